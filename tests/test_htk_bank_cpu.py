"""The HTK filterbank compiled into the log-mel kernel (csrc/htk_bank.h,
written by log_mel_front_b200/gen_htk_bank.py) against the oracle's
``mel_filter_bank`` (egemma2_audio.rs): every literal in the header is the
float32 rounding of the oracle's float64 weight, no nonzero weight is
missing, the header is what the generator writes today, and the per-warp
band split covers every band once."""
import os
import re

import numpy as np

from log_mel_front_b200 import gen_htk_bank as G
from oracle import oracle as O


def _header_terms():
    """(band, bin, weight) triples read back from the header's code."""
    src = open(G.HEADER).read()
    out = []
    for b, expr in re.findall(r"o\[(\d+)\] = log_floor_sum\((.*)\);", src):
        for k, w in re.findall(r"m\[(\d+)\](?:\]|,| \*) ?(0x[0-9a-fp.+-]+)f", expr):
            out.append((int(b), int(k), float.fromhex(w)))
    return out


def test_header_is_current():
    assert open(G.HEADER).read() == G.render()


def test_header_weights_are_the_oracle_bank_in_float32():
    M = O.mel_filter_bank()
    terms = _header_terms()
    assert len(terms) == int((M > 0).sum()) == 506
    seen = np.zeros_like(M, dtype=bool)
    for b, k, w in terms:
        assert not seen[k, b]
        seen[k, b] = True
        assert np.float32(M[k, b]) == np.float32(w), (b, k)
    assert np.all(seen == (M > 0))


def test_warp_split_covers_every_band_once():
    split = G.warp_split(G.bank())
    assert split[0] == 0 and split[-1] == 128 and len(split) == 9
    assert all(a <= b for a, b in zip(split, split[1:]))
    src = open(G.HEADER).read()
    bands = [int(b) for b in re.findall(r"o\[(\d+)\] =", src)]
    assert sorted(bands) == list(range(128))
    # balance: no warp does more than 1.5x the mean number of multiply-adds
    per = [sum(len(G.bank()[b][1]) for b in range(split[w], split[w + 1])) for w in range(8)]
    assert max(per) <= 1.5 * 506 / 8, per
