// Channel mixdown and band-limited resampling (egemma2_audio.rs, to_mono_16k
// and resample_hq): mono = float32 channel average; with the rates reduced by
// their gcd to o (in) and p (out), output n sits at input position n o / p and
//   y[n] = sum_m x[m] c sinc(t) I0(beta sqrt(1 - (t/64)^2)) / I0(beta),
//   t = (m - n o / p) c,   c = 0.958 min(o, p) / o,   |t| < 64 zero crossings,
// with ceil(p N / o) outputs and samples outside the clip taken as zero.
//
// Outputs are taken four at a time: unit u covers n = 4u .. 4u+3. Units of
// the same type T = u mod NT (NT = p / gcd(p, 4)) have the same taps, and
// consecutive units of one type sit D = 4 o / gcd(p, 4) input samples apart
// (one frame of 441 samples for 44.1 kHz, 12 samples for 48 kHz). k_rs_table
// evaluates, once per call and in float64, the taps of the four outputs of
// every type at every input offset i of their common window (lo_T + i,
// W_pad offsets), and stores them as one float4 per (T, i); zero outside each
// output's 64 zero crossings.
//
// The FIR works on tiles of Q consecutive units of each of up to eight types
// of one clip: the input span the tile touches and the types' tap rows sit in
// shared memory, and a warp takes a (type, 32-unit group) item with lane =
// unit, so for every input offset the warp reads one float4 of taps (the same
// shared-memory address for all lanes: a broadcast) and each lane one input
// sample, and does four FMAs. k_rs_fir_pipe, the persistent form, keeps one
// type group's tap rows for all its tiles, copies the next tile's span while
// it computes the current one, and splits each item's offset window over two
// warps. k_rs_fir, one CTA per tile, serves the plans whose tap rows and two
// spans do not fit: when the span does not fit (large D, as for co-prime
// rates) it reads the input from global memory, and when the tap rows do not
// fit it reads them from global memory too: correct, and slower.
//
// Rates whose repeating row of outputs is short (at most 160 outputs, a
// multiple of 16: 44.1, 48, 32, 24, 8, 96 kHz ...) take the tensor-core form
// instead (k_rs_btc builds its taps, k_rs_fir_tc computes; see the section
// before launch_rs_btc): the same sums as products of bf16-split operands.
#include <cmath>

#include "ae_internal.h"
#include "common.cuh"

namespace ae {

namespace {
constexpr double kRsWidth = 64.0;
constexpr double kRsRolloff = 0.958;
constexpr double kRsBeta = 12.8;
constexpr int kRsThreads = 256;
constexpr int kRsWarps = kRsThreads / 32;
constexpr size_t kRsSmemMax = 200 * 1024;  // staged input + staged output per CTA
constexpr size_t kRsPipeSmemMax = 220 * 1024;  // tap rows + two input spans (persistent form)
constexpr int kRsTcMaxN = 160;   // outputs per row of the tensor-core form
constexpr int kRsTcMaxK = 4096;  // inputs per row
}  // namespace

// I0(x) = sum_k ((x / 2)^2)^k / (k!)^2, summed while the terms still count.
__device__ double rs_bessel_i0(double x) {
  const double q = 0.25 * x * x;
  double term = 1.0, sum = 1.0;
  for (int k = 1; k < 400; ++k) {
    term *= q / ((double)k * (double)k);
    sum += term;
    if (term < sum * 1e-17) break;
  }
  return sum;
}

// One thread per (type T, offset i): the taps of outputs U T + r, r < U, at
// input lo_T + i (relative to the unit's base q D), lo_T = floor(U T o / p -
// 64 / c), stored as U / 4 float4. Output U T + r sits at input position
// U T o / p + r o / p.
__global__ void k_rs_table(float4 *__restrict__ coef, int32_t *__restrict__ lo, int U, int o, int p, int NT, int W_pad,
                           double c, double half, double i0b) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)NT * W_pad) return;
  const int T = (int)(idx / W_pad), i = (int)(idx % W_pad);
  const double frac = (double)U * (double)T * (double)o / (double)p;
  const int l0 = (int)floor(frac - half);
  if (i == 0) lo[T] = l0;
  for (int j = 0; j < U / 4; ++j) {
    double v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = 4 * j + k;
      const double t = ((double)(l0 + i) - frac - (double)r * (double)o / (double)p) * c;
      v[k] = 0.0;
      if (fabs(t) < kRsWidth) {
        const double q = t / kRsWidth;
        const double win = rs_bessel_i0(kRsBeta * sqrt(1.0 - q * q)) / i0b;
        const double pt = M_PI * t;
        const double sinc = pt == 0.0 ? 1.0 : sin(pt) / pt;
        v[k] = sinc * win * c;
      }
    }
    coef[idx * (U / 4) + j] = make_float4((float)v[0], (float)v[1], (float)v[2], (float)v[3]);
  }
}

// mono[i] = (x_0[i] + ... + x_{C-1}[i]) / C in float32, channel order.
__global__ void k_rs_mix(const float *__restrict__ x, int channels, int64_t ch_stride, int64_t n,
                         float *__restrict__ mono) {
  const float n_ch = (float)channels;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float s = x[i];
    for (int ch = 1; ch < channels; ++ch) s += x[ch * ch_stride + i];
    mono[i] = s / n_ch;
  }
}

struct RsArgs {
  const float *x;           // mono input, packed clips
  float *y;                 // packed outputs
  const float4 *coef;       // [NT][W_pad]: taps of the unit's four outputs
  const int32_t *lo;        // [NT]
  const int64_t *in_off;    // [B + 1] input sample offsets
  const int64_t *out_off;   // [B + 1] output sample offsets
  const int32_t *tile_off;  // [B + 1] tile offsets
  int n_clips, NT, D, W_pad, Q, TG, n_groups;
  int lo_min, span;         // span: staged inputs per tile (0: read from global memory)
  int stage_coef;           // the group's tap rows live in shared memory
  int n_tiles;              // tiles of the call (each covers Q units of every type of one clip)
};

// Clip of a tile (the last clip whose first tile is <= tile; empty clips own
// no tiles) and the tile's first unit and first input index within its clip.
struct RsTile {
  int64_t in0, n_in, out0, n_out, q0, base;
};
__device__ __forceinline__ RsTile rs_tile(const RsArgs &a, int tile) {
  int l = 0, h = a.n_clips;
  while (h - l > 1) {
    const int mid = (l + h) >> 1;
    if (a.tile_off[mid] <= tile) l = mid; else h = mid;
  }
  RsTile r;
  r.in0 = a.in_off[l];
  r.n_in = a.in_off[l + 1] - r.in0;
  r.out0 = a.out_off[l];
  r.n_out = a.out_off[l + 1] - r.out0;
  r.q0 = (int64_t)(tile - a.tile_off[l]) * a.Q;
  r.base = r.q0 * a.D + a.lo_min;
  return r;
}

// 4-byte asynchronous copy global -> shared; with valid == false nothing is
// read and the destination is zero-filled.
__device__ __forceinline__ void cp_async4(float *dst, const float *src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Partial FIR of one warp item over input offsets [i0, i1) (both even) from
// staged taps ([offset][U / 4] float4) and a staged input span: lane = unit,
// U outputs per lane, two partial sums each (even and odd offsets).
template <int U>
__device__ __forceinline__ void rs_partial(const RsArgs &a, const RsTile &r, const float *span, const float4 *cT,
                                           int T, int ql, int i0, int i1, float (&acc)[U]) {
  constexpr int V = U / 4;
  const int64_t m0 = (r.q0 + ql) * a.D + a.lo[T];
  const float *xr = span + (m0 - r.base);
  // two outputs' taps against the same input sample per packed two-lane FMA
  // (each lane a fused multiply-add, as fmaf)
  float2 e[U / 2], d[U / 2];
#pragma unroll
  for (int k = 0; k < U / 2; ++k) e[k] = d[k] = make_float2(0.f, 0.f);
#pragma unroll 4
  for (int i = i0; i < i1; i += 2) {
    const float x0 = xr[i], x1 = xr[i + 1];
    const float2 xx0 = make_float2(x0, x0), xx1 = make_float2(x1, x1);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float4 w0 = cT[i * V + j], w1 = cT[(i + 1) * V + j];
      e[2 * j] = __ffma2_rn(make_float2(w0.x, w0.y), xx0, e[2 * j]);
      e[2 * j + 1] = __ffma2_rn(make_float2(w0.z, w0.w), xx0, e[2 * j + 1]);
      d[2 * j] = __ffma2_rn(make_float2(w1.x, w1.y), xx1, d[2 * j]);
      d[2 * j + 1] = __ffma2_rn(make_float2(w1.z, w1.w), xx1, d[2 * j + 1]);
    }
  }
#pragma unroll
  for (int k = 0; k < U / 2; ++k) {
    acc[2 * k] = e[k].x + d[k].x;
    acc[2 * k + 1] = e[k].y + d[k].y;
  }
}

// Persistent form, for plans whose group tap rows and two input spans fit in
// shared memory: CTA b serves type group b mod n_groups for the tiles
// b / n_groups, + per, ... of the whole call. The group's tap rows are staged
// once; the input span of the next tile is copied asynchronously (4 bytes a
// lane, coalesced, zero-filled outside the clip) while the current tile is
// computed, so the copies hide behind the multiply-adds. Each (type, 32-unit)
// item is split over PARTS warps, one per slice of the offset window, so that
// 16 warps keep the shared-memory loads' latency covered; the other slices'
// sums meet the first's in shared memory. With U = 8 outputs per unit a warp
// loads two broadcast float4 of taps and one input sample per offset for
// eight multiply-adds (U = 4: one and one for four).
constexpr int kRsPipeThreads = 512;

template <int U, int PARTS>
__global__ void __launch_bounds__(kRsPipeThreads) k_rs_fir_pipe(const RsArgs a, int per) {
  constexpr int V = U / 4, ITEMS = kRsPipeThreads / 32 / PARTS;
  extern __shared__ __align__(16) float rs_smem[];
  const int g = blockIdx.x % a.n_groups;
  int t = blockIdx.x / a.n_groups;
  if (t >= a.n_tiles) return;
  const int T0 = g * a.TG, n_types = min(a.TG, a.NT - T0);
  float4 *cs = reinterpret_cast<float4 *>(rs_smem);                        // [TG][W_pad][V]
  float4 *red = cs + (int64_t)a.TG * a.W_pad * V;                           // [PARTS - 1][ITEMS][32][V]
  float *buf0 = reinterpret_cast<float *>(red + (PARTS - 1) * ITEMS * 32 * V);  // two input spans
  auto stage = [&](int tile, float *dst) {
    const RsTile r = rs_tile(a, tile);
    const float *xin = a.x + r.in0;
    for (int i = threadIdx.x; i < a.span; i += kRsPipeThreads) {
      const int64_t m = r.base + i;
      const bool ok = m >= 0 && m < r.n_in;
      cp_async4(dst + i, ok ? xin + m : a.x, ok);
    }
  };
  stage(t, buf0);
  cp_async_commit();
  {
    const float4 *src = a.coef + (int64_t)T0 * a.W_pad * V;
    for (int i = threadIdx.x; i < n_types * a.W_pad * V; i += kRsPipeThreads) cs[i] = __ldg(src + i);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = (a.Q / 32) * n_types;
  const int item = warp % ITEMS, part = warp / ITEMS;
  const int pw = a.W_pad / PARTS;  // W_pad is a multiple of 8: every slice is even
  const int tl = item % n_types, ql = (item / n_types) * 32 + lane;
  for (int k = 0; t < a.n_tiles; ++k, t += per) {
    if (t + per < a.n_tiles) stage(t + per, buf0 + ((k + 1) & 1) * a.span);
    cp_async_commit();  // possibly empty: keeps one group per iteration
    cp_async_wait_1();  // this tile's span has landed (this thread's copies)
    __syncthreads();    // ... and every thread's
    const RsTile r = rs_tile(a, t);
    float acc[U];
    if (item < items) {
      rs_partial<U>(a, r, buf0 + (k & 1) * a.span, cs + (int64_t)tl * a.W_pad * V, T0 + tl, ql, part * pw,
                    (part + 1) * pw, acc);
      if (part > 0) {
        float4 *dst = red + (((part - 1) * ITEMS + item) * 32 + lane) * V;
#pragma unroll
        for (int j = 0; j < V; ++j) dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
      }
    }
    __syncthreads();
    if (item < items && part == 0) {
#pragma unroll
      for (int q = 1; q < PARTS; ++q) {
        const float4 *src = red + (((q - 1) * ITEMS + item) * 32 + lane) * V;
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const float4 u = src[j];
          acc[4 * j] += u.x;
          acc[4 * j + 1] += u.y;
          acc[4 * j + 2] += u.z;
          acc[4 * j + 3] += u.w;
        }
      }
      const int64_t n0 = ((r.q0 + ql) * a.NT + T0 + tl) * U;  // first output of the unit
#pragma unroll
      for (int j = 0; j < U; ++j)
        if (n0 + j < r.n_out) a.y[r.out0 + n0 + j] = acc[j];
    }
    __syncthreads();  // the span buffer is refilled and red rewritten on the next tiles
  }
}

// Per-tile form (one CTA per tile and type group), for plans the persistent form
// cannot hold: spans read from global memory, or tap rows too large to stage twice.
__global__ void __launch_bounds__(kRsThreads) k_rs_fir(const RsArgs a) {
  extern __shared__ __align__(16) float rs_smem[];
  // tile = (clip, block of Q units of each type, group of TG types)
  const int tile = blockIdx.x / a.n_groups, tg = blockIdx.x % a.n_groups;
  int c = 0;
  {
    int l = 0, h = a.n_clips;  // last clip whose first tile is <= tile
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (a.tile_off[mid] <= tile) l = mid; else h = mid;
    }
    c = l;
  }
  const int64_t in0 = a.in_off[c], n_in = a.in_off[c + 1] - in0;
  const int64_t out0 = a.out_off[c], n_out = a.out_off[c + 1] - out0;
  const int64_t q0 = (int64_t)(tile - a.tile_off[c]) * a.Q;
  const int64_t base = q0 * a.D + a.lo_min;  // first input index the tile touches
  const int T0 = tg * a.TG, n_types = min(a.TG, a.NT - T0);
  const float *xin = a.x + in0;
  float4 *cs = reinterpret_cast<float4 *>(rs_smem + a.span);  // [TG][W_pad] tap rows (stage_coef)
  for (int i = threadIdx.x; i < a.span; i += kRsThreads) {
    const int64_t m = base + i;
    rs_smem[i] = (m >= 0 && m < n_in) ? __ldg(xin + m) : 0.f;
  }
  if (a.stage_coef) {
    const float4 *src = a.coef + (int64_t)T0 * a.W_pad;
    for (int i = threadIdx.x; i < n_types * a.W_pad; i += kRsThreads) cs[i] = __ldg(src + i);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = a.Q / 32, items = groups * n_types;
  for (int item = warp; item < items; item += kRsWarps) {
    const int tl = item % n_types, g = item / n_types, T = T0 + tl;
    const int ql = g * 32 + lane;  // unit of type T within the tile
    const float4 *cT = a.stage_coef ? cs + (int64_t)tl * a.W_pad : a.coef + (int64_t)T * a.W_pad;
    const int64_t m0 = (q0 + ql) * a.D + a.lo[T];  // input index of offset 0
    // two partial sums (even and odd offsets) per output
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f), d = e;
    if (a.span > 0) {
      const float *xr = rs_smem + (m0 - base);
#pragma unroll 4
      for (int i = 0; i < a.W_pad; i += 2) {
        const float4 w0 = cT[i], w1 = cT[i + 1];
        const float x0 = xr[i], x1 = xr[i + 1];
        e.x = fmaf(w0.x, x0, e.x);
        e.y = fmaf(w0.y, x0, e.y);
        e.z = fmaf(w0.z, x0, e.z);
        e.w = fmaf(w0.w, x0, e.w);
        d.x = fmaf(w1.x, x1, d.x);
        d.y = fmaf(w1.y, x1, d.y);
        d.z = fmaf(w1.z, x1, d.z);
        d.w = fmaf(w1.w, x1, d.w);
      }
    } else {
      for (int i = 0; i < a.W_pad; i += 2) {
        const float4 w0 = cT[i], w1 = cT[i + 1];
        const int64_t m = m0 + i;
        const float x0 = (m >= 0 && m < n_in) ? __ldg(xin + m) : 0.f;
        const float x1 = (m + 1 >= 0 && m + 1 < n_in) ? __ldg(xin + m + 1) : 0.f;
        e.x = fmaf(w0.x, x0, e.x);
        e.y = fmaf(w0.y, x0, e.y);
        e.z = fmaf(w0.z, x0, e.z);
        e.w = fmaf(w0.w, x0, e.w);
        d.x = fmaf(w1.x, x1, d.x);
        d.y = fmaf(w1.y, x1, d.y);
        d.z = fmaf(w1.z, x1, d.z);
        d.w = fmaf(w1.w, x1, d.w);
      }
    }
    const float r4[4] = {e.x + d.x, e.y + d.y, e.z + d.z, e.w + d.w};
    const int64_t n0 = ((q0 + ql) * a.NT + T) * 4;  // first output of the unit
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if (n0 + r < n_out) a.y[out0 + n0 + r] = r4[r];
  }
}

int64_t rs_len(int64_t n, int rate_in, int rate_out) {
  if (n < 0 || rate_in <= 0 || rate_out <= 0) return -1;
  if (rate_in == rate_out || n == 0) return n;
  int64_t a = rate_in, b = rate_out;
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  const int64_t o = rate_in / a, p = rate_out / a;
  return (p * n + o - 1) / o;
}

// The plan for units of U outputs; `items` caps the (type, 32-unit) items of
// a tile (the warps of the per-tile form, or 16 warps / parts in the
// persistent form).
static RsPlan rs_plan_u(int rate_in, int rate_out, int U, int items, int parts) {
  RsPlan pl;
  pl.U = U;
  pl.parts = parts;
  int64_t a = rate_in, b = rate_out;
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  pl.o = (int)(rate_in / a);
  pl.p = (int)(rate_out / a);
  pl.c = kRsRolloff * (double)std::min(pl.o, pl.p) / (double)pl.o;
  pl.half = kRsWidth / pl.c;
  int gu = U;  // gcd(p, U), U a power of two
  while (pl.p % gu) gu /= 2;
  pl.NT = pl.p / gu;
  pl.D = (int)((int64_t)U * pl.o / gu);
  // a unit's U outputs span (U - 1) o / p input samples; each reaches half to either side
  pl.W = (int)std::ceil(2.0 * pl.half + (double)(U - 1) * pl.o / pl.p) + 3;
  pl.W_pad = (pl.W + 7) & ~7;
  pl.lo_min = (int)std::floor(-pl.half) - 1;  // <= lo_T for every type
  // a tile: Q units of each of (up to) TG types, at most `items` (type,
  // 32-unit group) items; the staged input span and the group's tap rows
  // within the shared-memory budget
  pl.TG = std::min(pl.NT, items);
  pl.n_groups = (pl.NT + pl.TG - 1) / pl.TG;
  int groups = std::max(1, items / pl.TG);
  // lo_T < U T o / p <= D - U o / p, so offsets stay below Q D + W_pad - lo_min
  auto span_of = [&](int q) -> int64_t { return (int64_t)q * pl.D + pl.W_pad - pl.lo_min + 2; };
  const int64_t coef_bytes = 4 * (int64_t)U * pl.TG * pl.W_pad;
  while (groups > 1 && 4 * span_of(32 * groups) + coef_bytes > (int64_t)kRsSmemMax) groups /= 2;
  pl.Q = 32 * groups;
  pl.stage_coef = coef_bytes <= (int64_t)kRsSmemMax / 2;
  const int64_t span_b = 4 * span_of(pl.Q);
  pl.span = span_b + (pl.stage_coef ? coef_bytes : 0) <= (int64_t)kRsSmemMax ? (int)span_of(pl.Q) : 0;
  pl.span = (pl.span + 3) & ~3;  // the tap rows that follow stay 16-byte aligned
  pl.smem = 4 * (size_t)pl.span + (pl.stage_coef ? (size_t)coef_bytes : 0);
  // the persistent form keeps the tap rows, the other slices' sums and two input spans
  const size_t red_bytes = 4 * (size_t)U * 32 * (size_t)(kRsPipeThreads / 32 / parts) * (size_t)(parts - 1);
  pl.smem_pipe = 8 * (size_t)pl.span + (size_t)coef_bytes + red_bytes;
  pl.pipe = pl.stage_coef && pl.span > 0 && pl.smem_pipe <= kRsPipeSmemMax;
  return pl;
}

RsPlan rs_plan(int rate_in, int rate_out) {
  // eight outputs per unit in the persistent form when it fits (4 items of
  // 4 warps each), else four (8 items of 2 warps, or the per-tile form)
  RsPlan pl = rs_plan_u(rate_in, rate_out, 8, 4, 4);
  if (!pl.pipe) pl = rs_plan_u(rate_in, rate_out, 4, kRsWarps, 2);
  // the tensor-core form when a row of outputs that repeats the same taps
  // (a multiple of p) holds at most 160 and a multiple of 16 of them
  int g16 = 16;
  while (pl.p % g16) g16 /= 2;
  const int64_t N = (int64_t)pl.p * (16 / g16);
  if (rate_in != rate_out && N <= kRsTcMaxN) {
    const int64_t D = N * pl.o / pl.p;
    const int lo = (int)std::floor(-pl.half) - 1;
    const int hi = (int)std::ceil((double)(N - 1) * pl.o / pl.p + pl.half) + 1;
    const int64_t K = ((int64_t)(hi - lo + 1) + 63) / 64 * 64;
    if (D <= (1 << 20) && K <= kRsTcMaxK) {
      pl.tc = true;
      pl.tcN = (int)N;
      pl.tcD = (int)D;
      pl.tcLo = lo;
      pl.tcK = (int)K;
    }
  }
  return pl;
}

cudaError_t launch_rs_table(const RsPlan &pl, float *coef, int32_t *lo, cudaStream_t s) {
  const int64_t n = (int64_t)pl.NT * pl.W_pad;
  const double i0b = [] {
    double q = 0.25 * kRsBeta * kRsBeta, term = 1.0, sum = 1.0;
    for (int k = 1; k < 400; ++k) {
      term *= q / ((double)k * (double)k);
      sum += term;
      if (term < sum * 1e-17) break;
    }
    return sum;
  }();
  return launch_k(k_rs_table, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, reinterpret_cast<float4 *>(coef),
                  lo, pl.U, pl.o, pl.p, pl.NT, pl.W_pad, pl.c, pl.half, i0b);
}

cudaError_t launch_rs_mix(const float *x, int channels, int64_t ch_stride, int64_t n, float *mono, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
  return launch_k(k_rs_mix, dim3((unsigned)blocks), dim3(256), 0, s, x, channels, ch_stride, n, mono);
}

cudaError_t launch_rs_fir(const RsPlan &pl, const float *mono, float *y, const float *coef, const int32_t *lo,
                          const int64_t *in_off, const int64_t *out_off, const int32_t *tile_off, int n_clips,
                          int n_tiles, cudaStream_t s) {
  if (n_tiles <= 0) return cudaSuccess;
  RsArgs a;
  a.x = mono;
  a.y = y;
  a.coef = reinterpret_cast<const float4 *>(coef);
  a.lo = lo;
  a.in_off = in_off;
  a.out_off = out_off;
  a.tile_off = tile_off;
  a.n_clips = n_clips;
  a.NT = pl.NT;
  a.D = pl.D;
  a.W_pad = pl.W_pad;
  a.Q = pl.Q;
  a.TG = pl.TG;
  a.n_groups = pl.n_groups;
  a.lo_min = pl.lo_min;
  a.span = pl.span;
  a.stage_coef = pl.stage_coef ? 1 : 0;
  a.n_tiles = n_tiles;
  if (pl.pipe) {
    auto kern = pl.U == 8 ? k_rs_fir_pipe<8, 4> : k_rs_fir_pipe<4, 2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_pipe);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRsPipeThreads, pl.smem_pipe)) !=
        cudaSuccess)
      return e;
    // CTAs per type group: every resident slot busy, but no more than the tiles
    const int per = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sms * std::max(per_sm, 1) / pl.n_groups,
                                                                 n_tiles));
    return launch_k(kern, dim3((unsigned)(per * pl.n_groups)), dim3(kRsPipeThreads), pl.smem_pipe, s, a, per);
  }
  if (pl.smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_rs_fir, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRsSmemMax);
    if (e != cudaSuccess) return e;
  }
  return launch_k(k_rs_fir, dim3((unsigned)((int64_t)n_tiles * pl.n_groups)), dim3(kRsThreads), pl.smem, s, a);
}

// ------------------------------------------------------------------ tensor-core form

// The FIR as a product: row r of outputs r N .. r N + N - 1 (N = tcN) reads
// the inputs r D + lo .. r D + lo + K - 1 (D = tcD, lo = tcLo, K = tcK), with
// the same taps for every row, so Y[rows][N] = X[rows][K] B^T with B[N][K]
// the taps of each output of a row at each input offset (zero outside its 64
// zero crossings). Both operands are split into bf16 parts (hi = bf16(v), lo =
// bf16(v - hi), v = hi + lo to about 2^-18 relative) and the product is taken
// as X_hi B_hi + X_hi B_lo + X_lo B_hi + X_lo B_lo, accumulated in float32 on
// the tensor cores.

// B's two parts, [N][K] bf16 each (hi first), the taps in float64 as the
// other table's: t = (lo + k - j o / p) c for output j of a row, input k.
__global__ void k_rs_btc(bf16 *__restrict__ bmat, int N, int K, int lo, int o, int p, double c, double i0b) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)N * K) return;
  const int j = (int)(idx / K), k = (int)(idx % K);
  const double t = ((double)(lo + k) - (double)j * (double)o / (double)p) * c;
  double v = 0.0;
  if (fabs(t) < kRsWidth) {
    const double q = t / kRsWidth;
    const double win = rs_bessel_i0(kRsBeta * sqrt(1.0 - q * q)) / i0b;
    const double pt = M_PI * t;
    v = (pt == 0.0 ? 1.0 : sin(pt) / pt) * win * c;
  }
  const bf16 hi = __double2bfloat16(v);
  bmat[idx] = hi;
  bmat[(int64_t)N * K + idx] = __double2bfloat16(v - (double)__bfloat162float(hi));
}

struct RsTcArgs {
  const float *x;
  float *y;
  const int64_t *in_off, *out_off;
  const int32_t *tile_off;  // [B + 1] tiles of 128 rows
  int n_clips, n_tiles, N, D, lo, kb_n;
};

namespace {
constexpr int kTcThreads = 256;
constexpr uint32_t kTcA = 128 * 128;             // one part of A: 128 rows x 64 bf16
constexpr uint32_t kTcB = kRsTcMaxN * 128;       // one part of B: up to 160 rows x 64 bf16
constexpr uint32_t kTcOffB = 2 * 2 * kTcA;       // A: [2 stages][hi, lo]
constexpr uint32_t kTcOffBar = kTcOffB + 2 * 2 * kTcB;  // B: [2 stages][hi, lo]
constexpr size_t kTcSmem = kTcOffBar + 64 + 1024;
static_assert(kTcOffB % 1024 == 0 && kTcOffBar % 1024 == 0, "swizzle atoms");
static_assert(kTcSmem <= 227 * 1024, "one CTA per SM");
}  // namespace

struct RsTcTile {
  int64_t in0, n_in, out0, n_out, rows, r0;
};
__device__ __forceinline__ RsTcTile rs_tc_tile(const RsTcArgs &a, int tile) {
  int l = 0, h = a.n_clips;
  while (h - l > 1) {
    const int mid = (l + h) >> 1;
    if (a.tile_off[mid] <= tile) l = mid; else h = mid;
  }
  RsTcTile r;
  r.in0 = a.in_off[l];
  r.n_in = a.in_off[l + 1] - r.in0;
  r.out0 = a.out_off[l];
  r.n_out = a.out_off[l + 1] - r.out0;
  r.rows = (r.n_out + a.N - 1) / a.N;
  r.r0 = (int64_t)(tile - a.tile_off[l]) * 128;
  return r;
}

// Persistent CTAs over tiles of 128 rows, walked as one sequence of steps
// (tile, 64-input k-block). Thread t owns inputs 4 (t mod 16) .. + 3 of rows
// t / 16 + 16 i of every k-block: it loads them two steps ahead into one of
// three register sets (the loop is unrolled three times, so no set is copied),
// splits the current set into A's two parts, and B's two parts arrive by TMA;
// one thread issues the four products into the tile's accumulator (N
// tensor-memory columns), and all threads drain it after the tile's last step.
__global__ void __launch_bounds__(kTcThreads, 1) k_rs_fir_tc(const __grid_constant__ CUtensorMap tmB, const RsTcArgs a,
                                                            unsigned *status) {
  extern __shared__ uint8_t tc_raw_smem[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(tc_raw_smem) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kTcOffBar), *empty = full + 2, *accb = full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 5);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.N, D = a.D, kb_n = a.kb_n;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accb, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_bf16_f32(128, N);
  const int my_tiles = (int)blockIdx.x < a.n_tiles ? (a.n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int64_t n_steps = (int64_t)my_tiles * kb_n;
  const int qd = tid & 15, rw0 = tid >> 4;

  // tile records of the step being computed and of the one being loaded
  RsTcTile tc_cur{}, tc_ld{};
  int ld_tile = -1;
  auto tile_of_step = [&](int64_t st) { return (int)blockIdx.x + (int)(st / kb_n) * (int)gridDim.x; };
  auto load = [&](int64_t st, float (&v)[32]) {
    const int tile = tile_of_step(st), kb = (int)(st % kb_n);
    if (tile != ld_tile) {
      tc_ld = rs_tc_tile(a, tile);
      ld_tile = tile;
    }
    const RsTcTile &T = tc_ld;
    const int64_t first = T.r0 * D + a.lo + 64 * kb, last = (T.r0 + 127) * D + a.lo + 64 * kb + 63;
    const float *xin = a.x + T.in0;
    int64_t m = (T.r0 + rw0) * D + a.lo + 64 * kb + 4 * qd;
    if (T.r0 + 127 < T.rows && first >= 0 && last < T.n_in) {
#pragma unroll
      for (int i = 0; i < 8; ++i, m += 16 * (int64_t)D) {
#pragma unroll
        for (int u = 0; u < 4; ++u) v[4 * i + u] = __ldg(xin + m + u);
      }
    } else {
      int64_t r = T.r0 + rw0;
#pragma unroll
      for (int i = 0; i < 8; ++i, m += 16 * (int64_t)D, r += 16) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool ok = r < T.rows && m + u >= 0 && m + u < T.n_in;
          v[4 * i + u] = ok ? __ldg(xin + m + u) : 0.f;
        }
      }
    }
  };
  int ntile = 0;
  bool ok = true;
  // one step: s's inputs are in `cur`; s + 2's are loaded into `nxt`
  auto step = [&](int64_t sidx, float (&cur)[32], float (&nxt)[32]) {
    if (!ok) return;
    const int st = (int)(sidx & 1), kb = (int)(sidx % kb_n);
    if (kb == 0) tc_cur = rs_tc_tile(a, tile_of_step(sidx));
    if (sidx + 2 < n_steps) load(sidx + 2, nxt);
    bool good = true;
    if (tid == 0 && sidx >= 2) good = mbar_wait(&empty[st], (uint32_t)(((sidx >> 1) - 1) & 1));  // stage st is free
    if (!__syncthreads_and(good)) {
      ok = false;
      return;
    }
    if (tid == 0) {
      mbar_arrive_expect_tx(&full[st], 2u * (uint32_t)N * 128u);
      tma_load_2d(smem + kTcOffB + (2 * st) * kTcB, &tmB, 64 * kb, 0, &full[st]);
      tma_load_2d(smem + kTcOffB + (2 * st + 1) * kTcB, &tmB, 64 * kb, N, &full[st]);
    }
    {  // split into A's parts: row rw0 + 16 i, inputs 4 qd .. 4 qd + 3 (half a 16-byte granule)
      uint8_t *ahi = smem + (2 * st) * kTcA, *alo = smem + (2 * st + 1) * kTcA;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = rw0 + 16 * i;
        const float *v = cur + 4 * i;
        const float h0 = __bfloat162float(__float2bfloat16_rn(v[0])), h1 = __bfloat162float(__float2bfloat16_rn(v[1]));
        const float h2 = __bfloat162float(__float2bfloat16_rn(v[2])), h3 = __bfloat162float(__float2bfloat16_rn(v[3]));
        const uint32_t off = row * 128 + (((qd >> 1) ^ (row & 7)) << 4) + (qd & 1) * 8;
        *reinterpret_cast<uint2 *>(ahi + off) = make_uint2(pack_bf16(h0, h1), pack_bf16(h2, h3));
        *reinterpret_cast<uint2 *>(alo + off) =
            make_uint2(pack_bf16(v[0] - h0, v[1] - h1), pack_bf16(v[2] - h2, v[3] - h3));
      }
    }
    fence_async_smem();
    __syncthreads();  // A's parts are written
    if (tid == 0) {
      if (!mbar_wait(&full[st], (uint32_t)((sidx >> 1) & 1))) {
        atomicOr(status, kStatusWaitTimeout);
      } else {
        tc_fence_after();
        const uint32_t ahi = smem_u32(smem + (2 * st) * kTcA), alo = smem_u32(smem + (2 * st + 1) * kTcA);
        const uint32_t bhi = smem_u32(smem + kTcOffB + (2 * st) * kTcB), blo = smem_u32(smem + kTcOffB + (2 * st + 1) * kTcB);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          tc_mma_bf16(tmem, sw128_desc(ahi + ks * 32), sw128_desc(bhi + ks * 32), idesc, (kb | ks) != 0 ? 1u : 0u);
          tc_mma_bf16(tmem, sw128_desc(ahi + ks * 32), sw128_desc(blo + ks * 32), idesc, 1u);
          tc_mma_bf16(tmem, sw128_desc(alo + ks * 32), sw128_desc(bhi + ks * 32), idesc, 1u);
          tc_mma_bf16(tmem, sw128_desc(alo + ks * 32), sw128_desc(blo + ks * 32), idesc, 1u);
        }
      }
      tc_commit(&empty[st]);
      if (kb + 1 == kb_n) tc_commit(accb);
    }
    if (kb + 1 < kb_n) return;
    // the tile's last step: drain (warp w reads lanes 32 (w & 3) .. + 31, columns of half w >> 2)
    const bool got = mbar_wait(accb, (uint32_t)(ntile & 1));
    if (!__syncthreads_and(got)) {
      ok = false;
      return;
    }
    tc_fence_after();
    {
      const int q = warp & 3, half = warp >> 2, ncol = N / 2;  // N / 2 is a multiple of 8
      const int64_t r = tc_cur.r0 + 32 * q + lane;
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * ncol);
      for (int c0 = 0; c0 < ncol; c0 += 8) {
        uint32_t v[8];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
            : "r"(taddr + c0));
        tmem_ld_wait();
        if (r < tc_cur.rows) {
          const int64_t n0 = r * N + half * ncol + c0;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (n0 + u < tc_cur.n_out) a.y[tc_cur.out0 + n0 + u] = __uint_as_float(v[u]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the accumulator is read: the next tile's first product may overwrite it
    ++ntile;
  };
  float va[32], vb[32], vc[32];
  if (n_steps > 0) load(0, va);
  if (n_steps > 1) load(1, vb);
  for (int64_t sidx = 0; sidx < n_steps && ok; sidx += 3) {
    step(sidx, va, vc);
    if (sidx + 1 < n_steps) step(sidx + 1, vb, va);
    if (sidx + 2 < n_steps) step(sidx + 2, vc, vb);
  }
  if (!ok && tid == 0) atomicOr(status, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_rs_btc(const RsPlan &pl, void *bmat, cudaStream_t s) {
  const int64_t n = (int64_t)pl.tcN * pl.tcK;
  const double i0b = [] {
    double q = 0.25 * kRsBeta * kRsBeta, term = 1.0, sum = 1.0;
    for (int k = 1; k < 400; ++k) {
      term *= q / ((double)k * (double)k);
      sum += term;
      if (term < sum * 1e-17) break;
    }
    return sum;
  }();
  return launch_k(k_rs_btc, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, static_cast<bf16 *>(bmat), pl.tcN,
                  pl.tcK, pl.tcLo, pl.o, pl.p, pl.c, i0b);
}

cudaError_t launch_rs_fir_tc(const RsPlan &pl, const float *mono, float *y, void *bmat, const int64_t *in_off,
                             const int64_t *out_off, const int32_t *tile_off, int n_clips, int n_tiles,
                             cudaStream_t s) {
  if (n_tiles <= 0) return cudaSuccess;
  CUtensorMap tmB;  // both parts as one [2 N][K] bf16 matrix, boxes of 64 inputs x N rows
  if (!make_tmap_2d_bf16(&tmB, bmat, (uint64_t)pl.tcK, (uint64_t)2 * pl.tcN, (uint64_t)pl.tcK * 2, 64,
                         (uint32_t)pl.tcN))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr{0};
  if (const cudaError_t e = smem_attr(k_rs_fir_tc, kTcSmem, attr)) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  RsTcArgs a;
  a.x = mono;
  a.y = y;
  a.in_off = in_off;
  a.out_off = out_off;
  a.tile_off = tile_off;
  a.n_clips = n_clips;
  a.n_tiles = n_tiles;
  a.N = pl.tcN;
  a.D = pl.tcD;
  a.lo = pl.tcLo;
  a.kb_n = pl.tcK / 64;
  const int grid = n_tiles < sms ? n_tiles : sms;
  return launch_k(k_rs_fir_tc, dim3((unsigned)grid), dim3(kTcThreads), kTcSmem, s, tmB, a, device_status_word());
}

}  // namespace ae
