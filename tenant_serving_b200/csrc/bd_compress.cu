// bd_compress: the compress half of BitDelta on sm_100a.
//
// Method ("bitdelta" page, "How BitDelta Works" 1-3 and "Safety Benefits: 1. Outlier
// Clipping"; per-axis vectors from "Per-Axis Weight Deltas", "Key Contributions" 1):
//   delta = W_fine - W_base; optional clamp to [mean - k std, mean + k std] over the whole
//   matrix; scale = mean |delta_c| over each group / row / column / the whole matrix;
//   sign bit = !(delta_c < 0), packed LSB-first along d_in into uint32 words.
//
// Kernels (all HBM-bound streams; 16-byte coalesced loads of both inputs):
//   k_delta_stats      clip statistics: sums of the shifted
//                      delta and of its square, in fp64 per element, one pair per block;
//                      the last block merges the pairs in a fixed order -> mean, std, lo,
//                      hi and the fp32 thresholds the main pass compares with.
//   k_scale_signpack   main pass for GROUP / ROW / TENSOR: a warp streams a segment of
//                      one row, 16 bytes per lane per input; signs are packed with two
//                      (bf16) or three (fp32) xor-shuffles of per-lane bit masks; group
//                      sums are xor-shuffle trees; row / tensor sums go to fp64 partials.
//   k_col_scale_signpack  COL mode: a CTA of 8 warps walks a tile of rows of one column
//                      chunk, each warp its own rows with 8 rows in flight (fp32 sums over
//                      those 8, fp64 across them); the warps' column sums are added in
//                      shared memory into one fp64 partial per column and CTA.
//   k_scale_final      fixed-order reduction of the partials into row / column / tensor
//                      scales (deterministic, no atomics).
//   k_block_final      BLOCK mode: the main pass writes each row's group means; the
//                      block scale is their mean over the block's rows, in fp64 and in
//                      row order.
#include "bd_internal.cuh"

#include <math.h>

namespace bd {

struct ClipParams {
  double mean, stddev, lo, hi;
  float lo_up;   // smallest float >= lo:  x < lo  <=>  x < lo_up   (x a float)
  float hi_dn;   // largest float <= hi:   x > hi  <=>  x > hi_dn
  float lo_val;  // value a clamped-low entry takes (lo rounded, sign kept)
  float hi_val;  // value a clamped-high entry takes
};

// ------------------------------------------------------------------------------------
// element access: 16 bytes of W_base and W_fine -> VEC deltas in fp32
// ------------------------------------------------------------------------------------
template <bool BF16>
struct Vec;
template <>
struct Vec<true> {  // 8 bf16 per 16 bytes
  static constexpr int N = 8;
  __device__ __forceinline__ static void delta(const uint4& b, const uint4& f, float* d) {
    const uint32_t bb[4] = {b.x, b.y, b.z, b.w};
    const uint32_t ff[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      d[2 * k] = bf16lo(ff[k]) - bf16lo(bb[k]);
      d[2 * k + 1] = bf16hi(ff[k]) - bf16hi(bb[k]);
    }
  }
  // exact differences in fp64
  __device__ __forceinline__ static void delta64(const uint4& b, const uint4& f, double* d) {
    const uint32_t bb[4] = {b.x, b.y, b.z, b.w};
    const uint32_t ff[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      d[2 * k] = (double)bf16lo(ff[k]) - (double)bf16lo(bb[k]);
      d[2 * k + 1] = (double)bf16hi(ff[k]) - (double)bf16hi(bb[k]);
    }
  }
};
template <>
struct Vec<false> {  // 4 fp32 per 16 bytes
  static constexpr int N = 4;
  __device__ __forceinline__ static void delta(const uint4& b, const uint4& f, float* d) {
    d[0] = __uint_as_float(f.x) - __uint_as_float(b.x);
    d[1] = __uint_as_float(f.y) - __uint_as_float(b.y);
    d[2] = __uint_as_float(f.z) - __uint_as_float(b.z);
    d[3] = __uint_as_float(f.w) - __uint_as_float(b.w);
  }
  __device__ __forceinline__ static void delta64(const uint4& b, const uint4& f, double* d) {
    d[0] = (double)__uint_as_float(f.x) - (double)__uint_as_float(b.x);
    d[1] = (double)__uint_as_float(f.y) - (double)__uint_as_float(b.y);
    d[2] = (double)__uint_as_float(f.z) - (double)__uint_as_float(b.z);
    d[3] = (double)__uint_as_float(f.w) - (double)__uint_as_float(b.w);
  }
};

// The four fp32 values the main pass needs from ClipParams.
struct ClipF {
  float lo_up, hi_dn, lo_val, hi_val;
};
__device__ __forceinline__ ClipF load_clip(const ClipParams* c) {
  return ClipF{c->lo_up, c->hi_dn, c->lo_val, c->hi_val};
}

__device__ __forceinline__ float clamp_delta(float d, const ClipF& c) {
  // Comparisons against the float thresholds are exactly the comparisons of the float
  // delta with the fp64 bounds; the replacement keeps the sign of the fp64 bound.
  return d < c.lo_up ? c.lo_val : (d > c.hi_dn ? c.hi_val : d);
}

// ------------------------------------------------------------------------------------
// whole-matrix mean / std for the clip: fp64 shifted sums, finished by the last block
// ------------------------------------------------------------------------------------
// mean, unbiased std, bounds and the fp32 comparison values from the whole-matrix sums of
// (delta - shift) and (delta - shift)^2
__device__ void finish_clip(double S1, double S2, double shift, int64_t n, double k,
                            ClipParams* __restrict__ out, double* __restrict__ stats_out) {
  const double dn = (double)n;
  const double mean = shift + S1 / dn;
  double sd = 0.0;
  if (n > 1) {
    double var = (S2 - S1 * (S1 / dn)) / (dn - 1.0);
    sd = var > 0.0 ? sqrt(var) : 0.0;
  }
  const double lo = mean - k * sd, hi = mean + k * sd;
  ClipParams c;
  c.mean = mean;
  c.stddev = sd;
  c.lo = lo;
  c.hi = hi;
  c.lo_up = __double2float_ru(lo);
  c.hi_dn = __double2float_rd(hi);
  float lv = __double2float_rn(lo), hv = __double2float_rn(hi);
  // keep the sign of the fp64 bound if rounding flushed it to zero
  if (lo < 0.0 && lv == 0.0f) lv = -1.401298464e-45f;
  if (hi < 0.0 && hv == 0.0f) hv = -1.401298464e-45f;
  if (lo >= 0.0 && lv == 0.0f) lv = 0.0f;
  if (hi >= 0.0 && hv == 0.0f) hv = 0.0f;
  c.lo_val = lv;
  c.hi_val = hv;
  *out = c;
  if (stats_out) {
    stats_out[0] = mean;
    stats_out[1] = sd;
    stats_out[2] = lo;
    stats_out[3] = hi;
  }
}

// Block (256 threads) sums of this thread's (s1, s2) -> partials[blockIdx.x]; the last
// block to get there (ticket on *counter, which the call zeroed) adds all partials in
// index order (strided per-thread sums, then a fixed tree: deterministic), finishes the
// clip parameters and puts the counter back to zero.
__device__ void stats_block_finish(double s1, double s2, double* __restrict__ partials,
                                   unsigned int* __restrict__ counter, double shift, int64_t n,
                                   double k, ClipParams* __restrict__ out,
                                   double* __restrict__ stats_out) {
  __shared__ double sh1[256], sh2[256];
  __shared__ bool last;
  s1 = warp_sum_d(s1);
  s2 = warp_sum_d(s2);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    sh1[w] = s1;
    sh2[w] = s2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t1 = 0.0, t2 = 0.0;
    for (int q = 0; q < (int)(blockDim.x >> 5); ++q) {
      t1 += sh1[q];
      t2 += sh2[q];
    }
    partials[2 * blockIdx.x] = t1;
    partials[2 * blockIdx.x + 1] = t2;
    __threadfence();
    last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  double t1 = 0.0, t2 = 0.0;
  for (int q = threadIdx.x; q < (int)gridDim.x; q += blockDim.x) {
    t1 += __ldcg(partials + 2 * q);
    t2 += __ldcg(partials + 2 * q + 1);
  }
  sh1[threadIdx.x] = t1;
  sh2[threadIdx.x] = t2;
  __syncthreads();
  for (int st = 128; st > 0; st >>= 1) {
    if ((int)threadIdx.x < st) {
      sh1[threadIdx.x] += sh1[threadIdx.x + st];
      sh2[threadIdx.x] += sh2[threadIdx.x + st];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    finish_clip(sh1[0], sh2[0], shift, n, k, out, stats_out);
    *counter = 0u;
  }
}

// Statistics pass (ROW / COL / TENSOR modes with the clip): every element's exact fp64
// delta, shifted by the delta of element 0, summed in fp64.
template <bool BF16>
__global__ void __launch_bounds__(256) k_delta_stats(const uint4* __restrict__ wb,
                                                     const uint4* __restrict__ wf,
                                                     int64_t nvec, int64_t n, double k,
                                                     double* __restrict__ partials,
                                                     unsigned int* __restrict__ counter,
                                                     ClipParams* __restrict__ clip_out,
                                                     double* __restrict__ stats_out) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  using V = Vec<BF16>;
  // shift: delta of element 0 (every thread computes the same value); sums of the
  // shifted deltas are accumulated in fp64 per element
  double shift;
  {
    double d0[V::N];
    V::delta64(wb[0], wf[0], d0);
    shift = d0[0];
  }
  double s1 = 0.0, s2 = 0.0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 b[4], f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      b[u] = ldg_stream(wb + i + u * stride);
      f[u] = ldg_stream(wf + i + u * stride);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      double d[V::N];
      V::delta64(b[u], f[u], d);  // exact difference of the stored values
#pragma unroll
      for (int q = 0; q < V::N; ++q) {
        const double t = d[q] - shift;
        s1 += t;
        s2 = fma(t, t, s2);
      }
    }
  }
  for (; i < nvec; i += stride) {
    double d[V::N];
    V::delta64(ldg_stream(wb + i), ldg_stream(wf + i), d);
#pragma unroll
    for (int q = 0; q < V::N; ++q) {
      const double t = d[q] - shift;
      s1 += t;
      s2 = fma(t, t, s2);
    }
  }
  stats_block_finish(s1, s2, partials, counter, shift, n, k, clip_out, stats_out);
}

// ------------------------------------------------------------------------------------
// main pass for GROUP / ROW / TENSOR
// ------------------------------------------------------------------------------------
// A task is (row, segment of seg_chunks chunks); a chunk is 32 lanes x 16 bytes. Column
// arithmetic is 32-bit (d_in < 2^31 is checked on the host) and the group size is a power
// of two, so group indices are shifts.
template <bool BF16, int SEGC, bool CLIP, bool GROUP>
__global__ void __launch_bounds__(256, 4) k_scale_signpack(
    const uint8_t* __restrict__ wb, const uint8_t* __restrict__ wf, int64_t d_out, int d_in,
    int lg, int seg_chunks, int nseg, const ClipParams* __restrict__ clipp,
    uint32_t* __restrict__ signs, float* __restrict__ scales, double* __restrict__ partials) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  using V = Vec<BF16>;
  constexpr int VEC = V::N;
  constexpr int CHUNK = 32 * VEC;             // columns per chunk
  constexpr int LPW = 32 / VEC;               // lanes per 32-bit sign word
  constexpr int ESZ = BF16 ? 2 : 4;
  const int lane = threadIdx.x & 31;
  const int64_t task = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (task >= d_out * (int64_t)nseg) return;
  const int64_t row = task / nseg;
  const int seg = (int)(task - row * nseg);

  ClipF cp{0.f, 0.f, 0.f, 0.f};
  if (CLIP) cp = load_clip(clipp);

  const uint8_t* rb = wb + row * (int64_t)d_in * ESZ;
  const uint8_t* rf = wf + row * (int64_t)d_in * ESZ;
  uint32_t* srow = signs + row * (int64_t)(d_in >> 5);
  const int G = 1 << lg;
  float* srow_s = GROUP ? scales + row * (int64_t)(d_in >> lg) : nullptr;
  const float invG = 1.0f / (float)G;  // exact: G is a power of two
  const int lpg = G / VEC;              // lanes per group when G <= CHUNK
  const int col_seg0 = seg * seg_chunks * CHUNK;

  double acc_row = 0.0;   // ROW / TENSOR: this lane's share of the segment sum
  double acc_grp = 0.0;   // GROUP with G > CHUNK: running group sum (all lanes equal)

  for (int c0 = 0; c0 < seg_chunks; c0 += SEGC) {
    uint4 b[SEGC], f[SEGC];
    bool valid[SEGC];
#pragma unroll
    for (int u = 0; u < SEGC; ++u) {
      const int col = col_seg0 + (c0 + u) * CHUNK + lane * VEC;
      valid[u] = (c0 + u < seg_chunks) && col < d_in;
      if (valid[u]) {
        b[u] = ldg_stream(rb + (int64_t)col * ESZ);
        f[u] = ldg_stream(rf + (int64_t)col * ESZ);
      }
    }
#pragma unroll
    for (int u = 0; u < SEGC; ++u) {
      const int chunk_col0 = col_seg0 + (c0 + u) * CHUNK;
      if (c0 + u >= seg_chunks || chunk_col0 >= d_in) break;  // warp-uniform
      const int col = chunk_col0 + lane * VEC;
      uint32_t m = 0;
      float a = 0.f;
      if (valid[u]) {
        float d[VEC];
        V::delta(b[u], f[u], d);
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
          const float dc = CLIP ? clamp_delta(d[k], cp) : d[k];
          m |= (dc < 0.f ? 0u : 1u) << k;
          a += fabsf(dc);
        }
      }
      // pack: LPW lanes x VEC bits -> one word, lane order = column order (LSB first)
      uint32_t v = m << (VEC * (lane & (LPW - 1)));
#pragma unroll
      for (int o = 1; o < LPW; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
      if (valid[u] && (lane & (LPW - 1)) == 0) srow[col >> 5] = v;

      if (GROUP) {
        if (G <= CHUNK) {
          float s = a;
          for (int o = 1; o < lpg; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (valid[u] && (lane & (lpg - 1)) == 0) srow_s[col >> lg] = s * invG;
        } else {
          const float s = warp_sum_f(a);
          acc_grp += (double)s;
          if (((chunk_col0 + CHUNK) & (G - 1)) == 0 || chunk_col0 + CHUNK >= d_in) {
            if (lane == 0) srow_s[chunk_col0 >> lg] = (float)(acc_grp * (double)invG);
            acc_grp = 0.0;
          }
        }
      } else {
        acc_row += (double)a;
      }
    }
  }
  if (!GROUP) {
    acc_row = warp_sum_d(acc_row);
    if (lane == 0) partials[row * nseg + seg] = acc_row;
  }
}

// ------------------------------------------------------------------------------------
// COL mode: per-column sums over row tiles
// ------------------------------------------------------------------------------------
// A CTA of 8 warps takes 8 x tile_rows consecutive rows of one column chunk (CHUNK
// columns, VEC per lane). Warp w walks rows w * tile_rows .. of them with UR rows of both
// inputs in flight; the |delta| of a column over those UR rows is summed in fp32 and added
// to the lane's fp64 sums. The CTA then adds its 8 warps' sums in warp order into one fp64
// partial per column: colpart[cta tile][column].
template <bool BF16, bool CLIP>
__global__ void __launch_bounds__(256, 2) k_col_scale_signpack(
    const uint8_t* __restrict__ wb, const uint8_t* __restrict__ wf, int64_t d_out, int64_t d_in,
    int tile_rows, int64_t nchunks, const ClipParams* __restrict__ clipp,
    uint32_t* __restrict__ signs, double* __restrict__ colpart) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  using V = Vec<BF16>;
  constexpr int VEC = V::N;
  constexpr int CHUNK = 32 * VEC;
  constexpr int LPW = 32 / VEC;
  constexpr int ESZ = BF16 ? 2 : 4;
  constexpr int UR = 8;  // rows in flight per warp
  __shared__ double red[8][CHUNK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tile = blockIdx.x / nchunks;
  const int64_t chunk = blockIdx.x % nchunks;
  const int64_t col = chunk * CHUNK + lane * VEC;
  const bool valid = col < d_in;
  ClipF cp{0.f, 0.f, 0.f, 0.f};
  if (CLIP) cp = load_clip(clipp);
  double acc[VEC];
#pragma unroll
  for (int k = 0; k < VEC; ++k) acc[k] = 0.0;
  const int64_t r0 = (tile * 8 + warp) * (int64_t)tile_rows;
  const int64_t r1 = min(d_out, r0 + tile_rows);
  const int64_t words_per_row = d_in >> 5;
  const int64_t rstride = d_in * ESZ;
  const uint8_t* pb = wb + (r0 * d_in + col) * ESZ;
  const uint8_t* pf = wf + (r0 * d_in + col) * ESZ;
  for (int64_t r = r0; r < r1; r += UR, pb += UR * rstride, pf += UR * rstride) {
    uint4 b[UR], f[UR];
#pragma unroll
    for (int u = 0; u < UR; ++u) {
      if (valid && r + u < r1) {
        b[u] = ldg_stream(pb + u * rstride);
        f[u] = ldg_stream(pf + u * rstride);
      }
    }
    float sum[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) sum[k] = 0.f;
#pragma unroll
    for (int u = 0; u < UR; ++u) {
      if (r + u >= r1) break;  // warp-uniform
      uint32_t m = 0;
      if (valid) {
        float d[VEC];
        V::delta(b[u], f[u], d);
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
          const float dc = CLIP ? clamp_delta(d[k], cp) : d[k];
          m |= (dc < 0.f ? 0u : 1u) << k;
          sum[k] += fabsf(dc);
        }
      }
      uint32_t v = m << (VEC * (lane % LPW));
#pragma unroll
      for (int o = 1; o < LPW; o <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
      if (valid && (lane % LPW) == 0) signs[(r + u) * words_per_row + (col >> 5)] = v;
    }
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[k] += (double)sum[k];
  }
#pragma unroll
  for (int k = 0; k < VEC; ++k) red[warp][lane * VEC + k] = acc[k];
  __syncthreads();
  for (int c = threadIdx.x; c < CHUNK; c += blockDim.x) {
    const int64_t cc = chunk * CHUNK + c;
    if (cc < d_in) {
      double t = 0.0;
#pragma unroll
      for (int w = 0; w < 8; ++w) t += red[w][c];
      colpart[tile * d_in + cc] = t;
    }
  }
}

// ------------------------------------------------------------------------------------
// fixed-order reductions of the partial sums
// ------------------------------------------------------------------------------------
// ROW: scales[r] = sum_s partials[r][s] / d_in (one thread per row)
__global__ void k_row_final(const double* __restrict__ partials, int nseg, int64_t d_out,
                            int64_t d_in, float* __restrict__ scales) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= d_out) return;
  double s = 0.0;
  for (int k = 0; k < nseg; ++k) s += partials[r * nseg + k];
  scales[r] = (float)(s / (double)d_in);
}

// COL: scales[i] = sum_t colpart[t][i] / d_out. Block (32 x 8 threads) per 32 columns:
// thread (x, y) sums tiles y, y + 8, ... of column x, then the 8 partial sums are added in
// y order (deterministic).
__global__ void __launch_bounds__(256) k_col_final(const double* __restrict__ colpart, int64_t ntile, int64_t d_out,
                                                   int64_t d_in, float* __restrict__ scales) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  __shared__ double part[8][33];
  const int64_t i = (int64_t)blockIdx.x * 32 + threadIdx.x;
  double sum = 0.0;
  if (i < d_in)
    for (int64_t t = threadIdx.y; t < ntile; t += 8) sum += colpart[t * d_in + i];
  part[threadIdx.y][threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.y == 0 && i < d_in) {
    double tot = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) tot += part[k][threadIdx.x];
    scales[i] = (float)(tot / (double)d_out);
  }
}

// BLOCK: scales[rb][g] = mean over rows r of row block rb of rowmean[r][g] (each row mean
// is over G entries, so this is the mean over the block's entries). Block (32 x 8
// threads) per (row block, 32 groups): thread (x, y) sums rows y, y + 8, ... of group x in
// fp64, then the 8 partial sums are added in y order (deterministic).
__global__ void __launch_bounds__(256) k_block_final(const float* __restrict__ rowmean, int64_t d_out, int64_t ngc,
                                                     int G, float* __restrict__ scales) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  __shared__ double part[8][33];
  const int64_t rb = blockIdx.x;
  const int64_t g = (int64_t)blockIdx.y * 32 + threadIdx.x;
  const int64_t r0 = rb * G, r1 = r0 + G < d_out ? r0 + G : d_out;
  double sum = 0.0;
  if (g < ngc)
    for (int64_t r = r0 + threadIdx.y; r < r1; r += 8) sum += (double)rowmean[r * ngc + g];
  part[threadIdx.y][threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.y == 0 && g < ngc) {
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += part[k][threadIdx.x];
    scales[rb * ngc + g] = (float)(t / (double)(r1 - r0));
  }
}

// TENSOR: one block; strided per-thread sums then a fixed tree
__global__ void k_tensor_final(const double* __restrict__ partials, int64_t n, double count,
                               float* __restrict__ scales) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  __shared__ double sh[256];
  double s = 0.0;
  for (int64_t k = threadIdx.x; k < n; k += blockDim.x) s += partials[k];
  sh[threadIdx.x] = s;
  __syncthreads();
  for (int st = 128; st > 0; st >>= 1) {
    if ((int)threadIdx.x < st) sh[threadIdx.x] += sh[threadIdx.x + st];
    __syncthreads();
  }
  if (threadIdx.x == 0) scales[0] = (float)(sh[0] / count);
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
namespace {

struct CompressPlan {
  bool bf16;
  int chunk;          // columns per warp chunk
  int seg_chunks;     // chunks per task (GROUP / ROW / TENSOR)
  int nseg;           // tasks per row
  int stats_blocks;   // blocks of the stats pass
  int main_blocks;    // blocks of the main pass (GROUP / ROW / TENSOR)
  int col_tile;       // rows per tile (COL)
  int64_t nchunks;    // chunks per row
  int64_t ntile;      // row tiles (COL)
  size_t off_clip, off_cnt, off_stats, off_part, total;
};

bd_status plan_compress(int32_t dtype, int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg,
                        CompressPlan* p) {
  if (!cfg) return BD_ERR_NULL;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_DTYPE;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (d_in > ((int64_t)1 << 30) || d_out > ((int64_t)1 << 40)) return BD_ERR_SHAPE;
  if (cfg->mode < BD_SCALE_GROUP || cfg->mode > BD_SCALE_BLOCK) return BD_ERR_CONFIG;
  if (cfg->clip != 0 && cfg->clip != 1) return BD_ERR_CONFIG;
  if (cfg->clip && !(cfg->clip_k >= 0.0f)) return BD_ERR_CONFIG;
  const int64_t G = cfg->group_size;
  const bool grouped = cfg->mode == BD_SCALE_GROUP || cfg->mode == BD_SCALE_BLOCK;
  if (!scale_mode_ok(cfg->mode, cfg->group_size, d_in)) return BD_ERR_CONFIG;
  if (cfg->mode == BD_SCALE_BLOCK &&
      ((d_out + G - 1) / G > 0x7FFFFFFF || (d_in / G + 31) / 32 > 65535))  // the block reduction's grid
    return BD_ERR_SHAPE;
  p->bf16 = dtype == BD_BF16;
  p->chunk = p->bf16 ? 256 : 128;
  p->nchunks = (d_in + p->chunk - 1) / p->chunk;
  const int sms = sm_count();
  const int64_t target_tasks = (int64_t)sms * 64;  // warps in flight we want
  int segc = 4;
  while (segc > 1 && d_out * ((p->nchunks + segc - 1) / segc) < target_tasks) segc >>= 1;
  if (grouped && G > p->chunk) {
    const int need = (int)(G / p->chunk);
    segc = ((segc + need - 1) / need) * need;
  }
  p->seg_chunks = segc;
  p->nseg = (int)((p->nchunks + segc - 1) / segc);
  p->stats_blocks = sms * 4;
  p->main_blocks = (int)((d_out * (int64_t)p->nseg + 7) / 8);
  // COL: CTAs of 8 warps x tile rows, tile 8..64 rows: the longest that still gives
  // every SM 8 CTAs (else 8)
  int tile = 64;
  while (tile > 8 && ((d_out + 8 * tile - 1) / (8 * tile)) * p->nchunks < (int64_t)sms * 8) tile >>= 1;
  p->col_tile = tile;
  p->ntile = (d_out + 8 * tile - 1) / (8 * tile);
  // one-dimensional grids of the main passes
  if ((d_out * (int64_t)p->nseg + 7) / 8 > 0x7FFFFFFF || p->ntile * p->nchunks > 0x7FFFFFFF) return BD_ERR_SHAPE;
  size_t off = kStatusBytes;
  p->off_clip = off;
  off = align_up(off + sizeof(ClipParams), 256);
  p->off_cnt = off;
  off = align_up(off + sizeof(unsigned int), 256);
  p->off_stats = off;
  off = align_up(off + (size_t)p->stats_blocks * 2 * sizeof(double), 256);
  p->off_part = off;
  size_t part = 0;
  if (cfg->mode == BD_SCALE_ROW || cfg->mode == BD_SCALE_TENSOR)
    part = (size_t)d_out * p->nseg * sizeof(double);
  else if (cfg->mode == BD_SCALE_COL)
    part = (size_t)p->ntile * d_in * sizeof(double);
  else if (cfg->mode == BD_SCALE_BLOCK)
    part = (size_t)d_out * (size_t)(d_in / G) * sizeof(float);  // row group means
  off = align_up(off + part, 256);
  p->total = off;
  return BD_OK;
}

template <bool BF16>
bd_status launch_compress(const CompressPlan& p, const void* w_base, const void* w_fine,
                          int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg,
                          uint32_t* signs, float* scales, double* stats_out, uint8_t* ws,
                          cudaStream_t s) {
  ClipParams* clipp = nullptr;
  const int64_t nvec = d_out * d_in * (BF16 ? 2 : 4) / 16;
  const bool clip = cfg->clip != 0;
  unsigned int* counter = reinterpret_cast<unsigned int*>(ws + p.off_cnt);
  double* stat_parts = reinterpret_cast<double*>(ws + p.off_stats);
  if (clip) {
    clipp = reinterpret_cast<ClipParams*>(ws + p.off_clip);
    // the last-block ticket of the statistics starts from zero in every call
    BD_CUDA_TRY(cudaMemsetAsync(counter, 0, sizeof(unsigned int), s));
  }
  if (clip) {
    launch_begin(K_DELTA_STATS, s);
    BD_CUDA_TRY(launch_pdl(k_delta_stats<BF16>, dim3(p.stats_blocks), dim3(256), 0, s, (const uint4*)w_base,
                           (const uint4*)w_fine, nvec, d_out * d_in, (double)cfg->clip_k, stat_parts, counter,
                           clipp, stats_out));
    launch_end(K_DELTA_STATS, s);
    BD_LAUNCH_CHECK();
  }
  double* part = reinterpret_cast<double*>(ws + p.off_part);
  if (cfg->mode == BD_SCALE_COL) {
    const int64_t blocks = p.ntile * p.nchunks;  // grid limit checked in the plan
    launch_begin(K_COL_SCALE_SIGNPACK, s);
    auto kcol = clip ? k_col_scale_signpack<BF16, true> : k_col_scale_signpack<BF16, false>;
    BD_CUDA_TRY(launch_pdl(kcol, dim3((unsigned)blocks), dim3(256), 0, s, (const uint8_t*)w_base,
                           (const uint8_t*)w_fine, d_out, d_in, p.col_tile, p.nchunks, (const ClipParams*)clipp,
                           signs, part));
    launch_end(K_COL_SCALE_SIGNPACK, s);
    BD_LAUNCH_CHECK();
    launch_begin(K_SCALE_FINAL, s);
    BD_CUDA_TRY(launch_pdl(k_col_final, dim3((unsigned)((d_in + 31) / 32)), dim3(32, 8), 0, s, (const double*)part,
                           p.ntile, d_out, d_in, scales));
    launch_end(K_SCALE_FINAL, s);
    BD_LAUNCH_CHECK();
    return BD_OK;
  }
  const unsigned blocks = (unsigned)p.main_blocks;
  const bool group = cfg->mode == BD_SCALE_GROUP || cfg->mode == BD_SCALE_BLOCK;
  int lg = 0;
  if (group)
    while ((1 << lg) < cfg->group_size) ++lg;
  const int din = (int)d_in;
  // BLOCK: the per-row group means go to the workspace, the block means follow
  float* group_out = cfg->mode == BD_SCALE_BLOCK ? reinterpret_cast<float*>(part) : scales;
#define BD_SIGNPACK(SEGC, CLIP, GRP)                                                                    \
  BD_CUDA_TRY(launch_pdl(k_scale_signpack<BF16, SEGC, CLIP, GRP>, dim3(blocks), dim3(256), 0, s,           \
                         (const uint8_t*)w_base, (const uint8_t*)w_fine, d_out, din, lg, p.seg_chunks,     \
                         p.nseg, (const ClipParams*)clipp, signs, group_out, part))
  launch_begin(K_SCALE_SIGNPACK, s);
  if (p.seg_chunks >= 4) {
    if (clip) { if (group) BD_SIGNPACK(4, true, true); else BD_SIGNPACK(4, true, false); }
    else { if (group) BD_SIGNPACK(4, false, true); else BD_SIGNPACK(4, false, false); }
  } else {
    if (clip) { if (group) BD_SIGNPACK(2, true, true); else BD_SIGNPACK(2, true, false); }
    else { if (group) BD_SIGNPACK(2, false, true); else BD_SIGNPACK(2, false, false); }
  }
#undef BD_SIGNPACK
  launch_end(K_SCALE_SIGNPACK, s);
  BD_LAUNCH_CHECK();
  if (cfg->mode == BD_SCALE_ROW) {
    launch_begin(K_SCALE_FINAL, s);
    BD_CUDA_TRY(launch_pdl(k_row_final, dim3((unsigned)((d_out + 255) / 256)), dim3(256), 0, s, (const double*)part,
                           p.nseg, d_out, d_in, scales));
    launch_end(K_SCALE_FINAL, s);
    BD_LAUNCH_CHECK();
  } else if (cfg->mode == BD_SCALE_BLOCK) {
    const int64_t ngc = d_in >> lg;
    launch_begin(K_SCALE_FINAL, s);
    const int64_t nrb = (d_out + cfg->group_size - 1) / cfg->group_size;  // grid limits checked in the plan
    BD_CUDA_TRY(launch_pdl(k_block_final, dim3((unsigned)nrb, (unsigned)((ngc + 31) / 32)), dim3(32, 8), 0, s,
                           reinterpret_cast<const float*>(part), d_out, ngc, (int)cfg->group_size, scales));
    launch_end(K_SCALE_FINAL, s);
    BD_LAUNCH_CHECK();
  } else if (cfg->mode == BD_SCALE_TENSOR) {
    launch_begin(K_SCALE_FINAL, s);
    BD_CUDA_TRY(launch_pdl(k_tensor_final, dim3(1), dim3(256), 0, s, (const double*)part, d_out * (int64_t)p.nseg,
                           (double)d_out * (double)d_in, scales));
    launch_end(K_SCALE_FINAL, s);
    BD_LAUNCH_CHECK();
  }
  return BD_OK;
}

// Host-side checks of a compress call (nothing is launched); fills the plan.
bd_status compress_check(const void* w_base, const void* w_fine, int32_t dtype, int64_t d_out,
                         int64_t d_in, const bd_compress_cfg* cfg, const uint32_t* signs_out,
                         const float* scales_out, const double* stats_out, CompressPlan* p) {
  bd_status st = plan_compress(dtype, d_out, d_in, cfg, p);
  if (st != BD_OK) return st;
  if (!w_base || !w_fine || !signs_out || !scales_out) return BD_ERR_NULL;
  if (!aligned16(w_base) || !aligned16(w_fine) || !aligned16(signs_out) || !aligned16(scales_out))
    return BD_ERR_ALIGN;
  if (stats_out && (reinterpret_cast<uintptr_t>(stats_out) & 7u)) return BD_ERR_ALIGN;
  return BD_OK;
}

bd_status compress_run(const CompressPlan& p, const void* w_base, const void* w_fine, int64_t d_out,
                       int64_t d_in, const bd_compress_cfg* cfg, uint32_t* signs_out, float* scales_out,
                       double* stats_out, void* workspace, size_t ws_bytes, cudaStream_t s) {
  if (!workspace || ws_bytes < p.total) return BD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BD_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (p.bf16)
    return launch_compress<true>(p, w_base, w_fine, d_out, d_in, cfg, signs_out, scales_out,
                                 stats_out, ws, s);
  return launch_compress<false>(p, w_base, w_fine, d_out, d_in, cfg, signs_out, scales_out,
                                stats_out, ws, s);
}

}  // namespace

bd_status compress_impl(const void* w_base, const void* w_fine, int32_t dtype, int64_t d_out,
                        int64_t d_in, const bd_compress_cfg* cfg, uint32_t* signs_out,
                        float* scales_out, double* stats_out, void* workspace, size_t ws_bytes,
                        cudaStream_t s) {
  CompressPlan p;
  bd_status st = compress_check(w_base, w_fine, dtype, d_out, d_in, cfg, signs_out, scales_out,
                                stats_out, &p);
  if (st != BD_OK) return st;
  return compress_run(p, w_base, w_fine, d_out, d_in, cfg, signs_out, scales_out, stats_out,
                      workspace, ws_bytes, s);
}

size_t compress_workspace_size(int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg) {
  CompressPlan p;
  if (plan_compress(BD_BF16, d_out, d_in, cfg, &p) != BD_OK) return 0;
  CompressPlan q;
  plan_compress(BD_F32, d_out, d_in, cfg, &q);
  return p.total > q.total ? p.total : q.total;
}

}  // namespace bd

extern "C" bd_status bd_compress(const void* w_base, const void* w_fine, int32_t dtype,
                                 int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg,
                                 uint32_t* signs_out, float* scales_out, double* stats_out,
                                 void* workspace, size_t ws_bytes, void* stream) {
  return bd::compress_impl(w_base, w_fine, dtype, d_out, d_in, cfg, signs_out, scales_out,
                           stats_out, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" size_t bd_compress_workspace_size(int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg) {
  return bd::compress_workspace_size(d_out, d_in, cfg);
}

// ------------------------------------------------------------------------------------
// bd_compress_noalloc: bd_compress for callers that cannot allocate device memory.
// Its scratch is a fixed array in this library's device image instead of a caller
// workspace. Every GPU that loads the library holds the array until the process exits.
// ------------------------------------------------------------------------------------
#include <mutex>

namespace bd {

constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;  // BD_NOALLOC_SCRATCH_BYTES

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device (with
// that device current) and cached. The cached address belongs to the device's context of
// the time: after cudaDeviceReset the library must be reloaded before this call is used.
static bd_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    (void)cudaGetLastError();
    return BD_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return BD_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return BD_OK;
}

}  // namespace bd

extern "C" bd_status bd_compress_noalloc(const void* w_base, const void* w_fine, int32_t dtype,
                                         int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg,
                                         uint32_t* signs_out, float* scales_out,
                                         double* stats_out, void* stream) {
  // the arguments first, as for bd_compress
  bd::CompressPlan p;
  bd_status st = bd::compress_check(w_base, w_fine, dtype, d_out, d_in, cfg, signs_out, scales_out,
                                    stats_out, &p);
  if (st != BD_OK) return st;
  if (p.total > bd::kNoAllocScratchBytes) return BD_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = bd::noalloc_scratch(&scratch);
  if (st != BD_OK) return st;
  return bd::compress_run(p, w_base, w_fine, d_out, d_in, cfg, signs_out, scales_out, stats_out, scratch,
                          bd::kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}
