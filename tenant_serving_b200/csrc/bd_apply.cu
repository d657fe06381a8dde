// bd_apply_multi: y_t = W_base x_t + Delta_hat_{u(t)} x_t for a batch of mixed tenants.
//
// "BitDelta Guide", "Systems Mechanics: 1. Decoupled Forward Pass" (shared base product,
// per-tenant delta product) and "2. Fused Dequantization ..." (sign bits stay packed in
// HBM and are expanded on chip). The pages give no kernel for this GPU; the design here:
//
//   k_tenant_bucket  one CTA: counting sort of the tenant ids into segments (tenant,
//                    start, length) and a token permutation. Invalid ids set a status
//                    bit and join the base-only segment. No host synchronisation.
//   base product     bf16: tcgen05 tensor-core GEMM (bd_base_tc.cu), fp32: k_base_gemv.
//                    Both write fp32 partial sums y_part[kz][t][row].
//   k_delta_lut      one CTA per (segment, 1024-row block): streams the tenant's sign
//                    words through shared memory 256 columns at a time and, per token,
//                    turns every byte of signs into ONE table lookup: for each 8-column
//                    chunk a 256-entry table holds sum_j (+/-) x_j for every sign
//                    pattern (built per window from two 16-entry nibble tables). The
//                    lookup order is rotated by row so the 32 lanes of a warp always hit
//                    32 different banks. Group scales multiply per 32-bit word, column
//                    scales are folded into x before the tables are built, row / tensor
//                    scales multiply at the end. The epilogue adds the base partial sums
//                    in a fixed order and writes y (bf16 or fp32) in request order.
#include "bd_internal.cuh"

namespace bd {

struct TcPlan {
  int n_tile, tiles_n, tiles_m, kblocks, kb_per_split, ksplit, stages;
  size_t smem;
};
TcPlan plan_base_tc(int64_t d_out, int64_t d_in, int64_t batch);
bd_status launch_base_tc(const TcPlan& p, const void* w_base, const void* x, int64_t d_out,
                         int64_t d_in, int64_t batch, float* y_part, uint32_t* status,
                         cudaStream_t s);

constexpr int kMaxTenants = 16384;
constexpr int kMaxBatch = 65536;

// ------------------------------------------------------------------------------------
// segments
// ------------------------------------------------------------------------------------
struct SegTable {
  int32_t n_seg;
  int32_t pad[3];
  // followed in memory by: tenant[max_seg], start[max_seg], len[max_seg], perm[batch]
};

__global__ void __launch_bounds__(1024) k_tenant_bucket(const int32_t* __restrict__ ids, int batch,
                                                        int n_tenants, int max_seg,
                                                        int32_t* __restrict__ seg_base,
                                                        uint32_t* __restrict__ status) {
  extern __shared__ int32_t cnt[];  // n_tenants + 1 counters (last = base only)
  __shared__ int32_t warp_tot[32], warp_seg[32];
  __shared__ int32_t bad;
  const int nkeys = n_tenants + 1;
  int32_t* seg_tenant = seg_base + 4;
  int32_t* seg_start = seg_tenant + max_seg;
  int32_t* seg_len = seg_start + max_seg;
  int32_t* perm = seg_len + max_seg;
  if (threadIdx.x == 0) {
    status[0] = 0;  // the status word reports this call
    bad = 0;
  }
  for (int k = threadIdx.x; k < nkeys; k += blockDim.x) cnt[k] = 0;
  __syncthreads();
  for (int t = threadIdx.x; t < batch; t += blockDim.x) {
    int u = ids[t];
    if (u < -1 || u >= n_tenants) {
      bad = 1;
      u = -1;
    }
    atomicAdd(&cnt[u < 0 ? n_tenants : u], 1);
  }
  __syncthreads();
  // exclusive scan of counts and of "count > 0" (segment index), contiguous per thread
  const int per = (nkeys + blockDim.x - 1) / blockDim.x;
  const int k0 = threadIdx.x * per, k1 = min(nkeys, k0 + per);
  int tot = 0, nz = 0;
  for (int k = k0; k < k1; ++k) {
    tot += cnt[k];
    nz += cnt[k] > 0;
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int itot = tot, inz = nz;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int a = __shfl_up_sync(0xffffffffu, itot, o), b = __shfl_up_sync(0xffffffffu, inz, o);
    if (lane >= o) {
      itot += a;
      inz += b;
    }
  }
  if (lane == 31) {
    warp_tot[w] = itot;
    warp_seg[w] = inz;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    int a = lane < nw ? warp_tot[lane] : 0, b = lane < nw ? warp_seg[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int c = __shfl_up_sync(0xffffffffu, a, o), d = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        a += c;
        b += d;
      }
    }
    if (lane < nw) {
      warp_tot[lane] = a;
      warp_seg[lane] = b;
    }
  }
  __syncthreads();
  int off = itot - tot + (w > 0 ? warp_tot[w - 1] : 0);
  int sidx = inz - nz + (w > 0 ? warp_seg[w - 1] : 0);
  for (int k = k0; k < k1; ++k) {
    const int c = cnt[k];
    if (c > 0) {
      seg_tenant[sidx] = (k == n_tenants) ? -1 : k;
      seg_start[sidx] = off;
      seg_len[sidx] = c;
      ++sidx;
    }
    cnt[k] = off;  // becomes the scatter cursor
    off += c;
  }
  if (threadIdx.x == blockDim.x - 1) seg_base[0] = sidx;  // last thread holds the total
  __syncthreads();
  for (int t = threadIdx.x; t < batch; t += blockDim.x) {
    int u = ids[t];
    if (u < -1 || u >= n_tenants) u = -1;
    const int pos = atomicAdd(&cnt[u < 0 ? n_tenants : u], 1);
    perm[pos] = t;
  }
  if (threadIdx.x == 0 && bad) atomicOr(status, BD_DEV_TENANT_RANGE);
}

// ------------------------------------------------------------------------------------
// fp32 base product on CUDA cores (small problems; the bf16 path uses tensor cores)
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_base_gemv_f32(const float* __restrict__ W,
                                                       const float* __restrict__ X, int64_t d_out,
                                                       int64_t d_in, int batch,
                                                       float* __restrict__ y_part) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= d_out) return;
  const float* wr = W + row * d_in;
  for (int t0 = 0; t0 < batch; t0 += 8) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int64_t k = lane * 4; k < d_in; k += 128) {
      const float4 w = *reinterpret_cast<const float4*>(wr + k);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (t0 + j < batch) {
          const float4 x = *reinterpret_cast<const float4*>(X + (int64_t)(t0 + j) * d_in + k);
          acc[j] = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, acc[j]))));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = warp_sum_f(acc[j]);
      if (lane == 0 && t0 + j < batch) y_part[(int64_t)(t0 + j) * d_out + row] = v;
    }
  }
}

// ------------------------------------------------------------------------------------
// delta product with per-chunk sign lookup tables
// ------------------------------------------------------------------------------------
constexpr int LUT_R = 1024;                 // rows per CTA
constexpr int LUT_THREADS = 512;            // 16 warps
constexpr int LUT_WARPS = LUT_THREADS / 32;
constexpr int LUT_TT = 4;                   // tokens per pass (two 64 KB table pages)
constexpr int LUT_W = 256;                  // columns per window (8 sign words per row)
constexpr int LUT_NQ = LUT_R / (LUT_WARPS * 4);  // row quads per warp
constexpr int LUT_PAGE = 65536;             // bytes: 256 sign patterns x 64 slots x 4 B
constexpr int LUT_BITS_BYTES = LUT_R * 32;  // one window of sign words for LUT_R rows
constexpr size_t LUT_SMEM = (size_t)(LUT_TT / 2) * LUT_PAGE + 2 * LUT_BITS_BYTES + 64;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool XBF16>
__device__ __forceinline__ void load_x8(const void* x, int64_t off, float* v) {
  if (XBF16) {
    const uint4 q = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + off);
    const uint32_t a[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = bf16lo(a[k]);
      v[2 * k + 1] = bf16hi(a[k]);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + off);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ float ld_scale(const void* s, bool f16, int64_t i) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

template <bool XBF16>
__global__ void __launch_bounds__(LUT_THREADS, 1) k_delta_lut(
    const bd_tenant* __restrict__ tenants, int n_tenants, bool scale_f16,
    const int32_t* __restrict__ seg_base, int max_seg, const void* __restrict__ x,
    const float* __restrict__ y_part, int ksplit, int64_t d_out, int64_t d_in, int batch,
    void* __restrict__ y, bool y_bf16, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int seg = blockIdx.y;
  const int n_seg = seg_base[0];
  if (seg >= n_seg) return;
  const int32_t* seg_tenant = seg_base + 4;
  const int32_t* seg_start = seg_tenant + max_seg;
  const int32_t* seg_len = seg_start + max_seg;
  const int32_t* perm = seg_len + max_seg;
  const int u_in = seg_tenant[seg];
  const int start = seg_start[seg], len = seg_len[seg];
  const int64_t r0 = (int64_t)blockIdx.x * LUT_R;
  const int rows = (int)min((int64_t)LUT_R, d_out - r0);

  float* lut = reinterpret_cast<float*>(smem);
  uint8_t* bits_s = smem + (size_t)(LUT_TT / 2) * LUT_PAGE;
  float* out_s = lut;  // reused after the last window
  int* tok_s = reinterpret_cast<int*>(bits_s + 2 * LUT_BITS_BYTES);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane >> 3;        // row inside the warp's row quad
  const int wd = lane & 7;        // sign word inside the 256-column window
  const int64_t wpr = d_in >> 5;  // sign words per row
  const int nwin = (int)((d_in + LUT_W - 1) / LUT_W);

  bd_tenant T;
  int mode = BD_SCALE_GROUP, G = 128;
  int u = u_in;
  if (u >= 0) {
    T = tenants[u];
    mode = T.mode;
    G = T.group_size;
    // the table lives in device memory, so its records are checked here
    const bool ok_mode = mode >= BD_SCALE_GROUP && mode <= BD_SCALE_TENSOR;
    const bool ok_group = mode != BD_SCALE_GROUP ||
                          (G >= 32 && (G & (G - 1)) == 0 && (d_in % G) == 0);
    const bool ok_ptr = T.signs != nullptr && T.scales != nullptr &&
                        ((reinterpret_cast<uintptr_t>(T.signs) | reinterpret_cast<uintptr_t>(T.scales)) & 15u) == 0;
    if (!(ok_mode && ok_group && ok_ptr)) {
      if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, BD_DEV_TENANT_RECORD);
      u = -1;  // base product only
    }
  }

  // per-lane lookup constants: byte order rotated by q so a warp hits 32 distinct banks
  uint32_t sel[4], slot[2][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int b = (j + q) & 3;
    sel[j] = 0x7604u | ((uint32_t)b << 4);
    slot[0][j] = 4u * (uint32_t)(4 * wd + b);
    slot[1][j] = 4u * (uint32_t)(32 + 4 * wd + b);
  }

  for (int tg = 0; tg < len; tg += LUT_TT) {
    const int ntok = min(LUT_TT, len - tg);
    if (tid < LUT_TT) tok_s[tid] = tid < ntok ? perm[start + tg + tid] : -1;
    float acc[LUT_NQ][LUT_TT];
#pragma unroll
    for (int i = 0; i < LUT_NQ; ++i)
#pragma unroll
      for (int t = 0; t < LUT_TT; ++t) acc[i][t] = 0.f;
    __syncthreads();

    if (u >= 0) {
      // stage window 0 of sign words
      // 16-byte copies when every row starts 16-byte aligned and windows are whole
      // (d_in % 256 == 0), else one 4-byte copy per sign word.
      const bool whole = (d_in % LUT_W) == 0;
      auto stage = [&](int win, int buf) {
        uint8_t* dst = bits_s + (size_t)buf * LUT_BITS_BYTES;
        const int64_t w0 = (int64_t)win * (LUT_W / 32);
        if (whole) {
          for (int i = tid; i < LUT_R * 2; i += LUT_THREADS) {
            const int rl = i >> 1, half = i & 1;
            if (rl < rows) cp_async16(dst + rl * 32 + half * 16, T.signs + (r0 + rl) * wpr + w0 + half * 4);
          }
        } else {
          for (int i = tid; i < LUT_R * 8; i += LUT_THREADS) {
            const int rl = i >> 3, k = i & 7;
            if (rl < rows && w0 + k < wpr) cp_async4(dst + rl * 32 + k * 4, T.signs + (r0 + rl) * wpr + w0 + k);
          }
        }
      };
      stage(0, 0);
      cp_async_commit();
      for (int win = 0; win < nwin; ++win) {
        if (win + 1 < nwin) stage(win + 1, (win + 1) & 1);
        cp_async_commit();
        // ---- build the tables of this window: T[v][slot], slot = 32*(tt&1) + chunk
        {
          const int c = lane;      // chunk (8 columns) of the window
          const int h = warp;      // high nibble of the sign byte this thread fills
          const int64_t col = (int64_t)win * LUT_W + 8 * c;
#pragma unroll
          for (int tt = 0; tt < LUT_TT; ++tt) {
            if (tt < ntok) {
              const int t = tok_s[tt];
              float xv[8];
              if (col < d_in) {
                load_x8<XBF16>(x, (int64_t)t * d_in + col, xv);
                if (mode == BD_SCALE_COL) {
#pragma unroll
                  for (int k = 0; k < 8; ++k) xv[k] *= ld_scale(T.scales, scale_f16, col + k);
                }
              } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) xv[k] = 0.f;
              }
              float p01[4], p23[4];
#pragma unroll
              for (int n = 0; n < 4; ++n) {
                p01[n] = ((n & 1) ? xv[0] : -xv[0]) + ((n & 2) ? xv[1] : -xv[1]);
                p23[n] = ((n & 1) ? xv[2] : -xv[2]) + ((n & 2) ? xv[3] : -xv[3]);
              }
              const float hi = (((h & 1) ? xv[4] : -xv[4]) + ((h & 2) ? xv[5] : -xv[5])) +
                               (((h & 4) ? xv[6] : -xv[6]) + ((h & 8) ? xv[7] : -xv[7]));
              float* page = lut + (size_t)(tt >> 1) * (LUT_PAGE / 4);
              const int sl = 32 * (tt & 1) + c;
#pragma unroll
              for (int n = 0; n < 16; ++n) {
                const float lo = p01[n & 3] + p23[n >> 2];
                page[((h << 4) | n) * 64 + sl] = lo + hi;
              }
            }
          }
        }
        if (win + 1 < nwin) cp_async_wait<1>();
        else cp_async_wait<0>();
        __syncthreads();
        // ---- lookups
        const uint32_t* wbuf = reinterpret_cast<const uint32_t*>(bits_s + (size_t)(win & 1) * LUT_BITS_BYTES);
        const int64_t wcol = (int64_t)win * LUT_W + 32 * wd;
        const bool wvalid = wcol < d_in;
#pragma unroll
        for (int iq = 0; iq < LUT_NQ; ++iq) {
          const int rl = (warp * LUT_NQ + iq) * 4 + q;
          if (rl < rows && wvalid) {
            const uint32_t word = wbuf[rl * 8 + wd];
            float s = 1.f;
            if (mode == BD_SCALE_GROUP)
              s = ld_scale(T.scales, scale_f16, (r0 + rl) * (d_in / G) + wcol / G);
#pragma unroll
            for (int tt = 0; tt < LUT_TT; ++tt) {
              const uint8_t* page = reinterpret_cast<const uint8_t*>(lut) + (size_t)(tt >> 1) * LUT_PAGE;
              float p = 0.f;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t idx = __byte_perm(word, slot[tt & 1][j], sel[j]);
                p += *reinterpret_cast<const float*>(page + idx);
              }
              acc[iq][tt] = fmaf(s, p, acc[iq][tt]);
            }
          }
        }
        __syncthreads();
      }
    }
    // ---- reduce the 8 lanes of each row and stage per-token results
#pragma unroll
    for (int iq = 0; iq < LUT_NQ; ++iq) {
#pragma unroll
      for (int tt = 0; tt < LUT_TT; ++tt) {
        float v = acc[iq][tt];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        const int rl = (warp * LUT_NQ + iq) * 4 + q;
        if (wd == 0) out_s[tt * LUT_R + rl] = v;
      }
    }
    __syncthreads();
    // ---- combine with the base product and write y in request order
    float rs = 1.f;
    if (u >= 0 && mode == BD_SCALE_TENSOR) rs = ld_scale(T.scales, scale_f16, 0);
    for (int tt = 0; tt < ntok; ++tt) {
      const int t = tok_s[tt];
      for (int rl = tid; rl < rows; rl += LUT_THREADS) {
        const int64_t row = r0 + rl;
        float base = 0.f;
        for (int kz = 0; kz < ksplit; ++kz) base += y_part[((int64_t)kz * batch + t) * d_out + row];
        float d = 0.f;
        if (u >= 0) {
          float sc = rs;
          if (mode == BD_SCALE_ROW) sc = ld_scale(T.scales, scale_f16, row);
          d = sc * out_s[tt * LUT_R + rl];
        }
        const float v = base + d;
        if (y_bf16)
          reinterpret_cast<uint16_t*>(y)[(int64_t)t * d_out + row] = (uint16_t)f2bf_bits(v);
        else
          reinterpret_cast<float*>(y)[(int64_t)t * d_out + row] = v;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
namespace {
struct ApplyLayout {
  int max_seg;
  TcPlan tc;
  int ksplit;
  size_t off_seg, off_part, total;
};

ApplyLayout layout_apply(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants, bool tc) {
  ApplyLayout L;
  L.max_seg = (int)(batch < (int64_t)n_tenants + 1 ? batch : (int64_t)n_tenants + 1);
  if (L.max_seg < 1) L.max_seg = 1;
  L.ksplit = 1;
  if (tc) {
    L.tc = plan_base_tc(d_out, d_in, batch);
    L.ksplit = L.tc.ksplit;
  }
  size_t off = kStatusBytes;
  L.off_seg = off;
  off = align_up(off + (16 + 3 * (size_t)L.max_seg * 4 + (size_t)batch * 4), 256);
  L.off_part = off;
  off = align_up(off + (size_t)L.ksplit * batch * d_out * sizeof(float), 256);
  L.total = off;
  return L;
}
}  // namespace

size_t apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants) {
  if (d_out < 1 || d_in < 32 || batch < 0 || n_tenants < 0) return 0;
  const size_t a = layout_apply(d_out, d_in, batch, n_tenants, true).total;
  const size_t b = layout_apply(d_out, d_in, batch, n_tenants, false).total;
  return a > b ? a : b;
}

bd_status apply_impl(const void* w_base, int32_t w_dtype, int64_t d_out, int64_t d_in,
                     const bd_tenant* tenants, int32_t n_tenants, int32_t scale_dtype,
                     const int32_t* tenant_ids, const void* x, int64_t batch, void* y,
                     int32_t y_dtype, void* workspace, size_t ws_bytes, cudaStream_t s) {
  if (w_dtype != BD_BF16 && w_dtype != BD_F32) return BD_ERR_DTYPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if (y_dtype != BD_BF16 && y_dtype != BD_F32) return BD_ERR_DTYPE;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (batch < 0 || batch > kMaxBatch || n_tenants < 0 || n_tenants > kMaxTenants) return BD_ERR_SHAPE;
  if (batch == 0) return BD_OK;
  if (!w_base || !x || !y || !tenant_ids) return BD_ERR_NULL;
  if (n_tenants > 0 && !tenants) return BD_ERR_NULL;
  if (!aligned16(w_base) || !aligned16(x) || !aligned16(y) || !aligned16(tenant_ids) ||
      (tenants && (reinterpret_cast<uintptr_t>(tenants) & 7u)))
    return BD_ERR_ALIGN;
  const bool tc = w_dtype == BD_BF16;
  ApplyLayout L = layout_apply(d_out, d_in, batch, n_tenants, tc);
  if (!workspace || ws_bytes < L.total) return BD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BD_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  int32_t* seg = reinterpret_cast<int32_t*>(ws + L.off_seg);
  float* y_part = reinterpret_cast<float*>(ws + L.off_part);

  // 1. bucket tokens by tenant
  const size_t bucket_smem = (size_t)(n_tenants + 1) * sizeof(int32_t);
  static bool bucket_attr = false;
  if (!bucket_attr) {
    if (cudaFuncSetAttribute(k_tenant_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (kMaxTenants + 1) * (int)sizeof(int32_t)) != cudaSuccess) {
      (void)cudaGetLastError();
      return BD_ERR_CUDA;
    }
    bucket_attr = true;
  }
  launch_begin(K_TENANT_BUCKET, s);
  k_tenant_bucket<<<1, 1024, bucket_smem, s>>>(tenant_ids, (int)batch, n_tenants, L.max_seg, seg,
                                               status);
  launch_end(K_TENANT_BUCKET, s);
  BD_LAUNCH_CHECK();

  // 2. base product (fp32 partial sums)
  if (tc) {
    bd_status st = launch_base_tc(L.tc, w_base, x, d_out, d_in, batch, y_part, status, s);
    if (st != BD_OK) return st;
  } else {
    const int64_t blocks = (d_out * 32 + 255) / 256;
    launch_begin(K_BASE_GEMV, s);
    k_base_gemv_f32<<<(unsigned)blocks, 256, 0, s>>>((const float*)w_base, (const float*)x, d_out,
                                                     d_in, (int)batch, y_part);
    launch_end(K_BASE_GEMV, s);
    BD_LAUNCH_CHECK();
  }

  // 3. delta product per (segment, row block) fused with the combine
  static bool lut_attr[2] = {false, false};
  auto kfn = tc ? k_delta_lut<true> : k_delta_lut<false>;
  if (!lut_attr[tc ? 1 : 0]) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LUT_SMEM) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return BD_ERR_CUDA;
    }
    lut_attr[tc ? 1 : 0] = true;
  }
  dim3 grid((unsigned)((d_out + LUT_R - 1) / LUT_R), (unsigned)L.max_seg);
  launch_begin(K_DELTA_LUT, s);
  kfn<<<grid, LUT_THREADS, LUT_SMEM, s>>>(tenants, n_tenants, scale_dtype == BD_F16, seg, L.max_seg,
                                          x, y_part, L.ksplit, d_out, d_in, (int)batch, y,
                                          y_dtype == BD_BF16, status);
  launch_end(K_DELTA_LUT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd

extern "C" size_t bd_apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch,
                                          int32_t n_tenants) {
  return bd::apply_workspace_size(d_out, d_in, batch, n_tenants);
}

extern "C" bd_status bd_apply_multi(const void* w_base, int32_t w_dtype, int64_t d_out,
                                    int64_t d_in, const bd_tenant* tenants, int32_t n_tenants,
                                    int32_t scale_dtype, const int32_t* tenant_ids, const void* x,
                                    int64_t batch, void* y, int32_t y_dtype, void* workspace,
                                    size_t ws_bytes, void* stream) {
  return bd::apply_impl(w_base, w_dtype, d_out, d_in, tenants, n_tenants, scale_dtype, tenant_ids,
                        x, batch, y, y_dtype, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}
