// E4M3 base weights with per-row scales under the delta path: quantization of a base
// matrix, the activations as two e4m3 limbs, and the base product on the tensor cores
// (tcgen05.mma kind::f8f6f4).
//
// "BitDelta Guide", "3. Quantized Base Model Compatibility (BitDelta + GPTQ / QuIP#)": the
// 1-bit delta is applied on top of quantized base weights; "Per-Axis Weight Deltas for
// Frequent Model Updates", Future Directions: FP8 co-design. The base is stored as e4m3
// codes q[o][i] and one fp32 scale s_o per output row, W_hat = s_o * q, half the bytes of
// a bf16 base.
//
// The tensor cores take both operands of a kind::f8f6f4 product in an 8-bit format, so
// every activation row x_t (bf16) is first written as x_t = 2^e_t (hi + lo), hi and lo
// e4m3 and 2^e_t a power of two that brings max|x_t| into [128, 256): hi is x_t / 2^e_t
// rounded to e4m3, lo the e4m3 rounding of the (exact) remainder. Four significant bits
// each cover the eight of a bf16 value, so the pair is exact except where the remainder
// falls below e4m3's subnormal range (|x| < 2^-9 * 2^e_t, i.e. below ~max|x_t| / 2^16),
// whose error is bounded by 2^-10 * 2^e_t. The product runs over 2B token columns (hi and
// lo side by side) with fp32 accumulation in tensor memory; the epilogue adds the two
// columns of a token and applies s_o * 2^e_t.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

#include <cuda_fp8.h>

namespace bd {

constexpr float kE4M3Max = 448.f;
constexpr int F8_BM = 128;  // rows per CTA (MMA M)
constexpr int F8_BK = 128;  // K per stage: 128 e4m3 = one 128-byte swizzle row

__device__ __forceinline__ uint32_t e4m3_code(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}

// 8 consecutive values of a row (d_in % 32 == 0, so 8 never straddle the end)
template <bool BF16>
__device__ __forceinline__ void load8(const void* row, int64_t k, float* v) {
  if (BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(row) + k);
    const uint32_t a[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = bf16lo(a[j]);
      v[2 * j + 1] = bf16hi(a[j]);
    }
  } else {
    const float4 p = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row) + k);
    const float4 q = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row) + k + 4);
    v[0] = p.x; v[1] = p.y; v[2] = p.z; v[3] = p.w;
    v[4] = q.x; v[5] = q.y; v[6] = q.z; v[7] = q.w;
  }
}

__device__ __forceinline__ float block_max(float m, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = m;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint2 pack8(const uint32_t* c) {
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// ------------------------------------------------------------------------------------
// per-row quantization: s_o = max_i |W[o,i]| / 448 and q = e4m3(W / s_o), both quotients
// IEEE fp32 divisions, rounding to nearest even with saturation at 448; a zero row has
// scale 0 and codes 0
// ------------------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) k_quantize_fp8(const void* __restrict__ w, int64_t d_out, int64_t d_in,
                                                      uint8_t* __restrict__ codes, float* __restrict__ scales) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  __shared__ float red[8];
  for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
    const uint8_t* wr = reinterpret_cast<const uint8_t*>(w) + row * d_in * (BF16 ? 2 : 4);
    float m = 0.f;
    for (int64_t k = (int64_t)threadIdx.x * 8; k < d_in; k += 256 * 8) {
      float v[8];
      load8<BF16>(wr, k, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    m = block_max(m, red);
    const float s = m / kE4M3Max;
    if (threadIdx.x == 0) scales[row] = s;
    for (int64_t k = (int64_t)threadIdx.x * 8; k < d_in; k += 256 * 8) {
      float v[8];
      load8<BF16>(wr, k, v);
      uint32_t c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) c[j] = s > 0.f ? e4m3_code(v[j] / s) : 0u;
      *reinterpret_cast<uint2*>(codes + row * d_in + k) = pack8(c);
    }
  }
}

// ------------------------------------------------------------------------------------
// activations -> limbs. Token t of the batch sits in N tile j = t / h at column
// c = t % h of that tile's tokens; in the tile's operand rows, 16-token group g = c / 16
// has its hi limbs at rows 32 g + (c % 16) and its lo limbs 16 rows further, so one
// 32-column read of the accumulator holds both columns of 16 tokens. Padding tokens
// (t >= batch) get zero rows.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_x_limbs(const uint16_t* __restrict__ x, int64_t d_in, int batch, int h,
                                                 int n_tile, uint8_t* __restrict__ x8, float* __restrict__ xmul) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  __shared__ float red[4];
  const int t = blockIdx.x;
  const int j = t / h, c = t % h;
  uint8_t* hi = x8 + ((int64_t)j * n_tile + 32 * (c / 16) + (c % 16)) * d_in;
  uint8_t* lo = hi + 16 * d_in;
  if (t >= batch) {
    for (int64_t k = (int64_t)threadIdx.x * 8; k < d_in; k += 128 * 8) {
      *reinterpret_cast<uint2*>(hi + k) = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(lo + k) = make_uint2(0u, 0u);
    }
    if (threadIdx.x == 0) xmul[t] = 0.f;
    return;
  }
  const uint16_t* xr = x + (int64_t)t * d_in;
  float m = 0.f;
  for (int64_t k = (int64_t)threadIdx.x * 8; k < d_in; k += 128 * 8) {
    float v[8];
    load8<true>(xr, k, v);
#pragma unroll
    for (int q = 0; q < 8; ++q) m = fmaxf(m, fabsf(v[q]));
  }
  m = block_max(m, red);
  // e = floor(log2 m) - 7, so that m / 2^e lies in [128, 256); kept in [-120, 120]
  int e = 0;
  if (m > 0.f) {
    e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127 - 7;
    e = e < -120 ? -120 : (e > 120 ? 120 : e);
  }
  const float down = __uint_as_float((uint32_t)(127 - e) << 23);
  if (threadIdx.x == 0) xmul[t] = __uint_as_float((uint32_t)(127 + e) << 23);
  for (int64_t k = (int64_t)threadIdx.x * 8; k < d_in; k += 128 * 8) {
    float v[8];
    load8<true>(xr, k, v);
    uint32_t ch[8], cl[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float a = v[q] * down;  // exact: a power of two
      ch[q] = e4m3_code(a);
      cl[q] = e4m3_code(a - e4m3_to_float(ch[q]));  // the remainder is exact in fp32
    }
    *reinterpret_cast<uint2*>(hi + k) = pack8(ch);
    *reinterpret_cast<uint2*>(lo + k) = pack8(cl);
  }
}

// ------------------------------------------------------------------------------------
// base product: one CTA per (N tile, 128-row block, K range). Warp 0 issues TMA loads of
// the codes [128 x 128] and the limb rows [n_tile x 128] (128-byte swizzle), warp 1 the
// MMAs (M=128, N=n_tile, K=32, e4m3 x e4m3, fp32 in tensor memory); the epilogue writes
// y_part[kz][t][row] = s_row * 2^e_t * (acc_hi + acc_lo).
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1) k_base_fp8(const __grid_constant__ CUtensorMap tm_w,
                                                     const __grid_constant__ CUtensorMap tm_x,
                                                     const float* __restrict__ w_scales,
                                                     const float* __restrict__ xmul, int64_t d_out, int batch,
                                                     int h, int n_tile, int stages, int kblocks, int kb_per_split,
                                                     float* __restrict__ y_part, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t a_bytes = F8_BM * F8_BK;  // 16 KB
  const uint32_t b_bytes = (uint32_t)n_tile * F8_BK;
  uint8_t* sa = smem;
  uint8_t* sb = smem + (size_t)stages * a_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + (size_t)stages * b_bytes);
  uint64_t* empty = full + stages;
  uint64_t* done = empty + stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued_out = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_blk = blockIdx.x, m_blk = blockIdx.y, kz = blockIdx.z;
  const int kb0 = kz * kb_per_split;
  const int kb1 = min(kblocks, kb0 + kb_per_split);
  const int nkb = kb1 - kb0;  // >= 1 by construction on the host
  uint32_t tcols = 32;
  while (tcols < (uint32_t)n_tile) tcols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *issued_out = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) tmem_alloc(tmem_slot, tcols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_wait();  // the set-up above overlaps the previous kernel on the stream
  pdl_trigger();

  bool timed_out = false;
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        if (i >= stages && !mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          timed_out = true;
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
        tma_load_2d(sa + (size_t)s * a_bytes, &tm_w, &full[s], (kb0 + i) * F8_BK, m_blk * F8_BM);
        tma_load_2d(sb + (size_t)s * b_bytes, &tm_x, &full[s], (kb0 + i) * F8_BK, n_blk * n_tile);
        ++issued;
      }
      *issued_out = issued;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_e4m3(F8_BM, n_tile);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          timed_out = true;
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad = umma_desc_sw128(smem_u32(sa + (size_t)s * a_bytes));
        const uint64_t bdsc = umma_desc_sw128(smem_u32(sb + (size_t)s * b_bytes));
#pragma unroll
        for (int k = 0; k < F8_BK / 32; ++k) {
          // advance 32 elements (32 bytes) along K inside the swizzled 128-byte row
          umma_f8(tmem_d, ad + (uint64_t)(2 * k), bdsc + (uint64_t)(2 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(done);
    }
    __syncwarp();
  }

  const bool ok = mbar_wait(done, 0, nullptr);
  tc_fence_after();
  if (!ok) timed_out = true;
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (ok && !aborted) {
    const int64_t row = (int64_t)m_blk * F8_BM + warp * 32 + lane;
    const float s_row = row < d_out ? w_scales[row] : 0.f;
    const uint32_t lane_addr = tmem_d + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < n_tile; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(lane_addr + (uint32_t)c0, r);
      if (row < d_out) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int t = n_blk * h + c0 / 2 + jj;
          if (t < batch) {
            const float v = __uint_as_float(r[jj]) + __uint_as_float(r[16 + jj]);
            y_part[((int64_t)kz * batch + t) * d_out + row] = s_row * xmul[t] * v;
          }
        }
      }
    }
  }
  if (timed_out || aborted) {
    if (threadIdx.x == 0) {
      atomicOr(status, BD_DEV_TIMEOUT);
      // every TMA load this CTA issued lands before its shared memory goes away
      const int issued = *issued_out;
      for (int i = 0; i < issued; ++i) mbar_wait(&full[i % stages], (uint32_t)(i / stages) & 1u, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_d, tcols);
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
static bool encode_u8_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)F8_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

Fp8Plan plan_base_fp8(int64_t d_out, int64_t d_in, int64_t batch) {
  Fp8Plan p;
  p.tiles_n = (int)((batch + 127) / 128);
  const int per = (int)((batch + p.tiles_n - 1) / p.tiles_n);
  p.h = ((per + 15) / 16) * 16;
  p.n_tile = 2 * p.h;
  p.tiles_m = (int)((d_out + F8_BM - 1) / F8_BM);
  p.kblocks = (int)((d_in + F8_BK - 1) / F8_BK);
  // K splits as for the bf16 product: waves of one CTA per SM times the K blocks of a
  // CTA, each split charged the write and re-read of its fp32 partial sums
  const int sms = sm_count();
  const int base_ctas = p.tiles_m * p.tiles_n;
  const double kb_seconds = 4.0 * (p.n_tile / 2 > 46 ? p.n_tile / 2 : 46) / 1.9e9;
  const double split_units = 8.0 * (double)batch * (double)d_out / 5e12 / kb_seconds;
  int best_kb = p.kblocks;
  double best_cost = 1e30;
  for (int k = 1; k <= 16; ++k) {
    const int kb_per = (p.kblocks + k - 1) / k;
    if (k > 1 && kb_per < 4) break;
    const int splits = (p.kblocks + kb_per - 1) / kb_per;
    const int64_t waves = ((int64_t)base_ctas * splits + sms - 1) / sms;
    const double cost = (double)waves * kb_per + (splits - 1) * split_units;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_kb = kb_per;
    }
  }
  p.kb_per_split = best_kb;
  p.ksplit = (p.kblocks + best_kb - 1) / best_kb;
  const size_t stage_bytes = (size_t)F8_BM * F8_BK + (size_t)p.n_tile * F8_BK;
  int st = (int)((200 * 1024) / stage_bytes);
  if (st > 8) st = 8;
  if (st < 2) st = 2;
  p.stages = st;
  p.smem = 1024 + (size_t)st * stage_bytes + (2 * st + 1) * 8 + 16;
  p.x8_bytes = (size_t)p.tiles_n * p.n_tile * d_in;
  p.xmul_count = p.tiles_n * p.h;
  return p;
}

bd_status launch_base_fp8(const Fp8Plan& p, const uint8_t* codes, const float* w_scales, const void* x,
                          int64_t d_out, int64_t d_in, int64_t batch, uint8_t* x8, float* xmul, float* y_part,
                          uint32_t* status, cudaStream_t s) {
  launch_begin(K_X_LIMBS, s);
  BD_CUDA_TRY(launch_pdl(k_x_limbs, dim3((unsigned)(p.tiles_n * p.h)), dim3(128), 0, s,
                         static_cast<const uint16_t*>(x), d_in, (int)batch, p.h, p.n_tile, x8, xmul));
  launch_end(K_X_LIMBS, s);
  BD_LAUNCH_CHECK();
  CUtensorMap tw, tx;
  if (!encode_u8_2d(&tw, codes, d_out, d_in, F8_BM)) return BD_ERR_CUDA;
  if (!encode_u8_2d(&tx, x8, (int64_t)p.tiles_n * p.n_tile, d_in, p.n_tile)) return BD_ERR_CUDA;
  static std::atomic<uint64_t> attr_set{0};
  if (!ensure_dyn_smem(k_base_fp8, 227 * 1024, attr_set)) return BD_ERR_CUDA;
  if (p.tiles_m > 65535) return BD_ERR_SHAPE;
  dim3 grid(p.tiles_n, p.tiles_m, p.ksplit);
  launch_begin(K_BASE_FP8, s);
  BD_CUDA_TRY(launch_pdl(k_base_fp8, grid, dim3(128), p.smem, s, tw, tx, w_scales, (const float*)xmul, d_out,
                         (int)batch, p.h, p.n_tile, p.stages, p.kblocks, p.kb_per_split, y_part, status));
  launch_end(K_BASE_FP8, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd

extern "C" bd_status bd_quantize_base_fp8(const void* w, int32_t w_dtype, int64_t d_out, int64_t d_in,
                                          uint8_t* codes, float* scales, void* stream) {
  using namespace bd;
  if (!w || !codes || !scales) return BD_ERR_NULL;
  if (w_dtype != BD_BF16 && w_dtype != BD_F32) return BD_ERR_DTYPE;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return BD_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int64_t blocks = d_out;
  const int cap = sm_count() * 8;
  if (blocks > cap) blocks = cap;
  launch_begin(K_QUANT_FP8, s);
  if (w_dtype == BD_BF16)
    BD_CUDA_TRY(launch_pdl(k_quantize_fp8<true>, dim3((unsigned)blocks), dim3(256), 0, s, w, d_out, d_in, codes,
                           scales));
  else
    BD_CUDA_TRY(launch_pdl(k_quantize_fp8<false>, dim3((unsigned)blocks), dim3(256), 0, s, w, d_out, d_in, codes,
                           scales));
  launch_end(K_QUANT_FP8, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}
