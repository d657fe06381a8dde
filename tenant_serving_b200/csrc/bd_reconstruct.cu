// bd_reconstruct: Delta_hat = sign * scale ("bitdelta" page, "4. Reconstruction") and,
// with W_base given, the personalised weight W_base + Delta_hat ("5. Serving").
// Write-bound stream: one thread expands one byte of sign bits (8 columns) and stores
// 16 (bf16) or 32 (fp32) bytes.
#include "bd_internal.cuh"

namespace bd {

__device__ __forceinline__ float load_scale(const void* sc, bool f16, int64_t idx) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(sc)[idx])
             : reinterpret_cast<const float*>(sc)[idx];
}

__global__ void __launch_bounds__(256) k_reconstruct(
    const uint8_t* __restrict__ signs, const void* __restrict__ scales, bool scale_f16, int mode,
    int group, int64_t d_out, int64_t d_in, const void* __restrict__ w_base, bool w_bf16,
    void* __restrict__ out, bool out_bf16) {
  const int64_t nbytes = d_out * (d_in >> 3);
  const int64_t bytes_per_row = d_in >> 3;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbytes;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / bytes_per_row;
    const int64_t col = (i - row * bytes_per_row) * 8;
    const uint32_t bits = signs[i];  // byte i = columns 8*(i%bpr) .. +7, LSB first
    float s[8];
    if (mode == BD_SCALE_COL) {
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = load_scale(scales, scale_f16, col + k);
    } else {
      int64_t idx = 0;
      if (mode == BD_SCALE_GROUP) idx = row * (d_in / group) + col / group;
      else if (mode == BD_SCALE_BLOCK) idx = (row / group) * (d_in / group) + col / group;
      else if (mode == BD_SCALE_ROW) idx = row;
      const float sv = load_scale(scales, scale_f16, idx);
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = sv;
    }
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = ((bits >> k) & 1u) ? s[k] : -s[k];
    const int64_t e0 = row * d_in + col;
    if (w_base) {
      if (w_bf16) {
        const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(w_base) + e0);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[2 * k] += bf16lo(ww[k]);
          v[2 * k + 1] += bf16hi(ww[k]);
        }
      } else {
        const float4* wp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(w_base) + e0);
        const float4 a = wp[0], b = wp[1];
        v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
        v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
      }
    }
    if (out_bf16) {
      uint4 o;
      o.x = f2bf_bits(v[0]) | (f2bf_bits(v[1]) << 16);
      o.y = f2bf_bits(v[2]) | (f2bf_bits(v[3]) << 16);
      o.z = f2bf_bits(v[4]) | (f2bf_bits(v[5]) << 16);
      o.w = f2bf_bits(v[6]) | (f2bf_bits(v[7]) << 16);
      *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + e0) = o;
    } else {
      float4* op = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e0);
      op[0] = make_float4(v[0], v[1], v[2], v[3]);
      op[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

}  // namespace bd

extern "C" bd_status bd_reconstruct(const uint32_t* signs, const void* scales, int32_t scale_dtype,
                                    int32_t mode, int32_t group_size, int64_t d_out, int64_t d_in,
                                    const void* w_base, int32_t w_dtype, void* out,
                                    int32_t out_dtype, void* stream) {
  using namespace bd;
  if (!signs || !scales || !out) return BD_ERR_NULL;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (scale_dtype != BD_F32 && scale_dtype != BD_F16) return BD_ERR_DTYPE;
  if (out_dtype != BD_F32 && out_dtype != BD_BF16) return BD_ERR_DTYPE;
  if (w_base && w_dtype != BD_F32 && w_dtype != BD_BF16) return BD_ERR_DTYPE;
  if (!scale_mode_ok(mode, group_size, d_in)) return BD_ERR_CONFIG;
  if (!aligned16(signs) || !aligned16(scales) || !aligned16(out) || (w_base && !aligned16(w_base)))
    return BD_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nbytes = d_out * (d_in >> 3);
  int64_t blocks = (nbytes + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 16;
  if (blocks > cap) blocks = cap;
  launch_begin(K_RECONSTRUCT, s);
  k_reconstruct<<<(unsigned)blocks, 256, 0, s>>>(
      reinterpret_cast<const uint8_t*>(signs), scales, scale_dtype == BD_F16, mode, group_size,
      d_out, d_in, w_base, w_dtype == BD_BF16, out, out_dtype == BD_BF16);
  launch_end(K_RECONSTRUCT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}
