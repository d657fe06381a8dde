// bd_prepare_tenant: rewrite a tenant's sign words (and group-128 scales) into the tiled
// serving layout read by the apply kernel: tiles of 512 rows x 256 columns, each tile one
// contiguous block, so a stage of the apply kernel is one 16 KB (signs) + 2-4 KB (scales)
// copy instead of 512 scattered row pieces. A pure permutation of the stored values.
#include "bd_internal.cuh"

namespace bd {

constexpr int64_t kTileRows = 512;
constexpr int64_t kTileCols = 256;

__host__ __device__ inline int64_t n_row_tiles(int64_t d_out) { return (d_out + kTileRows - 1) / kTileRows; }
__host__ __device__ inline int64_t n_col_tiles(int64_t d_in) { return (d_in + kTileCols - 1) / kTileCols; }

size_t prepared_signs_bytes(int64_t d_out, int64_t d_in) {
  return (size_t)(n_row_tiles(d_out) * n_col_tiles(d_in) * 4096 * 4);
}

static size_t plain_scale_elems(int64_t d_out, int64_t d_in, int32_t mode, int32_t G) {
  return (size_t)scale_count(mode, G, d_out, d_in);
}

size_t prepared_scales_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t G, int32_t sdt) {
  const size_t ssz = sdt == BD_F16 ? 2 : 4;
  if (mode == BD_SCALE_GROUP && G == 128)
    return (size_t)(n_row_tiles(d_out) * n_col_tiles(d_in) * 1024) * ssz;
  return align_up(plain_scale_elems(d_out, d_in, mode, G) * ssz, 16);
}

__global__ void k_prepare_signs(const uint32_t* __restrict__ signs, int64_t d_out, int64_t d_in,
                                uint32_t* __restrict__ out, int64_t total) {
  const int64_t wpr = d_in >> 5, nwin = n_col_tiles(d_in);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = i >> 12;
    const int within = (int)(i & 4095);
    const int64_t rb = tile / nwin, win = tile - rb * nwin;
    const int64_t row = rb * kTileRows + (within >> 3);
    const int64_t word = win * 8 + (within & 7);
    out[i] = (row < d_out && word < wpr) ? signs[row * wpr + word] : 0u;
  }
}

template <typename S>
__global__ void k_prepare_scales128(const S* __restrict__ sc, int64_t d_out, int64_t d_in,
                                    S* __restrict__ out, int64_t total) {
  const int64_t gpr = d_in / 128, nwin = n_col_tiles(d_in);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = i >> 10;
    const int within = (int)(i & 1023);
    const int64_t rb = tile / nwin, win = tile - rb * nwin;
    const int64_t row = rb * kTileRows + (within >> 1);
    const int64_t g = win * 2 + (within & 1);
    out[i] = (row < d_out && g < gpr) ? sc[row * gpr + g] : S(0);
  }
}

}  // namespace bd

extern "C" size_t bd_prepared_signs_bytes(int64_t d_out, int64_t d_in) {
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return 0;
  return bd::prepared_signs_bytes(d_out, d_in);
}

extern "C" size_t bd_prepared_scales_bytes(int64_t d_out, int64_t d_in, int32_t mode,
                                           int32_t group_size, int32_t scale_dtype) {
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return 0;
  if (!bd::scale_mode_ok(mode, group_size, d_in)) return 0;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return 0;
  return bd::prepared_scales_bytes(d_out, d_in, mode, group_size, scale_dtype);
}

extern "C" bd_status bd_prepare_tenant(const uint32_t* signs, const void* scales,
                                       int32_t scale_dtype, int32_t mode, int32_t group_size,
                                       int64_t d_out, int64_t d_in, uint32_t* signs_out,
                                       void* scales_out, void* stream) {
  using namespace bd;
  if (!signs || !scales || !signs_out || !scales_out) return BD_ERR_NULL;
  if (d_out < 1 || d_in < 32 || (d_in % 32) != 0) return BD_ERR_SHAPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if (!scale_mode_ok(mode, group_size, d_in)) return BD_ERR_CONFIG;
  if (!aligned16(signs) || !aligned16(scales) || !aligned16(signs_out) || !aligned16(scales_out))
    return BD_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t words = (int64_t)(prepared_signs_bytes(d_out, d_in) / 4);
  const int cap = sm_count() * 8;
  int64_t blocks = (words + 255) / 256;
  if (blocks > cap) blocks = cap;
  launch_begin(K_PREPARE, s);
  k_prepare_signs<<<(unsigned)blocks, 256, 0, s>>>(signs, d_out, d_in, signs_out, words);
  launch_end(K_PREPARE, s);
  BD_LAUNCH_CHECK();
  if (mode == BD_SCALE_GROUP && group_size == 128) {
    const int64_t n = n_row_tiles(d_out) * n_col_tiles(d_in) * 1024;
    int64_t b2 = (n + 255) / 256;
    if (b2 > cap) b2 = cap;
    launch_begin(K_PREPARE, s);
    if (scale_dtype == BD_F16)
      k_prepare_scales128<__half><<<(unsigned)b2, 256, 0, s>>>(
          static_cast<const __half*>(scales), d_out, d_in, static_cast<__half*>(scales_out), n);
    else
      k_prepare_scales128<float><<<(unsigned)b2, 256, 0, s>>>(
          static_cast<const float*>(scales), d_out, d_in, static_cast<float*>(scales_out), n);
    launch_end(K_PREPARE, s);
    BD_LAUNCH_CHECK();
  } else {
    const size_t bytes = plain_scale_elems(d_out, d_in, mode, group_size) * (scale_dtype == BD_F16 ? 2 : 4);
    BD_CUDA_TRY(cudaMemcpyAsync(scales_out, scales, bytes, cudaMemcpyDeviceToDevice, s));
  }
  return BD_OK;
}
