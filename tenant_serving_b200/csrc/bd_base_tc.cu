// Base product Y_base = X W_base^T on the 5th-generation tensor cores.
//
// "BitDelta Guide", "Systems Mechanics: 1. Decoupled Forward Pass": the shared base is
// applied once to the whole batch. One CTA owns a 128-row block of W_base and an
// N-column block of tokens (N = the batch rounded up to 16, at most 256) and a range of
// K. Warp 0 issues TMA tile loads of W_base [128 x 64] and X [N x 64] (128-byte
// swizzle) into a ring of shared-memory stages; warp 1 issues tcgen05.mma (M=128, N,
// K=16, bf16 in, fp32 accumulate in tensor memory) and releases each stage with
// tcgen05.commit; then all four warps read the accumulator with tcgen05.ld (one TMEM
// lane = one output row) and store fp32 partial sums y_part[kz][token][row].
// K is split across CTAs when the row blocks alone would leave SMs idle; the partial
// sums are added in a fixed order by the consumer.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

namespace bd {

constexpr int TC_BM = 128;   // rows per CTA (MMA M)
constexpr int TC_BK = 64;    // K per stage: 64 bf16 = one 128-byte swizzle row

__global__ void __launch_bounds__(128, 1) k_base_tc(const __grid_constant__ CUtensorMap tm_w,
                                                    const __grid_constant__ CUtensorMap tm_x,
                                                    int64_t d_out, int batch, int n_tile,
                                                    int stages, int kblocks, int kb_per_split,
                                                    float* __restrict__ y_part,
                                                    uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t a_bytes = TC_BM * TC_BK * 2;    // 16 KB
  const uint32_t b_bytes = (uint32_t)n_tile * TC_BK * 2;
  uint8_t* sa = smem;
  uint8_t* sb = smem + (size_t)stages * a_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + (size_t)stages * b_bytes);
  uint64_t* empty = full + stages;
  uint64_t* done = empty + stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued_out = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the N blocks of one row block are neighbours in launch order, so they stream the same
  // W_base tiles at about the same time and all but the first read them from L2
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
        tma_load_2d(sa + (size_t)s * a_bytes, &tm_w, &full[s], (kb0 + i) * TC_BK, m_blk * TC_BM);
        tma_load_2d(sb + (size_t)s * b_bytes, &tm_x, &full[s], (kb0 + i) * TC_BK, n_blk * n_tile);
        ++issued;
      }
      *issued_out = issued;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(TC_BM, n_tile, true);
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
        for (int k = 0; k < TC_BK / 16; ++k) {
          // advance 16 elements (32 bytes) along K inside the swizzled 128-byte row
          umma_f16(tmem_d, ad + (uint64_t)(2 * k), bdsc + (uint64_t)(2 * k), idesc,
                   (i > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(done);  // fires when every MMA issued above has completed
    }
    __syncwarp();
  }

  // epilogue: thread (warp w, lane l) owns accumulator lane 32w + l = output row
  const bool ok = mbar_wait(done, 0, nullptr);
  tc_fence_after();
  if (!ok) timed_out = true;
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (ok && !aborted) {
    const int64_t row = (int64_t)m_blk * TC_BM + warp * 32 + lane;
    const uint32_t lane_addr = tmem_d + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < n_tile; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(lane_addr + (uint32_t)c0, r);
      if (row < d_out) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = n_blk * n_tile + c0 + j;
          if (c0 + j < n_tile && t < batch)
            y_part[((int64_t)kz * batch + t) * d_out + row] = __uint_as_float(r[j]);
        }
      }
    }
  }
  if (timed_out || aborted) {
    if (threadIdx.x == 0) atomicOr(status, BD_DEV_TIMEOUT);
    // let every TMA load this CTA issued land before its shared memory goes away
    if (threadIdx.x == 0) {
      const int issued = *issued_out;
      for (int i = 0; i < issued; ++i) {
        const int s = i % stages;
        const uint32_t ph = (uint32_t)(i / stages) & 1u;
        // a completed phase of parity ph means load i landed; bounded either way
        mbar_wait(&full[s], ph, nullptr);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_d, tcols);
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
// bf16 row-major [rows][cols] tensor, box [box_rows][64 cols], 128-byte swizzle
static bool encode_bf16_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                           int box_rows) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)TC_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

TcPlan plan_base_tc(int64_t d_out, int64_t d_in, int64_t batch) {
  TcPlan p;
  p.tiles_n = (int)((batch + 255) / 256);
  int per = (int)((batch + p.tiles_n - 1) / p.tiles_n);
  p.n_tile = ((per + 15) / 16) * 16;
  p.tiles_m = (int)((d_out + TC_BM - 1) / TC_BM);
  p.kblocks = (int)((d_in + TC_BK - 1) / TC_BK);
  // K splits: one CTA per SM at a time, so the time goes as the number of waves times the
  // K blocks of a CTA. Each extra split also writes and re-reads batch x d_out fp32
  // partial sums; that traffic (at ~5 TB/s) is charged in units of one K block's MMA
  // time (4 MMAs of N/2 cycles, at least ~46 cycles each, at ~1.9 GHz). At least 4 K
  // blocks per CTA.
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
  const size_t stage_bytes = (size_t)TC_BM * TC_BK * 2 + (size_t)p.n_tile * TC_BK * 2;
  int st = (int)((200 * 1024) / stage_bytes);
  if (st > 8) st = 8;
  if (st < 2) st = 2;
  p.stages = st;
  p.smem = 1024 + (size_t)st * stage_bytes + (2 * st + 1) * 8 + 16;
  return p;
}

bd_status launch_base_tc(const TcPlan& p, const void* w_base, const void* x, int64_t d_out,
                         int64_t d_in, int64_t batch, float* y_part, uint32_t* status,
                         cudaStream_t s) {
  CUtensorMap tw, tx;
  if (!encode_bf16_2d(&tw, w_base, d_out, d_in, TC_BM)) return BD_ERR_CUDA;
  if (!encode_bf16_2d(&tx, x, batch, d_in, p.n_tile)) return BD_ERR_CUDA;
  static std::atomic<uint64_t> attr_set{0};
  if (!ensure_dyn_smem(k_base_tc, 227 * 1024, attr_set)) return BD_ERR_CUDA;

  if (p.tiles_m > 65535) return BD_ERR_SHAPE;  // row blocks run along grid y
  dim3 grid(p.tiles_n, p.tiles_m, p.ksplit);
  launch_begin(K_BASE_TC, s);
  BD_CUDA_TRY(launch_pdl(k_base_tc, grid, dim3(128), p.smem, s, tw, tx, d_out, (int)batch, p.n_tile, p.stages,
                         p.kblocks, p.kb_per_split, y_part, status));
  launch_end(K_BASE_TC, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd
