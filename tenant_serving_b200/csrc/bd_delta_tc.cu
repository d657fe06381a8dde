// Tensor-core delta product for tenants with several tokens in the batch.
//
// "BitDelta Guide", "Systems Mechanics: 2. Fused Dequantization": the sign bits stay
// packed in HBM and are expanded on chip. For a tenant u with n_u tokens the delta is a
// dense contraction  D[128 rows x N] = A_u[128 x K] * X_u^T, A_u = +/-s (the scale of
// the row's group, or of the row, or the tensor), X_u = the tenant's tokens. Here:
//   - a loader warp streams the tenant's sign words (and group-128 scales) in 256-column
//     windows of the tiled serving layout (one 4 KB bulk copy per 128 rows) into a
//     shared-memory ring, and the tokens X_u by TMA;
//   - eight warps expand A (one thread per row and per half of a 64-column stage) in
//     registers as fp16 +/-s, exact because the scales are fp16, and store it straight
//     into tensor memory with tcgen05.st: A never touches shared memory. Column 32b + q of
//     a sign word goes to K position 32b + 2q and column 32b + q + 16 to 32b + 2q + 1, so
//     each 32-bit register of two halves is one shift and one LOP3 of the word;
//   - X is gathered once per call in the same column order (k_tc_gather) as fp16 of
//     x * 2^e_t, with 2^e_t per token chosen so the largest |x| stays below 2^15: bf16
//     values are then exact in fp16 (tiny ones lose only sub-2^-24 bits). For a tenant
//     with column scales the gather multiplies each x_i by s_i first (A is then +/-1):
//     Delta_hat x = sign . (s * x); the fp16 rounding of s_i x_i is the one inexact step
//     (relative 2^-11 per product);
//   - one thread issues tcgen05.mma with A from tensor memory and B from shared memory
//     (M=128, N = n_u rounded to 16, K=16, fp32 accumulation in tensor memory); four
//     more warps read the accumulator, multiply by 2^-e_t (exact), add the base product
//     and write y. The accumulator is double buffered so that this epilogue overlaps
//     the next tile's MMAs.
// Tenants qualify when they are stored in the tiled serving layout, their scales are
// fp16 and in GROUP or BLOCK (group >= 64), ROW, COL or TENSOR mode, and d_in % 64 == 0;
// the planner sends the rest to the lookup-table kernel.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

namespace bd {

constexpr int DT_BM = 128;            // rows per work item
constexpr int DT_BK = 64;             // K per stage (64 fp16 = one 128-byte swizzle row)
constexpr int DT_KPW = 4;             // stages per 256-column window
constexpr int DT_NMAX = kTcSegTokens;  // tokens per segment
constexpr int DT_AW = 2;              // A ring depth in windows (tensor memory)
constexpr int DT_XW_MAX = 8;          // X ring depth in windows (shared memory), fewer for wide segments
constexpr int DT_WSLOTS = 16;         // sign-window ring depth (64 KB of signs in flight)
constexpr int DT_WDONE = 8;           // "window's MMAs done" barriers (>= A and X ring depths)
// a window waits on wdone of window w - ring depth; the slot may not be reused by a later
// window before that wait, which holds while both ring depths are <= DT_WDONE
static_assert(DT_XW_MAX <= DT_WDONE && DT_AW <= DT_WDONE, "window-done ring too short");
constexpr int DT_THREADS = 15 * 32;   // 0-7 expand A, 8-11 epilogue, 12 MMA, 13 X loader, 14 sign loader
constexpr uint32_t DT_TMEM_COLS = 512;  // [0,256): two accumulators, [256,512): A ring (2 windows)
constexpr uint32_t DT_ACC_STRIDE = 128;
constexpr uint32_t DT_A_COL0 = 256;
constexpr uint32_t DT_WIN_SIGN_BYTES = 4096;  // 128 rows x 8 words
constexpr uint32_t DT_WIN_SCALE_BYTES = 512;  // 128 rows x 2 fp16 (tiled group-128 scales)

// ------------------------------------------------------------------------------------
// gather: X_u rows for every tensor-core segment, permuted and scaled into fp16 range
// ------------------------------------------------------------------------------------
// seg arrays: tc_tenant, tc_start, tc_count, tc_xrow (Xg row of the segment's first token).
// One CTA of DT_GATHER_THREADS per Xg row (blockIdx.x: the row within its segment,
// blockIdx.y: the segment): every thread takes 32-column blocks tid, tid + 128, ... of
// the token, so the row's largest |value| is one pass of short per-thread loops and a CTA
// reduction; the second pass re-reads the row (from L1 / L2) to scale and write it.
constexpr int DT_GATHER_THREADS = 128;
__global__ void __launch_bounds__(DT_GATHER_THREADS) k_tc_gather(const int32_t* __restrict__ seg_base,
                                                                 int max_groups, int max_tc,
                                                                 const bd_tenant* __restrict__ tc_rec,
                                                                 const uint16_t* __restrict__ x, int64_t d_in,
                                                                 __half* __restrict__ xg, float* __restrict__ xinv) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  const int n_tc = seg_base[1];
  const int sidx = blockIdx.y;
  if (sidx >= n_tc) return;
  const int32_t* tc = seg_base + kSegHeader + 3 * max_groups;  // tc_tenant, then the arrays below
  const int32_t* tc_start = tc + max_tc;
  const int32_t* tc_count = tc_start + max_tc;
  const int32_t* tc_xrow = tc_count + max_tc;
  const int32_t* permv = tc_xrow + max_tc;
  const int count = tc_count[sidx];
  const int npad = (count + 15) & ~15;
  const int r = blockIdx.x;
  if (r >= npad) return;  // CTA-uniform
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t xr = tc_xrow[sidx] + r;
  __half* out = xg + xr * d_in;
  const int nblk = (int)(d_in >> 5);
  if (r >= count) {
    for (int b = tid; b < nblk; b += DT_GATHER_THREADS) {
      uint4* o = reinterpret_cast<uint4*>(out + 32 * b);
      o[0] = o[1] = o[2] = o[3] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) xinv[xr] = 0.f;
    return;
  }
  const int t = permv[tc_start[sidx] + r];
  const uint16_t* xt = x + (int64_t)t * d_in;
  // column scales of the segment's tenant (fp16), folded into its activations
  const bool col = tc_rec[sidx].mode == BD_SCALE_COL;
  const uint16_t* cs = static_cast<const uint16_t*>(tc_rec[sidx].scales);
  // 32 values of column block b: x, times the column scale for a COL tenant
  auto load32 = [&](int b, float* v) {
    const uint4* p = reinterpret_cast<const uint4*>(xt + 32 * b);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 w = p[k];
      const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * k + 2 * j] = bf16lo(a[j]);
        v[8 * k + 2 * j + 1] = bf16hi(a[j]);
      }
    }
    if (col) {
      const uint4* q = reinterpret_cast<const uint4*>(cs + 32 * b);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 w = q[k];
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = *reinterpret_cast<const __half2*>(&a[j]);
          v[8 * k + 2 * j] *= __low2float(h);
          v[8 * k + 2 * j + 1] *= __high2float(h);
        }
      }
    }
  };
  // largest |x| (|s x| for a COL tenant) of the token
  __shared__ float wmax[DT_GATHER_THREADS / 32];
  float m = 0.f;
#pragma unroll 2
  for (int b = tid; b < nblk; b += DT_GATHER_THREADS) {
    float v[32];
    load32(b, v);
#pragma unroll
    for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(v[k]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < DT_GATHER_THREADS / 32; ++w) m = fmaxf(m, wmax[w]);
  int e = 0;
  if (m > 0.f) {
    int E;
    frexpf(m, &E);   // m < 2^E
    e = 15 - E;      // m * 2^e < 2^15
    if (e > 126) e = 126;  // keep 2^e finite (tokens of only subnormal-sized values)
  }
  const float sc = ldexpf(1.f, e);
#pragma unroll 2
  for (int b = tid; b < nblk; b += DT_GATHER_THREADS) {
    float v[32];
    load32(b, v);
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] *= sc;
    // K position 2q <- column q, 2q + 1 <- column q + 16
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const __half2 h = __floats2half2_rn(v[q], v[q + 16]);
      o[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + 32 * b);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
    dst[3] = make_uint4(o[12], o[13], o[14], o[15]);
  }
  if (tid == 0) xinv[xr] = ldexpf(1.f, -e);
}

// ------------------------------------------------------------------------------------
// the tensor-core delta kernel
// ------------------------------------------------------------------------------------
// Persistent: work item = (segment, 128-row tile), items dealt round-robin to the CTAs.
// All rings run across items.

// 32 lanes x 16 consecutive 32-bit columns of tensor memory from 16 registers per thread.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns of tensor memory into 16 registers per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16; ACC = 0 overwrites D
template <int ACC>
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "n"(ACC)
      : "memory");
}

struct TcSegs {
  const int32_t *start, *count, *xrow, *perm;
};
__device__ __forceinline__ TcSegs tc_segs(const int32_t* seg_base, int max_groups, int max_tc) {
  TcSegs g;
  const int32_t* tenant = seg_base + kSegHeader + 3 * max_groups;
  g.start = tenant + max_tc;
  g.count = g.start + max_tc;
  g.xrow = g.count + max_tc;
  g.perm = g.xrow + max_tc;
  return g;
}

// ring position: slot and the parity of its current fill
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  int n = 0;  // fills so far
  __device__ __forceinline__ void next(int slots) {
    ++n;
    if (++slot == slots) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// what every role needs to know about a work item; all loads independent of one another,
// so the next item's are issued one item ahead
struct Item {
  bd_tenant T;
  int64_t row0;
  int start, count, xrow;
};
__device__ __forceinline__ Item load_item(const TcSegs& sg, const bd_tenant* __restrict__ tc_rec,
                                          int it, int mtiles) {
  Item m;
  const int sidx = it / mtiles;
  m.row0 = (int64_t)(it - sidx * mtiles) * DT_BM;
  const uint4* rp = reinterpret_cast<const uint4*>(tc_rec + sidx);
  const uint4 a = rp[0], b = rp[1];
  m.T.signs = reinterpret_cast<const uint32_t*>((uint64_t)a.x | ((uint64_t)a.y << 32));
  m.T.scales = reinterpret_cast<const void*>((uint64_t)a.z | ((uint64_t)a.w << 32));
  m.T.mode = (int32_t)b.x;
  m.T.group_size = (int32_t)b.y;
  m.T.layout = (int32_t)b.z;
  m.T.reserved = (int32_t)b.w;
  m.start = sg.start[sidx];
  m.count = sg.count[sidx];
  m.xrow = sg.xrow[sidx];
  return m;
}

__global__ void __launch_bounds__(DT_THREADS, 1) k_delta_tc(
    const __grid_constant__ CUtensorMap tm_x, const bd_tenant* __restrict__ tc_rec,
    const int32_t* __restrict__ seg_base, int max_groups, int max_tc,
    const float* __restrict__ xinv, const float* __restrict__ y_part, int ksplit, int64_t d_out,
    int64_t d_in, int batch, void* __restrict__ y, bool y_bf16, int nmax, int xwin,
    uint32_t* __restrict__ status) {
  pdl_wait();  // inputs may come from the previous kernel on the stream
  pdl_trigger();
  const int n_tc = seg_base[1];
  const int mtiles = (int)((d_out + DT_BM - 1) / DT_BM);
  const int items = n_tc * mtiles;
  if ((int)blockIdx.x >= items) return;  // whole CTA, before any barrier or TMEM use
  const int nloc = (items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const TcSegs sg = tc_segs(seg_base, max_groups, max_tc);
  const int nkb = (int)(d_in / DT_BK);
  const int nwin = (nkb + DT_KPW - 1) / DT_KPW;
  auto item_index = [&](int i) { return (int)blockIdx.x + i * (int)gridDim.x; };

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t b_bytes = (uint32_t)nmax * DT_BK * 2;  // one stage of X: nmax rows x 128 B
  const uint32_t xw_bytes = b_bytes * DT_KPW;            // one window of X
  uint8_t* sb = smem;
  uint8_t* sw = sb + (size_t)xwin * xw_bytes;
  uint8_t* ss = sw + (size_t)DT_WSLOTS * DT_WIN_SIGN_BYTES;
  // full_x: X window landed (TMA); full_a: the producers stored the window's A and saw its
  // X land (one barrier for the MMA issuer to wait on); wdone[w % DT_WDONE]: window w's
  // MMAs completed, which frees both its A slot and its X slot
  uint64_t* full_x = reinterpret_cast<uint64_t*>(ss + (size_t)DT_WSLOTS * DT_WIN_SCALE_BYTES);
  uint64_t* wdone = full_x + DT_XW_MAX;
  uint64_t* full_a = wdone + DT_WDONE;
  uint64_t* full_w = full_a + DT_AW;
  uint64_t* empty_w = full_w + DT_WSLOTS;
  uint64_t* acc_full = empty_w + DT_WSLOTS;  // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < xwin; ++i) mbar_init(&full_x[i], 1);
    for (int i = 0; i < DT_WDONE; ++i) mbar_init(&wdone[i], 1);
    for (int i = 0; i < DT_AW; ++i) mbar_init(&full_a[i], 256);
    for (int i = 0; i < DT_WSLOTS; ++i) {
      mbar_init(&full_w[i], 1);
      mbar_init(&empty_w[i], 256);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 12) tmem_alloc(tmem_slot, DT_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 8) {
    // ---------------- A producers: thread = (row, half of each stage) ----------------
    const int q4 = warp & 3, h = warp >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t a_lane = tmem_base + ((uint32_t)(q4 * 32) << 16) + DT_A_COL0 + (uint32_t)(16 * h);
    Ring A, W, X;  // A: window count and A slot; X: the window's X slot
    bool stop = false;
    Item nxt = load_item(sg, tc_rec, item_index(0), mtiles);
    for (int i = 0; i < nloc && !stop; ++i) {
      const Item cur = nxt;
      if (i + 1 < nloc) nxt = load_item(sg, tc_rec, item_index(i + 1), mtiles);
      const bd_tenant& T = cur.T;
      const int64_t row = cur.row0 + r;
      const bool live = row < d_out;
      const uint16_t* sc16 = static_cast<const uint16_t*>(T.scales);
      // scale source: 0 = tiled group-128 scales in the window ring, 1 = one load per
      // stage (other group sizes, and G x G blocks), 2 = one value for the whole item
      // (row / tensor)
      const bool blockwise = T.mode == BD_SCALE_BLOCK;
      const int kind = T.mode == BD_SCALE_GROUP ? (T.group_size == 128 ? 0 : 1) : (blockwise ? 1 : 2);
      const int gshift = (T.mode == BD_SCALE_GROUP || blockwise) ? __ffs(T.group_size) - 1 : 0;
      const int64_t srow = blockwise ? (row >> gshift) : row;  // BLOCK: G x G blocks
      uint32_t s_item = 0;
      // (a COL tenant's scales are in its gathered activations: A = +/-1)
      if (kind == 2 && live) s_item = T.mode == BD_SCALE_COL ? 0x3C00u : sc16[T.mode == BD_SCALE_ROW ? row : 0];
      auto stage_scale = [&](int kb) -> uint32_t {
        if (!live || kb >= nkb) return 0u;
        return sc16[srow * (d_in >> gshift) + (((int64_t)kb * DT_BK) >> gshift)];
      };
      uint32_t pre[DT_KPW] = {0, 0, 0, 0};  // kind 1: scales of the next window, loaded ahead
      if (kind == 1) {
#pragma unroll
        for (int j = 0; j < DT_KPW; ++j) pre[j] = stage_scale(j);
      }
      for (int win = 0; win < nwin; ++win) {
        // tcgen05.st below is warp-collective: every decision to stop is taken by the warp
        if (!__all_sync(0xffffffffu, mbar_wait(&full_w[W.slot], W.phase, abort_flag))) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        const uint8_t* wrow = sw + (size_t)W.slot * DT_WIN_SIGN_BYTES + (size_t)r * 32;
        const uint4 lo = *reinterpret_cast<const uint4*>(wrow);
        const uint4 hi = *reinterpret_cast<const uint4*>(wrow + 16);
        uint32_t wsel[DT_KPW];
        wsel[0] = h ? lo.y : lo.x;
        wsel[1] = h ? lo.w : lo.z;
        wsel[2] = h ? hi.y : hi.x;
        wsel[3] = h ? hi.w : hi.z;
        uint32_t scl[DT_KPW];
        if (kind == 0) {
          const uint32_t sp = *reinterpret_cast<const uint32_t*>(ss + (size_t)W.slot * DT_WIN_SCALE_BYTES + (size_t)r * 4);
          scl[0] = scl[1] = sp & 0xFFFFu;
          scl[2] = scl[3] = sp >> 16;
        } else if (kind == 1) {
#pragma unroll
          for (int j = 0; j < DT_KPW; ++j) {
            scl[j] = pre[j];
            pre[j] = stage_scale((win + 1) * DT_KPW + j);
          }
        } else {
#pragma unroll
          for (int j = 0; j < DT_KPW; ++j) scl[j] = s_item;
        }
        mbar_arrive(&empty_w[W.slot]);
        W.next(DT_WSLOTS);
        if (!live) {
#pragma unroll
          for (int j = 0; j < DT_KPW; ++j) wsel[j] = 0u, scl[j] = 0u;
        }
        // the A window slot must have been read by the MMAs of two windows ago
        if (A.n >= DT_AW) {
          const int pw = A.n - DT_AW;
          if (!__all_sync(0xffffffffu, mbar_wait(&wdone[pw % DT_WDONE],
                                                 (uint32_t)(pw / DT_WDONE) & 1u, abort_flag))) {
            *abort_flag = 1;
            stop = true;
            break;
          }
        }
        tc_fence_after();
        const uint32_t abase = a_lane + (uint32_t)A.slot * (DT_KPW * 32u);
#pragma unroll
        for (int j = 0; j < DT_KPW; ++j) {
          // a partial last window leaves its tail stages unwritten; the MMAs skip them
          const uint32_t w = wsel[j];
          const uint32_t s2 = scl[j] | (scl[j] << 16);
          uint32_t v[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            // bits q and q + 16 to the sign positions 15 and 31 of the pair: a clear bit
            // (delta < 0) flips the sign of the scale
            const uint32_t t = w << (15 - q);
            v[q] = s2 ^ (~t & 0x80008000u);
          }
          tmem_st16(abase + (uint32_t)j * 32u, v);
        }
        tmem_wait_st();
        // publish the window once its X has landed too, so that the MMA issuer waits once
        if (!__all_sync(0xffffffffu, mbar_wait(&full_x[X.slot], X.phase, abort_flag))) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        tc_fence_before();
        mbar_arrive(&full_a[A.slot]);
        A.next(DT_AW);
        X.next(xwin);
      }
    }
    tmem_wait_st();
  } else if (warp < 12) {
    // ---------------- epilogue: thread = row of the tile ----------------
    const int q4 = warp - 8;
    const int er = q4 * 32 + lane;
    Item nxt = load_item(sg, tc_rec, item_index(0), mtiles);
    for (int i = 0; i < nloc; ++i) {
      const Item cur = nxt;
      if (i + 1 < nloc) nxt = load_item(sg, tc_rec, item_index(i + 1), mtiles);
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (uint32_t)(i >> 1) & 1u, abort_flag))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int64_t row = cur.row0 + er;
      const int npad = (cur.count + 15) & ~15;
      const uint32_t lane_addr =
          tmem_base + (uint32_t)ab * DT_ACC_STRIDE + ((uint32_t)(q4 * 32) << 16);
      for (int c0 = 0; c0 < npad; c0 += 16) {
        uint32_t rr[16];
        tmem_ld16(lane_addr + (uint32_t)c0, rr);
        if (row < d_out) {
          // 16 tokens at a time: token ids and 2^-e first, then every split-K partial of
          // all 16 outputs as independent loads, then the stores
          int tok[16];
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = c0 + j;
            const bool ok = c < cur.count;
            tok[j] = ok ? sg.perm[cur.start + c] : 0;
            v[j] = ok ? __uint_as_float(rr[j]) * xinv[cur.xrow + c] : 0.f;
          }
          for (int kz = 0; kz < ksplit; ++kz) {
            const float* part = y_part + (int64_t)kz * batch * d_out + row;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < cur.count) v[j] += part[(int64_t)tok[j] * d_out];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < cur.count) {
              if (y_bf16)
                reinterpret_cast<uint16_t*>(y)[(int64_t)tok[j] * d_out + row] = (uint16_t)f2bf_bits(v[j]);
              else
                reinterpret_cast<float*>(y)[(int64_t)tok[j] * d_out + row] = v[j];
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  } else if (warp == 12) {
    if (lane == 0) {
      // ---------------- MMA issuer: 16 MMAs per window ----------------
      Ring A, X;
      bool stop = false;
      int ncount = sg.count[item_index(0) / mtiles];
      const uint32_t sb_addr = smem_u32(sb);
      for (int i = 0; i < nloc && !stop; ++i) {
        const int ab = i & 1;
        const int npad = (ncount + 15) & ~15;
        if (i + 1 < nloc) ncount = sg.count[item_index(i + 1) / mtiles];
        if (i >= 2 && !mbar_wait(&acc_empty[ab], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = umma_idesc_f16(DT_BM, npad, false);
        const uint32_t d_tmem = tmem_base + (uint32_t)ab * DT_ACC_STRIDE;
        for (int win = 0; win < nwin; ++win) {
          if (!mbar_wait(&full_a[A.slot], A.phase, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = tmem_base + DT_A_COL0 + (uint32_t)A.slot * (DT_KPW * 32u);
          const uint64_t b0 = umma_desc_sw128(sb_addr + (uint32_t)X.slot * xw_bytes);
          const int nst = min(DT_KPW, nkb - win * DT_KPW);
          if (win == 0)
            umma_f16_ts<0>(d_tmem, a0, b0, idesc);
          else
            umma_f16_ts<1>(d_tmem, a0, b0, idesc);
#pragma unroll
          for (int k = 1; k < DT_KPW * 4; ++k) {
            // stage j = k / 4 (32 TMEM columns, b_bytes of X), K step k % 4 (8 columns, 32 B)
            if (k / 4 < nst)
              umma_f16_ts<1>(d_tmem, a0 + (uint32_t)((k / 4) * 32 + (k % 4) * 8),
                             b0 + (uint64_t)(((k / 4) * b_bytes + (k % 4) * 32) >> 4), idesc);
          }
          umma_commit(&wdone[A.n % DT_WDONE]);  // frees this window's A and X slots
          A.next(DT_AW);
          X.next(xwin);
        }
        if (!stop) umma_commit(&acc_full[ab]);
      }
      // no MMA may be in flight when the CTA leaves
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else if (warp == 13) {
    if (lane == 0) {
      // ---------------- X loader: one window (4 stages) of the segment's tokens per fill ----------------
      Ring X;
      bool stop = false;
      int ncount = sg.count[item_index(0) / mtiles], nxrow = sg.xrow[item_index(0) / mtiles];
      for (int i = 0; i < nloc && !stop; ++i) {
        const int npad = (ncount + 15) & ~15;
        const int xrow = nxrow;
        if (i + 1 < nloc) {
          const int sn = item_index(i + 1) / mtiles;
          ncount = sg.count[sn];
          nxrow = sg.xrow[sn];
        }
        for (int win = 0; win < nwin; ++win) {
          // the slot's previous fill (window X.n - xwin) must have been read by its MMAs
          if (X.n >= xwin && !mbar_wait(&wdone[(X.n - xwin) % DT_WDONE],
                                        (uint32_t)((X.n - xwin) / DT_WDONE) & 1u, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          const int nst = min(DT_KPW, nkb - win * DT_KPW);
          mbar_arrive_expect_tx(&full_x[X.slot], (uint32_t)(nst * npad) * DT_BK * 2);
          for (int j = 0; j < nst; ++j)
            for (int jr = 0; jr < npad; jr += 16)
              tma_load_2d(sb + (size_t)X.slot * xw_bytes + (size_t)j * b_bytes + (size_t)jr * 128,
                          &tm_x, &full_x[X.slot], (win * DT_KPW + j) * DT_BK, xrow + jr);
          X.next(xwin);
        }
      }
      // every copy issued must have landed before the CTA leaves: wait for the last fill
      // of each slot (a fill that was already consumed returns at once)
      for (int k = 1; k <= xwin && k <= X.n; ++k) {
        const int f = X.n - k;
        mbar_wait(&full_x[f % xwin], (uint32_t)(f / xwin) & 1u, nullptr);
      }
    }
  } else if (lane == 0) {
    // ---------------- sign loader: one window (128 rows x 256 columns) per copy ----------------
    Ring W;
    bool stop = false;
    Item nxt = load_item(sg, tc_rec, item_index(0), mtiles);
    for (int i = 0; i < nloc && !stop; ++i) {
      const Item cur = nxt;
      if (i + 1 < nloc) nxt = load_item(sg, tc_rec, item_index(i + 1), mtiles);
      const bd_tenant& T = cur.T;
      const bool tiled_scales = T.mode == BD_SCALE_GROUP && T.group_size == 128;
      const int64_t tile_row = (cur.row0 >> 9) * nwin;
      const uint32_t wbytes = DT_WIN_SIGN_BYTES + (tiled_scales ? DT_WIN_SCALE_BYTES : 0u);
      for (int win = 0; win < nwin; ++win) {
        if (W.n >= DT_WSLOTS && !mbar_wait(&empty_w[W.slot], W.phase ^ 1u, abort_flag)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        const int64_t tile = tile_row + win;
        mbar_arrive_expect_tx(&full_w[W.slot], wbytes);
        bulk_load(sw + (size_t)W.slot * DT_WIN_SIGN_BYTES,
                  T.signs + tile * 4096 + (cur.row0 & 511) * 8, DT_WIN_SIGN_BYTES, &full_w[W.slot]);
        if (tiled_scales)
          bulk_load(ss + (size_t)W.slot * DT_WIN_SCALE_BYTES,
                    static_cast<const uint16_t*>(T.scales) + tile * 1024 + (cur.row0 & 511) * 2,
                    DT_WIN_SCALE_BYTES, &full_w[W.slot]);
        W.next(DT_WSLOTS);
      }
    }
    for (int k = 1; k <= DT_WSLOTS && k <= W.n; ++k) {
      const int f = W.n - k;
      mbar_wait(&full_w[f % DT_WSLOTS], (uint32_t)(f / DT_WSLOTS) & 1u, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0 && tid == 0) atomicOr(status, BD_DEV_TIMEOUT);
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem_base, DT_TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------

size_t delta_tc_smem(int nmax, int xwin) {
  size_t need = 1024 + (size_t)xwin * DT_KPW * nmax * DT_BK * 2 +
                (size_t)DT_WSLOTS * (DT_WIN_SIGN_BYTES + DT_WIN_SCALE_BYTES) +
                (size_t)(DT_XW_MAX + DT_WDONE + DT_AW + 2 * DT_WSLOTS + 5) * 8 + 16;
  // at least half of the SM's shared memory: one CTA per SM, so that the 512 tensor-memory
  // columns each CTA allocates never wait on a co-resident CTA
  return need < 120 * 1024 ? 120 * 1024 : need;
}

int delta_tc_xwin(int nmax) {
  int w = DT_XW_MAX;
  while (w > 2 && delta_tc_smem(nmax, w) > 220 * 1024) --w;
  return w;
}

bd_status launch_delta_tc(const bd_tenant* tc_rec, const int32_t* seg, int max_groups, int max_tc,
                          const void* x, int64_t d_out, int64_t d_in, int64_t batch, __half* xg,
                          int64_t xg_rows, float* xinv, const float* y_part, int ksplit, void* y,
                          bool y_bf16, uint32_t* status, cudaStream_t s) {
  if (max_tc <= 0) return BD_OK;
  // 1. gather X of the tensor-core segments
  dim3 gg(DT_NMAX, (unsigned)max_tc);  // one CTA per Xg row
  launch_begin(K_TC_GATHER, s);
  BD_CUDA_TRY(launch_pdl(k_tc_gather, gg, dim3(DT_GATHER_THREADS), 0, s, seg, max_groups, max_tc, tc_rec,
                         static_cast<const uint16_t*>(x), d_in, xg, xinv));
  launch_end(K_TC_GATHER, s);
  BD_LAUNCH_CHECK();
  // 2. tensor-core delta + combine
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return BD_ERR_CUDA;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)xg_rows};
  cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
  cuuint32_t box[2] = {(cuuint32_t)DT_BK, 16};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xg, dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return BD_ERR_CUDA;
  int nmax = (int)((batch + 15) / 16) * 16;
  if (nmax > DT_NMAX) nmax = DT_NMAX;
  const int xwin = delta_tc_xwin(nmax);
  const size_t smem = delta_tc_smem(nmax, xwin);
  static std::atomic<uint64_t> attr{0};
  if (!ensure_dyn_smem(k_delta_tc, 227 * 1024, attr)) return BD_ERR_CUDA;

  const int64_t mtiles = (d_out + DT_BM - 1) / DT_BM;
  int64_t grid = (int64_t)sm_count();
  if (grid > mtiles * max_tc) grid = mtiles * max_tc;
  launch_begin(K_DELTA_TC, s);
  BD_CUDA_TRY(launch_pdl(k_delta_tc, dim3((unsigned)grid), dim3(DT_THREADS), smem, s, tm, tc_rec, seg, max_groups,
                         max_tc, (const float*)xinv, y_part, ksplit, d_out, d_in, (int)batch, y, y_bf16, nmax, xwin,
                         status));
  launch_end(K_DELTA_TC, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd
