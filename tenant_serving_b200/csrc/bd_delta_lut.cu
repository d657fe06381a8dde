// Lookup-table delta product for tenants with few tokens in the batch (bd_apply_multi).
//
// "BitDelta Guide", "Systems Mechanics: 2. Fused Dequantization": the packed sign bits are
// streamed from HBM once and expanded on chip. For a lookup group (NT <= 4 tokens of one
// tenant) the delta of one output row is
//     y_t[row] = sum_chunk s(row, chunk) * T_t[v(row, chunk)][chunk]
// where a chunk is 8 consecutive columns, v(row, chunk) the row's sign byte of that chunk
// and T_t[v][chunk] = sum_j (bit j of v ? +x_t : -x_t)[8 chunk + j]: for every chunk a
// 256-entry table of all signed sums, built in shared memory once per 256-column window.
// One byte of signs then costs one shared-memory read per token instead of eight
// multiply-adds, and all NT tokens are served by one pass over the tenant's bits.
//
// Organisation: persistent, one CTA per SM, 17 warps.
//   warp 16, producer: walks this CTA's share of the (lookup group, 512-row tile) units,
//     cut into pieces of <= DL_PMAX consecutive tiles of one group. For every (window,
//     tile) of a piece it fills one stage of a ring: a header, the tile's 16 KB of sign
//     words (one bulk copy from the tiled serving layout, or 512 row copies of 32 bytes
//     from the row-major layout) and the tile's group-128 scales. Per window, the x slices
//     of the group's tokens (and column scales) go to a two-slot ring of their own.
//   warps 0-15, consumers: warp w owns rows 32w..32w+31 of every tile, one row per lane.
//     At the first tile of a window they rebuild the tables (warp w fills the 16 sign
//     patterns whose high nibble is w); then each lane turns its row's 32 sign bytes into
//     32 * NT table reads. Lane l takes word (i + l/4) % 8 at slot i and byte (j + l) % 4
//     at step j, so the 32 lanes of a warp always read 32 different chunks; with tables
//     laid out [v][chunk], one bank per chunk, the reads are conflict free. One PRMT of
//     the sign word with a per-lane constant gives v * 256 + 4 * chunk directly.
//     Running sums per (tile, token) live in tensor memory (4 columns per tile in the
//     warp's 128-column block), so one build of a window's tables serves every tile of a
//     piece. At the end of a piece each lane adds the base product's partial sums and
//     writes y for its rows, in request order.
// Every wait is bounded; on a timeout the kernel sets BD_DEV_TIMEOUT, lets its copies
// land, frees its tensor memory and returns.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

namespace bd {

constexpr int DL_CWARPS = 16;                       // consumer warps
constexpr int DL_THREADS = (DL_CWARPS + 1) * 32;    // + the producer warp
constexpr int DL_ROWS = 512;                        // rows per tile = 32 per consumer warp
constexpr int DL_W = 256;                           // columns per window (32 chunks)
constexpr int DL_PMAX = 32;                         // tiles per piece (4 TMEM columns each)
constexpr int DL_STAGES = 4;
constexpr uint32_t DL_TABLE_BYTES = 2 * 65536;      // page 0: tokens 0, 1; page 1: tokens 2, 3
constexpr uint32_t DL_SIGN_BYTES = 16384;           // [512 rows][8 words]
constexpr uint32_t DL_SC_OFF = 16384;               // [512 rows][2] group-128 scales
constexpr uint32_t DL_SC_BYTES = 4096;
constexpr uint32_t DL_HDR_OFF = DL_SC_OFF + DL_SC_BYTES;
constexpr uint32_t DL_STAGE_BYTES = DL_HDR_OFF + 128;
constexpr uint32_t DL_XTOK_BYTES = 1024;            // one token's window of x (256 x fp32 max)
constexpr uint32_t DL_XCS_OFF = 4 * DL_XTOK_BYTES;  // column scales of the window
constexpr uint32_t DL_XSLOT_BYTES = DL_XCS_OFF + 1024;
constexpr uint32_t DL_TMEM_COLS = 512;
constexpr size_t DL_SMEM = 128 + DL_TABLE_BYTES + DL_STAGES * DL_STAGE_BYTES + 2 * DL_XSLOT_BYTES + 256;
static_assert(DL_SMEM <= 227 * 1024, "shared memory layout too large");

// header flags
constexpr int F_WIN0 = 1;      // first tile of a window: rebuild the tables
constexpr int F_LAST = 2;      // last stage of a piece: write y
constexpr int F_BASE = 4;      // base-only piece (no delta): write y from the base product
constexpr int F_END = 8;       // no more work for this CTA
constexpr int F_FIRSTWIN = 16; // window 0: the running sums start here
// sign sources
constexpr int SS_STAGED = 0;   // in the stage (bulk copies)
constexpr int SS_DIRECT = 1;   // each lane loads its row's words from global memory
// scale kinds
constexpr int SK_STAGED = 0;   // group-128 scales in the stage ([row][2])
constexpr int SK_GLOBAL = 1;   // group scales loaded from global memory per word
constexpr int SK_NONE = 2;     // row / tensor (applied at the end) or column (folded into x)

// Work weight of one (group, tile) unit of class k (groups of 4, 3, 2, 1 tokens, then
// base-only groups): about the shared-memory reads of its lookups plus its sign stream.
__host__ __device__ constexpr int lut_class_weight(int k) { return k < 4 ? 17 - 4 * k : 1; }

struct DlHdr {
  const void* scales;
  const uint32_t* signs;
  int32_t flags, nt, p, P;
  int32_t tile0, win, mode, skind;
  int32_t lg, ssrc, pad0, pad1;
  int32_t tok[4];
};
static_assert(sizeof(DlHdr) <= 128, "stage header too large");

// ------------------------------------------------------------------------------------
// small device helpers
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
template <int OFF>
__device__ __forceinline__ float lds_off(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32f(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
// All consumer warps meet on `bar` (count DL_CWARPS, one arrive per warp); the wait is
// bounded, so a warp that gave up cannot leave the others blocked. Warp-uniform result.
__device__ __forceinline__ bool consumer_sync(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}
// 32 lanes x 4 columns of tensor memory <-> 4 registers per thread
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3]))
               : "memory");
}
__device__ __forceinline__ void tmem_ld4_issue(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st4() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ldg_scale(const void* s, bool f16, int64_t i) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

// ------------------------------------------------------------------------------------
// the lookups of one row-window: 8 sign words, NT tokens
// ------------------------------------------------------------------------------------
// wd[i]: sign word (i + sigma) % 8 of the row; sc[i]: its scale; K[i] byte j: 4 * chunk of
// (slot i, step j); sel[j]: PRMT selector -> byte 0 = K byte j, byte 1 = the sign byte of
// step j, bytes 2-3 = 0 (sign replicate of K byte j, which is < 128). The table entry of
// token t sits at tbase + v * 256 + 4 * chunk + (t & 1) * 128 + (t >> 1) * 65536.
template <int NT>
__device__ __forceinline__ void lut_row_window(const uint32_t (&wd)[8], const float (&sc)[8],
                                               const uint32_t (&K)[8], const uint32_t (&sel)[4],
                                               uint32_t tbase, float (&part)[4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float a[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) a[t] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t addr = tbase + prmt(wd[i], K[i], sel[j]);
      a[0] += lds_off<0>(addr);
      if (NT > 1) a[NT > 1 ? 1 : 0] += lds_off<128>(addr);
      if (NT > 2) a[NT > 2 ? 2 : 0] += lds_off<65536>(addr);
      if (NT > 3) a[NT > 3 ? 3 : 0] += lds_off<65536 + 128>(addr);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) part[t] = fmaf(sc[i], a[t], part[t]);
  }
}

// Tables of one window for the group's tokens, from the x slice (and column scales) in
// slot xs. Thread (warp h, lane c): chunk c, sign patterns with high nibble h.
template <bool XBF16>
__device__ __forceinline__ void lut_build(uint32_t tbase, uint32_t xs, int nt, bool col_mode,
                                          bool cs_f16, int64_t col0, int64_t d_in) {
  const int c = threadIdx.x & 31, h = threadIdx.x >> 5;
  const bool valid = col0 + 8 * c < d_in;  // d_in % 32 == 0: a chunk is all in or all out
  float cs[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) cs[k] = 1.f;
  if (col_mode && valid) {
    if (cs_f16) {
      uint4 v;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(xs + DL_XCS_OFF + 16u * c));
      const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&a[k]);
        cs[2 * k] = __low2float(hh);
        cs[2 * k + 1] = __high2float(hh);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) cs[k] = __uint_as_float(lds32(xs + DL_XCS_OFF + 32u * c + 4u * k));
    }
  }
  for (int t = 0; t < nt; ++t) {
    float xv[8];
    if (valid) {
      const uint32_t xa = xs + (uint32_t)t * DL_XTOK_BYTES;
      if (XBF16) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(xa + 16u * c));
        const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          xv[2 * k] = bf16lo(a[k]);
          xv[2 * k + 1] = bf16hi(a[k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) xv[k] = __uint_as_float(lds32(xa + 32u * c + 4u * k));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) xv[k] *= cs[k];
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
    const uint32_t base = tbase + (uint32_t)(t >> 1) * 65536u + (uint32_t)(t & 1) * 128u +
                          (uint32_t)(16 * h) * 256u + 4u * (uint32_t)c;
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) sts32f(base + (uint32_t)lo * 256u, (p01[lo & 3] + p23[lo >> 2]) + hi);
  }
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------
struct DlRing {
  int slot = 0;
  uint32_t phase = 0;
  int n = 0;
  __device__ __forceinline__ void next(int slots) {
    ++n;
    if (++slot == slots) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

template <bool XBF16>
__global__ void __launch_bounds__(DL_THREADS, 1) k_delta_lut(
    const bd_tenant* __restrict__ tenants, bool scale_f16, const int32_t* __restrict__ seg_base,
    int max_groups, int max_tc, const void* __restrict__ x, const float* __restrict__ y_part,
    int ksplit, int64_t d_out, int64_t d_in, int batch, void* __restrict__ y, bool y_bf16,
    uint32_t* __restrict__ status) {
  extern __shared__ uint8_t dl_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dl_smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t tbase = smem_u32(sm);
  uint8_t* stages = sm + DL_TABLE_BYTES;
  uint8_t* xslots = stages + DL_STAGES * DL_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(xslots + 2 * DL_XSLOT_BYTES);
  uint64_t* empty = full + DL_STAGES;
  uint64_t* xfull = empty + DL_STAGES;
  uint64_t* xempty = xfull + 2;
  uint64_t* cbar = xempty + 2;  // [2]: consumers before / after a table build
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cbar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < DL_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], DL_CWARPS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], DL_CWARPS);
      mbar_init(&cbar[i], DL_CWARPS);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == DL_CWARPS) tmem_alloc(tmem_slot, DL_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int32_t* grp_tenant = seg_base + kSegHeader;
  const int32_t* grp_start = grp_tenant + max_groups;
  const int32_t* grp_len = grp_start + max_groups;
  const int32_t* perm = grp_len + max_groups + 4 * max_tc;
  const int nwin = (int)((d_in + DL_W - 1) / DL_W);
  const int tiles = (int)((d_out + DL_ROWS - 1) / DL_ROWS);
  const int64_t wpr = d_in >> 5;

  if (warp == DL_CWARPS) {
    // ================================ producer ================================
    // class k: lookup groups of 4, 3, 2, 1 tokens of a tenant, then base-only groups;
    // a (group, tile) unit weighs about its shared-memory reads
    int64_t W = 0;
    for (int k = 0; k < kLutClasses; ++k) W += (int64_t)seg_base[2 + k] * tiles * lut_class_weight(k);
    const int64_t r0 = W * (int64_t)blockIdx.x / gridDim.x;
    const int64_t r1 = W * ((int64_t)blockIdx.x + 1) / gridDim.x;
    const int ssz = scale_f16 ? 2 : 4;
    const int xb = XBF16 ? 2 : 4;
    DlRing S, X;
    bool stop = false;

    // wait for a free stage; false on abort / timeout (warp-uniform)
    auto acquire = [&]() -> bool {
      bool ok = true;
      if (lane == 0 && S.n >= DL_STAGES) ok = mbar_wait(&empty[S.slot], S.phase ^ 1u, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok && lane == 0) *abort_flag = 1;
      return ok;
    };

    int64_t Ck = 0;  // weight before class k
    int Sk = 0;      // first group of class k
    for (int k = 0; k < kLutClasses && !stop; ++k) {
      const int nk = seg_base[2 + k];
      const int wk = lut_class_weight(k);
      const int64_t Ck1 = Ck + (int64_t)nk * tiles * wk;
      const int64_t lo = r0 > Ck ? r0 : Ck, hi = r1 < Ck1 ? r1 : Ck1;
      const int64_t cbase = Ck;
      const int sbase = Sk;
      Ck = Ck1;
      Sk += nk;
      if (lo >= hi) continue;
      // units whose start offset cbase + j * wk lies in [lo, hi)
      const int64_t j1 = (hi - cbase + wk - 1) / wk;
      int64_t j = (lo - cbase + wk - 1) / wk;
      while (j < j1 && !stop) {
        const int item = sbase + (int)(j / tiles);
        const int tile0 = (int)(j % tiles);
        int P = tiles - tile0;
        if (P > DL_PMAX) P = DL_PMAX;
        if ((int64_t)P > j1 - j) P = (int)(j1 - j);
        j += P;
        // ---- the group and its tenant record
        const int u0 = grp_tenant[item];
        const int nt = grp_len[item];
        int tok[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) tok[q] = q < nt ? perm[grp_start[item] + q] : 0;
        bd_tenant T{};
        int u = u0;
        if (u >= 0) {
          T = tenants[u];
          const bool ok_mode = T.mode >= BD_SCALE_GROUP && T.mode <= BD_SCALE_TENSOR;
          const bool ok_group = T.mode != BD_SCALE_GROUP ||
                                (T.group_size >= 32 && (T.group_size & (T.group_size - 1)) == 0 &&
                                 (d_in % T.group_size) == 0);
          const bool ok_ptr = T.signs != nullptr && T.scales != nullptr &&
                              ((reinterpret_cast<uintptr_t>(T.signs) |
                                reinterpret_cast<uintptr_t>(T.scales)) & 15u) == 0;
          const bool ok_layout = (T.layout == BD_LAYOUT_ROWMAJOR || T.layout == BD_LAYOUT_TILED) &&
                                 T.reserved == 0;
          if (!(ok_mode && ok_group && ok_ptr && ok_layout)) {
            if (lane == 0) atomicOr(status, BD_DEV_TENANT_RECORD);
            u = -1;
          }
        }
        if (u < 0) {
          // base-only piece: one header-only stage
          if (!acquire()) { stop = true; break; }
          if (lane == 0) {
            DlHdr* H = reinterpret_cast<DlHdr*>(stages + S.slot * DL_STAGE_BYTES + DL_HDR_OFF);
            H->flags = F_BASE | F_LAST;
            H->nt = nt;
            H->p = 0;
            H->P = P;
            H->tile0 = tile0;
            H->win = 0;
            H->mode = BD_SCALE_GROUP;
            H->skind = SK_NONE;
            H->lg = 0;
            H->ssrc = SS_STAGED;
            H->scales = nullptr;
            H->signs = nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) H->tok[q] = tok[q];
            mbar_arrive(&full[S.slot]);
          }
          __syncwarp();
          S.next(DL_STAGES);
          continue;
        }
        int lg = 0;
        if (T.mode == BD_SCALE_GROUP)
          while ((1 << lg) < T.group_size) ++lg;
        const bool tiled = T.layout == BD_LAYOUT_TILED;
        const int skind = T.mode != BD_SCALE_GROUP ? SK_NONE
                          : ((T.group_size == 128 && tiled) ? SK_STAGED : SK_GLOBAL);
        const int ssrc = (tiled || (d_in % DL_W) == 0) ? SS_STAGED : SS_DIRECT;
        for (int win = 0; win < nwin && !stop; ++win) {
          // ---- x slices (and column scales) of this window
          const int64_t col0 = (int64_t)win * DL_W;
          const int ncols = (int)((d_in - col0) < DL_W ? (d_in - col0) : DL_W);
          {
            bool ok = true;
            if (lane == 0 && X.n >= 2) ok = mbar_wait(&xempty[X.slot], X.phase ^ 1u, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
              if (lane == 0) *abort_flag = 1;
              stop = true;
              break;
            }
            if (lane == 0) {
              uint8_t* xs = xslots + X.slot * DL_XSLOT_BYTES;
              const uint32_t xbytes = (uint32_t)(ncols * xb);
              const uint32_t cbytes = T.mode == BD_SCALE_COL ? (uint32_t)(ncols * ssz) : 0u;
              mbar_arrive_expect_tx(&xfull[X.slot], xbytes * (uint32_t)nt + cbytes);
              for (int q = 0; q < nt; ++q)
                bulk_load(xs + q * DL_XTOK_BYTES,
                          reinterpret_cast<const uint8_t*>(x) + ((int64_t)tok[q] * d_in + col0) * xb,
                          xbytes, &xfull[X.slot]);
              if (cbytes)
                bulk_load(xs + DL_XCS_OFF, reinterpret_cast<const uint8_t*>(T.scales) + col0 * ssz,
                          cbytes, &xfull[X.slot]);
            }
            __syncwarp();
            X.next(2);
          }
          for (int p = 0; p < P; ++p) {
            if (!acquire()) { stop = true; break; }
            const int tile = tile0 + p;
            uint8_t* st = stages + S.slot * DL_STAGE_BYTES;
            const int rows = (int)((d_out - (int64_t)tile * DL_ROWS) < DL_ROWS ? (d_out - (int64_t)tile * DL_ROWS)
                                                                                : DL_ROWS);
            uint32_t bytes = 0;
            if (ssrc == SS_STAGED) bytes += tiled ? DL_SIGN_BYTES : (uint32_t)rows * 32u;
            if (skind == SK_STAGED) bytes += 1024u * (uint32_t)ssz;
            if (lane == 0) {
              DlHdr* H = reinterpret_cast<DlHdr*>(st + DL_HDR_OFF);
              int f = 0;
              if (p == 0) f |= F_WIN0;
              if (win == 0) f |= F_FIRSTWIN;
              if (win == nwin - 1 && p == P - 1) f |= F_LAST;
              H->flags = f;
              H->nt = nt;
              H->p = p;
              H->P = P;
              H->tile0 = tile0;
              H->win = win;
              H->mode = T.mode;
              H->skind = skind;
              H->lg = lg;
              H->ssrc = ssrc;
              H->scales = T.scales;
              H->signs = T.signs;
#pragma unroll
              for (int q = 0; q < 4; ++q) H->tok[q] = tok[q];
              if (bytes) mbar_arrive_expect_tx(&full[S.slot], bytes);
              else mbar_arrive(&full[S.slot]);
              if (ssrc == SS_STAGED && tiled)
                bulk_load(st, T.signs + ((int64_t)tile * nwin + win) * 4096, DL_SIGN_BYTES, &full[S.slot]);
              if (skind == SK_STAGED)
                bulk_load(st + DL_SC_OFF,
                          reinterpret_cast<const uint8_t*>(T.scales) + ((int64_t)tile * nwin + win) * 1024 * ssz,
                          1024u * (uint32_t)ssz, &full[S.slot]);
            }
            __syncwarp();
            if (ssrc == SS_STAGED && !tiled) {
              // row-major, d_in % 256 == 0: one 32-byte copy per row (16-byte aligned)
              for (int r = lane; r < rows; r += 32)
                bulk_load(st + r * 32, T.signs + ((int64_t)tile * DL_ROWS + r) * wpr + (int64_t)win * 8, 32u,
                          &full[S.slot]);
            }
            __syncwarp();
            S.next(DL_STAGES);
          }
        }
      }
    }
    // end marker; after an abort there is none: the consumers see the abort flag instead
    if (!stop && acquire()) {
      if (lane == 0) {
        DlHdr* H = reinterpret_cast<DlHdr*>(stages + S.slot * DL_STAGE_BYTES + DL_HDR_OFF);
        H->flags = F_END;
        mbar_arrive(&full[S.slot]);
      }
      __syncwarp();
      S.next(DL_STAGES);
    }
    // every copy issued must land before the CTA leaves: the last fill of each stage and
    // of each x slot completes its phase (bounded; a phase already completed returns at once)
    if (lane == 0) {
      for (int q = 1; q <= DL_STAGES && q <= S.n; ++q) {
        const int f = S.n - q;
        mbar_wait(&full[f % DL_STAGES], (uint32_t)(f / DL_STAGES) & 1u, nullptr);
      }
      for (int q = 1; q <= 2 && q <= X.n; ++q) {
        const int f = X.n - q;
        mbar_wait(&xfull[f % 2], (uint32_t)(f / 2) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ================================ consumers ================================
    const int sig = lane >> 2, rho = lane & 3;
    uint32_t K[8], sel[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b = (uint32_t)((j + rho) & 3);
      const uint32_t kb = 4u + (uint32_t)j;
      sel[j] = kb | (b << 4) | ((0x8u | kb) << 8) | ((0x8u | kb) << 12);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t wi = (uint32_t)((i + sig) & 7);
      uint32_t v = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) v |= (4u * (4u * wi + (uint32_t)((j + rho) & 3))) << (8 * j);
      K[i] = v;
    }
    const uint32_t t_lane = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(warp >> 2) * 128u;
    const int r_in = warp * 32 + lane;  // row inside a tile
    DlRing S, X;
    bool dead = false;
    for (;;) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(&full[S.slot], S.phase, abort_flag));
      if (!got) {
        if (lane == 0) *abort_flag = 1;
        dead = true;
        break;
      }
      const uint8_t* st = stages + S.slot * DL_STAGE_BYTES;
      const DlHdr* H = reinterpret_cast<const DlHdr*>(st + DL_HDR_OFF);
      const int flags = H->flags;
      if (flags & F_END) break;
      const int nt = H->nt, p = H->p, P = H->P, tile0 = H->tile0, win = H->win, mode = H->mode;
      const int skind = H->skind, lg = H->lg, ssrc = H->ssrc;
      const void* scales = H->scales;
      const uint32_t* signs = H->signs;
      int tok[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) tok[q] = H->tok[q];

      if (!(flags & F_BASE)) {
        if (flags & F_WIN0) {
          // new window: wait for its x, rebuild the tables once every warp is done with
          // the previous window's lookups
          const bool xok = __all_sync(0xffffffffu, mbar_wait(&xfull[X.slot], X.phase, abort_flag));
          if (!xok) {
            if (lane == 0) *abort_flag = 1;
            dead = true;
            break;
          }
          // X.n counts the windows seen: both meeting barriers flip phase once per window
          const uint32_t cpar = (uint32_t)X.n & 1u;
          if (!consumer_sync(&cbar[0], cpar, abort_flag)) {
            if (lane == 0) *abort_flag = 1;
            dead = true;
            break;
          }
          lut_build<XBF16>(tbase, smem_u32(xslots + X.slot * DL_XSLOT_BYTES), nt, mode == BD_SCALE_COL,
                           scale_f16, (int64_t)win * DL_W, d_in);
          __syncwarp();
          if (lane == 0) mbar_arrive(&xempty[X.slot]);
          X.next(2);
          if (!consumer_sync(&cbar[1], cpar, abort_flag)) {
            if (lane == 0) *abort_flag = 1;
            dead = true;
            break;
          }
        }
        const int64_t row = (int64_t)(tile0 + p) * DL_ROWS + r_in;
        const bool live = row < d_out;
        // the row's 8 sign words, rotated by sigma
        uint32_t wd[8];
        if (ssrc == SS_STAGED) {
          const uint32_t wrow = smem_u32(st) + (uint32_t)r_in * 32u;
#pragma unroll
          for (int i = 0; i < 8; ++i) wd[i] = lds32(wrow + 4u * (uint32_t)((i + sig) & 7));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int64_t wi = (int64_t)win * 8 + ((i + sig) & 7);
            wd[i] = (live && wi < wpr) ? signs[row * wpr + wi] : 0u;
          }
        }
        // the scale of each word
        float sc[8];
        if (skind == SK_STAGED) {
          const uint32_t sa = smem_u32(st) + DL_SC_OFF + (uint32_t)r_in * (scale_f16 ? 4u : 8u);
          float s0, s1;
          if (scale_f16) {
            const uint32_t v = lds32(sa);
            s0 = __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu)));
            s1 = __half2float(__ushort_as_half((unsigned short)(v >> 16)));
          } else {
            s0 = __uint_as_float(lds32(sa));
            s1 = __uint_as_float(lds32(sa + 4u));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = ((i + sig) & 7) < 4 ? s0 : s1;
        } else if (skind == SK_GLOBAL) {
          const int64_t gpr = d_in >> lg;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int64_t col = (int64_t)win * DL_W + 32 * ((i + sig) & 7);
            sc[i] = (live && col < d_in) ? ldg_scale(scales, scale_f16, row * gpr + (col >> lg)) : 0.f;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = 1.f;
        }
        const uint32_t tcol = t_lane + 4u * (uint32_t)p;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
        if (!(flags & F_FIRSTWIN)) {
          // running sums of this tile from the previous windows
          uint32_t old[4];
          tmem_wait_st4();
          tmem_ld4_issue(tcol, old);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) part[q] = __uint_as_float(old[q]);
        }
        switch (nt) {
          case 1: lut_row_window<1>(wd, sc, K, sel, tbase, part); break;
          case 2: lut_row_window<2>(wd, sc, K, sel, tbase, part); break;
          case 3: lut_row_window<3>(wd, sc, K, sel, tbase, part); break;
          default: lut_row_window<4>(wd, sc, K, sel, tbase, part); break;
        }
        tmem_st4(tcol, part);
      }
      // the stage is consumed (its header was copied to registers above)
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[S.slot]);
      S.next(DL_STAGES);

      if (flags & F_LAST) {
        // ---- end of a piece: y = base partial sums + delta, rows of this lane
        const bool base_only = (flags & F_BASE) != 0;
        if (!base_only) tmem_wait_st4();
        float rs = 1.f;
        if (!base_only && mode == BD_SCALE_TENSOR) rs = ldg_scale(scales, scale_f16, 0);
        for (int p0 = 0; p0 < P; p0 += 8) {
          uint32_t acc[32];
          if (!base_only) {
            tmem_ld32(t_lane + 4u * (uint32_t)p0, acc);  // includes the wait
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) acc[q] = 0u;
          }
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) {
            if (p0 + pp >= P) break;
            const int64_t row = (int64_t)(tile0 + p0 + pp) * DL_ROWS + r_in;
            if (row >= d_out) continue;
            float s_row = rs;
            if (!base_only && mode == BD_SCALE_ROW) s_row = ldg_scale(scales, scale_f16, row);
            float bsum[4] = {0.f, 0.f, 0.f, 0.f};
            for (int kz = 0; kz < ksplit; ++kz) {
              const float* part = y_part + (int64_t)kz * batch * d_out + row;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (q < nt) bsum[q] += part[(int64_t)tok[q] * d_out];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (q < nt) {
                const float v = bsum[q] + (base_only ? 0.f : s_row * __uint_as_float(acc[4 * pp + q]));
                if (y_bf16)
                  reinterpret_cast<uint16_t*>(y)[(int64_t)tok[q] * d_out + row] = (uint16_t)f2bf_bits(v);
                else
                  reinterpret_cast<float*>(y)[(int64_t)tok[q] * d_out + row] = v;
              }
            }
          }
        }
      }
    }
    (void)dead;
    tmem_wait_st4();
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0 && tid == 0) atomicOr(status, BD_DEV_TIMEOUT);
  if (warp == DL_CWARPS) {
    tc_fence_after();
    tmem_dealloc(tmem_base, DL_TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
size_t delta_lut_smem() { return DL_SMEM; }

bd_status launch_delta_lut(bool xbf16, const bd_tenant* tenants, bool scale_f16, const int32_t* seg,
                           int max_groups, int max_tc, const void* x, const float* y_part, int ksplit,
                           int64_t d_out, int64_t d_in, int64_t batch, void* y, bool y_bf16,
                           uint32_t* status, cudaStream_t s) {
  auto kfn = xbf16 ? k_delta_lut<true> : k_delta_lut<false>;
  static std::atomic<uint64_t> attr[2];
  if (!ensure_dyn_smem(kfn, (int)DL_SMEM, attr[xbf16 ? 1 : 0])) return BD_ERR_CUDA;
  launch_begin(K_DELTA_LUT, s);
  kfn<<<(unsigned)sm_count(), DL_THREADS, DL_SMEM, s>>>(tenants, scale_f16, seg, max_groups, max_tc, x,
                                                       y_part, ksplit, d_out, d_in, (int)batch, y, y_bf16,
                                                       status);
  launch_end(K_DELTA_LUT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd
