// Lookup-table delta product for tenants with few tokens in the batch (bd_apply_multi).
//
// "BitDelta Guide", "Systems Mechanics: 2. Fused Dequantization": the packed sign bits are
// streamed from HBM once and expanded on chip. For a lookup group (NT <= 4 tokens of one
// tenant) the delta of one output row is
//     y_t[row] = sum_chunk s(row, chunk) * T_t[v(row, chunk)][chunk]
// where a chunk is 8 consecutive columns, v(row, chunk) the row's sign byte of that chunk
// and T_t[v][chunk] = sum_j (bit j of v ? +x_t : -x_t)[8 chunk + j]: for every chunk a
// 256-entry table of all signed sums, built in shared memory once per 256-column window.
// One byte of signs then costs one shared-memory read per token (one 8-byte read per pair
// of tokens) instead of eight multiply-adds, and all NT tokens are served by one pass over
// the tenant's bits.
//
// Organisation: persistent, one CTA per SM, 9 warps.
//   Work: (lookup group, K chunk, 512-row tile) units, split over the CTAs by a cost model
//     (a group of NT tokens costs about what its table reads cost, times the windows of a
//     chunk); a CTA walks its share in pieces of <= DL_PMAX consecutive tiles of one group
//     and chunk and hands each to the consumers through a small descriptor ring. A unit
//     covers all of d_in, or one of kc K chunks when the call has too few (group, tile)
//     units to fill the SMs.
//   K chunks: each chunk of a tile leaves its 512 x 4 running sums in the workspace; the
//     CTA that completes a tile adds them in chunk order and writes y.
//   warp 8, producer: for every (window, tile) of a piece fills one stage of a ring with
//     the tile's 16 KB of sign words (one bulk copy from the tiled serving layout, or 512
//     row copies of 32 bytes from the row-major layout) and its group-128 scales; per
//     window, the x slices of the group's tokens (and column scales) go to a two-slot
//     ring of their own, DL_XSLOTS windows deep.
//   warps 0-7, consumers: warp w owns rows 32w + l and 256 + 32w + l of every tile (lane
//     l). At the first tile of a window they rebuild the tables, then each lane turns its
//     rows' sign bytes into table reads. Lane l takes word (i + l/4) % 8 at slot i and byte
//     (j + l) % 4 at step j, so a warp's 32 lanes always address 32 different chunks and
//     the reads are bank-conflict free. The tables sit on a 64 KB boundary: one PRMT of the
//     sign word with a per-lane constant gives the whole shared address of an entry.
//     Running sums per (tile, row, token) live in tensor memory, so one build of a
//     window's tables serves every tile of a piece. At the end of a piece each lane adds
//     the base product's partial sums and writes y for its rows, in request order.
// Every wait is bounded; on a timeout the kernel sets BD_DEV_TIMEOUT, lets its copies
// land, frees its tensor memory and returns.
#include "bd_internal.cuh"
#include "bd_tc.cuh"

namespace bd {

#ifndef BD_LUT_CWARPS
#define BD_LUT_CWARPS 8
#endif
constexpr int DL_CWARPS = BD_LUT_CWARPS;            // consumer warps (8 or 16)
constexpr int DL_THREADS = (DL_CWARPS + 1) * 32;    // + the producer warp
constexpr int DL_ROWS = kLutTileRows;               // rows per tile (512)
constexpr int DL_RPL = DL_ROWS / (32 * DL_CWARPS);  // rows of a tile per consumer lane
constexpr int DL_NIB = 16 / DL_CWARPS;              // table high nibbles built per warp
// tensor memory of a consumer warp: its lane quadrant (warp % 4) and a block of columns;
// a tile's running sums take 4 columns per row of the lane (tokens 0-3)
constexpr uint32_t DL_TBLK = 512u / (DL_CWARPS / 4);
constexpr uint32_t DL_TSTRIDE = 4u * DL_RPL;
static_assert(DL_CWARPS == 8 || DL_CWARPS == 16, "8 or 16 consumer warps");
constexpr int DL_W = kLutWindow;                    // columns per window (256: 32 chunks)
constexpr int DL_PMAX = 32;                         // tiles per piece (DL_TSTRIDE TMEM columns each)
static_assert(DL_PMAX * 4 * DL_RPL <= (int)(512u / (DL_CWARPS / 4)), "running sums fit the warp's columns");
constexpr int DL_MAX_STAGES = 4;
constexpr uint32_t DL_PAGE = 65536;                 // one page of tables (256 v x 256 B)
constexpr uint32_t DL_TABLE_BYTES = 2 * DL_PAGE;    // page 0: tokens 0, 1; page 1: tokens 2, 3
constexpr uint32_t DL_SIGN_BYTES = 16384;           // [512 rows][8 words]
constexpr uint32_t DL_SC_OFF = 16384;               // [512 rows][2] group-128 scales
constexpr uint32_t DL_STAGE_BYTES = DL_SC_OFF + 4096;
constexpr int DL_XSLOTS = 4;                        // x ring depth in windows
// one x slot: 4 tokens' window of x (256 columns) + the window's column scales (fp32 max)
__host__ __device__ constexpr uint32_t dl_xtok_bytes(bool xbf16) { return xbf16 ? 512u : 1024u; }
__host__ __device__ constexpr uint32_t dl_xcs_off(bool xbf16) { return 4u * dl_xtok_bytes(xbf16); }
__host__ __device__ constexpr uint32_t dl_xslot_bytes(bool xbf16) { return dl_xcs_off(xbf16) + 1024u; }
// after the tables: the x slots, then the piece descriptors, barriers and flags
__host__ __device__ constexpr uint32_t dl_fixed_bytes(bool xbf16) { return DL_XSLOTS * dl_xslot_bytes(xbf16) + 640u; }
constexpr uint32_t DL_TMEM_COLS = 512;
constexpr int DL_SMEM = 227 * 1024;                 // the whole per-CTA shared memory
static_assert(DL_STAGE_BYTES % 128 == 0 && dl_fixed_bytes(true) % 128 == 0 && dl_fixed_bytes(false) % 128 == 0,
              "16-byte aligned copies");

// sign sources
constexpr int SS_STAGED = 0;   // in the stage (bulk copies)
constexpr int SS_DIRECT = 1;   // each lane loads its rows' words from global memory
// scale kinds
constexpr int SK_STAGED = 0;   // group-128 scales in the stage ([row][2])
constexpr int SK_GLOBAL = 1;   // group scales loaded from global memory per word
constexpr int SK_NONE = 2;     // row / tensor (applied at the end) or column (folded into x)

// Work weight of one (group, tile) unit of class k (groups of 4, 3, 2, 1 tokens, then
// base-only groups) over all of d_in: its time relative to a one-token unit, fitted to
// per-CTA busy time measured on B200 over the four fused Llama-3-8B calls (4 tokens
// 1.7-2.2, 3 tokens 1.5-2.0, 2 tokens 1.15-1.25; a base-only unit only writes y).
__host__ __device__ constexpr int lut_class_weight(int k) {
  return k == 0 ? 19 : (k == 1 ? 17 : (k == 2 ? 12 : (k == 3 ? 10 : 1)));
}

// Shared-memory layout of the kernel, from the address where its dynamic window starts:
// the tables on the first 64 KB boundary, ring stages below them and after them, the x
// slots and barriers right after the tables. The same arithmetic runs on the host (launch
// check) and in the kernel.
struct DlLayout {
  uint32_t tbase, fixed, stage0_lo, stage0_hi;
  int n_lo, stages;
};
__host__ __device__ inline DlLayout dl_layout(uint32_t raw_base, uint32_t raw_bytes, bool xbf16) {
  DlLayout L;
  const uint32_t base = (raw_base + 127u) & ~127u;
  const uint32_t end = raw_base + raw_bytes;
  L.tbase = (base + DL_PAGE - 1) & ~(DL_PAGE - 1);
  L.fixed = L.tbase + DL_TABLE_BYTES;
  L.stage0_lo = base;
  L.stage0_hi = L.fixed + dl_fixed_bytes(xbf16);
  L.n_lo = (int)((L.tbase - base) / DL_STAGE_BYTES);
  const int n_hi = L.stage0_hi <= end ? (int)((end - L.stage0_hi) / DL_STAGE_BYTES) : -1000;
  int n = L.n_lo + n_hi;
  if (n > DL_MAX_STAGES) n = DL_MAX_STAGES;
  L.stages = n;  // < 2: the layout does not fit
  return L;
}
__device__ __forceinline__ uint32_t dl_stage_addr(const DlLayout& L, int i) {
  return i < L.n_lo ? L.stage0_lo + (uint32_t)i * DL_STAGE_BYTES
                    : L.stage0_hi + (uint32_t)(i - L.n_lo) * DL_STAGE_BYTES;
}

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
template <int OFF>
__device__ __forceinline__ float2 lds2_off(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(v.x), "=f"(v.y) : "r"(a), "n"(OFF));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32f(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts64f(uint32_t a, float x, float y) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(x), "f"(y) : "memory");
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
__device__ __forceinline__ void tmem_ld4_wait(uint32_t taddr, float* v) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int q = 0; q < 4; ++q) v[q] = __uint_as_float(r[q]);
}
// 32 lanes x 8 columns of tensor memory <-> 8 registers per thread
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}
__device__ __forceinline__ void tmem_ld8_wait(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = __uint_as_float(r[q]);
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 32 lanes x 8 (or 4) columns of tensor memory -> registers, without waiting: the registers
// hold the values only after tmem_ld_tile_wait on them (the wait takes them as operands,
// so no use can be scheduled before it). Lets a tile's table reads overlap the load.
__device__ __forceinline__ void tmem_ld_tile_async(uint32_t taddr, uint32_t* r) {
  if (DL_RPL == 2)
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  else
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_tile_wait(uint32_t* r) {
  if (DL_RPL == 2)
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
  else
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]) : : "memory");
}
// the running sums of one tile (DL_TSTRIDE columns)
__device__ __forceinline__ void tmem_st_tile(uint32_t taddr, const float* v) {
  if (DL_RPL == 2) tmem_st8(taddr, v);
  else tmem_st4(taddr, v);
}
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float* v) {
  if (DL_RPL == 2) tmem_ld8_wait(taddr, v);
  else tmem_ld4_wait(taddr, v);
}

__device__ __forceinline__ float ldg_scale(const void* s, bool f16, int64_t i) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

// ------------------------------------------------------------------------------------
// the walk over this CTA's (group, tile) units
// ------------------------------------------------------------------------------------
struct DlPiece {
  bd_tenant T;
  int item, tile0, P, nt, u, skind, ssrc, lg;
  int w0, w1, chunk, kc;  // windows [w0, w1) = K chunk `chunk` of kc
  int tok[4];
};

// Units of class k: (group, K chunk, tile), tile fastest. Tenant classes are cut into
// kc K chunks of wpc windows each (kc from the plan); base-only groups are not cut. With
// kc > 1 a unit weighs its class weight times the windows it covers (base-only: times all
// of them); with kc = 1 the class weights alone (the CTA boundaries then fall where the
// weights were fitted, which measured best).
struct DlWalk {
  int64_t r0, r1, Ck, j, j1, cbase;
  int k, Sk, sbase, wk, tiles, kc, wpc, nwin, ukc;
};

__device__ __forceinline__ int dl_unit_weight(int k, int wpc, int nwin) {
  return wpc == nwin ? lut_class_weight(k) : lut_class_weight(k) * (k < kLutClasses - 1 ? wpc : nwin);
}

// split: the launch may cut units into K chunks (else every unit covers all of d_in)
__device__ __forceinline__ void walk_init(DlWalk& w, const int32_t* seg_base, int tiles, int nwin, bool split) {
  int kc = split ? seg_base[2 + kLutClasses] : 1;
  if (kc < 1 || kc > kLutMaxChunks || nwin % kc != 0) kc = 1;  // (the planner only writes valid values)
  w.kc = kc;
  w.nwin = nwin;
  w.wpc = nwin / kc;
  int64_t W = 0;
  for (int k = 0; k < kLutClasses; ++k)
    W += (int64_t)seg_base[2 + k] * tiles * (k < kLutClasses - 1 ? kc : 1) * dl_unit_weight(k, w.wpc, nwin);
  w.r0 = W * (int64_t)blockIdx.x / gridDim.x;
  w.r1 = W * ((int64_t)blockIdx.x + 1) / gridDim.x;
  w.Ck = 0;
  w.Sk = 0;
  w.k = -1;
  w.j = w.j1 = 0;
  w.cbase = 0;
  w.sbase = 0;
  w.wk = 1;
  w.ukc = 1;
  w.tiles = tiles;
}

// Next piece of this CTA's share; false when there is none. Deterministic: every lane of
// the producer warp gets the same sequence. *bad is set for an invalid record.
__device__ __forceinline__ bool walk_next(DlWalk& w, const int32_t* __restrict__ seg_base, const int32_t* __restrict__ grp_tenant,
                          const int32_t* __restrict__ grp_start, const int32_t* __restrict__ grp_len,
                          const int32_t* __restrict__ perm, const bd_tenant* __restrict__ tenants,
                          int64_t d_in, DlPiece& pc, bool* bad) {
  while (w.j >= w.j1) {
    if (++w.k >= kLutClasses) return false;
    const int nk = seg_base[2 + w.k];
    w.wk = dl_unit_weight(w.k, w.wpc, w.nwin);
    w.ukc = w.k < kLutClasses - 1 ? w.kc : 1;
    const int64_t Ck1 = w.Ck + (int64_t)nk * w.ukc * w.tiles * w.wk;
    const int64_t lo = w.r0 > w.Ck ? w.r0 : w.Ck, hi = w.r1 < Ck1 ? w.r1 : Ck1;
    w.cbase = w.Ck;
    w.sbase = w.Sk;
    w.Ck = Ck1;
    w.Sk += nk;
    if (lo < hi) {
      // the units whose start offset cbase + j * wk lies in [lo, hi)
      w.j = (lo - w.cbase + w.wk - 1) / w.wk;
      w.j1 = (hi - w.cbase + w.wk - 1) / w.wk;
    } else {
      w.j = w.j1 = 0;
    }
  }
  const int64_t per_item = (int64_t)w.ukc * w.tiles;
  pc.item = w.sbase + (int)(w.j / per_item);
  const int64_t rem = w.j % per_item;
  pc.chunk = (int)(rem / w.tiles);
  pc.kc = w.ukc;
  pc.tile0 = (int)(rem % w.tiles);
  pc.w0 = w.ukc > 1 ? pc.chunk * w.wpc : 0;
  pc.w1 = w.ukc > 1 ? pc.w0 + w.wpc : w.nwin;
  int P = w.tiles - pc.tile0;
  if (P > DL_PMAX) P = DL_PMAX;
  if ((int64_t)P > w.j1 - w.j) P = (int)(w.j1 - w.j);
  pc.P = P;
  w.j += P;
  pc.nt = grp_len[pc.item];
  const int gs = grp_start[pc.item];
#pragma unroll
  for (int t = 0; t < 4; ++t) pc.tok[t] = t < pc.nt ? perm[gs + t] : 0;
  pc.u = grp_tenant[pc.item];
  *bad = false;
  if (pc.u >= 0) {
    pc.T = tenants[pc.u];
    const bd_tenant& T = pc.T;
    const bool ok_mode = scale_mode_ok(T.mode, T.group_size, d_in);
    const bool ok_ptr = T.signs != nullptr && T.scales != nullptr &&
                        ((reinterpret_cast<uintptr_t>(T.signs) | reinterpret_cast<uintptr_t>(T.scales)) & 15u) == 0;
    const bool ok_layout = (T.layout == BD_LAYOUT_ROWMAJOR || T.layout == BD_LAYOUT_TILED) && T.reserved == 0;
    if (!(ok_mode && ok_ptr && ok_layout)) {
      *bad = true;
      pc.u = -1;
    }
  }
  pc.lg = 0;
  pc.skind = SK_NONE;
  pc.ssrc = SS_STAGED;
  if (pc.u >= 0) {
    const bd_tenant& T = pc.T;
    if (T.mode == BD_SCALE_GROUP || T.mode == BD_SCALE_BLOCK)
      while ((1 << pc.lg) < T.group_size) ++pc.lg;
    const bool tiled = T.layout == BD_LAYOUT_TILED;
    pc.skind = T.mode == BD_SCALE_BLOCK ? SK_GLOBAL
               : T.mode != BD_SCALE_GROUP ? SK_NONE : ((T.group_size == 128 && tiled) ? SK_STAGED : SK_GLOBAL);
    pc.ssrc = (tiled || (d_in % DL_W) == 0) ? SS_STAGED : SS_DIRECT;
  }
  return true;
}

// ------------------------------------------------------------------------------------
// tables and lookups
// ------------------------------------------------------------------------------------
// Table entry of (sign byte v, chunk c, token t), offset from the table base:
//   NT = 1 : v * 256 + 8 * (c & 15) + 4 * (c >> 4)              (32 chunks on 32 banks)
//   NT >= 2: (t >> 1) * 65536 + v * 256 + 8 * c + 4 * (t & 1)   (token pairs side by side)
__host__ __device__ __forceinline__ uint32_t dl_chunk_off(int c, bool single) {
  return single ? (uint32_t)(8 * (c & 15) + 4 * (c >> 4)) : (uint32_t)(8 * c);
}

// The lookups of one row-window: wd[i] = sign word (i + sigma) % 8 of the row, sc[i] its
// scale. part[t] += sum over the window of sc * (table entry), token t; the even and odd
// words accumulate in two independent chains (shorter dependency chains per lane).
template <int NT>
__device__ __forceinline__ void lut_row(const uint32_t (&wd)[8], const float (&sc)[8], const uint32_t (&K)[8][2],
                                        const uint32_t (&sel)[4], float* part) {
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // the word's four table reads per token, added as a tree (two dependent adds, not four)
    float2 e[4], f[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t addr = prmt(wd[i], K[i][j >> 1], sel[j]);
      if (NT == 1) {
        e[j].x = lds_off<0>(addr);
      } else {
        e[j] = lds2_off<0>(addr);
        if (NT == 3) f[j].x = lds_off<(int)DL_PAGE>(addr);
        if (NT == 4) f[j] = lds2_off<(int)DL_PAGE>(addr);
      }
    }
    // even and odd words in two chains of running sums, added at the end
    float* a = acc[i & 1];
    a[0] = fmaf(sc[i], (e[0].x + e[1].x) + (e[2].x + e[3].x), a[0]);
    if (NT > 1) a[1] = fmaf(sc[i], (e[0].y + e[1].y) + (e[2].y + e[3].y), a[1]);
    if (NT > 2) a[2] = fmaf(sc[i], (f[0].x + f[1].x) + (f[2].x + f[3].x), a[2]);
    if (NT > 3) a[3] = fmaf(sc[i], (f[0].y + f[1].y) + (f[2].y + f[3].y), a[3]);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) part[t] += acc[0][t] + acc[1][t];
}

// Tables of one window for the group's tokens, from the x slice (and column scales) in
// slot xs. Thread (warp h8, lane c): chunk c, the sign patterns whose high nibble is
// h8 + DL_CWARPS * k, k < DL_NIB.
template <bool XBF16>
__device__ __forceinline__ void lut_build(uint32_t tbase, uint32_t xs, int nt, bool col_mode, bool cs_f16,
                                          int64_t col0, int64_t d_in) {
  const int c = threadIdx.x & 31, h8 = threadIdx.x >> 5;
  const bool valid = col0 + 8 * c < d_in;  // d_in % 32 == 0: a chunk is all in or all out
  float cs[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) cs[k] = 1.f;
  if (col_mode && valid) {
    if (cs_f16) {
      const uint4 v = lds128(xs + dl_xcs_off(XBF16) + 16u * c);
      const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&a[k]);
        cs[2 * k] = __low2float(hh);
        cs[2 * k + 1] = __high2float(hh);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) cs[k] = __uint_as_float(lds32(xs + dl_xcs_off(XBF16) + 32u * c + 4u * k));
    }
  }
  const bool single = nt == 1;
  const uint32_t coff = dl_chunk_off(c, single);
  for (int t0 = 0; t0 < nt; t0 += 2) {
    // tokens t0 and t0 + 1 (the second one absent for an odd count: zero entries)
    float lo16[2][16], hi[2][DL_NIB];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float xv[8];
      if (valid && t0 + q < nt) {
        const uint32_t xa = xs + (uint32_t)(t0 + q) * dl_xtok_bytes(XBF16);
        if (XBF16) {
          const uint4 v = lds128(xa + 16u * c);
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
#pragma unroll
      for (int lo = 0; lo < 16; ++lo) lo16[q][lo] = p01[lo & 3] + p23[lo >> 2];
#pragma unroll
      for (int hh = 0; hh < DL_NIB; ++hh) {
        const int h = h8 + DL_CWARPS * hh;
        hi[q][hh] = (((h & 1) ? xv[4] : -xv[4]) + ((h & 2) ? xv[5] : -xv[5])) +
                    (((h & 4) ? xv[6] : -xv[6]) + ((h & 8) ? xv[7] : -xv[7]));
      }
    }
    const uint32_t page = tbase + (uint32_t)(t0 >> 1) * DL_PAGE + coff;
#pragma unroll
    for (int hh = 0; hh < DL_NIB; ++hh) {
      const uint32_t rowb = page + (uint32_t)(16 * (h8 + DL_CWARPS * hh)) * 256u;
#pragma unroll
      for (int lo = 0; lo < 16; ++lo) {
        if (single)
          sts32f(rowb + (uint32_t)lo * 256u, lo16[0][lo] + hi[0][hh]);
        else
          sts64f(rowb + (uint32_t)lo * 256u, lo16[0][lo] + hi[0][hh], lo16[1][lo] + hi[1][hh]);
      }
    }
  }
}

// Per-lane PRMT constants for a table layout. K[i][h] bytes 0, 1: the entry offsets of
// the chunks of (slot i, steps 2h and 2h + 1); bytes 2, 3: the table base >> 16.
// sel[j]: byte 0 <- K byte (j & 1), byte 1 <- sign byte (j + rho) % 4 of the word,
// bytes 2, 3 <- K bytes 2, 3.
__device__ __forceinline__ void dl_lane_consts(int lane, uint32_t tbase, bool single, uint32_t (&K)[8][2],
                                               uint32_t (&sel)[4]) {
  const int sig = lane >> 2, rho = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t b = (uint32_t)((j + rho) & 3);
    sel[j] = (4u + (uint32_t)(j & 1)) | (b << 4) | (6u << 8) | (7u << 12);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int wi = (i + sig) & 7;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t o0 = dl_chunk_off(4 * wi + ((2 * h + rho) & 3), single);
      const uint32_t o1 = dl_chunk_off(4 * wi + ((2 * h + 1 + rho) & 3), single);
      K[i][h] = o0 | (o1 << 8) | (tbase & 0xFFFF0000u);
    }
  }
}

// What the consumers need of a piece; written by the producer into a small ring.
struct DlDesc {
  const uint32_t* signs;
  const void* scales;
  int32_t tile0, P, nt, u;  // u: tenant, -1 base only, -2 end of this CTA's work
  int32_t mode, skind, ssrc, lg;
  int32_t tok[4];
};
static_assert(sizeof(DlDesc) == 64, "descriptor slot size");
// K-chunk part of a piece's descriptor (only kernels launched with K chunks use it)
struct DlSplit {
  int32_t w0, w1, item, kc;  // windows [w0, w1); lookup group; K chunks of its units
  int32_t chunk, pad[3];
};
static_assert(sizeof(DlSplit) == 32, "split slot size");

constexpr int DL_DSLOTS = 4;
// the fixed region after the x slots: descriptors, split slots, barriers, three words
static_assert(DL_DSLOTS * (sizeof(DlDesc) + sizeof(DlSplit)) +
                      (2 * DL_MAX_STAGES + 2 * DL_XSLOTS + 2 * DL_DSLOTS + 4) * sizeof(uint64_t) + 12 <=
                  dl_fixed_bytes(true) - DL_XSLOTS * dl_xslot_bytes(true),
              "fixed shared-memory region");

// One row-window of a stage: its sign words, their scales, the lookups into part[0..3].
__device__ __forceinline__ void dl_row_window(const DlDesc& D, uint32_t st, int r_in, int tile, int win, int nt,
                                              int sig, uint32_t hi_slots, bool scale_f16, int64_t d_out,
                                              int64_t d_in, int64_t wpr, const uint32_t (&K)[8][2],
                                              const uint32_t (&sel)[4], float* part) {
  const int64_t row = (int64_t)tile * DL_ROWS + r_in;
  const bool live = row < d_out;
  uint32_t wd[8];
  if (D.ssrc == SS_STAGED) {
    const uint32_t wrow = st + (uint32_t)r_in * 32u;
#pragma unroll
    for (int i = 0; i < 8; ++i) wd[i] = lds32(wrow + 4u * (uint32_t)((i + sig) & 7));
  } else {
    const uint32_t* signs = D.signs;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t wi = (int64_t)win * 8 + ((i + sig) & 7);
      wd[i] = (live && wi < wpr) ? signs[row * wpr + wi] : 0u;
    }
  }
  float sc[8];
  const int skind = D.skind;
  if (skind == SK_STAGED) {
    const uint32_t sa = st + DL_SC_OFF + (uint32_t)r_in * (scale_f16 ? 4u : 8u);
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
    for (int i = 0; i < 8; ++i) sc[i] = ((hi_slots >> i) & 1u) ? s1 : s0;
  } else if (skind == SK_GLOBAL) {
    const int lg = D.lg;
    const void* scales = D.scales;
    const int64_t gpr = d_in >> lg;
    const int64_t srow = D.mode == BD_SCALE_BLOCK ? (row >> lg) : row;  // BLOCK: G x G blocks
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t col = (int64_t)win * DL_W + 32 * ((i + sig) & 7);
      sc[i] = (live && col < d_in) ? ldg_scale(scales, scale_f16, srow * gpr + (col >> lg)) : 0.f;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i] = 1.f;
  }
  switch (nt) {
    case 1: lut_row<1>(wd, sc, K, sel, part); break;
    case 2: lut_row<2>(wd, sc, K, sel, part); break;
    case 3: lut_row<3>(wd, sc, K, sel, part); break;
    default: lut_row<4>(wd, sc, K, sel, part); break;
  }
}

// End of a piece whose units are K chunks (Q.kc > 1). Every consumer lane stores the
// running sums of its rows (4 tokens, unscaled) into the unit's slot
// lut_part[((item * tiles + tile) * kc + chunk) * 512 + row][4]; after a barrier, lane p of
// warp 0 counts the arrival at tile p; the CTA that completes a tile's count then reads
// the kc slots of that tile in chunk order, applies the row / tensor scale, adds the base
// partial sums and writes y. Warp-uniform; false when a bounded barrier gave up.
__device__ __noinline__ bool dl_split_epilogue(const DlDesc& D, const DlSplit& Q, int P, int tiles, uint32_t t_lane,
                                               int r_lo, int lane,
                                               int warp, float* __restrict__ lut_part, int32_t* __restrict__ lut_cnt,
                                               int split_cap, const float* __restrict__ y_part, int ksplit, int batch,
                                               int64_t d_out, float rs, bool scale_f16, void* __restrict__ y,
                                               bool y_bf16, uint64_t* bars, uint32_t parity,
                                               volatile uint32_t* last_mask, const volatile int* abort_flag,
                                               uint32_t* __restrict__ status) {
  constexpr int PT = 32 / DL_TSTRIDE;
  const int kc = Q.kc, nt = D.nt;
  const int64_t unit0 = (int64_t)Q.item * tiles + D.tile0;  // (group, tile) of the piece's first tile
  const bool fits = (unit0 + P) * kc <= (int64_t)split_cap;  // guaranteed by the planner
  if (!fits && lane == 0 && warp == 0) atomicOr(status, BD_DEV_INTERNAL);
  for (int p0 = 0; p0 < P; p0 += PT) {
    uint32_t acc[32];
    tmem_ld32(t_lane + DL_TSTRIDE * (uint32_t)p0, acc);
#pragma unroll
    for (int pp = 0; pp < PT; ++pp)
#pragma unroll
      for (int h = 0; h < DL_RPL; ++h) {
        if (p0 + pp >= P || !fits) continue;
        const int r_in = r_lo + 32 * DL_CWARPS * h;
        const int64_t slot = (unit0 + p0 + pp) * kc + Q.chunk;
        const int b = DL_TSTRIDE * pp + 4 * h;
        __stcg(reinterpret_cast<float4*>(lut_part + (slot * DL_ROWS + r_in) * 4),
               make_float4(__uint_as_float(acc[b]), __uint_as_float(acc[b + 1]), __uint_as_float(acc[b + 2]),
                           __uint_as_float(acc[b + 3])));
      }
  }
  __threadfence();  // the slot is visible device-wide before this CTA's arrival is counted
  if (!consumer_sync(&bars[0], parity, abort_flag)) return false;
  if (warp == 0) {
    bool last = false;
    if (lane < P && fits) last = atomicAdd(&lut_cnt[unit0 + lane], 1) == kc - 1;
    const uint32_t m = __ballot_sync(0xffffffffu, last);
    if (lane == 0) *last_mask = m;
  }
  if (!consumer_sync(&bars[1], parity, abort_flag)) return false;
  const uint32_t m = *last_mask;
  if (m == 0) return true;
  __threadfence();  // the other chunks' slots are read after their arrivals were seen
  const int mode = D.mode;
  for (int p = 0; p < P; ++p) {
    if (!((m >> p) & 1u)) continue;
#pragma unroll
    for (int h = 0; h < DL_RPL; ++h) {
      const int r_in = r_lo + 32 * DL_CWARPS * h;
      const int64_t row = (int64_t)(D.tile0 + p) * DL_ROWS + r_in;
      if (row >= d_out) continue;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = 0; c < kc; ++c) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(lut_part + (((unit0 + p) * kc + c) * DL_ROWS + r_in) * 4));
        d[0] += v.x;
        d[1] += v.y;
        d[2] += v.z;
        d[3] += v.w;
      }
      const float s_row = mode == BD_SCALE_ROW ? ldg_scale(D.scales, scale_f16, row) : rs;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q >= nt) continue;
        const int64_t t = D.tok[q];
        float v = 0.f;
        for (int kz = 0; kz < ksplit; ++kz) v += y_part[((int64_t)kz * batch + t) * d_out + row];
        v += s_row * d[q];
        if (y_bf16)
          reinterpret_cast<uint16_t*>(y)[t * d_out + row] = (uint16_t)f2bf_bits(v);
        else
          reinterpret_cast<float*>(y)[t * d_out + row] = v;
      }
    }
  }
  return true;
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

// SPLIT: the planner may have cut units into K chunks (the launch has too few units for
// the SMs otherwise); without it the kernel keeps the plain whole-d_in code paths.
template <bool XBF16, bool SPLIT>
__global__ void __launch_bounds__(DL_THREADS, 1) k_delta_lut(
    const bd_tenant* __restrict__ tenants, bool scale_f16, const int32_t* __restrict__ seg_base,
    int max_groups, int max_tc, const void* __restrict__ x, const float* __restrict__ y_part,
    int ksplit, int64_t d_out, int64_t d_in, int batch, void* __restrict__ y, bool y_bf16,
    float* __restrict__ lut_part, int32_t* __restrict__ lut_cnt, int split_cap,
    uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t dl_smem_raw[];
  const uint32_t raw = smem_u32(dl_smem_raw);
  const DlLayout L = dl_layout(raw, DL_SMEM, XBF16);
  constexpr uint32_t XTOK = dl_xtok_bytes(XBF16), XCS = dl_xcs_off(XBF16), XSLOT = dl_xslot_bytes(XBF16);
  if (L.stages < 2) {  // checked on the host before the launch
    if (threadIdx.x == 0) atomicOr(status, BD_DEV_INTERNAL);
    return;
  }
  uint8_t* gen = dl_smem_raw - raw;  // generic pointer of shared address 0
  const uint32_t xslot0 = L.fixed;
  DlDesc* desc = reinterpret_cast<DlDesc*>(gen + L.fixed + DL_XSLOTS * XSLOT);
  DlSplit* dsplit = reinterpret_cast<DlSplit*>(desc + DL_DSLOTS);
  uint64_t* full = reinterpret_cast<uint64_t*>(dsplit + DL_DSLOTS);
  uint64_t* empty = full + DL_MAX_STAGES;
  uint64_t* xfull = empty + DL_MAX_STAGES;
  uint64_t* xempty = xfull + DL_XSLOTS;
  uint64_t* dfull = xempty + DL_XSLOTS;
  uint64_t* dempty = dfull + DL_DSLOTS;
  // [4]: consumers before / after a table build; around the arrival counts of split units
  uint64_t* cbar = dempty + DL_DSLOTS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cbar + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* last_mask = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
  const int NS = L.stages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < DL_MAX_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], DL_CWARPS);
    }
    for (int i = 0; i < DL_XSLOTS; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], DL_CWARPS);
    }
    for (int i = 0; i < DL_DSLOTS; ++i) {
      mbar_init(&dfull[i], 1);
      mbar_init(&dempty[i], DL_CWARPS);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&cbar[i], DL_CWARPS);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == DL_CWARPS) tmem_alloc(tmem_slot, DL_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the set-up above overlaps the previous kernel on the stream; its outputs (the plan, the
  // base partial sums) are read only after this
  pdl_wait();
  pdl_trigger();

  const int nwin = (int)((d_in + DL_W - 1) / DL_W);
  const int tiles = (int)((d_out + DL_ROWS - 1) / DL_ROWS);
  const int64_t wpr = d_in >> 5;
  const int ssz = scale_f16 ? 2 : 4;

  if (warp == DL_CWARPS) {
    // ================================ producer ================================
    const int32_t* grp_tenant = seg_base + kSegHeader;
    const int32_t* grp_start = grp_tenant + max_groups;
    const int32_t* grp_len = grp_start + max_groups;
    const int32_t* perm = grp_len + max_groups + 4 * max_tc;
    DlWalk walk;
    walk_init(walk, seg_base, tiles, nwin, SPLIT);
    DlPiece pc;
    bool bad = false;
    const int xb = XBF16 ? 2 : 4;
    DlRing S, X, Dr;
    bool stop = false;
    // a free descriptor slot (warp-uniform; false on abort / timeout)
    auto take_desc = [&]() -> bool {
      bool ok = true;
      if (lane == 0 && Dr.n >= DL_DSLOTS) ok = mbar_wait(&dempty[Dr.slot], Dr.phase ^ 1u, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok && lane == 0) *abort_flag = 1;
      return ok;
    };
    for (;;) {
      const bool more = walk_next(walk, seg_base, grp_tenant, grp_start, grp_len, perm, tenants, d_in, pc, &bad);
      if (!take_desc()) {
        stop = true;
        break;
      }
      if (lane == 0) {
        DlDesc& D = desc[Dr.slot];
        if (!more) {
          D.u = -2;
        } else {
          if (bad) atomicOr(status, BD_DEV_TENANT_RECORD);
          D.signs = pc.T.signs;
          D.scales = pc.T.scales;
          D.tile0 = pc.tile0;
          D.P = pc.P;
          D.nt = pc.nt;
          D.u = pc.u;
          D.mode = pc.u >= 0 ? pc.T.mode : (int)BD_SCALE_GROUP;
          D.skind = pc.skind;
          D.ssrc = pc.ssrc;
          D.lg = pc.lg;
          if (SPLIT) {
            DlSplit& Q = dsplit[Dr.slot];
            Q.w0 = pc.w0;
            Q.w1 = pc.w1;
            Q.item = pc.item;
            Q.kc = pc.kc;
            Q.chunk = pc.chunk;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) D.tok[q] = pc.tok[q];
        }
        mbar_arrive(&dfull[Dr.slot]);
      }
      __syncwarp();
      Dr.next(DL_DSLOTS);
      if (!more) break;
      if (pc.u < 0) continue;  // base-only piece: the consumers write it without stages
      const bd_tenant& T = pc.T;
      const bool tiled = T.layout == BD_LAYOUT_TILED;
      const int wbeg = SPLIT ? pc.w0 : 0, wend = SPLIT ? pc.w1 : nwin;
      for (int win = wbeg; win < wend && !stop; ++win) {
        // ---- x slices (and column scales) of this window
        const int64_t col0 = (int64_t)win * DL_W;
        const int ncols = (int)((d_in - col0) < DL_W ? (d_in - col0) : DL_W);
        {
          bool ok = true;
          if (lane == 0 && X.n >= DL_XSLOTS) ok = mbar_wait(&xempty[X.slot], X.phase ^ 1u, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) {
            if (lane == 0) *abort_flag = 1;
            stop = true;
            break;
          }
          if (lane == 0) {
            uint8_t* xs = gen + xslot0 + X.slot * XSLOT;
            const uint32_t xbytes = (uint32_t)(ncols * xb);
            const uint32_t cbytes = T.mode == BD_SCALE_COL ? (uint32_t)(ncols * ssz) : 0u;
            mbar_arrive_expect_tx(&xfull[X.slot], xbytes * (uint32_t)pc.nt + cbytes);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q < pc.nt)
                bulk_load(xs + q * XTOK,
                          reinterpret_cast<const uint8_t*>(x) + ((int64_t)pc.tok[q] * d_in + col0) * xb, xbytes,
                          &xfull[X.slot]);
            if (cbytes)
              bulk_load(xs + XCS, reinterpret_cast<const uint8_t*>(T.scales) + col0 * ssz, cbytes, &xfull[X.slot]);
          }
          __syncwarp();
          X.next(DL_XSLOTS);
        }
        for (int p = 0; p < pc.P; ++p) {
          bool ok = true;
          if (lane == 0 && S.n >= NS) ok = mbar_wait(&empty[S.slot], S.phase ^ 1u, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) {
            if (lane == 0) *abort_flag = 1;
            stop = true;
            break;
          }
          const int tile = pc.tile0 + p;
          uint8_t* st = gen + dl_stage_addr(L, S.slot);
          const int rows = (int)((d_out - (int64_t)tile * DL_ROWS) < DL_ROWS ? (d_out - (int64_t)tile * DL_ROWS)
                                                                              : DL_ROWS);
          uint32_t bytes = 0;
          if (pc.ssrc == SS_STAGED) bytes += tiled ? DL_SIGN_BYTES : (uint32_t)rows * 32u;
          if (pc.skind == SK_STAGED) bytes += 1024u * (uint32_t)ssz;
          if (lane == 0) {
            if (bytes) mbar_arrive_expect_tx(&full[S.slot], bytes);
            else mbar_arrive(&full[S.slot]);
            if (pc.ssrc == SS_STAGED && tiled)
              bulk_load(st, T.signs + ((int64_t)tile * nwin + win) * 4096, DL_SIGN_BYTES, &full[S.slot]);
            if (pc.skind == SK_STAGED)
              bulk_load(st + DL_SC_OFF,
                        reinterpret_cast<const uint8_t*>(T.scales) + ((int64_t)tile * nwin + win) * 1024 * ssz,
                        1024u * (uint32_t)ssz, &full[S.slot]);
          }
          __syncwarp();
          if (pc.ssrc == SS_STAGED && !tiled) {
            // row-major, d_in % 256 == 0: one 32-byte copy per row (16-byte aligned)
            for (int r = lane; r < rows; r += 32)
              bulk_load(st + r * 32, T.signs + ((int64_t)tile * DL_ROWS + r) * wpr + (int64_t)win * 8, 32u,
                        &full[S.slot]);
          }
          __syncwarp();
          S.next(NS);
        }
      }
      if (stop) break;
    }
    // every copy issued must land before the CTA leaves: the last fill of each stage and
    // of each x slot completes its phase (bounded; a phase already completed returns at once)
    if (lane == 0) {
      for (int q = 1; q <= NS && q <= S.n; ++q) {
        const int f = S.n - q;
        mbar_wait(&full[f % NS], (uint32_t)(f / NS) & 1u, nullptr);
      }
      for (int q = 1; q <= DL_XSLOTS && q <= X.n; ++q) {
        const int f = X.n - q;
        mbar_wait(&xfull[f % DL_XSLOTS], (uint32_t)(f / DL_XSLOTS) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ================================ consumers ================================
    // lane constants: rotation sigma (words), which slots hold words 4-7 of a window, the
    // PRMT constants of the table layout in use (recomputed when a piece changes it)
    const int sig = lane >> 2;
    uint32_t hi_slots = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) hi_slots |= (((i + sig) & 7) >= 4 ? 1u : 0u) << i;
    uint32_t K[8][2], sel[4];
    int k_single = -1;
    // tensor memory: lane quadrant warp % 4, column block warp / 4; tile p, row h of the
    // lane, token t at column DL_TSTRIDE * p + 4h + t
    const uint32_t t_lane = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(warp >> 2) * DL_TBLK;
    const int r_lo = warp * 32 + lane;  // rows r_lo + 32 * DL_CWARPS * h of each tile, h < DL_RPL
    DlRing S, X, Dr;
    int nsplit = 0;  // split pieces finished (phase of the two epilogue barriers)
    for (;;) {
      if (!__all_sync(0xffffffffu, mbar_wait(&dfull[Dr.slot], Dr.phase, abort_flag))) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const DlDesc& D = desc[Dr.slot];
      const int u = D.u;
      if (u == -2) break;
      const int nt = D.nt, P = D.P, tile0 = D.tile0;
      bool dead = false;
      if (u >= 0) {
        const bool single = nt == 1;
        if ((int)single != k_single) {
          dl_lane_consts(lane, L.tbase, single, K, sel);
          k_single = (int)single;
        }
        const int wbeg = SPLIT ? dsplit[Dr.slot].w0 : 0, wend = SPLIT ? dsplit[Dr.slot].w1 : nwin;
        for (int win = wbeg; win < wend && !dead; ++win) {
          // new window: wait for its x, rebuild the tables once every warp is done with
          // the previous window's lookups
          const bool xok = __all_sync(0xffffffffu, mbar_wait(&xfull[X.slot], X.phase, abort_flag));
          const uint32_t cpar = (uint32_t)X.n & 1u;  // both meeting barriers flip once per window
          if (!xok || !consumer_sync(&cbar[0], cpar, abort_flag)) {
            dead = true;
            break;
          }
          lut_build<XBF16>(L.tbase, xslot0 + X.slot * XSLOT, nt, D.mode == BD_SCALE_COL, scale_f16,
                           (int64_t)win * DL_W, d_in);
          __syncwarp();
          if (lane == 0) mbar_arrive(&xempty[X.slot]);
          X.next(DL_XSLOTS);
          if (!consumer_sync(&cbar[1], cpar, abort_flag)) {
            dead = true;
            break;
          }
          // the previous window's stores of the running sums are complete before they are
          // read back below
          if (win > wbeg) tmem_wait_st();
          for (int p = 0; p < P; ++p) {
            if (!__all_sync(0xffffffffu, mbar_wait(&full[S.slot], S.phase, abort_flag))) {
              dead = true;
              break;
            }
            const uint32_t st = dl_stage_addr(L, S.slot);
            float part[4 * DL_RPL];
#pragma unroll
            for (int q = 0; q < 4 * DL_RPL; ++q) part[q] = 0.f;
            const uint32_t tcol = t_lane + DL_TSTRIDE * (uint32_t)p;
            // the running sums of this tile from the previous windows load while the
            // window's table reads run; they are added at the end
            uint32_t prev[4 * DL_RPL];
            const bool carry = win > wbeg;
            if (carry) tmem_ld_tile_async(tcol, prev);
#pragma unroll
            for (int h = 0; h < DL_RPL; ++h)
              dl_row_window(D, st, r_lo + 32 * DL_CWARPS * h, tile0 + p, win, nt, sig, hi_slots, scale_f16, d_out,
                            d_in, wpr, K, sel, part + 4 * h);
            if (carry) {
              tmem_ld_tile_wait(prev);
#pragma unroll
              for (int q = 0; q < 4 * DL_RPL; ++q) part[q] += __uint_as_float(prev[q]);
            }
            tmem_st_tile(tcol, part);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[S.slot]);
            S.next(NS);
          }
        }
        if (dead) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        tmem_wait_st();
      }
      // ---- end of a piece: y = base partial sums + delta, rows of this lane. Several
      // tiles at a time: their running sums in one tensor-memory read and all their base
      // partial sums as independent loads before any store.
      const bool base_only = u < 0;
      const int mode = D.mode;
      const void* scales = D.scales;
      float rs = 1.f;
      if (!base_only && mode == BD_SCALE_TENSOR) rs = ldg_scale(scales, scale_f16, 0);
      constexpr int PT = 32 / DL_TSTRIDE;  // tiles per 32-column read
      const bool split = SPLIT && !base_only && dsplit[Dr.slot].kc > 1;
      if (split) {
        // ---- a K chunk of split units: its running sums go to the unit's partial slot;
        // the last chunk to arrive at a tile adds all chunks in chunk order (the result
        // does not depend on which CTA arrives last) and writes y
        if (!dl_split_epilogue(D, dsplit[Dr.slot], P, tiles, t_lane, r_lo, lane, warp, lut_part, lut_cnt, split_cap, y_part, ksplit,
                               batch, d_out, rs, scale_f16, y, y_bf16, &cbar[2], (uint32_t)(nsplit & 1), last_mask,
                               abort_flag, status)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        ++nsplit;
      } else {
        for (int p0 = 0; p0 < P; p0 += PT) {
          uint32_t acc[32];  // tile p0 + pp, row h, token q at DL_TSTRIDE * pp + 4 h + q
          if (!base_only) {
            tmem_ld32(t_lane + DL_TSTRIDE * (uint32_t)p0, acc);
          } else {
  #pragma unroll
            for (int q = 0; q < 32; ++q) acc[q] = 0u;
          }
          float bsum[PT][DL_RPL][4];
  #pragma unroll
          for (int pp = 0; pp < PT; ++pp)
  #pragma unroll
            for (int h = 0; h < DL_RPL; ++h)
  #pragma unroll
              for (int q = 0; q < 4; ++q) bsum[pp][h][q] = 0.f;
          for (int kz = 0; kz < ksplit; ++kz) {
            const float* part = y_part + (int64_t)kz * batch * d_out;
  #pragma unroll
            for (int pp = 0; pp < PT; ++pp)
  #pragma unroll
              for (int h = 0; h < DL_RPL; ++h) {
                const int64_t row = (int64_t)(tile0 + p0 + pp) * DL_ROWS + r_lo + 32 * DL_CWARPS * h;
                if (p0 + pp < P && row < d_out) {
  #pragma unroll
                  for (int q = 0; q < 4; ++q)
                    if (q < nt) bsum[pp][h][q] += part[(int64_t)D.tok[q] * d_out + row];
                }
              }
          }
  #pragma unroll
          for (int pp = 0; pp < PT; ++pp)
  #pragma unroll
            for (int h = 0; h < DL_RPL; ++h) {
              const int64_t row = (int64_t)(tile0 + p0 + pp) * DL_ROWS + r_lo + 32 * DL_CWARPS * h;
              if (p0 + pp >= P || row >= d_out) continue;
              float s_row = rs;
              if (!base_only && mode == BD_SCALE_ROW) s_row = ldg_scale(scales, scale_f16, row);
  #pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (q < nt) {
                  const float v =
                      bsum[pp][h][q] + (base_only ? 0.f : s_row * __uint_as_float(acc[DL_TSTRIDE * pp + 4 * h + q]));
                  const int64_t t = D.tok[q];
                  if (y_bf16)
                    reinterpret_cast<uint16_t*>(y)[t * d_out + row] = (uint16_t)f2bf_bits(v);
                  else
                    reinterpret_cast<float*>(y)[t * d_out + row] = v;
                }
              }
            }
        }
      }
      // the descriptor is no longer read
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[Dr.slot]);
      Dr.next(DL_DSLOTS);
    }
    tmem_wait_st();
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
// The kernel's layout needs its dynamic window to start low enough that the tables (on a
// 64 KB boundary) and at least two ring stages fit: checked once per device from the
// kernel's static shared memory and the device's reserved shared memory per block.
static bool dl_layout_fits(const void* fn, bool xbf16, int v) {
  static std::atomic<uint64_t> ok_bits[4], bad_bits[4];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (ok_bits[v].load() & bit)) return true;
  if (bit && (bad_bits[v].load() & bit)) return false;
  cudaFuncAttributes fa;
  int reserved = 0;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  const uint32_t start = (uint32_t)reserved + (uint32_t)fa.sharedSizeBytes;
  const bool fits = dl_layout(start, DL_SMEM, xbf16).stages >= 2;
  if (bit) (fits ? ok_bits[v] : bad_bits[v]).fetch_or(bit);
  return fits;
}

bd_status launch_delta_lut(bool xbf16, const bd_tenant* tenants, bool scale_f16, const int32_t* seg,
                           int max_groups, int max_tc, const void* x, const float* y_part, int ksplit,
                           int64_t d_out, int64_t d_in, int64_t batch, void* y, bool y_bf16,
                           float* lut_part, int32_t* lut_cnt, int split_cap, uint32_t* status,
                           cudaStream_t s) {
  // the K-chunk variant when the planner cuts units for any plan of this shape (at most
  // max_groups tenant groups of ceil(d_out / 512) tiles, fewer than kLutMinUnitsPerCta per
  // CTA), and for long rows (>= 32 windows), where a plan with few units is worth cutting
  // even if most plans of the shape are not
  const int64_t tiles = (d_out + DL_ROWS - 1) / DL_ROWS, nwin = (d_in + DL_W - 1) / DL_W;
  const bool split = split_cap >= 2 && nwin >= 4 &&
                     ((int64_t)max_groups * tiles < (int64_t)kLutMinUnitsPerCta * sm_count() || nwin >= 32);
  auto kfn = xbf16 ? (split ? k_delta_lut<true, true> : k_delta_lut<true, false>)
                   : (split ? k_delta_lut<false, true> : k_delta_lut<false, false>);
  const int v = (xbf16 ? 1 : 0) + (split ? 2 : 0);
  static std::atomic<uint64_t> attr[4];
  if (!ensure_dyn_smem(kfn, DL_SMEM, attr[v])) return BD_ERR_CUDA;
  if (!dl_layout_fits(reinterpret_cast<const void*>(kfn), xbf16, v)) return BD_ERR_INTERNAL;
  launch_begin(K_DELTA_LUT, s);
  BD_CUDA_TRY(launch_pdl(kfn, dim3((unsigned)sm_count()), dim3(DL_THREADS), DL_SMEM, s, tenants, scale_f16, seg,
                         max_groups, max_tc, x, y_part, ksplit, d_out, d_in, (int)batch, y, y_bf16, lut_part, lut_cnt,
                         split_cap, status));
  launch_end(K_DELTA_LUT, s);
  BD_LAUNCH_CHECK();
  return BD_OK;
}

}  // namespace bd
