/*
 * bitdelta.h — C ABI of the B200 (sm_100a) BitDelta library (libbitdelta.so).
 *
 * Two halves of one method:
 *   compress : Delta = W_fine - W_base, optional k-sigma clip, abs-mean scales, sign bits
 *              ("bitdelta" page, "How BitDelta Works" 1-4 and "Safety Benefits:
 *              1. Outlier Clipping"; "Per-Axis Weight Deltas", "Key Contributions" 1).
 *   apply    : y_t = W_base x_t + Delta_hat_{u(t)} x_t for a batch whose tokens belong to
 *              different tenants u ("BitDelta Guide: 1-Bit Delta Quantization for LLM
 *              Serving", "Systems Mechanics: 1. Decoupled Forward Pass").
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless the argument says "host". The caller owns and
 *     allocates every buffer (workspace included); the library never allocates device
 *     memory and never frees a caller's buffer.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream). Nothing synchronises the host except bd_get_status and
 *     bd_profile_collect, which say so.
 *   - Argument errors that the host can see are returned before anything is launched and
 *     leave outputs untouched. Errors only the device can see (a tenant id out of range,
 *     a wait that ran out) set bits in a status word inside the workspace; no kernel
 *     traps. Read it with bd_get_status.
 *   - Matrices are [d_out][d_in] row-major (the [Out, In] layout of an nn.Linear weight).
 *   - Sign words: uint32 signs[d_out][d_in/32], packed along the input axis; column
 *     32*w + j of a row is bit j of its word w (least significant bit first). Bit 1 means
 *     +1 and bit 0 means -1; sign(0) = +1 (-0.0 included), i.e. bit = !(delta_c < 0).
 *   - Alignment: every pointer to a matrix, sign array or scale array must be 16-byte
 *     aligned (128-bit loads and bulk copies), else BD_ERR_ALIGN.
 *   - Shapes: d_out >= 1, d_in >= 32 and d_in % 32 == 0, else BD_ERR_SHAPE.
 *
 * The float arithmetic (fp32 accumulation) and what each result is compared with are
 * described per call below.
 */
#ifndef BITDELTA_H
#define BITDELTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------------------------- */
/* status, types                                                                       */
/* ---------------------------------------------------------------------------------- */
typedef enum {
  BD_OK = 0,
  BD_ERR_NULL = 1,          /* a required pointer is NULL                              */
  BD_ERR_SHAPE = 2,         /* sizes out of range or not divisible as required        */
  BD_ERR_DTYPE = 3,         /* a dtype code the call does not accept                   */
  BD_ERR_ALIGN = 4,         /* a pointer is not 16-byte aligned                        */
  BD_ERR_CONFIG = 5,        /* bad compress config / scale mode / group size           */
  BD_ERR_CUDA = 6,          /* a CUDA runtime call failed (launch error etc.)          */
  BD_ERR_TENANT_RANGE = 7,  /* device status: a tenant id outside [-1, n_tenants)      */
  BD_ERR_TIMEOUT = 8,       /* device status: a bounded wait gave up                   */
  BD_ERR_WORKSPACE = 9,     /* workspace NULL or smaller than the *_workspace_size     */
  BD_ERR_TENANT_RECORD = 10,/* device status: a bd_tenant record is invalid            */
  BD_ERR_INTERNAL = 11      /* device status: a kernel's layout self-check failed       */
} bd_status;

typedef enum { BD_F32 = 0, BD_BF16 = 1, BD_F16 = 2 } bd_dtype;

/* Scale granularity.
 *  GROUP : one scale per contiguous run of group_size entries along d_in,
 *          scales[d_out][d_in/group_size] ("2. Group Quantization", default 128).
 *  ROW   : one scale per output row, scales[d_out]  (the 1 x d_out vector of
 *          "Per-Axis Weight Deltas").
 *  COL   : one scale per input column, scales[d_in] (the d_in x 1 vector).
 *  TENSOR: one scalar alpha for the whole matrix, scales[1] ("BitDelta Guide",
 *          "2. Optimal L2 Norm Initialization").
 *  BLOCK : one scale per square block of group_size rows x group_size columns,
 *          scales[ceil(d_out/group_size)][d_in/group_size]; the last row block holds
 *          the remaining d_out % group_size rows ("Per-Axis Weight Deltas", Future
 *          Directions: blockwise per-group scaling, read as the row group extended to a
 *          square block).
 * Every scale is the abs-mean of its slice of the clipped delta, the L2-optimal
 * value for fixed signs. GROUP and BLOCK need group_size a power of two >= 32 that
 * divides d_in. */
typedef enum { BD_SCALE_GROUP = 0, BD_SCALE_ROW = 1, BD_SCALE_COL = 2, BD_SCALE_TENSOR = 3,
               BD_SCALE_BLOCK = 4 } bd_scale_mode;

/* Device status bits (bd_get_status). */
#define BD_DEV_TENANT_RANGE 0x1u  /* some token had a tenant id outside [-1, n_tenants) */
#define BD_DEV_TIMEOUT      0x2u  /* a bounded wait inside a kernel gave up              */
#define BD_DEV_TENANT_RECORD 0x4u /* a bd_tenant record had a bad mode, group size or
                                     NULL / misaligned pointer; its tokens got the base
                                     product only                                      */
#define BD_DEV_INTERNAL     0x8u  /* a kernel's shared-memory layout self-check failed and
                                     it returned without writing its outputs            */

/* ---------------------------------------------------------------------------------- */
/* compress                                                                            */
/* ---------------------------------------------------------------------------------- */
typedef struct {
  int32_t group_size; /* GROUP mode: power of two, 32 <= G, G divides d_in. Ignored otherwise. */
  int32_t mode;       /* bd_scale_mode                                                    */
  int32_t clip;       /* 0: no clip; 1: clamp delta to [mean - k*std, mean + k*std]       */
  float clip_k;       /* k of the clip (the pages use 3; 2 for "aggressive")            */
} bd_compress_cfg;

/* Bytes of workspace bd_compress needs for this shape and config (0 is possible). */
size_t bd_compress_workspace_size(int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg /* host */);

/* bd_compress — the compress half: Delta = W_fine - W_base (computed in fp32 from the
 * stored values), optional whole-matrix k-sigma clip with the unbiased (N-1) standard
 * deviation accumulated in fp64, abs-mean scales over the clipped delta (fp32 sums in a
 * fixed tree order, so results are deterministic), and sign bits of the clipped delta.
 * Follows "bitdelta" page, "1. Delta Computation", "2. Group Quantization",
 * "3. 1-bit Quantization", "Outlier Clipping", and the per-axis vectors of "Per-Axis
 * Weight Deltas".
 *
 *   w_base, w_fine : [d_out][d_in], dtype BD_F32 or BD_BF16.
 *   cfg            : host pointer; see bd_compress_cfg.
 *   signs_out      : uint32[d_out][d_in/32], fully overwritten.
 *   scales_out     : fp32, [d_out][d_in/G] (GROUP), [d_out] (ROW), [d_in] (COL), [1] (TENSOR).
 *   stats_out      : optional (may be NULL) fp64[4] = {mean, std, lo, hi} of the delta;
 *                    written only when cfg->clip is set.
 *   workspace      : device scratch of bd_compress_workspace_size() bytes (16-byte aligned);
 *                    may be NULL only when that size is 0.
 * Signs are bit-exact with the fp64 definition (the sign of an fp32 difference is the
 * sign of the exact difference); scales agree with it to ~1e-6 relative.
 * Returns BD_OK or a host-detected error; nothing is written on error. */
bd_status bd_compress(const void* w_base, const void* w_fine, int32_t dtype, int64_t d_out,
                      int64_t d_in, const bd_compress_cfg* cfg, uint32_t* signs_out,
                      float* scales_out, double* stats_out, void* workspace, size_t ws_bytes,
                      void* stream);

/* bd_compress_noalloc — the same computation, arguments and results as bd_compress,
 * but with no workspace argument and no device allocation anywhere on its path.
 * There is no counterpart on the method's source pages; this entry point exists for
 * callers that cannot allocate device memory themselves: code embedded in a host
 * runtime that owns all device memory and forbids raw cudaMalloc, or a latency-critical
 * loop where an allocation (which may synchronise the device) is not acceptable.
 * Its scratch is one fixed array of BD_NOALLOC_SCRATCH_BYTES in the library's device
 * image; every GPU that loads the library holds it until the process exits.
 *   - Shapes and configs whose scratch need (bd_compress_workspace_size) exceeds
 *     BD_NOALLOC_SCRATCH_BYTES are rejected with BD_ERR_WORKSPACE before any launch.
 *     GROUP mode needs about 10 KB at any size; ROW / TENSOR need 8 bytes per row per
 *     column segment (every Llama-3-8B projection fits); COL needs 8 bytes per column
 *     per tile of rows and BLOCK 4 bytes per (row, group), so large COL and BLOCK
 *     problems do not fit.
 *   - The first call on each device looks up the array's device address (with that
 *     device current) and caches it; make that first call before any stream capture.
 *     The cached address does not survive cudaDeviceReset: after a reset, use
 *     bd_compress (or a process that loads the library afresh).
 *   - Every call shares the one array and it keeps the last call's contents; nothing in
 *     it has to start at zero. Calls whose execution overlaps on the GPU (other streams,
 *     other host threads) race on it: serialise them.
 * The caller still passes inputs and outputs, as for bd_compress. */
#define BD_NOALLOC_SCRATCH_BYTES ((size_t)1 << 20)
bd_status bd_compress_noalloc(const void* w_base, const void* w_fine, int32_t dtype,
                              int64_t d_out, int64_t d_in, const bd_compress_cfg* cfg,
                              uint32_t* signs_out, float* scales_out, double* stats_out,
                              void* stream);

/* ---------------------------------------------------------------------------------- */
/* reconstruct                                                                         */
/* ---------------------------------------------------------------------------------- */
/* bd_reconstruct — Delta_hat = sign * scale ("4. Reconstruction"); with w_base given,
 * the personalised weight W_base + Delta_hat ("5. Serving").
 *   signs      : uint32[d_out][d_in/32].
 *   scales     : per `mode` as in bd_compress, dtype scale_dtype (BD_F32 or BD_F16).
 *   w_base     : optional [d_out][d_in] of w_dtype (BD_F32 or BD_BF16), or NULL.
 *   out        : [d_out][d_in] of out_dtype (BD_F32 or BD_BF16; bf16 is rounded to nearest
 *                even from the fp32 value).
 * The fp32 result is exact for fp16/fp32 scales when w_base is NULL. */
bd_status bd_reconstruct(const uint32_t* signs, const void* scales, int32_t scale_dtype,
                         int32_t mode, int32_t group_size, int64_t d_out, int64_t d_in,
                         const void* w_base, int32_t w_dtype, void* out, int32_t out_dtype,
                         void* stream);

/* ---------------------------------------------------------------------------------- */
/* multi-tenant apply                                                                  */
/* ---------------------------------------------------------------------------------- */
/* Storage layouts of a tenant's sign words (and group-128 scales) for bd_apply_multi.
 *  ROWMAJOR : signs uint32[d_out][d_in/32] exactly as bd_compress writes them; scales as
 *             bd_compress writes them (converted to the call's scale_dtype).
 *  TILED    : the serving layout written by bd_prepare_tenant. The matrix is cut into
 *             tiles of 512 rows x 256 columns (8 sign words); tile (rb, w) is 4096
 *             consecutive words [row 0..511][word 0..7] at word offset
 *             (rb * ceil(d_in/256) + w) * 4096, rows past d_out and words past d_in/32
 *             zero. For GROUP scales with group_size 128 the scales are tiled the same
 *             way: tile (rb, w) holds [row 0..511][2 scales] at element offset
 *             (rb * ceil(d_in/256) + w) * 1024. Other scale modes keep their plain layout.
 *  The same bits in either layout give the same result; TILED lets every 512-row stage
 *  of the apply kernel arrive as one contiguous 16 KB block. */
#define BD_LAYOUT_ROWMAJOR 0
#define BD_LAYOUT_TILED 1

/* One resident tenant variant of one projection. An array of these lives in DEVICE
 * memory and is read by the kernels (the host never dereferences it). */
typedef struct {
  const uint32_t* signs;  /* device, per `layout`, 16-byte aligned                       */
  const void* scales;     /* device, per `mode` and `layout`, dtype = the call's scale_dtype */
  int32_t mode;           /* bd_scale_mode                                               */
  int32_t group_size;     /* GROUP mode: power of two, 32 <= G, G divides d_in           */
  int32_t layout;         /* BD_LAYOUT_ROWMAJOR or BD_LAYOUT_TILED                        */
  int32_t reserved;       /* must be 0                                                   */
} bd_tenant;

/* Bytes of the TILED sign words and scales of one tenant (bd_prepare_tenant outputs). */
size_t bd_prepared_signs_bytes(int64_t d_out, int64_t d_in);
size_t bd_prepared_scales_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t group_size,
                                int32_t scale_dtype);

/* bd_prepare_tenant — rewrite one tenant's sign words (uint32[d_out][d_in/32], as
 * bd_compress writes them) and scales (dtype scale_dtype, BD_F16 or BD_F32) into the
 * TILED serving layout described above: a pure re-ordering, no value changes. Scales of
 * modes other than GROUP-128 are copied unchanged. Outputs must not overlap the inputs;
 * sizes are bd_prepared_signs_bytes / bd_prepared_scales_bytes. Done once when a tenant
 * is loaded, not per batch. */
bd_status bd_prepare_tenant(const uint32_t* signs, const void* scales, int32_t scale_dtype,
                            int32_t mode, int32_t group_size, int64_t d_out, int64_t d_in,
                            uint32_t* signs_out, void* scales_out, void* stream);

/* The many-token threshold built into the library: a tenant with at least this many
 * tokens in a batch (and a record the tensor-core path supports) goes to the tensor-core
 * delta; every other tenant goes through the lookup-table delta, at most 4 of its tokens
 * per pass over its bits (a tenant with 5 to 8 tokens is read twice). */
int32_t bd_tc_min_tokens(void);

/* ---------------------------------------------------------------------------------- */
/* host-resident tenant cache and packed-delta loader                                  */
/* ---------------------------------------------------------------------------------- */
/* "Per-Axis Weight Deltas", Key Contributions item 4 and Implementation details: packed
 * deltas (1-bit signs along the input axis + fp16 scale vectors) go to the GPU in a single
 * non-blocking transfer per module, with no dense reconstruction. "BitDelta Guide",
 * "3. Dynamic Model Hot-Swapping and Multi-Tenant Batching": deltas are pre-cached in GPU
 * memory or streamed from host CPU memory.
 *
 * A module is one projection of one layer. Every tenant is kept in host memory as one
 * packed RECORD per module: the TILED sign words (bd_prepared_signs_bytes bytes), then its
 * scales in the TILED layout (bd_prepared_scales_bytes bytes), i.e. the two outputs of
 * bd_prepare_tenant placed back to back. The GPU holds n_slots tenant slots; the cache maps
 * the tenants of each batch onto slots (least recently used slot evicted first) and loads
 * a missing tenant with one cudaMemcpyAsync per module. The caller allocates every buffer
 * (a device pool and pinned host staging); the cache object itself is host memory that
 * bd_cache_create allocates and bd_cache_destroy frees. Not thread-safe: one host thread
 * per cache. */
typedef struct {
  int64_t d_out, d_in;     /* the module's shape: d_out >= 1, d_in >= 32, d_in % 32 == 0    */
  int32_t min_group_size;  /* smallest GROUP size a record may use (power of two >= 32 that
                              divides d_in), or 0 when no record uses GROUP scales          */
  int32_t reserved;        /* 0 */
} bd_cache_module;

typedef struct bd_cache bd_cache;  /* opaque */

/* Bytes of one packed record (0 for an invalid shape, mode, group size or dtype). */
size_t bd_cache_record_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t group_size,
                             int32_t scale_dtype);

/* bd_prepare_record_host — host-side packing of one module of one tenant: sign words
 * uint32[d_out][d_in/32] (as bd_compress writes them) and scales (BD_F16 / BD_F32, plain
 * layout) into a packed record of bd_cache_record_bytes bytes at `record` (host memory).
 * The bytes are those bd_prepare_tenant writes on the device. Pure host code, no CUDA.
 * BD_ERR_WORKSPACE when record_bytes is too small. */
bd_status bd_prepare_record_host(const uint32_t* signs, const void* scales, int32_t scale_dtype,
                                 int32_t mode, int32_t group_size, int64_t d_out, int64_t d_in,
                                 void* record, size_t record_bytes);

/* Device pool bytes for n_slots slots of these modules (tables first, then the slots);
 * pinned host staging bytes (two copies of the tables). 0 for invalid arguments. */
size_t bd_cache_pool_bytes(const bd_cache_module* modules, int32_t n_modules, int32_t n_slots,
                           int32_t scale_dtype);
size_t bd_cache_staging_bytes(int32_t n_modules, int32_t n_slots);

/* bd_cache_create — a cache for n_host_tenants tenants (ids 0 .. n_host_tenants-1) over
 * n_modules modules, every tenant's scales of dtype scale_dtype.
 *   pool    : device, >= bd_cache_pool_bytes, 256-byte aligned; owned by the caller and
 *             written only by the cache's copies.
 *   staging : host, pinned (cudaHostAlloc / pin_memory), >= bd_cache_staging_bytes,
 *             16-byte aligned.
 * Makes no CUDA call (events are created on the first bd_cache_prefetch).
 * Errors: BD_ERR_NULL, BD_ERR_SHAPE, BD_ERR_DTYPE, BD_ERR_ALIGN, BD_ERR_WORKSPACE. */
bd_status bd_cache_create(const bd_cache_module* modules, int32_t n_modules, int32_t scale_dtype,
                          int32_t n_host_tenants, int32_t n_slots, void* pool, size_t pool_bytes,
                          void* staging, size_t staging_bytes, bd_cache** out);
/* Waits for the cache's copies in flight, then frees the host object. */
bd_status bd_cache_destroy(bd_cache* cache);

/* bd_cache_register — the packed record of (tenant, module) in host memory, with its scale
 * mode and group size. The memory must stay valid and unchanged while the cache exists;
 * pinned memory makes the copies asynchronous. A tenant that is resident on the GPU cannot
 * be re-registered (BD_ERR_CONFIG). */
bd_status bd_cache_register(bd_cache* cache, int32_t tenant, int32_t module, const void* record_host,
                            int32_t mode, int32_t group_size);

/* The device table of `module`: bd_cache_slots() bd_tenant records, one per slot, to pass
 * to bd_apply_multi as `tenants` (n_tenants = bd_cache_slots()) with the slot ids from
 * bd_cache_prefetch as `tenant_ids`. NULL for a bad module. */
const bd_tenant* bd_cache_table(const bd_cache* cache, int32_t module);
int32_t bd_cache_slots(const bd_cache* cache);

/* bd_cache_assign — host part of a prefetch, no CUDA call: maps the batch's tenant ids
 * (host int32[batch], -1 = base only) onto slots. Resident tenants are hits; every other
 * distinct tenant takes the least recently used slot not held by an unreleased batch
 * (empty slots first, then the lowest slot index among equals) and is listed in
 * loads[2k] = tenant, loads[2k+1] = slot (host, room for 2 * n_slots ints, may be NULL).
 * Writes slot_ids[t] (host int32[batch]; -1 for -1) and a ticket for the batch, which
 * holds its slots until bd_cache_release. At most 4 batches may be held at once. The
 * loads are left to the caller (bd_cache_prefetch is assign + loads).
 * Errors (nothing changed): BD_ERR_TENANT_RANGE (an id outside [-1, n_host_tenants)),
 * BD_ERR_TENANT_RECORD (a tenant without a record for every module), BD_ERR_CONFIG (not
 * enough free slots for the batch's missing tenants, or 4 batches held). */
bd_status bd_cache_assign(bd_cache* cache, const int32_t* tenant_ids, int64_t batch, int32_t* slot_ids,
                          int32_t* loads, int32_t* n_loads, int64_t* ticket);

/* bd_cache_prefetch — bd_cache_assign, then the loads on copy_stream: for each missing
 * tenant, after the last batch that read its slot has been released, one cudaMemcpyAsync
 * per module from its host record into the slot; then one copy of the changed tables.
 * The batch's ticket records when its copies are done. Issue it for the next batch while
 * the current one computes. A CUDA error returns BD_ERR_CUDA; the batch's new slots are
 * then marked empty and its ticket is closed. */
bd_status bd_cache_prefetch(bd_cache* cache, const int32_t* tenant_ids, int64_t batch, int32_t* slot_ids,
                            int32_t* n_loads, int64_t* ticket, void* copy_stream);
/* Makes compute_stream wait for the ticket's copies (no host wait). acquire and release
 * of a cache's batches go to one compute stream. BD_ERR_CONFIG for a ticket not held. */
bd_status bd_cache_acquire(bd_cache* cache, int64_t ticket, void* compute_stream);
/* Marks the end of the ticket's use on compute_stream (after its bd_apply_multi calls):
 * its slots may be refilled once compute_stream has passed this point. */
bd_status bd_cache_release(bd_cache* cache, int64_t ticket, void* compute_stream);

/* slot_tenant (host int32[n_slots], may be NULL): the tenant in each slot (-1 empty);
 * stats (host int64[4], may be NULL): hits, misses, bytes copied, copies issued. */
bd_status bd_cache_resident(const bd_cache* cache, int32_t* slot_tenant, int64_t* stats);

/* Bytes of workspace bd_apply_multi needs. */
size_t bd_apply_workspace_size(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants);

/* bd_apply_multi — decomposed multi-tenant forward of one linear projection:
 *     y[t] = W_base x[t] + Delta_hat_{u(t)} x[t],   u(t) = tenant_ids[t]
 * ("BitDelta Guide", "Systems Mechanics: 1. Decoupled Forward Pass", and "2. Fused
 * Dequantization": sign bits stay packed in memory and are unpacked on chip).
 * The base product W_base X is computed once for the whole batch; the tokens are
 * grouped by tenant on the device (no host synchronisation). Two delta kernels share the
 * work, chosen per tenant on the device:
 *   - a tenant with at least bd_tc_min_tokens() tokens in the batch (9 as built),
 *     stored in the TILED layout with
 *     fp16 scales in GROUP or BLOCK (group_size >= 64), ROW, COL or TENSOR mode (bf16
 *     activations and d_in % 64 == 0), is a dense product on the tensor cores, in
 *     segments of <= 64 of its tokens; its activations are scaled per token by a power of
 *     two into fp16 for that product (exact for bf16 values in fp16's normal range; for
 *     COL scales the activations are multiplied by the column scales first, and that
 *     product is rounded to fp16, a relative error of at most 2^-11 per element);
 *   - every other tenant goes through the sign lookup-table kernel, its packed signs and
 *     scales streamed once per group of <= 4 of its tokens (once in all when it has at
 *     most 4 tokens in the batch).
 *
 *   w_base      : [d_out][d_in], w_dtype BD_BF16 (tensor-core path) or BD_F32.
 *   tenants     : device array of n_tenants bd_tenant records (n_tenants >= 0).
 *   scale_dtype : BD_F16 or BD_F32, for every tenant's scales.
 *   tenant_ids  : device int32[batch]; -1 = base model only. Ids outside [-1, n_tenants)
 *                 set BD_DEV_TENANT_RANGE and that token gets the base product only.
 *                 A tenant record that is invalid (mode, group size, NULL or unaligned
 *                 pointer) sets BD_DEV_TENANT_RECORD and its tokens get the base only.
 *   x           : [batch][d_in], same dtype as w_base.
 *   y           : [batch][d_out], y_dtype BD_BF16 (round to nearest even) or BD_F32.
 *   workspace   : bd_apply_workspace_size() bytes, 16-byte aligned. Its status word is
 *                 reset by this call, so bd_get_status reports the latest call.
 * Products are accumulated in fp32. batch may be 0 (nothing is launched).
 * Returns BD_OK or a host-detected error. */
bd_status bd_apply_multi(const void* w_base, int32_t w_dtype, int64_t d_out, int64_t d_in,
                         const bd_tenant* tenants, int32_t n_tenants, int32_t scale_dtype,
                         const int32_t* tenant_ids, const void* x, int64_t batch, void* y,
                         int32_t y_dtype, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------- */
/* e4m3 base weights                                                                   */
/* ---------------------------------------------------------------------------------- */
/* "BitDelta Guide", "3. Quantized Base Model Compatibility (BitDelta + GPTQ / QuIP#)":
 * the 1-bit delta is applied on top of quantized base weights; "Per-Axis Weight Deltas",
 * Future Directions: FP8 co-design. The base is held as OCP E4M3 codes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits; largest finite 448; S.1111.111 NaN) with one
 * fp32 scale per output row: W_hat[o][i] = scales[o] * e4m3(codes[o][i]).
 *
 * bd_quantize_base_fp8 — scales[o] = max_i |w[o][i]| / 448 and codes[o][i] = e4m3 of
 * w[o][i] / scales[o], both quotients IEEE fp32 divisions, the rounding to nearest even
 * with saturation at +-448 and the sign kept; a row of zeros gets scale 0 and codes 0.
 *   w      : device [d_out][d_in], w_dtype BD_BF16 or BD_F32, 16-byte aligned.
 *   codes  : device uint8 [d_out][d_in], 16-byte aligned.  scales : device fp32 [d_out].
 * d_in % 32 == 0. Asynchronous on `stream`. */
bd_status bd_quantize_base_fp8(const void* w, int32_t w_dtype, int64_t d_out, int64_t d_in,
                               uint8_t* codes, float* scales, void* stream);

/* Bytes of workspace bd_apply_multi_fp8 needs. */
size_t bd_apply_fp8_workspace_size(int64_t d_out, int64_t d_in, int64_t batch, int32_t n_tenants);

/* bd_apply_multi_fp8 — bd_apply_multi with an e4m3 base:
 *     y[t] = W_hat x[t] + Delta_hat_{u(t)} x[t].
 * Same tenants, ids, output and status rules as bd_apply_multi; x is bf16 [batch][d_in].
 * The base product runs on the tensor cores in e4m3 x e4m3 with fp32 accumulation: each
 * x[t] is written as 2^e_t (hi + lo), hi and lo e4m3 and 2^e_t the power of two that puts
 * max|x[t]| in [128, 256). This is exact for bf16 values down to about max|x[t]| / 2^16;
 * smaller ones carry an error of at most 2^-10 * 2^e_t.
 *   w_codes  : device uint8 [d_out][d_in] (bd_quantize_base_fp8), 16-byte aligned.
 *   w_scales : device fp32 [d_out], 4-byte aligned.
 *   workspace: bd_apply_fp8_workspace_size() bytes. */
bd_status bd_apply_multi_fp8(const uint8_t* w_codes, const float* w_scales, int64_t d_out, int64_t d_in,
                             const bd_tenant* tenants, int32_t n_tenants, int32_t scale_dtype,
                             const int32_t* tenant_ids, const void* x, int64_t batch, void* y,
                             int32_t y_dtype, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------- */
/* status, diagnostics                                                                 */
/* ---------------------------------------------------------------------------------- */
/* Copies the device status word of a workspace (compress or apply) to *flags (host)
 * and SYNCHRONISES `stream`. Returns BD_ERR_INTERNAL, BD_ERR_TIMEOUT,
 * BD_ERR_TENANT_RECORD or BD_ERR_TENANT_RANGE (in that order of precedence) when the
 * corresponding bit is set, BD_OK when none is. */
bd_status bd_get_status(const void* workspace, uint32_t* flags /* host, may be NULL */,
                        void* stream);

/* Static description of a status code. */
const char* bd_status_string(int32_t status);

/* Kernel launch accounting: the number of kernels this library has launched since it
 * was loaded (all calls, all streams). */
int64_t bd_launch_count(void);

/* bd_selftest_wait_timeout — exercises the failure-detection path of the kernels'
 * bounded waits on the device, without a fault. The method's pages have no counterpart;
 * this is a test aid. It launches one kernel whose thread waits on a barrier that nothing
 * ever completes, through the same bounded wait the tensor-core kernels use; after
 * limit_cycles SM clock cycles the wait gives up, BD_DEV_TIMEOUT is set in the status
 * word of `workspace` (cleared first) and the kernel ends normally, so the context stays
 * usable. Read the outcome with bd_get_status (BD_ERR_TIMEOUT).
 *   workspace    : device, >= 256 bytes, 16-byte aligned (its status block is used).
 *   limit_cycles : 1 .. 4e9 (the kernels' own limit, ~2 s); BD_ERR_CONFIG otherwise. */
bd_status bd_selftest_wait_timeout(void* workspace, size_t ws_bytes, int64_t limit_cycles,
                                   void* stream);

/* Optional per-kernel timing. While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on its launch stream (at most `capacity`
 * launches are recorded; later ones are counted but not timed). bd_profile_collect
 * SYNCHRONISES on the recorded events, writes per kernel kind the number of timed
 * launches and their summed duration in milliseconds, clears the records and returns
 * the number of kernel kinds (array length written, <= max_kinds). */
bd_status bd_profile_enable(int32_t on, int32_t capacity);
int32_t bd_profile_collect(int64_t* launches /* host */, double* total_ms /* host */,
                           int32_t max_kinds);
const char* bd_kernel_name(int32_t kind);

#ifdef __cplusplus
}
#endif
#endif /* BITDELTA_H */
