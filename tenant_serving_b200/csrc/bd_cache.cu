// Host-resident tenant cache and packed-delta loader.
//
// "Per-Axis Weight Deltas", Key Contributions item 4 and Implementation details: a
// tenant's packed module (1-bit signs packed along the input axis plus its fp16 scale
// vector) moves to the GPU in a single non-blocking transfer per module, without dense
// reconstruction. "BitDelta Guide", "3. Dynamic Model Hot-Swapping and Multi-Tenant
// Batching": deltas are pre-cached in GPU memory or streamed from host CPU memory.
//
// Design. Every tenant lives in host memory as one packed record per module (layer x
// projection): the serving layout's tiled sign words followed by its scales, so one
// cudaMemcpyAsync moves one module. The GPU holds n_slots tenant slots in a caller-owned
// device pool; slot s's record of module m always sits at the same device address, and a
// device table per module (n_slots bd_tenant records, at the start of the pool) is what
// bd_apply_multi reads. A batch is mapped onto slots by its composition: resident tenants
// are hits, missing ones evict the least recently used slot that no unreleased batch
// holds. Loads go on a copy stream; a batch's compute stream waits for its own loads
// only (acquire), and a slot's old contents are overwritten only after the compute
// stream has finished the last batch that read them (release).
#include "bd_internal.cuh"

#include <cstring>
#include <new>
#include <vector>

namespace bd {
size_t prepared_signs_bytes(int64_t d_out, int64_t d_in);
size_t prepared_scales_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t G, int32_t sdt);
}  // namespace bd

struct bd_cache {
  struct Module {
    int64_t d_out, d_in;
    int32_t min_group;
    size_t signs_bytes, region_bytes, offset;  // offset of the module's region in a slot
  };
  struct Entry {
    const void* host = nullptr;  // packed record in host memory
    int32_t mode = -1, group_size = 0;
    size_t bytes = 0;
  };
  std::vector<Module> mods;
  int32_t scale_dtype = BD_F16;
  int32_t n_host = 0, n_slots = 0;
  uint8_t* pool = nullptr;
  size_t pool_bytes = 0, tables_bytes = 0, slot_bytes = 0;
  uint8_t* staging = nullptr;  // two pinned copies of the tables (double buffered)
  std::vector<Entry> entries;  // [tenant][module]
  std::vector<bd_tenant> tables;  // authoritative host copy, [module][slot]
  // slot state
  std::vector<int32_t> slot_tenant;  // -1: empty
  std::vector<int64_t> slot_stamp;   // batch sequence number of the last use (-1: never)
  std::vector<int64_t> slot_hold;    // ticket holding the slot until its release (-1: none)
  std::vector<int32_t> slot_done;    // release event index of the last batch that read it (-1: none)
  std::vector<int32_t> tenant_slot;  // -1: not resident
  // tickets (batches assigned and not yet released)
  static constexpr int kTickets = 4;
  int64_t next_ticket = 0;
  bool ticket_open[kTickets] = {false, false, false, false};
  int64_t ticket_id[kTickets] = {-1, -1, -1, -1};
  std::vector<int32_t> ticket_slots[kTickets];
  // CUDA events, created on first use (the host logic needs no device)
  bool events_ready = false;
  cudaEvent_t ready_ev[kTickets] = {}, done_ev[kTickets] = {}, mirror_ev[2] = {};
  bool mirror_pending[2] = {false, false};
  int mirror_next = 0;
  // statistics
  int64_t hits = 0, misses = 0, bytes_loaded = 0, copies = 0;
};

namespace {

constexpr size_t kRegionAlign = 256;

size_t record_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t G, int32_t sdt) {
  return bd::align_up(bd::prepared_signs_bytes(d_out, d_in), 16) +
         bd::prepared_scales_bytes(d_out, d_in, mode, G, sdt);
}

bool shape_ok(int64_t d_out, int64_t d_in) { return d_out >= 1 && d_in >= 32 && (d_in % 32) == 0; }

bool mode_ok(int64_t d_in, int32_t mode, int32_t G) { return bd::scale_mode_ok(mode, G, d_in); }

// The largest record a tenant of this module may have: every scale mode, group sizes from
// min_group up to d_in.
size_t region_bytes(int64_t d_out, int64_t d_in, int32_t min_group, int32_t sdt) {
  size_t m = 0;
  for (int32_t mode = BD_SCALE_ROW; mode <= BD_SCALE_TENSOR; ++mode) {
    const size_t b = record_bytes(d_out, d_in, mode, 0, sdt);
    if (b > m) m = b;
  }
  for (int64_t G = min_group; G <= d_in; G *= 2) {
    if (d_in % G) continue;
    for (int32_t mode : {(int32_t)BD_SCALE_GROUP, (int32_t)BD_SCALE_BLOCK}) {
      const size_t b = record_bytes(d_out, d_in, mode, (int32_t)G, sdt);
      if (b > m) m = b;
    }
  }
  return bd::align_up(m, kRegionAlign);
}

bool layout_modules(const bd_cache_module* modules, int32_t n_modules, int32_t sdt,
                    std::vector<bd_cache::Module>* out, size_t* slot_bytes) {
  size_t off = 0;
  for (int32_t m = 0; m < n_modules; ++m) {
    const bd_cache_module& M = modules[m];
    if (!shape_ok(M.d_out, M.d_in)) return false;
    if (M.min_group_size != 0 && !mode_ok(M.d_in, BD_SCALE_GROUP, M.min_group_size)) return false;
    bd_cache::Module mm;
    mm.d_out = M.d_out;
    mm.d_in = M.d_in;
    mm.min_group = M.min_group_size ? M.min_group_size : (int32_t)M.d_in;  // 0: no GROUP records
    mm.signs_bytes = bd::align_up(bd::prepared_signs_bytes(M.d_out, M.d_in), 16);
    mm.region_bytes = region_bytes(M.d_out, M.d_in, mm.min_group, sdt);
    mm.offset = off;
    off += mm.region_bytes;
    if (out) out->push_back(mm);
  }
  *slot_bytes = off;
  return true;
}

size_t tables_bytes_for(int32_t n_modules, int32_t n_slots) {
  return bd::align_up((size_t)n_modules * (size_t)n_slots * sizeof(bd_tenant), kRegionAlign);
}

bool ensure_events(bd_cache* c) {
  if (c->events_ready) return true;
  for (int i = 0; i < bd_cache::kTickets; ++i) {
    if (cudaEventCreateWithFlags(&c->ready_ev[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->done_ev[i], cudaEventDisableTiming) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
  }
  for (int i = 0; i < 2; ++i)
    if (cudaEventCreateWithFlags(&c->mirror_ev[i], cudaEventDisableTiming) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
  c->events_ready = true;
  return true;
}

int ticket_index(const bd_cache* c, int64_t ticket) {
  for (int i = 0; i < bd_cache::kTickets; ++i)
    if (c->ticket_open[i] && c->ticket_id[i] == ticket) return i;
  return -1;
}

}  // namespace

// ------------------------------------------------------------------------------------
// host-side record preparation
// ------------------------------------------------------------------------------------
extern "C" size_t bd_cache_record_bytes(int64_t d_out, int64_t d_in, int32_t mode, int32_t group_size,
                                        int32_t scale_dtype) {
  if (!shape_ok(d_out, d_in) || !mode_ok(d_in, mode, group_size)) return 0;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return 0;
  return record_bytes(d_out, d_in, mode, group_size, scale_dtype);
}

extern "C" bd_status bd_prepare_record_host(const uint32_t* signs, const void* scales, int32_t scale_dtype,
                                            int32_t mode, int32_t group_size, int64_t d_out, int64_t d_in,
                                            void* record, size_t record_bytes_given) {
  if (!signs || !scales || !record) return BD_ERR_NULL;
  if (!shape_ok(d_out, d_in)) return BD_ERR_SHAPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if (!mode_ok(d_in, mode, group_size)) return BD_ERR_CONFIG;
  const size_t need = record_bytes(d_out, d_in, mode, group_size, scale_dtype);
  if (record_bytes_given < need) return BD_ERR_WORKSPACE;
  // signs: tiles of 512 rows x 8 words, tile (rb, w) at word (rb * nwin + w) * 4096
  const int64_t wpr = d_in / 32, nwin = (d_in + 255) / 256, nrt = (d_out + 511) / 512;
  uint32_t* out = static_cast<uint32_t*>(record);
  for (int64_t rb = 0; rb < nrt; ++rb)
    for (int64_t w = 0; w < nwin; ++w) {
      uint32_t* tile = out + (rb * nwin + w) * 4096;
      for (int64_t r = 0; r < 512; ++r) {
        const int64_t row = rb * 512 + r;
        for (int64_t k = 0; k < 8; ++k) {
          const int64_t word = w * 8 + k;
          tile[r * 8 + k] = (row < d_out && word < wpr) ? signs[row * wpr + word] : 0u;
        }
      }
    }
  const size_t sb = bd::align_up(bd::prepared_signs_bytes(d_out, d_in), 16);
  std::memset(static_cast<uint8_t*>(record) + bd::prepared_signs_bytes(d_out, d_in), 0,
              sb - bd::prepared_signs_bytes(d_out, d_in));
  uint8_t* sc_out = static_cast<uint8_t*>(record) + sb;
  const size_t ssz = scale_dtype == BD_F16 ? 2 : 4;
  const size_t sc_bytes = bd::prepared_scales_bytes(d_out, d_in, mode, group_size, scale_dtype);
  std::memset(sc_out, 0, sc_bytes);
  const uint8_t* sc_in = static_cast<const uint8_t*>(scales);
  if (mode == BD_SCALE_GROUP && group_size == 128) {
    // tile (rb, w): [row 0..511][2 groups] at element (rb * nwin + w) * 1024
    const int64_t gpr = d_in / 128;
    for (int64_t rb = 0; rb < nrt; ++rb)
      for (int64_t w = 0; w < nwin; ++w)
        for (int64_t r = 0; r < 512; ++r)
          for (int64_t k = 0; k < 2; ++k) {
            const int64_t row = rb * 512 + r, g = w * 2 + k;
            if (row < d_out && g < gpr)
              std::memcpy(sc_out + ((rb * nwin + w) * 1024 + r * 2 + k) * ssz, sc_in + (row * gpr + g) * ssz, ssz);
          }
  } else {
    const size_t n = (size_t)bd::scale_count(mode, group_size, d_out, d_in);
    std::memcpy(sc_out, sc_in, n * ssz);
  }
  return BD_OK;
}

// ------------------------------------------------------------------------------------
// the cache
// ------------------------------------------------------------------------------------
extern "C" size_t bd_cache_pool_bytes(const bd_cache_module* modules, int32_t n_modules, int32_t n_slots,
                                      int32_t scale_dtype) {
  if (!modules || n_modules < 1 || n_slots < 1) return 0;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return 0;
  size_t slot = 0;
  if (!layout_modules(modules, n_modules, scale_dtype, nullptr, &slot)) return 0;
  return tables_bytes_for(n_modules, n_slots) + slot * (size_t)n_slots;
}

extern "C" size_t bd_cache_staging_bytes(int32_t n_modules, int32_t n_slots) {
  if (n_modules < 1 || n_slots < 1) return 0;
  return 2 * tables_bytes_for(n_modules, n_slots);
}

extern "C" bd_status bd_cache_create(const bd_cache_module* modules, int32_t n_modules, int32_t scale_dtype,
                                     int32_t n_host_tenants, int32_t n_slots, void* pool, size_t pool_bytes,
                                     void* staging, size_t staging_bytes, bd_cache** out) {
  if (!out) return BD_ERR_NULL;
  *out = nullptr;
  if (!modules || !pool || !staging) return BD_ERR_NULL;
  if (n_modules < 1 || n_host_tenants < 1 || n_slots < 1) return BD_ERR_SHAPE;
  if (scale_dtype != BD_F16 && scale_dtype != BD_F32) return BD_ERR_DTYPE;
  if ((reinterpret_cast<uintptr_t>(pool) & (kRegionAlign - 1)) != 0 || !bd::aligned16(staging)) return BD_ERR_ALIGN;
  bd_cache* c = new (std::nothrow) bd_cache();
  if (!c) return BD_ERR_INTERNAL;
  if (!layout_modules(modules, n_modules, scale_dtype, &c->mods, &c->slot_bytes)) {
    delete c;
    return BD_ERR_SHAPE;
  }
  c->tables_bytes = tables_bytes_for(n_modules, n_slots);
  const size_t need = c->tables_bytes + c->slot_bytes * (size_t)n_slots;
  if (pool_bytes < need || staging_bytes < 2 * c->tables_bytes) {
    delete c;
    return BD_ERR_WORKSPACE;
  }
  c->scale_dtype = scale_dtype;
  c->n_host = n_host_tenants;
  c->n_slots = n_slots;
  c->pool = static_cast<uint8_t*>(pool);
  c->pool_bytes = pool_bytes;
  c->staging = static_cast<uint8_t*>(staging);
  c->entries.assign((size_t)n_host_tenants * n_modules, bd_cache::Entry());
  c->slot_tenant.assign(n_slots, -1);
  c->slot_stamp.assign(n_slots, -1);
  c->slot_hold.assign(n_slots, -1);
  c->slot_done.assign(n_slots, -1);
  c->tenant_slot.assign(n_host_tenants, -1);
  // every record points at its slot's region: valid (GROUP with the module's G, or ROW)
  // though never read before a tenant is loaded there
  c->tables.resize((size_t)n_modules * n_slots);
  for (int32_t m = 0; m < n_modules; ++m)
    for (int32_t s = 0; s < n_slots; ++s) {
      const bd_cache::Module& M = c->mods[m];
      uint8_t* base = c->pool + c->tables_bytes + (size_t)s * c->slot_bytes + M.offset;
      bd_tenant& t = c->tables[(size_t)m * n_slots + s];
      t.signs = reinterpret_cast<const uint32_t*>(base);
      t.scales = base + M.signs_bytes;
      t.mode = BD_SCALE_ROW;
      t.group_size = 0;
      t.layout = BD_LAYOUT_TILED;
      t.reserved = 0;
    }
  *out = c;
  return BD_OK;
}

extern "C" bd_status bd_cache_destroy(bd_cache* c) {
  if (!c) return BD_ERR_NULL;
  bd_status st = BD_OK;
  if (c->events_ready) {
    // copies may still read the host records and the staging tables
    for (int i = 0; i < 2; ++i)
      if (cudaEventSynchronize(c->mirror_ev[i]) != cudaSuccess) st = BD_ERR_CUDA;
    for (int i = 0; i < bd_cache::kTickets; ++i) {
      if (cudaEventSynchronize(c->ready_ev[i]) != cudaSuccess) st = BD_ERR_CUDA;
      cudaEventDestroy(c->ready_ev[i]);
      cudaEventDestroy(c->done_ev[i]);
    }
    for (int i = 0; i < 2; ++i) cudaEventDestroy(c->mirror_ev[i]);
    (void)cudaGetLastError();
  }
  delete c;
  return st;
}

extern "C" bd_status bd_cache_register(bd_cache* c, int32_t tenant, int32_t module, const void* record_host,
                                       int32_t mode, int32_t group_size) {
  if (!c || !record_host) return BD_ERR_NULL;
  if (tenant < 0 || tenant >= c->n_host) return BD_ERR_TENANT_RANGE;
  if (module < 0 || module >= (int32_t)c->mods.size()) return BD_ERR_SHAPE;
  const bd_cache::Module& M = c->mods[module];
  if (!mode_ok(M.d_in, mode, group_size)) return BD_ERR_CONFIG;
  if ((mode == BD_SCALE_GROUP || mode == BD_SCALE_BLOCK) && group_size < M.min_group) return BD_ERR_CONFIG;
  if (!bd::aligned16(record_host)) return BD_ERR_ALIGN;
  if (c->tenant_slot[tenant] >= 0) return BD_ERR_CONFIG;  // resident: its slot still holds the old record
  bd_cache::Entry& e = c->entries[(size_t)tenant * c->mods.size() + module];
  e.host = record_host;
  e.mode = mode;
  e.group_size = (mode == BD_SCALE_GROUP || mode == BD_SCALE_BLOCK) ? group_size : 0;
  e.bytes = record_bytes(M.d_out, M.d_in, mode, group_size, c->scale_dtype);
  return BD_OK;
}

extern "C" const bd_tenant* bd_cache_table(const bd_cache* c, int32_t module) {
  if (!c || module < 0 || module >= (int32_t)c->mods.size()) return nullptr;
  return reinterpret_cast<const bd_tenant*>(c->pool) + (size_t)module * c->n_slots;
}

extern "C" int32_t bd_cache_slots(const bd_cache* c) { return c ? c->n_slots : 0; }

extern "C" bd_status bd_cache_assign(bd_cache* c, const int32_t* tenant_ids, int64_t batch, int32_t* slot_ids,
                                     int32_t* loads, int32_t* n_loads, int64_t* ticket) {
  if (!c || !n_loads || !ticket || (batch > 0 && (!tenant_ids || !slot_ids))) return BD_ERR_NULL;
  if (batch < 0) return BD_ERR_SHAPE;
  *n_loads = 0;
  *ticket = -1;
  int free_ticket = -1;
  for (int i = 0; i < bd_cache::kTickets; ++i)
    if (!c->ticket_open[i]) {
      free_ticket = i;
      break;
    }
  if (free_ticket < 0) return BD_ERR_CONFIG;  // too many batches assigned and not released
  const int32_t nm = (int32_t)c->mods.size();
  // validate everything before any state changes
  std::vector<int32_t> distinct;
  std::vector<uint8_t> seen(c->n_host, 0);
  for (int64_t t = 0; t < batch; ++t) {
    const int32_t u = tenant_ids[t];
    if (u == -1) continue;
    if (u < 0 || u >= c->n_host) return BD_ERR_TENANT_RANGE;
    if (seen[u]) continue;
    seen[u] = 1;
    for (int32_t m = 0; m < nm; ++m)
      if (!c->entries[(size_t)u * nm + m].host) return BD_ERR_TENANT_RECORD;
    distinct.push_back(u);
  }
  // slots this batch may not take: held by unreleased batches, or holding a tenant of
  // this batch
  const int64_t stamp = c->next_ticket;
  std::vector<uint8_t> taken(c->n_slots, 0);
  int32_t need = 0;
  for (int32_t u : distinct) {
    if (c->tenant_slot[u] >= 0) taken[c->tenant_slot[u]] = 1;
    else ++need;
  }
  std::vector<int32_t> victims;
  if (need > 0) {
    // least recently used first (never-used slots have stamp -1), lowest index on ties
    std::vector<int32_t> cand;
    for (int32_t s = 0; s < c->n_slots; ++s)
      if (!taken[s] && c->slot_hold[s] < 0) cand.push_back(s);
    if ((int32_t)cand.size() < need) return BD_ERR_CONFIG;  // not enough free slots
    for (int32_t k = 0; k < need; ++k) {
      int best = -1;
      for (int i = 0; i < (int)cand.size(); ++i) {
        if (cand[i] < 0) continue;
        if (best < 0 || c->slot_stamp[cand[i]] < c->slot_stamp[cand[best]]) best = i;
      }
      victims.push_back(cand[best]);
      cand[best] = -1;
    }
  }
  // commit
  std::vector<int32_t>& held = c->ticket_slots[free_ticket];
  held.clear();
  int32_t nv = 0;
  for (int32_t u : distinct) {
    int32_t s = c->tenant_slot[u];
    if (s >= 0) {
      ++c->hits;
    } else {
      s = victims[nv++];
      const int32_t old = c->slot_tenant[s];
      if (old >= 0) c->tenant_slot[old] = -1;
      c->slot_tenant[s] = u;
      c->tenant_slot[u] = s;
      if (loads) {
        loads[2 * (*n_loads)] = u;
        loads[2 * (*n_loads) + 1] = s;
      }
      ++*n_loads;
      ++c->misses;
      for (int32_t m = 0; m < nm; ++m) {
        const bd_cache::Entry& e = c->entries[(size_t)u * nm + m];
        bd_tenant& rec = c->tables[(size_t)m * c->n_slots + s];
        rec.mode = e.mode;
        rec.group_size = e.group_size;
      }
    }
    c->slot_stamp[s] = stamp;
    c->slot_hold[s] = stamp;
    held.push_back(s);
  }
  for (int64_t t = 0; t < batch; ++t) {
    const int32_t u = tenant_ids[t];
    slot_ids[t] = u == -1 ? -1 : c->tenant_slot[u];
  }
  c->ticket_open[free_ticket] = true;
  c->ticket_id[free_ticket] = stamp;
  c->next_ticket++;
  *ticket = stamp;
  return BD_OK;
}

namespace {
// Undo a batch whose copies could not all be issued: its loaded slots become empty (their
// contents are unknown) and its ticket is closed without a release event.
void drop_batch(bd_cache* c, int64_t ticket, const std::vector<int32_t>& loads, int32_t n_loads) {
  for (int32_t k = 0; k < n_loads; ++k) {
    const int32_t u = loads[2 * k], slot = loads[2 * k + 1];
    c->tenant_slot[u] = -1;
    c->slot_tenant[slot] = -1;
    c->slot_stamp[slot] = -1;
  }
  const int ti = ticket_index(c, ticket);
  if (ti < 0) return;
  for (int32_t s : c->ticket_slots[ti])
    if (c->slot_hold[s] == ticket) c->slot_hold[s] = -1;
  c->ticket_open[ti] = false;
  c->ticket_slots[ti].clear();
}

bd_status issue_loads(bd_cache* c, const std::vector<int32_t>& loads, int32_t n_loads, int ti, cudaStream_t s) {
  const int32_t nm = (int32_t)c->mods.size();
  for (int32_t k = 0; k < n_loads; ++k) {
    const int32_t u = loads[2 * k], slot = loads[2 * k + 1];
    // the slot's previous contents are overwritten only after the last batch that read
    // them has finished on its compute stream
    if (c->slot_done[slot] >= 0) BD_CUDA_TRY(cudaStreamWaitEvent(s, c->done_ev[c->slot_done[slot]], 0));
    uint8_t* base = c->pool + c->tables_bytes + (size_t)slot * c->slot_bytes;
    for (int32_t m = 0; m < nm; ++m) {
      const bd_cache::Entry& e = c->entries[(size_t)u * nm + m];
      // one transfer per module: its tiled signs and its scales together
      BD_CUDA_TRY(cudaMemcpyAsync(base + c->mods[m].offset, e.host, e.bytes, cudaMemcpyHostToDevice, s));
      c->bytes_loaded += (int64_t)e.bytes;
      c->copies++;
    }
  }
  if (n_loads > 0) {
    // the device tables: the authoritative host copy through one of two pinned buffers
    const int b = c->mirror_next;
    c->mirror_next ^= 1;
    if (c->mirror_pending[b]) BD_CUDA_TRY(cudaEventSynchronize(c->mirror_ev[b]));
    uint8_t* mirror = c->staging + (size_t)b * c->tables_bytes;
    const size_t tb = c->tables.size() * sizeof(bd_tenant);
    std::memcpy(mirror, c->tables.data(), tb);
    BD_CUDA_TRY(cudaMemcpyAsync(c->pool, mirror, tb, cudaMemcpyHostToDevice, s));
    BD_CUDA_TRY(cudaEventRecord(c->mirror_ev[b], s));
    c->mirror_pending[b] = true;
    c->copies++;
  }
  BD_CUDA_TRY(cudaEventRecord(c->ready_ev[ti], s));
  return BD_OK;
}
}  // namespace

extern "C" bd_status bd_cache_prefetch(bd_cache* c, const int32_t* tenant_ids, int64_t batch, int32_t* slot_ids,
                                       int32_t* n_loads, int64_t* ticket, void* copy_stream) {
  if (!c || !n_loads || !ticket) return BD_ERR_NULL;
  if (!ensure_events(c)) return BD_ERR_CUDA;
  std::vector<int32_t> loads(2 * (size_t)c->n_slots);
  const bd_status st = bd_cache_assign(c, tenant_ids, batch, slot_ids, loads.data(), n_loads, ticket);
  if (st != BD_OK) return st;
  const bd_status st2 = issue_loads(c, loads, *n_loads, ticket_index(c, *ticket), static_cast<cudaStream_t>(copy_stream));
  if (st2 != BD_OK) {
    drop_batch(c, *ticket, loads, *n_loads);
    *ticket = -1;
  }
  return st2;
}

extern "C" bd_status bd_cache_acquire(bd_cache* c, int64_t ticket, void* compute_stream) {
  if (!c) return BD_ERR_NULL;
  const int ti = ticket_index(c, ticket);
  if (ti < 0) return BD_ERR_CONFIG;
  if (!c->events_ready) return BD_OK;  // no copy was ever issued (assign-only use)
  BD_CUDA_TRY(cudaStreamWaitEvent(static_cast<cudaStream_t>(compute_stream), c->ready_ev[ti], 0));
  return BD_OK;
}

extern "C" bd_status bd_cache_release(bd_cache* c, int64_t ticket, void* compute_stream) {
  if (!c) return BD_ERR_NULL;
  const int ti = ticket_index(c, ticket);
  if (ti < 0) return BD_ERR_CONFIG;
  if (c->events_ready) BD_CUDA_TRY(cudaEventRecord(c->done_ev[ti], static_cast<cudaStream_t>(compute_stream)));
  for (int32_t s : c->ticket_slots[ti]) {
    if (c->events_ready) c->slot_done[s] = ti;
    if (c->slot_hold[s] == ticket) c->slot_hold[s] = -1;
  }
  // a slot also held by another unreleased batch keeps that hold
  for (int i = 0; i < bd_cache::kTickets; ++i)
    if (i != ti && c->ticket_open[i])
      for (int32_t s : c->ticket_slots[i])
        if (c->slot_hold[s] < 0) c->slot_hold[s] = c->ticket_id[i];
  c->ticket_open[ti] = false;
  c->ticket_slots[ti].clear();
  return BD_OK;
}

extern "C" bd_status bd_cache_resident(const bd_cache* c, int32_t* slot_tenant, int64_t* stats) {
  if (!c) return BD_ERR_NULL;
  if (slot_tenant)
    for (int32_t s = 0; s < c->n_slots; ++s) slot_tenant[s] = c->slot_tenant[s];
  if (stats) {
    stats[0] = c->hits;
    stats[1] = c->misses;
    stats[2] = c->bytes_loaded;
    stats[3] = c->copies;
  }
  return BD_OK;
}
