// A8 — expert slot cache on the GPU over a pinned host pool (ExactMoE
// paper, Abstract: the experts live in pinned host memory and a slot cache
// of configurable size holds some of them on the GPU; Figure 1 caption: the
// host pool holds every packed expert, and a miss copies its packed codes and
// scales; Figure 2 caption: once the cache holds all experts no hit rate is
// counted; Table 1: slot counts 8/16/32/64 with hit rate and H2D traffic).
//
// Host side: one LRU per layer over `slots` device records. A miss evicts the
// least recently used slot that the current step does not need and is filled
// with one cudaMemcpyAsync of the expert's whole record (packed codes and
// scales, no dequantised copy) on a side stream. The layer's device table
// expert -> slot names exactly the experts of the last lookup; when a step
// needs more experts than there are slots (Figure 1 caption: the active
// experts run in waves sized to the cache), slot_cache_plan_waves splits it, and the
// step's experts outside the current wave are marked MOE_SLOT_SKIP, so each
// wave's grouped FFN call computes that wave's experts and no other. The table
// is rewritten by a one-block kernel on the compute stream, after the
// previous reader of the table, whose argument carries the whole table, so no
// host buffer has to outlive the call.
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace moe {

struct SlotTable {
  int32_t slot_of[MAX_E];
};

__global__ void write_slot_table_kernel(int32_t *dst, int E, const SlotTable table) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) dst[e] = table.slot_of[e];
}

}  // namespace moe

struct moe_slot_cache {
  int layers, E, slots;
  int64_t rec;
  const uint8_t *pool;
  uint8_t *dev_slots;
  int32_t *dev_table;
  bool resident;
  bool simulate;  // created without memory: policy and counters only
  // per layer
  std::vector<std::vector<int32_t>> owner;     // [layer][slot] expert or -1
  std::vector<std::vector<int32_t>> where;     // [layer][expert] slot or -1
  std::vector<std::vector<uint8_t>> loaded;    // [layer][expert] (resident mode)
  std::vector<std::vector<uint64_t>> stamp;    // [layer][slot] last step that used it
  std::vector<uint64_t> step;                  // [layer]
  std::vector<cudaEvent_t> released, filled;   // [layer], created on first use
  std::vector<bool> release_recorded;
  // misses of the last lookup per layer, for rollback if the fill fails
  std::vector<std::vector<int32_t>> pending_ids, pending_slots;
  std::vector<std::vector<int32_t>> step_ids;    // [layer] distinct ids of the last lookup
  std::vector<std::vector<uint8_t>> planned;     // [layer][expert] in the step last planned in waves
  std::vector<std::vector<int32_t>> table_host;  // [layer] the device table as last written (empty: unknown)
  uint64_t hits = 0, misses = 0, h2d_bytes = 0;
  int inject_fail = 0;
};

extern "C" int slot_cache_create(moe_slot_cache **out, int layers, int E, int slots, int64_t record_bytes,
                                 const void *pinned_pool, void *device_slots, int32_t *expert_slot) {
  using namespace moe;
  if (!out) return set_error(MOE_ERR_INVALID_ARG, "slot_cache_create: out is NULL");
  *out = nullptr;
  if (layers < 1 || E < 1 || E > MAX_E || slots < 1 || record_bytes < 256 || record_bytes % 256)
    return set_error(MOE_ERR_SHAPE, "slot_cache_create: layers=%d E=%d slots=%d record_bytes=%lld", layers, E, slots,
                     (long long)record_bytes);
  const bool simulate = !pinned_pool && !device_slots && !expert_slot;
  if (!simulate && (!pinned_pool || !device_slots || !expert_slot))
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_create: NULL pointer (pass all three memories, or none to "
                     "simulate the policy)");
  moe_slot_cache *c = new moe_slot_cache();
  c->layers = layers; c->E = E; c->slots = slots; c->rec = record_bytes;
  c->pool = static_cast<const uint8_t *>(pinned_pool);
  c->dev_slots = static_cast<uint8_t *>(device_slots);
  c->dev_table = expert_slot;
  c->resident = slots >= E;
  c->simulate = simulate;
  c->owner.assign(layers, std::vector<int32_t>(slots, -1));
  c->where.assign(layers, std::vector<int32_t>(E, -1));
  c->loaded.assign(layers, std::vector<uint8_t>(E, 0));
  c->stamp.assign(layers, std::vector<uint64_t>(slots, 0));
  c->step.assign(layers, 0);
  c->released.assign(layers, nullptr);
  c->filled.assign(layers, nullptr);
  c->release_recorded.assign(layers, false);
  c->pending_ids.assign(layers, {});
  c->pending_slots.assign(layers, {});
  c->step_ids.assign(layers, {});
  c->planned.assign(layers, std::vector<uint8_t>(E, 0));
  c->table_host.assign(layers, {});
  if (c->resident) {
    for (int l = 0; l < layers; ++l)
      for (int e = 0; e < E; ++e) { c->owner[l][e] = e; c->where[l][e] = e; }
  }
  *out = c;
  return MOE_OK;
}

// Undoes the slot assignments of the layer's last lookup whose records were
// never copied (a failed fill, or a lookup that no fill followed): those
// experts and their slots go back to empty, so a later lookup misses them
// again instead of reading a slot that holds stale bytes.
static void rollback(moe_slot_cache *c, int layer) {
  auto &ids = c->pending_ids[layer];
  auto &sl = c->pending_slots[layer];
  for (size_t i = 0; i < ids.size(); ++i) {
    if (c->resident) { c->loaded[layer][ids[i]] = 0; continue; }
    c->where[layer][ids[i]] = -1;
    c->owner[layer][sl[i]] = -1;
  }
  ids.clear();
  sl.clear();
}

extern "C" int slot_cache_lookup(moe_slot_cache *c, int layer, const int32_t *ids, int n, int32_t *slot_of_id,
                                 int32_t *miss_ids, int *n_miss) {
  moe::NvtxScope nvtx_scope("slot_cache_lookup");
  using namespace moe;
  if (!c || !n_miss || (n > 0 && (!ids || !slot_of_id || !miss_ids)))
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_lookup: NULL pointer");
  if (layer < 0 || layer >= c->layers || n < 0)
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_lookup: layer=%d n=%d", layer, n);
  *n_miss = 0;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->E) return set_error(MOE_ERR_INVALID_ARG, "slot_cache_lookup: id %d out of range", ids[i]);
  auto &owner = c->owner[layer];
  auto &where = c->where[layer];
  auto &stamp = c->stamp[layer];
  rollback(c, layer);  // the previous lookup's misses were never filled
  const uint64_t now = ++c->step[layer];

  // distinct ids, first occurrence order
  std::vector<int32_t> uniq;
  std::vector<uint8_t> seen(c->E, 0);
  for (int i = 0; i < n; ++i)
    if (!seen[ids[i]]) { seen[ids[i]] = 1; uniq.push_back(ids[i]); }
  if (int(uniq.size()) > c->slots)
    return set_error(MOE_ERR_CAPACITY, "slot_cache_lookup: %d distinct experts > %d slots (plan waves with "
                     "slot_cache_plan_waves)", int(uniq.size()), c->slots);
  c->step_ids[layer] = uniq;
  for (int32_t e : uniq)  // a lookup outside the planned step ends that plan
    if (!c->planned[layer][e]) { std::fill(c->planned[layer].begin(), c->planned[layer].end(), 0); break; }

  if (c->resident) {  // every expert owns its slot; only first touches load
    for (int32_t e : uniq)
      if (!c->loaded[layer][e]) {
        miss_ids[(*n_miss)++] = e;
        c->pending_ids[layer].push_back(e);
        c->pending_slots[layer].push_back(e);
        c->loaded[layer][e] = 1;
      }
    for (int i = 0; i < n; ++i) slot_of_id[i] = ids[i];
    return MOE_OK;
  }

  // hits first, so their slots are protected from eviction this step
  std::vector<int32_t> missing;
  for (int32_t e : uniq) {
    if (where[e] >= 0) { stamp[where[e]] = now; ++c->hits; }
    else missing.push_back(e);
  }
  for (int32_t e : missing) {
    int victim = -1;
    for (int s = 0; s < c->slots; ++s) {  // a free slot, else the least recently used
      if (stamp[s] == now) continue;
      if (owner[s] < 0) { victim = s; break; }
      if (victim < 0 || stamp[s] < stamp[victim]) victim = s;
    }
    if (victim < 0) return set_error(MOE_ERR_CAPACITY, "slot_cache_lookup: no evictable slot");
    if (owner[victim] >= 0) where[owner[victim]] = -1;
    owner[victim] = e;
    where[e] = victim;
    stamp[victim] = now;
    ++c->misses;
    miss_ids[(*n_miss)++] = e;
    c->pending_ids[layer].push_back(e);
    c->pending_slots[layer].push_back(victim);
  }
  for (int i = 0; i < n; ++i) slot_of_id[i] = where[ids[i]];
  return MOE_OK;
}

static int ensure_events(moe_slot_cache *c, int layer) {
  using namespace moe;
  if (!c->filled[layer]) {
    cudaError_t e = cudaEventCreateWithFlags(&c->filled[layer], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->released[layer], cudaEventDisableTiming);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "slot_cache: event creation: %s", cudaGetErrorString(e));
  }
  return MOE_OK;
}

extern "C" int slot_cache_fill(moe_slot_cache *c, int layer, const int32_t *miss_ids, int n_miss, moe_stream_t side,
                               moe_stream_t compute) {
  moe::NvtxScope nvtx_scope("slot_cache_fill");
  using namespace moe;
  if (!c || (n_miss > 0 && !miss_ids)) return set_error(MOE_ERR_INVALID_ARG, "slot_cache_fill: NULL pointer");
  if (layer < 0 || layer >= c->layers || n_miss < 0)
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_fill: layer=%d n_miss=%d", layer, n_miss);
  for (int i = 0; i < n_miss; ++i)
    if (miss_ids[i] < 0 || miss_ids[i] >= c->E || c->where[layer][miss_ids[i]] < 0)
      return set_error(MOE_ERR_INVALID_ARG, "slot_cache_fill: id %d was not assigned a slot by slot_cache_lookup",
                       miss_ids[i]);
  if (n_miss > 0 && c->inject_fail > 0) {
    --c->inject_fail;
    rollback(c, layer);
    return set_error(MOE_ERR_CUDA, "slot_cache_fill: injected fill failure (layer %d)", layer);
  }
  // the table the FFN reads: the last lookup's experts in their slots, the
  // other experts of a step planned in waves skipped, every other expert
  // absent (-1: flagged if a token selects it)
  std::vector<int32_t> table(c->E, -1);
  for (int x = 0; x < c->E; ++x)
    if (c->planned[layer][x]) table[x] = MOE_SLOT_SKIP;
  for (int32_t x : c->step_ids[layer]) table[x] = c->where[layer][x];
  const bool table_changed = table != c->table_host[layer];
  if (c->simulate) {  // no memory: the misses count as copied
    c->h2d_bytes += uint64_t(n_miss) * uint64_t(c->rec);
    c->pending_ids[layer].clear();
    c->pending_slots[layer].clear();
    c->table_host[layer] = table;
    return MOE_OK;
  }
  if (n_miss == 0 && !table_changed) return MOE_OK;
  cudaStream_t s = as_stream(side), cs = as_stream(compute);
  cudaError_t e = cudaSuccess;
  if (n_miss > 0) {
    int st = ensure_events(c, layer);
    if (st != MOE_OK) { rollback(c, layer); return st; }
    if (c->release_recorded[layer]) e = cudaStreamWaitEvent(s, c->released[layer], 0);
    for (int i = 0; i < n_miss && e == cudaSuccess; ++i) {
      const int id = miss_ids[i];
      const int slot = c->where[layer][id];
      uint8_t *dst = c->dev_slots + (int64_t(layer) * c->slots + slot) * c->rec;
      const uint8_t *src = c->pool + (int64_t(layer) * c->E + id) * c->rec;
      e = cudaMemcpyAsync(dst, src, size_t(c->rec), cudaMemcpyHostToDevice, s);
    }
    if (e != cudaSuccess) {
      rollback(c, layer);
      return set_error(MOE_ERR_CUDA, "slot_cache_fill: copy: %s", cudaGetErrorString(e));
    }
    e = cudaEventRecord(c->filled[layer], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, c->filled[layer], 0);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "slot_cache_fill: %s", cudaGetErrorString(e));
    c->h2d_bytes += uint64_t(n_miss) * uint64_t(c->rec);
  }
  c->pending_ids[layer].clear();
  c->pending_slots[layer].clear();
  if (table_changed) {
    SlotTable t;
    for (int x = 0; x < c->E; ++x) t.slot_of[x] = table[x];
    write_slot_table_kernel<<<1, 256, 0, cs>>>(c->dev_table + int64_t(layer) * c->E, c->E, t);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      c->table_host[layer].clear();
      return set_error(MOE_ERR_CUDA, "slot_cache_fill: table: %s", cudaGetErrorString(e));
    }
    count_launches(1);
    c->table_host[layer] = table;
  }
  return MOE_OK;
}

extern "C" int slot_cache_plan_waves(moe_slot_cache *c, int layer, const int32_t *ids, int n,
                                     int32_t *wave_ids, int32_t *wave_start, int *n_waves) {
  moe::NvtxScope nvtx_scope("slot_cache_plan_waves");
  using namespace moe;
  if (!c || !n_waves || (n > 0 && (!ids || !wave_ids || !wave_start)))
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_plan_waves: NULL pointer");
  if (layer < 0 || layer >= c->layers || n < 0)
    return set_error(MOE_ERR_INVALID_ARG, "slot_cache_plan_waves: layer=%d n=%d", layer, n);
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->E)
      return set_error(MOE_ERR_INVALID_ARG, "slot_cache_plan_waves: id %d out of range", ids[i]);
  *n_waves = 0;
  if (n == 0) return MOE_OK;
  // distinct ids, first occurrence order; those whose records are in a slot
  // (copied by a completed fill) come first, so they run before any eviction
  std::vector<uint8_t> seen(c->E, 0), pending(c->E, 0);
  for (int32_t x : c->pending_ids[layer]) pending[x] = 1;
  std::vector<int32_t> held, absent;
  for (int i = 0; i < n; ++i) {
    const int x = ids[i];
    if (seen[x]) continue;
    seen[x] = 1;
    const bool in_slot = c->resident ? c->loaded[layer][x] != 0 : c->where[layer][x] >= 0;
    (in_slot && !pending[x] ? held : absent).push_back(x);
  }
  int m = 0;
  for (int32_t x : held) wave_ids[m++] = x;
  for (int32_t x : absent) wave_ids[m++] = x;
  for (int x = 0; x < c->E; ++x) c->planned[layer][x] = seen[x];
  int w = 0;
  for (int start = 0; start < m; start += c->slots) wave_start[w++] = start;
  wave_start[w] = m;
  *n_waves = w;
  return MOE_OK;
}

extern "C" int slot_cache_release(moe_slot_cache *c, int layer, moe_stream_t compute) {
  moe::NvtxScope nvtx_scope("slot_cache_release");
  using namespace moe;
  if (!c || layer < 0 || layer >= c->layers) return set_error(MOE_ERR_INVALID_ARG, "slot_cache_release: bad argument");
  if (c->simulate) return MOE_OK;
  int st = ensure_events(c, layer);
  if (st != MOE_OK) return st;
  cudaError_t e = cudaEventRecord(c->released[layer], as_stream(compute));
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "slot_cache_release: %s", cudaGetErrorString(e));
  c->release_recorded[layer] = true;
  return MOE_OK;
}

extern "C" int slot_cache_stats(const moe_slot_cache *c, uint64_t *hits, uint64_t *misses, uint64_t *h2d_bytes) {
  if (!c) return moe::set_error(MOE_ERR_INVALID_ARG, "slot_cache_stats: NULL cache");
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (h2d_bytes) *h2d_bytes = c->h2d_bytes;
  return MOE_OK;
}

extern "C" int slot_cache_inject_fill_failure(moe_slot_cache *c, int count) {
  if (!c || count < 0) return moe::set_error(MOE_ERR_INVALID_ARG, "slot_cache_inject_fill_failure: bad argument");
  c->inject_fail = count;
  return MOE_OK;
}

extern "C" void slot_cache_destroy(moe_slot_cache *c) {
  if (!c) return;
  for (cudaEvent_t ev : c->filled) if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : c->released) if (ev) cudaEventDestroy(ev);
  delete c;
}
