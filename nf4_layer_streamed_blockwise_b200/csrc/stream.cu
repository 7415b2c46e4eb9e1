// Layer-streaming scheduler: page-locked host layer records -> a ring of HBM
// slots on a copy stream, ordered against the compute stream with events only
// (no host synchronisation inside a training step).
//
// Invariants:
//  * a slot is overwritten only after the compute stream has passed the point
//    where the slot's previous occupant was released (slot_free event);
//  * compute on a layer starts only after that layer's upload completed
//    (up_done event);
//  * the layer currently being computed is never evicted.
// The pages' design (a pair of GPU buffers allocated up front, stream_buffers
// 2..8, a page-locked store so that the copy overlaps compute) is kept; their
// silent fallback to pageable memory becomes LSQ_ENOTPINNED.
#include <vector>

#include "host_common.h"

struct lsq_stream {
  int n_layers = 0, n_slots = 0;
  size_t record_bytes = 0;
  std::vector<void*> slots;
  std::vector<const void*> host;
  cudaStream_t compute = nullptr, copy = nullptr;
  std::vector<int> slot_layer;         // layer held by a slot, -1 if none
  std::vector<int64_t> slot_tick;      // last step() use, for LRU
  std::vector<int> layer_slot;         // slot holding a layer, -1 if none
  std::vector<char> used_since_upload; // stepped since its last upload
  std::vector<char> free_recorded;     // slot_free[slot] has been recorded
  std::vector<cudaEvent_t> up_start, up_done, slot_free;
  int cur = -1;  // layer of the last step()
  int64_t tick = 0, uploads = 0, bytes = 0, reused = 0;
};

namespace lsq {
namespace sched {

static lsq_status upload(lsq_stream* st, int layer, int slot) {
  const int old = st->slot_layer[slot];
  if (old >= 0) st->layer_slot[old] = -1;
  if (st->free_recorded[slot]) LSQ_CUDA_TRY(cudaStreamWaitEvent(st->copy, st->slot_free[slot], 0));
  LSQ_CUDA_TRY(cudaEventRecord(st->up_start[layer], st->copy));
  LSQ_CUDA_TRY(cudaMemcpyAsync(st->slots[slot], st->host[layer], st->record_bytes, cudaMemcpyHostToDevice, st->copy));
  LSQ_CUDA_TRY(cudaEventRecord(st->up_done[layer], st->copy));
  st->slot_layer[slot] = layer;
  st->layer_slot[layer] = slot;
  st->used_since_upload[layer] = 0;
  st->uploads += 1;
  st->bytes += (int64_t)st->record_bytes;
  return LSQ_OK;
}

// an empty slot if any, else the least recently used one; `keep` is excluded
static int victim(const lsq_stream* st, int keep) {
  int best = -1;
  for (int s = 0; s < st->n_slots; ++s) {
    if (s == keep) continue;
    if (st->slot_layer[s] < 0) return s;
    if (best < 0 || st->slot_tick[s] < st->slot_tick[best]) best = s;
  }
  return best;
}

static bool is_pinned_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

static void destroy_events(lsq_stream* st) {
  for (auto* v : {&st->up_start, &st->up_done, &st->slot_free})
    for (cudaEvent_t e : *v)
      if (e) cudaEventDestroy(e);
}

}  // namespace sched
}  // namespace lsq

using namespace lsq;
using namespace lsq::sched;

extern "C" lsq_status lsq_stream_create(const lsq_stream_cfg* cfg, lsq_cuda_stream compute, lsq_cuda_stream copy,
                                        lsq_stream** out) {
  if (!cfg || !out || !cfg->slots || !cfg->host_records) return fail(LSQ_EINVAL, "lsq_stream_create: NULL argument");
  *out = nullptr;
  if (cfg->n_layers < 1 || cfg->record_bytes == 0) return fail(LSQ_EINVAL, "lsq_stream_create: empty model");
  if (cfg->n_slots < 2 || (cfg->n_slots > 8 && cfg->n_slots != cfg->n_layers))
    return fail(LSQ_EINVAL, "lsq_stream_create: n_slots must be 2..8 or n_layers (resident), got %d", cfg->n_slots);
  if ((cudaStream_t)compute == (cudaStream_t)copy)
    return fail(LSQ_EINVAL, "lsq_stream_create: the copy stream must differ from the compute stream");
  lsq_status s = check_device();
  if (s != LSQ_OK) return s;
  for (int i = 0; i < cfg->n_slots; ++i) {
    const void* p = cfg->slots[i];
    cudaPointerAttributes a;
    if (!p || !aligned(p, 256) || cudaPointerGetAttributes(&a, p) != cudaSuccess || a.type != cudaMemoryTypeDevice) {
      cudaGetLastError();
      return fail(LSQ_EINVAL, "lsq_stream_create: slot %d is not a 256-byte aligned device pointer", i);
    }
  }
  for (int l = 0; l < cfg->n_layers; ++l) {
    const char* h = static_cast<const char*>(cfg->host_records[l]);
    if (!h) return fail(LSQ_EINVAL, "lsq_stream_create: record %d is NULL", l);
    if (!is_pinned_host(h) || !is_pinned_host(h + cfg->record_bytes - 1))
      return fail(LSQ_ENOTPINNED, "lsq_stream_create: record %d is not page-locked host memory", l);
  }
  lsq_stream* st = new lsq_stream();
  st->n_layers = cfg->n_layers;
  st->n_slots = cfg->n_slots;
  st->record_bytes = cfg->record_bytes;
  st->slots.assign(cfg->slots, cfg->slots + cfg->n_slots);
  st->host.assign(cfg->host_records, cfg->host_records + cfg->n_layers);
  st->compute = (cudaStream_t)compute;
  st->copy = (cudaStream_t)copy;
  st->slot_layer.assign(st->n_slots, -1);
  st->slot_tick.assign(st->n_slots, 0);
  st->free_recorded.assign(st->n_slots, 0);
  st->layer_slot.assign(st->n_layers, -1);
  st->used_since_upload.assign(st->n_layers, 0);
  st->up_start.assign(st->n_layers, nullptr);
  st->up_done.assign(st->n_layers, nullptr);
  st->slot_free.assign(st->n_slots, nullptr);
  cudaError_t e = cudaSuccess;
  for (int l = 0; l < st->n_layers && e == cudaSuccess; ++l) {
    e = cudaEventCreate(&st->up_start[l]);
    if (e == cudaSuccess) e = cudaEventCreate(&st->up_done[l]);
  }
  for (int i = 0; i < st->n_slots && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(&st->slot_free[i], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    destroy_events(st);
    delete st;
    return cuda_fail(e, "lsq_stream_create: cudaEventCreate");
  }
  *out = st;
  return LSQ_OK;
}

extern "C" lsq_status lsq_layer_upload_async(lsq_stream* st, int32_t layer, int32_t slot) {
  if (!st) return fail(LSQ_EINVAL, "lsq_layer_upload_async: NULL scheduler");
  if (layer < 0 || layer >= st->n_layers || slot < 0 || slot >= st->n_slots)
    return fail(LSQ_EINVAL, "lsq_layer_upload_async: layer %d / slot %d out of range", layer, slot);
  if (st->cur >= 0 && st->layer_slot[st->cur] == slot && st->cur != layer)
    return fail(LSQ_ESTATE, "lsq_layer_upload_async: slot %d holds layer %d, which is in use", slot, st->cur);
  if (st->layer_slot[layer] == slot) return LSQ_OK;  // already there
  if (st->layer_slot[layer] >= 0) {                 // move: forget the old copy
    st->slot_layer[st->layer_slot[layer]] = -1;
    st->layer_slot[layer] = -1;
  }
  return upload(st, layer, slot);
}

extern "C" lsq_status lsq_stream_step(lsq_stream* st, int32_t layer, int32_t direction, void** slot_ptr) {
  if (!st || !slot_ptr) return fail(LSQ_EINVAL, "lsq_stream_step: NULL argument");
  if (layer < 0 || layer >= st->n_layers) return fail(LSQ_EINVAL, "lsq_stream_step: layer %d out of range", layer);
  if (direction != 1 && direction != -1) return fail(LSQ_EINVAL, "lsq_stream_step: direction must be +1 or -1");
  lsq_status s;
  // release the previous layer once the compute work enqueued so far is done
  if (st->cur >= 0 && st->cur != layer && st->layer_slot[st->cur] >= 0) {
    const int ps = st->layer_slot[st->cur];
    LSQ_CUDA_TRY(cudaEventRecord(st->slot_free[ps], st->compute));
    st->free_recorded[ps] = 1;
  }
  if (st->layer_slot[layer] < 0) {
    const int v = victim(st, -1);
    if ((s = upload(st, layer, v)) != LSQ_OK) return s;
  } else if (st->used_since_upload[layer]) {
    st->reused += 1;
  }
  const int slot = st->layer_slot[layer];
  LSQ_CUDA_TRY(cudaStreamWaitEvent(st->compute, st->up_done[layer], 0));
  st->slot_tick[slot] = ++st->tick;
  st->used_since_upload[layer] = 1;
  st->cur = layer;
  const int nxt = layer + direction;
  if (nxt >= 0 && nxt < st->n_layers && st->layer_slot[nxt] < 0) {
    const int v = victim(st, slot);
    if (v >= 0 && (s = upload(st, nxt, v)) != LSQ_OK) return s;
  }
  *slot_ptr = st->slots[slot];
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_stats(const lsq_stream* st, int64_t* uploads, int64_t* bytes, int64_t* reused) {
  if (!st || !uploads || !bytes || !reused) return fail(LSQ_EINVAL, "lsq_stream_stats: NULL argument");
  *uploads = st->uploads;
  *bytes = st->bytes;
  *reused = st->reused;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_upload_ms(lsq_stream* st, int32_t layer, float* ms) {
  if (!st || !ms) return fail(LSQ_EINVAL, "lsq_stream_upload_ms: NULL argument");
  if (layer < 0 || layer >= st->n_layers) return fail(LSQ_EINVAL, "lsq_stream_upload_ms: layer out of range");
  LSQ_CUDA_TRY(cudaEventSynchronize(st->up_done[layer]));
  LSQ_CUDA_TRY(cudaEventElapsedTime(ms, st->up_start[layer], st->up_done[layer]));
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_reset(lsq_stream* st) {
  if (!st) return fail(LSQ_EINVAL, "lsq_stream_reset: NULL scheduler");
  LSQ_CUDA_TRY(cudaStreamSynchronize(st->copy));
  LSQ_CUDA_TRY(cudaStreamSynchronize(st->compute));
  std::fill(st->slot_layer.begin(), st->slot_layer.end(), -1);
  std::fill(st->layer_slot.begin(), st->layer_slot.end(), -1);
  std::fill(st->slot_tick.begin(), st->slot_tick.end(), 0);
  std::fill(st->free_recorded.begin(), st->free_recorded.end(), 0);
  std::fill(st->used_since_upload.begin(), st->used_since_upload.end(), 0);
  st->cur = -1;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_destroy(lsq_stream* st) {
  if (!st) return LSQ_OK;
  cudaStreamSynchronize(st->copy);
  destroy_events(st);
  delete st;
  return LSQ_OK;
}
