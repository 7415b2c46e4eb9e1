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
//
// The slot policy (which slot to fill, how far to prefetch) is a CUDA-free
// core that emits actions; the scheduler executes them with CUDA calls and
// lsq_stream_simulate returns them, so the policy is testable without a GPU.
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <chrono>
#include <condition_variable>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "host_common.h"

namespace lsq {
namespace sched {

enum ActKind { RELEASE = 1, UPLOAD = 2, WAIT = 3 };
struct Act {
  int kind, layer, slot;
};

struct Policy {
  int n_layers = 0, n_slots = 0;
  std::vector<int> slot_layer;         // layer held by a slot, -1 if none
  std::vector<int64_t> slot_tick;      // last step() use, for LRU
  std::vector<int> layer_slot;         // slot holding a layer, -1 if none
  std::vector<char> used_since_upload; // stepped since its last upload
  int cur = -1;                        // layer of the last step()
  int64_t tick = 0, uploads = 0, reused = 0;

  void init(int L, int S) {
    n_layers = L;
    n_slots = S;
    slot_layer.assign(S, -1);
    slot_tick.assign(S, 0);
    layer_slot.assign(L, -1);
    used_since_upload.assign(L, 0);
    cur = -1;
    tick = uploads = reused = 0;
  }

  // An empty slot if any, else the least recently used one, skipping slots
  // whose layer is in `keep` (the layer in use and those prefetched ahead).
  int victim(const int* keep, int nkeep) const {
    int best = -1;
    for (int s = 0; s < n_slots; ++s) {
      bool kept = false;
      for (int i = 0; i < nkeep; ++i) kept |= (keep[i] >= 0 && slot_layer[s] == keep[i]);
      if (kept) continue;
      if (slot_layer[s] < 0) return s;
      if (best < 0 || slot_tick[s] < slot_tick[best]) best = s;
    }
    return best;
  }

  void place(int layer, int slot, std::vector<Act>& out) {
    const int old = slot_layer[slot];
    if (old >= 0) layer_slot[old] = -1;
    if (layer_slot[layer] >= 0) slot_layer[layer_slot[layer]] = -1;
    slot_layer[slot] = layer;
    layer_slot[layer] = slot;
    used_since_upload[layer] = 0;
    uploads += 1;
    out.push_back({UPLOAD, layer, slot});
  }

  // Begin compute on `layer` walking in `direction`; appends the actions.
  void step(int layer, int direction, std::vector<Act>& out) {
    if (cur >= 0 && cur != layer && layer_slot[cur] >= 0) out.push_back({RELEASE, cur, layer_slot[cur]});
    if (layer_slot[layer] < 0) {
      place(layer, victim(nullptr, 0), out);
    } else if (used_since_upload[layer]) {
      reused += 1;
    }
    const int slot = layer_slot[layer];
    out.push_back({WAIT, layer, slot});
    slot_tick[slot] = ++tick;
    used_since_upload[layer] = 1;
    cur = layer;
    // prefetch up to n_slots - 1 layers ahead in the walking direction
    int keep[8] = {layer, -1, -1, -1, -1, -1, -1, -1};
    int nkeep = 1;
    const int ahead = n_slots - 1 < 7 ? n_slots - 1 : 7;
    for (int k = 1; k <= ahead; ++k) {
      const int nxt = layer + k * direction;
      if (nxt < 0 || nxt >= n_layers) break;
      if (layer_slot[nxt] < 0) {
        const int v = victim(keep, nkeep);
        if (v < 0) break;
        place(nxt, v, out);
      }
      keep[nkeep++] = nxt;
    }
  }
};

}  // namespace sched
}  // namespace lsq

namespace lsq {
namespace disk {

// Disk tier: layer parts are read from a store file into a ring of
// page-locked staging buffers by a small pool of host threads, in the order
// the scheduler submits them; the copy stream waits for each part with a host
// function before its host-to-device copy and hands the buffer back with
// another one after it.  Part t (the t-th upload) uses buffer t % n; the
// readers fill it only once part t - n has been handed back, and each reader
// thread reads one contiguous piece of every part, in part order.  Every wait
// is bounded (kWaitS); a wait that runs out, or a failed read, sets an error
// that the next scheduler call returns.
constexpr int kWaitS = 120;

struct Reader {
  int fd = -1;
  size_t part_bytes = 0;           // bytes per upload (this rank's part of a record)
  std::vector<void*> staging;      // page-locked, part_bytes each
  int nthreads = 0;
  std::mutex mu;
  std::condition_variable cv;
  std::vector<int> job_layer;      // layer of each submitted part (index = ticket)
  std::vector<int64_t> filled;     // per buffer: the ticket whose bytes it holds, -1 none
  std::vector<int64_t> released;   // per buffer: the last ticket handed back by the copy stream
  std::vector<int> pieces;         // per buffer: pieces of the pending ticket read so far
  bool stop = false;
  lsq_status error = LSQ_OK;
  std::string errmsg;
  std::vector<std::thread> threads;
  int64_t bytes_read = 0;

  int n() const { return (int)staging.size(); }

  void set_error(lsq_status e, const std::string& m) {
    if (error == LSQ_OK) {
      error = e;
      errmsg = m;
    }
    cv.notify_all();
  }

  int64_t submit(int layer) {
    std::lock_guard<std::mutex> g(mu);
    job_layer.push_back(layer);
    cv.notify_all();
    return (int64_t)job_layer.size() - 1;
  }

  void worker(int w) {
    const size_t per = (part_bytes + nthreads - 1) / nthreads;
    const size_t lo = std::min(part_bytes, (size_t)w * per), hi = std::min(part_bytes, lo + per);
    for (int64_t t = 0;; ++t) {
      const int b = (int)(t % n());
      int layer;
      {
        std::unique_lock<std::mutex> g(mu);
        // the part is submitted and its buffer handed back by part t - n
        for (;;) {
          const bool ok = cv.wait_for(g, std::chrono::seconds(kWaitS), [&] {
            return stop || error != LSQ_OK || ((int64_t)job_layer.size() > t && released[b] >= t - n());
          });
          if (stop || error != LSQ_OK) return;
          if (ok) break;
          if ((int64_t)job_layer.size() > t) {
            set_error(LSQ_ETIMEOUT, "disk tier: a staging buffer was not handed back in time");
            return;
          }
          // idle (nothing submitted yet): keep waiting on the host
        }
        layer = job_layer[t];
      }
      char* dst = static_cast<char*>(staging[b]) + lo;
      off_t off = (off_t)((uint64_t)layer * part_bytes + lo);
      size_t left = hi - lo;
      while (left > 0) {
        const ssize_t r = pread(fd, dst, left, off);
        if (r <= 0) {
          std::lock_guard<std::mutex> g(mu);
          set_error(LSQ_EINVAL, std::string("disk tier: read of layer ") + std::to_string(layer) + " failed: " +
                                    (r == 0 ? "end of file" : std::strerror(errno)));
          return;
        }
        dst += r;
        off += r;
        left -= (size_t)r;
      }
      std::lock_guard<std::mutex> g(mu);
      bytes_read += (int64_t)(hi - lo);
      if (++pieces[b] == nthreads) {
        pieces[b] = 0;
        filled[b] = t;
        cv.notify_all();
      }
    }
  }

  // host-function side (copy stream): wait until part t is in its buffer
  void wait_filled(int64_t t) {
    const int b = (int)(t % n());
    std::unique_lock<std::mutex> g(mu);
    if (!cv.wait_for(g, std::chrono::seconds(kWaitS), [&] { return stop || error != LSQ_OK || filled[b] == t; }))
      set_error(LSQ_ETIMEOUT, "disk tier: a layer part was not read in time");
  }
  void release(int64_t t) {
    std::lock_guard<std::mutex> g(mu);
    released[t % n()] = t;
    cv.notify_all();
  }

  void shutdown() {
    {
      std::lock_guard<std::mutex> g(mu);
      stop = true;
    }
    cv.notify_all();
    for (auto& th : threads)
      if (th.joinable()) th.join();
    threads.clear();
    if (fd >= 0) close(fd);
    fd = -1;
  }
};

struct HostArg {
  Reader* r;
  int64_t t;
};
static void CUDART_CB wait_filled_cb(void* p) {
  HostArg* a = static_cast<HostArg*>(p);
  a->r->wait_filled(a->t);
  delete a;
}
static void CUDART_CB release_cb(void* p) {
  HostArg* a = static_cast<HostArg*>(p);
  a->r->release(a->t);
  delete a;
}

}  // namespace disk
}  // namespace lsq

struct lsq_stream {
  lsq::sched::Policy pol;
  lsq::disk::Reader* reader = nullptr;  // disk tier, else records come from host_records
  size_t record_bytes = 0;
  // sharded upload: this rank copies shard_bytes at shard_rank * shard_bytes; gather completes the slot
  size_t shard_bytes = 0;
  int shard_rank = 0;
  lsq_gather_fn gather = nullptr;
  void* gather_user = nullptr;
  std::vector<void*> slots;
  std::vector<const void*> host;
  cudaStream_t compute = nullptr, copy = nullptr;
  std::vector<char> free_recorded;  // slot_free[slot] has been recorded
  std::vector<cudaEvent_t> up_start, up_done, slot_free;
  int64_t bytes = 0;
  std::vector<lsq::sched::Act> acts;
  // double-quantised absmax: expanded to fp32 inside the slot after each upload
  int n_expand = 0;
  uint64_t ex_codes[8], ex_params[8], ex_out[8];
  int64_t ex_nb[8];
  int64_t expands = 0;
  // exposed-copy timing: a pair of timing events around each compute-stream wait on an upload
  int direction = 0;                 // walking direction of the lsq_stream_step being executed
  std::vector<cudaEvent_t> wev;      // 2 per kept wait
  std::vector<int> wdir;             // direction of each kept wait
  int n_wait = 0, n_wait_dropped = 0;
  // stream capture of one step (lsq_stream_capture_begin / _end): the copy stream joins the compute
  // stream's capture; only events recorded inside it order work inside it
  bool capturing = false;
  std::vector<char> cap_up, cap_free;  // up_done[layer] / slot_free[slot] recorded in this capture
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
  std::vector<int> cap_state;          // the policy's slot map when the capture began
  // events last recorded inside a capture cannot be waited on or timed outside it: the first eager
  // use after a capture records them again on the compute stream (after every replay queued there)
  std::vector<char> stale_up, stale_free;
  std::vector<char> untimed;           // the layer's upload events were re-recorded, not timed
};

namespace lsq {
namespace sched {

// Re-record, at the current point of the compute stream, the events a capture left behind: a
// release or an upload recorded in a captured step is complete once the compute stream passes the
// graph launches queued on it (the graph joins the copy stream back before it ends).
static lsq_status refresh_after_capture(lsq_stream* st) {
  for (size_t s = 0; s < st->stale_free.size(); ++s)
    if (st->stale_free[s]) LSQ_CUDA_TRY(cudaEventRecord(st->slot_free[s], st->compute));
  for (size_t l = 0; l < st->stale_up.size(); ++l)
    if (st->stale_up[l]) {
      LSQ_CUDA_TRY(cudaEventRecord(st->up_start[l], st->compute));
      LSQ_CUDA_TRY(cudaEventRecord(st->up_done[l], st->compute));
      st->untimed[l] = 1;
    }
  st->stale_free.clear();
  st->stale_up.clear();
  return LSQ_OK;
}

static lsq_status execute(lsq_stream* st) {
  if (!st->capturing && (!st->stale_free.empty() || !st->stale_up.empty())) {
    lsq_status s = refresh_after_capture(st);
    if (s != LSQ_OK) return s;
  }
  for (const Act& a : st->acts) {
    if (a.kind == RELEASE) {
      LSQ_CUDA_TRY(cudaEventRecord(st->slot_free[a.slot], st->compute));
      st->free_recorded[a.slot] = 1;
      if (st->capturing) st->cap_free[a.slot] = 1;
    } else if (a.kind == UPLOAD) {
      // in a capture, a release recorded before it is already ordered: the graph starts after the
      // compute stream's earlier work
      if (st->free_recorded[a.slot] && (!st->capturing || st->cap_free[a.slot]))
        LSQ_CUDA_TRY(cudaStreamWaitEvent(st->copy, st->slot_free[a.slot], 0));
      LSQ_CUDA_TRY(cudaEventRecord(st->up_start[a.layer], st->copy));
      char* dst = static_cast<char*>(st->slots[a.slot]) + (size_t)st->shard_rank * st->shard_bytes;
      if (st->reader) {
        disk::Reader* r = st->reader;
        const int64_t t = r->submit(a.layer);
        LSQ_CUDA_TRY(cudaLaunchHostFunc(st->copy, disk::wait_filled_cb, new disk::HostArg{r, t}));
        LSQ_CUDA_TRY(cudaMemcpyAsync(dst, r->staging[t % r->n()], st->shard_bytes, cudaMemcpyHostToDevice,
                                     st->copy));
        LSQ_CUDA_TRY(cudaLaunchHostFunc(st->copy, disk::release_cb, new disk::HostArg{r, t}));
      } else {
        LSQ_CUDA_TRY(cudaMemcpyAsync(dst, st->host[a.layer], st->shard_bytes, cudaMemcpyHostToDevice, st->copy));
      }
      if (st->gather) {
        const int32_t rc = st->gather(st->gather_user, a.layer, a.slot, st->slots[a.slot], st->record_bytes,
                                      (lsq_cuda_stream)st->copy);
        if (rc != 0) return fail(LSQ_ECALLBACK, "gather callback returned %d for layer %d", rc, a.layer);
      }
      if (st->n_expand > 0) {
        lsq_status s = dq::launch_expand(static_cast<const char*>(st->slots[a.slot]), st->ex_codes, st->ex_params,
                                         st->ex_out, st->ex_nb, st->n_expand, st->copy);
        if (s != LSQ_OK) return s;
        st->expands += 1;
      }
      LSQ_CUDA_TRY(cudaEventRecord(st->up_done[a.layer], st->copy));
      if (st->capturing) st->cap_up[a.layer] = 1;
      st->untimed[a.layer] = 0;
      st->bytes += (int64_t)st->shard_bytes;
    } else if (a.kind == WAIT) {
      // in a capture, an upload recorded before it is complete when the graph starts (the caller
      // orders the compute stream after the copy stream's earlier work)
      if (st->capturing && !st->cap_up[a.layer]) continue;
      const bool timed = !st->wev.empty();
      const bool kept = timed && 2 * (size_t)st->n_wait < st->wev.size();
      if (kept) LSQ_CUDA_TRY(cudaEventRecord(st->wev[2 * st->n_wait], st->compute));
      LSQ_CUDA_TRY(cudaStreamWaitEvent(st->compute, st->up_done[a.layer], 0));
      if (kept) {
        LSQ_CUDA_TRY(cudaEventRecord(st->wev[2 * st->n_wait + 1], st->compute));
        st->wdir[st->n_wait++] = st->direction;
      } else if (timed) {
        st->n_wait_dropped += 1;
      }
    }
  }
  st->acts.clear();
  return LSQ_OK;
}

static bool is_pinned_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// the disk tier's first error, if any (returned by the next scheduler call)
static lsq_status disk_status(lsq_stream* st) {
  if (!st->reader) return LSQ_OK;
  std::lock_guard<std::mutex> g(st->reader->mu);
  if (st->reader->error == LSQ_OK) return LSQ_OK;
  return fail(st->reader->error, "%s", st->reader->errmsg.c_str());
}

static void destroy_wait_events(lsq_stream* st) {
  for (cudaEvent_t e : st->wev)
    if (e) cudaEventDestroy(e);
  st->wev.clear();
  st->wdir.clear();
  st->n_wait = st->n_wait_dropped = 0;
}

static void destroy_events(lsq_stream* st) {
  destroy_wait_events(st);
  for (auto* v : {&st->up_start, &st->up_done, &st->slot_free})
    for (cudaEvent_t e : *v)
      if (e) cudaEventDestroy(e);
  if (st->fork_ev) cudaEventDestroy(st->fork_ev);
  if (st->join_ev) cudaEventDestroy(st->join_ev);
  st->fork_ev = st->join_ev = nullptr;
}

// The part of the policy's state that a step's actions depend on: which layer each slot holds, the
// slots' LRU order, the layers stepped since their upload, the current layer.  (The tick counter
// itself grows without bound; only the order it gives matters.)
static std::vector<int> slot_map(const Policy& p) {
  std::vector<int> v(p.slot_layer);
  for (int s = 0; s < p.n_slots; ++s) {
    int rank = 0;
    for (int t = 0; t < p.n_slots; ++t) rank += p.slot_tick[t] < p.slot_tick[s];
    v.push_back(rank);
  }
  for (char u : p.used_since_upload) v.push_back(u);
  v.push_back(p.cur);
  return v;
}

static bool valid_slots(int n_layers, int n_slots) {
  return n_slots >= 2 && (n_slots <= 8 || n_slots == n_layers);
}

}  // namespace sched
}  // namespace lsq

using namespace lsq;
using namespace lsq::sched;

extern "C" lsq_status lsq_stream_create(const lsq_stream_cfg* cfg, lsq_cuda_stream compute, lsq_cuda_stream copy,
                                        lsq_stream** out) {
  if (!cfg || !out || !cfg->slots || (!cfg->host_records && !cfg->disk_path))
    return fail(LSQ_EINVAL, "lsq_stream_create: NULL argument");
  if (cfg->host_records && cfg->disk_path)
    return fail(LSQ_EINVAL, "lsq_stream_create: give host_records or disk_path, not both");
  *out = nullptr;
  if (cfg->n_layers < 1 || cfg->record_bytes == 0) return fail(LSQ_EINVAL, "lsq_stream_create: empty model");
  if (!valid_slots(cfg->n_layers, cfg->n_slots))
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
  const int world = cfg->shard_world > 1 ? cfg->shard_world : 1;
  if (cfg->shard_world < 0 || cfg->shard_rank < 0 || cfg->shard_rank >= world)
    return fail(LSQ_EINVAL, "lsq_stream_create: shard rank %d of %d", cfg->shard_rank, cfg->shard_world);
  if (world > 1 && !cfg->gather) return fail(LSQ_EINVAL, "lsq_stream_create: sharded upload needs a gather callback");
  if (cfg->record_bytes % (256 * (size_t)world) != 0)
    return fail(LSQ_EINVAL, "lsq_stream_create: record_bytes must be a multiple of 256 x shard_world");
  const size_t shard = cfg->record_bytes / world;
  for (int l = 0; cfg->host_records && l < cfg->n_layers; ++l) {
    const char* h = static_cast<const char*>(cfg->host_records[l]);
    if (!h) return fail(LSQ_EINVAL, "lsq_stream_create: record %d is NULL", l);
    if (!is_pinned_host(h) || !is_pinned_host(h + shard - 1))
      return fail(LSQ_ENOTPINNED, "lsq_stream_create: record %d is not page-locked host memory", l);
  }
  disk::Reader* reader = nullptr;
  if (cfg->disk_path) {
    if (cfg->n_staging < 2 || cfg->n_staging > 8 || !cfg->staging || cfg->disk_threads < 1 || cfg->disk_threads > 16)
      return fail(LSQ_EINVAL, "lsq_stream_create: the disk tier needs 2..8 staging buffers and 1..16 threads");
    for (int i = 0; i < cfg->n_staging; ++i) {
      const char* h = static_cast<const char*>(cfg->staging[i]);
      if (!h || !is_pinned_host(h) || !is_pinned_host(h + shard - 1))
        return fail(LSQ_ENOTPINNED, "lsq_stream_create: staging buffer %d is not page-locked host memory", i);
    }
    const int fd = open(cfg->disk_path, O_RDONLY | O_CLOEXEC);
    if (fd < 0) return fail(LSQ_EINVAL, "lsq_stream_create: cannot open %s: %s", cfg->disk_path, std::strerror(errno));
    struct stat sb;
    if (fstat(fd, &sb) != 0 || (uint64_t)sb.st_size < (uint64_t)cfg->n_layers * shard) {
      close(fd);
      return fail(LSQ_EINVAL, "lsq_stream_create: %s holds less than %d layer parts of %zu bytes", cfg->disk_path,
                  cfg->n_layers, shard);
    }
    posix_fadvise(fd, 0, 0, POSIX_FADV_SEQUENTIAL);
    reader = new disk::Reader();
    reader->fd = fd;
    reader->part_bytes = shard;
    reader->staging.assign(cfg->staging, cfg->staging + cfg->n_staging);
    reader->nthreads = cfg->disk_threads;
    reader->filled.assign(cfg->n_staging, -1);
    reader->released.assign(cfg->n_staging, -1);
    for (int b = 0; b < cfg->n_staging; ++b) reader->released[b] = b - cfg->n_staging;  // never used yet
    reader->pieces.assign(cfg->n_staging, 0);
    for (int w = 0; w < reader->nthreads; ++w) reader->threads.emplace_back(&disk::Reader::worker, reader, w);
  }
  lsq_stream* st = new lsq_stream();
  st->reader = reader;
  st->pol.init(cfg->n_layers, cfg->n_slots);
  st->record_bytes = cfg->record_bytes;
  st->shard_bytes = shard;
  st->shard_rank = cfg->shard_rank;
  st->gather = cfg->gather;
  st->gather_user = cfg->gather_user;
  st->slots.assign(cfg->slots, cfg->slots + cfg->n_slots);
  if (cfg->host_records) st->host.assign(cfg->host_records, cfg->host_records + cfg->n_layers);
  st->compute = (cudaStream_t)compute;
  st->copy = (cudaStream_t)copy;
  st->free_recorded.assign(cfg->n_slots, 0);
  st->up_start.assign(cfg->n_layers, nullptr);
  st->up_done.assign(cfg->n_layers, nullptr);
  st->untimed.assign(cfg->n_layers, 0);
  st->slot_free.assign(cfg->n_slots, nullptr);
  cudaError_t e = cudaSuccess;
  for (int l = 0; l < cfg->n_layers && e == cudaSuccess; ++l) {
    e = cudaEventCreate(&st->up_start[l]);
    if (e == cudaSuccess) e = cudaEventCreate(&st->up_done[l]);
  }
  for (int i = 0; i < cfg->n_slots && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(&st->slot_free[i], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->fork_ev, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->join_ev, cudaEventDisableTiming);
  // every slot starts out released at this point of the compute stream, so the first upload into it
  // waits for the work queued there so far: the caller's allocator may have handed out the slots'
  // memory while kernels that still write its previous contents are queued on that stream
  for (int i = 0; i < cfg->n_slots && e == cudaSuccess; ++i) {
    e = cudaEventRecord(st->slot_free[i], st->compute);
    st->free_recorded[i] = 1;
  }
  if (e != cudaSuccess) {
    destroy_events(st);
    if (st->reader) {
      st->reader->shutdown();
      delete st->reader;
    }
    delete st;
    return cuda_fail(e, "lsq_stream_create: event create / record");
  }
  *out = st;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_set_absmax_expand(lsq_stream* st, const lsq_absmax_dq_item* items,
                                                  int32_t n_items, size_t slot_bytes) {
  if (!st || (n_items > 0 && !items)) return fail(LSQ_EINVAL, "lsq_stream_set_absmax_expand: NULL argument");
  if (n_items < 0 || n_items > 8) return fail(LSQ_EINVAL, "lsq_stream_set_absmax_expand: 0..8 items, got %d", n_items);
  if (st->pol.uploads > 0) return fail(LSQ_ESTATE, "lsq_stream_set_absmax_expand: call before the first upload");
  const uint64_t rec = st->record_bytes;
  for (int k = 0; k < n_items; ++k) {
    const lsq_absmax_dq_item& it = items[k];
    const uint64_t nb = (uint64_t)it.nb, nblk = (nb + 255) / 256;
    if (it.nb < 1 || it.codes_off + nb > rec || it.params_off % 8 || it.params_off + 8 * nblk > rec ||
        it.out_off % 4 || it.out_off < rec || it.out_off + 4 * nb > slot_bytes)
      return fail(LSQ_EINVAL,
                  "lsq_stream_set_absmax_expand: item %d out of bounds (codes and params inside the record, "
                  "params 8-byte aligned, output 4-byte aligned between the record's end and slot_bytes)", k);
    for (int j = 0; j < k; ++j)
      if (it.out_off < items[j].out_off + 4 * (uint64_t)items[j].nb && items[j].out_off < it.out_off + 4 * nb)
        return fail(LSQ_EINVAL, "lsq_stream_set_absmax_expand: outputs of items %d and %d overlap", j, k);
  }
  st->n_expand = n_items;
  for (int k = 0; k < n_items; ++k) {
    st->ex_codes[k] = items[k].codes_off;
    st->ex_params[k] = items[k].params_off;
    st->ex_out[k] = items[k].out_off;
    st->ex_nb[k] = items[k].nb;
  }
  return LSQ_OK;
}

extern "C" lsq_status lsq_layer_upload_async(lsq_stream* st, int32_t layer, int32_t slot) {
  if (!st) return fail(LSQ_EINVAL, "lsq_layer_upload_async: NULL scheduler");
  Policy& p = st->pol;
  if (layer < 0 || layer >= p.n_layers || slot < 0 || slot >= p.n_slots)
    return fail(LSQ_EINVAL, "lsq_layer_upload_async: layer %d / slot %d out of range", layer, slot);
  if (p.cur >= 0 && p.layer_slot[p.cur] == slot && p.cur != layer)
    return fail(LSQ_ESTATE, "lsq_layer_upload_async: slot %d holds layer %d, which is in use", slot, p.cur);
  if (p.layer_slot[layer] == slot) return LSQ_OK;  // already there
  lsq_status ds = disk_status(st);
  if (ds != LSQ_OK) return ds;
  p.place(layer, slot, st->acts);
  return execute(st);
}

extern "C" lsq_status lsq_stream_step(lsq_stream* st, int32_t layer, int32_t direction, void** slot_ptr) {
  if (!st || !slot_ptr) return fail(LSQ_EINVAL, "lsq_stream_step: NULL argument");
  if (layer < 0 || layer >= st->pol.n_layers) return fail(LSQ_EINVAL, "lsq_stream_step: layer %d out of range", layer);
  if (direction != 1 && direction != -1) return fail(LSQ_EINVAL, "lsq_stream_step: direction must be +1 or -1");
  lsq_status ds = disk_status(st);
  if (ds != LSQ_OK) return ds;
  st->pol.step(layer, direction, st->acts);
  st->direction = direction;
  lsq_status s = execute(st);
  if (s != LSQ_OK) return s;
  *slot_ptr = st->slots[st->pol.layer_slot[layer]];
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_simulate(int32_t n_layers, int32_t n_slots, int32_t n_steps, const int32_t* layers,
                                          const int32_t* directions, int32_t* actions, int32_t max_actions,
                                          int32_t* n_actions) {
  if (!layers || !directions || !actions || !n_actions) return fail(LSQ_EINVAL, "lsq_stream_simulate: NULL argument");
  if (n_layers < 1 || !valid_slots(n_layers, n_slots) || n_steps < 0 || max_actions < 0)
    return fail(LSQ_EINVAL, "lsq_stream_simulate: bad sizes");
  Policy p;
  p.init(n_layers, n_slots);
  std::vector<Act> acts;
  for (int i = 0; i < n_steps; ++i) {
    if (layers[i] < 0 || layers[i] >= n_layers || (directions[i] != 1 && directions[i] != -1))
      return fail(LSQ_EINVAL, "lsq_stream_simulate: step %d out of range", i);
    p.step(layers[i], directions[i], acts);
  }
  if ((int64_t)acts.size() > max_actions)
    return fail(LSQ_EINVAL, "lsq_stream_simulate: %zu actions exceed max_actions", acts.size());
  for (size_t i = 0; i < acts.size(); ++i) {
    actions[3 * i] = acts[i].kind;
    actions[3 * i + 1] = acts[i].layer;
    actions[3 * i + 2] = acts[i].slot;
  }
  *n_actions = (int32_t)acts.size();
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_stats(const lsq_stream* st, int64_t* uploads, int64_t* bytes, int64_t* reused) {
  if (!st || !uploads || !bytes || !reused) return fail(LSQ_EINVAL, "lsq_stream_stats: NULL argument");
  *uploads = st->pol.uploads;
  *bytes = st->bytes;
  *reused = st->pol.reused;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_upload_ms(lsq_stream* st, int32_t layer, float* ms) {
  if (!st || !ms) return fail(LSQ_EINVAL, "lsq_stream_upload_ms: NULL argument");
  if (layer < 0 || layer >= st->pol.n_layers) return fail(LSQ_EINVAL, "lsq_stream_upload_ms: layer out of range");
  if (st->capturing || ((size_t)layer < st->stale_up.size() && st->stale_up[layer]) || st->untimed[layer])
    return fail(LSQ_ESTATE, "lsq_stream_upload_ms: layer %d was last uploaded inside a captured step", layer);
  LSQ_CUDA_TRY(cudaEventSynchronize(st->up_done[layer]));
  LSQ_CUDA_TRY(cudaEventElapsedTime(ms, st->up_start[layer], st->up_done[layer]));
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_time_waits(lsq_stream* st, int32_t capacity) {
  if (!st) return fail(LSQ_EINVAL, "lsq_stream_time_waits: NULL scheduler");
  if (capacity < 0 || capacity > (1 << 20)) return fail(LSQ_EINVAL, "lsq_stream_time_waits: capacity %d", capacity);
  if (st->capturing) return fail(LSQ_ESTATE, "lsq_stream_time_waits: a capture is open");
  LSQ_CUDA_TRY(cudaStreamSynchronize(st->compute));  // no kept wait is still pending on the old events
  destroy_wait_events(st);
  if (capacity == 0) return LSQ_OK;
  st->wev.assign(2 * (size_t)capacity, nullptr);
  st->wdir.assign(capacity, 0);
  for (size_t i = 0; i < st->wev.size(); ++i) {
    cudaError_t e = cudaEventCreate(&st->wev[i]);
    if (e != cudaSuccess) {
      st->wev[i] = nullptr;
      destroy_wait_events(st);
      return cuda_fail(e, "lsq_stream_time_waits: event create");
    }
  }
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_wait_ms(lsq_stream* st, float* fwd_ms, float* bwd_ms, int32_t* n_waits,
                                         int32_t* n_dropped) {
  if (!st || !fwd_ms || !bwd_ms || !n_waits || !n_dropped) return fail(LSQ_EINVAL, "lsq_stream_wait_ms: NULL argument");
  if (st->wev.empty()) return fail(LSQ_ESTATE, "lsq_stream_wait_ms: wait timing is off (lsq_stream_time_waits)");
  double f = 0.0, b = 0.0;
  for (int i = 0; i < st->n_wait; ++i) {
    float ms = 0.0f;
    LSQ_CUDA_TRY(cudaEventSynchronize(st->wev[2 * i + 1]));
    LSQ_CUDA_TRY(cudaEventElapsedTime(&ms, st->wev[2 * i], st->wev[2 * i + 1]));
    (st->wdir[i] > 0 ? f : b) += ms;
  }
  *fwd_ms = (float)f;
  *bwd_ms = (float)b;
  *n_waits = st->n_wait;
  *n_dropped = st->n_wait_dropped;
  st->n_wait = st->n_wait_dropped = 0;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_reset(lsq_stream* st) {
  if (!st) return fail(LSQ_EINVAL, "lsq_stream_reset: NULL scheduler");
  if (st->capturing) return fail(LSQ_ESTATE, "lsq_stream_reset: a capture is open");
  LSQ_CUDA_TRY(cudaStreamSynchronize(st->copy));
  LSQ_CUDA_TRY(cudaStreamSynchronize(st->compute));
  const int64_t up = st->pol.uploads, re = st->pol.reused;
  st->pol.init(st->pol.n_layers, st->pol.n_slots);
  st->pol.uploads = up;
  st->pol.reused = re;
  std::fill(st->free_recorded.begin(), st->free_recorded.end(), 0);
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_capture_begin(lsq_stream* st) {
  if (!st) return fail(LSQ_EINVAL, "lsq_stream_capture_begin: NULL scheduler");
  if (st->capturing) return fail(LSQ_ESTATE, "lsq_stream_capture_begin: a capture is already open");
  if (st->reader || st->gather)
    return fail(LSQ_EINVAL, "lsq_stream_capture_begin: the disk tier and sharded uploads do host work in each step");
  if (!st->wev.empty()) return fail(LSQ_EINVAL, "lsq_stream_capture_begin: exposed-copy timing is on");
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  LSQ_CUDA_TRY(cudaStreamIsCapturing(st->compute, &cs));
  if (cs != cudaStreamCaptureStatusActive)
    return fail(LSQ_ESTATE, "lsq_stream_capture_begin: the compute stream is not being captured");
  st->cap_up.assign(st->pol.n_layers, 0);
  st->cap_free.assign(st->pol.n_slots, 0);
  LSQ_CUDA_TRY(cudaEventRecord(st->fork_ev, st->compute));
  LSQ_CUDA_TRY(cudaStreamWaitEvent(st->copy, st->fork_ev, 0));
  st->cap_state = slot_map(st->pol);
  st->capturing = true;
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_capture_end(lsq_stream* st) {
  if (!st) return fail(LSQ_EINVAL, "lsq_stream_capture_end: NULL scheduler");
  if (!st->capturing) return fail(LSQ_ESTATE, "lsq_stream_capture_end: no capture is open");
  st->capturing = false;
  st->stale_up = st->cap_up;
  st->stale_free = st->cap_free;
  LSQ_CUDA_TRY(cudaEventRecord(st->join_ev, st->copy));
  LSQ_CUDA_TRY(cudaStreamWaitEvent(st->compute, st->join_ev, 0));
  if (slot_map(st->pol) != st->cap_state)
    return fail(LSQ_ESTATE, "lsq_stream_capture_end: the captured steps leave the slots holding other layers than "
                "at the start, so a replay would compute on the wrong records (capture after a full warm-up step)");
  return LSQ_OK;
}

extern "C" lsq_status lsq_stream_destroy(lsq_stream* st) {
  if (!st) return LSQ_OK;
  cudaStreamSynchronize(st->copy);  // every host function of the disk tier has run
  if (st->reader) {
    st->reader->shutdown();
    delete st->reader;
  }
  destroy_events(st);
  delete st;
  return LSQ_OK;
}
