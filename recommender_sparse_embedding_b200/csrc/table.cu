// table.cu -- host side of the embedding engine: the C ABI of include/recis.h,
// table and batch lifetimes, EmbeddingBlocks growth, IDMap growth, error
// reporting and kernel tracing.
//
// EmbeddingBlocks (RecIS README, Key optimisations > Efficient dynamic
// embedding: contiguous chunked memory blocks that grow on demand) are
// physical allocations (cuMemCreate) mapped one after another into a single
// reserved virtual range, so a row is found as base + row * stride with no
// block table and growth maps a new block without copying.
//
// The host never waits for the device in steady state: it keeps an upper bound
// of the live rows (previous bound + N per lookup), tightened whenever the
// event recorded after the last call has completed (the kernels write the live
// row count and an error flag into host-mapped memory).  Only when the bound
// says the row space or the IDMap could overflow does it synchronise, read the
// exact count and grow.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace recis {

namespace {
thread_local std::string g_err;

std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::atomic<int64_t> g_launches{0};
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

int* g_feat_status[128] = {nullptr};
std::mutex g_feat_mu;

std::atomic<int> g_spin_limit{kSpinLimit};
std::atomic<int64_t> g_map_limit{0};

constexpr double kMaxLoad = 0.5;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void set_error(const std::string& msg) { g_err = msg; }

int spin_limit() { return g_spin_limit.load(std::memory_order_relaxed); }
int64_t map_limit_bytes() { return g_map_limit.load(std::memory_order_relaxed); }

recis_status cuda_fail(cudaError_t e, const char* what) {
  set_error(std::string(what) + ": " + cudaGetErrorString(e));
  return RECIS_ERR_CUDA;
}

// Driver entry points, resolved through the runtime so that the library has no
// link-time dependency on libcuda (it loads on machines without a driver).
struct Drv {
  decltype(&::cuMemAddressReserve) MemAddressReserve = nullptr;
  decltype(&::cuMemAddressFree) MemAddressFree = nullptr;
  decltype(&::cuMemCreate) MemCreate = nullptr;
  decltype(&::cuMemRelease) MemRelease = nullptr;
  decltype(&::cuMemMap) MemMap = nullptr;
  decltype(&::cuMemUnmap) MemUnmap = nullptr;
  decltype(&::cuMemSetAccess) MemSetAccess = nullptr;
  decltype(&::cuMemGetAllocationGranularity) MemGetAllocationGranularity = nullptr;
  decltype(&::cuGetErrorString) GetErrorString = nullptr;
  decltype(&::cuDeviceGet) DeviceGet = nullptr;
  decltype(&::cuDeviceGetAttribute) DeviceGetAttribute = nullptr;
  bool ok = false;
};

static const Drv& drv() {
  static Drv d = [] {
    Drv x;
    auto get = [](const char* name, void** fn) {
      cudaDriverEntryPointQueryResult q;
      return cudaGetDriverEntryPointByVersion(name, fn, 12000, cudaEnableDefault, &q) ==
                 cudaSuccess &&
             q == cudaDriverEntryPointSuccess && *fn != nullptr;
    };
    x.ok = get("cuMemAddressReserve", (void**)&x.MemAddressReserve) &&
           get("cuMemAddressFree", (void**)&x.MemAddressFree) &&
           get("cuMemCreate", (void**)&x.MemCreate) && get("cuMemRelease", (void**)&x.MemRelease) &&
           get("cuMemMap", (void**)&x.MemMap) && get("cuMemUnmap", (void**)&x.MemUnmap) &&
           get("cuMemSetAccess", (void**)&x.MemSetAccess) &&
           get("cuMemGetAllocationGranularity", (void**)&x.MemGetAllocationGranularity) &&
           get("cuGetErrorString", (void**)&x.GetErrorString) && get("cuDeviceGet", (void**)&x.DeviceGet) &&
           get("cuDeviceGetAttribute", (void**)&x.DeviceGetAttribute);
    return x;
  }();
  return d;
}

static recis_status cu_fail(CUresult r, const char* what) {
  const char* s = nullptr;
  if (drv().GetErrorString) drv().GetErrorString(r, &s);
  set_error(std::string(what) + ": " + (s ? s : "CUDA driver error"));
  return r == CUDA_ERROR_OUT_OF_MEMORY ? RECIS_ERR_OOM : RECIS_ERR_CUDA;
}

LaunchScope::LaunchScope(const char* n, cudaStream_t s) : name(n), stream(s), slot(-1) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_prof_on.load(std::memory_order_relaxed)) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    ProfRec r{n, pool_event(), pool_event()};
    cudaEventRecord(r.a, s);
    g_prof.push_back(r);
    slot = (int)g_prof.size() - 1;
  }
}

LaunchScope::~LaunchScope() {
  if (slot >= 0) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (slot < (int)g_prof.size()) cudaEventRecord(g_prof[slot].b, stream);
  }
}

// ---------------------------------------------------------------- VMM blocks
static recis_status vmm_reserve(VmmArray& a, size_t bytes) {
  const CUresult r = drv().MemAddressReserve(&a.va, bytes, 0, 0, 0);
  if (r != CUDA_SUCCESS) return cu_fail(r, "cuMemAddressReserve");
  a.reserved = bytes;
  a.mapped = 0;
  return RECIS_OK;
}

static recis_status vmm_map_to(VmmArray& a, size_t bytes, int dev) {
  if (bytes <= a.mapped) return RECIS_OK;
  if (bytes > a.reserved) {
    set_error("EmbeddingBlocks: address space reservation exhausted (raise max_rows)");
    return RECIS_ERR_TABLE_FULL;
  }
  const size_t sz = bytes - a.mapped;
  const int64_t cap = map_limit_bytes();
  if (cap > 0 && (int64_t)bytes > cap) {
    set_error("EmbeddingBlocks: mapping refused by the test cap on mapped bytes");
    return RECIS_ERR_OOM;
  }
  CUmemAllocationProp prop = {};
  prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
  if (a.host_numa >= 0) {  // host memory, reached by the GPU through the mapping
    prop.location.type = CU_MEM_LOCATION_TYPE_HOST_NUMA;
    prop.location.id = a.host_numa;
  } else {
    prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    prop.location.id = dev;
  }
  CUmemGenericAllocationHandle h;
  CUresult r = drv().MemCreate(&h, sz, &prop, 0);
  if (r != CUDA_SUCCESS) return cu_fail(r, "cuMemCreate (EmbeddingBlock)");
  r = drv().MemMap(a.va + a.mapped, sz, 0, h, 0);
  if (r != CUDA_SUCCESS) {
    drv().MemRelease(h);
    return cu_fail(r, "cuMemMap");
  }
  CUmemAccessDesc acc = {};
  acc.location.type = CU_MEM_LOCATION_TYPE_DEVICE;  // the GPU reads and writes every block
  acc.location.id = dev;
  acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;
  r = drv().MemSetAccess(a.va + a.mapped, sz, &acc, 1);
  if (r != CUDA_SUCCESS) {
    drv().MemUnmap(a.va + a.mapped, sz);
    drv().MemRelease(h);
    return cu_fail(r, "cuMemSetAccess");
  }
  a.handles.push_back(h);
  a.sizes.push_back(sz);
  a.mapped = bytes;
  return RECIS_OK;
}

static void vmm_release(VmmArray& a) {
  size_t off = 0;
  for (size_t i = 0; i < a.handles.size(); ++i) {
    drv().MemUnmap(a.va + off, a.sizes[i]);
    drv().MemRelease(a.handles[i]);
    off += a.sizes[i];
  }
  a.handles.clear();
  a.sizes.clear();
  if (a.va) drv().MemAddressFree(a.va, a.reserved);
  a.va = 0;
  a.reserved = a.mapped = 0;
}

static size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

// Map blocks until at least `rows` rows are backed.
static recis_status grow_rows(recis_table* t, int64_t rows) {
  if (rows <= t->mapped_rows) return RECIS_OK;
  if (rows > t->max_rows) {
    set_error("table full: live rows would exceed max_rows");
    return RECIS_ERR_TABLE_FULL;
  }
  // grow by whole blocks, at least a quarter of the current size
  int64_t target = std::max<int64_t>(rows, t->mapped_rows + t->mapped_rows / 4);
  target = (target + t->block_rows - 1) / t->block_rows * t->block_rows;
  target = std::min<int64_t>(target, t->max_rows);
  const size_t rb = round_up((size_t)target * t->row_bytes, t->gran);
  recis_status st = vmm_map_to(t->rows, std::min(rb, t->rows.reserved), t->dev);
  if (st != RECIS_OK) return st;
  const int64_t backed = (int64_t)(t->rows.mapped / t->row_bytes);
  const size_t kb = round_up((size_t)backed * sizeof(int64_t), t->gran);
  st = vmm_map_to(t->keys, std::min(kb, t->keys.reserved), t->dev);
  if (st != RECIS_OK) return st;
  int64_t m = std::min<int64_t>(backed, (int64_t)(t->keys.mapped / sizeof(int64_t)));
  if (t->cfg.evictable) {
    const size_t sb = round_up((size_t)m * sizeof(uint32_t), t->gran);
    st = vmm_map_to(t->seen, std::min(sb, t->seen.reserved), t->dev);
    if (st != RECIS_OK) return st;
    m = std::min<int64_t>(m, (int64_t)(t->seen.mapped / sizeof(uint32_t)));
  }
  // rows past max_rows stay unused even where a block's rounding backs them
  t->mapped_rows = std::min<int64_t>(m, t->max_rows);
  return RECIS_OK;
}

// A slot array of cap slots: device memory, or mapped pinned host memory for
// a host-placed IDMap (*host receives its host address, else null).
static cudaError_t alloc_slots(recis_table* t, int64_t cap, Slot** dev_ptr, Slot** host) {
  *host = nullptr;
  if (!(t->cfg.placement & RECIS_PLACE_IDMAP_HOST)) return cudaMalloc(dev_ptr, sizeof(Slot) * cap);
  cudaError_t e = cudaHostAlloc(host, sizeof(Slot) * cap, cudaHostAllocMapped);
  if (e != cudaSuccess) return e;
  e = cudaHostGetDevicePointer((void**)dev_ptr, *host, 0);
  if (e != cudaSuccess) {
    cudaFreeHost(*host);
    *host = nullptr;
  }
  return e;
}

static void free_slots(Slot* dev_ptr, Slot* host) {
  if (host) cudaFreeHost(host);
  else cudaFree(dev_ptr);
}

// IDMap growth: a new slot array, every live (key, row) re-inserted.
static recis_status grow_idmap(recis_table* t, int64_t keys_needed, cudaStream_t s) {
  int64_t cap = t->capacity;
  while ((double)keys_needed > kMaxLoad * (double)cap) cap *= 2;
  if (cap == t->capacity) return RECIS_OK;
  Slot* ns = nullptr;
  Slot* ns_host = nullptr;
  cudaError_t e = alloc_slots(t, cap, &ns, &ns_host);
  if (e != cudaSuccess) {
    set_error("IDMap growth: allocation failed");
    return RECIS_ERR_OOM;
  }
  e = cudaMemsetAsync(ns, 0xff, sizeof(Slot) * cap, s);
  if (e != cudaSuccess) return cuda_fail(e, "IDMap growth memset");
  Slot* old = t->slots;
  Slot* old_host = t->slots_host;
  const int64_t old_cap = t->capacity;
  t->slots = ns;
  t->slots_host = ns_host;
  t->capacity = cap;
  // the rehash drops tombstones and counts the slots it fills
  e = cudaMemsetAsync(&t->dstate->slots_used, 0, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return cuda_fail(e, "IDMap growth memset");
  e = launch_rehash(t, old, old_cap, s);
  if (e != cudaSuccess) return cuda_fail(e, "IDMap rehash");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "IDMap rehash");
  free_slots(old, old_host);
  unsigned long long used = 0;
  e = cudaMemcpy(&used, &t->dstate->slots_used, sizeof(used), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "IDMap rehash count");
  t->slots_upper = (int64_t)used;
  return RECIS_OK;
}

// Tighten the live-row bound with the newest progress event that has completed:
// the host-mapped count then covers at least every call up to that event.
static void refresh_mirror(recis_table* t) {
  for (int i = 0; i < t->ring_live; ++i) {
    const int k = (t->ring_next - 1 - i + recis_table::kRing) % recis_table::kRing;
    if (cudaEventQuery(t->ring[k]) == cudaSuccess) {
      const int64_t bound = (int64_t)t->mirror->next_free + (t->cum_issued - t->ring_cum[k]);
      if (bound < t->rows_upper) t->rows_upper = bound;
      const int64_t sbound = (int64_t)t->mirror->slots_used + (t->cum_issued - t->ring_cum[k]);
      if (sbound < t->slots_upper) t->slots_upper = sbound;
      t->ring_live = i;  // this event and older ones are consumed
      return;
    }
  }
}

static recis_status decode_status(int bits) {
  if (bits & kErrReservedKey) {
    set_error("an input key equals the reserved value -1");
    return RECIS_ERR_RESERVED_KEY;
  }
  if (bits & kErrTableFull) {
    set_error("table full: IDMap probe limit or row space exhausted");
    return RECIS_ERR_TABLE_FULL;
  }
  if (bits & kErrTimeout) {
    set_error("a bounded device-side wait gave up");
    return RECIS_ERR_TIMEOUT;
  }
  if (bits & kErrTagOverflow) {
    set_error("a transformed feature value is wider than its tag field");
    return RECIS_ERR_INVALID_ARG;
  }
  if (bits & kErrDuplicateImport) {
    set_error("import: key already present");
    return RECIS_ERR_INVALID_ARG;
  }
  if (bits & kErrBadOffsets) {
    set_error("bag offsets are not non-decreasing from 0 to N");
    return RECIS_ERR_INVALID_ARG;
  }
  return RECIS_OK;
}

// Synchronise the stream, read and clear the table's device status.
static recis_status take_status(recis_table* t, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  DevState h;
  e = cudaMemcpy(&h, t->dstate, sizeof(DevState), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  t->rows_upper = (int64_t)h.next_free;
  t->slots_upper = (int64_t)h.slots_used;
  t->ring_live = 0;
  t->mirror->error_seen = 0;
  if (h.status) {
    const int zero = 0;
    e = cudaMemcpy(&t->dstate->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  return decode_status(h.status);
}

// An error raised by earlier work that has finished is returned by the next call.
static recis_status pending_error(recis_table* t, cudaStream_t s) {
  if (t->mirror->error_seen) return take_status(t, s);
  return RECIS_OK;
}

// Make room for up to `n_new` new keys without waiting in the common case.
// device_checked: the call's kernels reject it as a whole when its actual new
// keys do not fit the mapped rows, so a bound past max_rows maps up to
// max_rows and lets the device decide; otherwise such a bound is an error.
static recis_status reserve(recis_table* t, int64_t n_new, cudaStream_t s,
                            bool device_checked = false) {
  refresh_mirror(t);
  int64_t need = t->rows_upper + n_new;
  if (device_checked) need = std::min(need, std::max(t->max_rows, t->rows_upper));
  // IDMap slots: keys with rows, candidates and tombstones all hold one
  const int64_t slots_need = std::max(need, t->slots_upper + n_new);
  if (need > t->mapped_rows || (double)slots_need > kMaxLoad * (double)t->capacity) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    DevState h;
    e = cudaMemcpy(&h, t->dstate, sizeof(DevState), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "row count read");
    t->rows_upper = (int64_t)h.next_free;
    t->slots_upper = (int64_t)h.slots_used;
    t->ring_live = 0;
    need = t->rows_upper + n_new;
    if (device_checked) need = std::min(need, std::max(t->max_rows, t->rows_upper));
    recis_status st = grow_rows(t, need);
    if (st != RECIS_OK) return st;
    st = grow_idmap(t, std::max(need, t->slots_upper + n_new), s);
    if (st != RECIS_OK) return st;
  }
  return RECIS_OK;
}

static void after_call(recis_table* t, int64_t n_new_bound, cudaStream_t s) {
  t->rows_upper += n_new_bound;
  t->slots_upper += n_new_bound;
  t->cum_issued += n_new_bound;
  const int k = t->ring_next;
  if (cudaEventRecord(t->ring[k], s) == cudaSuccess) {
    t->ring_cum[k] = t->cum_issued;
    t->ring_next = (k + 1) % recis_table::kRing;
    t->ring_live = std::min(t->ring_live + 1, recis_table::kRing);
  }
}

// ---------------------------------------------------------------- batch scratch
template <typename T>
static cudaError_t realloc_dev(T*& p, size_t count, bool zero) {
  if (p) cudaFree(p);
  p = nullptr;
  cudaError_t e = cudaMalloc(&p, sizeof(T) * std::max<size_t>(count, 1));
  if (e != cudaSuccess) return e;
  if (zero) e = cudaMemset(p, 0, sizeof(T) * std::max<size_t>(count, 1));
  return e;
}

int64_t unique_tiles_for(int64_t N);

recis_status batch_ensure(recis_batch* b, int64_t N, int64_t nbags, int D) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (b->dev >= 0 && b->dev != dev) {
    set_error("batch used on a different device than it was first used on");
    return RECIS_ERR_INVALID_ARG;
  }
  b->dev = dev;
  cudaError_t e = cudaSuccess;
  if (!b->ctl) {
    if ((e = realloc_dev(b->ctl, 1, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    if ((e = realloc_dev(b->bdev, 1, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    if ((e = realloc_dev(b->ss, 1, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
  }
  if (N > b->capN) {
    const int64_t cap = std::max<int64_t>(N + N / 4, 1 << 12);
    // index buffers start zeroed: even after a failed call every index read
    // from them stays inside its buffer
    for (int i = 0; i < 2; ++i) {
      if ((e = realloc_dev(b->kbuf[i], cap, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
      if ((e = realloc_dev(b->vbuf[i], cap, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    }
    if ((e = realloc_dev(b->uniq, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->rows, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->inv, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->seg_of, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->ss_meta, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->seg_start, cap + 1, true)) != cudaSuccess ||
        (e = realloc_dev(b->spos, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->gsrc, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->gfirst, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->bag_of, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->socc, cap, true)) != cudaSuccess ||
        (e = realloc_dev(b->multi_keys, cap / 2 + 1, false)) != cudaSuccess)
      return cuda_fail(e, "batch alloc");
    const int64_t st = (cap + kSortTile - 1) / kSortTile;
    if ((e = realloc_dev(b->sort_lookback, (size_t)st * 256, true)) != cudaSuccess)
      return cuda_fail(e, "batch alloc");
    b->sort_lookback_tiles = st;
    const int64_t ut = unique_tiles_for(cap);
    if ((e = realloc_dev(b->seg_lookback, (size_t)ut, true)) != cudaSuccess)
      return cuda_fail(e, "batch alloc");
    b->capN = cap;
  }
  b->seg_lookback_tiles = unique_tiles_for(N);
  if (nbags > b->capBags) {
    const int64_t cap = std::max<int64_t>(nbags + nbags / 4, 1 << 12);
    if ((e = realloc_dev(b->bag_counter, cap, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capBags = cap;
  }
  if (!b->side) {
    if ((e = cudaStreamCreateWithFlags(&b->side, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&b->ev_fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&b->ev_join, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&b->ev_pfork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&b->ev_probe, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "batch stream");
  }
  if (N > kSampleSortMaxN && N > b->capPocc) {
    const int64_t cap = N + N / 8;
    if ((e = realloc_dev(b->pocc, cap, false)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capPocc = cap;
  }
  if (N <= kSampleSortMaxN) {
    const int64_t th = samplesort_tiles_for(N) * kMaxBucketSlots;
    if (th > b->ss_th_cap) {
      const int64_t cap = th + th / 4;
      if ((e = realloc_dev(b->ss_th, cap, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
      b->ss_th_cap = cap;
    }
  }
  const int64_t cf = pool_chunk_for(N, D), cu = update_chunk_for(N, D);
  if ((N + cf - 1) / cf + 1 > b->capChunks) {
    const int64_t cap = (N + cf - 1) / cf + 1 + 1024;
    if ((e = realloc_dev(b->chunk_bag, cap, true)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capChunks = cap;
  }
  const int64_t nch = std::max((N + cf - 1) / cf, (N + cu - 1) / cu);
  const int64_t need = nch * 2 * D;
  if (need > b->capPartials) {
    const int64_t cap = need + need / 4 + 1024;
    if ((e = realloc_dev(b->partials, cap, false)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capPartials = cap;
  }
  // reduced gradients of long segments: one row per kShortSeg positions (a
  // long segment is the only one starting in its row's positions); the list
  // of long segments crossing a span end: at most one per span
  const int64_t gneed = ((N + kShortSeg - 1) / kShortSeg + 1) * (int64_t)D;
  if (gneed > b->capGbuf) {
    const int64_t cap = gneed + gneed / 4;
    if ((e = realloc_dev(b->gbuf, cap, false)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capGbuf = cap;
  }
  const int64_t sneed = (N + cu - 1) / cu + 1;
  if (sneed > b->capSegs) {
    const int64_t cap = sneed + sneed / 4;
    if ((e = realloc_dev(b->long_segs, cap, false)) != cudaSuccess) return cuda_fail(e, "batch alloc");
    b->capSegs = cap;
  }
  return RECIS_OK;
}

static void batch_free(recis_batch* b) {
  for (int i = 0; i < 2; ++i) {
    cudaFree(b->kbuf[i]);
    cudaFree(b->vbuf[i]);
  }
  cudaFree(b->sort_lookback);
  cudaFree(b->ctl);
  cudaFree(b->ss);
  cudaFree(b->ss_th);
  cudaFree(b->ss_meta);
  cudaFree(b->seg_lookback);
  cudaFree(b->uniq);
  cudaFree(b->rows);
  cudaFree(b->inv);
  cudaFree(b->seg_of);
  cudaFree(b->seg_start);
  cudaFree(b->spos);
  cudaFree(b->gsrc);
  cudaFree(b->gfirst);
  cudaFree(b->bag_counter);
  cudaFree(b->partials);
  cudaFree(b->gbuf);
  cudaFree(b->multi_keys);
  cudaFree(b->long_segs);
  cudaFree(b->bdev);
  cudaFree(b->chunk_bag);
  cudaFree(b->bag_of);
  cudaFree(b->pocc);
  cudaFree(b->socc);
  cudaFree(b->part_hist);
  cudaFree(b->dstate_local);
  if (b->side) cudaStreamDestroy(b->side);
  if (b->ev_fork) cudaEventDestroy(b->ev_fork);
  if (b->ev_join) cudaEventDestroy(b->ev_join);
  if (b->ev_pfork) cudaEventDestroy(b->ev_pfork);
  if (b->ev_probe) cudaEventDestroy(b->ev_probe);
}

static recis_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10) {
    set_error("this library is built for sm_100a (B200); the current device is not");
    return RECIS_ERR_NO_DEVICE;
  }
  return RECIS_OK;
}

// the shared forward / insert path
static recis_status lookup_impl(const LookupArgs& a, cudaStream_t s) {
  recis_table* t = a.t;
  recis_batch* b = a.b;
  recis_status st = pending_error(t, s);
  if (st != RECIS_OK) return st;
  st = reserve(t, a.N, s, a.N <= kSampleSortMaxN);
  if (st != RECIS_OK) return st;
  st = batch_ensure(b, a.N, (int64_t)a.F * a.B, t->D);
  if (st != RECIS_OK) return st;
  b->table = t;
  b->N = a.N;
  b->F = a.F;
  b->B = a.B;
  b->combiner = a.combiner;
  b->keys = a.keys;
  b->bag_offsets = a.bag_offsets;
  b->have_lookup = true;
  if (++b->call_seq == 0) b->call_seq = 1;
  t->clock += 1;  // this call's lookups touch rows at this clock
  cudaError_t e;
  const bool pool = a.pooled_out || a.unpooled_out;
  const int64_t cf = pool_chunk_for(a.N, t->D);
  if (pool) {
    // bag preparation on the side stream, overlapping the dedup
    if ((e = cudaEventRecord(b->ev_fork, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(b->side, b->ev_fork, 0)) != cudaSuccess ||
        (e = launch_bag_prep(a, cf, b->side)) != cudaSuccess ||
        (e = cudaEventRecord(b->ev_join, b->side)) != cudaSuccess)
      return cuda_fail(e, "bag preparation");
  }
  if (a.N > 0) {
    if (a.N <= kSampleSortMaxN) {
      if ((e = launch_sample_dedup(b, t, a.keys, a.N, a.insert, s)) != cudaSuccess)
        return cuda_fail(e, "dedup launch");
    } else {
      if ((e = launch_sort(b, t, a.keys, a.N, s)) != cudaSuccess) return cuda_fail(e, "sort launch");
      if ((e = launch_unique_insert(b, t, a.N, a.insert, s)) != cudaSuccess)
        return cuda_fail(e, "unique launch");
    }
    if (a.rows_out && (e = launch_rows_per_key(b, a.N, a.rows_out, s)) != cudaSuccess)
      return cuda_fail(e, "rows launch");
  } else {
    if ((e = cudaMemsetAsync(b->bdev, 0, sizeof(BatchDev), s)) != cudaSuccess)
      return cuda_fail(e, "memset");
  }
  if (pool) {
    if ((e = cudaStreamWaitEvent(s, b->ev_join, 0)) != cudaSuccess) return cuda_fail(e, "join");
    if ((e = launch_pool(a, cf, s)) != cudaSuccess) return cuda_fail(e, "pool launch");
  }
  after_call(t, a.N, s);
  return RECIS_OK;
}

// Synchronous: rows in use (live rows and the freed rows below them) and live
// rows of a table.
recis_status table_counts(recis_table* t, cudaStream_t s, int64_t* in_use, int64_t* live) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  DevState h;
  e = cudaMemcpy(&h, t->dstate, sizeof(DevState), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "size read");
  if (in_use) *in_use = (int64_t)h.next_free;
  if (live) *live = (int64_t)h.next_free - (int64_t)(h.free_tail - h.free_head);
  return RECIS_OK;
}

}  // namespace recis

using namespace recis;

extern "C" {

const char* recis_last_error_string(void) { return g_err.c_str(); }

recis_status recis_debug_set(int32_t what, int64_t value) {
  switch (what) {
    case RECIS_DEBUG_SPIN_LIMIT:
      if (value < 0 || value > INT32_MAX) return RECIS_ERR_INVALID_ARG;
      g_spin_limit.store(value == 0 ? kSpinLimit : (int)value);
      return RECIS_OK;
    case RECIS_DEBUG_MAP_LIMIT:
      if (value < 0) return RECIS_ERR_INVALID_ARG;
      g_map_limit.store(value);
      return RECIS_OK;
    default:
      set_error("debug_set: unknown setting");
      return RECIS_ERR_INVALID_ARG;
  }
}

int64_t recis_launch_count(void) { return g_launches.load(); }

recis_status recis_profile_enable(int32_t on) {
  g_prof_on.store(on != 0);
  return RECIS_OK;
}

int32_t recis_profile_collect(const char** names, int64_t* launches, double* total_ms,
                              int32_t max) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::vector<const char*> nm;
  std::vector<int64_t> cnt;
  std::vector<double> ms;
  for (auto& r : g_prof) {
    cudaEventSynchronize(r.b);
    float t = 0.f;
    cudaEventElapsedTime(&t, r.a, r.b);
    size_t i = 0;
    while (i < nm.size() && std::strcmp(nm[i], r.name) != 0) ++i;
    if (i == nm.size()) {
      nm.push_back(r.name);
      cnt.push_back(0);
      ms.push_back(0.0);
    }
    cnt[i] += 1;
    ms[i] += t;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  const int32_t n = (int32_t)std::min<size_t>(nm.size(), (size_t)std::max(max, 0));
  for (int32_t i = 0; i < n; ++i) {
    if (names) names[i] = nm[i];
    if (launches) launches[i] = cnt[i];
    if (total_ms) total_ms[i] = ms[i];
  }
  return n;
}

recis_status recis_feature_hash(const recis_feature_op* ops, int32_t F, const int64_t* values,
                                const int64_t* feat_offsets, int64_t* keys_out,
                                recis_stream_t stream) {
  if (F < 0 || F > 4096 || (F > 0 && (!ops || !feat_offsets))) {
    set_error("feature_hash: bad F, ops or feat_offsets");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(values, 8) || misaligned(keys_out, 8)) {
    set_error("feature_hash: values and keys_out must be 8-byte aligned");
    return RECIS_ERR_INVALID_ARG;
  }
  if (F == 0) return RECIS_OK;
  if (feat_offsets[0] != 0) {
    set_error("feature_hash: feat_offsets[0] must be 0");
    return RECIS_ERR_INVALID_ARG;
  }
  for (int f = 0; f < F; ++f) {
    const recis_feature_op& o = ops[f];
    if (feat_offsets[f + 1] < feat_offsets[f]) {
      set_error("feature_hash: feat_offsets must be non-decreasing");
      return RECIS_ERR_INVALID_ARG;
    }
    if ((o.flags & ~(RECIS_BUCKETIZE | RECIS_HASH | RECIS_MOD | RECIS_TAG | RECIS_FLOAT)) ||
        ((o.flags & RECIS_BUCKETIZE) && (o.flags & (RECIS_HASH | RECIS_MOD))) ||
        ((o.flags & RECIS_FLOAT) && !(o.flags & RECIS_BUCKETIZE)) ||
        ((o.flags & RECIS_BUCKETIZE) && o.n_bound > 0 && misaligned(o.boundaries, 8)) ||
        ((o.flags & RECIS_MOD) && o.mod == 0) ||
        ((o.flags & RECIS_BUCKETIZE) && (o.n_bound < 0 || (o.n_bound > 0 && !o.boundaries))) ||
        ((o.flags & RECIS_TAG) &&
         (o.tag_shift < 1 || o.tag_shift > 62 || o.tag >= (1ULL << (63 - o.tag_shift))))) {
      set_error("feature_hash: invalid feature op " + std::to_string(f));
      return RECIS_ERR_INVALID_ARG;
    }
  }
  if (feat_offsets[F] > 0 && (!values || !keys_out)) {
    set_error("feature_hash: null values or keys_out");
    return RECIS_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return RECIS_ERR_NO_DEVICE;
  {
    std::lock_guard<std::mutex> lk(g_feat_mu);
    if (!g_feat_status[dev]) {
      int* p = nullptr;
      cudaError_t e = cudaMalloc(&p, sizeof(int));
      if (e != cudaSuccess) return cuda_fail(e, "feature status alloc");
      cudaMemset(p, 0, sizeof(int));
      g_feat_status[dev] = p;
    }
  }
  const cudaError_t e = launch_feature_hash(ops, F, values, feat_offsets, keys_out,
                                            g_feat_status[dev], (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "feature_hash launch");
  return RECIS_OK;
}

recis_status recis_feature_status_sync(recis_stream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128 || !g_feat_status[dev]) return RECIS_OK;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h = 0;
  e = cudaMemcpy(&h, g_feat_status[dev], sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (h) cudaMemset(g_feat_status[dev], 0, sizeof(int));
  return decode_status(h);
}

recis_status recis_table_create(const recis_table_config* cfg, recis_stream_t stream,
                                recis_table_t* out) {
  if (!cfg || !out) {
    set_error("table_create: null argument");
    return RECIS_ERR_INVALID_ARG;
  }
  *out = nullptr;
  if (cfg->dim < 4 || cfg->dim > 1024 || cfg->dim % 4 != 0 ||
      (cfg->optimizer != RECIS_ADAGRAD && cfg->optimizer != RECIS_ADAM) ||
      cfg->initial_capacity < 0 || cfg->block_rows < 0 || cfg->max_rows < 0 ||
      !(cfg->eps >= 0.0) || !std::isfinite(cfg->lr) || cfg->admit_threshold < 0 ||
      cfg->admit_threshold > kMaxAdmitThreshold || (cfg->evictable != 0 && cfg->evictable != 1)) {
    set_error("table_create: invalid config (dim must be a multiple of 4 in [4, 1024])");
    return RECIS_ERR_INVALID_ARG;
  }
  recis_status st = check_device();
  if (st != RECIS_OK) return st;
  cudaFree(0);  // make the primary context current
  if (!drv().ok) {
    set_error("CUDA driver virtual-memory entry points unavailable");
    return RECIS_ERR_CUDA;
  }
  CUresult r = CUDA_SUCCESS;

  recis_table* t = new recis_table();
  t->cfg = *cfg;
  cudaGetDevice(&t->dev);
  t->D = cfg->dim;
  t->s = cfg->optimizer == RECIS_ADAGRAD ? 1 : 2;
  t->row_floats = t->D * (1 + t->s);
  t->row_bytes = sizeof(float) * t->row_floats;
  const double scale = cfg->init_scale > 0 ? cfg->init_scale : 1.0 / std::sqrt((double)t->D);
  t->init_two_s = 2.0f * (float)scale;
  t->block_rows = cfg->block_rows > 0 ? cfg->block_rows : 65536;
  t->max_rows = cfg->max_rows > 0 ? cfg->max_rows : (int64_t)1 << 28;
  if (t->max_rows > INT32_MAX) t->max_rows = INT32_MAX;  // row offsets are 31-bit in the kernels

  if (cfg->placement & ~(RECIS_PLACE_BLOCKS_HOST | RECIS_PLACE_IDMAP_HOST)) {
    delete t;
    set_error("table_create: unknown placement flags");
    return RECIS_ERR_INVALID_ARG;
  }
  if (cfg->placement & RECIS_PLACE_IDMAP_HOST) {
    int native = 0;
    cudaDeviceGetAttribute(&native, cudaDevAttrHostNativeAtomicSupported, t->dev);
    if (!native) {
      delete t;
      set_error("table_create: an IDMap in host memory needs native GPU atomics on host memory, "
                "which this system does not provide");
      return RECIS_ERR_INVALID_ARG;
    }
  }
  int host_numa = -1;
  if (cfg->placement & RECIS_PLACE_BLOCKS_HOST) {
    CUdevice cd = 0;
    int vmm_host = 0, numa = -1;
    if (drv().DeviceGet(&cd, t->dev) == CUDA_SUCCESS) {
      drv().DeviceGetAttribute(&vmm_host, CU_DEVICE_ATTRIBUTE_HOST_NUMA_VIRTUAL_MEMORY_MANAGEMENT_SUPPORTED, cd);
      drv().DeviceGetAttribute(&numa, CU_DEVICE_ATTRIBUTE_HOST_NUMA_ID, cd);
    }
    if (!vmm_host) {
      delete t;
      set_error("table_create: EmbeddingBlocks in host memory need host-NUMA virtual-memory mappings, "
                "which this driver and device do not provide");
      return RECIS_ERR_INVALID_ARG;
    }
    host_numa = numa < 0 ? 0 : numa;
    t->rows.host_numa = t->keys.host_numa = t->seen.host_numa = host_numa;
  }
  CUmemAllocationProp prop = {};
  prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
  prop.location.type = host_numa >= 0 ? CU_MEM_LOCATION_TYPE_HOST_NUMA : CU_MEM_LOCATION_TYPE_DEVICE;
  prop.location.id = host_numa >= 0 ? host_numa : t->dev;
  r = drv().MemGetAllocationGranularity(&t->gran, &prop, CU_MEM_ALLOC_GRANULARITY_RECOMMENDED);
  if (r != CUDA_SUCCESS) {
    delete t;
    return cu_fail(r, "cuMemGetAllocationGranularity");
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if ((st = vmm_reserve(t->rows, round_up((size_t)t->max_rows * t->row_bytes, t->gran))) != RECIS_OK ||
      (st = vmm_reserve(t->keys, round_up((size_t)t->max_rows * sizeof(int64_t), t->gran))) != RECIS_OK ||
      (cfg->evictable &&
       (st = vmm_reserve(t->seen, round_up((size_t)t->max_rows * sizeof(uint32_t), t->gran))) != RECIS_OK))
    goto fail;
  if ((st = grow_rows(t, std::max<int64_t>(cfg->initial_capacity, 1))) != RECIS_OK) goto fail;
  {
    int64_t cap = 1024;
    while ((double)cfg->initial_capacity > kMaxLoad * (double)cap) cap *= 2;
    t->capacity = cap;
    if ((e = alloc_slots(t, cap, &t->slots, &t->slots_host)) != cudaSuccess) {
      st = RECIS_ERR_OOM;
      set_error("IDMap allocation failed");
      goto fail;
    }
    if ((e = cudaMemsetAsync(t->slots, 0xff, sizeof(Slot) * cap, s)) != cudaSuccess) {
      st = cuda_fail(e, "IDMap init");
      goto fail;
    }
  }
  if ((e = cudaMalloc(&t->dstate, sizeof(DevState))) != cudaSuccess ||
      (e = cudaMemsetAsync(t->dstate, 0, sizeof(DevState), s)) != cudaSuccess ||
      (e = cudaHostAlloc(&t->mirror, sizeof(HostMirror), cudaHostAllocMapped)) != cudaSuccess ||
      (e = cudaHostGetDevicePointer((void**)&t->mirror_dev, t->mirror, 0)) != cudaSuccess) {
    st = cuda_fail(e, "table state allocation");
    goto fail;
  }
  std::memset((void*)t->mirror, 0, sizeof(HostMirror));
  for (int k = 0; k < recis_table::kRing; ++k) {
    if ((e = cudaEventCreateWithFlags(&t->ring[k], cudaEventDisableTiming)) != cudaSuccess) {
      st = cuda_fail(e, "event creation");
      goto fail;
    }
  }
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) {
    st = cuda_fail(e, "table init");
    goto fail;
  }
  *out = t;
  return RECIS_OK;
fail:
  recis_table_destroy(t);
  return st;
}

recis_status recis_table_destroy(recis_table_t t) {
  if (!t) return RECIS_OK;
  cudaDeviceSynchronize();
  vmm_release(t->rows);
  vmm_release(t->keys);
  vmm_release(t->seen);
  cudaFree(t->free_rows);
  free_slots(t->slots, t->slots_host);
  cudaFree(t->dstate);
  if (t->mirror) cudaFreeHost((void*)t->mirror);
  for (int k = 0; k < recis_table::kRing; ++k)
    if (t->ring[k]) cudaEventDestroy(t->ring[k]);
  delete t;
  return RECIS_OK;
}

recis_status recis_batch_create(recis_batch_t* out) {
  if (!out) return RECIS_ERR_INVALID_ARG;
  *out = new recis_batch();
  return RECIS_OK;
}

recis_status recis_batch_destroy(recis_batch_t b) {
  if (!b) return RECIS_OK;
  cudaDeviceSynchronize();
  batch_free(b);
  delete b;
  return RECIS_OK;
}

static recis_status check_lookup_args(recis_table_t t, recis_batch_t b, const int64_t* keys,
                                      int64_t N, const int64_t* bag_offsets, int32_t F, int64_t B,
                                      int32_t combiner, bool need_bags) {
  if (!t || !b) {
    set_error("null table or batch");
    return RECIS_ERR_INVALID_ARG;
  }
  if (N < 0 || N >= ((int64_t)1 << 30) || (N > 0 && !keys)) {
    set_error("N must be in [0, 2^30) and keys non-null");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(keys, 8) || misaligned(bag_offsets, 8)) {
    set_error("keys and bag_offsets must be 8-byte aligned");
    return RECIS_ERR_INVALID_ARG;
  }
  if (need_bags) {
    if (F < 0 || B < 0 || (int64_t)F * B >= ((int64_t)1 << 31) ||
        (combiner != RECIS_SUM && combiner != RECIS_MEAN)) {
      set_error("bad F, B or combiner");
      return RECIS_ERR_INVALID_ARG;
    }
    const int64_t nb = (int64_t)F * B;
    if ((nb > 0 && !bag_offsets) || (nb == 0 && N > 0)) {
      set_error("bag_offsets missing, or N > 0 with no bags");
      return RECIS_ERR_INVALID_ARG;
    }
  }
  return RECIS_OK;
}

recis_status recis_lookup_pooled(recis_table_t t, recis_batch_t b, const int64_t* keys, int64_t N,
                                 const int64_t* bag_offsets, int32_t F, int64_t B,
                                 int32_t combiner, float* pooled_out, float* unpooled_out,
                                 recis_stream_t stream) {
  recis_status st = check_lookup_args(t, b, keys, N, bag_offsets, F, B, combiner, true);
  if (st != RECIS_OK) return st;
  if (!pooled_out && !unpooled_out) {
    set_error("lookup_pooled: pooled_out and unpooled_out are both null");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(pooled_out, 16) || misaligned(unpooled_out, 16)) {
    set_error("lookup_pooled: pooled_out and unpooled_out must be 16-byte aligned");
    return RECIS_ERR_INVALID_ARG;
  }
  LookupArgs a{t, b, keys, N, bag_offsets, F, B, combiner, pooled_out, unpooled_out, nullptr, false};
  return lookup_impl(a, (cudaStream_t)stream);
}

recis_status recis_table_insert(recis_table_t t, recis_batch_t b, const int64_t* keys, int64_t N,
                                int64_t* rows_out, recis_stream_t stream) {
  recis_status st = check_lookup_args(t, b, keys, N, nullptr, 0, 0, RECIS_SUM, false);
  if (st != RECIS_OK) return st;
  if (misaligned(rows_out, 8)) {
    set_error("table_insert: rows_out must be 8-byte aligned");
    return RECIS_ERR_INVALID_ARG;
  }
  LookupArgs a{t, b, keys, N, nullptr, 0, 0, RECIS_SUM, nullptr, nullptr, rows_out, true};
  st = lookup_impl(a, (cudaStream_t)stream);
  b->have_lookup = false;  // no bags: nothing to back-propagate
  return st;
}

recis_status recis_backward_update(recis_table_t t, recis_batch_t b, const float* grad_pooled,
                                   const float* grad_unpooled, recis_stream_t stream) {
  if (!t || !b || !b->have_lookup || b->table != t) {
    set_error("backward_update: the batch holds no lookup of this table");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(grad_pooled, 16) || misaligned(grad_unpooled, 16)) {
    set_error("backward_update: grad_pooled and grad_unpooled must be 16-byte aligned");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  recis_status st = pending_error(t, s);
  if (st != RECIS_OK) return st;
  float lr_t = (float)t->cfg.lr, inv_sqrt_bc2 = 1.0f;
  if (t->cfg.optimizer == RECIS_ADAM) {
    t->step += 1;
    const double bc1 = 1.0 - std::pow(t->cfg.beta1, (double)t->step);
    const double bc2 = 1.0 - std::pow(t->cfg.beta2, (double)t->step);
    lr_t = (float)(t->cfg.lr / bc1);
    inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  }
  if (b->N > 0) {
    const cudaError_t e = launch_update(t, b, grad_pooled, grad_unpooled,
                                       update_chunk_for(b->N, t->D), lr_t, inv_sqrt_bc2, s);
    if (e != cudaSuccess) return cuda_fail(e, "update launch");
  }
  after_call(t, 0, s);
  return RECIS_OK;
}

recis_status recis_table_reserve(recis_table_t t, int64_t rows, recis_stream_t stream) {
  if (!t || rows < 0) {
    set_error("table_reserve: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  recis_status st = take_status(t, s);  // waits for the stream; exact live rows
  if (st != RECIS_OK) return st;
  const int64_t target = std::max(rows, t->rows_upper);
  st = grow_rows(t, target);
  if (st != RECIS_OK) return st;
  return grow_idmap(t, target, s);
}

recis_status recis_table_status_sync(recis_table_t t, recis_stream_t stream) {
  if (!t) return RECIS_ERR_INVALID_ARG;
  return take_status(t, (cudaStream_t)stream);
}


recis_status recis_table_size(recis_table_t t, int64_t* n_out, int64_t* step_out,
                              recis_stream_t stream) {
  if (!t) return RECIS_ERR_INVALID_ARG;
  recis_status st = table_counts(t, (cudaStream_t)stream, nullptr, n_out);
  if (st != RECIS_OK) return st;
  if (step_out) *step_out = t->step;
  return RECIS_OK;
}

recis_status recis_table_clock(recis_table_t t, int64_t* clock_out) {
  if (!t || !clock_out) return RECIS_ERR_INVALID_ARG;
  *clock_out = t->clock;
  return RECIS_OK;
}

recis_status recis_table_export(recis_table_t t, int64_t* keys, float* emb, float* state,
                                int64_t capacity, int64_t* n_out, int64_t* step_out,
                                recis_stream_t stream) {
  if (!t || capacity < 0) return RECIS_ERR_INVALID_ARG;
  int64_t in_use = 0, n = 0;
  recis_status st = table_counts(t, (cudaStream_t)stream, &in_use, &n);
  if (st != RECIS_OK) return st;
  if (n_out) *n_out = n;
  if (step_out) *step_out = t->step;
  const int64_t m = std::min(n, capacity);
  if (m == 0) return RECIS_OK;
  // the live rows (freed rows hold key -1) in ascending row order, in chunks
  const int64_t chunk = std::max<int64_t>(1, ((int64_t)64 << 20) / (int64_t)t->row_bytes);
  std::vector<int64_t> kb((size_t)std::min(chunk, in_use));
  std::vector<float> buf((emb || state) ? (size_t)std::min(chunk, in_use) * t->row_floats : 0);
  int64_t k = 0;
  for (int64_t r0 = 0; r0 < in_use && k < m; r0 += chunk) {
    const int64_t nr = std::min(chunk, in_use - r0);
    cudaError_t e = cudaMemcpy(kb.data(), (const int64_t*)t->keys.va + r0, sizeof(int64_t) * nr,
                               cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "export keys");
    if (emb || state) {
      e = cudaMemcpy(buf.data(), (const char*)t->rows.va + (size_t)r0 * t->row_bytes,
                     (size_t)nr * t->row_bytes, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return cuda_fail(e, "export rows");
    }
    for (int64_t i = 0; i < nr && k < m; ++i) {
      if (kb[i] == kEmptyKey) continue;
      if (keys) keys[k] = kb[i];
      const float* src = buf.data() + (size_t)i * t->row_floats;
      if (emb) std::memcpy(emb + (size_t)k * t->D, src, sizeof(float) * t->D);
      if (state) std::memcpy(state + (size_t)k * t->s * t->D, src + t->D, sizeof(float) * t->s * t->D);
      ++k;
    }
  }
  return RECIS_OK;
}

recis_status recis_table_import(recis_table_t t, const int64_t* keys, const float* emb,
                                const float* state, int64_t n, int64_t step,
                                recis_stream_t stream) {
  if (!t || n < 0 || (n > 0 && (!keys || !emb)) || step < 0) {
    set_error("import: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  for (int64_t i = 0; i < n; ++i)
    if (keys[i] == kEmptyKey) {
      set_error("import: reserved key -1");
      return RECIS_ERR_RESERVED_KEY;
    }
  recis_status st = pending_error(t, s);
  if (st != RECIS_OK) return st;
  st = reserve(t, n, s);
  if (st != RECIS_OK) return st;
  int64_t row0 = 0;  // imported rows go after every row in use
  st = table_counts(t, s, &row0, nullptr);
  if (st != RECIS_OK) return st;
  if (row0 + n > t->mapped_rows) {
    st = grow_rows(t, row0 + n);
    if (st != RECIS_OK) return st;
  }
  cudaError_t e;
  if (n > 0) {
    const int64_t chunk = std::max<int64_t>(1, ((int64_t)64 << 20) / (int64_t)t->row_bytes);
    std::vector<float> buf((size_t)std::min(chunk, n) * t->row_floats);
    for (int64_t r0 = 0; r0 < n; r0 += chunk) {
      const int64_t nr = std::min(chunk, n - r0);
      for (int64_t i = 0; i < nr; ++i) {
        float* dst = buf.data() + (size_t)i * t->row_floats;
        std::memcpy(dst, emb + (size_t)(r0 + i) * t->D, sizeof(float) * t->D);
        if (state) {
          std::memcpy(dst + t->D, state + (size_t)(r0 + i) * t->s * t->D,
                      sizeof(float) * t->s * t->D);
        } else {
          const float v = t->cfg.optimizer == RECIS_ADAGRAD ? (float)t->cfg.adagrad_init_acc : 0.f;
          for (int j = 0; j < t->s * t->D; ++j) dst[t->D + j] = v;
        }
      }
      e = cudaMemcpy((char*)t->rows.va + (size_t)(row0 + r0) * t->row_bytes, buf.data(),
                     (size_t)nr * t->row_bytes, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) return cuda_fail(e, "import rows");
    }
    int64_t* dkeys = nullptr;
    if ((e = cudaMalloc(&dkeys, sizeof(int64_t) * n)) != cudaSuccess) return cuda_fail(e, "import");
    e = cudaMemcpy(dkeys, keys, sizeof(int64_t) * n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = launch_import(t, dkeys, n, row0, t->clock, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(dkeys);
    if (e != cudaSuccess) return cuda_fail(e, "import");
    DevState h{};
    h.next_free = (unsigned long long)(row0 + n);
    e = cudaMemcpy(&t->dstate->next_free, &h.next_free, sizeof(h.next_free), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "import");
  }
  t->step = step;
  return take_status(t, s);
}

recis_status recis_batch_get_unique(recis_batch_t b, int64_t* uniq_out, int32_t* inv_out,
                                    int64_t* rows_out, int64_t capacity, int64_t* U_out,
                                    int64_t* n_new_out, recis_stream_t stream) {
  if (!b || !b->ctl || capacity < 0) return RECIS_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  BatchDev h;
  e = cudaMemcpy(&h, b->bdev, sizeof(BatchDev), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "batch read");
  const int64_t U = b->N > 0 ? (int64_t)h.U : 0;
  const int64_t m = std::min(U, capacity);
  if (uniq_out && m > 0 &&
      (e = cudaMemcpyAsync(uniq_out, b->uniq, sizeof(int64_t) * m, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy uniq");
  if (rows_out && m > 0 &&
      (e = cudaMemcpyAsync(rows_out, b->rows, sizeof(int64_t) * m, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy rows");
  if (inv_out && b->N > 0 &&
      (e = cudaMemcpyAsync(inv_out, b->inv, sizeof(int32_t) * b->N, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy inv");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (U_out) *U_out = U;
  if (n_new_out) *n_new_out = b->N > 0 ? (int64_t)h.n_new : 0;
  return RECIS_OK;
}

}  // extern "C"
