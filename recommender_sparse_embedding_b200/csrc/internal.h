// internal.h -- host-side structures and kernel launchers of the embedding engine.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/recis.h"
#include "common.cuh"

namespace recis {

// ---------------------------------------------------------------- sort
constexpr int kSortBits = 8;
constexpr int kSortPasses = 64 / kSortBits;
constexpr int kSortBlock = 256;
constexpr int kSortItems = 12;
constexpr int kSortTile = kSortBlock * kSortItems;  // 3072 keys per tile

// Per-call control block of the sort and of the unique pass.  The first
// kCtlZeroBytes bytes are cleared before every lookup.
struct SortCtl {
  unsigned int hist[kSortPasses][256];
  unsigned int tile_counter[kSortPasses];
  unsigned int ticket;
  unsigned int seg_tile_counter;
  unsigned int pad0[6];
  // written by the last CTA of the histogram kernel
  unsigned int active[kSortPasses];   // pass p moves keys (its digit is not constant)
  unsigned int ordinal[kSortPasses];  // number of active passes before p
  unsigned int n_active;
  unsigned int pad1[15];
  unsigned int base[kSortPasses][256];  // first output position of each digit
};
constexpr size_t kCtlZeroBytes = offsetof(SortCtl, active);

// Control block of the sample-sort dedup (samplesort.cu).  Every field is
// written by the kernels of each call before it is read; nothing is cleared
// on the host.
constexpr int kMaxSplitters = 2048;       // distinct splitters <= 2047
constexpr int kMaxBucketSlots = 4096;     // buckets 0 .. 2 * nsplit (<= 4094)
constexpr int kMaxSample = 8192;          // sample size of the largest batches
// Segments (occurrences of one unique key) longer than this are summed by a
// separate chunked reduction in the backward; the dedup marks their positions.
constexpr int kShortSeg = 16;
struct SsCtl {
  unsigned nsplit, nb, nbp, pad0;         // splitters, buckets, buckets rounded up to 32
  unsigned ticket_scan, ticket_local, pad1, pad2;
  uint64_t samp[kMaxSample];              // the sorted sample (ukey order)
  uint64_t cand[2][kMaxSplitters];  // candidate splitters of this call and the next
  unsigned tot[kMaxBucketSlots];          // keys per bucket
  unsigned base[kMaxBucketSlots];         // first sorted position of each bucket
  unsigned hcnt[kMaxBucketSlots];         // distinct keys (heads) per bucket
  unsigned ncnt[kMaxBucketSlots];         // new keys per bucket
  unsigned hpre[kMaxBucketSlots];         // heads in earlier buckets of the same local CTA
  unsigned npre[kMaxBucketSlots];         // new keys in earlier buckets of the same local CTA
  unsigned long long cta_tot[kMaxBucketSlots / 2];  // per local CTA: new keys << 32 | heads
  unsigned long long cta_pre[kMaxBucketSlots / 2];  // the same, summed over earlier local CTAs
};
constexpr int64_t kSampleSortMaxN = (int64_t)1600 * 1000;  // larger batches use the radix sort

// Per-batch device scalars.
struct BatchDev {
  unsigned long long row_base;  // table's next_free when the lookup started
  unsigned long long free_base; // table's free_head when the lookup started
  unsigned long long free_avail;// freed rows queued then (free_tail - free_head)
  unsigned int U;               // unique keys of the last lookup (0 when it was rejected)
  unsigned int n_new;           // new keys of the last lookup
  unsigned int nseg_med;        // long segments cut by seg_reduce span ends, combined by one lane group
  unsigned int nseg_huge;       // ... over many spans, combined by a whole CTA
  unsigned int seg_work;        // work counter of the combine
  unsigned int nmulti;          // keys seen 2 to kShortSeg times (sample-sort path)
  unsigned int reject_call;     // call number of a lookup rejected as a whole (reserved key,
                                // or its new keys overflow the row space)
};

// ---------------------------------------------------------------- table
struct VmmArray {
  CUdeviceptr va = 0;
  size_t reserved = 0;   // bytes of address space
  size_t mapped = 0;     // bytes backed by physical blocks
  int host_numa = -1;    // >= 0: blocks are host memory of this NUMA node
  std::vector<CUmemGenericAllocationHandle> handles;
  std::vector<size_t> sizes;
};

}  // namespace recis

struct recis_table {
  int dev = 0;
  recis_table_config cfg{};
  int D = 0, s = 0, row_floats = 0;
  size_t row_bytes = 0;
  float init_two_s = 0.f;
  size_t gran = 0;              // VMM granularity
  int64_t block_rows = 0;
  int64_t max_rows = 0;
  int64_t mapped_rows = 0;
  recis::VmmArray rows;         // [row][emb D | state s*D] fp32
  recis::VmmArray keys;         // [row] int64, key of each row (-1: freed)
  recis::VmmArray seen;         // [row] uint32, clock of the last lookup that touched it (evictable tables)
  int32_t* free_rows = nullptr; // queue of freed rows (DevState free_head .. free_tail)
  int64_t free_cap = 0;         // entries of free_rows
  int64_t clock = 0;            // lookups so far
  int64_t slots_upper = 0;      // upper bound on IDMap slots holding a key
  recis::Slot* slots = nullptr; // IDMap (device address; mapped pinned host memory with PLACE_IDMAP_HOST)
  recis::Slot* slots_host = nullptr;  // host address of a host-placed IDMap
  int64_t capacity = 0;         // slots, power of two
  recis::DevState* dstate = nullptr;
  recis::HostMirror* mirror = nullptr;  // host-mapped
  recis::HostMirror* mirror_dev = nullptr;
  // progress events: ring[k] recorded after a call, when cum_issued was ring_cum[k]
  static constexpr int kRing = 8;
  cudaEvent_t ring[kRing] = {};
  int64_t ring_cum[kRing] = {};
  int ring_next = 0;
  int ring_live = 0;            // recorded events not yet consumed (newest first)
  int64_t cum_issued = 0;       // sum of N over all lookups issued
  int64_t rows_upper = 0;       // upper bound on live rows
  int64_t step = 0;             // Adam step counter
};

struct recis_batch {
  int dev = -1;
  int64_t capN = 0;             // occurrence capacity of the N-sized buffers
  int64_t capBags = 0;
  int64_t capPartials = 0;      // doubles
  uint64_t* kbuf[2] = {nullptr, nullptr};
  uint32_t* vbuf[2] = {nullptr, nullptr};
  unsigned long long* sort_lookback = nullptr;  // [tiles][256], epoch-tagged
  int64_t sort_lookback_tiles = 0;
  recis::SortCtl* ctl = nullptr;
  unsigned long long* seg_lookback = nullptr;   // [tiles], cleared per call (follows ctl)
  recis::SsCtl* ss = nullptr;                    // sample-sort control
  uint32_t* ss_th = nullptr;                     // [tiles][2048] tile histograms
  uint64_t* ss_meta = nullptr;                   // [capN] per sorted position
  int64_t ss_th_cap = 0;
  int64_t seg_lookback_tiles = 0;
  int64_t* uniq = nullptr;
  int64_t* rows = nullptr;
  int32_t* inv = nullptr;
  int32_t* seg_of = nullptr;    // segment (unique index) of each sorted position
  int32_t* seg_start = nullptr; // [U+1] first sorted position of each unique
  uint32_t* spos = nullptr;     // [capN] sorted position of each occurrence
  int4* gsrc = nullptr;         // [capN] per sorted position: {gradient row, bag length, occurrence, 0}
  int4* gfirst = nullptr;       // [capN] per unique key: the same, of one of its occurrences
  int32_t* chunk_bag = nullptr; // bag of each pool chunk's first occurrence
  int32_t* bag_of = nullptr;    // [capN] bag of every occurrence (written beside the dedup)
  int64_t* pocc = nullptr;      // [capN] IDMap result of each head, by sorted position (radix-sort path)
  int64_t capPocc = 0;
  // table-less dedup of the sharded path (recis_batch_dedup, recis_reduce_grad)
  int32_t* socc = nullptr;      // [capN] occurrence at each sorted position
  recis::DevState* dstate_local = nullptr;  // status word of the batch's own calls
  int64_t dedup_N = -1;         // occurrences of the last batch dedup (-1: none)
  unsigned* part_hist = nullptr;  // recis_partition_keys: per-tile owner counts, then offsets
  int64_t capPart = 0;
  int64_t capChunks = 0;
  cudaStream_t side = nullptr;  // bag preparation runs here, beside the dedup
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaEvent_t ev_pfork = nullptr, ev_probe = nullptr;  // IDMap probes beside the sort
  int cand_parity = 0;          // which candidate array the next call reads
  int64_t cand_n = 0;           // batch size that wrote it (0: none yet)
  int cand_splits = 0;          // its splitter slots (quantiles written: cand_splits - 1)
  int32_t* bag_counter = nullptr;  // [capBags]
  double* partials = nullptr;
  float* gbuf = nullptr;          // [chunks][D] reduced gradients of long segments
  int32_t* multi_keys = nullptr;  // [N/2] unique keys seen 2 to kShortSeg times (sample-sort path)
  int2* long_segs = nullptr;      // [capSegs] {start, end} of long segments cut by span ends
  int64_t capSegs = 0;
  int64_t capGbuf = 0;            // floats
  recis::BatchDev* bdev = nullptr;
  uint32_t epoch = 0;
  uint32_t call_seq = 0;          // number of the current lookup on this batch (never 0)
  // the last lookup, for the backward
  recis_table* table = nullptr;
  int64_t N = 0;
  int32_t F = 0;
  int64_t B = 0;
  int32_t combiner = 0;
  const int64_t* keys = nullptr;
  const int64_t* bag_offsets = nullptr;
  bool have_lookup = false;
  bool backward_done = true;
};

namespace recis {

void set_error(const std::string& msg);

// Device arrays are read and written with vector loads and copies: int64
// arrays must be 8-byte aligned, float rows 16-byte aligned.  True when p
// (non-null) is not a multiple of `bytes`, a power of two.
inline bool misaligned(const void* p, uintptr_t bytes) { return ((uintptr_t)p & (bytes - 1)) != 0; }

// Test hooks (recis_debug_set): the bound of the device-side spin-waits, and
// a cap on the EmbeddingBlock bytes a table may map (0 = none).
int spin_limit();
int64_t map_limit_bytes();

// Launches kernel<<<grid, block, smem, s>>>(args...) with programmatic
// stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}
recis_status cuda_fail(cudaError_t e, const char* what);

// launch bookkeeping (tracing)
struct LaunchScope {
  LaunchScope(const char* name, cudaStream_t s);
  ~LaunchScope();
  const char* name;
  cudaStream_t stream;
  int slot;
};

// ---- launchers (each returns the CUDA error of the launch)
cudaError_t launch_feature_hash(const recis_feature_op* ops, int F, const int64_t* values,
                                const int64_t* feat_offsets, int64_t* keys_out, int* dev_status,
                                cudaStream_t s);

struct LookupArgs {
  recis_table* t;
  recis_batch* b;
  const int64_t* keys;
  int64_t N;
  const int64_t* bag_offsets;
  int32_t F;
  int64_t B;
  int32_t combiner;
  float* pooled_out;
  float* unpooled_out;
  int64_t* rows_out;  // insert path: row per occurrence
  bool insert;        // bulk insert (keys may arrive sorted): fresh splitters, none kept
};

cudaError_t launch_sort(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N,
                        cudaStream_t s);
cudaError_t launch_unique_insert(recis_batch* b, recis_table* t, int64_t N, bool insert, cudaStream_t s);
cudaError_t launch_sample_dedup(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N,
                                bool insert, cudaStream_t s);
int samplesort_splits_for(int64_t N);
int64_t samplesort_tiles_for(int64_t N);
cudaError_t launch_pool(const LookupArgs& a, int64_t chunk, cudaStream_t s);
cudaError_t launch_bag_prep(const LookupArgs& a, int64_t chunk, cudaStream_t s);
cudaError_t launch_rows_per_key(recis_batch* b, int64_t N, int64_t* rows_out, cudaStream_t s);
cudaError_t launch_update(recis_table* t, recis_batch* b, const float* grad_pooled,
                          const float* grad_unpooled, int64_t chunk, float lr_t, float inv_sqrt_bc2,
                          cudaStream_t s);
cudaError_t launch_import(recis_table* t, const int64_t* keys, int64_t n, int64_t row0,
                          int64_t clock, cudaStream_t s);
recis_status table_counts(recis_table* t, cudaStream_t s, int64_t* in_use, int64_t* live);
recis_status batch_ensure(recis_batch* b, int64_t N, int64_t nbags, int D);
cudaError_t launch_rehash(recis_table* t, const Slot* old_slots, int64_t old_cap, cudaStream_t s);

int64_t pool_chunk_for(int64_t N, int D);
int64_t update_chunk_for(int64_t N, int D);

}  // namespace recis
