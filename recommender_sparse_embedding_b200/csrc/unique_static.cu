// unique_static.cu -- an allocation-free dedup entry point (recis_unique_static).
//
// Who needs it: callers that must not allocate device memory -- code running
// inside another framework's memory pool that forbids foreign cudaMalloc
// calls, callers that record work into a CUDA graph with allocation disabled,
// or processes that budget device memory up front and treat any later
// allocation as a failure.  The regular path keeps its scratch in a
// recis_batch_t that grows with cudaMalloc; this variant keeps all of it in
// one file-scope __device__ array of fixed size instead, so it never
// allocates.  The price: that array is reserved on every GPU that loads the
// library, for as long as the process lives, and N is capped.
//
// It runs the same sort kernels as the regular path (launch_sort, pointed at
// the static array), then its own dedup-only variant of the unique pass: no
// IDMap, no rows, just the ascending unique keys, the inverse index and U.
#include <mutex>

#include "internal.h"

namespace recis {

namespace {

constexpr int64_t kStaticMaxKeys = (int64_t)1 << 18;  // 262,144 keys per call
constexpr int kUoBlock = 256, kUoItems = 4, kUoTile = kUoBlock * kUoItems;
constexpr int64_t kStaticSortTiles = (kStaticMaxKeys + kSortTile - 1) / kSortTile;
constexpr int64_t kStaticUniqueTiles = (kStaticMaxKeys + kUoTile - 1) / kUoTile;

struct StaticScratch {
  SortCtl ctl;
  DevState st;
  BatchDev bdev;
  unsigned long long seg_lookback[kStaticUniqueTiles];
  unsigned long long sort_lookback[kStaticSortTiles * 256];
  uint64_t kbuf[2][kStaticMaxKeys];
  uint32_t vbuf[2][kStaticMaxKeys];
};

// The scratch: about 6.3 MB per GPU, zero at module load.
static __device__ __align__(256) unsigned char g_unique_scratch[sizeof(StaticScratch)];

std::mutex g_setup_mu;
StaticScratch* g_scratch_addr[128] = {nullptr};
uint32_t g_epoch[128] = {0};

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Dedup-only pass over the sorted (key, occurrence) pairs: head flags, a
// decoupled look-back over tiles for the unique index, then uniq / inv.  The
// last tile (which knows the total after its look-back) writes U, or -1 when a
// bounded wait gave up here or in the sort.
__global__ void __launch_bounds__(kUoBlock) unique_only_kernel(
    const int64_t* __restrict__ in_keys, StaticScratch* sc, int64_t N, int64_t* uniq,
    int32_t* inv, int64_t* U_out, int spin_max) {
  __shared__ uint64_t s_last[kUoBlock];
  __shared__ unsigned s_scan[kUoBlock / 32];
  __shared__ unsigned s_tile;
  __shared__ unsigned long long s_prefix;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(&sc->ctl.seg_tile_counter, 1u);
  __syncthreads();
  const unsigned tile = s_tile;
  const unsigned na = sc->ctl.n_active;
  const uint64_t* ks = na == 0 ? nullptr : sc->kbuf[(na - 1) & 1];
  const uint32_t* vs = na == 0 ? nullptr : sc->vbuf[(na - 1) & 1];
  const int64_t tbase = (int64_t)tile * kUoTile;
  const int64_t pos0 = tbase + (int64_t)tid * kUoItems;
  uint64_t k[kUoItems];
  uint32_t v[kUoItems];
#pragma unroll
  for (int j = 0; j < kUoItems; ++j) {
    const int64_t pos = pos0 + j;
    k[j] = pos < N ? (ks ? ks[pos] : to_ukey(in_keys[pos])) : 0;
    v[j] = pos < N ? (vs ? vs[pos] : (uint32_t)pos) : 0;
  }
  s_last[tid] = k[kUoItems - 1];
  __syncthreads();
  bool have_prev = true;
  uint64_t prev = 0;
  if (tid > 0)
    prev = s_last[tid - 1];
  else if (tbase > 0)
    prev = ks ? ks[tbase - 1] : to_ukey(in_keys[tbase - 1]);
  else
    have_prev = false;
  bool head[kUoItems];
  unsigned nh = 0;
#pragma unroll
  for (int j = 0; j < kUoItems; ++j) {
    const uint64_t pk = j == 0 ? prev : k[j - 1];
    head[j] = pos0 + j < N && (!(j == 0 ? have_prev : true) || pk != k[j]);
    nh += head[j];
  }
  unsigned x = nh;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_scan[w] = x;
  __syncthreads();
  unsigned wpre = 0, tot = 0;
#pragma unroll
  for (int ww = 0; ww < kUoBlock / 32; ++ww) {
    if (ww < w) wpre += s_scan[ww];
    tot += s_scan[ww];
  }
  const unsigned excl = wpre + x - nh;
  if (tid == 0) {
    unsigned long long* my = sc->seg_lookback + tile;
    unsigned long long hx = 0;
    if (tile == 0) {
      st_relaxed(my, (2ULL << 62) | tot);
    } else {
      st_relaxed(my, (1ULL << 62) | tot);
      int64_t t = (int64_t)tile - 1;
      int spins = 0;
      while (t >= 0) {
        const unsigned long long e = ld_relaxed(sc->seg_lookback + t);
        const unsigned long long flag = e >> 62;
        if (flag == 0) {
          if (++spins > spin_max) {
            atomicOr(&sc->st.status, kErrTimeout);
            break;
          }
          __nanosleep(32);
          continue;
        }
        hx += e & 0xffffffffULL;
        if (flag == 2) break;
        --t;
      }
      st_relaxed(my, (2ULL << 62) | (hx + tot));
    }
    s_prefix = hx;
  }
  __syncthreads();
  unsigned hrun = (unsigned)s_prefix + excl;
#pragma unroll
  for (int j = 0; j < kUoItems; ++j) {
    const int64_t pos = pos0 + j;
    if (pos >= N) break;
    if (head[j]) {
      uniq[hrun] = from_ukey(k[j]);
      ++hrun;
    }
    if (v[j] < (uint64_t)N) inv[v[j]] = (int32_t)(hrun - 1);
  }
  if (tile == gridDim.x - 1 && tid == 0) {
    __threadfence();
    const bool failed = (*(volatile int*)&sc->st.status & kErrTimeout) != 0;
    *U_out = failed ? -1 : (int64_t)(s_prefix + tot);
  }
}

}  // namespace

}  // namespace recis

using namespace recis;

extern "C" recis_status recis_unique_static(const int64_t* keys, int64_t N, int64_t* uniq_out,
                                            int32_t* inv_out, int64_t* U_out,
                                            recis_stream_t stream) {
  if (N < 0 || N > kStaticMaxKeys) {
    set_error("recis_unique_static: N must be in [0, 262144] (the size of its static scratch)");
    return RECIS_ERR_INVALID_ARG;
  }
  if (!U_out || (N > 0 && (!keys || !uniq_out || !inv_out))) {
    set_error("recis_unique_static: null argument");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(keys, 8) || misaligned(uniq_out, 8) || misaligned(inv_out, 4) || misaligned(U_out, 8)) {
    set_error("recis_unique_static: misaligned array (int64 arrays 8-byte, inv_out 4-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return RECIS_ERR_NO_DEVICE;
  cudaStream_t s = (cudaStream_t)stream;
  StaticScratch* sc = nullptr;
  uint32_t epoch = 0;
  {
    // set-up, once per device with that device current: the host needs the
    // device address of the array (its host-side name is only a stand-in)
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_unique_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static scratch)");
      g_scratch_addr[dev] = static_cast<StaticScratch*>(p);
    }
    sc = g_scratch_addr[dev];
    // this call's sort tags its passes epoch+1, epoch+2, ... skipping 0 (see
    // launch_sort, which also clears the look-back array when the tag wraps);
    // the next call starts where this one ends
    epoch = g_epoch[dev];
    uint32_t last = epoch;
    for (int p = 0; p < kSortPasses; ++p) {
      last += 1;
      if (last == 0) last = 1;
    }
    g_epoch[dev] = last;
  }
  if (N == 0) {
    e = cudaMemsetAsync(U_out, 0, sizeof(int64_t), s);
    return e == cudaSuccess ? RECIS_OK : cuda_fail(e, "cudaMemsetAsync");
  }
  e = cudaMemsetAsync(&sc->st, 0, sizeof(DevState), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  // the regular sort kernels, pointed at the static scratch
  recis_batch b;
  recis_table t;
  b.kbuf[0] = sc->kbuf[0];
  b.kbuf[1] = sc->kbuf[1];
  b.vbuf[0] = sc->vbuf[0];
  b.vbuf[1] = sc->vbuf[1];
  b.sort_lookback = sc->sort_lookback;
  b.sort_lookback_tiles = kStaticSortTiles;
  b.ctl = &sc->ctl;
  b.seg_lookback = sc->seg_lookback;
  b.seg_lookback_tiles = (N + kUoTile - 1) / kUoTile;
  b.bdev = &sc->bdev;
  b.epoch = epoch;
  t.dstate = &sc->st;
  t.mirror_dev = nullptr;
  e = launch_sort(&b, &t, keys, N, s);
  if (e != cudaSuccess) return cuda_fail(e, "sort launch");
  const unsigned tiles = (unsigned)((N + kUoTile - 1) / kUoTile);
  unique_only_kernel<<<tiles, kUoBlock, 0, s>>>(keys, sc, N, uniq_out, inv_out, U_out, spin_limit());
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "unique launch");
  return RECIS_OK;
}
