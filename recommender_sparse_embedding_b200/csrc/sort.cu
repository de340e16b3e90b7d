// sort.cu -- stable LSD radix sort of (key, occurrence index) pairs: the first
// half of the dedup step (RecIS README, Key optimisations > Distributed
// optimisation: requests are merged and deduplicated before the lookup).
//
// Design (one-sweep LSD radix sort, 8-bit digits):
//   * sort_hist_kernel reads the keys once and builds the histograms of all
//     eight digit positions; its last CTA marks the passes whose digit is the
//     same for every key as inactive (they would not move anything) and writes
//     each active pass's digit bases.  It also checks for the reserved key and
//     snapshots the table's next free row for the unique pass.
//   * sort_pass_kernel runs once per digit position.  A CTA takes the next tile
//     id from an atomic counter (so every earlier tile is already running),
//     ranks its 2048 keys with warp match/ballot, publishes its digit counts,
//     and resolves its global offsets by decoupled look-back over the earlier
//     tiles' published counts (bounded wait).  The tile is reordered in shared
//     memory so the scatter writes runs of consecutive addresses.
// Keys are mapped to unsigned order (sign bit flipped); values are the
// occurrence indices (generated in the first active pass).
#include "internal.h"

namespace recis {

namespace {

constexpr unsigned kFlagAgg = 1u, kFlagIncl = 2u;

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__global__ void __launch_bounds__(256) sort_hist_kernel(const int64_t* __restrict__ keys,
                                                        int64_t N, SortCtl* ctl, DevState* st,
                                                        HostMirror* mirror, BatchDev* bdev,
                                                        uint32_t call_id) {
  constexpr int kPer = 8;  // keys per thread per round, all loaded before they are counted
  __shared__ unsigned int sh[kSortPasses][256];
  __shared__ bool s_last;
  for (int i = threadIdx.x; i < kSortPasses * 256; i += blockDim.x) (&sh[0][0])[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  bool reserved = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * kPer;
  // warp-uniform trip count so that the votes see the whole warp
  const int64_t base0 = ((int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) * kPer;
  for (int64_t wb = base0; wb < N; wb += stride) {
    int64_t k[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int64_t i = wb + j * 32 + lane;
      k[j] = i < N ? __ldcs(keys + i) : 0;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const bool valid = wb + j * 32 + lane < N;
      reserved |= valid && (k[j] == kEmptyKey);
      const uint64_t u = to_ukey(k[j]);
      const bool full = __all_sync(0xffffffffu, valid);
#pragma unroll
      for (int p = 0; p < kSortPasses; ++p) {
        const unsigned d = (unsigned)(u >> (p * kSortBits)) & 255u;
        // a digit the whole warp shares (the constant high digits of tagged
        // keys) is one add of 32; the others one shared atomic per key
        if (full && __all_sync(0xffffffffu, d == __shfl_sync(0xffffffffu, d, 0))) {
          if (lane == 0) atomicAdd(&sh[p][d], 32u);
        } else if (valid) {
          atomicAdd(&sh[p][d], 1u);
        }
      }
    }
  }
  if (__any_sync(0xffffffffu, reserved) && lane == 0) {
    bdev->reject_call = call_id;  // the unique pass then inserts nothing
    raise_error(st, mirror, kErrReservedKey);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kSortPasses * 256; i += blockDim.x) {
    const unsigned c = (&sh[0][0])[i];
    if (c) atomicAdd(&(&ctl->hist[0][0])[i], c);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&ctl->ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last CTA plans the passes: warp p scans the 256 digit counts of pass p
  __shared__ unsigned int s_active[kSortPasses];
  const int wp = threadIdx.x >> 5;  // blockDim == 256: one warp per pass
  unsigned c[8];
  unsigned run = 0;
  bool one_bucket = false;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    c[q] = __ldcg(&ctl->hist[wp][lane * 8 + q]);
    one_bucket |= c[q] == (unsigned)N;
    run += c[q];
  }
  unsigned x = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  unsigned base = x - run;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    ctl->base[wp][lane * 8 + q] = base;
    base += c[q];
  }
  one_bucket = __any_sync(0xffffffffu, one_bucket);
  if (lane == 0) s_active[wp] = one_bucket ? 0u : 1u;
  __syncthreads();
  if (threadIdx.x == 0) {
    bdev->row_base = *(volatile unsigned long long*)&st->next_free;
    const unsigned long long fh = *(volatile unsigned long long*)&st->free_head;
    bdev->free_base = fh;
    bdev->free_avail = *(volatile unsigned long long*)&st->free_tail - fh;
    bdev->nseg_med = 0;  // the backward's long-segment lists start empty
    bdev->nseg_huge = 0;
    bdev->seg_work = 0;
    unsigned n = 0;
    for (int p = 0; p < kSortPasses; ++p) {
      ctl->active[p] = s_active[p];
      ctl->ordinal[p] = n;
      n += s_active[p];
    }
    ctl->n_active = n;
  }
}

// four CTAs per SM (64 registers a thread): 11 % faster on the 32.8M-key
// step than three with 80 registers, the look-back waits of more tiles
// overlapping
__global__ void __launch_bounds__(kSortBlock, 4) sort_pass_kernel(
    int P, const int64_t* __restrict__ in_keys, uint64_t* kb0, uint64_t* kb1, uint32_t* vb0,
    uint32_t* vb1, int64_t N, SortCtl* ctl, unsigned long long* lookback, uint32_t epoch,
    DevState* st, HostMirror* mirror, int spin_max) {
  if (!ctl->active[P]) return;
  const unsigned ord = ctl->ordinal[P];
  const uint64_t* ksrc = (ord & 1) ? kb0 : kb1;  // ord-1 parity
  const uint32_t* vsrc = (ord & 1) ? vb0 : vb1;
  uint64_t* kdst = (ord & 1) ? kb1 : kb0;
  uint32_t* vdst = (ord & 1) ? vb1 : vb0;
  const bool from_input = ord == 0;

  __shared__ uint64_t s_keys[kSortTile];
  __shared__ uint32_t s_vals[kSortTile];
  __shared__ unsigned int s_whist[kSortBlock / 32][256];
  __shared__ unsigned int s_doff[256];
  __shared__ int s_glob[256];
  __shared__ unsigned int s_wsum[kSortBlock / 32];
  __shared__ unsigned int s_tile;

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < (kSortBlock / 32) * 256; i += kSortBlock) (&s_whist[0][0])[i] = 0;
  if (tid == 0) s_tile = atomicAdd(&ctl->tile_counter[P], 1u);
  __syncthreads();
  const unsigned tile = s_tile;
  const int64_t tbase = (int64_t)tile * kSortTile;
  const int shift = P * kSortBits;

  uint64_t k[kSortItems];
  uint32_t v[kSortItems];
  unsigned rank[kSortItems];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t pos = tbase + w * (kSortItems * 32) + j * 32 + lane;
    if (pos < N) {
      if (from_input) {
        k[j] = to_ukey(in_keys[pos]);
        v[j] = (uint32_t)pos;
      } else {
        k[j] = ksrc[pos];
        v[j] = vsrc[pos];
      }
    } else {
      k[j] = ~0ULL;  // padding sorts after every valid key of digit 255
      v[j] = 0xffffffffu;
    }
  }
  // rank of each key among the warp's keys of its digit, in (item, lane)
  // order.  match_any finds the lanes sharing a digit; it is quick on these
  // keys, whose warps hold few distinct digits (hot keys, and the digit
  // order of the passes before); eight ballots on the digit bits measured
  // slower here, though faster on uniformly random keys.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const unsigned d = (unsigned)(k[j] >> shift) & 255u;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const int leader = __ffs(peers) - 1;
    unsigned old = 0;
    if (lane == leader) {
      old = s_whist[w][d];
      s_whist[w][d] = old + __popc(peers);
    }
    old = __shfl_sync(0xffffffffu, old, leader);
    rank[j] = old + __popc(peers & lt);
    __syncwarp();
  }
  __syncthreads();
  // per digit: counts over warps -> exclusive prefix per warp, tile total
  const int d = tid;  // kSortBlock == 256
  unsigned total = 0;
#pragma unroll
  for (int ww = 0; ww < kSortBlock / 32; ++ww) {
    const unsigned c = s_whist[ww][d];
    s_whist[ww][d] = total;
    total += c;
  }
  // publish this tile's count of digit d
  unsigned long long* my = lookback + (size_t)tile * 256 + d;
  const unsigned long long tag = (unsigned long long)epoch << 32;
  if (tile == 0)
    st_relaxed(my, tag | ((unsigned long long)kFlagIncl << 30) | total);
  else
    st_relaxed(my, tag | ((unsigned long long)kFlagAgg << 30) | total);
  // tile-local exclusive scan over digits
  {
    unsigned x = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) s_wsum[w] = x;
    __syncthreads();
    unsigned pre = 0;
#pragma unroll
    for (int ww = 0; ww < kSortBlock / 32; ++ww)
      if (ww < w) pre += s_wsum[ww];
    s_doff[d] = pre + x - total;
  }
  // decoupled look-back for digit d: kWin predecessor entries are loaded at
  // once, then consumed nearest first until an inclusive one is met (a window
  // of 4 measured faster than 1 or 16 on 32.8M keys)
  unsigned excl = 0;
  if (tile > 0) {
    constexpr int kWin = 4;
    int64_t t = (int64_t)tile - 1;
    int spins = 0;
    bool done = false;
    while (!done) {
      unsigned long long e[kWin];
#pragma unroll
      for (int w = 0; w < kWin; ++w)
        e[w] = (t - w >= 0) ? ld_relaxed(lookback + (size_t)(t - w) * 256 + d) : 0ULL;
#pragma unroll
      for (int w = 0; w < kWin; ++w) {
        if (done) break;
        if (t - w < 0) {  // unreachable: tile 0 publishes an inclusive count
          done = true;
          break;
        }
        unsigned long long v = e[w];
        while ((uint32_t)(v >> 32) != epoch || ((v >> 30) & 3u) == 0) {
          if (++spins > spin_max) {
            raise_error(st, mirror, kErrTimeout);
            done = true;
            break;
          }
          __nanosleep(32);
          v = ld_relaxed(lookback + (size_t)(t - w) * 256 + d);
        }
        if (done) break;
        excl += (unsigned)(v & 0x3fffffffu);
        if (((v >> 30) & 3u) == kFlagIncl) done = true;
      }
      t -= kWin;
    }
    st_relaxed(my, tag | ((unsigned long long)kFlagIncl << 30) | (excl + total));
  }
  s_glob[d] = (int)(ctl->base[P][d] + excl) - (int)s_doff[d];
  __syncthreads();
  // reorder the tile in shared memory
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const unsigned dd = (unsigned)(k[j] >> shift) & 255u;
    const unsigned sp = s_doff[dd] + s_whist[w][dd] + rank[j];
    s_keys[sp] = k[j];
    s_vals[sp] = v[j];
  }
  __syncthreads();
  const int64_t valid = N - tbase < kSortTile ? N - tbase : kSortTile;
  for (int sidx = tid; sidx < valid; sidx += kSortBlock) {
    const uint64_t kk = s_keys[sidx];
    const unsigned dd = (unsigned)(kk >> shift) & 255u;
    const int g = s_glob[dd] + sidx;
    if ((unsigned)g < (unsigned)N) {  // always true unless the keys changed under the sort
      kdst[g] = kk;
      vdst[g] = s_vals[sidx];
    }
  }
}

}  // namespace

cudaError_t launch_sort(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N,
                        cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(b->ctl, 0, kCtlZeroBytes, s);
  if (e != cudaSuccess) return e;
  if (b->seg_lookback_tiles > 0) {
    e = cudaMemsetAsync(b->seg_lookback, 0, sizeof(unsigned long long) * b->seg_lookback_tiles, s);
    if (e != cudaSuccess) return e;
  }
  {
    int64_t blocks = (N + 2047) / 2048;  // 8 keys per thread
    if (blocks > 8 * kSMs) blocks = 8 * kSMs;
    if (blocks < 1) blocks = 1;
    LaunchScope ls("sort_hist", s);
    sort_hist_kernel<<<(unsigned)blocks, 256, 0, s>>>(keys, N, b->ctl, t->dstate, t->mirror_dev,
                                                      b->bdev, b->call_seq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t tiles = (N + kSortTile - 1) / kSortTile;
  for (int p = 0; p < kSortPasses; ++p) {
    b->epoch += 1;
    if (b->epoch == 0) {
      // the tag wrapped: entries left by passes 2^32 tags ago could carry the
      // tag about to be used, so the look-back array starts over from zero
      // (stream-ordered after every earlier pass)
      b->epoch = 1;
      e = cudaMemsetAsync(b->sort_lookback, 0,
                          sizeof(unsigned long long) * 256 * (size_t)b->sort_lookback_tiles, s);
      if (e != cudaSuccess) return e;
    }
    LaunchScope ls("sort_pass", s);
    sort_pass_kernel<<<(unsigned)tiles, kSortBlock, 0, s>>>(
        p, keys, b->kbuf[0], b->kbuf[1], b->vbuf[0], b->vbuf[1], N, b->ctl, b->sort_lookback,
        b->epoch, t->dstate, t->mirror_dev, spin_limit());
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace recis
