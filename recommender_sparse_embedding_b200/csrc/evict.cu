// evict.cu -- feature eviction (RecIS README, Core architecture > Embedding
// Engine: the table supports feature eviction and admission policies).
//
// recis_table_evict removes every key whose last lookup came before a given
// clock.  Three launches, synchronous:
//   evict_mark   over the IDMap slots: a key with a row last touched before
//                the clock becomes a tombstone (its slot keeps the key, so no
//                other key's probe chain is cut), its row's key becomes -1 and
//                its last-lookup clock the freed mark; a candidate last seen
//                before the clock becomes a tombstone too;
//   evict_count  per block of 1024 rows, the rows freed just now;
//   evict_list   (after the host's prefix over the block counts) appends the
//                freed rows to the free-row queue in ascending row order and
//                clears their mark.
// Later lookups give queued rows to their new keys, oldest first.
#include <algorithm>
#include <vector>

#include "internal.h"

namespace recis {
namespace {

constexpr int kEvictBlock = 1024;

__global__ void __launch_bounds__(256) evict_mark_kernel(Slot* slots, int64_t cap, int64_t* row_keys,
                                                         uint32_t* seen, uint64_t min_clock) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < cap; i += stride) {
    const longlong2 sv = __ldcg(reinterpret_cast<const longlong2*>(slots + i));
    if (sv.x == kEmptyKey) continue;
    if (sv.y >= 0) {
      if ((uint64_t)seen[sv.y] < min_clock) {
        slots[i].row = kTombRow;
        row_keys[sv.y] = kEmptyKey;
        seen[sv.y] = kFreedMark;
      }
    } else if (is_cand_row(sv.y) && cand_clock(sv.y) < min_clock) {
      slots[i].row = kTombRow;
    }
  }
}

__global__ void __launch_bounds__(256) evict_count_kernel(const uint32_t* seen, int64_t n, unsigned* counts) {
  __shared__ unsigned s_n;
  if (threadIdx.x == 0) s_n = 0;
  __syncthreads();
  const int64_t r0 = (int64_t)blockIdx.x * kEvictBlock;
  unsigned c = 0;
  for (int i = threadIdx.x; i < kEvictBlock; i += blockDim.x)
    c += (r0 + i < n && seen[r0 + i] == kFreedMark) ? 1u : 0u;
  atomicAdd(&s_n, c);
  __syncthreads();
  if (threadIdx.x == 0) counts[blockIdx.x] = s_n;
}

// One CTA of 1024 threads per block of rows: a stable compaction of the
// marked rows (rank = marked rows before it in the block).
__global__ void __launch_bounds__(kEvictBlock) evict_list_kernel(uint32_t* seen, int64_t n,
                                                                 const unsigned* offsets, int32_t* out) {
  __shared__ unsigned s_warp[kEvictBlock / 32];
  const int64_t r = (int64_t)blockIdx.x * kEvictBlock + threadIdx.x;
  const bool marked = r < n && seen[r] == kFreedMark;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, marked);
  if (lane == 0) s_warp[w] = __popc(bal);
  __syncthreads();
  unsigned before = 0;
  for (int i = 0; i < w; ++i) before += s_warp[i];
  if (marked) {
    out[offsets[blockIdx.x] + before + __popc(bal & ((1u << lane) - 1u))] = (int32_t)r;
    seen[r] = 0;
  }
}

}  // namespace
}  // namespace recis

using namespace recis;

extern "C" recis_status recis_table_evict(recis_table_t t, int64_t min_clock, int64_t* n_evicted,
                                          recis_stream_t stream) {
  if (!t || min_clock < 0) {
    set_error("table_evict: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  if (!t->cfg.evictable) {
    set_error("table_evict: the table was created without evictable = 1");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  int64_t in_use = 0;
  recis_status st = table_counts(t, s, &in_use, nullptr);
  if (st != RECIS_OK) return st;
  cudaError_t e;
  {
    int64_t blocks = (t->capacity + 255) / 256;
    if (blocks > 16 * kSMs) blocks = 16 * kSMs;
    LaunchScope ls("evict_mark", s);
    evict_mark_kernel<<<(unsigned)blocks, 256, 0, s>>>(t->slots, t->capacity,
                                                       reinterpret_cast<int64_t*>(t->keys.va),
                                                       reinterpret_cast<uint32_t*>(t->seen.va),
                                                       (uint64_t)min_clock);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "evict launch");
  }
  const int64_t nblk = (in_use + kEvictBlock - 1) / kEvictBlock;
  int64_t total = 0;
  if (nblk > 0) {
    unsigned* dcnt = nullptr;
    if ((e = cudaMalloc(&dcnt, sizeof(unsigned) * nblk * 2)) != cudaSuccess) return cuda_fail(e, "evict alloc");
    std::vector<unsigned> cnt((size_t)nblk), off((size_t)nblk);
    {
      LaunchScope ls("evict_count", s);
      evict_count_kernel<<<(unsigned)nblk, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(t->seen.va), in_use,
                                                        dcnt);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemcpyAsync(cnt.data(), dcnt, sizeof(unsigned) * nblk, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    DevState h{};
    if (e == cudaSuccess) e = cudaMemcpy(&h, t->dstate, sizeof(DevState), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
      cudaFree(dcnt);
      return cuda_fail(e, "evict count");
    }
    for (int64_t i = 0; i < nblk; ++i) {
      off[i] = (unsigned)total;
      total += cnt[i];
    }
    // the queue: rows not yet reused move to the front of a buffer with room
    // for the new ones behind them
    const int64_t keep = (int64_t)(h.free_tail - h.free_head);
    if (total > 0) {
      int32_t* q = t->free_rows;
      if (keep + total > t->free_cap || h.free_head > 0) {
        const int64_t cap = std::max<int64_t>(keep + total + (keep + total) / 4, 1024);
        if ((e = cudaMalloc(&q, sizeof(int32_t) * cap)) != cudaSuccess) {
          cudaFree(dcnt);
          return cuda_fail(e, "evict queue alloc");
        }
        if (keep > 0)
          e = cudaMemcpyAsync(q, t->free_rows + h.free_head, sizeof(int32_t) * keep, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
          cudaFree(q);
          cudaFree(dcnt);
          return cuda_fail(e, "evict queue copy");
        }
        cudaFree(t->free_rows);
        t->free_rows = q;
        t->free_cap = cap;
      }
      for (int64_t i = 0; i < nblk; ++i) off[i] += (unsigned)keep;
      e = cudaMemcpyAsync(dcnt + nblk, off.data(), sizeof(unsigned) * nblk, cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess) {
        LaunchScope ls("evict_list", s);
        evict_list_kernel<<<(unsigned)nblk, kEvictBlock, 0, s>>>(reinterpret_cast<uint32_t*>(t->seen.va), in_use,
                                                                 dcnt + nblk, t->free_rows);
        e = cudaGetLastError();
      }
      unsigned long long ht[2] = {0ULL, (unsigned long long)(keep + total)};
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(&t->dstate->free_head, ht, sizeof(ht), cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    cudaFree(dcnt);
    if (e != cudaSuccess) return cuda_fail(e, "evict list");
  }
  if (n_evicted) *n_evicted = total;
  return RECIS_OK;
}
