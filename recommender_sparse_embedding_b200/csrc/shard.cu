// shard.cu -- building blocks of sharded tables (RecIS README, Key
// optimisations > Distributed optimisation: parameters are split evenly over
// the compute nodes; each node merges and deduplicates its requests, sends
// them to the nodes that own the IDs and fetches the embeddings back with an
// All-to-All collective).
//
// A requesting GPU dedups its batch (recis_batch_dedup), groups its unique
// keys by owner (recis_partition_keys), exchanges them, and pools the rows the
// owners send back (recis_pool_rows); in the backward it sums each unique
// key's gradient over its occurrences (recis_reduce_grad) in the order the
// keys were sent, for the return exchange.  Owners serve their share through
// the ordinary table calls (a lookup with one bag per received key, then a
// backward with the received gradients as unpooled gradients).  The
// exchanges themselves are NCCL all-to-alls issued by the caller.
#include <algorithm>
#include <vector>

#include "internal.h"

namespace recis {

cudaError_t launch_sort(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N, cudaStream_t s);

namespace {

constexpr int kDdBlock = 256, kDdItems = 4, kDdTile = kDdBlock * kDdItems;  // as the unique pass's tiles
constexpr int kMaxOwners = 256;
constexpr int kPartTile = 1024;

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

struct DedupParams {
  const int64_t* keys;
  int64_t N;
  SortCtl* ctl;
  const uint64_t* kb0;
  const uint64_t* kb1;
  const uint32_t* vb0;
  const uint32_t* vb1;
  unsigned long long* lookback;  // [tiles], cleared by the sort launch
  int64_t* uniq;
  int32_t* inv;
  int32_t* seg_start;            // [U + 1]
  int32_t* socc;                 // [N] occurrence at each sorted position
  int64_t* U_out;
  BatchDev* bdev;
  DevState* st;
  int spin_max;
};

// Dedup only, over the sorted (key, occurrence) pairs: heads numbered by a
// decoupled look-back over tiles; unique keys, inverse index, segment starts
// and the occurrence at each sorted position.  The last tile writes U (or -1
// when a bounded wait gave up).
__global__ void __launch_bounds__(kDdBlock) dedup_kernel(const __grid_constant__ DedupParams p) {
  __shared__ uint64_t s_last[kDdBlock];
  __shared__ unsigned s_scan[kDdBlock / 32];
  __shared__ unsigned s_tile;
  __shared__ unsigned long long s_prefix;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(&p.ctl->seg_tile_counter, 1u);
  __syncthreads();
  const unsigned tile = s_tile;
  const unsigned na = p.ctl->n_active;
  const uint64_t* ks = na == 0 ? nullptr : (((na - 1) & 1) ? p.kb1 : p.kb0);
  const uint32_t* vs = na == 0 ? nullptr : (((na - 1) & 1) ? p.vb1 : p.vb0);
  const int64_t N = p.N;
  const int64_t tbase = (int64_t)tile * kDdTile;
  const int64_t pos0 = tbase + (int64_t)tid * kDdItems;
  uint64_t k[kDdItems];
  uint32_t v[kDdItems];
#pragma unroll
  for (int j = 0; j < kDdItems; ++j) {
    const int64_t pos = pos0 + j;
    k[j] = pos < N ? (ks ? ks[pos] : to_ukey(p.keys[pos])) : 0;
    v[j] = pos < N ? (vs ? vs[pos] : (uint32_t)pos) : 0;
  }
  s_last[tid] = k[kDdItems - 1];
  __syncthreads();
  bool have_prev = true;
  uint64_t prev = 0;
  if (tid > 0) prev = s_last[tid - 1];
  else if (tbase > 0) prev = ks ? ks[tbase - 1] : to_ukey(p.keys[tbase - 1]);
  else have_prev = false;
  bool head[kDdItems];
  unsigned nh = 0;
#pragma unroll
  for (int j = 0; j < kDdItems; ++j) {
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
  for (int ww = 0; ww < kDdBlock / 32; ++ww) {
    if (ww < w) wpre += s_scan[ww];
    tot += s_scan[ww];
  }
  const unsigned excl = wpre + x - nh;
  if (tid == 0) {
    unsigned long long* my = p.lookback + tile;
    unsigned long long hx = 0;
    if (tile == 0) {
      st_relaxed_u64(my, (2ULL << 62) | tot);
    } else {
      st_relaxed_u64(my, (1ULL << 62) | tot);
      int64_t t = (int64_t)tile - 1;
      int spins = 0;
      while (t >= 0) {
        const unsigned long long e = ld_relaxed_u64(p.lookback + t);
        const unsigned long long flag = e >> 62;
        if (flag == 0) {
          if (++spins > p.spin_max) {
            atomicOr(&p.st->status, kErrTimeout);
            break;
          }
          __nanosleep(32);
          continue;
        }
        hx += e & 0xffffffffULL;
        if (flag == 2) break;
        --t;
      }
      st_relaxed_u64(my, (2ULL << 62) | (hx + tot));
    }
    s_prefix = hx;
  }
  __syncthreads();
  unsigned hrun = (unsigned)s_prefix + excl;
#pragma unroll
  for (int j = 0; j < kDdItems; ++j) {
    const int64_t pos = pos0 + j;
    if (pos >= N) break;
    if (head[j]) {
      p.uniq[hrun] = from_ukey(k[j]);
      p.seg_start[hrun] = (int32_t)pos;
      ++hrun;
    }
    p.socc[pos] = (int32_t)v[j];
    if (v[j] < (uint64_t)N) p.inv[v[j]] = (int32_t)(hrun - 1);
  }
  if (tile == gridDim.x - 1 && tid == 0) {
    __threadfence();
    const bool failed = (*(volatile int*)&p.st->status & kErrTimeout) != 0;
    const unsigned long long U = s_prefix + tot;
    p.seg_start[U] = (int32_t)N;
    p.bdev->U = failed ? 0u : (unsigned)U;
    *p.U_out = failed ? -1 : (int64_t)U;
  }
}

// owner of a key: the table-slot hash, so that keys spread evenly
__device__ __forceinline__ int owner_of(int64_t key, uint64_t salt, int G) {
  return (int)(mix64((uint64_t)key ^ salt) % (uint64_t)G);
}

// per tile of kPartTile keys: the count of each owner (row `tile` of hist)
__global__ void __launch_bounds__(kPartTile) part_count_kernel(const int64_t* keys, int64_t n, int G, uint64_t salt,
                                                               unsigned* hist) {
  __shared__ unsigned s_h[kMaxOwners];
  for (int i = threadIdx.x; i < G; i += kPartTile) s_h[i] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * kPartTile + threadIdx.x;
  if (i < n) atomicAdd(&s_h[owner_of(keys[i], salt, G)], 1u);
  __syncthreads();
  for (int o = threadIdx.x; o < G; o += kPartTile) hist[(size_t)blockIdx.x * G + o] = s_h[o];
}

// stable scatter by owner: a key's place = its owner's offset for its tile +
// the keys of the same owner before it in the tile (warp match + per-warp
// counts)
__global__ void __launch_bounds__(kPartTile) part_scatter_kernel(const int64_t* keys, int64_t n, int G, uint64_t salt,
                                                                 const unsigned* offs, int64_t* out_keys,
                                                                 int32_t* out_pos) {
  __shared__ unsigned s_w[kPartTile / 32][kMaxOwners];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < (kPartTile / 32) * G; i += kPartTile) (&s_w[0][0])[(i / G) * kMaxOwners + i % G] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * kPartTile + tid;
  const bool ok = i < n;
  const int64_t key = ok ? keys[i] : 0;
  const int o = ok ? owner_of(key, salt, G) : kMaxOwners;  // an invalid owner matches no valid one
  const unsigned peers = __match_any_sync(0xffffffffu, o);
  const unsigned rank_w = __popc(peers & ((1u << lane) - 1u));
  if (ok && lane == __ffs(peers) - 1) s_w[w][o] = __popc(peers);
  __syncthreads();
  if (ok) {
    unsigned before = 0;
    for (int ww = 0; ww < w; ++ww) before += s_w[ww][o];
    const unsigned at = offs[(size_t)blockIdx.x * G + o] + before + rank_w;
    out_keys[at] = key;
    out_pos[i] = (int32_t)at;
  }
}

// one warp per bag: the sum (or mean) of the rows of its occurrences, in fp64,
// rounded once; rows of unique key u sit at row rix[u] (or u)
__global__ void __launch_bounds__(256) pool_rows_kernel(const float* rows, const int32_t* rix, const int32_t* inv,
                                                        const int64_t* offs, int32_t F, int64_t B, int D,
                                                        int mean, float* pooled) {
  const int lane = threadIdx.x & 31;
  const int64_t nb = (int64_t)F * B;
  const int64_t warps = (int64_t)gridDim.x * blockDim.x / 32;
  for (int64_t j = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; j < nb; j += warps) {
    const int64_t lo = offs[j], hi = offs[j + 1];
    const int64_t f = j / B, b = j - f * B;
    float* out = pooled + (b * F + f) * (int64_t)D;
    for (int c = lane; c < D; c += 32) {
      double acc = 0.0;
      for (int64_t i = lo; i < hi; ++i) {
        const int32_t u = __ldg(inv + i);
        const int64_t r = rix ? __ldg(rix + u) : u;
        acc += (double)__ldg(rows + r * D + c);
      }
      if (mean && hi > lo) acc /= (double)(hi - lo);
      out[c] = (float)acc;
    }
  }
}

// one warp per unique key: its gradient, summed over its occurrences in
// occurrence order in fp64 and rounded once, written at row oix[u] (or u)
__global__ void __launch_bounds__(256) reduce_grad_kernel(const int32_t* seg_start, const int32_t* socc,
                                                          const BatchDev* bdev, const int64_t* offs, int32_t F,
                                                          int64_t B, int D, int mean, const float* gp,
                                                          const float* gu, const int32_t* oix, float* out) {
  const int lane = threadIdx.x & 31;
  const int64_t U = (int64_t)bdev->U;
  const int64_t nb = (int64_t)F * B;
  const int64_t warps = (int64_t)gridDim.x * blockDim.x / 32;
  for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; u < U; u += warps) {
    const int32_t s0 = __ldg(seg_start + u), s1 = __ldg(seg_start + u + 1);
    float* o = out + (int64_t)(oix ? __ldg(oix + u) : u) * D;
    for (int c0 = 0; c0 < D; c0 += 32) {
      const int c = c0 + lane;
      double acc = 0.0;
      for (int32_t q = s0; q < s1; ++q) {
        const int32_t occ = __ldg(socc + q);
        if (gp) {
          // the bag of the occurrence: offs[lo] <= occ < offs[lo + 1] (the
          // search keeps offs[lo] <= occ < offs[hi], so empty bags are passed)
          int64_t lo = 0, hi = nb;
          while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if (__ldg(offs + mid) <= occ) lo = mid; else hi = mid;
          }
          const int64_t f = lo / B, b = lo - f * B;
          if (c < D) {
            double t = (double)__ldg(gp + (b * F + f) * D + c);
            if (mean) t /= (double)(__ldg(offs + lo + 1) - __ldg(offs + lo));
            acc += t;
          }
        }
        if (gu && c < D) acc += (double)__ldg(gu + (int64_t)occ * D + c);
      }
      if (c < D) o[c] = (float)acc;
    }
  }
}

}  // namespace
}  // namespace recis

using namespace recis;

extern "C" recis_status recis_batch_dedup(recis_batch_t b, const int64_t* keys, int64_t N, int64_t* uniq_out,
                                          int32_t* inv_out, int64_t* U_out, recis_stream_t stream) {
  if (!b || N < 0 || N >= ((int64_t)1 << 30) || !U_out || (N > 0 && (!keys || !uniq_out || !inv_out))) {
    set_error("batch_dedup: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(keys, 8) || misaligned(uniq_out, 8) || misaligned(inv_out, 4) || misaligned(U_out, 8)) {
    set_error("batch_dedup: misaligned array (int64 arrays 8-byte, inv_out 4-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  recis_status st = batch_ensure(b, N, 0, 4);
  if (st != RECIS_OK) return st;
  cudaError_t e;
  if (!b->dstate_local) {
    if ((e = cudaMalloc(&b->dstate_local, sizeof(DevState))) != cudaSuccess) return cuda_fail(e, "batch alloc");
  }
  if ((e = cudaMemsetAsync(b->dstate_local, 0, sizeof(DevState), s)) != cudaSuccess) return cuda_fail(e, "memset");
  b->have_lookup = false;
  b->dedup_N = N;
  if (N == 0) {
    if ((e = cudaMemsetAsync(U_out, 0, sizeof(int64_t), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(b->bdev, 0, sizeof(BatchDev), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(b->seg_start, 0, sizeof(int32_t), s)) != cudaSuccess)
      return cuda_fail(e, "memset");
    return RECIS_OK;
  }
  recis_table t;  // the sort only reports into a status word
  t.dstate = b->dstate_local;
  t.mirror_dev = nullptr;
  if ((e = launch_sort(b, &t, keys, N, s)) != cudaSuccess) return cuda_fail(e, "sort launch");
  DedupParams p;
  p.keys = keys;
  p.N = N;
  p.ctl = b->ctl;
  p.kb0 = b->kbuf[0];
  p.kb1 = b->kbuf[1];
  p.vb0 = b->vbuf[0];
  p.vb1 = b->vbuf[1];
  p.lookback = b->seg_lookback;
  p.uniq = uniq_out;
  p.inv = inv_out;
  p.seg_start = b->seg_start;
  p.socc = b->socc;
  p.U_out = U_out;
  p.bdev = b->bdev;
  p.st = b->dstate_local;
  p.spin_max = spin_limit();
  LaunchScope ls("batch_dedup", s);
  dedup_kernel<<<(unsigned)((N + kDdTile - 1) / kDdTile), kDdBlock, 0, s>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RECIS_OK : cuda_fail(e, "dedup launch");
}

extern "C" recis_status recis_partition_keys(recis_batch_t b, const int64_t* keys, int64_t n, int32_t G,
                                             uint64_t salt, int64_t* out_keys, int32_t* out_pos,
                                             int64_t* counts_out, recis_stream_t stream) {
  if (!b || n < 0 || n >= ((int64_t)1 << 31) || G < 1 || G > kMaxOwners || !counts_out ||
      (n > 0 && (!keys || !out_keys || !out_pos))) {
    set_error("partition_keys: bad arguments (G must be in 1..256)");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(keys, 8) || misaligned(out_keys, 8) || misaligned(out_pos, 4) || misaligned(counts_out, 8)) {
    set_error("partition_keys: misaligned array (int64 arrays 8-byte, out_pos 4-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t tiles = (n + kPartTile - 1) / kPartTile;
  std::vector<int64_t> counts((size_t)G, 0);
  cudaError_t e;
  if (tiles > 0) {
    if (tiles * G > b->capPart) {
      const int64_t cap = tiles * G + tiles * G / 4 + 1024;
      cudaFree(b->part_hist);
      b->part_hist = nullptr;
      if ((e = cudaMalloc(&b->part_hist, sizeof(unsigned) * cap)) != cudaSuccess) return cuda_fail(e, "partition alloc");
      b->capPart = cap;
    }
    {
      LaunchScope ls("partition_count", s);
      part_count_kernel<<<(unsigned)tiles, kPartTile, 0, s>>>(keys, n, G, salt, b->part_hist);
    }
    std::vector<unsigned> h((size_t)(tiles * G));
    if ((e = cudaGetLastError()) != cudaSuccess ||
        (e = cudaMemcpyAsync(h.data(), b->part_hist, sizeof(unsigned) * h.size(), cudaMemcpyDeviceToHost, s)) !=
            cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
      return cuda_fail(e, "partition count");
    // offsets: owner-major, tiles in order within an owner (a stable partition)
    unsigned run = 0;
    for (int o = 0; o < G; ++o) {
      for (int64_t c = 0; c < tiles; ++c) {
        const unsigned x = h[(size_t)c * G + o];
        h[(size_t)c * G + o] = run;
        run += x;
        counts[o] += x;
      }
    }
    if ((e = cudaMemcpyAsync(b->part_hist, h.data(), sizeof(unsigned) * h.size(), cudaMemcpyHostToDevice, s)) !=
        cudaSuccess)
      return cuda_fail(e, "partition offsets");
    {
      LaunchScope ls("partition_scatter", s);
      part_scatter_kernel<<<(unsigned)tiles, kPartTile, 0, s>>>(keys, n, G, salt, b->part_hist, out_keys, out_pos);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "partition scatter");
  }
  if ((e = cudaMemcpyAsync(counts_out, counts.data(), sizeof(int64_t) * G, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
      (e = cudaStreamSynchronize(s)) != cudaSuccess)
    return cuda_fail(e, "partition counts");
  return RECIS_OK;
}

extern "C" recis_status recis_pool_rows(const float* rows, const int32_t* row_of_unique, const int32_t* inv,
                                        const int64_t* bag_offsets, int32_t F, int64_t B, int32_t D,
                                        int32_t combiner, float* pooled_out, recis_stream_t stream) {
  if (F < 0 || B < 0 || D < 1 || (combiner != RECIS_SUM && combiner != RECIS_MEAN) ||
      ((int64_t)F * B > 0 && (!bag_offsets || !pooled_out))) {
    set_error("pool_rows: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(rows, 16) || misaligned(pooled_out, 16) || misaligned(bag_offsets, 8) ||
      misaligned(row_of_unique, 4) || misaligned(inv, 4)) {
    set_error("pool_rows: misaligned array (float rows 16-byte, bag_offsets 8-byte, indices 4-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  const int64_t nb = (int64_t)F * B;
  if (nb == 0) return RECIS_OK;
  int64_t blocks = (nb * 32 + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  cudaStream_t s = (cudaStream_t)stream;
  LaunchScope ls("pool_rows", s);
  pool_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(rows, row_of_unique, inv, bag_offsets, F, B, D,
                                                    combiner == RECIS_MEAN, pooled_out);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RECIS_OK : cuda_fail(e, "pool_rows launch");
}

extern "C" recis_status recis_reduce_grad(recis_batch_t b, const int64_t* bag_offsets, int32_t F, int64_t B,
                                          int32_t D, int32_t combiner, const float* grad_pooled,
                                          const float* grad_unpooled, const int32_t* out_index, float* grad_out,
                                          recis_stream_t stream) {
  if (!b || b->dedup_N < 0 || F < 0 || B < 0 || D < 1 || (combiner != RECIS_SUM && combiner != RECIS_MEAN) ||
      !grad_out || (grad_pooled && !bag_offsets)) {
    set_error("reduce_grad: bad arguments, or the batch holds no recis_batch_dedup");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(grad_pooled, 16) || misaligned(grad_unpooled, 16) || misaligned(grad_out, 16) ||
      misaligned(bag_offsets, 8) || misaligned(out_index, 4)) {
    set_error("reduce_grad: misaligned array (float rows 16-byte, bag_offsets 8-byte, out_index 4-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  if (b->dedup_N == 0) return RECIS_OK;
  int64_t blocks = (b->dedup_N * 32 + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  cudaStream_t s = (cudaStream_t)stream;
  LaunchScope ls("reduce_grad", s);
  reduce_grad_kernel<<<(unsigned)blocks, 256, 0, s>>>(b->seg_start, b->socc, b->bdev, bag_offsets, F, B, D,
                                                      combiner == RECIS_MEAN, grad_pooled, grad_unpooled,
                                                      out_index, grad_out);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RECIS_OK : cuda_fail(e, "reduce_grad launch");
}
