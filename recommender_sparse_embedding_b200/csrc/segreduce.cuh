// segreduce.cuh -- shared machinery of the two segmented reductions (bag
// pooling in the forward, per-unique gradient reduction in the backward).
//
// The positions [0, N) are cut into fixed chunks of C positions; one group of
// G lanes walks one chunk in order, 16 bytes (one float4 column) per lane, so
// the work is balanced whatever the bag or segment lengths are.  A segment
// that lies inside one chunk is finished by that group.  A segment cut by
// chunk boundaries leaves one partial sum per chunk it touches (slot 0 when it
// is the chunk's first segment, slot 1 otherwise); the group that arrives last
// (atomic ticket per segment, reset by that group) adds the partials in chunk
// order, so results are deterministic and no per-element atomics are used.
#pragma once
#include "internal.h"

namespace recis {

template <int G>
struct GroupCtx {
  int lane;        // lane within the group
  unsigned mask;   // lanes of this group within the warp
  int shift;       // first lane of the group within the warp
  __device__ __forceinline__ GroupCtx() {
    const int wl = threadIdx.x & 31;
    lane = wl & (G - 1);
    shift = wl & ~(G - 1);
    mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << shift);
  }
  template <typename T>
  __device__ __forceinline__ T bcast(T v, int src) const {
    return __shfl_sync(mask, v, src, G);
  }
  __device__ __forceinline__ unsigned ballot(bool pr) const {
    return (__ballot_sync(mask, pr) >> shift) & ((G == 32) ? 0xffffffffu : ((1u << G) - 1u));
  }
};

__device__ __forceinline__ float4 f4_zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }

// fp64 accumulator of one 16-byte column (4 floats).  Bags of thousands of
// rows and hot keys with tens of thousands of occurrences are summed in double
// and rounded once, so the fp32 result does not depend on the length of the
// sum.
struct Acc4 {
  double x, y, z, w;
};
__device__ __forceinline__ Acc4 acc_zero() { return Acc4{0.0, 0.0, 0.0, 0.0}; }
__device__ __forceinline__ void acc_add(Acc4& a, const float4& b) {
  a.x += (double)b.x;
  a.y += (double)b.y;
  a.z += (double)b.z;
  a.w += (double)b.w;
}
__device__ __forceinline__ void acc_add(Acc4& a, const Acc4& b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}
__device__ __forceinline__ float4 acc_round(const Acc4& a) {
  return make_float4((float)a.x, (float)a.y, (float)a.z, (float)a.w);
}

// Last-arrival combine of a split segment.  Every group that touched the
// segment calls this once with its partial; returns true in the group that
// must finish the segment, with the full sum in acc.  Partials are fp64,
// 32 bytes per column, two slots of D doubles per chunk.
template <int G, int VPL, int NB = 1>
__device__ __forceinline__ bool combine_split(const GroupCtx<G>& g, Acc4 (&acc)[VPL],
                                              double* partials, int32_t* counters, int64_t seg,
                                              int64_t chunk, bool first_of_chunk,
                                              int64_t seg_start, int64_t seg_end, int64_t C,
                                              int ncol) {
  const int slot = first_of_chunk ? 0 : 1;
  const int64_t D = (int64_t)ncol * 4;
  double* mine = partials + (chunk * 2 + slot) * D;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col < ncol) {
      double2* d = reinterpret_cast<double2*>(mine) + 2 * col;
      __stcg(d, make_double2(acc[v].x, acc[v].y));
      __stcg(d + 1, make_double2(acc[v].z, acc[v].w));
    }
  }
  __threadfence();
  __syncwarp(g.mask);
  int ticket = 0;
  if (g.lane == 0) ticket = atomicAdd(&counters[seg], 1);
  ticket = g.bcast(ticket, 0);
  const int64_t c0 = seg_start / C, c1 = (seg_end - 1) / C;
  if (ticket != (int)(c1 - c0)) return false;
  __threadfence();
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  // the partials in chunk order, NB chunks' loads in flight at a time
  for (int64_t cb = c0; cb <= c1; cb += NB) {
    double2 pa[NB][VPL], pb[NB][VPL];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int64_t cc = cb + t;
      const int sl = (cc == c0 && seg_start != c0 * C) ? 1 : 0;
      const double* src = partials + (cc * 2 + sl) * D;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (cc <= c1 && col < ncol) {
          pa[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col);
          pb[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col + 1);
        } else {
          pa[t][v] = make_double2(0.0, 0.0);
          pb[t][v] = make_double2(0.0, 0.0);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      if (cb + t > c1) break;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc_add(acc[v], Acc4{pa[t][v].x, pa[t][v].y, pb[t][v].x, pb[t][v].y});
    }
  }
  if (g.lane == 0) counters[seg] = 0;
  return true;
}

}  // namespace recis

namespace recis {

// Sums the fp64 partials of chunks lo..hi (slot of each chunk as in
// combine_split) in chunk order, NB chunks' loads in flight at a time.
template <int G, int VPL, int NB>
__device__ __forceinline__ void sum_partials(const GroupCtx<G>& g, Acc4 (&acc)[VPL], const double* partials,
                                             int64_t lo, int64_t hi, int64_t c0, bool c0_slot1, int ncol) {
  const int64_t D = (int64_t)ncol * 4;
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  for (int64_t cb = lo; cb <= hi; cb += NB) {
    double2 pa[NB][VPL], pb[NB][VPL];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int64_t cc = cb + t;
      const int sl = (cc == c0 && c0_slot1) ? 1 : 0;
      const double* src = partials + (cc * 2 + sl) * D;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (cc <= hi && col < ncol) {
          pa[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col);
          pb[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col + 1);
        } else {
          pa[t][v] = make_double2(0.0, 0.0);
          pb[t][v] = make_double2(0.0, 0.0);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      if (cb + t > hi) break;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc_add(acc[v], Acc4{pa[t][v].x, pa[t][v].y, pb[t][v].x, pb[t][v].y});
    }
  }
}

// Two-level last-arrival combine of a segment cut into chunks of C
// positions, for segments of thousands of chunks.  Chunks are grouped in
// blocks of BLK; every group that touched the segment calls this once with
// its chunk's partial.  The last arrival among the segment's chunks of one
// block (ticket in block_counters at the block's first chunk of the
// segment) adds them in chunk order and stores the block sum over that
// chunk's partial; the last block (ticket in seg_counters) adds the block
// sums in block order.  Returns true in the group that must finish the
// segment, with the full sum in acc.  Tickets reset themselves.
template <int G, int VPL, int NB, int BLK>
__device__ __forceinline__ bool combine_split2(const GroupCtx<G>& g, Acc4 (&acc)[VPL], double* partials,
                                               int32_t* block_counters, int32_t* seg_counters, int64_t seg,
                                               int64_t chunk, bool first_of_chunk, int64_t seg_start,
                                               int64_t seg_end, int64_t C, int ncol) {
  const int64_t D = (int64_t)ncol * 4;
  const int slot = first_of_chunk ? 0 : 1;
  double* mine = partials + (chunk * 2 + slot) * D;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col < ncol) {
      double2* d = reinterpret_cast<double2*>(mine) + 2 * col;
      __stcg(d, make_double2(acc[v].x, acc[v].y));
      __stcg(d + 1, make_double2(acc[v].z, acc[v].w));
    }
  }
  const int64_t c0 = seg_start / C, c1 = (seg_end - 1) / C;
  const bool c0_slot1 = seg_start != c0 * C;
  const int64_t blk = chunk / BLK;
  const int64_t lo = c0 > blk * BLK ? c0 : blk * BLK;
  const int64_t hi = c1 < (blk + 1) * BLK - 1 ? c1 : (blk + 1) * BLK - 1;
  const int lo_slot = (lo == c0 && c0_slot1) ? 1 : 0;
  __threadfence();
  __syncwarp(g.mask);
  if (hi > lo) {
    int ticket = 0;
    if (g.lane == 0) ticket = atomicAdd(&block_counters[lo * 2 + lo_slot], 1);
    ticket = g.bcast(ticket, 0);
    if (ticket != (int)(hi - lo)) return false;
    __threadfence();
    sum_partials<G, VPL, NB>(g, acc, partials, lo, hi, c0, c0_slot1, ncol);
    if (g.lane == 0) block_counters[lo * 2 + lo_slot] = 0;
    // the block sum replaces the partial of the block's first chunk
    double* dst = partials + (lo * 2 + lo_slot) * D;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      if (col < ncol) {
        double2* d = reinterpret_cast<double2*>(dst) + 2 * col;
        __stcg(d, make_double2(acc[v].x, acc[v].y));
        __stcg(d + 1, make_double2(acc[v].z, acc[v].w));
      }
    }
    __threadfence();
    __syncwarp(g.mask);
  }
  const int64_t b0 = c0 / BLK, b1 = c1 / BLK;
  if (b0 == b1) {
    if (hi == lo) sum_partials<G, VPL, NB>(g, acc, partials, lo, lo, c0, c0_slot1, ncol);
    return true;
  }
  int ticket = 0;
  if (g.lane == 0) ticket = atomicAdd(&seg_counters[seg], 1);
  ticket = g.bcast(ticket, 0);
  if (ticket != (int)(b1 - b0)) return false;
  __threadfence();
  // block sums in block order, NB blocks' loads in flight at a time
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  for (int64_t bc = b0; bc <= b1; bc += NB) {
    double2 pa[NB][VPL], pb[NB][VPL];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int64_t bb = bc + t;
      const int64_t l = c0 > bb * BLK ? c0 : bb * BLK;
      const int sl = (l == c0 && c0_slot1) ? 1 : 0;
      const double* src = partials + (l * 2 + sl) * D;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (bb <= b1 && col < ncol) {
          pa[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col);
          pb[t][v] = __ldcg(reinterpret_cast<const double2*>(src) + 2 * col + 1);
        } else {
          pa[t][v] = make_double2(0.0, 0.0);
          pb[t][v] = make_double2(0.0, 0.0);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      if (bc + t > b1) break;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc_add(acc[v], Acc4{pa[t][v].x, pa[t][v].y, pb[t][v].x, pb[t][v].y});
    }
  }
  if (g.lane == 0) seg_counters[seg] = 0;
  return true;
}

}  // namespace recis
