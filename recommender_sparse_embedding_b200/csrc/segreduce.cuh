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
