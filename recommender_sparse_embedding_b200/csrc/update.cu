// update.cu -- backward: per-unique gradient reduction and the sparse
// optimiser row update (RecIS README, Key optimisations > Operator
// implementation: reductions merged at warp level rather than by per-element
// atomics; > Efficient dynamic embedding: optimiser state stored beside the
// parameters in the EmbeddingBlocks).
//
// The dedup left the sorted positions grouped by unique key: segment u spans
// sorted positions seg_start[u] .. seg_start[u+1]-1, and the pooling
// recorded each position's gradient source (pooled-gradient row, bag length,
// occurrence).  The gradient of u is
//   g(u) = sum over its positions of grad_pooled[bag] * (1 or 1/length)
//          + grad_unpooled[occurrence],
// summed in fp64 in position order and rounded once to fp32.  Three launches:
//   seg_partial  segments longer than kShortSeg (hot keys): the positions
//                are cut into spans; each lane group sums its span's part
//                of every long segment in fp64, storing g(u) in gbuf at row
//                seg_start[u] / kChunk when the segment lies inside the span
//                (a long segment is the only long one starting in its
//                kChunk positions), else a partial;
//   seg_combine  adds the partials of each segment cut by span ends in a
//                fixed order and stores g(u) in gbuf;
//   row_update  one lane group per unique key loads the row [emb | state],
//               sums the key's gradient terms itself when the segment is
//               short (all loads issued before the sum) or reads gbuf, and
//               applies Adagrad or Adam in place.  Keys seen 2 to kShortSeg
//               times come from the dedup's list, spread evenly over the
//               groups, when there are a few per group.
// No float atomics anywhere; the result does not depend on scheduling.
#include <algorithm>

#include "segreduce.cuh"

namespace recis {

constexpr int kChunk = 16;  // positions per gbuf row; seg_reduce spans are multiples of it
static_assert(kChunk <= kShortSeg + 1, "kChunk positions must hold at most one long segment start");
static_assert(kChunk == kShortSeg, "gbuf holds one row per kShortSeg positions");

struct UpdateParams {
  int64_t N;
  int32_t ncol;             // D / 4
  int32_t mean;
  int32_t row_floats;
  int64_t span;             // seg_reduce positions per lane group (a multiple of kChunk)
  const int4* gsrc;         // [N] per sorted position: {gradient row, bag length, occurrence, 0}
  const int4* gfirst;       // [U] per unique key: gsrc of one of its occurrences
  const int32_t* seg_of;    // [N] sorted position -> unique index
  const int32_t* seg_start; // [U+1]
  const int64_t* rows;      // [U]
  BatchDev* bdev;           // U of the lookup; the long-segment list counters
  const float* gp;          // grad_pooled [B][F][D] or null
  const float* gu;          // grad_unpooled [N][D] or null
  float* gbuf;              // [N / kChunk + 1][D] reduced gradients of long segments
  float* row_data;
  double* partials;         // [spans][2][D]
  int2* long_segs;          // [seg_cap] long segments crossing a span end: the CTA-combined ones
                            // from the back, the others from the front
  int64_t seg_cap;
  DevState* st;             // status word (a bounded wait that gave up)
  HostMirror* mirror;
  int spin_max;             // polls before a wait gives up
  const int32_t* multi_keys;  // keys seen 2 to kShortSeg times (bdev->nmulti of them), or null
  // optimiser
  float lr;        // Adagrad: lr; Adam: lr / (1 - beta1^t)
  float eps;
  float beta1, beta2;
  float omb1, omb2;  // 1 - beta1, 1 - beta2 (formed in double, rounded once)
  float inv_sqrt_bc2;  // Adam: 1 / sqrt(1 - beta2^t) (formed in double, rounded once)
};

// gradient rows each lane loads before adding (fewer for wide rows: registers)
template <int VPL, bool BOTH = false>
constexpr int kRowsInFlight = VPL >= 4 ? 1 : ((VPL == 2 ? 2 : 4) / (BOTH ? 2 : 1));

// Gradient source of one position: row of grad_pooled, its scale (1, or
// 1/length for mean pooling) and the occurrence (row of grad_unpooled).
struct Src {
  int32_t gr;
  int32_t occ;
  double scale;
};

__device__ __forceinline__ Src make_src(const UpdateParams& p, int4 v) {
  Src s;
  s.gr = v.x;
  s.occ = v.z;
  s.scale = p.mean ? 1.0 / (double)v.y : 1.0;
  return s;
}

// Adds the terms of `count` (<= K) positions whose sources sit in lanes
// first .. first+count-1 to acc; every lane loads its 16-byte columns of all
// the rows before adding.  GP / GU: pooled / unpooled gradient present.
template <int G, int VPL, int K, bool GP, bool GU>
__device__ __forceinline__ void add_terms(const GroupCtx<G>& g, const UpdateParams& p, const Src& my,
                                          int first, int count, Acc4 (&acc)[VPL]) {
  const int64_t D = (int64_t)p.ncol * 4;
  float4 tp[K][VPL], tu[K][VPL];
  double sc[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const bool valid = k < count;
    const int src = valid ? first + k : first;
    const int32_t gr = GP ? g.bcast(my.gr, src) : 0;
    const int32_t oc = GU ? g.bcast(my.occ, src) : 0;
    sc[k] = (GP && p.mean) ? g.bcast(my.scale, src) : 1.0;
    const float4* gps = reinterpret_cast<const float4*>(p.gp + (int64_t)gr * D);
    const float4* gus = reinterpret_cast<const float4*>(p.gu + (int64_t)oc * D);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      const bool ok = valid && col < p.ncol;
      tp[k][v] = (GP && ok) ? __ldcs(gps + col) : f4_zero();
      tu[k][v] = (GU && ok) ? __ldcs(gus + col) : f4_zero();
    }
  }
#pragma unroll
  for (int k = 0; k < K; ++k) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      // one term per position: pooled gradient * scale + unpooled gradient
      acc[v].x += (GP ? (double)tp[k][v].x * sc[k] : 0.0) + (GU ? (double)tu[k][v].x : 0.0);
      acc[v].y += (GP ? (double)tp[k][v].y * sc[k] : 0.0) + (GU ? (double)tu[k][v].y : 0.0);
      acc[v].z += (GP ? (double)tp[k][v].z * sc[k] : 0.0) + (GU ? (double)tu[k][v].z : 0.0);
      acc[v].w += (GP ? (double)tp[k][v].w * sc[k] : 0.0) + (GU ? (double)tu[k][v].w : 0.0);
    }
  }
}

// ------------------------------------------------------------------ seg_reduce
// Long segments (more than kShortSeg positions: hot keys).  The sorted
// positions are cut into spans of p.span positions (a multiple of kChunk),
// one lane group per span.  The group walks its span a step of Q positions
// (one or a few per lane) at a time, with three steps in flight: the rows
// of step k, the segment bounds of step k+1 and the segments and gradient
// sources of step k+2.  A position is long when its segment is; the
// gradient rows of a step's long positions are copied into shared memory by
// bulk copies (cp.async when the gradients are not device memory), up to
// PR positions at once (one slot per position, row and
// lane), then added in position order into one fp64 sum per segment run.
// A run's sum is
//   - the segment's gradient, rounded once and stored in gbuf at row
//     start / kChunk, when the segment lies inside the span;
//   - else a partial of the span: slot 0 for the segment that began before
//     the span, slot 1 for the one that begins in it and runs past its end.
// seg_partial lists the segment as {start, end} at its first span;
// seg_combine adds its partials in a fixed order -- slot 1 of its first
// span, then slot 0 of each following span -- with one lane group, or for a
// segment of many spans with a whole CTA: lane group j takes terms j,
// j + groups, ..., and the groups' sums are added in group order.  No
// tickets, fences or float atomics; the result does not depend on
// scheduling.
constexpr int kHugeTerms = 16;  // partials above which a whole CTA combines a segment

// Positions per step: one per lane (at least kChunk, at most 4 per lane).
template <int G>
struct SegStep {
  static constexpr int Q = G >= kChunk ? G : (4 * G < kChunk ? 4 * G : kChunk);
  static constexpr int E = Q / G;  // positions per lane
};

// A step's positions, loaded in two stages: the segment and the gradient
// source of each position, then its segment's bounds.
template <int E>
struct StepA {
  int32_t seg[E];
  int4 src[E];
};
template <int E>
struct StepB {
  int32_t seg[E], st[E], en[E];
  int4 src[E];
};

// a[e] for a run-time e without local-memory indexing
template <int E, typename T>
__device__ __forceinline__ T pick(const T (&a)[E], int e) {
  T v = a[0];
#pragma unroll
  for (int i = 1; i < E; ++i)
    if (i == e) v = a[i];
  return v;
}

template <int G, int E>
__device__ __forceinline__ void load_step_a(const GroupCtx<G>& g, const UpdateParams& p, int64_t base,
                                            int64_t end, StepA<E>& a) {
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t q = base + g.lane + e * G;
    a.seg[e] = -1;
    a.src[e] = make_int4(0, 1, 0, 0);
    if (q < end) {
      a.seg[e] = __ldg(p.seg_of + q);
      a.src[e] = __ldg(p.gsrc + q);
    }
  }
}

template <int E>
__device__ __forceinline__ void load_step_b(const UpdateParams& p, const StepA<E>& a, StepB<E>& b) {
#pragma unroll
  for (int e = 0; e < E; ++e) {
    b.seg[e] = a.seg[e];
    b.src[e] = a.src[e];
    b.st[e] = b.en[e] = 0;
    if (a.seg[e] >= 0) {
      b.st[e] = __ldg(p.seg_start + a.seg[e]);
      b.en[e] = __ldg(p.seg_start + a.seg[e] + 1);
    }
  }
}

// the pooled gradient's scale of each position: 1 / bag length (mean
// pooling), else 1
template <int E>
__device__ __forceinline__ void step_scales(const UpdateParams& p, const StepB<E>& b, double (&sc)[E]) {
#pragma unroll
  for (int e = 0; e < E; ++e) sc[e] = (p.mean && b.src[e].y > 0) ? 1.0 / (double)b.src[e].y : 1.0;
}

// bit t (t >= 1): position t of the step lies in another segment than
// position t - 1
template <int G, int E>
__device__ __forceinline__ unsigned run_starts(const GroupCtx<G>& g, const StepB<E>& b) {
  unsigned m = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int32_t up = __shfl_up_sync(g.mask, b.seg[e], 1, G);
    const int32_t wrap = g.bcast(b.seg[e > 0 ? e - 1 : 0], G - 1);
    const int32_t prev = g.lane > 0 ? up : (e > 0 ? wrap : b.seg[e]);
    m |= g.ballot(b.seg[e] != prev) << (e * G);
  }
  return m;
}

// bit t (t = lane + e * G): position t of the step lies in a long segment
template <int G, int E>
__device__ __forceinline__ unsigned long_mask(const GroupCtx<G>& g, const StepB<E>& b) {
  unsigned m = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) m |= g.ballot(b.seg[e] >= 0 && b.en[e] - b.st[e] > kShortSeg) << (e * G);
  return m;
}

template <int G, int VPL>
__device__ __forceinline__ void store_gbuf(const GroupCtx<G>& g, const UpdateParams& p, int64_t start,
                                           const Acc4 (&acc)[VPL]) {
  float4* dst = reinterpret_cast<float4*>(p.gbuf + (start / kChunk) * (int64_t)p.ncol * 4);
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col < p.ncol) __stcg(dst + col, acc_round(acc[v]));
  }
}

// resident CTAs per SM (registers: several positions per lane for narrow
// rows, many accumulators for wide ones)
template <int G, int VPL>
constexpr int kPartialCtas = VPL >= 4 ? 1 : (G < 8 ? 2 : 3);

// Staging: kChunk 16-byte slots per lane, PR long positions' rows at a time.
__device__ __forceinline__ void cp_async16_(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

// TMA: the gradient rows are copied by the bulk-copy engine (gradients in
// device memory), else by cp.async (any memory the GPU can address).
template <int G, int VPL, bool GP, bool GU, bool TMA>
__global__ void __launch_bounds__(256, kPartialCtas<G, VPL>) seg_partial_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  constexpr int NRW = (GP && GU) ? 2 : 1;  // gradient rows per position
  constexpr int PR = kChunk / (VPL * NRW) > 0 ? kChunk / (VPL * NRW) : 1;  // positions staged at once
  constexpr int Q = SegStep<G>::Q, E = SegStep<G>::E;
  extern __shared__ float4 s_rows[];  // [groups of the CTA][kChunk][G]
  __shared__ uint64_t s_mbar[256];     // one transaction barrier per group
  const GroupCtx<G> g;
  float4* rows = s_rows + (size_t)(threadIdx.x / G) * kChunk * G;
  uint64_t* mbar = s_mbar + threadIdx.x / G;
  const int64_t span = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const int64_t p0 = span * p.span;
  if (p0 >= p.N) return;
  if (TMA && g.lane == 0) mbar_init(mbar, 1);
  __syncwarp(g.mask);
  unsigned phase = 0;
  const unsigned row_bytes = (unsigned)p.ncol * 16u;
  const int64_t p1 = p0 + p.span < p.N ? p0 + p.span : p.N;
  const int64_t D = (int64_t)p.ncol * 4;
  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  int32_t cur = -1, cst = 0, cen = 0;
  auto flush = [&]() {
    if (cst >= p0 && cen <= p1) {
      store_gbuf<G, VPL>(g, p, cst, acc);
    } else {
      const int slot = cst < p0 ? 0 : 1;
      double2* dst = reinterpret_cast<double2*>(p.partials + (span * 2 + slot) * D);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (col < p.ncol) {
          __stcg(dst + 2 * col, make_double2(acc[v].x, acc[v].y));
          __stcg(dst + 2 * col + 1, make_double2(acc[v].z, acc[v].w));
        }
      }
      // listed at its first span: segments of many spans from the back
      if (slot == 1 && g.lane == 0) {
        if ((cen - 1) / p.span - cst / p.span + 1 > kHugeTerms)
          p.long_segs[p.seg_cap - 1 - atomicAdd(&p.bdev->nseg_huge, 1u)] = make_int2(cst, cen);
        else
          p.long_segs[atomicAdd(&p.bdev->nseg_med, 1u)] = make_int2(cst, cen);
      }
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  };
  // three steps in flight: rows of step k, bounds of step k+1, segments of step k+2
  StepA<E> a1, a2;
  StepB<E> cur_b, nxt_b;
  load_step_a<G, E>(g, p, p0, p1, a1);
  load_step_b<E>(p, a1, cur_b);
  load_step_a<G, E>(g, p, p0 + Q, p1, a1);
  unsigned mask = long_mask<G, E>(g, cur_b);
  unsigned runs = run_starts<G, E>(g, cur_b);
  double scale[E];
  if (GP) step_scales<E>(p, cur_b, scale);
  for (int64_t base = p0; base < p1; base += Q) {
    const int32_t first_seg = g.bcast(cur_b.seg[0], 0);
    bool ahead = false;  // next steps' loads issued
    unsigned rem = mask;
    do {
      // the next PR long positions of the step: rows into shared memory
      unsigned piece = rem;  // a step's positions fit in one piece when PR >= Q
      if (PR < Q && __popc(rem) > PR) {
        piece = 0;
        unsigned r = rem;
        for (int u = 0; u < PR; ++u) {
          piece |= r & (0u - r);
          r &= r - 1;
        }
      }
      rem &= ~piece;
      // the piece's rows into slot u = the position's rank in the piece
      if (TMA) {
        // each lane copies the rows of its own positions, one bulk copy per row
        if (piece) {
          __syncwarp(g.mask);  // the group has read the previous piece
          fence_async_smem();
          if (g.lane == 0) mbar_arrive_expect(mbar, (unsigned)__popc(piece) * NRW * row_bytes);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int t = g.lane + e * G;
            if (t < 32 && ((piece >> t) & 1u)) {
              const int u = __popc(piece & ((1u << t) - 1u));
              if (GP) bulk_row(rows + (u * NRW) * VPL * G, p.gp + (int64_t)cur_b.src[e].x * D, row_bytes, mbar);
              if (GU)
                bulk_row(rows + (u * NRW + (GP ? 1 : 0)) * VPL * G, p.gu + (int64_t)cur_b.src[e].z * D,
                         row_bytes, mbar);
            }
          }
        }
      } else {
        // 16 bytes per lane and row, by cp.async
        int u = 0;
        for (unsigned m = piece; m; m &= m - 1, ++u) {
          const int t = __ffs(m) - 1;
          const int e = t / G, l = t % G;
          const int4 sv = pick(cur_b.src, e);
          if (GP) {
            const float* r = p.gp + (int64_t)g.bcast(sv.x, l) * D;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
              const int col = g.lane + v * G;
              if (col < p.ncol) cp_async16_(rows + ((u * NRW) * VPL + v) * G + g.lane, r + 4 * col);
            }
          }
          if (GU) {
            const float* r = p.gu + (int64_t)g.bcast(sv.z, l) * D;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
              const int col = g.lane + v * G;
              if (col < p.ncol)
                cp_async16_(rows + ((u * NRW + (GP ? 1 : 0)) * VPL + v) * G + g.lane, r + 4 * col);
            }
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      if (!ahead) {
        load_step_b<E>(p, a1, nxt_b);
        load_step_a<G, E>(g, p, base + 2 * Q, p1, a2);
        ahead = true;
      }
      if (!TMA) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      } else if (piece) {
        if (!mbar_wait(mbar, phase, p.spin_max)) {
          // the copies did not land in time: reported, and waited for once
          // more before the slots are read or written again
          if (g.lane == 0) raise_error(p.st, p.mirror, kErrTimeout);
          mbar_wait(mbar, phase, p.spin_max);
        }
        phase ^= 1u;
      }
      // the piece's positions in order, one segment run at a time
      int u = 0;
      for (unsigned m = piece; m; m &= m - 1, ++u) {
        const int t = __ffs(m) - 1;
        const int e = t / G, l = t % G;
        // a new segment run: the step's first position in another segment
        // than the last one added, or a segment start within the step
        if (t == 0 ? first_seg != cur : ((runs >> t) & 1u) != 0u) {
          if (cur >= 0) flush();
          cur = g.bcast(pick(cur_b.seg, e), l);
          cst = g.bcast(pick(cur_b.st, e), l);
          cen = g.bcast(pick(cur_b.en, e), l);
        }
        const double sc = (GP && p.mean) ? g.bcast(pick(scale, e), l) : 1.0;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          const int col = g.lane + v * G;
          if (col < p.ncol) {
            const float4 x = GP ? rows[((u * NRW) * VPL + v) * G + g.lane] : f4_zero();
            const float4 y = GU ? rows[((u * NRW + (GP ? 1 : 0)) * VPL + v) * G + g.lane] : f4_zero();
            // one term per position: pooled gradient * scale + unpooled gradient
            acc[v].x += (GP ? (double)x.x * sc : 0.0) + (GU ? (double)y.x : 0.0);
            acc[v].y += (GP ? (double)x.y * sc : 0.0) + (GU ? (double)y.y : 0.0);
            acc[v].z += (GP ? (double)x.z * sc : 0.0) + (GU ? (double)y.z : 0.0);
            acc[v].w += (GP ? (double)x.w * sc : 0.0) + (GU ? (double)y.w : 0.0);
          }
        }
      }
    } while (rem);
    cur_b = nxt_b;
    a1 = a2;
    mask = long_mask<G, E>(g, cur_b);
    runs = run_starts<G, E>(g, cur_b);
    if (GP) step_scales<E>(p, cur_b, scale);
  }
  if (cur >= 0) flush();
  pdl_trigger();
}

__device__ __forceinline__ int64_t min_i64(int64_t a, int64_t b) { return a < b ? a : b; }

// Terms i = i0, i0 + stride, ... (< n) of a listed segment whose first span
// is c0, added in that order: term 0 is slot 1 of span c0, term i slot 0 of
// span c0 + i; NB terms' loads in flight at a time.
template <int G, int VPL, int NB>
__device__ __forceinline__ void add_span_partials(const GroupCtx<G>& g, const UpdateParams& p, int64_t c0,
                                                  int64_t n, int64_t i0, int64_t stride, Acc4 (&acc)[VPL]) {
  const int64_t D = (int64_t)p.ncol * 4;
  for (int64_t ib = i0; ib < n; ib += NB * stride) {
    double2 pa[NB][VPL], pb[NB][VPL];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const int64_t i = ib + t * stride;
      const double2* src = reinterpret_cast<const double2*>(p.partials + ((c0 + i) * 2 + (i == 0 ? 1 : 0)) * D);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (i < n && col < p.ncol) {
          pa[t][v] = __ldcg(src + 2 * col);
          pb[t][v] = __ldcg(src + 2 * col + 1);
        } else {
          pa[t][v] = make_double2(0.0, 0.0);
          pb[t][v] = make_double2(0.0, 0.0);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      if (ib + t * stride >= n) break;
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc_add(acc[v], Acc4{pa[t][v].x, pa[t][v].y, pb[t][v].x, pb[t][v].y});
    }
  }
}

// A persistent grid takes work items from a counter: first the segments of
// many spans (one CTA each), then the others (one lane group each, a CTA's
// groups taking consecutive list entries).
template <int G, int VPL>
__global__ void __launch_bounds__(256) seg_combine_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  constexpr int NB = VPL >= 4 ? 2 : 4;
  const GroupCtx<G> g;
  const int grp = threadIdx.x / G, ngrp = blockDim.x / G;
  const int64_t cap = p.seg_cap;
  const int64_t spans = (p.N + p.span - 1) / p.span;
  int64_t nmed = p.bdev->nseg_med, nhuge = p.bdev->nseg_huge;
  if (nmed > cap) nmed = cap;
  if (nhuge > cap - nmed) nhuge = cap - nmed;
  const int64_t items = nhuge + (nmed + ngrp - 1) / ngrp;
  __shared__ unsigned s_item;
  extern __shared__ Acc4 s_part[];  // [groups][VPL][G]
  for (;;) {
    __syncthreads();  // the previous item's s_part and s_item are read
    if (threadIdx.x == 0) s_item = atomicAdd(&p.bdev->seg_work, 1u);
    __syncthreads();
    const int64_t item = s_item;
    if (item >= items) break;
    Acc4 acc[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
    if (item < nhuge) {
      const int2 sg = p.long_segs[cap - 1 - item];
      const int64_t c0 = sg.x / p.span, n = min_i64((sg.y - 1) / p.span + 1, spans) - c0;
      add_span_partials<G, VPL, NB>(g, p, c0, n, grp, ngrp, acc);
#pragma unroll
      for (int v = 0; v < VPL; ++v) s_part[(grp * VPL + v) * G + g.lane] = acc[v];
      __syncthreads();
      if (grp == 0) {
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
        for (int j = 0; j < ngrp; ++j) {
#pragma unroll
          for (int v = 0; v < VPL; ++v) acc_add(acc[v], s_part[(j * VPL + v) * G + g.lane]);
        }
        store_gbuf<G, VPL>(g, p, sg.x, acc);
      }
    } else {
      const int64_t j = (item - nhuge) * ngrp + grp;
      if (j < nmed) {
        const int2 sg = p.long_segs[j];
        const int64_t c0 = sg.x / p.span, n = min_i64((sg.y - 1) / p.span + 1, spans) - c0;
        add_span_partials<G, VPL, NB>(g, p, c0, n, 0, 1, acc);
        store_gbuf<G, VPL>(g, p, sg.x, acc);
      }
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ row_update
// Row data of one unique key: emb and the optimiser state, VPL 16-byte
// columns per lane.
template <int VPL, bool ADAM>
struct RowRegs {
  float4 w[VPL], s1[VPL], s2[ADAM ? VPL : 1];
};

template <int G, int VPL, bool ADAM>
__device__ __forceinline__ void load_row(const GroupCtx<G>& g, const UpdateParams& p, int64_t row,
                                         RowRegs<VPL, ADAM>& r) {
  const int D = p.ncol * 4;
  const float* base = p.row_data + (row < 0 ? 0 : row) * (int64_t)p.row_floats;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (row >= 0 && col < p.ncol) {
      r.w[v] = __ldcs(reinterpret_cast<const float4*>(base) + col);
      r.s1[v] = __ldcs(reinterpret_cast<const float4*>(base + D) + col);
      if (ADAM) r.s2[v] = __ldcs(reinterpret_cast<const float4*>(base + 2 * D) + col);
    }
  }
}

// g rounded once to fp32, then the optimiser in fp32 in the order written:
//   Adagrad  acc += g^2;  w -= lr g / (sqrt(acc) + eps)
//   Adam     m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
//            w -= (lr / (1-b1^t)) m / (sqrt(v) / sqrt(1-b2^t) + eps)
template <int G, int VPL, bool ADAM>
__device__ __forceinline__ void apply_update(const GroupCtx<G>& g, const UpdateParams& p, int64_t row,
                                             const RowRegs<VPL, ADAM>& r, const float4 (&grad)[VPL]) {
  if (row < 0) return;
  float* base = p.row_data + row * p.row_floats;
  const int D = p.ncol * 4;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col >= p.ncol) continue;
    const float gg[4] = {grad[v].x, grad[v].y, grad[v].z, grad[v].w};
    float ww[4] = {r.w[v].x, r.w[v].y, r.w[v].z, r.w[v].w};
    float a1[4] = {r.s1[v].x, r.s1[v].y, r.s1[v].z, r.s1[v].w};
    // the step lr * x / denom: the quotient by __fdividef (within 2 ulp;
    // denom >= eps is far from its overflow range)
    if (!ADAM) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float acc = a1[e] + gg[e] * gg[e];
        ww[e] = ww[e] - __fdividef(p.lr * gg[e], sqrtf(acc) + p.eps);
        a1[e] = acc;
      }
    } else {
      float a2[4] = {r.s2[v].x, r.s2[v].y, r.s2[v].z, r.s2[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = p.beta1 * a1[e] + p.omb1 * gg[e];
        const float vv = p.beta2 * a2[e] + p.omb2 * (gg[e] * gg[e]);
        ww[e] = ww[e] - __fdividef(p.lr * m, fmaf(sqrtf(vv), p.inv_sqrt_bc2, p.eps));
        a1[e] = m;
        a2[e] = vv;
      }
      __stcs(reinterpret_cast<float4*>(base + 2 * D) + col, make_float4(a2[0], a2[1], a2[2], a2[3]));
    }
    __stcs(reinterpret_cast<float4*>(base + D) + col, make_float4(a1[0], a1[1], a1[2], a1[3]));
    __stcs(reinterpret_cast<float4*>(base) + col, make_float4(ww[0], ww[1], ww[2], ww[3]));
  }
}

// One group of G lanes per unique key u (U from the lookup).  The first
// loads (segment bounds, row offset, and the source of a singleton's one
// occurrence) are independent; the row loads go out next, together with the
// gradient rows of a singleton.  A longer short segment resolves its
// positions' sources one per lane and loads several rows at a time; a long
// segment's sum is read from gbuf.
// Gradient of key (s0, s1, first) into acc: a singleton's one term (its
// pooled gradient row already staged in shared memory when staged != null),
// a long segment's sum from gbuf, else the terms gathered here (the first G
// positions' source records already loaded into rec0 when have0).
template <int G, int VPL, bool GP, bool GU>
__device__ __forceinline__ void key_grad(const GroupCtx<G>& g, const UpdateParams& p, int32_t s0,
                                         int32_t s1, int4 first, const float4* staged, int stride,
                                         float4 (&out)[VPL], int4 rec0 = make_int4(0, 1, 0, 0),
                                         bool have0 = false) {
  const int64_t D = (int64_t)p.ncol * 4;
  const int len = s1 - s0;
  constexpr int K = kRowsInFlight<VPL, GP && GU>;
  if (len == 1 && staged && !p.mean) {
    // a singleton's one pooled-gradient term, exactly
#pragma unroll
    for (int v = 0; v < VPL; ++v) out[v] = staged[v * stride];
    return;
  }
  if (len > kShortSeg) {
    const float4* src = reinterpret_cast<const float4*>(p.gbuf + (int64_t)(s0 / kChunk) * D);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      out[v] = col < p.ncol ? __ldcg(src + col) : f4_zero();
    }
    return;
  }
  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  if (len == 1) {
    if (staged) {
      const double sc = 1.0 / (double)first.y;  // mean pooling
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const float4 t = staged[v * stride];
        acc[v] = Acc4{(double)t.x * sc, (double)t.y * sc, (double)t.z * sc, (double)t.w * sc};
      }
    } else {
      add_terms<G, VPL, 1, GP, GU>(g, p, make_src(p, first), 0, 1, acc);
    }
  } else {
    for (int base = 0; base < len; base += G) {
      const int m = len - base < G ? len - base : G;
      Src s{0, 0, 1.0};
      if (base == 0 && have0)
        s = make_src(p, rec0);  // lanes >= m hold {0, 1, 0, 0}: the same unused source
      else if (g.lane < m)
        s = make_src(p, __ldg(p.gsrc + s0 + base + g.lane));
      for (int k0 = 0; k0 < m; k0 += K)
        add_terms<G, VPL, K, GP, GU>(g, p, s, k0, m - k0 < K ? m - k0 : K, acc);
    }
  }
#pragma unroll
  for (int v = 0; v < VPL; ++v) out[v] = acc_round(acc[v]);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// a hint: the 128-byte line holding a into L2
__device__ __forceinline__ void prefetch_l2(const void* a) { asm volatile("prefetch.global.L2 [%0];" ::"l"(a)); }

// Indices of one key: segment bounds, row offset (positions and rows fit in
// 32 bits: N < 2^31, rows < 2^31) and the source of one of its occurrences.
struct __align__(16) KeyIdx {
  int32_t s0, s1, row, pad;
  int4 first;
};

__device__ __forceinline__ KeyIdx key_idx(const UpdateParams& p, int64_t u) {
  KeyIdx k;
  k.pad = 0;
  k.s0 = __ldg(p.seg_start + u);
  k.s1 = __ldg(p.seg_start + u + 1);
  k.row = (int32_t)__ldg(p.rows + u);
  k.first = __ldg(p.gfirst + u);
  return k;
}

// The listed keys (seen 2 to kShortSeg times) i = gid, gid + groups, ...:
// indices, row and gradient rows loaded, then the update.  Kept out of line
// so that the staged key walk of the row update is allocated on its own.
template <int G, int VPL, bool ADAM, bool GP, bool GU>
__device__ __noinline__ void update_listed(const UpdateParams& p, int64_t gid, int64_t groups, int64_t nm) {
  const GroupCtx<G> g;
  for (int64_t i = gid; i < nm; i += groups) {
    const KeyIdx k = key_idx(p, __ldg(p.multi_keys + i));
    RowRegs<VPL, ADAM> r;
    load_row<G, VPL, ADAM>(g, p, k.row, r);
    float4 grad[VPL];
    key_grad<G, VPL, GP, GU>(g, p, k.s0, k.s1, k.first, nullptr, 0, grad);
    apply_update<G, VPL, ADAM>(g, p, k.row, r, grad);
  }
}

// A persistent grid of G-lane groups walks the unique keys u = gid, gid +
// groups, ... (U from the lookup), S keys deep: while key u is
// updated, the next S-1 keys' rows [emb | state] (and a singleton's
// pooled gradient row) are in flight into shared memory, and the key after
// those has its indices loaded.  TMA: the group's lane 0 copies each row with
// one bulk copy on the stage's transaction barrier, which every lane waits
// on.  Otherwise each lane copies (cp.async) and reads back only its own
// 16-byte columns, so a lane's own wait is enough for the data.  A key's
// indices are shared by the group through shared memory (written by its
// lane 0, read after __syncwarp).  Other keys' gradients (repeated keys,
// long segments, unpooled gradients) are gathered while the key is updated.
// Pipeline depth: 4 when each group walks many keys (long-sequence batches),
// 2 otherwise (measured: 3 or 4 keys deep, or a fourth CTA per SM, only
// lengthen every request on the 26-feature step).
// AHEAD (S >= 3, gradients in device memory and too large for L2, keys seen
// 2 to kShortSeg times not listed): their gathers run ahead of the walk too.
// While key k is updated, the source records of key k+2's first G positions
// are loaded (one per lane) and, with key k+1's records in hand, key k+1's
// gradient rows are prefetched into L2, so that its gather starts from
// registers and L2 instead of two dependent DRAM round trips (measured on
// the large-table step: 3.32 -> 2.92 ms; where the gradients sit in L2 the
// extra work only costs).
template <int G, int VPL, bool ADAM, bool GP, bool GU, int S, bool TMA, bool AHEAD = false>
__global__ void __launch_bounds__(256, 3) row_update_kernel(const __grid_constant__ UpdateParams p) {
  static_assert(!AHEAD || (S >= 3 && TMA), "look-ahead needs key k+2 issued and device-memory gradients");
  pdl_wait();
  constexpr int NR = ADAM ? 3 : 2;             // row slices: emb, state(s)
  constexpr int NS = NR * VPL + VPL;           // staged float4 per thread per stage
  // [S][NS][blockDim] float4 (TMA: [S][groups][NS * G], each row contiguous
  // followed by the gradient row), then [S][groups] keys, then (TMA)
  // [S][groups] transaction barriers
  extern __shared__ float4 s_stage[];
  const GroupCtx<G> g;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int grp = tid / G, ngrp = nt / G;
  const int64_t groups = (int64_t)gridDim.x * blockDim.x / G;
  const int64_t U = (int64_t)p.bdev->U;
  const int D = p.ncol * 4;
  const int64_t u0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  // Keys seen 2 to kShortSeg times first, spread evenly over the groups,
  // when there are a few per group: their gradient rows are gathered when
  // the key is updated, so drawn by the stride below they would pile up in
  // some groups.  The walk then skips them.  (With many per group the walk's
  // staging is worth more than the balance; every group decides alike.)
  const int64_t nm = p.multi_keys ? (int64_t)p.bdev->nmulti : 0;
  const bool listed = p.multi_keys != nullptr && nm <= 4 * groups;
  if (listed) update_listed<G, VPL, ADAM, GP, GU>(p, u0, groups, nm);
  auto is_listed = [&](const KeyIdx& k) { return listed && k.s1 - k.s0 > 1 && k.s1 - k.s0 <= kShortSeg; };
  if (u0 >= U) return;
  KeyIdx* s_keys = reinterpret_cast<KeyIdx*>(s_stage + S * NS * nt);
  uint64_t* s_mbar = reinterpret_cast<uint64_t*>(s_keys + S * ngrp);
  auto key_slot = [&](int st) -> KeyIdx* { return s_keys + st * ngrp + grp; };
  auto mbar = [&](int st) -> uint64_t* { return s_mbar + st * ngrp + grp; };
  // this lane's 16-byte column of row slice sl (the gradient row: sl = NR * VPL)
  auto slot = [&](int stage, int sl) -> float4* {
    if (TMA) {
      float4* region = s_stage + (size_t)(stage * ngrp + grp) * NS * G;
      const int r = sl / VPL, v = sl % VPL;
      return region + (r < NR ? r * p.ncol : NR * VPL * G) + g.lane + v * G;
    }
    return s_stage + ((stage * NS + sl) * nt + tid);
  };
  const int stride = TMA ? G : nt;  // between a lane's columns v and v + 1
  const unsigned row_bytes = (unsigned)p.row_floats * 4u;
  if (TMA) {
    if (g.lane == 0)
      for (int st = 0; st < S; ++st) mbar_init(mbar(st), 1);
    __syncwarp(g.mask);
  }
  auto issue = [&](int stage, const KeyIdx& k) {
    const bool copy = k.row >= 0 && !is_listed(k);
    const bool stage_grad = GP && !GU && k.s1 - k.s0 == 1;
    const float* base = p.row_data + (int64_t)(k.row < 0 ? 0 : k.row) * p.row_floats;
    const float* gsrc_row = p.gp + (int64_t)k.first.x * D;
    if (TMA) {
      // the whole row [emb | state] and a singleton's gradient row by the
      // bulk-copy engine, one instruction each; one barrier phase per issue
      if (g.lane == 0) {
        *key_slot(stage) = k;
        fence_async_smem();
        mbar_arrive_expect(mbar(stage), copy ? row_bytes + (stage_grad ? (unsigned)D * 4u : 0u) : 0u);
        if (copy) {
          float4* region = s_stage + (size_t)(stage * ngrp + grp) * NS * G;
          bulk_row(region, base, row_bytes, mbar(stage));
          if (stage_grad) bulk_row(region + NR * VPL * G, gsrc_row, (unsigned)D * 4u, mbar(stage));
        }
      }
      return;
    }
    if (g.lane == 0) *key_slot(stage) = k;
    if (!copy) return;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      if (col < p.ncol) {
#pragma unroll
        for (int r = 0; r < NR; ++r) cp_async16(slot(stage, r * VPL + v), base + r * D + 4 * col);
        if (stage_grad) cp_async16(slot(stage, NR * VPL + v), gsrc_row + 4 * col);
      }
    }
  };
  auto idx_of = [&](int64_t k) -> KeyIdx {
    const int64_t uk = u0 + k * groups;
    return uk < U ? key_idx(p, uk) : KeyIdx{0, 1, -1, 0, make_int4(0, 1, 0, 0)};
  };
  auto gathers = [&](const KeyIdx& k) { return k.s1 - k.s0 > 1 && k.s1 - k.s0 <= kShortSeg && !is_listed(k); };
  auto load_rec = [&](const KeyIdx& k) -> int4 {
    return gathers(k) && g.lane < k.s1 - k.s0 ? __ldg(p.gsrc + k.s0 + g.lane) : make_int4(0, 1, 0, 0);
  };
  auto prefetch_rows = [&](const KeyIdx& k, int4 rec) {
    if (k.row < 0 || !gathers(k) || g.lane >= k.s1 - k.s0) return;
    for (int off = 0; off < D * 4; off += 128) {
      if (GP) prefetch_l2(p.gp + (int64_t)rec.x * D + off / 4);
      if (GU) prefetch_l2(p.gu + (int64_t)rec.z * D + off / 4);
    }
  };
  // AHEAD: the source records of key k (rec_cur) and of key k+1 (rec_nxt)
  int4 rec_cur = make_int4(0, 1, 0, 0), rec_nxt = make_int4(0, 1, 0, 0);
  if constexpr (AHEAD) {
    rec_cur = load_rec(idx_of(0));
    rec_nxt = load_rec(idx_of(1));
  }
#pragma unroll
  for (int k = 0; k < S - 1; ++k) {
    issue(k, idx_of(k));
    if (!TMA) cp_async_commit();
  }
  KeyIdx pre = idx_of(S - 1);
  for (int64_t k = 0; u0 + k * groups < U; ++k) {
    __syncwarp(g.mask);  // every lane is done with the slot about to be reused
    issue((int)((k + S - 1) % S), pre);
    if (!TMA) cp_async_commit();
    pre = idx_of(k + S);
    __syncwarp(g.mask);
    const int stage = (int)(k % S);
    const KeyIdx cur = *key_slot(stage);
    const bool staged_grad = GP && !GU && cur.s1 - cur.s0 == 1;
    const int4 rec = rec_cur;
    if constexpr (AHEAD) {
      // keys k+1 and k+2 sit in their stages' slots (issued S-1 keys ahead)
      rec_cur = rec_nxt;
      prefetch_rows(*key_slot((int)((k + 1) % S)), rec_cur);
      rec_nxt = load_rec(*key_slot((int)((k + 2) % S)));
    }
    float4 grad[VPL];
    if (TMA) {
      // the (k / S)-th use of this stage's barrier
      const unsigned parity = (unsigned)((k / S) & 1);
      if (!mbar_wait(mbar(stage), parity, p.spin_max)) {
        if (g.lane == 0) raise_error(p.st, p.mirror, kErrTimeout);
        mbar_wait(mbar(stage), parity, p.spin_max);
      }
    } else {
      cp_async_wait<S - 1>();
    }
    if (is_listed(cur)) continue;  // updated above
    key_grad<G, VPL, GP, GU>(g, p, cur.s0, cur.s1, cur.first,
                             staged_grad ? slot(stage, NR * VPL) : nullptr, stride, grad, rec, AHEAD && gathers(cur));
    if (cur.row >= 0) {
      RowRegs<VPL, ADAM> r;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        r.w[v] = *slot(stage, 0 * VPL + v);
        r.s1[v] = *slot(stage, 1 * VPL + v);
        if (ADAM) r.s2[v] = *slot(stage, 2 * VPL + v);
      }
      apply_update<G, VPL, ADAM>(g, p, cur.row, r, grad);
    }
  }
  pdl_trigger();
}

// Rows wider than one 16-byte column per lane (D > 128): the same walk over
// keys with the row loaded into registers (staging would need too much
// shared memory).
template <int G, int VPL, bool ADAM, bool GP, bool GU>
__global__ void __launch_bounds__(256, 2) row_update_wide_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  const GroupCtx<G> g;
  const int64_t groups = (int64_t)gridDim.x * blockDim.x / G;
  const int64_t U = (int64_t)p.bdev->U;
  for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G; u < U; u += groups) {
    const KeyIdx k = key_idx(p, u);
    RowRegs<VPL, ADAM> r;
    load_row<G, VPL, ADAM>(g, p, k.row, r);
    float4 grad[VPL];
    key_grad<G, VPL, GP, GU>(g, p, k.s0, k.s1, k.first, nullptr, 0, grad);
    apply_update<G, VPL, ADAM>(g, p, k.row, r, grad);
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ host
int group_lanes_for(int D);

// gradient bytes above which the row update prefetches gathers (half of L2)
constexpr int64_t kAheadGradBytes = 64ll << 20;

// seg_reduce span: kChunk * 2^k positions (at most 8 steps), as long as 16K
// lane groups remain to fill the GPU
int64_t update_chunk_for(int64_t N, int) {
  int64_t span = kChunk;
  while (span < 8 * kChunk && (N + 2 * span - 1) / (2 * span) >= 16384) span *= 2;
  return span;
}

// sets a kernel's dynamic shared memory limit once per device
template <typename K>
static cudaError_t smem_attr(K kernel, size_t smem, bool (&done)[64]) {
  if (smem <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

template <int G, int VPL, bool GP, bool GU>
static cudaError_t launch_update_g(const UpdateParams& p, bool adam, int64_t ucap, bool tma, bool rows_tma,
                                   bool ahead_ok, cudaStream_t s) {
  {
    // one lane group per span; one staging slot per position, row and lane
    constexpr size_t smem = (size_t)256 * kChunk * sizeof(float4);
    static bool attr[64] = {false}, attr_t[64] = {false};
    cudaError_t e = tma ? smem_attr(seg_partial_kernel<G, VPL, GP, GU, true>, smem, attr_t)
                        : smem_attr(seg_partial_kernel<G, VPL, GP, GU, false>, smem, attr);
    if (e != cudaSuccess) return e;
    const int64_t spans = (p.N + p.span - 1) / p.span;
    const unsigned blocks = (unsigned)std::max<int64_t>(1, (spans * G + 255) / 256);
    {
      LaunchScope ls("seg_partial", s);
      e = tma ? launch_pdl(seg_partial_kernel<G, VPL, GP, GU, true>, blocks, 256, smem, s, p)
              : launch_pdl(seg_partial_kernel<G, VPL, GP, GU, false>, blocks, 256, smem, s, p);
      if (e != cudaSuccess) return e;
    }
    constexpr size_t csmem = (size_t)256 * VPL * sizeof(Acc4);
    static bool cattr[64] = {false};
    if ((e = smem_attr(seg_combine_kernel<G, VPL>, csmem, cattr)) != cudaSuccess) return e;
    int64_t cblocks = 4 * (int64_t)kSMs;
    if (cblocks > spans) cblocks = spans;
    LaunchScope ls("seg_combine", s);
    e = launch_pdl(seg_combine_kernel<G, VPL>, (unsigned)(cblocks < 1 ? 1 : cblocks), 256, csmem, s, p);
    if (e != cudaSuccess) return e;
  }
  // persistent: as many CTAs as fit at once (U is known only on the device)
  int64_t blocks = (ucap * G + 255) / 256;
  const int64_t resident = (int64_t)kSMs * (VPL == 1 ? 3 : 2);
  if (blocks > resident) blocks = resident;
  if (blocks < 1) blocks = 1;
  LaunchScope ls("row_update", s);
  if constexpr (VPL == 1) {
    // keys per group decide the depth (U <= ucap)
    const bool deep = ucap / (blocks * (256 / G)) >= 64;
    const bool ahead = deep && rows_tma && ahead_ok;
    const int S = deep ? 4 : 2;
    const int ns = ((adam ? 3 : 2) * VPL + VPL);
    const size_t smem = (size_t)S * ns * 256 * sizeof(float4) + (size_t)S * (256 / G) * sizeof(KeyIdx) +
                        (rows_tma ? (size_t)S * (256 / G) * sizeof(uint64_t) : 0);
    cudaError_t e;
    auto go = [&](auto kernel) -> cudaError_t {
      cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
      return launch_pdl(kernel, (unsigned)blocks, 256, smem, s, p);
    };
    if (rows_tma) {
      if (adam)
        e = ahead  ? go(row_update_kernel<G, VPL, true, GP, GU, 4, true, true>)
            : deep ? go(row_update_kernel<G, VPL, true, GP, GU, 4, true>)
                   : go(row_update_kernel<G, VPL, true, GP, GU, 2, true>);
      else
        e = ahead  ? go(row_update_kernel<G, VPL, false, GP, GU, 4, true, true>)
            : deep ? go(row_update_kernel<G, VPL, false, GP, GU, 4, true>)
                   : go(row_update_kernel<G, VPL, false, GP, GU, 2, true>);
    } else {
      if (adam)
        e = deep ? go(row_update_kernel<G, VPL, true, GP, GU, 4, false>)
                 : go(row_update_kernel<G, VPL, true, GP, GU, 2, false>);
      else
        e = deep ? go(row_update_kernel<G, VPL, false, GP, GU, 4, false>)
                 : go(row_update_kernel<G, VPL, false, GP, GU, 2, false>);
    }
    if (e != cudaSuccess) return e;
  } else {
    if (adam)
      return launch_pdl(row_update_wide_kernel<G, VPL, true, GP, GU>, (unsigned)blocks, 256, 0, s, p);
    else
      return launch_pdl(row_update_wide_kernel<G, VPL, false, GP, GU>, (unsigned)blocks, 256, 0, s, p);
  }
  return cudaGetLastError();
}

template <int G, int VPL>
static cudaError_t launch_update_t(const UpdateParams& p, bool adam, int64_t ucap, bool tma, bool rows_tma,
                                   bool ahead_ok, cudaStream_t s) {
  if (p.gp && p.gu) return launch_update_g<G, VPL, true, true>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (p.gp) return launch_update_g<G, VPL, true, false>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (p.gu) return launch_update_g<G, VPL, false, true>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  return launch_update_g<G, VPL, false, false>(p, adam, ucap, tma, rows_tma, ahead_ok, s);  // touched rows, zero gradient
}

// device memory of this GPU's own address space (allocations and VMM
// mappings of device memory): the bulk-copy engine reads it; other memory
// (host-mapped, managed) takes the cp.async path
static bool device_memory(const void* ptr) {
  if (!ptr) return true;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

cudaError_t launch_update(recis_table* t, recis_batch* b, const float* grad_pooled,
                          const float* grad_unpooled, int64_t span, float lr_t, float inv_sqrt_bc2,
                          cudaStream_t s) {
  UpdateParams p;
  p.N = b->N;
  p.ncol = t->D / 4;
  p.mean = b->combiner == RECIS_MEAN;
  p.row_floats = t->row_floats;
  p.span = span;
  p.gsrc = b->gsrc;
  p.gfirst = b->gfirst;
  // keys seen 2 to kShortSeg times are listed by the sample-sort dedup
  p.multi_keys = b->N <= kSampleSortMaxN ? b->multi_keys : nullptr;
  p.seg_of = b->seg_of;
  p.seg_start = b->seg_start;
  p.rows = b->rows;
  p.bdev = b->bdev;
  p.gp = grad_pooled;
  p.gu = grad_unpooled;
  p.gbuf = b->gbuf;
  p.row_data = reinterpret_cast<float*>(t->rows.va);
  p.partials = b->partials;
  p.long_segs = b->long_segs;
  p.seg_cap = b->capSegs;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  p.spin_max = spin_limit();
  p.lr = lr_t;
  p.eps = (float)t->cfg.eps;
  p.beta1 = (float)t->cfg.beta1;
  p.beta2 = (float)t->cfg.beta2;
  p.omb1 = (float)(1.0 - t->cfg.beta1);
  p.omb2 = (float)(1.0 - t->cfg.beta2);
  p.inv_sqrt_bc2 = inv_sqrt_bc2;
  if (p.N == 0) return cudaSuccess;
  const bool adam = t->cfg.optimizer == RECIS_ADAM;
  const int64_t ucap = b->N;  // U <= N; groups past U return at once
  // bulk copies for gradients in device memory, and for rows too when the
  // EmbeddingBlocks are device memory
  const bool tma = device_memory(grad_pooled) && device_memory(grad_unpooled);
  const bool rows_tma = tma && t->rows.host_numa < 0;
  // the row update gathers ahead when the keys seen a few times are not
  // listed and the gradients are too large to stay in L2
  const int64_t grad_bytes = (grad_pooled ? (int64_t)b->F * b->B * t->D * 4 : 0) +
                             (grad_unpooled ? b->N * t->D * 4 : 0);
  const bool ahead_ok = p.multi_keys == nullptr && grad_bytes > kAheadGradBytes;
  const int ncol = p.ncol;
  if (ncol <= 1) return launch_update_t<1, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 2) return launch_update_t<2, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 4) return launch_update_t<4, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 8) return launch_update_t<8, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 16) return launch_update_t<16, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 32) return launch_update_t<32, 1>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 64) return launch_update_t<32, 2>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  if (ncol <= 128) return launch_update_t<32, 4>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
  return launch_update_t<32, 8>(p, adam, ucap, tma, rows_tma, ahead_ok, s);
}

}  // namespace recis
