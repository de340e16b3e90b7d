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
// summed in fp64 in position order and rounded once to fp32.  Two launches:
//   seg_reduce  segments longer than kShortSeg (hot keys) are cut into
//               chunks of kChunk positions; each lane group sums its chunk's
//               part of a segment into an fp64 partial; the group that
//               arrives last adds the partials in chunk order (for a segment
//               of more than 64 chunks, in two levels: per block of 32
//               chunks, then the block sums in block order) and stores g(u)
//               in gbuf at row seg_start[u] / kChunk (a long segment is the
//               only long one starting in its chunk).
//   row_update  one lane group per unique key loads the row [emb | state],
//               sums the key's gradient terms itself when the segment is
//               short (all loads issued before the sum) or reads gbuf, and
//               applies Adagrad or Adam in place.  Keys seen 2 to kShortSeg
//               times come from the dedup's list, spread evenly over the
//               groups, when there are a few per group.
// No float atomics anywhere; the result does not depend on scheduling.
#include "segreduce.cuh"

namespace recis {

constexpr int kChunk = 16;  // seg_reduce positions per group (<= kShortSeg + 1)
static_assert(kChunk <= kShortSeg + 1, "a chunk must hold at most one long segment start");
static_assert(kChunk == kShortSeg, "the dedup lists long chunks of kShortSeg positions");
constexpr int kCombineBlock = 32;  // chunks per block of the two-level combine

struct UpdateParams {
  int64_t N;
  int32_t ncol;             // D / 4
  int32_t mean;
  int32_t row_floats;
  int64_t nchunks;          // seg_reduce chunks
  const int4* gsrc;         // [N] per sorted position: {gradient row, bag length, occurrence, 0}
  const int4* gfirst;       // [U] per unique key: gsrc of one of its occurrences
  const uint64_t* meta;     // [N] per sorted position, bit 63: long segment (null: use seg_start)
  const int32_t* long_chunks;  // chunks holding a long segment, bdev->nlong of them (or null)
  const int32_t* seg_of;    // [N] sorted position -> unique index
  const int32_t* seg_start; // [U+1]
  const int64_t* rows;      // [U]
  const BatchDev* bdev;     // U of the lookup
  const float* gp;          // grad_pooled [B][F][D] or null
  const float* gu;          // grad_unpooled [N][D] or null
  float* gbuf;              // [nchunks][D] reduced gradients of long segments
  float* row_data;
  double* partials;         // [nchunks][2][D]
  int32_t* counters;        // [U] last-arrival tickets (self-resetting)
  int32_t* chunk_counters;  // [nchunks][2] block-level tickets (self-resetting)
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
// One group per chunk of kChunk sorted positions.  Lanes resolve G positions
// at a time: the long-segment mark (or, without marks, the segment's bounds),
// the segment and the gradient source; positions of short segments are
// skipped, so a chunk without a long segment ends after one load.  A chunk
// meets at most two long segments (one ending, one starting); each gets one
// partial per chunk, in slot 0 if it starts at or before the chunk's first
// position, else slot 1.
template <int G, int VPL, bool GP, bool GU>
__device__ __forceinline__ void reduce_chunk(const GroupCtx<G>& g, const UpdateParams& p, int64_t chunk) {
  const int64_t D = (int64_t)p.ncol * 4;
  const int64_t p0 = chunk * kChunk;
  const int64_t p1 = p0 + kChunk < p.N ? p0 + kChunk : p.N;
  if (!p.meta && !p.long_chunks) {
    // no marks from the dedup: a segment lying wholly inside the chunk is
    // short (kChunk <= kShortSeg), so only the segments of the chunk's first
    // and last positions can be long; a chunk where neither is ends here
    bool lng = false;
    for (int e = g.lane; e < 2; e += G) {
      const int32_t sg = __ldg(p.seg_of + (e == 0 ? p0 : p1 - 1));
      lng |= __ldg(p.seg_start + sg + 1) - __ldg(p.seg_start + sg) > kShortSeg;
    }
    if (!g.ballot(lng)) return;
  }
  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  int32_t cur = -1;
  int64_t cst = 0, cen = 0;
  auto flush = [&]() {
    // segments of up to two blocks of chunks: one last-arrival combine;
    // longer ones (hot keys of long sequences): two levels
    const bool two_level = (cen - 1) / kChunk - cst / kChunk >= 2 * kCombineBlock;
    if (two_level ? combine_split2<G, VPL, VPL >= 4 ? 1 : 4 / VPL, kCombineBlock>(
                        g, acc, p.partials, p.chunk_counters, p.counters, cur, chunk, cst <= p0, cst, cen,
                        kChunk, p.ncol)
                  : combine_split<G, VPL, VPL >= 4 ? 1 : 4 / VPL>(g, acc, p.partials, p.counters, cur, chunk,
                                                                 cst <= p0, cst, cen, kChunk, p.ncol)) {
      float4* dst = reinterpret_cast<float4*>(p.gbuf + (cst / kChunk) * D);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (col < p.ncol) __stcg(dst + col, acc_round(acc[v]));
      }
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  };
  for (int64_t sub = p0; sub < p1; sub += G) {
    const int64_t q = sub + g.lane;
    bool maybe = q < p1;
    if (maybe && p.meta) maybe = (__ldg(p.meta + q) >> 63) != 0;
    if (!g.ballot(maybe)) continue;
    int32_t seg = -1, st = 0, en = 0;
    Src s{0, 0, 1.0};
    if (maybe) {
      seg = __ldg(p.seg_of + q);
      s = make_src(p, __ldg(p.gsrc + q));
      st = __ldg(p.seg_start + seg);
      en = __ldg(p.seg_start + seg + 1);
    }
    const bool is_long = maybe && en - st > kShortSeg;
    unsigned rest = g.ballot(is_long);
    while (rest) {
      const int a = __ffs(rest) - 1;
      const int32_t sg = g.bcast(seg, a);
      const unsigned same = g.ballot(is_long && seg == sg);  // lanes a .. a+cnt-1
      const int cnt = __popc(same);
      if (sg != cur) {
        if (cur >= 0) flush();
        cur = sg;
        cst = g.bcast(st, a);
        cen = g.bcast(en, a);
      }
      constexpr int K = kRowsInFlight<VPL, GP && GU>;
      for (int k0 = 0; k0 < cnt; k0 += K)
        add_terms<G, VPL, K, GP, GU>(g, p, s, a + k0, cnt - k0 < K ? cnt - k0 : K, acc);
      rest &= ~same;
    }
  }
  if (cur >= 0) flush();
}

// With the dedup's list of chunks holding a long segment, a persistent grid
// of groups walks the list; without it, one group per chunk.
// resident CTAs of 256 threads per SM of the long-segment reduction
template <int VPL>
constexpr int kSegReduceCtas = VPL == 1 ? 3 : (VPL == 2 ? 2 : 1);

template <int G, int VPL, bool GP, bool GU>
__global__ void __launch_bounds__(256, kSegReduceCtas<VPL>)
    seg_reduce_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  const GroupCtx<G> g;
  const int64_t gid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (p.long_chunks) {
    const int64_t n = (int64_t)p.bdev->nlong;
    const int64_t groups = (int64_t)gridDim.x * blockDim.x / G;
    for (int64_t i = gid; i < n; i += groups) reduce_chunk<G, VPL, GP, GU>(g, p, __ldg(p.long_chunks + i));
  } else if (gid < p.nchunks) {
    reduce_chunk<G, VPL, GP, GU>(g, p, gid);
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ seg_reduce, staged
// The same reduction for one 16-byte column per lane (D = 4G) and one kind of
// gradient (pooled or unpooled), G >= 8: groups walk the listed chunks (one
// each when the grid covers the list); a chunk's positions are resolved by
// the group (each lane kChunk / G of them), and the gradient rows of all its
// long positions are copied into shared memory by cp.async at once, one slot
// per position and lane, so a chunk costs one round trip for its rows instead
// of one per few rows.  Each lane copies and reads back only its own columns.
__device__ __forceinline__ void cp_async16_(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

template <int G>
struct ChunkPos {
  static constexpr int E = G >= kChunk ? 1 : kChunk / G;  // positions per lane
  int32_t seg[E], st[E], en[E], src[E];
  double scale[E];
  unsigned mask;  // bit t: position t of the chunk is in a long segment
};

template <int G, bool GP>
__device__ __forceinline__ void chunk_indices(const GroupCtx<G>& g, const UpdateParams& p, int64_t chunk,
                                              ChunkPos<G>& c) {
  constexpr int E = ChunkPos<G>::E;
  const int64_t p0 = chunk * kChunk;
  bool lng[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int t = g.lane + e * G;
    const int64_t q = p0 + t;
    lng[e] = false;
    c.seg[e] = 0;
    c.st[e] = c.en[e] = c.src[e] = 0;
    c.scale[e] = 1.0;
    if (chunk >= 0 && t < kChunk && q < p.N) {
      const bool marked = p.meta ? (__ldg(p.meta + q) >> 63) != 0 : true;
      const int32_t sg = __ldg(p.seg_of + q);
      const int4 gs = __ldg(p.gsrc + q);
      const int32_t a = __ldg(p.seg_start + sg), b = __ldg(p.seg_start + sg + 1);
      lng[e] = marked && b - a > kShortSeg;
      c.seg[e] = sg;
      c.st[e] = a;
      c.en[e] = b;
      c.src[e] = GP ? gs.x : gs.z;
      c.scale[e] = (GP && p.mean) ? 1.0 / (double)gs.y : 1.0;
    }
  }
  c.mask = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) c.mask |= g.ballot(lng[e]) << (e * G);
}

template <int G, bool GP>
__global__ void __launch_bounds__(256, 3) seg_reduce_staged_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  constexpr int E = ChunkPos<G>::E;
  extern __shared__ float4 s_rows[];  // [groups of the CTA][kChunk][G]
  const GroupCtx<G> g;
  float4* rows = s_rows + (size_t)(threadIdx.x / G) * kChunk * G;
  const int64_t groups = (int64_t)gridDim.x * blockDim.x / G;
  const int64_t gid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const int64_t n = (int64_t)p.bdev->nlong;
  const int64_t D = (int64_t)p.ncol * 4;
  const float* grad = GP ? p.gp : p.gu;
  auto chunk_of = [&](int64_t i) -> int64_t { return i < n ? (int64_t)__ldg(p.long_chunks + i) : -1; };
  ChunkPos<G> cur;
  int64_t i = gid;
  int64_t chunk = chunk_of(i);
  chunk_indices<G, GP>(g, p, chunk, cur);
  while (chunk >= 0) {
    // this chunk's gradient rows into shared memory
    for (unsigned m = cur.mask; m; m &= m - 1) {
      const int t = __ffs(m) - 1;
      const int32_t src = g.bcast(t / G == 0 ? cur.src[0] : cur.src[E - 1], t % G);
      if (g.lane < p.ncol) cp_async16_(rows + t * G + g.lane, grad + (int64_t)src * D + 4 * g.lane);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    // the next chunk's positions meanwhile
    const int64_t next = chunk_of(i + groups);
    ChunkPos<G> nxt;
    chunk_indices<G, GP>(g, p, next, nxt);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // the long positions in order, one segment run at a time
    const int64_t p0 = chunk * kChunk;
    Acc4 acc = acc_zero();
    int32_t sg = -1, cst = 0, cen = 0;
    auto flush = [&]() {
      Acc4 a1[1] = {acc};
      const bool two_level = (cen - 1) / kChunk - cst / kChunk >= 2 * kCombineBlock;
      if (two_level ? combine_split2<G, 1, 2, kCombineBlock>(g, a1, p.partials, p.chunk_counters, p.counters,
                                                            sg, chunk, cst <= p0, cst, cen, kChunk, p.ncol)
                    : combine_split<G, 1, 2>(g, a1, p.partials, p.counters, sg, chunk, cst <= p0, cst, cen,
                                             kChunk, p.ncol)) {
        if (g.lane < p.ncol) __stcg(reinterpret_cast<float4*>(p.gbuf + (cst / kChunk) * D) + g.lane,
                                    acc_round(a1[0]));
      }
      acc = acc_zero();
    };
    for (unsigned m = cur.mask; m; m &= m - 1) {
      const int t = __ffs(m) - 1;
      const int e = t / G, l = t % G;
      const int32_t s = g.bcast(e == 0 ? cur.seg[0] : cur.seg[E - 1], l);
      if (s != sg) {
        if (sg >= 0) flush();
        sg = s;
        cst = g.bcast(e == 0 ? cur.st[0] : cur.st[E - 1], l);
        cen = g.bcast(e == 0 ? cur.en[0] : cur.en[E - 1], l);
      }
      const double sc = g.bcast(e == 0 ? cur.scale[0] : cur.scale[E - 1], l);
      if (g.lane < p.ncol) {
        const float4 v = rows[t * G + g.lane];
        acc.x += (double)v.x * sc;
        acc.y += (double)v.y * sc;
        acc.z += (double)v.z * sc;
        acc.w += (double)v.w * sc;
      }
    }
    if (sg >= 0) flush();
    i += groups;
    chunk = next;
    cur = nxt;
  }
  pdl_trigger();
}

// Chunks of kChunk positions holding a position of a long segment, listed
// for the staged reduction when the dedup listed none (the radix path): only
// the segments of a chunk's first and last positions can be long (a segment
// lying wholly inside a chunk is short).  The list's order depends on
// scheduling; every chunk's partial and every combine do not.
__global__ void __launch_bounds__(256) list_long_chunks_kernel(const __grid_constant__ UpdateParams p,
                                                               int32_t* out, BatchDev* bdev) {
  pdl_wait();
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  bool lng = false;
  if (c < p.nchunks) {
    const int64_t p0 = c * kChunk, p1 = p0 + kChunk < p.N ? p0 + kChunk : p.N;
    const int32_t a = __ldg(p.seg_of + p0), b = __ldg(p.seg_of + p1 - 1);
    lng = __ldg(p.seg_start + a + 1) - __ldg(p.seg_start + a) > kShortSeg ||
          __ldg(p.seg_start + b + 1) - __ldg(p.seg_start + b) > kShortSeg;
  }
  const unsigned bal = __ballot_sync(0xffffffffu, lng);
  const int lane = threadIdx.x & 31;
  unsigned at = 0;
  if (lane == 0 && bal) at = atomicAdd(&bdev->nlong, (unsigned)__popc(bal));
  at = __shfl_sync(0xffffffffu, at, 0);
  if (lng) out[at + __popc(bal & ((1u << lane) - 1u))] = (int32_t)c;
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
// a long segment's sum from gbuf, else the terms gathered here.
template <int G, int VPL, bool GP, bool GU>
__device__ __forceinline__ void key_grad(const GroupCtx<G>& g, const UpdateParams& p, int32_t s0,
                                         int32_t s1, int4 first, const float4* staged, int stride,
                                         float4 (&out)[VPL]) {
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
      if (g.lane < m) s = make_src(p, __ldg(p.gsrc + s0 + base + g.lane));
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
// pooled gradient row) are in flight into shared memory by cp.async, and the
// key after those has its indices loaded.  Each lane copies and reads back
// only its own 16-byte columns, so a lane's own wait is enough for the data;
// a key's indices are shared by the group through shared memory (written by
// its lane 0, read after __syncwarp).  Other keys' gradients (repeated keys,
// long segments, unpooled gradients) are gathered while the key is updated.
// Pipeline depth: 4 when each group walks many keys (long-sequence batches),
// 2 otherwise (measured: 3 or 4 keys deep, or a fourth CTA per SM, only
// lengthen every request on the 26-feature step).
template <int G, int VPL, bool ADAM, bool GP, bool GU, int S>
__global__ void __launch_bounds__(256, 3) row_update_kernel(const __grid_constant__ UpdateParams p) {
  pdl_wait();
  constexpr int NR = ADAM ? 3 : 2;             // row slices: emb, state(s)
  constexpr int NS = NR * VPL + VPL;           // staged float4 per thread per stage
  extern __shared__ float4 s_stage[];          // [S][NS][blockDim], then [S][groups] keys
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
  auto key_slot = [&](int st) -> KeyIdx* { return s_keys + st * ngrp + grp; };
  auto slot = [&](int stage, int sl) -> float4* { return s_stage + ((stage * NS + sl) * nt + tid); };
  auto issue = [&](int stage, const KeyIdx& k) {
    if (g.lane == 0) *key_slot(stage) = k;
    if (k.row < 0 || is_listed(k)) return;
    const float* base = p.row_data + (int64_t)k.row * p.row_floats;
    const bool stage_grad = GP && !GU && k.s1 - k.s0 == 1;
    const float* gsrc_row = p.gp + (int64_t)k.first.x * D;
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
#pragma unroll
  for (int k = 0; k < S - 1; ++k) {
    issue(k, idx_of(k));
    cp_async_commit();
  }
  KeyIdx pre = idx_of(S - 1);
  for (int64_t k = 0; u0 + k * groups < U; ++k) {
    __syncwarp(g.mask);  // every lane is done with the slot about to be reused
    issue((int)((k + S - 1) % S), pre);
    cp_async_commit();
    pre = idx_of(k + S);
    __syncwarp(g.mask);
    const int stage = (int)(k % S);
    const KeyIdx cur = *key_slot(stage);
    const bool staged_grad = GP && !GU && cur.s1 - cur.s0 == 1;
    float4 grad[VPL];
    cp_async_wait<S - 1>();
    if (is_listed(cur)) continue;  // updated above
    key_grad<G, VPL, GP, GU>(g, p, cur.s0, cur.s1, cur.first,
                             staged_grad ? slot(stage, NR * VPL) : nullptr, nt, grad);
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

int64_t update_chunk_for(int64_t, int) { return kChunk; }

template <int G, int VPL, bool GP, bool GU>
static cudaError_t launch_update_g(const UpdateParams& p, bool adam, int64_t ucap, cudaStream_t s) {
  if constexpr (VPL == 1 && G >= 8 && GP != GU) {
    if (p.long_chunks) {
      constexpr size_t smem = (size_t)256 * kChunk * sizeof(float4);  // one slot per position and lane
      static bool attr[64] = {false};
      int dev = 0;
      cudaGetDevice(&dev);
      if (dev < 0 || dev >= 64 || !attr[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(seg_reduce_staged_kernel<G, GP>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr[dev] = true;
      }
      // one group per chunk (the list holds at most nchunks; groups past its
      // length return at once): many groups in flight hide the combines'
      // fences and ticket round trips
      LaunchScope ls("seg_reduce", s);
      const int64_t blocks = (p.nchunks * G + 255) / 256;
      const cudaError_t e = launch_pdl(seg_reduce_staged_kernel<G, GP>, (unsigned)(blocks < 1 ? 1 : blocks), 256,
                                       smem, s, p);
      if (e != cudaSuccess) return e;
    }
  } else {
    int64_t blocks = (p.nchunks * G + 255) / 256;
    if (p.long_chunks && blocks > kSegReduceCtas<VPL> * kSMs) blocks = kSegReduceCtas<VPL> * kSMs;
    if (blocks < 1) blocks = 1;
    LaunchScope ls("seg_reduce", s);
    const cudaError_t e = launch_pdl(seg_reduce_kernel<G, VPL, GP, GU>, (unsigned)blocks, 256, 0, s, p);
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
    const int S = deep ? 4 : 2;
    const int ns = ((adam ? 3 : 2) * VPL + VPL);
    const size_t smem = (size_t)S * ns * 256 * sizeof(float4) + (size_t)S * (256 / G) * sizeof(KeyIdx);
    cudaError_t e;
    auto go = [&](auto kernel) -> cudaError_t {
      cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
      return launch_pdl(kernel, (unsigned)blocks, 256, smem, s, p);
    };
    if (adam)
      e = deep ? go(row_update_kernel<G, VPL, true, GP, GU, 4>) : go(row_update_kernel<G, VPL, true, GP, GU, 2>);
    else
      e = deep ? go(row_update_kernel<G, VPL, false, GP, GU, 4>) : go(row_update_kernel<G, VPL, false, GP, GU, 2>);
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
static cudaError_t launch_update_t(const UpdateParams& p, bool adam, int64_t ucap, cudaStream_t s) {
  if (p.gp && p.gu) return launch_update_g<G, VPL, true, true>(p, adam, ucap, s);
  if (p.gp) return launch_update_g<G, VPL, true, false>(p, adam, ucap, s);
  if (p.gu) return launch_update_g<G, VPL, false, true>(p, adam, ucap, s);
  return launch_update_g<G, VPL, false, false>(p, adam, ucap, s);  // touched rows, zero gradient
}

cudaError_t launch_update(recis_table* t, recis_batch* b, const float* grad_pooled,
                          const float* grad_unpooled, int64_t, float lr_t, float inv_sqrt_bc2,
                          cudaStream_t s) {
  UpdateParams p;
  p.N = b->N;
  p.ncol = t->D / 4;
  p.mean = b->combiner == RECIS_MEAN;
  p.row_floats = t->row_floats;
  p.nchunks = (b->N + kChunk - 1) / kChunk;
  p.gsrc = b->gsrc;
  p.gfirst = b->gfirst;
  // long-segment marks and the long-chunk list come from the sample-sort dedup
  p.meta = b->N <= kSampleSortMaxN ? b->ss_meta : nullptr;
  p.long_chunks = b->N <= kSampleSortMaxN ? b->long_chunks : nullptr;
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
  p.counters = b->seg_counter;
  p.chunk_counters = b->chunk_counter;
  p.lr = lr_t;
  p.eps = (float)t->cfg.eps;
  p.beta1 = (float)t->cfg.beta1;
  p.beta2 = (float)t->cfg.beta2;
  p.omb1 = (float)(1.0 - t->cfg.beta1);
  p.omb2 = (float)(1.0 - t->cfg.beta2);
  p.inv_sqrt_bc2 = inv_sqrt_bc2;
  if (p.N == 0) return cudaSuccess;
  if (!p.long_chunks) {
    // the radix-path dedup lists no chunks: list those holding a long segment
    cudaError_t e = cudaMemsetAsync(&b->bdev->nlong, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    LaunchScope ls("list_long", s);
    list_long_chunks_kernel<<<(unsigned)((p.nchunks + 255) / 256), 256, 0, s>>>(p, b->long_chunks, b->bdev);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.long_chunks = b->long_chunks;
  }
  const bool adam = t->cfg.optimizer == RECIS_ADAM;
  const int64_t ucap = b->N;  // U <= N; groups past U return at once
  const int ncol = p.ncol;
  if (ncol <= 1) return launch_update_t<1, 1>(p, adam, ucap, s);
  if (ncol <= 2) return launch_update_t<2, 1>(p, adam, ucap, s);
  if (ncol <= 4) return launch_update_t<4, 1>(p, adam, ucap, s);
  if (ncol <= 8) return launch_update_t<8, 1>(p, adam, ucap, s);
  if (ncol <= 16) return launch_update_t<16, 1>(p, adam, ucap, s);
  if (ncol <= 32) return launch_update_t<32, 1>(p, adam, ucap, s);
  if (ncol <= 64) return launch_update_t<32, 2>(p, adam, ucap, s);
  if (ncol <= 128) return launch_update_t<32, 4>(p, adam, ucap, s);
  return launch_update_t<32, 8>(p, adam, ucap, s);
}

}  // namespace recis
