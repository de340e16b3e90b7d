// pool.cu -- forward gather + bag pooling from the EmbeddingBlocks (RecIS
// README, Key optimisations > Efficient dynamic embedding: rows are read at the
// offsets the IDMap returned; > Operator implementation: vectorised memory
// access).
//
// Bags are contiguous ranges of occurrences, so the forward is a segmented
// reduction over occurrence order (segreduce.cuh): a group of G lanes owns a
// chunk of C occurrences, each lane one 16-byte column of the row.  The bag
// preparation (beside the dedup) writes the bag of every occurrence; the
// group resolves G positions at a time, one per lane (row, sorted position,
// unique key, bag and its bounds, two sub-blocks ahead), writes their
// gradient-source records lane-parallel, marks the positions that end a bag
// in one ballot, and copies the sub-block's rows into shared memory by
// cp.async at once (one round trip per sub-block), so the walk itself only
// adds rows and flushes at the
// marks.  A chunk whose bags all hold one occurrence (one-hot features) is a
// plain gather.
// Outputs: pooled rows [B][F][D] (sum, or mean = sum / length), optional
// unpooled rows [N][D], and the gradient source of every occurrence for the
// backward.
// Empty bags are written as zeros by a grid-stride prologue.
#include <climits>

#include "segreduce.cuh"

namespace recis {

struct PoolParams {
  int64_t N;
  int64_t nbags;
  int64_t B;
  int32_t F;
  int32_t ncol;    // D / 4
  int64_t C;       // chunk length
  int64_t nchunks;
  int32_t mean;
  int32_t row_floats;
  const int64_t* offs;   // bag offsets [nbags + 1]
  const int32_t* inv;    // [N]
  const int64_t* rows;   // [U]
  const float* row_data;
  float* pooled;         // [B][F][D] or null
  float* unpooled;       // [N][D] or null
  const uint32_t* spos;  // [N] sorted position of each occurrence
  const int64_t* pocc;   // [N] IDMap result of each occurrence (row if >= 0), or null
  int4* gsrc;            // [N] per sorted position: {gradient row b*F+f, bag length, occurrence, 0}
  int4* gfirst;          // [U] per unique key: the same, of one of its occurrences
  int32_t* chunk_bag;    // [nchunks] bag of each chunk's first occurrence
  int32_t* bag_of;       // [N] bag of every occurrence
  double* partials;
  int32_t* counters;     // [nbags]
  DevState* st;
  HostMirror* mirror;
  int spin_max;          // polls before a wait gives up
  uint64_t b_magic;      // ceil(2^64 / B) for B >= 2 (quotient by B as a high multiply), 0 for B = 1
};

// j / B for 0 <= j < 2^32: floor(j * ceil(2^64 / B) / 2^64) is exact, the
// rounding of the magic number adding less than 2^-32 to a quotient whose
// fraction is at most 1 - 1/B (division by invariant integers using
// multiplication, Granlund and Montgomery 1994).
__device__ __forceinline__ int div_b(const PoolParams& p, int j) {
  return p.b_magic ? (int)__umul64hi((unsigned long long)(unsigned)j, p.b_magic) : j;
}

// Bag preparation, one thread per bag (runs beside the dedup on a side
// stream): checks the offsets, writes the bag of every occurrence and of every
// chunk's first occurrence, and zeroes the pooled output of empty bags.  A bag
// of more than 32 occurrences has its bag ids written by the whole warp.
__global__ void __launch_bounds__(256) bag_prep_kernel(const __grid_constant__ PoolParams p) {
  const int64_t D = (int64_t)p.ncol * 4;
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (blockIdx.x == 0 && threadIdx.x == 0 &&
      (p.offs[0] != 0 || p.offs[p.nbags] != p.N))
    raise_error(p.st, p.mirror, kErrBadOffsets);
  // warp-uniform trip count, so the warp can share out its long bags
  for (int64_t j0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); j0 < p.nbags; j0 += stride) {
    const int64_t j = j0 + lane;
    int64_t lo = 0, hi = 0;
    if (j < p.nbags) {
      lo = p.offs[j];
      hi = p.offs[j + 1];
      if (lo < 0 || hi < lo || hi > p.N) {
        raise_error(p.st, p.mirror, kErrBadOffsets);
        lo = hi = 0;
      } else if (hi == lo) {
        if (p.pooled) {
          const int64_t f = j / p.B, b = j - f * p.B;
          float4* o = reinterpret_cast<float4*>(p.pooled + (b * p.F + f) * D);
          for (int c = 0; c < p.ncol; ++c) o[c] = f4_zero();
        }
      } else {
        for (int64_t c = (lo + p.C - 1) / p.C; c * p.C < hi; ++c) p.chunk_bag[c] = (int32_t)j;
        if (hi - lo <= 32)
          for (int64_t q = lo; q < hi; ++q) p.bag_of[q] = (int32_t)j;
      }
    }
    unsigned lng = __ballot_sync(0xffffffffu, hi - lo > 32);
    while (lng) {
      const int l = __ffs(lng) - 1;
      const int64_t a = __shfl_sync(0xffffffffu, lo, l), e = __shfl_sync(0xffffffffu, hi, l);
      const int32_t jl = (int32_t)(j0 + l);
      for (int64_t q = a + lane; q < e; q += 32) p.bag_of[q] = jl;
      lng &= lng - 1;
    }
  }
}

// rows per lane staged at once by the bag walk: a sub-block (G), at most
// 16 16-byte slots per lane
template <int G, int VPL>
__host__ __device__ constexpr int pool_piece() {
  return 16 / VPL < G ? 16 / VPL : G;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// TMA: the bag walk's rows are copied by the bulk-copy engine (EmbeddingBlocks
// in device memory), else by cp.async.
template <int G, int VPL, bool TMA>
__global__ void __launch_bounds__(256, VPL == 1 ? 3 : (VPL == 2 ? 2 : 1))
    pool_kernel(const __grid_constant__ PoolParams p) {
  pdl_wait();
  // all positions, bags and rows fit in 32 bits (N < 2^30, F*B < 2^31,
  // rows < 2^31), so the walk runs on 32-bit integers
  const int ncol = p.ncol;
  const int D = ncol * 4;
  const GroupCtx<G> g;
  const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (chunk >= p.nchunks) return;
  const int N = (int)p.N, nbags = (int)p.nbags, C = (int)p.C, B = (int)p.B, F = p.F;
  const int p0 = (int)chunk * C;
  const int p1 = p0 + C < N ? p0 + C : N;

  // Row, sorted position and unique index of the G positions of one
  // sub-block, one position per lane.  The row of an occurrence whose key
  // was already present comes straight from the IDMap result of the dedup.
  struct Ids {
    int row, spos, seg;
  };
  int lim = p1;  // positions below lim are walked (the bag walk moves it to a bag end)
  auto resolve = [&](int sub) {
    Ids r{-1, 0, 0};
    const int q = sub + g.lane;
    if (q < lim) {
      r.seg = __ldg(p.inv + q);
      r.spos = (int)__ldg(p.spos + q);
      const int64_t pr = p.pocc ? __ldcg(p.pocc + q) : -2;
      r.row = pr >= 0 ? (int)pr : (int)__ldg(p.rows + r.seg);
    }
    return r;
  };
  // bag of a position and its bounds (bag_of is written beside the dedup)
  struct Bag {
    int j, lo, hi;
  };
  auto bag_at = [&](int sub) {
    Bag r{0, 0, 0};
    const int q = sub + g.lane;
    if (q < lim) {
      int j = __ldg(p.bag_of + q);
      if (j < 0 || j >= nbags) j = 0;  // only with malformed bag offsets (reported by the preparation)
      r.j = j;
      r.lo = (int)__ldg(p.offs + j);
      r.hi = (int)__ldg(p.offs + j + 1);
    }
    return r;
  };
  // the ids of the first sub-block are in flight while the bag walk starts
  const Ids ids0 = resolve(p0);

  // bag containing p0 (precomputed), its start, and the ends of the G bags
  // from it on (for the one-hot test)
  int j0 = p.chunk_bag[chunk];
  if (j0 < 0 || j0 >= nbags) {  // only with malformed offsets
    if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
    j0 = 0;
  }
  const int cur_start = (int)p.offs[j0];
  const int wend = (j0 + g.lane < nbags) ? (int)p.offs[j0 + g.lane + 1] : INT_MAX;

  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();

  // the pooled row of bag j (sum, or mean over its len occurrences)
  auto store_bag = [&](int j, int len) {
    if (!p.pooled) return;
    const int f = div_b(p, j);
    float4* o = reinterpret_cast<float4*>(p.pooled + (int64_t)((j - f * B) * F + f) * D);
    const double dlen = (double)len;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      if (col < ncol) {
        Acc4 r = acc[v];
        if (p.mean) {
          r.x /= dlen;
          r.y /= dlen;
          r.z /= dlen;
          r.w /= dlen;
        }
        __stcs(o + col, acc_round(r));
      }
    }
  };

  extern __shared__ float4 s_ring[];  // [groups][PR][VPL][G] staged rows of the bag walk
  const int m = p1 - p0;

  // A chunk whose bags each hold exactly one occurrence (one-hot features, or
  // a one-hot stretch of a multi-hot one) is a plain gather: position p0 + t
  // is bag j0 + t, and the pooled row (sum, or mean over one row) is the row
  // itself.  K row loads per lane are in flight at once.
  bool onehot = cur_start == p0;
  for (int s = 0; onehot && s < m; s += G) {
    const int e = s == 0 ? wend
                         : ((j0 + s + g.lane < nbags) ? (int)p.offs[j0 + s + g.lane + 1] : INT_MAX);
    onehot = g.ballot(s + g.lane < m && e != p0 + s + g.lane + 1) == 0u;
  }
  if (onehot) {
    constexpr int K = (VPL >= 8 ? 1 : 8 / VPL) < G ? (VPL >= 8 ? 1 : 8 / VPL) : G;
    for (int s = 0; s < m; s += G) {
      const Ids ids = s == 0 ? ids0 : resolve(p0 + s);
      int out = 0;  // pooled row b*F+f of this lane's bag
      if (s + g.lane < m) {
        const int j = j0 + s + g.lane;
        const int f = div_b(p, j);
        out = (j - f * B) * F + f;
        const int4 src = make_int4(out, 1, p0 + s + g.lane, 0);
        p.gsrc[ids.spos] = src;
        p.gfirst[ids.seg] = src;
      }
      const int cnt = m - s < G ? m - s : G;
      for (int t0 = 0; t0 < cnt; t0 += K) {
        float4 val[K][VPL];
#pragma unroll
        for (int u = 0; u < K; ++u) {
          const int row = g.bcast(ids.row, (t0 + u) % G);
          const bool ok = t0 + u < cnt && row >= 0;
          const float4* src =
              reinterpret_cast<const float4*>(p.row_data + (int64_t)(ok ? row : 0) * p.row_floats);
#pragma unroll
          for (int v = 0; v < VPL; ++v) {
            const int col = g.lane + v * G;
            val[u][v] = (ok && col < ncol) ? __ldcg(src + col) : f4_zero();
          }
        }
#pragma unroll
        for (int u = 0; u < K; ++u) {
          if (t0 + u >= cnt) break;
          const int ob = g.bcast(out, (t0 + u) % G);
          if (p.pooled) {
            float4* o = reinterpret_cast<float4*>(p.pooled + (int64_t)ob * D);
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
              const int col = g.lane + v * G;
              if (col < ncol) __stcs(o + col, val[u][v]);
            }
          }
          if (p.unpooled) {
            float4* o = reinterpret_cast<float4*>(p.unpooled + (int64_t)(p0 + s + t0 + u) * D);
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
              const int col = g.lane + v * G;
              if (col < ncol) __stcs(o + col, val[u][v]);
            }
          }
        }
      }
    }
    pdl_trigger();
    return;
  }

  // The bag walk, one sub-block of G positions at a time (one per lane,
  // resolved one sub-block ahead): the positions' gradient sources are
  // written by their own lanes, and `ends` marks the positions after which
  // the running sum is flushed -- the last position of a bag, or of the
  // chunk.  The sub-block's rows are copied into shared memory by cp.async,
  // PR rows per lane at once (one round trip), while the sub-block after the
  // next one is resolved; then they are added in position order.
  // Bags of at most C/2 occurrences are never cut: the chunk walks from the
  // first bag that starts in it to the end of the last one that starts in
  // it (a bag crossing the chunk's start belongs to the chunk before);
  // longer bags are cut at chunk ends and combined from partials.  (Whole
  // bags of up to 2C made the chunks' work too uneven: slower on bags of 1
  // to 100 occurrences.)
  const int lcap = C / 2;
  int q0 = p0, q1 = p1;
  {
    const int hi0 = (int)p.offs[j0 + 1];
    if (cur_start < p0 && hi0 - cur_start <= lcap) q0 = hi0;
    if (p1 < N) {
      int j1 = p.chunk_bag[chunk + 1];
      if (j1 < 0 || j1 >= nbags) j1 = 0;  // only with malformed offsets (reported above)
      const int lo1 = (int)p.offs[j1], hi1 = (int)p.offs[j1 + 1];
      if (lo1 < p1 && hi1 - lo1 <= lcap && hi1 <= N) q1 = hi1;
    }
  }
  if (q0 >= q1) {
    pdl_trigger();
    return;
  }
  lim = q1;
  auto flush_bag = [&](int j, int lo, int hi) {
    if (!(lo >= 0 && lo < hi && hi <= N)) {  // malformed bag offsets
      if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
    } else if (lo >= q0 && hi <= q1) {
      store_bag(j, hi - lo);
    } else if (combine_split<G, VPL>(g, acc, p.partials, p.counters, j, chunk, lo <= p0, lo, hi, C,
                                     ncol)) {
      store_bag(j, hi - lo);
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  };
  auto emit = [&](int sub, const Ids& ids, const Bag& bg) {
    const int q = sub + g.lane;
    if (q < q1) {
      const int f = div_b(p, bg.j);
      const int4 src = make_int4((bg.j - f * B) * F + f, bg.hi - bg.lo, q, 0);
      p.gsrc[ids.spos] = src;
      p.gfirst[ids.seg] = src;
    }
    return g.ballot(q < q1 && (q + 1 == bg.hi || q + 1 == q1));
  };
  constexpr int PR = pool_piece<G, VPL>();  // rows per lane staged at once
  float4* stage = s_ring + (size_t)(threadIdx.x / G) * PR * VPL * G;
  __shared__ uint64_t s_mbar[256];  // TMA: one transaction barrier per group
  uint64_t* mbar = s_mbar + threadIdx.x / G;
  unsigned phase = 0;
  const unsigned row_bytes = (unsigned)ncol * 16u;
  if (TMA) {
    if (g.lane == 0) mbar_init(mbar, 1);
    __syncwarp(g.mask);
  }
  Ids cur_ids = (q0 == p0 && q1 == p1) ? ids0 : resolve(q0), nxt_ids = resolve(q0 + G);
  Bag cur_bag = bag_at(q0), nxt_bag = bag_at(q0 + G);
  for (int sub = q0; sub < q1; sub += G) {
    const unsigned ends = emit(sub, cur_ids, cur_bag);
    const unsigned has_row = g.ballot(cur_ids.row >= 0);
    const int cnt = q1 - sub < G ? q1 - sub : G;
    Ids nn_ids{-1, 0, 0};
    Bag nn_bag{0, 0, 0};
    for (int r0 = 0; r0 < cnt; r0 += PR) {
      const int pc = cnt - r0 < PR ? cnt - r0 : PR;
      unsigned nrows = 0;
      if (TMA) {
        // each lane copies its own position's row, one bulk copy
        const bool mine = g.lane >= r0 && g.lane < r0 + pc && cur_ids.row >= 0;
        nrows = (unsigned)__popc(g.ballot(mine));
        if (nrows) {
          __syncwarp(g.mask);  // the group has read the previous piece
          fence_async_smem();
          if (g.lane == 0) mbar_arrive_expect(mbar, nrows * row_bytes);
          if (mine)
            bulk_row(stage + (g.lane - r0) * VPL * G, p.row_data + (int64_t)cur_ids.row * p.row_floats, row_bytes,
                     mbar);
        }
      } else {
        for (int u = 0; u < pc; ++u) {
          const int row = g.bcast(cur_ids.row, r0 + u);
          if (row >= 0) {
            const float4* src = reinterpret_cast<const float4*>(p.row_data + (int64_t)row * p.row_floats);
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
              const int col = g.lane + v * G;
              if (col < ncol) cp_async16(stage + (u * VPL + v) * G + g.lane, src + col);
            }
          }
        }
        cp_async_commit();
      }
      if (r0 == 0) {  // the sub-block after the next one, while the rows are in flight
        nn_ids = resolve(sub + 2 * G);
        nn_bag = bag_at(sub + 2 * G);
      }
      if (!TMA) {
        cp_async_wait<0>();
      } else if (nrows) {
        if (!mbar_wait(mbar, phase, p.spin_max)) {
          // the copies did not land in time: reported, and waited for once
          // more before the slots are read or written again
          if (g.lane == 0) raise_error(p.st, p.mirror, kErrTimeout);
          mbar_wait(mbar, phase, p.spin_max);
        }
        phase ^= 1u;
      }
      for (int u = 0; u < pc; ++u) {
        const int t = r0 + u;
        const bool ok = (has_row >> t) & 1u;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          const int col = g.lane + v * G;
          const float4 val = (ok && col < ncol) ? stage[(u * VPL + v) * G + g.lane] : f4_zero();
          acc_add(acc[v], val);
          if (p.unpooled && col < ncol)
            __stcs(reinterpret_cast<float4*>(p.unpooled + (int64_t)(sub + t) * D) + col, val);
        }
        if ((ends >> t) & 1u)
          flush_bag(g.bcast(cur_bag.j, t), g.bcast(cur_bag.lo, t), g.bcast(cur_bag.hi, t));
      }
    }
    cur_ids = nxt_ids;
    cur_bag = nxt_bag;
    nxt_ids = nn_ids;
    nxt_bag = nn_bag;
  }
  pdl_trigger();
}

template <int G, int VPL>
static cudaError_t launch_pool_t(const PoolParams& p, bool tma, cudaStream_t s) {
  const int64_t threads = p.nchunks * G;
  int64_t blocks = (threads + 255) / 256;
  if (blocks < 1) blocks = 1;
  const size_t smem = (size_t)pool_piece<G, VPL>() * VPL * 256 * sizeof(float4);
  const auto kernel = tma ? pool_kernel<G, VPL, true> : pool_kernel<G, VPL, false>;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  LaunchScope ls("gather_pool", s);
  return launch_pdl(kernel, (unsigned)blocks, 256, smem, s, p);
}

int group_lanes_for(int D) {
  const int ncol = D / 4;
  int G = 1;
  while (G < ncol && G < 32) G <<= 1;
  return G;
}

int64_t pool_chunk_for(int64_t N, int D) {
  const int G = group_lanes_for(D);
  // enough groups for about one wave of the kernel's resident threads (3, 2
  // or 1 CTAs of 256 per SM by row width, as its launch bounds say), so each
  // group walks as long a chunk as that allows
  const int ncol = D / 4;
  const int vpl = ncol <= 32 ? 1 : (ncol <= 64 ? 2 : 4);
  const int64_t resident = (int64_t)kSMs * 256 * (vpl == 1 ? 3 : (vpl == 2 ? 2 : 1));
  int64_t C = 8;
  while (C < 256 && (N / (C * 2)) * G >= resident) C *= 2;
  return C;
}

static PoolParams pool_params(const LookupArgs& a, int64_t chunk) {
  recis_table* t = a.t;
  recis_batch* b = a.b;
  PoolParams p;
  p.N = a.N;
  p.nbags = (int64_t)a.F * a.B;
  p.B = a.B;
  p.F = a.F;
  p.ncol = t->D / 4;
  p.C = chunk;
  p.nchunks = (a.N + chunk - 1) / chunk;
  p.mean = a.combiner == RECIS_MEAN;
  p.row_floats = t->row_floats;
  p.offs = a.bag_offsets;
  p.inv = b->inv;
  p.rows = b->rows;
  p.row_data = reinterpret_cast<const float*>(t->rows.va);
  p.pooled = a.pooled_out;
  p.unpooled = a.unpooled_out;
  p.spos = b->spos;
  p.pocc = a.N <= kSampleSortMaxN ? reinterpret_cast<const int64_t*>(b->kbuf[1]) : nullptr;
  p.gsrc = b->gsrc;
  p.gfirst = b->gfirst;
  p.chunk_bag = b->chunk_bag;
  p.bag_of = b->bag_of;
  p.partials = b->partials;
  p.counters = b->bag_counter;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  p.spin_max = spin_limit();
  // ceil(2^64 / B) = floor((2^64 - 1) / B) + 1 (B >= 2; 2^64 itself for B = 1)
  p.b_magic = a.B >= 2 ? ~0ULL / (uint64_t)a.B + 1 : 0;
  return p;
}

cudaError_t launch_bag_prep(const LookupArgs& a, int64_t chunk, cudaStream_t s) {
  const PoolParams p = pool_params(a, chunk);
  if (p.nbags == 0) return cudaSuccess;
  int64_t blocks = (p.nbags + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  LaunchScope ls("bag_prep", s);
  bag_prep_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_pool(const LookupArgs& a, int64_t chunk, cudaStream_t s) {
  const PoolParams p = pool_params(a, chunk);
  if (p.nchunks == 0) return cudaSuccess;
  const int ncol = p.ncol;
  const bool tma = a.t->rows.host_numa < 0;  // EmbeddingBlocks in device memory
  if (ncol <= 1) return launch_pool_t<1, 1>(p, tma, s);
  if (ncol <= 2) return launch_pool_t<2, 1>(p, tma, s);
  if (ncol <= 4) return launch_pool_t<4, 1>(p, tma, s);
  if (ncol <= 8) return launch_pool_t<8, 1>(p, tma, s);
  if (ncol <= 16) return launch_pool_t<16, 1>(p, tma, s);
  if (ncol <= 32) return launch_pool_t<32, 1>(p, tma, s);
  if (ncol <= 64) return launch_pool_t<32, 2>(p, tma, s);
  if (ncol <= 128) return launch_pool_t<32, 4>(p, tma, s);
  return launch_pool_t<32, 8>(p, tma, s);
}

}  // namespace recis
