// pool.cu -- forward gather + bag pooling from the EmbeddingBlocks (RecIS
// README, Key optimisations > Efficient dynamic embedding: rows are read at the
// offsets the IDMap returned; > Operator implementation: vectorised memory
// access).
//
// Bags are contiguous ranges of occurrences, so the forward is a segmented
// reduction over occurrence order (segreduce.cuh): a group of G lanes owns a
// chunk of C occurrences, each lane one 16-byte column of the row.  Rows
// stream through a ring of R slots per lane in shared memory (cp.async), so R
// row loads per lane are in flight while the group adds.  The bag of the
// chunk's first occurrence comes from the bag preparation; later bag
// boundaries come from a window of G bag ends held one per lane.  A chunk
// whose bags all hold one occurrence (one-hot features) is a plain gather.
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
  double* partials;
  int32_t* counters;     // [nbags]
  DevState* st;
  HostMirror* mirror;
};

// Bag preparation, one thread per bag (runs beside the dedup on a side
// stream): checks the offsets, writes the bag of every chunk's first
// occurrence, and zeroes the pooled output of empty bags.
__global__ void __launch_bounds__(256) bag_prep_kernel(const __grid_constant__ PoolParams p) {
  const int64_t D = (int64_t)p.ncol * 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (blockIdx.x == 0 && threadIdx.x == 0 &&
      (p.offs[0] != 0 || p.offs[p.nbags] != p.N))
    raise_error(p.st, p.mirror, kErrBadOffsets);
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < p.nbags; j += stride) {
    const int64_t lo = p.offs[j], hi = p.offs[j + 1];
    if (lo < 0 || hi < lo || hi > p.N) {
      raise_error(p.st, p.mirror, kErrBadOffsets);
      continue;
    }
    if (hi == lo) {
      if (p.pooled) {
        const int64_t f = j / p.B, b = j - f * p.B;
        float4* o = reinterpret_cast<float4*>(p.pooled + (b * p.F + f) * D);
        for (int c = 0; c < p.ncol; ++c) o[c] = f4_zero();
      }
      continue;
    }
    for (int64_t c = (lo + p.C - 1) / p.C; c * p.C < hi; ++c) p.chunk_bag[c] = (int32_t)j;
  }
}

// depth of the row ring: up to 8 rows, at most one sub-block (G) ahead
template <int G, int VPL>
__host__ __device__ constexpr int pool_ring() {
  return (VPL >= 4 ? 2 : (VPL == 2 ? 4 : 8)) < G ? (VPL >= 4 ? 2 : (VPL == 2 ? 4 : 8)) : G;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int G, int VPL>
__global__ void __launch_bounds__(256, VPL == 1 ? 3 : (VPL == 2 ? 2 : 1))
    pool_kernel(const __grid_constant__ PoolParams p) {
  pdl_wait();
  constexpr int R = pool_ring<G, VPL>();  // rows in flight per group
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
  auto resolve = [&](int sub) {
    Ids r{-1, 0, 0};
    const int q = sub + g.lane;
    if (q < p1) {
      r.seg = __ldg(p.inv + q);
      r.spos = (int)__ldg(p.spos + q);
      const int64_t pr = p.pocc ? __ldcg(p.pocc + q) : -2;
      r.row = pr >= 0 ? (int)pr : (int)__ldg(p.rows + r.seg);
    }
    return r;
  };
  // the ids of the first sub-block are in flight while the bag walk starts
  const Ids ids0 = resolve(p0);

  // bag containing p0 (precomputed), its start, and a window of G bag ends
  int j0 = p.chunk_bag[chunk];
  if (j0 < 0 || j0 >= nbags) {  // only with malformed offsets
    if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
    j0 = 0;
  }
  int cur = j0;
  int cf = cur / B, cb = cur - cf * B;  // feature and sample of the current bag
  int cur_start = (int)p.offs[j0];
  int wbase = j0;
  int wend = (wbase + g.lane < nbags) ? (int)p.offs[wbase + g.lane + 1] : INT_MAX;
  int cur_end = g.bcast(wend, 0);

  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  bool has = false;

  auto epilogue = [&]() {
    if (!p.pooled) return;
    float4* o = reinterpret_cast<float4*>(p.pooled + (int64_t)(cb * F + cf) * D);
    const double dlen = (double)(cur_end - cur_start);
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
  auto flush = [&]() {
    if (!has) return;
    if (!(cur_start >= 0 && cur_start < cur_end && cur_end <= N)) {  // malformed bag offsets
      if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
    } else if (cur_start >= p0 && cur_end <= p1) {
      epilogue();
    } else if (combine_split<G, VPL>(g, acc, p.partials, p.counters, cur, chunk, cur == j0,
                                     cur_start, cur_end, C, ncol)) {
      epilogue();
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
    has = false;
  };

  // rows stream through a ring of R slots per lane in shared memory: row t+R
  // is in flight (cp.async) while row t is added
  extern __shared__ float4 s_ring[];  // [R][VPL][blockDim]
  auto slot = [&](int r, int v) -> float4* {
    return s_ring + ((r * VPL + v) * (int)blockDim.x + (int)threadIdx.x);
  };
  auto issue = [&](int t, int row) {
    if (row >= 0) {
      const float4* src = reinterpret_cast<const float4*>(p.row_data + (int64_t)row * p.row_floats);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (col < ncol) cp_async16(slot(t % R, v), src + col);
      }
    }
    cp_async_commit();
  };
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
        const int f = j / B;
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

  Ids cur_ids = ids0, nxt_ids = resolve(p0 + G);
#pragma unroll
  for (int t = 0; t < R; ++t) issue(t, t < m ? g.bcast(cur_ids.row, t) : -1);
  for (int t = 0; t < m; ++t) {
    const int pos = p0 + t;
    const int ln = t % G;
    const int row = g.bcast(cur_ids.row, ln);
    const int spos = g.bcast(cur_ids.spos, ln);
    const int seg = g.bcast(cur_ids.seg, ln);
    cp_async_wait<R - 1>();
    float4 val[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      val[v] = (row >= 0 && col < ncol) ? *slot(t % R, v) : f4_zero();
    }
    // the row R positions ahead (in this sub-block or the next) into the slot just read
    const int ta = t + R;
    int arow = -1;
    if (ta < m) arow = (ta / G == t / G) ? g.bcast(cur_ids.row, ta % G) : g.bcast(nxt_ids.row, ta % G);
    issue(ta, arow);
    while (pos >= cur_end) {  // leave the current bag (and any empty ones)
      flush();
      if (cur + 1 >= nbags) {  // only reachable with malformed bag offsets
        if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
        cur_end = INT_MAX;
        break;
      }
      ++cur;
      if (++cb == B) {
        cb = 0;
        ++cf;
      }
      cur_start = cur_end;
      if (cur - wbase >= G) {
        wbase = cur;
        wend = (wbase + g.lane < nbags) ? (int)p.offs[wbase + g.lane + 1] : INT_MAX;
      }
      cur_end = g.bcast(wend, cur - wbase);
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc_add(acc[v], val[v]);
    has = true;
    if (p.unpooled) {
      float4* dst = reinterpret_cast<float4*>(p.unpooled + (int64_t)pos * D);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        if (col < ncol) __stcs(dst + col, val[v]);
      }
    }
    // for the backward: this occurrence's gradient source, by sorted
    // position and by unique key
    if (g.lane == 0) {
      const int4 src = make_int4(cb * F + cf, cur_end - cur_start, pos, 0);
      p.gsrc[spos] = src;
      p.gfirst[seg] = src;
    }
    if (ln == G - 1) {  // next sub-block
      cur_ids = nxt_ids;
      nxt_ids = resolve(p0 + t + 1 + G);
    }
  }
  flush();
  pdl_trigger();
}

template <int G, int VPL>
static cudaError_t launch_pool_t(const PoolParams& p, cudaStream_t s) {
  const int64_t threads = p.nchunks * G;
  int64_t blocks = (threads + 255) / 256;
  if (blocks < 1) blocks = 1;
  const size_t smem = (size_t)pool_ring<G, VPL>() * VPL * 256 * sizeof(float4);
  const cudaError_t e =
      cudaFuncSetAttribute(pool_kernel<G, VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  LaunchScope ls("gather_pool", s);
  return launch_pdl(pool_kernel<G, VPL>, (unsigned)blocks, 256, smem, s, p);
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
  p.partials = b->partials;
  p.counters = b->bag_counter;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
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
  if (ncol <= 1) return launch_pool_t<1, 1>(p, s);
  if (ncol <= 2) return launch_pool_t<2, 1>(p, s);
  if (ncol <= 4) return launch_pool_t<4, 1>(p, s);
  if (ncol <= 8) return launch_pool_t<8, 1>(p, s);
  if (ncol <= 16) return launch_pool_t<16, 1>(p, s);
  if (ncol <= 32) return launch_pool_t<32, 1>(p, s);
  if (ncol <= 64) return launch_pool_t<32, 2>(p, s);
  if (ncol <= 128) return launch_pool_t<32, 4>(p, s);
  return launch_pool_t<32, 8>(p, s);
}

}  // namespace recis
