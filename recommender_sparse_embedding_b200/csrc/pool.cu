// pool.cu -- forward gather + bag pooling from the EmbeddingBlocks (RecIS
// README, Key optimisations > Efficient dynamic embedding: rows are read at the
// offsets the IDMap returned; > Operator implementation: vectorised memory
// access).
//
// Bags are contiguous ranges of occurrences, so the forward is a segmented
// reduction over occurrence order (segreduce.cuh): a group of G lanes owns a
// chunk of C occurrences, each lane one 16-byte column of the row.  Per batch
// of K occurrences the group issues the index loads (inverse index, then row
// offset) and then all K row loads before it accumulates, so every lane keeps
// K independent 16-byte loads in flight.  The bag of the chunk's first
// occurrence is found by a G-ary search over the bag offsets; later bag
// boundaries come from a window of G bag ends held one per lane.
// Outputs: pooled rows [B][F][D] (sum, or mean = sum / length), optional
// unpooled rows [N][D], and the bag of every occurrence for the backward.
// Empty bags are written as zeros by a grid-stride prologue.
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
  int32_t* occ_bag;      // [N]
  double* partials;
  int32_t* counters;     // [nbags]
  DevState* st;
  HostMirror* mirror;
};

template <int G, int VPL>
__global__ void __launch_bounds__(256) pool_kernel(const __grid_constant__ PoolParams p) {
  constexpr int K = VPL >= 8 ? 1 : 8 / VPL;
  const int64_t D = (int64_t)p.ncol * 4;
  // prologue: zero the output of empty bags
  if (p.pooled) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < p.nbags; j += stride) {
      if (p.offs[j] == p.offs[j + 1]) {
        const int64_t f = j / p.B, b = j - f * p.B;
        float4* o = reinterpret_cast<float4*>(p.pooled + (b * p.F + f) * D);
        for (int c = 0; c < p.ncol; ++c) o[c] = f4_zero();
      }
    }
  }
  const GroupCtx<G> g;
  const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (chunk >= p.nchunks) return;
  const int64_t p0 = chunk * p.C;
  const int64_t p1 = p0 + p.C < p.N ? p0 + p.C : p.N;

  // bag containing p0: last j with offs[j] <= p0 (offs[nbags] = N > p0)
  int64_t lo = 0, hi = p.nbags;
  while (hi - lo > 1) {
    const int64_t span = hi - lo;
    const int64_t piv = lo + ((int64_t)(g.lane + 1) * span) / (G + 1);
    const bool pr = p.offs[piv] <= p0;
    const int cnt = __popc(g.ballot(pr));
    const int64_t nlo = cnt > 0 ? g.bcast(piv, cnt - 1) : lo;
    const int64_t nhi = cnt < G ? g.bcast(piv, cnt < G ? cnt : 0) : hi;
    lo = nlo;
    hi = nhi;
  }
  const int64_t j0 = lo;
  int64_t cur = j0;
  int64_t cur_start = p.offs[j0];
  // window: lane l holds the end of bag wbase + l
  int64_t wbase = j0;
  int64_t wend = (wbase + g.lane < p.nbags) ? p.offs[wbase + g.lane + 1] : INT64_MAX;
  int64_t cur_end = g.bcast(wend, 0);

  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  bool has = false;

  auto epilogue = [&](int64_t bag, int64_t len) {
    if (!p.pooled) return;
    const int64_t f = bag / p.B, b = bag - f * p.B;
    float4* o = reinterpret_cast<float4*>(p.pooled + (b * p.F + f) * D);
    const double dlen = (double)len;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int col = g.lane + v * G;
      if (col < p.ncol) {
        Acc4 r = acc[v];
        if (p.mean) {
          r.x /= dlen;
          r.y /= dlen;
          r.z /= dlen;
          r.w /= dlen;
        }
        o[col] = acc_round(r);
      }
    }
  };
  auto flush = [&]() {
    if (!has) return;
    if (!(cur_start >= 0 && cur_start < cur_end && cur_end <= p.N)) {  // malformed bag offsets
      if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
      has = false;
      return;
    }
    const bool complete = cur_start >= p0 && cur_end <= p1;
    if (complete) {
      epilogue(cur, cur_end - cur_start);
    } else if (combine_split<G, VPL>(g, acc, p.partials, p.counters, cur, chunk, cur == j0,
                                     cur_start, cur_end, p.C, p.ncol)) {
      epilogue(cur, cur_end - cur_start);
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
    has = false;
  };

  for (int64_t pb = p0; pb < p1; pb += K) {
    int64_t r[K];
#pragma unroll
    for (int k = 0; k < K; ++k) r[k] = (pb + k < p1) ? (int64_t)p.inv[pb + k] : -1;
#pragma unroll
    for (int k = 0; k < K; ++k) r[k] = r[k] >= 0 ? p.rows[r[k]] : -1;
    float4 val[K][VPL];
#pragma unroll
    for (int k = 0; k < K; ++k) {
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        val[k][v] = (r[k] >= 0 && col < p.ncol)
                        ? __ldg(reinterpret_cast<const float4*>(p.row_data + r[k] * p.row_floats) + col)
                        : f4_zero();
      }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int64_t pos = pb + k;
      if (pos >= p1) break;
      while (pos >= cur_end) {  // leave the current bag (and any empty ones)
        flush();
        if (cur + 1 >= p.nbags) {  // only reachable with malformed bag offsets
          if (g.lane == 0) raise_error(p.st, p.mirror, kErrBadOffsets);
          cur_end = INT64_MAX;
          break;
        }
        ++cur;
        cur_start = cur_end;
        if (cur - wbase >= G) {
          wbase = cur;
          wend = (wbase + g.lane < p.nbags) ? p.offs[wbase + g.lane + 1] : INT64_MAX;
        }
        cur_end = g.bcast(wend, (int)(cur - wbase));
      }
#pragma unroll
      for (int v = 0; v < VPL; ++v) acc_add(acc[v], val[k][v]);
      has = true;
      if (p.unpooled) {
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          const int col = g.lane + v * G;
          if (col < p.ncol) __stcs(reinterpret_cast<float4*>(p.unpooled + pos * D) + col, val[k][v]);
        }
      }
      if (g.lane == 0) p.occ_bag[pos] = (int32_t)cur;
    }
  }
  flush();
}

template <int G, int VPL>
static cudaError_t launch_pool_t(const PoolParams& p, cudaStream_t s) {
  const int64_t threads = p.nchunks * G;
  int64_t blocks = (threads + 255) / 256;
  if (blocks < 1) blocks = 1;
  LaunchScope ls("gather_pool", s);
  pool_kernel<G, VPL><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

int group_lanes_for(int D) {
  const int ncol = D / 4;
  int G = 1;
  while (G < ncol && G < 32) G <<= 1;
  return G;
}

int64_t pool_chunk_for(int64_t N, int D) {
  const int G = group_lanes_for(D);
  // enough groups for about one full wave of 148 SMs x 2048 threads
  int64_t C = 8;
  while (C < 256 && (N / (C * 2)) * G >= (int64_t)kSMs * 2048) C *= 2;
  return C;
}

cudaError_t launch_pool(const LookupArgs& a, int64_t chunk, cudaStream_t s) {
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
  p.occ_bag = b->occ_bag;
  p.partials = b->partials;
  p.counters = b->bag_counter;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  if (p.nchunks == 0 && !(p.pooled && p.nbags > 0)) return cudaSuccess;
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
