// update.cu -- backward: per-unique gradient reduction fused with the sparse
// optimiser row update (RecIS README, Key optimisations > Operator
// implementation: reductions merged at warp level rather than by per-element
// atomics; > Efficient dynamic embedding: optimiser state stored beside the
// parameters in the EmbeddingBlocks).
//
// The sorted positions of the dedup are already grouped by unique key, so the
// backward is a segmented reduction over sorted order (segreduce.cuh).  For
// sorted position q (occurrence i = vals[q], its bag from the forward) the term is
//   grad_pooled[b][f] * (1 or 1/length) + grad_unpooled[i];
// a group sums the terms of each unique key in its chunk in position order and
// then applies Adagrad or Adam to that key's row [emb | state] in place.  Keys
// whose occurrences cross chunk boundaries are combined by the last-arriving
// group, which also applies the update, so every touched row is updated
// exactly once.
#include "segreduce.cuh"

namespace recis {

struct UpdateParams {
  int64_t N;
  int64_t B;
  int32_t F;
  int32_t ncol;
  int64_t C;
  int64_t nchunks;
  int32_t mean;
  int32_t row_floats;
  const uint32_t* vals;     // sorted occurrence indices
  const int32_t* seg_of;    // [N] sorted position -> unique index
  const int32_t* seg_start; // [U+1]
  const int2* occ_info;     // [N] {gradient row, bag length}
  const int64_t* offs;      // bag offsets
  const int64_t* rows;      // [U]
  const float* gp;          // grad_pooled [B][F][D] or null
  const float* gu;          // grad_unpooled [N][D] or null
  float* row_data;
  double* partials;
  int32_t* counters;        // [U]
  // optimiser
  float lr;        // Adagrad: lr; Adam: lr / (1 - beta1^t)
  float eps;
  float beta1, beta2;
  float omb1, omb2;  // 1 - beta1, 1 - beta2 (formed in double, rounded once)
  float sqrt_bc2;  // Adam: sqrt(1 - beta2^t)
};

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
      r.w[v] = __ldcg(reinterpret_cast<const float4*>(base) + col);
      r.s1[v] = __ldcg(reinterpret_cast<const float4*>(base + D) + col);
      if (ADAM) r.s2[v] = __ldcg(reinterpret_cast<const float4*>(base + 2 * D) + col);
    }
  }
}

template <int G, int VPL, bool ADAM>
__device__ __forceinline__ void apply_update(const GroupCtx<G>& g, const UpdateParams& p,
                                             int64_t row, const RowRegs<VPL, ADAM>& r,
                                             const Acc4 (&grad)[VPL]) {
  if (row < 0) return;
  float* base = p.row_data + row * p.row_floats;
  const int D = p.ncol * 4;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col >= p.ncol) continue;
    const float gg[4] = {(float)grad[v].x, (float)grad[v].y, (float)grad[v].z, (float)grad[v].w};
    float ww[4] = {r.w[v].x, r.w[v].y, r.w[v].z, r.w[v].w};
    float a1[4] = {r.s1[v].x, r.s1[v].y, r.s1[v].z, r.s1[v].w};
    if (!ADAM) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float acc = a1[e] + gg[e] * gg[e];
        ww[e] = ww[e] - p.lr * gg[e] / (sqrtf(acc) + p.eps);
        a1[e] = acc;
      }
    } else {
      float a2[4] = {r.s2[v].x, r.s2[v].y, r.s2[v].z, r.s2[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = p.beta1 * a1[e] + p.omb1 * gg[e];
        const float vv = p.beta2 * a2[e] + p.omb2 * (gg[e] * gg[e]);
        ww[e] = ww[e] - p.lr * m / (sqrtf(vv) / p.sqrt_bc2 + p.eps);
        a1[e] = m;
        a2[e] = vv;
      }
      __stcg(reinterpret_cast<float4*>(base + 2 * D) + col, make_float4(a2[0], a2[1], a2[2], a2[3]));
    }
    __stcg(reinterpret_cast<float4*>(base + D) + col, make_float4(a1[0], a1[1], a1[2], a1[3]));
    __stcg(reinterpret_cast<float4*>(base) + col, make_float4(ww[0], ww[1], ww[2], ww[3]));
  }
}

// One group per chunk of C sorted positions.  Index work is lane-parallel:
// for G positions at a time each lane resolves one position (sorted position
// -> occurrence -> bag -> gradient row), then the group streams the gradient
// rows RB at a time, every lane loading its 16-byte column of each.  The
// chunk's unique keys are consecutive segment ids s0..s_last; their row
// offsets are fetched one per lane, and the row of the next key is loaded
// while the current key's terms are summed, so the epilogue rarely waits.
template <int G, int VPL, bool ADAM>
__global__ void __launch_bounds__(256, VPL == 1 ? 3 : (VPL == 2 ? 2 : 1))
    update_kernel(const __grid_constant__ UpdateParams p) {
  constexpr int RB = VPL >= 2 ? 1 : 2;  // gradient rows in flight per lane
  const GroupCtx<G> g;
  const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (chunk >= p.nchunks) return;
  const int64_t D = (int64_t)p.ncol * 4;
  const uint32_t* vals = p.vals;
  const int64_t p0 = chunk * p.C;
  const int64_t p1 = p0 + p.C < p.N ? p0 + p.C : p.N;
  const int32_t s0 = __ldg(p.seg_of + p0);
  const int32_t s_last = __ldg(p.seg_of + p1 - 1);
  const bool s0_starts_here = __ldg(p.seg_start + s0) == p0;
  const int32_t after = p1 < p.N ? __ldg(p.seg_of + p1) : -1;
  int32_t wbase = s0;
  int64_t wrow = (s0 + g.lane <= s_last) ? __ldg(p.rows + s0 + g.lane) : -1;

  int32_t cur = s0;
  bool cur_starts_here = s0_starts_here;
  int64_t cur_row = g.bcast(wrow, 0);
  RowRegs<VPL, ADAM> rcur, rnext;
  load_row<G, VPL, ADAM>(g, p, cur_row, rcur);
  int64_t next_row = -1;
  auto fetch_next = [&]() {  // row of cur + 1, if it belongs to this chunk
    next_row = -1;
    if (cur + 1 <= s_last) {
      if (cur + 1 - wbase >= G) {
        wbase = cur + 1;
        wrow = (wbase + g.lane <= s_last) ? __ldg(p.rows + wbase + g.lane) : -1;
      }
      next_row = g.bcast(wrow, cur + 1 - wbase);
      load_row<G, VPL, ADAM>(g, p, next_row, rnext);
    }
  };
  fetch_next();

  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();

  auto finish = [&](bool ends_here) {
    if (cur_starts_here && ends_here) {
      apply_update<G, VPL, ADAM>(g, p, cur_row, rcur, acc);
    } else {
      const int64_t st = p.seg_start[cur], en = p.seg_start[cur + 1];
      if (combine_split<G, VPL>(g, acc, p.partials, p.counters, cur, chunk, cur == s0, st, en,
                                p.C, p.ncol))
        apply_update<G, VPL, ADAM>(g, p, cur_row, rcur, acc);
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  };

  for (int64_t sub = p0; sub < p1; sub += G) {
    // lane-parallel resolution of positions sub .. sub+G-1
    const int64_t q = sub + g.lane;
    const bool ok = q < p1;
    const int32_t my_seg = ok ? __ldg(p.seg_of + q) : -1;
    const int32_t my_occ = ok ? (int32_t)__ldg(vals + q) : -1;
    int32_t my_gprow = -1;
    double my_scale = 1.0;
    if (ok && p.gp) {
      const int2 oi = __ldg(p.occ_info + my_occ);
      my_gprow = oi.x;
      if (p.mean) my_scale = 1.0 / (double)oi.y;
    }
    const int m = (int)((p1 - sub) < G ? (p1 - sub) : G);
    for (int kb = 0; kb < m; kb += RB) {
      float4 tp[RB][VPL], tu[RB][VPL];
      int32_t sg[RB];
      double sc[RB];
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        const int src = kb + k < m ? kb + k : 0;
        const int32_t gr = g.bcast(my_gprow, src);
        const int32_t oc = g.bcast(my_occ, src);
        sg[k] = g.bcast(my_seg, src);
        sc[k] = p.mean ? g.bcast(my_scale, src) : 1.0;
        const bool valid = kb + k < m;
        const float4* gps = reinterpret_cast<const float4*>(p.gp + (int64_t)gr * D);
        const float4* gus = reinterpret_cast<const float4*>(p.gu + (int64_t)oc * D);
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          const int col = g.lane + v * G;
          tp[k][v] = (valid && col < p.ncol && gr >= 0) ? __ldcs(gps + col) : f4_zero();
          tu[k][v] = (valid && col < p.ncol && p.gu) ? __ldcs(gus + col) : f4_zero();
        }
      }
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        if (kb + k >= m) break;
        if (sg[k] != cur) {
          finish(true);
          cur = sg[k];
          cur_starts_here = true;
          cur_row = next_row;
          rcur = rnext;
          fetch_next();
        }
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
          acc[v].x += (double)tp[k][v].x * sc[k] + (double)tu[k][v].x;
          acc[v].y += (double)tp[k][v].y * sc[k] + (double)tu[k][v].y;
          acc[v].z += (double)tp[k][v].z * sc[k] + (double)tu[k][v].z;
          acc[v].w += (double)tp[k][v].w * sc[k] + (double)tu[k][v].w;
        }
      }
    }
  }
  finish(after != cur);
}

template <int G, int VPL>
static cudaError_t launch_update_t(const UpdateParams& p, bool adam, cudaStream_t s) {
  const int64_t threads = p.nchunks * G;
  int64_t blocks = (threads + 255) / 256;
  if (blocks < 1) blocks = 1;
  LaunchScope ls("reduce_update", s);
  if (adam)
    update_kernel<G, VPL, true><<<(unsigned)blocks, 256, 0, s>>>(p);
  else
    update_kernel<G, VPL, false><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

int group_lanes_for(int D);

int64_t update_chunk_for(int64_t N, int D) {
  const int G = group_lanes_for(D);
  int64_t C = 8;
  while (C < 256 && (N / (C * 2)) * G >= (int64_t)kSMs * 2048) C *= 2;
  return C;
}

cudaError_t launch_update(recis_table* t, recis_batch* b, const float* grad_pooled,
                          const float* grad_unpooled, int64_t chunk, float lr_t, float sqrt_bc2,
                          cudaStream_t s) {
  UpdateParams p;
  p.N = b->N;
  p.B = b->B;
  p.F = b->F;
  p.ncol = t->D / 4;
  p.C = chunk;
  p.nchunks = (b->N + chunk - 1) / chunk;
  p.mean = b->combiner == RECIS_MEAN;
  p.row_floats = t->row_floats;
  p.vals = b->svals;
  p.seg_of = b->seg_of;
  p.seg_start = b->seg_start;
  p.occ_info = b->occ_info;
  p.offs = b->bag_offsets;
  p.rows = b->rows;
  p.gp = grad_pooled;
  p.gu = grad_unpooled;
  p.row_data = reinterpret_cast<float*>(t->rows.va);
  p.partials = b->partials;
  p.counters = b->seg_counter;
  p.lr = lr_t;
  p.eps = (float)t->cfg.eps;
  p.beta1 = (float)t->cfg.beta1;
  p.beta2 = (float)t->cfg.beta2;
  p.omb1 = (float)(1.0 - t->cfg.beta1);
  p.omb2 = (float)(1.0 - t->cfg.beta2);
  p.sqrt_bc2 = sqrt_bc2;
  if (p.nchunks == 0) return cudaSuccess;
  const bool adam = t->cfg.optimizer == RECIS_ADAM;
  const int ncol = p.ncol;
  if (ncol <= 1) return launch_update_t<1, 1>(p, adam, s);
  if (ncol <= 2) return launch_update_t<2, 1>(p, adam, s);
  if (ncol <= 4) return launch_update_t<4, 1>(p, adam, s);
  if (ncol <= 8) return launch_update_t<8, 1>(p, adam, s);
  if (ncol <= 16) return launch_update_t<16, 1>(p, adam, s);
  if (ncol <= 32) return launch_update_t<32, 1>(p, adam, s);
  if (ncol <= 64) return launch_update_t<32, 2>(p, adam, s);
  if (ncol <= 128) return launch_update_t<32, 4>(p, adam, s);
  return launch_update_t<32, 8>(p, adam, s);
}

}  // namespace recis
