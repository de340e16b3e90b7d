// update.cu -- backward: per-unique gradient reduction fused with the sparse
// optimiser row update (RecIS README, Key optimisations > Operator
// implementation: reductions merged at warp level rather than by per-element
// atomics; > Efficient dynamic embedding: optimiser state stored beside the
// parameters in the EmbeddingBlocks).
//
// The sorted positions of the dedup are already grouped by unique key, so the
// backward is a segmented reduction over sorted order (segreduce.cuh).  For
// sorted position q (occurrence i = vals[q], bag = occ_bag[i]) the term is
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
  const int32_t* occ_bag;   // [N]
  const int64_t* offs;      // bag offsets
  const int64_t* rows;      // [U]
  const float* gp;          // grad_pooled [B][F][D] or null
  const float* gu;          // grad_unpooled [N][D] or null
  float* row_data;
  double* partials;
  int32_t* counters;        // [U]
  const SortCtl* ctl;
  const uint32_t* vb0;
  const uint32_t* vb1;
  // optimiser
  float lr;        // Adagrad: lr; Adam: lr / (1 - beta1^t)
  float eps;
  float beta1, beta2;
  float omb1, omb2;  // 1 - beta1, 1 - beta2 (formed in double, rounded once)
  float sqrt_bc2;  // Adam: sqrt(1 - beta2^t)
};

template <int G, int VPL, bool ADAM>
__device__ __forceinline__ void apply_update(const GroupCtx<G>& g, const UpdateParams& p,
                                             int64_t row, const Acc4 (&grad)[VPL]) {
  if (row < 0) return;
  float* base = p.row_data + row * p.row_floats;
  const int D = p.ncol * 4;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int col = g.lane + v * G;
    if (col >= p.ncol) continue;
    float4* wp = reinterpret_cast<float4*>(base) + col;
    float4* s1p = reinterpret_cast<float4*>(base + D) + col;
    float4 w = *wp, s1 = *s1p;
    const float gg[4] = {(float)grad[v].x, (float)grad[v].y, (float)grad[v].z, (float)grad[v].w};
    float ww[4] = {w.x, w.y, w.z, w.w};
    float a1[4] = {s1.x, s1.y, s1.z, s1.w};
    if (!ADAM) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float acc = a1[e] + gg[e] * gg[e];
        ww[e] = ww[e] - p.lr * gg[e] / (sqrtf(acc) + p.eps);
        a1[e] = acc;
      }
    } else {
      float4* s2p = reinterpret_cast<float4*>(base + 2 * D) + col;
      const float4 s2 = *s2p;
      float a2[4] = {s2.x, s2.y, s2.z, s2.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = p.beta1 * a1[e] + p.omb1 * gg[e];
        const float vv = p.beta2 * a2[e] + p.omb2 * (gg[e] * gg[e]);
        ww[e] = ww[e] - p.lr * m / (sqrtf(vv) / p.sqrt_bc2 + p.eps);
        a1[e] = m;
        a2[e] = vv;
      }
      *s2p = make_float4(a2[0], a2[1], a2[2], a2[3]);
    }
    *s1p = make_float4(a1[0], a1[1], a1[2], a1[3]);
    *wp = make_float4(ww[0], ww[1], ww[2], ww[3]);
  }
}

template <int G, int VPL, bool ADAM>
__global__ void __launch_bounds__(256) update_kernel(const __grid_constant__ UpdateParams p) {
  constexpr int K = VPL >= 4 ? 1 : 4 / VPL;
  const GroupCtx<G> g;
  const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  if (chunk >= p.nchunks) return;
  const int64_t D = (int64_t)p.ncol * 4;
  const unsigned na = p.ctl->n_active;
  const uint32_t* vals = na == 0 ? nullptr : (((na - 1) & 1) ? p.vb1 : p.vb0);
  const int64_t p0 = chunk * p.C;
  const int64_t p1 = p0 + p.C < p.N ? p0 + p.C : p.N;
  const int32_t s0 = p.seg_of[p0];
  const bool s0_starts_here = p.seg_start[s0] == p0;
  const int32_t after = p1 < p.N ? p.seg_of[p1] : -1;

  int32_t cur = s0;
  bool cur_starts_here = s0_starts_here;
  Acc4 acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();

  auto finish = [&](bool ends_here) {
    const int64_t row = p.rows[cur];
    if (cur_starts_here && ends_here) {
      apply_update<G, VPL, ADAM>(g, p, row, acc);
    } else {
      const int64_t st = p.seg_start[cur], en = p.seg_start[cur + 1];
      if (combine_split<G, VPL>(g, acc, p.partials, p.counters, cur, chunk, cur == s0, st, en,
                                p.C, p.ncol))
        apply_update<G, VPL, ADAM>(g, p, row, acc);
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = acc_zero();
  };

  for (int64_t pb = p0; pb < p1; pb += K) {
    int32_t sg[K];
    int64_t occ[K];
    double scale[K];
    int64_t gprow[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int64_t q = pb + k;
      const bool ok = q < p1;
      sg[k] = ok ? p.seg_of[q] : -1;
      occ[k] = ok ? (vals ? (int64_t)vals[q] : q) : -1;
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      scale[k] = 1.0;
      gprow[k] = -1;
      if (occ[k] >= 0 && p.gp) {
        const int64_t bag = p.occ_bag[occ[k]];
        const int64_t f = bag / p.B, b = bag - f * p.B;
        gprow[k] = b * p.F + f;
        if (p.mean) scale[k] = 1.0 / (double)(p.offs[bag + 1] - p.offs[bag]);
      }
    }
    float4 tp[K][VPL], tu[K][VPL];
#pragma unroll
    for (int k = 0; k < K; ++k) {
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int col = g.lane + v * G;
        tp[k][v] = (col < p.ncol && gprow[k] >= 0)
                       ? __ldg(reinterpret_cast<const float4*>(p.gp + gprow[k] * D) + col)
                       : f4_zero();
        tu[k][v] = (col < p.ncol && p.gu && occ[k] >= 0)
                       ? __ldg(reinterpret_cast<const float4*>(p.gu + occ[k] * D) + col)
                       : f4_zero();
      }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (pb + k >= p1) break;
      if (sg[k] != cur) {
        finish(true);
        cur = sg[k];
        cur_starts_here = true;
      }
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        acc[v].x += (double)tp[k][v].x * scale[k] + (double)tu[k][v].x;
        acc[v].y += (double)tp[k][v].y * scale[k] + (double)tu[k][v].y;
        acc[v].z += (double)tp[k][v].z * scale[k] + (double)tu[k][v].z;
        acc[v].w += (double)tp[k][v].w * scale[k] + (double)tu[k][v].w;
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
  p.vals = nullptr;
  p.seg_of = b->seg_of;
  p.seg_start = b->seg_start;
  p.occ_bag = b->occ_bag;
  p.offs = b->bag_offsets;
  p.rows = b->rows;
  p.gp = grad_pooled;
  p.gu = grad_unpooled;
  p.row_data = reinterpret_cast<float*>(t->rows.va);
  p.partials = b->partials;
  p.counters = b->seg_counter;
  p.ctl = b->ctl;
  p.vb0 = b->vbuf[0];
  p.vb1 = b->vbuf[1];
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
