// rows.cu -- row-level access to the EmbeddingBlocks by row offset (RecIS
// README, Key optimisations > Efficient dynamic embedding: the second-level
// store holds the embedding parameters and the optimiser state of each ID
// side by side).
//
// recis_table_read_rows gathers chosen rows -- their key, emb and optimiser
// state -- into caller device buffers, one 16-byte column per thread, so a
// caller can inspect or save part of a table that is too large to export.
#include "internal.h"

namespace recis {

namespace {

// One thread per 16-byte column of the output rows; column c of row i is
// thread i * cols + c, cols = row_floats / 4 (emb columns first, then state).
__global__ void __launch_bounds__(256) read_rows_kernel(const float* __restrict__ row_data,
                                                        const int64_t* __restrict__ row_keys,
                                                        int64_t live, int row_floats, int D,
                                                        const int64_t* __restrict__ rows, int64_t n,
                                                        int64_t* keys_out, float* emb_out,
                                                        float* state_out) {
  const int cols = row_floats >> 2, dcols = D >> 2;
  const int64_t total = n * cols;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
    const int64_t i = t / cols;
    const int c = (int)(t - i * cols);
    const int64_t r = __ldg(rows + i);
    const bool ok = r >= 0 && r < live;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok) v = __ldcg(reinterpret_cast<const float4*>(row_data + r * (int64_t)row_floats) + c);
    if (c < dcols) {
      if (emb_out) reinterpret_cast<float4*>(emb_out + i * (int64_t)D)[c] = v;
    } else if (state_out) {
      reinterpret_cast<float4*>(state_out + i * (int64_t)(row_floats - D))[c - dcols] = v;
    }
    if (c == 0 && keys_out) keys_out[i] = ok ? __ldcg(row_keys + r) : kEmptyKey;
  }
}

}  // namespace

}  // namespace recis

using namespace recis;

extern "C" recis_status recis_table_read_rows(recis_table_t t, const int64_t* rows, int64_t n,
                                              int64_t* keys_out, float* emb_out, float* state_out,
                                              recis_stream_t stream) {
  if (!t || n < 0 || (n > 0 && !rows)) {
    set_error("read_rows: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  if (misaligned(rows, 8) || misaligned(keys_out, 8) || misaligned(emb_out, 16) || misaligned(state_out, 16)) {
    set_error("read_rows: misaligned array (int64 arrays 8-byte, float rows 16-byte)");
    return RECIS_ERR_INVALID_ARG;
  }
  if (n == 0 || (!keys_out && !emb_out && !state_out)) return RECIS_OK;
  cudaStream_t s = (cudaStream_t)stream;
  // rows at or past the live count read as key -1 and zeros; the live count
  // is exact once the table's earlier work has finished
  int64_t live = 0;  // rows in use (a freed row reads as key -1)
  recis_status st = table_counts(t, s, &live, nullptr);
  if (st != RECIS_OK) return st;
  const int64_t total = n * (t->row_floats / 4);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  LaunchScope ls("read_rows", s);
  read_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      reinterpret_cast<const float*>(t->rows.va), reinterpret_cast<const int64_t*>(t->keys.va),
      live, t->row_floats, t->D, rows, n, keys_out, emb_out, state_out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "read_rows launch");
  return RECIS_OK;
}
