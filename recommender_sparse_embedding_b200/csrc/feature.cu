// feature.cu -- fused feature transform (RecIS README, Core architecture >
// Feature Engine: Hash / Mod / Bucketize, with automatic operator fusion).
//
// One launch transforms up to kFeatPerLaunch features: every value finds its
// feature by a binary search over the offsets held in the kernel's parameter
// space, then applies bucketize (of int64 or, with RECIS_FLOAT, of float64
// values) or hash -> mod, then the feature tag.  The
// kernel streams 16 bytes per value (8 in, 8 out), four values per thread
// in flight.
#include "internal.h"

namespace recis {

constexpr int kFeatPerLaunch = 128;

struct FeatOpDev {
  uint32_t flags;
  int32_t n_bound;
  uint64_t seed;
  uint64_t mod;        // modulus, or mask + 1 when pow2
  uint64_t tag_bits;   // tag << shift
  uint64_t limit;      // 2^shift
  const int64_t* bounds;
};
constexpr uint32_t kModPow2 = 1u << 31;  // internal flag: mod is a power of two

struct FeatParams {
  int F;
  int pad;
  int64_t offs[kFeatPerLaunch + 1];
  FeatOpDev ops[kFeatPerLaunch];
};

constexpr int kFeatItems = 4;  // values per thread per round, all loaded before any is transformed

// the transform of value x of feature op
__device__ __forceinline__ int64_t feature_key(const FeatOpDev& op, int64_t x, int* status) {
  uint64_t v;
  if (op.flags & RECIS_BUCKETIZE) {
    // count of boundaries <= x: the boundaries are sorted, so the ones <= x
    // come first (a NaN x, as a double, compares below none of them: 0)
    const bool fl = (op.flags & RECIS_FLOAT) != 0;
    const double xd = __longlong_as_double(x);
    int l = 0, r = op.n_bound;
    while (l < r) {
      const int m = (l + r) >> 1;
      const int64_t bm = __ldg(op.bounds + m);
      if (fl ? __longlong_as_double(bm) <= xd : bm <= x) l = m + 1; else r = m;
    }
    v = (uint64_t)l;
  } else {
    v = (uint64_t)x;
    if (op.flags & RECIS_HASH) v = mix64(v ^ op.seed);
    if (op.flags & RECIS_MOD) v = (op.flags & kModPow2) ? (v & (op.mod - 1)) : (v % op.mod);
  }
  if (!(op.flags & RECIS_TAG)) return (int64_t)v;
  if (v >= op.limit) {
    atomicOr(status, kErrTagOverflow);
    return kEmptyKey;
  }
  return (int64_t)(op.tag_bits | v);
}

__global__ void __launch_bounds__(256) feature_hash_kernel(const __grid_constant__ FeatParams p,
                                                           const int64_t* __restrict__ values,
                                                           int64_t* __restrict__ keys,
                                                           int* __restrict__ status) {
  pdl_wait();
  const int64_t lo = p.offs[0], hi = p.offs[p.F];
  constexpr int64_t kRound = 256 * kFeatItems;
  const int64_t stride = (int64_t)gridDim.x * kRound;
  for (int64_t base = lo + (int64_t)blockIdx.x * kRound + threadIdx.x; base < hi; base += stride) {
    int64_t x[kFeatItems];
#pragma unroll
    for (int j = 0; j < kFeatItems; ++j) {
      const int64_t i = base + j * 256;
      x[j] = i < hi ? __ldcs(values + i) : 0;
    }
#pragma unroll
    for (int j = 0; j < kFeatItems; ++j) {
      const int64_t i = base + j * 256;
      if (i >= hi) break;
      // feature of value i: last f with offs[f] <= i (and offs[f+1] > i)
      int a = 0, b = p.F;  // invariant: offs[a] <= i < offs[b]
      while (b - a > 1) {
        const int m = (a + b) >> 1;
        if (p.offs[m] <= i) a = m; else b = m;
      }
      __stcs(keys + i, feature_key(p.ops[a], x[j], status));
    }
  }
  pdl_trigger();
}

cudaError_t launch_feature_hash(const recis_feature_op* ops, int F, const int64_t* values,
                                const int64_t* feat_offsets, int64_t* keys_out, int* dev_status,
                                cudaStream_t s) {
  for (int f0 = 0; f0 < F; f0 += kFeatPerLaunch) {
    const int nf = F - f0 < kFeatPerLaunch ? F - f0 : kFeatPerLaunch;
    FeatParams p;
    p.F = nf;
    p.pad = 0;
    for (int f = 0; f <= nf; ++f) p.offs[f] = feat_offsets[f0 + f];
    for (int f = 0; f < nf; ++f) {
      const recis_feature_op& o = ops[f0 + f];
      FeatOpDev& d = p.ops[f];
      d.flags = o.flags;
      d.n_bound = o.n_bound;
      d.seed = o.hash_seed;
      d.mod = o.mod;
      if ((o.flags & RECIS_MOD) && (o.mod & (o.mod - 1)) == 0) d.flags |= kModPow2;
      d.tag_bits = (o.flags & RECIS_TAG) ? (o.tag << o.tag_shift) : 0;
      d.limit = (o.flags & RECIS_TAG) ? (1ULL << o.tag_shift) : 0;
      d.bounds = o.boundaries;
    }
    const int64_t n = p.offs[nf] - p.offs[0];
    if (n <= 0) continue;
    int64_t blocks = (n + 256 * kFeatItems - 1) / (256 * kFeatItems);
    const int64_t cap = (int64_t)kSMs * 8;
    if (blocks > cap) blocks = cap;
    LaunchScope ls("feature_hash", s);
    const cudaError_t le = launch_pdl(feature_hash_kernel, (unsigned)blocks, 256, 0, s, p, values, keys_out,
                                      dev_status);
    if (le != cudaSuccess) return le;
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace recis
