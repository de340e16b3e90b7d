// samplesort.cu -- dedup + IDMap find-or-insert for batches of up to 2^19
// keys in three launches (RecIS README, Key optimisations > Distributed
// optimisation: merged requests deduplicated; > Efficient dynamic embedding:
// IDMap first-level store, EmbeddingBlocks second-level store).
//
// It produces exactly what the radix-sort path (sort.cu + unique.cu) produces
// -- unique keys ascending, inverse index, rows (new keys in ascending key
// order), segment starts, segment of each sorted position, occurrence of each
// sorted position, initialised new rows -- but replaces the eight digit
// passes by one bucket pass:
//   ss_plan     every CTA sorts the same 2048-key sample (bitonic network in
//               shared memory) and takes up to 255 distinct splitters; key k
//               goes to bucket 2r + [k == splitter r], r = #splitters < k, so
//               buckets are ordered, and a key equal to a splitter (a hot key)
//               gets a bucket of its own.  The CTAs then histogram their
//               slice of the keys; the last CTA scans the histogram.
//   ss_scatter  one stable pass moving (key, occurrence) into bucket order:
//               warp match/ballot ranking, decoupled look-back over tiles.
//   ss_local    one CTA per bucket: sorts the bucket in shared memory by
//               (key, occurrence) (an ascending-only bitonic network), finds
//               the heads, probes the IDMap, resolves its unique/new prefix by
//               look-back over buckets, writes all outputs and initialises
//               its new rows.  A bucket larger than shared memory (possible
//               only for adversarial key orders) is sorted by the same
//               network in global memory and streamed.
#include <climits>

#include "internal.h"

namespace recis {

namespace {

constexpr int kSsSample = 2048;
constexpr int kSsSplit = 255;         // at most 255 distinct splitters
constexpr int kSsDigits = 512;        // buckets 0 .. 2*nsplit (<= 510)
constexpr int kSsBlock = 256;         // scatter CTA
constexpr int kSsItems = 8;
constexpr int kSsTile = kSsBlock * kSsItems;  // 2048 keys per scatter tile
constexpr int kLocBlock = 512;        // local CTA
constexpr int kLocCap = 3072;         // bucket elements held in shared memory
constexpr int kMaxProbes = 1 << 16;
constexpr unsigned long long kAgg = 1ULL << 62, kIncl = 2ULL << 62;
constexpr unsigned kFlagAgg = 1u, kFlagIncl = 2u;

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// bucket of ukey u: 2r + [u == split[r]], r = number of splitters < u
__device__ __forceinline__ unsigned bucket_of(const uint64_t* split, int nsplit, uint64_t u) {
  int lo = 0, hi = nsplit;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (split[mid] < u) lo = mid + 1; else hi = mid;
  }
  return 2u * (unsigned)lo + ((lo < nsplit && split[lo] == u) ? 1u : 0u);
}

// Ascending bitonic network on n elements (any n): for each merge size k the
// first stage compares i with its mirror i ^ (k-1), later stages compare i
// with i ^ d; every comparator puts the smaller (key, idx) at the lower index,
// so a partner past the end behaves as +infinity and is skipped.  All threads
// of the block must call it.
template <typename KeyPtr, typename IdxPtr>
__device__ void bitonic_sort(KeyPtr key, IdxPtr idx, int n) {
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int k = 2; k <= n2; k <<= 1) {
    for (int d = k >> 1; d > 0; d >>= 1) {
      const bool mirror = d == (k >> 1);
      for (int t = threadIdx.x; t < (n2 >> 1); t += blockDim.x) {
        // t-th pair: lower index i has bit d clear
        const int i = ((t & ~(d - 1)) << 1) | (t & (d - 1));
        const int j = mirror ? (i ^ (k - 1)) : (i | d);
        if (j < n) {
          const uint64_t ki = key[i], kj = key[j];
          const uint32_t ii = idx[i], ij = idx[j];
          if (kj < ki || (kj == ki && ij < ii)) {
            key[i] = kj;
            key[j] = ki;
            idx[i] = ij;
            idx[j] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
}

// IDMap find-or-insert (the same protocol as the radix path).
__device__ __forceinline__ bool idmap_probe(Slot* slots, uint64_t mask, int64_t key,
                                            int64_t* slot, int64_t* row) {
  uint64_t h = mix64((uint64_t)key ^ kSlotSalt) & mask;
  const int64_t limit = (int64_t)mask + 1 < kMaxProbes ? (int64_t)mask + 1 : kMaxProbes;
  for (int64_t n = 0; n < limit; ++n) {
    const longlong2 sv = __ldcg(reinterpret_cast<const longlong2*>(slots + h));
    if (sv.x == key) {
      *slot = (int64_t)h;
      *row = sv.y;
      return false;
    }
    if (sv.x == kEmptyKey) {
      const unsigned long long old = atomicCAS(reinterpret_cast<unsigned long long*>(&slots[h].key),
                                               (unsigned long long)kEmptyKey,
                                               (unsigned long long)key);
      if ((int64_t)old == kEmptyKey) {
        *slot = (int64_t)h;
        *row = -1;
        return true;
      }
      if ((int64_t)old == key) {
        *slot = (int64_t)h;
        *row = __ldcg(&slots[h].row);
        return false;
      }
    }
    h = (h + 1) & mask;
  }
  *slot = -1;
  *row = -1;
  return false;
}

}  // namespace

struct SsParams {
  const int64_t* keys;
  int64_t N;
  SsCtl* ctl;
  uint64_t* kb0;
  uint32_t* vb0;
  uint64_t* kb1;            // scratch for oversized buckets
  uint32_t* vb1;
  unsigned long long* lookback;  // scatter look-back [tiles][512], epoch-tagged
  uint32_t epoch;
  // table
  Slot* slots;
  uint64_t slot_mask;
  float* row_data;
  int64_t* row_keys;
  int64_t mapped_rows;
  int row_floats;
  int D;
  int adagrad;
  float acc0;
  float two_s;
  uint64_t init_seed;
  // outputs
  int64_t* uniq;
  int64_t* rows;
  int32_t* inv;
  int32_t* seg_of;
  uint32_t* svals;
  int32_t* seg_start;
  BatchDev* bdev;
  DevState* st;
  HostMirror* mirror;
};

// ------------------------------------------------------------------ plan
__global__ void __launch_bounds__(512) ss_plan_kernel(const __grid_constant__ SsParams p) {
  __shared__ uint64_t s_samp[kSsSample];
  __shared__ uint32_t s_sidx[kSsSample];
  __shared__ uint64_t s_split[kSsSplit];
  __shared__ unsigned s_hist[kSsDigits];
  __shared__ int s_nsplit;
  __shared__ bool s_last;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int64_t N = p.N;
  for (int k = tid; k < kSsSample; k += blockDim.x) {
    const int64_t pos = (int64_t)(((unsigned long long)k * (unsigned long long)N) / kSsSample);
    s_samp[k] = to_ukey(p.keys[pos]);
    s_sidx[k] = (uint32_t)k;
  }
  for (int k = tid; k < kSsDigits; k += blockDim.x) s_hist[k] = 0;
  __syncthreads();
  bitonic_sort(s_samp, s_sidx, kSsSample);
  // candidates: every 8th sample; keep the distinct ones (warp 0 compacts)
  if (w == 0) {
    int n = 0;
    uint64_t prev = 0;
    bool have = false;
    for (int base = 0; base < kSsSplit; base += 32) {
      const int i = base + lane;
      const uint64_t c = i < kSsSplit ? s_samp[(i + 1) * (kSsSample / (kSsSplit + 1)) - 1] : 0;
      const uint64_t pc = __shfl_up_sync(0xffffffffu, c, 1);
      const bool first = i < kSsSplit && (lane == 0 ? (!have || c != prev) : c != pc);
      const unsigned bal = __ballot_sync(0xffffffffu, first);
      if (first) s_split[n + __popc(bal & ((1u << lane) - 1u))] = c;
      n += __popc(bal);
      prev = __shfl_sync(0xffffffffu, c, 31);
      have = true;
    }
    if (lane == 0) s_nsplit = n;
  }
  __syncthreads();
  const int nsplit = s_nsplit;
  if (blockIdx.x == 0) {
    for (int i = tid; i < nsplit; i += blockDim.x) p.ctl->split[i] = s_split[i];
    if (tid == 0) p.ctl->nsplit = (unsigned)nsplit;
  }
  // histogram of this CTA's slice
  bool reserved = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < N; i += stride) {
    const int64_t k = p.keys[i];
    reserved |= k == kEmptyKey;
    atomicAdd(&s_hist[bucket_of(s_split, nsplit, to_ukey(k))], 1u);
  }
  if (__any_sync(0xffffffffu, reserved) && lane == 0) raise_error(p.st, p.mirror, kErrReservedKey);
  __syncthreads();
  for (int k = tid; k < kSsDigits; k += blockDim.x)
    if (s_hist[k]) atomicAdd(&p.ctl->hist[k], s_hist[k]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&p.ctl->ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last CTA: exclusive scan of the bucket counts (warp 0, 16 per lane)
  if (w == 0) {
    unsigned c[16], run = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      c[q] = __ldcg(&p.ctl->hist[lane * 16 + q]);
      run += c[q];
    }
    unsigned x = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    unsigned b = x - run;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      p.ctl->base[lane * 16 + q] = b;
      b += c[q];
    }
    if (lane == 0) p.bdev->row_base = *(volatile unsigned long long*)&p.st->next_free;
  }
}

// ------------------------------------------------------------------ scatter
__global__ void __launch_bounds__(kSsBlock) ss_scatter_kernel(const __grid_constant__ SsParams p) {
  __shared__ uint64_t s_keys[kSsTile];
  __shared__ uint32_t s_vals[kSsTile];
  __shared__ unsigned s_whist[kSsBlock / 32][kSsDigits];
  __shared__ unsigned s_doff[kSsDigits];
  __shared__ int s_glob[kSsDigits];
  __shared__ uint64_t s_split[kSsSplit];
  __shared__ unsigned s_wsum[kSsBlock / 32];
  __shared__ unsigned s_tile;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nsplit = (int)p.ctl->nsplit;
  for (int i = tid; i < nsplit; i += kSsBlock) s_split[i] = p.ctl->split[i];
  for (int i = tid; i < (kSsBlock / 32) * kSsDigits; i += kSsBlock) (&s_whist[0][0])[i] = 0;
  if (tid == 0) s_tile = atomicAdd(&p.ctl->tile_counter, 1u);
  __syncthreads();
  const unsigned tile = s_tile;
  const int64_t tbase = (int64_t)tile * kSsTile;
  const int64_t N = p.N;

  uint64_t k[kSsItems];
  uint32_t v[kSsItems];
  unsigned d[kSsItems], rank[kSsItems];
#pragma unroll
  for (int j = 0; j < kSsItems; ++j) {
    const int64_t pos = tbase + w * (kSsItems * 32) + j * 32 + lane;
    if (pos < N) {
      k[j] = to_ukey(p.keys[pos]);
      v[j] = (uint32_t)pos;
    } else {
      k[j] = ~0ULL;
      v[j] = 0xffffffffu;
    }
  }
#pragma unroll
  for (int j = 0; j < kSsItems; ++j) {
    const int64_t pos = tbase + w * (kSsItems * 32) + j * 32 + lane;
    // padding goes to digit 511, after every real bucket
    d[j] = pos < N ? bucket_of(s_split, nsplit, k[j]) : (unsigned)(kSsDigits - 1);
  }
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kSsItems; ++j) {
    const unsigned peers = __match_any_sync(0xffffffffu, d[j]);
    const int leader = __ffs(peers) - 1;
    unsigned old = 0;
    if (lane == leader) {
      old = s_whist[w][d[j]];
      s_whist[w][d[j]] = old + __popc(peers);
    }
    old = __shfl_sync(0xffffffffu, old, leader);
    rank[j] = old + __popc(peers & lt);
    __syncwarp();
  }
  __syncthreads();
  // two digits per thread: totals over warps, prefix per warp
  unsigned total[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int dd = tid + h * kSsBlock;
    unsigned t = 0;
#pragma unroll
    for (int ww = 0; ww < kSsBlock / 32; ++ww) {
      const unsigned c = s_whist[ww][dd];
      s_whist[ww][dd] = t;
      t += c;
    }
    total[h] = t;
    unsigned long long* my = p.lookback + (size_t)tile * kSsDigits + dd;
    const unsigned long long tag = (unsigned long long)p.epoch << 32;
    st_relaxed(my, tag | ((unsigned long long)(tile == 0 ? kFlagIncl : kFlagAgg) << 30) | t);
  }
  {
    // low half: digits 0..255 in thread order
    unsigned x = total[0];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) s_wsum[w] = x;
    __syncthreads();
    unsigned pre = 0, lowsum = 0;
#pragma unroll
    for (int ww = 0; ww < kSsBlock / 32; ++ww) {
      if (ww < w) pre += s_wsum[ww];
      lowsum += s_wsum[ww];
    }
    s_doff[tid] = pre + x - total[0];
    __syncthreads();
    // high half: digits 256..511
    unsigned y2 = total[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, y2, off);
      if (lane >= off) y2 += y;
    }
    if (lane == 31) s_wsum[w] = y2;
    __syncthreads();
    unsigned pre2 = 0;
#pragma unroll
    for (int ww = 0; ww < kSsBlock / 32; ++ww)
      if (ww < w) pre2 += s_wsum[ww];
    s_doff[tid + kSsBlock] = lowsum + pre2 + y2 - total[1];
  }
  // decoupled look-back, two digits per thread
  int spins = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int dd = tid + h * kSsBlock;
    unsigned excl = 0;
    if (tile > 0) {
      constexpr int kWin = 8;
      int64_t t = (int64_t)tile - 1;
      bool done = false;
      while (!done) {
        unsigned long long e[kWin];
#pragma unroll
        for (int q = 0; q < kWin; ++q)
          e[q] = (t - q >= 0) ? ld_relaxed(p.lookback + (size_t)(t - q) * kSsDigits + dd) : 0ULL;
#pragma unroll
        for (int q = 0; q < kWin; ++q) {
          if (done) break;
          if (t - q < 0) {
            done = true;
            break;
          }
          unsigned long long val = e[q];
          while ((uint32_t)(val >> 32) != p.epoch || ((val >> 30) & 3u) == 0) {
            if (++spins > kSpinLimit) {
              raise_error(p.st, p.mirror, kErrTimeout);
              done = true;
              break;
            }
            __nanosleep(32);
            val = ld_relaxed(p.lookback + (size_t)(t - q) * kSsDigits + dd);
          }
          if (done) break;
          excl += (unsigned)(val & 0x3fffffffu);
          if (((val >> 30) & 3u) == kFlagIncl) done = true;
        }
        t -= kWin;
      }
      const unsigned long long tag = (unsigned long long)p.epoch << 32;
      st_relaxed(p.lookback + (size_t)tile * kSsDigits + dd,
                 tag | ((unsigned long long)kFlagIncl << 30) | (excl + total[h]));
    }
    s_glob[dd] = (int)(p.ctl->base[dd] + excl) - (int)s_doff[dd];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kSsItems; ++j) {
    const unsigned sp = s_doff[d[j]] + s_whist[w][d[j]] + rank[j];
    s_keys[sp] = k[j];
    s_vals[sp] = v[j];
  }
  __syncthreads();
  const int64_t valid = N - tbase < kSsTile ? N - tbase : kSsTile;
  for (int sidx = tid; sidx < valid; sidx += kSsBlock) {
    const int g = s_glob[bucket_of(s_split, nsplit, s_keys[sidx])] + sidx;
    if ((unsigned)g < (unsigned)N) {
      p.kb0[g] = s_keys[sidx];
      p.vb0[g] = s_vals[sidx];
    }
  }
}

// ------------------------------------------------------------------ local
struct LocalShared {
  uint64_t key[kLocCap];
  uint32_t idx[kLocCap];
  int32_t init_pos[kLocCap];  // sorted position of each new head (its key is kb0[pos])
  int32_t init_row[kLocCap];
  unsigned scan[kLocBlock / 32];
  unsigned long long prefix;
  unsigned bucket;
  int ninit;
};

__device__ __forceinline__ unsigned block_excl_scan(unsigned x, unsigned* s_scan, unsigned* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned y = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned z = __shfl_up_sync(0xffffffffu, y, off);
    if (lane >= off) y += z;
  }
  __syncthreads();
  if (lane == 31) s_scan[w] = y;
  __syncthreads();
  unsigned pre = 0, tot = 0;
  for (int ww = 0; ww < (int)(blockDim.x >> 5); ++ww) {
    const unsigned c = s_scan[ww];
    if (ww < w) pre += c;
    tot += c;
  }
  *total = tot;
  return pre + y - x;
}

// look-back over buckets by warp 0: (heads, new) prefix of this bucket
__device__ __forceinline__ void bucket_lookback(const SsParams& p, unsigned b, unsigned long long tH,
                                                unsigned long long tN, LocalShared& sh) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  unsigned long long* lb = p.ctl->blb;
  unsigned long long hx = 0, nx = 0;
  if (b == 0) {
    if (lane == 0) st_relaxed(lb, kIncl | (tH << 31) | tN);
  } else {
    if (lane == 0) st_relaxed(lb + b, kAgg | (tH << 31) | tN);
    int64_t t = (int64_t)b - 1;
    int spins = 0;
    bool done = false;
    while (!done) {
      const int64_t idx = t - lane;
      unsigned long long e = idx >= 0 ? ld_relaxed(lb + idx) : kIncl;
      while (!__all_sync(0xffffffffu, (e >> 62) != 0)) {
        if (++spins > kSpinLimit) break;
        __nanosleep(32);
        if ((e >> 62) == 0) e = ld_relaxed(lb + idx);
      }
      if (spins > kSpinLimit) {
        if (lane == 0) raise_error(p.st, p.mirror, kErrTimeout);
        break;
      }
      const unsigned incl = __ballot_sync(0xffffffffu, (e >> 62) == 2);
      const int stop = incl ? __ffs(incl) - 1 : 31;
      unsigned long long h = lane <= stop ? (e >> 31) & 0x7fffffffULL : 0;
      unsigned long long n = lane <= stop ? e & 0x7fffffffULL : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        h += __shfl_xor_sync(0xffffffffu, h, off);
        n += __shfl_xor_sync(0xffffffffu, n, off);
      }
      hx += h;
      nx += n;
      done = incl != 0;
      t -= 32;
    }
    if (lane == 0) st_relaxed(lb + b, kIncl | ((hx + tH) << 31) | (nx + tN));
  }
  if (lane == 0) sh.prefix = (hx << 32) | nx;
}

// outputs of one head / element (shared by the in-memory and streamed paths)
__device__ __forceinline__ void write_head(const SsParams& p, LocalShared& sh, uint64_t ukey,
                                           unsigned seg, int64_t pos, bool isnew, int64_t slot,
                                           int64_t row, unsigned new_rank, int32_t key_at) {
  const int64_t key = from_ukey(ukey);
  int64_t r = row;
  if (isnew) {
    r = (int64_t)(p.bdev->row_base + new_rank);
    if (r >= p.mapped_rows) {
      raise_error(p.st, p.mirror, kErrTableFull);
      r = -1;
    } else {
      p.slots[slot].row = r;
      p.row_keys[r] = key;
      const int q = atomicAdd(&sh.ninit, 1);
      if (q < kLocCap) {
        sh.init_pos[q] = key_at;
        sh.init_row[q] = (int32_t)r;
      }
    }
  }
  p.uniq[seg] = key;
  p.rows[seg] = r;
  p.seg_start[seg] = (int32_t)pos;
}

// keys: where init_pos points (the bucket in shared memory, or the sorted
// keys in global memory for a streamed bucket)
__device__ void init_rows(const SsParams& p, LocalShared& sh, const uint64_t* keys) {
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nf4 = p.row_floats >> 2, ncol = p.D >> 2;
  const float sv = p.adagrad ? p.acc0 : 0.0f;
  const int n = sh.ninit < kLocCap ? sh.ninit : kLocCap;
  for (int r = w; r < n; r += kLocBlock / 32) {
    const uint64_t base = mix64((uint64_t)from_ukey(keys[sh.init_pos[r]]) ^ p.init_seed);
    float4* dst = reinterpret_cast<float4*>(p.row_data + (int64_t)sh.init_row[r] * p.row_floats);
    for (int c = lane; c < nf4; c += 32) {
      float4 o;
      if (c < ncol) {
        o.x = init_value(base, 4 * c + 0, p.two_s);
        o.y = init_value(base, 4 * c + 1, p.two_s);
        o.z = init_value(base, 4 * c + 2, p.two_s);
        o.w = init_value(base, 4 * c + 3, p.two_s);
      } else {
        o = make_float4(sv, sv, sv, sv);
      }
      dst[c] = o;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) sh.ninit = 0;
  __syncthreads();
}

__global__ void __launch_bounds__(kLocBlock) ss_local_kernel(const __grid_constant__ SsParams p) {
  extern __shared__ __align__(16) unsigned char s_raw[];
  LocalShared& sh = *reinterpret_cast<LocalShared*>(s_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    sh.bucket = atomicAdd(&p.ctl->bucket_counter, 1u);
    sh.ninit = 0;
  }
  __syncthreads();
  const unsigned b = sh.bucket;
  const int nsplit = (int)p.ctl->nsplit;
  const unsigned nb = 2u * (unsigned)nsplit + 1u;
  const int64_t off = p.ctl->base[b];
  const int64_t m = b < nb ? (int64_t)p.ctl->hist[b] : 0;
  const bool eq_bucket = (b & 1u) != 0;
  const int64_t N = p.N;

  if (m <= kLocCap) {
    // ---- in shared memory: load, sort, heads, probes
    for (int i = tid; i < m; i += kLocBlock) {
      sh.key[i] = p.kb0[off + i];
      sh.idx[i] = p.vb0[off + i];
    }
    __syncthreads();
    if (!eq_bucket && m > 1) bitonic_sort(sh.key, sh.idx, (int)m);
    // each thread: 8 consecutive sorted elements
    constexpr int kPer = kLocCap / kLocBlock;
    const int i0 = tid * kPer;
    bool head[kPer], isnew[kPer];
    int64_t slot[kPer], row[kPer];
    unsigned nh = 0, nn = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = i0 + j;
      head[j] = i < m && (i == 0 || sh.key[i] != sh.key[i - 1]);
      isnew[j] = false;
      slot[j] = -1;
      row[j] = -1;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (head[j] && from_ukey(sh.key[i0 + j]) != kEmptyKey) {
        isnew[j] = idmap_probe(p.slots, p.slot_mask, from_ukey(sh.key[i0 + j]), &slot[j], &row[j]);
        if (slot[j] < 0) raise_error(p.st, p.mirror, kErrTableFull);
      }
      nh += head[j];
      nn += isnew[j];
    }
    unsigned totH, totN;
    const unsigned exH = block_excl_scan(nh, sh.scan, &totH);
    const unsigned exN = block_excl_scan(nn, sh.scan, &totN);
    __syncthreads();
    bucket_lookback(p, b, totH, totN, sh);
    __syncthreads();
    const unsigned Hx = (unsigned)(sh.prefix >> 32), Nx = (unsigned)(sh.prefix & 0xffffffffULL);
    unsigned hrun = Hx + exH, nrun = Nx + exN;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = i0 + j;
      if (i >= m) break;
      const int64_t pos = off + i;
      if (head[j]) {
        write_head(p, sh, sh.key[i], hrun, pos, isnew[j], slot[j], row[j], nrun, i);
        nrun += isnew[j];
        ++hrun;
      }
      const unsigned seg = hrun - 1;
      const uint32_t occ = sh.idx[i];
      p.seg_of[pos] = (int32_t)seg;
      p.svals[pos] = occ;
      if (occ < (uint64_t)N) p.inv[occ] = (int32_t)seg;
    }
    if (b == gridDim.x - 1 && tid == 0) {
      // the last bucket CTA knows the totals
      const unsigned long long U = (unsigned long long)Hx + totH, nnew = (unsigned long long)Nx + totN;
      p.bdev->U = (unsigned)U;
      p.bdev->n_new = (unsigned)nnew;
      unsigned long long nf = p.bdev->row_base + nnew;
      if (nf > (unsigned long long)p.mapped_rows) nf = (unsigned long long)p.mapped_rows;
      p.st->next_free = nf;
      if (p.mirror) {
        p.mirror->next_free = nf;
        __threadfence_system();
      }
      p.seg_start[U] = (int32_t)N;
    }
    init_rows(p, sh, sh.key);
    return;
  }

  // ---- oversized bucket, streamed from global memory
  if (!eq_bucket) bitonic_sort(p.kb0 + off, p.vb0 + off, (int)m);
  __threadfence_block();
  __syncthreads();
  // sweep 1: heads, probes (kept in kb1/vb1 of the same range), counts
  unsigned long long cH = 0, cN = 0;
  for (int64_t c0 = 0; c0 < m; c0 += kLocBlock) {
    const int64_t i = c0 + tid;
    bool hd = false, nw = false;
    if (i < m) {
      const uint64_t u = p.kb0[off + i];
      hd = i == 0 || u != p.kb0[off + i - 1];
      int64_t slot = -1, row = -1;
      if (hd && from_ukey(u) != kEmptyKey) {
        nw = idmap_probe(p.slots, p.slot_mask, from_ukey(u), &slot, &row);
        if (slot < 0) raise_error(p.st, p.mirror, kErrTableFull);
      }
      p.kb1[off + i] = (uint64_t)(nw ? slot : row);
      p.vb1[off + i] = (hd ? 1u : 0u) | (nw ? 2u : 0u);
    }
    unsigned t1, t2;
    block_excl_scan(hd ? 1u : 0u, sh.scan, &t1);
    block_excl_scan(nw ? 1u : 0u, sh.scan, &t2);
    cH += t1;
    cN += t2;
  }
  __syncthreads();
  bucket_lookback(p, b, cH, cN, sh);
  __syncthreads();
  const unsigned Hx = (unsigned)(sh.prefix >> 32), Nx = (unsigned)(sh.prefix & 0xffffffffULL);
  // sweep 2: outputs
  unsigned hcarry = Hx, ncarry = Nx;
  for (int64_t c0 = 0; c0 < m; c0 += kLocBlock) {
    const int64_t i = c0 + tid;
    const uint32_t fl = i < m ? p.vb1[off + i] : 0u;
    const bool hd = fl & 1u, nw = (fl & 2u) != 0;
    unsigned t1, t2;
    const unsigned eh = block_excl_scan(hd ? 1u : 0u, sh.scan, &t1);
    const unsigned en = block_excl_scan(nw ? 1u : 0u, sh.scan, &t2);
    if (i < m) {
      const int64_t pos = off + i;
      const uint64_t u = p.kb0[pos];
      const int64_t sr = (int64_t)p.kb1[pos];
      if (hd)
        write_head(p, sh, u, hcarry + eh, pos, nw, nw ? sr : -1, nw ? -1 : sr, ncarry + en,
                   (int32_t)pos);
      // the segment of element i: heads up to and including i, minus one
      const unsigned seg = hcarry + eh + (hd ? 1u : 0u) - 1u;
      const uint32_t occ = p.vb0[pos];
      p.seg_of[pos] = (int32_t)seg;
      p.svals[pos] = occ;
      if (occ < (uint64_t)N) p.inv[occ] = (int32_t)seg;
    }
    hcarry += t1;
    ncarry += t2;
    __syncthreads();
    if (sh.ninit >= kLocCap - kLocBlock) init_rows(p, sh, p.kb0);
  }
  if (b == gridDim.x - 1 && tid == 0) {
    const unsigned long long U = hcarry, nnew = ncarry;
    p.bdev->U = (unsigned)U;
    p.bdev->n_new = (unsigned)nnew;
    unsigned long long nf = p.bdev->row_base + nnew;
    if (nf > (unsigned long long)p.mapped_rows) nf = (unsigned long long)p.mapped_rows;
    p.st->next_free = nf;
    if (p.mirror) {
      p.mirror->next_free = nf;
      __threadfence_system();
    }
    p.seg_start[U] = (int32_t)N;
  }
  init_rows(p, sh, p.kb0);
}

cudaError_t launch_sample_dedup(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N,
                                cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(b->ss, 0, kSsCtlZeroBytes, s);
  if (e != cudaSuccess) return e;
  b->epoch += 1;
  if (b->epoch == 0) b->epoch = 1;
  SsParams p;
  p.keys = keys;
  p.N = N;
  p.ctl = b->ss;
  p.kb0 = b->kbuf[0];
  p.vb0 = b->vbuf[0];
  p.kb1 = b->kbuf[1];
  p.vb1 = b->vbuf[1];
  p.lookback = b->ss_lookback;
  p.epoch = b->epoch;
  p.slots = t->slots;
  p.slot_mask = (uint64_t)t->capacity - 1;
  p.row_data = reinterpret_cast<float*>(t->rows.va);
  p.row_keys = reinterpret_cast<int64_t*>(t->keys.va);
  p.mapped_rows = t->mapped_rows;
  p.row_floats = t->row_floats;
  p.D = t->D;
  p.adagrad = t->cfg.optimizer == RECIS_ADAGRAD;
  p.acc0 = (float)t->cfg.adagrad_init_acc;
  p.two_s = t->init_two_s;
  p.init_seed = t->cfg.init_seed;
  p.uniq = b->uniq;
  p.rows = b->rows;
  p.inv = b->inv;
  p.seg_of = b->seg_of;
  p.svals = b->svals;
  p.seg_start = b->seg_start;
  p.bdev = b->bdev;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  {
    int64_t blocks = (N + 4095) / 4096;
    if (blocks > 2 * kSMs) blocks = 2 * kSMs;
    if (blocks < 1) blocks = 1;
    LaunchScope ls("ss_plan", s);
    ss_plan_kernel<<<(unsigned)blocks, 512, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const int64_t tiles = (N + kSsTile - 1) / kSsTile;
    LaunchScope ls("ss_scatter", s);
    ss_scatter_kernel<<<(unsigned)tiles, kSsBlock, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    static bool attr_set[128] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 128 && !attr_set[dev]) {
      e = cudaFuncSetAttribute(ss_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)sizeof(LocalShared));
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    LaunchScope ls("ss_local", s);
    ss_local_kernel<<<kSsDigits - 1, kLocBlock, sizeof(LocalShared), s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace recis
