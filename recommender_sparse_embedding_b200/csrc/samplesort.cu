// samplesort.cu -- dedup + IDMap find-or-insert for batches of up to
// kSampleSortMaxN keys (RecIS README, Key optimisations > Distributed
// optimisation: merged requests deduplicated; > Efficient dynamic embedding:
// IDMap first-level store, EmbeddingBlocks second-level store).
//
// It produces exactly what the radix-sort path (sort.cu + unique.cu) produces:
// unique keys ascending, inverse index, rows (new keys get rows in ascending
// key order), segment starts, the segment and the occurrence of each sorted
// position, and initialised new rows.  The digit passes are replaced by six
// short launches, none of which waits on another CTA:
//   ss_rank      a strided sample of the keys (2048 to 8192 by batch size) is
//                sorted by ranking: every sample's rank is its count of
//                smaller samples (ties by position), spread over many CTAs.
//   ss_count     per tile of 2048 keys: up to 1023 distinct splitters from the
//                sorted sample, the bucket of every key (key u goes to bucket
//                2r + [u == split[r]], r = #splitters < u, so buckets are
//                ordered by key and a key equal to a splitter -- a hot key --
//                has a bucket of its own), the tile's bucket histogram, and
//                the IDMap find-or-insert of every occurrence (a missing key
//                claims a free slot by CAS; its row is assigned later).
//   ss_tilescan  per bucket, the exclusive prefix of the tile histograms (so
//                the scatter is stable); the last CTA scans the bucket totals
//                into bucket starts.
//   ss_scatter   moves (key, occurrence) into bucket order, stably.
//   ss_local     sorts every key-range bucket by (key, occurrence): one warp
//                per bucket of up to 512 keys, in registers; the whole CTA in
//                shared memory for larger ones.  An equality bucket holds one
//                key, already in occurrence order.  Heads (first position of
//                each distinct key) and new keys are numbered within the
//                bucket; the last CTA scans the per-bucket counts.
//   ss_finish    a flat pass over the sorted positions writes every output and
//                initialises the new rows.
// A key-range bucket larger than shared memory (only for adversarial key
// orders) is sorted by the same network in global memory.
#include <climits>

#include "internal.h"

namespace recis {

namespace {

constexpr int kRankThreads = 256;
constexpr int kCountThreads = 256;
constexpr int kCountItems = 8;
constexpr int kTile = kCountThreads * kCountItems;  // 2048 keys per count/scatter tile
constexpr int kFinThreads = 256;
constexpr int kFinItems = 2;
constexpr int kSub = kFinThreads * kFinItems;       // sorted positions per finish CTA
constexpr int kMaxProbes = 1 << 16;

// IDMap probe result of a head: row >= 0 for a key already present; -2 - slot
// for a new key whose slot this call claimed; -1 when there is no row
// (reserved key, or the IDMap was exhausted).
__device__ __forceinline__ int64_t encode_new(int64_t slot) { return -2 - slot; }

// bucket of ukey u: 2r + [u == split[r]], r = number of splitters < u
__device__ __forceinline__ unsigned bucket_of(const uint64_t* split, int nsplit, uint64_t u) {
  int lo = 0, hi = nsplit;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (split[mid] < u) lo = mid + 1; else hi = mid;
  }
  return 2u * (unsigned)lo + ((lo < nsplit && split[lo] == u) ? 1u : 0u);
}

// Ascending bitonic network (mirror form) on n elements in shared memory: for
// merge size k the first stage compares i with i ^ (k-1), later stages i with
// i | d; every comparator puts the smaller element at the lower index, so a
// partner past the end behaves as +infinity and is skipped.  Comparator t acts
// on i = 2t - (t mod d) and its partner; the comparators of one 64-element
// block are t in [32a, 32a+32), so warp a mod (NT/32) owns block a in every
// stage whose partners stay inside a block (k <= 64, or d <= 32) and those
// stages need only __syncwarp; the others end with __syncthreads.  PAIRS
// orders by (key, idx), otherwise by key alone (idx unused).  All threads of
// the block call it; it returns after a final __syncthreads.
template <int NT, bool PAIRS, typename KeyPtr, typename IdxPtr>
__device__ void staged_sort(KeyPtr key, IdxPtr idx, int n) {
  int n2 = 64;
  while (n2 < n) n2 <<= 1;
  const int half = n2 >> 1;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  bool prev_local = false;
  for (int k = 2; k <= n2; k <<= 1) {
    for (int d = k >> 1; d > 0; d >>= 1) {
      const bool mirror = d == (k >> 1);
      const bool local = mirror ? k <= 64 : d <= 32;
      if (!local && prev_local) __syncthreads();
      const int t0 = local ? lane + 32 * w : (int)threadIdx.x;
      for (int t = t0; t < half; t += NT) {
        const int i = ((t & ~(d - 1)) << 1) | (t & (d - 1));
        const int j = mirror ? (i ^ (k - 1)) : (i | d);
        if (j < n) {
          const uint64_t ki = key[i], kj = key[j];
          if (PAIRS) {
            const uint32_t ii = idx[i], ij = idx[j];
            if (kj < ki || (kj == ki && ij < ii)) {
              key[i] = kj;
              key[j] = ki;
              idx[i] = ij;
              idx[j] = ii;
            }
          } else if (kj < ki) {
            key[i] = kj;
            key[j] = ki;
          }
        }
      }
      if (local) __syncwarp(); else __syncthreads();
      prev_local = local;
    }
  }
  __syncthreads();
}

// IDMap find-or-insert: linear probing from slot h = H(key ^ salt); a free
// slot is claimed by a 64-bit CAS on its key.  Returns the row of a key
// already present, -2 - slot for a key claimed in this call (its row is -1
// until the call assigns it, whichever occurrence claimed it), or -1 when
// the probe limit was reached.
__device__ __forceinline__ int64_t idmap_resolve(Slot* slots, uint64_t mask, int64_t key, uint64_t h,
                                                 longlong2 sv) {
  const int64_t limit = (int64_t)mask + 1 < kMaxProbes ? (int64_t)mask + 1 : kMaxProbes;
  for (int64_t n = 0; n < limit; ++n) {
    if (n > 0) sv = __ldcg(reinterpret_cast<const longlong2*>(slots + h));
    if (sv.x == key) {
      const int64_t row = sv.y >= 0 ? sv.y : __ldcg(&slots[h].row);
      return row >= 0 ? row : encode_new((int64_t)h);
    }
    if (sv.x == kEmptyKey) {
      const unsigned long long old = atomicCAS(reinterpret_cast<unsigned long long*>(&slots[h].key),
                                               (unsigned long long)kEmptyKey,
                                               (unsigned long long)key);
      if ((int64_t)old == kEmptyKey) return encode_new((int64_t)h);
      if ((int64_t)old == key) {
        const int64_t row = __ldcg(&slots[h].row);
        return row >= 0 ? row : encode_new((int64_t)h);
      }
    }
    h = (h + 1) & mask;
  }
  return -1;
}

// exclusive block scan of one value per thread; *total gets the block sum
template <int NT>
__device__ __forceinline__ unsigned block_excl_scan(unsigned x, unsigned* s_warp, unsigned* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned y = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned z = __shfl_up_sync(0xffffffffu, y, off);
    if (lane >= off) y += z;
  }
  __syncthreads();
  if (lane == 31) s_warp[w] = y;
  __syncthreads();
  unsigned pre = 0, tot = 0;
#pragma unroll
  for (int ww = 0; ww < NT / 32; ++ww) {
    const unsigned c = s_warp[ww];
    pre += ww < w ? c : 0u;
    tot += c;
  }
  *total = tot;
  return pre + y - x;
}

// exclusive block scan of two values per thread at once (low and high 32 bits)
template <int NT>
__device__ __forceinline__ unsigned long long block_excl_scan2(unsigned long long x,
                                                               unsigned long long* s_warp,
                                                               unsigned long long* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned long long y = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long z = __shfl_up_sync(0xffffffffu, y, off);
    if (lane >= off) y += z;
  }
  __syncthreads();
  if (lane == 31) s_warp[w] = y;
  __syncthreads();
  unsigned long long pre = 0, tot = 0;
#pragma unroll
  for (int ww = 0; ww < NT / 32; ++ww) {
    const unsigned long long c = s_warp[ww];
    pre += ww < w ? c : 0ull;
    tot += c;
  }
  *total = tot;
  return pre + y - x;
}

}  // namespace

struct SsParams {
  const int64_t* keys;
  int64_t N;
  int splits;               // splitter slots S + 1
  int nsample;              // sample size
  int tiles;                // count/scatter tiles
  int max_buckets;          // 2S + 1
  SsCtl* ctl;
  const uint64_t* cand;     // candidate splitters: cand[(i+1)*cand_step - 1], i < S, ascending
  int cand_step;
  uint64_t* cand_next;      // [S] quantiles of this call's sorted keys, for the next call
  uint32_t* th;             // [tiles][nbp] tile histograms, then their column prefix
  uint16_t* bkt;            // [N] bucket of each key
  uint64_t* kb;             // [N] ukeys in bucket order, then sorted
  uint32_t* vb;             // [N] occurrence of each position
  int64_t* pocc;            // [N] IDMap result of each occurrence (see idmap_resolve)
  uint64_t* meta;           // [N] per sorted position, see pack_meta
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
  uint32_t* spos;
  int32_t* seg_of;
  uint32_t* svals;
  int32_t* seg_start;
  BatchDev* bdev;
  int32_t* long_chunks;     // chunks (kShortSeg positions) holding a long segment
  DevState* st;
  HostMirror* mirror;
};

// Per sorted position, written by ss_local: the bucket, the position's
// segment within the bucket (1-based count of heads up to it), for a head
// whether its key is new and the 1-based count of new heads up to it, and in
// bit 63 whether the position's segment is longer than kShortSeg.
constexpr uint64_t kMetaLong = 1ULL << 63;
__device__ __forceinline__ uint64_t pack_meta(unsigned b, unsigned lh, unsigned lnew, bool head,
                                              bool isnew) {
  return ((uint64_t)b << 44) | ((uint64_t)head << 43) | ((uint64_t)isnew << 42) |
         ((uint64_t)lnew << 21) | (uint64_t)lh;
}

// ------------------------------------------------------------------ rank
// Sample k is the key at position floor(k N / ns).  CTA c ranks samples
// [32c, 32c+32): 8 threads per sample each count the smaller samples (ties
// broken by sample index) in one eighth of the sample, and the sum is the
// sample's place in ctl->samp.
__global__ void __launch_bounds__(kRankThreads) ss_rank_kernel(const __grid_constant__ SsParams p) {
  extern __shared__ __align__(16) uint64_t s_samp[];  // [nsample]
  const int tid = threadIdx.x;
  const int ns = p.nsample;
  const unsigned long long N = (unsigned long long)p.N;
  const int lg = 31 - __clz(ns);  // ns is a power of two
  for (int k = tid; k < ns; k += kRankThreads)
    s_samp[k] = to_ukey(__ldg(p.keys + (int64_t)(((unsigned long long)k * N) >> lg)));
  __syncthreads();
  const int i = (int)blockIdx.x * 32 + (tid >> 3);
  const int part = tid & 7;
  const uint64_t v = s_samp[i];
  unsigned cnt = 0;
#pragma unroll 8
  for (int j = part; j < ns; j += 8) {
    const uint64_t sj = s_samp[j];
    cnt += (sj < v || (sj == v && j < i)) ? 1u : 0u;
  }
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 4);
  if (part == 0) p.ctl->samp[cnt] = v;
}

// ------------------------------------------------------------------ count
// Per tile of 2048 keys: the splitters (the S candidates, ascending; a run of
// equal candidates keeps its first), the bucket of each key (kept for the
// scatter) and the tile's bucket histogram (row `tile` of th).  CTA 0 resets
// the call's tickets and records where this call's new rows start.
__global__ void __launch_bounds__(kCountThreads) ss_count_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  __shared__ uint64_t s_split[kMaxSplitters];
  __shared__ unsigned s_hist[kMaxBucketSlots];
  __shared__ unsigned s_warp[kCountThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int64_t pos0 = (int64_t)blockIdx.x * kTile + w * (kCountItems * 32) + lane;
  int64_t k[kCountItems];
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const int64_t pos = pos0 + j * 32;
    k[j] = pos < p.N ? __ldcs(p.keys + pos) : 0;
  }
  // splitters: 4 candidates per thread, in order
  const int S = p.splits - 1, step = p.cand_step;
  constexpr int kCand = kMaxSplitters / kCountThreads;  // 4
  uint64_t c[kCand];
  unsigned keepm = 0, nkeep = 0;
#pragma unroll
  for (int q = 0; q < kCand; ++q) {
    const int ci = tid * kCand + q;
    if (ci < S) {
      c[q] = __ldcg(p.cand + (ci + 1) * step - 1);
      const bool keep = ci == 0 || c[q] != __ldcg(p.cand + ci * step - 1);
      keepm |= keep ? (1u << q) : 0u;
      nkeep += keep ? 1u : 0u;
    }
  }
  unsigned nsplit;
  unsigned at = block_excl_scan<kCountThreads>(nkeep, s_warp, &nsplit);
#pragma unroll
  for (int q = 0; q < kCand; ++q)
    if (keepm & (1u << q)) s_split[at++] = c[q];
  const int nb = 2 * (int)nsplit + 1;
  const int nbp = (nb + 31) & ~31;
  for (int i = tid; i < nbp; i += kCountThreads) s_hist[i] = 0;
  if (blockIdx.x == 0 && tid == 0) {
    p.ctl->nsplit = nsplit;
    p.ctl->nb = (unsigned)nb;
    p.ctl->nbp = (unsigned)nbp;
    p.ctl->ticket_scan = 0;
    p.ctl->ticket_local = 0;
    p.bdev->row_base = *(volatile unsigned long long*)&p.st->next_free;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const int64_t pos = pos0 + j * 32;
    if (pos < p.N) {
      const unsigned b = bucket_of(s_split, (int)nsplit, to_ukey(k[j]));
      p.bkt[pos] = (uint16_t)b;
      atomicAdd(&s_hist[b], 1u);
    }
  }
  __syncthreads();
  uint32_t* row = p.th + (size_t)blockIdx.x * nbp;
  for (int i = tid; i < nbp; i += kCountThreads) row[i] = s_hist[i];
  pdl_trigger();
}

// ------------------------------------------------------------------ probe
// IDMap find-or-insert of every occurrence (runs on a second stream beside
// count, tile scan and scatter): two keys per thread, both first slots loaded
// before either is resolved.  A missing key claims a free slot by CAS; every
// occurrence of it then sees the slot with row -1 and records -2 - slot.
constexpr int kProbeThreads = 256;
constexpr int kProbeItems = 2;
__global__ void __launch_bounds__(kProbeThreads) ss_probe_kernel(const __grid_constant__ SsParams p) {
  const int64_t pos0 = (int64_t)blockIdx.x * (kProbeThreads * kProbeItems) + threadIdx.x;
  int64_t k[kProbeItems];
  uint64_t h[kProbeItems];
  longlong2 sv[kProbeItems];
#pragma unroll
  for (int j = 0; j < kProbeItems; ++j) {
    const int64_t pos = pos0 + j * kProbeThreads;
    k[j] = pos < p.N ? __ldcs(p.keys + pos) : kEmptyKey;
    h[j] = mix64((uint64_t)k[j] ^ kSlotSalt) & p.slot_mask;
    if (k[j] != kEmptyKey) sv[j] = __ldcg(reinterpret_cast<const longlong2*>(p.slots + h[j]));
  }
  bool reserved = false;
#pragma unroll
  for (int j = 0; j < kProbeItems; ++j) {
    const int64_t pos = pos0 + j * kProbeThreads;
    if (pos >= p.N) continue;
    int64_t r = -1;
    if (k[j] == kEmptyKey) {
      reserved = true;
    } else {
      r = idmap_resolve(p.slots, p.slot_mask, k[j], h[j], sv[j]);
      if (r == -1) raise_error(p.st, p.mirror, kErrTableFull);
    }
    p.pocc[pos] = r;
  }
  if (reserved) raise_error(p.st, p.mirror, kErrReservedKey);
}

// ------------------------------------------------------------------ tile scan
// CTA c owns buckets 32c .. 32c+31 (one per lane); warp w owns a contiguous
// range of tiles.  Turns th[t][b] into the exclusive prefix over tiles and
// writes the bucket totals; the last CTA scans the totals into bucket starts.
__global__ void __launch_bounds__(1024) ss_tilescan_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  __shared__ unsigned s_part[32][33];
  __shared__ unsigned s_warp[32];
  __shared__ bool s_last;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nbp = (int)p.ctl->nbp;
  const int T = p.tiles;
  const int per = (T + 31) / 32;
  const int ta = w * per, tb = ta + per < T ? ta + per : T;
  if ((int)blockIdx.x * 32 < nbp) {
    const int b = (int)blockIdx.x * 32 + lane;
    unsigned sum = 0;
#pragma unroll 4
    for (int t = ta; t < tb; ++t) sum += __ldcg(p.th + (size_t)t * nbp + b);
    s_part[w][lane] = sum;
    __syncthreads();
    if (w == 0) {
      unsigned run = 0;
      for (int ww = 0; ww < 32; ++ww) {
        const unsigned c = s_part[ww][lane];
        s_part[ww][lane] = run;
        run += c;
      }
      p.ctl->tot[b] = run;
    }
    __syncthreads();
    unsigned run = s_part[w][lane];
    for (int t = ta; t < tb; ++t) {
      uint32_t* q = p.th + (size_t)t * nbp + b;
      const unsigned c = __ldcg(q);
      *q = run;
      run += c;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&p.ctl->ticket_scan, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // bucket starts: two consecutive buckets per thread
  const int nb = (int)p.ctl->nb;
  unsigned c[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int b = 2 * tid + h;
    c[h] = b < nb ? __ldcg(&p.ctl->tot[b]) : 0u;
  }
  unsigned total;
  const unsigned ex = block_excl_scan<1024>(c[0] + c[1], s_warp, &total);
  if (2 * tid < nb) p.ctl->base[2 * tid] = ex;
  if (2 * tid + 1 < nb) p.ctl->base[2 * tid + 1] = ex + c[0];
  pdl_trigger();
}

// ------------------------------------------------------------------ scatter
// Stable move of (ukey, occurrence) into bucket order.  Within a tile, warp w
// holds keys w*256 .. w*256+255 (item j of lane l is key w*256 + 32j + l);
// ranks within a warp come from match_any over the items in order, ranks
// across warps from a prefix over per-warp bucket counters.
__global__ void __launch_bounds__(kCountThreads) ss_scatter_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  extern __shared__ unsigned s_wc[];  // [8][nbp] per-warp counters, then destinations
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nbp = (int)p.ctl->nbp;
  const int64_t pos0 = (int64_t)blockIdx.x * kTile + w * (kCountItems * 32) + lane;
  uint64_t k[kCountItems];
  unsigned b[kCountItems], rank[kCountItems];
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const int64_t pos = pos0 + j * 32;
    const bool ok = pos < p.N;
    k[j] = ok ? to_ukey(__ldcs(p.keys + pos)) : 0;
    b[j] = ok ? (unsigned)p.bkt[pos] : 0xffffffffu;
  }
  for (int i = tid; i < (kCountThreads / 32) * nbp; i += kCountThreads) s_wc[i] = 0;
  __syncthreads();
  unsigned* mine = s_wc + w * nbp;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const unsigned peers = __match_any_sync(0xffffffffu, b[j]);
    const int leader = __ffs(peers) - 1;
    const unsigned before = b[j] != 0xffffffffu ? mine[b[j]] : 0u;
    rank[j] = before + __popc(peers & lt);
    __syncwarp();
    if (lane == leader && b[j] != 0xffffffffu) mine[b[j]] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  const uint32_t* th_row = p.th + (size_t)blockIdx.x * nbp;
  const int nb = (int)p.ctl->nb;
  for (int i = tid; i < nbp; i += kCountThreads) {
    unsigned run = __ldcg(th_row + i) + (i < nb ? __ldcg(&p.ctl->base[i]) : 0u);
#pragma unroll
    for (int ww = 0; ww < kCountThreads / 32; ++ww) {
      const unsigned c = s_wc[ww * nbp + i];
      s_wc[ww * nbp + i] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    if (b[j] == 0xffffffffu) continue;
    const unsigned dst = mine[b[j]] + rank[j];
    if (dst < (unsigned)p.N) {
      p.kb[dst] = k[j];
      p.vb[dst] = (uint32_t)(pos0 + j * 32);
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ local
template <int NT, int CAP>
struct LocalShared {
  uint64_t key[CAP];
  uint32_t idx[CAP];
  uint32_t loc[CAP];    // per position: lh | lnew << 13 | head << 26 | new << 27
  uint8_t hlong[CAP];   // per bucket-local segment: longer than kShortSeg
  unsigned long long warp[NT / 32];
  bool last;
};

// Number heads and new keys of a sorted bucket (in shared memory, or in
// global memory for an oversized one) in rounds of NT positions, write the
// sorted keys and occurrences (from shared memory) and every position's meta.
// A segment is long when the key 16 positions after its head is the same.
template <int NT, int CAP>
__device__ void block_number(const SsParams& p, LocalShared<NT, CAP>& sh, unsigned b, int64_t m,
                             int64_t off, bool in_smem) {
  const int tid = threadIdx.x;
  unsigned long long carry = 0;
  for (int64_t c0 = 0; c0 < m; c0 += NT) {
    const int64_t i = c0 + tid;
    unsigned f = 0;
    uint64_t u = 0;
    uint32_t occ = 0;
    bool lng = false;
    if (i < m) {
      u = in_smem ? sh.key[i] : __ldcg(p.kb + off + i);
      occ = in_smem ? sh.idx[i] : __ldcg(p.vb + off + i);
      const uint64_t before = i == 0 ? 0 : (in_smem ? sh.key[i - 1] : __ldcg(p.kb + off + i - 1));
      if (i == 0 || u != before) {
        f = 1u | (__ldcg(p.pocc + occ) <= -2 ? 2u : 0u);
        const int64_t j = i + kShortSeg;
        lng = j < m && (in_smem ? sh.key[j] : __ldcg(p.kb + off + j)) == u;
      }
    }
    unsigned long long tot;
    const unsigned long long ex =
        carry + block_excl_scan2<NT>(((unsigned long long)(f >> 1) << 32) | (f & 1u), sh.warp, &tot);
    if (i < m) {
      const unsigned lh = (unsigned)(ex & 0xffffffffULL) + (f & 1u);
      const unsigned ln = (unsigned)(ex >> 32) + (f >> 1);
      if (in_smem) {
        p.kb[off + i] = u;
        p.vb[off + i] = occ;
        sh.loc[i] = lh | (ln << 13) | ((f & 1u) << 26) | ((f >> 1) << 27);
        if (f & 1u) sh.hlong[lh - 1] = lng ? 1 : 0;
      } else {
        p.meta[off + i] = pack_meta(b, lh, ln, f & 1u, (f >> 1) != 0);
      }
    }
    carry += tot;
  }
  if (tid == 0) {
    p.ctl->hcnt[b] = (unsigned)(carry & 0xffffffffULL);
    p.ctl->ncnt[b] = (unsigned)(carry >> 32);
  }
  __syncthreads();
  if (in_smem) {
    for (int i = tid; i < m; i += NT) {
      const uint32_t v = sh.loc[i];
      const unsigned lh = v & 0x1fffu;
      const uint64_t mt = pack_meta(b, lh, (v >> 13) & 0x1fffu, (v >> 26) & 1u, (v >> 27) & 1u);
      p.meta[off + i] = mt | (sh.hlong[lh - 1] ? kMetaLong : 0ULL);
    }
  } else {
    // oversized bucket (adversarial key order): a head of a long segment marks
    // its positions
    __threadfence_block();
    for (int64_t i = tid; i < m; i += NT) {
      const uint64_t u = __ldcg(p.kb + off + i);
      if ((i == 0 || u != __ldcg(p.kb + off + i - 1)) && i + kShortSeg < m &&
          __ldcg(p.kb + off + i + kShortSeg) == u) {
        for (int64_t j = i; j < m && __ldcg(p.kb + off + j) == u; ++j) p.meta[off + j] |= kMetaLong;
      }
    }
  }
}

// One CTA per key-range bucket and the equality bucket after it.  A
// key-range bucket is sorted by (key, occurrence) in
// shared memory (oversized ones in global memory), then numbered; an
// equality bucket holds one key, already in occurrence order (stable
// scatter).  The last CTA scans the bucket counts into the call's segment and
// new-row prefixes.
template <int NT, int CAP>
__global__ void __launch_bounds__(NT) ss_local_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  extern __shared__ __align__(16) unsigned char s_raw[];
  LocalShared<NT, CAP>& sh = *reinterpret_cast<LocalShared<NT, CAP>*>(s_raw);
  const int tid = threadIdx.x;
  const unsigned nb = p.ctl->nb;
  // CTA c: key-range bucket 2c, then equality bucket 2c+1
  for (unsigned b = 2 * blockIdx.x; b < 2 * blockIdx.x + 2 && b < nb; ++b) {
    const int64_t m = (int64_t)p.ctl->tot[b];
    const int64_t off = (int64_t)p.ctl->base[b];
    if (m == 0) {
      if (tid == 0) {
        p.ctl->hcnt[b] = 0;
        p.ctl->ncnt[b] = 0;
      }
    } else if (b & 1u) {
      const bool isnew = __ldcg(p.pocc + __ldcg(p.vb + off)) <= -2;
      const uint64_t lng = m > kShortSeg ? kMetaLong : 0ULL;
      for (int64_t i = tid; i < m; i += NT)
        p.meta[off + i] = pack_meta(b, 1u, isnew ? 1u : 0u, i == 0, i == 0 && isnew) | lng;
      if (tid == 0) {
        p.ctl->hcnt[b] = 1;
        p.ctl->ncnt[b] = isnew ? 1u : 0u;
      }
    } else if (m <= CAP) {
      for (int i = tid; i < m; i += NT) {
        sh.key[i] = __ldcg(p.kb + off + i);
        sh.idx[i] = __ldcg(p.vb + off + i);
      }
      __syncthreads();
      staged_sort<NT, true>(sh.key, sh.idx, (int)m);
      block_number<NT, CAP>(p, sh, b, m, off, true);
    } else {
      staged_sort<NT, true>(p.kb + off, p.vb + off, (int)m);
      __threadfence_block();
      block_number<NT, CAP>(p, sh, b, m, off, false);
    }
    __syncthreads();
  }
  // the last CTA scans the bucket counts and publishes the call's totals
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(&p.ctl->ticket_local, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  // thread t owns buckets PER*t .. PER*t+PER-1: all loads at once, a serial
  // scan of its own, one block scan
  constexpr int PER = (kMaxBucketSlots + NT - 1) / NT;
  unsigned long long v[PER], own = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const unsigned i = (unsigned)(tid * PER + q);
    v[q] = i < nb ? ((unsigned long long)__ldcg(&p.ctl->ncnt[i]) << 32) | __ldcg(&p.ctl->hcnt[i]) : 0ULL;
  }
#pragma unroll
  for (int q = 0; q < PER; ++q) own += v[q];
  unsigned long long carry;
  unsigned long long ex = block_excl_scan2<NT>(own, sh.warp, &carry);
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const unsigned i = (unsigned)(tid * PER + q);
    if (i < nb) {
      p.ctl->hpre[i] = (unsigned)(ex & 0xffffffffULL);
      p.ctl->npre[i] = (unsigned)(ex >> 32);
    }
    ex += v[q];
  }
  if (tid == 0) {
    const unsigned long long U = carry & 0xffffffffULL, nnew = carry >> 32;
    p.bdev->U = (unsigned)U;
    p.bdev->n_new = (unsigned)nnew;
    p.bdev->nlong = 0;
    unsigned long long nf = p.bdev->row_base + nnew;
    if (nf > (unsigned long long)p.mapped_rows) nf = (unsigned long long)p.mapped_rows;
    p.st->next_free = nf;
    if (p.mirror) {
      p.mirror->next_free = nf;
      __threadfence_system();
    }
    p.seg_start[U] = (int32_t)p.N;
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ finish
struct FinishShared {
  int64_t init_key[kFinThreads * kFinItems];
  int32_t init_row[kFinThreads * kFinItems];
  unsigned chunk_long;  // bit c: chunk c (kShortSeg positions) of this CTA holds a long segment
  int ninit;
};
static_assert(kSub / kShortSeg <= 32, "one bit per chunk of a finish CTA");

// Flat pass over the sorted positions, kSub per CTA (position blk*kSub +
// j*256 + t for item j of thread t): segment of every position from its
// bucket's prefix, all outputs, and the initialisation of the new rows.
__global__ void __launch_bounds__(kFinThreads) ss_finish_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  __shared__ FinishShared sh;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) {
    sh.ninit = 0;
    sh.chunk_long = 0;
  }
  __syncthreads();
  const int64_t q0 = (int64_t)blockIdx.x * kSub + tid;
  const uint64_t row_base = p.bdev->row_base;
  uint64_t mt[kFinItems];
  uint32_t occ[kFinItems];
#pragma unroll
  for (int j = 0; j < kFinItems; ++j) {
    const int64_t q = q0 + j * kFinThreads;
    if (q < p.N) {
      mt[j] = __ldcs(p.meta + q);
      occ[j] = __ldcs(p.vb + q);
    }
  }
#pragma unroll
  for (int j = 0; j < kFinItems; ++j) {
    const int64_t q = q0 + j * kFinThreads;
    if (q >= p.N) break;
    const uint64_t m = mt[j];
    if (m >> 63) atomicOr(&sh.chunk_long, 1u << ((tid + j * kFinThreads) / kShortSeg));
    const unsigned b = (unsigned)(m >> 44) & 0xfffu;
    const unsigned lh = (unsigned)(m & 0x1fffffULL);
    const unsigned seg = __ldg(&p.ctl->hpre[b]) + lh - 1u;
    p.seg_of[q] = (int32_t)seg;
    p.svals[q] = occ[j];
    if (occ[j] < (uint32_t)p.N) {
      p.inv[occ[j]] = (int32_t)seg;
      p.spos[occ[j]] = (uint32_t)q;
    }
    if ((m >> 43) & 1u) {
      const int64_t key = from_ukey(__ldcs(p.kb + q));
      int64_t row = __ldcg(p.pocc + occ[j]);
      if ((m >> 42) & 1u) {
        const int64_t slot = -2 - row;
        const unsigned ln = (unsigned)((m >> 21) & 0x1fffffULL);
        row = (int64_t)(row_base + __ldg(&p.ctl->npre[b]) + ln - 1u);
        if (row >= p.mapped_rows) {
          raise_error(p.st, p.mirror, kErrTableFull);
          row = -1;
        } else {
          p.slots[slot].row = row;
          p.row_keys[row] = key;
          const int at = atomicAdd(&sh.ninit, 1);
          sh.init_key[at] = key;
          sh.init_row[at] = (int32_t)row;
        }
      }
      p.uniq[seg] = key;
      p.rows[seg] = row;
      p.seg_start[seg] = (int32_t)q;
    }
  }
  // chunks of this CTA holding a long segment, for the backward's reduction
  __syncthreads();
  if (w == 0) {
    const bool has = (sh.chunk_long >> lane) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, has);
    unsigned at = 0;
    if (lane == 0 && bal) at = atomicAdd(&p.bdev->nlong, (unsigned)__popc(bal));
    at = __shfl_sync(0xffffffffu, at, 0);
    if (has)
      p.long_chunks[at + __popc(bal & ((1u << lane) - 1u))] =
          (int32_t)(blockIdx.x * (kSub / kShortSeg) + lane);
  }
  // the next call's candidate splitters: quantiles of this call's sorted keys
  if (blockIdx.x == 0) {
    const unsigned long long N = (unsigned long long)p.N;
    for (int i = tid; i < p.splits - 1; i += kFinThreads) {
      const unsigned long long q = ((unsigned long long)(i + 1) * N) / (unsigned long long)p.splits;
      p.cand_next[i] = __ldcg(p.kb + (q > 0 ? q - 1 : 0));
    }
  }
  __syncthreads();
  // initialise the new rows: one warp per row, one 16-byte column per lane
  const int n = sh.ninit;
  const int nf4 = p.row_floats >> 2, ncol = p.D >> 2;
  const float sv = p.adagrad ? p.acc0 : 0.0f;
  for (int rr = w; rr < n; rr += kFinThreads / 32) {
    const uint64_t base = mix64((uint64_t)sh.init_key[rr] ^ p.init_seed);
    float4* dst = reinterpret_cast<float4*>(p.row_data + (int64_t)sh.init_row[rr] * p.row_floats);
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
  pdl_trigger();
}

// ------------------------------------------------------------------ host
int samplesort_splits_for(int64_t) { return kMaxSplitters; }

int64_t samplesort_tiles_for(int64_t N) { return (N + kTile - 1) / kTile; }

static int sample_size_for(int64_t N) {
  if (N <= 262144) return 2048;
  if (N <= 524288) return 4096;
  return 8192;
}

template <typename K>
static cudaError_t set_smem(K kernel, int bytes, bool* done, int dev) {
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

template <int NT, int CAP>
static cudaError_t launch_local(const SsParams& p, int dev, cudaStream_t s) {
  static bool attr[64] = {false};
  cudaError_t e = set_smem(ss_local_kernel<NT, CAP>, (int)sizeof(LocalShared<NT, CAP>), attr, dev);
  if (e != cudaSuccess) return e;
  LaunchScope ls("ss_local", s);
  return launch_pdl(ss_local_kernel<NT, CAP>, (unsigned)((p.max_buckets + 1) / 2), NT,
                    sizeof(LocalShared<NT, CAP>), s, p);
}

cudaError_t launch_sample_dedup(recis_batch* b, recis_table* t, const int64_t* keys, int64_t N,
                                bool insert, cudaStream_t s) {
  SsParams p;
  p.keys = keys;
  p.N = N;
  p.splits = samplesort_splits_for(N);
  p.nsample = sample_size_for(N);
  p.tiles = (int)samplesort_tiles_for(N);
  p.max_buckets = 2 * (p.splits - 1) + 1;
  p.ctl = b->ss;
  p.th = b->ss_th;
  p.bkt = reinterpret_cast<uint16_t*>(b->vbuf[1]);
  p.kb = b->kbuf[0];
  p.vb = b->vbuf[0];
  p.pocc = reinterpret_cast<int64_t*>(b->kbuf[1]);
  p.meta = b->ss_meta;
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
  p.spos = b->spos;
  p.seg_of = b->seg_of;
  p.svals = b->svals;
  p.seg_start = b->seg_start;
  p.bdev = b->bdev;
  p.long_chunks = b->long_chunks;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool rank_attr[64] = {false}, scatter_attr[64] = {false};
  const int nbp_max = (p.max_buckets + 31) & ~31;
  // splitters: quantiles of the previous call on this batch when its size was
  // comparable (batches of one training stream share their key
  // distribution), else a sorted sample of this call's keys.  A bulk insert
  // never reuses and leaves nothing to reuse: its key chunks may arrive
  // sorted, one key range after another, where old quantiles would put a
  // whole call into one bucket.
  const int cur = b->cand_parity;
  const bool reuse = !insert && b->cand_n > 0 && b->cand_n >= N / 2 && b->cand_n <= 2 * N;
  p.cand_next = b->ss->cand[cur ^ 1];
  if (reuse) {
    p.cand = b->ss->cand[cur];
    p.cand_step = 1;
  } else {
    p.cand = b->ss->samp;
    p.cand_step = p.nsample / p.splits;
    if ((e = set_smem(ss_rank_kernel, kMaxSample * (int)sizeof(uint64_t), rank_attr, dev)) != cudaSuccess)
      return e;
    LaunchScope ls("ss_rank", s);
    ss_rank_kernel<<<(unsigned)(p.nsample / 32), kRankThreads, p.nsample * sizeof(uint64_t), s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  b->cand_parity = cur ^ 1;
  b->cand_n = insert ? 0 : N;
  // IDMap probes of every occurrence on the side stream, beside the sort
  if ((e = cudaEventRecord(b->ev_pfork, s)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(b->side, b->ev_pfork, 0)) != cudaSuccess)
    return e;
  {
    LaunchScope ls("ss_probe", b->side);
    const int64_t per = kProbeThreads * kProbeItems;
    ss_probe_kernel<<<(unsigned)((N + per - 1) / per), kProbeThreads, 0, b->side>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = cudaEventRecord(b->ev_probe, b->side)) != cudaSuccess) return e;
  {
    LaunchScope ls("ss_count", s);
    if ((e = launch_pdl(ss_count_kernel, (unsigned)p.tiles, kCountThreads, 0, s, p)) != cudaSuccess) return e;
  }
  {
    LaunchScope ls("ss_tilescan", s);
    if ((e = launch_pdl(ss_tilescan_kernel, (unsigned)(nbp_max / 32), 1024, 0, s, p)) != cudaSuccess) return e;
  }
  {
    const int smem = (kCountThreads / 32) * nbp_max * (int)sizeof(unsigned);
    if ((e = set_smem(ss_scatter_kernel, smem, scatter_attr, dev)) != cudaSuccess) return e;
    LaunchScope ls("ss_scatter", s);
    if ((e = launch_pdl(ss_scatter_kernel, (unsigned)p.tiles, kCountThreads, smem, s, p)) != cudaSuccess) return e;
  }
  if ((e = cudaStreamWaitEvent(s, b->ev_probe, 0)) != cudaSuccess) return e;
  if (N <= 524288)
    e = launch_local<128, 2048>(p, dev, s);
  else
    e = launch_local<512, 4096>(p, dev, s);
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("ss_finish", s);
    if ((e = launch_pdl(ss_finish_kernel, (unsigned)((N + kSub - 1) / kSub), kFinThreads, 0, s, p)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace recis
