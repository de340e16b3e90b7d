// samplesort.cu -- dedup + IDMap find-or-insert for batches of up to
// kSampleSortMaxN keys (RecIS README, Key optimisations > Distributed
// optimisation: merged requests deduplicated; > Efficient dynamic embedding:
// IDMap first-level store, EmbeddingBlocks second-level store).
//
// It produces exactly what the radix-sort path (sort.cu + unique.cu) produces:
// unique keys ascending, inverse index, rows (new keys get rows in ascending
// key order), segment starts, the segment of each sorted position, the
// sorted position of each occurrence, and initialised new rows; besides,
// the marks and lists the backward uses (positions in long segments, chunks
// holding one, keys seen 2 to kShortSeg times).  The digit passes are
// replaced by short launches, none of which waits on another CTA:
//   ss_rank      (first call of a batch) a strided sample of 4096 or 8192
//                keys is sorted by ranking: every sample's rank is its count
//                of smaller samples (ties by position), over many CTAs.
//   ss_probe     (second stream, beside the three below) the IDMap
//                find-or-insert of every occurrence: a missing key claims a
//                free slot by CAS; its row is assigned by ss_finish.
//   ss_count     per tile of 2048 keys: up to 2047 (batches of at most
//                327680 keys) or 1023 distinct splitters from the sorted
//                sample or the previous call's quantiles, the bucket of every
//                key (key u goes to bucket 2r + [u == split[r]],
//                r = #splitters < u, so buckets are ordered by key and a key
//                equal to a splitter -- a hot key -- has a bucket of its
//                own), and the tile's bucket histogram.
//   ss_tilescan  per bucket, the exclusive prefix of the tile histograms (so
//                the scatter is stable); the last CTA scans the bucket totals
//                into bucket starts.
//   ss_scatter   moves (key, occurrence) into bucket order, stably.
//   ss_local     sorts every key-range bucket by (key, occurrence): one warp
//                per bucket (batches of at most 327680 keys: 64-bit words of
//                key and position in registers, up to 16 per lane), else one
//                CTA per bucket (up to 4 pairs per thread in registers, or
//                shared memory); an equality bucket holds one key, already
//                in occurrence order.  Heads (first position of each distinct
//                key) and new keys are numbered within the bucket and the
//                bucket counts summed within the CTA; the CTA totals are
//                scanned by the last CTA (one CTA per bucket) or by every
//                finish CTA (one warp per bucket: a few hundred totals).
//   ss_finish    a flat pass over the sorted positions writes every output and
//                initialises the new rows.
// A key-range bucket larger than shared memory (only for adversarial key
// orders) is sorted by the CTA network in global memory.
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

// (key, idx) of the lower position of a comparator keeps the smaller pair
__device__ __forceinline__ bool pair_less(uint64_t ka, uint32_t xa, uint64_t kb, uint32_t xb) {
  return ka < kb || (ka == kb && xa < xb);
}

// The same network on NT*E elements held in registers, element i = E*t + e
// in element e of thread t.  A comparator whose block (k for the first stage
// of a merge, 2d otherwise) fits in one thread is a register swap; one that
// fits in E*32 elements pairs lanes of a warp by shuffles (first stage: lane
// t ^ (k/E - 1), element E-1-e; otherwise lane t ^ (d/E), element e); the rest
// exchange through shared memory sk/sx (NT*E entries).  Ends with the sorted
// elements in sk/sx and a __syncthreads.
template <int NT, int E>
__device__ void reg_sort(uint64_t (&k)[E], uint32_t (&x)[E], uint64_t* sk, uint32_t* sx) {
  const int t = threadIdx.x, lane = t & 31;
#pragma unroll
  for (int kk = 2; kk <= NT * E; kk <<= 1) {
#pragma unroll
    for (int d = kk >> 1; d > 0; d >>= 1) {
      const bool mirror = d == (kk >> 1);
      const int span = mirror ? kk : 2 * d;
      if (span <= E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int f = mirror ? (e ^ (kk - 1)) : (e ^ d);
          if (f > e && pair_less(k[f], x[f], k[e], x[e])) {
            const uint64_t tk = k[e];
            const uint32_t tx = x[e];
            k[e] = k[f];
            x[e] = x[f];
            k[f] = tk;
            x[f] = tx;
          }
        }
      } else if (span <= 32 * E) {
        const int lm = mirror ? (kk / E - 1) : (d / E);
        // this lane holds the lower positions of its pairs
        const bool low = (lane & (mirror ? kk / (2 * E) : d / E)) == 0;
        uint64_t nk[E];
        uint32_t nx[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int send = mirror ? (E - 1 - e) : e;
          const uint64_t pk = __shfl_xor_sync(0xffffffffu, k[send], lm);
          const uint32_t px = __shfl_xor_sync(0xffffffffu, x[send], lm);
          const bool pl = pair_less(pk, px, k[e], x[e]);
          const bool take = low ? pl : !pl;
          nk[e] = take ? pk : k[e];
          nx[e] = take ? px : x[e];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
          k[e] = nk[e];
          x[e] = nx[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          sk[E * t + e] = k[e];
          sx[E * t + e] = x[e];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = E * t + e;
          const int j = mirror ? (i ^ (kk - 1)) : (i ^ d);
          const uint64_t pk = sk[j];
          const uint32_t px = sx[j];
          const bool pl = pair_less(pk, px, k[e], x[e]);
          const bool take = i < j ? pl : !pl;
          if (take) {
            k[e] = pk;
            x[e] = px;
          }
        }
        __syncthreads();
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    sk[E * t + e] = k[e];
    sx[E * t + e] = x[e];
  }
  __syncthreads();
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
  int local_bpc_shift;      // log2 of the buckets per CTA of the local kernel
  int local_ctas;           // CTAs of the local kernel
  int finish_scans;         // the finish kernel scans the local CTAs' totals
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
  int32_t* seg_start;
  BatchDev* bdev;
  int32_t* multi_keys;      // keys seen 2 to kShortSeg times (appended by ss_finish)
  DevState* st;
  HostMirror* mirror;
  uint32_t call_id;         // this lookup's number on the batch (BatchDev::reject_call)
  int admit;                // admission threshold (>= 1)
  uint64_t clock;           // this lookup's clock
  uint32_t* seen;           // [row] clock of the last lookup that touched the row, or null
  const int32_t* free_rows; // queue of freed rows (bdev->free_base .. + free_avail)
};

// New rows a call takes past the table's end: its new keys beyond the freed
// rows it reuses.
__device__ __forceinline__ unsigned long long fresh_rows(unsigned long long nnew, unsigned long long avail) {
  return nnew > avail ? nnew - avail : 0ULL;
}

// A lookup is rejected as a whole when one of its keys is the reserved -1
// (marked by the probe kernel) or when its new keys would not fit the mapped
// row space: then no key is inserted (the slots its probes claimed are given
// back), no row is created, and U = 0, so the matching backward updates no row.
__device__ __forceinline__ bool call_rejected(const SsParams& p, unsigned long long tot,
                                              unsigned long long row_base) {
  return __ldcg(&p.bdev->reject_call) == p.call_id ||
         row_base + fresh_rows(tot >> 32, p.bdev->free_avail) > (unsigned long long)p.mapped_rows;
}

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
  // splitters: up to 8 candidates per thread, in order
  const int S = p.splits - 1, step = p.cand_step;
  constexpr int kCand = kMaxSplitters / kCountThreads;  // 8
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
    p.bdev->nseg_med = 0;  // the backward's long-segment lists start empty
    p.bdev->nseg_huge = 0;
    p.bdev->seg_work = 0;
    p.bdev->nmulti = 0;
    p.bdev->row_base = *(volatile unsigned long long*)&p.st->next_free;
    const unsigned long long fh = *(volatile unsigned long long*)&p.st->free_head;
    p.bdev->free_base = fh;
    p.bdev->free_avail = *(volatile unsigned long long*)&p.st->free_tail - fh;
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
// occurrence of a key without a row records its slot and whether this call
// admits it (the count of lookups it appeared in reaches the threshold).  All
// occurrences of a key see the same slot state, so they agree.  Claims are
// counted per CTA and added to the table's slot count once.
constexpr int kProbeThreads = 256;
constexpr int kProbeItems = 2;
__global__ void __launch_bounds__(kProbeThreads) ss_probe_kernel(const __grid_constant__ SsParams p) {
  __shared__ unsigned s_claims;
  if (threadIdx.x == 0) s_claims = 0;
  __syncthreads();
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
      const Probe pr = idmap_probe(p.slots, p.slot_mask, k[j], h[j], sv[j], true, &s_claims);
      if (pr.limit) raise_error(p.st, p.mirror, kErrTableFull);
      else if (pr.row >= 0) r = pr.row;
      else r = pr.prior + 1 >= p.admit ? -2 - pr.slot : kCandPocc - pr.slot;
    }
    p.pocc[pos] = r;
  }
  if (reserved) {
    p.bdev->reject_call = p.call_id;
    raise_error(p.st, p.mirror, kErrReservedKey);
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_claims) atomicAdd(&p.st->slots_used, (unsigned long long)s_claims);
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
  // bucket starts: consecutive buckets per thread
  constexpr int PER = kMaxBucketSlots / 1024;
  const int nb = (int)p.ctl->nb;
  unsigned c[PER], own = 0;
#pragma unroll
  for (int h = 0; h < PER; ++h) {
    const int b = PER * tid + h;
    c[h] = b < nb ? __ldcg(&p.ctl->tot[b]) : 0u;
    own += c[h];
  }
  unsigned total;
  unsigned ex = block_excl_scan<1024>(own, s_warp, &total);
#pragma unroll
  for (int h = 0; h < PER; ++h) {
    const int b = PER * tid + h;
    if (b < nb) p.ctl->base[b] = ex;
    ex += c[h];
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ scatter
// Stable move of (ukey, occurrence) into bucket order.  Within a tile, warp w
// holds keys w*256 .. w*256+255 (item j of lane l is key w*256 + 32j + l);
// ranks within a warp come from the lanes sharing a bucket (ballots on its
// bits) over the items in order, ranks
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
  // lanes holding the same bucket: 12 ballots on the bucket's bits (buckets
  // are below 4095; a missing key takes 4095), all items first
  unsigned peers[kCountItems];
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const unsigned bb = b[j] != 0xffffffffu ? b[j] : 4095u;
    unsigned pm = 0xffffffffu;
#pragma unroll
    for (int q = 0; q < 12; ++q) {
      const unsigned bal = __ballot_sync(0xffffffffu, (bb >> q) & 1u);
      pm &= ((bb >> q) & 1u) ? bal : ~bal;
    }
    peers[j] = pm;
  }
#pragma unroll
  for (int j = 0; j < kCountItems; ++j) {
    const int leader = __ffs(peers[j]) - 1;
    const unsigned before = b[j] != 0xffffffffu ? mine[b[j]] : 0u;
    rank[j] = before + __popc(peers[j] & lt);
    __syncwarp();
    if (lane == leader && b[j] != 0xffffffffu) mine[b[j]] = before + __popc(peers[j]);
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

// Sort a bucket of up to NT*E keys in registers (positions past m are
// padded with the largest pair); leaves it in sk/sx.
template <int NT, int E>
__device__ void reg_load_sort(const SsParams& p, uint64_t* sk, uint32_t* sx, int64_t m, int64_t off) {
  uint64_t k[E];
  uint32_t x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = E * (int)threadIdx.x + e;
    k[e] = i < m ? __ldcg(p.kb + off + i) : ~0ULL;
    x[e] = i < m ? __ldcg(p.vb + off + i) : ~0u;
  }
  reg_sort<NT, E>(k, x, sk, sx);
}

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
        f = 1u | (pocc_new(__ldcg(p.pocc + occ)) ? 2u : 0u);
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

// Equality bucket b (one key, m > 0 positions, already in occurrence order
// from the stable scatter; isnew: the key was claimed by this call): one
// segment, numbered by threads first, first + stride, ...; `first == 0` also
// writes the bucket's counts.
__device__ __forceinline__ void local_equal(const SsParams& p, unsigned b, int64_t m, int64_t off,
                                            bool isnew, int first, int stride) {
  const uint64_t lng = m > kShortSeg ? kMetaLong : 0ULL;
  for (int64_t i = first; i < m; i += stride)
    p.meta[off + i] = pack_meta(b, 1u, isnew ? 1u : 0u, i == 0, i == 0 && isnew) | lng;
  if (first == 0) {
    p.ctl->hcnt[b] = 1;
    p.ctl->ncnt[b] = isnew ? 1u : 0u;
  }
}

// Key-range bucket b (m > 0) by the whole CTA: sorted by (key, occurrence) in
// registers (up to 4 keys per thread), in shared memory, or in global memory
// for an oversized one (adversarial key orders), then numbered.
template <int NT, int CAP>
__device__ void local_range_block(const SsParams& p, LocalShared<NT, CAP>& sh, unsigned b, int64_t m,
                                  int64_t off) {
  const int tid = threadIdx.x;
  if (m <= NT * 4) {
    if (m <= NT * 2) reg_load_sort<NT, 2>(p, sh.key, sh.idx, m, off);
    else reg_load_sort<NT, 4>(p, sh.key, sh.idx, m, off);
    block_number<NT, CAP>(p, sh, b, m, off, true);
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
}

// Bucket prefixes, first level: every local CTA turns the counts of its BPC
// buckets into prefixes within the CTA and publishes its total.  The finish
// kernel scans the CTA totals; a bucket's place is then the CTA prefix plus
// hpre[b] (heads), and the same for new keys.  Called by every thread after
// its CTA's buckets are written.
template <int BPC>
__device__ __forceinline__ void local_publish(const SsParams& p) {
  if (threadIdx.x != 0) return;
  const unsigned nb = p.ctl->nb;
  const unsigned b0 = blockIdx.x * BPC;
  unsigned long long v[BPC], run = 0;
#pragma unroll
  for (int j = 0; j < BPC; ++j) {
    const unsigned b = b0 + j;
    v[j] = b < nb ? ((unsigned long long)__ldcg(&p.ctl->ncnt[b]) << 32) | __ldcg(&p.ctl->hcnt[b]) : 0ULL;
  }
#pragma unroll
  for (int j = 0; j < BPC; ++j) {
    if (b0 + j < nb) {
      p.ctl->hpre[b0 + j] = (unsigned)(run & 0xffffffffULL);
      p.ctl->npre[b0 + j] = (unsigned)(run >> 32);
    }
    run += v[j];
  }
  p.ctl->cta_tot[blockIdx.x] = run;
}

// The call's totals (tot = new keys << 32 | heads), published by one thread;
// a rejected call publishes U = 0 and no new rows, and marks the batch.
__device__ __forceinline__ void publish_totals(const SsParams& p, unsigned long long tot,
                                               unsigned long long row_base) {
  const unsigned long long U = tot & 0xffffffffULL;
  unsigned long long nnew = tot >> 32;
  const bool rejected = call_rejected(p, tot, row_base);
  if (rejected) {
    if (__ldcg(&p.bdev->reject_call) != p.call_id) raise_error(p.st, p.mirror, kErrTableFull);
    p.bdev->reject_call = p.call_id;
    nnew = 0;
  }
  p.bdev->U = rejected ? 0u : (unsigned)U;
  p.bdev->n_new = (unsigned)nnew;
  // new keys take the queued freed rows first, then rows past the end
  const unsigned long long avail = p.bdev->free_avail;
  const unsigned long long nf = row_base + fresh_rows(nnew, avail);
  p.st->next_free = nf;
  p.st->free_head = p.bdev->free_base + (nnew < avail ? nnew : avail);
  if (p.mirror) {
    p.mirror->next_free = nf;
    p.mirror->slots_used = *(volatile unsigned long long*)&p.st->slots_used;
    __threadfence_system();
  }
  p.seg_start[U] = (int32_t)p.N;
}

// Exclusive scan of the local CTAs' totals by one block of NT threads
// (thread t owns per consecutive ones); dst(i, prefix) receives each prefix.
// Returns the grand total.
template <int NT, typename Dst>
__device__ __forceinline__ unsigned long long scan_cta_totals(const SsParams& p, unsigned long long* s_warp,
                                                              Dst dst) {
  constexpr int kPer = (kMaxBucketSlots / 2 + NT - 1) / NT;
  const int tid = threadIdx.x;
  const int G = p.local_ctas;
  const int per = (G + NT - 1) / NT;
  unsigned long long v[kPer], own = 0;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int i = tid * per + r;
    v[r] = (r < per && i < G) ? __ldcg(&p.ctl->cta_tot[i]) : 0ULL;
    own += v[r];
  }
  unsigned long long tot;
  unsigned long long ex = block_excl_scan2<NT>(own, s_warp, &tot);
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int i = tid * per + r;
    if (r < per && i < G) dst(i, ex);
    ex += v[r];
  }
  return tot;
}

// One CTA per key-range bucket and the equality bucket after it (larger
// batches, whose buckets hold hundreds to thousands of keys).
template <int NT, int CAP>
__global__ void __launch_bounds__(NT, NT >= 512 ? 2 : 4) ss_local_kernel(const __grid_constant__ SsParams p) {
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
      local_equal(p, b, m, off, pocc_new(__ldcg(p.pocc + __ldcg(p.vb + off))), tid, NT);
    } else {
      local_range_block<NT, CAP>(p, sh, b, m, off);
    }
    __syncthreads();
  }
  local_publish<2>(p);
  // the last CTA to finish scans the CTA totals (the finish kernel reads
  // the prefixes per position)
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(&p.ctl->ticket_local, 1u) == gridDim.x - 1;
  __syncthreads();
  if (sh.last) {
    __threadfence();
    const unsigned long long tot =
        scan_cta_totals<NT>(p, sh.warp, [&](int i, unsigned long long v) { p.ctl->cta_pre[i] = v; });
    if (tid == 0) publish_totals(p, tot, p.bdev->row_base);
  }
  pdl_trigger();
}

// ------------------------------------------------------------------ local, one warp per bucket
// For batches of up to kLocalWarpMaxN keys (2047 splitters: key-range
// buckets of about 100 keys), one warp sorts and numbers one bucket.  A bucket of m <= 32E keys (E = 4, 8 or 16 per lane)
// whose keys span less than 2^55 is sorted as single 64-bit words
// (u - min) << log2(32E) | position: the positions are distinct and in
// occurrence order (stable scatter), so the word order is the (key,
// occurrence) order.  Lane l holds positions E*l .. E*l+E-1; the network is
// the one of reg_sort on one warp.
constexpr int64_t kLocalWarpMaxN = 327680;  // batches whose buckets go one per warp
constexpr int kLocalWarps = 4;
constexpr int kLocalWarpThreads = 32 * kLocalWarps;
constexpr int kWarpSortMax = 512;

template <int CAP>
struct LocalWarpShared {
  LocalShared<kLocalWarpThreads, CAP> blk;        // buckets left to the whole CTA
  uint32_t idx[kLocalWarps][kWarpSortMax];        // occurrence of every bucket position
  uint8_t hl[kLocalWarps][kWarpSortMax];          // per bucket-local segment: long
  unsigned fallback;                              // bit w: warp w left its bucket to the CTA
};

__device__ __forceinline__ uint64_t u64_min(uint64_t a, uint64_t b) { return a < b ? a : b; }
__device__ __forceinline__ uint64_t u64_max(uint64_t a, uint64_t b) { return a < b ? b : a; }

template <int E>
__device__ __forceinline__ void warp_sort_unrolled(uint64_t (&c)[E]) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 2; kk <= 32 * E; kk <<= 1) {
#pragma unroll
    for (int d = kk >> 1; d > 0; d >>= 1) {
      const bool mirror = d == (kk >> 1);
      if ((mirror ? kk : 2 * d) <= E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int f = mirror ? (e ^ (kk - 1)) : (e ^ d);
          if (f > e) {
            const uint64_t lo = u64_min(c[e], c[f]), hi = u64_max(c[e], c[f]);
            c[e] = lo;
            c[f] = hi;
          }
        }
      } else if (mirror) {
        // lane ^ (kk/E - 1): my element e meets its element E-1-e
        const int lm = kk / E - 1;
        const bool low = (lane & (kk / (2 * E))) == 0;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          const uint64_t a = __shfl_xor_sync(kFull, c[E - 1 - e], lm);
          const uint64_t b = __shfl_xor_sync(kFull, c[e], lm);
          c[e] = low ? u64_min(c[e], a) : u64_max(c[e], a);
          c[E - 1 - e] = low ? u64_min(c[E - 1 - e], b) : u64_max(c[E - 1 - e], b);
        }
      } else {
        const int lm = d / E;
        const bool low = (lane & lm) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint64_t a = __shfl_xor_sync(kFull, c[e], lm);
          c[e] = low ? u64_min(c[e], a) : u64_max(c[e], a);
        }
      }
    }
  }
}

// one stage whose comparators lie inside a thread: partner e ^ (V-1) (first
// stage of a merge of V) or e ^ V
template <int E, bool MIRROR, int V>
__device__ __forceinline__ void thread_stage(uint64_t (&c)[E]) {
  if constexpr ((MIRROR ? V : 2 * V) <= E) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int f = MIRROR ? (e ^ (V - 1)) : (e ^ V);
      if (f > e) {
        const uint64_t lo = u64_min(c[e], c[f]), hi = u64_max(c[e], c[f]);
        c[e] = lo;
        c[f] = hi;
      }
    }
  }
}

// The same network with its stages in a loop (compact code for the rare
// buckets of up to 512 keys)
template <int E>
__device__ void warp_sort_loop(uint64_t (&c)[E]) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  for (int kk = 2; kk <= 32 * E; kk <<= 1) {
    for (int d = kk >> 1; d > 0; d >>= 1) {
      const bool mirror = d == (kk >> 1);
      if ((mirror ? kk : 2 * d) <= E) {
        if (mirror) {
          switch (kk) {
            case 2: thread_stage<E, true, 2>(c); break;
            case 4: thread_stage<E, true, 4>(c); break;
            case 8: thread_stage<E, true, 8>(c); break;
            default: thread_stage<E, true, 16>(c); break;
          }
        } else {
          switch (d) {
            case 1: thread_stage<E, false, 1>(c); break;
            case 2: thread_stage<E, false, 2>(c); break;
            case 4: thread_stage<E, false, 4>(c); break;
            default: thread_stage<E, false, 8>(c); break;
          }
        }
      } else if (mirror) {
        const int lm = kk / E - 1;
        const bool low = (lane & (kk / (2 * E))) == 0;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          const uint64_t a = __shfl_xor_sync(kFull, c[E - 1 - e], lm);
          const uint64_t b = __shfl_xor_sync(kFull, c[e], lm);
          c[e] = low ? u64_min(c[e], a) : u64_max(c[e], a);
          c[E - 1 - e] = low ? u64_min(c[E - 1 - e], b) : u64_max(c[E - 1 - e], b);
        }
      } else {
        const int lm = d / E;
        const bool low = (lane & lm) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint64_t a = __shfl_xor_sync(kFull, c[e], lm);
          c[e] = low ? u64_min(c[e], a) : u64_max(c[e], a);
        }
      }
    }
  }
}

template <int E>
__device__ __forceinline__ void warp_sort(uint64_t (&c)[E]) {
  if constexpr (E <= 8) warp_sort_unrolled<E>(c);
  else warp_sort_loop<E>(c);
}

// Key-range bucket b (0 < m <= 32E) by one warp: sort, number heads and new
// keys, write the sorted keys, occurrences and meta.  Returns false, having
// written nothing, when the bucket's keys span 2^55 or more.  *extra (when
// not null) is loaded into extra_val together with the heads' IDMap results.
template <int E>
__device__ bool local_range_warp(const SsParams& p, unsigned b, int m, int64_t off, uint32_t* widx,
                                 uint8_t* whl, const int64_t* extra, int64_t& extra_val) {
  constexpr unsigned kFull = 0xffffffffu;
  constexpr int PB = E == 4 ? 7 : (E == 8 ? 8 : 9);  // position bits
  static_assert((32 * E) == (1 << PB), "one position per low bit pattern");
  const int lane = threadIdx.x & 31;
  uint64_t c[E];
  uint64_t lo = ~0ULL, hi = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = E * lane + e;
    c[e] = 0;
    if (i < m) {
      c[e] = __ldcg(p.kb + off + i);
      widx[i] = __ldcg(p.vb + off + i);
      lo = u64_min(lo, c[e]);
      hi = u64_max(hi, c[e]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = u64_min(lo, __shfl_xor_sync(kFull, lo, o));
    hi = u64_max(hi, __shfl_xor_sync(kFull, hi, o));
  }
  if (hi - lo >= (1ULL << 55)) return false;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = E * lane + e;
    c[e] = i < m ? ((c[e] - lo) << PB) | (uint64_t)i : ~0ULL;
  }
  warp_sort<E>(c);
  __syncwarp();
  // heads (first position of a key), new keys, and long segments (the key 16
  // positions after the head is the same)
  const uint64_t before = __shfl_up_sync(kFull, c[E - 1] >> PB, 1);
  uint32_t occ[E];
  unsigned hmask = 0, nmask = 0, lmask = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = E * lane + e;
    const uint64_t rel = c[e] >> PB;
    const uint64_t after16 = __shfl_down_sync(kFull, rel, kShortSeg / E);
    occ[e] = i < m ? widx[c[e] & ((1u << PB) - 1u)] : 0u;
    const uint64_t prev = e == 0 ? before : (c[e - 1] >> PB);
    if (i < m && (i == 0 || rel != prev)) {
      hmask |= 1u << e;
      if (i + kShortSeg < m && after16 == rel) lmask |= 1u << e;
    }
  }
  // the IDMap results of the heads (and the caller's extra one), all in
  // flight at once
  int64_t pv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) pv[e] = ((hmask >> e) & 1u) ? __ldcg(p.pocc + occ[e]) : 0;
  if (extra) extra_val = __ldcg(extra);
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (pocc_new(pv[e])) nmask |= 1u << e;
  const unsigned long long own = ((unsigned long long)__popc(nmask) << 32) | (unsigned)__popc(hmask);
  unsigned long long y = own;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long z = __shfl_up_sync(kFull, y, o);
    if (lane >= o) y += z;
  }
  const unsigned long long total = __shfl_sync(kFull, y, 31);
  const unsigned lh0 = (unsigned)((y - own) & 0xffffffffULL), ln0 = (unsigned)((y - own) >> 32);
  unsigned lh = lh0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    lh += (hmask >> e) & 1u;
    if ((hmask >> e) & 1u) whl[lh - 1] = (uint8_t)((lmask >> e) & 1u);
  }
  __syncwarp();
  lh = lh0;
  unsigned ln = ln0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = E * lane + e;
    lh += (hmask >> e) & 1u;
    ln += (nmask >> e) & 1u;
    if (i < m) {
      p.kb[off + i] = lo + (c[e] >> PB);
      p.vb[off + i] = occ[e];
      p.meta[off + i] = pack_meta(b, lh, ln, (hmask >> e) & 1u, (nmask >> e) & 1u) |
                        (whl[lh - 1] ? kMetaLong : 0ULL);
    }
  }
  if (lane == 0) {
    p.ctl->hcnt[b] = (unsigned)(total & 0xffffffffULL);
    p.ctl->ncnt[b] = (unsigned)(total >> 32);
  }
  return true;
}

// Warp w of CTA c: key-range bucket 2q and equality bucket 2q+1 of pair
// q = 4c + w.  Key-range buckets too large (over 512 keys) or too wide for
// one warp are then done by the whole CTA, one after another.
template <int CAP>
__global__ void __launch_bounds__(kLocalWarpThreads) ss_local_warp_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  extern __shared__ __align__(16) unsigned char s_raw[];
  LocalWarpShared<CAP>& sh = *reinterpret_cast<LocalWarpShared<CAP>*>(s_raw);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned nb = p.ctl->nb;
  if (tid == 0) sh.fallback = 0;
  __syncthreads();
  const unsigned q = kLocalWarps * blockIdx.x + w;
  // both buckets' sizes and starts, and the equality bucket's first
  // occurrence, are loaded at once (the control arrays hold every slot)
  const unsigned br = 2 * q, be = 2 * q + 1;
  const bool has_r = br < nb, has_e = be < nb;
  const int64_t mr = (int64_t)__ldcg(&p.ctl->tot[br]), offr = (int64_t)__ldcg(&p.ctl->base[br]);
  const int64_t me = (int64_t)__ldcg(&p.ctl->tot[be]), offe = (int64_t)__ldcg(&p.ctl->base[be]);
  const bool eq = has_e && me > 0;
  const int64_t* eq_pocc = eq ? p.pocc + __ldcg(p.vb + offe) : nullptr;
  int64_t eq_val = 0;
  bool eq_loaded = false;
  if (has_r && mr == 0) {
    if (lane == 0) {
      p.ctl->hcnt[br] = 0;
      p.ctl->ncnt[br] = 0;
    }
  } else if (has_r) {
    bool done = false;
    if (mr <= 128)
      done = local_range_warp<4>(p, br, (int)mr, offr, sh.idx[w], sh.hl[w], eq_pocc, eq_val);
    else if (mr <= 256)
      done = local_range_warp<8>(p, br, (int)mr, offr, sh.idx[w], sh.hl[w], eq_pocc, eq_val);
    else if (mr <= 512)
      done = local_range_warp<16>(p, br, (int)mr, offr, sh.idx[w], sh.hl[w], eq_pocc, eq_val);
    eq_loaded = done;
    if (!done && lane == 0) atomicOr(&sh.fallback, 1u << w);
  }
  if (eq) {
    if (!eq_loaded) eq_val = __ldcg(eq_pocc);
    local_equal(p, be, me, offe, pocc_new(eq_val), lane, 32);
  } else if (has_e && lane == 0) {
    p.ctl->hcnt[be] = 0;
    p.ctl->ncnt[be] = 0;
  }
  __syncthreads();
  for (unsigned fb = sh.fallback; fb; fb &= fb - 1) {
    const unsigned b = 2 * (kLocalWarps * blockIdx.x + (unsigned)(__ffs(fb) - 1));
    local_range_block<kLocalWarpThreads, CAP>(p, sh.blk, b, (int64_t)p.ctl->tot[b],
                                              (int64_t)p.ctl->base[b]);
    __syncthreads();
  }
  local_publish<2 * kLocalWarps>(p);
  pdl_trigger();
}

// ------------------------------------------------------------------ finish
struct FinishShared {
  int64_t init_key[kFinThreads * kFinItems];
  int32_t init_row[kFinThreads * kFinItems];
  unsigned long long cpre[kMaxBucketSlots / 2];  // per local CTA: new keys << 32 | heads before it
  unsigned long long warp[kFinThreads / 32];
  int ninit;
  unsigned heads[kSub / 32];        // bit i: position i of this CTA is a head
  int32_t multi[kSub / 2];          // keys of this CTA seen 2 to kShortSeg times
  int nmulti;
  unsigned multi_base;
};
static_assert(kSub / kShortSeg <= 32, "one bit per chunk of a finish CTA");

// Flat pass over the sorted positions, kSub per CTA (position blk*kSub +
// j*256 + t for item j of thread t): segment of every position from its
// bucket's prefix, all outputs, and the initialisation of the new rows.
__global__ void __launch_bounds__(kFinThreads, 3) ss_finish_kernel(const __grid_constant__ SsParams p) {
  pdl_wait();
  __shared__ FinishShared sh;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) {
    sh.ninit = 0;
    sh.nmulti = 0;
  }
  __syncthreads();
  const int64_t q0 = (int64_t)blockIdx.x * kSub + tid;
  const uint64_t row_base = p.bdev->row_base;
  unsigned sh_unclaim = 0;  // slots this thread gave back (a rejected call)
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
  // second level of the bucket prefixes, after the one-warp local kernel:
  // every CTA scans the local CTAs' totals and CTA 0 publishes the call's
  // totals (after the CTA local kernel its last CTA did both)
  bool rejected;
  if (p.finish_scans) {
    const unsigned long long tot = scan_cta_totals<kFinThreads>(
        p, sh.warp, [&](int i, unsigned long long v) { sh.cpre[i] = v; });
    rejected = call_rejected(p, tot, row_base);
    if (blockIdx.x == 0 && tid == 0) publish_totals(p, tot, row_base);
  } else {
    rejected = __ldcg(&p.bdev->reject_call) == p.call_id;  // published by the local kernel
  }
  // head bits of this CTA's positions (position j*kFinThreads + 32w + lane)
#pragma unroll
  for (int j = 0; j < kFinItems; ++j) {
    const int64_t q = q0 + j * kFinThreads;
    const unsigned hb = __ballot_sync(0xffffffffu, q < p.N && ((mt[j] >> 43) & 1u));
    if (lane == 0) sh.heads[(j * kFinThreads) / 32 + w] = hb;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kFinItems; ++j) {
    const int64_t q = q0 + j * kFinThreads;
    if (q >= p.N) break;
    const uint64_t m = mt[j];
    const unsigned b = (unsigned)(m >> 44) & 0xfffu;
    const unsigned lh = (unsigned)(m & 0x1fffffULL);
    const unsigned long long cpre = p.finish_scans ? sh.cpre[b >> p.local_bpc_shift]
                                                   : __ldg(&p.ctl->cta_pre[b >> p.local_bpc_shift]);
    const unsigned seg = (unsigned)(cpre & 0xffffffffULL) + __ldg(&p.ctl->hpre[b]) + lh - 1u;
    p.seg_of[q] = (int32_t)seg;
    if (occ[j] < (uint32_t)p.N) {
      p.inv[occ[j]] = (int32_t)seg;
      p.spos[occ[j]] = (uint32_t)q;
    }
    if ((m >> 43) & 1u) {
      const int64_t key = from_ukey(__ldcs(p.kb + q));
      int64_t row = __ldcg(p.pocc + occ[j]);
      if ((m >> 42) & 1u) {
        // admitted by this call: the k-th new key (ascending key order) takes
        // the k-th queued freed row, or a row past the end
        const int64_t slot = -2 - row;
        const unsigned ln = (unsigned)((m >> 21) & 0x1fffffULL);
        const unsigned long long k = (cpre >> 32) + __ldg(&p.ctl->npre[b]) + ln - 1u;
        const unsigned long long avail = p.bdev->free_avail;
        row = k < avail ? (int64_t)__ldg(p.free_rows + p.bdev->free_base + k)
                        : (int64_t)(row_base + (k - avail));
        if (rejected) {
          sh_unclaim += idmap_give_back(p.slots, slot);
          row = -1;
        } else if (row >= p.mapped_rows) {
          raise_error(p.st, p.mirror, kErrTableFull);
          row = -1;
        } else {
          p.slots[slot].row = row;
          p.row_keys[row] = key;
          if (p.seen) p.seen[row] = (uint32_t)p.clock;
          const int at = atomicAdd(&sh.ninit, 1);
          sh.init_key[at] = key;
          sh.init_row[at] = (int32_t)row;
        }
      } else if (pocc_cand(row)) {
        // stays a candidate: one more lookup counted, at this clock
        const int64_t slot = kCandPocc - row;
        if (rejected) sh_unclaim += idmap_give_back(p.slots, slot);
        else p.slots[slot].row = cand_row(p.clock, prior_count(__ldcg(&p.slots[slot].row)) + 1);
        row = -1;
      } else if (row >= 0 && p.seen && !rejected) {
        p.seen[row] = (uint32_t)p.clock;
      }
      p.uniq[seg] = key;
      p.rows[seg] = row;
      p.seg_start[seg] = (int32_t)q;
      // a short segment (not long) whose next position is no head holds 2 to
      // kShortSeg occurrences: listed for the row update
      if (p.multi_keys && !rejected && !(m >> 63)) {
        const int i = tid + j * kFinThreads + 1;  // next position within this CTA
        bool next_head;
        if (q + 1 >= p.N) next_head = true;
        else if (i < kSub) next_head = (sh.heads[i >> 5] >> (i & 31)) & 1u;
        else next_head = (__ldcs(p.meta + q + 1) >> 43) & 1u;
        if (!next_head) sh.multi[atomicAdd(&sh.nmulti, 1)] = (int32_t)seg;
      }
    }
  }
  if (sh_unclaim) atomicAdd(&p.st->slots_used, (unsigned long long)(0ULL - sh_unclaim));
  // this CTA's keys seen 2 to kShortSeg times, for the backward's row update
  __syncthreads();
  if (tid == 0 && sh.nmulti > 0) sh.multi_base = atomicAdd(&p.bdev->nmulti, (unsigned)sh.nmulti);
  __syncthreads();
  for (int i = tid; i < sh.nmulti; i += kFinThreads) p.multi_keys[sh.multi_base + i] = sh.multi[i];
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
// splitter slots: key-range buckets of about 100 keys for batches the
// one-warp local sort takes, else about N / 1023
int samplesort_splits_for(int64_t N) { return N <= kLocalWarpMaxN ? 2048 : 1024; }

int64_t samplesort_tiles_for(int64_t N) { return (N + kTile - 1) / kTile; }

// sample of the first call: at least two keys per splitter slot
static int sample_size_for(int64_t N) {
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
  return launch_pdl(ss_local_kernel<NT, CAP>, (unsigned)p.local_ctas, NT, sizeof(LocalShared<NT, CAP>), s,
                    p);
}

template <int CAP>
static cudaError_t launch_local_warp(const SsParams& p, int dev, cudaStream_t s) {
  static bool attr[64] = {false};
  cudaError_t e = set_smem(ss_local_warp_kernel<CAP>, (int)sizeof(LocalWarpShared<CAP>), attr, dev);
  if (e != cudaSuccess) return e;
  LaunchScope ls("ss_local", s);
  return launch_pdl(ss_local_warp_kernel<CAP>, (unsigned)p.local_ctas, kLocalWarpThreads,
                    sizeof(LocalWarpShared<CAP>), s, p);
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
  static_assert(2 * kLocalWarps == 8, "buckets per CTA of the one-warp local kernel");
  p.local_bpc_shift = N <= kLocalWarpMaxN ? 3 : 1;  // 8 or 2 buckets per local CTA
  p.local_ctas = (p.max_buckets + 1) / 2;            // bucket pairs
  if (N <= kLocalWarpMaxN) p.local_ctas = (p.local_ctas + kLocalWarps - 1) / kLocalWarps;
  p.finish_scans = N <= kLocalWarpMaxN ? 1 : 0;
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
  p.seg_start = b->seg_start;
  p.bdev = b->bdev;
  p.multi_keys = b->multi_keys;
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  p.call_id = b->call_seq;
  // a bulk insert pre-loads: its keys are admitted at once
  p.admit = (!insert && t->cfg.admit_threshold > 1) ? t->cfg.admit_threshold : 1;
  p.clock = (uint64_t)t->clock;
  p.seen = t->cfg.evictable ? reinterpret_cast<uint32_t*>(t->seen.va) : nullptr;
  p.free_rows = t->free_rows;

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
  // The previous quantiles serve when they are at least as many as this
  // call's splitters (every (prev / splits)-th of them).
  const int cur = b->cand_parity;
  const bool reuse = !insert && b->cand_n > 0 && b->cand_n >= N / 2 && b->cand_n <= 2 * N &&
                     b->cand_splits >= p.splits;
  p.cand_next = b->ss->cand[cur ^ 1];
  if (reuse) {
    p.cand = b->ss->cand[cur];
    p.cand_step = b->cand_splits / p.splits;
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
  b->cand_splits = p.splits;
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
    if ((e = set_smem(ss_scatter_kernel, (kCountThreads / 32) * kMaxBucketSlots * (int)sizeof(unsigned),
                      scatter_attr, dev)) != cudaSuccess)
      return e;
    LaunchScope ls("ss_scatter", s);
    if ((e = launch_pdl(ss_scatter_kernel, (unsigned)p.tiles, kCountThreads, smem, s, p)) != cudaSuccess) return e;
  }
  if ((e = cudaStreamWaitEvent(s, b->ev_probe, 0)) != cudaSuccess) return e;
  if (N <= kLocalWarpMaxN)
    e = launch_local_warp<2048>(p, dev, s);
  else if (N <= 524288)
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
