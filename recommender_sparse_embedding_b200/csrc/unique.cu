// unique.cu -- the second half of the dedup step fused with the IDMap
// find-or-insert and the initialisation of new rows (RecIS README, Key
// optimisations > Efficient dynamic embedding: IDMap = first-level store,
// feature ID -> offset; EmbeddingBlocks = second-level store of parameters and
// optimiser state).
//
// One pass over the sorted (key, occurrence) pairs, 1024 positions per tile:
//   1. head flags (first position of each distinct key);
//   2. each head probes the IDMap (open addressing, linear probing, 16-byte
//      slots {key, row}); a missing key is claimed with a 64-bit CAS;
//   3. the tile publishes (heads, new keys) and resolves its prefix by
//      decoupled look-back, which numbers the unique keys in ascending order
//      and gives new keys consecutive rows in ascending key order after the
//      table's live rows;
//   4. writes uniq / rows / segment starts / inverse index, the row of each
//      new slot and the key of each new row, and initialises the new rows
//      (seeded hash of the key; optimiser state at its initial value).
// The last tile publishes U, the new-key count and the table's next free row.
#include "internal.h"

namespace recis {

namespace {

constexpr int kUqBlock = 256, kUqItems = 4, kUqTile = kUqBlock * kUqItems;
constexpr int kHpItems = 2;  // sorted positions per thread of the head probe (4 or 8 measured slower)
constexpr unsigned long long kUqAgg = 1ULL << 62, kUqIncl = 2ULL << 62;

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

}  // namespace

struct UniqueParams {
  const int64_t* in_keys;
  const uint64_t* kb0;
  const uint64_t* kb1;
  const uint32_t* vb0;
  const uint32_t* vb1;
  int64_t N;
  SortCtl* ctl;
  unsigned long long* lookback;
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
  int64_t* uniq;
  int64_t* rows;
  int32_t* inv;
  uint32_t* spos;           // [N] sorted position of each occurrence
  int32_t* seg_of;
  int32_t* seg_start;
  BatchDev* bdev;
  DevState* st;
  HostMirror* mirror;
  uint32_t call_id;
  int spin_max;             // polls before a look-back wait gives up
  int admit;                // admission threshold (>= 1)
  uint64_t clock;           // this lookup's clock
  uint32_t* seen;           // [row] last-lookup clock of each row, or null
  const int32_t* free_rows; // queue of freed rows (bdev->free_base .. + free_avail)
  int64_t* pocc;            // [N] IDMap result of each head, at its sorted position
};

// IDMap find-or-insert of every head (first position of a key) of the
// sorted keys, with admission, before the unique pass: the result lands at
// the head's sorted position (pocc[pos], as the probe kernel of the sample
// sort encodes it), so the unique pass reads it coalesced and its look-back
// never waits on a probe.  A call rejected for a reserved key (found by the
// histogram pass) only looks keys up.
__global__ void __launch_bounds__(kUqBlock) head_probe_kernel(const __grid_constant__ UniqueParams p) {
  __shared__ unsigned s_claims;
  if (threadIdx.x == 0) s_claims = 0;
  __syncthreads();
  const int64_t N = p.N;
  const unsigned na = p.ctl->n_active;
  const uint64_t* ks = na == 0 ? nullptr : (((na - 1) & 1) ? p.kb1 : p.kb0);
  const bool rejected = __ldcg(&p.bdev->reject_call) == p.call_id;
  const int64_t pos0 = ((int64_t)blockIdx.x * kUqBlock + threadIdx.x) * kHpItems;
  uint64_t k[kHpItems + 1];
#pragma unroll
  for (int j = 0; j <= kHpItems; ++j) {
    const int64_t pos = pos0 + j - 1;
    k[j] = (pos >= 0 && pos < N) ? (ks ? ks[pos] : to_ukey(p.in_keys[pos])) : 0;
  }
  bool head[kHpItems];
  uint64_t h[kHpItems];
  longlong2 sv[kHpItems];
#pragma unroll
  for (int j = 0; j < kHpItems; ++j) {
    const int64_t pos = pos0 + j;
    head[j] = pos < N && (pos == 0 || k[j] != k[j + 1]);
    h[j] = mix64((uint64_t)from_ukey(k[j + 1]) ^ kSlotSalt) & p.slot_mask;
    if (head[j] && from_ukey(k[j + 1]) != kEmptyKey)
      sv[j] = __ldcg(reinterpret_cast<const longlong2*>(p.slots + h[j]));
  }
#pragma unroll
  for (int j = 0; j < kHpItems; ++j) {
    if (!head[j]) continue;
    int64_t r = -1;  // the reserved key (reported by the histogram pass) has no row
    if (from_ukey(k[j + 1]) != kEmptyKey) {
      const Probe pr = idmap_probe(p.slots, p.slot_mask, from_ukey(k[j + 1]), h[j], sv[j], !rejected, &s_claims);
      if (pr.limit) raise_error(p.st, p.mirror, kErrTableFull);
      else if (pr.row >= 0) r = pr.row;
      else if (pr.slot >= 0) r = pr.prior + 1 >= p.admit ? -2 - pr.slot : kCandPocc - pr.slot;
    }
    p.pocc[pos0 + j] = r;
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_claims) atomicAdd(&p.st->slots_used, (unsigned long long)s_claims);
}

__global__ void __launch_bounds__(kUqBlock) unique_insert_kernel(const __grid_constant__ UniqueParams p) {
  __shared__ uint64_t s_last[kUqBlock];
  __shared__ unsigned s_scan[kUqBlock / 32];
  __shared__ unsigned s_tile;
  __shared__ unsigned long long s_prefix;
  __shared__ int s_ninit;
  __shared__ unsigned s_unclaim;
  __shared__ int64_t s_init_key[kUqTile];
  __shared__ int64_t s_init_row[kUqTile];

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) {
    s_tile = atomicAdd(&p.ctl->seg_tile_counter, 1u);
    s_ninit = 0;
    s_unclaim = 0;
  }
  __syncthreads();
  const unsigned tile = s_tile;
  const int64_t N = p.N;
  const unsigned na = p.ctl->n_active;
  const uint64_t* ks = na == 0 ? nullptr : (((na - 1) & 1) ? p.kb1 : p.kb0);
  const uint32_t* vs = na == 0 ? nullptr : (((na - 1) & 1) ? p.vb1 : p.vb0);
  const int64_t tbase = (int64_t)tile * kUqTile;
  const int64_t pos0 = tbase + (int64_t)tid * kUqItems;

  uint64_t k[kUqItems];
  uint32_t v[kUqItems];
#pragma unroll
  for (int j = 0; j < kUqItems; ++j) {
    const int64_t pos = pos0 + j;
    if (pos < N) {
      k[j] = ks ? ks[pos] : to_ukey(p.in_keys[pos]);
      v[j] = vs ? vs[pos] : (uint32_t)pos;
    } else {
      k[j] = 0;
      v[j] = 0;
    }
  }
  s_last[tid] = k[kUqItems - 1];
  __syncthreads();
  uint64_t prev;
  bool have_prev;
  if (tid > 0) {
    prev = s_last[tid - 1];
    have_prev = true;
  } else if (tbase > 0) {
    prev = ks ? ks[tbase - 1] : to_ukey(p.in_keys[tbase - 1]);
    have_prev = true;
  } else {
    prev = 0;
    have_prev = false;
  }

  // a batch holding the reserved key (found by the histogram pass and the
  // probe) is rejected as a whole: the probe's claims are given back
  const bool rejected = __ldcg(&p.bdev->reject_call) == p.call_id;
  // the heads' IDMap results, recorded at their sorted positions by head_probe
  bool head[kUqItems], isnew[kUqItems];
  int64_t pv[kUqItems];
  unsigned nh = 0, nn = 0;
#pragma unroll
  for (int j = 0; j < kUqItems; ++j) {
    const int64_t pos = pos0 + j;
    const uint64_t pk = j == 0 ? prev : k[j - 1];
    head[j] = pos < N && (!(j == 0 ? have_prev : true) || pk != k[j]);
    pv[j] = head[j] ? __ldcg(p.pocc + pos) : -1;
  }
#pragma unroll
  for (int j = 0; j < kUqItems; ++j) {
    isnew[j] = !rejected && pocc_new(pv[j]);  // admitted by this call: gets a row
    if (head[j]) {
      ++nh;
      nn += isnew[j];
    }
  }
  // block exclusive scan of (heads, new) packed as heads | new << 16
  const unsigned mine = nh | (nn << 16);
  unsigned x = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_scan[w] = x;
  __syncthreads();
  unsigned wpre = 0, tot = 0;
#pragma unroll
  for (int ww = 0; ww < kUqBlock / 32; ++ww) {
    const unsigned c = s_scan[ww];
    if (ww < w) wpre += c;
    tot += c;
  }
  const unsigned excl_thread = wpre + x - mine;
  const unsigned long long tH = tot & 0xffffu, tN = tot >> 16;

  if (w == 0) {
    // decoupled look-back by warp 0: 32 predecessor tiles per step
    unsigned long long* my = p.lookback + tile;
    unsigned long long hx = 0, nx = 0;
    if (tile == 0) {
      if (lane == 0) st_relaxed(my, kUqIncl | (tH << 31) | tN);
    } else {
      if (lane == 0) st_relaxed(my, kUqAgg | (tH << 31) | tN);
      int64_t t = (int64_t)tile - 1;
      int spins = 0;
      bool done = false;
      while (!done) {
        const int64_t idx = t - lane;
        unsigned long long e = idx >= 0 ? ld_relaxed(p.lookback + idx) : kUqIncl;
        while (!__all_sync(0xffffffffu, (e >> 62) != 0)) {
          if (++spins > p.spin_max) break;
          __nanosleep(32);
          if ((e >> 62) == 0) e = ld_relaxed(p.lookback + idx);
        }
        if (spins > p.spin_max) {
          if (lane == 0) raise_error(p.st, p.mirror, kErrTimeout);
          break;
        }
        const unsigned incl = __ballot_sync(0xffffffffu, (e >> 62) == 2);
        const int stop = incl ? __ffs(incl) - 1 : 31;  // nearest inclusive entry
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
      if (lane == 0) st_relaxed(my, kUqIncl | ((hx + tH) << 31) | (nx + tN));
    }
    if (lane == 0) s_prefix = (hx << 32) | nx;
  }
  __syncthreads();
  const unsigned long long Hx = s_prefix >> 32, Nx = s_prefix & 0xffffffffULL;
  const unsigned long long row_base = p.bdev->row_base;

  unsigned hrun = Hx + (excl_thread & 0xffffu);
  unsigned nrun = (unsigned)Nx + (excl_thread >> 16);
#pragma unroll
  for (int j = 0; j < kUqItems; ++j) {
    const int64_t pos = pos0 + j;
    if (pos >= N) break;
    if (head[j]) {
      const unsigned seg = hrun;
      int64_t r = pv[j] >= 0 ? pv[j] : -1;
      if (isnew[j]) {
        // the k-th new key takes the k-th queued freed row, or a row past the end
        const int64_t slot = -2 - pv[j];
        const unsigned long long kk = nrun, avail = p.bdev->free_avail;
        r = kk < avail ? (int64_t)__ldg(p.free_rows + p.bdev->free_base + kk)
                       : (int64_t)(row_base + (kk - avail));
        ++nrun;
        if (r >= p.mapped_rows) {
          raise_error(p.st, p.mirror, kErrTableFull);
          r = -1;
        } else {
          p.slots[slot].row = r;
          p.row_keys[r] = from_ukey(k[j]);
          if (p.seen) p.seen[r] = (uint32_t)p.clock;
          const int q = atomicAdd(&s_ninit, 1);
          s_init_key[q] = from_ukey(k[j]);
          s_init_row[q] = r;
        }
      } else if (pv[j] <= -2) {
        // no row: a rejected call gives its claims back; otherwise the key
        // stays a candidate with one more lookup counted, at this clock
        const int64_t slot = pocc_new(pv[j]) ? -2 - pv[j] : kCandPocc - pv[j];
        if (rejected) atomicAdd(&s_unclaim, idmap_give_back(p.slots, slot));
        else p.slots[slot].row = cand_row(p.clock, prior_count(__ldcg(&p.slots[slot].row)) + 1);
      } else if (r >= 0 && p.seen && !rejected) {
        p.seen[r] = (uint32_t)p.clock;
      }
      p.uniq[seg] = from_ukey(k[j]);
      p.rows[seg] = r;
      p.seg_start[seg] = (int32_t)pos;
      ++hrun;
    }
    const int32_t seg = (int32_t)(hrun - 1);
    p.seg_of[pos] = seg;
    if (v[j] < (uint64_t)N) {
      p.inv[v[j]] = seg;
      p.spos[v[j]] = (uint32_t)pos;
    }
  }
  __syncthreads();
  if (tid == 0 && s_unclaim) atomicAdd(&p.st->slots_used, 0ULL - (unsigned long long)s_unclaim);
  if (tile == gridDim.x - 1 && tid == 0) {
    const unsigned long long U = Hx + tH, nnew = Nx + tN;
    p.bdev->U = rejected ? 0u : (unsigned)U;
    p.bdev->n_new = (unsigned)nnew;
    const unsigned long long avail = p.bdev->free_avail;
    unsigned long long nf = row_base + (nnew > avail ? nnew - avail : 0ULL);
    if (nf > (unsigned long long)p.mapped_rows) nf = (unsigned long long)p.mapped_rows;
    p.st->next_free = nf;
    p.st->free_head = p.bdev->free_base + (nnew < avail ? nnew : avail);
    if (p.mirror) {
      p.mirror->next_free = nf;
      p.mirror->slots_used = *(volatile unsigned long long*)&p.st->slots_used;
      __threadfence_system();
    }
    p.seg_start[U] = (int32_t)N;
  }
  __syncthreads();
  // initialise this tile's new rows: one warp per row, 16 bytes per lane per
  // step; the key's base hash is formed once per row
  const int nf4 = p.row_floats >> 2;
  const int ncol = p.D >> 2;
  const float sv = p.adagrad ? p.acc0 : 0.0f;
  for (int r = w; r < s_ninit; r += kUqBlock / 32) {
    const uint64_t base = mix64((uint64_t)s_init_key[r] ^ p.init_seed);
    float4* dst = reinterpret_cast<float4*>(p.row_data + s_init_row[r] * (int64_t)p.row_floats);
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
}

__global__ void rows_per_key_kernel(const int32_t* __restrict__ inv, const int64_t* __restrict__ rows,
                                    int64_t N, int64_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < N; i += stride)
    out[i] = rows[inv[i]];
}

cudaError_t launch_unique_insert(recis_batch* b, recis_table* t, int64_t N, bool insert, cudaStream_t s) {
  UniqueParams p;
  p.in_keys = b->keys;
  p.kb0 = b->kbuf[0];
  p.kb1 = b->kbuf[1];
  p.vb0 = b->vbuf[0];
  p.vb1 = b->vbuf[1];
  p.N = N;
  p.ctl = b->ctl;
  p.lookback = b->seg_lookback;
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
  p.st = t->dstate;
  p.mirror = t->mirror_dev;
  p.call_id = b->call_seq;
  p.spin_max = spin_limit();
  // a bulk insert pre-loads: its keys are admitted at once
  p.admit = (!insert && t->cfg.admit_threshold > 1) ? t->cfg.admit_threshold : 1;
  p.clock = (uint64_t)t->clock;
  p.seen = t->cfg.evictable ? reinterpret_cast<uint32_t*>(t->seen.va) : nullptr;
  p.free_rows = t->free_rows;
  p.pocc = b->pocc;
  const int64_t tiles = (N + kUqTile - 1) / kUqTile;
  {
    LaunchScope ls("head_probe", s);
    head_probe_kernel<<<(unsigned)((N + kUqBlock * kHpItems - 1) / (kUqBlock * kHpItems)), kUqBlock, 0, s>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  LaunchScope ls("unique_insert", s);
  unique_insert_kernel<<<(unsigned)tiles, kUqBlock, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_rows_per_key(recis_batch* b, int64_t N, int64_t* rows_out, cudaStream_t s) {
  int64_t blocks = (N + 255) / 256;
  if (blocks > 8 * kSMs) blocks = 8 * kSMs;
  LaunchScope ls("rows_per_key", s);
  rows_per_key_kernel<<<(unsigned)blocks, 256, 0, s>>>(b->inv, b->rows, N, rows_out);
  return cudaGetLastError();
}

// Every key of the old slot array into the new one with its row state (a row
// or a candidate count); tombstones are dropped.  Counts the slots filled.
__global__ void rehash_kernel(const Slot* __restrict__ old_slots, int64_t old_cap, Slot* slots,
                              uint64_t mask, DevState* st, HostMirror* mirror) {
  __shared__ unsigned s_claims;
  if (threadIdx.x == 0) s_claims = 0;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < old_cap; i += stride) {
    const Slot sl = old_slots[i];
    if (sl.key == kEmptyKey || sl.row == kTombRow) continue;
    const uint64_t h = mix64((uint64_t)sl.key ^ kSlotSalt) & mask;
    const Probe pr = idmap_probe(slots, mask, sl.key, h, __ldcg(reinterpret_cast<const longlong2*>(slots + h)),
                                 true, &s_claims);
    if (pr.slot >= 0 && pr.row < 0 && pr.prior == 0) slots[pr.slot].row = sl.row;
    else raise_error(st, mirror, pr.limit ? kErrTableFull : kErrDuplicateImport);
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_claims) atomicAdd(&st->slots_used, (unsigned long long)s_claims);
}

// Imported keys get rows row0 + i; a key already holding a row is an error, a
// candidate or an evicted key is admitted with its imported row.
__global__ void import_kernel(const int64_t* __restrict__ keys, int64_t n, int64_t row0,
                              Slot* slots, uint64_t mask, int64_t* row_keys, uint32_t* seen,
                              uint32_t clock, DevState* st, HostMirror* mirror) {
  __shared__ unsigned s_claims;
  if (threadIdx.x == 0) s_claims = 0;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t h = mix64((uint64_t)keys[i] ^ kSlotSalt) & mask;
    const Probe pr = idmap_probe(slots, mask, keys[i], h, __ldcg(reinterpret_cast<const longlong2*>(slots + h)),
                                 true, &s_claims);
    if (pr.slot >= 0 && pr.row < 0) {
      slots[pr.slot].row = row0 + i;
      row_keys[row0 + i] = keys[i];
      if (seen) seen[row0 + i] = clock;
    } else {
      raise_error(st, mirror, pr.limit ? kErrTableFull : kErrDuplicateImport);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_claims) atomicAdd(&st->slots_used, (unsigned long long)s_claims);
}

cudaError_t launch_rehash(recis_table* t, const Slot* old_slots, int64_t old_cap, cudaStream_t s) {
  int64_t blocks = (old_cap + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  LaunchScope ls("idmap_rehash", s);
  rehash_kernel<<<(unsigned)blocks, 256, 0, s>>>(old_slots, old_cap, t->slots,
                                                 (uint64_t)t->capacity - 1, t->dstate,
                                                 t->mirror_dev);
  return cudaGetLastError();
}

cudaError_t launch_import(recis_table* t, const int64_t* keys, int64_t n, int64_t row0,
                          int64_t clock, cudaStream_t s) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 16 * kSMs) blocks = 16 * kSMs;
  if (blocks < 1) return cudaSuccess;
  LaunchScope ls("idmap_import", s);
  import_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      keys, n, row0, t->slots, (uint64_t)t->capacity - 1, reinterpret_cast<int64_t*>(t->keys.va),
      t->cfg.evictable ? reinterpret_cast<uint32_t*>(t->seen.va) : nullptr, (uint32_t)clock, t->dstate,
      t->mirror_dev);
  return cudaGetLastError();
}

int64_t unique_tiles_for(int64_t N) { return (N + kUqTile - 1) / kUqTile; }

}  // namespace recis
