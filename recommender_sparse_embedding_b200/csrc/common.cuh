// common.cuh -- device-side helpers shared by the kernels of the embedding engine.
#pragma once
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

namespace recis {

constexpr int kSMs = 148;  // B200
constexpr int64_t kEmptyKey = -1;

// device-detected error bits (table or batch status word)
enum : int {
  kErrReservedKey = 1,
  kErrTableFull = 2,
  kErrTimeout = 4,
  kErrTagOverflow = 8,
  kErrDuplicateImport = 16,
  kErrBadOffsets = 32,
};

// Bound for every spin-wait on another CTA's progress: after this many polls
// (with a short sleep each) the waiter records kErrTimeout and moves on.  The
// kernels take the bound as an argument (spin_limit()), which a test may lower
// through recis_debug_set to make a wait give up.
constexpr int kSpinLimit = 1 << 22;

// H: SplitMix64 finaliser (Steele, Lea & Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014).  The feature Hash op, the row initialiser
// and the IDMap slot hash all use it.
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

// IDMap slot salt: decorrelates the slot index from keys that are themselves
// outputs of the feature hash.
constexpr uint64_t kSlotSalt = 0x2545F4914F6CDD1DULL;

struct __align__(16) Slot {
  int64_t key;  // kEmptyKey when free
  int64_t row;  // see the row states below
};

// Row field of a slot whose key is set (admission and eviction: RecIS README,
// Core architecture > Embedding Engine, feature eviction and admission):
//   >= 0          the key's row;
//   -1            claimed by the running call, no row yet;
//   kTombRow      the key was evicted: it keeps its slot (so no other key's
//                 probe chain is cut) and has no row; if it comes back it
//                 takes this slot again;
//   kReclaimRow   an evicted key's slot taken again by the running call;
//   candidate     a key seen by earlier lookups but not admitted yet:
//                 -2 - (clock << 16 | count), count = lookups it appeared in
//                 (1 .. 65535), clock = the last of them (< 2^40).
constexpr int64_t kTombRow = INT64_MIN;
constexpr int64_t kReclaimRow = INT64_MIN + 1;
constexpr int kMaxAdmitThreshold = 65535;
__host__ __device__ __forceinline__ bool is_cand_row(int64_t r) { return r <= -2 && r > kReclaimRow; }
__host__ __device__ __forceinline__ int cand_count(int64_t r) { return (int)((-2 - r) & 0xffff); }
__host__ __device__ __forceinline__ uint64_t cand_clock(int64_t r) { return (uint64_t)(-2 - r) >> 16; }
__host__ __device__ __forceinline__ int64_t cand_row(uint64_t clock, int count) {
  return -2 - (int64_t)((clock << 16) | (uint64_t)(count < 0xffff ? count : 0xffff));
}
// lookups the key had appeared in before the running call, from its row field
__host__ __device__ __forceinline__ int prior_count(int64_t r) { return is_cand_row(r) ? cand_count(r) : 0; }
// last-lookup clock of a row freed by an eviction that has not yet joined
// the free-row queue
constexpr uint32_t kFreedMark = 0xffffffffu;

// Table-wide device state.
struct DevState {
  unsigned long long next_free;   // rows in use: live rows and freed rows below it
  int status;                     // OR of error bits
  int pad;
  unsigned long long slots_used;  // IDMap slots holding a key (tombstones included)
  unsigned long long free_head;   // freed rows not yet reused: queue [free_head, free_tail)
  unsigned long long free_tail;
};

// Host-mapped mirror: written by kernels so the host can read progress and
// errors after an event, without a device synchronisation.
struct HostMirror {
  volatile unsigned long long next_free;
  volatile int error_seen;
  volatile int pad;
  volatile unsigned long long slots_used;
};

// Result of an IDMap probe for one key.
struct Probe {
  int64_t row;   // the key's row (>= 0), or -1 when it has none
  int64_t slot;  // its slot when it has no row (claimed, candidate or reclaimed); -1 otherwise
  int prior;     // lookups it appeared in before this call (candidates; 0 otherwise)
  bool limit;    // the probe limit was reached (the IDMap is too full)
};

constexpr int kProbeLimit = 1 << 16;

// IDMap result of one occurrence, as the probe kernel records it: the key's
// row (>= 0); -2 - slot for a key without a row that this call admits (it
// gets a row); kCandPocc - slot for one that stays a candidate; -1 when there
// is no row and no slot (reserved key, or the IDMap was exhausted).
constexpr int64_t kCandPocc = -((int64_t)1 << 40) - 2;
__device__ __forceinline__ bool pocc_new(int64_t v) { return v <= -2 && v > kCandPocc; }
__device__ __forceinline__ bool pocc_cand(int64_t v) { return v <= kCandPocc; }

// IDMap find-or-insert with admission: linear probing from slot h (sv = the
// slot already loaded there).  A key found with a row returns it; a key
// without one (claimed by this call, a candidate, or evicted -- an evicted
// key's slot is reclaimed for it) returns its slot and its prior count; a
// missing key claims the first free slot by a 64-bit CAS on its key (each
// claim adds one to *claims).  With insert false nothing is claimed and a
// missing or evicted key returns row -1 and slot -1.
__device__ __forceinline__ Probe idmap_probe(Slot* slots, uint64_t mask, int64_t key, uint64_t h,
                                             longlong2 sv, bool insert, unsigned* claims) {
  const int64_t limit = (int64_t)mask + 1 < kProbeLimit ? (int64_t)mask + 1 : kProbeLimit;
  for (int64_t n = 0; n < limit; ++n) {
    if (n > 0) sv = __ldcg(reinterpret_cast<const longlong2*>(slots + h));
    bool mine = sv.x == key;
    if (!mine && sv.x == kEmptyKey) {
      if (!insert) return Probe{-1, -1, 0, false};
      const unsigned long long old = atomicCAS(reinterpret_cast<unsigned long long*>(&slots[h].key),
                                               (unsigned long long)kEmptyKey, (unsigned long long)key);
      if ((int64_t)old == kEmptyKey) {
        atomicAdd(claims, 1u);
        return Probe{-1, (int64_t)h, 0, false};
      }
      mine = (int64_t)old == key;
    }
    if (mine) {
      const int64_t r = sv.x == key && sv.y >= 0 ? sv.y : __ldcg(&slots[h].row);
      if (r >= 0) return Probe{r, -1, 0, false};
      if (r == kTombRow || r == kReclaimRow) {
        if (!insert) return Probe{-1, -1, 0, false};
        if (r == kTombRow)
          atomicCAS(reinterpret_cast<unsigned long long*>(&slots[h].row), (unsigned long long)kTombRow,
                    (unsigned long long)kReclaimRow);
        return Probe{-1, (int64_t)h, 0, false};
      }
      return Probe{-1, (int64_t)h, prior_count(r), false};  // claimed by this call (-1) or a candidate
    }
    h = (h + 1) & mask;
  }
  return Probe{-1, -1, 0, true};
}

// Gives back a slot the running call took for a key it then did not keep (a
// rejected call): a fresh claim empties it again (returns 1, one slot less in
// use), a reclaimed evicted key's slot becomes a tombstone again; a
// candidate's slot keeps its state.  Every key claimed by the call is newer
// than every key that stays, so emptying its slot cuts no probe chain.
__device__ __forceinline__ unsigned idmap_give_back(Slot* slots, int64_t slot) {
  const int64_t r = __ldcg(&slots[slot].row);
  if (r == -1) {
    slots[slot].key = kEmptyKey;
    return 1u;
  }
  if (r == kReclaimRow) slots[slot].row = kTombRow;
  return 0u;
}

__device__ __forceinline__ void raise_error(DevState* st, HostMirror* mirror, int bit) {
  atomicOr(&st->status, bit);
  if (mirror) mirror->error_seen = 1;
}

// signed int64 -> order-preserving uint64
__device__ __forceinline__ uint64_t to_ukey(int64_t k) { return (uint64_t)k ^ 0x8000000000000000ULL; }
__device__ __forceinline__ int64_t from_ukey(uint64_t u) { return (int64_t)(u ^ 0x8000000000000000ULL); }

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Row init: emb[j] = (u - 1/2) * 2s with u = (H(H(key ^ seed) + j) >> 40) * 2^-24.
// (u - 0.5f) is exact in fp32 and the product is rounded once.
__device__ __forceinline__ float init_value(uint64_t base, int j, float two_s) {
  const uint64_t h = mix64(base + (uint64_t)j);
  const float u = (float)(uint32_t)(h >> 40) * (1.0f / 16777216.0f);
  return __fmul_rn(u - 0.5f, two_s);
}

// Programmatic dependent launch.  Kernels of the step are launched with the
// programmatic-serialization attribute (launch_pdl): a kernel may be
// scheduled while its predecessor in the stream is still running, so its
// first statement waits for the predecessor's completion and memory
// (griddepcontrol.wait), and a CTA whose stores are done lets the successor
// start launching (griddepcontrol.launch_dependents).  Without the
// attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- row gathers by the bulk-copy (TMA) engine: one instruction moves a
// whole contiguous row from global into shared memory and counts its bytes
// on a shared-memory transaction barrier (mbarrier).  Addresses and sizes
// are multiples of 16 bytes; no cluster multicast.
__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* mbar, unsigned arrivals) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(arrivals) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// one arrival that also expects `bytes` of bulk copies in this phase
__device__ __forceinline__ void mbar_arrive_expect(uint64_t* mbar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(mbar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_row(void* dst, const void* src, unsigned bytes, uint64_t* mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(mbar))
               : "memory");
}
// orders this thread's earlier shared-memory reads before later bulk copies
// into the same bytes
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(mbar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `parity` to complete, polling at most `limit`
// times (each poll itself waits a short while in hardware); false when it
// gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, unsigned parity, int limit) {
  for (int i = 0; i < limit; ++i)
    if (mbar_try_wait(mbar, parity)) return true;
  return false;
}

}  // namespace recis
