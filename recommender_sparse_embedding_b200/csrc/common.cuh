// common.cuh -- device-side helpers shared by the kernels of the embedding engine.
#pragma once
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
  int64_t row;
};

// Table-wide device state.
struct DevState {
  unsigned long long next_free;  // number of live rows
  int status;                    // OR of error bits
  int pad;
};

// Host-mapped mirror: written by kernels so the host can read progress and
// errors after an event, without a device synchronisation.
struct HostMirror {
  volatile unsigned long long next_free;
  volatile int error_seen;
  volatile int pad;
};

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

}  // namespace recis
