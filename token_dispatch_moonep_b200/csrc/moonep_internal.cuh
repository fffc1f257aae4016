// Internal definitions shared by the libmoonep.so translation units: arena and
// workspace layout, config validation, device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "moonep.h"

namespace moonep {

// Diagnostics set by moonep_debug_set_wait (process-wide, host side): the
// time limit of every bounded in-kernel wait, and the phantom count that
// forces a wait to run out (tests only).
long long debug_wait_limit_ns();
int debug_phantom();

// Unique id of the calling thread's current CUDA context (the driver never
// reuses one within a process, so a device reset or a second context on the
// same device gives a new id); 0 if it cannot be queried.  Host state that
// belongs to one context (a kernel's attributes, a device symbol's address)
// is cached under this id.
unsigned long long current_context_id();

constexpr int kMaxDevices = 128;  // device ordinals the host-side caches cover

// Streaming multiprocessors of the current device (cached per device; 148 on B200).
int current_sm_count();

constexpr int kPlanThreads = 512;   // threads per CTA of the plan kernel
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPairsPerThread = 16;  // most pairs per thread in one plan chunk
constexpr size_t kAlignBytes = 256;

// ----------------------------------------------------------------- config ---
struct Dims {
  int64_t R, E, K, S, H, B, A, L, SK, N, NvS, NCMAX, PMAX;  // NCMAX: most plan chunks (512 pairs each)
  int mode;
  uint32_t magicL;  // ceil(2^32 / L) for L > 1: e / L == __umulhi(e, magicL) for e < 2^22
};

__host__ __device__ inline int64_t nvs_of(int64_t S, int64_t K, int64_t E, int64_t A) {
  int64_t sk = S * K;
  return sk + (A - 1) * (sk < E ? sk : E);
}

// Validates everything that does not depend on H; returns false on a bad config.
inline bool make_dims(const moonep_config_t *c, Dims *d) {
  if (!c) return false;
  if (c->R < 1 || c->E < 1 || c->E % c->R != 0) return false;
  if (c->E > MOONEP_MAX_EXPERTS) return false;
  if (c->K < 1 || c->K > c->E || c->K > MOONEP_MAX_TOPK) return false;
  if (c->S < 0 || c->budget < 0 || c->budget > c->E) return false;
  if (c->mode != MOONEP_MODE_TRAIN && c->mode != MOONEP_MODE_INFER) return false;
  if (c->align < 1 || c->align > 4096) return false;
  d->R = c->R; d->E = c->E; d->K = c->K; d->S = c->S; d->H = c->H;
  d->B = c->budget; d->A = c->align; d->mode = c->mode;
  d->L = d->E / d->R;
  d->SK = d->S * d->K;
  d->N = d->R * d->SK;
  d->NvS = nvs_of(d->S, d->K, d->E, d->A);
  if (d->N >= (int64_t(1) << 31) || d->R * d->NvS >= (int64_t(1) << 31)) return false;
  d->NCMAX = d->N > 0 ? (d->N + kPlanThreads - 1) / kPlanThreads : 1;
  d->PMAX = d->E + d->R;
  d->magicL = d->L > 1 ? (uint32_t)(0xFFFFFFFFu / (uint32_t)d->L) + 1u : 0u;
  return true;
}

// ------------------------------------------------------------ plan arena ---
enum ArenaField {
  F_SLOT_OF, F_SLOT_SRC, F_EXPERT_COUNT, F_RANK_LOAD, F_OVERFLOW, F_DEFICIT, F_N_SEG,
  F_SEG_EXPERT, F_SEG_START, F_SEG_LEN, F_SEG_KIND, F_SEG_WSLOT,
  F_PIECE_EXPERT, F_PIECE_RANK, F_PIECE_START, F_PIECE_LEN, F_PIECE_WSLOT, F_PIECE_OSTART,
  F_EXP_PIECE_BEGIN, F_EXP_PIECE_END, F_REP_EXPERT, F_REPLICATED, F_SCALARS,
  F_COUNT
};

enum Scalar { S_N_PIECE = 0, S_N_REMOTE = 1, S_N_LOCAL = 2, S_N_REPLICATED = 3, S_BAD = 4 };

inline size_t align_up(size_t v) { return (v + kAlignBytes - 1) / kAlignBytes * kAlignBytes; }

struct ArenaLayout {
  size_t off[F_COUNT];
  size_t total;
  explicit ArenaLayout(const Dims &d) {
    const int64_t n[F_COUNT] = {
        d.N, d.R * d.NvS, d.E, d.R, d.R, d.R, d.R,
        d.R * d.E, d.R * d.E, d.R * d.E, d.R * d.E, d.R * d.E,
        d.PMAX, d.PMAX, d.PMAX, d.PMAX, d.PMAX, d.PMAX,
        d.E, d.E, d.R * d.B, d.E, 8};
    size_t o = 0;
    for (int i = 0; i < F_COUNT; i++) {
      off[i] = o;
      o += align_up(size_t(n[i] > 0 ? n[i] : 1) * sizeof(int32_t));
    }
    total = o;
  }
};

// Device-side bundle of arena pointers.
struct PlanPtrs {
  int32_t *f[F_COUNT];
};

inline PlanPtrs plan_ptrs(const Dims &d, const void *arena) {
  ArenaLayout lay(d);
  PlanPtrs p;
  for (int i = 0; i < F_COUNT; i++)
    p.f[i] = reinterpret_cast<int32_t *>(const_cast<char *>(static_cast<const char *>(arena)) + lay.off[i]);
  return p;
}

// -------------------------------------------------------------- workspace ---
// Plan scratch: sync words (generation, done, state, tables-done, two totals
// tags), two expert-total buffers (each kTotalCopies partial copies of
// MOONEP_MAX_EXPERTS counts) at a fixed offset
// (so that a call with another config finds them where the last call left them),
// per-chunk arrival epochs (plus slots for diagnostic phantom arrivals), per-chunk
// bad-id marks, per-chunk histograms, stable ranks, placement constants.
constexpr int kSyncWords = 16;
constexpr int kSyncMaxPhantom = 32;
constexpr int kTotalCopies = 16;  // chunk k adds its counts into copy k % 16 (spreads the atomics)

enum WsField {
  W_SYNC, W_TOTALS, W_ARRIVE, W_BADMARK, W_HIST, W_RANK, W_EXP_KEPT, W_EXP_ROW0, W_EXP_OSTART,
  W_PIECE_GROW, W_COUNT
};

struct WsLayout {
  size_t off[W_COUNT];
  size_t total;
  explicit WsLayout(const Dims &d) {
    const size_t n[W_COUNT] = {
        size_t(kSyncWords) * sizeof(int32_t),
        size_t(2 * kTotalCopies * MOONEP_MAX_EXPERTS) * sizeof(int32_t),
        size_t(d.NCMAX + kSyncMaxPhantom) * sizeof(int32_t),
        size_t(d.NCMAX) * sizeof(int32_t),
        size_t(d.E * d.NCMAX) * sizeof(int32_t),
        size_t(d.N > 0 ? d.N : 1) * sizeof(uint16_t),
        size_t(d.E) * sizeof(int32_t), size_t(d.E) * sizeof(int32_t), size_t(d.E) * sizeof(int32_t),
        size_t(d.PMAX) * sizeof(int32_t)};
    size_t o = 0;
    for (int i = 0; i < W_COUNT; i++) {
      off[i] = o;
      o += align_up(n[i]);
    }
    total = o;
  }
};

// ---------------------------------------------------------------- helpers ---
__device__ __forceinline__ void set_status(int32_t *st, int32_t bits) {
  if (st) atomicOr(st, bits);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// home rank of expert e (e / L) without a division
__device__ __forceinline__ int home_of(const Dims &d, int e) {
  return d.L == 1 ? e : (int)__umulhi((unsigned)e, d.magicL);
}

// bf16 pairs packed in a 32-bit word: exact widening, and round-to-nearest-even packing
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 l = __float2bfloat16_rn(lo);
  const __nv_bfloat16 h = __float2bfloat16_rn(hi);
  return (uint32_t)__bfloat16_as_ushort(l) | ((uint32_t)__bfloat16_as_ushort(h) << 16);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

inline cudaStream_t to_cuda(moonep_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace moonep
