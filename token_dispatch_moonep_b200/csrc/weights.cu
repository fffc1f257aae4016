// The weight matrix of every entry of the plan's per-rank segment tables ("Moonshot AI
// Open-Sources MoonEP", replica-slot paragraph: a duplicated expert computes on its
// receiving rank with a local copy of its weights, held in one of the rank's replica
// slots, and past the slot budget reads them on its home rank).  The expert computation
// between dispatch and combine needs, for each segment, the rows it owns (seg_start,
// seg_len) and the weights it multiplies them with; this table gives the latter as
// device pointers, written on the device so that no host read of the plan is needed.
#include "moonep_internal.cuh"

namespace moonep {
namespace {

constexpr int kWeightThreads = 256;

// One thread per segment-table entry q = d * E + i: a replica piece reads its rank's
// slot rep_w[d][j], a native segment and a remote piece the home row w[e], an unused
// entry nothing (null).  Entries that name an expert or a slot out of range are null
// and set MOONEP_DEV_BAD_PLAN.
__global__ void __launch_bounds__(kWeightThreads)
segment_weights_kernel(const int32_t *__restrict__ seg_expert, const int32_t *__restrict__ seg_kind,
                       const int32_t *__restrict__ seg_wslot, const uint16_t *w,
                       const uint16_t *rep_w, int64_t W, int R, int E, int B,
                       const uint16_t **out, int32_t *status) {
  // launched with programmatic stream serialisation: nothing is read before the kernel
  // ahead of it in the stream (the plan) has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t q = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x;
  if (q >= (int64_t)R * E) return;
  const int64_t d = q / E;
  const int kind = seg_kind[q];
  const uint16_t *p = nullptr;
  bool bad = false;
  if (kind == MOONEP_SEG_REPLICA) {
    const int j = seg_wslot[q];
    if (j >= 0 && j < B) p = rep_w + (d * B + j) * W;
    else bad = true;
  } else if (kind == MOONEP_SEG_NATIVE || kind == MOONEP_SEG_REMOTE) {
    const int e = seg_expert[q];
    if (e >= 0 && e < E) p = w + (int64_t)e * W;
    else bad = true;
  }
  out[q] = p;
  if (bad) atomicOr(status, MOONEP_DEV_BAD_PLAN);
}

}  // namespace
}  // namespace moonep

using namespace moonep;

extern "C" moonep_status_t moonep_segment_weights(const moonep_config_t *cfg, const void *plan_arena,
                                                  const uint16_t *weights, const uint16_t *rep_weights,
                                                  int64_t W, const uint16_t **seg_weights,
                                                  int32_t *dev_status, moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d) || !plan_arena || !aligned256(plan_arena) || !weights || W < 1 ||
      !seg_weights || (reinterpret_cast<uintptr_t>(seg_weights) & 7u) != 0 || !dev_status ||
      (d.B > 0 && !rep_weights))
    return MOONEP_ERR_INVALID_ARG;
  const PlanPtrs P = plan_ptrs(d, plan_arena);
  const int64_t n = d.R * d.E;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((n + kWeightThreads - 1) / kWeightThreads));
  lc.blockDim = dim3(kWeightThreads);
  lc.stream = to_cuda(stream);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &lc, segment_weights_kernel, (const int32_t *)P.f[F_SEG_EXPERT], (const int32_t *)P.f[F_SEG_KIND],
      (const int32_t *)P.f[F_SEG_WSLOT], weights, rep_weights, W, (int)d.R, (int)d.E, (int)d.B,
      seg_weights, dev_status);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOONEP_ERR_CUDA;
  }
  return MOONEP_OK;
}
