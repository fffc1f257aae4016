// Data-movement kernels of the MoonEP hot path: zero-copy dispatch, combine,
// combine-backward, reduce_grad, and the "next" rows (weight prefetch,
// dispatch-backward, the copy-through-buffer comparison path).  All are
// HBM-bound row moves with O(1) arithmetic per byte; tensor cores are not
// involved.
//
// Rows are moved as 16-byte vectors (8 bf16).  A warp owns a token (dispatch:
// half a row of one; combine: half a row when the batch is small;
// combine-backward: two warps per token): lane k (< K) holds the token's k-th
// slot and gate and broadcasts them with shuffles.
// reduce_grad (over bf16 or fp32 gradient rows) streams through shared memory
// with bulk asynchronous copies.  Rows whose byte length or base address is not
// 16-byte aligned take a scalar (one value per lane) path.
#include <cuda_bf16.h>

#include <mutex>
#include <utility>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kThreads = kWarpsPerBlock * 32;

// Programmatic dependent launch.  Every kernel here is launched with
// programmatic stream serialisation, so the GPU may start it while the kernel
// before it in the stream drains; its first instruction waits until that
// kernel has completed and its memory is visible, so no read or write moves
// ahead of it.  This hides most of the launch gap between back-to-back kernels.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
void launch(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
            Args &&...args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(block);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);  // errors: cudaGetLastError
}

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// slot of pair (t, lane) for lanes < K, validated against the buffer; -1 otherwise
__device__ __forceinline__ int load_slot(const int32_t *slot_of, int64_t t, int K, int64_t nrows,
                                         int32_t *status) {
  const int lane = threadIdx.x & 31;
  int s = -1;
  if (lane < K) {
    s = __ldg(slot_of + t * K + lane);
    if (s >= nrows || s < -1) {
      set_status(status, MOONEP_DEV_BAD_PLAN);
      s = -1;
    }
  }
  return s;
}

// ------------------------------------------------------------- dispatch ---
// One warp per (token, column chunk).  A row of nvec vectors is cut into nch
// equal chunks of cl <= 32*U vectors; the warp loads its chunk once (U vectors
// per lane in flight) and stores it to the token's K slots.  Small units keep
// every SM busy to the end of the launch and a chunk is never a partial loop.
template <int U>
__global__ void __launch_bounds__(kThreads)
dispatch_chunk_kernel(const int32_t *__restrict__ slot_of, const uint4 *__restrict__ x,
                      uint4 *__restrict__ recv, int64_t T, int K, int64_t nvec, int64_t nch,
                      int64_t cl, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  const int64_t nunits = T * nch;
  for (int64_t w = warp_g; w < nunits; w += nwarps) {
    const int64_t t = w / nch;
    const int64_t c0 = (w - t * nch) * cl;
    const int64_t c1 = c0 + cl < nvec ? c0 + cl : nvec;
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const uint4 *src = x + t * nvec;
    uint4 buf[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = c0 + u * 32 + lane;
      if (v < c1) buf[u] = __ldcs(src + v);
    }
    for (int k = 0; k < K; k++) {
      const int row = __shfl_sync(0xffffffffu, my_slot, k);
      if (row < 0) continue;
      uint4 *dst = recv + (int64_t)row * nvec;
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int64_t v = c0 + u * 32 + lane;
        if (v < c1) dst[v] = buf[u];
      }
    }
  }
}

// chunking of a row of nvec vectors for dispatch_chunk_kernel<U>
struct RowChunks {
  int64_t nch, cl;
};
template <int U>
RowChunks row_chunks(int64_t nvec) {
  RowChunks r;
  r.nch = (nvec + 32 * U - 1) / (32 * U);
  if (r.nch < 1) r.nch = 1;
  r.cl = (nvec + r.nch - 1) / r.nch;
  return r;
}
constexpr int kDispatchU = 14;

__global__ void __launch_bounds__(kThreads)
dispatch_scalar_kernel(const int32_t *__restrict__ slot_of, const uint16_t *__restrict__ x,
                       uint16_t *__restrict__ recv, int64_t T, int K, int64_t H, int64_t nrows,
                       int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t t = warp_g; t < T; t += nwarps) {
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    for (int64_t h0 = 0; h0 < H; h0 += 32) {
      const int64_t h = h0 + lane;
      const uint16_t v = h < H ? x[t * H + h] : 0;
      for (int k = 0; k < K; k++) {
        const int row = __shfl_sync(0xffffffffu, my_slot, k);
        if (row >= 0 && h < H) recv[(int64_t)row * H + h] = v;
      }
    }
  }
}

// -------------------------------------------------------------- combine ---
template <int U>
__global__ void __launch_bounds__(kThreads)
combine_vec_kernel(const int32_t *__restrict__ slot_of, const uint4 *__restrict__ y,
                   const float *__restrict__ gates, uint4 *__restrict__ out, int64_t T, int K,
                   int64_t nvec, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t t = warp_g; t < T; t += nwarps) {
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const float my_w = lane < K ? (gates ? __ldg(gates + t * K + lane) : 1.f) : 0.f;
    for (int64_t v0 = 0; v0 < nvec; v0 += 32 * U) {
      float acc[U][8];
#pragma unroll
      for (int u = 0; u < U; u++)
#pragma unroll
        for (int i = 0; i < 8; i++) acc[u][i] = 0.f;
      for (int k = 0; k < K; k++) {
        const int row = __shfl_sync(0xffffffffu, my_slot, k);
        const float w = __shfl_sync(0xffffffffu, my_w, k);
        if (row < 0) continue;
        const uint4 *src = y + (int64_t)row * nvec;
        uint4 q[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
          const int64_t v = v0 + u * 32 + lane;
          if (v < nvec) q[u] = __ldcs(src + v);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
          const uint32_t wd[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
          for (int i = 0; i < 4; i++) {
            acc[u][2 * i] = __fmaf_rn(w, bf16_lo(wd[i]), acc[u][2 * i]);
            acc[u][2 * i + 1] = __fmaf_rn(w, bf16_hi(wd[i]), acc[u][2 * i + 1]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int64_t v = v0 + u * 32 + lane;
        if (v < nvec) {
          uint4 o;
          o.x = pack_bf16x2(acc[u][0], acc[u][1]);
          o.y = pack_bf16x2(acc[u][2], acc[u][3]);
          o.z = pack_bf16x2(acc[u][4], acc[u][5]);
          o.w = pack_bf16x2(acc[u][6], acc[u][7]);
          out[t * nvec + v] = o;
        }
      }
    }
  }
}

// K <= KMAX: the K rows of a column chunk are loaded before any arithmetic, so
// a warp keeps K*U 16-byte loads in flight.  A warp's unit is a token, or with
// split = 1 one half of its columns [c0, c0 + cl) (small batches: twice the units,
// so the last wave of warps is not left half empty).
template <int U, int KMAX>
__global__ void __launch_bounds__(kThreads)
combine_vec_k_kernel(const int32_t *__restrict__ slot_of, const uint4 *__restrict__ y,
                     const float *__restrict__ gates, uint4 *__restrict__ out, int64_t T, int K,
                     int64_t nvec, int split, int64_t cl, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  const int64_t nunits = T << split;
  for (int64_t w = warp_g; w < nunits; w += nwarps) {
    const int64_t t = w >> split;
    const int64_t c0 = (w - (t << split)) * cl;
    const int64_t c1 = c0 + cl < nvec ? c0 + cl : nvec;
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const float my_w = lane < K ? (gates ? __ldg(gates + t * K + lane) : 1.f) : 0.f;
    int rows[KMAX];
    float ws[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; k++) {
      rows[k] = __shfl_sync(0xffffffffu, my_slot, k);
      ws[k] = __shfl_sync(0xffffffffu, my_w, k);
    }
    for (int64_t v0 = c0; v0 < c1; v0 += 32 * U) {
      uint4 q[KMAX][U];
#pragma unroll
      for (int k = 0; k < KMAX; k++)
#pragma unroll
        for (int u = 0; u < U; u++) {
          const int64_t v = v0 + u * 32 + lane;
          q[k][u] = (rows[k] >= 0 && v < c1) ? __ldcs(y + (int64_t)rows[k] * nvec + v)
                                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int64_t v = v0 + u * 32 + lane;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] = 0.f;
#pragma unroll
        for (int k = 0; k < KMAX; k++) {
          if (rows[k] < 0) continue;  // k >= K, or a pair without a slot
          const uint32_t wd[4] = {q[k][u].x, q[k][u].y, q[k][u].z, q[k][u].w};
#pragma unroll
          for (int i = 0; i < 4; i++) {
            acc[2 * i] = __fmaf_rn(ws[k], bf16_lo(wd[i]), acc[2 * i]);
            acc[2 * i + 1] = __fmaf_rn(ws[k], bf16_hi(wd[i]), acc[2 * i + 1]);
          }
        }
        if (v < c1) {
          uint4 o;
          o.x = pack_bf16x2(acc[0], acc[1]);
          o.y = pack_bf16x2(acc[2], acc[3]);
          o.z = pack_bf16x2(acc[4], acc[5]);
          o.w = pack_bf16x2(acc[6], acc[7]);
          out[t * nvec + v] = o;
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
combine_scalar_kernel(const int32_t *__restrict__ slot_of, const uint16_t *__restrict__ y,
                      const float *__restrict__ gates, uint16_t *__restrict__ out, int64_t T, int K,
                      int64_t H, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t t = warp_g; t < T; t += nwarps) {
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const float my_w = lane < K ? (gates ? gates[t * K + lane] : 1.f) : 0.f;
    for (int64_t h0 = 0; h0 < H; h0 += 32) {
      const int64_t h = h0 + lane;
      float acc = 0.f;
      for (int k = 0; k < K; k++) {
        const int row = __shfl_sync(0xffffffffu, my_slot, k);
        const float w = __shfl_sync(0xffffffffu, my_w, k);
        if (row >= 0 && h < H) acc = __fmaf_rn(w, bf16_to_f(y[(int64_t)row * H + h]), acc);
      }
      if (h < H) out[t * H + h] = f_to_bf16(acc);
    }
  }
}

// ----------------------------------------------------- combine-backward ---
// dy[slot_k] = bf16(w_k * dout[t]); dgates[t,k] = <dout[t], y[slot_k]> (fp32, lane
// partials then a warp tree).  One k at a time; the dout row is re-read from
// cache for each k.
template <int U>
__global__ void __launch_bounds__(kThreads)
combine_bwd_vec_kernel(const int32_t *__restrict__ slot_of, const uint4 *__restrict__ dout,
                       const uint4 *__restrict__ y, const float *__restrict__ gates,
                       uint4 *__restrict__ dy, float *__restrict__ dgates, int64_t T, int K,
                       int64_t nvec, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t t = warp_g; t < T; t += nwarps) {
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const float my_w = lane < K ? (gates ? __ldg(gates + t * K + lane) : 1.f) : 0.f;
    const uint4 *g = dout + t * nvec;
    float my_dg = 0.f;
    for (int k = 0; k < K; k++) {
      const int row = __shfl_sync(0xffffffffu, my_slot, k);
      const float w = __shfl_sync(0xffffffffu, my_w, k);
      float part = 0.f;
      if (row >= 0) {
        const uint4 *yr = y + (int64_t)row * nvec;
        uint4 *dr = dy + (int64_t)row * nvec;
        for (int64_t v0 = 0; v0 < nvec; v0 += 32 * U) {
          uint4 gq[U], yq[U];
#pragma unroll
          for (int u = 0; u < U; u++) {
            const int64_t v = v0 + u * 32 + lane;
            if (v < nvec) {
              gq[u] = __ldg(g + v);
              yq[u] = __ldcs(yr + v);
            }
          }
#pragma unroll
          for (int u = 0; u < U; u++) {
            const int64_t v = v0 + u * 32 + lane;
            if (v < nvec) {
              const uint32_t gw[4] = {gq[u].x, gq[u].y, gq[u].z, gq[u].w};
              const uint32_t yw[4] = {yq[u].x, yq[u].y, yq[u].z, yq[u].w};
              uint32_t o[4];
#pragma unroll
              for (int i = 0; i < 4; i++) {
                const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
                part = __fmaf_rn(g0, bf16_lo(yw[i]), part);
                part = __fmaf_rn(g1, bf16_hi(yw[i]), part);
                o[i] = pack_bf16x2(__fmul_rn(w, g0), __fmul_rn(w, g1));
              }
              dr[v] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane == k) my_dg = part;
    }
    if (lane < K) dgates[t * K + lane] = my_dg;
  }
}

// K <= KMAX, two warps per token: each warp of a pair takes half of the row's
// columns (twice the warps in flight for the same bytes).  Each warp reduces
// its per-k dot partials with a warp tree; the pair's two partials are added in
// fixed order through shared memory, so dgates are deterministic.
template <int U, int KMAX>
__global__ void __launch_bounds__(kThreads)
combine_bwd_split_kernel(const int32_t *__restrict__ slot_of, const uint4 *__restrict__ dout,
                         const uint4 *__restrict__ y, const float *__restrict__ gates,
                         uint4 *__restrict__ dy, float *__restrict__ dgates, int64_t T, int K,
                         int64_t nvec, int64_t nrows, int32_t *status) {
  pdl_wait();
  __shared__ float red[kWarpsPerBlock][KMAX];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int half = wib & 1;
  const int64_t unit = ((int64_t)blockIdx.x * kWarpsPerBlock + wib) >> 1;
  const int64_t nunits = (int64_t)gridDim.x * kWarpsPerBlock / 2;
  const int64_t cols = (nvec + 1) / 2;
  const int64_t c0 = half * cols, c1 = c0 + cols < nvec ? c0 + cols : nvec;
  for (int64_t t0 = 0; t0 < T; t0 += nunits) {  // same trip count for every warp of the block
    const int64_t t = t0 + unit;
    const bool act = t < T;
    int my_slot = -1;
    float my_w = 0.f;
    if (act) {
      my_slot = load_slot(slot_of, t, K, nrows, status);
      my_w = lane < K ? __ldg(gates + t * K + lane) : 0.f;
    }
    int rows[KMAX];
    float ws[KMAX], part[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; k++) {
      rows[k] = __shfl_sync(0xffffffffu, my_slot, k);
      ws[k] = __shfl_sync(0xffffffffu, my_w, k);
      part[k] = 0.f;
    }
    if (act) {
      const uint4 *g = dout + t * nvec;
      for (int64_t v0 = c0; v0 < c1; v0 += 32 * U) {
        uint4 gq[U], yq[KMAX][U];
#pragma unroll
        for (int u = 0; u < U; u++) {
          const int64_t v = v0 + u * 32 + lane;
          gq[u] = v < c1 ? __ldcs(g + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < KMAX; k++)
#pragma unroll
          for (int u = 0; u < U; u++) {
            const int64_t v = v0 + u * 32 + lane;
            yq[k][u] = (rows[k] >= 0 && v < c1) ? __ldcs(y + (int64_t)rows[k] * nvec + v)
                                                : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
        for (int k = 0; k < KMAX; k++) {
          if (rows[k] < 0) continue;
          uint4 *dr = dy + (int64_t)rows[k] * nvec;
#pragma unroll
          for (int u = 0; u < U; u++) {
            const int64_t v = v0 + u * 32 + lane;
            if (v >= c1) continue;
            const uint32_t gw[4] = {gq[u].x, gq[u].y, gq[u].z, gq[u].w};
            const uint32_t yw[4] = {yq[k][u].x, yq[k][u].y, yq[k][u].z, yq[k][u].w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
              const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
              part[k] = __fmaf_rn(g0, bf16_lo(yw[i]), part[k]);
              part[k] = __fmaf_rn(g1, bf16_hi(yw[i]), part[k]);
              o[i] = pack_bf16x2(__fmul_rn(ws[k], g0), __fmul_rn(ws[k], g1));
            }
            dr[v] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < KMAX; k++) {
      float p = part[k];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0) red[wib][k] = p;
    }
    __syncthreads();
    if (half == 0 && act && lane < K) dgates[t * K + lane] = red[wib][lane] + red[wib + 1][lane];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads)
combine_bwd_scalar_kernel(const int32_t *__restrict__ slot_of, const uint16_t *__restrict__ dout,
                          const uint16_t *__restrict__ y, const float *__restrict__ gates,
                          uint16_t *__restrict__ dy, float *__restrict__ dgates, int64_t T, int K,
                          int64_t H, int64_t nrows, int32_t *status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t t = warp_g; t < T; t += nwarps) {
    const int my_slot = load_slot(slot_of, t, K, nrows, status);
    const float my_w = lane < K ? (gates ? gates[t * K + lane] : 1.f) : 0.f;
    float my_dg = 0.f;
    for (int k = 0; k < K; k++) {
      const int row = __shfl_sync(0xffffffffu, my_slot, k);
      const float w = __shfl_sync(0xffffffffu, my_w, k);
      float part = 0.f;
      if (row >= 0) {
        for (int64_t h = lane; h < H; h += 32) {
          const float g = bf16_to_f(dout[t * H + h]);
          part = __fmaf_rn(g, bf16_to_f(y[(int64_t)row * H + h]), part);
          dy[(int64_t)row * H + h] = f_to_bf16(__fmul_rn(w, g));
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane == k) my_dg = part;
    }
    if (lane < K) dgates[t * K + lane] = my_dg;
  }
}

// ----------------------------------------------------------- reduce_grad ---
// A shared-memory pipeline fed by bulk asynchronous copies.  Work units are
// (replicated expert, 8 KB chunk of its row); a unit is one or more stages:
// the first holds the home chunk and the expert's first three local replica
// chunks, each further stage the next four.  One producer thread per CTA
// issues cp.async.bulk copies (completion counted in bytes on the stage's
// mbarrier); eight consumer warps add the stage's rows in fp32 in piece order
// and, after the unit's last stage, store the result over the home chunk (bf16
// gradients: rounded once to bf16; fp32 gradient buffers: the fp32 sum itself).
// Three stages of four chunks per CTA and two CTAs per SM keep up to 192 KB
// per SM in flight with no registers held for it (measured against 4 stages
// of 3 chunks: equal at 10 pieces over 6 experts, 6% faster at 59 over 54).
// Every wait is bounded (moonep_debug_set_wait's limit); a wait that gives up
// sets MOONEP_DEV_TIMEOUT, and the producer waits (bounded) for its copies
// before the CTA exits.
namespace rg {
constexpr int kChunk = 8192;             // bytes of a row per unit
constexpr int kSlots = 4;                // chunks per stage
constexpr int kStages = 3;
constexpr int kConsumerWarps = 8;
constexpr int kThreadsRg = (kConsumerWarps + 1) * 32;
constexpr int kSmem = kStages * kSlots * kChunk;
constexpr int kPieceCache = 64;          // local pieces of one expert kept in shared memory
constexpr int kVecPerLane = kChunk / 16 / (kConsumerWarps * 32);
static_assert(kVecPerLane * 16 * kConsumerWarps * 32 == kChunk, "chunk split over consumer lanes");

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// true once the phase of the given parity has completed; false after limit_ns
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_test(bar, parity))
    if ((long long)(now_ns() - t0) > limit_ns) return false;
  return true;
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

struct Tables {
  const int32_t *replicated, *scalars, *pbeg, *pend, *prank, *pwslot;
  int R, E, B, PMAX;
  long long wait_ns;  // limit of every mbarrier wait
  int phantom_tx;     // bytes the first stage expects beyond its copies (0; tests force a timeout)
};

// Expert of replicated entry i and its piece range; false if the tables are inconsistent.
__device__ __forceinline__ bool expert_of(const Tables &t, int64_t i, int *e, int *b, int *en) {
  *e = t.replicated[i];
  if (*e < 0 || *e >= t.E) return false;
  *b = t.pbeg[*e];
  *en = t.pend[*e];
  return *b >= 0 && *en <= t.PMAX && *en >= *b;
}
// Stages of a unit with nl local pieces: the first holds the home chunk and
// up to slots - 1 pieces, every further stage up to slots pieces.
__device__ __forceinline__ int stages_of(int nl, int slots) {
  return nl <= slots - 1 ? 1 : 1 + (nl - (slots - 1) + slots - 1) / slots;
}
__device__ __forceinline__ bool local_piece(const Tables &t, int pc, int *row) {
  const int ws = t.pwslot[pc], rk = t.prank[pc];
  *row = rk * t.B + ws;
  return ws >= 0 && ws < t.B && rk >= 0 && rk < t.R;
}
}  // namespace rg

// kF32: fp32 gradient rows (4 values per 16-byte vector) instead of bf16 (8); the
// sums are the same fp32 additions in the same order, with no rounding to bf16.
template <bool kF32>
__global__ void __launch_bounds__(rg::kThreadsRg, 1)
reduce_grad_bulk_kernel(rg::Tables t, const uint4 *__restrict__ rep, uint4 *__restrict__ home,
                        int64_t nvec, int32_t *status) {
  using namespace rg;
  constexpr int kEl = kF32 ? 4 : 8;  // values per 16-byte vector
  pdl_wait();
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ int pcache[kPieceCache];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int64_t n_exp = t.scalars[S_N_REPLICATED];
  if (n_exp < 0 || n_exp > t.E) {
    if (blockIdx.x == 0 && tid == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
    n_exp = 0;
  }
  const int64_t rowbytes = nvec * 16;
  const int64_t nch = (rowbytes + kChunk - 1) / kChunk;
  const int64_t total = n_exp * nch;
  if (tid == 0) {
    for (int s = 0; s < kStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // Both roles walk the same sequence: units u = blockIdx.x + j * gridDim.x,
  // each split into stages_of(local pieces, kSlots) stages, stage k of the
  // sequence in buffer k % kStages.
  if (warp == kConsumerWarps) {  // ------------------------------- producer
    if (lane != 0) return;
    int64_t k = 0, cur = -1;
    int e = 0, b = 0, en = 0, nl = 0;
    bool good = false, ok = true;
    for (int64_t u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const int64_t i = u / nch;
      if (i != cur) {  // a new expert: list its local pieces once
        cur = i;
        good = expert_of(t, i, &e, &b, &en);
        nl = 0;
        for (int pc = b; good && pc < en; pc++) {
          int row;
          if (!local_piece(t, pc, &row)) continue;
          if (nl < kPieceCache) pcache[nl] = row;
          nl++;
        }
      }
      if (!good) continue;
      const int64_t off = (u % nch) * kChunk;
      const uint32_t bytes = (uint32_t)(rowbytes - off < kChunk ? rowbytes - off : kChunk);
      const int ng = stages_of(nl, kSlots);
      int li = 0, pc = b;
      for (int g = 0; g < ng; g++, k++) {
        const int s = (int)(k % kStages);
        if (!mbar_wait(&empty[s], (uint32_t)((k / kStages) & 1) ^ 1u, t.wait_ns)) {
          ok = false;
          break;
        }
        const uint8_t *src[kSlots];
        int ns = 0;
        if (g == 0) src[ns++] = reinterpret_cast<const uint8_t *>(home + (int64_t)e * nvec) + off;
        while (ns < kSlots && li < nl) {
          int row = 0;
          if (nl <= kPieceCache) {
            row = pcache[li];
          } else {  // more local pieces than the cache holds: walk the tables again
            while (pc < en && !local_piece(t, pc, &row)) pc++;
            pc++;
          }
          li++;
          src[ns++] = reinterpret_cast<const uint8_t *>(rep + (int64_t)row * nvec) + off;
        }
        mbar_expect_tx(&full[s], bytes * (uint32_t)ns + (k == 0 ? (uint32_t)t.phantom_tx : 0u));
        uint8_t *dst = stage_mem + (size_t)s * kSlots * kChunk;
        for (int q = 0; q < ns; q++) bulk_load(dst + (size_t)q * kChunk, src[q], bytes, &full[s]);
      }
    }
    if (!ok) set_status(status, MOONEP_DEV_TIMEOUT);
    for (int64_t j = k > kStages ? k - kStages : 0; j < k; j++)  // copies land before exit
      mbar_wait(&full[j % kStages], (uint32_t)((j / kStages) & 1), t.wait_ns);
    return;
  }

  // ------------------------------------------------------------- consumers
  int64_t k = 0, cur = -1;
  int e = 0, nl = 0;
  bool good = false, ok = true;
  for (int64_t u = blockIdx.x; u < total && ok; u += gridDim.x) {
    const int64_t i = u / nch;
    if (i != cur) {
      cur = i;
      int b = 0, en = 0;
      good = expert_of(t, i, &e, &b, &en);
      nl = 0;
      for (int pc = b; good && pc < en; pc++) {
        int row;
        nl += local_piece(t, pc, &row) ? 1 : 0;
      }
      if (!good && warp == 0 && lane == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
    }
    if (!good) continue;
    const int64_t off = (u % nch) * kChunk;
    const int64_t nv = (rowbytes - off < kChunk ? rowbytes - off : kChunk) / 16;
    const int ng = stages_of(nl, kSlots);
    float acc[kVecPerLane][kEl];
    int left = nl;
    for (int g = 0; g < ng; g++, k++) {
      const int s = (int)(k % kStages);
      if (!mbar_wait(&full[s], (uint32_t)((k / kStages) & 1), t.wait_ns)) {
        ok = false;
        break;
      }
      const uint4 *slot = reinterpret_cast<const uint4 *>(stage_mem + (size_t)s * kSlots * kChunk);
      int q = 0;
      if (g == 0) {  // the home chunk starts the sum
#pragma unroll
        for (int j = 0; j < kVecPerLane; j++) {
          const int64_t v = (warp * kVecPerLane + j) * 32 + lane;
          const uint4 h = v < nv ? slot[v] : make_uint4(0, 0, 0, 0);
          const uint32_t wd[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
          for (int w = 0; w < 4; w++) {
            if constexpr (kF32) {
              acc[j][w] = __uint_as_float(wd[w]);
            } else {
              acc[j][2 * w] = bf16_lo(wd[w]);
              acc[j][2 * w + 1] = bf16_hi(wd[w]);
            }
          }
        }
        q = 1;
      }
      const int cap = g == 0 ? kSlots - 1 : kSlots;  // the first stage also holds the home chunk
      const int np = left < cap ? left : cap;
      left -= np;
      for (int pq = 0; pq < np; pq++, q++) {  // replicas in piece order
        const uint4 *sl = slot + (int64_t)q * (kChunk / 16);
#pragma unroll
        for (int j = 0; j < kVecPerLane; j++) {
          const int64_t v = (warp * kVecPerLane + j) * 32 + lane;
          const uint4 r = v < nv ? sl[v] : make_uint4(0, 0, 0, 0);
          const uint32_t wd[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int w = 0; w < 4; w++) {
            if constexpr (kF32) {
              acc[j][w] = __fadd_rn(acc[j][w], __uint_as_float(wd[w]));
            } else {
              acc[j][2 * w] = __fadd_rn(acc[j][2 * w], bf16_lo(wd[w]));
              acc[j][2 * w + 1] = __fadd_rn(acc[j][2 * w + 1], bf16_hi(wd[w]));
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!ok) break;
    uint4 *hrow = home + (int64_t)e * nvec + off / 16;
#pragma unroll
    for (int j = 0; j < kVecPerLane; j++) {
      const int64_t v = (warp * kVecPerLane + j) * 32 + lane;
      if (v < nv) {
        uint4 o;
        if constexpr (kF32) {
          o = make_uint4(__float_as_uint(acc[j][0]), __float_as_uint(acc[j][1]),
                         __float_as_uint(acc[j][2]), __float_as_uint(acc[j][3]));
        } else {
          o.x = pack_bf16x2(acc[j][0], acc[j][1]);
          o.y = pack_bf16x2(acc[j][2], acc[j][3]);
          o.z = pack_bf16x2(acc[j][4], acc[j][5]);
          o.w = pack_bf16x2(acc[j][6], acc[j][7]);
        }
        hrow[v] = o;
      }
    }
  }
  if (!ok && lane == 0) set_status(status, MOONEP_DEV_TIMEOUT);
}

// ------------------------------------------------ copy-through-buffer mode ---
// The zero_copy=False comparison path: pairs first land in a per-rank
// communication buffer in arrival order, then a permute copies them into the
// expert-ordered dispatch buffer (and back out before combine).
//
// comm_place: 64 tokens per CTA; each pair reserves its row in its destination
// rank's part of the buffer: a shared-memory count per destination, one global
// reservation per (CTA, destination), then the CTA-local position.  Arrival
// order inside a rank is unspecified (as it is for a real receiver).
constexpr int kCommTokensPerBlock = 64;

__global__ void __launch_bounds__(512)
comm_place_kernel(const int32_t *__restrict__ slot_of, int32_t *__restrict__ comm_index,
                  int32_t *__restrict__ counters, int64_t T, int K, int R, int64_t NvS,
                  int32_t *status) {
  pdl_wait();
  extern __shared__ int cs[];  // [R] local counts, then [R] global bases
  int *cnt = cs, *base = cs + R;
  for (int d = threadIdx.x; d < R; d += blockDim.x) cnt[d] = 0;
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * kCommTokensPerBlock;
  const int64_t np = (int64_t)kCommTokensPerBlock * K;
  const int64_t nrows = (int64_t)R * NvS;
  for (int64_t i = threadIdx.x; i < np; i += blockDim.x) {
    const int64_t p = t0 * K + i;
    if (p >= T * K) break;
    const int row = slot_of[p];
    if (row < 0 || row >= nrows) continue;
    atomicAdd(&cnt[row / NvS], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    base[d] = cnt[d] ? atomicAdd(&counters[d], cnt[d]) : 0;
    cnt[d] = 0;
  }
  __syncthreads();
  for (int64_t i = threadIdx.x; i < np; i += blockDim.x) {
    const int64_t p = t0 * K + i;
    if (p >= T * K) break;
    const int row = slot_of[p];
    if (row < 0 || row >= nrows) {
      comm_index[p] = -1;
      continue;
    }
    const int d = (int)(row / NvS);
    const int pos = base[d] + atomicAdd(&cnt[d], 1);
    if (pos >= NvS) {  // impossible when every rank receives S*K pairs
      set_status(status, MOONEP_DEV_BAD_PLAN);
      comm_index[p] = -1;
      continue;
    }
    comm_index[p] = (int32_t)(d * NvS + pos);
  }
}

// dst[dst_index[p]] = src[src_index[p]] for every pair, one warp per pair (rows of nvec vectors)
__global__ void __launch_bounds__(kThreads)
permute_rows_kernel(const int32_t *__restrict__ src_index, const int32_t *__restrict__ dst_index,
                    const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t npairs,
                    int64_t nvec, int64_t nrows) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t p = warp_g; p < npairs; p += nwarps) {
    const int a = __ldg(src_index + p), b = __ldg(dst_index + p);
    if (a < 0 || b < 0 || a >= nrows || b >= nrows) continue;
    const uint4 *s = src + (int64_t)a * nvec;
    uint4 *d = dst + (int64_t)b * nvec;
    for (int64_t v0 = 0; v0 < nvec; v0 += 32 * 4) {
      uint4 q[4];
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const int64_t v = v0 + u * 32 + lane;
        if (v < nvec) q[u] = __ldcs(s + v);
      }
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const int64_t v = v0 + u * 32 + lane;
        if (v < nvec) d[v] = q[u];
      }
    }
  }
}

// -------------------------------------------------------- prefetch_weight ---
// Work units: (replicated expert, warp-chunk of 32*U column vectors).  The home
// weight vectors are read once and stored into every local replica slot of the
// expert (the expert's pieces with a weight slot).
template <int U>
__global__ void __launch_bounds__(kThreads)
prefetch_weight_vec_kernel(const int32_t *__restrict__ replicated, const int32_t *__restrict__ scalars,
                           const int32_t *__restrict__ pbeg, const int32_t *__restrict__ pend,
                           const int32_t *__restrict__ prank, const int32_t *__restrict__ pwslot,
                           const uint4 *__restrict__ w, uint4 *__restrict__ rep_w, int64_t nvec,
                           int R, int E, int B, int PMAX, int32_t *status) {
  pdl_wait();
  int64_t n_exp = scalars[S_N_REPLICATED];
  if (n_exp < 0 || n_exp > E) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
    n_exp = 0;
  }
  const int64_t per_exp = (nvec + 32 * U - 1) / (32 * U);
  const int64_t total = n_exp * per_exp;
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerBlock;
  for (int64_t wk = warp_g; wk < total; wk += nwarps) {
    const int e = replicated[wk / per_exp];
    const int64_t v0 = (wk % per_exp) * 32 * U;
    const int b = e >= 0 && e < E ? pbeg[e] : 0, en = e >= 0 && e < E ? pend[e] : -1;
    if (e < 0 || e >= E || b < 0 || en > PMAX || en < b) {
      if (lane == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
      continue;
    }
    const uint4 *src = w + (int64_t)e * nvec;
    uint4 q[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t v = v0 + u * 32 + lane;
      q[u] = v < nvec ? __ldcs(src + v) : make_uint4(0, 0, 0, 0);
    }
    for (int pc = b; pc < en; pc++) {
      const int ws = pwslot[pc], rk = prank[pc];
      if (ws < 0) continue;
      if (ws >= B || rk < 0 || rk >= R) {
        if (lane == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
        continue;
      }
      uint4 *dst = rep_w + ((int64_t)rk * B + ws) * nvec;
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int64_t v = v0 + u * 32 + lane;
        if (v < nvec) dst[v] = q[u];
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
prefetch_weight_scalar_kernel(const int32_t *__restrict__ replicated, const int32_t *__restrict__ scalars,
                              const int32_t *__restrict__ pbeg, const int32_t *__restrict__ pend,
                              const int32_t *__restrict__ prank, const int32_t *__restrict__ pwslot,
                              const uint16_t *__restrict__ w, uint16_t *__restrict__ rep_w, int64_t W,
                              int R, int E, int B, int PMAX, int32_t *status) {
  pdl_wait();
  int64_t n_exp = scalars[S_N_REPLICATED];
  if (n_exp < 0 || n_exp > E) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
    n_exp = 0;
  }
  const int64_t total = n_exp * W;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
    const int e = replicated[q / W];
    const int64_t c = q % W;
    const int b = e >= 0 && e < E ? pbeg[e] : 0, en = e >= 0 && e < E ? pend[e] : -1;
    if (e < 0 || e >= E || b < 0 || en > PMAX || en < b) {
      set_status(status, MOONEP_DEV_BAD_PLAN);
      continue;
    }
    const uint16_t v = w[(int64_t)e * W + c];
    for (int pc = b; pc < en; pc++) {
      const int ws = pwslot[pc], rk = prank[pc];
      if (ws < 0) continue;
      if (ws >= B || rk < 0 || rk >= R) {
        set_status(status, MOONEP_DEV_BAD_PLAN);
        continue;
      }
      rep_w[((int64_t)rk * B + ws) * W + c] = v;
    }
  }
}

// reduce_grad's scalar path (rows not in whole aligned 16-byte vectors): one value of
// a replicated expert's row per thread, the same fp32 additions in piece order.
// Gradient values of either type read as fp32 and stored back in their own type.
__device__ __forceinline__ float grad_to_f(uint16_t b) { return bf16_to_f(b); }
__device__ __forceinline__ float grad_to_f(float v) { return v; }
__device__ __forceinline__ void grad_store(uint16_t *p, float v) { *p = f_to_bf16(v); }
__device__ __forceinline__ void grad_store(float *p, float v) { *p = v; }

template <class T>
__global__ void __launch_bounds__(kThreads)
reduce_grad_scalar_kernel(const int32_t *__restrict__ replicated, const int32_t *__restrict__ scalars,
                          const int32_t *__restrict__ pbeg, const int32_t *__restrict__ pend,
                          const int32_t *__restrict__ prank, const int32_t *__restrict__ pwslot,
                          const T *__restrict__ rep, T *__restrict__ home, int64_t P,
                          int R, int E, int B, int PMAX, int32_t *status) {
  pdl_wait();
  int64_t n_exp = scalars[S_N_REPLICATED];
  if (n_exp < 0 || n_exp > E) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, MOONEP_DEV_BAD_PLAN);
    n_exp = 0;
  }
  const int64_t total = n_exp * P;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
    const int e = replicated[q / P];
    const int64_t c = q % P;
    const int b = e >= 0 && e < E ? pbeg[e] : 0, en = e >= 0 && e < E ? pend[e] : -1;
    if (e < 0 || e >= E || b < 0 || en > PMAX || en < b) {
      set_status(status, MOONEP_DEV_BAD_PLAN);
      continue;
    }
    float acc = grad_to_f(home[(int64_t)e * P + c]);
    for (int pc = b; pc < en; pc++) {
      const int ws = pwslot[pc], rk = prank[pc];
      if (ws < 0) continue;
      if (ws >= B || rk < 0 || rk >= R) {
        set_status(status, MOONEP_DEV_BAD_PLAN);
        continue;
      }
      acc = __fadd_rn(acc, grad_to_f(rep[((int64_t)rk * B + ws) * P + c]));
    }
    grad_store(home + (int64_t)e * P + c, acc);
  }
}

int num_sms() { return current_sm_count(); }

// Co-resident CTAs per SM of reduce_grad_bulk_kernel<kF32>, -1 on a CUDA error.  Its
// shared memory limit is a per-context function attribute: it is raised once per CUDA
// context and the occupancy answer is kept with the context id, per device and per
// instantiation.
template <bool kF32>
int rg_blocks_per_sm() {
  static std::mutex mu;
  static unsigned long long ctx_of[kMaxDevices];
  static int per_sm_of[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return -1;
  }
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(mu);
  if (ctx != 0 && ctx_of[dev] == ctx && per_sm_of[dev] > 0) return per_sm_of[dev];
  int per_sm = 0;
  if (cudaFuncSetAttribute(reduce_grad_bulk_kernel<kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           rg::kSmem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reduce_grad_bulk_kernel<kF32>, rg::kThreadsRg,
                                                    rg::kSmem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    return -1;
  }
  ctx_of[dev] = ctx;
  per_sm_of[dev] = per_sm;
  return per_sm;
}

// combine_vec_k_kernel's units: whole tokens, or column halves (split = 1) when the
// tokens would fill fewer than eight waves of the resident warps (two 8-warp CTAs per
// SM); a half is a multiple of 64 vectors, the kernel's column step.
struct CombineSplit {
  int split;
  int64_t cl;
};
CombineSplit combine_split(int64_t T, int64_t nvec) {
  const int64_t resident = (int64_t)num_sms() * 2 * kWarpsPerBlock;
  if (T >= 8 * resident || nvec < 128) return {0, nvec};
  return {1, ((nvec + 1) / 2 + 63) / 64 * 64};
}

unsigned token_grid(int64_t T) {
  int64_t blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int64_t cap = (int64_t)num_sms() * 64;
  if (blocks > cap) blocks = cap;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

bool data_dims(const moonep_config_t *cfg, Dims *d) {
  return make_dims(cfg, d) && d->H >= 1;
}

}  // namespace

}  // namespace moonep

using namespace moonep;

extern "C" moonep_status_t moonep_dispatch(const moonep_config_t *cfg, const void *plan_arena,
                                           const uint16_t *x, uint16_t *recv, int32_t *dev_status,
                                           moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!x || !recv || !aligned256(plan_arena)) return MOONEP_ERR_INVALID_ARG;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS;
  if (d.H % 8 == 0 && aligned16(x) && aligned16(recv)) {
    const RowChunks rc = row_chunks<kDispatchU>(d.H / 8);
    launch(dispatch_chunk_kernel<kDispatchU>, token_grid(T * rc.nch), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(recv), T,
        (int)d.K, d.H / 8, rc.nch, rc.cl, nrows, dev_status);
  } else {
    launch(dispatch_scalar_kernel, token_grid(T), kThreads, 0, st, P.f[F_SLOT_OF], x, recv, T, (int)d.K,
        d.H, nrows, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" moonep_status_t moonep_combine(const moonep_config_t *cfg, const void *plan_arena,
                                          const uint16_t *y, const float *gates, uint16_t *out,
                                          int32_t *dev_status, moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!y || !gates || !out || !aligned256(plan_arena)) return MOONEP_ERR_INVALID_ARG;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS;
  if (d.H % 8 == 0 && aligned16(y) && aligned16(out) && d.K <= 8) {
    const CombineSplit cs = combine_split(T, d.H / 8);
    launch((combine_vec_k_kernel<2, 8>), token_grid(T << cs.split), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(y), gates, reinterpret_cast<uint4 *>(out),
        T, (int)d.K, d.H / 8, cs.split, cs.cl, nrows, dev_status);
  } else if (d.H % 8 == 0 && aligned16(y) && aligned16(out)) {
    launch(combine_vec_kernel<4>, token_grid(T), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(y), gates, reinterpret_cast<uint4 *>(out),
        T, (int)d.K, d.H / 8, nrows, dev_status);
  } else {
    launch(combine_scalar_kernel, token_grid(T), kThreads, 0, st, P.f[F_SLOT_OF], y, gates, out, T,
        (int)d.K, d.H, nrows, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" moonep_status_t moonep_combine_backward(const moonep_config_t *cfg,
                                                   const void *plan_arena, const uint16_t *dout,
                                                   const uint16_t *y, const float *gates,
                                                   uint16_t *dy, float *dgates,
                                                   int32_t *dev_status, moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!dout || !y || !gates || !dy || !dgates || !aligned256(plan_arena))
    return MOONEP_ERR_INVALID_ARG;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS;
  const bool vec = d.H % 8 == 0 && aligned16(dout) && aligned16(y) && aligned16(dy);
  if (vec && d.K <= 8) {
    // two warps per token measured 6.5 TB/s against 6.1 for one
    launch((combine_bwd_split_kernel<2, 8>), token_grid(2 * T), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(dout), reinterpret_cast<const uint4 *>(y),
        gates, reinterpret_cast<uint4 *>(dy), dgates, T, (int)d.K, d.H / 8, nrows, dev_status);
  } else if (vec) {
    launch(combine_bwd_vec_kernel<4>, token_grid(T), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(dout), reinterpret_cast<const uint4 *>(y),
        gates, reinterpret_cast<uint4 *>(dy), dgates, T, (int)d.K, d.H / 8, nrows, dev_status);
  } else {
    launch(combine_bwd_scalar_kernel, token_grid(T), kThreads, 0, st,
        P.f[F_SLOT_OF], dout, y, gates, dy, dgates, T, (int)d.K, d.H, nrows, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

namespace {
// reduce_grad over gradient rows of T (bf16 bits or fp32): the bulk-copy pipeline when
// rows are whole 16-byte vectors at 16-byte aligned bases, else the scalar kernel.
template <class T>
moonep_status_t reduce_grad_impl(const moonep_config_t *cfg, const void *plan_arena, const T *rep_grads,
                                 T *home_grads, int64_t P_elems, int32_t *dev_status,
                                 moonep_stream_t stream) {
  constexpr bool kF32 = sizeof(T) == 4;
  constexpr int64_t kPerVec = 16 / sizeof(T);
  Dims d;
  if (!make_dims(cfg, &d) || !plan_arena || !dev_status || P_elems < 1)
    return MOONEP_ERR_INVALID_ARG;
  if (!home_grads || (d.B > 0 && !rep_grads) || !aligned256(plan_arena))
    return MOONEP_ERR_INVALID_ARG;
  if (d.B == 0) return MOONEP_OK;  // no replica slots, nothing to fold
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  if (P_elems % kPerVec == 0 && aligned16(rep_grads) && aligned16(home_grads)) {
    const int per_sm = rg_blocks_per_sm<kF32>();
    if (per_sm < 1) return MOONEP_ERR_CUDA;
    const rg::Tables t{P.f[F_REPLICATED], P.f[F_SCALARS], P.f[F_EXP_PIECE_BEGIN],
                       P.f[F_EXP_PIECE_END], P.f[F_PIECE_RANK], P.f[F_PIECE_WSLOT],
                       (int)d.R, (int)d.E, (int)d.B, (int)d.PMAX, debug_wait_limit_ns(),
                       debug_phantom() > 0 ? 16 * debug_phantom() : 0};
    launch(reduce_grad_bulk_kernel<kF32>, (unsigned)(num_sms() * per_sm), rg::kThreadsRg, rg::kSmem, st,
        t, reinterpret_cast<const uint4 *>(rep_grads), reinterpret_cast<uint4 *>(home_grads),
        P_elems / kPerVec, dev_status);
  } else {
    launch(reduce_grad_scalar_kernel<T>, (unsigned)num_sms() * 8, kThreads, 0, st,
        P.f[F_REPLICATED], P.f[F_SCALARS], P.f[F_EXP_PIECE_BEGIN], P.f[F_EXP_PIECE_END],
        P.f[F_PIECE_RANK], P.f[F_PIECE_WSLOT], rep_grads, home_grads, P_elems, (int)d.R,
        (int)d.E, (int)d.B, (int)d.PMAX, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}
}  // namespace

extern "C" moonep_status_t moonep_reduce_grad(const moonep_config_t *cfg, const void *plan_arena,
                                              const uint16_t *rep_grads, uint16_t *home_grads,
                                              int64_t P_elems, int32_t *dev_status,
                                              moonep_stream_t stream) {
  return reduce_grad_impl(cfg, plan_arena, rep_grads, home_grads, P_elems, dev_status, stream);
}

extern "C" moonep_status_t moonep_reduce_grad_f32(const moonep_config_t *cfg, const void *plan_arena,
                                                  const float *rep_grads, float *home_grads,
                                                  int64_t P_elems, int32_t *dev_status,
                                                  moonep_stream_t stream) {
  return reduce_grad_impl(cfg, plan_arena, rep_grads, home_grads, P_elems, dev_status, stream);
}

extern "C" moonep_status_t moonep_dispatch_backward(const moonep_config_t *cfg,
                                                    const void *plan_arena, const uint16_t *d_recv,
                                                    uint16_t *dx, int32_t *dev_status,
                                                    moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!d_recv || !dx || !aligned256(plan_arena)) return MOONEP_ERR_INVALID_ARG;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS;
  // the combine kernels with unit weights: fmaf(1, y, acc) rounds like acc + y
  if (d.H % 8 == 0 && aligned16(d_recv) && aligned16(dx) && d.K <= 8) {
    const CombineSplit cs = combine_split(T, d.H / 8);
    launch((combine_vec_k_kernel<2, 8>), token_grid(T << cs.split), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(d_recv), nullptr,
        reinterpret_cast<uint4 *>(dx), T, (int)d.K, d.H / 8, cs.split, cs.cl, nrows, dev_status);
  } else if (d.H % 8 == 0 && aligned16(d_recv) && aligned16(dx)) {
    launch(combine_vec_kernel<4>, token_grid(T), kThreads, 0, st,
        P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(d_recv), nullptr,
        reinterpret_cast<uint4 *>(dx), T, (int)d.K, d.H / 8, nrows, dev_status);
  } else {
    launch(combine_scalar_kernel, token_grid(T), kThreads, 0, st, P.f[F_SLOT_OF], d_recv, nullptr, dx,
        T, (int)d.K, d.H, nrows, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" moonep_status_t moonep_prefetch_weight(const moonep_config_t *cfg,
                                                  const void *plan_arena, const uint16_t *weights,
                                                  uint16_t *rep_weights, int64_t W,
                                                  int32_t *dev_status, moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d) || !plan_arena || !dev_status || W < 1) return MOONEP_ERR_INVALID_ARG;
  if (!weights || (d.B > 0 && !rep_weights) || !aligned256(plan_arena))
    return MOONEP_ERR_INVALID_ARG;
  if (d.B == 0) return MOONEP_OK;  // no replica slots: every duplicate reads remotely
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  if (W % 8 == 0 && aligned16(weights) && aligned16(rep_weights)) {
    // many small blocks: the block scheduler balances the expert-major units
    const unsigned grid = (unsigned)num_sms() * 64;
    launch(prefetch_weight_vec_kernel<8>, grid, kThreads, 0, st,
        P.f[F_REPLICATED], P.f[F_SCALARS], P.f[F_EXP_PIECE_BEGIN], P.f[F_EXP_PIECE_END],
        P.f[F_PIECE_RANK], P.f[F_PIECE_WSLOT], reinterpret_cast<const uint4 *>(weights),
        reinterpret_cast<uint4 *>(rep_weights), W / 8, (int)d.R, (int)d.E, (int)d.B, (int)d.PMAX,
        dev_status);
  } else {
    launch(prefetch_weight_scalar_kernel, (unsigned)num_sms() * 8, kThreads, 0, st,
        P.f[F_REPLICATED], P.f[F_SCALARS], P.f[F_EXP_PIECE_BEGIN], P.f[F_EXP_PIECE_END],
        P.f[F_PIECE_RANK], P.f[F_PIECE_WSLOT], weights, rep_weights, W, (int)d.R, (int)d.E,
        (int)d.B, (int)d.PMAX, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

namespace {
unsigned pair_grid(int64_t npairs) {
  int64_t blocks = (npairs + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int64_t cap = (int64_t)num_sms() * 64;
  if (blocks > cap) blocks = cap;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}
}  // namespace

extern "C" moonep_status_t moonep_dispatch_via_buffer(const moonep_config_t *cfg,
                                                      const void *plan_arena, const uint16_t *x,
                                                      uint16_t *comm, int32_t *comm_index,
                                                      uint16_t *recv, int32_t *dev_status,
                                                      moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!x || !comm || !comm_index || !recv || !aligned256(plan_arena)) return MOONEP_ERR_INVALID_ARG;
  if (d.H % 8 != 0 || !aligned16(x) || !aligned16(comm) || !aligned16(recv))
    return MOONEP_ERR_UNSUPPORTED;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS, N = T * d.K;
  int32_t *counters = comm_index + N;
  if (cudaMemsetAsync(counters, 0, sizeof(int32_t) * d.R, st) != cudaSuccess) return MOONEP_ERR_CUDA;
  const unsigned blocks = (unsigned)((T + kCommTokensPerBlock - 1) / kCommTokensPerBlock);
  launch(comm_place_kernel, blocks, 512, 2 * d.R * sizeof(int), st, P.f[F_SLOT_OF], comm_index, counters,
      T, (int)d.K, (int)d.R, d.NvS,
      dev_status);
  // the sender writes rows into the receivers' communication buffers
  const RowChunks rc = row_chunks<kDispatchU>(d.H / 8);
  launch(dispatch_chunk_kernel<kDispatchU>, token_grid(T * rc.nch), kThreads, 0, st,
      comm_index, reinterpret_cast<const uint4 *>(x), reinterpret_cast<uint4 *>(comm), T, (int)d.K,
      d.H / 8, rc.nch, rc.cl, nrows, dev_status);
  // the receiver permutes them into expert order
  launch(permute_rows_kernel, pair_grid(N), kThreads, 0, st,
      comm_index, P.f[F_SLOT_OF], reinterpret_cast<const uint4 *>(comm),
      reinterpret_cast<uint4 *>(recv), N, d.H / 8, nrows);
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" moonep_status_t moonep_combine_via_buffer(const moonep_config_t *cfg,
                                                     const void *plan_arena, const uint16_t *y,
                                                     const float *gates, const int32_t *comm_index,
                                                     uint16_t *comm, uint16_t *out,
                                                     int32_t *dev_status, moonep_stream_t stream) {
  Dims d;
  if (!data_dims(cfg, &d) || !plan_arena || !dev_status) return MOONEP_ERR_INVALID_ARG;
  const int64_t T = d.R * d.S;
  if (T == 0) return MOONEP_OK;
  if (!y || !gates || !comm_index || !comm || !out || !aligned256(plan_arena))
    return MOONEP_ERR_INVALID_ARG;
  if (d.H % 8 != 0 || !aligned16(y) || !aligned16(comm) || !aligned16(out))
    return MOONEP_ERR_UNSUPPORTED;
  PlanPtrs P = plan_ptrs(d, plan_arena);
  cudaStream_t st = to_cuda(stream);
  const int64_t nrows = d.R * d.NvS, N = T * d.K;
  // the expert ranks permute their outputs back into arrival order
  launch(permute_rows_kernel, pair_grid(N), kThreads, 0, st,
      P.f[F_SLOT_OF], comm_index, reinterpret_cast<const uint4 *>(y), reinterpret_cast<uint4 *>(comm),
      N, d.H / 8, nrows);
  // and the source ranks combine from the communication buffer
  if (d.K <= 8) {
    const CombineSplit cs = combine_split(T, d.H / 8);
    launch((combine_vec_k_kernel<2, 8>), token_grid(T << cs.split), kThreads, 0, st,
        comm_index, reinterpret_cast<const uint4 *>(comm), gates, reinterpret_cast<uint4 *>(out), T,
        (int)d.K, d.H / 8, cs.split, cs.cl, nrows, dev_status);
  } else {
    launch(combine_vec_kernel<4>, token_grid(T), kThreads, 0, st,
        comm_index, reinterpret_cast<const uint4 *>(comm), gates, reinterpret_cast<uint4 *>(out), T,
        (int)d.K, d.H / 8, nrows, dev_status);
  }
  return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" const char *moonep_status_string(moonep_status_t s) {
  switch (s) {
    case MOONEP_OK: return "ok";
    case MOONEP_ERR_INVALID_ARG: return "invalid argument (config out of range, null or misaligned pointer)";
    case MOONEP_ERR_CUDA: return "CUDA launch or runtime error";
    case MOONEP_ERR_UNSUPPORTED: return "sizes past the supported limits";
  }
  return "unknown status";
}
