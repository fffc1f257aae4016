// Balanced plan for MoonEP-style expert parallelism ("Moonshot AI Open-Sources
// MoonEP": every rank receives exactly S*K token-slots, overloaded experts are
// duplicated onto underloaded ranks within a replica-slot budget;
// "MoonshotAI/MoonEP 딥다이브" §4 pattern 1: planned once per layer, reused).
//
// Two kernels:
//   plan_hist_solve  one CTA per chunk of 8192 (rank, token, k) pairs.  Each CTA
//                    builds its chunk's per-expert histogram and the stable rank
//                    of every pair among the chunk's pairs of the same expert
//                    (warp-private counters + __match_any_sync, so a hot expert
//                    never serialises on an atomic).  The last CTA to finish
//                    (arrival counter; no CTA ever waits for another) scans the
//                    histograms per expert into per-chunk bases and solves the
//                    O(E + R) balance problem in shared memory.
//   plan_place       every pair's final row: position inside its expert's list
//                    = chunk base + stable rank; the first kept_e positions stay
//                    in the home segment, the rest map through the piece table.
#include <atomic>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

__device__ __forceinline__ int roundup_i(int v, int a) { return (v + a - 1) / a * a; }

// Exclusive scan of s[0, n) in shared memory, in place; every thread of the block
// calls it.  scratch: 33 ints of shared memory.  Returns the total.
__device__ int block_excl_scan(int *s, int n, int *scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int b = tid * per < n ? tid * per : n;
  const int e = b + per < n ? b + per : n;
  int sum = 0;
  for (int i = b; i < e; i++) sum += s[i];
  const int incl = warp_incl_scan(sum);
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nwarps ? scratch[lane] : 0;
    const int wi = warp_incl_scan(v);
    if (lane < nwarps) scratch[lane] = wi - v;
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  int run = scratch[warp] + incl - sum;
  for (int i = b; i < e; i++) {
    const int v = s[i];
    s[i] = run;
    run += v;
  }
  const int total = scratch[32];
  __syncthreads();
  return total;
}

// first index i in [0, n) with a[i] > v (n if none); a non-decreasing
__device__ __forceinline__ int upper_bound_i(const int *a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > v) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// first index i in [0, n) with a[i] >= v
__device__ __forceinline__ int lower_bound_i(const int *a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] >= v) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// --------------------------------------------------------------- the solve --
// Runs in the last CTA of plan_hist_solve.  hist[c*E + e] holds chunk c's
// count of expert e on entry and the exclusive per-expert prefix on exit.
__device__ void solve(const Dims &d, int *smem, PlanPtrs P, int32_t *wsflags, int32_t *hist,
                      int32_t *exp_kept, int32_t *exp_row0, int32_t *exp_ostart,
                      int32_t *piece_grow, int32_t *status) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int E = (int)d.E, R = (int)d.R, L = (int)d.L, A = (int)d.A, B = (int)d.B;
  const int SK = (int)d.SK, NvS = (int)d.NvS;
  const int64_t NC = d.NC;
  const int PMAX = (int)d.PMAX;

  int *s = smem;
  int *s_cnt = s; s += E;
  int *s_cst = s; s += E;   // offset of the expert's list inside its home stream
  int *s_kept = s; s += E;
  int *s_ost = s; s += E;   // offset of the expert's first leaving entry in the overflow stream
  int *s_npc = s; s += E;   // pieces of the expert
  int *s_pbeg = s; s += E;  // first piece id of the expert
  int *s_nst = s; s += E;   // start row of the expert's native segment within its rank
  int *s_i0 = s; s += E;    // first receiver index of the expert's pieces
  int *s_flag = s; s += E;  // expert has a local replica piece
  int *s_load = s; s += R;
  int *s_hbase = s; s += R;
  int *s_over = s; s += R;
  int *s_def = s; s += R;
  int *s_obase = s; s += R;
  int *s_dbase = s; s += R;
  int *s_ridx = s; s += R;  // receiver index of a rank, -1 if it receives nothing
  int *s_nbase = s; s += R;
  int *s_ntot = s; s += R;  // rows used by the rank's native segments
  int *s_rrank = s; s += R; // per receiver index i (< n_recv)
  int *s_rbase = s; s += R;
  int *s_rend = s; s += R;
  int *s_rfirst = s; s += R;
  int *s_rcount = s; s += R;
  int *s_rpbase = s; s += R;
  int *s_pexp = s; s += PMAX;
  int *s_precv = s; s += PMAX;
  int *s_post = s; s += PMAX;
  int *s_plen = s; s += PMAX;
  int *s_pj = s; s += PMAX;
  int *s_pst = s; s += PMAX;
  int *scratch = s; s += 40;  // [0..32] scan scratch, [33..39] block-wide values

  const bool bad_ids = __ldcg(wsflags + 1) != 0;

  // S1: per-expert exclusive scan over chunks; G lanes share one expert column.
  {
    int G = 1;
    while (G < 32 && 2 * G * E <= nt) G *= 2;
    const int grp = tid / G, sub = tid % G, ngrp = nt / G;
    const int per = (int)((NC + G - 1) / G);
    for (int e0 = 0; e0 < E; e0 += ngrp) {
      const int e = e0 + grp;
      const bool act = e < E;
      const int c0 = sub * per;
      const int c1 = (int)(c0 + per < NC ? c0 + per : NC);
      int sum = 0;
      if (act) {
        int c = c0;
        for (; c + 16 <= c1; c += 16) {
          int v[16];
#pragma unroll
          for (int u = 0; u < 16; u++) v[u] = __ldcg(hist + (int64_t)(c + u) * E + e);
#pragma unroll
          for (int u = 0; u < 16; u++) sum += v[u];
        }
        for (; c < c1; c++) sum += __ldcg(hist + (int64_t)c * E + e);
      }
      // exclusive scan of the G partial sums inside the group
      int incl = sum;
      for (int o = 1; o < G; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o, G);
        if (sub >= o) incl += n;
      }
      int run = incl - sum;
      const int total = __shfl_sync(0xffffffffu, incl, G - 1, G);
      if (act) {
        int c = c0;
        for (; c + 16 <= c1; c += 16) {
          int v[16];
#pragma unroll
          for (int u = 0; u < 16; u++) v[u] = __ldcg(hist + (int64_t)(c + u) * E + e);
#pragma unroll
          for (int u = 0; u < 16; u++) {
            hist[(int64_t)(c + u) * E + e] = run;
            run += v[u];
          }
        }
        for (; c < c1; c++) {
          const int v = __ldcg(hist + (int64_t)c * E + e);
          hist[(int64_t)c * E + e] = run;
          run += v;
        }
        if (sub == 0) s_cnt[e] = total;
      }
    }
  }
  __syncthreads();

  // S2: rank loads and each expert's offset inside its home stream
  for (int e = tid; e < E; e += nt) s_cst[e] = s_cnt[e];
  __syncthreads();
  const int total_pairs = block_excl_scan(s_cst, E, scratch);
  for (int h = tid; h < R; h += nt) {
    const int lo = s_cst[h * L];
    const int hi = (h + 1) * L < E ? s_cst[(h + 1) * L] : total_pairs;
    s_hbase[h] = lo;
    s_load[h] = hi - lo;
    s_over[h] = hi - lo > SK ? hi - lo - SK : 0;
    s_def[h] = hi - lo < SK ? SK - (hi - lo) : 0;
    s_obase[h] = s_over[h];
    s_dbase[h] = s_def[h];
    s_ridx[h] = s_def[h] > 0 ? 1 : 0;
  }
  __syncthreads();
  for (int e = tid; e < E; e += nt) s_cst[e] -= s_hbase[e / L];
  block_excl_scan(s_obase, R, scratch);
  block_excl_scan(s_dbase, R, scratch);
  const int n_recv = block_excl_scan(s_ridx, R, scratch);
  for (int h = tid; h < R; h += nt) {
    if (s_def[h] > 0) {
      const int i = s_ridx[h];
      s_rrank[i] = h;
      s_rbase[i] = s_dbase[h];
      s_rend[i] = s_dbase[h] + s_def[h];
      s_rfirst[i] = 0;
      s_rcount[i] = 0;
    } else {
      s_ridx[h] = -1;
    }
  }
  __syncthreads();

  // S3: kept rows, overflow position and piece count of every expert
  for (int e = tid; e < E; e += nt) {
    const int cnt = s_cnt[e], cst = s_cst[e], h = e / L;
    int kept = SK - cst;
    kept = kept < 0 ? 0 : (kept > cnt ? cnt : kept);
    const int ovf = cnt - kept;
    const int ost = s_obase[h] + (cst > SK ? cst - SK : 0);
    s_kept[e] = kept;
    s_ost[e] = ost;
    int npc = 0, i0 = 0;
    if (ovf > 0 && !bad_ids && n_recv > 0) {
      i0 = upper_bound_i(s_rend, n_recv, ost);
      int i1 = lower_bound_i(s_rend, n_recv, ost + ovf);
      if (i1 >= n_recv) i1 = n_recv - 1;
      if (i0 < n_recv) npc = i1 - i0 + 1;
    }
    s_npc[e] = npc;
    s_pbeg[e] = npc;
    s_i0[e] = i0;
    s_nst[e] = roundup_i(kept, A);
  }
  __syncthreads();
  int n_piece = block_excl_scan(s_pbeg, E, scratch);
  if (n_piece > PMAX) n_piece = PMAX;  // cannot happen: pieces <= experts + receivers - 1
  const int native_rows = block_excl_scan(s_nst, E, scratch);
  for (int h = tid; h < R; h += nt) {
    const int lo = s_nst[h * L];
    const int hi = (h + 1) * L < E ? s_nst[(h + 1) * L] : native_rows;
    s_nbase[h] = lo;
    s_ntot[h] = hi - lo;
  }
  __syncthreads();
  for (int e = tid; e < E; e += nt) s_nst[e] -= s_nbase[e / L];

  // S4: pieces = intersections of expert overflow ranges with receiver ranges
  for (int e = tid; e < E; e += nt) {
    const int npc = s_npc[e];
    if (npc == 0) continue;
    const int ost = s_ost[e], oend = ost + (s_cnt[e] - s_kept[e]);
    for (int q = 0; q < npc; q++) {
      const int i = s_i0[e] + q, pid = s_pbeg[e] + q;
      if (pid >= PMAX) break;
      const int os = ost > s_rbase[i] ? ost : s_rbase[i];
      const int oe = oend < s_rend[i] ? oend : s_rend[i];
      s_pexp[pid] = e;
      s_precv[pid] = i;
      s_post[pid] = os;
      s_plen[pid] = oe - os;
      if (os == s_rbase[i]) s_rfirst[i] = pid;
    }
  }
  __syncthreads();
  for (int pid = tid; pid < n_piece; pid += nt) {
    const int i = s_precv[pid];
    const int j = pid - s_rfirst[i];
    s_pj[pid] = j;
    if (s_post[pid] + s_plen[pid] == s_rend[i]) s_rcount[i] = j + 1;
    s_pst[pid] = roundup_i(s_plen[pid], A);
  }
  __syncthreads();
  block_excl_scan(s_pst, n_piece, scratch);
  for (int i = tid; i < n_recv; i += nt) s_rpbase[i] = s_pst[s_rfirst[i]];
  if (tid == 0) { scratch[33] = 0; scratch[34] = 0; scratch[35] = 0; scratch[36] = 0; }
  __syncthreads();
  for (int pid = tid; pid < n_piece; pid += nt) {
    const int i = s_precv[pid];
    s_pst[pid] = s_ntot[s_rrank[i]] + s_pst[pid] - s_rpbase[i];
  }
  __syncthreads();

  // capacity: every rank's rows must end inside NvS (true by construction)
  for (int h = tid; h < R; h += nt) {
    int used = s_ntot[h];
    const int i = s_ridx[h];
    if (i >= 0 && s_rcount[i] > 0) {
      const int last = s_rfirst[i] + s_rcount[i] - 1;
      used = s_pst[last] + s_plen[last];
    }
    if (used > NvS) atomicOr(&scratch[33], 1);
  }
  // remote pieces and experts with a local replica
  for (int e = tid; e < E; e += nt) s_flag[e] = 0;
  __syncthreads();
  for (int pid = tid; pid < n_piece; pid += nt) {
    if (s_pj[pid] >= B) atomicAdd(&scratch[34], 1);
    else s_flag[s_pexp[pid]] = 1;
  }
  __syncthreads();
  const bool capacity_bad = scratch[33] != 0;
  const int n_remote = scratch[34];
  // compact list of experts with a local replica (ascending)
  for (int e = tid; e < E; e += nt) s_i0[e] = s_flag[e];
  __syncthreads();
  const int n_replicated = block_excl_scan(s_i0, E, scratch);

  // S5: outputs
  int32_t *o_count = P.f[F_EXPERT_COUNT];
  for (int e = tid; e < E; e += nt) {
    const int h = e / L;
    o_count[e] = s_cnt[e];
    P.f[F_EXP_PIECE_BEGIN][e] = s_pbeg[e];
    P.f[F_EXP_PIECE_END][e] = s_pbeg[e] + s_npc[e];
    exp_kept[e] = s_kept[e];
    exp_row0[e] = h * NvS + s_nst[e];
    exp_ostart[e] = s_ost[e];
    const int si = h * E + (e - h * L);
    P.f[F_SEG_EXPERT][si] = e;
    P.f[F_SEG_START][si] = s_nst[e];
    P.f[F_SEG_LEN][si] = s_kept[e];
    P.f[F_SEG_KIND][si] = MOONEP_SEG_NATIVE;
    P.f[F_SEG_WSLOT][si] = -1;
    if (s_flag[e]) P.f[F_REPLICATED][s_i0[e]] = e;
  }
  for (int h = tid; h < R; h += nt) {
    P.f[F_RANK_LOAD][h] = s_load[h];
    P.f[F_OVERFLOW][h] = s_over[h];
    P.f[F_DEFICIT][h] = s_def[h];
    const int i = s_ridx[h];
    P.f[F_N_SEG][h] = L + (i >= 0 ? s_rcount[i] : 0);
  }
  for (int pid = tid; pid < n_piece; pid += nt) {
    const int i = s_precv[pid], dr = s_rrank[i], j = s_pj[pid];
    const int e = s_pexp[pid];
    const int ws = j < B ? j : -1;
    P.f[F_PIECE_EXPERT][pid] = e;
    P.f[F_PIECE_RANK][pid] = dr;
    P.f[F_PIECE_START][pid] = s_pst[pid];
    P.f[F_PIECE_LEN][pid] = s_plen[pid];
    P.f[F_PIECE_WSLOT][pid] = ws;
    P.f[F_PIECE_OSTART][pid] = s_post[pid];
    piece_grow[pid] = dr * NvS + s_pst[pid];
    if (L + j < E) {
      const int si = dr * E + L + j;
      P.f[F_SEG_EXPERT][si] = e;
      P.f[F_SEG_START][si] = s_pst[pid];
      P.f[F_SEG_LEN][si] = s_plen[pid];
      P.f[F_SEG_KIND][si] = ws >= 0 ? MOONEP_SEG_REPLICA : MOONEP_SEG_REMOTE;
      P.f[F_SEG_WSLOT][si] = ws;
    }
  }
  for (int64_t q = tid; q < d.R * d.E; q += nt) {
    const int h = (int)(q / E), i = (int)(q % E);
    const int ri = s_ridx[h];
    const int nseg = L + (ri >= 0 ? s_rcount[ri] : 0);
    if (i >= nseg) {
      P.f[F_SEG_EXPERT][q] = -1;
      P.f[F_SEG_START][q] = 0;
      P.f[F_SEG_LEN][q] = 0;
      P.f[F_SEG_KIND][q] = -1;
      P.f[F_SEG_WSLOT][q] = -1;
    }
  }
  for (int64_t q = tid; q < d.R * d.B; q += nt) {
    const int h = (int)(q / B), j = (int)(q % B);
    const int ri = s_ridx[h];
    P.f[F_REP_EXPERT][q] = (ri >= 0 && j < s_rcount[ri]) ? s_pexp[s_rfirst[ri] + j] : -1;
  }
  if (tid == 0) {
    int32_t *sc = P.f[F_SCALARS];
    sc[S_N_PIECE] = n_piece;
    sc[S_N_REMOTE] = n_remote;
    sc[S_N_LOCAL] = n_piece - n_remote;
    sc[S_N_REPLICATED] = n_replicated;
    sc[S_BAD] = (bad_ids ? 1 : 0) | (capacity_bad ? 2 : 0);
    sc[5] = sc[6] = sc[7] = 0;
    if (capacity_bad) {
      wsflags[2] = 1;
      set_status(status, MOONEP_DEV_CAPACITY);
    }
    if (d.mode == MOONEP_MODE_TRAIN && n_remote > 0) set_status(status, MOONEP_DEV_BUDGET);
  }
}

// ----------------------------------------------------- histogram + solve ---
__global__ void __launch_bounds__(kPlanThreads)
plan_hist_solve_kernel(Dims d, const int32_t *__restrict__ idx, PlanPtrs P, int32_t *wsflags,
                       int32_t *hist, uint16_t *rank_out, int32_t *exp_kept, int32_t *exp_row0,
                       int32_t *exp_ostart, int32_t *piece_grow, int32_t *status) {
  extern __shared__ int smem[];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = (int)d.E;
  const int64_t c = blockIdx.x;

  int *wh = smem;  // [kPlanWarps][E] warp-private running counts
  for (int i = tid; i < kPlanWarps * E; i += kPlanThreads) wh[i] = 0;
  __syncthreads();

  const int64_t base = c * kChunk + (int64_t)warp * (32 * kPairsPerThread);
  int ev[kPairsPerThread];
  int rk[kPairsPerThread];
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    const int64_t p = base + j * 32 + lane;
    int e = -2;  // past the end
    if (p < d.N) {
      e = __ldcs(idx + p);
      if (e < 0 || e >= E) {
        bad = true;
        e = -1;
      }
    }
    ev[j] = e;
  }
  int *myh = wh + warp * E;
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    const int e = ev[j];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int prev = e >= 0 ? myh[e] : 0;
    const int r = __popc(peers & lanemask_lt());
    rk[j] = prev + r;
    __syncwarp();
    if (e >= 0 && r == 0) myh[e] = prev + __popc(peers);
    __syncwarp();
  }
  if (bad) {
    set_status(status, MOONEP_DEV_BAD_EXPERT_ID);
    atomicOr(wsflags + 1, 1);
  }
  __syncthreads();
  // per expert: exclusive prefix over warps, chunk total
  for (int e = tid; e < E; e += kPlanThreads) {
    int acc = 0;
    for (int w = 0; w < kPlanWarps; w++) {
      const int v = wh[w * E + e];
      wh[w * E + e] = acc;
      acc += v;
    }
    hist[c * E + e] = acc;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    const int64_t p = base + j * 32 + lane;
    if (ev[j] >= 0) rank_out[p] = (uint16_t)(myh[ev[j]] + rk[j]);
  }

  // arrival: the last CTA solves (nobody waits)
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(wsflags, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  solve(d, smem, P, wsflags, hist, exp_kept, exp_row0, exp_ostart, piece_grow, status);
}

// ---------------------------------------------------------------- placing ---
__global__ void __launch_bounds__(kPlaceThreads)
plan_place_kernel(Dims d, const int32_t *__restrict__ idx, PlanPtrs P, const int32_t *wsflags,
                  const int32_t *__restrict__ hist, const uint16_t *__restrict__ rank_in,
                  const int32_t *__restrict__ exp_kept, const int32_t *__restrict__ exp_row0,
                  const int32_t *__restrict__ exp_ostart, const int32_t *__restrict__ piece_grow) {
  const bool invalid = (wsflags[1] | wsflags[2]) != 0;
  const int E = (int)d.E;
  int32_t *slot_of = P.f[F_SLOT_OF];
  int32_t *slot_src = P.f[F_SLOT_SRC];
  const int32_t *pbeg = P.f[F_EXP_PIECE_BEGIN];
  const int32_t *pend = P.f[F_EXP_PIECE_END];
  const int32_t *post = P.f[F_PIECE_OSTART];
  const int64_t nrows = d.R * d.NvS;
  const int64_t p0 = (int64_t)blockIdx.x * kPlacePairsPerBlock + threadIdx.x;
#pragma unroll
  for (int j = 0; j < kPlacePairsPerThread; j++) {
    const int64_t p = p0 + j * kPlaceThreads;
    if (p >= d.N) break;
    if (invalid) {
      slot_of[p] = -1;
      continue;
    }
    const int e = __ldcs(idx + p);
    const int pos = hist[(p / kChunk) * E + e] + rank_in[p];
    const int kept = exp_kept[e];
    int row = -1;
    if (pos < kept) {
      row = exp_row0[e] + pos;
    } else {
      const int o = exp_ostart[e] + (pos - kept);
      int lo = pbeg[e], hi = pend[e] - 1;  // last piece with ostart <= o
      if (lo >= 0 && hi >= lo && hi < d.PMAX) {
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (post[mid] <= o) lo = mid; else hi = mid - 1;
        }
        row = piece_grow[lo] + (o - post[lo]);
      }
    }
    if (row < 0 || row >= nrows) row = -1;  // unreachable for a consistent plan
    slot_of[p] = row;
    if (row >= 0) slot_src[row] = (int32_t)p;
  }
  // rows that hold no pair: everything after a bad plan, padding when A > 1
  if (invalid || d.A > 1) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nrows; q += stride) {
      if (invalid) {
        slot_src[q] = -1;
        continue;
      }
      const int h = (int)(q / d.NvS), row = (int)(q % d.NvS);
      const int nseg = P.f[F_N_SEG][h];
      const int32_t *st = P.f[F_SEG_START] + (int64_t)h * E;
      const int32_t *ln = P.f[F_SEG_LEN] + (int64_t)h * E;
      // last segment with start <= row
      int lo = 0, hi = nseg - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (st[mid] <= row) lo = mid; else hi = mid - 1;
      }
      // among segments sharing that start (empty ones), the non-empty one is last
      const bool inside = nseg > 0 && st[lo] <= row && row < st[lo] + ln[lo];
      if (!inside) slot_src[q] = -1;
    }
  }
}

size_t solve_smem_bytes(const Dims &d) {
  const size_t hist_phase = size_t(kPlanWarps) * d.E * sizeof(int);
  const size_t solve_phase = (9 * d.E + 16 * d.R + 6 * d.PMAX + 40) * sizeof(int);
  return hist_phase > solve_phase ? hist_phase : solve_phase;
}

}  // namespace

}  // namespace moonep

using namespace moonep;

extern "C" int64_t moonep_nvs(const moonep_config_t *cfg) {
  Dims d;
  if (!make_dims(cfg, &d)) return -1;
  return d.NvS;
}

extern "C" size_t moonep_plan_bytes(const moonep_config_t *cfg) {
  Dims d;
  if (!make_dims(cfg, &d)) return 0;
  return ArenaLayout(d).total;
}

extern "C" size_t moonep_workspace_bytes(const moonep_config_t *cfg) {
  Dims d;
  if (!make_dims(cfg, &d)) return 0;
  return WsLayout(d).total;
}

extern "C" moonep_status_t moonep_plan_view(const moonep_config_t *cfg, const void *plan_arena,
                                            moonep_plan_view_t *out) {
  Dims d;
  if (!make_dims(cfg, &d) || !plan_arena || !out) return MOONEP_ERR_INVALID_ARG;
  PlanPtrs p = plan_ptrs(d, plan_arena);
  out->slot_of = p.f[F_SLOT_OF];
  out->slot_src = p.f[F_SLOT_SRC];
  out->expert_count = p.f[F_EXPERT_COUNT];
  out->rank_load = p.f[F_RANK_LOAD];
  out->overflow = p.f[F_OVERFLOW];
  out->deficit = p.f[F_DEFICIT];
  out->n_seg = p.f[F_N_SEG];
  out->seg_expert = p.f[F_SEG_EXPERT];
  out->seg_start = p.f[F_SEG_START];
  out->seg_len = p.f[F_SEG_LEN];
  out->seg_kind = p.f[F_SEG_KIND];
  out->seg_wslot = p.f[F_SEG_WSLOT];
  out->piece_expert = p.f[F_PIECE_EXPERT];
  out->piece_rank = p.f[F_PIECE_RANK];
  out->piece_start = p.f[F_PIECE_START];
  out->piece_len = p.f[F_PIECE_LEN];
  out->piece_wslot = p.f[F_PIECE_WSLOT];
  out->piece_ostart = p.f[F_PIECE_OSTART];
  out->expert_piece_begin = p.f[F_EXP_PIECE_BEGIN];
  out->expert_piece_end = p.f[F_EXP_PIECE_END];
  out->rep_expert = p.f[F_REP_EXPERT];
  out->replicated_experts = p.f[F_REPLICATED];
  out->scalars = p.f[F_SCALARS];
  out->nvs = d.NvS;
  out->max_pieces = (int32_t)d.PMAX;
  return MOONEP_OK;
}

extern "C" moonep_status_t moonep_plan(const moonep_config_t *cfg, const int32_t *topk_idx,
                                       void *plan_arena, void *workspace, int32_t *dev_status,
                                       moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d)) return MOONEP_ERR_INVALID_ARG;
  if (!plan_arena || !workspace || !dev_status || (d.N > 0 && !topk_idx))
    return MOONEP_ERR_INVALID_ARG;
  if (!aligned256(plan_arena) || !aligned256(workspace)) return MOONEP_ERR_INVALID_ARG;
  cudaStream_t st = to_cuda(stream);
  PlanPtrs P = plan_ptrs(d, plan_arena);
  WsLayout wl(d);
  char *ws = static_cast<char *>(workspace);
  int32_t *wsflags = reinterpret_cast<int32_t *>(ws + wl.off[W_COUNTER]);
  int32_t *hist = reinterpret_cast<int32_t *>(ws + wl.off[W_HIST]);
  uint16_t *rank = reinterpret_cast<uint16_t *>(ws + wl.off[W_RANK]);
  int32_t *kept = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_KEPT]);
  int32_t *row0 = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_ROW0]);
  int32_t *ostart = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_OSTART]);
  int32_t *grow = reinterpret_cast<int32_t *>(ws + wl.off[W_PIECE_GROW]);

  if (cudaMemsetAsync(wsflags, 0, 8 * sizeof(int32_t), st) != cudaSuccess) return MOONEP_ERR_CUDA;
  const size_t smem = solve_smem_bytes(d);
  if (smem > 48 * 1024) {
    if (smem > 227 * 1024) return MOONEP_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(plan_hist_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOONEP_ERR_CUDA;
  }
  plan_hist_solve_kernel<<<(unsigned)d.NC, kPlanThreads, smem, st>>>(
      d, topk_idx, P, wsflags, hist, rank, kept, row0, ostart, grow, dev_status);
  if (cudaGetLastError() != cudaSuccess) return MOONEP_ERR_CUDA;
  int64_t blocks = (d.N + kPlacePairsPerBlock - 1) / kPlacePairsPerBlock;
  if (d.A > 1 && blocks < 148) blocks = 148;
  if (blocks < 1) blocks = 1;
  plan_place_kernel<<<(unsigned)blocks, kPlaceThreads, 0, st>>>(d, topk_idx, P, wsflags, hist, rank,
                                                                 kept, row0, ostart, grow);
  if (cudaGetLastError() != cudaSuccess) return MOONEP_ERR_CUDA;
  return MOONEP_OK;
}

// ------------------------------------------------ allocation-free variant ---
// Scratch for moonep_plan_static: a fixed device array that lives as long as
// the library is loaded.  Host code cannot use the symbol itself as a device
// pointer; its device address is looked up once per device.
static __device__ __align__(256) unsigned char g_plan_scratch[MOONEP_STATIC_WORKSPACE_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::atomic<void *> g_plan_scratch_addr[kMaxDevices];
}  // namespace

extern "C" moonep_status_t moonep_plan_static(const moonep_config_t *cfg, const int32_t *topk_idx,
                                              void *plan_arena, int32_t *dev_status,
                                              moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d)) return MOONEP_ERR_INVALID_ARG;
  if (WsLayout(d).total > (size_t)MOONEP_STATIC_WORKSPACE_BYTES) return MOONEP_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOONEP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOONEP_ERR_UNSUPPORTED;
  void *scratch = g_plan_scratch_addr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    if (cudaGetSymbolAddress(&scratch, g_plan_scratch) != cudaSuccess || !scratch)
      return MOONEP_ERR_CUDA;
    g_plan_scratch_addr[dev].store(scratch, std::memory_order_release);
  }
  // the ordinary plan with the static array as its workspace (it resets the
  // arrival counter and flags itself; every other scratch word is written
  // before it is read)
  return moonep_plan(cfg, topk_idx, plan_arena, scratch, dev_status, stream);
}
