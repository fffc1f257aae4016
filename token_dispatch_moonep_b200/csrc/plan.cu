// Balanced plan for MoonEP-style expert parallelism ("Moonshot AI Open-Sources
// MoonEP": every rank receives exactly S*K token-slots, overloaded experts are
// duplicated onto underloaded ranks within a replica-slot budget;
// "MoonshotAI/MoonEP 딥다이브" §4 pattern 1: planned once per layer, reused).
//
// The rule (pairs of an expert in (rank, token, k) order; each home rank keeps the
// first S*K entries of its experts' lists in ascending expert order; the rest, over
// ranks ascending, fill the underloaded ranks in ascending order; pieces, budget and
// alignment as in include/moonep.h) is computed by one cooperative kernel:
//
// plan_kernel (chunks <= co-resident CTAs): CTA k owns chunk k of 512*ppt pairs.
//   count    warp-private per-expert counters in shared memory give every pair its
//            stable rank among the chunk's pairs of the same expert (lanes with
//            equal ids found by one ballot per bit of the id: a fixed cost however
//            many distinct ids a warp holds, no atomics).
//   publish  the chunk's counts are added by atomics into one of 16 spread copies
//            of the expert totals (a buffer per epoch parity, zeroed by the launch
//            before), the histogram is stored as a uint16 row, and one release
//            store of an arrival flag publishes both.
//   gather   once every flag shows this launch's epoch (warp 0 polls), warps 0..7
//            read the totals while warps 8..15 sum the rows before or after the
//            chunk (the nearer end) into its pairs' base offsets.  The first launch
//            on a workspace has no zeroed totals and sums every row instead.
//   solve    each CTA solves the O(E + R) problem itself with block scans; all
//            CTAs reach the same tables, so nobody waits for anybody again.
//   place    each CTA places its own pairs straight from its shared memory.
//   tables   the user-facing tables, spread over the warps of all CTAs; the last
//            CTA lists the replicated experts.
// The kernel's code is fetched anew on every launch (inside a step the data kernels
// have streamed gigabytes through L2 since the last plan), so loops that run once or
// twice per thread stay rolled and the table phase keeps to 32-bit indices.
// plan_multichunk_kernel (larger batches): CTA 0 solves, CTAs 1..W are workers
//            with several chunks each; workers keep stable ranks in the workspace,
//            the solver turns the histograms into per-chunk bases and publishes the
//            placement tables with a done flag.
// Flags carry a per-launch epoch derived from a generation word on the device,
// so graph replays and reused workspaces need no memset; every wait is bounded
// in time and reports MOONEP_DEV_TIMEOUT instead of hanging.
#include <atomic>
#include <mutex>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

// process-wide diagnostics (moonep_debug_set_wait)
std::atomic<long long> g_wait_limit_ns{200LL * 1000 * 1000};
std::atomic<int> g_phantom_arrivals{0};
std::atomic<bool> g_plan_pdl{true};

constexpr int kStBad = 1, kStCapacity = 2, kStTimeout = 8;
// Odd step between launch epochs: values left in a reused workspace (previous
// epochs, constant fills, zeros) never equal the next epoch by accident.
constexpr unsigned kEpochStep = 0x9E3779B1u;
constexpr int kSyncGen = 0, kSyncDone = 1, kSyncState = 2, kSyncTables = 3;
// tags of the two expert-total buffers: the epoch of the launch each was zeroed for
constexpr int kSyncTotTag = 4;

struct PlanArgs {
  Dims d;
  int ppt;        // pairs per thread of a chunk
  int workers;    // CTAs 1..workers
  int64_t ch;     // pairs per chunk (512 * ppt)
  int64_t nc;     // chunks
  const int32_t *idx;
  PlanPtrs P;
  int32_t *sync;     // generation, done, state, tables-done, totals tags
  int32_t *totals;   // [2][kTotalCopies][MOONEP_MAX_EXPERTS] expert totals, a buffer per epoch parity
  int32_t *arrive;   // [nc + phantom] per-chunk arrival epochs
  int32_t *badmark;  // [nc]
  int32_t *hist;     // [nc][E] chunk histograms (rewritten as bases when chunks > workers)
  uint16_t *rank;    // [N] stable ranks (only when a worker has several chunks)
  int32_t *exp_kept, *exp_row0, *exp_ostart, *piece_grow;
  int32_t *status;
  long long wait_ns;
  int phantom;
};

__device__ __forceinline__ int roundup_i(int v, int a) { return (v + a - 1) / a * a; }

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int32_t *p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_relaxed(const int32_t *p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Warp-wide bounded wait until flags[0, n) all equal v.  False on timeout.  Each
// lane issues the loads of its (up to 16) flags of a 512-flag block together, so a
// polling round costs one L2 round trip; one fence once everything has arrived.
__device__ bool warp_wait_all(const int32_t *flags, int64_t n, int v, long long limit_ns) {
  const int lane = threadIdx.x & 31;
  const unsigned long long t0 = now_ns();
  int64_t from = 0;  // flags before `from` are known to have arrived
  for (;;) {
    int got[16];
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const int64_t c = from + j * 32 + lane;
      got[j] = c < n ? ld_relaxed(flags + c) : v;
    }
    bool mine = true;
#pragma unroll
    for (int j = 0; j < 16; j++) mine &= got[j] == v;
    if (__all_sync(0xffffffffu, mine)) {
      from += 16 * 32;
      if (from >= n) {
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        return true;
      }
      continue;
    }
    if ((long long)(now_ns() - t0) > limit_ns) return false;
  }
}

// Exclusive scans of NA arrays a[k][0, n) in shared memory, in place, one pass;
// every thread of the block calls it.  scratch: 4*33 ints.  Totals in tot.
template <int NA>
__device__ void block_excl_scan(int *const (&a)[NA], int n, int *scratch, int (&tot)[NA]) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int b = tid * per < n ? tid * per : n;
  const int e = b + per < n ? b + per : n;
  int sum[NA], incl[NA];
#pragma unroll
  for (int k = 0; k < NA; k++) {
    sum[k] = 0;
    for (int i = b; i < e; i++) sum[k] += a[k][i];
    incl[k] = warp_incl_scan(sum[k]);
    if (lane == 31) scratch[k * 33 + warp] = incl[k];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < NA; k++) {
      const int v = lane < nwarps ? scratch[k * 33 + lane] : 0;
      const int wi = warp_incl_scan(v);
      if (lane < nwarps) scratch[k * 33 + lane] = wi - v;
      if (lane == 31) scratch[k * 33 + 32] = wi;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < NA; k++) {
    int run = scratch[k * 33 + warp] + incl[k] - sum[k];
    for (int i = b; i < e; i++) {
      const int v = a[k][i];
      a[k][i] = run;
      run += v;
    }
    tot[k] = scratch[k * 33 + 32];
  }
  __syncthreads();
}

// first i in [0, n) with a[i] > v (n if none); a non-decreasing
__device__ __forceinline__ int upper_bound_i(const int *a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > v) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// out[e] = sum of hist rows [0, nrows) at column e (E columns).  Rows are read
// as 16-byte vectors when E % 4 == 0, many rows in flight per thread.
// red: 4*blockDim.x ints of shared scratch.  Ends with __syncthreads().
__device__ void column_sums(const int32_t *hist, int E, int64_t nrows, int *out, int *red) {
  const int tid = threadIdx.x, nt = blockDim.x;
  if ((E & 3) == 0 && E / 4 <= nt) {
    const int E4 = E / 4, groups = nt / E4;
    const int g = tid / E4, col = tid % E4;
    int4 acc = make_int4(0, 0, 0, 0);
    if (g < groups) {
      const int4 *h4 = reinterpret_cast<const int4 *>(hist);
      for (int64_t r0 = g; r0 < nrows; r0 += (int64_t)groups * 8) {
        int4 v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
          const int64_t r = r0 + (int64_t)u * groups;
          v[u] = r < nrows ? __ldcg(h4 + r * E4 + col) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
          acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
        }
      }
      reinterpret_cast<int4 *>(red)[g * E4 + col] = acc;
    }
    __syncthreads();
    for (int e = tid; e < E; e += nt) {
      int s = 0;
      for (int q = 0; q < groups; q++) s += red[q * E + e];
      out[e] = s;
    }
  } else {
    for (int e = tid; e < E; e += nt) {
      int s = 0;
      for (int64_t r = 0; r < nrows; r++) s += __ldcg(hist + r * E + e);
      out[e] = s;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------- worker counting ---
// Histogram of chunk k and the stable rank of each of its pairs among the
// chunk's pairs of the same expert.  Pair of (warp w, step j, lane l) is
// k*ch + w*32*ppt + j*32 + l.  ev[j]: expert id, -1 bad id, -2 past the end.
// kU16: the histogram row is written as uint16 (a chunk holds at most 8192 pairs).
// pre(): run by every thread once the loads are issued, before the first barrier.
// tot(): after that barrier, where to add the chunk's count of each expert by
// atomics (null: nowhere).
// The caller puts a block barrier after the call before wh is written again.
template <bool kU16, class Pre, class Tot>
__device__ __forceinline__ bool count_chunk(const PlanArgs &a, int64_t k, int *wh,
                                            int (&ev)[kPairsPerThread], int (&rk)[kPairsPerThread],
                                            Pre pre, Tot tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = (int)a.d.E, ppt = a.ppt;
  for (int i = tid; i < kPlanWarps * E; i += kPlanThreads) wh[i] = 0;
  const int64_t base = k * a.ch + (int64_t)warp * 32 * ppt;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    const int64_t p = base + j * 32 + lane;
    int e = -2;
    if (j < ppt && p < a.d.N) {
      e = __ldcs(a.idx + p);
      if (e < 0 || e >= E) {
        bad = true;
        e = -1;
      }
    }
    ev[j] = e;
  }
  pre();
  __syncthreads();
  int32_t *const tot_dst = tot();
  int *myh = wh + warp * E;
  const uint32_t lt = lanemask_lt();
  // lanes holding the same id: one ballot per bit of the key id + 2 (id -1: a bad id,
  // -2: past the end), a fixed cost however many distinct ids the warp holds
  const int nbits = 32 - __clz(E + 1);
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    if (j >= ppt) break;  // uniform across the block
    const int e = ev[j];
    const unsigned key = (unsigned)(e + 2);
    uint32_t peers = 0xffffffffu;
    for (int b = 0; b < nbits; b++) {
      const uint32_t ones = __ballot_sync(0xffffffffu, (key >> b) & 1u);
      peers &= ((key >> b) & 1u) ? ones : ~ones;
    }
    const int prev = e >= 0 ? myh[e] : 0;
    const int r = __popc(peers & lt);
    rk[j] = prev + r;
    __syncwarp();
    if (e >= 0 && r == 0) myh[e] = prev + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPlanThreads) {
    int acc = 0;
#pragma unroll
    for (int w = 0; w < kPlanWarps; w++) {
      const int v = wh[w * E + e];
      wh[w * E + e] = acc;
      acc += v;
    }
    if (kU16)
      reinterpret_cast<uint16_t *>(a.hist)[k * E + e] = (uint16_t)acc;
    else
      a.hist[k * E + e] = acc;
    if (tot_dst && acc) atomicAdd(tot_dst + e, acc);
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++)
    if (ev[j] >= 0) rk[j] += myh[ev[j]];
  return bad;
}

// ------------------------------------------------------------ the solve ---
struct SolveSmem {
  int *cnt, *cst, *kept, *ovf, *oend, *npc, *nst, *i0, *flag, *npcn;  // [E]
  int *load, *over, *def, *ridx, *ntot, *nseg, *rrank, *rbase, *rend, *rfirst, *tmp;  // [R]
  int *pexp, *precv, *post, *plen, *pst;  // [PMAX]
  int *scratch, *misc, *red;  // 4*33, 8, 4*kPlanThreads
};

__device__ __forceinline__ SolveSmem carve(const Dims &d, int *s) {
  const int E = (int)d.E, R = (int)d.R, PM = (int)d.PMAX;
  SolveSmem m;
  int **ea[10] = {&m.cnt, &m.cst, &m.kept, &m.ovf, &m.oend, &m.npc, &m.nst, &m.i0, &m.flag, &m.npcn};
  for (int i = 0; i < 10; i++) { *ea[i] = s; s += E; }
  int **ra[11] = {&m.load, &m.over, &m.def, &m.ridx, &m.ntot, &m.nseg, &m.rrank, &m.rbase, &m.rend,
                  &m.rfirst, &m.tmp};
  for (int i = 0; i < 11; i++) { *ra[i] = s; s += R; }
  int **pa[5] = {&m.pexp, &m.precv, &m.post, &m.plen, &m.pst};
  for (int i = 0; i < 5; i++) { *pa[i] = s; s += PM; }
  m.scratch = s; s += 4 * 33;
  m.misc = s; s += 8;
  s = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(s) + 15) & ~uintptr_t(15));
  m.red = s;
  return m;
}

__host__ __device__ inline size_t solve_smem_ints(const Dims &d) {
  return 10 * d.E + 11 * d.R + 5 * d.PMAX + 4 * 33 + 8 + 4 + 4 * kPlanThreads;
}

// Solver side of the arrivals when every worker has one chunk: warp w waits
// for chunks w, w + 16, ... (and the phantom arrivals of the timeout test) and
// adds each chunk's histogram into its own partial row part[w][E] as soon as
// the chunk's flag shows this launch's epoch, so most of the summing overlaps
// the wait.  Then cnt[e] = sum of the 16 partials.  part may alias cnt (each
// column is reduced by one thread).  Returns kStTimeout / kStBad bits.
__device__ int gather_counts(const PlanArgs &a, int epoch, int *part, int *cnt, int *flags) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = (int)a.d.E;
  const int64_t ntot = a.nc + a.phantom;
  if (tid == 0) flags[0] = 0;
  for (int e = lane; e < E; e += 32) part[warp * E + e] = 0;
  __syncthreads();
  int st = 0;
  const unsigned long long t0 = now_ns();
  // a bad id does not stop the gathering: the generation word may only advance
  // once every CTA has arrived (and so has read it)
  for (int64_t c0 = warp; c0 < ntot && !(st & kStTimeout); c0 += (int64_t)kPlanWarps * 32) {
    const int64_t c = c0 + (int64_t)kPlanWarps * lane;  // this lane's chunk in the batch
    bool pend = c < ntot;
    unsigned pending = __ballot_sync(0xffffffffu, pend);
    while (pending) {
      const bool arrived = pend && ld_relaxed(a.arrive + c) == epoch;
      unsigned got = __ballot_sync(0xffffffffu, arrived);
      if (!got) {
        if ((long long)(now_ns() - t0) > a.wait_ns) {
          st = kStTimeout;
          break;
        }
        __nanosleep(32);
        continue;
      }
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      pending &= ~got;
      if (arrived) pend = false;
      bool bad = arrived && c < a.nc && __ldcg(a.badmark + c) == epoch;
      if (__any_sync(0xffffffffu, bad)) st |= kStBad;
      while (got) {  // add up to four arrived chunks per pass, their loads in flight together
        int64_t cj[4];
        int n = 0;
        while (got && n < 4) {
          const int j = __ffs(got) - 1;
          got &= got - 1;
          const int64_t cc = c0 + (int64_t)kPlanWarps * j;
          if (cc < a.nc) cj[n++] = cc;
        }
        for (int qb = 0; qb < E; qb += 32 * 8) {
          int v[4][8];
#pragma unroll
          for (int i = 0; i < 4; i++)
#pragma unroll
            for (int q = 0; q < 8; q++) {
              const int col = qb + q * 32 + lane;
              v[i][q] = (i < n && col < E) ? __ldcg(a.hist + cj[i] * E + col) : 0;
            }
#pragma unroll
          for (int q = 0; q < 8; q++) {
            const int col = qb + q * 32 + lane;
            if (col < E) part[warp * E + col] += v[0][q] + v[1][q] + v[2][q] + v[3][q];
          }
        }
      }
    }
  }
  if (lane == 0 && st) atomicOr(flags, st);
  __syncthreads();
  st = flags[0];
  for (int e = tid; e < E; e += kPlanThreads) {
    int sum = 0;
#pragma unroll
    for (int w = 0; w < kPlanWarps; w++) sum += part[w * E + e];
    cnt[e] = sum;
  }
  __syncthreads();
  return st;
}

// Per-expert exclusive scan of the histograms over chunks, in place (the
// bases of chunks when workers hold several chunks); counts into cnt.
__device__ void chunk_bases(const PlanArgs &a, int *cnt) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int E = (int)a.d.E;
  const int64_t NC = a.nc;
  for (int e = tid; e < E; e += nt) {
    int run = 0;
    for (int64_t c = 0; c < NC; c += 16) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; u++) v[u] = c + u < NC ? __ldcg(a.hist + (c + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 16; u++) {
        if (c + u < NC) a.hist[(c + u) * E + e] = run;
        run += v[u];
      }
    }
    cnt[e] = run;
  }
  __syncthreads();
}

// The part of the solve placement depends on.  Returns state bits (thread 0).
__device__ int solve_core(const PlanArgs &a, const SolveSmem &m) {
  const Dims &d = a.d;
  const PlanPtrs &P = a.P;
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int E = (int)d.E, R = (int)d.R, L = (int)d.L, A = (int)d.A;
  const int SK = (int)d.SK, NvS = (int)d.NvS, PM = (int)d.PMAX;

  // rank loads from the global prefix of counts
  for (int e = tid; e < E; e += nt) m.cst[e] = m.cnt[e];
  if (tid == 0) { m.misc[1] = 0; m.misc[2] = 0; }
  {
    int *arr[1] = {m.cst};
    int tot[1];
    __syncthreads();
    block_excl_scan<1>(arr, E, m.scratch, tot);
    for (int h = tid; h < R; h += nt) {
      const int lo = m.cst[h * L];
      m.load[h] = ((h + 1) * L < E ? m.cst[(h + 1) * L] : tot[0]) - lo;
    }
  }
  __syncthreads();
  // overflow / deficit bases, receiver compaction: one warp, ceil(R/32)
  // consecutive ranks per lane, three warp scans
  if (warp == 0) {
    const int per = (R + 31) / 32;
    const int h0 = lane * per < R ? lane * per : R;
    const int h1 = h0 + per < R ? h0 + per : R;
    int sov = 0, sdf = 0, srf = 0;
    for (int h = h0; h < h1; h++) {
      const int ld = m.load[h];
      sov += ld > SK ? ld - SK : 0;
      sdf += ld < SK ? SK - ld : 0;
      srf += ld < SK ? 1 : 0;
    }
    const int iov = warp_incl_scan(sov), idf = warp_incl_scan(sdf), irf = warp_incl_scan(srf);
    int ov = iov - sov, df = idf - sdf, rf = irf - srf;  // exclusive bases of this lane's ranks
    for (int h = h0; h < h1; h++) {
      const int ld = m.load[h];
      const int o = ld > SK ? ld - SK : 0, dd = ld < SK ? SK - ld : 0;
      m.over[h] = ov;
      m.def[h] = df;
      if (dd > 0) {
        m.ridx[h] = rf;
        m.rrank[rf] = h;
        m.rbase[rf] = df;
        m.rend[rf] = df + dd;
        rf++;
      } else {
        m.ridx[h] = -1;
      }
      ov += o;
      df += dd;
    }
    if (lane == 31) m.misc[0] = irf;
  }
  __syncthreads();
  const int n_recv = m.misc[0];

  // per expert: kept rows, overflow range, pieces
  for (int e = tid; e < E; e += nt) {
    const int h = e / L;
    const int cnt = m.cnt[e];
    const int cst = m.cst[e] - m.cst[h * L];
    int kept = SK - cst;
    kept = kept < 0 ? 0 : (kept > cnt ? cnt : kept);
    const int ovf = cnt - kept;
    const int ost = m.over[h] + (cst > SK ? cst - SK : 0);
    m.kept[e] = kept;
    m.ovf[e] = ovf;
    m.oend[e] = ost + ovf;
    int npc = 0, i0 = 0;
    if (ovf > 0 && n_recv > 0) {
      i0 = upper_bound_i(m.rend, n_recv, ost);
      int i1 = upper_bound_i(m.rend, n_recv, ost + ovf - 1);
      if (i1 >= n_recv) i1 = n_recv - 1;
      if (i0 < n_recv) npc = i1 - i0 + 1;
    }
    m.npc[e] = npc;
    m.npcn[e] = npc;
    m.i0[e] = i0;
    m.nst[e] = A > 1 ? roundup_i(kept, A) : (cst < SK ? cst : SK);  // A = 1: kept rows are a prefix
  }
  int n_piece;
  __syncthreads();
  if (A > 1) {
    int *arr[2] = {m.npc, m.nst};
    int tot[2];
    block_excl_scan<2>(arr, E, m.scratch, tot);
    n_piece = tot[0];
    for (int h = tid; h < R; h += nt) {
      const int lo = m.nst[h * L];
      m.ntot[h] = ((h + 1) * L < E ? m.nst[(h + 1) * L] : tot[1]) - lo;
      m.tmp[h] = lo;
    }
    __syncthreads();
    for (int e = tid; e < E; e += nt) m.nst[e] -= m.tmp[e / L];
  } else {
    int *arr[1] = {m.npc};
    int tot[1];
    block_excl_scan<1>(arr, E, m.scratch, tot);
    n_piece = tot[0];
    for (int h = tid; h < R; h += nt) m.ntot[h] = m.load[h] < SK ? m.load[h] : SK;
  }
  if (n_piece > PM) n_piece = PM;  // cannot happen: pieces <= experts + receivers - 1
  if (tid == 0) m.misc[3] = n_piece;
  __syncthreads();

  // placement tables: per expert, then per piece, one thread each.  The expert
  // of piece pid is the last e with first-piece id npc[e] <= pid (npc is the
  // exclusive scan of the piece counts, so that expert has a piece).
  for (int e = tid; e < E; e += nt) {
    const int h = e / L;
    a.exp_kept[e] = m.kept[e];
    a.exp_row0[e] = h * NvS + m.nst[e];
    a.exp_ostart[e] = m.oend[e] - m.ovf[e];
    P.f[F_EXP_PIECE_BEGIN][e] = m.npc[e];
    P.f[F_EXP_PIECE_END][e] = m.npc[e] + m.npcn[e];
  }
  for (int pid = tid; pid < n_piece; pid += nt) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (m.npc[mid] <= pid) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int q = pid - m.npc[e];
    const int i = m.i0[e] + q;
    if (q < 0 || q >= m.npcn[e] || i >= n_recv) continue;
    const int ost = m.oend[e] - m.ovf[e];
    const int os = ost > m.rbase[i] ? ost : m.rbase[i];
    const int oe = m.oend[e] < m.rend[i] ? m.oend[e] : m.rend[i];
    const int dr = m.rrank[i];
    int start;
    if (A == 1) {
      start = m.ntot[dr] + (os - m.rbase[i]);
    } else {  // earlier pieces of receiver i: from the expert holding rbase up to e-1
      const int ef = upper_bound_i(m.oend, E, m.rbase[i]);
      start = m.ntot[dr];
      if (ef < e) {
        start += roundup_i(m.oend[ef] - m.rbase[i], A);
        for (int e2 = ef + 1; e2 < e; e2++) start += roundup_i(m.ovf[e2], A);
      }
    }
    m.pexp[pid] = e;
    m.precv[pid] = i;
    m.post[pid] = os;
    m.plen[pid] = oe - os;
    m.pst[pid] = start;
    P.f[F_PIECE_OSTART][pid] = os;
    a.piece_grow[pid] = dr * NvS + start;
    if (start + (oe - os) > NvS) m.misc[1] = 1;
  }
  for (int h = tid; h < R; h += nt)
    if (m.ntot[h] > NvS) m.misc[1] = 1;
  __syncthreads();
  // segments per rank (published with the placement tables: the workers fill
  // the unused segment entries and replica slots from it)
  for (int i = tid; i < n_recv; i += nt) {  // first and last piece of each receiver
    const int ef = upper_bound_i(m.oend, E, m.rbase[i]);
    m.rfirst[i] = ef < E ? m.npc[ef] + (i - m.i0[ef]) : 0;
    const int el = upper_bound_i(m.oend, E, m.rend[i] - 1);
    const int last = el < E ? m.npc[el] + (i - m.i0[el]) : -1;
    m.nseg[m.rrank[i]] = L + (last - m.rfirst[i] + 1);
  }
  for (int h = tid; h < R; h += nt)
    if (m.ridx[h] < 0) m.nseg[h] = L;
  __syncthreads();
  for (int h = tid; h < R; h += nt) P.f[F_N_SEG][h] = m.nseg[h];
  return m.misc[1] ? kStCapacity : 0;
}

// Every other plan table (after the done flag; placement does not read them).
__device__ void solve_outputs(const PlanArgs &a, const SolveSmem &m) {
  const Dims &d = a.d;
  const PlanPtrs &P = a.P;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int E = (int)d.E, R = (int)d.R, L = (int)d.L, B = (int)d.B, SK = (int)d.SK;
  const int n_piece = m.misc[3];

  for (int e = tid; e < E; e += nt) m.flag[e] = 0;
  __syncthreads();
  for (int pid = tid; pid < n_piece; pid += nt) {
    const int i = m.precv[pid], e = m.pexp[pid];
    const int dr = m.rrank[i], j = pid - m.rfirst[i];
    const int ws = j < B ? j : -1;
    P.f[F_PIECE_EXPERT][pid] = e;
    P.f[F_PIECE_RANK][pid] = dr;
    P.f[F_PIECE_START][pid] = m.pst[pid];
    P.f[F_PIECE_LEN][pid] = m.plen[pid];
    P.f[F_PIECE_WSLOT][pid] = ws;
    if (j >= 0 && L + j < E) {
      const int sj = dr * E + L + j;
      P.f[F_SEG_EXPERT][sj] = e;
      P.f[F_SEG_START][sj] = m.pst[pid];
      P.f[F_SEG_LEN][sj] = m.plen[pid];
      P.f[F_SEG_KIND][sj] = ws >= 0 ? MOONEP_SEG_REPLICA : MOONEP_SEG_REMOTE;
      P.f[F_SEG_WSLOT][sj] = ws;
    }
    if (ws >= 0) {
      P.f[F_REP_EXPERT][(int64_t)dr * B + j] = e;
      m.flag[e] = 1;
    } else {
      atomicAdd(&m.misc[2], 1);
    }
  }
  for (int e = tid; e < E; e += nt) {
    const int h = e / L, si = h * E + (e - h * L);
    P.f[F_EXPERT_COUNT][e] = m.cnt[e];
    P.f[F_SEG_EXPERT][si] = e;
    P.f[F_SEG_START][si] = m.nst[e];
    P.f[F_SEG_LEN][si] = m.kept[e];
    P.f[F_SEG_KIND][si] = MOONEP_SEG_NATIVE;
    P.f[F_SEG_WSLOT][si] = -1;
  }
  for (int h = tid; h < R; h += nt) {
    const int ld = m.load[h];
    P.f[F_RANK_LOAD][h] = ld;
    P.f[F_OVERFLOW][h] = ld > SK ? ld - SK : 0;
    P.f[F_DEFICIT][h] = ld < SK ? SK - ld : 0;
  }
  __syncthreads();
  for (int e = tid; e < E; e += nt) m.i0[e] = m.flag[e];  // keep the flags across the scan
  {
    int *arr[1] = {m.flag};
    int tot[1];
    __syncthreads();
    block_excl_scan<1>(arr, E, m.scratch, tot);
    for (int e = tid; e < E; e += nt)
      if (m.i0[e]) P.f[F_REPLICATED][m.flag[e]] = e;
    if (tid == 0) m.misc[4] = tot[0];
  }
  __syncthreads();
  if (tid == 0) {
    const int n_remote = m.misc[2];
    int32_t *sc = P.f[F_SCALARS];
    sc[S_N_PIECE] = n_piece;
    sc[S_N_REMOTE] = n_remote;
    sc[S_N_LOCAL] = n_piece - n_remote;
    sc[S_N_REPLICATED] = m.misc[4];
    sc[S_BAD] = 0;
    sc[5] = sc[6] = sc[7] = 0;
    if (d.mode == MOONEP_MODE_TRAIN && n_remote > 0) set_status(a.status, MOONEP_DEV_BUDGET);
  }
}

// -------------------------------------------------------------- placing ---
// tables: base[E] kept[E] row0[E] ostart[E] piece_begin[E] piece_end[E]
//         piece_ostart[PMAX] piece_row[PMAX]
__device__ __forceinline__ void place_chunk(const PlanArgs &a, int64_t k, const int *t, bool from_regs,
                                            const int (&ev)[kPairsPerThread],
                                            const int (&rk)[kPairsPerThread]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Dims &d = a.d;
  const int E = (int)d.E, PM = (int)d.PMAX, ppt = a.ppt;
  const int *t_base = t, *t_kept = t + E, *t_row0 = t + 2 * E, *t_ost = t + 3 * E;
  const int *t_pb = t + 4 * E, *t_pe = t + 5 * E, *t_post = t + 6 * E, *t_prow = t + 6 * E + PM;
  int32_t *slot_of = a.P.f[F_SLOT_OF];
  int32_t *slot_src = a.P.f[F_SLOT_SRC];
  const int64_t nrows = d.R * d.NvS;
  const int64_t base = k * a.ch + (int64_t)warp * 32 * ppt;
#pragma unroll
  for (int j = 0; j < kPairsPerThread; j++) {
    if (j >= ppt) break;
    const int64_t p = base + j * 32 + lane;
    if (p >= d.N) continue;
    const int e = from_regs ? ev[j] : __ldcs(a.idx + p);
    const int r = from_regs ? rk[j] : (int)a.rank[p];
    const int pos = t_base[e] + r;
    const int kept = t_kept[e];
    int row = -1;
    if (pos < kept) {
      row = t_row0[e] + pos;
    } else {
      const int o = t_ost[e] + (pos - kept);
      int lo = t_pb[e], hi = t_pe[e] - 1;  // last piece with ostart <= o
      if (lo >= 0 && hi >= lo && hi < PM) {
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (t_post[mid] <= o) lo = mid; else hi = mid - 1;
        }
        row = t_prow[lo] + (o - t_post[lo]);
      }
    }
    if (row < 0 || row >= nrows) row = -1;  // unreachable for a consistent plan
    slot_of[p] = row;
    if (row >= 0) slot_src[row] = (int32_t)p;
  }
}

__device__ __forceinline__ bool wait_flag(const int32_t *flag, int v, long long limit_ns) {
  const unsigned long long t0 = now_ns();
  while (ld_acquire(flag) != v) {
    if ((long long)(now_ns() - t0) > limit_ns) return false;
    __nanosleep(64);
  }
  return true;
}

__global__ void __launch_bounds__(kPlanThreads) plan_multichunk_kernel(PlanArgs a) {
  // launched with programmatic stream serialisation: wait here until the
  // kernel before it in the stream (the router's top-k, the previous layer)
  // has completed and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) int smem[];
  __shared__ int s_epoch, s_state, s_ok;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Dims &d = a.d;
  const int E = (int)d.E, PM = (int)d.PMAX;
  int32_t *gen = a.sync + kSyncGen, *done = a.sync + kSyncDone;
  int32_t *state_w = a.sync + kSyncState, *tables = a.sync + kSyncTables;

  // the generation word: workers need it only when they publish, so its load
  // overlaps their counting
  int gen_v = 0;
  if (tid == 0) gen_v = *((volatile int32_t *)gen);

  // ================================================================ solver ==
  if (blockIdx.x == 0) {
    if (tid == 0) s_epoch = (int)((unsigned)gen_v + kEpochStep);
    __syncthreads();
    const int epoch = s_epoch;
    SolveSmem m = carve(d, smem);
    int st;
    if (a.nc <= a.workers) {
      st = gather_counts(a, epoch, smem, m.cnt, &s_state);
    } else {
      if (warp == 0) {
        const bool ok = warp_wait_all(a.arrive, a.nc + a.phantom, epoch, a.wait_ns);
        bool b = false;
        for (int64_t c = lane; c < a.nc; c += 32) b |= __ldcg(a.badmark + c) == epoch;
        b = __any_sync(0xffffffffu, b);
        if (lane == 0) s_state = (ok ? 0 : kStTimeout) | (b ? kStBad : 0);
      }
      __syncthreads();
      st = s_state;
      if (st == 0) chunk_bases(a, m.cnt);
    }
    if (tid == 0) *((volatile int32_t *)gen) = epoch;  // every CTA read it before arriving
    if (st == 0) st = solve_core(a, m);
    if (tid == 0) {
      if (st & kStTimeout) set_status(a.status, MOONEP_DEV_TIMEOUT);
      if (st & kStCapacity) set_status(a.status, MOONEP_DEV_CAPACITY);
      if (st) {
        int32_t *sc = a.P.f[F_SCALARS];
        for (int i = 0; i < 8; i++) sc[i] = 0;
        sc[S_BAD] = st;
      }
      *state_w = st;
      __threadfence();
      st_release(done, epoch);
    }
    if (st == 0) solve_outputs(a, m);
    if (d.A > 1) {  // only the padding fill (A > 1) waits for the finished tables
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        st_release(tables, epoch);
      }
    }
    return;
  }

  // =============================================================== workers ==
  const int wk = blockIdx.x - 1, W = a.workers;
  const bool single = a.nc <= W;  // at most one chunk per worker: ids and ranks stay in registers
  int ev[kPairsPerThread], rk[kPairsPerThread];
  int epoch = 0;
  bool have_epoch = false;
  for (int64_t k = wk; k < a.nc; k += W) {
    const bool bad = __syncthreads_or(count_chunk<false>(
        a, k, smem, ev, rk, [] {}, []() -> int32_t * { return nullptr; }));
    if (!have_epoch) {
      if (tid == 0) s_epoch = (int)((unsigned)gen_v + kEpochStep);
      __syncthreads();
      epoch = s_epoch;
      have_epoch = true;
    }
    if (!single) {
      const int64_t base = k * a.ch + (int64_t)warp * 32 * a.ppt;
#pragma unroll
      for (int j = 0; j < kPairsPerThread; j++)
        if (j < a.ppt && ev[j] >= 0) a.rank[base + j * 32 + lane] = (uint16_t)rk[j];
      __syncthreads();
    }
    if (tid == 0) {
      if (bad) set_status(a.status, MOONEP_DEV_BAD_EXPERT_ID);
      a.badmark[k] = bad ? epoch : ~epoch;
      __threadfence();
      st_release(a.arrive + k, epoch);
    }
  }
  if (!have_epoch) {  // a worker without a chunk
    if (tid == 0) s_epoch = (int)((unsigned)gen_v + kEpochStep);
    __syncthreads();
    epoch = s_epoch;
  }
  int *tb = smem;  // placement tables, see place_chunk
  // base offsets of my chunk: sums of the histograms of the chunks before it
  // (overlaps the solve; with several chunks per worker the solver writes them)
  bool ok = true;
  if (single && wk < a.nc) {
    if (warp == 0) {
      const bool w = warp_wait_all(a.arrive, wk, epoch, a.wait_ns);
      if (lane == 0) s_ok = w;
    }
    __syncthreads();
    ok = s_ok;
    int *red = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(tb + 6 * E + 2 * PM) + 15) &
                                       ~uintptr_t(15));
    if (ok) column_sums(a.hist, E, wk, tb, red);
  }
  if (tid == 0) {
    const bool w = wait_flag(done, epoch, a.wait_ns);
    s_state = w ? __ldcg(state_w) : kStTimeout;
    if (!w || !ok) set_status(a.status, MOONEP_DEV_TIMEOUT);
  }
  __syncthreads();
  const bool invalid = s_state != 0 || !ok;

  if (!invalid) {
    for (int e = tid; e < E; e += kPlanThreads) {
      tb[E + e] = __ldcg(a.exp_kept + e);
      tb[2 * E + e] = __ldcg(a.exp_row0 + e);
      tb[3 * E + e] = __ldcg(a.exp_ostart + e);
      tb[4 * E + e] = __ldcg(a.P.f[F_EXP_PIECE_BEGIN] + e);
      tb[5 * E + e] = __ldcg(a.P.f[F_EXP_PIECE_END] + e);
    }
    for (int i = tid; i < PM; i += kPlanThreads) {
      tb[6 * E + i] = __ldcg(a.P.f[F_PIECE_OSTART] + i);
      tb[6 * E + PM + i] = __ldcg(a.piece_grow + i);
    }
    __syncthreads();
    for (int64_t k = wk; k < a.nc; k += W) {
      if (!single) {
        for (int e = tid; e < E; e += kPlanThreads) tb[e] = __ldcg(a.hist + k * E + e);
        __syncthreads();
      }
      place_chunk(a, k, tb, single, ev, rk);
      if (!single) __syncthreads();
    }
  } else {
    int32_t *slot_of = a.P.f[F_SLOT_OF];
    for (int64_t k = wk; k < a.nc; k += W)
      for (int64_t p = k * a.ch + tid; p < (k + 1) * a.ch && p < d.N; p += kPlanThreads) slot_of[p] = -1;
  }

  // unused segment entries and free replica slots (from the published n_seg)
  if (!invalid) {
    const int L = (int)d.L, B = (int)d.B;
    for (int h = wk; h < (int)d.R; h += W) {
      const int ns = __ldcg(a.P.f[F_N_SEG] + h);
      for (int i = ns + tid; i < E; i += kPlanThreads) {
        const int64_t q = (int64_t)h * E + i;
        a.P.f[F_SEG_EXPERT][q] = -1;
        a.P.f[F_SEG_START][q] = 0;
        a.P.f[F_SEG_LEN][q] = 0;
        a.P.f[F_SEG_KIND][q] = -1;
        a.P.f[F_SEG_WSLOT][q] = -1;
      }
      for (int j = (ns - L) + tid; j < B; j += kPlanThreads)
        if (j >= 0) a.P.f[F_REP_EXPERT][(int64_t)h * B + j] = -1;
    }
  }

  // rows that hold no pair: everything after an invalid plan, padding when A > 1
  if (invalid || d.A > 1) {
    if (!invalid) {
      if (tid == 0) s_ok = wait_flag(tables, epoch, a.wait_ns);
      __syncthreads();
      if (!s_ok) {
        if (tid == 0) set_status(a.status, MOONEP_DEV_TIMEOUT);
        return;
      }
    }
    const int64_t nrows = d.R * d.NvS;
    const int64_t stride = (int64_t)W * blockDim.x;
    int32_t *slot_src = a.P.f[F_SLOT_SRC];
    for (int64_t q = (int64_t)wk * blockDim.x + tid; q < nrows; q += stride) {
      if (invalid) {
        slot_src[q] = -1;
        continue;
      }
      const int h = (int)(q / d.NvS), row = (int)(q % d.NvS);
      const int nseg = __ldcg(a.P.f[F_N_SEG] + h);
      const int32_t *st = a.P.f[F_SEG_START] + (int64_t)h * E;
      const int32_t *ln = a.P.f[F_SEG_LEN] + (int64_t)h * E;
      int lo = 0, hi = nseg - 1;  // last segment with start <= row
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldcg(st + mid) <= row) lo = mid; else hi = mid - 1;
      }
      const bool inside = nseg > 0 && __ldcg(st + lo) <= row && row < __ldcg(st + lo) + __ldcg(ln + lo);
      if (!inside) slot_src[q] = -1;
    }
  }
}

// ============================================ one chunk per CTA, every CTA solves ===
// plan_kernel (phases at the top of this file): its shared-memory state.  One
// grid-wide exchange (the arrivals) per plan; every CTA then holds the whole solve.
struct FastSmem {
  int *cnt, *base, *gcst, *kept, *ovf, *oend, *nst, *row0, *npc, *i0, *pid0, *eflag, *epos;  // [E]
  int *load, *over, *def, *ridx, *ntot, *nseg, *rrank, *rbase, *rend, *rfirst, *rlast;  // [R]
  int *pexp, *precv, *post, *plen, *pst, *prow, *pscan;  // [PMAX]
  int *misc;     // [16]: 0 receivers, 1 pieces, 2 capacity, 3 gather state, 4 remote pieces
  int *scratch;  // 20 * kPlanWarps: the areas of the block scans
  int *tmp;      // per-warp histograms [16][E] while counting, then gather partials
};

enum FastMisc { M_NRECV = 0, M_NPIECE = 1, M_CAP = 2, M_STATE = 3, M_NREMOTE = 4 };

__host__ __device__ inline size_t fast_tmp_ints(const Dims &d) {
  const size_t hist = size_t(kPlanWarps) * d.E;
  const size_t gather = 2 * size_t(8 * kPlanThreads > d.E ? 8 * kPlanThreads : d.E);
  return hist > gather ? hist : gather;
}

__host__ __device__ inline size_t fast_smem_ints(const Dims &d) {
  return 13 * d.E + 11 * d.R + 7 * d.PMAX + 16 + 20 * kPlanWarps + 4 + fast_tmp_ints(d);
}

__device__ __forceinline__ FastSmem carve_fast(const Dims &d, int *s) {
  const int E = (int)d.E, R = (int)d.R, PM = (int)d.PMAX;
  FastSmem m;
  int **ea[13] = {&m.cnt, &m.base, &m.gcst, &m.kept, &m.ovf, &m.oend, &m.nst, &m.row0, &m.npc,
                  &m.i0, &m.pid0, &m.eflag, &m.epos};
  for (int i = 0; i < 13; i++) { *ea[i] = s; s += E; }
  int **ra[11] = {&m.load, &m.over, &m.def, &m.ridx, &m.ntot, &m.nseg, &m.rrank, &m.rbase,
                  &m.rend, &m.rfirst, &m.rlast};
  for (int i = 0; i < 11; i++) { *ra[i] = s; s += R; }
  int **pa[7] = {&m.pexp, &m.precv, &m.post, &m.plen, &m.pst, &m.prow, &m.pscan};
  for (int i = 0; i < 7; i++) { *pa[i] = s; s += PM; }
  m.misc = s; s += 16;
  m.scratch = s; s += 20 * kPlanWarps;
  s = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(s) + 15) & ~uintptr_t(15));
  m.tmp = s;
  return m;
}

// Sums of every chunk's histogram (uint16 rows): m.cnt[e] over all chunks and m.base[e]
// over the chunks before chunk k.  Warp 0 alone polls the arrival flags (every CTA polling
// with every thread would pile thousands of loads per round onto the same few L2 lines);
// once all chunks (and the test-only phantom arrivals) show this launch's epoch, all
// threads load the rows together.  A row is U = E / V units of V counts (V = 8: one
// 16-byte load); thread group g (G groups of U threads, or one group when U >
// kPlanThreads) takes chunks g, g + G, ...  Returns the state bits (kStTimeout, kStBad).
template <int V>
__device__ int gather_all(const PlanArgs &a, int64_t k, int epoch, const FastSmem &m) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int E = (int)a.d.E;
  const uint16_t *hist = reinterpret_cast<const uint16_t *>(a.hist);
  if (tid < 32) {
    const bool ok = warp_wait_all(a.arrive, a.nc + a.phantom, epoch, a.wait_ns);
    if (lane == 0) m.misc[M_STATE] = ok ? 0 : kStTimeout;
  }
  __syncthreads();
  if (m.misc[M_STATE]) return kStTimeout;
  const int U = E / V;
  const int gw = U < kPlanThreads ? U : kPlanThreads;  // threads per group
  const int G = kPlanThreads / gw;
  const int g = tid / gw, u0 = tid % gw;
  const int NU = (U + gw - 1) / gw;                    // units per thread (1, or 2 when V == 1)
  constexpr int QN = V == 8 ? 1 : 2;                   // E <= 1024: U <= 128 units of 8 counts
  int tot[QN][V], pre[QN][V];
#pragma unroll
  for (int q = 0; q < QN; q++)
#pragma unroll
    for (int v = 0; v < V; v++) tot[q][v] = pre[q][v] = 0;
  bool bad = false;
  if (g < G) {
    for (int64_t r0 = g; r0 < a.nc; r0 += 8LL * G) {
      uint32_t vals[8][QN][V == 8 ? 4 : 1];
#pragma unroll
      for (int j = 0; j < 8; j++) {  // the batch's loads first, then the sums
        const int64_t r = r0 + (int64_t)j * G;
#pragma unroll
        for (int q = 0; q < QN; q++) {
          const int u = u0 + q * gw;
          const bool in = r < a.nc && q < NU && u < U;
          if constexpr (V == 8) {
            const uint4 t = in ? __ldcg(reinterpret_cast<const uint4 *>(hist + r * E) + u)
                               : make_uint4(0, 0, 0, 0);
            vals[j][q][0] = t.x;
            vals[j][q][1] = t.y;
            vals[j][q][2] = t.z;
            vals[j][q][3] = t.w;
          } else {
            vals[j][q][0] = in ? __ldcg(hist + r * E + u) : 0u;
          }
        }
        if (u0 == 0 && r < a.nc) bad |= __ldcg(a.badmark + r) == epoch;
      }
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const int64_t r = r0 + (int64_t)j * G;
#pragma unroll
        for (int q = 0; q < QN; q++)
#pragma unroll
          for (int v = 0; v < V; v++) {
            const int c = V == 8 ? (int)((vals[j][q][v >> 1] >> ((v & 1) * 16)) & 0xffffu)
                                 : (int)vals[j][q][0];
            tot[q][v] += c;
            if (r < k) pre[q][v] += c;
          }
      }
    }
  }
  if (bad) atomicOr(&m.misc[M_STATE], kStBad);
  // partial sums of the groups, then one thread per expert adds them up
  int *ptot = m.tmp, *ppre = m.tmp + G * E;
  if (g < G) {
#pragma unroll
    for (int q = 0; q < QN; q++) {
      const int u = u0 + q * gw;
      if (q >= NU || u >= U) break;
#pragma unroll
      for (int v = 0; v < V; v++) {
        ptot[g * E + u * V + v] = tot[q][v];
        ppre[g * E + u * V + v] = pre[q][v];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPlanThreads) {
    int t = 0, p = 0;
    for (int q = 0; q < G; q++) {
      t += ptot[q * E + e];
      p += ppre[q * E + e];
    }
    m.cnt[e] = t;
    m.base[e] = p;
  }
  __syncthreads();
  return m.misc[M_STATE];
}

// Barrier of the first NT threads of the block: __syncthreads for the whole block,
// else named barrier BAR (the other threads of the block do other work meanwhile).
template <int NT, int BAR>
__device__ __forceinline__ void group_sync() {
  if (NT == kPlanThreads) __syncthreads();
  else asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Expert e's total: the sum of its kTotalCopies partial copies (loads in flight together).
__device__ __forceinline__ int total_of(const int32_t *totals, int e) {
  int v[kTotalCopies];
#pragma unroll
  for (int c = 0; c < kTotalCopies; c++) v[c] = __ldcg(totals + c * MOONEP_MAX_EXPERTS + e);
  int s = 0;
#pragma unroll
  for (int c = 0; c < kTotalCopies; c++) s += v[c];
  return s;
}

// Warps 8..15 of the split gather: m.base[e] = pairs of expert e in the chunks before
// chunk k, read from the nearer end: the rows before k when k < nc / 2, else the
// totals less the rows from k on (no CTA reads more than half the rows).  A row is
// U = E / V units of V counts; G groups of the 256 threads take rows r, r + G, ...
template <int V>
__device__ void chunk_bases_split(const PlanArgs &a, int64_t k, const int32_t *totals,
                                  const FastSmem &m) {
  constexpr int NT = kPlanThreads / 2;
  const int tb = threadIdx.x - NT;
  const int E = (int)a.d.E;
  const uint16_t *hist = reinterpret_cast<const uint16_t *>(a.hist);
  const bool suffix = 2 * k >= a.nc;
  const int64_t r_lo = suffix ? k : 0, r_hi = suffix ? a.nc : k;
  const int U = E / V;
  const int gw = U < NT ? U : NT;
  const int G = NT / gw;
  const int g = tb / gw, u0 = tb % gw;
  const int NU = (U + gw - 1) / gw;
  constexpr int QN = V == 8 ? 1 : 4;  // E <= 1024: U <= 128 units of 8, or <= 1024 of 1
  int acc[QN][V];
#pragma unroll
  for (int q = 0; q < QN; q++)
#pragma unroll
    for (int v = 0; v < V; v++) acc[q][v] = 0;
  if (g < G) {
    for (int64_t r0 = r_lo + g; r0 < r_hi; r0 += 8LL * G) {
      uint32_t vals[8][QN][V == 8 ? 4 : 1];
#pragma unroll
      for (int j = 0; j < 8; j++) {  // the batch's loads first, then the sums
        const int64_t r = r0 + (int64_t)j * G;
#pragma unroll
        for (int q = 0; q < QN; q++) {
          const int u = u0 + q * gw;
          const bool in = r < r_hi && q < NU && u < U;
          if constexpr (V == 8) {
            const uint4 t = in ? __ldcg(reinterpret_cast<const uint4 *>(hist + r * E) + u)
                               : make_uint4(0, 0, 0, 0);
            vals[j][q][0] = t.x;
            vals[j][q][1] = t.y;
            vals[j][q][2] = t.z;
            vals[j][q][3] = t.w;
          } else {
            vals[j][q][0] = in ? __ldcg(hist + r * E + u) : 0u;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; j++)
#pragma unroll
        for (int q = 0; q < QN; q++)
#pragma unroll
          for (int v = 0; v < V; v++)
            acc[q][v] += V == 8 ? (int)((vals[j][q][v >> 1] >> ((v & 1) * 16)) & 0xffffu)
                                : (int)vals[j][q][0];
    }
#pragma unroll
    for (int q = 0; q < QN; q++) {
      const int u = u0 + q * gw;
      if (q >= NU || u >= U) break;
#pragma unroll
      for (int v = 0; v < V; v++) m.tmp[g * E + u * V + v] = acc[q][v];
    }
  }
  group_sync<NT, 2>();
  for (int e = tb; e < E; e += NT) {
    int sum = 0;
    for (int q = 0; q < G; q++) sum += m.tmp[q * E + e];
    m.base[e] = suffix ? total_of(totals, e) - sum : sum;
  }
}

// first i in [0, n) with a[i] > v (n if none); a non-decreasing.  The steps depend only
// on n (no data-dependent branches): the same trip count for every thread.
__device__ __forceinline__ int upper_bound_bf(const int *a, int n, int v) {
  if (n <= 0) return 0;
  const int *base = a;
  int len = n;
  while (len > 1) {
    const int half = len >> 1;
    base = base[half] <= v ? base + half : base;
    len -= half;
  }
  return (int)(base - a) + (*base <= v ? 1 : 0);
}

// Exclusive scan over the NT threads of NA values per thread, in thread order, with
// the totals: one barrier.  Each call passes its own scratch area (NA * kPlanWarps
// ints) so that no second barrier is needed before the area is written again.
template <int NA, int NT, int BAR>
__device__ __forceinline__ void block_scan(const int (&v)[NA], int (&ex)[NA], int (&tot)[NA],
                                           int *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc[NA];
#pragma unroll
  for (int k = 0; k < NA; k++) inc[k] = warp_incl_scan(v[k]);
  if (lane == 31)
#pragma unroll
    for (int k = 0; k < NA; k++) scratch[k * kPlanWarps + warp] = inc[k];
  group_sync<NT, BAR>();
#pragma unroll
  for (int k = 0; k < NA; k++) {
    int off = 0, t = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; w++) {
      const int x = scratch[k * kPlanWarps + w];
      off += w < warp ? x : 0;
      t += x;
    }
    ex[k] = off + inc[k] - v[k];
    tot[k] = t;
  }
}

// Thread t's contiguous share [b, e) of n elements among NT threads.
template <int NT>
__device__ __forceinline__ void share_of(int n, int &b, int &e) {
  const int per = (n + NT - 1) / NT;
  b = min((int)threadIdx.x * per, n);
  e = min(b + per, n);
}

// The balance problem, from m.cnt, by the first NT threads of the block (the fixed
// rule of the plan; see the file header): block scans over experts, ranks and pieces,
// one thread per element in between.  Writes the solve state into shared memory; misc[M_CAP] != 0 if a rank
// would pass NvS rows or the tables do not fit together (unreachable).  A thread's
// loops run once or twice, so they stay rolled: the plan's code is fetched anew on
// every launch, and unrolled copies would only lengthen that fetch.
template <int NT, int BAR>
__device__ void solve_fast(const Dims &d, const FastSmem &m) {
  const int tid = threadIdx.x;
  const int E = (int)d.E, R = (int)d.R, L = (int)d.L, A = (int)d.A, B = (int)d.B;
  const int SK = (int)d.SK, NvS = (int)d.NvS, PM = (int)d.PMAX;
  int *scr = m.scratch;  // scan areas of 4 * kPlanWarps ints
  int eb, ee, hb, he;
  share_of<NT>(E, eb, ee);
  share_of<NT>(R, hb, he);
  // (1) one scan for two prefixes: the expert counts (global exclusive prefix) and, over
  //     the ranks, overflow, deficit and receivers (rank loads are sums of their experts'
  //     counts); then the receivers (ranks below S*K) in rank order
  int n_recv;
  {
    int v[4] = {0, 0, 0, 0}, ex[4], tot[4];
#pragma unroll 1
    for (int e = eb; e < ee; e++) v[0] += m.cnt[e];
#pragma unroll 1
    for (int h = hb; h < he; h++) {
      int ld = 0;
      for (int e = h * L; e < (h + 1) * L; e++) ld += m.cnt[e];
      m.load[h] = ld;
      v[1] += ld > SK ? ld - SK : 0;
      v[2] += ld < SK ? SK - ld : 0;
      v[3] += ld < SK ? 1 : 0;
    }
    block_scan<4, NT, BAR>(v, ex, tot, scr);
    int run = ex[0];
#pragma unroll 1
    for (int e = eb; e < ee; e++) {
      m.gcst[e] = run;
      run += m.cnt[e];
    }
    int ov = ex[1], df = ex[2], rf = ex[3];
#pragma unroll 1
    for (int h = hb; h < he; h++) {
      const int ld = m.load[h];
      const int o = ld > SK ? ld - SK : 0, dd = ld < SK ? SK - ld : 0;
      m.over[h] = ov;
      m.def[h] = df;
      m.nseg[h] = L;
      if (dd > 0) {
        m.ridx[h] = rf;
        m.rrank[rf] = h;
        m.rbase[rf] = df;
        m.rend[rf] = df + dd;
        rf++;
      } else {
        m.ridx[h] = -1;
      }
      ov += o;
      df += dd;
    }
    n_recv = tot[3];
    if (tid == 0) {
      m.misc[M_CAP] = 0;
      m.misc[M_NREMOTE] = 0;
    }
  }
  group_sync<NT, BAR>();
  // (2) per expert: rows kept at home, its range [oend - ovf, oend) of the overflow
  //     stream, the receivers it reaches (one piece each); piece ids and padded kept rows
  //     by one scan
  int n_piece, padtot;
  {
    int v[2] = {0, 0}, ex[2], tot[2];
#pragma unroll 1
    for (int e = eb; e < ee; e++) {
      const int h = home_of(d, e);
      const int c = m.cnt[e];
      const int cl = m.gcst[e] - m.gcst[h * L];
      int kept = SK - cl;
      kept = kept < 0 ? 0 : (kept > c ? c : kept);
      const int ovf = c - kept;
      const int ost = m.over[h] + (cl > SK ? cl - SK : 0);
      int npc = 0, i0 = 0;
      if (ovf > 0 && n_recv > 0) {
        i0 = upper_bound_bf(m.rend, n_recv, ost);
        int i1 = upper_bound_bf(m.rend, n_recv, ost + ovf - 1);
        if (i1 >= n_recv) i1 = n_recv - 1;
        if (i0 < n_recv) npc = i1 - i0 + 1;
      }
      m.kept[e] = kept;
      m.ovf[e] = ovf;
      m.oend[e] = ost + ovf;
      m.npc[e] = npc;
      m.i0[e] = i0;
      m.eflag[e] = 0;
      v[0] += npc;
      v[1] += A > 1 ? roundup_i(kept, A) : kept;
    }
#pragma unroll 1
    for (int i = tid; i < n_recv; i += NT) m.rfirst[i] = m.rlast[i] = -1;  // set by its pieces
    block_scan<2, NT, BAR>(v, ex, tot, scr + 4 * kPlanWarps);
    int rp = ex[0], rk = ex[1];
#pragma unroll 1
    for (int e = eb; e < ee; e++) {
      m.pid0[e] = rp;
      rp += m.npc[e];
      m.epos[e] = rk;  // global prefix of the padded kept rows
      const int kept = m.kept[e];
      rk += A > 1 ? roundup_i(kept, A) : kept;
    }
    n_piece = tot[0] < PM ? tot[0] : PM;  // pieces <= experts + receivers - 1 < PMAX
    padtot = tot[1];
  }
  group_sync<NT, BAR>();
  // (3) one task per thread: an expert's segment start and first row; a rank's native
  //     rows; a piece's expert, receiver and range (a piece that starts at its
  //     receiver's base is the receiver's first, one that ends at its end the last)
  int bad = 0;
#pragma unroll 1
  for (int t = tid; t < E + R + n_piece; t += NT) {
    if (t < E) {
      const int e = t, h = home_of(d, e);
      const int nst = m.epos[e] - m.epos[h * L];
      m.nst[e] = nst;
      m.row0[e] = h * NvS + nst;
    } else if (t < E + R) {
      const int h = t - E;
      m.ntot[h] = ((h + 1) * L < E ? m.epos[(h + 1) * L] : padtot) - m.epos[h * L];
    } else {
      const int pid = t - E - R;
      const int e = upper_bound_bf(m.pid0, E, pid) - 1;  // its expert: the last first-id <= pid
      int i = e < 0 ? -1 : m.i0[e] + (pid - m.pid0[e]);
      if (e < 0 || i < 0 || i >= n_recv || pid - m.pid0[e] >= m.npc[e]) {
        bad = 1;
        i = 0;
      }
      const int ee2 = e < 0 ? 0 : e;
      const int ost = m.oend[ee2] - m.ovf[ee2];
      const int os = ost > m.rbase[i] ? ost : m.rbase[i];
      const int oe = m.oend[ee2] < m.rend[i] ? m.oend[ee2] : m.rend[i];
      m.pexp[pid] = ee2;
      m.precv[pid] = i;
      m.post[pid] = os;
      m.plen[pid] = oe - os;
      m.pscan[pid] = A > 1 ? roundup_i(oe - os, A) : oe - os;
      if (os == m.rbase[i]) m.rfirst[i] = pid;
      if (oe == m.rend[i]) m.rlast[i] = pid;
    }
  }
  if (bad) atomicOr(&m.misc[M_CAP], 1);
  group_sync<NT, BAR>();
  // (4) alignment > 1: a piece's start is its receiver's native rows plus the padded
  //     lengths of the receiver's earlier pieces (a scan over the pieces)
  if (A > 1) {
    int pb, pe;
    share_of<NT>(n_piece, pb, pe);
    int v[1] = {0}, ex[1], tot[1];
#pragma unroll 1
    for (int pid = pb; pid < pe; pid++) v[0] += m.pscan[pid];
    block_scan<1, NT, BAR>(v, ex, tot, scr + 8 * kPlanWarps);
    group_sync<NT, BAR>();  // every thread has read its values before they are overwritten
    int run = ex[0];
#pragma unroll 1
    for (int pid = pb; pid < pe; pid++) {
      const int x = m.pscan[pid];
      m.pscan[pid] = run;
      run += x;
    }
    group_sync<NT, BAR>();
  }
  // (5) one piece per thread: its first row within the receiving rank (alignment 1: the
  //     receiver's rows follow its native rows in overflow-stream order), capacity,
  //     local-replica flags, remote pieces; one receiver per thread: its segment count
  int cap = 0, nrem = 0;
#pragma unroll 1
  for (int pid = tid; pid < n_piece; pid += NT) {
    const int i = m.precv[pid], first = m.rfirst[i], dr = m.rrank[i];
    if (first < 0 || pid < first) {
      cap = 1;
      continue;
    }
    const int st = A > 1 ? m.ntot[dr] + m.pscan[pid] - m.pscan[first]
                         : m.ntot[dr] + (m.post[pid] - m.rbase[i]);
    m.pst[pid] = st;
    m.prow[pid] = dr * NvS + st;
    if (st + m.plen[pid] > NvS) cap = 1;
    if (pid - first < B) m.eflag[m.pexp[pid]] = 1;
    else nrem++;
  }
#pragma unroll 1
  for (int i = tid; i < n_recv; i += NT) {
    const int first = m.rfirst[i], last = m.rlast[i];
    if (first < 0 || last < first || L + (last - first + 1) > E) cap = 1;
    else m.nseg[m.rrank[i]] = L + (last - first + 1);
  }
#pragma unroll 1
  for (int h = tid; h < R; h += NT)
    if (m.ntot[h] > NvS) cap = 1;
  if (cap) atomicOr(&m.misc[M_CAP], 1);
  if (nrem) atomicAdd(&m.misc[M_NREMOTE], nrem);
  if (tid == 0) {
    m.misc[M_NRECV] = n_recv;
    m.misc[M_NPIECE] = n_piece;
  }
  group_sync<NT, BAR>();
}

// The gather when this launch's expert totals were added up by atomics (every chunk
// adds its counts before it arrives): warp 0 waits for the arrivals; then warps 0..7
// read the totals and solve while warps 8..15 work out the chunk's base offsets.
// Returns the state bits (kStTimeout, kStBad); the solve is done when it returns 0.
template <int V>
__device__ int gather_split(const PlanArgs &a, int64_t k, int epoch, const int32_t *totals,
                            const FastSmem &m) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = (int)a.d.E;
  if (tid < 32) {
    const bool ok = warp_wait_all(a.arrive, a.nc + a.phantom, epoch, a.wait_ns);
    if (lane == 0) m.misc[M_STATE] = ok ? 0 : kStTimeout;
  }
  __syncthreads();
  if (m.misc[M_STATE]) return kStTimeout;
  if (warp < kPlanWarps / 2) {
    constexpr int NT = kPlanThreads / 2;
    // the first bad-id mark is loaded with the totals (one L2 round trip for both)
    const bool has_mark = tid < a.nc;
    const int mark = has_mark ? __ldcg(a.badmark + tid) : 0;
    for (int e = tid; e < E; e += NT) m.cnt[e] = total_of(totals, e);
    bool bad = has_mark && mark == epoch;
    for (int64_t c = tid + NT; c < a.nc; c += NT) bad |= __ldcg(a.badmark + c) == epoch;
    if (bad) atomicOr(&m.misc[M_STATE], kStBad);
    group_sync<NT, 1>();
    if (m.misc[M_STATE] == 0) solve_fast<NT, 1>(a.d, m);
  } else {
    chunk_bases_split<V>(a, k, totals, m);
  }
  __syncthreads();
  return m.misc[M_STATE];
}

// Row of a pair at position pos of expert e's list (solve state in shared memory).
__device__ __forceinline__ int fast_row(const FastSmem &m, int e, int pos) {
  const int kept = m.kept[e];
  if (pos < kept) return m.row0[e] + pos;
  const int o = m.oend[e] - m.ovf[e] + (pos - kept);
  int lo = m.pid0[e], hi = lo + m.npc[e] - 1;  // the last piece of e starting at or before o
  if (hi < lo) return -1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (m.post[mid] <= o) lo = mid; else hi = mid - 1;
  }
  return m.prow[lo] + (o - m.post[lo]);
}

// True if row `row` of rank h holds a pair (inside a segment), false for padding.
__device__ __forceinline__ bool fast_row_used(const Dims &d, const FastSmem &m, int h, int row) {
  const int L = (int)d.L;
  if (row < m.ntot[h]) {  // native segments: the last expert starting at or before row
    int lo = h * L, hi = h * L + L - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (m.nst[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return row < m.nst[lo] + m.kept[lo];
  }
  const int i = m.ridx[h];
  if (i < 0) return false;
  int lo = m.rfirst[i], hi = lo + (m.nseg[h] - L) - 1;
  if (hi < lo) return false;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (m.pst[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return m.pst[lo] <= row && row < m.pst[lo] + m.plen[lo];
}

// The user-facing tables, shared over the CTAs (every CTA holds the whole solve).  Every
// index fits in 32 bits (R * NvS < 2^31 is checked on the host); the loops run a handful
// of times per thread and stay rolled: the code of the plan is fetched from L2 (or
// DRAM, after a step's kernels have streamed through it) on every launch, so its size
// is latency.
__device__ void fast_tables(const PlanArgs &a, const FastSmem &m) {
  const Dims &d = a.d;
  const PlanPtrs &P = a.P;
  const int tid = threadIdx.x;
  const int E = (int)d.E, R = (int)d.R, L = (int)d.L, B = (int)d.B, SK = (int)d.SK;
  const int n_piece = min(m.misc[M_NPIECE], (int)d.PMAX);
  // item i of a table goes to warp i / 32 counted across the CTAs first (warp w of CTA b
  // is warp w * gridDim + b): the stores spread over every SM, 32 to a line
  const int gt = ((tid >> 5) * (int)gridDim.x + (int)blockIdx.x) * 32 + (tid & 31);
  const int stride = (int)gridDim.x * kPlanThreads;
#pragma unroll 1
  for (int e = gt; e < E; e += stride) {
    const int h = home_of(d, e);
    const int si = h * E + (e - h * L);
    P.f[F_EXPERT_COUNT][e] = m.cnt[e];
    P.f[F_EXP_PIECE_BEGIN][e] = m.pid0[e];
    P.f[F_EXP_PIECE_END][e] = m.pid0[e] + m.npc[e];
    P.f[F_SEG_EXPERT][si] = e;
    P.f[F_SEG_START][si] = m.nst[e];
    P.f[F_SEG_LEN][si] = m.kept[e];
    P.f[F_SEG_KIND][si] = MOONEP_SEG_NATIVE;
    P.f[F_SEG_WSLOT][si] = -1;
  }
#pragma unroll 1
  for (int pid = gt; pid < n_piece; pid += stride) {
    const int i = m.precv[pid], dr = m.rrank[i], j = pid - m.rfirst[i], e = m.pexp[pid];
    const int ws = j < B ? j : -1;
    P.f[F_PIECE_EXPERT][pid] = e;
    P.f[F_PIECE_RANK][pid] = dr;
    P.f[F_PIECE_START][pid] = m.pst[pid];
    P.f[F_PIECE_LEN][pid] = m.plen[pid];
    P.f[F_PIECE_WSLOT][pid] = ws;
    P.f[F_PIECE_OSTART][pid] = m.post[pid];
    if (j >= 0 && L + j < E) {
      const int sj = dr * E + L + j;
      P.f[F_SEG_EXPERT][sj] = e;
      P.f[F_SEG_START][sj] = m.pst[pid];
      P.f[F_SEG_LEN][sj] = m.plen[pid];
      P.f[F_SEG_KIND][sj] = ws >= 0 ? MOONEP_SEG_REPLICA : MOONEP_SEG_REMOTE;
      P.f[F_SEG_WSLOT][sj] = ws;
    }
    if (ws >= 0) P.f[F_REP_EXPERT][dr * B + j] = e;
  }
#pragma unroll 1
  for (int h = gt; h < R; h += stride) {
    const int ld = m.load[h];
    P.f[F_RANK_LOAD][h] = ld;
    P.f[F_OVERFLOW][h] = ld > SK ? ld - SK : 0;
    P.f[F_DEFICIT][h] = ld < SK ? SK - ld : 0;
    P.f[F_N_SEG][h] = m.nseg[h];
  }
#pragma unroll 1
  for (int q = gt; q < R * E; q += stride) {  // unused segment entries
    const int h = q / E, i = q - h * E;
    if (i >= m.nseg[h]) {
      P.f[F_SEG_EXPERT][q] = -1;
      P.f[F_SEG_START][q] = 0;
      P.f[F_SEG_LEN][q] = 0;
      P.f[F_SEG_KIND][q] = -1;
      P.f[F_SEG_WSLOT][q] = -1;
    }
  }
#pragma unroll 1
  for (int q = gt; q < R * B; q += stride) {  // free replica weight slots
    const int h = q / B, j = q - h * B;
    if (j >= m.nseg[h] - L) P.f[F_REP_EXPERT][q] = -1;
  }
  if (d.A > 1) {  // padding rows hold no pair
    int32_t *slot_src = P.f[F_SLOT_SRC];
    const int NvS = (int)d.NvS, rows = (int)(d.R * d.NvS);
#pragma unroll 1
    for (int q = gt; q < rows; q += stride) {
      const int h = q / NvS;
      if (!fast_row_used(d, m, h, q - h * NvS)) slot_src[q] = -1;
    }
  }
  if (blockIdx.x == gridDim.x - 1) {  // the last chunk is the smallest: this CTA adds the rest
    // the replicated experts in ascending order: a ballot per warp of 32 experts, the
    // warps' counts added up in shared memory
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = lanemask_lt();
    int carry = 0;
#pragma unroll 1
    for (int e0 = 0; e0 < E; e0 += kPlanThreads) {
      const int e = e0 + tid;
      const bool f = e < E && m.eflag[e];
      const uint32_t b = __ballot_sync(0xffffffffu, f);
      if (lane == 0) m.scratch[warp] = __popc(b);
      __syncthreads();
      int before = carry, all = 0;
#pragma unroll
      for (int w = 0; w < kPlanWarps; w++) {
        const int x = m.scratch[w];
        before += w < warp ? x : 0;
        all += x;
      }
      if (f) P.f[F_REPLICATED][before + __popc(b & lt)] = e;
      carry += all;
      __syncthreads();
    }
    if (tid == 0) {
      const int n_remote = m.misc[M_NREMOTE];
      int32_t *sc = P.f[F_SCALARS];
      sc[S_N_PIECE] = n_piece;
      sc[S_N_REMOTE] = n_remote;
      sc[S_N_LOCAL] = n_piece - n_remote;
      sc[S_N_REPLICATED] = carry;
      sc[S_BAD] = 0;
      sc[5] = sc[6] = sc[7] = 0;
      if (d.mode == MOONEP_MODE_TRAIN && n_remote > 0) set_status(a.status, MOONEP_DEV_BUDGET);
    }
  }
}

// Data phases of the fused forward layer (plan_fused_kernel): the buffers of the
// identity-expert layer and the dispatch chunking of a token row.
struct FusedArgs {
  const float *gates;  // [N]
  const uint4 *x;      // [R*S, H/8]
  uint4 *recv;         // [R*NvS, H/8]
  uint4 *out;          // [R*S, H/8]
  int64_t nvec;        // H / 8
  int64_t nch;         // column chunks a token row is cut into for dispatch
  int64_t cl;          // vectors per chunk (<= 32 * kFusedU)
};
constexpr int kFusedU = 14;  // dispatch: 16-byte vectors per lane of a column chunk

// Zero-copy dispatch of this CTA's tokens [t0, t1): a warp loads a column chunk of a
// token row once (kFusedU vectors per lane in flight) and stores it to the token's K
// rows (srow: the rows of the chunk's pairs, pair order).
__device__ void fused_dispatch(const FusedArgs &f, int64_t t0, int64_t t1, int K, const int *srow) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nunits = (t1 - t0) * f.nch;
  for (int64_t u = warp; u < nunits; u += kPlanWarps) {
    const int64_t tl = u / f.nch, t = t0 + tl;
    const int64_t c0 = (u - tl * f.nch) * f.cl;
    const int64_t c1 = c0 + f.cl < f.nvec ? c0 + f.cl : f.nvec;
    const uint4 *src = f.x + t * f.nvec;
    uint4 buf[kFusedU];
#pragma unroll
    for (int q = 0; q < kFusedU; q++) {
      const int64_t v = c0 + q * 32 + lane;
      if (v < c1) buf[q] = __ldcs(src + v);
    }
    for (int k = 0; k < K; k++) {
      const int row = srow[tl * K + k];
      if (row < 0) continue;
      uint4 *dst = f.recv + (int64_t)row * f.nvec;
#pragma unroll
      for (int q = 0; q < kFusedU; q++) {
        const int64_t v = c0 + q * 32 + lane;
        if (v < c1) dst[v] = buf[q];
      }
    }
  }
}

// Combine of this CTA's tokens from the rows it has just dispatched (identity expert:
// y = recv): a warp per token, the K rows of a column chunk loaded before any
// arithmetic, fused multiply-adds in ascending k, one rounding to bf16.
__device__ void fused_combine(const FusedArgs &f, int64_t t0, int64_t t1, int K, const int *srow) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t t = t0 + warp; t < t1; t += kPlanWarps) {
    const int my_slot = lane < K ? srow[(t - t0) * K + lane] : -1;
    const float my_w = lane < K ? __ldg(f.gates + t * K + lane) : 0.f;
    int rows[8];
    float ws[8];
#pragma unroll
    for (int k = 0; k < 8; k++) {
      rows[k] = __shfl_sync(0xffffffffu, my_slot, k);
      ws[k] = __shfl_sync(0xffffffffu, my_w, k);
    }
    for (int64_t v0 = 0; v0 < f.nvec; v0 += 64) {
      uint4 q[8][2];
#pragma unroll
      for (int k = 0; k < 8; k++)
#pragma unroll
        for (int uu = 0; uu < 2; uu++) {
          const int64_t v = v0 + uu * 32 + lane;
          q[k][uu] = (rows[k] >= 0 && v < f.nvec) ? __ldcg(f.recv + (int64_t)rows[k] * f.nvec + v)
                                                  : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int uu = 0; uu < 2; uu++) {
        const int64_t v = v0 + uu * 32 + lane;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; k++) {
          if (rows[k] < 0) continue;  // k >= K, or a pair without a slot
          const uint32_t wd[4] = {q[k][uu].x, q[k][uu].y, q[k][uu].z, q[k][uu].w};
#pragma unroll
          for (int i = 0; i < 4; i++) {
            acc[2 * i] = __fmaf_rn(ws[k], bf16_lo(wd[i]), acc[2 * i]);
            acc[2 * i + 1] = __fmaf_rn(ws[k], bf16_hi(wd[i]), acc[2 * i + 1]);
          }
        }
        if (v < f.nvec) {
          uint4 o;
          o.x = pack_bf16x2(acc[0], acc[1]);
          o.y = pack_bf16x2(acc[2], acc[3]);
          o.z = pack_bf16x2(acc[4], acc[5]);
          o.w = pack_bf16x2(acc[6], acc[7]);
          f.out[t * f.nvec + v] = o;
        }
      }
    }
  }
}

// kFused: the plan followed, in the same launch, by the dispatch of this CTA's tokens
// and the combine of the same tokens (identity expert; a chunk holds whole tokens).
template <bool kFused>
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs a, FusedArgs f) {
  // launched with programmatic stream serialisation: wait here until the kernel
  // before it in the stream (the router's top-k, the previous layer) has completed
  // and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) int smem[];
  __shared__ int s_epoch, s_fast;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Dims &d = a.d;
  const int64_t k = blockIdx.x;  // this CTA's chunk
  const FastSmem m = carve_fast(d, smem);
  int32_t *gen = a.sync + kSyncGen;
  // the generation word and the two totals tags: needed only when the chunk is
  // published, so their loads overlap the counting (the previous launch has completed,
  // so plain loads see its writes)
  int gen_v = 0, tag0 = 0, tag1 = 0;
  if (tid == 0) {
    gen_v = *((volatile int32_t *)gen);
    tag0 = *((volatile int32_t *)(a.sync + kSyncTotTag));
    tag1 = *((volatile int32_t *)(a.sync + kSyncTotTag + 1));
  }
  int ev[kPairsPerThread], rk[kPairsPerThread];
  // the epoch, once the ids' loads are in flight; the chunk's counts go by atomics
  // into copy k % 16 of this epoch's totals buffer as soon as they are summed, if that
  // buffer was zeroed for exactly this epoch by the launch before (else: first use of
  // the workspace, or it ran another kernel)
  const bool bad = __syncthreads_or(count_chunk<true>(
      a, k, m.tmp, ev, rk,
      [&] {
        if (tid == 0) {
          const int e = (int)((unsigned)gen_v + kEpochStep);
          s_epoch = e;
          s_fast = ((e & 1) ? tag1 : tag0) == e;
        }
      },
      [&]() -> int32_t * {
        return s_fast ? a.totals + ((s_epoch & 1) * kTotalCopies + k % kTotalCopies) * MOONEP_MAX_EXPERTS
                      : nullptr;
      }));
  const int epoch = s_epoch;
  const bool fast = s_fast;
  int32_t *totals = a.totals + (epoch & 1) * kTotalCopies * MOONEP_MAX_EXPERTS;
  if (tid == 0) {
    if (bad) set_status(a.status, MOONEP_DEV_BAD_EXPERT_ID);
    a.badmark[k] = bad ? epoch : ~epoch;
    // the histogram row and the totals were written by every thread before the
    // barriers above; the release store orders all of it (barrier, then release:
    // cumulative) before the flag
    st_release(a.arrive + k, epoch);
  }
  {
    // zero this CTA's share of the other totals buffer for the next launch (nobody uses
    // it in this one): warps 1.. do it while warp 0 polls the arrivals.  Every CTA gets
    // here, and the next launch reads the buffer and its tag only after this grid has
    // completed, so no ordering inside this launch is needed.
    const int nxt = (epoch & 1) ^ 1;
    int4 *other = reinterpret_cast<int4 *>(a.totals + nxt * kTotalCopies * MOONEP_MAX_EXPERTS);
    constexpr int n4 = kTotalCopies * MOONEP_MAX_EXPERTS / 4;
    const int per = (n4 + (int)gridDim.x - 1) / (int)gridDim.x;
    const int z0 = (int)k * per, z1 = z0 + per < n4 ? z0 + per : n4;
    if (warp > 0)
      for (int i = z0 + tid - 32; i < z1; i += kPlanThreads - 32) other[i] = make_int4(0, 0, 0, 0);
    if (k == 0 && tid == 0)
      *((volatile int32_t *)(a.sync + kSyncTotTag + nxt)) = (int)((unsigned)epoch + kEpochStep);
  }
  int st;
  if (fast)
    st = (d.E & 7) == 0 ? gather_split<8>(a, k, epoch, totals, m) : gather_split<1>(a, k, epoch, totals, m);
  else
    st = (d.E & 7) == 0 ? gather_all<8>(a, k, epoch, m) : gather_all<1>(a, k, epoch, m);
  // every CTA has arrived, so every CTA has read the generation word; a bad id
  // does not stop this, the next launch must get a new epoch in any case
  if (k == 0 && tid == 0) *((volatile int32_t *)gen) = epoch;
  if (st == 0) {
    if (!fast) solve_fast<kPlanThreads, 0>(d, m);
    if (m.misc[M_CAP]) st = kStCapacity;
  }
  int32_t *slot_of = a.P.f[F_SLOT_OF];
  if (st) {  // an invalid plan: no pair has a slot, no row a pair
    const int64_t p0 = k * a.ch, p1 = (k + 1) * a.ch < d.N ? (k + 1) * a.ch : d.N;
    for (int64_t p = p0 + tid; p < p1; p += kPlanThreads) slot_of[p] = -1;
    int32_t *slot_src = a.P.f[F_SLOT_SRC];
    for (int64_t q = k * kPlanThreads + tid; q < d.R * d.NvS; q += (int64_t)gridDim.x * kPlanThreads)
      slot_src[q] = -1;
    if (tid == 0) {
      if (st & kStTimeout) set_status(a.status, MOONEP_DEV_TIMEOUT);
      if (k == 0) {
        if (st & kStCapacity) set_status(a.status, MOONEP_DEV_CAPACITY);
        int32_t *sc = a.P.f[F_SCALARS];
        for (int i = 0; i < 8; i++) sc[i] = 0;
        sc[S_BAD] = st;
      }
    }
    if (kFused) {  // as the separate calls would: nothing dispatched, every output row zero
      const int64_t t0 = k * a.ch / d.K;
      const int64_t t1 = ((k + 1) * a.ch < d.N ? (k + 1) * a.ch : d.N) / d.K;
      for (int64_t q = t0 * f.nvec + tid; q < t1 * f.nvec; q += kPlanThreads) f.out[q] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  // place this chunk's pairs
  {
    int32_t *slot_src = a.P.f[F_SLOT_SRC];
    const int64_t nrows = d.R * d.NvS;
    const int64_t base = k * a.ch + (int64_t)warp * 32 * a.ppt;
#pragma unroll
    for (int j = 0; j < kPairsPerThread; j++) {
      if (j >= a.ppt) break;
      const int64_t p = base + j * 32 + lane;
      if (p >= d.N) continue;
      const int e = ev[j];
      int row = e >= 0 ? fast_row(m, e, m.base[e] + rk[j]) : -1;
      if (row < 0 || row >= nrows) row = -1;  // unreachable for a consistent plan
      slot_of[p] = row;
      if (row >= 0) slot_src[row] = (int32_t)p;
      if (kFused) m.tmp[p - k * a.ch] = row;  // the chunk's rows, pair order
    }
  }
  if (kFused) {
    // a chunk holds whole tokens (K divides 512): every row a token's combine reads was
    // written by this CTA's dispatch, so a CTA barrier orders the two phases
    const int K = (int)d.K;
    const int64_t t0 = k * a.ch / K;
    const int64_t t1 = ((k + 1) * a.ch < d.N ? (k + 1) * a.ch : d.N) / K;
    __syncthreads();
    fused_dispatch(f, t0, t1, K, m.tmp);
    __syncthreads();
    fused_combine(f, t0, t1, K, m.tmp);
  }
  fast_tables(a, m);
}


size_t plan_multichunk_smem_bytes(const Dims &d) {
  const size_t worker = std::max<size_t>(size_t(kPlanWarps) * d.E,
                                         6 * d.E + 2 * d.PMAX + 4 + 4 * kPlanThreads);
  const size_t solver = solve_smem_ints(d);
  return std::max(worker, solver) * sizeof(int) + 16;
}

size_t plan_smem_bytes(const Dims &d) { return fast_smem_ints(d) * sizeof(int) + 16; }

// Host-side launch facts of the two plan kernels, cached per device for the
// context they were taken in (a kernel's dynamic shared memory limit is a
// per-context attribute): SM count, the opt-in shared memory limit, and
// co-resident CTAs per SM for the dynamic shared memory sizes seen so far.
struct KernelLaunchInfo {
  int limit = 0;          // largest dynamic shared memory a launch may request
  bool attr_set = false;  // that limit has been set on the kernel in this context
  size_t occ_smem[8] = {};
  int occ_ctas[8] = {};
  int occ_n = 0;
};
struct DeviceLaunchInfo {
  unsigned long long ctx = 0;
  int sms = 0;
  KernelLaunchInfo k[3];  // 0: plan_kernel<false>, 1: plan_multichunk_kernel, 2: plan_kernel<true>
};
std::mutex g_launch_mu;
DeviceLaunchInfo g_launch[kMaxDevices];

// Co-resident CTAs per SM of kernel `which` with `smem` bytes of dynamic shared
// memory (the kernel's limit raised first when past 48 KB); 0 if it does not
// fit, -1 on a CUDA error.  *sms receives the SM count.
template <typename F>
int plan_ctas_per_sm(F f, int which, int dev, size_t smem, int *sms) {
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_launch_mu);
  DeviceLaunchInfo &di = g_launch[dev];
  if (ctx == 0 || di.ctx != ctx) {  // first call in this context (or no context id)
    di = DeviceLaunchInfo();
    di.ctx = ctx;
  }
  if (di.sms == 0 && (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) !=
                          cudaSuccess || di.sms <= 0)) {
    cudaGetLastError();
    di.sms = 0;
    return -1;
  }
  *sms = di.sms;
  KernelLaunchInfo &ki = di.k[which];
  if (ki.limit == 0) {
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, f) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    ki.limit = optin - (int)fa.sharedSizeBytes;
    if (ki.limit <= 0) return -1;
  }
  if (smem > size_t(ki.limit)) return 0;
  // the device's whole limit, so concurrent callers with other configs never lower
  // it under each other
  if (smem > 48 * 1024 && !ki.attr_set) {
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, ki.limit) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    ki.attr_set = true;
  }
  for (int i = 0; i < ki.occ_n; i++)
    if (ki.occ_smem[i] == smem) return ki.occ_ctas[i];
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kPlanThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  const int slot = ki.occ_n < 8 ? ki.occ_n++ : int(smem % 8);
  ki.occ_smem[slot] = smem;
  ki.occ_ctas[slot] = per_sm;
  return per_sm;
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

namespace moonep {
namespace {
// The plan launch shared by moonep_plan and moonep_fused_forward (fused != nullptr: the
// one-chunk-per-CTA kernel with the data phases, or MOONEP_ERR_UNSUPPORTED when the
// chunks do not fit on the co-resident CTAs).  Arguments were checked by the caller.
moonep_status_t launch_plan(const Dims &d, const int32_t *topk_idx, void *plan_arena,
                            void *workspace, int32_t *dev_status, moonep_stream_t stream,
                            const FusedArgs *fused) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOONEP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOONEP_ERR_UNSUPPORTED;

  // one chunk per CTA when the chunks fit on the co-resident CTAs: pairs spread
  // over them, 512..8192 pairs a chunk (a cooperative launch guarantees that the
  // CTAs run at the same time)
  int sms = 0;
  const size_t smem = plan_smem_bytes(d);
  const int per_sm = fused ? plan_ctas_per_sm(plan_kernel<true>, 2, dev, smem, &sms)
                           : plan_ctas_per_sm(plan_kernel<false>, 0, dev, smem, &sms);
  if (per_sm < 0) return MOONEP_ERR_CUDA;
  PlanArgs a;
  a.d = d;
  bool one_chunk_per_cta = false;
  size_t kernel_smem = smem;
  if (per_sm > 0) {
    const int64_t coresident = (int64_t)sms * per_sm;
    int64_t ppt = (d.N + coresident * kPlanThreads - 1) / (coresident * kPlanThreads);
    ppt = ppt < 1 ? 1 : ppt;
    if (ppt <= kPairsPerThread) {
      one_chunk_per_cta = true;
      a.ppt = (int)ppt;
      a.ch = ppt * kPlanThreads;
      a.nc = d.N > 0 ? (d.N + a.ch - 1) / a.ch : 1;
      a.workers = (int)a.nc;
    }
  }
  if (!one_chunk_per_cta) {
    if (fused) return MOONEP_ERR_UNSUPPORTED;
    // chunks outnumber the co-resident CTAs: one solving CTA, workers with
    // several chunks each
    kernel_smem = plan_multichunk_smem_bytes(d);
    const int ms = plan_ctas_per_sm(plan_multichunk_kernel, 1, dev, kernel_smem, &sms);
    if (ms < 0) return MOONEP_ERR_CUDA;
    if (ms == 0) return MOONEP_ERR_UNSUPPORTED;
    const int64_t coresident = (int64_t)sms * ms;
    if (coresident < 2) return MOONEP_ERR_UNSUPPORTED;
    const int64_t wmax = coresident - 1;
    int64_t ppt = (d.N + wmax * kPlanThreads - 1) / (wmax * kPlanThreads);
    ppt = ppt < 1 ? 1 : (ppt > kPairsPerThread ? kPairsPerThread : ppt);
    a.ppt = (int)ppt;
    a.ch = ppt * kPlanThreads;
    a.nc = d.N > 0 ? (d.N + a.ch - 1) / a.ch : 1;
    a.workers = (int)(a.nc < wmax ? a.nc : wmax);
  }
  if (a.nc > d.NCMAX) return MOONEP_ERR_UNSUPPORTED;  // cannot happen: chunks >= 512 pairs
  a.idx = topk_idx;
  a.P = plan_ptrs(d, plan_arena);
  WsLayout wl(d);
  char *ws = static_cast<char *>(workspace);
  a.sync = reinterpret_cast<int32_t *>(ws + wl.off[W_SYNC]);
  a.totals = reinterpret_cast<int32_t *>(ws + wl.off[W_TOTALS]);
  a.arrive = reinterpret_cast<int32_t *>(ws + wl.off[W_ARRIVE]);
  a.badmark = reinterpret_cast<int32_t *>(ws + wl.off[W_BADMARK]);
  a.hist = reinterpret_cast<int32_t *>(ws + wl.off[W_HIST]);
  a.rank = reinterpret_cast<uint16_t *>(ws + wl.off[W_RANK]);
  a.exp_kept = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_KEPT]);
  a.exp_row0 = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_ROW0]);
  a.exp_ostart = reinterpret_cast<int32_t *>(ws + wl.off[W_EXP_OSTART]);
  a.piece_grow = reinterpret_cast<int32_t *>(ws + wl.off[W_PIECE_GROW]);
  a.status = dev_status;
  a.wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  a.phantom = g_phantom_arrivals.load(std::memory_order_relaxed);
  const FusedArgs f = fused ? *fused : FusedArgs{};

  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(one_chunk_per_cta ? a.nc : a.workers + 1));
  lc.blockDim = dim3(kPlanThreads);
  lc.dynamicSmemBytes = kernel_smem;
  lc.stream = to_cuda(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  auto go = [&]() {
    if (!one_chunk_per_cta) return cudaLaunchKernelEx(&lc, plan_multichunk_kernel, a);
    return fused ? cudaLaunchKernelEx(&lc, plan_kernel<true>, a, f)
                 : cudaLaunchKernelEx(&lc, plan_kernel<false>, a, f);
  };
  // programmatic dependent launch hides the launch gap after the previous
  // kernel; without it (a runtime that refuses the pair) the launch is plain
  lc.numAttrs = g_plan_pdl.load(std::memory_order_relaxed) ? 2 : 1;
  if (go() == cudaSuccess) return MOONEP_OK;
  cudaGetLastError();
  if (lc.numAttrs == 2) {
    g_plan_pdl.store(false);
    lc.numAttrs = 1;
    if (go() == cudaSuccess) return MOONEP_OK;
    cudaGetLastError();
  }
  return MOONEP_ERR_CUDA;
}
}  // namespace
}  // namespace moonep

extern "C" moonep_status_t moonep_plan(const moonep_config_t *cfg, const int32_t *topk_idx,
                                       void *plan_arena, void *workspace, int32_t *dev_status,
                                       moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d)) return MOONEP_ERR_INVALID_ARG;
  if (!plan_arena || !workspace || !dev_status || (d.N > 0 && !topk_idx))
    return MOONEP_ERR_INVALID_ARG;
  if (!aligned256(plan_arena) || !aligned256(workspace)) return MOONEP_ERR_INVALID_ARG;
  return launch_plan(d, topk_idx, plan_arena, workspace, dev_status, stream, nullptr);
}

extern "C" moonep_status_t moonep_fused_forward(const moonep_config_t *cfg, const int32_t *topk_idx,
                                                const float *gates, const uint16_t *x,
                                                void *plan_arena, void *workspace, uint16_t *recv,
                                                uint16_t *out, int32_t *dev_status,
                                                moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d) || d.H < 1) return MOONEP_ERR_INVALID_ARG;
  if (!plan_arena || !workspace || !dev_status) return MOONEP_ERR_INVALID_ARG;
  if (d.N > 0 && (!topk_idx || !gates || !x || !recv || !out)) return MOONEP_ERR_INVALID_ARG;
  if (!aligned256(plan_arena) || !aligned256(workspace)) return MOONEP_ERR_INVALID_ARG;
  // whole tokens per chunk (chunks are multiples of 512 pairs), 16-byte rows, K <= 8
  if (kPlanThreads % d.K != 0 || d.K > 8 || d.H % 8 != 0) return MOONEP_ERR_UNSUPPORTED;
  if (d.N > 0 && (!aligned16(x) || !aligned16(recv) || !aligned16(out))) return MOONEP_ERR_UNSUPPORTED;
  FusedArgs f;
  f.gates = gates;
  f.x = reinterpret_cast<const uint4 *>(x);
  f.recv = reinterpret_cast<uint4 *>(recv);
  f.out = reinterpret_cast<uint4 *>(out);
  f.nvec = d.H / 8;
  f.nch = (f.nvec + 32 * kFusedU - 1) / (32 * kFusedU);
  f.cl = (f.nvec + f.nch - 1) / f.nch;
  return launch_plan(d, topk_idx, plan_arena, workspace, dev_status, stream, &f);
}

namespace moonep {
long long debug_wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
int debug_phantom() { return g_phantom_arrivals.load(std::memory_order_relaxed); }

namespace {
// driver entry points (no link-time dependency on libcuda)
typedef int (*CtxGetCurrentFn)(void **ctx);
typedef int (*CtxGetIdFn)(void *ctx, unsigned long long *id);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_fns_once;
}  // namespace

unsigned long long current_context_id() {
  std::call_once(g_ctx_fns_once, [] {
    void *f = nullptr, *g = nullptr;
    cudaDriverEntryPointQueryResult qf = cudaDriverEntryPointSymbolNotFound, qg = qf;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &qf) == cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &g, cudaEnableDefault, &qg) == cudaSuccess &&
        qf == cudaDriverEntryPointSuccess && qg == cudaDriverEntryPointSuccess && f && g) {
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(g);
    }
    cudaGetLastError();
  });
  if (!g_ctx_get_current || !g_ctx_get_id) return 0;
  void *ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_get_current(&ctx) != 0 || !ctx || g_ctx_get_id(ctx, &id) != 0) return 0;
  return id;
}

int current_sm_count() {
  static std::atomic<int> sms[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 148;
  }
  int v = sms[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return 148;
    }
    sms[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}
}  // namespace moonep

extern "C" moonep_status_t moonep_debug_set_wait(int64_t limit_ns, int32_t phantom_arrivals) {
  if (limit_ns < 0 || phantom_arrivals < 0 || phantom_arrivals > kSyncMaxPhantom)
    return MOONEP_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_ns);
  g_phantom_arrivals.store(phantom_arrivals);
  return MOONEP_OK;
}

// ------------------------------------------------ allocation-free variant ---
// Scratch for moonep_plan_static: a fixed device array that lives as long as
// the library is loaded.  Host code cannot use the symbol itself as a device
// pointer: its device address is looked up with cudaGetSymbolAddress.  That
// address belongs to one context's copy of the module (a device reset, or a
// second context on the same device, loads the module again, possibly
// elsewhere), so it is cached per device together with the id of the context
// it was looked up in, and looked up again whenever the current context's id
// differs.
static __device__ __align__(256) unsigned char g_plan_scratch[MOONEP_STATIC_WORKSPACE_BYTES];

namespace {
struct ScratchAddr {
  unsigned long long ctx_id;
  void *addr;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch_addr[kMaxDevices];

// Device address of g_plan_scratch in the current context; nullptr on error.
void *static_scratch(int dev) {
  unsigned long long id = current_context_id();
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (id != 0 && g_scratch_addr[dev].ctx_id == id) return g_scratch_addr[dev].addr;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return nullptr;
  }
  id = current_context_id();  // the lookup makes the device's context current if it was not
  if (id != 0) {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    g_scratch_addr[dev] = {id, p};
  }
  return p;
}
}  // namespace

extern "C" moonep_status_t moonep_plan_static(const moonep_config_t *cfg, const int32_t *topk_idx,
                                              void *plan_arena, int32_t *dev_status,
                                              moonep_stream_t stream) {
  Dims d;
  if (!make_dims(cfg, &d)) return MOONEP_ERR_INVALID_ARG;
  // every host-checkable argument first: nothing below runs for a bad call
  if (!plan_arena || !dev_status || (d.N > 0 && !topk_idx) || !aligned256(plan_arena))
    return MOONEP_ERR_INVALID_ARG;
  if (WsLayout(d).total > (size_t)MOONEP_STATIC_WORKSPACE_BYTES) return MOONEP_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOONEP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOONEP_ERR_UNSUPPORTED;
  void *scratch = static_scratch(dev);
  if (!scratch) return MOONEP_ERR_CUDA;
  // the ordinary plan with the static array as its workspace: every scratch
  // word it reads is written earlier in the same call, and its arrival flags
  // are tagged with a per-launch epoch, so nothing needs clearing
  return moonep_plan(cfg, topk_idx, plan_arena, scratch, dev_status, stream);
}
