/*
 * moonep.h — C ABI of libmoonep.so: the data-parallel hot path of MoonEP-style
 * perfectly balanced expert parallelism on one B200.  The R expert-parallel
 * ranks of a layer are R partitions of one device's memory.
 *
 * Steps (in pipeline order, "MoonshotAI/MoonEP 딥다이브" §5 file order):
 *   moonep_plan              router top-k -> static balanced plan (every rank gets S*K rows)
 *   moonep_dispatch          zero-copy scatter of token rows into expert-ordered slots
 *   moonep_combine           gate-weighted gather-sum of expert outputs back to tokens
 *   moonep_combine_backward  gradients of combine w.r.t. expert outputs and gates
 *   moonep_reduce_grad       fold replica-expert gradients into their home experts
 *                            (moonep_reduce_grad_f32: the same over fp32 gradient buffers)
 *   moonep_dispatch_backward gradient of dispatch (sum of a token's K slot gradients)
 *   moonep_prefetch_weight   copy duplicated experts' weights into replica slots
 *   moonep_segment_weights   the weight matrix each segment's expert computation reads
 *   moonep_fused_forward     plan + dispatch + combine of the identity expert in one launch
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and frees every buffer (device memory
 *     for tensors, the plan arena and the workspace).  The library never
 *     allocates, frees or synchronises the host.
 *   - Streams: every call only enqueues work on `stream` (0 = legacy default
 *     stream) and returns; results are valid once that stream reaches them.
 *   - Return value: host-checkable errors (bad config, null or misaligned
 *     pointer, launch failure).  On any non-OK return nothing was enqueued
 *     except possibly work that ran before a launch failure.
 *   - Device status: data-dependent errors found by the kernels are OR-ed into
 *     the caller's device int32 `*dev_status` (MOONEP_DEV_* bits).  The caller
 *     zeroes it once and reads it whenever it chooses.
 *   - bf16 tensors are passed as uint16_t bit patterns, row-major, rows
 *     contiguous.  Row counts use the symbols of moonep_config_t.
 *   - Alignment: every pointer is aligned to its element type, as C requires
 *     of a typed pointer (2 bytes for bf16, 4 for int32 and fp32).  The calls
 *     check null pointers and the 256-byte alignment of the plan arena and the
 *     workspace.  Rows whose byte length or base is not a multiple of 16 take a
 *     scalar path.  Element alignment itself is not checked.
 *   - Layouts: topk_idx int32 [R, S, K]; gates fp32 [R, S, K]; x / out / dout
 *     bf16 [R, S, H]; the dispatch buffer bf16 [R, NvS, H] (rank d owns rows
 *     d*NvS .. d*NvS+NvS-1); replica gradients bf16 [R, budget, P]; home
 *     gradients bf16 [E, P] (expert e at row e; its home rank is e / (E/R)).
 */
#ifndef MOONEP_H
#define MOONEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the ABI are exported; everything else in the library is hidden. */
#if defined(__GNUC__)
#define MOONEP_API __attribute__((visibility("default")))
#else
#define MOONEP_API
#endif

/* A CUDA stream handle (the same object as cudaStream_t / CUstream). */
typedef struct CUstream_st *moonep_stream_t;

#define MOONEP_MODE_TRAIN 0 /* replica budget must hold every duplicate locally */
#define MOONEP_MODE_INFER 1 /* pieces past the budget become remote reads */

/* Largest supported sizes (shared-memory tables of the planning kernel). */
#define MOONEP_MAX_EXPERTS 1024
#define MOONEP_MAX_TOPK 32

typedef struct moonep_config {
  int32_t R;      /* expert-parallel ranks, >= 1 */
  int32_t E;      /* experts, multiple of R; expert e lives on rank e / (E/R) */
  int32_t K;      /* experts per token, 1 <= K <= min(E, MOONEP_MAX_TOPK) */
  int32_t S;      /* tokens per rank, >= 0 */
  int32_t H;      /* hidden size (bf16 elements per row), >= 1 for data calls */
  int32_t budget; /* replica weight slots per rank, 0 <= budget <= E */
  int32_t mode;   /* MOONEP_MODE_TRAIN or MOONEP_MODE_INFER */
  int32_t align;  /* segment alignment A in rows, 1 <= A <= 4096 (1: NvS = S*K) */
} moonep_config_t;

typedef enum moonep_status {
  MOONEP_OK = 0,
  MOONEP_ERR_INVALID_ARG = 1, /* config out of range, null or misaligned pointer */
  MOONEP_ERR_CUDA = 2,        /* a CUDA launch or runtime call failed */
  MOONEP_ERR_UNSUPPORTED = 3  /* sizes past the documented limits */
} moonep_status_t;

/* Bits OR-ed into *dev_status by the kernels. */
#define MOONEP_DEV_BAD_EXPERT_ID 0x1 /* a topk_idx entry outside [0, E): plan marks all pairs -1 */
#define MOONEP_DEV_CAPACITY 0x2      /* a rank's segments would pass NvS rows (never by design) */
#define MOONEP_DEV_BUDGET 0x4        /* TRAIN mode and a replica piece had no local weight slot */
#define MOONEP_DEV_TIMEOUT 0x8       /* a bounded wait inside a kernel gave up */
#define MOONEP_DEV_BAD_PLAN 0x10     /* a data call met a slot outside [-1, R*NvS) */

/* Segment kinds in the plan's per-rank segment table. */
#define MOONEP_SEG_NATIVE 0  /* the rank's own expert */
#define MOONEP_SEG_REPLICA 1 /* a duplicated expert whose weights sit in local slot `wslot` */
#define MOONEP_SEG_REMOTE 2  /* a duplicated expert past the budget: weights read remotely */

/* Device pointers into a plan arena (filled by moonep_plan_view; host-only call).
 * Sizes: N = R*S*K pairs, P_MAX = E + R pieces.  Pair p = (r*S + s)*K + k. */
typedef struct moonep_plan_view {
  int32_t *slot_of;            /* [N] global row d*NvS + row of pair p (-1 only after a bad id) */
  int32_t *slot_src;           /* [R*NvS] pair id held by each row, -1 for padding */
  int32_t *expert_count;       /* [E] pairs routed to each expert (utilisation) */
  int32_t *rank_load;          /* [R] pairs whose expert lives on each rank */
  int32_t *overflow;           /* [R] max(0, load - S*K) */
  int32_t *deficit;            /* [R] max(0, S*K - load) */
  int32_t *n_seg;              /* [R] valid entries of each rank's segment table */
  int32_t *seg_expert;         /* [R*E] segment i of rank d at d*E+i: expert (-1 unused) */
  int32_t *seg_start;          /* [R*E] first row within the rank (multiple of A) */
  int32_t *seg_len;            /* [R*E] rows */
  int32_t *seg_kind;           /* [R*E] MOONEP_SEG_* (-1 unused) */
  int32_t *seg_wslot;          /* [R*E] replica weight slot, -1 for native / remote */
  int32_t *piece_expert;       /* [P_MAX] replica pieces in overflow-stream order; entries of
                                  every piece table at index >= scalars[0] are unspecified */
  int32_t *piece_rank;         /* [P_MAX] receiving rank */
  int32_t *piece_start;        /* [P_MAX] first row within the receiving rank */
  int32_t *piece_len;          /* [P_MAX] rows */
  int32_t *piece_wslot;        /* [P_MAX] local weight slot or -1 (remote) */
  int32_t *piece_ostart;       /* [P_MAX] offset of the piece in the overflow stream */
  int32_t *expert_piece_begin; /* [E] pieces of expert e are [begin, end) */
  int32_t *expert_piece_end;   /* [E] */
  int32_t *rep_expert;         /* [R*budget] expert in weight slot j of rank d, -1 if free */
  int32_t *replicated_experts; /* [E] experts with >= 1 local replica, ascending; count in
                                  scalars[3], later entries unspecified */
  int32_t *scalars;            /* [8] 0 n_piece, 1 n_remote, 2 n_local_pieces, 3 n_replicated */
  int64_t nvs;                 /* rows per rank */
  int32_t max_pieces;          /* P_MAX */
} moonep_plan_view_t;

/* Rows per rank of the dispatch buffer: NvS = S*K + (A-1)*min(E, S*K).
 * Fixed by the config alone, whatever the routing ("MoonshotAI/MoonEP 딥다이브"
 * §4 pattern 2: NvS = S x K + alignment padding).  Returns -1 for a bad config. */
MOONEP_API int64_t moonep_nvs(const moonep_config_t *cfg);

/* Bytes of the plan arena (device, 256-byte aligned base) for this config; 0 if invalid. */
MOONEP_API size_t moonep_plan_bytes(const moonep_config_t *cfg);

/* Bytes of scratch the plan needs (device, 256-byte aligned base); 0 if invalid.
 * Contents need no initialisation: any bytes are valid before a call.  A call
 * leaves state for the next call on the same workspace (a generation word and
 * expert totals zeroed ahead, at fixed offsets, for any config); a call that
 * finds none (the first on a workspace) takes a slower gather with the same
 * result.  Calls that share a workspace must be ordered on the GPU. */
MOONEP_API size_t moonep_workspace_bytes(const moonep_config_t *cfg);

/* Plan ("Moonshot AI Open-Sources MoonEP", S x K and replica-slot paragraphs;
 * "MoonshotAI/MoonEP 딥다이브" §4 pattern 1: computed once per layer in forward
 * and reused by combine and both backward passes).
 * Rule: pairs routed to expert e are listed in (rank, token, k) order; each home
 * rank keeps the first S*K entries of its experts' lists taken in ascending
 * expert order; the remaining entries, concatenated over ranks ascending, fill
 * the underloaded ranks in ascending order; each receiver's run splits into
 * same-expert pieces, piece j using weight slot j if j < budget (else remote).
 * Rank d's rows: native experts ascending, then pieces; segments start at
 * multiples of A.  Every rank then holds exactly S*K valid rows.
 *   topk_idx   device int32 [R*S*K] (may be NULL when S == 0)
 *   plan_arena device, moonep_plan_bytes(cfg) bytes, 256-byte aligned; written
 *   workspace  device, moonep_workspace_bytes(cfg) bytes, 256-byte aligned
 *   dev_status device int32, bits OR-ed: BAD_EXPERT_ID, BUDGET, CAPACITY, TIMEOUT
 * Enqueues one cooperative kernel (its CTAs are co-resident and wait for each
 * other with bounded waits, see moonep_debug_set_wait). */
MOONEP_API moonep_status_t moonep_plan(const moonep_config_t *cfg, const int32_t *topk_idx, void *plan_arena,
                            void *workspace, int32_t *dev_status, moonep_stream_t stream);

/* Allocation-free variant of moonep_plan.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory on their
 * own — for example a plugin running inside another engine that only hands it
 * the tensors of one call, or a serving loop that reserved all device memory up
 * front and must not call cudaMalloc (which can also synchronise the device)
 * while it runs.  Such a caller passes only inputs and outputs; the plan's
 * scratch is a fixed array of MOONEP_STATIC_WORKSPACE_BYTES inside the library
 * (a device global that every GPU which loads the library keeps until exit).
 *   - Same arguments and results as moonep_plan, without `workspace`.
 *   - Configs whose moonep_workspace_bytes() exceeds the array are rejected
 *     with MOONEP_ERR_UNSUPPORTED before anything is enqueued.
 *   - Host-checkable arguments (config, null or misaligned pointers, size)
 *     are checked before any CUDA call.
 *   - The first call in a CUDA context (with the device current) looks up the
 *     array's device address in that context and caches it under the
 *     context's id; a device reset or another context on the same device has
 *     a new id, so the first call there looks it up again.  Make the first
 *     call in each context before any stream capture.  Nothing is allocated
 *     or freed, ever.
 *   - All calls on a device share the one array and find it as the previous
 *     call left it; no word of it needs to start at zero (each is written
 *     before it is read in the same call, and the arrival flags carry a
 *     per-launch epoch).  Calls whose execution overlaps on the GPU (other
 *     streams, concurrent graphs) race and must be ordered by the caller. */
#define MOONEP_STATIC_WORKSPACE_BYTES (4u << 20)

MOONEP_API moonep_status_t moonep_plan_static(const moonep_config_t *cfg, const int32_t *topk_idx,
                                              void *plan_arena, int32_t *dev_status,
                                              moonep_stream_t stream);

/* Diagnostics for the bounded in-kernel waits (process-wide, host-side).
 * The plan is one cooperative launch whose CTAs wait for every CTA's arrival
 * (batches of more chunks than co-resident CTAs also wait for the solving CTA);
 * reduce_grad's pipeline waits on shared-memory barriers for its bulk copies.
 * Each wait gives up after `limit_ns` nanoseconds (default 200 ms) and sets
 * MOONEP_DEV_TIMEOUT instead of hanging (a timed-out plan is invalid:
 * slot_of = -1).  `phantom_arrivals` (tests only, 0..32) forces the timeout:
 * the plan's CTAs also wait for that many arrivals that no CTA ever makes, and
 * each reduce_grad CTA's first stage expects 16 bytes per phantom arrival more
 * than its copies deliver. */
MOONEP_API moonep_status_t moonep_debug_set_wait(int64_t limit_ns, int32_t phantom_arrivals);

/* Fill `out` with device pointers into `plan_arena` (pure host arithmetic). */
MOONEP_API moonep_status_t moonep_plan_view(const moonep_config_t *cfg, const void *plan_arena,
                                 moonep_plan_view_t *out);

/* Zero-copy dispatch ("MoonshotAI/MoonEP 딥다이브" §2②: each token is written
 * straight into its final expert-ordered position, no permute afterwards):
 *   recv[slot_of[p]] = x[p / K]   bit copy of H bf16 values, for every pair p.
 *   x    device bf16 [R*S, H];  recv device bf16 [R*NvS, H] (padding rows untouched)
 * x and recv must not overlap. */
MOONEP_API moonep_status_t moonep_dispatch(const moonep_config_t *cfg, const void *plan_arena,
                                const uint16_t *x, uint16_t *recv, int32_t *dev_status,
                                moonep_stream_t stream);

/* Combine ("MoonshotAI/MoonEP 딥다이브" §3③ combine; §8 exercise C):
 *   out[t] = bf16( sum_{k=0..K-1} gates[t,k] * y[slot_of[t*K+k]] )
 * accumulated in fp32 with fused multiply-adds in ascending k, rounded once to
 * bf16 (nearest-even).  y device bf16 [R*NvS, H] (may be the dispatch buffer:
 * identity expert); gates device fp32 [R*S*K]; out device bf16 [R*S, H]. */
MOONEP_API moonep_status_t moonep_combine(const moonep_config_t *cfg, const void *plan_arena,
                               const uint16_t *y, const float *gates, uint16_t *out,
                               int32_t *dev_status, moonep_stream_t stream);

/* Backward of combine (reuses the forward plan, §4 pattern 1):
 *   dy[slot_of[t*K+k]] = bf16( gates[t,k] * dout[t] )       (one fp32 product)
 *   dgates[t*K+k]      = sum_h dout[t,h] * y[slot_of[t*K+k], h]   (fp32)
 * dout bf16 [R*S, H]; y bf16 [R*NvS, H]; dy bf16 [R*NvS, H] (padding untouched;
 * must not overlap y); dgates fp32 [R*S*K]. */
MOONEP_API moonep_status_t moonep_combine_backward(const moonep_config_t *cfg, const void *plan_arena,
                                        const uint16_t *dout, const uint16_t *y,
                                        const float *gates, uint16_t *dy, float *dgates,
                                        int32_t *dev_status, moonep_stream_t stream);

/* reduce_grad ("MoonshotAI/MoonEP 딥다이브" §4 pattern 3: replica gradients live
 * in a separate buffer and are added into the home expert's gradient, so training
 * equals no replication):
 *   for each expert e with local replica pieces (plan order = ascending rank d):
 *     home[e, :] = bf16( float(home[e, :]) + sum_d float(rep[d, wslot_d(e), :]) )
 * in fp32, in place.  rep_grads device bf16 [R, budget, P]; home_grads device
 * bf16 [E, P]; P >= 1 elements per expert gradient.  Remote pieces have no
 * replica slot and contribute nothing (TRAIN plans flag them as BUDGET).
 * With P % 8 == 0 and 16-byte aligned buffers the kernel stages rows in shared
 * memory with bulk asynchronous copies; its internal waits are bounded and one
 * that gives up (not possible with a consistent plan) sets MOONEP_DEV_TIMEOUT.
 * dev_status bits: BAD_PLAN (inconsistent plan tables), TIMEOUT. */
MOONEP_API moonep_status_t moonep_reduce_grad(const moonep_config_t *cfg, const void *plan_arena,
                                   const uint16_t *rep_grads, uint16_t *home_grads, int64_t P,
                                   int32_t *dev_status, moonep_stream_t stream);

/* reduce_grad over fp32 gradient buffers (the same section of the deep-dive page; for
 * a training step that keeps its expert gradients in fp32):
 *   for each expert e with local replica pieces (plan order = ascending rank d):
 *     home[e, :] = home[e, :] + sum_d rep[d, wslot_d(e), :]
 * fp32 additions starting from home[e, :], pieces in that order, in place; no bf16
 * rounding anywhere.  rep_grads device fp32 [R, budget, P]; home_grads device fp32
 * [E, P]; P >= 1.  Rows are staged in shared memory by bulk copies when P % 4 == 0
 * and both buffers are 16-byte aligned, else a scalar kernel does the same sums.
 * Arguments, errors and dev_status bits as for moonep_reduce_grad. */
MOONEP_API moonep_status_t moonep_reduce_grad_f32(const moonep_config_t *cfg, const void *plan_arena,
                                       const float *rep_grads, float *home_grads, int64_t P,
                                       int32_t *dev_status, moonep_stream_t stream);

/* Backward of dispatch (reuses the forward plan, "MoonshotAI/MoonEP 딥다이브" §4
 * pattern 1): the gradient of each token row is the sum of the gradients of
 * the K slots it was sent to,
 *   dx[t] = bf16( sum_{k=0..K-1} d_recv[slot_of[t*K+k]] )
 * accumulated in fp32 in ascending k, rounded once (nearest-even).
 * d_recv bf16 [R*NvS, H]; dx bf16 [R*S, H]. */
MOONEP_API moonep_status_t moonep_dispatch_backward(const moonep_config_t *cfg,
                                                    const void *plan_arena, const uint16_t *d_recv,
                                                    uint16_t *dx, int32_t *dev_status,
                                                    moonep_stream_t stream);

/* Replica weight prefetch ("Moonshot AI Open-Sources MoonEP", S x K paragraph:
 * duplicated experts are prefetched before computation starts; the
 * replica-slot paragraph: E/R slots in training, 3-4 in inference with remote
 * reads past the budget; Buffer.prefetch_weight, "MoonshotAI/MoonEP 딥다이브" §3③):
 *   rep_weights[d, j, :] = weights[e, :] for every piece of expert e that holds
 *   local weight slot j on rank d (a bit copy; each home row is read once).
 * Remote pieces (weight slot -1 in the plan) are not copied: their segments
 * read weights[e] on the home rank.  weights bf16 [E, W]; rep_weights bf16
 * [R, budget, W] (slots without a piece are left untouched); W >= 1. */
MOONEP_API moonep_status_t moonep_prefetch_weight(const moonep_config_t *cfg,
                                                  const void *plan_arena, const uint16_t *weights,
                                                  uint16_t *rep_weights, int64_t W,
                                                  int32_t *dev_status, moonep_stream_t stream);

/* The weights each entry of the plan's segment tables computes with, for the expert
 * computation between dispatch and combine (same page, replica-slot paragraph: a
 * duplicated expert runs on its receiving rank with the weights prefetched into a
 * local slot, and past the slot budget reads them on its home rank).  Entry
 * q = d*E + i of rank d's segment table gets:
 *   MOONEP_SEG_REPLICA  rep_weights + (d*budget + seg_wslot[q]) * W
 *   MOONEP_SEG_NATIVE   weights + seg_expert[q] * W
 *   MOONEP_SEG_REMOTE   weights + seg_expert[q] * W  (the home copy, read remotely)
 *   unused              NULL
 * Written on the device (no host read of the plan), so a grouped expert kernel can
 * take the rows [seg_start, seg_start + seg_len) of each segment and this pointer.
 *   weights      device bf16 [E, W] (home expert weights; only addresses are formed)
 *   rep_weights  device bf16 [R, budget, W] (may be NULL when budget == 0)
 *   seg_weights  device, R*E pointers, 8-byte aligned; written
 * An entry naming an expert or a slot out of range is NULL and sets
 * MOONEP_DEV_BAD_PLAN. */
MOONEP_API moonep_status_t moonep_segment_weights(const moonep_config_t *cfg, const void *plan_arena,
                                                  const uint16_t *weights, const uint16_t *rep_weights,
                                                  int64_t W, const uint16_t **seg_weights,
                                                  int32_t *dev_status, moonep_stream_t stream);

/* The zero_copy=False comparison path ("MoonshotAI/MoonEP 딥다이브" §6: the
 * zero_copy=True option removes a copy; §8 exercise D measures the epilogue
 * copy it saves).  Rows first land in a per-rank communication buffer `comm`
 * (bf16 [R*NvS, H]) in arrival order, then a permute copies them into the
 * expert-ordered `recv`.  The result is bit-identical to moonep_dispatch; only
 * the extra copy differs.
 *   comm_index  device int32 [R*S*K + R]: on return the comm row of every pair
 *               (order inside a rank unspecified); the last R words are counters
 *   requires H % 8 == 0 and 16-byte aligned x, comm, recv (else UNSUPPORTED).
 * Enqueues a 4-byte-per-rank memset and three kernels. */
MOONEP_API moonep_status_t moonep_dispatch_via_buffer(const moonep_config_t *cfg,
                                                      const void *plan_arena, const uint16_t *x,
                                                      uint16_t *comm, int32_t *comm_index,
                                                      uint16_t *recv, int32_t *dev_status,
                                                      moonep_stream_t stream);

/* The matching combine of the comparison path: the expert outputs y (expert
 * order) are permuted back into `comm` at the rows comm_index gives (as left
 * by moonep_dispatch_via_buffer), then combined from there.  Bit-identical to
 * moonep_combine. */
MOONEP_API moonep_status_t moonep_combine_via_buffer(const moonep_config_t *cfg,
                                                     const void *plan_arena, const uint16_t *y,
                                                     const float *gates, const int32_t *comm_index,
                                                     uint16_t *comm, uint16_t *out,
                                                     int32_t *dev_status, moonep_stream_t stream);

/* The forward layer of the identity expert in one launch, for small batches where
 * launch and hand-off latency matter (the decode path: "Moonshot AI Open-Sources
 * MoonEP", replica-slot paragraph, inference with a few replica slots): moonep_plan,
 * then moonep_dispatch of x into recv, then moonep_combine of y = recv, with the same
 * results bit for bit as those three calls.  Each CTA of the plan's one-chunk-per-CTA
 * launch dispatches and combines the tokens of its own chunk right after placing
 * them: under the identity expert a token's combine reads only rows that the same
 * CTA has just written, so no second grid-wide exchange is needed.  (With a real
 * expert between dispatch and combine this call does not apply.)
 *   topk_idx, gates, x, plan_arena, workspace, dev_status: as for moonep_plan /
 *   moonep_dispatch / moonep_combine; recv bf16 [R*NvS, H] (padding rows untouched);
 *   out bf16 [R*S, H].  The plan tables are complete when the launch ends.
 * MOONEP_ERR_UNSUPPORTED when K does not divide 512 or K > 8 (a chunk must hold whole
 * tokens), H % 8 != 0, x / recv / out not 16-byte aligned, or the batch needs more
 * chunks than co-resident CTAs (more than about 148 * 8192 pairs): use the separate
 * calls then.  A plan that fails (bad expert id, timeout) dispatches nothing and
 * writes zero output rows, as the separate calls would. */
MOONEP_API moonep_status_t moonep_fused_forward(const moonep_config_t *cfg, const int32_t *topk_idx,
                                                const float *gates, const uint16_t *x,
                                                void *plan_arena, void *workspace, uint16_t *recv,
                                                uint16_t *out, int32_t *dev_status,
                                                moonep_stream_t stream);

/* Static description of a status code. */
MOONEP_API const char *moonep_status_string(moonep_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOONEP_H */
