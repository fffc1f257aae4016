/*
 * moonep_oracle.c — plain, slow CPU oracle for the MoonEP balanced expert-parallel
 * hot path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product path never does.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * What it follows.  The pages describe the outcome of MoonEP's planner, not its
 * code:
 *   - "Moonshot AI Open-Sources MoonEP" (the S x K paragraph): every rank
 *     receives exactly S*K token-slots however skewed the routing, by
 *     duplicating overloaded experts onto other ranks; the replica-slot
 *     paragraph: E/R weight slots per rank in training, 3-4 in inference with
 *     remote reads past the budget.
 *   - "MoonshotAI/MoonEP 딥다이브" §2② (zero copy: each token is written
 *     straight to its final expert-ordered slot, the buffer view feeds the
 *     experts), §4 pattern 1 (plan once, reuse in combine and backward),
 *     pattern 2 (fixed NvS = S*K + alignment padding rows), pattern 3
 *     (replica gradients are summed back into the home expert, identical to no
 *     replication), §8 exercise C (dispatch -> no-op -> combine is the identity
 *     on the gate-weighted sum).
 * The pages fix no tie-breaks.  This oracle takes one fixed, deterministic rule:
 *   1. list_e = the (rank, token, k) pairs routed to expert e, in that
 *      lexicographic order; count[e] = |list_e|.
 *   2. Expert e lives on home rank e / L (L = E/R).  load_h = sum of the counts
 *      of rank h's experts; overflow_h = max(0, load_h - S*K);
 *      deficit_h = max(0, S*K - load_h).
 *   3. stream_h = list_e for rank h's experts in ascending e, concatenated.  Its
 *      first S*K entries stay home; the remaining overflow_h entries leave.
 *   4. The global overflow stream O is the concatenation, over h ascending, of
 *      the leaving entries.  Underloaded ranks d, ascending, each take the next
 *      deficit_d entries of O.
 *   5. A receiver's run is split into maximal same-expert pieces; piece j of a
 *      receiver uses local replica weight slot j if j < budget, else it is a
 *      REMOTE piece (weights read from the home rank).  In training mode a
 *      REMOTE piece is reported as a budget error; the plan is still produced.
 *   6. Rank d's rows: its native experts dL..dL+L-1 ascending (possibly empty),
 *      then its pieces in O order.  Segment i starts at the sum of
 *      roundup(len, A) over the segments before it (A = alignment).
 *      NvS = S*K + (A-1) * min(E, S*K).
 *   7. slot_of[pair] = d*NvS + start(segment) + index within the segment;
 *      slot_src[d*NvS + row] = flat pair id (r*S + s)*K + k, or -1 for padding.
 * Data steps:
 *   dispatch   recv[slot_of[p]] = x[token(p)]                (bit copy)
 *   combine    acc = 0; for k: acc = fmaf(w_k, y[slot_k], acc); out = bf16(acc)
 *              (fp32 accumulation in k order, the precision the method fixes)
 *   combine-bw dY[slot_k] = bf16(w_k * dOut[t]) (one fp32 product);
 *              dgate[t,k] = sum_h dOut[t,h] * y[slot_k,h] accumulated in double
 *   reduce_grad home[e] = bf16(float(home[e]) + sum over e's local replica pieces,
 *              in O order (ascending receiver), of float(rep[d][slot]))
 *   reduce_grad over fp32 gradient buffers: the same sum in the same order, with
 *              fp32 gradients in and out (no bf16 rounding anywhere)
 *   dispatch-bw dx[t] = bf16( sum_k float(dRecv[slot_k]) ), fp32 adds in k order (the
 *              adjoint of dispatch; the backward pass reuses the forward plan, §4 pattern 1)
 *   prefetch   rep_w[d][j] = w[e] for every local replica piece (d, j) of expert e
 *              (the duplicated experts' weights are fetched before compute: news page,
 *              S x K paragraph; Buffer.prefetch_weight, deep-dive §3③)
 * bf16 rounding is round-to-nearest-even on the fp32 bit pattern.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* status values returned by the oracle (its own numbering) */
#define ORC_OK 0
#define ORC_INVALID_ARG 1
#define ORC_BAD_EXPERT_ID 2
#define ORC_BUDGET 4
#define ORC_CAPACITY 8

#define KIND_NATIVE 0
#define KIND_REPLICA 1
#define KIND_REMOTE 2

typedef struct {
  int32_t R, E, K, S, H, budget, mode, align;
} orc_config;

/* Every array is caller-allocated on the host with the stated length. */
typedef struct {
  int32_t *expert_count;  /* [E] */
  int32_t *rank_load;     /* [R] */
  int32_t *overflow;      /* [R] */
  int32_t *deficit;       /* [R] */
  int32_t *n_seg;         /* [R] */
  int32_t *seg_expert;    /* [R*E]  segment i of rank d at d*E + i */
  int32_t *seg_start;     /* [R*E]  first row within rank d */
  int32_t *seg_len;       /* [R*E] */
  int32_t *seg_kind;      /* [R*E]  KIND_* */
  int32_t *seg_wslot;     /* [R*E]  replica weight slot, -1 for native / remote */
  int32_t *n_piece;       /* [1] */
  int32_t *piece_expert;  /* [E+R] pieces in O order */
  int32_t *piece_rank;    /* [E+R] receiving rank */
  int32_t *piece_start;   /* [E+R] first row within the receiving rank */
  int32_t *piece_len;     /* [E+R] */
  int32_t *piece_wslot;   /* [E+R] */
  int32_t *piece_ostart;  /* [E+R] position of the piece's first entry in O */
  int32_t *rep_expert;    /* [R*budget] expert held in weight slot j of rank d, -1 if none */
  int32_t *n_remote;      /* [1] */
  int32_t *slot_of;       /* [R*S*K] */
  int32_t *slot_src;      /* [R*NvS] */
} orc_plan_out;

static int64_t roundup64(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

int64_t orc_nvs(const orc_config *c) {
  int64_t sk = (int64_t)c->S * c->K;
  int64_t a = c->align;
  int64_t m = sk < c->E ? sk : c->E;
  return sk + (a - 1) * m;
}

int orc_validate(const orc_config *c) {
  if (c->R < 1 || c->E < 1 || c->E % c->R != 0) return ORC_INVALID_ARG;
  if (c->K < 1 || c->K > c->E || c->S < 0 || c->budget < 0 || c->align < 1) return ORC_INVALID_ARG;
  if (c->mode != 0 && c->mode != 1) return ORC_INVALID_ARG;
  return ORC_OK;
}

/* ------------------------------------------------------------------ plan --- */
int orc_plan(const orc_config *c, const int32_t *topk_idx, orc_plan_out *out) {
  int st = orc_validate(c);
  if (st != ORC_OK) return st;
  const int64_t R = c->R, E = c->E, K = c->K, S = c->S, A = c->align, B = c->budget;
  const int64_t L = E / R;
  const int64_t SK = (int64_t)S * K;
  const int64_t npairs = (int64_t)R * S * K;
  const int64_t NvS = orc_nvs(c);
  int64_t p, e, h, d, i;

  for (p = 0; p < npairs; p++)
    if (topk_idx[p] < 0 || topk_idx[p] >= E) return ORC_BAD_EXPERT_ID;

  /* step 1: per-expert lists in (rank, token, k) order (stable bucket fill) */
  int64_t *list_begin = calloc((size_t)E + 1, sizeof(int64_t));
  int64_t *fill = calloc((size_t)E, sizeof(int64_t));
  int64_t *list = malloc((size_t)(npairs ? npairs : 1) * sizeof(int64_t));
  for (e = 0; e < E; e++) out->expert_count[e] = 0;
  for (p = 0; p < npairs; p++) out->expert_count[topk_idx[p]]++;
  for (e = 0; e < E; e++) list_begin[e + 1] = list_begin[e] + out->expert_count[e];
  for (p = 0; p < npairs; p++) {
    e = topk_idx[p];
    list[list_begin[e] + fill[e]] = p;
    fill[e]++;
  }

  /* step 2: loads, overflow, deficit */
  int64_t total_over = 0, total_def = 0;
  for (h = 0; h < R; h++) {
    int64_t load = 0;
    for (e = h * L; e < (h + 1) * L; e++) load += out->expert_count[e];
    out->rank_load[h] = (int32_t)load;
    out->overflow[h] = (int32_t)(load > SK ? load - SK : 0);
    out->deficit[h] = (int32_t)(load < SK ? SK - load : 0);
    total_over += out->overflow[h];
    total_def += out->deficit[h];
  }
  if (total_over != total_def) { /* cannot happen: total load is R*S*K */
    free(list_begin); free(fill); free(list);
    return ORC_INVALID_ARG;
  }

  /* step 3 + 4: walk each home stream; first S*K entries stay, the tail joins O.
     kept[e] = how many of e's entries stay home. O holds pair ids, O_expert their expert. */
  int64_t *kept = calloc((size_t)E, sizeof(int64_t));
  int64_t *O = malloc((size_t)(total_over ? total_over : 1) * sizeof(int64_t));
  int32_t *O_expert = malloc((size_t)(total_over ? total_over : 1) * sizeof(int32_t));
  int64_t n_O = 0;
  for (h = 0; h < R; h++) {
    int64_t t = 0; /* position in stream_h */
    for (e = h * L; e < (h + 1) * L; e++) {
      for (i = list_begin[e]; i < list_begin[e + 1]; i++) {
        if (t < SK) {
          kept[e]++;
        } else {
          O[n_O] = list[i];
          O_expert[n_O] = (int32_t)e;
          n_O++;
        }
        t++;
      }
    }
  }

  /* step 4 + 5: receivers take consecutive runs of O; runs split into pieces */
  int64_t n_piece = 0;
  for (i = 0; i < R * B; i++) out->rep_expert[i] = -1;
  int32_t *pieces_of_rank = calloc((size_t)(R > 0 ? R : 1), sizeof(int32_t));
  int64_t *first_piece_of_rank = calloc((size_t)(R > 0 ? R : 1), sizeof(int64_t));
  int64_t remote = 0;
  int64_t o = 0;
  for (d = 0; d < R; d++) {
    int64_t need = out->deficit[d];
    first_piece_of_rank[d] = n_piece;
    int64_t j = 0;
    while (need > 0) {
      int32_t ex = O_expert[o];
      int64_t len = 0;
      int64_t ostart = o;
      while (need > 0 && O_expert[o] == ex) { o++; need--; len++; }
      out->piece_expert[n_piece] = ex;
      out->piece_rank[n_piece] = (int32_t)d;
      out->piece_len[n_piece] = (int32_t)len;
      out->piece_ostart[n_piece] = (int32_t)ostart;
      if (j < B) {
        out->piece_wslot[n_piece] = (int32_t)j;
        out->rep_expert[d * B + j] = ex;
      } else {
        out->piece_wslot[n_piece] = -1;
        remote++;
      }
      n_piece++;
      j++;
    }
    pieces_of_rank[d] = (int32_t)j;
  }
  *out->n_piece = (int32_t)n_piece;
  *out->n_remote = (int32_t)remote;

  /* step 6: segment layout of every rank */
  int capacity_bad = 0;
  int64_t *native_start = calloc((size_t)E, sizeof(int64_t));
  for (d = 0; d < R; d++) {
    int64_t cursor = 0;
    int32_t nseg = 0;
    for (e = d * L; e < (d + 1) * L; e++) {
      int64_t idx = d * E + nseg;
      out->seg_expert[idx] = (int32_t)e;
      out->seg_start[idx] = (int32_t)cursor;
      out->seg_len[idx] = (int32_t)kept[e];
      out->seg_kind[idx] = KIND_NATIVE;
      out->seg_wslot[idx] = -1;
      native_start[e] = cursor;
      cursor += roundup64(kept[e], A);
      nseg++;
    }
    for (i = first_piece_of_rank[d]; i < first_piece_of_rank[d] + pieces_of_rank[d]; i++) {
      int64_t idx = d * E + nseg;
      out->seg_expert[idx] = out->piece_expert[i];
      out->seg_start[idx] = (int32_t)cursor;
      out->seg_len[idx] = out->piece_len[i];
      out->seg_kind[idx] = out->piece_wslot[i] >= 0 ? KIND_REPLICA : KIND_REMOTE;
      out->seg_wslot[idx] = out->piece_wslot[i];
      out->piece_start[i] = (int32_t)cursor;
      cursor += roundup64(out->piece_len[i], A);
      nseg++;
    }
    out->n_seg[d] = nseg;
    for (i = nseg; i < E; i++) {
      out->seg_expert[d * E + i] = -1;
      out->seg_start[d * E + i] = 0;
      out->seg_len[d * E + i] = 0;
      out->seg_kind[d * E + i] = -1;
      out->seg_wslot[d * E + i] = -1;
    }
    /* the last segment's rows must end inside NvS */
    int64_t used = 0;
    for (i = 0; i < nseg; i++) {
      int64_t end = out->seg_start[d * E + i] + out->seg_len[d * E + i];
      if (end > used) used = end;
    }
    if (used > NvS) capacity_bad = 1;
  }

  /* step 7: slot of every pair, source of every row */
  for (i = 0; i < R * NvS; i++) out->slot_src[i] = -1;
  if (!capacity_bad) {
    for (e = 0; e < E; e++) {
      int64_t home = e / L;
      for (i = 0; i < kept[e]; i++) {
        int64_t pair = list[list_begin[e] + i];
        int64_t row = home * NvS + native_start[e] + i;
        out->slot_of[pair] = (int32_t)row;
        out->slot_src[row] = (int32_t)pair;
      }
    }
    for (i = 0; i < n_piece; i++) {
      int64_t r = out->piece_rank[i];
      for (int64_t q = 0; q < out->piece_len[i]; q++) {
        int64_t pair = O[out->piece_ostart[i] + q];
        int64_t row = r * NvS + out->piece_start[i] + q;
        out->slot_of[pair] = (int32_t)row;
        out->slot_src[row] = (int32_t)pair;
      }
    }
  }

  free(list_begin); free(fill); free(list); free(kept); free(O); free(O_expert);
  free(pieces_of_rank); free(first_piece_of_rank); free(native_start);
  if (capacity_bad) return ORC_CAPACITY;
  if (c->mode == 0 && remote > 0) return ORC_BUDGET;
  return ORC_OK;
}

/* ------------------------------------------------------------ bf16 <-> f32 --- */
float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
    return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays a quiet NaN */
  /* round to nearest, ties to even, on the 16 bits that are dropped */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* -------------------------------------------------------------- dispatch --- */
/* recv[slot_of[p]] = x[p / K] for every pair; rows not named by a slot are left alone. */
void orc_dispatch(const orc_config *c, const int32_t *slot_of, const uint16_t *x, uint16_t *recv) {
  const int64_t npairs = (int64_t)c->R * c->S * c->K;
  const int64_t H = c->H;
  for (int64_t p = 0; p < npairs; p++) {
    int64_t t = p / c->K;
    int64_t row = slot_of[p];
    for (int64_t h = 0; h < H; h++) recv[row * H + h] = x[t * H + h];
  }
}

/* ---------------------------------------------------------------- combine --- */
/* out[t] = bf16( sum_k w[t,k] * y[slot_of[t,k]] ), fp32 fused multiply-add in k order. */
void orc_combine_tokens(const orc_config *c, const int32_t *slot_of, const uint16_t *y,
                        const float *gates, const int64_t *tokens, int64_t n_tokens,
                        uint16_t *out) {
  const int64_t K = c->K, H = c->H;
  for (int64_t n = 0; n < n_tokens; n++) {
    int64_t t = tokens ? tokens[n] : n;
    for (int64_t h = 0; h < H; h++) {
      float acc = 0.0f;
      for (int64_t k = 0; k < K; k++) {
        int64_t row = slot_of[t * K + k];
        acc = fmaf(gates[t * K + k], orc_bf16_to_f32(y[row * H + h]), acc);
      }
      out[n * H + h] = orc_f32_to_bf16(acc);
    }
  }
}

/* ------------------------------------------------------- combine-backward --- */
/* dY[slot_of[t,k]] = bf16(w[t,k] * dOut[t]);  dgate[t,k] = <dOut[t], y[slot_of[t,k]]> */
void orc_combine_backward_tokens(const orc_config *c, const int32_t *slot_of,
                                 const uint16_t *dout, const uint16_t *y, const float *gates,
                                 const int64_t *tokens, int64_t n_tokens,
                                 uint16_t *dy_rows /* [n_tokens*K, H] */, float *dgates) {
  const int64_t K = c->K, H = c->H;
  for (int64_t n = 0; n < n_tokens; n++) {
    int64_t t = tokens ? tokens[n] : n;
    for (int64_t k = 0; k < K; k++) {
      int64_t row = slot_of[t * K + k];
      float w = gates[t * K + k];
      double dot = 0.0;
      for (int64_t h = 0; h < H; h++) {
        float g = orc_bf16_to_f32(dout[t * H + h]);
        float prod = w * g;
        dy_rows[(n * K + k) * H + h] = orc_f32_to_bf16(prod);
        dot += (double)g * (double)orc_bf16_to_f32(y[row * H + h]);
      }
      dgates[n * K + k] = (float)dot;
    }
  }
}

/* ------------------------------------------------------------ reduce_grad --- */
/* For every expert e: home[e] = bf16( float(home[e]) + sum of its local replica
   pieces' gradients, pieces taken in O order ).  rep is [R, budget, P], home [E, P]. */
void orc_reduce_grad(const orc_config *c, const int32_t *piece_expert, const int32_t *piece_rank,
                     const int32_t *piece_wslot, int32_t n_piece, const uint16_t *rep,
                     uint16_t *home, int64_t P) {
  const int64_t B = c->budget;
  for (int64_t e = 0; e < c->E; e++) {
    int has = 0;
    for (int32_t i = 0; i < n_piece; i++)
      if (piece_expert[i] == e && piece_wslot[i] >= 0) has = 1;
    if (!has) continue;
    for (int64_t q = 0; q < P; q++) {
      float acc = orc_bf16_to_f32(home[e * P + q]);
      for (int32_t i = 0; i < n_piece; i++) {
        if (piece_expert[i] != e || piece_wslot[i] < 0) continue;
        int64_t slot = (int64_t)piece_rank[i] * B + piece_wslot[i];
        acc = acc + orc_bf16_to_f32(rep[slot * P + q]);
      }
      home[e * P + q] = orc_f32_to_bf16(acc);
    }
  }
}

/* For every expert e with a local replica piece, over fp32 gradient buffers:
   home[e] = home[e] + the pieces' gradients, fp32 additions starting from home[e]
   and taking the pieces in O order (ascending receiver), with no rounding to bf16
   ("MoonshotAI/MoonEP 딥다이브" §4 pattern 3: replica gradients are added into
   the home expert's gradient; a training step that keeps its expert gradients in
   fp32 buffers folds them there).  rep is [R, budget, P], home [E, P]. */
void orc_reduce_grad_f32(const orc_config *c, const int32_t *piece_expert, const int32_t *piece_rank,
                         const int32_t *piece_wslot, int32_t n_piece, const float *rep, float *home,
                         int64_t P) {
  const int64_t B = c->budget;
  for (int64_t e = 0; e < c->E; e++) {
    for (int64_t q = 0; q < P; q++) {
      float acc = home[e * P + q];
      for (int32_t i = 0; i < n_piece; i++) {
        if (piece_expert[i] != e || piece_wslot[i] < 0) continue;
        int64_t slot = (int64_t)piece_rank[i] * B + piece_wslot[i];
        acc = acc + rep[slot * P + q];
      }
      home[e * P + q] = acc;
    }
  }
}

/* ------------------------------------------------------ dispatch-backward --- */
/* dx[t] = bf16( sum_k float(drecv[slot_of[t,k]]) ), fp32 additions in k order. */
void orc_dispatch_backward_tokens(const orc_config *c, const int32_t *slot_of,
                                  const uint16_t *drecv, const int64_t *tokens, int64_t n_tokens,
                                  uint16_t *dx) {
  const int64_t K = c->K, H = c->H;
  for (int64_t n = 0; n < n_tokens; n++) {
    int64_t t = tokens ? tokens[n] : n;
    for (int64_t h = 0; h < H; h++) {
      float acc = 0.0f;
      for (int64_t k = 0; k < K; k++) {
        int64_t row = slot_of[t * K + k];
        acc = acc + orc_bf16_to_f32(drecv[row * H + h]);
      }
      dx[n * H + h] = orc_f32_to_bf16(acc);
    }
  }
}

/* -------------------------------------------------------- segment_weights --- */
/* The weight matrix each entry of the per-rank segment tables computes with: a
   native segment reads its home expert's weights w[e]; a replica piece reads its
   rank's local slot rep_w[d][j]; a remote piece (no local slot, past the budget)
   reads the home weights w[e] on the home rank; an unused entry reads nothing.
   buf[q] = 0 for w, 1 for rep_w, -1 for none; off[q] = the matrix's first
   element in that buffer (row * W), -1 for none.  q = d * E + i. */
void orc_segment_weights(const orc_config *c, const int32_t *seg_expert, const int32_t *seg_kind,
                         const int32_t *seg_wslot, int64_t W, int32_t *buf, int64_t *off) {
  const int64_t R = c->R, E = c->E, B = c->budget;
  for (int64_t d = 0; d < R; d++) {
    for (int64_t i = 0; i < E; i++) {
      const int64_t q = d * E + i;
      if (seg_kind[q] == KIND_REPLICA) {
        buf[q] = 1;
        off[q] = (d * B + seg_wslot[q]) * W;
      } else if (seg_kind[q] == KIND_NATIVE || seg_kind[q] == KIND_REMOTE) {
        buf[q] = 0;
        off[q] = (int64_t)seg_expert[q] * W;
      } else {
        buf[q] = -1;
        off[q] = -1;
      }
    }
  }
}

/* --------------------------------------------------------- prefetch_weight --- */
/* For every piece with a local weight slot: rep_w[rank][slot] = w[expert] (W elements).
   rep_w is [R, budget, W]; w is [E, W]. */
void orc_prefetch_weight(const orc_config *c, const int32_t *piece_expert,
                         const int32_t *piece_rank, const int32_t *piece_wslot, int32_t n_piece,
                         const uint16_t *w, uint16_t *rep_w, int64_t W) {
  const int64_t B = c->budget;
  for (int32_t i = 0; i < n_piece; i++) {
    if (piece_wslot[i] < 0) continue;
    int64_t slot = (int64_t)piece_rank[i] * B + piece_wslot[i];
    for (int64_t q = 0; q < W; q++) rep_w[slot * W + q] = w[(int64_t)piece_expert[i] * W + q];
  }
}
