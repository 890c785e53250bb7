/*
 * CPU oracle for the MoE expert-parallel token round trip.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library) never calls it and shares no code with it.
 *
 * It computes, slowly and directly, what the round trip computes:
 *   route    -> top-k expert ids per token + softmax over the k chosen logits
 *   index    -> per-expert counts, exclusive offsets, per-rank counts and
 *               offsets, per-(source rank, expert) counts, and the stable
 *               slot <-> row permutation
 *   dispatch -> copy of each token row to every row it was dispatched to
 *   ffn      -> per-row SwiGLU expert MLP, in float64
 *   combine  -> weighted sum of a token's k expert outputs, in float64
 *
 * Floating point is float64 throughout (inputs are widened exactly); the
 * pages fix no precision.  Notation: T tokens, H hidden, I intermediate,
 * E experts, k experts per token, R logical EP ranks, S = T*k slots; slot
 * s = t*k + j is the j-th choice of token t.
 *
 * Sources (page title, section):
 *  [EPRT]  "EP: Partition Experts and Route Tokens" -- sections "Send tokens
 *          to experts and return their results", "Return multiple expert
 *          results to the same token", "Equal expert counts can receive
 *          different token counts".
 *  [NEURON] "Expert Parallelism (EP)" (vLLM on Neuron design note) --
 *          sections "Weight Layout Across Ranks", "Collective Patterns /
 *          Prefill (CTE kernel)", "Why a Single All-Reduce/Reduce-Scatter
 *          Works", "Limitations" (items 1, 3 and 4).
 *  [WIKI]  "什么是专家并行（Expert Parallelism）？" -- sections "工作机制"
 *          (how it works) and "边界与常见误解" (third point): an expert-
 *          parallel load balancer redistributes hot and cold experts over
 *          the GPUs to keep their utilisation balanced.
 *  [SWIGLU] Shazeer, "GLU Variants Improve Transformer" (2020): FFN_SwiGLU(x)
 *          = (SiLU(x W) * (x V)) W2, SiLU(z) = z * sigmoid(z).  The pages call
 *          each expert "an MLP"; the layer shapes name its form SwiGLU.
 *
 * Parity pins: every function here is checked by the not-gpu tests against
 * the pages' worked examples, closed forms and a dense brute-force MoE.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

static double orc_load(const void* base, int dtype, size_t i) {
  if (dtype == ORC_F32) return (double)((const float*)base)[i];
  uint32_t u = (uint32_t)((const uint16_t*)base)[i] << 16; /* exact widening */
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---------------------------------------------------------- router logits
 * [NEURON] "Router Weights": every token is scored against all E experts;
 * the affinity of token t for expert e is the dot product of the token's
 * activation with expert e's router vector, plus the expert's bias:
 *   logits[t][e] = round_f32( sum_h x[t][h] * w[e][h] + bias[e] )
 * summed in float64 over ascending h from the given (bf16 or float32) values,
 * rounded once to float32.  w is [E][H] (row e = expert e); bias may be NULL.
 * Returns 0, or -1 for bad sizes.
 */
int oracle_router_logits(const void* x, int xdt, const void* w, int wdt, const double* bias, int T, int H, int E,
                         float* logits) {
  if (T < 0 || H < 1 || E < 1) return -1;
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += orc_load(x, xdt, (size_t)t * H + h) * orc_load(w, wdt, (size_t)e * H + h);
      if (bias) acc += bias[e];
      logits[(size_t)t * E + e] = (float)acc;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ route
 * [EPRT] "Send tokens ...": the router chooses each token's expert(s) from
 * all E experts; Top-1 uses combination weight one.  "Return multiple ...":
 * with Top-2 the token's results are combined with per-expert weights kept
 * apart from the expert choice.  Weight rule: softmax over the k selected
 * logits (which gives exactly 1 for k = 1).
 *
 * Order: experts sorted by logit descending; equal logits (IEEE ==, so
 * -0 == +0) keep the lower expert id first.  Plain repeated selection.
 * Returns 0, or -1 for bad sizes.
 */
int oracle_route(const float* logits, int T, int E, int k, int32_t* ids, float* w) {
  if (T < 0 || E < 1 || k < 1 || k > E || k > 64) return -1;
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep lower id */
      }
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    double m = (double)l[ids[(size_t)t * k]];
    double z = 0.0;
    double ex[64];
    for (int j = 0; j < k && j < 64; ++j) {
      ex[j] = exp((double)l[ids[(size_t)t * k + j]] - m);
      z += ex[j];
    }
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(ex[j] / z);
  }
  free(taken);
  return 0;
}

/* Source rank of token t when T tokens are split into R contiguous, as-equal-
 * as-possible ranges (t in [ceil(rT/R), ceil((r+1)T/R)) belongs to rank r).
 * With R | T this is t / (T/R): tokens 0..T/R-1 on rank 0, and so on, as in
 * [EPRT] "Replicate attention ...": each GPU holds its own tokens. */
int oracle_src_rank(int t, int T, int R) { return (int)(((int64_t)t * R) / T); }

/* ------------------------------------------------------------------ index
 * [EPRT] "Send tokens ...": dispatch groups token vectors by the selected
 * expert and keeps each result's association to its original token;
 * "Equal expert counts ...": experts and ranks receive unequal counts.
 * [NEURON] "Limitations" 3-4: rank r owns experts [r*E/R, (r+1)*E/R).
 *
 * Rows are ordered by (expert, token): expert e's rows start at the
 * exclusive prefix sum of the counts of experts < e, and within an expert
 * the rows follow token order (a stable grouping).  Because experts are
 * placed contiguously, that order is also rank-major.
 *
 * Slots whose id is outside [0, E) are dropped: not counted, slot_to_row
 * = -1.  row_to_slot entries past the last placed row are -1.
 * src_expert_counts may be NULL.  Returns the number of dropped slots, or
 * -1 for bad sizes.
 */
int oracle_dispatch_index(const int32_t* ids, int T, int k, int E, int R,
                          int32_t* expert_counts, int32_t* expert_offsets,
                          int32_t* rank_counts, int32_t* rank_offsets,
                          int32_t* slot_to_row, int32_t* row_to_slot,
                          int32_t* src_expert_counts) {
  if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return -1;
  const int S = T * k, EL = E / R;
  int dropped = 0;
  for (int e = 0; e < E; ++e) expert_counts[e] = 0;
  for (int s = 0; s < S; ++s) {
    if (ids[s] < 0 || ids[s] >= E) { ++dropped; continue; }
    expert_counts[ids[s]] += 1;
  }
  expert_offsets[0] = 0;
  for (int e = 0; e < E; ++e) expert_offsets[e + 1] = expert_offsets[e] + expert_counts[e];
  for (int r = 0; r < R; ++r) {
    rank_counts[r] = 0;
    for (int e = r * EL; e < (r + 1) * EL; ++e) rank_counts[r] += expert_counts[e];
  }
  rank_offsets[0] = 0;
  for (int r = 0; r < R; ++r) rank_offsets[r + 1] = rank_offsets[r] + rank_counts[r];

  int32_t* cursor = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int s = 0; s < S; ++s) row_to_slot[s] = -1;
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int s = t * k + j, e = ids[s];
      if (e < 0 || e >= E) { slot_to_row[s] = -1; continue; }
      int row = expert_offsets[e] + cursor[e]++;
      slot_to_row[s] = row;
      row_to_slot[row] = s;
    }
  }
  free(cursor);
  if (src_expert_counts) {
    memset(src_expert_counts, 0, sizeof(int32_t) * (size_t)R * E);
    for (int s = 0; s < S; ++s) {
      int e = ids[s];
      if (e < 0 || e >= E) continue;
      src_expert_counts[(size_t)oracle_src_rank(s / k, T, R) * E + e] += 1;
    }
  }
  return dropped;
}

/* ---------------------------------------------------------------- dispatch
 * [EPRT] "Send tokens ...": experts receive the token input vectors (not the
 * router scores).  x_disp[slot_to_row[s]] = x[s / k], a byte copy. */
void oracle_dispatch_rows(const void* x, size_t row_bytes, int T, int k,
                          const int32_t* slot_to_row, void* x_disp) {
  for (int s = 0; s < T * k; ++s) {
    if (slot_to_row[s] < 0) continue;
    memcpy((char*)x_disp + (size_t)slot_to_row[s] * row_bytes,
           (const char*)x + (size_t)(s / k) * row_bytes, row_bytes);
  }
}

/* --------------------------------------------------------------------- ffn
 * [EPRT] "Send tokens ...": an expert transforms each of its rows on its
 * own (rows are stacked only to batch the work).  [SWIGLU]:
 *   g = x . Wg_e,  u = x . Wu_e          (Wg_e, Wu_e: [H, I], row-major)
 *   a = SiLU(g) * u,  SiLU(z) = z / (1 + exp(-z))
 *   y = a . Wd_e                          (Wd_e: [I, H], row-major)
 * All sums in float64, ascending index.
 *
 * Computes n rows: row i has input x_rows[i*H ..] (dtype xdt), expert
 * row_expert[i]; w_gate[e], w_up[e], w_down[e] point at expert e's matrices
 * (dtype wdt; entries of unused experts may be NULL).  a_out (n x I, may be
 * NULL) receives the SwiGLU activations, y_out (n x H) the outputs.
 */
void oracle_ffn_rows(const void* x_rows, int xdt, const int32_t* row_expert, int n,
                     const void* const* w_gate, const void* const* w_up,
                     const void* const* w_down, int wdt, int H, int I,
                     double* a_out, double* y_out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n; ++i) {
    int e = row_expert[i];
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    double* g = (double*)calloc((size_t)I, sizeof(double));
    double* u = (double*)calloc((size_t)I, sizeof(double));
    double* y = y_out + (size_t)i * H;
    for (int h = 0; h < H; ++h) x[h] = orc_load(x_rows, xdt, (size_t)i * H + h);
    for (int h = 0; h < H; ++h) {
      for (int c = 0; c < I; ++c) {
        g[c] += x[h] * orc_load(w_gate[e], wdt, (size_t)h * I + c);
        u[c] += x[h] * orc_load(w_up[e], wdt, (size_t)h * I + c);
      }
    }
    for (int c = 0; c < I; ++c) {
      g[c] = g[c] / (1.0 + exp(-g[c])) * u[c];
      if (a_out) a_out[(size_t)i * I + c] = g[c];
    }
    for (int h = 0; h < H; ++h) y[h] = 0.0;
    for (int c = 0; c < I; ++c)
      for (int h = 0; h < H; ++h) y[h] += g[c] * orc_load(w_down[e], wdt, (size_t)c * H + h);
    free(x);
    free(g);
    free(u);
  }
}

/* ----------------------------------------------------------------- combine
 * [EPRT] "Send tokens ...": results return to their original tokens and
 * original order; "Return multiple ...": y(t) = sum_j w[t,j] * u_j, e.g.
 * y(A2) = 0.7 u0 + 0.3 u2.  Sum in float64 over j ascending.
 * y_disp holds float64 expert outputs indexed by row; slots with
 * slot_to_row < 0 contribute nothing. */
void oracle_combine(const double* y_disp, const float* topk_w, const int32_t* slot_to_row,
                    int T, int k, int H, double* y) {
  for (int t = 0; t < T; ++t) {
    double* out = y + (size_t)t * H;
    for (int h = 0; h < H; ++h) out[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      int row = slot_to_row[(size_t)t * k + j];
      if (row < 0) continue;
      double wj = (double)topk_w[(size_t)t * k + j];
      for (int h = 0; h < H; ++h) out[h] += wj * y_disp[(size_t)row * H + h];
    }
  }
}

/* ------------------------------------------------ masking: rank partials
 * [NEURON] "Collective Patterns / Prefill (CTE kernel)", steps 5-6, and "Why
 * a Single All-Reduce/Reduce-Scatter Works": in the masking form every rank
 * runs all T tokens against its own experts only, and a token none of whose
 * chosen experts sit on rank r gets zeros from r ("Tokens not routed to a
 * rank's experts produce zero output").  With rank r owning experts
 * [r*E/R, (r+1)*E/R) ("Limitations" 3-4), rank r's partial output is
 *   part[r][t] = sum over j (ascending) with ids[t*k+j] / (E/R) == r of
 *                w[t*k+j] * y_disp[slot_to_row[t*k+j]],
 * the expert output of each slot weighted by its affinity.  Slots with
 * slot_to_row < 0 (dropped) contribute nothing.  part is [R][T][H], float64.
 * Returns 0, or -1 for bad sizes. */
int oracle_rank_partials(const double* y_disp, const float* topk_w, const int32_t* ids,
                         const int32_t* slot_to_row, int T, int k, int H, int E, int R, double* part) {
  if (T < 0 || k < 1 || H < 1 || E < 1 || R < 1 || E % R != 0) return -1;
  const int EL = E / R;
  for (int r = 0; r < R; ++r) {
    for (int t = 0; t < T; ++t) {
      double* out = part + ((size_t)r * T + t) * H;
      for (int h = 0; h < H; ++h) out[h] = 0.0;
      for (int j = 0; j < k; ++j) {
        const int s = t * k + j, e = ids[s], row = slot_to_row[s];
        if (row < 0 || e < 0 || e >= E || e / EL != r) continue;
        const double affinity = (double)topk_w[s];
        for (int h = 0; h < H; ++h) out[h] += affinity * y_disp[(size_t)row * H + h];
      }
    }
  }
  return 0;
}

/* The reduction of the masking form (the reduce-scatter of "Collective
 * Patterns / Prefill", all-reduce in decode): y[t] = sum over r ascending of
 * part[r][t].  float64. */
void oracle_reduce_ranks(const double* part, int T, int H, int R, double* y) {
  for (int t = 0; t < T; ++t)
    for (int h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int r = 0; r < R; ++r) acc += part[((size_t)r * T + t) * H + h];
      y[(size_t)t * H + h] = acc;
    }
}

/* ------------------------------------------ expert-parallel exchange plan
 * [EPRT] "Send tokens to experts and return their results": each GPU routes
 * its own tokens and sends each token vector to the GPU that holds its
 * selected expert; destinations receive different counts (an exchange by
 * destination); results return to their source GPU and original token.
 * "Return multiple expert results to the same token": input delivery is
 * shared when two selected experts reside on the same GPU, and the source
 * forms the weighted sum of the token's results.  [NEURON] "Limitations"
 * 3-4: rank d holds experts [d*E/R, (d+1)*E/R).
 *
 * Plan of one source rank with T tokens (ids [T][k] global expert ids,
 * w [T][k] weights):
 *   J(t, d)        = the choices j (ascending) of token t with ids[t][j] on d;
 *   send_counts[d] = #{t : J(t, d) non-empty}: token t's row goes to d once;
 *   send rows are ordered by destination, then by token: send_offsets is the
 *   exclusive prefix sum of send_counts, and the row of (t, d) is
 *   send_offsets[d] + #{t' < t : J(t', d) non-empty};
 *   slot_send_row[t*k + j] = that row for d = ids[t][j] / (E/R) (-1 for an
 *   id outside [0, E));
 *   row_token[row]          = t;
 *   row_ids[row][i], row_w[row][i] (i < k): for the i-th choice j of J(t, d),
 *   the expert's local id ids[t][j] - d*E/R and the weight w[t][j]; -1 and 0
 *   past |J(t, d)|.
 * Arrays sized for T*k rows (the most there can be).  Returns the number of
 * send rows, or -1 for bad sizes. */
int oracle_ep_plan(const int32_t* ids, const float* w, int T, int k, int E, int R, int32_t* send_counts,
                   int32_t* send_offsets, int32_t* slot_send_row, int32_t* row_token, int32_t* row_ids,
                   float* row_w) {
  if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return -1;
  const int EL = E / R;
  for (int d = 0; d < R; ++d) {
    send_counts[d] = 0;
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j) {
        const int e = ids[(size_t)t * k + j];
        if (e >= 0 && e < E && e / EL == d) {
          send_counts[d] += 1;
          break;
        }
      }
  }
  send_offsets[0] = 0;
  for (int d = 0; d < R; ++d) send_offsets[d + 1] = send_offsets[d] + send_counts[d];
  for (int s = 0; s < T * k; ++s) slot_send_row[s] = -1;
  for (int d = 0; d < R; ++d) {
    int row = send_offsets[d];
    for (int t = 0; t < T; ++t) {
      int n = 0;
      for (int j = 0; j < k; ++j) {
        const int e = ids[(size_t)t * k + j];
        if (e < 0 || e >= E || e / EL != d) continue;
        row_ids[(size_t)row * k + n] = e - d * EL;
        row_w[(size_t)row * k + n] = w[(size_t)t * k + j];
        slot_send_row[(size_t)t * k + j] = row;
        n += 1;
      }
      if (n == 0) continue;
      for (int i = n; i < k; ++i) {
        row_ids[(size_t)row * k + i] = -1;
        row_w[(size_t)row * k + i] = 0.0f;
      }
      row_token[row] = t;
      row += 1;
    }
  }
  return send_offsets[R];
}

/* ----------------------------------------------------------------- EPLB
 * [WIKI] "工作机制" / "边界与常见误解" (third point): routing is dynamic, so
 * the per-expert token counts drift and a balancer redistributes hot and
 * cold experts over the GPUs; [NEURON] "Limitations" 3: the static layout
 * (rank r owns experts [r*E/R, (r+1)*E/R)) has no replication and no
 * dynamic balancing.  The pages give no algorithm; this is the plainest
 * reading, with every tie fixed so that results are exact integers:
 *
 *  plan (from measured per-expert loads, R ranks of `slots` physical expert
 *  slots each, P = R * slots >= E):
 *   1. every expert gets one replica; each of the P - E extra replicas goes
 *      to the expert with the largest load per replica, load[e] / n[e]
 *      (compared exactly as load[a] * n[b] vs load[b] * n[a]), ties to the
 *      lower expert id;
 *   2. replica j of expert e is given the share
 *      load[e] / n[e] + (j < load[e] % n[e]) (integer division: an even
 *      split of the expert's load);
 *   3. replicas are placed one by one in order of decreasing share (ties:
 *      lower expert id, then lower replica index), each on the rank with
 *      the least placed share that still has a free slot (ties: lower
 *      rank); it takes that rank's next slot, physical id rank*slots + i.
 *  Outputs: phys_to_logical[P]; replica_offsets[E+1] (prefix sums of n) and
 *  replicas[P] (physical ids of expert e's replicas j = 0..n[e]-1 at
 *  replica_offsets[e] + j).  Returns -1 if P < E or a size is < 1.
 *
 *  remap (per step): slot t*k+j with logical expert e goes to replica
 *  t mod n[e] of e (round robin over token indices); ids outside [0, E)
 *  map to -1.
 */
int oracle_eplb_plan(const int64_t* load, int E, int R, int slots, int32_t* phys_to_logical,
                     int32_t* replica_offsets, int32_t* replicas) {
  if (E < 1 || R < 1 || slots < 1) return -1;
  const int P = R * slots;
  if (P < E) return -1;
  int* n = (int*)malloc(sizeof(int) * (size_t)E);
  for (int e = 0; e < E; ++e) n[e] = 1;
  for (int extra = 0; extra < P - E; ++extra) {
    int best = 0;
    for (int e = 1; e < E; ++e)
      if (load[e] * (int64_t)n[best] > load[best] * (int64_t)n[e]) best = e;
    n[best] += 1;
  }
  replica_offsets[0] = 0;
  for (int e = 0; e < E; ++e) replica_offsets[e + 1] = replica_offsets[e] + n[e];
  /* the P replicas as (expert, index, share) */
  int* item_e = (int*)malloc(sizeof(int) * (size_t)P);
  int* item_j = (int*)malloc(sizeof(int) * (size_t)P);
  int64_t* share = (int64_t*)malloc(sizeof(int64_t) * (size_t)P);
  char* placed = (char*)calloc((size_t)P, 1);
  int m = 0;
  for (int e = 0; e < E; ++e)
    for (int j = 0; j < n[e]; ++j) {
      item_e[m] = e;
      item_j[m] = j;
      share[m] = load[e] / n[e] + (j < load[e] % n[e] ? 1 : 0);
      ++m;
    }
  int64_t* rank_load = (int64_t*)calloc((size_t)R, sizeof(int64_t));
  int* used = (int*)calloc((size_t)R, sizeof(int));
  for (int step = 0; step < P; ++step) {
    /* next: the unplaced item of largest share; items are listed by
       (expert, index) ascending, so the first maximum wins ties */
    int pick = -1;
    for (int i = 0; i < P; ++i)
      if (!placed[i] && (pick < 0 || share[i] > share[pick])) pick = i;
    placed[pick] = 1;
    int r_best = -1;
    for (int r = 0; r < R; ++r)
      if (used[r] < slots && (r_best < 0 || rank_load[r] < rank_load[r_best])) r_best = r;
    const int phys = r_best * slots + used[r_best];
    used[r_best] += 1;
    rank_load[r_best] += share[pick];
    phys_to_logical[phys] = item_e[pick];
    replicas[replica_offsets[item_e[pick]] + item_j[pick]] = phys;
  }
  free(n);
  free(item_e);
  free(item_j);
  free(share);
  free(placed);
  free(rank_load);
  free(used);
  return 0;
}

void oracle_eplb_remap(const int32_t* ids, int T, int k, int E, const int32_t* replica_offsets,
                       const int32_t* replicas, int32_t* phys_ids) {
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      int out = -1;
      if (e >= 0 && e < E) {
        const int n = replica_offsets[e + 1] - replica_offsets[e];
        out = replicas[replica_offsets[e] + t % n];
      }
      phys_ids[(size_t)t * k + j] = out;
    }
}
