/*
 * moe_b200.h -- C ABI of the MoE expert-parallel token round trip on one
 * NVIDIA B200 (sm_100a).
 *
 * One MoE layer's token round trip, as four calls:
 *
 *   moe_route      logits -> top-k expert ids + softmax-over-top-k weights
 *   moe_dispatch   expert histogram, exclusive scan, stable scatter of token
 *                  rows into an expert-contiguous (= rank-major) buffer,
 *                  per-expert / per-rank / per-(source rank, expert) counts
 *   moe_expert_ffn grouped SwiGLU expert MLP over the ragged expert segments
 *                  (also callable as its two halves, moe_ffn_gate_up and
 *                  moe_ffn_down)
 *   moe_combine    gather each token's k expert outputs, weight them by the
 *                  router weights, sum, and write them in original token order
 *
 * and, beside them: moe_router_topk (router affinities on tensor cores fused
 * with the top-k), an index-only moe_dispatch with moe_ffn_gate_up_gather /
 * moe_expert_ffn_gather (the row scatter fused into the gate/up projection),
 * moe_eplb_plan / moe_eplb_remap / moe_eplb_replicate (replicas of hot
 * experts placed over the logical ranks), and moe_combine_rank_partials /
 * moe_reduce_rank_partials (the masking form: per-rank partial outputs and
 * their rank-ordered sum), and moe_ep_* (the exchange of rows between ranks
 * for expert parallelism over several GPUs).
 *
 * Sources (page title, section):
 *  [EPRT]   "EP: Partition Experts and Route Tokens": "Send tokens to experts
 *           and return their results" (route, dispatch, per-expert batched
 *           MLP, return in original order), "Return multiple expert results
 *           to the same token" (Top-2 weighted sum), "Equal expert counts can
 *           receive different token counts" (unequal per-expert/per-rank
 *           counts).
 *  [NEURON] "Expert Parallelism (EP)" (vLLM on Neuron): "Weight Layout Across
 *           Ranks" and "Limitations" 1, 3, 4 (E divisible by the EP degree;
 *           rank r owns experts [r*E/R, (r+1)*E/R), contiguous placement);
 *           "Router Weights" (every rank scores all E experts).
 *  [SWIGLU] Shazeer, "GLU Variants Improve Transformer" (2020): the expert
 *           MLP y = (SiLU(x Wg) * (x Wu)) Wd.
 *
 * Conventions for every call:
 *  - T tokens, H hidden, I intermediate, E experts, k experts per token
 *    (1 <= k <= min(E, 8)), R logical EP ranks (E % R == 0), S = T*k slots.
 *    Slot s = t*k + j is token t's j-th choice.
 *  - All array arguments are DEVICE pointers owned by the caller, row-major,
 *    except where a call says HOST (moe_eplb_plan's arrays, the
 *    phys_to_logical table of moe_eplb_replicate, moe_ep_plan_host's and
 *    moe_ep_exchange_offsets' arrays, moe_ep_pack's per-destination pointer
 *    tables); activation and weight
 *    buffers (and the workspace) 16-byte aligned, int32/float32 index and
 *    weight arrays 4-byte aligned.  The library never allocates, frees or
 *    copies to the host, and never synchronises, except moe_get_error.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously on it.
 *  - Invalid arguments are rejected on the host before anything is enqueued
 *    (MOE_ERR_INVALID_ARG; moe_last_error_message() names the argument).
 *    A failed launch returns MOE_ERR_CUDA.
 *  - Data-dependent problems found on the device (an expert id outside
 *    [0, E), inconsistent expert offsets, a row index out of range, a
 *    bounded wait that ran out) never fault: the offending item is skipped,
 *    a bit is set in a per-device error word, and moe_get_error() reports it.
 *  - dtype is MOE_F32 (float32) or MOE_BF16 (bfloat16) for activations and
 *    expert weights; logits and combination weights are always float32;
 *    all accumulation is float32.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* rejected on the host, nothing enqueued */
  MOE_ERR_UNSUPPORTED = 2, /* valid request the library does not implement */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE = 4,      /* the device flagged bad data (see moe_get_error) */
  MOE_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out */
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Version of this ABI (bumped on any signature change). */
int moe_abi_version(void);

/* Static text for a status code. */
const char* moe_status_string(int status);

/* Text describing the last non-OK status returned on this host thread. */
const char* moe_last_error_message(void);

/*
 * moe_route -- [EPRT] "Send tokens ...": each token picks its experts from
 * all E scores; "Return multiple ...": the combination weights are kept apart
 * from the choice.  Weight rule: softmax over the k selected logits (k = 1
 * gives exactly 1.0).
 *   logits   [T, E] float32 (router affinities, finite)
 *   topk_ids [T, k] int32   out: experts by logit descending; equal logits
 *                                (-0 == +0) put the lower id first
 *   topk_w   [T, k] float32 out: exp(l_j - l_0) / sum_i exp(l_i - l_0)
 * Constraints: T >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 8).
 */
moe_status moe_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                     void* stream);

/*
 * moe_router_topk -- [NEURON] "Router Weights": every token is scored against
 * all E experts, logits = x W_r^T (+ bias); then exactly moe_route on those
 * logits.  The affinity matrix runs on tensor cores: bf16 products summed in
 * float32 (order of the tensor-core accumulation), plus the bias in float32.
 *   x        [T, H] bf16          token activations
 *   w_router [E, H] bf16          row e = expert e's router vector
 *   bias     [E] float32 or NULL  added to every token's logits
 *   logits   [T, E] float32 or NULL  out (optional): the affinities used
 *   topk_ids [T, k] int32, topk_w [T, k] float32  out: as moe_route, and
 *            bit-identical to moe_route applied to the logits written here
 * Constraints: T >= 0, 1 <= E <= 256, 1 <= k <= min(E, 8), H a positive
 * multiple of 8; x, w_router 16-byte aligned.
 */
moe_status moe_router_topk(const void* x, const void* w_router, const float* bias, int T, int H, int E, int k,
                           float* logits, int32_t* topk_ids, float* topk_w, void* stream);

/*
 * Bytes of device workspace moe_dispatch needs for these sizes.  The
 * workspace must be zero-filled once before its first use; every call leaves
 * it ready for the next, a call whose grid barrier timed out included (the
 * last of its CTAs to finish zeroes the barrier's counters).  Calls sharing a
 * workspace must not overlap.
 */
size_t moe_dispatch_workspace_bytes(int T, int k, int E, int R);

/*
 * moe_dispatch -- [EPRT] "Send tokens ...": dispatch groups token vectors by
 * selected expert and tracks each row's source token; [NEURON] "Limitations"
 * 3-4: rank r owns experts [r*E/R, (r+1)*E/R), so expert-major order is also
 * rank-major, the layout of an all-to-all send buffer.
 *   x                 [T, H] dtype     token rows
 *   topk_ids          [T, k] int32     from moe_route
 *   x_disp            [S, H] dtype     out: x_disp[slot_to_row[s]] = x[s / k]
 *   expert_counts     [E]     int32    out: rows per expert
 *   expert_offsets    [E + 1] int32    out: exclusive prefix sum of counts
 *   rank_counts       [R]     int32    out: rows per logical rank
 *   rank_offsets      [R + 1] int32    out: exclusive prefix sum
 *   slot_to_row       [S]     int32    out: row of slot s (-1 if dropped)
 *   row_to_slot       [S]     int32    out: inverse (-1 past the last row)
 *   src_expert_counts [R, E]  int32    out (may be NULL): rows of expert e
 *                                      whose token comes from source rank r;
 *                                      token t's source rank is t*R/T
 *                                      (contiguous, as-equal-as-possible
 *                                      ranges: the all-to-all send splits)
 *   workspace / workspace_bytes        scratch from moe_dispatch_workspace_bytes
 * Rows are ordered by (expert, token): stable in token order within each
 * expert.  Slots with an id outside [0, E) are dropped (not counted,
 * slot_to_row = -1) and flagged in the device error word.
 * Index-only dispatch: x and x_disp both NULL computes every output but
 * x_disp (the counts, offsets and permutation) and moves no rows; the gate/up
 * projection then gathers the rows itself (moe_ffn_gate_up_gather).  Exactly
 * one of them NULL is MOE_ERR_INVALID_ARG.
 * Constraints: H * sizeof(dtype) % 16 == 0, E % R == 0, E <= 1024,
 * 1 <= k <= min(E, 8), S < 2^31.
 */
moe_status moe_dispatch(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                        void* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                        int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                        int32_t* src_expert_counts, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_route_count + moe_dispatch_counted -- moe_route and moe_dispatch with
 * the dispatch's counting moved into the routing kernel.  The router already
 * holds each token's choices; counting them there (per chunk of slots: the
 * experts' counts and each slot's stable rank among the chunk's slots of its
 * expert, into the dispatch workspace) leaves the dispatch kernel only the
 * scan of the chunk counts, the permutation and the row copy, with no grid
 * barrier before its copy when the count table is small (chunks x E <= 8192).
 *
 * The pair counts in chunks of at most 128 slots (moe_dispatch: 512), so the
 * routing kernel has a CTA per chunk and a warp per token.
 *
 * moe_route_count: exactly moe_route (same ids and weights, bit for bit),
 * plus that counting into `workspace` (moe_route_count_workspace_bytes(T, k,
 * E, R) bytes, zero-filled once, as moe_dispatch's).  Ids outside [0, E)
 * cannot arise from finite logits.
 * moe_dispatch_counted: moe_dispatch's arguments and results (its workspace
 * sized by moe_route_count_workspace_bytes), for the topk_ids that
 * moe_route_count last wrote with this workspace and the same T, k, E, R (it
 * may be called again on them: the counting is kept).
 * Counts that do not belong to the ids given never move a row outside its
 * expert's segment: such slots are dropped and flagged (bit 2).
 */
size_t moe_route_count_workspace_bytes(int T, int k, int E, int R);
moe_status moe_route_count(const float* logits, int T, int E, int k, int R, int32_t* topk_ids, float* topk_w,
                           void* workspace, size_t workspace_bytes, void* stream);
moe_status moe_dispatch_counted(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                                void* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                                int32_t* src_expert_counts, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_dispatch_noalloc -- moe_dispatch for callers that cannot allocate.
 * (The pages have no counterpart: this is a deployment variant of this
 * library's dispatch.)
 *
 * Same arguments and results as moe_dispatch, without the workspace: some
 * callers have no way to pass one in and may not call cudaMalloc where they
 * call us (a host framework that owns all device memory, or a hot path that
 * must not take cudaMalloc's implicit synchronisation).  The scratch lives in
 * a fixed array of MOE_DISPATCH_NOALLOC_SCRATCH_BYTES bytes inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  This call allocates nothing and frees nothing.
 *  - Sizes whose moe_dispatch_workspace_bytes(T, k, E, R) exceeds the
 *    maximum are rejected with MOE_ERR_INVALID_ARG (use moe_dispatch then).
 *  - The first call in a CUDA context (a device's primary context, or another
 *    context current at the call) looks up the array's device address there
 *    with cudaGetSymbolAddress; make that first call before any stream
 *    capture.  Later calls in the same context reuse the address.  A new
 *    context (for instance the primary context recreated after
 *    cudaDeviceReset) has a new id and gets a new lookup, so an address from
 *    a destroyed context is never reused.
 *  - A rejected call (MOE_ERR_INVALID_ARG) enqueues nothing and leaves the
 *    array untouched.
 *  - Every call on a device shares the one array and finds it as the last
 *    call left it; the call clears the part that must start at zero.  Calls
 *    that overlap on the GPU (other streams, other host threads) race on it:
 *    serialise them.
 */
#define MOE_DISPATCH_NOALLOC_SCRATCH_BYTES (2u << 20)
moe_status moe_dispatch_noalloc(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E,
                                int R, void* x_disp, int32_t* expert_counts, int32_t* expert_offsets,
                                int32_t* rank_counts, int32_t* rank_offsets, int32_t* slot_to_row,
                                int32_t* row_to_slot, int32_t* src_expert_counts, void* stream);

/*
 * moe_expert_ffn -- [EPRT] "Send tokens ...": each expert's rows are stacked
 * and multiplied by that expert's weights, with no mixing across rows;
 * [SWIGLU]:  h = SiLU(x_disp Wg_e) * (x_disp Wu_e),  y_disp = h Wd_e
 * for every row in expert e's segment [expert_offsets[e], expert_offsets[e+1]).
 *   x_disp         [S, H] dtype
 *   w_gate, w_up   [E, H, I] dtype     (expert e's [H, I] matrix at e*H*I)
 *   w_down         [E, I, H] dtype
 *   expert_offsets [E + 1] int32       from moe_dispatch (read on the device)
 *   h              [S, I] dtype        out: SwiGLU activations (rounded to
 *                                      dtype), the intermediate of the pair
 *   y_disp         [S, H] dtype        out: expert outputs
 * Rows outside [expert_offsets[0], expert_offsets[E]) are not written.
 * bf16 runs on tcgen05 tensor cores (float32 accumulate in TMEM), float32 on
 * CUDA cores.  Constraints: H % 8 == 0, I % 8 == 0 (bf16); H % 4, I % 4 (f32).
 */
moe_status moe_expert_ffn(const void* x_disp, int dtype, const void* w_gate, const void* w_up,
                          const void* w_down, const int32_t* expert_offsets, int E, int H, int I, int S, void* h,
                          void* y_disp, void* stream);

/*
 * Tile shape of the bf16 expert FFN (moe_expert_ffn, moe_ffn_gate_up,
 * moe_ffn_down and their _gather forms).  One setting for the whole process,
 * read at each call.
 *   MOE_FFN_TILING_AUTO    per projection: pair tiles when S >= 448 * E for
 *                          gate/up and S >= 384 * E for down (enough rows per
 *                          expert that padding each expert to 256 rows costs
 *                          little), else single tiles.  The default.
 *   MOE_FFN_TILING_SINGLE  128-row tiles, one SM per tile.
 *   MOE_FFN_TILING_PAIR    256-row tiles computed by a cluster of two SMs
 *                          (tcgen05 cta_group::2; each SM loads half of the
 *                          weight tile); an expert's last tile with at most
 *                          128 rows left uses an M = 128 pair MMA.
 * Both shapes form the same products and accumulate them in float32 in the
 * same K order.  float32 calls ignore the setting.
 * moe_set_ffn_tiling returns MOE_ERR_INVALID_ARG for any other mode and keeps
 * the old one.  moe_ffn_tiling_for returns the shape (SINGLE or PAIR) that a
 * bf16 call of `projection` (MOE_FFN_GATE_UP or MOE_FFN_DOWN) with E experts
 * and S rows would use now, or -1 for E <= 0, S < 0 or another projection.
 */
#define MOE_FFN_TILING_AUTO 0
#define MOE_FFN_TILING_SINGLE 1
#define MOE_FFN_TILING_PAIR 2
#define MOE_FFN_GATE_UP 0
#define MOE_FFN_DOWN 1
moe_status moe_set_ffn_tiling(int mode);
int moe_get_ffn_tiling(void);
int moe_ffn_tiling_for(int E, int S, int projection);

/* First half of moe_expert_ffn: h = SiLU(x_disp Wg_e) * (x_disp Wu_e). */
moe_status moe_ffn_gate_up(const void* x_disp, int dtype, const void* w_gate, const void* w_up,
                           const int32_t* expert_offsets, int E, int H, int I, int S, void* h, void* stream);

/* Second half of moe_expert_ffn: y_disp = h Wd_e. */
moe_status moe_ffn_down(const void* h, int dtype, const void* w_down, const int32_t* expert_offsets, int E, int H,
                        int I, int S, void* y_disp, void* stream);

/*
 * moe_ffn_down_combine + moe_combine_finalize -- moe_ffn_down fused with
 * moe_combine ([EPRT] "Send tokens ...": results return to their source
 * tokens; "Return multiple ...": y(t) = sum_j w_j u_j): the down projection's
 * epilogue multiplies each row's output by its slot's weight and adds it into
 * a float32 accumulator by token, so y_disp is never written or read.
 *   row_to_slot [S] int32, topk_w [T, k] float32   from moe_dispatch / moe_route
 *   y_acc       [T, H] float32: zero on entry to the first call (the finalize
 *               leaves it zero again); gets  sum_j w[t][j] * (h Wd)[row of t*k+j]
 * moe_combine_finalize: y[t] = y_acc[t] rounded to bf16, then y_acc = 0.
 * The additions are float32 atomics (red.global.add.v4.f32): their order,
 * hence the last bits of y, is not fixed from run to run (moe_combine sums in
 * j order).  Single-CTA tiles whatever the tiling setting; bf16 only
 * (MOE_ERR_UNSUPPORTED otherwise).  A row whose slot is outside [0, T*k) is
 * skipped and flagged (bit 4).  Pays where the accumulator stays in L2 (few
 * tokens, e.g. decode); elsewhere its T*H*4 bytes of reductions cost more than
 * the combine they replace.
 */
moe_status moe_ffn_down_combine(const void* h, int dtype, const void* w_down, const int32_t* expert_offsets, int E,
                                int H, int I, int S, const int32_t* row_to_slot, const float* topk_w, int T, int k,
                                float* y_acc, void* stream);
moe_status moe_combine_finalize(float* y_acc, int dtype, int T, int H, void* y, void* stream);

/*
 * moe_ffn_gate_up_gather -- moe_ffn_gate_up fused with the row scatter of
 * moe_dispatch ([EPRT] "Send tokens ...": a dispatched row is a copy of its
 * token's row): the A operand of dispatched row r is read straight from x,
 *   h[r] = SiLU(x[row_to_slot[r] / k] Wg_e) * (x[row_to_slot[r] / k] Wu_e),
 * so x_disp is never written or read.  bf16: 128 extra threads per CTA copy
 * each k-block's token rows into the swizzled A tile with 16-byte cp.async
 * (the weights still arrive by TMA); float32 indexes x on CUDA cores.
 * Measured against moe_dispatch + moe_ffn_gate_up: faster end to end where
 * the FFN streams weights (few rows per expert), slower (~10% on the gate/up
 * projection) where it is tensor-bound.
 *   x              [T, H] dtype        token rows (moe_dispatch's x)
 *   row_to_slot    [S] int32           from moe_dispatch (index-only is enough)
 *   k              top-k of the routing (slot s belongs to token s / k)
 *   the rest as moe_ffn_gate_up; S <= T * k.
 * The result equals moe_ffn_gate_up on the x_disp that moe_dispatch writes,
 * bit for bit (same products, same K order, same tile shape).  A row whose
 * slot is outside [0, T * k) reads token 0 and is flagged (bit 4).
 */
moe_status moe_ffn_gate_up_gather(const void* x, int dtype, int T, const int32_t* row_to_slot, int k,
                                  const void* w_gate, const void* w_up, const int32_t* expert_offsets, int E, int H,
                                  int I, int S, void* h, void* stream);

/* moe_expert_ffn with the gathering gate/up projection: moe_ffn_gate_up_gather, then moe_ffn_down. */
moe_status moe_expert_ffn_gather(const void* x, int dtype, int T, const int32_t* row_to_slot, int k,
                                 const void* w_gate, const void* w_up, const void* w_down,
                                 const int32_t* expert_offsets, int E, int H, int I, int S, void* h, void* y_disp,
                                 void* stream);

/*
 * moe_combine -- [EPRT] "Send tokens ...": results return to their source
 * tokens in original order; "Return multiple ...": y(t) = sum_j w_j u_j.
 *   y_disp      [S, H] dtype
 *   topk_w      [T, k] float32
 *   slot_to_row [S] int32              from moe_dispatch
 *   y           [T, H] dtype           out: float32 sum over j = 0..k-1 in
 *                                      order, rounded once to dtype
 * A slot whose row is outside [0, S) contributes nothing and is flagged.
 */
moe_status moe_combine(const void* y_disp, int dtype, const float* topk_w, const int32_t* slot_to_row, int T, int k,
                       int H, void* y, void* stream);

/*
 * The masking form of expert parallelism -- [NEURON] "Collective Patterns /
 * Prefill (CTE kernel)" steps 5-6 and "Why a Single All-Reduce/Reduce-Scatter
 * Works": every rank runs all tokens against its own experts only, tokens not
 * routed to them get zeros from it, and a reduce-scatter (prefill) or
 * all-reduce (decode) sums the ranks' partial outputs.  One GPU holds the R
 * logical ranks' partials as R planes of one buffer.
 *
 * moe_combine_rank_partials: for every rank r and token t,
 *   y_part[r][t] = sum over j with topk_ids[t][j] / (E / R) == r of
 *                  topk_w[t][j] * y_disp[slot_to_row[t*k + j]]
 * (float32, j ascending, rounded once to dtype; zero where rank r owns none
 * of the token's experts).
 *   y_disp      [S, H] dtype     expert outputs (moe_expert_ffn)
 *   topk_w      [T, k] float32, topk_ids [T, k] int32   (moe_route)
 *   slot_to_row [S] int32        (moe_dispatch; -1 = dropped slot, skipped)
 *   y_part      [R, T, H] dtype  out
 * A slot whose row is outside [0, S), or whose id is outside [0, E) with a
 * row other than -1, contributes nothing and is flagged (bit 4).
 *
 * moe_reduce_rank_partials: y[t] = sum over r = 0 .. R-1 of y_part[r][t]
 * (float32, rank order, rounded once to dtype).
 *   y_part [R, T, H] dtype, y [T, H] dtype out.
 * Constraints: H * sizeof(dtype) % 16 == 0; 1 <= k <= 8; E % R == 0,
 * E <= 1024 (R <= 1024 for the reduction).
 */
moe_status moe_combine_rank_partials(const void* y_disp, int dtype, const float* topk_w, const int32_t* topk_ids,
                                    const int32_t* slot_to_row, int T, int k, int H, int E, int R, void* y_part,
                                    void* stream);
moe_status moe_reduce_rank_partials(const void* y_part, int dtype, int T, int H, int R, void* y, void* stream);

/*
 * Expert-parallel exchange between ranks -- [EPRT] "Send tokens ...": each
 * GPU routes its own tokens and sends each token vector to the GPU holding
 * its selected expert (an exchange by destination with unequal counts);
 * results return to the source GPU and token, which forms the weighted sum.
 * "Return multiple ...": input delivery is shared when two selected experts
 * sit on the same GPU.  [NEURON] "Limitations" 3-4: rank d holds experts
 * [d*E/R, (d+1)*E/R) (EL = E/R local experts).
 *
 * One layer over R ranks (R <= 64), every rank a source and a destination:
 *   source s:  moe_route; moe_ep_plan; (counts exchange: every rank gets all
 *              R send_counts vectors); moe_ep_exchange_offsets; moe_ep_pack
 *              into the destinations' receive buffers (peer memory), or into
 *              a local buffer for a staged all-to-all;
 *   (all ranks: barrier, or the all-to-all itself)
 *   destination d: moe_ep_recv_index over its received rows; the gathering
 *              gate/up projection (moe_ffn_gate_up_gather with x = received
 *              rows, row_to_slot from moe_ep_recv_index, k) and moe_ffn_down
 *              with its EL local experts' weights; moe_combine(y_gemm,
 *              recv_w, slot_to_row, T_recv, k) gives one partial per received
 *              row (the weighted sum over the row's local experts); the
 *              partials of source s (rows [recv_base[s], recv_base[s+1]))
 *              return to s's return buffer at ret_base[s];
 *   (barrier)
 *   source s:  moe_combine(y_ret, ones [T, k], ret_row, T, k) sums each
 *              token's partials: its output.
 * The library moves no rows between GPUs by itself except through the peer
 * pointers given to moe_ep_pack; barriers and the counts exchange belong to
 * the caller (NCCL, or a host process group).
 *
 * moe_ep_plan (device) / moe_ep_plan_host (HOST arrays, no device work): the
 * send plan of one source rank with T tokens.  One send row per (token t,
 * destination d holding any of t's experts), ordered by d, then t:
 *   topk_ids, topk_w [T, k]  from moe_route (global expert ids)
 *   send_counts  [R]         out: rows for each destination
 *   send_offsets [R + 1]     out: exclusive prefix sum of send_counts
 *   slot_send_row [T * k]    out: send row of slot t*k+j's (t, d) pair
 *   ret_row      [T * k]     out: that row for the first choice of t on each
 *                            destination, -1 for its other choices there (so
 *                            a token's partials are each summed once)
 *   row_token    [T * min(k, R)] out: token of each send row
 *   row_ids      [T * min(k, R), k] out: the token's local expert ids on the
 *                            row's destination (id - d*EL), in top-k order,
 *                            -1 past the last
 *   row_w        [T * min(k, R), k] float32 out: their weights, 0 past the last
 *   workspace    moe_ep_plan_workspace_bytes(T, R) bytes (no zeroing needed)
 * Ids outside [0, E) are dropped (their slots' rows are -1) and flagged
 * (device: bit 1 of the error word; host: MOE_ERR_DEVICE).  Two kernels.
 *
 * moe_ep_exchange_offsets (HOST arrays): from counts [R][R] (row s = source
 * s's send_counts) for rank `rank`:
 *   dst_base[d]  = sum_{s < rank} counts[s][d]  (where rank's rows start in
 *                  d's receive buffer)
 *   recv_base[s] = sum_{s' < s} counts[s'][rank]  ([R + 1]; recv_base[R]
 *                  rows are received)
 *   ret_base[s]  = sum_{d < rank} counts[s][d]  (where rank's partials for
 *                  source s go in s's return buffer)
 *
 * moe_ep_pack: every send row r of destination d goes to
 *   dst_x[d]   row dst_base[d] + r - send_offsets[d]  (x[row_token[r]])
 *   dst_ids[d], dst_w[d] at the same row: row_ids[r], row_w[r]
 * dst_x, dst_ids, dst_w, dst_cap are HOST arrays of R entries (device
 * pointers, possibly peers' memory; dst_cap[d] rows each); dst_base is a
 * DEVICE array [R] (moe_ep_exchange_offsets' dst_base, or send_offsets for a
 * local staging buffer).  A destination row beyond dst_cap[d] is skipped and
 * flagged (bit 4).  16-byte vector copies, a warp per (row, column slice).
 *
 * moe_ep_recv_index: the received rows' counting sort by local expert:
 *   recv_ids       [T_recv, k]  received row_ids (-1 = padding, never
 *                               flagged; rows past the received count must
 *                               be all -1); k may exceed EL (a row holds at
 *                               most min(k, EL) local ids)
 *   expert_counts  [EL], expert_offsets [EL + 1]  out
 *   slot_to_row    [T_recv * k] out: GEMM row of (received row q, choice i),
 *                               -1 for padding
 *   row_to_slot    [T_recv * k] out: q*k + i of each GEMM row
 *   workspace      moe_dispatch_workspace_bytes(T_recv, k, EL, 1) bytes,
 *                  zero-filled once (as moe_dispatch's)
 * GEMM rows are ordered by (local expert, received row): stable.
 *
 * moe_enable_peer_access (host; enqueues nothing): lets kernels launched on
 * the CURRENT device load and store memory that lives on device peer_device
 * (a peer's receive buffers given to moe_ep_pack), i.e.
 * cudaDeviceEnablePeerAccess from the current device.  peer_device equal to
 * the current device, or access already enabled, is MOE_OK; a pair of
 * devices without peer capability is MOE_ERR_UNSUPPORTED; peer_device < 0 or
 * not below the device count is MOE_ERR_INVALID_ARG.
 */
size_t moe_ep_plan_workspace_bytes(int T, int R);
moe_status moe_ep_plan(const int32_t* topk_ids, const float* topk_w, int T, int k, int E, int R,
                       int32_t* send_counts, int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row,
                       int32_t* row_token, int32_t* row_ids, float* row_w, void* workspace, size_t workspace_bytes,
                       void* stream);
moe_status moe_ep_plan_host(const int32_t* topk_ids, const float* topk_w, int T, int k, int E, int R,
                            int32_t* send_counts, int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row,
                            int32_t* row_token, int32_t* row_ids, float* row_w);
moe_status moe_ep_exchange_offsets(const int32_t* counts, int R, int rank, int32_t* dst_base, int32_t* recv_base,
                                   int32_t* ret_base);
moe_status moe_ep_pack(const void* x, int dtype, int T, int H, int k, int R, const int32_t* send_offsets,
                       const int32_t* dst_base, const int32_t* row_token, const int32_t* row_ids, const float* row_w,
                       void* const* dst_x, int32_t* const* dst_ids, float* const* dst_w, const int32_t* dst_cap,
                       void* stream);
moe_status moe_ep_recv_index(const int32_t* recv_ids, int T_recv, int k, int EL, int32_t* expert_counts,
                             int32_t* expert_offsets, int32_t* slot_to_row, int32_t* row_to_slot, void* workspace,
                             size_t workspace_bytes, void* stream);
moe_status moe_enable_peer_access(int peer_device);

/*
 * Expert placement with replicas -- an expert-parallel load balancer:
 * "什么是专家并行（Expert Parallelism）？", "工作机制" and "边界与常见误解"
 * (third point): routing is dynamic, so a balancer redistributes hot and cold
 * experts over the GPUs to keep their utilisation balanced ("Expert
 * Parallelism (EP)", "Limitations" 3: the static layout has neither).
 *
 * moe_eplb_plan (HOST arrays, runs on the CPU, no device work): from
 * measured per-expert loads (e.g. expert_counts of earlier steps) place
 * P = R * slots_per_rank physical experts, rank r holding physical ids
 * [r * slots_per_rank, (r + 1) * slots_per_rank):
 *   1. every expert gets one replica; each extra slot goes to the expert
 *      with the largest load per replica (load[a] * n[b] vs load[b] * n[a]),
 *      ties to the lower id;
 *   2. replica j of expert e carries the share load[e] / n[e] +
 *      (j < load[e] % n[e]);
 *   3. largest share first (ties: lower expert, lower replica), each replica
 *      takes the next slot of the rank with the least placed share that has
 *      a free slot (ties: lower rank).
 *   load            [E] int64, each in [0, 2^40)
 *   phys_to_logical [P] int32 out: expert whose weights physical id p holds
 *   replica_offsets [E + 1] int32 out: prefix sums of the replica counts
 *   replicas        [P] int32 out: physical ids of expert e's replicas at
 *                   replica_offsets[e] + j, j = 0 .. n_e - 1
 * Needs E, R, slots_per_rank >= 1 and E <= P <= 2^20, else
 * MOE_ERR_INVALID_ARG.  The result is an exact function of the inputs.
 *
 * moe_eplb_remap (device): phys_ids[t*k + j] = replicas[replica_offsets[e] +
 * t mod n_e] for e = topk_ids[t*k + j] (a token's slots go round robin over
 * the expert's replicas).  Ids outside [0, E) give -1 and set bit 1 of the
 * error word; inconsistent replica tables give -1 and set bit 2.  Feed
 * phys_ids to moe_dispatch with P experts and R ranks: the per-rank counts
 * are then those of the plan.
 *
 * moe_eplb_replicate (device copies, phys_to_logical is a HOST array): the
 * weights of the P physical experts, w_phys[p] = w[phys_to_logical[p]], each
 * expert_bytes long (one cudaMemcpyAsync each).  A replica holds its
 * expert's weights, so the round trip over the physical experts gives the
 * same outputs, bit for bit, as the one over the logical experts.
 */
moe_status moe_eplb_plan(const int64_t* load, int E, int R, int slots_per_rank, int32_t* phys_to_logical,
                         int32_t* replica_offsets, int32_t* replicas);
moe_status moe_eplb_remap(const int32_t* topk_ids, int T, int k, int E, const int32_t* replica_offsets,
                          const int32_t* replicas, int P, int32_t* phys_ids, void* stream);
moe_status moe_eplb_replicate(const void* w, size_t expert_bytes, int E, const int32_t* phys_to_logical, int P,
                              void* w_phys, void* stream);

/*
 * Synchronise `stream`, then read and clear the current device's error word.
 * Returns MOE_OK, MOE_ERR_DEVICE (bad ids/offsets/rows were skipped),
 * MOE_ERR_TIMEOUT (a bounded wait ran out; outputs of that call are
 * incomplete) or MOE_ERR_CUDA.  `*bits_out` (may be NULL) receives the raw
 * word: 1 bad expert id, 2 bad expert offsets, 4 bad combine row, 8 timeout.
 */
moe_status moe_get_error(void* stream, uint32_t* bits_out);

/*
 * Self-test of the device-side bounded waits (no counterpart on the pages:
 * failure detection of this library).  Enqueues one kernel whose single
 * waiting thread waits on a barrier that nothing completes; after limit_us
 * microseconds (1 .. 1e6) the wait gives up, sets the timeout bit and the
 * kernel returns, leaving the context usable.  A following moe_get_error()
 * returns MOE_ERR_TIMEOUT.
 */
moe_status moe_selftest_wait_timeout(unsigned int limit_us, void* stream);

/*
 * Self-test of moe_dispatch's recovery from a grid-barrier timeout (no
 * counterpart on the pages: failure detection of this library).  Same
 * arguments as moe_dispatch (T >= 1), plus limit_us (1 .. 1e6) for each
 * grid-barrier wait.  It presets the workspace's barrier arrival count to a
 * value no arrival sequence completes, then launches the dispatch kernel:
 * every CTA's first barrier wait runs out after limit_us, the timeout bit is
 * set, the outputs of this call are incomplete, and the kernel's exit
 * restores the workspace.  A following moe_get_error() returns
 * MOE_ERR_TIMEOUT, and a following moe_dispatch on the same workspace gives
 * complete, correct results.
 */
moe_status moe_selftest_dispatch_timeout(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k,
                                         int E, int R, void* x_disp, int32_t* expert_counts,
                                         int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets,
                                         int32_t* slot_to_row, int32_t* row_to_slot, int32_t* src_expert_counts,
                                         void* workspace, size_t workspace_bytes, unsigned int limit_us,
                                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
