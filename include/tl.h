/*
 * tl.h -- C ABI of libtl.so: per-lane-depth decode of a weight-shared looped
 * transformer on NVIDIA B200 (sm_100a).
 *
 * The model ("Benchmark Comparison" (vs generic runtimes), "Where Generic
 * Runtimes Lose On Looped Checkpoints"):
 *     embed -> pre blocks -> shared loop block x L -> head
 * L is a runtime argument over the same weights ("Dynamic-L Inference", "The
 * Core Idea"); each lane of a batch has its own L ("Dynamic-L Inference",
 * "L-Aware Batching").  Every pre block and every (loop iteration, body layer)
 * keeps its own K/V cache ("Benchmark Comparison" (measured benchmarks),
 * section 9, storage for "2 pre + 8 loop" blocks).  Lanes advance one loop
 * iteration per step, each at its own iteration index, and the exit decision of
 * a step is taken on the device before the next step is formed ("Depth-adaptive
 * Inference of Looped Language Models via Continuous Depth Batching", CDB
 * design).  Early exit on the relative L2 change of the hidden state and the
 * monotonic L clamp follow "CLI Reference", "generate" options
 * --early-exit-patience / -min-L / -tau / -peek-every.
 *
 * Block (per layer): a = RMSNorm(x; g1); [q|k|v] = a Wqkv^T; RoPE(q, k, pos);
 * o = causal softmax(q k^T / sqrt(hd)) v over the layer's cache slot;
 * x += o Wo^T; b = RMSNorm(x; g2); x += (silu(b Wg^T) * (b Wu^T)) Wd^T.
 * Head: logits = RMSNorm(h; g_final) Whead^T; greedy token = argmax (lowest id
 * on ties).  RoPE pairs (i, i + hd/2) with angle pos * base^(-2i/hd).
 *
 * Conventions for every call:
 *   - Return value: TL_OK (0) or a negative tl_status.  No call aborts, exits
 *     or throws.  tl_strerror() names a status.
 *   - Memory: the caller owns all memory.  Device memory comes from one
 *     caller-allocated workspace of tl_workspace_bytes() bytes given to
 *     tl_create(); pointers named dev_* are device pointers the caller owns;
 *     host_* are host pointers, read or written before the call returns unless
 *     stated otherwise.
 *   - Streams: every device operation is enqueued on the stream given to
 *     tl_create() (a cudaStream_t passed as void*; NULL = legacy default
 *     stream).  Device outputs are valid once the caller synchronises that
 *     stream.
 *   - Numbers: the residual stream, norms, softmax and every accumulation are
 *     FP32; the K/V cache and tensor-core operands are FP16; INT4 weights are
 *     dequantised exactly as (u - 8) * scale.
 */
#ifndef TL_H
#define TL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tl_status {
    TL_OK = 0,
    TL_EINVAL = -1,    /* bad argument, shape or configuration */
    TL_ENOMEM = -2,    /* workspace too small, or KV page pool exhausted */
    TL_ESTATE = -3,    /* call not valid in the context's current state */
    TL_EKV = -4,       /* a lane's L would rise above the depth its cache holds */
    TL_ECUDA = -5,     /* a CUDA runtime call failed (see tl_last_cuda_error) */
    TL_ETIMEOUT = -6,  /* a bounded device wait ran out */
    TL_EDEVICE = -7    /* a kernel recorded an out-of-range index in the status word */
} tl_status;

typedef enum tl_weight_fmt {
    TL_FMT_INT4 = 0,   /* packed nibbles u in [0,15], value (u - 8) * fp16 scale per group */
    TL_FMT_BF16 = 1    /* bfloat16 bit patterns */
} tl_weight_fmt;

/* Model and capacity.  d = n_heads * head_dim with head_dim 32, 64 or 128;
 * d and ffn multiples of 64 (the tensor-core projections take K in 64-wide
 * blocks); for INT4, group a multiple of 32 dividing d and ffn, with at
 * most 32 groups across d and across ffn.
 *
 * act_split: the tensor-core projections (rows above 8) multiply fp16 copies
 * of the activations.  Split, each copy is hi = fp16(x) and lo = fp16(x - hi)
 * and the projection sums both products (twice the MMAs), which keeps the
 * activations' fp32 precision to ~2^-22; single, one fp16 rounding (2^-11)
 * per projection input.  Automatic: split when a token's path crosses more
 * than 48 blocks (n_pre + L_max * n_loop_layers): the error of single fp16
 * grows with depth, and at 96 blocks (a 24-layer body at L = 4) it takes the
 * logits past relative L2 2e-3 from the exact model.  The few-row CUDA-core
 * projections keep fp32 activations either way. */
typedef struct tl_config {
    int32_t vocab;
    int32_t d;
    int32_t n_heads;
    int32_t ffn;
    int32_t n_pre;            /* pre blocks (own weights, own KV)                 */
    int32_t n_loop_layers;    /* layers in the shared loop body                   */
    int32_t fmt_pre;          /* tl_weight_fmt of pre-block matrices              */
    int32_t fmt_loop;         /* tl_weight_fmt of loop-body matrices              */
    int32_t fmt_embed_head;   /* tl_weight_fmt of embedding and head              */
    int32_t group;            /* INT4 group size along K (multiple of 32)         */
    float rms_eps;
    float rope_base;
    int32_t max_lanes;        /* lanes held at once                               */
    int32_t max_seq;          /* prompt + generated tokens per lane               */
    int32_t L_max;            /* largest per-lane loop count                      */
    int32_t kv_page_tokens;   /* tokens per KV page (power of two, >= 32)         */
    int32_t kv_pool_pages;    /* pages in the pool; 0 = one per lane/slot/page    */
    int32_t max_prefill_tokens; /* prompt rows one prefill call computes, summed
                                   over its lanes; 0 = max_seq                   */
    int32_t act_split;        /* activations for the tensor-core projections:
                                 0 automatic, 1 split, 2 single fp16 (below)     */
} tl_config;

typedef struct tl_ctx tl_ctx;

typedef struct tl_stats {
    int64_t loop_steps;          /* loop steps run (tl_loop_step + inside tl_decode) */
    int64_t lane_iterations;     /* sum over steps of lanes that ran an iteration */
    int64_t tokens_emitted;      /* greedy tokens written by tl_decode/tl_generate */
    int64_t prefill_tokens;      /* prompt positions run by tl_prefill          */
    int64_t kernel_launches;     /* kernels this library launched               */
    int32_t device_status;       /* last status word read back (0 = clean)      */
    int32_t kv_pages_used;
    int32_t entry_in_boundary;   /* the last decode ran entering lanes' first loop
                                    iteration in the boundary stage (1) or at the
                                    next tick (0); see tl_set_tick_overlap      */
    int32_t tick_layout;         /* the layout the last decode ran: 1, 2 or 3 (see
                                    tl_set_tick_overlap)                         */
    int64_t boundary_stages;     /* boundary stages launched apart from the loop
                                    steps (layout 3; in layouts 1 and 2 every tick
                                    holds one)                                    */
} tl_stats;

/* ---------------------------------------------------------------- sizes -- */

/* Bytes of device workspace tl_create() needs for cfg.  TL_EINVAL on a bad cfg. */
int tl_workspace_bytes(const tl_config* cfg, size_t* out_bytes);

/* Bytes of the weight blob for cfg (layout below).  Host-only; no CUDA call. */
int tl_weights_bytes(const tl_config* cfg, size_t* out_bytes);

/*
 * Weight blob layout (little endian, no padding):
 *   header: 8 bytes "TLWBLOB1", then the model fields of tl_config (vocab ..
 *           rope_base: ten int32 then two float32, declaration order; 48 bytes);
 *   matrices in this order: embed [V,d]; for each pre block then each loop
 *   layer: wqkv [3d,d] (rows q|k|v), wo [d,d], wg [F,d], wu [F,d], wd [d,F];
 *   head [V,d].  An INT4 matrix [N,K] is N*K/2 bytes of packed nibbles (row
 *   major; element 2i in the low nibble of byte i, 2i+1 in the high nibble)
 *   followed by N*(K/group) fp16 scales (row major).  A BF16 matrix is N*K
 *   uint16 bit patterns (row major);
 *   gains: for each pre block then loop layer g1[d], g2[d]; then g_final[d];
 *   fp32.
 * The INT4 convention (stored nibble u = code + 8, value (u - 8) * scale) is
 * "Benchmark Comparison" (measured benchmarks) section 5's symmetric form; the
 * nibble order is "CLI Reference", TINYLOOP_KV_INT4's.
 */

/* -------------------------------------------------------------- context -- */

/* Carve the caller's workspace (>= tl_workspace_bytes, 256-byte aligned) and
 * bind the stream.  The workspace must stay allocated until tl_destroy().
 * Launches initialisation kernels (RoPE table, page table, lane state).
 * Kernels launch with programmatic dependent launch (each may start while
 * its predecessor finishes); the environment variable TL_PDL=0, read here,
 * launches them fully serialised instead.
 * TL_EINVAL bad cfg/pointer; TL_ENOMEM workspace too small; TL_ECUDA. */
int tl_create(const tl_config* cfg, void* dev_workspace, size_t workspace_bytes,
              void* cuda_stream, tl_ctx** out_ctx);

/* Frees host-side state only (the workspace stays the caller's). */
int tl_destroy(tl_ctx* ctx);

/* Copy a weight blob (host memory, tl_weights_bytes(cfg) bytes, header must
 * match cfg) into the workspace's device layout.  The caller keeps the host
 * buffer.  Synchronous with respect to the host buffer.  TL_EINVAL on size,
 * magic or config mismatch. */
int tl_load_weights(tl_ctx* ctx, const void* host_blob, size_t bytes);

/* ------------------------------------------------------ weight preparation -- */

/* Symmetric per-group INT4 quantisation on the device ("Benchmark Comparison"
 * (measured benchmarks), section 7: per-group min-max, no calibration):
 * per row n and group j, scale = fp16_rne(max|w| / 7); code =
 * clamp(rint(w / scale), -7, 7) with the division in fp64 at the fp16 scale's
 * value (0 when scale is 0); stored nibble = code + 8.
 * dev_w: fp64 [N, K] row major.  dev_packed: [N, K/2] bytes; dev_scales: fp16
 * bits [N, K/group].  K % group == 0, group % 32 == 0.  Enqueued on
 * cuda_stream.  TL_EINVAL on bad sizes. */
int tl_quantize_int4(const double* dev_w, int64_t N, int64_t K, int32_t group,
                     uint8_t* dev_packed, uint16_t* dev_scales, void* cuda_stream);

/* Dequantise packed INT4 back to fp32 (exact): out[n,k] = (u - 8) * scale. */
int tl_dequant_int4(const uint8_t* dev_packed, const uint16_t* dev_scales, int64_t N,
                    int64_t K, int32_t group, float* dev_out, void* cuda_stream);

/* Round fp64 to the nearest bfloat16 (ties to even); dev_out: bf16 bits [n]. */
int tl_round_bf16(const double* dev_w, int64_t n, uint16_t* dev_out, void* cuda_stream);

/* ------------------------------------------------------------ lanes -- */

/* Run a lane's prompt ("CLI Reference", "benchmark": forward scoring over a
 * token sequence at --loops L): embed, pre blocks, then L loop iterations over
 * all T positions as one causal batch, filling the lane's K/V for the pre
 * blocks and iterations 1..L.  The lane becomes ready for its first greedy
 * token (tl_head_logits / tl_decode) with cap L.  Early exit does not apply to
 * the prompt.
 *   lane: 0..max_lanes-1 (any earlier content of the lane is dropped);
 *   host_tokens: int32 [T], ids in [0, vocab); 1 <= T <= max_seq, and the
 *     positions it computes (T minus the shared ones) <= max_prefill_tokens;
 *   L: 1..L_max;
 *   share_prefix_from_lane: -1, or a lane whose prompt starts with the same
 *     tokens and was prefilled at L' >= L; its full KV pages covering the first
 *     shared_tokens positions are mapped (reference counted) instead of being
 *     recomputed ("Benchmark Comparison" (measured benchmarks), section 2,
 *     SHARED prefix reuse); shared_tokens is rounded down to whole pages;
 *   dev_hidden_out: NULL or fp32 [T, d], the final hidden rows (before the
 *     head norm) of the positions computed (all T without a shared prefix).
 *   The donor must not be re-prefilled while lanes map its pages.
 * TL_EINVAL bad lane/T/L/token; TL_ENOMEM page pool exhausted. */
int tl_prefill(tl_ctx* ctx, int32_t lane, const int32_t* host_tokens, int32_t T, int32_t L,
               int32_t share_prefix_from_lane, int32_t shared_tokens, float* dev_hidden_out);

/* tl_prefill for n lanes in one pass: every block runs once over the rows of
 * all n prompts (a wide causal batch on the tensor cores), iteration l over
 * the lanes whose L exceeds l; attention stays per lane.  Same result per
 * lane as n tl_prefill calls.  This is the prompt side of L-aware batching
 * ("Dynamic-L Inference", "L-Aware Batching": one batch call with a loop
 * count per lane).
 *   lanes: host int32 [n], distinct, 0..max_lanes-1;
 *   host_tokens: the n prompts back to back, lane i's T[i] ids after lane
 *     i-1's;
 *   T, L: host int32 [n], as for tl_prefill;
 *   share_prefix_from_lane, shared_tokens: as for tl_prefill, applied to
 *     every lane of the batch (the donor must not be one of them).
 *   The positions computed, summed over the lanes, must be <=
 *   max_prefill_tokens.
 * TL_EINVAL bad arguments (nothing is changed); TL_ENOMEM page pool
 * exhausted (the batch's lanes are left empty). */
int tl_prefill_batch(tl_ctx* ctx, int32_t n, const int32_t* lanes, const int32_t* host_tokens,
                     const int32_t* T, const int32_t* L, int32_t share_prefix_from_lane,
                     int32_t shared_tokens);

/* Early-exit parameters for all lanes ("CLI Reference", generate options):
 * probe at iteration l when l > min_L and (l - min_L - 1) % peek_every == 0;
 * a probe with delta = ||h_l - h_{l-1}|| / ||h_{l-1}|| < tau extends the
 * streak, any other probe resets it; exit once streak >= patience.
 * tau <= 0 or patience == 0 disables it.  peek_every >= 1.  Replaces the
 * logit-margin mode. */
int tl_set_early_exit(tl_ctx* ctx, double tau, int32_t min_L, int32_t patience, int32_t peek_every);

/* Logit-margin early exit for all lanes ("CLI Reference",
 * --early-exit-logit-margin, and its "Current Behavior" note that this is the
 * mode that fires): the same probe schedule, streak and patience as
 * tl_set_early_exit, but a probe's metric is the head's top-1 minus top-2
 * logit (final RMSNorm and head projection of the lane's hidden state at that
 * iteration, a full head pass per probe) and the probe succeeds when the
 * margin is at least `margin` (the pages say the loop stops when the model is
 * confidently predicting one token; "at least the threshold" is the reading
 * taken).  Replaces the hidden-state mode; margin <= 0 or patience == 0
 * disables early exit.  peek_every >= 1. */
int tl_set_early_exit_logit_margin(tl_ctx* ctx, double margin, int32_t min_L, int32_t patience,
                                   int32_t peek_every);

/* L warmup for all lanes ("Dynamic-L Inference", L scheduling: the first N
 * tokens at a shallow depth, the rest at full depth; "CLI Reference",
 * --l-warmup-tokens / --l-warmup-L): decode tokens 1..warmup_tokens after the
 * prompt's token run min(warmup_L, L requested) iterations (early exit may
 * stop them sooner) and do not lower the lane's cap; later tokens run min(L
 * requested, cap) as usual.  A later token's deeper iteration l, at a
 * position that a warmup token computed only to depth D < l, attends to that
 * position's K/V of iteration D (the deepest iteration holding it; the pages
 * do not say, this is the reading taken): when a warmup token's loop ends,
 * its K/V are copied into the slots of the iterations above D.  warmup_tokens
 * = 0 disables it (the default).  Takes effect for tokens entered afterwards.
 * TL_EINVAL for warmup_tokens < 0 or warmup_L < 1. */
int tl_set_l_warmup(tl_ctx* ctx, int32_t warmup_tokens, int32_t warmup_L);

/* One loop step: every lane with dev_active_mask[lane] != 0 that is in its
 * loop phase runs its next loop iteration (all body layers), at its own
 * iteration index; then the device applies the early-exit rule.
 *   dev_per_lane_L: NULL, or int32 [max_lanes] requested L per lane; a lane
 *     whose request rose above the depth its cache holds sets TL_EKV in the
 *     status word and does not run;
 *   dev_active_mask: NULL (= all lanes) or uint8 [max_lanes];
 *   dev_exit_mask_out: NULL or uint8 [max_lanes]: 1 where the lane's loop for
 *     its current token finished in this step (early exit or L reached),
 *     0 elsewhere.
 * Device-side only: the host never waits. */
int tl_loop_step(tl_ctx* ctx, const int32_t* dev_per_lane_L, const uint8_t* dev_active_mask,
                 uint8_t* dev_exit_mask_out);

/* Boundary stage, head: for lanes with dev_lane_mask[lane] != 0 (NULL = all
 * lanes whose loop finished), final RMSNorm + head projection + greedy argmax.
 *   dev_logits: NULL or fp32 [max_lanes, vocab] (rows of other lanes untouched);
 *   dev_argmax: NULL or int32 [max_lanes]. */
int tl_head_logits(tl_ctx* ctx, const uint8_t* dev_lane_mask, float* dev_logits, int32_t* dev_argmax);

/* Boundary stage, token entry: for lanes with dev_lane_mask[lane] != 0, record
 * that the lane's last loop ran to its finished depth (the lane's cap becomes
 * that depth), advance its position, embed dev_tokens[lane] (int32
 * [max_lanes]) and run the pre blocks, leaving the lane at the start of its
 * loop.  Lets a caller drive decode with its own tokens (teacher forcing). */
int tl_embed_next(tl_ctx* ctx, const uint8_t* dev_lane_mask, const int32_t* dev_tokens);

/* Greedy continuous-depth decode of lanes 0..n_lanes-1, all prefilled.
 * Emits n_new tokens per lane: the first from the lane's current hidden state
 * (its prompt), each later one after a loop of min(L_requested, cap)
 * iterations or fewer under early exit.  Steps run until every lane has
 * emitted n_new tokens; lanes leave and re-enter the loop batch on the device.
 *   host_per_lane_L: int32 [n_lanes] requested L (<= the prefill L);
 *   dev_tokens_out / dev_depths_out: int32 [n_lanes, n_new] (NULL allowed):
 *     the tokens and the iterations run behind each (the prefill L for the
 *     first token).
 * TL_EKV when a request exceeds the lane's cache depth. */
int tl_decode(tl_ctx* ctx, const int32_t* host_per_lane_L, int32_t n_lanes, int32_t n_new,
              int32_t* dev_tokens_out, int32_t* dev_depths_out);

/* End to end from host memory ("Dynamic-L Inference", "L-Aware Batching":
 * generate_batch(prompts, per_lane_loops)): copy prompts to the device,
 * prefill every lane at its L (as tl_prefill_batch, as many lanes per pass as
 * max_prefill_tokens allows), decode n_new tokens per lane, copy tokens and
 * depths back.  host_prompts: int32 [n_lanes, T]; outputs int32 [n_lanes,
 * n_new] in host memory (pinned memory makes the copies asynchronous-capable).
 * Returns after the results are in host memory. */
int tl_generate(tl_ctx* ctx, const int32_t* host_prompts, int32_t n_lanes, int32_t T,
                const int32_t* host_per_lane_L, int32_t n_new, int32_t* host_tokens_out,
                int32_t* host_depths_out);

/* Self-speculative greedy decode of one lane ("CLI Reference", speculate:
 * --draft-loops, --verify-loops, --draft-ahead at temperature 0; the same
 * weights and one KV cache serve both depths).  The lane must be at a
 * boundary with no token taken since its prompt: freshly prefilled
 * (tl_prefill / tl_prefill_batch) at L >= max(L_draft, L_verify), or left so
 * by a previous tl_speculate.
 * Its first token comes from the prompt's last position; then each round
 * drafts up to draft_ahead tokens at L_draft, one position at a time (every
 * greedy token fed back on the device), runs the drafted positions again at
 * L_verify as one causal batch (embed, pre blocks, L_verify iterations,
 * rewriting their K/V in every slot), keeps the drafted tokens up to the first
 * one the verify pass's greedy choice differs from and takes the verify
 * pass's token there, and continues from the last kept position.  With greedy
 * choices the tokens are those of a plain decode at L_verify; the draft only
 * decides how many positions one verify pass covers.  Early exit and L warmup
 * are off for the call.  One host synchronisation per round.
 *   host_tokens_out: int32 [n_new]; host_rounds_out: NULL or the number of
 *   verify rounds.  Positions up to prompt length + n_new - 2 are written, so
 *   that must stay below max_seq; draft_ahead <= max_lanes and <=
 *   max_prefill_tokens.  Afterwards the lane is at its last kept position
 *   with cap L_verify, as after a prompt: a following tl_decode or
 *   tl_speculate starts there, so its first token is this call's last.
 * TL_ESTATE if the lane is not at such a boundary; TL_EKV if a depth exceeds
 * its cache; TL_EINVAL on bad arguments. */
int tl_speculate(tl_ctx* ctx, int32_t lane, int32_t n_new, int32_t L_draft, int32_t L_verify, int32_t draft_ahead,
                 int32_t* host_tokens_out, int32_t* host_rounds_out);

/* Layout of a decode tick ("Depth-adaptive Inference of Looped Language
 * Models via Continuous Depth Batching": boundary stages queued apart from
 * loop steps, with scheduling overlapping GPU work).  In modes 1 and 2 every
 * tick runs two concurrent branches on disjoint lanes and ends when both
 * have: the boundary stage (head, greedy token, embedding and pre blocks of
 * the lanes whose loop finished) and one loop iteration of the lanes in their
 * loop.  mode 1: a lane that takes a token also runs its first loop
 * iteration in that boundary stage (a token costs its depth in ticks); mode
 * 2: it joins the loop step at the next tick (one tick more per token, a
 * shorter boundary stage).  mode 3: the two run on two streams at their own
 * cadence with no join per tick; each boundary stage takes the lanes whose
 * loop has finished when it starts and hands those that continue to the loop
 * when their pre blocks are done (needs CUDA graphs, else mode 2 runs).
 * mode 0 (default) chooses per decode call: mode 3 for 32+ lanes with mean
 * requested L of 6 or more, mode 1 otherwise.  Results per lane do not
 * depend on it beyond the rounding differences of batch width: in a decode
 * of more than 8 lanes the loop steps always run on the tensor cores (fp16
 * activation copies), while a boundary stage of at most 8 rows takes fp32
 * activations and a wider one fp16, and attention's context split follows
 * the step's row count; in mode 3 the widths depend on timing.  See
 * tl_stats.tick_layout.  TL_EINVAL for other modes. */
int tl_set_tick_overlap(tl_ctx* ctx, int32_t mode);

/* Shared-prefix ("cascade") attention in decode steps (default on; "Benchmark
 * Comparison" (measured benchmarks), section 2: one cached prefix serves many
 * requests, and in a looped model every loop iteration of them).  When every
 * lane that maps shared prefix pages (tl_prefill with share_prefix_from_lane)
 * maps the same donor's prefix of the same length, each decode attention step
 * first attends all such rows at one loop iteration to the prefix together
 * on the tensor cores (head widths 64 and 128), reading each prefix page once
 * per step instead of once per lane, and then each row's own positions; the
 * two are merged by log-sum-exp.  Same result up to summation order.
 * enabled = 0 attends every lane's whole context on its own. */
int tl_set_cascade(tl_ctx* ctx, int32_t enabled);

/* Replay of decode ticks as CUDA graphs (default on): each tick of tl_decode /
 * tl_generate is one captured graph whose conditional nodes, set on the
 * device from the live row counts, skip empty stages and pick the CUDA-core or
 * tensor-core variant of a stage.  enabled = 0 launches every kernel of a tick
 * individually instead (same kernels and results; what profilers that cannot
 * look inside graphs with conditional nodes need).  Timing with
 * tl_profile_begin also launches individually. */
int tl_set_graphs(tl_ctx* ctx, int32_t enabled);

/* ------------------------------------------------- lane-state checkpoint -- */

/* Bytes of a lane-state snapshot: the scheduling state and the fp32 hidden row
 * of every lane (max_lanes * (52 + 4 d)).  The KV cache is not part of it: a
 * decode started from a restored snapshot rewrites every position past the
 * saved ones before reading it, and positions at or before them are never
 * written by decode. */
int tl_lane_state_bytes(tl_ctx* ctx, size_t* out_bytes);

/* Copy the lane states into dev_dst (device, tl_lane_state_bytes bytes),
 * enqueued on the context's stream. */
int tl_lane_state_save(tl_ctx* ctx, void* dev_dst);

/* Restore lane states saved by tl_lane_state_save on this context. */
int tl_lane_state_load(tl_ctx* ctx, const void* dev_src);

/* ------------------------------------------------------------ profiling -- */

typedef enum tl_prof_kind {
    TL_PROF_NONE = 0,
    TL_PROF_ATTN = 1,   /* per-iteration attention launches                  */
    TL_PROF_PROJ = 2,   /* block projections (QKV, O, gate/up, down)         */
    TL_PROF_HEAD = 3    /* head projection + argmax partials                 */
} tl_prof_kind;

/* Time every launch group of the kinds in kind_mask (bit k = tl_prof_kind k)
 * with CUDA events on the context's stream until tl_profile_end.  A group is
 * one attention launch, or the one or two kernels of one projection.  Cost:
 * two event records per group; the host waits only when 4096 groups are
 * outstanding.  TL_EINVAL for bits outside kinds 1..3. */
int tl_profile_begin(tl_ctx* ctx, int32_t kind_mask);

/* Stop timing.  out_groups / out_total_ms (nullable) receive 4 entries indexed
 * by tl_prof_kind: groups timed and their summed device time in ms. */
int tl_profile_end(tl_ctx* ctx, int64_t* out_groups, double* out_total_ms);

/* ------------------------------------------------ allocation-free head -- */

/* Greedy LM head for callers that cannot allocate device memory.  The pages
 * have no counterpart for this call: it exists because some callers cannot
 * allocate device memory at the time they need the head (a serving loop that
 * reserved all its memory at start-up and forbids allocation afterwards, a
 * host framework whose allocator owns every cudaMalloc, or code that runs
 * while a stream is being captured, where cudaMalloc is not allowed), and
 * tl_head_logits needs the scratch space of a tl_create workspace.
 *
 * Computes, for r < rows: logits[r] = RMSNorm(h[r]; g_final, rms_eps) W^T and
 * argmax[r] = the lowest id among the largest logits.  Enqueued on
 * cuda_stream; calls no cudaMalloc / cudaFree and no allocating routine.
 *   dev_h: fp32 [rows][d] hidden rows (before the final norm);
 *   dev_g_final: fp32 [d];
 *   dev_head_packed: INT4 head [V][d/2] in the weight blob's packing (element
 *     2i in the low nibble of byte i), 16-byte aligned;
 *   dev_head_scales: fp16 bits [V][d/group];
 *   dev_logits: NULL or fp32 [rows][V]; dev_argmax: int32 [rows].
 * Its scratch is one fixed array in device global memory defined by the
 * library (about 1.5 MB, held on every GPU that loads the library until the
 * process exits): rows <= 64, d <= 4096 and V <= 262144, else TL_ENOMEM with
 * nothing enqueued.  Every call shares that array and it keeps the last
 * call's contents (each call writes all it reads); calls whose kernels
 * overlap on the GPU (unordered streams) race on it.  The first call on a
 * device looks up the array's device address with that device current; make
 * that first call before any stream capture begins.  TL_EINVAL on NULL inputs,
 * d or group not multiples of 32, group not dividing d, a head pointer not
 * 16-byte aligned or another pointer not aligned to its element size
 * (nothing is enqueued). */
int tl_head_argmax_static(const float* dev_h, int32_t rows, const float* dev_g_final, float rms_eps,
                          const uint8_t* dev_head_packed, const uint16_t* dev_head_scales, int32_t V,
                          int32_t d, int32_t group, float* dev_logits, int32_t* dev_argmax, void* cuda_stream);

/* ---------------------------------------------------------- measurement -- */

/* Read-bandwidth probe (a measurement aid, not a step of the model; the pages
 * relate the loop block's cost to where its weights are read from,
 * "Benchmark Comparison" (measured benchmarks), section 6, L2 residency):
 * 4 CTAs per SM read dev_src[0 .. bytes) with 16-byte loads, reps times over,
 * and write one word per CTA into dev_sink.  The caller times it with events
 * on cuda_stream: a buffer well under the L2 capacity gives the L2 read
 * bandwidth (after a first pass), one far larger than L2 the HBM read
 * bandwidth.  dev_src 16-byte aligned, bytes a multiple of 16, reps >= 1,
 * n_sink >= 4 x the SM count; TL_EINVAL otherwise (nothing enqueued). */
int tl_read_probe(const void* dev_src, size_t bytes, int32_t reps, uint32_t* dev_sink, int32_t n_sink,
                  void* cuda_stream);

/* -------------------------------------------------------------- misc -- */

/* Counters; also reads back and clears the device status word (synchronises
 * the stream). */
int tl_stats_get(tl_ctx* ctx, tl_stats* out);

/* Name of a tl_status. */
const char* tl_strerror(int status);

/* The last CUDA error string recorded by this thread ("" if none). */
const char* tl_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TL_H */
