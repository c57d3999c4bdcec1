// libtl runtime: workspace carve-up, weight loading, KV page allocation,
// prefill, loop steps, boundary stages and the continuous-depth decode loop.
// Every call below enqueues kernels on the context's stream; the only host
// waits are the lagged "lanes still alive" polls of tl_decode and the explicit
// synchronisations of tl_generate / tl_stats_get.
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <array>
#include <cstring>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_util.h"
#include "attn_decode.cuh"
#include "attn_split.cuh"
#include "attn_tc.cuh"
#include "gemv_stream.cuh"
#include "kernels.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm_wide.cuh"

namespace tl {

static thread_local std::string g_cuda_err;

int check_cuda(cudaError_t e) {
  if (e == cudaSuccess) return TL_OK;
  g_cuda_err = cudaGetErrorString(e);
  return TL_ECUDA;
}

static size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

static bool cfg_valid(const tl_config* c) {
  if (!c) return false;
  if (c->vocab <= 0 || c->d <= 0 || c->n_heads <= 0 || c->ffn <= 0 || c->n_pre < 0 || c->n_loop_layers < 1)
    return false;
  if (c->d % c->n_heads) return false;
  const int hd = c->d / c->n_heads;
  if (hd != 32 && hd != 64 && hd != 128) return false;
  // the tensor-core projections step through K in 64-wide blocks (K is d or ffn)
  if (c->d % 64 || c->ffn % 64) return false;
  const int fmts[3] = {c->fmt_pre, c->fmt_loop, c->fmt_embed_head};
  bool any_int4 = false;
  for (int f : fmts) {
    if (f != TL_FMT_INT4 && f != TL_FMT_BF16) return false;
    any_int4 |= f == TL_FMT_INT4;
  }
  if (any_int4 && (c->group <= 0 || c->group % 32 || c->d % c->group || c->ffn % c->group)) return false;
  // the decode tensor-core kernel stages a row's scale groups for its K range in shared memory
  if (any_int4 && (c->d / c->group > TC_SC_MAX - 1 || c->ffn / c->group > TC_SC_MAX - 1)) return false;
  if (!(c->rms_eps >= 0.f) || !(c->rope_base > 0.f)) return false;
  if (c->max_lanes < 1 || c->max_lanes > 1024 || c->max_seq < 1 || c->L_max < 1) return false;
  if (c->kv_page_tokens < 32 || (c->kv_page_tokens & (c->kv_page_tokens - 1))) return false;
  if (c->kv_pool_pages < 0 || c->max_prefill_tokens < 0) return false;
  if (c->act_split < 0 || c->act_split > 2) return false;
  return true;
}

// Split activations for the tensor cores (act16_put): on when asked, or
// automatically when a token's path crosses more than kSplitDepth blocks.
// Measured with the oracle on the 1.4B-class shape (24-layer body, L = 2, a
// 1,088-position context): fp16 activations alone put the first token's
// logits at relative L2 1.9e-3 from the fp64 result, fp16 K/V 1.2e-3, fp16
// attention probabilities 0.9e-3, all three 2.4e-3 (the GPU: 2.39e-3),
// against a bar of 2e-3; the 407M-class model at L = 32 (34 blocks) stays
// at 1.5e-3 with fp16 activations.
constexpr int kSplitDepth = 48;

// Blocks with a resident fp16 copy of their matrices: all of them (pre blocks
// first, then the loop body's layers).  The tensor-core projections read the
// copy; the few-row GEMV reads the INT4 or BF16 weights themselves.
static int n_f16_blocks(const tl_config* c) { return c->n_pre + c->n_loop_layers; }
static int act_split_on(const tl_config* c) {
  if (c->act_split != 0) return c->act_split == 1 ? 1 : 0;
  return c->n_pre + c->L_max * c->n_loop_layers > kSplitDepth ? 1 : 0;
}

// TMA row coordinates into the KV pool are 32-bit signed.
static bool kv_rows_ok(const tl_config* c, int64_t n_pages) {
  return n_pages * 2 * c->n_heads * (int64_t)c->kv_page_tokens < (int64_t(1) << 31);
}

static size_t mat_bytes(const tl_config* c, int fmt, int64_t N, int64_t K) {
  if (fmt == TL_FMT_INT4) return (size_t)(N * K / 2) + (size_t)(N * (K / c->group)) * 2;
  return (size_t)(N * K) * 2;
}

struct MatSpec {
  int fmt;
  int64_t N, K;
};

static std::vector<MatSpec> mat_specs(const tl_config* c) {
  std::vector<MatSpec> v;
  const int64_t d = c->d, F = c->ffn, V = c->vocab;
  v.push_back({c->fmt_embed_head, V, d});
  for (int b = 0; b < c->n_pre + c->n_loop_layers; ++b) {
    const int f = b < c->n_pre ? c->fmt_pre : c->fmt_loop;
    v.push_back({f, 3 * d, d});
    v.push_back({f, d, d});
    v.push_back({f, F, d});
    v.push_back({f, F, d});
    v.push_back({f, d, F});
  }
  v.push_back({c->fmt_embed_head, V, d});
  return v;
}

static constexpr size_t kBlobHeader = 8 + 48;

static size_t blob_bytes(const tl_config* c) {
  size_t s = kBlobHeader;
  for (const auto& m : mat_specs(c)) s += mat_bytes(c, m.fmt, m.N, m.K);
  s += (size_t)(2 * (c->n_pre + c->n_loop_layers) + 1) * c->d * 4;
  return s;
}

// ------------------------------------------------- tensor-core tiling ----

constexpr int kGemvMaxRows = 8;  // row counts the CUDA-core GEMV takes; more go to the tensor cores
enum ProjPath { PATH_AUTO = 0, PATH_GEMV = 1, PATH_TC = 2 };
// head GEMV: output features per warp (its registers hold that many raw chunks
// and 8 row accumulators each)
constexpr int head_rpw(int fmt) { return fmt == TL_FMT_INT4 ? 4 : 2; }

// Activation rows per tensor-core tile.  The gate/up pair stays at 128 above
// 128 rows: its 256-row tile cannot split K (the pair's partial tiles would
// need 256 KB of shared memory), which left a 256-row step with one CTA per
// 128 weight rows (44 CTAs for a 5,632-wide FFN: 74 us per launch).
static int tc_nt(int max_rows, int nmat = 1) {
  if (max_rows <= 64) return 64;
  return (max_rows <= 128 || nmat == 2) ? 128 : 256;
}

template <int NMAT, int FMT>
static bool tc_split_ok(int nt) {
  return nt == 64 ? TcCfg<64, NMAT, FMT>::SPLIT_OK
                  : (nt == 128 ? TcCfg<128, NMAT, FMT>::SPLIT_OK : TcCfg<256, NMAT, FMT>::SPLIT_OK);
}

// Split of the K loop (the cluster size, <= 8) so that the grid fills the 148
// SMs (two CTAs per SM fit for the 64-row single-matrix tile).  Every split
// keeps >= 2 k-blocks; its INT4 scale groups stay within TC_SC_MAX because the
// configuration allows at most TC_SC_MAX - 1 groups over the whole K.
static int tc_splits(int N, int K, int max_rows, int nmat, int fmt, int group) {
  const int nt = tc_nt(max_rows, nmat);
  const bool ok = nmat == 1 ? (fmt == TL_FMT_INT4 ? tc_split_ok<1, TL_FMT_INT4>(nt)
                                                 : (fmt == FMT_F16 ? tc_split_ok<1, FMT_F16>(nt)
                                                                   : tc_split_ok<1, TL_FMT_BF16>(nt)))
                            : (fmt == TL_FMT_INT4 ? tc_split_ok<2, TL_FMT_INT4>(nt)
                                                 : (fmt == FMT_F16 ? tc_split_ok<2, FMT_F16>(nt)
                                                                   : tc_split_ok<2, TL_FMT_BF16>(nt)));
  const int m_tiles = (N + 127) / 128, n_tiles = (max_rows + nt - 1) / nt;
  const int kb = K / 64;
  const int slots = (nmat == 1 && nt == 64) ? 296 : 148;
  int best = 1;
  for (int s = 2; s <= 8 && ok; ++s) {
    if (kb % s || kb / s < 2) continue;
    if ((int64_t)m_tiles * n_tiles * s <= slots) best = s;
  }
  return best;
}

// ------------------------------------------------ streamed GEMV geometry ----

struct GsChoice {
  bool ok;
  GsPlan pl;
  int smem, grid;
};

// Blocks of fb output features (>= 8, a multiple of 8, ~16 KB of weights) and
// as many ring stages as fit beside the 8-row activation tile.
static GsChoice gs_plan(int fmt, int N, int K, int group, int nmat, int n_sms, int cap = 220 * 1024) {
  GsChoice c{};
  const int row = fmt == TL_FMT_INT4 ? K / 2 : 2 * K;
  const int sc = fmt == TL_FMT_INT4 ? (K / group) * 2 : 0;
  int fb = (16384 / (row + sc)) / 8 * 8;
  if (fb < 8) fb = 8;
  const int stage = (fb * (row + sc) + 127) / 128 * 128;
  const int xs = 8 * K * 4;
  int stages = (cap - xs - 512) / (nmat * stage);
  if (stages < 2) stages = (220 * 1024 - xs - 512) / (nmat * stage);  // the cap is a preference
  if (stages > 8) stages = 8;
  if (stages < 2) return c;
  if (((int64_t)(N % fb) * sc) % 16) return c;  // the last block's scales must be a 16-byte multiple
  c.pl.fb = fb;
  c.pl.stages = stages;
  c.pl.stage_bytes = stage;
  c.pl.row_bytes = row;
  c.pl.sc_row_bytes = sc;
  c.pl.xs_offset = stages * nmat * stage;
  c.pl.bar_offset = c.pl.xs_offset + xs;
  c.smem = c.pl.bar_offset + 2 * stages * 8 + 16;
  const int nblocks = (N + fb - 1) / fb;
  c.grid = nblocks < n_sms ? nblocks : n_sms;
  c.ok = true;
  return c;
}

// Offsets of every workspace region (computed identically by tl_workspace_bytes and tl_create).
struct Layout {
  int n_slots, pages_per_seq, n_pages, max_rows, n_parts, max_prefill;
  size_t page_elems;
  std::vector<size_t> mat_off;  // per matrix
  size_t gains, rope, page_table, kv, lanes, h, h_in, hrows, rows[6], act_a, act_qkv, act_q, act_o, act_u,
      act_a16, act_o16, act_u16, attn_part, attn_counters, part_val, part_idx, tok_stage, L_stage,
      mask_stage, pf_n, pf_tiles, pf_info, probe_logits, margin_lane, spec, lane_shared, casc,
      f16blk, out_tok, out_dep, status, counters, body_kernels, alive, b_act_a, b_act_qkv, b_act_q, b_act_o, b_act_u,
      b_act_a16, b_act_o16, b_act_u16, b_attn_part, b_attn_counters, b_part_val, b_part_idx, b_casc, total;
};

static Layout make_layout(const tl_config* c) {
  Layout L;
  const int hd = c->d / c->n_heads;
  L.max_prefill = c->max_prefill_tokens ? c->max_prefill_tokens : c->max_seq;
  L.n_slots = c->n_pre + c->L_max * c->n_loop_layers;
  L.pages_per_seq = (c->max_seq + c->kv_page_tokens - 1) / c->kv_page_tokens;
  L.n_pages = c->kv_pool_pages ? c->kv_pool_pages : c->max_lanes * L.n_slots * L.pages_per_seq;
  L.page_elems = (size_t)2 * c->n_heads * c->kv_page_tokens * hd;
  L.max_rows = c->max_lanes > L.max_prefill ? c->max_lanes : L.max_prefill;
  L.n_parts = (c->vocab + GEMV_WARPS * 2 - 1) / (GEMV_WARPS * 2);  // the smallest head_rpw
  if (L.n_parts < 1024) L.n_parts = 1024;                            // streamed GEMV: one per SM
  if (L.n_parts < (c->vocab + 127) / 128) L.n_parts = (c->vocab + 127) / 128;  // tensor-core head: one per tile
  size_t o = 0;
  for (const auto& m : mat_specs(c)) {
    L.mat_off.push_back(o);
    o = align_up(o + mat_bytes(c, m.fmt, m.N, m.K));
  }
  const size_t d = c->d, F = c->ffn, R = L.max_rows, lanes = c->max_lanes;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.gains = take((size_t)(2 * (c->n_pre + c->n_loop_layers) + 1) * d * 4);
  L.rope = take((size_t)c->max_seq * (hd / 2) * 8);
  L.page_table = take(lanes * L.n_slots * L.pages_per_seq * 4);
  L.kv = take((size_t)L.n_pages * L.page_elems * 2);
  L.lanes = take(lanes * sizeof(LaneState));
  L.h = take(lanes * d * 4);
  L.h_in = take(lanes * d * 4);
  L.hrows = take((size_t)L.max_prefill * d * 4);
  for (int i = 0; i < 6; ++i) L.rows[i] = take(4 + 3 * R * 4 + 16);
  L.act_a = take(R * d * 4);
  L.act_qkv = take(R * 3 * d * 4);
  L.act_q = take(R * d * 4);
  L.act_o = take(R * d * 4);
  L.act_u = take(R * F * 4);
  const size_t s16 = (size_t)1 << act_split_on(c);  // [hi | lo] rows with split activations
  L.act_a16 = take(R * d * 2 * s16);
  L.act_o16 = take(R * d * 2 * s16);
  L.act_u16 = take(R * F * 2 * s16);
  L.attn_part = take(lanes * c->n_heads * kAttnPieces * (hd + 2) * 4);
  L.attn_counters = take(lanes * c->n_heads * 4);
  L.part_val = take(lanes * L.n_parts * 4);
  L.part_idx = take(lanes * L.n_parts * 4);
  L.tok_stage = take(R * 4);
  L.L_stage = take(lanes * 4);
  L.mask_stage = take(lanes);
  L.pf_n = take((size_t)(c->L_max + 2) * 4);
  L.pf_tiles = take((R / 64 + lanes + 2) * 8);
  L.pf_info = take(lanes * 16);
  L.probe_logits = take(lanes * (size_t)c->vocab * 4);
  L.margin_lane = take(lanes * 4);
  L.spec = take((lanes + 3 * L.max_prefill + 8) * 4);
  L.lane_shared = take(lanes * 4);
  L.casc = take(lanes * c->n_heads * (hd + 2) * 4);
  // prompt batches wide enough for the persistent GEMM: one block's five matrices in fp16
  // a resident fp16 copy of every block matrix (BF16: the same bytes per weight; INT4: four times, 100 MB
  // at the 407M-class shape), so the tensor-core projections load weight tiles straight into the MMA layout
  // instead of converting them every step (64 lanes: 33.8k -> 36.0k tokens/s; 1.4B-class BF16, 256 lanes:
  // 5.9k -> 8.6k)
  L.f16blk = take((size_t)n_f16_blocks(c) * (4 * d * d + 3 * d * F) * 2);
  L.out_tok = take(lanes * (size_t)c->max_seq * 4);
  L.out_dep = take(lanes * (size_t)c->max_seq * 4);
  L.status = take(4);
  L.counters = take(4 * 8);
  L.body_kernels = take(8 * 4);
  L.alive = take(8);  // alive lanes, loop rows
  // the decode boundary stage's own scratch (rows = lanes)
  L.b_act_a = take(lanes * d * 4);
  L.b_act_qkv = take(lanes * 3 * d * 4);
  L.b_act_q = take(lanes * d * 4);
  L.b_act_o = take(lanes * d * 4);
  L.b_act_u = take(lanes * F * 4);
  L.b_act_a16 = take(lanes * d * 2 * s16);
  L.b_act_o16 = take(lanes * d * 2 * s16);
  L.b_act_u16 = take(lanes * F * 2 * s16);
  L.b_attn_part = take(lanes * c->n_heads * kAttnPieces * (hd + 2) * 4);
  L.b_attn_counters = take(lanes * c->n_heads * 4);
  L.b_part_val = take(lanes * L.n_parts * 4);
  L.b_part_idx = take(lanes * L.n_parts * 4);
  L.b_casc = take(lanes * c->n_heads * (hd + 2) * 4);
  L.total = o;
  return L;
}

struct BlockW {
  MatView wqkv, wo, wg, wu, wd;
  const float *g1, *g2;
  CUtensorMap mqkv, mo, mg, mu, md;  // TMA maps of the raw weight tiles
  const BlockW* f16 = nullptr;       // the resident fp16 copy the tensor-core projections read
};

// Row-wise scratch of one stream of projection / attention / head kernels.  A
// decode tick runs its boundary stage (head, token, embedding, pre blocks of
// the entering lanes) and its loop iteration as two concurrent branches, each
// with its own set; prompts and single calls use the main set.
struct Scratch {
  int rows;                        // rows the activation buffers hold
  float *act_a, *act_qkv, *act_q, *act_o, *act_u;
  __half *act_a16, *act_o16, *act_u16;
  float* attn_part;                // decode attention split / piece partials
  int32_t* attn_counters;
  float* part_val;                 // head argmax partials
  int32_t* part_idx;
  int32_t* head_nparts;            // device: partial count written by the head kernel that ran
  float* casc;                     // shared-prefix attention partials
  CUtensorMap xmap[3][3];          // [a16, o16, u16][NT 64, 128, 256]
  int gs_cap;                      // shared memory the streamed GEMV may take per CTA
  int gs_ctas;                     // CTAs (SMs) the streamed GEMV may take
  Rows probe;                      // logit-margin probe rows of this stream's loop iterations
};

}  // namespace tl

using namespace tl;

struct tl_ctx {
  tl_config cfg;
  Layout lay;
  cudaStream_t stream;
  char* ws;
  size_t ws_bytes;
  int hd;
  bool loaded = false;
  int split16 = 0;  // tensor-core activation copies as [hi | lo] (act_split_on)
  MatView embed, head;
  std::vector<BlockW> pre, loop;
  const float* g_final;
  KVGeom kv;
  float2* rope;
  int32_t* page_table;
  LaneState* lanes;
  float *h, *h_in, *hrows;
  Rows rows[6];  // 0 loop, 1 boundary, 2 entered, 3 prefill / mask, 4 / 5 logit-margin probes (per scratch)
  Scratch scr[2];       // 0 main (prompts, loop iterations), 1 a decode tick's boundary stage
  Scratch* sc = nullptr;  // the set the next launches use
  float* probe_logits;  // [lanes][vocab] head logits of the lanes probing in margin mode
  float* margin_lane;   // [lanes] their top-1 minus top-2 margins
  int32_t* spec;        // speculation: [lanes] token per lane, then drafted, verify-input and verify tokens
  int32_t* lane_shared; // [lanes] shared-prefix positions each lane maps (device copy of h_lane_shared)
  std::vector<int32_t> h_lane_shared, h_lane_donor;
  bool cascade_enabled = true;  // tl_set_cascade
  bool cascade_active = false;  // enabled, and the lanes that share map one donor's prefix of one length
  std::vector<BlockW> blk16;    // resident fp16 copies of the blocks (see BlockW::f16)
  int32_t *tok_stage, *L_stage, *out_tok, *out_dep, *status, *alive;
  int32_t* pf_n;     // prompt batches: row count of each stage (stage l = loop iteration l)
  int2* pf_tiles;    // prompt batches: attention tiles (first row, rows)
  int32_t* pf_info;  // prompt batches: per lane (lane, last row, last position, L)
  uint8_t* mask_stage;
  unsigned long long* counters;  // 0 lane iterations, 1 tokens, 2 kernels run inside conditional graph bodies
  int32_t* body_kernels;          // [stage][variant] kernels of each conditional body (graph ticks)
  EEParams ee{0.0, 2, 0, 1, 0, 0, 0.0};
  WarmParams warm{0, 2};
  int n_sms = 148;
  int head_parts = 0;  // partial results per row written by the head projection
  CUtensorMap mhead;   // TMA map of the head's raw weight tiles
  CUtensorMap kvmap;   // TMA map of the KV pool: rows of hd fp16, tiles of kAttnUK rows (swizzled)
  // CUDA graph of one decode tick (captured on cap_stream, replayed on stream)
  cudaStream_t cap_stream = nullptr, cap_body = nullptr, cap_stream2 = nullptr;
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;  // the tick graph's boundary branch
  cudaGraphExec_t tick_exec = nullptr;
  int tick_lanes = 0, tick_new = 0;
  int32_t *tick_tok = nullptr, *tick_dep = nullptr;
  EEParams tick_ee{};
  WarmParams tick_warm{};
  bool tick_cascade = false;
  int tick_entry = -1, tick_layout = 0;
  int overlap_mode = 0;   // tl_set_tick_overlap: 0 automatic, 1 entering lanes iterate in the boundary stage, 2 next
                          // tick, 3 boundary stages apart from the loop steps
  int entry_iter = 1;     // resolved for the running decode: 1 = first iteration in the boundary stage
  int layout = 1;         // resolved for the running decode: 1, 2 or 3 as overlap_mode
  // asynchronous stages (layout 3): the loop step's graph on `stream`, the boundary stage's on bstream
  cudaStream_t bstream = nullptr;
  cudaEvent_t b_ev[4] = {nullptr, nullptr, nullptr, nullptr};
  cudaGraphExec_t loop_exec = nullptr, bnd_exec = nullptr;
  int64_t loop_launches = 0, bnd_launches = 0;  // plain kernel nodes of each
  int hold_entered = 0;   // head_finalize keeps continuing lanes claimed (boundary stage of layout 3)
  int64_t tick_launches = 0;
  int64_t tick_loop_kernels = 0;  // plain kernel nodes of a tick graph (outside conditional bodies)
  bool graphs_enabled = true;
  bool pdl = true;  // programmatic dependent launch between consecutive kernels
  int prio = 0;     // launch priority of the next kernels (0: the stream's)
  int prio_hi = 0;  // the device's highest priority: a decode tick's boundary stage
  // host state
  std::vector<int32_t> h_page_table;  // [lanes][slots][pages]
  std::vector<int32_t> refcount;      // per page
  std::vector<int32_t> free_pages;
  std::vector<int32_t> lane_L;        // prefill depth per lane (0 = empty)
  int32_t* pinned_alive = nullptr;    // ring of (alive lanes, loop rows)
  cudaEvent_t alive_ev[4];
  int64_t steps = 0, prefill_tokens = 0, launches = 0, bnd_stages = 0;
  // profiling ring (tl_profile_begin / tl_profile_end)
  int prof_mask = 0;
  std::vector<std::array<cudaEvent_t, 2>> prof_ev;
  std::vector<int> prof_kind_of;
  int64_t prof_head = 0, prof_tail = 0, prof_groups[4] = {0, 0, 0, 0};
  double prof_ms[4] = {0, 0, 0, 0};
};

static constexpr int kAliveRing = 4;
static constexpr int kBRing = 4;  // boundary stages queued at once, at most (layout 3)
static constexpr int kLoopStepsPerGraph = 6;  // layout 3
static constexpr int kProfRing = 4096;

namespace {

// -------------------------------------------------------------- launches ----

int launch_err(tl_ctx* c) {
  c->launches++;
  return check_cuda(cudaGetLastError());
}

// Every kernel of the library goes through here: cudaLaunchKernelEx with
// programmatic stream serialization (each kernel waits for its predecessor
// with griddepcontrol.wait before touching its outputs, and lets its successor
// start its prologue early), unless the context turned that off.
template <typename... KArgs, typename... Args>
int launch_k(tl_ctx* c, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, Args... args) {
  cudaLaunchConfig_t lc{};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = c->stream;
  cudaLaunchAttribute at[2];
  int na = 0;
  if (c->pdl) {
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (c->prio) {
    at[na].id = cudaLaunchAttributePriority;
    at[na].val.priority = c->prio;
    ++na;
  }
  lc.attrs = at;
  lc.numAttrs = na;
  TL_CUDA(cudaLaunchKernelEx(&lc, kern, args...));
  return launch_err(c);
}

// Per-kind device time: event pairs around every launch group of a profiled
// kind, kept in a ring; the host folds in the oldest pair only when the ring is
// full, so timing adds no wait until thousands of groups are in flight.
int prof_fold_oldest(tl_ctx* c) {
  const int i = (int)(c->prof_tail % kProfRing);
  TL_CUDA(cudaEventSynchronize(c->prof_ev[i][1]));
  float ms = 0.f;
  TL_CUDA(cudaEventElapsedTime(&ms, c->prof_ev[i][0], c->prof_ev[i][1]));
  c->prof_ms[c->prof_kind_of[i]] += ms;
  c->prof_tail++;
  return TL_OK;
}

bool prof_on(tl_ctx* c, int kind) { return kind > 0 && kind < 4 && ((c->prof_mask >> kind) & 1); }

int prof_start(tl_ctx* c, int kind) {
  if (!prof_on(c, kind)) return TL_OK;
  if (c->prof_head - c->prof_tail == kProfRing) TL_TRY(prof_fold_oldest(c));
  const int i = (int)(c->prof_head % kProfRing);
  c->prof_kind_of[i] = kind;
  return check_cuda(cudaEventRecord(c->prof_ev[i][0], c->stream));
}

int prof_stop(tl_ctx* c, int kind) {
  if (!prof_on(c, kind)) return TL_OK;
  TL_CUDA(cudaEventRecord(c->prof_ev[c->prof_head % kProfRing][1], c->stream));
  c->prof_head++;
  c->prof_groups[kind]++;
  return TL_OK;
}

// Kernel attributes (shared-memory opt-in) are per device: each launch helper
// keeps one bit per device ordinal (< 64) for "already set on this device".
static int current_device() {
  int dev = 0;
  return (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) ? dev : 0;
}
static bool attr_needed(uint64_t* done_mask) {
  const uint64_t bit = 1ull << current_device();
  if (*done_mask & bit) return false;
  *done_mask |= bit;
  return true;
}

template <int FMT, int EPI, int RPW = 1>
int gemv_launch(tl_ctx* c, const float* X, const int32_t* n_rows, const MatView& W, const MatView& W2,
                const ProjOut& o, int skip_above) {
  const size_t smem = (size_t)8 * W.K * 4;
  auto kern = gemv_kernel<FMT, EPI, RPW>;
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
  }
  if (smem > 200 * 1024) return TL_EINVAL;
  const unsigned grid = (unsigned)((W.N + GEMV_WARPS * RPW - 1) / (GEMV_WARPS * RPW));
  TL_TRY(launch_k(c, kern, dim3(grid), dim3(GEMV_WARPS * 32), smem, X, n_rows, W, W2, o, skip_above));
  return TL_OK;
}

template <int FMT, int EPI>
int gemv_stream_launch(tl_ctx* c, const GsChoice& g, const float* X, const int32_t* n_rows, const MatView& W,
                       const MatView& W2, const ProjOut& o, int skip_above, const GsNorm& nrm) {
  auto kern = gemv_stream_kernel<FMT, EPI>;
  static int attr_smem[64] = {0};  // per instantiation and device: largest opt-in requested so far
  const int dev = current_device();
  if (g.smem > attr_smem[dev]) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, g.smem));
    attr_smem[dev] = g.smem;
  }
  TL_TRY(launch_k(c, kern, dim3(g.grid), dim3(GS_THREADS), g.smem, X, n_rows, W, W2, o, skip_above, g.pl, nrm,
                  c->status));
  return TL_OK;
}

// Few-row projection: the streamed GEMV where its ring fits, else the
// register-blocked CUDA-core GEMV.  nrm (streamed GEMV only): X is the
// residual and the kernel applies the RMSNorm itself.
template <int FMT, int EPI, int RPW>
int small_rows_proj(tl_ctx* c, const float* X, const int32_t* n, const MatView& W, const MatView& W2, ProjOut o,
                    int skip, const GsNorm* nrm) {
  const GsChoice g = gs_plan(FMT, W.N, W.K, W.group, EPI == EPI_SWIGLU ? 2 : 1, c->sc->gs_ctas, c->sc->gs_cap);
  if (g.ok) {
    if (EPI == EPI_ARGMAX) o.n_parts = g.grid;
    return gemv_stream_launch<FMT, EPI>(c, g, X, n, W, W2, o, skip, nrm ? *nrm : GsNorm{});
  }
  if (nrm) return TL_EINVAL;  // callers check gemv_norms_itself first
  if (EPI == EPI_ARGMAX) o.n_parts = (W.N + GEMV_WARPS * RPW - 1) / (GEMV_WARPS * RPW);
  return gemv_launch<FMT, EPI, RPW>(c, X, n, W, W2, o, skip);
}

template <int NT, int NMAT, int FMT, int EPI>
int tc_launch_t(tl_ctx* c, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                const TcParams& p, dim3 grid) {
  using Cf = TcCfg<NT, NMAT, FMT>;
  auto kern = tc_gemm_kernel<NT, NMAT, FMT, EPI>;
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM));
  }
  cudaLaunchConfig_t lc{};
  lc.gridDim = grid;
  lc.blockDim = dim3(256, 1, 1);
  lc.dynamicSmemBytes = Cf::SMEM;
  lc.stream = c->stream;
  cudaLaunchAttribute at[3];
  at[0].id = cudaLaunchAttributeClusterDimension;  // the split-K CTAs of a tile share a cluster
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = grid.z;
  int na = 1;
  if (c->pdl) {
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (c->prio) {
    at[na].id = cudaLaunchAttributePriority;
    at[na].val.priority = c->prio;
    ++na;
  }
  lc.attrs = at;
  lc.numAttrs = na;
  TL_CUDA(cudaLaunchKernelEx(&lc, kern, mw, mw2, mx, p));
  return launch_err(c);
}

template <int NMAT, int FMT, int EPI>
int tc_launch_nt(tl_ctx* c, int nt, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                 const TcParams& p, dim3 grid) {
  if (nt == 64) return tc_launch_t<64, NMAT, FMT, EPI>(c, mw, mw2, mx, p, grid);
  if (nt == 128) return tc_launch_t<128, NMAT, FMT, EPI>(c, mw, mw2, mx, p, grid);
  return tc_launch_t<256, NMAT, FMT, EPI>(c, mw, mw2, mx, p, grid);
}

// Persistent tensor-core projection for many rows (prompt batches).
template <int NMAT, int FMT, int EPI>
int tc_wide_launch(tl_ctx* c, int max_rows, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                   const TcParams& p) {
  using Cf = TcWideCfg<NMAT, FMT>;
  auto kern = tc_gemm_wide_kernel<NMAT, FMT, EPI>;
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM));
  }
  const int64_t tiles = (int64_t)((p.N + 127) / 128) * ((max_rows + Cf::NT - 1) / Cf::NT);
  const int grid = (int)(tiles < c->n_sms ? tiles : c->n_sms);
  return launch_k(c, kern, dim3(grid), dim3(Cf::THREADS), Cf::SMEM, mw, mw2, mx, p);
}

// Rows from which prompt projections take the persistent kernel.
constexpr int kWideRows = 512;

// Tensor-core projection reading the fp16 copy `xsel` of the activations
// (0: norm output, 1: attention output, 2: SwiGLU output).
int tc_proj(tl_ctx* c, int max_rows, int xsel, const int32_t* n, const MatView& W, const CUtensorMap& mw,
            const MatView* W2, const CUtensorMap* mw2, const ProjOut& o, __half* out16, int skip) {
  const int nmat = W2 ? 2 : 1;
  const int nt = tc_nt(max_rows, nmat);
  const int S = o.epi == EPI_ARGMAX ? 1 : tc_splits(W.N, W.K << c->split16, max_rows, nmat, W.fmt, W.group);
  dim3 grid((W.N + 127) / 128, (max_rows + nt - 1) / nt, S);
  TcParams p{};
  p.n_rows = n;
  p.skip_at_or_below = skip;
  p.N = W.N;
  p.K = W.K;
  p.group = W.group;
  p.kb_wrap = W.K / 64;
  p.split16 = c->split16;
  p.kb_per_split = ((W.K / 64) << c->split16) / S;
  p.scales = W.s;
  p.scales2 = W2 ? W2->s : nullptr;
  p.o = o;
  p.out16 = out16;
  p.status = c->status;
  const CUtensorMap& m2 = mw2 ? *mw2 : mw;
  if (max_rows >= kWideRows && o.epi != EPI_ARGMAX) {
    p.kb_per_split = (W.K / 64) << c->split16;
    const CUtensorMap& mxw = c->sc->xmap[xsel][nmat == 1 ? 2 : 1];  // 256-row tiles, 128 for the gate/up pair
    if (W.fmt == FMT_F16) {
      if (o.epi == EPI_SWIGLU) return tc_wide_launch<2, FMT_F16, EPI_SWIGLU>(c, max_rows, mw, m2, mxw, p);
      if (o.epi == EPI_RESID) return tc_wide_launch<1, FMT_F16, EPI_RESID>(c, max_rows, mw, m2, mxw, p);
      return tc_wide_launch<1, FMT_F16, EPI_STORE>(c, max_rows, mw, m2, mxw, p);
    }
    if (W.fmt == TL_FMT_INT4) {
      if (o.epi == EPI_SWIGLU) return tc_wide_launch<2, TL_FMT_INT4, EPI_SWIGLU>(c, max_rows, mw, m2, mxw, p);
      if (o.epi == EPI_RESID) return tc_wide_launch<1, TL_FMT_INT4, EPI_RESID>(c, max_rows, mw, m2, mxw, p);
      return tc_wide_launch<1, TL_FMT_INT4, EPI_STORE>(c, max_rows, mw, m2, mxw, p);
    }
    if (o.epi == EPI_SWIGLU) return tc_wide_launch<2, TL_FMT_BF16, EPI_SWIGLU>(c, max_rows, mw, m2, mxw, p);
    if (o.epi == EPI_RESID) return tc_wide_launch<1, TL_FMT_BF16, EPI_RESID>(c, max_rows, mw, m2, mxw, p);
    return tc_wide_launch<1, TL_FMT_BF16, EPI_STORE>(c, max_rows, mw, m2, mxw, p);
  }
  const CUtensorMap& mx = c->sc->xmap[xsel][nt == 64 ? 0 : (nt == 128 ? 1 : 2)];
  if (W.fmt == FMT_F16) {  // (block matrices only: the head keeps its own format)
    if (o.epi == EPI_ARGMAX) return TL_EINVAL;
    if (o.epi == EPI_SWIGLU) return tc_launch_nt<2, FMT_F16, EPI_SWIGLU>(c, nt, mw, m2, mx, p, grid);
    if (o.epi == EPI_RESID) return tc_launch_nt<1, FMT_F16, EPI_RESID>(c, nt, mw, m2, mx, p, grid);
    return tc_launch_nt<1, FMT_F16, EPI_STORE>(c, nt, mw, m2, mx, p, grid);
  }
  if (W.fmt == TL_FMT_INT4) {
    if (o.epi == EPI_ARGMAX) return tc_launch_nt<1, TL_FMT_INT4, EPI_ARGMAX>(c, nt, mw, m2, mx, p, grid);
    if (o.epi == EPI_SWIGLU) return tc_launch_nt<2, TL_FMT_INT4, EPI_SWIGLU>(c, nt, mw, m2, mx, p, grid);
    if (o.epi == EPI_RESID) return tc_launch_nt<1, TL_FMT_INT4, EPI_RESID>(c, nt, mw, m2, mx, p, grid);
    return tc_launch_nt<1, TL_FMT_INT4, EPI_STORE>(c, nt, mw, m2, mx, p, grid);
  }
  if (o.epi == EPI_ARGMAX) return tc_launch_nt<1, TL_FMT_BF16, EPI_ARGMAX>(c, nt, mw, m2, mx, p, grid);
  if (o.epi == EPI_SWIGLU) return tc_launch_nt<2, TL_FMT_BF16, EPI_SWIGLU>(c, nt, mw, m2, mx, p, grid);
  if (o.epi == EPI_RESID) return tc_launch_nt<1, TL_FMT_BF16, EPI_RESID>(c, nt, mw, m2, mx, p, grid);
  return tc_launch_nt<1, TL_FMT_BF16, EPI_STORE>(c, nt, mw, m2, mx, p, grid);
}

// Projection over the device-side row count: the CUDA-core GEMV takes up to 8
// rows (exact fp32 weights and activations); larger counts go to the tensor
// cores.  PATH_AUTO (only an upper bound known on the host): both are launched
// and the one that does not apply returns at once.  PATH_GEMV / PATH_TC: the
// caller knows which applies (prompts, or a graph branch chosen on the
// device), and only that one is launched.  nrm: see small_rows_proj (the
// tensor-core variant reads the fp16 copy of a separate norm kernel).
// tw (optional): the matrices and maps the tensor-core variant reads instead (a BF16 block's resident
// fp16 copy; the GEMV keeps the exact BF16 weights).
struct TcTwin {
  const MatView* W;
  const CUtensorMap* mw;
  const MatView* W2;
  const CUtensorMap* mw2;
};

int proj(tl_ctx* c, int max_rows, int path, const float* X, int xsel, const int32_t* n, const MatView& W,
         const CUtensorMap* mw, const MatView* W2, const CUtensorMap* mw2, ProjOut o, __half* out16,
         int prof_kind = TL_PROF_PROJ, const GsNorm* nrm = nullptr, const TcTwin* tw = nullptr) {
  const MatView& w2 = W2 ? *W2 : W;
  TL_TRY(prof_start(c, prof_kind));
  const bool argmax = o.epi == EPI_ARGMAX;
  const bool use_tc = max_rows > kGemvMaxRows && path != PATH_GEMV;
  const bool use_gemv = !use_tc || path == PATH_AUTO;
  if (use_gemv) {
    const int skip = use_tc ? kGemvMaxRows : 0;
    int st;
    if (W.fmt == TL_FMT_INT4) {
      switch (o.epi) {
        case EPI_STORE: st = small_rows_proj<TL_FMT_INT4, EPI_STORE, 1>(c, X, n, W, w2, o, skip, nrm); break;
        case EPI_RESID: st = small_rows_proj<TL_FMT_INT4, EPI_RESID, 1>(c, X, n, W, w2, o, skip, nrm); break;
        case EPI_SWIGLU: st = small_rows_proj<TL_FMT_INT4, EPI_SWIGLU, 1>(c, X, n, W, w2, o, skip, nrm); break;
        default: st = small_rows_proj<TL_FMT_INT4, EPI_ARGMAX, head_rpw(TL_FMT_INT4)>(c, X, n, W, w2, o, skip, nrm); break;
      }
    } else {
      switch (o.epi) {
        case EPI_STORE: st = small_rows_proj<TL_FMT_BF16, EPI_STORE, 1>(c, X, n, W, w2, o, skip, nrm); break;
        case EPI_RESID: st = small_rows_proj<TL_FMT_BF16, EPI_RESID, 1>(c, X, n, W, w2, o, skip, nrm); break;
        case EPI_SWIGLU: st = small_rows_proj<TL_FMT_BF16, EPI_SWIGLU, 1>(c, X, n, W, w2, o, skip, nrm); break;
        default: st = small_rows_proj<TL_FMT_BF16, EPI_ARGMAX, head_rpw(TL_FMT_BF16)>(c, X, n, W, w2, o, skip, nrm); break;
      }
    }
    TL_TRY(st);
  }
  if (use_tc) {
    if (argmax) o.n_parts = (W.N + 127) / 128;  // one partial per 128-row tile
    if (tw)
      TL_TRY(tc_proj(c, max_rows, xsel, n, *tw->W, *tw->mw, tw->W2, tw->mw2, o, out16,
                     path == PATH_AUTO ? kGemvMaxRows : 0));
    else
      TL_TRY(tc_proj(c, max_rows, xsel, n, W, *mw, W2, mw2, o, out16, path == PATH_AUTO ? kGemvMaxRows : 0));
  }
  return prof_stop(c, prof_kind);
}

template <int HD>
int attn_tc_launch(tl_ctx* c, const AttnTcParams& p, dim3 grid) {
  auto kern = attn_tc_kernel<HD>;
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnTcCfg<HD>::SMEM));
  }
  return launch_k(c, kern, grid, dim3(256), (size_t)AttnTcCfg<HD>::SMEM, c->kvmap, p);
}

template <int HD>
int attn_launch_t(tl_ctx* c, const Rows& rows, int slot_base, int slot_stride, bool cascade) {
  auto kern = attn_decode_kernel<HD>;
  const int smem = attn_smem_bytes<HD>(c->cfg.max_lanes);
  static int attr_smem[64] = {0};  // per instantiation and device: largest opt-in requested so far
  const int dev = current_device();
  if (smem > attr_smem[dev]) {
    TL_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    attr_smem[dev] = smem;
  }
  return launch_k(c, kern, dim3(c->n_sms), dim3(AttnCfg<HD>::WARPS * 32), (size_t)smem, c->kvmap,
                  (const float*)c->sc->act_qkv, c->sc->act_o, c->sc->act_o16, rows, c->kv, (const float2*)c->rope, slot_base,
                  slot_stride, c->sc->attn_part, c->sc->attn_counters, c->status,
                  cascade ? (const int32_t*)c->lane_shared : (const int32_t*)nullptr, (const float*)c->sc->casc,
                  c->split16);
}

// Shared-prefix ("cascade") pass of a decode step: for every loop iteration
// value, all rows whose lanes map the shared prefix attend to it together on
// the tensor cores, 128 rows per CTA; partials go to c->sc->casc.
int cascade_launch(tl_ctx* c, int max_rows, const Rows& rows, int slot_base, int slot_stride) {
  AttnTcParams p{};
  p.q = c->sc->act_qkv;
  p.rope = c->rope;
  p.rows = rows;
  p.mode = 1;
  p.lane_shared = c->lane_shared;
  p.chunks = (max_rows + 127) / 128;
  p.casc = c->sc->casc;
  p.g = c->kv;
  p.slot_base = slot_base;
  p.slot_stride = slot_stride;
  p.status = c->status;
  const int groups = slot_stride > 0 ? c->cfg.L_max : 1;
  const dim3 grid(groups * p.chunks, c->cfg.n_heads);
  return c->hd == 64 ? attn_tc_launch<64>(c, p, grid) : attn_tc_launch<128>(c, p, grid);
}

// Decode attention (one query row per (row, head)) over the rows of `rows`.
// Decode attention over the rows of `rows`.  Steps with a shared-prefix
// cascade take the balanced persistent kernel (which merges the cascade's
// partials); the others the split-context kernel, whose small CTAs measured
// faster around the neighbouring projections in CUDA-graph ticks (64 lanes:
// 346 against 358 ms per decode pass; one lane at L = 8: 1,609 against 1,516
// tokens/s), with the same per-kind kernel time.
template <int HD>
int attn_split_launch(tl_ctx* c, dim3 grid, const Rows& rows, int slot_base, int slot_stride) {
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(attn_split_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kAttnSplitSmem<HD>));
  }
  return launch_k(c, attn_split_kernel<HD>, grid, dim3(128), kAttnSplitSmem<HD>, (const float*)c->sc->act_qkv,
                  c->sc->act_o, c->sc->act_o16, rows, c->kv, (const float2*)c->rope, slot_base, slot_stride,
                  c->sc->attn_part, c->sc->attn_counters, c->status, c->split16);
}

int attn_launch(tl_ctx* c, int max_rows, const Rows& rows, int slot_base, int slot_stride) {
  TL_TRY(prof_start(c, TL_PROF_ATTN));
  const bool cascade = c->cascade_active && c->hd >= 64;
  int st;
  if (cascade) {
    TL_TRY(cascade_launch(c, max_rows, rows, slot_base, slot_stride));
    st = c->hd == 64 ? attn_launch_t<64>(c, rows, slot_base, slot_stride, true)
                     : attn_launch_t<128>(c, rows, slot_base, slot_stride, true);
  } else {
    int ks = (kAttnCtaTarget + max_rows * c->cfg.n_heads - 1) / (max_rows * c->cfg.n_heads);
    ks = ks < 1 ? 1 : (ks > kAttnPieces ? kAttnPieces : ks);
    if (max_rows > 1) ks = ks < 4 ? 4 : ks;
    const dim3 grid(max_rows, c->cfg.n_heads, ks);
    switch (c->hd) {
      case 32: st = attn_split_launch<32>(c, grid, rows, slot_base, slot_stride); break;
      case 64: st = attn_split_launch<64>(c, grid, rows, slot_base, slot_stride); break;
      default: st = attn_split_launch<128>(c, grid, rows, slot_base, slot_stride); break;
    }
  }
  TL_TRY(st);
  return prof_stop(c, TL_PROF_ATTN);
}

// Causal attention over a prompt block (rows of one lane, consecutive positions).
template <int HD>
int attn_prefill_launch_hd(tl_ctx* c, int max_rows, const Rows& rows, int slot, const int2* tiles, int n_tiles) {
  const size_t smem = (size_t)(3 * HD * 64 + 64 * 65) * 4;
  static uint64_t attr_done = 0;  // per instantiation: one bit per device
  if (attr_needed(&attr_done)) {
    TL_CUDA(cudaFuncSetAttribute(attn_prefill_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  }
  dim3 grid(tiles ? n_tiles : (max_rows + 63) / 64, c->cfg.n_heads);
  TL_TRY(launch_k(c, attn_prefill_kernel<HD>, dim3(grid), dim3(256), smem, c->sc->act_q, c->sc->act_o, c->sc->act_o16, rows,
                  tiles, c->kv, slot, c->status, c->split16));
  return TL_OK;
}

// Prompt rows per attention tile: 128 for the tensor-core kernel (head widths 64 and 128), 64 otherwise.
int prompt_tile_rows(const tl_ctx* c) { return c->hd >= 64 ? 128 : 64; }

int attn_prefill_launch(tl_ctx* c, int max_rows, const Rows& rows, int slot, const int2* tiles, int n_tiles) {
  TL_TRY(prof_start(c, TL_PROF_ATTN));
  int st;
  if (c->hd >= 64 && tiles) {  // tensor cores: 128-row tiles (prompt_tile_rows)
    AttnTcParams p{};
    p.q = c->sc->act_q;
    p.rope = c->rope;
    p.rows = rows;
    p.tiles = tiles;
    p.mode = 0;
    p.o = c->sc->act_o;
    p.o16 = c->sc->act_o16;
    p.split16 = c->split16;
    p.g = c->kv;
    p.slot_base = slot;
    p.slot_stride = 0;
    p.status = c->status;
    const dim3 grid(n_tiles, c->cfg.n_heads);
    st = c->hd == 64 ? attn_tc_launch<64>(c, p, grid) : attn_tc_launch<128>(c, p, grid);
  } else {
    switch (c->hd) {
      case 32: st = attn_prefill_launch_hd<32>(c, max_rows, rows, slot, tiles, n_tiles); break;
      case 64: st = attn_prefill_launch_hd<64>(c, max_rows, rows, slot, tiles, n_tiles); break;
      default: st = attn_prefill_launch_hd<128>(c, max_rows, rows, slot, tiles, n_tiles); break;
    }
  }
  TL_TRY(st);
  return prof_stop(c, TL_PROF_ATTN);
}

// Whether the few-row GEMV for W (nmat matrices) applies the RMSNorm in its
// own activation staging (the streamed GEMV does; its fallback does not).
bool gemv_norms_itself(tl_ctx* c, const MatView& W, int nmat) {
  return gs_plan(W.fmt, W.N, W.K, W.group, nmat, c->sc->gs_ctas, c->sc->gs_cap).ok;
}

// RMSNorm(hbuf rows) * g feeding a projection of W on `path`.  Returns the
// GEMV's activation source and norm arguments; launches the separate norm
// kernel (fp32 act_a + fp16 act_a16, and the h_in copy) only where a
// projection that needs it can run: the tensor-core variant (more than 8 rows)
// or a GEMV that does not normalise itself.
// A prompt projection's residual left for the next norm kernel to add: h[row
// r] += add[r] for r < *n (at most `rows` rows).
struct PendingAdd {
  const float* add = nullptr;
  const int32_t* n = nullptr;
  int rows = 0;
};

int norm_for_proj(tl_ctx* c, int max_rows, int path, const int32_t* n, float* hbuf, const int32_t* map,
                  const float* g, float* h_in, const MatView& W, int nmat, const float** X, GsNorm* nrm,
                  bool* use_nrm, const PendingAdd& pend = PendingAdd{}) {
  const bool fused = path != PATH_TC && gemv_norms_itself(c, W, nmat) && !pend.add;
  const bool tc_possible = path != PATH_GEMV && max_rows > kGemvMaxRows;
  *use_nrm = fused;
  *nrm = GsNorm{g, map, c->cfg.rms_eps, h_in};
  *X = fused ? hbuf : c->sc->act_a;
  if (!fused || tc_possible) {
    const int min_rows = (fused && path == PATH_AUTO) ? kGemvMaxRows : 0;  // <= 8 rows: the GEMV normalises
    const int grid = pend.rows > max_rows ? pend.rows : max_rows;
    TL_TRY(launch_k(c, rmsnorm_rows_kernel, dim3(grid), dim3(256), 0, hbuf, map, n, c->cfg.d, g, c->cfg.rms_eps,
                    c->sc->act_a, h_in, c->sc->act_a16, nullptr, 0, min_rows, pend.add, pend.n, c->split16));
  }
  return TL_OK;
}

// One transformer block on the rows of `rows`; hidden rows live in hbuf
// (indexed through map, or by row when map is null).
// prompt = rows are runs of consecutive positions of one lane each, attended
// causally in the n_tiles tiles of `tiles`.
// Prompt batches (pend != null): the residual projections of blocks wide
// enough for the persistent kernel store their output (in act_q, free after
// attention) instead of adding it into hbuf, and the next norm kernel adds it
// (the norm after the attention, then the next block's first norm, or the
// caller after the last block, from *pend).
int run_block(tl_ctx* c, const Rows& rows, int max_rows, float* hbuf, const int32_t* map, const BlockW& w,
              int slot_base, int slot_stride, float* h_in, bool prompt = false, int path = PATH_AUTO,
              const int2* tiles = nullptr, int n_tiles = 0, PendingAdd* pend = nullptr) {
  if (prompt) path = max_rows > kGemvMaxRows ? PATH_TC : PATH_GEMV;
  const int d = c->cfg.d, F = c->cfg.ffn;
  const bool defer = pend && prompt && max_rows >= kWideRows;
  const BlockW& pw = w;  // the GEMV's matrices; the tensor-core variants read the block's resident fp16 copy
  const BlockW* tb = w.f16;
  const TcTwin t_qkv{tb ? &tb->wqkv : nullptr, tb ? &tb->mqkv : nullptr, nullptr, nullptr};
  const TcTwin t_o{tb ? &tb->wo : nullptr, tb ? &tb->mo : nullptr, nullptr, nullptr};
  const TcTwin t_gu{tb ? &tb->wg : nullptr, tb ? &tb->mg : nullptr, tb ? &tb->wu : nullptr, tb ? &tb->mu : nullptr};
  const TcTwin t_d{tb ? &tb->wd : nullptr, tb ? &tb->md : nullptr, nullptr, nullptr};
  const float* X = nullptr;
  GsNorm nrm{};
  bool use_nrm = false;
  TL_TRY(norm_for_proj(c, max_rows, path, rows.n, hbuf, map, w.g1, h_in, w.wqkv, 1, &X, &nrm, &use_nrm,
                       pend ? *pend : PendingAdd{}));
  if (pend) *pend = PendingAdd{};
  ProjOut o{};
  o.epi = EPI_STORE;
  o.out = c->sc->act_qkv;
  o.ldo = 3 * d;
  TL_TRY(proj(c, max_rows, path, X, 0, rows.n, pw.wqkv, &pw.mqkv, nullptr, nullptr, o, nullptr, TL_PROF_PROJ,
              use_nrm ? &nrm : nullptr, tb ? &t_qkv : nullptr));
  if (prompt) {
    TL_TRY(launch_k(c, rope_kv_kernel, dim3(max_rows), dim3(d / 2), 0, c->sc->act_qkv, c->sc->act_q, rows, c->kv, c->rope,
                    slot_base, slot_stride, nullptr, c->status));
    TL_TRY(attn_prefill_launch(c, max_rows, rows, slot_base, tiles, n_tiles));
  } else {
    TL_TRY(attn_launch(c, max_rows, rows, slot_base, slot_stride));  // RoPE and the KV append run inside
  }
  ProjOut r{};
  r.epi = EPI_RESID;
  r.h = hbuf;
  r.map = map;
  if (defer) {  // stored, added by the next norm
    r.epi = EPI_STORE;
    r.out = c->sc->act_q;
    r.ldo = d;
  }
  TL_TRY(proj(c, max_rows, path, c->sc->act_o, 1, rows.n, pw.wo, &pw.mo, nullptr, nullptr, r, nullptr, TL_PROF_PROJ,
              nullptr, tb ? &t_o : nullptr));
  TL_TRY(norm_for_proj(c, max_rows, path, rows.n, hbuf, map, w.g2, nullptr, w.wg, 2, &X, &nrm, &use_nrm,
                       defer ? PendingAdd{c->sc->act_q, rows.n, max_rows} : PendingAdd{}));
  ProjOut sw{};
  sw.epi = EPI_SWIGLU;
  // only the tensor-core variant runs here: the down projection reads the fp16 copy alone
  sw.out = (path == PATH_TC && max_rows > kGemvMaxRows) ? nullptr : c->sc->act_u;
  sw.ldo = F;
  TL_TRY(proj(c, max_rows, path, X, 0, rows.n, pw.wg, &pw.mg, &pw.wu, &pw.mu, sw, c->sc->act_u16, TL_PROF_PROJ,
              use_nrm ? &nrm : nullptr, tb ? &t_gu : nullptr));
  TL_TRY(proj(c, max_rows, path, c->sc->act_u, 2, rows.n, pw.wd, &pw.md, nullptr, nullptr, r, nullptr, TL_PROF_PROJ,
              nullptr, tb ? &t_d : nullptr));
  if (defer) *pend = PendingAdd{c->sc->act_q, rows.n, max_rows};
  return TL_OK;
}

// Row table `which` from lanes 0..n_consider-1 (all lanes when n_consider <= 0);
// optionally sets a conditional graph node's value from the row count.
int build_rows(tl_ctx* c, int which, int sel, const uint8_t* mask, const int32_t* per_lane_L, uint8_t* exit_mask,
               int32_t* alive, int n_consider = 0, cudaGraphConditionalHandle cond = 0, int cond_mode = COND_NONE,
               const int32_t* body_kernels = nullptr) {
  const int n = n_consider > 0 ? n_consider : c->cfg.max_lanes;
  TL_TRY(launch_k(c, build_rows_kernel, dim3(1), dim3(1024), 0, c->lanes, n, sel, mask, per_lane_L, c->rows[which], exit_mask,
                                               alive, c->status, cond, cond_mode, kGemvMaxRows, body_kernels,
                                               &c->counters[2]));
  return TL_OK;
}

// Logit-margin probes ("CLI Reference", --early-exit-logit-margin: a head
// projection per peek): the loop rows whose iteration is a probe go into
// rows[4]; the final norm and the head (the boundary stage's kernels) write
// their logits, and margin_kernel reduces each to its top-1 minus top-2.  The
// probe count is known only on the device, so unless the loop rows fit the
// GEMV (then so do the probes) both head variants are launched and the one
// that does not apply returns at once.
int probe_head(tl_ctx* c, int max_rows, int path, const Rows& loop_rows) {
  const Rows& P = c->sc->probe;
  TL_TRY(launch_k(c, probe_rows_kernel, dim3(1), dim3(1024), 0, loop_rows, (const LaneState*)c->lanes, c->ee, P));
  const int ppath = path == PATH_GEMV ? PATH_GEMV : PATH_AUTO;
  const float* X = nullptr;
  GsNorm nrm{};
  bool use_nrm = false;
  TL_TRY(norm_for_proj(c, max_rows, ppath, P.n, c->h, P.lane, c->g_final, nullptr, c->head, 1, &X, &nrm, &use_nrm));
  ProjOut o{};
  o.epi = EPI_ARGMAX;
  o.logits = c->probe_logits;
  o.lmap = P.lane;
  o.ldo = c->cfg.vocab;
  o.part_val = c->sc->part_val;
  o.part_idx = c->sc->part_idx;
  o.n_parts_dev = c->sc->head_nparts;
  TL_TRY(proj(c, max_rows, ppath, X, 0, P.n, c->head, &c->mhead, nullptr, nullptr, o, nullptr, TL_PROF_HEAD,
              use_nrm ? &nrm : nullptr));
  return launch_k(c, margin_kernel, dim3(max_rows), dim3(256), 0, P, (const float*)c->probe_logits, c->cfg.vocab,
                  c->margin_lane);
}

// Projection path of a decode's loop steps when both variants would be
// launched (plain graph nodes, individual launches): a decode wider than 8
// lanes runs them on the tensor cores whatever the step's row count.  The GEMV
// variant launched beside them (returning at once above 8 rows) still held its
// SMs' shared memory while it waited for its predecessor: 64 lanes measured
// 36.0k against 42.0k tokens/s.  It also makes a row's projections independent
// of how many rows share its step.
static int loop_path(int n_lanes) { return n_lanes > kGemvMaxRows ? PATH_TC : PATH_AUTO; }

// One loop iteration for the lanes selected into rows[table] (0: the loop
// table; 2: the lanes entering at a decode tick's boundary stage).
int loop_iteration(tl_ctx* c, int max_rows, uint8_t* exit_mask, int path = PATH_AUTO, int table = 0) {
  const Rows& R = c->rows[table];
  const int Lb = c->cfg.n_loop_layers;
  for (int m = 0; m < Lb; ++m)
    TL_TRY(run_block(c, R, max_rows, c->h, R.lane, c->loop[m], c->cfg.n_pre + m, Lb, m == 0 ? c->h_in : nullptr,
                     false, path));
  if (c->ee.enabled && c->ee.use_margin) TL_TRY(probe_head(c, max_rows, path, R));
  TL_TRY(launch_k(c, exit_update_kernel, dim3(max_rows), dim3(256), 0, R, c->lanes, (const float*)c->h,
                  (const float*)c->h_in, c->cfg.d, c->ee, exit_mask, &c->counters[0], c->warm, c->kv, c->cfg.n_pre,
                  c->cfg.n_loop_layers, c->status, (const float*)c->margin_lane));
  c->steps++;
  return TL_OK;
}

// Pre blocks for the lanes in rows[2] (lanes that just took a token).
int pre_blocks(tl_ctx* c, int max_rows, int path = PATH_AUTO) {
  const Rows& E = c->rows[2];
  for (int b = 0; b < c->cfg.n_pre; ++b)
    TL_TRY(run_block(c, E, max_rows, c->h, E.lane, c->pre[b], b, 0, nullptr, false, path));
  return TL_OK;
}

int pre_blocks_for_entered(tl_ctx* c, int max_rows) {
  TL_TRY(build_rows(c, 2, SEL_ENTERED, nullptr, nullptr, nullptr, nullptr, max_rows));
  return pre_blocks(c, max_rows);
}

// Boundary stage, head part, for the lanes in rows[1]: final norm, head,
// argmax, and in decode mode the token bookkeeping and embedding.
int head_core(tl_ctx* c, int max_rows, int mode, float* logits, int32_t* argmax, int32_t* tok_out, int32_t* dep_out,
              int n_new, int path = PATH_AUTO, int mark_entered = 1) {
  const Rows& B = c->rows[1];
  const float* X = nullptr;
  GsNorm nrm{};
  bool use_nrm = false;
  TL_TRY(norm_for_proj(c, max_rows, path, B.n, c->h, B.lane, c->g_final, nullptr, c->head, 1, &X, &nrm, &use_nrm));
  ProjOut o{};
  o.epi = EPI_ARGMAX;
  o.logits = logits;
  o.lmap = B.lane;
  o.ldo = c->cfg.vocab;
  o.part_val = c->sc->part_val;
  o.part_idx = c->sc->part_idx;
  o.n_parts_dev = c->sc->head_nparts;
  TL_TRY(proj(c, max_rows, path, X, 0, B.n, c->head, &c->mhead, nullptr, nullptr, o, nullptr, TL_PROF_HEAD,
              use_nrm ? &nrm : nullptr));
  TL_TRY(launch_k(c, head_finalize_kernel, dim3(max_rows), dim3(256), 0, B, c->lanes, c->sc->part_val, c->sc->part_idx, c->sc->head_nparts, mode,
                                                        argmax, tok_out, dep_out, n_new, c->embed, c->h, c->cfg.d,
                                                        c->cfg.max_seq, mark_entered, c->status, &c->counters[1],
                                                        c->warm, (int32_t)c->hold_entered));
  return TL_OK;
}

// Whole boundary stage: head, then (decode mode) pre blocks for the lanes that took a token.
int head_stage(tl_ctx* c, int max_rows, int mode, float* logits, int32_t* argmax, int32_t* tok_out,
               int32_t* dep_out, int n_new) {
  TL_TRY(head_core(c, max_rows, mode, logits, argmax, tok_out, dep_out, n_new));
  if (mode == HEAD_DECODE) return pre_blocks_for_entered(c, max_rows);
  return TL_OK;
}

// ------------------------------------------------------------ KV pages ----

void release_lane_pages(tl_ctx* c, int lane) {
  const int per_lane = c->lay.n_slots * c->lay.pages_per_seq;
  int32_t* t = &c->h_page_table[(size_t)lane * per_lane];
  for (int i = 0; i < per_lane; ++i) {
    if (t[i] >= 0 && --c->refcount[t[i]] == 0) c->free_pages.push_back(t[i]);
    t[i] = -1;
  }
  c->lane_L[lane] = 0;
  c->h_lane_shared[lane] = 0;
  c->h_lane_donor[lane] = -1;
}

// Shared-prefix attention runs as a cascade when enabled and every lane that
// maps shared pages maps the same donor's prefix of the same length (the
// tensor-core pass reads one page list per loop iteration).  Copies the
// per-lane lengths to the device.
int update_cascade(tl_ctx* c) {
  int donor = -1, len = 0;
  bool one = true, any = false;
  for (int i = 0; i < c->cfg.max_lanes; ++i) {
    if (c->h_lane_shared[i] == 0) continue;
    if (!any) {
      donor = c->h_lane_donor[i];
      len = c->h_lane_shared[i];
      any = true;
    } else if (c->h_lane_donor[i] != donor || c->h_lane_shared[i] != len) {
      one = false;
    }
  }
  c->cascade_active = c->cascade_enabled && any && one && c->hd >= 64;
  return check_cuda(cudaMemcpyAsync(c->lane_shared, c->h_lane_shared.data(), (size_t)c->cfg.max_lanes * 4,
                                    cudaMemcpyHostToDevice, c->stream));
}

// --------------------------------------------------------- tensor maps ----

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major 2D map: `inner` elements per row, `outer` rows, row pitch in bytes.
int encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = tensor_map_encoder();
  if (!fn) {
    g_cuda_err = "cuTensorMapEncodeTiled entry point unavailable";
    return TL_ECUDA;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_cuda_err = "cuTensorMapEncodeTiled failed";
    return TL_ECUDA;
  }
  return TL_OK;
}

// Raw weight tiles: INT4 128 rows x 32 bytes, BF16 128 rows x 64 elements; unswizzled.
int encode_weight_map(CUtensorMap* m, const MatView& W) {
  if (W.fmt == TL_FMT_INT4)
    return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.q, (uint64_t)W.K / 2, (uint64_t)W.N, (uint64_t)W.K / 2, 32,
                     128, CU_TENSOR_MAP_SWIZZLE_NONE);
  return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, W.bf, (uint64_t)W.K, (uint64_t)W.N, (uint64_t)W.K * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

int encode_all_maps(tl_ctx* c) {
  for (auto* v : {&c->pre, &c->loop})
    for (BlockW& b : *v) {
      TL_TRY(encode_weight_map(&b.mqkv, b.wqkv));
      TL_TRY(encode_weight_map(&b.mo, b.wo));
      TL_TRY(encode_weight_map(&b.mg, b.wg));
      TL_TRY(encode_weight_map(&b.mu, b.wu));
      TL_TRY(encode_weight_map(&b.md, b.wd));
    }
  TL_TRY(encode_weight_map(&c->mhead, c->head));
  for (BlockW& b : c->blk16) {  // fp16 tiles of 128 rows x 64 K, in the MMA's swizzled layout
    const MatView* mv5[5] = {&b.wqkv, &b.wo, &b.wg, &b.wu, &b.wd};
    CUtensorMap* mp5[5] = {&b.mqkv, &b.mo, &b.mg, &b.mu, &b.md};
    for (int i = 0; i < 5; ++i)
      TL_TRY(encode_2d(mp5[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, mv5[i]->bf, (uint64_t)mv5[i]->K, (uint64_t)mv5[i]->N,
                       (uint64_t)mv5[i]->K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
  }
  {  // KV pool as rows of hd fp16: a page is [K: H x P rows][V: H x P rows]
    const uint64_t pool_rows = (uint64_t)c->lay.n_pages * 2 * c->cfg.n_heads * c->cfg.kv_page_tokens;
    const uint32_t cols = c->hd > 64 ? 64 : (uint32_t)c->hd;
    TL_TRY(encode_2d(&c->kvmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c->kv.pool, (uint64_t)c->hd, pool_rows,
                     (uint64_t)c->hd * 2, cols, (uint32_t)kAttnUK,
                     cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B));
  }
  for (Scratch& sc : c->scr) {
    const __half* xs[3] = {sc.act_a16, sc.act_o16, sc.act_u16};
    const int ks[3] = {c->cfg.d, c->cfg.d, c->cfg.ffn};
    const int nts[3] = {64, 128, 256};
    for (int x = 0; x < 3; ++x)
      for (int i = 0; i < 3; ++i)
        TL_TRY(encode_2d(&sc.xmap[x][i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xs[x], (uint64_t)ks[x] << c->split16,
                         (uint64_t)sc.rows, ((uint64_t)ks[x] << c->split16) * 2, 64, nts[i],
                         CU_TENSOR_MAP_SWIZZLE_128B));
  }
  return TL_OK;
}

}  // namespace

// ============================================================== C ABI ====

extern "C" int tl_workspace_bytes(const tl_config* cfg, size_t* out) {
  if (!cfg_valid(cfg) || !out) return TL_EINVAL;
  const Layout lay = make_layout(cfg);
  if (!kv_rows_ok(cfg, lay.n_pages)) return TL_EINVAL;
  *out = lay.total;
  return TL_OK;
}

extern "C" int tl_weights_bytes(const tl_config* cfg, size_t* out) {
  if (!cfg_valid(cfg) || !out) return TL_EINVAL;
  *out = blob_bytes(cfg);
  return TL_OK;
}

extern "C" const char* tl_strerror(int s) {
  switch (s) {
    case TL_OK: return "ok";
    case TL_EINVAL: return "invalid argument";
    case TL_ENOMEM: return "out of memory (workspace or KV page pool)";
    case TL_ESTATE: return "invalid state for this call";
    case TL_EKV: return "requested depth exceeds the lane's KV cache";
    case TL_ECUDA: return "CUDA error";
    case TL_ETIMEOUT: return "device wait timed out";
    case TL_EDEVICE: return "device reported an out-of-range index";
    default: return "unknown status";
  }
}

extern "C" const char* tl_last_cuda_error(void) { return g_cuda_err.c_str(); }

__global__ void rope_table_kernel(float2* t, int max_seq, int half, double base) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)max_seq * half) return;
  const int p = (int)(i / half), k = (int)(i % half);
  const double theta = pow(base, -2.0 * k / (2.0 * half));
  double s, co;
  sincos((double)p * theta, &s, &co);
  t[i] = make_float2((float)co, (float)s);
}

__global__ void lanes_init_kernel(LaneState* l, int n) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    LaneState z{};
    z.phase = PH_IDLE;
    z.token = -1;
    l[i] = z;
  }
}

extern "C" int tl_create(const tl_config* cfg, void* dev_ws, size_t bytes, void* stream, tl_ctx** out) {
  if (!cfg_valid(cfg) || !dev_ws || !out || ((uintptr_t)dev_ws & 255)) return TL_EINVAL;
  Layout lay = make_layout(cfg);
  if (!kv_rows_ok(cfg, lay.n_pages)) return TL_EINVAL;
  if (bytes < lay.total) return TL_ENOMEM;
  tl_ctx* c = new tl_ctx();
  c->sc = &c->scr[0];
  c->cfg = *cfg;
  c->lay = lay;
  c->stream = (cudaStream_t)stream;
  c->ws = (char*)dev_ws;
  c->ws_bytes = bytes;
  c->hd = cfg->d / cfg->n_heads;
  c->split16 = act_split_on(cfg);
  if (const char* e = std::getenv("TL_PDL")) c->pdl = std::strcmp(e, "0") != 0;
  char* w = c->ws;
  // weight views
  auto specs = mat_specs(cfg);
  std::vector<MatView> mv;
  for (size_t i = 0; i < specs.size(); ++i) {
    MatView m{};
    m.fmt = specs[i].fmt;
    m.N = (int)specs[i].N;
    m.K = (int)specs[i].K;
    m.group = cfg->group;
    char* p = w + lay.mat_off[i];
    if (m.fmt == TL_FMT_INT4) {
      m.q = (const uint8_t*)p;
      m.s = (const __half*)(p + (size_t)m.N * m.K / 2);
    } else {
      m.bf = (const uint16_t*)p;
    }
    mv.push_back(m);
  }
  const float* gains = (const float*)(w + lay.gains);
  c->embed = mv[0];
  c->head = mv.back();
  const int nb = cfg->n_pre + cfg->n_loop_layers;
  for (int b = 0; b < nb; ++b) {
    BlockW bw{mv[1 + 5 * b], mv[2 + 5 * b], mv[3 + 5 * b], mv[4 + 5 * b], mv[5 + 5 * b],
              gains + (size_t)(2 * b) * cfg->d, gains + (size_t)(2 * b + 1) * cfg->d};
    (b < cfg->n_pre ? c->pre : c->loop).push_back(bw);
  }
  {  // resident fp16 copies of the blocks, in block order (filled by tl_load_weights)
    const int64_t d = cfg->d, F = cfg->ffn;
    const int64_t off[5] = {0, 3 * d * d, 4 * d * d, 4 * d * d + F * d, 4 * d * d + 2 * F * d};
    const int64_t NN[5] = {3 * d, d, F, F, d}, KK[5] = {d, d, d, d, F};
    c->blk16.reserve(nb);  // (BlockW::f16 points into it)
    __half* base = (__half*)(w + lay.f16blk);
    for (int b = 0; b < nb; ++b) {
      BlockW& src = b < cfg->n_pre ? c->pre[b] : c->loop[b - cfg->n_pre];
      BlockW cp = src;
      MatView* mv5[5] = {&cp.wqkv, &cp.wo, &cp.wg, &cp.wu, &cp.wd};
      for (int i = 0; i < 5; ++i) {
        mv5[i]->fmt = FMT_F16;
        mv5[i]->N = (int)NN[i];
        mv5[i]->K = (int)KK[i];
        mv5[i]->bf = reinterpret_cast<const uint16_t*>(base + off[i]);
      }
      base += 4 * d * d + 3 * d * F;
      c->blk16.push_back(cp);
      src.f16 = &c->blk16.back();
    }
  }
  c->g_final = gains + (size_t)(2 * nb) * cfg->d;
  c->rope = (float2*)(w + lay.rope);
  c->page_table = (int32_t*)(w + lay.page_table);
  c->kv.pool = (__half*)(w + lay.kv);
  c->kv.page_table = c->page_table;
  c->kv.n_slots = lay.n_slots;
  c->kv.pages_per_seq = lay.pages_per_seq;
  c->kv.page_tokens = cfg->kv_page_tokens;
  int sh = 0;
  while ((1 << sh) < cfg->kv_page_tokens) ++sh;
  c->kv.page_shift = sh;
  c->kv.n_pages = lay.n_pages;
  c->kv.H = cfg->n_heads;
  c->kv.hd = c->hd;
  c->kv.page_elems = (int64_t)lay.page_elems;
  c->lanes = (LaneState*)(w + lay.lanes);
  c->h = (float*)(w + lay.h);
  c->h_in = (float*)(w + lay.h_in);
  c->hrows = (float*)(w + lay.hrows);
  for (int i = 0; i < 6; ++i) {
    int32_t* base = (int32_t*)(w + lay.rows[i]);
    c->rows[i].n = base;
    c->rows[i].lane = base + 4;
    c->rows[i].pos = base + 4 + lay.max_rows;
    c->rows[i].iter = base + 4 + 2 * lay.max_rows;
  }
  c->sc->act_a = (float*)(w + lay.act_a);
  c->sc->act_qkv = (float*)(w + lay.act_qkv);
  c->sc->act_q = (float*)(w + lay.act_q);
  c->sc->act_o = (float*)(w + lay.act_o);
  c->sc->act_u = (float*)(w + lay.act_u);
  c->sc->act_a16 = (__half*)(w + lay.act_a16);
  c->sc->act_o16 = (__half*)(w + lay.act_o16);
  c->sc->act_u16 = (__half*)(w + lay.act_u16);
  c->sc->attn_part = (float*)(w + lay.attn_part);
  c->sc->attn_counters = (int32_t*)(w + lay.attn_counters);
  c->sc->part_val = (float*)(w + lay.part_val);
  c->sc->part_idx = (int32_t*)(w + lay.part_idx);
  c->tok_stage = (int32_t*)(w + lay.tok_stage);
  c->L_stage = (int32_t*)(w + lay.L_stage);
  c->pf_n = (int32_t*)(w + lay.pf_n);
  c->pf_tiles = (int2*)(w + lay.pf_tiles);
  c->pf_info = (int32_t*)(w + lay.pf_info);
  c->probe_logits = (float*)(w + lay.probe_logits);
  c->margin_lane = (float*)(w + lay.margin_lane);
  c->spec = (int32_t*)(w + lay.spec);
  c->lane_shared = (int32_t*)(w + lay.lane_shared);
  c->sc->casc = (float*)(w + lay.casc);
  c->mask_stage = (uint8_t*)(w + lay.mask_stage);
  c->out_tok = (int32_t*)(w + lay.out_tok);
  c->out_dep = (int32_t*)(w + lay.out_dep);
  c->status = (int32_t*)(w + lay.status);
  c->counters = (unsigned long long*)(w + lay.counters);
  c->body_kernels = (int32_t*)(w + lay.body_kernels);
  c->sc->head_nparts = c->body_kernels + 7;
  c->scr[0].rows = lay.max_rows;
  c->scr[0].gs_cap = 220 * 1024;
  c->scr[0].probe = c->rows[4];
  c->scr[1].probe = c->rows[5];
  {
    Scratch& b = c->scr[1];
    b.rows = cfg->max_lanes;
    b.act_a = (float*)(w + lay.b_act_a);
    b.act_qkv = (float*)(w + lay.b_act_qkv);
    b.act_q = (float*)(w + lay.b_act_q);
    b.act_o = (float*)(w + lay.b_act_o);
    b.act_u = (float*)(w + lay.b_act_u);
    b.act_a16 = (__half*)(w + lay.b_act_a16);
    b.act_o16 = (__half*)(w + lay.b_act_o16);
    b.act_u16 = (__half*)(w + lay.b_act_u16);
    b.attn_part = (float*)(w + lay.b_attn_part);
    b.attn_counters = (int32_t*)(w + lay.b_attn_counters);
    b.part_val = (float*)(w + lay.b_part_val);
    b.part_idx = (int32_t*)(w + lay.b_part_idx);
    b.head_nparts = c->body_kernels + 6;
    b.casc = (float*)(w + lay.b_casc);
    // a smaller streamed-GEMV ring, so the concurrent loop branch's kernels find room beside it (the
    // GEMV on half of the SMs instead measured slower: 22.9k against 24.1k tokens/s on 64 lanes)
    b.gs_cap = 100 * 1024;
  }
  c->alive = (int32_t*)(w + lay.alive);
  {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
      c->n_sms = sms;
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess) c->prio_hi = hi;
    c->scr[0].gs_ctas = c->n_sms;
    c->scr[1].gs_ctas = c->n_sms;
    const GsChoice g = gs_plan(c->head.fmt, c->head.N, c->head.K, c->head.group, 1, c->n_sms);
    const int rpw = head_rpw(c->head.fmt);
    c->head_parts = g.ok ? g.grid : (c->head.N + GEMV_WARPS * rpw - 1) / (GEMV_WARPS * rpw);
  }
  // host-side page allocator
  const size_t per_lane = (size_t)lay.n_slots * lay.pages_per_seq;
  c->h_page_table.assign(per_lane * cfg->max_lanes, -1);
  c->refcount.assign(lay.n_pages, 0);
  c->free_pages.reserve(lay.n_pages);
  for (int p = lay.n_pages - 1; p >= 0; --p) c->free_pages.push_back(p);
  c->lane_L.assign(cfg->max_lanes, 0);
  c->h_lane_shared.assign(cfg->max_lanes, 0);
  c->h_lane_donor.assign(cfg->max_lanes, -1);
  int st = TL_OK;
  do {
    const int half = c->hd / 2;
    const int64_t n = (int64_t)cfg->max_seq * half;
    if ((st = launch_k(c, rope_table_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, c->rope, cfg->max_seq,
                       half, (double)cfg->rope_base)) != TL_OK)
      break;
    if ((st = launch_k(c, lanes_init_kernel, dim3((cfg->max_lanes + 255) / 256), dim3(256), 0, c->lanes,
                       cfg->max_lanes)) != TL_OK)
      break;
    if ((st = check_cuda(cudaMemsetAsync(w + lay.page_table, 0xFF, per_lane * cfg->max_lanes * 4, c->stream))) != TL_OK) break;
    if ((st = check_cuda(cudaMemsetAsync(c->status, 0, 4, c->stream))) != TL_OK) break;
    if ((st = check_cuda(cudaMemsetAsync(c->lane_shared, 0, (size_t)cfg->max_lanes * 4, c->stream))) != TL_OK) break;
    if ((st = check_cuda(cudaMemsetAsync(c->counters, 0, 32, c->stream))) != TL_OK) break;
    if ((st = check_cuda(cudaMemsetAsync(c->scr[0].attn_counters, 0, (size_t)cfg->max_lanes * cfg->n_heads * 4, c->stream))) != TL_OK) break;
    if ((st = check_cuda(cudaMemsetAsync(c->scr[1].attn_counters, 0, (size_t)cfg->max_lanes * cfg->n_heads * 4, c->stream))) != TL_OK) break;
    if ((st = encode_all_maps(c)) != TL_OK) break;
    for (int i = 0; i < 6; ++i)
      if ((st = check_cuda(cudaMemsetAsync(c->rows[i].n, 0, 4, c->stream))) != TL_OK) break;
    if (st != TL_OK) break;
    if ((st = check_cuda(cudaHostAlloc((void**)&c->pinned_alive, 2 * kAliveRing * sizeof(int32_t), cudaHostAllocDefault))) != TL_OK) break;
    for (int i = 0; i < kAliveRing; ++i)
      if ((st = check_cuda(cudaEventCreateWithFlags(&c->alive_ev[i], cudaEventDisableTiming))) != TL_OK) break;
    if (st != TL_OK) break;
    if ((st = check_cuda(cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking))) != TL_OK) break;
    if ((st = check_cuda(cudaStreamCreateWithFlags(&c->cap_body, cudaStreamNonBlocking))) != TL_OK) break;
    if ((st = check_cuda(cudaStreamCreateWithFlags(&c->cap_stream2, cudaStreamNonBlocking))) != TL_OK) break;
    if ((st = check_cuda(cudaEventCreateWithFlags(&c->fork_ev, cudaEventDisableTiming))) != TL_OK) break;
    if ((st = check_cuda(cudaEventCreateWithFlags(&c->join_ev, cudaEventDisableTiming))) != TL_OK) break;
    if ((st = check_cuda(cudaStreamCreateWithFlags(&c->bstream, cudaStreamNonBlocking))) != TL_OK) break;
    for (int i = 0; i < kBRing; ++i)
      if ((st = check_cuda(cudaEventCreateWithFlags(&c->b_ev[i], cudaEventDisableTiming))) != TL_OK) break;
    if (st != TL_OK) break;
  } while (0);
  if (st != TL_OK) {
    if (c->pinned_alive) cudaFreeHost(c->pinned_alive);
    delete c;
    return st;
  }
  *out = c;
  return TL_OK;
}

extern "C" int tl_destroy(tl_ctx* c) {
  if (!c) return TL_EINVAL;
  cudaStreamSynchronize(c->stream);
  if (c->tick_exec) cudaGraphExecDestroy(c->tick_exec);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  if (c->cap_body) cudaStreamDestroy(c->cap_body);
  if (c->cap_stream2) cudaStreamDestroy(c->cap_stream2);
  if (c->fork_ev) cudaEventDestroy(c->fork_ev);
  if (c->join_ev) cudaEventDestroy(c->join_ev);
  if (c->loop_exec) cudaGraphExecDestroy(c->loop_exec);
  if (c->bnd_exec) cudaGraphExecDestroy(c->bnd_exec);
  if (c->bstream) cudaStreamDestroy(c->bstream);
  for (int i = 0; i < kBRing; ++i)
    if (c->b_ev[i]) cudaEventDestroy(c->b_ev[i]);
  for (int i = 0; i < kAliveRing; ++i) cudaEventDestroy(c->alive_ev[i]);
  for (auto& e : c->prof_ev) {
    cudaEventDestroy(e[0]);
    cudaEventDestroy(e[1]);
  }
  if (c->pinned_alive) cudaFreeHost(c->pinned_alive);
  delete c;
  return TL_OK;
}

extern "C" int tl_load_weights(tl_ctx* c, const void* blob, size_t bytes) {
  if (!c || !blob) return TL_EINVAL;
  const tl_config* cfg = &c->cfg;
  if (bytes != blob_bytes(cfg)) return TL_EINVAL;
  const char* b = (const char*)blob;
  if (memcmp(b, "TLWBLOB1", 8) != 0) return TL_EINVAL;
  int32_t hdr_i[10];
  float hdr_f[2];
  memcpy(hdr_i, b + 8, 40);
  memcpy(hdr_f, b + 48, 8);
  const int32_t want[10] = {cfg->vocab, cfg->d, cfg->n_heads, cfg->ffn, cfg->n_pre, cfg->n_loop_layers,
                            cfg->fmt_pre, cfg->fmt_loop, cfg->fmt_embed_head, cfg->group};
  if (memcmp(hdr_i, want, 40) != 0 || hdr_f[0] != cfg->rms_eps || hdr_f[1] != cfg->rope_base) return TL_EINVAL;
  size_t off = kBlobHeader;
  auto specs = mat_specs(cfg);
  for (size_t i = 0; i < specs.size(); ++i) {
    const size_t n = mat_bytes(cfg, specs[i].fmt, specs[i].N, specs[i].K);
    TL_CUDA(cudaMemcpyAsync(c->ws + c->lay.mat_off[i], b + off, n, cudaMemcpyHostToDevice, c->stream));
    off += n;
  }
  const size_t gb = (size_t)(2 * (cfg->n_pre + cfg->n_loop_layers) + 1) * cfg->d * 4;
  TL_CUDA(cudaMemcpyAsync(c->ws + c->lay.gains, b + off, gb, cudaMemcpyHostToDevice, c->stream));
  // INT4 matrices into the device nibble order
  std::vector<const MatView*> mats = {&c->embed, &c->head};
  for (auto* v : {&c->pre, &c->loop})
    for (const BlockW& bw : *v)
      for (const MatView* m : {&bw.wqkv, &bw.wo, &bw.wg, &bw.wu, &bw.wd}) mats.push_back(m);
  for (const MatView* m : mats) {
    if (m->fmt != TL_FMT_INT4) continue;
    const int64_t words = (int64_t)m->N * m->K / 8;
    TL_TRY(launch_k(c, int4_repack_kernel, dim3((unsigned)((words + 255) / 256)), dim3(256), 0, (uint32_t*)m->q, words));
  }
  // the blocks' resident fp16 copies (the conversion the tensor-core kernels applied per tile)
  for (auto* v : {&c->pre, &c->loop})
    for (const BlockW& bw : *v) {
      if (!bw.f16) continue;
      const MatView* src[5] = {&bw.wqkv, &bw.wo, &bw.wg, &bw.wu, &bw.wd};
      const MatView* dst[5] = {&bw.f16->wqkv, &bw.f16->wo, &bw.f16->wg, &bw.f16->wu, &bw.f16->wd};
      for (int i = 0; i < 5; ++i) {
        const int64_t words = (int64_t)src[i]->N * src[i]->K / 8;
        TL_TRY(launch_k(c, stage_f16_kernel, dim3((unsigned)((words + 255) / 256)), dim3(256), 0, *src[i],
                        const_cast<__half*>(reinterpret_cast<const __half*>(dst[i]->bf))));
      }
    }
  TL_CUDA(cudaStreamSynchronize(c->stream));
  c->loaded = true;
  return TL_OK;
}

extern "C" int tl_set_early_exit(tl_ctx* c, double tau, int32_t min_L, int32_t patience, int32_t peek_every) {
  if (!c || peek_every < 1 || min_L < 0 || patience < 0) return TL_EINVAL;
  c->ee.tau = tau;
  c->ee.min_L = min_L;
  c->ee.patience = patience;
  c->ee.peek_every = peek_every;
  c->ee.enabled = (tau > 0.0 && patience > 0) ? 1 : 0;
  c->ee.use_margin = 0;
  c->ee.margin = 0.0;
  return TL_OK;
}

extern "C" int tl_set_early_exit_logit_margin(tl_ctx* c, double margin, int32_t min_L, int32_t patience,
                                              int32_t peek_every) {
  if (!c || peek_every < 1 || min_L < 0 || patience < 0) return TL_EINVAL;
  c->ee.tau = 0.0;
  c->ee.min_L = min_L;
  c->ee.patience = patience;
  c->ee.peek_every = peek_every;
  c->ee.enabled = (margin > 0.0 && patience > 0) ? 1 : 0;
  c->ee.use_margin = 1;
  c->ee.margin = margin;
  return TL_OK;
}

extern "C" int tl_set_l_warmup(tl_ctx* c, int32_t warmup_tokens, int32_t warmup_L) {
  if (!c || warmup_tokens < 0 || warmup_L < 1) return TL_EINVAL;
  c->warm.tokens = warmup_tokens;
  c->warm.L = warmup_L;
  return TL_OK;
}

// Prompts of several lanes in one pass over the weights.  Every block runs
// once on the rows of all lanes (the loop's iteration l on the lanes whose L
// exceeds l: lanes are ordered by L, deepest first, so those rows are a prefix
// of the row table); attention runs per lane, in tiles of up to 64 rows that
// never straddle two lanes.
struct PromptLane {
  int lane;
  const int32_t* tokens;
  int T, L;
};

static int prefill_impl(tl_ctx* c, const std::vector<PromptLane>& in, int32_t share_from, int32_t shared_tokens,
                        float* dev_hidden_out) {
  const tl_config& cfg = c->cfg;
  const int n = (int)in.size();
  if (n < 1 || n > cfg.max_lanes) return TL_EINVAL;
  const int P = cfg.n_pre, Lb = cfg.n_loop_layers, pps = c->lay.pages_per_seq, pt = cfg.kv_page_tokens;
  std::vector<char> seen(cfg.max_lanes, 0);
  std::vector<int> share_pages(n, 0);
  int64_t total = 0;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    const PromptLane& p = in[i];
    if (p.lane < 0 || p.lane >= cfg.max_lanes || seen[p.lane] || !p.tokens || p.T < 1 || p.T > cfg.max_seq ||
        p.L < 1 || p.L > cfg.L_max)
      return TL_EINVAL;
    seen[p.lane] = 1;
    for (int t = 0; t < p.T; ++t)
      if (p.tokens[t] < 0 || p.tokens[t] >= cfg.vocab) return TL_EINVAL;
    if (share_from >= 0) {
      // the donor keeps its pages: it is not re-run in this batch and holds every slot this lane needs
      if (share_from >= cfg.max_lanes || share_from == p.lane || c->lane_L[share_from] < p.L || shared_tokens < 0 ||
          shared_tokens > p.T)
        return TL_EINVAL;
      // whole pages only, and never the last prompt position (this lane computes it)
      share_pages[i] = (shared_tokens < p.T ? shared_tokens : p.T - 1) / pt;
    }
    total += p.T - share_pages[i] * pt;
    need += (int64_t)(P + p.L * Lb) * (pps - share_pages[i]);
  }
  if (share_from >= 0 && seen[share_from]) return TL_EINVAL;
  if (total > c->lay.max_prefill) return TL_EINVAL;
  // pages: slots of the pre blocks and of iterations 1..L, for every position up to max_seq
  for (int i = 0; i < n; ++i) release_lane_pages(c, in[i].lane);
  if ((int64_t)c->free_pages.size() < need) {
    update_cascade(c);
    return TL_ENOMEM;
  }
  const size_t per_lane = (size_t)c->lay.n_slots * pps;
  for (int i = 0; i < n; ++i) {
    const int used_slots = P + in[i].L * Lb;
    int32_t* t = &c->h_page_table[(size_t)in[i].lane * per_lane];
    const int32_t* donor = share_from >= 0 ? &c->h_page_table[(size_t)share_from * per_lane] : nullptr;
    for (int sl = 0; sl < used_slots; ++sl)
      for (int pg = 0; pg < pps; ++pg) {
        int32_t id;
        if (pg < share_pages[i]) {
          id = donor[(size_t)sl * pps + pg];
        } else {
          id = c->free_pages.back();
          c->free_pages.pop_back();
        }
        c->refcount[id]++;
        t[(size_t)sl * pps + pg] = id;
      }
    c->lane_L[in[i].lane] = in[i].L;
    c->h_lane_shared[in[i].lane] = share_pages[i] * pt;
    c->h_lane_donor[in[i].lane] = share_pages[i] > 0 ? share_from : -1;
    TL_CUDA(cudaMemcpyAsync(c->page_table + (size_t)in[i].lane * per_lane, t, per_lane * 4, cudaMemcpyHostToDevice,
                            c->stream));
  }
  TL_TRY(update_cascade(c));
  // row table (deepest lanes first), tokens, attention tiles, per-lane finish info
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return in[a].L > in[b].L; });
  std::vector<int32_t> r_lane, r_pos, r_iter, tok, info;
  std::vector<int2> tiles;
  std::vector<int64_t> rows_upto(n + 1, 0), tiles_upto(n + 1, 0);
  r_lane.reserve(total);
  r_pos.reserve(total);
  tok.reserve(total);
  for (int k = 0; k < n; ++k) {
    const PromptLane& p = in[order[k]];
    const int pos0 = share_pages[order[k]] * pt, Tn = p.T - pos0;
    const int row0 = (int)r_lane.size();
    for (int t = 0; t < Tn; ++t) {
      r_lane.push_back(p.lane);
      r_pos.push_back(pos0 + t);
      tok.push_back(p.tokens[pos0 + t]);
    }
    const int tr = prompt_tile_rows(c);
    for (int t0 = 0; t0 < Tn; t0 += tr) tiles.push_back(make_int2(row0 + t0, Tn - t0 < tr ? Tn - t0 : tr));
    info.insert(info.end(), {p.lane, row0 + Tn - 1, p.T - 1, p.L});
    rows_upto[k + 1] = (int64_t)r_lane.size();
    tiles_upto[k + 1] = (int64_t)tiles.size();
  }
  r_iter.assign(total, 0);
  const int Lmax = in[order[0]].L;
  std::vector<int32_t> stage_rows(Lmax + 1, 0), stage_tiles(Lmax);  // stage_rows[Lmax] = 0
  for (int l = 0; l < Lmax; ++l) {
    int k = 0;
    while (k < n && in[order[k]].L > l) ++k;  // lanes 0..k-1 of the order run iteration l
    stage_rows[l] = (int32_t)rows_upto[k];
    stage_tiles[l] = (int32_t)tiles_upto[k];
  }
  const Rows& R = c->rows[3];
  TL_CUDA(cudaMemcpyAsync(R.lane, r_lane.data(), total * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(R.pos, r_pos.data(), total * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(R.iter, r_iter.data(), total * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->tok_stage, tok.data(), total * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->pf_tiles, tiles.data(), tiles.size() * sizeof(int2), cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->pf_info, info.data(), info.size() * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->pf_n, stage_rows.data(), (Lmax + 1) * 4, cudaMemcpyHostToDevice, c->stream));
  Rows Rs = R;
  Rs.n = c->pf_n;  // stage 0: every row (every lane has L >= 1)
  const int all = (int)total;
  TL_TRY(launch_k(c, embed_rows_kernel, dim3(all), dim3(256), 0, c->embed, c->tok_stage, all, cfg.d, c->hrows,
                  c->status));
  PendingAdd pend;
  for (int b = 0; b < P; ++b)
    TL_TRY(run_block(c, Rs, all, c->hrows, nullptr, c->pre[b], b, 0, nullptr, true, PATH_AUTO, c->pf_tiles,
                     stage_tiles[0], &pend));
  for (int l = 0; l < Lmax; ++l) {
    Rs.n = c->pf_n + l;
    for (int m = 0; m < Lb; ++m)
      TL_TRY(run_block(c, Rs, stage_rows[l], c->hrows, nullptr, c->loop[m], P + l * Lb + m, 0, nullptr, true,
                       PATH_AUTO, c->pf_tiles, stage_tiles[l], &pend));
  }
  if (pend.add)  // the last block's residual (the norm kernel with no rows to normalise only adds)
    TL_TRY(launch_k(c, rmsnorm_rows_kernel, dim3(pend.rows), dim3(256), 0, c->hrows, (const int32_t*)nullptr,
                    (const int32_t*)(c->pf_n + Lmax), cfg.d, (const float*)nullptr, cfg.rms_eps, (float*)nullptr,
                    (float*)nullptr, (__half*)nullptr, (float*)nullptr, 0, 0, pend.add, pend.n, 0));
  TL_TRY(launch_k(c, prefill_finish_batch_kernel, dim3(n), dim3(256), 0, c->lanes, c->pf_info, n, c->hrows, c->h,
                  cfg.d));
  if (dev_hidden_out)
    TL_CUDA(cudaMemcpyAsync(dev_hidden_out, c->hrows, (size_t)total * cfg.d * 4, cudaMemcpyDeviceToDevice,
                            c->stream));
  c->prefill_tokens += total;
  // the host tables above are pageable: the copies have consumed them by the time cudaMemcpyAsync returns
  return TL_OK;
}

extern "C" int tl_prefill(tl_ctx* c, int32_t lane, const int32_t* host_tokens, int32_t T, int32_t L,
                          int32_t share_from, int32_t shared_tokens, float* dev_hidden_out) {
  if (!c || !host_tokens) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  return prefill_impl(c, {PromptLane{lane, host_tokens, T, L}}, share_from, shared_tokens, dev_hidden_out);
}

extern "C" int tl_prefill_batch(tl_ctx* c, int32_t n, const int32_t* lanes, const int32_t* host_tokens,
                                const int32_t* T, const int32_t* L, int32_t share_from, int32_t shared_tokens) {
  if (!c || !lanes || !host_tokens || !T || !L || n < 1) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  std::vector<PromptLane> in(n);
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    if (T[i] < 1) return TL_EINVAL;
    in[i] = PromptLane{lanes[i], host_tokens + off, T[i], L[i]};
    off += (size_t)T[i];
  }
  return prefill_impl(c, in, share_from, shared_tokens, nullptr);
}

// ------------------------------------------------------ self-speculation ----

// Positions pos0 .. pos0 + k - 1 of one lane (their tokens already in
// c->tok_stage) through embed, the pre blocks and L loop iterations as one
// causal batch over the lane's own pages (the cache of earlier positions is
// read, these positions' K/V rewritten for every slot they reach); the final
// hidden rows are left in c->hrows.  The lane state is not touched.
static int rerun_positions(tl_ctx* c, int lane, int pos0, int k, int L) {
  const tl_config& cfg = c->cfg;
  const int P = cfg.n_pre, Lb = cfg.n_loop_layers;
  std::vector<int32_t> r_lane(k, lane), r_pos(k), r_iter(k, 0), stage_rows(L + 1, k);
  stage_rows[L] = 0;
  for (int i = 0; i < k; ++i) r_pos[i] = pos0 + i;
  std::vector<int2> tiles;
  const int tr = prompt_tile_rows(c);
  for (int t0 = 0; t0 < k; t0 += tr) tiles.push_back(make_int2(t0, k - t0 < tr ? k - t0 : tr));
  const Rows& R = c->rows[3];
  TL_CUDA(cudaMemcpyAsync(R.lane, r_lane.data(), k * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(R.pos, r_pos.data(), k * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(R.iter, r_iter.data(), k * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->pf_tiles, tiles.data(), tiles.size() * sizeof(int2), cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->pf_n, stage_rows.data(), (L + 1) * 4, cudaMemcpyHostToDevice, c->stream));
  Rows Rs = R;
  Rs.n = c->pf_n;
  const int nt = (int)tiles.size();
  TL_TRY(launch_k(c, embed_rows_kernel, dim3(k), dim3(256), 0, c->embed, (const int32_t*)c->tok_stage, k, cfg.d,
                  c->hrows, c->status));
  PendingAdd pend;
  for (int b = 0; b < P; ++b)
    TL_TRY(run_block(c, Rs, k, c->hrows, nullptr, c->pre[b], b, 0, nullptr, true, PATH_AUTO, c->pf_tiles, nt, &pend));
  for (int l = 0; l < L; ++l) {
    Rs.n = c->pf_n + l;
    for (int m = 0; m < Lb; ++m)
      TL_TRY(run_block(c, Rs, k, c->hrows, nullptr, c->loop[m], P + l * Lb + m, 0, nullptr, true, PATH_AUTO,
                       c->pf_tiles, nt, &pend));
  }
  if (pend.add)
    TL_TRY(launch_k(c, rmsnorm_rows_kernel, dim3(pend.rows), dim3(256), 0, c->hrows, (const int32_t*)nullptr,
                    (const int32_t*)(c->pf_n + L), cfg.d, (const float*)nullptr, cfg.rms_eps, (float*)nullptr,
                    (float*)nullptr, (__half*)nullptr, (float*)nullptr, 0, 0, pend.add, pend.n, 0));
  c->prefill_tokens += k;
  return TL_OK;
}

// Greedy head over hidden rows 0 .. k - 1 of c->hrows: dev_argmax[r] for each row.
static int head_hrows(tl_ctx* c, int k, int32_t* dev_argmax) {
  const Rows& T4 = c->rows[4];
  std::vector<int32_t> ident(k);
  for (int i = 0; i < k; ++i) ident[i] = i;
  TL_CUDA(cudaMemcpyAsync(T4.lane, ident.data(), k * 4, cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(T4.n, &k, 4, cudaMemcpyHostToDevice, c->stream));
  const float* X = nullptr;
  GsNorm nrm{};
  bool use_nrm = false;
  TL_TRY(norm_for_proj(c, k, PATH_AUTO, T4.n, c->hrows, nullptr, c->g_final, nullptr, c->head, 1, &X, &nrm, &use_nrm));
  ProjOut o{};
  o.epi = EPI_ARGMAX;
  o.lmap = T4.lane;
  o.ldo = c->cfg.vocab;
  o.part_val = c->sc->part_val;
  o.part_idx = c->sc->part_idx;
  o.n_parts_dev = c->sc->head_nparts;
  TL_TRY(proj(c, k, PATH_AUTO, X, 0, T4.n, c->head, &c->mhead, nullptr, nullptr, o, nullptr, TL_PROF_HEAD,
              use_nrm ? &nrm : nullptr));
  return launch_k(c, head_finalize_kernel, dim3(k), dim3(256), 0, T4, c->lanes, (const float*)c->sc->part_val,
                  (const int32_t*)c->sc->part_idx, (const int32_t*)c->sc->head_nparts, (int32_t)HEAD_ONLY, dev_argmax,
                  (int32_t*)nullptr, (int32_t*)nullptr, 0, c->embed, c->h, c->cfg.d, c->cfg.max_seq, 0, c->status,
                  (unsigned long long*)nullptr, c->warm, (int32_t)0);
}

static int speculate_impl(tl_ctx* c, int lane, int n_new, int Ld, int Lv, int ahead, int32_t* out, int32_t* rounds_out) {
  const tl_config& cfg = c->cfg;
  LaneState st{};
  TL_CUDA(cudaMemcpyAsync(&st, c->lanes + lane, sizeof(st), cudaMemcpyDeviceToHost, c->stream));
  TL_CUDA(cudaStreamSynchronize(c->stream));
  if (st.phase != PH_BOUNDARY || st.taken != 0 || st.depth < Lv) return TL_ESTATE;
  const int T = st.pos + 1;
  if (T + n_new - 1 > cfg.max_seq) return TL_EINVAL;
  int32_t* tok = c->spec;                   // [lanes] the token each lane takes next (embed input, head output)
  int32_t* drafted = c->spec + cfg.max_lanes;  // [ahead]
  int32_t* verify = drafted + c->lay.max_prefill;  // [ahead] the verify pass's greedy tokens
  std::vector<uint8_t> mask(cfg.max_lanes, 0);
  mask[lane] = 1;
  TL_CUDA(cudaMemcpyAsync(c->mask_stage, mask.data(), cfg.max_lanes, cudaMemcpyHostToDevice, c->stream));
  std::vector<int32_t> Lreq(cfg.max_lanes, Ld);
  TL_CUDA(cudaMemcpyAsync(c->L_stage, Lreq.data(), cfg.max_lanes * 4, cudaMemcpyHostToDevice, c->stream));
  // token 0 from the prompt's last position
  TL_TRY(build_rows(c, 1, SEL_MASK, c->mask_stage, nullptr, nullptr, nullptr));
  TL_TRY(head_stage(c, cfg.max_lanes, HEAD_ONLY, nullptr, tok, nullptr, nullptr, 0));
  int32_t t0 = 0;
  TL_CUDA(cudaMemcpyAsync(&t0, tok + lane, 4, cudaMemcpyDeviceToHost, c->stream));
  TL_CUDA(cudaStreamSynchronize(c->stream));
  std::vector<int32_t> tokens{t0};
  std::vector<int32_t> hd(ahead), hv(ahead);
  int rounds = 0;
  while ((int)tokens.size() < n_new) {
    ++rounds;
    const int p0 = T + (int)tokens.size() - 1;  // position of the last token taken, not computed yet
    const int k = std::min(ahead, n_new - (int)tokens.size());
    TL_CUDA(cudaMemcpyAsync(tok + lane, &tokens.back(), 4, cudaMemcpyHostToDevice, c->stream));
    // draft: one position at a time at L_draft, each greedy token fed straight back on the device
    for (int j = 0; j < k; ++j) {
      TL_TRY(launch_k(c, embed_next_kernel, dim3(cfg.max_lanes), dim3(256), 0, c->lanes, cfg.max_lanes,
                      (const uint8_t*)c->mask_stage, (const int32_t*)tok, c->embed, c->h, cfg.d, cfg.max_seq, c->status,
                      c->warm));
      TL_TRY(pre_blocks_for_entered(c, cfg.max_lanes));
      for (int l = 0; l < Ld; ++l) {
        TL_TRY(build_rows(c, 0, SEL_LOOP, c->mask_stage, l == 0 ? c->L_stage : nullptr, nullptr, nullptr));
        TL_TRY(loop_iteration(c, cfg.max_lanes, nullptr));
      }
      TL_TRY(build_rows(c, 1, SEL_MASK, c->mask_stage, nullptr, nullptr, nullptr));
      TL_TRY(head_stage(c, cfg.max_lanes, HEAD_ONLY, nullptr, tok, nullptr, nullptr, 0));
      TL_CUDA(cudaMemcpyAsync(drafted + j, tok + lane, 4, cudaMemcpyDeviceToDevice, c->stream));
    }
    // verify: the k positions together at L_verify, inputs = the last token taken, then the drafts
    TL_CUDA(cudaMemcpyAsync(c->tok_stage, &tokens.back(), 4, cudaMemcpyHostToDevice, c->stream));
    if (k > 1)
      TL_CUDA(cudaMemcpyAsync(c->tok_stage + 1, drafted, (size_t)(k - 1) * 4, cudaMemcpyDeviceToDevice, c->stream));
    TL_TRY(rerun_positions(c, lane, p0, k, Lv));
    TL_TRY(head_hrows(c, k, verify));
    TL_CUDA(cudaMemcpyAsync(hd.data(), drafted, (size_t)k * 4, cudaMemcpyDeviceToHost, c->stream));
    TL_CUDA(cudaMemcpyAsync(hv.data(), verify, (size_t)k * 4, cudaMemcpyDeviceToHost, c->stream));
    TL_CUDA(cudaStreamSynchronize(c->stream));
    int taken = 0;
    for (int j = 0; j < k; ++j) {
      tokens.push_back(hv[j]);
      ++taken;
      if (hv[j] != hd[j]) break;
    }
    // the lane continues from the last kept position, computed at L_verify by the verify pass
    const int32_t info[4] = {lane, taken - 1, p0 + taken - 1, Lv};
    TL_CUDA(cudaMemcpyAsync(c->pf_info, info, sizeof(info), cudaMemcpyHostToDevice, c->stream));
    TL_TRY(launch_k(c, prefill_finish_batch_kernel, dim3(1), dim3(256), 0, c->lanes, (const int32_t*)c->pf_info, 1,
                    (const float*)c->hrows, c->h, cfg.d));
  }
  TL_CUDA(cudaStreamSynchronize(c->stream));
  std::memcpy(out, tokens.data(), (size_t)n_new * 4);
  if (rounds_out) *rounds_out = rounds;
  return TL_OK;
}

extern "C" int tl_speculate(tl_ctx* c, int32_t lane, int32_t n_new, int32_t L_draft, int32_t L_verify,
                            int32_t draft_ahead, int32_t* host_tokens_out, int32_t* host_rounds_out) {
  if (!c || !host_tokens_out) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  if (lane < 0 || lane >= c->cfg.max_lanes || n_new < 1 || L_draft < 1 || L_verify < 1 || draft_ahead < 1 ||
      L_draft > c->cfg.L_max || L_verify > c->cfg.L_max || draft_ahead > c->lay.max_prefill ||
      draft_ahead > c->cfg.max_lanes)
    return TL_EINVAL;
  if (c->lane_L[lane] == 0) return TL_ESTATE;
  if (L_verify > c->lane_L[lane] || L_draft > c->lane_L[lane]) return TL_EKV;
  // the oracle's speculation has no early exit and no warmup: both are off for its duration
  const EEParams ee = c->ee;
  const WarmParams wp = c->warm;
  c->ee.enabled = 0;
  c->warm.tokens = 0;
  const int st = speculate_impl(c, lane, n_new, L_draft, L_verify, draft_ahead, host_tokens_out, host_rounds_out);
  c->ee = ee;
  c->warm = wp;
  return st;
}

extern "C" int tl_loop_step(tl_ctx* c, const int32_t* dev_L, const uint8_t* dev_mask, uint8_t* dev_exit) {
  if (!c) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  TL_TRY(build_rows(c, 0, SEL_LOOP, dev_mask, dev_L, dev_exit, nullptr));
  return loop_iteration(c, c->cfg.max_lanes, dev_exit);
}

extern "C" int tl_head_logits(tl_ctx* c, const uint8_t* dev_mask, float* dev_logits, int32_t* dev_argmax) {
  if (!c) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  TL_TRY(build_rows(c, 1, dev_mask ? SEL_MASK : SEL_BOUNDARY, dev_mask, nullptr, nullptr, nullptr));
  return head_stage(c, c->cfg.max_lanes, HEAD_ONLY, dev_logits, dev_argmax, nullptr, nullptr, 0);
}

extern "C" int tl_embed_next(tl_ctx* c, const uint8_t* dev_mask, const int32_t* dev_tokens) {
  if (!c || !dev_tokens) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  TL_TRY(launch_k(c, embed_next_kernel, dim3(c->cfg.max_lanes), dim3(256), 0, c->lanes, c->cfg.max_lanes, dev_mask, dev_tokens,
                                                             c->embed, c->h, c->cfg.d, c->cfg.max_seq, c->status,
                                                             c->warm));
  return pre_blocks_for_entered(c, c->cfg.max_lanes);
}

// The tick's three row tables (boundary -> rows[1], entered -> rows[2],
// loop -> rows[0]) and alive count from one kernel; with conditional nodes it
// also chooses their bodies.
static int plan_tick(tl_ctx* c, int n_lanes, const TickConds& tc, int32_t which = 3) {
  return launch_k(c, plan_tick_kernel, dim3(1), dim3(1024), 0, c->lanes, n_lanes, c->rows[1], c->rows[2], c->rows[0],
                  c->alive, c->cfg.max_seq, tc, kGemvMaxRows, c->body_kernels, &c->counters[2], which);
}

// One decode tick: the boundary stage (head, tokens, embedding, pre blocks
// and the first loop iteration of the lanes that take a token) and one loop
// iteration for the lanes already in their loop.  The two touch disjoint
// lanes and use separate scratch; launched one after the other here, they are
// concurrent branches of the tick graph.
static int enqueue_tick(tl_ctx* c, int n_lanes, int n_new, int32_t* tok_out, int32_t* dep_out) {
  TL_TRY(plan_tick(c, n_lanes, TickConds{}));
  c->sc = &c->scr[1];
  c->prio = c->prio_hi;
  int st = head_core(c, n_lanes, HEAD_DECODE, nullptr, nullptr, tok_out, dep_out, n_new, PATH_AUTO, 0);
  if (st == TL_OK) st = pre_blocks(c, n_lanes);
  if (st == TL_OK && c->entry_iter) st = loop_iteration(c, n_lanes, nullptr, PATH_AUTO, 2);
  c->sc = &c->scr[0];
  c->prio = 0;
  TL_TRY(st);
  return loop_iteration(c, n_lanes, nullptr, loop_path(n_lanes));
}

static bool same_ee(const EEParams& a, const EEParams& b) {
  return a.tau == b.tau && a.min_L == b.min_L && a.patience == b.patience && a.peek_every == b.peek_every &&
         a.enabled == b.enabled && a.use_margin == b.use_margin && a.margin == b.margin;
}

// Conditional node after the current position of the capture on `s`.
static int add_conditional(cudaStream_t s, cudaGraphConditionalHandle h, cudaGraphConditionalNodeType type, int size,
                           cudaGraph_t* bodies) {
  cudaStreamCaptureStatus st;
  cudaGraph_t g = nullptr;
  const cudaGraphNode_t* deps = nullptr;
  size_t nd = 0;
  TL_CUDA(cudaStreamGetCaptureInfo(s, &st, nullptr, &g, &deps, &nd));
  cudaGraphNodeParams p{};
  p.type = cudaGraphNodeTypeConditional;
  p.conditional.handle = h;
  p.conditional.type = type;
  p.conditional.size = size;
  cudaGraphNode_t node;
  TL_CUDA(cudaGraphAddNode(&node, g, deps, nd, &p));
  for (int i = 0; i < size; ++i) bodies[i] = p.conditional.phGraph_out[i];
  TL_CUDA(cudaStreamUpdateCaptureDependencies(s, &node, 1, cudaStreamSetCaptureDependencies));
  return TL_OK;
}

static int new_handle(cudaStream_t s, cudaGraphConditionalHandle* h) {
  cudaStreamCaptureStatus st;
  cudaGraph_t g = nullptr;
  TL_CUDA(cudaStreamGetCaptureInfo(s, &st, nullptr, &g, nullptr, nullptr));
  TL_CUDA(cudaGraphConditionalHandleCreate(h, g, 0, cudaGraphCondAssignDefault));
  return TL_OK;
}

// Captures fn() into an (empty) body graph; *n_kernels = kernels it launched.
template <class F>
static int capture_body(tl_ctx* c, cudaGraph_t body, int64_t* n_kernels, F fn) {
  TL_CUDA(cudaStreamBeginCaptureToGraph(c->cap_body, body, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal));
  cudaStream_t saved = c->stream;
  c->stream = c->cap_body;
  const int64_t l0 = c->launches;
  const int st = fn();
  *n_kernels = c->launches - l0;
  c->stream = saved;
  cudaGraph_t out = nullptr;
  const cudaError_t e = cudaStreamEndCapture(c->cap_body, &out);
  TL_TRY(st);
  return check_cuda(e);
}

// The tick as a CUDA graph with device-chosen branches: one planning kernel
// builds the three row tables and sets one conditional node per stage, so a
// stage with no rows runs nothing and a stage runs either its CUDA-core GEMV
// variant (<= 8 rows) or its tensor-core variant, never both.  Every kernel
// reads its row count from device memory, so one capture serves every tick of
// a decode with the same lanes, token budget, outputs and early-exit
// parameters.
//   plan -+-> SWITCH { norm, head, argmax + token + embedding: GEMV | tensor cores }
//         |     -> SWITCH { entering lanes: pre blocks + first loop iteration: GEMV | TC }  (boundary scratch)
//         +-> loop body + exit rule of the other lanes: plain nodes (loop_path) for a body of
//             <= 2 layers, else SWITCH { GEMV | tensor cores }                            (main scratch)
//   (the two branches join at the end of the tick: "Depth-adaptive Inference of Looped Language Models via
//   Continuous Depth Batching", boundary stages queued apart from loop steps, overlapped with them)
static int capture_tick(tl_ctx* c, int n_lanes, int n_new, int32_t* tok_out, int32_t* dep_out, int32_t* kcount) {
  TickConds tc{};
  // a short loop body runs as plain kernel nodes (below), so its handle is not needed
  const bool plain_loop = c->cfg.n_loop_layers <= 2;
  for (int t = 0; t < (plain_loop ? 2 : 3); ++t) TL_TRY(new_handle(c->stream, &tc.h[t]));
  tc.use = plain_loop ? 3 : 7;
  TL_TRY(plan_tick(c, n_lanes, tc));
  cudaGraph_t body[2];
  int64_t nk[2] = {0, 0};
  // fork: the boundary stage on its own capture stream (and scratch), concurrent with the loop iteration
  cudaStream_t main_s = c->stream;
  TL_CUDA(cudaEventRecord(c->fork_ev, main_s));
  TL_CUDA(cudaStreamWaitEvent(c->cap_stream2, c->fork_ev, 0));
  c->stream = c->cap_stream2;
  c->sc = &c->scr[1];
  // the boundary stage's kernels at the device's highest priority: their CTAs are dispatched ahead of the
  // loop step's pending ones
  c->prio = c->prio_hi;
  // boundary rows -> head (CUDA-core GEMV for <= 8 rows, tensor cores above)
  TL_TRY(add_conditional(c->stream, tc.h[0], cudaGraphCondTypeSwitch, 2, body));
  TL_TRY(capture_body(c, body[0], &nk[0], [&] {
    return head_core(c, n_lanes, HEAD_DECODE, nullptr, nullptr, tok_out, dep_out, n_new, PATH_GEMV, 0);
  }));
  TL_TRY(capture_body(c, body[1], &nk[1], [&] {
    return head_core(c, n_lanes, HEAD_DECODE, nullptr, nullptr, tok_out, dep_out, n_new, PATH_TC, 0);
  }));
  kcount[0] = (int32_t)nk[0];
  kcount[1] = (int32_t)nk[1];
  // entered rows -> pre blocks and their first loop iteration
  TL_TRY(add_conditional(c->stream, tc.h[1], cudaGraphCondTypeSwitch, 2, body));
  TL_TRY(capture_body(c, body[0], &nk[0], [&] {
    const int st = pre_blocks(c, n_lanes, PATH_GEMV);
    return (st != TL_OK || !c->entry_iter) ? st : loop_iteration(c, n_lanes, nullptr, PATH_GEMV, 2);
  }));
  TL_TRY(capture_body(c, body[1], &nk[1], [&] {
    const int st = pre_blocks(c, n_lanes, PATH_TC);
    return (st != TL_OK || !c->entry_iter) ? st : loop_iteration(c, n_lanes, nullptr, PATH_TC, 2);
  }));
  kcount[2] = (int32_t)nk[0];
  kcount[3] = (int32_t)nk[1];
  // join point of the boundary branch; the loop branch continues on the main capture stream
  TL_CUDA(cudaEventRecord(c->join_ev, c->cap_stream2));
  c->stream = main_s;
  c->sc = &c->scr[0];
  c->prio = 0;
  // loop rows -> loop body.  The bodies of a graph's conditional nodes were measured to start one after
  // another (each once the previous body's last kernel was launched), which kept this branch waiting for
  // the boundary stage's head.  So a short body runs as plain kernel nodes, which start at once, on the
  // projection path loop_path chooses; a long body (the 24-layer one) keeps its conditional node, where
  // doubling every projection's launches measured slower (7.0k against 7.9k tokens/s on 256 lanes).  Plain nodes for the boundary
  // stage too measured slower again (2.0k against 1.8k tokens/s for one lane at L = 8).
  c->tick_loop_kernels = 0;
  kcount[4] = kcount[5] = 0;
  if (plain_loop) {
    const int64_t l0 = c->launches;
    TL_TRY(loop_iteration(c, n_lanes, nullptr, loop_path(n_lanes)));
    c->tick_loop_kernels = c->launches - l0;
  } else {
    TL_TRY(add_conditional(c->stream, tc.h[2], cudaGraphCondTypeSwitch, 2, body));
    TL_TRY(capture_body(c, body[0], &nk[0], [&] { return loop_iteration(c, n_lanes, nullptr, PATH_GEMV); }));
    TL_TRY(capture_body(c, body[1], &nk[1], [&] { return loop_iteration(c, n_lanes, nullptr, PATH_TC); }));
    kcount[4] = (int32_t)nk[0];
    kcount[5] = (int32_t)nk[1];
  }
  TL_CUDA(cudaStreamWaitEvent(c->stream, c->join_ev, 0));
  return TL_OK;
}

// Layout 3 ("Depth-adaptive Inference of Looped Language Models via
// Continuous Depth Batching": boundary stages queued apart from the loop
// steps): two graphs on two streams with no join per tick.  The loop step's
// graph plans the lanes in their loop and runs one iteration for them; the
// boundary stage's graph claims the lanes whose loop finished, runs their
// head, token and embedding and, for those that continue, their pre blocks,
// then hands them to the loop (release_rows_kernel).  A lane's phase word
// orders the hand-offs, so a lane's own steps keep their order while the two
// streams run side by side at their own cadence.
// kLoopStepsPerGraph loop steps per graph launch (each plans its own rows):
// fewer graph boundaries, each of which cost ~10 us between two steps.  A
// boundary stage is launched (at most) once per graph launch, so the count
// also sets the boundary stages' cadence.  Measured at 64 lanes with the
// current kernels: 41.4-41.8k tokens/s with 4 steps per graph (2,556 steps
// per pass), 45.7-46.1k with 6 (2,310), 41.1k with 8 (3,072: empty steps at
// the end of a decode cost more than they save).
static int capture_loop_step(tl_ctx* c, int n_lanes, int32_t* kcount) {
  const bool plain_loop = c->cfg.n_loop_layers <= 2;  // as in the tick graph
  const int64_t l0 = c->launches;
  for (int k = 0; k < kLoopStepsPerGraph; ++k) {
    TickConds tc{};
    if (!plain_loop) TL_TRY(new_handle(c->stream, &tc.h[2]));
    tc.use = plain_loop ? 0 : 4;
    TL_TRY(plan_tick(c, n_lanes, tc, 2));
    if (plain_loop) {
      TL_TRY(loop_iteration(c, n_lanes, nullptr, loop_path(n_lanes)));
    } else {
      cudaGraph_t body[2];
      int64_t nk[2] = {0, 0};
      TL_TRY(add_conditional(c->stream, tc.h[2], cudaGraphCondTypeSwitch, 2, body));
      TL_TRY(capture_body(c, body[0], &nk[0], [&] { return loop_iteration(c, n_lanes, nullptr, PATH_GEMV); }));
      TL_TRY(capture_body(c, body[1], &nk[1], [&] { return loop_iteration(c, n_lanes, nullptr, PATH_TC); }));
      kcount[4] = (int32_t)nk[0];
      kcount[5] = (int32_t)nk[1];
    }
  }
  c->loop_launches = c->launches - l0;  // plain nodes (kernels in the chosen body are counted on the device)
  return TL_OK;
}

static int capture_boundary_stage(tl_ctx* c, int n_lanes, int n_new, int32_t* tok_out, int32_t* dep_out,
                                  int32_t* kcount) {
  TickConds tc{};
  for (int t = 0; t < 2; ++t) TL_TRY(new_handle(c->stream, &tc.h[t]));
  tc.use = 3;
  cudaGraph_t body[2];
  int64_t nk[2] = {0, 0};
  const int64_t l0 = c->launches;
  TL_TRY(plan_tick(c, n_lanes, tc, 1));
  TL_TRY(add_conditional(c->stream, tc.h[0], cudaGraphCondTypeSwitch, 2, body));
  TL_TRY(capture_body(c, body[0], &nk[0], [&] {
    return head_core(c, n_lanes, HEAD_DECODE, nullptr, nullptr, tok_out, dep_out, n_new, PATH_GEMV, 0);
  }));
  TL_TRY(capture_body(c, body[1], &nk[1], [&] {
    return head_core(c, n_lanes, HEAD_DECODE, nullptr, nullptr, tok_out, dep_out, n_new, PATH_TC, 0);
  }));
  kcount[0] = (int32_t)nk[0];
  kcount[1] = (int32_t)nk[1];
  TL_TRY(add_conditional(c->stream, tc.h[1], cudaGraphCondTypeSwitch, 2, body));
  TL_TRY(capture_body(c, body[0], &nk[0], [&] { return pre_blocks(c, n_lanes, PATH_GEMV); }));
  TL_TRY(capture_body(c, body[1], &nk[1], [&] { return pre_blocks(c, n_lanes, PATH_TC); }));
  kcount[2] = (int32_t)nk[0];
  kcount[3] = (int32_t)nk[1];
  TL_TRY(launch_k(c, release_rows_kernel, dim3((n_lanes + 255) / 256), dim3(256), 0, c->rows[2], c->lanes));
  c->bnd_launches = c->launches - l0;
  return TL_OK;
}

// Captures fn() as a graph on cap_stream and instantiates it into *exec.
template <class F>
static int capture_graph(tl_ctx* c, cudaGraphExec_t* exec, F fn) {
  cudaStream_t saved = c->stream;
  TL_CUDA(cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
  c->stream = c->cap_stream;
  const int st = fn();
  c->stream = saved;
  c->sc = &c->scr[0];
  c->prio = 0;
  c->hold_entered = 0;
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(c->cap_stream, &g);
  if (st != TL_OK) {
    if (g) cudaGraphDestroy(g);
    return st;
  }
  TL_CUDA(e);
  const cudaError_t ei = cudaGraphInstantiate(exec, g, 0);
  cudaGraphDestroy(g);
  return check_cuda(ei);
}

static int tick_graph(tl_ctx* c, int n_lanes, int n_new, int32_t* tok_out, int32_t* dep_out) {
  const bool async = c->layout == 3;
  if ((async ? (c->loop_exec && c->bnd_exec) : c->tick_exec != nullptr) && c->tick_lanes == n_lanes &&
      c->tick_new == n_new && c->tick_tok == tok_out && c->tick_dep == dep_out && same_ee(c->tick_ee, c->ee) &&
      c->tick_warm.tokens == c->warm.tokens && c->tick_warm.L == c->warm.L &&
      c->tick_cascade == c->cascade_active && c->tick_entry == c->entry_iter && c->tick_layout == c->layout)
    return TL_OK;
  for (cudaGraphExec_t* g : {&c->tick_exec, &c->loop_exec, &c->bnd_exec})
    if (*g) {
      cudaGraphExecDestroy(*g);
      *g = nullptr;
    }
  const int64_t l0 = c->launches, s0 = c->steps;
  int32_t kcount[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int st = TL_OK;
  if (async) {
    st = capture_graph(c, &c->loop_exec, [&] { return capture_loop_step(c, n_lanes, kcount); });
    if (st == TL_OK)
      st = capture_graph(c, &c->bnd_exec, [&] {
        c->sc = &c->scr[1];
        c->prio = c->prio_hi;
        c->hold_entered = 1;
        return capture_boundary_stage(c, n_lanes, n_new, tok_out, dep_out, kcount);
      });
  } else {
    st = capture_graph(c, &c->tick_exec, [&] { return capture_tick(c, n_lanes, n_new, tok_out, dep_out, kcount); });
  }
  c->launches = l0;
  c->steps = s0;
  TL_TRY(st);
  // the row-table kernels add the chosen bodies' kernel counts on the device
  TL_CUDA(cudaMemcpyAsync(c->body_kernels, kcount, sizeof(kcount), cudaMemcpyHostToDevice, c->stream));
  TL_CUDA(cudaStreamSynchronize(c->stream));
  c->tick_lanes = n_lanes;
  c->tick_new = n_new;
  c->tick_tok = tok_out;
  c->tick_dep = dep_out;
  c->tick_ee = c->ee;
  c->tick_warm = c->warm;
  c->tick_cascade = c->cascade_active;
  c->tick_entry = c->entry_iter;
  c->tick_layout = c->layout;
  c->tick_launches = 1 + c->tick_loop_kernels;  // the planning kernel and the loop step's plain nodes
  return TL_OK;
}

// Where a decode's entering lanes run their first loop iteration, and whether
// boundary stages run apart from the loop steps.  In the boundary stage (same
// tick) a token costs its depth in ticks; at the next tick it costs one tick
// more, but the boundary stage is shorter and runs beside the loop step.  On
// their own stream (layout 3) the loop steps no longer wait for the boundary
// stage at every tick, and a lane waits for it only when its own loop has
// finished.  Measured on the B200: 64 lanes at L ~ Poisson(8): 29.0k tokens/s
// with layout 3, 25.6k with layout 2, 24.1k with layout 1; one lane at L = 8:
// 1,829 with layout 1, 1,715 with layout 2; 256 lanes at L in 1..4: 7.9k with
// layout 1, 7.3k with layouts 2 and 3.  Automatic: layout 3 for batches of
// 32+ lanes whose mean L is 6 or more, else layout 1.
static void resolve_entry(tl_ctx* c, const int32_t* host_L, int n_lanes) {
  int mode = c->overlap_mode;
  if (mode == 0) {
    double sum = 0;
    for (int i = 0; i < n_lanes; ++i) sum += host_L[i];
    mode = (n_lanes >= 32 && sum >= 6.0 * n_lanes) ? 3 : 1;
  }
  // the asynchronous layout needs graphs; run individually, its stages take layout 2's order
  if (mode == 3 && !(c->graphs_enabled && c->prof_mask == 0)) mode = 2;
  c->layout = mode;
  c->entry_iter = mode == 1 ? 1 : 0;
}

// Layout 3's host loop: loop steps on `stream` as in the tick loop; a
// boundary stage on bstream whenever fewer than two are queued there.  When
// the loop found no rows (all live lanes at or in a boundary stage), the next
// step waits for the last queued boundary stage.
static int decode_async(tl_ctx* c, int n_lanes, int n_new) {
  TL_CUDA(cudaEventRecord(c->fork_ev, c->stream));  // the boundary stream starts after the decode's set-up
  TL_CUDA(cudaStreamWaitEvent(c->bstream, c->fork_ev, 0));
  int64_t nb = 0;
  auto launch_bnd = [&]() -> int {
    TL_CUDA(cudaGraphLaunch(c->bnd_exec, c->bstream));
    TL_CUDA(cudaEventRecord(c->b_ev[nb % kBRing], c->bstream));
    ++nb;
    c->bnd_stages++;
    c->launches += c->bnd_launches;
    return TL_OK;
  };
  auto run = [&]() -> int {
    TL_TRY(launch_bnd());
    // safety bound only: a step with rows advances some lane by an iteration, and empty steps are followed
    // by a wait for the boundary stream
    const int64_t max_ticks = ((int64_t)n_lanes * n_new * (c->cfg.L_max + 1) + 4) * (kAliveRing + 1);
    for (int64_t t = 0; t < max_ticks; ++t) {
      if (t >= kAliveRing - 1) {
        const int64_t q = (t - (kAliveRing - 1)) % kAliveRing;
        TL_CUDA(cudaEventSynchronize(c->alive_ev[q]));
        if (c->pinned_alive[2 * q] == 0) break;
        if (c->pinned_alive[2 * q + 1] == 0) TL_CUDA(cudaStreamWaitEvent(c->stream, c->b_ev[(nb - 1) % kBRing], 0));
      }
      TL_CUDA(cudaGraphLaunch(c->loop_exec, c->stream));
      c->launches += c->loop_launches;
      c->steps += kLoopStepsPerGraph;
      TL_CUDA(cudaMemcpyAsync(&c->pinned_alive[2 * (t % kAliveRing)], c->alive, 8, cudaMemcpyDeviceToHost,
                              c->stream));
      TL_CUDA(cudaEventRecord(c->alive_ev[t % kAliveRing], c->stream));
      if (nb < 2) {
        TL_TRY(launch_bnd());
      } else {
        const cudaError_t q = cudaEventQuery(c->b_ev[(nb - 2) % kBRing]);
        if (q == cudaSuccess) TL_TRY(launch_bnd());
        else if (q != cudaErrorNotReady) return check_cuda(q);
      }
    }
    return TL_OK;
  };
  const int st = run();
  // the decode ends when both streams have, on every path
  TL_CUDA(cudaEventRecord(c->join_ev, c->bstream));
  TL_CUDA(cudaStreamWaitEvent(c->stream, c->join_ev, 0));
  return st;
}

static int decode_impl(tl_ctx* c, int n_lanes, int n_new, int32_t* tok_out, int32_t* dep_out) {
  TL_TRY(launch_k(c, decode_init_kernel, dim3((n_lanes + 255) / 256), dim3(256), 0, c->lanes, n_lanes, c->L_stage, n_new, c->status));
  // per-kind event profiling needs individual launches; otherwise replay a captured tick
  const bool graphs = c->prof_mask == 0 && c->graphs_enabled;
  if (graphs) TL_TRY(tick_graph(c, n_lanes, n_new, tok_out, dep_out));
  if (c->layout == 3) return decode_async(c, n_lanes, n_new);
  // upper bound on ticks: every token runs at most L_max iterations, plus the first
  const int64_t max_ticks = (int64_t)n_new * (c->cfg.L_max + 2) + 4;
  for (int64_t t = 0; t < max_ticks; ++t) {
    // lagged poll: tick t - (ring-1) must be known before launching tick t
    if (t >= kAliveRing - 1) {
      const int64_t q = t - (kAliveRing - 1);
      TL_CUDA(cudaEventSynchronize(c->alive_ev[q % kAliveRing]));
      if (c->pinned_alive[2 * (q % kAliveRing)] == 0) break;
    }
    if (graphs) {
      TL_CUDA(cudaGraphLaunch(c->tick_exec, c->stream));
      c->launches += c->tick_launches;
      c->steps++;
    } else {
      TL_TRY(enqueue_tick(c, n_lanes, n_new, tok_out, dep_out));
    }
    // the alive count was written by the tick's first kernel
    TL_CUDA(cudaMemcpyAsync(&c->pinned_alive[2 * (t % kAliveRing)], c->alive, 8, cudaMemcpyDeviceToHost, c->stream));
    TL_CUDA(cudaEventRecord(c->alive_ev[t % kAliveRing], c->stream));
  }
  return TL_OK;
}

extern "C" int tl_decode(tl_ctx* c, const int32_t* host_L, int32_t n_lanes, int32_t n_new, int32_t* tok_out,
                         int32_t* dep_out) {
  if (!c || !host_L) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  if (n_lanes < 1 || n_lanes > c->cfg.max_lanes || n_new < 1) return TL_EINVAL;
  for (int i = 0; i < n_lanes; ++i) {
    if (host_L[i] < 1 || host_L[i] > c->cfg.L_max) return TL_EINVAL;
    if (c->lane_L[i] == 0) return TL_ESTATE;
    if (host_L[i] > c->lane_L[i]) return TL_EKV;
  }
  TL_CUDA(cudaMemcpyAsync(c->L_stage, host_L, (size_t)n_lanes * 4, cudaMemcpyHostToDevice, c->stream));
  resolve_entry(c, host_L, n_lanes);
  return decode_impl(c, n_lanes, n_new, tok_out, dep_out);
}

extern "C" int tl_generate(tl_ctx* c, const int32_t* host_prompts, int32_t n_lanes, int32_t T,
                           const int32_t* host_L, int32_t n_new, int32_t* host_tok, int32_t* host_dep) {
  if (!c || !host_prompts || !host_L || !host_tok) return TL_EINVAL;
  if (!c->loaded) return TL_ESTATE;
  if (n_lanes < 1 || n_lanes > c->cfg.max_lanes || n_new < 1 || T < 1 || T + n_new - 1 > c->cfg.max_seq)
    return TL_EINVAL;
  if (T > c->lay.max_prefill) return TL_EINVAL;
  // prompts in batches of as many lanes as the prompt rows allow
  const int per_batch = (int)(c->lay.max_prefill / T);
  for (int i0 = 0; i0 < n_lanes; i0 += per_batch) {
    std::vector<PromptLane> in;
    for (int i = i0; i < n_lanes && i < i0 + per_batch; ++i)
      in.push_back(PromptLane{i, host_prompts + (size_t)i * T, T, host_L[i]});
    TL_TRY(prefill_impl(c, in, -1, 0, nullptr));
  }
  TL_CUDA(cudaMemcpyAsync(c->L_stage, host_L, (size_t)n_lanes * 4, cudaMemcpyHostToDevice, c->stream));
  resolve_entry(c, host_L, n_lanes);
  TL_TRY(decode_impl(c, n_lanes, n_new, c->out_tok, c->out_dep));
  TL_CUDA(cudaMemcpyAsync(host_tok, c->out_tok, (size_t)n_lanes * n_new * 4, cudaMemcpyDeviceToHost, c->stream));
  if (host_dep)
    TL_CUDA(cudaMemcpyAsync(host_dep, c->out_dep, (size_t)n_lanes * n_new * 4, cudaMemcpyDeviceToHost, c->stream));
  TL_CUDA(cudaStreamSynchronize(c->stream));
  return TL_OK;
}

extern "C" int tl_stats_get(tl_ctx* c, tl_stats* out) {
  if (!c || !out) return TL_EINVAL;
  unsigned long long ctr[4];
  int32_t st = 0;
  TL_CUDA(cudaMemcpyAsync(ctr, c->counters, 32, cudaMemcpyDeviceToHost, c->stream));
  TL_CUDA(cudaMemcpyAsync(&st, c->status, 4, cudaMemcpyDeviceToHost, c->stream));
  TL_CUDA(cudaMemsetAsync(c->status, 0, 4, c->stream));
  TL_CUDA(cudaStreamSynchronize(c->stream));
  out->loop_steps = c->steps;
  out->lane_iterations = (int64_t)ctr[0];
  out->tokens_emitted = (int64_t)ctr[1];
  out->prefill_tokens = c->prefill_tokens;
  out->kernel_launches = c->launches + (int64_t)ctr[2];
  out->device_status = st;
  out->kv_pages_used = c->lay.n_pages - (int32_t)c->free_pages.size();
  out->entry_in_boundary = c->entry_iter;
  out->tick_layout = c->layout;
  out->boundary_stages = c->bnd_stages;
  return TL_OK;
}

extern "C" int tl_lane_state_bytes(tl_ctx* c, size_t* out) {
  if (!c || !out) return TL_EINVAL;
  *out = (size_t)c->cfg.max_lanes * (sizeof(LaneState) + (size_t)c->cfg.d * 4);
  return TL_OK;
}

extern "C" int tl_lane_state_save(tl_ctx* c, void* dev_dst) {
  if (!c || !dev_dst) return TL_EINVAL;
  const size_t a = (size_t)c->cfg.max_lanes * sizeof(LaneState), b = (size_t)c->cfg.max_lanes * c->cfg.d * 4;
  TL_CUDA(cudaMemcpyAsync(dev_dst, c->lanes, a, cudaMemcpyDeviceToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync((char*)dev_dst + a, c->h, b, cudaMemcpyDeviceToDevice, c->stream));
  return TL_OK;
}

extern "C" int tl_lane_state_load(tl_ctx* c, const void* dev_src) {
  if (!c || !dev_src) return TL_EINVAL;
  const size_t a = (size_t)c->cfg.max_lanes * sizeof(LaneState), b = (size_t)c->cfg.max_lanes * c->cfg.d * 4;
  TL_CUDA(cudaMemcpyAsync(c->lanes, dev_src, a, cudaMemcpyDeviceToDevice, c->stream));
  TL_CUDA(cudaMemcpyAsync(c->h, (const char*)dev_src + a, b, cudaMemcpyDeviceToDevice, c->stream));
  return TL_OK;
}

extern "C" int tl_profile_begin(tl_ctx* c, int32_t kind_mask) {
  if (!c || (kind_mask & ~0xE)) return TL_EINVAL;
  if (c->prof_ev.empty()) {
    c->prof_ev.resize(kProfRing);
    c->prof_kind_of.assign(kProfRing, 0);
    for (auto& e : c->prof_ev) {
      TL_CUDA(cudaEventCreate(&e[0]));
      TL_CUDA(cudaEventCreate(&e[1]));
    }
  }
  c->prof_mask = kind_mask;
  c->prof_head = c->prof_tail = 0;
  for (int k = 0; k < 4; ++k) {
    c->prof_groups[k] = 0;
    c->prof_ms[k] = 0.0;
  }
  return TL_OK;
}

extern "C" int tl_profile_end(tl_ctx* c, int64_t* groups, double* total_ms) {
  if (!c) return TL_EINVAL;
  while (c->prof_tail < c->prof_head) TL_TRY(prof_fold_oldest(c));
  for (int k = 0; k < 4; ++k) {
    if (groups) groups[k] = c->prof_groups[k];
    if (total_ms) total_ms[k] = c->prof_ms[k];
  }
  c->prof_mask = 0;
  return TL_OK;
}

extern "C" int tl_set_tick_overlap(tl_ctx* c, int32_t mode) {
  if (!c || mode < 0 || mode > 3) return TL_EINVAL;
  c->overlap_mode = mode;
  return TL_OK;
}

extern "C" int tl_set_cascade(tl_ctx* c, int32_t enabled) {
  if (!c) return TL_EINVAL;
  c->cascade_enabled = enabled != 0;
  return update_cascade(c);
}

extern "C" int tl_set_graphs(tl_ctx* c, int32_t enabled) {
  if (!c) return TL_EINVAL;
  c->graphs_enabled = enabled != 0;
  return TL_OK;
}
