// Decode-path kernels: lane compaction, RMSNorm, projections (W4A16 / BF16),
// RoPE + KV append, paged per-iteration attention, early-exit rule, head
// argmax and the boundary-stage transitions.
//
// Model block and head: see include/tl.h.  Every kernel that depends on a row
// count reads it from device memory (Rows::n) so a step can be replayed with
// no host involvement; grids are sized for the largest row count.
#pragma once

#include "common.cuh"

namespace tl {

// ------------------------------------------------------------- weights ----

struct MatView {
  int32_t fmt;          // TL_FMT_INT4 / TL_FMT_BF16
  int32_t N, K, group;
  const uint8_t* q;     // INT4 packed [N][K/2]
  const __half* s;      // INT4 scales [N][K/group]
  const uint16_t* bf;   // BF16 [N][K]
};

enum Epi : int32_t { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_ARGMAX = 3 };

// Output side of a projection.  Row r of the activations is output row r; for
// EPI_RESID it is added into h[map ? map[r] : r][:]; for EPI_ARGMAX each CTA
// writes its best (value, index) per row into part_*[r * n_parts + blockIdx.x]
// and, when logits != null, the logits into logits[lmap[r] * ldo + n].
struct ProjOut {
  int32_t epi;
  float* out;            // EPI_STORE / EPI_SWIGLU: [rows][ldo]
  int32_t ldo;
  float* h;              // EPI_RESID: residual rows, leading dimension N
  const int32_t* map;    // EPI_RESID row -> h row (null = identity)
  float* logits;         // EPI_ARGMAX (nullable)
  const int32_t* lmap;   // EPI_ARGMAX row -> logits row
  float* part_val;
  int32_t* part_idx;
  int32_t n_parts;
  int32_t* n_parts_dev;  // EPI_ARGMAX: the kernel that did the work stores n_parts here
};

// Orders (value, index) pairs: larger value first, lower index on ties.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// ---------------------------------------------------------- row tables ----

enum RowSel : int32_t { SEL_LOOP = 0, SEL_BOUNDARY = 1, SEL_ENTERED = 2, SEL_MASK = 3 };

// One CTA of 1024 threads; thread i looks at lane i.  Selects lanes, writes the
// compacted row table (lane order), and for SEL_LOOP copies h -> h_in (the loop
// input that the relative-L2 test compares against).  SEL_LOOP also applies an
// optional per-lane L request: a request above the lane's cap sets ST_EKV and
// keeps the lane out; a request at or below the iterations already done
// finishes the lane's loop without running.
// Conditional graph nodes driven by a row table (cond_mode): 1 = IF (rows > 0);
// 2 = SWITCH over (rows <= 8 -> body 0, CUDA-core GEMV variant; rows > 8 ->
// body 1, tensor-core variant; no rows -> no body).  body_kernels[v] is the
// number of kernels body v launches; it is added to *kernel_count.
enum CondMode : int32_t { COND_NONE = 0, COND_IF = 1, COND_SWITCH = 2 };

__global__ void build_rows_kernel(LaneState* __restrict__ lanes, int n_lanes, int32_t sel,
                                  const uint8_t* __restrict__ mask, const int32_t* __restrict__ per_lane_L,
                                  Rows rows, uint8_t* __restrict__ exit_mask_out, int32_t* __restrict__ alive,
                                  int32_t* __restrict__ status, cudaGraphConditionalHandle cond, int32_t cond_mode,
                                  int32_t gemv_max_rows, const int32_t* __restrict__ body_kernels,
                                  unsigned long long* __restrict__ kernel_count) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int32_t warp_cnt[32];
  __shared__ int32_t alive_cnt;
  const int i = threadIdx.x;
  if (i == 0) alive_cnt = 0;
  __syncthreads();
  int take = 0;
  if (i < n_lanes) {
    LaneState& st = lanes[i];
    const bool on = (mask == nullptr) || mask[i] != 0;
    if (st.phase == PH_LOOP || st.phase == PH_BOUNDARY) atomicAdd(&alive_cnt, 1);
    if (sel == SEL_LOOP) {
      if (exit_mask_out && on) exit_mask_out[i] = 0;
      if (on && st.phase == PH_LOOP) {
        take = 1;
        if (per_lane_L) {
          const int L = per_lane_L[i];
          if (L < 1 || L > st.L_cap) {
            set_status(status, ST_EKV);
            take = 0;
          } else {
            st.L_req = L;
            st.L_run = L;
            if (st.iter >= L) {  // already ran what is now requested: loop finished
              st.phase = PH_BOUNDARY;
              st.depth = st.iter;
              if (exit_mask_out) exit_mask_out[i] = 1;
              take = 0;
            }
          }
        }
      }
    } else if (sel == SEL_BOUNDARY) {
      take = on && st.phase == PH_BOUNDARY;
    } else if (sel == SEL_ENTERED) {
      take = st.entered;
      st.entered = 0;
    } else {
      take = on;
    }
  }
  // block-wide exclusive scan of `take`
  const int lane = i & 31, w = i >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (lane == 0) warp_cnt[w] = __popc(bal);
  __syncthreads();
  if (w == 0) {
    int v = warp_cnt[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    warp_cnt[lane] = v;  // inclusive
  }
  __syncthreads();
  const int base = (w == 0) ? 0 : warp_cnt[w - 1];
  const int r = base + __popc(bal & ((1u << lane) - 1u));
  if (take) {
    rows.lane[r] = i;
    rows.pos[r] = lanes[i].pos;
    rows.iter[r] = lanes[i].iter;
  }
  if (i == 0) {
    const int n = warp_cnt[31];
    rows.n[0] = n;
    if (alive) alive[0] = alive_cnt;
    if (cond_mode == COND_IF) {
      cudaGraphSetConditional(cond, n > 0 ? 1u : 0u);
      if (n > 0) atomicAdd(kernel_count, (unsigned long long)body_kernels[0]);
    } else if (cond_mode == COND_SWITCH) {
      const unsigned v = n == 0 ? 2u : (n <= gemv_max_rows ? 0u : 1u);
      cudaGraphSetConditional(cond, v);
      if (v < 2) atomicAdd(kernel_count, (unsigned long long)body_kernels[v]);
    }
  }
}

// The three row tables of a decode tick from the lane states at its start,
// in lane order, decided one stage ahead: boundary rows (loop finished: head,
// token), entered rows (boundary lanes that will take a token and continue:
// their pre blocks and first loop iteration run at position pos + 1, in the
// boundary stage) and loop rows (lanes already in their loop), so the
// boundary stage and the loop step touch disjoint lanes and run
// concurrently.  Whether a boundary lane continues
// is fixed before its head runs, by the same test head_finalize_kernel applies
// (n_emitted + 1 < n_target and pos + 1 < max_seq).  alive = lanes in their
// loop or at a boundary.  With conditional graph nodes, sets the SWITCH value
// of each table whose bit is set in cond.use, as build_rows_kernel does.
// which: bit 0 plans the boundary and entered tables, bit 1 the loop table
// and the alive count (both: one tick); a boundary plan alone (the stage runs
// apart from the loop steps) also claims its lanes (PH_CLAIMED), and alive
// then counts claimed lanes too.  alive[1] = loop rows.  One CTA of 1024
// threads; thread i looks at lane i.
struct TickConds {
  cudaGraphConditionalHandle h[3];  // boundary, entered, loop
  int32_t use;                      // bit t: h[t] is a live handle
};

__global__ void plan_tick_kernel(LaneState* lanes, int n_lanes, Rows boundary, Rows entered, Rows loop,
                                 int32_t* __restrict__ alive, int max_seq, TickConds cond, int32_t gemv_max_rows,
                                 const int32_t* __restrict__ body_kernels,
                                 unsigned long long* __restrict__ kernel_count, int32_t which) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int32_t cnt[3][32];
  const int i = threadIdx.x, lane = i & 31, w = i >> 5;
  int take[3] = {0, 0, 0}, live = 0, pos = 0, iter = 0;
  if (i < n_lanes) {
    const int ph = phase_acquire(&lanes[i].phase);
    const LaneState st = lanes[i];
    pos = st.pos;
    iter = st.iter;
    const bool b = ph == PH_BOUNDARY;
    const bool e = b && st.n_emitted + 1 < st.n_target && st.pos + 1 < max_seq;
    take[0] = (which & 1) && b;
    take[1] = (which & 1) && e;
    take[2] = (which & 2) && ph == PH_LOOP;  // entering lanes join the loop at the next tick
    live = ph == PH_LOOP || b || ph == PH_CLAIMED;
    if (which == 1 && b) lanes[i].phase = PH_CLAIMED;
  }
  unsigned bal[3];
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    bal[t] = __ballot_sync(0xffffffffu, take[t]);
    if (lane == 0) cnt[t][w] = __popc(bal[t]);
  }
  const unsigned live_bal = __ballot_sync(0xffffffffu, live);
  __shared__ int32_t live_cnt[32];
  if (lane == 0) live_cnt[w] = __popc(live_bal);
  __syncthreads();
  if (w < 3) {  // warp t scans table t's per-warp counts
    int v = cnt[w][lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    cnt[w][lane] = v;  // inclusive
  } else if (w == 3) {
    const int v = warp_sum(live_cnt[lane]);
    if (lane == 0) live_cnt[0] = v;
  }
  __syncthreads();
  const unsigned below = (1u << lane) - 1u;
  const Rows* tab[3] = {&boundary, &entered, &loop};
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    if (take[t]) {
      const int r = (w == 0 ? 0 : cnt[t][w - 1]) + __popc(bal[t] & below);
      const bool fresh = t == 1;  // entering: next position, iteration 0
      tab[t]->lane[r] = i;
      tab[t]->pos[r] = fresh ? pos + 1 : pos;
      tab[t]->iter[r] = fresh ? 0 : iter;
    }
  }
  if (i == 0) {
    int n[3];
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      n[t] = cnt[t][31];
      if ((which >> (t == 2 ? 1 : 0)) & 1) tab[t]->n[0] = n[t];
    }
    if (alive && (which & 2)) {
      alive[0] = live_cnt[0];
      alive[1] = n[2];
    }
    unsigned long long k = 0;
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      if (!((cond.use >> t) & 1)) continue;
      const unsigned v = n[t] == 0 ? 2u : (n[t] <= gemv_max_rows ? 0u : 1u);
      cudaGraphSetConditional(cond.h[t], v);
      if (v < 2) k += (unsigned long long)body_kernels[2 * t + v];
    }
    if (k) atomicAdd(kernel_count, k);
  }
}

// --------------------------------------------------------------- norms ----

// out[r] = RMSNorm(h[map ? map[r] : r]) * g, fp32 (and an fp16 copy for the
// tensor-core projections when out16 is given, split into hi and lo halves
// with split16, see act16_put).  One CTA per row.  When h_in is
// given, also copies the source row there (indexed like h); when zero_rows is
// given, clears row r of that [rows][zero_cols] accumulator, which the next
// (split-K) projection adds into.  Does nothing more when the row count is
// at most min_rows (those counts are served by a GEMV that normalises by
// itself).  add (prompt batches): first h[row r] += add[r] for every r <
// *n_add, the residual of a projection that stored its output instead of
// adding it (the grid covers those rows too).
__global__ void rmsnorm_rows_kernel(float* __restrict__ h, const int32_t* __restrict__ map,
                                    const int32_t* __restrict__ n_rows, int d, const float* __restrict__ g,
                                    float eps, float* __restrict__ out, float* __restrict__ h_in,
                                    __half* __restrict__ out16, float* __restrict__ zero_rows, int zero_cols,
                                    int min_rows, const float* __restrict__ add, const int32_t* __restrict__ n_add,
                                    int split16) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int n = n_rows[0];
  if (add && r < n_add[0]) {  // deferred residual of the previous projection: h[row r] += add[r]
    float* hx = h + (int64_t)(map ? map[r] : r) * d;
    for (int k = threadIdx.x; k < d; k += blockDim.x) hx[k] += add[(int64_t)r * d + k];
    __syncthreads();
  }
  if (r >= n || n <= min_rows) return;
  const int src = map ? map[r] : r;
  const float* x = h + (int64_t)src * d;
  float ss = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) ss += x[k] * x[k];
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    const float v = x[k];
    const float y = v * inv * g[k];
    out[(int64_t)r * d + k] = y;
    if (out16) act16_put(out16, r, d, k, y, split16);
    if (h_in) h_in[(int64_t)src * d + k] = v;
  }
  if (zero_rows)
    for (int k = threadIdx.x; k < zero_cols; k += blockDim.x) zero_rows[(int64_t)r * zero_cols + k] = 0.f;
}

// ------------------------------------------------------------ embedding ----

// h[dst] = dequantised embedding row of token; one CTA per row.
__device__ __forceinline__ void embed_row(const MatView& E, int tok, float* __restrict__ dst, int d) {
  if (E.fmt == TL_FMT_INT4) {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(E.q + (int64_t)tok * (d / 2));
    const __half* s = E.s + (int64_t)tok * (d / E.group);
    for (int wi = threadIdx.x; wi < d / 8; wi += blockDim.x) {
      const uint32_t w = q[wi];
      const float sc = __half2float(s[(8 * wi) / E.group]);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[8 * wi + e] = nib_to_f(w, 4 * nib_pos(e)) * sc;
    }
  } else {
    const uint16_t* p = E.bf + (int64_t)tok * d;
    for (int k = threadIdx.x; k < d; k += blockDim.x) dst[k] = bf16_bits_to_f(p[k]);
  }
}

__global__ void embed_rows_kernel(MatView E, const int32_t* __restrict__ tokens, int n, int d,
                                  float* __restrict__ h, int32_t* __restrict__ status) {
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x;
  if (r >= n) return;
  int tok = tokens[r];
  if (tok < 0 || tok >= E.N) { set_status(status, ST_BAD_TOKEN); tok = 0; }
  embed_row(E, tok, h + (int64_t)r * d, d);
}

// ---------------------------------------------------------- GEMV (few rows) ----
//
// y[r][n] = sum_k x[r][k] * W[n][k] for R activation rows at a time held in
// shared memory (fp32, 16-byte slots XOR-swizzled so that 32 lanes reading
// consecutive 128-byte segments do not collide on banks).  One warp per output
// feature (two for EPI_SWIGLU: gate row n and up row n), 8 warps per CTA; each
// lane owns 32-element chunks of K: 16 bytes of INT4 (one fp16 scale per chunk,
// since the group is a multiple of 32) or 64 bytes of BF16.  INT4 values are
// (u - 8) exactly in fp32; the group scale multiplies each chunk's partial sum.

constexpr int GEMV_WARPS = 8;

__device__ __forceinline__ int swz_slot(int f) { return (f & ~7) | ((f & 7) ^ ((f >> 3) & 7)); }

// Raw bytes of one 32-element chunk of a weight row: INT4 16 bytes, BF16 64.
template <int FMT>
struct Chunk {
  uint4 v[FMT == TL_FMT_INT4 ? 1 : 4];
  float sc;
};

template <int FMT>
__device__ __forceinline__ void load_chunk_raw(const MatView& W, int n, int c, Chunk<FMT>& ch) {
  if constexpr (FMT == TL_FMT_INT4) {
    ch.v[0] = __ldg(reinterpret_cast<const uint4*>(W.q + (int64_t)n * (W.K / 2) + c * 16));
    ch.sc = __half2float(W.s[(int64_t)n * (W.K / W.group) + (c * 32) / W.group]);
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(W.bf + (int64_t)n * W.K + c * 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) ch.v[j] = __ldg(p + j);
    ch.sc = 1.f;
  }
}

template <int FMT>
__device__ __forceinline__ void unpack_chunk(const Chunk<FMT>& ch, float (&w)[32]) {
  if constexpr (FMT == TL_FMT_INT4) {
    const uint32_t u[4] = {ch.v[0].x, ch.v[0].y, ch.v[0].z, ch.v[0].w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) w[8 * j + e] = nib_to_f(u[j], 4 * nib_pos(e));
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t u[4] = {ch.v[j].x, ch.v[j].y, ch.v[j].z, ch.v[j].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[8 * j + 2 * e] = __uint_as_float(u[e] << 16);
        w[8 * j + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
      }
    }
  }
}

template <int R>
__device__ __forceinline__ void dot_chunk(const float* __restrict__ xs, int K, int c, const float (&w)[32],
                                          float sc, float (&acc)[R]) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float4* row = reinterpret_cast<const float4*>(xs + r * K);
    float p = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 x = row[swz_slot(8 * c + j)];
      p = fmaf(w[4 * j], x.x, p);
      p = fmaf(w[4 * j + 1], x.y, p);
      p = fmaf(w[4 * j + 2], x.z, p);
      p = fmaf(w[4 * j + 3], x.w, p);
    }
    acc[r] = fmaf(p, sc, acc[r]);
  }
}

// One warp owns RPW consecutive output features (for EPI_SWIGLU: gate row n
// and up row n, RPW = 1); a lane loads the raw chunks of all of them before
// using any, so a warp keeps RPW (x2) 16-byte loads in flight per lane.
template <int FMT, int R, int EPI, int RPW>
__device__ __forceinline__ void gemv_rows(const float* __restrict__ xs, int r0, int rows, const MatView& W,
                                          const MatView& W2, const ProjOut& o, float (*best_v)[8],
                                          int (*best_i)[8]) {
  const int K = W.K, N = W.N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbase = (blockIdx.x * GEMV_WARPS + warp) * RPW;
  const int nch = K / 32;
  float acc[RPW][R], acc2[R];
#pragma unroll
  for (int f = 0; f < RPW; ++f)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[f][r] = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) acc2[r] = 0.f;
  for (int c = lane; c < nch; c += 32) {
    Chunk<FMT> ch[RPW];
#pragma unroll
    for (int f = 0; f < RPW; ++f)
      if (nbase + f < N) load_chunk_raw<FMT>(W, nbase + f, c, ch[f]);
    Chunk<FMT> ch2;
    if constexpr (EPI == EPI_SWIGLU)
      if (nbase < N) load_chunk_raw<FMT>(W2, nbase, c, ch2);
#pragma unroll
    for (int f = 0; f < RPW; ++f) {
      if (nbase + f < N) {
        float w[32];
        unpack_chunk<FMT>(ch[f], w);
        dot_chunk<R>(xs, K, c, w, ch[f].sc, acc[f]);
      }
    }
    if constexpr (EPI == EPI_SWIGLU) {
      if (nbase < N) {
        float w[32];
        unpack_chunk<FMT>(ch2, w);
        dot_chunk<R>(xs, K, c, w, ch2.sc, acc2);
      }
    }
  }
#pragma unroll
  for (int f = 0; f < RPW; ++f)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[f][r] = warp_sum(acc[f][r]);
  if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll
    for (int r = 0; r < R; ++r) acc2[r] = warp_sum(acc2[r]);
  }
  if constexpr (EPI == EPI_ARGMAX) {
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int f = 0; f < RPW; ++f)
          if (nbase + f < N && better(acc[f][r], nbase + f, bv, bi)) { bv = acc[f][r]; bi = nbase + f; }
        best_v[warp][r] = bv;
        best_i[warp][r] = bi;
      }
    }
    if (o.logits && lane < R && r0 + lane < rows) {
#pragma unroll
      for (int f = 0; f < RPW; ++f) {
        float v = acc[f][0];
#pragma unroll
        for (int r = 1; r < R; ++r) if (lane == r) v = acc[f][r];
        if (nbase + f < N) o.logits[(int64_t)o.lmap[r0 + lane] * o.ldo + nbase + f] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < R && r0 + threadIdx.x < rows) {
      const int r = threadIdx.x;
      float bv = best_v[0][r];
      int bi = best_i[0][r];
      for (int ww = 1; ww < GEMV_WARPS; ++ww)
        if (better(best_v[ww][r], best_i[ww][r], bv, bi)) { bv = best_v[ww][r]; bi = best_i[ww][r]; }
      o.part_val[(int64_t)(r0 + r) * o.n_parts + blockIdx.x] = bv;
      o.part_idx[(int64_t)(r0 + r) * o.n_parts + blockIdx.x] = bi;
    }
  } else if (lane < R && r0 + lane < rows) {
    const int r = r0 + lane;
#pragma unroll
    for (int f = 0; f < RPW; ++f) {
      const int n = nbase + f;
      if (n >= N) continue;
      float v = acc[f][0], v2 = acc2[0];
#pragma unroll
      for (int rr = 1; rr < R; ++rr)
        if (lane == rr) { v = acc[f][rr]; v2 = acc2[rr]; }
      if constexpr (EPI == EPI_STORE) {
        o.out[(int64_t)r * o.ldo + n] = v;
      } else if constexpr (EPI == EPI_SWIGLU) {
        o.out[(int64_t)r * o.ldo + n] = silu_f(v) * v2;
      } else {
        const int hr = o.map ? o.map[r] : r;
        o.h[(int64_t)hr * N + n] += v;
      }
    }
  }
}

// Rows are taken 8 at a time (fewer for the last chunk, dispatched to a body
// compiled for that count).  With skip_above > 0 the kernel does nothing when
// the row count exceeds it (the tensor-core kernel launched beside it takes
// those).  A CTA covers GEMV_WARPS * RPW output features.
template <int FMT, int EPI, int RPW>
__global__ void __launch_bounds__(GEMV_WARPS * 32)
gemv_kernel(const float* __restrict__ X, const int32_t* __restrict__ n_rows, MatView W, MatView W2, ProjOut o,
            int skip_above) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ float4 smem4[];
  float* xs = reinterpret_cast<float*>(smem4);
  __shared__ float best_v[GEMV_WARPS][8];
  __shared__ int best_i[GEMV_WARPS][8];
  const int K = W.K;
  const int rows = n_rows[0];
  if (skip_above > 0 && rows > skip_above) return;
  for (int r0 = 0; r0 < rows; r0 += 8) {
    const int nr = min(8, rows - r0);
    __syncthreads();
    for (int f = threadIdx.x; f < nr * K / 4; f += blockDim.x) {
      const int r = f / (K / 4), fi = f % (K / 4);
      smem4[r * (K / 4) + swz_slot(fi)] = reinterpret_cast<const float4*>(X + (int64_t)(r0 + r) * K)[fi];
    }
    __syncthreads();
    switch (nr) {
      case 1: gemv_rows<FMT, 1, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 2: gemv_rows<FMT, 2, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 3: gemv_rows<FMT, 3, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 4: gemv_rows<FMT, 4, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 5: gemv_rows<FMT, 5, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 6: gemv_rows<FMT, 6, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      case 7: gemv_rows<FMT, 7, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
      default: gemv_rows<FMT, 8, EPI, RPW>(xs, r0, rows, W, W2, o, best_v, best_i); break;
    }
  }
}

// --------------------------------------------------------- RoPE + KV ----

// q_out[r] = RoPE(q), and K = RoPE(k), V = v appended (fp16) to the page of
// (lane, slot, pos).  slot = slot_base + iter * slot_stride.  One CTA per row,
// d/2 threads: thread t rotates pair (i, i + hd/2) of head t / (hd/2).
__global__ void rope_kv_kernel(const float* __restrict__ qkv, float* __restrict__ q_out, Rows rows, KVGeom g,
                               const float2* __restrict__ rope_cs, int slot_base, int slot_stride,
                               const int32_t* __restrict__ map_lane, int32_t* __restrict__ status) {
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x;
  if (r >= rows.n[0]) return;
  const int d = g.H * g.hd, half = g.hd / 2;
  const int t = threadIdx.x;
  if (t >= d / 2) return;
  const int h = t / half, i = t % half;
  const int pos = rows.pos[r];
  const int lane = map_lane ? map_lane[r] : rows.lane[r];
  const int slot = slot_base + rows.iter[r] * slot_stride;
  const float2 cs = rope_cs[(int64_t)pos * half + i];
  const float* src = qkv + (int64_t)r * 3 * d;
  const int c0 = h * g.hd + i, c1 = c0 + half;
  const float q0 = src[c0], q1 = src[c1];
  q_out[(int64_t)r * d + c0] = q0 * cs.x - q1 * cs.y;
  q_out[(int64_t)r * d + c1] = q1 * cs.x + q0 * cs.y;
  const float k0 = src[d + c0], k1 = src[d + c1];
  __half* kp = kv_k_ptr(g, lane, slot, pos, h, status);
  if (kp) {
    __half* vp = kp + (int64_t)g.H * g.page_tokens * g.hd;
    kp[i] = __float2half_rn(k0 * cs.x - k1 * cs.y);
    kp[i + half] = __float2half_rn(k1 * cs.x + k0 * cs.y);
    vp[i] = __float2half_rn(src[2 * d + c0]);
    vp[i + half] = __float2half_rn(src[2 * d + c1]);
  }
}

// --------------------------------------------------- prefill attention ----
//
// Causal attention for blocks of consecutive prompt rows of one lane each: CTA
// (qb, h) takes query tile qb = tiles[qb] = (first row, row count <= 64) of
// the row table (every row of a tile belongs to one lane and the positions
// rows.pos[r] are consecutive; tiles == null: rows 64 qb .. 64 qb + 63 of a
// one-lane table) and walks key blocks of 64 positions from 0 up to its last
// query position, staging K and V once per block in shared memory (fp32) and
// keeping a running max / sum per query row.  256 threads: for the scores
// thread (ty, tx) owns rows 4ty..4ty+3 and keys 4tx..4tx+3; for the output it
// owns the same rows and dims tx*HD/16 .. +HD/16.
template <int HD>
__global__ void __launch_bounds__(256)
attn_prefill_kernel(const float* __restrict__ q, float* __restrict__ o, __half* __restrict__ o16, Rows rows,
                    const int2* __restrict__ tiles, KVGeom g, int slot, int32_t* __restrict__ status, int split16) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int BQ = 64, BK = 64, DPT = HD / 16;
  extern __shared__ float4 smem_pf[];
  float* Qs = reinterpret_cast<float*>(smem_pf);  // [HD][BQ]  (pre-scaled)
  float* Ks = Qs + HD * BQ;                        // [HD][BK]
  float* Vs = Ks + HD * BK;                        // [BK][HD]
  float* Ps = Vs + BK * HD;                        // [BQ][BK + 1]
  const int n = rows.n[0];
  const int2 tile = tiles ? tiles[blockIdx.x] : make_int2(blockIdx.x * BQ, min(BQ, n - (int)blockIdx.x * BQ));
  const int r0 = tile.x, h = blockIdx.y;
  if (r0 >= n || tile.y <= 0) return;
  const int ln = rows.lane[r0];
  const int d = g.H * HD;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int nq = min(min(BQ, tile.y), n - r0);
  const int pos_first = rows.pos[r0];
  const int pos_last = pos_first + nq - 1;
  const float scale = rsqrtf((float)HD);
  for (int i = threadIdx.x; i < BQ * HD; i += 256) {
    const int r = i / HD, dd = i % HD;
    Qs[dd * BQ + r] = (r < nq) ? q[(int64_t)(r0 + r) * d + h * HD + dd] * scale : 0.f;
  }
  float m[4], l[4], acc[4][DPT];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int j = 0; j < DPT; ++j) acc[i][j] = 0.f;
  }
  const int nkb = pos_last / BK + 1;
  for (int kb = 0; kb < nkb; ++kb) {
    const int k0 = kb * BK;
    __syncthreads();
    // stage K (transposed) and V for key positions k0 .. k0+63 (<= pos_last)
    for (int i = threadIdx.x; i < BK * (HD / 8); i += 256) {
      const int kr = i / (HD / 8), c8 = i % (HD / 8);
      const int kp = k0 + kr;
      float kv[8], vv[8];
      const __half* kptr = (kp <= pos_last) ? kv_k_ptr(g, ln, slot, kp, h, status) : nullptr;
      if (kptr) {
        const uint4 ku = *reinterpret_cast<const uint4*>(kptr + c8 * 8);
        const uint4 vu = *reinterpret_cast<const uint4*>(kptr + (int64_t)g.H * g.page_tokens * HD + c8 * 8);
        const __half2* kh = reinterpret_cast<const __half2*>(&ku);
        const __half2* vh = reinterpret_cast<const __half2*>(&vu);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = __half22float2(kh[e]), b = __half22float2(vh[e]);
          kv[2 * e] = a.x; kv[2 * e + 1] = a.y; vv[2 * e] = b.x; vv[2 * e + 1] = b.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[e] = vv[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        Ks[(c8 * 8 + e) * BK + kr] = kv[e];
        Vs[kr * HD + c8 * 8 + e] = vv[e];
      }
    }
    __syncthreads();
    // scores
    float sc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll 8
    for (int dd = 0; dd < HD; ++dd) {
      const float4 a = *reinterpret_cast<const float4*>(&Qs[dd * BQ + ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Ks[dd * BK + tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[i][j] = fmaf(av[i], bv[j], sc[i][j]);
    }
    // causal mask, online softmax per row (the 16 threads of a row group share it)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qp = pos_first + ty * 4 + i;
      float mb = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kp = k0 + tx * 4 + j;
        if (kp > qp) sc[i][j] = -INFINITY;
        mb = fmaxf(mb, sc[i][j]);
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      const float mn = fmaxf(m[i], mb);
      float ps = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float pv = (sc[i][j] == -INFINITY) ? 0.f : expf(sc[i][j] - mn);
        Ps[(ty * 4 + i) * (BK + 1) + tx * 4 + j] = pv;
        ps += pv;
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      const float corr = (m[i] == -INFINITY) ? 0.f : expf(m[i] - mn);
      l[i] = l[i] * corr + ps;
      m[i] = mn;
#pragma unroll
      for (int j = 0; j < DPT; ++j) acc[i][j] *= corr;
    }
    __syncthreads();
    // output: acc[r][dims] += P[r][k] V[k][dims]
#pragma unroll 4
    for (int k = 0; k < BK; ++k) {
      float vv[DPT];
#pragma unroll
      for (int j = 0; j < DPT; ++j) vv[j] = Vs[k * HD + tx * DPT + j];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pk = Ps[(ty * 4 + i) * (BK + 1) + k];
#pragma unroll
        for (int j = 0; j < DPT; ++j) acc[i][j] = fmaf(pk, vv[j], acc[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= nq) continue;
    const float inv = 1.f / l[i];
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      o[(int64_t)(r0 + r) * d + h * HD + tx * DPT + j] = acc[i][j] * inv;
      act16_put(o16, r0 + r, d, h * HD + tx * DPT + j, acc[i][j] * inv, split16);
    }
  }
}

// ----------------------------------------------------------- exit rule ----
//
// After a loop iteration of the row's lane: delta = ||h - h_in|| / ||h_in||
// (sums in fp64); probe at iteration l when l > min_L and (l - min_L - 1) %
// peek_every == 0; a probe with delta < tau extends the streak, any other
// probe resets it; the lane's loop finishes on streak >= patience or when l
// reaches L_run.  In logit-margin mode ("CLI Reference",
// --early-exit-logit-margin) the probe's metric is margin_lane[lane], the top-1
// minus top-2 logit of the head at this iteration (margin_kernel), and it
// succeeds when the margin is at least the threshold.  One CTA per row.
//
// L warmup: when a warmup token's loop finishes at depth D below the lane's
// requested L, the K/V it wrote at its position for iteration D (every body
// layer) are copied into the slots of iterations D+1 .. L_req, so a later,
// deeper token attends there to the deepest iteration that computed the
// position (the pages do not say what it should read; this is the reading
// taken).  Positions are written once, so the copy stays valid.
__global__ void exit_update_kernel(Rows rows, LaneState* __restrict__ lanes, const float* __restrict__ h,
                                   const float* __restrict__ h_in, int d, EEParams ee,
                                   uint8_t* __restrict__ exit_mask_out, unsigned long long* __restrict__ lane_iters,
                                   WarmParams wp, KVGeom g, int n_pre, int n_loop_layers, int32_t* __restrict__ status,
                                   const float* __restrict__ margin_lane) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ double red[32];
  __shared__ int fill_from, fill_to;
  const int r = blockIdx.x;
  if (r >= rows.n[0]) return;
  const int ln = rows.lane[r];
  LaneState& st = lanes[ln];
  const int l = st.iter + 1;
  const bool probe = ee_probe(ee, l);
  double num = 0.0, den = 0.0;
  if (probe && !ee.use_margin) {
    const float* a = h + (int64_t)ln * d;
    const float* b = h_in + (int64_t)ln * d;
    for (int k = threadIdx.x; k < d; k += blockDim.x) {
      const double x = a[k], y = b[k];
      num += (x - y) * (x - y);
      den += y * y;
    }
    num = block_sum_d(num, red);
    den = block_sum_d(den, red);
  }
  if (threadIdx.x == 0) {
    bool ex = false;
    if (probe) {
      const bool below = ee.use_margin ? ((double)margin_lane[ln] >= ee.margin)
                                       : ((den > 0.0) && (sqrt(num / den) < ee.tau));
      st.streak = below ? st.streak + 1 : 0;
      ex = st.streak >= ee.patience;
    }
    st.iter = l;
    const bool fin = ex || l >= st.L_run;
    if (fin) {
      st.depth = l;
      phase_release(&st.phase, PH_BOUNDARY);  // a boundary stage may take the lane from here on
    }
    if (exit_mask_out) exit_mask_out[ln] = fin ? 1 : 0;
    if (lane_iters) atomicAdd(lane_iters, 1ull);
    fill_from = (fin && warm_token(wp, st.taken) && l < st.L_req) ? l : 0;
    fill_to = st.L_req;
  }
  __syncthreads();
  if (fill_from == 0) return;
  // copy K and V of this position from iteration fill_from into iterations fill_from+1 .. fill_to
  const int pos = rows.pos[r];
  const int hd = g.hd, per_head = 2 * hd;  // K then V elements of one head
  const int per_slot = g.H * per_head;
  const int total = (fill_to - fill_from) * n_loop_layers * per_slot;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int e = i % per_slot, q = i / per_slot;
    const int m = q % n_loop_layers, it = fill_from + 1 + q / n_loop_layers;
    const int hh = e / per_head, k = e % per_head;
    const int src_slot = n_pre + (fill_from - 1) * n_loop_layers + m;
    const int dst_slot = n_pre + (it - 1) * n_loop_layers + m;
    const __half* sp = kv_k_ptr(g, ln, src_slot, pos, hh, status);
    __half* dp = kv_k_ptr(g, ln, dst_slot, pos, hh, status);
    if (!sp || !dp) continue;
    const int64_t v_off = (int64_t)g.H * g.page_tokens * hd;  // V row of the same head and position
    if (k < hd) dp[k] = sp[k];
    else dp[v_off + k - hd] = sp[v_off + k - hd];
  }
}

// ---------------------------------------------------- logit-margin probe ----
//
// Rows of the loop table whose iteration just run (lane's iter + 1) is a probe
// of the exit rule, compacted in row order into `probe` (one CTA of 1024
// threads; thread i looks at loop row i).
__global__ void probe_rows_kernel(Rows loop, const LaneState* __restrict__ lanes, EEParams ee, Rows probe) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int32_t cnt[32];
  const int i = threadIdx.x, lane = i & 31, w = i >> 5;
  const int n = loop.n[0];
  int take = 0, ln = 0;
  if (i < n) {
    ln = loop.lane[i];
    take = ee_probe(ee, lanes[ln].iter + 1);
  }
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (lane == 0) cnt[w] = __popc(bal);
  __syncthreads();
  if (w == 0) {
    int v = cnt[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    cnt[lane] = v;
  }
  __syncthreads();
  if (take) {
    const int r = (w == 0 ? 0 : cnt[w - 1]) + __popc(bal & ((1u << lane) - 1u));
    probe.lane[r] = ln;
    probe.pos[r] = loop.pos[i];
    probe.iter[r] = loop.iter[i];
  }
  if (i == 0) probe.n[0] = cnt[31];
}

// margin_lane[lane] = top-1 minus top-2 of logits[lane][0..V) for every probe
// row (equal maxima give 0).  One CTA per row.
__global__ void margin_kernel(Rows probe, const float* __restrict__ logits, int V, float* __restrict__ margin_lane) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float s1[32], s2[32];
  const int r = blockIdx.x;
  if (r >= probe.n[0]) return;
  const int ln = probe.lane[r];
  const float* x = logits + (int64_t)ln * V;
  float a1 = -INFINITY, a2 = -INFINITY;  // the two largest values seen (a multiset)
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float y = x[v];
    if (y > a1) { a2 = a1; a1 = y; } else if (y > a2) { a2 = y; }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float b1 = __shfl_xor_sync(0xffffffffu, a1, off), b2 = __shfl_xor_sync(0xffffffffu, a2, off);
    const float n1 = fmaxf(a1, b1), n2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
    a1 = n1;
    a2 = n2;
  }
  if ((threadIdx.x & 31) == 0) { s1[threadIdx.x >> 5] = a1; s2[threadIdx.x >> 5] = a2; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
      const float n1 = fmaxf(a1, s1[w]), n2 = fmaxf(fminf(a1, s1[w]), fmaxf(a2, s2[w]));
      a1 = n1;
      a2 = n2;
    }
    margin_lane[ln] = a1 - a2;
  }
}

// ------------------------------------------------------------- boundary ----

enum HeadMode : int32_t { HEAD_ONLY = 0, HEAD_DECODE = 1 };

// Argmax over the head's partial results for each boundary row; HEAD_DECODE
// also records the token and the depth behind it, and either retires the lane
// or moves it to its next position: cap = depth (monotonic clamp), L_run =
// min(L_req, cap), embed the token, and (mark_entered) flag it for a later
// SEL_ENTERED table; a decode tick plans its entered rows beforehand and
// passes 0.  One CTA per row.
__global__ void head_finalize_kernel(Rows rows, LaneState* __restrict__ lanes, const float* __restrict__ part_val,
                                     const int32_t* __restrict__ part_idx, const int32_t* __restrict__ n_parts_dev,
                                     int32_t mode,
                                     int32_t* __restrict__ argmax_out, int32_t* __restrict__ tokens_out,
                                     int32_t* __restrict__ depths_out, int n_new, MatView E, float* __restrict__ h,
                                     int d, int max_seq, int32_t mark_entered, int32_t* __restrict__ status,
                                     unsigned long long* __restrict__ tok_count, WarmParams wp, int32_t hold) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int tok_s;
  __shared__ int go_s;
  const int r = blockIdx.x;
  if (r >= rows.n[0]) return;
  const int ln = rows.lane[r];
  const int n_parts = n_parts_dev[0];
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int p = threadIdx.x; p < n_parts; p += blockDim.x) {
    const float v = part_val[(int64_t)r * n_parts + p];
    const int i = part_idx[(int64_t)r * n_parts + p];
    if (better(v, i, bv, bi)) { bv = v; bi = i; }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
  }
  if ((threadIdx.x & 31) == 0) { sv[threadIdx.x >> 5] = bv; si[threadIdx.x >> 5] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (better(sv[w], si[w], bv, bi)) { bv = sv[w]; bi = si[w]; }
    if (bi < 0 || bi >= E.N) { set_status(status, ST_BAD_TOKEN); bi = 0; }
    tok_s = bi;
    go_s = 0;
    if (argmax_out) argmax_out[ln] = bi;
    if (mode == HEAD_DECODE) {
      LaneState& st = lanes[ln];
      if (tokens_out) tokens_out[(int64_t)ln * n_new + st.n_emitted] = bi;
      if (depths_out) depths_out[(int64_t)ln * n_new + st.n_emitted] = st.depth;
      st.n_emitted += 1;
      if (tok_count) atomicAdd(tok_count, 1ull);
      if (st.n_emitted >= st.n_target) {
        st.phase = PH_DONE;
      } else if (st.pos + 1 >= max_seq) {
        set_status(status, ST_BAD_POS);
        st.phase = PH_DONE;
      } else {
        if (!warm_token(wp, st.taken)) st.L_cap = st.depth;  // a warmup token's depth does not lower the cap
        st.taken += 1;
        st.L_run = warm_token(wp, st.taken) ? min(wp.L, st.L_req) : min(st.L_req, st.L_cap);
        st.pos += 1;
        st.iter = 0;
        st.streak = 0;
        st.token = bi;
        st.phase = hold ? PH_CLAIMED : PH_LOOP;  // held: release_rows_kernel hands it to the loop
        st.entered = mark_entered;
        go_s = 1;
      }
    }
  }
  __syncthreads();
  if (go_s) embed_row(E, tok_s, h + (int64_t)ln * d, d);
}

// Teacher-forced token entry for masked lanes (see tl_embed_next).  One CTA per lane.
__global__ void embed_next_kernel(LaneState* __restrict__ lanes, int n_lanes, const uint8_t* __restrict__ mask,
                                  const int32_t* __restrict__ tokens, MatView E, float* __restrict__ h, int d,
                                  int max_seq, int32_t* __restrict__ status, WarmParams wp) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int tok_s, go_s;
  const int ln = blockIdx.x;
  if (ln >= n_lanes) return;
  if (threadIdx.x == 0) {
    go_s = 0;
    LaneState& st = lanes[ln];
    if ((mask == nullptr || mask[ln]) && st.phase != PH_IDLE) {
      int tok = tokens[ln];
      if (tok < 0 || tok >= E.N) { set_status(status, ST_BAD_TOKEN); tok = 0; }
      if (st.pos + 1 >= max_seq) {
        set_status(status, ST_BAD_POS);
      } else {
        if (!warm_token(wp, st.taken)) st.L_cap = st.depth;
        st.taken += 1;
        st.L_run = warm_token(wp, st.taken) ? min(wp.L, st.L_req) : min(st.L_req, st.L_cap);
        st.pos += 1;
        st.iter = 0;
        st.streak = 0;
        st.token = tok;
        st.phase = PH_LOOP;
        st.entered = 1;
        tok_s = tok;
        go_s = 1;
      }
    }
  }
  __syncthreads();
  if (go_s) embed_row(E, tok_s, h + (int64_t)ln * d, d);
}

// End of a boundary stage that runs apart from the loop steps: the entered
// lanes (their token, embedding and pre blocks done by the kernels before this
// one) go to the loop.  One thread per row.
__global__ void release_rows_kernel(Rows rows, LaneState* lanes) {
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows.n[0]) return;
  phase_release(&lanes[rows.lane[r]].phase, PH_LOOP);
}

// Lanes of a decode call: set the request and token budget.  A request above
// the lane's cap sets ST_EKV and leaves the lane out.
__global__ void decode_init_kernel(LaneState* __restrict__ lanes, int n_lanes, const int32_t* __restrict__ req_L,
                                   int n_new, int32_t* __restrict__ status) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_lanes) return;
  LaneState& st = lanes[i];
  const int L = req_L[i];
  if (st.phase != PH_BOUNDARY || L < 1 || L > st.L_cap) {
    set_status(status, ST_EKV);
    st.phase = PH_DONE;
    return;
  }
  st.L_req = L;
  st.n_emitted = 0;
  st.n_target = n_new;
}

// Lane states after a batch of prompts: lane lanes[i] takes hidden row
// last_row[i] of hrows (its position last_pos[i]), cap = depth = L[i].
__global__ void prefill_finish_batch_kernel(LaneState* __restrict__ lanes, const int32_t* __restrict__ info, int n,
                                            const float* __restrict__ hrows, float* __restrict__ h, int d) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x;
  if (i >= n) return;
  const int ln = info[4 * i], last_row = info[4 * i + 1], last_pos = info[4 * i + 2], L = info[4 * i + 3];
  for (int k = threadIdx.x; k < d; k += blockDim.x) h[(int64_t)ln * d + k] = hrows[(int64_t)last_row * d + k];
  if (threadIdx.x == 0) {
    LaneState& st = lanes[ln];
    st.L_req = L;
    st.L_cap = L;
    st.L_run = L;
    st.iter = 0;
    st.pos = last_pos;
    st.streak = 0;
    st.phase = PH_BOUNDARY;
    st.depth = L;
    st.n_emitted = 0;
    st.n_target = 0;
    st.token = -1;
    st.entered = 0;
    st.taken = 0;
  }
}

}  // namespace tl
