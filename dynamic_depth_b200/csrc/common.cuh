// Shared device helpers and the device-side state layout of libtl.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/tl.h"

namespace tl {

// Status-word bits written by kernels (never __trap/assert: a bad index is
// recorded and the access skipped).
enum : int32_t {
  ST_BAD_PAGE = 1 << 0,     // page id outside the pool
  ST_BAD_POS = 1 << 1,      // position >= max_seq
  ST_BAD_SLOT = 1 << 2,     // KV slot outside the table
  ST_BAD_TOKEN = 1 << 3,    // token id outside [0, vocab)
  ST_EKV = 1 << 4,          // lane asked for more iterations than its cache holds
  ST_BAD_ROW = 1 << 5,      // row table larger than its buffers
};

// PH_CLAIMED: taken by a boundary stage that runs apart from the loop steps
// (asynchronous decode stages); the stage hands the lane back as PH_LOOP when
// its pre blocks are done, or retires it as PH_DONE.
enum LanePhase : int32_t { PH_IDLE = 0, PH_LOOP = 1, PH_BOUNDARY = 2, PH_DONE = 3, PH_CLAIMED = 4 };

// A lane's phase is the hand-off word between concurrently running stages:
// the writer orders every other write of the lane before it (release), the
// reader reads it before the lane's other fields (acquire).
// fp16 copy of an activation for the tensor cores, row `row` of a [rows][cols]
// activation.  With split16 a row holds [hi | lo] (2 * cols halves): hi =
// fp16(v), lo = fp16(v - hi); a projection that multiplies both halves by the
// same weights and sums (a K of 2 * cols) sees the fp32 activation to within
// ~2^-22 relative instead of fp16's 2^-11.
__device__ __forceinline__ void act16_put(__half* base, int64_t row, int cols, int col, float v, int split16) {
  __half* p = base + row * ((int64_t)cols << split16) + col;
  const __half hi = __float2half_rn(v);
  *p = hi;
  if (split16) p[cols] = __float2half_rn(v - __half2float(hi));
}

// Eight consecutive columns col0 .. col0 + 7 (col0 a multiple of 8) as act16_put does, in 16-byte stores.
__device__ __forceinline__ void act16_put8(__half* base, int64_t row, int cols, int col0, const float (&v)[8],
                                           int split16) {
  __half* p = base + row * ((int64_t)cols << split16) + col0;
  __half2 hi[4], lo[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    hi[e] = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
    const float2 f = __half22float2(hi[e]);
    lo[e] = __floats2half2_rn(v[2 * e] - f.x, v[2 * e + 1] - f.y);
  }
  *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(hi);
  if (split16) *reinterpret_cast<uint4*>(p + cols) = *reinterpret_cast<const uint4*>(lo);
}

__device__ __forceinline__ int32_t phase_acquire(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void phase_release(int32_t* p, int32_t v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One lane's scheduling state, resident in device memory.
struct LaneState {
  int32_t L_req;      // requested loop count
  int32_t L_cap;      // monotonic clamp: iterations the cache holds for new positions
  int32_t L_run;      // iterations planned for the current token: min(L_req, L_cap)
  int32_t iter;       // iterations done for the current token
  int32_t pos;        // position of the row the lane is computing
  int32_t streak;     // early-exit streak
  int32_t phase;      // LanePhase
  int32_t depth;      // iterations behind the lane's current hidden state
  int32_t n_emitted;  // tokens emitted by the running decode
  int32_t n_target;   // tokens to emit
  int32_t token;      // last token fed (or emitted)
  int32_t entered;    // set when the lane just took a token and still needs its pre blocks
  int32_t taken;      // tokens taken after the prompt: the token being computed is number `taken` (0 = prompt)
};

// L warmup ("Dynamic-L Inference", L scheduling; "CLI Reference",
// --l-warmup-tokens / --l-warmup-L): decode tokens 1..tokens run min(L, L_req)
// iterations and leave the cap alone; tokens == 0 disables it.
struct WarmParams {
  int32_t tokens;
  int32_t L;
};

__device__ __forceinline__ bool warm_token(const WarmParams& w, int t) { return t >= 1 && t <= w.tokens; }

// Early-exit parameters, copied by value into kernels.
struct EEParams {
  double tau;
  int32_t min_L;
  int32_t patience;
  int32_t peek_every;
  int32_t enabled;
  int32_t use_margin;  // 1: the probe's metric is the head's top-1 minus top-2 logit margin
  double margin;       // margin mode: a probe succeeds when the margin is at least this
};

// Whether iteration l (1-based) of a token is a probe of the exit rule.
__device__ __forceinline__ bool ee_probe(const EEParams& ee, int l) {
  return ee.enabled && l > ee.min_L && ((l - ee.min_L - 1) % ee.peek_every) == 0;
}

// Compacted rows of one launch group: row r computes for lane row_lane[r] at
// position row_pos[r], loop iteration row_iter[r] (0-based).
struct Rows {
  int32_t* n;        // device scalar: number of valid rows
  int32_t* lane;
  int32_t* pos;
  int32_t* iter;
};

// KV cache geometry.  A page holds kv_page_tokens positions of one (lane,
// slot): K as [H][P][hd] fp16 then V as [H][P][hd] fp16.
struct KVGeom {
  __half* pool;
  const int32_t* page_table;   // [max_lanes][n_slots][pages_per_seq]
  int32_t n_slots;
  int32_t pages_per_seq;
  int32_t page_tokens;
  int32_t page_shift;          // log2(page_tokens)
  int32_t n_pages;
  int32_t H, hd;
  int64_t page_elems;          // 2 * H * P * hd
};

__device__ __forceinline__ void set_status(int32_t* st, int32_t bit) { atomicOr(st, bit); }

// Programmatic dependent launch: a kernel lets the next kernel of the stream
// start its independent prologue at once (launch_dependents), and waits for
// the previous kernel's completion and memory (wait) before it touches
// anything that kernel or an earlier one wrote.  Both are no-ops when the
// launch did not ask for programmatic serialization.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024).  `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.f;
  if (w == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}
__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.0;
  if (w == 0) t = warp_sum_d(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// (u - 8) as an exact float for a nibble u in [0,15]: 2^23 + u read as float, minus 2^23 + 8.
__device__ __forceinline__ float nib_to_f(uint32_t w, int sh) {
  return __uint_as_float(((w >> sh) & 0xFu) | 0x4B000000u) - 8388616.0f;
}

__device__ __forceinline__ float bf16_bits_to_f(uint32_t b) { return __uint_as_float(b << 16); }

// Nibble holding element e (0..7) of an 8-element word in the device INT4
// layout: element 2i in nibble i, element 2i+1 in nibble i + 4 (the loader
// repacks the blob's plain order into this one).
__device__ __forceinline__ constexpr int nib_pos(int e) { return (e & 1) ? (e >> 1) + 4 : (e >> 1); }

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

// Address of (slot, lane, pos) K row for head h; V follows at + H*P*hd.
__device__ __forceinline__ __half* kv_k_ptr(const KVGeom& g, int lane, int slot, int pos, int h,
                                            int32_t* status) {
  if (slot < 0 || slot >= g.n_slots) { set_status(status, ST_BAD_SLOT); return nullptr; }
  const int pg = pos >> g.page_shift;
  if (pos < 0 || pg >= g.pages_per_seq) { set_status(status, ST_BAD_POS); return nullptr; }
  const int page = g.page_table[((int64_t)lane * g.n_slots + slot) * g.pages_per_seq + pg];
  if (page < 0 || page >= g.n_pages) { set_status(status, ST_BAD_PAGE); return nullptr; }
  const int off = pos & (g.page_tokens - 1);
  return g.pool + (int64_t)page * g.page_elems + ((int64_t)h * g.page_tokens + off) * g.hd;
}

}  // namespace tl
