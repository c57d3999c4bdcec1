// Decode attention over the paged per-iteration KV cache, balanced over the
// whole GPU.
//
// o[r][h] = softmax(q k^T / sqrt(hd)) v over positions 0..pos of row r's
// (lane, slot) cache, with RoPE of q and k and the append of the row's own
// K/V folded in (one query row per (row, head); the slot is slot_base +
// iter * slot_stride).
//
// Work decomposition.  Every (row, head) is cut into key blocks ("units") of
// UK consecutive positions (UK divides the page size, so a unit lies in one
// page); the units of all rows and heads are flattened in (row, head, block)
// order and cut into equal contiguous ranges, one per warp of a persistent
// grid (one CTA of 4 or 8 warps per SM).  A warp streams its range through a private
// ring of shared-memory stages filled by TMA tile loads (K then V of one unit,
// 128-byte or 64-byte swizzled so the per-key reads below hit distinct banks),
// keeping STAGES units in flight, and runs an online softmax over the units of
// each (row, head) it meets.  A (row, head) that one warp covers entirely is
// written out directly; one that a warp boundary cuts produces a partial
// (max, sum, unnormalised output) per piece, and the last piece to finish (an
// atomic count per (row, head)) merges them in piece order, so the result
// does not depend on which warp finishes first.  No warp ever waits for
// another.  Units per warp are raised when needed so a (row, head) never has
// more than kAttnPieces pieces.
//
// Shared prefixes ("Benchmark Comparison" (measured benchmarks), section 2):
// when lane_shared is given, a row whose lane maps lane_shared[lane] positions
// of a shared prefix skips them (the cascade pass of attn_tc_kernel attended
// all such rows against the prefix at once and left a partial per (row,
// head) in casc); its output merges that partial with its own positions by
// log-sum-exp.
//
// The unit that holds position pos is processed by exactly one warp: it
// rotates that position's key, writes K and V to the cache for later steps and
// patches them into its shared-memory copy of the unit (the TMA may have read
// the row before or after the write), so no other CTA needs them in this
// launch.
//
// Inside a warp (UK = 32 keys per unit), lane j scores key j, reading its key
// row chunk by chunk through the swizzle, with the rotated, pre-scaled query in
// registers.  For the value sum the warp is split into G = 32 / (hd / 8) key
// groups of hd / 8 lanes: lane (group g, chunk c) owns the 8 output dimensions
// of 16-byte chunk c and sums keys g, g + G, ... of the unit (the lanes of one
// group read one whole value row, no bank conflict); the groups' sums are
// added once per (row, head) run, not per unit.  Every wait is bounded
// (~1.5 s); on expiry the warp records ST_TIMEOUT, lets its copies in flight
// land and leaves.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace tl {

constexpr int kAttnPieces = 8;   // pieces a (row, head) may be cut into
constexpr int kAttnUK = 32;      // keys per unit (divides every page size, which is >= 32)

template <int HD>
struct AttnCfg {
  static constexpr int UK = kAttnUK;
  static constexpr int COLS = HD > 64 ? 64 : HD;            // dimensions per TMA tile row
  static constexpr int HALVES = HD / COLS;                  // tiles per key row (hd 128: two)
  static constexpr int ROW_BYTES = COLS * 2;                // 128 B (swizzle 128B) or 64 B (64B)
  static constexpr int TILE_BYTES = UK * ROW_BYTES;
  static constexpr int UNIT_BYTES = 2 * HALVES * TILE_BYTES;  // K tiles then V tiles
  static constexpr int RING = 192 * 1024;                   // all warps' stages
  static constexpr int WARPS = RING / (3 * UNIT_BYTES) > 8 ? 8 : RING / (3 * UNIT_BYTES);
  static constexpr int STAGES = RING / (WARPS * UNIT_BYTES) > 6 ? 6 : RING / (WARPS * UNIT_BYTES);
  static constexpr int LPR = HD / 8;                        // lanes per value row (one 16-byte chunk each)
  static constexpr int G = 32 / LPR;                        // key groups of the value sum
  static constexpr int SMEM_FIXED = 1024 + WARPS * STAGES * 8 + 64;
  static_assert(STAGES >= 2 && WARPS >= 4, "attention ring too small");
  static_assert(TILE_BYTES % 1024 == 0 || (ROW_BYTES == 64 && TILE_BYTES % 512 == 0), "tile alignment");
};

// Byte offset of 16-byte chunk c of row j inside a swizzled tile.
template <int ROW_BYTES>
__device__ __forceinline__ int swz_chunk(int j, int c) {
  if constexpr (ROW_BYTES == 128) return j * 128 + ((c ^ (j & 7)) << 4);
  else return j * 64 + ((c ^ ((j >> 1) & 3)) << 4);
}

// Dynamic shared memory bytes of the kernel for a given row capacity.
template <int HD>
constexpr int attn_smem_bytes(int max_rows) {
  return AttnCfg<HD>::WARPS * AttnCfg<HD>::STAGES * AttnCfg<HD>::UNIT_BYTES + AttnCfg<HD>::SMEM_FIXED +
         4 * (max_rows + 1);
}

template <int HD>
__global__ void __launch_bounds__(AttnCfg<HD>::WARPS * 32, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap kvmap, const float* __restrict__ qkv, float* __restrict__ o,
                   __half* __restrict__ o16, Rows rows, KVGeom g, const float2* __restrict__ rope_cs, int slot_base,
                   int slot_stride, float* __restrict__ part, int32_t* __restrict__ counters,
                   int32_t* __restrict__ status, const int32_t* __restrict__ lane_shared,
                   const float* __restrict__ casc, int split16) {
  using C = AttnCfg<HD>;
  constexpr int UK = C::UK, STAGES = C::STAGES, WARPS = C::WARPS, HALF = HD / 2, LPR = C::LPR, G = C::G;
  constexpr int CPT = C::COLS / 8;  // 16-byte chunks per tile row
  extern __shared__ __align__(1024) uint8_t smem_attn[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_attn) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + WARPS * STAGES * C::UNIT_BYTES);  // [warp][stage]
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(full + WARPS * STAGES);
  int32_t* ubase = reinterpret_cast<int32_t*>(full + WARPS * STAGES) + 16;  // [n + 1] units before row r
  __shared__ int32_t red_i[WARPS];
  __shared__ int32_t red_m[WARPS];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = g.H, d = H * HD;
  // shared-prefix rows (lane_shared != null): their first lane_shared[lane] positions were attended by the
  // cascade pass, whose partial (max, sum, output) in casc is merged in here; this kernel takes the rest
  auto first_block = [&](int r) { return lane_shared ? lane_shared[rows.lane[r]] / UK : 0; };
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < WARPS * STAGES; ++i) mbar_init(smem_u32(&full[i]), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_wait();
  const int n = rows.n[0];
  // units per row (ceil((pos + 1) / UK)) and their exclusive scan, times H
  {
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    const int r0 = threadIdx.x * per, r1 = min(n, r0 + per);
    int s = 0, mx = 0;
    for (int r = r0; r < r1; ++r) {
      const int nu = (rows.pos[r] + UK) / UK - first_block(r);
      s += nu;
      mx = max(mx, nu);
    }
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    int wmx = mx;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wmx = max(wmx, __shfl_xor_sync(0xffffffffu, wmx, off));
    if (lane == 31) red_i[warp] = incl;
    if (lane == 0) red_m[warp] = wmx;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += red_i[w];
    int run = before + incl - s;
    for (int r = r0; r < r1; ++r) {
      ubase[r] = run * H;
      run += (rows.pos[r] + UK) / UK - first_block(r);
    }
    if (threadIdx.x == blockDim.x - 1) ubase[n] = (before + incl) * H;
    __syncthreads();
  }
  if (n <= 0) return;
  int max_nu = 0;
  for (int w = 0; w < WARPS; ++w) max_nu = max(max_nu, red_m[w]);
  const int U = ubase[n];
  const int W = gridDim.x * WARPS;
  int upw = (U + W - 1) / W;
  upw = max(upw, (max_nu + kAttnPieces - 2) / (kAttnPieces - 1));
  upw = max(upw, 1);
  const int gw = blockIdx.x * WARPS + warp;
  const int u_begin = gw * upw, u_end = min(U, u_begin + upw);
  if (u_begin >= U) return;

  // (row, head, block) of a flat unit index
  auto locate = [&](int u, int& r, int& h, int& b) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ubase[mid] <= u) lo = mid; else hi = mid - 1;
    }
    r = lo;
    const int nu = (ubase[r + 1] - ubase[r]) / H;
    const int rem = u - ubase[r];
    h = rem / nu;
    b = rem % nu;
  };

  uint8_t* wring = ring + warp * STAGES * C::UNIT_BYTES;
  uint64_t* wfull = full + warp * STAGES;
  const int64_t head_rows = (int64_t)g.page_tokens;          // rows of one head's block inside a page
  const int64_t page_rows = (int64_t)2 * H * g.page_tokens;  // K then V
  // TMA loads of unit (r, h, b) into stage s (lane 0 only)
  auto issue = [&](int r, int h, int b, int s) {
    const int ln = rows.lane[r];
    const int slot = slot_base + rows.iter[r] * slot_stride;
    const int p0 = (first_block(r) + b) * UK;
    const int pg = p0 >> g.page_shift;
    int page = -1;
    if (slot >= 0 && slot < g.n_slots && pg < g.pages_per_seq)
      page = g.page_table[((int64_t)ln * g.n_slots + slot) * g.pages_per_seq + pg];
    const uint32_t fb = smem_u32(&wfull[s]);
    if (page < 0 || page >= g.n_pages) {  // recorded; the stage completes with nothing loaded
      set_status(status, ST_BAD_PAGE);
      mbar_arrive(fb);
      return;
    }
    const int64_t y = (int64_t)page * page_rows + h * head_rows + (p0 & (g.page_tokens - 1));
    mbar_expect_tx(fb, C::UNIT_BYTES);
    uint8_t* st = wring + s * C::UNIT_BYTES;
#pragma unroll
    for (int t = 0; t < C::HALVES; ++t) {
      tma_load_2d(smem_u32(st + t * C::TILE_BYTES), &kvmap, t * C::COLS, (int)y, fb);
      tma_load_2d(smem_u32(st + (C::HALVES + t) * C::TILE_BYTES), &kvmap, t * C::COLS, (int)(y + H * head_rows), fb);
    }
  };
  // the issue cursor runs ahead of the consumer over the same flat order
  int ir = 0, ih = 0, ib = 0;
  locate(u_begin, ir, ih, ib);
  auto advance = [&](int& rr, int& hh, int& bb) {
    if (++bb == (ubase[rr + 1] - ubase[rr]) / H) {
      bb = 0;
      if (++hh == H) {
        hh = 0;
        ++rr;
      }
    }
  };

  const int n_units = u_end - u_begin;
  if (lane == 0)
    for (int i = 0; i < min(STAGES, n_units); ++i) {
      issue(ir, ih, ib, i);
      advance(ir, ih, ib);
    }
  __syncwarp();

  // scores in the log2 domain: q carries log2(e) / sqrt(hd), so exp2 of differences gives the softmax weights
  const float scale = rsqrtf((float)HD) * 1.4426950408889634f;
  // value-sum role of this lane: 16-byte chunk vc of the value row (tile vt, chunk vcc), key group kg
  const int vc = lane % LPR, kg = lane / LPR;
  const int vt = vc / CPT, vcc = vc % CPT;
  // this lane's swizzled byte offsets: its key row's chunks (scores) and its value chunk of each key it sums
  int koff[CPT], voff[UK / G];
#pragma unroll
  for (int c = 0; c < CPT; ++c) koff[c] = swz_chunk<C::ROW_BYTES>(lane, c);
#pragma unroll
  for (int t = 0; t < UK / G; ++t) voff[t] = swz_chunk<C::ROW_BYTES>(kg + G * t, vcc);
  float q[HD];
  float m = -INFINITY, l = 0.f, acc[8];
  int r = 0, h = 0, b = 0, nu = 1, run_first = 0, ctx = 0, pos = 0, ln = 0, fb = 0;
  locate(u_begin, r, h, b);
  bool aborted = false;
  int consumed = 0;
  for (int i = 0; i < n_units; ++i) {
    const int u = u_begin + i;
    const int s = i % STAGES;
    if (i == 0 || b == 0) {  // a new (row, head): rotated, pre-scaled query; fresh softmax state
      nu = (ubase[r + 1] - ubase[r]) / H;
      pos = rows.pos[r];
      ln = rows.lane[r];
      ctx = pos + 1;
      fb = first_block(r);
      run_first = b;
      const float* src = qkv + (int64_t)r * 3 * d + h * HD;
      // lane l rotates pairs (l + 32 k, l + 32 k + HD/2); then every lane gathers the whole vector
      constexpr int NK = (HALF + 31) / 32;
      float qa[NK], qb[NK];
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        const int i0 = lane + 32 * k;
        qa[k] = qb[k] = 0.f;
        if (i0 < HALF) {
          const float2 cs = rope_cs[(int64_t)pos * HALF + i0];
          const float x0 = src[i0], x1 = src[i0 + HALF];
          qa[k] = (x0 * cs.x - x1 * cs.y) * scale;
          qb[k] = (x1 * cs.x + x0 * cs.y) * scale;
        }
      }
#pragma unroll
      for (int e = 0; e < HALF; ++e) {
        q[e] = __shfl_sync(0xffffffffu, qa[e / 32], e % 32);
        q[e + HALF] = __shfl_sync(0xffffffffu, qb[e / 32], e % 32);
      }
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    }
    if (!mbar_wait_warp(smem_u32(&wfull[s]), (i / STAGES) & 1, abort_flag)) { aborted = true; break; }
    consumed = i + 1;
    uint8_t* st = wring + s * C::UNIT_BYTES;
    const int nvalid = min(UK, ctx - (fb + b) * UK);
    if (b == nu - 1) {
      // this unit holds position pos: rotate its key, append K/V to the cache, patch the staged copy
      const int j = pos - (fb + b) * UK;
      const float* src = qkv + (int64_t)r * 3 * d + h * HD;
      __half* kp = kv_k_ptr(g, ln, slot_base + rows.iter[r] * slot_stride, pos, h, status);
      __half* vp = kp ? kp + (int64_t)H * g.page_tokens * HD : nullptr;
#pragma unroll
      for (int k = 0; k < (HALF + 31) / 32; ++k) {
        const int i0 = lane + 32 * k;
        if (i0 < HALF) {
          const float2 cs = rope_cs[(int64_t)pos * HALF + i0];
          const float k0 = src[d + i0], k1 = src[d + i0 + HALF];
          const __half ka = __float2half_rn(k0 * cs.x - k1 * cs.y), kb = __float2half_rn(k1 * cs.x + k0 * cs.y);
          const __half va = __float2half_rn(src[2 * d + i0]), vb = __float2half_rn(src[2 * d + i0 + HALF]);
          if (kp) {
            kp[i0] = ka;
            kp[i0 + HALF] = kb;
            vp[i0] = va;
            vp[i0 + HALF] = vb;
          }
          // element e of the row lives in tile e / COLS, chunk (e % COLS) / 8, slot e % 8
          const int es[2] = {i0, i0 + HALF};
          const __half kh[2] = {ka, kb}, vh[2] = {va, vb};
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int e = es[z], t = e / C::COLS, ee = e % C::COLS;
            const int off = swz_chunk<C::ROW_BYTES>(j, ee >> 3) + (ee & 7) * 2;
            *reinterpret_cast<__half*>(st + t * C::TILE_BYTES + off) = kh[z];
            *reinterpret_cast<__half*>(st + (C::HALVES + t) * C::TILE_BYTES + off) = vh[z];
          }
        }
      }
      __syncwarp();
    }
    // score of key `lane`
    float dot = 0.f;
#pragma unroll
    for (int t = 0; t < C::HALVES; ++t) {
      const uint8_t* tile = st + t * C::TILE_BYTES;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const uint4 kv = *reinterpret_cast<const uint4*>(tile + koff[c]);
        const __half2* hv = reinterpret_cast<const __half2*>(&kv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          dot = fmaf(q[t * C::COLS + 8 * c + 2 * e], f.x, dot);
          dot = fmaf(q[t * C::COLS + 8 * c + 2 * e + 1], f.y, dot);
        }
      }
    }
    const bool valid = lane < nvalid;
    const float sc = valid ? dot : -INFINITY;
    const float mn = fmaxf(m, warp_max(sc));
    const float p = valid ? exp2f(sc - mn) : 0.f;
    const float corr = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    l = l * corr + warp_sum(p);
    m = mn;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= corr;
    // value sum: keys kg, kg + G, ... of the unit, this lane's 8 dimensions
    {
      // keys past nvalid have p = 0, but their stale bytes may not be finite: skip them
      const uint8_t* vtile = st + (C::HALVES + vt) * C::TILE_BYTES;
      const bool full_unit = nvalid == UK;
#pragma unroll
      for (int t = 0; t < UK / G; ++t) {
        const int j = kg + G * t;
        const float pj = __shfl_sync(0xffffffffu, p, j);
        if (full_unit || j < nvalid) {
          const uint4 vv = *reinterpret_cast<const uint4*>(vtile + voff[t]);
          const __half2* hv = reinterpret_cast<const __half2*>(&vv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(hv[e]);
            acc[2 * e] = fmaf(pj, f.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(pj, f.y, acc[2 * e + 1]);
          }
        }
      }
    }
    // the stage is free: order this warp's reads before the next TMA write into it, then refill
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (lane == 0 && i + STAGES < n_units) {
      issue(ir, ih, ib, s);
      advance(ir, ih, ib);
    }
    __syncwarp();
    // end of this warp's run over (r, h): write the output or a piece
    if (b == nu - 1 || i == n_units - 1) {
      float tot[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float v = acc[e];
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        tot[e] = v;
      }
      const int dim0 = vc * 8;  // this lane's dimensions (lanes of key group 0 write)
      if (run_first == 0 && b == nu - 1) {
        if (kg == 0) {
          float Lt = l, fo = 1.f;
          if (fb > 0) {  // merge the shared-prefix partial
            const float* cp = casc + ((int64_t)r * H + h) * (HD + 2);
            const float mc = cp[0], M = fmaxf(m, mc);
            fo = exp2f(m - M);
            const float fc = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
            Lt = l * fo + cp[1] * fc;
#pragma unroll
            for (int e = 0; e < 8; ++e) tot[e] = tot[e] * fo + cp[2 + dim0 + e] * fc;
          }
          const float inv = 1.f / Lt;
          float4* op = reinterpret_cast<float4*>(o + (int64_t)r * d + h * HD + dim0);
          op[0] = make_float4(tot[0] * inv, tot[1] * inv, tot[2] * inv, tot[3] * inv);
          op[1] = make_float4(tot[4] * inv, tot[5] * inv, tot[6] * inv, tot[7] * inv);
          float ov[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) ov[e] = tot[e] * inv;
          act16_put8(o16, r, d, h * HD + dim0, ov, split16);
        }
      } else {
        const int first_unit = ubase[r] + h * nu;  // flat index of block 0 of (r, h)
        const int w_first = first_unit / upw, w_last = (first_unit + nu - 1) / upw;
        const int piece = gw - w_first, n_pieces = w_last - w_first + 1;
        float* mine = part + ((int64_t)(r * H + h) * kAttnPieces + piece) * (HD + 2);
        if (kg == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mine[2 + dim0 + e] = tot[e];
        }
        if (lane == 0) {
          mine[0] = m;
          mine[1] = l;
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(&counters[r * H + h], 1) == n_pieces - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          const float* base = part + (int64_t)(r * H + h) * kAttnPieces * (HD + 2);
          // the pieces in order, then the shared-prefix partial when the row has one
          const float* cp = fb > 0 ? casc + ((int64_t)r * H + h) * (HD + 2) : nullptr;
          const int n_all = n_pieces + (cp ? 1 : 0);
          auto piece_ptr = [&](int z) { return z < n_pieces ? base + z * (HD + 2) : cp; };
          float M = -INFINITY;
          for (int z = 0; z < n_all; ++z) M = fmaxf(M, __ldcg(piece_ptr(z)));
          float Lt = 0.f, outv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) outv[e] = 0.f;
          for (int z = 0; z < n_all; ++z) {
            const float* pz = piece_ptr(z);
            const float mz = __ldcg(pz);
            const float f = (mz == -INFINITY) ? 0.f : exp2f(mz - M);
            Lt += __ldcg(pz + 1) * f;
            if (kg == 0) {
#pragma unroll
              for (int e = 0; e < 8; ++e) outv[e] += __ldcg(pz + 2 + dim0 + e) * f;
            }
          }
          if (kg == 0) {
            const float inv = 1.f / Lt;
            float4* op = reinterpret_cast<float4*>(o + (int64_t)r * d + h * HD + dim0);
            op[0] = make_float4(outv[0] * inv, outv[1] * inv, outv[2] * inv, outv[3] * inv);
            op[1] = make_float4(outv[4] * inv, outv[5] * inv, outv[6] * inv, outv[7] * inv);
            float ov[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[e] = outv[e] * inv;
            act16_put8(o16, r, d, h * HD + dim0, ov, split16);
          }
          if (lane == 0) counters[r * H + h] = 0;
        }
      }
    }
    // advance to the next unit of the flat order
    if (++b == nu) {
      b = 0;
      if (++h == H) {
        h = 0;
        ++r;
      }
    }
  }
  if (aborted && lane == 0) {
    set_status(status, ST_TIMEOUT);
    // copies already issued land before the CTA's shared memory is released
    volatile int32_t never = 0;
    const int issued = min(n_units, consumed + STAGES);
    for (int i = consumed; i < issued; ++i) mbar_wait(smem_u32(&wfull[i % STAGES]), (i / STAGES) & 1, &never);
  }
}

}  // namespace tl
