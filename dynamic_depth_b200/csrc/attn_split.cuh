// Decode attention with the context split over CTAs: one CTA of 4 warps per
// (row, head, split).  Used for decode steps without a shared prefix (the
// balanced kernel of attn_decode.cuh serves shared-prefix steps, whose cascade
// partial it merges): at a few rows its small CTAs start and finish sooner
// around the neighbouring projections than the persistent kernel's.
#pragma once

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace tl {

// ------------------------------------------------------------- attention ----
//
// o[r][h] = softmax(q k^T / sqrt(hd)) v over positions 0..pos of the row's
// (lane, slot) cache, with RoPE and the KV append of the row's own position
// folded in: every CTA rotates its head's query from the projection output
// (qkv, [rows][3d]), and the CTA of the last split, whose key range holds
// position pos, first rotates and stores that position's key and value, then
// reads them back with the rest of its range (ordered by __syncthreads within
// the CTA; no other CTA reads that position).  One CTA of 4 warps per
// (row, head, split): the key
// blocks of 32 positions are divided into S contiguous ranges, S chosen on the
// device from the live row count so that few rows still spread over the SMs
// (S <= gridDim.z).  Inside a CTA warp w takes blocks w, w+4, ..., streamed
// through its own two-stage shared-memory ring: one key per lane for the
// scores, then every lane owns hd/32 output dimensions for the value sum;
// running max and sum are merged across warps, and across splits by the last
// CTA of the (row, head) to finish, in split order.  Requires kv_page_tokens
// >= 32 (a block lies in one page).
// Working CTAs the context split aims for: four per SM on 148 SMs (a
// larger target, 12 per SM, split the 64-row case in two and measured
// slower: the split partials and their combine cost more than the waves save).
constexpr int kAttnCtaTarget = 4 * 148;

// Keys of one ring stage: 32 (one per lane) at head dim 32, 16 (two lanes per
// key) at 64, 8 (four lanes per key) at 128: 2 KB of keys and 2 KB of values.
template <int HD>
constexpr int kAttnKeys = HD >= 128 ? 8 : (HD >= 64 ? 16 : 32);
// Bytes of one stage's keys (or values) of one head.
template <int HD>
constexpr int kAttnBlockBytes = kAttnKeys<HD> * HD * 2;
// Ring stages per warp: two, so a CTA takes 32 KB and six share an SM; the
// CTAs of a 64-row step then run in about one wave.  Measured at 64 lanes
// (hd 64): 34.0k tokens/s with 2 stages of 16 keys, 32.7k with 3, 31.5-32.0k
// with 4 (three CTAs per SM); 8-key stages 33.0-33.6k.
template <int HD>
constexpr int kAttnStages = 2;
// Dynamic shared memory of attn_split_kernel: per warp, its stages of keys and values.
template <int HD>
constexpr int kAttnSplitSmem = 4 * kAttnStages<HD> * 2 * kAttnBlockBytes<HD>;

extern __shared__ __align__(16) uint8_t attn_split_smem[];

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Stored position of 16-byte chunk c of key row r: the eight rows one
// shared-memory access phase reads (lane = row) land in eight different bank
// groups.
template <int HD>
__device__ __forceinline__ int attn_swz(int c, int r) {
  return HD == 32 ? (c ^ ((r >> 1) & 3)) : (c ^ (r & 7));
}

// The keys and values of sub-block sb (positions sb*KEYS ..) of one head into
// a ring stage: keys at row stride HD*2 bytes with swizzled chunks, then
// values unswizzled; rows at or past ctx are zero-filled (no global read).
// false when the page table has no page there (status set).
template <int HD>
__device__ __forceinline__ bool attn_issue_block(uint8_t* stage, const KVGeom& g, int ln, int slot, int sb, int ctx,
                                                 int h, int32_t* status) {
  constexpr int KEYS = kAttnKeys<HD>;
  const __half* kbase = kv_k_ptr(g, ln, slot, sb * KEYS, h, status);
  if (!kbase) return false;
  const __half* vbase = kbase + (int64_t)g.H * g.page_tokens * HD;
  const int lane = threadIdx.x & 31;
  const int nk = min(KEYS, ctx - sb * KEYS);
  constexpr int CPR = HD / 8;
#pragma unroll
  for (int q = lane; q < KEYS * CPR; q += 32) {
    const int row = q / CPR, c = q % CPR;
    const int bytes = row < nk ? 16 : 0;
    cp_async16(stage + row * HD * 2 + attn_swz<HD>(c, row) * 16, kbase + row * HD + c * 8, bytes);
    cp_async16(stage + kAttnBlockBytes<HD> + row * HD * 2 + c * 16, vbase + row * HD + c * 8, bytes);
  }
  return true;
}

template <int HD>
__global__ void __launch_bounds__(128)
attn_split_kernel(const float* __restrict__ qkv, float* __restrict__ o, __half* __restrict__ o16, Rows rows,
                   KVGeom g, const float2* __restrict__ rope_cs, int slot_base, int slot_stride,
                   float* __restrict__ part, int32_t* __restrict__ counters, int32_t* __restrict__ status,
                   int split16) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int DPL = HD / 32;  // output dims per lane
  __shared__ float qs[HD];
  __shared__ float wm[4], wl[4];
  __shared__ float wacc[4][HD];
  __shared__ int last_s;
  const int r = blockIdx.x, h = blockIdx.y, z = blockIdx.z;
  const int n = rows.n[0];
  if (r >= n) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = g.H * HD;
  const int pos = rows.pos[r];
  const int ln = rows.lane[r];
  const int slot = slot_base + rows.iter[r] * slot_stride;
  const int ctx = pos + 1;
  const int nblk = (ctx + 31) / 32;
  int S = (kAttnCtaTarget + n * g.H - 1) / (n * g.H);
  S = min(min(S, (int)gridDim.z), nblk);
  if (z >= S) return;
  const int b0 = (z * nblk) / S, b1 = ((z + 1) * nblk) / S;
  const float scale = rsqrtf((float)HD);
  {
    constexpr int HALF = HD / 2;
    const float* src = qkv + (int64_t)r * 3 * d + h * HD;
    const int i = threadIdx.x;
    if (i < HALF) {
      const float2 cs = rope_cs[(int64_t)pos * HALF + i];
      const float q0 = src[i], q1 = src[i + HALF];
      qs[i] = (q0 * cs.x - q1 * cs.y) * scale;
      qs[i + HALF] = (q1 * cs.x + q0 * cs.y) * scale;
      if (z == S - 1) {  // this split's range ends at pos: append the row's key and value
        __half* kp = kv_k_ptr(g, ln, slot, pos, h, status);
        if (kp) {
          __half* vp = kp + (int64_t)g.H * g.page_tokens * HD;
          const float k0 = src[d + i], k1 = src[d + i + HALF];
          kp[i] = __float2half_rn(k0 * cs.x - k1 * cs.y);
          kp[i + HALF] = __float2half_rn(k1 * cs.x + k0 * cs.y);
          vp[i] = __float2half_rn(src[2 * d + i]);
          vp[i + HALF] = __float2half_rn(src[2 * d + i + HALF]);
        }
      }
    }
  }
  __syncthreads();
  float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  // Each warp streams its sub-blocks through a ring of NS shared-memory
  // stages (cp.async, 16-byte chunks): NS - 1 sub-blocks' keys and values are
  // in flight while the current one is scored and summed.
  constexpr int KEYS = kAttnKeys<HD>;
  constexpr int LPK = 32 / KEYS;       // lanes per key (their partial dots are summed)
  constexpr int CPL = HD / 8 / LPK;    // 16-byte chunks of a key row per lane
  constexpr int NS = kAttnStages<HD>;
  constexpr int BB = kAttnBlockBytes<HD>;
  uint8_t* ring = attn_split_smem + (size_t)warp * NS * 2 * BB;
  const int key = lane % KEYS, half = lane / KEYS;
  // the split's 32-position blocks b0 .. b1 as sub-blocks of KEYS positions; this warp's are sb0, sb0 + 4, ...
  const int sb1 = min(b1 * (32 / KEYS), (ctx + KEYS - 1) / KEYS);
  const int sb0 = b0 * (32 / KEYS) + warp;
  int avail = sb0 < sb1 ? (sb1 - sb0 + 3) / 4 : 0;  // a sub-block without a page ends the range
#pragma unroll
  for (int i = 0; i < NS - 1; ++i) {
    if (i < avail && !attn_issue_block<HD>(ring + i * 2 * BB, g, ln, slot, sb0 + 4 * i, ctx, h, status)) avail = i;
    cp_async_commit();
  }
  for (int i = 0; i < avail; ++i) {
    const int ip = i + NS - 1;
    if (ip < avail && !attn_issue_block<HD>(ring + (ip % NS) * 2 * BB, g, ln, slot, sb0 + 4 * ip, ctx, h, status))
      avail = ip;
    cp_async_commit();
    cp_async_wait<NS - 1>();  // sub-block i's copies (each lane's own) have landed
    __syncwarp();             // ... and every lane's are visible to the warp
    const int sb = sb0 + 4 * i;
    const uint8_t* ks = ring + (i % NS) * 2 * BB;
    const uint8_t* vs = ks + BB;
    const int j = sb * KEYS + key;
    float s = -INFINITY;
    {
      float dot = 0.f;
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) {
        const int c = half * CPL + cc;
        const uint4 kv = *reinterpret_cast<const uint4*>(ks + key * HD * 2 + attn_swz<HD>(c, key) * 16);
        const __half2* hv = reinterpret_cast<const __half2*>(&kv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          dot = fmaf(qs[8 * c + 2 * e], f.x, dot);
          dot = fmaf(qs[8 * c + 2 * e + 1], f.y, dot);
        }
      }
      if constexpr (LPK >= 2) dot += __shfl_xor_sync(0xffffffffu, dot, 16);
      if constexpr (LPK >= 4) dot += __shfl_xor_sync(0xffffffffu, dot, 8);
      if (j < ctx) s = dot;
    }
    const float mb = warp_max(s);
    const float mn = fmaxf(m, mb);
    const float p = (j < ctx && half == 0) ? expf(s - mn) : 0.f;  // one lane per key carries its weight
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] *= corr;
    m = mn;
#pragma unroll 8
    for (int jj = 0; jj < KEYS; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const uint8_t* vr = vs + jj * HD * 2 + lane * DPL * 2;  // rows past the context were zero-filled
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vr);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
        acc[0] = fmaf(pj, f0.x, acc[0]);
        acc[1] = fmaf(pj, f0.y, acc[1]);
        acc[2] = fmaf(pj, f1.x, acc[2]);
        acc[3] = fmaf(pj, f1.y, acc[3]);
      } else if constexpr (DPL == 2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(vr));
        acc[0] = fmaf(pj, f.x, acc[0]);
        acc[1] = fmaf(pj, f.y, acc[1]);
      } else {
        acc[0] = fmaf(pj, __half2float(*reinterpret_cast<const __half*>(vr)), acc[0]);
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  if (lane == 0) { wm[warp] = m; wl[warp] = l; }
#pragma unroll
  for (int e = 0; e < DPL; ++e) wacc[warp][lane * DPL + e] = acc[e];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w]);
  float Lsum = 0.f;
  float f[4];
  for (int w = 0; w < 4; ++w) {
    f[w] = (wm[w] == -INFINITY) ? 0.f : expf(wm[w] - M);
    Lsum += wl[w] * f[w];
  }
  if (S == 1) {
    for (int i = threadIdx.x; i < HD; i += blockDim.x) {
      float v = 0.f;
      for (int w = 0; w < 4; ++w) v += wacc[w][i] * f[w];
      o[(int64_t)r * d + h * HD + i] = v / Lsum;
      act16_put(o16, r, d, h * HD + i, v / Lsum, split16);
    }
    return;
  }
  // split partial: (max, sum, unnormalised output) for this key range
  float* mine = part + (((int64_t)r * g.H + h) * gridDim.z + z) * (HD + 2);
  for (int i = threadIdx.x; i < HD; i += blockDim.x) {
    float v = 0.f;
    for (int w = 0; w < 4; ++w) v += wacc[w][i] * f[w];
    mine[2 + i] = v;
  }
  if (threadIdx.x == 0) { mine[0] = M; mine[1] = Lsum; }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_s = (atomicAdd(&counters[r * g.H + h], 1) == S - 1);
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  const float* base = part + ((int64_t)r * g.H + h) * gridDim.z * (HD + 2);
  float Mx = -INFINITY;
  for (int zz = 0; zz < S; ++zz) Mx = fmaxf(Mx, __ldcg(base + zz * (HD + 2)));
  float Lt = 0.f;
  for (int zz = 0; zz < S; ++zz) {
    const float mz = __ldcg(base + zz * (HD + 2));
    Lt += __ldcg(base + zz * (HD + 2) + 1) * ((mz == -INFINITY) ? 0.f : expf(mz - Mx));
  }
  for (int i = threadIdx.x; i < HD; i += blockDim.x) {
    float v = 0.f;
    for (int zz = 0; zz < S; ++zz) {
      const float mz = __ldcg(base + zz * (HD + 2));
      v += __ldcg(base + zz * (HD + 2) + 2 + i) * ((mz == -INFINITY) ? 0.f : expf(mz - Mx));
    }
    o[(int64_t)r * d + h * HD + i] = v / Lt;
    act16_put(o16, r, d, h * HD + i, v / Lt, split16);
  }
  if (threadIdx.x == 0) counters[r * g.H + h] = 0;
}


}  // namespace tl
