// Decode attention with the context split over CTAs: one CTA of 4 warps per
// (row, head, split).  Used for decode steps without a shared prefix (the
// balanced kernel of attn_decode.cuh serves shared-prefix steps, whose cascade
// partial it merges): at a few rows its small CTAs start and finish sooner
// around the neighbouring projections than the persistent kernel's.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

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
// (S <= gridDim.z).  Inside a CTA warp w takes blocks w, w+4, ...: one key per
// lane for the scores, then every lane owns hd/32 output dimensions for the
// value sum (all 32 value loads of a block issued together); running max and
// sum are merged across warps, and across splits by the last CTA of the
// (row, head) to finish, in split order.  Requires kv_page_tokens >= 32.
// Working CTAs the context split aims for: four per SM on 148 SMs (a
// larger target, 12 per SM, split the 64-row case in two and measured
// slower: the split partials and their combine cost more than the waves save).
constexpr int kAttnCtaTarget = 4 * 148;

template <int HD>
__global__ void __launch_bounds__(128)
attn_split_kernel(const float* __restrict__ qkv, float* __restrict__ o, __half* __restrict__ o16, Rows rows,
                   KVGeom g, const float2* __restrict__ rope_cs, int slot_base, int slot_stride,
                   float* __restrict__ part, int32_t* __restrict__ counters, int32_t* __restrict__ status) {
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
  for (int kb = b0 + warp; kb < b1; kb += 4) {
    const __half* kbase = kv_k_ptr(g, ln, slot, kb * 32, h, status);
    if (!kbase) break;
    const __half* vbase = kbase + (int64_t)g.H * g.page_tokens * HD;
    const int j = kb * 32 + lane;
    const int nk = min(32, ctx - kb * 32);
    // the block's values, loaded together with its keys (neither depends on the scores)
    constexpr int VW = DPL >= 2 ? DPL / 2 : 1;  // 32-bit words of values per lane per key
    uint32_t vraw[32][VW];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      if (jj < nk) {
        if constexpr (DPL >= 2) {
#pragma unroll
          for (int e = 0; e < VW; ++e)
            vraw[jj][e] = reinterpret_cast<const uint32_t*>(vbase + (int64_t)jj * HD + lane * DPL)[e];
        } else {
          vraw[jj][0] = __half_as_ushort(vbase[(int64_t)jj * HD + lane]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < VW; ++e) vraw[jj][e] = 0u;
      }
    }
    float s = -INFINITY;
    if (j < ctx) {
      const uint4* kr = reinterpret_cast<const uint4*>(kbase + (int64_t)lane * HD);
      uint4 kv[HD / 8];
#pragma unroll
      for (int c = 0; c < HD / 8; ++c) kv[c] = kr[c];
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < HD / 8; ++c) {
        const __half2* hv = reinterpret_cast<const __half2*>(&kv[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          dot = fmaf(qs[8 * c + 2 * e], f.x, dot);
          dot = fmaf(qs[8 * c + 2 * e + 1], f.y, dot);
        }
      }
      s = dot;
    }
    const float mb = warp_max(s);
    const float mn = fmaxf(m, mb);
    const float p = (j < ctx) ? expf(s - mn) : 0.f;
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] *= corr;
    m = mn;
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      if constexpr (DPL >= 2) {
#pragma unroll
        for (int e = 0; e < VW; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&vraw[jj][e]));
          acc[2 * e] = fmaf(pj, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(pj, f.y, acc[2 * e + 1]);
        }
      } else {
        acc[0] = fmaf(pj, __half2float(__ushort_as_half((unsigned short)vraw[jj][0])), acc[0]);
      }
    }
  }
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
      o16[(int64_t)r * d + h * HD + i] = __float2half_rn(v / Lsum);
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
    o16[(int64_t)r * d + h * HD + i] = __float2half_rn(v / Lt);
  }
  if (threadIdx.x == 0) counters[r * g.H + h] = 0;
}


}  // namespace tl
