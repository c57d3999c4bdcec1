// Weight-streaming GEMV for few activation rows (decode): y[r] = W x[r] for
// r < rows <= 8 per pass, W INT4 (exact (u - 8) * scale) or BF16, fp32
// activations and accumulation.
//
// One persistent CTA per SM.  Weight rows of a matrix are contiguous, so a
// block of fb consecutive output features is one contiguous byte range (plus
// its fp16 scales): a producer warp streams blocks into a ring of shared-memory
// stages with cp.async.bulk (untiled TMA, no multicast), several stages ahead,
// while 8 consumer warps turn each stage into outputs.  The activation rows
// are staged once per CTA (fp32, 16-byte slots XOR-swizzled as in the
// CUDA-core GEMV), optionally normalised on the way in (GsNorm).  A consumer
// warp owns whole output features: every lane
// takes 32-element chunks of the row from shared memory, and one warp
// reduction per (feature, row) finishes it.  Memory parallelism comes from the
// bulk copies in flight (tens of KB per SM), not from registers.
#pragma once

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace tl {

constexpr int GS_CONSUMERS = 8;
constexpr int GS_THREADS = (GS_CONSUMERS + 1) * 32;

// Host-computed geometry of one launch.
struct GsPlan {
  int32_t fb;            // output features per block
  int32_t stages;
  int32_t stage_bytes;   // per matrix (weights then scales), multiple of 128
  int32_t row_bytes;     // packed bytes of one weight row
  int32_t sc_row_bytes;  // fp16 scale bytes of one row (INT4), else 0
  int32_t xs_offset;     // activation tile offset in dynamic shared memory
  int32_t bar_offset;
};

template <int FMT, int R, int EPI>
__device__ __forceinline__ void gs_feature(const uint8_t* __restrict__ wrow, const uint8_t* __restrict__ srow,
                                           const uint8_t* __restrict__ wrow2, const uint8_t* __restrict__ srow2,
                                           const float* __restrict__ xs, int K, int group, float (&acc)[R],
                                           float (&acc2)[R]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = acc2[r] = 0.f;
  for (int c = lane; c < K / 32; c += 32) {
    Chunk<FMT> ch;
    if constexpr (FMT == TL_FMT_INT4) {
      ch.v[0] = *reinterpret_cast<const uint4*>(wrow + c * 16);
      ch.sc = __half2float(*reinterpret_cast<const __half*>(srow + ((c * 32) / group) * 2));
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) ch.v[j] = *reinterpret_cast<const uint4*>(wrow + c * 64 + j * 16);
      ch.sc = 1.f;
    }
    float w[32];
    unpack_chunk<FMT>(ch, w);
    dot_chunk<R>(xs, K, c, w, ch.sc, acc);
    if constexpr (EPI == EPI_SWIGLU) {
      if constexpr (FMT == TL_FMT_INT4) {
        ch.v[0] = *reinterpret_cast<const uint4*>(wrow2 + c * 16);
        ch.sc = __half2float(*reinterpret_cast<const __half*>(srow2 + ((c * 32) / group) * 2));
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) ch.v[j] = *reinterpret_cast<const uint4*>(wrow2 + c * 64 + j * 16);
      }
      unpack_chunk<FMT>(ch, w);
      dot_chunk<R>(xs, K, c, w, ch.sc, acc2);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    acc[r] = warp_sum(acc[r]);
    if constexpr (EPI == EPI_SWIGLU) acc2[r] = warp_sum(acc2[r]);
  }
}

// Consumer warp: all features of stage `s` (block b) assigned to this warp.
template <int FMT, int R, int EPI>
__device__ __forceinline__ void gs_consume(const uint8_t* __restrict__ stage, int stage_bytes, int b, int nrow,
                                           const GsPlan& pl, const MatView& W, const float* __restrict__ xs, int r0,
                                           int rows, const ProjOut& o, float (&bv)[8], int (&bi)[8]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = W.K;
  for (int f = warp; f < nrow; f += GS_CONSUMERS) {
    const int n = b * pl.fb + f;
    const uint8_t* wrow = stage + (size_t)f * pl.row_bytes;
    const uint8_t* srow = stage + (size_t)pl.fb * pl.row_bytes + (size_t)f * pl.sc_row_bytes;
    const uint8_t* stage2 = stage + stage_bytes;
    const uint8_t* wrow2 = stage2 + (size_t)f * pl.row_bytes;
    const uint8_t* srow2 = stage2 + (size_t)pl.fb * pl.row_bytes + (size_t)f * pl.sc_row_bytes;
    float acc[R], acc2[R];
    gs_feature<FMT, R, EPI>(wrow, srow, wrow2, srow2, xs, K, W.group, acc, acc2);
    if constexpr (EPI == EPI_ARGMAX) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (better(acc[r], n, bv[r], bi[r])) { bv[r] = acc[r]; bi[r] = n; }
      if (o.logits && lane < R && r0 + lane < rows) {
        float v = acc[0];
#pragma unroll
        for (int r = 1; r < R; ++r) if (lane == r) v = acc[r];
        o.logits[(int64_t)o.lmap[r0 + lane] * o.ldo + n] = v;
      }
    } else if (lane < R && r0 + lane < rows) {
      float v = acc[0], v2 = acc2[0];
#pragma unroll
      for (int r = 1; r < R; ++r)
        if (lane == r) { v = acc[r]; v2 = acc2[r]; }
      const int row = r0 + lane;
      if constexpr (EPI == EPI_STORE) {
        o.out[(int64_t)row * o.ldo + n] = v;
      } else if constexpr (EPI == EPI_SWIGLU) {
        o.out[(int64_t)row * o.ldo + n] = silu_f(v) * v2;
      } else {
        const int hr = o.map ? o.map[row] : row;
        o.h[(int64_t)hr * W.N + n] += v;
      }
    }
  }
}

// Producer: request weight block b (and its scales) into stage s.
template <int FMT, int NMAT>
__device__ __forceinline__ void gs_issue(const MatView& W, const MatView& W2, const GsPlan& pl, uint8_t* ring,
                                         uint64_t* full, int s, int rd, int b) {
  (void)rd;
  const int N = W.N;
  const int nrow = min(pl.fb, N - b * pl.fb);
  const uint32_t wbytes = (uint32_t)nrow * pl.row_bytes, sbytes = (uint32_t)nrow * pl.sc_row_bytes;
  const uint32_t fb = smem_u32(&full[s]);
  mbar_expect_tx(fb, NMAT * (wbytes + sbytes));
#pragma unroll
  for (int mat = 0; mat < NMAT; ++mat) {
    const MatView& M = mat == 0 ? W : W2;
    uint8_t* dst = ring + (size_t)(s * NMAT + mat) * pl.stage_bytes;
    const uint8_t* src = (FMT == TL_FMT_INT4) ? M.q : reinterpret_cast<const uint8_t*>(M.bf);
    bulk_load(smem_u32(dst), src + (size_t)b * pl.fb * pl.row_bytes, wbytes, fb);
    if (FMT == TL_FMT_INT4)
      bulk_load(smem_u32(dst + (size_t)pl.fb * pl.row_bytes),
                reinterpret_cast<const uint8_t*>(M.s) + (size_t)b * pl.fb * pl.sc_row_bytes, sbytes, fb);
  }
}

// RMSNorm folded into the activation staging (g != null): X holds the
// residual rows h, row r of this projection is h row map[r] (row r when map is
// null), and each CTA stages x * rsqrt(mean(x^2) + eps) * g itself; CTA 0 also
// copies the raw rows to h_in (indexed like h) when h_in is given.
struct GsNorm {
  const float* g;
  const int32_t* map;
  float eps;
  float* h_in;
};

template <int FMT, int EPI>
__global__ void __launch_bounds__(GS_THREADS, 1)
gemv_stream_kernel(const float* __restrict__ X, const int32_t* __restrict__ n_rows, MatView W, MatView W2, ProjOut o,
                   int skip_above, GsPlan pl, GsNorm nrm, int32_t* __restrict__ status) {
  constexpr int NMAT = (EPI == EPI_SWIGLU) ? 2 : 1;
  extern __shared__ __align__(128) uint8_t gs_smem[];
  uint8_t* ring = gs_smem;
  float* xs = reinterpret_cast<float*>(gs_smem + pl.xs_offset);
  uint64_t* full = reinterpret_cast<uint64_t*>(gs_smem + pl.bar_offset);
  uint64_t* empty = full + pl.stages;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(empty + pl.stages);
  __shared__ float best_v[GS_CONSUMERS][8];
  __shared__ int best_i[GS_CONSUMERS][8];
  __shared__ float inv_s[8];

  const int K = W.K, N = W.N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblocks = (N + pl.fb - 1) / pl.fb;
  pdl_launch_dependents();
  if ((int)blockIdx.x >= nblocks) return;
  const int my_blocks = (nblocks - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < pl.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), GS_CONSUMERS);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Weights depend on no earlier kernel: when this launch certainly runs (no
  // row-count skip), the first blocks are requested before waiting for the
  // previous kernel.
  const int pre = (skip_above == 0) ? min(my_blocks, pl.stages) : 0;
  if (warp == GS_CONSUMERS && lane == 0)
    for (int i = 0; i < pre; ++i) gs_issue<FMT, NMAT>(W, W2, pl, ring, full, i, i, blockIdx.x + i * gridDim.x);
  pdl_wait();
  const int rows = n_rows[0];
  if ((skip_above > 0 && rows > skip_above) || rows <= 0) {
    if (warp == GS_CONSUMERS && lane == 0) {  // let the early copies land before leaving
      volatile int32_t never = 0;
      for (int i = 0; i < pre; ++i) mbar_wait(smem_u32(&full[i]), 0, &never);
    }
    return;
  }
  int it = 0;  // pipeline position, continued across row chunks
  for (int r0 = 0; r0 < rows; r0 += 8) {
    const int nr = min(8, rows - r0);
    float4* xs4 = reinterpret_cast<float4*>(xs);
    const bool copy_in = nrm.h_in && blockIdx.x == 0;
    for (int f = threadIdx.x; f < nr * K / 4; f += blockDim.x) {
      const int r = f / (K / 4), fi = f % (K / 4);
      const int src = nrm.map ? nrm.map[r0 + r] : r0 + r;
      const float4 v = reinterpret_cast<const float4*>(X + (int64_t)src * K)[fi];
      xs4[r * (K / 4) + swz_slot(fi)] = v;
      if (copy_in) reinterpret_cast<float4*>(nrm.h_in + (int64_t)src * K)[fi] = v;
    }
    __syncthreads();
    if (nrm.g) {
      if (warp < nr) {  // warp r: sum of squares of row r
        float ss = 0.f;
        for (int q = lane; q < K / 4; q += 32) {
          const float4 v = xs4[warp * (K / 4) + q];
          ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        }
        ss = warp_sum(ss);
        if (lane == 0) inv_s[warp] = rsqrtf(ss / (float)K + nrm.eps);
      }
      __syncthreads();
      for (int f = threadIdx.x; f < nr * K / 4; f += blockDim.x) {
        const int r = f / (K / 4), fi = f % (K / 4);
        const float inv = inv_s[r];
        const float4 gg = reinterpret_cast<const float4*>(nrm.g)[fi];
        float4& v = xs4[r * (K / 4) + swz_slot(fi)];
        v.x = v.x * inv * gg.x;
        v.y = v.y * inv * gg.y;
        v.z = v.z * inv * gg.z;
        v.w = v.w * inv * gg.w;
      }
      __syncthreads();
    }
    if (warp == GS_CONSUMERS) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        for (int i = 0; i < my_blocks; ++i) {
          const int g = it + i, s = g % pl.stages, rd = g / pl.stages;
          if (g < pre) continue;  // requested before the dependency wait
          if (rd > 0 && !mbar_wait(smem_u32(&empty[s]), (rd - 1) & 1, abort_flag)) break;
          gs_issue<FMT, NMAT>(W, W2, pl, ring, full, s, rd, blockIdx.x + i * gridDim.x);
        }
      }
    } else {
      // ----------------------------------------------------------- consumers
      float bv[8];
      int bi[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) { bv[r] = -INFINITY; bi[r] = 0x7fffffff; }
      for (int i = 0; i < my_blocks; ++i) {
        const int g = it + i, s = g % pl.stages, rd = g / pl.stages;
        if (!mbar_wait(smem_u32(&full[s]), rd & 1, abort_flag)) break;
        const int b = blockIdx.x + i * gridDim.x;
        const int nrow = min(pl.fb, N - b * pl.fb);
        const uint8_t* stage = ring + (size_t)(s * NMAT) * pl.stage_bytes;
        switch (nr) {
          case 1: gs_consume<FMT, 1, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 2: gs_consume<FMT, 2, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 3: gs_consume<FMT, 3, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 4: gs_consume<FMT, 4, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 5: gs_consume<FMT, 5, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 6: gs_consume<FMT, 6, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          case 7: gs_consume<FMT, 7, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
          default: gs_consume<FMT, 8, EPI>(stage, pl.stage_bytes, b, nrow, pl, W, xs, r0, rows, o, bv, bi); break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      }
      if constexpr (EPI == EPI_ARGMAX) {
        if (lane == 0)
#pragma unroll
          for (int r = 0; r < 8; ++r) { best_v[warp][r] = bv[r]; best_i[warp][r] = bi[r]; }
      }
    }
    it += my_blocks;
    __syncthreads();
    if constexpr (EPI == EPI_ARGMAX) {
      if (blockIdx.x == 0 && threadIdx.x == 0 && o.n_parts_dev) o.n_parts_dev[0] = o.n_parts;
      if (threadIdx.x < nr) {
        const int r = threadIdx.x;
        float v = best_v[0][r];
        int ix = best_i[0][r];
        for (int w = 1; w < GS_CONSUMERS; ++w)
          if (better(best_v[w][r], best_i[w][r], v, ix)) { v = best_v[w][r]; ix = best_i[w][r]; }
        o.part_val[(int64_t)(r0 + r) * o.n_parts + blockIdx.x] = v;
        o.part_idx[(int64_t)(r0 + r) * o.n_parts + blockIdx.x] = ix;
      }
      __syncthreads();
    }
    if (*abort_flag) break;
  }
  if (threadIdx.x == 0 && *abort_flag) {
    atomicOr(status, ST_TIMEOUT);
    // let copies already issued land before the CTA's shared memory is released
    volatile int32_t never = 0;
    for (int g = (it > pl.stages ? it - pl.stages : 0); g < it; ++g)
      mbar_wait(smem_u32(&full[g % pl.stages]), (g / pl.stages) & 1, &never);
  }
}

}  // namespace tl
