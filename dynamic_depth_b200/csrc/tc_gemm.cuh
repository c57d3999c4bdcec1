// W4A16 / BF16 projection on the 5th-generation tensor cores (tcgen05 + TMEM).
// (The TMA and MMA warps run their loops with all lanes; one elected lane issues.)
//
// Y[rows, N] = X[rows, K] * W[N, K]^T computed as its transpose: the weight
// tile is the 128-row M operand and the activation rows are the N operand
// (NT = 64, 128 or 256 rows), so decode batches of a few dozen lanes still fill
// an M=128 instruction while the kernel streams each weight byte once.
//
// Per CTA (256 threads): warp 0 issues TMA loads of the raw weight tile (INT4
// nibbles or BF16, unswizzled) and of the fp16 activation tile (SWIZZLE_128B)
// into a ring of stages; warps 4-7 convert the raw weight tile to fp16 in the
// canonical K-major SWIZZLE_128B layout (INT4: (u - 8) * scale rounded once to
// fp16) and later run the epilogue; warp 1 issues tcgen05.mma (K = 16 per
// instruction, 4 per 64-wide k-block) into a TMEM accumulator and commits each
// stage back to the producer; warp 2 owns the TMEM allocation.  Split-K CTAs
// of one output tile form a thread-block cluster: each parks its fp32 partial
// tile in its own shared memory, and after a cluster barrier CTA z reduces the
// z-th slice of the tile's rows over the cluster's shared memory in split
// order (deterministic, no global scratch) and applies the epilogue (store,
// residual add, or silu(gate) * up).  Every mbarrier wait is bounded (~1.5 s
// of %globaltimer); on expiry the CTA records ST_TIMEOUT in the status word and
// still reaches both cluster barriers.
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace tl {

struct TcParams {
  const int32_t* n_rows;   // device scalar
  int32_t skip_at_or_below;
  int32_t N, K, group;
  int32_t kb_per_split;    // 64-wide k-blocks per split
  int32_t kb_wrap;         // k-blocks of the weights, K / 64
  int32_t split16;         // activation rows are [hi | lo] (see act16_put): 2 * kb_wrap k-steps (below)
  const __half* scales;    // INT4: [N][K/group]
  const __half* scales2;   // second matrix (gate/up pair)
  ProjOut o;               // EPI_STORE / EPI_SWIGLU: o.out [rows][ldo]; EPI_RESID: o.h / o.map
  __half* out16;           // fp16 copy of the EPI_SWIGLU output (the next projection's operand)
  int32_t* status;
};

constexpr int TC_SC_MAX = 33;  // scale groups per CTA row

// Weights already in fp16 (a block's resident copy, see stage_f16_kernel): the
// weight tile arrives by TMA in the canonical MMA layout and nothing is
// converted.
constexpr int FMT_F16 = 2;

// k-step j of a projection: weight block tc_wblock, activation block
// tc_xblock.  With split activations a weight block's hi and lo products run
// back to back (steps 2w and 2w + 1), so its second read comes from L2 and a
// CTA's k-steps cover a contiguous range of weight blocks.
__device__ __forceinline__ int tc_wblock(const TcParams& p, int j) { return j >> p.split16; }
__device__ __forceinline__ int tc_xblock(const TcParams& p, int j) {
  return p.split16 ? (j & 1) * p.kb_wrap + (j >> 1) : j;
}

template <int NT, int NMAT, int FMT>
struct TcCfg {
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = NT * 64 * 2;
  static constexpr int RAW_BYTES = (FMT == TL_FMT_INT4) ? 128 * 32 : (FMT == FMT_F16 ? 0 : 128 * 128);
  static constexpr int SC_BYTES = (FMT == TL_FMT_INT4) ? NMAT * 128 * TC_SC_MAX * 2 : 0;
  static constexpr int stage_bytes = NMAT * (A_BYTES + RAW_BYTES) + B_BYTES;
  static constexpr int fixed = SC_BYTES + 256 + 1024;
  // the 64-row single-matrix tile (decode batches) keeps 3 stages so two CTAs share an SM
  static constexpr int CAP = (NT == 64 && NMAT == 1) ? 3 : 4;
  static constexpr int STAGES = ((220 * 1024 - fixed) / stage_bytes) >= CAP ? CAP : ((220 * 1024 - fixed) / stage_bytes);
  static constexpr int SMEM = STAGES * stage_bytes + fixed;
  static constexpr int TMEM_COLS = (NMAT * NT <= 32) ? 32 : NMAT * NT;
  // split-K parks a [NMAT][NT][128] fp32 partial tile in the stage buffers
  static constexpr bool SPLIT_OK = NMAT * NT * 128 * 4 <= STAGES * stage_bytes;
  static_assert(STAGES >= 2, "tile does not fit in shared memory");
  // TMEM is allocated before the programmatic-dependency wait, so a CTA may
  // allocate while a CTA of the previous kernel on its SM still has to.  Any
  // tile holding more than 64 columns must leave no room for a second
  // tensor-core CTA on its SM (two CTAs above 114 KB exceed the SM's 228 KB);
  // two 64-column CTAs fit TMEM's 512 columns together.
  static_assert(TMEM_COLS <= 64 || SMEM > 114 * 1024, "TMEM could be oversubscribed by co-resident CTAs");
};

// K-major, SWIZZLE_128B canonical layout: 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

template <int NT>
__device__ __forceinline__ constexpr uint32_t umma_idesc_f16() {
  // D fp32, A/B fp16, both K-major, N = NT, M = 128
  return (1u << 4) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// INT4 device layout: in each 32-bit word of 8 consecutive k, element 2i is
// nibble i and element 2i+1 is nibble i + 4 (see the load-time repack), so
// (w >> 4i) & 0x000F000F is the pair (2i, 2i+1) as two 16-bit lanes.
__device__ __forceinline__ uint4 int4_word_to_half8(uint32_t w, __half2 s2) {
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t bits = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;  // (1024 + u) in each half
    __half2 h = *reinterpret_cast<const __half2*>(&bits);
    h = __hmul2(__hsub2(h, off), s2);  // (u - 8) exact, then one rounding of (u - 8) * s
    out[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ uint4 bf16x8_to_half8(uint4 v) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(__uint_as_float(in[i] << 16), __uint_as_float(in[i] & 0xFFFF0000u));
    out[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// Final value of one output element (SPLIT: the SwiGLU output's fp16 copy as
// hi and lo halves; a compile-time choice, which callers make once per row
// group: a per-element choice measured 13-20 % slower in the prompt GEMM).
template <int EPI, bool SPLIT = false>
__device__ __forceinline__ void tc_emit(const TcParams& p, int row, int m, float v, float v2) {
  const ProjOut& o = p.o;
  if constexpr (EPI == EPI_STORE) {
    o.out[(int64_t)row * o.ldo + m] = v;
  } else if constexpr (EPI == EPI_SWIGLU) {
    const float u = silu_f(v) * v2;
    if (o.out) o.out[(int64_t)row * o.ldo + m] = u;
    if (p.out16) {
      if constexpr (SPLIT) act16_put(p.out16, row, o.ldo, m, u, 1);
      else p.out16[(int64_t)row * o.ldo + m] = __float2half_rn(u);
    }
  } else if constexpr (EPI == EPI_RESID) {
    const int hr = o.map ? o.map[row] : row;
    o.h[(int64_t)hr * p.N + m] += v;
  }
}

// Final values of n consecutive activation rows (row0 .. row0+n-1) at output
// m.  The residual form loads all n residual elements before storing any, so
// the n read-modify-writes overlap instead of running one after another.
template <int EPI, int NV>
__device__ __forceinline__ void tc_emit_rows(const TcParams& p, int row0, int n, int m, const float (&v)[NV],
                                             const float (&v2)[NV]) {
  if constexpr (EPI == EPI_RESID) {
    const ProjOut& o = p.o;
    float* dst[NV];
    float hv[NV];
#pragma unroll
    for (int e = 0; e < NV; ++e) {
      const int hr = e < n ? (o.map ? o.map[row0 + e] : row0 + e) : 0;
      dst[e] = o.h + (int64_t)hr * p.N + m;
      hv[e] = e < n ? *dst[e] : 0.f;
    }
#pragma unroll
    for (int e = 0; e < NV; ++e)
      if (e < n) *dst[e] = hv[e] + v[e];
  } else if (EPI == EPI_SWIGLU && p.split16) {
#pragma unroll
    for (int e = 0; e < NV; ++e)
      if (e < n) tc_emit<EPI, true>(p, row0 + e, m, v[e], v2[e]);
  } else {
#pragma unroll
    for (int e = 0; e < NV; ++e)
      if (e < n) tc_emit<EPI, false>(p, row0 + e, m, v[e], v2[e]);
  }
}

template <int NT, int NMAT, int FMT, int EPI>
__global__ void __launch_bounds__(256, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapW2,
               const __grid_constant__ CUtensorMap mapX, TcParams p) {
  using C = TcCfg<NT, NMAT, FMT>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;                                          // [STAGES][NMAT][A_BYTES]
  uint8_t* sB = sA + STAGES * NMAT * C::A_BYTES;               // [STAGES][B_BYTES]
  uint8_t* sRaw = sB + STAGES * C::B_BYTES;                    // [STAGES][NMAT][RAW_BYTES]
  __half* sSc = reinterpret_cast<__half*>(sRaw + STAGES * NMAT * C::RAW_BYTES);  // [NMAT][128][TC_SC_MAX]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sSc) + C::SC_BYTES);
  uint64_t* full = bars;                // TMA landed (raw W + X)
  uint64_t* afull = bars + STAGES;      // fp16 weight tile converted
  uint64_t* empty = bars + 2 * STAGES;  // MMAs of the stage finished
  uint64_t* accfull = bars + 3 * STAGES;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + 3 * STAGES + 1);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * NT;
  const int nkb = p.kb_per_split, kb0 = blockIdx.z * nkb;
  const int S = gridDim.z;                      // split-K CTAs of this tile = cluster size
  float* red = reinterpret_cast<float*>(sA);    // [NMAT][NT][128] partial tile after the main loop
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&afull[s]), 4);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accfull), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32((const void*)tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  // Weight tiles depend on no earlier kernel: when this launch certainly runs
  // (no row-count skip), the first stages are requested before waiting for
  // the previous kernel.  Their barriers expect the weight bytes now and get
  // their arrival (with the activation bytes) after the wait.
  const int pre = (p.skip_at_or_below == 0) ? min(nkb, STAGES) : 0;
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      const uint32_t fb = smem_u32(&full[i]);
      const int kbw = tc_wblock(p, kb0 + i);
      if constexpr (FMT == FMT_F16) {  // straight into the MMA's A tiles
        mbar_add_tx(fb, NMAT * C::A_BYTES);
        tma_load_2d(smem_u32(sA + (i * NMAT + 0) * C::A_BYTES), &mapW, kbw * 64, m0, fb);
        if constexpr (NMAT == 2) tma_load_2d(smem_u32(sA + (i * NMAT + 1) * C::A_BYTES), &mapW2, kbw * 64, m0, fb);
      } else {
        mbar_add_tx(fb, NMAT * C::RAW_BYTES);
        const int wx = (FMT == TL_FMT_INT4) ? kbw * 32 : kbw * 64;
        tma_load_2d(smem_u32(sRaw + (i * NMAT + 0) * C::RAW_BYTES), &mapW, wx, m0, fb);
        if constexpr (NMAT == 2) tma_load_2d(smem_u32(sRaw + (i * NMAT + 1) * C::RAW_BYTES), &mapW2, wx, m0, fb);
      }
    }
  }
  pdl_wait();
  const int rows = p.n_rows[0];
  const bool active = !(rows <= p.skip_at_or_below || n0 >= rows);
  const int ncols = active ? min(NT, rows - n0) : 0;

  if (!active) {
    if (warp == 0 && lane == 0) {  // nothing to compute: let the early weight copies land, then leave
      for (int i = 0; i < pre; ++i) {
        mbar_arrive(smem_u32(&full[i]));
        volatile int32_t never = 0;
        mbar_wait(smem_u32(&full[i]), 0, &never);
      }
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    // the whole warp runs the loop (waits included); one elected lane issues
    int issued = 0;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % STAGES, r = i / STAGES;
      const int kb = kb0 + i;
      const uint32_t fb = smem_u32(&full[s]);
      if (i >= pre && r > 0 && !mbar_wait_warp(smem_u32(&empty[s]), (r - 1) & 1, abort_flag)) break;
      if (elect_one()) {
        if (i < pre) {
          mbar_expect_tx(fb, C::B_BYTES);
        } else if constexpr (FMT == FMT_F16) {
          mbar_expect_tx(fb, NMAT * C::A_BYTES + C::B_BYTES);
          const int kbw = tc_wblock(p, kb);
          tma_load_2d(smem_u32(sA + (s * NMAT + 0) * C::A_BYTES), &mapW, kbw * 64, m0, fb);
          if constexpr (NMAT == 2) tma_load_2d(smem_u32(sA + (s * NMAT + 1) * C::A_BYTES), &mapW2, kbw * 64, m0, fb);
        } else {
          mbar_expect_tx(fb, NMAT * C::RAW_BYTES + C::B_BYTES);
          const int kbw = tc_wblock(p, kb);
          const int wx = (FMT == TL_FMT_INT4) ? kbw * 32 : kbw * 64;
          tma_load_2d(smem_u32(sRaw + (s * NMAT + 0) * C::RAW_BYTES), &mapW, wx, m0, fb);
          if constexpr (NMAT == 2) tma_load_2d(smem_u32(sRaw + (s * NMAT + 1) * C::RAW_BYTES), &mapW2, wx, m0, fb);
        }
        tma_load_2d(smem_u32(sB + s * C::B_BYTES), &mapX, tc_xblock(p, kb) * 64, n0, fb);
      }
      __syncwarp();
      issued = i + 1;
    }
    if (*abort_flag && lane == 0) {  // let copies already in flight land before the CTA leaves
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
        volatile int32_t never = 0;
        mbar_wait(smem_u32(&full[i % STAGES]), (i / STAGES) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc = umma_idesc_f16<NT>();
    for (int i = 0; i < nkb; ++i) {
      const int s = i % STAGES, r = i / STAGES;
      if (FMT != FMT_F16 && !mbar_wait_warp(smem_u32(&afull[s]), r & 1, abort_flag)) break;
      if (!mbar_wait_warp(smem_u32(&full[s]), r & 1, abort_flag)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t b_addr = smem_u32(sB + s * C::B_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bdesc = umma_desc(b_addr + kk * 32);
#pragma unroll
          for (int mat = 0; mat < NMAT; ++mat) {
            const uint64_t adesc = umma_desc(smem_u32(sA + (s * NMAT + mat) * C::A_BYTES) + kk * 32);
            umma_f16(tmem + mat * NT, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&empty[s]));
      }
      __syncwarp();
    }
    if (elect_one()) umma_commit(smem_u32(accfull));
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------- convert + epilogue
    const int t = threadIdx.x - 128;  // weight row within the tile == TMEM lane
    const int q = warp - 4;
    const int gfirst = (FMT == TL_FMT_INT4) ? (tc_wblock(p, kb0) * 64) / p.group : 0;
    if constexpr (FMT == TL_FMT_INT4) {
      // this row's group scales for the CTA's K range (while the first TMA is in flight)
      const int glast = ((tc_wblock(p, kb0 + nkb - 1) + 1) * 64 - 1) / p.group;
      for (int mat = 0; mat < NMAT; ++mat) {
        const __half* sc = mat == 0 ? p.scales : p.scales2;
        const int64_t rowoff = (int64_t)(m0 + t) * (p.K / p.group);
        for (int j = 0; j <= glast - gfirst && j < TC_SC_MAX; ++j)
          sSc[(mat * 128 + t) * TC_SC_MAX + j] = (m0 + t < p.N) ? sc[rowoff + gfirst + j] : __float2half(0.f);
      }
    }
    bool ok = true;
    for (int i = 0; i < (FMT == FMT_F16 ? 0 : nkb) && ok; ++i) {  // (fp16 weights: nothing to convert)
      const int s = i % STAGES, r = i / STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full[s]), r & 1, abort_flag))) { ok = false; break; }
#pragma unroll
      for (int mat = 0; mat < NMAT; ++mat) {
        uint8_t* arow = sA + (s * NMAT + mat) * C::A_BYTES + t * 128;
        const uint8_t* raw = sRaw + (s * NMAT + mat) * C::RAW_BYTES;
        if constexpr (FMT == TL_FMT_INT4) {
          const uint4 w0 = *reinterpret_cast<const uint4*>(raw + t * 32);
          const uint4 w1 = *reinterpret_cast<const uint4*>(raw + t * 32 + 16);
          const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          const int kbase = tc_wblock(p, kb0 + i) * 64;
          const __half* srow = sSc + (mat * 128 + t) * TC_SC_MAX;
          if (p.group % 64 == 0) {  // the k-block lies inside one scale group
            const __half sc = srow[kbase / p.group - gfirst];
            const __half2 s2 = __halves2half2(sc, sc);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(arow + ((c ^ (t & 7)) << 4)) = int4_word_to_half8(w[c], s2);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const __half sc = srow[(kbase + 8 * c) / p.group - gfirst];
              *reinterpret_cast<uint4*>(arow + ((c ^ (t & 7)) << 4)) = int4_word_to_half8(w[c], __halves2half2(sc, sc));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(raw + t * 128 + c * 16);
            *reinterpret_cast<uint4*>(arow + ((c ^ (t & 7)) << 4)) = bf16x8_to_half8(v);
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&afull[s]));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(smem_u32(accfull), 0, abort_flag))) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int m = m0 + t;
      const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
      if constexpr (EPI == EPI_ARGMAX) {
        // per activation row: the best (value, index) of this tile's 128 outputs
        float* bv_s = reinterpret_cast<float*>(sA);          // [4 warps][NT]
        int* bi_s = reinterpret_cast<int*>(sA) + 4 * NT;      // [4 warps][NT]
        for (int j = 0; j < ncols; j += 8) {
          float v[8];
          tmem_ld8(tl + j, v);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (j + e >= ncols) break;
            float bv = (m < p.N) ? v[e] : -INFINITY;
            int bi = (m < p.N) ? m : 0x7fffffff;
            if (p.o.logits && m < p.N) p.o.logits[(int64_t)p.o.lmap[n0 + j + e] * p.o.ldo + m] = v[e];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
              if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if (lane == 0) { bv_s[q * NT + j + e] = bv; bi_s[q * NT + j + e] = bi; }
          }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        for (int c = t; c < ncols; c += 128) {  // activation rows of the tile (up to NT = 256): 128 threads
          float bv = bv_s[c];
          int bi = bi_s[c];
          for (int w = 1; w < 4; ++w)
            if (better(bv_s[w * NT + c], bi_s[w * NT + c], bv, bi)) { bv = bv_s[w * NT + c]; bi = bi_s[w * NT + c]; }
          p.o.part_val[(int64_t)(n0 + c) * p.o.n_parts + blockIdx.x] = bv;
          p.o.part_idx[(int64_t)(n0 + c) * p.o.n_parts + blockIdx.x] = bi;
        }
        if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0 && p.o.n_parts_dev) p.o.n_parts_dev[0] = p.o.n_parts;
      } else
      for (int j = 0; j < ncols; j += 8) {
        float v[8], v2[8];
        tmem_ld8(tl + j, v);
        if constexpr (NMAT == 2) tmem_ld8(tl + NT + j, v2);
        if (S == 1) {
          if constexpr (NMAT == 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) v2[e] = 0.f;
          }
          if (m < p.N) tc_emit_rows<EPI, 8>(p, n0 + j, min(8, ncols - j), m, v, v2);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            red[(j + e) * 128 + t] = v[e];
            if constexpr (NMAT == 2) red[(NT + j + e) * 128 + t] = v2[e];
          }
        }
      }
    }
  }
  if (active && S > 1) {
    // split-K: reduce this CTA's slice of rows over the cluster's partial tiles
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int z = blockIdx.z;
    const int f0 = (z * 128) / S, nf = ((z + 1) * 128) / S - f0;
    const float* rz[8];
#pragma unroll
    for (int zz = 0; zz < 8; ++zz) rz[zz] = cluster.map_shared_rank(red, zz < S ? zz : 0);
    for (int i = threadIdx.x; i < nf * ncols; i += blockDim.x) {
      const int tt = f0 + i % nf, j = i / nf;
      float pa[8], pb[8];
#pragma unroll
      for (int zz = 0; zz < 8; ++zz) {  // all remote loads first, then the sum in split order
        pa[zz] = zz < S ? rz[zz][j * 128 + tt] : 0.f;
        if constexpr (NMAT == 2) pb[zz] = zz < S ? rz[zz][(NT + j) * 128 + tt] : 0.f;
      }
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int zz = 0; zz < 8; ++zz) {
        if (zz < S) {
          a += pa[zz];
          if constexpr (NMAT == 2) b += pb[zz];
        }
      }
      if (m0 + tt < p.N) {
        if (p.split16) tc_emit<EPI, true>(p, n0 + j, m0 + tt, a, b);
        else tc_emit<EPI, false>(p, n0 + j, m0 + tt, a, b);
      }
    }
    cluster.sync();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, ST_TIMEOUT);
  if (warp == 2) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// Load-time repack of an INT4 matrix (standard packing: element e of each
// 8-element word in nibble e) into the device layout used above and by the
// CUDA-core kernels (element 2i in nibble i, 2i+1 in nibble i + 4).  In place.
__global__ void int4_repack_kernel(uint32_t* __restrict__ w, int64_t n_words) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_words) return;
  const uint32_t x = w[i];
  uint32_t y = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    y |= ((x >> (4 * e)) & 0xFu) << (4 * nib_pos(e));
  }
  w[i] = y;
}

}  // namespace tl
