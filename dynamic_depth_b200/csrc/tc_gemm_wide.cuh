// Projection over many activation rows (prompts): a persistent tcgen05 GEMM.
//
// Y[rows, N] = X[rows, K] * W[N, K]^T as its transpose, like tc_gemm_kernel:
// the weight tile is the M = 128 operand and NT activation rows the N
// operand (NT = 256 for one matrix, 128 for the gate/up pair, so every tile
// is 128 x 256 MMA columns).  Unlike the decode kernel, one CTA per SM loops
// over output tiles (weight tile fastest, so the CTAs of a wave share their
// activation tiles in L2) with the full K per tile, and the tile's epilogue
// overlaps the next tile's main loop: the TMEM accumulator is double
// buffered (2 x 256 columns).
//
// Warp roles (384 threads; one lane of the producer and of the MMA warp runs
// the whole issue loop): warp 0 issues the TMA loads (raw weight tile and
// fp16 activation tile per 64-wide k-block) into a ring of stages; warps 4-7
// convert the raw weight tile to fp16 in the canonical K-major SWIZZLE_128B
// layout (INT4: (u - 8) * scale rounded once to fp16, scales read from
// global memory one k-block ahead); warp 1 issues the MMAs (4 per k-block and matrix) and
// commits stages back to the producer and finished accumulators to the
// epilogue; warps 8-11 read the accumulator (TMEM lane quadrant = warp % 4)
// and apply the epilogue; warp 2 owns the TMEM allocation.  Every mbarrier
// wait is bounded (~1.5 s); on expiry the CTA records ST_TIMEOUT, lets its
// copies in flight land and frees its TMEM.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tc_gemm.cuh"

namespace tl {

template <int NMAT, int FMT>
struct TcWideCfg {
  static constexpr int NT = 256 / NMAT;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = NT * 64 * 2;
  static constexpr int RAW_BYTES = (FMT == TL_FMT_INT4) ? 128 * 32 : (FMT == FMT_F16 ? 0 : 128 * 128);
  // 64-wide k-blocks per pipeline stage (two per stage, with only two stages fitting, measured slower:
  // 766 against 837 TFLOP/s on the 64 x 512-token prompt pass)
  static constexpr int KPS = 1;
  static constexpr int stage_bytes = NMAT * (KPS * A_BYTES + RAW_BYTES) + KPS * B_BYTES;
  static constexpr int LIMIT = 227 * 1024;  // opt-in shared memory per CTA
  static constexpr int RESERVE = 2048;      // 1024-byte alignment slack + barriers
  static constexpr int FIT = (LIMIT - RESERVE) / stage_bytes;
  static constexpr int STAGES = FIT > 4 ? 4 : FIT;
  static constexpr int SMEM = STAGES * stage_bytes + RESERVE;
  static constexpr int TMEM_COLS = 512;     // two accumulators of NMAT x NT columns
  static constexpr int THREADS = 384;
  static_assert(STAGES >= 2, "tile does not fit in shared memory");
  static_assert(2 * NMAT * NT == TMEM_COLS, "double-buffered accumulator must fill TMEM exactly");
  // one CTA per SM (shared memory), so its 512 TMEM columns are never contended
  static_assert(SMEM > LIMIT / 2, "a second CTA could share the SM and its TMEM");
};

// 32 consecutive accumulator columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int NMAT, int FMT, int EPI>
__global__ void __launch_bounds__(384, 1)
tc_gemm_wide_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapW2,
                    const __grid_constant__ CUtensorMap mapX, TcParams p) {
  using C = TcWideCfg<NMAT, FMT>;
  constexpr int NT = C::NT, STAGES = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_wide[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_wide) + 1023) & ~uintptr_t(1023));
  constexpr int KPS = C::KPS;
  uint8_t* sA = base;                                  // [STAGES][NMAT][KPS][A_BYTES] fp16 weight tiles
  uint8_t* sB = sA + STAGES * NMAT * KPS * C::A_BYTES;  // [STAGES][KPS][B_BYTES] fp16 activation tiles
  uint8_t* sRaw = sB + STAGES * KPS * C::B_BYTES;      // [STAGES][NMAT][RAW_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + STAGES * NMAT * C::RAW_BYTES);
  uint64_t* full = bars;                  // TMA landed
  uint64_t* afull = bars + STAGES;        // weight tile converted
  uint64_t* empty = bars + 2 * STAGES;    // MMAs of the stage finished
  uint64_t* accfull = bars + 3 * STAGES;  // [2] accumulator complete
  uint64_t* accempty = accfull + 2;       // [2] accumulator read out
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(accempty + 2);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&afull[s]), 4);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accfull[b]), 1);
      mbar_init(smem_u32(&accempty[b]), 4);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  const int rows = p.n_rows[0];
  const int m_tiles = (p.N + 127) / 128;
  const int n_tiles = rows > p.skip_at_or_below ? (rows + NT - 1) / NT : 0;
  const int n_total = m_tiles * n_tiles;
  const int nkb = p.kb_wrap << p.split16;  // k-steps (split activations: two per weight block, tc_xblock)
  const int nks = (nkb + KPS - 1) / KPS;  // pipeline steps per tile

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    // one lane runs the whole producer loop
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_total && ok; t += gridDim.x) {
        const int m0 = (t % m_tiles) * 128, n0 = (t / m_tiles) * NT;
        for (int ks = 0; ks < nks; ++ks, ++g) {
          const int s = g % STAGES, r = g / STAGES;
          if (r > 0 && !mbar_wait(smem_u32(&empty[s]), (r - 1) & 1, abort_flag)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[s]);
          const int nq = min(KPS, nkb - ks * KPS);  // k-blocks in this step
          if constexpr (FMT == FMT_F16) {  // fp16 weight tiles straight into the MMA layout
            mbar_expect_tx(fb, nq * (NMAT * C::A_BYTES + C::B_BYTES));
            for (int q = 0; q < nq; ++q) {
              const int kb = ks * KPS + q, kbw = tc_wblock(p, kb);
              tma_load_2d(smem_u32(sA + ((s * NMAT + 0) * KPS + q) * C::A_BYTES), &mapW, kbw * 64, m0, fb);
              if constexpr (NMAT == 2)
                tma_load_2d(smem_u32(sA + ((s * NMAT + 1) * KPS + q) * C::A_BYTES), &mapW2, kbw * 64, m0, fb);
              tma_load_2d(smem_u32(sB + (s * KPS + q) * C::B_BYTES), &mapX, tc_xblock(p, kb) * 64, n0, fb);
            }
          } else {
            const int kb = ks, kbw = tc_wblock(p, kb);
            mbar_expect_tx(fb, NMAT * C::RAW_BYTES + C::B_BYTES);
            const int wx = (FMT == TL_FMT_INT4) ? kbw * 32 : kbw * 64;
            tma_load_2d(smem_u32(sRaw + (s * NMAT + 0) * C::RAW_BYTES), &mapW, wx, m0, fb);
            if constexpr (NMAT == 2) tma_load_2d(smem_u32(sRaw + (s * NMAT + 1) * C::RAW_BYTES), &mapW2, wx, m0, fb);
            tma_load_2d(smem_u32(sB + s * C::B_BYTES), &mapX, tc_xblock(p, kb) * 64, n0, fb);
          }
        }
      }
      if (*abort_flag) {  // let copies already in flight land before the CTA leaves
        for (int i = (g > STAGES ? g - STAGES : 0); i < g; ++i) {
          volatile int32_t never = 0;
          mbar_wait(smem_u32(&full[i % STAGES]), (i / STAGES) & 1, &never);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    // one lane runs the whole issue loop: no warp-wide step (shuffle, elect, sync) between k-blocks, so the
    // next MMAs follow a completed barrier as closely as possible
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_f16<NT>();
      int g = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_total && ok; t += gridDim.x, ++it) {
        const int buf = it & 1, use = it >> 1;
        if (use > 0 && !mbar_wait(smem_u32(&accempty[buf]), (use - 1) & 1, abort_flag)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t acc = tmem + (uint32_t)(buf * NMAT * NT);
        for (int ks = 0; ks < nks; ++ks, ++g) {
          const int s = g % STAGES, r = g / STAGES;
          if ((FMT != FMT_F16 && !mbar_wait(smem_u32(&afull[s]), r & 1, abort_flag)) ||
              !mbar_wait(smem_u32(&full[s]), r & 1, abort_flag)) {
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const int nq = min(KPS, nkb - ks * KPS);
          for (int q = 0; q < nq; ++q) {
            const uint32_t b_addr = smem_u32(sB + (s * KPS + q) * C::B_BYTES);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bdesc = umma_desc(b_addr + kk * 32);
#pragma unroll
              for (int mat = 0; mat < NMAT; ++mat) {
                const uint64_t adesc = umma_desc(smem_u32(sA + ((s * NMAT + mat) * KPS + q) * C::A_BYTES) + kk * 32);
                umma_f16(acc + mat * NT, adesc, bdesc, idesc, (ks > 0 || q > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          umma_commit(smem_u32(&empty[s]));
        }
        if (ok) umma_commit(smem_u32(&accfull[buf]));
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8 && FMT != FMT_F16) {
    // ------------------------------------------------------------ convert
    const int tr = threadIdx.x - 128;  // weight row within the tile
    const int gpr = (FMT == TL_FMT_INT4) ? p.K / p.group : 0;
    const bool whole_groups = (FMT == TL_FMT_INT4) && p.group % 64 == 0;
    // INT4: this row's scales of a k-block, fetched one k-block ahead of their use
    auto fetch_scales = [&](int t, int kb_act, __half (&out)[NMAT][8]) {
      const int m = (t % m_tiles) * 128 + tr;
      const int kb = tc_wblock(p, kb_act);
#pragma unroll
      for (int mat = 0; mat < NMAT; ++mat) {
        const __half* sc = (mat == 0 ? p.scales : p.scales2) + (int64_t)m * gpr;
#pragma unroll
        if (whole_groups) {  // the k-block lies inside one scale group: one load
          const __half h = (m < p.N) ? sc[(kb * 64) / p.group] : __float2half(0.f);
#pragma unroll
          for (int c = 0; c < 8; ++c) out[mat][c] = h;
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) out[mat][c] = (m < p.N) ? sc[(kb * 64 + 8 * c) / p.group] : __float2half(0.f);
        }
      }
    };
    __half sc_cur[NMAT][8], sc_nxt[NMAT][8];
    if constexpr (FMT == TL_FMT_INT4) {
      if ((int)blockIdx.x < n_total) fetch_scales(blockIdx.x, 0, sc_cur);
    }
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_total && ok; t += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        const int s = g % STAGES, r = g / STAGES;
        if constexpr (FMT == TL_FMT_INT4) {
          const int tn = kb + 1 < nkb ? t : t + (int)gridDim.x, kn = kb + 1 < nkb ? kb + 1 : 0;
          if (tn < n_total) fetch_scales(tn, kn, sc_nxt);
        }
        __half2 sc2[NMAT][8];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
          for (int c = 0; c < 8; ++c) sc2[mat][c] = __halves2half2(sc_cur[mat][c], sc_cur[mat][c]);
        // every lane waits (each reads the landed tile); the warp leaves together
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full[s]), r & 1, abort_flag))) { ok = false; break; }
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
          uint8_t* arow = sA + (s * NMAT + mat) * C::A_BYTES + tr * 128;
          const uint8_t* raw = sRaw + (s * NMAT + mat) * C::RAW_BYTES;
          if constexpr (FMT == TL_FMT_INT4) {
            const uint4 w0 = *reinterpret_cast<const uint4*>(raw + tr * 32);
            const uint4 w1 = *reinterpret_cast<const uint4*>(raw + tr * 32 + 16);
            const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(arow + ((c ^ (tr & 7)) << 4)) = int4_word_to_half8(w[c], sc2[mat][c]);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 v = *reinterpret_cast<const uint4*>(raw + tr * 128 + c * 16);
              *reinterpret_cast<uint4*>(arow + ((c ^ (tr & 7)) << 4)) = bf16x8_to_half8(v);
            }
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&afull[s]));
        if constexpr (FMT == TL_FMT_INT4) {
#pragma unroll
          for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int c = 0; c < 8; ++c) sc_cur[mat][c] = sc_nxt[mat][c];
        }
      }
    }
  } else if (warp >= 8) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    const int tr = q * 32 + lane;
    int it = 0;
    for (int t = blockIdx.x; t < n_total; t += gridDim.x, ++it) {
      const int buf = it & 1, use = it >> 1;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&accfull[buf]), use & 1, abort_flag))) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int m = (t % m_tiles) * 128 + tr, n0 = (t / m_tiles) * NT;
      const int ncols = min(NT, rows - n0);
      const uint32_t acc = tmem + (uint32_t)(buf * NMAT * NT) + ((uint32_t)(q * 32) << 16);
      for (int j = 0; j < ncols; j += 32) {
        float v[32], v2[32];
        tmem_ld32(acc + j, v);
        if constexpr (NMAT == 2) {
          tmem_ld32(acc + NT + j, v2);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v2[e] = 0.f;
        }
        if (m < p.N) tc_emit_rows<EPI, 32>(p, n0 + j, min(32, ncols - j), m, v, v2);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&accempty[buf]));
    }
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

// The resident fp16 copy of one block matrix (made at weight load): out [N][K]
// fp16 with exactly the values the converting kernels build in shared memory
// (INT4: (u - 8) exact, times the fp16 group scale, rounded once; BF16: the
// same value in fp16).  One thread per 8 consecutive elements.
__global__ void stage_f16_kernel(MatView W, __half* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8-element word
  const int64_t words = (int64_t)W.N * W.K / 8;
  if (i >= words) return;
  const int64_t n = i / (W.K / 8), w = i % (W.K / 8);
  uint4 v;
  if (W.fmt == TL_FMT_INT4) {
    const uint32_t word = reinterpret_cast<const uint32_t*>(W.q)[i];
    const __half sc = W.s[n * (W.K / W.group) + (8 * w) / W.group];
    v = int4_word_to_half8(word, __halves2half2(sc, sc));
  } else {
    v = bf16x8_to_half8(reinterpret_cast<const uint4*>(W.bf)[i]);
  }
  reinterpret_cast<uint4*>(out)[i] = v;
}

}  // namespace tl
