// Attention on the 5th-generation tensor cores (tcgen05 + TMEM) for blocks of
// up to 128 query rows that read one KV slot of one cache: a prompt tile
// (consecutive positions of one lane, causal) or, for decode rows whose caches
// map the same shared-prefix pages, all such rows at one loop iteration
// against the shared prefix ("Benchmark Comparison" (measured benchmarks),
// section 2: one cached prefix serves many requests, and on a looped model
// every loop iteration).
//
// Per CTA (one 128-row query tile, one head), flash-attention style over key
// blocks of 64 positions:
//   S = Q K^T             tcgen05.mma, M = 128 query rows, N = 64 keys, K = hd
//   p = exp2(S - m_run)   one thread per query row (TMEM lane), online max/sum
//   O_j = P V             tcgen05.mma, M = 128, N = hd, K = 64 keys
//   O = O * corr + O_j    in the softmax threads' registers
// Q (rotated, scaled by log2(e)/sqrt(hd), fp16) and P (fp16) sit in shared
// memory in the canonical K-major 128-byte-swizzled layout; K tiles arrive by
// TMA in the same layout (keys as rows, the B operand K-major); V tiles arrive
// by TMA as rows of keys, i.e. the B operand of P V in its N-major
// ("MN-major") form.  S and O_j live in TMEM, double buffered so the MMA warp
// computes S of block j+1 while the softmax warps work on block j.
//
// Warp roles (256 threads): warp 0 TMA producer (K, V of each block into a
// 3-stage ring), warp 1 MMA issuer (one elected lane), warp 2 TMEM allocator,
// warps 4-7 query rows (load Q, softmax, write P, accumulate O, epilogue).
// Every wait is bounded (~1.5 s); on expiry the CTA records ST_TIMEOUT, lets
// its copies land and frees its TMEM.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tc_gemm.cuh"

namespace tl {

template <int HD>
struct AttnTcCfg {
  static constexpr int BM = 128, BN = 64;
  static constexpr int CT = HD / 64;                    // 64-wide column tiles of a row
  static constexpr int Q_BYTES = BM * HD * 2;           // CT tiles of [128 x 64] fp16
  static constexpr int KV_TILE = BN * 128;              // [64 keys x 64 cols] fp16 = 8 KB
  static constexpr int STAGE = 2 * CT * KV_TILE;        // K tiles, then V tiles
  static constexpr int STAGES = 3;
  static constexpr int P_BYTES = BM * BN * 2;           // [128 x 64] fp16 = 16 KB
  static constexpr int SMEM = 1024 + Q_BYTES + STAGES * STAGE + 2 * P_BYTES + 512 + 4 * 128;
  static constexpr int TMEM_COLS = HD == 64 ? 256 : 512;  // S[2] (64 each), then O_j[2] (HD each)
  static_assert(HD == 64 || HD == 128, "tensor-core attention takes head widths 64 and 128");
};

struct AttnTcParams {
  const float* q;                // mode 0: rotated q rows [rows][d]; mode 1: projection rows [rows][3d]
  const float2* rope;            // mode 1: RoPE table [max_seq][hd/2]
  Rows rows;
  const int2* tiles;             // mode 0: (first row, rows) of each tile
  int32_t mode;                  // 0 prompt tiles (causal), 1 shared-prefix groups
  const int32_t* lane_shared;    // mode 1: shared prefix positions per lane (0 = none)
  int32_t chunks;                // mode 1: CTAs per loop iteration (128-row chunks of the rows)
  float* casc;                   // mode 1: [rows][H][hd + 2] partial (max, sum, output)
  float* o;                      // mode 0: output rows [rows][d]
  __half* o16;                   // mode 0: fp16 copy (hi and lo halves with split16)
  int32_t split16;
  KVGeom g;
  int32_t slot_base, slot_stride;
  int32_t* status;
};

// Instruction descriptor: D fp32, A/B fp16, A K-major, B K-major (b_mn = 0) or N-major (b_mn = 1).
__device__ __forceinline__ constexpr uint32_t attn_idesc(int M, int N, int b_mn) {
  return (1u << 4) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory descriptor of a 128-byte-swizzled tile: lbo / sbo in bytes.
__device__ __forceinline__ uint64_t attn_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tmem_ld32_att(uint32_t taddr, float (&v)[32]) {
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

template <int HD>
__global__ void __launch_bounds__(256, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap kvmap, AttnTcParams p) {
  using C = AttnTcCfg<HD>;
  constexpr int BM = C::BM, BN = C::BN, CT = C::CT, STAGES = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_atc[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_atc) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;                              // [CT][128 x 64] fp16
  uint8_t* sKV = sQ + C::Q_BYTES;                  // [STAGES][K tiles (CT), V tiles (CT)]
  uint8_t* sP = sKV + STAGES * C::STAGE;           // [2][128 x 64] fp16
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * C::P_BYTES);
  uint64_t* full = bars;                 // [STAGES] K/V landed
  uint64_t* empty = bars + STAGES;       // [STAGES] both MMAs of the stage done
  uint64_t* s_full = bars + 2 * STAGES;  // [2] S of a block in TMEM
  uint64_t* p_full = s_full + 2;         // [2] P written (S buffer free)
  uint64_t* o_full = p_full + 2;         // [2] O_j in TMEM
  uint64_t* o_free = o_full + 2;         // [2] O_j read
  uint64_t* q_full = o_free + 2;         // Q written
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(q_full + 1);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  int32_t* sh_rows = reinterpret_cast<int32_t*>(bars + 64);  // [128] row index of each query row (-1: none)
  __shared__ int32_t sh_cnt, sh_lane, sh_kend, sh_iter;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const KVGeom& g = p.g;
  const int H = g.H, d = H * HD;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&s_full[b]), 1);
      mbar_init(smem_u32(&p_full[b]), 4);
      mbar_init(smem_u32(&o_full[b]), 1);
      mbar_init(smem_u32(&o_free[b]), 4);
    }
    mbar_init(smem_u32(q_full), 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32((const void*)tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  // ------------------------------------------------------------- the tile's rows
  if (p.mode == 0) {
    if (threadIdx.x == 0) {
      const int2 t = p.tiles[blockIdx.x];
      const int n = p.rows.n[0];
      int cnt = (t.x < n) ? min(min(t.y, BM), n - t.x) : 0;
      sh_cnt = cnt;
      sh_lane = cnt > 0 ? p.rows.lane[t.x] : 0;
      sh_iter = cnt > 0 ? p.rows.iter[t.x] : 0;
      sh_kend = cnt > 0 ? p.rows.pos[t.x + cnt - 1] + 1 : 0;
    }
    __syncthreads();
    if (threadIdx.x < BM) sh_rows[threadIdx.x] = threadIdx.x < sh_cnt ? p.tiles[blockIdx.x].x + threadIdx.x : -1;
  } else {
    // group = blockIdx.x / tiles_per_group: loop iteration; chunk = the rest; rows of that iteration whose lane maps
    // a shared prefix, in row order
    const int n = p.rows.n[0];
    const int iter = blockIdx.x / p.chunks, chunk = blockIdx.x % p.chunks;
    __shared__ int32_t wcnt[8];
    if (threadIdx.x == 0) sh_cnt = 0;
    __syncthreads();
    int seen = 0;  // rows of this iteration before the current 256-row window
    for (int w0 = 0; w0 < n; w0 += 256) {
      const int r = w0 + threadIdx.x;
      int take = 0;
      if (r < n) take = p.rows.iter[r] == iter && p.lane_shared[p.rows.lane[r]] > 0;
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      if (lane == 0) wcnt[warp] = __popc(bal);
      __syncthreads();
      int before = seen;
      for (int w = 0; w < warp; ++w) before += wcnt[w];
      const int idx = before + __popc(bal & ((1u << lane) - 1u));
      if (take && idx >= chunk * BM && idx < (chunk + 1) * BM) sh_rows[idx - chunk * BM] = r;
      int tot = 0;
      for (int w = 0; w < 8; ++w) tot += wcnt[w];
      seen += tot;
      __syncthreads();
    }
    const int cnt = max(0, min(BM, seen - chunk * BM));
    if (threadIdx.x < BM && threadIdx.x >= cnt) sh_rows[threadIdx.x] = -1;
    if (threadIdx.x == 0) {
      sh_cnt = cnt;
      sh_iter = iter;
      sh_lane = cnt > 0 ? p.rows.lane[sh_rows[0]] : 0;
      sh_kend = cnt > 0 ? p.lane_shared[sh_lane] : 0;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const int cnt = sh_cnt, kend = sh_kend;
  const int nkb = (kend + BN - 1) / BN;
  const int slot = p.slot_base + sh_iter * p.slot_stride;
  const int ln0 = sh_lane;

  if (cnt > 0 && nkb > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA
      const int64_t head_rows = g.page_tokens, page_rows = (int64_t)2 * H * g.page_tokens;
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < nkb && ok; ++j) {
        const int s = j % STAGES, r = j / STAGES;
        if (r > 0 && !mbar_wait_warp(smem_u32(&empty[s]), (r - 1) & 1, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          const uint32_t fb = smem_u32(&full[s]);
          uint32_t bytes = 0;
          int64_t ys[2];
          for (int b = 0; b < 2; ++b) {  // two 32-key boxes per block (a box never crosses a page)
            const int pos = j * BN + 32 * b;
            const int pg = pos >> g.page_shift;
            int page = -1;
            if (slot >= 0 && slot < g.n_slots && pg < g.pages_per_seq)
              page = g.page_table[((int64_t)ln0 * g.n_slots + slot) * g.pages_per_seq + pg];
            ys[b] = (page >= 0 && page < g.n_pages) ? (int64_t)page * page_rows + h * head_rows + (pos & (g.page_tokens - 1)) : -1;
            if (ys[b] < 0 && pos < kend) set_status(p.status, ST_BAD_PAGE);
            if (ys[b] >= 0) bytes += 2 * CT * 32 * 128;
          }
          mbar_expect_tx(fb, bytes);
          uint8_t* st = sKV + s * C::STAGE;
          for (int b = 0; b < 2; ++b) {
            if (ys[b] < 0) continue;
            for (int ct = 0; ct < CT; ++ct) {
              tma_load_2d(smem_u32(st + ct * C::KV_TILE + b * 32 * 128), &kvmap, ct * 64, (int)ys[b], fb);
              tma_load_2d(smem_u32(st + (CT + ct) * C::KV_TILE + b * 32 * 128), &kvmap, ct * 64,
                          (int)(ys[b] + H * head_rows), fb);
            }
          }
          if (bytes == 0) mbar_arrive(fb);
        }
        __syncwarp();
        issued = j + 1;
      }
      if (*abort_flag && lane == 0) {
        volatile int32_t never = 0;
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(smem_u32(&full[i % STAGES]), (i / STAGES) & 1, &never);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA
      constexpr uint32_t idesc_s = attn_idesc(BM, BN, 0);
      constexpr uint32_t idesc_o = attn_idesc(BM, HD, 1);
      bool ok = mbar_wait_warp(smem_u32(q_full), 0, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j % STAGES, buf = j & 1;
        if (!mbar_wait_warp(smem_u32(&full[s]), (j / STAGES) & 1, abort_flag)) return false;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint8_t* st = sKV + s * C::STAGE;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t a = attn_desc(smem_u32(sQ + (kk / 4) * (BM * 128)) + (kk % 4) * 32, 16, 1024);
            const uint64_t b = attn_desc(smem_u32(st + (kk / 4) * C::KV_TILE) + (kk % 4) * 32, 16, 1024);
            umma_f16(tmem + buf * BN, a, b, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&s_full[buf]));
        }
        __syncwarp();
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nkb && ok; ++j) {
        const int s = j % STAGES, buf = j & 1;
        if (j + 1 < nkb && !issue_s(j + 1)) break;
        if (!mbar_wait_warp(smem_u32(&p_full[buf]), (j >> 1) & 1, abort_flag)) break;
        if (j >= 2 && !mbar_wait_warp(smem_u32(&o_free[buf]), ((j >> 1) - 1) & 1, abort_flag)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint8_t* vt = sKV + s * C::STAGE + CT * C::KV_TILE;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t a = attn_desc(smem_u32(sP + buf * C::P_BYTES) + kk * 32, 16, 1024);
            // V: rows of keys (K), 64 values of N per 128-byte row; 8-key groups 1024 B apart, the second
            // 64-wide N tile (hd 128) one V tile further
            const uint64_t b = attn_desc(smem_u32(vt) + kk * 16 * 128, C::KV_TILE, 1024);
            umma_f16(tmem + 2 * BN + buf * HD, a, b, idesc_o, kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&o_full[buf]));
          umma_commit(smem_u32(&empty[s]));
        }
        __syncwarp();
      }
    } else if (warp >= 4) {
      // ------------------------------------------------------ query rows (softmax)
      const int t = threadIdx.x - 128;  // query row == TMEM lane
      const int q4 = warp - 4;
      const int row = sh_rows[t];
      const float scale = rsqrtf((float)HD) * 1.4426950408889634f;
      int qpos = 0;
      // Q row t: rotated (mode 1: from the projection), scaled, fp16, K-major swizzled
      {
        float qv[HD];
        if (row >= 0) {
          qpos = p.rows.pos[row];
          if (p.mode == 0) {
            const float* src = p.q + (int64_t)row * d + h * HD;
#pragma unroll
            for (int e = 0; e < HD; ++e) qv[e] = src[e] * scale;
          } else {
            const float* src = p.q + (int64_t)row * 3 * d + h * HD;
            const float2* cs = p.rope + (int64_t)qpos * (HD / 2);
#pragma unroll
            for (int i = 0; i < HD / 2; ++i) {
              const float2 c = cs[i];
              const float x0 = src[i], x1 = src[i + HD / 2];
              qv[i] = (x0 * c.x - x1 * c.y) * scale;
              qv[i + HD / 2] = (x1 * c.x + x0 * c.y) * scale;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < HD; ++e) qv[e] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < HD / 8; ++c) {
          __half2 hv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) hv[e] = __floats2half2_rn(qv[8 * c + 2 * e], qv[8 * c + 2 * e + 1]);
          uint8_t* dst = sQ + (c / 8) * (BM * 128) + t * 128 + (((c % 8) ^ (t & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(hv);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(q_full));
      const bool causal = p.mode == 0;
      float m = -INFINITY, l = 0.f, O[HD];
#pragma unroll
      for (int e = 0; e < HD; ++e) O[e] = 0.f;
      const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
      bool ok = true;
      for (int j = 0; j < nkb; ++j) {
        const int buf = j & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&s_full[buf]), (j >> 1) & 1, abort_flag))) { ok = false; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // two passes over the row's 64 scores (read twice from TMEM): the block maximum, then P
        const int vis = row < 0 ? 0 : min(kend, causal ? qpos + 1 : kend) - j * BN;  // visible keys of the block
        float mb = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float sv[32];
          tmem_ld32_att(tl + buf * BN + 32 * hh, sv);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * hh + i < vis) mb = fmaxf(mb, sv[i]);
        }
        const float mn = fmaxf(m, mb);
        const float corr = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        float rs = 0.f;
        uint8_t* prow = sP + buf * C::P_BYTES + t * 128;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float sv[32];
          tmem_ld32_att(tl + buf * BN + 32 * hh, sv);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            __half2 hv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = 8 * c + 2 * e;
              const float p0 = (32 * hh + i0 < vis) ? exp2f(sv[i0] - mn) : 0.f;
              const float p1 = (32 * hh + i0 + 1 < vis) ? exp2f(sv[i0 + 1] - mn) : 0.f;
              rs += p0 + p1;
              hv[e] = __floats2half2_rn(p0, p1);
            }
            const int cc = 4 * hh + c;
            *reinterpret_cast<uint4*>(prow + ((cc ^ (t & 7)) << 4)) = *reinterpret_cast<const uint4*>(hv);
          }
        }
        if (j == nkb - 1 && kend < (j + 1) * BN) {
          // keys past the end were never written: clear their V rows (p = 0 there, but 0 * NaN is not 0)
          const int first = kend - j * BN;
          uint8_t* vt = sKV + (j % STAGES) * C::STAGE + CT * C::KV_TILE;
          for (int i = t; i < (BN - first) * CT * 8; i += BM) {
            const int rr = first + i / (CT * 8), cc = i % (CT * 8);
            *reinterpret_cast<uint4*>(vt + (cc / 8) * C::KV_TILE + rr * 128 + ((cc % 8) << 4)) = make_uint4(0, 0, 0, 0);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[buf]));
        l = l * corr + rs;
        m = mn;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&o_full[buf]), (j >> 1) & 1, abort_flag))) { ok = false; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          float ov[32];
          tmem_ld32_att(tl + 2 * BN + buf * HD + c0, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) O[c0 + i] = O[c0 + i] * corr + ov[i];
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&o_free[buf]));
      }
      if (ok && row >= 0) {
        if (p.mode == 0) {
          const float inv = 1.f / l;
          float* od = p.o + (int64_t)row * d + h * HD;
#pragma unroll
          for (int e = 0; e < HD; e += 8) {
            float ov[8];
#pragma unroll
            for (int f = 0; f < 8; ++f) ov[f] = O[e + f] * inv;
            *reinterpret_cast<float4*>(od + e) = make_float4(ov[0], ov[1], ov[2], ov[3]);
            *reinterpret_cast<float4*>(od + e + 4) = make_float4(ov[4], ov[5], ov[6], ov[7]);
            act16_put8(p.o16, row, d, h * HD + e, ov, p.split16);
          }
        } else {
          float* dst = p.casc + ((int64_t)row * H + h) * (HD + 2);
          dst[0] = m;
          dst[1] = l;
#pragma unroll
          for (int e = 0; e < HD; ++e) dst[2 + e] = O[e];
        }
      }
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

}  // namespace tl
