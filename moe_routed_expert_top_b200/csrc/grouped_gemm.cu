// grouped_gemm.cu - persistent grouped GEMM C = A @ B[e]^T for sm_100a.
//
// What it computes: for every expert e, the rows of A that belong to e (a
// contiguous range in expert order) times expert e's weight matrix B[e]
// (TileOPs PR #1580 "Grouped-GEMM TMA OOB zero-fill + unpermute out=",
// Grouped-GEMM kernel). The work split follows the dispatch tables of the
// TileLang tutorial "Example 07: MoE dispatch contract and quantised GEMM"
// section 1: M-block bx belongs to expert group_idx_for_bx[bx] and starts at
// row m_start = bx*128 - group_padded_offsets[g] + group_offsets[g]; experts
// with no rows own no M-block and are never scheduled (pypto-lib PR #809,
// empty routed experts skip all compute).
//
// How (B200-first, not the pages' SM90 design):
//   * one persistent CTA per SM walks the tile list tile = (expert, n-block,
//     m-block) with m-blocks of one expert and one n-block adjacent, so CTAs
//     running at the same time share weight tiles through L2;
//   * warp 0 issues TMA loads (128-byte swizzle) into a STAGES-deep shared
//     memory ring; the A descriptor spans all rows, so the ragged tail past the
//     last row is zero-filled by the hardware and rows of the next expert that
//     fall inside a 128-row box are computed and then masked at the store;
//   * warp 1 allocates tensor memory and issues tcgen05.mma (M=128, N=BN,
//     fp32 accumulators in TMEM), double-buffered so the epilogue of one tile
//     overlaps the main loop of the next;
//   * warps 2-5 (one thread per accumulator row) read TMEM with tcgen05.ld and
//     run the epilogue: a bf16 store, SiLU(gate)*up (gate and up columns of the
//     same output column sit in one accumulator, BN/2 apart), or SiLU(gate)*up
//     quantised to E4M3 with one fp32 scale per 1x128 tile (XTuner PR #2089,
//     fused SwiGLU + per-tile quantisation);
//   * FP8 mode: E4M3 x E4M3 MMAs accumulate each 128-wide K-block in its own
//     TMEM buffer (4 in flight); the epilogue applies that block's activation
//     and weight scales and sums the blocks in fp32 registers.
// Every wait is bounded: on timeout the kernel flags MOE_DEV_TIMEOUT, drains
// its in-flight TMA copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

struct GemmParams {
  int M_dense;  // rows in dense mode
  int N;        // rows of B per expert
  int K;
  int E;
  const int32_t* group_sizes;  // grouped mode; null in dense mode
  const int32_t* group_offsets;
  const int32_t* group_padded;
  const int32_t* idx_for_bx;
  int M_blk;
  int rows_total;  // rows of A and C: no tile reads or writes past it
  void* C;
  int ldc;  // output row length in elements
  int out_f32;  // store epilogues: 1 = fp32 C, 0 = bf16 C
  float* C_scales;
  int ld_cscales;
  float* debug_h;
  const float* A_scales;
  const float* B_scales;
  int32_t* status;
};

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int kMode, int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr bool kFp8In = (kMode == kModeFp8Store);
  static constexpr bool kSwiglu = (kMode == kModeSwiglu || kMode == kModeSwigluFp8);
  static constexpr int BK = kFp8In ? 128 : 64;  // elements in one 128-byte smem row
  static constexpr int UMMA_K = kFp8In ? 32 : 16;
  static constexpr int K_STEPS = BK / UMMA_K;   // MMAs per stage
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = cmin(8, (196 * 1024) / STAGE_BYTES);
  static constexpr int NUM_ACC = kFp8In ? 4 : 2;
  static constexpr int TMEM_COLS = pow2_at_least(NUM_ACC * BN);
  static constexpr int OUT_COLS = kSwiglu ? BN / 2 : BN;  // output columns per tile
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NUM_ACC + 1;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
  static constexpr uint32_t IDESC = kFp8In ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, BN);
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128");
  static_assert(TMEM_COLS <= 512, "tensor memory");
  static_assert(!kFp8In || BN == 128, "FP8 mode uses 128-column tiles (one weight scale block)");
  static_assert(kMode != kModeSwigluFp8 || BN == 256, "1x128 quant tiles need 128 h columns");
};

struct TileInfo {
  int e;
  int nb;
  int m_start;
  int rows;
};

// Decode persistent tile index t. Identical in all three roles, so they agree
// on every tile (and on skipping a tile whose tables are inconsistent).
__device__ __forceinline__ bool decode_tile(const GemmParams& p, int NB, int t, TileInfo& ti) {
  if (p.group_padded == nullptr) {
    const int mblocks = (p.M_dense + 127) / 128;
    const int nb = t / mblocks;
    const int mb = t - nb * mblocks;
    ti.e = 0;
    ti.nb = nb;
    ti.m_start = mb * 128;
    ti.rows = cmin(128, p.M_dense - mb * 128);
    return true;
  }
  const int bx = t / NB;
  if (bx >= p.M_blk) return false;
  const int e = __ldg(p.idx_for_bx + bx);
  if (e < 0 || e >= p.E) return false;
  const int b0 = __ldg(p.group_padded + e) >> 7;
  const int mblocks = (__ldg(p.group_padded + e + 1) >> 7) - b0;
  const int local = t - b0 * NB;
  if (mblocks <= 0 || local < 0 || local >= mblocks * NB) return false;
  const int nb = local / mblocks;
  const int mb = local - nb * mblocks;
  ti.e = e;
  ti.nb = nb;
  ti.m_start = __ldg(p.group_offsets + e) + mb * 128;
  ti.rows = cmin(128, __ldg(p.group_sizes + e) - mb * 128);
  if (ti.m_start < 0 || ti.m_start + ti.rows > p.rows_total) {
    // tables inconsistent with the row count: skip the tile in every role
    if (threadIdx.x == 0) atomicOr(p.status, MOE_DEV_BAD_TABLES_FLAG);
    return false;
  }
  return ti.rows > 0;
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

template <int kMode, int BN>
__global__ void __launch_bounds__(192, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  using Cfg = GemmCfg<kMode, BN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int NUM_ACC = Cfg::NUM_ACC;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * STAGES;
  const uint32_t tfull0 = empty0 + 8 * STAGES;
  const uint32_t tempty0 = tfull0 + 8 * NUM_ACC;
  const uint32_t drain_bar = tempty0 + 8 * NUM_ACC;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 4);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int NB = (Cfg::kSwiglu ? (p.N / 2) : p.N) / Cfg::OUT_COLS;
  int total_tiles;
  if (p.group_padded == nullptr) {
    total_tiles = ((p.M_dense + 127) / 128) * NB;
  } else {
    total_tiles = (__ldg(p.group_padded + p.E) >> 7) * NB;
  }
  const int KB = p.K / Cfg::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      const uint64_t pol_w = l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        TileInfo ti;
        if (!decode_tile(p, NB, t, ti)) continue;
        const int half_n = p.N / 2;
        const int brow = ti.e * p.N + ti.nb * (Cfg::kSwiglu ? BN / 2 : BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
          const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_BYTES);
          tma_load_2d(a_dst, &tmA, kb * Cfg::BK, ti.m_start, fb, pol_act);
          if constexpr (Cfg::kSwiglu) {
            tma_load_2d(b_dst, &tmB, kb * Cfg::BK, brow, fb, pol_w);
            tma_load_2d(b_dst + (BN / 2) * 128, &tmB, kb * Cfg::BK, brow + half_n, fb, pol_w);
          } else {
            tma_load_2d(b_dst, &tmB, kb * Cfg::BK, brow, fb, pol_w);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain: every issued copy lands before shared memory goes away
        const uint32_t n = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
        int s = stage;
        uint32_t ph = phase;
        for (uint32_t i = 0; i < n; ++i) {
          if (--s < 0) {
            s = STAGES - 1;
            ph ^= 1u;
          }
          mbar_wait_drain(full0 + 8 * s, ph);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        TileInfo ti;
        if (!decode_tile(p, NB, t, ti)) continue;
        if constexpr (!Cfg::kFp8In) {
          if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
            const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
            for (int k = 0; k < Cfg::K_STEPS; ++k) {
              // +32 bytes along K inside the 128-byte swizzled row = +2 in the address field
              mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, Cfg::IDESC, (kb | k) != 0 ? 1u : 0u);
            }
            mma_commit(empty0 + 8 * stage);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(tfull0 + 8 * acc);
          if (++acc == NUM_ACC) {
            acc = 0;
            acc_phase ^= 1u;
          }
        } else {
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.status) ||
                !mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
            const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
            const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
            for (int k = 0; k < Cfg::K_STEPS; ++k) {
              mma_fp8(d, adesc + 2 * k, bdesc + 2 * k, Cfg::IDESC, k != 0 ? 1u : 0u);
            }
            mma_commit(empty0 + 8 * stage);
            mma_commit(tfull0 + 8 * acc);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            if (++acc == NUM_ACC) {
              acc = 0;
              acc_phase ^= 1u;
            }
          }
        }
      }
      // all MMAs this thread issued complete before tensor memory is freed
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      TileInfo ti;
      if (!decode_tile(p, NB, t, ti)) continue;
      const bool valid = r < ti.rows;
      const int64_t row = static_cast<int64_t>(ti.m_start) + r;
      if constexpr (!Cfg::kFp8In) {
        if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t tb = lane_base + static_cast<uint32_t>(acc * BN);
        if constexpr (kMode == kModeStore) {
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (p.out_f32) {
              if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.C) + row * p.ldc +
                                                      ti.nb * BN + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
              }
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) +
                                                      row * p.ldc + ti.nb * BN + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
              }
            }
          }
        } else if constexpr (kMode == kModeSwiglu) {
          constexpr int HN = BN / 2;
          __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C);
          uint32_t g[32], u[32], gn[32], un[32];
          tmem_ld32(tb, g);
          tmem_ld32(tb + HN, u);
          tmem_ld_wait();
#pragma unroll 1
          for (int c = 0; c < HN / 32; ++c) {
            // the next chunk's TMEM loads run while this chunk is computed and stored
            const bool more = c + 1 < HN / 32;
            if (more) {
              tmem_ld32(tb + (c + 1) * 32, gn);
              tmem_ld32(tb + HN + (c + 1) * 32, un);
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 =
                  silu_f32(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(C + row * p.ldc + ti.nb * HN + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
            if (more) {
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                g[i] = gn[i];
                u[i] = un[i];
              }
            }
          }
        } else {  // kModeSwigluFp8: 128 h columns = one 1x128 quantisation tile
          constexpr int HN = BN / 2;
          float h[HN];
          float amax = 0.0f;
#pragma unroll
          for (int c = 0; c < HN / 32; ++c) {
            uint32_t g[32], u[32];
            tmem_ld32(tb + c * 32, g);
            tmem_ld32(tb + HN + c * 32, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float hv = silu_f32(__uint_as_float(g[i])) * __uint_as_float(u[i]);
              h[c * 32 + i] = hv;
              amax = fmaxf(amax, fabsf(hv));
            }
          }
          if (valid) {
            const float s = amax / 448.0f;
            uint8_t* Cq = static_cast<uint8_t*>(p.C) + row * p.ldc + ti.nb * HN;
#pragma unroll
            for (int c = 0; c < HN / 16; ++c) {
              uint32_t w4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t lo, hi;
                if (amax > 0.0f) {
                  lo = cvt_e4m3x2(h[c * 16 + 4 * i] / s, h[c * 16 + 4 * i + 1] / s);
                  hi = cvt_e4m3x2(h[c * 16 + 4 * i + 2] / s, h[c * 16 + 4 * i + 3] / s);
                } else {
                  lo = hi = 0u;
                }
                w4[i] = lo | (hi << 16);
              }
              reinterpret_cast<uint4*>(Cq)[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            p.C_scales[row * p.ld_cscales + ti.nb] = amax > 0.0f ? s : 0.0f;
            if (p.debug_h != nullptr) {
              float4* dh = reinterpret_cast<float4*>(p.debug_h + row * p.ldc + ti.nb * HN);
#pragma unroll
              for (int i = 0; i < HN / 4; ++i)
                dh[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
        if (++acc == NUM_ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      } else {
        // FP8 block-scaled: sum over K-blocks of sa[row,kb] * sw[e,nb,kb] * (A_kb B_kb^T)
        const int KBS = p.K / 128;
        const float* sa = p.A_scales + (valid ? row : 0) * KBS;
        const float* sw = p.B_scales + (static_cast<int64_t>(ti.e) * (p.N / 128) + ti.nb) * KBS;
        float accv[BN];
#pragma unroll
        for (int i = 0; i < BN; ++i) accv[i] = 0.0f;
        float sa_next = valid ? __ldg(sa) : 0.0f;
        float sw_next = __ldg(sw);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          const float scale = sa_next * sw_next;
          if (kb + 1 < KB) {
            sa_next = valid ? __ldg(sa + kb + 1) : 0.0f;
            sw_next = __ldg(sw + kb + 1);
          }
          if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tb = lane_base + static_cast<uint32_t>(acc * BN);
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              accv[c * 32 + i] = fmaf(scale, __uint_as_float(v[i]), accv[c * 32 + i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
          if (++acc == NUM_ACC) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
        if (!ok) break;
        if (valid) {
          if (p.out_f32) {
            float4* dst =
                reinterpret_cast<float4*>(static_cast<float*>(p.C) + row * p.ldc + ti.nb * BN);
#pragma unroll
            for (int i = 0; i < BN / 4; ++i)
              dst[i] = make_float4(accv[4 * i], accv[4 * i + 1], accv[4 * i + 2], accv[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + row * p.ldc +
                                                  ti.nb * BN);
#pragma unroll
            for (int i = 0; i < BN / 8; ++i)
              dst[i] = make_uint4(pack_bf16x2(accv[8 * i], accv[8 * i + 1]),
                                  pack_bf16x2(accv[8 * i + 2], accv[8 * i + 3]),
                                  pack_bf16x2(accv[8 * i + 4], accv[8 * i + 5]),
                                  pack_bf16x2(accv[8 * i + 6], accv[8 * i + 7]));
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D K-major tensor [rows, K] with a box of box_rows x (128 bytes), 128-byte swizzle,
// zero fill out of bounds.
static bool encode_2d(CUtensorMap* map, const void* base, bool fp8, uint64_t K, uint64_t rows,
                      uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  const uint32_t elt = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * elt};
  cuuint32_t box[2] = {128 / elt, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

template <int kMode, int BN>
static cudaError_t run_gemm(const GemmLaunch& L, cudaStream_t stream) {
  using Cfg = GemmCfg<kMode, BN>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kMode, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const bool grouped = L.group_padded != nullptr;
  const int E = grouped ? L.E : 1;
  CUtensorMap tmA, tmB;
  const uint32_t b_box_rows = Cfg::kSwiglu ? BN / 2 : BN;
  if (!encode_2d(&tmA, L.A, Cfg::kFp8In, L.K, L.rows, 128) ||
      !encode_2d(&tmB, L.B, Cfg::kFp8In, L.K, static_cast<uint64_t>(E) * L.N, b_box_rows))
    return cudaErrorInvalidValue;

  GemmParams p{};
  p.M_dense = grouped ? 0 : L.rows;
  p.N = L.N;
  p.K = L.K;
  p.E = E;
  p.group_sizes = L.group_sizes;
  p.group_offsets = L.group_offsets;
  p.group_padded = L.group_padded;
  p.idx_for_bx = L.idx_for_bx;
  p.M_blk = L.M_blk;
  p.rows_total = L.rows;
  p.C = L.C;
  const int out_n = Cfg::kSwiglu ? L.N / 2 : L.N;
  p.ldc = out_n;
  p.out_f32 = L.out_f32;
  p.C_scales = L.C_scales;
  p.ld_cscales = out_n / 128;
  p.debug_h = L.debug_h;
  p.A_scales = L.A_scales;
  p.B_scales = L.B_scales;
  p.status = L.status;

  const int NB = out_n / Cfg::OUT_COLS;
  const long long mblocks_ub = grouped ? static_cast<long long>(L.M_blk) : (L.rows + 127) / 128;
  const long long tiles_ub = mblocks_ub * NB;
  int sms = device_sm_count();
  if (L.max_ctas > 0 && L.max_ctas < sms) sms = L.max_ctas;
  const int grid = static_cast<int>(tiles_ub < sms ? (tiles_ub > 0 ? tiles_ub : 1) : sms);
  grouped_gemm_kernel<kMode, BN><<<grid, 192, Cfg::SMEM_BYTES, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(const GemmLaunch& L, cudaStream_t stream) {
  // B as a strided view (a tensor-parallel shard) is read by the pair tiling only
  const bool b_view = L.ldb != 0 || L.up_off != 0 || L.b_rows != 0;
  if (L.gather || b_view || L.tiling == kTilingWeightsPair ||
      (L.tiling == kTilingAuto && grouped_gemm_pair_preferred(L)))
    return grouped_gemm_pair_supported(L) ? launch_grouped_gemm_pair(L, stream)
                                          : cudaErrorNotSupported;
  if (grouped_gemm_t_supported(L) &&
      (L.tiling == kTilingWeights || (L.tiling == kTilingAuto && grouped_gemm_t_preferred(L))))
    return launch_grouped_gemm_t(L, stream);
  if (L.tiling == kTilingWeights) return cudaErrorNotSupported;
  // the weighted (pair-order) store and the f16e format are built into the
  // weight-row tilings only
  if (L.weighted || L.out_f16e) return cudaErrorNotSupported;
  switch (L.mode) {
    case kModeStore:
      if (L.N % 256 == 0) return run_gemm<kModeStore, 256>(L, stream);
      if (L.N % 128 == 0) return run_gemm<kModeStore, 128>(L, stream);
      return run_gemm<kModeStore, 64>(L, stream);
    case kModeSwiglu: {
      // Small expert groups (decode): every tile streams its full weight slab,
      // so 64-column h tiles halve the tile cost and cut the idle tail of the
      // last wave of the persistent grid.
      const bool small_groups = L.group_padded != nullptr && L.rows < 64 * L.E;
      if ((L.N / 2) % 128 == 0 && !small_groups) return run_gemm<kModeSwiglu, 256>(L, stream);
      return run_gemm<kModeSwiglu, 128>(L, stream);
    }
    case kModeSwigluFp8:
      return run_gemm<kModeSwigluFp8, 256>(L, stream);
    case kModeFp8Store:
      return run_gemm<kModeFp8Store, 128>(L, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace moe

namespace moe {

bool grouped_gemm_f16e_supported(const GemmLaunch& L) {
  if (!L.out_f16e) return false;
  // the dispatch of launch_grouped_gemm, for a launch that stores f16e
  const bool b_view = L.ldb != 0 || L.up_off != 0 || L.b_rows != 0;
  if (L.gather || b_view || L.tiling == kTilingWeightsPair ||
      (L.tiling == kTilingAuto && grouped_gemm_pair_preferred(L)))
    return grouped_gemm_pair_supported(L);
  return grouped_gemm_t_supported(L) &&
         (L.tiling == kTilingWeights || (L.tiling == kTilingAuto && grouped_gemm_t_preferred(L)));
}

}  // namespace moe
