// grouped_gemm_t.cu - the grouped GEMM with weights on the MMA's M side
// ("transposed" tiles): D^T[w, t] = sum_k W[e][w, k] * X[t, k].
//
// Same operation as grouped_gemm.cu (TileOPs PR #1580 "Grouped-GEMM TMA OOB
// zero-fill + unpermute out=", Grouped-GEMM kernel: C[e] = A[e] @ B[e]^T over
// each expert's rows), tiled the other way round: a tile is 128 weight rows x
// up to TN token rows of one expert. The MMA's N is the tile's token count
// rounded up to 16, so the tensor work follows the real group sizes instead of
// padding every expert to 128-row blocks, and a small group (decode) loads
// only as many token rows as it has (TMA boxes of 32/64/128/256 rows).
//
// Tiles are ordered (expert, weight block, token chunk), token chunks
// innermost, so the chunks that share a weight block run at the same time and
// read it once from HBM. Empty experts own no tile (pypto-lib PR #809).
//
// Modes:
//   store  : C [rows, N] (fp32 or bf16) = X @ W[e]^T; weight block = 128 rows.
//   swiglu : h bf16 [rows, F] = SiLU(G[:, :F]) * G[:, F:], G = X @ W[e]^T with
//            W[e] = [gate rows; up rows] (TileOPs PR #778, Design); a weight
//            block stacks 64 gate rows over the matching 64 up rows, so one
//            M=128 MMA produces both and the epilogue pairs lane r with lane
//            r + 64 through shared memory (XTuner PR #2089, SiLU(gate)*up).
// Warp roles and the bounded-wait/teardown protocol are those of
// grouped_gemm.cu: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer,
// warps 2-5 epilogue (TMEM lane = weight row), two TMEM accumulators. The FP8
// mode adds a scale warp (6), a second MMA issuer (7) and a second epilogue
// group (8-11), 384 threads.
// The epilogue stages 32 token rows at a time in shared memory and writes
// them row-major with 16-byte stores, masking rows past the tile's tokens.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "f16e.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

enum TMode { kTStore = 0, kTSwiglu = 1, kTFp8Store = 2 };

constexpr int kXBoxes = 4;  // token-tile TMA boxes of 32, 64, 128, 256 rows

struct TParams {
  int M_dense;  // rows in dense mode (group tables null)
  int N;        // rows of W per expert
  int K;
  int E;
  const int32_t* group_sizes;
  const int32_t* group_offsets;
  int rows_total;
  void* C;
  int ldc;      // output row length in elements
  int out_f32;  // store modes: fp32 C
  int out_f16e;     // store modes: C fp16 + C_exps int8 [rows, ldc / 128] (f16e.cuh)
  int8_t* C_exps;
  const float* A_scales;  // FP8: activation scales [rows, KBS]
  const float* B_scales;  // FP8: weight block scales [E, N/128, KBS]
  int KBS;                // FP8: K / 128
  int32_t* status;
  // weighted store: C row pair_of_row[r] = row_scale * row_w[pair] * result row r
  int weighted;
  const int32_t* pair_of_row;
  const float* row_w;
  float row_scale;
};

__host__ __device__ constexpr int tmin(int a, int b) { return a < b ? a : b; }

template <int kMode, int TN>
struct TCfg {
  static constexpr bool kFp8 = kMode == kTFp8Store;
  static constexpr int BK = kFp8 ? 128 : 64;  // elements per 128-byte smem row
  static constexpr int K_STEPS = 4;           // MMAs (K = 16 bf16 / 32 e4m3) per stage
  static constexpr int A_BYTES = 128 * 128;     // weight tile: 128 rows x 128 B
  static constexpr int B_BYTES = TN * 128;      // token tile: up to TN rows x 128 B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = tmin(8, ((kFp8 ? 192 : 200) * 1024) / STAGE_BYTES);
  // FP8: one TMEM buffer per 128-wide K-block, as many in flight as 512 columns
  // hold (the MMA -> epilogue -> release round trip per K-block is latency
  // bound); bf16: 2 tile buffers
  static constexpr int NUM_ACC = kFp8 ? 512 / TN : 2;
  static constexpr int TMEM_COLS = NUM_ACC * TN;
  // 32 token rows x 128 fp32, then the tile's row destinations and factors
  // (weighted store)
  static constexpr int STAGE_OUT_BYTES = 32 * 128 * 4 + 2 * TN * 4;
  // FP8: a scale warp (warp 6) prepares each tile's sa * sw products one tile
  // ahead in a ring of two slots of TN x MAX_KBS fp32, a second MMA issuer
  // (warp 7) takes every other K-block, and a second epilogue group (warps
  // 8-11) takes the tile's token columns 32..63
  static constexpr int kThreads = kFp8 ? 384 : 192;
  static constexpr int MAX_KBS = 16;                    // FP8: K <= 2048
  static constexpr int SA_SLOT = TN * MAX_KBS;          // floats per slot
  static constexpr int SA_BYTES = kFp8 ? 2 * SA_SLOT * 4 : 0;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NUM_ACC + 1 + (kFp8 ? 4 : 0);
  static constexpr int MAX_E = 1024;
  // ... + barriers + TMEM slot and flags + cpre[E + 1] + soff[E + 1]
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGE_OUT_BYTES + SA_BYTES +
                                    NUM_BARS * 8 + 16 + 2 * (MAX_E + 8) * 4;
  static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "tensor memory");
  static_assert(!kFp8 || TN <= 64, "FP8 keeps TN columns per K-block buffer, 4 buffers");
  static constexpr int WROWS = (kMode == kTSwiglu) ? 64 : 128;  // output columns per tile
  static_assert(TN % 32 == 0 && TN >= 32 && TN <= 256, "token tile");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct TTile {
  int e, wb, m0, nt;
  int chunks;  // token tiles of this expert (tiles that read the same weights)
};

// Tile t -> (expert, weight block, token chunk). cpre[e] = token chunks of the
// experts before e and soff[e] = group_offsets[e] (both in shared memory, built
// at kernel start); WB weight blocks. A CTA visits its tiles in increasing
// order, so each warp keeps the expert of its last tile in `ecur` and only
// moves it forward: no search and no global load per tile.
__device__ __forceinline__ bool t_decode(const TParams& p, const int* cpre, const int* soff,
                                         int WB, int TN, int t, int& ecur, TTile& ti) {
  while (WB * cpre[ecur + 1] <= t) ++ecur;  // experts without chunks are passed over
  const int e = ecur;
  const int chunks = cpre[e + 1] - cpre[e];
  const int local = t - WB * cpre[e];
  const int wb = local / chunks;
  const int c = local - wb * chunks;
  const int off = soff[e];
  const int size = soff[e + 1] - off;
  ti.e = e;
  ti.wb = wb;
  ti.chunks = chunks;
  ti.m0 = off + c * TN;
  ti.nt = tmin(TN, size - c * TN);
  if (ti.nt <= 0 || ti.m0 < 0 || ti.m0 + ti.nt > p.rows_total) {
    if (threadIdx.x == 0 && ti.nt > 0) atomicOr(p.status, MOE_DEV_BAD_TABLES_FLAG);
    return false;
  }
  return true;
}

__device__ __forceinline__ int xbox_for(int n) {  // smallest box (32/64/128/256) holding n rows
  return n <= 32 ? 0 : n <= 64 ? 1 : n <= 128 ? 2 : 3;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// FP8: the second epilogue group's barrier, and both groups' (256 threads)
__device__ __forceinline__ void epi_bar_g1() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void epi_bar_all() { asm volatile("bar.sync 3, 256;" ::: "memory"); }

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Weighted store: the destination row (flat pair index, -1 = none) and the
// factor row_scale * row_w[pair] of a tile's rows row0 .. row0 + rows - 1,
// loaded by the 128 epilogue threads when the tile starts, so the loads' latency
// passes while the tile's MMAs run; read after the barrier that precedes the
// first store.
__device__ __forceinline__ void stage_row_info(const TParams& p, int et, int rows, int row0,
                                               int* sDst, float* sFac) {
  for (int i = et; i < rows; i += 128) {
    const int pr = __ldg(p.pair_of_row + row0 + i);
    sDst[i] = pr;
    sFac[i] = pr >= 0 ? p.row_scale * __ldg(p.row_w + pr) : 0.0f;
  }
}

// Write `rows` staged token rows (sOut[i][0..128), fp32) to C rows row0.. at
// column col0, fp32, bf16 or f16e, 16-byte stores; 128 epilogue threads (et). A
// weighted store writes row i to sDst[i], scaled by sFac[i].
__device__ __forceinline__ void store_rows(const TParams& p, const float* sOut, int et, int rows,
                                           int row0, int col0, const int* sDst,
                                           const float* sFac) {
  if (p.out_f16e) {
    // a row's 128 columns (one f16e block) over 16 lanes of a half warp; every
    // lane encodes, whether or not its row is stored
    const int c8 = et & 15;
    float v[4][8];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const float4* src = reinterpret_cast<const float4*>(sOut + (pass * 8 + (et >> 4)) * 128 + c8 * 8);
      const float4 a = src[0], b = src[1];
      v[pass][0] = a.x; v[pass][1] = a.y; v[pass][2] = a.z; v[pass][3] = a.w;
      v[pass][4] = b.x; v[pass][5] = b.y; v[pass][6] = b.z; v[pass][7] = b.w;
    }
    uint4 pk[4];
    int e[4];
    f16e_encode8xn<4>(v, pk, e);
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int i = pass * 8 + (et >> 4);
      if (i < rows) {
        const int64_t row = row0 + i;
        __half* dst = static_cast<__half*>(p.C) + row * p.ldc + col0;
        reinterpret_cast<uint4*>(dst)[c8] = pk[pass];
        if (c8 == 0) p.C_exps[row * (p.ldc / 128) + col0 / 128] = static_cast<int8_t>(e[pass]);
      }
    }
    return;
  }
  if (p.out_f32) {
#pragma unroll
    for (int pass = 0; pass < 8; ++pass) {
      const int i = pass * 4 + (et >> 5);
      const int c4 = et & 31;
      if (i < rows) {
        float4 val = reinterpret_cast<const float4*>(sOut + i * 128)[c4];
        int drow = row0 + i;
        if (p.weighted) {
          drow = sDst[i];
          const float f = sFac[i];
          if (drow < 0) continue;
          val = make_float4(val.x * f, val.y * f, val.z * f, val.w * f);
        }
        float* dst = static_cast<float*>(p.C) + static_cast<int64_t>(drow) * p.ldc + col0;
        reinterpret_cast<float4*>(dst)[c4] = val;
      }
    }
  } else {
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int i = pass * 8 + (et >> 4);
      const int c8 = et & 15;
      if (i < rows) {
        const float* src = sOut + i * 128 + c8 * 8;
        int drow = row0 + i;
        float f = 1.0f;
        if (p.weighted) {
          drow = sDst[i];
          f = sFac[i];
          if (drow < 0) continue;
        }
        const uint4 val =
            p.weighted ? make_uint4(pack_bf16x2(src[0] * f, src[1] * f),
                                    pack_bf16x2(src[2] * f, src[3] * f),
                                    pack_bf16x2(src[4] * f, src[5] * f),
                                    pack_bf16x2(src[6] * f, src[7] * f))
                       : make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                                    pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
        __nv_bfloat16* dst =
            static_cast<__nv_bfloat16*>(p.C) + static_cast<int64_t>(drow) * p.ldc + col0;
        reinterpret_cast<uint4*>(dst)[c8] = val;
      }
    }
  }
}

template <int kMode, int TN>
__global__ void __launch_bounds__(TCfg<kMode, TN>::kThreads, 1)
    grouped_gemm_t_kernel(const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmX0,
                          const __grid_constant__ CUtensorMap tmX1,
                          const __grid_constant__ CUtensorMap tmX2,
                          const __grid_constant__ CUtensorMap tmX3, const TParams p) {
  using Cfg = TCfg<kMode, TN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int NUM_ACC = Cfg::NUM_ACC;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                                   // weight tiles
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;           // token tiles
  float* sOut = reinterpret_cast<float*>(sB + STAGES * Cfg::B_BYTES);  // [32][128]
  int* sDst = reinterpret_cast<int*>(sOut + 32 * 128);  // weighted store: the tile's row info
  float* sFac = reinterpret_cast<float*>(sDst + TN);
  // FP8: sa * sw of a tile's tokens, K-block major [KBS][TN], two slots
  float* sSa = sOut + 32 * 128 + 2 * TN;
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sOut) +
                                               Cfg::STAGE_OUT_BYTES + Cfg::SA_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // set only by epilogue threads, read only after their shared barrier: the four
  // epilogue warps always agree on whether to stop
  volatile int* epi_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* cpre = reinterpret_cast<int*>(tmem_slot + 4);  // [E + 1]
  int* soff = cpre + Cfg::MAX_E + 8;                    // [E + 1]: group_offsets

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * STAGES;
  const uint32_t tfull0 = empty0 + 8 * STAGES;
  const uint32_t tempty0 = tfull0 + 8 * NUM_ACC;
  const uint32_t drain_bar = tempty0 + 8 * NUM_ACC;
  const uint32_t scl_full0 = drain_bar + 8;      // FP8: slot filled by the scale warp
  const uint32_t scl_empty0 = scl_full0 + 16;    // FP8: slot released by the epilogue
  constexpr int kThreads = Cfg::kThreads;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = p.group_sizes ? p.E : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, Cfg::kFp8 ? 8 : 4);  // epilogue warps
    }
    mbar_init(drain_bar, Cfg::kFp8 ? 2 : 1);  // one commit per MMA issuer
    if constexpr (Cfg::kFp8) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(scl_full0 + 8 * i, 1);
        mbar_init(scl_empty0 + 8 * i, 1);
      }
    }
    *abort_flag = 0;
    *epi_abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX0);
    tma_prefetch_desc(&tmX1);
    tma_prefetch_desc(&tmX2);
    tma_prefetch_desc(&tmX3);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  // token chunks per expert -> exclusive prefix cpre[0..E] (all threads)
  {
    const int per = (E + kThreads - 1) / kThreads;
    const int beg = threadIdx.x * per;
    int local = 0;
    for (int i = 0; i < per && beg + i < E; ++i) {
      const int s = p.group_sizes ? __ldg(p.group_sizes + beg + i) : p.M_dense;
      local += (s + TN - 1) / TN;
    }
    int inc = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    int* wsum = reinterpret_cast<int*>(sOut);  // scratch before the epilogue uses it
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int run = before + inc - local;
    for (int i = 0; i < per && beg + i < E; ++i) {
      cpre[beg + i] = run;
      const int s = p.group_sizes ? __ldg(p.group_sizes + beg + i) : p.M_dense;
      run += (s + TN - 1) / TN;
    }
    if (threadIdx.x == kThreads - 1) cpre[E] = before + inc;
    for (int i = threadIdx.x; i <= E; i += kThreads)
      soff[i] = p.group_offsets ? __ldg(p.group_offsets + i) : (i == 0 ? 0 : p.M_dense);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int WB = (kMode == kTSwiglu) ? (p.N / 2) / 64 : p.N / 128;
  const int total_tiles = WB * cpre[E];
  const int KB = p.K / Cfg::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      const uint64_t pol_w1 = l2_policy_by_code(MOE_W_POLICY_SINGLE);
      const uint64_t pol_wn = l2_policy_by_code(MOE_W_POLICY_MULTI);
      const CUtensorMap* xmaps[kXBoxes] = {&tmX0, &tmX1, &tmX2, &tmX3};
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      int ecur = 0;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        TTile ti;
        if (!t_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
        const int nmma = (ti.nt + 15) & ~15;
        const int xb = xbox_for(nmma);
        const uint32_t bytes = Cfg::A_BYTES + (32u << xb) * 128u;
        const int wrow = ti.e * p.N + ti.wb * Cfg::WROWS;
        const uint64_t pol_w = ti.chunks > 1 ? pol_wn : pol_w1;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
          if constexpr (kMode == kTSwiglu) {
            tma_load_2d(a_dst, &tmW, kb * Cfg::BK, wrow, fb, pol_w);                  // gate
            tma_load_2d(a_dst + 64 * 128, &tmW, kb * Cfg::BK, wrow + p.N / 2, fb, pol_w);  // up
          } else {
            tma_load_2d(a_dst, &tmW, kb * Cfg::BK, wrow, fb, pol_w);
          }
          tma_load_2d(smem_u32(sB + stage * Cfg::B_BYTES), xmaps[xb], kb * Cfg::BK, ti.m0, fb,
                      pol_act);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
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
  } else if (warp == 1 || (Cfg::kFp8 && warp == 7)) {
    // ------------------------------------------------------------ MMA issuer(s)
    if (lane == 0) {
      // FP8: two issuers (warps 1 and 7) take the K-blocks of even and odd
      // running index; each K-block has its own TMEM buffer and commit, so
      // while one thread waits on the tensor pipe the other prepares the next
      const int issuer = warp == 1 ? 0 : 1;
      int nk = 0;  // running K-block index over the CTA's tiles
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int ecur = 0;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        TTile ti;
        if (!t_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
        const int nmma = (ti.nt + 15) & ~15;
        if constexpr (Cfg::kFp8) {
          // one TMEM buffer per 128-wide K-block: the epilogue scales and sums them
          const uint32_t idesc8 = idesc_e4m3_f32(128, nmma);
          for (int kb = 0; kb < KB; ++kb, ++nk) {
            if ((nk & 1) == issuer) {
              if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.status) ||
                  !mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d = tmem_base + static_cast<uint32_t>(acc * TN);
              const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
              const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
              for (int k = 0; k < Cfg::K_STEPS; ++k)
                mma_fp8(d, adesc + 2 * k, bdesc + 2 * k, idesc8, k != 0 ? 1u : 0u);
              // the stage is released as soon as these MMAs complete, not when
              // the epilogue gets to this K-block's buffer: the ring keeps its
              // depth while the epilogue lags
              mma_commit(empty0 + 8 * stage);
              mma_commit(tfull0 + 8 * acc);
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            if (++acc == NUM_ACC) {
              acc = 0;
              acc_phase ^= 1u;
            }
          }
          continue;
        }
        const uint32_t idesc = idesc_bf16_f32(128, nmma);
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * TN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * Cfg::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
          for (int k = 0; k < Cfg::K_STEPS; ++k)
            mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
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
      }
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ scale warp (FP8)
    // For each tile, one tile ahead of the epilogue: s[kb][t] = sw[e, wb, kb] *
    // sa[m0 + t, kb] into the next slot of the two-slot ring, K-block major so
    // the epilogue reads each K-block's column scales as 16-byte broadcasts. It
    // keeps the global loads' latency off the epilogue's path.
    if constexpr (Cfg::kFp8) {
      int ecur = 0;
      int slot = 0;
      uint32_t sphase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        TTile ti;
        if (!t_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
        uint32_t got = 1;
        if (lane == 0) got = mbar_wait(scl_empty0 + 8 * slot, sphase ^ 1u, abort_flag, p.status);
        if (!__shfl_sync(0xffffffffu, got, 0)) break;
        float* dst = sSa + slot * Cfg::SA_SLOT;
        const int nsa = ti.nt * p.KBS;
        const float* gsa = p.A_scales + static_cast<int64_t>(ti.m0) * p.KBS;
        const float* gsw =
            p.B_scales + (static_cast<int64_t>(ti.e) * (p.N / 128) + ti.wb) * p.KBS;
        // 8 independent loads in flight per lane per round (at most 4 rounds)
        for (int base = 0; base < nsa; base += 8 * 32) {
          float a[8], b[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = base + j * 32 + lane;
            const bool in = i < nsa;
            a[j] = in ? __ldg(gsa + i) : 0.0f;
            b[j] = in ? __ldg(gsw + (i % p.KBS)) : 0.0f;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = base + j * 32 + lane;
            if (i < nsa) {
              const int tok = i / p.KBS;
              const int kb = i - tok * p.KBS;
              dst[kb * TN + tok] = a[j] * b[j];
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(scl_full0 + 8 * slot);
        if (++slot == 2) {
          slot = 0;
          sphase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row of this thread's TMEM lane
    // FP8: two groups, warps 2-5 (token columns 0..31) and 8-11 (32..63)
    const int grp = (Cfg::kFp8 && warp >= 8) ? 1 : 0;
    const int et = threadIdx.x - (grp ? 256 : 64);  // 0..127 within the group
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int acc = 0;
    uint32_t acc_phase = 0;
    int sslot = 0;  // FP8: the scale ring's slot of the next tile, and its phase
    uint32_t sphase = 0;
    int ecur = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      TTile ti;
      if (!t_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
      if (kMode != kTSwiglu && p.weighted && grp == 0)
        stage_row_info(p, et, ti.nt, ti.m0, sDst, sFac);
      if constexpr (Cfg::kFp8) {
        // y[t, w] = sum_kb sw[e, wb, kb] * sa[t, kb] * (Wq_kb Xq_kb^T)[w, t], with
        // the tile's products sw * sa prepared by the scale warp in slot sslot;
        // group grp holds token columns 32*grp .. 32*grp+31
        const float* sS = sSa + sslot * Cfg::SA_SLOT;
        if (!mbar_wait(scl_full0 + 8 * sslot, sphase, abort_flag, p.status)) *epi_abort = 1;
        epi_bar_all();  // both groups arrive here whether their waits succeeded or not
        if (*epi_abort) break;
        const bool mine = grp * 32 < ti.nt;  // uniform across the group
        float accv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) accv[i] = 0.0f;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (mine) {
            const uint32_t tbk = lane_base + static_cast<uint32_t>(acc * TN + grp * 32);
            const float4* s4 = reinterpret_cast<const float4*>(sS + kb * TN + grp * 32);
            uint32_t v[32];
            tmem_ld32(tbk, v);
            tmem_ld_wait();
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
              const float4 sc = s4[i4];
              accv[i4 * 4 + 0] = fmaf(sc.x, __uint_as_float(v[i4 * 4 + 0]), accv[i4 * 4 + 0]);
              accv[i4 * 4 + 1] = fmaf(sc.y, __uint_as_float(v[i4 * 4 + 1]), accv[i4 * 4 + 1]);
              accv[i4 * 4 + 2] = fmaf(sc.z, __uint_as_float(v[i4 * 4 + 2]), accv[i4 * 4 + 2]);
              accv[i4 * 4 + 3] = fmaf(sc.w, __uint_as_float(v[i4 * 4 + 3]), accv[i4 * 4 + 3]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
          if (++acc == NUM_ACC) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
        if (!ok) *epi_abort = 1;
        epi_bar_all();
        if (*epi_abort) break;
        // every epilogue thread is done with the slot: the scale warp may refill it
        if (grp == 0 && et == 0) mbar_arrive(scl_empty0 + 8 * sslot);
        if (++sslot == 2) {
          sslot = 0;
          sphase ^= 1u;
        }
        // the groups store their 32 token rows in turn through sOut
        if (grp == 1) epi_bar_all();
        if (mine) {
#pragma unroll
          for (int i = 0; i < 32; ++i) sOut[i * 128 + r] = accv[i];
          if (grp == 0) epi_bar(); else epi_bar_g1();
          store_rows(p, sOut, et, tmin(32, ti.nt - grp * 32), ti.m0 + grp * 32, ti.wb * 128,
                     sDst + grp * 32, sFac + grp * 32);
        }
        if (grp == 0) epi_bar_all();
        epi_bar_all();  // sOut and the row info are rewritten for the next tile
        continue;
      }
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status)) *epi_abort = 1;
      epi_bar();  // every epilogue warp arrives here whether its wait succeeded or not
      if (*epi_abort) break;
      tc_fence_after();
      const uint32_t tb = lane_base + static_cast<uint32_t>(acc * TN);
      uint32_t v[32], vn[32];
      tmem_ld32(tb, v);
      tmem_ld_wait();
      for (int j0 = 0; j0 < ti.nt; j0 += 32) {
        // the next slab's TMEM load runs while this slab is staged and stored
        const bool more = j0 + 32 < ti.nt;
        if (more) tmem_ld32(tb + j0 + 32, vn);
        // sOut[i][r] = D[r][j0 + i]: token row i, weight row r
#pragma unroll
        for (int i = 0; i < 32; ++i) sOut[i * 128 + r] = __uint_as_float(v[i]);
        const int rows = tmin(32, ti.nt - j0);
        epi_bar();
        if constexpr (kMode == kTStore) {
          // a token row = 128 fp32 (32 x 16 B, 4 rows per pass) or 128 bf16
          // (16 x 16 B, 8 rows per pass)
          store_rows(p, sOut, et, rows, ti.m0 + j0, ti.wb * 128, sDst + j0, sFac + j0);
        } else {
          // swiglu: gate = weight rows 0..63, up = rows 64..127 of the block;
          // h row = 64 bf16 = 8 x 16 B; 16 rows per pass
#pragma unroll
          for (int pass = 0; pass < 2; ++pass) {
            const int i = pass * 16 + (et >> 3);
            const int c8 = et & 7;
            if (i < rows) {
              const float* g = sOut + i * 128 + c8 * 8;
              const float* u = g + 64;
              uint32_t pk[4];
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2)
                pk[k2] = pack_bf16x2(silu(g[2 * k2]) * u[2 * k2], silu(g[2 * k2 + 1]) * u[2 * k2 + 1]);
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) +
                                   static_cast<int64_t>(ti.m0 + j0 + i) * p.ldc + ti.wb * 64;
              reinterpret_cast<uint4*>(dst)[c8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
        epi_bar();  // sOut is rewritten by the next slab
        if (more) {
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = vn[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// K-major [rows, K] tensor of bf16 (or e4m3 bytes), boxes of 128 bytes x box_rows,
// 128-byte swizzle, zero fill out of bounds.
bool encode_kmajor_2d(CUtensorMap* map, const void* base, bool fp8, uint64_t K, uint64_t rows,
                      uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t elt = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * elt};
  cuuint32_t box[2] = {128 / elt, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kMode, int TN>
cudaError_t run_t(const GemmLaunch& L, cudaStream_t stream) {
  using Cfg = TCfg<kMode, TN>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_t_kernel<kMode, TN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const bool grouped = L.group_sizes != nullptr;
  const int E = grouped ? L.E : 1;
  CUtensorMap tmW, tmX[kXBoxes];
  const uint32_t wbox = kMode == kTSwiglu ? 64 : 128;
  if (!encode_kmajor_2d(&tmW, L.B, Cfg::kFp8, L.K, static_cast<uint64_t>(E) * L.N, wbox))
    return cudaErrorInvalidValue;
  for (int i = 0; i < kXBoxes; ++i)
    if (!encode_kmajor_2d(&tmX[i], L.A, Cfg::kFp8, L.K, L.rows, 32u << i))
      return cudaErrorInvalidValue;
  TParams p{};
  p.M_dense = grouped ? 0 : L.rows;
  p.N = L.N;
  p.K = L.K;
  p.E = E;
  p.group_sizes = L.group_sizes;
  p.group_offsets = L.group_offsets;
  p.rows_total = L.rows;
  p.C = L.C;
  p.ldc = kMode == kTSwiglu ? L.N / 2 : L.N;
  p.out_f32 = L.out_f32;
  p.out_f16e = L.out_f16e;
  p.C_exps = L.C_exps;
  p.A_scales = L.A_scales;
  p.B_scales = L.B_scales;
  p.KBS = L.K / 128;
  p.status = L.status;
  p.weighted = L.weighted;
  p.pair_of_row = L.pair_of_row;
  p.row_w = L.row_weights;
  p.row_scale = L.row_scale;
  const int WB = kMode == kTSwiglu ? (L.N / 2) / 64 : L.N / 128;
  const long long chunks_ub = grouped ? (static_cast<long long>(L.rows) + TN - 1) / TN + E
                                      : (static_cast<long long>(L.rows) + TN - 1) / TN;
  const long long tiles_ub = chunks_ub * WB;
  int sms = device_sm_count();
  if (L.max_ctas > 0 && L.max_ctas < sms) sms = L.max_ctas;
  const int grid = static_cast<int>(tiles_ub < sms ? (tiles_ub > 0 ? tiles_ub : 1) : sms);
  grouped_gemm_t_kernel<kMode, TN><<<grid, Cfg::kThreads, Cfg::SMEM_BYTES, stream>>>(
      tmW, tmX[0], tmX[1], tmX[2], tmX[3], p);
  return cudaGetLastError();
}

}  // namespace

bool grouped_gemm_t_supported(const GemmLaunch& L) {
  if (L.E > 1024) return false;
  if (L.out_f16e && ((L.mode != kModeStore && L.mode != kModeFp8Store) || L.weighted ||
                     L.out_f32 || L.C_exps == nullptr))
    return false;
  if (L.weighted && (L.pair_of_row == nullptr || L.row_weights == nullptr ||
                     L.group_sizes == nullptr ||
                     (L.mode != kModeStore && L.mode != kModeFp8Store)))
    return false;
  if (L.mode == kModeFp8Store)
    return L.A_scales != nullptr && L.B_scales != nullptr && L.N % 128 == 0 &&
           L.K % 128 == 0 && L.K <= 128 * TCfg<kTFp8Store, 64>::MAX_KBS;
  if (L.A_scales != nullptr || L.B_scales != nullptr) return false;
  if (L.mode == kModeStore) return L.N % 128 == 0 && L.K % 64 == 0;
  if (L.mode == kModeSwiglu) return (L.N / 2) % 64 == 0 && L.N % 2 == 0 && L.K % 64 == 0;
  return false;
}

cudaError_t launch_grouped_gemm_t(const GemmLaunch& L, cudaStream_t stream) {
  // Token tile sized to the groups: small groups (decode) keep 64-row token
  // tiles so 8 stages fit and more weight bytes stay in flight per SM.
  const bool small = L.group_sizes != nullptr && L.rows <= 64 * L.E;
  if (L.mode == kModeSwiglu)
    return small ? run_t<kTSwiglu, 64>(L, stream) : run_t<kTSwiglu, 256>(L, stream);
  if (L.mode == kModeStore)
    return small ? run_t<kTStore, 64>(L, stream) : run_t<kTStore, 256>(L, stream);
  if (L.mode == kModeFp8Store) return run_t<kTFp8Store, 64>(L, stream);
  return cudaErrorInvalidValue;
}

bool grouped_gemm_t_preferred(const GemmLaunch& L) {
  // measured on B200: weight-row tiles win for the down/store GEMM at every
  // group size once the token tile fits the groups, and for SwiGLU on small
  // groups; token-row tiles keep SwiGLU on large groups (their epilogue needs
  // no shared-memory pairing of gate and up)
  if (L.mode == kModeStore || L.mode == kModeFp8Store) return true;
  return L.group_sizes != nullptr && L.rows <= 64 * L.E;
}

}  // namespace moe
