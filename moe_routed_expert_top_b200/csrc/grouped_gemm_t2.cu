// grouped_gemm_t2.cu - weight-row tiles computed by a pair of CTAs (a cluster
// of two on one TPC) with cta_group::2 MMAs.
//
// Same operation and tile order as grouped_gemm_t.cu (TileOPs PR #1580
// "Grouped-GEMM TMA OOB zero-fill + unpermute out=", Grouped-GEMM kernel:
// C[e] = A[e] @ B[e]^T over each expert's rows): a pair tile is 256 weight rows
// x up to TN tokens of one expert. Each CTA of the pair loads its own 128
// weight rows and its own half of the token rows (no multicast: every CTA
// fetches its own tiles); the leader CTA issues the M=256 MMA, which reads both
// CTAs' shared memory and leaves each CTA's 128 rows x N columns in that CTA's
// tensor memory. Per CTA and per 64-wide K step this moves 16 KB of weights +
// TN/2 token rows instead of 16 KB + TN rows, for the same MMA work.
//
// Pair protocol:
//   * both CTAs' TMA loads complete on the leader's `full` barrier (the leader
//     alone arms it with the bytes of both halves);
//   * the leader's MMA commits to `empty` and `tfull` in both CTAs (multicast
//     commit), so each producer and each epilogue waits on local barriers;
//   * both CTAs' epilogue warps release an accumulator on the leader's `tempty`
//     barrier (8 arrivals);
//   * a cluster barrier after barrier initialisation and another before tensor
//     memory is freed keep either CTA from touching the other's shared memory
//     outside the kernel's lifetime.
// Modes: store (fp32 or bf16 C) and SwiGLU (64 gate rows stacked over the
// matching 64 up rows in each CTA's half; TileOPs PR #778, Design; XTuner
// PR #2089, SiLU(gate)*up). Every wait is bounded (4 s) and sets
// MOE_DEV_TIMEOUT on expiry.
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

enum PMode { kPStore = 0, kPSwiglu = 1 };

constexpr int kPXBoxes = 4;  // boxes of 16, 32, 64, 128 rows for a CTA's half of the tokens

struct PParams {
  int M_dense;
  int N;  // rows of W per expert
  int K;
  int E;
  const int32_t* group_sizes;
  const int32_t* group_offsets;
  int rows_total;
  void* C;
  int ldc;
  int out_f32;
  int out_f16e;     // C fp16 + C_exps int8 [rows, ldc / 128] (f16e.cuh)
  int8_t* C_exps;
  int32_t* status;
  // gather mode: token row r is hidden[pair_of_row[r] / top_k] (K columns)
  const __nv_bfloat16* hidden;
  const int32_t* pair_of_row;
  int top_k;
  int hidden_rows;
  int up_off;  // SwiGLU: rows from a gate row of W to its up row
  // weighted store: C row pair_of_row[r] = row_scale * row_w[pair] * result row r
  int weighted;
  const float* row_w;
  float row_scale;
};

__host__ __device__ constexpr int pmin(int a, int b) { return a < b ? a : b; }

template <int kMode, int TN>
struct PCfg {
  static constexpr int BK = 64;
  static constexpr int K_STEPS = 4;
  static constexpr int A_BYTES = 128 * 128;       // this CTA's 128 weight rows
  static constexpr int B_BYTES = (TN / 2) * 128;  // this CTA's half of the token rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = pmin(8, (200 * 1024) / STAGE_BYTES);
  static constexpr int NUM_ACC = 2;
  static constexpr int TMEM_COLS = 2 * TN;
  // 32 token rows x 128 fp32 (16 per epilogue group), then each group's copy
  // of the tile's row destinations and factors (weighted store)
  static constexpr int STAGE_OUT_BYTES = 32 * 128 * 4 + 4 * TN * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NUM_ACC + 1;
  static constexpr int MAX_E = 1024;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGE_OUT_BYTES +
                                    NUM_BARS * 8 + 16 + 2 * (MAX_E + 8) * 4;
  static constexpr int PAIR_COLS = (kMode == kPSwiglu) ? 128 : 256;  // output columns per pair tile
  static constexpr int CTA_COLS = PAIR_COLS / 2;
  static_assert(TN % 32 == 0 && TN >= 32 && TN <= 256, "token tile");
  static_assert(TMEM_COLS <= 512, "tensor memory");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct PTile {
  int e, wb, m0, nt;
  int chunks;  // token tiles of this expert (tiles that read the same weights)
};

// Tile t -> (expert, weight block, token chunk), from cpre (token chunks of the
// experts before e) and soff (group_offsets), both in shared memory. A pair
// visits its tiles in increasing order, so each warp keeps the expert of its
// last tile in `ecur` and only moves it forward.
__device__ __forceinline__ bool p_decode(const PParams& p, const int* cpre, const int* soff,
                                         int WB, int TN, int t, int& ecur, PTile& ti) {
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
  // the expert's tokens split evenly over its tiles (in multiples of 32)
  const int ts = pmin(TN, ((size + chunks - 1) / chunks + 31) & ~31);
  ti.m0 = off + c * ts;
  ti.nt = pmin(ts, size - c * ts);
  if (ti.nt <= 0 || ti.m0 < 0 || ti.m0 + ti.nt > p.rows_total) {
    if (threadIdx.x == 0 && ti.nt > 0) atomicOr(p.status, MOE_DEV_BAD_TABLES_FLAG);
    return false;
  }
  return true;
}

__device__ __forceinline__ int half_box(int half) {  // smallest of 16/32/64/128 rows >= half
  return half <= 16 ? 0 : half <= 32 ? 1 : half <= 64 ? 2 : 3;
}

// Named barrier of epilogue group g (its 128 threads).
__device__ __forceinline__ void pgroup_bar(int g) {
  if (g == 0)
    asm volatile("bar.sync 1, 128;" ::: "memory");
  else
    asm volatile("bar.sync 2, 128;" ::: "memory");
}

__device__ __forceinline__ float psilu(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ void pair_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// Threads per CTA: producer warp, MMA warp, two groups of 4 epilogue warps.
constexpr int kPairThreads = 320;  // TMA, MMA, two groups of 4 epilogue warps

template <int kMode, int TN, bool kGather>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmW,
                             const __grid_constant__ CUtensorMap tmX0,
                             const __grid_constant__ CUtensorMap tmX1,
                             const __grid_constant__ CUtensorMap tmX2,
                             const __grid_constant__ CUtensorMap tmX3, const PParams p) {
  using Cfg = PCfg<kMode, TN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int NUM_ACC = Cfg::NUM_ACC;
  constexpr int kThreads = kPairThreads;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  float* sOut = reinterpret_cast<float*>(sB + STAGES * Cfg::B_BYTES);
  int* sDst = reinterpret_cast<int*>(sOut + 32 * 128);  // weighted store: [2][TN] row info
  float* sFac = reinterpret_cast<float*>(sDst + 2 * TN);   // [2][TN]
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sOut) + Cfg::STAGE_OUT_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* cpre = reinterpret_cast<int*>(tmem_slot + 4);  // [E + 1]
  int* soff = cpre + Cfg::MAX_E + 8;                    // [E + 1]: group_offsets

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * STAGES;
  const uint32_t tfull0 = empty0 + 8 * STAGES;
  const uint32_t tempty0 = tfull0 + 8 * NUM_ACC;
  const uint32_t drain_bar = tempty0 + 8 * NUM_ACC;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = p.group_sizes ? p.E : 1;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 16);  // 8 epilogue warps in each CTA of the pair
    }
    mbar_init(drain_bar, 1);
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
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
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
    int* wsum = reinterpret_cast<int*>(sOut);
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
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or load completion
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int WB = (kMode == kPSwiglu) ? (p.N / 2) / 128 : p.N / 256;
  const int total_tiles = WB * cpre[E];
  const int KB = p.K / Cfg::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // Lane 0 waits for free stages and loads the weight rows (and the token
    // rows as one box). Gather mode: the token rows are hidden-state rows
    // picked through pair_of_row, and lane l fetches rows 4l..4l+3 of this
    // CTA's half with one four-row TMA gather (512 B of the 128-byte-swizzled
    // tile: the same bytes in the same place as the box load).
    if (kGather || lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      const uint64_t pol_w1 = l2_policy_by_code(MOE_W_POLICY_SINGLE);
      const uint64_t pol_wn = l2_policy_by_code(MOE_W_POLICY_MULTI);
      const CUtensorMap* xmaps[kPXBoxes] = {&tmX0, &tmX1, &tmX2, &tmX3};
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;  // stages whose loads this CTA issued
      bool ok = true;
      int ecur = 0;
      for (int t = pair; ok && t < total_tiles; t += npairs) {
        PTile ti;
        if (!p_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
        const int nmma = (ti.nt + 31) & ~31;
        const int half = nmma / 2;
        const int xb = half_box(half);
        const uint32_t x_bytes = kGather ? static_cast<uint32_t>(half) * 128u : (16u << xb) * 128u;
        const uint32_t bytes_pair = 2u * (Cfg::A_BYTES + x_bytes);
        const int wrow = ti.e * p.N + ti.wb * Cfg::PAIR_COLS +
                         static_cast<int>(rank) * (kMode == kPSwiglu ? 64 : 128);
        const uint64_t pol_w = ti.chunks > 1 ? pol_wn : pol_w1;
        const int trow = ti.m0 + static_cast<int>(rank) * half;
        const bool gather_lane = kGather && 4 * lane < half;
        int g[4] = {0, 0, 0, 0};
        if (gather_lane) {
          // rows past the tile's tokens repeat its first token: they only feed
          // MMA columns that are never stored
          auto token_of = [&](int row) {
            const int v = __ldg(p.pair_of_row + row) / p.top_k;
            return v < 0 ? 0 : (v >= p.hidden_rows ? p.hidden_rows - 1 : v);
          };
          const int first = token_of(ti.m0);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = trow - ti.m0 + 4 * lane + j;  // row within the tile
            g[j] = i < ti.nt ? token_of(ti.m0 + i) : first;
          }
        }
        for (int kb = 0; kb < KB; ++kb) {
          uint32_t got = 1;
          if (lane == 0) got = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status);
          if constexpr (kGather) got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          const uint32_t fb_local = full0 + 8 * stage;
          const uint32_t fb = cluster_map_shared(fb_local, 0);
          const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_BYTES);
          if (lane == 0) {
            if (leader) mbar_arrive_expect_tx(fb_local, bytes_pair);
            const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
            if constexpr (kMode == kPSwiglu) {
              tma_load_2d_pair(a_dst, &tmW, kb * Cfg::BK, wrow, fb, pol_w);
              tma_load_2d_pair(a_dst + 64 * 128, &tmW, kb * Cfg::BK, wrow + p.up_off, fb, pol_w);
            } else {
              tma_load_2d_pair(a_dst, &tmW, kb * Cfg::BK, wrow, fb, pol_w);
            }
            if constexpr (!kGather)
              tma_load_2d_pair(b_dst, xmaps[xb], kb * Cfg::BK, trow, fb, pol_act);
          }
          if (gather_lane)
            tma_gather4_pair(b_dst + lane * 512, &tmX0, kb * Cfg::BK, g[0], g[1], g[2], g[3], fb,
                             pol_act);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && lane == 0) {
        // A wait gave up: the copies of the last min(issued, STAGES) stages may
        // still be in flight into this CTA's shared memory, completing on the
        // leader's `full` barriers. The leader waits for those phases (it armed
        // each with both halves' bytes, so they complete once both CTAs' copies
        // of the stage have landed); the other CTA cannot wait on the leader's
        // barriers and instead waits for the MMA's release of each stage on its
        // own `empty` barriers (a release means both halves landed and were
        // read). One shared time limit bounds the whole drain; the cluster
        // barrier at the end keeps both CTAs alive until both have drained.
        const uint32_t n = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        int s = stage;
        uint32_t ph = phase;
        for (uint32_t i = 0; i < n; ++i) {
          if (--s < 0) {
            s = STAGES - 1;
            ph ^= 1u;
          }
          if (leader)
            mbar_wait_until(full0 + 8 * s, ph, deadline);
          else
            mbar_wait_until(empty0 + 8 * s, ph, deadline);
        }
      }
      // every load this CTA issued has been consumed (its stage released) before leaving
      if (ok && lane == 0) {
        for (int i = 0; i < STAGES; ++i) {
          mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int ecur = 0;
      for (int t = pair; ok && t < total_tiles; t += npairs) {
        PTile ti;
        if (!p_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
        const int nmma = (ti.nt + 31) & ~31;
        const uint32_t idesc = idesc_bf16_f32(256, nmma);
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
            mma_bf16_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair_mc(empty0 + 8 * stage, 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(tfull0 + 8 * acc, 0x3);
        if (++acc == NUM_ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      pair_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Two groups of four warps (2-5 and 6-9). In each 32-token slab of a tile,
    // group g takes tokens 16g .. 16g+15: its own TMEM columns, its own 16 rows
    // of sOut and its own named barrier, so one group's stores and barrier
    // waits overlap the other's TMEM loads. Warp w reads TMEM lanes
    // 32*(w%4) .. +31 (its weight rows).
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int et = threadIdx.x - 64 - 128 * grp;  // 0..127 within the group
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float* gOut = sOut + grp * 16 * 128;
    int* gDst = sDst + grp * TN;
    float* gFac = sFac + grp * TN;
    int acc = 0;
    uint32_t acc_phase = 0;
    int ecur = 0;
    for (int t = pair; t < total_tiles; t += npairs) {
      PTile ti;
      if (!p_decode(p, cpre, soff, WB, TN, t, ecur, ti)) continue;
      if (kMode == kPStore && p.weighted) {
        // the tile's row destinations (flat pair index, -1 = none) and factors,
        // loaded while its MMAs run; read after the first slab's barrier
        for (int i = et; i < ti.nt; i += 128) {
          const int pr = __ldg(p.pair_of_row + ti.m0 + i);
          gDst[i] = pr;
          gFac[i] = pr >= 0 ? p.row_scale * __ldg(p.row_w + pr) : 0.0f;
        }
      }
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.status)) *epi_abort = 1;
      pgroup_bar(grp);
      if (*epi_abort) break;
      tc_fence_after();
      const uint32_t tb = lane_base + static_cast<uint32_t>(acc * TN + 16 * grp);
      const int col0 = ti.wb * Cfg::PAIR_COLS + static_cast<int>(rank) * Cfg::CTA_COLS;
      uint32_t v[16], vn[16];
      tmem_ld16(tb, v);
      tmem_ld_wait();
      for (int j0 = 0; j0 < ti.nt; j0 += 32) {
        const bool more = j0 + 32 < ti.nt;
        if (more) tmem_ld16(tb + j0 + 32, vn);
#pragma unroll
        for (int i = 0; i < 16; ++i) gOut[i * 128 + r] = __uint_as_float(v[i]);
        const int jg = j0 + 16 * grp;  // the group's first token of this slab
        const int rows = pmin(16, ti.nt - jg);  // may be <= 0: nothing to store
        pgroup_bar(grp);
        if constexpr (kMode == kPStore) {
          if (p.out_f32) {
#pragma unroll
            for (int pass = 0; pass < 4; ++pass) {
              const int i = pass * 4 + (et >> 5);
              const int c4 = et & 31;
              if (i < rows) {
                float4 val = reinterpret_cast<const float4*>(gOut + i * 128)[c4];
                int drow = ti.m0 + jg + i;
                if (p.weighted) {
                  drow = gDst[jg + i];
                  const float f = gFac[jg + i];
                  if (drow < 0) continue;
                  val = make_float4(val.x * f, val.y * f, val.z * f, val.w * f);
                }
                float* dst = static_cast<float*>(p.C) + static_cast<int64_t>(drow) * p.ldc + col0;
                reinterpret_cast<float4*>(dst)[c4] = val;
              }
            }
          } else if (p.out_f16e) {
            // f16e: a row's 128 columns are this CTA's output block, held by 16
            // lanes of a half warp (8 columns each); every lane encodes
            const int c8 = et & 15;
            float fv[2][8];
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
              const float4* src =
                  reinterpret_cast<const float4*>(gOut + (pass * 8 + (et >> 4)) * 128 + c8 * 8);
              const float4 a = src[0], b = src[1];
              fv[pass][0] = a.x; fv[pass][1] = a.y; fv[pass][2] = a.z; fv[pass][3] = a.w;
              fv[pass][4] = b.x; fv[pass][5] = b.y; fv[pass][6] = b.z; fv[pass][7] = b.w;
            }
            uint4 pk[2];
            int e[2];
            f16e_encode8xn<2>(fv, pk, e);
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
              const int i = pass * 8 + (et >> 4);
              if (i < rows) {
                const int64_t row = ti.m0 + jg + i;
                __half* dst = static_cast<__half*>(p.C) + row * p.ldc + col0;
                reinterpret_cast<uint4*>(dst)[c8] = pk[pass];
                if (c8 == 0)
                  p.C_exps[row * (p.ldc / 128) + col0 / 128] = static_cast<int8_t>(e[pass]);
              }
            }
          } else {
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
              const int i = pass * 8 + (et >> 4);
              const int c8 = et & 15;
              if (i < rows) {
                const float* src = gOut + i * 128 + c8 * 8;
                int drow = ti.m0 + jg + i;
                float f = 1.0f;
                if (p.weighted) {
                  drow = gDst[jg + i];
                  f = gFac[jg + i];
                  if (drow < 0) continue;
                }
                const uint4 val =
                    p.weighted ? make_uint4(pack_bf16x2(src[0] * f, src[1] * f),
                                            pack_bf16x2(src[2] * f, src[3] * f),
                                            pack_bf16x2(src[4] * f, src[5] * f),
                                            pack_bf16x2(src[6] * f, src[7] * f))
                               : make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                                            pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) +
                                     static_cast<int64_t>(drow) * p.ldc + col0;
                reinterpret_cast<uint4*>(dst)[c8] = val;
              }
            }
          }
        } else {
          // swiglu: gate = weight rows 0..63, up = rows 64..127 of this CTA's
          // block; an h row = 64 bf16 = 8 x 16 B; 16 rows per pass
          const int i = et >> 3;
          const int c8 = et & 7;
          if (i < rows) {
            const float* g = gOut + i * 128 + c8 * 8;
            const float* u = g + 64;
            uint32_t pk[4];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2)
              pk[k2] = pack_bf16x2(psilu(g[2 * k2]) * u[2 * k2],
                                   psilu(g[2 * k2 + 1]) * u[2 * k2 + 1]);
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) +
                                 static_cast<int64_t>(ti.m0 + jg + i) * p.ldc + col0;
            reinterpret_cast<uint4*>(dst)[c8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        pgroup_bar(grp);  // the group's rows of sOut are rewritten by its next slab
        if (more) {
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = vn[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map_shared(tempty0 + 8 * acc, 0));
      if (++acc == NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  cluster_sync();  // neither CTA frees tensor memory or exits while its pair still runs
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 p_encode_fn() {
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

// Tensor map of a bf16 matrix of `rows` rows of K elements, `ld` elements apart.
bool p_encode(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
              uint64_t ld) {
  auto fn = p_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kMode, int TN, bool kGather>
cudaError_t run_pair(const GemmLaunch& L, cudaStream_t stream) {
  using Cfg = PCfg<kMode, TN>;
  constexpr int kThreads = kPairThreads;
  static int max_pairs_cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (max_pairs_cache[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<kMode, TN, kGather>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // pairs that can be resident at once (a pair needs both SMs of one TPC free)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(device_sm_count() & ~1));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<kMode, TN, kGather>, &cfg);
    if (e != cudaSuccess) return e;
    max_pairs_cache[dev] = n > 0 ? n : 1;
  }
  const bool grouped = L.group_sizes != nullptr;
  const int E = grouped ? L.E : 1;
  // rows of the A operand in memory: the hidden states in gather mode
  const int a_rows = kGather ? L.a_rows : L.rows;
  CUtensorMap tmW, tmX[kPXBoxes];
  const uint64_t b_rows = L.b_rows > 0 ? static_cast<uint64_t>(L.b_rows) : static_cast<uint64_t>(E) * L.N;
  const uint64_t ldb = L.ldb > 0 ? static_cast<uint64_t>(L.ldb) : static_cast<uint64_t>(L.K);
  if (!p_encode(&tmW, L.B, L.K, b_rows, kMode == kPSwiglu ? 64 : 128, ldb))
    return cudaErrorInvalidValue;
  // gather mode: map 0 is the hidden states with a one-row-high box (four-row gathers)
  for (int i = 0; i < kPXBoxes; ++i)
    if (!p_encode(&tmX[i], L.A, L.K, a_rows, kGather && i == 0 ? 1u : 16u << i, L.K))
      return cudaErrorInvalidValue;
  PParams p{};
  p.M_dense = grouped ? 0 : L.rows;
  p.N = L.N;
  p.K = L.K;
  p.E = E;
  p.group_sizes = L.group_sizes;
  p.group_offsets = L.group_offsets;
  p.rows_total = L.rows;
  p.C = L.C;
  p.ldc = kMode == kPSwiglu ? L.N / 2 : L.N;
  p.out_f32 = L.out_f32;
  p.out_f16e = L.out_f16e;
  p.C_exps = L.C_exps;
  p.status = L.status;
  p.hidden = static_cast<const __nv_bfloat16*>(L.A);
  p.pair_of_row = L.pair_of_row;
  p.top_k = L.top_k;
  p.hidden_rows = a_rows;
  p.up_off = L.up_off > 0 ? L.up_off : L.N / 2;
  p.weighted = L.weighted;
  p.row_w = L.row_weights;
  p.row_scale = L.row_scale;
  const int WB = kMode == kPSwiglu ? (L.N / 2) / 128 : L.N / 256;
  const long long chunks_ub = grouped ? (static_cast<long long>(L.rows) + TN - 1) / TN + E
                                      : (static_cast<long long>(L.rows) + TN - 1) / TN;
  const long long pairs_ub = chunks_ub * WB;
  int max_pairs = max_pairs_cache[dev];
  if (L.max_ctas > 0 && L.max_ctas / 2 < max_pairs) max_pairs = L.max_ctas / 2 > 0 ? L.max_ctas / 2 : 1;
  const int pairs = static_cast<int>(pairs_ub < max_pairs ? (pairs_ub > 0 ? pairs_ub : 1) : max_pairs);
  grouped_gemm_pair_kernel<kMode, TN, kGather><<<2 * pairs, kThreads, Cfg::SMEM_BYTES, stream>>>(
      tmW, tmX[0], tmX[1], tmX[2], tmX[3], p);
  return cudaGetLastError();
}

template <int kMode, int TN>
cudaError_t run_pair_g(const GemmLaunch& L, cudaStream_t stream) {
  return L.gather ? run_pair<kMode, TN, true>(L, stream) : run_pair<kMode, TN, false>(L, stream);
}

}  // namespace

bool grouped_gemm_pair_supported(const GemmLaunch& L) {
  if (L.A_scales != nullptr || L.B_scales != nullptr || L.E > 1024) return false;
  if (L.weighted && (L.pair_of_row == nullptr || L.row_weights == nullptr ||
                     L.group_sizes == nullptr || L.mode != kModeStore))
    return false;
  // gathering needs the group tables and the row -> pair map
  if (L.gather && (L.group_sizes == nullptr || L.pair_of_row == nullptr || L.top_k <= 0 ||
                   L.a_rows <= 0))
    return false;
  // a strided view of B: rows at least K long, 16-byte row pitch
  if (L.ldb != 0 && (L.ldb < L.K || L.ldb % 8 != 0)) return false;
  if (L.out_f16e && (L.mode != kModeStore || L.weighted || L.out_f32 || L.C_exps == nullptr))
    return false;
  if (L.mode == kModeStore) return L.N % 256 == 0 && L.K % 64 == 0 && L.up_off == 0;
  if (L.mode == kModeSwiglu) return (L.N / 2) % 128 == 0 && L.K % 64 == 0;
  return false;
}

// Measured on B200 with the bf16 workloads (interleaved runs): pairs beat the
// single-CTA weight-row and token-row tilings once experts hold more than 64
// rows on average (prefill; down projection by 10-30%), and are on par or
// slightly behind below that (decode), where the single-CTA kernel's 64-token
// tiles fit the groups better.
bool grouped_gemm_pair_preferred(const GemmLaunch& L) {
  if (!grouped_gemm_pair_supported(L)) return false;
  return L.group_sizes == nullptr || L.rows > 64 * L.E;
}

cudaError_t launch_grouped_gemm_pair(const GemmLaunch& L, cudaStream_t stream) {
  const bool small = L.group_sizes != nullptr && L.rows <= 64 * L.E;
  // A dense problem too small to give three quarters of the CTA pairs a
  // 256-token tile (a tensor-parallel rank's shared expert, few tokens) takes
  // 128-token tiles: twice the tiles, and the MMA still runs at its full rate
  // from N = 128 (one rank of tp 8 at Kimi-K2's shared expert: 36 -> 72 tiles).
  bool mid = false;
  if (!small && L.group_sizes == nullptr && L.rows > 128) {
    const long long wb = L.mode == kModeSwiglu ? (L.N / 2) / 128 : L.N / 256;
    const long long tiles256 = wb * ((static_cast<long long>(L.rows) + 255) / 256);
    mid = tiles256 * 4 < static_cast<long long>(device_sm_count() / 2) * 3;
  }
  if (L.mode == kModeSwiglu)
    return small ? run_pair_g<kPSwiglu, 64>(L, stream)
                 : mid ? run_pair_g<kPSwiglu, 128>(L, stream)
                       : run_pair_g<kPSwiglu, 256>(L, stream);
  if (L.mode == kModeStore)
    return small ? run_pair_g<kPStore, 64>(L, stream)
                 : mid ? run_pair_g<kPStore, 128>(L, stream)
                       : run_pair_g<kPStore, 256>(L, stream);
  return cudaErrorInvalidValue;
}

}  // namespace moe
