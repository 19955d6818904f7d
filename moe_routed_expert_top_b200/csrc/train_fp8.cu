// train_fp8.cu - training-side FP8 activation layouts and the SwiGLU backward
// (XTuner PR #2089 "Fuse MoE activation FP8 quantization kernels", Changes):
//
//  * dual-layout quantisation of an activation x [M, K] in one pass over x:
//    the forward layout (codes [M, K], one scale per 1x128 row tile, as
//    per_tile_quant) and a transposed, expert-padded copy for the
//    weight-gradient GEMM, which contracts over tokens: xT [K, Mp] with the
//    rows of each expert starting a fresh 128-token block (expand_128x), one
//    scale per 128x128 block (trans_per_block) or per 1x128 tile of an xT row
//    (trans_per_tile). The padded token axis is the block layout of the
//    TileLang tutorial "Example 07" section 1 (block_token 128): block bx
//    belongs to expert group_idx_for_bx[bx] and holds its rows from
//    m_start = bx*128 - group_padded_offsets[g] + group_offsets[g];
//  * the same with x = SiLU(gate) * up computed in fp32 from gate_up
//    (swiglu_per_tile_quant_with_trans_per_block): no bf16 h is written;
//  * swiglu_backward: grad_gate_up [M, 2F] from gate_up and dL/dh in one pass.
//
// Scale rule everywhere (as in the forward quantiser): s = amax / 448 with
// IEEE division, codes = e4m3_rn_satfinite(x / s), an all-zero tile or block
// has s = 0 and codes 0; padding tokens are zeros.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

// The tile is staged in shared memory for the transposed pass: the SwiGLU
// form as fp32 h (129 words per row), the plain form as its bf16 input rows
// (136 elements per row, 16-byte aligned), which halves the footprint and
// doubles the CTAs per SM.
constexpr int kTileStride = 129;
constexpr int kTileStrideBf16 = 136;
__host__ __device__ constexpr int dual_smem(bool swiglu) {
  return (swiglu ? 128 * kTileStride * 4 : 128 * kTileStrideBf16 * 2) + 512 * 4;  // + reduce
}

struct DualParams {
  int M;  // rows of x
  int K;  // columns of the quantised activation (SwiGLU: F)
  int E;
  const int32_t* sizes;  // grouped mode; null in dense mode
  const int32_t* offsets;
  const int32_t* padded;
  const int32_t* idx_for_bx;
  int M_blk;                 // 128-token blocks on the padded axis
  const __nv_bfloat16* x;    // [M, K], or gate_up [M, 2K] in SwiGLU mode
  uint8_t* q;                // [M, K]
  float* s;                  // [M, K / 128]
  uint8_t* qT;               // [K, 128 * M_blk]
  float* sT;                 // per block [K / 128, M_blk]; per tile [K, M_blk]
  float* debug_h;            // SwiGLU mode: fp32 h [M, K], or null
};

__device__ __forceinline__ void unpack8(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = bf16lo_to_f32(w[j]);
    f[2 * j + 1] = bf16hi_to_f32(w[j]);
  }
}

// x / s rounded to nearest even, from y = RN(1/s): q0 = RN(x*y) lies within
// 2 ulp of x/s; each correction q += RN(x - s*q) * y, with the residual
// x - s*q exact in one FMA, is Markstein's division step (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): after the first q is within one
// ulp and the second gives the correctly rounded quotient, provided the
// residual does not underflow. With s >= 2^-90 it cannot wherever the
// quotient reaches 2^-11 (below that every value encodes to a signed zero in
// E4M3), so callers use this for s >= 2^-90 and plain division otherwise.
// A zero x keeps its sign (q0 is that zero).
__device__ __forceinline__ float div_by_scale(float x, float s, float y) {
  const float q0 = x * y;
  const float q1 = fmaf(fmaf(-q0, s, x), y, q0);
  const float q2 = fmaf(fmaf(-q1, s, x), y, q1);
  return q0 == 0.0f ? q0 : q2;
}

constexpr float kFastDivMinScale = 8.0779356e-28f;  // 2^-90

// 32 values -> 32 E4M3 codes (scale s, or all zero when amax == 0) as 2 x 16 B.
__device__ __forceinline__ void encode32(const float* v, float amax, float s, uint4* out) {
  uint32_t w[8];
  if (amax > 0.0f && s >= kFastDivMinScale) {
    const float y = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = static_cast<uint32_t>(cvt_e4m3x2(div_by_scale(v[4 * j], s, y),
                                              div_by_scale(v[4 * j + 1], s, y))) |
             (static_cast<uint32_t>(cvt_e4m3x2(div_by_scale(v[4 * j + 2], s, y),
                                               div_by_scale(v[4 * j + 3], s, y)))
              << 16);
  } else if (amax > 0.0f) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = static_cast<uint32_t>(cvt_e4m3x2(v[4 * j] / s, v[4 * j + 1] / s)) |
             (static_cast<uint32_t>(cvt_e4m3x2(v[4 * j + 2] / s, v[4 * j + 3] / s)) << 16);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = 0u;
  }
  out[0] = make_uint4(w[0], w[1], w[2], w[3]);
  out[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

constexpr int kDualThreads = 512;

// One CTA per (128-token block bx of the padded axis, 128-column block kb);
// 512 threads, 32 values each. Phase A: thread (row i = t/4, quarter t%4)
// reads 32 values of its row, writes their row-layout codes (each row segment
// of 128 is one 1x128 tile, its amax shared by the row's 4 threads) and stages
// the values in shared memory. Phase B: thread (column c = t%128, token
// quarter t/128) reads 32 staged values down its column and writes them as 32
// contiguous codes of xT row kb*128 + c.
template <bool kSwiglu, bool kTransBlock>
__global__ void __launch_bounds__(kDualThreads, 2) quant_dual_kernel(const DualParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* tile = reinterpret_cast<float*>(smem_raw);                  // SwiGLU: [128][129] fp32
  __nv_bfloat16* tile16 = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // plain: [128][136] bf16
  float* red = reinterpret_cast<float*>(smem_raw + dual_smem(kSwiglu) - kDualThreads * 4);
  const int bx = blockIdx.x;
  const int kb = blockIdx.y;
  const int t = threadIdx.x;

  int m_start = 0, rows = 0;
  if (p.idx_for_bx != nullptr) {
    const int g = __ldg(p.idx_for_bx + bx);
    if (g >= 0 && g < p.E) {
      const int local = bx * 128 - __ldg(p.padded + g);
      const int size = __ldg(p.sizes + g);
      m_start = __ldg(p.offsets + g) + local;
      rows = local < 0 ? 0 : min(max(size - local, 0), 128);
    }
  } else {
    m_start = bx * 128;
    rows = max(0, min(128, p.M - m_start));
  }
  if (m_start < 0 || m_start + rows > p.M) rows = 0;  // inconsistent tables: zeros only
  const int KB = p.K / 128;

  // ---------------------------------------------------------------- phase A
  {
    const int i = t >> 2;
    const int qq = t & 3;
    const int col = kb * 128 + qq * 32;
    float v[32];
    const bool live = i < rows;
    if (live) {
      const int64_t r = static_cast<int64_t>(m_start + i);
      if constexpr (kSwiglu) {
        const uint4* gsrc = reinterpret_cast<const uint4*>(p.x + r * 2 * p.K + col);
        const uint4* usrc = reinterpret_cast<const uint4*>(p.x + r * 2 * p.K + p.K + col);
        uint4 graw[4], uraw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          graw[j] = __ldg(gsrc + j);
          uraw[j] = __ldg(usrc + j);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float g[8], u[8];
          unpack8(graw[j], g);
          unpack8(uraw[j], u);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[8 * j + e] = g[e] / (1.0f + expf(-g[e])) * u[e];
        }
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + r * p.K + col);
        uint4 raw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = __ldg(src + j);
        uint4* st = reinterpret_cast<uint4*>(tile16 + i * kTileStrideBf16 + qq * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          st[j] = raw[j];
          unpack8(raw[j], v + 8 * j);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
      if constexpr (!kSwiglu) {
        uint4* st = reinterpret_cast<uint4*>(tile16 + i * kTileStrideBf16 + qq * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) st[j] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float s = amax / 448.0f;
    if (live) {
      const int64_t r = static_cast<int64_t>(m_start + i);
      uint4 codes[2];
      encode32(v, amax, s, codes);
      uint4* dst = reinterpret_cast<uint4*>(p.q + r * p.K + col);
      dst[0] = codes[0];
      dst[1] = codes[1];
      if (qq == 0) p.s[r * KB + kb] = amax > 0.0f ? s : 0.0f;
      if (kSwiglu && p.debug_h != nullptr) {
        float4* hd = reinterpret_cast<float4*>(p.debug_h + r * p.K + col);
#pragma unroll
        for (int j = 0; j < 8; ++j) hd[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
    }
    if constexpr (kSwiglu) {
#pragma unroll
      for (int j = 0; j < 32; ++j) tile[i * kTileStride + qq * 32 + j] = v[j];
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase B
  const int c = t & 127;
  const int tq = t >> 7;
  float w[32];
  if constexpr (kSwiglu) {
#pragma unroll
    for (int r = 0; r < 32; ++r) w[r] = tile[(tq * 32 + r) * kTileStride + c];
  } else {
#pragma unroll
    for (int r = 0; r < 32; ++r) w[r] = __bfloat162float(tile16[(tq * 32 + r) * kTileStrideBf16 + c]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int r = 0; r < 32; ++r) amax = fmaxf(amax, fabsf(w[r]));
  if constexpr (kTransBlock) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((t & 31) == 0) red[t >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int wi = 1; wi < kDualThreads / 32; ++wi) amax = fmaxf(amax, red[wi]);
  } else {
    red[t] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[c], red[c + 128]), fmaxf(red[c + 256], red[c + 384]));
  }
  const float s = amax / 448.0f;
  uint4 codes[2];
  encode32(w, amax, s, codes);
  const int64_t ldT = static_cast<int64_t>(p.M_blk) * 128;
  uint4* dst = reinterpret_cast<uint4*>(p.qT + static_cast<int64_t>(kb * 128 + c) * ldT +
                                        static_cast<int64_t>(bx) * 128 + tq * 32);
  dst[0] = codes[0];
  dst[1] = codes[1];
  const float sv = amax > 0.0f ? s : 0.0f;
  if constexpr (kTransBlock) {
    if (t == 0) p.sT[static_cast<int64_t>(kb) * p.M_blk + bx] = sv;
  } else {
    if (tq == 0) p.sT[static_cast<int64_t>(kb * 128 + c) * p.M_blk + bx] = sv;
  }
}

// grad_gate_up [M, 2F] from gate_up [M, 2F] and grad_h [M, F]; 8 columns per
// thread and step, fp32 arithmetic, bf16 results.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(long long n8, int F8,
                                                              const uint4* __restrict__ gu,
                                                              const uint4* __restrict__ dh,
                                                              uint4* __restrict__ out) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += stride) {
    const long long r = i / F8;
    const int c8 = static_cast<int>(i - r * F8);
    float g[8], u[8], d[8];
    unpack8(__ldg(gu + r * 2 * F8 + c8), g);
    unpack8(__ldg(gu + r * 2 * F8 + F8 + c8), u);
    unpack8(__ldg(dh + r * F8 + c8), d);
    uint32_t og[4], ou[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float a[2], b[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x = g[2 * j + e];
        const float sg = 1.0f / (1.0f + expf(-x));
        a[e] = d[2 * j + e] * u[2 * j + e] * (sg * (1.0f + x * (1.0f - sg)));
        b[e] = d[2 * j + e] * (x * sg);
      }
      og[j] = pack_bf16x2(a[0], a[1]);
      ou[j] = pack_bf16x2(b[0], b[1]);
    }
    out[r * 2 * F8 + c8] = make_uint4(og[0], og[1], og[2], og[3]);
    out[r * 2 * F8 + F8 + c8] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
}

template <bool kSwiglu, bool kTransBlock>
cudaError_t run_dual(const DualParams& p, cudaStream_t stream) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(quant_dual_kernel<kSwiglu, kTransBlock>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, dual_smem(kSwiglu));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const dim3 grid(static_cast<unsigned>(p.M_blk), static_cast<unsigned>(p.K / 128));
  quant_dual_kernel<kSwiglu, kTransBlock><<<grid, kDualThreads, dual_smem(kSwiglu), stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_dual(const DualLaunch& L, cudaStream_t stream) {
  if (L.M_blk <= 0 || L.K <= 0) return cudaSuccess;
  DualParams p;
  p.M = L.M;
  p.K = L.K;
  p.E = L.E;
  p.sizes = L.sizes;
  p.offsets = L.offsets;
  p.padded = L.padded;
  p.idx_for_bx = L.idx_for_bx;
  p.M_blk = L.M_blk;
  p.x = static_cast<const __nv_bfloat16*>(L.x);
  p.q = L.q;
  p.s = L.s;
  p.qT = L.qT;
  p.sT = L.sT;
  p.debug_h = L.debug_h;
  if (L.swiglu)
    return L.trans_block ? run_dual<true, true>(p, stream) : run_dual<true, false>(p, stream);
  return L.trans_block ? run_dual<false, true>(p, stream) : run_dual<false, false>(p, stream);
}

cudaError_t launch_swiglu_backward(int M, int F, const void* gate_up, const void* grad_h,
                                   void* grad_gate_up, cudaStream_t stream) {
  if (M <= 0 || F <= 0) return cudaSuccess;
  const long long n8 = static_cast<long long>(M) * (F / 8);
  const long long want = (n8 + 255) / 256;
  const long long cap = static_cast<long long>(device_sm_count()) * 8;
  const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
  swiglu_backward_kernel<<<blocks, 256, 0, stream>>>(
      n8, F / 8, static_cast<const uint4*>(gate_up), static_cast<const uint4*>(grad_h),
      static_cast<uint4*>(grad_gate_up));
  return cudaGetLastError();
}

}  // namespace moe
