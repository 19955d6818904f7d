// elementwise.cu - a7 weighted unpermute and the combine of pre-weighted rows,
// a5 standalone SwiGLU(+E4M3 1x128 quantisation), and the offline 128x128
// block quantisation of FP8 weights.
// All three are HBM-streaming kernels: 16-byte vector loads/stores, fp32 math.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "f16e.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// a7: out[t] = bf16( scale * sum_j w[t,j] * y[row_of_pair[t*k+j]] + addend[t] )
// (TileOPs PR #1580, Unpermute: scaling folded in before the cast/store; the
// result is written straight into the caller's output buffer). y and the
// addend are fp32 (the down GEMM's accumulator, not rounded in between). One
// thread per 8 columns of one token; fp32 accumulation in slot order j.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) unpermute_kernel(const float4* __restrict__ y,
                                                        const int32_t* __restrict__ row_of_pair,
                                                        const float* __restrict__ w, int k,
                                                        int P, int H8, float scale,
                                                        const float4* __restrict__ addend,
                                                        uint4* __restrict__ out, int cblocks) {
  // one block per (token, 128 groups of 8 columns): a flat grid, so T is not
  // bound by the 65535 limit of a grid's y extent
  const int t = static_cast<int>(blockIdx.x / cblocks);
  const int c = static_cast<int>(blockIdx.x % cblocks) * blockDim.x + threadIdx.x;  // 8-column group
  if (c >= H8) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  const int64_t pbase = static_cast<int64_t>(t) * k;
  // slots in groups of 8: all row indices, then all loads, then the FMAs in
  // slot order, so each thread keeps 16 independent 16-byte loads in flight
  for (int j0 = 0; j0 < k; j0 += 8) {
    int rows[8];
    float wts[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = j0 + j < k;
      const int r = in ? __ldg(row_of_pair + pbase + j0 + j) : -1;
      rows[j] = (r >= 0 && r < P) ? r : -1;
      wts[j] = in ? __ldg(w + pbase + j0 + j) : 0.0f;
    }
    float4 va[8], vb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (rows[j] >= 0) {
        const float4* src = y + (static_cast<int64_t>(rows[j]) * H8 + c) * 2;
        va[j] = __ldg(src);
        vb[j] = __ldg(src + 1);
      } else {
        va[j] = vb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        wts[j] = 0.0f;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j0 + j >= k) break;
      if (rows[j] < 0) continue;
      const float wt = wts[j];
      acc[0] = fmaf(wt, va[j].x, acc[0]);
      acc[1] = fmaf(wt, va[j].y, acc[1]);
      acc[2] = fmaf(wt, va[j].z, acc[2]);
      acc[3] = fmaf(wt, va[j].w, acc[3]);
      acc[4] = fmaf(wt, vb[j].x, acc[4]);
      acc[5] = fmaf(wt, vb[j].y, acc[5]);
      acc[6] = fmaf(wt, vb[j].z, acc[6]);
      acc[7] = fmaf(wt, vb[j].w, acc[7]);
    }
  }
  float v[8];
  if (addend != nullptr) {
    const float4* ad = addend + (static_cast<int64_t>(t) * H8 + c) * 2;
    const float4 a = __ldg(ad), b = __ldg(ad + 1);
    const float add[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf(scale, acc[i], add[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = scale * acc[i];
  }
  out[static_cast<int64_t>(t) * H8 + c] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                     pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

cudaError_t launch_unpermute(const float* y, const int32_t* row_of_pair, const float* weights,
                             int T, int k, int H, float scale, const float* addend, void* out,
                             cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int H8 = H / 8;
  const int cblocks = (H8 + 127) / 128;
  const long long blocks = static_cast<long long>(T) * cblocks;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  unpermute_kernel<<<static_cast<unsigned>(blocks), 128, 0, stream>>>(
      reinterpret_cast<const float4*>(y), row_of_pair, weights, k, T * k, H8, scale,
      reinterpret_cast<const float4*>(addend), static_cast<uint4*>(out), cblocks);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// a7 from the down GEMM's f16e rows (f16e.cuh): y = y16 * 2^e with one int8
// exponent per row and 128-column block. Each row is decoded to its fp32
// value (exact) before the same fp32 sums in slot order as above; the row
// reads are 16 bytes per 8 columns instead of 32.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) unpermute_f16e_kernel(
    const uint4* __restrict__ y16, const int8_t* __restrict__ y_exp,
    const int32_t* __restrict__ row_of_pair, const float* __restrict__ w, int k, int P, int H8,
    float scale, const float4* __restrict__ addend, uint4* __restrict__ out, int cblocks) {
  const int t = static_cast<int>(blockIdx.x / cblocks);
  const int c = static_cast<int>(blockIdx.x % cblocks) * blockDim.x + threadIdx.x;  // 8-column group
  if (c >= H8) return;
  const int HB = H8 / 16;  // 128-column blocks per row
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  const int64_t pbase = static_cast<int64_t>(t) * k;
  for (int j0 = 0; j0 < k; j0 += 8) {
    int rows[8];
    float wts[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = j0 + j < k;
      const int r = in ? __ldg(row_of_pair + pbase + j0 + j) : -1;
      rows[j] = (r >= 0 && r < P) ? r : -1;
      wts[j] = in ? __ldg(w + pbase + j0 + j) : 0.0f;
    }
    uint4 va[8];
    int ex[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (rows[j] >= 0) {
        va[j] = __ldg(y16 + static_cast<int64_t>(rows[j]) * H8 + c);
        ex[j] = __ldg(y_exp + static_cast<int64_t>(rows[j]) * HB + (c >> 4));
      } else {
        va[j] = make_uint4(0u, 0u, 0u, 0u);
        ex[j] = 0;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j0 + j >= k) break;
      if (rows[j] < 0) continue;
      const float s2 = f16e_pow2(ex[j]);
      const uint32_t wd[4] = {va[j].x, va[j].y, va[j].z, va[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[q]));
        acc[2 * q] = fmaf(wts[j], f.x * s2, acc[2 * q]);
        acc[2 * q + 1] = fmaf(wts[j], f.y * s2, acc[2 * q + 1]);
      }
    }
  }
  float v[8];
  if (addend != nullptr) {
    const float4* ad = addend + (static_cast<int64_t>(t) * H8 + c) * 2;
    const float4 a = __ldg(ad), b = __ldg(ad + 1);
    const float add[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf(scale, acc[i], add[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = scale * acc[i];
  }
  out[static_cast<int64_t>(t) * H8 + c] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                     pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// The same for k <= 8 as a persistent grid (8 blocks per SM) that walks its
// (token, 128-column block) items in order and loads the next item's row
// indices and weights while the current item's rows are in flight, so the
// two dependent loads of an item (indices, then rows) do not add up. Same
// arithmetic in the same order: results are identical.
template <bool kAddend>
__global__ void __launch_bounds__(128, 8) unpermute_f16e_pipe_kernel(
    const uint4* __restrict__ y16, const int8_t* __restrict__ y_exp,
    const int32_t* __restrict__ row_of_pair, const float* __restrict__ w, int k, int P, int H8,
    float scale, const float4* __restrict__ addend, uint4* __restrict__ out, int cblocks,
    long long items) {
  const int HB = H8 / 16;
  int nrows[8];
  float nwts[8];
  auto load_idx = [&](long long item) {
    const int64_t pbase = (item / cblocks) * k;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = j < k;
      const int r = in ? __ldg(row_of_pair + pbase + j) : -1;
      nrows[j] = (r >= 0 && r < P) ? r : -1;
      nwts[j] = in ? __ldg(w + pbase + j) : 0.0f;
    }
  };
  long long item = blockIdx.x;
  if (item < items) load_idx(item);
  for (; item < items; item += gridDim.x) {
    int rows[8];
    float wts[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rows[j] = nrows[j];
      wts[j] = nwts[j];
    }
    const int64_t t = item / cblocks;
    const int c = static_cast<int>(item - t * cblocks) * blockDim.x + threadIdx.x;
    const bool col = c < H8;
    uint4 va[8];
    int ex[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (col && rows[j] >= 0) {
        va[j] = __ldg(y16 + static_cast<int64_t>(rows[j]) * H8 + c);
        ex[j] = __ldg(y_exp + static_cast<int64_t>(rows[j]) * HB + (c >> 4));
      } else {
        va[j] = make_uint4(0u, 0u, 0u, 0u);
        ex[j] = 0;
      }
    }
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (kAddend && col) {
      const float4* ad = addend + (t * H8 + c) * 2;
      a = __ldg(ad);
      b = __ldg(ad + 1);
    }
    if (item + gridDim.x < items) load_idx(item + gridDim.x);
    if (!col) continue;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= k) break;
      if (rows[j] < 0) continue;
      const float s2 = f16e_pow2(ex[j]);
      const uint32_t wd[4] = {va[j].x, va[j].y, va[j].z, va[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[q]));
        acc[2 * q] = fmaf(wts[j], f.x * s2, acc[2 * q]);
        acc[2 * q + 1] = fmaf(wts[j], f.y * s2, acc[2 * q + 1]);
      }
    }
    float v[8];
    if constexpr (kAddend) {
      const float add[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = fmaf(scale, acc[i], add[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = scale * acc[i];
    }
    out[t * H8 + c] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                 pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
}

cudaError_t launch_unpermute_f16e(const void* y16, const int8_t* y_exp, const int32_t* row_of_pair,
                                  const float* weights, int T, int k, int H, float scale,
                                  const float* addend, void* out, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int H8 = H / 8;
  const int cblocks = (H8 + 127) / 128;
  const long long blocks = static_cast<long long>(T) * cblocks;
  if (k <= 8) {
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    const unsigned grid = static_cast<unsigned>(blocks < cap ? blocks : cap);
    const float4* ad = reinterpret_cast<const float4*>(addend);
    if (addend != nullptr)
      unpermute_f16e_pipe_kernel<true><<<grid, 128, 0, stream>>>(
          static_cast<const uint4*>(y16), y_exp, row_of_pair, weights, k, T * k, H8, scale, ad,
          static_cast<uint4*>(out), cblocks, blocks);
    else
      unpermute_f16e_pipe_kernel<false><<<grid, 128, 0, stream>>>(
          static_cast<const uint4*>(y16), y_exp, row_of_pair, weights, k, T * k, H8, scale, ad,
          static_cast<uint4*>(out), cblocks, blocks);
    return cudaGetLastError();
  }
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  unpermute_f16e_kernel<<<static_cast<unsigned>(blocks), 128, 0, stream>>>(
      static_cast<const uint4*>(y16), y_exp, row_of_pair, weights, k, T * k, H8, scale,
      reinterpret_cast<const float4*>(addend), static_cast<uint4*>(out), cblocks);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Combine of weighted rows (the unpermute's gather-reduce once the routing
// weight and scale were applied in the down GEMM's epilogue; TileOPs PR #1580,
// Unpermute, with the weight fold of the down projection's row scale):
//   out[t] = bf16( sum_{j<k} y_w[t*k+j] + addend[t] )
// y_w bf16 or fp32 [T*k, H] in flat pair order; pairs without a row
// (row_of_pair -1) contribute nothing. fp32 sums in slot order j, then the
// addend: the result does not depend on scheduling. One thread per 8 columns
// of one token.
// ---------------------------------------------------------------------------
template <bool kF32>
__global__ void __launch_bounds__(128) combine_kernel(const uint4* __restrict__ y_w,
                                                      const int32_t* __restrict__ row_of_pair,
                                                      int k, int H8,
                                                      const float4* __restrict__ addend,
                                                      uint4* __restrict__ out, int cblocks) {
  constexpr int kVec = kF32 ? 2 : 1;  // 16-byte vectors per 8 columns
  const int t = static_cast<int>(blockIdx.x / cblocks);
  const int c = static_cast<int>(blockIdx.x % cblocks) * blockDim.x + threadIdx.x;
  if (c >= H8) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  const int64_t pbase = static_cast<int64_t>(t) * k;
  for (int j0 = 0; j0 < k; j0 += 8) {
    // all row checks, then all loads, then the adds in slot order: up to 8
    // independent 16-byte loads in flight per thread
    bool has[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) has[j] = j0 + j < k && __ldg(row_of_pair + pbase + j0 + j) >= 0;
    uint4 v[8][kVec];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int u = 0; u < kVec; ++u)
        v[j][u] = has[j] ? __ldg(y_w + ((pbase + j0 + j) * H8 + c) * kVec + u)
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (!has[j]) continue;
      if constexpr (kF32) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          acc[4 * u + 0] += __uint_as_float(v[j][u].x);
          acc[4 * u + 1] += __uint_as_float(v[j][u].y);
          acc[4 * u + 2] += __uint_as_float(v[j][u].z);
          acc[4 * u + 3] += __uint_as_float(v[j][u].w);
        }
      } else {
        const uint32_t w4[4] = {v[j][0].x, v[j][0].y, v[j][0].z, v[j][0].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] += bf16lo_to_f32(w4[q]);
          acc[2 * q + 1] += bf16hi_to_f32(w4[q]);
        }
      }
    }
  }
  if (addend != nullptr) {
    const float4* ad = addend + (static_cast<int64_t>(t) * H8 + c) * 2;
    const float4 a = __ldg(ad), b = __ldg(ad + 1);
    const float add[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += add[i];
  }
  out[static_cast<int64_t>(t) * H8 + c] =
      make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                 pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

cudaError_t launch_combine(const void* y_w, bool y_f32, const int32_t* row_of_pair, int T, int k,
                           int H, const float* addend, void* out, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int H8 = H / 8;
  const int cblocks = (H8 + 127) / 128;
  const long long blocks = static_cast<long long>(T) * cblocks;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  auto kern = y_f32 ? combine_kernel<true> : combine_kernel<false>;
  kern<<<static_cast<unsigned>(blocks), 128, 0, stream>>>(
      static_cast<const uint4*>(y_w), row_of_pair, k, H8, reinterpret_cast<const float4*>(addend),
      static_cast<uint4*>(out), cblocks);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// a5 standalone: h = SiLU(gate) * up (XTuner PR #2089, Changes), stored as
// bf16, or quantised per row and 128-column tile: s = amax/448,
// q = e4m3_rn_satfinite(h/s), s = 0 and q = 0 for an all-zero tile. One warp
// per (row, tile), 4 columns per lane.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) swiglu_quant_kernel(int M, int F,
                                                           const __nv_bfloat16* __restrict__ gu,
                                                           const float* __restrict__ hin,
                                                           int out_fp8, void* __restrict__ out,
                                                           float* __restrict__ scales) {
  const int ntiles = (F + 127) / 128;
  const long long gw = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(M) * ntiles) return;
  const int r = static_cast<int>(gw / ntiles);
  const int tile = static_cast<int>(gw - static_cast<long long>(r) * ntiles);
  const int col = tile * 128 + lane * 4;
  const bool active = col < F;  // F % 4 == 0: all four columns valid or none
  float h[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (active) {
    if (gu != nullptr) {
      const uint2 gv = *reinterpret_cast<const uint2*>(gu + static_cast<int64_t>(r) * 2 * F + col);
      const uint2 uv =
          *reinterpret_cast<const uint2*>(gu + static_cast<int64_t>(r) * 2 * F + F + col);
      const float g[4] = {bf16lo_to_f32(gv.x), bf16hi_to_f32(gv.x), bf16lo_to_f32(gv.y),
                          bf16hi_to_f32(gv.y)};
      const float u[4] = {bf16lo_to_f32(uv.x), bf16hi_to_f32(uv.x), bf16lo_to_f32(uv.y),
                          bf16hi_to_f32(uv.y)};
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = g[i] / (1.0f + expf(-g[i])) * u[i];
    } else {
      const float4 v = *reinterpret_cast<const float4*>(hin + static_cast<int64_t>(r) * F + col);
      h[0] = v.x;
      h[1] = v.y;
      h[2] = v.z;
      h[3] = v.w;
    }
  }
  if (!out_fp8) {
    if (active) {
      uint2 o = make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + static_cast<int64_t>(r) * F +
                                col) = o;
    }
    return;
  }
  float amax = fmaxf(fmaxf(fabsf(h[0]), fabsf(h[1])), fmaxf(fabsf(h[2]), fabsf(h[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax / 448.0f;
  if (active) {
    uint32_t code = 0;
    if (amax > 0.0f)
      code = static_cast<uint32_t>(cvt_e4m3x2(h[0] / s, h[1] / s)) |
             (static_cast<uint32_t>(cvt_e4m3x2(h[2] / s, h[3] / s)) << 16);
    *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + static_cast<int64_t>(r) * F + col) =
        code;
  }
  if (lane == 0) scales[static_cast<int64_t>(r) * ntiles + tile] = amax > 0.0f ? s : 0.0f;
}

cudaError_t launch_swiglu_quant(int M, int F, const void* gate_up, const float* h, int out_fp8,
                                void* out, float* scales, cudaStream_t stream) {
  if (M <= 0 || F <= 0) return cudaSuccess;
  const long long warps = static_cast<long long>(M) * ((F + 127) / 128);
  const long long blocks = (warps + 7) / 8;
  swiglu_quant_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      M, F, static_cast<const __nv_bfloat16*>(gate_up), h, out_fp8, out, scales);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 128x128 block quantisation of weights w [batch, N, K] (bf16) to E4M3 codes
// and fp32 block scales. One CTA per block; thread i handles row i/2,
// columns (i%2)*64 .. +64.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint4* __restrict__ w, int N,
                                                           int K, uint8_t* __restrict__ q,
                                                           float* __restrict__ scales) {
  const int kb = blockIdx.x, nb = blockIdx.y, b = blockIdx.z;
  const int nbk = K / 128, nbn = N / 128;
  const int tid = threadIdx.x;
  const int r = nb * 128 + (tid >> 1);
  const int c0 = kb * 128 + (tid & 1) * 64;
  const int64_t base = (static_cast<int64_t>(b) * N + r) * K + c0;  // element index
  const uint4* src = w + base / 8;
  float v[64];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 x = __ldg(src + i);
    const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16lo_to_f32(u[j]);
      v[8 * i + 2 * j + 1] = bf16hi_to_f32(u[j]);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float s_max[8];
  if ((tid & 31) == 0) s_max[tid >> 5] = amax;
  __syncthreads();
  amax = s_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, s_max[i]);
  const float s = amax / 448.0f;
  uint4* dst = reinterpret_cast<uint4*>(q + base);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t wd[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float* x = v + 16 * i + 4 * j;
      wd[j] = amax > 0.0f ? (static_cast<uint32_t>(cvt_e4m3x2(x[0] / s, x[1] / s)) |
                             (static_cast<uint32_t>(cvt_e4m3x2(x[2] / s, x[3] / s)) << 16))
                          : 0u;
    }
    dst[i] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
  }
  if (tid == 0)
    scales[(static_cast<int64_t>(b) * nbn + nb) * nbk + kb] = amax > 0.0f ? s : 0.0f;
}

cudaError_t launch_quantize_weight(int batch, int N, int K, const void* w, uint8_t* q,
                                   float* scales, cudaStream_t stream) {
  if (batch <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  dim3 grid(K / 128, N / 128, batch);
  quant_weight_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(w), N, K, q, scales);
  return cudaGetLastError();
}

}  // namespace moe
