// route_permute.cu - a1 top-k routing and a3 the permute gather (a2, the
// dispatch tables, is in tables.cu).
//
// Built with --fmad=false: the routing weights use only explicitly rounded
// float32 operations (__fmul_rn / __fadd_rn / __fsub_rn / __fdiv_rn), so they
// are reproducible bit for bit.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "internal.h"
#include "status.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// a1: routing
// ---------------------------------------------------------------------------

// exp(x) in float32 (Cody & Waite, "Software Manual for the Elementary
// Functions", 1980, range reduction; Taylor polynomial of degree 7):
//   n = rint(x * log2 e); r = (x - n*ln2_hi) - n*ln2_lo, ln2_hi = 355/512
//   (exact product for |n| < 2^15); p = sum_{i<=7} r^i / i! by Horner;
//   result = (p * 2^(n - floor(n/2))) * 2^floor(n/2): the first product is
//   exact, the second is the single final rounding (also into subnormals).
// The argument is clamped to [-104, 89] first (exp underflows to 0 below and
// overflows to +inf above). NaN inputs are outside the supported domain.
__device__ __forceinline__ float moe_expf(float x) {
  const float kLog2e = 0x1.715476p+0f;
  const float kLn2Hi = 0x1.630000p-1f;  // 0.693359375
  const float kLn2Lo = -0x1.bd0106p-13f;
  x = fminf(fmaxf(x, -104.0f), 89.0f);
  const float n = rintf(__fmul_rn(x, kLog2e));
  float r = __fsub_rn(x, __fmul_rn(n, kLn2Hi));
  r = __fsub_rn(r, __fmul_rn(n, kLn2Lo));
  float p = 0x1.a01a02p-13f;                     // 1/7!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.6c16c2p-10f);  // 1/6!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.111112p-7f);   // 1/5!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-5f);   // 1/4!
  p = __fadd_rn(__fmul_rn(p, r), 0x1.555556p-3f);   // 1/3!
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);             // 1/2!
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);             // 1/1!
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);             // 1/0!
  const int ni = static_cast<int>(n);
  const int lo = ni >> 1;  // floor(n/2)
  const int hi = ni - lo;
  const float s_hi = __int_as_float((hi + 127) << 23);
  const float s_lo = __int_as_float((lo + 127) << 23);
  return __fmul_rn(__fmul_rn(p, s_hi), s_lo);
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// One warp per token: k rounds of a warp-wide arg-max over the not yet taken
// experts (largest logit, then lowest index), then the weights.
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T,
                                                         int E, int k, int score_fn,
                                                         int renormalize, int32_t* __restrict__ ids,
                                                         float* __restrict__ weights) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* row = logits + static_cast<int64_t>(t) * E;
  uint32_t taken = 0;  // bit i: expert lane + 32*i already picked (E <= 1024)
  float my_val = 0.0f;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    for (int i = 0, e = lane; e < E; ++i, e += 32) {
      if ((taken >> i) & 1u) continue;
      const float v = __ldg(row + e);
      if (better(v, e, bv, bi)) {
        bv = v;
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= 0 && bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      my_val = bv;
      my_idx = bi;
    }
  }
  const float top = __shfl_sync(0xffffffffu, my_val, 0);
  float w = 0.0f;
  if (score_fn == 0) {
    const float ev = moe_expf(__fsub_rn(my_val, top));
    float den = 0.0f;
    if (renormalize) {
      for (int j = 0; j < k; ++j) den = __fadd_rn(den, __shfl_sync(0xffffffffu, ev, j));
    } else {
      if (lane == 0)
        for (int e = 0; e < E; ++e) den = __fadd_rn(den, moe_expf(__fsub_rn(__ldg(row + e), top)));
      den = __shfl_sync(0xffffffffu, den, 0);
    }
    w = __fdiv_rn(ev, den);
  } else {
    const float sv = __fdiv_rn(1.0f, __fadd_rn(1.0f, moe_expf(-my_val)));
    if (renormalize) {
      float den = 0.0f;
      for (int j = 0; j < k; ++j) den = __fadd_rn(den, __shfl_sync(0xffffffffu, sv, j));
      w = __fdiv_rn(sv, den);
    } else {
      w = sv;
    }
  }
  if (lane < k) {
    ids[static_cast<int64_t>(t) * k + lane] = my_idx;
    weights[static_cast<int64_t>(t) * k + lane] = w;
  }
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int score_fn,
                              int renormalize, int32_t* ids, float* weights, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int warps = 8;
  route_topk_kernel<<<(T + warps - 1) / warps, warps * 32, 0, stream>>>(
      logits, T, E, k, score_fn, renormalize, ids, weights);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// a3: permute gather, x_perm[r] = hidden[pair_of_row[r] / k], 16-byte vectors
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ hidden,
                                                          const int32_t* __restrict__ pair_of_row,
                                                          int P, int k, int H8,
                                                          uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < P; r += warps_total) {
    const int p = __ldg(pair_of_row + r);
    if (p < 0 || p >= P) continue;
    const uint4* src = hidden + static_cast<int64_t>(p / k) * H8;
    uint4* dst = x_perm + static_cast<int64_t>(r) * H8;
    int c = lane;
    for (; c + 96 < H8; c += 128) {
      const uint4 a = __ldg(src + c), b = __ldg(src + c + 32), d = __ldg(src + c + 64),
                  e = __ldg(src + c + 96);
      dst[c] = a;
      dst[c + 32] = b;
      dst[c + 64] = d;
      dst[c + 96] = e;
    }
    for (; c < H8; c += 32) dst[c] = __ldg(src + c);
  }
}

cudaError_t launch_gather_rows(const void* hidden, const int32_t* pair_of_row, int P, int k,
                               int H, void* x_perm, cudaStream_t stream) {
  if (P <= 0) return cudaSuccess;
  const int H8 = H / 8;
  const int rows_per_block = 8;
  int blocks = (P + rows_per_block - 1) / rows_per_block;
  const int cap = device_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  gather_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(hidden), pair_of_row,
                                                 P, k, H8, static_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
