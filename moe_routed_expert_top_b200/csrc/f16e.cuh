// f16e.cuh - a block floating-point format for the down GEMM's output rows:
// fp16 values with one int8 power-of-two exponent per row and 128-column block,
//   y[r, c] = C16[r, c] * 2^e[r, c / 128].
// The exponent puts the block's largest magnitude in [2^14, 2^15), so every
// value keeps fp16's 11 significant bits relative to itself (values more than
// 2^28 below the block maximum become fp16 subnormals or zero) while the block
// may hold any fp32 range. Encoding scales by an exact power of two and rounds
// once to fp16 (to nearest even); decoding is exact. Half the bytes of fp32,
// with 8x the precision of bf16.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace moe {

constexpr int kF16eMinExp = -100;  // keeps 2^-e a normal fp32 for tiny blocks

// Exponent of a block whose largest magnitude is amax (0 for an all-zero block).
__device__ __forceinline__ int f16e_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const int e2 = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127;  // floor(log2)
  const int e = (e2 < -126 ? -126 : e2) - 14;  // subnormal amax: treated as 2^-126
  return e < kF16eMinExp ? kF16eMinExp : e;
}

// 2^x as an fp32, for x in [-126, 127].
__device__ __forceinline__ float f16e_pow2(int x) {
  return __uint_as_float(static_cast<uint32_t>(x + 127) << 23);
}

// Encodes NP rows' blocks at once (the NP row passes of a slab). Each row's
// 128-column block is spread over 16 consecutive lanes of a half warp, 8
// columns each (v[q]: this lane's 8 values of pass q); every lane of the warp
// must call this. Returns each block's exponent (the same in its 16 lanes)
// and this lane's 8 fp16 codes per pass. The NP half-warp reductions are
// interleaved so that their shuffle latencies overlap.
template <int NP>
__device__ __forceinline__ void f16e_encode8xn(const float (&v)[NP][8], uint4 (&out)[NP],
                                               int (&e)[NP]) {
  float amax[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    amax[q] = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax[q] = fmaxf(amax[q], fabsf(v[q][i]));
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
    for (int q = 0; q < NP; ++q)
      amax[q] = fmaxf(amax[q], __shfl_xor_sync(0xffffffffu, amax[q], off));
  }
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    e[q] = f16e_exponent(amax[q]);
    const float s = f16e_pow2(-e[q]);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = __floats2half2_rn(v[q][2 * i] * s, v[q][2 * i + 1] * s);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    out[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace moe
