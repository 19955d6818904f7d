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

// Plain form: each CTA is persistent and streams its tiles (128 padded
// tokens x 128 columns) through a ring of NS shared-memory stages filled with
// cp.async, NS - 1 tiles ahead of the one it quantises, so the copies of the
// next tiles are in flight while a tile is encoded. Padding rows of an
// expert's last block are zero-filled by the copy. A stage row holds the
// tile's 128 bf16 values plus 16 bytes of padding; its 16-byte chunks are
// permuted (chunk_pos) so that the row-pass reads (4 threads per row, 16 bytes
// each) and the column-pass reads are free of bank conflicts. The rows and
// the block of each of the CTA's tiles are looked up once, before the loop.
struct DualCfg {
  static constexpr int NS = 3;
  static constexpr int ROW_BYTES = 272;
  static constexpr int IN_BYTES = 128 * ROW_BYTES;
  static constexpr int RED_BYTES = 512 * 8;  // per-tile column maxima: 2 slots x 4 x 64 float2
  static constexpr int META_TILES = 512;  // tiles per CTA with precomputed rows
  static constexpr int SMEM = NS * IN_BYTES + RED_BYTES + META_TILES * 8;
};

// SwiGLU form: one CTA per tile. The row pass writes its fp32 h into a shared
// tile of 128 rows of 528 bytes, 16-byte chunk k of row quarter qq at chunk
// qq*8 + (k ^ 2qq), which keeps both the row pass's 16-byte stores and the
// column pass's reads free of bank conflicts.
constexpr int kHRowBytes = 528;
constexpr int kSwigluSmem = 128 * kHRowBytes + 512 * 4;

// Position of 16-byte chunk L (0..15) of a staged 256-byte row: the second
// half's chunks are swapped in fours, so that the row pass (two threads per
// row, 16-byte reads) and the column pass (4-byte reads, a warp across 64
// columns of one row) are free of bank conflicts with rows 17 chunks apart.
__device__ __forceinline__ int chunk_pos(int L) { return L ^ ((L >> 1) & 4); }

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

// x / s rounded to nearest even for two values, given ns = -s and
// y = RN(1/s), with packed fp32x2 arithmetic (two lanes per instruction).
// q0 = RN(x*y) lies within 2 ulp of x/s; each correction
// q <- RN(q + y*(x - s*q)), the residual exact in one FMA, is Markstein's
// division step (P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): after the
// first q is within one ulp and the second gives the correctly rounded
// quotient, provided the residual does not underflow. With s >= 2^-90 it
// cannot wherever the quotient reaches 2^-11 (below that every value encodes
// to a signed zero in E4M3), so callers use this for s >= 2^-90 and plain
// division otherwise. The residual is rounded toward -infinity: an exact
// residual is unaffected, and for a zero x the residual is -0, which keeps
// the sign of q0 = x*y (+-0) through both steps.
__device__ __forceinline__ void div2(float xa, float xb, float ns, float y, float& qa, float& qb) {
  asm("{\n.reg .b64 x, q, r, s2, y2;\n"
      "mov.b64 x, {%2, %3};\n"
      "mov.b64 s2, {%4, %4};\n"
      "mov.b64 y2, {%5, %5};\n"
      "mul.rn.f32x2 q, x, y2;\n"
      "fma.rm.f32x2 r, q, s2, x;\n"
      "fma.rn.f32x2 q, r, y2, q;\n"
      "fma.rm.f32x2 r, q, s2, x;\n"
      "fma.rn.f32x2 q, r, y2, q;\n"
      "mov.b64 {%0, %1}, q;\n}"
      : "=f"(qa), "=f"(qb)
      : "f"(xa), "f"(xb), "f"(ns), "f"(y));
}

constexpr float kFastDivMinScale = 8.0779356e-28f;  // 2^-90

// N values get(0) .. get(N - 1) -> N E4M3 codes of x / s (all zero when
// amax == 0) as N / 4 words.
template <int N, class Get>
__device__ __forceinline__ void encode(Get get, float amax, float s, uint32_t* w) {
  if (amax > 0.0f && s >= kFastDivMinScale) {
    const float y = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < N / 4; ++j) {
      float q0, q1, q2, q3;
      div2(get(4 * j), get(4 * j + 1), -s, y, q0, q1);
      div2(get(4 * j + 2), get(4 * j + 3), -s, y, q2, q3);
      w[j] = cvt_e4m3x4(q0, q1, q2, q3);
    }
  } else if (amax > 0.0f) {
#pragma unroll
    for (int j = 0; j < N / 4; ++j)
      w[j] = cvt_e4m3x4(get(4 * j) / s, get(4 * j + 1) / s, get(4 * j + 2) / s, get(4 * j + 3) / s);
  } else {
#pragma unroll
    for (int j = 0; j < N / 4; ++j) w[j] = 0u;
  }
}

// Two lists of N values with their own scales, sharing one fast path.
template <int N, class GetA, class GetB>
__device__ __forceinline__ void encode2(GetA geta, float aa, float sa, GetB getb, float ab, float sb,
                                        uint32_t* wa, uint32_t* wb) {
  if (aa > 0.0f && ab > 0.0f && sa >= kFastDivMinScale && sb >= kFastDivMinScale) {
    const float ya = __frcp_rn(sa);
    const float yb = sa == sb ? ya : __frcp_rn(sb);
#pragma unroll
    for (int j = 0; j < N / 4; ++j) {
      float q0, q1, q2, q3;
      div2(geta(4 * j), geta(4 * j + 1), -sa, ya, q0, q1);
      div2(geta(4 * j + 2), geta(4 * j + 3), -sa, ya, q2, q3);
      wa[j] = cvt_e4m3x4(q0, q1, q2, q3);
      div2(getb(4 * j), getb(4 * j + 1), -sb, yb, q0, q1);
      div2(getb(4 * j + 2), getb(4 * j + 3), -sb, yb, q2, q3);
      wb[j] = cvt_e4m3x4(q0, q1, q2, q3);
    }
  } else {
    encode<N>(geta, aa, sa, wa);
    encode<N>(getb, ab, sb, wb);
  }
}

// Running maximum of |x| over packed bf16 pairs, the two lanes kept apart
// (max.xorsign.abs: the sign bits of the result carry no meaning).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t m, uint32_t w) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(w));
  return r;
}
// The same over n words (n a multiple of 4) in four independent chains.
template <int n>
__device__ __forceinline__ uint32_t absmax_tree(const uint32_t* w) {
  uint32_t m[4] = {w[0], w[1], w[2], w[3]};
#pragma unroll
  for (int k = 4; k < n; ++k) m[k & 3] = bf16x2_absmax(m[k & 3], w[k]);
  return bf16x2_absmax(bf16x2_absmax(m[0], m[1]), bf16x2_absmax(m[2], m[3]));
}
__device__ __forceinline__ float absmax_lo(uint32_t m) { return __uint_as_float((m << 16) & 0x7FFFFFFFu); }
__device__ __forceinline__ float absmax_hi(uint32_t m) { return __uint_as_float(m & 0x7FFF0000u); }

constexpr int kDualThreads = 512;

// Rows of x that 128-token block bx of the padded axis holds: m_start and the
// count (0 for a padding-only block, or when the tables are inconsistent).
__device__ __forceinline__ void dual_block_rows(const DualParams& p, int bx, int& m_start,
                                                int& rows) {
  m_start = 0;
  rows = 0;
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
  if (m_start < 0 || m_start + rows > p.M) rows = 0;
}

// Plain form, persistent: CTA b takes tiles b, b + G, b + 2G, ... (tile =
// bx * KB + kb of 128-token block bx and 128-column block kb); 256 threads,
// 64 values each per pass. Row pass: thread (row i = t/2, half h = t%2)
// takes the 64 values of its half row and writes their row-layout codes (the
// row's two threads share the 1x128 tile's amax). Column pass: thread
// (column pair cp = t%64, token quarter tq = t/64) takes columns 2cp and
// 2cp+1 for tokens tq*32 .. tq*32+31 (one 4-byte shared read per token) and
// writes each column's 32 codes to xT rows kb*128 + 2cp and + 1. The passes
// are software pipelined: between two barriers a thread runs the row pass of
// tile j + 1 and then the column pass of tile j. The 128x128 block amax
// (per-block scales) is the maximum of the row tiles' amax, reduced in the
// row pass into the tile's shared slot (three, by tile index mod 3).
constexpr int kPlainThreads = 256;

template <bool kTransBlock>
__global__ void __launch_bounds__(kPlainThreads, 2) quant_dual_kernel(const DualParams p) {
  using C = DualCfg;
  static_assert(C::NS == 3, "the pipelined loop below assumes three stages");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* red = reinterpret_cast<float*>(smem_raw + C::NS * C::IN_BYTES);
  uint2* meta = reinterpret_cast<uint2*>(smem_raw + C::NS * C::IN_BYTES + C::RED_BYTES);
  const int t = threadIdx.x;
  const int KB = p.K / 128;
  const int tiles = p.M_blk * KB;
  const int G = static_cast<int>(gridDim.x);
  const int b = static_cast<int>(blockIdx.x);
  const int n_my = b < tiles ? (tiles - 1 - b) / G + 1 : 0;

  // (m_start, bx | rows << 24) of the CTA's tile j
  auto tile_meta = [&](int j) -> uint2 {
    const int bx = (b + j * G) / KB;
    int m_start, rows;
    dual_block_rows(p, bx, m_start, rows);
    return make_uint2(static_cast<uint32_t>(m_start),
                      static_cast<uint32_t>(bx) | (static_cast<uint32_t>(rows) << 24));
  };
  for (int j = t; j < n_my && j < C::META_TILES; j += kPlainThreads) meta[j] = tile_meta(j);
  if (kTransBlock && t < 3) red[t] = 0.0f;  // block-amax slots
  __syncthreads();  // meta and the slots are read by every thread from here on
  auto get_meta = [&](int j) -> uint2 { return j < C::META_TILES ? meta[j] : tile_meta(j); };

  // Copies tile j into stage `stage` (one commit group per call, empty past
  // the CTA's last tile): thread t copies chunk t%16 of rows t/16 + 16k.
  const int L = t & 15;
  const int64_t ld = p.K;
  auto issue = [&](int j, int stage) {
    if (j < n_my) {
      const uint2 m = get_meta(j);
      const int bx = static_cast<int>(m.y & 0xFFFFFFu);
      const int rows = static_cast<int>(m.y >> 24);
      const int kb = b + j * G - bx * KB;
      const __nv_bfloat16* src0 =
          p.x + (static_cast<int64_t>(static_cast<int>(m.x)) + (t >> 4)) * ld + kb * 128 + L * 8;
      uint8_t* dst0 = smem_raw + stage * C::IN_BYTES + (t >> 4) * C::ROW_BYTES + chunk_pos(L) * 16;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool live = (t >> 4) + k * 16 < rows;
        cp_async16(dst0 + k * 16 * C::ROW_BYTES, live ? src0 + k * 16 * ld : p.x, live ? 16u : 0u);
      }
    }
    cp_async_commit();
  };

  const int i = t >> 1;  // row pass
  const int h = t & 1;
  auto row_pass = [&](int j, int stage) {
    const uint2 m = get_meta(j);
    const int bx = static_cast<int>(m.y & 0xFFFFFFu);
    const int rows = static_cast<int>(m.y >> 24);
    const int kb = b + j * G - bx * KB;
    const uint8_t* srow = smem_raw + stage * C::IN_BYTES + i * C::ROW_BYTES + h * 128;
    uint32_t w[32];  // bf16 pairs: columns h*64 + 2k, + 2k + 1
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {  // chunk_pos(h * 8 + jj) = h * 8 + (jj ^ 4h)
      const uint4 u = *reinterpret_cast<const uint4*>(srow + (jj ^ (h * 4)) * 16);
      w[4 * jj] = u.x;
      w[4 * jj + 1] = u.y;
      w[4 * jj + 2] = u.z;
      w[4 * jj + 3] = u.w;
    }
    const uint32_t mx = absmax_tree<32>(w);
    float amax = fmaxf(absmax_lo(mx), absmax_hi(mx));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    if (i < rows) {
      const float s = amax / 448.0f;
      const int64_t r = static_cast<int64_t>(static_cast<int>(m.x) + i);
      uint32_t codes[16];
      encode<64>([&](int k) { return k & 1 ? bf16hi_to_f32(w[k >> 1]) : bf16lo_to_f32(w[k >> 1]); },
                 amax, s, codes);
      uint4* dst = reinterpret_cast<uint4*>(p.q + r * ld + kb * 128 + h * 64);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        dst[k] = make_uint4(codes[4 * k], codes[4 * k + 1], codes[4 * k + 2], codes[4 * k + 3]);
      if (h == 0) p.s[r * KB + kb] = amax > 0.0f ? s : 0.0f;
    }
    if constexpr (kTransBlock) {
#pragma unroll
      for (int off = 16; off > 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      // non-negative floats order as their bit patterns
      if ((t & 31) == 0) atomicMax(reinterpret_cast<int*>(red) + stage, __float_as_int(amax));
    }
  };

  const int cp = t & 63;  // column pass
  const int tq = t >> 6;
  const int coff = chunk_pos(cp >> 2) * 16 + (cp & 3) * 4;
  const int64_t ldT = static_cast<int64_t>(p.M_blk) * 128;
  auto col_pass = [&](int j, int stage) {
    const uint2 m = get_meta(j);
    const int bx = static_cast<int>(m.y & 0xFFFFFFu);
    const int kb = b + j * G - bx * KB;
    const uint8_t* st = smem_raw + stage * C::IN_BYTES + tq * 32 * C::ROW_BYTES + coff;
    uint32_t wd[32];  // token tq*32 + r: (column 2cp, column 2cp + 1)
#pragma unroll
    for (int r = 0; r < 32; ++r) wd[r] = *reinterpret_cast<const uint32_t*>(st + r * C::ROW_BYTES);
    float a0, a1;
    if constexpr (kTransBlock) {
      a0 = a1 = red[stage];
      if (t == 0) red[stage == 0 ? 2 : stage - 1] = 0.0f;  // slot of tile j + 2
    } else {
      // the column maxima of this tile's four token quarters, left in slot
      // j & 1 by colmax_pass one barrier earlier
      const float2* slot = reinterpret_cast<const float2*>(red) + (j & 1) * 256;
      a0 = a1 = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 q2 = slot[k * 64 + cp];
        a0 = fmaxf(a0, q2.x);
        a1 = fmaxf(a1, q2.y);
      }
    }
    const float s0 = a0 / 448.0f;
    const float s1 = kTransBlock ? s0 : a1 / 448.0f;
    uint32_t c0[8], c1[8];
    encode2<32>([&](int r) { return bf16lo_to_f32(wd[r]); }, a0, s0,
                [&](int r) { return bf16hi_to_f32(wd[r]); }, a1, s1, c0, c1);
    uint4* dst = reinterpret_cast<uint4*>(p.qT + static_cast<int64_t>(kb * 128 + 2 * cp) * ldT +
                                          static_cast<int64_t>(bx) * 128 + tq * 32);
    dst[0] = make_uint4(c0[0], c0[1], c0[2], c0[3]);
    dst[1] = make_uint4(c0[4], c0[5], c0[6], c0[7]);
    uint4* dst1 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst) + ldT);
    dst1[0] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
    dst1[1] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
    if constexpr (kTransBlock) {
      if (t == 0) p.sT[static_cast<int64_t>(kb) * p.M_blk + bx] = a0 > 0.0f ? s0 : 0.0f;
    } else {
      if (tq == 0) {
        p.sT[static_cast<int64_t>(kb * 128 + 2 * cp) * p.M_blk + bx] = a0 > 0.0f ? s0 : 0.0f;
        p.sT[static_cast<int64_t>(kb * 128 + 2 * cp + 1) * p.M_blk + bx] = a1 > 0.0f ? s1 : 0.0f;
      }
    }
  };

  // Per-tile scales: each thread's maxima of columns 2cp, 2cp+1 over its 32
  // tokens of tile j, into slot j & 1, one barrier before tile j's column
  // pass reads the four token quarters' values.
  auto colmax_pass = [&](int j, int stage) {
    const uint8_t* st = smem_raw + stage * C::IN_BYTES + tq * 32 * C::ROW_BYTES + coff;
    uint32_t wd[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) wd[r] = *reinterpret_cast<const uint32_t*>(st + r * C::ROW_BYTES);
    const uint32_t mx = absmax_tree<32>(wd);
    reinterpret_cast<float2*>(red)[(j & 1) * 256 + tq * 64 + cp] =
        make_float2(absmax_lo(mx), absmax_hi(mx));
  };

  issue(0, 0);
  issue(1, 1);
  cp_async_wait<1>();  // tile 0 has landed
  __syncthreads();
  if (n_my > 0) {
    row_pass(0, 0);
    if constexpr (!kTransBlock) colmax_pass(0, 0);
  }
  int stage = 0;  // stage (and block-amax slot) of tile j: j mod 3
  for (int j = 0; j + 1 < n_my; ++j) {
    cp_async_wait<0>();  // tile j + 1 has landed
    __syncthreads();     // row pass j and column pass j - 1 are done everywhere
    const int s1 = stage == 2 ? 0 : stage + 1;
    const int s2 = s1 == 2 ? 0 : s1 + 1;
    issue(j + 2, s2);  // into the stage column pass j - 1 released
    row_pass(j + 1, s1);
    if constexpr (!kTransBlock) colmax_pass(j + 1, s1);
    col_pass(j, stage);
    stage = s1;
  }
  if (n_my > 0) {  // the last tile's column pass
    cp_async_wait<0>();
    __syncthreads();
    col_pass(n_my - 1, stage);
  }
  cp_async_wait<0>();
}

// SwiGLU form: one CTA per (128-token block bx, 128-column block kb) of h =
// SiLU(gate) * up; the same two passes, the row pass reading gate and up from
// global memory and staging h (fp32) for the column pass. SiLU(g) is
// g / (1 + e^-g) with the hardware exponential and reciprocal (h is checked
// against the oracle's float64 SwiGLU within 1e-5 relative; every code is
// exact for the h the kernel computed).
template <bool kTransBlock>
__global__ void __launch_bounds__(kDualThreads, 2) swiglu_quant_dual_kernel(const DualParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* red = reinterpret_cast<float*>(smem_raw + 128 * kHRowBytes);
  const int bx = blockIdx.x;
  const int kb = blockIdx.y;
  const int t = threadIdx.x;
  int m_start, rows;
  dual_block_rows(p, bx, m_start, rows);
  const int KB = p.K / 128;

  // ---------------------------------------------------------------- row pass
  {
    const int i = t >> 2;
    const int qq = t & 3;
    const int col = kb * 128 + qq * 32;
    float v[32];
    const bool live = i < rows;
    if (live) {
      const int64_t r = static_cast<int64_t>(m_start + i);
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
        for (int e = 0; e < 8; ++e) v[8 * j + e] = __fdividef(g[e], 1.0f + __expf(-g[e])) * u[e];
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (live) {
      const float s = amax / 448.0f;
      const int64_t r = static_cast<int64_t>(m_start + i);
      uint32_t codes[8];
      encode<32>([&](int k) { return v[k]; }, amax, s, codes);
      uint4* dst = reinterpret_cast<uint4*>(p.q + r * p.K + col);
      dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
      dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
      if (qq == 0) p.s[r * KB + kb] = amax > 0.0f ? s : 0.0f;
      if (p.debug_h != nullptr) {
        float4* hd = reinterpret_cast<float4*>(p.debug_h + r * p.K + col);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          hd[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
    }
    uint8_t* hrow = smem_raw + i * kHRowBytes;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<float4*>(hrow + (qq * 8 + (k ^ (2 * qq))) * 16) =
          make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    if constexpr (kTransBlock) {
#pragma unroll
      for (int off = 16; off > 2; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if ((t & 31) == 0) red[t >> 5] = amax;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------- column pass
  const int c = t & 127;
  const int tq = t >> 7;
  const int hoff = ((c >> 5) * 8 + (((c >> 2) & 7) ^ ((c >> 5) * 2))) * 16 + (c & 3) * 4;
  float w[32];
#pragma unroll
  for (int r = 0; r < 32; ++r)
    w[r] = *reinterpret_cast<const float*>(smem_raw + (tq * 32 + r) * kHRowBytes + hoff);
  float amax;
  if constexpr (kTransBlock) {
    amax = red[t & 15];
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  } else {
    amax = 0.0f;
#pragma unroll
    for (int r = 0; r < 32; ++r) amax = fmaxf(amax, fabsf(w[r]));
    red[t] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[c], red[c + 128]), fmaxf(red[c + 256], red[c + 384]));
  }
  const float s = amax / 448.0f;
  uint32_t codes[8];
  encode<32>([&](int k) { return w[k]; }, amax, s, codes);
  const int64_t ldT = static_cast<int64_t>(p.M_blk) * 128;
  uint4* dst = reinterpret_cast<uint4*>(p.qT + static_cast<int64_t>(kb * 128 + c) * ldT +
                                        static_cast<int64_t>(bx) * 128 + tq * 32);
  dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
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

template <bool kTransBlock>
cudaError_t run_dual(const DualParams& p, cudaStream_t stream) {
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int ctas = 2;
  if (dev >= 0 && dev < 64) {
    if (per_sm[dev] == 0) {
      cudaError_t e = cudaFuncSetAttribute(quant_dual_kernel<kTransBlock>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, DualCfg::SMEM);
      if (e != cudaSuccess) return e;
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quant_dual_kernel<kTransBlock>,
                                                        kPlainThreads, DualCfg::SMEM);
      if (e != cudaSuccess) return e;
      per_sm[dev] = n > 0 ? n : 1;
    }
    ctas = per_sm[dev];
  }
  const long long tiles = static_cast<long long>(p.M_blk) * (p.K / 128);
  const long long cap = static_cast<long long>(device_sm_count()) * ctas;
  const unsigned grid = static_cast<unsigned>(tiles < cap ? tiles : cap);
  quant_dual_kernel<kTransBlock><<<grid, kPlainThreads, DualCfg::SMEM, stream>>>(p);
  return cudaGetLastError();
}

template <bool kTransBlock>
cudaError_t run_swiglu_dual(const DualParams& p, cudaStream_t stream) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(swiglu_quant_dual_kernel<kTransBlock>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSwigluSmem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const dim3 grid(static_cast<unsigned>(p.M_blk), static_cast<unsigned>(p.K / 128));
  swiglu_quant_dual_kernel<kTransBlock><<<grid, kDualThreads, kSwigluSmem, stream>>>(p);
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
    return L.trans_block ? run_swiglu_dual<true>(p, stream) : run_swiglu_dual<false>(p, stream);
  return L.trans_block ? run_dual<true>(p, stream) : run_dual<false>(p, stream);
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
