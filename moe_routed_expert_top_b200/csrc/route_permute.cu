// route_permute.cu - a1 top-k routing, a2 dispatch tables + stable
// permutation, a3 permute gather.
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
// a2: histogram + stable scan -> tables and permutation (one CTA, no host sync)
// ---------------------------------------------------------------------------
// The P pairs are cut into 32 contiguous segments, one per warp. Pass 1: each
// warp counts its segment per expert (32 pairs at a time; __match_any_sync
// groups equal ids, the group's lowest lane adds the group size). A per-expert
// scan over the 32 warp counts and a block scan over experts give every
// (warp, expert) its first row. Pass 2: each warp walks its segment again in
// order; a pair's row is its (warp, expert) base plus the number of earlier
// lanes in its match group. Rows therefore follow flat pair order inside each
// expert (a stable sort by expert).

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

__global__ void __launch_bounds__(1024) tables_kernel(
    const int32_t* __restrict__ ids, int P, int E, int pad, int M_blk, int32_t* __restrict__ sizes,
    int32_t* __restrict__ offsets, int32_t* __restrict__ padded, int32_t* __restrict__ idx_for_bx,
    int32_t* __restrict__ row_of_pair, int32_t* __restrict__ pair_of_row,
    int32_t* __restrict__ status) {
  extern __shared__ int smem[];
  int* hist = smem;                  // [32][E]: per-warp counts, then bases
  int* s_off = hist + 32 * E;        // [E + 1]
  int* s_pad = s_off + E + 1;        // [E + 1]
  int* s_tot = s_pad + E + 1;        // [2][32] warp totals of the two scans
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  for (int i = tid; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  const int seg = (P + 31) / 32;
  const int beg = warp * seg;
  const int end = min(P, beg + seg);
  bool bad = false;
  for (int base = beg; base < end; base += 32) {
    const int p = base + lane;
    int id = -1;
    if (p < end) {
      id = __ldg(ids + p);
      if (id < 0 || id >= E) {
        bad = true;
        id = -1;
      }
    }
    const unsigned mask = __match_any_sync(0xffffffffu, id);
    if (id >= 0 && lane == __ffs(mask) - 1) hist[warp * E + id] += __popc(mask);
    __syncwarp();
  }
  if (bad) atomicOr(status, MOE_DEV_BAD_EXPERT_ID_FLAG);
  __syncthreads();

  // per expert: exclusive scan over warps (in place), total size
  int size = 0;
  if (tid < E) {
    for (int w = 0; w < 32; ++w) {
      const int c = hist[w * E + tid];
      hist[w * E + tid] = size;
      size += c;
    }
  }
  const int padsz = (size + pad - 1) / pad * pad;
  // block exclusive scans of size and padded size over experts (E <= 1024)
  const int inc_s = warp_incl_scan(size, lane);
  const int inc_p = warp_incl_scan(padsz, lane);
  if (lane == 31) {
    s_tot[warp] = inc_s;
    s_tot[32 + warp] = inc_p;
  }
  __syncthreads();
  if (warp == 0) {
    const int a = warp_incl_scan(s_tot[lane], lane);
    const int b = warp_incl_scan(s_tot[32 + lane], lane);
    __syncwarp();
    s_tot[lane] = a;
    s_tot[32 + lane] = b;
  }
  __syncthreads();
  const int ex_s = inc_s - size + (warp > 0 ? s_tot[warp - 1] : 0);
  const int ex_p = inc_p - padsz + (warp > 0 ? s_tot[32 + warp - 1] : 0);
  if (tid < E) {
    s_off[tid] = ex_s;
    s_pad[tid] = ex_p;
    sizes[tid] = size;
    offsets[tid] = ex_s;
    padded[tid] = ex_p;
    if (tid == E - 1) {
      s_off[E] = ex_s + size;
      s_pad[E] = ex_p + padsz;
      offsets[E] = ex_s + size;
      padded[E] = ex_p + padsz;
    }
  }
  __syncthreads();
  if (tid < E) {
    for (int w = 0; w < 32; ++w) hist[w * E + tid] += s_off[tid];
  }
  __syncthreads();

  for (int base = beg; base < end; base += 32) {
    const int p = base + lane;
    int id = -1;
    if (p < end) {
      id = __ldg(ids + p);
      if (id < 0 || id >= E) id = -1;
    }
    const unsigned mask = __match_any_sync(0xffffffffu, id);
    const int rank = __popc(mask & ((1u << lane) - 1u));
    if (id >= 0) {
      const int row = hist[warp * E + id] + rank;
      row_of_pair[p] = row;
      pair_of_row[row] = p;
    } else if (p < end) {
      row_of_pair[p] = -1;
    }
    __syncwarp();
    if (id >= 0 && lane == __ffs(mask) - 1) hist[warp * E + id] += __popc(mask);
    __syncwarp();
  }
  // rows left empty by skipped (out-of-range) pairs
  for (int r = s_off[E] + tid; r < P; r += blockDim.x) pair_of_row[r] = -1;

  // M-block -> expert: largest g with padded[g] <= bx * pad
  for (int bx = tid; bx < M_blk; bx += blockDim.x) {
    const long long x = static_cast<long long>(bx) * pad;
    int lo = 0, hi = E - 1;  // s_pad[0] = 0 <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pad[mid] <= x)
        lo = mid;
      else
        hi = mid - 1;
    }
    idx_for_bx[bx] = lo;
  }
}

cudaError_t launch_tables(const int32_t* ids, int P, int E, int padding_M, int M_blk,
                          int32_t* sizes, int32_t* offsets, int32_t* padded, int32_t* idx_for_bx,
                          int32_t* row_of_pair, int32_t* pair_of_row, int32_t* status,
                          cudaStream_t stream) {
  const size_t smem = (static_cast<size_t>(32) * E + 2 * (E + 1) + 64) * sizeof(int);
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tables_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(32 * 1024 * 4 + 2 * 1025 * 4 + 64 * 4));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  tables_kernel<<<1, 1024, smem, stream>>>(ids, P, E, padding_M, M_blk, sizes, offsets, padded,
                                           idx_for_bx, row_of_pair, pair_of_row, status);
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
