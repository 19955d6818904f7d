// tables.cu - a2: histogram + stable scan -> the four dispatch tables and the
// expert-sorted permutation (TileLang tutorial "Example 07: MoE dispatch
// contract and quantised GEMM", section 1), on the device, with no host sync.
//
// Pairs p = t*k + j are cut into chunks of 1024*R consecutive pairs (R pairs
// per thread, R chosen so there are at most 64 chunks); inside a chunk, warp w
// owns the contiguous sub-range [w*32R, (w+1)*32R) and walks it 32 pairs at a
// time, in order.
//   kernel 1 (one CTA per chunk): per-chunk expert counts -> chunk_counts.
//   kernel 2 (one CTA per chunk): every CTA re-derives the global tables from
//     chunk_counts (per-expert totals, an exclusive scan over experts, and the
//     sum of counts of the chunks before its own), then ranks its pairs: a
//     pair's row is group_offsets[e] + (pairs of e in earlier chunks) + (pairs
//     of e in earlier warps of this chunk) + (earlier pairs of e in this warp).
//     Rows therefore follow the flat pair order inside each expert (a stable
//     sort by expert); no atomics decide any order, so the result is
//     deterministic. CTA 0 also writes group_sizes, group_offsets,
//     group_padded_offsets and group_idx_for_bx.
// Ids outside [0, E) are skipped (row_of_pair = -1) and flagged in *status;
// rows left empty by them get pair_of_row = -1.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "status.cuh"

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxChunks = 64;

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Block-wide exclusive scan of one value per thread (blockDim == 1024).
// Returns the exclusive prefix; *total receives the sum over the block.
__device__ __forceinline__ int block_excl_scan(int v, int* s_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_incl_scan(v, lane);
  if (lane == 31) s_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int t = warp_incl_scan(s_tot[lane], lane);
    __syncwarp();
    s_tot[lane] = t;
  }
  __syncthreads();
  const int ex = inc - v + (warp > 0 ? s_tot[warp - 1] : 0);
  *total = s_tot[31];
  __syncthreads();
  return ex;
}

__device__ __forceinline__ int load_id(const int32_t* ids, int p, int end, int E, bool* bad) {
  if (p >= end) return -1;
  const int id = __ldg(ids + p);
  if (id < 0 || id >= E) {
    *bad = true;
    return -1;
  }
  return id;
}

__global__ void __launch_bounds__(kThreads) chunk_hist_kernel(const int32_t* __restrict__ ids, int P,
                                                              int E, int R,
                                                              int32_t* __restrict__ chunk_counts,
                                                              int32_t* __restrict__ status) {
  extern __shared__ int cnt[];  // [E]
  for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = 0;
  __syncthreads();
  const int chunk = blockIdx.x;
  const int beg = chunk * kThreads * R;
  const int end = min(P, beg + kThreads * R);
  bool bad = false;
  for (int i = beg + threadIdx.x; i < end; i += kThreads) {
    const int id = load_id(ids, i, end, E, &bad);
    if (id >= 0) atomicAdd(&cnt[id], 1);  // a count: the order of the adds does not matter
  }
  if (bad) atomicOr(status, MOE_DEV_BAD_EXPERT_ID_FLAG);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    chunk_counts[static_cast<int64_t>(chunk) * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kThreads) chunk_rank_kernel(
    const int32_t* __restrict__ ids, int P, int E, int R, int nchunks, int pad, int M_blk,
    const int32_t* __restrict__ chunk_counts, int32_t* __restrict__ sizes,
    int32_t* __restrict__ offsets, int32_t* __restrict__ padded, int32_t* __restrict__ idx_for_bx,
    int32_t* __restrict__ row_of_pair, int32_t* __restrict__ pair_of_row) {
  extern __shared__ int smem[];
  int* hist = smem;              // [32][E] per-warp counts, then per-warp bases
  int* s_pad = hist + 32 * E;    // [E + 1]
  int* s_tot = s_pad + E + 1;    // [32]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;
  const int cbeg = chunk * kThreads * R;
  const int cend = min(P, cbeg + kThreads * R);
  const int wbeg = cbeg + warp * 32 * R;
  const int wend = min(cend, wbeg + 32 * R);

  for (int i = tid; i < 32 * E; i += kThreads) hist[i] = 0;
  __syncthreads();
  // per-warp counts of this chunk
  for (int base = wbeg; base < wend; base += 32) {
    bool bad = false;
    const int id = load_id(ids, base + lane, wend, E, &bad);
    const unsigned mask = __match_any_sync(0xffffffffu, id);
    if (id >= 0 && lane == __ffs(mask) - 1) hist[warp * E + id] += __popc(mask);
    __syncwarp();
  }
  // global tables from the chunk counts (every CTA derives the same values)
  int size = 0, before = 0;
  if (tid < E) {
    int c = 0;
    for (; c + 4 <= nchunks; c += 4) {
      const int a0 = __ldg(chunk_counts + static_cast<int64_t>(c) * E + tid);
      const int a1 = __ldg(chunk_counts + static_cast<int64_t>(c + 1) * E + tid);
      const int a2 = __ldg(chunk_counts + static_cast<int64_t>(c + 2) * E + tid);
      const int a3 = __ldg(chunk_counts + static_cast<int64_t>(c + 3) * E + tid);
      before += (c < chunk ? a0 : 0) + (c + 1 < chunk ? a1 : 0) + (c + 2 < chunk ? a2 : 0) +
                (c + 3 < chunk ? a3 : 0);
      size += a0 + a1 + a2 + a3;
    }
    for (; c < nchunks; ++c) {
      const int a = __ldg(chunk_counts + static_cast<int64_t>(c) * E + tid);
      before += c < chunk ? a : 0;
      size += a;
    }
  }
  const int padsz = (size + pad - 1) / pad * pad;
  int total = 0, total_pad = 0;
  const int off = block_excl_scan(size, s_tot, &total);
  const int poff = block_excl_scan(padsz, s_tot, &total_pad);
  if (tid < E) {
    s_pad[tid] = poff;
    if (tid == E - 1) s_pad[E] = poff + padsz;
    // bases of this chunk's warps for expert tid
    int run = off + before;
    for (int w = 0; w < 32; ++w) {
      const int c = hist[w * E + tid];
      hist[w * E + tid] = run;
      run += c;
    }
    if (chunk == 0) {
      sizes[tid] = size;
      offsets[tid] = off;
      padded[tid] = poff;
      if (tid == E - 1) {
        offsets[E] = total;
        padded[E] = total_pad;
      }
    }
  }
  __syncthreads();
  // rows, in flat order within each expert
  for (int base = wbeg; base < wend; base += 32) {
    bool bad = false;
    const int p = base + lane;
    const int id = load_id(ids, p, wend, E, &bad);
    const unsigned mask = __match_any_sync(0xffffffffu, id);
    if (id >= 0) {
      const int row = hist[warp * E + id] + __popc(mask & ((1u << lane) - 1u));
      row_of_pair[p] = row;
      pair_of_row[row] = p;
    } else if (p < wend) {
      row_of_pair[p] = -1;
    }
    __syncwarp();
    if (id >= 0 && lane == __ffs(mask) - 1) hist[warp * E + id] += __popc(mask);
    __syncwarp();
  }
  if (chunk == 0) {
    // rows left empty by skipped (out-of-range) pairs
    for (int r = total + tid; r < P; r += kThreads) pair_of_row[r] = -1;
    // M-block -> expert: the largest g with padded[g] <= bx * pad
    for (int bx = tid; bx < M_blk; bx += kThreads) {
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
}

}  // namespace

int tables_chunk_rounds(int P) {
  const int per = kThreads * kMaxChunks;
  return P <= per ? 1 : (P + per - 1) / per;
}

int tables_num_chunks(int P) {
  const int R = tables_chunk_rounds(P);
  return (P + kThreads * R - 1) / (kThreads * R);
}

cudaError_t launch_tables(const int32_t* ids, int P, int E, int padding_M, int M_blk,
                          int32_t* sizes, int32_t* offsets, int32_t* padded, int32_t* idx_for_bx,
                          int32_t* row_of_pair, int32_t* pair_of_row, int32_t* chunk_counts,
                          int32_t* status, cudaStream_t stream) {
  if (P <= 0) return cudaSuccess;
  const int R = tables_chunk_rounds(P);
  const int nchunks = tables_num_chunks(P);
  const size_t smem1 = static_cast<size_t>(E) * sizeof(int);
  const size_t smem2 = (static_cast<size_t>(32) * E + (E + 1) + 32) * sizeof(int);
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    const int max2 = static_cast<int>((32 * 1024 + 1025 + 32) * sizeof(int));
    cudaError_t e = cudaFuncSetAttribute(chunk_rank_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, max2);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  chunk_hist_kernel<<<nchunks, kThreads, smem1, stream>>>(ids, P, E, R, chunk_counts, status);
  chunk_rank_kernel<<<nchunks, kThreads, smem2, stream>>>(ids, P, E, R, nchunks, padding_M, M_blk,
                                                          chunk_counts, sizes, offsets, padded,
                                                          idx_for_bx, row_of_pair, pair_of_row);
  return cudaGetLastError();
}

}  // namespace moe
