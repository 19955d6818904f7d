// ep.cu - the two index/row kernels expert parallelism needs around the
// existing path: experts split over ranks, tokens dispatched to the ranks
// that own their experts and the results combined back (pypto-lib PR #809
// "predicate empty routed-expert stages": a dispatch step producing per-expert
// counts and gathered rows for each rank's local experts, whose routed stages
// then skip empty experts):
//
//  * split_ids: a global expert id e becomes (rank e / E_local, local expert
//    e % E_local); ids outside [0, world * E_local) get rank `world` (which the
//    table builder then flags as a bad id) and local id 0;
//  * gather_rows: dst[r] = src[map[r]] for rows of any multiple of 4 bytes
//    (16-byte vectors when the row allows), a negative map entry gives a zero
//    row, an entry >= n_src gives a zero row and sets MOE_DEV_BAD_TABLES.
#include <cuda_runtime.h>

#include "internal.h"
#include "status.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) split_ids_kernel(int n, int E_local, int world,
                                                        const int32_t* __restrict__ ids,
                                                        int32_t* __restrict__ rank_ids,
                                                        int32_t* __restrict__ local_ids) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int e = ids[i];
  const bool ok = e >= 0 && e < world * E_local;
  const int r = ok ? e / E_local : world;
  rank_ids[i] = r;
  local_ids[i] = ok ? e - r * E_local : 0;
}

template <typename V>
__global__ void __launch_bounds__(256) gather_rows_kernel_v(int n_dst, int n_src, int row_v,
                                                            const int32_t* __restrict__ map,
                                                            const V* __restrict__ src,
                                                            V* __restrict__ dst,
                                                            int32_t* status) {
  // one warp per destination row, grid-stride over rows
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < n_dst; r += warps) {
    const int s = __ldg(map + r);
    const bool ok = s >= 0 && s < n_src;
    if (s >= n_src && lane == 0 && status != nullptr) atomicOr(status, MOE_DEV_BAD_TABLES_FLAG);
    V* d = dst + static_cast<int64_t>(r) * row_v;
    if (ok) {
      const V* p = src + static_cast<int64_t>(s) * row_v;
      for (int c = lane; c < row_v; c += 32) d[c] = __ldg(p + c);
    } else {
      V z;
      memset(&z, 0, sizeof(V));
      for (int c = lane; c < row_v; c += 32) d[c] = z;
    }
  }
}

}  // namespace

cudaError_t launch_split_ids(int n, int E_local, int world, const int32_t* ids, int32_t* rank_ids,
                             int32_t* local_ids, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  split_ids_kernel<<<(n + 255) / 256, 256, 0, stream>>>(n, E_local, world, ids, rank_ids,
                                                        local_ids);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows_any(int n_dst, int n_src, long long row_bytes, const int32_t* map,
                                   const void* src, void* dst, int32_t* status,
                                   cudaStream_t stream) {
  if (n_dst <= 0) return cudaSuccess;
  long long blocks = (static_cast<long long>(n_dst) + 7) / 8;  // 8 warps per block
  const long long cap = static_cast<long long>(device_sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  const unsigned g = static_cast<unsigned>(blocks);
  const bool vec16 = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
  if (vec16)
    gather_rows_kernel_v<uint4><<<g, 256, 0, stream>>>(
        n_dst, n_src, static_cast<int>(row_bytes / 16), map, static_cast<const uint4*>(src),
        static_cast<uint4*>(dst), status);
  else
    gather_rows_kernel_v<uint32_t><<<g, 256, 0, stream>>>(
        n_dst, n_src, static_cast<int>(row_bytes / 4), map, static_cast<const uint32_t*>(src),
        static_cast<uint32_t*>(dst), status);
  return cudaGetLastError();
}

}  // namespace moe
