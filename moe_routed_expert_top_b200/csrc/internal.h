// internal.h - launch helpers shared by the C-ABI layer (api.cu) and the
// kernel translation units. Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

enum GemmMode { kModeStore = 0, kModeSwiglu = 1, kModeSwigluFp8 = 2, kModeFp8Store = 3 };

struct GemmLaunch {
  int mode = kModeStore;
  int tiling = 0;  // GemmTiling
  // grouped mode: tables non-null, rows = P; dense mode: tables null, rows = M
  int rows = 0;
  int N = 0;  // rows of B per expert
  int K = 0;
  int E = 1;
  const void* A = nullptr;
  const void* B = nullptr;
  const float* A_scales = nullptr;  // fp8 mode [rows, K/128]
  const float* B_scales = nullptr;  // fp8 mode [E, N/128, K/128]
  const int32_t* group_sizes = nullptr;
  const int32_t* group_offsets = nullptr;
  const int32_t* group_padded = nullptr;
  const int32_t* idx_for_bx = nullptr;
  int M_blk = 0;  // length of idx_for_bx (grouped mode)
  void* C = nullptr;
  int out_f32 = 0;  // store modes: fp32 C instead of bf16
  // store modes: C fp16 with one int8 power-of-two exponent per row and
  // 128-column block in C_exps [rows, N / 128] (f16e.cuh); weight-row and
  // pair tilings, not with the weighted store
  int out_f16e = 0;
  int8_t* C_exps = nullptr;
  float* C_scales = nullptr;
  float* debug_h = nullptr;
  int32_t* status = nullptr;
  // gather mode (weight-row pair tiling only): A is the hidden states
  // [a_rows, K] and row r of the grouped problem is A[pair_of_row[r] / top_k]
  int gather = 0;
  const int32_t* pair_of_row = nullptr;
  int top_k = 0;
  int a_rows = 0;
  // B as a view into a larger matrix (weight-row pair tiling only; 0 = the
  // default): ldb = elements between consecutive B rows (default K); up_off =
  // rows from a gate row to its up row in SwiGLU mode (default N / 2); b_rows =
  // rows addressable from B (default E * N). A tensor-parallel shard of a
  // complete weight is addressed in place this way.
  int ldb = 0;
  int up_off = 0;
  long long b_rows = 0;
  // weighted store (store modes, bf16 or fp32 C, grouped; weight-row tilings only):
  // row r of the result goes to C row pair_of_row[r] (flat pair order),
  // multiplied by row_scale * row_weights[pair_of_row[r]]; rows with no pair
  // (-1) are skipped
  int weighted = 0;
  const float* row_weights = nullptr;
  float row_scale = 1.0f;
  // at most this many CTAs (0 = one per SM): leaves SMs to a kernel that runs
  // beside this one on another stream
  int max_ctas = 0;
};

// Tiling of the grouped GEMM: token-row tiles (grouped_gemm.cu), weight-row
// tiles with the tokens on the MMA's N side (grouped_gemm_t.cu), or the same
// weight-row tiles computed by CTA pairs with 256-row MMAs (grouped_gemm_t2.cu).
enum GemmTiling { kTilingAuto = 0, kTilingRows = 1, kTilingWeights = 2, kTilingWeightsPair = 3 };

// Each returns cudaSuccess or the launch error.
cudaError_t launch_grouped_gemm(const GemmLaunch& L, cudaStream_t stream);
cudaError_t launch_grouped_gemm_t(const GemmLaunch& L, cudaStream_t stream);
bool grouped_gemm_t_supported(const GemmLaunch& L);
bool grouped_gemm_t_preferred(const GemmLaunch& L);
cudaError_t launch_grouped_gemm_pair(const GemmLaunch& L, cudaStream_t stream);
bool grouped_gemm_pair_supported(const GemmLaunch& L);
bool grouped_gemm_pair_preferred(const GemmLaunch& L);
// Whether the automatic (or requested) tiling of L stores the f16e format.
bool grouped_gemm_f16e_supported(const GemmLaunch& L);

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int score_fn,
                              int renormalize, int32_t* ids, float* weights, cudaStream_t stream);

// chunk_counts: scratch of tables_num_chunks(P) * E int32
cudaError_t launch_tables(const int32_t* ids, int P, int E, int padding_M, int M_blk,
                          int32_t* sizes, int32_t* offsets, int32_t* padded, int32_t* idx_for_bx,
                          int32_t* row_of_pair, int32_t* pair_of_row, int32_t* chunk_counts,
                          int32_t* status, cudaStream_t stream);
int tables_num_chunks(int P);

cudaError_t launch_gather_rows(const void* hidden, const int32_t* pair_of_row, int P, int k,
                               int H, void* x_perm, cudaStream_t stream);

// y fp32 [T*k, H]; addend fp32 [T, H] or null; out bf16 [T, H]
cudaError_t launch_unpermute(const float* y, const int32_t* row_of_pair, const float* weights,
                             int T, int k, int H, float scale, const float* addend, void* out,
                             cudaStream_t stream);
// The same from the down GEMM's f16e output: y16 fp16 [T*k, H], y_exp int8
// [T*k, H/128], y = y16 * 2^y_exp.
cudaError_t launch_unpermute_f16e(const void* y16, const int8_t* y_exp, const int32_t* row_of_pair,
                                  const float* weights, int T, int k, int H, float scale,
                                  const float* addend, void* out, cudaStream_t stream);
cudaError_t launch_combine(const void* y_w, bool y_f32, const int32_t* row_of_pair, int T, int k,
                           int H, const float* addend, void* out, cudaStream_t stream);

cudaError_t launch_swiglu_quant(int M, int F, const void* gate_up, const float* h, int out_fp8,
                                void* out, float* scales, cudaStream_t stream);

cudaError_t launch_quantize_weight(int batch, int N, int K, const void* w, uint8_t* q,
                                   float* scales, cudaStream_t stream);

// Training-side FP8 dual-layout quantisation (train_fp8.cu).
struct DualLaunch {
  int M = 0;  // rows of x
  int K = 0;  // columns of the quantised activation (SwiGLU: F)
  int E = 1;
  const int32_t* sizes = nullptr;  // grouped mode (all four non-null) or dense (all null)
  const int32_t* offsets = nullptr;
  const int32_t* padded = nullptr;
  const int32_t* idx_for_bx = nullptr;
  int M_blk = 0;  // 128-token blocks of the padded axis (qT row pitch / 128)
  const void* x = nullptr;  // bf16 [M, K], or gate_up bf16 [M, 2K] when swiglu
  int swiglu = 0;
  int trans_block = 1;  // 1: 128x128 block scales of xT; 0: 1x128 tile scales
  uint8_t* q = nullptr;
  float* s = nullptr;
  uint8_t* qT = nullptr;
  float* sT = nullptr;
  float* debug_h = nullptr;
};
cudaError_t launch_quant_dual(const DualLaunch& L, cudaStream_t stream);
cudaError_t launch_swiglu_backward(int M, int F, const void* gate_up, const void* grad_h,
                                   void* grad_gate_up, cudaStream_t stream);

// Expert parallelism helpers (ep.cu).
cudaError_t launch_split_ids(int n, int E_local, int world, const int32_t* ids, int32_t* rank_ids,
                             int32_t* local_ids, cudaStream_t stream);
cudaError_t launch_gather_rows_any(int n_dst, int n_src, long long row_bytes, const int32_t* map,
                                   const void* src, void* dst, int32_t* status,
                                   cudaStream_t stream);

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

}  // namespace moe
