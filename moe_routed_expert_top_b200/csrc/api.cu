// api.cu - the extern "C" entry points declared in include/moe.h: argument
// validation, table/workspace layout, and the launch sequence of the whole
// routed-experts forward. No allocation, no host synchronisation: every call
// only enqueues kernels on the caller's stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "moe.h"

namespace {

thread_local char g_last_error[256] = "";
thread_local int32_t g_last_launches = 0;

moe_status cuda_fail(cudaError_t e) {
  std::strncpy(g_last_error, cudaGetErrorString(e), sizeof(g_last_error) - 1);
  g_last_error[sizeof(g_last_error) - 1] = '\0';
  return MOE_ERR_CUDA;
}

#define MOE_CUDA_TRY(expr)                  \
  do {                                      \
    cudaError_t _e = (expr);                \
    if (_e != cudaSuccess) return cuda_fail(_e); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxPairs = (1ll << 31) - (1ll << 20);

// Shape rules shared by every call that takes a moe_problem.
moe_status check_problem(const moe_problem* pr, bool need_gemm) {
  if (pr == nullptr) return MOE_ERR_INVALID_ARG;
  if (pr->T < 0 || pr->H <= 0 || pr->F <= 0 || pr->E <= 0 || pr->top_k <= 0 ||
      pr->padding_M <= 0 || pr->F_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (pr->score_fn != MOE_SCORE_SOFTMAX && pr->score_fn != MOE_SCORE_SIGMOID)
    return MOE_ERR_INVALID_ARG;
  if (pr->E > 1024 || pr->top_k > 32) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(pr->T) * pr->top_k > kMaxPairs) return MOE_ERR_UNSUPPORTED;
  if (pr->padding_M > (1 << 20)) return MOE_ERR_UNSUPPORTED;
  if (need_gemm) {
    // a token's k experts are distinct; tables over given ids accept repeats
    // (the groups can be ranks, as in expert parallelism)
    if (pr->top_k > pr->E) return MOE_ERR_UNSUPPORTED;
    if (pr->padding_M != 128) return MOE_ERR_UNSUPPORTED;
    if (pr->H % 64 != 0 || pr->F % 64 != 0 || pr->F_shared % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (pr->down_fp8 && (pr->H % 128 != 0 || pr->F % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// A second stream per device on which the forward runs the shared expert beside
// the routed GEMMs (created on first use outside stream capture; null if it
// does not exist yet and may not be created now, or if creating it fails: the
// forward then runs everything on the caller's stream).
cudaStream_t side_stream(bool may_create) {
  static cudaStream_t streams[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (streams[dev] == nullptr && may_create) {
    cudaStream_t t = nullptr;
    if (cudaStreamCreateWithFlags(&t, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    streams[dev] = t;
  }
  return streams[dev];
}

// An event released when the forward returns (also on its error paths);
// destroying an event whose record and waits are enqueued is allowed.
struct EventGuard {
  cudaEvent_t e = nullptr;
  bool create() {
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess) return true;
    e = nullptr;
    cudaGetLastError();
    return false;
  }
  ~EventGuard() {
    if (e != nullptr) cudaEventDestroy(e);
  }
};

// SMs given to the shared expert while the routed GEMMs run on the others, so
// that both finish at about the same time: the shared MLP is compute-bound
// (its FLOPs at about 0.9 PFLOP/s, the dense rate its tiles reach on B200),
// the routed GEMMs stream the touched experts' weights at about 5.8 TB/s.
// Even (the shared GEMMs run on CTA pairs), at least 2, at most a quarter.
int shared_sms(const moe_problem* pr, int sms) {
  const double shared_s = 6.0 * pr->T * static_cast<double>(pr->H) * pr->F_shared / 0.9e15;
  const double touched = pr->E < static_cast<int64_t>(pr->T) * pr->top_k
                             ? pr->E
                             : static_cast<double>(pr->T) * pr->top_k;
  const double routed_s = touched * 3.0 * pr->H * static_cast<double>(pr->F) *
                          (pr->down_fp8 ? 1.67 : 2.0) / 5.8e12;
  int k = static_cast<int>(sms * shared_s / (routed_s > 0 ? routed_s : 1e-9) + 0.5);
  k &= ~1;
  if (k < 2) k = 2;
  if (k > sms / 4) k = (sms / 4) & ~1;
  return k;
}

void fill_layout(const moe_problem* pr, moe_tables_layout* L) {
  const int64_t E = pr->E;
  const int64_t P = static_cast<int64_t>(pr->T) * pr->top_k;
  const int64_t M_blk = (P + pr->padding_M - 1) / pr->padding_M + E;
  int64_t o = 0;
  L->group_sizes = o;
  o += round_up(E, 4);
  L->group_offsets = o;
  o += round_up(E + 1, 4);
  L->group_padded_offsets = o;
  o += round_up(E + 1, 4);
  L->group_idx_for_bx = o;
  o += round_up(M_blk, 4);
  L->row_of_pair = o;
  o += round_up(P, 4);
  L->pair_of_row = o;
  o += round_up(P, 4);
  L->chunk_counts = o;
  o += round_up(static_cast<int64_t>(moe::tables_num_chunks(static_cast<int>(P))) * E, 4);
  L->total_int32 = o;
  L->M_blk = static_cast<int32_t>(M_blk);
  L->P = static_cast<int32_t>(P);
}

struct WorkspacePlan {
  int64_t status = 0, tables = 0, x_perm = 0, h = 0, h_scales = 0, y = 0, y_exp = 0, hs = 0, ys = 0,
          total = 0;
};

WorkspacePlan plan_workspace(const moe_problem* pr) {
  moe_tables_layout L;
  fill_layout(pr, &L);
  const int64_t P = L.P, T = pr->T, H = pr->H, F = pr->F, Fs = pr->F_shared;
  WorkspacePlan w;
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o = round_up(o + bytes, 1024);
    return at;
  };
  w.status = take(256);
  w.tables = take(L.total_int32 * 4);
  w.x_perm = take(P * H * 2);
  w.h = take(P * F * (pr->down_fp8 ? 1 : 2));
  w.h_scales = take(pr->down_fp8 ? P * (F / 128) * 4 : 0);
  // the down GEMM's output: fp32 [P, H], or f16e (fp16 [P, H] in the same
  // region + int8 exponents [P, H/128])
  w.y = take(P * H * 4);
  w.y_exp = take(P * ((H + 127) / 128));
  w.hs = take(Fs ? T * Fs * 2 : 0);
  w.ys = take(Fs ? T * H * 4 : 0);
  w.total = o;
  return w;
}

}  // namespace

extern "C" {

moe_status moe_get_tables_layout(const moe_problem* prob, moe_tables_layout* out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  fill_layout(prob, out);
  return MOE_OK;
}

size_t moe_workspace_bytes(const moe_problem* prob) {
  if (check_problem(prob, true) != MOE_OK) return 0;
  return static_cast<size_t>(plan_workspace(prob).total);
}

moe_status moe_route_topk(const moe_problem* prob, const float* logits, int32_t* topk_ids,
                          float* topk_weights, moe_stream_t stream) {
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (prob->top_k > prob->E) return MOE_ERR_UNSUPPORTED;  // k distinct experts
  if (prob->T == 0) return MOE_OK;
  if (logits == nullptr || topk_ids == nullptr || topk_weights == nullptr)
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_route_topk(logits, prob->T, prob->E, prob->top_k, prob->score_fn,
                                      prob->renormalize, topk_ids, topk_weights,
                                      reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_route_permute(const moe_problem* prob, const float* logits, int32_t* topk_ids,
                             float* topk_weights, const void* hidden, void* x_perm,
                             int32_t* tables, int32_t* dev_status, moe_stream_t stream) {
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (logits != nullptr && prob->top_k > prob->E) return MOE_ERR_UNSUPPORTED;
  if (prob->T == 0) return MOE_OK;
  if (topk_ids == nullptr || tables == nullptr || dev_status == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (logits != nullptr && topk_weights == nullptr) return MOE_ERR_INVALID_ARG;
  if (hidden != nullptr && (x_perm == nullptr || !aligned16(hidden) || !aligned16(x_perm) ||
                            prob->H % 8 != 0))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  moe_tables_layout L;
  fill_layout(prob, &L);
  if (logits != nullptr)
    MOE_CUDA_TRY(moe::launch_route_topk(logits, prob->T, prob->E, prob->top_k, prob->score_fn,
                                        prob->renormalize, topk_ids, topk_weights, st));
  MOE_CUDA_TRY(moe::launch_tables(topk_ids, L.P, prob->E, prob->padding_M, L.M_blk,
                                  tables + L.group_sizes, tables + L.group_offsets,
                                  tables + L.group_padded_offsets, tables + L.group_idx_for_bx,
                                  tables + L.row_of_pair, tables + L.pair_of_row,
                                  tables + L.chunk_counts, dev_status, st));
  if (hidden != nullptr)
    MOE_CUDA_TRY(moe::launch_gather_rows(hidden, tables + L.pair_of_row, L.P, prob->top_k,
                                         prob->H, x_perm, st));
  return MOE_OK;
}

moe_status moe_grouped_gemm(const moe_problem* prob, int32_t M_rows, int32_t N, int32_t K,
                            const void* A, const float* A_scales, const void* B,
                            const float* B_scales, const int32_t* tables, int32_t epilogue,
                            void* C, float* C_scales, float* debug_h, int32_t* dev_status,
                            moe_stream_t stream) {
  if (A == nullptr || B == nullptr || C == nullptr || dev_status == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return MOE_ERR_INVALID_ARG;
  const bool fp8 = A_scales != nullptr || B_scales != nullptr;
  if (fp8 && (A_scales == nullptr || B_scales == nullptr)) return MOE_ERR_INVALID_ARG;
  moe::GemmLaunch g;
  if ((epilogue & ~(MOE_A_GATHER | 0xFF)) != 0) return MOE_ERR_INVALID_ARG;
  const int tiling = (epilogue >> 4) & 0xF;
  g.gather = (epilogue & MOE_A_GATHER) != 0;
  epilogue &= 0xF;
  if (tiling > moe::kTilingWeightsPair) return MOE_ERR_INVALID_ARG;
  g.tiling = tiling;
  if (tables != nullptr) {
    moe_status s = check_problem(prob, false);
    if (s != MOE_OK) return s;
    if (prob->padding_M != 128) return MOE_ERR_UNSUPPORTED;
    moe_tables_layout L;
    fill_layout(prob, &L);
    g.rows = L.P;
    g.E = prob->E;
    g.group_sizes = tables + L.group_sizes;
    g.group_offsets = tables + L.group_offsets;
    g.group_padded = tables + L.group_padded_offsets;
    g.idx_for_bx = tables + L.group_idx_for_bx;
    g.M_blk = L.M_blk;
    if (g.gather) {
      g.pair_of_row = tables + L.pair_of_row;
      g.top_k = prob->top_k;
      g.a_rows = prob->T;
      if (K != prob->H) return MOE_ERR_INVALID_ARG;  // gathered rows are whole hidden rows
    }
  } else {
    if (g.gather) return MOE_ERR_INVALID_ARG;  // gathering follows the group tables
    if (M_rows < 0) return MOE_ERR_INVALID_ARG;
    g.rows = M_rows;
    g.E = 1;
  }
  if (g.rows == 0) return MOE_OK;
  if (epilogue == MOE_EPI_STORE_F16E) {
    // fp16 + one int8 exponent per row and 128 columns, into C and C_scales
    if (C_scales == nullptr) return MOE_ERR_INVALID_ARG;
    if (N % 128 != 0) return MOE_ERR_UNSUPPORTED;
    g.out_f16e = 1;
    g.C_exps = reinterpret_cast<int8_t*>(C_scales);
  }
  if (fp8) {
    if (epilogue != MOE_EPI_STORE && epilogue != MOE_EPI_STORE_F32 &&
        epilogue != MOE_EPI_STORE_F16E)
      return MOE_ERR_UNSUPPORTED;
    if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_UNSUPPORTED;
    g.mode = moe::kModeFp8Store;
    g.out_f32 = epilogue == MOE_EPI_STORE_F32;
  } else {
    if (K % 64 != 0) return MOE_ERR_UNSUPPORTED;
    switch (epilogue) {
      case MOE_EPI_STORE:
      case MOE_EPI_STORE_F32:
      case MOE_EPI_STORE_F16E:
        if (N % 64 != 0) return MOE_ERR_UNSUPPORTED;
        g.mode = moe::kModeStore;
        g.out_f32 = epilogue == MOE_EPI_STORE_F32;
        break;
      case MOE_EPI_SWIGLU:
        if (N % 128 != 0) return MOE_ERR_UNSUPPORTED;  // F = N/2 multiple of 64
        g.mode = moe::kModeSwiglu;
        break;
      case MOE_EPI_SWIGLU_FP8:
        if (N % 256 != 0) return MOE_ERR_UNSUPPORTED;  // F multiple of 128
        if (C_scales == nullptr) return MOE_ERR_INVALID_ARG;
        if (debug_h != nullptr && !aligned16(debug_h)) return MOE_ERR_INVALID_ARG;
        g.mode = moe::kModeSwigluFp8;
        break;
      default:
        return MOE_ERR_INVALID_ARG;
    }
  }
  g.N = N;
  g.K = K;
  g.A = A;
  g.B = B;
  g.A_scales = A_scales;
  g.B_scales = B_scales;
  g.C = C;
  g.C_scales = C_scales;
  g.debug_h = debug_h;
  g.status = dev_status;
  if (g.tiling == moe::kTilingWeights && !moe::grouped_gemm_t_supported(g))
    return MOE_ERR_UNSUPPORTED;
  if (g.tiling == moe::kTilingWeightsPair && !moe::grouped_gemm_pair_supported(g))
    return MOE_ERR_UNSUPPORTED;
  if (g.out_f16e && !moe::grouped_gemm_f16e_supported(g)) return MOE_ERR_UNSUPPORTED;
  // gathering is built into the weight-row pair tiling only
  if (g.gather && ((g.tiling != moe::kTilingAuto && g.tiling != moe::kTilingWeightsPair) ||
                   !moe::grouped_gemm_pair_supported(g)))
    return MOE_ERR_UNSUPPORTED;
  MOE_CUDA_TRY(moe::launch_grouped_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_swiglu_quant(int32_t M, int32_t F, const void* gate_up, const float* h,
                            int32_t out_fp8, void* out, float* scales, moe_stream_t stream) {
  if (M < 0 || F <= 0 || F % 4 != 0) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  if ((gate_up == nullptr) == (h == nullptr)) return MOE_ERR_INVALID_ARG;
  if (gate_up == nullptr && !out_fp8) return MOE_ERR_INVALID_ARG;
  if (out_fp8 && scales == nullptr) return MOE_ERR_INVALID_ARG;
  if ((gate_up && !aligned16(gate_up)) || (h && !aligned16(h)) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_swiglu_quant(M, F, gate_up, h, out_fp8 ? 1 : 0, out, scales,
                                        reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_unpermute(const moe_problem* prob, const float* y, const int32_t* tables,
                         const float* topk_weights, float scale, const float* addend, void* out,
                         moe_stream_t stream) {
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (prob->T == 0) return MOE_OK;
  if (y == nullptr || tables == nullptr || topk_weights == nullptr || out == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (prob->H % 8 != 0 || !aligned16(y) || !aligned16(out) || (addend && !aligned16(addend)))
    return MOE_ERR_INVALID_ARG;
  moe_tables_layout L;
  fill_layout(prob, &L);
  MOE_CUDA_TRY(moe::launch_unpermute(y, tables + L.row_of_pair, topk_weights, prob->T,
                                     prob->top_k, prob->H, scale, addend, out,
                                     reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_unpermute_f16e(const moe_problem* prob, const void* y16, const int8_t* y_exp,
                              const int32_t* tables, const float* topk_weights, float scale,
                              const float* addend, void* out, moe_stream_t stream) {
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (prob->T == 0) return MOE_OK;
  if (y16 == nullptr || y_exp == nullptr || tables == nullptr || topk_weights == nullptr ||
      out == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (prob->H % 128 != 0 || !aligned16(y16) || !aligned16(out) || (addend && !aligned16(addend)))
    return MOE_ERR_INVALID_ARG;
  moe_tables_layout L;
  fill_layout(prob, &L);
  MOE_CUDA_TRY(moe::launch_unpermute_f16e(y16, y_exp, tables + L.row_of_pair, topk_weights,
                                          prob->T, prob->top_k, prob->H, scale, addend, out,
                                          reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_down_gemm_weighted(const moe_problem* prob, int32_t N, int32_t K, const void* A,
                                  const float* A_scales, const void* B, const float* B_scales,
                                  const int32_t* tables, const float* topk_weights, float scale,
                                  int32_t epilogue, void* y_w, int32_t* dev_status,
                                  moe_stream_t stream) {
  if (A == nullptr || B == nullptr || tables == nullptr || topk_weights == nullptr ||
      y_w == nullptr || dev_status == nullptr)
    return MOE_ERR_INVALID_ARG;
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (prob->padding_M != 128) return MOE_ERR_UNSUPPORTED;
  if (N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(y_w)) return MOE_ERR_INVALID_ARG;
  if ((epilogue & ~0xFF) != 0) return MOE_ERR_INVALID_ARG;
  const int t = (epilogue >> 4) & 0xF;
  const int epi = epilogue & 0xF;
  if (epi != MOE_EPI_STORE && epi != MOE_EPI_STORE_F32) return MOE_ERR_INVALID_ARG;
  if (t > moe::kTilingWeightsPair) return MOE_ERR_INVALID_ARG;
  if (t == moe::kTilingRows) return MOE_ERR_UNSUPPORTED;
  const bool fp8 = A_scales != nullptr || B_scales != nullptr;
  if (fp8 && (A_scales == nullptr || B_scales == nullptr)) return MOE_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % (fp8 ? 128 : 64) != 0) return MOE_ERR_UNSUPPORTED;
  moe_tables_layout L;
  fill_layout(prob, &L);
  if (L.P == 0) return MOE_OK;
  moe::GemmLaunch g;
  g.tiling = t;
  g.mode = fp8 ? moe::kModeFp8Store : moe::kModeStore;
  g.rows = L.P;
  g.E = prob->E;
  g.group_sizes = tables + L.group_sizes;
  g.group_offsets = tables + L.group_offsets;
  g.group_padded = tables + L.group_padded_offsets;
  g.idx_for_bx = tables + L.group_idx_for_bx;
  g.M_blk = L.M_blk;
  g.N = N;
  g.K = K;
  g.A = A;
  g.B = B;
  g.A_scales = A_scales;
  g.B_scales = B_scales;
  g.C = y_w;
  g.out_f32 = epi == MOE_EPI_STORE_F32;
  g.status = dev_status;
  g.weighted = 1;
  g.pair_of_row = tables + L.pair_of_row;
  g.row_weights = topk_weights;
  g.row_scale = scale;
  if (t == moe::kTilingWeights && !moe::grouped_gemm_t_supported(g)) return MOE_ERR_UNSUPPORTED;
  if (t == moe::kTilingWeightsPair && !moe::grouped_gemm_pair_supported(g))
    return MOE_ERR_UNSUPPORTED;
  if (t == moe::kTilingAuto && !moe::grouped_gemm_t_supported(g) &&
      !moe::grouped_gemm_pair_supported(g))
    return MOE_ERR_UNSUPPORTED;
  MOE_CUDA_TRY(moe::launch_grouped_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_combine(const moe_problem* prob, const void* y_w, int32_t y_f32,
                       const int32_t* tables, const float* addend, void* out,
                       moe_stream_t stream) {
  moe_status s = check_problem(prob, false);
  if (s != MOE_OK) return s;
  if (prob->T == 0) return MOE_OK;
  if (y_w == nullptr || tables == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if (prob->H % 8 != 0 || !aligned16(y_w) || !aligned16(out) || (addend && !aligned16(addend)))
    return MOE_ERR_INVALID_ARG;
  moe_tables_layout L;
  fill_layout(prob, &L);
  MOE_CUDA_TRY(moe::launch_combine(y_w, y_f32 != 0, tables + L.row_of_pair, prob->T, prob->top_k,
                                   prob->H, addend, out, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_quantize_weight_128x128(int32_t batch, int32_t N, int32_t K, const void* w,
                                       uint8_t* q, float* scales, moe_stream_t stream) {
  if (batch < 0 || N < 0 || K < 0 || w == nullptr || q == nullptr || scales == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (batch > 65535 || N / 128 > 65535) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(w) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_quantize_weight(batch, N, K, w, q, scales,
                                           reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_experts_forward(const moe_problem* prob, const void* hidden,
                               const int32_t* topk_ids, const float* topk_weights,
                               const void* w_gate_up, const void* w_down,
                               const float* w_down_scales, const void* ws_gate_up,
                               const void* ws_down, float scale, void* out, void* workspace,
                               size_t ws_bytes, moe_stream_t stream) {
  g_last_launches = 0;
  moe_status s = check_problem(prob, true);
  if (s != MOE_OK) return s;
  if (prob->T == 0) return MOE_OK;
  if (hidden == nullptr || topk_ids == nullptr || topk_weights == nullptr ||
      w_gate_up == nullptr || w_down == nullptr || out == nullptr || workspace == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (prob->down_fp8 && w_down_scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (prob->F_shared > 0 && (ws_gate_up == nullptr || ws_down == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out) ||
      !aligned16(workspace) || (ws_gate_up && !aligned16(ws_gate_up)) ||
      (ws_down && !aligned16(ws_down)))
    return MOE_ERR_INVALID_ARG;
  const WorkspacePlan w = plan_workspace(prob);
  if (ws_bytes < static_cast<size_t>(w.total)) return MOE_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(base + w.status);
  int32_t* tables = reinterpret_cast<int32_t*>(base + w.tables);
  void* x_perm = base + w.x_perm;
  void* h = base + w.h;
  float* h_scales = reinterpret_cast<float*>(base + w.h_scales);
  float* y = reinterpret_cast<float*>(base + w.y);
  moe_tables_layout L;
  fill_layout(prob, &L);
  const int T = prob->T, H = prob->H, F = prob->F, E = prob->E, k = prob->top_k;

  MOE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), st));

  // shared expert (a dense SwiGLU MLP on all tokens, added in the unpermute).
  // Where the routed experts hold few rows each (at most 64 on average, the
  // single-CTA weight-row tiling) their GEMMs are bound by weight bytes while
  // the shared MLP is compute-bound, so it runs on its own stream and a few
  // SMs beside them, joined before the unpermute: Kimi-K2 (T 512, 384
  // experts) 5.14 vs 5.28 ms per layer. With more rows per expert the routed
  // GEMMs need all SMs (DeepSeek-V3 prefill, 128 rows per expert: 4.75 with
  // 16 SMs given away, 4.72 serial), and the shared expert runs after them.
  const float* addend = nullptr;
  EventGuard fork, join;
  bool beside = false;
  int routed_ctas = 0;
  if (prob->F_shared > 0) {
    moe::GemmLaunch d;
    d.rows = T;
    d.E = 1;
    d.status = status;
    d.mode = moe::kModeSwiglu;
    d.N = 2 * prob->F_shared;
    d.K = H;
    d.A = hidden;
    d.B = ws_gate_up;
    d.C = base + w.hs;
    // a stream is not created while the caller's stream is being captured
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
      cudaGetLastError();
      cap = cudaStreamCaptureStatusActive;
    }
    cudaStream_t side = static_cast<int64_t>(T) * k <= 64LL * E
                            ? side_stream(cap == cudaStreamCaptureStatusNone)
                            : nullptr;
    beside = side != nullptr && fork.create() && join.create();
    cudaStream_t sst = st;
    if (beside) {
      const int sms = moe::device_sm_count();
      d.max_ctas = shared_sms(prob, sms);
      routed_ctas = sms - d.max_ctas;
      sst = side;
      MOE_CUDA_TRY(cudaEventRecord(fork.e, st));
      MOE_CUDA_TRY(cudaStreamWaitEvent(side, fork.e, 0));
    }
    MOE_CUDA_TRY(moe::launch_grouped_gemm(d, sst));
    d.mode = moe::kModeStore;
    d.N = H;
    d.K = prob->F_shared;
    d.A = base + w.hs;
    d.B = ws_down;
    d.C = base + w.ys;
    d.out_f32 = 1;
    MOE_CUDA_TRY(moe::launch_grouped_gemm(d, sst));
    if (beside) MOE_CUDA_TRY(cudaEventRecord(join.e, side));
    addend = reinterpret_cast<const float*>(base + w.ys);
    g_last_launches += 2;
  }

  // a2 + a3
  MOE_CUDA_TRY(moe::launch_tables(topk_ids, L.P, E, prob->padding_M, L.M_blk,
                                  tables + L.group_sizes, tables + L.group_offsets,
                                  tables + L.group_padded_offsets, tables + L.group_idx_for_bx,
                                  tables + L.row_of_pair, tables + L.pair_of_row,
                                  tables + L.chunk_counts, status, st));
  g_last_launches += 2;

  moe::GemmLaunch g;
  g.rows = L.P;
  g.E = E;
  g.group_sizes = tables + L.group_sizes;
  g.group_offsets = tables + L.group_offsets;
  g.group_padded = tables + L.group_padded_offsets;
  g.idx_for_bx = tables + L.group_idx_for_bx;
  g.M_blk = L.M_blk;
  g.status = status;
  g.max_ctas = routed_ctas;
  // a4 + a5: gate+up with the SwiGLU (+ FP8 1x128) epilogue
  g.mode = prob->down_fp8 ? moe::kModeSwigluFp8 : moe::kModeSwiglu;
  g.N = 2 * F;
  g.K = H;
  g.B = w_gate_up;
  g.C = h;
  g.C_scales = prob->down_fp8 ? h_scales : nullptr;
  // a3: the gather kernel writes x_perm once. (Gathering inside the GEMM,
  // MOE_A_GATHER, re-fetches every token row once per weight block with
  // four-row TMA gathers and measured about 2x slower end to end on B200.)
  MOE_CUDA_TRY(moe::launch_gather_rows(hidden, tables + L.pair_of_row, L.P, k, H, x_perm, st));
  g_last_launches += 1;
  g.A = x_perm;
  MOE_CUDA_TRY(moe::launch_grouped_gemm(g, st));
  // a6: down, fp32 rows in expert order for the weighted unpermute. (Folding
  // the routing weight into this epilogue, moe_down_gemm_weighted, writes the
  // rows in flat pair order: in fp32 that measured as fast on DeepSeek shapes
  // but slower on Qwen3 prefill, where the scattered 512-byte row segments
  // cost more than the combine saves; in bf16 it is faster but its per-term
  // rounding exceeds the output tolerance on rare DeepSeek outputs.)
  g.mode = prob->down_fp8 ? moe::kModeFp8Store : moe::kModeStore;
  g.N = H;
  g.K = F;
  g.A = h;
  g.B = w_down;
  g.A_scales = prob->down_fp8 ? h_scales : nullptr;
  g.B_scales = prob->down_fp8 ? w_down_scales : nullptr;
  g.C_scales = nullptr;
  // y in f16e (half the bytes of fp32, 11 significant bits per value) wherever
  // the down GEMM's tiling stores it, else fp32. Down GEMM + unpermute on B200,
  // f16e against fp32 (us): qwen3_prefill 136 + 42 vs 136 + 60, qwen3_decode
  // 77 + 12 vs 83 + 15, dsv3_decode_fp8 552 + 23 vs 548 + 33, dsv3_prefill
  // 1381 + 124 vs 1406 + 173.
  int8_t* y_exp = reinterpret_cast<int8_t*>(base + w.y_exp);
  g.C = y;
  g.out_f16e = 1;
  g.C_exps = y_exp;
  const bool f16e = moe::grouped_gemm_f16e_supported(g);
  if (!f16e) {
    g.out_f16e = 0;
    g.C_exps = nullptr;
    g.out_f32 = 1;
  }
  MOE_CUDA_TRY(moe::launch_grouped_gemm(g, st));
  g_last_launches += 2;

  if (beside) MOE_CUDA_TRY(cudaStreamWaitEvent(st, join.e, 0));
  // a7
  if (f16e)
    MOE_CUDA_TRY(moe::launch_unpermute_f16e(y, y_exp, tables + L.row_of_pair, topk_weights, T, k,
                                            H, scale, addend, out, st));
  else
    MOE_CUDA_TRY(moe::launch_unpermute(y, tables + L.row_of_pair, topk_weights, T, k, H, scale,
                                       addend, out, st));
  g_last_launches += 1;
  return MOE_OK;
}

size_t moe_shared_workspace_bytes(int32_t T, int32_t H, int32_t F_s, int32_t tp_size) {
  if (T < 0 || H <= 0 || F_s <= 0 || tp_size <= 0 || F_s % tp_size != 0) return 0;
  const int64_t Fp = F_s / tp_size;
  return static_cast<size_t>(1024 + round_up(static_cast<int64_t>(T) * Fp * 2, 1024));
}

moe_status moe_shared_expert_forward(int32_t T, int32_t H, int32_t F_s, int32_t tp_size,
                                     int32_t tp_rank, const void* hidden, const void* w_gate_up,
                                     const void* w_down, int32_t out_f32, void* out,
                                     void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (hidden == nullptr || w_gate_up == nullptr || w_down == nullptr || out == nullptr ||
      workspace == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out) ||
      !aligned16(workspace))
    return MOE_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || H % 64 != 0 || F_s <= 0 || tp_size <= 0 || tp_rank < 0 ||
      tp_rank >= tp_size || F_s % tp_size != 0)
    return MOE_ERR_INVALID_ARG;
  const int64_t Fp = F_s / tp_size;
  if (Fp % 64 != 0) return MOE_ERR_INVALID_ARG;
  if (tp_size > 1 && (H % 256 != 0 || Fp % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < moe_shared_workspace_bytes(T, H, F_s, tp_size)) return MOE_ERR_WORKSPACE;
  g_last_launches = 0;
  if (T == 0) return MOE_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  void* h = base + 1024;
  MOE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
  const size_t r = static_cast<size_t>(tp_rank);
  // gate+up with the SwiGLU epilogue: this rank's gate rows and, F_s rows
  // further, its up rows, addressed in the complete w_gate_up
  moe::GemmLaunch d;
  d.rows = T;
  d.E = 1;
  d.status = status;
  d.mode = moe::kModeSwiglu;
  d.N = static_cast<int>(2 * Fp);
  d.K = H;
  d.A = hidden;
  d.B = static_cast<const uint16_t*>(w_gate_up) + r * Fp * H;  // bf16 elements
  if (tp_size > 1) {
    d.up_off = F_s;
    d.b_rows = 2LL * F_s - static_cast<long long>(r) * Fp;
  }
  d.C = h;
  if (tp_size > 1 && !moe::grouped_gemm_pair_supported(d)) return MOE_ERR_UNSUPPORTED;
  MOE_CUDA_TRY(moe::launch_grouped_gemm(d, st));
  // down: this rank's F_p columns of the complete w_down (row pitch F_s)
  d.mode = moe::kModeStore;
  d.N = H;
  d.K = static_cast<int>(Fp);
  d.A = h;
  d.B = static_cast<const uint16_t*>(w_down) + r * Fp;
  d.up_off = 0;
  d.b_rows = 0;
  if (tp_size > 1) d.ldb = F_s;
  d.C = out;
  d.out_f32 = out_f32 != 0;
  if (tp_size > 1 && !moe::grouped_gemm_pair_supported(d)) return MOE_ERR_UNSUPPORTED;
  MOE_CUDA_TRY(moe::launch_grouped_gemm(d, st));
  g_last_launches = 2;
  return MOE_OK;
}

int32_t moe_dual_blocks(const moe_problem* prob, int32_t M) {
  if (M < 0) return -1;
  if (prob == nullptr) return (M + 127) / 128;
  if (check_problem(prob, false) != MOE_OK || prob->padding_M != 128) return -1;
  if (static_cast<int64_t>(prob->T) * prob->top_k != M) return -1;
  moe_tables_layout L;
  fill_layout(prob, &L);
  return L.M_blk;
}

namespace {

moe_status quant_dual_common(const moe_problem* prob, const int32_t* tables, int32_t M,
                             int32_t K, const void* x, int32_t trans_mode, uint8_t* q, float* s,
                             uint8_t* qT, float* sT, float* debug_h, int swiglu,
                             moe_stream_t stream) {
  if ((prob == nullptr) != (tables == nullptr)) return MOE_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (trans_mode != MOE_TRANS_PER_BLOCK && trans_mode != MOE_TRANS_PER_TILE)
    return MOE_ERR_INVALID_ARG;
  const int32_t M_blk = moe_dual_blocks(prob, M);
  if (M_blk < 0) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  if (x == nullptr || q == nullptr || s == nullptr || qT == nullptr || sT == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(qT) || (debug_h && !aligned16(debug_h)))
    return MOE_ERR_INVALID_ARG;
  moe::DualLaunch d;
  d.M = M;
  d.K = K;
  d.M_blk = M_blk;
  if (prob != nullptr) {
    moe_tables_layout L;
    fill_layout(prob, &L);
    d.E = prob->E;
    d.sizes = tables + L.group_sizes;
    d.offsets = tables + L.group_offsets;
    d.padded = tables + L.group_padded_offsets;
    d.idx_for_bx = tables + L.group_idx_for_bx;
  }
  d.x = x;
  d.swiglu = swiglu;
  d.trans_block = trans_mode == MOE_TRANS_PER_BLOCK;
  d.q = q;
  d.s = s;
  d.qT = qT;
  d.sT = sT;
  d.debug_h = debug_h;
  MOE_CUDA_TRY(moe::launch_quant_dual(d, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

}  // namespace

moe_status moe_quant_dual(const moe_problem* prob, const int32_t* tables, int32_t M, int32_t K,
                          const void* x, int32_t trans_mode, uint8_t* q, float* s, uint8_t* qT,
                          float* sT, moe_stream_t stream) {
  return quant_dual_common(prob, tables, M, K, x, trans_mode, q, s, qT, sT, nullptr, 0, stream);
}

moe_status moe_swiglu_quant_dual(const moe_problem* prob, const int32_t* tables, int32_t M,
                                 int32_t F, const void* gate_up, int32_t trans_mode, uint8_t* q,
                                 float* s, uint8_t* qT, float* sT, float* debug_h,
                                 moe_stream_t stream) {
  return quant_dual_common(prob, tables, M, F, gate_up, trans_mode, q, s, qT, sT, debug_h, 1,
                           stream);
}

moe_status moe_swiglu_backward(int32_t M, int32_t F, const void* gate_up, const void* grad_h,
                               void* grad_gate_up, moe_stream_t stream) {
  if (M < 0 || F <= 0 || F % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  if (gate_up == nullptr || grad_h == nullptr || grad_gate_up == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(gate_up) || !aligned16(grad_h) || !aligned16(grad_gate_up))
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_swiglu_backward(M, F, gate_up, grad_h, grad_gate_up,
                                           reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_ep_split_ids(int32_t n, int32_t E_local, int32_t world, const int32_t* ids,
                            int32_t* rank_ids, int32_t* local_ids, moe_stream_t stream) {
  if (n < 0 || E_local < 1 || world < 1) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(E_local) * world > (1ll << 30)) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (ids == nullptr || rank_ids == nullptr || local_ids == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_split_ids(n, E_local, world, ids, rank_ids, local_ids,
                                     reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_gather_rows(int32_t n_dst, int32_t n_src, int64_t row_bytes, const int32_t* map,
                           const void* src, void* dst, int32_t* dev_status, moe_stream_t stream) {
  if (n_dst < 0 || n_src < 0 || row_bytes <= 0 || row_bytes % 4 != 0) return MOE_ERR_INVALID_ARG;
  if (row_bytes / 4 > (1ll << 30)) return MOE_ERR_INVALID_ARG;
  if (n_dst == 0) return MOE_OK;
  if (map == nullptr || dst == nullptr || (n_src > 0 && src == nullptr)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dst) & 3) != 0 || (reinterpret_cast<uintptr_t>(src) & 3) != 0)
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(moe::launch_gather_rows_any(n_dst, n_src, row_bytes, map, src, dst, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_decode_device_status(int32_t dev_status) {
  if (dev_status == 0) return MOE_OK;
  if (dev_status & MOE_DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
  return MOE_ERR_DEVICE_FLAG;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE_FLAG: return "MOE_ERR_DEVICE_FLAG";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_cuda_error(void) { return g_last_error; }

int32_t moe_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
