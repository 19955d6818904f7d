/*
 * moe.h - C ABI of the B200 (sm_100a) routed mixture-of-experts expert forward.
 *
 * The library runs, on one GPU and on the caller's CUDA stream:
 *   a1 top-k routing of router logits (softmax or sigmoid scores, optionally
 *      renormalised over the k picks);
 *   a2 the expert-sorted permutation and its dispatch tables (group_sizes,
 *      group_offsets, group_padded_offsets, group_idx_for_bx) from a chunked
 *      histogram + stable scan on the device, with no host synchronisation;
 *   a3 the permute gather of token rows into expert order;
 *   a4 a persistent grouped gate+up GEMM on tcgen05 tensor cores (TMEM
 *      accumulators, TMA loads whose out-of-bounds zero fill covers ragged
 *      expert tails);
 *   a5 SiLU(gate)*up in that GEMM's epilogue, optionally quantised to FP8
 *      E4M3 with one fp32 scale per 1x128 tile;
 *   a6 a grouped down GEMM, bf16 or FP8 with 128x128 block-scaled weights;
 *   a7 a weighted unpermute that folds in routed_scaling_factor.
 *
 * Sources of the operations (web pages, cited by title and section):
 *   [TUT07]  TileLang tutorial "Example 07: MoE dispatch contract and
 *            quantised GEMM", section 1 (moe_dispatch_contract.py: the four
 *            tables, m_start recovery, the 9-token example) and section 2
 *            (skeletons.py: routed grouped GEMM -> SiLU -> down -> weighted
 *            write-back).
 *   [PR1580] TileOPs PR #1580 "Grouped-GEMM TMA OOB zero-fill + unpermute
 *            out=": Grouped-GEMM kernel (C[e] = A[e] @ B[e]^T, A descriptor over
 *            all rows, hardware zero fill of the partial last tile, no padding
 *            copies or host sync) and Unpermute (out= buffer, scaling folded in
 *            before the cast/store).
 *   [PR778]  TileOPs PR #778 "SharedFusedMoE with native shared expert kernel
 *            and TP support": Design (caller passes complete weights; merged
 *            gate_up weight holds gate rows then up rows; shared expert
 *            gate+up -> SiLU-mul -> down added to the routed output).
 *   [PR2089] XTuner PR #2089 "Fuse MoE activation FP8 quantization kernels":
 *            Changes (SiLU(gate)*up fused with W2-input 1x128 per-tile FP8
 *            quantisation, no bf16 activation materialised).
 *   [PR809]  pypto-lib PR #809 "predicate empty routed-expert stages": experts
 *            with zero rows skip all compute.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller (PyTorch
 *     supplies them). Row-major, densely packed, 16-byte aligned. bf16 values
 *     are passed as `const void*` / `void*` (2 bytes each, IEEE bfloat16).
 *   - The library never allocates, frees or synchronises. Every call only
 *     enqueues work on `stream` (NULL = the legacy default stream); a return of
 *     MOE_OK means "validated and enqueued".
 *   - Synchronous errors (bad arguments, unsupported shapes, a CUDA launch
 *     error) are returned as moe_status before or at launch.
 *   - Errors only the device can see (an expert id outside [0, E), a pipeline
 *     wait that exceeded its time limit) are OR-ed as MOE_DEV_* flags into the
 *     caller's int32 `dev_status` word, to be read after the stream is
 *     synchronised. Kernels never trap: an out-of-range id is skipped, a wait
 *     that times out makes the kernel drain its in-flight copies, free its
 *     tensor memory and return.
 *   - Symbols: T tokens, k = top_k, E experts, H hidden size, F expert FFN size,
 *     P = T*k (token, expert) pairs.
 */
#ifndef MOE_B200_MOE_H_
#define MOE_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,   /* null pointer, negative size, misaligned pointer, bad enum */
  MOE_ERR_UNSUPPORTED = -2,   /* shape outside what the kernels handle (see each call) */
  MOE_ERR_WORKSPACE = -3,     /* workspace smaller than moe_workspace_bytes() */
  MOE_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed (message: moe_last_cuda_error) */
  MOE_ERR_TIMEOUT = -5,       /* reported by moe_decode_device_status for MOE_DEV_TIMEOUT */
  MOE_ERR_DEVICE_FLAG = -6    /* reported by moe_decode_device_status for other device flags */
} moe_status;

/* Flags OR-ed into the int32 device status word. */
enum {
  MOE_DEV_BAD_EXPERT_ID = 1,  /* a topk id outside [0, E): that pair was skipped */
  MOE_DEV_TIMEOUT = 2,        /* a kernel's bounded wait ran out; its outputs are invalid */
  MOE_DEV_BAD_TABLES = 4      /* group tables inconsistent with the GEMM's shape */
};

enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };

/* Epilogues of moe_grouped_gemm. */
enum {
  MOE_EPI_STORE = 0,       /* C bf16 [rows, N] = A @ B^T */
  MOE_EPI_SWIGLU = 1,      /* C bf16 [rows, N/2] = SiLU(G[:, :N/2]) * G[:, N/2:] */
  MOE_EPI_SWIGLU_FP8 = 2,  /* C e4m3 [rows, N/2] + C_scales fp32 [rows, N/256] */
  MOE_EPI_STORE_F32 = 3,   /* C fp32 [rows, N] = A @ B^T (the accumulator, unrounded) */
  MOE_EPI_STORE_F16E = 4   /* C fp16 [rows, N] and one int8 exponent per row and 128
                              columns in C_scales (read as int8_t [rows, N/128]):
                              A @ B^T = C * 2^e (see moe_unpermute_f16e) */
};

/* Tiling choice, OR-ed into moe_grouped_gemm's `epilogue` argument. Both
 * compute the same result.
 *   MOE_TILE_AUTO        the library's choice: weight-row pairs for bf16 problems
 *                        whose experts average more than 64 rows (and dense
 *                        problems), else weight rows where supported, else
 *                        token rows
 *   MOE_TILE_TOKEN_ROWS  128 token rows x N columns per tile (every epilogue)
 *   MOE_TILE_WEIGHT_ROWS 128 weight rows x (the expert's tokens, <= 256, rounded
 *                        up to 16) per tile: MMA work follows the real group
 *                        sizes; MOE_EPI_STORE / STORE_F32 (N % 128 == 0; in
 *                        FP8 mode also K <= 2048) or bf16 MOE_EPI_SWIGLU
 *                        (N % 128 == 0) only, else MOE_ERR_UNSUPPORTED.
 *   MOE_TILE_WEIGHT_ROWS_PAIR  256 weight rows x (tokens, <= 256) per tile,
 *                        computed by two CTAs of a cluster with one 256-row
 *                        MMA (each CTA fetches half of the weight rows and half
 *                        of the token rows); bf16 only: MOE_EPI_STORE /
 *                        STORE_F32 (N % 256 == 0) or MOE_EPI_SWIGLU
 *                        (N % 256 == 0), K % 64 == 0, E <= 1024, else
 *                        MOE_ERR_UNSUPPORTED. */
enum {
  MOE_TILE_AUTO = 0x00,
  MOE_TILE_TOKEN_ROWS = 0x10,
  MOE_TILE_WEIGHT_ROWS = 0x20,
  MOE_TILE_WEIGHT_ROWS_PAIR = 0x30
};

/* Flag OR-ed into moe_grouped_gemm's `epilogue`: the permutation is fused into
 * the GEMM. A is then the hidden states bf16 [prob->T, K] (K == prob->H) and
 * row r of the grouped problem is A[pair_of_row[r] / top_k] (pair_of_row from
 * `tables`), the rows x_perm would hold (TileOPs PR #1580, copy elimination;
 * TileLang tutorial "Example 07", section 1, permutation). Grouped mode, bf16,
 * the weight-row pair tiling only (MOE_TILE_AUTO or MOE_TILE_WEIGHT_ROWS_PAIR
 * with its shape rules), else MOE_ERR_UNSUPPORTED; without tables
 * MOE_ERR_INVALID_ARG. The rows are fetched with four-row TMA gathers once per
 * weight block; on B200 this measured slower than writing x_perm once with
 * moe_route_permute, so moe_experts_forward does not use it. */
enum { MOE_A_GATHER = 0x100 };

/* One MoE layer's shape and routing options. */
typedef struct moe_problem {
  int32_t T;            /* tokens (>= 0; 0 is a no-op) */
  int32_t H;            /* hidden size: multiple of 64 (of 128 with down_fp8) */
  int32_t F;            /* expert FFN size: multiple of 64 (of 128 with down_fp8) */
  int32_t E;            /* routed experts, 1..1024 */
  int32_t top_k;        /* 1..32; at most E for routing and the forward (k distinct
                           experts); tables, GEMMs and unpermute over given ids
                           accept repeated groups (e.g. the ranks of expert
                           parallelism) */
  int32_t padding_M;    /* group_padded_offsets alignment = M-block height
                           ("block_token" in [TUT07]); the GEMMs need 128 */
  int32_t score_fn;     /* MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID */
  int32_t renormalize;  /* 1: weights renormalised over the k picks */
  float routed_scaling_factor; /* applied in the unpermute (a7), not in routing */
  int32_t down_fp8;     /* 1: FP8 1x128 activations and 128x128 block-scaled down weights */
  int32_t F_shared;     /* shared expert FFN size (multiple of 64), 0 = none */
} moe_problem;

/* Layout of the int32 dispatch-table buffer written by moe_route_permute.
 * Offsets are in int32 elements from the buffer's start ([TUT07] section 1):
 *   group_sizes[E]            pairs routed to each expert
 *   group_offsets[E+1]        exclusive scan of sizes; [E] = P
 *   group_padded_offsets[E+1] exclusive scan of ceil(size/padding_M)*padding_M
 *   group_idx_for_bx[M_blk]   M-block -> expert: the largest g whose padded
 *                             offset is <= bx*padding_M; M_blk = ceil(P/padding_M)+E
 *   row_of_pair[P]            permuted row of flat pair p = t*k + j; experts in
 *                             index order, pairs of one expert in flat order
 *   pair_of_row[P]            inverse permutation (-1 for rows left empty by
 *                             out-of-range ids)
 *   chunk_counts[...]         scratch of the table builder (per-chunk expert
 *                             counts); contents unspecified */
typedef struct moe_tables_layout {
  int64_t group_sizes;
  int64_t group_offsets;
  int64_t group_padded_offsets;
  int64_t group_idx_for_bx;
  int64_t row_of_pair;
  int64_t pair_of_row;
  int64_t chunk_counts;
  int64_t total_int32;  /* elements the buffer must hold */
  int32_t M_blk;
  int32_t P;
} moe_tables_layout;

/* Fills *out for `prob`. Errors: MOE_ERR_INVALID_ARG for null or bad sizes. */
moe_status moe_get_tables_layout(const moe_problem* prob, moe_tables_layout* out);

/* Bytes of device workspace moe_experts_forward needs for `prob` (0 on a bad
 * problem). The first 4 bytes of the workspace are the call's int32 device
 * status word (see MOE_DEV_*); the rest holds the tables, the permuted rows,
 * the SwiGLU output (bf16, or e4m3 codes + fp32 scales), the down output and
 * the shared expert's intermediates, each 1024-byte aligned. */
size_t moe_workspace_bytes(const moe_problem* prob);

/* a1: top-k routing ([PR778] Benchmark: sigmoid routing for DeepSeek/Kimi-K2).
 * logits fp32 [T, E] -> topk_ids int32 [T, k] (largest logit first; equal
 * logits: lower expert index first) and topk_weights fp32 [T, k]:
 *   softmax+renorm: w_j = e_j / sum_{i<k} e_i, e_j = exp(l_j - l_top1)
 *   softmax:        w_j = exp(l_j - max l) / sum over all E (index order)
 *   sigmoid:        s_j = 1/(1+exp(-l_j)); renorm w_j = s_j / sum_{i<k} s_i
 * in float32 with a fixed exp (Cody-Waite reduction, degree-7 Taylor), sums
 * in slot order, IEEE division: results are reproducible bit for bit.
 * routed_scaling_factor is NOT applied here. */
moe_status moe_route_topk(const moe_problem* prob, const float* logits,
                          int32_t* topk_ids, float* topk_weights, moe_stream_t stream);

/* a1 (optional) + a2 + a3 ([TUT07] section 1; [PR1580] no host sync).
 * If `logits` is non-null, routes first (as moe_route_topk) into topk_ids /
 * topk_weights; otherwise topk_ids [T, k] is an input and topk_weights unused.
 * Writes the dispatch tables into `tables` (moe_tables_layout) and, if
 * `hidden` [T, H] bf16 is non-null, x_perm [P, H] bf16 with
 * x_perm[row_of_pair[p]] = hidden[p / k]. Any padding_M >= 1 is accepted.
 * Device flags: MOE_DEV_BAD_EXPERT_ID into *dev_status (required). */
moe_status moe_route_permute(const moe_problem* prob, const float* logits,
                             int32_t* topk_ids, float* topk_weights,
                             const void* hidden, void* x_perm, int32_t* tables,
                             int32_t* dev_status, moe_stream_t stream);

/* a4 / a6: grouped GEMM C = A @ B[e]^T over each expert's rows
 * ([PR1580] Grouped-GEMM kernel), persistent, tcgen05 + TMEM + TMA.
 *   tables non-null (grouped): A [P, K] rows in expert order (P = T*k of
 *     `prob`), B [E, N, K]; M-block bx covers rows of expert group_idx_for_bx[bx]
 *     (padding_M must be 128); experts with no rows are never scheduled.
 *   tables null (dense, one group): A [M_rows, K], B [N, K].
 * bf16 mode (A_scales == B_scales == NULL): A, B bf16; K % 64 == 0.
 *   MOE_EPI_STORE:      C bf16 [rows, N], N % 64 == 0.
 *   MOE_EPI_STORE_F32:  C fp32 [rows, N], N % 64 == 0.
 *   MOE_EPI_SWIGLU:     N = 2F with gate = B rows [0,F), up = rows [F,2F)
 *                       ([PR778] Design); C bf16 [rows, F]; F % 64 == 0.
 *   MOE_EPI_SWIGLU_FP8: as SWIGLU, then per row and 128-column tile
 *                       s = amax/448, q = e4m3_rn_satfinite(h/s) (s = 0, q = 0
 *                       for an all-zero tile) ([PR2089] Changes); C e4m3 codes
 *                       [rows, F], C_scales fp32 [rows, F/128]; F % 128 == 0.
 *                       debug_h (nullable) receives the fp32 h [rows, F].
 * FP8 mode (A_scales and B_scales non-null): A e4m3 [rows, K] with A_scales
 *   fp32 [rows, K/128]; B e4m3 [E, N, K] with B_scales fp32 [E, N/128, K/128];
 *   C [rows, N] = sum over K-blocks kb of sa[r,kb]*sb[n/128,kb]*(A_kb @ B_kb^T),
 *   bf16 with MOE_EPI_STORE or fp32 with MOE_EPI_STORE_F32; N % 128 == 0,
 *   K % 128 == 0.
 * MOE_EPI_STORE_F16E (bf16 or FP8 operands): C fp16 [rows, N] and int8
 *   exponents in C_scales [rows, N/128], result = C * 2^e per row and
 *   128-column block (see moe_unpermute_f16e); N % 128 == 0; the weight-row
 *   and weight-row pair tilings only (MOE_TILE_TOKEN_ROWS, or an automatic
 *   choice of it: MOE_ERR_UNSUPPORTED).
 * Device flags: MOE_DEV_TIMEOUT into *dev_status (required). */
moe_status moe_grouped_gemm(const moe_problem* prob, int32_t M_rows, int32_t N, int32_t K,
                            const void* A, const float* A_scales,
                            const void* B, const float* B_scales,
                            const int32_t* tables, int32_t epilogue,
                            void* C, float* C_scales, float* debug_h,
                            int32_t* dev_status, moe_stream_t stream);

/* a5 standalone ([PR2089] Changes): SwiGLU and/or 1x128 FP8 quantisation.
 *   gate_up bf16 [M, 2F] non-null: h = SiLU(gate_up[:, :F]) * gate_up[:, F:]
 *     in fp32; out_fp8 == 0 -> out bf16 [M, F] (round to nearest even);
 *     out_fp8 == 1 -> out e4m3 [M, F] + scales fp32 [M, ceil(F/128)].
 *   gate_up NULL, h fp32 [M, F] non-null: quantise h (out_fp8 must be 1).
 * Quantisation rule as MOE_EPI_SWIGLU_FP8; a partial last tile takes amax
 * over its valid columns. F % 4 == 0. */
moe_status moe_swiglu_quant(int32_t M, int32_t F, const void* gate_up, const float* h,
                            int32_t out_fp8, void* out, float* scales, moe_stream_t stream);

/* a7 ([PR1580] Unpermute): out bf16 [T, H] =
 *   RNE_bf16( scale * sum_{j<k} topk_weights[t,j] * y[row_of_pair[t*k+j]] + addend[t] )
 * with the sum in fp32 in slot order j; y fp32 [P, H] (the down GEMM's
 * MOE_EPI_STORE_F32 output: kept unrounded so a bf16 intermediate adds no
 * error before the single final cast); addend fp32 [T, H] or NULL; tables as
 * written by moe_route_permute (row -1 contributes nothing). */
moe_status moe_unpermute(const moe_problem* prob, const float* y, const int32_t* tables,
                         const float* topk_weights, float scale, const float* addend,
                         void* out, moe_stream_t stream);

/* a7 from the down GEMM's MOE_EPI_STORE_F16E output (no counterpart on the
 * pages, which hand a bf16 y to the unpermute): y16 fp16 [P, H] and y_exp int8
 * [P, H/128] with y[r, c] = y16[r, c] * 2^y_exp[r, c/128]. The exponent of a
 * row's 128-column block puts the block's largest magnitude in [2^14, 2^15),
 * so every value keeps 11 significant bits (8x bf16's precision) at any fp32
 * range, in half the bytes of fp32; moe_experts_forward stores y this way when
 * its down GEMM's tiling supports it. Otherwise as moe_unpermute: each row is
 * decoded exactly to fp32, then out[t] = RNE_bf16(scale * sum_j w[t,j] *
 * y[row_of_pair[t*k+j]] + addend[t]) with fp32 sums in slot order. Needs
 * H % 128 == 0 and 16-byte-aligned y16, out and addend, else
 * MOE_ERR_INVALID_ARG. */
moe_status moe_unpermute_f16e(const moe_problem* prob, const void* y16, const int8_t* y_exp,
                              const int32_t* tables, const float* topk_weights, float scale,
                              const float* addend, void* out, moe_stream_t stream);

/* a6 with the routing weight folded into the epilogue ([PR1580] Unpermute's
 * scale folding, applied one step earlier, as the down projection's per-row
 * scale × routing weight of [PR778]): for every permuted row r with a pair
 * p = pair_of_row[r] (from `tables`),
 *   y_w [P, N], row p = scale * topk_weights[p] * (A @ B[e]^T)[r]
 * i.e. the down GEMM's rows, weighted, in flat pair order p = t*k + j; rows of
 * pairs without a permuted row are not written. `epilogue` = MOE_EPI_STORE
 * (y_w bf16, rounded to nearest even: half the bytes, the rounding of the bf16
 * y that [PR1580]'s unpermute reads) or MOE_EPI_STORE_F32 (y_w fp32, unrounded), OR-ed with
 * MOE_TILE_AUTO, MOE_TILE_WEIGHT_ROWS or MOE_TILE_WEIGHT_ROWS_PAIR and their
 * shape rules (N % 128 == 0; pairs: bf16 operands, N % 256 == 0);
 * MOE_TILE_TOKEN_ROWS: MOE_ERR_UNSUPPORTED. A, A_scales, B, B_scales as for
 * moe_grouped_gemm's store epilogues (bf16, or FP8 block-scaled with
 * K <= 2048); tables as written by moe_route_permute (padding_M 128);
 * topk_weights fp32 [T, k]. Device flags: MOE_DEV_TIMEOUT into *dev_status
 * (required). */
moe_status moe_down_gemm_weighted(const moe_problem* prob, int32_t N, int32_t K, const void* A,
                                  const float* A_scales, const void* B, const float* B_scales,
                                  const int32_t* tables, const float* topk_weights, float scale,
                                  int32_t epilogue, void* y_w, int32_t* dev_status,
                                  moe_stream_t stream);

/* a7 after moe_down_gemm_weighted: the deterministic combine
 *   out bf16 [T, H] = RNE_bf16( sum_{j<k} y_w[t*k+j] + addend[t] )
 * with fp32 sums in slot order j, then the addend (fp32 [T, H] or NULL);
 * pairs with row_of_pair == -1 contribute nothing. y_w [T*k, H] fp32
 * (y_f32 != 0) or bf16; H % 8 == 0. */
moe_status moe_combine(const moe_problem* prob, const void* y_w, int32_t y_f32,
                       const int32_t* tables, const float* addend, void* out,
                       moe_stream_t stream);

/* Offline weight preparation for the FP8 down GEMM: for each of `batch`
 * matrices w bf16 [N, K], per 128x128 block s = amax/448 and
 * q = e4m3_rn_satfinite(w/s) (all-zero block: s = 0, q = 0); q uint8
 * [batch, N, K], scales fp32 [batch, ceil(N/128), ceil(K/128)]. */
moe_status moe_quantize_weight_128x128(int32_t batch, int32_t N, int32_t K, const void* w,
                                       uint8_t* q, float* scales, moe_stream_t stream);

/* The whole routed-experts forward (a2..a7, plus the shared expert when
 * prob->F_shared > 0): from given topk_ids / topk_weights [T, k],
 *   out bf16 [T, H] = RNE_bf16( scale * sum_j w[t,j] * MLP_{e(t,j)}(hidden[t])
 *                               + shared_MLP(hidden[t]) )
 * with MLP_e(x) = W_down[e] (bf16(SiLU(G_gate) * G_up)), G = W_gate_up[e] x.
 *   w_gate_up bf16 [E, 2F, H]; w_down bf16 [E, H, F], or with prob->down_fp8
 *   e4m3 [E, H, F] plus w_down_scales fp32 [E, H/128, F/128] (see
 *   moe_quantize_weight_128x128); ws_gate_up bf16 [2F_s, H], ws_down bf16
 *   [H, F_s] when F_shared > 0 (else NULL).
 * Needs prob->padding_M == 128. `workspace` (ws_bytes >= moe_workspace_bytes)
 * is caller-owned device memory; its first int32 is this call's device status
 * (zeroed by the call, then OR-ed with MOE_DEV_* flags).
 * Streams: everything is ordered on `stream`. When F_shared > 0 and the routed
 * experts average at most 64 rows (T*k <= 64*E), the shared expert's two GEMMs
 * run on a second, library-owned stream of the current device (created on first
 * use outside stream capture, never destroyed; while `stream` is being captured
 * and that stream does not exist yet, they run on `stream`), forked from
 * `stream` by an event before them and joined
 * back by an event before the unpermute; the routed GEMMs then use the other SMs.
 * Under CUDA graph capture of `stream` the fork and join are graph edges. */
moe_status moe_experts_forward(const moe_problem* prob, const void* hidden,
                               const int32_t* topk_ids, const float* topk_weights,
                               const void* w_gate_up, const void* w_down,
                               const float* w_down_scales,
                               const void* ws_gate_up, const void* ws_down,
                               float scale, void* out, void* workspace, size_t ws_bytes,
                               moe_stream_t stream);

/* One tensor-parallel rank's share of the shared expert, a dense SwiGLU MLP on
 * all tokens (TileOPs PR #778 "SharedFusedMoE with native shared expert kernel
 * and TP support": Design, TP split convention, Partial output contract).
 * The caller passes the COMPLETE weights; rank r of tp_size owns
 * F_p = F_s / tp_size FFN columns:
 *   gate rows [r*F_p, (r+1)*F_p) and up rows F_s + [r*F_p, (r+1)*F_p) of
 *   w_gate_up bf16 [2*F_s, H] (column parallel), and columns
 *   [r*F_p, (r+1)*F_p) of w_down bf16 [H, F_s] (row parallel),
 * all read in place (no slice copies), and writes
 *   out [T, H] = bf16(SiLU(x Wg^T) * (x Wu^T)) Wd^T   (this rank's slices)
 * as fp32 (out_f32 = 1) or bf16 (0). With tp_size > 1, `out` is a partial
 * sum: the caller all-reduces it over the ranks and adds the routed output.
 * Errors: null or unaligned pointers, T < 0, H or F_p not a multiple of 64,
 * tp_rank outside [0, tp_size), F_s % tp_size != 0 -> MOE_ERR_INVALID_ARG;
 * tp_size > 1 also needs H % 256 == 0 and F_p % 128 == 0, else
 * MOE_ERR_UNSUPPORTED; ws_bytes < moe_shared_workspace_bytes ->
 * MOE_ERR_WORKSPACE. `workspace` holds h and the device status word (its
 * first int32, zeroed by the call). T == 0 enqueues nothing. */
size_t moe_shared_workspace_bytes(int32_t T, int32_t H, int32_t F_s, int32_t tp_size);
moe_status moe_shared_expert_forward(int32_t T, int32_t H, int32_t F_s, int32_t tp_size,
                                     int32_t tp_rank, const void* hidden, const void* w_gate_up,
                                     const void* w_down, int32_t out_f32, void* out,
                                     void* workspace, size_t ws_bytes, moe_stream_t stream);

/* ---- Training-side FP8 activation layouts (XTuner PR #2089 "Fuse MoE
 * activation FP8 quantization kernels", Changes) --------------------------
 *
 * moe_quant_dual quantises an activation x bf16 [M, K] in one pass into
 *   - the forward layout: q e4m3 [M, K], s fp32 [M, K/128] (one scale per
 *     1x128 row tile; per_tile_quant), and
 *   - a transposed, expert-padded copy for the weight-gradient GEMM:
 *     qT e4m3 [K, 128*M_blk] where the rows of each expert start a fresh
 *     128-token block (expand_128x): row r of expert g lands in column
 *     group_padded_offsets[g] + (r - group_offsets[g]) (the block layout of
 *     the TileLang tutorial "Example 07" section 1 with block_token 128);
 *     padding columns are 0. Scales sT fp32 [K/128, M_blk] (trans_mode
 *     MOE_TRANS_PER_BLOCK: one per 128x128 block) or [K, M_blk]
 *     (MOE_TRANS_PER_TILE: one per 1x128 tile of a qT row).
 * Scale rule: s = amax/448 (IEEE division), code = e4m3_rn_satfinite(x/s),
 * all-zero tile/block: s = 0 and codes 0.
 * Grouped mode: prob (padding_M 128) and `tables` from moe_route_permute,
 * M == prob->T * prob->top_k, M_blk = the tables' M_blk. Dense mode (prob
 * and tables NULL): one group, M_blk = ceil(M/128). Needs K % 128 == 0 and
 * 16-byte-aligned pointers, else MOE_ERR_INVALID_ARG; M == 0 is a no-op.
 * moe_dual_blocks returns M_blk (or -1 for invalid arguments). */
enum { MOE_TRANS_PER_BLOCK = 0, MOE_TRANS_PER_TILE = 1 };
int32_t moe_dual_blocks(const moe_problem* prob, int32_t M);
moe_status moe_quant_dual(const moe_problem* prob, const int32_t* tables, int32_t M, int32_t K,
                          const void* x, int32_t trans_mode, uint8_t* q, float* s, uint8_t* qT,
                          float* sT, moe_stream_t stream);

/* The same with x = SiLU(gate) * up computed in fp32 from gate_up bf16
 * [M, 2F] (gate columns first) and never stored in bf16
 * (swiglu_per_tile_quant_with_trans_per_block / _per_tile); K = F. debug_h,
 * if not NULL, receives the fp32 h [M, F]. */
moe_status moe_swiglu_quant_dual(const moe_problem* prob, const int32_t* tables, int32_t M,
                                 int32_t F, const void* gate_up, int32_t trans_mode, uint8_t* q,
                                 float* s, uint8_t* qT, float* sT, float* debug_h,
                                 moe_stream_t stream);

/* Backward of h = SiLU(gate) * up (swiglu_backward): from gate_up bf16
 * [M, 2F] and grad_h bf16 [M, F], grad_gate_up bf16 [M, 2F] with
 *   grad_gate = grad_h * up * s * (1 + g * (1 - s)),  grad_up = grad_h * g * s,
 * s = 1 / (1 + e^-g), fp32 arithmetic. F % 8 == 0, 16-byte-aligned pointers,
 * else MOE_ERR_INVALID_ARG; M == 0 is a no-op. */
moe_status moe_swiglu_backward(int32_t M, int32_t F, const void* gate_up, const void* grad_h,
                               void* grad_gate_up, moe_stream_t stream);

/* ---- Expert parallelism helpers (experts split over `world` ranks of
 * E_local experts each; pypto-lib PR #809 "predicate empty routed-expert
 * stages": dispatch to the ranks owning the experts, per-rank expert counts,
 * empty local experts skipped). The exchange itself is the caller's
 * all-to-all; the rest of the path is the entry points above. -------------
 *
 * moe_ep_split_ids: for n expert ids, rank_ids[i] = id / E_local and
 * local_ids[i] = id % E_local; an id outside [0, world*E_local) gets rank
 * `world` (flagged by moe_route_permute as a bad id when the ranks are used
 * as its groups) and local id 0. n < 0, E_local < 1, world < 1 or null
 * pointers -> MOE_ERR_INVALID_ARG; n == 0 is a no-op. */
moe_status moe_ep_split_ids(int32_t n, int32_t E_local, int32_t world, const int32_t* ids,
                            int32_t* rank_ids, int32_t* local_ids, moe_stream_t stream);

/* moe_gather_rows: dst row r = src row map[r] for n_dst rows of row_bytes
 * bytes (a multiple of 4); map[r] < 0 gives a zero row; map[r] >= n_src gives
 * a zero row and ORs MOE_DEV_BAD_TABLES into *dev_status (if not NULL).
 * Caller-owned device memory; rows do not overlap between src and dst. */
moe_status moe_gather_rows(int32_t n_dst, int32_t n_src, int64_t row_bytes, const int32_t* map,
                           const void* src, void* dst, int32_t* dev_status, moe_stream_t stream);

/* Capacity of the library's built-in scratch area used by
 * moe_experts_forward_noalloc: 64 MiB of device memory. */
#define MOE_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* moe_experts_forward without a caller-supplied workspace: the pages have no
 * counterpart; this exists for callers that cannot allocate device memory.
 * Some callers have no way to obtain a scratch buffer: a plug-in running
 * inside a host program that owns every device allocation through its own
 * allocator and forbids others, or a service whose device-memory budget is
 * fixed when it starts. This call takes the same arguments as
 * moe_experts_forward minus (workspace, ws_bytes) and keeps its workspace in a
 * file-scope device array of MOE_NOALLOC_SCRATCH_BYTES bytes inside the
 * library; every GPU that loads the library holds that array until the
 * process exits.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library
 *     routine. Its first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - Problems whose moe_workspace_bytes() exceeds MOE_NOALLOC_SCRATCH_BYTES
 *     are rejected with MOE_ERR_WORKSPACE before anything is enqueued.
 *   - All calls share the one array and it keeps the last call's contents;
 *     the call itself clears what must start at zero (the status word).
 *     Calls whose work overlaps on the GPU (different streams, or different
 *     host threads on one device) race on the array: serialise them.
 *   - The device status word (MOE_DEV_* flags of the last call) is the
 *     array's first int32; moe_noalloc_read_status copies it out.
 *   - Argument and shape checks are moe_experts_forward's (T == 0 enqueues
 *     nothing and touches no device). */
moe_status moe_experts_forward_noalloc(const moe_problem* prob, const void* hidden,
                                       const int32_t* topk_ids, const float* topk_weights,
                                       const void* w_gate_up, const void* w_down,
                                       const float* w_down_scales,
                                       const void* ws_gate_up, const void* ws_down,
                                       float scale, void* out, moe_stream_t stream);

/* Copies the device status word of the last moe_experts_forward_noalloc call
 * on the current device (its MOE_DEV_* flags) into *host_status, with one
 * cudaMemcpyAsync on `stream`. Enqueue it after that call on the same stream;
 * *host_status is valid once the stream has been synchronised (decode it with
 * moe_decode_device_status). No counterpart on the pages. Errors: NULL
 * host_status -> MOE_ERR_INVALID_ARG; a failed CUDA call -> MOE_ERR_CUDA. */
moe_status moe_noalloc_read_status(int32_t* host_status, moe_stream_t stream);

/* Self-test of the bounded pipeline wait (no counterpart on the pages; the
 * pages' kernels have no time limits). Every wait on an mbarrier in this
 * library's kernels gives up after a fixed limit, ORs MOE_DEV_TIMEOUT into the
 * status word, raises its CTA's abort flag so the CTA's other waiting threads
 * stop too, drains what it has in flight against one deadline and frees its
 * tensor memory. This call runs that same wait in a one-CTA kernel on
 * mbarriers that nothing ever arrives on, with `limit_ns` (1e3 .. 1e9) in place
 * of the production limit, so a caller can check on its own GPU that a stalled
 * pipeline ends with a flag and a usable context. The kernel issues no copy
 * and no MMA. After the stream is synchronised: *dev_status has
 * MOE_DEV_TIMEOUT set, and dev_result int64 [6] (device memory, 8-byte
 * aligned) holds {first wait returned true (0 expected), its duration in ns
 * (>= limit_ns expected), a second thread's wait returned true (0 expected),
 * its duration in ns (the abort flag ended it, well before its own limit of
 * 10 * limit_ns), the teardown drain returned true (0 expected), its duration
 * in ns (>= limit_ns expected)}. The kernel takes about 2 * limit_ns.
 * Errors: NULL or misaligned pointers, limit_ns out of range ->
 * MOE_ERR_INVALID_ARG; a launch error -> MOE_ERR_CUDA. */
moe_status moe_selftest_bounded_wait(int64_t limit_ns, int32_t* dev_status, int64_t* dev_result,
                                     moe_stream_t stream);

/* Maps a device status word (copied to the host after a sync) to a status:
 * MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_FLAG. */
moe_status moe_decode_device_status(int32_t dev_status);

/* Static, human-readable name of a status. */
const char* moe_status_string(moe_status status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* moe_last_cuda_error(void);

/* Kernels the last moe_experts_forward call on this thread enqueued. */
int32_t moe_last_launch_count(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MOE_B200_MOE_H_ */
