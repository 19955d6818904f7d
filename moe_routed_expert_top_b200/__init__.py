"""Python binding of the B200 routed mixture-of-experts expert forward.

A thin ctypes layer over ``libmoe_b200.so`` (declared in ``include/moe.h``):
each function has the name of the C entry point, takes torch tensors (or
None), passes their device pointers and the current CUDA stream, and raises
``MoeError`` on a non-OK status. Every step of the path runs in the library's
CUDA kernels; there is no fallback. If the library is not built the first call
raises ``MoeLibraryMissing`` (build it with ``python -m
moe_routed_expert_top_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MoeError", "MoeLibraryMissing", "Problem", "make_problem", "lib", "library_path",
    "moe_get_tables_layout", "moe_workspace_bytes", "moe_route_topk", "moe_route_permute",
    "moe_grouped_gemm", "moe_swiglu_quant", "moe_unpermute", "moe_quantize_weight_128x128",
    "moe_experts_forward", "moe_decode_device_status", "moe_status_string",
    "moe_last_launch_count", "moe_shared_workspace_bytes", "moe_shared_expert_forward",
    "moe_dual_blocks", "moe_quant_dual", "moe_swiglu_quant_dual", "moe_swiglu_backward",
    "moe_ep_split_ids", "moe_gather_rows", "moe_down_gemm_weighted", "moe_combine",
    "moe_experts_forward_noalloc", "moe_noalloc_read_status", "moe_selftest_bounded_wait",
    "moe_unpermute_f16e", "EXPORTED_SYMBOLS",
    "MOE_OK", "MOE_EPI_STORE", "MOE_EPI_SWIGLU", "MOE_EPI_SWIGLU_FP8", "MOE_EPI_STORE_F32",
    "MOE_SCORE_SOFTMAX", "MOE_SCORE_SIGMOID", "MOE_DEV_BAD_EXPERT_ID", "MOE_DEV_TIMEOUT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = -1, -2, -3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_FLAG = -4, -5, -6
MOE_DEV_BAD_EXPERT_ID, MOE_DEV_TIMEOUT, MOE_DEV_BAD_TABLES = 1, 2, 4
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
MOE_EPI_STORE, MOE_EPI_SWIGLU, MOE_EPI_SWIGLU_FP8, MOE_EPI_STORE_F32 = 0, 1, 2, 3
MOE_EPI_STORE_F16E = 4
MOE_TILE_AUTO, MOE_TILE_TOKEN_ROWS, MOE_TILE_WEIGHT_ROWS = 0x00, 0x10, 0x20
MOE_TILE_WEIGHT_ROWS_PAIR = 0x30
MOE_A_GATHER = 0x100  # moe_grouped_gemm: A = hidden states, rows gathered through the tables
MOE_TRANS_PER_BLOCK, MOE_TRANS_PER_TILE = 0, 1

EXPORTED_SYMBOLS = (
    "moe_get_tables_layout", "moe_workspace_bytes", "moe_route_topk", "moe_route_permute",
    "moe_grouped_gemm", "moe_swiglu_quant", "moe_unpermute", "moe_quantize_weight_128x128",
    "moe_experts_forward", "moe_decode_device_status", "moe_status_string",
    "moe_last_cuda_error", "moe_last_launch_count", "moe_experts_forward_noalloc",
    "moe_shared_workspace_bytes", "moe_shared_expert_forward",
    "moe_dual_blocks", "moe_quant_dual", "moe_swiglu_quant_dual", "moe_swiglu_backward",
    "moe_ep_split_ids", "moe_gather_rows", "moe_down_gemm_weighted", "moe_combine",
    "moe_noalloc_read_status", "moe_selftest_bounded_wait", "moe_unpermute_f16e",
)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        name = _status_name(status)
        super().__init__(f"{where}: {name}{(' (' + detail + ')') if detail else ''}")


class MoeLibraryMissing(RuntimeError):
    pass


class Problem(ctypes.Structure):
    """Mirror of ``moe_problem``."""
    _fields_ = [
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("F", ctypes.c_int32),
        ("E", ctypes.c_int32), ("top_k", ctypes.c_int32), ("padding_M", ctypes.c_int32),
        ("score_fn", ctypes.c_int32), ("renormalize", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_float), ("down_fp8", ctypes.c_int32),
        ("F_shared", ctypes.c_int32),
    ]


class TablesLayout(ctypes.Structure):
    _fields_ = [
        ("group_sizes", ctypes.c_int64), ("group_offsets", ctypes.c_int64),
        ("group_padded_offsets", ctypes.c_int64), ("group_idx_for_bx", ctypes.c_int64),
        ("row_of_pair", ctypes.c_int64), ("pair_of_row", ctypes.c_int64),
        ("chunk_counts", ctypes.c_int64), ("total_int32", ctypes.c_int64), ("M_blk", ctypes.c_int32), ("P", ctypes.c_int32),
    ]


def make_problem(T, H, F, E, top_k, padding_M=128, score_fn="softmax", renormalize=True,
                 routed_scaling_factor=1.0, down_fp8=False, F_shared=0) -> Problem:
    sf = {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}.get(score_fn, score_fn)
    return Problem(int(T), int(H), int(F), int(E), int(top_k), int(padding_M), int(sf),
                   int(bool(renormalize)), float(routed_scaling_factor), int(bool(down_fp8)),
                   int(F_shared))


_LIB = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """The loaded library (raises MoeLibraryMissing if it was never built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(library_path):
        raise MoeLibraryMissing(
            f"{library_path} not found: build it with `python -m moe_routed_expert_top_b200.build`")
    L = ctypes.CDLL(library_path)
    PP = ctypes.POINTER(Problem)
    sig = {
        "moe_get_tables_layout": (ctypes.c_int, [PP, ctypes.POINTER(TablesLayout)]),
        "moe_workspace_bytes": (ctypes.c_size_t, [PP]),
        "moe_route_topk": (ctypes.c_int, [PP, _P, _P, _P, _P]),
        "moe_route_permute": (ctypes.c_int, [PP, _P, _P, _P, _P, _P, _P, _P, _P]),
        "moe_grouped_gemm": (ctypes.c_int, [PP, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P,
                                            _P]),
        "moe_swiglu_quant": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, _P, _P,
                                            ctypes.c_int32, _P, _P, _P]),
        "moe_unpermute": (ctypes.c_int, [PP, _P, _P, _P, ctypes.c_float, _P, _P, _P]),
        "moe_unpermute_f16e": (ctypes.c_int, [PP, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P]),
        "moe_down_gemm_weighted": (ctypes.c_int, [PP, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                                  _P, _P, _P, _P, ctypes.c_float, ctypes.c_int32,
                                                  _P, _P, _P]),
        "moe_combine": (ctypes.c_int, [PP, _P, ctypes.c_int32, _P, _P, _P, _P]),
        "moe_quantize_weight_128x128": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32,
                                                       ctypes.c_int32, _P, _P, _P, _P]),
        "moe_experts_forward": (ctypes.c_int, [PP, _P, _P, _P, _P, _P, _P, _P, _P,
                                               ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
        "moe_experts_forward_noalloc": (ctypes.c_int, [PP, _P, _P, _P, _P, _P, _P, _P, _P,
                                                       ctypes.c_float, _P, _P]),
        "moe_shared_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32] * 4),
        "moe_shared_expert_forward": (ctypes.c_int, [ctypes.c_int32] * 5 + [_P, _P, _P,
                                                                            ctypes.c_int32, _P,
                                                                            _P, ctypes.c_size_t,
                                                                            _P]),
        "moe_dual_blocks": (ctypes.c_int32, [PP, ctypes.c_int32]),
        "moe_quant_dual": (ctypes.c_int, [PP, _P, ctypes.c_int32, ctypes.c_int32, _P,
                                          ctypes.c_int32, _P, _P, _P, _P, _P]),
        "moe_swiglu_quant_dual": (ctypes.c_int, [PP, _P, ctypes.c_int32, ctypes.c_int32, _P,
                                                 ctypes.c_int32, _P, _P, _P, _P, _P, _P]),
        "moe_swiglu_backward": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P]),
        "moe_ep_split_ids": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P,
                                            _P, _P, _P]),
        "moe_gather_rows": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _P, _P,
                                           _P, _P, _P]),
        "moe_noalloc_read_status": (ctypes.c_int, [_P, _P]),
        "moe_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_int64, _P, _P, _P]),
        "moe_decode_device_status": (ctypes.c_int, [ctypes.c_int32]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_last_cuda_error": (ctypes.c_char_p, []),
        "moe_last_launch_count": (ctypes.c_int32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _LIB = L
    return L


def _status_name(s: int) -> str:
    try:
        return lib().moe_status_string(int(s)).decode()
    except Exception:  # pragma: no cover - library missing
        return str(s)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        detail = ""
        if status == MOE_ERR_CUDA:
            detail = lib().moe_last_cuda_error().decode()
        raise MoeError(status, where, detail)


def moe_get_tables_layout(prob: Problem) -> dict:
    out = TablesLayout()
    _check(lib().moe_get_tables_layout(ctypes.byref(prob), ctypes.byref(out)),
           "moe_get_tables_layout")
    return {f: getattr(out, f) for f, _ in TablesLayout._fields_}


def moe_workspace_bytes(prob: Problem) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(prob)))


def moe_route_topk(prob, logits, topk_ids, topk_weights, stream=None):
    _check(lib().moe_route_topk(ctypes.byref(prob), _ptr(logits), _ptr(topk_ids),
                                _ptr(topk_weights), _stream(stream)), "moe_route_topk")


def moe_route_permute(prob, logits, topk_ids, topk_weights, hidden, x_perm, tables, dev_status,
                      stream=None):
    _check(lib().moe_route_permute(ctypes.byref(prob), _ptr(logits), _ptr(topk_ids),
                                   _ptr(topk_weights), _ptr(hidden), _ptr(x_perm), _ptr(tables),
                                   _ptr(dev_status), _stream(stream)), "moe_route_permute")


def moe_grouped_gemm(prob, M_rows, N, K, A, A_scales, B, B_scales, tables, epilogue, C,
                     C_scales, debug_h, dev_status, stream=None):
    _check(lib().moe_grouped_gemm(ctypes.byref(prob) if prob is not None else None, int(M_rows),
                                  int(N), int(K), _ptr(A), _ptr(A_scales), _ptr(B),
                                  _ptr(B_scales), _ptr(tables), int(epilogue), _ptr(C),
                                  _ptr(C_scales), _ptr(debug_h), _ptr(dev_status),
                                  _stream(stream)), "moe_grouped_gemm")


def moe_swiglu_quant(M, F, gate_up, h, out_fp8, out, scales, stream=None):
    _check(lib().moe_swiglu_quant(int(M), int(F), _ptr(gate_up), _ptr(h), int(bool(out_fp8)),
                                  _ptr(out), _ptr(scales), _stream(stream)), "moe_swiglu_quant")


def moe_unpermute(prob, y, tables, topk_weights, scale, addend, out, stream=None):
    _check(lib().moe_unpermute(ctypes.byref(prob), _ptr(y), _ptr(tables), _ptr(topk_weights),
                               float(scale), _ptr(addend), _ptr(out), _stream(stream)),
           "moe_unpermute")


def moe_unpermute_f16e(prob, y16, y_exp, tables, topk_weights, scale, addend, out, stream=None):
    _check(lib().moe_unpermute_f16e(ctypes.byref(prob), _ptr(y16), _ptr(y_exp), _ptr(tables),
                                    _ptr(topk_weights), float(scale), _ptr(addend), _ptr(out),
                                    _stream(stream)), "moe_unpermute_f16e")


def moe_down_gemm_weighted(prob, N, K, A, A_scales, B, B_scales, tables, topk_weights, scale,
                           epilogue, y_w, dev_status, stream=None):
    _check(lib().moe_down_gemm_weighted(ctypes.byref(prob), int(N), int(K), _ptr(A),
                                        _ptr(A_scales), _ptr(B), _ptr(B_scales), _ptr(tables),
                                        _ptr(topk_weights), float(scale), int(epilogue),
                                        _ptr(y_w), _ptr(dev_status), _stream(stream)),
           "moe_down_gemm_weighted")


def moe_combine(prob, y_w, tables, addend, out, stream=None):
    """y_w fp32 or bf16 (taken from the tensor's dtype)."""
    import torch
    _check(lib().moe_combine(ctypes.byref(prob), _ptr(y_w), int(y_w.dtype == torch.float32),
                             _ptr(tables), _ptr(addend), _ptr(out), _stream(stream)),
           "moe_combine")


def moe_quantize_weight_128x128(batch, N, K, w, q, scales, stream=None):
    _check(lib().moe_quantize_weight_128x128(int(batch), int(N), int(K), _ptr(w), _ptr(q),
                                             _ptr(scales), _stream(stream)),
           "moe_quantize_weight_128x128")


def moe_experts_forward(prob, hidden, topk_ids, topk_weights, w_gate_up, w_down, w_down_scales,
                        ws_gate_up, ws_down, scale, out, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().moe_experts_forward(ctypes.byref(prob), _ptr(hidden), _ptr(topk_ids),
                                     _ptr(topk_weights), _ptr(w_gate_up), _ptr(w_down),
                                     _ptr(w_down_scales), _ptr(ws_gate_up), _ptr(ws_down),
                                     float(scale), _ptr(out), _ptr(workspace), int(ws_bytes),
                                     _stream(stream)), "moe_experts_forward")


def moe_experts_forward_noalloc(prob, hidden, topk_ids, topk_weights, w_gate_up, w_down,
                                w_down_scales, ws_gate_up, ws_down, scale, out, stream=None):
    _check(lib().moe_experts_forward_noalloc(ctypes.byref(prob), _ptr(hidden), _ptr(topk_ids),
                                             _ptr(topk_weights), _ptr(w_gate_up), _ptr(w_down),
                                             _ptr(w_down_scales), _ptr(ws_gate_up), _ptr(ws_down),
                                             float(scale), _ptr(out), _stream(stream)),
           "moe_experts_forward_noalloc")


def moe_noalloc_read_status(stream=None) -> int:
    """The status word of the last moe_experts_forward_noalloc call (synchronises
    the stream to read it)."""
    import torch
    v = ctypes.c_int32(-1)
    _check(lib().moe_noalloc_read_status(ctypes.byref(v), _stream(stream)),
           "moe_noalloc_read_status")
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    return int(v.value)


def moe_selftest_bounded_wait(limit_ns, dev_status, dev_result, stream=None):
    _check(lib().moe_selftest_bounded_wait(int(limit_ns), _ptr(dev_status), _ptr(dev_result),
                                           _stream(stream)), "moe_selftest_bounded_wait")


def moe_shared_workspace_bytes(T, H, F_s, tp_size=1) -> int:
    return int(lib().moe_shared_workspace_bytes(int(T), int(H), int(F_s), int(tp_size)))


def moe_shared_expert_forward(T, H, F_s, tp_size, tp_rank, hidden, w_gate_up, w_down, out_f32,
                              out, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().moe_shared_expert_forward(int(T), int(H), int(F_s), int(tp_size), int(tp_rank),
                                           _ptr(hidden), _ptr(w_gate_up), _ptr(w_down),
                                           int(out_f32), _ptr(out), _ptr(workspace),
                                           int(ws_bytes), _stream(stream)),
           "moe_shared_expert_forward")


def moe_dual_blocks(prob, M) -> int:
    """128-token blocks of the padded token axis of moe_quant_dual (qT row pitch / 128)."""
    return int(lib().moe_dual_blocks(ctypes.byref(prob) if prob is not None else None, int(M)))


def moe_quant_dual(prob, tables, M, K, x, trans_mode, q, s, qT, sT, stream=None):
    _check(lib().moe_quant_dual(ctypes.byref(prob) if prob is not None else None, _ptr(tables),
                                int(M), int(K), _ptr(x), int(trans_mode), _ptr(q), _ptr(s),
                                _ptr(qT), _ptr(sT), _stream(stream)), "moe_quant_dual")


def moe_swiglu_quant_dual(prob, tables, M, F, gate_up, trans_mode, q, s, qT, sT, debug_h=None,
                          stream=None):
    _check(lib().moe_swiglu_quant_dual(ctypes.byref(prob) if prob is not None else None,
                                       _ptr(tables), int(M), int(F), _ptr(gate_up),
                                       int(trans_mode), _ptr(q), _ptr(s), _ptr(qT), _ptr(sT),
                                       _ptr(debug_h), _stream(stream)), "moe_swiglu_quant_dual")


def moe_swiglu_backward(M, F, gate_up, grad_h, grad_gate_up, stream=None):
    _check(lib().moe_swiglu_backward(int(M), int(F), _ptr(gate_up), _ptr(grad_h),
                                     _ptr(grad_gate_up), _stream(stream)), "moe_swiglu_backward")


def moe_ep_split_ids(n, E_local, world, ids, rank_ids, local_ids, stream=None):
    _check(lib().moe_ep_split_ids(int(n), int(E_local), int(world), _ptr(ids), _ptr(rank_ids),
                                  _ptr(local_ids), _stream(stream)), "moe_ep_split_ids")


def moe_gather_rows(n_dst, n_src, row_bytes, map_, src, dst, dev_status=None, stream=None):
    _check(lib().moe_gather_rows(int(n_dst), int(n_src), int(row_bytes), _ptr(map_), _ptr(src),
                                 _ptr(dst), _ptr(dev_status), _stream(stream)), "moe_gather_rows")


def moe_decode_device_status(dev_status: int) -> int:
    return int(lib().moe_decode_device_status(int(dev_status)))


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_last_launch_count() -> int:
    return int(lib().moe_last_launch_count())
