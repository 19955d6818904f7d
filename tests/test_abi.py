"""The C-ABI library loads and exports every entry point include/moe.h declares;
host-side argument validation and layout logic (no GPU needed: nothing here
launches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def M():
    from moe_routed_expert_top_b200 import build
    build.build()
    import moe_routed_expert_top_b200 as m
    return m


def test_library_exports_every_declared_symbol(M):
    L = M.lib()
    declared = _header_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(M.EXPORTED_SYMBOLS)


def test_library_has_no_cuda_driver_load_dependency(M):
    # loads on a machine without a GPU driver: the runtime is linked statically
    ctypes.CDLL(M.library_path)


def test_status_strings_and_device_status_decoding(M):
    assert M.moe_status_string(0) == "MOE_OK"
    assert M.moe_status_string(-3) == "MOE_ERR_WORKSPACE"
    assert M.moe_decode_device_status(0) == 0
    assert M.moe_decode_device_status(M.MOE_DEV_TIMEOUT) == -5
    assert M.moe_decode_device_status(M.MOE_DEV_BAD_EXPERT_ID) == -6
    assert M.moe_decode_device_status(M.MOE_DEV_TIMEOUT | 1) == -5


def test_tables_layout_matches_tutorial_counts(M):
    p = M.make_problem(T=9, H=128, F=64, E=4, top_k=2, padding_M=128)
    L = M.moe_get_tables_layout(p)
    assert L["M_blk"] == 5 and L["P"] == 18
    offs = [L[k] for k in ("group_sizes", "group_offsets", "group_padded_offsets",
                           "group_idx_for_bx", "row_of_pair", "pair_of_row")]
    assert offs == sorted(offs)
    assert all(o % 4 == 0 for o in offs)        # 16-byte aligned sections
    assert L["group_offsets"] - L["group_sizes"] >= 4
    assert L["group_idx_for_bx"] - L["group_padded_offsets"] >= 5
    assert L["total_int32"] >= L["pair_of_row"] + 18


def test_workspace_bytes_covers_intermediates(M):
    for fp8, Fs in ((False, 0), (True, 0), (False, 2048)):
        p = M.make_problem(T=512, H=7168, F=2048, E=256, top_k=8, down_fp8=fp8, F_shared=Fs)
        ws = M.moe_workspace_bytes(p)
        P = 512 * 8
        need = P * 7168 * 2 * 2 + P * 2048 * (1 if fp8 else 2)
        if Fs:
            need += 512 * Fs * 2 + 512 * 7168 * 2
        assert ws >= need
        assert ws % 1024 == 0


@pytest.mark.parametrize("kw,status", [
    (dict(E=0), -1), (dict(E=1025), -2), (dict(top_k=33), -2), (dict(top_k=9, E=8), -2),
    (dict(T=-1), -1), (dict(score_fn=7), -1), (dict(H=100), -2), (dict(padding_M=64), -2),
    (dict(down_fp8=True, F=192), -2),
])
def test_problem_validation(M, kw, status):
    base = dict(T=16, H=256, F=256, E=8, top_k=2)
    base.update(kw)
    p = M.make_problem(**base)
    # moe_workspace_bytes returns 0 for a problem the forward cannot run
    assert M.moe_workspace_bytes(p) == 0
    r = M.lib().moe_experts_forward(ctypes.byref(p), 16, 16, 16, 16, 16, None, None, None,
                                    ctypes.c_float(1.0), 16, 16, ctypes.c_size_t(1 << 30), None)
    assert r == status


def test_null_pointer_and_workspace_errors(M):
    p = M.make_problem(T=16, H=256, F=256, E=8, top_k=2)
    L = M.lib()
    assert L.moe_route_topk(ctypes.byref(p), None, 16, 16, None) == -1
    assert L.moe_route_permute(ctypes.byref(p), None, None, None, None, None, 16, 16, None) == -1
    assert L.moe_unpermute(ctypes.byref(p), None, 16, 16, ctypes.c_float(1.0), None, 16, None) == -1
    # workspace too small is caught before anything is enqueued
    assert L.moe_experts_forward(ctypes.byref(p), 16, 16, 16, 16, 16, None, None, None,
                                 ctypes.c_float(1.0), 16, 16, ctypes.c_size_t(1024), None) == -3
    # misaligned pointer
    assert L.moe_experts_forward(ctypes.byref(p), 18, 16, 16, 16, 16, None, None, None,
                                 ctypes.c_float(1.0), 16, 16, ctypes.c_size_t(1 << 30), None) == -1
    # FP8 down needs its scales; shared expert needs both weights
    p8 = M.make_problem(T=16, H=256, F=256, E=8, top_k=2, down_fp8=True)
    assert L.moe_experts_forward(ctypes.byref(p8), 16, 16, 16, 16, 16, None, None, None,
                                 ctypes.c_float(1.0), 16, 16, ctypes.c_size_t(1 << 30), None) == -1
    ps = M.make_problem(T=16, H=256, F=256, E=8, top_k=2, F_shared=128)
    assert L.moe_experts_forward(ctypes.byref(ps), 16, 16, 16, 16, 16, None, 16, None,
                                 ctypes.c_float(1.0), 16, 16, ctypes.c_size_t(1 << 30), None) == -1
    # grouped GEMM: bad epilogue, unsupported K, FP8 with a non-store epilogue
    assert L.moe_grouped_gemm(None, 128, 256, 256, 16, None, 16, None, None, 9, 16, None, None,
                              16, None) == -1
    assert L.moe_grouped_gemm(None, 128, 256, 96, 16, None, 16, None, None, 0, 16, None, None,
                              16, None) == -2
    assert L.moe_grouped_gemm(None, 128, 256, 256, 16, 16, 16, 16, None, 1, 16, None, None,
                              16, None) == -2
    # swiglu_quant: exactly one of gate_up / h; quantising h needs out_fp8
    assert L.moe_swiglu_quant(4, 128, None, None, 1, 16, 16, None) == -1
    assert L.moe_swiglu_quant(4, 128, None, 16, 0, 16, 16, None) == -1
    assert L.moe_swiglu_quant(4, 126, 16, None, 0, 16, None, None) == -1


def test_empty_batch_is_a_no_op(M):
    p = M.make_problem(T=0, H=256, F=256, E=8, top_k=2)
    L = M.lib()
    assert L.moe_route_topk(ctypes.byref(p), None, None, None, None) == 0
    assert L.moe_experts_forward(ctypes.byref(p), None, None, None, None, None, None, None, None,
                                 ctypes.c_float(1.0), None, None, ctypes.c_size_t(0), None) == 0


def test_weighted_down_and_combine_validation(M):
    """moe_down_gemm_weighted and moe_combine reject bad arguments on the host,
    before anything is enqueued, and treat an empty batch as a no-op."""
    p = M.make_problem(T=16, H=256, F=256, E=8, top_k=2)
    L = M.lib()
    f1 = ctypes.c_float(1.0)

    def dw(prob, N=256, K=256, A=16, As=None, B=16, Bs=None, tables=16, w=16, epi=0, y=16, st=16):
        return L.moe_down_gemm_weighted(ctypes.byref(prob), N, K, A, As, B, Bs, tables, w, f1,
                                        epi, y, st, None)

    assert dw(p, A=None) == -1
    assert dw(p, tables=None) == -1
    assert dw(p, w=None) == -1
    assert dw(p, st=None) == -1
    assert dw(p, y=18) == -1                     # misaligned output
    assert dw(p, epi=M.MOE_EPI_SWIGLU) == -1     # store epilogues only
    assert dw(p, epi=0x100) == -1                # no gather flag here
    assert dw(p, epi=M.MOE_TILE_TOKEN_ROWS) == -2
    assert dw(p, N=192) == -2                    # weight-row tilings need N % 128 == 0
    assert dw(p, K=96) == -2
    assert dw(p, As=16) == -1                    # FP8 needs both scale arrays
    assert dw(M.make_problem(T=16, H=256, F=256, E=8, top_k=2, padding_M=64)) == -2
    assert dw(M.make_problem(T=0, H=256, F=256, E=8, top_k=2)) == 0

    def cb(prob, y=16, f32=0, tables=16, add=None, out=16):
        return L.moe_combine(ctypes.byref(prob), y, f32, tables, add, out, None)

    assert cb(p, y=None) == -1
    assert cb(p, tables=None) == -1
    assert cb(p, out=None) == -1
    assert cb(p, out=24) == -1                   # misaligned
    assert cb(p, add=8) == -1
    assert cb(M.make_problem(T=16, H=100, F=256, E=8, top_k=2)) == -1   # H % 8
    assert cb(M.make_problem(T=0, H=256, F=256, E=8, top_k=2)) == 0


def test_noalloc_validates_like_the_workspace_forward(M):
    """moe_experts_forward_noalloc leaves every argument and shape check to
    moe_experts_forward: an invalid problem gets that call's status even at
    T = 0, a valid T = 0 problem is a no-op that touches no device, and a
    problem too large for the built-in scratch array is MOE_ERR_WORKSPACE."""
    L = M.lib()
    f1 = ctypes.c_float(1.0)

    def na(prob):
        return L.moe_experts_forward_noalloc(ctypes.byref(prob), None, None, None, None, None,
                                             None, None, None, f1, None, None)

    assert L.moe_experts_forward_noalloc(None, None, None, None, None, None, None, None, None,
                                         f1, None, None) == M.MOE_ERR_INVALID_ARG
    for kw, status in ((dict(E=0), -1), (dict(E=1025), -2), (dict(top_k=9, E=8), -2),
                       (dict(H=100), -2), (dict(score_fn=7), -1)):
        base = dict(T=0, H=256, F=256, E=8, top_k=2)
        base.update(kw)
        assert na(M.make_problem(**base)) == status, kw
    assert na(M.make_problem(T=0, H=256, F=256, E=8, top_k=2)) == M.MOE_OK
    big = M.make_problem(T=4096, H=2048, F=768, E=128, top_k=8)
    assert M.moe_workspace_bytes(big) > 64 * 1024 * 1024
    assert na(big) == M.MOE_ERR_WORKSPACE
    assert L.moe_noalloc_read_status(None, None) == M.MOE_ERR_INVALID_ARG


def test_selftest_bounded_wait_validation(M):
    L = M.lib()
    assert L.moe_selftest_bounded_wait(1000000, None, 16, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(1000000, 16, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(1000000, 16, 20, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(999, 16, 16, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(2000000000, 16, 16, None) == M.MOE_ERR_INVALID_ARG
