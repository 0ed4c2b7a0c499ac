"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/bitlinear.h declares, and rejects bad arguments before any
CUDA call is made."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def L():
    from bit_weight_linear_b200 import build as b
    b.build()
    import bit_weight_linear_b200 as blw
    return blw.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:bl|ob|billm)_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ["bl_pack_ternary", "ob_pack_sign", "bl_quant_act", "bl_ternary_linear", "ob_linear"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    import bit_weight_linear_b200 as blw
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in blw.ABI, f"binding lacks {name}"


def test_status_strings(L):
    assert L.bl_status_string(0) == b"BL_OK"
    assert L.bl_status_string(2).startswith(b"BL_ERR_SHAPE")
    assert L.bl_status_string(99) == b"unknown bl_status"
    assert L.bl_abi_version() == 100


def test_workspace_sizes(L):
    assert L.bl_ternary_workspace_bytes(1, 4096, 4096) == 4096 + 256 + 256
    assert L.bl_ternary_workspace_bytes(8, 4096, 4096) == 8 * 4096 + 256 + 256
    assert L.ob_workspace_bytes(16, 4096, 4096) == 3 * 16 * 4096 + 256 + 256   # three limb planes
    assert L.bl_ternary_workspace_bytes(1, 100, 16) == 0       # bad K
    assert L.bl_ternary_workspace_bytes(1, 128, 24) == 0       # bad N (not a multiple of 16)
    assert L.ob_workspace_bytes(1, 128, -16) == 0
    assert L.ob_workspace_bytes(1, 65536 + 128, 16) == 0        # OneBit K limit
    for v in (L.bl_ternary_workspace_bytes(3, 384, 16), L.ob_workspace_bytes(5, 640, 32)):
        assert v % 256 == 0


A = ctypes.c_void_p(0x10000)       # aligned fake device address (never dereferenced)
MIS = ctypes.c_void_p(0x10004)     # misaligned


@pytest.mark.parametrize("M,K,N", [(1, 100, 16), (1, 0, 16), (1, 128, 15), (-1, 128, 16),
                                   (1, 128, -16), (1, 64, 16)])
def test_shape_rules(L, M, K, N):
    assert L.bl_ternary_linear(A, M, K, N, A, 1.0, A, None, A, 1 << 30, None) == 2
    assert L.ob_linear(A, M, K, N, A, A, A, A, A, 1 << 30, None) == 2


def test_shape_checks_of_packers_and_quant(L):
    assert L.bl_pack_ternary(A, 16, 100, A, None) == 2
    assert L.ob_pack_sign(A, 17, 128, A, None) == 2
    assert L.bl_quant_act(A, 1, 96, A, A, None) == 2


def test_empty_inputs_are_noops(L):
    assert L.bl_ternary_linear(None, 0, 128, 16, None, 1.0, None, None, None, 0, None) == 0
    assert L.bl_ternary_linear(None, 4, 128, 0, None, 1.0, None, None, None, 0, None) == 0
    assert L.ob_linear(None, 0, 128, 16, None, None, None, None, None, 0, None) == 0
    assert L.bl_quant_act(None, 0, 128, None, None, None) == 0
    assert L.bl_pack_ternary(None, 0, 128, None, None) == 0


def test_null_alignment_and_workspace(L):
    assert L.bl_ternary_linear(None, 1, 128, 16, A, 1.0, A, None, A, 1 << 20, None) == 1
    assert L.bl_ternary_linear(MIS, 1, 128, 16, A, 1.0, A, None, A, 1 << 20, None) == 3
    assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, MIS, A, 1 << 20, None) == 3
    assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, None, None, 1 << 20, None) == 7
    need = L.bl_ternary_workspace_bytes(1, 128, 16)
    assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, None, A, need - 1, None) == 7
    assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, None, MIS, need, None) == 3
    assert L.ob_linear(A, 1, 128, 16, A, None, A, A, A, 1 << 20, None) == 1
    assert L.ob_linear(A, 1, 128, 16, A, A, MIS, A, A, 1 << 20, None) == 3
    assert L.ob_linear(A, 1, 128, 16, A, A, A, A, A, 10, None) == 7
    assert L.ob_linear(A, 1, 65536 + 128, 16, A, A, A, A, A, 1 << 30, None) == 2
    assert L.bl_quant_act(A, 1, 128, None, A, None) == 1
    assert L.bl_pack_ternary(A, 16, 128, MIS, None) == 3


def test_python_binding_refuses_cpu_tensors():
    import torch
    import bit_weight_linear_b200 as blw
    with pytest.raises(ValueError):
        blw.bl_quant_act(torch.zeros((1, 128), dtype=torch.float16))


@pytest.mark.parametrize("mode,code", [("cuda", 5), ("timeout", 6)])
def test_fault_injection_hook(L, monkeypatch, mode, code):
    """BL_FAULT_INJECT makes every launching entry point return the injected
    error after its argument checks and before any CUDA call (so this runs
    without a GPU); bad arguments still win, and unsetting it restores the
    normal behaviour."""
    monkeypatch.setenv("BL_FAULT_INJECT", mode)
    assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, None, A, 1 << 20, None) == code
    assert L.ob_linear(A, 1, 128, 16, A, A, A, A, A, 1 << 20, None) == code
    assert L.bl_quant_act(A, 1, 128, A, A, None) == code
    assert L.bl_pack_ternary(A, 16, 128, A, None) == code
    assert L.ob_pack_sign(A, 16, 128, A, None) == code
    assert L.bl_ternary_linear_noalloc(A, 1, 128, 16, A, 1.0, A, None, None) == code
    assert L.bl_ternary_linear(A, 1, 100, 16, A, 1.0, A, None, A, 1 << 20, None) == 2
    assert L.bl_ternary_linear(None, 0, 128, 16, None, 1.0, None, None, None, 0, None) == 0
    monkeypatch.setenv("BL_FAULT_INJECT", "")
    # with no GPU the call now fails in the CUDA runtime, not in the hook
    if not __import__("torch").cuda.is_available():
        assert L.bl_ternary_linear(A, 1, 128, 16, A, 1.0, A, None, A, 1 << 20, None) == 5


def test_chain_build_rejects_bad_layers(L):
    """bl_chain_build validates every layer before any CUDA call."""
    import bit_weight_linear_b200 as blw
    n = 2
    arr = (blw.ChainLayer * n)()
    for j in range(n):
        arr[j].x, arr[j].src, arr[j].K, arr[j].N = 0x10000, -1, 128, 16
        arr[j].w, arr[j].y, arr[j].src2 = 0x10000, 0x10000, -1
    plan = blw.ChainPlan()
    buf = ctypes.c_void_p(0x100000)
    nb = L.bl_chain_bytes(n)
    assert nb > 0 and L.bl_chain_bytes(0) == 0 and L.bl_chain_bytes(2049) == 0
    assert L.bl_chain_build(0, None, n, buf, nb, ctypes.byref(plan), None) == 1
    assert L.bl_chain_build(2, arr, n, buf, nb, ctypes.byref(plan), None) == 2       # bad form
    assert L.bl_chain_build(0, arr, n, ctypes.c_void_p(0x100010), nb, ctypes.byref(plan), None) == 3
    arr[1].src = 1                                  # not an earlier layer
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].src, arr[1].K = 0, 256                   # K must equal the source's N
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].K, arr[1].N, arr[1].src = 128, 16, -1
    arr[0].K = 100                                  # K % 128
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[0].K, arr[0].x = 128, None                  # a given input needs x
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 1
    arr[0].x = 0x10004                              # misaligned
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 3
    arr[0].x = 0x10000
    assert L.bl_chain_build(1, arr, n, buf, nb, ctypes.byref(plan), None) == 1       # OneBit needs g, h
    assert L.bl_chain_build(0, arr, n, buf, nb - 1, ctypes.byref(plan), None) == 7
    # fused prologues: SwiGLU needs src >= 0 and an earlier src2 of the same width
    arr[1].src2 = 0                                 # src2 without src
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].src, arr[1].x, arr[1].src2 = 0, None, 1  # src2 not an earlier layer
    arr[0].N = 128
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].src2, arr[1].norm_w, arr[1].norm_eps = 0, 0x20000, -1.0    # eps < 0
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].norm_eps, arr[1].norm_w = 1e-6, 0x20002                    # misaligned weight
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 3
    # a fused row must fit the registers of the prologue: 17920 ternary
    arr[0].N = arr[1].K = 18048
    arr[1].norm_w, arr[1].src2 = 0x20000, -1
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].norm_w = None
    arr[1].swiglu_buf = 0x30000                     # a SwiGLU buffer without src2
    assert L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None) == 2
    arr[1].swiglu_buf = None                        # unfused, the same row is fine
    r = L.bl_chain_build(0, arr, n, buf, nb, ctypes.byref(plan), None)
    assert r != 2


def test_svid_rejects_bad_arguments(L):
    """ob_svid validates shape, iteration limits, pointers and workspace before
    any CUDA call."""
    ws = L.ob_svid_workspace_bytes(64, 256)
    assert ws > 0 and ws % 256 == 0
    assert L.ob_svid_workspace_bytes(24, 256) == 0               # N % 16
    assert L.ob_svid_workspace_bytes(64, 100) == 0               # K % 128
    assert L.ob_svid_workspace_bytes(524288 + 16, 128) == 0      # N limit
    args = lambda **kw: [kw.get("W", A), kw.get("N", 64), kw.get("K", 256), kw.get("it", 10),
                         kw.get("tol", 1e-12), kw.get("s1", A), kw.get("g", A), kw.get("h", A),
                         kw.get("a", None), kw.get("b", None), None, None, kw.get("ws", A),
                         kw.get("nws", ws), None]
    assert L.ob_svid(*args(N=0)) == 0                             # empty: no-op
    assert L.ob_svid(*args(K=100)) == 2
    assert L.ob_svid(*args(it=0)) == 2
    assert L.ob_svid(*args(tol=-1.0)) == 2
    assert L.ob_svid(*args(tol=float("nan"))) == 2
    assert L.ob_svid(*args(W=None)) == 1
    assert L.ob_svid(*args(g=None)) == 1
    assert L.ob_svid(*args(h=ctypes.c_void_p(0x10002))) == 3
    assert L.ob_svid(*args(a=ctypes.c_void_p(0x10008))) == 3
    assert L.ob_svid(*args(nws=ws - 1)) == 7
    assert L.ob_svid(*args(ws=None)) == 7


def test_billm_rejects_bad_arguments(L):
    ws = L.billm_workspace_bytes(4, 256, 32)
    assert ws > 0 and ws % 256 == 0
    assert L.billm_workspace_bytes(4, 100, 32) == 0
    assert L.billm_workspace_bytes(4, 65536 + 128, 32) == 0
    assert L.billm_linear(A, 4, 256, 24, A, A, A, A, ws, None) == 2           # N % 16
    assert L.billm_linear(A, 0, 256, 32, A, A, A, A, ws, None) == 0           # empty
    assert L.billm_linear(None, 4, 256, 32, A, A, A, A, ws, None) == 1
    assert L.billm_linear(A, 4, 256, 32, A, ctypes.c_void_p(0x10002), A, A, ws, None) == 3
    assert L.billm_linear(A, 4, 256, 32, A, A, A, A, ws - 1, None) == 7
    assert L.billm_binarize(A, 32, 100, A, A, None, None, None) == 2
    assert L.billm_binarize(A, 32, 128, None, A, None, None, None) == 1
    assert L.billm_binarize(A, 32, 128, A, A, ctypes.c_void_p(0x10008), None, None) == 3


def test_chain_run_host_rejects_bad_arguments(L):
    """bl_chain_run_host validates the plan and every copy before any CUDA call."""
    import bit_weight_linear_b200 as blw
    plan = blw.ChainPlan()
    plan.form, plan.n_layers, plan.fused = 0, 1, 0
    buf = ctypes.c_void_p(0x100000)
    cp = (blw.Copy * 1)()
    cp[0] = blw.Copy(0x10000, 0x20000, 64)
    assert L.bl_chain_run_host(None, buf, cp, 1, cp, 1, None) == 1
    assert L.bl_chain_run_host(ctypes.byref(plan), ctypes.c_void_p(0x100010), cp, 1, cp, 1, None) == 3
    assert L.bl_chain_run_host(ctypes.byref(plan), buf, cp, -1, cp, 1, None) == 2
    assert L.bl_chain_run_host(ctypes.byref(plan), buf, None, 1, cp, 1, None) == 1
    bad = (blw.Copy * 1)()
    bad[0] = blw.Copy(None, 0x20000, 64)
    assert L.bl_chain_run_host(ctypes.byref(plan), buf, bad, 1, cp, 1, None) == 1
    assert L.bl_chain_run_host(ctypes.byref(plan), buf, cp, 1, bad, 1, None) == 1
    plan.fused = 2
    assert L.bl_chain_run_host(ctypes.byref(plan), buf, cp, 1, cp, 1, None) == 2
