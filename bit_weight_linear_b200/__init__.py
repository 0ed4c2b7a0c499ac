"""bit_weight_linear_b200 -- B200-native extreme-low-bit linear layers.

Two forward forms that replace ``nn.Linear``:

* BitLinear (BitNet b1.58): ternary weights packed 2 bits each, activations
  quantised per token to int8 (absmax, Q_b = 127, no zero point), exact int32
  contraction, fp16 output -- ``bl_pack_ternary``, ``bl_quant_act``,
  ``bl_ternary_linear``.
* OneBit: y = ((x * g) S^T) * h with a 1-bit sign matrix S and fp16 value
  vectors g, h -- ``ob_pack_sign``, ``ob_linear``.

This module is argument marshalling only: every step runs in the CUDA kernels
of ``libbitlinear.so`` (C ABI declared in ``include/bitlinear.h``), called
through ctypes on torch's current stream.  torch supplies device memory and
streams.  There is no CPU fallback: if the library is missing or no CUDA
device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

BL_OK = 0
STATUS_NAMES = {0: "BL_OK", 1: "BL_ERR_NULL", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN",
                4: "BL_ERR_INVALID_VALUE", 5: "BL_ERR_CUDA", 6: "BL_ERR_TIMEOUT",
                7: "BL_ERR_WORKSPACE", 8: "BL_ERR_SCRATCH_LIMIT"}

# Entry points declared in include/bitlinear.h: name -> (argtypes, restype)
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class ChainLayer(ctypes.Structure):
    """bl_chain_layer (include/bitlinear.h)."""
    _fields_ = [("x", _P), ("src", _I), ("K", _I), ("N", _I), ("w", _P), ("w_scale", ctypes.c_float),
                ("g", _P), ("h", _P), ("y", _P), ("acc_out", _P), ("src2", _I), ("norm_w", _P),
                ("norm_eps", ctypes.c_float), ("swiglu_buf", _P)]


class Copy(ctypes.Structure):
    """bl_copy (include/bitlinear.h)."""
    _fields_ = [("src", _P), ("dst", _P), ("bytes", _SZ)]


class ChainPlan(ctypes.Structure):
    """bl_chain_plan (include/bitlinear.h)."""
    _fields_ = [("form", _I), ("n_layers", _I), ("sm_count", _I), ("kmax", _I), ("slots", _I),
                ("smem_bytes", _I), ("fused", _I)]
ABI = {
    "bl_status_string": ([_I], ctypes.c_char_p),
    "bl_abi_version": ([], _I),
    "bl_pack_ternary": ([_P, _I, _I, _P, _P], _I),
    "ob_pack_sign": ([_P, _I, _I, _P, _P], _I),
    "bl_quant_act": ([_P, _I, _I, _P, _P, _P], _I),
    "bl_ternary_workspace_bytes": ([_I, _I, _I], _SZ),
    "bl_ternary_linear": ([_P, _I, _I, _I, _P, ctypes.c_float, _P, _P, _P, _SZ, _P], _I),
    "ob_workspace_bytes": ([_I, _I, _I], _SZ),
    "ob_linear": ([_P, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "bl_device_status": ([_P], _I),
    "bl_prefill_plan": ([_I, _I, _I, _I, _I, _P], _I),
    "bl_ternary_linear_noalloc": ([_P, _I, _I, _I, _P, ctypes.c_float, _P, _P, _P], _I),
    "bl_debug_stall_next_launch": ([ctypes.c_ulonglong], _I),
    "ob_svid_workspace_bytes": ([_I, _I], _SZ),
    "ob_svid": ([_P, _I, _I, _I, ctypes.c_double, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "billm_workspace_bytes": ([_I, _I, _I], _SZ),
    "billm_linear": ([_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "billm_binarize": ([_P, _I, _I, _P, _P, _P, _P, _P], _I),
    "bl_chain_run_host": ([_P, _P, _P, _I, _P, _I, _P], _I),
    "bl_chain_bytes": ([_I], _SZ),
    "bl_chain_build": ([_I, _P, _I, _P, _SZ, _P, _P], _I),
    "bl_chain_run": ([_P, _P, _P], _I),
}


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbitlinear.so not built at {LIB_PATH}; run "
                              "`python -m bit_weight_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in ABI.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != BL_OK:
        raise BitLinearError(fn, status)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts: torch.Tensor):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("bit_weight_linear_b200 runs on CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")


def bl_pack_ternary(w: torch.Tensor) -> torch.Tensor:
    """int8 [N,K] in {-1,0,1} (CUDA) -> packed words [N, K/16] (int32 storage of uint32)."""
    _need_cuda(w)
    assert w.dtype == torch.int8 and w.dim() == 2
    N, K = w.shape
    w2 = torch.empty((N, K // 16), dtype=torch.int32, device=w.device)
    _check("bl_pack_ternary", lib().bl_pack_ternary(_ptr(w), N, K, _ptr(w2), _stream()))
    return w2


def ob_pack_sign(w: torch.Tensor) -> torch.Tensor:
    """fp16 [N,K] (CUDA) -> packed sign bits [N, K/32] (int32 storage of uint32)."""
    _need_cuda(w)
    assert w.dtype == torch.float16 and w.dim() == 2
    N, K = w.shape
    s1 = torch.empty((N, K // 32), dtype=torch.int32, device=w.device)
    _check("ob_pack_sign", lib().ob_pack_sign(_ptr(w), N, K, _ptr(s1), _stream()))
    return s1


def ob_svid(W: torch.Tensor, max_iter: int = 1000, tol: float = 1e-12, return_ab: bool = False):
    """SVID of fp32 W [N,K] (CUDA) on the device: returns (s1 packed signs
    [N, K/32], g fp16 [K], h fp16 [N], sigma, iterations), plus fp64 a [N] and
    b [K] when return_ab."""
    _need_cuda(W)
    assert W.dtype == torch.float32 and W.dim() == 2
    N, K = W.shape
    dev = W.device
    s1 = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
    g = torch.empty((K,), dtype=torch.float16, device=dev)
    h = torch.empty((N,), dtype=torch.float16, device=dev)
    a = torch.empty((N,), dtype=torch.float64, device=dev) if return_ab else None
    b = torch.empty((K,), dtype=torch.float64, device=dev) if return_ab else None
    nws = int(lib().ob_svid_workspace_bytes(N, K))
    if nws == 0:
        raise BitLinearError("ob_svid", 2)
    ws = torch.empty((nws,), dtype=torch.uint8, device=dev)
    sigma, iters = ctypes.c_double(0.0), ctypes.c_int(0)
    _check("ob_svid", lib().ob_svid(_ptr(W), N, K, int(max_iter), float(tol), _ptr(s1), _ptr(g), _ptr(h),
                                    _ptr(a), _ptr(b), ctypes.byref(sigma), ctypes.byref(iters), _ptr(ws),
                                    nws, _stream()))
    out = (s1, g, h, sigma.value, iters.value)
    return out + (a, b) if return_ab else out


def billm_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().billm_workspace_bytes(M, K, N))


def billm_binarize(W: torch.Tensor, return_alpha64: bool = False):
    """Residual binarisation of fp32 W [N,K] (CUDA): returns (b2 stacked sign
    planes [2N, K/32], alpha fp16 [2N]), plus fp64 alpha_o, alpha_r [N] when
    return_alpha64."""
    _need_cuda(W)
    assert W.dtype == torch.float32 and W.dim() == 2
    N, K = W.shape
    b2 = torch.empty((2 * N, K // 32), dtype=torch.int32, device=W.device)
    alpha = torch.empty((2 * N,), dtype=torch.float16, device=W.device)
    ao = torch.empty((N,), dtype=torch.float64, device=W.device) if return_alpha64 else None
    ar = torch.empty((N,), dtype=torch.float64, device=W.device) if return_alpha64 else None
    _check("billm_binarize", lib().billm_binarize(_ptr(W), N, K, _ptr(b2), _ptr(alpha), _ptr(ao), _ptr(ar),
                                                  _stream()))
    return (b2, alpha, ao, ar) if return_alpha64 else (b2, alpha)


def billm_linear(x: torch.Tensor, b2: torch.Tensor, alpha: torch.Tensor, *,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """Two-plane binary forward: y = alpha_o * (x B_o^T) + alpha_r * (x B_r^T),
    fp16 in/out; b2 = [B_o; B_r] packed [2N, K/32], alpha = [alpha_o; alpha_r]."""
    _need_cuda(x, b2, alpha)
    M, K = x.shape
    N = b2.shape[0] // 2
    nws = int(lib().billm_workspace_bytes(M, K, N))
    if nws == 0 and M > 0 and N > 0:
        raise BitLinearError("billm_linear", 2)
    ws = workspace if workspace is not None else torch.empty((max(nws, 1),), dtype=torch.uint8,
                                                             device=x.device)
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check("billm_linear", lib().billm_linear(_ptr(x), M, K, N, _ptr(b2), _ptr(alpha), _ptr(y), _ptr(ws),
                                              ws.numel(), _stream()))
    return y


def bl_quant_act(x: torch.Tensor):
    """fp16 [M,K] -> (q int8 [M,K], scale fp32 [M]) by per-token absmax (Q_b = 127)."""
    _need_cuda(x)
    assert x.dtype == torch.float16 and x.dim() == 2
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("bl_quant_act", lib().bl_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s), _stream()))
    return q, s


def bl_ternary_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().bl_ternary_workspace_bytes(M, K, N))


def ob_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().ob_workspace_bytes(M, K, N))


def _workspace(nbytes: int, device, workspace: torch.Tensor | None) -> torch.Tensor:
    if workspace is not None:
        return workspace
    return torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=device)


def bl_ternary_linear(x: torch.Tensor, w2: torch.Tensor, w_scale: float, *,
                      return_acc: bool = False, workspace: torch.Tensor | None = None,
                      out: torch.Tensor | None = None):
    """BitLinear forward: fp16 x [M,K], packed w2 [N,K/16] -> fp16 y [M,N] (and int32 acc)."""
    _need_cuda(x, w2)
    M, K = x.shape
    N = w2.shape[0]
    if w2.shape[1] * 16 != K:
        raise ValueError("w2 must be [N, K/16]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device) if return_acc else None
    nbytes = bl_ternary_workspace_bytes(M, K, N)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bl_ternary_linear(_ptr(x), M, K, N, _ptr(w2), float(w_scale), _ptr(y), _ptr(acc),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check("bl_ternary_linear", st)
    return (y, acc) if return_acc else y


def ob_linear(x: torch.Tensor, s1: torch.Tensor, g: torch.Tensor, h: torch.Tensor, *,
              workspace: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """OneBit forward: y = ((x * g) S^T) * h, fp16 in/out, packed S [N, K/32]."""
    _need_cuda(x, s1, g, h)
    M, K = x.shape
    N = s1.shape[0]
    if s1.shape[1] * 32 != K or g.shape != (K,) or h.shape != (N,):
        raise ValueError("shapes: s1 [N,K/32], g [K], h [N]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    nbytes = ob_workspace_bytes(M, K, N)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().ob_linear(_ptr(x), M, K, N, _ptr(s1), _ptr(g), _ptr(h), _ptr(y), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream())
    _check("ob_linear", st)
    return y


def bl_ternary_linear_noalloc(x: torch.Tensor, w2: torch.Tensor, w_scale: float, *,
                              return_acc: bool = False, out: torch.Tensor | None = None):
    """BitLinear forward without a workspace, for callers that cannot allocate device
    memory where they run the layer: the library's fixed scratch array stands in
    for it (M*K up to about 16.7 million; calls that overlap on the GPU race on
    the shared array).  Same result as ``bl_ternary_linear``."""
    _need_cuda(x, w2)
    M, K = x.shape
    N = w2.shape[0]
    if w2.shape[1] * 16 != K:
        raise ValueError("w2 must be [N, K/16]")
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device) if return_acc else None
    st = lib().bl_ternary_linear_noalloc(_ptr(x), M, K, N, _ptr(w2), float(w_scale), _ptr(y),
                                         _ptr(acc), _stream())
    _check("bl_ternary_linear_noalloc", st)
    return (y, acc) if return_acc else y


class Chain:
    """A decode chain built on the device (bl_chain_build): the single-token
    forward of a list of layers in one persistent launch per run().  Holds the
    device descriptor buffer and the plan; keeps the layers' tensors alive."""

    def __init__(self, form: int, layers: list[dict]):
        """layers: dicts with K, N, w (packed, CUDA), y (fp16 [N] or [1, N],
        CUDA), and either x (fp16 [K], CUDA) or src (index of an earlier
        layer); optional src2 (SwiGLU of the outputs of src and src2) with an
        optional swiglu_buf (fp16 [K] scratch: the SwiGLU is then evaluated once
        per element), norm_w (fp16 [K] RMSNorm weight) and norm_eps; ternary:
        w_scale, optional acc_out (int32 [N]); OneBit: g, h."""
        n = len(layers)
        arr = (ChainLayer * n)()
        self._keep = []
        dev = None
        for j, d in enumerate(layers):
            ts = [d.get(k) for k in ("x", "w", "g", "h", "y", "acc_out", "norm_w", "swiglu_buf")]
            _need_cuda(*[t for t in ts if t is not None])
            self._keep.extend(t for t in ts if t is not None)
            dev = dev or d["w"].device
            arr[j].x = None if d.get("x") is None else d["x"].data_ptr()
            arr[j].src = int(d.get("src", -1))
            arr[j].K, arr[j].N = int(d["K"]), int(d["N"])
            arr[j].w = d["w"].data_ptr()
            arr[j].w_scale = float(d.get("w_scale", 0.0))
            arr[j].g = None if d.get("g") is None else d["g"].data_ptr()
            arr[j].h = None if d.get("h") is None else d["h"].data_ptr()
            arr[j].y = d["y"].data_ptr()
            arr[j].acc_out = None if d.get("acc_out") is None else d["acc_out"].data_ptr()
            arr[j].src2 = int(d.get("src2", -1))
            arr[j].norm_w = None if d.get("norm_w") is None else d["norm_w"].data_ptr()
            arr[j].norm_eps = float(d.get("norm_eps", 0.0))
            arr[j].swiglu_buf = None if d.get("swiglu_buf") is None else d["swiglu_buf"].data_ptr()
        nbytes = int(lib().bl_chain_bytes(n))
        if nbytes == 0:
            raise ValueError("chain length out of range")
        self.buf = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
        self.plan = ChainPlan()
        _check("bl_chain_build", lib().bl_chain_build(form, arr, n, _ptr(self.buf), nbytes,
                                                      ctypes.byref(self.plan), _stream()))

    def run(self):
        """One decode step over the chain on torch's current stream."""
        _check("bl_chain_run", lib().bl_chain_run(ctypes.byref(self.plan), _ptr(self.buf),
                                                  _stream()))

    def run_host(self, inputs, outputs):
        """One decode step with host buffers on torch's current stream: inputs
        are (host tensor, device tensor) pairs copied to the device first,
        outputs (device tensor, host tensor) pairs copied back after the run.
        Host tensors should be pinned; nothing is synchronised."""
        for h, d in list(inputs) + [(h, d) for d, h in outputs]:
            if h.is_cuda or not d.is_cuda or not h.is_contiguous() or not d.is_contiguous():
                raise ValueError("run_host takes contiguous (host, device) tensor pairs")
            if h.numel() * h.element_size() != d.numel() * d.element_size():
                raise ValueError("host and device buffers differ in size")
        ins = (Copy * max(1, len(inputs)))()
        for i, (h, d) in enumerate(inputs):
            ins[i] = Copy(h.data_ptr(), d.data_ptr(), h.numel() * h.element_size())
        outs = (Copy * max(1, len(outputs)))()
        for i, (d, h) in enumerate(outputs):
            outs[i] = Copy(d.data_ptr(), h.data_ptr(), d.numel() * d.element_size())
        _check("bl_chain_run_host", lib().bl_chain_run_host(ctypes.byref(self.plan), _ptr(self.buf), ins,
                                                            len(inputs), outs, len(outputs), _stream()))


def bl_device_status() -> int:
    return int(lib().bl_device_status(_stream()))


__all__ = ["bl_pack_ternary", "ob_pack_sign", "bl_quant_act", "bl_ternary_linear",
           "ob_linear", "bl_ternary_workspace_bytes", "ob_workspace_bytes",
           "bl_device_status", "bl_ternary_linear_noalloc", "Chain", "BitLinearError", "lib", "ABI"]
