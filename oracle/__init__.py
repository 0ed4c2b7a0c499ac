"""The oracle: a plain, slow CPU restatement of the extreme-low-bit linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline / reference leg may import this package.  The
product path (``bit_weight_linear_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``oref.c`` (scalar C, IEEE fp32 without contraction,
fp64 where the pages fix no precision); this module only marshals numpy arrays
through ctypes.  ``build()`` compiles ``liboref.so`` next to this file.

Pages followed (cited by title and section):

* BitNet b1.58 -- "微软、国科大开启1Bit时代：大模型转三进制，速度快4倍能耗降至1/41",
  section "BitNet b1.58 介绍" (ternary weights, per-token symmetric int8
  activations, no zero point, no bias), "内存和延迟" (2-bit kernel).
* OneBit -- "清华、哈工大把大模型压缩到了1bit，把大模型放在手机里跑的愿望就快要实现了！",
  sections "1. 新的 1bit 结构" (+-1 matrix, FP16 value vectors g and h, the
  4096x4096 storage example), "2. 基于 SVID 初始化量化模型" (sign times a rank-1
  approximation of |W|; order swap), "3. 通过知识蒸馏迁移原模型能力" (save the
  post-Sign() parameters).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboref.so")
_OMP_LIB_PATH = os.path.join(_HERE, "liboref_omp.so")   # the same source with -fopenmp
_SRC = os.path.join(_HERE, "oref.c")

OREF_OK, OREF_ERR_SHAPE, OREF_ERR_VALUE, OREF_ERR_ALLOC = 0, -1, -2, -3

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations", "-Wall", "-Wno-unknown-pragmas"]


def _build_one(path: str, extra, force: bool) -> str:
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= max(os.path.getmtime(_SRC),
                                              os.path.getmtime(os.path.join(_HERE, "oref.h")))):
        return path
    tmp = path + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, *extra, "-o", tmp, _SRC, "-lm"], cwd=_HERE)
    os.replace(tmp, path)
    return path


def build(force: bool = False) -> str:
    """Compile ``oref.c`` into ``liboref.so`` (one core) and ``liboref_omp.so``
    (output rows on all host cores, OpenMP); returns the first library's path."""
    _build_one(_OMP_LIB_PATH, ["-fopenmp"], force)
    return _build_one(_LIB_PATH, [], force)


_lib = None
_omp_lib = None


def lib(parallel: bool = False) -> ctypes.CDLL:
    """The oracle library: single-threaded, or (parallel=True) the OpenMP build
    whose linear forms spread output rows over the host cores."""
    global _lib, _omp_lib
    if parallel:
        if _omp_lib is None:
            build()
            _omp_lib = _declare(ctypes.CDLL(_OMP_LIB_PATH))
        return _omp_lib
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def omp_threads() -> int:
    """Threads the OpenMP build uses (OMP_NUM_THREADS, else the host's cores)."""
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.oref_half_to_double.argtypes = [ctypes.c_uint16]
    L.oref_half_to_double.restype = ctypes.c_double
    L.oref_double_to_half.argtypes = [ctypes.c_double]
    L.oref_double_to_half.restype = ctypes.c_uint16
    L.oref_float_to_half.argtypes = [ctypes.c_float]
    L.oref_float_to_half.restype = ctypes.c_uint16
    L.oref_pack_ternary.argtypes = [P, I, I, P]
    L.oref_pack_sign.argtypes = [P, I, I, P]
    L.oref_quant_act.argtypes = [P, I, I, P, P]
    L.oref_ternary_linear.argtypes = [P, I, I, I, P, ctypes.c_float, P, P]
    L.oref_ob_linear.argtypes = [P, I, I, I, P, P, P, P, P]
    L.oref_svid.argtypes = [P, I, I, P, P, P, P, I, ctypes.c_double]
    L.oref_rmsnorm.argtypes = [P, I, I, P, ctypes.c_double, P]
    L.oref_swiglu.argtypes = [P, P, I, P]
    L.oref_billm_binarize.argtypes = [P, I, I, P, P, P, P]
    L.oref_billm_linear.argtypes = [P, I, I, I, P, P, P, P, P, P]
    L.oref_onebit_bits.argtypes = [ctypes.c_int64, ctypes.c_int64]
    L.oref_onebit_bits.restype = ctypes.c_int64
    L.oref_onebit_params.argtypes = [ctypes.c_int64, ctypes.c_int64]
    L.oref_onebit_params.restype = ctypes.c_int64
    for f in ("oref_pack_ternary", "oref_pack_sign", "oref_quant_act",
              "oref_ternary_linear", "oref_ob_linear", "oref_svid", "oref_rmsnorm", "oref_swiglu",
              "oref_billm_binarize", "oref_billm_linear"):
        getattr(L, f).restype = I
    return L


class OracleError(RuntimeError):
    pass


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise OracleError(f"{what}: oracle error {rc}")
    return rc


def _half_bits(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.float16:
        return _c(x.view(np.uint16), np.uint16)
    if x.dtype == np.uint16:
        return _c(x, np.uint16)
    raise TypeError("expected float16 (or its uint16 bit pattern)")


def half_to_double(bits: int) -> float:
    return lib().oref_half_to_double(int(bits))


def double_to_half(v: float) -> int:
    return lib().oref_double_to_half(float(v))


def float_to_half(v: float) -> int:
    return lib().oref_float_to_half(float(v))


def pack_ternary(w: np.ndarray) -> np.ndarray:
    """int8 [N,K] in {-1,0,1} -> uint32 [N, K/16] (2-bit codes t+1)."""
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.zeros((N, K // 16), dtype=np.uint32)
    _check(lib().oref_pack_ternary(_p(w), N, K, _p(out)), "pack_ternary")
    return out


def pack_sign(w: np.ndarray) -> np.ndarray:
    """fp16 [N,K] -> uint32 [N, K/32]; bit set iff w >= 0 (sign(0) = +1)."""
    wb = _half_bits(w)
    N, K = wb.shape
    out = np.zeros((N, K // 32), dtype=np.uint32)
    _check(lib().oref_pack_sign(_p(wb), N, K, _p(out)), "pack_sign")
    return out


def quant_act(x: np.ndarray):
    """fp16 [M,K] -> (q int8 [M,K], s fp32 [M])."""
    xb = _half_bits(x)
    M, K = xb.shape
    q = np.zeros((M, K), dtype=np.int8)
    s = np.zeros((M,), dtype=np.float32)
    _check(lib().oref_quant_act(_p(xb), M, K, _p(q), _p(s)), "quant_act")
    return q, s


def ternary_linear(x: np.ndarray, w2: np.ndarray, w_scale: float, parallel: bool = False):
    """BitLinear forward: returns (y fp16 [M,N], acc int32 [M,N]).  parallel:
    the OpenMP build (output rows on all host cores, same results)."""
    xb = _half_bits(x)
    w2 = _c(w2, np.uint32)
    M, K = xb.shape
    N = w2.shape[0]
    assert w2.shape[1] * 16 == K
    y = np.zeros((M, N), dtype=np.uint16)
    acc = np.zeros((M, N), dtype=np.int32)
    _check(lib(parallel).oref_ternary_linear(_p(xb), M, K, N, _p(w2), float(w_scale), _p(y), _p(acc)),
           "ternary_linear")
    return y.view(np.float16), acc


def ob_linear(x: np.ndarray, s1: np.ndarray, g: np.ndarray, h: np.ndarray,
              parallel: bool = False):
    """OneBit forward: returns (y fp16 [M,N], z fp64 [M,N] before fp16 rounding).
    parallel: the OpenMP build (output rows on all host cores, same results)."""
    xb = _half_bits(x)
    s1 = _c(s1, np.uint32)
    gb = _half_bits(g)
    hb = _half_bits(h)
    M, K = xb.shape
    N = s1.shape[0]
    assert s1.shape[1] * 32 == K and gb.shape == (K,) and hb.shape == (N,)
    y = np.zeros((M, N), dtype=np.uint16)
    z = np.zeros((M, N), dtype=np.float64)
    _check(lib(parallel).oref_ob_linear(_p(xb), M, K, N, _p(s1), _p(gb), _p(hb), _p(y), _p(z)),
           "ob_linear")
    return y.view(np.float16), z


def svid(W: np.ndarray, max_iter: int = 1000, tol: float = 1e-12):
    """SVID of fp32 W [N,K]: returns (S int8 +-1, a fp64 [N], b fp64 [K], sigma, iters)."""
    W = _c(W, np.float32)
    N, K = W.shape
    S = np.zeros((N, K), dtype=np.int8)
    a = np.zeros((N,), dtype=np.float64)
    b = np.zeros((K,), dtype=np.float64)
    sig = ctypes.c_double(0.0)
    it = _check(lib().oref_svid(_p(W), N, K, _p(S), _p(a), _p(b), ctypes.byref(sig),
                                int(max_iter), float(tol)), "svid")
    return S, a, b, sig.value, it


def billm_binarize(W: np.ndarray):
    """BiLLM binary residual approximation of fp32 W [N,K]:
    returns (B_o int8 +-1 [N,K], B_r int8 +-1 [N,K], alpha_o fp64 [N], alpha_r fp64 [N])."""
    W = _c(W, np.float32)
    N, K = W.shape
    Bo = np.zeros((N, K), dtype=np.int8)
    Br = np.zeros((N, K), dtype=np.int8)
    ao = np.zeros((N,), dtype=np.float64)
    ar = np.zeros((N,), dtype=np.float64)
    _check(lib().oref_billm_binarize(_p(W), N, K, _p(Bo), _p(Br), _p(ao), _p(ar)), "billm_binarize")
    return Bo, Br, ao, ar


def billm_linear(x: np.ndarray, bo1: np.ndarray, br1: np.ndarray, alpha_o: np.ndarray,
                 alpha_r: np.ndarray, parallel: bool = False):
    """Two-plane binary linear: returns (y fp16 [M,N], z fp64 [M,N]) for fp16 x
    [M,K], packed sign planes [N, K/32] and fp16 scales [N]."""
    xb = _half_bits(np.atleast_2d(x))
    bo1, br1 = _c(bo1, np.uint32), _c(br1, np.uint32)
    aob, arb = _half_bits(alpha_o), _half_bits(alpha_r)
    M, K = xb.shape
    N = bo1.shape[0]
    assert bo1.shape == (N, K // 32) and br1.shape == bo1.shape and aob.shape == (N,) and arb.shape == (N,)
    y = np.zeros((M, N), dtype=np.uint16)
    z = np.zeros((M, N), dtype=np.float64)
    _check(lib(parallel).oref_billm_linear(_p(xb), M, K, N, _p(bo1), _p(br1), _p(aob), _p(arb), _p(y),
                                           _p(z)), "billm_linear")
    return y.view(np.float16), z


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of each token (row) of fp16 x [M,K] with fp16 weight gamma [K] -> fp16 [M,K]."""
    xb = _half_bits(np.atleast_2d(x))
    gb = _half_bits(gamma)
    M, K = xb.shape
    assert gb.shape == (K,)
    y = np.zeros((M, K), dtype=np.uint16)
    _check(lib().oref_rmsnorm(_p(xb), M, K, _p(gb), float(eps), _p(y)), "rmsnorm")
    return y.view(np.float16)


def swiglu(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """fp16((a / (1 + exp(-a))) * b), elementwise over fp16 arrays of one shape."""
    ab = _half_bits(a).reshape(-1)
    bb = _half_bits(b).reshape(-1)
    assert ab.shape == bb.shape
    y = np.zeros(ab.shape, dtype=np.uint16)
    _check(lib().oref_swiglu(_p(ab), _p(bb), ab.size, _p(y)), "swiglu")
    return y.view(np.float16).reshape(np.asarray(a).shape)


def onebit_bits(N: int, K: int) -> int:
    return lib().oref_onebit_bits(N, K)


def onebit_params(N: int, K: int) -> int:
    return lib().oref_onebit_params(N, K)
