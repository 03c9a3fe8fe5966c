"""fp64 CPU oracle for residual binarization -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the bench's CPU-baseline leg may
import this module. The product (the CUDA library and its Python binding)
never imports it and shares no code with it.

The arithmetic lives in ``rb_oracle.c`` (plain C, fp64, OpenMP over rows);
this wrapper only converts numpy arrays and loads the shared object, building
it with gcc on first use. See ``rb_oracle.c`` for the passages each function
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rb_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile rb_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64, i32 = ctypes.c_int64, ctypes.c_int32
            lib.rbo_pack.argtypes = [p, i64, i64, i32, i64, p, p, p]
            lib.rbo_pack.restype = ctypes.c_int
            lib.rbo_matvec.argtypes = [p, p, i64, i64, i32, i64, p, i64, p, p]
            lib.rbo_matvec.restype = ctypes.c_int
            lib.rbo_pack_fixed.argtypes = [p, i64, i64, i32, p, p, p, p]
            lib.rbo_pack_fixed.restype = ctypes.c_int
            lib.rbo_dual_matvec.argtypes = [p, p, i64, i64, i32, p, i64, p, p]
            lib.rbo_dual_matvec.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def pack(W: np.ndarray, n_paths: int, group: int = 0, want_rabs: bool = False):
    """Derive N residual sign planes and scales from one weight matrix.

    W: (M, K) float16/float32/float64. group: 0 for one scale per row, else the
    number of columns per scale. Returns (planes uint32 [N, M, K/32],
    alpha float64 [N, M, K/G], rabs float64 [N, M, K] or None).
    """
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = W.shape
    G = K if group == 0 else group
    planes = np.zeros((n_paths, M, K // 32), dtype=np.uint32)
    alpha = np.zeros((n_paths, M, K // G), dtype=np.float64)
    rabs = np.zeros((n_paths, M, K), dtype=np.float64) if want_rabs else None
    rc = _load().rbo_pack(_ptr(W), M, K, n_paths, G, _ptr(planes), _ptr(alpha),
                          _ptr(rabs) if rabs is not None else None)
    if rc != 0:
        raise ValueError(f"bad shape M={M} K={K} N={n_paths} G={G}")
    return planes, alpha, rabs


def matvec(planes: np.ndarray, alpha: np.ndarray, x: np.ndarray):
    """y[t, i] = sum_k sum_j alpha_k[i, g(j)] * (+-1) * x[t, j] and its tolerance scale.

    planes uint32 [N, M, K/32]; alpha [N, M, K/G] (any float dtype, widened to
    fp64); x [T, K]. Returns (y float64 [T, M], denom float64 [T, M]).
    """
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float64)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    N, M, W32 = planes.shape
    K = W32 * 32
    G = K // alpha.shape[2]
    T = x.shape[0]
    if x.shape[1] != K or alpha.shape[:2] != (N, M):
        raise ValueError("shape mismatch")
    y = np.zeros((T, M), dtype=np.float64)
    den = np.zeros((T, M), dtype=np.float64)
    rc = _load().rbo_matvec(_ptr(planes), _ptr(alpha), M, K, N, G, _ptr(x), T, _ptr(y), _ptr(den))
    if rc != 0:
        raise ValueError("bad shape")
    return y, den


def pack_fixed(W: np.ndarray, h: np.ndarray, g: np.ndarray | None = None, want_rabs: bool = False):
    """Sign planes of the dual-scale block for given scales (RaBiT 4.1-4.2).

    W (M, K); h (N, M) output-channel scales; g (N, K) input-channel scales or
    None (all ones). R_0 = W, B_k = sign(R_{k-1}),
    R_k = R_{k-1} - h_k[i] g_k[j] B_k. Returns (planes uint32 [N, M, K/32],
    rabs float64 [N, M, K] or None).
    """
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = W.shape
    h = np.ascontiguousarray(h, dtype=np.float64)
    N = h.shape[0]
    if h.shape != (N, M):
        raise ValueError("h must be (N, M)")
    if g is not None:
        g = np.ascontiguousarray(g, dtype=np.float64)
        if g.shape != (N, K):
            raise ValueError("g must be (N, K)")
    planes = np.zeros((N, M, K // 32), dtype=np.uint32)
    rabs = np.zeros((N, M, K), dtype=np.float64) if want_rabs else None
    rc = _load().rbo_pack_fixed(_ptr(W), M, K, N, _ptr(h), _ptr(g) if g is not None else None, _ptr(planes),
                                _ptr(rabs) if rabs is not None else None)
    if rc != 0:
        raise ValueError(f"bad shape M={M} K={K} N={N}")
    return planes, rabs


def dual_inputs(g: np.ndarray | None, x: np.ndarray, n_paths: int) -> np.ndarray:
    """x_k = g_k (.) x rounded to the nearest fp16 (the activation the binary
    core of path k sees): [N, T, K] float64 holding fp16 values."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if g is None:
        g = np.ones((n_paths, x.shape[1]))
    g = np.asarray(g, dtype=np.float64)
    return (g[:, None, :] * x[None, :, :]).astype(np.float16).astype(np.float64)


def dual_matvec(planes: np.ndarray, h: np.ndarray, xk: np.ndarray):
    """y[t, i] = sum_k h_k[i] sum_j (+-1) xk[k, t, j] and its tolerance scale.

    planes uint32 [N, M, K/32]; h [N, M]; xk [N, T, K] (from dual_inputs).
    Returns (y float64 [T, M], denom float64 [T, M]).
    """
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    h = np.ascontiguousarray(h, dtype=np.float64)
    xk = np.ascontiguousarray(xk, dtype=np.float64)
    N, M, W32 = planes.shape
    K = W32 * 32
    T = xk.shape[1]
    if h.shape != (N, M) or xk.shape != (N, T, K):
        raise ValueError("shape mismatch")
    y = np.zeros((T, M), dtype=np.float64)
    den = np.zeros((T, M), dtype=np.float64)
    rc = _load().rbo_dual_matvec(_ptr(planes), _ptr(h), M, K, N, _ptr(xk), T, _ptr(y), _ptr(den))
    if rc != 0:
        raise ValueError("bad shape")
    return y, den


def reconstruct_f16(planes: np.ndarray, alpha: np.ndarray) -> np.ndarray:
    """W^ = sum_k alpha_k (.) B_k (RaBiT 4.1), summed exactly in fp64 and
    rounded once to the nearest fp16: the operand of the reconstruct-once
    contraction. planes uint32 [N, M, K/32]; alpha [N, M, K/G]. Returns
    float16 [M, K]."""
    planes = np.ascontiguousarray(planes, dtype="<u4")
    N, M, W32 = planes.shape
    K = W32 * 32
    G = K // alpha.shape[2]
    bits = np.unpackbits(planes.view(np.uint8), axis=-1, bitorder="little").reshape(N, M, K)
    signs = np.where(bits == 1, 1.0, -1.0)
    What = (np.repeat(np.asarray(alpha, dtype=np.float64), G, axis=2) * signs).sum(0)
    return What.astype(np.float16)


def dense_matvec(W: np.ndarray, x: np.ndarray):
    """y = x W^T in fp64 (BLAS) for a dense weight, with the tolerance scale
    D = |x| |W|^T. W [M, K]; x [T, K]. Returns (y [T, M], D [T, M])."""
    W = np.asarray(W, dtype=np.float64)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    return x @ W.T, np.abs(x) @ np.abs(W).T


def silu_gate(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """h = silu(g) u = g u / (1 + e^-g) in fp64: the gate of the gated MLP
    block of the Llama models whose decode RaBiT section 5 times (the pages
    do not print the block; this is that architecture's SiLU gate)."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * np.asarray(u, dtype=np.float64)


def swiglu_matvec(planes: np.ndarray, alpha: np.ndarray, x: np.ndarray):
    """The gated pair evaluated from its planes: planes [2N, M, K/32] and
    alpha [2N, M, K/G] hold the gate G's N paths, then the up projection
    U's. g = G x and u = U x are the pinned matvec of each half; h =
    silu_gate(g, u). Returns (h, g, u, Dg, Du), fp64 [T, M]; Dg, Du are the
    matvec tolerance scales of g and u."""
    n2 = planes.shape[0]
    if n2 % 2:
        raise ValueError("expected the gate's and the up projection's paths")
    n = n2 // 2
    g, dg = matvec(planes[:n], alpha[:n], x)
    u, du = matvec(planes[n:], alpha[n:], x)
    return silu_gate(g, u), g, u, dg, du


def alpha_to_f16(alpha: np.ndarray) -> np.ndarray:
    """Round fp64 scales to the nearest fp16 (ties to even): the stored fp16 copy."""
    return np.asarray(alpha, dtype=np.float64).astype(np.float16)


from .compare import (  # noqa: E402,F401
    compare_planes,
    compare_scales,
    compare_scales_f16,
    compare_outputs,
)
