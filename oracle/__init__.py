"""MixQ CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and the two share no code.

This module only marshals numpy arrays into the plain C oracle in
``mixq_oracle.c`` (built by :func:`build`); every step of the arithmetic lives
in that C file, which cites the passages it follows.  fp16 arrays cross the
boundary as their raw binary16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mixq_oracle.c")
_LIB = os.path.join(_HERE, "libmixq_oracle.so")
# A planted-mistake build of the oracle (oracle/mutation_check.py) is loaded in
# place of the real one when this names its shared library.
_LIB_OVERRIDE = os.environ.get("MIXQ_ORACLE_LIB")
GROUP = 128
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-Wall", "-Wextra"]

_ERRORS = {1: "invalid argument", 2: "non-finite input", 3: "int32 overflow"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: -O2, no fp contraction, no fast-math, OpenMP."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.run(["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"], check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB_OVERRIDE or _LIB)
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: {_ERRORS.get(rc, rc)}")


def _f16bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.float16
    return x.view(np.uint16)


def _idx(idx) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))


def k_out_pad(k_out: int) -> int:
    """Outlier slice width rounded up to a multiple of 64 (zero filled)."""
    return (k_out + 63) // 64 * 64


def prepack_w8(W: np.ndarray, idx):
    """Per-output-channel INT8 weights + outlier weight columns.

    Returns (Wq int8 [N,K], s_w f32 [N], W_out f16 [N,K_out_pad])."""
    lib = _load()
    N, K = W.shape
    idx = _idx(idx)
    ko, kp = len(idx), k_out_pad(len(idx))
    Wq = np.empty((N, K), np.int8)
    s_w = np.empty(N, np.float32)
    W_out = np.zeros((N, kp), np.uint16)
    rc = lib.oracle_prepack_w8(_p(_f16bits(W)), N, K, _p(idx), ko, kp, _p(Wq), _p(s_w), _p(W_out))
    _check(rc, "prepack_w8")
    return Wq, s_w, W_out.view(np.float16)


def prepack_w4(Wq8: np.ndarray):
    """Progressive level-2 (group 128) of INT8 codes.

    Returns logical (q u8 [N,K], s2 u8 [N,K/128], z2 u8 [N,K/128], w8eff int8 [N,K])."""
    lib = _load()
    Wq8 = np.ascontiguousarray(Wq8, dtype=np.int8)
    N, K = Wq8.shape
    q = np.empty((N, K), np.uint8)
    s2 = np.empty((N, K // GROUP), np.uint8)
    z2 = np.empty((N, K // GROUP), np.uint8)
    w8 = np.empty((N, K), np.int8)
    rc = lib.oracle_prepack_w4(_p(Wq8), N, K, _p(q), _p(s2), _p(z2), _p(w8))
    _check(rc, "prepack_w4")
    return q, s2, z2, w8


def prepack_w4b(W: np.ndarray):
    """4-bit reading B: per (row, group of 128) fp16 scale and integer zero.

    Returns logical (q u8 [N,K], s_g f16 [N,K/128], z_g u8 [N,K/128])."""
    lib = _load()
    N, K = W.shape
    q = np.empty((N, K), np.uint8)
    s_g = np.empty((N, K // GROUP), np.uint16)
    z_g = np.empty((N, K // GROUP), np.uint8)
    rc = lib.oracle_prepack_w4b(_p(_f16bits(W)), N, K, _p(q), _p(s_g), _p(z_g))
    _check(rc, "prepack_w4b")
    return q, s_g.view(np.float16), z_g


def linear_w4b(Xq, s_x, X_out, q, s_g, z_g, W_out, m0: int = 0, m1: int | None = None):
    """Layer output (fp64) with reading-B weights for rows [m0,m1).

    Returns (part int32 [m1-m0, N, K/128] per-group partial sums, y f64 [m1-m0, N])."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    q = np.ascontiguousarray(q, dtype=np.uint8)
    z_g = np.ascontiguousarray(z_g, dtype=np.uint8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    M, K = Xq.shape
    N = q.shape[0]
    kp = 0 if X_out is None else X_out.shape[1]
    xo = _f16bits(X_out) if kp else None
    wo = _f16bits(W_out) if kp else None
    m1 = M if m1 is None else m1
    part = np.empty((m1 - m0, N, K // GROUP), np.int32)
    y = np.empty((m1 - m0, N), np.float64)
    rc = lib.oracle_linear_w4b(_p(Xq), _p(s_x), _p(xo), _p(q), _p(_f16bits(s_g)), _p(z_g),
                               _p(wo), M, N, K, kp, m0, m1, _p(part), _p(y))
    _check(rc, "linear_w4b")
    return part, y


def linear_w4b_points(Xq, s_x, X_out, q, s_g, z_g, W_out, ms, ns):
    """Reading-B layer output (fp64) and per-group partial sums at sampled points."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    q = np.ascontiguousarray(q, dtype=np.uint8)
    z_g = np.ascontiguousarray(z_g, dtype=np.uint8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    ms = _idx(ms)
    ns = _idx(ns)
    M, K = Xq.shape
    N = q.shape[0]
    kp = 0 if X_out is None else X_out.shape[1]
    xo = _f16bits(X_out) if kp else None
    wo = _f16bits(W_out) if kp else None
    part = np.empty((len(ms), K // GROUP), np.int32)
    y = np.empty(len(ms), np.float64)
    rc = lib.oracle_linear_w4b_points(_p(Xq), _p(s_x), _p(xo), _p(q), _p(_f16bits(s_g)), _p(z_g),
                                      _p(wo), M, N, K, kp, _p(ms), _p(ns), len(ms), _p(part),
                                      _p(y))
    _check(rc, "linear_w4b_points")
    return part, y


def quantize_act(X: np.ndarray, idx, T: float):
    """Per-token INT8 activations, outlier gather, detection bitmap, flags.

    Returns (Xq int8 [M,K], s_x f32 [M], X_out f16 [M,K_out_pad],
             bitmap u32 [ceil(K/32)], flags int32 [2])."""
    lib = _load()
    M, K = X.shape
    idx = _idx(idx)
    ko, kp = len(idx), k_out_pad(len(idx))
    Xq = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    X_out = np.zeros((M, kp), np.uint16)
    bitmap = np.zeros((K + 31) // 32, np.uint32)
    flags = np.zeros(2, np.int32)
    rc = lib.oracle_quantize_act(_p(_f16bits(X)), M, K, K, _p(idx), ko, kp, ctypes.c_float(T),
                                 _p(Xq), _p(s_x), _p(X_out), _p(bitmap), _p(flags))
    _check(rc, "quantize_act")
    return Xq, s_x, X_out.view(np.float16), bitmap, flags


def rmsnorm(X: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMS-normalised tokens Y = fp16(X / sqrt(mean(X^2) + eps) * g), fp64 inside."""
    lib = _load()
    M, K = X.shape
    Y = np.empty((M, K), np.uint16)
    lib.oracle_rmsnorm.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p]
    rc = lib.oracle_rmsnorm(_p(_f16bits(X)), M, K, K, _p(_f16bits(np.asarray(g, np.float16))),
                            float(eps), _p(Y))
    _check(rc, "rmsnorm")
    return Y.view(np.float16)


def gemm_i32(Xq: np.ndarray, Wq: np.ndarray, m0: int = 0, m1: int | None = None):
    """Exact INT32 accumulators acc[m,n] = sum_k Xq[m,k]*Wq[n,k] for rows [m0,m1)."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    m1 = M if m1 is None else m1
    acc = np.empty((m1 - m0, N), np.int32)
    _check(lib.oracle_gemm_i32(_p(Xq), _p(Wq), M, N, K, m0, m1, _p(acc)), "gemm_i32")
    return acc


def linear(Xq, s_x, X_out, Wq, s_w, W_out, m0: int = 0, m1: int | None = None):
    """Mixed-precision layer output in fp64 for rows [m0,m1). Returns (acc, y)."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = Xq.shape
    N = Wq.shape[0]
    kp = 0 if X_out is None else X_out.shape[1]
    xo = _f16bits(X_out) if kp else None
    wo = _f16bits(W_out) if kp else None
    m1 = M if m1 is None else m1
    acc = np.empty((m1 - m0, N), np.int32)
    y = np.empty((m1 - m0, N), np.float64)
    rc = lib.oracle_linear(_p(Xq), _p(s_x), _p(xo), _p(Wq), _p(s_w), _p(wo), M, N, K, kp, m0, m1,
                           _p(acc), _p(y))
    _check(rc, "linear")
    return acc, y


def linear_points(Xq, s_x, X_out, Wq, s_w, W_out, ms, ns):
    """Mixed-precision layer output (fp64) and INT32 acc at sampled points."""
    lib = _load()
    Xq = np.ascontiguousarray(Xq, dtype=np.int8)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    ms = _idx(ms)
    ns = _idx(ns)
    M, K = Xq.shape
    N = Wq.shape[0]
    kp = 0 if X_out is None else X_out.shape[1]
    xo = _f16bits(X_out) if kp else None
    wo = _f16bits(W_out) if kp else None
    acc = np.empty(len(ms), np.int32)
    y = np.empty(len(ms), np.float64)
    rc = lib.oracle_linear_points(_p(Xq), _p(s_x), _p(xo), _p(Wq), _p(s_w), _p(wo), M, N, K, kp,
                                  _p(ms), _p(ns), len(ms), _p(acc), _p(y))
    _check(rc, "linear_points")
    return acc, y


def round_f16(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to fp16 (nearest even) in one step."""
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, np.uint16)
    lib.oracle_round_f16(_p(y), ctypes.c_longlong(y.size), _p(out))
    return out.view(np.float16)
