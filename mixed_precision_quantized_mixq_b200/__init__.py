"""Python binding of libmixq.so (the C ABI in include/mixq.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  The binding
refuses to run if libmixq.so is missing or no sm_100 GPU is present; there is
no CPU fallback.

Low-level calls keep the C names (``mixq_quantize_act`` ...) and take torch
tensors; :class:`PackedWeights`, :func:`prepack`, :func:`quantize_act`,
:func:`gemm` and :func:`linear` are thin conveniences over them.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmixq.so")

MIXQ_W8, MIXQ_W4G128, MIXQ_W4G128_F16S = 0, 1, 2
STATUS = {0: "MIXQ_OK", 1: "MIXQ_ERR_INVALID_ARG", 2: "MIXQ_ERR_UNSUPPORTED_SHAPE",
          3: "MIXQ_ERR_MISALIGNED", 4: "MIXQ_ERR_CUDA", 5: "MIXQ_ERR_TIMEOUT",
          6: "MIXQ_ERR_NO_DEVICE"}
GROUP = 128

_c = ctypes
_VP, _I, _F, _SZ, _U64 = _c.c_void_p, _c.c_int, _c.c_float, _c.c_size_t, _c.c_uint64
_SIGNATURES = {
    "mixq_last_error": (_c.c_char_p, []),
    "mixq_version": (_I, []),
    "mixq_prepack_size": (_I, [_I, _I, _I, _I, _c.POINTER(_SZ), _c.POINTER(_SZ), _c.POINTER(_SZ)]),
    "mixq_prepack_weights": (_I, [_I, _VP, _I, _I, _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP]),
    "mixq_quantize_act": (_I, [_VP, _I, _I, _I, _VP, _I, _F, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "mixq_quantize_act_static": (_I, [_VP, _I, _I, _I, _VP, _I, _F, _VP, _VP, _VP, _VP, _VP, _VP,
                                      _VP]),
    "mixq_rmsnorm_quantize_act": (_I, [_VP, _I, _I, _I, _VP, _F, _VP, _I, _VP, _I, _F, _VP, _VP,
                                       _VP, _VP, _VP, _VP, _VP]),
    "mixq_merge_outliers": (_I, [_VP, _I, _VP, _I, _VP, _c.POINTER(_I)]),
    "mixq_extract_outlier_weights": (_I, [_VP, _I, _I, _VP, _I, _VP, _VP, _VP]),
    "mixq_gemm_w8a8o16": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _VP,
                               _VP]),
    "mixq_gemm_w4a8o16": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I,
                               _VP, _VP]),
    "mixq_gemm_w4a8o16_f16s": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I,
                                    _VP, _VP]),
    "mixq_gemm_workspace_size": (_SZ, [_I, _I, _I]),
    "mixq_gemm_plan": (_I, [_I, _I, _I, _I, _I, _c.POINTER(_I), _c.POINTER(_I), _c.POINTER(_I)]),
    "mixq_debug_gemm_i32": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _I, _I, _I, _VP, _VP]),
    "mixq_debug_max_active_clusters": (_I, [_I, _I, _I, _I, _c.POINTER(_I)]),
    "mixq_debug_unpack_w8": (_I, [_I, _I, _VP, _VP, _VP]),
    "mixq_debug_unpack_w4": (_I, [_I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "mixq_debug_mma_rate": (_I, [_I, _I, _c.POINTER(_c.c_double), _VP, _VP]),
    "mixq_debug_gemm_stall": (_I, [_I, _I, _I, _VP, _VP, _VP, _VP, _VP, _I, _U64, _VP, _VP]),
}


class MixqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmixq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixed_precision_quantized_mixq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise MixqError(rc, lib().mixq_last_error().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def k_out_pad(k_out: int) -> int:
    return (k_out + 63) // 64 * 64


# ------------------------------------------------------------- raw C names
def mixq_prepack_size(mode: int, N: int, K: int, K_out: int):
    a, b, c = _SZ(), _SZ(), _SZ()
    _check(lib().mixq_prepack_size(mode, N, K, K_out, ctypes.byref(a), ctypes.byref(b),
                                   ctypes.byref(c)))
    return a.value, b.value, c.value


def mixq_prepack_weights(mode, W, idx, Wq, s_w, grp, W_out, status, stream=None):
    N, K = W.shape
    _check(lib().mixq_prepack_weights(mode, _ptr(W), N, K, _ptr(idx), 0 if idx is None else idx.numel(),
                                      _ptr(Wq), _ptr(s_w), _ptr(grp), _ptr(W_out), _ptr(status),
                                      _stream(stream)))


def mixq_quantize_act(X, idx, threshold, Xq, s_x, X_out, bitmap, flags, status, stream=None):
    M, K = X.shape
    _check(lib().mixq_quantize_act(_ptr(X), M, K, X.stride(0), _ptr(idx),
                                   0 if idx is None else idx.numel(), float(threshold), _ptr(Xq),
                                   _ptr(s_x), _ptr(X_out), _ptr(bitmap), _ptr(flags), _ptr(status),
                                   _stream(stream)))


def mixq_quantize_act_static(X, idx, threshold, Xq, s_x, X_out, bitmap, flags, status,
                             stream=None):
    """mixq_quantize_act with its completion ticket in the library's own static
    scratch: flags has two words, and the call allocates nothing."""
    M, K = X.shape
    _check(lib().mixq_quantize_act_static(_ptr(X), M, K, X.stride(0), _ptr(idx),
                                          0 if idx is None else idx.numel(), float(threshold),
                                          _ptr(Xq), _ptr(s_x), _ptr(X_out), _ptr(bitmap),
                                          _ptr(flags), _ptr(status), _stream(stream)))


def mixq_rmsnorm_quantize_act(X, gamma, eps, Xn, idx, threshold, Xq, s_x, X_out, bitmap, flags,
                              status, stream=None):
    M, K = X.shape
    _check(lib().mixq_rmsnorm_quantize_act(_ptr(X), M, K, X.stride(0), _ptr(gamma), float(eps),
                                           _ptr(Xn), 0 if Xn is None else Xn.stride(0), _ptr(idx),
                                           0 if idx is None else idx.numel(), float(threshold),
                                           _ptr(Xq), _ptr(s_x), _ptr(X_out), _ptr(bitmap),
                                           _ptr(flags), _ptr(status), _stream(stream)))


def mixq_gemm_w8a8o16(M, N, K, K_out, Xq, s_x, X_out, Wq, s_w, W_out, flags, Y, status,
                      stream=None):
    _check(lib().mixq_gemm_w8a8o16(M, N, K, K_out, _ptr(Xq), _ptr(s_x), _ptr(X_out), _ptr(Wq),
                                   _ptr(s_w), _ptr(W_out), _ptr(flags), _ptr(Y), Y.stride(0),
                                   _ptr(status), _stream(stream)))


def mixq_gemm_w4a8o16(M, N, K, K_out, Xq, s_x, X_out, Wq4, grp, s_w, W_out, flags, Y, status,
                      stream=None):
    _check(lib().mixq_gemm_w4a8o16(M, N, K, K_out, _ptr(Xq), _ptr(s_x), _ptr(X_out), _ptr(Wq4),
                                   _ptr(grp), _ptr(s_w), _ptr(W_out), _ptr(flags), _ptr(Y),
                                   Y.stride(0), _ptr(status), _stream(stream)))


def mixq_gemm_w4a8o16_f16s(M, N, K, K_out, Xq, s_x, X_out, Wq4, grp, W_out, flags, Y, status,
                           stream=None):
    _check(lib().mixq_gemm_w4a8o16_f16s(M, N, K, K_out, _ptr(Xq), _ptr(s_x), _ptr(X_out),
                                        _ptr(Wq4), _ptr(grp), _ptr(W_out), _ptr(flags), _ptr(Y),
                                        Y.stride(0), _ptr(status), _stream(stream)))


def mixq_gemm_plan(mode: int, M: int, N: int, K: int, num_sms: int = 0):
    bn, split, ctas = _I(), _I(), _I()
    _check(lib().mixq_gemm_plan(mode, M, N, K, num_sms, ctypes.byref(bn), ctypes.byref(split),
                                ctypes.byref(ctas)))
    return bn.value, split.value, ctas.value


def mixq_debug_gemm_i32(mode, Xq, Wq, grp, acc, N, bn=0, split=0, status=None, stream=None):
    M, K = Xq.shape
    _check(lib().mixq_debug_gemm_i32(mode, M, N, K, _ptr(Xq), _ptr(Wq), _ptr(grp), _ptr(acc),
                                     acc.stride(0), bn, split, _ptr(status), _stream(stream)))


def mixq_debug_max_active_clusters(mode: int, bn: int, split: int, small_m: int = 0) -> int:
    n = _I()
    _check(lib().mixq_debug_max_active_clusters(mode, bn, split, small_m, ctypes.byref(n)))
    return n.value


def mixq_debug_unpack_w8(N, K, Wq, out, stream=None):
    _check(lib().mixq_debug_unpack_w8(N, K, _ptr(Wq), _ptr(out), _stream(stream)))


def mixq_debug_unpack_w4(N, K, Wq4, grp, q, s2, z2, status=None, stream=None):
    _check(lib().mixq_debug_unpack_w4(N, K, _ptr(Wq4), _ptr(grp), _ptr(q), _ptr(s2), _ptr(z2),
                                      _ptr(status), _stream(stream)))


def mixq_debug_gemm_stall(Xq, Wq, s_x, s_w, Y, wait_limit_ns, status, stream=None):
    M, K = Xq.shape
    N = Wq.shape[0]
    _check(lib().mixq_debug_gemm_stall(M, N, K, _ptr(Xq), _ptr(Wq), _ptr(s_x), _ptr(s_w), _ptr(Y),
                                       Y.stride(0), int(wait_limit_ns), _ptr(status),
                                       _stream(stream)))


def mixq_debug_mma_rate(kind: int, iters: int, status=None, stream=None) -> float:
    """Launch the tensor-core rate loop (kind 0 = kind::i8, 1 = kind::f16); returns the
    operations the launch performs (time it with events on the stream)."""
    ops = _c.c_double()
    _check(lib().mixq_debug_mma_rate(kind, iters, ctypes.byref(ops), _ptr(status),
                                     _stream(stream)))
    return ops.value


# ------------------------------------------------------------ conveniences
def _require_cuda():
    import torch
    if not torch.cuda.is_available():
        raise MixqError(6, "no CUDA device: the MixQ layer runs only on an sm_100 GPU")
    return torch


@dataclass
class PackedWeights:
    """Prepacked layer weights (all device tensors)."""
    mode: int
    N: int
    K: int
    idx: "object"      # int32 [K_out]
    Wq: "object"       # tiled codes: int8 [N*K] (W8) or uint8 [N*K/2] (4-bit), see mixq.h
    s_w: "object"      # fp32 [N], or None (MIXQ_W4G128_F16S)
    grp: "object"      # fp16 [K/128, N, 2] group pairs (4-bit) or None
    W_out: "object"    # fp16 [N, K_out_pad] or None

    @property
    def k_out(self) -> int:
        return self.idx.numel()


def merge_outliers(bitmap, idx, K: int):
    """Sorted union of the outlier channels idx and the channels set in a detection
    bitmap (both device tensors), as a new device int32 tensor (host merge, one sync)."""
    import numpy as np
    torch = _require_cuda()
    bm = bitmap.detach().to("cpu").contiguous().view(torch.int32).numpy().view(np.uint32)
    old = idx.detach().to("cpu", torch.int32).contiguous().numpy()
    out = np.empty(K, dtype=np.int32)
    n = _I()
    _check(lib().mixq_merge_outliers(bm.ctypes.data, K, old.ctypes.data if old.size else None,
                                     old.size, out.ctypes.data, ctypes.byref(n)))
    return torch.from_numpy(out[:n.value].copy()).to(idx.device if idx.numel() else bitmap.device)


def update_outliers(w: PackedWeights, W, idx_new, status=None, stream=None) -> PackedWeights:
    """The same prepacked codes with the outlier columns rebuilt for a new outlier set
    (W: the layer's fp16 weights [N, K] on the device)."""
    torch = _require_cuda()
    idx_new = torch.as_tensor(idx_new, dtype=torch.int32, device=W.device).contiguous()
    ko = idx_new.numel()
    W_out = torch.empty((w.N, k_out_pad(ko)), dtype=torch.float16, device=W.device) if ko else None
    if ko:
        _check(lib().mixq_extract_outlier_weights(_ptr(W.contiguous()), w.N, w.K, _ptr(idx_new), ko,
                                                  _ptr(W_out), _ptr(status), _stream(stream)))
    return PackedWeights(w.mode, w.N, w.K, idx_new, w.Wq, w.s_w, w.grp, W_out)


def column_shard(N: int, rank: int, world: int) -> tuple[int, int]:
    """Output channels [n0, n1) that one rank holds in an N-split (column-parallel)
    layer: equal shards of whole 128-channel weight tiles."""
    if world < 1 or not 0 <= rank < world or N % (128 * world):
        raise ValueError(f"N = {N} does not split into {world} shards of whole 128-channel tiles")
    per = N // world
    return rank * per, (rank + 1) * per


def prepack_shard(W, idx, mode: int, rank: int, world: int, status=None,
                  stream=None) -> PackedWeights:
    """Prepack this rank's rows of W [N, K] for an N-split layer (each output channel
    is quantized on its own, so a shard's codes equal those rows of the full prepack)."""
    n0, n1 = column_shard(W.shape[0], rank, world)
    return prepack(W[n0:n1], idx, mode, status=status, stream=stream)


def gather_columns(Y_local, world: int, group=None):
    """All-gather the [M, N/world] output shards of an N-split layer into [M, N] in rank
    order, over torch.distributed (NCCL between GPUs)."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(Y_local) for _ in range(world)]
    dist.all_gather(parts, Y_local.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def status_tensor(device=None):
    torch = _require_cuda()
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def check_status(status) -> None:
    """Raise if a kernel recorded a device-side error in `status` (syncs)."""
    v = int(status.item())
    if v != 0:
        raise MixqError(v, "device-side error recorded by a kernel")


def prepack(W, idx, mode: int = MIXQ_W8, status=None, stream=None) -> PackedWeights:
    """Quantize fp16 weights W [N, K] (device) for the layer; idx = sorted outlier channels."""
    torch = _require_cuda()
    N, K = W.shape
    dev = W.device
    idx = torch.as_tensor(idx, dtype=torch.int32, device=dev).contiguous()
    ko = idx.numel()
    if mode == MIXQ_W8:
        Wq = torch.empty(N * K, dtype=torch.int8, device=dev)
        grp = None
    else:
        Wq = torch.empty(N * K // 2, dtype=torch.uint8, device=dev)
        grp = torch.empty((K // GROUP, N, 2), dtype=torch.float16, device=dev)
    s_w = torch.empty(N, dtype=torch.float32, device=dev) if mode != MIXQ_W4G128_F16S else None
    W_out = torch.empty((N, k_out_pad(ko)), dtype=torch.float16, device=dev) if ko else None
    mixq_prepack_weights(mode, W.contiguous(), idx if ko else None, Wq, s_w, grp, W_out, status,
                         stream)
    return PackedWeights(mode, N, K, idx, Wq, s_w, grp, W_out)


@dataclass
class QuantAct:
    Xq: "object"      # int8 [M, K]
    s_x: "object"     # fp32 [M]
    X_out: "object"   # fp16 [M, K_out_pad] or None
    bitmap: "object"  # int32 view of uint32 [K/32]
    flags: "object"   # int32 [4]


def quantize_act(X, idx, threshold: float = 6.0, out: QuantAct | None = None, status=None,
                 stream=None) -> QuantAct:
    torch = _require_cuda()
    M, K = X.shape
    dev = X.device
    ko = idx.numel()
    if out is None:
        out = QuantAct(torch.empty((M, K), dtype=torch.int8, device=dev),
                       torch.empty(M, dtype=torch.float32, device=dev),
                       torch.empty((M, k_out_pad(ko)), dtype=torch.float16, device=dev) if ko else None,
                       torch.empty(K // 32, dtype=torch.int32, device=dev),
                       torch.empty(4, dtype=torch.int32, device=dev))
    mixq_quantize_act(X, idx if ko else None, threshold, out.Xq, out.s_x, out.X_out, out.bitmap,
                      out.flags, status, stream)
    return out


def rmsnorm_quantize_act(X, gamma, eps: float, idx, threshold: float = 6.0,
                         out: QuantAct | None = None, Xn=None, status=None,
                         stream=None) -> QuantAct:
    """RMS-normalise each token (gain gamma, eps) and run the activation pass on
    the result in the same kernel; Xn (optional) receives the normalised tokens."""
    torch = _require_cuda()
    M, K = X.shape
    dev = X.device
    ko = idx.numel()
    if out is None:
        out = QuantAct(torch.empty((M, K), dtype=torch.int8, device=dev),
                       torch.empty(M, dtype=torch.float32, device=dev),
                       torch.empty((M, k_out_pad(ko)), dtype=torch.float16, device=dev) if ko else None,
                       torch.empty(K // 32, dtype=torch.int32, device=dev),
                       torch.empty(4, dtype=torch.int32, device=dev))
    mixq_rmsnorm_quantize_act(X, gamma, eps, Xn, idx if ko else None, threshold, out.Xq, out.s_x,
                              out.X_out, out.bitmap, out.flags, status, stream)
    return out


def gemm(q: QuantAct, w: PackedWeights, Y=None, status=None, stream=None):
    torch = _require_cuda()
    M, K = q.Xq.shape
    if Y is None:
        Y = torch.empty((M, w.N), dtype=torch.float16, device=q.Xq.device)
    if w.mode == MIXQ_W8:
        mixq_gemm_w8a8o16(M, w.N, K, w.k_out, q.Xq, q.s_x, q.X_out, w.Wq, w.s_w, w.W_out, q.flags,
                          Y, status, stream)
    elif w.mode == MIXQ_W4G128:
        mixq_gemm_w4a8o16(M, w.N, K, w.k_out, q.Xq, q.s_x, q.X_out, w.Wq, w.grp, w.s_w, w.W_out,
                          q.flags, Y, status, stream)
    else:
        mixq_gemm_w4a8o16_f16s(M, w.N, K, w.k_out, q.Xq, q.s_x, q.X_out, w.Wq, w.grp, w.W_out,
                               q.flags, Y, status, stream)
    return Y


def linear(X, w: PackedWeights, threshold: float = 6.0, status=None, stream=None):
    """Y = MixQ layer(X) for fp16 X [M, K] on the device: quantize, then GEMM."""
    q = quantize_act(X, w.idx, threshold, status=status, stream=stream)
    return gemm(q, w, status=status, stream=stream), q
