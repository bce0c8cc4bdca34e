"""Shared test helpers: run the CUDA path through the C ABI binding and the
oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import numpy as np

import oracle

# FP16 output tolerance of the layer (the target's statement): |Y - y| <= max(1e-3, 1e-2 |y|)
ATOL, RTOL = 1e-3, 1e-2


def y_close(Y: np.ndarray, y: np.ndarray) -> np.ndarray:
    return np.abs(Y.astype(np.float64) - y) <= np.maximum(ATOL, RTOL * np.abs(y))


def assert_y_close(Y, y, what=""):
    ok = y_close(Y, y)
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        detail = ", ".join(f"{tuple(b)}: got {Y[tuple(b)]} want {y[tuple(b)]}" for b in bad)
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outputs out of tolerance "
                             f"({detail})")


def oracle_weights(W: np.ndarray, idx, mode: str):
    """Oracle prepack: (effective int8 weights, s_w, W_out, extras)."""
    Wq8, s_w, W_out = oracle.prepack_w8(W, idx)
    if mode == "w8":
        return Wq8, s_w, W_out, {"Wq8": Wq8}
    q, s2, z2, w8eff = oracle.prepack_w4(Wq8)
    return w8eff, s_w, W_out, {"Wq8": Wq8, "q": q, "s2": s2, "z2": z2}


def oracle_layer(X, W, idx, mode: str, T: float, rows=None):
    """Oracle of the whole layer; rows=None -> every row, else a (m0, m1) window."""
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, T)
    Weff, s_w, W_out, extra = oracle_weights(W, idx, mode)
    m0, m1 = (0, X.shape[0]) if rows is None else rows
    xo = X_out if X_out.shape[1] else None
    wo = W_out if W_out.shape[1] else None
    acc, y = oracle.linear(Xq, s_x, xo, Weff, s_w, wo, m0, m1)
    return dict(Xq=Xq, s_x=s_x, X_out=X_out, bitmap=bitmap, flags=flags, Weff=Weff, s_w=s_w,
                W_out=W_out, acc=acc, y=y, **extra)


class Gpu:
    """Runs the CUDA path on device tensors (imports torch lazily)."""

    def __init__(self):
        import torch
        import mixed_precision_quantized_mixq_b200 as mq
        self.torch, self.mq = torch, mq

    def dev(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a)).cuda()

    def layer(self, X, W, idx, mode: str, T: float):
        torch, mq = self.torch, self.mq
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        Xd, Wd = self.dev(X), self.dev(W)
        idxd = self.dev(np.asarray(idx, np.int32))
        w = mq.prepack(Wd, idxd, mq.MIXQ_W8 if mode == "w8" else mq.MIXQ_W4G128, status=status)
        Y, q = mq.linear(Xd, w, T, status=status)
        torch.cuda.synchronize()
        out = dict(Y=Y.cpu().numpy(), Xq=q.Xq.cpu().numpy(), s_x=q.s_x.cpu().numpy(),
                   X_out=(q.X_out.cpu().numpy() if q.X_out is not None
                          else np.zeros((X.shape[0], 0), np.float16)),
                   bitmap=q.bitmap.cpu().numpy().view(np.uint32), flags=q.flags.cpu().numpy(),
                   s_w=w.s_w.cpu().numpy(),
                   W_out=(w.W_out.cpu().numpy() if w.W_out is not None
                          else np.zeros((W.shape[0], 0), np.float16)),
                   status=int(status.item()), packed=w)
        if mode == "w8":
            out["Wq"] = self.unpack_w8(w)
        return out

    def unpack_w8(self, w):
        torch, mq = self.torch, self.mq
        out = torch.empty((w.N, w.K), dtype=torch.int8, device="cuda")
        mq.mixq_debug_unpack_w8(w.N, w.K, w.Wq, out)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def unpack_w4(self, w):
        torch, mq = self.torch, self.mq
        N, K = w.N, w.K
        q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        s2 = torch.empty((N, K // 128), dtype=torch.uint8, device="cuda")
        z2 = torch.empty((N, K // 128), dtype=torch.uint8, device="cuda")
        mq.mixq_debug_unpack_w4(N, K, w.Wq, w.grp, q, s2, z2)
        torch.cuda.synchronize()
        return q.cpu().numpy(), s2.cpu().numpy(), z2.cpu().numpy()

    def acc_i32(self, Xq, w, bn=0, split=0):
        torch, mq = self.torch, self.mq
        M = Xq.shape[0]
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        acc = torch.full((M, w.N), -7, dtype=torch.int32, device="cuda")
        mq.mixq_debug_gemm_i32(w.mode, Xq if isinstance(Xq, torch.Tensor) else self.dev(Xq), w.Wq,
                               w.grp, acc, w.N, bn, split, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        return acc.cpu().numpy()
