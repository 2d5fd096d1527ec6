"""One mixture-of-experts feed-forward layer (forward + backward) on a B200.

Python binding of libmoe (see include/moe.h).  The functions here carry the
C entry points' names and only marshal arguments: PyTorch provides device
memory, streams and output allocation; every step of the layer runs in the
library's sm_100a kernels.  There is no CPU fallback: without the built
library (or without a GPU) the calls raise.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (MOE_BF16, MOE_MXFP8, MOE_EPI_NONE, MOE_EPI_SWIGLU, MOE_EPI_SWIGLU_BWD,  # noqa: F401
                   MOE_ROUTE_GIVEN, MOE_ROUTE_ROUTER, MOE_DEV_BAD_EXPERT, MOE_DEV_DUP_EXPERT,
                   MOE_DEV_TIMEOUT, MOE_DEV_NONFINITE, MoeError, LayerDesc, LayerWeights,
                   LayerGrads, CtxView)

__all__ = ["moe_route", "moe_permute", "moe_permute_mx", "mx_quantize", "mx_quantize_dual", "moe_grouped_gemm_fwd",
           "moe_grouped_gemm_dgrad", "moe_grouped_gemm_wgrad", "moe_grouped_gemm_fwd_gather",
           "moe_grouped_gemm_wgrad_gather", "moe_unpermute_combine",
           "moe_combine_bwd", "moe_combine_bwd_mx", "moe_unpermute_sum", "moe_router_wgrad", "MoELayer",
           "a_pad_max", "MoeError"]


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes device tensors (got a CPU tensor)")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def a_pad_max(T: int, k: int, E: int, align: int = 128) -> int:
    """Host-known bound on the padded permuted row count, rounded to 128."""
    a = T * k + E * (align - 1)
    return (a + 127) // 128 * 128


def _dev(t):
    return t.device


# ---------------------------------------------------------------- routing
def moe_route(x, Wr, bias, k: int, E: int, *, topk_idx=None, gates=None, align: int = 128,
              want_logits: bool = True, status=None, stream=None) -> dict:
    """Router (x, Wr, bias) or given routing (topk_idx, gates) -> routing
    metadata, all on the device.  Returns a dict of tensors."""
    given = topk_idx is not None
    dev = (topk_idx if given else x).device
    T = topk_idx.shape[0] if given else x.shape[0]
    d = 0 if x is None else x.shape[1]
    A = a_pad_max(T, k, E, align)
    i32 = dict(dtype=torch.int32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "topk_idx": topk_idx if given else torch.empty((T, k), **i32),
        "gates": gates if given else torch.empty((T, k), **f32),
        "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
        "poff": torch.empty(E + 1, **i32), "dst": torch.empty((T, k), **i32),
        "src": torch.empty(A, **i32), "A_pad_max": A,
        "logits": torch.empty((T, E), **f32) if (want_logits and not given) else None,
    }
    ws_bytes = _lib.lib().moe_route_workspace_size(T, 0 if given else d, E)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    _lib.call("moe_route", _p(x), _p(Wr), _p(bias), T, d, E, k, align,
              _lib.MOE_ROUTE_GIVEN if given else _lib.MOE_ROUTE_ROUTER,
              _p(out["topk_idx"]), _p(out["gates"]), _p(out["counts"]), _p(out["offsets"]),
              _p(out["poff"]), _p(out["dst"]), _p(out["src"]), A, _p(out["logits"]),
              _p(ws), ws_bytes, _p(status), _s(stream))
    return out


def moe_permute(x, meta: dict, k: int, E: int, *, mx: bool = False, stream=None):
    """Xp[dst[t,j]] = x[t]; pad rows zero.  With mx=True also the MX codes
    and (tensor-core layout) scales of Xp along d."""
    T, d = x.shape
    A = meta["A_pad_max"]
    Xp = torch.empty((A, d), dtype=torch.bfloat16, device=x.device)
    Xq = torch.empty((A, d), dtype=torch.uint8, device=x.device) if mx else None
    Xs = torch.empty(A * d // 32, dtype=torch.uint8, device=x.device) if mx else None
    _lib.call("moe_permute", _p(x), _p(meta["dst"]), _p(meta["offsets"]), _p(meta["poff"]), T, k,
              d, E, A, _p(Xp), _p(Xq), _p(Xs), _s(stream))
    return (Xp, Xq, Xs) if mx else Xp


def moe_permute_mx(x, meta: dict, E: int, *, stream=None):
    """Dispatch straight into MX codes: returns (codes, scales) of the
    permuted rows along d and (codes, scales) down the rows."""
    T, d = x.shape
    A = meta["A_pad_max"]
    mk = lambda *s: torch.empty(s, dtype=torch.uint8, device=x.device)  # noqa: E731
    q, qs, qT, qTs = mk(A, d), mk(A * d // 32), mk(A, d), mk(A * d // 32)
    _lib.call("moe_permute_mx", _p(x), _p(meta["src"]), _p(meta["poff"]), T, d, E, A, _p(q),
              _p(qs), _p(qT), _p(qTs), _s(stream))
    return (q, qs), (qT, qTs)


def moe_combine_bwd_mx(dout, gates, meta: dict, E: int, *, stream=None):
    """dY rows (gate-scaled dout, bf16-rounded) straight into MX codes:
    (codes, scales) along d and (codes, scales) down the rows."""
    T, d = dout.shape
    k = meta["topk_idx"].shape[1]
    A = meta["A_pad_max"]
    mk = lambda *s: torch.empty(s, dtype=torch.uint8, device=dout.device)  # noqa: E731
    q, qs, qT, qTs = mk(A, d), mk(A * d // 32), mk(A, d), mk(A * d // 32)
    _lib.call("moe_combine_bwd_mx", _p(dout), _p(gates), _p(meta["topk_idx"]), _p(meta["src"]),
              _p(meta["poff"]), T, k, d, E, A, _p(q), _p(qs), _p(qT), _p(qTs), _s(stream))
    return (q, qs), (qT, qTs)


def mx_quantize(t, axis: int, *, nrows=None, codes=None, scales=None, stream=None):
    """MX codes [R, C] and scales (R*C/32 bytes, tensor-core layout) of a
    bf16 [R, C] tensor, blocks along a row (axis 0) or down a column (axis 1)."""
    R, C = t.shape
    codes = torch.empty((R, C), dtype=torch.uint8, device=t.device) if codes is None else codes
    scales = torch.empty(R * C // 32, dtype=torch.uint8, device=t.device) if scales is None else scales
    _lib.call("mx_quantize", _p(t), R, C, axis, None, 0, _p(nrows), _p(codes), _p(scales),
              _s(stream))
    return codes, scales


def mx_quantize_dual(t, *, nrows=None, stream=None):
    """Both MX quantisations of a bf16 [R, C] tensor in one pass:
    (codes, scales) along rows (axis 0) and (codes, scales) down columns."""
    R, C = t.shape
    mk = lambda *s: torch.empty(s, dtype=torch.uint8, device=t.device)
    cr, sr, cc, sc = mk(R, C), mk(R * C // 32), mk(R, C), mk(R * C // 32)
    _lib.call("mx_quantize_dual", _p(t), R, C, _p(nrows), _p(cr), _p(sr), _p(cc), _p(sc),
              _s(stream))
    return (cr, sr), (cc, sc)


# ------------------------------------------------------------ grouped GEMM
def moe_grouped_gemm_fwd(A, B, poff, E: int, *, epilogue=MOE_EPI_NONE, B3=None, A_sc=None,
                         B_sc=None, B3_sc=None, want_aux=True, status=None, stream=None):
    """Rows of group e: C = A B[e] (EPI_NONE) or silu(A B[e]) * (A B3[e])
    (EPI_SWIGLU, also returns aux = [A B | A B3]).  MX when scales are given."""
    mx = A_sc is not None
    Ap, K = A.shape
    N = B.shape[2]
    C = torch.empty((Ap, N), dtype=torch.bfloat16, device=A.device)
    aux = None
    if epilogue == MOE_EPI_SWIGLU and want_aux:
        aux = torch.empty((Ap, 2 * N), dtype=torch.bfloat16, device=A.device)
    _lib.call("moe_grouped_gemm_fwd", MOE_MXFP8 if mx else MOE_BF16, _p(A), _p(A_sc), _p(B),
              _p(B_sc), _p(B3), _p(B3_sc), _p(poff), E, Ap, N, K, epilogue, _p(C), _p(aux),
              _p(status), _s(stream))
    return (C, aux) if epilogue == MOE_EPI_SWIGLU else C


def moe_grouped_gemm_dgrad(dC, B, poff, E: int, *, epilogue=MOE_EPI_NONE, B3=None, aux=None,
                           dC_sc=None, B_sc=None, B3_sc=None, status=None, stream=None):
    """dA = dC B[e]^T (+ dC[:, N:] B3[e]^T), or the SwiGLU-backward epilogue."""
    mx = dC_sc is not None
    Ap = dC.shape[0]
    K, N = B.shape[1], B.shape[2]
    cols = 2 * K if epilogue == MOE_EPI_SWIGLU_BWD else K
    dA = torch.empty((Ap, cols), dtype=torch.bfloat16, device=dC.device)
    _lib.call("moe_grouped_gemm_dgrad", MOE_MXFP8 if mx else MOE_BF16, _p(dC), _p(dC_sc), _p(B),
              _p(B_sc), _p(B3), _p(B3_sc), _p(poff), E, Ap, N, K, epilogue, _p(aux), _p(dA),
              _p(status), _s(stream))
    return dA


def moe_grouped_gemm_wgrad(A, dC, poff, E: int, *, split: bool = False, A_sc=None, dC_sc=None,
                           status=None, stream=None):
    """dB[e] = A_e^T dC_e over the rows of group e (two outputs when split)."""
    mx = A_sc is not None
    Ap, K = A.shape
    N = dC.shape[1] // (2 if split else 1)
    dB = torch.empty((E, K, N), dtype=torch.bfloat16, device=A.device)
    dB3 = torch.empty((E, K, N), dtype=torch.bfloat16, device=A.device) if split else None
    _lib.call("moe_grouped_gemm_wgrad", MOE_MXFP8 if mx else MOE_BF16, _p(A), _p(A_sc), _p(dC),
              _p(dC_sc), _p(poff), E, Ap, K, N, _p(dB), _p(dB3), _p(status), _s(stream))
    return (dB, dB3) if split else dB


def moe_grouped_gemm_fwd_gather(x, src, B, poff, E: int, A_pad_max: int, *,
                                epilogue=MOE_EPI_NONE, B3=None, want_aux=True, status=None,
                                stream=None):
    """moe_grouped_gemm_fwd (BF16) with row r of A read as x[src[r]] (zero
    for src[r] < 0): the dispatch fused into the GEMM's loads."""
    T, K = x.shape
    N = B.shape[2]
    C = torch.empty((A_pad_max, N), dtype=torch.bfloat16, device=x.device)
    aux = None
    if epilogue == MOE_EPI_SWIGLU and want_aux:
        aux = torch.empty((A_pad_max, 2 * N), dtype=torch.bfloat16, device=x.device)
    _lib.call("moe_grouped_gemm_fwd_gather", _p(x), T, _p(src), _p(B), _p(B3), _p(poff), E,
              A_pad_max, N, K, epilogue, _p(C), _p(aux), _p(status), _s(stream))
    return (C, aux) if epilogue == MOE_EPI_SWIGLU else C


def moe_grouped_gemm_fwd_swiglu_mxq(A, A_sc, B, B_sc, B3, B3_sc, poff, E: int, *, status=None,
                                    stream=None):
    """MXFP8 GEMM1 + SwiGLU whose h leaves as MX codes: returns aux = [H1 |
    H3] bf16 and (h codes, h scales) along F and (codes, scales) down the rows."""
    Ap, K = A.shape
    F = B.shape[2]
    dev = A.device
    aux = torch.empty((Ap, 2 * F), dtype=torch.bfloat16, device=dev)
    mk = lambda *s: torch.empty(s, dtype=torch.uint8, device=dev)  # noqa: E731
    hq, hs, hTq, hTs = mk(Ap, F), mk(Ap * F // 32), mk(Ap, F), mk(Ap * F // 32)
    _lib.call("moe_grouped_gemm_fwd_swiglu_mxq", _p(A), _p(A_sc), _p(B), _p(B_sc), _p(B3),
              _p(B3_sc), _p(poff), E, Ap, F, K, _p(aux), _p(hq), _p(hs), _p(hTq), _p(hTs),
              _p(status), _s(stream))
    return aux, (hq, hs), (hTq, hTs)


def moe_grouped_gemm_dgrad_swiglu_mxq(dC, dC_sc, B, B_sc, aux, poff, E: int, *, status=None,
                                      stream=None):
    """MXFP8 GEMM2 dgrad + SwiGLU backward whose dA = [dA1 | dA3] leaves as MX
    codes: returns (codes, scales) along 2F and (codes, scales) down the rows.
    B: W2 codes [E, F, d] quantised along d."""
    Ap, N = dC.shape
    K = B.shape[1]
    dev = dC.device
    mk = lambda *s: torch.empty(s, dtype=torch.uint8, device=dev)  # noqa: E731
    q, qs, qT, qTs = mk(Ap, 2 * K), mk(Ap * 2 * K // 32), mk(Ap, 2 * K), mk(Ap * 2 * K // 32)
    _lib.call("moe_grouped_gemm_dgrad_swiglu_mxq", _p(dC), _p(dC_sc), _p(B), _p(B_sc), _p(poff),
              E, Ap, N, K, _p(aux), _p(q), _p(qs), _p(qT), _p(qTs), _p(status), _s(stream))
    return (q, qs), (qT, qTs)


def moe_grouped_gemm_wgrad_gather(x, src, dC, poff, E: int, *, offsets=None, split: bool = False,
                                  status=None, stream=None):
    """moe_grouped_gemm_wgrad (BF16) with A row r read as x[src[r]]."""
    T, K = x.shape
    Ap = dC.shape[0]
    N = dC.shape[1] // (2 if split else 1)
    dB = torch.empty((E, K, N), dtype=torch.bfloat16, device=x.device)
    dB3 = torch.empty((E, K, N), dtype=torch.bfloat16, device=x.device) if split else None
    _lib.call("moe_grouped_gemm_wgrad_gather", _p(x), T, _p(src), _p(dC), _p(poff), _p(offsets),
              E, Ap, K, N, _p(dB), _p(dB3), _p(status), _s(stream))
    return (dB, dB3) if split else dB


def moe_grouped_gemm_tn(X, W, poff, E: int, *, epilogue=MOE_EPI_NONE, W3=None,
                        w_kmajor: bool = False, offsets=None, row_scale=None, col_vec=None,
                        status=None, stream=None):
    """Tokens-N grouped GEMM (BF16): only the real rows of each group are
    multiplied (``offsets``), the padding rows of the output are zeros.
    SwiGLU: returns (h, aux); otherwise C."""
    Ap, K = X.shape
    N = W.shape[1] if w_kmajor else W.shape[2]
    C = torch.empty((Ap, N), dtype=torch.bfloat16, device=X.device)
    aux = None
    if epilogue == MOE_EPI_SWIGLU:
        aux = torch.empty((Ap, 2 * N), dtype=torch.bfloat16, device=X.device)
    _lib.call("moe_grouped_gemm_tn", epilogue, _p(X), _p(W), _p(W3), 1 if w_kmajor else 0,
              _p(poff), _p(offsets), E, Ap, N, K, _p(C), _p(aux), _p(row_scale), _p(col_vec),
              _p(status), _s(stream))
    return (C, aux) if epilogue == MOE_EPI_SWIGLU else C


# ---------------------------------------------------- combine and backward
def moe_unpermute_combine(Y, gates, dst, *, stream=None):
    T, k = dst.shape
    d = Y.shape[1]
    out = torch.empty((T, d), dtype=torch.bfloat16, device=Y.device)
    _lib.call("moe_unpermute_combine", _p(Y), _p(gates), _p(dst), T, k, d, _p(out), _s(stream))
    return out


def moe_combine_bwd(dout, Y, gates, meta: dict, E: int, *, router: bool = True, stream=None):
    T, k = meta["dst"].shape
    d = dout.shape[1]
    dev = dout.device
    dY = torch.empty_like(Y)
    dg = torch.empty((T, k), dtype=torch.float32, device=dev)
    dl = torch.empty((T, k), dtype=torch.float32, device=dev) if router else None
    dl_rows = torch.zeros(Y.shape[0], dtype=torch.float32, device=dev) if router else None
    _lib.call("moe_combine_bwd", _p(dout), _p(Y), _p(gates), _p(meta["dst"]), _p(meta["offsets"]),
              _p(meta["poff"]), T, k, d, E, _p(dY), _p(dg), _p(dl), _p(dl_rows), _s(stream))
    return dY, dg, dl, dl_rows


def moe_unpermute_sum(dXp, dst, *, topk_idx=None, dl=None, Wr=None, E: int = 0, stream=None):
    T, k = dst.shape
    d = dXp.shape[1]
    dx = torch.empty((T, d), dtype=torch.bfloat16, device=dXp.device)
    ws_bytes = _lib.lib().moe_unpermute_sum_workspace_size(d, max(E, 1))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dXp.device) if Wr is not None else None
    _lib.call("moe_unpermute_sum", _p(dXp), _p(dst), _p(topk_idx), _p(dl), _p(Wr), T, k, d,
              max(E, 1), _p(dx), _p(ws), ws_bytes if ws is not None else 0, _s(stream))
    return dx


def moe_router_wgrad(x, meta: dict, dl_rows, E: int, *, stream=None):
    T, d = x.shape
    A = meta["A_pad_max"]
    dWr = torch.empty((d, E), dtype=torch.float32, device=x.device)
    ws_bytes = _lib.lib().moe_router_wgrad_workspace_size(d, A)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    _lib.call("moe_router_wgrad", _p(x), _p(meta["src"]), _p(dl_rows), _p(meta["offsets"]),
              _p(meta["poff"]), T, d, E, A, _p(dWr), _p(ws), ws_bytes, _s(stream))
    return dWr


# ------------------------------------------------------------- the layer
class MoELayer:
    """The whole layer over caller-owned weights, with one context buffer
    that holds everything the backward needs."""

    def __init__(self, *, T, d, E, k, F, W1, W3, W2, Wr=None, bias=None, topk_idx=None,
                 gates=None, mx=False, align=128):
        self.desc = LayerDesc(T, d, E, k, F, align,
                              MOE_ROUTE_GIVEN if topk_idx is not None else MOE_ROUTE_ROUTER,
                              MOE_MXFP8 if mx else MOE_BF16)
        self.cfg = dict(T=T, d=d, E=E, k=k, F=F, mx=mx)
        self._keep = [W1, W3, W2, Wr, bias, topk_idx, gates]
        self.weights = LayerWeights(*[None if t is None else _p(t).value
                                      for t in (Wr, bias, W1, W3, W2, topk_idx, gates)])
        dev = W1.device
        self.ctx_bytes = _lib.lib().moe_layer_ctx_bytes(ctypes.byref(self.desc))
        if self.ctx_bytes == 0:
            raise MoeError("moe_layer_ctx_bytes", _lib.MOE_ERR_INVALID_ARG,
                           "layer description rejected (align 128, d % 256, F % 256, "
                           "k <= min(E,16), router E <= 512)")
        self.ctx = torch.empty(self.ctx_bytes + 256, dtype=torch.uint8, device=dev)
        base = self.ctx.data_ptr()
        self._ctx_ptr = (base + 255) // 256 * 256
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dW1 = torch.empty_like(W1)
        self.dW3 = torch.empty_like(W3)
        self.dW2 = torch.empty_like(W2)
        self.dWr = torch.empty((d, E), dtype=torch.float32, device=dev) if Wr is not None else None
        self.grads = LayerGrads(_p(self.dW1).value, _p(self.dW3).value, _p(self.dW2).value,
                                None if self.dWr is None else _p(self.dWr).value)

    def view(self) -> CtxView:
        v = CtxView()
        _lib.call("moe_layer_ctx_view", ctypes.byref(self.desc), ctypes.c_void_p(self._ctx_ptr),
                  ctypes.byref(v))
        return v

    def forward(self, x, out=None, stream=None):
        out = torch.empty_like(x) if out is None else out
        _lib.call("moe_layer_fwd", ctypes.byref(self.desc), ctypes.byref(self.weights), _p(x),
                  _p(out), ctypes.c_void_p(self._ctx_ptr), self.ctx_bytes, _p(self.status),
                  _s(stream))
        return out

    def backward(self, x, dout, dx=None, stream=None):
        dx = torch.empty_like(dout) if dx is None else dx
        _lib.call("moe_layer_bwd", ctypes.byref(self.desc), ctypes.byref(self.weights), _p(x),
                  ctypes.c_void_p(self._ctx_ptr), self.ctx_bytes, _p(dout), _p(dx),
                  ctypes.byref(self.grads), _p(self.status), _s(stream))
        return dx

    def step_host(self, x_host, dout_host, out_host, dx_host, x_dev, dout_dev, out_dev, dx_dev,
                  stream=None):
        """fwd + bwd from host buffers (copies inside the call; the host
        outputs are complete after step_host_sync and a stream sync)."""
        hp = lambda t: ctypes.c_void_p(t.data_ptr())
        _lib.call("moe_layer_step_host", ctypes.byref(self.desc), ctypes.byref(self.weights),
                  hp(x_host), hp(dout_host), hp(out_host), hp(dx_host), _p(x_dev), _p(dout_dev),
                  _p(out_dev), _p(dx_dev), ctypes.c_void_p(self._ctx_ptr), self.ctx_bytes,
                  ctypes.byref(self.grads), _p(self.status), _s(stream))

    @staticmethod
    def step_host_sync(stream=None):
        """Orders `stream` after every download step_host has queued on the
        current device; synchronise the stream afterwards to read the host
        outputs."""
        _lib.call("moe_layer_step_host_sync", _s(stream))

    def ctx_tensor(self, name: str, shape, dtype) -> torch.Tensor:
        """A view of one saved buffer of the context (for inspection)."""
        v = self.view()
        ptr = getattr(v, name)
        if not ptr:
            raise KeyError(name)
        off = ptr - self.ctx.data_ptr()
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        return self.ctx[off:off + nbytes].view(dtype).view(*shape)
