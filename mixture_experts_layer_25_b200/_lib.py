"""ctypes loader of libmoe.so: raw C entry points and the C structs.

Argument marshalling only; every step of the layer runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB_PATH may name another build of the same library (e.g. a variant
# compiled with different tuning constants)
LIB_PATH = os.environ.get("MOE_LIB_PATH") or os.path.join(_HERE, "libmoe.so")

P = ctypes.c_void_p
I = ctypes.c_int
Z = ctypes.c_size_t

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = 0, 1, 2, 3, 4
MOE_DEV_BAD_EXPERT, MOE_DEV_DUP_EXPERT, MOE_DEV_TIMEOUT, MOE_DEV_NONFINITE = 1, 2, 4, 8
MOE_ROUTE_ROUTER, MOE_ROUTE_GIVEN = 0, 1
MOE_BF16, MOE_MXFP8 = 0, 1
MOE_EPI_NONE, MOE_EPI_SWIGLU, MOE_EPI_SWIGLU_BWD = 0, 1, 2


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


class LayerDesc(ctypes.Structure):
    _fields_ = [(n, I) for n in ("T", "d", "E", "k", "F", "align", "route_mode", "dtype")]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, P) for n in ("Wr", "bias", "W1", "W3", "W2", "topk_idx", "gates")]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, P) for n in ("dW1", "dW3", "dW2", "dWr")]


CTX_PTRS = ["topk_idx", "counts", "offsets", "poff", "dst", "src",
            "gates", "logits", "dg", "dl", "dl_rows",
            "Xp", "H13", "h", "Y", "dY", "dA13", "dXp",
            "Xp_q", "Xp_s", "W13_q", "W13_s", "W2_q", "W2_s", "h_q", "h_s",
            "dY_q", "dY_s", "W13t_q", "W13t_s", "W2t_q", "W2t_s", "dA_q", "dA_s",
            "hT_q", "hT_s", "dYT_q", "dYT_s", "XpT_q", "XpT_s", "dAT_q", "dAT_s"]


class CtxView(ctypes.Structure):
    _fields_ = [(n, P) for n in CTX_PTRS] + [("ws", P), ("ws_bytes", Z), ("A_pad_max", I)]


_SIGS = {
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_version": (ctypes.c_char_p, []),
    "moe_launch_count": (ctypes.c_ulonglong, []),
    "moe_set_stage_events": (None, [ctypes.POINTER(P), I]),
    "moe_route_workspace_size": (Z, [I, I, I]),
    "moe_route": (I, [P, P, P, I, I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, Z, P, P]),
    "moe_route_noalloc": (I, [P, P, P, I, I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P]),
    "moe_permute": (I, [P, P, P, P, I, I, I, I, I, P, P, P, P]),
    "mx_quantize": (I, [P, I, I, I, P, I, P, P, P, P]),
    "mx_quantize_dual": (I, [P, I, I, P, P, P, P, P, P]),
    "moe_grouped_gemm_fwd": (I, [I, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P]),
    "moe_grouped_gemm_dgrad": (I, [I, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P]),
    "moe_grouped_gemm_wgrad": (I, [I, P, P, P, P, P, I, I, I, I, P, P, P, P]),
    "moe_grouped_gemm_tn": (I, [I, P, P, P, I, P, P, I, I, I, I, P, P, P, P, P, P]),
    "moe_grouped_gemm_fwd_gather": (I, [P, I, P, P, P, P, I, I, I, I, I, P, P, P, P]),
    "moe_permute_mx": (I, [P, P, P, I, I, I, I, P, P, P, P, P]),
    "moe_combine_bwd_mx": (I, [P, P, P, P, P, I, I, I, I, I, P, P, P, P, P]),
    "moe_grouped_gemm_fwd_swiglu_mxq": (I, [P, P, P, P, P, P, P, I, I, I, I, P, P, P, P, P, P, P]),
    "moe_grouped_gemm_dgrad_swiglu_mxq": (I, [P, P, P, P, P, I, I, I, I, P, P, P, P, P, P, P]),
    "moe_grouped_gemm_wgrad_gather": (I, [P, I, P, P, P, P, I, I, I, I, P, P, P, P]),
    "moe_selftest_wait_timeout": (I, [P, ctypes.c_uint64, P]),
    "moe_unpermute_combine": (I, [P, P, P, I, I, I, P, P]),
    "moe_combine_bwd": (I, [P, P, P, P, P, P, I, I, I, I, P, P, P, P, P]),
    "moe_unpermute_sum_workspace_size": (Z, [I, I]),
    "moe_unpermute_sum": (I, [P, P, P, P, P, I, I, I, I, P, P, Z, P]),
    "moe_router_wgrad_workspace_size": (Z, [I, I]),
    "moe_router_wgrad": (I, [P, P, P, P, P, I, I, I, I, P, P, Z, P]),
    "moe_layer_ctx_bytes": (Z, [ctypes.POINTER(LayerDesc)]),
    "moe_layer_ctx_view": (I, [ctypes.POINTER(LayerDesc), P, ctypes.POINTER(CtxView)]),
    "moe_layer_fwd": (I, [ctypes.POINTER(LayerDesc), ctypes.POINTER(LayerWeights), P, P, P, Z, P, P]),
    "moe_layer_bwd": (I, [ctypes.POINTER(LayerDesc), ctypes.POINTER(LayerWeights), P, P, Z, P, P,
                          ctypes.POINTER(LayerGrads), P, P]),
    "moe_layer_step_host": (I, [ctypes.POINTER(LayerDesc), ctypes.POINTER(LayerWeights), P, P, P, P,
                                P, P, P, P, P, Z, ctypes.POINTER(LayerGrads), P, P]),
    "moe_layer_step_host_sync": (I, [P]),
}

_lib = None


def lib():
    """The loaded library (built in-tree by ``python -m mixture_experts_layer_25_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixture_experts_layer_25_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def call(name: str, *args) -> None:
    """Call a status-returning entry point; raise MoeError on failure."""
    code = getattr(lib(), name)(*args)
    if code != MOE_OK:
        raise MoeError(name, code, lib().moe_last_error().decode())


STAGES = ["route", "permute", "quant_w_fwd", "gemm1_swiglu", "quant_h", "gemm2", "combine",
          "combine_bwd", "quant_dgrad2", "gemm2_dgrad_swiglu_bwd", "quant_wgrad2", "gemm2_wgrad",
          "quant_dgrad1", "gemm1_dgrad", "quant_wgrad1", "gemm1_wgrad", "unpermute_sum",
          "router_wgrad"]


def exported_names() -> list[str]:
    return list(_SIGS)
