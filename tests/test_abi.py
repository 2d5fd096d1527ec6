"""The C-ABI library loads on a CPU-only host and exports every symbol the
header declares; host-only size queries work without a GPU."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_25_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^MOE_API [^(]*?\b((?:moe|mx)_\w+)\(", src, re.M)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_layer_25_b200 import build
    build.build()


def test_header_declares_the_call_list():
    names = _declared()
    for n in ("moe_route", "moe_permute", "mx_quantize", "moe_grouped_gemm_fwd",
              "moe_grouped_gemm_dgrad", "moe_grouped_gemm_wgrad", "moe_unpermute_combine",
              "moe_layer_fwd", "moe_layer_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) == set(_lib.exported_names())


def test_host_size_queries():
    lib = _lib.lib()
    # given routing (d = 0): 32-token block histograms
    assert lib.moe_route_workspace_size(16384, 0, 128) == 512 * 128 * 4
    # tensor-core router: 128-token block histograms + W_r split in 2 bf16 parts
    assert lib.moe_route_workspace_size(16384, 2048, 128) == 128 * 128 * 4 + 2 * 2048 * 128 * 2
    assert lib.moe_route_workspace_size(0, 2048, 128) == 0
    assert lib.moe_unpermute_sum_workspace_size(2048, 128) == 2048 * 128 * 4
    d = _lib.LayerDesc(16384, 2048, 128, 4, 1024, 128, 0, 0)
    n = lib.moe_layer_ctx_bytes(ctypes.byref(d))
    A = 16384 * 4 + 128 * 127
    assert n > A * 2048 * 2 * 4          # Xp, Y, dY + H13/h/dA13
    d.dtype = 1
    assert lib.moe_layer_ctx_bytes(ctypes.byref(d)) > n
    for bad in (dict(align=64), dict(d=2000), dict(k=0), dict(E=2000), dict(F=100)):
        b = _lib.LayerDesc(16384, 2048, 128, 4, 1024, 128, 0, 0)
        for kk, v in bad.items():
            setattr(b, kk, v)
        assert lib.moe_layer_ctx_bytes(ctypes.byref(b)) == 0


def test_version_and_error_string():
    lib = _lib.lib()
    assert b"sm_100a" in lib.moe_version()
    assert isinstance(lib.moe_last_error(), bytes)


def test_argument_errors_need_no_gpu():
    # argument validation happens on the host before anything is enqueued
    lib = _lib.lib()
    code = lib.moe_route(None, None, None, 0, 0, 0, 0, 128, 0, None, None, None, None, None,
                         None, None, 0, None, None, 0, None, None)
    assert code == _lib.MOE_ERR_INVALID_ARG
    assert b"bad T/E/k" in lib.moe_last_error()
    code = lib.mx_quantize(None, 100, 128, 0, None, 0, None, None, None, None)
    assert code == _lib.MOE_ERR_INVALID_ARG


def test_grouped_gemm_argument_errors_need_no_gpu():
    lib = _lib.lib()
    fake = ctypes.c_void_p(256)     # never dereferenced: the checks fail first
    # E out of range
    assert lib.moe_grouped_gemm_tn(0, fake, fake, None, 0, fake, None, 0, 128, 128, 64, fake,
                                   None, None, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    # K not a multiple of 64
    assert lib.moe_grouped_gemm_tn(0, fake, fake, None, 0, fake, None, 4, 128, 128, 100, fake,
                                   None, None, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    # SwiGLU without W3 / aux
    assert lib.moe_grouped_gemm_tn(1, fake, fake, None, 0, fake, None, 4, 128, 128, 64, fake,
                                   None, None, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    # a rank-1 term needs both vectors
    assert lib.moe_grouped_gemm_tn(0, fake, fake, None, 1, fake, None, 4, 128, 128, 64, fake,
                                   None, fake, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    # A_pad_max not a multiple of 128
    assert lib.moe_grouped_gemm_fwd(0, fake, None, fake, None, None, None, fake, 4, 100, 256, 64,
                                    0, fake, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_gemm_wgrad(0, fake, None, fake, None, fake, 4, 128, 100, 256, fake,
                                      None, None, None) == _lib.MOE_ERR_INVALID_ARG
