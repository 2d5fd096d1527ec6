"""moe_route_noalloc: routing for callers that cannot allocate device memory
while they run (a pooling allocator owns the device memory, or a
latency-critical loop must not call cudaMalloc).  Its scratch is a fixed
array the library keeps in device memory, shared by every call.  The test
makes two calls in a row on different inputs (the second smaller, so scratch
left over from the first would show) and compares each with the ordinary
moe_route (caller workspace) on the same input, through the C ABI.  It is
collected last, needs nothing from other test files, and runs alone or after
them."""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("mixture_experts_layer_25_b200")
from mixture_experts_layer_25_b200 import _lib  # noqa: E402


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _case(mode, call):
    """Input of the call-th call: a different size and different data."""
    if mode == "router":
        T, d, E, k = (4096, 2048, 128, 4) if call == 0 else (1000, 2048, 128, 4)
        x = moe_inputs.random_bf16((T, d), 21 + 10 * call, device="cuda")
        g = torch.Generator(device="cuda"); g.manual_seed(22 + 10 * call)
        Wr = torch.randn((d, E), generator=g, device="cuda") * 0.02
        return dict(T=T, d=d, E=E, k=k, x=x, Wr=Wr, topk=None, gates=None)
    T, E, k = (8192, 384, 8) if call == 0 else (3000, 384, 8)
    idx, gates = moe_inputs.random_routing(T, E, k, 23 + 10 * call)
    return dict(T=T, d=0, E=E, k=k, x=None, Wr=None, topk=torch.from_numpy(idx).cuda(),
                gates=torch.from_numpy(gates).cuda())


def _fresh_outputs(c):
    T, E, k = c["T"], c["E"], c["k"]
    A = moe.a_pad_max(T, k, E)
    i32 = lambda *s: torch.full(s, -7, dtype=torch.int32, device="cuda")
    o = dict(counts=i32(E), offsets=i32(E + 1), poff=i32(E + 1), dst=i32(T, k), src=i32(A), A=A)
    if c["topk"] is None:
        o["topk_idx"] = i32(T, k)
        o["gates"] = torch.full((T, k), -7.0, device="cuda")
        o["logits"] = torch.full((T, E), -7.0, device="cuda")
    else:
        o["topk_idx"], o["gates"], o["logits"] = c["topk"], c["gates"], None
    return o


@pytest.mark.parametrize("mode", ["router", "given"])
def test_noalloc_route_matches_route_on_two_calls(mode):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        c = _case(mode, call)
        ref = moe.moe_route(c["x"], c["Wr"], None, c["k"], c["E"], topk_idx=c["topk"],
                            gates=c["gates"])
        torch.cuda.synchronize()
        o = _fresh_outputs(c)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        _lib.call("moe_route_noalloc", _p(c["x"]), _p(c["Wr"]), None, c["T"], c["d"], c["E"],
                  c["k"], 128, _lib.MOE_ROUTE_ROUTER if mode == "router" else _lib.MOE_ROUTE_GIVEN,
                  _p(o["topk_idx"]), _p(o["gates"]), _p(o["counts"]), _p(o["offsets"]),
                  _p(o["poff"]), _p(o["dst"]), _p(o["src"]), o["A"], _p(o["logits"]), _p(st),
                  stream)
        torch.cuda.synchronize()
        assert st.item() == 0
        for n in ("topk_idx", "counts", "offsets", "poff", "dst", "src"):
            assert torch.equal(o[n], ref[n]), n
        if mode == "router":
            for n in ("gates", "logits"):
                a, b = o[n].double().cpu().numpy(), ref[n].double().cpu().numpy()
                assert np.max(np.abs(a - b)) / np.max(np.abs(b)) < 1e-5, n


def test_noalloc_route_rejects_problems_beyond_its_fixed_scratch():
    E = 128
    T = (4 << 20) // (E * 4) * 32 + 32         # given routing: one 32-token block too many
    assert _lib.lib().moe_route_workspace_size(T, 0, E) > (4 << 20)
    code = _lib.lib().moe_route_noalloc(None, None, None, T, 0, E, 4, 128, 1, None, None,
                                        None, None, None, None, None, 0, None, None, None)
    assert code == _lib.MOE_ERR_INVALID_ARG
    assert b"fixed array" in _lib.lib().moe_last_error()
