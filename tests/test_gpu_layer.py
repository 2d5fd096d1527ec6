"""GPU parity of the whole layer (moe_layer_fwd + moe_layer_bwd through the C
ABI) against the oracle: the tiny layer element by element; the full-size
layers on sampled tokens and experts.

Routing reading: the device computes logits in fp32.  The strict check runs
the oracle's routing on the device's logits (bit-exact metadata); the
full-size checks use the oracle's own fp64 routing and skip the rare
near-tie tokens, whose choice may legitimately differ."""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from gpu_util import f64, np_i, rel_err

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("mixture_experts_layer_25_b200")


def _layer(cfg, inp):
    return moe.MoELayer(T=cfg.T, d=cfg.d, E=cfg.E, k=cfg.k, F=cfg.F, W1=inp["W1"], W3=inp["W3"],
                        W2=inp["W2"], Wr=inp["Wr"] if cfg.routing == "router" else None,
                        bias=inp["bias"], topk_idx=inp.get("topk_idx"), gates=inp.get("gates"),
                        mx=cfg.mx)


def _run(cfg, inp):
    L = _layer(cfg, inp)
    out = L.forward(inp["x"])
    dx = L.backward(inp["x"], inp["dout"])
    torch.cuda.synchronize()
    assert L.status.item() == 0
    return L, out, dx


@pytest.mark.parametrize("variant", ["bf16", "mx", "given", "skewed", "one_token", "ragged",
                                     "k_equals_E", "single_expert", "mx_ragged", "many_experts"])
def test_tiny_layer_element_by_element(variant):
    cfg = moe_inputs.CONFIGS["tiny"]
    if variant == "many_experts":
        # the largest expert count the layer's router takes (512): the SIMT
        # router, most groups empty or with a few rows, the tokens-N GEMMs
        cfg = cfg.with_(T=512, E=512, k=4, F=256)
    if variant == "one_token":
        cfg = cfg.with_(T=1)
    if variant in ("ragged", "mx_ragged"):
        cfg = cfg.with_(T=333, mx=variant == "mx_ragged")
    if variant == "k_equals_E":
        cfg = cfg.with_(T=200, k=8)
    if variant == "single_expert":
        cfg = cfg.with_(T=100, E=1, k=1)
    if variant == "mx":
        cfg = cfg.with_(mx=True)
    if variant == "given":
        cfg = cfg.with_(routing="random")
    if variant == "skewed":
        cfg = cfg.with_(bias="zipf", E=8)
    inp = moe_inputs.make_layer_inputs(cfg, "cuda")
    L, out, dx = _run(cfg, inp)
    T, E, k = cfg.T, cfg.E, cfg.k
    W = [f64(inp[n]) for n in ("W1", "W3", "W2")]
    if cfg.routing == "router":
        logits = L.ctx_tensor("logits", (T, E), torch.float32)
        ctx = oracle.layer_forward(f64(inp["x"]), *W, k, Wr=f64(inp["Wr"]),
                                   bias=moe_inputs.to_f64(inp["bias"]), logits=f64(logits),
                                   mx=cfg.mx)
    else:
        ctx = oracle.layer_forward(f64(inp["x"]), *W, k, topk_idx=np_i(inp["topk_idx"]),
                                   gates=f64(inp["gates"]), mx=cfg.mx)
    g = oracle.layer_backward(ctx, f64(inp["dout"]))
    # routing metadata bit-exact
    np.testing.assert_array_equal(np_i(L.ctx_tensor("topk_idx", (T, k), torch.int32)), ctx["topk_idx"])
    np.testing.assert_array_equal(np_i(L.ctx_tensor("dst", (T, k), torch.int32)), ctx["meta"]["dst"])
    np.testing.assert_array_equal(np_i(L.ctx_tensor("poff", (E + 1,), torch.int32)), ctx["meta"]["poff"])
    tol = 3e-2 if cfg.mx else 1e-2
    errs = {
        "out": rel_err(f64(out), ctx["out"]),
        "dx": rel_err(f64(dx), g["dx"]),
        "dW1": rel_err(f64(L.dW1), g["dW1"]),
        "dW3": rel_err(f64(L.dW3), g["dW3"]),
        "dW2": rel_err(f64(L.dW2), g["dW2"]),
    }
    if cfg.routing == "router":
        errs["dWr"] = rel_err(L.dWr.cpu().numpy(), g["dWr"])
    print(variant, {n: f"{e:.2e}" for n, e in errs.items()})
    bad = {n: e for n, e in errs.items() if not e < tol}
    assert not bad, errs


def _oracle_on_tokens(cfg, inp, cache, toks, only_expert=None):
    """Oracle fwd + bwd of the sub-batch `toks` (each token's result does not
    depend on the other tokens), over the experts these tokens choose.  With
    given routing and `only_expert`, each token keeps just its assignment to
    that expert: the expert's weight gradients depend on nothing else."""
    x = f64(inp["x"][toks]); dout = f64(inp["dout"][toks])
    if only_expert is not None and cfg.routing != "router":
        idx = np_i(inp["topk_idx"][toks]); gg = f64(inp["gates"][toks])
        slot = np.argmax(idx == only_expert, axis=1)
        S = np.array([only_expert])
        Ws = [cache["W"](n, S) for n in ("W1", "W3", "W2")]
        ctx = oracle.layer_forward(x, *Ws, 1, topk_idx=np.zeros((len(toks), 1), np.int32),
                                   gates=gg[np.arange(len(toks)), slot][:, None], mx=cfg.mx)
        return ctx, oracle.layer_backward(ctx, dout), S, {only_expert: 0}
    if cfg.routing == "router":
        Wr, b = cache["Wr"], cache["b"]
        idx = oracle.topk_select(oracle.router_logits(x, Wr, b), cfg.k)
    else:
        idx = np_i(inp["topk_idx"][toks]); g = f64(inp["gates"][toks])
    S = np.unique(idx)
    pos = {int(e): i for i, e in enumerate(S)}
    Ws = [cache["W"](n, S) for n in ("W1", "W3", "W2")]
    if cfg.routing == "router":
        ctx = oracle.layer_forward(x, *Ws, cfg.k, Wr=Wr[:, S], bias=None if b is None else b[S],
                                   mx=cfg.mx)
    else:
        ci = np.vectorize(pos.get)(idx).astype(np.int32)
        ctx = oracle.layer_forward(x, *Ws, cfg.k, topk_idx=ci, gates=g, mx=cfg.mx)
    return ctx, oracle.layer_backward(ctx, dout), S, pos


@pytest.mark.parametrize("name", ["olmo128", "olmo128_mx", "skewed", "trillion", "trillion_mx"])
def test_full_size_layer_sampled(name):
    cfg = moe_inputs.CONFIGS[name]
    inp = moe_inputs.make_layer_inputs(cfg, "cuda")
    L, out, dx = _run(cfg, inp)
    T, E, k = cfg.T, cfg.E, cfg.k
    cache = {"Wr": f64(inp["Wr"]), "b": moe_inputs.to_f64(inp["bias"])}
    wcache = {}

    def W(n, S):
        key = (n, tuple(S.tolist()))
        if key not in wcache:
            wcache.clear()
            wcache[key] = inp[n][torch.from_numpy(S).cuda()].to(torch.float64).cpu().numpy()
        return wcache[key]
    cache["W"] = W
    tol = 3e-2 if cfg.mx else 1e-2
    topk = np_i(L.ctx_tensor("topk_idx", (T, k), torch.int32))
    # routing metadata bit-exact against the oracle's counting sort
    meta = oracle.routing_metadata(topk, E, 128)
    np.testing.assert_array_equal(np_i(L.ctx_tensor("dst", (T, k), torch.int32)), meta["dst"])
    np.testing.assert_array_equal(np_i(L.ctx_tensor("counts", (E,), torch.int32)), meta["counts"])
    # sampled tokens: out and dx rows
    rng = np.random.default_rng(cfg.index)
    # the oracle holds the fp64 weights of every expert the sampled tokens
    # use (about 0.3 GB each at d = 6144, and MX quantises each along both K)
    n_tok = 24 if cfg.d <= 2048 else (2 if cfg.mx else 3)
    toks = np.sort(rng.choice(T, n_tok, replace=False))
    ctx, g, S, pos = _oracle_on_tokens(cfg, inp, cache, toks)
    same = np.all(S[ctx["topk_idx"]] == topk[toks], axis=1)
    assert same.sum() >= len(toks) - 1           # at most a near-tie
    assert rel_err(f64(out[toks])[same], ctx["out"][same]) < tol
    assert rel_err(f64(dx[toks])[same], g["dx"][same]) < tol
    # sampled experts: every weight gradient of the expert (and its router column)
    counts = meta["counts"]
    cand = [e for e in np.argsort(-counts)[:3].tolist() + [int(rng.integers(E))] if counts[e] > 0]
    for e in cand[:2]:
        grp = meta["src"][meta["poff"][e]:meta["poff"][e] + counts[e]]
        ctx, g, S, pos = _oracle_on_tokens(cfg, inp, cache, grp, only_expert=e)
        if cfg.routing == "router" and not np.all(S[ctx["topk_idx"]] == topk[grp]):
            continue                             # a near-tie token in the group
        i = pos[e]
        assert rel_err(f64(L.dW1[e]), g["dW1"][i]) < tol, ("dW1", e)
        assert rel_err(f64(L.dW3[e]), g["dW3"][i]) < tol, ("dW3", e)
        assert rel_err(f64(L.dW2[e]), g["dW2"][i]) < tol, ("dW2", e)
        if cfg.routing == "router":
            assert rel_err(L.dWr[:, e].cpu().numpy(), g["dWr"][:, i]) < tol, ("dWr", e)


def test_host_buffer_step_matches_device_step():
    cfg = moe_inputs.CONFIGS["tiny"]
    inp = moe_inputs.make_layer_inputs(cfg, "cuda")
    L, out, dx = _run(cfg, inp)
    xh = inp["x"].cpu().pin_memory(); dh = inp["dout"].cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory(); dxh = torch.empty_like(xh).pin_memory()
    bufs = [torch.empty_like(inp["x"]) for _ in range(4)]
    L.step_host(xh, dh, oh, dxh, *bufs)
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu()) and torch.equal(dxh, dx.cpu())


@pytest.mark.gpu
@pytest.mark.parametrize("mx", [False, True])
def test_host_buffer_steps_back_to_back(mx):
    """Four host-buffer steps queued without a host sync, on three different
    inputs and two alternating sets of device buffers (each step's uploads
    may run under the previous step's backward, its forward under the
    previous step's downloads): after step_host_sync and a synchronisation
    of the stream alone, every step's out and dx, and the last step's
    weight gradients, equal the device-resident step on the same input."""
    cfg = moe_inputs.CONFIGS["olmo128"].with_(T=4096, mx=mx)
    inp = moe_inputs.make_layer_inputs(cfg, "cuda")
    xs = [torch.roll(inp["x"], 37 * i, 0).contiguous() for i in range(3)]
    ds = [torch.roll(inp["dout"], 101 * i, 0).contiguous() for i in range(3)]
    order = [0, 1, 2, 1]
    ref = {}
    for i in sorted(set(order)):
        Li, oi, di = _run(cfg, dict(inp, x=xs[i], dout=ds[i]))
        ref[i] = (oi.cpu(), di.cpu(), Li.dW1.cpu(), Li.dW2.cpu())
        del Li
    L = _layer(cfg, inp)
    host = [(xs[i].cpu().pin_memory(), ds[i].cpu().pin_memory()) for i in range(3)]
    outs = [(torch.empty_like(host[0][0]).pin_memory(), torch.empty_like(host[0][0]).pin_memory())
            for _ in order]
    bufs = [[torch.empty_like(inp["x"]) for _ in range(4)] for _ in range(2)]
    stream = torch.cuda.current_stream()
    for n, i in enumerate(order):
        L.step_host(host[i][0], host[i][1], outs[n][0], outs[n][1], *bufs[n % 2])
    L.step_host_sync()                   # the stream, not the device, is synchronised
    stream.synchronize()
    assert L.status.item() == 0
    for n, i in enumerate(order):
        assert torch.equal(outs[n][0], ref[i][0]), ("out", n)
        assert torch.equal(outs[n][1], ref[i][1]), ("dx", n)
    assert torch.equal(L.dW1.cpu(), ref[order[-1]][2]) and torch.equal(L.dW2.cpu(), ref[order[-1]][3])
