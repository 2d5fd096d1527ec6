"""Pins of the oracle's layer forward/backward: dense special cases, a
library autograd of the dense mixture, central finite differences and
token-permutation invariance."""
import numpy as np
import pytest
import torch

import oracle


def _layer(T, d, E, F, seed, wr_std=1.0):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d))
    W1 = rng.normal(size=(E, d, F)) * 0.3
    W3 = rng.normal(size=(E, d, F)) * 0.3
    W2 = rng.normal(size=(E, F, d)) * 0.3
    Wr = rng.normal(size=(d, E)) * wr_std
    dout = rng.normal(size=(T, d))
    return x, W1, W3, W2, Wr, dout


def test_single_expert_is_dense_swiglu():
    x, W1, W3, W2, Wr, _ = _layer(9, 8, 1, 6, 0)
    ctx = oracle.layer_forward(x, W1, W3, W2, 1, Wr=Wr, align=4)
    H1, H3 = x @ W1[0], x @ W3[0]
    dense = (H1 / (1 + np.exp(-H1)) * H3) @ W2[0]
    np.testing.assert_allclose(ctx["out"], dense, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(ctx["gates"], 1.0)


def test_k_equals_E_is_dense_mixture():
    T, d, E, F = 11, 8, 4, 6
    x, W1, W3, W2, Wr, _ = _layer(T, d, E, F, 1)
    ctx = oracle.layer_forward(x, W1, W3, W2, E, Wr=Wr, align=8)
    L = x @ Wr
    p = np.exp(L) / np.exp(L).sum(1, keepdims=True)
    dense = np.zeros((T, d))
    for e in range(E):
        H1, H3 = x @ W1[e], x @ W3[e]
        dense += p[:, e:e + 1] * ((H1 / (1 + np.exp(-H1)) * H3) @ W2[e])
    np.testing.assert_allclose(ctx["out"], dense, rtol=1e-12, atol=1e-12)


def test_backward_matches_torch_autograd_dense_mixture():
    """k = E: every expert is chosen and the gates are the full softmax, so
    the layer is a smooth dense mixture that torch's fp64 autograd can
    differentiate independently."""
    T, d, E, F = 7, 6, 3, 5
    x, W1, W3, W2, Wr, dout = _layer(T, d, E, F, 2)
    ctx = oracle.layer_forward(x, W1, W3, W2, E, Wr=Wr, align=4)
    g = oracle.layer_backward(ctx, dout)
    tx, t1, t3, t2, tr = [torch.tensor(a, dtype=torch.float64, requires_grad=True)
                          for a in (x, W1, W3, W2, Wr)]
    p = torch.softmax(tx @ tr, dim=1)
    out = sum(p[:, e:e + 1] * ((torch.nn.functional.silu(tx @ t1[e]) * (tx @ t3[e])) @ t2[e])
              for e in range(E))
    (out * torch.tensor(dout)).sum().backward()
    for name, t in (("dx", tx), ("dW1", t1), ("dW3", t3), ("dW2", t2), ("dWr", tr)):
        np.testing.assert_allclose(g[name], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def _loss(x, W1, W3, W2, Wr, dout, k, align):
    return float(np.sum(oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=align)["out"] * dout))


def test_backward_central_finite_differences():
    T, d, E, F, k, align = 6, 8, 4, 6, 2, 4
    x, W1, W3, W2, Wr, dout = _layer(T, d, E, F, 3, wr_std=2.0)
    L = x @ Wr
    srt = np.sort(L, axis=1)[:, ::-1]
    assert np.min(srt[:, k - 1] - srt[:, k]) > 1e-3   # no near-tie: top-k stays put
    ctx = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=align)
    g = oracle.layer_backward(ctx, dout)
    eps = 1e-6
    args = dict(x=x, W1=W1, W3=W3, W2=W2, Wr=Wr)
    names = {"x": "dx", "W1": "dW1", "W3": "dW3", "W2": "dW2", "Wr": "dWr"}
    for pname, arr in args.items():
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = arr[i]
            arr[i] = old + eps
            fp = _loss(**args, dout=dout, k=k, align=align)
            arr[i] = old - eps
            fm = _loss(**args, dout=dout, k=k, align=align)
            arr[i] = old
            num[i] = (fp - fm) / (2 * eps)
        ana = g[names[pname]]
        rel = np.max(np.abs(ana - num)) / np.max(np.abs(num))
        assert rel <= 1e-6, (pname, rel)


def test_gate_gradient_is_dot_of_dout_and_expert_output():
    T, d, E, F, k = 5, 4, 3, 4, 2
    x, W1, W3, W2, Wr, dout = _layer(T, d, E, F, 4)
    ctx = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=2)
    g = oracle.layer_backward(ctx, dout)
    # perturb a gate directly: out moves by eps * Y row
    for t in range(T):
        for j in range(k):
            y = ctx["Y"][ctx["meta"]["dst"][t, j]]
            assert abs(g["dg"][t, j] - float(dout[t] @ y)) < 1e-12


def test_token_permutation_invariance():
    T, d, E, F, k = 40, 8, 6, 6, 2
    x, W1, W3, W2, Wr, dout = _layer(T, d, E, F, 5)
    perm = np.random.default_rng(9).permutation(T)
    a = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=4)
    b = oracle.layer_forward(x[perm], W1, W3, W2, k, Wr=Wr, align=4)
    np.testing.assert_allclose(b["out"], a["out"][perm], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(b["topk_idx"], a["topk_idx"][perm])
    ga = oracle.layer_backward(a, dout)
    gb = oracle.layer_backward(b, dout[perm])
    np.testing.assert_allclose(gb["dx"], ga["dx"][perm], rtol=1e-11, atol=1e-12)
    for n in ("dW1", "dW3", "dW2", "dWr"):
        np.testing.assert_allclose(gb[n], ga[n], rtol=1e-11, atol=1e-12)
    # every group of b holds the same tokens (renamed), in ascending order
    mb = b["meta"]
    inv = np.argsort(perm)
    for e in range(E):
        ra = a["meta"]["src"][a["meta"]["poff"][e]:a["meta"]["poff"][e] + a["meta"]["counts"][e]]
        rb = mb["src"][mb["poff"][e]:mb["poff"][e] + mb["counts"][e]]
        assert sorted(inv[ra].tolist()) == rb.tolist()


def test_given_routing_uses_given_gates():
    T, d, E, F, k = 6, 4, 5, 4, 2
    x, W1, W3, W2, _, dout = _layer(T, d, E, F, 6)
    idx = np.array([[0, 1], [4, 2], [3, 0], [1, 3], [2, 4], [0, 2]], dtype=np.int32)
    gates = np.full((T, k), 0.5)
    ctx = oracle.layer_forward(x, W1, W3, W2, k, topk_idx=idx, gates=gates, align=4)
    ref = np.zeros((T, d))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            H1, H3 = x[t] @ W1[e], x[t] @ W3[e]
            ref[t] += 0.5 * ((H1 / (1 + np.exp(-H1)) * H3) @ W2[e])
    np.testing.assert_allclose(ctx["out"], ref, rtol=1e-12, atol=1e-13)
    g = oracle.layer_backward(ctx, dout)
    assert "dWr" not in g


def test_round_bf16_against_torch():
    rng = np.random.default_rng(0)
    v = (rng.normal(size=10000) * np.exp(rng.normal(size=10000) * 5)).astype(np.float32).astype(np.float64)
    ref = torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(v), ref)


def test_grouped_matmuls_equal_block_diagonal_dense_products():
    """Grouped products equal one dense product with a block-diagonal
    operand built from the groups (a plain library matmul)."""
    rng = np.random.default_rng(7)
    E, K, N = 3, 5, 4
    poff = np.array([0, 2, 2, 6])           # group 1 empty
    A = rng.normal(size=(6, K)); B = rng.normal(size=(E, K, N)); dC = rng.normal(size=(6, N))
    # dense: rows of group e use columns block e of a [6, E*K] expanded A
    Aexp = np.zeros((6, E * K))
    for e in range(E):
        Aexp[poff[e]:poff[e + 1], e * K:(e + 1) * K] = A[poff[e]:poff[e + 1]]
    Bstack = B.reshape(E * K, N)
    np.testing.assert_allclose(oracle.grouped_matmul(A, B, poff), Aexp @ Bstack, rtol=1e-13)
    np.testing.assert_allclose(oracle.grouped_matmul_t(dC, B, poff) , (dC @ Bstack.T).reshape(6, E, K)[np.arange(6), [0, 0, 2, 2, 2, 2]], rtol=1e-13)
    dB = oracle.grouped_wgrad(A, dC, poff, E)
    np.testing.assert_allclose(dB.reshape(E * K, N), Aexp.T @ dC, rtol=1e-13, atol=1e-14)
    assert np.all(dB[1] == 0)


def test_backward_pieces_compose_to_layer_backward():
    T, d, E, F, k = 9, 6, 4, 5, 2
    x, W1, W3, W2, Wr, dout = _layer(T, d, E, F, 8)
    ctx = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=2)
    g = oracle.layer_backward(ctx, dout)
    # SwiGLU backward against the closed form of d(silu(a) b)
    a = np.linspace(-4, 4, 17)
    s = 1 / (1 + np.exp(-a))
    d1, d3 = oracle.swiglu_backward(np.ones_like(a), a, np.full_like(a, 2.0))
    np.testing.assert_allclose(d1, 2.0 * (s + a * s * (1 - s)), rtol=1e-14)
    np.testing.assert_allclose(d3, a * s, rtol=1e-14)
    # dY rows are gate-scaled dout rows
    for t in range(T):
        for j in range(k):
            np.testing.assert_allclose(g["dY"][ctx["meta"]["dst"][t, j]], ctx["gates"][t, j] * dout[t])
