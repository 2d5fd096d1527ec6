"""Pins of the oracle's router, top-k, gates and routing metadata against
hand-worked cases, brute-force per-token loops and the routing invariants."""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute_topk(row, k):
    """Pure-Python selection: k times, take the largest remaining value,
    the lowest index among equals."""
    chosen = []
    for _ in range(k):
        best = None
        for e, v in enumerate(row):
            if e in chosen:
                continue
            if best is None or v > row[best]:
                best = e
        chosen.append(best)
    return chosen


def _brute_gates(row, chosen):
    z = sum(math.exp(row[e]) for e in range(len(row)))       # full softmax
    p = [math.exp(row[e]) / z for e in chosen]
    s = sum(p)
    return [q / s for q in p]                                 # renormalised


def test_topk_golden_cases():
    n = 0
    for line in open(os.path.join(GOLDEN, "topk_cases.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, logits, idx, gates = [p.strip() for p in line.split("|")]
        L = np.array([[float(v) for v in logits.split()]])
        got_i = oracle.topk_select(L, int(k))
        got_g = oracle.gates_from_logits(L, got_i)
        assert got_i[0].tolist() == [int(v) for v in idx.split()], line
        np.testing.assert_allclose(got_g[0], [float(v) for v in gates.split()], rtol=1e-14)
        n += 1
    assert n >= 7


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    T, E, k = 200, 9, 3
    # coarse values force many exact ties
    L = rng.integers(-3, 4, size=(T, E)).astype(np.float64) * 0.5
    idx = oracle.topk_select(L, k)
    g = oracle.gates_from_logits(L, idx)
    for t in range(T):
        row = L[t].tolist()
        ch = _brute_topk(row, k)
        assert idx[t].tolist() == ch
        np.testing.assert_allclose(g[t], _brute_gates(row, ch), rtol=1e-12)


def test_gates_invariants():
    rng = np.random.default_rng(5)
    L = rng.normal(size=(500, 16)) * 3
    idx = oracle.topk_select(L, 4)
    g = oracle.gates_from_logits(L, idx)
    assert np.all(g >= 0)
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-14)
    # k distinct experts per token, in descending logit order
    for t in range(len(L)):
        assert len(set(idx[t].tolist())) == 4
        v = L[t, idx[t]]
        assert np.all(np.diff(v) <= 0)
    # gates descend with the logits
    assert np.all(np.diff(g, axis=1) <= 1e-15)


def test_router_logits_closed_form():
    # one-hot tokens pick rows of Wr; the bias shifts every row
    d, E = 6, 5
    rng = np.random.default_rng(1)
    Wr = rng.normal(size=(d, E))
    b = rng.normal(size=E)
    x = np.eye(d)
    np.testing.assert_array_equal(oracle.router_logits(x, Wr), Wr)
    np.testing.assert_array_equal(oracle.router_logits(x, Wr, b), Wr + b)


def _check_metadata(idx, E, align, meta):
    T, k = idx.shape
    counts, offsets, poff = meta["counts"], meta["offsets"], meta["poff"]
    dst, src = meta["dst"], meta["src"]
    # counts by direct tally
    assert counts.tolist() == [int(np.sum(idx == e)) for e in range(E)]
    assert counts.sum() == T * k
    assert offsets[0] == 0 and np.all(np.diff(offsets) == counts)
    pc = [(-(-c // align)) * align for c in counts]
    assert poff[0] == 0 and np.diff(poff).tolist() == pc
    assert np.all(poff % align == 0)
    # dst is a bijection onto the real (non-pad) rows, src inverts it
    flat = dst.reshape(-1)
    assert len(set(flat.tolist())) == T * k
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            r = dst[t, j]
            assert poff[e] <= r < poff[e] + counts[e]
            assert src[r] == t
    # pad rows are marked -1, real rows are the first counts[e] of a group
    for e in range(E):
        assert np.all(src[poff[e]:poff[e] + counts[e]] >= 0)
        assert np.all(src[poff[e] + counts[e]:poff[e + 1]] == -1)
        # stable: tokens ascend inside a group
        assert np.all(np.diff(src[poff[e]:poff[e] + counts[e]]) > 0)


@pytest.mark.parametrize("T,E,k,align", [(1, 4, 2, 128), (7, 5, 3, 4), (300, 16, 4, 128),
                                         (129, 8, 8, 32), (50, 64, 2, 128)])
def test_routing_metadata_invariants(T, E, k, align):
    rng = np.random.default_rng(T * 31 + E)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    meta = oracle.routing_metadata(idx, E, align)
    _check_metadata(idx, E, align, meta)


def test_routing_metadata_hand_case():
    # tokens 0..3, k=2, E=3, align=2
    idx = np.array([[2, 0], [0, 1], [2, 1], [0, 2]])
    m = oracle.routing_metadata(idx, 3, 2)
    assert m["counts"].tolist() == [3, 2, 3]
    assert m["offsets"].tolist() == [0, 3, 5, 8]
    assert m["poff"].tolist() == [0, 4, 6, 10]
    # expert 0 rows 0..2 take tokens 0,1,3; expert 1 rows 4,5 tokens 1,2;
    # expert 2 rows 6..8 tokens 0,2,3
    assert m["dst"].tolist() == [[6, 0], [1, 4], [7, 5], [2, 8]]
    assert m["src"].tolist() == [0, 1, 3, -1, 1, 2, 0, 2, 3, -1]


def test_permute_rows():
    idx = np.array([[1, 0], [1, 2]])
    m = oracle.routing_metadata(idx, 3, 2)
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    Xp = oracle.permute_rows(x, m)
    # expert 0: token 0 + pad; expert 1: tokens 0, 1; expert 2: token 1 + pad
    np.testing.assert_array_equal(Xp, [[1, 2], [0, 0], [1, 2], [3, 4], [3, 4], [0, 0]])
