"""GPU parity of the tcgen05 grouped GEMMs (fwd / dgrad / wgrad, BF16 and
MXFP8) against the oracle's grouped products, on ragged groups with empty
experts, several tiles and a partial last tile per group."""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from gpu_util import f64, rel_err, scales_to_plain

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("mixture_experts_layer_25_b200")


def _groups(counts, extra_rows=256):
    counts = np.asarray(counts)
    padded = -(-counts // 128) * 128
    poff = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    A = int(poff[-1]) + extra_rows
    real = np.zeros(A, bool)
    for e, c in enumerate(counts):
        real[poff[e]:poff[e] + c] = True
    return poff, A, real


def _act(A, cols, real, seed, scale=1.0):
    t = moe_inputs.random_bf16((A, cols), seed, std=scale, device="cuda")
    t[torch.from_numpy(~real).cuda()] = 0     # pad rows are zero, as the library keeps them
    return t


def _w(E, r, c, seed):
    return moe_inputs.random_bf16((E, r, c), seed, std=0.05, device="cuda")


COUNTS = [0, 5, 300, 128, 1, 0, 513]


@pytest.mark.parametrize("mx", [False, True])
def test_fwd_plain(mx):
    E, K, N = len(COUNTS), 512, 512
    poff, A, real = _groups(COUNTS)
    X = _act(A, K, real, 1)
    B = _w(E, K, N, 2)
    P = int(poff[-1])
    tp = torch.from_numpy(poff).cuda()
    if not mx:
        C = moe.moe_grouped_gemm_fwd(X, B, tp, E)
        ref = oracle.grouped_matmul(f64(X), f64(B), poff)
    else:
        Xq, Xs = moe.mx_quantize(X, 0)
        Bq, Bs = moe.mx_quantize(B.view(E * K, N), 1)
        C = moe.moe_grouped_gemm_fwd(Xq, Bq.view(E, K, N), tp, E, A_sc=Xs, B_sc=Bs)
        Xd = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(f64(X)))
        Bd = oracle.mx_dequantize_cols(*oracle.mx_quantize_cols_grouped(f64(B).reshape(E * K, N), [0, E * K]))
        ref = oracle.grouped_matmul(Xd, Bd.reshape(E, K, N), poff)
    torch.cuda.synchronize()
    err = rel_err(f64(C[:P]), ref[:P])
    assert err < (1e-2 if not mx else 3e-2), err


@pytest.mark.parametrize("mx", [False, True])
def test_fwd_swiglu(mx):
    E, K, F = len(COUNTS), 256, 384
    poff, A, real = _groups(COUNTS)
    X = _act(A, K, real, 3)
    W1, W3 = _w(E, K, F, 4), _w(E, K, F, 5)
    P = int(poff[-1])
    tp = torch.from_numpy(poff).cuda()
    if not mx:
        h, aux = moe.moe_grouped_gemm_fwd(X, W1, tp, E, epilogue=moe.MOE_EPI_SWIGLU, B3=W3)
        Xd, W1d, W3d = f64(X), f64(W1), f64(W3)
    else:
        Xq, Xs = moe.mx_quantize(X, 0)
        W1q, W1s = moe.mx_quantize(W1.view(E * K, F), 1)
        W3q, W3s = moe.mx_quantize(W3.view(E * K, F), 1)
        h, aux = moe.moe_grouped_gemm_fwd(Xq, W1q.view(E, K, F), tp, E, epilogue=moe.MOE_EPI_SWIGLU,
                                          B3=W3q.view(E, K, F), A_sc=Xs, B_sc=W1s, B3_sc=W3s)
        Xd = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(f64(X)))
        q = lambda W: oracle.mx_dequantize_cols(*oracle.mx_quantize_cols_grouped(
            f64(W).reshape(E * K, F), [0, E * K])).reshape(E, K, F)
        W1d, W3d = q(W1), q(W3)
    torch.cuda.synchronize()
    H1 = oracle.grouped_matmul(Xd, W1d, poff)
    H3 = oracle.grouped_matmul(Xd, W3d, poff)
    tol = 1e-2 if not mx else 3e-2
    assert rel_err(f64(aux[:P, :F]), H1[:P]) < tol
    assert rel_err(f64(aux[:P, F:]), H3[:P]) < tol
    assert rel_err(f64(h[:P]), (oracle.silu(H1) * H3)[:P]) < tol


@pytest.mark.parametrize("mx", [False, True])
@pytest.mark.parametrize("dual", [False, True])
def test_dgrad(mx, dual):
    E, K, N = len(COUNTS), 512, 256
    poff, A, real = _groups(COUNTS)
    dC = _act(A, 2 * N if dual else N, real, 6)
    B, B3 = _w(E, K, N, 7), (_w(E, K, N, 8) if dual else None)
    P = int(poff[-1])
    tp = torch.from_numpy(poff).cuda()
    if not mx:
        dA = moe.moe_grouped_gemm_dgrad(dC, B, tp, E, B3=B3)
        dCd, Bd = f64(dC), f64(B)
        B3d = f64(B3) if dual else None
    else:
        dCq, dCs = moe.mx_quantize(dC, 0)
        Bq, Bs = moe.mx_quantize(B.view(E * K, N), 0)
        B3q, B3s = (moe.mx_quantize(B3.view(E * K, N), 0) if dual else (None, None))
        dA = moe.moe_grouped_gemm_dgrad(dCq, Bq.view(E, K, N), tp, E,
                                        B3=None if B3q is None else B3q.view(E, K, N),
                                        dC_sc=dCs, B_sc=Bs, B3_sc=B3s)
        dCd = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(f64(dC)))
        q = lambda W: oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(
            f64(W).reshape(E * K, N))).reshape(E, K, N)
        Bd = q(B)
        B3d = q(B3) if dual else None
    torch.cuda.synchronize()
    ref = oracle.grouped_matmul_t(dCd[:, :N], Bd, poff)
    if dual:
        ref += oracle.grouped_matmul_t(dCd[:, N:], B3d, poff)
    assert rel_err(f64(dA[:P]), ref[:P]) < (1e-2 if not mx else 3e-2)


@pytest.mark.parametrize("mx", [False, True])
def test_dgrad_swiglu_bwd(mx):
    E, F, d = len(COUNTS), 256, 512
    poff, A, real = _groups(COUNTS)
    dY = _act(A, d, real, 9)
    W2 = _w(E, F, d, 10)
    H13 = _act(A, 2 * F, real, 11, scale=2.0)
    P = int(poff[-1])
    tp = torch.from_numpy(poff).cuda()
    if not mx:
        dA = moe.moe_grouped_gemm_dgrad(dY, W2, tp, E, epilogue=moe.MOE_EPI_SWIGLU_BWD, aux=H13)
        dYd, W2d = f64(dY), f64(W2)
    else:
        dYq, dYs = moe.mx_quantize(dY, 0)
        Wq, Ws = moe.mx_quantize(W2.view(E * F, d), 0)
        dA = moe.moe_grouped_gemm_dgrad(dYq, Wq.view(E, F, d), tp, E,
                                        epilogue=moe.MOE_EPI_SWIGLU_BWD, aux=H13, dC_sc=dYs, B_sc=Ws)
        dYd = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(f64(dY)))
        W2d = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(f64(W2).reshape(E * F, d))).reshape(E, F, d)
    torch.cuda.synchronize()
    dh = oracle.grouped_matmul_t(dYd, W2d, poff)
    H = f64(H13)
    d1, d3 = oracle.swiglu_backward(dh, H[:, :F], H[:, F:])
    tol = 1e-2 if not mx else 3e-2
    assert rel_err(f64(dA[:P, :F]), d1[:P]) < tol
    assert rel_err(f64(dA[:P, F:]), d3[:P]) < tol


@pytest.mark.parametrize("mx", [False, True])
@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("K", [256, 384])
def test_wgrad(mx, split, K):
    """K % 256 == 0 in BF16 runs on SM pairs (256 x 256 tiles), K = 384 on
    single SMs."""
    E, N = len(COUNTS), 256
    poff, A, real = _groups(COUNTS)
    X = _act(A, K, real, 12)
    dC = _act(A, 2 * N if split else N, real, 13)
    tp = torch.from_numpy(poff).cuda()
    if not mx:
        r = moe.moe_grouped_gemm_wgrad(X, dC, tp, E, split=split)
        Xd, dCd = f64(X), f64(dC)
    else:
        Xq, Xs = moe.mx_quantize(X, 1)
        dCq, dCs = moe.mx_quantize(dC, 1)
        r = moe.moe_grouped_gemm_wgrad(Xq, dCq, tp, E, split=split, A_sc=Xs, dC_sc=dCs)
        Xd = oracle.mx_dequantize_cols(*oracle.mx_quantize_cols_grouped(f64(X), [0, A]))
        dCd = oracle.mx_dequantize_cols(*oracle.mx_quantize_cols_grouped(f64(dC), [0, A]))
    torch.cuda.synchronize()
    ref = oracle.grouped_wgrad(Xd, dCd, poff, E)
    tol = 1e-2 if not mx else 3e-2
    if split:
        dB, dB3 = r
        assert rel_err(f64(dB), ref[:, :, :N]) < tol
        assert rel_err(f64(dB3), ref[:, :, N:]) < tol
    else:
        assert rel_err(f64(r), ref) < tol
    got = f64(r[0] if split else r)
    assert np.all(got[0] == 0) and np.all(got[5] == 0)      # empty experts


def test_fwd_full_width_sampled_experts():
    """The 128-expert layer's GEMM1 shape (K = 2048, N = 2F = 2048) with
    ~512 rows per expert; checked on a sample of experts."""
    E, K, F = 128, 2048, 1024
    rng = np.random.default_rng(0)
    counts = rng.multinomial(65536, np.ones(E) / E)
    poff, A, real = _groups(counts, extra_rows=0)
    X = _act(A, K, real, 14)
    W1, W3 = _w(E, K, F, 15), _w(E, K, F, 16)
    tp = torch.from_numpy(poff).cuda()
    h, aux = moe.moe_grouped_gemm_fwd(X, W1, tp, E, epilogue=moe.MOE_EPI_SWIGLU, B3=W3)
    torch.cuda.synchronize()
    for e in (0, 37, 127):
        a, b = int(poff[e]), int(poff[e]) + int(counts[e])
        Xe = f64(X[a:b])
        H1 = Xe @ f64(W1[e]); H3 = Xe @ f64(W3[e])
        assert rel_err(f64(h[a:b]), oracle.silu(H1) * H3) < 1e-2
        assert rel_err(f64(aux[a:b, :F]), H1) < 1e-2


# ------------------------------------------------ tokens-N grouped GEMM (BF16)
# groups with 1, 2 and 3 token blocks, a block of 5 rows (MMA N = 16), and a
# last block whose padding runs past 256 rows (385 rows: blocks of 224 and 161)
COUNTS_TN = [0, 5, 300, 128, 1, 0, 513, 700, 256, 257, 385]


def _tn_setup(counts, cols, seed, garbage):
    poff, A, real = _groups(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    X = moe_inputs.random_bf16((A, cols), seed, device="cuda")
    # padding rows hold garbage: they must be neither multiplied nor copied
    X[torch.from_numpy(~real).cuda()] = 100.0 if garbage else 0.0
    return poff, offs, A, real, X


def _pad_rows(poff, real):
    P = int(poff[-1])
    return ~real[:P]


@pytest.mark.parametrize("with_offsets", [True, False])
def test_tn_fwd_swiglu(with_offsets):
    E, K, F = len(COUNTS_TN), 256, 384
    poff, offs, A, real, X = _tn_setup(COUNTS_TN, K, 21, with_offsets)
    W1, W3 = _w(E, K, F, 22), _w(E, K, F, 23)
    tp, to = torch.from_numpy(poff).cuda(), torch.from_numpy(offs).cuda()
    h, aux = moe.moe_grouped_gemm_tn(X, W1, tp, E, epilogue=moe.MOE_EPI_SWIGLU, W3=W3,
                                     offsets=to if with_offsets else None)
    torch.cuda.synchronize()
    P = int(poff[-1])
    Xd = f64(X)
    Xd[~real] = 0.0
    H1 = oracle.grouped_matmul(Xd, f64(W1), poff)
    H3 = oracle.grouped_matmul(Xd, f64(W3), poff)
    r = real[:P]
    assert rel_err(f64(aux[:P, :F])[r], H1[:P][r]) < 1e-2
    assert rel_err(f64(aux[:P, F:])[r], H3[:P][r]) < 1e-2
    assert rel_err(f64(h[:P])[r], (oracle.silu(H1) * H3)[:P][r]) < 1e-2
    pad = _pad_rows(poff, real)
    assert np.all(f64(h[:P])[pad] == 0) and np.all(f64(aux[:P])[pad] == 0)


def test_tn_fwd_plain():
    E, K, N = len(COUNTS_TN), 512, 512
    poff, offs, A, real, X = _tn_setup(COUNTS_TN, K, 24, True)
    W = _w(E, K, N, 25)
    tp, to = torch.from_numpy(poff).cuda(), torch.from_numpy(offs).cuda()
    C = moe.moe_grouped_gemm_tn(X, W, tp, E, offsets=to)
    torch.cuda.synchronize()
    P = int(poff[-1])
    Xd = f64(X)
    Xd[~real] = 0.0
    ref = oracle.grouped_matmul(Xd, f64(W), poff)
    r = real[:P]
    assert rel_err(f64(C[:P])[r], ref[:P][r]) < 1e-2
    assert np.all(f64(C[:P])[_pad_rows(poff, real)] == 0)


@pytest.mark.parametrize("rank1", [False, True])
def test_tn_dgrad_dual(rank1):
    """dA = dC[:, :Kw] W^T + dC[:, Kw:] W3^T (+ row_scale x col_vec), the
    GEMM1 dgrad of the layer with the router's share of dx."""
    E, Nout, Kw = len(COUNTS_TN), 512, 256
    poff, offs, A, real, X = _tn_setup(COUNTS_TN, 2 * Kw, 26, True)
    W, W3 = _w(E, Nout, Kw, 27), _w(E, Nout, Kw, 28)
    tp, to = torch.from_numpy(poff).cuda(), torch.from_numpy(offs).cuda()
    g = torch.Generator(device="cuda"); g.manual_seed(29)
    rs = torch.randn(A, generator=g, device="cuda") if rank1 else None
    cv = torch.randn((E, Nout), generator=g, device="cuda") * 0.02 if rank1 else None
    C = moe.moe_grouped_gemm_tn(X, W, tp, E, W3=W3, w_kmajor=True, offsets=to, row_scale=rs,
                                col_vec=cv)
    torch.cuda.synchronize()
    P = int(poff[-1])
    Xd = f64(X)
    Xd[~real] = 0.0
    ref = (oracle.grouped_matmul_t(Xd[:, :Kw], f64(W), poff) +
           oracle.grouped_matmul_t(Xd[:, Kw:], f64(W3), poff))
    if rank1:
        rsd, cvd = rs.double().cpu().numpy(), cv.double().cpu().numpy()
        for e in range(E):
            ref[poff[e]:poff[e + 1]] += np.outer(rsd[poff[e]:poff[e + 1]], cvd[e])
    r = real[:P]
    assert rel_err(f64(C[:P])[r], ref[:P][r]) < 1e-2
    assert np.all(f64(C[:P])[_pad_rows(poff, real)] == 0)


def test_max_expert_count():
    """E = 1024 groups (the kernels' limit), most of them empty: the tile
    schedules of both GEMM kernels and the tokens-N kernel's per-expert
    tables at their largest."""
    E, K, N = 1024, 256, 256
    counts = np.zeros(E, np.int64)
    counts[[0, 17, 511, 1023]] = [5, 300, 129, 64]
    poff, A, real = _groups(counts, extra_rows=0)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    X = _act(A, K, real, 31)
    W = _w(E, K, N, 32)
    tp, to = torch.from_numpy(poff).cuda(), torch.from_numpy(offs).cuda()
    C = moe.moe_grouped_gemm_fwd(X, W, tp, E)
    Ct = moe.moe_grouped_gemm_tn(X, W, tp, E, offsets=to)
    torch.cuda.synchronize()
    ref = oracle.grouped_matmul(f64(X), f64(W), poff)
    P = int(poff[-1])
    assert rel_err(f64(C[:P]), ref[:P]) < 1e-2
    assert rel_err(f64(Ct[:P]), ref[:P]) < 1e-2


def _routed(T, E, k, d, seed):
    idx, gates = moe_inputs.random_routing(T, E, k, seed)
    meta = moe.moe_route(None, None, None, k, E, topk_idx=torch.from_numpy(idx).cuda(),
                         gates=torch.from_numpy(gates).cuda())
    x = moe_inputs.random_bf16((T, d), seed + 1, device="cuda")
    ref = oracle.routing_metadata(idx, E, 128)
    return x, meta, ref


@pytest.mark.parametrize("T,E,k", [(700, 16, 4), (1, 8, 2), (3000, 64, 3)])
def test_fwd_gather_equals_fwd_on_permuted_rows(T, E, k):
    """The dispatch fused into the GEMM: A rows gathered from x by src give
    the same products as the GEMM on the permuted buffer (bit for bit: the
    same operands reach the same MMAs) and match the oracle."""
    d, F = 512, 256
    x, meta, ref = _routed(T, E, k, d, 30 + T)
    A = meta["A_pad_max"]
    W1, W3, W2 = _w(E, d, F, 31), _w(E, d, F, 32), _w(E, d, 512, 33)   # W2 as a [d, 512] map
    poff = meta["poff"]
    P = int(ref["poff"][E])
    Xp = moe.moe_permute(x, meta, k, E)
    h, aux = moe.moe_grouped_gemm_fwd(Xp, W1, poff, E, epilogue=moe.MOE_EPI_SWIGLU, B3=W3)
    hg, auxg = moe.moe_grouped_gemm_fwd_gather(x, meta["src"], W1, poff, E, A,
                                               epilogue=moe.MOE_EPI_SWIGLU, B3=W3)
    C = moe.moe_grouped_gemm_fwd(Xp, W2, poff, E)
    Cg = moe.moe_grouped_gemm_fwd_gather(x, meta["src"], W2, poff, E, A)
    torch.cuda.synchronize()
    assert torch.equal(hg[:P], h[:P]) and torch.equal(auxg[:P], aux[:P])
    assert torch.equal(Cg[:P], C[:P])
    Xp64 = oracle.permute_rows(f64(x), ref)
    H1 = oracle.grouped_matmul(Xp64, f64(W1), ref["poff"])
    H3 = oracle.grouped_matmul(Xp64, f64(W3), ref["poff"])
    assert rel_err(f64(hg[:P]), oracle.silu(H1) * H3) < 1e-2
    assert rel_err(f64(Cg[:P]), oracle.grouped_matmul(Xp64, f64(W2), ref["poff"])) < 1e-2
    pad = torch.from_numpy(ref["src"] < 0).cuda()
    assert torch.all(hg[:P][pad] == 0)


@pytest.mark.parametrize("T,E,k", [(700, 16, 4), (1, 8, 2), (3000, 64, 3)])
def test_wgrad_gather_equals_wgrad_on_permuted_rows(T, E, k):
    # d = 384: both forms run on single SMs (the permuted form takes SM
    # pairs when d % 256 == 0), so the same MMAs see the same operands
    d, F = 384, 256
    x, meta, ref = _routed(T, E, k, d, 40 + T)
    A = meta["A_pad_max"]
    real = np.zeros(A, bool)
    real[:len(ref["src"])] = ref["src"] >= 0
    dA = _act(A, 2 * F, real, 41)
    Xp = moe.moe_permute(x, meta, k, E)
    dW1, dW3 = moe.moe_grouped_gemm_wgrad(Xp, dA, meta["poff"], E, split=True)
    g1, g3 = moe.moe_grouped_gemm_wgrad_gather(x, meta["src"], dA, meta["poff"], E,
                                               offsets=meta["offsets"], split=True)
    torch.cuda.synchronize()
    assert torch.equal(g1, dW1) and torch.equal(g3, dW3)
    Xp64 = oracle.permute_rows(f64(x), ref)
    dA64 = f64(dA)[:len(ref["src"])]
    ref1 = oracle.grouped_wgrad(Xp64, dA64[:, :F], ref["poff"], E)
    ref3 = oracle.grouped_wgrad(Xp64, dA64[:, F:], ref["poff"], E)
    assert rel_err(f64(g1), ref1) < 1e-2 and rel_err(f64(g3), ref3) < 1e-2
    empty = np.nonzero(ref["counts"] == 0)[0]
    for e in empty:
        assert torch.all(g1[e] == 0) and torch.all(g3[e] == 0)


def _same_codes(q_fused, q_ref, R, C, axis, P):
    """Fused-epilogue MX codes and scales equal the quantiser's on rows < P."""
    (cf, sf), (cr, sr) = q_fused, q_ref
    assert torch.equal(cf[:P], cr[:P])
    pf, pr = scales_to_plain(sf, R, C, axis), scales_to_plain(sr, R, C, axis)
    rows = P if axis == 0 else P // 32
    np.testing.assert_array_equal(pf[:rows], pr[:rows])


def test_fwd_swiglu_mxq_equals_quantised_h():
    """GEMM1 + SwiGLU in MXFP8 with h quantised in the epilogue: codes and
    scales along F and down the rows are bit-identical to mx_quantize_dual
    of the h the plain MX call stores, and [H1 | H3] is the same."""
    E, K, F = len(COUNTS), 256, 256
    poff, A, real = _groups(COUNTS)
    X = _act(A, K, real, 50)
    W1, W3 = _w(E, K, F, 51), _w(E, K, F, 52)
    tp = torch.from_numpy(poff).cuda()
    P = int(poff[-1])
    Xq, Xs = moe.mx_quantize(X, 0)
    W1q, W1s = moe.mx_quantize(W1.view(E * K, F), 1)
    W3q, W3s = moe.mx_quantize(W3.view(E * K, F), 1)
    h, aux = moe.moe_grouped_gemm_fwd(Xq, W1q.view(E, K, F), tp, E, epilogue=moe.MOE_EPI_SWIGLU,
                                      B3=W3q.view(E, K, F), A_sc=Xs, B_sc=W1s, B3_sc=W3s)
    aux2, qrow, qcol = moe.moe_grouped_gemm_fwd_swiglu_mxq(Xq, Xs, W1q.view(E, K, F), W1s,
                                                           W3q.view(E, K, F), W3s, tp, E)
    ref_row, ref_col = moe.mx_quantize_dual(h)
    torch.cuda.synchronize()
    assert torch.equal(aux2[:P], aux[:P])
    _same_codes(qrow, ref_row, A, F, 0, P)
    _same_codes(qcol, ref_col, A, F, 1, P)


def test_dgrad_swiglu_mxq_equals_quantised_dA():
    """GEMM2 dgrad + SwiGLU backward in MXFP8 with dA quantised in the
    epilogue: bit-identical to mx_quantize_dual of the stored dA."""
    E, F, d = len(COUNTS), 256, 512
    poff, A, real = _groups(COUNTS)
    dY = _act(A, d, real, 53)
    W2 = _w(E, F, d, 54)
    H13 = _act(A, 2 * F, real, 55, scale=2.0)
    P = int(poff[-1])
    tp = torch.from_numpy(poff).cuda()
    dYq, dYs = moe.mx_quantize(dY, 0)
    Wq, Ws = moe.mx_quantize(W2.view(E * F, d), 0)
    dA = moe.moe_grouped_gemm_dgrad(dYq, Wq.view(E, F, d), tp, E, epilogue=moe.MOE_EPI_SWIGLU_BWD,
                                    aux=H13, dC_sc=dYs, B_sc=Ws)
    qrow, qcol = moe.moe_grouped_gemm_dgrad_swiglu_mxq(dYq, dYs, Wq.view(E, F, d), Ws, H13, tp, E)
    ref_row, ref_col = moe.mx_quantize_dual(dA)
    torch.cuda.synchronize()
    _same_codes(qrow, ref_row, A, 2 * F, 0, P)
    _same_codes(qcol, ref_col, A, 2 * F, 1, P)
