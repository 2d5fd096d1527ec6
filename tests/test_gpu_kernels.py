"""GPU parity of the routing, dispatch, combine, backward and MX kernels
against the CPU oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from gpu_util import f64, np_i, rel_err, scales_to_plain

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("mixture_experts_layer_25_b200")
U = 2.0 ** -24


def _router_inputs(T, d, E, seed, bias=False):
    x = moe_inputs.random_bf16((T, d), seed, device="cuda")
    g = torch.Generator(device="cuda"); g.manual_seed(seed + 1)
    Wr = (torch.randn((d, E), generator=g, device="cuda") * 0.02).contiguous()
    b = None
    if bias:
        rng = np.random.default_rng(seed + 2)
        rank = rng.permutation(E) + 1
        b = torch.tensor(3.0 * np.log(rank.astype(np.float64) ** -1.2), dtype=torch.float32).cuda()
    return x, Wr, b


def _check_metadata(meta, idx, E):
    """GPU metadata bit-exact against the oracle's counting sort of idx."""
    ref = oracle.routing_metadata(idx, E, 128)
    assert np_i(meta["counts"]).tolist() == ref["counts"].tolist()
    assert np_i(meta["offsets"]).tolist() == ref["offsets"].tolist()
    assert np_i(meta["poff"]).tolist() == ref["poff"].tolist()
    np.testing.assert_array_equal(np_i(meta["dst"]), ref["dst"])
    src = np_i(meta["src"])
    P = int(ref["poff"][E])
    np.testing.assert_array_equal(src[:P], ref["src"])
    assert np.all(src[P:] == -1)
    return ref


@pytest.mark.parametrize("T,d,E,k,bias", [
    (1024, 256, 8, 2, False),     # the tiny layer
    (37, 64, 5, 3, False),        # ragged: one partial routing block (CUDA-core path)
    (37, 128, 8, 2, False),       # ragged, tensor-core path
    (300, 256, 64, 8, True),      # k = 8 on the tensor-core path
    (200, 64, 136, 3, False),     # E > 128: CUDA-core path
    (1000, 128, 16, 4, True),
    (4096, 2048, 128, 4, True),   # skewed load, many empty experts
    (16384, 2048, 128, 4, False), # the 128-expert layer at full size
])
def test_route_router_mode(T, d, E, k, bias):
    x, Wr, b = _router_inputs(T, d, E, 11 + T, bias)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    meta = moe.moe_route(x, Wr, b, k, E, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Lg = f64(meta["logits"])
    idx_g = np_i(meta["topk_idx"])
    # (i) strict: the oracle's selection and metadata on the device's logits
    idx_o = oracle.topk_select(Lg, k)
    np.testing.assert_array_equal(idx_g, idx_o)
    assert rel_err(f64(meta["gates"]), oracle.gates_from_logits(Lg, idx_o)) < 1e-5
    _check_metadata(meta, idx_o, E)
    # (ii) end to end: fp32 logits within the fp32 dot-product bound of the
    # fp64 logits; only near-tie tokens may choose differently (a tie at the
    # selection boundary changes the set, one inside the top k its order)
    x64, W64 = f64(x), f64(Wr)
    b64 = None if b is None else f64(b)
    L64 = oracle.router_logits(x64, W64, b64)
    bound = 4 * d * U * (np.abs(x64) @ np.abs(W64)) + 4 * U * np.abs(L64)
    assert np.all(np.abs(Lg - L64) <= bound)
    srt = -np.sort(-L64, axis=1)
    kk = min(k + 1, E)
    near = np.any(srt[:, :kk - 1] - srt[:, 1:kk] < 2 * bound.max(axis=1)[:, None], axis=1)
    differ = np.any(oracle.topk_select(L64, k) != idx_g, axis=1)
    assert not np.any(differ & ~near)
    if bias:
        assert np.sum(np_i(meta["counts"]) == 0) >= 1


@pytest.mark.parametrize("T,E,k", [(8192, 384, 8), (100, 7, 7), (1, 4, 2), (3000, 64, 1)])
def test_route_given_mode(T, E, k):
    idx, gates = moe_inputs.random_routing(T, E, k, 5 + T)
    ti = torch.from_numpy(idx).cuda()
    tg = torch.from_numpy(gates).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    meta = moe.moe_route(None, None, None, k, E, topk_idx=ti, gates=tg, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    _check_metadata(meta, idx, E)


def test_route_given_mode_rejects_bad_experts():
    idx, gates = moe_inputs.random_routing(64, 8, 3, 1)
    idx[5, 1] = 8          # out of range
    idx[9, 2] = idx[9, 0]  # repeated inside a token
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    meta = moe.moe_route(None, None, None, 3, 8, topk_idx=torch.from_numpy(idx).cuda(),
                         gates=torch.from_numpy(gates).cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == (moe.MOE_DEV_BAD_EXPERT | moe.MOE_DEV_DUP_EXPERT)
    dst = np_i(meta["dst"])
    assert dst[5, 1] == -1 and dst[9, 2] == -1
    counts = np_i(meta["counts"])
    assert counts.sum() == 64 * 3 - 2
    src = np_i(meta["src"])
    valid = dst[dst >= 0]
    assert len(set(valid.tolist())) == len(valid) and np.all(src[valid] >= 0)


def _meta_for(T, E, k, seed):
    idx, gates = moe_inputs.random_routing(T, E, k, seed)
    meta = moe.moe_route(None, None, None, k, E, topk_idx=torch.from_numpy(idx).cuda(),
                         gates=torch.from_numpy(gates).cuda())
    return idx, gates, meta


@pytest.mark.parametrize("T,d,E,k", [(1024, 256, 8, 2), (333, 2048, 64, 4), (50, 6144, 384, 8),
                                     (5000, 2048, 128, 4), (700, 1024, 16, 3), (1, 2048, 8, 4)])
def test_permute_bit_exact_and_pad_rows_zero(T, d, E, k):
    idx, gates, meta = _meta_for(T, E, k, 3)
    x = moe_inputs.random_bf16((T, d), 7, device="cuda")
    Xp = moe.moe_permute(x, meta, k, E)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    P = int(ref["poff"][E])
    np.testing.assert_array_equal(f64(Xp[:P]), oracle.permute_rows(f64(x), ref))


def test_permute_fused_mx_codes():
    T, d, E, k = 700, 512, 16, 4
    idx, gates, meta = _meta_for(T, E, k, 4)
    x = moe_inputs.random_bf16((T, d), 8, device="cuda")
    x[3, :64] = 0          # an all-zero block
    x[4, :32] *= 1e-30     # tiny values
    Xp, Xq, Xs = moe.moe_permute(x, meta, k, E, mx=True)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    P = int(ref["poff"][E])
    Xp64 = oracle.permute_rows(f64(x), ref)
    c, s = oracle.mx_quantize_rows(Xp64)
    np.testing.assert_array_equal(Xq[:P].cpu().numpy(), c)
    A = meta["A_pad_max"]
    np.testing.assert_array_equal(scales_to_plain(Xs, A, d, 0)[:P], s)


@pytest.mark.parametrize("T,d,E,k", [(700, 512, 16, 4), (1, 256, 8, 2), (64, 6144, 384, 8),
                                     (3000, 2048, 128, 4)])
def test_permute_mx_codes_both_axes(T, d, E, k):
    """Dispatch straight into MX codes: along d and down the rows, bit-exact
    against the oracle's quantisers applied to the oracle's permuted rows."""
    idx, gates, meta = _meta_for(T, E, k, 6 + T)
    x = moe_inputs.random_bf16((T, d), 9 + T, device="cuda")
    x[0, :64] = 0                                   # zero blocks
    (q, qs), (qT, qTs) = moe.moe_permute_mx(x, meta, E)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    P = int(ref["poff"][E])
    A = meta["A_pad_max"]
    Xp64 = oracle.permute_rows(f64(x), ref)
    c0, s0 = oracle.mx_quantize_rows(Xp64)
    c1, s1 = oracle.mx_quantize_cols_grouped(Xp64, ref["poff"])
    np.testing.assert_array_equal(q[:P].cpu().numpy(), c0)
    np.testing.assert_array_equal(scales_to_plain(qs, A, d, 0)[:P], s0)
    np.testing.assert_array_equal(qT[:P].cpu().numpy(), c1)
    np.testing.assert_array_equal(scales_to_plain(qTs, A, d, 1)[:P // 32], s1)


@pytest.mark.parametrize("T,d,E,k", [(700, 512, 16, 4), (1, 256, 8, 2), (64, 6144, 384, 8)])
def test_combine_bwd_mx_codes_both_axes(T, d, E, k):
    """The backward's gate-scaled rows straight into MX codes: bit-exact
    against the oracle's quantisers of the bf16-rounded dY rows."""
    idx, gates, meta = _meta_for(T, E, k, 16 + T)
    dout = moe_inputs.random_bf16((T, d), 19 + T, device="cuda")
    (q, qs), (qT, qTs) = moe.moe_combine_bwd_mx(dout, meta["gates"], meta, E)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    P = int(ref["poff"][E])
    A = meta["A_pad_max"]
    # dY as the kernel forms it, g * dout in fp32 then rounded to bf16: the
    # codes are integer decisions taken in the kernel's precision
    g32 = meta["gates"].cpu().numpy().astype(np.float32)
    d32 = f64(dout).astype(np.float32)
    dY = np.zeros((P, d))
    for j in range(k):
        prod = torch.from_numpy(g32[:, j:j + 1] * d32).to(torch.bfloat16).to(torch.float64)
        dY[ref["dst"][:, j]] = prod.numpy()
    c0, s0 = oracle.mx_quantize_rows(dY)
    c1, s1 = oracle.mx_quantize_cols_grouped(dY, ref["poff"])
    np.testing.assert_array_equal(q[:P].cpu().numpy(), c0)
    np.testing.assert_array_equal(scales_to_plain(qs, A, d, 0)[:P], s0)
    np.testing.assert_array_equal(qT[:P].cpu().numpy(), c1)
    np.testing.assert_array_equal(scales_to_plain(qTs, A, d, 1)[:P // 32], s1)


@pytest.mark.parametrize("R,C,axis", [(256, 512, 0), (512, 384, 1), (128, 128, 0), (384, 2048, 1)])
def test_mx_quantize_bit_exact(R, C, axis):
    g = torch.Generator(device="cuda"); g.manual_seed(R + C + axis)
    v = torch.randn((R, C), generator=g, device="cuda") * torch.exp(
        torch.randn((R, 1), generator=g, device="cuda") * 3)
    v = v.to(torch.bfloat16)
    v[0, :32] = 0
    v[1, 5] = -0.0
    v[2, :] = -v[2, :].abs() * 1e-6
    v[5, 7] = 300.0
    v[6, 0] = 400.0        # a negative value that rounds to zero keeps its sign
    v[6, 1] = -1e-5
    codes, scales = moe.mx_quantize(v, axis)
    torch.cuda.synchronize()
    v64 = f64(v)
    if axis == 0:
        c, s = oracle.mx_quantize_rows(v64)
    else:
        c, s = oracle.mx_quantize_cols_grouped(v64, np.array([0, R]))
    np.testing.assert_array_equal(codes.cpu().numpy(), c)
    np.testing.assert_array_equal(scales_to_plain(scales, R, C, axis), s)


@pytest.mark.parametrize("R,C", [(256, 512), (384, 384), (128, 2048)])
def test_mx_quantize_dual_equals_both_axes(R, C):
    g = torch.Generator(device="cuda"); g.manual_seed(R * 7 + C)
    v = (torch.randn((R, C), generator=g, device="cuda") *
         torch.exp(torch.randn((R, 1), generator=g, device="cuda") * 3)).to(torch.bfloat16)
    v[3, :40] = 0
    v[7, 9] = -1e-30
    (cr, sr), (cc, sc) = moe.mx_quantize_dual(v)
    torch.cuda.synchronize()
    v64 = f64(v)
    c0, s0 = oracle.mx_quantize_rows(v64)
    c1, s1 = oracle.mx_quantize_cols_grouped(v64, np.array([0, R]))
    np.testing.assert_array_equal(cr.cpu().numpy(), c0)
    np.testing.assert_array_equal(scales_to_plain(sr, R, C, 0), s0)
    np.testing.assert_array_equal(cc.cpu().numpy(), c1)
    np.testing.assert_array_equal(scales_to_plain(sc, R, C, 1), s1)


@pytest.mark.parametrize("R,C,n", [(384, 256, 200), (256, 512, 129), (512, 128, 64)])
def test_mx_quantize_dual_partial_rows(R, C, n):
    """mx_quantize_dual with a device row count n < R: rows below n get the
    codes and row scales of the full quantisation; a 32-row column block
    that starts below n gets the full block's column scale (rows at and
    beyond n are still part of its maximum); a block of a processed 128-row
    tile that starts at or beyond n gets scale byte 0."""
    g = torch.Generator(device="cuda"); g.manual_seed(R + C + n)
    v = (torch.randn((R, C), generator=g, device="cuda") *
         torch.exp(torch.randn((R, 1), generator=g, device="cuda") * 2)).to(torch.bfloat16)
    nrows = torch.tensor([n], dtype=torch.int32, device="cuda")
    (cr, sr), (cc, sc) = moe.mx_quantize_dual(v, nrows=nrows)
    torch.cuda.synchronize()
    v64 = f64(v)
    c0, s0 = oracle.mx_quantize_rows(v64)
    c1, s1 = oracle.mx_quantize_cols_grouped(v64, np.array([0, R]))
    np.testing.assert_array_equal(cr.cpu().numpy()[:n], c0[:n])
    np.testing.assert_array_equal(scales_to_plain(sr, R, C, 0)[:n], s0[:n])
    np.testing.assert_array_equal(cc.cpu().numpy()[:n], c1[:n])
    col = scales_to_plain(sc, R, C, 1)          # [R / 32, C]
    live = -(-n // 32)                          # blocks starting below n
    np.testing.assert_array_equal(col[:live], s1[:live])
    tiles_end = -(-n // 128) * 4                # blocks of the processed tiles
    assert np.all(col[live:tiles_end] == 0)


def _every_finite_bf16_in_blocks():
    """Blocks of 32 that hold every finite bf16 value (both zeros and the
    subnormals included) in several roles, as float64 [n_blocks, 32]:
    * each value v as its block's maximum, with 31 companions v * (-1)^j
      2^(-j/2) rounded to bf16 (down to E4M3 subnormals and to zero);
    * each value v with |v| <= M as an ordinary element of a block whose
      maximum is a fixed M (the largest finite bf16, 1, 1.5, 2^100, 2^-120 and
      the subnormal 2^-130), 31 values per block, either sign of M."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    v = f[np.isfinite(f)].astype(np.float64)
    to_bf16 = lambda a: torch.tensor(a).to(torch.bfloat16).to(torch.float64).numpy()  # noqa: E731
    j = np.arange(1, 32)
    comp = to_bf16(v[:, None] * ((-1.0) ** j * 2.0 ** (-j / 2.0))[None, :])
    fam = [np.concatenate([v[:, None], comp], axis=1)]
    bmax = float(np.max(v))
    for i, M in enumerate([bmax, 1.0, 1.5, 2.0 ** 100, 2.0 ** -120, 2.0 ** -130]):
        u = v[np.abs(v) <= M]
        n = -(-len(u) // 31)
        body = np.concatenate([u, np.zeros(n * 31 - len(u))]).reshape(n, 31)
        head = np.full((n, 1), M if i % 2 == 0 else -M)
        fam.append(np.concatenate([head, body], axis=1))
    return np.concatenate(fam, axis=0)


def _blocks_as(blocks, axis, C=128):
    """[n, 32] blocks -> a [R, C] array (R, C multiples of 128) whose 32-blocks
    along rows (axis 0) or down columns (axis 1) are the given blocks, in
    order, padded with zero blocks."""
    per = C // 32 if axis == 0 else C
    n = -(-len(blocks) // per)
    rows_per = 1 if axis == 0 else 32
    R = -(-n * rows_per // 128) * 128
    pad = R // rows_per * per - len(blocks)
    b = np.concatenate([blocks, np.zeros((pad, 32))], axis=0)
    if axis == 0:
        return b.reshape(R, C)
    return b.reshape(R // 32, C, 32).transpose(0, 2, 1).reshape(R, C)


def test_mx_quantisers_on_every_finite_bf16_value():
    """Every finite bf16 value through the row and column quantisers, the
    dual quantiser (both arrangements) and the permute's fused MX codes,
    bit-exact against the oracle's quantiser."""
    blocks = _every_finite_bf16_in_blocks()
    for axis in (0, 1):
        a = _blocks_as(blocks, axis)
        R, C = a.shape
        t = torch.tensor(a).to(torch.bfloat16).cuda()
        np.testing.assert_array_equal(f64(t), a)             # every value is a bf16 number
        if axis == 0:
            c_ref, s_ref = oracle.mx_quantize_rows(a)
        else:
            c_ref, s_ref = oracle.mx_quantize_cols_grouped(a, np.array([0, R]))
        codes, scales = moe.mx_quantize(t, axis)
        (cr, sr), (cc, sc) = moe.mx_quantize_dual(t)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
        np.testing.assert_array_equal(scales_to_plain(scales, R, C, axis), s_ref)
        c0, s0 = oracle.mx_quantize_rows(a)
        c1, s1 = oracle.mx_quantize_cols_grouped(a, np.array([0, R]))
        np.testing.assert_array_equal(cr.cpu().numpy(), c0)
        np.testing.assert_array_equal(scales_to_plain(sr, R, C, 0), s0)
        np.testing.assert_array_equal(cc.cpu().numpy(), c1)
        np.testing.assert_array_equal(scales_to_plain(sc, R, C, 1), s1)
    # the permute's fused quantisation: the rows of the axis-0 arrangement
    # as tokens, each routed to k = 2 of 8 experts
    x64 = _blocks_as(blocks, 0)
    T, d = x64.shape
    x = torch.tensor(x64).to(torch.bfloat16).cuda()
    idx, gates, meta = _meta_for(T, 8, 2, 5)
    Xp, Xq, Xs = moe.moe_permute(x, meta, 2, 8, mx=True)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, 8, 128)
    P = int(ref["poff"][8])
    c, s = oracle.mx_quantize_rows(oracle.permute_rows(x64, ref))
    np.testing.assert_array_equal(Xq[:P].cpu().numpy(), c)
    np.testing.assert_array_equal(scales_to_plain(Xs, meta["A_pad_max"], d, 0)[:P], s)


@pytest.mark.parametrize("T,d,E,k", [(1024, 256, 8, 2), (257, 2048, 32, 4), (64, 6144, 384, 8),
                                     (3000, 1024, 16, 3), (5000, 2048, 64, 4), (1, 2048, 8, 4)])
def test_combine_and_its_backward(T, d, E, k):
    """Gate-weighted combine and its backward against the oracle; the cases
    cover both backward kernels (persistent with prefetch for d <= 2048 and
    k <= 4, one token per team otherwise), several persistent sweeps
    (T = 3000, 5000), two tokens per block (d = 1024), k = 3 and T = 1."""
    idx, gates, meta = _meta_for(T, E, k, 5)
    A = meta["A_pad_max"]
    Y = moe_inputs.random_bf16((A, d), 9, device="cuda")
    dout = moe_inputs.random_bf16((T, d), 10, device="cuda")
    tg = torch.from_numpy(gates).cuda()
    out = moe.moe_unpermute_combine(Y, tg, meta["dst"])
    dY, dg, dl, dl_rows = moe.moe_combine_bwd(dout, Y, tg, meta, E)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    dst = ref["dst"]
    Y64, g64 = f64(Y), gates.astype(np.float64)
    assert rel_err(f64(out), oracle.combine(Y64, g64, dst)) < 1e-2
    dY_o, dg_o = oracle.combine_backward(f64(dout), Y64, g64, dst)
    P = int(ref["poff"][E])
    assert rel_err(f64(dY[:P]), dY_o[:P]) < 1e-2
    pad = ref["src"] < 0
    assert np.all(f64(dY[:P])[pad] == 0)
    assert np.all(dl_rows.cpu().numpy()[:P][pad] == 0)      # pad rows of dl_rows are zero too
    assert rel_err(dg.cpu().numpy(), dg_o) < 1e-4
    dl_o = oracle.gate_logit_grad(g64, dg_o)
    assert rel_err(dl.cpu().numpy(), dl_o) < 1e-4
    np.testing.assert_allclose(dl_rows.cpu().numpy()[dst], dl.cpu().numpy(), rtol=0, atol=0)


@pytest.mark.parametrize("T,d,E,k", [(1024, 256, 8, 2), (300, 2048, 128, 4), (5000, 2048, 64, 4),
                                     (777, 1024, 16, 3), (1, 2048, 8, 4), (96, 6144, 384, 8)])
def test_unpermute_sum_and_router_grads(T, d, E, k):
    idx, gates, meta = _meta_for(T, E, k, 6)
    A = meta["A_pad_max"]
    dXp = moe_inputs.random_bf16((A, d), 12, device="cuda")
    x = moe_inputs.random_bf16((T, d), 13, device="cuda")
    g = torch.Generator(device="cuda"); g.manual_seed(14)
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.02
    dl = torch.randn((T, k), generator=g, device="cuda")
    dl_rows = torch.zeros(A, dtype=torch.float32, device="cuda")
    dst_t = meta["dst"].long()
    dl_rows[dst_t.reshape(-1)] = dl.reshape(-1)
    dx_plain = moe.moe_unpermute_sum(dXp, meta["dst"])
    dx = moe.moe_unpermute_sum(dXp, meta["dst"], topk_idx=meta["topk_idx"], dl=dl, Wr=Wr, E=E)
    dWr = moe.moe_router_wgrad(x, meta, dl_rows, E)
    torch.cuda.synchronize()
    ref = oracle.routing_metadata(idx, E, 128)
    dxs = oracle.unpermute_sum(f64(dXp), ref["dst"])
    assert rel_err(f64(dx_plain), dxs) < 1e-2
    dWr_o, dxr = oracle.router_backward(f64(x), f64(Wr), idx, dl.cpu().numpy().astype(np.float64))
    assert rel_err(f64(dx), dxs + dxr) < 1e-2
    assert rel_err(dWr.cpu().numpy(), dWr_o) < 1e-4


def test_bounded_wait_reports_timeout_and_keeps_the_context_usable():
    """Failure detection without a fault: a wait that nothing satisfies gives
    up after 50 ms with MOE_DEV_TIMEOUT; the next launches still work."""
    import ctypes
    from mixture_experts_layer_25_b200 import _lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    _lib.call("moe_selftest_wait_timeout", ctypes.c_void_p(st.data_ptr()), 50_000_000, stream)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_DEV_TIMEOUT
    x = moe_inputs.random_bf16((128, 128), 3, device="cuda")
    q, s = moe.mx_quantize(x, 0)       # the context is still usable
    torch.cuda.synchronize()
    c, _ = oracle.mx_quantize_rows(f64(x))
    np.testing.assert_array_equal(q.cpu().numpy(), c)
