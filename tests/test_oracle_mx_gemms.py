"""Pins of the oracle's MXFP8 expert GEMMs: which axis each operand is
quantised along, and where the layer rounds to bf16 before quantising.

Two kinds of pin:

* exactness: for each of the six per-group GEMMs, operands that are exact
  MX numbers in blocks of 32 along that GEMM's K but NOT along the other
  axis.  Quantising along K leaves them unchanged, so the MX product equals
  the fp64 product bit for bit (the fp64 sums are exact at these sizes);
  quantising along the other axis changes them and the equality fails.
* brute force: a tiny MX layer, forward and backward, where every GEMM
  output is recomputed from its inputs with an independent quantiser (the
  E4M3 value set decoded by torch's float8_e4m3fn, a nearest-value search
  per element, the scale from the block maximum's binary exponent) applied
  block by block along that GEMM's K, after rounding each operand the device
  stores in bf16 with torch's own bf16 conversion.

Source of the format: [OC3-ja] "MXFP8による精度最適化" (MXFP8 expert GEMMs,
E4M3 elements with one power-of-two scale per 32 elements along K).
"""
import math

import numpy as np
import torch

import oracle

# E4M3 values by code, decoded by torch (independent of oracle.mx)
_CODES = torch.arange(256, dtype=torch.uint8)
_TABLE = _CODES.view(torch.float8_e4m3fn).to(torch.float64).numpy()
_POS = np.arange(0x7F)                 # non-negative finite codes 0 .. 126
_POS_VAL = _TABLE[_POS]


# --------------------------------------------------------------------------
# exactness pins
# --------------------------------------------------------------------------

def _exact_along(shape, axis, rng, scales=(-6, -5, -4, -3)):
    """Random values that are exact MX numbers for blocks of 32 along
    `axis` (0: 32 consecutive rows of a column; 1: 32 consecutive columns of
    a row).  Each block draws its own scale 2^s and holds one +-448 2^s
    element, so its MX scale is exactly 2^s; the other elements are E4M3
    values (subnormals included) times 2^s.  Blocks along the other axis mix
    scales, so a small element meets a larger block maximum there and loses
    bits."""
    R, C = shape
    v = np.empty(shape)
    if axis == 0:
        nb = R // 32
        for b in range(nb):
            for c in range(C):
                s = rng.choice(scales)
                codes = rng.integers(1, 0x7F, size=32)
                blk = _TABLE[codes] * np.where(rng.random(32) < 0.5, -1.0, 1.0)
                blk[rng.integers(32)] = 448.0 * (1 if rng.random() < 0.5 else -1)
                v[32 * b:32 * b + 32, c] = blk * 2.0 ** s
    else:
        return _exact_along((C, R), 0, rng, scales).T.copy()
    return v


def _q(v, axis):
    """The oracle's MX round trip along `axis` (blocks of 32)."""
    if axis == 1:
        c, s = oracle.mx_quantize_rows(v)
        return oracle.mx_dequantize_rows(c, s)
    c, s = oracle.mx_quantize_cols_grouped(v, np.array([0, v.shape[0]]))
    return oracle.mx_dequantize_cols(c, s)


def _check_exact(v, k_axis):
    """v is unchanged by quantising along k_axis and changed along the other."""
    np.testing.assert_array_equal(_q(v, k_axis), v)
    assert np.any(_q(v, 1 - k_axis) != v), "operand is exact along both axes: pin has no teeth"


def test_gemm1_fwd_quantises_x_along_d_and_weights_down_d():
    rng = np.random.default_rng(10)
    M, d, F = 64, 96, 64
    Xe = _exact_along((M, d), 1, rng)
    W1, W3 = _exact_along((d, F), 0, rng), _exact_along((d, F), 0, rng)
    for v, ax in ((Xe, 1), (W1, 0), (W3, 0)):
        _check_exact(v, ax)
    H1, H3 = oracle.gemm1_fwd(Xe, W1, W3, mx=True)
    np.testing.assert_array_equal(H1, Xe @ W1)
    np.testing.assert_array_equal(H3, Xe @ W3)


def test_gemm2_fwd_quantises_h_along_F_and_W2_down_F():
    rng = np.random.default_rng(11)
    M, F, d = 64, 96, 64
    he, W2 = _exact_along((M, F), 1, rng), _exact_along((F, d), 0, rng)
    _check_exact(he, 1); _check_exact(W2, 0)
    np.testing.assert_array_equal(oracle.gemm2_fwd(he, W2, mx=True), he @ W2)


def test_gemm2_dgrad_quantises_dY_and_W2_along_d():
    rng = np.random.default_rng(12)
    M, F, d = 64, 64, 96
    dYe, W2 = _exact_along((M, d), 1, rng), _exact_along((F, d), 1, rng)
    _check_exact(dYe, 1); _check_exact(W2, 1)
    np.testing.assert_array_equal(oracle.gemm2_dgrad(dYe, W2, mx=True), dYe @ W2.T)


def test_gemm2_wgrad_quantises_h_and_dY_down_the_group_rows():
    rng = np.random.default_rng(13)
    M, F, d = 96, 64, 64
    he, dYe = _exact_along((M, F), 0, rng), _exact_along((M, d), 0, rng)
    _check_exact(he, 0); _check_exact(dYe, 0)
    np.testing.assert_array_equal(oracle.gemm2_wgrad(he, dYe, mx=True), he.T @ dYe)


def test_gemm1_dgrad_quantises_dA_and_weights_along_F():
    rng = np.random.default_rng(14)
    M, F, d = 64, 96, 64
    dA1, dA3 = _exact_along((M, F), 1, rng), _exact_along((M, F), 1, rng)
    W1, W3 = _exact_along((d, F), 1, rng), _exact_along((d, F), 1, rng)
    for v in (dA1, dA3, W1, W3):
        _check_exact(v, 1)
    np.testing.assert_array_equal(oracle.gemm1_dgrad(dA1, dA3, W1, W3, mx=True),
                                  dA1 @ W1.T + dA3 @ W3.T)


def test_gemm1_wgrad_quantises_x_and_dA_down_the_group_rows():
    rng = np.random.default_rng(15)
    M, F, d = 96, 64, 64
    Xe = _exact_along((M, d), 0, rng)
    dA1, dA3 = _exact_along((M, F), 0, rng), _exact_along((M, F), 0, rng)
    for v in (Xe, dA1, dA3):
        _check_exact(v, 0)
    dW1, dW3 = oracle.gemm1_wgrad(Xe, dA1, dA3, mx=True)
    np.testing.assert_array_equal(dW1, Xe.T @ dA1)
    np.testing.assert_array_equal(dW3, Xe.T @ dA3)


def test_exact_operands_along_the_wrong_axis_are_not_exact_products():
    """The converse: operands exact only along the other axis give an MX
    product that differs from the fp64 one (so the pins above would catch
    an oracle that quantised along the wrong axis)."""
    rng = np.random.default_rng(16)
    he, W2 = _exact_along((64, 96), 0, rng), _exact_along((96, 64), 1, rng)
    assert np.any(oracle.gemm2_fwd(he, W2, mx=True) != he @ W2)


# --------------------------------------------------------------------------
# brute-force pin of the whole MX layer, GEMM by GEMM
# --------------------------------------------------------------------------

def _bf16(v):
    return torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()


def _brute_block(blk):
    """Dequantised MX block: scale 2^s with s = floor(log2 amax) - 8
    (clamped to [-127, 127]; zero block -> 2^-127), each element the nearest
    E4M3 value of v / 2^s (equal distance -> even code, beyond 448 -> 448)."""
    amax = float(np.max(np.abs(blk)))
    if amax == 0.0:
        return np.zeros_like(blk)
    _, ex = math.frexp(amax)            # amax = m 2^ex, m in [0.5, 1)
    s = min(127, max(-127, (ex - 1) - 8))
    q = np.minimum(np.abs(blk) / 2.0 ** s, 448.0)
    dist = np.abs(q[:, None] - _POS_VAL[None, :])
    best = dist == dist.min(axis=1, keepdims=True)
    even = best & (_POS[None, :] % 2 == 0)
    pick = np.where(even.any(1), np.argmax(even, 1), np.argmax(best, 1))
    return np.copysign(_POS_VAL[pick], blk) * 2.0 ** s


def _brute_q(v, axis):
    """Blocks of 32 along `axis` of v (rows or columns), each on its own."""
    v = np.asarray(v, np.float64)
    out = np.empty_like(v)
    if axis == 1:
        for r in range(v.shape[0]):
            for c in range(0, v.shape[1], 32):
                out[r, c:c + 32] = _brute_block(v[r, c:c + 32])
    else:
        for c in range(v.shape[1]):
            for r in range(0, v.shape[0], 32):
                out[r:r + 32, c] = _brute_block(v[r:r + 32, c])
    return out


def _brute_gemm(a, b):
    """a [M, K] @ b [K, N] with a quantised along its rows and b down its
    columns, both in blocks of 32 along K."""
    return _brute_q(a, 1) @ _brute_q(b, 0)


def _close(got, want, what):
    scale = max(float(np.max(np.abs(want))), 1e-300)
    err = float(np.max(np.abs(got - want))) / scale
    assert err <= 1e-12, f"{what}: rel err {err:.3e}"


def test_mx_layer_every_gemm_against_brute_force_quantisation():
    """Forward and backward of a tiny MX layer (router mode, ragged groups
    padded to 32 rows): each GEMM output against the brute-force GEMM of
    its own inputs, each operand quantised along that GEMM's K after the
    device's bf16 rounding (h, dY, the saved H1/H3, dh and dA are stored in
    bf16 first; x and the weights are bf16 inputs)."""
    rng = np.random.default_rng(20)
    T, d, E, F, k = 72, 64, 4, 64, 2
    f = lambda a: _bf16(a)   # noqa: E731  (inputs are bf16 numbers)
    x = f(rng.normal(size=(T, d)))
    W1 = f(rng.normal(size=(E, d, F)) * 0.2)
    W3 = f(rng.normal(size=(E, d, F)) * 0.2)
    W2 = f(rng.normal(size=(E, F, d)) * 0.2)
    Wr = rng.normal(size=(d, E))
    dout = f(rng.normal(size=(T, d)))
    bias = np.array([2.0, 0.5, 0.0, -3.0])        # uneven loads: groups of 64 and 32 rows
    ctx = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, bias=bias, align=32, mx=True)
    g = oracle.layer_backward(ctx, dout)
    poff, dst = ctx["meta"]["poff"], ctx["meta"]["dst"]
    assert len(set(np.diff(poff).tolist())) > 1       # groups of different sizes

    # dY: gate-scaled dout rows rounded to bf16, pad rows zero
    dY = np.zeros_like(g["dY"])
    for j in range(k):
        dY[dst[:, j]] = _bf16(ctx["gates"][:, j:j + 1] * dout)
    np.testing.assert_array_equal(g["dY"], dY)

    for e in range(E):
        a, b = int(poff[e]), int(poff[e + 1])
        if a == b:
            continue
        Xe, H1, H3 = ctx["Xp"][a:b], ctx["H1"][a:b], ctx["H3"][a:b]
        _close(H1, _brute_gemm(Xe, W1[e]), "GEMM1 H1")
        _close(H3, _brute_gemm(Xe, W3[e]), "GEMM1 H3")
        he = _bf16(H1 / (1.0 + np.exp(-H1)) * H3)
        _close(ctx["Y"][a:b], _brute_gemm(he, W2[e]), "GEMM2")
        dYe = dY[a:b]
        dh = g["dh"][a:b]
        _close(dh, _bf16(_brute_gemm(dYe, W2[e].T)), "GEMM2 dgrad (bf16 output)")
        _close(g["dW2"][e], _brute_gemm(he.T, dYe), "GEMM2 wgrad")
        # SwiGLU backward from the stored H1/H3, result stored in bf16
        z, u = _bf16(H1), _bf16(H3)
        sg = 1.0 / (1.0 + np.exp(-z))
        dA1 = _bf16(dh * u * sg * (1.0 + z * (1.0 - sg)))
        dA3 = _bf16(dh * z * sg)
        _close(g["dA1"][a:b], dA1, "dA1")
        _close(g["dA3"][a:b], dA3, "dA3")
        _close(g["dXp"][a:b], _brute_gemm(dA1, W1[e].T) + _brute_gemm(dA3, W3[e].T),
               "GEMM1 dgrad")
        _close(g["dW1"][e], _brute_gemm(Xe.T, dA1), "GEMM1 wgrad W1")
        _close(g["dW3"][e], _brute_gemm(Xe.T, dA3), "GEMM1 wgrad W3")


def test_brute_force_quantiser_matches_torch_fp8_conversion():
    """The test's own quantiser agrees with torch's float8_e4m3fn rounding
    (nearest, ties to even) on the scaled values of random blocks that stay
    below 448 after scaling."""
    rng = np.random.default_rng(21)
    v = _bf16(rng.normal(size=(16, 64)) * np.exp(rng.normal(size=(16, 1)) * 3))
    got = _brute_q(v, 1)
    for r in range(16):
        for c in range(0, 64, 32):
            blk = v[r, c:c + 32]
            _, ex = math.frexp(float(np.max(np.abs(blk))))
            s = ex - 1 - 8
            q = torch.tensor(np.clip(blk / 2.0 ** s, -448.0, 448.0))
            ref = q.to(torch.float8_e4m3fn).to(torch.float64).numpy() * 2.0 ** s
            np.testing.assert_array_equal(got[r, c:c + 32], ref)
