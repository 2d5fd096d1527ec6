"""Pins of the oracle's MX (E4M3 + E8M0, 32-element block) quantiser:
hand-derived encodings and scales, an exhaustive sweep of every finite bf16
value against a brute-force nearest-code search over the decode table,
exactly representable blocks, and the layout relation between the row- and
column-blocked forms."""
import os

import numpy as np
import torch

import oracle
from oracle import mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("#") or not line.strip():
            continue
        yield line.split()


def test_e4m3_golden_cases():
    n = 0
    for val, code, *_ in _rows("mx_e4m3_cases.txt"):
        got = int(mx.e4m3_encode(np.array([float(val)]))[0])
        assert got == int(code, 16), (val, hex(got), code)
        n += 1
    assert n >= 20


def test_scale_golden_cases():
    for amax, byte, *_ in _rows("mx_scale_cases.txt"):
        s = int(mx.mx_scale_exponent(np.array([float(amax)]))[0])
        assert s + 127 == int(byte), (amax, s + 127, byte)


def test_decode_table_structure():
    t = mx.e4m3_decode_table()
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    fin = np.isfinite(t)
    assert fin.sum() == 254
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)                 # codes 0..126 increase
    np.testing.assert_array_equal(t[0x80:0xFF], -pos)


def _brute_encode(q):
    """Nearest finite code by exhaustive search; equal distance -> even code;
    beyond 448 -> 448; sign from q."""
    t = mx.e4m3_decode_table()
    codes = np.arange(0x7F)                         # non-negative finite codes
    vals = t[codes]
    a = np.minimum(np.abs(q), 448.0)
    dist = np.abs(a[:, None] - vals[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among tied candidates prefer the one with an even code
    even = cand & (codes[None, :] % 2 == 0)
    pick = np.where(even.any(1), np.argmax(even, 1), np.argmax(cand, 1))
    out = codes[pick] | np.where(np.signbit(q), 0x80, 0)
    return out.astype(np.uint8)


def test_e4m3_encode_exhaustive_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    v = f[np.isfinite(f)].astype(np.float64)
    v = v[np.abs(v) < 2.0 ** 12]                    # includes the saturating range
    np.testing.assert_array_equal(mx.e4m3_encode(v), _brute_encode(v))


def test_every_bf16_value_in_a_unit_amax_block():
    """Each finite bf16 value v with |v| <= 1 placed in a block whose amax
    is 1 (scale 2^-8): the code is the brute-force code of 256 v."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    v = f[np.isfinite(f)].astype(np.float64)
    v = v[np.abs(v) <= 1.0]
    n = (len(v) + 30) // 31
    pad = np.zeros(n * 31 - len(v))
    body = np.concatenate([v, pad]).reshape(n, 31)
    blocks = np.concatenate([np.ones((n, 1)), body], axis=1)      # amax = 1
    codes, scales = mx.mx_quantize_rows(blocks)
    assert np.all(scales == 119)
    np.testing.assert_array_equal(codes[:, 1:].reshape(-1)[:len(v)], _brute_encode(256.0 * v))


def test_random_blocks_against_direct_rule():
    rng = np.random.default_rng(0)
    v = rng.normal(size=(64, 256)) * np.exp(rng.normal(size=(64, 1)) * 4)
    v = torch.tensor(v).to(torch.bfloat16).to(torch.float64).numpy()
    codes, scales = mx.mx_quantize_rows(v)
    for r in range(v.shape[0]):
        for b in range(v.shape[1] // 32):
            blk = v[r, 32 * b:32 * b + 32]
            amax = np.max(np.abs(blk))
            e = int(np.floor(np.log2(amax)))       # fine for normal amax
            s = max(-127, min(127, e - 8))
            assert scales[r, b] == s + 127
            np.testing.assert_array_equal(codes[r, 32 * b:32 * b + 32], _brute_encode(blk / 2.0 ** s))


def test_exactly_representable_block_round_trips():
    t = mx.e4m3_decode_table()
    rng = np.random.default_rng(1)
    for s in (-20, -8, 0, 5, 40):
        c = rng.integers(0, 0x7F, size=(8, 32))
        c[:, 0] = 0x7E                              # amax = 448 * 2^s -> scale 2^s
        sign = np.where(rng.random((8, 32)) < 0.5, -1.0, 1.0)
        v = sign * t[c] * 2.0 ** s
        codes, scales = mx.mx_quantize_rows(v)
        assert np.all(scales == s + 127)
        np.testing.assert_array_equal(mx.mx_dequantize_rows(codes, scales), v)


def test_zero_block_and_error_bound():
    v = np.zeros((2, 64)); v[1, 32:] = np.linspace(-3, 3, 32)
    codes, scales = mx.mx_quantize_rows(v)
    assert scales[0].tolist() == [0, 0] and scales[1, 0] == 0
    assert np.all(codes[0] == 0)
    # relative error of a normal-range element is at most half a mantissa step
    rng = np.random.default_rng(2)
    w = rng.normal(size=(128, 128))
    c, s = mx.mx_quantize_rows(w)
    back = mx.mx_dequantize_rows(c, s)
    X = np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32, axis=1)
    normal = np.abs(w) >= X * 2.0 ** -6
    sat = np.abs(w) > X * 448.0        # the rule saturates (448, 512) * X to 448 X
    assert sat.sum() > 0 and np.all(back[sat] == np.sign(w[sat]) * 448.0 * X[sat])
    ok = normal & ~sat
    assert np.all(np.abs(back - w)[ok] <= np.abs(w)[ok] * 2.0 ** -4)
    assert np.all(np.abs(back - w)[~normal] <= X[~normal] * 2.0 ** -10)


def test_column_blocks_are_row_blocks_of_the_transpose():
    rng = np.random.default_rng(3)
    v = rng.normal(size=(256, 96))
    cc, sc = mx.mx_quantize_cols_grouped(v, np.array([0, 128, 256]))
    cr, sr = mx.mx_quantize_rows(v.T.copy())
    np.testing.assert_array_equal(cc, cr.T)
    np.testing.assert_array_equal(sc, sr.T)
    np.testing.assert_array_equal(mx.mx_dequantize_cols(cc, sc), mx.mx_dequantize_rows(cr, sr).T)


def _mx_exact(shape, axis_blocks_rows, rng, s=-6):
    """Values that are exact MX numbers for blocks of 32 along the chosen
    axis: E4M3 values times 2^s with a 448 * 2^s element in every block."""
    t = mx.e4m3_decode_table()
    c = rng.integers(0, 0x7F, size=shape)
    v = t[c] * np.where(rng.random(shape) < 0.5, -1.0, 1.0) * 2.0 ** s
    if axis_blocks_rows:       # blocks of 32 consecutive rows
        v[::32, :] = 448.0 * 2.0 ** s
    else:                      # blocks of 32 consecutive columns
        v[:, ::32] = 448.0 * 2.0 ** s
    return v


def test_mx_layer_first_gemm_is_exact_on_mx_exact_inputs():
    """With x exact along d and W1/W3 exact down d, the MX quantiser leaves
    GEMM1's operands unchanged, so H1/H3 of the MX layer equal the fp64 ones;
    the second GEMM then differs only by quantising h and W2."""
    rng = np.random.default_rng(4)
    T, d, E, F, k = 16, 64, 2, 64, 1
    x = _mx_exact((T, d), False, rng)
    W1 = np.stack([_mx_exact((d, F), True, rng) for _ in range(E)])
    W3 = np.stack([_mx_exact((d, F), True, rng) for _ in range(E)])
    W2 = np.stack([_mx_exact((F, d), True, rng) for _ in range(E)])
    Wr = rng.normal(size=(d, E))
    a = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=32, mx=False)
    b = oracle.layer_forward(x, W1, W3, W2, k, Wr=Wr, align=32, mx=True)
    np.testing.assert_array_equal(a["H1"], b["H1"])
    np.testing.assert_array_equal(a["H3"], b["H3"])
    err = np.max(np.abs(a["out"] - b["out"])) / np.max(np.abs(a["out"]))
    assert 0 < err < 0.1
