"""fp64 oracle of one MoE feed-forward layer, forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring for the page citations
[OC3-ja], [OC3-hu], [JUPITER] and for who may import this).

Notation: T tokens, d model width, E experts, k experts per token, F expert
hidden width; A = T*k assignments.  Everything is float64 unless it is an
index.  Rounding to bf16 is NOT emulated in the BF16 path (the tolerance
covers it); the MXFP8 path quantises each GEMM operand along that GEMM's K
with the MX rule in ``oracle.mx``, rounds the tensors it quantises to bf16
first (the device stores them in bf16 before quantising), and lets the saved
H1/H3 enter the SwiGLU backward at their stored bf16 precision: quantisation
turns a one-ulp bf16 difference into a one-ulp E4M3 difference, so the MX
operands must be the same values on both sides.
"""
from __future__ import annotations

import numpy as np

from . import mx as _mx


# --------------------------------------------------------------------------
# elementwise helpers
# --------------------------------------------------------------------------

def silu(z):
    """SiLU / swish, z * sigmoid(z), in fp64."""
    return z / (1.0 + np.exp(-z))


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def round_bf16(v):
    """Round fp64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits (7 stored).  Done on the exact binary
    significand from frexp, so it is exact for every finite input in bf16's
    normal range (inputs here never leave it)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)               # v = m * 2^e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0) / 256.0   # keep 8 significant bits, half-to-even
    return np.ldexp(r, e)


# --------------------------------------------------------------------------
# router: logits, top-k, gates   ([OC3-hu] first section: k experts chosen
# per token; [JUPITER] model paragraph: top-8 of 384)
# --------------------------------------------------------------------------

def router_logits(x, Wr, bias=None):
    """logit[t,e] = sum_i x[t,i] * Wr[i,e] (+ bias[e])."""
    L = np.asarray(x, np.float64) @ np.asarray(Wr, np.float64)
    if bias is not None:
        L = L + np.asarray(bias, np.float64)[None, :]
    return L


def topk_select(logits, k):
    """Indices of the k largest logits per token, largest first; equal
    values are ordered by the lower expert index.

    Softmax is strictly increasing, so ranking logits ranks probabilities.
    A stable sort of the negated logits keeps equal values in index order."""
    order = np.argsort(-np.asarray(logits, np.float64), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gates_from_logits(logits, idx):
    """Softmax over all E followed by renormalisation over the chosen k,
    which equals a softmax over the chosen logits alone:
    g[t,j] = exp(L[t,sel_j]) / sum_j' exp(L[t,sel_j'])."""
    Ls = np.take_along_axis(np.asarray(logits, np.float64), idx.astype(np.int64), axis=1)
    m = Ls.max(axis=1, keepdims=True)
    w = np.exp(Ls - m)
    return w / w.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# routing metadata   ([OC3-ja] "ルーティングと計算の最適化": routing metadata is
# kept on the GPU; token rows are written straight into each expert's input
# buffer)
# --------------------------------------------------------------------------

def routing_metadata(idx, E, align=128):
    """Counting sort of the T*k assignments by expert, stable in token order.

    counts[e]   number of assignments to expert e
    offsets     exclusive scan of counts (length E+1)
    poff        exclusive scan of counts rounded up to `align` (length E+1):
                group e occupies rows [poff[e], poff[e+1]) of the permuted
                buffer, real rows first, then zero pad rows
    dst[t,j]    row of assignment (t,j): poff[e] + #{t' < t : e chosen by t'}
    src[r]      token of permuted row r, -1 for pad rows (length poff[E])
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = np.zeros(E, np.int64)
    for t in range(T):
        for j in range(k):
            counts[int(idx[t, j])] += 1
    offsets = np.zeros(E + 1, np.int64)
    poff = np.zeros(E + 1, np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
        padded = -(-counts[e] // align) * align
        poff[e + 1] = poff[e] + padded
    seen = np.zeros(E, np.int64)
    dst = np.zeros((T, k), np.int64)
    src = np.full(int(poff[E]), -1, np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            r = poff[e] + seen[e]
            seen[e] += 1
            dst[t, j] = r
            src[r] = t
    return dict(counts=counts, offsets=offsets, poff=poff, dst=dst, src=src,
                E=E, align=align)


def permute_rows(x, meta):
    """Expert-contiguous input buffer: Xp[dst[t,j]] = x[t], pad rows zero."""
    x = np.asarray(x, np.float64)
    src = meta["src"]
    Xp = np.zeros((len(src), x.shape[1]), np.float64)
    real = src >= 0
    Xp[real] = x[src[real]]
    return Xp


# --------------------------------------------------------------------------
# expert MLPs as grouped GEMMs ([OC3-ja]: many small per-expert matmuls
# batched into one grouped GEMM); SwiGLU experts: h = silu(x W1) * (x W3),
# y = h W2
# --------------------------------------------------------------------------

def _q_rows(v):
    """MX round trip with 32-element blocks along the last axis."""
    c, s = _mx.mx_quantize_rows(v)
    return _mx.mx_dequantize_rows(c, s)


def _q_cols(v):
    """MX round trip with 32-row blocks along the first axis."""
    c, s = _mx.mx_quantize_cols_grouped(v, np.array([0, v.shape[0]]))
    return _mx.mx_dequantize_cols(c, s)


def _gemm(a, b, mx, a_blocks_along, b_blocks_along):
    """a @ b in fp64; in MX mode each operand first goes through the MX
    quantiser along the shared K axis ('rows' = blocks along the last axis,
    'cols' = blocks of 32 rows)."""
    if mx:
        a = _q_rows(a) if a_blocks_along == "rows" else _q_cols(a)
        b = _q_rows(b) if b_blocks_along == "rows" else _q_cols(b)
    return a @ b


# The six expert GEMMs of one group ([OC3-ja] "MXFP8による精度最適化": the
# expert feed-forward matmuls run in MXFP8).  In MX mode each operand is
# quantised in blocks of 32 along that GEMM's reduction axis K: for a
# row-major a [M, K] that is along its rows ('rows'), for b [K, N] down its
# columns ('cols').  Xe, he, dYe, dA1, dA3 are the group's rows.

def gemm1_fwd(Xe, W1e, W3e, mx=False):
    """H1 = Xe W1e, H3 = Xe W3e; K = d."""
    return _gemm(Xe, W1e, mx, "rows", "cols"), _gemm(Xe, W3e, mx, "rows", "cols")


def gemm2_fwd(he, W2e, mx=False):
    """Y = he W2e; K = F."""
    return _gemm(he, W2e, mx, "rows", "cols")


def gemm2_dgrad(dYe, W2e, mx=False):
    """dh = dYe W2e^T; K = d."""
    return _gemm(dYe, W2e.T, mx, "rows", "cols")


def gemm2_wgrad(he, dYe, mx=False):
    """dW2e = he^T dYe; K = the group's rows (blocks of 32 rows from the
    group's first row)."""
    return _gemm(he.T, dYe, mx, "rows", "cols")


def gemm1_dgrad(dA1, dA3, W1e, W3e, mx=False):
    """dXe = dA1 W1e^T + dA3 W3e^T, i.e. [dA1 | dA3] [W1e | W3e]^T; K = 2F
    (F is a multiple of 32, so no block straddles the two halves)."""
    return _gemm(dA1, W1e.T, mx, "rows", "cols") + _gemm(dA3, W3e.T, mx, "rows", "cols")


def gemm1_wgrad(Xe, dA1, dA3, mx=False):
    """dW1e = Xe^T dA1, dW3e = Xe^T dA3; K = the group's rows."""
    return _gemm(Xe.T, dA1, mx, "rows", "cols"), _gemm(Xe.T, dA3, mx, "rows", "cols")


def expert_forward(Xp, W1, W3, W2, poff, mx=False):
    """Per group e (rows poff[e]..poff[e+1]): H1 = Xe W1[e], H3 = Xe W3[e],
    h = silu(H1) * H3, Y = h W2[e].  Returns (H1, H3, h, Y) over all rows."""
    A_pad = Xp.shape[0]
    E, d, F = W1.shape
    H1 = np.zeros((A_pad, F)); H3 = np.zeros((A_pad, F))
    h = np.zeros((A_pad, F)); Y = np.zeros((A_pad, W2.shape[2]))
    for e in range(E):
        a, b = int(poff[e]), int(poff[e + 1])
        if a == b:
            continue
        Xe = Xp[a:b]
        H1[a:b], H3[a:b] = gemm1_fwd(Xe, W1[e], W3[e], mx)
        h[a:b] = silu(H1[a:b]) * H3[a:b]
        he = round_bf16(h[a:b]) if mx else h[a:b]
        Y[a:b] = gemm2_fwd(he, W2[e], mx)
    return H1, H3, h, Y


def combine(Y, gates, dst):
    """out[t] = sum_j gates[t,j] * Y[dst[t,j]] (slot order j = 0..k-1)."""
    T, k = dst.shape
    out = np.zeros((T, Y.shape[1]))
    for j in range(k):
        out += gates[:, j:j + 1] * Y[dst[:, j]]
    return out


def layer_forward(x, W1, W3, W2, k, Wr=None, bias=None, topk_idx=None,
                  gates=None, logits=None, align=128, mx=False):
    """Whole forward pass.  Routing is either computed (router mode: from
    ``logits`` if given, else from x, Wr, bias) or given (``topk_idx`` and
    ``gates``, the random-routing stress workload of [OC3-ja] "実証されたスケール").
    Returns a context dict holding every intermediate."""
    x = np.asarray(x, np.float64)
    W1 = np.asarray(W1, np.float64); W3 = np.asarray(W3, np.float64)
    W2 = np.asarray(W2, np.float64)
    E = W1.shape[0]
    if topk_idx is None:
        L = router_logits(x, Wr, bias) if logits is None else np.asarray(logits, np.float64)
        idx = topk_select(L, k)
        g = gates_from_logits(L, idx)
        router = True
    else:
        L = None
        idx = np.asarray(topk_idx).astype(np.int32)
        g = np.asarray(gates, np.float64)
        router = False
    meta = routing_metadata(idx, E, align)
    Xp = permute_rows(x, meta)
    H1, H3, h, Y = expert_forward(Xp, W1, W3, W2, meta["poff"], mx=mx)
    out = combine(Y, g, meta["dst"])
    return dict(x=x, W1=W1, W3=W3, W2=W2, Wr=None if Wr is None else np.asarray(Wr, np.float64),
                logits=L, topk_idx=idx, gates=g, meta=meta, Xp=Xp, H1=H1, H3=H3,
                h=h, Y=Y, out=out, router=router, mx=mx, k=k)


def grouped_matmul(A, B, poff):
    """C[r] = A[r] @ B[e] for every row r of group e (rows poff[e]..poff[e+1])."""
    A = np.asarray(A, np.float64)
    C = np.zeros((A.shape[0], B.shape[2]))
    for e in range(B.shape[0]):
        a, b = int(poff[e]), int(poff[e + 1])
        if a < b:
            C[a:b] = A[a:b] @ np.asarray(B[e], np.float64)
    return C


def grouped_matmul_t(dC, B, poff):
    """dA[r] = dC[r] @ B[e]^T for every row r of group e."""
    dC = np.asarray(dC, np.float64)
    dA = np.zeros((dC.shape[0], B.shape[1]))
    for e in range(B.shape[0]):
        a, b = int(poff[e]), int(poff[e + 1])
        if a < b:
            dA[a:b] = dC[a:b] @ np.asarray(B[e], np.float64).T
    return dA


def grouped_wgrad(A, dC, poff, E):
    """dB[e] = A_e^T @ dC_e, summed over the rows of group e (zero if empty)."""
    A = np.asarray(A, np.float64); dC = np.asarray(dC, np.float64)
    dB = np.zeros((E, A.shape[1], dC.shape[1]))
    for e in range(E):
        a, b = int(poff[e]), int(poff[e + 1])
        if a < b:
            dB[e] = A[a:b].T @ dC[a:b]
    return dB


def swiglu_backward(dh, H1, H3):
    """h = silu(H1) * H3:  dH1 = dh * H3 * s * (1 + H1 (1 - s)),
    dH3 = dh * H1 * s, with s = sigmoid(H1)."""
    s = _sigmoid(H1)
    return dh * H3 * s * (1.0 + H1 * (1.0 - s)), dh * H1 * s


def combine_backward(dout, Y, gates, dst):
    """Backward of out[t] = sum_j g[t,j] Y[dst[t,j]]:
    dY[dst[t,j]] = g[t,j] dout[t] (other rows zero), dg[t,j] = <dout[t], Y[dst[t,j]]>."""
    dout = np.asarray(dout, np.float64)
    T, k = dst.shape
    dY = np.zeros((Y.shape[0], dout.shape[1]))
    dg = np.zeros((T, k))
    for j in range(k):
        dY[dst[:, j]] = gates[:, j:j + 1] * dout
        dg[:, j] = np.sum(dout * Y[dst[:, j]], axis=1)
    return dY, dg


def gate_logit_grad(gates, dg):
    """Gates are a softmax over the chosen logits, so the chosen logits get
    dl_j = g_j (dg_j - sum_i g_i dg_i)."""
    return gates * (dg - np.sum(gates * dg, axis=1, keepdims=True))


def unpermute_sum(dXp, dst):
    """dx[t] = sum_j dXp[dst[t,j]]."""
    T, k = dst.shape
    dx = np.zeros((T, dXp.shape[1]))
    for j in range(k):
        dx += dXp[dst[:, j]]
    return dx


def router_backward(x, Wr, idx, dl):
    """Logits L = x Wr (+ b): with dL[t, idx[t,j]] = dl[t,j] and zero
    elsewhere, dWr = x^T dL and the input gradient dL Wr^T."""
    T, k = idx.shape
    E = Wr.shape[1]
    dL = np.zeros((T, E))
    for j in range(k):
        dL[np.arange(T), idx[:, j].astype(np.int64)] += dl[:, j]
    return np.asarray(x, np.float64).T @ dL, dL @ np.asarray(Wr, np.float64).T


def layer_backward(ctx, dout):
    """Gradients of <dout, out> with respect to x, W1, W3, W2 and (router
    mode) Wr, plus the gate gradient dg.  The top-k choice is piecewise
    constant, so only the chosen logits receive gradient; the bias is a
    constant."""
    dout = np.asarray(dout, np.float64)
    mx = ctx["mx"]
    meta = ctx["meta"]; dst = meta["dst"]; poff = meta["poff"]
    g = ctx["gates"]; Y = ctx["Y"]; Xp = ctx["Xp"]
    H1, H3, h = ctx["H1"], ctx["H3"], ctx["h"]
    W1, W3, W2 = ctx["W1"], ctx["W3"], ctx["W2"]
    E = W1.shape[0]

    dY, dg = combine_backward(dout, Y, g, dst)
    if mx:
        dY = round_bf16(dY)

    dW1 = np.zeros_like(W1); dW3 = np.zeros_like(W3); dW2 = np.zeros_like(W2)
    dXp = np.zeros_like(Xp)
    dh = np.zeros_like(h); dA1 = np.zeros_like(h); dA3 = np.zeros_like(h)
    for e in range(E):
        a, b = int(poff[e]), int(poff[e + 1])
        if a == b:
            continue
        dYe = dY[a:b]
        he = round_bf16(h[a:b]) if mx else h[a:b]
        dh[a:b] = gemm2_dgrad(dYe, W2[e], mx)
        dW2[e] = gemm2_wgrad(he, dYe, mx)
        if mx:
            # an MXFP8 GEMM accumulates in fp32 and outputs bf16, dh included;
            # the saved activations enter the backward at their stored (bf16)
            # precision, and dA is stored in bf16 before it is quantised, so
            # the quantised dA operands are the device's
            dh[a:b] = round_bf16(dh[a:b])
            g1, g3 = swiglu_backward(dh[a:b], round_bf16(H1[a:b]), round_bf16(H3[a:b]))
            dA1[a:b], dA3[a:b] = round_bf16(g1), round_bf16(g3)
        else:
            dA1[a:b], dA3[a:b] = swiglu_backward(dh[a:b], H1[a:b], H3[a:b])
        dXp[a:b] = gemm1_dgrad(dA1[a:b], dA3[a:b], W1[e], W3[e], mx)
        dW1[e], dW3[e] = gemm1_wgrad(Xp[a:b], dA1[a:b], dA3[a:b], mx)

    dx = unpermute_sum(dXp, dst)
    out = dict(dx=dx, dW1=dW1, dW3=dW3, dW2=dW2, dg=dg, dY=dY, dXp=dXp, dh=dh, dA1=dA1,
               dA3=dA3)
    if ctx["router"]:
        dl = gate_logit_grad(g, dg)
        dWr, dx_r = router_backward(ctx["x"], ctx["Wr"], ctx["topk_idx"], dl)
        out["dWr"] = dWr
        out["dx"] = dx + dx_r
        out["dl"] = dl
    return out
