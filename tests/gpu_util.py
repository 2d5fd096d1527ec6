"""Helpers shared by the GPU parity tests (index maps and error norms only)."""
import numpy as np
import torch

import moe_inputs


def rel_err(got, ref):
    """max |got - ref| / max |ref| over the whole tensor."""
    got = np.asarray(got, np.float64); ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / (den if den > 0 else 1.0))


def f64(t):
    return moe_inputs.to_f64(t)


def np_i(t):
    return t.detach().cpu().numpy().astype(np.int64)


def scales_to_plain(sc, R, C, axis):
    """Tensor-core scale layout (library header) -> plain scales:
    axis 0: [R, C/32] (block along a row); axis 1: [R/32, C]."""
    sc = sc.detach().cpu().numpy().reshape(-1)
    K, MN = (C, R) if axis == 0 else (R, C)
    mn = np.arange(MN)[:, None]
    kb = np.arange(K // 32)[None, :]
    off = ((mn // 128) * (K // 128) + kb // 4) * 512 + (mn % 32) * 16 + ((mn // 32) % 4) * 4 + kb % 4
    v = sc[off]
    return v if axis == 0 else v.T


def plain_to_scales(plain, R, C, axis):
    """Inverse of scales_to_plain (numpy uint8 -> flat uint8 array)."""
    K, MN = (C, R) if axis == 0 else (R, C)
    p = plain if axis == 0 else plain.T
    out = np.zeros(R * C // 32, np.uint8)
    mn = np.arange(MN)[:, None]
    kb = np.arange(K // 32)[None, :]
    off = ((mn // 128) * (K // 128) + kb // 4) * 512 + (mn % 32) * 16 + ((mn // 32) % 4) * 4 + kb % 4
    out[off] = p
    return out


def cuda(a, dtype=None):
    t = torch.as_tensor(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()
