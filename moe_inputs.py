"""Seeded synthetic inputs for the MoE feed-forward layer.

This module only draws random numbers and lays them out; it contains none of
the layer's arithmetic.  Both the CPU oracle's tests and the CUDA path's tests
(and ``bench.py``) take their inputs from here, so the two sides see the very
same bits.

Workloads (shapes chosen for the single-GPU layer; the Olmo-core 3 and the
JUPITER/TorchTitan write-ups give the 128-expert top-4 and the 384-expert top-8
d_model=6144 settings, "Routing and compute optimisation" and "Experimental
model" sections):

===========  =====  =====  ===  ==  =====  =======  ==========================
name         T      d      E    k   F      routing  note
===========  =====  =====  ===  ==  =====  =======  ==========================
tiny         1024   256    8    2   512    router   small case, full oracle
olmo128      16384  2048   128  4   1024   router   the headline workload
olmo128_mx   16384  2048   128  4   1024   router   both GEMMs in MXFP8
skewed       16384  2048   128  4   1024   router   Zipf(1.2) logit bias
trillion     8192   6144   384  8   2048   random   random routing (stress)
===========  =====  =====  ===  ==  =====  =======  ==========================

Recipe (each tensor seeded with ``1000 * config_index + tensor_id``):
  x ~ N(0,1) rounded to bf16; W1, W3 [E,d,F] and W2 [E,F,d] ~ N(0, 0.02) in
  bf16; router W_r [d,E] ~ N(0, 0.02) fp32; upstream grad dout ~ N(0,1) bf16;
  skewed bias b_e = 3*log(rank_e^-1.2) with rank a seeded permutation of 1..E;
  random routing draws k distinct experts per token uniformly (in drawn order)
  and gates U(0,1) renormalised to sum 1 (fp32).

Large tensors are drawn with torch's seeded generator on the device that will
hold them (``torch.Generator(device)``), so a full-size workload never crosses
PCIe; a tensor drawn on a given device type with a given seed is reproducible.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    index: int
    T: int
    d: int
    E: int
    k: int
    F: int
    routing: str = "router"   # "router" | "random"
    mx: bool = False          # grouped GEMMs in MXFP8
    bias: str | None = None   # None | "zipf"
    align: int = 128

    @property
    def A(self) -> int:
        return self.T * self.k

    @property
    def A_pad_max(self) -> int:
        # every group padded up to `align` rows: at most align-1 pad rows each
        return self.T * self.k + self.E * (self.align - 1)

    def with_(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": LayerConfig("tiny", 0, 1024, 256, 8, 2, 512),
    "olmo128": LayerConfig("olmo128", 1, 16384, 2048, 128, 4, 1024),
    "olmo128_mx": LayerConfig("olmo128_mx", 2, 16384, 2048, 128, 4, 1024, mx=True),
    "skewed": LayerConfig("skewed", 3, 16384, 2048, 128, 4, 1024, bias="zipf"),
    "trillion": LayerConfig("trillion", 4, 8192, 6144, 384, 8, 2048, routing="random"),
    "trillion_mx": LayerConfig("trillion_mx", 4, 8192, 6144, 384, 8, 2048,
                               routing="random", mx=True),
}

# tensor ids (seed = 1000 * config index + id)
_X, _W1, _W3, _W2, _WR, _DOUT, _BIAS, _ROUTE = range(1, 9)


def seed_of(cfg: LayerConfig, tensor_id: int, salt: int = 0) -> int:
    return 1000 * cfg.index + tensor_id + 100000 * salt


def _normal(shape, std, seed, device, dtype):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_layer_inputs(cfg: LayerConfig, device="cpu", salt: int = 0,
                      with_weights: bool = True) -> dict:
    """All inputs of one fwd+bwd step as torch tensors on ``device``.

    Keys: x [T,d] bf16, W1/W3 [E,d,F] bf16, W2 [E,F,d] bf16, Wr [d,E] f32,
    bias [E] f32 or None, dout [T,d] bf16, and for random routing
    topk_idx [T,k] int32 and gates [T,k] f32.
    """
    dev = torch.device(device)
    s = lambda tid: seed_of(cfg, tid, salt)
    out = {
        "x": _normal((cfg.T, cfg.d), 1.0, s(_X), dev, torch.bfloat16),
        "dout": _normal((cfg.T, cfg.d), 1.0, s(_DOUT), dev, torch.bfloat16),
        "Wr": _normal((cfg.d, cfg.E), 0.02, s(_WR), dev, torch.float32),
        "bias": None,
    }
    if with_weights:
        out["W1"] = _normal((cfg.E, cfg.d, cfg.F), 0.02, s(_W1), dev, torch.bfloat16)
        out["W3"] = _normal((cfg.E, cfg.d, cfg.F), 0.02, s(_W3), dev, torch.bfloat16)
        out["W2"] = _normal((cfg.E, cfg.F, cfg.d), 0.02, s(_W2), dev, torch.bfloat16)
    if cfg.bias == "zipf":
        rng = np.random.default_rng(s(_BIAS))
        rank = rng.permutation(cfg.E) + 1
        b = 3.0 * np.log(rank.astype(np.float64) ** -1.2)
        out["bias"] = torch.from_numpy(b.astype(np.float32)).to(dev)
    if cfg.routing == "random":
        idx, gates = random_routing(cfg.T, cfg.E, cfg.k, s(_ROUTE))
        out["topk_idx"] = torch.from_numpy(idx).to(dev)
        out["gates"] = torch.from_numpy(gates).to(dev)
    return out


def random_routing(T: int, E: int, k: int, seed: int):
    """k distinct experts per token, uniform without replacement, in drawn
    order; gates U(0,1) renormalised to sum 1 (stored as fp32)."""
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E))
    idx = np.argsort(keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    u = rng.random((T, k))
    gates = (u / u.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, gates


def bf16_bits_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a bf16 tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


def to_f64(t) -> np.ndarray | None:
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t)
    return t.detach().to("cpu").numpy().astype(np.float64)


def random_bf16(shape, seed, std=1.0, device="cpu") -> torch.Tensor:
    return _normal(shape, std, seed, torch.device(device), torch.bfloat16)
