"""CPU oracle for the MoE feed-forward layer (TEST INFRASTRUCTURE ONLY).

Plain, slow, fp64 NumPy restatement of what the layer computes.  Only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it; the library never does, and it imports nothing from the library.

Sources, cited by page title and section:

* [OC3-ja]  "Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ"
  (agentlenshq.com) -- sections "ルーティングと計算の最適化" (routing kept on the
  GPU, rows written straight into the experts' input buffers, grouped GEMM),
  "MXFP8による精度最適化" (MXFP8), "実証されたスケール" (random routing).
* [OC3-hu]  "Az Ai2 megnyitotta az Olmo-core 3 MoE-tréningrendszerét"
  (aihirek.info) -- first section (8 -> 128 experts, four chosen per token).
* [JUPITER] "PyTorch、欧州の公共スパコンで約1兆パラメータMoEを訓練" (cctest.ai)
  -- model paragraph (384 experts, top-8, hidden 6144).

The pages name the steps but never write the formulas; the layer definition
this oracle follows (softmax over E, top-k with ties to the lower expert index,
gates renormalised over the chosen k, SwiGLU experts, gate-weighted sum, the
OCP MX scale rule) is the stated workload definition of the layer.

Pins (tests/test_oracle_*.py, ``-m "not gpu"``): brute-force per-token loops,
routing invariants, dense special cases (E=1,k=1 and k=E), central finite
differences for every gradient, token-permutation invariance, and for the MX
quantiser hand-derived cases plus an exhaustive bf16 sweep against a
brute-force nearest-code search.
"""
from .moe_oracle import (  # noqa: F401
    router_logits, topk_select, gates_from_logits, routing_metadata,
    permute_rows, expert_forward, combine, layer_forward, layer_backward,
    silu, round_bf16, grouped_matmul, grouped_matmul_t, grouped_wgrad, swiglu_backward,
    combine_backward, gate_logit_grad, unpermute_sum, router_backward,
    gemm1_fwd, gemm2_fwd, gemm2_dgrad, gemm2_wgrad, gemm1_dgrad, gemm1_wgrad,
)
from .mx import (  # noqa: F401
    e4m3_decode_table, e4m3_encode, mx_scale_exponent, mx_quantize_rows,
    mx_quantize_cols_grouped, mx_dequantize_rows, mx_dequantize_cols,
)
