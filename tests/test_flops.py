"""The benchmark's FLOP accounting against the pages' worked examples and the
survey-level totals derived from the path's definitions."""
import json
import os

import pytest

from contextual_sparsity_lora_b200 import flops

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def test_estimator_cost_ratio_worked_example():
    g = GOLD["estimator_cost_ratio"]
    assert flops.estimator_cost_ratio(g["d_in"], g["d_out"], g["k"]) == pytest.approx(g["ratio"], abs=g["abs_tol"])


def test_dense_warmup_bound_worked_example():
    g = GOLD["dense_warmup_bound"]
    assert flops.dense_warmup_speedup_bound(g["p"], g["s"]) == pytest.approx(g["bound"], abs=g["abs_tol"])


@pytest.mark.parametrize("ratio,n_keep,tflop", [(1.0, 14336, 2.886), (0.7, 10036, 2.237),
                                                  (0.5, 7168, 1.804), (0.3, 4301, 1.371)])
def test_ffn_main_branch_totals(ratio, n_keep, tflop):
    w = flops.ffn_block(4096, 14336, 4096, 3072, n_keep, 32, 8)
    # 12 D F (T_out + T_ctx n / F)
    assert w["main"] / 1e12 == pytest.approx(tflop, abs=2e-3)
    assert w["lora"] / 1e9 == pytest.approx(43.5, abs=0.1)


def test_attention_projection_totals():
    w = flops.attn_proj_block(4096, 32, 8, 128, 4096, 3072, 512, 512, 32, 8)
    assert w["main"] / 1e12 == pytest.approx(0.430, abs=2e-3)
    dense = flops.attn_proj_block(4096, 32, 8, 128, 4096, 3072, 1024, 1024, 32, 8)
    assert dense["main"] / 1e12 == pytest.approx(0.687, abs=2e-3)


def test_factor_memory_worked_example():
    """The factors of the estimated projections (q, k, v, gate, up) of LLaMA2-7B at k = 8 in
    16-bit storage come to the page's approximate total."""
    g = GOLD["factor_memory"]
    b = flops.estimator_factor_bytes(g["n_layers"], g["projections"], g["k"], g["bytes_per_param"])
    assert b / 1e6 == pytest.approx(g["approx_mb"], rel=g["rel_tol"])
