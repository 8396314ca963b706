"""Host-side logic of the fine-tuning step (no GPU): the per-layer keep tables, the learning-rate
schedule against the oracle's, and the per-layer weight generator's exact factors."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import inputs
from contextual_sparsity_lora_b200.model import cosine_lr, layerwise_keep, llama3_8b_math10k_keep


def test_layerwise_table():
    keep = layerwise_keep()
    assert len(keep) == 32
    assert all(k == (1.0, 1.0) for k in keep[:8])
    assert all(k == (0.6, 0.6) for k in keep[8:20])
    assert all(k == (0.35, 0.35) for k in keep[20:])


def test_math10k_table_counts():
    keep = llama3_8b_math10k_keep()
    assert sum(1 for a, f in keep if f < 1.0) == 28
    assert sum(1 for a, f in keep if a < 1.0) == 14


@pytest.mark.parametrize("n_steps,warm", [(20, 0.04), (100, 0.04), (7, 0.5), (3, 1.0)])
def test_cosine_lr_matches_oracle(n_steps, warm):
    for t in range(1, n_steps + 1):
        assert cosine_lr(t, n_steps, 3e-4, warm) == pytest.approx(oracle.cosine_lr(t, n_steps, 3e-4, warm),
                                                                  rel=1e-12, abs=1e-24)


def test_signed_permutation_keeps_spectrum_and_exact_factors():
    gen = inputs.generator(5)
    w = inputs.spectral_weight(48, 40, 0.5, 6, gen, "cpu", torch.float64, torch.float64)
    p = inputs.signed_permutation(w, gen)
    W = p.W.numpy()
    sv = np.linalg.svd(W, compute_uv=False)
    np.testing.assert_allclose(sv, w.s.numpy()[: len(sv)], rtol=1e-12)
    # W_A W_B is the rank-6 Eckart-Young truncation of the permuted weight (math convention W.T)
    U, s, Vt = np.linalg.svd(W.T)
    trunc = (U[:, :6] * s[:6]) @ Vt[:6]
    np.testing.assert_allclose(p.W_A.numpy() @ p.W_B.numpy(), trunc, atol=1e-12)
    assert not np.allclose(W, w.W.numpy())
