"""Data-parallel estimator path on one GPU: the rank-local criterion statistics
(sl_svd_estimate_partials) and the scores from their sum (sl_svd_scores_from_partials).

A whole batch computed in one call, and the same batch split into two parts whose statistics
are added (what the all-reduce over two ranks does), must give the same scores and index sets
as the fp64 oracle over the whole batch; the blocks' data-parallel wiring is exercised with a
stand-in for the process group that adds a second rank's statistics."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks
from gpu_helpers import FP32_TOL, attn_problem, ffn_problem, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


def ffn_factors(p):
    wa = [cu(p["gate"].W_A), cu(p["up"].W_A)]
    wb = [cu(p["gate"].W_B), cu(p["up"].W_B)]
    return wa, wb


@pytest.mark.parametrize("T,C,D,F,k", [(424, 300, 512, 1000, 8), (4096, 3072, 4096, 14336, 8)])
def test_swiglu_partials_then_scores_equal_direct_estimate(T, C, D, F, k):
    p = ffn_problem(T, C, D, F, 32, k, seed=21)
    wa, wb = ffn_factors(p)
    x = cu(p["x"])
    ws = B.Workspace()
    direct = torch.empty(F, device=DEV)
    B.sl_svd_estimate(ws, B.SL_CRIT_SWIGLU_L2, x[:C], C, wa, wb, k, direct)
    n = B.sl_svd_partials_count(B.SL_CRIT_SWIGLU_L2, wb, k)
    assert n == F
    part = torch.empty(n, dtype=torch.float64, device=DEV)
    B.sl_svd_estimate_partials(ws, B.SL_CRIT_SWIGLU_L2, x[:C], C, wa, wb, k, part)
    sc = torch.empty(F, device=DEV)
    B.sl_svd_scores_from_partials(B.SL_CRIT_SWIGLU_L2, wb, k, part, sc)
    assert torch.equal(sc, direct)  # same sums, same root


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4)])
def test_qk_partials_then_scores_equal_direct_estimate(hq, hkv):
    T, C, D, hd, k = 424, 300, 512, 64, 8
    p = attn_problem(T, C, D, hq, hkv, hd, 32, k, seed=22)
    w = p["w"]
    wa = [cu(w[n].W_A) for n in "qkv"]
    wb = [cu(w[n].W_B) for n in "qkv"]
    x = cu(p["x"])
    ws = B.Workspace()
    nu = hkv * hd
    s_qk, s_v = torch.empty(nu, device=DEV), torch.empty(nu, device=DEV)
    B.sl_svd_estimate(ws, B.SL_CRIT_QK, x[:C], C, wa, wb, k, s_qk, scores_v=s_v, n_q_heads=hq, n_kv_heads=hkv,
                      head_dim=hd)
    n = B.sl_svd_partials_count(B.SL_CRIT_QK, wb, k)
    assert n == (3 * k) ** 2
    part = torch.empty(n, dtype=torch.float64, device=DEV)
    B.sl_svd_estimate_partials(ws, B.SL_CRIT_QK, x[:C], C, wa, wb, k, part, n_q_heads=hq, n_kv_heads=hkv,
                               head_dim=hd)
    g = part.view(3 * k, 3 * k)
    assert torch.equal(g, g.T)  # a Gram matrix
    a_qk, a_v = torch.empty(nu, device=DEV), torch.empty(nu, device=DEV)
    B.sl_svd_scores_from_partials(B.SL_CRIT_QK, wb, k, part, a_qk, scores_v=a_v, n_q_heads=hq, n_kv_heads=hkv,
                                  head_dim=hd)
    assert torch.equal(a_qk, s_qk) and torch.equal(a_v, s_v)


def test_two_rank_split_matches_the_whole_batch_oracle():
    """Context rows split over two 'ranks' (unequal, ragged parts): the summed statistics give
    the oracle's scores and index sets over all context rows."""
    T, C, D, F, k = 424, 300, 512, 1000, 8
    p = ffn_problem(T, C, D, F, 32, k, seed=23)
    wa, wb = ffn_factors(p)
    x = cu(p["x"])
    ws = B.Workspace()
    c1 = 136
    parts = []
    for lo, hi in ((0, c1), (c1, C)):
        t = torch.empty(F, dtype=torch.float64, device=DEV)
        B.sl_svd_estimate_partials(ws, B.SL_CRIT_SWIGLU_L2, x[lo:hi], hi - lo, wa, wb, k, t)
        parts.append(t)
    total = parts[0] + parts[1]
    sc = torch.empty(F, device=DEV)
    B.sl_svd_scores_from_partials(B.SL_CRIT_SWIGLU_L2, wb, k, total, sc)
    s_w, idx_w = oracle.ffn_select(p["x"], p["ctx"], (p["gate"].W_A, p["gate"].W_B), (p["up"].W_A, p["up"].W_B),
                                   0.5)
    assert rel_fro(sc, s_w) < FP32_TOL
    nk = B.sl_keep_count(0.5, F)
    sig = torch.empty(F, dtype=torch.int32, device=DEV)
    B.sl_select_channels(sc, nk, sig)
    np.testing.assert_array_equal(sig.cpu().numpy()[:nk], oracle.select_top(sc.cpu().numpy().astype(np.float64), nk))

    # attention: the Gram matrices of the parts add up
    hq, hkv, hd = 8, 2, 64
    pa = attn_problem(T, C, D, hq, hkv, hd, 32, k, seed=24)
    wa3 = [cu(pa["w"][n].W_A) for n in "qkv"]
    wb3 = [cu(pa["w"][n].W_B) for n in "qkv"]
    xa = cu(pa["x"])
    grams = []
    for lo, hi in ((0, c1), (c1, C)):
        t = torch.empty((3 * k) ** 2, dtype=torch.float64, device=DEV)
        B.sl_svd_estimate_partials(ws, B.SL_CRIT_QK, xa[lo:hi], hi - lo, wa3, wb3, k, t, n_q_heads=hq,
                                   n_kv_heads=hkv, head_dim=hd)
        grams.append(t)
    nu = hkv * hd
    s_qk, s_v = torch.empty(nu, device=DEV), torch.empty(nu, device=DEV)
    B.sl_svd_scores_from_partials(B.SL_CRIT_QK, wb3, k, grams[0] + grams[1], s_qk, scores_v=s_v, n_q_heads=hq,
                                  n_kv_heads=hkv, head_dim=hd)
    want = oracle.attn_select(pa["x"], pa["ctx"], *((pa["w"][n].W_A, pa["w"][n].W_B) for n in "qkv"), hq, hkv, hd,
                              0.5)
    assert rel_fro(s_qk, want["s_qk"]) < FP32_TOL
    assert rel_fro(s_v, want["s_v"]) < FP32_TOL


def test_rank_without_context_rows_contributes_zero():
    F, k = 1000, 8
    p = ffn_problem(64, 0, 512, F, 32, k, seed=25)
    wa, wb = ffn_factors(p)
    x = cu(p["x"])
    t = torch.full((F,), 7.0, dtype=torch.float64, device=DEV)
    B.sl_svd_estimate_partials(B.Workspace(), B.SL_CRIT_SWIGLU_L2, x[:0], 0, wa, wb, k, t)
    assert torch.count_nonzero(t).item() == 0


class _SecondRank:
    """Stands in for a two-rank process group: all_reduce adds what the other rank would
    contribute (its criterion statistics; ones for the gradients)."""

    world = 2
    active = True

    def __init__(self, other_stats, other_grad):
        self.other = other_stats
        self.other_grad = other_grad
        self.calls = []

    def all_reduce(self, t):
        self.calls.append((t.dtype, t.numel()))
        if t.dtype == torch.float64:
            t += self.other
        else:
            t += self.other_grad


def test_ffn_block_data_parallel_wiring():
    """FFNBlock with a data-parallel group: its selection is the oracle's over both ranks'
    context rows, and its gradients pass through one all-reduce after the backward."""
    T, C, D, F, r, k = 424, 300, 512, 1000, 32, 8
    p = ffn_problem(T, C, D, F, r, k, seed=26)
    q = ffn_problem(T, C, D, F, r, k, seed=27)  # the other rank's batch (same weights below)
    wa, wb = ffn_factors(p)
    other = torch.empty(F, dtype=torch.float64, device=DEV)
    B.sl_svd_estimate_partials(B.Workspace(), B.SL_CRIT_SWIGLU_L2, cu(q["x"])[:C], C, wa, wb, k, other)
    dp = _SecondRank(other, 1.0)
    dp0 = _SecondRank(other, 0.0)
    blk = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5, DEV, dp=dp)
    own = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5, DEV, dp=dp0)
    x, dy = cu(p["x"]), cu(p["dy"])
    blk.step(x, dy)
    own.step(x, dy)
    torch.cuda.synchronize()
    assert dp.calls == [(torch.float64, F), (torch.float32, blk.grads.flat.numel())]
    X2 = np.concatenate([oracle.f64(p["x"])[:C], oracle.f64(q["x"])[:C]])
    s_w, idx_w = oracle.ffn_select(X2, np.ones(2 * C, dtype=bool), (p["gate"].W_A, p["gate"].W_B),
                                   (p["up"].W_A, p["up"].W_B), 0.5)
    assert rel_fro(blk.scores, s_w) < FP32_TOL
    nk = blk.n_keep
    np.testing.assert_array_equal(blk.sigma.cpu().numpy()[:nk],
                                  oracle.select_top(blk.scores.cpu().numpy().astype(np.float64), nk))
    # both blocks chose the union's channels; the gradients left the step summed with the
    # other rank's (here: ones)
    assert torch.equal(blk.sigma, own.sigma)
    assert rel_fro(blk.grads.flat - 1.0, own.grads.flat) < 1e-5
