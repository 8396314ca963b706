"""Criterion variants of the criterion ablation (Table 10 of the walkthrough): the Wanda-style
FFN criterion, head-level QK selection and random selection, through the C ABI and through the
blocks, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks
from gpu_helpers import BF16_TOL, FP32_TOL, attn_problem, ffn_problem, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


@pytest.mark.parametrize("C,D,F", [(300, 512, 1000), (97, 264, 72), (3072, 4096, 14336)])
def test_wanda_scores_match_oracle(C, D, F):
    p = ffn_problem(C + 16, C, D, F, 8, 8, seed=31)
    x = cu(p["x"])
    wg, wu = cu(p["gate"].W), cu(p["up"].W)
    sc = torch.empty(F, device=DEV)
    B.sl_wanda_scores(B.Workspace(), x[:C], C, [wg, wu], sc)
    want = oracle.wanda_scores(oracle.f64(x)[:C], [wg, wu])
    assert rel_fro(sc, want) < FP32_TOL
    # one weight: its own term
    s1 = torch.empty(F, device=DEV)
    B.sl_wanda_scores(B.Workspace(), x[:C], C, [wg], s1)
    assert rel_fro(s1, oracle.wanda_scores(oracle.f64(x)[:C], [wg])) < FP32_TOL


@pytest.mark.parametrize("hkv,hd,hpg,keep", [(8, 128, 4, 4), (8, 128, 4, 1), (40, 128, 1, 16), (5, 3, 2, 5)])
def test_select_heads_bit_exact(hkv, hd, hpg, keep):
    rng = np.random.default_rng(hkv * 100 + keep)
    s = rng.random(hkv * hd).astype(np.float32)
    s[rng.random(s.size) < 0.02] = np.nan
    if hkv > 2:  # two heads with equal sums: ties go to the lower head
        s[hd:2 * hd] = s[2 * hd:3 * hd]
    sc = torch.tensor(s, device=DEV)
    sig_k = torch.empty(hkv * hd, dtype=torch.int32, device=DEV)
    sig_q = torch.empty(hkv * hpg * hd, dtype=torch.int32, device=DEV)
    B.sl_select_heads(sc, hkv, hd, keep, sig_k, hpg, sig_q)
    # head sums as the kernel forms them (fp64 over the fp32 scores, then fp32)
    h = np.array([np.float32(np.sum(s[g * hd:(g + 1) * hd].astype(np.float64))) for g in range(hkv)])
    heads = oracle.select_top(h.astype(np.float64), keep)
    units = (heads[:, None] * hd + np.arange(hd)[None, :]).reshape(-1)
    got_k = sig_k.cpu().numpy()
    np.testing.assert_array_equal(got_k[: keep * hd], units)
    np.testing.assert_array_equal(got_k[keep * hd:], oracle.complement(units, hkv * hd))
    got_q = sig_q.cpu().numpy()
    qch = oracle.expand_units(units, hkv * hpg, hkv, hd)
    np.testing.assert_array_equal(got_q[: keep * hpg * hd], qch)
    np.testing.assert_array_equal(got_q[keep * hpg * hd:], oracle.complement(qch, hkv * hpg * hd))
    # with finite scores the oracle's own head-level selection agrees
    if not np.isnan(s).any():
        np.testing.assert_array_equal(units, oracle.select_heads(s, hkv, hd, keep))


def test_ffn_block_wanda_criterion_step():
    T, C, D, F, r, k = 424, 300, 512, 1000, 32, 8
    p = ffn_problem(T, C, D, F, r, k, seed=32)
    blk = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5, DEV,
                          criterion="wanda")
    x, dy = cu(p["x"]), cu(p["dy"])
    blk.step(x, dy)
    torch.cuda.synchronize()
    want = oracle.wanda_scores(oracle.f64(p["x"])[:C], [blk.Wg, blk.Wu])
    assert rel_fro(blk.scores, want) < FP32_TOL
    nk = blk.n_keep
    idx = blk.sigma.cpu().numpy()[:nk].astype(np.int64)
    np.testing.assert_array_equal(idx, oracle.select_top(blk.scores.cpu().numpy().astype(np.float64), nk))
    fwd = oracle.ffn_fwd(p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0, idx)
    assert rel_fro(blk.y, fwd["Y"]) < BF16_TOL


def test_ffn_block_random_criterion_is_seeded():
    T, C, D, F, r, k = 424, 300, 512, 1000, 32, 8
    p = ffn_problem(T, C, D, F, r, k, seed=33)
    mk = lambda seed: blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5,
                                      DEV, criterion="random", seed=seed)
    a, b, c = mk(7), mk(7), mk(8)
    x, dy = cu(p["x"]), cu(p["dy"])
    for blk in (a, b, c):
        blk.step(x, dy)
    torch.cuda.synchronize()
    assert torch.equal(a.sigma, b.sigma) and not torch.equal(a.sigma, c.sigma)
    sc = a.scores.cpu().numpy()
    assert sc.min() >= 0.0 and sc.max() < 1.0
    nk = a.n_keep
    np.testing.assert_array_equal(a.sigma.cpu().numpy()[:nk], oracle.select_top(sc.astype(np.float64), nk))
    idx = a.sigma.cpu().numpy()[:nk].astype(np.int64)
    fwd = oracle.ffn_fwd(p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0, idx)
    assert rel_fro(a.y, fwd["Y"]) < BF16_TOL


@pytest.mark.parametrize("qk,vo", [("head", "l2"), ("random", "random"), ("channel", "random")])
def test_attn_block_criterion_variants_step(qk, vo):
    T, C, D, hq, hkv, hd, r, k = 424, 300, 512, 8, 2, 64, 32, 8
    p = attn_problem(T, C, D, hq, hkv, hd, r, k, seed=34)
    w, lo = p["w"], p["lora"]
    blk = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], 2.0, k, hq, hkv,
                               hd, T, C, 0.5, DEV, qk_criterion=qk, vo_criterion=vo, seed=3)
    x, xo = cu(p["x"]), cu(p["x_o"])
    blk.step(x, xo, cu(p["dy"]), cu(p["dq"]), cu(p["dk"]), cu(p["dv"]))
    torch.cuda.synchronize()
    s_qk = blk.s_qk.cpu().numpy().astype(np.float64)
    if qk == "head":
        sel = oracle.attn_select(p["x"], p["ctx"], *((w[n].W_A, w[n].W_B) for n in "qkv"), hq, hkv, hd, 0.5)
        assert rel_fro(blk.s_qk, sel["s_qk"]) < FP32_TOL
        nk = blk.n_keep_heads * hd
        h = np.array([np.float32(np.sum(blk.s_qk.cpu().numpy()[g * hd:(g + 1) * hd].astype(np.float64)))
                      for g in range(hkv)])
        heads = oracle.select_top(h.astype(np.float64), blk.n_keep_heads)
        units = (heads[:, None] * hd + np.arange(hd)[None, :]).reshape(-1)
    else:
        nk = blk.n_keep_qk
        units = oracle.select_top(s_qk, nk)
    np.testing.assert_array_equal(blk.sig_k.cpu().numpy()[:nk], units)
    idx_q = oracle.expand_units(units, hq, hkv, hd)
    np.testing.assert_array_equal(blk.sig_q.cpu().numpy()[: nk * (hq // hkv)], idx_q)
    q_want = oracle.sparse_linear_fwd(p["x"], w["q"].W, *lo["q"], 2.0, p["ctx"], idx_q, "out")
    assert rel_fro(blk.q, q_want) < BF16_TOL
