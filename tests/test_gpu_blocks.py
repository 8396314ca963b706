"""Whole fine-tuning steps of the FFN and attention-projection blocks (every stage of the
path through the C ABI) against the fp64 oracle: small multi-tile cases with ragged
tails, the degenerate token splits, keep ratio 1, and the full LLaMA3-8B sizes on
sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks, inputs
from gpu_helpers import BF16_TOL, FP32_TOL, attn_problem, ffn_problem, rel_fro, unsigma

pytestmark = pytest.mark.gpu
DEV = "cuda"


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


def check_selection(scores_gpu, sigma_gpu, n_keep, scores_oracle):
    """Indices: bit-exact against the oracle's selection on the GPU's fp32 scores; against the
    oracle's own scores, any disagreement must sit within 1e-5 relative of the n-th score."""
    sc = scores_gpu.cpu().numpy().astype(np.float64)
    got = sigma_gpu.cpu().numpy()[:n_keep]
    np.testing.assert_array_equal(got, oracle.select_top(sc, n_keep))
    want = oracle.select_top(scores_oracle, n_keep)
    diff = np.setxor1d(got, want)
    if diff.size:
        thr = np.sort(scores_oracle)[::-1][n_keep - 1]
        assert np.all(np.abs(scores_oracle[diff] - thr) <= 1e-5 * abs(thr)), "selection differs beyond ties"


def run_ffn(T, C, D, F, r, k, ratio, seed, zero_b=False):
    p = ffn_problem(T, C, D, F, r, k, seed, zero_b=zero_b)
    blk = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, ratio, DEV)
    xg, dyg = cu(p["x"]), cu(p["dy"])
    blk.step(xg, dyg)
    torch.cuda.synchronize()
    return p, blk


def check_ffn(p, blk, ratio):
    T, C, F = blk.n_tok, blk.n_ctx, blk.F
    if blk.dense:
        idx = np.arange(F)
    elif C == 0:
        idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)   # unused: no context rows
    else:
        s_w, _ = oracle.ffn_select(p["x"], p["ctx"], (p["gate"].W_A, p["gate"].W_B), (p["up"].W_A, p["up"].W_B),
                                   ratio)
        assert rel_fro(blk.scores, s_w) < FP32_TOL
        check_selection(blk.scores, blk.sigma, blk.n_keep, s_w)
        idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    args = (p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0, idx)
    fwd = oracle.ffn_fwd(*args)
    bwd = oracle.ffn_bwd(p["x"], p["dy"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"],
                         2.0, idx, fwd=fwd)
    sig = blk.sigma
    assert rel_fro(unsigma(blk.g, sig, C), fwd["G"]) < BF16_TOL
    assert rel_fro(unsigma(blk.u, sig, C), fwd["U"]) < BF16_TOL
    assert rel_fro(unsigma(blk.h, sig, C), fwd["H"]) < BF16_TOL
    assert rel_fro(blk.y, fwd["Y"]) < BF16_TOL
    assert rel_fro(unsigma(blk.dg, sig, C), bwd["dG"]) < BF16_TOL
    assert rel_fro(unsigma(blk.du, sig, C), bwd["dU"]) < BF16_TOL
    assert rel_fro(blk.dx, bwd["dX"]) < BF16_TOL
    for n in ("g", "u", "d"):
        assert rel_fro(getattr(blk, "dA_" + n), bwd["dA_" + n]) < BF16_TOL, n
        if np.abs(bwd["dB_" + n]).max() > 0:
            assert rel_fro(getattr(blk, "dB_" + n), bwd["dB_" + n]) < BF16_TOL, n
    # output rows never depend on the index set
    dense = oracle.ffn_fwd(p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0,
                           np.arange(F))
    assert rel_fro(oracle.f64(blk.y)[C:], dense["Y"][C:]) < BF16_TOL


@pytest.mark.parametrize("T,C,D,F,ratio", [(424, 300, 512, 1000, 0.5), (424, 300, 512, 1000, 0.3),
                                            (424, 300, 512, 1000, 1.0), (200, 200, 256, 688, 0.5),
                                            (200, 0, 256, 688, 0.5), (136, 8, 264, 520, 0.05)])
def test_ffn_step_matches_oracle(T, C, D, F, ratio):
    p, blk = run_ffn(T, C, D, F, 32, 8, ratio, seed=20)
    check_ffn(p, blk, ratio)


def test_ffn_step_main_branch_only():
    """LoRA B = 0 removes the LoRA output, so the sliced main branch alone is compared."""
    p, blk = run_ffn(424, 300, 512, 1000, 32, 8, 0.5, seed=21, zero_b=True)
    check_ffn(p, blk, 0.5)


def test_tiny_fp32_config_step():
    """The tiny SwiGLU configuration (fp32 weights and activations): fp32 estimator, bf16 GEMM path."""
    cfg = inputs.TINY_FFN
    d = inputs.make_ffn_inputs(cfg, seed=0)
    perm = inputs.context_first_order(d["ctx_mask"])
    x32 = d["x"][perm]
    C = int(d["ctx_mask"].sum())
    blk = blocks.FFNBlock(d["gate"], d["up"], d["down"], d["lora_gate"], d["lora_up"], d["lora_down"],
                          cfg.lora_scale, cfg.k, cfg.n_tok, C, cfg.ratio, DEV)
    blk.step(cu(x32), cu(d["dy"][perm]), x_est=cu(x32, torch.float32))
    torch.cuda.synchronize()
    ctx = np.arange(cfg.n_tok) < C
    s_w, _ = oracle.ffn_select(x32, ctx, (d["gate"].W_A, d["gate"].W_B), (d["up"].W_A, d["up"].W_B), cfg.ratio)
    assert rel_fro(blk.scores, s_w) < FP32_TOL
    check_selection(blk.scores, blk.sigma, blk.n_keep, s_w)
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    bf = lambda t: t.to(torch.bfloat16)  # the GEMM path consumes bf16 copies
    fwd = oracle.ffn_fwd(bf(x32), ctx, bf(d["gate"].W), bf(d["up"].W), bf(d["down"].W), d["lora_gate"], d["lora_up"],
                         d["lora_down"], cfg.lora_scale, idx)
    assert rel_fro(blk.y, fwd["Y"]) < BF16_TOL


def run_attn(T, C, D, hq, hkv, hd, ratio, seed, zero_b=False):
    p = attn_problem(T, C, D, hq, hkv, hd, 32, 8, seed, zero_b=zero_b)
    w, lo = p["w"], p["lora"]
    blk = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], 2.0, 8, hq, hkv,
                               hd, T, C, ratio, DEV)
    blk.step(cu(p["x"]), cu(p["x_o"]), cu(p["dy"]), cu(p["dq"]), cu(p["dk"]), cu(p["dv"]))
    torch.cuda.synchronize()
    return p, blk


def check_attn(p, blk, ratio):
    C, hq, hkv, hd = blk.n_ctx, blk.hq, blk.hkv, blk.hd
    w, lo, ctx = p["w"], p["lora"], p["ctx"]
    if blk.dense or C == 0:
        idx = {n: np.arange(blk.Dq if n in "qo" else blk.Dkv) for n in "qkvo"}
    else:
        sel = oracle.attn_select(p["x"], ctx, (w["q"].W_A, w["q"].W_B), (w["k"].W_A, w["k"].W_B),
                                 (w["v"].W_A, w["v"].W_B), hq, hkv, hd, ratio)
        assert rel_fro(blk.s_qk, sel["s_qk"]) < FP32_TOL
        assert rel_fro(blk.s_v, sel["s_v"]) < FP32_TOL
        check_selection(blk.s_qk, blk.sig_k, blk.n_keep_u, sel["s_qk"])
        check_selection(blk.s_v, blk.sig_v, blk.n_keep_u, sel["s_v"])
        u_qk = blk.sig_k.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
        u_v = blk.sig_v.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
        idx = {"q": oracle.expand_units(u_qk, hq, hkv, hd), "k": u_qk, "v": u_v,
               "o": oracle.expand_units(u_v, hq, hkv, hd)}
        np.testing.assert_array_equal(blk.sig_q.cpu().numpy()[: len(idx["q"])], idx["q"])
        np.testing.assert_array_equal(blk.sig_o.cpu().numpy()[: len(idx["o"])], idx["o"])
    outs = {"q": blk.q, "k": blk.kk, "v": blk.vv}
    for n in "qkv":
        want = oracle.sparse_linear_fwd(p["x"], w[n].W, *lo[n], 2.0, ctx, idx[n], "out")
        assert rel_fro(outs[n], want) < BF16_TOL, n
    y = oracle.sparse_linear_fwd(p["x_o"], w["o"].W, *lo["o"], 2.0, ctx, idx["o"], "in")
    assert rel_fro(blk.y, y) < BF16_TOL
    dxo, dAo, dBo = oracle.sparse_linear_bwd(p["x_o"], p["dy"], w["o"].W, *lo["o"], 2.0, ctx, idx["o"], "in")
    assert rel_fro(blk.dx_o, dxo) < BF16_TOL
    assert rel_fro(blk.dA["o"], dAo) < BF16_TOL
    assert rel_fro(blk.dB["o"], dBo) < BF16_TOL
    dx = 0
    for n, g in (("q", "dq"), ("k", "dk"), ("v", "dv")):
        dxn, dAn, dBn = oracle.sparse_linear_bwd(p["x"], p[g], w[n].W, *lo[n], 2.0, ctx, idx[n], "out")
        dx = dx + dxn
        assert rel_fro(blk.dA[n], dAn) < BF16_TOL, n
        assert rel_fro(blk.dB[n], dBn) < BF16_TOL, n
    assert rel_fro(blk.dx, dx) < BF16_TOL


@pytest.mark.parametrize("T,C,D,hq,hkv,hd,ratio", [(424, 300, 512, 8, 2, 64, 0.5), (424, 300, 512, 4, 4, 128, 0.4),
                                                    (424, 300, 512, 8, 2, 64, 1.0), (256, 256, 256, 4, 2, 64, 0.5),
                                                    (256, 0, 256, 4, 2, 64, 0.5)])
def test_attn_step_matches_oracle(T, C, D, hq, hkv, hd, ratio):
    p, blk = run_attn(T, C, D, hq, hkv, hd, ratio, seed=30)
    check_attn(p, blk, ratio)


def test_attn_step_main_branch_only():
    p, blk = run_attn(424, 300, 512, 8, 2, 64, 0.5, seed=31, zero_b=True)
    check_attn(p, blk, 0.5)
