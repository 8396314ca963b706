"""Full model sizes: LLaMA3-8B in the launch configuration the benchmark times (8 x 512
tokens, 3072 context + 1024 output, keep ratio 0.5, GQA 32/8, estimator rank 8) and the
LLaMA2-13B layer (4 x 1024 tokens, 3072 context + 1024 output, keep ratio 0.4, MHA 40 x 128,
FFN 13824, estimator rank 16). The estimator scores and the selection are checked in full;
the row-independent outputs (g, u, h, y, dx of the FFN; q, k, v, y, dx_o, dx of the
attention projections) are checked on sampled context and output rows, which the oracle
can compute one row at a time."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import blocks, inputs
from gpu_helpers import BF16_TOL, FP32_TOL, rel_fro, unsigma

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample_rows(T, C, n, seed):
    rng = np.random.default_rng(seed)
    ctx = rng.choice(C, n // 2, replace=False)
    out = C + rng.choice(T - C, n - n // 2, replace=False)
    return np.sort(np.concatenate([ctx, out]))


@pytest.mark.parametrize("cfg", [inputs.LLAMA3_8B_FFN, inputs.LLAMA2_13B_FFN], ids=lambda c: c.name)
def test_ffn_full_size(cfg):
    d = inputs.make_ffn_inputs(cfg, seed=1, device=DEV)
    perm = inputs.context_first_order(d["ctx_mask"])
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    x, dy = d["x"][perm].contiguous(), d["dy"][perm].contiguous()
    blk = blocks.FFNBlock(d["gate"], d["up"], d["down"], d["lora_gate"], d["lora_up"], d["lora_down"],
                          cfg.lora_scale, cfg.k, T, C, cfg.ratio, DEV)
    blk.step(x, dy)
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    ctx = np.arange(T) < C
    s_w, _ = oracle.ffn_select(x, ctx, (d["gate"].W_A, d["gate"].W_B), (d["up"].W_A, d["up"].W_B), cfg.ratio)
    assert rel_fro(blk.scores, s_w) < FP32_TOL
    sc = blk.scores.cpu().numpy().astype(np.float64)
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    np.testing.assert_array_equal(idx, oracle.select_top(sc, blk.n_keep))
    rows = sample_rows(T, C, 48, 0)
    xr, dyr, cr = x[rows].cpu(), dy[rows].cpu(), ctx[rows]
    W = lambda w: w.W.cpu()
    L = lambda p: (p[0].cpu(), p[1].cpu())
    args = (xr, cr, W(d["gate"]), W(d["up"]), W(d["down"]), L(d["lora_gate"]), L(d["lora_up"]),
            L(d["lora_down"]), cfg.lora_scale, idx)
    fwd = oracle.ffn_fwd(*args)
    bwd = oracle.ffn_bwd(xr, dyr, cr, W(d["gate"]), W(d["up"]), W(d["down"]), L(d["lora_gate"]),
                         L(d["lora_up"]), L(d["lora_down"]), cfg.lora_scale, idx, fwd=fwd)
    n_ctx_rows = int(cr.sum())
    sig = blk.sigma

    def nat(t):  # natural-layout sampled rows of a sigma-layout activation
        sub = t[rows]
        return unsigma(sub, sig, n_ctx_rows)

    assert rel_fro(nat(blk.g), fwd["G"]) < BF16_TOL
    assert rel_fro(nat(blk.u), fwd["U"]) < BF16_TOL
    assert rel_fro(nat(blk.h), fwd["H"]) < BF16_TOL
    assert rel_fro(blk.y[rows], fwd["Y"]) < BF16_TOL
    assert rel_fro(nat(blk.dg), bwd["dG"]) < BF16_TOL
    assert rel_fro(blk.dx[rows], bwd["dX"]) < BF16_TOL


@pytest.mark.parametrize("cfg", [inputs.LLAMA3_8B_ATTN, inputs.LLAMA2_13B_ATTN], ids=lambda c: c.name)
def test_attn_full_size(cfg):
    d = inputs.make_attn_inputs(cfg, seed=2, device=DEV)
    perm = inputs.context_first_order(d["ctx_mask"])
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    t = {k: d[k][perm].contiguous() for k in ("x", "x_o", "dq", "dk", "dv", "dy")}
    blk = blocks.AttnProjBlock(d["q"], d["k"], d["v"], d["o"], d["lora_q"], d["lora_k"], d["lora_v"], d["lora_o"],
                               cfg.lora_scale, cfg.k, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, T, C, cfg.ratio,
                               DEV)
    blk.step(t["x"], t["x_o"], t["dy"], t["dq"], t["dk"], t["dv"])
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    ctx = np.arange(T) < C
    F = lambda n: (d[n].W_A, d[n].W_B)
    sel = oracle.attn_select(t["x"], ctx, F("q"), F("k"), F("v"), cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim,
                             cfg.ratio)
    assert rel_fro(blk.s_qk, sel["s_qk"]) < FP32_TOL
    assert rel_fro(blk.s_v, sel["s_v"]) < FP32_TOL
    u_qk = blk.sig_k.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
    u_v = blk.sig_v.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
    np.testing.assert_array_equal(u_qk, oracle.select_top(blk.s_qk.cpu().numpy().astype(np.float64), blk.n_keep_u))
    np.testing.assert_array_equal(u_v, oracle.select_top(blk.s_v.cpu().numpy().astype(np.float64), blk.n_keep_u))
    hq, hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    idx = {"q": oracle.expand_units(u_qk, hq, hkv, hd), "k": u_qk, "v": u_v, "o": oracle.expand_units(u_v, hq, hkv, hd)}
    rows = sample_rows(T, C, 48, 1)
    cr = ctx[rows]
    lo = {n: (d["lora_" + n][0].cpu(), d["lora_" + n][1].cpu()) for n in "qkvo"}
    outs = {"q": blk.q, "k": blk.kk, "v": blk.vv}
    xr = t["x"][rows].cpu()
    for n in "qkv":
        want = oracle.sparse_linear_fwd(xr, d[n].W.cpu(), *lo[n], cfg.lora_scale, cr, idx[n], "out")
        assert rel_fro(outs[n][rows], want) < BF16_TOL, n
    xo = t["x_o"][rows].cpu()
    assert rel_fro(blk.y[rows], oracle.sparse_linear_fwd(xo, d["o"].W.cpu(), *lo["o"], cfg.lora_scale, cr, idx["o"],
                                                         "in")) < BF16_TOL
    dxo, _, _ = oracle.sparse_linear_bwd(xo, t["dy"][rows].cpu(), d["o"].W.cpu(), *lo["o"], cfg.lora_scale, cr,
                                         idx["o"], "in")
    assert rel_fro(blk.dx_o[rows], dxo) < BF16_TOL
    dx = 0
    for n, g in (("q", "dq"), ("k", "dk"), ("v", "dv")):
        dx = dx + oracle.sparse_linear_bwd(xr, t[g][rows].cpu(), d[n].W.cpu(), *lo[n], cfg.lora_scale, cr, idx[n],
                                           "out")[0]
    assert rel_fro(blk.dx[rows], dx) < BF16_TOL
