"""Full model sizes with the frozen branch checked on its own, and the LoRA gradients over the
whole batch.

With the workload's generators the LoRA term of an output is about ten times the sliced main
branch, so a relative error bound on y = main + LoRA would let a large main-branch error through.
Here every LoRA B is zero: y, g, u, h and dx are the sliced frozen products alone (plus, in
dx, nothing from LoRA since dy B = 0), compared element by element on sampled context and
output rows with the CTA-pair GEMM forced to each tile height (256- and 512-row tiles).

The LoRA gradients dA, dB are sums over all tokens, so they are compared with the oracle run over
the whole batch: the four attention adapters (rank-32 products, cheap in fp64) and the three FFN
adapters (one fp64 forward and backward of the FFN block on every row).

Sizes: the LLaMA3-8B blocks (8 x 512 tokens, 3072 context + 1024 output, GQA 32/8, FFN 14336,
estimator rank 8) at keep 0.5 and 0.3, and the LLaMA2-13B blocks (4 x 1024 tokens, MHA 40 x 128,
FFN 13824, estimator rank 16) at keep 0.4.
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks, inputs
from gpu_helpers import BF16_TOL, rel_fro, unsigma

pytestmark = pytest.mark.gpu
DEV = "cuda"
TILE_ROWS = (256, 512)


def sample_rows(T, C, n, seed):
    rng = np.random.default_rng(seed)
    ctx = rng.choice(C, n // 2, replace=False)
    out = C + rng.choice(T - C, n - n // 2, replace=False)
    return np.sort(np.concatenate([ctx, out]))


def assert_close_elementwise(got, want, name, tol=BF16_TOL):
    """Element by element: |got - want| <= tol (|want| + rms of want's row), every row's relative
    Frobenius error <= tol, and the whole block's <= tol."""
    g, w = oracle.f64(got), oracle.f64(want)
    assert g.shape == w.shape, name
    rms = np.sqrt(np.mean(w * w, axis=1, keepdims=True))
    bad = np.abs(g - w) > tol * (np.abs(w) + rms)
    assert not bad.any(), f"{name}: {int(bad.sum())} elements outside tolerance, first at {np.argwhere(bad)[0]}"
    row_err = np.linalg.norm(g - w, axis=1) / np.maximum(np.linalg.norm(w, axis=1), 1e-30)
    assert row_err.max() <= tol, f"{name}: row error {row_err.max():.3g}"
    assert rel_fro(g, w) <= tol, name


def zero_b(pair):
    a, b = pair
    return a, torch.zeros_like(b)


_CACHE = {}


def ffn_case(cfg, seed):
    key = ("ffn", cfg.name, seed)
    if key not in _CACHE:
        _CACHE.clear()
        d = inputs.make_ffn_inputs(cfg, seed=seed, device=DEV)
        perm = inputs.context_first_order(d["ctx_mask"])
        host = {n: d[n].W.cpu() for n in ("gate", "up", "down")}
        _CACHE[key] = (d, perm, host)
    return _CACHE[key]


def attn_case(cfg, seed):
    key = ("attn", cfg.name, seed)
    if key not in _CACHE:
        _CACHE.clear()
        d = inputs.make_attn_inputs(cfg, seed=seed, device=DEV)
        perm = inputs.context_first_order(d["ctx_mask"])
        host = {n: d[n].W.cpu() for n in "qkvo"}
        _CACHE[key] = (d, perm, host)
    return _CACHE[key]


FFN_CASES = [(inputs.LLAMA3_8B_FFN, 0.5), (inputs.LLAMA3_8B_FFN, 0.3), (inputs.LLAMA2_13B_FFN, 0.4)]
ATTN_CASES = [(inputs.LLAMA3_8B_ATTN, 0.5), (inputs.LLAMA2_13B_ATTN, 0.4)]


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
@pytest.mark.parametrize("cfg,ratio", FFN_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_ffn_full_size_main_branch(cfg, ratio, tile_rows):
    d, perm, host = ffn_case(cfg, 3)
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    x, dy = d["x"][perm].contiguous(), d["dy"][perm].contiguous()
    lg, lu, ld = zero_b(d["lora_gate"]), zero_b(d["lora_up"]), zero_b(d["lora_down"])
    with B.pair_tile_rows(tile_rows):
        blk = blocks.FFNBlock(d["gate"], d["up"], d["down"], lg, lu, ld, cfg.lora_scale, cfg.k, T, C, ratio, DEV)
        blk.step(x, dy)
        torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    np.testing.assert_array_equal(idx, oracle.select_top(blk.scores.cpu().numpy().astype(np.float64), blk.n_keep))
    rows = sample_rows(T, C, 48, 5)
    ctx = np.arange(T) < C
    xr, dyr, cr = x[rows].cpu(), dy[rows].cpu(), ctx[rows]
    L = lambda p: (p[0].cpu(), p[1].cpu())
    args = (xr, cr, host["gate"], host["up"], host["down"], L(lg), L(lu), L(ld), cfg.lora_scale, idx)
    fwd = oracle.ffn_fwd(*args)
    bwd = oracle.ffn_bwd(xr, dyr, cr, host["gate"], host["up"], host["down"], L(lg), L(lu), L(ld), cfg.lora_scale,
                         idx, fwd=fwd)
    n_ctx_rows = int(cr.sum())

    def nat(t):
        return unsigma(t[rows], blk.sigma, n_ctx_rows)

    for got, want, name in ((nat(blk.g), fwd["G"], "g"), (nat(blk.u), fwd["U"], "u"), (nat(blk.h), fwd["H"], "h"),
                            (blk.y[rows], fwd["Y"], "y"), (nat(blk.dg), bwd["dG"], "dg"),
                            (nat(blk.du), bwd["dU"], "du"), (blk.dx[rows], bwd["dX"], "dx")):
        assert_close_elementwise(got, want, f"{name} ({tile_rows}-row tiles)")
    # dropped context channels carry no main-branch value: with B = 0 they are exactly zero
    drop = blk.sigma.cpu().numpy()[blk.n_keep:]
    gctx = oracle.f64(blk.g[:C].cpu())
    assert np.all(gctx[:, blk.n_keep:] == 0.0), "dropped context channels of g"
    assert drop.size == cfg.inter - blk.n_keep


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
@pytest.mark.parametrize("cfg,ratio", ATTN_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_attn_full_size_main_branch(cfg, ratio, tile_rows):
    d, perm, host = attn_case(cfg, 4)
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    t = {k: d[k][perm].contiguous() for k in ("x", "x_o", "dq", "dk", "dv", "dy")}
    lo = {n: zero_b(d["lora_" + n]) for n in "qkvo"}
    with B.pair_tile_rows(tile_rows):
        blk = blocks.AttnProjBlock(d["q"], d["k"], d["v"], d["o"], lo["q"], lo["k"], lo["v"], lo["o"], cfg.lora_scale,
                                   cfg.k, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, T, C, ratio, DEV)
        blk.step(t["x"], t["x_o"], t["dy"], t["dq"], t["dk"], t["dv"])
        torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    hq, hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    u_qk = blk.sig_k.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
    u_v = blk.sig_v.cpu().numpy()[: blk.n_keep_u].astype(np.int64)
    idx = {"q": oracle.expand_units(u_qk, hq, hkv, hd), "k": u_qk, "v": u_v, "o": oracle.expand_units(u_v, hq, hkv, hd)}
    rows = sample_rows(T, C, 48, 6)
    cr = (np.arange(T) < C)[rows]
    L = {n: (lo[n][0].cpu(), lo[n][1].cpu()) for n in "qkvo"}
    xr, xo = t["x"][rows].cpu(), t["x_o"][rows].cpu()
    outs = {"q": blk.q, "k": blk.kk, "v": blk.vv}
    for n in "qkv":
        want = oracle.sparse_linear_fwd(xr, host[n], *L[n], cfg.lora_scale, cr, idx[n], "out")
        assert_close_elementwise(outs[n][rows], want, f"{n} ({tile_rows}-row tiles)")
    want = oracle.sparse_linear_fwd(xo, host["o"], *L["o"], cfg.lora_scale, cr, idx["o"], "in")
    assert_close_elementwise(blk.y[rows], want, f"y ({tile_rows}-row tiles)")
    dxo = oracle.sparse_linear_bwd(xo, t["dy"][rows].cpu(), host["o"], *L["o"], cfg.lora_scale, cr, idx["o"], "in")[0]
    assert_close_elementwise(blk.dx_o[rows], dxo, f"dx_o ({tile_rows}-row tiles)")
    dx = 0
    for n, g in (("q", "dq"), ("k", "dk"), ("v", "dv")):
        dx = dx + oracle.sparse_linear_bwd(xr, t[g][rows].cpu(), host[n], *L[n], cfg.lora_scale, cr, idx[n], "out")[0]
    assert_close_elementwise(blk.dx[rows], dx, f"dx ({tile_rows}-row tiles)")


@pytest.mark.parametrize("cfg", [inputs.LLAMA3_8B_ATTN, inputs.LLAMA2_13B_ATTN], ids=lambda c: c.name)
def test_attn_full_size_lora_gradients(cfg):
    """dA, dB of q, k, v, o over all tokens against the oracle's sums over the whole batch (with the
    GPU's index sets; the LoRA gradients do not depend on them, since they read x, x_o and the
    upstream gradients only)."""
    d, perm, host = attn_case(cfg, 4)
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    t = {k: d[k][perm].contiguous() for k in ("x", "x_o", "dq", "dk", "dv", "dy")}
    blk = blocks.AttnProjBlock(d["q"], d["k"], d["v"], d["o"], d["lora_q"], d["lora_k"], d["lora_v"], d["lora_o"],
                               cfg.lora_scale, cfg.k, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, T, C, cfg.ratio,
                               DEV)
    blk.step(t["x"], t["x_o"], t["dy"], t["dq"], t["dk"], t["dv"])
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    s = cfg.lora_scale
    x, xo = oracle.f64(t["x"]), oracle.f64(t["x_o"])
    for n, xin, g in (("q", x, "dq"), ("k", x, "dk"), ("v", x, "dv"), ("o", xo, "dy")):
        A, Bm = oracle.f64(d["lora_" + n][0]), oracle.f64(d["lora_" + n][1])
        dy = oracle.f64(t[g])
        dA = s * (dy @ Bm).T @ xin          # s (dy B)^T x
        dB = s * dy.T @ (xin @ A.T)         # s dy^T (x A^T)
        assert rel_fro(blk.dA[n], dA) < BF16_TOL, f"dA_{n}"
        assert rel_fro(blk.dB[n], dB) < BF16_TOL, f"dB_{n}"


@pytest.mark.parametrize("cfg", [inputs.LLAMA3_8B_FFN], ids=lambda c: c.name)
def test_ffn_full_size_lora_gradients(cfg):
    """dA, dB of gate, up, down over all 4096 tokens: one fp64 forward and backward of the FFN block
    on every row (the GPU's index set)."""
    d, perm, host = ffn_case(cfg, 3)
    C = int(d["ctx_mask"].sum())
    T = cfg.n_tok
    x, dy = d["x"][perm].contiguous(), d["dy"][perm].contiguous()
    blk = blocks.FFNBlock(d["gate"], d["up"], d["down"], d["lora_gate"], d["lora_up"], d["lora_down"],
                          cfg.lora_scale, cfg.k, T, C, cfg.ratio, DEV)
    blk.step(x, dy)
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    ctx = np.arange(T) < C
    L = lambda p: (p[0].cpu(), p[1].cpu())
    lg, lu, ld = L(d["lora_gate"]), L(d["lora_up"]), L(d["lora_down"])
    xc, dyc = x.cpu(), dy.cpu()
    fwd = oracle.ffn_fwd(xc, ctx, host["gate"], host["up"], host["down"], lg, lu, ld, cfg.lora_scale, idx)
    bwd = oracle.ffn_bwd(xc, dyc, ctx, host["gate"], host["up"], host["down"], lg, lu, ld, cfg.lora_scale, idx,
                         fwd=fwd)
    for n in ("g", "u", "d"):
        assert rel_fro(getattr(blk, "dA_" + n), bwd["dA_" + n]) < BF16_TOL, f"dA_{n}"
        assert rel_fro(getattr(blk, "dB_" + n), bwd["dB_" + n]) < BF16_TOL, f"dB_{n}"
    assert rel_fro(blk.y, fwd["Y"]) < BF16_TOL
    assert rel_fro(blk.dx, bwd["dX"]) < BF16_TOL
