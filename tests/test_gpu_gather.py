"""Kept weight rows read in place by the GEMM (row-gather copies through sigma) against the
same sliced products on a compacted copy of those rows, and against the fp64 oracle.

Both forms put the same bf16 rows in the same places of the tensor cores' operand tiles, so
the sliced products agree bit for bit. The shapes make the gather take every path it has:
kept counts that end inside a group of four rows and inside a tile (rows past the kept count
read the zero row), MN-major column blocks past the weight's width (widths that are whole
64-column blocks but not whole 256-column tiles), both CTA-pair tile heights and the one-CTA
kernel (tile rows 128).
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks, inputs
from gpu_helpers import BF16_TOL, attn_problem, ffn_problem, rel_fro, unsigma

pytestmark = pytest.mark.gpu
DEV = "cuda"
TILE_ROWS = [0, 128, 256, 512]


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


def sigma_from(idx, n):
    idx = np.asarray(idx, dtype=np.int64)
    return torch.tensor(np.concatenate([idx, oracle.complement(idx, n)]), dtype=torch.int32, device=DEV)


def _lora_fwd(ws, lin, xg, C, r, layout=B.SL_LAYOUT_NATURAL, ch=None):
    T = xg.shape[0]
    xa, xa_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa, in_layout=layout, in_ch=ch)
    return xa_s


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
@pytest.mark.parametrize("layout", [B.SL_LAYOUT_NATURAL, B.SL_LAYOUT_SIGMA])
def test_out_slice_gather_equals_compact(tile_rows, layout):
    """q/k/v-like products: y (N = kept output channels gathered, K-major) and dx (K = kept
    channels gathered, MN-major over d_in = 640, so the last tile's second CTA reads only zero
    column blocks)."""
    T, C, D, Do, r, nk = 424, 300, 640, 1000, 32, 437
    gen = inputs.generator(41)
    w = inputs.spectral_weight(Do, D, 0.5, 8, gen, "cpu", torch.float64, torch.bfloat16)
    A, Bm = inputs.lora_pair(Do, D, r, 0.02, gen)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    s, ctx = 2.0, np.arange(T) < C
    idx = np.sort(np.random.default_rng(42).choice(Do, nk, replace=False))
    sig = sigma_from(idx, Do)
    ws = B.Workspace()
    Wg, Ag, Bg, xg = cu(w.W), cu(A), cu(Bm), cu(x)
    w_kept = Wg[sig[:nk].long()].contiguous()
    lin_g = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_OUT)
    lin_c = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_OUT, w_kept=w_kept)
    ch = B.channels_desc(sig, nk)
    dy_in = dy.clone()
    if layout == B.SL_LAYOUT_SIGMA:
        dy_in[:C] = dy[:C][:, sig.cpu().long()]
    dyg = cu(dy_in)
    with B.pair_tile_rows(tile_rows):
        xa_s = _lora_fwd(ws, lin_g, xg, C, r)
        ys, dxs = [], []
        for lin in (lin_g, lin_c):
            y = torch.full((T, Do), float("nan"), device=DEV, dtype=torch.bfloat16)
            B.sl_sparse_linear_fwd(ws, [lin], [ch], B.SL_EPI_NONE, xg, C, xa_s, [y], out_layout=layout)
            ys.append(y)
        dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
        dA, dB = torch.empty(r, D, device=DEV), torch.empty(Do, r, device=DEV)
        B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin_g], xg, C, xa_s, dy=[dyg], out_layout=layout, out_ch=[ch],
                          dya=[dya], dya_s=[dya_s], dA=[dA], dB=[dB])
        for lin in (lin_g, lin_c):
            dx = torch.full((T, D), float("nan"), device=DEV, dtype=torch.bfloat16)
            B.sl_sparse_linear_bwd(ws, [lin], [ch], B.SL_EPI_NONE, [dyg], C, [dya_s], dx=dx, in_layout=layout)
            dxs.append(dx)
    torch.cuda.synchronize()
    assert ws.read_device_flag() == 0
    assert torch.equal(ys[0], ys[1])
    assert torch.equal(dxs[0], dxs[1])
    want = oracle.sparse_linear_fwd(x, w.W, A, Bm, s, ctx, idx, "out")
    got = oracle.f64(ys[0]) if layout == B.SL_LAYOUT_NATURAL else unsigma(ys[0], sig, C)
    assert np.isfinite(got).all()
    assert rel_fro(got, want) < BF16_TOL
    dX, _, _ = oracle.sparse_linear_bwd(x, dy, w.W, A, Bm, s, ctx, idx, "out")
    assert rel_fro(dxs[0], dX) < BF16_TOL


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
@pytest.mark.parametrize("layout", [B.SL_LAYOUT_NATURAL, B.SL_LAYOUT_SIGMA])
def test_in_slice_gather_equals_compact(tile_rows, layout):
    """o/down-like products: y (K = kept input channels gathered from W^T, MN-major over
    d_out = 640) and dx (N = kept input channels gathered from W^T, K-major)."""
    T, C, Di, Do, r, nk = 424, 300, 1000, 640, 32, 437
    gen = inputs.generator(43)
    w = inputs.spectral_weight(Do, Di, 0.5, 8, gen, "cpu", torch.float64, torch.bfloat16)
    A, Bm = inputs.lora_pair(Do, Di, r, 0.02, gen)
    x = inputs.activations_student_t(T, Di, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    s, ctx = 2.0, np.arange(T) < C
    idx = np.sort(np.random.default_rng(44).choice(Di, nk, replace=False))
    sig = sigma_from(idx, Di)
    ws = B.Workspace()
    Wg, Ag, Bg = cu(w.W), cu(A), cu(Bm)
    Wt = torch.empty(Di, Do, device=DEV, dtype=torch.bfloat16)
    B.sl_prepare_weight(Wg, Wt)
    w_kept = Wt[sig[:nk].long()].contiguous()
    lin_g = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_IN, w_t=Wt)
    lin_c = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_IN, w_t=Wt, w_kept=w_kept)
    ch = B.channels_desc(sig, nk)
    x_in = x.clone()
    if layout == B.SL_LAYOUT_SIGMA:
        x_in[:C] = x[:C][:, sig.cpu().long()]
    xg, dyg = cu(x_in), cu(dy)
    with B.pair_tile_rows(tile_rows):
        xa_s = _lora_fwd(ws, lin_g, xg, C, r, layout, ch)
        ys, dxs = [], []
        for lin in (lin_g, lin_c):
            y = torch.full((T, Do), float("nan"), device=DEV, dtype=torch.bfloat16)
            B.sl_sparse_linear_fwd(ws, [lin], [ch], B.SL_EPI_NONE, xg, C, xa_s, [y], in_layout=layout)
            ys.append(y)
        dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
        dA, dB = torch.empty(r, Di, device=DEV), torch.empty(Do, r, device=DEV)
        B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin_g], xg, C, xa_s, in_layout=layout, in_ch=ch, dy=[dyg], dya=[dya],
                          dya_s=[dya_s], dA=[dA], dB=[dB])
        for lin in (lin_g, lin_c):
            dx = torch.full((T, Di), float("nan"), device=DEV, dtype=torch.bfloat16)
            B.sl_sparse_linear_bwd(ws, [lin], [ch], B.SL_EPI_NONE, [dyg], C, [dya_s], dx=dx, out_layout=layout)
            dxs.append(dx)
    torch.cuda.synchronize()
    assert ws.read_device_flag() == 0
    assert torch.equal(ys[0], ys[1])
    assert torch.equal(dxs[0], dxs[1])
    assert rel_fro(ys[0], oracle.sparse_linear_fwd(x, w.W, A, Bm, s, ctx, idx, "in")) < BF16_TOL
    dX, _, _ = oracle.sparse_linear_bwd(x, dy, w.W, A, Bm, s, ctx, idx, "in")
    got = oracle.f64(dxs[0]) if layout == B.SL_LAYOUT_NATURAL else unsigma(dxs[0], sig, C)
    assert rel_fro(got, dX) < BF16_TOL


def _grads_close(a, b):
    # dB and the inputs of dx pass through fp32 reductions whose order is not fixed
    # (the fused LoRA backward), so the backward side is compared within rounding
    return rel_fro(a, b) < 1e-3


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
def test_ffn_block_gather_equals_compact(tile_rows):
    """The SwiGLU block: paired gate/up tiles gathered from both weights with one sigma, the
    down product gathered from W^T, the SwiGLU backward and the gate/up input gradient."""
    T, C, D, F, r, k = 424, 300, 512, 1000, 32, 8
    p = ffn_problem(T, C, D, F, r, k, seed=45)
    outs = []
    with B.pair_tile_rows(tile_rows):
        for kr in ("gather", "compact"):
            blk = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5, DEV,
                                  kept_rows=kr)
            blk.step(cu(p["x"]), cu(p["dy"]))
            torch.cuda.synchronize()
            assert blk.read_device_flag() == 0
            outs.append(blk)
    g, c = outs
    assert torch.equal(g.sigma, c.sigma)
    for name in ("g", "u", "h", "y"):
        assert torch.equal(getattr(g, name), getattr(c, name)), name
    for name in ("dg", "du", "dx"):
        assert _grads_close(getattr(g, name), getattr(c, name)), name
    assert _grads_close(g.grads.flat, c.grads.flat)
    idx = g.sigma.cpu().numpy()[: g.n_keep].astype(np.int64)
    fwd = oracle.ffn_fwd(p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0, idx)
    assert rel_fro(g.y, fwd["Y"]) < BF16_TOL


@pytest.mark.parametrize("tile_rows", TILE_ROWS)
def test_attention_block_gather_equals_compact(tile_rows):
    """q/k/v (GQA expansion of the kept KV units to the query side, natural-layout scatter) and
    o gathered from W^T."""
    T, C, D, hq, hkv, hd, r, k = 424, 300, 512, 8, 2, 64, 32, 8
    a = attn_problem(T, C, D, hq, hkv, hd, r, k, seed=46)
    w, lo = a["w"], a["lora"]
    outs = []
    with B.pair_tile_rows(tile_rows):
        for kr in ("gather", "compact"):
            ab = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], 2.0, k, hq,
                                      hkv, hd, T, C, 0.5, DEV, kept_rows=kr)
            ab.step(cu(a["x"]), cu(a["x_o"]), cu(a["dy"]), cu(a["dq"]), cu(a["dk"]), cu(a["dv"]))
            torch.cuda.synchronize()
            assert ab.read_device_flag() == 0
            outs.append(ab)
    g, c = outs
    for name in ("sig_q", "sig_k", "sig_v", "sig_o"):
        assert torch.equal(getattr(g, name), getattr(c, name)), name
    for name in ("q", "kk", "vv", "y"):
        assert torch.equal(getattr(g, name), getattr(c, name)), name
    for name in ("dx", "dx_o"):
        assert _grads_close(getattr(g, name), getattr(c, name)), name
    assert _grads_close(g.grads.flat, c.grads.flat)
    u_v = g.sig_v.cpu().numpy()[: g.n_keep_u].astype(np.int64)
    idx_o = oracle.expand_units(u_v, hq, hkv, hd)
    want = oracle.sparse_linear_fwd(a["x_o"], w["o"].W, *lo["o"], 2.0, a["ctx"], idx_o, "in")
    assert rel_fro(g.y, want) < BF16_TOL
