"""A whole decoder layer around the sparse projections (RMSNorm, sparse q/k/v, causal GQA
attention, sparse o, residual, RMSNorm, sparse FFN, residual), forward and backward, against
the fp64 oracle of the same layer with the index sets the GPU chose (their validity is
checked against the oracle's scores)."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import blocks, inputs
from contextual_sparsity_lora_b200.layer import DecoderLayer
from gpu_helpers import BF16_TOL, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def build(n_seq, S, n_out, D, hq, hkv, hd, F, r, k, ratio, seed, io_layout="natural"):
    gen = inputs.generator(seed)
    Dq, Dkv = hq * hd, hkv * hd
    shapes = {"q": (Dq, D), "k": (Dkv, D), "v": (Dkv, D), "o": (D, Dq), "gate": (F, D), "up": (F, D), "down": (D, F)}
    w = {n: inputs.spectral_weight(do, di, 0.5, k, gen, "cpu", torch.float64, torch.bfloat16)
         for n, (do, di) in shapes.items()}
    lora = {n: inputs.lora_pair(do, di, r, 0.02, gen) for n, (do, di) in shapes.items()}
    g1 = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    g2 = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    T = n_seq * S
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, D, generator=gen).to(torch.bfloat16)
    ctx = np.tile(np.arange(S) < S - n_out, n_seq)
    perm = inputs.context_first_order(torch.from_numpy(ctx)).numpy()
    C = int(ctx.sum())
    attn = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lora["q"], lora["k"], lora["v"], lora["o"], 2.0, k,
                                hq, hkv, hd, T, C, ratio, DEV, io_layout=io_layout)
    ffn = blocks.FFNBlock(w["gate"], w["up"], w["down"], lora["gate"], lora["up"], lora["down"], 2.0, k, T, C, ratio,
                          DEV)
    layer = DecoderLayer(attn, ffn, g1, g2, perm, n_seq)
    return dict(w=w, lora=lora, g1=g1, g2=g2, x=x, dy=dy, ctx=ctx, perm=perm, layer=layer, attn=attn,
                ffn=ffn, heads=(hq, hkv, hd), n_seq=n_seq)


@pytest.mark.parametrize("io_layout", ["natural", "sigma"])
@pytest.mark.parametrize("n_seq,S,n_out,D,hq,hkv,hd,F", [(2, 64, 16, 256, 4, 2, 32, 512), (3, 40, 8, 128, 2, 2, 64, 264)])
def test_decoder_layer_matches_oracle(n_seq, S, n_out, D, hq, hkv, hd, F, io_layout):
    """Both interface layouts of the attention block: natural channels, or the sigma layout with
    the layer's permutations converting the context rows' channel order."""
    p = build(n_seq, S, n_out, D, hq, hkv, hd, F, 16, 8, 0.5, seed=61, io_layout=io_layout)
    perm = p["perm"]
    pt = torch.from_numpy(perm)
    x_cf = p["x"][pt].to(DEV).contiguous()
    dy_cf = p["dy"][pt].to(DEV).contiguous()
    layer, attn, ffn = p["layer"], p["attn"], p["ffn"]
    layer.step(x_cf, dy_cf)
    torch.cuda.synchronize()

    def nat(t):  # context-first rows -> sequence order
        out = np.empty(tuple(t.shape), dtype=np.float64)
        out[perm] = oracle.f64(t)
        return out

    idx = {"q": attn.sig_q.cpu().numpy()[: attn.ch["q"].n_keep].astype(np.int64),
           "k": attn.sig_k.cpu().numpy()[: attn.ch["k"].n_keep].astype(np.int64),
           "v": attn.sig_v.cpu().numpy()[: attn.ch["v"].n_keep].astype(np.int64),
           "o": attn.sig_o.cpu().numpy()[: attn.ch["o"].n_keep].astype(np.int64),
           "ffn": ffn.sigma.cpu().numpy()[: ffn.n_keep].astype(np.int64)}
    w = {n: v.W for n, v in p["w"].items()}
    ref = oracle.decoder_layer(p["x"], p["dy"], p["ctx"], n_seq, w, p["lora"], (p["g1"], p["g2"]), 1e-5, 2.0,
                               p["heads"], 0.5, idx=dict(idx))
    # the selections read the normalised inputs: the GPU's scores against the oracle's on the
    # oracle's own normalised rows (bf16 rounding of h1, h2 sets the tolerance)
    fac = {n: (p["w"][n].W_A, p["w"][n].W_B) for n in ("q", "k", "v", "gate", "up")}
    sel = oracle.attn_select(ref["H1"], p["ctx"], fac["q"], fac["k"], fac["v"], hq, hkv, hd, 0.5)
    assert rel_fro(attn.s_qk, sel["s_qk"]) < BF16_TOL
    assert rel_fro(attn.s_v, sel["s_v"]) < BF16_TOL
    s_f, _ = oracle.ffn_select(ref["H2"], p["ctx"], fac["gate"], fac["up"], 0.5)
    assert rel_fro(ffn.scores, s_f) < BF16_TOL
    np.testing.assert_array_equal(idx["ffn"], oracle.select_top(ffn.scores.cpu().numpy().astype(np.float64),
                                                                 ffn.n_keep))
    # forward and backward of the layer
    assert rel_fro(nat(layer.h1), ref["H1"]) < BF16_TOL
    assert rel_fro(nat(layer.x2), ref["X2"]) < BF16_TOL
    assert rel_fro(nat(layer.y), ref["Y"]) < BF16_TOL
    assert rel_fro(nat(layer.dx), ref["dX"]) < BF16_TOL
    for n in "qkvo":
        assert rel_fro(attn.dA[n], ref["dA_" + n]) < BF16_TOL, n
        assert rel_fro(attn.dB[n], ref["dB_" + n]) < BF16_TOL, n
    for n, a, b in (("gate", ffn.dA_g, ffn.dB_g), ("up", ffn.dA_u, ffn.dB_u), ("down", ffn.dA_d, ffn.dB_d)):
        assert rel_fro(a, ref["dA_" + n]) < BF16_TOL, n
        assert rel_fro(b, ref["dB_" + n]) < BF16_TOL, n


def test_rmsnorm_and_add_rows_match_oracle():
    from contextual_sparsity_lora_b200 import binding as B
    gen = inputs.generator(62)
    T, D = 37, 264
    x = torch.randn(T, D, generator=gen).to(torch.bfloat16).to(DEV)
    res = torch.randn(T, D, generator=gen).to(torch.bfloat16).to(DEV)
    g = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16).to(DEV)
    dy = torch.randn(T, D, generator=gen).to(torch.bfloat16).to(DEV)
    y, s = torch.empty_like(x), torch.empty_like(x)
    rstd = torch.empty(T, device=DEV)
    B.sl_rmsnorm_fwd(x, g, 1e-5, y, rstd, res=res, sum_out=s)
    s_ref = oracle.f64(x) + oracle.f64(res)
    assert rel_fro(s, s_ref) < 1e-2
    assert rel_fro(y, oracle.rmsnorm(s, g, 1e-5)) < 1e-2
    dx = torch.empty_like(x)
    B.sl_rmsnorm_bwd(dy, s, g, rstd, dx, dres=res)
    assert rel_fro(dx, oracle.rmsnorm_bwd(dy, s, g, 1e-5) + oracle.f64(res)) < 1e-2
    out = torch.empty_like(x)
    B.sl_add_rows(x, res, out)
    assert rel_fro(out, s_ref) < 1e-2
