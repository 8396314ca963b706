"""The whole decoder layer at full model sizes: LLaMA3-8B (8 x 512 tokens, 3072 context + 1024
output, GQA 32/8 x 128, FFN 14336, estimator rank 8, keep 0.5) and the LLaMA2-13B layer (4 x 1024
tokens, MHA 40 x 128, FFN 13824, estimator rank 16, keep 0.4).

The selections are checked on the whole batch: the GPU's attention and FFN scores against
the oracle's criteria applied to the GPU's own normalised rows h1 and h2 (fp32 arithmetic on
the same bf16 inputs), and each index set against the oracle's top-n of the GPU's scores
(exact). With those index sets fixed, the rows of one sequence depend on that sequence alone
(the projections and RMSNorm are row-wise, the attention is causal within the sequence), so
the oracle computes h1, x2, y and dx for whole sampled sequences, forward and backward."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import blocks, inputs
from contextual_sparsity_lora_b200.layer import DecoderLayer
from gpu_helpers import BF16_TOL, FP32_TOL, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("ac,fc,seqs", [(inputs.LLAMA3_8B_ATTN, inputs.LLAMA3_8B_FFN, (0, 7)),
                                        (inputs.LLAMA2_13B_ATTN, inputs.LLAMA2_13B_FFN, (2,))],
                         ids=["llama3-8b", "llama2-13b"])
def test_decoder_layer_full_size(ac, fc, seqs):
    da = inputs.make_attn_inputs(ac, seed=3, device=DEV)
    df = inputs.make_ffn_inputs(fc, seed=4, device=DEV)
    mask = da["ctx_mask"]
    perm = inputs.context_first_order(mask)
    C, T, D = int(mask.sum()), ac.n_tok, ac.hidden
    hq, hkv, hd = ac.n_q_heads, ac.n_kv_heads, ac.head_dim
    gen = inputs.generator(5)
    g1 = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    g2 = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    attn = blocks.AttnProjBlock(da["q"], da["k"], da["v"], da["o"], da["lora_q"], da["lora_k"], da["lora_v"],
                                da["lora_o"], ac.lora_scale, ac.k, hq, hkv, hd, T, C, ac.ratio, DEV, io_layout="sigma")
    ffn = blocks.FFNBlock(df["gate"], df["up"], df["down"], df["lora_gate"], df["lora_up"], df["lora_down"],
                          fc.lora_scale, fc.k, T, C, fc.ratio, DEV)
    p_np = perm.cpu().numpy()
    layer = DecoderLayer(attn, ffn, g1, g2, p_np, ac.batch)
    x, dy = da["x"], da["dy"]  # sequence order
    layer.step(x[perm].contiguous(), dy[perm].contiguous())
    torch.cuda.synchronize()
    assert attn.read_device_flag() == 0 and ffn.read_device_flag() == 0

    def nat(t):  # context-first rows -> sequence order
        out = np.empty(tuple(t.shape), dtype=np.float64)
        out[p_np] = oracle.f64(t)
        return out

    ctx = mask.cpu().numpy()
    h1, h2 = nat(layer.h1), nat(layer.h2)
    sel = oracle.attn_select(h1, ctx, (da["q"].W_A, da["q"].W_B), (da["k"].W_A, da["k"].W_B),
                             (da["v"].W_A, da["v"].W_B), hq, hkv, hd, ac.ratio)
    assert rel_fro(attn.s_qk, sel["s_qk"]) < FP32_TOL
    assert rel_fro(attn.s_v, sel["s_v"]) < FP32_TOL
    s_f, _ = oracle.ffn_select(h2, ctx, (df["gate"].W_A, df["gate"].W_B), (df["up"].W_A, df["up"].W_B), fc.ratio)
    assert rel_fro(ffn.scores, s_f) < FP32_TOL
    idx = {"q": attn.sig_q.cpu().numpy()[: attn.ch["q"].n_keep].astype(np.int64),
           "k": attn.sig_k.cpu().numpy()[: attn.ch["k"].n_keep].astype(np.int64),
           "v": attn.sig_v.cpu().numpy()[: attn.ch["v"].n_keep].astype(np.int64),
           "o": attn.sig_o.cpu().numpy()[: attn.ch["o"].n_keep].astype(np.int64),
           "ffn": ffn.sigma.cpu().numpy()[: ffn.n_keep].astype(np.int64)}
    f32 = lambda t: t.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(idx["ffn"], oracle.select_top(f32(ffn.scores), ffn.n_keep))
    np.testing.assert_array_equal(idx["k"], oracle.select_top(f32(attn.s_qk), attn.ch["k"].n_keep))
    np.testing.assert_array_equal(idx["v"], oracle.select_top(f32(attn.s_v), attn.ch["v"].n_keep))

    w = {"q": da["q"].W, "k": da["k"].W, "v": da["v"].W, "o": da["o"].W, "gate": df["gate"].W, "up": df["up"].W,
         "down": df["down"].W}
    lora = {"q": da["lora_q"], "k": da["lora_k"], "v": da["lora_v"], "o": da["lora_o"], "gate": df["lora_gate"],
            "up": df["lora_up"], "down": df["lora_down"]}
    got = {n: nat(t) for n, t in (("H1", layer.h1), ("X2", layer.x2), ("Y", layer.y), ("dX", layer.dx))}
    S = ac.seq
    for s in seqs:
        rows = np.arange(s * S, (s + 1) * S)
        ref = oracle.decoder_layer(x[rows].cpu(), dy[rows].cpu(), ctx[rows], 1, w, lora, (g1, g2), 1e-5,
                                   ac.lora_scale, (hq, hkv, hd), ac.ratio, idx=dict(idx))
        for n in ("H1", "X2", "Y", "dX"):
            assert rel_fro(got[n][rows], ref[n]) < BF16_TOL, (s, n)
