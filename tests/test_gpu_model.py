"""A whole fine-tuning step of a small stack of decoder layers (embedding, layers with a per-layer
keep table, final RMSNorm, LM head, cross-entropy on the output rows, backward, AdamW) against
the fp64 oracle with the index sets each layer's GPU selection chose; the progressive schedule's
dense steps; the AdamW update."""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import inputs
from contextual_sparsity_lora_b200.model import SparseLoRAModel, llama3_8b_math10k_keep
from gpu_helpers import BF16_TOL, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def build(keep, seed=71):
    gen = inputs.generator(seed)
    n_seq, S, n_out, D, hq, hkv, hd, F, r, k, V = 2, 48, 16, 128, 2, 1, 64, 256, 8, 8, 512
    shapes = {"q": (hq * hd, D), "k": (hkv * hd, D), "v": (hkv * hd, D), "o": (D, hq * hd), "gate": (F, D),
              "up": (F, D), "down": (D, F)}
    frozen = {n: inputs.spectral_weight(do, di, 0.5, k, gen, "cpu", torch.float64, torch.bfloat16)
              for n, (do, di) in shapes.items()}
    frozen["embed"] = (torch.randn(V, D, generator=gen)).to(torch.bfloat16)
    frozen["lm_head"] = (0.05 * torch.randn(V, D, generator=gen)).to(torch.bfloat16)
    frozen["gamma_f"] = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)
    loras = [{n: inputs.lora_pair(do, di, r, 0.02, gen) for n, (do, di) in shapes.items()} for _ in keep]
    gammas = [((1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16),
               (1.0 + 0.1 * torch.randn(D, generator=gen)).to(torch.bfloat16)) for _ in keep]
    T = n_seq * S
    ctx = np.tile(np.arange(S) < S - n_out, n_seq)
    perm = inputs.context_first_order(torch.from_numpy(ctx)).numpy()
    C = int(ctx.sum())
    ids = torch.randint(0, V, (T,), generator=gen)
    targets = torch.randint(0, V, (T - C,), generator=gen)  # one per output row, sequence order
    model = SparseLoRAModel(frozen, loras, gammas, keep, perm, C, n_seq, (hq, hkv, hd), k, 2.0, DEV)
    return dict(frozen=frozen, loras=loras, gammas=gammas, ctx=ctx, perm=perm, ids=ids, targets=targets, model=model,
                n_seq=n_seq, heads=(hq, hkv, hd), C=C)


def run_and_check(p, dense):
    model, perm = p["model"], p["perm"]
    pt = torch.from_numpy(perm)
    ids_cf = p["ids"][pt].to(torch.int32).to(DEV)
    # the output rows of the context-first order are the output rows in sequence order
    model.set_dense(dense)
    loss = model.forward_backward(ids_cf, p["targets"].to(DEV))
    torch.cuda.synchronize()
    layers = []
    for lay in model.layers:
        at, ff = lay.attn, lay.ffn
        idx = {"q": at.sig_q.cpu().numpy()[: at.ch["q"].n_keep].astype(np.int64),
               "k": at.sig_k.cpu().numpy()[: at.ch["k"].n_keep].astype(np.int64),
               "v": at.sig_v.cpu().numpy()[: at.ch["v"].n_keep].astype(np.int64),
               "o": at.sig_o.cpu().numpy()[: at.ch["o"].n_keep].astype(np.int64),
               "ffn": ff.sigma.cpu().numpy()[: ff.n_keep].astype(np.int64)}
        if ff.dense:
            idx["ffn"] = np.arange(ff.F)
        if at.dense:
            idx.update(q=np.arange(at.Dq), k=np.arange(at.Dkv), v=np.arange(at.Dkv), o=np.arange(at.Dq))
        layers.append(idx)
    w = {n: v.W for n, v in p["frozen"].items() if n not in ("embed", "lm_head", "gamma_f")}
    L = [dict(w=w, lora=p["loras"][i], gammas=p["gammas"][i], idx=layers[i]) for i in range(len(layers))]
    ref_loss, grads = oracle.model_step(p["ids"].numpy(), p["targets"].numpy(), p["ctx"], p["n_seq"],
                                        p["frozen"]["embed"], p["frozen"]["lm_head"], p["frozen"]["gamma_f"], L, 1e-5,
                                        2.0, p["heads"])
    assert abs(float(loss) - ref_loss) <= 2e-2 * abs(ref_loss)
    for i, lay in enumerate(model.layers):
        at, ff = lay.attn, lay.ffn
        for n in "qkvo":
            assert rel_fro(at.dA[n], grads[i]["dA_" + n]) < BF16_TOL, (i, n)
            assert rel_fro(at.dB[n], grads[i]["dB_" + n]) < BF16_TOL, (i, n)
        for n, a, b in (("gate", ff.dA_g, ff.dB_g), ("up", ff.dA_u, ff.dB_u), ("down", ff.dA_d, ff.dB_d)):
            assert rel_fro(a, grads[i]["dA_" + n]) < BF16_TOL, (i, n)
            assert rel_fro(b, grads[i]["dB_" + n]) < BF16_TOL, (i, n)
    return model


def test_model_step_matches_oracle_with_per_layer_keep_table():
    p = build([(1.0, 1.0), (0.5, 0.5), (0.25, 0.3)])
    model = run_and_check(p, dense=False)
    assert model.layers[0].ffn.dense and not model.layers[2].ffn.dense


def test_progressive_schedule_dense_steps_match_dense_oracle():
    p = build([(0.5, 0.5), (0.25, 0.3)], seed=72)
    model = run_and_check(p, dense=True)
    assert all(lay.attn.dense and lay.ffn.dense for lay in model.layers)
    model.set_dense(False)
    assert not model.layers[0].ffn.dense


def test_adamw_update_matches_oracle():
    p = build([(0.5, 0.5)], seed=73)
    model = run_and_check(p, dense=False)
    blk, master, m, v = model.opt[1]  # the FFN block of layer 0
    p0, g = master.clone(), blk.grads.flat.clone()
    model.optimizer_step(1, 1e-3, weight_decay=0.01)
    torch.cuda.synchronize()
    want, _, _ = oracle.adamw(p0, g, np.zeros(g.numel()), np.zeros(g.numel()), 1, 1e-3, 0.9, 0.999, 1e-8, 0.01)
    np.testing.assert_allclose(master.cpu().numpy(), want, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(blk.params.flat.float().cpu().numpy(), master.cpu().numpy(), rtol=1e-2, atol=1e-6)


def test_keep_table_reading():
    keep = llama3_8b_math10k_keep()
    assert len(keep) == 32
    # layers numbered from 1: L1, L2 dense; FFN 1% kept on L3-L30; QKVO 25% kept on L14-19, 21-23, 25-29
    assert keep[0] == (1.0, 1.0) and keep[1] == (1.0, 1.0) and keep[2] == (1.0, 0.01)
    assert keep[13] == (0.25, 0.01) and keep[19] == (1.0, 0.01) and keep[28] == (0.25, 0.01)
    assert keep[29] == (1.0, 0.01) and keep[30] == (1.0, 1.0)
