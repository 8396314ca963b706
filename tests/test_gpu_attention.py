"""The attention core of the decoder layer (sl_attention_fwd, sl_attention_bwd) against the fp64
oracle's causal grouped-query attention and its backward, on the same bf16 inputs.

Shapes: sequences shorter than one 128-token tile and ragged multi-tile lengths, head dimensions 32,
64 and 128 (below, at and above one 64-element chunk), grouped (GQA) and plain multi-head; the
LLaMA3-8B layer's 8 x 512 tokens with 32 query / 8 key-value heads of 128, and the LLaMA2-13B
layer's 4 x 1024 tokens with 40 heads of 128, checked on a subset of heads that the oracle
computes in full (every sequence, every position). Outputs are bf16: relative Frobenius error at
most 2e-2 per checked head group; element by element within 2e-2 (o, dv) or 1e-1 (dq, dk) of the
value plus the row's RMS."""
import math

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from gpu_helpers import BF16_TOL, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def close(got, want, name, tol=BF16_TOL, elem_tol=BF16_TOL):
    """Relative Frobenius error at most tol, and element by element within elem_tol (|value| + row
    RMS) plus 1e-3 of the matrix RMS (rows that cancel to zero exactly in fp64, e.g. dq of a
    sequence's first query, whose only key is itself, keep the fp32 rounding of dP - D)."""
    g, w = oracle.f64(got), oracle.f64(want)
    rms = np.sqrt(np.mean(w * w, axis=1, keepdims=True))
    floor = 1e-3 * np.sqrt(np.mean(w * w))
    ratio = np.abs(g - w) / (np.abs(w) + rms + floor / elem_tol)
    assert rel_fro(g, w) < tol, f"{name}: relative error {rel_fro(g, w):.3g}"
    bad = ratio > elem_tol
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {ratio.size} elements outside tolerance, worst ratio "
                           f"{ratio.max():.3g} at {np.unravel_index(ratio.argmax(), ratio.shape)}")


def run(n_seq, S, hq, hkv, hd, seed, heads=None):
    g = torch.Generator().manual_seed(seed)
    T = n_seq * S
    q = torch.randn(T, hq * hd, generator=g).to(torch.bfloat16)
    k = torch.randn(T, hkv * hd, generator=g).to(torch.bfloat16)
    v = torch.randn(T, hkv * hd, generator=g).to(torch.bfloat16)
    do = torch.randn(T, hq * hd, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o = torch.full((T, hq * hd), float("nan"), device=DEV, dtype=torch.bfloat16)
    lse = torch.full((hq, T), float("nan"), device=DEV)
    ws = B.Workspace()
    B.sl_attention_fwd(ws, qd, kd, vd, n_seq, hq, hkv, hd, o, lse)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(vd, float("nan"))
    B.sl_attention_bwd(ws, qd, kd, vd, o, dod, lse, n_seq, hq, hkv, hd, dq, dk, dv)
    torch.cuda.synchronize()
    assert ws.read_device_flag() == 0
    hpg = hq // hkv
    groups = sorted(set(range(hkv)) if heads is None else {h // hpg for h in heads})
    for gi in groups:
        hs = list(range(gi * hpg, (gi + 1) * hpg))
        cq = np.concatenate([np.arange(h * hd, (h + 1) * hd) for h in hs])
        ck = np.arange(gi * hd, (gi + 1) * hd)
        Q, K, V, dO = oracle.f64(q)[:, cq], oracle.f64(k)[:, ck], oracle.f64(v)[:, ck], oracle.f64(do)[:, cq]
        O, P = oracle.attention(Q, K, V, n_seq, hpg, 1, hd)
        dQ, dK, dV = oracle.attention_bwd(dO, Q, K, V, P, n_seq, hpg, 1, hd)
        close(o.cpu()[:, cq], O, f"o group {gi}")
        # dS enters the dQ and dK products rounded to bf16 (as P enters P V) and D = rowsum(dO O) is
        # formed from the bf16 O, and each row of dS sums to zero, so dq and dk are sums of
        # cancelling terms: over millions of elements the tail reaches about 5e-2 of the row's scale
        # (an fp64 emulation of those roundings gives the same spread); the whole matrices stay
        # within 2e-2, and a masking or indexing error moves elements by far more than 1e-1
        close(dq.cpu()[:, cq], dQ, f"dq group {gi}", elem_tol=1e-1)
        close(dk.cpu()[:, ck], dK, f"dk group {gi}", elem_tol=1e-1)
        close(dv.cpu()[:, ck], dV, f"dv group {gi}")
        # the row log-sum-exp of the scaled scores, from the oracle's probabilities' normaliser
        Sc = np.zeros((hpg, T))
        for b in range(n_seq):
            rows = slice(b * S, (b + 1) * S)
            for j, h in enumerate(hs):
                s = Q[rows, j * hd:(j + 1) * hd] @ K[rows].T / math.sqrt(hd)
                s = np.where(np.tril(np.ones((S, S), dtype=bool)), s, -np.inf)
                m = s.max(axis=1)
                Sc[j, rows] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        np.testing.assert_allclose(lse.cpu().numpy()[hs], Sc, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("n_seq,S,hq,hkv,hd", [(2, 64, 4, 2, 32), (3, 40, 2, 2, 64), (2, 300, 4, 1, 128),
                                                (1, 257, 2, 2, 128), (2, 128, 6, 3, 96), (2, 200, 4, 2, 40),
                                                (1, 130, 2, 1, 8)])
def test_attention_matches_oracle(n_seq, S, hq, hkv, hd):
    run(n_seq, S, hq, hkv, hd, seed=S + hd)


@pytest.mark.parametrize("n_seq,S,hq,hkv,hd,heads", [(8, 512, 32, 8, 128, (0, 13, 31)), (4, 1024, 40, 40, 128, (0, 39))],
                         ids=["llama3-8b", "llama2-13b"])
def test_attention_full_size(n_seq, S, hq, hkv, hd, heads):
    run(n_seq, S, hq, hkv, hd, seed=7, heads=heads)
