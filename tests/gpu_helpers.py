"""Shared helpers of the GPU parity tests: seeded problem construction and comparisons."""
import numpy as np
import torch

import oracle
from contextual_sparsity_lora_b200 import inputs

BF16_TOL = 2e-2   # relative Frobenius error, outputs rounded through bf16 tensor-core GEMMs
FP32_TOL = 1e-5   # relative Frobenius error, fp32 accumulations of exact inputs (scores, x A^T)


def rel_fro(got, want) -> float:
    got, want = oracle.f64(got), oracle.f64(want)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def unsigma(t, sigma, n_ctx):
    """Natural-layout copy of a sigma-layout activation (context rows permuted by sigma)."""
    out = oracle.f64(t).copy()
    sig = sigma.cpu().numpy().astype(np.int64)
    ctx = out[:n_ctx].copy()
    nat = np.empty_like(ctx)
    nat[:, sig] = ctx
    out[:n_ctx] = nat
    return out


def ffn_problem(T, n_ctx, D, F, r, k, seed, zero_b=False, alpha=0.5, device="cuda"):
    """Weights and tensors of a SwiGLU FFN step in context-first row order."""
    gen = inputs.generator(seed)
    gate = inputs.spectral_weight(F, D, alpha, k, gen, "cpu", torch.float64, torch.bfloat16)
    up = inputs.spectral_weight(F, D, alpha, k, gen, "cpu", torch.float64, torch.bfloat16)
    down = inputs.spectral_weight(D, F, alpha, k, gen, "cpu", torch.float64, torch.bfloat16)
    lg = inputs.lora_pair(F, D, r, 0.02, gen)
    lu = inputs.lora_pair(F, D, r, 0.02, gen)
    ld = inputs.lora_pair(D, F, r, 0.02, gen)
    if zero_b:
        lg, lu, ld = ((a, torch.zeros_like(b)) for a, b in (lg, lu, ld))
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, D, generator=gen).to(torch.bfloat16)
    ctx = np.zeros(T, dtype=bool)
    ctx[:n_ctx] = True
    return dict(gate=gate, up=up, down=down, lg=lg, lu=lu, ld=ld, x=x, dy=dy, ctx=ctx)


def attn_problem(T, n_ctx, D, hq, hkv, hd, r, k, seed, zero_b=False, alpha=0.5):
    gen = inputs.generator(seed)
    Dq, Dkv = hq * hd, hkv * hd
    w = {n: inputs.spectral_weight(do, di, alpha, k, gen, "cpu", torch.float64, torch.bfloat16)
         for n, do, di in (("q", Dq, D), ("k", Dkv, D), ("v", Dkv, D), ("o", D, Dq))}
    lo = {}
    for n, do, di in (("q", Dq, D), ("k", Dkv, D), ("v", Dkv, D), ("o", D, Dq)):
        a, b = inputs.lora_pair(do, di, r, 0.02, gen)
        lo[n] = (a, torch.zeros_like(b) if zero_b else b)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    x_o = inputs.activations_student_t(T, Dq, 4, 0.01, 30.0, gen)
    g = {n: torch.randn(T, d, generator=gen).to(torch.bfloat16) for n, d in (("dq", Dq), ("dk", Dkv), ("dv", Dkv),
                                                                              ("dy", D))}
    ctx = np.zeros(T, dtype=bool)
    ctx[:n_ctx] = True
    return dict(w=w, lora=lo, x=x, x_o=x_o, ctx=ctx, **g)
