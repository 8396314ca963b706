"""Seeded synthetic inputs shared by the CUDA path's tests, the benchmark and the oracle's tests.

This module only draws random numbers and assembles them into tensors with the
shapes, spectra and value distributions of the workloads the SparseLoRA pages
describe (LLaMA-style projections fine-tuned with LoRA). It holds none of the
method's arithmetic: no estimator, criterion, selection, sliced product or
LoRA product is computed here.

Frozen weights are built from a known singular value decomposition so that the
offline rank-k factors the method keeps next to every weight (its offline SVD
step, out of the hot path) can be emitted exactly, in the split the pages give:
W_A = U[:, :k] diag(sqrt(s[:k])) and W_B = diag(sqrt(s[:k])) V[:, :k]^T
("SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
paper-graph-ui walkthrough, section "SVD Sparsity Estimator", pre-computation).

Conventions
-----------
* Weights are returned in nn.Linear storage order, ``W[d_out, d_in]``; the
  pages' math convention is ``W_math = W.T`` with ``y = x W_math``.
* ``W_A`` is ``[d_in, k]`` and ``W_B`` is ``[k, d_out]``, both in the math
  convention, so that ``x @ W_A @ W_B`` approximates ``x @ W.T``.
* LoRA adapters follow the usual layout ``A[r, d_in]``, ``B[d_out, r]``.
* Tokens are produced in sequence order ``[batch * seq, d]`` together with a
  boolean context mask (True = context token, False = output/loss token; the
  last ``n_out`` tokens of every sequence are output tokens).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


def generator(seed: int, device: str | torch.device = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device, dtype):
    return torch.randn(*shape, generator=gen, device=device, dtype=dtype)


def orthonormal_columns(rows: int, cols: int, gen, device="cpu", dtype=torch.float64) -> torch.Tensor:
    """Haar-distributed matrix with orthonormal columns: QR of a Gaussian matrix,
    with the signs fixed so that diag(R) > 0 (which makes Q unique)."""
    g = _randn((rows, cols), gen, device, dtype)
    q, r = torch.linalg.qr(g, mode="reduced")
    d = torch.sign(torch.diagonal(r))
    d[d == 0] = 1
    return q * d.unsqueeze(0)


@dataclass
class SpectralWeight:
    W: torch.Tensor        # [d_out, d_in], storage dtype
    W_A: torch.Tensor      # [d_in, k], storage dtype
    W_B: torch.Tensor      # [k, d_out], storage dtype
    s: torch.Tensor        # singular values, float64 on CPU, descending
    U: torch.Tensor | None = None   # [d_in, r] left singular vectors of W_math (kept only if asked)
    V: torch.Tensor | None = None   # [d_out, r] right singular vectors of W_math


def spectral_weight(d_out: int, d_in: int, alpha: float, k: int, gen, device="cpu",
                    work_dtype=torch.float64, store_dtype=torch.bfloat16,
                    keep_factors: bool = False) -> SpectralWeight:
    """W_math = U diag(s) V^T with random orthonormal U [d_in, r], V [d_out, r] and
    s_i = i^(-alpha), i = 1..r, r = min(d_in, d_out)."""
    r = min(d_in, d_out)
    s = torch.arange(1, r + 1, dtype=torch.float64).pow(-alpha)
    U = orthonormal_columns(d_in, r, gen, device, work_dtype)
    V = orthonormal_columns(d_out, r, gen, device, work_dtype)
    sd = s.to(device=device, dtype=work_dtype)
    W = (V * sd.unsqueeze(0)) @ U.T                       # [d_out, d_in] = W_math^T
    rs = sd[:k].sqrt()
    W_A = U[:, :k] * rs.unsqueeze(0)                      # [d_in, k]
    W_B = rs.unsqueeze(1) * V[:, :k].T                    # [k, d_out]
    out = SpectralWeight(W=W.to(store_dtype), W_A=W_A.to(store_dtype), W_B=W_B.to(store_dtype), s=s)
    if keep_factors:
        out.U, out.V = U, V
    return out


def signed_permutation(w: SpectralWeight, gen) -> SpectralWeight:
    """Another weight of the same spectrum: W' = P_out W P_in^T with random signed permutations
    P_out, P_in (orthogonal), so U' = P_in U and V' = P_out V stay orthonormal and the factors
    move with them (rows of W_A, columns of W_B), exactly, in any storage dtype. One spectral
    draw thus gives distinct per-layer weights without a new orthogonalisation."""
    d_out, d_in = w.W.shape
    dev = w.W.device
    po = torch.randperm(d_out, generator=gen).to(dev)
    pi = torch.randperm(d_in, generator=gen).to(dev)
    so = (torch.randint(0, 2, (d_out,), generator=gen) * 2 - 1).to(device=dev, dtype=w.W.dtype)
    si = (torch.randint(0, 2, (d_in,), generator=gen) * 2 - 1).to(device=dev, dtype=w.W.dtype)
    W = w.W[po][:, pi] * so[:, None] * si[None, :]
    W_A = w.W_A[pi] * si.to(w.W_A.dtype)[:, None]
    W_B = w.W_B[:, po] * so.to(w.W_B.dtype)[None, :]
    return SpectralWeight(W=W.contiguous(), W_A=W_A.contiguous(), W_B=W_B.contiguous(), s=w.s)


def lora_pair(d_out: int, d_in: int, r: int, std: float, gen, device="cpu", dtype=torch.bfloat16):
    """LoRA adapter A [r, d_in], B [d_out, r], both i.i.d. N(0, std^2)."""
    A = _randn((r, d_in), gen, device, torch.float32) * std
    B = _randn((d_out, r), gen, device, torch.float32) * std
    return A.to(dtype), B.to(dtype)


def activations_gaussian_outliers(n_tok: int, d: int, n_outlier: int, factor: float, gen,
                                  device="cpu", dtype=torch.float32) -> torch.Tensor:
    """N(0, 1) activations with ``n_outlier`` randomly chosen input channels scaled by ``factor``."""
    x = _randn((n_tok, d), gen, device, torch.float32)
    ch = torch.randperm(d, generator=gen, device=device)[:n_outlier]
    x[:, ch] *= factor
    return x.to(dtype)


def activations_student_t(n_tok: int, d: int, nu: int, outlier_frac: float, factor: float, gen,
                          device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """Heavy-tailed activations: Student-t with integer ``nu`` degrees of freedom
    (a standard normal over sqrt(chi^2_nu / nu), the chi^2 drawn as a sum of
    ``nu`` squared normals), with round(outlier_frac * d) channels scaled by ``factor``."""
    z = _randn((n_tok, d), gen, device, torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(int(nu)):
        e = _randn((n_tok, d), gen, device, torch.float32)
        chi2.addcmul_(e, e)
    x = z / torch.sqrt(chi2 / nu)
    n_out = int(round(outlier_frac * d))
    ch = torch.randperm(d, generator=gen, device=device)[:n_out]
    x[:, ch] *= factor
    return x.to(dtype)


def context_mask(batch: int, seq: int, n_out: int, device="cpu") -> torch.Tensor:
    """True for context tokens; the last ``n_out`` tokens of every sequence are output tokens."""
    m = torch.ones(batch, seq, dtype=torch.bool, device=device)
    m[:, seq - n_out:] = False
    return m.reshape(-1)


def context_first_order(mask: torch.Tensor) -> torch.Tensor:
    """Row order that lists all context rows first (in sequence order), then all output rows."""
    idx = torch.arange(mask.numel(), device=mask.device)
    return torch.cat([idx[mask], idx[~mask]])


# ---------------------------------------------------------------------------
# Workload configurations (shapes and distributions of the pages' settings)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class FFNConfig:
    name: str
    hidden: int
    inter: int
    batch: int
    seq: int
    n_out: int          # output tokens per sequence
    r: int              # LoRA rank
    k: int              # estimator rank
    ratio: float        # keep ratio
    alpha: float        # spectrum decay s_i = i^-alpha
    lora_std: float = 0.02
    lora_scale: float = 2.0
    fp32: bool = False  # tiny oracle config stores weights/activations in fp32

    @property
    def n_tok(self):
        return self.batch * self.seq


@dataclass(frozen=True)
class AttnConfig:
    name: str
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    batch: int
    seq: int
    n_out: int
    r: int
    k: int
    ratio: float
    alpha: float = 0.5
    lora_std: float = 0.02
    lora_scale: float = 2.0

    @property
    def n_tok(self):
        return self.batch * self.seq


TINY_FFN = FFNConfig("tiny-swiglu-ffn-d256-f688", hidden=256, inter=688, batch=2, seq=64, n_out=16,
                     r=8, k=8, ratio=0.5, alpha=0.7, fp32=True)
LLAMA3_8B_ATTN = AttnConfig("llama3-8b-attn-proj-b8s512", hidden=4096, n_q_heads=32, n_kv_heads=8,
                            head_dim=128, batch=8, seq=512, n_out=128, r=32, k=8, ratio=0.5)
LLAMA3_8B_FFN = FFNConfig("llama3-8b-swiglu-ffn-b8s512", hidden=4096, inter=14336, batch=8, seq=512,
                          n_out=128, r=32, k=8, ratio=0.5, alpha=0.5)
LLAMA2_13B_ATTN = AttnConfig("llama2-13b-attn-proj-b4s1024", hidden=5120, n_q_heads=40, n_kv_heads=40,
                             head_dim=128, batch=4, seq=1024, n_out=256, r=32, k=16, ratio=0.4)
LLAMA2_13B_FFN = FFNConfig("llama2-13b-swiglu-ffn-b4s1024", hidden=5120, inter=13824, batch=4, seq=1024,
                           n_out=256, r=32, k=16, ratio=0.4, alpha=0.5)


def make_ffn_inputs(cfg: FFNConfig, seed: int, device="cpu", work_dtype=None):
    """All inputs of one SwiGLU FFN block fine-tuning step, in sequence token order."""
    gen = generator(seed, device)
    store = torch.float32 if cfg.fp32 else torch.bfloat16
    if work_dtype is None:
        work_dtype = torch.float64 if str(device) == "cpu" else torch.float32
    D, F = cfg.hidden, cfg.inter
    gate = spectral_weight(F, D, cfg.alpha, cfg.k, gen, device, work_dtype, store)
    up = spectral_weight(F, D, cfg.alpha, cfg.k, gen, device, work_dtype, store)
    down = spectral_weight(D, F, cfg.alpha, cfg.k, gen, device, work_dtype, store)
    lg = lora_pair(F, D, cfg.r, cfg.lora_std, gen, device, torch.bfloat16)
    lu = lora_pair(F, D, cfg.r, cfg.lora_std, gen, device, torch.bfloat16)
    ld = lora_pair(D, F, cfg.r, cfg.lora_std, gen, device, torch.bfloat16)
    if cfg.fp32:
        x = activations_gaussian_outliers(cfg.n_tok, D, 4, 20.0, gen, device, torch.float32)
    else:
        x = activations_student_t(cfg.n_tok, D, 4, 0.01, 30.0, gen, device, torch.bfloat16)
    dy = _randn((cfg.n_tok, D), gen, device, torch.float32).to(store)
    mask = context_mask(cfg.batch, cfg.seq, cfg.n_out, device)
    return dict(x=x, dy=dy, ctx_mask=mask, gate=gate, up=up, down=down,
                lora_gate=lg, lora_up=lu, lora_down=ld)


def make_attn_inputs(cfg: AttnConfig, seed: int, device="cpu", work_dtype=None):
    """All inputs of one attention-projection block step (q, k, v, o). The attention
    core itself is not part of the path: its output ``x_o`` (input of o) and the
    gradients ``dq, dk, dv`` it would send back are drawn as synthetic tensors."""
    gen = generator(seed, device)
    if work_dtype is None:
        work_dtype = torch.float64 if str(device) == "cpu" else torch.float32
    D, hd = cfg.hidden, cfg.head_dim
    dq_, dkv = cfg.n_q_heads * hd, cfg.n_kv_heads * hd
    wq = spectral_weight(dq_, D, cfg.alpha, cfg.k, gen, device, work_dtype)
    wk = spectral_weight(dkv, D, cfg.alpha, cfg.k, gen, device, work_dtype)
    wv = spectral_weight(dkv, D, cfg.alpha, cfg.k, gen, device, work_dtype)
    wo = spectral_weight(D, dq_, cfg.alpha, cfg.k, gen, device, work_dtype)
    lq = lora_pair(dq_, D, cfg.r, cfg.lora_std, gen, device)
    lk = lora_pair(dkv, D, cfg.r, cfg.lora_std, gen, device)
    lv = lora_pair(dkv, D, cfg.r, cfg.lora_std, gen, device)
    lo = lora_pair(D, dq_, cfg.r, cfg.lora_std, gen, device)
    x = activations_student_t(cfg.n_tok, D, 4, 0.01, 30.0, gen, device)
    x_o = activations_student_t(cfg.n_tok, dq_, 4, 0.01, 30.0, gen, device)
    dq = _randn((cfg.n_tok, dq_), gen, device, torch.float32).to(torch.bfloat16)
    dk = _randn((cfg.n_tok, dkv), gen, device, torch.float32).to(torch.bfloat16)
    dv = _randn((cfg.n_tok, dkv), gen, device, torch.float32).to(torch.bfloat16)
    dy = _randn((cfg.n_tok, D), gen, device, torch.float32).to(torch.bfloat16)
    mask = context_mask(cfg.batch, cfg.seq, cfg.n_out, device)
    return dict(x=x, x_o=x_o, dq=dq, dk=dk, dv=dv, dy=dy, ctx_mask=mask,
                q=wq, k=wk, v=wv, o=wo, lora_q=lq, lora_k=lk, lora_v=lv, lora_o=lo)


def scaled(cfg, **changes):
    """A copy of a config with some fields replaced (e.g. smaller token counts for tests)."""
    from dataclasses import replace
    return replace(cfg, **changes)
