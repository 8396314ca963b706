"""A whole fine-tuning step of a LLaMA-style model with SparseLoRA ([WT] "Putting It All
Together"; "Layer Sensitivity Analysis" for the per-layer ratios; "Step Sensitivity and
Progressive Sparse Fine-Tuning" for the dense first steps):

    x = embedding[ids]; for each layer: x = DecoderLayer(x) with the layer's keep ratios;
    logits = RMSNorm(x) W_lm^T on the output rows; loss = cross-entropy(logits, targets);
    backward through every layer; AdamW on every LoRA matrix.

Per-layer keep ratios (attention q/k/v/o, FFN) come from a table; the first steps of a run are
dense (progressive schedule). Every projection, RMSNorm, residual, the embedding gather and
AdamW run in libsparselora's kernels; the attention core and the frozen LM head's product with
its cross-entropy are torch library calls (like cuBLAS), outside the method's steps."""
from __future__ import annotations

import math

import torch

from . import binding as B
from .blocks import AttnProjBlock, FFNBlock
from .layer import DecoderLayer


def llama3_8b_math10k_keep(n_layers: int = 32):
    """Keep ratios per layer (attention, FFN) from the walkthrough's reading of the LLaMA3-8B /
    Math10K configuration ([WT] "Converting sensitivity curves to sparsity configurations"): FFN
    sparsity 99% on layers L3-L30, QKVO sparsity 75% on L14-L19, L21-L23, L25-L29, the other
    layers dense (layers numbered from 1)."""
    out = []
    for i in range(1, n_layers + 1):
        ffn = 0.01 if 3 <= i <= 30 else 1.0
        attn = 0.25 if (14 <= i <= 19 or 21 <= i <= 23 or 25 <= i <= 29) else 1.0
        out.append((attn, ffn))
    return out


def layerwise_keep(n_layers: int = 32, dense_layers: int = 8, mid_end: int = 20, mid_keep: float = 0.6,
                   deep_keep: float = 0.35):
    """A non-uniform keep table over a 32-layer LLaMA3-8B (layers numbered from 0): layers
    0-7 dense, 8-19 at keep 0.6, 20-31 at keep 0.35, the same ratio on the attention
    projections and the FFN ([WT] "Layer Sensitivity Analysis and Non-Uniform Sparsity":
    deeper layers tolerate more sparsity, so shallow layers stay dense)."""
    out = []
    for i in range(n_layers):
        k = 1.0 if i < dense_layers else (mid_keep if i < mid_end else deep_keep)
        out.append((k, k))
    return out


def cosine_lr(step: int, n_steps: int, peak: float, warmup_frac: float = 0.04) -> float:
    """Learning rate of 1-based `step` of `n_steps` ([WT] "Step Sensitivity and Progressive
    Sparse Fine-Tuning", the schedule of Table 11): linear warm-up to `peak` over the first
    ceil(warmup_frac * n_steps) steps, then cosine decay to 0 at the last step."""
    n_warm = math.ceil(warmup_frac * n_steps)
    if step <= n_warm:
        return peak * step / n_warm
    if n_steps == n_warm:
        return peak
    t = (step - n_warm) / (n_steps - n_warm)
    return 0.5 * peak * (1.0 + math.cos(math.pi * t))


class SparseLoRAModel:
    def __init__(self, frozen, loras, gammas, keep, perm, n_ctx, n_seq, heads, est_k, lora_scale, device="cuda",
                 eps=1e-5):
        """frozen: dict with "embed" [V, D], "lm_head" [V, D], "gamma_f" [D] and the projection
        weights "q","k","v","o","gate","up","down" (SpectralWeight-like: .W, .W_A, .W_B), shared by
        every layer or a list of such dicts (one per layer); loras: per layer a dict of (A, B);
        gammas: per layer (g1, g2); keep: per layer (attn_keep, ffn_keep); perm: context-first
        row order of the batch (n_seq sequences); heads: (n_q_heads, n_kv_heads, head_dim)."""
        bf = torch.bfloat16
        self.device = device
        self.eps = eps
        self.n_layers = len(keep)
        self.keep = list(keep)
        hq, hkv, hd = heads
        T = len(perm)
        self.T, self.C = T, n_ctx
        self.embed = frozen["embed"].to(device=device, dtype=bf).contiguous()
        self.lm_head = frozen["lm_head"].to(device=device, dtype=bf).contiguous()
        self.gamma_f = frozen["gamma_f"].to(device=device, dtype=bf).contiguous()
        self.D = self.embed.shape[1]
        self.layers = []
        for i in range(self.n_layers):
            w = frozen["layers"][i] if "layers" in frozen else frozen
            lo = loras[i]
            attn = AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], lora_scale, est_k,
                                 hq, hkv, hd, T, n_ctx, keep[i][0], device, io_layout="sigma")
            ffn = FFNBlock(w["gate"], w["up"], w["down"], lo["gate"], lo["up"], lo["down"], lora_scale, est_k, T, n_ctx,
                           keep[i][1], device)
            self.layers.append(DecoderLayer(attn, ffn, gammas[i][0], gammas[i][1], perm, n_seq, eps))
        # fp32 master copies of every LoRA matrix and their AdamW moments, in the blocks' flat layout
        self.opt = []
        for lay in self.layers:
            for blk in (lay.attn, lay.ffn):
                master = blk.params.flat.float()
                self.opt.append((blk, master, torch.zeros_like(master), torch.zeros_like(master)))
        e = lambda *sh, dt=bf: torch.empty(*sh, dtype=dt, device=device)
        self.x0 = e(T, self.D)
        self.hf, self.dhf, self.dx_top = e(T, self.D), e(T, self.D), e(T, self.D)
        self.rstd_f = e(T, dt=torch.float32)
        self.loss = torch.zeros((), dtype=torch.float32, device=device)

    def set_dense(self, on: bool):
        for lay in self.layers:
            lay.attn.set_dense(on)
            lay.ffn.set_dense(on)

    def forward_backward(self, ids_cf, targets_out):
        """ids_cf: int32 [T] token ids in context-first order; targets_out: int64 [T - C], the
        next-token targets of the output rows (rows C..T-1 of the context-first order)."""
        B.sl_permute_rows(self.embed, ids_cf, self.x0)
        x = self.x0
        for lay in self.layers:
            x = lay.forward(x)
        self.x_top = x
        B.sl_rmsnorm_fwd(x, self.gamma_f, self.eps, self.hf, self.rstd_f)
        h_out = self.hf[self.C:]
        logits = torch.matmul(h_out, self.lm_head.t()).float()
        n_out = logits.shape[0]
        lse = torch.logsumexp(logits, dim=1)
        self.loss.copy_((lse - logits.gather(1, targets_out[:, None])[:, 0]).mean())
        dlogits = torch.softmax(logits, dim=1)
        dlogits[torch.arange(n_out, device=logits.device), targets_out] -= 1.0
        dlogits /= n_out
        self.dhf.zero_()
        self.dhf[self.C:] = torch.matmul(dlogits.to(torch.bfloat16), self.lm_head)
        B.sl_rmsnorm_bwd(self.dhf, x, self.gamma_f, self.rstd_f, self.dx_top)
        dx = self.dx_top
        for lay in reversed(self.layers):
            dx = lay.backward(dx)
        return self.loss

    def optimizer_step(self, step: int, lr: float, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0):
        for blk, master, m, v in self.opt:
            B.sl_adamw_step(master, blk.grads.flat, m, v, step, lr, betas[0], betas[1], eps, weight_decay,
                            params_bf16=blk.params.flat)

    def step(self, ids_cf, targets_out, step: int, n_steps: int, lr: float, dense_frac: float = 0.1,
             warmup_frac: float = 0.04):
        """One fine-tuning step (1-based `step` of `n_steps`): dense while step <= ceil(dense_frac *
        n_steps), then with the per-layer keep ratios; AdamW at the cosine schedule's rate for
        this step, peak `lr`."""
        self.set_dense(step <= math.ceil(dense_frac * n_steps))
        loss = self.forward_backward(ids_cf, targets_out)
        self.optimizer_step(step, cosine_lr(step, n_steps, lr, warmup_frac))
        return loss
