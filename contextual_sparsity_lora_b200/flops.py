"""Algorithmic work of one SparseLoRA layer step (host-side accounting for the benchmark).

Counts follow the definitions of the path, not what a kernel happens to execute
(padding, zero-filled tails and recomputation are not counted):

* frozen branch, one projection, forward + input-gradient backward:
  4 * D_in * D_out * T_out  (dense output rows)  +  4 * D_in * n_kept * T_ctx
  (the kept channels on context rows); no weight gradient is formed.
* LoRA, one projection, forward + backward: 6 * T * r * (D_in + D_out)
  (x A^T, (xA^T) B^T, dy B, dy^T xa, dya^T x, dya A).
* estimator (forward only, context rows): 2 * T_ctx * k * (D_in + D_out) per
  estimated projection, the cost the pages give.

Cost model of the estimator ("SparseLoRA: Accelerating LLM Fine-Tuning with
Contextual Sparsity", paper-graph-ui walkthrough, section "SVD Sparsity
Estimator", cost analysis): low-rank over dense is k (D_in + D_out) / (D_in D_out).
Dense warm-up bound (same page, "Step Sensitivity and Progressive Sparse
Fine-Tuning"): overall speedup 1 / (p + (1 - p) / s).
"""
from __future__ import annotations


def estimator_cost_ratio(d_in: int, d_out: int, k: int) -> float:
    return k * (d_in + d_out) / (d_in * d_out)


def dense_warmup_speedup_bound(p: float, s: float) -> float:
    return 1.0 / (p + (1.0 - p) / s)


def estimator_factor_bytes(n_layers: int, projections, k: int, bytes_per_param: int = 2) -> int:
    """Memory of the offline rank-k factors W_A [d_in, k] and W_B [k, d_out]: k (d_in + d_out)
    parameters per estimated projection (same page, memory overhead), over `n_layers` layers
    with the (d_in, d_out) pairs in `projections`."""
    return n_layers * sum(k * (di + do) for di, do in projections) * bytes_per_param


def frozen_fwd_bwd(d_in: int, d_out: int, n_tok: int, n_ctx: int, n_kept_of_sliced_side: int,
                   sliced_side_size: int) -> float:
    """Frozen-branch FLOPs of one projection; the kept count is on the sliced side
    (output channels or input channels), whose full size is ``sliced_side_size``."""
    full = 2.0 * d_in * d_out
    frac = n_kept_of_sliced_side / sliced_side_size
    return 2.0 * full * ((n_tok - n_ctx) + n_ctx * frac)


def lora_fwd_bwd(d_in: int, d_out: int, n_tok: int, r: int) -> float:
    return 6.0 * n_tok * r * (d_in + d_out)


def estimator(d_in: int, d_outs, n_ctx: int, k: int) -> float:
    return sum(2.0 * n_ctx * k * (d_in + d) for d in d_outs)


def ffn_block(hidden: int, inter: int, n_tok: int, n_ctx: int, n_keep: int, r: int, k: int,
              with_estimator: bool = True) -> dict:
    main = 2 * frozen_fwd_bwd(hidden, inter, n_tok, n_ctx, n_keep, inter) \
        + frozen_fwd_bwd(inter, hidden, n_tok, n_ctx, n_keep, inter)
    lora = 2 * lora_fwd_bwd(hidden, inter, n_tok, r) + lora_fwd_bwd(inter, hidden, n_tok, r)
    est = estimator(hidden, (inter, inter), n_ctx, k) if with_estimator else 0.0
    return dict(main=main, lora=lora, estimator=est, total=main + lora + est)


def attn_proj_block(hidden: int, n_q_heads: int, n_kv_heads: int, head_dim: int, n_tok: int,
                    n_ctx: int, n_keep_units: int, n_keep_units_v: int, r: int, k: int,
                    with_estimator: bool = True) -> dict:
    dq, dkv = n_q_heads * head_dim, n_kv_heads * head_dim
    units = n_kv_heads * head_dim
    main = frozen_fwd_bwd(hidden, dq, n_tok, n_ctx, n_keep_units, units) \
        + frozen_fwd_bwd(hidden, dkv, n_tok, n_ctx, n_keep_units, units) \
        + frozen_fwd_bwd(hidden, dkv, n_tok, n_ctx, n_keep_units_v, units) \
        + frozen_fwd_bwd(dq, hidden, n_tok, n_ctx, n_keep_units_v, units)
    lora = lora_fwd_bwd(hidden, dq, n_tok, r) + 2 * lora_fwd_bwd(hidden, dkv, n_tok, r) \
        + lora_fwd_bwd(dq, hidden, n_tok, r)
    est = estimator(hidden, (dq, dkv, dkv), n_ctx, k) if with_estimator else 0.0
    return dict(main=main, lora=lora, estimator=est, total=main + lora + est)


def lora_skinny_bytes(ops) -> float:
    """Minimum HBM bytes of the LoRA products that are not fused into the sliced GEMMs
    (x A^T, dy B, dy^T xa, dya^T x): every large operand read once per direction.
    ops: (n_tok, d_in, (d_out, ...)) per group of adapters sharing one input; bf16."""
    total = 0.0
    for n_tok, d_in, d_outs in ops:
        total += 2.0 * n_tok * d_in * 2          # x: forward (x A^T) and backward (dya^T x)
        total += sum(2.0 * n_tok * d for d in d_outs)  # dy: read once for dy B and dy^T xa
    return total

