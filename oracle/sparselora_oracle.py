"""Plain, slow, fp64 CPU oracle of SparseLoRA's sparse frozen-branch linear layer.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module. The product path (the CUDA
library and its binding) never calls it, and it shares no code with them.

Everything here is float64 NumPy, written as the plain definitions the pages
give, in their order and notation, so that it can be checked by eye. Sources
(cited by page title and section):

[WT]  "SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
      paper-graph-ui walkthrough, section 3.4 "Detailed, Sentence-Based
      Technical Breakdown", with its parts "Oracle Sparse Neuron Selection
      Criteria", "SVD Sparsity Estimator" (runtime usage, Algorithm 1; cost
      analysis), "Token Sensitivity and Context-Output Aware Sparsity"
      (Figure 8) and "Putting It All Together"; section 3.2 "Big-Picture
      Architecture" for the backward pass.
[PN]  "SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
      zhaoyang97 Paper-Notes (ICML 2025), section 方法详解 (method details):
      sparse neuron selection criteria and SVD sparsity estimator.

Conventions: the pages write a linear layer as y = x W with
W in R^{D_in x D_out}. This oracle takes weights in nn.Linear storage order,
``W[D_out, D_in]`` and uses ``W_math = W.T``. LoRA: ``A[r, D_in]``,
``B[D_out, r]``, y += scale * (x A^T) B^T. Tokens are rows; ``ctx`` is a
boolean row mask (True = context token, False = output token).

Readings where the pages are silent or ambiguous:
  R1  W_B = diag(sqrt(s_k)) V[:, :k]^T with V the right singular vectors, so
      that W_A W_B is the Eckart-Young rank-k truncation.
  R3  Scores are reduced over the context rows of the layer's own input, all
      sequences of the batch jointly (one index set per batch).
  R4  V/O: scores are the L2 norms of the estimated V output channels; the
      kept V channels keep the matching O input columns (every query head of
      the group under GQA).
  R5  QK under GQA: the selection unit is a KV channel (g, d); its score is
      ||K_hat[:, (g, d)]|| * sum_{h in g} ||Q_hat[:, (h, d)]||. Equal head
      counts reduce this to s = q * k exactly.
  R6  Dropped channels of the frozen branch are zero on context rows; the
      dense LoRA output is added on every row; in the FFN the down
      projection's LoRA sees the full h.
  R7  n = ceil(ratio * N - 1e-9), clamped to [1, N].
  R8  Exactly n channels are kept: order by score descending, ties to the
      lower index, NaN below every number; the kept set is returned ascending.
  R9  The index set is a constant for the backward pass.

  R13 Head-level QK variant (criterion ablation, Table 10): a KV head's score is the sum
      of its head_dim unit scores; whole heads are kept (top n_heads_keep, ties to the lower
      head index) with every channel of the head.
  R14 Wanda-style channel criterion (criterion ablation, Table 10; Wanda's importance
      |W[i, j]| ||X[:, j]||_2): the channel score sums it over the channel's row of the
      frozen weight, over every projection that shares the index set (gate and up), with the
      feature norms over the context rows of the layer input.

  R16 The decoder layer around the projections (NEXT-1): LLaMA's pre-norm layer with RMSNorm
      (frozen gain), causal grouped-query attention without a positional encoding (the pages
      do not say how rotary embeddings meet channel sparsity), residual connections; the
      selections read the normalised layer inputs.
  R17 In the layer, output rows attend to context keys and values computed with the sparse
      projections, as the per-layer split implies (R12).
  R19 The model step's loss is the mean cross-entropy of the LM head's logits over the output
      rows only (next-token targets given per output row); the LM head is frozen.
  R21 Learning rate: cosine decay to 0 at the last step after a linear warm-up over
      ceil(0.04 n_steps) steps (the warm-up reaches the peak at its last step).

Parity unpinned (no printed value or closed form pins them):
the GQA aggregation of R5 and the V-space reading of R4.
"""
from __future__ import annotations

import math

import numpy as np


def f64(a) -> np.ndarray:
    """Upcast a NumPy array or a torch tensor (any float dtype, any device) to float64 NumPy."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        if a.dtype.is_floating_point:
            a = a.double()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Activation
# ---------------------------------------------------------------------------

def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def silu(z):
    """SiLU(z) = z * sigmoid(z) [WT, FFN structure: h = SiLU(x W_gate) * (x W_up)]."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def silu_grad(z):
    """d/dz SiLU(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    z = np.asarray(z, dtype=np.float64)
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


# ---------------------------------------------------------------------------
# Offline factors and the estimator  [WT "SVD Sparsity Estimator"; PN SVD 稀疏估计器]
# ---------------------------------------------------------------------------

def svd_factors(W, k):
    """Offline rank-k factors of a frozen weight (nn.Linear storage W[D_out, D_in]).

    W_math = U S V^T; W_A = U[:, :k] diag(sqrt(S[:k])) in R^{D_in x k};
    W_B = diag(sqrt(S[:k])) V[:, :k]^T in R^{k x D_out} (reading R1).
    Returns (W_A, W_B, S) with S all singular values, descending."""
    Wm = f64(W).T
    U, S, Vt = np.linalg.svd(Wm, full_matrices=False)
    rs = np.sqrt(S[:k])
    W_A = U[:, :k] * rs[None, :]
    W_B = rs[:, None] * Vt[:k, :]
    return W_A, W_B, S


def estimate(X_ctx, W_A, W_B):
    """Low-rank output estimate y_hat = (x W_A) W_B, in that order [WT Algorithm 1]."""
    return (f64(X_ctx) @ f64(W_A)) @ f64(W_B)


# ---------------------------------------------------------------------------
# Criteria  [WT "Oracle Sparse Neuron Selection Criteria"; PN 稀疏神经元选择准则]
# ---------------------------------------------------------------------------

def score_l2(Y):
    """Per-channel L2 norm over all (batch, sequence) rows: s_i = sqrt(sum_t Y[t, i]^2)."""
    Y = f64(Y)
    return np.sqrt(np.sum(Y * Y, axis=0))


def score_swiglu(G, U):
    """FFN criterion: L2 norm per intermediate channel of h = SiLU(G) * U."""
    return score_l2(silu(f64(G)) * f64(U))


def score_qk(Q, K, n_q_heads, n_kv_heads, head_dim):
    """QK criterion s = ||Q||_2 * ||K||_2 per channel, with channel norms taken over
    rows [WT "Computing the QK norm oracle"; PN QK Norm 准则]. Under grouped-query
    attention the unit is a KV channel (g, d) and the query side sums the norms of
    the group's query heads at the same head dimension (reading R5).
    Returns scores over n_kv_heads * head_dim units, unit index g * head_dim + d."""
    return qk_from_sumsq(sumsq(Q), sumsq(K), n_q_heads, n_kv_heads, head_dim)


# ---------------------------------------------------------------------------
# Sufficient statistics for ranks that each hold part of the batch's context rows.
# Every criterion above is built from per-channel sums of squares over the context
# rows, and a sum over all rows is the sum of the sums over disjoint parts of them:
# the ranks add their statistics and every rank then derives the scores of the
# whole batch (one index set per batch, reading R3).
# ---------------------------------------------------------------------------

def sumsq(Y):
    """Per-channel sum of squares over rows: sum_t Y[t, i]^2 (score_l2 before the root)."""
    Y = f64(Y)
    return np.sum(Y * Y, axis=0)


def qk_from_sumsq(q2, k2, n_q_heads, n_kv_heads, head_dim):
    """The QK scores (reading R5) from the per-channel sums of squares of Q_hat and K_hat."""
    q = np.sqrt(f64(q2)).reshape(n_q_heads, head_dim)
    k = np.sqrt(f64(k2)).reshape(n_kv_heads, head_dim)
    group = n_q_heads // n_kv_heads
    q_group = q.reshape(n_kv_heads, group, head_dim).sum(axis=1)
    return (q_group * k).reshape(-1)


def wanda_scores(X_ctx, Ws):
    """Wanda-style channel scores (reading R14): s_i = sum_p sum_j |W_p[i, j]| ||X[:, j]||_2,
    W_p in nn.Linear storage [D_out, D_in], norms over the rows of X_ctx."""
    n = np.sqrt(np.sum(f64(X_ctx) ** 2, axis=0))
    return sum(np.abs(f64(W)) @ n for W in Ws)


# ---------------------------------------------------------------------------
# Selection  [WT Algorithm 1: keep the top ceil(r * D_out) channels; PN top-n]
# ---------------------------------------------------------------------------

def keep_count(ratio, n):
    """n_keep = ceil(ratio * n), guarded against binary rounding, clamped to [1, n] (R7)."""
    c = int(math.ceil(float(ratio) * int(n) - 1e-9))
    return max(1, min(int(n), c))


def select_top(scores, n_keep):
    """Indices of the n_keep largest scores; ties to the lower index, NaN below every
    number (R8). Returned ascending."""
    s = f64(scores)
    n = s.shape[0]
    nan = np.isnan(s)
    neg = np.where(nan, 0.0, -s)            # ascending -s == descending s
    order = np.lexsort((np.arange(n), neg, nan))
    return np.sort(order[:n_keep]).astype(np.int64)


def complement(idx, n):
    mask = np.ones(n, dtype=bool)
    mask[np.asarray(idx, dtype=np.int64)] = False
    return np.nonzero(mask)[0].astype(np.int64)


def expand_units(units, n_q_heads, n_kv_heads, head_dim):
    """Channels of a query-side projection (Q rows, O input columns) kept by a set of
    KV units (g, d): every query head h of group g keeps (h, d) (readings R4, R5).
    Returned ascending."""
    kept = np.zeros(n_kv_heads * head_dim, dtype=bool)
    kept[np.asarray(units, dtype=np.int64)] = True
    group = n_q_heads // n_kv_heads
    out = []
    for h in range(n_q_heads):
        g = h // group
        for d in range(head_dim):
            if kept[g * head_dim + d]:
                out.append(h * head_dim + d)
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# Sparse frozen branch + dense LoRA  [WT Algorithm 1, Figure 8, section 3.2]
# ---------------------------------------------------------------------------

def select_heads(unit_scores, n_kv_heads, head_dim, n_keep_heads):
    """Head-level QK selection (reading R13): head score = sum of its unit scores; the
    n_keep_heads best heads (select_top order) keep all their channels. Returns the kept KV
    channels ascending."""
    h = f64(unit_scores).reshape(n_kv_heads, head_dim).sum(axis=1)
    heads = select_top(h, n_keep_heads)
    return (heads[:, None] * head_dim + np.arange(head_dim)[None, :]).reshape(-1)


def sliced_weight(W, idx, slice_kind):
    """W_math restricted to the kept channels, with dropped channels set to zero:
    'out' keeps output channels (columns of W_math; gate, up, q, k, v),
    'in' keeps input channels (rows of W_math; down, o)."""
    Wm = f64(W).T
    keep = np.zeros(Wm.shape[1] if slice_kind == "out" else Wm.shape[0], dtype=bool)
    keep[np.asarray(idx, dtype=np.int64)] = True
    Wt = np.zeros_like(Wm)
    if slice_kind == "out":
        Wt[:, keep] = Wm[:, keep]
    elif slice_kind == "in":
        Wt[keep, :] = Wm[keep, :]
    else:
        raise ValueError(slice_kind)
    return Wt


def sparse_linear_fwd(X, W, A, B, scale, ctx, idx, slice_kind):
    """y = x W_sliced on context rows, y = x W on output rows, plus the dense LoRA
    output scale * (x A^T) B^T on every row (reading R6)."""
    X = f64(X)
    ctx = np.asarray(ctx, dtype=bool)
    Wm = f64(W).T
    Wt = sliced_weight(W, idx, slice_kind)
    Y = np.empty((X.shape[0], Wm.shape[1]))
    Y[ctx] = X[ctx] @ Wt
    Y[~ctx] = X[~ctx] @ Wm
    Y += scale * (X @ f64(A).T) @ f64(B).T
    return Y


def sparse_linear_bwd(X, dY, W, A, B, scale, ctx, idx, slice_kind):
    """Backward of sparse_linear_fwd with the index set held fixed (R9). The frozen
    weight gets no gradient; the input gradient flows through the kept channels on
    context rows and through the dense weight on output rows; the LoRA gradients are
    dense. Returns (dX, dA, dB)."""
    X, dY = f64(X), f64(dY)
    ctx = np.asarray(ctx, dtype=bool)
    A, B = f64(A), f64(B)
    Wm = f64(W).T
    Wt = sliced_weight(W, idx, slice_kind)
    dX = np.empty_like(X)
    dX[ctx] = dY[ctx] @ Wt.T
    dX[~ctx] = dY[~ctx] @ Wm.T
    xa = X @ A.T                  # [T, r]
    dya = scale * (dY @ B)        # [T, r]
    dX += dya @ A
    dB = scale * dY.T @ xa
    dA = dya.T @ X
    return dX, dA, dB


# ---------------------------------------------------------------------------
# Blocks
# ---------------------------------------------------------------------------

def ffn_select(X, ctx, gate_f, up_f, ratio):
    """FFN estimator + criterion + selection: scores from the estimated SiLU(gate) * up
    on context rows; one index set over the intermediate channels for gate, up and
    down [WT "FFN structure ...", "Putting It All Together"]. gate_f / up_f are
    (W_A, W_B) pairs. Returns (scores, idx)."""
    Xc = f64(X)[np.asarray(ctx, dtype=bool)]
    G_hat = estimate(Xc, *gate_f)
    U_hat = estimate(Xc, *up_f)
    s = score_swiglu(G_hat, U_hat)
    return s, select_top(s, keep_count(ratio, s.shape[0]))


def ffn_fwd(X, ctx, Wg, Wu, Wd, lora_g, lora_u, lora_d, scale, idx):
    """SwiGLU FFN block: G, U through gate/up sliced to idx on output channels,
    H = SiLU(G) * U, Y through down sliced to idx on input channels. lora_* are (A, B)."""
    G = sparse_linear_fwd(X, Wg, *lora_g, scale, ctx, idx, "out")
    U = sparse_linear_fwd(X, Wu, *lora_u, scale, ctx, idx, "out")
    H = silu(G) * U
    Y = sparse_linear_fwd(H, Wd, *lora_d, scale, ctx, idx, "in")
    return dict(G=G, U=U, H=H, Y=Y)


def ffn_bwd(X, dY, ctx, Wg, Wu, Wd, lora_g, lora_u, lora_d, scale, idx, fwd=None):
    """Backward of ffn_fwd for the given output gradient; returns dX and every LoRA gradient."""
    if fwd is None:
        fwd = ffn_fwd(X, ctx, Wg, Wu, Wd, lora_g, lora_u, lora_d, scale, idx)
    G, U, H = fwd["G"], fwd["U"], fwd["H"]
    dH, dA_d, dB_d = sparse_linear_bwd(H, dY, Wd, *lora_d, scale, ctx, idx, "in")
    dG = dH * U * silu_grad(G)
    dU = dH * silu(G)
    dXg, dA_g, dB_g = sparse_linear_bwd(X, dG, Wg, *lora_g, scale, ctx, idx, "out")
    dXu, dA_u, dB_u = sparse_linear_bwd(X, dU, Wu, *lora_u, scale, ctx, idx, "out")
    return dict(dX=dXg + dXu, dH=dH, dG=dG, dU=dU, dA_g=dA_g, dB_g=dB_g, dA_u=dA_u, dB_u=dB_u,
                dA_d=dA_d, dB_d=dB_d)


def attn_select(X, ctx, q_f, k_f, v_f, n_q_heads, n_kv_heads, head_dim, ratio):
    """Attention projections: QK criterion on the estimated Q, K; L2 criterion on the
    estimated V (reading R4); keep counts over the KV units. Returns a dict with the
    scores and the index sets of q, k, v (output channels) and o (input channels)."""
    Xc = f64(X)[np.asarray(ctx, dtype=bool)]
    Q_hat = estimate(Xc, *q_f)
    K_hat = estimate(Xc, *k_f)
    V_hat = estimate(Xc, *v_f)
    s_qk = score_qk(Q_hat, K_hat, n_q_heads, n_kv_heads, head_dim)
    s_v = score_l2(V_hat)
    n_units = n_kv_heads * head_dim
    u_qk = select_top(s_qk, keep_count(ratio, n_units))
    u_v = select_top(s_v, keep_count(ratio, n_units))
    return dict(s_qk=s_qk, s_v=s_v, units_qk=u_qk, units_v=u_v,
                idx_q=expand_units(u_qk, n_q_heads, n_kv_heads, head_dim), idx_k=u_qk,
                idx_v=u_v, idx_o=expand_units(u_v, n_q_heads, n_kv_heads, head_dim))


# ---------------------------------------------------------------------------
# The decoder layer around the sparse projections (NEXT-1): RMSNorm, causal GQA attention,
# residual connections  [WT "Putting It All Together"; R16, R17]
# ---------------------------------------------------------------------------

def rmsnorm(X, gamma, eps):
    """y = x / sqrt(mean_j x_j^2 + eps) * gamma, per row (LLaMA's RMSNorm, frozen gain)."""
    X = f64(X)
    r = 1.0 / np.sqrt(np.mean(X * X, axis=1, keepdims=True) + eps)
    return X * r * f64(gamma)[None, :]


def rmsnorm_bwd(dY, X, gamma, eps):
    """dX of rmsnorm for the upstream gradient dY (the gain is frozen)."""
    X, dY, g = f64(X), f64(dY), f64(gamma)[None, :]
    d = X.shape[1]
    r = 1.0 / np.sqrt(np.mean(X * X, axis=1, keepdims=True) + eps)
    gd = g * dY
    return r * gd - X * r ** 3 * np.sum(X * gd, axis=1, keepdims=True) / d


def attention(Q, K, V, n_seq, n_q_heads, n_kv_heads, head_dim):
    """Causal scaled dot-product attention per sequence (rows sequence-major, n_seq sequences
    of equal length), grouped-query: query head h reads KV head h // (n_q_heads // n_kv_heads).
    Returns (O, P) with P the attention probabilities [n_seq, n_q_heads, S, S]."""
    Q, K, V = f64(Q), f64(K), f64(V)
    T = Q.shape[0]
    S = T // n_seq
    hpg = n_q_heads // n_kv_heads
    O = np.zeros((T, n_q_heads * head_dim))
    P = np.zeros((n_seq, n_q_heads, S, S))
    mask = np.tril(np.ones((S, S), dtype=bool))
    for b in range(n_seq):
        rows = slice(b * S, (b + 1) * S)
        for h in range(n_q_heads):
            g = h // hpg
            q = Q[rows, h * head_dim:(h + 1) * head_dim]
            k = K[rows, g * head_dim:(g + 1) * head_dim]
            v = V[rows, g * head_dim:(g + 1) * head_dim]
            sc = q @ k.T / math.sqrt(head_dim)
            sc = np.where(mask, sc, -np.inf)
            sc = sc - sc.max(axis=1, keepdims=True)
            e = np.exp(sc)
            p = e / e.sum(axis=1, keepdims=True)
            P[b, h] = p
            O[rows, h * head_dim:(h + 1) * head_dim] = p @ v
    return O, P


def attention_bwd(dO, Q, K, V, P, n_seq, n_q_heads, n_kv_heads, head_dim):
    """Gradients of attention() for the upstream gradient dO (softmax backward
    dS = P * (dP - rowsum(dP * P)))."""
    dO, Q, K, V = f64(dO), f64(Q), f64(K), f64(V)
    T = Q.shape[0]
    S = T // n_seq
    hpg = n_q_heads // n_kv_heads
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(n_seq):
        rows = slice(b * S, (b + 1) * S)
        for h in range(n_q_heads):
            g = h // hpg
            qs, ks = slice(h * head_dim, (h + 1) * head_dim), slice(g * head_dim, (g + 1) * head_dim)
            p = P[b, h]
            do = dO[rows, qs]
            dV[rows, ks] += p.T @ do
            dp = do @ V[rows, ks].T
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
            dQ[rows, qs] = ds @ K[rows, ks] / math.sqrt(head_dim)
            dK[rows, ks] += ds.T @ Q[rows, qs] / math.sqrt(head_dim)
    return dQ, dK, dV


def decoder_layer(X, dY, ctx, n_seq, w, lora, gammas, eps, scale, heads, ratio, est_k_factors=None, idx=None):
    """One decoder layer around the sparse projections, forward and backward:
      h1 = rmsnorm(X, g1); q, k, v = sparse projections of h1 (QK / V criteria on h1's context
      rows); O = attention(q, k, v); x2 = X + o(O); h2 = rmsnorm(x2, g2); Y = x2 + FFN(h2)
      (SwiGLU criterion on h2's context rows).
    w: frozen weights {"q","k","v","o","gate","up","down"} (nn.Linear storage); lora: (A, B)
    per projection; heads = (n_q_heads, n_kv_heads, head_dim); est_k_factors: (W_A, W_B) per
    estimated projection (q, k, v, gate, up) for the selection, or idx: fixed index sets
    {"q","k","v","o","ffn"} (e.g. the ones a GPU run chose). Returns the forward values, the
    index sets, dX and every LoRA gradient."""
    hq, hkv, hd = heads
    X = f64(X)
    H1 = rmsnorm(X, gammas[0], eps)
    if idx is None:
        sel = attn_select(H1, ctx, est_k_factors["q"], est_k_factors["k"], est_k_factors["v"], hq, hkv, hd, ratio)
        idx = {"q": sel["idx_q"], "k": sel["idx_k"], "v": sel["idx_v"], "o": sel["idx_o"]}
    Qm = sparse_linear_fwd(H1, w["q"], *lora["q"], scale, ctx, idx["q"], "out")
    Km = sparse_linear_fwd(H1, w["k"], *lora["k"], scale, ctx, idx["k"], "out")
    Vm = sparse_linear_fwd(H1, w["v"], *lora["v"], scale, ctx, idx["v"], "out")
    O, P = attention(Qm, Km, Vm, n_seq, hq, hkv, hd)
    Om = sparse_linear_fwd(O, w["o"], *lora["o"], scale, ctx, idx["o"], "in")
    X2 = X + Om
    H2 = rmsnorm(X2, gammas[1], eps)
    if "ffn" not in idx:
        _, idx["ffn"] = ffn_select(H2, ctx, est_k_factors["gate"], est_k_factors["up"], ratio)
    fwd_f = ffn_fwd(H2, ctx, w["gate"], w["up"], w["down"], lora["gate"], lora["up"], lora["down"], scale, idx["ffn"])
    Y = X2 + fwd_f["Y"]
    # backward
    dY = f64(dY)
    bf = ffn_bwd(H2, dY, ctx, w["gate"], w["up"], w["down"], lora["gate"], lora["up"], lora["down"], scale,
                 idx["ffn"], fwd=fwd_f)
    dX2 = dY + rmsnorm_bwd(bf["dX"], X2, gammas[1], eps)
    dO, dA_o, dB_o = sparse_linear_bwd(O, dX2, w["o"], *lora["o"], scale, ctx, idx["o"], "in")
    dQ, dK, dV = attention_bwd(dO, Qm, Km, Vm, P, n_seq, hq, hkv, hd)
    grads = {"dA_o": dA_o, "dB_o": dB_o, "dA_gate": bf["dA_g"], "dB_gate": bf["dB_g"], "dA_up": bf["dA_u"],
             "dB_up": bf["dB_u"], "dA_down": bf["dA_d"], "dB_down": bf["dB_d"]}
    dH1 = np.zeros_like(H1)
    for n, dm in (("q", dQ), ("k", dK), ("v", dV)):
        dx, da, db = sparse_linear_bwd(H1, dm, w[n], *lora[n], scale, ctx, idx[n], "out")
        dH1 += dx
        grads["dA_" + n], grads["dB_" + n] = da, db
    dX = dX2 + rmsnorm_bwd(dH1, X, gammas[0], eps)
    return dict(Y=Y, dX=dX, H1=H1, H2=H2, X2=X2, O=O, Q=Qm, K=Km, V=Vm, idx=idx, **grads)


def model_step(ids, targets_out, ctx, n_seq, embed, lm_head, gamma_f, layers, eps, scale, heads):
    """Loss and LoRA gradients of a stack of decoder layers (NEXT-2): X_0 = embed[ids]; each
    layer as decoder_layer with its index sets; H = rmsnorm(X_L, gamma_f); cross-entropy of
    H W_lm^T against targets_out on the output rows (mean over them); backward through every
    layer. layers: list of dicts w, lora, gammas, idx. Rows in sequence order; targets_out in
    the order of the output rows. Returns (loss, per-layer gradient dicts)."""
    X = f64(embed)[np.asarray(ids)]
    xs = []
    for L in layers:
        xs.append(X)
        X = decoder_layer(X, np.zeros_like(X), ctx, n_seq, L["w"], L["lora"], L["gammas"], eps, scale, heads, 0.0,
                          idx=dict(L["idx"]))["Y"]
    H = rmsnorm(X, gamma_f, eps)
    out = ~np.asarray(ctx, dtype=bool)
    logits = H[out] @ f64(lm_head).T
    m = logits.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(logits - m).sum(axis=1, keepdims=True)))[:, 0]
    t = np.asarray(targets_out)
    loss = float(np.mean(lse - logits[np.arange(len(t)), t]))
    p = np.exp(logits - lse[:, None])
    p[np.arange(len(t)), t] -= 1.0
    p /= len(t)
    dH = np.zeros_like(H)
    dH[out] = p @ f64(lm_head)
    dX = rmsnorm_bwd(dH, X, gamma_f, eps)
    grads = [None] * len(layers)
    for l in range(len(layers) - 1, -1, -1):
        L = layers[l]
        res = decoder_layer(xs[l], dX, ctx, n_seq, L["w"], L["lora"], L["gammas"], eps, scale, heads, 0.0,
                            idx=dict(L["idx"]))
        grads[l] = res
        dX = res["dX"]
    return loss, grads


def adamw(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    """One AdamW update (decoupled weight decay, bias-corrected moments); returns (p, m, v)."""
    p, g, m, v = f64(p), f64(g), f64(m), f64(v)
    p = p - lr * weight_decay * p
    m = beta1 * m + (1 - beta1) * g
    v = beta2 * v + (1 - beta2) * g * g
    mh = m / (1 - beta1 ** step)
    vh = v / (1 - beta2 ** step)
    return p - lr * mh / (np.sqrt(vh) + eps), m, v


def cosine_lr(step, n_steps, peak, warmup_frac):
    """Learning rate at 1-based `step` of `n_steps` under a cosine schedule with linear warm-up
    ([WT] "Step Sensitivity and Progressive Sparse Fine-Tuning", interaction with the learning
    rate schedule: Table 11's cosine scheduler with a 4% warm-up ratio; reading R21): the rate
    climbs as a straight line from 0 to `peak` across the first ceil(warmup_frac * n_steps)
    steps, then follows half a cosine period from `peak` down to 0 at the last step."""
    n_warm = math.ceil(warmup_frac * n_steps)
    if step <= n_warm:
        return peak * (step / n_warm)
    if n_steps == n_warm:
        return peak
    phase = (step - n_warm) / (n_steps - n_warm)  # 0 just after the warm-up, 1 at the last step
    return peak * (math.cos(math.pi * phase) + 1.0) / 2.0


def dense_lora_reference(X, dY, W, A, B, scale):
    """Dense LoRA layer (keep ratio 1): y = x W + scale (x A^T) B^T and its backward."""
    X = f64(X)
    n = f64(W).shape[0]
    allc = np.ones(X.shape[0], dtype=bool)
    idx = np.arange(n)
    Y = sparse_linear_fwd(X, W, A, B, scale, allc, idx, "out")
    dX, dA, dB = sparse_linear_bwd(X, dY, W, A, B, scale, allc, idx, "out")
    return Y, dX, dA, dB
