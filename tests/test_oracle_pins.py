"""Pins of the fp64 oracle against what the SparseLoRA pages and the mathematics fix:
worked examples computed by hand (tests/golden/worked_examples.json), closed forms
(Eckart-Young, full-rank estimator), special cases (keep ratio 1 = dense LoRA, equal
head counts = MHA formula), brute force on tiny inputs and central finite differences.
No GPU is needed."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def arr(x):
    return np.asarray([[float(v) for v in row] for row in x]) if isinstance(x[0], list) else \
        np.asarray([float(v) for v in x])


# --------------------------------------------------------------------------- worked examples

def test_l2_norm_worked_example():
    g = GOLD["l2_norm"]
    np.testing.assert_allclose(oracle.score_l2(arr(g["Y"])), g["scores"], rtol=0, atol=1e-15)


def test_qk_norm_worked_example_mha():
    g = GOLD["qk_norm"]
    s = oracle.score_qk(arr(g["Q"]), arr(g["K"]), n_q_heads=1, n_kv_heads=1, head_dim=2)
    np.testing.assert_allclose(s, g["scores"], rtol=0, atol=1e-15)


def test_qk_norm_worked_example_gqa():
    g = GOLD["qk_norm_gqa"]
    s = oracle.score_qk(arr(g["Q"]), arr(g["K"]), g["n_q_heads"], g["n_kv_heads"], g["head_dim"])
    np.testing.assert_allclose(s, g["scores"], rtol=0, atol=1e-15)


def test_silu_values():
    g = GOLD["silu"]
    np.testing.assert_allclose(oracle.silu(np.array(g["z"])), g["value"], rtol=1e-15, atol=0)


def test_select_worked_example():
    g = GOLD["select_top"]
    s = np.array([float(v) for v in g["scores"]])
    for n, want in g["cases"]:
        assert oracle.select_top(s, n).tolist() == want


def test_keep_count_worked_examples():
    for ratio, n, want in GOLD["keep_count"]["cases"]:
        assert oracle.keep_count(ratio, n) == want


@pytest.mark.parametrize("name", ["linear_out_slice", "linear_in_slice"])
def test_linear_worked_example(name):
    g = GOLD[name]
    kind = "out" if name == "linear_out_slice" else "in"
    X, W, A, B = (arr(g[k]) for k in ("X", "W", "A", "B"))
    ctx = np.array(g["ctx"])
    Y = oracle.sparse_linear_fwd(X, W, A, B, g["scale"], ctx, g["idx"], kind)
    np.testing.assert_allclose(Y, arr(g["Y"]), rtol=0, atol=1e-14)
    if "dY" in g:
        dX, dA, dB = oracle.sparse_linear_bwd(X, arr(g["dY"]), W, A, B, g["scale"], ctx, g["idx"], kind)
        np.testing.assert_allclose(dX, arr(g["dX"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(dA, arr(g["dA"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(dB, arr(g["dB"]), rtol=0, atol=1e-14)


# --------------------------------------------------------------------------- estimator / factors

def _f64_weight(d_out, d_in, alpha, k, seed):
    gen = inputs.generator(seed)
    return inputs.spectral_weight(d_out, d_in, alpha, k, gen, "cpu", torch.float64, torch.float64,
                                  keep_factors=True)


@pytest.mark.parametrize("shape", [(96, 40), (40, 96), (64, 64)])
def test_svd_factors_recover_known_spectrum(shape):
    d_out, d_in = shape
    k = 8
    w = _f64_weight(d_out, d_in, 0.7, k, seed=3)
    W_A, W_B, S = oracle.svd_factors(w.W, k)
    s = w.s.numpy()
    np.testing.assert_allclose(S, s, rtol=1e-12, atol=1e-14)
    # W_A W_B is the rank-k truncation U_k S_k V_k^T (sign flips of singular vectors cancel)
    Uk, Vk = w.U.numpy()[:, :k], w.V.numpy()[:, :k]
    np.testing.assert_allclose(W_A @ W_B, (Uk * s[:k]) @ Vk.T, rtol=0, atol=1e-12)
    # the generator's emitted factors give the same product
    np.testing.assert_allclose(w.W_A.numpy() @ w.W_B.numpy(), W_A @ W_B, rtol=0, atol=1e-12)
    # Eckart-Young: squared Frobenius error of the truncation = sum of the discarded s_i^2
    err = np.sum((oracle.f64(w.W).T - W_A @ W_B) ** 2)
    assert err == pytest.approx(np.sum(s[k:] ** 2), rel=1e-10)


def test_full_rank_estimator_equals_dense_output():
    """With k = min(D_in, D_out) the estimate is x W exactly, so estimated scores are the
    oracle criterion on true activations."""
    d_out, d_in = 48, 32
    w = _f64_weight(d_out, d_in, 0.5, min(d_in, d_out), seed=5)
    x = np.random.default_rng(1).standard_normal((20, d_in))
    Y = x @ oracle.f64(w.W).T
    Yh = oracle.estimate(x, w.W_A, w.W_B)
    np.testing.assert_allclose(Yh, Y, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.score_l2(Yh), oracle.score_l2(Y), rtol=1e-12)


def test_estimate_order_is_associative_product():
    rng = np.random.default_rng(2)
    x, wa, wb = rng.standard_normal((7, 11)), rng.standard_normal((11, 3)), rng.standard_normal((3, 13))
    np.testing.assert_allclose(oracle.estimate(x, wa, wb), x @ (wa @ wb), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- criteria

def test_l2_closed_form_constant_columns():
    c = np.array([0.0, -2.0, 3.5, 1e-3])
    T = 37
    Y = np.ones((T, 1)) * c[None, :]
    np.testing.assert_allclose(oracle.score_l2(Y), np.abs(c) * math.sqrt(T), rtol=1e-14)


def test_swiglu_criterion_special_cases():
    T = 9
    G = np.zeros((T, 3))
    G[:, 1] = 50.0       # SiLU(50) = 50 to fp64 precision
    G[:, 2] = -50.0      # SiLU(-50) ~ -50 e^-50
    U = np.full((T, 3), 2.0)
    s = oracle.score_swiglu(G, U)
    assert s[0] == 0.0
    assert s[1] == pytest.approx(100.0 * math.sqrt(T), rel=1e-14)
    assert s[2] == pytest.approx(100.0 * math.exp(-50.0) * math.sqrt(T), rel=1e-10)


def test_qk_group_size_one_is_mha_formula():
    rng = np.random.default_rng(4)
    Q, K = rng.standard_normal((15, 12)), rng.standard_normal((15, 12))
    s = oracle.score_qk(Q, K, n_q_heads=3, n_kv_heads=3, head_dim=4)
    q = np.sqrt((Q ** 2).sum(0))
    k = np.sqrt((K ** 2).sum(0))
    np.testing.assert_allclose(s, q * k, rtol=1e-14)


def test_qk_gqa_is_sum_over_group():
    rng = np.random.default_rng(6)
    nq, nkv, hd = 4, 2, 3
    Q, K = rng.standard_normal((10, nq * hd)), rng.standard_normal((10, nkv * hd))
    s = oracle.score_qk(Q, K, nq, nkv, hd)
    for g in range(nkv):
        for d in range(hd):
            qs = sum(np.linalg.norm(Q[:, h * hd + d]) for h in range(g * 2, g * 2 + 2))
            assert s[g * hd + d] == pytest.approx(qs * np.linalg.norm(K[:, g * hd + d]), rel=1e-13)


def test_gram_identity_for_linear_criteria():
    """sum_t (Z b_i)_t^2 = b_i^T (Z^T Z) b_i: the token reduction of a linear criterion
    collapses to a k x k Gram matrix (exact algebra)."""
    rng = np.random.default_rng(7)
    Z, Wb = rng.standard_normal((50, 8)), rng.standard_normal((8, 30))
    G = Z.T @ Z
    quad = np.einsum("ki,kl,li->i", Wb, G, Wb)
    np.testing.assert_allclose(np.sqrt(quad), oracle.score_l2(Z @ Wb), rtol=1e-12)


# --------------------------------------------------------------------------- selection

def _brute_force_valid(scores, n, idx):
    """Every kept score beats every dropped one under (score desc, index asc, NaN last)."""
    def key(i):
        v = scores[i]
        return (1, 0.0, i) if math.isnan(v) else (0, -v, i)
    kept = set(idx.tolist())
    assert len(kept) == n == len(idx)
    assert list(idx) == sorted(idx)
    worst_kept = max(key(i) for i in kept)
    for j in range(len(scores)):
        if j not in kept:
            assert key(j) > worst_kept


def test_select_brute_force_tiny_exhaustive():
    vals = [0.0, 1.0, 1.0, float("nan"), -float("inf"), 2.5]
    for perm in set(itertools.permutations(vals)):
        s = np.array(perm)
        for n in range(1, len(s) + 1):
            _brute_force_valid(s, n, oracle.select_top(s, n))


def test_select_brute_force_random_with_duplicates():
    rng = np.random.default_rng(8)
    for trial in range(200):
        N = int(rng.integers(1, 40))
        s = rng.integers(0, 5, N).astype(float)     # many ties
        n = int(rng.integers(1, N + 1))
        idx = oracle.select_top(s, n)
        _brute_force_valid(s, n, idx)
        # reference by full sort on (score desc, index asc)
        order = sorted(range(N), key=lambda i: (-s[i], i))[:n]
        assert idx.tolist() == sorted(order)


def test_expand_units_mha_identity_and_gqa():
    u = np.array([0, 3, 5])
    np.testing.assert_array_equal(oracle.expand_units(u, 2, 2, 3), u)
    # 4 query heads over 2 KV heads, head_dim 3: unit (g=0, d=0) -> heads 0,1 at d=0; (1, 2) -> heads 2,3 at d=2
    got = oracle.expand_units(np.array([0, 5]), 4, 2, 3)
    assert got.tolist() == [0, 3, 8, 11]


# --------------------------------------------------------------------------- sparse linear

def _rand_linear(rng, T, d_in, d_out, r):
    return (rng.standard_normal((T, d_in)), rng.standard_normal((d_out, d_in)),
            rng.standard_normal((r, d_in)), rng.standard_normal((d_out, r)), rng.standard_normal((T, d_out)))


@pytest.mark.parametrize("kind", ["out", "in"])
def test_sliced_equals_compact_submatrix_product(kind):
    """Kept channels form a dense submatrix: compute it on the compact submatrix and
    compare with the masked-weight definition."""
    rng = np.random.default_rng(9)
    T, d_in, d_out, r = 12, 10, 14, 3
    X, W, A, B, dY = _rand_linear(rng, T, d_in, d_out, r)
    ctx = np.ones(T, dtype=bool)
    n_side = d_out if kind == "out" else d_in
    idx = np.sort(rng.choice(n_side, 5, replace=False))
    Y = oracle.sparse_linear_fwd(X, W, A, B, 0.0, ctx, idx, kind)
    Wm = W.T
    if kind == "out":
        want = np.zeros((T, d_out))
        want[:, idx] = X @ Wm[:, idx]
    else:
        want = X[:, idx] @ Wm[idx, :]
    np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["out", "in"])
def test_output_rows_do_not_depend_on_index_set(kind):
    rng = np.random.default_rng(10)
    T, d_in, d_out, r = 16, 9, 11, 2
    X, W, A, B, dY = _rand_linear(rng, T, d_in, d_out, r)
    ctx = rng.random(T) < 0.6
    n_side = d_out if kind == "out" else d_in
    i1, i2 = np.array([0, 1]), np.arange(n_side)
    y1 = oracle.sparse_linear_fwd(X, W, A, B, 1.5, ctx, i1, kind)
    y2 = oracle.sparse_linear_fwd(X, W, A, B, 1.5, ctx, i2, kind)
    np.testing.assert_array_equal(y1[~ctx], y2[~ctx])
    g1 = oracle.sparse_linear_bwd(X, dY, W, A, B, 1.5, ctx, i1, kind)[0]
    g2 = oracle.sparse_linear_bwd(X, dY, W, A, B, 1.5, ctx, i2, kind)[0]
    np.testing.assert_array_equal(g1[~ctx], g2[~ctx])


def test_keep_ratio_one_is_dense_lora():
    rng = np.random.default_rng(11)
    T, d_in, d_out, r = 13, 8, 6, 2
    X, W, A, B, dY = _rand_linear(rng, T, d_in, d_out, r)
    ctx = rng.random(T) < 0.5
    Y, dX, dA, dB = oracle.dense_lora_reference(X, dY, W, A, B, 2.0)
    for kind, n in (("out", d_out), ("in", d_in)):
        idx = np.arange(n)
        np.testing.assert_allclose(oracle.sparse_linear_fwd(X, W, A, B, 2.0, ctx, idx, kind), Y, rtol=1e-13)
        got = oracle.sparse_linear_bwd(X, dY, W, A, B, 2.0, ctx, idx, kind)
        for a, b in zip(got, (dX, dA, dB)):
            np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("kind", ["out", "in"])
def test_linear_backward_matches_finite_differences(kind):
    rng = np.random.default_rng(12)
    T, d_in, d_out, r = 6, 5, 7, 2
    X, W, A, B, dY = _rand_linear(rng, T, d_in, d_out, r)
    ctx = np.array([True, True, False, True, False, True])
    n_side = d_out if kind == "out" else d_in
    idx = np.array([1, 3, 4])
    assert idx.max() < n_side

    def loss():
        return float(np.sum(dY * oracle.sparse_linear_fwd(X, W, A, B, 0.7, ctx, idx, kind)))
    dX, dA, dB = oracle.sparse_linear_bwd(X, dY, W, A, B, 0.7, ctx, idx, kind)
    np.testing.assert_allclose(dX, _fd(loss, X), rtol=1e-7, atol=1e-7)
    np.testing.assert_allclose(dA, _fd(loss, A), rtol=1e-7, atol=1e-7)
    np.testing.assert_allclose(dB, _fd(loss, B), rtol=1e-7, atol=1e-7)


def test_silu_grad_matches_finite_differences():
    z = np.linspace(-8, 8, 33)
    fd = (oracle.silu(z + 1e-6) - oracle.silu(z - 1e-6)) / 2e-6
    np.testing.assert_allclose(oracle.silu_grad(z), fd, rtol=1e-7, atol=1e-9)


# --------------------------------------------------------------------------- FFN block

def _tiny_ffn(seed=0, T=10, D=6, F=9, r=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, D))
    Wg, Wu, Wd = rng.standard_normal((F, D)), rng.standard_normal((F, D)), rng.standard_normal((D, F))
    lg = (rng.standard_normal((r, D)), rng.standard_normal((F, r)))
    lu = (rng.standard_normal((r, D)), rng.standard_normal((F, r)))
    ld = (rng.standard_normal((r, F)), rng.standard_normal((D, r)))
    ctx = rng.random(T) < 0.6
    dY = rng.standard_normal((T, D))
    return X, Wg, Wu, Wd, lg, lu, ld, ctx, dY


def test_ffn_keep_ratio_one_is_dense_swiglu_lora():
    X, Wg, Wu, Wd, lg, lu, ld, ctx, dY = _tiny_ffn()
    s = 1.3
    out = oracle.ffn_fwd(X, ctx, Wg, Wu, Wd, lg, lu, ld, s, np.arange(Wg.shape[0]))
    G = X @ Wg.T + s * (X @ lg[0].T) @ lg[1].T
    U = X @ Wu.T + s * (X @ lu[0].T) @ lu[1].T
    H = G / (1 + np.exp(-G)) * U
    Y = H @ Wd.T + s * (H @ ld[0].T) @ ld[1].T
    np.testing.assert_allclose(out["Y"], Y, rtol=1e-12, atol=1e-12)


def test_ffn_index_coupling():
    """One index set: gate/up keep idx output channels, down keeps idx input channels;
    on context rows the dropped intermediate channels carry only the LoRA terms, and
    down's frozen branch reads only H[:, idx] while its LoRA reads the full H."""
    X, Wg, Wu, Wd, lg, lu, ld, ctx, dY = _tiny_ffn(1)
    s = 0.9
    idx = np.array([0, 2, 3, 7])
    drop = oracle.complement(idx, Wg.shape[0])
    out = oracle.ffn_fwd(X, ctx, Wg, Wu, Wd, lg, lu, ld, s, idx)
    G, H, Y = out["G"], out["H"], out["Y"]
    np.testing.assert_allclose(G[ctx][:, drop], (s * (X @ lg[0].T) @ lg[1].T)[ctx][:, drop], rtol=1e-12)
    want = H[ctx][:, idx] @ Wd.T[idx, :] + s * (H[ctx] @ ld[0].T) @ ld[1].T
    np.testing.assert_allclose(Y[ctx], want, rtol=1e-12, atol=1e-12)


def test_ffn_backward_matches_finite_differences():
    X, Wg, Wu, Wd, lg, lu, ld, ctx, dY = _tiny_ffn(2, T=5, D=4, F=6, r=2)
    s = 0.8
    idx = np.array([1, 2, 5])

    def loss():
        return float(np.sum(dY * oracle.ffn_fwd(X, ctx, Wg, Wu, Wd, lg, lu, ld, s, idx)["Y"]))
    g = oracle.ffn_bwd(X, dY, ctx, Wg, Wu, Wd, lg, lu, ld, s, idx)
    np.testing.assert_allclose(g["dX"], _fd(loss, X), rtol=1e-6, atol=1e-7)
    for name, arrs in (("g", lg), ("u", lu), ("d", ld)):
        np.testing.assert_allclose(g["dA_" + name], _fd(loss, arrs[0]), rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(g["dB_" + name], _fd(loss, arrs[1]), rtol=1e-6, atol=1e-7)


def test_ffn_select_on_tiny_config_is_valid():
    cfg = inputs.TINY_FFN
    d = inputs.make_ffn_inputs(cfg, seed=0)
    s, idx = oracle.ffn_select(d["x"], d["ctx_mask"], (d["gate"].W_A, d["gate"].W_B),
                               (d["up"].W_A, d["up"].W_B), cfg.ratio)
    assert idx.shape[0] == oracle.keep_count(cfg.ratio, cfg.inter) == 344
    _brute_force_valid(s, 344, idx)


def test_context_first_permutation_equivalence():
    """Linear layers are row-independent: running on the context-first row order and
    un-permuting gives the sequence-order result."""
    X, Wg, Wu, Wd, lg, lu, ld, ctx, dY = _tiny_ffn(3)
    idx = np.array([0, 4, 5])
    perm = np.concatenate([np.nonzero(ctx)[0], np.nonzero(~ctx)[0]])
    a = oracle.ffn_fwd(X, ctx, Wg, Wu, Wd, lg, lu, ld, 1.0, idx)["Y"]
    b = oracle.ffn_fwd(X[perm], ctx[perm], Wg, Wu, Wd, lg, lu, ld, 1.0, idx)["Y"]
    inv = np.argsort(perm)
    np.testing.assert_allclose(b[inv], a, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- attention projections

def test_attn_select_mha_reduces_to_plain_qk():
    rng = np.random.default_rng(13)
    T, D, h, hd, k = 20, 16, 2, 4, 3
    X = rng.standard_normal((T, D))
    ctx = np.ones(T, dtype=bool)
    fs = [(rng.standard_normal((D, k)), rng.standard_normal((k, h * hd))) for _ in range(3)]
    out = oracle.attn_select(X, ctx, *fs, h, h, hd, 0.5)
    Q, K = X @ fs[0][0] @ fs[0][1], X @ fs[1][0] @ fs[1][1]
    s = np.linalg.norm(Q, axis=0) * np.linalg.norm(K, axis=0)
    np.testing.assert_allclose(out["s_qk"], s, rtol=1e-12)
    np.testing.assert_array_equal(out["idx_q"], out["idx_k"])
    np.testing.assert_array_equal(out["idx_o"], out["idx_v"])


def test_sum_of_squares_statistics_add_over_row_parts():
    """The per-channel statistics of data-parallel ranks: the sum over all rows is the sum of
    the sums over any split of the rows, and the root is the L2 criterion."""
    rng = np.random.default_rng(5)
    Y = rng.standard_normal((37, 11))
    np.testing.assert_allclose(oracle.sumsq(Y), oracle.score_l2(Y) ** 2, rtol=1e-13)
    for cut in (0, 1, 18, 37):
        np.testing.assert_allclose(oracle.sumsq(Y[:cut]) + oracle.sumsq(Y[cut:]), oracle.sumsq(Y), rtol=1e-13)
    # columns of constant value c over n rows: n c^2
    np.testing.assert_allclose(oracle.sumsq(np.full((6, 3), 2.5)), np.full(3, 6 * 2.5 ** 2), rtol=0)


# ----------------------------------------------------------------------- criterion variants

def test_wanda_scores_brute_force_tiny():
    """Wanda-style channel scores (R14) against explicit loops over rows, columns and tokens."""
    rng = np.random.default_rng(41)
    X = rng.standard_normal((5, 4))
    Ws = [rng.standard_normal((3, 4)), rng.standard_normal((3, 4))]
    want = np.zeros(3)
    for i in range(3):
        for W in Ws:
            for j in range(4):
                norm = 0.0
                for t in range(5):
                    norm += X[t, j] * X[t, j]
                want[i] += abs(W[i, j]) * norm ** 0.5
    np.testing.assert_allclose(oracle.wanda_scores(X, Ws), want, rtol=1e-13)


def test_wanda_scores_closed_forms():
    # constant columns c_j over T rows give norms sqrt(T) |c_j|; W = I picks them out
    T, c = 9, np.array([2.0, -3.0, 0.5])
    X = np.tile(c, (T, 1))
    np.testing.assert_allclose(oracle.wanda_scores(X, [np.eye(3)]), np.sqrt(T) * np.abs(c), rtol=1e-14)
    # homogeneous in |W| and in |X|
    rng = np.random.default_rng(42)
    X, W = rng.standard_normal((7, 6)), rng.standard_normal((4, 6))
    base = oracle.wanda_scores(X, [W])
    np.testing.assert_allclose(oracle.wanda_scores(-3.0 * X, [W]), 3.0 * base, rtol=1e-13)
    np.testing.assert_allclose(oracle.wanda_scores(X, [-0.5 * W]), 0.5 * base, rtol=1e-13)
    np.testing.assert_allclose(oracle.wanda_scores(X, [W, W]), 2.0 * base, rtol=1e-13)


def test_select_heads_special_cases():
    # head_dim 1: whole heads are single units, so this is the plain top-n
    s = np.array([0.3, 2.0, 1.1, 2.0, -1.0])
    np.testing.assert_array_equal(oracle.select_heads(s, 5, 1, 2), oracle.select_top(s, 2))
    # equal head sums: the lower heads
    np.testing.assert_array_equal(oracle.select_heads(np.ones(12), 3, 4, 2), np.arange(8))
    # a head with the largest single unit but the smaller sum loses to the head with the larger sum
    s = np.array([10.0, 0.0, 0.0, 0.0, 3.0, 3.0, 3.0, 3.0])
    np.testing.assert_array_equal(oracle.select_heads(s, 2, 4, 1), np.arange(4, 8))
    np.testing.assert_array_equal(oracle.select_top(s, 4), np.array([0, 4, 5, 6]))


# ----------------------------------------------------------------------- decoder layer (NEXT-1)

def test_rmsnorm_closed_forms():
    g = np.array([1.0, 2.0, -0.5, 3.0])
    # a constant row c: mean(x^2) = c^2, so y = c / sqrt(c^2 + eps) * gamma
    c, eps = 2.5, 1e-6
    np.testing.assert_allclose(oracle.rmsnorm(np.full((1, 4), c), g, eps)[0], c / np.sqrt(c * c + eps) * g,
                               rtol=1e-14)
    # eps = 0: invariant to scaling the row
    rng = np.random.default_rng(51)
    X = rng.standard_normal((3, 4))
    np.testing.assert_allclose(oracle.rmsnorm(7.0 * X, g, 0.0), oracle.rmsnorm(X, g, 0.0), rtol=1e-13)
    # rows of +-1: y = x * gamma
    X = np.array([[1.0, -1.0, 1.0, -1.0]])
    np.testing.assert_allclose(oracle.rmsnorm(X, g, 0.0), X * g, rtol=1e-15)


def test_rmsnorm_backward_matches_finite_differences():
    rng = np.random.default_rng(52)
    X, dY, g = rng.standard_normal((3, 6)), rng.standard_normal((3, 6)), rng.standard_normal(6)
    eps, h = 1e-5, 1e-6
    num = np.zeros_like(X)
    for i in range(X.shape[0]):
        for j in range(X.shape[1]):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, j] += h
            Xm[i, j] -= h
            num[i, j] = (np.sum(dY * oracle.rmsnorm(Xp, g, eps)) - np.sum(dY * oracle.rmsnorm(Xm, g, eps))) / (2 * h)
    np.testing.assert_allclose(oracle.rmsnorm_bwd(dY, X, g, eps), num, rtol=1e-7, atol=1e-8)


def test_attention_closed_forms():
    rng = np.random.default_rng(53)
    n_seq, S, hq, hkv, hd = 2, 5, 4, 2, 3
    T = n_seq * S
    V = rng.standard_normal((T, hkv * hd))
    # zero queries: causal uniform weights, O[i] = mean of V over positions 0..i of the sequence
    O, _ = oracle.attention(np.zeros((T, hq * hd)), rng.standard_normal((T, hkv * hd)), V, n_seq, hq, hkv, hd)
    for b in range(n_seq):
        for i in range(S):
            for h in range(hq):
                g = h // (hq // hkv)
                want = V[b * S:b * S + i + 1, g * hd:(g + 1) * hd].mean(axis=0)
                np.testing.assert_allclose(O[b * S + i, h * hd:(h + 1) * hd], want, rtol=1e-13)
    # the first token of every sequence attends only to itself
    Q, K = rng.standard_normal((T, hq * hd)), rng.standard_normal((T, hkv * hd))
    O, _ = oracle.attention(Q, K, V, n_seq, hq, hkv, hd)
    for b in range(n_seq):
        for h in range(hq):
            g = h // (hq // hkv)
            np.testing.assert_allclose(O[b * S, h * hd:(h + 1) * hd], V[b * S, g * hd:(g + 1) * hd], rtol=1e-14)


def test_attention_backward_matches_finite_differences():
    rng = np.random.default_rng(54)
    n_seq, S, hq, hkv, hd = 2, 3, 2, 1, 2
    T = n_seq * S
    Q, K, V = (rng.standard_normal((T, n * hd)) for n in (hq, hkv, hkv))
    dO = rng.standard_normal((T, hq * hd))
    _, P = oracle.attention(Q, K, V, n_seq, hq, hkv, hd)
    dQ, dK, dV = oracle.attention_bwd(dO, Q, K, V, P, n_seq, hq, hkv, hd)
    h = 1e-6

    def loss(Q, K, V):
        return np.sum(dO * oracle.attention(Q, K, V, n_seq, hq, hkv, hd)[0])

    for M, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        num = np.zeros_like(M)
        for i in range(M.shape[0]):
            for j in range(M.shape[1]):
                args_p = [Q.copy(), K.copy(), V.copy()]
                args_m = [Q.copy(), K.copy(), V.copy()]
                args_p[which][i, j] += h
                args_m[which][i, j] -= h
                num[i, j] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-8)


def test_decoder_layer_backward_matches_finite_differences():
    """dX and two LoRA gradients of the whole layer (fixed index sets, R9) against central
    differences of the layer's output."""
    rng = np.random.default_rng(55)
    n_seq, S, D, hq, hkv, hd, F, r = 2, 3, 8, 2, 1, 4, 12, 2
    T = n_seq * S
    Dq, Dkv = hq * hd, hkv * hd
    shapes = {"q": (Dq, D), "k": (Dkv, D), "v": (Dkv, D), "o": (D, Dq), "gate": (F, D), "up": (F, D), "down": (D, F)}
    w = {n: 0.3 * rng.standard_normal(s) for n, s in shapes.items()}
    lora = {n: (0.3 * rng.standard_normal((r, s[1])), 0.3 * rng.standard_normal((s[0], r))) for n, s in shapes.items()}
    gammas = (1.0 + 0.1 * rng.standard_normal(D), 1.0 + 0.1 * rng.standard_normal(D))
    ctx = np.tile(np.array([True, True, False]), n_seq)
    idx = {"q": np.array([0, 1, 4, 5]), "k": np.array([0, 1]), "v": np.array([1, 3]), "o": np.array([1, 3, 5, 7]),
           "ffn": np.array([0, 2, 3, 7, 8, 11])}
    X, dY = rng.standard_normal((T, D)), rng.standard_normal((T, D))
    res = oracle.decoder_layer(X, dY, ctx, n_seq, w, lora, gammas, 1e-5, 2.0, (hq, hkv, hd), 0.5, idx=dict(idx))

    def loss(X, lora):
        out = oracle.decoder_layer(X, np.zeros_like(dY), ctx, n_seq, w, lora, gammas, 1e-5, 2.0, (hq, hkv, hd), 0.5,
                                   idx=dict(idx))
        return np.sum(dY * out["Y"])

    h = 1e-6
    num = np.zeros_like(X)
    for i in range(T):
        for j in range(D):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, j] += h
            Xm[i, j] -= h
            num[i, j] = (loss(Xp, lora) - loss(Xm, lora)) / (2 * h)
    np.testing.assert_allclose(res["dX"], num, rtol=1e-5, atol=1e-7)
    for name, which in (("q", 0), ("down", 1)):
        M = lora[name][which]
        G = res[("dA_" if which == 0 else "dB_") + name]
        numg = np.zeros_like(M)
        for i in range(M.shape[0]):
            for j in range(M.shape[1]):
                lp = {k: (a.copy(), b.copy()) for k, (a, b) in lora.items()}
                lm = {k: (a.copy(), b.copy()) for k, (a, b) in lora.items()}
                lp[name][which][i, j] += h
                lm[name][which][i, j] -= h
                numg[i, j] = (loss(X, lp) - loss(X, lm)) / (2 * h)
        np.testing.assert_allclose(G, numg, rtol=1e-5, atol=1e-7)


def test_adamw_closed_forms():
    # first step, no decay: m_hat = g, v_hat = g^2, so p moves by -lr * g / (|g| + eps)
    p, g = np.array([1.0, -2.0, 0.5]), np.array([0.3, -4.0, 0.0])
    q, m, v = oracle.adamw(p, g, np.zeros(3), np.zeros(3), 1, 0.1, 0.9, 0.999, 1e-8, 0.0)
    np.testing.assert_allclose(q, p - 0.1 * g / (np.abs(g) + 1e-8), rtol=1e-12)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-15)
    # zero gradient, decay only
    q, _, _ = oracle.adamw(p, np.zeros(3), np.zeros(3), np.zeros(3), 3, 0.01, 0.9, 0.999, 1e-8, 0.1)
    np.testing.assert_allclose(q, p * (1 - 0.01 * 0.1), rtol=1e-15)


def test_model_step_one_layer_equals_layer_and_loss_gradient():
    """A one-layer stack: the loss gradient reaching the layer is the cross-entropy gradient through
    the final RMSNorm, checked by central differences of the loss in the layer's output."""
    rng = np.random.default_rng(56)
    n_seq, S, D, hq, hkv, hd, F, r, V = 1, 4, 8, 2, 1, 4, 12, 2, 11
    T = n_seq * S
    shapes = {"q": (hq * hd, D), "k": (hkv * hd, D), "v": (hkv * hd, D), "o": (D, hq * hd), "gate": (F, D),
              "up": (F, D), "down": (D, F)}
    w = {n: 0.3 * rng.standard_normal(s) for n, s in shapes.items()}
    lora = {n: (0.3 * rng.standard_normal((r, s[1])), 0.3 * rng.standard_normal((s[0], r))) for n, s in shapes.items()}
    gammas = (1.0 + 0.1 * rng.standard_normal(D), 1.0 + 0.1 * rng.standard_normal(D))
    ctx = np.array([True, True, False, False])
    idx = {"q": np.arange(8), "k": np.arange(4), "v": np.arange(4), "o": np.arange(8), "ffn": np.arange(12)}
    embed, lm_head, gf = rng.standard_normal((V, D)), rng.standard_normal((V, D)), 1.0 + 0.1 * rng.standard_normal(D)
    ids, tgt = rng.integers(0, V, T), rng.integers(0, V, 2)
    layers = [dict(w=w, lora=lora, gammas=gammas, idx=idx)]
    loss, grads = oracle.model_step(ids, tgt, ctx, n_seq, embed, lm_head, gf, layers, 1e-5, 2.0, (hq, hkv, hd))

    def loss_of(lo):
        L = [dict(w=w, lora=lo, gammas=gammas, idx=idx)]
        return oracle.model_step(ids, tgt, ctx, n_seq, embed, lm_head, gf, L, 1e-5, 2.0, (hq, hkv, hd))[0]

    h = 1e-6
    for name in ("q", "down"):
        M = lora[name][1]
        num = np.zeros_like(M)
        for i in range(M.shape[0]):
            for j in range(M.shape[1]):
                lp = {k: (a.copy(), b.copy()) for k, (a, b) in lora.items()}
                lm = {k: (a.copy(), b.copy()) for k, (a, b) in lora.items()}
                lp[name][1][i, j] += h
                lm[name][1][i, j] -= h
                num[i, j] = (loss_of(lp) - loss_of(lm)) / (2 * h)
        np.testing.assert_allclose(grads[0]["dB_" + name], num, rtol=1e-5, atol=1e-8)


def test_cosine_lr_closed_forms():
    # 100 steps, 4% warm-up: 4 warm-up steps reaching the peak at step 4; the cosine half-period
    # over steps 4..100 is at its midpoint (peak / 2) at step 52 and reaches 0 at step 100
    f = lambda t: oracle.cosine_lr(t, 100, 2e-4, 0.04)
    assert f(1) == pytest.approx(0.5e-4, rel=1e-15)
    assert f(4) == pytest.approx(2e-4, rel=1e-15)
    assert f(52) == pytest.approx(1e-4, rel=1e-12)
    assert f(100) == pytest.approx(0.0, abs=1e-20)
    # a third of the decay: (cos(pi / 3) + 1) / 2 = 3/4 of the peak
    assert f(4 + 32) == pytest.approx(0.75 * 2e-4, rel=1e-12)
    rates = [f(t) for t in range(4, 101)]
    assert all(a >= b for a, b in zip(rates, rates[1:]))
    # 20 steps: ceil(0.8) = 1 warm-up step, so the first step already runs at the peak
    assert oracle.cosine_lr(1, 20, 1.0, 0.04) == 1.0
    assert oracle.cosine_lr(20, 20, 1.0, 0.04) == pytest.approx(0.0, abs=1e-15)


def test_sigmoid_identities():
    # sigma(z) + sigma(-z) = 1, sigma(0) = 1/2, no overflow at large |z|, sigma(log 3) = 3/4
    z = np.array([-800.0, -30.0, -1.5, 0.0, 1.5, 30.0, 800.0, np.log(3.0)])
    s = oracle.sigmoid(z)
    assert np.all(np.isfinite(s))
    np.testing.assert_allclose(s + oracle.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    assert s[3] == 0.5 and s[0] == 0.0 and s[6] == 1.0
    assert s[7] == pytest.approx(0.75, rel=1e-15)


def test_sliced_weight_zeroes_the_dropped_channels():
    W = np.arange(12.0).reshape(3, 4)  # nn.Linear storage [d_out = 3, d_in = 4]; W_math = W.T [4, 3]
    out = oracle.sliced_weight(W, np.array([0, 2]), "out")
    np.testing.assert_array_equal(out, np.array([[0, 0, 8], [1, 0, 9], [2, 0, 10], [3, 0, 11]], dtype=float))
    inn = oracle.sliced_weight(W, np.array([1, 3]), "in")
    np.testing.assert_array_equal(inn, np.array([[0, 0, 0], [1, 5, 9], [0, 0, 0], [3, 7, 11]], dtype=float))


# ---------------------------------------------------------------------------
# Closed forms of the decoder layer and of the model step: forward values that follow from the
# layer's structure alone (pre-norm RMSNorm, residual connections from the layer input and from
# the attention sum, causal attention within each sequence, SwiGLU, loss on the output rows), so
# that a composition mistake mirrored in the backward still fails.
# ---------------------------------------------------------------------------

def _sign_rows(rng, T, D):
    """Rows of +-1 entries: mean square exactly 1, so RMSNorm with eps = 0 and unit gain is the
    identity on them."""
    return rng.choice([-1.0, 1.0], size=(T, D))


def _layer_weights(D, hq, hkv, hd, F, r, rng, zero=True):
    Dq, Dkv = hq * hd, hkv * hd
    shapes = {"q": (Dq, D), "k": (Dkv, D), "v": (Dkv, D), "o": (D, Dq), "gate": (F, D), "up": (F, D), "down": (D, F)}
    w = {n: np.zeros(s) for n, s in shapes.items()}
    # LoRA B = 0 (the adapter adds nothing), A random (its input path still runs)
    lora = {n: (rng.standard_normal((r, s[1])), np.zeros((s[0], r))) for n, s in shapes.items()}
    full = {"q": np.arange(Dq), "k": np.arange(Dkv), "v": np.arange(Dkv), "o": np.arange(Dq), "ffn": np.arange(F)}
    return w, lora, full


def test_decoder_layer_zero_projections_is_identity():
    """Every frozen weight zero and every LoRA B zero: each branch adds exactly zero, so the layer
    passes X through its two residual connections (Y = X) and the gradient through them
    (dX = dY), for any gains and any index sets."""
    rng = np.random.default_rng(61)
    n_seq, S, D, hq, hkv, hd, F, r = 2, 4, 8, 2, 1, 4, 12, 2
    T = n_seq * S
    w, lora, _ = _layer_weights(D, hq, hkv, hd, F, r, rng)
    gammas = (1.0 + 0.3 * rng.standard_normal(D), 1.0 + 0.3 * rng.standard_normal(D))
    ctx = np.tile(np.array([True, True, True, False]), n_seq)
    idx = {"q": np.array([1, 2, 5, 6]), "k": np.array([1, 2]), "v": np.array([0, 3]), "o": np.array([0, 3, 4, 7]),
           "ffn": np.array([0, 1, 5, 6, 9, 10])}
    X, dY = rng.standard_normal((T, D)), rng.standard_normal((T, D))
    res = oracle.decoder_layer(X, dY, ctx, n_seq, w, lora, gammas, 1e-5, 2.0, (hq, hkv, hd), 0.5, idx=dict(idx))
    np.testing.assert_array_equal(res["Y"], X)
    np.testing.assert_array_equal(res["dX"], dY)
    for n in ("q", "k", "v", "o", "gate", "up", "down"):
        np.testing.assert_array_equal(res["dA_" + n], 0.0)


def test_decoder_layer_attention_branch_closed_form():
    """Attention branch alone, MHA with D = heads x head_dim: W_q = W_k = 0 (uniform causal
    weights), W_v = W_o = I, the FFN zero, every LoRA B zero, all channels kept. On rows of +-1
    with eps = 0 and unit gains the pre-norm is the identity, so the layer is
    Y_t = X_t + mean_{s <= t, same sequence} X_s. Its backward: with J_t = I - x_t x_t^T / D the
    Jacobian of RMSNorm at such a row, dX_t = dY_t + J_t sum_{u >= t, same sequence} dY_u / (pos(u) + 1).
    A post-norm layer, a residual taken after the norm, a non-causal or cross-sequence mask, or a
    missing residual gives another Y."""
    rng = np.random.default_rng(62)
    n_seq, S, hq, hd, F, r = 2, 5, 2, 3, 4, 2
    D = hq * hd
    T = n_seq * S
    w, lora, full = _layer_weights(D, hq, hq, hd, F, r, rng)
    w["v"] = np.eye(D)
    w["o"] = np.eye(D)
    ones = (np.ones(D), np.ones(D))
    ctx = np.tile(np.array([True, True, True, False, False]), n_seq)
    X = _sign_rows(rng, T, D)
    dY = rng.standard_normal((T, D))
    res = oracle.decoder_layer(X, dY, ctx, n_seq, w, lora, ones, 0.0, 2.0, (hq, hq, hd), 1.0, idx=dict(full))
    Y = np.empty_like(X)
    dX = np.empty_like(X)
    for b in range(n_seq):
        for i in range(S):
            t = b * S + i
            Y[t] = X[t] + X[b * S:t + 1].sum(axis=0) / (i + 1)
            acc = sum(dY[b * S + j] / (j + 1) for j in range(i, S))
            J = np.eye(D) - np.outer(X[t], X[t]) / D
            dX[t] = dY[t] + J @ acc
    np.testing.assert_allclose(res["Y"], Y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(res["dX"], dX, rtol=1e-12, atol=1e-12)


def test_decoder_layer_ffn_branch_closed_form():
    """FFN branch alone: attention weights zero, W_up = I, W_gate = c I, W_down = I (F = D), LoRA
    B zero, all channels kept; rows of +-1, eps = 0, unit gains. Then Y = X + SiLU(c X) * X, and
    for x = +-1 that is x + c * sigmoid(c x) (SiLU(c) for x = 1, -SiLU(-c) = c sigmoid(-c) for
    x = -1)."""
    rng = np.random.default_rng(63)
    n_seq, S, D, hq, hkv, hd, r = 2, 3, 6, 2, 1, 3, 2
    T = n_seq * S
    c = 1.7
    w, lora, full = _layer_weights(D, hq, hkv, hd, D, r, rng)
    w["up"] = np.eye(D)
    w["gate"] = c * np.eye(D)
    w["down"] = np.eye(D)
    ones = (np.ones(D), np.ones(D))
    ctx = np.tile(np.array([True, True, False]), n_seq)
    X = _sign_rows(rng, T, D)
    res = oracle.decoder_layer(X, np.zeros((T, D)), ctx, n_seq, w, lora, ones, 0.0, 2.0, (hq, hkv, hd), 1.0,
                               idx=dict(full))
    want = X + c / (1.0 + np.exp(-c * X))
    np.testing.assert_allclose(res["Y"], want, rtol=1e-14, atol=1e-14)


def _identity_model(rng, n_layers, D, hq, hkv, hd, F, r):
    layers = []
    for _ in range(n_layers):
        w, lora, full = _layer_weights(D, hq, hkv, hd, F, r, rng)
        layers.append(dict(w=w, lora=lora, gammas=(1.0 + 0.2 * rng.standard_normal(D),) * 2, idx=full))
    return layers


def test_model_step_zero_head_loss_is_log_vocab():
    """A zero LM head gives all-zero logits: the mean cross-entropy over the output rows is ln V
    exactly, whatever the layers, ids and targets."""
    rng = np.random.default_rng(64)
    n_seq, S, D, hq, hkv, hd, F, r, V = 2, 4, 8, 2, 1, 4, 12, 2, 37
    T = n_seq * S
    layers = _identity_model(rng, 2, D, hq, hkv, hd, F, r)
    for L in layers:  # non-trivial layers: the head alone fixes the loss
        L["w"] = {n: 0.3 * rng.standard_normal(a.shape) for n, a in L["w"].items()}
    ctx = np.tile(np.array([True, True, True, False]), n_seq)
    embed = rng.standard_normal((V, D))
    ids, tgt = rng.integers(0, V, T), rng.integers(0, V, int((~ctx).sum()))
    loss, _ = oracle.model_step(ids, tgt, ctx, n_seq, embed, np.zeros((V, D)), np.ones(D), layers, 1e-5, 2.0,
                                (hq, hkv, hd))
    assert abs(loss - math.log(V)) < 1e-13


def test_model_step_signed_one_hot_head_closed_form():
    """Identity layers (zero weights, zero LoRA B), embedding rows of +-1, eps = 0 and unit final
    gain make the final hidden state H_t = E[id_t] exactly. With V = 2 D and LM-head rows e_j
    (v = j) and -e_j (v = D + j), every row's logits are D values +1 and D values -1, so
    logsumexp = ln D + ln(e + 1/e); the loss is the mean over the output rows (in their order) of
    that minus the target's logit +-H_t[j]."""
    rng = np.random.default_rng(65)
    n_seq, S, D, hq, hkv, hd, F, r = 2, 4, 6, 2, 1, 3, 8, 2
    V = 2 * D
    T = n_seq * S
    layers = _identity_model(rng, 2, D, hq, hkv, hd, F, r)
    ctx = np.tile(np.array([True, False, True, False]), n_seq)
    embed = _sign_rows(rng, V, D)
    head = np.concatenate([np.eye(D), -np.eye(D)])
    ids = rng.integers(0, V, T)
    out_rows = np.flatnonzero(~ctx)
    tgt = rng.integers(0, V, out_rows.size)
    loss, _ = oracle.model_step(ids, tgt, ctx, n_seq, embed, head, np.ones(D), layers, 0.0, 2.0, (hq, hkv, hd))
    lse = math.log(D) + math.log(math.e + 1.0 / math.e)
    want = np.mean([lse - (embed[ids[t], v] if v < D else -embed[ids[t], v - D]) for t, v in zip(out_rows, tgt)])
    assert abs(loss - want) < 1e-13
