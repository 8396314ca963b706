"""CUDA path (through the C ABI) against the fp64 oracle on seeded inputs.

Sizes span several 128-row / 256-column tiles and end in ragged tails. Tolerances:
relative Frobenius error <= 1e-5 for fp32 quantities computed from exact inputs
(estimator scores), <= 2e-2 for values that pass through bf16 tensor-core GEMMs;
channel indices bit-exact when both sides select from the same fp32 scores.
"""
import numpy as np
import pytest
import torch

import oracle
from contextual_sparsity_lora_b200 import binding as B
from contextual_sparsity_lora_b200 import blocks, inputs
from gpu_helpers import BF16_TOL, FP32_TOL, attn_problem, ffn_problem, rel_fro, unsigma

pytestmark = pytest.mark.gpu
DEV = "cuda"


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


def sigma_from(idx, n):
    idx = np.asarray(idx, dtype=np.int64)
    return torch.tensor(np.concatenate([idx, oracle.complement(idx, n)]), dtype=torch.int32, device=DEV)


def rand_idx(n, n_keep, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, n_keep, replace=False))


# ------------------------------------------------------------------------------------------ LoRA

@pytest.mark.parametrize("T,n_ctx,D,rs", [(424, 300, 512, (32,)), (424, 300, 512, (32, 32, 32)),
                                           (130, 0, 264, (8, 16))])
def test_lora_fwd_xa(T, n_ctx, D, rs):
    gen = inputs.generator(1)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    As = [inputs.lora_pair(64, D, r, 0.02, gen) for r in rs]
    ws = B.Workspace()
    R = sum(rs)
    xa = torch.empty(T, R, device=DEV)
    xa_s = torch.empty(T, R, device=DEV, dtype=torch.bfloat16)
    w0 = cu(torch.zeros(64, D))
    dev_ab = [(cu(a), cu(b)) for a, b in As]   # device copies stay alive for the call
    lins = [B.linear_desc(w0, a, b, 2.0, B.SL_SLICE_OUT) for a, b in dev_ab]
    xg = cu(x)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, lins, xg, n_ctx, xa_s, xa=xa)
    want = oracle.f64(x) @ np.concatenate([oracle.f64(a) for a, b in As], 0).T
    assert rel_fro(xa, want) < FP32_TOL
    assert rel_fro(xa_s, 2.0 * want) < BF16_TOL


def test_lora_bwd_natural_and_sigma():
    T, C, D, Do, r = 424, 300, 512, 1000, 32
    gen = inputs.generator(2)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    A, Bm = inputs.lora_pair(Do, D, r, 0.02, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    s = 2.0
    xg, Ag, Bg, dyg = cu(x), cu(A), cu(Bm), cu(dy)
    ws = B.Workspace()
    lin = B.linear_desc(cu(torch.zeros(Do, D)), Ag, Bg, s, B.SL_SLICE_OUT)
    xa = torch.empty(T, r, device=DEV)
    xa_s = torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa)
    X, dY, A64, B64 = (oracle.f64(t) for t in (x, dy, A, Bm))
    # natural layout
    dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    dA, dB = torch.empty(r, D, device=DEV), torch.empty(Do, r, device=DEV)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin], xg, C, xa_s, dy=[dyg], dya=[dya], dya_s=[dya_s], dA=[dA], dB=[dB])
    assert rel_fro(dya, s * dY @ B64) < FP32_TOL * 10
    assert rel_fro(dB, s * dY.T @ (X @ A64.T)) < BF16_TOL
    assert rel_fro(dA, (s * dY @ B64).T @ X) < BF16_TOL
    # sigma layout on the output side: dy's context rows permuted by sigma
    idx = rand_idx(Do, 437, 3)
    sig = sigma_from(idx, Do)
    dy_sig = dy.clone()
    dy_sig[:C] = dy[:C][:, sig.cpu().long()]
    ch = B.channels_desc(sig, 437)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin], xg, C, xa_s, dy=[cu(dy_sig)], out_layout=B.SL_LAYOUT_SIGMA,
                      out_ch=[ch], dya=[dya], dya_s=[dya_s], dA=[dA], dB=[dB])
    assert rel_fro(dya, s * dY @ B64) < FP32_TOL * 10
    assert rel_fro(dB, s * dY.T @ (X @ A64.T)) < BF16_TOL
    assert rel_fro(dA, (s * dY @ B64).T @ X) < BF16_TOL


# ------------------------------------------------------------------------------------------ sparse linear

@pytest.mark.parametrize("layout", [B.SL_LAYOUT_NATURAL, B.SL_LAYOUT_SIGMA])
@pytest.mark.parametrize("zero_b", [False, True])
def test_sparse_linear_out_slice_fwd_bwd(layout, zero_b):
    T, C, D, Do, r, nk = 424, 300, 512, 1000, 32, 437
    gen = inputs.generator(4)
    w = inputs.spectral_weight(Do, D, 0.5, 8, gen, "cpu", torch.float64, torch.bfloat16)
    A, Bm = inputs.lora_pair(Do, D, r, 0.02, gen)
    if zero_b:
        Bm = torch.zeros_like(Bm)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    s, ctx = 2.0, np.arange(T) < C
    idx = rand_idx(Do, nk, 5)
    sig = sigma_from(idx, Do)
    ws = B.Workspace()
    Wg, Ag, Bg, xg = cu(w.W), cu(A), cu(Bm), cu(x)
    lin = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_OUT)
    ch = B.channels_desc(sig, nk)
    xa, xa_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa)
    y = torch.full((T, Do), float("nan"), device=DEV, dtype=torch.bfloat16)
    B.sl_sparse_linear_fwd(ws, [lin], [ch], B.SL_EPI_NONE, xg, C, xa_s, [y], out_layout=layout)
    want = oracle.sparse_linear_fwd(x, w.W, A, Bm, s, ctx, idx, "out")
    got = oracle.f64(y) if layout == B.SL_LAYOUT_NATURAL else unsigma(y, sig, C)
    assert np.isfinite(got).all()
    assert rel_fro(got, want) < BF16_TOL
    # backward: dy given in the same layout
    dy_in = dy.clone()
    if layout == B.SL_LAYOUT_SIGMA:
        dy_in[:C] = dy[:C][:, sig.cpu().long()]
    dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    dA, dB = torch.empty(r, D, device=DEV), torch.empty(Do, r, device=DEV)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin], xg, C, xa_s, dy=[cu(dy_in)], out_layout=layout, out_ch=[ch],
                      dya=[dya], dya_s=[dya_s], dA=[dA], dB=[dB])
    dx = torch.full((T, D), float("nan"), device=DEV, dtype=torch.bfloat16)
    B.sl_sparse_linear_bwd(ws, [lin], [ch], B.SL_EPI_NONE, [cu(dy_in)], C, [dya_s], dx=dx, in_layout=layout)
    dX, dA_w, dB_w = oracle.sparse_linear_bwd(x, dy, w.W, A, Bm, s, ctx, idx, "out")
    assert rel_fro(dx, dX) < BF16_TOL
    assert rel_fro(dA, dA_w) < BF16_TOL
    if not zero_b:
        assert rel_fro(dB, dB_w) < BF16_TOL


@pytest.mark.parametrize("layout", [B.SL_LAYOUT_NATURAL, B.SL_LAYOUT_SIGMA])
def test_sparse_linear_in_slice_fwd_bwd(layout):
    T, C, Di, Do, r, nk = 424, 300, 1000, 512, 32, 437
    gen = inputs.generator(6)
    w = inputs.spectral_weight(Do, Di, 0.5, 8, gen, "cpu", torch.float64, torch.bfloat16)
    A, Bm = inputs.lora_pair(Do, Di, r, 0.02, gen)
    x = inputs.activations_student_t(T, Di, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    s, ctx = 2.0, np.arange(T) < C
    idx = rand_idx(Di, nk, 7)
    sig = sigma_from(idx, Di)
    ws = B.Workspace()
    Wg, Ag, Bg = cu(w.W), cu(A), cu(Bm)
    Wt = torch.empty(Di, Do, device=DEV, dtype=torch.bfloat16)
    B.sl_prepare_weight(Wg, Wt)
    assert torch.equal(Wt, Wg.t())
    lin = B.linear_desc(Wg, Ag, Bg, s, B.SL_SLICE_IN, w_t=Wt)
    ch = B.channels_desc(sig, nk)
    x_in = x.clone()
    if layout == B.SL_LAYOUT_SIGMA:
        x_in[:C] = x[:C][:, sig.cpu().long()]
    xg = cu(x_in)
    xa, xa_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa, in_layout=layout, in_ch=ch)
    assert rel_fro(xa, oracle.f64(x) @ oracle.f64(A).T) < FP32_TOL
    y = torch.full((T, Do), float("nan"), device=DEV, dtype=torch.bfloat16)
    B.sl_sparse_linear_fwd(ws, [lin], [ch], B.SL_EPI_NONE, xg, C, xa_s, [y], in_layout=layout)
    assert rel_fro(y, oracle.sparse_linear_fwd(x, w.W, A, Bm, s, ctx, idx, "in")) < BF16_TOL
    dyg = cu(dy)
    dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    dA, dB = torch.empty(r, Di, device=DEV), torch.empty(Do, r, device=DEV)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin], xg, C, xa_s, in_layout=layout, in_ch=ch, dy=[dyg], dya=[dya],
                      dya_s=[dya_s], dA=[dA], dB=[dB])
    dx = torch.full((T, Di), float("nan"), device=DEV, dtype=torch.bfloat16)
    B.sl_sparse_linear_bwd(ws, [lin], [ch], B.SL_EPI_NONE, [dyg], C, [dya_s], dx=dx, out_layout=layout)
    dX, dA_w, dB_w = oracle.sparse_linear_bwd(x, dy, w.W, A, Bm, s, ctx, idx, "in")
    got = oracle.f64(dx) if layout == B.SL_LAYOUT_NATURAL else unsigma(dx, sig, C)
    assert rel_fro(got, dX) < BF16_TOL
    assert rel_fro(dA, dA_w) < BF16_TOL
    assert rel_fro(dB, dB_w) < BF16_TOL


# ------------------------------------------------------------------------------------------ estimator / select

def test_estimator_swiglu_scores_and_select():
    T, C, D, F, k = 424, 300, 512, 1000, 8
    p = ffn_problem(T, C, D, F, 32, k, seed=8)
    ws = B.Workspace()
    xg = cu(p["x"])
    scores = torch.empty(F, device=DEV)
    B.sl_svd_estimate(ws, B.SL_CRIT_SWIGLU_L2, xg[:C], C, [cu(p["gate"].W_A), cu(p["up"].W_A)],
                      [cu(p["gate"].W_B), cu(p["up"].W_B)], k, scores)
    s_w, idx_w = oracle.ffn_select(p["x"], p["ctx"], (p["gate"].W_A, p["gate"].W_B), (p["up"].W_A, p["up"].W_B), 0.5)
    assert rel_fro(scores, s_w) < FP32_TOL
    nk = oracle.keep_count(0.5, F)
    sig = torch.empty(F, dtype=torch.int32, device=DEV)
    B.sl_select_channels(scores, nk, sig)
    got = sig.cpu().numpy()
    sc = scores.cpu().numpy().astype(np.float64)
    want = oracle.select_top(sc, nk)
    np.testing.assert_array_equal(got[:nk], want)
    np.testing.assert_array_equal(got[nk:], oracle.complement(want, F))


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4)])
def test_estimator_qk_and_v_scores(hq, hkv):
    T, C, D, hd, k = 424, 300, 512, 64, 8
    p = attn_problem(T, C, D, hq, hkv, hd, 32, k, seed=9)
    ws = B.Workspace()
    xg = cu(p["x"])
    nu = hkv * hd
    s_qk, s_v = torch.empty(nu, device=DEV), torch.empty(nu, device=DEV)
    w = p["w"]
    B.sl_svd_estimate(ws, B.SL_CRIT_QK, xg[:C], C, [cu(w[n].W_A) for n in "qkv"], [cu(w[n].W_B) for n in "qkv"], k,
                      s_qk, scores_v=s_v, n_q_heads=hq, n_kv_heads=hkv, head_dim=hd)
    want = oracle.attn_select(p["x"], p["ctx"], (w["q"].W_A, w["q"].W_B), (w["k"].W_A, w["k"].W_B),
                              (w["v"].W_A, w["v"].W_B), hq, hkv, hd, 0.5)
    assert rel_fro(s_qk, want["s_qk"]) < FP32_TOL
    assert rel_fro(s_v, want["s_v"]) < FP32_TOL
    nk = oracle.keep_count(0.5, nu)
    sk, sq = torch.empty(nu, dtype=torch.int32, device=DEV), torch.empty(hq * hd, dtype=torch.int32, device=DEV)
    B.sl_select_channels(s_qk, nk, sk, hq // hkv, hd, sq)
    units = oracle.select_top(s_qk.cpu().numpy().astype(np.float64), nk)
    np.testing.assert_array_equal(sk.cpu().numpy()[:nk], units)
    qi = oracle.expand_units(units, hq, hkv, hd)
    np.testing.assert_array_equal(sq.cpu().numpy()[: len(qi)], qi)
    np.testing.assert_array_equal(sq.cpu().numpy()[len(qi):], oracle.complement(qi, hq * hd))


def test_estimator_l2_fp32_inputs():
    """The tiny fp32 configuration's estimator path (fp32 x and factors)."""
    T, C, D, Do, k = 128, 96, 256, 688, 8
    gen = inputs.generator(10)
    w = inputs.spectral_weight(Do, D, 0.7, k, gen, "cpu", torch.float64, torch.float32)
    x = inputs.activations_gaussian_outliers(T, D, 4, 20.0, gen)
    ws = B.Workspace()
    s = torch.empty(Do, device=DEV)
    B.sl_svd_estimate(ws, B.SL_CRIT_L2, cu(x, torch.float32)[:C], C, [cu(w.W_A, torch.float32)],
                      [cu(w.W_B, torch.float32)], k, s)
    want = oracle.score_l2(oracle.estimate(oracle.f64(x)[:C], w.W_A, w.W_B))
    assert rel_fro(s, want) < FP32_TOL


@pytest.mark.parametrize("n,n_keep", [(1, 1), (7, 3), (1000, 1), (1000, 1000), (1025, 513), (4096, 4095),
                                        (14336, 7168), (16384, 5000), (16385, 8000), (40960, 12345)])
def test_select_edge_cases_bit_exact(n, n_keep):
    rng = np.random.default_rng(n + n_keep)
    s = rng.integers(0, 50, n).astype(np.float32)          # heavy ties
    s[rng.random(n) < 0.05] = np.nan
    s[rng.random(n) < 0.02] = -np.inf
    s[rng.random(n) < 0.02] = -0.0
    s[rng.random(n) < 0.02] = 0.0
    sc = torch.tensor(s, device=DEV)
    sig = torch.empty(n, dtype=torch.int32, device=DEV)
    B.sl_select_channels(sc, n_keep, sig)
    want = oracle.select_top(s.astype(np.float64), n_keep)
    got = sig.cpu().numpy()
    np.testing.assert_array_equal(got[:n_keep], want)
    np.testing.assert_array_equal(got[n_keep:], oracle.complement(want, n))


@pytest.mark.parametrize("n,n_keep", [(1024, 512), (4096, 1229), (14336, 4301), (14336, 10036), (20000, 7)])
def test_select_continuous_scores_bit_exact(n, n_keep):
    """Distinct scores spread over a narrow range (criterion-like): the threshold search
    mostly ends on a threshold with exactly n_keep scores at or above it."""
    rng = np.random.default_rng(7 * n + n_keep)
    s = (1.0 + rng.standard_normal(n) ** 2).astype(np.float32)
    sc = torch.tensor(s, device=DEV)
    sig = torch.empty(n, dtype=torch.int32, device=DEV)
    B.sl_select_channels(sc, n_keep, sig)
    want = oracle.select_top(s.astype(np.float64), n_keep)
    got = sig.cpu().numpy()
    np.testing.assert_array_equal(got[:n_keep], want)
    np.testing.assert_array_equal(got[n_keep:], oracle.complement(want, n))


def test_select_all_equal_scores_at_the_size_limit():
    """Every score equal at n = 40960: the threshold is that score and the tied count (40960)
    exceeds 2^15, which a signed 16-bit half of a packed count would overflow; the lowest
    n_keep indices are kept."""
    n, n_keep = 40960, 20000
    sc = torch.full((n,), 1.5, device=DEV)
    sig = torch.empty(n, dtype=torch.int32, device=DEV)
    B.sl_select_channels(sc, n_keep, sig)
    np.testing.assert_array_equal(sig.cpu().numpy(), np.arange(n))
    s = np.full(n, 2.0, np.float32)
    s[:5] = 3.0  # five above the tie, then 39955 tied
    sig2 = torch.empty(n, dtype=torch.int32, device=DEV)
    B.sl_select_channels(torch.tensor(s, device=DEV), 35000, sig2)
    want = oracle.select_top(s.astype(np.float64), 35000)
    np.testing.assert_array_equal(sig2.cpu().numpy()[:35000], want)
    np.testing.assert_array_equal(sig2.cpu().numpy()[35000:], oracle.complement(want, n))


@pytest.mark.parametrize("hkv,hd,hpg,keep", [(8, 128, 4, 0.5), (8, 128, 4, 0.05), (2, 64, 8, 0.7), (40, 128, 1, 0.4),
                                              (3, 96, 3, 0.33), (5, 8, 2, 1.0)])
def test_select_query_side_set_bit_exact(hkv, hd, hpg, keep):
    """The query-side set of a KV-unit selection (GQA expansion) against the oracle's expansion:
    query channel (h, d) kept iff unit (h / hpg, d) is; kept then dropped, each ascending."""
    n = hkv * hd
    n_keep = max(1, int(round(keep * n)))
    rng = np.random.default_rng(n + hpg)
    s = (1.0 + rng.standard_normal(n) ** 2).astype(np.float32)
    sig = torch.empty(n, dtype=torch.int32, device=DEV)
    wide = torch.empty(n * hpg, dtype=torch.int32, device=DEV)
    B.sl_select_channels(torch.tensor(s, device=DEV), n_keep, sig, hpg, hd, wide)
    units = oracle.select_top(s.astype(np.float64), n_keep)
    np.testing.assert_array_equal(sig.cpu().numpy()[:n_keep], units)
    kept_q = oracle.expand_units(units, hkv * hpg, hkv, hd)
    got = wide.cpu().numpy()
    np.testing.assert_array_equal(got[: len(kept_q)], kept_q)
    np.testing.assert_array_equal(got[len(kept_q):], oracle.complement(kept_q, n * hpg))


def test_select_and_estimate_are_deterministic():
    T, C, D, F, k = 424, 300, 512, 1000, 8
    p = ffn_problem(T, C, D, F, 32, k, seed=11)
    ws = B.Workspace()
    xg = cu(p["x"])
    outs = []
    for _ in range(2):
        sc = torch.empty(F, device=DEV)
        B.sl_svd_estimate(ws, B.SL_CRIT_SWIGLU_L2, xg[:C], C, [cu(p["gate"].W_A), cu(p["up"].W_A)],
                          [cu(p["gate"].W_B), cu(p["up"].W_B)], k, sc)
        sig = torch.empty(F, dtype=torch.int32, device=DEV)
        B.sl_select_channels(sc, 500, sig)
        outs.append((sc.cpu(), sig.cpu()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_gather_rows_batch_is_exact():
    """Several row gathers in one launch: ragged row counts, a width that is not a multiple of
    8 (scalar copies), a strided destination and an empty job, against NumPy indexing."""
    from contextual_sparsity_lora_b200 import binding as B
    rng = np.random.default_rng(81)
    shapes = [(300, 64, 120), (77, 203, 77), (5, 13, 0), (1000, 40, 999)]  # (src rows, cols, gathered rows)
    srcs, perms, dsts, want = [], [], [], []
    for rows, cols, n in shapes:
        src = torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)).to(torch.bfloat16)
        p = rng.permutation(rows)[:n].astype(np.int32)
        wide = torch.zeros(max(n, 1), cols + 24, dtype=torch.bfloat16, device=DEV)
        srcs.append(src.to(DEV))
        perms.append(torch.from_numpy(p).to(DEV))
        dsts.append(wide[:n, :cols] if n else wide[:0, :cols])
        want.append(src.view(torch.int16).numpy()[p])
    B.sl_gather_rows_batch(srcs, perms, dsts)
    torch.cuda.synchronize()
    for d, w in zip(dsts, want):
        np.testing.assert_array_equal(d.cpu().view(torch.int16).numpy(), w)
    with pytest.raises(RuntimeError):
        B.sl_gather_rows_batch(srcs * 3, perms * 3, dsts * 3)  # more than 8 jobs


# ------------------------------------------------------------- SiLU in the far negative tail

@pytest.mark.parametrize("tile_rows", [256, 512])
def test_swiglu_epilogues_elementwise_on_negative_gates(tile_rows):
    """The SwiGLU epilogues evaluate the logistic function on every element. Gate pre-activations
    spread over [-24, 3] (most of them strongly negative, where SiLU(g) is tiny) are checked
    element by element at relative error 2e-2: h = SiLU(g) u (formed from the fp32 accumulators)
    against the oracle's fp64 H, and the backward's dg = dh u SiLU'(g), du = dh SiLU(g) against
    the oracle's formulas applied to the g, u the forward stored (bf16) and to the oracle's dh.
    A logistic function with a fixed absolute error (such as one built on 1 + tanh(g/2)) fails
    this test below g = -8."""
    T, C, D, F, r, k = 256, 192, 256, 512, 16, 8
    gen = inputs.generator(71)
    absn = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64).abs()
    x = absn(T, D).to(torch.bfloat16)                       # non-negative inputs: no cancellation in g
    a = torch.linspace(-30.0, 4.0, F, dtype=torch.float64)[torch.randperm(F, generator=gen)]
    Wg = (a[:, None] * absn(F, D) * 1.25 / D).to(torch.bfloat16)
    # up rows of one sign each: u has no cancellation either, so its fp32 accumulation error stays
    # at a few ulp of u and the relative error of h = SiLU(g) u isolates the logistic function
    sgn = torch.where(torch.rand(F, generator=gen, dtype=torch.float64) < 0.5, -1.0, 1.0)
    Wu = (sgn[:, None] * absn(F, D) * 2.0 / D).to(torch.bfloat16)
    Wd = (torch.randn(D, F, generator=gen, dtype=torch.float64) / F ** 0.5).to(torch.bfloat16)

    def sw(W):
        WA = torch.randn(W.shape[1], k, generator=gen, dtype=torch.float64) / 16
        WB = torch.randn(k, W.shape[0], generator=gen, dtype=torch.float64) / 16
        return inputs.SpectralWeight(W=W, W_A=WA.to(torch.bfloat16), W_B=WB.to(torch.bfloat16), s=torch.ones(k))

    zl = lambda do, di: (inputs.lora_pair(do, di, r, 0.02, gen)[0], torch.zeros(do, r, dtype=torch.bfloat16))
    lg, lu, ld = zl(F, D), zl(F, D), zl(D, F)
    dy = torch.randn(T, D, generator=gen).to(torch.bfloat16)
    from contextual_sparsity_lora_b200 import blocks
    with B.pair_tile_rows(tile_rows):
        blk = blocks.FFNBlock(sw(Wg), sw(Wu), sw(Wd), lg, lu, ld, 2.0, k, T, C, 0.5, DEV)
        blk.step(cu(x), cu(dy))
        torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    ctx = np.arange(T) < C
    fwd = oracle.ffn_fwd(x, ctx, Wg, Wu, Wd, lg, lu, ld, 2.0, idx)
    G = fwd["G"]
    live = G != 0.0   # dropped context channels are exactly 0 (LoRA B = 0)
    assert (G[live] < -8).mean() > 0.5, "most gates in the far negative tail"
    h = unsigma(blk.h, blk.sigma, C)
    rel = np.abs(h[live] - fwd["H"][live]) / np.abs(fwd["H"][live])
    assert rel.max() < 2e-2, f"h: worst relative error {rel.max():.3g}"
    # backward epilogue: the oracle's SwiGLU backward on the stored bf16 g and u, with the oracle's
    # dh = dY W_down (sliced on the context rows; LoRA B = 0 adds nothing)
    g16, u16 = unsigma(blk.g, blk.sigma, C), unsigma(blk.u, blk.sigma, C)
    dH = oracle.sparse_linear_bwd(fwd["H"], dy, Wd, ld[0], ld[1], 2.0, ctx, idx, "in")[0]
    rms = np.sqrt(np.mean(dH * dH))
    for got, fac, name in ((unsigma(blk.dg, blk.sigma, C), u16 * oracle.silu_grad(g16), "dg"),
                           (unsigma(blk.du, blk.sigma, C), oracle.silu(g16), "du")):
        want = dH * fac
        # 2e-2 relative, plus a floor for the fp32 accumulation error of dh where dh itself is ~0
        bad = live & (np.abs(got - want) > 2e-2 * np.abs(want) + 1e-4 * np.abs(fac) * rms)
        assert not bad.any(), f"{name}: {int(bad.sum())} elements outside tolerance"


# ------------------------------------------------- stage 1 inside the LoRA forward, criteria from Z

@pytest.mark.parametrize("T,C,D,crit,k,r", [(424, 300, 512, "qk", 8, 32), (424, 300, 512, "swiglu", 8, 32),
                                            (300, 200, 64, "swiglu", 4, 16), (200, 130, 256, "qk", 16, 8),
                                            (256, 0, 256, "swiglu", 8, 16)])
def test_lora_fwd_estimate_and_scores_from_z(T, C, D, crit, k, r):
    """sl_lora_fwd_estimate: x A^T of the adapters and Z = X_ctx W_A from one skinny product (split-K
    and, at d_in = 64, the unsplit epilogue); sl_svd_scores_from_z: the criteria from that Z,
    against the oracle's estimator on the same context rows (QK with GQA, SwiGLU)."""
    gen = inputs.generator(81 + k)
    hq, hkv, hd = 4, 2, 32
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    if crit == "qk":
        outs = (hq * hd, hkv * hd, hkv * hd)
    else:
        outs = (384, 384)
    fac = [inputs.spectral_weight(n, D, 0.5, k, gen, "cpu", torch.float64, torch.bfloat16) for n in outs]
    ads = [inputs.lora_pair(n, D, r, 0.02, gen) for n in outs]
    mk = len(outs) * k
    xg = cu(x)
    dev_ab = [(cu(a), cu(b)) for a, b in ads]
    lins = [B.linear_desc(cu(torch.zeros(n, D)), a, b, 2.0, B.SL_SLICE_OUT) for (a, b), n in zip(dev_ab, outs)]
    WA = [cu(f.W_A) for f in fac]
    WB = [cu(f.W_B) for f in fac]
    WAt = torch.empty(mk, D, device=DEV, dtype=torch.bfloat16)
    for j, w in enumerate(WA):
        B.sl_prepare_weight(w, WAt[j * k:(j + 1) * k])
    R = r * len(outs)
    xa = torch.full((T, R), float("nan"), device=DEV)
    xa_s = torch.full((T, R), float("nan"), device=DEV, dtype=torch.bfloat16)
    z = torch.full((max(C, 1), mk), float("nan"), device=DEV)
    ws = B.Workspace()
    B.sl_lora_fwd_estimate(ws, lins, xg, C, xa_s, xa, len(outs), k, WAt, z)
    torch.cuda.synchronize()
    X = oracle.f64(x)
    want_xa = X @ np.concatenate([oracle.f64(a) for a, _ in ads], 0).T
    assert rel_fro(xa, want_xa) < FP32_TOL
    assert rel_fro(xa_s, 2.0 * want_xa) < BF16_TOL
    if C == 0:
        assert torch.isnan(z).all()  # no context rows: Z untouched
        return
    want_z = X[:C] @ np.concatenate([oracle.f64(f.W_A) for f in fac], 1)
    assert rel_fro(z, want_z) < FP32_TOL
    ctx = np.arange(T) < C
    if crit == "qk":
        s_qk = torch.empty(hkv * hd, device=DEV)
        s_v = torch.empty(hkv * hd, device=DEV)
        B.sl_svd_scores_from_z(ws, B.SL_CRIT_QK, WB, k, z, C, s_qk, scores_v=s_v, n_q_heads=hq, n_kv_heads=hkv,
                               head_dim=hd)
        sel = oracle.attn_select(x, ctx, (fac[0].W_A, fac[0].W_B), (fac[1].W_A, fac[1].W_B), (fac[2].W_A, fac[2].W_B),
                                 hq, hkv, hd, 0.5)
        assert rel_fro(s_qk, sel["s_qk"]) < FP32_TOL
        assert rel_fro(s_v, sel["s_v"]) < FP32_TOL
    else:
        sc = torch.empty(outs[0], device=DEV)
        B.sl_svd_scores_from_z(ws, B.SL_CRIT_SWIGLU_L2, WB, k, z, C, sc)
        s_w, _ = oracle.ffn_select(x, ctx, (fac[0].W_A, fac[0].W_B), (fac[1].W_A, fac[1].W_B), 0.5)
        assert rel_fro(sc, s_w) < FP32_TOL
    assert ws.read_device_flag() == 0


@pytest.mark.parametrize("to_sigma", [True, False])
@pytest.mark.parametrize("n_cols", [8, 1024, 4096, 5120])
def test_permute_rows_sigma_is_exact(to_sigma, n_cols):
    """Row permutation with the context rows' channel order converted to or from the sigma
    layout, against NumPy indexing (bit-exact: it only moves bf16 values)."""
    n_rows, n_ctx = 300, 217
    rng = np.random.default_rng(n_cols + int(to_sigma))
    src = torch.randn(n_rows + 5, n_cols, device=DEV).to(torch.bfloat16)
    perm = rng.permutation(n_rows).astype(np.int32)
    sig = rng.permutation(n_cols).astype(np.int32)
    dst = torch.full((n_rows, n_cols), 7.0, device=DEV, dtype=torch.bfloat16)
    B.sl_permute_rows_sigma(src, torch.tensor(perm, device=DEV), dst, torch.tensor(sig, device=DEV), n_ctx, to_sigma)
    s = src.float().cpu().numpy()
    want = s[perm].copy()
    for i in range(n_rows):
        if to_sigma and i < n_ctx:
            want[i] = s[perm[i]][sig]
        elif not to_sigma and perm[i] < n_ctx:
            want[i, sig] = s[perm[i]]
    np.testing.assert_array_equal(dst.float().cpu().numpy(), want)


def test_attention_block_sigma_layout_matches_natural():
    """The attention block with its interfaces in the sigma layout against the natural layout on
    the same inputs: q, k, v and dx_o equal after the layout conversion (the same GEMM tiles,
    bulk instead of scattered stores); y, dx and the gradients within fp32 summation-order
    rounding (x_o A^T over permuted channels, the fused LoRA backward's unordered sums)."""
    T, C, D, hq, hkv, hd, r, k = 424, 300, 512, 8, 2, 64, 32, 8
    a = attn_problem(T, C, D, hq, hkv, hd, r, k, seed=47)
    w, lo = a["w"], a["lora"]
    blks = {}
    for lay in ("natural", "sigma"):
        blks[lay] = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], 2.0, k, hq,
                                         hkv, hd, T, C, 0.5, DEV, io_layout=lay)
    nb, sb = blks["natural"], blks["sigma"]
    xg = cu(a["x"])
    nb.forward_qkv(xg)
    sb.forward_qkv(xg)
    torch.cuda.synchronize()
    for name in ("sig_q", "sig_k", "sig_v", "sig_o"):
        assert torch.equal(getattr(nb, name), getattr(sb, name)), name
    for t_n, t_s, name in ((nb.q, sb.q, "q"), (nb.kk, sb.kk, "k"), (nb.vv, sb.vv, "v")):
        np.testing.assert_array_equal(oracle.f64(t_n), unsigma(t_s, sb.sigma_of(name), C))

    def to_sig(t, name):  # natural -> sigma layout on the context rows
        out = t.clone()
        sig = sb.sigma_of(name).long()
        out[:C] = t[:C][:, sig]
        return out
    x_o = cu(a["x_o"])
    nb.forward_o(x_o)
    sb.forward_o(to_sig(x_o, "o"))
    dy = cu(a["dy"])
    nb.backward_o(dy)
    sb.backward_o(dy)
    dq, dk, dv = cu(a["dq"]), cu(a["dk"]), cu(a["dv"])
    nb.backward_qkv(dq, dk, dv)
    sb.backward_qkv(to_sig(dq, "q"), to_sig(dk, "k"), to_sig(dv, "v"))
    torch.cuda.synchronize()
    assert nb.read_device_flag() == 0 and sb.read_device_flag() == 0
    # x_o A^T sums the context rows' channels in another order in the sigma layout (permuted A)
    assert rel_fro(sb.y, nb.y) < 1e-3
    np.testing.assert_array_equal(oracle.f64(nb.dx_o), unsigma(sb.dx_o, sb.sigma_of("o"), C))
    assert rel_fro(sb.dx, nb.dx) < 1e-3
    assert rel_fro(sb.grads.flat, nb.grads.flat) < 1e-3
