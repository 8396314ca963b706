"""The debug build (libsparselora_debug.so, device-side bounds checks) on the GPU.

Valid inputs: a small FFN block step and attention-projection block step through the debug
library give the oracle's results and leave every error word at zero.

Out-of-range indices: a channel set (sigma) or gather list with one entry past the extent it
indexes is handed to the debug library ONLY; every device access that entry drives is one of the
checked ones (row and column gathers, output column and row maps, dB rows), so the failing check
skips the access and the call records its code instead of reading or writing outside the
caller's buffers. The release library is never given such an index.
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
BAD_GATHER_ROW, BAD_GATHER_COL, BAD_COL_MAP, BAD_ROW_MAP, BAD_DB_ROW = 0x101, 0x102, 0x103, 0x104, 0x105


@pytest.fixture
def debug_lib():
    with B.using_library(B.DEBUG_LIB_PATH) as L:
        assert L.sl_debug_bounds_enabled() == 1
        assert B.sl_read_debug_flag() == 0
        yield L


def cu(t, dtype=torch.bfloat16):
    return t.to(device=DEV, dtype=dtype).contiguous()


def test_debug_library_valid_ffn_and_attention_steps(debug_lib):
    T, C, D, F, r, k = 424, 300, 512, 1000, 32, 8
    p = ffn_problem(T, C, D, F, r, k, seed=21)
    blk = blocks.FFNBlock(p["gate"], p["up"], p["down"], p["lg"], p["lu"], p["ld"], 2.0, k, T, C, 0.5, DEV)
    blk.step(cu(p["x"]), cu(p["dy"]))
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0
    idx = blk.sigma.cpu().numpy()[: blk.n_keep].astype(np.int64)
    s_w, _ = oracle.ffn_select(p["x"], p["ctx"], (p["gate"].W_A, p["gate"].W_B), (p["up"].W_A, p["up"].W_B), 0.5)
    assert rel_fro(blk.scores, s_w) < FP32_TOL
    fwd = oracle.ffn_fwd(p["x"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"], 2.0, idx)
    bwd = oracle.ffn_bwd(p["x"], p["dy"], p["ctx"], p["gate"].W, p["up"].W, p["down"].W, p["lg"], p["lu"], p["ld"],
                         2.0, idx, fwd=fwd)
    assert rel_fro(unsigma(blk.h, blk.sigma, C), fwd["H"]) < BF16_TOL
    assert rel_fro(blk.y, fwd["Y"]) < BF16_TOL
    assert rel_fro(blk.dx, bwd["dX"]) < BF16_TOL
    for n in ("g", "u", "d"):
        assert rel_fro(getattr(blk, "dA_" + n), bwd["dA_" + n]) < BF16_TOL
        assert rel_fro(getattr(blk, "dB_" + n), bwd["dB_" + n]) < BF16_TOL
    hq, hkv, hd = 8, 2, 64
    a = attn_problem(T, C, D, hq, hkv, hd, r, k, seed=22)
    w, lo = a["w"], a["lora"]
    ab = blocks.AttnProjBlock(w["q"], w["k"], w["v"], w["o"], lo["q"], lo["k"], lo["v"], lo["o"], 2.0, k, hq, hkv, hd,
                              T, C, 0.5, DEV)
    ab.step(cu(a["x"]), cu(a["x_o"]), cu(a["dy"]), cu(a["dq"]), cu(a["dk"]), cu(a["dv"]))
    torch.cuda.synchronize()
    assert ab.read_device_flag() == 0
    u_v = ab.sig_v.cpu().numpy()[: ab.n_keep_u].astype(np.int64)
    idx_o = oracle.expand_units(u_v, hq, hkv, hd)
    want = oracle.sparse_linear_fwd(a["x_o"], w["o"].W, *lo["o"], 2.0, a["ctx"], idx_o, "in")
    assert rel_fro(ab.y, want) < BF16_TOL
    assert B.sl_read_debug_flag() == 0


def test_debug_gather_rows_batch_skips_an_out_of_range_row(debug_lib):
    """One perm entry equal to the source's row count: that destination row is left as it was,
    every other row is gathered, and the debug word holds the row-gather code."""
    n_src, n_cols, n = 64, 128, 16
    src = torch.randn(n_src, n_cols, device=DEV).to(torch.bfloat16)
    perm = torch.randperm(n_src, device=DEV)[:n].to(torch.int32)
    perm[5] = n_src
    dst = torch.full((n, n_cols), 7.0, device=DEV, dtype=torch.bfloat16)
    B.sl_gather_rows_batch([src], [perm], [dst])
    assert B.sl_read_debug_flag() == BAD_GATHER_ROW
    assert B.sl_read_debug_flag() == 0  # the read clears it
    ok = torch.arange(n, device=DEV) != 5
    assert torch.equal(dst[ok], src[perm[ok].long()])
    assert bool((dst[5] == 7.0).all())
    # sl_permute_rows: the same check against its row count
    out = torch.full((n_src, n_cols), 3.0, device=DEV, dtype=torch.bfloat16)
    pr = torch.arange(n_src, device=DEV, dtype=torch.int32).flip(0).contiguous()
    pr[0] = -1
    B.sl_permute_rows(src, pr, out)
    assert B.sl_read_debug_flag() == BAD_GATHER_ROW
    assert bool((out[0] == 3.0).all())
    assert torch.equal(out[1:], src[pr[1:].long()])


def _bad_sigma(n, n_keep, bad_pos, seed):
    rng = np.random.default_rng(seed)
    idx = np.sort(rng.choice(n, n_keep, replace=False))
    sig = np.concatenate([idx, oracle.complement(idx, n)]).astype(np.int32)
    sig[bad_pos] = n  # one past the last channel
    return torch.tensor(sig, device=DEV)


@pytest.mark.parametrize("bad_pos", [3, 900])
def test_debug_sparse_linear_with_an_out_of_range_channel(debug_lib, bad_pos):
    """sigma with one entry = d_out, among the kept channels (3) or the dropped ones (900), handed to
    the forward with the kept rows gathered inside the call and the natural output layout: the kept
    row gather, the sigma-ordered LoRA B gather and the output column scatter all read that entry and
    all check it; the workspace records a bad-index code and the step completes."""
    T, C, D, Do, r, nk = 424, 300, 512, 1000, 32, 437
    gen = inputs.generator(23)
    w = inputs.spectral_weight(Do, D, 0.5, 8, gen, "cpu", torch.float64, torch.bfloat16)
    A, Bm = inputs.lora_pair(Do, D, r, 0.02, gen)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    ws = B.Workspace()
    Wg, Ag, Bg, xg = cu(w.W), cu(A), cu(Bm), cu(x)
    lin = B.linear_desc(Wg, Ag, Bg, 2.0, B.SL_SLICE_OUT)
    sig = _bad_sigma(Do, nk, bad_pos, 24)
    ch = B.channels_desc(sig, nk)
    xa, xa_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa)
    y = torch.zeros(T, Do, device=DEV, dtype=torch.bfloat16)
    B.sl_sparse_linear_fwd(ws, [lin], [ch], B.SL_EPI_NONE, xg, C, xa_s, [y], out_layout=B.SL_LAYOUT_NATURAL)
    torch.cuda.synchronize()
    code = ws.read_device_flag()
    assert code in (BAD_GATHER_ROW, BAD_COL_MAP), hex(code)
    # output rows do not read sigma: they are the dense product
    want = oracle.sparse_linear_fwd(x[C:], w.W, A, Bm, 2.0, np.zeros(T - C, dtype=bool), np.arange(Do), "out")
    assert rel_fro(y[C:], want) < BF16_TOL


def test_debug_lora_backward_with_an_out_of_range_channel(debug_lib):
    """The LoRA backward with dy in the sigma layout of a set holding one entry = d_out: the LoRA B
    gather and the fused kernel's dB rows read that entry and check it."""
    T, C, D, Do, r, nk = 424, 300, 512, 1000, 32, 437
    gen = inputs.generator(25)
    A, Bm = inputs.lora_pair(Do, D, r, 0.02, gen)
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen)
    dy = torch.randn(T, Do, generator=gen).to(torch.bfloat16)
    ws = B.Workspace()
    lin = B.linear_desc(cu(torch.zeros(Do, D)), cu(A), cu(Bm), 2.0, B.SL_SLICE_OUT)
    sig = _bad_sigma(Do, nk, 10, 26)
    ch = B.channels_desc(sig, nk)
    xg = cu(x)
    xa, xa_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lin], xg, C, xa_s, xa=xa)
    dya, dya_s = torch.empty(T, r, device=DEV), torch.empty(T, r, device=DEV, dtype=torch.bfloat16)
    dA, dB = torch.empty(r, D, device=DEV), torch.empty(Do, r, device=DEV)
    B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lin], xg, C, xa_s, dy=[cu(dy)], out_layout=B.SL_LAYOUT_SIGMA,
                      out_ch=[ch], dya=[dya], dya_s=[dya_s], dA=[dA], dB=[dB])
    torch.cuda.synchronize()
    code = ws.read_device_flag()
    assert code in (BAD_GATHER_ROW, BAD_DB_ROW), hex(code)
