"""The C ABI without a GPU: the in-tree library loads, exports every function the header
declares, and rejects invalid arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from contextual_sparsity_lora_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparselora.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SL_API\s+[\w\s\*]+?\b(sl_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from contextual_sparsity_lora_b200 import build
        build.build()
    return B.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTED)


def test_status_strings_and_version(lib):
    assert B.status_string(B.SL_OK) == "ok"
    assert "workspace" in B.status_string(B.SL_ERR_WORKSPACE)
    assert B.sl_version() >= 1


@pytest.mark.parametrize("ratio,n,want", [(0.7, 14336, 10036), (0.3, 14336, 4301), (0.5, 1024, 512),
                                          (0.4, 13824, 5530), (1.0, 7, 7), (1e-6, 10, 1), (0.5, 0, 0)])
def test_keep_count_host(lib, ratio, n, want):
    assert B.sl_keep_count(ratio, n) == want


def _ws(ptr=None, nbytes=0):
    return B.SlWorkspaceC(ptr, nbytes, 0)


def test_estimate_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    fake = 0x10000  # never dereferenced: validation fails first
    wa = (P * 2)(fake, fake)
    wb = (P * 2)(fake, fake)
    dout = (ctypes.c_int64 * 2)(64, 64)
    ws = _ws()
    f = lib.sl_svd_estimate
    # null x
    assert f(B.SL_CRIT_L2, B.SL_DT_BF16, None, 8, 64, 64, 1, wa, wb, dout, 8, 0, 0, 0, P(fake), None,
             ctypes.byref(ws), None) == B.SL_ERR_INVALID_ARG
    # misaligned leading dimension
    assert f(B.SL_CRIT_L2, B.SL_DT_BF16, P(fake), 8, 64, 66, 1, wa, wb, dout, 8, 0, 0, 0, P(fake), None,
             ctypes.byref(ws), None) == B.SL_ERR_ALIGNMENT
    # rank too large
    assert f(B.SL_CRIT_L2, B.SL_DT_BF16, P(fake), 8, 64, 64, 1, wa, wb, dout, 32, 0, 0, 0, P(fake), None,
             ctypes.byref(ws), None) == B.SL_ERR_SHAPE
    # QK with inconsistent heads
    assert f(B.SL_CRIT_QK, B.SL_DT_BF16, P(fake), 8, 64, 64, 2, wa, wb, dout, 8, 3, 2, 32, P(fake), None,
             ctypes.byref(ws), None) == B.SL_ERR_SHAPE
    # missing workspace: reports the size it needs
    assert f(B.SL_CRIT_SWIGLU_L2, B.SL_DT_BF16, P(fake), 8, 64, 64, 2, wa, wb, dout, 8, 0, 0, 0, P(fake), None,
             ctypes.byref(ws), None) == B.SL_ERR_WORKSPACE
    assert ws.needed > 256


def test_select_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    f = lib.sl_select_channels
    assert f(None, 10, 5, P(0x10000), 0, 0, None, None) == B.SL_ERR_INVALID_ARG
    assert f(P(0x10000), 10, 0, P(0x10000), 0, 0, None, None) == B.SL_ERR_SHAPE
    assert f(P(0x10000), 10, 11, P(0x10000), 0, 0, None, None) == B.SL_ERR_SHAPE
    assert f(P(0x10000), 1 << 20, 5, P(0x10000), 0, 0, None, None) == B.SL_ERR_SHAPE
    assert f(P(0x10000), 12, 5, P(0x10000), 2, 5, None, None) == B.SL_ERR_INVALID_ARG


def _linear(fake, d_in=64, d_out=64, r=8, slice_kind=B.SL_SLICE_OUT, w_t=None):
    return B.SlLinearC(fake, w_t, d_in, d_out, slice_kind, r, fake, fake, 2.0, 0)


def test_linear_calls_reject_bad_arguments(lib):
    fake = 0x10000
    P = ctypes.c_void_p
    ch = B.SlChannelsC(fake, 64, 32)
    ys = (P * 1)(fake)
    ld = (ctypes.c_int64 * 1)(64)
    ws = _ws()
    fwd = lib.sl_sparse_linear_fwd
    lin = (B.SlLinearC * 1)(_linear(fake))
    chs = (B.SlChannelsC * 1)(ch)
    # context rows beyond the token count
    assert fwd(1, lin, chs, B.SL_EPI_NONE, P(fake), 64, 10, 11, 0, 0, P(fake), 8, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_SHAPE
    # LoRA rank not a multiple of 8
    bad = (B.SlLinearC * 1)(_linear(fake, r=12))
    assert fwd(1, bad, chs, B.SL_EPI_NONE, P(fake), 64, 10, 5, 0, 0, P(fake), 16, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_INVALID_ARG
    # channel count larger than the sliced side
    chs_bad = (B.SlChannelsC * 1)(B.SlChannelsC(fake, 64, 65))
    assert fwd(1, lin, chs_bad, B.SL_EPI_NONE, P(fake), 64, 10, 5, 0, 0, P(fake), 8, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_INVALID_ARG
    # misaligned pointer
    assert fwd(1, lin, chs, B.SL_EPI_NONE, P(fake + 2), 64, 10, 5, 0, 0, P(fake), 8, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_ALIGNMENT
    # input-sliced layer without its transposed weight
    lin_in = (B.SlLinearC * 1)(_linear(fake, slice_kind=B.SL_SLICE_IN))
    assert fwd(1, lin_in, chs, B.SL_EPI_NONE, P(fake), 64, 10, 5, 0, 0, P(fake), 8, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_INVALID_ARG
    # workspace query for a valid call
    assert fwd(1, lin, chs, B.SL_EPI_NONE, P(fake), 64, 10, 5, 0, 0, P(fake), 8, ys, ld, ctypes.byref(ws),
               None) == B.SL_ERR_WORKSPACE
    assert ws.needed > 256
    bwd = lib.sl_sparse_linear_bwd
    dys = (P * 1)(fake)
    assert bwd(4, lin, chs, B.SL_EPI_NONE, dys, ld, 10, 5, 0, 0, (P * 1)(fake), P(fake), 64, None, None,
               ctypes.byref(ws), None) == B.SL_ERR_INVALID_ARG
    lora = lib.sl_lora_fwd_bwd
    assert lora(B.SL_LORA_FWD, 0, lin, P(fake), 64, 10, 5, 0, None, P(fake), P(fake), 8, None, None, 0, None,
                None, None, None, None, ctypes.byref(ws), None) == B.SL_ERR_INVALID_ARG


def test_workspace_init_and_profile_hooks_host_side(lib):
    ws = _ws()
    assert lib.sl_workspace_init(ctypes.byref(ws), None) == B.SL_ERR_WORKSPACE
    assert lib.sl_profile_enable(0) == B.SL_OK
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_double()
    assert lib.sl_profile_read(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == B.SL_OK
    assert lib.sl_profile_read(None, None, None) == B.SL_ERR_INVALID_ARG


def test_layer_and_optimizer_entries_reject_bad_arguments(lib):
    """RMSNorm, residual add, AdamW, head-level selection, Wanda scores and the batched row
    gather check their arguments before any launch (fake device addresses are never touched)."""
    P = ctypes.c_void_p
    a, odd = P(0x10000), P(0x10002)  # 16-byte aligned / not
    # sl_rmsnorm_fwd(x, ldx, res, ldr, sum_out, lds, gamma, eps, y, ldy, rstd, n_rows, d, stream)
    f = lib.sl_rmsnorm_fwd
    assert f(None, 64, None, 0, None, 0, a, 1e-5, a, 64, a, 4, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, a, 64, None, 0, a, 1e-5, a, 64, a, 4, 64, None) == B.SL_ERR_INVALID_ARG  # res without sum_out
    assert f(a, 64, None, 0, None, 0, a, 1e-5, a, 64, a, 0, 64, None) == B.SL_ERR_SHAPE
    assert f(a, 64, None, 0, None, 0, a, 1e-5, a, 64, a, 4, 60, None) == B.SL_ERR_SHAPE
    assert f(a, 64, None, 0, None, 0, a, -1.0, a, 64, a, 4, 64, None) == B.SL_ERR_SHAPE
    assert f(odd, 64, None, 0, None, 0, a, 1e-5, a, 64, a, 4, 64, None) == B.SL_ERR_ALIGNMENT
    # sl_rmsnorm_bwd(dy, lddy, x, ldx, gamma, rstd, dres, ldr, dx, lddx, n_rows, d, stream)
    g = lib.sl_rmsnorm_bwd
    assert g(a, 64, a, 64, a, None, None, 0, a, 64, 4, 64, None) == B.SL_ERR_INVALID_ARG
    assert g(a, 64, a, 32, a, a, None, 0, a, 64, 4, 64, None) == B.SL_ERR_ALIGNMENT  # ld below d
    # sl_add_rows(a, lda, b, ldb, out, ldo, n_rows, d, stream)
    h = lib.sl_add_rows
    assert h(a, 64, None, 64, a, 64, 4, 64, None) == B.SL_ERR_INVALID_ARG
    assert h(a, 64, a, 64, a, 64, 4, 12, None) == B.SL_ERR_SHAPE
    # sl_adamw_step(p, g, m, v, p_bf16, n, lr, b1, b2, eps, wd, step, stream)
    w = lib.sl_adamw_step
    assert w(a, a, None, a, None, 10, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == B.SL_ERR_INVALID_ARG
    assert w(a, a, a, a, None, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, None) == B.SL_ERR_SHAPE
    assert w(a, a, a, a, None, 10, 1e-3, 1.0, 0.999, 1e-8, 0.0, 1, None) == B.SL_ERR_SHAPE
    assert w(a, a, a, a, None, 10, -1.0, 0.9, 0.999, 1e-8, 0.0, 1, None) == B.SL_ERR_SHAPE
    assert w(a, a, a, a, None, 10, 1e-3, 0.9, 0.999, 1e-8, 0.0, 0, None) == B.SL_ERR_SHAPE
    # sl_select_heads(scores, n_heads, head_dim, n_keep_heads, heads_per_group, sigma, sigma_wide, stream)
    sh = lib.sl_select_heads
    assert sh(None, 8, 128, 2, 4, a, None, None) == B.SL_ERR_INVALID_ARG
    assert sh(a, 8, 128, 9, 4, a, None, None) == B.SL_ERR_SHAPE
    assert sh(a, 0, 128, 1, 4, a, None, None) == B.SL_ERR_SHAPE
    assert sh(a, 8, 128, 2, 0, a, a, None) == B.SL_ERR_INVALID_ARG  # query side without a group size
    # sl_wanda_scores(x, n_ctx, d_in, ldx, n_proj, w, d_out, ldw, scores, ws, stream)
    wa = lib.sl_wanda_scores
    ws = B.SlWorkspaceC(None, 0, 0)
    wp = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    assert wa(a, 16, 64, 64, 0, wp, 32, 64, a, ctypes.byref(ws), None) == B.SL_ERR_INVALID_ARG
    assert wa(a, 0, 64, 64, 2, wp, 32, 64, a, ctypes.byref(ws), None) == B.SL_ERR_SHAPE
    assert wa(a, 16, 60, 64, 2, wp, 32, 64, a, ctypes.byref(ws), None) == B.SL_ERR_ALIGNMENT
    assert wa(a, 16, 64, 64, 2, wp, 32, 64, a, ctypes.byref(ws), None) == B.SL_ERR_WORKSPACE
    # sl_gather_rows_batch(n, src[], ld_src[], src_rows[], perm[], n_rows[], n_cols[], dst[], ld_dst[], stream)
    gb = lib.sl_gather_rows_batch
    ptrs = lambda *v: (ctypes.c_void_p * len(v))(*v)
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)
    ok = dict(src=ptrs(0x10000), ld=i64(64), srows=i64(16), perm=ptrs(0x20000), rows=i64(4), cols=i64(64),
              dst=ptrs(0x30000))
    args = lambda n, **k: [n] + [k.get(x, ok[x]) for x in ("src", "ld", "srows", "perm", "rows", "cols", "dst")] + \
        [k.get("ldd", i64(64)), None]
    assert gb(*args(0)) == B.SL_ERR_INVALID_ARG
    assert gb(*args(9)) == B.SL_ERR_INVALID_ARG
    assert gb(*args(1, perm=ptrs(None))) == B.SL_ERR_INVALID_ARG
    assert gb(*args(1, srows=None)) == B.SL_ERR_INVALID_ARG
    assert gb(*args(1, rows=i64(-1))) == B.SL_ERR_SHAPE
    assert gb(*args(1, cols=i64(0))) == B.SL_ERR_SHAPE
    assert gb(*args(1, srows=i64(0))) == B.SL_ERR_SHAPE
    assert gb(*args(1, ldd=i64(32))) == B.SL_ERR_SHAPE
    # a job without rows launches nothing, whatever its pointers
    assert gb(*args(1, rows=i64(0), src=ptrs(None), perm=ptrs(None), dst=ptrs(None))) == B.SL_OK


def test_pair_tile_rows_setting_host_side(lib):
    """The tile-height setting accepts 0 (chosen per launch), 128 (no CTA pairs), 256 and 512,
    and nothing else."""
    for rows in (128, 256, 512, 0):
        assert lib.sl_set_pair_tile_rows(rows) == B.SL_OK
    for rows in (-1, 1, 64, 384, 1024):
        assert lib.sl_set_pair_tile_rows(rows) == B.SL_ERR_INVALID_ARG
    assert lib.sl_set_pair_tile_rows(0) == B.SL_OK


def test_debug_build_exports_and_flags_host_side():
    """The debug build exports the same entry points and says it checks bounds; the release build
    says it does not, and its debug word always reads 0."""
    if not os.path.exists(B.DEBUG_LIB_PATH):
        pytest.skip("debug library not built")
    dbg = B.load(B.DEBUG_LIB_PATH)
    for name in B.EXPORTED:
        getattr(dbg, name)
    assert dbg.sl_debug_bounds_enabled() == 1
    rel = B.load(B.LIB_PATH)
    assert rel.sl_debug_bounds_enabled() == 0
    code = ctypes.c_int32(-1)
    assert rel.sl_read_debug_flag(ctypes.byref(code), None) == B.SL_OK and code.value == 0
    assert rel.sl_read_debug_flag(None, None) == B.SL_ERR_INVALID_ARG


def test_permute_rows_rejects_bad_arguments(lib):
    """sl_permute_rows(src, ld_src, src_rows, perm, n_rows, n_cols, dst, ld_dst, stream): host checks
    only; nothing is launched."""
    P = ctypes.c_void_p
    f = lib.sl_permute_rows
    a = P(0x10000)
    assert f(None, 64, 8, a, 4, 64, a, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, 8, None, 4, 64, a, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, 0, a, 4, 64, a, 64, None) == B.SL_ERR_SHAPE
    assert f(a, 64, 8, a, 0, 64, a, 64, None) == B.SL_ERR_SHAPE
    assert f(a, 32, 8, a, 4, 64, a, 64, None) == B.SL_ERR_SHAPE


def test_permute_rows_sigma_rejects_bad_arguments(lib):
    """sl_permute_rows_sigma(src, ld_src, src_rows, perm, n_rows, n_cols, sigma, n_ctx, to_sigma, dst,
    ld_dst, stream): host checks only; nothing is launched."""
    P = ctypes.c_void_p
    f = lib.sl_permute_rows_sigma
    a, odd = P(0x10000), P(0x10008)
    assert f(None, 64, 8, a, 4, 64, a, 2, 1, a, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, 8, a, 4, 64, None, 2, 1, a, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, 8, a, 4, 64, a, 2, 1, None, 64, None) == B.SL_ERR_INVALID_ARG
    assert f(a, 64, 0, a, 4, 64, a, 2, 1, a, 64, None) == B.SL_ERR_SHAPE
    assert f(a, 64, 8, a, 4, 64, a, -1, 1, a, 64, None) == B.SL_ERR_SHAPE
    assert f(a, 1 << 15, 8, a, 4, 16392, a, 2, 1, a, 1 << 15, None) == B.SL_ERR_SHAPE  # wider than 16384
    assert f(a, 60, 8, a, 4, 60, a, 2, 1, a, 64, None) == B.SL_ERR_ALIGNMENT
    assert f(odd, 64, 8, a, 4, 64, a, 2, 1, a, 64, None) == B.SL_ERR_ALIGNMENT
