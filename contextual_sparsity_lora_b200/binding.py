"""ctypes binding of libsparselora.so. Same names as the C ABI (include/sparselora.h);
argument marshalling only: tensors are passed as device pointers, the stream is
torch's current stream, and every computation happens in the library's kernels.

The library must have been built in-tree (``python -m contextual_sparsity_lora_b200.build``);
there is no fallback: a missing library raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparselora.so")

SL_OK, SL_ERR_INVALID_ARG, SL_ERR_SHAPE, SL_ERR_ALIGNMENT, SL_ERR_WORKSPACE, SL_ERR_UNSUPPORTED, SL_ERR_CUDA, \
    SL_ERR_DEVICE_FLAG = range(8)
SL_CRIT_L2, SL_CRIT_SWIGLU_L2, SL_CRIT_QK = 0, 1, 2
SL_DT_BF16, SL_DT_F32 = 0, 1
SL_SLICE_OUT, SL_SLICE_IN = 0, 1
SL_LAYOUT_NATURAL, SL_LAYOUT_SIGMA = 0, 1
SL_EPI_NONE, SL_EPI_SWIGLU = 0, 1
SL_LORA_FWD, SL_LORA_BWD = 0, 1

EXPORTED = ("sl_status_string", "sl_version", "sl_keep_count", "sl_workspace_init", "sl_read_device_flag",
            "sl_svd_estimate", "sl_select_channels", "sl_lora_fwd_bwd", "sl_sparse_linear_fwd",
            "sl_sparse_linear_bwd", "sl_prepare_weight", "sl_permute_rows", "sl_profile_enable", "sl_profile_read",
            "sl_svd_estimate_noalloc", "sl_profile_launches", "sl_svd_partials_count", "sl_svd_estimate_partials",
            "sl_svd_scores_from_partials", "sl_select_heads", "sl_wanda_scores", "sl_rmsnorm_fwd", "sl_rmsnorm_bwd",
            "sl_add_rows", "sl_adamw_step", "sl_gather_rows_batch", "sl_set_pair_tile_rows",
            "sl_debug_bounds_enabled", "sl_read_debug_flag", "sl_attention_fwd", "sl_attention_bwd",
            "sl_lora_fwd_estimate", "sl_svd_scores_from_z", "sl_permute_rows_sigma")


class SlWorkspaceC(ctypes.Structure):
    _fields_ = [("ptr", c_void_p), ("bytes", c_size_t), ("needed", c_size_t)]


class SlLinearC(ctypes.Structure):
    _fields_ = [("w", c_void_p), ("w_t", c_void_p), ("d_in", c_int64), ("d_out", c_int64), ("slice", c_int32),
                ("r", c_int32), ("lora_a", c_void_p), ("lora_b", c_void_p), ("lora_scale", c_float),
                ("pad_", c_int32), ("w_kept", c_void_p)]


class SlChannelsC(ctypes.Structure):
    _fields_ = [("sigma", c_void_p), ("n_side", c_int64), ("n_keep", c_int64)]


class SparseLoRAError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} (status {code})")


DEBUG_LIB_PATH = os.path.join(_HERE, "libsparselora_debug.so")

_lib = None


def lib():
    """The library every wrapper below calls (the in-tree release build unless `using_library`
    selected another one)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


class using_library:
    """Context manager: the wrappers call the library at `path` (e.g. DEBUG_LIB_PATH, the build
    with device-side bounds checks) inside the block."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def load(path):
    """Load a build of the library and declare its entry points' argument types."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m contextual_sparsity_lora_b200.build`")
    L = ctypes.CDLL(path)
    P = c_void_p
    L.sl_status_string.restype = c_char_p
    L.sl_status_string.argtypes = [c_int32]
    L.sl_version.restype = c_int32
    L.sl_keep_count.restype = c_int64
    L.sl_keep_count.argtypes = [c_double, c_int64]
    L.sl_workspace_init.argtypes = [POINTER(SlWorkspaceC), P]
    L.sl_read_device_flag.argtypes = [POINTER(SlWorkspaceC), POINTER(c_int32), P]
    L.sl_svd_estimate.argtypes = [c_int32, c_int32, P, c_int64, c_int64, c_int64, c_int32, POINTER(c_void_p),
                                  POINTER(c_void_p), POINTER(c_int64), c_int32, c_int32, c_int32, c_int32, P, P,
                                  POINTER(SlWorkspaceC), P]
    L.sl_svd_partials_count.restype = c_int64
    L.sl_svd_partials_count.argtypes = [c_int32, c_int32, POINTER(c_int64), c_int32]
    L.sl_svd_estimate_partials.argtypes = [c_int32, c_int32, P, c_int64, c_int64, c_int64, c_int32,
                                           POINTER(c_void_p), POINTER(c_void_p), POINTER(c_int64), c_int32,
                                           c_int32, c_int32, c_int32, P, POINTER(SlWorkspaceC), P]
    L.sl_svd_scores_from_partials.argtypes = [c_int32, c_int32, c_int32, POINTER(c_void_p), POINTER(c_int64),
                                              c_int32, c_int32, c_int32, c_int32, P, P, P, P]
    L.sl_select_channels.argtypes = [P, c_int64, c_int64, P, c_int32, c_int32, P, P]
    L.sl_select_heads.argtypes = [P, c_int32, c_int32, c_int32, c_int32, P, P, P]
    L.sl_rmsnorm_fwd.argtypes = [P, c_int64, P, c_int64, P, c_int64, P, c_float, P, c_int64, P, c_int64, c_int64, P]
    L.sl_rmsnorm_bwd.argtypes = [P, c_int64, P, c_int64, P, P, P, c_int64, P, c_int64, c_int64, c_int64, P]
    L.sl_add_rows.argtypes = [P, c_int64, P, c_int64, P, c_int64, c_int64, c_int64, P]
    L.sl_adamw_step.argtypes = [P, P, P, P, P, c_int64, c_float, c_float, c_float, c_float, c_float, c_int32, P]
    L.sl_wanda_scores.argtypes = [P, c_int64, c_int64, c_int64, c_int32, POINTER(c_void_p), c_int64, c_int64, P,
                                  POINTER(SlWorkspaceC), P]
    L.sl_lora_fwd_bwd.argtypes = [c_int32, c_int32, POINTER(SlLinearC), P, c_int64, c_int64, c_int64, c_int32,
                                  POINTER(SlChannelsC), P, P, c_int64, POINTER(c_void_p), POINTER(c_int64),
                                  c_int32, POINTER(SlChannelsC), POINTER(c_void_p), POINTER(c_void_p),
                                  POINTER(c_void_p), POINTER(c_void_p), POINTER(SlWorkspaceC), P]
    L.sl_sparse_linear_fwd.argtypes = [c_int32, POINTER(SlLinearC), POINTER(SlChannelsC), c_int32, P, c_int64,
                                       c_int64, c_int64, c_int32, c_int32, P, c_int64, POINTER(c_void_p),
                                       POINTER(c_int64), POINTER(SlWorkspaceC), P]
    L.sl_sparse_linear_bwd.argtypes = [c_int32, POINTER(SlLinearC), POINTER(SlChannelsC), c_int32,
                                       POINTER(c_void_p), POINTER(c_int64), c_int64, c_int64, c_int32, c_int32,
                                       POINTER(c_void_p), P, c_int64, POINTER(c_void_p), POINTER(c_void_p),
                                       POINTER(SlWorkspaceC), P]
    L.sl_prepare_weight.argtypes = [P, c_int64, c_int64, P, P]
    L.sl_profile_enable.argtypes = [c_int32]
    L.sl_profile_read.argtypes = [POINTER(c_int64), POINTER(c_int64), POINTER(c_double)]
    L.sl_permute_rows.argtypes = [P, c_int64, c_int64, P, c_int64, c_int64, P, c_int64, P]
    L.sl_permute_rows_sigma.argtypes = [P, c_int64, c_int64, P, c_int64, c_int64, P, c_int64, c_int32, P, c_int64,
                                        P]
    L.sl_gather_rows_batch.argtypes = [c_int32, P, P, P, P, P, P, P, P, P]
    L.sl_debug_bounds_enabled.restype = c_int32
    L.sl_lora_fwd_estimate.argtypes = [c_int32, POINTER(SlLinearC), P, c_int64, c_int64, c_int64, P, P, c_int64,
                                       c_int32, c_int32, P, c_int64, P, c_int64, POINTER(SlWorkspaceC), P]
    L.sl_svd_scores_from_z.argtypes = [c_int32, c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, c_int32, c_int32,
                                       c_int32, P, c_int64, c_int64, P, P, POINTER(SlWorkspaceC), P]
    L.sl_attention_fwd.argtypes = [P, P, P, c_int64, c_int64, c_int32, c_int32, c_int32, c_int32, c_int32, P, P,
                                   POINTER(SlWorkspaceC), P]
    L.sl_attention_bwd.argtypes = [P, P, P, P, P, P, c_int64, c_int64, c_int32, c_int32, c_int32, c_int32, c_int32,
                                   P, P, P, POINTER(SlWorkspaceC), P]
    L.sl_read_debug_flag.argtypes = [POINTER(c_int32), P]
    L.sl_set_pair_tile_rows.argtypes = [c_int32]
    for n in EXPORTED:
        if n not in ("sl_status_string", "sl_version", "sl_keep_count", "sl_svd_partials_count",
                     "sl_debug_bounds_enabled"):
            getattr(L, n).restype = c_int32
    return L


def status_string(code: int) -> str:
    return lib().sl_status_string(int(code)).decode()


def _check(fn, code):
    if code != SL_OK:
        raise SparseLoRAError(fn, code)


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream():
    return c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptrs(ts):
    return (c_void_p * max(1, len(ts)))(*[None if t is None else t.data_ptr() for t in ts])


def _i64s(vs):
    return (c_int64 * max(1, len(vs)))(*[int(v) for v in vs])


class Workspace:
    """Caller-owned scratch memory for the library (a torch byte buffer that grows on demand)."""

    def __init__(self, device="cuda", nbytes: int = 1 << 20):
        self.device = device
        self.buf = None
        self._alloc(nbytes)

    def _alloc(self, nbytes):
        self.buf = torch.empty(int(nbytes), dtype=torch.uint8, device=self.device)
        self.c = SlWorkspaceC(self.buf.data_ptr(), self.buf.numel(), 0)
        _check("sl_workspace_init", lib().sl_workspace_init(ctypes.byref(self.c), _stream()))

    def call(self, fn_name, *args):
        """Run one library call with this workspace, growing it once if the call asks for more."""
        fn = getattr(lib(), fn_name)
        code = fn(*args, ctypes.byref(self.c), _stream())
        if code == SL_ERR_WORKSPACE and self.c.needed > self.c.bytes:
            self._alloc(self.c.needed + (1 << 20))
            code = fn(*args, ctypes.byref(self.c), _stream())
        _check(fn_name, code)

    def read_device_flag(self) -> int:
        v = c_int32(0)
        code = lib().sl_read_device_flag(ctypes.byref(self.c), ctypes.byref(v), _stream())
        if code not in (SL_OK, SL_ERR_DEVICE_FLAG):
            _check("sl_read_device_flag", code)
        return int(v.value)


def linear_desc(w, lora_a, lora_b, lora_scale, slice_kind, w_t=None, w_kept=None) -> SlLinearC:
    d_out, d_in = w.shape
    return SlLinearC(w.data_ptr(), None if w_t is None else w_t.data_ptr(), d_in, d_out, slice_kind,
                     lora_a.shape[0], lora_a.data_ptr(), lora_b.data_ptr(), float(lora_scale), 0,
                     None if w_kept is None else w_kept.data_ptr())


def channels_desc(sigma, n_keep) -> SlChannelsC:
    return SlChannelsC(sigma.data_ptr(), sigma.numel(), int(n_keep))


def _arr(cls, items):
    return (cls * max(1, len(items)))(*items)


# ---------------------------------------------------------------------------- entry points

def sl_version() -> int:
    return int(lib().sl_version())


def sl_keep_count(ratio: float, n: int) -> int:
    return int(lib().sl_keep_count(float(ratio), int(n)))


def sl_svd_estimate(ws: Workspace, crit, x, n_ctx, w_a, w_b, k, scores, scores_v=None, n_q_heads=0,
                    n_kv_heads=0, head_dim=0):
    dtype = SL_DT_F32 if x.dtype == torch.float32 else SL_DT_BF16
    d_out = [t.shape[1] for t in w_b]
    ws.call("sl_svd_estimate", crit, dtype, _ptr(x), int(n_ctx), x.shape[1], x.stride(0), len(w_a), _ptrs(w_a),
            _ptrs(w_b), _i64s(d_out), int(k), int(n_q_heads), int(n_kv_heads), int(head_dim), _ptr(scores),
            _ptr(scores_v))


def sl_svd_estimate_noalloc(crit, x, n_ctx, w_a, w_b, k, scores, scores_v=None, n_q_heads=0, n_kv_heads=0,
                            head_dim=0, device_flag=None):
    """sl_svd_estimate on the library's fixed scratch array (no workspace, no allocation).
    Returns the scratch bytes the call needed; device_flag: optional int32 CUDA tensor that
    receives the call's device error word."""
    dtype = SL_DT_F32 if x.dtype == torch.float32 else SL_DT_BF16
    d_out = [t.shape[1] for t in w_b]
    needed = c_int64(0)
    _check("sl_svd_estimate_noalloc",
           lib().sl_svd_estimate_noalloc(crit, dtype, _ptr(x), int(n_ctx), x.shape[1], x.stride(0), len(w_a),
                                         _ptrs(w_a), _ptrs(w_b), _i64s(d_out), int(k), int(n_q_heads),
                                         int(n_kv_heads), int(head_dim), _ptr(scores), _ptr(scores_v),
                                         ctypes.byref(needed), _ptr(device_flag), _stream()))
    return int(needed.value)


def sl_lora_fwd_estimate(ws: Workspace, lins, x, n_ctx, xa_s, xa, n_proj, k, w_a_t, z):
    """x A^T of the adapters (xa, xa_s) and the estimator's Z = X_ctx W_A (z [n_ctx, n_proj k] fp32)
    from one pass over x; w_a_t [n_proj k, d_in] bf16 stacks the transposed factors."""
    ws.call("sl_lora_fwd_estimate", len(lins), _arr(SlLinearC, list(lins)), _ptr(x), x.stride(0), x.shape[0],
            int(n_ctx), _ptr(xa), _ptr(xa_s), xa_s.stride(0), int(n_proj), int(k), _ptr(w_a_t), w_a_t.stride(0),
            _ptr(z), z.stride(0))


def sl_svd_scores_from_z(ws: Workspace, crit, w_b, k, z, n_ctx, scores, scores_v=None, n_q_heads=0, n_kv_heads=0,
                         head_dim=0):
    ws.call("sl_svd_scores_from_z", int(crit), len(w_b), _ptrs(list(w_b)), _i64s([t.shape[1] for t in w_b]), int(k),
            int(n_q_heads), int(n_kv_heads), int(head_dim), _ptr(z), z.stride(0), int(n_ctx), _ptr(scores),
            _ptr(scores_v))


def sl_svd_partials_count(crit, w_b, k):
    d_out = [t.shape[1] for t in w_b]
    return int(lib().sl_svd_partials_count(crit, len(w_b), _i64s(d_out), int(k)))


def sl_svd_estimate_partials(ws: Workspace, crit, x, n_ctx, w_a, w_b, k, partials, n_q_heads=0, n_kv_heads=0,
                             head_dim=0):
    """The rank-local criterion statistics (fp64 `partials`, sl_svd_partials_count elements)."""
    dtype = SL_DT_F32 if x.dtype == torch.float32 else SL_DT_BF16
    d_out = [t.shape[1] for t in w_b]
    ws.call("sl_svd_estimate_partials", crit, dtype, _ptr(x), int(n_ctx), x.shape[1], x.stride(0), len(w_a),
            _ptrs(w_a), _ptrs(w_b), _i64s(d_out), int(k), int(n_q_heads), int(n_kv_heads), int(head_dim),
            _ptr(partials))


def sl_svd_scores_from_partials(crit, w_b, k, partials, scores, scores_v=None, n_q_heads=0, n_kv_heads=0,
                                head_dim=0):
    dtype = SL_DT_F32 if w_b[0].dtype == torch.float32 else SL_DT_BF16
    d_out = [t.shape[1] for t in w_b]
    _check("sl_svd_scores_from_partials",
           lib().sl_svd_scores_from_partials(crit, dtype, len(w_b), _ptrs(w_b), _i64s(d_out), int(k), int(n_q_heads),
                                             int(n_kv_heads), int(head_dim), _ptr(partials), _ptr(scores),
                                             _ptr(scores_v), _stream()))


def sl_select_channels(scores, n_keep, sigma, heads_per_group=0, head_dim=0, sigma_wide=None):
    _check("sl_select_channels",
           lib().sl_select_channels(_ptr(scores), scores.numel(), int(n_keep), _ptr(sigma), int(heads_per_group),
                                    int(head_dim), _ptr(sigma_wide), _stream()))


def sl_select_heads(scores, n_heads, head_dim, n_keep_heads, sigma, heads_per_group=0, sigma_wide=None):
    _check("sl_select_heads",
           lib().sl_select_heads(_ptr(scores), int(n_heads), int(head_dim), int(n_keep_heads), int(heads_per_group),
                                 _ptr(sigma), _ptr(sigma_wide), _stream()))


def sl_wanda_scores(ws: Workspace, x, n_ctx, w, scores):
    """Wanda-style channel scores over the context rows x[:n_ctx] for the weights w (one index set)."""
    ws.call("sl_wanda_scores", _ptr(x), int(n_ctx), x.shape[1], x.stride(0), len(w), _ptrs(w), w[0].shape[0],
            w[0].stride(0), _ptr(scores))


def sl_rmsnorm_fwd(x, gamma, eps, y, rstd, res=None, sum_out=None):
    _check("sl_rmsnorm_fwd",
           lib().sl_rmsnorm_fwd(_ptr(x), x.stride(0), _ptr(res), res.stride(0) if res is not None else 0,
                                _ptr(sum_out), sum_out.stride(0) if sum_out is not None else 0, _ptr(gamma),
                                float(eps), _ptr(y), y.stride(0), _ptr(rstd), x.shape[0], x.shape[1], _stream()))


def sl_rmsnorm_bwd(dy, x, gamma, rstd, dx, dres=None):
    _check("sl_rmsnorm_bwd",
           lib().sl_rmsnorm_bwd(_ptr(dy), dy.stride(0), _ptr(x), x.stride(0), _ptr(gamma), _ptr(rstd), _ptr(dres),
                                dres.stride(0) if dres is not None else 0, _ptr(dx), dx.stride(0), x.shape[0],
                                x.shape[1], _stream()))


def sl_add_rows(a, b, out):
    _check("sl_add_rows", lib().sl_add_rows(_ptr(a), a.stride(0), _ptr(b), b.stride(0), _ptr(out), out.stride(0),
                                            a.shape[0], a.shape[1], _stream()))


def sl_adamw_step(params, grads, m, v, step, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
                  params_bf16=None):
    _check("sl_adamw_step", lib().sl_adamw_step(_ptr(params), _ptr(grads), _ptr(m), _ptr(v), _ptr(params_bf16),
                                                params.numel(), float(lr), float(beta1), float(beta2), float(eps),
                                                float(weight_decay), int(step), _stream()))


def sl_lora_fwd_bwd(ws: Workspace, mode, lins, x, n_ctx, xa_s, xa=None, in_layout=SL_LAYOUT_NATURAL, in_ch=None,
                    dy=(), out_layout=SL_LAYOUT_NATURAL, out_ch=(), dya=(), dya_s=(), dA=(), dB=()):
    lin_arr = _arr(SlLinearC, list(lins))
    in_c = ctypes.byref(in_ch) if in_ch is not None else None
    out_arr = _arr(SlChannelsC, list(out_ch)) if out_ch else None
    ws.call("sl_lora_fwd_bwd", mode, len(lins), lin_arr, _ptr(x), x.stride(0), x.shape[0], int(n_ctx), in_layout,
            in_c, _ptr(xa), _ptr(xa_s), xa_s.stride(0), _ptrs(list(dy)), _i64s([t.stride(0) for t in dy]),
            out_layout, out_arr, _ptrs(list(dya)), _ptrs(list(dya_s)), _ptrs(list(dA)), _ptrs(list(dB)))


def sl_sparse_linear_fwd(ws: Workspace, lins, chans, epi, x, n_ctx, xa_s, ys, in_layout=SL_LAYOUT_NATURAL,
                         out_layout=SL_LAYOUT_NATURAL):
    ws.call("sl_sparse_linear_fwd", len(lins), _arr(SlLinearC, list(lins)), _arr(SlChannelsC, list(chans)), epi,
            _ptr(x), x.stride(0), x.shape[0], int(n_ctx), in_layout, out_layout, _ptr(xa_s), xa_s.stride(0),
            _ptrs(list(ys)), _i64s([t.stride(0) for t in ys]))


def sl_sparse_linear_bwd(ws: Workspace, lins, chans, epi, dys, n_ctx, dya_s, dx=None, in_layout=SL_LAYOUT_NATURAL,
                         out_layout=SL_LAYOUT_NATURAL, aux=(), aux_out=()):
    ld = dx.stride(0) if dx is not None else aux_out[0].stride(0)
    ws.call("sl_sparse_linear_bwd", len(lins), _arr(SlLinearC, list(lins)), _arr(SlChannelsC, list(chans)), epi,
            _ptrs(list(dys)), _i64s([t.stride(0) for t in dys]), dys[0].shape[0], int(n_ctx), in_layout,
            out_layout, _ptrs(list(dya_s)), _ptr(dx), ld, _ptrs(list(aux)), _ptrs(list(aux_out)))


def sl_prepare_weight(w, w_t):
    d_out, d_in = w.shape
    _check("sl_prepare_weight", lib().sl_prepare_weight(_ptr(w), d_out, d_in, _ptr(w_t), _stream()))


def sl_permute_rows(src, perm, dst):
    """dst[i, :] = src[perm[i], :] for i < perm.numel() (src may have more rows than dst)."""
    _check("sl_permute_rows", lib().sl_permute_rows(_ptr(src), src.stride(0), src.shape[0], _ptr(perm), perm.numel(),
                                                    src.shape[1], _ptr(dst), dst.stride(0), _stream()))


def sl_permute_rows_sigma(src, perm, dst, sigma, n_ctx, to_sigma):
    """Row permutation with the sigma-layout channel order on context rows: to_sigma, destination
    rows i < n_ctx get dst[i, p] = src[perm[i], sigma[p]]; else source rows perm[i] < n_ctx are in
    the sigma layout and dst[i, sigma[p]] = src[perm[i], p]; other rows are copied."""
    _check("sl_permute_rows_sigma",
           lib().sl_permute_rows_sigma(_ptr(src), src.stride(0), src.shape[0], _ptr(perm), perm.numel(), src.shape[1],
                                       _ptr(sigma), int(n_ctx), 1 if to_sigma else 0, _ptr(dst), dst.stride(0),
                                       _stream()))


def sl_gather_rows_batch(srcs, perms, dsts):
    """dst_q[i, :] = src_q[perm_q[i], :] for every q, in one launch (at most 8 gathers);
    perm_q holds one int32 index per row of dst_q."""
    n = len(srcs)
    _check("sl_gather_rows_batch", lib().sl_gather_rows_batch(
        n, _ptrs(srcs), _i64s([t.stride(0) for t in srcs]), _i64s([t.shape[0] for t in srcs]), _ptrs(perms),
        _i64s([t.numel() for t in perms]), _i64s([t.shape[1] for t in srcs]), _ptrs(dsts),
        _i64s([t.stride(0) for t in dsts]), _stream()))


def sl_debug_bounds_enabled() -> bool:
    return bool(lib().sl_debug_bounds_enabled())


def sl_read_debug_flag() -> int:
    """Code recorded by a failed bounds check of the entries without a workspace (debug build),
    cleared by the read; 0 when none (always 0 in the release build). Synchronises."""
    code = c_int32(0)
    rc = lib().sl_read_debug_flag(ctypes.byref(code), _stream())
    if rc not in (SL_OK, SL_ERR_DEVICE_FLAG):
        _check("sl_read_debug_flag", rc)
    return int(code.value)


def sl_attention_fwd(ws: Workspace, q, k, v, n_seq, n_q_heads, n_kv_heads, head_dim, o, lse):
    """Causal GQA attention over n_seq equal-length sequences (rows in sequence order): o and the
    per-row log-sum-exp lse [n_q_heads, T] for the backward."""
    ws.call("sl_attention_fwd", _ptr(q), _ptr(k), _ptr(v), q.stride(0), k.stride(0), int(n_seq),
            q.shape[0] // int(n_seq), int(n_q_heads), int(n_kv_heads), int(head_dim), _ptr(o), _ptr(lse))


def sl_attention_bwd(ws: Workspace, q, k, v, o, d_o, lse, n_seq, n_q_heads, n_kv_heads, head_dim, dq, dk, dv):
    ws.call("sl_attention_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), q.stride(0), k.stride(0),
            int(n_seq), q.shape[0] // int(n_seq), int(n_q_heads), int(n_kv_heads), int(head_dim), _ptr(dq), _ptr(dk),
            _ptr(dv))


def sl_set_pair_tile_rows(rows: int):
    """Tile height of the CTA-pair GEMM for later launches: 256, 512, 128 (no CTA pairs: the
    one-CTA kernel), or 0 (chosen per launch)."""
    _check("sl_set_pair_tile_rows", lib().sl_set_pair_tile_rows(int(rows)))


class pair_tile_rows:
    """Context manager that forces the CTA-pair tile height inside a block of calls (and
    restores the per-launch choice after it)."""

    def __init__(self, rows: int):
        self.rows = int(rows)

    def __enter__(self):
        sl_set_pair_tile_rows(self.rows)
        return self

    def __exit__(self, *exc):
        sl_set_pair_tile_rows(0)


def sl_profile_enable(on: bool):
    _check("sl_profile_enable", lib().sl_profile_enable(1 if on else 0))


def sl_profile_launches(capacity=4096):
    """[(milliseconds, kind)] of the GEMM-engine launches recorded since the last read
    (kind 0: one-CTA, 1: CTA pairs 256-row tiles, 2: CTA pairs 512-row tiles)."""
    ms = (ctypes.c_double * capacity)()
    kind = (ctypes.c_int32 * capacity)()
    n = c_int64(0)
    _check("sl_profile_launches", lib().sl_profile_launches(capacity, ms, kind, ctypes.byref(n)))
    return [(float(ms[i]), int(kind[i])) for i in range(min(n.value, capacity))]


def sl_profile_read():
    """(kernel launches, GEMM-engine launches, GEMM-engine milliseconds) since the last read."""
    a, b, c = c_int64(0), c_int64(0), c_double(0.0)
    _check("sl_profile_read", lib().sl_profile_read(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return int(a.value), int(b.value), float(c.value)
