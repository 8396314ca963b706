"""One fine-tuning step of a SparseLoRA FFN block or attention-projection block,
composed from the C ABI calls (no arithmetic here: buffers are allocated with torch,
every stage runs in libsparselora's kernels).

Rows are in context-first order (context rows [0, n_ctx), then output rows).
Dense mode (keep ratio 1, no estimator) is the dense-LoRA baseline on the same kernels.
"""
from __future__ import annotations

import torch

from . import binding as B


# Where the sliced products find the kept weight rows: in a compacted copy made once per step
# ("compact", the default: the tiled operand loads of the copy outrun the row-gather copies), or
# in place through sigma ("gather": tile::gather4 copies of four 128-byte rows each).
KEPT_ROWS = ("compact", "gather")


def _empty(shape, dtype, device):
    return torch.empty(*shape, dtype=dtype, device=device)


class _Side:
    """A second stream for a chain of calls that does not depend on the main chain (and the
    workspace it needs: concurrent calls must not share scratch). `fork` makes the side
    stream wait for the work queued so far; `join` makes the main stream wait for the side
    chain. Inside CUDA-graph capture this becomes two parallel branches of the graph."""

    def __init__(self, device):
        self.stream = torch.cuda.Stream(device=device)
        self.ws = B.Workspace(device)

    def fork(self):
        self.stream.wait_stream(torch.cuda.current_stream())
        return torch.cuda.stream(self.stream)

    def join(self):
        torch.cuda.current_stream().wait_stream(self.stream)

    def mark(self):
        """An event after the work queued on the side stream so far (wait on it with
        torch.cuda.current_stream().wait_event to join only that part)."""
        ev = torch.cuda.Event()
        ev.record(self.stream)
        return ev


class DataParallel:
    """Ranks that each hold part of one global batch ([WT] "Oracle Sparse Neuron Selection
    Criteria": one index set per batch). The criterion statistics of each rank's context rows
    (sl_svd_estimate_partials) are summed over the ranks before the scores and the top-n, so
    every rank keeps the same channels; the LoRA gradients (sums over tokens) are summed over
    the ranks after the backward. One fp64 all-reduce per block for the statistics (the FFN's
    per-channel sums of squares, or the attention block's Gram matrix) and one fp32 all-reduce
    per block for its gradients. world == 1 leaves every path as on one GPU."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1

    @property
    def active(self) -> bool:
        return self.world > 1

    def all_reduce(self, t):
        if self.world > 1:
            import torch.distributed as dist
            dist.all_reduce(t, group=self.group)


class _GradBuffer:
    """One flat buffer holding a block's LoRA matrices (gradients in fp32, or the parameters'
    bf16 working copy with initial values), so that one collective or one optimiser launch
    covers them all; views start on 64-element boundaries (16-byte alignment and more), and the
    gradient and parameter buffers of a block share the layout."""

    def __init__(self, shapes, device, dtype=torch.float32, init=None):
        self.offsets, n = [], 0
        for sh in shapes:
            self.offsets.append(n)
            cnt = 1
            for d in sh:
                cnt *= d
            n += (cnt + 63) // 64 * 64
        self.flat = torch.zeros(n, dtype=dtype, device=device)
        self.views = [self.flat[o:o + sh[0] * sh[1]].view(*sh) for o, sh in zip(self.offsets, shapes)]
        if init is not None:
            for v, t in zip(self.views, init):
                v.copy_(t.to(device=device, dtype=dtype))


class FFNBlock:
    """SwiGLU FFN: gate/up (output channels sliced), down (input channels sliced), one
    index set shared by all three; L2 criterion on the estimated SiLU(gate) * up."""

    CRITERIA = ("svd", "wanda", "random")

    def __init__(self, gate, up, down, lora_gate, lora_up, lora_down, lora_scale, k, n_tok, n_ctx, ratio,
                 device="cuda", dense=False, dp=None, criterion="svd", seed=0, kept_rows="compact"):
        """criterion: "svd" (SwiGLU L2 of the SVD estimate, the method's criterion), or the
        criterion ablation's alternatives "wanda" (Wanda-style channel scores of the frozen
        gate/up weights) and "random" (uniform scores from a generator seeded with `seed`).
        kept_rows: "compact" (a compacted copy of the kept rows, rebuilt once per step and
        shared by the forward and backward products; the faster form on B200) or "gather" (the
        sliced products read the kept weight rows in place, through sigma, with the GEMM's
        row-gather copies)."""
        if criterion not in self.CRITERIA:
            raise ValueError(f"criterion {criterion!r} not in {self.CRITERIA}")
        if kept_rows not in KEPT_ROWS:
            raise ValueError(f"kept_rows {kept_rows!r} not in {KEPT_ROWS}")
        self.kept_rows = kept_rows
        if criterion != "svd" and dp is not None and dp.active:
            raise ValueError("the ablation criteria run on one rank")
        self.criterion = criterion
        self.rng = torch.Generator(device=device)
        self.rng.manual_seed(int(seed))
        bf = torch.bfloat16
        self.device = device
        self.D = gate.W.shape[1]
        self.F = gate.W.shape[0]
        self.k = k
        self.n_tok, self.n_ctx = n_tok, n_ctx
        self.dense = dense or ratio >= 1.0
        self.n_keep = self.F if self.dense else B.sl_keep_count(ratio, self.F)
        dev = lambda t: t.to(device=device, dtype=bf).contiguous()
        self.Wg, self.Wu, self.Wd = dev(gate.W), dev(up.W), dev(down.W)
        self.est_dtype = torch.float32 if gate.W_A.dtype == torch.float32 else bf
        ed = lambda t: t.to(device=device, dtype=self.est_dtype).contiguous()
        self.WAg, self.WBg, self.WAu, self.WBu = ed(gate.W_A), ed(gate.W_B), ed(up.W_A), ed(up.W_B)
        r_, D_, F_ = lora_gate[0].shape[0], gate.W.shape[1], gate.W.shape[0]
        # LoRA matrices in the order and layout of the gradient buffer (A_d, B_d, A_g, B_g, A_u, B_u)
        self.params = _GradBuffer([(r_, F_), (D_, r_), (r_, D_), (F_, r_), (r_, D_), (F_, r_)], device, torch.bfloat16,
                                  init=[lora_down[0], lora_down[1], lora_gate[0], lora_gate[1], lora_up[0],
                                        lora_up[1]])
        self.Ad, self.Bd, self.Ag, self.Bg, self.Au, self.Bu = self.params.views
        self.r = self.Ag.shape[0]
        self.scale = float(lora_scale)
        self.Wd_t = _empty((self.F, self.D), bf, device)
        B.sl_prepare_weight(self.Wd, self.Wd_t)
        self.ws = B.Workspace(device)
        self.side = _Side(device)
        self.concurrent = True  # independent chains on a second stream
        T, D, F, r = n_tok, self.D, self.F, self.r
        f32 = torch.float32
        self.scores = _empty((F,), f32, device)
        self.sigma = torch.arange(F, dtype=torch.int32, device=device)
        self.xa_gu, self.xa_s_gu = _empty((T, 2 * r), f32, device), _empty((T, 2 * r), bf, device)
        self.g, self.u, self.h = (_empty((T, F), bf, device) for _ in range(3))
        self.xa_d, self.xa_s_d = _empty((T, r), f32, device), _empty((T, r), bf, device)
        self.y = _empty((T, D), bf, device)
        self.dya_d, self.dya_s_d = _empty((T, r), f32, device), _empty((T, r), bf, device)
        self.dg, self.du = _empty((T, F), bf, device), _empty((T, F), bf, device)
        self.dya_g, self.dya_s_g = _empty((T, r), f32, device), _empty((T, r), bf, device)
        self.dya_u, self.dya_s_u = _empty((T, r), f32, device), _empty((T, r), bf, device)
        self.grads = _GradBuffer([(r, F), (D, r), (r, D), (F, r), (r, D), (F, r)], device)
        self.dA_d, self.dB_d, self.dA_g, self.dB_g, self.dA_u, self.dB_u = self.grads.views
        self.dp = dp if dp is not None and dp.active else None
        self.est_part = _empty((F,), torch.float64, device) if self.dp else None
        self.dx = _empty((T, D), bf, device)
        # the estimator's stage 1 inside the gate/up x A^T launch (one pass over x): single rank,
        # the method's criterion, bf16 factors
        self.fold = (criterion == "svd" and self.dp is None and self.est_dtype == bf and self.k in (4, 8, 16)
                     and n_ctx > 0 and not self.dense)
        if self.fold:
            self.WAt = _empty((2 * self.k, D), bf, device)  # [W_A(gate)^T; W_A(up)^T]
            B.sl_prepare_weight(self.WAg, self.WAt[: self.k])
            B.sl_prepare_weight(self.WAu, self.WAt[self.k:])
            self.z = _empty((n_ctx, 2 * self.k), f32, device)
        # kept rows of the sliced weights: read in place by the GEMM (None), or a compacted copy
        # rebuilt once per step and shared by the forward and backward calls (the weights
        # themselves when nothing is dropped)
        if self.dense:
            self.Wg_k, self.Wu_k, self.Wd_k = self.Wg, self.Wu, self.Wd_t
        elif kept_rows == "gather":
            self.Wg_k = self.Wu_k = self.Wd_k = None
        else:
            nk = self.n_keep
            self.Wg_k, self.Wu_k, self.Wd_k = (_empty((nk, D), bf, device) for _ in range(3))
        self._descs()

    def _descs(self):
        s = self.scale
        lin = lambda wk_g, wk_u, wk_d: (
            B.linear_desc(self.Wg, self.Ag, self.Bg, s, B.SL_SLICE_OUT, w_kept=wk_g),
            B.linear_desc(self.Wu, self.Au, self.Bu, s, B.SL_SLICE_OUT, w_kept=wk_u),
            B.linear_desc(self.Wd, self.Ad, self.Bd, s, B.SL_SLICE_IN, w_t=self.Wd_t, w_kept=wk_d))
        self._sparse = lin(self.Wg_k, self.Wu_k, self.Wd_k) + (B.channels_desc(self.sigma, self.n_keep),)
        self._sigma_id = torch.arange(self.F, dtype=torch.int32, device=self.device)
        self._dense = lin(self.Wg, self.Wu, self.Wd_t) + (B.channels_desc(self._sigma_id, self.F),)
        self._always_dense = self.dense
        self.lin_g, self.lin_u, self.lin_d, self.ch = self._dense if self.dense else self._sparse

    def set_dense(self, on: bool):
        """Run the next steps densely (the progressive schedule's first steps, [WT] "Step
        Sensitivity and Progressive Sparse Fine-Tuning") or back with the block's keep ratio."""
        self.dense = bool(on) or self._always_dense
        self.lin_g, self.lin_u, self.lin_d, self.ch = self._dense if self.dense else self._sparse

    def estimate(self, x):
        """a1 + a2: SwiGLU-L2 scores of the estimated gate/up outputs on x's context rows (or
        the ablation criterion's scores)."""
        if self.criterion == "wanda":
            B.sl_wanda_scores(self.ws, x[: self.n_ctx], self.n_ctx, [self.Wg, self.Wu], self.scores)
            return
        if self.criterion == "random":
            self.scores.uniform_(generator=self.rng)
            return
        xe = x if self.est_dtype == torch.bfloat16 else self.x_est
        if self.dp:  # statistics of this rank's context rows, summed over the ranks
            B.sl_svd_estimate_partials(self.ws, B.SL_CRIT_SWIGLU_L2, xe[: self.n_ctx], self.n_ctx,
                                       [self.WAg, self.WAu], [self.WBg, self.WBu], self.k, self.est_part)
            self.dp.all_reduce(self.est_part)
            B.sl_svd_scores_from_partials(B.SL_CRIT_SWIGLU_L2, [self.WBg, self.WBu], self.k, self.est_part,
                                          self.scores)
            return
        B.sl_svd_estimate(self.ws, B.SL_CRIT_SWIGLU_L2, xe[: self.n_ctx], self.n_ctx, [self.WAg, self.WAu],
                          [self.WBg, self.WBu], self.k, self.scores)

    def choose(self):
        """a3: the kept channel set (self.sigma) from self.scores."""
        B.sl_select_channels(self.scores, self.n_keep, self.sigma)

    def compact(self):
        """The kept weight rows of gate, up (rows of W) and down (rows of W^T) for this step
        (nothing to do when the GEMM gathers them)."""
        if self.Wg_k is None or self.dense:
            return
        kept = self.sigma[: self.n_keep]
        B.sl_gather_rows_batch([self.Wg, self.Wu, self.Wd_t], [kept] * 3, [self.Wg_k, self.Wu_k, self.Wd_k])

    def _compact_gu(self):
        if self.Wg_k is not None:
            kept = self.sigma[: self.n_keep]
            B.sl_gather_rows_batch([self.Wg, self.Wu], [kept] * 2, [self.Wg_k, self.Wu_k])

    def _compact_d(self):
        """The down projection's kept rows, on the second stream when the block runs chains
        concurrently (needed only by the down product); True when it forked."""
        if self.Wd_k is None:
            return False
        kept = self.sigma[: self.n_keep]
        if self.concurrent:
            with self.side.fork():
                B.sl_permute_rows(self.Wd_t, kept, self.Wd_k)
            return True
        B.sl_permute_rows(self.Wd_t, kept, self.Wd_k)
        return False

    def select(self, x):
        """a1 + a2 + a3 on the context rows of x, then the kept weight rows."""
        self.estimate(x)
        self.choose()
        self.compact()

    def forward(self, x, x_est=None):
        """x: bf16 [n_tok, D] context-first. x_est: optional fp32 copy for an fp32 estimator."""
        self.x = x
        self.x_est = x_est
        C = self.n_ctx
        lay = B.SL_LAYOUT_NATURAL if self.dense else B.SL_LAYOUT_SIGMA
        # no context rows: nothing to score, every row is dense (data-parallel ranks still take
        # part in the selection of the batch)
        down_side = False
        if not self.dense and self.fold and x_est is None:
            # x A^T of gate/up and the estimator's Z from one pass over x, then the criterion
            # from Z, the selection and the kept rows (down's on the second stream)
            B.sl_lora_fwd_estimate(self.ws, [self.lin_g, self.lin_u], x, C, self.xa_s_gu, self.xa_gu, 2, self.k,
                                   self.WAt, self.z)
            B.sl_svd_scores_from_z(self.ws, B.SL_CRIT_SWIGLU_L2, [self.WBg, self.WBu], self.k, self.z, C,
                                   self.scores)
            self.choose()
            self._compact_gu()
            down_side = self._compact_d()
        elif not self.dense and (C > 0 or self.dp):
            if self.concurrent:  # x A^T of gate/up does not depend on the selection
                with self.side.fork():
                    B.sl_lora_fwd_bwd(self.side.ws, B.SL_LORA_FWD, [self.lin_g, self.lin_u], x, C, self.xa_s_gu,
                                      xa=self.xa_gu)
                lora_done = self.side.mark()
                self.estimate(x)
                self.choose()
                self._compact_gu()
                down_side = self._compact_d()
                torch.cuda.current_stream().wait_event(lora_done)
            else:
                self.select(x)
                B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_FWD, [self.lin_g, self.lin_u], x, C, self.xa_s_gu,
                                  xa=self.xa_gu)
        else:
            B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_FWD, [self.lin_g, self.lin_u], x, C, self.xa_s_gu, xa=self.xa_gu)
        B.sl_sparse_linear_fwd(self.ws, [self.lin_g, self.lin_u], [self.ch], B.SL_EPI_SWIGLU, x, C, self.xa_s_gu,
                               [self.g, self.u, self.h], out_layout=B.SL_LAYOUT_SIGMA)
        if down_side:
            self.side.join()
        B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_FWD, [self.lin_d], self.h, C, self.xa_s_d, xa=self.xa_d,
                          in_layout=lay, in_ch=self.ch)
        B.sl_sparse_linear_fwd(self.ws, [self.lin_d], [self.ch], B.SL_EPI_NONE, self.h, C, self.xa_s_d, [self.y],
                               in_layout=B.SL_LAYOUT_SIGMA)
        return self.y

    def backward(self, dy):
        C = self.n_ctx
        lay = B.SL_LAYOUT_NATURAL if self.dense else B.SL_LAYOUT_SIGMA
        B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_BWD, [self.lin_d], self.h, C, self.xa_s_d, in_layout=lay,
                          in_ch=self.ch, dy=[dy], dya=[self.dya_d], dya_s=[self.dya_s_d], dA=[self.dA_d],
                          dB=[self.dB_d])
        B.sl_sparse_linear_bwd(self.ws, [self.lin_d], [self.ch], B.SL_EPI_SWIGLU, [dy], C, [self.dya_s_d],
                               aux=[self.g, self.u], aux_out=[self.dg, self.du], out_layout=B.SL_LAYOUT_SIGMA)
        B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_BWD, [self.lin_g, self.lin_u], self.x, C, self.xa_s_gu,
                          dy=[self.dg, self.du], out_layout=lay, out_ch=[self.ch, self.ch],
                          dya=[self.dya_g, self.dya_u], dya_s=[self.dya_s_g, self.dya_s_u],
                          dA=[self.dA_g, self.dA_u], dB=[self.dB_g, self.dB_u])
        B.sl_sparse_linear_bwd(self.ws, [self.lin_g, self.lin_u], [self.ch, self.ch], B.SL_EPI_NONE,
                               [self.dg, self.du], C, [self.dya_s_g, self.dya_s_u], dx=self.dx,
                               in_layout=B.SL_LAYOUT_SIGMA)
        return self.dx

    def read_device_flag(self) -> int:
        """Device error word of both workspaces (0: no device-side timeout); synchronises."""
        return self.ws.read_device_flag() or self.side.ws.read_device_flag()

    def step(self, x, dy, x_est=None):
        self.forward(x, x_est)
        dx = self.backward(dy)
        if self.dp:
            self.dp.all_reduce(self.grads.flat)
        return dx


class AttnProjBlock:
    """q, k, v (output channels sliced) and o (input channels sliced). QK criterion over
    KV units for q/k, L2 criterion on the estimated V for v/o. The attention core is not
    part of the path: its output x_o and its gradients dq, dk, dv are inputs."""

    def __init__(self, q, k, v, o, lora_q, lora_k, lora_v, lora_o, lora_scale, est_k, n_q_heads, n_kv_heads,
                 head_dim, n_tok, n_ctx, ratio, device="cuda", dense=False, dp=None, qk_criterion="channel",
                 vo_criterion="l2", seed=0, kept_rows="compact", io_layout="natural"):
        """qk_criterion: "channel" (the method's QK norm per KV channel), or the criterion
        ablation's "head" (whole KV heads by the summed QK norm) and "random"; vo_criterion:
        "l2" (the method's) or "random" (uniform scores from a generator seeded with `seed`).
        kept_rows: "compact" (a compacted copy per step, shared by forward and backward; the
        faster form on B200) or "gather" (the sliced products read the kept weight rows in place
        through sigma). io_layout: the channel order of the context rows of q, k, v (outputs),
        x_o (input), dx_o (output) and dq, dk, dv (inputs): "natural", or "sigma" (channel
        sigma[p] in column p, the order the sliced products read and write, so no column scatter
        or gather runs; sl_permute_rows_sigma converts while it reorders the rows, as the decoder
        layer does)."""
        if qk_criterion not in ("channel", "head", "random") or vo_criterion not in ("l2", "random"):
            raise ValueError(f"criteria {qk_criterion!r}, {vo_criterion!r}")
        if kept_rows not in KEPT_ROWS:
            raise ValueError(f"kept_rows {kept_rows!r} not in {KEPT_ROWS}")
        if io_layout not in ("natural", "sigma"):
            raise ValueError(f"io_layout {io_layout!r}")
        self.kept_rows = kept_rows
        self.io_layout = io_layout
        self.lay = B.SL_LAYOUT_SIGMA if io_layout == "sigma" else B.SL_LAYOUT_NATURAL
        if (qk_criterion, vo_criterion) != ("channel", "l2") and dp is not None and dp.active:
            raise ValueError("the ablation criteria run on one rank")
        self.qk_criterion, self.vo_criterion = qk_criterion, vo_criterion
        self.rng = torch.Generator(device=device)
        self.rng.manual_seed(int(seed))
        bf, f32 = torch.bfloat16, torch.float32
        dev = lambda t: t.to(device=device, dtype=bf).contiguous()
        self.device = device
        self.D = q.W.shape[1]
        self.hq, self.hkv, self.hd = n_q_heads, n_kv_heads, head_dim
        self.hpg = n_q_heads // n_kv_heads
        self.Dq, self.Dkv = n_q_heads * head_dim, n_kv_heads * head_dim
        self.k = est_k
        self.n_tok, self.n_ctx = n_tok, n_ctx
        self.dense = dense or ratio >= 1.0
        self.n_units = self.Dkv
        self.n_keep_u = self.n_units if self.dense else B.sl_keep_count(ratio, self.n_units)
        # kept KV units of q/k (whole heads for the head-level criterion) and of v/o
        self.n_keep_heads = self.hkv if self.dense else B.sl_keep_count(ratio, self.hkv)
        self.n_keep_qk = self.n_keep_heads * head_dim if qk_criterion == "head" else self.n_keep_u
        self.n_keep_vo = self.n_keep_u
        self.Wq, self.Wk, self.Wv, self.Wo = dev(q.W), dev(k.W), dev(v.W), dev(o.W)
        self.WA = [dev(q.W_A), dev(k.W_A), dev(v.W_A)]
        self.WB = [dev(q.W_B), dev(k.W_B), dev(v.W_B)]
        loras = dict(zip("qkvo", (lora_q, lora_k, lora_v, lora_o)))
        # LoRA matrices in the order and layout of the gradient buffer (A_q..A_o, then B_q..B_o)
        self.params = _GradBuffer([tuple(loras[n][0].shape) for n in "qkvo"] + [tuple(loras[n][1].shape) for n in "qkvo"],
                                  device, torch.bfloat16, init=[loras[n][0] for n in "qkvo"] + [loras[n][1] for n in "qkvo"])
        self.L = {n: (self.params.views[i], self.params.views[4 + i]) for i, n in enumerate("qkvo")}
        self.r = self.L["q"][0].shape[0]
        self.scale = float(lora_scale)
        self.Wo_t = _empty((self.Dq, self.D), bf, device)
        B.sl_prepare_weight(self.Wo, self.Wo_t)
        self.ws = B.Workspace(device)
        self.side = _Side(device)
        self.concurrent = True  # independent chains on a second stream
        T, D, r = n_tok, self.D, self.r
        self.s_qk, self.s_v = _empty((self.n_units,), f32, device), _empty((self.n_units,), f32, device)
        ar = lambda n: torch.arange(n, dtype=torch.int32, device=device)
        self.sig_k, self.sig_q = ar(self.Dkv), ar(self.Dq)
        self.sig_v, self.sig_o = ar(self.Dkv), ar(self.Dq)
        self.xa_qkv, self.xa_s_qkv = _empty((T, 3 * r), f32, device), _empty((T, 3 * r), bf, device)
        self.q, self.kk, self.vv = _empty((T, self.Dq), bf, device), _empty((T, self.Dkv), bf, device), \
            _empty((T, self.Dkv), bf, device)
        self.xa_o, self.xa_s_o = _empty((T, r), f32, device), _empty((T, r), bf, device)
        self.y = _empty((T, D), bf, device)
        self.dya = {n: (_empty((T, r), f32, device), _empty((T, r), bf, device)) for n in "qkvo"}
        d_ins = {"q": D, "k": D, "v": D, "o": self.Dq}
        d_outs = {"q": self.Dq, "k": self.Dkv, "v": self.Dkv, "o": D}
        self.grads = _GradBuffer([(r, d_ins[n]) for n in "qkvo"] + [(d_outs[n], r) for n in "qkvo"], device)
        self.dA = dict(zip("qkvo", self.grads.views[:4]))
        self.dB = dict(zip("qkvo", self.grads.views[4:]))
        self.dp = dp if dp is not None and dp.active else None
        self.est_part = _empty((B.sl_svd_partials_count(B.SL_CRIT_QK, self.WB, self.k),), torch.float64,
                               device) if self.dp else None
        self.dx_o = _empty((T, self.Dq), bf, device)
        self.dx = _empty((T, D), bf, device)
        # the estimator's stage 1 inside the q/k/v x A^T launch (one pass over x): single rank, the
        # method's criteria, factor widths the fused product takes
        self.fold = ((qk_criterion, vo_criterion) == ("channel", "l2") and self.dp is None and est_k % 4 == 0
                     and 3 * est_k <= 64 and n_ctx > 0 and not self.dense)
        if self.fold:
            self.WAt = _empty((3 * est_k, D), bf, device)  # [W_A(q)^T; W_A(k)^T; W_A(v)^T]
            for j in range(3):
                B.sl_prepare_weight(self.WA[j], self.WAt[j * est_k:(j + 1) * est_k])
            self.z = _empty((n_ctx, 3 * est_k), f32, device)
        s = self.scale
        # kept rows of the sliced weights (rows of W for q, k, v; rows of W^T for o): read in
        # place by the GEMM (None), or a copy rebuilt once per step after the selection and
        # shared by the forward and backward calls
        nq, nu = self.n_keep_qk * self.hpg, self.n_keep_qk
        nv, no = self.n_keep_vo, self.n_keep_vo * self.hpg
        if self.dense:
            self.W_k = {"q": self.Wq, "k": self.Wk, "v": self.Wv, "o": self.Wo_t}
        elif kept_rows == "gather":
            self.W_k = {n: None for n in "qkvo"}
        else:
            self.W_k = {"q": _empty((nq, D), bf, device), "k": _empty((nu, D), bf, device),
                        "v": _empty((nv, D), bf, device), "o": _empty((no, D), bf, device)}
        lin = lambda wk: {
            "q": B.linear_desc(self.Wq, *self.L["q"], s, B.SL_SLICE_OUT, w_kept=wk["q"]),
            "k": B.linear_desc(self.Wk, *self.L["k"], s, B.SL_SLICE_OUT, w_kept=wk["k"]),
            "v": B.linear_desc(self.Wv, *self.L["v"], s, B.SL_SLICE_OUT, w_kept=wk["v"]),
            "o": B.linear_desc(self.Wo, *self.L["o"], s, B.SL_SLICE_IN, w_t=self.Wo_t, w_kept=wk["o"]),
        }
        self._lin_sparse = lin(self.W_k)
        self._ch_sparse = {
            "q": B.channels_desc(self.sig_q, self.n_keep_qk * self.hpg),
            "k": B.channels_desc(self.sig_k, self.n_keep_qk),
            "v": B.channels_desc(self.sig_v, self.n_keep_vo),
            "o": B.channels_desc(self.sig_o, self.n_keep_vo * self.hpg),
        }
        self._ids = {"q": ar(self.Dq), "kv": ar(self.Dkv)}
        self._lin_dense = lin({"q": self.Wq, "k": self.Wk, "v": self.Wv, "o": self.Wo_t})
        self._ch_dense = {"q": B.channels_desc(self._ids["q"], self.Dq), "k": B.channels_desc(self._ids["kv"], self.Dkv),
                          "v": B.channels_desc(self._ids["kv"], self.Dkv), "o": B.channels_desc(self._ids["q"], self.Dq)}
        self._always_dense = self.dense
        self.lin, self.ch = (self._lin_dense, self._ch_dense) if self.dense else (self._lin_sparse, self._ch_sparse)

    def estimate(self, x):
        """a1 + a2: QK scores over KV units and V scores from one pass over x's context rows
        (random scores replace them for the ablation's random criteria)."""
        C = self.n_ctx
        if self.qk_criterion == "random" or self.vo_criterion == "random":
            if (self.qk_criterion, self.vo_criterion) != ("random", "random"):
                B.sl_svd_estimate(self.ws, B.SL_CRIT_QK, x[:C], C, self.WA, self.WB, self.k, self.s_qk,
                                  scores_v=self.s_v, n_q_heads=self.hq, n_kv_heads=self.hkv, head_dim=self.hd)
            if self.qk_criterion == "random":
                self.s_qk.uniform_(generator=self.rng)
            if self.vo_criterion == "random":
                self.s_v.uniform_(generator=self.rng)
            return
        if self.dp:  # Gram matrix of this rank's Z, summed over the ranks
            B.sl_svd_estimate_partials(self.ws, B.SL_CRIT_QK, x[:C], C, self.WA, self.WB, self.k, self.est_part,
                                       n_q_heads=self.hq, n_kv_heads=self.hkv, head_dim=self.hd)
            self.dp.all_reduce(self.est_part)
            B.sl_svd_scores_from_partials(B.SL_CRIT_QK, self.WB, self.k, self.est_part, self.s_qk, scores_v=self.s_v,
                                          n_q_heads=self.hq, n_kv_heads=self.hkv, head_dim=self.hd)
            return
        B.sl_svd_estimate(self.ws, B.SL_CRIT_QK, x[:C], C, self.WA, self.WB, self.k, self.s_qk, scores_v=self.s_v,
                          n_q_heads=self.hq, n_kv_heads=self.hkv, head_dim=self.hd)

    def _estimate_fused(self, x, ws):
        """x A^T of q, k, v together with the estimator's Z (one pass over x), then the QK and V
        scores from Z."""
        C = self.n_ctx
        lq, lk, lv = (self.lin[n] for n in "qkv")
        B.sl_lora_fwd_estimate(ws, [lq, lk, lv], x, C, self.xa_s_qkv, self.xa_qkv, 3, self.k, self.WAt, self.z)
        B.sl_svd_scores_from_z(ws, B.SL_CRIT_QK, self.WB, self.k, self.z, C, self.s_qk, scores_v=self.s_v,
                               n_q_heads=self.hq, n_kv_heads=self.hkv, head_dim=self.hd)

    def _choose_and_compact(self):
        """The q/k and v/o selections with their kept weight rows: two independent chains (the
        v/o one on the second stream when concurrent)."""
        if self.concurrent:
            with self.side.fork():
                self._vo_chain()
            self._qk_chain()
            self.side.join()
        else:
            self.choose()
            self.compact()

    def _select_qk(self):
        if self.qk_criterion == "head":
            B.sl_select_heads(self.s_qk, self.hkv, self.hd, self.n_keep_heads, self.sig_k, self.hpg, self.sig_q)
        else:
            B.sl_select_channels(self.s_qk, self.n_keep_qk, self.sig_k, self.hpg, self.hd, self.sig_q)

    def _select_vo(self):
        B.sl_select_channels(self.s_v, self.n_keep_vo, self.sig_v, self.hpg, self.hd, self.sig_o)

    def set_dense(self, on: bool):
        """Run the next steps densely (the progressive schedule's first steps) or back with the
        block's keep ratios."""
        self.dense = bool(on) or self._always_dense
        self.lin, self.ch = (self._lin_dense, self._ch_dense) if self.dense else (self._lin_sparse, self._ch_sparse)

    def _kept_rows(self, names):
        """The kept weight rows of the named projections (rows of W; for o, rows of W^T), one
        launch; nothing when the GEMM gathers them."""
        if self.W_k[names[0]] is None or self.dense:
            return
        src = {"q": (self.Wq, self.sig_q), "k": (self.Wk, self.sig_k), "v": (self.Wv, self.sig_v),
               "o": (self.Wo_t, self.sig_o)}
        B.sl_gather_rows_batch([src[n][0] for n in names], [src[n][1][: self.ch[n].n_keep] for n in names],
                               [self.W_k[n] for n in names])

    def _qk_chain(self):
        self._select_qk()
        self._kept_rows("qk")

    def _vo_chain(self):
        self._select_vo()
        self._kept_rows("vo")

    def choose(self):
        """a3: the q/k set from the QK scores and the v/o set from the V scores."""
        self._select_qk()
        self._select_vo()

    def compact(self):
        """The kept weight rows of q, k, v (rows of W) and o (rows of W^T) for this step."""
        self._kept_rows("qkvo")

    def select(self, x):
        """a1 + a2, then the q/k and v/o selections with their kept weight rows: two
        independent chains (the v/o one on the second stream when concurrent)."""
        self.estimate(x)
        if self.concurrent:
            with self.side.fork():
                self._vo_chain()
            self._qk_chain()
            self.side.join()
        else:
            self.choose()
            self.compact()

    def forward(self, x, x_o):
        C = self.n_ctx
        self.x, self.x_o = x, x_o
        lq, lk, lv, lo = (self.lin[n] for n in "qkvo")
        sel = not self.dense and (C > 0 or self.dp is not None)

        def o_lora(ws):
            B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lo], x_o, C, self.xa_s_o, xa=self.xa_o, in_layout=self.lay,
                              in_ch=self.ch["o"])

        # x_o A^T does not depend on the selection in the natural layout; in the sigma layout x_o's
        # context columns follow the v/o set, so it runs after the selection (beside the q/k/v
        # products when the block runs chains concurrently)
        early_o = self.lay == B.SL_LAYOUT_NATURAL or not sel

        def qkv_lora(ws):
            B.sl_lora_fwd_bwd(ws, B.SL_LORA_FWD, [lq, lk, lv], x, C, self.xa_s_qkv, xa=self.xa_qkv)

        if sel and self.fold:
            if self.concurrent and early_o:
                with self.side.fork():
                    o_lora(self.side.ws)
                o_done = self.side.mark()
                self._estimate_fused(x, self.ws)
                self._choose_and_compact()
                torch.cuda.current_stream().wait_event(o_done)
            else:
                if early_o:
                    o_lora(self.ws)
                self._estimate_fused(x, self.ws)
                self._choose_and_compact()
        elif sel and self.concurrent:
            with self.side.fork():
                qkv_lora(self.side.ws)
                if early_o:
                    o_lora(self.side.ws)
            self.select(x)
            self.side.join()
        else:
            if sel:
                self.select(x)
            qkv_lora(self.ws)
            if early_o:
                o_lora(self.ws)
        late_side = not early_o and self.concurrent
        if late_side:
            with self.side.fork():
                o_lora(self.side.ws)
        elif not early_o:
            o_lora(self.ws)
        B.sl_sparse_linear_fwd(self.ws, [lq, lk, lv], [self.ch[n] for n in "qkv"], B.SL_EPI_NONE, x, C,
                               self.xa_s_qkv, [self.q, self.kk, self.vv], out_layout=self.lay)
        if late_side:
            self.side.join()
        B.sl_sparse_linear_fwd(self.ws, [lo], [self.ch["o"]], B.SL_EPI_NONE, x_o, C, self.xa_s_o, [self.y],
                               in_layout=self.lay)
        return self.y

    def _o_backward(self, ws, dy):
        """o's LoRA gradients and its input gradient dx_o."""
        lo = self.lin["o"]
        C = self.n_ctx
        B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lo], self.x_o, C, self.xa_s_o, in_layout=self.lay, in_ch=self.ch["o"],
                          dy=[dy], dya=[self.dya["o"][0]], dya_s=[self.dya["o"][1]], dA=[self.dA["o"]],
                          dB=[self.dB["o"]])
        B.sl_sparse_linear_bwd(ws, [lo], [self.ch["o"]], B.SL_EPI_NONE, [dy], C, [self.dya["o"][1]],
                               dx=self.dx_o, out_layout=self.lay)

    def _qkv_backward(self, ws, dq, dk, dv):
        """q, k, v LoRA gradients and dx."""
        lq, lk, lv = (self.lin[n] for n in "qkv")
        C = self.n_ctx
        B.sl_lora_fwd_bwd(ws, B.SL_LORA_BWD, [lq, lk, lv], self.x, C, self.xa_s_qkv, dy=[dq, dk, dv],
                          out_layout=self.lay, out_ch=[self.ch[n] for n in "qkv"],
                          dya=[self.dya[n][0] for n in "qkv"], dya_s=[self.dya[n][1] for n in "qkv"],
                          dA=[self.dA[n] for n in "qkv"], dB=[self.dB[n] for n in "qkv"])
        B.sl_sparse_linear_bwd(ws, [lq, lk, lv], [self.ch[n] for n in "qkv"], B.SL_EPI_NONE, [dq, dk, dv], C,
                               [self.dya[n][1] for n in "qkv"], dx=self.dx, in_layout=self.lay)

    def backward(self, dy, dq, dk, dv):
        if self.concurrent:  # the o chain and the q/k/v chain are independent
            with self.side.fork():
                self._o_backward(self.side.ws, dy)
            self._qkv_backward(self.ws, dq, dk, dv)
            self.side.join()
        else:
            self._o_backward(self.ws, dy)
            self._qkv_backward(self.ws, dq, dk, dv)
        return self.dx, self.dx_o

    # ---- the same step in the order of a decoder layer, where the attention core sits between
    # q/k/v and o: forward_qkv, forward_o, then backward_o, backward_qkv

    def forward_qkv(self, x):
        """The selection on x's context rows and q, k, v (context rows in the block's io_layout)."""
        C = self.n_ctx
        self.x = x
        lq, lk, lv = (self.lin[n] for n in "qkv")
        sel = not self.dense and (C > 0 or self.dp is not None)
        if sel and self.fold:
            self._estimate_fused(x, self.ws)
            self._choose_and_compact()
        elif sel and self.concurrent:
            with self.side.fork():
                B.sl_lora_fwd_bwd(self.side.ws, B.SL_LORA_FWD, [lq, lk, lv], x, C, self.xa_s_qkv, xa=self.xa_qkv)
            self.select(x)
            self.side.join()
        else:
            if sel:
                self.select(x)
            B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_FWD, [lq, lk, lv], x, C, self.xa_s_qkv, xa=self.xa_qkv)
        B.sl_sparse_linear_fwd(self.ws, [lq, lk, lv], [self.ch[n] for n in "qkv"], B.SL_EPI_NONE, x, C,
                               self.xa_s_qkv, [self.q, self.kk, self.vv], out_layout=self.lay)
        return self.q, self.kk, self.vv

    def forward_o(self, x_o):
        """o of the attention output x_o (its input channels sliced by the v/o selection)."""
        C = self.n_ctx
        self.x_o = x_o
        lo = self.lin["o"]
        B.sl_lora_fwd_bwd(self.ws, B.SL_LORA_FWD, [lo], x_o, C, self.xa_s_o, xa=self.xa_o, in_layout=self.lay,
                          in_ch=self.ch["o"])
        B.sl_sparse_linear_fwd(self.ws, [lo], [self.ch["o"]], B.SL_EPI_NONE, x_o, C, self.xa_s_o, [self.y],
                               in_layout=self.lay)
        return self.y

    def backward_o(self, dy):
        self._o_backward(self.ws, dy)
        return self.dx_o

    def backward_qkv(self, dq, dk, dv):
        self._qkv_backward(self.ws, dq, dk, dv)
        return self.dx

    def sigma_of(self, name):
        """The channel set in force for projection `name` ("q", "k", "v", "o"): its sigma tensor
        (the identity in dense steps)."""
        if self.dense:
            return self._ids["q" if name in "qo" else "kv"]
        return {"q": self.sig_q, "k": self.sig_k, "v": self.sig_v, "o": self.sig_o}[name]

    def read_device_flag(self) -> int:
        """Device error word of both workspaces (0: no device-side timeout); synchronises."""
        return self.ws.read_device_flag() or self.side.ws.read_device_flag()

    def step(self, x, x_o, dy, dq, dk, dv):
        self.forward(x, x_o)
        dx = self.backward(dy, dq, dk, dv)
        if self.dp:
            self.dp.all_reduce(self.grads.flat)
        return dx
