"""One LLaMA-style decoder layer around the sparse projections, forward and backward
([WT] "Putting It All Together": the sparse q/k/v/o and FFN projections inside the model's
layers; the per-layer context/output split, so output rows attend to context keys and values
computed with the sparse projections).

    h1 = RMSNorm(x, g1); q, k, v = sparse projections of h1; a = causal GQA attention(q, k, v)
    x2 = x + o(a); h2 = RMSNorm(x2, g2); y = x2 + FFN(h2)

RMSNorm, the residual adds, every projection and the causal grouped-query attention core
(sl_attention_fwd / sl_attention_bwd, tcgen05 kernels) run in libsparselora's kernels. Rows are
in context-first order like the blocks' (sl_permute_rows moves q, k, v to sequence order for the
attention core and its output back; when the attention block keeps its interfaces in the sigma
layout, sl_permute_rows_sigma also restores or applies the channel order of the context rows in
the same pass). No rotary positional encoding: the pages do not say how it
meets channel sparsity (a rotation mixes channel pairs that the selection may split)."""
from __future__ import annotations

import torch

from . import binding as B
from .blocks import AttnProjBlock, FFNBlock


class DecoderLayer:
    def __init__(self, attn: AttnProjBlock, ffn: FFNBlock, gamma1, gamma2, perm, n_seq: int, eps: float = 1e-5):
        """attn, ffn: the layer's projection blocks (same n_tok and n_ctx); gamma1, gamma2: frozen
        RMSNorm gains [D]; perm: int64 [n_tok], context-first position p holds sequence-order row
        perm[p] (rows of n_seq sequences of equal length)."""
        dev = attn.device
        self.attn, self.ffn = attn, ffn
        self.g1 = gamma1.to(device=dev, dtype=torch.bfloat16).contiguous()
        self.g2 = gamma2.to(device=dev, dtype=torch.bfloat16).contiguous()
        self.eps = float(eps)
        self.n_seq = int(n_seq)
        T, D = attn.n_tok, attn.D
        self.T, self.D = T, D
        self.S = T // self.n_seq
        perm = torch.as_tensor(perm, dtype=torch.int64, device=dev)
        inv = torch.empty_like(perm)
        inv[perm] = torch.arange(T, device=dev)
        self.perm = perm.to(torch.int32).contiguous()  # sequence-order row of each context-first row
        self.inv = inv.to(torch.int32).contiguous()    # context-first row of each sequence-order row
        bf, f32 = torch.bfloat16, torch.float32
        e = lambda *sh, dt=bf: torch.empty(*sh, dtype=dt, device=dev)
        self.h1, self.x2, self.h2, self.y = e(T, D), e(T, D), e(T, D), e(T, D)
        self.rstd1, self.rstd2 = e(T, dt=f32), e(T, dt=f32)
        Dq, Dkv = attn.Dq, attn.Dkv
        self.q_nat, self.k_nat, self.v_nat = e(T, Dq), e(T, Dkv), e(T, Dkv)
        self.a_nat, self.a_cf = e(T, Dq), e(T, Dq)
        self.lse = e(attn.hq, T, dt=f32)
        self.da_nat = e(T, Dq)
        self.dq_nat, self.dk_nat, self.dv_nat = e(T, Dq), e(T, Dkv), e(T, Dkv)
        self.dq_cf, self.dk_cf, self.dv_cf = e(T, Dq), e(T, Dkv), e(T, Dkv)
        self.dx2, self.dx = e(T, D), e(T, D)
        self.ws = B.Workspace(dev)  # the attention core's scratch (the dq accumulator) and error word

    def _to_seq(self, src, dst, name):
        """Context-first rows -> sequence order; with the block's sigma layout, the context rows'
        channels also return to natural order (projection `name`'s channel set)."""
        at = self.attn
        if at.io_layout == "sigma":
            B.sl_permute_rows_sigma(src, self.inv, dst, at.sigma_of(name), at.n_ctx, to_sigma=False)
        else:
            B.sl_permute_rows(src, self.inv, dst)

    def _to_cf(self, src, dst, name):
        """Sequence order -> context-first rows (in the block's sigma layout when it uses one)."""
        at = self.attn
        if at.io_layout == "sigma":
            B.sl_permute_rows_sigma(src, self.perm, dst, at.sigma_of(name), at.n_ctx, to_sigma=True)
        else:
            B.sl_permute_rows(src, self.perm, dst)

    def forward(self, x):
        at = self.attn
        B.sl_rmsnorm_fwd(x, self.g1, self.eps, self.h1, self.rstd1)
        q, k, v = at.forward_qkv(self.h1)
        for src, dst, name in ((q, self.q_nat, "q"), (k, self.k_nat, "k"), (v, self.v_nat, "v")):
            self._to_seq(src, dst, name)
        B.sl_attention_fwd(self.ws, self.q_nat, self.k_nat, self.v_nat, self.n_seq, at.hq, at.hkv, at.hd, self.a_nat,
                           self.lse)
        self._to_cf(self.a_nat, self.a_cf, "o")
        o = at.forward_o(self.a_cf)
        # x2 = x + o (the residual stream) and h2 = RMSNorm(x2) in one pass
        B.sl_rmsnorm_fwd(o, self.g2, self.eps, self.h2, self.rstd2, res=x, sum_out=self.x2)
        f = self.ffn.forward(self.h2)
        B.sl_add_rows(self.x2, f, self.y)
        self.x = x
        return self.y

    def backward(self, dy):
        at = self.attn
        dh2 = self.ffn.backward(dy)
        B.sl_rmsnorm_bwd(dh2, self.x2, self.g2, self.rstd2, self.dx2, dres=dy)
        da_cf = at.backward_o(self.dx2)
        self._to_seq(da_cf, self.da_nat, "o")
        B.sl_attention_bwd(self.ws, self.q_nat, self.k_nat, self.v_nat, self.a_nat, self.da_nat, self.lse, self.n_seq,
                           at.hq, at.hkv, at.hd, self.dq_nat, self.dk_nat, self.dv_nat)
        for src, dst, name in ((self.dq_nat, self.dq_cf, "q"), (self.dk_nat, self.dk_cf, "k"),
                               (self.dv_nat, self.dv_cf, "v")):
            self._to_cf(src, dst, name)
        dh1 = at.backward_qkv(self.dq_cf, self.dk_cf, self.dv_cf)
        B.sl_rmsnorm_bwd(dh1, self.x, self.g1, self.rstd1, self.dx, dres=self.dx2)
        return self.dx

    def read_device_flag(self) -> int:
        """Device error word of the attention core's workspace (0: no device-side timeout); synchronises."""
        return self.ws.read_device_flag()

    def step(self, x, dy):
        self.forward(x)
        return self.backward(dy)
