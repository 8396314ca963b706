"""Benchmark: SparseLoRA layer fine-tuning step (forward + backward) tokens/s at LLaMA3-8B shapes.

One step = every stage of the hot path for one LLaMA3-8B decoder layer's seven
projections over one batch of 8 x 512 tokens (last 128 of each sequence are output
tokens): the attention projections q/k/v/o (QK criterion for q/k, L2 criterion on
the estimated V for v/o, GQA 32/8 heads x 128) and the SwiGLU FFN gate/up/down
(L2 criterion on the estimated SiLU(gate) * up), keep ratio 0.5, LoRA rank 32 on
all seven, estimator rank 8. The attention core between q/k/v and o is not part of
the path; its output and gradients are synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sparselora|reference]

Multi-GPU (torchrun, one rank per GPU): each rank runs the step on its own batch
(weak scaling, no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import math
import json
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from contextual_sparsity_lora_b200 import flops, inputs  # noqa: E402

METRIC = "sparse-LoRA layer fwd+bwd tokens/s at LLaMA3-8B shapes"
UNIT = "tokens/s"
WORKLOAD = "llama3-8b-layer-7proj-b8s512-keep0.5"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sparselora", choices=["sparselora", "reference"])
    ap.add_argument("--ratio", type=float, default=0.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-LoRA companion measurement")
    ap.add_argument("--no-layer", action="store_true", help="skip the whole-decoder-layer measurement")
    ap.add_argument("--no-model", action="store_true", help="skip the 32-layer fine-tuning run")
    ap.add_argument("--no-sweep", action="store_true", help="skip the keep-ratio sweep and the LLaMA2-13B layer")
    ap.add_argument("--attention-only", action="store_true",
                    help="time only the causal GQA attention core at the LLaMA3-8B layer's shape and print it")
    ap.add_argument("--stages-only", action="store_true",
                    help="time only the selection stages (estimator, criterion, top-n, compaction) of both blocks "
                         "and print them; no step, no headline line")
    return ap.parse_args()


def dist_setup(n_gpus, cpu_only=False):
    """Process group of a torchrun launch (none for one process). The reference arm runs on the
    host cores only, so it takes gloo even on a GPU machine."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and not cpu_only else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every `interval` seconds while the
    timed region runs, read-only through NVML (nvidia-smi's query loop as the fallback)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, index, interval=0.005):
        self.index = index
        self.interval = interval
        self.samples = []   # (sm_mhz, max_mhz, reasons bitmask)
        self.source = None
        self._stop = threading.Event()
        self.thread = None
        self.proc = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                             int(get_reasons(h))))
                    except Exception:
                        pass
                    self._stop.wait(self.interval)
            self.source = f"NVML every {self.interval * 1e3:.0f} ms"
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        except Exception:
            self._start_smi()
        return self

    def _start_smi(self):
        fields = "clocks.sm,clocks.max.sm,clocks_event_reasons.active"
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={fields}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi -lms 20"

            def read():
                for line in self.proc.stdout:
                    parts = [q.strip() for q in line.split(",")]
                    try:
                        self.samples.append((float(parts[0]), float(parts[1]), int(parts[2], 16)))
                    except Exception:
                        pass
            self.thread = threading.Thread(target=read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def __exit__(self, *a):
        self._stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = sorted(float(x[0]) for x in self.samples)
        reasons = sorted({name for x in self.samples for bit, name in self.REASONS.items() if x[2] & bit})
        return {"sm_mhz": sm[len(sm) // 2], "sm_min_mhz": sm[0], "sm_max_mhz": max(float(x[1]) for x in self.samples),
                "reasons": reasons, "samples": len(self.samples), "source": self.source}


def make_layer(ratio, seed_w, seed_x, device, dense=False, dp=None, cfgs=None, kept_rows="compact"):
    """The two blocks of one layer (LLaMA3-8B unless `cfgs` = (attention config, FFN config))
    plus their per-step inputs (context-first rows). dp: a blocks.DataParallel over the ranks
    (one index set per global batch), or None. kept_rows: where the sliced products read the
    kept weight rows (blocks.KEPT_ROWS)."""
    from contextual_sparsity_lora_b200 import blocks
    ac, fc = cfgs if cfgs else (inputs.LLAMA3_8B_ATTN, inputs.LLAMA3_8B_FFN)
    da = inputs.make_attn_inputs(ac, seed_w, device=device)
    df = inputs.make_ffn_inputs(fc, seed_w + 1, device=device)
    perm = inputs.context_first_order(da["ctx_mask"])
    C = int(da["ctx_mask"].sum())
    attn = blocks.AttnProjBlock(da["q"], da["k"], da["v"], da["o"], da["lora_q"], da["lora_k"], da["lora_v"],
                                da["lora_o"], ac.lora_scale, ac.k, ac.n_q_heads, ac.n_kv_heads, ac.head_dim,
                                ac.n_tok, C, ratio, device, dense=dense, dp=dp, kept_rows=kept_rows, io_layout="sigma")
    ffn = blocks.FFNBlock(df["gate"], df["up"], df["down"], df["lora_gate"], df["lora_up"], df["lora_down"],
                          fc.lora_scale, fc.k, fc.n_tok, C, ratio, device, dense=dense, dp=dp, kept_rows=kept_rows)
    if seed_x != seed_w:  # per-rank batches
        dx = inputs.make_attn_inputs(ac, seed_x, device=device)
        for key in ("x", "x_o", "dq", "dk", "dv", "dy"):
            da[key] = dx[key]
        df["x"], df["dy"] = dx["x"], dx["dy"]
    step_in = {k: da[k][perm].contiguous() for k in ("x", "x_o", "dq", "dk", "dv", "dy")}
    step_in["ffn_x"] = df["x"][perm].contiguous()
    step_in["ffn_dy"] = df["dy"][perm].contiguous()
    return attn, ffn, step_in, C, (ac, fc), (da, df, perm)


def run_step(attn, ffn, s):
    attn.step(s["x"], s["x_o"], s["dy"], s["dq"], s["dk"], s["dv"])
    ffn.step(s["ffn_x"], s["ffn_dy"])


def algorithmic_flops(ac, fc, C, ratio, dense):
    T = ac.n_tok
    nu = ac.n_kv_heads * ac.head_dim
    nk_u = nu if dense else inputs_keep(ratio, nu)
    nk_f = fc.inter if dense else inputs_keep(ratio, fc.inter)
    a = flops.attn_proj_block(ac.hidden, ac.n_q_heads, ac.n_kv_heads, ac.head_dim, T, C, nk_u, nk_u, ac.r, ac.k,
                              with_estimator=not dense)
    f = flops.ffn_block(fc.hidden, fc.inter, T, C, nk_f, fc.r, fc.k, with_estimator=not dense)
    return {k: a[k] + f[k] for k in a}


def inputs_keep(ratio, n):
    from contextual_sparsity_lora_b200 import binding as B
    return B.sl_keep_count(ratio, n)


def capture_graph(fn, warm=True):
    """Capture one call of fn (all library launches on torch's current stream) as a CUDA graph."""
    if warm:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


# DRAM bytes (read + write) of gemm_pair_kernel per launch, the mean over the 8 CTA-pair
# launches of one step of this workload, from an ncu capture of one step's CTA-pair launches
# (dram__bytes_read.sum + dram__bytes_write.sum: 3014.7 MB per step). Valid for the kernel
# as captured; to be set to None when the kernel changes.
PAIR_DRAM_BYTES_PER_LAUNCH = 2985.1e6 / 8
PAIR_DRAM_SOURCE = "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean of the step's 8 launches"
# SHA-256 (first 16 hex digits) of the sources that define gemm_pair_kernel, as they were when the
# figure above was captured; when the sources differ the figure is stale and is reported as null.
PAIR_DRAM_SOURCES = ("sl_gemm.cu", "sl_gemm.h", "sl_ptx.cuh", "sl_internal.h")
PAIR_DRAM_SOURCE_SHA = "19ffcbf8776d459a"


def pair_sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in PAIR_DRAM_SOURCES:
        with open(os.path.join(ROOT, "contextual_sparsity_lora_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def pair_traffic():
    """(bytes per launch or None, source note) for the roofline's traffic key."""
    sha = pair_sources_sha()
    if sha == PAIR_DRAM_SOURCE_SHA:
        return PAIR_DRAM_BYTES_PER_LAUNCH, f"{PAIR_DRAM_SOURCE} (sources {sha})"
    return None, f"no capture of the current kernel sources ({sha}); the last capture was of {PAIR_DRAM_SOURCE_SHA}"


def capture_or_eager(fn, world):
    """A replay callable for one step: its CUDA graph, or with N > 1 (NCCL collectives inside
    the step), the eager step when the collectives cannot be captured. Returns (callable,
    captured)."""
    if world == 1:
        return capture_graph(fn, warm=False).replay, True
    try:
        g = capture_graph(fn, warm=False)
        _GRAPHS.append(g)  # released before the process group is destroyed
        return g.replay, True
    except Exception as e:  # noqa: BLE001 - any capture failure falls back to the eager step
        print(f"rank step not captured ({type(e).__name__}: {e}); timing the eager step", file=sys.stderr)
        torch.cuda.synchronize()
        return fn, False


_GRAPHS = []


def time_steps(fn, K, W, world, device):
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    barrier(world)
    return max_over_ranks(ms, world, device)


def stage_times(attn, ffn, s, reps, device, hbm_gbs, step_ms):
    """Device time of the selection stages of both blocks, each captured alone in a CUDA graph
    (`inner` back-to-back copies of the stage per graph, so that the host's graph launches do not
    pace tiny stages) and replayed `reps` times. The step runs the estimator's stage 1 (a1, Z =
    X_ctx W_A) as extra columns of the LoRA x A^T launch that streams the same rows
    (sl_lora_fwd_estimate): its cost is the difference between that launch and the x A^T launch
    alone. Then a2 (sl_svd_scores_from_z: the criterion from Z), a3 (sl_select_channels) and the
    per-step compaction of the kept weight rows. The standalone estimator (sl_svd_estimate: its own
    pass over X_ctx, then the criterion) is timed beside it for reference."""
    from contextual_sparsity_lora_b200 import binding as B
    inner = 10

    def graph_us(fn):
        fn()

        def many():
            for _ in range(inner):
                fn()
        g = capture_graph(many, warm=False)
        return time_steps(g.replay, reps, 3, 1, device) / (reps * inner) * 1e3

    out = {}
    total = 0.0
    for name, blk, x in (("attn", attn, s["x"]), ("ffn", ffn, s["ffn_x"])):
        C, D = blk.n_ctx, x.shape[1]
        T = x.shape[0]
        if name == "attn":
            lins = [blk.lin[n] for n in "qkv"]
            xa, xa_s, crit, n_proj = blk.xa_qkv, blk.xa_s_qkv, B.SL_CRIT_QK, 3
            kw = dict(scores_v=blk.s_v, n_q_heads=blk.hq, n_kv_heads=blk.hkv, head_dim=blk.hd)
            sc, WB = blk.s_qk, blk.WB
        else:
            lins = [blk.lin_g, blk.lin_u]
            xa, xa_s, crit, n_proj = blk.xa_gu, blk.xa_s_gu, B.SL_CRIT_SWIGLU_L2, 2
            kw = {}
            sc, WB = blk.scores, [blk.WBg, blk.WBu]
        lora_us = graph_us(lambda: B.sl_lora_fwd_bwd(blk.ws, B.SL_LORA_FWD, lins, x, C, xa_s, xa=xa))
        fused_us = graph_us(lambda: B.sl_lora_fwd_estimate(blk.ws, lins, x, C, xa_s, xa, n_proj, blk.k, blk.WAt,
                                                          blk.z))
        a2 = graph_us(lambda: B.sl_svd_scores_from_z(blk.ws, crit, WB, blk.k, blk.z, C, sc, **kw))
        sel = graph_us(blk.choose)
        # kept weight rows: read in place by the sliced products (no launch), or compacted per step
        comp = graph_us(blk.compact) if blk.kept_rows == "compact" else 0.0
        standalone = graph_us(lambda: blk.estimate(x))
        a1 = max(fused_us - lora_us, 0.0)
        fused_bytes = T * D * 2 + (sum(l.r for l in lins) + n_proj * blk.k) * D * 2
        out[name] = {"a1_marginal_us": a1, "lora_x_at_us": lora_us, "lora_x_at_with_z_us": fused_us,
                     "fused_launch_bytes": fused_bytes, "fused_launch_GBs": fused_bytes / (fused_us * 1e3),
                     "fused_launch_frac_of_hbm": fused_bytes / (fused_us * 1e3) / hbm_gbs,
                     "a2_criterion_us": a2, "a3_select_us": sel, "kept_rows": blk.kept_rows,
                     "compact_weights_us": comp,
                     "standalone_estimator_us": standalone}
        total += a1 + a2 + sel
    # criterion ablation variants (not on the step's path): the Wanda-style FFN criterion
    # (reads X_ctx and the gate and up weights once) and the head-level QK selection
    C, D, F = ffn.n_ctx, ffn.D, ffn.F
    ws = B.Workspace(device)
    wanda_sc = torch.empty(F, device=device)
    xf = s["ffn_x"]
    w_us = graph_us(lambda: B.sl_wanda_scores(ws, xf[:C], C, [ffn.Wg, ffn.Wu], wanda_sc))
    w_bytes = C * D * 2 + 2 * F * D * 2
    sig_k = torch.empty_like(attn.sig_k)
    sig_q = torch.empty_like(attn.sig_q)
    h_us = graph_us(lambda: B.sl_select_heads(attn.s_qk, attn.hkv, attn.hd, attn.n_keep_heads, sig_k, attn.hpg,
                                              sig_q))
    out["variants"] = {"ffn_wanda_scores_us": w_us, "ffn_wanda_bytes": w_bytes,
                       "ffn_wanda_GBs": w_bytes / (w_us * 1e3), "ffn_wanda_frac_of_hbm": w_bytes / (w_us * 1e3) / hbm_gbs,
                       "qk_head_select_us": h_us}
    out["estimator_and_select_us"] = total
    if step_ms:
        out["estimator_and_select_pct_of_step"] = 100.0 * total / (step_ms * 1e3)
    out["timing"] = ("each stage alone, 10 copies per CUDA graph, replayed; device time between events; "
                     "a1 = the x A^T launch with Z minus the x A^T launch alone")
    return out


def rank_sweep(fc, x, C, device, ks=(4, 8, 16), reps=20):
    """Estimator rank k against cost and fidelity on the LLaMA3-8B FFN (the sweep the pages leave
    open): for each k, the device time of estimator + selection (10 copies per CUDA graph) and
    how well the estimated kept set matches the kept set of the exact criterion,
    ||SiLU(X_ctx W_g^T)[:, i] * (X_ctx W_u^T)[:, i]||_2 computed with full products (torch,
    evaluation only): the recall of the exact top-n and the share of the exact top-n's squared
    criterion mass the estimated set holds. One spectral draw with rank-16 factors; ranks 4 and
    8 are its truncations (the leading singular triplets), so every k sees the same weights."""
    from contextual_sparsity_lora_b200 import blocks
    d = inputs.make_ffn_inputs(inputs.scaled(fc, k=max(ks)), 1, device=device)
    T = fc.n_tok
    xc = x[:C].float()
    g = xc @ d["gate"].W.float().t()
    u = xc @ d["up"].W.float().t()
    s_true = (torch.nn.functional.silu(g) * u).pow(2).sum(0)
    del g, u, xc
    out = {}
    for k in ks:
        cut = lambda w: inputs.SpectralWeight(W=w.W, W_A=w.W_A[:, :k].contiguous(), W_B=w.W_B[:k].contiguous(), s=w.s)
        blk = blocks.FFNBlock(cut(d["gate"]), cut(d["up"]), cut(d["down"]), d["lora_gate"], d["lora_up"],
                              d["lora_down"], fc.lora_scale, k, T, C, fc.ratio, device)

        def sel():
            blk.estimate(x)
            blk.choose()
        sel()
        g10 = capture_graph(lambda: [sel() for _ in range(10)], warm=False)
        us = time_steps(g10.replay, reps, 3, 1, device) / (reps * 10) * 1e3
        n = blk.n_keep
        top = torch.topk(s_true, n).indices
        kept = blk.sigma[:n].long()
        out[f"k{k}"] = {"estimate_select_us": us,
                        "recall_of_exact_top_n": float(torch.isin(kept, top).float().mean()),
                        "exact_mass_share": float(s_true[kept].sum() / s_true[top].sum())}
        del g10, blk
        torch.cuda.synchronize()
    out["workload"] = (f"LLaMA3-8B FFN, {C} context rows, keep {fc.ratio}; synthetic weights with singular "
                       f"values i^-{fc.alpha}")
    return out


def cpu_baseline(da, df, ratio, n_tokens=512, n_seqs=1):
    """The fp64 oracle on the host cores over a bounded sample: ``n_tokens`` consecutive
    tokens of the first sequence, the window placed so that context and output tokens keep the
    workload's proportion (the whole sequence at 512: 384 context + 128 output; at 128:
    96 + 32), through both blocks, estimator to LoRA gradients."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    ac, fc = inputs.LLAMA3_8B_ATTN, inputs.LLAMA3_8B_FFN
    S = int(n_tokens)
    n_o = round(S * ac.n_out / ac.seq)             # output tokens of the window
    end = ac.seq - ac.n_out + n_o
    sl = slice(end - S, end)                       # sequence order, ends n_o tokens into the output part
    ctx = da["ctx_mask"][sl].cpu().numpy()
    f64 = oracle.f64
    X = f64(da["x"][sl]); XO = f64(da["x_o"][sl]); dq = f64(da["dq"][sl]); dk = f64(da["dk"][sl])
    dv = f64(da["dv"][sl]); dyo = f64(da["dy"][sl]); Xf = f64(df["x"][sl]); dyf = f64(df["dy"][sl])
    W = {n: f64(da[n].W) for n in "qkvo"}
    F = {n: (f64(da[n].W_A), f64(da[n].W_B)) for n in "qkv"}
    L = {n: (f64(da["lora_" + n][0]), f64(da["lora_" + n][1])) for n in "qkvo"}
    Wf = {n: f64(df[n].W) for n in ("gate", "up", "down")}
    Ff = {n: (f64(df[n].W_A), f64(df[n].W_B)) for n in ("gate", "up")}
    Lf = {n: (f64(df["lora_" + n][0]), f64(df["lora_" + n][1])) for n in ("gate", "up", "down")}
    s = ac.lora_scale
    t0 = time.perf_counter()
    for _ in range(n_seqs):
        _oracle_layer(oracle, X, XO, dq, dk, dv, dyo, Xf, dyf, ctx, W, F, L, Wf, Ff, Lf, s, ac, ratio)
    dt = time.perf_counter() - t0
    S = S * n_seqs
    return {"value": S / dt, "unit": UNIT, "cores": int(threads), "blas_threads": int(threads), "kind": "oracle",
            "sample": f"{S} tokens ({n_seqs} x {S // n_seqs} of one sequence, {int(ctx.sum())} context + "
                      f"{S // n_seqs - int(ctx.sum())} output each) through both blocks, fp64 NumPy, {dt:.1f} s",
            "seconds": dt, "host_cpus": os.cpu_count()}


def _oracle_layer(oracle, X, XO, dq, dk, dv, dyo, Xf, dyf, ctx, W, F, L, Wf, Ff, Lf, s, ac, ratio):
    sel = oracle.attn_select(X, ctx, F["q"], F["k"], F["v"], ac.n_q_heads, ac.n_kv_heads, ac.head_dim, ratio)
    for n, xin, kind in (("q", X, "out"), ("k", X, "out"), ("v", X, "out"), ("o", XO, "in")):
        oracle.sparse_linear_fwd(xin, W[n], *L[n], s, ctx, sel["idx_" + n], kind)
    for n, xin, g, kind in (("q", X, dq, "out"), ("k", X, dk, "out"), ("v", X, dv, "out"), ("o", XO, dyo, "in")):
        oracle.sparse_linear_bwd(xin, g, W[n], *L[n], s, ctx, sel["idx_" + n], kind)
    _, idx = oracle.ffn_select(Xf, ctx, Ff["gate"], Ff["up"], ratio)
    fwd = oracle.ffn_fwd(Xf, ctx, Wf["gate"], Wf["up"], Wf["down"], Lf["gate"], Lf["up"], Lf["down"], s, idx)
    oracle.ffn_bwd(Xf, dyf, ctx, Wf["gate"], Wf["up"], Wf["down"], Lf["gate"], Lf["up"], Lf["down"], s, idx, fwd=fwd)


def model_measure(da, df, perm, C, ac, fc, device, keep, n_steps=20, vocab=128256, peak_lr=1e-4):
    """A 20-step fine-tuning run of a 32-layer LLaMA3-8B-shaped model: embedding, 32 decoder
    layers with the per-layer keep table `keep`, final RMSNorm, LM head with cross-entropy on the
    output rows, backward, AdamW on every LoRA matrix at the cosine schedule's rate; the first
    10% of the steps dense (progressive schedule). Each layer's frozen projection weights are a
    random signed permutation of one decaying-spectrum draw per projection (distinct weights of
    the same spectrum, exact factors); LoRA matrices and RMSNorm gains are per layer. Each
    mode's forward + backward is one CUDA graph (captured once); AdamW runs per block between
    replays, all inside the timed region."""
    from contextual_sparsity_lora_b200.model import SparseLoRAModel, cosine_lr
    gen = torch.Generator(device="cpu")
    gen.manual_seed(91)
    D, n_layers = ac.hidden, len(keep)
    base = {"q": da["q"], "k": da["k"], "v": da["v"], "o": da["o"], "gate": df["gate"], "up": df["up"],
            "down": df["down"]}
    frozen = {"layers": [{n: inputs.signed_permutation(w, gen) for n, w in base.items()} for _ in range(n_layers)]}
    frozen["embed"] = torch.randn(vocab, D, device=device, dtype=torch.bfloat16)
    frozen["lm_head"] = 0.02 * torch.randn(vocab, D, device=device, dtype=torch.bfloat16)
    frozen["gamma_f"] = torch.ones(D, dtype=torch.bfloat16)
    shapes = {n: tuple(w.W.shape) for n, w in base.items()}
    loras = [{n: inputs.lora_pair(do, di, ac.r, 0.02, gen) for n, (do, di) in shapes.items()} for _ in range(n_layers)]
    gammas = [(torch.ones(D, dtype=torch.bfloat16), torch.ones(D, dtype=torch.bfloat16)) for _ in range(n_layers)]
    model = SparseLoRAModel(frozen, loras, gammas, keep, perm.cpu().numpy(), C, ac.batch,
                            (ac.n_q_heads, ac.n_kv_heads, ac.head_dim), ac.k, ac.lora_scale, device)
    del frozen
    T = ac.n_tok
    ids_cf = torch.randint(0, vocab, (T,), generator=gen).to(torch.int32).to(device)
    targets = torch.randint(0, vocab, (T - C,), generator=gen).to(device)
    graphs = {}
    for dense in (True, False):
        model.set_dense(dense)
        for _ in range(2):
            model.forward_backward(ids_cf, targets)
        torch.cuda.synchronize()
        graphs[dense] = capture_graph(lambda: model.forward_backward(ids_cf, targets), warm=False)
    n_dense = math.ceil(0.1 * n_steps)
    times, losses = [], []
    for step in range(1, n_steps + 1):
        dense = step <= n_dense
        model.set_dense(dense)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graphs[dense].replay()
        model.optimizer_step(step, cosine_lr(step, n_steps, peak_lr))
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        losses.append(float(model.loss))
    total = sum(times)
    sparse_ms = sum(times[n_dense:]) / (n_steps - n_dense)
    dense_ms = sum(times[:n_dense]) / n_dense
    del graphs, model
    torch.cuda.synchronize()
    return {"value": n_steps * T / (total / 1e3), "unit": UNIT, "steps": n_steps, "dense_steps": n_dense,
            "ms_per_sparse_step": sparse_ms, "ms_per_dense_step": dense_ms,
            "sparse_vs_dense_speedup": dense_ms / sparse_ms, "run_vs_all_dense_speedup": n_steps * dense_ms / total,
            "loss_first": losses[0], "loss_last": losses[-1], "layers": n_layers, "vocab": vocab,
            "lr": f"AdamW, cosine schedule, 4% warm-up, peak {peak_lr}",
            "frozen_weights": "per layer: a random signed permutation of one decaying-spectrum draw per projection",
            "lm_head_and_cross_entropy": "torch (library)",
            "attention_core": "sl_attention_fwd / sl_attention_bwd (tcgen05, causal GQA)"}


def full_layer_measure(attn, ffn, step_in, perm, ac, K, W, device):
    """The whole decoder layer around the same blocks (RMSNorm, sparse q/k/v, causal GQA
    attention core, sparse o, residual, RMSNorm, sparse FFN, residual), forward and backward
    on the step's 8 x 512 tokens: context, not the headline."""
    from contextual_sparsity_lora_b200.layer import DecoderLayer
    gen = torch.Generator(device="cpu")
    gen.manual_seed(77)
    g1 = 1.0 + 0.1 * torch.randn(ac.hidden, generator=gen)
    g2 = 1.0 + 0.1 * torch.randn(ac.hidden, generator=gen)
    layer = DecoderLayer(attn, ffn, g1, g2, perm, ac.batch)
    x, dy = step_in["x"], step_in["dy"]
    for _ in range(2):
        layer.step(x, dy)
    torch.cuda.synchronize()
    replay = capture_graph(lambda: layer.step(x, dy), warm=False).replay
    ms = time_steps(replay, K, W, 1, device) / K
    return {"value": ac.n_tok / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "cuda_graph": True,
            "attention_core": attention_core_measure(layer, ac, K, W, device),
            "layer": "RMSNorm, sparse q/k/v, attention, sparse o, residual, RMSNorm, sparse SwiGLU FFN, residual"}


def attention_core_times(ws, q, k, v, o, d_o, lse, dq, dk, dv, n_seq, S, hq, hkv, hd, K, W, device):
    """sl_attention_fwd and sl_attention_bwd on the given buffers, each captured in a CUDA graph of
    10 calls: device time per call and TFLOP/s of the causal products (forward Q K^T and P V,
    backward the recomputed Q K^T, dO V^T, P^T dO, dS^T Q and dS K: 2 and 5 products of 2 hd FLOP
    per visible (query, key) pair)."""
    from contextual_sparsity_lora_b200 import binding as B
    pairs = n_seq * hq * S * (S + 1) / 2

    def fwd():
        B.sl_attention_fwd(ws, q, k, v, n_seq, hq, hkv, hd, o, lse)

    def bwd():
        B.sl_attention_bwd(ws, q, k, v, o, d_o, lse, n_seq, hq, hkv, hd, dq, dk, dv)

    out = {"kernels": "attn_fwd_kernel, attn_bwd_kernel (tcgen05, TMEM accumulators)",
           "shape": f"{n_seq} x {S} tokens, {hq} query / {hkv} key-value heads of {hd}, causal"}
    peak = float(load_peaks()[0].get("bf16_tflops", 1590.0))
    for name, fn, n_prod in (("fwd", fwd, 2), ("bwd", bwd, 5)):
        fn()
        g = capture_graph(lambda: [fn() for _ in range(10)], warm=False)
        us = time_steps(g.replay, K, W, 1, device) / (10 * K) * 1e3
        del g
        tf = n_prod * 2.0 * hd * pairs / (us * 1e-6) / 1e12
        out[f"{name}_us"] = us
        out[f"{name}_tflops"] = tf
        out[f"{name}_frac_of_bf16_peak"] = tf / peak
    return out


def attention_core_measure(layer, ac, K, W, device):
    """The layer's attention core alone, on the layer's own q, k, v, o, dO buffers after a step."""
    at = layer.attn
    return attention_core_times(layer.ws, layer.q_nat, layer.k_nat, layer.v_nat, layer.a_nat, layer.da_nat,
                                layer.lse, layer.dq_nat, layer.dk_nat, layer.dv_nat, layer.n_seq, layer.S, at.hq,
                                at.hkv, at.hd, K, W, device)


def attention_only(device, K, W):
    """The attention core alone at the LLaMA3-8B layer's shape (8 sequences of 512 tokens, 32
    query and 8 key-value heads of 128) on seeded normal q, k, v and dO (about 0.1 GB on the
    device): the small case for profiling the attention kernels."""
    from contextual_sparsity_lora_b200 import binding as B
    ac = inputs.LLAMA3_8B_ATTN
    T, hq, hkv, hd = ac.n_tok, ac.n_q_heads, ac.n_kv_heads, ac.head_dim
    g = torch.Generator(device=device)
    g.manual_seed(5)
    rnd = lambda n: torch.randn(T, n, generator=g, device=device).to(torch.bfloat16)
    q, k, v, d_o = rnd(hq * hd), rnd(hkv * hd), rnd(hkv * hd), rnd(hq * hd)
    o, dq = torch.empty_like(q), torch.empty_like(q)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    lse = torch.empty(hq, T, device=device)
    return attention_core_times(B.Workspace(device), q, k, v, o, d_o, lse, dq, dk, dv, ac.batch, ac.seq, hq, hkv, hd,
                                K, W, device)


def e2e_measure(attn, ffn, step_in, K, W, world, device, eager=False):
    """Same step through the public API with host buffers: every step copies that step's inputs
    from pinned host memory and reads the LoRA gradients back. The copies run on a second stream
    and are double-buffered: the inputs of step i+1 go into one device buffer while step i
    computes on the other, and the gradients of step i (snapshotted on the device) return to the
    host during step i+1. eager=False replays one captured graph of the step per input buffer;
    eager=True calls the library entries step by step (the host-side cost of every ABI call:
    argument checks, tensor-map encoding, marshalling, launches) with the same copies.
    Returns (ms per step, H2D bytes per step, D2H bytes per step)."""
    host = {k: v.cpu().pin_memory() for k, v in step_in.items()}
    bufs = [{k: torch.empty_like(v) for k, v in step_in.items()} for _ in range(2)]
    grads = [attn.dA[n] for n in "qkvo"] + [attn.dB[n] for n in "qkvo"] + \
        [ffn.dA_g, ffn.dB_g, ffn.dA_u, ffn.dB_u, ffn.dA_d, ffn.dB_d]
    snap = [torch.empty_like(g) for g in grads]
    host_out = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in grads]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(g.numel() * g.element_size() for g in grads)
    for b in bufs:
        for k in host:
            b[k].copy_(host[k])
    for _ in range(2):
        run_step(attn, ffn, bufs[0])
    torch.cuda.synchronize()
    if eager:
        replays = [(lambda b=b: run_step(attn, ffn, b)) for b in bufs]
    else:
        replays = [capture_or_eager(lambda b=b: run_step(attn, ffn, b), world)[0] for b in bufs]
    main = torch.cuda.current_stream()
    h2d_s = torch.cuda.Stream(device=device)   # inputs in
    d2h_s = torch.cuda.Stream(device=device)   # gradients out (its own stream: the two directions overlap)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer j have landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step that read buffer j has finished
    ev_snap, ev_out = torch.cuda.Event(), torch.cuda.Event()
    for e in ev_in + ev_done + [ev_out]:
        e.record(main)
    state = {"i": 0}

    def step():
        j = state["i"] % 2
        with torch.cuda.stream(h2d_s):     # step i+1's inputs into the other buffer, during step i
            h2d_s.wait_event(ev_done[1 - j])   # the buffer is free once the step that read it finished
            for k in host:
                bufs[1 - j][k].copy_(host[k], non_blocking=True)
            ev_in[1 - j].record(h2d_s)
        main.wait_event(ev_in[j])
        replays[j]()
        ev_done[j].record(main)
        main.wait_event(ev_out)            # the previous step's gradients have left the snapshot
        for d, g in zip(snap, grads):
            d.copy_(g)
        ev_snap.record(main)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_snap)
            for h, d in zip(host_out, snap):
                h.copy_(d, non_blocking=True)
            ev_out.record(d2h_s)
        state["i"] += 1

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for _ in range(K):
        step()
    main.wait_stream(h2d_s)                # the last step's copies belong to the timed region
    main.wait_stream(d2h_s)
    e1.record(main)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    barrier(world)
    return ms / K, h2d, d2h


def sweep_measure(device, K, W):
    """Keep-ratio sweep of the LLaMA3-8B workload (the pages' operating points at several
    sparsities): for keep 1.0 (dense LoRA on the same kernels, no estimator), 0.7, 0.5 and 0.3,
    the FFN block alone and the whole 7-projection step, each one CUDA graph replayed K times."""
    out = {}
    ac, fc = inputs.LLAMA3_8B_ATTN, inputs.LLAMA3_8B_FFN
    for ratio in (1.0, 0.7, 0.5, 0.3):
        attn, ffn, s_in, C, _, _ = make_layer(ratio, 0, 1000, device, dense=ratio >= 1.0)
        for _ in range(3):
            run_step(attn, ffn, s_in)
        torch.cuda.synchronize()
        g_all = capture_graph(lambda: run_step(attn, ffn, s_in), warm=False)
        ms_all = time_steps(g_all.replay, K, W, 1, device) / K
        del g_all
        g_ffn = capture_graph(lambda: ffn.step(s_in["ffn_x"], s_in["ffn_dy"]), warm=False)
        ms_ffn = time_steps(g_ffn.replay, K, W, 1, device) / K
        del g_ffn
        fl = algorithmic_flops(ac, fc, C, ratio, dense=ratio >= 1.0)
        nk = fc.inter if ratio >= 1.0 else inputs_keep(ratio, fc.inter)
        f = flops.ffn_block(fc.hidden, fc.inter, fc.n_tok, C, nk, fc.r, fc.k, with_estimator=ratio < 1.0)
        out[f"keep{ratio}"] = {"step_ms": ms_all, "step_tokens_per_s": ac.n_tok / (ms_all / 1e3),
                               "step_effective_tflops": fl["total"] / (ms_all / 1e3) / 1e12,
                               "ffn_ms": ms_ffn, "ffn_tokens_per_s": fc.n_tok / (ms_ffn / 1e3),
                               "ffn_effective_tflops": f["total"] / (ms_ffn / 1e3) / 1e12}
        del attn, ffn, s_in
        torch.cuda.synchronize()
    out["workload"] = "LLaMA3-8B, 8 x 512 tokens (last 128 output), LoRA rank 32, estimator rank 8"
    return out


def llama2_13b_measure(device, K, W):
    """The LLaMA2-13B layer's seven projections (4 x 1024 tokens, last 256 output; MHA 40 x 128,
    FFN 13824; LoRA rank 32, estimator rank 16) at keep 0.4, and densely (keep 1, no estimator)."""
    ac, fc = inputs.LLAMA2_13B_ATTN, inputs.LLAMA2_13B_FFN
    res = {}
    for name, ratio, dense in (("sparse", ac.ratio, False), ("dense_lora", 1.0, True)):
        attn, ffn, s_in, C, _, _ = make_layer(ratio, 0, 1000, device, dense=dense, cfgs=(ac, fc))
        for _ in range(3):
            run_step(attn, ffn, s_in)
        torch.cuda.synchronize()
        g = capture_graph(lambda: run_step(attn, ffn, s_in), warm=False)
        ms = time_steps(g.replay, K, W, 1, device) / K
        fl = algorithmic_flops(ac, fc, C, ratio, dense=dense)
        res[name] = {"ms_per_step": ms, "tokens_per_s": ac.n_tok / (ms / 1e3),
                     "effective_tflops": fl["total"] / (ms / 1e3) / 1e12,
                     "algorithmic_tflop_per_step": fl["total"] / 1e12}
        del g, attn, ffn, s_in
        torch.cuda.synchronize()
    res["speedup_vs_dense_lora"] = res["dense_lora"]["ms_per_step"] / res["sparse"]["ms_per_step"]
    res["workload"] = "llama2-13b-layer-7proj-b4s1024-keep0.4-k16"
    return res


def cpu_tiny_single_core(repeats=3):
    """The fp64 oracle on one host thread (BLAS limited to one thread) for the tiny fp32 FFN
    configuration (hidden 256, FFN 688, 2 x 64 tokens, last 16 output, LoRA rank 8, estimator
    rank 8, keep 0.5): estimator, selection, forward and backward of the block."""
    import numpy as np
    import oracle
    from threadpoolctl import threadpool_limits
    cfg = inputs.TINY_FFN
    d = inputs.make_ffn_inputs(cfg, seed=0, device="cpu")
    ctx = d["ctx_mask"].numpy()
    X, dY = oracle.f64(d["x"]), oracle.f64(d["dy"])
    W = {n: oracle.f64(d[n].W) for n in ("gate", "up", "down")}
    Fa = {n: (oracle.f64(d[n].W_A), oracle.f64(d[n].W_B)) for n in ("gate", "up")}
    L = {n: (oracle.f64(d["lora_" + n][0]), oracle.f64(d["lora_" + n][1])) for n in ("gate", "up", "down")}
    times = []
    with threadpool_limits(limits=1):
        for _ in range(repeats):
            t0 = time.perf_counter()
            _, idx = oracle.ffn_select(X, ctx, Fa["gate"], Fa["up"], cfg.ratio)
            fwd = oracle.ffn_fwd(X, ctx, W["gate"], W["up"], W["down"], L["gate"], L["up"], L["down"],
                                 cfg.lora_scale, idx)
            oracle.ffn_bwd(X, dY, ctx, W["gate"], W["up"], W["down"], L["gate"], L["up"], L["down"],
                           cfg.lora_scale, idx, fwd=fwd)
            times.append(time.perf_counter() - t0)
    t = min(times)
    return {"value": cfg.n_tok / t, "unit": UNIT, "seconds": t, "threads": 1, "blas_threads": 1,
            "workload": cfg.name, "repeats": repeats, "np_version": np.__version__}


def reference_arm(args, rank, world):
    """The oracle timed on this machine's host cores (rank 0 only) over bounded samples."""
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    device = "cuda" if torch.cuda.is_available() else "cpu"
    ac = inputs.LLAMA3_8B_ATTN
    da = inputs.make_attn_inputs(ac, 0, device=device)
    df = inputs.make_ffn_inputs(inputs.LLAMA3_8B_FFN, 1, device=device)
    n_tok = 128
    times = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(da, df, args.ratio, n_tokens=n_tok)
        if i >= args.warmup:
            times.append(cb["seconds"])
    per = sum(times) / len(times)
    value = n_tok / per
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "seq_len": ac.seq, "sample_tokens_per_step": n_tok},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_setup(args.gpus, cpu_only=args.impl == "reference")
    if args.impl == "reference":
        try:
            reference_arm(args, rank, world)
        finally:
            dist_teardown(world)
        return
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    from contextual_sparsity_lora_b200 import binding as B
    from contextual_sparsity_lora_b200 import blocks
    B.lib()
    if args.attention_only:
        if rank == 0:
            print(json.dumps({"attention_core": attention_only(device, args.steps, max(args.warmup, 3))}))
        barrier(world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    # N > 1: every rank takes its own 4096-token share of the global batch; the criterion
    # statistics and the LoRA gradients are summed over the ranks (NCCL all-reduce)
    dp = blocks.DataParallel() if world > 1 else None
    attn, ffn, step_in, C, (ac, fc), (da, df, perm) = make_layer(args.ratio, 0, 1000 + rank, device, dp=dp)
    T = ac.n_tok
    B.sl_profile_enable(False)
    for _ in range(max(args.warmup, 3)):   # eager warm-up: sizes every workspace
        run_step(attn, ffn, step_in)
    torch.cuda.synchronize()
    B.sl_profile_read()
    if args.stages_only:
        if rank == 0:
            attn.dp = ffn.dp = None  # rank-local stages only: no collective inside the stage graphs
            print(json.dumps({"stages": stage_times(attn, ffn, step_in, 50, device,
                                                    float(load_peaks()[0].get("hbm_gbs", 6650.0)), None)}))
        barrier(world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    # The step is captured once into a CUDA graph and replayed; every replay runs every
    # kernel. The headline graph carries no event nodes. A second capture of the same step,
    # with the library's launch counting and an event pair around each GEMM-engine launch,
    # is replayed over its own K timed steps for the roofline's kernel durations.
    graph, use_graph = capture_or_eager(lambda: run_step(attn, ffn, step_in), world)
    n_launch_headline = None
    if use_graph:
        # the headline step's own launch count: a discarded capture of the same (concurrent)
        # step with the library's launch counting on
        B.sl_profile_read()
        B.sl_profile_enable(True)
        cnt_graph, _ = capture_or_eager(lambda: run_step(attn, ffn, step_in), world)
        B.sl_profile_enable(False)
        cnt_graph()  # one replay records the capture's event pairs, which the read waits for
        torch.cuda.synchronize()
        n_launch_headline = B.sl_profile_read()[0]
        del cnt_graph  # before the profiled copy's capture reuses the library's event pairs
        torch.cuda.synchronize()
    # (the profiled copy runs each block's chains in order, so that no concurrent kernel
    # stretches a GEMM-engine launch's event-timed duration)
    attn.concurrent = ffn.concurrent = False
    B.sl_profile_enable(True)
    prof_graph, _ = capture_or_eager(lambda: run_step(attn, ffn, step_in), world) if use_graph else (graph, False)
    B.sl_profile_enable(False)
    attn.concurrent = ffn.concurrent = True
    with ClockSampler(local) as clk:
        ms = time_steps(graph, args.steps, args.warmup, world, device)
    torch.cuda.synchronize()
    prof_ms = time_steps(prof_graph, args.steps, args.warmup, world, device)
    torch.cuda.synchronize()
    # GEMM-engine durations of the profiled copy's last replay, per launch and in total; the
    # launch count is the headline graph's (the profiled copy's when the step is not captured)
    per_launch = B.sl_profile_launches()
    n_launch_step, n_gemm, gemm_ms = B.sl_profile_read()
    if n_launch_headline is not None:
        n_launch_step = n_launch_headline
    pair_ms = sum(m for m, k in per_launch if k in (1, 2))
    pair_n = sum(1 for _, k in per_launch if k in (1, 2))
    skinny_ms = sum(m for m, k in per_launch if k in (0, 3, 4))
    skinny_n = sum(1 for _, k in per_launch if k in (0, 3, 4))
    del prof_graph
    n_launch = n_launch_step * args.steps
    ms_step = ms / args.steps
    value = world * T / (ms_step / 1e3)
    fl = algorithmic_flops(ac, fc, C, args.ratio, dense=False)
    # dominant kernel: the CTA-pair GEMM launches (the sliced main-branch products with the
    # LoRA up-projections fused as K extensions: y += xa_s B^T, dx += dya_s A, i.e. one third
    # of the LoRA FLOPs); the one-CTA launches (rank-r LoRA products, estimator stage 1)
    # are HBM-bound and reported apart
    pair_flops = fl["main"] + fl["lora"] / 3.0
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops"))
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
    traffic, traffic_src = pair_traffic()
    achieved = pair_flops / (pair_ms / 1e3) / 1e12 if pair_ms > 0 else None
    skinny_bytes = flops.lora_skinny_bytes([(T, ac.hidden, (ac.n_q_heads * ac.head_dim, 2 * ac.n_kv_heads * ac.head_dim)),
                                            (T, ac.n_q_heads * ac.head_dim, (ac.hidden,)),
                                            (T, fc.hidden, (2 * fc.inter,)), (T, fc.inter, (fc.hidden,))])
    # (the estimator's stage 1 rides in the x A^T launches of q/k/v and gate/up: no bytes of its own)
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": 8 * world, "seq_len": ac.seq, "tokens_per_rank": T,
                   "context_tokens_per_rank": C, "keep_ratio": args.ratio, "lora_rank": ac.r,
                   "estimator_rank": ac.k, "parallelism": f"dp{world}",
                   "exchange": ("per block: fp64 all-reduce of the criterion statistics (one index set per "
                                "global batch), fp32 all-reduce of the LoRA gradients") if world > 1 else "none",
                   "l2": "per-step working set ~1.4 GB > 126 MB L2; no flush"},
        "roofline": {"bound": "tensor", "kernel": "sl::gemm_pair_kernel (CTA-pair tcgen05 GEMM: sliced products)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": (achieved / peak) if achieved else None,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "peak_source": f"{src} bf16_tflops (burst: the step's timed region lasts well under the "
                                    f"seconds-long loop of the sustained figure)",
                     "frac_of_sustained": (achieved / peak_sus) if achieved else None,
                     "algorithmic_tflop_per_launch": pair_flops / 1e12 / max(pair_n, 1),
                     "launches_per_step": pair_n, "ms_per_launch": pair_ms / max(pair_n, 1),
                     "gemm_engine_ms_per_step": gemm_ms, "gemm_engine_launches_per_step": n_gemm,
                     "skinny_lora_and_stage1": {"bound": "hbm", "ms_per_step": skinny_ms,
                                                "what": "one-CTA rank-r launches (x A^T with the estimator's Z, "
                                                        "dA = dya^T x) and the fused LoRA backward",
                                                "launches_per_step": skinny_n,
                                                "algorithmic_bytes_per_step": skinny_bytes,
                                                "achieved_GBs": skinny_bytes / (skinny_ms * 1e6) if skinny_ms else None,
                                                "peak_GBs": hbm,
                                                "frac": skinny_bytes / (skinny_ms * 1e6) / hbm if skinny_ms else None},
                     "timing": "event pair around each GEMM-engine launch, in a separately captured "
                               "copy of the step replayed over its own timed steps",
                     "profiled_step_ms": prof_ms / args.steps,
                     "algorithmic_tflop_per_step": pair_flops / 1e12},
        "gpu_launches": n_launch,
        "gpu_launches_per_step": n_launch_step, "cuda_graph": use_graph,
        "effective_tflops": fl["total"] / (ms_step / 1e3) / 1e12,
        "clocks": clk.summary(),
    }
    if rank == 0:
        saved = (attn.dp, ffn.dp)
        attn.dp = ffn.dp = None  # rank-local stages only: no collective inside the stage graphs
        line["stages"] = stage_times(attn, ffn, step_in, 50, device, float(peaks.get("hbm_gbs", 6650.0)), ms_step)
        if world == 1:
            line["stages"]["estimator_rank_sweep"] = rank_sweep(fc, step_in["ffn_x"], C, device)
        attn.dp, ffn.dp = saved
    barrier(world)
    # dense LoRA on the same kernels (keep ratio 1, no estimator): context, not the headline
    if not args.no_dense:
        d_attn, d_ffn, _, _, _, _ = make_layer(1.0, 0, 1000 + rank, device, dense=True, dp=dp)
        for _ in range(3):
            run_step(d_attn, d_ffn, step_in)
        d_graph, _ = capture_or_eager(lambda: run_step(d_attn, d_ffn, step_in), world)
        d_ms = time_steps(d_graph, args.steps, max(args.warmup, 3), world, device)
        d_fl = algorithmic_flops(ac, fc, C, 1.0, dense=True)
        line["dense_lora"] = {"value": world * T / (d_ms / args.steps / 1e3), "unit": UNIT,
                              "ms_per_step": d_ms / args.steps,
                              "effective_tflops": d_fl["total"] / (d_ms / args.steps / 1e3) / 1e12}
        line["speedup_vs_dense_lora"] = line["dense_lora"]["ms_per_step"] / ms_step
        del d_attn, d_ffn, d_graph
        # the same sparse step with the kept weight rows read in place by the GEMM's row-gather
        # copies instead of the per-step compacted copy: context, not the headline
        c_attn, c_ffn, _, _, _, _ = make_layer(args.ratio, 0, 1000 + rank, device, dp=dp, kept_rows="gather")
        for _ in range(3):
            run_step(c_attn, c_ffn, step_in)
        c_graph, _ = capture_or_eager(lambda: run_step(c_attn, c_ffn, step_in), world)
        c_ms = time_steps(c_graph, args.steps, max(args.warmup, 3), world, device)
        line["kept_rows_gathered"] = {"ms_per_step": c_ms / args.steps, "value": world * T / (c_ms / args.steps / 1e3),
                                      "unit": UNIT, "step_ms_ratio_to_compacted": c_ms / args.steps / ms_step,
                                      "what": "kept weight rows read in place by tile::gather4 operand copies"}
        del c_attn, c_ffn, c_graph
    if world == 1 and not args.no_model:
        from contextual_sparsity_lora_b200.model import layerwise_keep, llama3_8b_math10k_keep
        line["model_32_layers"] = model_measure(da, df, perm, C, ac, fc, device, layerwise_keep())
        line["model_32_layers"]["keep_table"] = "layers 0-7 dense, 8-19 keep 0.6, 20-31 keep 0.35 (attention and FFN)"
        m10 = model_measure(da, df, perm, C, ac, fc, device, llama3_8b_math10k_keep())
        m10["keep_table"] = "FFN keep 0.01 on L3-L30, QKVO keep 0.25 on L14-19, L21-23, L25-29, else dense (from 1)"
        line["model_32_layers_math10k_table"] = m10
    if world == 1 and not args.no_layer:
        line["full_layer"] = full_layer_measure(attn, ffn, step_in, perm, ac, args.steps, max(args.warmup, 3), device)
    if world == 1 and not args.no_sweep:
        line["sweep"] = sweep_measure(device, args.steps, max(args.warmup, 3))
        line["llama2_13b_layer"] = llama2_13b_measure(device, args.steps, max(args.warmup, 3))
    if not args.no_e2e:
        how = ("inputs from pinned host memory on a copy stream into two device buffers (step i+1's copy "
               "overlaps step i), LoRA gradients snapshotted on the device and read back on a third stream "
               "during the next step")
        e2e_ms, h2d, d2h = e2e_measure(attn, ffn, step_in, args.steps, max(args.warmup, 3), world, device)
        line["e2e"] = {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "copies": how,
                       "step": "one CUDA graph of the step per input buffer"}
        ee_ms, _, _ = e2e_measure(attn, ffn, step_in, args.steps, max(args.warmup, 3), world, device, eager=True)
        line["e2e_eager"] = {"value": world * T / (ee_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                             "d2h_bytes_per_step": d2h, "ms_per_step": ee_ms, "copies": how,
                             "step": "every library entry called from Python per step (no graph): argument "
                                     "checks, tensor-map encoding and ctypes marshalling included"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(da, df, args.ratio, n_tokens=512, n_seqs=3).items()
                                if k != "seconds"}
        line["cpu_baseline"]["single_core_tiny_ffn"] = cpu_tiny_single_core()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graph, prof_graph
        _GRAPHS.clear()
        torch.cuda.synchronize()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
