"""sl_svd_estimate_noalloc: the estimator on the library's fixed scratch array.

Collected last on purpose: it must give the workspace entry's scores both in a fresh
process and after every other test has run kernels on the device. The GPU cases call the
entry through the C ABI (ctypes) several times in a row, each time on new inputs and
another scratch layout, so that contents left in the shared array by the previous call
cannot leak into the next one."""
import ctypes

import pytest
import torch

from contextual_sparsity_lora_b200 import binding as B

FP32_TOL = 1e-5  # relative Frobenius error allowed between two fp32 score vectors


def _rel(got, want):
    got, want = got.double(), want.double()
    return float((got - want).norm() / want.norm().clamp_min(1e-300))


def test_rejects_shapes_beyond_the_fixed_scratch():
    """Host-side: too many context rows for the 8 MiB array is refused before any device work,
    with the bytes it would need reported; argument errors pass through unchanged."""
    lib = B.lib()
    P = ctypes.c_void_p
    fake = 0x10000  # never dereferenced: the call returns before touching the device
    wa = (P * 3)(fake, fake, fake)
    wb = (P * 3)(fake, fake, fake)
    dout = (ctypes.c_int64 * 3)(4096, 1024, 1024)
    need = ctypes.c_int64(-1)
    f = lib.sl_svd_estimate_noalloc
    rc = f(B.SL_CRIT_QK, B.SL_DT_BF16, P(fake), 1 << 20, 4096, 4096, 3, wa, wb, dout, 8, 32, 8, 128, P(fake),
           P(fake), ctypes.byref(need), None, None)
    assert rc == B.SL_ERR_WORKSPACE
    assert need.value > 8 << 20
    need.value = -1
    rc = f(B.SL_CRIT_QK, B.SL_DT_BF16, None, 64, 4096, 4096, 3, wa, wb, dout, 8, 32, 8, 128, P(fake), P(fake),
           ctypes.byref(need), None, None)
    assert rc == B.SL_ERR_INVALID_ARG
    assert need.value == -1


def _ffn_case(seed, n_ctx=3072, d=4096, f=14336, k=8, dev="cuda"):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(n_ctx, d, generator=g) * 0.5).to(torch.bfloat16).to(dev)
    wa = [(torch.randn(d, k, generator=g) / d ** 0.5).to(torch.bfloat16).to(dev) for _ in range(2)]
    wb = [torch.randn(k, f, generator=g).to(torch.bfloat16).to(dev) for _ in range(2)]
    return dict(crit=B.SL_CRIT_SWIGLU_L2, x=x, n_ctx=n_ctx, w_a=wa, w_b=wb, k=k, outs=[f], heads=(0, 0, 0))


def _attn_case(seed, n_ctx=2000, d=4096, hq=32, hkv=8, hd=128, k=8, dev="cuda"):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(n_ctx, d, generator=g) * 0.5).to(torch.bfloat16).to(dev)
    dims = (hq * hd, hkv * hd, hkv * hd)
    wa = [(torch.randn(d, k, generator=g) / d ** 0.5).to(torch.bfloat16).to(dev) for _ in dims]
    wb = [torch.randn(k, n, generator=g).to(torch.bfloat16).to(dev) for n in dims]
    return dict(crit=B.SL_CRIT_QK, x=x, n_ctx=n_ctx, w_a=wa, w_b=wb, k=k, outs=[hkv * hd, hkv * hd],
                heads=(hq, hkv, hd))


def _l2_fp32_case(seed, n_ctx=96, d=256, n=688, k=8, dev="cuda"):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n_ctx, d, generator=g).to(dev)
    wa = [(torch.randn(d, k, generator=g) / d ** 0.5).to(dev)]
    wb = [torch.randn(k, n, generator=g).to(dev)]
    return dict(crit=B.SL_CRIT_L2, x=x, n_ctx=n_ctx, w_a=wa, w_b=wb, k=k, outs=[n], heads=(0, 0, 0))


def _scores(case, fn):
    outs = [torch.full((n,), float("nan"), device="cuda") for n in case["outs"]]
    hq, hkv, hd = case["heads"]
    fn(case["crit"], case["x"], case["n_ctx"], case["w_a"], case["w_b"], case["k"], outs[0],
       outs[1] if len(outs) > 1 else None, hq, hkv, hd)
    return outs


def _other_library_work():
    """Kernels of other entries first (a small FFN block step: estimator with a workspace,
    selection, sparse GEMMs, LoRA backward), so the case where the fixed array follows other
    work on the device is exercised inside this test, not only through collection order."""
    import numpy as np  # noqa: F401
    from contextual_sparsity_lora_b200 import blocks, inputs
    T, C, D, F, r, k = 256, 192, 256, 512, 16, 8
    gen = inputs.generator(9)
    w = [inputs.spectral_weight(a, b, 0.5, k, gen, "cpu", torch.float64) for a, b in ((F, D), (F, D), (D, F))]
    lo = [inputs.lora_pair(a, b, r, 0.02, gen) for a, b in ((F, D), (F, D), (D, F))]
    blk = blocks.FFNBlock(*w, *lo, 2.0, k, T, C, 0.5, "cuda")
    x = inputs.activations_student_t(T, D, 4, 0.01, 30.0, gen).cuda()
    blk.step(x, torch.randn(T, D, generator=gen).to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    assert blk.read_device_flag() == 0


def _memory_state():
    torch.cuda.synchronize()
    free, _ = torch.cuda.mem_get_info()
    return free, torch.cuda.memory_allocated(), torch.cuda.memory_reserved()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_consecutive_calls():
    """Scores equal to the workspace entry's, bit for bit, on calls in a row over new inputs and
    differently sized scratch layouts; and the calls allocate nothing: device free memory (as the
    driver reports it) and torch's allocator counters are unchanged across them."""
    _other_library_work()
    ws = B.Workspace()
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")

    def with_ws(crit, x, n_ctx, w_a, w_b, k, s, sv, hq, hkv, hd):
        B.sl_svd_estimate(ws, crit, x, n_ctx, w_a, w_b, k, s, scores_v=sv, n_q_heads=hq, n_kv_heads=hkv,
                          head_dim=hd)

    needed = []

    def no_alloc(crit, x, n_ctx, w_a, w_b, k, s, sv, hq, hkv, hd):
        needed.append(B.sl_svd_estimate_noalloc(crit, x, n_ctx, w_a, w_b, k, s, scores_v=sv, n_q_heads=hq,
                                                n_kv_heads=hkv, head_dim=hd, device_flag=flag))

    cases = [_ffn_case(1), _attn_case(2), _ffn_case(3), _l2_fp32_case(4), _attn_case(5)]
    wants = [_scores(c, with_ws) for c in cases]
    outs = [[torch.full((n,), float("nan"), device="cuda") for n in c["outs"]] for c in cases]

    def run(case, out):
        for o in out:
            o.fill_(float("nan"))
        hq, hkv, hd = case["heads"]
        no_alloc(case["crit"], case["x"], case["n_ctx"], case["w_a"], case["w_b"], case["k"], out[0],
                 out[1] if len(out) > 1 else None, hq, hkv, hd)

    # first round: every kernel involved has been loaded and run once
    for case, out in zip(cases, outs):
        run(case, out)
    # two more rounds of consecutive calls on the shared array; the results and device flags are
    # copied into buffers allocated beforehand, and compared only after the second snapshot, so
    # that nothing in between allocates on the test's side either
    kept = [[[torch.empty_like(o) for o in out] for out in outs] for _ in range(2)]
    flags = torch.full((2, len(cases)), -1, dtype=torch.int32, device="cuda")
    before = _memory_state()
    for rep in range(2):
        for i, (case, out) in enumerate(zip(cases, outs)):
            flag.fill_(-1)
            run(case, out)
            flags[rep, i].copy_(flag[0])
            for dst, src in zip(kept[rep][i], out):
                dst.copy_(src)
    after = _memory_state()
    assert after == before, f"memory changed across the calls: {before} -> {after}"
    assert bool((flags == 0).all()), f"device flags {flags.tolist()}"
    for rep in range(2):
        for got, want in zip(kept[rep], wants):
            for g_, w_ in zip(got, want):
                assert torch.isfinite(g_).all()
                assert _rel(g_, w_) < FP32_TOL
                assert torch.equal(g_, w_)  # same kernels, fixed-order sums
    assert all(0 < n <= 8 << 20 for n in needed)
    assert len(set(needed)) > 1
