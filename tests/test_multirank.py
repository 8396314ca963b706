"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (one process each, as
torchrun would start them) go through bench.py's rendezvous, barrier and max-over-ranks
reduction, which the N-GPU timing uses (each rank times its own replica of the step; the
job's time is the slowest rank's)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    # each rank reports a different time; every rank must see the slowest one
    t = bench.max_over_ranks(10.0 + 5.0 * rank, w, "cpu")
    bench.barrier(w)
    out[rank] = t
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    bench.barrier(1)


def _dp_rank_main(rank, world, port, out):
    """Two ranks, each with half of the batch's sequences: the rank-local statistics of the
    criteria (oracle), summed by the blocks' own `DataParallel` object (the fp64 all-reduce the
    library's blocks issue), give every rank the scores and the index sets of the whole batch."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from contextual_sparsity_lora_b200 import blocks, inputs

    dist.init_process_group("gloo")
    dp = blocks.DataParallel()
    assert dp.world == world and dp.active
    gen = inputs.generator(3)
    D, F, hq, hkv, hd, k = 64, 96, 4, 2, 8, 8
    x = inputs.activations_student_t(8 * 16, D, 4, 0.03, 30.0, gen)  # 8 sequences of 16 tokens
    ctx = np.tile(np.arange(16) < 12, 8)
    fac = {n: oracle.svd_factors(inputs.spectral_weight(o, D, 0.5, k, gen, "cpu", torch.float64,
                                                        torch.float32).W, k)[:2]
           for n, o in (("gate", F), ("up", F), ("q", hq * hd), ("k", hkv * hd), ("v", hkv * hd))}
    X = oracle.f64(x)

    def stats(rows):
        Xc = X[rows & ctx]
        G, U = oracle.estimate(Xc, *fac["gate"]), oracle.estimate(Xc, *fac["up"])
        Q, K, V = (oracle.estimate(Xc, *fac[n]) for n in "qkv")
        return np.concatenate([oracle.sumsq(oracle.silu(G) * U), oracle.sumsq(Q), oracle.sumsq(K),
                               oracle.sumsq(V)])

    mine = np.arange(8 * 16) // 64 == rank  # rank r holds sequences 4r .. 4r + 3
    t = torch.tensor(stats(mine), dtype=torch.float64)
    dp.all_reduce(t)  # sum over the ranks
    s = t.numpy()
    f2, q2, k2, v2 = np.split(s, np.cumsum([F, hq * hd, hkv * hd]))
    s_ffn = np.sqrt(f2)
    s_qk = oracle.qk_from_sumsq(q2, k2, hq, hkv, hd)
    s_v = np.sqrt(v2)
    sel = [oracle.select_top(v, oracle.keep_count(0.5, v.shape[0])) for v in (s_ffn, s_qk, s_v)]
    out[rank] = (s_ffn, s_qk, s_v, sel)
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_data_parallel_ranks_select_the_batch_index_sets():
    import numpy as np

    import oracle
    from contextual_sparsity_lora_b200 import inputs
    import torch

    ctx_ = mp.get_context("spawn")
    with ctx_.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_dp_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    # both ranks agree exactly
    for a, b in zip(res[0][:3], res[1][:3]):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(res[0][3], res[1][3]):
        np.testing.assert_array_equal(a, b)
    # and equal the single-process criterion over the whole batch
    gen = inputs.generator(3)
    D, F, hq, hkv, hd, k = 64, 96, 4, 2, 8, 8
    x = inputs.activations_student_t(8 * 16, D, 4, 0.03, 30.0, gen)
    ctx = np.tile(np.arange(16) < 12, 8)
    fac = {n: oracle.svd_factors(inputs.spectral_weight(o, D, 0.5, k, gen, "cpu", torch.float64,
                                                        torch.float32).W, k)[:2]
           for n, o in (("gate", F), ("up", F), ("q", hq * hd), ("k", hkv * hd), ("v", hkv * hd))}
    s_ffn, _ = oracle.ffn_select(x, ctx, fac["gate"], fac["up"], 0.5)
    sel = oracle.attn_select(x, ctx, fac["q"], fac["k"], fac["v"], hq, hkv, hd, 0.5)
    np.testing.assert_allclose(res[0][0], s_ffn, rtol=1e-12)
    np.testing.assert_allclose(res[0][1], sel["s_qk"], rtol=1e-12)
    np.testing.assert_allclose(res[0][2], sel["s_v"], rtol=1e-12)
    np.testing.assert_array_equal(res[0][3][0], oracle.select_top(s_ffn, oracle.keep_count(0.5, F)))
    np.testing.assert_array_equal(res[0][3][1], sel["units_qk"])
    np.testing.assert_array_equal(res[0][3][2], sel["units_v"])


def _ref_rank_main(rank, world, port, out):
    """One rank of `torchrun ... bench.py --impl reference --gpus 2`: rank 0 prints the line."""
    import contextlib
    import io

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    # no --gpus flag: the line's n_gpus is the launch's world size
    sys.argv = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"]
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main()
    import torch.distributed as dist
    out[rank] = buf.getvalue()
    out[f"group_left_{rank}"] = not dist.is_initialized()


@pytest.mark.timeout(300)
def test_reference_arm_under_two_ranks_prints_once():
    import json

    ctx_ = mp.get_context("spawn")
    with ctx_.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_ref_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[1].strip() == ""
    lines = [l for l in res[0].splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert res["group_left_0"] and res["group_left_1"], "both ranks destroy the process group"


def _grad_rank_main(rank, world, port, out):
    """One rank's LoRA gradients in a block's flat buffer, summed by `DataParallel` (the one
    fp32 all-reduce per block after the backward)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    from contextual_sparsity_lora_b200 import blocks

    dist.init_process_group("gloo")
    dp = blocks.DataParallel()
    shapes = [(32, 100), (7, 9), (64, 32)]  # A of 32 x 100, an odd-sized block, B of 64 x 32
    buf = blocks._GradBuffer(shapes, "cpu")
    g = torch.Generator().manual_seed(100 + rank)
    mine = [torch.randn(*sh, generator=g) for sh in shapes]
    for v, m in zip(buf.views, mine):
        v.copy_(m)
    dp.all_reduce(buf.flat)
    out[rank] = ([m.numpy() for m in mine], [v.clone().numpy() for v in buf.views], list(buf.offsets),
                 [v.data_ptr() - buf.flat.data_ptr() for v in buf.views])
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_data_parallel_sums_the_flat_gradient_buffer():
    import numpy as np

    ctx_ = mp.get_context("spawn")
    with ctx_.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_grad_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    mine0, got0, offsets, byte_offsets = res[0]
    mine1, got1, _, _ = res[1]
    for a, b, c, d in zip(mine0, mine1, got0, got1):
        np.testing.assert_array_equal(c, d)  # every rank holds the same sums
        np.testing.assert_allclose(c, a + b, rtol=1e-6, atol=1e-6)
    # the views start on 64-element boundaries of the one flat buffer (one collective covers all)
    assert all(o % 64 == 0 for o in offsets) and offsets == sorted(offsets)
    assert byte_offsets == [4 * o for o in offsets]


def test_data_parallel_without_a_process_group_is_one_rank():
    import torch

    from contextual_sparsity_lora_b200 import blocks

    dp = blocks.DataParallel()
    assert dp.world == 1 and not dp.active
    t = torch.arange(5, dtype=torch.float64)
    dp.all_reduce(t)  # no collective: unchanged
    assert t.tolist() == [0.0, 1.0, 2.0, 3.0, 4.0]
