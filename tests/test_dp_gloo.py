"""The data-parallel path with two gloo ranks on CPU.

Each rank takes its shard of the tokens, runs the fp64 oracle's backward on
it, and the adapter gradients are summed with lora_linear_layer_b200.dp's
all-reduce.  The summed dA, dB and the concatenated dX shards must equal the
oracle on the whole batch, and the timing reduction must return the maximum
over ranks.  The partials are summed in fp64, and in fp32 as the GPU path
does (lora_bwd_ex with fp32 gradients, summed before any rounding).  No GPU
is involved."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, M, q, dtype="float64", async_op=False):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle as O
    import workloads as WL
    from lora_linear_layer_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sh = WL.LayerShape(M, 48, 40, 8, 12.0)
        t = WL.make_layer_inputs(sh, seed=3, with_dy=True)          # same full batch on every rank
        f = lambda x: O.bf16_bits_to_f64(WL.bf16_bits(x))          # noqa: E731
        X, W, A, B, dY = (f(t[k]) for k in ("X", "W", "A", "B", "dY"))
        b, e = dp.shard_rows(M, world, rank)
        dX, dA, dB = O.lora_backward(X[b:e], W, A, B, dY[b:e], sh.alpha)
        dA_t = torch.from_numpy(dA.astype(dtype))
        dB_t = torch.from_numpy(dB.astype(dtype))
        works = dp.allreduce_adapter_grads(dA_t, dB_t, async_op=async_op)
        for w in works or []:
            w.wait()
        times = dp.max_over_ranks([1.0 + rank, 5.0 - rank])
        q.put((rank, b, e, dX, dA_t.numpy(), dB_t.numpy(), times))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,dtype,async_op", [(16, "float64", False), (23, "float64", False), (23, "float32", False),
                                              (23, "float32", True)])
def test_two_rank_backward_equals_full_batch(M, dtype, async_op):
    sys.path.insert(0, ROOT)
    import oracle as O
    import workloads as WL
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, M, q, dtype, async_op)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sh = WL.LayerShape(M, 48, 40, 8, 12.0)
    t = WL.make_layer_inputs(sh, seed=3, with_dy=True)
    f = lambda x: O.bf16_bits_to_f64(WL.bf16_bits(x))              # noqa: E731
    dX, dA, dB = O.lora_backward(*(f(t[k]) for k in ("X", "W", "A", "B", "dY")), sh.alpha)
    # shards cover the rows exactly once, in order
    assert [(r[1], r[2]) for r in res] == [(0, (M + 1) // 2), ((M + 1) // 2, M)]
    np.testing.assert_allclose(np.concatenate([r[3] for r in res]), dX, rtol=1e-12, atol=1e-12)
    tol = 1e-12 if dtype == "float64" else 2e-6    # a few fp32 roundings
    for r in res:   # every rank holds the full-batch sums after the all-reduce
        assert r[4].dtype == np.dtype(dtype) and r[5].dtype == np.dtype(dtype)
        np.testing.assert_allclose(r[4], dA, rtol=tol, atol=tol * np.abs(dA).max())
        np.testing.assert_allclose(r[5], dB, rtol=tol, atol=tol * np.abs(dB).max())
        assert r[6] == [2.0, 5.0]


def test_shard_rows_partition():
    sys.path.insert(0, ROOT)
    from lora_linear_layer_b200 import dp
    for M in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_rows(M, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(8, 2, 2)
