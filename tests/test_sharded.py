"""The sharded one-layer path on CPU: token shards summed by an all-reduce,
row shards quantized independently and gathered in rank order.

The ranks are gloo processes; each rank's compute steps are the oracle's, so
what is under test is the host logic of ``sharded.py`` (shard ranges, the
step sequence, the padded row gather).  The result must equal the oracle run
on the whole layer in one process.
"""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from post_weight_quantization_26_b200 import sharded  # noqa: E402


@pytest.mark.parametrize("n,world", [(10, 3), (0, 2), (2, 4), (4096, 8), (7, 1), (262144, 6)])
def test_shards_cover_the_range_once_and_balance(n, world):
    ranges = [sharded.shard(n, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_shard_rejects_bad_requests():
    for args in [(5, 0, 0), (5, 2, 2), (-1, 2, 0), (5, 2, -1)]:
        with pytest.raises(ValueError):
            sharded.shard(*args)


SPEC = dict(d_row=50, d_col=256, n_tokens=3001, group=64, sym=False, block=128, bits=4)


def _problem():
    from post_weight_quantization_26_b200 import synth
    spec = synth.tiny_spec(SPEC["d_row"], SPEC["d_col"], SPEC["n_tokens"], seed=17)
    return (synth.gen_tokens(spec).float().numpy().astype(np.float64),
            synth.gen_weight(spec).numpy().astype(np.float64))


def _oracle_steps(world):
    import torch
    import torch.distributed as dist

    from oracle import gptq_oracle as O

    def zeros_h(d):
        return torch.zeros((d, d), dtype=torch.float64)

    def accumulate(H, x):
        if len(x):
            H += torch.from_numpy(O.hessian(x))

    def allreduce_sum(H):
        if world > 1:
            dist.all_reduce(H, op=dist.ReduceOp.SUM)

    def prepare(H):
        hd, dead = O.dampen(H.numpy(), 0.01)
        return O.hinv_cholesky_upper(hd), dead

    def quantize(w, u, dead):
        codes, s, z, _, _ = O.gptq_quantize(w, u, SPEC["bits"], SPEC["group"], SPEC["sym"],
                                            SPEC["block"], dead=dead, dtype=np.float32)
        return (torch.from_numpy(np.asarray(codes, np.int64)),
                torch.from_numpy(np.asarray(s, np.float64)),
                torch.from_numpy(np.asarray(z, np.int64)))

    def allgather_rows(t):
        return sharded.gather_padded(t, world, "cpu")

    return sharded.Steps(zeros_h, accumulate, allreduce_sum, prepare, quantize, allgather_rows)


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    if world > 1:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=timedelta(seconds=120))
    try:
        x, w = _problem()
        t0, t1 = sharded.shard(len(x), world, rank)
        r0, r1 = sharded.shard(len(w), world, rank)
        codes, s, z, H = sharded.quantize_layer_sharded(
            _oracle_steps(world), x[t0:t1], w[r0:r1], x.shape[1])
        q.put((rank, codes.numpy(), s.numpy(), z.numpy(), H.numpy(), (t0, t1), (r0, r1)))
    finally:
        if world > 1:
            dist.destroy_process_group()


def _run(world):
    if world == 1:
        class Q(list):
            put = list.append
        q = Q()
        _rank(0, 1, 0, q)
        return q
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


@pytest.fixture(scope="module")
def whole_layer():
    from oracle import gptq_oracle as O
    x, w = _problem()
    h = O.hessian(x)
    ref = O.gptq(w, h, bits=SPEC["bits"], group=SPEC["group"], sym=SPEC["sym"],
                 block=SPEC["block"], damp_rel=0.01, dtype=np.float32)
    return h, ref


@pytest.mark.parametrize("world", [1, 2, 3])
def test_sharded_layer_equals_the_whole_layer(world, whole_layer):
    h_ref, ref = whole_layer
    res = _run(world)
    # token shards tile the calibration set, row shards tile W
    assert [r[5] for r in res] == [sharded.shard(SPEC["n_tokens"], world, k) for k in range(world)]
    assert [r[6] for r in res] == [sharded.shard(SPEC["d_row"], world, k) for k in range(world)]
    for rank, codes, s, z, H, _, _ in res:
        # every rank holds the full H (only the summation order differs) and
        # the gathered outputs of every rank, in rank order
        np.testing.assert_allclose(H, h_ref, rtol=1e-12, atol=1e-9)
        assert codes.shape == (SPEC["d_row"], SPEC["d_col"])
        assert np.array_equal(codes, ref["codes"])
        assert np.array_equal(z, ref["zeros"])
        np.testing.assert_allclose(s, ref["scales"], rtol=1e-12)
