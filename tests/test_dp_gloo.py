"""Data-parallel host logic on the CPU: token sharding and the weight-gradient
all-reduce, with two gloo ranks.  Each rank computes the weight gradient of
its token shard with the oracle; after the all-reduce every rank must hold
the full-token result (exactly, on inputs whose quantisation is exact)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_blockwise_scaled_b200.dp import shard_tokens


def test_shard_tokens_covers_whole_blocks():
    for tokens in (128, 1024, 16384, 128 * 7):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_tokens(tokens, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == tokens
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            assert all((s0 % 128 == 0) and (s1 % 128 == 0) for s0, s1 in spans)
            sizes = [s1 - s0 for s0, s1 in spans]
            assert max(sizes) - min(sizes) <= 128
    with pytest.raises(ValueError):
        shard_tokens(100, 0, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import oracle
    from fp8_blockwise_scaled_b200.dp import allreduce_weight_grads, shard_tokens
    from tests.oracle_pins import exact_case
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tokens, n_out, n_in = 640, 128, 256
        rng = np.random.default_rng(5)             # same inputs on every rank
        dy, _ = exact_case(rng, tokens, n_out, "col")
        x, _ = exact_case(rng, tokens, n_in, "col")
        t0, t1 = shard_tokens(tokens, rank, world)
        qa, sa = oracle.quantize_act_colwise_t(dy[t0:t1])
        qb, sb = oracle.quantize_act_colwise_t(x[t0:t1])
        part = torch.from_numpy(oracle.gemm(oracle.WGRAD, qa, sa, qb, sb))
        allreduce_weight_grads([part])
        qa, sa = oracle.quantize_act_colwise_t(dy)
        qb, sb = oracle.quantize_act_colwise_t(x)
        full = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)
        q.put((rank, bool(np.array_equal(part.numpy(), full)), (t0, t1)))
    finally:
        dist.destroy_process_group()


def test_weight_gradient_allreduce_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert all(ok for _, ok, _ in results)
    assert results[0][2] == (0, 384) and results[1][2] == (384, 640)
