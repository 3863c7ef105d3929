"""Data-parallel host logic on the CPU: token sharding and the weight-gradient
all-reduce, with two gloo ranks.  Each rank computes the weight gradient of
its token shard with the oracle and hands it over in the product's types: an
fp32 partial (what the WGRAD GEMM writes with fp32 output) and a bf16 result
buffer.  After the fp32 all-reduce and the single rounding every rank must
hold the full-token result rounded to bf16 (exactly, on inputs whose
quantisation and partial sums are exact)."""
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
        part = torch.from_numpy(oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)).to(torch.float32)
        out = torch.empty(part.shape, dtype=torch.bfloat16)
        allreduce_weight_grads([(part, out)], round_fn=lambda a, b: b.copy_(a.to(torch.bfloat16)))
        qa, sa = oracle.quantize_act_colwise_t(dy)
        qb, sb = oracle.quantize_act_colwise_t(x)
        full = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)
        # Every rank holds the fp32 sum of both ranks' fp32 partials (the same on both ranks,
        # within the fp32 rounding of the partials and of their sum from the exact full-token
        # result), rounded once to bf16.
        shares = []
        for r in range(world):
            s0, s1 = shard_tokens(tokens, r, world)
            a, b = oracle.quantize_act_colwise_t(dy[s0:s1]), oracle.quantize_act_colwise_t(x[s0:s1])
            shares.append(oracle.gemm(oracle.WGRAD, *a, *b).astype(np.float32))
        want32 = shares[0] + shares[1]
        ok = (bool(np.array_equal(part.numpy(), want32))
              and torch.equal(out, torch.from_numpy(want32).to(torch.bfloat16))
              and bool(np.all(np.abs(want32 - full) <= 2.0**-22 * (np.abs(shares[0]) + np.abs(shares[1])))))
        wrong_type = False
        try:
            allreduce_weight_grads([(out.float(), out.float())], round_fn=lambda a, b: None)
        except ValueError:
            wrong_type = True
        q.put((rank, ok and wrong_type, (t0, t1)))
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
