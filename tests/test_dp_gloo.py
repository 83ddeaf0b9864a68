"""Data-parallel host logic on CPU: two gloo ranks, no GPU.

Each rank takes its shard of the tokens, computes its LoRA gradients with the
oracle, writes them into a GradBucket and all-reduces it.  The sum over ranks
must equal the oracle's gradients of the whole batch, since dA = s V^T X and
dB = s dY^T U are sums over tokens.  max_over_ranks must return the largest
rank's value on every rank.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_nf4_quantized_17_b200 import dp

N, K, R, M, ALPHA = 24, 128, 4, 11, 8.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w_hat = oracle.compute_weight(oracle.quantize(w, 64, 256)).reshape(N, K)
    a = rng.standard_normal((R, K)) / np.sqrt(R)
    b = rng.standard_normal((N, R)) * 0.05
    x = rng.standard_normal((M, K))
    dy = rng.standard_normal((M, N))
    return w_hat, a, b, x, dy


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_hat, a, b, x, dy = _problem()
        lo, hi = dp.token_shard(M, rank, world)
        _, da, db = oracle.linear_bwd(w_hat, a, b, ALPHA, x[lo:hi], dy[lo:hi])
        bucket = dp.GradBucket(R, K, N, "cpu")
        bucket.dA.copy_(torch.from_numpy(np.asarray(da, np.float32)))
        bucket.dB.copy_(torch.from_numpy(np.asarray(db, np.float32)))
        bucket.allreduce()
        slowest = dp.max_over_ranks(10.0 + rank, "cpu")
        results[rank] = (bucket.dA.double().numpy(), bucket.dB.double().numpy(), slowest)
    finally:
        dist.destroy_process_group()


def _rank_entry(rank, world, port, queue):
    results = {}
    _rank_main(rank, world, port, results)
    queue.put((rank, results[rank]))


@pytest.mark.parametrize("world", [2])
def test_gradient_allreduce_equals_full_batch(world):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_entry, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, res = queue.get(timeout=120)
        got[rank] = res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w_hat, a, b, x, dy = _problem()
    _, da_ref, db_ref = oracle.linear_bwd(w_hat, a, b, ALPHA, x, dy)
    for rank in range(world):
        da, db, slowest = got[rank]
        # fp32 storage of each rank's part and an fp32 sum: relative 1e-6
        np.testing.assert_allclose(da, da_ref, rtol=1e-5, atol=1e-6 * np.abs(da_ref).max())
        np.testing.assert_allclose(db, db_ref, rtol=1e-5, atol=1e-6 * np.abs(db_ref).max())
        assert slowest == 10.0 + (world - 1)
    # every rank holds the same gradient after the exchange
    assert np.array_equal(got[0][0], got[1][0]) and np.array_equal(got[0][1], got[1][1])


# a small stack: 3 layers x 3 linears of different shapes (r, d_in, d_out)
STACK = [(4, 128, 24), (4, 64, 128), (8, 128, 64)]
LAYERS = 3
M_STACK = 13


def _stack_problem():
    rng = np.random.default_rng(11)
    layers = []
    for _ in range(LAYERS):
        row = []
        for r, k, n in STACK:
            w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
            w_hat = oracle.compute_weight(oracle.quantize(w, 64, 256)).reshape(n, k)
            row.append((w_hat, rng.standard_normal((r, k)) / np.sqrt(r),
                        rng.standard_normal((n, r)) * 0.05, rng.standard_normal((M_STACK, k)),
                        rng.standard_normal((M_STACK, n))))
        layers.append(row)
    return layers


def _stack_rank_main(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layers = _stack_problem()
        lo, hi = dp.token_shard(M_STACK, rank, world)
        buckets = [dp.LayerBucket(STACK, "cpu") for _ in range(LAYERS)]
        works = []
        # the bench's order: backward from the last layer down, each layer's
        # exchange started as soon as its gradients are written
        for l in reversed(range(LAYERS)):
            for j in reversed(range(len(STACK))):
                w_hat, a, b, x, dy = layers[l][j]
                _, da, db = oracle.linear_bwd(w_hat, a, b, ALPHA, x[lo:hi], dy[lo:hi])
                dA, dB = buckets[l].views[j]
                dA.copy_(torch.from_numpy(np.asarray(da, np.float32)))
                dB.copy_(torch.from_numpy(np.asarray(db, np.float32)))
            works.append(buckets[l].allreduce(async_op=True))
        for wk in works:
            wk.wait()
        queue.put((rank, [[(v[0].double().numpy(), v[1].double().numpy()) for v in bk.views]
                          for bk in buckets]))
    finally:
        dist.destroy_process_group()


def test_layer_buckets_exchanged_per_layer_equal_full_batch():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_stack_rank_main, args=(r, world, port, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, res = queue.get(timeout=120)
        got[rank] = res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    layers = _stack_problem()
    for l in range(LAYERS):
        for j in range(len(STACK)):
            w_hat, a, b, x, dy = layers[l][j]
            _, da_ref, db_ref = oracle.linear_bwd(w_hat, a, b, ALPHA, x, dy)
            for rank in range(world):
                da, db = got[rank][l][j]
                np.testing.assert_allclose(da, da_ref, rtol=1e-5, atol=1e-6 * np.abs(da_ref).max())
                np.testing.assert_allclose(db, db_ref, rtol=1e-5, atol=1e-6 * np.abs(db_ref).max())
            assert np.array_equal(got[0][l][j][0], got[1][l][j][0])


def test_layer_bucket_layout():
    bk = dp.LayerBucket(STACK + [(64, 8192, 22016)], "cpu")
    base = bk.flat.data_ptr()
    ends = []
    for (r, k, n), (dA, dB) in zip(STACK + [(64, 8192, 22016)], bk.views):
        assert dA.shape == (r, k) and dB.shape == (n, r)
        assert dA.is_contiguous() and dB.is_contiguous()
        for v in (dA, dB):
            assert (v.data_ptr() - base) % 256 == 0
            ends.append((v.data_ptr() - base, v.data_ptr() - base + 4 * v.numel()))
    ends.sort()
    for (a0, a1), (b0, b1) in zip(ends, ends[1:]):
        assert a1 <= b0  # disjoint, in order
    assert ends[-1][1] <= 4 * bk.flat.numel()
    # one rank: no collective, nothing to wait for
    assert bk.allreduce(async_op=True) is None


@pytest.mark.parametrize("total,world", [(4096, 2), (11, 2), (11, 4), (3, 8), (0, 2), (8192, 8)])
def test_token_shards_partition_the_batch(total, world):
    spans = [dp.token_shard(total, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == total
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_bucket_views_are_aligned_and_disjoint():
    bk = dp.GradBucket(16, 4096, 11008, "cpu")
    assert bk.dA.shape == (16, 4096) and bk.dB.shape == (11008, 16)
    assert bk.dA.is_contiguous() and bk.dB.is_contiguous()
    assert (bk.dB.data_ptr() - bk.flat.data_ptr()) % 256 == 0
    bk.dA.fill_(1.0)
    assert torch.count_nonzero(bk.dB) == 0
    with pytest.raises(ValueError):
        dp.token_shard(10, 2, 2)


def test_adapter_optimizer_layout_matches_the_gradient_bucket():
    # AdapterAdamW keeps A and B (fp32 master and bf16 views) at the offsets of
    # GradBucket, so that one flat AdamW step pairs every parameter with its
    # gradient; checked on the host (no kernel runs here)
    from bit_nf4_quantized_17_b200.optim import AdapterAdamW

    r, d_in, d_out = 8, 200, 72
    A = torch.randn(r, d_in).to(torch.bfloat16)
    B = torch.randn(d_out, r).to(torch.bfloat16)
    opt = AdapterAdamW(A, B, lr=1e-3)
    bucket = opt.grad_bucket()
    assert opt.master.shape == bucket.flat.shape
    assert torch.equal(opt.A, A) and torch.equal(opt.B, B)
    na = r * d_in
    assert torch.equal(opt.master[:na].view(r, d_in), A.float())
    assert torch.equal(opt.master[bucket.off_b:bucket.off_b + d_out * r].view(d_out, r), B.float())
    assert opt.A.data_ptr() == opt.bf16.data_ptr()
    assert opt.B.data_ptr() == opt.bf16.data_ptr() + 2 * bucket.off_b
    assert bucket.dB.data_ptr() == bucket.flat.data_ptr() + 4 * bucket.off_b
