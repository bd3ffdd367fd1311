"""Data-parallel path on CPU: two gloo ranks.

Tokens are sharded over the ranks and the adapter gradients are summed: the
weight gradients of the LoRA adapters contract over the token index
(mbrenndoerfer.com QLoRA essay, section "Low-Rank Adaptation (LoRA)": the
adapters are the only trained parameters; "QLoRA: Efficient Finetuning of
Quantized LLMs", abstract: gradients flow through the frozen 4-bit weight
into them), so the sum over ranks of the shard gradients is the gradient of
the whole batch.  Each rank computes its shard's gradients with the float64
oracle; the exchange goes through the library's data-parallel helpers.
"""

import importlib.util
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

HERE = os.path.dirname(os.path.abspath(__file__))
DP_PATH = os.path.join(HERE, "..", "bit_nf4_quantized_16_b200", "dp.py")


def _load_dp():
    # the helpers import nothing from the library: load the file directly so
    # the test needs neither the built library nor a GPU
    spec = importlib.util.spec_from_file_location("qlora_dp", DP_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(seed=3, M=37, N=48, K=64, r=8):
    rng = np.random.default_rng(seed)
    return {
        "X": rng.standard_normal((M, K)),
        "W": rng.standard_normal((N, K)) * 0.02,
        "A": rng.standard_normal((r, K)) / r,
        "B": rng.standard_normal((N, r)) * 0.01,
        "dY": rng.standard_normal((M, N)),
        "s": 2.0,
    }


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.join(HERE, ".."))
        from oracle import linear as olin
        dp = _load_dp()
        c = _case()
        M = c["X"].shape[0]
        a, b = dp.shard_tokens(M, rank, world)
        _, dA, dB = olin.backward(c["X"][a:b], c["W"], c["A"], c["B"], c["s"], c["dY"][a:b])
        flat = torch.from_numpy(np.concatenate([dA.ravel(), dB.ravel()])).to(torch.float64)
        dp.allreduce_adapter_grads(flat)
        t = dp.max_over_ranks(1.5 + rank)   # a per-rank step time
        out[rank] = (flat.numpy().copy(), t, (a, b))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_shard_tokens_partition():
    dp = _load_dp()
    for M in (0, 1, 7, 37, 4096):
        for world in (1, 2, 3, 8):
            shards = [dp.shard_tokens(M, r, world) for r in range(world)]
            assert shards[0][0] == 0 and shards[-1][1] == M
            for (a0, b0), (a1, b1) in zip(shards, shards[1:]):
                assert b0 == a1
            sizes = [b - a for a, b in shards]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_sum_to_the_full_batch_gradient():
    from oracle import linear as olin
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    c = _case()
    _, dA, dB = olin.backward(c["X"], c["W"], c["A"], c["B"], c["s"], c["dY"])
    want = np.concatenate([dA.ravel(), dB.ravel()])
    shards = []
    for rank in range(world):
        got, t, shard = out[rank]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
        assert t == 2.5          # max over ranks of 1.5 + rank
        shards.append(shard)
    assert shards == [(0, 19), (19, 37)]


def _worker_overlapped(rank, world, port, out):
    """Three linears' backward in reverse order; each linear's dA, dB are
    handed to the overlapped reducer as soon as they exist (views of one
    flattened buffer), and the reducer is waited on once at the end."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.join(HERE, ".."))
        from oracle import linear as olin
        dp = _load_dp()
        cases = [_case(seed=10 + i, N=48 + 8 * i, K=64 + 16 * i) for i in range(3)]
        sizes = [c["A"].size + c["B"].size for c in cases]
        flat = torch.zeros(sum(sizes), dtype=torch.float64)
        offs = np.cumsum([0] + sizes)
        red = dp.OverlappedGradSum()
        for i in reversed(range(3)):
            c = cases[i]
            a, b = dp.shard_tokens(c["X"].shape[0], rank, world)
            _, dA, dB = olin.backward(c["X"][a:b], c["W"], c["A"], c["B"], c["s"], c["dY"][a:b])
            view = flat[offs[i]: offs[i + 1]]
            view.copy_(torch.from_numpy(np.concatenate([dA.ravel(), dB.ravel()])))
            red.ready(view)
        red.wait()
        out[rank] = (flat.numpy().copy(), len(red.pending))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_overlapped_reduction_sums_every_linear():
    from oracle import linear as olin
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker_overlapped, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    want = []
    for i in range(3):
        c = _case(seed=10 + i, N=48 + 8 * i, K=64 + 16 * i)
        _, dA, dB = olin.backward(c["X"], c["W"], c["A"], c["B"], c["s"], c["dY"])
        want.append(np.concatenate([dA.ravel(), dB.ravel()]))
    want = np.concatenate(want)
    for rank in range(world):
        got, pending = out[rank]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
        assert pending == 0


def test_overlapped_reduction_is_a_no_op_on_one_rank():
    dp = _load_dp()
    red = dp.OverlappedGradSum()
    buf = torch.arange(6, dtype=torch.float32)
    red.ready(buf)
    red.wait()
    assert torch.equal(buf, torch.arange(6, dtype=torch.float32)) and red.pending == []
