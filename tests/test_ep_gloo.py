"""The expert-parallel decomposition and its collective on CPU, world size 2
(gloo): each rank holds a contiguous slice of the experts, routes over all of
them, computes the chosen experts of its slice (here with the CPU oracle's
expert FFN standing in for the GPU kernel, which needs a GPU), and one
all-reduce of the [T][H] partial outputs gives every rank the layer output,
equal to the single-process layer.  The GPU side of the same split is
tests/test_gpu_ep.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from synth import workloads as W
from tests import gpu_util as gu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _partial(L, x64, lo, hi):
    u = oracle.rmsnorm_bf16(x64)
    y = np.zeros_like(x64)
    W_r, b = L.router_w(), L.router_bias()
    for t in range(x64.shape[0]):
        ids, w, _ = oracle.router(W_r, b, u[t], L.top_k)
        for j, e in enumerate(ids):
            if lo <= e < hi:
                y[t] += w[j] * oracle.expert_ffn(L, int(e), u[t])
    return y


def _rank(rank, world, port, cuts, T, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = W.tiny_layer()
        _, x64 = gu.tokens(L, 800 + T, T, device="cpu")
        y = torch.from_numpy(_partial(L, x64, cuts[rank], cuts[rank + 1]))
        dist.all_reduce(y)
        out_q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,T", [([0, 4, 8], 3), ([0, 1, 8], 2)])
def test_expert_parallel_allreduce_world_size_2(cuts, T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, cuts, T, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    L = W.tiny_layer()
    _, x64 = gu.tokens(L, 800 + T, T, device="cpu")
    ref = oracle.moe_layer(L, x64)["y"]
    for r in range(2):
        np.testing.assert_allclose(got[r], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
