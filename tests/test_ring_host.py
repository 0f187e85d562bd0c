"""Host logic of sequence-sharded (ring) attention, without a GPU: the ring
schedule of exact_attention_109_b200.ring driven with the oracle's per-step
arithmetic must reproduce attention over the whole sequence -- run as G
virtual ranks in one process, and as two and three gloo ranks exchanging
key/value blocks and dK/dV accumulators point to point."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_attention_109_b200 import ring
from ring_oracle_ops import OracleOps

B, H, N, D_HEAD, SCALE = 1, 2, 24, 8, 0.3


def _inputs(seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, D_HEAD, generator=g, dtype=torch.float64) for _ in range(4)]


def _reference(q, k, v, dO, causal):
    o, lse = oracle.ref_fwd(q.numpy(), k.numpy(), v.numpy(), causal, SCALE)
    dq, dk, dv, _ = oracle.ref_bwd(q.numpy(), k.numpy(), v.numpy(), dO.numpy(), causal, SCALE)
    return o, lse, dq, dk, dv


def _close(a, b, tol=1e-5):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_local_ring_matches_whole_sequence(world, causal):
    q, k, v, dO = _inputs(10 + world)
    got = ring.local_ring_attention(q, k, v, dO, causal, SCALE, world, ops=OracleOps())
    for g, r in zip(got, _reference(q, k, v, dO, causal)):
        _close(g, r)


def test_local_ring_rejects_uneven_shards():
    q, k, v, dO = _inputs(1)
    with pytest.raises(ValueError):
        ring.local_ring_attention(q, k, v, dO, True, SCALE, 5, ops=OracleOps())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, dO = _inputs(77)
        n = N // world
        sl = slice(rank * n, (rank + 1) * n)
        mine = [t[:, :, sl].contiguous() for t in (q, k, v, dO)]
        o, lse = ring.run_nccl(ring.forward_program(mine[0], mine[1], mine[2], causal, SCALE,
                                                    rank, world, OracleOps()))
        dq, dk, dv = ring.run_nccl(ring.backward_program(mine[0], mine[1], mine[2], o, lse,
                                                         mine[3], causal, SCALE, rank, world,
                                                         OracleOps()))
        # the caller's shards are only read (received blocks go to buffers
        # of the ring's own)
        untouched = all(torch.equal(a, b[:, :, sl]) for a, b in zip(mine, (q, k, v, dO)))
        out[rank] = [t.numpy() for t in (o, lse, dq, dk, dv)] + [untouched]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_gloo_ring_matches_whole_sequence(world, causal):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, causal, out), nprocs=world, join=True)
        res = dict(out)
    q, k, v, dO = _inputs(77)
    ref = _reference(q, k, v, dO, causal)
    n = N // world
    for rank in range(world):
        sl = slice(rank * n, (rank + 1) * n)
        assert res[rank][-1], "the ring wrote into the caller's input shards"
        for g, r in zip(res[rank][:-1], ref):
            _close(g, r[:, :, sl] if r.ndim == 4 else r[:, :, sl])
