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


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_local_ring_matches_whole_sequence(world, causal, layout):
    q, k, v, dO = _inputs(10 + world)
    got = ring.local_ring_attention(q, k, v, dO, causal, SCALE, world, ops=OracleOps(),
                                    layout=layout)
    for g, r in zip(got, _reference(q, k, v, dO, causal)):
        _close(g, r)


class _CountingOps(OracleOps):
    """Counts the (query, key) pairs each virtual rank attends over."""

    def __init__(self):
        self.pairs = 0

    def _count(self, q, causal):
        n = q.shape[2]
        self.pairs += {0: n * n, 1: n * (n + 1) // 2, 2: n * (n - 1) // 2}[int(causal)]

    def fwd(self, q, k, v, causal, scale):
        self._count(q, causal)
        return super().fwd(q, k, v, causal, scale)


@pytest.mark.parametrize("world", [2, 4, 6])
def test_striped_causal_ring_is_balanced(world):
    """Under the causal mask the contiguous layout gives rank r work for r + 1
    shard pairs; the striped one gives rank r G n (n - 1) / 2 + (r + 1) n
    (query, key) pairs -- equal to within (G - 1) n, against n^2 per block --
    and the total over the ranks is the whole sequence's."""
    n = 8
    g = torch.Generator().manual_seed(3)
    q, k, v, dO = (torch.randn(1, 1, n * world, 4, generator=g, dtype=torch.float64)
                   for _ in range(4))
    work = {}
    for layout in ring.LAYOUTS:
        ops = [_CountingOps() for _ in range(world)]
        ring.local_ring_attention(q, k, v, dO, True, SCALE, world, ops=ops, layout=layout)
        work[layout] = [o.pairs for o in ops]
    N = n * world
    assert sum(work["striped"]) == sum(work["contiguous"]) == N * (N + 1) // 2
    assert work["striped"] == [world * n * (n - 1) // 2 + (r + 1) * n for r in range(world)]
    assert work["contiguous"] == [r * n * n + n * (n + 1) // 2 for r in range(world)]
    # striped: G half blocks per rank, against G - 1/2 whole blocks for the last
    # contiguous rank
    assert max(work["striped"]) <= world * n * (n + 1) // 2


def test_pair_masks():
    assert [ring.pair_mask(True, "striped", 2, s) for s in range(4)] == [1, 1, 1, 2]
    assert [ring.pair_mask(True, "contiguous", 2, s) for s in range(4)] == [0, 0, 1, None]
    assert ring.pair_mask(False, "striped", 0, 3) == 0
    with pytest.raises(ValueError):
        ring.pair_mask(True, "zigzag", 0, 0)


def test_local_ring_rejects_uneven_shards():
    q, k, v, dO = _inputs(1)
    with pytest.raises(ValueError):
        ring.local_ring_attention(q, k, v, dO, True, SCALE, 5, ops=OracleOps())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, layout, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, dO = _inputs(77)
        sl = _my_positions(rank, world, layout)
        mine = [t[:, :, sl].contiguous() for t in (q, k, v, dO)]
        o, lse = ring.run_nccl(ring.forward_program(mine[0], mine[1], mine[2], causal, SCALE,
                                                    rank, world, OracleOps(), layout))
        dq, dk, dv = ring.run_nccl(ring.backward_program(mine[0], mine[1], mine[2], o, lse,
                                                         mine[3], causal, SCALE, rank, world,
                                                         OracleOps(), layout))
        # the caller's shards are only read (received blocks go to buffers
        # of the ring's own)
        untouched = all(torch.equal(a, b[:, :, sl]) for a, b in zip(mine, (q, k, v, dO)))
        out[rank] = [t.numpy() for t in (o, lse, dq, dk, dv)] + [untouched]
    finally:
        dist.destroy_process_group()


def _my_positions(rank, world, layout):
    n = N // world
    return slice(rank, N, world) if layout == "striped" else slice(rank * n, (rank + 1) * n)


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_gloo_ring_matches_whole_sequence(world, causal, layout):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, causal, layout, out), nprocs=world, join=True)
        res = dict(out)
    q, k, v, dO = _inputs(77)
    ref = _reference(q, k, v, dO, causal)
    for rank in range(world):
        sl = _my_positions(rank, world, layout)
        assert res[rank][-1], "the ring wrote into the caller's input shards"
        for g, r in zip(res[rank][:-1], ref):
            _close(g, r[:, :, sl] if r.ndim == 4 else r[:, :, sl])
