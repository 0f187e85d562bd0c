"""Sequence-sharded attention across devices (Ring Attention).

Ring Attention with Blockwise Transformers (abstract): the sequence is spread
over a ring of devices; each device keeps its block of queries while the
key/value blocks travel around the ring, the transfer of the next block
overlapping the blockwise attention on the current one, so the context length
grows with the number of devices.  Every (query shard, key/value shard) pair
is an ordinary attention problem of the shard length, computed by the CUDA
library (``fa_fwd`` / ``fa_bwd_main_accumulate``); the pairs' results are
folded together with the log-sum-exp rule (``fa_lse_merge``).

Layouts of the sequence over a ring of G ranks (every rank holds n = N / G
positions as q, k, v, dO, O [B, H, n, d] bf16 and LSE [B, H, n] fp32):

* "contiguous": rank r holds positions [r n, (r+1) n).  Under the causal mask
  key shard j is fully visible to query shard r when j < r, causal when
  j = r and skipped when j > r, so rank r computes r + 1 pairs and the last
  rank's G pairs are the ring's critical path.
* "striped": rank r holds positions r, r + G, r + 2G, ... (local row i is
  position i G + r).  Key j of shard s is then visible to query i of shard r
  iff j G + s <= i G + r: j <= i when s <= r, j < i when s > r.  Every pair is
  half a block of work -- causal with or without its diagonal -- so every
  rank computes the same G half blocks and the causal ring is balanced (the
  striped layout of "Striped Attention: Faster Ring Attention for Causal
  Transformers", Brandon et al., 2023; not on the pages, which give only the
  Ring Attention abstract).

Each rank's schedule is written once, as a generator (``forward_program`` /
``backward_program``) that yields at its exchange points:
``("start", sends, recvs)`` posts one step of the rotation -- every tensor in
``sends`` goes to the next rank, every tensor in ``recvs`` is filled from the
previous rank -- and ``("wait",)`` waits for everything posted.  Two runners
drive it: ``run_nccl`` with torch.distributed point-to-point operations (one
process per GPU; over NVLink / NVSwitch with NCCL), and ``run_local``, which
runs G virtual ranks in lockstep in one process and performs each rotation
as device-to-device copies (the same bytes a ring would move), for checking
the whole scheme on one GPU.

The forward sends key/value blocks before computing on the current ones, so
transfer and compute overlap.  In the backward the dK/dV accumulators travel
with their key/value block and are sent after the block's gradient is added;
after G rotations every rank holds its own shard's accumulators again.

This module only marshals buffers and orders calls; all arithmetic runs in
the CUDA library (an ``ops`` object may be substituted to exercise the
schedule on CPU in tests).
"""
from __future__ import annotations

import torch

from . import api as _api


# ---------------------------------------------------------------- compute ops


class CudaOps:
    """The per-step arithmetic, through the library's C ABI."""

    def fwd(self, q, k, v, causal, scale):
        return _api.attention_forward(q, k, v, causal, scale)

    def merge(self, o_acc, lse_acc, o_part, lse_part, o_out, init):
        rows = lse_acc.numel()
        st = _api.fa_lse_merge(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(),
                               lse_part.data_ptr(), o_out.data_ptr() if o_out is not None else 0,
                               rows, o_acc.shape[-1], int(init),
                               torch.cuda.current_stream(o_acc.device).cuda_stream)
        _api._check(st, "fa_lse_merge")

    def bwd_prepare(self, o, lse, dO):
        B, H, n, d = o.shape
        nbytes = _api.fa_bwd_workspace_size(B, H, n, d)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=o.device)
        st = _api.fa_bwd_preprocess(o.data_ptr(), lse.data_ptr(), dO.data_ptr(), B, H, n, d,
                                    ws.data_ptr(), nbytes,
                                    torch.cuda.current_stream(o.device).cuda_stream)
        _api._check(st, "fa_bwd_preprocess")
        return ws

    def bwd_accumulate(self, ws, q, k, v, dO, dk_acc, dv_acc, causal, scale):
        B, H, n, d = q.shape
        st = _api.fa_bwd_main_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), dO.data_ptr(),
                                         dk_acc.data_ptr(), dv_acc.data_ptr(), B, H, n, d,
                                         int(causal), scale, ws.data_ptr(), ws.numel(),
                                         torch.cuda.current_stream(q.device).cuda_stream)
        _api._check(st, "fa_bwd_main_accumulate")

    def bwd_finish(self, ws, q, scale):
        B, H, n, d = q.shape
        dq = torch.empty_like(q)
        st = _api.fa_bwd_dq_convert(dq.data_ptr(), B, H, n, d, scale, ws.data_ptr(), ws.numel(),
                                    torch.cuda.current_stream(q.device).cuda_stream)
        _api._check(st, "fa_bwd_dq_convert")
        return dq

    def to_bf16(self, x):
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
        st = _api.fa_convert_f32_bf16(x.data_ptr(), out.data_ptr(), x.numel(),
                                      torch.cuda.current_stream(x.device).cuda_stream)
        _api._check(st, "fa_convert_f32_bf16")
        return out


# ---------------------------------------------------------------- schedules


LAYOUTS = ("contiguous", "striped")


def pair_mask(causal: bool, layout: str, rank: int, shard: int):
    """Mask of the pair (query shard `rank`, key shard `shard`) as the
    library's `causal` argument -- 0 none, 1 causal (j <= i), 2 causal
    without the diagonal (j < i) -- or None when no key of the shard is
    visible (the pair is skipped)."""
    if layout not in LAYOUTS:
        raise ValueError(f"unknown ring layout {layout!r}")
    if not causal:
        return 0
    if layout == "striped":
        return 1 if shard <= rank else 2
    if shard < rank:
        return 0
    return 1 if shard == rank else None


def _last_visible_step(causal: bool, layout: str, rank: int, world: int) -> int:
    # step s holds key shard (rank - s) mod world; contiguous causal ranks see
    # s = 0..rank, every other case sees every step
    return rank if (causal and layout == "contiguous") else world - 1


def forward_program(q, k, v, causal: bool, scale: float, rank: int, world: int, ops=None,
                    layout: str = "contiguous"):
    """Rank `rank`'s forward: returns (O bf16, LSE fp32) of its query shard.
    Step 0 is the rank's own key shard, where every query row sees at least
    its own key, so the first partial result folded in has a finite LSE."""
    ops = ops or CudaOps()
    B, H, n, d = q.shape
    o_acc = torch.empty((B, H, n, d), dtype=torch.float32, device=q.device)
    lse_acc = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    o_out = torch.empty_like(q)
    # The caller's k, v are only ever sent; received blocks alternate between
    # two buffers of our own (one while only two ranks rotate).
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    cur = (k, v)
    last = _last_visible_step(causal, layout, rank, world)
    first = True
    for s in range(world):
        shard = (rank - s) % world
        if s < world - 1:
            nxt = bufs[s % 2]
            yield ("start", list(cur), list(nxt))
        mask = pair_mask(causal, layout, rank, shard)
        if mask is not None:
            o_p, l_p = ops.fwd(q, cur[0], cur[1], mask, scale)
            ops.merge(o_acc, lse_acc, o_p, l_p, o_out if s == last else None, first)
            first = False
        if s < world - 1:
            yield ("wait",)
            cur = nxt
    return o_out, lse_acc


def backward_program(q, k, v, o, lse, dO, causal: bool, scale: float, rank: int, world: int,
                     ops=None, layout: str = "contiguous"):
    """Rank `rank`'s backward: returns (dQ, dK, dV) bf16 of its shards, given
    its query shard's final O and LSE (from forward_program)."""
    ops = ops or CudaOps()
    ws = ops.bwd_prepare(o, lse, dO)
    dk_acc = torch.zeros(k.shape, dtype=torch.float32, device=k.device)
    dv_acc = torch.zeros(v.shape, dtype=torch.float32, device=v.device)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    kv = (k, v)  # the caller's k, v are only sent, as in the forward
    acc = (dk_acc, dv_acc)
    acc_n = (torch.empty_like(dk_acc), torch.empty_like(dv_acc)) if world > 1 else None
    for s in range(world):
        shard = (rank - s) % world
        if s < world - 1:
            kv_n = bufs[s % 2]
            yield ("start", list(kv), list(kv_n))
        mask = pair_mask(causal, layout, rank, shard)
        if mask is not None:
            ops.bwd_accumulate(ws, q, kv[0], kv[1], dO, acc[0], acc[1], mask, scale)
        if world > 1:
            # the accumulators belong to key shard `shard`: pass them on; after
            # `world` rotations each is back with its owner
            yield ("start", list(acc), list(acc_n))
            yield ("wait",)
            acc, acc_n = acc_n, acc
            if s < world - 1:
                kv = kv_n
    dq = ops.bwd_finish(ws, q, scale)
    return dq, ops.to_bf16(acc[0]), ops.to_bf16(acc[1])


# ---------------------------------------------------------------- runners


def _peer(group, group_rank):
    import torch.distributed as dist
    return group_rank if group is None else dist.get_global_rank(group, group_rank)


def run_nccl(program, group=None):
    """Drive one rank's program with torch.distributed point-to-point
    operations (NCCL for CUDA tensors): "start" posts isend to rank+1 and irecv
    from rank-1 for each tensor; "wait" makes the current stream wait for
    all posted operations."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    nxt, prv = _peer(group, (rank + 1) % world), _peer(group, (rank - 1) % world)
    pending = []
    try:
        req = next(program)
        while True:
            if req[0] == "start":
                ops = []
                for snd, rcv in zip(req[1], req[2]):
                    ops.append(dist.P2POp(dist.isend, snd, nxt, group))
                    ops.append(dist.P2POp(dist.irecv, rcv, prv, group))
                pending += dist.batch_isend_irecv(ops)
            else:
                for w in pending:
                    w.wait()
                pending = []
            req = program.send(None)
    except StopIteration as stop:
        return stop.value


def run_local(programs):
    """Drive the programs of `len(programs)` virtual ranks in lockstep in one
    process: at each "wait", every rank's posted receive buffers are filled,
    by device copies, from the previous rank's posted send buffers."""
    G = len(programs)
    results = [None] * G
    reqs = []
    for p in programs:
        try:
            reqs.append(next(p))
        except StopIteration as stop:
            reqs.append(("done", stop.value))
    pending = [[] for _ in range(G)]
    while True:
        kinds = {r[0] for r in reqs}
        if kinds == {"done"}:
            return [r[1] for r in reqs]
        if len(kinds) != 1:
            raise RuntimeError(f"ring programs out of step: {sorted(kinds)}")
        kind = kinds.pop()
        if kind == "start":
            for r in range(G):
                pending[r].append((reqs[r][1], reqs[r][2]))
        else:
            for r in range(G):
                src = pending[(r - 1) % G]
                for (snd, _), (_, rcv) in zip(src, pending[r]):
                    for a, b in zip(snd, rcv):
                        b.copy_(a)
            pending = [[] for _ in range(G)]
        nxt = []
        for r, p in enumerate(programs):
            try:
                nxt.append(p.send(None))
            except StopIteration as stop:
                nxt.append(("done", stop.value))
        reqs = nxt


def local_ring_attention(q, k, v, dO, causal: bool, scale: float, world: int, ops=None,
                         layout: str = "contiguous"):
    """Forward and backward of attention over the whole [B, H, N, d] inputs,
    computed as a ring of `world` virtual ranks on this device (N divisible by
    world), the sequence laid out over the ranks as `layout` says.  `ops` is
    one ops object for every rank, or a list of one per rank.  Returns (O,
    LSE, dQ, dK, dV) for the whole sequence."""
    N = q.shape[2]
    if N % world:
        raise ValueError("sequence length must be divisible by the ring size")
    if layout not in LAYOUTS:
        raise ValueError(f"unknown ring layout {layout!r}")
    n = N // world
    if layout == "striped":
        sl = [slice(r, N, world) for r in range(world)]
    else:
        sl = [slice(r * n, (r + 1) * n) for r in range(world)]
    per_rank = ops if isinstance(ops, (list, tuple)) else [ops] * world
    shard = lambda t, r: t[:, :, sl[r]].contiguous()  # noqa: E731
    fwd = run_local([forward_program(shard(q, r), shard(k, r), shard(v, r), causal, scale, r,
                                     world, per_rank[r], layout) for r in range(world)])
    bwd = run_local([backward_program(shard(q, r), shard(k, r), shard(v, r), fwd[r][0],
                                      fwd[r][1], shard(dO, r), causal, scale, r, world,
                                      per_rank[r], layout) for r in range(world)])

    def gather(parts):
        out = torch.empty(parts[0].shape[:2] + (N,) + parts[0].shape[3:], dtype=parts[0].dtype,
                          device=parts[0].device)
        for r, part in enumerate(parts):
            out[:, :, sl[r]] = part
        return out

    return tuple(gather([res[i] for res in part]) for part, i in
                 ((fwd, 0), (fwd, 1), (bwd, 0), (bwd, 1), (bwd, 2)))
