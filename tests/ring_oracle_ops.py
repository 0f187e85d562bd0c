"""The per-step arithmetic of the ring schedule done by the fp64 oracle on CPU
tensors, with the same interface as exact_attention_109_b200.ring.CudaOps, so
that the ring's host logic (which shard when, the causal flags, the
rotations, the return of the dK/dV accumulators) can be checked without a
GPU.  Test infrastructure only."""
import numpy as np
import torch

import oracle


def _np(t):
    return t.detach().to(torch.float64).numpy()


class OracleOps:
    """`causal` is the library's mask argument: 0 none, 1 key j visible to
    query i iff j <= i, 2 iff j < i.  Mode 2 is the causal attention of
    queries 1..n-1 over keys 0..n-2 (query i sees keys j <= i - 1), with row 0
    seeing no key (O = 0, LSE = -inf; it adds nothing to any gradient)."""

    def fwd(self, q, k, v, causal, scale):
        if causal == 2:
            q, k, v = _np(q), _np(k), _np(v)
            o = np.zeros(q.shape)
            lse = np.full(q.shape[:3], -np.inf)
            if q.shape[2] > 1:
                o[:, :, 1:], lse[:, :, 1:] = oracle.ref_fwd(q[:, :, 1:], k[:, :, :-1],
                                                            v[:, :, :-1], True, scale)
            return torch.from_numpy(o), torch.from_numpy(lse)
        o, lse = oracle.ref_fwd(_np(q), _np(k), _np(v), bool(causal), scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o_acc, lse_acc, o_part, lse_part, o_out, init):
        if init:
            o, lse = _np(o_part), _np(lse_part)
        else:
            o, lse = oracle.ref_lse_merge(_np(o_acc), _np(lse_acc), _np(o_part), _np(lse_part))
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(lse))
        if o_out is not None:
            o_out.copy_(torch.from_numpy(o))

    def bwd_prepare(self, o, lse, dO):
        return {"lse": _np(lse), "D": np.sum(_np(o) * _np(dO), axis=-1),
                "dq": np.zeros(tuple(o.shape))}

    def bwd_accumulate(self, ws, q, k, v, dO, dk_acc, dv_acc, causal, scale):
        if causal == 2:
            q, k, v, dO = _np(q), _np(k), _np(v), _np(dO)
            dq, dk, dv = np.zeros(q.shape), np.zeros(q.shape), np.zeros(q.shape)
            if q.shape[2] > 1:
                dq[:, :, 1:], dk[:, :, :-1], dv[:, :, :-1] = oracle.ref_grads_given_stats(
                    q[:, :, 1:], k[:, :, :-1], v[:, :, :-1], dO[:, :, 1:],
                    ws["lse"][:, :, 1:], ws["D"][:, :, 1:], True, scale)
        else:
            dq, dk, dv = oracle.ref_grads_given_stats(_np(q), _np(k), _np(v), _np(dO),
                                                      ws["lse"], ws["D"], bool(causal), scale)
        ws["dq"] += dq
        dk_acc.copy_(torch.from_numpy(_np(dk_acc) + dk))
        dv_acc.copy_(torch.from_numpy(_np(dv_acc) + dv))

    def bwd_finish(self, ws, q, scale):
        return torch.from_numpy(ws["dq"]).to(q.dtype)

    def to_bf16(self, x):
        return x.to(torch.float64)
