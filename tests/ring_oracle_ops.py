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
    def fwd(self, q, k, v, causal, scale):
        o, lse = oracle.ref_fwd(_np(q), _np(k), _np(v), causal, scale)
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
        dq, dk, dv = oracle.ref_grads_given_stats(_np(q), _np(k), _np(v), _np(dO), ws["lse"],
                                                  ws["D"], causal, scale)
        ws["dq"] += dq
        dk_acc.copy_(torch.from_numpy(_np(dk_acc) + dk))
        dv_acc.copy_(torch.from_numpy(_np(dv_acc) + dv))

    def bwd_finish(self, ws, q, scale):
        return torch.from_numpy(ws["dq"]).to(q.dtype)

    def to_bf16(self, x):
        return x.to(torch.float64)
