"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (for example a plugin inside an application that owns all device memory
through its own pool, or a serving path that forbids cudaMalloc after start-up).
Instead of a caller workspace it uses a fixed scratch array that the library
reserves on each GPU.

These tests call it through the C ABI.  Before the checked shapes, a larger
problem with another padded length and head dimension runs through it, so the
scratch array holds a different layout when the checked calls start.  Then,
on two calls in a row (the second reuses what the first left behind), dK and
dV must equal those of the ordinary fa_bwd entry point with a caller workspace
bit for bit (both are deterministic), and dQ (whose fp32 reduction order
varies from run to run) must match fa_bwd's and the fp64 oracle's within the
gradient tolerance of the other parity tests.  A problem too large for the
scratch array is turned away before any work is enqueued.  This file is named
so that pytest collects it last.
"""
import pytest
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64
from parity_util import TOL_GRAD_MAX, Check

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _noalloc(q, k, v, o, lse, dO, causal, scale):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    status = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), dO.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), B, H, N, d, int(causal), scale, _stream())
    assert status == fa.FA_OK, fa.fa_strerror(status)
    assert fa.fa_get_device_error() == fa.FA_OK
    return dq, dk, dv


def _problem(B, H, N, d, causal, seed):
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=seed, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal, scale)
    return host, (q, k, v, o, lse, dO), scale


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 4, 1000, 128, True),
                                            (1, 3, 777, 64, False)])
def test_noalloc_matches_fa_bwd_on_two_calls(B, H, N, d, causal):
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES
    # fill the scratch array with another problem's layout first
    _, big, big_scale = _problem(2, 8, 3000, 192 - d, not causal, seed=7)
    assert (fa.fa_bwd_workspace_size(2, 8, 3000, 192 - d)
            <= fa.FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES)
    _noalloc(*big, not causal, big_scale)

    host, args, scale = _problem(B, H, N, d, causal, seed=31 + d)
    q, k, v, o, lse, dO = args
    ref = fa.attention_backward(q, k, v, o, lse, dO, causal, scale)  # caller workspace
    assert fa.fa_get_device_error() == fa.FA_OK
    exact = oracle.ref_bwd(*[to_f64(host[x]) for x in ("q", "k", "v", "dO")], causal,
                           scale)[:3]
    for _ in range(2):
        dq, dk, dv = _noalloc(*args, causal, scale)
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
        assert torch.isfinite(dq.float()).all()
        assert (dq.float() - ref[0].float()).abs().max().item() <= TOL_GRAD_MAX
        c = Check()
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), exact):
            c.grad(name, to_f64(got.cpu()), want)
        c.done()


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, H, N, d = 1, 1, 200_000, 128
    assert fa.fa_bwd_workspace_size(B, H, N, d) > fa.FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    status = fa.fa_bwd_noalloc(*([fake] * 9), B, H, N, d, 1, 0.1, 0)
    assert status == fa.FA_ERR_INVALID_ARG
    status = fa.fa_bwd_noalloc(*([fake] * 9), 1, 1, 128, 96, 1, 0.1, 0)
    assert status == fa.FA_ERR_UNSUPPORTED
