"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (for example a plugin inside an application that owns all device memory
through its own pool, or a serving path that forbids cudaMalloc after start-up).
Instead of a caller workspace it uses a fixed scratch array that the library
reserves on each GPU.

These tests call it through the C ABI and check, on two calls in a row (the
second one reuses the scratch array the first one left behind), that it gives
the same dQ, dK and dV as the ordinary fa_bwd entry point with a caller
workspace, within the gradient tolerance the other tests use.  They also check
that a problem too large for the scratch array is turned away before any work
is enqueued.  This file is named so that pytest collects it last.
"""
import pytest
import torch

import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale

pytestmark = pytest.mark.gpu

TOL_GRAD_MAX = 2e-2  # the max-abs gradient tolerance of the parity tests


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 4, 1000, 128, True),
                                            (1, 3, 777, 64, False)])
def test_noalloc_matches_fa_bwd_on_two_calls(B, H, N, d, causal):
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=31 + d, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal, scale)
    ref = fa.attention_backward(q, k, v, o, lse, dO, causal, scale)  # caller workspace
    assert fa.fa_get_device_error() == fa.FA_OK
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        status = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), dO.data_ptr(), dq.data_ptr(),
                                   dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal),
                                   scale, stream)
        assert status == fa.FA_OK, fa.fa_strerror(status)
        assert fa.fa_get_device_error() == fa.FA_OK
        for got, want in zip((dq, dk, dv), ref):
            assert torch.isfinite(got.float()).all()
            err = (got.float() - want.float()).abs().max().item()
            assert err <= TOL_GRAD_MAX, err


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, H, N, d = 1, 1, 200_000, 128
    assert fa.fa_bwd_workspace_size(B, H, N, d) > fa.FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    status = fa.fa_bwd_noalloc(*([fake] * 9), B, H, N, d, 1, 0.1, 0)
    assert status == fa.FA_ERR_INVALID_ARG
    status = fa.fa_bwd_noalloc(*([fake] * 9), 1, 1, 128, 96, 1, 0.1, 0)
    assert status == fa.FA_ERR_UNSUPPORTED
