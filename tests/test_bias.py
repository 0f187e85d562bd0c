"""Attention with an additive score bias on the GPU: fa_fwd_bias / fa_bwd_bias
against the oracle's ref_fwd_bias / ref_bwd_bias (pinned to brute force,
torch autograd and finite differences) on the same seeded bf16 inputs, for
full and broadcast biases, both masks, d = 64 and 128, ragged lengths, and
biases that hide keys with -inf.  Tolerances are those of the plain path;
dBias is a gradient (dS) and takes the gradient bound.  No oracle call is
given anything the CUDA path computed."""
import numpy as np
import pytest
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64
from parity_util import Check

pytestmark = pytest.mark.gpu


def _bias(shape, seed, hide=0.0):
    g = torch.Generator().manual_seed(seed)
    b = torch.randn(shape, generator=g) * 2.0
    if hide:
        n = shape[-1]
        drop = torch.rand(shape, generator=g) < hide
        drop &= ~torch.eye(n, dtype=torch.bool)  # every row keeps its own key
        b = b.masked_fill(drop, float("-inf"))
    return b.to(torch.bfloat16)


def _run(B, H, N, d, causal, bshape, seed, hide=0.0, backward=True):
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=seed, with_dout=True)
    bias = _bias(bshape, seed + 1, hide)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    bd = bias.cuda()
    o, lse = fa.attention_forward_bias(q, k, v, bd, causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    args = [to_f64(host[x]) for x in ("q", "k", "v")]
    o_ref, lse_ref = oracle.ref_fwd_bias(*args, to_f64(bias), causal, scale)
    c = Check()
    c.o(to_f64(o.cpu()), o_ref)
    c.lse(lse.cpu().double().numpy(), lse_ref)
    if not backward:
        return c.done()
    dq, dk, dv, db = fa.attention_backward_bias(q, k, v, bd, o, lse, dO, causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    refs = oracle.ref_bwd_bias(*args, to_f64(bias), to_f64(host["dO"]), causal, scale)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs[:3]):
        c.grad(name, to_f64(got.cpu()), ref)
    # dBias is dS itself, not damped by the 1/sqrt(d) of dQ and dK, and
    # D = rowsum(dO * O) enters it undamped: one bf16 ulp of one element of
    # the O a backward pass receives moves dS_ij by P_ij |dO| ulp, up to
    # ~0.03 in rows whose softmax is peaked.  So dBias is checked on a second
    # backward pass whose O and LSE inputs are the oracle's own forward
    # results in the formats the pass takes (O rounded to bf16, LSE to fp32),
    # against the oracle's dBias with D taken from that same bf16 O.  Both
    # sides then start from identical inputs; nothing computed by the CUDA
    # path enters the oracle.
    o_in = torch.from_numpy(o_ref).to(torch.bfloat16)
    lse_in = torch.from_numpy(lse_ref).to(torch.float32)
    dq2, dk2, dv2, db = fa.attention_backward_bias(q, k, v, bd, o_in.cuda(), lse_in.cuda(), dO,
                                                   causal, scale)
    assert fa.fa_get_device_error() == fa.FA_OK
    refs2 = oracle.ref_bwd_bias(*args, to_f64(bias), to_f64(host["dO"]), causal, scale,
                                o_given=to_f64(o_in))
    for name, got, ref in zip(("dq_oracle_o", "dk_oracle_o", "dv_oracle_o", "dbias"),
                              (dq2, dk2, dv2, db), refs2):
        c.grad(name, to_f64(got.cpu()), ref)
    return c.done()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [8, 128, 136, 256, 504, 640])
def test_bias_full_shape(N, causal, d):
    _run(2, 3, N, d, causal, (2, 3, N, N), seed=N + d + int(causal))


@pytest.mark.parametrize("bshape", [(1, 3), (1, 1), (2, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_bias_broadcast(bshape, causal):
    N = 384
    _run(2, 3, N, 128, causal, bshape + (N, N), seed=11 + int(causal))


@pytest.mark.parametrize("causal", [False, True])
def test_bias_hiding_keys_with_minus_infinity(causal):
    _run(1, 2, 520, 128, causal, (1, 2, 520, 520), seed=21, hide=0.3)


def test_bias_forward_long():
    for causal in (False, True):
        _run(1, 2, 2048, 128, causal, (1, 2, 2048, 2048), seed=31, backward=False)


def test_bias_backward_without_dbias_and_bad_sizes():
    B, H, N, d = 1, 2, 256, 64
    host = attention_inputs(B, H, N, d, seed=41, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    bias = _bias((1, 2, N, N), 42).cuda()
    o, lse = fa.attention_forward_bias(q, k, v, bias, True, 0.125)
    full = fa.attention_backward_bias(q, k, v, bias, o, lse, dO, True, 0.125)
    part = fa.attention_backward_bias(q, k, v, bias, o, lse, dO, True, 0.125, want_dbias=False)
    assert part[3] is None
    for a, b in zip(full[1:3], part[1:3]):
        assert torch.equal(a, b)
    q2 = torch.zeros(1, 1, 100, 64, dtype=torch.bfloat16, device="cuda")
    b2 = torch.zeros(1, 1, 100, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_forward_bias(q2, q2, q2, b2, False, 0.125)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
