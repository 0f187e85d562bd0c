"""Tensors beyond 2^31 elements: every offset of the last head exceeds the
32-bit range, so a 32-bit index anywhere in the forward, the backward or
their host set-up shows up as wrong rows there.  B=16, H=130, N=8192,
d=128 causal (2.18e9 elements per tensor, 4.4 GB), and B=66, H=256,
N=2048, d=64 causal (2.21e9 elements; the d = 64 kernels with two CTAs per
SM); the last head's sampled rows are checked against the oracle on a copy
of that head's inputs."""
import pytest
import torch

from exact_attention_109_b200.inputs import attention_inputs_device, default_scale
from parity_util import (check_backward_causal_tail, check_forward_sampled, run_backward,
                         run_forward)

pytestmark = pytest.mark.gpu


def test_beyond_2g_elements():
    B, H, N, d = 16, 130, 8192, 128
    assert B * H * N * d > 2 ** 31
    scale = default_scale(d)
    dev = attention_inputs_device(B, H, N, d, seed=12)
    o, lse = run_forward(dev, True, scale)
    dq, dk, dv = run_backward(dev, o, lse, True, scale)
    # the last head, as a one-head problem for the oracle checks
    host = {x: dev[x][-1:, -1:].cpu() for x in ("q", "k", "v", "dO")}
    del dev
    check_forward_sampled(host, o[-1:, -1:].cpu(), lse[-1:, -1:].cpu(), True, scale, [0], 24)
    check_backward_causal_tail(host, dq[-1:, -1:].cpu(), dk[-1:, -1:].cpu(), dv[-1:, -1:].cpu(),
                               scale, [0], 16, 512)


def test_beyond_2g_elements_d64():
    B, H, N, d = 66, 256, 2048, 64
    assert B * H * N * d > 2 ** 31
    scale = default_scale(d)
    dev = attention_inputs_device(B, H, N, d, seed=13)
    o, lse = run_forward(dev, True, scale)
    dq, dk, dv = run_backward(dev, o, lse, True, scale)
    host = {x: dev[x][-1:, -1:].cpu() for x in ("q", "k", "v", "dO")}
    del dev
    check_forward_sampled(host, o[-1:, -1:].cpu(), lse[-1:, -1:].cpu(), True, scale, [0], 24)
    check_backward_causal_tail(host, dq[-1:, -1:].cpu(), dk[-1:, -1:].cpu(), dv[-1:, -1:].cpu(),
                               scale, [0], 16, 512)
