"""Forward parity on the GPU: the CUDA path (through the C ABI) against the
fp64 oracle on the same seeded bf16 inputs.  The benchmark sweep's shapes are
in test_sweep_parity.py."""
import numpy as np
import pytest
import torch

import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import default_scale
from parity_util import (check_forward_full, check_forward_sampled, check_full, gpu_inputs,
                         run_backward, run_forward)

pytestmark = pytest.mark.gpu


def test_tiny_config_seed0():
    """B=1, H=2, N=128, d=64, non-causal, scale=1/sqrt(d), seed 0."""
    host, dev = gpu_inputs(1, 2, 128, 64, seed=0)
    o, lse = run_forward(dev, False, default_scale(64))
    check_forward_full(host, o, lse, False, default_scale(64))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 64, 127, 128, 129, 200, 255, 256, 257, 384,
                               511, 640, 1000])
def test_ragged_lengths(N, causal, d):
    host, dev = gpu_inputs(2, 3, N, d, seed=N + 17 * d + int(causal))
    o, lse = run_forward(dev, causal, default_scale(d))
    check_forward_full(host, o, lse, causal, default_scale(d))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(512, 128), (513, 128), (2048, 64), (2049, 64)])
def test_kernel_crossovers(N, d, causal):
    """fa_fwd picks its kernel by shape: the lengths on either side of each
    switch (d = 128: one-tile up to N = 512; d = 64: 64-key blocks up to
    N = 2048), whole tensors, forward and backward."""
    host, dev = gpu_inputs(1, 2, N, d, seed=N + 3 * d + int(causal), with_dout=True)
    scale = default_scale(d)
    o, lse = run_forward(dev, causal, scale)
    dq, dk, dv = run_backward(dev, o, lse, causal, scale)
    check_full(host, o, lse, dq, dk, dv, causal, scale)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_many_heads_and_batches(causal, d):
    """Exercises the flattened (batch*head, query-pair) grid decode."""
    host, dev = gpu_inputs(5, 7, 300, d, seed=11)
    o, lse = run_forward(dev, causal, default_scale(d))
    check_forward_full(host, o, lse, causal, default_scale(d))


def test_large_scores_and_other_scale():
    """Row-scaled inputs and a scale of 1 push exponents far from zero."""
    host, dev = gpu_inputs(1, 2, 700, 128, seed=5, dist="row_scaled")
    for causal in (False, True):
        o, lse = run_forward(dev, causal, 1.0)
        check_forward_full(host, o, lse, causal, 1.0)


def test_long_sequence_sampled():
    """B=1, H=16, d=128, N=65536, causal."""
    host, dev = gpu_inputs(1, 16, 65536, 128, seed=3)
    o, lse = run_forward(dev, True, default_scale(128))
    check_forward_sampled(host, o, lse, True, default_scale(128), [0, 15], 24)


def test_deterministic():
    host, dev = gpu_inputs(2, 4, 1000, 128, seed=9)
    o1, l1 = run_forward(dev, True, 0.1)
    o2, l2 = run_forward(dev, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_misaligned_pointer_is_rejected():
    host, dev = gpu_inputs(1, 1, 128, 64, seed=0)
    q = dev["q"]
    st = fa.fa_fwd(q.data_ptr() + 2, dev["k"].data_ptr(), dev["v"].data_ptr(),
                   q.data_ptr(), q.data_ptr(), 1, 1, 127, 64, 0, 0.125)
    assert st == fa.FA_ERR_MISALIGNED


def test_outputs_only_touch_their_rows():
    """Canaries past the end of O and LSE stay intact."""
    host, dev = gpu_inputs(1, 2, 300, 64, seed=2)
    o_big = torch.full((1 * 2 * 300 * 64 + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    lse_big = torch.full((600 + 64,), 7.0, dtype=torch.float32, device="cuda")
    o = o_big[: 2 * 300 * 64].view(1, 2, 300, 64)
    lse = lse_big[:600].view(1, 2, 300)
    fa.attention_forward(dev["q"], dev["k"], dev["v"], True, 0.125, out=o, lse=lse)
    assert fa.fa_get_device_error() == fa.FA_OK
    assert torch.all(o_big[2 * 300 * 64:] == 7.0)
    assert torch.all(lse_big[600:] == 7.0)
    check_forward_full(host, o, lse, True, 0.125)
