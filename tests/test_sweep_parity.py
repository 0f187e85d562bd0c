"""Forward and backward parity at every shape of the pages' kernel benchmark
(iplexlaw FlashAttention-2 blog, "Read the reported speed-ups with their
conditions": sequence lengths 512 to 16k, head dimension 64 and 128, causal
and non-causal, 16k tokens per batch) and of the two GPT-style layers, each at
its own batch and head count.

* N <= 2048: every element of O, LSE, dQ, dK and dV of every head is compared
  with the oracle's whole-tensor forward and backward.
* N >= 4096: exact oracle rows -- sampled query rows of O, LSE and dQ and
  sampled key rows of dK and dV -- in the first and the last head.

The shapes: B = 16384 / N and model width 2048 (H = 32 at d = 64, H = 16 at
d = 128); GPT layer (a) B=8 N=2048 H=16 and (b) B=2 N=8192 H=20, d = 128,
causal, row-scaled inputs.  The long single sequence (B=1 H=16 N=65536) is in
test_fwd.py / test_bwd.py."""
import pytest

from exact_attention_109_b200.inputs import default_scale
from parity_util import (check_backward_sampled, check_forward_sampled, check_full,
                         gpu_inputs, run_backward, run_forward)

pytestmark = pytest.mark.gpu

WIDTH, TOKENS = 2048, 16384


def _fwd_bwd(B, H, N, d, causal, seed, dist="normal"):
    scale = default_scale(d)
    host, dev = gpu_inputs(B, H, N, d, seed, dist=dist, with_dout=True)
    o, lse = run_forward(dev, causal, scale)
    dq, dk, dv = run_backward(dev, o, lse, causal, scale)
    del dev
    return host, o, lse, dq, dk, dv, scale


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [512, 1024, 2048])
def test_sweep_whole_tensors(N, causal, d):
    B, H = TOKENS // N, WIDTH // d
    host, o, lse, dq, dk, dv, scale = _fwd_bwd(B, H, N, d, causal, seed=2)
    check_full(host, o, lse, dq, dk, dv, causal, scale)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [4096, 8192, 16384])
def test_sweep_sampled_rows(N, causal, d):
    B, H = TOKENS // N, WIDTH // d
    host, o, lse, dq, dk, dv, scale = _fwd_bwd(B, H, N, d, causal, seed=2)
    heads = [0, B * H - 1]
    check_forward_sampled(host, o, lse, causal, scale, heads, 48)
    check_backward_sampled(host, dq, dk, dv, causal, scale, heads, 32)


def test_gpt_layer_a_whole_tensors():
    """Width 2048: B=8, H=16, N=2048, d=128, causal, row-scaled Q/K/V."""
    host, o, lse, dq, dk, dv, scale = _fwd_bwd(8, 16, 2048, 128, True, seed=4,
                                               dist="row_scaled")
    check_full(host, o, lse, dq, dk, dv, True, scale)


def test_gpt_layer_b_sampled_rows():
    """Width 2560: B=2, H=20, N=8192, d=128, causal, row-scaled Q/K/V."""
    host, o, lse, dq, dk, dv, scale = _fwd_bwd(2, 20, 8192, 128, True, seed=5,
                                               dist="row_scaled")
    heads = [0, 39]
    check_forward_sampled(host, o, lse, True, scale, heads, 48)
    check_backward_sampled(host, dq, dk, dv, True, scale, heads, 32)
