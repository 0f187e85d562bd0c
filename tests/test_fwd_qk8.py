"""The 8-bit score path on the GPU: fa_fwd_qk8 with e4m3 Q, K (per-tensor
descales) and bf16 V against the fp64 oracle run on the dequantised inputs,
within the forward tolerances of the bf16 path (the e4m3 products are exact
in the fp32 accumulator; P V is the bf16 path's)."""
import pytest
import torch

import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_e4m3, to_f64
from parity_util import check_forward_full, check_forward_sampled

pytestmark = pytest.mark.gpu


def _run(B, H, N, causal, seed, dist="normal", scale=None):
    d = 128
    scale = default_scale(d) if scale is None else scale
    host = attention_inputs(B, H, N, d, seed=seed, dist=dist)
    q8, qs = to_e4m3(host["q"])
    k8, ks = to_e4m3(host["k"])
    deq = {"q": (q8.to(torch.float64) * qs), "k": (k8.to(torch.float64) * ks), "v": host["v"]}
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.attention_forward_qk8(q8.cuda(), k8.cuda(), host["v"].cuda(), qs, ks, causal, scale,
                             out=o, lse=lse)
    status = fa.fa_get_device_error()
    assert status == fa.FA_OK, fa.fa_strerror(status)
    return deq, o, lse, scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 256, 300, 640, 1000, 2048])
def test_qk8_matches_oracle_on_dequantised_inputs(N, causal):
    deq, o, lse, scale = _run(2, 3, N, causal, seed=N + int(causal))
    check_forward_full(deq, o, lse, causal, scale)


def test_qk8_row_scaled_and_scale_one():
    for causal in (False, True):
        deq, o, lse, scale = _run(1, 2, 700, causal, seed=5, dist="row_scaled", scale=1.0)
        check_forward_full(deq, o, lse, causal, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_qk8_benchmark_shape_sampled(causal):
    """B=2 H=16 N=8192: exact oracle rows for a sample of rows of 4 heads."""
    deq, o, lse, scale = _run(2, 16, 8192, causal, seed=2)
    check_forward_sampled(deq, o, lse, causal, scale, heads=[0, 7, 19, 31], rows_per_head=24)


def test_qk8_rejects_bad_arguments():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.float8_e4m3fn, device="cuda")
    v = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_forward_qk8(q, q, v, 1.0, 1.0, False, 0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    q = torch.zeros(1, 1, 128, 128, dtype=torch.float8_e4m3fn, device="cuda")
    v = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_forward_qk8(q, q, v, 0.0, 1.0, False, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
