"""Decoding parity on the GPU: fa_fwd_decode (split-KV, through the C ABI)
against the fp64 oracle's decoding reference on the same seeded bf16 inputs.

Covers one query row and several (1, 2, 3, 4, 7, 16: one, two and several
four-row query groups, with a ragged last group), key counts that leave ragged
blocks and splits, caches allocated longer than the keys in use (the unused
rows hold NaN, so reading them would show), causal alignment of the query rows
with the last keys, a single split (no workspace) and many splits, and the
decoding shapes that the benchmark times, whole."""
import numpy as np
import pytest
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import decode_inputs, default_scale, to_f64
from parity_util import Check, max_abs

pytestmark = pytest.mark.gpu


def run_decode(host, causal, scale, kv_rows=None, n_keys=None, dist_fill=float("nan")):
    q = host["q"].cuda()
    B, H, Nk, d = host["k"].shape
    rows = kv_rows or Nk
    k = torch.full((B, H, rows, d), dist_fill, dtype=torch.bfloat16, device="cuda")
    v = torch.full_like(k, dist_fill)
    k[:, :, :Nk] = host["k"].cuda()
    v[:, :, :Nk] = host["v"].cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    need = fa.fa_decode_workspace_size(B, H, q.shape[2], Nk, d)
    ws = (torch.full((need // 4,), float("nan"), dtype=torch.float32, device="cuda")
          if need else None)
    fa.attention_decode(q, k, v, causal, scale, n_keys=Nk, out=out, lse=lse, workspace=ws)
    status = fa.fa_get_device_error()
    assert status == fa.FA_OK, fa.fa_strerror(status)
    return out, lse


def check_decode(host, o, lse, causal, scale):
    o_ref, lse_ref = oracle.ref_fwd_decode(to_f64(host["q"]), to_f64(host["k"]),
                                           to_f64(host["v"]), causal, scale)
    c = Check()
    c.o(to_f64(o.cpu()), o_ref)
    c.lse(lse.cpu().double().numpy(), lse_ref)
    return c.done()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 63), (1, 64), (1, 65), (1, 256), (1, 257),
                                   (1, 1000), (2, 2), (2, 777), (3, 3), (3, 300),
                                   (4, 129), (7, 4095), (16, 2000), (1, 20000)])
def test_ragged_decode(Nq, Nk, causal, d):
    host = decode_inputs(2, 3, Nq, Nk, d, seed=Nq * 1000 + Nk + d + int(causal))
    o, lse = run_decode(host, causal, default_scale(d))
    check_decode(host, o, lse, causal, default_scale(d))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq", [1, 4, 5])
def test_cache_longer_than_keys(Nq, d):
    """Only the first Nk rows of each head's cache are keys; the rest is NaN."""
    host = decode_inputs(2, 2, Nq, 1500, d, seed=40 + Nq)
    for causal in (False, True):
        o, lse = run_decode(host, causal, default_scale(d), kv_rows=2048)
        check_decode(host, o, lse, causal, default_scale(d))


@pytest.mark.parametrize("d", [64, 128])
def test_decode_equals_square_forward_when_nq_equals_nk(d):
    """With Nq = Nk the decoding mask is fa_fwd's j <= i; both paths agree
    with the oracle (and hence with each other)."""
    host = decode_inputs(1, 2, 200, 200, d, seed=9)
    for causal in (False, True):
        o, lse = run_decode(host, causal, default_scale(d))
        check_decode(host, o, lse, causal, default_scale(d))
        o2, lse2 = fa.attention_forward(host["q"].cuda(), host["k"].cuda(),
                                        host["v"].cuda(), causal, default_scale(d))
        assert max_abs(lse.cpu().double().numpy(), lse2.cpu().double().numpy()) <= 2e-3


def test_large_scores():
    """Row-scaled inputs with scale 1 push the scores far from zero, which
    exercises the deferred rescaling and the split merge."""
    host = decode_inputs(1, 4, 3, 9000, 128, seed=77, dist="row_scaled")
    for causal in (False, True):
        o, lse = run_decode(host, causal, 1.0)
        check_decode(host, o, lse, causal, 1.0)


def test_many_heads_one_key_block():
    host = decode_inputs(7, 9, 1, 40, 64, seed=5)
    o, lse = run_decode(host, False, default_scale(64))
    check_decode(host, o, lse, False, default_scale(64))


def test_repeated_calls_reuse_workspace():
    host = decode_inputs(2, 4, 1, 5000, 128, seed=8)
    first = run_decode(host, True, default_scale(128))
    second = run_decode(host, True, default_scale(128))
    assert torch.equal(first[0], second[0]) and torch.equal(first[1], second[1])


# The decoding workloads the benchmark times, checked whole: model width 2048
# (H = 16, d = 128), one query row per sequence.
@pytest.mark.parametrize("B,H,Nq,Nk", [(16, 16, 1, 8192), (1, 16, 1, 65536),
                                       (4, 16, 4, 16384)])
def test_benchmark_decode_shapes(B, H, Nq, Nk):
    host = decode_inputs(B, H, Nq, Nk, 128, seed=2024)
    o, lse = run_decode(host, True, default_scale(128))
    check_decode(host, o, lse, True, default_scale(128))


def test_decode_rejects_bad_arguments_on_device():
    q = torch.zeros(1, 1, 2, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_decode(q, k, k, True, 0.1)  # causal needs Nk >= Nq
    assert e.value.status == fa.FA_ERR_INVALID_ARG
