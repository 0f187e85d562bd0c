"""The all-8-bit forward on the GPU: fa_fwd_fp8 with e4m3 Q, K and V
(per-tensor descales), S = Q K^T and O += P V both on kind::f8f6f4 tensor
cores, against the fp64 oracle run on the dequantised inputs.

P is rounded to e4m3 inside the kernel, so the bf16 tolerances do not apply;
the contract stated in include/fa.h does, per element:
    |O - O_ref| <= 2^-3 * sum_j P_ij |v_j - O_ref,i| + 2^-8 |O_ref| + 4e-3,
with relative L2 of O <= 6e-2 and LSE max-abs <= 1e-3.  The first term is the
worst case of rounding every weight to e4m3 (2^-4 relative each, 2^-3 once
normalised by their rounded sum, since O is then an exact convex combination
of V rows); the second is the bf16 output rounding; the third covers the
weights below e4m3's normal range (2^-16 absolute each, random in sign) and
the fp32 accumulation.  P_ij here are the exact softmax weights, computed in
fp64 from the same dequantised inputs (they only size the bound; the expected
values come from the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_e4m3
from parity_util import Check

pytestmark = pytest.mark.gpu

REL_L2 = 6e-2


def _run(B, H, N, causal, seed, dist="normal", scale=None):
    d = 128
    scale = default_scale(d) if scale is None else scale
    host = attention_inputs(B, H, N, d, seed=seed, dist=dist)
    q8, qs = to_e4m3(host["q"])
    k8, ks = to_e4m3(host["k"])
    v8, vs = to_e4m3(host["v"])
    deq = {"q": q8.to(torch.float64).numpy() * qs, "k": k8.to(torch.float64).numpy() * ks,
           "v": v8.to(torch.float64).numpy() * vs}
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.attention_forward_fp8(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, causal, scale,
                             out=o, lse=lse)
    status = fa.fa_get_device_error()
    assert status == fa.FA_OK, fa.fa_strerror(status)
    return deq, o.cpu().to(torch.float64).numpy(), lse.cpu().double().numpy(), scale


def _bound(q, k, v, o_ref, rows, causal, scale):
    """2^-3 * sum_j P_ij |v_j - O_ref,i| + 2^-8 |O_ref,i| + 4e-3 for the given
    query rows of one head (q, k, v: [N, d]; o_ref: [len(rows), d])."""
    N = q.shape[0]
    out = np.empty_like(o_ref)
    for a in range(0, len(rows), 64):
        rr = rows[a:a + 64]
        s = scale * (q[rr] @ k.T)
        if causal:
            s = np.where(np.arange(N)[None, :] > rr[:, None], -np.inf, s)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        spread = np.einsum("ij,ijd->id", p, np.abs(v[None, :, :] - o_ref[a:a + 64, None, :]))
        out[a:a + 64] = 2.0 ** -3 * spread
    return out + 2.0 ** -8 * np.abs(o_ref) + 4e-3


def _check(deq, o, lse, causal, scale, heads=None, rows_per_head=None, seed=0):
    B, H, N, d = deq["q"].shape
    flat = {x: deq[x].reshape(B * H, N, d) for x in ("q", "k", "v")}
    og, lg = o.reshape(B * H, N, d), lse.reshape(B * H, N)
    rng = np.random.default_rng(seed)
    c = Check()
    worst = 0.0
    for bh in (range(B * H) if heads is None else heads):
        q, k, v = flat["q"][bh], flat["k"][bh], flat["v"][bh]
        if rows_per_head is None:
            rows = np.arange(N)
        else:
            rows = np.unique(np.concatenate([[0, 1, 127, 128, N - 1],
                                             rng.choice(N, rows_per_head, replace=False)]))
        o_ref, l_ref = oracle.ref_fwd_rows(q, k, v, rows, causal, scale)
        err = np.abs(og[bh][rows] - o_ref)
        ratio = float(np.max(err / _bound(q, k, v, o_ref, rows, causal, scale)))
        worst = max(worst, ratio)
        c.bound("o_err_over_bound", ratio, 1.0)
        c.bound("o_rel_l2", float(np.linalg.norm(og[bh][rows] - o_ref) /
                                  np.linalg.norm(o_ref)), REL_L2)
        c.lse(lg[bh][rows], l_ref)
    return c.done()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 300, 1000])
def test_fp8_matches_oracle_on_dequantised_inputs(N, causal):
    deq, o, lse, scale = _run(2, 3, N, causal, seed=N + 7 * int(causal))
    _check(deq, o, lse, causal, scale)


def test_fp8_row_scaled_and_scale_one():
    """Large scores: peaked softmax rows, frequent refreshes of the running max."""
    for causal in (False, True):
        deq, o, lse, scale = _run(1, 2, 700, causal, seed=5, dist="row_scaled", scale=1.0)
        _check(deq, o, lse, causal, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_benchmark_shape_sampled(causal):
    """B=2 H=16 N=8192 d=128: exact oracle rows for a sample of rows of 3 heads."""
    deq, o, lse, scale = _run(2, 16, 8192, causal, seed=2)
    _check(deq, o, lse, causal, scale, heads=[0, 13, 31], rows_per_head=48)


def test_fp8_rejects_bad_arguments():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_forward_fp8(q, q, q, 1.0, 1.0, 1.0, False, 0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    q = torch.zeros(1, 1, 128, 128, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.attention_forward_fp8(q, q, q, 1.0, 1.0, 0.0, False, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
