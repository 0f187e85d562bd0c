"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding, run the fp64 oracle on the same bf16 bits, and measure the error.

Tolerances (GPU result vs the fp64 oracle on the same seeded inputs):
  O:            max-abs <= 1e-2 and relative L2 <= 5e-3
  dQ, dK, dV:   max-abs <= 2e-2
  LSE:          max-abs <= 1e-3 (fp32 statistic; the kernel's error is ~1e-5)
Outputs are bf16, whose own rounding of an exact value is up to half an ulp:
0.0156 for |x| in [4, 8) and 0.031 above 8, at or above the 2e-2 bound.  The
max-abs bounds therefore apply to each element's error in excess of that
element's unavoidable rounding, |gpu - ref| - |bf16(ref) - ref| (the "excess");
the raw max-abs and the bf16 floor max|bf16(ref) - ref| are reported beside it.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64

TOL_O_MAX = 1e-2
TOL_O_REL_L2 = 5e-3
TOL_GRAD_MAX = 2e-2
TOL_LSE_MAX = 1e-3


def bf16_floor(ref: np.ndarray) -> float:
    r = torch.from_numpy(np.ascontiguousarray(ref)).to(torch.bfloat16).to(torch.float64)
    return float(np.max(np.abs(r.numpy() - ref))) if ref.size else 0.0


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    assert np.all(np.isfinite(a)), "non-finite values in GPU output"
    return float(np.max(np.abs(a - b)))


def max_excess(gpu, ref) -> float:
    """max over elements of |gpu - ref| - |bf16(ref) - ref|."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.ascontiguousarray(ref, dtype=np.float64)
    if gpu.size == 0:
        return 0.0
    assert np.all(np.isfinite(gpu)), "non-finite values in GPU output"
    rounded = torch.from_numpy(ref).to(torch.bfloat16).to(torch.float64).numpy()
    return float(np.max(np.abs(gpu - ref) - np.abs(rounded - ref)))


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def gpu_inputs(B, H, N, d, seed, dist="normal", with_dout=False):
    host = attention_inputs(B, H, N, d, seed, dist, with_dout)
    dev = {k: v.cuda() for k, v in host.items()}
    return host, dev


def run_forward(dev, causal, scale):
    q = dev["q"]
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    fa.attention_forward(q, dev["k"], dev["v"], causal, scale, out=out, lse=lse)
    status = fa.fa_get_device_error()
    assert status == fa.FA_OK, fa.fa_strerror(status)
    return out, lse


def run_backward(dev, out, lse, causal, scale):
    q = dev["q"]
    nan = float("nan")
    dq, dk, dv = (torch.full_like(q, nan) for _ in range(3))
    need = fa.fa_bwd_workspace_size(*q.shape)
    ws = torch.full((need // 4,), nan, dtype=torch.float32, device=q.device)
    fa.attention_backward(q, dev["k"], dev["v"], out, lse, dev["dO"], causal,
                          scale, dq=dq, dk=dk, dv=dv, workspace=ws)
    status = fa.fa_get_device_error()
    assert status == fa.FA_OK, fa.fa_strerror(status)
    return dq, dk, dv


def check_forward_full(host, o, lse, causal, scale):
    """Whole-tensor comparison; returns a dict of error figures."""
    o_ref, lse_ref = oracle.ref_fwd(to_f64(host["q"]), to_f64(host["k"]),
                                    to_f64(host["v"]), causal, scale)
    o_gpu = to_f64(o.cpu())
    lse_gpu = lse.cpu().double().numpy()
    res = {"o_excess": max_excess(o_gpu, o_ref), "o_max": max_abs(o_gpu, o_ref),
           "o_rel_l2": rel_l2(o_gpu, o_ref), "lse_max": max_abs(lse_gpu, lse_ref),
           "o_floor": bf16_floor(o_ref)}
    assert res["o_excess"] <= TOL_O_MAX, res
    assert res["o_rel_l2"] <= TOL_O_REL_L2, res
    assert res["lse_max"] <= TOL_LSE_MAX, res
    return res


def sample_rows(N, count, rng):
    fixed = [0, 1, 63, 64, 127, 128, 129, 255, 256, N - 2, N - 1]
    rows = set(r for r in fixed if 0 <= r < N)
    rows.update(rng.choice(N, size=min(count, N), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def check_forward_sampled(host, o, lse, causal, scale, heads, rows_per_head, seed=0):
    """Exact oracle rows for a sample of (head, row) pairs at any N."""
    B, H, N, d = host["q"].shape
    rng = np.random.default_rng(seed)
    q, k, v = (host[x].reshape(B * H, N, d) for x in "qkv")
    o_gpu = o.reshape(B * H, N, d)
    lse_gpu = lse.reshape(B * H, N)
    worst = {"o_excess": 0.0, "o_max": 0.0, "lse_max": 0.0, "o_rel_l2": 0.0}
    for bh in heads:
        rows = sample_rows(N, rows_per_head, rng)
        o_ref, l_ref = oracle.ref_fwd_rows(to_f64(q[bh]), to_f64(k[bh]),
                                           to_f64(v[bh]), rows, causal, scale)
        og = to_f64(o_gpu[bh][torch.from_numpy(rows).to(o.device)].cpu())
        lg = lse_gpu[bh][torch.from_numpy(rows).to(o.device)].cpu().double().numpy()
        worst["o_excess"] = max(worst["o_excess"], max_excess(og, o_ref))
        worst["o_max"] = max(worst["o_max"], max_abs(og, o_ref))
        worst["o_rel_l2"] = max(worst["o_rel_l2"], rel_l2(og, o_ref))
        worst["lse_max"] = max(worst["lse_max"], max_abs(lg, l_ref))
    assert worst["o_excess"] <= TOL_O_MAX, worst
    assert worst["o_rel_l2"] <= TOL_O_REL_L2, worst
    assert worst["lse_max"] <= TOL_LSE_MAX, worst
    return worst


def check_backward_heads(host, dq, dk, dv, causal, scale, heads):
    """Whole-head gradient comparison for the listed (flattened) heads."""
    B, H, N, d = host["q"].shape
    flat = {x: host[x].reshape(B * H, 1, N, d) for x in ("q", "k", "v", "dO")}
    res = {f"{n}_{m}": 0.0 for n in ("dq", "dk", "dv") for m in ("excess", "max")}
    res["floor"] = 0.0
    for bh in heads:
        args = [to_f64(flat[x][bh:bh + 1]) for x in ("q", "k", "v", "dO")]
        rq, rk, rv, _ = oracle.ref_bwd(*args, causal, scale)
        for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            g = to_f64(got.reshape(B * H, 1, N, d)[bh:bh + 1].cpu())
            res[name + "_excess"] = max(res[name + "_excess"], max_excess(g, ref))
            res[name + "_max"] = max(res[name + "_max"], max_abs(g, ref))
            res["floor"] = max(res["floor"], bf16_floor(ref))
    for name in ("dq", "dk", "dv"):
        assert res[name + "_excess"] <= TOL_GRAD_MAX, res
    return res


def check_backward_sampled(host, dq, dk, dv, causal, scale, heads, rows_per_head, seed=0):
    """Exact oracle dQ rows and dK/dV rows for sampled rows of whole heads."""
    B, H, N, d = host["q"].shape
    rng = np.random.default_rng(seed)
    flat = {x: host[x].reshape(B * H, N, d) for x in ("q", "k", "v", "dO")}
    res = {f"{n}_{m}": 0.0 for n in ("dq", "dk", "dv") for m in ("excess", "max")}
    for bh in heads:
        q, k, v, dO = (to_f64(flat[x][bh]) for x in ("q", "k", "v", "dO"))
        rows = sample_rows(N, rows_per_head, rng)
        idx = torch.from_numpy(rows)
        lse_h, D_h = oracle.ref_head_stats(q, k, v, dO, causal, scale)
        rdq = oracle.ref_dq_rows(q, k, v, dO, rows, causal, scale)
        rdk, rdv = oracle.ref_dkdv_rows(q, k, v, dO, lse_h, D_h, rows, causal, scale)
        for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            g = to_f64(got.reshape(B * H, N, d)[bh].cpu()[idx])
            res[name + "_excess"] = max(res[name + "_excess"], max_excess(g, ref))
            res[name + "_max"] = max(res[name + "_max"], max_abs(g, ref))
    for name in ("dq", "dk", "dv"):
        assert res[name + "_excess"] <= TOL_GRAD_MAX, res
    return res


def check_backward_causal_tail(host, dq, dk, dv, scale, heads, rows_per_head, tail, seed=0):
    """Causal mask at large N: exact oracle dQ for sampled query rows anywhere
    in each listed head, and exact dK/dV for sampled key rows among the last
    ``tail`` keys, which only meet the last ``tail`` queries (so the oracle
    needs the softmax statistics of those rows alone)."""
    B, H, N, d = host["q"].shape
    first = N - tail
    rng = np.random.default_rng(seed)
    flat = {x: host[x].reshape(B * H, N, d) for x in ("q", "k", "v", "dO")}
    res = {f"{n}_{m}": 0.0 for n in ("dq", "dk", "dv") for m in ("excess", "max")}
    for bh in heads:
        q, k, v, dO = (to_f64(flat[x][bh]) for x in ("q", "k", "v", "dO"))
        q_rows = sample_rows(N, rows_per_head, rng)
        k_rows = first + sample_rows(tail, rows_per_head, rng)
        lse_h, D_h = oracle.ref_head_stats(q, k, v, dO, True, scale, first=first)
        rdq = oracle.ref_dq_rows(q, k, v, dO, q_rows, True, scale)
        rdk, rdv = oracle.ref_dkdv_rows(q, k, v, dO, lse_h, D_h, k_rows, True, scale)
        for name, got, ref, rows in (("dq", dq, rdq, q_rows), ("dk", dk, rdk, k_rows),
                                     ("dv", dv, rdv, k_rows)):
            g = to_f64(got.reshape(B * H, N, d)[bh].cpu()[torch.from_numpy(rows)])
            res[name + "_excess"] = max(res[name + "_excess"], max_excess(g, ref))
            res[name + "_max"] = max(res[name + "_max"], max_abs(g, ref))
    for name in ("dq", "dk", "dv"):
        assert res[name + "_excess"] <= TOL_GRAD_MAX, res
    return res
