"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding, run the fp64 oracle on the same bf16 bits, and measure the error.

Tolerances (GPU result vs the fp64 oracle on the same seeded inputs):
  O:            max-abs <= 1e-2 and relative L2 <= 5e-3
  dQ, dK, dV:   max-abs <= 2e-2
  LSE:          max-abs <= 1e-3 (fp32 statistic; the kernel's error is ~1e-5)

The max-abs bounds are asserted on the raw error |gpu - ref| of every element
small enough for the bf16 output format to leave room for the arithmetic:
|ref| < 4 for O and |ref| < 2 for the gradients.  The error of a bf16 output
is its arithmetic error plus up to half an ulp of rounding; half an ulp is
2^-8 = 0.0039 for |x| in [1, 2), 2^-7 = 0.0078 in [2, 4) and 2^-6 = 0.0156
in [4, 8).  O's arithmetic stays within ~2e-3, so |ref| < 4 leaves it room.  The gradients'
arithmetic -- fp32 sums of products whose P and dS operands are rounded to
bf16, 2^-8 relative each, over up to N terms -- reaches ~0.016 at d = 64
with the causal mask (where dP = dO.v has standard deviation 8), so only
|ref| < 2 (half an ulp at most 2^-8 = 0.0039) leaves the bound for it.
From those magnitudes on the bound applies to the error in excess of that
element's own rounding, |gpu - ref| - |bf16(ref) - ref|.  Relative L2 is
always raw.  Every check records its figures -- raw max-abs over all
elements, over the raw-bound region and per magnitude band ([0,1), [1,2),
[2,4), [4,8), [8,inf)), the excess above the region, the bf16 floor,
relative L2 -- in ``parity_log``.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64
import parity_log

TOL_O_MAX = 1e-2
TOL_O_REL_L2 = 5e-3
TOL_GRAD_MAX = 2e-2
TOL_LSE_MAX = 1e-3
# Magnitude below which the max-abs bound holds for the raw error.
RAW_BELOW_O = 4.0
RAW_BELOW_GRAD = 2.0
BANDS = (0.0, 1.0, 2.0, 4.0, 8.0, float("inf"))


def bf16_round(ref: np.ndarray) -> np.ndarray:
    r = torch.from_numpy(np.ascontiguousarray(ref, dtype=np.float64))
    return r.to(torch.bfloat16).to(torch.float64).numpy()


def bf16_floor(ref: np.ndarray) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(bf16_round(ref) - ref))) if ref.size else 0.0


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    assert np.all(np.isfinite(a)), "non-finite values in GPU output"
    return float(np.max(np.abs(a - b)))


def max_excess(gpu, ref) -> float:
    """max over elements of |gpu - ref| - |bf16(ref) - ref|."""
    figs = error_figures(gpu, ref, raw_below=0.0)
    return figs["excess_above"]


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def error_figures(gpu, ref, raw_below: float) -> dict:
    """Raw max-abs over all elements ("max") and over |ref| < raw_below
    ("max_below"); max of |gpu-ref| - |bf16(ref)-ref| over |ref| >= raw_below
    ("excess_above", 0 when there is no such element); the bf16 floor
    max|bf16(ref) - ref| ("floor"); relative L2 ("rel_l2")."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if gpu.size == 0:
        return {"max": 0.0, "max_below": 0.0, "excess_above": 0.0, "floor": 0.0,
                "rel_l2": 0.0, "n_above": 0}
    assert np.all(np.isfinite(gpu)), "non-finite values in GPU output"
    err = np.abs(gpu - ref)
    floor = np.abs(bf16_round(ref) - ref)
    mag = np.abs(ref)
    below = mag < raw_below
    above = ~below
    figs = {
        "max": float(err.max()),
        "max_below": float(err[below].max()) if below.any() else 0.0,
        "excess_above": float((err - floor)[above].max()) if above.any() else 0.0,
        "floor": float(floor.max()),
        "rel_l2": rel_l2(gpu, ref),
        "n_above": int(above.sum()),
    }
    for lo, hi in zip(BANDS[:-1], BANDS[1:]):
        band = (mag >= lo) & (mag < hi)
        if band.any():
            figs[f"max_mag{lo:g}to{hi:g}"] = float(err[band].max())
    return figs


class Check:
    """Accumulates the figures of one parity check and the bounds they
    break; ``done()`` records them and fails the test on any breach."""

    def __init__(self):
        self.res: dict = {}
        self.fails: list = []

    def _merge(self, name, figs):
        for key, val in figs.items():
            k = f"{name}_{key}"
            self.res[k] = max(self.res.get(k, val), val)

    def output(self, name, gpu, ref, tol, raw_below, rel_tol=None):
        figs = error_figures(gpu, ref, raw_below)
        self._merge(name, figs)
        if figs["max_below"] > tol:
            self.fails.append(f"{name}: raw max-abs {figs['max_below']:.3g} > {tol} "
                              f"over |ref| < {raw_below}")
        if figs["excess_above"] > tol:
            self.fails.append(f"{name}: error beyond the bf16 floor "
                              f"{figs['excess_above']:.3g} > {tol} over |ref| >= {raw_below}")
        if rel_tol is not None and figs["rel_l2"] > rel_tol:
            self.fails.append(f"{name}: rel-L2 {figs['rel_l2']:.3g} > {rel_tol}")
        return figs

    def o(self, gpu, ref, name="o"):
        return self.output(name, gpu, ref, TOL_O_MAX, RAW_BELOW_O, TOL_O_REL_L2)

    def grad(self, name, gpu, ref):
        return self.output(name, gpu, ref, TOL_GRAD_MAX, RAW_BELOW_GRAD)

    def lse(self, gpu, ref, name="lse"):
        err = max_abs(gpu, ref)
        k = f"{name}_max"
        self.res[k] = max(self.res.get(k, err), err)
        if err > TOL_LSE_MAX:
            self.fails.append(f"{name}: max-abs {err:.3g} > {TOL_LSE_MAX}")
        return err

    def bound(self, name, value, limit):
        self.res[name] = max(self.res.get(name, value), value)
        if not value <= limit:
            self.fails.append(f"{name}: {value:.3g} > {limit}")

    def done(self):
        parity_log.record(self.res)
        assert not self.fails, (self.fails, self.res)
        return self.res


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
    """Whole-tensor comparison of O and LSE; returns the error figures."""
    o_ref, lse_ref = oracle.ref_fwd(to_f64(host["q"]), to_f64(host["k"]),
                                    to_f64(host["v"]), causal, scale)
    c = Check()
    c.o(to_f64(o.cpu()), o_ref)
    c.lse(lse.cpu().double().numpy(), lse_ref)
    return c.done()


def check_full(host, o, lse, dq, dk, dv, causal, scale):
    """Whole-tensor comparison of O, LSE, dQ, dK and dV (every element of
    every head) against one oracle forward and backward."""
    args = [to_f64(host[x]) for x in ("q", "k", "v")]
    o_ref, lse_ref = oracle.ref_fwd(*args, causal, scale)
    c = Check()
    c.o(to_f64(o.cpu()), o_ref)
    c.lse(lse.cpu().double().numpy(), lse_ref)
    del o_ref, lse_ref
    refs = oracle.ref_bwd(*args, to_f64(host["dO"]), causal, scale)[:3]
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        c.grad(name, to_f64(got.cpu()), ref)
    return c.done()


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
    c = Check()
    for bh in heads:
        rows = sample_rows(N, rows_per_head, rng)
        o_ref, l_ref = oracle.ref_fwd_rows(to_f64(q[bh]), to_f64(k[bh]),
                                           to_f64(v[bh]), rows, causal, scale)
        idx = torch.from_numpy(rows).to(o.device)
        c.o(to_f64(o_gpu[bh][idx].cpu()), o_ref)
        c.lse(lse_gpu[bh][idx].cpu().double().numpy(), l_ref)
    return c.done()


def check_backward_heads(host, dq, dk, dv, causal, scale, heads):
    """Whole-head gradient comparison for the listed (flattened) heads."""
    B, H, N, d = host["q"].shape
    flat = {x: host[x].reshape(B * H, 1, N, d) for x in ("q", "k", "v", "dO")}
    c = Check()
    for bh in heads:
        args = [to_f64(flat[x][bh:bh + 1]) for x in ("q", "k", "v", "dO")]
        rq, rk, rv, _ = oracle.ref_bwd(*args, causal, scale)
        for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            c.grad(name, to_f64(got.reshape(B * H, 1, N, d)[bh:bh + 1].cpu()), ref)
    return c.done()


def check_backward_sampled(host, dq, dk, dv, causal, scale, heads, rows_per_head, seed=0):
    """Exact oracle dQ rows and dK/dV rows for sampled rows of whole heads."""
    B, H, N, d = host["q"].shape
    rng = np.random.default_rng(seed)
    flat = {x: host[x].reshape(B * H, N, d) for x in ("q", "k", "v", "dO")}
    c = Check()
    for bh in heads:
        q, k, v, dO = (to_f64(flat[x][bh]) for x in ("q", "k", "v", "dO"))
        rows = sample_rows(N, rows_per_head, rng)
        idx = torch.from_numpy(rows)
        lse_h, D_h = oracle.ref_head_stats(q, k, v, dO, causal, scale)
        rdq = oracle.ref_dq_rows(q, k, v, dO, rows, causal, scale)
        rdk, rdv = oracle.ref_dkdv_rows(q, k, v, dO, lse_h, D_h, rows, causal, scale)
        for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            c.grad(name, to_f64(got.reshape(B * H, N, d)[bh].cpu()[idx]), ref)
    return c.done()


def check_backward_causal_tail(host, dq, dk, dv, scale, heads, rows_per_head, tail, seed=0):
    """Causal mask at large N: exact oracle dQ for sampled query rows anywhere
    in each listed head, and exact dK/dV for sampled key rows among the last
    ``tail`` keys, which only meet the last ``tail`` queries (so the oracle
    needs the softmax statistics of those rows alone)."""
    B, H, N, d = host["q"].shape
    first = N - tail
    rng = np.random.default_rng(seed)
    flat = {x: host[x].reshape(B * H, N, d) for x in ("q", "k", "v", "dO")}
    c = Check()
    for bh in heads:
        q, k, v, dO = (to_f64(flat[x][bh]) for x in ("q", "k", "v", "dO"))
        q_rows = sample_rows(N, rows_per_head, rng)
        k_rows = first + sample_rows(tail, rows_per_head, rng)
        lse_h, D_h = oracle.ref_head_stats(q, k, v, dO, True, scale, first=first)
        rdq = oracle.ref_dq_rows(q, k, v, dO, q_rows, True, scale)
        rdk, rdv = oracle.ref_dkdv_rows(q, k, v, dO, lse_h, D_h, k_rows, True, scale)
        for name, got, ref, rows in (("dq", dq, rdq, q_rows), ("dk", dk, rdk, k_rows),
                                     ("dv", dv, rdv, k_rows)):
            c.grad(name, to_f64(got.reshape(B * H, N, d)[bh].cpu()[torch.from_numpy(rows)]),
                   ref)
    return c.done()
