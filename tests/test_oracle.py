"""Pins for the fp64 CPU oracle (no GPU).

The oracle is the plain definition of attention (FlashAttention-2 abstract:
exact, "no approximation"); these tests tie it to things it does not compute
itself:

* brute force in 50-digit arithmetic (mpmath), summing exp(s) directly with no
  max shift, on tiny inputs -- forward O and LSE;
* numerical derivatives of L = sum(O * dO) of that brute force (central
  differences at 60 digits) -- all three gradients;
* an independent library routine (torch's fp64 scaled_dot_product_attention
  and autograd) at moderate sizes;
* closed forms: identical V rows, Q = 0, causal row 0, N = 1, a hand-derived
  two-key example (``tests/golden/worked_examples.txt``);
* invariants: rows of P sum to one, shift and permutation invariance,
  sum_j dV_j = sum_i dO_i, sum_j dK_j = 0, D_i = <dO_i, O_i>;
* the blockwise statement of the iplexlaw FlashAttention-2 blog ("Tiling
  preserves the attention calculation"): an online softmax that rescales its
  running statistics reproduces the oracle, while normalising each block on its
  own and adding does not;
* planted mistakes: each of several plausible slips, written into a copy of the
  oracle's C source, makes at least one pin fail.
"""
import math
import os
import re
import subprocess
import tempfile

import mpmath as mp
import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------------------
# independent references
# ----------------------------------------------------------------------------

def brute_forward(q, k, v, causal, scale, dps=50):
    """O and LSE of one head by direct high-precision summation (no max shift)."""
    with mp.workdps(dps):
        N, d = q.shape
        Q = [[mp.mpf(float(x)) for x in row] for row in q]
        K = [[mp.mpf(float(x)) for x in row] for row in k]
        V = [[mp.mpf(float(x)) for x in row] for row in v]
        sc = mp.mpf(float(scale))
        O = []
        LSE = []
        for i in range(N):
            keys = range(i + 1) if causal else range(N)
            w = [mp.exp(sc * mp.fsum(Q[i][t] * K[j][t] for t in range(d)))
                 for j in keys]
            Z = mp.fsum(w)
            O.append([mp.fsum(w[a] * V[j][t] for a, j in enumerate(keys)) / Z
                      for t in range(d)])
            LSE.append(mp.log(Z))
        return O, LSE


def brute_loss(q, k, v, dO, causal, scale):
    O, _ = brute_forward(q, k, v, causal, scale, dps=60)
    with mp.workdps(60):
        return mp.fsum(O[i][t] * mp.mpf(float(dO[i, t]))
                       for i in range(q.shape[0]) for t in range(q.shape[1]))


def numeric_grads(q, k, v, dO, causal, scale, h=mp.mpf("1e-25")):
    """Central differences of L = sum(O * dO) through the brute force."""
    grads = []
    with mp.workdps(60):
        for which in range(3):
            base = [q, k, v]
            g = np.zeros_like(base[which])
            for idx in np.ndindex(*base[which].shape):
                vals = []
                for sgn in (1, -1):
                    arrs = [np.array(a, dtype=object) for a in base]
                    arrs[which][idx] = mp.mpf(float(base[which][idx])) + sgn * h
                    vals.append(_brute_loss_obj(arrs, dO, causal, scale))
                g[idx] = float((vals[0] - vals[1]) / (2 * h))
            grads.append(g)
    return grads


def _brute_loss_obj(arrs, dO, causal, scale):
    q, k, v = arrs
    N, d = q.shape
    sc = mp.mpf(float(scale))
    total = mp.mpf(0)
    for i in range(N):
        keys = range(i + 1) if causal else range(N)
        w = [mp.exp(sc * mp.fsum(mp.mpf(q[i, t]) * mp.mpf(k[j, t])
                                  for t in range(d))) for j in keys]
        Z = mp.fsum(w)
        for t in range(d):
            o = mp.fsum(w[a] * mp.mpf(v[j, t]) for a, j in enumerate(keys)) / Z
            total += o * mp.mpf(float(dO[i, t]))
    return total


def torch_sdpa(q, k, v, dO, causal, scale):
    """torch's fp64 scaled_dot_product_attention forward and autograd grads."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=bool(causal), scale=float(scale))
    o.backward(torch.tensor(dO, dtype=torch.float64))
    return (o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(),
            tv.grad.numpy())


def rng_inputs(seed, B, H, N, d):
    r = np.random.default_rng(seed)
    return [r.standard_normal((B, H, N, d)) for _ in range(4)]


def rel_err(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ----------------------------------------------------------------------------
# the pin suite, written so the planted-mistake test can rerun it on a mutant
# ----------------------------------------------------------------------------

def pin_brute_forward(lib=None, tol=1e-13):
    failures = []
    for seed, (N, d) in enumerate([(1, 3), (3, 2), (7, 4), (8, 1)]):
        q, k, v, _ = rng_inputs(seed, 1, 2, N, d)
        for causal in (False, True):
            scale = 0.7
            o, lse = oracle.ref_fwd(q, k, v, causal, scale, lib=lib)
            for h in range(2):
                O, L = brute_forward(q[0, h], k[0, h], v[0, h], causal, scale)
                eo = rel_err(o[0, h], np.array(O, dtype=np.float64))
                el = rel_err(lse[0, h], np.array(L, dtype=np.float64))
                if not (eo <= tol and el <= tol):
                    failures.append((N, d, causal, h, eo, el))
                rows = np.arange(N)[::-1]
                o_r, l_r = oracle.ref_fwd_rows(q[0, h], k[0, h], v[0, h], rows,
                                               causal, scale, lib=lib)
                if not (rel_err(o_r, np.array(O, dtype=np.float64)[rows]) <= tol
                        and rel_err(l_r, np.array(L, dtype=np.float64)[rows]) <= tol):
                    failures.append(("rows", N, d, causal, h))
    return failures


def pin_numeric_grads(lib=None, tol=1e-11):
    failures = []
    for seed, (N, d) in enumerate([(5, 3), (4, 2)]):
        q, k, v, dO = rng_inputs(100 + seed, 1, 1, N, d)
        for causal in (False, True):
            scale = 0.9
            dq, dk, dv, D = oracle.ref_bwd(q, k, v, dO, causal, scale, lib=lib)
            gq, gk, gv = numeric_grads(q[0, 0], k[0, 0], v[0, 0], dO[0, 0],
                                       causal, scale)
            errs = [rel_err(dq[0, 0], gq), rel_err(dk[0, 0], gk),
                    rel_err(dv[0, 0], gv)]
            if max(errs) > tol:
                failures.append((N, d, causal, errs))
            # the sampled-row entry points reproduce the same gradients
            rows = np.arange(N)
            lse, Dh = oracle.ref_head_stats(q[0, 0], k[0, 0], v[0, 0], dO[0, 0],
                                            causal, scale, lib=lib)
            dq_r = oracle.ref_dq_rows(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], rows,
                                      causal, scale, lib=lib)
            dk_r, dv_r = oracle.ref_dkdv_rows(q[0, 0], k[0, 0], v[0, 0],
                                              dO[0, 0], lse, Dh, rows, causal,
                                              scale, lib=lib)
            errs = [rel_err(dq_r, gq), rel_err(dk_r, gk), rel_err(dv_r, gv)]
            if max(errs) > tol:
                failures.append(("rows", N, d, causal, errs))
    return failures


def pin_library_routine(lib=None, tol=1e-12):
    failures = []
    for causal in (False, True):
        q, k, v, dO = rng_inputs(7, 2, 2, 67, 16)
        scale = 0.25
        o, _ = oracle.ref_fwd(q, k, v, causal, scale, lib=lib)
        dq, dk, dv, _ = oracle.ref_bwd(q, k, v, dO, causal, scale, lib=lib)
        to, tdq, tdk, tdv = torch_sdpa(q, k, v, dO, causal, scale)
        errs = [rel_err(o, to), rel_err(dq, tdq), rel_err(dk, tdk),
                rel_err(dv, tdv)]
        if max(errs) > tol:
            failures.append((causal, errs))
    return failures


# ----------------------------------------------------------------------------
# tests
# ----------------------------------------------------------------------------

def test_brute_force_forward():
    assert pin_brute_forward() == []


def test_numeric_gradients():
    assert pin_numeric_grads() == []


def test_library_routine():
    assert pin_library_routine() == []


def _parse_worked_examples():
    path = os.path.join(HERE, "golden", "worked_examples.txt")
    cases = []
    cur = {}
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        key, val = [s.strip() for s in line.split("=", 1)]
        if key == "case":
            if cur:
                cases.append(cur)
            cur = {"name": val}
        else:
            cur[key] = val
    if cur:
        cases.append(cur)
    return cases


def _eval_expr(s):
    return eval(s, {"__builtins__": {}}, {"ln": math.log, "exp": math.exp,
                                         "sqrt": math.sqrt})


@pytest.mark.parametrize("case", _parse_worked_examples(), ids=lambda c: c["name"])
def test_worked_examples(case):
    """Hand-derived examples (derivations in the fixture file)."""
    N, d = int(case["N"]), int(case["d"])
    def mat(key):
        vals = [_eval_expr(x) for x in case[key].split(",")]
        return np.array(vals, dtype=np.float64).reshape(1, 1, N, d)
    q, k, v = mat("q"), mat("k"), mat("v")
    causal = case["causal"] == "1"
    scale = _eval_expr(case["scale"])
    o, lse = oracle.ref_fwd(q, k, v, causal, scale)
    O_exp = np.array([_eval_expr(x) for x in case["O"].split(",")]).reshape(N, d)
    L_exp = np.array([_eval_expr(x) for x in case["LSE"].split(",")])
    np.testing.assert_allclose(o[0, 0], O_exp, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], L_exp, rtol=1e-14, atol=1e-14)
    if "dO" in case:
        dO = mat("dO")
        dq, dk, dv, D = oracle.ref_bwd(q, k, v, dO, causal, scale)
        for key, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
            exp_ = np.array([_eval_expr(x) for x in case[key].split(",")])
            np.testing.assert_allclose(got[0, 0].ravel(), exp_, rtol=1e-13,
                                       atol=1e-14, err_msg=key)


def test_identical_value_rows():
    q, k, v, _ = rng_inputs(11, 1, 2, 50, 8)
    v[:] = v[:, :, :1, :]
    for causal in (False, True):
        o, _ = oracle.ref_fwd(q, k, v, causal, 0.5)
        np.testing.assert_allclose(o, np.broadcast_to(v[:, :, :1, :], o.shape),
                                   rtol=0, atol=1e-14)


def test_zero_query_gives_mean_of_values():
    _, k, v, _ = rng_inputs(12, 2, 1, 40, 6)
    q = np.zeros_like(k)
    o, lse = oracle.ref_fwd(q, k, v, False, 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True),
                                                  o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, np.log(40.0), atol=1e-14)
    o, lse = oracle.ref_fwd(q, k, v, True, 0.3)
    counts = np.arange(1, 41, dtype=np.float64)
    prefix = np.cumsum(v, axis=2) / counts[None, None, :, None]
    np.testing.assert_allclose(o, prefix, atol=1e-14)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(counts), lse.shape),
                               atol=1e-14)


def test_causal_row_zero_and_single_key():
    q, k, v, _ = rng_inputs(13, 1, 3, 30, 5)
    o, lse = oracle.ref_fwd(q, k, v, True, 0.4)
    np.testing.assert_array_equal(o[:, :, 0, :], v[:, :, 0, :])
    s00 = 0.4 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=1e-15, atol=1e-15)
    # N = 1: the single key gets all the weight, causal or not
    for causal in (False, True):
        o1, l1 = oracle.ref_fwd(q[:, :, :1], k[:, :, :1], v[:, :, :1], causal, 0.4)
        np.testing.assert_array_equal(o1, v[:, :, :1])
        np.testing.assert_allclose(l1, s00[..., None], rtol=1e-15, atol=1e-15)


def test_probability_rows_sum_to_one():
    q, k, v, _ = rng_inputs(14, 1, 2, 33, 4)
    v[..., 2] = 1.0
    for causal in (False, True):
        o, _ = oracle.ref_fwd(q, k, v, causal, 1.3)
        np.testing.assert_allclose(o[..., 2], 1.0, rtol=0, atol=2e-15)


def test_key_shift_invariance():
    q, k, v, _ = rng_inputs(15, 1, 2, 45, 8)
    u = np.random.default_rng(0).standard_normal(8)
    scale = 0.35
    for causal in (False, True):
        o, lse = oracle.ref_fwd(q, k, v, causal, scale)
        o2, lse2 = oracle.ref_fwd(q, k + u, v, causal, scale)
        np.testing.assert_allclose(o2, o, atol=1e-13)
        np.testing.assert_allclose(lse2 - lse, scale * (q @ u), atol=1e-12)


def test_key_value_permutation_equivariance():
    q, k, v, dO = rng_inputs(16, 1, 2, 37, 8)
    perm = np.random.default_rng(1).permutation(37)
    o, lse = oracle.ref_fwd(q, k, v, False, 0.5)
    o2, lse2 = oracle.ref_fwd(q, k[:, :, perm], v[:, :, perm], False, 0.5)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    _, dk, dv, _ = oracle.ref_bwd(q, k, v, dO, False, 0.5)
    _, dk2, dv2, _ = oracle.ref_bwd(q, k[:, :, perm], v[:, :, perm], dO, False, 0.5)
    np.testing.assert_allclose(dk2, dk[:, :, perm], atol=1e-13)
    np.testing.assert_allclose(dv2, dv[:, :, perm], atol=1e-13)


def test_gradient_invariants():
    q, k, v, dO = rng_inputs(17, 2, 2, 70, 16)
    for causal in (False, True):
        o, _ = oracle.ref_fwd(q, k, v, causal, 0.25)
        dq, dk, dv, D = oracle.ref_bwd(q, k, v, dO, causal, 0.25)
        # P rows sum to one, so the value gradients add up to the upstream sum
        np.testing.assert_allclose(dv.sum(axis=2), dO.sum(axis=2), atol=1e-12)
        # each row of dS sums to zero, hence the key gradients cancel
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        # D_i = sum_j P_ij dP_ij equals <dO_i, O_i>
        np.testing.assert_allclose(D, np.einsum("bhnd,bhnd->bhn", dO, o),
                                   atol=1e-12)


def _online_softmax_blocks(q, k, v, causal, scale, block, normalise_each=False):
    """The tiled computation described on the blog, on one head (numpy)."""
    N, d = q.shape
    O = np.zeros((N, d))
    LSE = np.zeros(N)
    for i in range(N):
        m, l, acc = -np.inf, 0.0, np.zeros(d)
        hi = i + 1 if causal else N
        for j0 in range(0, hi, block):
            j1 = min(j0 + block, hi)
            s = scale * (k[j0:j1] @ q[i])
            if normalise_each:
                p = np.exp(s - s.max())
                acc += (p / p.sum()) @ v[j0:j1]
                continue
            m_new = max(m, s.max())
            alpha = np.exp(m - m_new) if np.isfinite(m) else 0.0
            p = np.exp(s - m_new)
            l = alpha * l + p.sum()
            acc = alpha * acc + p @ v[j0:j1]
            m = m_new
        O[i] = acc if normalise_each else acc / l
        LSE[i] = m + np.log(l) if not normalise_each else np.nan
    return O, LSE


def test_online_softmax_matches_and_blockwise_normalisation_does_not():
    q, k, v, _ = rng_inputs(18, 1, 1, 64, 8)
    for causal in (False, True):
        o, lse = oracle.ref_fwd(q, k, v, causal, 0.6)
        O, L = _online_softmax_blocks(q[0, 0], k[0, 0], v[0, 0], causal, 0.6, 16)
        np.testing.assert_allclose(O, o[0, 0], atol=1e-12)
        np.testing.assert_allclose(L, lse[0, 0], atol=1e-12)
        Obad, _ = _online_softmax_blocks(q[0, 0], k[0, 0], v[0, 0], causal, 0.6,
                                         16, normalise_each=True)
        assert np.max(np.abs(Obad - o[0, 0])) > 1e-2


def test_tail_head_stats_serve_causal_tail_key_rows():
    """Statistics of the rows from `first` on equal the full ones there (NaN
    before), and under the causal mask they give the full dK/dV of the key
    rows from `first` on, since those keys only meet the later queries."""
    q, k, v, dO = rng_inputs(23, 1, 1, 150, 8)
    first = 97
    lse_f, D_f = oracle.ref_head_stats(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], True, 0.3)
    lse_t, D_t = oracle.ref_head_stats(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], True, 0.3,
                                       first=first)
    assert np.all(np.isnan(lse_t[:first])) and np.all(np.isnan(D_t[:first]))
    np.testing.assert_array_equal(lse_t[first:], lse_f[first:])
    np.testing.assert_array_equal(D_t[first:], D_f[first:])
    _, dk, dv, _ = oracle.ref_bwd(q, k, v, dO, True, 0.3)
    rows = np.array([first, 120, 149])
    dk_r, dv_r = oracle.ref_dkdv_rows(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], lse_t, D_t,
                                      rows, True, 0.3)
    np.testing.assert_allclose(dk_r, dk[0, 0, rows], atol=1e-13)
    np.testing.assert_allclose(dv_r, dv[0, 0, rows], atol=1e-13)
    with pytest.raises(ValueError):
        oracle.ref_head_stats(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], True, 0.3, first=151)


def test_sampled_rows_match_full_tensors():
    q, k, v, dO = rng_inputs(19, 1, 1, 150, 8)
    rows = np.array([0, 1, 63, 64, 127, 128, 149])
    for causal in (False, True):
        o, lse = oracle.ref_fwd(q, k, v, causal, 0.3)
        dq, dk, dv, D = oracle.ref_bwd(q, k, v, dO, causal, 0.3)
        o_r, l_r = oracle.ref_fwd_rows(q[0, 0], k[0, 0], v[0, 0], rows, causal, 0.3)
        np.testing.assert_allclose(o_r, o[0, 0, rows], atol=1e-14)
        np.testing.assert_allclose(l_r, lse[0, 0, rows], atol=1e-14)
        lse_h, D_h = oracle.ref_head_stats(q[0, 0], k[0, 0], v[0, 0], dO[0, 0],
                                           causal, 0.3)
        np.testing.assert_allclose(lse_h, lse[0, 0], atol=1e-14)
        np.testing.assert_allclose(D_h, D[0, 0], atol=1e-13)
        np.testing.assert_allclose(
            oracle.ref_dq_rows(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], rows, causal,
                               0.3), dq[0, 0, rows], atol=1e-13)
        dk_r, dv_r = oracle.ref_dkdv_rows(q[0, 0], k[0, 0], v[0, 0], dO[0, 0],
                                          lse_h, D_h, rows, causal, 0.3)
        np.testing.assert_allclose(dk_r, dk[0, 0, rows], atol=1e-13)
        np.testing.assert_allclose(dv_r, dv[0, 0, rows], atol=1e-13)


def test_empty_sequence():
    z = np.zeros((1, 2, 0, 8))
    o, lse = oracle.ref_fwd(z, z, z, True, 0.5)
    assert o.shape == (1, 2, 0, 8) and lse.shape == (1, 2, 0)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of the C source must fail at least one pin
# ----------------------------------------------------------------------------

MUTANTS = {
    "lse_drops_max": ("return m + log(z);", "return log(z);"),
    "causal_off_by_one": ("return causal ? i + 1 : N;", "return causal ? i : N;"),
    "softmax_grad_sign": ("const double ds = p[j] * (dp[j] - Di);",
                          "const double ds = p[j] * (dp[j] + Di);"),
    "dk_wrong_operand": ("dk_j[t] += ds * q_i[t];", "dk_j[t] += ds * k_j[t];"),
    "dq_missing_scale": ("for (int t = 0; t < d; ++t) dq_i[t] *= scale;", ""),
    "dv_wrong_operand": ("dv_j[t] += p[j] * do_i[t];", "dv_j[t] += p[j] * q_i[t];"),
    "no_normalisation": ("for (int j = 0; j < n; ++j) p[j] /= z;", ""),
    "dkdv_rows_skip_diagonal": ("for (int i = causal ? j : 0; i < N; ++i)",
                                "for (int i = causal ? j + 1 : 0; i < N; ++i)"),
    "rows_dq_drops_D": ("const double ds = p[j] * (dp[j] - Di);\n                for",
                        "const double ds = p[j] * dp[j];\n                for"),
    "decode_extent_off_by_one": ("const int n = causal ? i + offset + 1 : Nk;",
                                 "const int n = causal ? i + offset : Nk;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__),
                            "attention_ref.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "mutant.so"
    c_path.write_text(mutated)
    oracle.build(str(c_path), str(so_path))
    lib = oracle.open_library(str(so_path))
    with np.errstate(all="ignore"):
        caught = bool(pin_brute_forward(lib) or pin_numeric_grads(lib)
                      or pin_library_routine(lib) or pin_decode(lib))
    assert caught, f"planted mistake {name} passed every pin"


# ----------------------------------------------------------------------------
# decoding: Nq queries against Nk >= Nq keys, causal diagonal ending at the
# last key
# ----------------------------------------------------------------------------

def brute_decode(q, k, v, causal, scale, dps=50):
    """Direct 50-digit summation for Nq queries against Nk keys."""
    Nq, Nk, d = q.shape[0], k.shape[0], q.shape[1]
    O, L = [], []
    with mp.workdps(dps):
        sc = mp.mpf(float(scale))
        for i in range(Nq):
            n = i + Nk - Nq + 1 if causal else Nk
            w = [mp.exp(sc * mp.fsum(mp.mpf(float(q[i, t])) * mp.mpf(float(k[j, t]))
                                      for t in range(d))) for j in range(n)]
            Z = mp.fsum(w)
            O.append([float(mp.fsum(w[j] * mp.mpf(float(v[j, t])) for j in range(n)) / Z)
                      for t in range(d)])
            L.append(float(mp.log(Z)))
    return np.array(O, dtype=np.float64), np.array(L, dtype=np.float64)


def pin_decode(lib=None, tol=1e-13):
    failures = []
    for seed, (Nq, Nk, d) in enumerate([(1, 9, 3), (3, 7, 2), (4, 4, 4), (2, 11, 1)]):
        q, _, _, _ = rng_inputs(300 + seed, 1, 2, Nq, d)
        _, k, v, _ = rng_inputs(400 + seed, 1, 2, Nk, d)
        for causal in (False, True):
            o, lse = oracle.ref_fwd_decode(q, k, v, causal, 0.8, lib=lib)
            for h in range(2):
                O, L = brute_decode(q[0, h], k[0, h], v[0, h], causal, 0.8)
                if not (rel_err(o[0, h], O) <= tol and rel_err(lse[0, h], L) <= tol):
                    failures.append((Nq, Nk, d, causal, h))
    return failures


def test_decode_brute_force():
    assert pin_decode() == []


def test_decode_library_routine():
    q, _, _, _ = rng_inputs(500, 2, 3, 5, 16)
    _, k, v, _ = rng_inputs(501, 2, 3, 77, 16)
    for causal in (False, True):
        mask = None
        if causal:
            i = np.arange(5)[:, None]
            j = np.arange(77)[None, :]
            mask = torch.tensor(j <= i + 77 - 5)
        to = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=mask, scale=0.3)
        o, _ = oracle.ref_fwd_decode(q, k, v, causal, 0.3)
        assert rel_err(o, to.numpy()) <= 1e-12


def test_decode_closed_forms():
    _, k, v, _ = rng_inputs(502, 1, 2, 30, 6)
    q = np.zeros((1, 2, 4, 6))
    o, lse = oracle.ref_fwd_decode(q, k, v, True, 0.5)
    for i in range(4):            # Q = 0: mean of the visible values
        n = i + 30 - 4 + 1
        np.testing.assert_allclose(o[:, :, i], v[:, :, :n].mean(axis=2), atol=1e-14)
        np.testing.assert_allclose(lse[:, :, i], np.log(n), atol=1e-14)
    # the last query sees every key, causal or not; Nq == Nk reduces to ref_fwd
    q, k, v, _ = rng_inputs(503, 1, 2, 12, 5)
    oc, lc = oracle.ref_fwd_decode(q[:, :, -1:], k, v, True, 0.7)
    on, ln = oracle.ref_fwd_decode(q[:, :, -1:], k, v, False, 0.7)
    np.testing.assert_allclose(oc, on, atol=0)
    for causal in (False, True):
        a, la = oracle.ref_fwd_decode(q, k, v, causal, 0.7)
        b, lb = oracle.ref_fwd(q, k, v, causal, 0.7)
        np.testing.assert_allclose(a, b, atol=0)
        np.testing.assert_allclose(la, lb, atol=0)
    with pytest.raises(ValueError):
        oracle.ref_fwd_decode(q, k[:, :, :5], v[:, :, :5], True, 0.7)


# ----------------------------------------------------------------------------
# ring steps: the log-sum-exp merge and gradients under whole-row statistics
# ----------------------------------------------------------------------------

def test_lse_merge_against_brute_force():
    """Merging brute-force attention over two disjoint key sets reproduces
    brute-force attention over their union (no max shift, 50 digits)."""
    q, k, v, _ = rng_inputs(600, 1, 1, 3, 4)
    _, k2, v2, _ = rng_inputs(601, 1, 1, 7, 4)
    kk = np.concatenate([k[0, 0], k2[0, 0]])
    vv = np.concatenate([v[0, 0], v2[0, 0]])
    for a in (1, 3, 6):
        oa, la = brute_decode(q[0, 0], kk[:a], vv[:a], False, 0.9)
        ob, lb = brute_decode(q[0, 0], kk[a:], vv[a:], False, 0.9)
        o_all, l_all = brute_decode(q[0, 0], kk, vv, False, 0.9)
        o, l = oracle.ref_lse_merge(oa, la, ob, lb)
        assert rel_err(o, o_all) <= 1e-13 and rel_err(l, l_all) <= 1e-13
        # either order, and a three-way split folded left to right
        o2, l2 = oracle.ref_lse_merge(ob, lb, oa, la)
        assert rel_err(o2, o_all) <= 1e-13 and rel_err(l2, l_all) <= 1e-13
    oa, la = brute_decode(q[0, 0], kk[:2], vv[:2], False, 0.9)
    ob, lb = brute_decode(q[0, 0], kk[2:5], vv[2:5], False, 0.9)
    oc, lc = brute_decode(q[0, 0], kk[5:], vv[5:], False, 0.9)
    o, l = oracle.ref_lse_merge(*oracle.ref_lse_merge(oa, la, ob, lb), oc, lc)
    o_all, l_all = brute_decode(q[0, 0], kk, vv, False, 0.9)
    assert rel_err(o, o_all) <= 1e-13 and rel_err(l, l_all) <= 1e-13


def test_lse_merge_reproduces_sharded_causal_attention():
    """The ring decomposition of causal attention: query shard r attends to key
    shards j < r in full and to shard r causally; merging the pieces gives
    ref_fwd over the whole sequence."""
    q, k, v, _ = rng_inputs(602, 2, 2, 24, 8)
    o_ref, l_ref = oracle.ref_fwd(q, k, v, True, 0.4)
    G, n = 3, 8
    for r in range(G):
        qs = q[:, :, r * n:(r + 1) * n]
        acc = None
        for j in range(r + 1):
            ks, vs = k[:, :, j * n:(j + 1) * n], v[:, :, j * n:(j + 1) * n]
            part = oracle.ref_fwd(qs, ks, vs, j == r, 0.4)
            acc = part if acc is None else oracle.ref_lse_merge(*acc, *part)
        assert rel_err(acc[0], o_ref[:, :, r * n:(r + 1) * n]) <= 1e-12
        assert rel_err(acc[1], l_ref[:, :, r * n:(r + 1) * n]) <= 1e-12


def test_grads_given_stats_sum_to_full_gradient():
    """Per-shard gradients under the whole rows' LSE and D add up to ref_bwd
    (itself pinned to numerical derivatives above); with one block they are
    ref_bwd."""
    q, k, v, dO = rng_inputs(603, 1, 2, 24, 8)
    for causal in (False, True):
        o, lse = oracle.ref_fwd(q, k, v, causal, 0.35)
        D = np.sum(o * dO, axis=-1)
        rq, rk, rv, _ = oracle.ref_bwd(q, k, v, dO, causal, 0.35)
        gq, gk, gv = oracle.ref_grads_given_stats(q, k, v, dO, lse, D, causal, 0.35)
        assert rel_err(gq, rq) <= 1e-12 and rel_err(gk, rk) <= 1e-12 and rel_err(gv, rv) <= 1e-12
        G, n = 3, 8
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        for r in range(G):
            rs = slice(r * n, (r + 1) * n)
            for j in range(G):
                if causal and j > r:
                    continue
                js = slice(j * n, (j + 1) * n)
                a, b, c = oracle.ref_grads_given_stats(
                    q[:, :, rs], k[:, :, js], v[:, :, js], dO[:, :, rs], lse[:, :, rs],
                    D[:, :, rs], causal and j == r, 0.35)
                dq[:, :, rs] += a
                dk[:, :, js] += b
                dv[:, :, js] += c
        assert rel_err(dq, rq) <= 1e-12, causal
        assert rel_err(dk, rk) <= 1e-12, causal
        assert rel_err(dv, rv) <= 1e-12, causal


# ----------------------------------------------------------------------------
# additive score bias
# ----------------------------------------------------------------------------

def test_bias_zero_and_mask_reduce_to_plain_attention():
    q, k, v, dO = rng_inputs(700, 2, 3, 9, 4)
    zero = np.zeros((1, 1, 9, 9))
    for causal in (False, True):
        o, l = oracle.ref_fwd_bias(q, k, v, zero, causal, 0.6)
        o2, l2 = oracle.ref_fwd(q, k, v, causal, 0.6)
        assert rel_err(o, o2) <= 1e-13 and rel_err(l, l2) <= 1e-13
        g = oracle.ref_bwd_bias(q, k, v, zero, dO, causal, 0.6)
        g2 = oracle.ref_bwd(q, k, v, dO, causal, 0.6)
        for a, b in zip(g[:3], g2[:3]):
            assert rel_err(a, b) <= 1e-12
    # a bias of -inf above the diagonal is the causal mask
    mask = np.where(np.arange(9)[None, :] > np.arange(9)[:, None], -np.inf, 0.0)[None, None]
    o, l = oracle.ref_fwd_bias(q, k, v, mask, False, 0.6)
    o2, l2 = oracle.ref_fwd(q, k, v, True, 0.6)
    assert rel_err(o, o2) <= 1e-13 and rel_err(l, l2) <= 1e-13


def test_bias_row_constant_shifts_lse_only():
    q, k, v, _ = rng_inputs(701, 1, 2, 7, 3)
    c = np.random.default_rng(1).standard_normal((1, 2, 7, 1)) * 3
    bias = np.broadcast_to(c, (1, 2, 7, 7)).copy()
    o, l = oracle.ref_fwd_bias(q, k, v, bias, True, 0.5)
    o2, l2 = oracle.ref_fwd(q, k, v, True, 0.5)
    assert rel_err(o, o2) <= 1e-13
    np.testing.assert_allclose(l, l2 + c[..., 0], atol=1e-13)


def test_bias_against_brute_force():
    q, k, v, _ = rng_inputs(702, 1, 1, 5, 3)
    bias = np.random.default_rng(2).standard_normal((1, 1, 5, 5)) * 2
    for causal in (False, True):
        o, l = oracle.ref_fwd_bias(q, k, v, bias, causal, 0.7)
        with mp.workdps(50):
            for i in range(5):
                keys = range(i + 1) if causal else range(5)
                w = [mp.exp(mp.mpf(0.7) * mp.fsum(mp.mpf(float(q[0, 0, i, t])) *
                                                   mp.mpf(float(k[0, 0, j, t])) for t in range(3))
                            + mp.mpf(float(bias[0, 0, i, j]))) for j in keys]
                Z = mp.fsum(w)
                assert abs(float(mp.log(Z)) - l[0, 0, i]) <= 1e-13
                for t in range(3):
                    ref = float(mp.fsum(w[a] * mp.mpf(float(v[0, 0, j, t]))
                                        for a, j in enumerate(keys)) / Z)
                    assert abs(ref - o[0, 0, i, t]) <= 1e-13


def test_bias_against_torch_autograd():
    """torch's fp64 SDPA with a float additive mask, and autograd for the
    gradients of q, k, v and the mask (broadcast over the batch)."""
    q, k, v, dO = rng_inputs(703, 2, 3, 11, 5)
    bias = np.random.default_rng(3).standard_normal((1, 3, 11, 11))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    tb = torch.tensor(bias, requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tb, scale=0.45)
    (out * torch.tensor(dO)).sum().backward()
    o, _ = oracle.ref_fwd_bias(q, k, v, bias, False, 0.45)
    dq, dk, dv, db = oracle.ref_bwd_bias(q, k, v, bias, dO, False, 0.45)
    assert rel_err(o, out.detach().numpy()) <= 1e-12
    assert rel_err(dq, tq.grad.numpy()) <= 1e-11
    assert rel_err(dk, tk.grad.numpy()) <= 1e-11
    assert rel_err(dv, tv.grad.numpy()) <= 1e-11
    # the broadcast bias's gradient is dBias summed over the batch
    assert rel_err(db.sum(axis=0, keepdims=True), tb.grad.numpy()) <= 1e-11


def test_bias_gradient_by_finite_differences():
    q, k, v, dO = rng_inputs(704, 1, 1, 6, 3)
    bias = np.random.default_rng(4).standard_normal((1, 1, 6, 6))
    _, _, _, db = oracle.ref_bwd_bias(q, k, v, bias, dO, True, 0.8)
    h = 1e-6
    for (i, j) in [(0, 0), (3, 1), (5, 5), (5, 2), (2, 2)]:
        bp, bm = bias.copy(), bias.copy()
        bp[0, 0, i, j] += h
        bm[0, 0, i, j] -= h
        lp = np.sum(oracle.ref_fwd_bias(q, k, v, bp, True, 0.8)[0] * dO)
        lm = np.sum(oracle.ref_fwd_bias(q, k, v, bm, True, 0.8)[0] * dO)
        assert abs((lp - lm) / (2 * h) - db[0, 0, i, j]) <= 1e-7
    assert np.all(db[0, 0][np.triu_indices(6, 1)] == 0)  # hidden pairs
    # with the exact O passed as o_given nothing changes
    o, _ = oracle.ref_fwd_bias(q, k, v, bias, True, 0.8)
    db2 = oracle.ref_bwd_bias(q, k, v, bias, dO, True, 0.8, o_given=o)[3]
    assert rel_err(db2, db) <= 1e-14


def test_dbias_with_bf16_rounded_o_stays_within_the_rounding_bound():
    """The dBias reference of the GPU tests takes D = rowsum(dO * O) from the
    oracle's own O rounded to bf16 (the format the backward receives O in).
    bf16 keeps 8 significant bits, so |bf16(x) - x| <= 2^-8 |x| and
    dS_ij moves by at most P_ij * 2^-8 * sum_d |dO_id| |O_id|.  This pins
    that reference to the exact-D one within that bound, and shows that the
    rounding really reaches it (the model is not the exact D in disguise)."""
    q, k, v, dO = rng_inputs(705, 2, 3, 24, 16)
    bias = np.random.default_rng(5).standard_normal((2, 3, 24, 24)) * 2
    for causal in (False, True):
        o, lse = oracle.ref_fwd_bias(q, k, v, bias, causal, 0.6)
        o_bf16 = torch.from_numpy(o).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.all(np.abs(o_bf16 - o) <= 2.0 ** -8 * np.abs(o))
        db_exact = oracle.ref_bwd_bias(q, k, v, bias, dO, causal, 0.6)[3]
        db_model = oracle.ref_bwd_bias(q, k, v, bias, dO, causal, 0.6, o_given=o_bf16)[3]
        s = 0.6 * np.einsum("bhid,bhjd->bhij", q, k) + bias
        if causal:
            s = np.where(np.arange(24)[None, :] > np.arange(24)[:, None], -np.inf, s)
        p = np.exp(s - lse[..., None])
        bound = p * 2.0 ** -8 * np.sum(np.abs(dO) * np.abs(o), axis=-1, keepdims=True)
        diff = np.abs(db_model - db_exact)
        assert np.all(diff <= bound * (1 + 1e-9) + 1e-15)
        assert diff.max() > 0.05 * bound.max()
