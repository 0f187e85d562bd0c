"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

The plain definition of scaled-dot-product attention and its gradient, in
double precision, written in C (``attention_ref.c``) and loaded here with
ctypes.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this package.  It shares no code with the CUDA library
and never calls it; the CUDA library never calls it either.

Every function takes float64 numpy arrays in the [B,H,N,d] layout (LSE and D
are [B,H,N]) and returns float64 arrays.  Bf16 inputs are widened exactly by
the caller, so the oracle sees the same values the GPU does.

Parity pins: every function here is pinned by ``tests/test_oracle.py`` against
quantities fixed by mathematics rather than by this code (high-precision brute
force, numerical derivatives, closed forms, invariants and an independent
library routine).  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_ref.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_LL = ctypes.POINTER(ctypes.c_longlong)


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE double)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
           "-shared", "-fPIC", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def open_library(path: str):
    """Load an oracle build from ``path`` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    i, d = ctypes.c_int, ctypes.c_double
    lib.ref_fwd.argtypes = [_D, _D, _D, _D, _D, i, i, i, i, i, d]
    lib.ref_fwd.restype = i
    lib.ref_bwd.argtypes = [_D, _D, _D, _D, _D, _D, _D, _D, i, i, i, i, i, d]
    lib.ref_bwd.restype = i
    lib.ref_fwd_rows.argtypes = [_D, _D, _D, i, i, i, d, _LL, i, _D, _D]
    lib.ref_fwd_rows.restype = i
    lib.ref_head_stats.argtypes = [_D, _D, _D, _D, i, i, i, d, i, _D, _D]
    lib.ref_head_stats.restype = i
    lib.ref_dq_rows.argtypes = [_D, _D, _D, _D, i, i, i, d, _LL, i, _D]
    lib.ref_dq_rows.restype = i
    lib.ref_dkdv_rows.argtypes = [_D, _D, _D, _D, _D, _D, i, i, i, d, _LL, i,
                                  _D, _D]
    lib.ref_dkdv_rows.restype = None
    lib.ref_fwd_decode.argtypes = [_D, _D, _D, _D, _D, i, i, i, i, i, d]
    lib.ref_fwd_decode.restype = i
    lib.ref_num_threads.argtypes = []
    lib.ref_num_threads.restype = i
    return lib


def _load():
    global _lib
    if _lib is None:
        if (not os.path.exists(_LIB_PATH)
                or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
            build()
        _lib = open_library(_LIB_PATH)
    return _lib


def _f64(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float64)
    return a


def _p(a: np.ndarray):
    return a.ctypes.data_as(_D)


def num_threads() -> int:
    return _load().ref_num_threads()


def ref_fwd(q, k, v, causal: bool, scale: float, lib=None):
    """O and LSE of softmax(scale * Q K^T [causal]) V for [B,H,N,d] inputs."""
    lib = lib or _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    if N:
        rc = lib.ref_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, d,
                         int(bool(causal)), float(scale))
        if rc:
            raise MemoryError("oracle forward: allocation failed")
    return o, lse


def ref_bwd(q, k, v, dO, causal: bool, scale: float, lib=None):
    """dQ, dK, dV and D = rowsum(P * dP) for upstream gradient dO."""
    lib = lib or _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    D = np.empty((B, H, N), dtype=np.float64)
    if N:
        rc = lib.ref_bwd(_p(q), _p(k), _p(v), _p(dO), _p(dq), _p(dk), _p(dv),
                         _p(D), B, H, N, d, int(bool(causal)), float(scale))
        if rc:
            raise MemoryError("oracle backward: allocation failed")
    return dq, dk, dv, D


def _rows(rows) -> np.ndarray:
    return np.ascontiguousarray(rows, dtype=np.int64)


def ref_fwd_rows(q, k, v, rows, causal: bool, scale: float, lib=None):
    """O and LSE for the query ``rows`` of one head; q,k,v are [N,d]."""
    lib = lib or _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    r = _rows(rows)
    o = np.empty((len(r), d), dtype=np.float64)
    lse = np.empty(len(r), dtype=np.float64)
    rc = lib.ref_fwd_rows(_p(q), _p(k), _p(v), N, d, int(bool(causal)),
                          float(scale), r.ctypes.data_as(_LL), len(r), _p(o),
                          _p(lse))
    if rc:
        raise MemoryError("oracle: allocation failed")
    return o, lse


def ref_head_stats(q, k, v, dO, causal: bool, scale: float, lib=None, first: int = 0):
    """LSE_i and D_i for the query rows i >= ``first`` of one head ([N,d]
    inputs); earlier rows are NaN.  Under the causal mask these are all the
    statistics that dK/dV rows j >= ``first`` depend on."""
    lib = lib or _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    N, d = q.shape
    if not 0 <= first <= N:
        raise ValueError("first must lie in [0, N]")
    lse = np.full(N, np.nan, dtype=np.float64)
    D = np.full(N, np.nan, dtype=np.float64)
    rc = lib.ref_head_stats(_p(q), _p(k), _p(v), _p(dO), N, d,
                            int(bool(causal)), float(scale), int(first), _p(lse), _p(D))
    if rc:
        raise MemoryError("oracle: allocation failed")
    return lse, D


def ref_dq_rows(q, k, v, dO, rows, causal: bool, scale: float, lib=None):
    """dQ for the query ``rows`` of one head."""
    lib = lib or _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    N, d = q.shape
    r = _rows(rows)
    dq = np.empty((len(r), d), dtype=np.float64)
    rc = lib.ref_dq_rows(_p(q), _p(k), _p(v), _p(dO), N, d, int(bool(causal)),
                         float(scale), r.ctypes.data_as(_LL), len(r), _p(dq))
    if rc:
        raise MemoryError("oracle: allocation failed")
    return dq


def ref_dkdv_rows(q, k, v, dO, lse, D, rows, causal: bool, scale: float,
                  lib=None):
    """dK and dV for the key ``rows`` of one head, given all rows' LSE and D."""
    lib = lib or _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    lse, D = _f64(lse), _f64(D)
    N, d = q.shape
    r = _rows(rows)
    dk = np.empty((len(r), d), dtype=np.float64)
    dv = np.empty((len(r), d), dtype=np.float64)
    lib.ref_dkdv_rows(_p(q), _p(k), _p(v), _p(dO), _p(lse), _p(D), N, d,
                      int(bool(causal)), float(scale), r.ctypes.data_as(_LL),
                      len(r), _p(dk), _p(dv))
    return dk, dv


def ref_fwd_decode(q, k, v, causal: bool, scale: float, lib=None):
    """O and LSE for Nq queries against Nk keys ([B,H,Nq,d] and [B,H,Nk,d]);
    causal: query i sees key j iff j <= i + Nk - Nq."""
    lib = lib or _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    o = np.empty_like(q)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    rc = lib.ref_fwd_decode(_p(q), _p(k), _p(v), _p(o), _p(lse), B * H, Nq, Nk, d,
                            int(bool(causal)), float(scale))
    if rc == -2:
        raise ValueError("causal decoding needs Nk >= Nq")
    if rc:
        raise MemoryError("oracle: allocation failed")
    return o, lse


# ---------------------------------------------------------------- ring steps
#
# Ring Attention with Blockwise Transformers (abstract): the sequence is
# spread over devices, each keeps its query block while key/value blocks
# travel, and every block's attention is folded into the running result.
# The two functions below are the per-step arithmetic of that scheme written
# out in plain numpy (fp64); they are used to check the ring's host logic.

def ref_lse_merge(o_a, lse_a, o_b, lse_b):
    """Attention over the union of two disjoint key sets from the results over
    each: with M = max(lse_a, lse_b) and w = exp(lse - M),
    O = (w_a O_a + w_b O_b) / (w_a + w_b) and LSE = M + log(w_a + w_b)
    (the rescaling of the online softmax, iplexlaw blog "Tiling preserves the
    attention calculation").  o_*: [..., d], lse_*: [...] (natural log)."""
    o_a, lse_a, o_b, lse_b = (np.asarray(x, dtype=np.float64) for x in (o_a, lse_a, o_b, lse_b))
    m = np.maximum(lse_a, lse_b)
    wa = np.exp(lse_a - m)
    wb = np.exp(lse_b - m)
    o = (wa[..., None] * o_a + wb[..., None] * o_b) / (wa + wb)[..., None]
    return o, m + np.log(wa + wb)


def ref_grads_given_stats(q, k, v, dO, lse, D, causal: bool, scale: float):
    """dQ, dK, dV of one (query block, key block) pair when the softmax
    normaliser and D come from the whole row: P = exp(scale q.k - lse) over
    this block's keys, dP = dO V^T, dS = P * (dP - D), dQ = scale dS K,
    dK = scale dS^T Q, dV = P^T dO.  causal: key j of the block visible to
    query i iff j <= i (the block on the diagonal).  Summed over the key
    blocks of a row these are the gradient over all its keys.
    q, dO: [B,H,Nq,d]; k, v: [B,H,Nk,d]; lse, D: [B,H,Nq]."""
    q, k, v, dO, lse, D = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO, lse, D))
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        nq, nk = s.shape[-2], s.shape[-1]
        hidden = np.arange(nk)[None, :] > np.arange(nq)[:, None]
        s = np.where(hidden, -np.inf, s)
    p = np.exp(s - lse[..., None])
    dp = np.einsum("bhid,bhjd->bhij", dO, v)
    ds = p * (dp - D[..., None])
    dq = scale * np.einsum("bhij,bhjd->bhid", ds, k)
    dk = scale * np.einsum("bhij,bhid->bhjd", ds, q)
    dv = np.einsum("bhij,bhid->bhjd", p, dO)
    return dq, dk, dv


# ---------------------------------------------------------------- score bias
#
# Attention with an additive bias matrix on the query-key scores (the
# "attention with bias" blurb of the pages): s_ij = scale q_i.k_j + b_ij, then
# the mask, the softmax and P V as before.  Plain numpy, fp64, materialised
# scores and a two-pass softmax.

def _biased_scores(q, k, bias, causal, scale):
    q, k, bias = (np.asarray(x, dtype=np.float64) for x in (q, k, bias))
    s = scale * np.einsum("bhid,bhjd->bhij", q, k) + bias
    if causal:
        n = s.shape[-1]
        s = np.where(np.arange(n)[None, :] > np.arange(n)[:, None], -np.inf, s)
    return s


def ref_fwd_bias(q, k, v, bias, causal: bool, scale: float):
    """O and LSE (natural log) of softmax(scale Q K^T + bias [+ causal]) V.
    bias: [Bb, Hb, N, N] with Bb in {1, B}, Hb in {1, H} (broadcast)."""
    s = _biased_scores(q, k, bias, causal, scale)
    m = np.max(s, axis=-1, keepdims=True)
    p = np.exp(s - m)
    den = np.sum(p, axis=-1, keepdims=True)
    o = np.einsum("bhij,bhjd->bhid", p / den, np.asarray(v, dtype=np.float64))
    return o, (m + np.log(den))[..., 0]


def ref_bwd_bias(q, k, v, bias, dO, causal: bool, scale: float, o_given=None):
    """dQ, dK, dV and dBias ([B,H,N,N], per batch and head) of
    L = sum(O * dO): P = softmax(s), dP = dO V^T, D = rowsum(dO * O),
    dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO,
    dBias = dS.  o_given: take D from this O (the forward output a backward
    pass receives) instead of the exact one."""
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    s = _biased_scores(q, k, bias, causal, scale)
    m = np.max(s, axis=-1, keepdims=True)
    p = np.exp(s - m)
    p = p / np.sum(p, axis=-1, keepdims=True)
    o = np.einsum("bhij,bhjd->bhid", p, v)
    if o_given is not None:
        o = np.asarray(o_given, dtype=np.float64)
    dp = np.einsum("bhid,bhjd->bhij", dO, v)
    D = np.sum(dO * o, axis=-1, keepdims=True)
    ds = p * (dp - D)
    dq = scale * np.einsum("bhij,bhjd->bhid", ds, k)
    dk = scale * np.einsum("bhij,bhid->bhjd", ds, q)
    dv = np.einsum("bhij,bhid->bhjd", p, dO)
    return dq, dk, dv, ds
