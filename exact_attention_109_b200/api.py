"""ctypes binding of libfa_sm100.so -- argument marshalling only.

Every function here converts torch tensors (or raw integers) into the pointers
and sizes of the C ABI in ``include/fa.h`` and calls the entry point of the same
name.  All arithmetic happens in the CUDA kernels behind that ABI; there is no
fallback path, and a missing library raises ``FaError`` on first use.
"""
from __future__ import annotations

import ctypes
import os

import torch

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfa_sm100.so"
_lib = None


class FaError(RuntimeError):
    """A C entry point returned a status other than FA_OK."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_strerror(status) if _lib else status}")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def library():
    """Load the CUDA library (raises when it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise FaError(FA_ERR_UNSUPPORTED,
                      f"{_LIB_NAME} not built (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_fwd.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f,
                           vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    lib.fa_bwd_preprocess.restype = i
    lib.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    lib.fa_bwd_main.restype = i
    lib.fa_bwd_dq_convert.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
    lib.fa_bwd_dq_convert.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f,
                                   vp]
    lib.fa_bwd_noalloc.restype = i
    ll = ctypes.c_longlong
    lib.fa_decode_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_fwd_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, ll, i, i, f, vp, sz, vp]
    lib.fa_fwd_decode.restype = i
    ip = ctypes.POINTER(i)
    lib.fa_decode_split_plan.argtypes = [i, i, i, i, i, i, i, ip, ip, ip]
    lib.fa_decode_split_plan.restype = i
    lib.fa_lse_merge.argtypes = [vp, vp, vp, vp, vp, ll, i, i, vp]
    lib.fa_lse_merge.restype = i
    lib.fa_bwd_main_accumulate.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz,
                                           vp]
    lib.fa_bwd_main_accumulate.restype = i
    lib.fa_convert_f32_bf16.argtypes = [vp, vp, ll, vp]
    lib.fa_convert_f32_bf16.restype = i
    lib.fa_fwd_qk8.argtypes = [vp, vp, vp, f, f, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_fwd_qk8.restype = i
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_fwd_fp8.restype = i
    lib.fa_fwd_bias.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp]
    lib.fa_fwd_bias.restype = i
    lib.fa_bwd_bias.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                f, vp, sz, vp]
    lib.fa_bwd_bias.restype = i
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    lib.fa_selftest_wait_timeout.restype = i
    lib.fa_get_device_error.argtypes = [vp]
    lib.fa_get_device_error.restype = i
    lib.fa_strerror.argtypes = [i]
    lib.fa_strerror.restype = ctypes.c_char_p
    _lib = lib
    return lib


def fa_strerror(status: int) -> str:
    return library().fa_strerror(int(status)).decode()


def _check(status: int, where: str):
    if status != FA_OK:
        raise FaError(status, where)


# ---------------------------------------------------------------- raw entry points

def fa_fwd(q: int, k: int, v: int, o: int, lse: int, B: int, H: int, N: int,
           d: int, causal: int, scale: float, stream: int = 0) -> int:
    """Raw C call with device pointers as integers; returns the status."""
    return library().fa_fwd(q, k, v, o, lse, B, H, N, d, int(causal),
                            float(scale), stream or None)


def fa_bwd(q: int, k: int, v: int, o: int, lse: int, dO: int, dq: int, dk: int,
           dv: int, B: int, H: int, N: int, d: int, causal: int, scale: float,
           workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    """Raw C call with device pointers as integers; returns the status."""
    return library().fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d,
                            int(causal), float(scale), workspace,
                            int(workspace_bytes), stream or None)


def fa_bwd_preprocess(o: int, lse: int, dO: int, B: int, H: int, N: int, d: int,
                      workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return library().fa_bwd_preprocess(o, lse, dO, B, H, N, d, workspace,
                                       int(workspace_bytes), stream or None)


def fa_bwd_main(q: int, k: int, v: int, dO: int, dk: int, dv: int, B: int, H: int,
                N: int, d: int, causal: int, scale: float, workspace: int,
                workspace_bytes: int, stream: int = 0) -> int:
    return library().fa_bwd_main(q, k, v, dO, dk, dv, B, H, N, d, int(causal),
                                 float(scale), workspace, int(workspace_bytes),
                                 stream or None)


def fa_bwd_dq_convert(dq: int, B: int, H: int, N: int, d: int, scale: float,
                      workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return library().fa_bwd_dq_convert(dq, B, H, N, d, float(scale), workspace,
                                       int(workspace_bytes), stream or None)


def fa_bwd_noalloc(q: int, k: int, v: int, o: int, lse: int, dO: int, dq: int,
                   dk: int, dv: int, B: int, H: int, N: int, d: int, causal: int,
                   scale: float, stream: int = 0) -> int:
    """Raw C call of the backward pass that uses the library's own fixed scratch
    array instead of a caller workspace (for callers that cannot allocate);
    returns the status."""
    return library().fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d,
                                    int(causal), float(scale), stream or None)


# Size of the scratch array fa_bwd_noalloc uses (FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES).
FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES = 64 << 20


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_bwd_workspace_size(B, H, N, d))


def fa_decode_workspace_size(B: int, H: int, Nq: int, Nk: int, d: int) -> int:
    return int(library().fa_decode_workspace_size(B, H, Nq, Nk, d))


def fa_fwd_decode(q: int, k: int, v: int, o: int, lse: int, B: int, H: int, Nq: int,
                  Nk: int, kv_rows: int, d: int, causal: int, scale: float,
                  workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    """Raw C call with device pointers as integers; returns the status."""
    return library().fa_fwd_decode(q, k, v, o, lse, B, H, Nq, Nk, int(kv_rows), d,
                                   int(causal), float(scale), workspace or None,
                                   int(workspace_bytes), stream or None)


def fa_decode_split_plan(B: int, H: int, Nq: int, Nk: int, d: int, sm_count: int,
                         ctas_per_sm: int):
    """(status, query rows per CTA, key splits, keys per split) of the host
    split plan; pure host arithmetic, needs no GPU."""
    qg, ns, ch = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = library().fa_decode_split_plan(B, H, Nq, Nk, d, sm_count, ctas_per_sm,
                                        ctypes.byref(qg), ctypes.byref(ns),
                                        ctypes.byref(ch))
    return st, qg.value, ns.value, ch.value


def fa_fwd_qk8(q: int, k: int, v: int, q_descale: float, k_descale: float, o: int, lse: int,
               B: int, H: int, N: int, d: int, causal: int, scale: float, stream: int = 0) -> int:
    """Raw C call: forward pass with e4m3 Q and K; returns the status."""
    return library().fa_fwd_qk8(q, k, v, float(q_descale), float(k_descale), o, lse, B, H, N,
                                d, int(causal), float(scale), stream or None)


def fa_fwd_fp8(q: int, k: int, v: int, q_descale: float, k_descale: float, v_descale: float,
               o: int, lse: int, B: int, H: int, N: int, d: int, causal: int, scale: float,
               stream: int = 0) -> int:
    """Raw C call with device pointers as integers; returns the status."""
    return library().fa_fwd_fp8(q, k, v, float(q_descale), float(k_descale), float(v_descale),
                                o, lse, B, H, N, d, int(causal), float(scale), stream or None)


def fa_fwd_bias(q: int, k: int, v: int, bias: int, o: int, lse: int, B: int, H: int, N: int,
                d: int, bias_batch: int, bias_heads: int, causal: int, scale: float,
                stream: int = 0) -> int:
    """Raw C call: forward pass with an additive score bias."""
    return library().fa_fwd_bias(q, k, v, bias, o, lse, B, H, N, d, int(bias_batch),
                                 int(bias_heads), int(causal), float(scale), stream or None)


def fa_bwd_bias(q: int, k: int, v: int, bias: int, o: int, lse: int, dO: int, dq: int, dk: int,
                dv: int, dbias: int, B: int, H: int, N: int, d: int, bias_batch: int,
                bias_heads: int, causal: int, scale: float, workspace: int,
                workspace_bytes: int, stream: int = 0) -> int:
    """Raw C call: backward pass with an additive score bias (dbias may be 0)."""
    return library().fa_bwd_bias(q, k, v, bias, o, lse, dO, dq, dk, dv, dbias or None, B, H, N,
                                 d, int(bias_batch), int(bias_heads), int(causal), float(scale),
                                 workspace, int(workspace_bytes), stream or None)


def fa_lse_merge(o_acc: int, lse_acc: int, o_part: int, lse_part: int, o_out: int,
                 rows: int, d: int, init: int, stream: int = 0) -> int:
    """Raw C call: fold a partial (O, LSE) into a running fp32 one."""
    return library().fa_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out or None, int(rows),
                                  d, int(init), stream or None)


def fa_bwd_main_accumulate(q: int, k: int, v: int, dO: int, dk_acc: int, dv_acc: int, B: int,
                           H: int, N: int, d: int, causal: int, scale: float, workspace: int,
                           workspace_bytes: int, stream: int = 0) -> int:
    """Raw C call: fa_bwd_main adding dK, dV into fp32 accumulators."""
    return library().fa_bwd_main_accumulate(q, k, v, dO, dk_acc, dv_acc, B, H, N, d,
                                            int(causal), float(scale), workspace,
                                            int(workspace_bytes), stream or None)


def fa_convert_f32_bf16(src: int, dst: int, n: int, stream: int = 0) -> int:
    return library().fa_convert_f32_bf16(src, dst, int(n), stream or None)


def fa_selftest_wait_timeout(limit_us: int, stream: int = 0) -> int:
    """Raw C call: enqueue the bounded-wait self-test (see include/fa.h)."""
    return library().fa_selftest_wait_timeout(int(limit_us), stream or None)


def fa_get_device_error(stream: int = 0) -> int:
    return library().fa_get_device_error(stream or None)


# ---------------------------------------------------------------- tensor wrappers

def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(q.shape)


def _require(ts, shape, dtype, device):
    for name, t in ts.items():
        if t.dtype != dtype:
            raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
        if t.device != device:
            raise ValueError(f"{name}: expected device {device}, got {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {shape}, got {tuple(t.shape)}")


def attention_forward(q, k, v, causal: int, scale: float, out=None, lse=None,
                      stream=None):
    """O, LSE = fa_fwd(q, k, v) for CUDA bf16 [B,H,N,d] tensors.  causal:
    0 / False none, 1 / True key j visible to query i iff j <= i, 2 iff
    j < i (row 0 then sees no key: O = 0, LSE = -inf)."""
    B, H, N, d = _shape(q)
    _require({"q": q, "k": k, "v": v}, (B, H, N, d), torch.bfloat16, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _require({"out": out}, (B, H, N, d), torch.bfloat16, q.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q.device)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                  int(causal), scale, s), "fa_fwd")
    return out, lse


def attention_backward(q, k, v, out, lse, dO, causal: int, scale: float,
                       dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV = fa_bwd(...) for CUDA bf16 [B,H,N,d] tensors (causal as
    for attention_forward)."""
    B, H, N, d = _shape(q)
    _require({"q": q, "k": k, "v": v, "out": out, "dO": dO}, (B, H, N, d),
             torch.bfloat16, q.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _require({"dq": dq, "dk": dk, "dv": dv}, (B, H, N, d), torch.bfloat16,
             q.device)
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dO),
                  _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, int(causal), scale,
                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                  s), "fa_bwd")
    return dq, dk, dv


def attention_decode(q, k, v, causal: bool, scale: float, n_keys: int | None = None,
                     out=None, lse=None, workspace=None, stream=None):
    """O, LSE = fa_fwd_decode(q, k, v): q [B,H,Nq,d] against the first n_keys
    rows (default: all) of the cache tensors k, v [B,H,kv_rows,d] (CUDA bf16).
    With causal, query i sees key j iff j <= i + n_keys - Nq."""
    B, H, Nq, d = _shape(q)
    kv_rows = k.shape[2] if k.dim() == 4 else -1
    Nk = kv_rows if n_keys is None else int(n_keys)
    _require({"q": q}, (B, H, Nq, d), torch.bfloat16, q.device)
    _require({"k": k, "v": v}, (B, H, kv_rows, d), torch.bfloat16, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _require({"out": out}, (B, H, Nq, d), torch.bfloat16, q.device)
    _require({"lse": lse}, (B, H, Nq), torch.float32, q.device)
    need = fa_decode_workspace_size(B, H, Nq, Nk, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(fa_fwd_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nq, Nk,
                         kv_rows, d, int(causal), scale, ws_ptr, ws_bytes, s),
           "fa_fwd_decode")
    return out, lse


def attention_forward_qk8(q8, k8, v, q_descale: float, k_descale: float, causal: bool,
                          scale: float, out=None, lse=None, stream=None):
    """O, LSE = fa_fwd_qk8: q8, k8 CUDA float8_e4m3fn [B,H,N,d] with their
    per-tensor dequantisation factors, v CUDA bf16 [B,H,N,d]."""
    B, H, N, d = _shape(q8)
    _require({"q8": q8, "k8": k8}, (B, H, N, d), torch.float8_e4m3fn, q8.device)
    _require({"v": v}, (B, H, N, d), torch.bfloat16, q8.device)
    if out is None:
        out = torch.empty(v.shape, dtype=torch.bfloat16, device=v.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=v.device)
    _require({"out": out}, (B, H, N, d), torch.bfloat16, q8.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q8.device)
    s = (stream or torch.cuda.current_stream(v.device)).cuda_stream
    _check(fa_fwd_qk8(_ptr(q8), _ptr(k8), _ptr(v), q_descale, k_descale, _ptr(out), _ptr(lse),
                      B, H, N, d, int(causal), scale, s), "fa_fwd_qk8")
    return out, lse


def attention_forward_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
                          causal: bool, scale: float, out=None, lse=None, stream=None):
    """O, LSE = fa_fwd_fp8: q8, k8, v8 CUDA float8_e4m3fn [B,H,N,d] with their
    per-tensor dequantisation factors; O is bf16."""
    B, H, N, d = _shape(q8)
    _require({"q8": q8, "k8": k8, "v8": v8}, (B, H, N, d), torch.float8_e4m3fn, q8.device)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    _require({"out": out}, (B, H, N, d), torch.bfloat16, q8.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q8.device)
    s = (stream or torch.cuda.current_stream(q8.device)).cuda_stream
    _check(fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), q_descale, k_descale, v_descale, _ptr(out),
                      _ptr(lse), B, H, N, d, int(causal), scale, s), "fa_fwd_fp8")
    return out, lse


def _bias_flags(bias, B, H, N):
    if bias.dim() != 4 or tuple(bias.shape[2:]) != (N, N) or bias.shape[0] not in (1, B) \
            or bias.shape[1] not in (1, H):
        raise ValueError(f"bias: expected [B or 1, H or 1, {N}, {N}], got {tuple(bias.shape)}")
    if bias.dtype != torch.bfloat16 or not bias.is_contiguous():
        raise TypeError("bias: expected a contiguous bf16 tensor")
    return int(bias.shape[0] == B and B > 1), int(bias.shape[1] == H and H > 1)


def attention_forward_bias(q, k, v, bias, causal: bool, scale: float, out=None, lse=None,
                           stream=None):
    """O, LSE = fa_fwd_bias: scores scale * q.k + bias for CUDA bf16 [B,H,N,d]
    q, k, v and a bf16 bias [B or 1, H or 1, N, N]."""
    B, H, N, d = _shape(q)
    _require({"q": q, "k": k, "v": v}, (B, H, N, d), torch.bfloat16, q.device)
    bb, bh_ = _bias_flags(bias, B, H, N)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _require({"out": out}, (B, H, N, d), torch.bfloat16, q.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q.device)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(fa_fwd_bias(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(out), _ptr(lse), B, H, N, d,
                       bb, bh_, int(causal), scale, s), "fa_fwd_bias")
    return out, lse


def attention_backward_bias(q, k, v, bias, out, lse, dO, causal: bool, scale: float,
                            want_dbias: bool = True, workspace=None, stream=None):
    """dQ, dK, dV, dBias (or None) = fa_bwd_bias(...); dBias is [B,H,N,N] bf16."""
    B, H, N, d = _shape(q)
    _require({"q": q, "k": k, "v": v, "out": out, "dO": dO}, (B, H, N, d), torch.bfloat16,
             q.device)
    _require({"lse": lse}, (B, H, N), torch.float32, q.device)
    bb, bh_ = _bias_flags(bias, B, H, N)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dbias = torch.empty((B, H, N, N), dtype=torch.bfloat16, device=q.device) if want_dbias \
        else None
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(fa_bwd_bias(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(out), _ptr(lse), _ptr(dO),
                       _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias) if dbias is not None else 0,
                       B, H, N, d, bb, bh_, int(causal), scale, _ptr(workspace),
                       workspace.numel() * workspace.element_size(), s), "fa_bwd_bias")
    return dq, dk, dv, dbias
