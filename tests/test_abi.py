"""The C ABI without a GPU: the library loads, exports every function that
include/fa.h declares, reports workspace sizes, and rejects bad arguments
before touching the device.  (No compute call is made here.)"""
import ctypes
import os
import re

import pytest

import exact_attention_109_b200 as fa
from exact_attention_109_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.library()


def declared_functions():
    names = []
    for header in os.listdir(os.path.join(ROOT, "include")):
        if not header.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", header)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(",
                            text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_get_device_error",
            "fa_strerror"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_strerror(lib):
    for code in range(6):
        assert fa.fa_strerror(code).startswith("FA_")
    assert "unknown" in fa.fa_strerror(99)


def test_workspace_size_is_linear_in_n(lib):
    # FlashAttention-2 abstract: memory linear, not quadratic, in N.
    for d in (64, 128):
        s1 = fa.fa_bwd_workspace_size(2, 3, 1024, d)
        s2 = fa.fa_bwd_workspace_size(2, 3, 2048, d)
        assert s1 == 2 * 3 * 1024 * (d + 2) * 4
        assert s2 == 2 * s1
    # padding to a multiple of 128 rows
    assert fa.fa_bwd_workspace_size(1, 1, 1, 64) == 128 * 66 * 4
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 1, 128, 96) == 0


FAKE = 1 << 20  # aligned, never dereferenced: every case fails validation first


@pytest.mark.parametrize("kwargs,status", [
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(lse=0), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(causal=3), fa.FA_ERR_INVALID_ARG),
    (dict(causal=-1), fa.FA_ERR_INVALID_ARG),
    (dict(k=FAKE + 2), fa.FA_ERR_MISALIGNED),
    (dict(o=FAKE + 8), fa.FA_ERR_MISALIGNED),
])
def test_fwd_rejects_bad_arguments(lib, kwargs, status):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, N=128, d=64,
                causal=0, scale=0.125)
    args.update(kwargs)
    assert fa.fa_fwd(**args) == status


@pytest.mark.parametrize("kwargs,status", [
    (dict(dO=0), fa.FA_ERR_INVALID_ARG),
    (dict(workspace=0), fa.FA_ERR_INVALID_ARG),
    (dict(workspace_bytes=16), fa.FA_ERR_INVALID_ARG),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(dq=FAKE + 4), fa.FA_ERR_MISALIGNED),
    (dict(workspace=FAKE + 16), fa.FA_ERR_MISALIGNED),
    (dict(causal=3), fa.FA_ERR_INVALID_ARG),
])
def test_bwd_rejects_bad_arguments(lib, kwargs, status):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dO=FAKE, dq=FAKE,
                dk=FAKE, dv=FAKE, B=1, H=1, N=128, d=64, causal=1, scale=0.125,
                workspace=FAKE, workspace_bytes=1 << 20)
    args.update(kwargs)
    assert fa.fa_bwd(**args) == status


def test_valid_call_without_device_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    st = fa.fa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, 0.125)
    assert st in (fa.FA_ERR_CUDA, fa.FA_ERR_UNSUPPORTED)


def test_tensor_wrapper_validates_before_calling(lib):
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        fa.attention_forward(q, q, q, False, 0.125)
    with pytest.raises(ValueError):
        fa.attention_forward(q[0], q[0], q[0], False, 0.125)


@pytest.mark.parametrize("fn,kwargs,status", [
    ("pre", dict(o=0), fa.FA_ERR_INVALID_ARG),
    ("pre", dict(workspace_bytes=8), fa.FA_ERR_INVALID_ARG),
    ("pre", dict(dO=FAKE + 2), fa.FA_ERR_MISALIGNED),
    ("main", dict(dk=0), fa.FA_ERR_INVALID_ARG),
    ("main", dict(causal=-1), fa.FA_ERR_INVALID_ARG),
    ("main", dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
    ("main", dict(d=80), fa.FA_ERR_UNSUPPORTED),
    ("main", dict(workspace=FAKE + 64), fa.FA_ERR_MISALIGNED),
    ("conv", dict(dq=0), fa.FA_ERR_INVALID_ARG),
    ("conv", dict(N=-5), fa.FA_ERR_INVALID_ARG),
])
def test_bwd_stages_reject_bad_arguments(lib, fn, kwargs, status):
    base = dict(B=1, H=1, N=128, d=64, workspace=FAKE, workspace_bytes=1 << 20)
    if fn == "pre":
        a = dict(o=FAKE, lse=FAKE, dO=FAKE, **base)
        a.update(kwargs)
        assert fa.fa_bwd_preprocess(**a) == status
    elif fn == "main":
        a = dict(q=FAKE, k=FAKE, v=FAKE, dO=FAKE, dk=FAKE, dv=FAKE, causal=0,
                 scale=0.1, **base)
        a.update(kwargs)
        assert fa.fa_bwd_main(**a) == status
    else:
        a = dict(dq=FAKE, scale=0.1, **base)
        a.update(kwargs)
        assert fa.fa_bwd_dq_convert(**a) == status
