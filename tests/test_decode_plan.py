"""Host logic of split-KV decoding, without a GPU: the workspace size, the
work split fa_fwd_decode would launch, and argument rejection before any
device work."""
import itertools
import math

import pytest

import exact_attention_109_b200 as fa
from exact_attention_109_b200 import build as fa_build

FAKE = 1 << 20  # aligned, never dereferenced: every case fails validation first


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.library()


def test_workspace_size(lib):
    # one fp32 partial row (d values + its log-sum-exp) per query row and split;
    # at most ceil(Nk / 256) splits, and none (size 0) when Nk <= 256
    assert fa.fa_decode_workspace_size(2, 3, 1, 256, 128) == 0
    assert fa.fa_decode_workspace_size(2, 3, 1, 257, 128) == 2 * 3 * 1 * 2 * 129 * 4
    assert fa.fa_decode_workspace_size(1, 16, 4, 65536, 64) == 16 * 4 * 256 * 65 * 4
    assert fa.fa_decode_workspace_size(1, 1, 1, 1000, 96) == 0
    assert fa.fa_decode_workspace_size(1, 1, 0, 1000, 64) == 0


PLAN_CASES = list(itertools.product((1, 3, 16, 256), (1, 2, 3, 4, 5, 16),
                                    (1, 100, 256, 257, 4096, 8192, 65536, 1 << 20),
                                    (64, 128), ((148, 2), (148, 3), (132, 1))))


@pytest.mark.parametrize("BH,Nq,Nk,d,slots", PLAN_CASES)
def test_split_plan_invariants(lib, BH, Nq, Nk, d, slots):
    st, qg, ns, chunk = fa.fa_decode_split_plan(1, BH, Nq, Nk, d, *slots)
    assert st == fa.FA_OK
    assert qg == (1 if Nq == 1 else 2 if Nq == 2 else 4)
    assert chunk % 64 == 0 and chunk >= 64
    # the splits tile [0, Nk) exactly, none of them empty
    assert ns * chunk >= Nk and (ns - 1) * chunk < Nk
    if ns > 1:
        assert chunk >= 256 and ns <= math.ceil(Nk / 256)
        # the workspace covers the partials of every split
        need = BH * Nq * ns * (d + 1) * 4
        assert fa.fa_decode_workspace_size(1, BH, Nq, Nk, d) >= need


def test_split_plan_fills_the_gpu(lib):
    # few heads, long cache: the keys are split so that every SM streams
    st, qg, ns, chunk = fa.fa_decode_split_plan(1, 16, 1, 65536, 128, 148, 2)
    assert st == fa.FA_OK and 16 * ns >= 148
    # many heads: no split needed beyond what balances the waves
    st, qg, ns, chunk = fa.fa_decode_split_plan(64, 32, 1, 4096, 128, 148, 2)
    assert st == fa.FA_OK and ns <= 2


@pytest.mark.parametrize("kwargs,status", [
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(lse=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=0), fa.FA_ERR_INVALID_ARG),
    (dict(kv_rows=999), fa.FA_ERR_INVALID_ARG),
    (dict(causal=1, Nq=1001), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(workspace=0), fa.FA_ERR_INVALID_ARG),
    (dict(workspace_bytes=16), fa.FA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), fa.FA_ERR_MISALIGNED),
    (dict(workspace=FAKE + 16), fa.FA_ERR_MISALIGNED),
])
def test_decode_rejects_bad_arguments(lib, kwargs, status):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=2, Nq=1, Nk=1000,
                kv_rows=1000, d=128, causal=0, scale=0.1, workspace=FAKE,
                workspace_bytes=1 << 20)
    args.update(kwargs)
    assert fa.fa_fwd_decode(*args.values()) == status


def test_plan_rejects_bad_arguments(lib):
    assert fa.fa_decode_split_plan(1, 1, 1, 100, 128, 0, 2)[0] == fa.FA_ERR_INVALID_ARG
    assert fa.fa_decode_split_plan(1, 1, 1, 100, 96, 148, 2)[0] == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_decode_split_plan(1, 1, 0, 100, 64, 148, 2)[0] == fa.FA_ERR_INVALID_ARG
