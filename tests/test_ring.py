"""Sequence-sharded (ring) attention on the GPU: the log-sum-exp merge kernel,
the fp32-accumulating backward and the conversion kernel against the oracle,
and the whole ring scheme -- G virtual ranks on this GPU, every pair computed
by the CUDA kernels -- against the oracle's attention over the whole
sequence, within the tolerances of the other parity tests."""
import numpy as np
import pytest
import torch

import oracle
import exact_attention_109_b200 as fa
from exact_attention_109_b200 import ring
from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64
from parity_util import Check, max_abs, max_excess

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("d", [64, 128])
def test_lse_merge_kernel(d):
    g = torch.Generator().manual_seed(3)
    rows = 1000
    o_a = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    o_b = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    l_a = torch.randn(rows, generator=g) * 4
    l_b = torch.randn(rows, generator=g) * 4
    acc = torch.empty(rows, d, device="cuda")
    lacc = torch.empty(rows, device="cuda")
    out = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    oa, ob, la, lb = o_a.cuda(), o_b.cuda(), l_a.cuda(), l_b.cuda()
    assert fa.fa_lse_merge(acc.data_ptr(), lacc.data_ptr(), oa.data_ptr(), la.data_ptr(), 0,
                           rows, d, 1, _stream()) == fa.FA_OK
    assert torch.equal(acc.cpu(), o_a.float()) and torch.equal(lacc.cpu(), l_a)
    assert fa.fa_lse_merge(acc.data_ptr(), lacc.data_ptr(), ob.data_ptr(), lb.data_ptr(),
                           out.data_ptr(), rows, d, 0, _stream()) == fa.FA_OK
    torch.cuda.synchronize()
    ro, rl = oracle.ref_lse_merge(to_f64(o_a), to_f64(l_a), to_f64(o_b), to_f64(l_b))
    assert max_abs(acc.cpu().double().numpy(), ro) <= 1e-5
    assert max_abs(lacc.cpu().double().numpy(), rl) <= 1e-5
    assert max_excess(to_f64(out.cpu()), ro) <= 1e-5


def test_convert_kernel_rounds_like_torch():
    x = torch.randn(4096 * 8, device="cuda") * 100
    y = torch.empty(x.shape, dtype=torch.bfloat16, device="cuda")
    assert fa.fa_convert_f32_bf16(x.data_ptr(), y.data_ptr(), x.numel(), _stream()) == fa.FA_OK
    assert torch.equal(y, x.to(torch.bfloat16))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_accumulates_into_fp32(causal, d):
    """fa_bwd_main_accumulate adds exactly what fa_bwd_main would write."""
    B, H, N = 1, 3, 700
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=5, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal, scale)
    _, dk_ref, dv_ref = fa.attention_backward(q, k, v, o, lse, dO, causal, scale)
    nbytes = fa.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    base_k = torch.randn(B, H, N, d, device="cuda")
    base_v = torch.randn(B, H, N, d, device="cuda")
    dk_acc, dv_acc = base_k.clone(), base_v.clone()
    assert fa.fa_bwd_preprocess(o.data_ptr(), lse.data_ptr(), dO.data_ptr(), B, H, N, d,
                                ws.data_ptr(), nbytes, _stream()) == fa.FA_OK
    assert fa.fa_bwd_main_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), dO.data_ptr(),
                                     dk_acc.data_ptr(), dv_acc.data_ptr(), B, H, N, d,
                                     int(causal), scale, ws.data_ptr(), nbytes,
                                     _stream()) == fa.FA_OK
    assert fa.fa_get_device_error() == fa.FA_OK
    for got, base, ref in ((dk_acc, base_k, dk_ref), (dv_acc, base_v, dv_ref)):
        added = (got - base).cpu().double().numpy()
        # the bf16 path rounds once; the fp32 sum carries no such rounding
        assert max_excess(to_f64(ref.cpu()), added) <= 1e-3


def _check_whole(host, got, causal, scale):
    args = [to_f64(host[x]) for x in ("q", "k", "v")]
    o_ref, lse_ref = oracle.ref_fwd(*args, causal, scale)
    dq_ref, dk_ref, dv_ref, _ = oracle.ref_bwd(*args, to_f64(host["dO"]), causal, scale)
    o, lse, dq, dk, dv = got
    c = Check()
    c.o(to_f64(o.cpu()), o_ref)
    c.lse(lse.cpu().double().numpy(), lse_ref)
    for name, g, r in (("dq", dq, dq_ref), ("dk", dk, dk_ref), ("dv", dv, dv_ref)):
        c.grad(name, to_f64(g.cpu()), r)
    return c.done()


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world,N", [(1, 384), (2, 512), (3, 600), (4, 1024), (8, 1024)])
def test_local_ring_matches_whole_sequence(world, N, causal, d, layout):
    scale = default_scale(d)
    host = attention_inputs(1, 2, N, d, seed=world * 100 + N + d, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    got = ring.local_ring_attention(q, k, v, dO, causal, scale, world, layout=layout)
    assert fa.fa_get_device_error() == fa.FA_OK
    _check_whole(host, got, causal, scale)


@pytest.mark.parametrize("layout", ring.LAYOUTS)
def test_local_ring_long_sequence(layout):
    """4 virtual ranks of 2048 tokens (N = 8192), whole tensors checked."""
    d, causal = 128, True
    scale = default_scale(d)
    host = attention_inputs(1, 2, 8192, d, seed=9, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    got = ring.local_ring_attention(q, k, v, dO, causal, scale, 4, layout=layout)
    assert fa.fa_get_device_error() == fa.FA_OK
    _check_whole(host, got, causal, scale)
