"""No kernel writes outside its outputs: every output tensor is carved out of a
larger buffer whose margins hold a canary bit pattern, and after the call the
margins must be untouched -- for ragged lengths (rows past N in a tile), both
masks, both head dims, and every entry point that writes tensors (forward,
backward, decoding with split keys, bias and its gradient, the e4m3 path)."""
import pytest
import torch

import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import attention_inputs, decode_inputs, default_scale, to_e4m3

pytestmark = pytest.mark.gpu

PAD = 4096          # elements of canary before and after each output
CANARY16 = 0x7FC1   # a NaN payload no kernel produces
CANARY32 = 0x7FC12345


def _guarded(shape, dtype):
    n = 1
    for s in shape:
        n *= s
    if dtype == torch.float32:
        buf = torch.full((n + 2 * PAD,), CANARY32, dtype=torch.int32, device="cuda")
        view = buf.view(torch.float32)
    else:
        buf = torch.full((n + 2 * PAD,), CANARY16, dtype=torch.int16, device="cuda")
        view = buf.view(torch.bfloat16)
    return buf, view[PAD:PAD + n].view(shape)


def _intact(buf):
    c = CANARY32 if buf.dtype == torch.int32 else CANARY16
    return bool((buf[:PAD] == c).all()) and bool((buf[-PAD:] == c).all())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 129, 300])
def test_forward_backward_stay_inside(N, causal, d):
    B, H = 2, 3
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=N, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    bo, o = _guarded((B, H, N, d), torch.bfloat16)
    bl, lse = _guarded((B, H, N), torch.float32)
    fa.attention_forward(q, k, v, causal, scale, out=o, lse=lse)
    bq, dq = _guarded((B, H, N, d), torch.bfloat16)
    bk, dk = _guarded((B, H, N, d), torch.bfloat16)
    bv, dv = _guarded((B, H, N, d), torch.bfloat16)
    fa.attention_backward(q, k, v, o, lse, dO, causal, scale, dq=dq, dk=dk, dv=dv)
    assert fa.fa_get_device_error() == fa.FA_OK
    for b in (bo, bl, bq, bk, bv):
        assert _intact(b)
    assert torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()


@pytest.mark.parametrize("Nq,Nk", [(1, 777), (3, 5000), (5, 300)])
def test_decode_stays_inside(Nq, Nk):
    B, H, d = 2, 3, 128
    host = decode_inputs(B, H, Nq, Nk, d, seed=Nk)
    q, k, v = (host[x].cuda() for x in ("q", "k", "v"))
    bo, o = _guarded((B, H, Nq, d), torch.bfloat16)
    bl, lse = _guarded((B, H, Nq), torch.float32)
    need = fa.fa_decode_workspace_size(B, H, Nq, Nk, d)
    bw, ws = _guarded((max(need // 4, 1),), torch.float32)
    fa.attention_decode(q, k, v, True, default_scale(d), out=o, lse=lse,
                        workspace=ws.view(torch.uint8) if need else None)
    assert fa.fa_get_device_error() == fa.FA_OK
    for b in (bo, bl, bw):
        assert _intact(b)


def test_bias_and_e4m3_stay_inside():
    B, H, N, d = 1, 2, 136, 128
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, seed=5, with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    bias = (torch.randn(1, H, N, N) * 2).to(torch.bfloat16).cuda()
    o, lse = fa.attention_forward_bias(q, k, v, bias, True, scale)
    nbytes = fa.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    bdb, dbias = _guarded((B, H, N, N), torch.bfloat16)
    bq, dq = _guarded((B, H, N, d), torch.bfloat16)
    dk, dv = torch.empty_like(q), torch.empty_like(q)
    st = fa.fa_bwd_bias(q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(), o.data_ptr(),
                        lse.data_ptr(), dO.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                        dv.data_ptr(), dbias.data_ptr(), B, H, N, d, 0, 1, 1, scale,
                        ws.data_ptr(), nbytes, torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK
    q8, qs = to_e4m3(host["q"])
    k8, ks = to_e4m3(host["k"])
    bo, o8 = _guarded((B, H, N, d), torch.bfloat16)
    bl, l8 = _guarded((B, H, N), torch.float32)
    fa.attention_forward_qk8(q8.cuda(), k8.cuda(), v, qs, ks, True, scale, out=o8, lse=l8)
    assert fa.fa_get_device_error() == fa.FA_OK
    for b in (bdb, bq, bo, bl):
        assert _intact(b)
