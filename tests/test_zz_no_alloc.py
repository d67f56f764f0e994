"""The allocation-free activation quantiser (qvae_act_absmax_quant_noalloc).

It serves callers that cannot allocate device memory (a host runtime that owns
every buffer and passes a layer only its inputs and outputs).  Its scratch is a
fixed array inside the library, shared by every call, so the test makes two
calls in a row -- a large tensor, then a smaller one that launches fewer CTAs --
and checks both against the workspace entry point through the C ABI.  The file
name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from video_vae_decode_b200 import qvae
    qvae.lib()
    return qvae


def run_both(q, x):
    xq_ws, s_ws = q.act_absmax_quant(x)                       # caller workspace
    xq_na = torch.empty_like(xq_ws)
    s_na = torch.empty_like(s_ws)
    q.qvae_act_absmax_quant_noalloc(x, xq_na, s_na)           # fixed library scratch
    torch.cuda.synchronize()
    assert q.qvae_get_error() == 0
    assert s_na.cpu().numpy().view(np.uint32)[0] == s_ws.cpu().numpy().view(np.uint32)[0]
    assert torch.equal(xq_na, xq_ws)
    return s_na.item()


def test_noalloc_matches_workspace_entry_point_twice(q):
    g = torch.Generator().manual_seed(123)
    big = (torch.randn(6_291_456, generator=g) * 2).to(torch.bfloat16).cuda()
    big[12345] = 40.0                                          # far above any N(0, 4) sample
    small = (torch.randn(70_001, generator=g) * 0.5).to(torch.bfloat16).cuda()
    s1 = run_both(q, big)
    s2 = run_both(q, small)                                    # fewer CTAs: stale slots unused
    assert s1 == np.float32(40.0) / np.float32(127.0)
    assert s2 < s1


def test_noalloc_empty_and_bad_arguments(q):
    x = torch.zeros(0, dtype=torch.bfloat16, device="cuda")
    xq = torch.zeros(0, dtype=torch.int8, device="cuda")
    s = torch.full((1,), 7.0, device="cuda")
    q.qvae_act_absmax_quant_noalloc(x, xq, s)
    torch.cuda.synchronize()
    assert s.item() == 0.0
    L = q.lib()
    x16 = torch.zeros(32, dtype=torch.bfloat16, device="cuda")
    xq16 = torch.zeros(32, dtype=torch.int8, device="cuda")
    p = lambda t, off=0: None if t is None else t.data_ptr() + off
    assert L.qvae_act_absmax_quant_noalloc(p(x16), 16, p(xq16), None, None) == q.QVAE_ERR_ARG
    assert L.qvae_act_absmax_quant_noalloc(p(x16), -1, p(xq16), p(s), None) == q.QVAE_ERR_ARG
    assert L.qvae_act_absmax_quant_noalloc(p(x16, 2), 16, p(xq16), p(s), None) == q.QVAE_ERR_ALIGN
