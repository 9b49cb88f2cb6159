"""The no-allocation fused call (sparse_attn_topk_noalloc) against the regular
fused call, through the C ABI.

Some callers cannot allocate device memory -- for example a serving engine that
has reserved all free device memory for its own pool, or a latency-critical
caller that must not pay for cudaFree's device-wide synchronisation.  For them
the library keeps its scratch in a static device array.  This file checks that
two consecutive calls, which share that array, both write exactly the bytes of
the regular call (mask and output: the same kernels run on the same lists), and
that a wait that runs out inside them is reported through the call's own status
reader.  The file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc():
    L = bsa.lib()
    f = L.sparse_attn_topk_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, bsa.Shape, ctypes.c_float, ctypes.c_int, vp, vp, vp]
    s = L.sparse_attn_topk_noalloc_status
    s.restype = ctypes.c_int
    s.argtypes = [vp]
    return f, s


@pytest.mark.parametrize("B,H,N,d,topk,causal", [
    (2, 3, 3001, 128, 0.5, 0),
    (2, 3, 2500, 64, 0.3, 0),
    (1, 4, 2900, 64, 0.4, 1),
    # the scratch holds the score matrices of 5 of these 10 heads at a time, so
    # the selection runs in two chunks of 5 heads
    (1, 10, 75600, 64, 0.5, 0),
])
def test_noalloc_matches_fused_call_twice(B, H, N, d, topk, causal, cuda_device):
    f, status = _noalloc()
    wl = W.custom("na", B=B, H=H, d=d, N=N, seed=N + d)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ref_out, ref_mask = bsa.sparse_attn_topk(q, k, v, topk, bool(causal), return_mask=True)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        mask = torch.full_like(ref_mask, 7)
        st = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), bsa.Shape(*q.shape), topk, causal, out.data_ptr(),
               mask.data_ptr(), stream)
        assert st == 0, bsa.lib().bsa_last_error_message().decode()
        assert status(stream) == 0, bsa.lib().bsa_last_error_message().decode()
        assert torch.equal(mask, ref_mask), f"call {call}: mask differs"
        assert torch.equal(out, ref_out), f"call {call}: output differs"


def test_noalloc_reports_a_wait_that_ran_out(cuda_device):
    f, status = _noalloc()
    wl = W.custom("na_to", B=1, H=4, d=128, N=6000, seed=5)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ref = bsa.sparse_attn_topk(q, k, v, 0.5)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream().cuda_stream
    shape = bsa.Shape(*q.shape)
    try:
        bsa.set_wait_timeout_ns(1000)
        assert f(q.data_ptr(), k.data_ptr(), v.data_ptr(), shape, 0.5, 0, out.data_ptr(), None, stream) == 0
        assert status(stream) == 4  # BSA_ERR_TIMEOUT
        assert b"bounded wait" in bsa.lib().bsa_last_error_message()
    finally:
        bsa.set_wait_timeout_ns(0)  # the default limit
    assert f(q.data_ptr(), k.data_ptr(), v.data_ptr(), shape, 0.5, 0, out.data_ptr(), None, stream) == 0
    assert status(stream) == 0
    assert torch.equal(out, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    f, _ = _noalloc()
    # Distinct, never-dereferenced addresses 1 GiB apart (each tensor of this shape
    # is 774 MB): the call is rejected on the host before anything is launched.
    q, k, v, out = (g << 30 for g in (4, 5, 6, 7))
    st = f(q, k, v, bsa.Shape(1, 40, 75600, 128), 0.5, 0, out, None, None)
    assert st == 1
    assert "static scratch" in bsa.lib().bsa_last_error_message().decode()
