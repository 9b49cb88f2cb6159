"""The no-allocation fused call (sparse_attn_topk_noalloc) against the regular
fused call, through the C ABI.

Some callers cannot allocate device memory -- for example a serving engine that
has reserved all free device memory for its own pool, or a latency-critical
caller that must not pay for cudaFree's device-wide synchronisation.  For them
the library keeps its scratch in a static device array; this test checks that
two consecutive calls, which share that array, both reproduce the regular
call's mask exactly and its output within the parity tolerance.  The file is
named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from tests.parity import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


def _noalloc():
    L = bsa.lib()
    f = L.sparse_attn_topk_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, bsa.Shape, ctypes.c_float, ctypes.c_int, vp, vp, vp]
    return f


@pytest.mark.parametrize("B,H,N,d,topk", [
    (2, 3, 3001, 128, 0.5),
    (2, 3, 2500, 64, 0.3),
    # the scratch holds the score matrices of 4 of these 10 heads at a time, so
    # the selection runs in chunks of 4, 4 and 2 heads
    (1, 10, 75600, 64, 0.5),
])
def test_noalloc_matches_fused_call_twice(B, H, N, d, topk, cuda_device):
    f = _noalloc()
    wl = W.custom("na", B=B, H=H, d=d, N=N, seed=N + d)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ref_out, ref_mask = bsa.sparse_attn_topk(q, k, v, topk, return_mask=True)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        mask = torch.full_like(ref_mask, 7)
        st = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), bsa.Shape(*q.shape), topk, 0, out.data_ptr(),
               mask.data_ptr(), stream)
        assert st == 0, bsa.lib().bsa_last_error_message().decode()
        torch.cuda.synchronize()
        assert torch.equal(mask, ref_mask), f"call {call}: mask differs"
        err = (out.float() - ref_out.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, err.max().item())


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    f = _noalloc()
    # Distinct, never-dereferenced addresses 1 GiB apart (each tensor of this shape
    # is 774 MB): the call is rejected on the host before anything is launched.
    q, k, v, out = (g << 30 for g in (4, 5, 6, 7))
    st = f(q, k, v, bsa.Shape(1, 40, 75600, 128), 0.5, 0, out, None, None)
    assert st == 1
    assert "static scratch" in bsa.lib().bsa_last_error_message().decode()
