"""Failure detection without a GPU fault: every wait inside the attention kernel
is bounded.  With the limit forced down to 1 microsecond the pipeline's first
waits (TMA loads, tensor-core results) run out, the kernel records the timeout
in the workspace status word and returns early, and the host reads
BSA_ERR_TIMEOUT.  The context stays usable: with the default limit restored the
next call succeeds and matches the reference result."""
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_forced_wait_timeout_is_reported_and_context_survives(cuda_device):
    wl = W.custom("to", B=1, H=4, d=128, N=6000, seed=5)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    ref = bsa.sparse_attn_topk(q, k, v, 0.5, workspace=ws)
    bsa.last_device_status(ws)
    out = torch.empty_like(q)
    try:
        bsa.set_wait_timeout_ns(1000)
        bsa.sparse_attn_topk(q, k, v, 0.5, out=out, workspace=ws)
        with pytest.raises(bsa.BsaError) as e:
            bsa.last_device_status(ws)
        assert e.value.status == 4  # BSA_ERR_TIMEOUT
        assert "bounded wait" in str(e.value)
    finally:
        bsa.set_wait_timeout_ns(0)  # the default limit
    again = bsa.sparse_attn_topk(q, k, v, 0.5, out=out, workspace=ws)
    bsa.last_device_status(ws)  # no error recorded this time
    torch.cuda.synchronize()
    assert torch.equal(again, ref)


def test_check_true_raises_the_recorded_timeout(cuda_device):
    """With check=True the call itself reads the status word after launching, so a
    wait that ran out surfaces as BsaError(BSA_ERR_TIMEOUT) without a separate
    last_device_status; the default limit then gives a clean, identical result."""
    wl = W.custom("to2", B=1, H=2, d=64, N=4000, seed=9)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    ref = bsa.sparse_attn_topk(q, k, v, 0.5, workspace=ws, check=True)
    out = torch.empty_like(q)
    try:
        bsa.set_wait_timeout_ns(1000)
        with pytest.raises(bsa.BsaError) as e:
            bsa.sparse_attn_topk(q, k, v, 0.5, out=out, workspace=ws, check=True)
        assert e.value.status == 4
    finally:
        bsa.set_wait_timeout_ns(0)
    bsa.sparse_attn_topk(q, k, v, 0.5, out=out, workspace=ws, check=True)
    assert torch.equal(out, ref)
