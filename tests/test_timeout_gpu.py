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


def test_every_workspace_call_clears_the_status_word(cuda_device):
    """The status word describes the latest call on the workspace: each call that
    takes one clears the word before its kernels, the selection-only calls
    included (their kernels never set it).  A word left nonzero by earlier use of
    the memory must not be reported."""
    wl = W.custom("st", B=1, H=2, d=64, N=3000, seed=8)
    q, k, v = (t.cuda() for t in W.make_qkv(wl))
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    bsa.last_device_status(ws)  # a fresh workspace starts cleared
    mask = torch.ones(wl.B, wl.H, wl.Qb, wl.Kb, dtype=torch.uint8, device="cuda")
    calls = {
        "sparse_attn_select": lambda: bsa.sparse_attn_select(q, k, 0.5, workspace=ws),
        "sparse_attn_select_cdf": lambda: bsa.sparse_attn_select_cdf(q, k, 0.9, workspace=ws),
        "sparse_attn_block_scores": lambda: bsa.sparse_attn_block_scores(q, k, workspace=ws),
        "block_sparse_attn_plan": lambda: bsa.block_sparse_attn_plan(q, mask, workspace=ws),
        "block_sparse_attn_apply": lambda: bsa.block_sparse_attn_apply(q, k, v, ws),
        "block_sparse_attn_fwd": lambda: bsa.block_sparse_attn_fwd(q, k, v, mask, workspace=ws),
        "sparse_attn_topk": lambda: bsa.sparse_attn_topk(q, k, v, 0.5, workspace=ws),
        "sparse_attn_cdf": lambda: bsa.sparse_attn_cdf(q, k, v, 0.9, workspace=ws),
    }
    for name, call in calls.items():
        ws[:256].fill_(0xC0)  # a stale nonzero word, as reused memory may hold
        call()
        try:
            bsa.last_device_status(ws)
        except bsa.BsaError as e:
            raise AssertionError(f"{name} left the stale status word in place: {e}") from None
