"""The device calls are asynchronous on the caller's stream and neither allocate
nor synchronise, so a caller can capture them once in a CUDA graph and replay
them: the replay runs selection and attention again on whatever the captured
buffers hold and writes exactly the bytes the eager call writes."""
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _qkv(d, seed, H=3, N=2900):
    return [t.cuda() for t in W.make_qkv(W.custom("graph", B=1, H=H, d=d, N=N, seed=seed))]


@pytest.mark.parametrize("d,causal", [(128, False), (64, True)])
def test_fused_call_replays_from_a_cuda_graph(cuda_device, d, causal):
    q, k, v = _qkv(d, seed=5)
    B, H, N, _ = q.shape
    ws = bsa.make_workspace(B, H, N, d)
    out = torch.empty_like(q)
    ref = bsa.sparse_attn_topk(q, k, v, 0.4, causal).clone()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        bsa.sparse_attn_topk(q, k, v, 0.4, causal, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bsa.sparse_attn_topk(q, k, v, 0.4, causal, out=out, workspace=ws)

    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    bsa.last_device_status(ws)
    assert torch.equal(out, ref)

    # New inputs in the captured buffers: the replay selects and attends afresh.
    q2, k2, v2 = _qkv(d, seed=6)
    ref2 = bsa.sparse_attn_topk(q2, k2, v2, 0.4, causal)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    bsa.last_device_status(ws)
    assert torch.equal(out, ref2)


def test_plan_and_apply_replay_from_a_cuda_graph(cuda_device):
    """Plan reuse under a graph: the caller mask is compacted once outside, and the
    graph holds only the attention over that plan."""
    q, k, v = _qkv(128, seed=9, H=2, N=1500)
    B, H, N, d = q.shape
    Qb, Kb = bsa.block_counts(N)
    mask = (torch.rand(B, H, Qb, Kb, generator=torch.Generator().manual_seed(3)) < 0.4).to(torch.uint8).cuda()
    ws = bsa.make_workspace(B, H, N, d)
    bsa.block_sparse_attn_plan(q, mask, workspace=ws)
    ref = bsa.block_sparse_attn_fwd(q, k, v, mask_id=mask)
    out = torch.empty_like(q)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        bsa.block_sparse_attn_apply(q, k, v, ws, out=out)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bsa.block_sparse_attn_apply(q, k, v, ws, out=out)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    bsa.last_device_status(ws)
    assert torch.equal(out, ref)
