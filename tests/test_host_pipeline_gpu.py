"""sparse_attn_topk_host: the head-chunk pipelined call on pinned host buffers gives
exactly the bytes of sparse_attn_topk on device buffers (heads are independent,
so chunking changes nothing), for several chunkings, ragged shapes, d = 64 and
causal; pageable host memory is rejected."""
import ctypes

import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W


def _case(B, H, N, d, seed):
    wl = W.custom("host", B=B, H=H, d=d, N=N, seed=seed)
    return W.make_qkv(wl)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,topk,causal,chunks", [
    (1, 5, 3000, 128, 0.5, False, 0),
    (1, 5, 3000, 128, 0.5, False, 3),
    (1, 5, 3000, 128, 0.3, False, 64),
    (2, 3, 1111, 64, 0.5, True, 4),
    (1, 1, 65, 128, 1.0, False, 2),
])
def test_host_pipeline_matches_device_call(cuda_device, B, H, N, d, topk, causal, chunks):
    q, k, v = _case(B, H, N, d, seed=N + d + H)
    ref = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, causal)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    out = bsa.sparse_attn_topk_host(qp, kp, vp, topk, causal, chunks=chunks)
    assert out.is_pinned()
    assert torch.equal(out, ref.cpu())
    # a second call reusing the device buffers and workspace
    bufs = tuple(torch.empty_like(ref) for _ in range(4))
    ws = bsa.make_workspace(B, H, N, d)
    out2 = bsa.sparse_attn_topk_host(qp, kp, vp, topk, causal, device_buffers=bufs, workspace=ws,
                                     chunks=chunks)
    bsa.last_device_status(ws)
    assert torch.equal(out2, ref.cpu())


@pytest.mark.gpu
def test_host_pipeline_rejects_pageable_memory(cuda_device):
    q, k, v = _case(1, 2, 512, 64, seed=3)
    dev = [torch.empty_like(q, device="cuda") for _ in range(4)]
    out = torch.empty_like(q)  # pageable
    s = bsa.Shape(*q.shape)
    ws = bsa.make_workspace(*q.shape)
    L = bsa.lib()
    st = L.sparse_attn_topk_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), s, 0.5, 0, out.data_ptr(),
                                 *[t.data_ptr() for t in dev], ws.data_ptr(), ws.numel(), 0, None)
    assert st == 1
    assert b"page-locked" in L.bsa_last_error_message()


@pytest.mark.gpu
@pytest.mark.parametrize("causal,chunks", [(False, 0), (True, 3)])
def test_host_pipeline_leaves_every_heads_lists_in_the_workspace(cuda_device, causal, chunks):
    """Each chunk's selection writes its own heads of the full workspace layout, so
    after the call the kept-block lists of all heads are there, equal to those
    sparse_attn_topk leaves."""
    import numpy as np

    from tests.parity import workspace_lists

    B, H, N, d = 1, 7, 2900, 128
    q, k, v = _case(B, H, N, d, seed=77)
    ws_dev, ws_host = bsa.make_workspace(B, H, N, d), bsa.make_workspace(B, H, N, d)
    ref = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), 0.3, causal, workspace=ws_dev)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    bufs = tuple(torch.empty_like(ref) for _ in range(4))
    out = bsa.sparse_attn_topk_host(qp, kp, vp, 0.3, causal, device_buffers=bufs, workspace=ws_host,
                                    chunks=chunks)
    bsa.last_device_status(ws_host)
    assert torch.equal(out, ref.cpu())
    Qb, Kb = (N + 127) // 128, (N + 63) // 64
    idx_d, cnt_d = workspace_lists(ws_dev, B * H, Qb, Kb, d)
    idx_h, cnt_h = workspace_lists(ws_host, B * H, Qb, Kb, d)
    assert np.array_equal(cnt_h, cnt_d)
    valid = np.arange(Kb)[None, :] < cnt_d[:, None]
    assert np.array_equal(np.where(valid, idx_h, -1), np.where(valid, idx_d, -1))
