"""Parity at the largest sequence the library accepts (N = 131072, Kb = 2048 key
blocks, the top of the int16 index range and of the row kernels' shared-memory
sizing) and one below it (a ragged last block): selection in full against the
fp64 oracle, attention on sampled query blocks (the first, second, middle and
last, plus seeded random ones)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests.parity import assert_close, compare_cdf_masks, compare_masks, sampled_blocks

pytestmark = pytest.mark.gpu


def _rows(out, q, k, v, mask_ref, agree, blocks, N, causal=False):
    got, ref = [], []
    o = out.cpu()
    qh, kh, vh = O.to_f64(q[0, 0]), O.to_f64(k[0, 0]), O.to_f64(v[0, 0])
    for i in blocks:
        if not agree[0, 0, i]:
            continue
        lo, hi = 128 * i, min(N, 128 * i + 128)
        ref.append(O.attention_rows(qh, kh, vh, mask_ref[0, 0, i], i, causal=causal))
        got.append(o[0, 0, lo:hi].float().numpy())
    assert got, "no sampled block to compare"
    return np.concatenate(got), np.concatenate(ref)


@pytest.mark.parametrize("N,d,topk", [(131072, 128, 0.3), (131071, 64, 0.5)])
def test_topk_at_max_length(N, d, topk, cuda_device):
    wl = W.custom("maxn", B=1, H=1, d=d, N=N, seed=N % 1000 + d)
    q, k, v = W.make_qkv(wl)
    assert wl.Kb == 2048
    out, mask = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, return_mask=True)
    torch.cuda.synchronize()
    mref, P = O.select(q, k, topk)
    bad, _, _ = compare_masks(mask, mref, P, O.keep_count(topk, wl.Kb))
    assert bad == 0
    agree = np.all(mask.cpu().numpy() == mref, axis=-1)
    got, ref = _rows(out, q, k, v, mref, agree, sampled_blocks(wl.Qb, 4, seed=N), N)
    assert_close(got, ref, f"max-length topk {N, d}")


def test_cdf_at_max_length(cuda_device):
    N, d, tau = 131071, 128, 0.9
    wl = W.custom("maxc", B=1, H=1, d=d, N=N, seed=11)
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_cdf(q.cuda(), k.cuda(), v.cuda(), tau, return_mask=True)
    torch.cuda.synchronize()
    mref, P = O.select_cdf(q, k, tau)
    bad, _ = compare_cdf_masks(mask, mref, P, tau)
    assert bad == 0
    agree = np.all(mask.cpu().numpy() == mref, axis=-1)
    got, ref = _rows(out, q, k, v, mref, agree, sampled_blocks(wl.Qb, 4, seed=5), N)
    assert_close(got, ref, "max-length cdf")


def test_causal_topk_at_max_length(cuda_device):
    N, d, topk = 131072, 128, 0.5
    wl = W.custom("maxcausal", B=1, H=1, d=d, N=N, seed=17)
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, is_causal=True, return_mask=True)
    torch.cuda.synchronize()
    mref, P = O.select(q, k, topk, causal=True)
    mg = mask.cpu().numpy()
    for i in range(wl.Qb):
        E = O.causal_block_limit(i, wl.Kb)
        kk = O.keep_count(topk, E)
        assert np.all(mg[0, 0, i, E:] == 0) and mg[0, 0, i].sum() == kk
        if np.any(mg[0, 0, i] != mref[0, 0, i]):
            assert O.tie_exempt_rows(P[:, :, i:i + 1, :E], kk)[0, 0, 0]
    agree = np.all(mg == mref, axis=-1)
    got, ref = _rows(out, q, k, v, mref, agree, sampled_blocks(wl.Qb, 4, seed=9), N, causal=True)
    assert_close(got, ref, "max-length causal topk")


def test_host_call_at_max_length(cuda_device):
    N, d = 131072, 64
    wl = W.custom("maxhost", B=1, H=3, d=d, N=N, seed=23)
    q, k, v = W.make_qkv(wl)
    ref = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), 0.5)
    out = bsa.sparse_attn_topk_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), 0.5)
    assert torch.equal(out, ref.cpu())
