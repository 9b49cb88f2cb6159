"""GPU parity at the full sizes of the five video-shaped workloads, in the same calls
the benchmark times.  Selection masks are compared in full (bit-exact outside the
tie band); attention outputs in full for the tiny and CogVideoX-2B shapes and on a
fixed sample of query blocks ({0, 1, Qb/2, Qb-1} plus seeded random blocks,
including the ragged last block) for the N = 75600 and N = 118800 shapes, whose
full fp64 oracle would take hours.  The host-buffer call the benchmark's end-to-end
figure times is compared byte for byte with the device call at Wan2.1-14B size."""
import functools

import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests.parity import assert_close, compare_masks, sampled_blocks
from tests import parity as P

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=1)
def _inputs(name):
    wl = W.WORKLOADS[name]
    q, k, v = W.make_qkv(wl)
    return wl, (q, k, v), (q.cuda(), k.cuda(), v.cuda())


@functools.lru_cache(maxsize=4)
def _oracle_select(name, topk):
    wl, (q, k, _), _ = _inputs(name)
    return O.select(q, k, topk)


def _check_rows(out, wl, qkv_cpu, mask_ref, agree, heads, n_random, seed):
    """Compare sampled query blocks (where the GPU and oracle masks agree)."""
    q, k, v = qkv_cpu
    got_all, ref_all = [], []
    o = out.cpu()
    for b in range(wl.B):
        for h in heads:
            blocks = [i for i in sampled_blocks(wl.Qb, n_random, seed + 97 * h + b) if agree[b, h, i]]
            qh, kh, vh = O.to_f64(q[b, h]), O.to_f64(k[b, h]), O.to_f64(v[b, h])
            for i in blocks:
                lo, hi = 128 * i, min(wl.N, 128 * i + 128)
                ref_all.append(O.attention_rows(qh, kh, vh, mask_ref[b, h, i], i))
                got_all.append(o[b, h, lo:hi].float().numpy())
    return assert_close(np.concatenate(got_all), np.concatenate(ref_all), wl.name)


def _fused_case(name, topk, heads=None, n_random=4, full=False):
    wl, qkv_cpu, (q, k, v) = _inputs(name)
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out, mask = bsa.sparse_attn_topk(q, k, v, topk, return_mask=True, workspace=ws)
    bsa.last_device_status(ws)
    mref, P = _oracle_select(name, topk)
    kk = O.keep_count(topk, wl.Kb)
    bad, n_exempt, n_diff_exempt = compare_masks(mask, mref, P, kk)
    assert bad == 0, f"{bad} non-exempt mask rows differ"
    agree = np.all(mask.cpu().numpy() == mref, axis=-1)
    if full:
        ref = O.block_sparse_attention(*qkv_cpu, mref)
        rows = np.repeat(agree, 128, axis=2)[:, :, :wl.N]
        assert_close(out.float().cpu().numpy()[rows], ref[rows], name)
    else:
        _check_rows(out, wl, qkv_cpu, mref, agree, heads or range(wl.H), n_random, seed=int(topk * 1000))
    return n_exempt, n_diff_exempt


def test_cogvideox2b_fused_topk05_full():
    _fused_case("cogvideox2b", 0.5, full=True)


@pytest.mark.parametrize("topk", [1.0, 0.5, 0.3, 0.1])
def test_wan13b_fused_topk_sweep(topk):
    _fused_case("wan13b", topk, n_random=3)


def test_wan14b_fused_topk05():
    _fused_case("wan14b", 0.5, heads=[0, 7, 13, 21, 27, 39], n_random=6)


@pytest.mark.parametrize("density", [0.5, 0.1])
def test_wan14b_caller_mask(density):
    wl, qkv_cpu, (q, k, v) = _inputs("wan14b")
    mask = W.make_random_mask(wl, density)
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out = bsa.block_sparse_attn_fwd(q, k, v, mask.cuda(), workspace=ws)
    bsa.last_device_status(ws)
    # The caller mask passes bit-exactly into the kept-block lists.
    BH, Qb, Kb = wl.B * wl.H, wl.Qb, wl.Kb
    idx, cnt = P.workspace_lists(ws, BH, Qb, Kb, wl.d)
    m = mask.view(BH * Qb, Kb).numpy()
    assert np.array_equal(cnt, m.sum(1))
    order = np.argsort(m == 0, axis=1, kind="stable")
    valid = np.arange(Kb)[None, :] < cnt[:, None]
    assert np.array_equal(np.where(valid, idx, -1), np.where(valid, order, -1))
    agree = np.ones((wl.B, wl.H, Qb), dtype=bool)
    _check_rows(out, wl, qkv_cpu, mask.numpy(), agree, [0, 9, 19, 29, 39], 6, seed=int(density * 100))


def test_hunyuan13b_fused_topk01():
    _fused_case("hunyuan13b", 0.1, heads=[0, 5, 11, 17, 23], n_random=6)


def test_wan13b_fused_cdf09():
    from tests.parity import compare_cdf_masks

    wl, qkv_cpu, (q, k, v) = _inputs("wan13b")
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out, mask = bsa.sparse_attn_cdf(q, k, v, 0.9, return_mask=True, workspace=ws)
    bsa.last_device_status(ws)
    mref, P = O.cdf_mask(_oracle_select("wan13b", 1.0)[1], 0.9), _oracle_select("wan13b", 1.0)[1]
    bad, _ = compare_cdf_masks(mask, mref, P, 0.9)
    assert bad == 0
    agree = np.all(mask.cpu().numpy() == mref, axis=-1)
    _check_rows(out, wl, qkv_cpu, mref, agree, range(wl.H), 3, seed=90)


def test_wan14b_host_buffer_call_matches_device_call():
    """The end-to-end call the benchmark times (pinned host buffers, default head
    chunking) writes exactly the bytes of the device call at full Wan2.1-14B size;
    the device call itself is checked against the oracle above."""
    wl, (q, k, v), (qd, kd, vd) = _inputs("wan14b")
    ref = bsa.sparse_attn_topk(qd, kd, vd, 0.5)
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out = bsa.sparse_attn_topk_host(qp, kp, vp, 0.5, workspace=ws)
    bsa.last_device_status(ws)
    assert torch.equal(out, ref.cpu())
