"""GPU parity at the full sizes of the five video-shaped workloads, in the same calls
the benchmark times (the causal ones too).  Selection masks are compared in full (bit-exact outside the
tie band); attention outputs in full for the tiny and CogVideoX-2B shapes and on a
fixed sample of query blocks ({0, 1, Qb/2, Qb-1} plus seeded random blocks,
including the ragged last block) for the N = 75600 and N = 118800 shapes, whose
full fp64 oracle would take hours.  Every query block whose GPU mask differs from
the oracle's (inside the tie band) is compared too, against the oracle's attention
over the GPU mask.  The host-buffer call the benchmark's end-to-end
figure times is compared byte for byte with the device call at Wan2.1-14B size."""
import functools

import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests.parity import assert_close, sampled_blocks
from tests import parity as P

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=1)
def _inputs(name):
    wl = W.WORKLOADS[name]
    q, k, v = W.make_qkv(wl)
    return wl, (q, k, v), (q.cuda(), k.cuda(), v.cuda())


@functools.lru_cache(maxsize=4)
def _oracle_select(name, topk, causal=False):
    wl, (q, k, _), _ = _inputs(name)
    return O.select(q, k, topk, causal=causal)


def _check_rows(out, wl, qkv_cpu, mask_np, heads, n_random, seed, extra=None, what="", causal=False):
    """Compare sampled query blocks of the listed heads, plus every (b, h, i) in
    `extra` (the rows whose GPU mask differs from the oracle's), with the oracle's
    attention over `mask_np`."""
    q, k, v = qkv_cpu
    extra = extra or {}
    got_all, ref_all = [], []
    o = out.cpu()
    for b in range(wl.B):
        for h in range(wl.H):
            blocks = set(extra.get((b, h), []))
            if h in heads:
                blocks |= set(sampled_blocks(wl.Qb, n_random, seed + 97 * h + b))
            if not blocks:
                continue
            qh, kh, vh = O.to_f64(q[b, h]), O.to_f64(k[b, h]), O.to_f64(v[b, h])
            for i in sorted(blocks):
                lo, hi = 128 * i, min(wl.N, 128 * i + 128)
                ref_all.append(O.attention_rows(qh, kh, vh, mask_np[b, h, i], i, causal=causal))
                got_all.append(o[b, h, lo:hi].float().numpy())
    return assert_close(np.concatenate(got_all), np.concatenate(ref_all), what or wl.name)


def _differing(mc, mref, wl):
    return {(b, h): P.differing_blocks(mc, mref, b, h) for b in range(wl.B) for h in range(wl.H)}


def _fused_case(name, topk, heads=None, n_random=4, full=False, causal=False):
    wl, qkv_cpu, (q, k, v) = _inputs(name)
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out, mask = bsa.sparse_attn_topk(q, k, v, topk, causal, return_mask=True, workspace=ws)
    bsa.last_device_status(ws)
    mref, Pr = _oracle_select(name, topk, causal)
    what = f"{name} topk {topk}{' causal' if causal else ''}"
    mc = P.check_topk_mask(mask, mref, Pr, topk, causal=causal, what=what)
    print(f"{what}: {mc}")
    if full:
        ref = O.block_sparse_attention(*qkv_cpu, mc.mask, causal=causal)
        assert_close(out.float().cpu().numpy(), ref, f"{what}; {mc}")
    else:
        heads = set(heads if heads is not None else range(wl.H))
        _check_rows(out, wl, qkv_cpu, mc.mask, heads, n_random, seed=int(topk * 1000),
                    extra=_differing(mc, mref, wl), what=f"{what}; {mc}", causal=causal)
    return mc


def test_cogvideox2b_fused_topk05_full():
    _fused_case("cogvideox2b", 0.5, full=True)


def test_cogvideox2b_fused_topk05_causal_full():
    """The causal call of the d = 64 kernel at full size, every row: per-row top-k
    over the eligible blocks, the diagonal masked element by element."""
    _fused_case("cogvideox2b", 0.5, full=True, causal=True)


@pytest.mark.parametrize("topk", [1.0, 0.5, 0.3, 0.1])
def test_wan13b_fused_topk_sweep(topk):
    _fused_case("wan13b", topk, n_random=3)


def test_wan14b_fused_topk05():
    _fused_case("wan14b", 0.5, heads=[0, 7, 13, 21, 27, 39], n_random=6)


def test_wan14b_fused_topk05_causal():
    _fused_case("wan14b", 0.5, heads=[0, 13, 27, 39], n_random=6, causal=True)


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
    _check_rows(out, wl, qkv_cpu, mask.numpy(), {0, 9, 19, 29, 39}, 6, seed=int(density * 100))


def test_hunyuan13b_fused_topk01():
    _fused_case("hunyuan13b", 0.1, heads=[0, 5, 11, 17, 23], n_random=6)


def test_wan13b_fused_cdf09():
    wl, qkv_cpu, (q, k, v) = _inputs("wan13b")
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out, mask = bsa.sparse_attn_cdf(q, k, v, 0.9, return_mask=True, workspace=ws)
    bsa.last_device_status(ws)
    Pr = _oracle_select("wan13b", 1.0)[1]
    mref = O.cdf_mask(Pr, 0.9)
    mc = P.check_cdf_mask(mask, mref, Pr, 0.9, what="wan13b cdf 0.9")
    print(f"wan13b cdf 0.9: {mc}")
    _check_rows(out, wl, qkv_cpu, mc.mask, set(range(wl.H)), 3, seed=90,
                extra=_differing(mc, mref, wl), what=f"wan13b cdf; {mc}")


def test_cogvideox2b_fused_cdf09_full():
    """cdfthreshd at d = 64 and full CogVideoX-2B size, every row: the score-ordered
    prefix reaching 0.9 of the block-score mass, then attention over it."""
    wl, qkv_cpu, (q, k, v) = _inputs("cogvideox2b")
    ws = bsa.make_workspace(wl.B, wl.H, wl.N, wl.d)
    out, mask = bsa.sparse_attn_cdf(q, k, v, 0.9, return_mask=True, workspace=ws)
    bsa.last_device_status(ws)
    Pr = _oracle_select("cogvideox2b", 1.0)[1]
    mref = O.cdf_mask(Pr, 0.9)
    mc = P.check_cdf_mask(mask, mref, Pr, 0.9, what="cogvideox2b cdf 0.9")
    print(f"cogvideox2b cdf 0.9: {mc}")
    ref = O.block_sparse_attention(*qkv_cpu, mc.mask)
    assert_close(out.float().cpu().numpy(), ref, f"cogvideox2b cdf 0.9; {mc}")


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
