"""Parity at the largest sequence the library accepts (N = 131072, Kb = 2048 key
blocks, the top of the int16 index range and of the row kernels' shared-memory
sizing) and one below it (a ragged last block): selection in full against the
fp64 oracle, attention on sampled query blocks (the first, second, middle and
last, plus seeded random ones, and every block whose GPU mask differs from the
oracle's inside the tie band)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests import parity as P
from tests.parity import assert_close, sampled_blocks

pytestmark = pytest.mark.gpu


def _rows(out, q, k, v, mc, mask_ref, blocks, N, causal=False):
    """GPU and oracle rows of the sampled query blocks plus every block whose GPU
    mask differs from the oracle's; the oracle attends over the validated GPU mask."""
    got, ref = [], []
    o = out.cpu()
    qh, kh, vh = O.to_f64(q[0, 0]), O.to_f64(k[0, 0]), O.to_f64(v[0, 0])
    for i in sorted(set(blocks) | set(P.differing_blocks(mc, mask_ref, 0, 0))):
        lo, hi = 128 * i, min(N, 128 * i + 128)
        ref.append(O.attention_rows(qh, kh, vh, mc.mask[0, 0, i], i, causal=causal))
        got.append(o[0, 0, lo:hi].float().numpy())
    return np.concatenate(got), np.concatenate(ref)


@pytest.mark.parametrize("N,d,topk", [(131072, 128, 0.3), (131071, 64, 0.5)])
def test_topk_at_max_length(N, d, topk, cuda_device):
    wl = W.custom("maxn", B=1, H=1, d=d, N=N, seed=N % 1000 + d)
    q, k, v = W.make_qkv(wl)
    assert wl.Kb == 2048
    out, mask = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select(q, k, topk)
    mc = P.check_topk_mask(mask, mref, Pr, topk, what=f"max-length topk {N, d}")
    got, ref = _rows(out, q, k, v, mc, mref, sampled_blocks(wl.Qb, 4, seed=N), N)
    assert_close(got, ref, f"max-length topk {N, d}; {mc}")


def test_cdf_at_max_length(cuda_device):
    N, d, tau = 131071, 128, 0.9
    wl = W.custom("maxc", B=1, H=1, d=d, N=N, seed=11)
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_cdf(q.cuda(), k.cuda(), v.cuda(), tau, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select_cdf(q, k, tau)
    mc = P.check_cdf_mask(mask, mref, Pr, tau, what="max-length cdf")
    got, ref = _rows(out, q, k, v, mc, mref, sampled_blocks(wl.Qb, 4, seed=5), N)
    assert_close(got, ref, f"max-length cdf; {mc}")


def test_causal_topk_at_max_length(cuda_device):
    N, d, topk = 131072, 128, 0.5
    wl = W.custom("maxcausal", B=1, H=1, d=d, N=N, seed=17)
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), topk, is_causal=True, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select(q, k, topk, causal=True)
    mc = P.check_topk_mask(mask, mref, Pr, topk, causal=True, what="max-length causal topk")
    got, ref = _rows(out, q, k, v, mc, mref, sampled_blocks(wl.Qb, 4, seed=9), N, causal=True)
    assert_close(got, ref, f"max-length causal topk; {mc}")


def test_host_call_at_max_length(cuda_device):
    N, d = 131072, 64
    wl = W.custom("maxhost", B=1, H=3, d=d, N=N, seed=23)
    q, k, v = W.make_qkv(wl)
    ref = bsa.sparse_attn_topk(q.cuda(), k.cuda(), v.cuda(), 0.5)
    out = bsa.sparse_attn_topk_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), 0.5)
    assert torch.equal(out, ref.cpu())
