"""Plan reuse (the build_plan / apply_plan split of the AB-Attention README, "Use an
existing pipeline", with one plan refresh every few denoising steps as in its
"Paper settings, timing, and pipeline integration"): the kept-block lists made
once by a selection (or from a caller mask) are applied to several CHANGED
(q, k, v), and every apply is compared with the fp64 oracle's attention over the
stored mask.  In full at small ragged shapes; at the full Wan2.1-1.3B shape on
sampled query blocks of every head."""
import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests import parity as P
from tests.parity import assert_close, sampled_blocks

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,topk,causal", [
    (2, 3, 3001, 128, 0.4, False),
    (1, 3, 2500, 64, 0.3, False),
    (1, 2, 2900, 128, 0.5, True),
])
def test_select_once_apply_to_changed_inputs(B, H, N, d, topk, causal, cuda_device):
    wl0 = W.custom("plan", B=B, H=H, d=d, N=N, seed=N + d)
    q0, k0, _ = W.make_qkv(wl0)
    ws = bsa.make_workspace(B, H, N, d)
    mask = bsa.sparse_attn_select(q0.cuda(), k0.cuda(), topk, causal, workspace=ws)
    torch.cuda.synchronize()
    mref, Pr = O.select(q0, k0, topk, causal=causal)
    mc = P.check_topk_mask(mask, mref, Pr, topk, causal=causal, what="plan")
    out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    for step in range(1, 4):
        q, k, v = W.make_qkv(W.custom("plan", B=B, H=H, d=d, N=N, seed=N + d + 101 * step))
        bsa.block_sparse_attn_apply(q.cuda(), k.cuda(), v.cuda(), ws, causal, out=out, check=True)
        ref = O.block_sparse_attention(q, k, v, mc.mask, causal=causal)
        assert_close(out.float().cpu().numpy(), ref, f"apply {step} of a stored plan")


def test_caller_mask_plan_applied_to_changed_inputs(cuda_device):
    B, H, N, d = 1, 3, 2222, 64
    Qb, Kb = O.block_counts(N)
    mask = (torch.rand(B, H, Qb, Kb, generator=torch.Generator().manual_seed(8)) < 0.35).to(torch.uint8)
    mask[0, 1, 4] = 0  # an empty row: zeros on every apply
    ws = bsa.make_workspace(B, H, N, d)
    q0 = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    bsa.block_sparse_attn_plan(q0, mask.cuda(), workspace=ws)
    for step in range(3):
        q, k, v = W.make_qkv(W.custom("planm", B=B, H=H, d=d, N=N, seed=50 + step))
        out = bsa.block_sparse_attn_apply(q.cuda(), k.cuda(), v.cuda(), ws, check=True)
        got = out.float().cpu().numpy()
        assert np.all(got[0, 1, 4 * 128:5 * 128] == 0)
        assert_close(got, O.block_sparse_attention(q, k, v, mask.numpy()), f"caller-mask plan, apply {step}")


def test_plan_reuse_wan13b_full_size(cuda_device):
    """Wan2.1-1.3B shape at topk 0.5: the plan of the seed-0 inputs applied to the
    inputs of three other seeds, sampled blocks of every head against the oracle."""
    base = W.WORKLOADS["wan13b"]
    q0, k0, _ = W.make_qkv(base)
    ws = bsa.make_workspace(base.B, base.H, base.N, base.d)
    mask = bsa.sparse_attn_select(q0.cuda(), k0.cuda(), 0.5, workspace=ws)
    torch.cuda.synchronize()
    mref, Pr = O.select(q0, k0, 0.5)
    mc = P.check_topk_mask(mask, mref, Pr, 0.5, what="wan13b plan")
    del q0, k0
    out = torch.empty(base.B, base.H, base.N, base.d, dtype=torch.bfloat16, device="cuda")
    for step in (1, 2, 3):
        wl = W.Workload(base.name, B=base.B, H=base.H, d=base.d, grid=base.grid, seed=step)
        q, k, v = W.make_qkv(wl)
        bsa.block_sparse_attn_apply(q.cuda(), k.cuda(), v.cuda(), ws, out=out, check=True)
        o = out.cpu()
        got, ref = [], []
        for h in range(wl.H):
            qh, kh, vh = O.to_f64(q[0, h]), O.to_f64(k[0, h]), O.to_f64(v[0, h])
            for i in sampled_blocks(wl.Qb, 2, seed=17 * step + h):
                lo, hi = 128 * i, min(wl.N, 128 * i + 128)
                ref.append(O.attention_rows(qh, kh, vh, mc.mask[0, h, i], i))
                got.append(o[0, h, lo:hi].float().numpy())
        assert_close(np.concatenate(got), np.concatenate(ref), f"wan13b plan, apply {step}")
