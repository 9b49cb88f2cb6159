"""GPU parity against the fp64 oracle on small and ragged shapes, through the C ABI
(via the Python binding), plus edge cases: empty rows, single tiles, odd kept
counts, ragged last blocks, the dense limit, compaction exactness, output canary
and determinism."""
import numpy as np
import pytest
import torch

import block_sparse_attention_14_b200 as bsa
from block_sparse_attention_14_b200 import workloads as W
from oracle import bsa_oracle as O
from tests.parity import assert_close
from tests import parity as P

pytestmark = pytest.mark.gpu


def _qkv(B, H, N, d, seed, scale=1.0):
    """q, k ~ N(0, scale^2) (a larger scale sharpens the softmax); v ~ N(0, 1) as in
    the workloads, so |out| stays where a 2e-2 absolute bound is meaningful for bf16."""
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, d, generator=g) for _ in range(3))
    return [(q * scale).to(torch.bfloat16), (k * scale).to(torch.bfloat16), v.to(torch.bfloat16)]


def _cuda(*ts):
    return [t.cuda() for t in ts]


SHAPES = [(1, 2, 1024, 64), (1, 2, 1024, 128), (2, 3, 300, 64), (1, 2, 300, 128),
          (1, 1, 1, 64), (1, 1, 65, 128), (1, 2, 4113, 128), (1, 1, 2000, 64)]


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 257])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_sequences_through_the_whole_path(N, d, causal, cuda_device):
    """The degenerate lengths through selection and attention: one key block
    (flat top-k rows), a partial single query block, the 64- and 128-row block
    edges; the block dot products then see tiles almost entirely past the data."""
    B, H, topk = 1, 2, 0.5
    q, k, v = _qkv(B, H, N, d, seed=N * 7 + d + causal)
    out, mask = bsa.sparse_attn_topk(*_cuda(q, k, v), topk, causal, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select(q, k, topk, causal=causal)
    mc = P.check_topk_mask(mask, mref, Pr, topk, causal=causal, what=f"tiny N={N} d={d}")
    ref = O.block_sparse_attention(q, k, v, mc.mask, causal=causal)
    assert_close(out.float().cpu().numpy(), ref, f"tiny N={N} d={d} causal={causal}")


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 257])
@pytest.mark.parametrize("d", [64, 128])
def test_tiny_sequences_cdf_and_caller_mask(N, d, cuda_device):
    """The same lengths through cdfthreshd selection and through a caller's random
    mask (compaction; empty rows included)."""
    B, H = 1, 2
    q, k, v = _qkv(B, H, N, d, seed=N * 11 + d)
    out, mask = bsa.sparse_attn_cdf(*_cuda(q, k, v), 0.9, return_mask=True)
    torch.cuda.synchronize()
    Pr = O.select(q, k, 1.0)[1]
    mref = O.cdf_mask(Pr, 0.9)
    mc = P.check_cdf_mask(mask, mref, Pr, 0.9, what=f"tiny cdf N={N} d={d}")
    assert_close(out.float().cpu().numpy(), O.block_sparse_attention(q, k, v, mc.mask), f"tiny cdf N={N} d={d}")
    Qb, Kb = O.block_counts(N)
    g = torch.Generator().manual_seed(N + d)
    m = (torch.rand(B, H, Qb, Kb, generator=g) < 0.5).to(torch.uint8)
    out2 = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), m.cuda())
    torch.cuda.synchronize()
    assert_close(out2.float().cpu().numpy(), O.block_sparse_attention(q, k, v, m.numpy()), f"tiny mask N={N} d={d}")


@pytest.mark.parametrize("B,H,N,d", SHAPES)
def test_dense_mask_none_matches_oracle(B, H, N, d, cuda_device):
    q, k, v = _qkv(B, H, N, d, seed=N + d, scale=1.5)
    out = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), None)
    torch.cuda.synchronize()
    ref = O.dense_attention(q, k, v)
    assert_close(out.float().cpu().numpy(), ref, f"dense {B,H,N,d}")


@pytest.mark.parametrize("B,H,N,d,density", [(1, 3, 1000, 64, 0.3), (1, 3, 1000, 128, 0.3),
                                             (2, 2, 2081, 128, 0.5), (1, 2, 4096, 64, 0.1),
                                             (1, 2, 1537, 128, 0.05)])
def test_caller_mask_matches_oracle(B, H, N, d, density, cuda_device):
    q, k, v = _qkv(B, H, N, d, seed=7 * N + d, scale=2.0)
    Qb, Kb = O.block_counts(N)
    g = torch.Generator().manual_seed(N)
    mask = (torch.rand(B, H, Qb, Kb, generator=g) < density).to(torch.uint8)
    mask[0, 0, 0] = 0                  # empty row -> zero output
    mask[0, -1, -1] = 0
    mask[0, -1, -1, -1] = 1            # only the ragged last key block
    if Qb > 1:
        mask[0, 0, 1] = 0
        mask[0, 0, 1, Kb // 2] = 1     # a single kept tile (odd count)
        mask[-1, 0, 1] = 1             # a full row (dense)
    out = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), mask.cuda())
    torch.cuda.synchronize()
    ref = O.block_sparse_attention(q, k, v, mask.numpy())
    got = out.float().cpu().numpy()
    assert np.all(got[0, 0, :128] == 0), "empty row must be exactly zero"
    assert_close(got, ref, f"mask {B,H,N,d,density}")


def test_tiny_workload_fused_topk(cuda_device):
    wl = W.WORKLOADS["tiny"]
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_topk(*_cuda(q, k, v), topk=0.5, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select(q, k, 0.5)
    mc = P.check_topk_mask(mask, mref, Pr, 0.5, what="tiny")
    # every row, against the oracle's attention over the validated GPU mask
    ref = O.block_sparse_attention(q, k, v, mc.mask)
    assert_close(out.float().cpu().numpy(), ref, f"tiny fused; {mc}")


@pytest.mark.parametrize("N,d,topk", [(3000, 128, 0.3), (3000, 64, 0.5), (777, 128, 0.2),
                                      (8192, 128, 0.1), (5000, 64, 1.0)])
def test_fused_topk_matches_oracle(N, d, topk, cuda_device):
    wl = W.custom("c", B=1, H=3, d=d, N=N, seed=N)
    q, k, v = W.make_qkv(wl)
    out, mask = bsa.sparse_attn_topk(*_cuda(q, k, v), topk=topk, return_mask=True)
    torch.cuda.synchronize()
    mref, Pr = O.select(q, k, topk)
    mc = P.check_topk_mask(mask, mref, Pr, topk, what=f"fused {N,d,topk}")
    ref = O.block_sparse_attention(q, k, v, mc.mask)
    assert_close(out.float().cpu().numpy(), ref, f"fused {N,d,topk}; {mc}")


def test_select_equals_fused_mask_and_block_scores(cuda_device):
    wl = W.custom("s", B=2, H=2, d=128, N=2500, seed=3)
    q, k, v = _cuda(*W.make_qkv(wl))
    m1 = bsa.sparse_attn_select(q, k, 0.4)
    _, m2 = bsa.sparse_attn_topk(q, k, v, 0.4, return_mask=True)
    assert torch.equal(m1, m2)
    P = bsa.sparse_attn_block_scores(q, k)
    torch.cuda.synchronize()
    _, Pref = O.select(q.cpu(), k.cpu(), 0.4)
    Pg = P.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(Pg.sum(-1), 1.0, rtol=0, atol=1e-5)
    np.testing.assert_allclose(Pg, Pref, rtol=1e-4, atol=1e-7)


@pytest.mark.parametrize("B,H,N,d", [(1, 3, 20000, 128), (2, 2, 17776, 64), (1, 2, 1000, 128)])
def test_block_dot_products_match_fp64(B, H, N, d, cuda_device):
    """The raw block dot products Qbar_i . Kbar_j that the selection ranks, read from
    the workspace, against fp64 dot products of the oracle's pooled means: within
    4e-6 of |Qbar_i| |Kbar_j| (fp32-like; the tensor cores compute them from a TF32
    hi/lo split).  The shapes cover several 128 x 256 tiles with ragged edges in
    both directions, and a single partial tile."""
    wl = W.custom("dots", B=B, H=H, d=d, N=N, seed=N + d)
    q, k, _ = W.make_qkv(wl)
    Qb, Kb = O.block_counts(N)
    ws = bsa.make_workspace(B, H, N, d)
    bsa.sparse_attn_block_scores(q.cuda(), k.cuda(), workspace=ws)
    bsa.last_device_status(ws)
    r = lambda x: (x + 255) // 256 * 256
    BH, Kp = B * H, (Kb + 3) // 4 * 4
    o_s = 256 + r(BH * Qb * d * 4) + r(BH * Kb * d * 4)
    S = ws[o_s:o_s + BH * Qb * Kp * 4].view(torch.float32).view(B, H, Qb, Kp)[..., :Kb].cpu().numpy()
    qbar = O.pool_mean(O.to_f64(q), 128)
    kbar = O.pool_mean(O.to_f64(k), 64)
    S64 = np.einsum("bhid,bhjd->bhij", qbar, kbar)
    norm = np.linalg.norm(qbar, axis=-1)[..., :, None] * np.linalg.norm(kbar, axis=-1)[..., None, :]
    err = np.abs(S.astype(np.float64) - S64) / norm
    assert err.max() <= 4e-6, f"max error {err.max():.2e} of |Qbar||Kbar|"


def test_topk_one_equals_dense_bitwise(cuda_device):
    q, k, v = _cuda(*_qkv(1, 2, 3001, 128, seed=5))
    a = bsa.sparse_attn_topk(q, k, v, 1.0)
    b = bsa.block_sparse_attn_fwd(q, k, v, None)
    ones = torch.ones(1, 2, *O.block_counts(3001), dtype=torch.uint8, device="cuda")
    c = bsa.block_sparse_attn_fwd(q, k, v, ones)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(b, c)


def test_compaction_is_exact(cuda_device):
    B, H, N, d = 1, 4, 5000, 64
    q, k, v = _cuda(*_qkv(B, H, N, d, seed=11))
    Qb, Kb = O.block_counts(N)
    g = torch.Generator().manual_seed(2)
    mask = (torch.rand(B, H, Qb, Kb, generator=g) < 0.37).to(torch.uint8)
    mask[0, 1, 3] = 7  # any nonzero value means keep
    ws = bsa.make_workspace(B, H, N, d)
    bsa.block_sparse_attn_fwd(q, k, v, mask.cuda(), workspace=ws)
    torch.cuda.synchronize()
    BH = B * H
    idx, cnt = P.workspace_lists(ws, BH, Qb, Kb, d)
    m = mask.view(BH * Qb, Kb).numpy()
    for row in range(BH * Qb):
        want = np.flatnonzero(m[row])
        assert cnt[row] == want.size
        assert np.array_equal(idx[row, :cnt[row]], want)


def test_no_writes_outside_output_and_deterministic(cuda_device):
    B, H, N, d = 1, 3, 1111, 128
    q, k, v = _cuda(*_qkv(B, H, N, d, seed=13))
    n = B * H * N * d
    buf = torch.full((n + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[:n].view(B, H, N, d)
    bsa.sparse_attn_topk(q, k, v, 0.5, out=out)
    first = out.clone()
    bsa.sparse_attn_topk(q, k, v, 0.5, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[n:] == 7.0)
    assert torch.equal(first, out)


def test_status_ok_after_a_normal_call(cuda_device):
    q, k, v = _cuda(*_qkv(1, 1, 256, 64, seed=1))
    ws = bsa.make_workspace(1, 1, 256, 64)
    bsa.sparse_attn_topk(q, k, v, 0.5, workspace=ws)
    bsa.last_device_status(ws)  # raises on a recorded timeout
    with pytest.raises(bsa.BsaError) as e:
        bsa.sparse_attn_cdf(q, k, v, 0.9, is_causal=True)
    assert e.value.status == 2


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 1024, 64), (1, 2, 300, 128), (2, 2, 4113, 128), (1, 1, 65, 64)])
def test_causal_dense_matches_oracle(B, H, N, d, cuda_device):
    q, k, v = _qkv(B, H, N, d, seed=N + 3 * d, scale=1.5)
    out = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), None, is_causal=True)
    torch.cuda.synchronize()
    Qb, Kb = O.block_counts(N)
    ref = O.block_sparse_attention(q, k, v, np.ones((B, H, Qb, Kb), np.uint8), causal=True)
    assert_close(out.float().cpu().numpy(), ref, f"causal dense {B,H,N,d}")


@pytest.mark.parametrize("N,d,density", [(2000, 128, 0.5), (1537, 64, 0.3)])
def test_causal_caller_mask_matches_oracle(N, d, density, cuda_device):
    B, H = 1, 3
    q, k, v = _qkv(B, H, N, d, seed=11 * N + d, scale=2.0)
    Qb, Kb = O.block_counts(N)
    g = torch.Generator().manual_seed(N + 5)
    mask = (torch.rand(B, H, Qb, Kb, generator=g) < density).to(torch.uint8)
    mask[0, 0, 2] = 0
    mask[0, 0, 2, 5] = 1          # only the second diagonal block: rows 256..319 see nothing
    mask[0, 1, 3] = 0
    mask[0, 1, 3, 7] = 1
    mask[0, 1, 3, 9] = 1          # an ineligible block, ignored under causal attention
    out = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), mask.cuda(), is_causal=True)
    torch.cuda.synchronize()
    ref = O.block_sparse_attention(q, k, v, mask.numpy(), causal=True)
    got = out.float().cpu().numpy()
    assert np.all(got[0, 0, 256:320] == 0)
    assert_close(got, ref, f"causal mask {N,d,density}")


@pytest.mark.parametrize("N,d,topk", [(3000, 128, 0.5), (2500, 64, 0.3), (777, 128, 0.2)])
def test_causal_fused_topk_matches_oracle(N, d, topk, cuda_device):
    wl = W.custom("ct", B=1, H=3, d=d, N=N, seed=N + 7)
    q, k, v = W.make_qkv(wl)
    qc, kc, vc = _cuda(q, k, v)
    out, mask = bsa.sparse_attn_topk(qc, kc, vc, topk, is_causal=True, return_mask=True)
    m2 = bsa.sparse_attn_select(qc, kc, topk, is_causal=True)
    torch.cuda.synchronize()
    assert torch.equal(mask, m2)
    mref, Pr = O.select(q, k, topk, causal=True)
    # per-row k over the eligible blocks; rows may differ only within the tie band
    mc = P.check_topk_mask(mask, mref, Pr, topk, causal=True, what=f"causal topk {N,d,topk}")
    ref = O.block_sparse_attention(q, k, v, mc.mask, causal=True)
    assert_close(out.float().cpu().numpy(), ref, f"causal topk {N,d,topk}; {mc}")


@pytest.mark.parametrize("N,d,tau", [(3000, 128, 0.5), (3000, 128, 0.9), (2500, 64, 0.95), (777, 128, 0.3),
                                     (4096, 64, 1.0)])
def test_cdf_selection_and_attention_match_oracle(N, d, tau, cuda_device):
    wl = W.custom("cdf", B=1, H=3, d=d, N=N, seed=N + 1)
    q, k, v = W.make_qkv(wl)
    qc, kc, vc = _cuda(q, k, v)
    m1 = bsa.sparse_attn_select_cdf(qc, kc, tau)
    out, m2 = bsa.sparse_attn_cdf(qc, kc, vc, tau, return_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(m1, m2)
    mref, Pr = O.select_cdf(q, k, tau)
    mc = P.check_cdf_mask(m1, mref, Pr, tau, what=f"cdf {N,d,tau}")
    ref = O.block_sparse_attention(q, k, v, mc.mask)
    assert_close(out.float().cpu().numpy(), ref, f"cdf {N,d,tau}; {mc}")


@pytest.mark.parametrize("N,d,scale,causal,order", [(3000, 128, 4.0, False, "ascending"),
                                                    (3000, 64, 4.0, False, "ascending"),
                                                    (2500, 128, 4.0, True, "ascending"),
                                                    (3000, 128, 3.0, False, "random")])
def test_large_score_jumps_rescale_exactly(N, d, scale, causal, order, cuda_device):
    """Scores of tens to ~100 in log2 units that grow from one kept pair to the next:
    the running reference maximum is raised, and O and l rescaled, many times per
    row; the result must still match the fp64 oracle.  (Much larger scores make the
    fp32 accumulation of the tensor-core Q K^T product, not the softmax, the limit:
    at q, k ~ N(0, 36) with d = 64 the max-abs error reaches ~3e-2.)"""
    q, k, v = _qkv(1, 2, N, d, seed=N + d, scale=scale)
    if order == "ascending":
        # make later key blocks score higher for every query: add a ramp along the keys
        ramp = torch.linspace(0.0, 3.0 * scale, N).view(1, 1, N, 1)
        k = (k.float() + ramp * q.float().mean(dim=2, keepdim=True).sign()).to(torch.bfloat16)
    out = bsa.block_sparse_attn_fwd(*_cuda(q, k, v), None, is_causal=causal)
    torch.cuda.synchronize()
    Qb, Kb = O.block_counts(N)
    ones = np.ones((1, 2, Qb, Kb), dtype=np.uint8)
    ref = O.block_sparse_attention(q, k, v, ones, causal=causal)
    assert_close(out.float().cpu().numpy(), ref, f"large score jumps {N, d, scale, causal, order}")
