"""The seeded synthetic inputs: shapes, determinism and the recipe's structure.  No GPU."""
import torch

from block_sparse_attention_14_b200 import workloads as W


def test_config_shapes():
    assert (W.WORKLOADS["tiny"].N, W.WORKLOADS["tiny"].Qb, W.WORKLOADS["tiny"].Kb) == (1024, 8, 16)
    assert (W.WORKLOADS["cogvideox2b"].N, W.WORKLOADS["cogvideox2b"].Qb, W.WORKLOADS["cogvideox2b"].Kb) == (17776, 139, 278)
    assert (W.WORKLOADS["wan14b"].N, W.WORKLOADS["wan14b"].Qb, W.WORKLOADS["wan14b"].Kb) == (75600, 591, 1182)
    assert (W.WORKLOADS["hunyuan13b"].N, W.WORKLOADS["hunyuan13b"].Qb, W.WORKLOADS["hunyuan13b"].Kb) == (118800, 929, 1857)


def test_qkv_deterministic_bf16_contiguous():
    wl = W.WORKLOADS["tiny"]
    a = W.make_qkv(wl)
    b = W.make_qkv(wl)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 2, 1024, 64) and x.is_contiguous()
        assert torch.equal(x, y)
    q, k, v = a
    assert not torch.equal(q, k)
    # v ~ N(0, 1)
    assert abs(v.float().mean().item()) < 0.02 and abs(v.float().std().item() - 1) < 0.02


def test_field_is_spatially_coherent_and_text_is_noise():
    wl = W.WORKLOADS["cogvideox2b"]
    small = W.Workload("s", B=1, H=2, d=64, grid=(3, 8, 8), text=10)
    q, k, v = W.make_qkv(small)
    # neighbouring video tokens correlate far more than random text tokens do
    vid = q[0, 0, small.text:].float()
    c_near = torch.nn.functional.cosine_similarity(vid[:-1], vid[1:]).mean()
    txt = q[0, 0, :small.text].float()
    c_txt = torch.nn.functional.cosine_similarity(txt[:-1], txt[1:]).mean()
    assert c_near > 0.5 and abs(c_txt) < 0.3
    assert wl.text == 226


def test_random_mask_density():
    wl = W.Workload("m", B=1, H=4, d=64, grid=(1, 1, 64 * 200))
    m = W.make_random_mask(wl, 0.1)
    assert m.dtype == torch.uint8 and m.shape == (1, 4, wl.Qb, wl.Kb)
    assert set(m.unique().tolist()) <= {0, 1}
    assert abs(m.float().mean().item() - 0.1) < 0.01
