"""The C-ABI library loads, exports every entry point declared in include/bsa.h,
and rejects bad arguments on the host before touching a GPU.  No GPU needed."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_14_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)) - {"if", "sizeof"})


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert {"sparse_attn_select", "block_sparse_attn_fwd", "sparse_attn_topk",
            "bsa_workspace_bytes", "bsa_last_device_status"} <= set(names)
    L = bsa.lib()
    for n in names:
        assert hasattr(L, n), n
    assert L.bsa_abi_version() == 2


def test_status_strings():
    L = bsa.lib()
    for code, name in bsa.STATUS.items():
        assert L.bsa_status_string(code).decode() == name


def test_workspace_bytes():
    # status 256 + qbar + kbar + block scores (fp32, rows padded to 4) + idx (int16)
    # + cnt, each rounded up to 256 bytes
    def r(x):
        return (x + 255) // 256 * 256
    for B, H, N, d in [(1, 40, 75600, 128), (2, 30, 17776, 64), (1, 1, 1, 64), (1, 2, 1024, 64)]:
        BH, Qb, Kb = B * H, -(-N // 128), -(-N // 64)
        Kp = (Kb + 3) // 4 * 4
        want = (256 + r(BH * Qb * d * 4) + r(BH * Kb * d * 4) + r(BH * Qb * Kp * 4)
                + r(BH * Qb * Kb * 2) + r(BH * Qb * 4))
        assert bsa.workspace_bytes(B, H, N, d) == want
    for bad in [(0, 1, 64, 64), (1, 1, 64, 96), (1, 1, 131073, 64), (1, 1, 0, 128), (256, 256, 64, 64)]:
        assert bsa.workspace_bytes(*bad) == 0


# Distinct fake device addresses, far enough apart that no tensor of the shapes
# used here overlaps another (nothing is launched: every call is rejected on the host).
QA, KA, VA, OA = 1 << 30, (1 << 30) + (1 << 26), (1 << 30) + (2 << 26), (1 << 30) + (3 << 26)


def _call_topk(shape, topk=0.5, is_causal=0, q=QA, k=KA, v=VA, out=OA, ws=512, ws_bytes=None):
    L = bsa.lib()
    s = bsa.Shape(*shape)
    if ws_bytes is None:
        ws_bytes = L.bsa_workspace_bytes(s)
    return L.sparse_attn_topk(q, k, v, s, topk, is_causal, out, None, ws, ws_bytes, None)


def test_output_must_not_overlap_inputs():
    L = bsa.lib()
    s = bsa.Shape(1, 1, 128, 64)          # 16 KiB per tensor
    n = L.bsa_workspace_bytes(s)
    base = 1 << 20
    q, k, v, ws = base, base + (1 << 16), base + (2 << 16), base + (4 << 16)
    for out in (q, k + 4096, v - 4096):   # same as q, inside k, straddling into v
        assert L.sparse_attn_topk(q, k, v, s, 0.5, 0, out, None, ws, n, None) == 1
        assert b"overlaps" in L.bsa_last_error_message()
        assert L.block_sparse_attn_fwd(q, k, v, s, None, 0, out, ws, n, None) == 1
        assert L.block_sparse_attn_apply(q, k, v, s, 0, out, ws, n, None) == 1
    L.sparse_attn_topk_noalloc.argtypes = [ctypes.c_void_p] * 3 + [bsa.Shape, ctypes.c_float, ctypes.c_int] + [ctypes.c_void_p] * 3
    L.sparse_attn_topk_noalloc.restype = ctypes.c_int
    assert L.sparse_attn_topk_noalloc(q, k, v, s, 0.5, 0, k, None, None) == 1


@pytest.mark.parametrize("kw,code", [
    (dict(shape=(1, 1, 128, 96)), 1),              # d not 64/128
    (dict(shape=(1, 1, 0, 64)), 1),                 # empty sequence
    (dict(shape=(1, 1, 200000, 64)), 1),            # N too long
    (dict(shape=(1, 1, 128, 64), topk=0.0), 1),
    (dict(shape=(1, 1, 128, 64), topk=1.5), 1),
    (dict(shape=(1, 1, 128, 64), topk=float("nan")), 1),
    (dict(shape=(1, 1, 128, 64), q=None), 1),
    (dict(shape=(1, 1, 128, 64), v=VA + 8), 1),     # unaligned pointer
    (dict(shape=(1, 1, 128, 64), ws=None), 1),
    (dict(shape=(1, 1, 128, 64), ws=512 + 16), 1),  # workspace not 256-aligned
    (dict(shape=(1, 1, 128, 64), ws_bytes=100), 1),  # workspace too small
])
def test_fused_call_rejects_bad_arguments(kw, code):
    assert _call_topk(**kw) == code
    msg = bsa.lib().bsa_last_error_message().decode()
    assert msg != "" and "overlaps" not in msg


def test_other_calls_reject_bad_arguments():
    L = bsa.lib()
    s = bsa.Shape(1, 2, 300, 64)
    n = L.bsa_workspace_bytes(s)
    assert L.block_sparse_attn_fwd(256, 256, 256, s, None, 0, None, 512, n, None) == 1
    assert L.sparse_attn_select(256, 256, s, 0.5, 0, None, 512, n, None) == 1
    assert L.sparse_attn_select(256, 256, s, -1.0, 1, 1024, 512, n, None) == 1
    assert L.block_sparse_attn_plan(None, bsa.Shape(1, 1, 64, 96), 0, 512, n, None) == 1
    assert L.block_sparse_attn_apply(256, 256, 256, s, 0, None, 512, n, None) == 1
    na = L.sparse_attn_topk_noalloc
    na.restype = ctypes.c_int
    na.argtypes = [ctypes.c_void_p] * 3 + [bsa.Shape, ctypes.c_float, ctypes.c_int] + [ctypes.c_void_p] * 3
    assert na(QA, KA, VA, s, 0.0, 1, OA, None, None) == 1  # topk out of range
    assert na(QA, KA, VA, bsa.Shape(1, 2, 300, 80), 0.5, 1, OA, None, None) == 1  # d not 64/128
    assert L.sparse_attn_block_scores(256, 256, s, None, 512, n, None) == 1
    assert L.sparse_attn_block_scores(256, 256, bsa.Shape(1, 2, 300, 32), 1024, 512, n, None) == 1
    assert L.bsa_last_device_status(None, None) == 1
    assert L.sparse_attn_topk_host(None, 256, 256, s, 0.5, 0, 256, 256, 256, 256, 256, 512, n, 0, None) == 1


def test_binding_rejects_cpu_tensors():
    import torch

    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bsa.sparse_attn_topk(q, q, q, 0.5)


def test_cdf_calls_reject_bad_thresholds():
    L = bsa.lib()
    s = bsa.Shape(1, 2, 300, 64)
    n = L.bsa_workspace_bytes(s)
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert L.sparse_attn_select_cdf(256, 256, s, bad, 1024, 512, n, None) == 1
        assert L.sparse_attn_cdf(QA, KA, VA, s, bad, 0, OA, None, 512, n, None) == 1
        assert b"threshold" in L.bsa_last_error_message()
    assert L.sparse_attn_cdf(QA, KA, VA, s, 0.9, 1, OA, None, 512, n, None) == 2
    assert L.sparse_attn_select_cdf(256, 256, s, 0.9, None, 512, n, None) == 1
