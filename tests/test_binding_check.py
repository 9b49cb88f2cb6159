"""The binding's opt-in status check, without a GPU: with check=True a call reads
the device status word right after launching (bsa_last_device_status) and raises
BsaError on a recorded timeout; without it the call only launches.  The C library
is replaced by a fake that records the calls and returns the statuses a timed-out
kernel would leave."""
import pytest
import torch

import block_sparse_attention_14_b200 as bsa


class FakeLib:
    def __init__(self, device_status):
        self.device_status = device_status
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append(name)
            if name == "bsa_last_device_status":
                return self.device_status
            if name == "sparse_attn_topk_noalloc_status":
                return self.device_status
            if name == "bsa_last_error_message":
                return b"a bounded wait ran out (site 6, CTA 0)"
            return 0
        return f


@pytest.fixture
def fake(monkeypatch):
    def install(device_status):
        lib = FakeLib(device_status)
        monkeypatch.setattr(bsa, "lib", lambda: lib)
        monkeypatch.setattr(bsa, "_qkv", lambda *ts: None)
        monkeypatch.setattr(bsa, "_stream", lambda t: 0)
        return lib
    return install


def _args():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    ws = torch.zeros(1024, dtype=torch.uint8)
    return q, ws


@pytest.mark.parametrize("call", ["topk", "fwd", "cdf", "apply"])
def test_check_raises_on_a_recorded_timeout(fake, call):
    lib = fake(4)
    q, ws = _args()
    run = {
        "topk": lambda c: bsa.sparse_attn_topk(q, q, q, 0.5, workspace=ws, check=c),
        "fwd": lambda c: bsa.block_sparse_attn_fwd(q, q, q, None, workspace=ws, check=c),
        "cdf": lambda c: bsa.sparse_attn_cdf(q, q, q, 0.9, workspace=ws, check=c),
        "apply": lambda c: bsa.block_sparse_attn_apply(q, q, q, ws, check=c),
    }[call]
    run(False)  # launches only: no status read, no error
    assert "bsa_last_device_status" not in lib.calls
    with pytest.raises(bsa.BsaError) as e:
        run(True)
    assert e.value.status == 4 and "bounded wait" in str(e.value)
    assert lib.calls[-2] == "bsa_last_device_status"


def test_check_passes_when_the_status_is_clean(fake):
    lib = fake(0)
    q, ws = _args()
    bsa.sparse_attn_topk(q, q, q, 0.5, workspace=ws, check=True)
    assert lib.calls[-1] == "bsa_last_device_status"
