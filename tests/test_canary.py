"""The canary guards of the binding's debug mode, on the CPU: a guard follows every buffer the
binding allocates and qsa_check_canaries names a buffer whose guard was written."""
import pytest
import torch

from hybrid_sparse_attention_qsa_b200 import qsa as Q


def test_release_mode_allocates_plain_tensors(monkeypatch):
    monkeypatch.setattr(Q, "DEBUG", False)
    t = Q._empty(4, 6, dtype=torch.bfloat16, device="cpu")
    assert t.shape == (4, 6) and t._base is None
    assert Q.qsa_check_canaries() == 0


def test_guard_follows_the_last_byte_and_catches_a_one_byte_overrun(monkeypatch):
    monkeypatch.setattr(Q, "DEBUG", True)
    monkeypatch.setattr(Q, "_guards", [])
    t = Q._empty((3, 5), dtype=torch.float32, device="cpu", what="probe")
    u = Q._empty_like(torch.empty(7, dtype=torch.int32), what="other")
    assert t.shape == (3, 5) and t.dtype == torch.float32 and t.is_contiguous()
    t.fill_(-1.0)                 # writing the whole buffer leaves the guard alone
    u.fill_(-1)
    assert Q.qsa_check_canaries() == 2
    raw = t._base.view(torch.uint8)
    assert raw.numel() == 60 + Q.CANARY_BYTES
    assert t.data_ptr() == raw.data_ptr()
    raw[60] = 0                   # the first byte past the end
    with pytest.raises(RuntimeError, match=r"probe \(60 bytes\)"):
        Q.qsa_check_canaries()
    raw[60] = Q.CANARY_BYTE
    u._base.view(torch.uint8)[28 + Q.CANARY_BYTES - 1] = 1   # the guard's last byte
    with pytest.raises(RuntimeError, match="other"):
        Q.qsa_check_canaries()


def test_freed_buffers_are_not_checked(monkeypatch):
    monkeypatch.setattr(Q, "DEBUG", True)
    monkeypatch.setattr(Q, "_guards", [])
    t = Q._empty(8, dtype=torch.uint8, device="cpu")
    t._base[9] = 0   # a damaged guard, but the buffer is freed before the check
    del t
    assert Q.qsa_check_canaries() == 0
