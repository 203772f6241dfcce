"""Bounded device waits: the timeout path is observable from the host.

A wait that nothing completes (a self-test kernel, bounded at 1 ms) must
raise the library's timeout count, which bnb4_device_status reports once and
then clears; ordinary calls leave it clear.  No GPU fault, trap or hang is
involved: the waiting kernel returns on its own.
"""
import pytest

torch = pytest.importorskip("torch")

import bit_blockwise_weight_b200 as bnb4

pytestmark = pytest.mark.gpu

TIMEOUT = 8  # BNB4_ERR_TIMEOUT


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_clear_after_normal_calls():
    w = torch.randn(256 * 512, device="cuda") * 0.02
    p, a = bnb4.quantize_4bit(w, 64, "nf4")
    X = torch.randn(300, 512, device="cuda", dtype=torch.bfloat16)
    bnb4.gemm_4bit(X, p, a, 256)                       # tcgen05 kernel
    bnb4.gemm_4bit(X[:8].contiguous(), p, a, 256)      # small-M kernel
    assert bnb4.device_status() == bnb4.STATUS_OK


def test_timed_out_wait_is_reported_once():
    assert bnb4.device_status() == bnb4.STATUS_OK
    assert bnb4.bnb4_selftest_wait_timeout(_stream()) == bnb4.STATUS_OK
    assert bnb4.device_status() == TIMEOUT
    assert bnb4.device_status() == bnb4.STATUS_OK  # cleared by the read
    # the context is still usable
    x = torch.randn(4096, device="cuda", dtype=torch.bfloat16)
    p, a = bnb4.quantize_4bit(x, 64, "nf4")
    torch.cuda.synchronize()
    assert p.numel() == 2048 and a.numel() == 64


INDEX = 10  # BNB4_ERR_INDEX


def test_two_kinds_are_reported_one_after_the_other():
    """A timed-out wait and a bad embedding index raised before one status
    call: the more severe (timeout) is reported and cleared first, the index
    report is kept for the next call, then all is clear."""
    assert bnb4.device_status() == bnb4.STATUS_OK
    w = torch.randn(64 * 128, device="cuda") * 0.02
    p, a = bnb4.quantize_4bit(w, 64, "nf4")
    idx = torch.tensor([0, 64, 3], dtype=torch.int64, device="cuda")   # 64 is out of range
    bnb4.embedding_4bit(p, a, 64, 128, idx, 64, "nf4")
    assert bnb4.bnb4_selftest_wait_timeout(_stream()) == bnb4.STATUS_OK
    assert bnb4.device_status() == TIMEOUT
    assert bnb4.device_status() == INDEX
    assert bnb4.device_status() == bnb4.STATUS_OK
