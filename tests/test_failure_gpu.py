"""Failure detection without a GPU fault: the bounded device wait that every
kernel uses gives up on a barrier that nothing arrives at, reports
PSA_ERR_TIMEOUT through the status word and returns, and the context stays
usable for the next launch."""
import pytest
import torch

import shared_prefix_attention_b200 as psa

pytestmark = pytest.mark.gpu


def test_wait_completes_when_arrived():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    psa.wait_selftest(status, arrive=True)
    assert psa.read_status(status) == psa.PSA_OK


def test_wait_gives_up_and_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    psa.wait_selftest(status, arrive=False)
    end.record()
    assert psa.read_status(status) == psa.PSA_ERR_TIMEOUT
    # The wait lasted about the library's 2 s budget, not forever and not zero.
    assert 1500.0 < start.elapsed_time(end) < 20000.0
    # The context survived: a fresh status stays clean and ordinary work runs.
    status.zero_()
    psa.wait_selftest(status, arrive=True)
    assert psa.read_status(status) == psa.PSA_OK
    x = torch.arange(4, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum()) == 12.0


def test_status_keeps_first_error():
    status = torch.full((1,), psa.PSA_ERR_INVALID_ARG, dtype=torch.int32, device="cuda")
    psa.wait_selftest(status, arrive=False)
    assert psa.read_status(status) == psa.PSA_ERR_INVALID_ARG
