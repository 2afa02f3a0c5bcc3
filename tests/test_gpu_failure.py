"""Failure reporting on the GPU without a GPU fault: a bounded device-side wait
on a barrier phase that nothing completes must end, write CCA_DEV_TIMEOUT to
the status word, and leave the context usable (the next kernel runs normally)."""

import pytest
import torch

import chunk_causal_attention_b200 as cca

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda:0")
    cca.cca_selftest_bounded_wait(st, budget_cycles=2_000_000)  # about 1 ms
    torch.cuda.synchronize()
    assert int(st.item()) == cca.CCA_DEV_TIMEOUT
    # positive control: the same wait succeeds when the phase completes
    cca.cca_selftest_bounded_wait(st, budget_cycles=2_000_000, arrive_first=True)
    torch.cuda.synchronize()
    assert int(st.item()) == cca.CCA_DEV_OK
    # the context is still usable
    x = torch.arange(16, device="cuda:0", dtype=torch.float32)
    assert float(x.sum().item()) == 120.0


def test_bounded_wait_rejects_bad_budget():
    st = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    with pytest.raises(cca.CcaError):
        cca.cca_selftest_bounded_wait(st, budget_cycles=0)
