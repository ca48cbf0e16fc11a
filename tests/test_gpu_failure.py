"""Failure detection without a GPU fault: every device-side wait of the
kernels is bounded by a wall-clock limit and reports LBCA_ERR_TIMEOUT through
the status word.  Here a wait runs out on purpose (an mbarrier that nothing
arrives at, the kernels' own wait helper, a 20 ms limit): the status says so,
the kernel returns, and the context keeps working (a decode call after it
still matches the oracle)."""
import time

import pytest
import torch

from block_compressed_long_b200 import synth
from lbca_cases import DecodeRun, assert_close, f64, lib, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib()


def test_wait_that_runs_out_reports_timeout_and_the_context_survives(L):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    L.lbca_selftest_bounded_wait(False, 20_000_000, st)
    torch.cuda.synchronize()
    assert int(st.item()) == L.LBCA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    ok = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lbca_selftest_bounded_wait(True, 20_000_000, ok)  # the control: the barrier completes
    torch.cuda.synchronize()
    assert int(ok.item()) == 0
    # the context is intact: a decode step still runs and matches the oracle
    w = synth.scaled(synth.WORKLOADS["gqa_decode_32k"], ctx=(500, 500), steps=1)
    inp = synth.make(w)
    run = DecodeRun(L, w, inp, steps=1)
    got = run.step()
    torch.cuda.synchronize()
    assert_close(f64(got), oracle_decode(w, inp, 0), "bf16", "decode after a timed-out wait")
    assert int(run.status.item()) == 0


def test_selftest_rejects_bad_arguments(L):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(L.LbcaError):
        L.lbca_selftest_bounded_wait(False, 0, st)
    with pytest.raises(L.LbcaError):
        L.lbca_selftest_bounded_wait(False, 10 ** 10, st)
