"""The library's failure paths, exercised without faulting, trapping or hanging the GPU.

  * Bounded waits: with the wait limit shortened to 1 ms, a kernel that waits on a shared-memory barrier
    no thread arrives on, or on a device word nothing writes, must give up, return, and leave
    QLORA_STATUS_TIMEOUT in the status word (qlora_get_status -> QLORA_ERR_TIMEOUT); the context stays
    usable and the next codec call matches the oracle bit for bit.
  * Host-side fault injection (QLORA_FAULT_INJECT): the chosen call fails as a launch failure would,
    enqueues nothing, and the calls before and after it give the normal results.
"""
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_wait(lib):
    lib.set_wait_limit(1_000_000)            # 1 ms
    yield
    lib.set_wait_limit(0)                    # back to the default


@pytest.mark.parametrize("kind", ["mbarrier", "device_word"])
def test_bounded_wait_gives_up_and_reports_timeout(lib, short_wait, kind):
    assert lib.get_status() == 0
    k = lib.SELFTEST_MBARRIER if kind == "mbarrier" else lib.SELFTEST_DEVICE_WORD
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    lib.selftest_wait(k)
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    assert 0.9 <= ms < 1000.0, ms             # waited about the limit, then returned
    assert lib.get_status() & lib.STATUS_TIMEOUT
    assert lib.get_status() == 0             # reading clears the bit
    x = synth.sweep_f32(64 * 1000 + 5, seed=3, tensor_id=71)
    q = lib.quantize(torch.from_numpy(x).cuda())
    assert lib.get_status() == 0
    assert np.array_equal(q.codes.cpu().numpy(), O.quantize(x).codes)


def test_selftest_rejects_an_unknown_kind(lib):
    with pytest.raises(lib.QLoRAError) as e:
        lib.selftest_wait(7)
    assert e.value.code == -1
    with pytest.raises(lib.QLoRAError) as e:
        lib.set_wait_limit(10)                # below 1 us
    assert e.value.code == -1


def test_injected_launch_failure(lib, monkeypatch):
    case = synth.linear_case(T=5, N=256, K=192, r=8, alpha=16.0, seed=9)
    q = lib.quantize(torch.from_numpy(case["W"]).cuda())
    d = {k: case[k].cuda() for k in ("X", "A", "B")}
    n0 = lib.kernel_launches()
    monkeypatch.setenv("QLORA_FAULT_INJECT", "qlora_linear_fwd:2")
    Y1, U1 = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    n1 = lib.kernel_launches()
    assert n1 > n0
    with pytest.raises(lib.QLoRAError) as e:
        lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    assert e.value.code == -5
    assert lib.kernel_launches() == n1       # nothing was enqueued by the failed call
    Y3, U3 = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    monkeypatch.delenv("QLORA_FAULT_INJECT")
    assert lib.get_status() == 0
    assert torch.equal(Y1, Y3) and torch.equal(U1, U3)
