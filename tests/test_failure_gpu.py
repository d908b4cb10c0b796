"""Failure detection on the GPU without a GPU fault: every wait in the
kernels is bounded in time; when one runs out the kernel sets
PA_DEVERR_TIMEOUT in the device error word and returns, and the context
stays usable.  The test hook pa_test_wait_timeout makes both kinds of wait
(the decode pipeline's polling wait and the prefill pipeline's sleeping
wait) run out on an mbarrier that nothing arrives on, with a short limit;
the test reads the status through the C ABI and then runs a decode on the
same device, checked against the fp64 oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import paging

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_kv_attention_36_b200 import binding
    binding.pa_device_errors(clear=True)
    return binding


def test_bounded_waits_time_out_report_and_leave_the_device_usable(pa, oracle_lib):
    limit_ns = 20_000_000  # 20 ms per wait
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    pa.pa_test_wait_timeout(limit_ns)
    end.record()
    errs = pa.pa_device_errors(clear=True)
    assert errs == pa.PA_DEVERR_TIMEOUT
    # both waits ran for (at least) their limit before giving up
    assert start.elapsed_time(end) >= 2 * limit_ns * 1e-6 * 0.95
    assert pa.pa_device_errors(clear=True) == 0

    # the device and the library work as before
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("tiny", poison=True)
    kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
    oracle_lib.append(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), kb, vb)
    ref = oracle_lib.decode(paging.bits(w.q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    q, kc, vc = w.q.to(d), w.k_cache.to(d), w.v_cache.to(d)
    out = torch.full_like(q, float("nan"))
    pa.pa_append_decode(w.k_new.to(d), w.v_new.to(d), w.slot_mapping.to(d), q, kc, vc, w.block_tables.to(d),
                        w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any()
    assert (np.abs(got - ref) <= 1e-2 + 1e-2 * np.abs(ref)).all()
    assert pa.pa_device_errors(clear=True) == 0


def test_wait_limit_is_validated_on_the_host(pa):
    vp = ctypes.c_void_p
    assert pa.lib.pa_test_wait_timeout(999, vp(0)) == -2
    assert pa.lib.pa_test_wait_timeout(2_000_000_000, vp(0)) == -2
