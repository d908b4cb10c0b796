"""Allocation-free decode: pa_decode_static_ws.

Some callers cannot allocate device memory where they decode: a host runtime
or plugin that owns every device allocation and hands out none, or a
latency-critical loop in which cudaMalloc (which may block and synchronise
the device) is not allowed.  For them the library offers pa_decode_static_ws,
which keeps its scratch in a fixed array inside the library instead of a
caller workspace.  These tests call it through the C ABI and check that it
gives what pa_decode gives, on two calls in a row (the array keeps the
previous call's contents, so the second call proves the counters it needs
are cleared), and that an oversize problem is refused before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import paging

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-2


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_kv_attention_36_b200 import binding
    binding.pa_device_errors(clear=True)
    return binding


def _inputs(lens, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + 15) // 16 for L in lens) + 2
    (kp, vp), bt = paging.page([ks, vs], lens, 16, nb, g, poison=True)
    q = torch.randn((len(lens), Hq, D), generator=g).to(torch.bfloat16)
    d = torch.device("cuda")
    return (q.to(d), kp.to(d), vp.to(d), bt.to(d), torch.tensor(lens, dtype=torch.int32, device=d),
            D ** -0.5)


@pytest.mark.parametrize("lens,Hq,Hkv,D", [
    ([5000, 3, 700, 0, 1290, 17], 16, 4, 128),   # long context split across CTAs
    ([2048, 1, 4000, 64], 32, 4, 64),            # GQA group of 8
])
def test_static_scratch_decode_matches_pa_decode_on_two_calls(pa, lens, Hq, Hkv, D):
    q, kc, vc, bt, cl, scale = _inputs(lens, Hq, Hkv, D, seed=len(lens) + D)
    ref = torch.empty_like(q)
    pa.pa_decode(q, kc, vc, bt, cl, scale, ref)
    torch.cuda.synchronize()
    want = ref.to(torch.float64).cpu().numpy()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_static_ws(q, kc, vc, bt, cl, scale, out)
        torch.cuda.synchronize()
        got = out.to(torch.float64).cpu().numpy()
        assert not np.isnan(got).any()
        assert (np.abs(got - want) <= ATOL + RTOL * np.abs(want)).all()
    assert pa.pa_device_errors(clear=True) == 0


def test_static_scratch_refuses_oversize_problem(pa):
    # 300000 sequences x 8 kv heads of merge counters alone exceed the array;
    # the call must fail on the host, before touching the (fake) pointers
    dims = pa.pa_dims(300000, 32, 8, 128, 16, 1000, 8)
    vp = ctypes.c_void_p
    rc = pa.lib.pa_decode_static_ws(vp(256), vp(256), vp(256), vp(256), vp(256), 0.1, vp(256),
                                    ctypes.byref(dims), vp(0))
    assert rc == pa.PA_ERR_SCRATCH_LIMIT
    assert pa.pa_decode_workspace_bytes(dims) > pa.PA_STATIC_SCRATCH_BYTES
