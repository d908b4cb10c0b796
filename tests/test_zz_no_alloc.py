"""Allocation-free decode: pa_decode_static_ws.

Some callers cannot allocate device memory where they decode: a host runtime
or plugin that owns every device allocation and hands out none, or a
latency-critical loop in which cudaMalloc (which may block and synchronise
the device) is not allowed.  For them the library offers pa_decode_static_ws,
which keeps its scratch in a fixed array inside the library instead of a
caller workspace.  These tests call it through the C ABI and hold every
output to the fp64 oracle (|gpu - ref| <= 1e-2 + 1e-2*|ref| per element):
on two calls in a row; and on a small problem followed by the full-size
long/skewed batch, whose merge counters then sit where the small problem
left its split-KV partials (the array keeps the previous call's contents, so
this proves each call clears what must start at zero).  They also check
that a problem too large for the array is refused before any launch.
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


def _inputs(oracle_lib, lens, Hq, Hkv, D, seed):
    """A NaN-poisoned paged batch on the GPU and the oracle's decode of it."""
    g = torch.Generator().manual_seed(seed)
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + 15) // 16 for L in lens) + 2
    (kp, vp), bt = paging.page([ks, vs], lens, 16, nb, g, poison=True)
    q = torch.randn((len(lens), Hq, D), generator=g).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32)
    scale = D ** -0.5
    ref = oracle_lib.decode(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(), cl.numpy(), scale)
    d = torch.device("cuda")
    return (q.to(d), kp.to(d), vp.to(d), bt.to(d), cl.to(d), scale), ref


def _static_decode(pa, args):
    q, kc, vc, bt, cl, scale = args
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_static_ws(q, kc, vc, bt, cl, scale, out)
    torch.cuda.synchronize()
    return out


def _assert_close(out, ref):
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any(), "NaN in output"
    err = np.abs(got - ref)
    assert (err <= ATOL + RTOL * np.abs(ref)).all(), f"max err {err.max():.3g}"


@pytest.mark.parametrize("lens,Hq,Hkv,D", [
    ([5000, 3, 700, 0, 1290, 17], 16, 4, 128),   # long context split across CTAs
    ([2048, 1, 4000, 64], 32, 4, 64),            # GQA group of 8
])
def test_static_scratch_decode_matches_oracle_on_two_calls(pa, oracle_lib, lens, Hq, Hkv, D):
    args, ref = _inputs(oracle_lib, lens, Hq, Hkv, D, seed=len(lens) + D)
    for _ in range(2):
        _assert_close(_static_decode(pa, args), ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_static_scratch_small_then_long_batch(pa, oracle_lib):
    # a small problem split over many CTAs leaves partials at the front of the
    # array; the long/skewed batch (32 q / 8 kv heads, head_dim 128, one
    # 131072-token sequence) then keeps its merge counters there
    from paged_kv_attention_36_b200 import workloads
    small, small_ref = _inputs(oracle_lib, [1000, 300, 40, 17], 8, 2, 64, seed=31)
    _assert_close(_static_decode(pa, small), small_ref)
    w = workloads.make("longskew", poison=True)
    dims = pa.make_dims(w.q, w.k_cache, w.block_tables)
    assert pa.pa_decode_workspace_bytes(dims) <= pa.PA_STATIC_SCRATCH_BYTES
    ref = oracle_lib.decode(paging.bits(w.q), paging.bits(w.k_cache), paging.bits(w.v_cache),
                            w.block_tables.numpy(), w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    args = (w.q.to(d), w.k_cache.to(d), w.v_cache.to(d), w.block_tables.to(d), w.context_lens.to(d), w.scale)
    for _ in range(2):
        _assert_close(_static_decode(pa, args), ref)
    _assert_close(_static_decode(pa, small), small_ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_static_scratch_refuses_oversize_problem(pa):
    # 600000 sequences x 8 kv heads of merge counters alone exceed the array;
    # the call must fail on the host, before touching the (fake) pointers
    dims = pa.pa_dims(600000, 32, 8, 128, 16, 1000, 8)
    vp = ctypes.c_void_p
    rc = pa.lib.pa_decode_static_ws(vp(256), vp(256), vp(256), vp(256), vp(256), 0.1, vp(256),
                                    ctypes.byref(dims), vp(0))
    assert rc == pa.PA_ERR_SCRATCH_LIMIT
    assert pa.pa_decode_workspace_bytes(dims) > pa.PA_STATIC_SCRATCH_BYTES
