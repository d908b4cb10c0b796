"""CPU-side checks of the C-ABI library: it loads, exports every symbol
include/pa.h declares, and its host-side validation rejects bad arguments
before touching a GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def binding():
    from paged_kv_attention_36_b200 import build
    build.build()
    from paged_kv_attention_36_b200 import binding
    return binding


def _declared():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    return sorted(set(re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("pa_cache_append", "pa_decode", "pa_decode_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol(binding):
    declared = _declared()
    assert sorted(binding.EXPORTS) == declared
    for n in declared:
        assert hasattr(binding.lib, n), n


def test_status_strings(binding):
    for code in range(0, -8, -1):
        s = binding.pa_status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in binding.pa_status_string(-99)


def _dims(binding, **kw):
    d = dict(num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
             num_blocks=64, max_blocks_per_seq=7)
    d.update(kw)
    return binding.pa_dims(*[d[n] for n, _ in binding.pa_dims._fields_])


def _decode(binding, dims, q=16, k=16, v=16, bt=16, cl=16, out=16, ws=16, ws_bytes=1 << 30):
    vp = ctypes.c_void_p
    return binding.lib.pa_decode(vp(q), vp(k), vp(v), vp(bt), vp(cl), 0.125, vp(out),
                                 ctypes.byref(dims) if dims is not None else None, vp(ws), ws_bytes,
                                 vp(0))


def test_decode_host_validation(binding):
    # fake, never-dereferenced addresses: validation fails before any CUDA call
    assert _decode(binding, None) == -1                                   # NULL dims
    assert _decode(binding, _dims(binding, num_q_heads=6, num_kv_heads=4)) == -2
    assert _decode(binding, _dims(binding, head_dim=96)) == -3
    assert _decode(binding, _dims(binding, block_size=32)) == -3
    assert _decode(binding, _dims(binding, num_q_heads=16, num_kv_heads=1, head_dim=128)) == -3
    assert _decode(binding, _dims(binding, num_blocks=0)) == -2
    assert _decode(binding, _dims(binding), q=0) == -1
    assert _decode(binding, _dims(binding), out=8) == -4                 # misaligned
    assert _decode(binding, _dims(binding, num_seqs=0)) == 0             # nothing to do


def test_append_host_validation(binding):
    vp = ctypes.c_void_p
    d = _dims(binding)
    f = binding.lib.pa_cache_append
    assert f(vp(16), vp(16), vp(16), 3, vp(16), vp(16), None, vp(0)) == -1
    assert f(vp(16), vp(16), vp(16), -1, vp(16), vp(16), ctypes.byref(d), vp(0)) == -2
    assert f(vp(16), vp(16), vp(16), 3, vp(16), vp(16), ctypes.byref(_dims(binding, head_dim=12)),
             vp(0)) == -3
    assert f(vp(16), vp(0), vp(16), 3, vp(16), vp(16), ctypes.byref(d), vp(0)) == -1
    assert f(vp(16), vp(24), vp(16), 3, vp(16), vp(16), ctypes.byref(d), vp(0)) == -4
    assert f(vp(0), vp(0), vp(0), 0, vp(0), vp(0), ctypes.byref(d), vp(0)) == 0


def test_workspace_size_formula(binding):
    # counters (B*Hkv int32) + per-CTA two partial slots, each holding the query
    # heads of one head group (HG = 8 kv heads x G: HG*G*D floats + HG*G (m, l)
    # pairs) + per-CTA two first-level merge counters per head of the group
    d = _dims(binding, num_seqs=64, num_q_heads=32, num_kv_heads=8, head_dim=128)
    n = binding.pa_decode_workspace_bytes(d, 148)
    hG = 8 * 4
    need = 64 * 8 * 4 + 148 * 2 * hG * 128 * 4 + 148 * 2 * hG * 8 + 148 * 2 * 8 * 4
    assert need <= n <= need + 4 * 256  # + alignment and the fused path's grid barrier
    with pytest.raises(ValueError):
        binding.pa_decode_workspace_bytes(_dims(binding, num_kv_heads=3), 148)


def test_binding_rejects_host_tensors(binding):
    q = torch.zeros((1, 2, 64), dtype=torch.bfloat16)
    kc = torch.zeros((1, 1, 16, 64), dtype=torch.bfloat16)
    bt = torch.zeros((1, 1), dtype=torch.int32)
    cl = torch.ones(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.pa_decode(q, kc, kc, bt, cl, 0.125, q.clone(), workspace=torch.zeros(8, dtype=torch.uint8))
    with pytest.raises(TypeError):
        binding.pa_decode(q.float(), kc, kc, bt, cl, 0.125, q.clone())


def test_prefill_host_validation(binding):
    # fake, never-dereferenced addresses: every case is decided before any CUDA call
    vp = ctypes.c_void_p

    def call(dims, q=16, cu=16, mq=8, k=16, v=16, bt=16, cl=16, out=16):
        return binding.lib.pa_prefill(vp(q), vp(cu), mq, vp(k), vp(v), vp(bt), vp(cl), 0.125, vp(out),
                                      ctypes.byref(dims) if dims is not None else None, vp(0))
    assert call(None) == -1                                                   # NULL dims
    assert call(_dims(binding), mq=-1) == -2                                  # negative max_q_len
    assert call(_dims(binding, num_q_heads=6, num_kv_heads=4)) == -2
    assert call(_dims(binding, head_dim=96)) == -3
    assert call(_dims(binding, block_size=32)) == -3
    assert call(_dims(binding, num_q_heads=16, num_kv_heads=1)) == -3         # G = 16
    assert call(_dims(binding), mq=0) == 0                                    # nothing to do
    assert call(_dims(binding, num_seqs=0)) == 0
    assert call(_dims(binding, num_blocks=0)) == -2
    assert call(_dims(binding), cu=0) == -1
    assert call(_dims(binding), out=0) == -1
    assert call(_dims(binding), q=8) == -4                                    # misaligned
    assert call(_dims(binding), cu=2) == -4
    assert call(_dims(binding, num_blocks=1 << 27)) == -2                     # 2^32 cache rows


def test_fp8_host_validation(binding):
    vp = ctypes.c_void_p
    d = _dims(binding)
    app = binding.lib.pa_cache_append_fp8

    def a(dims, n=3, kn=16, vn=16, sm=16, kc=16, vc=16, ks=16, vs=16):
        return app(vp(kn), vp(vn), vp(sm), n, vp(kc), vp(vc), vp(ks), vp(vs),
                   ctypes.byref(dims) if dims is not None else None, vp(0))
    assert a(None) == -1
    assert a(d, n=-1) == -2
    assert a(_dims(binding, head_dim=12)) == -3
    assert a(_dims(binding, block_size=32)) == -3
    assert a(d, n=0) == 0
    assert a(d, ks=0) == -1
    assert a(d, kn=24) == -4
    assert a(d, vs=2) == -4

    dec = binding.lib.pa_decode_fp8

    def dd(dims, q=16, out=16):
        return dec(vp(q), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), 0.125, vp(out),
                   ctypes.byref(dims) if dims is not None else None, vp(16), 1 << 30, vp(0))
    assert dd(None) == -1
    assert dd(_dims(binding, num_q_heads=6, num_kv_heads=4)) == -2
    assert dd(_dims(binding, head_dim=96)) == -3
    assert dd(_dims(binding, num_seqs=0)) == 0
    assert dd(d, q=0) == -1
    assert dd(d, out=8) == -4


def test_shared_prefix_host_validation(binding):
    vp = ctypes.c_void_p
    f = binding.lib.pa_decode_shared_prefix

    def call(dims, n=0, groups=1, mgs=4, kn=16, q=16, out=16, go=16, gp=16):
        return f(vp(kn), vp(16), vp(16), n, vp(q), vp(16), vp(16), vp(16), vp(16), 0.125, vp(go), vp(gp), groups,
                 mgs, vp(out), ctypes.byref(dims) if dims is not None else None, vp(16), 1 << 30, vp(0))
    d = _dims(binding)
    assert call(None) == -1
    assert call(d, n=-1) == -2
    assert call(d, groups=-1) == -2
    assert call(d, mgs=0) == -2                                   # groups need a group size
    assert call(_dims(binding, num_q_heads=6, num_kv_heads=4)) == -2
    assert call(_dims(binding, head_dim=96)) == -3
    assert call(d, q=0) == -1
    assert call(d, out=8) == -4
    assert call(_dims(binding, num_seqs=0)) == 0                  # nothing to attend over, nothing to append


def test_binding_constants_match_the_header(binding):
    # the ctypes binding restates the header's #define values; they must agree
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    defs = dict(re.findall(r"#define\s+(PA_(?:DEVERR_\w+|STATIC_SCRATCH_BYTES))\s+(\S.*?)\s*(?:/\*|$)", src,
                           re.M))
    assert "PA_STATIC_SCRATCH_BYTES" in defs and "PA_DEVERR_TIMEOUT" in defs
    for name, val in defs.items():
        assert getattr(binding, name) == eval(val.replace("u", "")), name
