"""GPU parity of the fp8 (E4M3) KV cache against the fp64 oracle.

  * append: the E4M3 codes the library writes (k token-major, v transposed
    in the documented token order) are bit-identical to the oracle's, for
    every slot of each workload's pool (NaN-poisoned rows included) and for
    values that saturate;
  * decode: |gpu - ref| <= 1e-2 + 1e-2*|ref| per bf16 element against the
    oracle's decode of the same fp8 caches, on the five workloads' shapes
    and lengths, ragged and empty contexts, and poisoned unused slots.
"""
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


def _scales(Hkv):
    # one K and one V scale per kv head (not powers of two, so encoding rounds)
    g = np.arange(Hkv, dtype=np.float32)
    return (g + 4) / 32, (g + 3) / 24


def _pool_rows(cache):
    """[NB][Hkv][16][D] bf16 -> the pool as T = NB*16 appended rows [T][Hkv][D]."""
    NB, Hkv, bs, D = cache.shape
    return cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()


def _quantize_both(pa, oracle_lib, k_cache, v_cache, ks, vs):
    """Encode the whole pool on the GPU and in the oracle; assert identical."""
    NB, Hkv, bs, D = k_cache.shape
    kn, vn = _pool_rows(k_cache), _pool_rows(v_cache)
    slots = torch.arange(NB * bs, dtype=torch.int32)
    k8 = np.zeros((NB, Hkv, 16, D), np.uint8)
    v8 = np.zeros((NB, Hkv, D, 16), np.uint8)
    oracle_lib.append_fp8(paging.bits(kn), paging.bits(vn), slots.numpy(), k8, v8, ks, vs)
    d = torch.device("cuda")
    gk8 = torch.zeros((NB, Hkv, 16, D), dtype=torch.uint8, device=d)
    gv8 = torch.zeros((NB, Hkv, D, 16), dtype=torch.uint8, device=d)
    tks, tvs = torch.from_numpy(ks).to(d), torch.from_numpy(vs).to(d)
    pa.pa_cache_append_fp8(kn.to(d), vn.to(d), slots.to(d), gk8, gv8, tks, tvs)
    torch.cuda.synchronize()
    assert np.array_equal(gk8.cpu().numpy(), k8), "k codes differ from the oracle"
    assert np.array_equal(gv8.cpu().numpy(), v8), "v codes differ from the oracle"
    return k8, v8, gk8, gv8, tks, tvs


def _close(out, ref):
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any(), "NaN in output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance, max err {err.max():.3g}"


@pytest.mark.parametrize("name", ["tiny", "qwen3", "llama32", "longskew", "prefix"])
def test_fp8_append_and_decode_match_oracle(pa, oracle_lib, name):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make(name, poison=True)
    ks, vs = _scales(w.k_cache.shape[1])
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, w.k_cache, w.v_cache, ks, vs)
    ref = oracle_lib.decode_fp8(paging.bits(w.q), k8, v8, ks, vs, w.block_tables.numpy(),
                                w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    q = w.q.to(d)
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_fp8(q, gk8, gv8, tks, tvs, w.block_tables.to(d), w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("name", ["tiny", "qwen3", "llama32", "longskew", "prefix"])
def test_fp8_fused_append_decode_matches_oracle(pa, oracle_lib, name):
    # one launch (pa_append_decode_fp8): every CTA encodes a slice of the
    # step's new rows, then the decode reads the caches including them
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make(name, poison=True)
    ks, vs = _scales(w.k_cache.shape[1])
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, w.k_cache, w.v_cache, ks, vs)
    oracle_lib.append_fp8(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), k8, v8, ks, vs)
    ref = oracle_lib.decode_fp8(paging.bits(w.q), k8, v8, ks, vs, w.block_tables.numpy(),
                                w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    q = w.q.to(d)
    out = torch.full_like(q, float("nan"))
    pa.pa_append_decode_fp8(w.k_new.to(d), w.v_new.to(d), w.slot_mapping.to(d), q, gk8, gv8, tks, tvs,
                            w.block_tables.to(d), w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    assert np.array_equal(gk8.cpu().numpy(), k8), "k codes differ from the oracle append"
    assert np.array_equal(gv8.cpu().numpy(), v8), "v codes differ from the oracle append"
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_fp8_fused_reads_rows_written_by_other_ctas(pa, oracle_lib):
    # every new row goes to another sequence's last page (reversed slot
    # mapping), so the CTA that reads it is not the one that wrote it
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("llama32", poison=True)
    perm = torch.arange(w.q.shape[0] - 1, -1, -1)
    kn, vn, sm = w.k_new[perm].contiguous(), w.v_new[perm].contiguous(), w.slot_mapping[perm].contiguous()
    ks, vs = _scales(w.k_cache.shape[1])
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, w.k_cache, w.v_cache, ks, vs)
    oracle_lib.append_fp8(paging.bits(kn), paging.bits(vn), sm.numpy(), k8, v8, ks, vs)
    ref = oracle_lib.decode_fp8(paging.bits(w.q), k8, v8, ks, vs, w.block_tables.numpy(),
                                w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    q = w.q.to(d)
    out = torch.full_like(q, float("nan"))
    pa.pa_append_decode_fp8(kn.to(d), vn.to(d), sm.to(d), q, gk8, gv8, tks, tvs, w.block_tables.to(d),
                            w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    assert np.array_equal(gk8.cpu().numpy(), k8) and np.array_equal(gv8.cpu().numpy(), v8)
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_fp8_fused_large_batch(pa, oracle_lib):
    # 700 sequences (a tenth empty): more than a decode CTA's 288 threads, so
    # the share scan runs in chunks, and 700 new rows (the grid-barrier mode)
    from paged_kv_attention_36_b200 import workloads
    g = torch.Generator().manual_seed(77)
    lens = torch.randint(1, 201, (700,), generator=g)
    lens[torch.rand(700, generator=g) < 0.1] = 0
    w = workloads.make("qwen3", poison=True, context_lens=lens, seed=77)
    ks, vs = _scales(w.k_cache.shape[1])
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, w.k_cache, w.v_cache, ks, vs)
    oracle_lib.append_fp8(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), k8, v8, ks, vs)
    ref = oracle_lib.decode_fp8(paging.bits(w.q), k8, v8, ks, vs, w.block_tables.numpy(),
                                w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    q = w.q.to(d)
    out = torch.full_like(q, float("nan"))
    pa.pa_append_decode_fp8(w.k_new.to(d), w.v_new.to(d), w.slot_mapping.to(d), q, gk8, gv8, tks, tvs,
                            w.block_tables.to(d), w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    assert np.array_equal(gk8.cpu().numpy(), k8) and np.array_equal(gv8.cpu().numpy(), v8)
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("name", ["qwen3", "llama32"])
def test_fp8_fused_multi_token_append(pa, oracle_lib, name):
    # the last 3 positions of every sequence appended in one step: 180 tokens
    # (qwen3; each CTA writes the rows of the blocks it reads) or 384
    # (llama32; the grid barrier of a cooperative launch)
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make(name, poison=True)
    B, Hkv, D = w.q.shape[0], w.k_cache.shape[1], w.q.shape[2]
    seq = torch.arange(B).repeat(3)
    pos = w.context_lens.to(torch.int64)[seq] - 1 - torch.arange(3).repeat_interleave(B)
    sm = workloads.slots_for_positions(w.block_tables[seq], pos, 16)
    g = torch.Generator().manual_seed(62)
    kn = torch.randn((3 * B, Hkv, D), generator=g).to(torch.bfloat16)
    vn = torch.randn((3 * B, Hkv, D), generator=g).to(torch.bfloat16)
    ks, vs = _scales(Hkv)
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, w.k_cache, w.v_cache, ks, vs)
    oracle_lib.append_fp8(paging.bits(kn), paging.bits(vn), sm.numpy(), k8, v8, ks, vs)
    ref = oracle_lib.decode_fp8(paging.bits(w.q), k8, v8, ks, vs, w.block_tables.numpy(),
                                w.context_lens.numpy(), w.scale)
    d = torch.device("cuda")
    out = torch.full_like(w.q.to(d), float("nan"))
    pa.pa_append_decode_fp8(kn.to(d), vn.to(d), sm.to(d), w.q.to(d), gk8, gv8, tks, tvs, w.block_tables.to(d),
                            w.context_lens.to(d), w.scale, out)
    torch.cuda.synchronize()
    assert np.array_equal(gk8.cpu().numpy(), k8) and np.array_equal(gv8.cpu().numpy(), v8)
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 8, 2), (64, 32, 8), (128, 16, 8), (128, 8, 8), (64, 16, 2),
                                      (128, 64, 8)])
def test_fp8_ragged_shapes(pa, oracle_lib, D, Hq, Hkv):
    g = torch.Generator().manual_seed(D + Hq)
    lens = [1, 15, 16, 17, 100, 0, 257, 33]
    ks_ = paging.random_seqs(g, lens, Hkv, D)
    vs_ = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + 15) // 16 for L in lens) + 3
    (kp, vp), bt = paging.page([ks_, vs_], lens, 16, nb, g, poison=True)
    q = torch.randn((len(lens), Hq, D), generator=g).to(torch.bfloat16)
    ks, vs = _scales(Hkv)
    k8, v8, gk8, gv8, tks, tvs = _quantize_both(pa, oracle_lib, kp, vp, ks, vs)
    cl = torch.tensor(lens, dtype=torch.int32)
    ref = oracle_lib.decode_fp8(paging.bits(q), k8, v8, ks, vs, bt.numpy(), cl.numpy(), D ** -0.5)
    d = torch.device("cuda")
    out = torch.full_like(q.to(d), float("nan"))
    pa.pa_decode_fp8(q.to(d), gk8, gv8, tks, tvs, bt.to(d), cl.to(d), D ** -0.5, out)
    torch.cuda.synchronize()
    _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_fp8_append_saturates_like_the_oracle(pa, oracle_lib):
    # values far beyond 448 * scale (and tiny ones in the subnormal range)
    g = torch.Generator().manual_seed(8)
    NB, Hkv, D = 4, 2, 64
    k = (torch.randn((NB, Hkv, 16, D), generator=g) * 1000).to(torch.bfloat16)
    v = (torch.randn((NB, Hkv, 16, D), generator=g) * 1e-3).to(torch.bfloat16)
    ks = np.array([0.5, 1.0], np.float32)
    vs = np.array([1.0, 0.25], np.float32)
    k8, v8, *_ = _quantize_both(pa, oracle_lib, k, v, ks, vs)
    assert (k8 == 0x7E).any() and (k8 == 0xFE).any()  # both signs saturated
    assert ((v8 & 0x78) == 0).any()                     # subnormal codes
    assert pa.pa_device_errors(clear=True) == 0
