"""GPU parity of the multi-query (chunked prefill) attention over the paged
cache, through the C ABI, against the fp64 oracle: |gpu - ref| <= 1e-2 +
1e-2*|ref| per bf16 element.  Ragged chunks (1, 7, 16, 17, 200 and whole-
context query counts), every built head shape, poisoned unused rows,
sequences without queries, a loose max_q_len, many row tiles and pages, and
a chunk longer than its context (reported, not faulted).
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


def _case(pa, oracle_lib, lens, q_lens, Hq, Hkv, D, seed, max_q_len=None):
    g = torch.Generator().manual_seed(seed)
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + 15) // 16 for L in lens) + 3
    (kp, vp), bt = paging.page([ks, vs], lens, 16, nb, g, poison=True)
    q = torch.randn((sum(q_lens), Hq, D), generator=g).to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]), dtype=torch.int32)
    cl = torch.tensor(lens, dtype=torch.int32)
    scale = D ** -0.5
    ref = oracle_lib.prefill(paging.bits(q), cu.numpy(), paging.bits(kp), paging.bits(vp), bt.numpy(),
                             cl.numpy(), scale)
    d = torch.device("cuda")
    out = torch.full((q.shape[0], Hq, D), float("nan"), dtype=torch.bfloat16, device=d)
    pa.pa_prefill(q.to(d), cu.to(d), max(q_lens) if max_q_len is None else max_q_len, kp.to(d), vp.to(d),
                  bt.to(d), cl.to(d), scale, out)
    torch.cuda.synchronize()
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any(), "NaN in output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance, max err {err.max():.3g}"
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 8, 2), (64, 32, 8), (64, 8, 8), (64, 16, 2),
                                      (128, 16, 8), (128, 32, 8), (128, 8, 8), (128, 64, 8)])
def test_ragged_chunks(pa, oracle_lib, D, Hq, Hkv):
    lens = [40, 7, 300, 17, 64, 129, 1]
    q_lens = [13, 7, 200, 17, 1, 16, 1]   # 7 and 17: whole contexts
    _case(pa, oracle_lib, lens, q_lens, Hq, Hkv, D, seed=D + Hq)


def test_long_context_chunk_many_tiles(pa, oracle_lib):
    # 512 queries x 4 heads per kv head = 16 row tiles, 2000-token context (125 pages)
    _case(pa, oracle_lib, [2000, 600], [512, 100], 32, 8, 128, seed=7)


def test_single_query_chunks_and_sequences_without_queries(pa, oracle_lib):
    _case(pa, oracle_lib, [100, 33, 5, 16, 48], [1, 0, 1, 0, 1], 8, 2, 64, seed=8, max_q_len=40)


def test_whole_context_prefill(pa, oracle_lib):
    _case(pa, oracle_lib, [333], [333], 16, 8, 64, seed=9)


def test_chunk_longer_than_context_is_reported(pa):
    d = torch.device("cuda")
    NB, Hkv, D = 4, 2, 64
    kc = torch.zeros((NB, Hkv, 16, D), dtype=torch.bfloat16, device=d)
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device=d)
    cl = torch.tensor([10], dtype=torch.int32, device=d)
    cu = torch.tensor([0, 12], dtype=torch.int32, device=d)   # 12 queries, 10 tokens
    q = torch.zeros((12, 8, D), dtype=torch.bfloat16, device=d)
    out = torch.empty_like(q)
    pa.pa_prefill(q, cu, 12, kc, kc, bt, cl, 0.125, out)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_CONTEXT


@pytest.mark.parametrize("name", ["llama32", "qwen3"])
def test_bench_batch_sampled_rows(pa, oracle_lib, name):
    """The benchmark's own batch and launch (16 sequences, 512-token chunks
    after prior contexts U[512,3584]) on the GPU; per sequence its first and
    last query token and six seeded random ones are checked against the
    oracle.  Query token i of sequence b is, by definition, the decode of
    its q row over the first first_pos + i + 1 cached tokens (the oracle's
    prefill equals its decode bit for bit there), so the pinned decode oracle
    gives each sampled row without the whole O(chunk x context) reference."""
    from paged_kv_attention_36_b200 import workloads
    pb = workloads.make_prefill(name)
    d = torch.device("cuda")
    out = torch.full(pb.q.shape, float("nan"), dtype=torch.bfloat16, device=d)
    pa.pa_prefill(pb.q.to(d), pb.cu_q_lens.to(d), pb.max_q_len, pb.k_cache.to(d), pb.v_cache.to(d),
                  pb.block_tables.to(d), pb.context_lens.to(d), pb.scale, out)
    torch.cuda.synchronize()
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any(), "NaN in output"
    rng = np.random.default_rng(36)
    cu, cl = pb.cu_q_lens.numpy(), pb.context_lens.numpy()
    rows, lens, seqs = [], [], []
    for b in range(len(cl)):
        ql = int(cu[b + 1] - cu[b])
        first_pos = int(cl[b]) - ql
        for i in sorted({0, ql - 1, *rng.integers(0, ql, 6).tolist()}):
            rows.append(int(cu[b]) + i)
            lens.append(first_pos + i + 1)
            seqs.append(b)
    ref = oracle_lib.decode(paging.bits(pb.q[rows]), paging.bits(pb.k_cache), paging.bits(pb.v_cache),
                            pb.block_tables[seqs].numpy(), np.array(lens, dtype=np.int32), pb.scale)
    err = np.abs(got[rows] - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance, max err {err.max():.3g}"
    assert pa.pa_device_errors(clear=True) == 0
