"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

  * append: bit-exact, including every row it must not touch;
  * decode: |gpu - ref| <= 1e-2 + 1e-2*|ref| per bf16 element (the fp32
    path with a final bf16 rounding sits ~100x inside this bound);
  * split-KV partials (test hook): |gpu - ref| <= 1e-4*(|ref| + max|ref row|)
    for o, and 1e-4 relative for m and l;
on all five workloads at full size, plus ragged, empty, one-token, full-page
and poisoned cases and forced split points.
"""
import os

import numpy as np
import pytest
import torch

from tests import paging

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-2
PART_TOL = 1e-4

# PA_DECODE_MATH=simt (set for a child process by test_kernel_variants_gpu.py)
# selects the fp32 CUDA-core policy, built for head_dim * Hq/Hkv <= 256 only.
SIMT = os.environ.get("PA_DECODE_MATH") == "simt"


def _skip_unbuilt(Hq, Hkv, D):
    if SIMT and (Hq // Hkv) * D > 256:
        pytest.skip("the fp32 CUDA-core policy is built for head_dim * Hq/Hkv <= 256")


def _skip_unbuilt_workload(name):
    from paged_kv_attention_36_b200 import workloads
    s = workloads.SPECS[name]
    _skip_unbuilt(s.num_q_heads, s.num_kv_heads, s.head_dim)


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_kv_attention_36_b200 import binding
    binding.pa_device_errors(clear=True)
    return binding


def _oracle_step(oracle, w):
    """Oracle append (on a copy of the caches) then oracle decode."""
    kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
    oracle.append(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), kb, vb)
    ref = oracle.decode(paging.bits(w.q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(),
                        w.scale)
    return kb, vb, ref


def _to_dev(w):
    d = torch.device("cuda")
    return dict(q=w.q.to(d), k_cache=w.k_cache.to(d), v_cache=w.v_cache.to(d),
                block_tables=w.block_tables.to(d), context_lens=w.context_lens.to(d),
                k_new=w.k_new.to(d), v_new=w.v_new.to(d), slot_mapping=w.slot_mapping.to(d))


def _gpu_step(pa, t, scale, workspace=None):
    pa.pa_cache_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
    out = torch.empty_like(t["q"])
    pa.pa_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"], scale,
                 out, workspace=workspace)
    torch.cuda.synchronize()
    return out


def _assert_close(out, ref):
    got = out.to(torch.float64).cpu().numpy()
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not np.isnan(got).any(), "NaN in output"
    assert not bad.any(), (f"{bad.sum()} of {bad.size} elements outside tolerance; "
                           f"max err {err.max():.3g}, worst at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    return float(err.max())


def _assert_caches_equal(t, kb, vb):
    k_ref = torch.from_numpy(kb.view(np.int16)).cuda()
    v_ref = torch.from_numpy(vb.view(np.int16)).cuda()
    assert torch.equal(t["k_cache"].view(torch.int16), k_ref), "k_cache differs from the oracle append"
    assert torch.equal(t["v_cache"].view(torch.int16), v_ref), "v_cache differs from the oracle append"


@pytest.mark.parametrize("name", ["tiny", "qwen3", "llama32", "longskew", "prefix"])
def test_append_then_decode_matches_oracle(pa, oracle_lib, name):
    from paged_kv_attention_36_b200 import workloads
    _skip_unbuilt_workload(name)
    w = workloads.make(name, poison=True)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    out = _gpu_step(pa, t, w.scale)
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_repeat_calls_reuse_workspace(pa, oracle_lib):
    # the long/skewed batch splits its 131072-token sequence over many CTAs;
    # the merge counters must return to zero for the next call, every call
    # must match the oracle, and, since split pieces are combined in a fixed
    # order whatever order they finish in, the calls agree bit for bit
    from paged_kv_attention_36_b200 import workloads
    _skip_unbuilt_workload("longskew")
    w = workloads.make("longskew", poison=True)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
    ws = pa.alloc_workspace(dims)
    outs = [_gpu_step(pa, t, w.scale, workspace=ws) for _ in range(3)]
    for out in outs:
        _assert_close(out, ref)
    n_cnt = dims.num_seqs * dims.num_kv_heads
    assert int(ws[: 4 * n_cnt].view(torch.int32).abs().sum()) == 0
    assert all(torch.equal(o.view(torch.int16), outs[0].view(torch.int16)) for o in outs[1:])


def _case(oracle_lib, pa, lens, Hq, Hkv, D, seed, poison=True, num_ctas=None):
    _skip_unbuilt(Hq, Hkv, D)
    g = torch.Generator().manual_seed(seed)
    bs = 16
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + bs - 1) // bs for L in lens) + 3
    (kp, vp), bt = paging.page([ks, vs], lens, bs, nb, g, poison=poison)
    q = torch.randn((len(lens), Hq, D), generator=g).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32)
    scale = D ** -0.5
    ref = oracle_lib.decode(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(),
                            cl.numpy(), scale)
    d = torch.device("cuda")
    tq, tk, tv, tbt, tcl = q.to(d), kp.to(d), vp.to(d), bt.to(d), cl.to(d)
    out = torch.full_like(tq, float("nan"))
    if num_ctas is None:
        pa.pa_decode(tq, tk, tv, tbt, tcl, scale, out)
    else:
        dims = pa.make_dims(tq, tk, tbt)
        ws = pa.alloc_workspace(dims, num_ctas)
        cap = 16384
        G = Hq // Hkv
        meta = torch.zeros((cap, 4), dtype=torch.int32, device=d)
        so = torch.zeros((cap, G, D), dtype=torch.float32, device=d)
        sm = torch.zeros((cap, G), dtype=torch.float32, device=d)
        sl = torch.zeros((cap, G), dtype=torch.float32, device=d)
        cnt = torch.zeros(1, dtype=torch.int32, device=d)
        pa.pa_decode_partials(tq, tk, tv, tbt, tcl, scale, out, num_ctas, ws, cap, meta, so, sm, sl, cnt)
        torch.cuda.synchronize()
        n = int(cnt.item())
        assert 0 < n <= cap
        _check_segments(oracle_lib, q, kp, vp, bt, cl, scale, lens, Hkv, G,
                        meta[:n].cpu().numpy(), so[:n].cpu().numpy(), sm[:n].cpu().numpy(),
                        sl[:n].cpu().numpy())
    torch.cuda.synchronize()
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def _check_segments(oracle_lib, q, kp, vp, bt, cl, scale, lens, Hkv, G, meta, so, sm, sl):
    # coverage: for each (b, g) the segments tile [0, L) exactly
    cover = {}
    for b, g, t0, t1 in meta.tolist():
        assert 0 <= t0 < t1 <= lens[b]
        cover.setdefault((b, g), []).append((t0, t1))
    for b, L in enumerate(lens):
        for g in range(Hkv):
            segs = sorted(cover.get((b, g), []))
            if L == 0:
                assert not segs
                continue
            assert segs[0][0] == 0 and segs[-1][1] == L
            assert all(a[1] == c[0] for a, c in zip(segs, segs[1:]))
    # values: every (segment, query head) against the oracle's partial
    rb = np.repeat(meta[:, 0], G)
    rh = (meta[:, 1][:, None] * G + np.arange(G)[None, :]).reshape(-1)
    rt0 = np.repeat(meta[:, 2], G)
    rt1 = np.repeat(meta[:, 3], G)
    o, m, l = oracle_lib.partials(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(),
                                  cl.numpy(), scale, rb, rh, rt0, rt1)
    go = so.reshape(-1, so.shape[-1]).astype(np.float64)
    row_scale = np.abs(o).max(axis=1, keepdims=True)
    assert (np.abs(go - o) <= PART_TOL * (np.abs(o) + row_scale)).all(), np.abs(go - o).max()
    np.testing.assert_allclose(sm.reshape(-1), m, rtol=PART_TOL, atol=PART_TOL)
    np.testing.assert_allclose(sl.reshape(-1), l, rtol=PART_TOL)


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 8, 2), (64, 32, 8), (64, 8, 8), (64, 16, 2),
                                      (128, 16, 8), (128, 32, 8), (128, 8, 8)])
def test_ragged_shapes(pa, oracle_lib, D, Hq, Hkv):
    lens = [1, 15, 16, 17, 100, 257, 33, 2]
    _case(oracle_lib, pa, lens, Hq, Hkv, D, seed=D + Hq + Hkv)


def test_empty_and_single_token_contexts(pa, oracle_lib):
    # context_len 0 -> zeros; context_len 1 -> exactly bf16(V_0)
    lens = [0, 1, 0, 5, 1]
    _case(oracle_lib, pa, lens, 8, 2, 64, seed=3)


def test_all_contexts_empty(pa, oracle_lib):
    _case(oracle_lib, pa, [0, 0, 0], 8, 2, 64, seed=4)


def test_context_len_one_is_exact(pa, oracle_lib):
    _skip_unbuilt(8, 2, 128)
    g = torch.Generator().manual_seed(5)
    lens = [1, 1, 1, 1]
    ks = paging.random_seqs(g, lens, 2, 128)
    vs = paging.random_seqs(g, lens, 2, 128)
    (kp, vp), bt = paging.page([ks, vs], lens, 16, 6, g)
    q = torch.randn((4, 8, 128), generator=g).to(torch.bfloat16)
    d = torch.device("cuda")
    out = torch.empty((4, 8, 128), dtype=torch.bfloat16, device=d)
    pa.pa_decode(q.to(d), kp.to(d), vp.to(d), bt.to(d), torch.tensor(lens, dtype=torch.int32, device=d),
                 0.1, out)
    torch.cuda.synchronize()
    for b in range(4):
        for h in range(8):
            assert torch.equal(out[b, h].cpu(), vs[b][h // 4, 0])


@pytest.mark.parametrize("num_ctas", [1, 3, 7, 40, 148, 600])
def test_forced_splits_partials_and_merge(pa, oracle_lib, num_ctas):
    lens = [700, 3, 0, 1024, 129, 2000, 16]
    _case(oracle_lib, pa, lens, 16, 4, 64, seed=100 + num_ctas, num_ctas=num_ctas)


@pytest.mark.parametrize("num_ctas", [5, 148])
def test_forced_splits_head_dim_128(pa, oracle_lib, num_ctas):
    lens = [1500, 1, 333, 64]
    _case(oracle_lib, pa, lens, 32, 8, 128, seed=200 + num_ctas, num_ctas=num_ctas)


@pytest.mark.parametrize("num_ctas", [17, 600, 1024])
def test_split_merge_levels(pa, oracle_lib, num_ctas):
    # one sequence cut into num_ctas pieces: 17 needs the second merge level
    # by one piece, 600 and 1024 give 38 and 64 runs of 16 (the most the
    # second level takes)
    lens = [16 * 1100, 5]
    _case(oracle_lib, pa, lens, 16, 8, 64, seed=300 + num_ctas, num_ctas=num_ctas)


def test_long_single_sequence(pa, oracle_lib):
    # one sequence spread over every CTA, with outlier keys
    lens = [65536]
    _case(oracle_lib, pa, lens, 8, 2, 128, seed=9)


def test_non_default_stream(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("tiny", poison=True)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        pa.pa_cache_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
        out = torch.empty_like(t["q"])
        pa.pa_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"], w.scale, out)
    s.synchronize()
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)


def test_device_errors_are_reported_not_faulted(pa):
    # out-of-range block ids and lengths are caught by the kernel's own checks:
    # the bad id is redirected to block 0, the length clamped, the bit set.
    d = torch.device("cuda")
    q = torch.randn((2, 8, 64), device=d).to(torch.bfloat16)
    kc = torch.randn((4, 2, 16, 64), device=d).to(torch.bfloat16)
    bt = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device=d)    # 9 >= NB
    cl = torch.tensor([20, 5], dtype=torch.int32, device=d)
    out = torch.empty_like(q)
    pa.pa_device_errors(clear=True)
    pa.pa_decode(q, kc, kc, bt, cl, 0.125, out)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_BLOCK_ID
    cl2 = torch.tensor([40, 5], dtype=torch.int32, device=d)           # > M*bs = 32
    bt2 = torch.tensor([[0, 3], [1, 2]], dtype=torch.int32, device=d)
    pa.pa_decode(q, kc, kc, bt2, cl2, 0.125, out)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_CONTEXT
    kn = torch.randn((2, 2, 64), device=d).to(torch.bfloat16)
    sm = torch.tensor([3, 4 * 16], dtype=torch.int32, device=d)        # second slot past the pool
    pa.pa_cache_append(kn, kn, sm, kc, kc)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_SLOT


def test_append_skips_padding_and_touches_nothing_else(pa, oracle_lib):
    g = torch.Generator().manual_seed(12)
    NB, Hkv, bs, D, T = 10, 4, 16, 128, 9
    kc = torch.randn((NB, Hkv, bs, D), generator=g).to(torch.bfloat16)
    vc = torch.randn((NB, Hkv, bs, D), generator=g).to(torch.bfloat16)
    kn = torch.randn((T, Hkv, D), generator=g).to(torch.bfloat16)
    vn = torch.randn((T, Hkv, D), generator=g).to(torch.bfloat16)
    slots = torch.tensor([5, -1, 159, 0, 16, -7, 77, 78, 100], dtype=torch.int32)
    kb, vb = paging.bits(kc).copy(), paging.bits(vc).copy()
    oracle_lib.append(paging.bits(kn), paging.bits(vn), slots.numpy(), kb, vb)
    d = torch.device("cuda")
    t = dict(k_cache=kc.to(d), v_cache=vc.to(d))
    pa.pa_cache_append(kn.to(d), vn.to(d), slots.to(d), t["k_cache"], t["v_cache"])
    torch.cuda.synchronize()
    _assert_caches_equal(t, kb, vb)


@pytest.mark.parametrize("name", ["tiny", "qwen3", "llama32", "longskew", "prefix"])
def test_fused_append_decode_matches_oracle(pa, oracle_lib, name):
    # one launch: every CTA appends a slice of the rows, a grid barrier, then decode
    from paged_kv_attention_36_b200 import workloads
    _skip_unbuilt_workload(name)
    w = workloads.make(name, poison=True)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    out = torch.empty_like(t["q"])
    pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                        t["block_tables"], t["context_lens"], w.scale, out)
    torch.cuda.synchronize()
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_fused_repeat_calls_reset_the_grid_barrier(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("qwen3", poison=True)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
    ws = pa.alloc_workspace(dims)
    for _ in range(4):
        out = torch.empty_like(t["q"])
        pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"],
                            t["v_cache"], t["block_tables"], t["context_lens"], w.scale, out, workspace=ws)
        torch.cuda.synchronize()
        _assert_close(out, ref)
        assert int(ws[-256:].view(torch.int32).abs().sum()) == 0  # barrier counters back to zero
    _assert_caches_equal(t, kb, vb)
    assert pa.pa_device_errors(clear=True) == 0


def test_fused_append_reads_rows_written_by_other_ctas(pa, oracle_lib):
    # slots of tokens appended to sequences whose pages other CTAs read:
    # every token goes to a different sequence's last page, in reverse order
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("llama32", poison=True)
    perm = torch.arange(w.q.shape[0] - 1, -1, -1)
    w.k_new, w.v_new = w.k_new[perm].contiguous(), w.v_new[perm].contiguous()
    w.slot_mapping = w.slot_mapping[perm].contiguous()
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    out = torch.empty_like(t["q"])
    pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                        t["block_tables"], t["context_lens"], w.scale, out)
    torch.cuda.synchronize()
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)


def _multi_token_step(w, per_seq, seed):
    """The last per_seq positions of every sequence appended this step, in
    position-major order, with fresh rows: T = per_seq * B tokens."""
    from paged_kv_attention_36_b200 import workloads
    B, Hkv, D = w.q.shape[0], w.k_cache.shape[1], w.q.shape[2]
    seq = torch.arange(B).repeat(per_seq)
    pos = w.context_lens.to(torch.int64)[seq] - 1 - torch.arange(per_seq).repeat_interleave(B)
    slots = workloads.slots_for_positions(w.block_tables[seq], pos, 16)
    g = torch.Generator().manual_seed(seed)
    w.k_new = torch.randn((per_seq * B, Hkv, D), generator=g).to(torch.bfloat16)
    w.v_new = torch.randn((per_seq * B, Hkv, D), generator=g).to(torch.bfloat16)
    w.slot_mapping = slots
    return w


@pytest.mark.parametrize("name,per_seq", [("qwen3", 3), ("llama32", 3)])
def test_fused_multi_token_append(pa, oracle_lib, name, per_seq):
    # several new tokens per sequence: qwen3 gives 180 (at most 256: every CTA
    # writes the rows of the blocks it reads itself), llama32 384 (the grid
    # barrier of a cooperative launch)
    from paged_kv_attention_36_b200 import workloads
    _skip_unbuilt_workload(name)
    w = _multi_token_step(workloads.make(name, poison=True), per_seq, seed=61)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    out = torch.full_like(t["q"], float("nan"))
    pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                        t["block_tables"], t["context_lens"], w.scale, out)
    torch.cuda.synchronize()
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def _large_batch(name, B, hi, seed):
    """B sequences of U[1, hi] tokens, a tenth of them empty."""
    from paged_kv_attention_36_b200 import workloads
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(1, hi + 1, (B,), generator=g)
    lens[torch.rand(B, generator=g) < 0.1] = 0
    return workloads.make(name, poison=True, context_lens=lens, seed=seed)


@pytest.mark.parametrize("name,B,hi", [("tiny", 1000, 120), ("qwen3", 600, 300)])
def test_large_batch_scans_in_chunks(pa, oracle_lib, name, B, hi):
    # more sequences than a decode CTA has threads (288): the scan of the
    # work line and the search for each CTA's first sequence run over
    # several chunks; fused, the B new rows take the grid-barrier mode
    _skip_unbuilt_workload(name)
    w = _large_batch(name, B, hi, seed=B + hi)
    kb, vb, ref = _oracle_step(oracle_lib, w)
    t = _to_dev(w)
    _assert_close(_gpu_step(pa, t, w.scale), ref)
    _assert_caches_equal(t, kb, vb)
    t = _to_dev(w)
    out = torch.full_like(t["q"], float("nan"))
    pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                        t["block_tables"], t["context_lens"], w.scale, out)
    torch.cuda.synchronize()
    _assert_caches_equal(t, kb, vb)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_fused_reports_bad_slot(pa):
    d = torch.device("cuda")
    q = torch.randn((2, 8, 64), device=d).to(torch.bfloat16)
    kc = torch.randn((4, 2, 16, 64), device=d).to(torch.bfloat16)
    bt = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device=d)
    cl = torch.tensor([20, 5], dtype=torch.int32, device=d)
    kn = torch.randn((2, 2, 64), device=d).to(torch.bfloat16)
    sm = torch.tensor([3, 4 * 16 + 1], dtype=torch.int32, device=d)   # second slot past the pool
    out = torch.empty_like(q)
    pa.pa_device_errors(clear=True)
    pa.pa_append_decode(kn, kn, sm, q, kc, kc.clone(), bt, cl, 0.125, out)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_SLOT
