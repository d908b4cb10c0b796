"""CUDA-graph capture of the decode step (the pages' engines replay a
captured decode to cut launch latency: miniVLLM docs index, "What is
miniVLLM?": CUDA graph optimization for low-latency decode).

Every C-ABI call is asynchronous, allocates nothing and never synchronises,
so a whole step can be captured on a torch stream and replayed.  These
tests capture (1) the fused append + decode (a cooperative launch with a
grid barrier in the workspace), (2) the shared-prefix step (the prefix pass
and the decode launched as its programmatic dependent), (3) the two-call
step (append, then decode), (4) the fused fp8 append + decode and (5) the
multi-query prefill; they replay
each several times with new inputs written into the captured buffers and
compare every replay with the fp64 oracle.  Replays reuse the workspace,
so they also prove that every call leaves its counters and barrier at zero.
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


def _close(out, ref):
    got = out.to(torch.float64).cpu().numpy()
    assert not np.isnan(got).any()
    assert (np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)).all(), float(np.abs(got - ref).max())


def _oracle(oracle, w, q, k_new, v_new):
    kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
    oracle.append(paging.bits(k_new), paging.bits(v_new), w.slot_mapping.numpy(), kb, vb)
    return oracle.decode(paging.bits(q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(), w.scale)


def _run(pa, oracle_lib, w, step, replays=3):
    """Capture `step(t, out)` once, then replay it with fresh q / new rows."""
    d = torch.device("cuda")
    t = {k: getattr(w, k).to(d) for k in ("q", "k_cache", "v_cache", "block_tables", "context_lens", "k_new",
                                          "v_new", "slot_mapping")}
    if w.num_groups:
        t["group_offsets"], t["group_prefix_pages"] = w.group_offsets.to(d), w.group_prefix_pages.to(d)
    out = torch.empty_like(t["q"])
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step(t, out)  # warm-up outside capture (first-call attribute set-up)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step(t, out)
    gen = torch.Generator().manual_seed(77)
    for _ in range(replays):
        q = torch.randn(w.q.shape, generator=gen).to(torch.bfloat16)
        kn = torch.randn(w.k_new.shape, generator=gen).to(torch.bfloat16)
        vn = torch.randn(w.v_new.shape, generator=gen).to(torch.bfloat16)
        t["q"].copy_(q)
        t["k_new"].copy_(kn)
        t["v_new"].copy_(vn)
        g.replay()
        torch.cuda.synchronize()
        _close(out, _oracle(oracle_lib, w, q, kn, vn))
    assert pa.pa_device_errors(clear=True) == 0


def test_graph_fused_append_decode(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("qwen3", poison=True)

    def step(t, out):
        dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
        if not hasattr(step, "ws"):
            step.ws = pa.alloc_workspace(dims)
        pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                            t["block_tables"], t["context_lens"], w.scale, out, workspace=step.ws)
    _run(pa, oracle_lib, w, step)


def test_graph_fused_append_decode_barrier_mode(pa, oracle_lib):
    # more than 256 new rows (the last 3 positions of each of 128 sequences):
    # the fused step's CTAs meet at a grid barrier, a cooperative launch,
    # captured and replayed; every replay must leave the barrier at zero
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("llama32", poison=True)
    B = w.q.shape[0]
    seq = torch.arange(B).repeat(3)
    pos = w.context_lens.to(torch.int64)[seq] - 1 - torch.arange(3).repeat_interleave(B)
    w.slot_mapping = workloads.slots_for_positions(w.block_tables[seq], pos, 16)
    g0 = torch.Generator().manual_seed(79)
    w.k_new = torch.randn((3 * B,) + tuple(w.k_new.shape[1:]), generator=g0).to(torch.bfloat16)
    w.v_new = torch.randn((3 * B,) + tuple(w.v_new.shape[1:]), generator=g0).to(torch.bfloat16)

    def step(t, out):
        dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
        if not hasattr(step, "ws"):
            step.ws = pa.alloc_workspace(dims)
        pa.pa_append_decode(t["k_new"], t["v_new"], t["slot_mapping"], t["q"], t["k_cache"], t["v_cache"],
                            t["block_tables"], t["context_lens"], w.scale, out, workspace=step.ws)
    _run(pa, oracle_lib, w, step, replays=2)
    assert int(step.ws[-256:].view(torch.int32).abs().sum()) == 0


def test_graph_two_call_step(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("longskew", poison=True)

    def step(t, out):
        dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
        if not hasattr(step, "ws"):
            step.ws = pa.alloc_workspace(dims)
        pa.pa_cache_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
        pa.pa_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"], w.scale, out,
                     workspace=step.ws)
    _run(pa, oracle_lib, w, step, replays=2)


def test_graph_shared_prefix_step(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("prefix", poison=True)

    def step(t, out):
        dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
        if not hasattr(step, "ws"):
            step.ws = torch.zeros(pa.pa_decode_shared_prefix_workspace_bytes(dims, w.num_groups, w.max_group_size),
                                  dtype=torch.uint8, device="cuda")
        pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                                   w.scale, t["group_offsets"], t["group_prefix_pages"], w.max_group_size, out,
                                   k_new=t["k_new"], v_new=t["v_new"], slot_mapping=t["slot_mapping"],
                                   workspace=step.ws)
    _run(pa, oracle_lib, w, step)


def test_graph_fused_fp8_step(pa, oracle_lib):
    """The fused fp8 step (pa_append_decode_fp8) captured once and replayed
    with new q and new rows; each replay against the oracle's fp8 append and
    decode of the same rows."""
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("llama32", poison=True)
    NB, Hkv, bs, D = w.k_cache.shape
    gsc = np.arange(Hkv, dtype=np.float32)
    ks, vs = (gsc + 4) / 32, (gsc + 3) / 24
    rows_k = w.k_cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
    rows_v = w.v_cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
    slots = torch.arange(NB * bs, dtype=torch.int32)
    k8 = np.zeros((NB, Hkv, 16, D), np.uint8)
    v8 = np.zeros((NB, Hkv, D, 16), np.uint8)
    oracle_lib.append_fp8(paging.bits(rows_k), paging.bits(rows_v), slots.numpy(), k8, v8, ks, vs)
    d = torch.device("cuda")
    t = {"q": w.q.to(d), "kn": w.k_new.to(d), "vn": w.v_new.to(d), "sm": w.slot_mapping.to(d),
         "k8": torch.from_numpy(k8).to(d), "v8": torch.from_numpy(v8).to(d), "ks": torch.from_numpy(ks).to(d),
         "vs": torch.from_numpy(vs).to(d), "bt": w.block_tables.to(d), "cl": w.context_lens.to(d)}
    out = torch.empty_like(t["q"])
    dims = pa.pa_dims(w.q.shape[0], w.q.shape[1], Hkv, D, 16, NB, w.block_tables.shape[1])
    ws = pa.alloc_workspace(dims)

    def step():
        pa.pa_append_decode_fp8(t["kn"], t["vn"], t["sm"], t["q"], t["k8"], t["v8"], t["ks"], t["vs"], t["bt"],
                                t["cl"], w.scale, out, workspace=ws)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step()  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    gen = torch.Generator().manual_seed(78)
    for _ in range(3):
        q = torch.randn(w.q.shape, generator=gen).to(torch.bfloat16)
        kn = torch.randn(w.k_new.shape, generator=gen).to(torch.bfloat16)
        vn = torch.randn(w.v_new.shape, generator=gen).to(torch.bfloat16)
        t["q"].copy_(q)
        t["kn"].copy_(kn)
        t["vn"].copy_(vn)
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        rk, rv = k8.copy(), v8.copy()
        oracle_lib.append_fp8(paging.bits(kn), paging.bits(vn), w.slot_mapping.numpy(), rk, rv, ks, vs)
        assert np.array_equal(t["k8"].cpu().numpy(), rk) and np.array_equal(t["v8"].cpu().numpy(), rv)
        ref = oracle_lib.decode_fp8(paging.bits(q), rk, rv, ks, vs, w.block_tables.numpy(), w.context_lens.numpy(),
                                    w.scale)
        _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_graph_prefill(pa, oracle_lib):
    """The multi-query prefill (tcgen05 kernel) captured once and replayed
    with new query rows; each replay against the oracle's prefill."""
    g0 = torch.Generator().manual_seed(88)
    lens, q_lens, Hq, Hkv, D = [300, 47, 1000, 16], [64, 47, 200, 1], 16, 8, 128
    ks = paging.random_seqs(g0, lens, Hkv, D)
    vs = paging.random_seqs(g0, lens, Hkv, D)
    nb = sum((L + 15) // 16 for L in lens) + 3
    (kp, vp), bt = paging.page([ks, vs], lens, 16, nb, g0, poison=True)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]), dtype=torch.int32)
    cl = torch.tensor(lens, dtype=torch.int32)
    d = torch.device("cuda")
    t = {"q": torch.zeros((sum(q_lens), Hq, D), dtype=torch.bfloat16, device=d), "cu": cu.to(d), "k": kp.to(d),
         "v": vp.to(d), "bt": bt.to(d), "cl": cl.to(d)}
    out = torch.empty_like(t["q"])
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())

    def step():
        pa.pa_prefill(t["q"], t["cu"], max(q_lens), t["k"], t["v"], t["bt"], t["cl"], D ** -0.5, out)
    with torch.cuda.stream(stream):
        step()  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(3):
        q = torch.randn(t["q"].shape, generator=g0).to(torch.bfloat16)
        t["q"].copy_(q)
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        ref = oracle_lib.prefill(paging.bits(q), cu.numpy(), paging.bits(kp), paging.bits(vp), bt.numpy(),
                                 cl.numpy(), D ** -0.5)
        _close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0
