"""GPU parity of the shared-prefix ("cascade") decode: the prefix pass plus
the decode over each member's own pages, through the C ABI, against the
fp64 oracle's plain decode of the same batch (the grouping changes the
order of the work, not the result).  Tolerance as for the decode:
|gpu - ref| <= 1e-2 + 1e-2*|ref| per bf16 element.

Covered: the prefix-shared batch at full size (fused append, and decode
alone), every built head shape, members whose whole context is the prefix,
groups of one, groups that share nothing, sequences outside any group,
empty contexts, more key ranges than prefix pages, a member long enough to
be split over many CTAs, repeated calls on one workspace, and the contract
breaches that fall back to a plain decode of the member (a context shorter
than the prefix, a group larger than max_group_size) or are only reported
(a member whose table does not hold the prefix blocks).
"""
import os

import numpy as np
import pytest
import torch

from tests import paging

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-2

# PA_DECODE_MATH=simt (set for a child process by test_kernel_variants_gpu.py)
# selects the fp32 CUDA-core decode policy, built for head_dim * Hq/Hkv <= 256.
SIMT = os.environ.get("PA_DECODE_MATH") == "simt"


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_kv_attention_36_b200 import binding
    binding.pa_device_errors(clear=True)
    return binding


def _assert_close(out, ref):
    got = out.to(torch.float64).cpu().numpy()
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    assert not np.isnan(got).any(), "NaN in output"
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} elements outside tolerance; max err {err.max():.3g}, "
                           f"worst at {np.unravel_index(np.argmax(err - bound), err.shape)}")


def _dev(w):
    d = torch.device("cuda")
    names = ("q", "k_cache", "v_cache", "block_tables", "context_lens", "k_new", "v_new", "slot_mapping",
             "group_offsets", "group_prefix_pages")
    return {k: getattr(w, k).to(d) for k in names if getattr(w, k) is not None}


def _ref(oracle, w):
    return oracle.decode(paging.bits(w.q), paging.bits(w.k_cache), paging.bits(w.v_cache),
                         w.block_tables.numpy(), w.context_lens.numpy(), w.scale)


def _decode(pa, t, w, max_group_size=None, workspace=None):
    out = torch.full_like(t["q"], float("nan"))
    mgs = w.max_group_size if max_group_size is None else max_group_size
    pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                               w.scale, t["group_offsets"], t["group_prefix_pages"], mgs, out,
                               workspace=workspace)
    torch.cuda.synchronize()
    return out


def test_prefix_batch_fused_append_matches_oracle(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("prefix", poison=True)
    assert w.num_groups == 2 and w.max_group_size == 128
    kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
    oracle_lib.append(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), kb, vb)
    ref = oracle_lib.decode(paging.bits(w.q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(), w.scale)
    t = _dev(w)
    out = torch.full_like(t["q"], float("nan"))
    pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                               w.scale, t["group_offsets"], t["group_prefix_pages"], w.max_group_size, out,
                               k_new=t["k_new"], v_new=t["v_new"], slot_mapping=t["slot_mapping"])
    torch.cuda.synchronize()
    assert torch.equal(t["k_cache"].view(torch.int16).cpu(), torch.from_numpy(kb.view(np.int16)))
    assert torch.equal(t["v_cache"].view(torch.int16).cpu(), torch.from_numpy(vb.view(np.int16)))
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_prefix_batch_decode_alone_and_repeat(pa, oracle_lib):
    # decode only (the appended rows are not used: context_lens stay those of
    # the batch, whose last row is the one the append would write, so write
    # it first with the library's own append)
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("prefix", poison=True)
    t = _dev(w)
    pa.pa_cache_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
    w.k_cache, w.v_cache = t["k_cache"].cpu(), t["v_cache"].cpu()
    ref = _ref(oracle_lib, w)
    dims = pa.make_dims(t["q"], t["k_cache"], t["block_tables"])
    ws = torch.zeros(pa.pa_decode_shared_prefix_workspace_bytes(dims, w.num_groups, w.max_group_size),
                     dtype=torch.uint8, device="cuda")
    outs = [_decode(pa, t, w, workspace=ws) for _ in range(3)]
    for out in outs:
        _assert_close(out, ref)
    n_cnt = dims.num_seqs * dims.num_kv_heads
    assert int(ws[: 4 * n_cnt].view(torch.int32).abs().sum()) == 0
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("heads", [(16, 8, 128), (32, 8, 64), (8, 8, 64), (16, 2, 64), (8, 8, 128),
                                   (32, 8, 128), (64, 8, 128)])
def test_group_shapes(pa, oracle_lib, heads):
    # groups of 5 (ragged suffixes), 1, 17 (crosses a 128-row tile at G = 8),
    # a group sharing nothing, ungrouped tails including an empty context
    from paged_kv_attention_36_b200 import workloads
    if SIMT and (heads[0] // heads[1]) * heads[2] > 256:
        pytest.skip("the fp32 CUDA-core policy is built for head_dim * Hq/Hkv <= 256")
    g = torch.Generator().manual_seed(sum(heads))
    groups = [(5, 6), (1, 3), (17, 2), (3, 0)]
    n = sum(m for m, _ in groups)
    suffix = torch.randint(1, 90, (n,), generator=g).tolist()
    w = workloads.make_grouped("qwen3", groups, suffix, tail_lens=[40, 0, 17], poison=True, heads=heads)
    ref = _ref(oracle_lib, w)
    out = _decode(pa, _dev(w), w)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("fused", [False, True])
def test_large_grouped_batch(pa, oracle_lib, fused):
    # 330 members in two groups plus 30 sequences in none: more sequences
    # than a decode CTA's 288 threads (the share scan runs in chunks); fused,
    # the 360 new rows are more than the decode appends itself, so the
    # prefix pass writes them and the decode waits for it (their slots are
    # past the shared blocks: a private suffix of at least one token)
    from paged_kv_attention_36_b200 import workloads
    g = torch.Generator().manual_seed(91)
    suffix = torch.randint(1 if fused else 0, 60, (330,), generator=g).tolist()
    tails = torch.randint(0, 90, (30,), generator=g).tolist()
    w = workloads.make_grouped("tiny", [(150, 3), (180, 2)], suffix, tail_lens=tails, poison=True)
    t = _dev(w)
    if fused:
        kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
        oracle_lib.append(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), kb, vb)
        ref = oracle_lib.decode(paging.bits(w.q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(),
                                w.scale)
        out = torch.full_like(t["q"], float("nan"))
        pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                                   w.scale, t["group_offsets"], t["group_prefix_pages"], w.max_group_size, out,
                                   k_new=t["k_new"], v_new=t["v_new"], slot_mapping=t["slot_mapping"])
        torch.cuda.synchronize()
        assert torch.equal(t["k_cache"].view(torch.int16).cpu(), torch.from_numpy(kb.view(np.int16)))
        assert torch.equal(t["v_cache"].view(torch.int16).cpu(), torch.from_numpy(vb.view(np.int16)))
    else:
        ref = _ref(oracle_lib, w)
        out = _decode(pa, t, w)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


@pytest.mark.parametrize("fused", [False, True])
def test_many_groups(pa, oracle_lib, fused):
    # ten groups, one of them empty and one sharing nothing: more groups than
    # the decode reads in one round, so sequences find theirs by bisection
    from paged_kv_attention_36_b200 import workloads
    g = torch.Generator().manual_seed(93)
    groups = [(2, 1), (3, 2), (1, 1), (0, 2), (4, 3), (2, 0), (1, 1), (3, 1), (2, 2), (5, 1)]
    n = sum(m for m, _ in groups)
    suffix = torch.randint(1, 50, (n,), generator=g).tolist()
    w = workloads.make_grouped("tiny", groups, suffix, tail_lens=[9, 0], poison=True)
    t = _dev(w)
    if fused:
        kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
        oracle_lib.append(paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy(), kb, vb)
        ref = oracle_lib.decode(paging.bits(w.q), kb, vb, w.block_tables.numpy(), w.context_lens.numpy(),
                                w.scale)
        out = torch.full_like(t["q"], float("nan"))
        pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                                   w.scale, t["group_offsets"], t["group_prefix_pages"], w.max_group_size, out,
                                   k_new=t["k_new"], v_new=t["v_new"], slot_mapping=t["slot_mapping"])
        torch.cuda.synchronize()
        assert torch.equal(t["k_cache"].view(torch.int16).cpu(), torch.from_numpy(kb.view(np.int16)))
    else:
        ref = _ref(oracle_lib, w)
        out = _decode(pa, t, w)
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_members_whose_context_is_the_prefix(pa, oracle_lib):
    # suffix 0: no own pages, the output is the prefix partials merged alone
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("qwen3", [(4, 5), (3, 1)], [0, 7, 0, 16, 0, 0, 1], tail_lens=[5], poison=True)
    ref = _ref(oracle_lib, w)
    _assert_close(_decode(pa, _dev(w), w), ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_more_key_ranges_than_prefix_pages(pa, oracle_lib):
    # one small group: the prefix pass splits the keys up to 16 ways, so most
    # ranges of a 2-page prefix are empty
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("tiny", [(2, 2)], [3, 20], poison=True)
    ref = _ref(oracle_lib, w)
    _assert_close(_decode(pa, _dev(w), w), ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_long_member_split_over_ctas(pa, oracle_lib):
    # a member with 40000 own tokens is split over many CTAs: only the piece
    # that starts at its first own page may carry the prefix
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("qwen3", [(3, 40)], [40000, 9, 300], tail_lens=[5000], poison=True)
    ref = _ref(oracle_lib, w)
    _assert_close(_decode(pa, _dev(w), w), ref)
    assert pa.pa_device_errors(clear=True) == 0


def test_context_shorter_than_prefix_falls_back(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("qwen3", [(4, 6)], [10, 20, 30, 40], poison=True)
    w.context_lens[2] = 6 * 16 - 5    # inside the shared blocks: decoded over its own table
    ref = _ref(oracle_lib, w)
    _assert_close(_decode(pa, _dev(w), w), ref)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_PREFIX


def test_group_larger_than_max_group_size_falls_back(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("qwen3", [(6, 4), (2, 3)], [5, 6, 7, 8, 9, 10, 11, 12], poison=True)
    ref = _ref(oracle_lib, w)
    _assert_close(_decode(pa, _dev(w), w, max_group_size=4), ref)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_PREFIX


def test_member_without_the_prefix_blocks_is_reported(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make_grouped("qwen3", [(3, 4)], [5, 6, 7])
    w.block_tables[1, 2] = w.block_tables[1, 4]  # member 1's third block is its own, not the group's
    _decode(pa, _dev(w), w)
    assert pa.pa_device_errors(clear=True) & pa.PA_DEVERR_PREFIX


def test_no_groups_is_plain_decode(pa, oracle_lib):
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make("qwen3", poison=True)
    t = _dev(w)
    pa.pa_cache_append(t["k_new"], t["v_new"], t["slot_mapping"], t["k_cache"], t["v_cache"])
    w.k_cache, w.v_cache = t["k_cache"].cpu(), t["v_cache"].cpu()
    ref = _ref(oracle_lib, w)
    empty_off = torch.zeros(1, dtype=torch.int32, device="cuda")
    empty_pp = torch.zeros(0, dtype=torch.int32, device="cuda")
    out = torch.full_like(t["q"], float("nan"))
    pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                               w.scale, empty_off, empty_pp, 0, out)
    torch.cuda.synchronize()
    _assert_close(out, ref)
    assert pa.pa_device_errors(clear=True) == 0
