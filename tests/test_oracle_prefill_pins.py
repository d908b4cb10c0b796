"""Pins of the oracle's multi-query (chunked prefill) attention (CPU only).

  * a library routine: torch scaled_dot_product_attention (fp64) on the
    contiguous K/V with the causal-offset mask (query i of a chunk of q_len
    sees keys 0 .. L - q_len + i), ragged batch, GQA, several block sizes;
  * q_len = 1 is the decode: bit-identical to the pinned decode oracle;
  * causality: changing K/V at positions after a query's own leaves that
    query's output bit-identical (and changing them at its own position
    does change it);
  * q_len = L with L = 1 returns V_0 exactly.
Each test names the mistake it would catch.
"""
import numpy as np
import torch

from tests import paging


def _batch(seed, lens, q_lens, Hq, Hkv, D, bs=16):
    g = torch.Generator().manual_seed(seed)
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + bs - 1) // bs for L in lens) + 2
    (kp, vp), bt = paging.page([ks, vs], lens, bs, nb, g, poison=True)
    total = sum(q_lens)
    q = torch.randn((total, Hq, D), generator=g).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    return ks, vs, kp, vp, bt, q, cu


def _sdpa_prefill(q, cu, ks, vs, lens, q_lens, scale):
    total, Hq, D = q.shape
    Hkv = ks[0].shape[0]
    G = Hq // Hkv
    out = np.zeros((total, Hq, D))
    for b, (L, n) in enumerate(zip(lens, q_lens)):
        if n == 0:
            continue
        k = ks[b].to(torch.float64).repeat_interleave(G, dim=0)        # [Hq][L][D]
        v = vs[b].to(torch.float64).repeat_interleave(G, dim=0)
        qq = q[cu[b]:cu[b + 1]].to(torch.float64).transpose(0, 1)      # [Hq][n][D]
        pos = torch.arange(L - n, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos                         # [n][L]
        o = torch.nn.functional.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=scale)
        out[cu[b]:cu[b + 1]] = o.transpose(0, 1).numpy()
    return out


def test_prefill_matches_library_sdpa_with_causal_offset(oracle_lib):
    # catches a mask without the offset (L - q_len), a mask off by one, a wrong
    # row -> sequence mapping in the packed q, the GQA mapping
    for bs, (Hq, Hkv, D) in ((16, (8, 2, 32)), (4, (6, 3, 16)), (32, (4, 4, 8))):
        lens = [40, 7, 64, 1, 33]
        q_lens = [13, 7, 1, 1, 0]
        ks, vs, kp, vp, bt, q, cu = _batch(11 + bs, lens, q_lens, Hq, Hkv, D, bs)
        scale = D ** -0.5
        got = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp), paging.bits(vp), bt.numpy(),
                                 np.array(lens, np.int32), scale)
        want = _sdpa_prefill(q, cu, ks, vs, lens, q_lens, scale)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_single_query_prefill_is_the_decode(oracle_lib):
    lens = [50, 17, 3]
    ks, vs, kp, vp, bt, q, cu = _batch(2, lens, [1, 1, 1], 8, 2, 32)
    cl = np.array(lens, np.int32)
    got = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp), paging.bits(vp), bt.numpy(), cl, 0.3)
    want = oracle_lib.decode(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(), cl, 0.3)
    assert np.array_equal(got, want)


def test_future_tokens_do_not_leak(oracle_lib):
    # catches a missing causal mask or one that admits the next position
    lens, q_lens = [48], [20]
    ks, vs, kp, vp, bt, q, cu = _batch(3, lens, q_lens, 4, 2, 16)
    cl = np.array(lens, np.int32)
    base = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp), paging.bits(vp), bt.numpy(), cl, 0.25)
    i = 5                          # query 5 sits at position 48 - 20 + 5 = 33
    pos = lens[0] - q_lens[0] + i
    kp2, vp2 = kp.clone(), vp.clone()
    blk, off = int(bt[0, (pos + 1) // 16]), (pos + 1) % 16
    kp2[blk, :, off] = kp2[blk, :, off] * 3        # position 34: in the future of query 5
    vp2[blk, :, off] = -vp2[blk, :, off]
    got = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp2), paging.bits(vp2), bt.numpy(), cl, 0.25)
    assert np.array_equal(got[: i + 1], base[: i + 1])      # queries 0 .. 5 see up to position 33
    assert not np.array_equal(got[i + 1], base[i + 1])      # query 6 sees position 34
    kp3 = kp.clone()
    blk, off = int(bt[0, pos // 16]), pos % 16
    kp3[blk, :, off] = kp3[blk, :, off] * 3                 # its own position
    got3 = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp3), paging.bits(vp), bt.numpy(), cl, 0.25)
    assert not np.array_equal(got3[i], base[i])


def test_first_token_of_a_full_prefill_is_v0(oracle_lib):
    lens, q_lens = [20], [20]
    ks, vs, kp, vp, bt, q, cu = _batch(4, lens, q_lens, 4, 1, 16)
    got = oracle_lib.prefill(paging.bits(q), cu, paging.bits(kp), paging.bits(vp), bt.numpy(),
                             np.array(lens, np.int32), 0.5)
    assert np.array_equal(got[0], vs[0][0, 0][None, :].expand(4, 16).to(torch.float64).numpy())
