"""Pins of the fp64 oracle to things other than itself (CPU only).

The pages name paged decode attention, the paged KV cache and the online
softmax but print no formula, tensor or worked example, so the oracle is
pinned by:
  * a library routine: torch's scaled_dot_product_attention (fp64, CPU) on
    the contiguous, un-paged K/V, with the GQA head mapping h -> h // G;
  * invariances: relabelling physical blocks, and re-paging with another
    block size, leave the output bit-identical;
  * closed forms: context_len == 1 gives V_0 exactly; equal keys or
    scale == 0 give the mean of V; a two-token example gives weights
    1/(1+e), e/(1+e); a dominant key gives its value;
  * the split/merge identity of flash-decoding partials;
  * an append round trip through the documented layout.
Each test names the mistake it would catch.
"""
import math

import numpy as np
import pytest
import torch

from tests import paging


def _decode(oracle, q, kp, vp, bt, lens, scale):
    return oracle.decode(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(),
                         np.asarray(lens, dtype=np.int32), scale)


def _sdpa(q, k_seqs, v_seqs, lens, scale):
    """torch SDPA (fp64) per sequence on contiguous K/V, kv heads expanded
    so that query head h reads kv head h // G."""
    B, Hq, D = q.shape
    Hkv = k_seqs[0].shape[0]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        if lens[b] == 0:
            continue
        k = k_seqs[b].to(torch.float64).repeat_interleave(G, dim=0)   # [Hq][L][D]
        v = v_seqs[b].to(torch.float64).repeat_interleave(G, dim=0)
        qq = q[b].to(torch.float64)[:, None, :]                        # [Hq][1][D]
        out[b] = torch.nn.functional.scaled_dot_product_attention(
            qq, k, v, scale=scale)[:, 0, :].numpy()
    return out


SHAPES = [
    # B, Hq, Hkv, D, bs, max_len
    (3, 4, 2, 4, 4, 40),
    (2, 8, 2, 64, 16, 40),
    (3, 6, 3, 8, 1, 12),
    (2, 4, 4, 16, 32, 70),
    (4, 8, 1, 128, 16, 33),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_matches_library_sdpa_on_contiguous_kv(oracle_lib, shape):
    # catches: wrong gather index (t / bs vs t % bs), transposed layout,
    # dropped or misapplied scale, wrong GQA mapping, unnormalised softmax
    B, Hq, Hkv, D, bs, max_len = shape
    g = torch.Generator().manual_seed(hash(shape) & 0xFFFF)
    lens = torch.randint(1, max_len + 1, (B,), generator=g).tolist()
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = sum((L + bs - 1) // bs for L in lens) + 5
    (kp, vp), bt = paging.page([ks, vs], lens, bs, nb, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    scale = 0.37
    got = _decode(oracle_lib, q, kp, vp, bt, lens, scale)
    ref = _sdpa(q, ks, vs, lens, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_large_logits_are_stable(oracle_lib):
    # catches: softmax without the max subtraction (exp overflows to inf)
    B, Hq, Hkv, D, bs = 2, 4, 2, 32, 16
    g = torch.Generator().manual_seed(7)
    lens = [37, 50]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 10, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    got = _decode(oracle_lib, q, kp, vp, bt, lens, 400.0)
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, _sdpa(q, ks, vs, lens, 400.0), rtol=1e-10, atol=1e-12)


def test_block_permutation_invariance(oracle_lib):
    # catches: any dependence on physical block ids beyond the gather
    B, Hq, Hkv, D, bs = 3, 8, 2, 64, 16
    g = torch.Generator().manual_seed(11)
    lens = [100, 17, 64]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    nb = 20
    (kp, vp), bt = paging.page([ks, vs], lens, bs, nb, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    base = _decode(oracle_lib, q, kp, vp, bt, lens, 0.125)
    perm = torch.randperm(nb, generator=g)
    kp2, vp2 = torch.empty_like(kp), torch.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    bt2 = bt.clone()
    used = bt != paging.PAD_BLOCK
    bt2[used] = perm[bt[used].long()].to(torch.int32)
    got = _decode(oracle_lib, q, kp2, vp2, bt2, lens, 0.125)
    assert np.array_equal(got, base)


def test_block_size_invariance(oracle_lib):
    # catches: page-boundary off-by-one, offset computed with the wrong block size
    B, Hq, Hkv, D = 2, 4, 2, 16
    g = torch.Generator().manual_seed(13)
    lens = [45, 33]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    outs = []
    for bs in (1, 4, 16, 32):
        nb = sum((L + bs - 1) // bs for L in lens) + 2
        (kp, vp), bt = paging.page([ks, vs], lens, bs, nb, g)
        outs.append(_decode(oracle_lib, q, kp, vp, bt, lens, 0.25))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_context_len_one_returns_v0_exactly(oracle_lib):
    # catches: softmax weight not exactly 1 for one token, wrong V row
    B, Hq, Hkv, D, bs = 3, 8, 2, 64, 16
    g = torch.Generator().manual_seed(17)
    lens = [1, 1, 1]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 8, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    got = _decode(oracle_lib, q, kp, vp, bt, lens, 0.125)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            assert np.array_equal(got[b, h], paging.to_f64(vs[b][h // G, 0]))


@pytest.mark.parametrize("mode", ["equal_keys", "zero_scale"])
def test_uniform_weights_give_mean_of_v(oracle_lib, mode):
    # catches: weights that do not sum to one, a dropped token, an extra token
    B, Hq, Hkv, D, bs = 2, 4, 2, 32, 16
    g = torch.Generator().manual_seed(19)
    lens = [29, 48]
    ks = paging.random_seqs(g, lens, Hkv, D)
    if mode == "equal_keys":
        ks = [k[:, :1, :].expand(-1, k.shape[1], -1).contiguous() for k in ks]
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 10, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    got = _decode(oracle_lib, q, kp, vp, bt, lens, 0.0 if mode == "zero_scale" else 0.2)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            mean = paging.to_f64(vs[b][h // G]).mean(axis=0)
            np.testing.assert_allclose(got[b, h], mean, rtol=1e-14, atol=1e-15)


def test_two_token_closed_form(oracle_lib):
    # logits (0, 1) -> weights (1, e) / (1 + e); V rows are the unit vectors,
    # so out = (1/(1+e), e/(1+e)).  catches: exp base, sign of the logit,
    # weights applied to the wrong rows
    D, bs = 2, 16
    q = torch.tensor([[[1.0, 0.0]]], dtype=torch.bfloat16)
    k = [torch.tensor([[[0.0, 0.0], [1.0, 0.0]]], dtype=torch.bfloat16)]
    v = [torch.tensor([[[1.0, 0.0], [0.0, 1.0]]], dtype=torch.bfloat16)]
    (kp, vp), bt = paging.page([k, v], [2], bs, 1, torch.Generator().manual_seed(0))
    got = _decode(oracle_lib, q, kp, vp, bt, [2], 1.0)
    e = math.e
    np.testing.assert_allclose(got[0, 0], [1 / (1 + e), e / (1 + e)], rtol=1e-15)


def test_dominant_key_selects_its_value(oracle_lib):
    # one key aligned with q and 64x larger -> its weight is 1 - O(e^-60)
    # catches: max taken over the wrong axis, weights not exponentiated
    D, bs, L = 16, 16, 40
    g = torch.Generator().manual_seed(23)
    q = torch.zeros((1, 1, D), dtype=torch.bfloat16)
    q[0, 0, 3] = 1.0
    k = torch.randn((1, L, D), generator=g).mul(0.01).to(torch.bfloat16)
    k[0, 21] = 0
    k[0, 21, 3] = 64.0
    v = torch.randn((1, L, D), generator=g).to(torch.bfloat16)
    (kp, vp), bt = paging.page([[k], [v]], [L], bs, 4, g)
    got = _decode(oracle_lib, q, kp, vp, bt, [L], 1.0)
    np.testing.assert_allclose(got[0, 0], paging.to_f64(v[0, 21]), rtol=1e-20, atol=1e-20)


def test_gqa_head_mapping(oracle_lib):
    # query head h must read kv head h // G (consecutive heads share a kv head)
    # catches: h % Hkv mapping
    B, Hq, Hkv, D, bs = 1, 6, 3, 16, 16
    g = torch.Generator().manual_seed(29)
    lens = [30]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 4, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    got = _decode(oracle_lib, q, kp, vp, bt, lens, 0.3)
    for h in range(Hq):
        kv = h // (Hq // Hkv)
        (kp1, vp1), bt1 = paging.page([[ks[0][kv:kv + 1]], [vs[0][kv:kv + 1]]], lens, bs, 4, g)
        one = _decode(oracle_lib, q[:, h:h + 1], kp1, vp1, bt1, lens, 0.3)
        assert np.array_equal(got[0, h], one[0, 0])


def test_split_partials_merge_to_full_decode(oracle_lib):
    # flash-decoding identity; catches: wrong rescale exp(m_i - M), l not
    # carried, empty ranges given weight
    B, Hq, Hkv, D, bs = 2, 4, 2, 64, 16
    g = torch.Generator().manual_seed(31)
    lens = [100, 57]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 12, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    full = _decode(oracle_lib, q, kp, vp, bt, lens, 0.125)
    for b, cuts in [(0, [0, 16, 16, 33, 80, 100]), (1, [0, 1, 40, 57])]:
        for h in range(Hq):
            rb = [b] * (len(cuts) - 1)
            rh = [h] * (len(cuts) - 1)
            o, m, l = oracle_lib.partials(paging.bits(q), paging.bits(kp), paging.bits(vp),
                                          bt.numpy(), np.asarray(lens, np.int32), 0.125,
                                          rb, rh, cuts[:-1], cuts[1:])
            merged = oracle_lib.lse_merge(o, m, l)
            np.testing.assert_allclose(merged, full[b, h], rtol=1e-12, atol=1e-14)


def test_single_token_partial_closed_form(oracle_lib):
    # one-token range: o = V_t, m = s_t, l = 1 exactly
    B, Hq, Hkv, D, bs = 1, 2, 1, 8, 4
    g = torch.Generator().manual_seed(37)
    lens = [9]
    ks = paging.random_seqs(g, lens, Hkv, D)
    vs = paging.random_seqs(g, lens, Hkv, D)
    (kp, vp), bt = paging.page([ks, vs], lens, bs, 5, g)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    o, m, l = oracle_lib.partials(paging.bits(q), paging.bits(kp), paging.bits(vp), bt.numpy(),
                                  np.asarray(lens, np.int32), 0.5, [0], [1], [6], [7])
    assert np.array_equal(o[0], paging.to_f64(vs[0][0, 6]))
    s = 0.5 * float((paging.to_f64(q[0, 1]) * paging.to_f64(ks[0][0, 6])).sum())
    assert m[0] == pytest.approx(s, rel=1e-15)
    assert l[0] == 1.0


def test_empty_context_gives_zero_and_reads_nothing(oracle_lib):
    # context_len 0: output 0 with no NaN even though every cache row is NaN
    # and every table entry is an out-of-range id
    B, Hq, Hkv, D, bs = 2, 4, 2, 16, 16
    kp = torch.zeros((3, Hkv, bs, D), dtype=torch.bfloat16)
    kp.view(torch.int16).fill_(paging.NAN_BITS)
    bt = torch.full((B, 2), paging.PAD_BLOCK, dtype=torch.int32)
    q = torch.ones((B, Hq, D), dtype=torch.bfloat16)
    got = _decode(oracle_lib, q, kp, kp.clone(), bt, [0, 0], 0.25)
    assert np.array_equal(got, np.zeros_like(got))


def test_block_id_out_of_range_is_reported(oracle_lib):
    B, Hq, Hkv, D, bs = 1, 2, 1, 8, 4
    kp = torch.zeros((2, Hkv, bs, D), dtype=torch.bfloat16)
    bt = torch.tensor([[0, 2]], dtype=torch.int32)      # block 2 does not exist
    q = torch.ones((B, Hq, D), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _decode(oracle_lib, q, kp, kp.clone(), bt, [6], 0.25)


def test_append_round_trip(oracle_lib):
    # rows land at block = slot // bs, offset = slot % bs of every kv head;
    # -1 slots are skipped; nothing else changes; a context of length one
    # over an appended slot decodes to the appended value exactly.
    NB, Hkv, bs, D, T = 6, 2, 16, 64, 5
    g = torch.Generator().manual_seed(41)
    kc = torch.zeros((NB, Hkv, bs, D), dtype=torch.bfloat16)
    kc.view(torch.int16).fill_(paging.NAN_BITS)
    vc = kc.clone()
    k_new = torch.randn((T, Hkv, D), generator=g).to(torch.bfloat16)
    v_new = torch.randn((T, Hkv, D), generator=g).to(torch.bfloat16)
    slots = np.array([3 * bs + 0, -1, 0 * bs + 15, 5 * bs + 7, 1 * bs + 0], dtype=np.int32)
    kb, vb = paging.bits(kc).copy(), paging.bits(vc).copy()
    oracle_lib.append(paging.bits(k_new), paging.bits(v_new), slots, kb, vb)
    expect_k, expect_v = paging.bits(kc).copy(), paging.bits(vc).copy()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        expect_k[s // bs, :, s % bs, :] = paging.bits(k_new)[t]
        expect_v[s // bs, :, s % bs, :] = paging.bits(v_new)[t]
    assert np.array_equal(kb, expect_k)
    assert np.array_equal(vb, expect_v)
    # decode a one-token context at slot 3*bs (token 0 of block 3)
    q = torch.randn((1, 2 * Hkv, D), generator=g).to(torch.bfloat16)
    bt = np.array([[3]], dtype=np.int32)
    out = oracle_lib.decode(paging.bits(q), kb, vb, bt, np.array([1], np.int32), 0.125)
    for h in range(2 * Hkv):
        assert np.array_equal(out[0, h], paging.to_f64(v_new[0, h // 2]))
