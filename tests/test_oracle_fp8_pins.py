"""Pins of the oracle's fp8 (OCP E4M3) KV-cache functions (CPU only).

  * the E4M3 code table against torch's float8_e4m3fn (an independent
    implementation of the format), all 256 codes;
  * the encoder against torch's conversion on random values and on every
    midpoint between neighbouring codes (ties to even), and against the
    format's definition at the edges: saturation beyond 448, NaN, signed
    zero, the smallest subnormal;
  * the append's byte layout on a hand-worked example, from the documented
    formulas (k token-major; v transposed with the token order
    pos(t) = 4*((t % 8) / 2) + 2*(t / 8) + t % 2);
  * the fp8 decode against the already pinned bf16 decode on caches holding
    the dequantized values, with power-of-two scales so that those values
    are exact in bf16.
Each test names the mistake it would catch.
"""
import numpy as np
import pytest
import torch

from tests import paging


def _torch_decode_codes(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def test_e4m3_code_table_matches_torch(oracle_lib):
    # catches a wrong exponent bias, a missing subnormal rule or a NaN code mix-up
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_lib.e4m3_decode(codes)
    want = _torch_decode_codes(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encoder_matches_torch_in_range(oracle_lib):
    # catches rounding toward zero or ties away from zero
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000) * s for s in (0.01, 1.0, 30.0, 120.0)]).astype(np.float32)
    x = x[np.abs(x) < 448.0]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle_lib.e4m3_encode(x), want)


def test_e4m3_midpoints_round_to_even(oracle_lib):
    # every value halfway between two neighbouring positive codes goes to the
    # code whose mantissa is even; just below / above go to the nearer one
    codes = np.arange(0, 0x7E, dtype=np.uint8)            # 0 .. 416 (0x7D), then 448
    lo = oracle_lib.e4m3_decode(codes)
    hi = oracle_lib.e4m3_decode(codes + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # midpoints are exact in fp32
    got = oracle_lib.e4m3_encode(mid)
    even = np.where(codes % 2 == 0, codes, codes + 1).astype(np.uint8)
    assert np.array_equal(got, even)
    below = np.nextafter(mid, np.float32(0)).astype(np.float32)
    above = np.nextafter(mid, np.float32(np.inf)).astype(np.float32)
    assert np.array_equal(oracle_lib.e4m3_encode(below), codes)
    assert np.array_equal(oracle_lib.e4m3_encode(above), (codes + 1).astype(np.uint8))


def test_e4m3_edges(oracle_lib):
    # catches a missing saturation (e.g. NaN or an overflow code for 500),
    # a lost sign, or a wrong smallest subnormal
    x = np.array([448, 464, 470, 479.9, 1000, 1e30, -1000, np.inf, -np.inf, np.nan,
                  0.0, -0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -11, 1.0, -1.0], dtype=np.float32)
    want = [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE, 0x7F,
            0x00, 0x80, 0x01, 0x00, 0x02, 0x00, 0x38, 0xB8]
    assert oracle_lib.e4m3_encode(x).tolist() == want


def _vt_pos(t):
    return 4 * ((t % 8) // 2) + 2 * (t // 8) + t % 2


def test_vt_position_is_a_permutation_of_16():
    assert sorted(_vt_pos(t) for t in range(16)) == list(range(16))
    assert [t for p in range(16) for t in range(16) if _vt_pos(t) == p] == \
        [0, 1, 8, 9, 2, 3, 10, 11, 4, 5, 12, 13, 6, 7, 14, 15]


def test_append_fp8_hand_example(oracle_lib):
    # two tokens, 2 kv heads, D = 16, 3 blocks: token 0 -> slot 21 (block 1,
    # offset 5), token 1 -> padding; k scale 0.5 / 2, v scale 0.25 / 4
    Hkv, D, NB = 2, 16, 3
    kn = torch.zeros((2, Hkv, D), dtype=torch.float32)
    vn = torch.zeros((2, Hkv, D), dtype=torch.float32)
    kn[0, 0] = torch.arange(D) * 0.25          # / 0.5 -> 0, 0.5, 1, ...
    kn[0, 1] = -torch.arange(D) * 4.0          # / 2   -> 0, -2, -4, ...
    vn[0, 0] = 1.0                              # / 0.25 -> 4
    vn[0, 1] = torch.arange(D) * 8.0           # / 4   -> 0, 2, 4, ...
    kb, vb = kn.to(torch.bfloat16), vn.to(torch.bfloat16)
    k8 = np.zeros((NB, Hkv, 16, D), dtype=np.uint8)
    v8 = np.zeros((NB, Hkv, D, 16), dtype=np.uint8)
    slots = np.array([21, -1], dtype=np.int32)
    oracle_lib.append_fp8(paging.bits(kb), paging.bits(vb), slots, k8, v8,
                          np.array([0.5, 2.0], np.float32), np.array([0.25, 4.0], np.float32))
    dec = oracle_lib.e4m3_decode
    assert np.array_equal(dec(k8[1, 0, 5]), np.arange(D) * 0.5)
    assert np.array_equal(dec(k8[1, 1, 5]), -np.arange(D) * 2.0)
    assert np.array_equal(dec(v8[1, 0, :, _vt_pos(5)]), np.full(D, 4.0))
    assert np.array_equal(dec(v8[1, 1, :, _vt_pos(5)]), np.arange(D) * 2.0)
    # nothing else was written
    k8[1, :, 5] = 0
    v8[1, :, :, _vt_pos(5)] = 0
    assert not k8.any() and not v8.any()


def test_decode_fp8_equals_bf16_decode_of_dequantized_cache(oracle_lib):
    # power-of-two scales keep the dequantized values exact in bf16, so the fp8
    # decode must equal the pinned bf16 decode bit for bit (catches a wrong V
    # transpose or token order, a scale applied to the wrong head or tensor)
    g = torch.Generator().manual_seed(5)
    B, Hq, Hkv, D, NB, M = 3, 8, 2, 32, 12, 4
    lens = np.array([17, 64, 1], dtype=np.int32)
    k8 = torch.randint(0, 256, (NB, Hkv, 16, D), generator=g, dtype=torch.uint8).numpy()
    v8 = torch.randint(0, 256, (NB, Hkv, D, 16), generator=g, dtype=torch.uint8).numpy()
    k8[(k8 & 0x7F) == 0x7F] = 0x10   # no NaN codes
    v8[(v8 & 0x7F) == 0x7F] = 0x10
    k8 = np.where((k8 & 0x78) == 0x78, k8 & 0xC7, k8)  # keep magnitudes moderate (no exponent 15)
    ks = np.array([2.0 ** -4, 2.0 ** -3], np.float32)
    vs = np.array([2.0 ** -2, 1.0], np.float32)
    perm = torch.randperm(NB, generator=g).numpy()
    bt = perm[: B * M].reshape(B, M).astype(np.int32)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    got = oracle_lib.decode_fp8(paging.bits(q), k8, v8, ks, vs, bt, lens, 0.2)
    # the bf16 caches of the same values
    kf = oracle_lib.e4m3_decode(k8) * ks[None, :, None, None]
    vt = oracle_lib.e4m3_decode(v8) * vs[None, :, None, None]                # [NB][Hkv][D][16 positions]
    order = [next(t for t in range(16) if _vt_pos(t) == p) for p in range(16)]
    vf = np.zeros((NB, Hkv, 16, D))
    for p_, t in enumerate(order):
        vf[:, :, t, :] = vt[:, :, :, p_]
    kbf = torch.from_numpy(kf).to(torch.bfloat16)
    vbf = torch.from_numpy(vf).to(torch.bfloat16)
    assert np.array_equal(kbf.to(torch.float64).numpy(), kf) and np.array_equal(vbf.to(torch.float64).numpy(), vf)
    want = oracle_lib.decode(paging.bits(q), paging.bits(kbf), paging.bits(vbf), bt, lens, 0.2)
    assert np.array_equal(got, want)
