"""fp64 CPU oracle for paged-KV decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the cpu-baseline / reference
leg of ``bench.py`` may import this package.  The product path
(``paged_kv_attention_36_b200``) never imports it and shares no code with it.

The arithmetic lives in ``pa_oracle.c`` (plain C, double precision); this
module only compiles it with gcc and marshals numpy arrays through ctypes.
Every function states the operation it mirrors; the C file cites the pages.

Inputs are bf16 tensors passed as their raw ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "libpa_oracle.so")

_ERRORS = {
    -1: "bad argument",
    -2: "block id out of range inside the context",
    -3: "context_len outside [0, max_blocks_per_seq * block_size]",
    -4: "append slot beyond the pool",
    -5: "out of memory",
}


def build(force: bool = False) -> str:
    """Compile ``pa_oracle.c`` into ``libpa_oracle.so`` (gcc, no fast-math,
    no FMA contraction, so every operation is the one written)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.pa_oracle_decode.argtypes = [vp] * 5 + [i64] * 7 + [dbl, vp, i32]
        lib.pa_oracle_decode.restype = i32
        lib.pa_oracle_partials.argtypes = [vp] * 5 + [i64] * 7 + [dbl] + [vp] * 4 + [i64] + [vp] * 3
        lib.pa_oracle_partials.restype = i32
        lib.pa_oracle_lse_merge.argtypes = [vp, vp, vp, i64, i64, vp]
        lib.pa_oracle_lse_merge.restype = i32
        lib.pa_oracle_append.argtypes = [vp, vp, vp, i64, vp, vp, i64, i64, i64, i64]
        lib.pa_oracle_append.restype = i32
        lib.pa_oracle_e4m3_encode_array.argtypes = [vp, i64, vp]
        lib.pa_oracle_e4m3_encode_array.restype = None
        lib.pa_oracle_e4m3_decode_array.argtypes = [vp, i64, vp]
        lib.pa_oracle_e4m3_decode_array.restype = None
        lib.pa_oracle_append_fp8.argtypes = [vp, vp, vp, i64, vp, vp, vp, vp, i64, i64, i64]
        lib.pa_oracle_append_fp8.restype = i32
        lib.pa_oracle_decode_fp8.argtypes = [vp] * 7 + [i64] * 6 + [dbl, vp, i32]
        lib.pa_oracle_decode_fp8.restype = i32
        lib.pa_oracle_prefill.argtypes = [vp] * 6 + [i64] * 7 + [dbl, vp, i32]
        lib.pa_oracle_prefill.restype = i32
        _lib = lib
    return _lib


def _check(rc: int) -> None:
    if rc != 0:
        raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs must be passed as uint16 bit patterns")
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q, k_cache, block_tables):
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    return B, Hq, Hkv, D, bs, NB, block_tables.shape[1]


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float,
           nthreads: int | None = None) -> np.ndarray:
    """out[b][h] = softmax(scale * q[b][h] . K_t) . V_t over the paged tokens
    t < context_lens[b] of kv head h // (Hq/Hkv); fp64, shape [B][Hq][D].

    q: [B][Hq][D] u16; k_cache, v_cache: [NB][Hkv][bs][D] u16;
    block_tables: [B][M] int32; context_lens: [B] int32."""
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    block_tables, context_lens = _i32(block_tables), _i32(context_lens)
    B, Hq, Hkv, D, bs, NB, M = _dims(q, k_cache, block_tables)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    rc = _load().pa_oracle_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                  _ptr(context_lens), B, Hq, Hkv, D, bs, NB, M, float(scale),
                                  _ptr(out), int(nthreads or default_threads()))
    _check(rc)
    return out


def partials(q, k_cache, v_cache, block_tables, context_lens, scale: float,
             rb, rh, rt0, rt1):
    """Split-KV partials for ranges (b, h, [t0, t1)): returns (o [n][D],
    m [n], l [n]) with o normalised, m the max logit and
    l = sum exp(s - m), all fp64."""
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    block_tables, context_lens = _i32(block_tables), _i32(context_lens)
    B, Hq, Hkv, D, bs, NB, M = _dims(q, k_cache, block_tables)
    rb, rh, rt0, rt1 = _i32(rb), _i32(rh), _i32(rt0), _i32(rt1)
    n = rb.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    m = np.zeros(n, dtype=np.float64)
    l = np.zeros(n, dtype=np.float64)
    rc = _load().pa_oracle_partials(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                    _ptr(context_lens), B, Hq, Hkv, D, bs, NB, M, float(scale),
                                    _ptr(rb), _ptr(rh), _ptr(rt0), _ptr(rt1), n,
                                    _ptr(o), _ptr(m), _ptr(l))
    _check(rc)
    return o, m, l


def lse_merge(o, m, l) -> np.ndarray:
    """Merge n partials (o [n][D], m [n], l [n]) of one row by log-sum-exp."""
    o = np.ascontiguousarray(o, dtype=np.float64)
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    n, D = o.shape
    out = np.zeros(D, dtype=np.float64)
    _check(_load().pa_oracle_lse_merge(_ptr(o), _ptr(m), _ptr(l), n, D, _ptr(out)))
    return out


def append(k_new, v_new, slot_mapping, k_cache, v_cache) -> None:
    """In place: k_cache[s // bs][g][s % bs] = k_new[t][g] (same for V) for
    every t with s = slot_mapping[t] >= 0.  Caches must be writable,
    C-contiguous uint16 arrays of shape [NB][Hkv][bs][D]."""
    k_new, v_new, slot_mapping = _u16(k_new), _u16(v_new), _i32(slot_mapping)
    for c in (k_cache, v_cache):
        if not (isinstance(c, np.ndarray) and c.dtype == np.uint16 and c.flags.c_contiguous):
            raise TypeError("caches must be C-contiguous uint16 numpy arrays")
    NB, Hkv, bs, D = k_cache.shape
    T = slot_mapping.shape[0]
    rc = _load().pa_oracle_append(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T,
                                  _ptr(k_cache), _ptr(v_cache), Hkv, D, bs, NB)
    _check(rc)


# ---------------------------------------------------------------------------
# fp8 (OCP E4M3) KV cache with per-kv-head scales; layouts in pa_oracle.c.

def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 codes (ties to even, |x| > 448 saturating, NaN -> 0x7F)
    of float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint8)
    _load().pa_oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    """Values (fp64) of E4M3 codes."""
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.zeros(c.shape, dtype=np.float64)
    _load().pa_oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def append_fp8(k_new, v_new, slot_mapping, k_cache8, v_cache8, k_scale, v_scale) -> None:
    """In place: encode token t's rows as e4m3(x / scale[g]) into slot
    slot_mapping[t] (>= 0) of the fp8 caches: k_cache8 [NB][Hkv][16][D],
    v_cache8 [NB][Hkv][D][16] (tokens in the transposed tile order)."""
    k_new, v_new, slot_mapping = _u16(k_new), _u16(v_new), _i32(slot_mapping)
    for c in (k_cache8, v_cache8):
        if not (isinstance(c, np.ndarray) and c.dtype == np.uint8 and c.flags.c_contiguous):
            raise TypeError("fp8 caches must be C-contiguous uint8 numpy arrays")
    NB, Hkv, bs, D = k_cache8.shape
    if bs != 16 or v_cache8.shape != (NB, Hkv, D, 16):
        raise ValueError("fp8 caches are [NB][Hkv][16][D] and [NB][Hkv][D][16]")
    ks = np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_scale, dtype=np.float32)
    T = slot_mapping.shape[0]
    _check(_load().pa_oracle_append_fp8(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(k_cache8),
                                        _ptr(v_cache8), _ptr(ks), _ptr(vs), Hkv, D, NB))


def decode_fp8(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, scale: float,
               nthreads: int | None = None) -> np.ndarray:
    """The decode over the dequantized fp8 caches (values e4m3(c) * scale[g]); fp64 [B][Hq][D]."""
    q = _u16(q)
    k8 = np.ascontiguousarray(k_cache8, dtype=np.uint8)
    v8 = np.ascontiguousarray(v_cache8, dtype=np.uint8)
    block_tables, context_lens = _i32(block_tables), _i32(context_lens)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k8.shape
    if D2 != D or bs != 16 or v8.shape != (NB, Hkv, D, 16) or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    ks = np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    _check(_load().pa_oracle_decode_fp8(_ptr(q), _ptr(k8), _ptr(v8), _ptr(ks), _ptr(vs), _ptr(block_tables),
                                        _ptr(context_lens), B, Hq, Hkv, D, NB, block_tables.shape[1],
                                        float(scale), _ptr(out), int(nthreads or default_threads())))
    return out


def prefill(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, scale: float,
            nthreads: int | None = None) -> np.ndarray:
    """Multi-query (chunked prefill) attention: q [total][Hq][D] u16 holds, for
    sequence b, rows cu_q_lens[b] .. cu_q_lens[b+1]-1, its last q_len_b
    tokens; token i (position L_b - q_len_b + i) attends to tokens 0 .. its
    position.  fp64 [total][Hq][D]."""
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    block_tables, context_lens, cu = _i32(block_tables), _i32(context_lens), _i32(cu_q_lens)
    total, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    B, M = block_tables.shape
    if D2 != D or cu.shape[0] != B + 1 or int(cu[-1]) != total:
        raise ValueError("shape mismatch")
    out = np.zeros((total, Hq, D), dtype=np.float64)
    _check(_load().pa_oracle_prefill(_ptr(q), _ptr(cu), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                     _ptr(context_lens), B, Hq, Hkv, D, bs, NB, M, float(scale), _ptr(out),
                                     int(nthreads or default_threads())))
    return out
