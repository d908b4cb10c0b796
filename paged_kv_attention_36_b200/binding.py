"""ctypes binding of libpa_b200.so (the C ABI declared in include/pa.h).

Argument marshalling only: every function checks the tensors' dtype,
device and contiguity, turns them into raw pointers plus a ``pa_dims``
struct and the current CUDA stream, calls the C entry point of the same
name, and raises ``PaError`` on a non-zero status.  All computation runs in
the library's CUDA kernels; if the library is missing this module raises at
import time instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_CONTEXT = 0x2
PA_DEVERR_SLOT = 0x4
PA_DEVERR_TIMEOUT = 0x8
PA_DEVERR_PREFIX = 0x10


class PaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {pa_status_string(code)} ({code})")
        self.code = code


class pa_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "num_blocks",
        "max_blocks_per_seq")]

    def __repr__(self):
        return "pa_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m paged_kv_attention_36_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    dp = ctypes.POINTER(pa_dims)
    lib.pa_cache_append.argtypes = [vp, vp, vp, i32, vp, vp, dp, vp]
    lib.pa_cache_append.restype = i32
    lib.pa_decode_workspace_bytes.argtypes = [dp, i32]
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode_default_ctas.argtypes = []
    lib.pa_decode_default_ctas.restype = i32
    lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, f32, vp, dp, vp, sz, vp]
    lib.pa_decode.restype = i32
    lib.pa_decode_partials.argtypes = [vp, vp, vp, vp, vp, f32, vp, dp, i32, vp, sz, i32,
                                       vp, vp, vp, vp, vp, vp]
    lib.pa_decode_partials.restype = i32
    lib.pa_append_decode.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, f32, vp, dp, vp, sz, vp]
    lib.pa_append_decode.restype = i32
    lib.pa_decode_shared_prefix_workspace_bytes.argtypes = [dp, i32, i32]
    lib.pa_decode_shared_prefix_workspace_bytes.restype = sz
    lib.pa_decode_shared_prefix.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, f32, vp, vp, i32, i32,
                                            vp, dp, vp, sz, vp]
    lib.pa_decode_shared_prefix.restype = i32
    lib.pa_cache_append_fp8.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, dp, vp]
    lib.pa_cache_append_fp8.restype = i32
    lib.pa_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, f32, vp, dp, vp, sz, vp]
    lib.pa_decode_fp8.restype = i32
    lib.pa_append_decode_fp8.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, f32, vp, dp, vp, sz, vp]
    lib.pa_append_decode_fp8.restype = i32
    lib.pa_prefill.argtypes = [vp, vp, i32, vp, vp, vp, vp, f32, vp, dp, vp]
    lib.pa_prefill.restype = i32
    lib.pa_decode_static_ws.argtypes = [vp, vp, vp, vp, vp, f32, vp, dp, vp]
    lib.pa_decode_static_ws.restype = i32
    lib.pa_test_wait_timeout.argtypes = [ctypes.c_int64, vp]
    lib.pa_test_wait_timeout.restype = i32
    lib.pa_device_errors.argtypes = [ctypes.POINTER(i32), i32]
    lib.pa_device_errors.restype = i32
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()

# Every symbol include/pa.h declares.
EXPORTS = ("pa_cache_append", "pa_decode_workspace_bytes", "pa_decode_default_ctas", "pa_decode",
           "pa_append_decode", "pa_decode_partials", "pa_decode_static_ws",
           "pa_decode_shared_prefix_workspace_bytes", "pa_decode_shared_prefix", "pa_cache_append_fp8",
           "pa_decode_fp8", "pa_append_decode_fp8", "pa_prefill", "pa_test_wait_timeout", "pa_device_errors", "pa_status_string")

PA_ERR_SCRATCH_LIMIT = -7
PA_STATIC_SCRATCH_BYTES = 16 << 20  # include/pa.h


def pa_status_string(code: int) -> str:
    return lib.pa_status_string(int(code)).decode()


def _check(code: int, what: str) -> None:
    if code != 0:
        raise PaError(code, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def make_dims(q: torch.Tensor, k_cache: torch.Tensor, block_tables: torch.Tensor) -> pa_dims:
    """pa_dims from q [B][Hq][D], a cache [NB][Hkv][bs][D] and block_tables [B][M]."""
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or block_tables.shape[0] != B:
        raise ValueError("q, cache and block_tables shapes disagree")
    return pa_dims(B, Hq, Hkv, D, bs, NB, block_tables.shape[1])


def pa_decode_workspace_bytes(dims: pa_dims, num_ctas: int = 0) -> int:
    n = lib.pa_decode_workspace_bytes(ctypes.byref(dims), int(num_ctas))
    if n == 0:
        raise ValueError(f"invalid dims {dims!r}")
    return int(n)


def pa_decode_default_ctas() -> int:
    n = lib.pa_decode_default_ctas()
    if n <= 0:
        raise RuntimeError("no CUDA device")
    return int(n)


def alloc_workspace(dims: pa_dims, num_ctas: int = 0, device=None) -> torch.Tensor:
    """A zero-filled device workspace (the C ABI never allocates)."""
    return torch.zeros(pa_decode_workspace_bytes(dims, num_ctas), dtype=torch.uint8,
                       device=device if device is not None else torch.device("cuda"))


def pa_cache_append(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """k_cache[s // bs][g][s % bs] = k_new[t][g] (v likewise) for s = slot_mapping[t] >= 0."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, torch.bfloat16, n, 3)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n, 4)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    T = slot_mapping.shape[0]
    if k_new.shape != v_new.shape or k_new.shape[0] != T or k_cache.shape != v_cache.shape:
        raise ValueError("append shapes disagree")
    NB, Hkv, bs, D = k_cache.shape
    if k_new.shape[1:] != (Hkv, D):
        raise ValueError("k_new rows must be [Hkv][D] of the cache")
    dims = pa_dims(0, Hkv, Hkv, D, bs, NB, 0)
    _check(lib.pa_cache_append(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(k_cache),
                               _ptr(v_cache), ctypes.byref(dims), _stream(stream)), "pa_cache_append")


def _decode_args(q, k_cache, v_cache, block_tables, context_lens, out):
    _need(q, torch.bfloat16, "q", 3)
    _need(out, torch.bfloat16, "out", 3)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(block_tables, torch.int32, "block_tables", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    if out.shape != q.shape or k_cache.shape != v_cache.shape or context_lens.shape[0] != q.shape[0]:
        raise ValueError("decode shapes disagree")
    return make_dims(q, k_cache, block_tables)


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
              workspace=None, stream=None) -> None:
    """out = paged decode attention (see include/pa.h).  ``workspace`` is a
    zero-initialised uint8 device tensor of pa_decode_workspace_bytes(dims)
    bytes; one is allocated when omitted."""
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    if workspace is None:
        workspace = alloc_workspace(dims, device=q.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(lib.pa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                         _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                         _ptr(workspace), workspace.numel(), _stream(stream)), "pa_decode")


def _append_args(k_new, v_new, slot_mapping, k_cache, v_cache):
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, torch.bfloat16, n, 3)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    T = slot_mapping.shape[0]
    NB, Hkv, bs, D = k_cache.shape
    if k_new.shape != v_new.shape or k_new.shape[0] != T or k_new.shape[1:] != (Hkv, D):
        raise ValueError("k_new/v_new must be [T][Hkv][D] of the cache")
    return T


def pa_append_decode(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens,
                     scale: float, out, workspace=None, stream=None) -> None:
    """One decode step in one launch: append the new K/V rows, then decode
    (see include/pa.h)."""
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    T = _append_args(k_new, v_new, slot_mapping, k_cache, v_cache)
    if workspace is None:
        workspace = alloc_workspace(dims, device=q.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(lib.pa_append_decode(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(q),
                                _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                                float(scale), _ptr(out), ctypes.byref(dims), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "pa_append_decode")


def prepare_append_decode(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens,
                          scale: float, out, workspace, stream=None) -> "Prepared":
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    T = _append_args(k_new, v_new, slot_mapping, k_cache, v_cache)
    _need(workspace, torch.uint8, "workspace", 1)
    p = Prepared(lib.pa_append_decode,
                 (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                  _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                  _ptr(workspace), workspace.numel(), _stream(stream)), "pa_append_decode")
    p._keep = (dims, k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, out,
               workspace)
    return p


def pa_decode_partials(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                       num_ctas: int, workspace, capacity: int, seg_meta, seg_o, seg_m, seg_l,
                       seg_count, stream=None) -> None:
    """Test hook: pa_decode on ``num_ctas`` CTAs that records each segment's
    split-KV partials (see include/pa.h)."""
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    _need(workspace, torch.uint8, "workspace", 1)
    _need(seg_meta, torch.int32, "seg_meta", 2)
    _need(seg_o, torch.float32, "seg_o", 3)
    _need(seg_m, torch.float32, "seg_m", 2)
    _need(seg_l, torch.float32, "seg_l", 2)
    _need(seg_count, torch.int32, "seg_count", 1)
    G = dims.num_q_heads // dims.num_kv_heads
    if seg_meta.shape[0] < capacity or seg_o.shape[0] < capacity or seg_o.shape[1:] != (G, dims.head_dim):
        raise ValueError("segment buffers smaller than capacity")
    _check(lib.pa_decode_partials(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                  _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                                  int(num_ctas), _ptr(workspace), workspace.numel(), int(capacity),
                                  _ptr(seg_meta), _ptr(seg_o), _ptr(seg_m), _ptr(seg_l),
                                  _ptr(seg_count), _stream(stream)), "pa_decode_partials")


def pa_decode_static_ws(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                        stream=None) -> None:
    """pa_decode without a caller workspace: the library's fixed scratch array
    is used instead, so nothing is allocated (for callers that cannot
    allocate device memory where they decode; see include/pa.h)."""
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    _check(lib.pa_decode_static_ws(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                   _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                                   _stream(stream)), "pa_decode_static_ws")


def pa_decode_shared_prefix_workspace_bytes(dims: pa_dims, num_groups: int, max_group_size: int) -> int:
    n = lib.pa_decode_shared_prefix_workspace_bytes(ctypes.byref(dims), int(num_groups), int(max_group_size))
    if n == 0:
        raise ValueError(f"invalid dims {dims!r} / groups ({num_groups}, {max_group_size})")
    return int(n)


def _prefix_args(group_offsets, group_prefix_pages, max_group_size):
    _need(group_offsets, torch.int32, "group_offsets", 1)
    _need(group_prefix_pages, torch.int32, "group_prefix_pages", 1)
    G = group_prefix_pages.shape[0]
    if group_offsets.shape[0] != G + 1:
        raise ValueError("group_offsets must have num_groups + 1 entries")
    if G > 0 and int(max_group_size) <= 0:
        raise ValueError("max_group_size must be positive")
    return G


def _shared_prefix_call(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens,
                        scale, group_offsets, group_prefix_pages, max_group_size, out, workspace, stream):
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    T = 0
    if slot_mapping is not None:
        T = _append_args(k_new, v_new, slot_mapping, k_cache, v_cache)
    ng = _prefix_args(group_offsets, group_prefix_pages, max_group_size)
    if workspace is None:
        workspace = torch.zeros(pa_decode_shared_prefix_workspace_bytes(dims, ng, max_group_size),
                                dtype=torch.uint8, device=q.device)
    _need(workspace, torch.uint8, "workspace", 1)
    args = (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(q), _ptr(k_cache), _ptr(v_cache),
            _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(group_offsets),
            _ptr(group_prefix_pages), ng, int(max_group_size), _ptr(out), ctypes.byref(dims),
            _ptr(workspace), workspace.numel(), _stream(stream))
    keep = (dims, k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens,
            group_offsets, group_prefix_pages, out, workspace)
    return args, keep


def pa_decode_shared_prefix(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                            group_offsets, group_prefix_pages, max_group_size: int, out,
                            k_new=None, v_new=None, slot_mapping=None, workspace=None, stream=None) -> None:
    """Decode of a batch whose groups of consecutive sequences share their
    first blocks: group i = sequences [group_offsets[i], group_offsets[i+1])
    sharing group_prefix_pages[i] blocks (see include/pa.h).  With
    ``slot_mapping`` given, the step's new K/V rows are appended first, in
    the same launch as the decode."""
    args, _ = _shared_prefix_call(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables,
                                  context_lens, scale, group_offsets, group_prefix_pages, max_group_size,
                                  out, workspace, stream)
    _check(lib.pa_decode_shared_prefix(*args), "pa_decode_shared_prefix")


def prepare_decode_shared_prefix(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                 group_offsets, group_prefix_pages, max_group_size: int, out, workspace,
                                 k_new=None, v_new=None, slot_mapping=None, stream=None) -> "Prepared":
    args, keep = _shared_prefix_call(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables,
                                     context_lens, scale, group_offsets, group_prefix_pages,
                                     max_group_size, out, workspace, stream)
    p = Prepared(lib.pa_decode_shared_prefix, args, "pa_decode_shared_prefix")
    p._keep = keep
    return p


# ---- fp8 (E4M3) caches -------------------------------------------------------

def _fp8_cache_args(k_cache8, v_cache8, k_scale, v_scale):
    _need(k_cache8, torch.uint8, "k_cache", 4)
    _need(v_cache8, torch.uint8, "v_cache", 4)
    NB, Hkv, bs, D = k_cache8.shape
    if bs != 16 or tuple(v_cache8.shape) != (NB, Hkv, D, 16):
        raise ValueError("fp8 caches are k [NB][Hkv][16][D] and v [NB][Hkv][D][16] (uint8)")
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, torch.float32, n, 1)
        if t.shape[0] != Hkv:
            raise ValueError(f"{n} must have one scale per kv head")
    return NB, Hkv, D


def pa_cache_append_fp8(k_new, v_new, slot_mapping, k_cache8, v_cache8, k_scale, v_scale, stream=None) -> None:
    """Encode each new bf16 row as E4M3 codes of x / scale[kv head] into its
    slot of the fp8 caches (see include/pa.h for the layouts)."""
    NB, Hkv, D = _fp8_cache_args(k_cache8, v_cache8, k_scale, v_scale)
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, torch.bfloat16, n, 3)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    T = slot_mapping.shape[0]
    if k_new.shape != v_new.shape or k_new.shape[0] != T or k_new.shape[1:] != (Hkv, D):
        raise ValueError("k_new/v_new must be [T][Hkv][D] of the cache")
    dims = pa_dims(0, Hkv, Hkv, D, 16, NB, 0)
    _check(lib.pa_cache_append_fp8(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(k_cache8),
                                   _ptr(v_cache8), _ptr(k_scale), _ptr(v_scale), ctypes.byref(dims),
                                   _stream(stream)), "pa_cache_append_fp8")


def _decode_fp8_args(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, out):
    NB, Hkv, D = _fp8_cache_args(k_cache8, v_cache8, k_scale, v_scale)
    _need(q, torch.bfloat16, "q", 3)
    _need(out, torch.bfloat16, "out", 3)
    _need(block_tables, torch.int32, "block_tables", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    B, Hq, D2 = q.shape
    if D2 != D or out.shape != q.shape or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("decode shapes disagree")
    return pa_dims(B, Hq, Hkv, D, 16, NB, block_tables.shape[1])


def pa_decode_fp8(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, scale: float, out,
                  workspace=None, stream=None) -> None:
    """Paged decode over fp8 (E4M3) caches with per-kv-head scales."""
    dims = _decode_fp8_args(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, out)
    if workspace is None:
        workspace = alloc_workspace(dims, device=q.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(lib.pa_decode_fp8(_ptr(q), _ptr(k_cache8), _ptr(v_cache8), _ptr(k_scale), _ptr(v_scale),
                             _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                             _ptr(workspace), workspace.numel(), _stream(stream)), "pa_decode_fp8")


def _append_decode_fp8_args(k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale, block_tables,
                            context_lens, out):
    dims = _decode_fp8_args(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, out)
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, torch.bfloat16, n, 3)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    T = slot_mapping.shape[0]
    if k_new.shape != v_new.shape or k_new.shape[0] != T or k_new.shape[1:] != (dims.num_kv_heads, dims.head_dim):
        raise ValueError("k_new/v_new must be [T][Hkv][D] of the cache")
    return dims, T


def pa_append_decode_fp8(k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale, block_tables,
                         context_lens, scale: float, out, workspace=None, stream=None) -> None:
    """pa_cache_append_fp8 then pa_decode_fp8, fused into one launch."""
    dims, T = _append_decode_fp8_args(k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale,
                                      block_tables, context_lens, out)
    if workspace is None:
        workspace = alloc_workspace(dims, device=q.device)
    _need(workspace, torch.uint8, "workspace", 1)
    _check(lib.pa_append_decode_fp8(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(q), _ptr(k_cache8),
                                    _ptr(v_cache8), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                    _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims), _ptr(workspace),
                                    workspace.numel(), _stream(stream)), "pa_append_decode_fp8")


def prepare_append_decode_fp8(k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale, block_tables,
                              context_lens, scale: float, out, workspace, stream=None) -> "Prepared":
    dims, T = _append_decode_fp8_args(k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale,
                                      block_tables, context_lens, out)
    _need(workspace, torch.uint8, "workspace", 1)
    p = Prepared(lib.pa_append_decode_fp8,
                 (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(q), _ptr(k_cache8), _ptr(v_cache8),
                  _ptr(k_scale), _ptr(v_scale), _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out),
                  ctypes.byref(dims), _ptr(workspace), workspace.numel(), _stream(stream)), "pa_append_decode_fp8")
    p._keep = (dims, k_new, v_new, slot_mapping, q, k_cache8, v_cache8, k_scale, v_scale, block_tables,
               context_lens, out, workspace)
    return p


def prepare_append_fp8(k_new, v_new, slot_mapping, k_cache8, v_cache8, k_scale, v_scale, stream=None) -> "Prepared":
    NB, Hkv, D = _fp8_cache_args(k_cache8, v_cache8, k_scale, v_scale)
    dims = pa_dims(0, Hkv, Hkv, D, 16, NB, 0)
    p = Prepared(lib.pa_cache_append_fp8,
                 (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), slot_mapping.shape[0], _ptr(k_cache8),
                  _ptr(v_cache8), _ptr(k_scale), _ptr(v_scale), ctypes.byref(dims), _stream(stream)),
                 "pa_cache_append_fp8")
    p._keep = (dims, k_new, v_new, slot_mapping, k_cache8, v_cache8, k_scale, v_scale)
    return p


def prepare_decode_fp8(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, scale: float, out,
                       workspace, stream=None) -> "Prepared":
    dims = _decode_fp8_args(q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, out)
    _need(workspace, torch.uint8, "workspace", 1)
    p = Prepared(lib.pa_decode_fp8,
                 (_ptr(q), _ptr(k_cache8), _ptr(v_cache8), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                  _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims), _ptr(workspace),
                  workspace.numel(), _stream(stream)), "pa_decode_fp8")
    p._keep = (dims, q, k_cache8, v_cache8, k_scale, v_scale, block_tables, context_lens, out, workspace)
    return p


def _prefill_args(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, out):
    _need(q, torch.bfloat16, "q", 3)
    _need(out, torch.bfloat16, "out", 3)
    _need(cu_q_lens, torch.int32, "cu_q_lens", 1)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(block_tables, torch.int32, "block_tables", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    B = block_tables.shape[0]
    if out.shape != q.shape or cu_q_lens.shape[0] != B + 1 or context_lens.shape[0] != B or \
            k_cache.shape != v_cache.shape or k_cache.shape[3] != q.shape[2]:
        raise ValueError("prefill shapes disagree")
    NB, Hkv, bs, D = k_cache.shape
    return pa_dims(B, q.shape[1], Hkv, D, bs, NB, block_tables.shape[1])


def pa_prefill(q, cu_q_lens, max_q_len: int, k_cache, v_cache, block_tables, context_lens, scale: float, out,
               stream=None) -> None:
    """Multi-query (chunked prefill) attention over the paged cache: the
    rows cu_q_lens[b] .. cu_q_lens[b+1]-1 of q are the last tokens of
    sequence b's context and attend causally (see include/pa.h)."""
    dims = _prefill_args(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, out)
    _check(lib.pa_prefill(_ptr(q), _ptr(cu_q_lens), int(max_q_len), _ptr(k_cache), _ptr(v_cache),
                          _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims),
                          _stream(stream)), "pa_prefill")


def prepare_prefill(q, cu_q_lens, max_q_len: int, k_cache, v_cache, block_tables, context_lens, scale: float,
                    out, stream=None) -> "Prepared":
    dims = _prefill_args(q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, out)
    p = Prepared(lib.pa_prefill,
                 (_ptr(q), _ptr(cu_q_lens), int(max_q_len), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                  _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(dims), _stream(stream)), "pa_prefill")
    p._keep = (dims, q, cu_q_lens, k_cache, v_cache, block_tables, context_lens, out)
    return p


def pa_test_wait_timeout(limit_ns: int, stream=None) -> None:
    """Test hook: one CTA whose bounded waits run out after limit_ns each
    (they set PA_DEVERR_TIMEOUT and return); see include/pa.h."""
    _check(lib.pa_test_wait_timeout(int(limit_ns), _stream(stream)), "pa_test_wait_timeout")


def pa_device_errors(clear: bool = False) -> int:
    """PA_DEVERR_* bits set on the current device since the last clear (synchronises)."""
    v = ctypes.c_int32(0)
    _check(lib.pa_device_errors(ctypes.byref(v), int(bool(clear))), "pa_device_errors")
    return int(v.value)


class Prepared:
    """A pa_cache_append / pa_decode call with its arguments marshalled
    once: calling it re-issues the same C call on the same tensors (their
    contents may change between calls, their storage may not).  Used where
    per-call Python overhead would otherwise leave the GPU idle."""

    def __init__(self, fn, args, what):
        self._fn, self._args, self._what, self._keep = fn, args, what, None

    def __call__(self):
        code = self._fn(*self._args)
        if code != 0:
            raise PaError(code, self._what)


def prepare_append(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None) -> Prepared:
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, torch.bfloat16, n, 3)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n, 4)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    NB, Hkv, bs, D = k_cache.shape
    dims = pa_dims(0, Hkv, Hkv, D, bs, NB, 0)
    p = Prepared(lib.pa_cache_append,
                 (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), slot_mapping.shape[0], _ptr(k_cache),
                  _ptr(v_cache), ctypes.byref(dims), _stream(stream)), "pa_cache_append")
    p._keep = (dims, k_new, v_new, slot_mapping, k_cache, v_cache)
    return p


def prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out, workspace,
                   stream=None) -> Prepared:
    dims = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    _need(workspace, torch.uint8, "workspace", 1)
    p = Prepared(lib.pa_decode,
                 (_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                  float(scale), _ptr(out), ctypes.byref(dims), _ptr(workspace), workspace.numel(),
                  _stream(stream)), "pa_decode")
    p._keep = (dims, q, k_cache, v_cache, block_tables, context_lens, out, workspace)
    return p
