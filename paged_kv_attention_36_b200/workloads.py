"""Seeded synthetic decode batches shaped like the pages' workloads.

This module only draws random inputs and builds block tables and slot
mappings (the bookkeeping a serving engine's block manager hands to the
kernels).  It holds none of the attention arithmetic, and it is shared by
the CUDA path's tests and bench and by the oracle's tests.

The pages measure on no public suite and print no tensors: miniVLLM's demo
runs a randomly initialised Qwen3 on two prompts repeated thirty times and
decodes up to 256 tokens (miniVLLM review, "What main.py actually does");
mini-sglang serves Qwen3-0.6B; tiny-vllm runs Llama 3.2 1B (tiny-vllm
write-up, "Diem noi bat").  The configurations below stand in for those
decode batches with their attention shapes (heads, head_dim, GQA group),
block size 16 and seeded N(0, 1) bf16 values.

All tensors are created on the CPU with a seeded ``torch.Generator``; the
caller moves them to a device.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BF16_NAN_BITS = 0x7FC0          # quiet NaN in bf16
POISON_BLOCK_ID = 0x7FFFFFFF    # block-table padding that must never be read


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int = 16
    description: str = ""


SPECS = {
    "tiny": WorkloadSpec(
        "tiny", 36000, 4, 8, 2, 64,
        description="batch 4, 8 q / 2 kv heads, head_dim 64, block 16, context_lens U[1,100], "
                    "64-block pool, block ids a seeded permutation, append 1 token/seq"),
    "qwen3": WorkloadSpec(
        "qwen3", 36001, 60, 16, 8, 128,
        description="Qwen3-0.6B-shaped decode: batch 60 (2 prompts x 30, no shared blocks), "
                    "16 q / 8 kv heads, head_dim 128, context_lens U[20,300], shuffled pool"),
    "llama32": WorkloadSpec(
        "llama32", 36002, 128, 32, 8, 64,
        description="Llama-3.2-1B-shaped decode: batch 128, 32 q / 8 kv heads, head_dim 64, "
                    "context_lens U[512,4096], blocks scattered over a pool 1.5x the need"),
    "longskew": WorkloadSpec(
        "longskew", 36003, 64, 32, 8, 128,
        description="long/skewed split-KV: 32 q / 8 kv heads, head_dim 128, one 131072-token "
                    "sequence and 63 of 1024, 1% outlier keys x8, shuffled pool"),
    "prefix": WorkloadSpec(
        "prefix", 36004, 256, 16, 8, 128,
        description="prefix-shared pages: batch 256, 16 q / 8 kv heads, head_dim 128, two "
                    "1024-token prefixes shared by 128 seqs each, private suffixes U[0,256], "
                    "append 1 token/seq then decode"),
}


@dataclasses.dataclass
class Workload:
    spec: WorkloadSpec
    q: torch.Tensor             # [B][Hq][D] bf16
    k_cache: torch.Tensor       # [NB][Hkv][bs][D] bf16
    v_cache: torch.Tensor       # [NB][Hkv][bs][D] bf16
    block_tables: torch.Tensor  # [B][M] int32
    context_lens: torch.Tensor  # [B] int32 (decode length, appended token included)
    k_new: torch.Tensor         # [B][Hkv][D] bf16: the token appended this step
    v_new: torch.Tensor         # [B][Hkv][D] bf16
    slot_mapping: torch.Tensor  # [B] int32: slot of position context_len - 1
    scale: float
    # shared prefixes: group i = sequences [group_offsets[i], group_offsets[i+1])
    # whose tables begin with the same group_prefix_pages[i] blocks
    group_offsets: torch.Tensor = None       # [num_groups + 1] int32
    group_prefix_pages: torch.Tensor = None  # [num_groups] int32

    @property
    def num_groups(self) -> int:
        return 0 if self.group_prefix_pages is None else int(self.group_prefix_pages.shape[0])

    @property
    def max_group_size(self) -> int:
        if self.num_groups == 0:
            return 0
        return int((self.group_offsets[1:] - self.group_offsets[:-1]).max().item())

    @property
    def dims(self):
        B, Hq, D = self.q.shape
        NB, Hkv, bs, _ = self.k_cache.shape
        return dict(num_seqs=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                    block_size=bs, num_blocks=NB, max_blocks_per_seq=self.block_tables.shape[1])


def _randn_bf16(gen: torch.Generator, shape) -> torch.Tensor:
    # fp32 N(0,1) draws rounded to nearest-even bf16
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def _pages(n_tokens: torch.Tensor, bs: int) -> torch.Tensor:
    return (n_tokens + bs - 1) // bs


def build_tables(block_lists, max_blocks: int) -> torch.Tensor:
    """Pack per-sequence lists of physical block ids into a [B][M] int32
    table padded with POISON_BLOCK_ID."""
    bt = torch.full((len(block_lists), max_blocks), POISON_BLOCK_ID, dtype=torch.int32)
    for b, ids in enumerate(block_lists):
        if len(ids):
            bt[b, :len(ids)] = torch.as_tensor(ids, dtype=torch.int32)
    return bt


def slots_for_positions(block_tables: torch.Tensor, positions: torch.Tensor, bs: int) -> torch.Tensor:
    """Slot of token position p of sequence b: block_tables[b][p // bs] * bs + p % bs
    (-1 where p < 0).  This is the slot mapping a block manager passes to the
    append."""
    B = positions.shape[0]
    pos = positions.to(torch.int64)
    valid = pos >= 0
    safe = torch.where(valid, pos, torch.zeros_like(pos))
    blk = block_tables.to(torch.int64)[torch.arange(B), safe // bs]
    slots = blk * bs + safe % bs
    return torch.where(valid, slots, torch.full_like(slots, -1)).to(torch.int32)


def make(name: str, *, poison: bool = False, seed: int | None = None,
         context_lens=None, num_seqs: int | None = None) -> Workload:
    """Build configuration ``name``.  ``poison`` fills every cache row no
    sequence reads with bf16 NaN, so any read past a context shows up.
    ``context_lens`` / ``num_seqs`` override the drawn lengths (edge cases)."""
    spec = SPECS[name]
    g = torch.Generator().manual_seed(spec.seed if seed is None else seed)
    B = spec.num_seqs if num_seqs is None else num_seqs
    Hq, Hkv, D, bs = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size

    shared_prefix_blocks = 0
    if context_lens is not None:
        lens = torch.as_tensor(context_lens, dtype=torch.int64)
        B = lens.shape[0]
    elif name == "tiny":
        lens = torch.randint(1, 101, (B,), generator=g, dtype=torch.int64)
    elif name == "qwen3":
        lens = torch.randint(20, 301, (B,), generator=g, dtype=torch.int64)
    elif name == "llama32":
        lens = torch.randint(512, 4097, (B,), generator=g, dtype=torch.int64)
    elif name == "longskew":
        lens = torch.full((B,), 1024, dtype=torch.int64)
        lens[0] = 131072
    elif name == "prefix":
        suffix = torch.randint(0, 257, (B,), generator=g, dtype=torch.int64)
        lens = 1024 + suffix + 1          # shared prefix + private suffix + appended token
        shared_prefix_blocks = 1024 // bs
    else:
        raise KeyError(name)

    pages = _pages(lens, bs)
    M = max(1, int(pages.max().item()) if B else 1)

    # ---- physical block assignment ------------------------------------
    if name == "prefix" and context_lens is None:
        n_groups = 2
        private = (pages - shared_prefix_blocks).clamp(min=0)
        need = n_groups * shared_prefix_blocks + int(private.sum().item())
        NB = need
        perm = torch.randperm(NB, generator=g).tolist()
        prefix_ids = [perm[i * shared_prefix_blocks:(i + 1) * shared_prefix_blocks]
                      for i in range(n_groups)]
        cursor = n_groups * shared_prefix_blocks
        lists = []
        for b in range(B):
            grp = 0 if b < B // 2 else 1
            n_priv = int(private[b].item())
            lists.append(prefix_ids[grp] + perm[cursor:cursor + n_priv])
            cursor += n_priv
    else:
        need = int(pages.sum().item())
        if name == "tiny" and context_lens is None:
            NB = 64
        elif name == "llama32":
            NB = int(math.ceil(1.5 * need))
        else:
            NB = max(need, 1)
        perm = torch.randperm(NB, generator=g).tolist()
        lists, cursor = [], 0
        for b in range(B):
            n = int(pages[b].item())
            lists.append(perm[cursor:cursor + n])
            cursor += n
    block_tables = build_tables(lists, M)
    w = _fill(spec, g, lens, lists, block_tables, NB, poison)
    if name == "prefix" and context_lens is None:
        w.group_offsets = torch.tensor([0, B // 2, B], dtype=torch.int32)
        w.group_prefix_pages = torch.tensor([shared_prefix_blocks] * 2, dtype=torch.int32)
    return w


def _fill(spec: WorkloadSpec, g: torch.Generator, lens: torch.Tensor, lists, block_tables: torch.Tensor,
          NB: int, poison: bool, num_seqs: int | None = None) -> Workload:
    """Draws q, the caches and the appended rows for a batch whose tables are
    built, poisons unread rows if asked, and derives the slot mapping."""
    B = lens.shape[0]
    Hq, Hkv, D, bs = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    name = spec.name

    # ---- values ----------------------------------------------------------
    q = _randn_bf16(g, (B, Hq, D))
    k_cache = _randn_bf16(g, (NB, Hkv, bs, D))
    v_cache = _randn_bf16(g, (NB, Hkv, bs, D))
    if name == "longskew":
        # 1% of (token row, kv head) keys scaled by 8 (a power of two: exact in bf16)
        outlier = torch.rand((NB, Hkv, bs), generator=g) < 0.01
        k_cache = torch.where(outlier[..., None], k_cache * 8, k_cache)
    k_new = _randn_bf16(g, (B, Hkv, D))
    v_new = _randn_bf16(g, (B, Hkv, D))

    if poison:
        used = torch.zeros((NB, bs), dtype=torch.bool)
        for b in range(B):
            L = int(lens[b].item())
            for j, blk in enumerate(lists[b]):
                n_valid = min(bs, L - j * bs)
                used[blk, :n_valid] = True
        nan = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)
        mask = (~used)[:, None, :, None].expand(NB, Hkv, bs, D)
        k_cache = torch.where(mask, nan, k_cache)
        v_cache = torch.where(mask, nan, v_cache)

    slot_mapping = slots_for_positions(block_tables, lens - 1, bs)
    return Workload(spec=spec, q=q, k_cache=k_cache.contiguous(), v_cache=v_cache.contiguous(),
                    block_tables=block_tables, context_lens=lens.to(torch.int32),
                    k_new=k_new, v_new=v_new, slot_mapping=slot_mapping,
                    scale=1.0 / math.sqrt(D))


def unique_kv_bytes(w: Workload) -> int:
    """Bytes of distinct K and V rows the decode must read: each physical
    (block, offset) row inside some context counts once per kv head."""
    bs = w.spec.block_size
    D = w.q.shape[2]
    NB, Hkv = w.k_cache.shape[0], w.k_cache.shape[1]
    used = torch.zeros(NB * bs, dtype=torch.bool)
    for b, L in enumerate(w.context_lens.tolist()):
        if L <= 0:
            continue
        t = torch.arange(L)
        blk = w.block_tables[b, t // bs].to(torch.int64)
        used[blk * bs + t % bs] = True
    return int(used.sum().item()) * Hkv * D * 2 * 2


def logical_kv_bytes(w: Workload) -> int:
    """K and V bytes summed over sequences (shared rows counted per reader)."""
    D = w.q.shape[2]
    Hkv = w.k_cache.shape[1]
    return int(w.context_lens.to(torch.int64).sum().item()) * Hkv * D * 2 * 2


def qo_bytes(w: Workload) -> int:
    """q read plus out written, bf16."""
    return 2 * w.q.numel() * 2


def append_bytes(w: Workload) -> int:
    """k_new/v_new read, their cache rows written, slot ids read."""
    n_valid = int((w.slot_mapping >= 0).sum().item())
    per_tok = w.k_new.shape[1] * w.k_new.shape[2] * 2 * 2
    return 2 * n_valid * per_tok + 4 * w.slot_mapping.numel()


def make_grouped(name: str, groups, suffix_lens, *, tail_lens=(), seed: int | None = None,
                 poison: bool = False, heads=None) -> Workload:
    """A batch with the head shapes of configuration ``name`` in which runs of
    consecutive sequences share their first blocks, as prefix caching
    leaves them.  ``groups`` = [(members, prefix_pages), ...]; member b of
    the groups has context prefix_pages * bs + suffix_lens[b] (0 makes the
    whole context the shared prefix); then one sequence in no group per
    entry of ``tail_lens``.  Block ids are a seeded permutation of a pool
    that holds exactly the needed blocks.  ``heads`` = (Hq, Hkv, D)
    overrides the configuration's head shapes."""
    spec = SPECS[name]
    if heads is not None:
        spec = dataclasses.replace(spec, num_q_heads=heads[0], num_kv_heads=heads[1], head_dim=heads[2])
    g = torch.Generator().manual_seed(spec.seed + 1000 if seed is None else seed)
    bs = spec.block_size
    n_members = sum(m for m, _ in groups)
    if len(suffix_lens) != n_members:
        raise ValueError("one suffix length per group member")
    lens, prefix_of = [], []
    for gi, (m, P) in enumerate(groups):
        for _ in range(m):
            prefix_of.append(gi)
    for b, sfx in enumerate(suffix_lens):
        lens.append(groups[prefix_of[b]][1] * bs + int(sfx))
    lens += [int(L) for L in tail_lens]
    lens_t = torch.tensor(lens, dtype=torch.int64)
    pages = _pages(lens_t, bs)
    private = [int(pages[b]) - (groups[prefix_of[b]][1] if b < n_members else 0) for b in range(len(lens))]
    NB = max(1, sum(P for _, P in groups) + sum(private))
    perm = torch.randperm(NB, generator=g).tolist()
    cursor, prefix_ids = 0, []
    for _, P in groups:
        prefix_ids.append(perm[cursor:cursor + P])
        cursor += P
    lists = []
    for b in range(len(lens)):
        shared = prefix_ids[prefix_of[b]] if b < n_members else []
        lists.append(shared + perm[cursor:cursor + private[b]])
        cursor += private[b]
    M = max(1, int(pages.max().item()) if len(lens) else 1)
    w = _fill(spec, g, lens_t, lists, build_tables(lists, M), NB, poison)
    offsets = [0]
    for m, _ in groups:
        offsets.append(offsets[-1] + m)
    w.group_offsets = torch.tensor(offsets, dtype=torch.int32)
    w.group_prefix_pages = torch.tensor([P for _, P in groups], dtype=torch.int32)
    return w


@dataclasses.dataclass
class PrefillBatch:
    """A chunked-prefill batch: sequence b's last q_len[b] cached tokens are
    its queries, rows cu_q_lens[b] .. cu_q_lens[b+1]-1 of q."""
    q: torch.Tensor             # [total][Hq][D] bf16
    cu_q_lens: torch.Tensor     # [B + 1] int32
    k_cache: torch.Tensor       # [NB][Hkv][16][D] bf16
    v_cache: torch.Tensor
    block_tables: torch.Tensor  # [B][M] int32
    context_lens: torch.Tensor  # [B] int32 (prior context + the chunk)
    scale: float
    description: str

    @property
    def max_q_len(self) -> int:
        return int((self.cu_q_lens[1:] - self.cu_q_lens[:-1]).max().item())


def make_prefill(name: str = "llama32", num_seqs: int = 16, chunk: int = 512, prior=(512, 3584),
                 seed: int | None = None) -> PrefillBatch:
    """Chunked prefill with the head shapes of configuration `name`: each of
    `num_seqs` sequences has a prior context U[prior] and a new chunk of
    `chunk` tokens (cached already), blocks scattered over a shuffled pool."""
    spec = SPECS[name]
    g = torch.Generator().manual_seed((spec.seed + 2000) if seed is None else seed)
    Hq, Hkv, D, bs = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    prior_lens = torch.randint(prior[0], prior[1] + 1, (num_seqs,), generator=g, dtype=torch.int64)
    lens = prior_lens + chunk
    pages = _pages(lens, bs)
    NB = int(pages.sum().item())
    perm = torch.randperm(NB, generator=g).tolist()
    lists, cursor = [], 0
    for b in range(num_seqs):
        n = int(pages[b].item())
        lists.append(perm[cursor:cursor + n])
        cursor += n
    bt = build_tables(lists, int(pages.max().item()))
    k_cache = _randn_bf16(g, (NB, Hkv, bs, D))
    v_cache = _randn_bf16(g, (NB, Hkv, bs, D))
    q = _randn_bf16(g, (num_seqs * chunk, Hq, D))
    cu = torch.arange(0, num_seqs + 1, dtype=torch.int32) * chunk
    desc = (f"chunked prefill, {spec.name} heads ({Hq} q / {Hkv} kv, head_dim {D}): {num_seqs} sequences, "
            f"{chunk}-token chunks after prior contexts U[{prior[0]},{prior[1]}], causal, block 16")
    return PrefillBatch(q=q, cu_q_lens=cu, k_cache=k_cache, v_cache=v_cache, block_tables=bt,
                        context_lens=lens.to(torch.int32), scale=1.0 / math.sqrt(D), description=desc)


def prefill_flops(b: PrefillBatch) -> int:
    """Multiply-adds x 2 of QK and PV: 4 * D flops per (query row, visible key)."""
    Hq, D = b.q.shape[1], b.q.shape[2]
    total = 0
    for i in range(b.cu_q_lens.shape[0] - 1):
        n = int(b.cu_q_lens[i + 1] - b.cu_q_lens[i])
        L = int(b.context_lens[i])
        # query j sees L - n + j + 1 keys
        total += n * (L - n + 1) + n * (n - 1) // 2
    return 4 * D * Hq * total
