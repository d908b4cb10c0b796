"""Test-side helpers: build paged pools from contiguous K/V (the documented
cache layout, cache[block][kv_head][offset][d]), and convert bf16 tensors
to and from their uint16 bit patterns for the oracle."""
from __future__ import annotations

import numpy as np
import torch

NAN_BITS = 0x7FC0
PAD_BLOCK = 0x7FFFFFFF


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy view of its bit patterns."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def page(planes, lens, bs: int, num_blocks: int, gen: torch.Generator, poison: bool = True):
    """Scatter per-sequence contiguous caches into paged pools that share
    one random block table.

    planes: list of per-sequence lists, planes[p][b] is [Hkv][L_b][D] bf16
    (e.g. planes = [K_seqs, V_seqs]).  Returns (pools, block_tables) with
    pools[p] of shape [NB][Hkv][bs][D]; unused rows are NaN when
    ``poison`` and unused table entries are PAD_BLOCK."""
    B = len(lens)
    Hkv, _, D = planes[0][0].shape
    pages = [(L + bs - 1) // bs for L in lens]
    M = max(1, max(pages) if pages else 1)
    assert sum(pages) <= num_blocks
    perm = torch.randperm(num_blocks, generator=gen).tolist()
    pools = []
    for _ in planes:
        pool = torch.zeros((num_blocks, Hkv, bs, D), dtype=torch.bfloat16)
        if poison:
            pool.view(torch.int16).fill_(NAN_BITS)
        pools.append(pool)
    bt = torch.full((B, M), PAD_BLOCK, dtype=torch.int32)
    cur = 0
    for b in range(B):
        for j in range(pages[b]):
            blk = perm[cur]
            cur += 1
            bt[b, j] = blk
            t0, t1 = j * bs, min(lens[b], (j + 1) * bs)
            for pool, seqs in zip(pools, planes):
                pool[blk, :, : t1 - t0, :] = seqs[b][:, t0:t1, :]
    return pools, bt


def contiguous(pool: torch.Tensor, bt: torch.Tensor, b: int, L: int) -> torch.Tensor:
    """[Hkv][L][D] rows of sequence b read back through its block table."""
    bs = pool.shape[2]
    if L == 0:
        return pool.new_zeros((pool.shape[1], 0, pool.shape[3]))
    rows = [pool[int(bt[b, t // bs]), :, t % bs, :] for t in range(L)]
    return torch.stack(rows, dim=1)


def random_seqs(gen, lens, Hkv, D):
    return [torch.randn((Hkv, L, D), generator=gen).to(torch.bfloat16) for L in lens]
