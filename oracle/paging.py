"""Paged cache layout: where a token's stored rows live in a block pool.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

[inferrs] "二、inferrs：TurboQuant 轻量推理服务器" manages the compressed cache
with PagedAttention but gives no page format.  The reading adopted: a pool
of fixed-size blocks, each array laid out [block][Hkv][block_size][...] like
a contiguous cache whose "batch" counts blocks; an int32 table
[batch][max_blocks] names, for sequence b, the block holding its tokens
[j * block_size, (j + 1) * block_size).  What is stored per token, and what
attention computes from it, does not change.

``gather`` reads one (sequence, kv head) token by token, which is the
definition; ``scatter`` writes a contiguous run block by block (the inverse,
written as slices), so a round trip through both pins each against the other.
"""

import numpy as np


def gather(pool, table, block_size, b, h, n):
    """Rows of tokens 0 .. n-1 of sequence b, kv head h: pool [blocks][Hkv][block_size][...]
    and table [batch][max_blocks] (any integer array).  A token whose block is
    outside the pool raises ValueError."""
    pool = np.asarray(pool)
    rows = []
    for t in range(n):
        blk = int(table[b][t // block_size])
        if not 0 <= blk < pool.shape[0]:
            raise ValueError("token %d of sequence %d: block %d outside the pool" % (t, b, blk))
        rows.append(pool[blk, h, t % block_size])
    return np.stack(rows) if rows else pool[:0, h, :0].reshape((0,) + pool.shape[3:])


def scatter(pool, table, block_size, b, h, rows):
    """Write rows [n][...] as tokens 0 .. n-1 of sequence b, kv head h into pool
    (in place), one block-sized slice at a time."""
    rows = np.asarray(rows)
    n = rows.shape[0]
    for j in range((n + block_size - 1) // block_size):
        blk = int(table[b][j])
        if not 0 <= blk < pool.shape[0]:
            raise ValueError("block %d of sequence %d: %d outside the pool" % (j, b, blk))
        seg = rows[j * block_size:(j + 1) * block_size]
        pool[blk, h, :seg.shape[0]] = seg
    return pool
