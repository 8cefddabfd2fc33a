"""The paged-cache layout in the oracle, pinned by a round trip, and the GPU
tests' gather helper checked against it (CPU only).

``oracle.paging.gather`` reads token by token; ``oracle.paging.scatter``
writes block-sized slices.  Writing sequences through random block tables
and reading them back must return them exactly, leave blocks no table names
untouched, and refuse a token whose block is outside the pool."""

import types

import numpy as np
import pytest
import torch

from bit_kv_cache_tq_b200 import tq
from oracle import paging


@pytest.mark.parametrize("bs,lens", [(16, [1, 16, 17, 100]), (48, [47, 48, 49, 300]), (256, [5, 700])])
def test_scatter_then_gather_round_trip(bs, lens):
    rng = np.random.default_rng(bs)
    hkv, width = 3, 5
    max_blocks = max((n + bs - 1) // bs for n in lens)
    num_blocks = len(lens) * max_blocks + 4
    table = rng.permutation(num_blocks)[: len(lens) * max_blocks].reshape(len(lens), max_blocks)
    pool = rng.integers(0, 256, size=(num_blocks, hkv, bs, width), dtype=np.int64)
    before = pool.copy()
    seqs = {(b, h): rng.integers(0, 256, size=(n, width)) for b, n in enumerate(lens) for h in range(hkv)}
    for (b, h), rows in seqs.items():
        paging.scatter(pool, table, bs, b, h, rows)
    for (b, h), rows in seqs.items():
        assert np.array_equal(paging.gather(pool, table, bs, b, h, rows.shape[0]), rows)
    # blocks no table names are untouched
    named = set(int(x) for b, n in enumerate(lens) for x in table[b][: (n + bs - 1) // bs])
    for blk in range(num_blocks):
        if blk not in named:
            assert np.array_equal(pool[blk], before[blk])


def test_gather_refuses_a_block_outside_the_pool():
    pool = np.zeros((4, 1, 16, 2))
    table = np.array([[2, -1, 3]])
    assert paging.gather(pool, table, 16, 0, 0, 16).shape == (16, 2)
    with pytest.raises(ValueError):
        paging.gather(pool, table, 16, 0, 0, 17)
    with pytest.raises(ValueError):
        paging.gather(pool, np.array([[4]]), 16, 0, 0, 1)


def test_gpu_tests_gather_helper_matches_the_oracle():
    """The tensor gather the paged GPU tests compare with (run here on CPU
    tensors) reads the same rows as the oracle's definition."""
    from test_gpu_paged import _gather
    rng = np.random.default_rng(5)
    hkv, bs, lens = 2, 16, [40, 7]
    max_blocks = 4
    num_blocks = len(lens) * max_blocks + 2
    table = rng.permutation(num_blocks)[: len(lens) * max_blocks].reshape(len(lens), max_blocks).astype(np.int32)
    for b, n in enumerate(lens):
        table[b, (n + bs - 1) // bs:] = -1

    def arr(*tail, dtype=torch.uint8):
        hi = 256 if dtype == torch.uint8 else 1 << 15
        return torch.from_numpy(rng.integers(0, hi, size=(num_blocks, hkv, bs) + tail)).to(dtype)

    pool = tq.CacheTensors(num_blocks, bs, arr(64), arr(dtype=torch.int16), arr(8), arr(dtype=torch.int16),
                           arr(32), arr(dtype=torch.int16), None)
    got = _gather(types.SimpleNamespace(hkv=hkv), pool, torch.from_numpy(table), max_blocks * bs)
    for name in ("k_codes", "k_norms", "k_qjl", "k_gamma", "v_codes", "v_norms"):
        for b, n in enumerate(lens):
            for h in range(hkv):
                want = paging.gather(getattr(pool, name).numpy(), table, bs, b, h, n)
                assert np.array_equal(getattr(got, name)[b, h, :n].numpy(), want), (name, b, h)
