"""Paged (block-table) cache through the C ABI.

A paged pool holds each sequence's tokens in blocks named by a block table,
[block][Hkv][block_size][...].  Gathering a sequence's blocks in table order
must give exactly the bytes a contiguous cache holds for the same inputs, and
decode attention over the pool must equal decode attention over the
contiguous cache (same kernel arithmetic on the same staged bytes) and the
oracle on the stored codes.  Tables are random permutations of the pool, with
blocks past a sequence's end left unmapped (-1) where the case allows."""

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq

pytestmark = pytest.mark.gpu


def _np64(x):
    return x.float().cpu().numpy().astype(np.float64)


def _table(bsz, max_blocks, bs, lens, seed, unmap_tail=True, spare=3):
    """A random block table; blocks at or past ceil(len / bs) are -1 when unmap_tail."""
    rng = np.random.default_rng(seed)
    num_blocks = bsz * max_blocks + spare
    perm = rng.permutation(num_blocks)[: bsz * max_blocks].reshape(bsz, max_blocks).astype(np.int32)
    if unmap_tail:
        for b, n in enumerate(lens):
            perm[b, (n + bs - 1) // bs:] = -1
    return torch.from_numpy(perm).cuda(), num_blocks


def _gather(layer, pool, table, cap):
    """The pool's blocks in table order as a contiguous cache [B][Hkv][cap]."""
    t = table.long().clamp(min=0)  # unmapped blocks gather block 0 (never compared)
    bsz, max_blocks = t.shape

    def g(x):
        if x is None:
            return None
        y = x[t]  # [B, max_blocks, Hkv, bs, ...]
        y = y.transpose(1, 2)  # [B, Hkv, max_blocks, bs, ...]
        return y.reshape(bsz, layer.hkv, max_blocks * pool.capacity, *x.shape[3:]).contiguous()

    return tq.CacheTensors(bsz, cap, g(pool.k_codes), g(pool.k_norms), g(pool.k_qjl), g(pool.k_gamma),
                           g(pool.v_codes), g(pool.v_norms), pool.qjl_matrix)


def _paged_prefill(layer, k, v, lens, bs, seed, unmap_tail=True):
    """Quantise the first lens[b] tokens of k, v ([B, T, Hkv, d]) of every
    sequence into a paged pool: one batch-1 call per sequence on its table row."""
    bsz = k.shape[0]
    max_blocks = (max(lens) + bs - 1) // bs + 1
    table, num_blocks = _table(bsz, max_blocks, bs, lens, seed, unmap_tail)
    pool = tq.alloc_cache(layer.params, num_blocks, bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b, n in enumerate(lens):
        tq.tq_quantize_append_paged(layer.params, layer.kcb, layer.vcb, k[b:b + 1, :n].cuda().contiguous(),
                                    v[b:b + 1, :n].cuda().contiguous(), zero, pool, table[b:b + 1], err)
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK and word == 0
    return pool, table, max_blocks * bs


def _contig_prefill(layer, k, v, lens, cap):
    """The same tokens into a contiguous cache (all T tokens written; only the
    first lens[b] are compared or attended)."""
    cache, st, word = H.gpu_quantize(layer, k, v, cap)
    assert st == tq.TQ_OK and word == 0
    return cache


def _assert_same_bytes(paged, contig, lens):
    for name in ("k_codes", "k_norms", "k_qjl", "k_gamma", "v_codes", "v_norms"):
        a, b = getattr(paged, name), getattr(contig, name)
        if a is None:
            continue
        for s, n in enumerate(lens):
            assert torch.equal(a[s, :, :n].cpu(), b[s, :, :n].cpu()), (name, s)


def _decode(layer, fn, q, store, table, lens, max_len):
    bsz = q.shape[0]
    ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, bsz, max_len), dtype=torch.uint8, device="cuda")
    out = torch.empty(bsz, layer.hq, layer.d, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    if table is None:
        fn(layer.params, layer.kcb, layer.vcb, q.cuda(), store, lens_t, max_len, out, ws, err)
    else:
        fn(layer.params, layer.kcb, layer.vcb, q.cuda(), store, table, lens_t, max_len, out, ws, err)
    st, word = tq.tq_read_device_error(err)
    return out.cpu().numpy(), st, word


CASES = {
    "k4v2_bs16": (dict(k_bits=4, v_bits=2), 32, 16),
    "k4v2_bs64": (dict(k_bits=4, v_bits=2), 32, 64),
    "k3qjl_v2_bs256_g8": (dict(k_bits=3, v_bits=2, qjl_dims=64), 64, 256),
    "int8k_v2_bs48": (dict(k_mode=tq.TQ_MODE_INT8, v_bits=2), 32, 48),
    "int8kv_bs128": (dict(k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8), 32, 128),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_paged_matches_contiguous_and_oracle(case):
    kw, hq, bs = CASES[case]
    layer = H.Layer(128, hq, 8, seed=21, **kw)
    lens = [1500, 777, 33]
    t = max(lens)
    k = inputs.lognormal_kv(len(lens), t, 8, 128, seed=21, layer=5, which=inputs.K)
    v = inputs.lognormal_kv(len(lens), t, 8, 128, seed=21, layer=5, which=inputs.V)
    q = inputs.queries(len(lens), hq, 128, seed=21, layer=5)
    pool, table, cap = _paged_prefill(layer, k, v, lens, bs, seed=21)
    contig = _contig_prefill(layer, k, v, lens, cap)
    gathered = _gather(layer, pool, table, cap)
    _assert_same_bytes(gathered, contig, lens)
    got, st, word = _decode(layer, tq.tq_decode_attention_paged, q, pool, table, lens, cap)
    assert st == tq.TQ_OK and word == 0
    want, st, word = _decode(layer, tq.tq_decode_attention, q, contig, None, lens, cap)
    assert st == tq.TQ_OK and word == 0
    assert np.array_equal(got, want)
    for b, n in enumerate(lens):  # the oracle on the stored codes
        ks = np.stack([H.stored_hat(layer, gathered, b, h, n, 0) for h in range(8)])[None]
        vs = np.stack([H.stored_hat(layer, gathered, b, h, n, 1) for h in range(8)])[None]
        ref = H.oracle_attention(layer, _np64(q[b:b + 1]), ks, vs, [n])
        assert H.rel_l2_per_vector(got[b:b + 1], ref["out"]).max() < H.ATTN_TOL


@pytest.mark.parametrize("bs", [16, 80])
def test_paged_append_step_matches_contiguous(bs):
    """The fused append-and-attend step on a pool: the new token lands in the
    block the table names, with the same bytes and the same output as on a
    contiguous cache."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=23)
    lens = [1201, 640, 2]  # after the append
    t = max(lens)
    k = inputs.lognormal_kv(len(lens), t, 8, 128, seed=23, layer=6, which=inputs.K)
    v = inputs.lognormal_kv(len(lens), t, 8, 128, seed=23, layer=6, which=inputs.V)
    kn = inputs.lognormal_kv(len(lens), 1, 8, 128, seed=23, layer=6, which=inputs.K, token_offset_seed=5)
    vn = inputs.lognormal_kv(len(lens), 1, 8, 128, seed=23, layer=6, which=inputs.V, token_offset_seed=5)
    q = inputs.queries(len(lens), 32, 128, seed=23, layer=6)
    prior = [n - 1 for n in lens]
    pool, table, cap = _paged_prefill(layer, k, v, prior, bs, seed=23, unmap_tail=False)
    contig = _contig_prefill(layer, k, v, prior, cap)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    outs = []
    for store, fn, extra in ((pool, tq.tq_append_decode_attention_paged, (table,)),
                             (contig, tq.tq_append_decode_attention, ())):
        ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, len(lens), cap), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty(len(lens), 32, 128, dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        fn(layer.params, layer.kcb, layer.vcb, kn.cuda(), vn.cuda(), q.cuda(), store, *extra, lens_t, cap, out, ws,
           err)
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK and word == 0
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    _assert_same_bytes(_gather(layer, pool, table, cap), contig, lens)


@pytest.mark.parametrize("lens,seq,block", [([900, 700], 1, 3), ([3000] * 8, 5, 26)])
def test_paged_unmapped_block_inside_a_sequence_is_reported(lens, seq, block):
    """A -1 entry below a sequence's length: the decode skips that block's
    copies and sets TQ_DEVERR_PAGE (no fault); the other sequences are exact.
    The first case puts the block in a chunk fetched before the length is
    known, the second in a later chunk of a split."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=25)
    bs = 64
    bsz, t = len(lens), max(lens)
    k = inputs.lognormal_kv(bsz, t, 8, 128, seed=25, layer=7, which=inputs.K)
    v = inputs.lognormal_kv(bsz, t, 8, 128, seed=25, layer=7, which=inputs.V)
    q = inputs.queries(bsz, 32, 128, seed=25, layer=7)
    pool, table, cap = _paged_prefill(layer, k, v, lens, bs, seed=25)
    contig = _contig_prefill(layer, k, v, lens, cap)
    broken = table.clone()
    broken[seq, block] = -1
    got, st, word = _decode(layer, tq.tq_decode_attention_paged, q, pool, broken, lens, cap)
    assert st == tq.TQ_ERR_DEVICE and word & tq.TQ_DEVERR_PAGE
    want, _, _ = _decode(layer, tq.tq_decode_attention, q, contig, None, lens, cap)
    others = [b for b in range(bsz) if b != seq]
    assert np.array_equal(got[others], want[others])
    # an append whose block is unmapped writes nothing and reports it
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kn = inputs.lognormal_kv(1, 1, 8, 128, seed=25, layer=7, which=inputs.K, token_offset_seed=2).cuda()
    before = pool.k_codes.clone()
    tq.tq_quantize_append_paged(layer.params, layer.kcb, layer.vcb, kn, kn,
                                torch.tensor([block * bs], dtype=torch.int32, device="cuda"), pool,
                                broken[seq:seq + 1], err)
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_ERR_DEVICE and word == tq.TQ_DEVERR_PAGE
    assert torch.equal(before, pool.k_codes)


def test_paged_rejects_configurations_outside_the_tensor_core_kernel():
    layer = H.Layer(64, 8, 2, k_bits=4, v_bits=2, seed=27)
    pool = tq.alloc_cache(layer.params, 4, 16)
    table = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    q = torch.zeros(1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TqError) as e:
        _decode(layer, tq.tq_decode_attention_paged, q, pool, table, [16], 64)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED


def test_max_seq_len_above_capacity():
    """max_seq_len only bounds the lengths: with a bound four times the
    capacity, splits start past the cache's end; nothing is read there and the
    outputs match the oracle as with the capacity itself."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=29)
    cap = 1024
    lens = [1024, 500]
    k = inputs.lognormal_kv(2, cap, 8, 128, seed=29, layer=8, which=inputs.K)
    v = inputs.lognormal_kv(2, cap, 8, 128, seed=29, layer=8, which=inputs.V)
    q = inputs.queries(2, 32, 128, seed=29, layer=8)
    cache, st, word = H.gpu_quantize(layer, k, v, cap)
    assert st == tq.TQ_OK
    a, st, word = H.gpu_decode(layer, q, cache, lens, max_len=cap)
    assert st == tq.TQ_OK and word == 0
    b, st, word = H.gpu_decode(layer, q, cache, lens, max_len=4 * cap)
    assert st == tq.TQ_OK and word == 0
    # the two bounds give different split plans (the fp16 rounding of p * ||v||
    # follows each split's running max), so both are held to the oracle
    for got in (a, b):
        for s, n in enumerate(lens):
            ks = np.stack([H.stored_hat(layer, cache, s, h, n, 0) for h in range(8)])[None]
            vs = np.stack([H.stored_hat(layer, cache, s, h, n, 1) for h in range(8)])[None]
            ref = H.oracle_attention(layer, _np64(q[s:s + 1]), ks, vs, [n])
            assert H.rel_l2_per_vector(got[s:s + 1], ref["out"]).max() < H.ATTN_TOL
