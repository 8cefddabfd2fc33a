"""tq_prefill_attention (append a chunk of tokens, then causal attention of
its queries over the compressed cache, on the tcgen05 tensor cores) against
the oracle: the appended codes follow the code rules, and every output row
matches the oracle's causal attention on the GPU's stored codes within 2e-3
relative L2.  Chunks span several 128-row query blocks and several 64-key
tiles with ragged ends."""

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq
from oracle import attention as oatt

pytestmark = pytest.mark.gpu


def _prefill_case(layer, starts, n_new, seed, prefill_tokens=None, dtype=torch.bfloat16, expect_word=0,
                  capacity=None):
    """Cache pre-filled with `starts[b]` tokens per sequence (GPU quantise),
    then one tq_prefill_attention call appending n_new fresh tokens (chunk
    and queries in `dtype`)."""
    bsz, hkv, d = len(starts), layer.hkv, layer.d
    cap = max(starts) + n_new + 40 if capacity is None else capacity
    pre = max(starts) if prefill_tokens is None else prefill_tokens
    k0 = inputs.lognormal_kv(bsz, max(pre, 1), hkv, d, seed=seed, layer=3, which=inputs.K)
    v0 = inputs.lognormal_kv(bsz, max(pre, 1), hkv, d, seed=seed, layer=3, which=inputs.V)
    cache, st, word = H.gpu_quantize(layer, k0, v0, cap)
    assert st == tq.TQ_OK and word == 0
    kn = inputs.lognormal_kv(bsz, n_new, hkv, d, seed=seed, layer=3, which=inputs.K, token_offset_seed=5).to(dtype)
    vn = inputs.lognormal_kv(bsz, n_new, hkv, d, seed=seed, layer=3, which=inputs.V, token_offset_seed=5).to(dtype)
    q = torch.randn(bsz, n_new, layer.hq, d, generator=torch.Generator().manual_seed(seed)).to(dtype)
    pos = torch.tensor(starts, dtype=torch.int32, device="cuda")
    out = torch.empty(bsz, n_new, layer.hq, d, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(tq.tq_prefill_workspace_bytes(layer.params, bsz, n_new), dtype=torch.uint8, device="cuda")
    tq.tq_prefill_attention(layer.params, layer.kcb, layer.vcb, kn.cuda(), vn.cuda(), q.cuda(), pos, cache, out, ws,
                            err)
    st, word = tq.tq_read_device_error(err)
    assert word == expect_word and st == (tq.TQ_OK if expect_word == 0 else tq.TQ_ERR_DEVICE), (st, word)
    return cache, out.cpu().numpy(), q, (kn, vn)


def _check_rows(layer, cache, out, q, starts, rows=None):
    """Oracle causal attention on the GPU's stored codes, row by row (all rows,
    or the sampled (b, j) pairs given)."""
    bsz, n_new = out.shape[0], out.shape[1]
    worst = 0.0
    for b in range(bsz):
        n = starts[b] + n_new
        khat = np.stack([H.stored_hat(layer, cache, b, h, n, 0) for h in range(layer.hkv)])[None]
        vhat = np.stack([H.stored_hat(layer, cache, b, h, n, 1) for h in range(layer.hkv)])[None]
        qb = q[b:b + 1].float().numpy().astype(np.float64)
        js = range(n_new) if rows is None else [j for (bb, j) in rows if bb == b]
        for j in js:
            ref = oatt.decode_attention(qb[:, j], khat, vhat, [starts[b] + j + 1], layer.params.sm_scale or None)["out"]
            rel = H.rel_l2_per_vector(out[b:b + 1, j], ref)
            worst = max(worst, rel.max())
    return worst


def _check_appended_codes(layer, cache, starts, n_new, kn, vn):
    for b, s0 in enumerate(starts):
        for which, x, codes, norms in ((0, kn, cache.k_codes, cache.k_norms), (1, vn, cache.v_codes, cache.v_norms)):
            for h in range(layer.hkv):
                rows = x[b, :, h].float().numpy().astype(np.float64)
                enc = layer.oracle_encode(rows, which)
                got = codes[b, h, s0:s0 + n_new].cpu().numpy()
                _, bits = layer.side(which)
                _, t_or = H.oracle_codebook(layer.d, bits)
                H.check_codes(got, enc, bits, layer.d, t_or)
                H.check_norms(norms[b, h, s0:s0 + n_new].cpu().numpy().view(np.uint16), enc["norm16"])


@pytest.mark.parametrize("hq,hkv,kb,vb", [(32, 8, 4, 2), (64, 8, 3, 2), (8, 8, 2, 4), (16, 1, 4, 3), (32, 8, 4, 4),
                                           (32, 8, 3, 3)])
def test_prefill_matches_oracle(hq, hkv, kb, vb):
    """Two sequences with different starts; 100 new tokens: several query
    blocks (128 / G tokens each) and a ragged last one; ~13 key tiles."""
    layer = H.Layer(128, hq, hkv, k_bits=kb, v_bits=vb, seed=21)
    starts = [700, 333]
    cache, out, q, (kn, vn) = _prefill_case(layer, starts, 100, seed=21)
    _check_appended_codes(layer, cache, starts, 100, kn, vn)
    worst = _check_rows(layer, cache, out, q, starts)
    assert worst < H.ATTN_TOL, worst


def test_prefill_chunk_of_one_is_a_decode_step():
    """One new token: the same as tq_append_decode_attention over start + 1."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=22)
    starts = [517]
    cache, out, q, (kn, vn) = _prefill_case(layer, starts, 1, seed=22)
    worst = _check_rows(layer, cache, out, q, starts)
    assert worst < H.ATTN_TOL, worst


def test_prefill_from_an_empty_cache():
    """Start 0: the chunk attends only to itself (causal within the chunk)."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=23)
    cache, out, q, _ = _prefill_case(layer, [0], 150, seed=23, prefill_tokens=1)
    worst = _check_rows(layer, cache, out, q, [0])
    assert worst < H.ATTN_TOL, worst


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_prefill_chunk_and_query_dtypes(dtype):
    """fp32 and fp16 chunks and queries (the kernel converts on load)."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=26)
    starts = [260]
    cache, out, q, (kn, vn) = _prefill_case(layer, starts, 70, seed=26, dtype=dtype)
    _check_appended_codes(layer, cache, starts, 70, kn, vn)
    worst = _check_rows(layer, cache, out, q, starts)
    assert worst < H.ATTN_TOL, worst


def test_prefill_flags_a_chunk_past_the_capacity():
    """A sequence whose chunk would end past the cache's capacity is refused
    on the device (TQ_DEVERR_POSITION): nothing of it is appended and its
    output rows are zero; the other sequence is unaffected."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=27)
    n_new = 60
    cap = 400 + n_new + 40
    starts = [400, cap - n_new + 1]
    cache, out, q, _ = _prefill_case(layer, starts, n_new, seed=27, prefill_tokens=400,
                                     expect_word=tq.TQ_DEVERR_POSITION, capacity=cap)
    assert np.all(out[1] == 0.0)
    assert np.all(cache.k_norms[1, :, cap - n_new:].cpu().numpy().view(np.uint16) == 0)
    worst = _check_rows(layer, cache, out[:1], q[:1], starts[:1])
    assert worst < H.ATTN_TOL, worst


def test_prefill_workspace_reused_across_chunks():
    """Two chunks in a row on one workspace that starts as arbitrary bytes.
    With 16 units of ~15 key tiles over one block per SM, most units are
    cut between blocks, so both calls go through the merge kernel."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=28)
    start, n1, n2 = 900, 40, 56
    cap = start + n1 + n2 + 40
    k0 = inputs.lognormal_kv(1, start, 8, 128, seed=28, layer=3, which=inputs.K)
    v0 = inputs.lognormal_kv(1, start, 8, 128, seed=28, layer=3, which=inputs.V)
    cache, st, word = H.gpu_quantize(layer, k0, v0, cap)
    assert st == tq.TQ_OK and word == 0
    nbytes = max(tq.tq_prefill_workspace_bytes(layer.params, 1, n) for n in (n1, n2))
    assert nbytes > 0
    ws = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    results = []
    for at, n in ((start, n1), (start + n1, n2)):
        kn = inputs.lognormal_kv(1, n, 8, 128, seed=28 + at, layer=3, which=inputs.K).cuda()
        vn = inputs.lognormal_kv(1, n, 8, 128, seed=28 + at, layer=3, which=inputs.V).cuda()
        q = torch.randn(1, n, 32, 128, generator=torch.Generator().manual_seed(at)).to(torch.bfloat16)
        out = torch.empty(1, n, 32, 128, dtype=torch.float32, device="cuda")
        pos = torch.tensor([at], dtype=torch.int32, device="cuda")
        tq.tq_prefill_attention(layer.params, layer.kcb, layer.vcb, kn, vn, q.cuda(), pos, cache, out, ws, err)
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK and word == 0, (st, word)
        results.append((at, q, out.cpu().numpy()))
    for at, q, out in results:
        worst = _check_rows(layer, cache, out, q, [at])
        assert worst < H.ATTN_TOL, (at, worst)


def test_prefill_inputs_written_by_the_kernels_just_before():
    """The chunk, the queries and the positions are produced on the stream by
    GPU kernels immediately before the call, behind a long matmul.  The
    attention and merge kernels start as programmatic dependents of the
    kernel before them; they must still see these inputs (the append only
    lets its dependent start after every earlier kernel has finished)."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=31)
    start, n = 777, 48
    k0 = inputs.lognormal_kv(1, start, 8, 128, seed=31, layer=3, which=inputs.K)
    v0 = inputs.lognormal_kv(1, start, 8, 128, seed=31, layer=3, which=inputs.V)
    cache, st, word = H.gpu_quantize(layer, k0, v0, start + n + 16)
    assert st == tq.TQ_OK and word == 0
    kn = inputs.lognormal_kv(1, n, 8, 128, seed=32, layer=3, which=inputs.K)
    vn = inputs.lognormal_kv(1, n, 8, 128, seed=32, layer=3, which=inputs.V)
    q = torch.randn(1, n, 32, 128, generator=torch.Generator().manual_seed(33)).to(torch.bfloat16)
    # device copies of the inputs, scaled by zero until the kernels below fill them
    kd, vd, qd = kn.cuda() * 0, vn.cuda() * 0, q.cuda() * 0
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc, vc, qc = kn.cuda(), vn.cuda(), q.cuda()
    big = torch.randn(4096, 4096, device="cuda")
    torch.cuda.synchronize()
    for _ in range(3):
        big = big @ big * (1.0 / 64.0)  # a few milliseconds of work ahead of the writes
    kd.copy_(kc * 1.0)
    vd.copy_(vc * 1.0)
    qd.copy_(qc * 1.0)
    pos.fill_(start)
    out = torch.empty(1, n, 32, 128, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_prefill_workspace_bytes(layer.params, 1, n), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_prefill_attention(layer.params, layer.kcb, layer.vcb, kd, vd, qd, pos, cache, out, ws, err)
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK and word == 0, (st, word)
    _check_appended_codes(layer, cache, [start], n, kn, vn)
    worst = _check_rows(layer, cache, out.cpu().numpy(), q, [start])
    assert worst < H.ATTN_TOL, worst


def test_prefill_whole_units_past_the_schedule():
    """More units than the shared schedule holds (a 16416-token chunk of 8
    kv heads in 32-token query blocks: 4104 > 4096 units): each block takes
    one whole unit and no workspace is needed; sampled rows against the
    oracle, the first and last of query blocks among them."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=29)
    n_new = 16416
    assert tq.tq_prefill_workspace_bytes(layer.params, 1, n_new) == 0
    cache, out, q, _ = _prefill_case(layer, [0], n_new, seed=29, prefill_tokens=1)
    gen = np.random.default_rng(29)
    rows = [(0, j) for j in (0, 31, 32, 8191, 8192, n_new - 1)]
    rows += [(0, int(j)) for j in sorted(gen.choice(n_new, size=6, replace=False))]
    worst = _check_rows(layer, cache, out, q, [0], rows=rows)
    assert worst < H.ATTN_TOL, worst


def test_prefill_workspace_argument_checks():
    """A missing, short or misaligned workspace is refused before anything
    is appended (the cache stays empty)."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=30)
    n = 64
    cache = tq.alloc_cache(layer.params, 1, 256)
    x = torch.zeros(1, n, 8, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, n, 32, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, n, 32, 128, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = tq.tq_prefill_workspace_bytes(layer.params, 1, n)
    big = torch.zeros(need + 16, dtype=torch.uint8, device="cuda")
    for ws, status in ((None, tq.TQ_ERR_INVALID_ARG), (big[:need - 16], tq.TQ_ERR_CAPACITY),
                       (big[1:need + 1], tq.TQ_ERR_ALIGNMENT)):
        with pytest.raises(tq.TqError) as ei:
            tq.tq_prefill_attention(layer.params, layer.kcb, layer.vcb, x, x, q, pos, cache, out, ws)
        assert ei.value.status == status
    assert not cache.k_norms.any()


@pytest.mark.slow
def test_prefill_llama8b_32k_chunk_sampled_rows():
    """Llama-3-8B-shaped layer, 32768 cached tokens, a 512-token chunk (the
    benchmark's prefill workload), 16 sampled rows against the oracle."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=24)
    starts = [32768]
    cache, out, q, _ = _prefill_case(layer, starts, 512, seed=24)
    gen = np.random.default_rng(24)
    rows = [(0, int(j)) for j in sorted(gen.choice(512, size=16, replace=False))] + [(0, 0), (0, 511)]
    worst = _check_rows(layer, cache, out, q, starts, rows=rows)
    assert worst < H.ATTN_TOL, worst


def test_prefill_rejects_unsupported_settings():
    layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=25)
    cache = tq.alloc_cache(layer.params, 1, 64)
    x = torch.zeros(1, 4, 8, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, 4, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 4, 64, 128, device="cuda")
    with pytest.raises(tq.TqError) as ei:
        tq.tq_prefill_attention(layer.params, layer.kcb, layer.vcb, x, x, q, torch.zeros(1, dtype=torch.int32,
                                device="cuda"), cache, out, None)
    assert ei.value.status == tq.TQ_ERR_UNSUPPORTED
