"""CUDA path vs the CPU oracle at the workloads' full sizes.

* Llama-3-8B-shaped layer (B=1, Hq=32, Hkv=8, d=128, 32768-token prefill plus
  one appended token, K4/V2), decoded with the benchmark's launch plan: every
  code, norm and output compared.
* The same layer with int8 keys and 2-bit values, and as an all-int8
  boundary layer, prefilled and then one fused append-and-attend step: every
  code, scale, norm and output compared.
* Batched ragged decode (B=16, lengths uniform in [2048, 8192], K3/V2): every
  code, norm and output compared.
* 70B-shaped long context (B=4, Hq=64, Hkv=8, 131072 tokens, K3 + 64-bit QJL,
  V2, Sparse V at 1e-6): the whole batch runs on the GPU; three (sequence, kv
  head) units are checked against the oracle (codes, QJL bits, the eight
  query heads of each unit with and without Sparse V).
* Bulk prefill quantise (262144 tokens x 8 heads, d = 128 and 256, a K4/V3
  turbo layer and an int8 boundary layer): the whole slab is quantised on the
  GPU; every 97th token is checked against the oracle.
"""

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq

pytestmark = pytest.mark.gpu


def _np64(x):
    return x.float().cpu().numpy().astype(np.float64)


def _check_rows(layer, which, x, codes, norms, qjl=None, gamma=None):
    """Rows x [N, d] (fp64) against the GPU's bytes for the same vectors."""
    enc = layer.oracle_encode(x, which)
    codes = np.asarray(codes)
    norms = np.asarray(norms).view(np.uint16)
    mode, bits = layer.side(which)
    if mode == tq.TQ_MODE_INT8:
        assert np.array_equal(codes, enc["bytes"])
        assert np.array_equal(norms, H.fp16_bits(enc["norm16"]))
        return enc
    _, t_or = H.oracle_codebook(layer.d, bits)
    _, _, mismatched = H.check_codes(codes, enc, bits, layer.d, t_or)
    H.check_norms(norms, enc["norm16"])
    if qjl is not None:
        H.check_qjl(np.asarray(qjl), np.asarray(gamma).view(np.uint16), enc, mismatched, layer.params.qjl_dims)
    return enc


def _unit_rows(cache, b, h, n, which):
    if which == 0:
        return (cache.k_codes[b, h, :n].cpu().numpy(), cache.k_norms[b, h, :n].cpu().numpy(),
                None if cache.k_qjl is None else cache.k_qjl[b, h, :n].cpu().numpy(),
                None if cache.k_gamma is None else cache.k_gamma[b, h, :n].cpu().numpy())
    return cache.v_codes[b, h, :n].cpu().numpy(), cache.v_norms[b, h, :n].cpu().numpy(), None, None


def _oracle_unit(layer, kx, vx, cache, b, h, n):
    """Check unit (b, h)'s first n tokens against the oracle's encoding; return
    the oracle's reconstruction of the GPU's stored K, V [n, d] (same codes)."""
    kc, kn, kq, kg = _unit_rows(cache, b, h, n, 0)
    vc, vn, _, _ = _unit_rows(cache, b, h, n, 1)
    _check_rows(layer, 0, kx, kc, kn, kq, kg)
    _check_rows(layer, 1, vx, vc, vn)
    return H.stored_hat(layer, cache, b, h, n, 0), H.stored_hat(layer, cache, b, h, n, 1)


def test_llama8b_layer_full_context():
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=1234)
    ctx = 32768
    t = ctx + 1
    cap = ctx + 26  # the benchmark's default capacity (and max_seq_len)
    k = inputs.lognormal_kv(1, t, 8, 128, seed=1234, layer=0, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, 128, seed=1234, layer=0, which=inputs.V)
    q = inputs.queries(1, 32, 128, seed=1234)
    cache = tq.alloc_cache(layer.params, 1, cap)
    cache, st, word = H.gpu_quantize(layer, k[:, :ctx], v[:, :ctx], cap, cache=cache)
    assert st == tq.TQ_OK and word == 0
    cache, st, word = H.gpu_quantize(layer, k[:, ctx:], v[:, ctx:], cap, cache=cache,
                                     positions=torch.tensor([ctx], dtype=torch.int32))
    assert st == tq.TQ_OK and word == 0
    got, st, word = H.gpu_decode(layer, q, cache, [t], max_len=cap)
    assert st == tq.TQ_OK and word == 0
    kn, vn = _np64(k), _np64(v)
    khat = np.empty((1, 8, t, 128))
    vhat = np.empty((1, 8, t, 128))
    for h in range(8):
        khat[0, h], vhat[0, h] = _oracle_unit(layer, kn[0, :, h], vn[0, :, h], cache, 0, h, t)
    ref = H.oracle_attention(layer, _np64(q), khat, vhat, [t])
    err = H.rel_l2_per_vector(got, ref["out"])
    assert err.max() < H.ATTN_TOL, err.max()


@pytest.mark.parametrize("v_mode", [tq.TQ_MODE_TURBO, tq.TQ_MODE_INT8])
def test_llama8b_int8_keys_full_context(v_mode):
    """The Llama-3-8B-shaped layer with int8 keys and 2-bit values (or int8
    values: a boundary layer): 32768 tokens prefilled, then one fused
    append-and-attend step; every code, scale, norm and output compared."""
    layer = H.Layer(128, 32, 8, k_mode=tq.TQ_MODE_INT8, v_mode=v_mode, v_bits=2, seed=4321)
    ctx = 32768
    t = ctx + 1
    cap = ctx + 8
    k = inputs.lognormal_kv(1, t, 8, 128, seed=4321, layer=0, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, 128, seed=4321, layer=0, which=inputs.V)
    q = inputs.queries(1, 32, 128, seed=4321)
    cache = tq.alloc_cache(layer.params, 1, cap)
    cache, st, word = H.gpu_quantize(layer, k[:, :ctx], v[:, :ctx], cap, cache=cache)
    assert st == tq.TQ_OK and word == 0
    ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, 1, cap), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, 32, 128, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_append_decode_attention(layer.params, layer.kcb, layer.vcb, k[:, ctx:].cuda(), v[:, ctx:].cuda(), q.cuda(),
                                  cache, torch.tensor([t], dtype=torch.int32, device="cuda"), cap, out, ws, err)
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK and word == 0
    got = out.cpu().numpy()
    kn, vn = _np64(k), _np64(v)
    khat = np.empty((1, 8, t, 128))
    vhat = np.empty((1, 8, t, 128))
    for h in range(8):
        khat[0, h], vhat[0, h] = _oracle_unit(layer, kn[0, :, h], vn[0, :, h], cache, 0, h, t)
    ref = H.oracle_attention(layer, _np64(q), khat, vhat, [t])
    err = H.rel_l2_per_vector(got, ref["out"])
    assert err.max() < H.ATTN_TOL, err.max()


def test_batched_ragged_full():
    layer = H.Layer(128, 32, 8, k_bits=3, v_bits=2, seed=77)
    bsz, t = 16, 8192
    lens = inputs.ragged_lengths(bsz, 2048, 8192, seed=0).tolist()
    k = inputs.lognormal_kv(bsz, t, 8, 128, seed=77, layer=1, which=inputs.K)
    v = inputs.lognormal_kv(bsz, t, 8, 128, seed=77, layer=1, which=inputs.V)
    q = inputs.queries(bsz, 32, 128, seed=77, layer=1)
    cache, st, word = H.gpu_quantize(layer, k, v, t)
    assert st == tq.TQ_OK and word == 0
    got, st, word = H.gpu_decode(layer, q, cache, lens, max_len=t)
    assert st == tq.TQ_OK and word == 0
    kn, vn = _np64(k), _np64(v)
    qn = _np64(q)
    errs = []
    for b in range(bsz):
        n = lens[b]
        khat = np.empty((1, 8, n, 128))
        vhat = np.empty((1, 8, n, 128))
        for h in range(8):
            khat[0, h], vhat[0, h] = _oracle_unit(layer, kn[b, :n, h], vn[b, :n, h], cache, b, h, n)
        ref = H.oracle_attention(layer, qn[b:b + 1], khat, vhat, [n])
        errs.append(H.rel_l2_per_vector(got[b:b + 1], ref["out"]).max())
    assert max(errs) < H.ATTN_TOL, max(errs)


def test_70b_long_context_sampled_units():
    tau = 1e-6
    layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=70, tau=tau)
    dense = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=70)
    bsz, t = 4, 131072
    k = inputs.lognormal_kv(bsz, t, 8, 128, seed=70, layer=40, which=inputs.K, device="cuda")
    v = inputs.lognormal_kv(bsz, t, 8, 128, seed=70, layer=40, which=inputs.V, device="cuda")
    q = inputs.queries(bsz, 64, 128, seed=70, layer=40)
    cache, st, word = H.gpu_quantize(layer, k, v, t)
    assert st == tq.TQ_OK and word == 0
    got_sparse, st, word = H.gpu_decode(layer, q, cache, [t] * bsz)
    assert st == tq.TQ_OK and word == 0
    got_dense, st, word = H.gpu_decode(dense, q, cache, [t] * bsz)
    assert st == tq.TQ_OK and word == 0
    qn = _np64(q)
    for b, h in ((0, 0), (2, 5), (3, 7)):
        khat, vhat = _oracle_unit(layer, _np64(k[b, :, h]), _np64(v[b, :, h]), cache, b, h, t)
        heads = slice(8 * h, 8 * h + 8)
        ref = H.oracle_attention(layer, qn[b:b + 1, heads], khat[None, None], vhat[None, None], [t], tau=tau)
        assert H.rel_l2_per_vector(got_dense[b, heads], ref["out"][0]).max() < H.ATTN_TOL
        g = got_sparse[b, heads]
        scale = np.linalg.norm(ref["out"][0], axis=-1)
        outside = np.maximum(ref["lo"][0] - g, 0.0) + np.maximum(g - ref["hi"][0], 0.0)
        assert (np.linalg.norm(outside, axis=-1) / scale).max() < H.ATTN_TOL


@pytest.mark.parametrize("d", [128, 256])
def test_bulk_prefill_quantize_full_slab(d):
    t, heads, stride = 262144, 8, 97
    k = inputs.lognormal_kv(1, t, heads, d, seed=5, layer=2, which=inputs.K, device="cuda")
    v = inputs.lognormal_kv(1, t, heads, d, seed=5, layer=2, which=inputs.V, device="cuda")
    sample = torch.arange(0, t, stride)
    ks = _np64(k[0, sample])  # [S, heads, d]
    vs = _np64(v[0, sample])
    for layer in (H.Layer(d, heads, heads, k_bits=4, v_bits=3, seed=2),
                  H.Layer(d, heads, heads, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8, seed=0)):
        cache, st, word = H.gpu_quantize(layer, k, v, t)
        assert st == tq.TQ_OK and word == 0
        idx = sample.cuda()
        for h in range(heads):
            _check_rows(layer, 0, ks[:, h], cache.k_codes[0, h, idx].cpu().numpy(),
                        cache.k_norms[0, h, idx].cpu().numpy())
            _check_rows(layer, 1, vs[:, h], cache.v_codes[0, h, idx].cpu().numpy(),
                        cache.v_norms[0, h, idx].cpu().numpy())
        del cache
        torch.cuda.empty_cache()
