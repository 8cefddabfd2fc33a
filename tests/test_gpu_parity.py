"""CUDA path vs the CPU oracle on seeded inputs (sizes the oracle finishes in
seconds, spanning several token splits and a ragged tail).  Every call goes
through the C ABI of libtq.so."""

import math

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq

pytestmark = pytest.mark.gpu


def _to_np(x):
    return x.float().cpu().numpy().astype(np.float64)


def _flat(x):
    """[B, T, Hkv, d] -> [B*Hkv*T, d] in cache order."""
    b, t, h, d = x.shape
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(b * h * t, d))


def _check_quantized(layer, cache, kx, vx, start=0):
    """Compare a GPU-filled cache with the oracle for tokens [start, start+T)."""
    b, t, hkv, d = kx.shape
    out = {}
    for which, x in ((0, kx), (1, vx)):
        enc = layer.oracle_encode(_flat(x), which)
        codes = (cache.k_codes if which == 0 else cache.v_codes)[:, :, start:start + t].cpu().numpy()
        norms = (cache.k_norms if which == 0 else cache.v_norms)[:, :, start:start + t].cpu().numpy()
        codes = codes.reshape(b * hkv * t, -1)
        norms = norms.reshape(-1).view(np.uint16)
        mode, bits = layer.side(which)
        if mode == tq.TQ_MODE_INT8:
            assert np.array_equal(codes, enc["bytes"])
            assert np.array_equal(norms, H.fp16_bits(enc["norm16"]))
            mismatched = np.zeros(codes.shape[0], dtype=bool)
        else:
            _, t_or = H.oracle_codebook(layer.d, bits)
            _, flips, mismatched = H.check_codes(codes, enc, bits, layer.d, t_or)
            H.check_norms(norms, enc["norm16"])
            out["flips%d" % which] = flips
        if which == 0 and layer.params.qjl_dims:
            qjl = cache.k_qjl[:, :, start:start + t].cpu().numpy().reshape(b * hkv * t, -1)
            gam = cache.k_gamma[:, :, start:start + t].cpu().numpy().reshape(-1).view(np.uint16)
            H.check_qjl(qjl, gam, enc, mismatched, layer.params.qjl_dims)
        out[which] = enc
    return out


def _oracle_hat(layer, enc, which, shape):
    b, hkv, t, d = shape
    return layer.oracle_decode(enc, which).reshape(b, hkv, t, d)


def _attention_case(layer, kx, vx, q, lens, tau=0.0):
    """Quantise on the GPU, check codes; attend on the GPU over (a) its own
    cache, against the oracle's attention on those stored codes, and (b) the
    oracle's codes uploaded, against the oracle's attention on its codes."""
    bsz, t, hkv, d = kx.shape
    cache, st, word = H.gpu_quantize(layer, kx, vx, t)
    assert st == tq.TQ_OK and word == 0
    enc = _check_quantized(layer, cache, _to_np(kx), _to_np(vx))
    khat = _oracle_hat(layer, enc[0], 0, (bsz, hkv, t, d))
    vhat = _oracle_hat(layer, enc[1], 1, (bsz, hkv, t, d))
    ref = H.oracle_attention(layer, _to_np(q), khat, vhat, lens, tau)
    want = ref["out"] if tau == 0 else ref["exact_sparse"]
    # (a) end to end, compared on the GPU's own stored codes (code parity passed above)
    got, st, word = H.gpu_decode(layer, q, cache, lens)
    assert st == tq.TQ_OK and word == 0
    ks = np.stack([np.stack([H.stored_hat(layer, cache, b, h, t, 0) for h in range(hkv)]) for b in range(bsz)])
    vs = np.stack([np.stack([H.stored_hat(layer, cache, b, h, t, 1) for h in range(hkv)]) for b in range(bsz)])
    ref_e2e = H.oracle_attention(layer, _to_np(q), ks, vs, lens, tau)
    err_e2e = H.rel_l2_per_vector(got, ref_e2e["out"] if tau == 0 else ref_e2e["exact_sparse"])
    # (b) on the oracle's own codes
    cache2 = tq.alloc_cache(layer.params, bsz, t)
    for b in range(bsz):
        for h in range(hkv):
            sel = slice((b * hkv + h) * t, (b * hkv + h + 1) * t)
            H.upload_oracle_cache(layer, cache2, b, h, {k: v[sel] for k, v in enc[0].items() if isinstance(v, np.ndarray)},
                                  {k: v[sel] for k, v in enc[1].items() if isinstance(v, np.ndarray)})
    got2, st, word = H.gpu_decode(layer, q, cache2, lens)
    assert st == tq.TQ_OK and word == 0
    err_same = H.rel_l2_per_vector(got2, want)
    return err_e2e, err_same, got2, ref, None


def test_single_head_fp32_k4_v2():
    """One head, d = 128, fp32 N(0,1) with four x20 outlier channels, 4096 tokens."""
    k, v, q, _ = inputs.single_head_fp32(seed=0)
    layer = H.Layer(128, 1, 1, k_bits=4, v_bits=2, seed=0)
    kx, vx = k[None, :, None, :], v[None, :, None, :]
    e2e, same, _, _, _ = _attention_case(layer, kx, vx, q[None, None, :], [4096])
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


def test_single_head_dequantize_matches_oracle():
    k, v, _, _ = inputs.single_head_fp32(seed=0)
    layer = H.Layer(128, 1, 1, k_bits=4, v_bits=2, seed=0)
    encs = [layer.oracle_encode(k.double().numpy(), 0), layer.oracle_encode(v.double().numpy(), 1)]
    cache = tq.alloc_cache(layer.params, 1, 4096)
    H.upload_oracle_cache(layer, cache, 0, 0, encs[0], encs[1])
    ko = torch.empty(4096, 1, 128, device="cuda")
    vo = torch.empty(4096, 1, 128, device="cuda")
    tq.tq_dequantize(layer.params, layer.kcb, layer.vcb, cache, 0, 0, 4096, ko, vo)
    torch.cuda.synchronize()
    for which, out in ((0, ko), (1, vo)):
        want = layer.oracle_decode(encs[which], which)
        got = out[:, 0].cpu().numpy()
        assert H.rel_l2_per_vector(got, want).max() < 1e-5


def test_llama8b_shaped_prefill_then_append():
    """B=1, Hq=32, Hkv=8 (GQA 4), d=128, bf16 log-normal; prefill 2999 tokens,
    append one, attend over 3000 (several splits and a ragged tail)."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=3)
    t = 3000
    k = inputs.lognormal_kv(1, t, 8, 128, seed=1, layer=3, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, 128, seed=1, layer=3, which=inputs.V)
    q = inputs.queries(1, 32, 128, seed=1, layer=3)
    cache = tq.alloc_cache(layer.params, 1, t)
    cache, st, word = H.gpu_quantize(layer, k[:, : t - 1], v[:, : t - 1], t, cache=cache)
    assert st == tq.TQ_OK
    cache, st, word = H.gpu_quantize(layer, k[:, t - 1:], v[:, t - 1:], t,
                                     positions=torch.tensor([t - 1], dtype=torch.int32), cache=cache)
    assert st == tq.TQ_OK and word == 0
    enc = _check_quantized(layer, cache, _to_np(k), _to_np(v))
    khat = _oracle_hat(layer, enc[0], 0, (1, 8, t, 128))
    vhat = _oracle_hat(layer, enc[1], 1, (1, 8, t, 128))
    ref = H.oracle_attention(layer, _to_np(q), khat, vhat, [t])
    got, st, word = H.gpu_decode(layer, q, cache, [t])
    assert st == tq.TQ_OK
    assert H.rel_l2_per_vector(got, ref["out"]).max() < H.ATTN_TOL
    # the appended token matters: attending over t-1 tokens gives another answer
    got_short, _, _ = H.gpu_decode(layer, q, cache, [t - 1])
    assert H.rel_l2_per_vector(got_short, got).max() > 1e-6


def test_batched_ragged_k3_v2():
    """B=5 ragged lengths, K 3-bit codes crossing byte boundaries, V 2-bit."""
    layer = H.Layer(128, 32, 8, k_bits=3, v_bits=2, seed=5)
    t = 1500
    lens = inputs.ragged_lengths(5, 200, t, seed=2).tolist()
    k = inputs.lognormal_kv(5, t, 8, 128, seed=2, layer=5, which=inputs.K)
    v = inputs.lognormal_kv(5, t, 8, 128, seed=2, layer=5, which=inputs.V)
    q = inputs.queries(5, 32, 128, seed=2, layer=5)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, lens)
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


def test_qjl_residual_group8():
    """K 3-bit + 64-dim QJL sign residual, V 2-bit, G = 8, two sequences."""
    layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=7)
    t = 1200
    k = inputs.lognormal_kv(2, t, 8, 128, seed=4, layer=7, which=inputs.K)
    v = inputs.lognormal_kv(2, t, 8, 128, seed=4, layer=7, which=inputs.V)
    q = inputs.queries(2, 64, 128, seed=4, layer=7)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, [t, t - 333])
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


def test_sparse_v_within_admissible_interval():
    """Sparse V on log-normal data: the output lies in the oracle's interval
    of every admissible skip set (each dropped weight < tau)."""
    layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=9, tau=1e-6)
    t = 2500
    k = inputs.lognormal_kv(1, t, 8, 128, seed=6, layer=9, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, 128, seed=6, layer=9, which=inputs.V)
    q = inputs.queries(1, 64, 128, seed=6, layer=9)
    cache, st, _ = H.gpu_quantize(layer, k, v, t)
    enc = _check_quantized(layer, cache, _to_np(k), _to_np(v))
    khat = _oracle_hat(layer, enc[0], 0, (1, 8, t, 128))
    vhat = _oracle_hat(layer, enc[1], 1, (1, 8, t, 128))
    ref = H.oracle_attention(layer, _to_np(q), khat, vhat, [t], tau=1e-6)
    got, st, _ = H.gpu_decode(layer, q, cache, [t])
    assert st == tq.TQ_OK
    scale = np.linalg.norm(ref["out"], axis=-1, keepdims=True)
    below = np.maximum(ref["lo"] - got, 0.0)
    above = np.maximum(got - ref["hi"], 0.0)
    outside = np.linalg.norm(below + above, axis=-1) / scale[..., 0]
    assert outside.max() < H.ATTN_TOL, outside.max()


# A dropped position's weight as the kernel sees it is below tau; the
# oracle's exact weight of the same position differs from the kernel's by the
# kernel's score error (fp16 centroids and query terms, about 1e-3 in the
# logit), so the oracle's weight stays below tau * (1 + 1e-2).
MASK_SLACK = 1e-2


@pytest.mark.parametrize("d", [128, 64])
def test_sparse_v_mask_is_admissible_and_exact(d):
    """Sparse V with the kernel's skip mask (d = 128: tensor-core kernel, the
    70B-shaped settings at small size; d = 64: the general kernels): every
    dropped position has exact weight below tau, the output equals the
    oracle's sum without exactly those positions (the denominator keeps
    them), and the gate fires on log-normal data."""
    if d == 128:
        layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=9, tau=1e-6)
    else:
        layer = H.Layer(64, 16, 4, k_bits=3, v_bits=2, seed=9, tau=1e-6)
    t = 2500
    k = inputs.lognormal_kv(1, t, layer.hkv, d, seed=6, layer=9, which=inputs.K)
    v = inputs.lognormal_kv(1, t, layer.hkv, d, seed=6, layer=9, which=inputs.V)
    q = inputs.queries(1, layer.hq, d, seed=6, layer=9)
    cache, st, _ = H.gpu_quantize(layer, k, v, t)
    enc = _check_quantized(layer, cache, _to_np(k), _to_np(v))
    khat = _oracle_hat(layer, enc[0], 0, (1, layer.hkv, t, d))
    vhat = _oracle_hat(layer, enc[1], 1, (1, layer.hkv, t, d))
    got, st, word, mask = H.gpu_decode(layer, q, cache, [t], with_mask=True)
    assert st == tq.TQ_OK and word == 0
    ref = H.oracle_attention(layer, _to_np(q), khat, vhat, [t], tau=1e-6, skip_mask=mask)
    assert ref["mask_max_weight"].max() < 1e-6 * (1 + MASK_SLACK), ref["mask_max_weight"].max()
    assert H.rel_l2_per_vector(got, ref["masked"]).max() < H.ATTN_TOL
    frac = mask.sum() / mask.size
    assert frac > 0.01, frac


def test_sparse_v_exact_on_separated_scores():
    """Scores built so that the skip set is unambiguous: 4 of every 16
    positions are 'hot' (scores ~ +8), the rest 'cold' (~ -8, weight < 1e-6
    for any admissible rule) with large values.  Skipping must drop exactly
    the cold positions: the output matches the oracle's exact Sparse-V sum,
    which differs from full attention by far more than the tolerance."""
    d, t = 128, 2000
    layer = H.Layer(d, 8, 1, k_bits=4, v_bits=4, seed=11, tau=1e-6)
    gen = torch.Generator().manual_seed(5)
    q = torch.randn(1, 8, d, generator=gen)
    qd = q[0, 0] / q[0, 0].norm()
    hot = (torch.arange(t) % 16) < 4
    a = 8.0 / (q[0, 0].norm() / math.sqrt(d))
    k = torch.where(hot[:, None], a * qd[None, :], -a * qd[None, :]) + 0.01 * torch.randn(t, d, generator=gen)
    v = torch.randn(t, d, generator=gen)
    v[~hot] = 6.0e4 / math.sqrt(d) * torch.sign(torch.randn(d, generator=gen))[None, :]
    q = q[:, :1].repeat(1, 8, 1)  # all heads share the query
    # nearly identical keys put whole columns of codes on the same boundaries,
    # so this case runs on the oracle's codes (uploaded), not on GPU quantisation
    enc = [layer.oracle_encode(k.double().numpy(), 0), layer.oracle_encode(v.double().numpy(), 1)]
    cache = tq.alloc_cache(layer.params, 1, t)
    H.upload_oracle_cache(layer, cache, 0, 0, enc[0], enc[1])
    khat = layer.oracle_decode(enc[0], 0)[None, None]
    vhat = layer.oracle_decode(enc[1], 1)[None, None]
    ref = H.oracle_attention(layer, _to_np(q), khat, vhat, [t], tau=1e-6)
    assert abs(ref["skip_fraction"] - 0.75) < 1e-9
    got, st, _, mask = H.gpu_decode(layer, q, cache, [t], with_mask=True)
    assert st == tq.TQ_OK
    assert H.rel_l2_per_vector(got, ref["exact_sparse"]).max() < H.ATTN_TOL
    assert H.rel_l2_per_vector(ref["exact_sparse"], ref["out"]).min() > 10 * H.ATTN_TOL
    # the kernel reports exactly the cold positions, for every head
    assert np.array_equal(mask, np.broadcast_to((~hot).numpy(), mask.shape))


@pytest.mark.parametrize("d", [128, 256])
def test_bulk_quantize_turbo_and_int8(d):
    """Prefill-style quantise: 3000 tokens x 8 heads, bf16; K4/V3 turbo layer
    and an int8 (per-vector absmax) boundary layer."""
    t = 3000
    k = inputs.lognormal_kv(1, t, 8, d, seed=8, layer=2, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, d, seed=8, layer=2, which=inputs.V)
    for layer in (H.Layer(d, 8, 8, k_bits=4, v_bits=3, seed=2),
                  H.Layer(d, 8, 8, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8, seed=0)):
        cache, st, word = H.gpu_quantize(layer, k, v, t)
        assert st == tq.TQ_OK and word == 0
        _check_quantized(layer, cache, _to_np(k), _to_np(v))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kb,vb", [(2, 3), (3, 4), (4, 2)])
def test_quantize_codes_every_width(d, kb, vb):
    """Every (head size, code width) pair through the quantise kernel's code
    grid: 333 tokens x 8 heads of bf16, K and V codes and norms against the
    oracle's code rule (2, 3 and 4 bits on each of d = 64, 128, 256)."""
    t = 333
    k = inputs.lognormal_kv(1, t, 8, d, seed=9, layer=kb, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, d, seed=9, layer=vb, which=inputs.V)
    layer = H.Layer(d, 8, 8, k_bits=kb, v_bits=vb, seed=3)
    cache, st, word = H.gpu_quantize(layer, k, v, t)
    assert st == tq.TQ_OK and word == 0
    _check_quantized(layer, cache, _to_np(k), _to_np(v))


def test_fp16_inputs_d64_group16():
    layer = H.Layer(64, 32, 2, k_bits=2, v_bits=4, seed=13)
    t = 700
    k = inputs.lognormal_kv(1, t, 2, 64, seed=9, layer=13, which=inputs.K, dtype=torch.float16)
    v = inputs.lognormal_kv(1, t, 2, 64, seed=9, layer=13, which=inputs.V, dtype=torch.float16)
    q = inputs.queries(1, 32, 64, seed=9, layer=13, dtype=torch.float16)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, [t])
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


@pytest.mark.parametrize("k_mode,v_mode", [(tq.TQ_MODE_INT8, tq.TQ_MODE_TURBO), (tq.TQ_MODE_TURBO, tq.TQ_MODE_INT8),
                                           (tq.TQ_MODE_INT8, tq.TQ_MODE_INT8)])
def test_attention_over_int8_sides(k_mode, v_mode):
    layer = H.Layer(128, 16, 4, k_bits=4, v_bits=2, k_mode=k_mode, v_mode=v_mode, seed=15)
    t = 900
    k = inputs.lognormal_kv(1, t, 4, 128, seed=10, layer=15, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 4, 128, seed=10, layer=15, which=inputs.V)
    q = inputs.queries(1, 16, 128, seed=10, layer=15)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, [t])
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


@pytest.mark.parametrize("hq,v_bits,lens", [(32, 2, [3001, 1700]), (64, 4, [1200, 1]), (16, 3, [777]),
                                           (32, "int8", [3001, 1700]), (64, "int8", [1200, 1]), (16, "int8", [777]),
                                           (128, 2, [900, 333]), (128, "int8", [900, 333]),
                                           (48, 2, [1000, 17]), (104, "int8", [700])])
def test_int8_keys_turbo_values_ragged(hq, v_bits, lens):
    """int8 keys beside turbo values (or int8 values: a boundary layer) in the
    tensor-core kernel: several chunks, ragged tails, a one-token sequence,
    GQA groups of 2, 4, 6, 8, 13 and 16 (groups above 4 combine the warps in
    passes of four heads, the last pass of 6 and 13 a partial one)."""
    if v_bits == "int8":
        layer = H.Layer(128, hq, 8, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8, seed=19)
    else:
        layer = H.Layer(128, hq, 8, k_mode=tq.TQ_MODE_INT8, v_bits=v_bits, seed=19)
    t = max(lens)
    k = inputs.lognormal_kv(len(lens), t, 8, 128, seed=19, layer=3, which=inputs.K)
    v = inputs.lognormal_kv(len(lens), t, 8, 128, seed=19, layer=3, which=inputs.V)
    q = inputs.queries(len(lens), hq, 128, seed=19, layer=3)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, lens)
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())


def test_zero_vectors_and_single_token():
    layer = H.Layer(128, 4, 1, k_bits=3, v_bits=2, seed=17)
    k = torch.zeros(1, 3, 1, 128)
    v = torch.zeros(1, 3, 1, 128)
    # a generic (non-constant) vector: a constant one puts several rotated
    # coordinates exactly on the zero boundary, where ties are arbitrary
    v[0, 1, 0, :] = torch.randn(128, generator=torch.Generator().manual_seed(3))
    cache, st, _ = H.gpu_quantize(layer, k, v, 3)
    assert st == tq.TQ_OK
    assert np.all(cache.k_norms.cpu().numpy() == 0)
    kc = H.unpack_codes(cache.k_codes[0, 0].cpu().numpy(), 3, 128)
    assert np.all(kc == 3)
    q = torch.randn(1, 4, 128)
    out, st, _ = H.gpu_decode(layer, q, cache, [3])
    vhat = layer.oracle_decode(layer.oracle_encode(v[0, :, 0].double().numpy(), 1), 1)
    assert np.allclose(out[0], vhat.mean(axis=0)[None, :], atol=1e-5)  # zero keys: uniform weights
    out1, st, _ = H.gpu_decode(layer, q, cache, [1])
    assert np.allclose(out1, 0.0, atol=1e-6)  # one token with a zero value


def test_device_errors_are_reported_not_trapped():
    layer = H.Layer(128, 8, 2, seed=19)
    k = inputs.lognormal_kv(2, 4, 2, 128, seed=1, layer=0, which=inputs.K)
    v = inputs.lognormal_kv(2, 4, 2, 128, seed=1, layer=0, which=inputs.V)
    cache = tq.alloc_cache(layer.params, 2, 16)
    cache, st, word = H.gpu_quantize(layer, k, v, 16, positions=torch.tensor([0, 13], dtype=torch.int32), cache=cache)
    assert st == tq.TQ_ERR_DEVICE and word & tq.TQ_DEVERR_POSITION
    assert np.all(cache.k_norms[1].cpu().numpy() == 0)  # sequence 1 untouched
    assert np.any(cache.k_norms[0, :, :4].cpu().numpy() != 0)  # sequence 0 written
    q = inputs.queries(2, 8, 128, seed=1)
    out, st, word = H.gpu_decode(layer, q, cache, [4, 0], max_len=16)
    assert st == tq.TQ_ERR_DEVICE and word & tq.TQ_DEVERR_SEQLEN
    assert np.all(out[1] == 0) and np.all(np.isfinite(out[0]))
    out, st, word = H.gpu_decode(layer, q, cache, [4, 17], max_len=16)
    assert st == tq.TQ_ERR_DEVICE and word & tq.TQ_DEVERR_SEQLEN
    # the context is still usable afterwards
    out, st, word = H.gpu_decode(layer, q, cache, [4, 4])
    assert st == tq.TQ_OK and word == 0


def test_decode_is_deterministic():
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=21)
    t = 2100
    k = inputs.lognormal_kv(1, t, 8, 128, seed=12, layer=21, which=inputs.K)
    v = inputs.lognormal_kv(1, t, 8, 128, seed=12, layer=21, which=inputs.V)
    q = inputs.queries(1, 32, 128, seed=12, layer=21)
    cache, _, _ = H.gpu_quantize(layer, k, v, t)
    a, _, _ = H.gpu_decode(layer, q, cache, [t])
    b, _, _ = H.gpu_decode(layer, q, cache, [t])
    assert np.array_equal(a, b)


def test_workspace_reused_across_batches_and_lengths():
    """One workspace, zeroed once, serves calls of different batch sizes and
    lengths in any order; each result equals that of a fresh workspace."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=22)
    t = 3000
    k = inputs.lognormal_kv(4, t, 8, 128, seed=13, layer=22, which=inputs.K)
    v = inputs.lognormal_kv(4, t, 8, 128, seed=13, layer=22, which=inputs.V)
    q = inputs.queries(4, 32, 128, seed=13, layer=22)
    wide, _, _ = H.gpu_quantize(layer, k, v, t)
    narrow, _, _ = H.gpu_quantize(layer, k[:1], v[:1], t)
    ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, 4, t), dtype=torch.uint8, device="cuda")
    calls = [(wide, q, [t, 2500, 1777, 64]), (narrow, q[:1], [700]), (wide, q, [2000, 1, 999, 1500]),
             (narrow, q[:1], [t]), (wide, q, [t, t, t, t]), (narrow, q[:1], [257])]
    for cache, qq, lens in calls:
        got, st, word = H.gpu_decode(layer, qq, cache, lens, ws=ws)
        assert st == tq.TQ_OK and word == 0
        fresh, _, _ = H.gpu_decode(layer, qq, cache, lens)
        assert np.array_equal(got, fresh), lens


def test_group16_d128():
    """d = 128 with 16 query heads per kv head (the tensor-core kernel with two
    8-head column tiles, its warps combined in four passes), fp32 queries,
    ragged lengths, K4/V3."""
    layer = H.Layer(128, 32, 2, k_bits=4, v_bits=3, seed=23)
    t = 1100
    k = inputs.lognormal_kv(2, t, 2, 128, seed=14, layer=23, which=inputs.K)
    v = inputs.lognormal_kv(2, t, 2, 128, seed=14, layer=23, which=inputs.V)
    q = inputs.queries(2, 32, 128, seed=14, layer=23, dtype=torch.float32)
    e2e, same, _, _, _ = _attention_case(layer, k, v, q, [t, 517])
    assert same.max() < H.ATTN_TOL and e2e.max() < H.ATTN_TOL, (same.max(), e2e.max())
