"""tq_append_decode_attention (append the step's token, then attend, in one
call) against the oracle: the appended token's codes, norms and QJL bits
follow the code rules, and the output matches the oracle's attention on the
GPU's stored codes.  The appended token is a fresh vector, so a missing cache
write cannot pass."""

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq

pytestmark = pytest.mark.gpu


def _np64(x):
    return x.float().cpu().numpy().astype(np.float64)


def _step_case(layer, t, lens, seed, dtype=torch.bfloat16):
    """Prefill t tokens per sequence with tq_quantize_append, then one fused
    step whose new token (a fresh vector) lands at lens[b] - 1."""
    bsz, hkv, d = len(lens), layer.hkv, layer.d
    k = inputs.lognormal_kv(bsz, t, hkv, d, seed=seed, layer=1, which=inputs.K, dtype=dtype)
    v = inputs.lognormal_kv(bsz, t, hkv, d, seed=seed, layer=1, which=inputs.V, dtype=dtype)
    kn = inputs.lognormal_kv(bsz, 1, hkv, d, seed=seed, layer=1, which=inputs.K, dtype=dtype, token_offset_seed=9)
    vn = inputs.lognormal_kv(bsz, 1, hkv, d, seed=seed, layer=1, which=inputs.V, dtype=dtype, token_offset_seed=9)
    q = inputs.queries(bsz, layer.hq, d, seed=seed, layer=1, dtype=dtype)
    cache, st, word = H.gpu_quantize(layer, k, v, t)
    assert st == tq.TQ_OK and word == 0
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, bsz, t), dtype=torch.uint8, device="cuda")
    out = torch.empty(bsz, layer.hq, d, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_append_decode_attention(layer.params, layer.kcb, layer.vcb, kn.cuda(), vn.cuda(), q.cuda(), cache, lens_t,
                                  t, out, ws, err)
    st, word = tq.tq_read_device_error(err)
    return cache, out.cpu().numpy(), st, word, (k, v, kn, vn, q)


def _check_appended(layer, cache, lens, kn, vn):
    """The appended token of every (b, kv head) against the oracle's encoding."""
    for b, n in enumerate(lens):
        for which, x, codes, norms in ((0, kn, cache.k_codes, cache.k_norms), (1, vn, cache.v_codes, cache.v_norms)):
            rows = _np64(x[b, 0])  # [Hkv, d]
            enc = layer.oracle_encode(rows, which)
            got_codes = codes[b, :, n - 1].cpu().numpy()
            got_norms = norms[b, :, n - 1].cpu().numpy().view(np.uint16)
            mode, bits = layer.side(which)
            if mode == tq.TQ_MODE_INT8:
                assert np.array_equal(got_codes, enc["bytes"])
                assert np.array_equal(got_norms, H.fp16_bits(enc["norm16"]))
                continue
            _, t_or = H.oracle_codebook(layer.d, bits)
            _, _, mism = H.check_codes(got_codes, enc, bits, layer.d, t_or)
            H.check_norms(got_norms, enc["norm16"])
            if which == 0 and layer.params.qjl_dims:
                H.check_qjl(cache.k_qjl[b, :, n - 1].cpu().numpy(), cache.k_gamma[b, :, n - 1].cpu().numpy(), enc,
                            mism, layer.params.qjl_dims)


def _check_attention(layer, cache, lens, q, got):
    bsz, hkv = len(lens), layer.hkv
    t = max(lens)
    for b, n in enumerate(lens):
        ks = np.stack([H.stored_hat(layer, cache, b, h, n, 0) for h in range(hkv)])[None]
        vs = np.stack([H.stored_hat(layer, cache, b, h, n, 1) for h in range(hkv)])[None]
        ref = H.oracle_attention(layer, _np64(q[b:b + 1]), ks, vs, [n])
        err = H.rel_l2_per_vector(got[b:b + 1], ref["out"])
        assert err.max() < H.ATTN_TOL, (b, err.max())


def test_step_llama8b_shaped():
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=41)
    lens = [3001]
    cache, got, st, word, (k, v, kn, vn, q) = _step_case(layer, 3001, lens, seed=41)
    assert st == tq.TQ_OK and word == 0
    _check_appended(layer, cache, lens, kn, vn)
    _check_attention(layer, cache, lens, q, got)


def test_step_qjl_group8_ragged():
    layer = H.Layer(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64, seed=43)
    lens = [1200, 867]
    cache, got, st, word, (k, v, kn, vn, q) = _step_case(layer, 1200, lens, seed=43)
    assert st == tq.TQ_OK and word == 0
    _check_appended(layer, cache, lens, kn, vn)
    _check_attention(layer, cache, lens, q, got)


@pytest.mark.parametrize("cfg", ["d64", "int8_v"])
def test_step_two_kernel_path(cfg):
    """Configurations outside the tensor-core kernel append with the quantise
    kernel and attend with the general kernels."""
    if cfg == "d64":
        layer = H.Layer(64, 8, 2, k_bits=4, v_bits=3, seed=45)
    else:
        layer = H.Layer(128, 16, 4, k_bits=4, v_mode=tq.TQ_MODE_INT8, seed=45)
    lens = [700, 350, 1]
    cache, got, st, word, (k, v, kn, vn, q) = _step_case(layer, 700, lens, seed=45)
    assert st == tq.TQ_OK and word == 0
    _check_appended(layer, cache, lens, kn, vn)
    _check_attention(layer, cache, lens, q, got)


@pytest.mark.parametrize("hq,v_bits", [(32, 2), (64, 3), (32, "int8")])
def test_step_int8_keys(hq, v_bits):
    """int8 keys with turbo values (the mixed setting), or with int8 values (a
    boundary layer), in the fused kernel: the appended rows are written as
    int8 bytes and fp16 scales, bit-exact with the oracle, and attention over
    the stored cache matches."""
    if v_bits == "int8":
        layer = H.Layer(128, hq, 8, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8, seed=51)
    else:
        layer = H.Layer(128, hq, 8, k_mode=tq.TQ_MODE_INT8, v_bits=v_bits, seed=51)
    lens = [2100, 1333, 5]
    cache, got, st, word, (k, v, kn, vn, q) = _step_case(layer, 2100, lens, seed=51)
    assert st == tq.TQ_OK and word == 0
    _check_appended(layer, cache, lens, kn, vn)
    _check_attention(layer, cache, lens, q, got)


def test_step_matches_separate_calls():
    """One fused call equals tq_quantize_append at seq_len - 1 followed by
    tq_decode_attention, on every output within the tolerance."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=47)
    t = 2600
    lens = [2600, 1999, 64]
    cache, got, st, word, (k, v, kn, vn, q) = _step_case(layer, t, lens, seed=47)
    assert st == tq.TQ_OK and word == 0
    sep, _, _ = H.gpu_quantize(layer, k, v, t)
    for b, n in enumerate(lens):  # one sequence at a time: the others' slots are untouched
        pos = torch.full((len(lens),), -1, dtype=torch.int32)
        pos[b] = n - 1
        kb = kn.clone()
        vb = vn.clone()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_append(layer.params, layer.kcb, layer.vcb, kb.cuda(), vb.cuda(), pos.cuda(), sep, err)
    want, st2, _ = H.gpu_decode(layer, q, sep, lens, max_len=t)
    assert st2 == tq.TQ_OK
    assert H.rel_l2_per_vector(got, want).max() < H.ATTN_TOL
    same = np.mean(sep.k_codes.cpu().numpy() == cache.k_codes.cpu().numpy())
    assert same > 0.9999, same


def test_step_bad_length_is_reported():
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=49)
    cache, got, st, word, _ = _step_case(layer, 256, [256, 0, 999], seed=49)
    assert st == tq.TQ_ERR_DEVICE and word & tq.TQ_DEVERR_SEQLEN


def test_early_prefetch_flag_same_results():
    """TQ_PARAM_PREFETCH_EARLY: two layers' steps alternate on one stream (the
    kernel before each call writes the other layer's cache, as the flag
    requires); every output equals the same sequence run without the flag."""
    t, steps = 1500, 3
    outs = {}
    for flags in (0, tq.TQ_PARAM_PREFETCH_EARLY):
        layers = [H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=60 + l) for l in range(2)]
        for layer in layers:
            layer.params.flags = flags
        ks = [inputs.lognormal_kv(1, t, 8, 128, seed=61, layer=l, which=inputs.K) for l in range(2)]
        vs = [inputs.lognormal_kv(1, t, 8, 128, seed=61, layer=l, which=inputs.V) for l in range(2)]
        caches = [H.gpu_quantize(layers[l], ks[l][:, : t - steps], vs[l][:, : t - steps], t)[0] for l in range(2)]
        torch.cuda.synchronize()
        ws = torch.zeros(tq.tq_decode_workspace_bytes(layers[0].params, 1, t), dtype=torch.uint8, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        res = []
        for i in range(steps):
            n = t - steps + i + 1
            lens = torch.tensor([n], dtype=torch.int32, device="cuda")
            for l in range(2):
                q = inputs.queries(1, 32, 128, seed=62, layer=l, step=i).cuda()
                out = torch.empty(1, 32, 128, dtype=torch.float32, device="cuda")
                tq.tq_append_decode_attention(layers[l].params, layers[l].kcb, layers[l].vcb,
                                              ks[l][:, n - 1:n].cuda(), vs[l][:, n - 1:n].cuda(), q, caches[l],
                                              lens, t, out, ws, err)
                res.append(out)
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK and word == 0
        outs[flags] = [r.cpu().numpy() for r in res]
    for a, b in zip(outs[0], outs[tq.TQ_PARAM_PREFETCH_EARLY]):
        assert np.array_equal(a, b)
