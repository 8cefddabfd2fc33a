"""tq_decode_attention_static (library-owned scratch, no allocation) against
tq_decode_attention on a caller workspace.  Collected last on purpose: it must
pass both alone and after every other GPU test has used the device."""

import ctypes

import numpy as np
import pytest
import torch

import harness as H
from bit_kv_cache_tq_b200 import inputs, tq

pytestmark = pytest.mark.gpu


def _static(layer, q, cache, lens, max_len=None, expect_word=0):
    lens_t = torch.as_tensor(np.asarray(lens), dtype=torch.int32).cuda()
    out = torch.empty(q.shape[0], layer.hq, layer.d, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_decode_attention_static(layer.params, layer.kcb, layer.vcb, q.cuda().contiguous(), cache, lens_t,
                                  int(max_len or max(lens)), out, err)
    st, word = tq.tq_read_device_error(err)
    assert word == expect_word and st == (tq.TQ_OK if expect_word == 0 else tq.TQ_ERR_DEVICE), (st, word)
    return out.cpu().numpy()


def test_static_scratch_matches_workspace_entry_point():
    """Both entry points run the same deterministic launches, so the outputs
    agree bit for bit: two calls in a row on one shape, then other batch
    sizes and lengths."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=31)
    t = 3000
    k = inputs.lognormal_kv(3, t, 8, 128, seed=31, layer=31, which=inputs.K)
    v = inputs.lognormal_kv(3, t, 8, 128, seed=31, layer=31, which=inputs.V)
    q = inputs.queries(3, 32, 128, seed=31, layer=31)
    wide, _, _ = H.gpu_quantize(layer, k, v, t)
    narrow, _, _ = H.gpu_quantize(layer, k[:1], v[:1], t)
    for cache, qq, lens in [(wide, q, [t, 1999, 700]), (wide, q, [t, 1999, 700]), (narrow, q[:1], [t]),
                            (wide, q, [64, t, 1])]:
        want, st, word = H.gpu_decode(layer, qq, cache, lens)
        assert st == tq.TQ_OK and word == 0
        got = _static(layer, qq, cache, lens)
        assert np.array_equal(got, want), (lens, np.abs(got - want).max())


def test_static_scratch_after_a_rejected_length():
    """A call whose device-side length check fails (sequence 1 longer than
    max_seq_len: TQ_DEVERR_SEQLEN, zeros for that sequence) leaves the shared
    array fit for the next call, which again matches the workspace entry
    point bit for bit."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=32)
    t = 2500
    k = inputs.lognormal_kv(2, t, 8, 128, seed=32, layer=32, which=inputs.K)
    v = inputs.lognormal_kv(2, t, 8, 128, seed=32, layer=32, which=inputs.V)
    q = inputs.queries(2, 32, 128, seed=32, layer=32)
    cache, _, _ = H.gpu_quantize(layer, k, v, t)
    bad = _static(layer, q, cache, [1000, t], max_len=2000, expect_word=tq.TQ_DEVERR_SEQLEN)
    assert np.all(bad[1] == 0.0)
    for lens in ([t, 1234], [t, 1234]):
        want, st, word = H.gpu_decode(layer, q, cache, lens)
        assert st == tq.TQ_OK and word == 0
        assert np.array_equal(_static(layer, q, cache, lens), want), lens


def test_static_call_repairs_dirty_counters():
    """Every counter word of the shared array set to 0xFFFFFFFF from the host
    (the state an interrupted call could leave, made without faulting the
    GPU): the next static call's own zero fill repairs what it uses, so two
    calls in a row still match the workspace entry point bit for bit; a fill
    with 0 resets the array outright."""
    layer = H.Layer(128, 32, 8, k_bits=4, v_bits=2, seed=33)
    t = 2200
    k = inputs.lognormal_kv(2, t, 8, 128, seed=33, layer=33, which=inputs.K)
    v = inputs.lognormal_kv(2, t, 8, 128, seed=33, layer=33, which=inputs.V)
    q = inputs.queries(2, 32, 128, seed=33, layer=33)
    cache, _, _ = H.gpu_quantize(layer, k, v, t)
    want, st, word = H.gpu_decode(layer, q, cache, [t, 1500])
    assert st == tq.TQ_OK and word == 0
    tq.tq_decode_static_fill(0xFF)
    for _ in range(2):
        assert np.array_equal(_static(layer, q, cache, [t, 1500]), want)
    tq.tq_decode_static_fill(0)
    assert np.array_equal(_static(layer, q, cache, [t, 1500]), want)


def test_static_scratch_rejects_calls_beyond_its_size():
    """1024 sequences x 64 query heads need more partials than the array holds;
    the call fails before any device work (the cache pointers are never read)."""
    p = tq.make_params(128, 64, 8)
    kcb, vcb = tq.tq_codebook_init(128, 4), tq.tq_codebook_init(128, 2)
    fake = 1 << 20
    cache = tq.tq_cache(1024, 16, fake, fake, None, None, fake, fake, None)
    st = tq.library().tq_decode_attention_static(ctypes.byref(p), ctypes.byref(kcb), ctypes.byref(vcb), fake,
                                                 tq.TQ_BF16, ctypes.byref(cache), fake, 16, fake, None, None)
    assert st == tq.TQ_ERR_CAPACITY
    need = tq.tq_decode_workspace_bytes(p, 1024, 16)
    assert need > tq.TQ_DECODE_STATIC_SCRATCH_BYTES
