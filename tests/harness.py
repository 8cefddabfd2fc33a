"""Helpers for the GPU parity tests: build caches from the oracle, compare a
GPU cache with the oracle's encoding under the stated rules.

Comparison rules (the contract of the method's parity):
* codes: bit-exact, except that a code may sit in the adjacent cell when
  the oracle's rotated unit coordinate lies within 1e-5 of the boundary
  between the two cells; such codes must be fewer than 1e-4 of all codes;
* norms (fp16): within 1 fp16 ulp of the oracle's fp16(fp64 norm);
* QJL sign bits: compared on vectors whose codes all match; a bit may
  differ only where |(S r)_j| < 1e-5 ||r|| (same 1e-4 budget); gamma within
  1 fp16 ulp;
* int8 codes and scales: bit-exact (both sides perform the same fp32 steps);
* attention outputs: relative L2 error <= 2e-3 per (batch, query head)
  vector against the oracle's attention on the same codes.
"""

import functools
import math

import numpy as np
import torch

from bit_kv_cache_tq_b200 import tq
from oracle import attention as oatt
from oracle import codebook as ocb
from oracle import quantize as oq
from oracle import rng as orng

CODE_WINDOW = 1e-5
FLIP_BUDGET = 1e-4
ATTN_TOL = 2e-3


@functools.lru_cache(maxsize=None)
def oracle_codebook(d, bits):
    return ocb.lloyd_max(d, bits)


@functools.lru_cache(maxsize=None)
def oracle_signs(seed, d):
    return orng.rotation_signs(seed, d)


@functools.lru_cache(maxsize=None)
def oracle_sketch(seed, m, d):
    return orng.qjl_matrix(seed, m, d)


class Layer:
    """Everything both sides need for one layer: params and the two codebooks."""

    def __init__(self, d, hq, hkv, k_bits=4, v_bits=2, k_mode=tq.TQ_MODE_TURBO, v_mode=tq.TQ_MODE_TURBO,
                 qjl_dims=0, seed=0, sm_scale=0.0, tau=0.0):
        self.params = tq.make_params(d, hq, hkv, k_bits, v_bits, k_mode, v_mode, qjl_dims, seed, sm_scale, tau)
        self.d, self.hq, self.hkv = d, hq, hkv
        self.kcb = tq.tq_codebook_init(d, k_bits) if k_mode == tq.TQ_MODE_TURBO else None
        self.vcb = tq.tq_codebook_init(d, v_bits) if v_mode == tq.TQ_MODE_TURBO else None

    def side(self, which):
        p = self.params
        mode, bits = (p.k_mode, p.k_bits) if which == 0 else (p.v_mode, p.v_bits)
        return mode, bits

    def oracle_encode(self, x, which):
        """x [N, d] (any float) -> dict of oracle results for side `which`."""
        x = np.asarray(x, dtype=np.float64)
        mode, bits = self.side(which)
        if mode == tq.TQ_MODE_INT8:
            q, scale16 = oq.encode_int8(x.astype(np.float32))
            return {"mode": mode, "bytes": q.astype(np.int8).view(np.uint8), "norm16": scale16, "q": q}
        c, t = oracle_codebook(self.d, bits)
        s = oracle_signs(self.params.seed, self.d)
        sk = oracle_sketch(self.params.seed, self.params.qjl_dims, self.d) if (which == 0 and self.params.qjl_dims) else None
        enc = oq.encode_turbo(x, s, c, t, bits, qjl=sk)
        enc["mode"] = mode
        enc["bytes"] = enc["packed"]
        return enc

    def oracle_decode(self, enc, which):
        mode, bits = self.side(which)
        if mode == tq.TQ_MODE_INT8:
            return oq.dequantize_int8(enc["q"], enc["norm16"])
        c, _ = oracle_codebook(self.d, bits)
        s = oracle_signs(self.params.seed, self.d)
        if which == 0 and self.params.qjl_dims:
            sk = oracle_sketch(self.params.seed, self.params.qjl_dims, self.d)
            return oq.dequantize_turbo(enc["codes"], enc["norm16"], s, c, qjl=sk, qjl_bits=enc["qjl_bits"],
                                       gamma16=enc["gamma16"])
        return oq.dequantize_turbo(enc["codes"], enc["norm16"], s, c)


def fp16_bits(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def unpack_codes(packed, bits, d):
    """Codes of LSB-first packed bytes [..., d*bits/8] (comparison helper)."""
    stream = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=-1, bitorder="little")
    planes = stream.reshape(stream.shape[:-1] + (d, bits)).astype(np.int64)
    return np.sum(planes << np.arange(bits), axis=-1)


def check_codes(gpu_bytes, enc, bits, d, boundaries):
    """Apply the code rule; return (n_codes, n_adjacent_in_window, mismatched_vector_mask)."""
    gpu_bytes = np.asarray(gpu_bytes, dtype=np.uint8)
    same = np.all(gpu_bytes == enc["bytes"], axis=-1)
    n_codes = enc["codes"].size
    if np.all(same):
        return n_codes, 0, ~same
    g = unpack_codes(gpu_bytes[~same], bits, d)
    o = enc["codes"][~same]
    y = enc["rotated"][~same]
    diff = g != o
    assert np.all(np.abs(g - o)[diff] == 1), "a code moved by more than one cell"
    lower = np.minimum(g, o)[diff]
    dist = np.abs(y[diff] - np.asarray(boundaries)[lower])
    assert np.all(dist < CODE_WINDOW), "a code differs away from a boundary (%g)" % dist.max()
    flips = int(diff.sum())
    assert flips < FLIP_BUDGET * n_codes + 1, "too many boundary flips: %d of %d" % (flips, n_codes)
    return n_codes, flips, ~same


def check_norms(gpu_bits, oracle_fp16):
    a = np.asarray(gpu_bits).astype(np.uint16).astype(np.int32)
    b = fp16_bits(oracle_fp16).astype(np.int32)
    assert np.all(np.abs(a - b) <= 1), "norm differs by more than 1 fp16 ulp"


def check_qjl(gpu_qjl, gpu_gamma, enc, mismatched, m):
    ok = ~mismatched
    bits_gpu = np.unpackbits(np.asarray(gpu_qjl, dtype=np.uint8)[ok], axis=-1, bitorder="little")[:, :m]
    bits_or = enc["qjl_bits"][ok]
    diff = bits_gpu != bits_or
    if diff.any():
        proj = np.abs(enc["projection"][ok][diff])
        rn = np.broadcast_to(enc["residual_norm"][ok][:, None], diff.shape)[diff]
        assert np.all(proj < CODE_WINDOW * rn), "a QJL bit differs away from zero"
        assert diff.sum() < FLIP_BUDGET * diff.size + 1
    check_norms(np.asarray(gpu_gamma)[ok], enc["gamma16"][ok])


def rel_l2_per_vector(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    num = np.linalg.norm(got - want, axis=-1)
    den = np.maximum(np.linalg.norm(want, axis=-1), 1e-30)
    return num / den


def upload_oracle_cache(layer, cache, b, h, k_enc, v_enc, start=0):
    """Write oracle encodings of sequence b, kv head h into the device cache."""
    n = k_enc["bytes"].shape[0]
    dev = cache.k_codes.device
    sl = slice(start, start + n)
    cache.k_codes[b, h, sl] = torch.from_numpy(np.ascontiguousarray(k_enc["bytes"])).to(dev)
    cache.k_norms[b, h, sl] = torch.from_numpy(fp16_bits(k_enc["norm16"]).view(np.int16)).to(dev)
    cache.v_codes[b, h, sl] = torch.from_numpy(np.ascontiguousarray(v_enc["bytes"])).to(dev)
    cache.v_norms[b, h, sl] = torch.from_numpy(fp16_bits(v_enc["norm16"]).view(np.int16)).to(dev)
    if layer.params.qjl_dims:
        cache.k_qjl[b, h, sl] = torch.from_numpy(np.ascontiguousarray(k_enc["qjl_packed"])).to(dev)
        cache.k_gamma[b, h, sl] = torch.from_numpy(fp16_bits(k_enc["gamma16"]).view(np.int16)).to(dev)


def gpu_quantize(layer, k, v, capacity, positions=None, cache=None):
    """Quantise k, v ([B, T, Hkv, d] torch, CPU or CUDA) into a (new) cache at positions."""
    bsz = k.shape[0]
    if cache is None:
        cache = tq.alloc_cache(layer.params, bsz, capacity)
    if positions is None:
        positions = torch.zeros(bsz, dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_append(layer.params, layer.kcb, layer.vcb, k.cuda().contiguous(), v.cuda().contiguous(),
                          positions.cuda(), cache, err)
    st, word = tq.tq_read_device_error(err)
    return cache, st, word


def gpu_decode(layer, q, cache, lens, max_len=None, ws=None, with_mask=False):
    """Decode attention through the C ABI; a fresh zeroed workspace unless `ws` is given.
    with_mask: also return the Sparse-V skip mask as bool [B, Hq, max_len]."""
    bsz = q.shape[0]
    lens_t = torch.as_tensor(np.asarray(lens), dtype=torch.int32).cuda()
    max_len = int(max(lens)) if max_len is None else max_len
    if ws is None:
        ws = torch.zeros(tq.tq_decode_workspace_bytes(layer.params, bsz, max_len), dtype=torch.uint8, device="cuda")
    out = torch.empty(bsz, layer.hq, layer.d, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mask = torch.zeros(bsz, layer.hq, (max_len + 31) // 32, dtype=torch.int32, device="cuda") if with_mask else None
    tq.tq_decode_attention(layer.params, layer.kcb, layer.vcb, q.cuda().contiguous(), cache, lens_t, max_len, out, ws,
                           err, skip_mask=mask)
    st, word = tq.tq_read_device_error(err)
    if with_mask:
        return out.cpu().numpy(), st, word, unpack_mask(mask.cpu().numpy(), max_len)
    return out.cpu().numpy(), st, word


def unpack_mask(words, n):
    """int32 words [B, Hq, W] (bit i % 32 of word i / 32 = position i) -> bool [B, Hq, n]."""
    w = words.astype(np.uint32)
    bits = (w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(w.shape[0], w.shape[1], -1)[..., :n].astype(bool)


def stored_hat(layer, cache, b, h, n, which):
    """The oracle's reconstruction of the GPU's own stored bytes (codes, norms,
    QJL bits, gamma) for tokens [0, n) of sequence b, kv head h: attention
    parity is measured on the same codes, after code parity has passed."""
    mode, bits = layer.side(which)
    if which == 0:
        raw, nrm = cache.k_codes[b, h, :n].cpu().numpy(), cache.k_norms[b, h, :n].cpu().numpy()
    else:
        raw, nrm = cache.v_codes[b, h, :n].cpu().numpy(), cache.v_norms[b, h, :n].cpu().numpy()
    norm16 = nrm.view(np.float16)
    if mode == tq.TQ_MODE_INT8:
        return layer.oracle_decode({"q": raw.view(np.int8).astype(np.int64), "norm16": norm16}, which)
    enc = {"codes": unpack_codes(raw, bits, layer.d), "norm16": norm16}
    if which == 0 and layer.params.qjl_dims:
        m = layer.params.qjl_dims
        z = cache.k_qjl[b, h, :n].cpu().numpy()
        enc["qjl_bits"] = np.unpackbits(z, axis=-1, bitorder="little")[:, :m]
        enc["gamma16"] = cache.k_gamma[b, h, :n].cpu().numpy().view(np.float16)
    return layer.oracle_decode(enc, which)


def oracle_attention(layer, q, khat, vhat, lens, tau=0.0, skip_mask=None):
    """q [B, Hq, d]; khat/vhat [B, Hkv, L, d] fp64; skip_mask bool [B, Hq, L] or None."""
    return oatt.decode_attention(np.asarray(q, dtype=np.float64), khat, vhat, lens,
                                 layer.params.sm_scale or None, sparse_tau=tau, skip_mask=skip_mask)
