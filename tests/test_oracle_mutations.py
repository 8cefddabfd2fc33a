"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutation is applied with monkeypatch to the oracle module in memory
and undone after the test.
"""

import math

import numpy as np
import pytest

import oracle_pins as P
from oracle import attention, codebook, quantize, rng, rotation


def _fails(fn, *args):
    with pytest.raises((AssertionError, ValueError, IndexError, ZeroDivisionError)):
        fn(*args)


def test_sign_layer_outside_the_transform(monkeypatch):
    def bad_rotate(x, signs):
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        return signs * (x @ rotation.hadamard(d).T) / np.sqrt(d)
    monkeypatch.setattr(rotation, "rotate", bad_rotate)
    _fails(P.pin_rotation_basis, rotation, rng)


def test_missing_normalisation(monkeypatch):
    def bad_rotate(x, signs):
        x = np.asarray(x, dtype=np.float64)
        return (x * signs) @ rotation.hadamard(x.shape[-1]).T
    monkeypatch.setattr(rotation, "rotate", bad_rotate)
    _fails(P.pin_rotation_orthogonal, rotation, rng)


def test_inverse_without_signs(monkeypatch):
    def bad_unrotate(y, signs):
        y = np.asarray(y, dtype=np.float64)
        d = y.shape[-1]
        return (y @ rotation.hadamard(d).T) / np.sqrt(d)
    monkeypatch.setattr(rotation, "unrotate", bad_unrotate)
    _fails(P.pin_rotation_orthogonal, rotation, rng)


def test_wrong_hadamard_order(monkeypatch):
    real = rotation.hadamard
    monkeypatch.setattr(rotation, "hadamard", lambda d: real(d)[::-1].copy())
    _fails(P.pin_hadamard, rotation)


def test_density_exponent_off_by_one(monkeypatch):
    def bad_density(x, d):
        x = np.asarray(x, dtype=np.float64)
        return codebook.density_constant(d) * np.clip(1 - x * x, 0, None) ** ((d - 2) / 2.0)
    monkeypatch.setattr(codebook, "density", bad_density)
    _fails(P.pin_density_moments, codebook)


def test_centroid_numerator_sign(monkeypatch):
    real = codebook.cell_moment
    monkeypatch.setattr(codebook, "cell_moment", lambda a, b, d: -real(a, b, d) if a > 0 else real(a, b, d))
    _fails(P.pin_uniform_case, codebook)


def test_boundary_not_midpoint(monkeypatch):
    real = codebook.lloyd_max

    def bad(d, bits, **kw):
        c, t = real(d, bits, **kw)
        return c, 0.9 * t
    monkeypatch.setattr(codebook, "lloyd_max", bad)
    _fails(P.pin_centroid_condition, codebook)


def test_code_tie_goes_up(monkeypatch):
    monkeypatch.setattr(quantize, "codes_from_rotated",
                        lambda y, t: np.sum(np.asarray(y)[..., None] >= np.asarray(t), axis=-1))
    _fails(P.pin_codes_nearest, quantize, codebook, rng)


def test_code_off_by_one(monkeypatch):
    monkeypatch.setattr(quantize, "codes_from_rotated",
                        lambda y, t: np.maximum(np.sum(np.asarray(y)[..., None] > np.asarray(t), axis=-1) - 1, 0))
    _fails(P.pin_codes_nearest, quantize, codebook, rng)


def test_msb_first_packing(monkeypatch):
    def bad_pack(codes, bits):
        codes = np.asarray(codes, dtype=np.int64)
        n = codes.shape[-1]
        planes = (codes[..., None] >> np.arange(bits)) & 1
        stream = planes.reshape(codes.shape[:-1] + (n * bits,)).astype(np.uint8)
        return np.packbits(stream, axis=-1, bitorder="big")
    monkeypatch.setattr(quantize, "pack", bad_pack)
    _fails(P.pin_pack_bigint, quantize)


def test_decode_drops_norm(monkeypatch):
    real = quantize.dequantize_turbo
    monkeypatch.setattr(quantize, "dequantize_turbo",
                        lambda codes, norm16, *a, **k: real(codes, np.ones_like(norm16), *a, **k))
    _fails(P.pin_dequant_nearest, quantize, codebook, rng)


def test_qjl_missing_sqrt_pi_over_2(monkeypatch):
    real = quantize.dequantize_turbo

    def bad(codes, norm16, signs, centroids, qjl=None, qjl_bits=None, gamma16=None):
        if qjl is not None:
            gamma16 = np.asarray(gamma16, dtype=np.float64) / math.sqrt(math.pi / 2.0)
        return real(codes, norm16, signs, centroids, qjl=qjl, qjl_bits=qjl_bits, gamma16=gamma16)
    monkeypatch.setattr(quantize, "dequantize_turbo", bad)
    _fails(P.pin_qjl_unbiased, quantize, codebook, rng)


def test_int8_round_half_away(monkeypatch):
    def bad(x):
        x32 = np.asarray(x, dtype=np.float32)
        scale16 = (np.max(np.abs(x32), axis=-1) / np.float32(127)).astype(np.float16)
        s = scale16.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.sign(x32 / s) * np.floor(np.abs(x32 / s) + 0.5)
        q = np.where(s > 0, np.clip(q, -127, 127), 0)
        return q.astype(np.int64), scale16
    monkeypatch.setattr(quantize, "encode_int8", bad)
    _fails(P.pin_int8_cases, quantize)


def test_gqa_interleaved_mapping(monkeypatch):
    real = attention.decode_attention

    def bad(q, k_hat, v_hat, lens, sm_scale=None, sparse_tau=0.0):
        hq, hkv = q.shape[1], k_hat.shape[1]
        g = hq // hkv
        order = [h % hkv * g + h // hkv for h in range(hq)] if g > 1 else list(range(hq))
        out = real(q, k_hat, v_hat, lens, sm_scale, sparse_tau)
        out["out"] = out["out"][:, order]
        return out
    monkeypatch.setattr(attention, "decode_attention", bad)
    _fails(P.pin_attention_special, attention)


def test_missing_softmax_scale(monkeypatch):
    real = attention.decode_attention
    monkeypatch.setattr(attention, "decode_attention",
                        lambda q, k, v, lens, sm_scale=None, sparse_tau=0.0: real(q, k, v, lens, 1.0, sparse_tau))
    _fails(P.pin_attention_special, attention)


def test_rotated_path_without_key_norm(monkeypatch):
    real = attention.attention_rotated
    monkeypatch.setattr(attention, "attention_rotated",
                        lambda q, s, ky, kn, vy, vn, sm_scale=None: real(q, s, ky, np.ones_like(kn), vy, vn, sm_scale))
    _fails(P.pin_rotated_domain, attention, quantize, codebook, rng)


def test_splitmix_wrong_increment(monkeypatch):
    monkeypatch.setattr(rng, "GOLDEN_GAMMA", 0x9E3779B97F4A7C13)
    _fails(P.pin_splitmix64, rng)


# ----------------------------------------------- random-number readings
def test_sign_from_bit_zero(monkeypatch):
    def bad_signs(seed, d):
        words = rng.splitmix64(seed, d)
        return np.array([-1.0 if w & 1 else 1.0 for w in words], dtype=np.float64)
    monkeypatch.setattr(rng, "rotation_signs", bad_signs)
    _fails(P.pin_first_signs, rng)


def test_sign_inverted(monkeypatch):
    real = rng.rotation_signs
    monkeypatch.setattr(rng, "rotation_signs", lambda seed, d: -real(seed, d))
    _fails(P.pin_first_signs, rng)


def _box_muller(seed, m, d, swap_u=False, sin_first=False, column_major=False):
    n = m * d
    words = rng.splitmix64(seed ^ rng.QJL_STREAM_XOR, n + 1)
    vals = []
    for k in range((n + 1) // 2):
        u1 = (words[2 * k] >> 11) * 2.0 ** -53
        u2 = (words[2 * k + 1] >> 11) * 2.0 ** -53
        if swap_u:
            u1, u2 = u2, u1
        r = math.sqrt(-2.0 * math.log(1.0 - u1))
        c, s = r * math.cos(2.0 * math.pi * u2), r * math.sin(2.0 * math.pi * u2)
        vals += [s, c] if sin_first else [c, s]
    a = np.array(vals[:n], dtype=np.float64).astype(np.float32).astype(np.float64)
    return a.reshape(d, m).T.copy() if column_major else a.reshape(m, d)


@pytest.mark.parametrize("kind", ["swap_u", "sin_first", "column_major"])
def test_box_muller_readings(monkeypatch, kind):
    monkeypatch.setattr(rng, "qjl_matrix", lambda seed, m, d: _box_muller(seed, m, d, **{kind: True}))
    _fails(P.pin_first_qjl_pair, rng)


def test_box_muller_control():
    # the helper above, with no mistake planted, passes the pin
    class R:
        pass
    r = R()
    r.qjl_matrix = lambda seed, m, d: _box_muller(seed, m, d)
    P.pin_first_qjl_pair(r)


def test_masked_sum_drops_from_denominator(monkeypatch):
    """Renormalising over the kept positions (dropping skipped positions from
    the denominator too) must fail a pin."""
    real = attention.decode_attention

    def bad(q, k_hat, v_hat, lens, sm_scale=None, sparse_tau=0.0, skip_mask=None):
        res = real(q, k_hat, v_hat, lens, sm_scale, sparse_tau, skip_mask)
        if skip_mask is not None:
            qd = np.asarray(q, dtype=np.float64)
            g = qd.shape[1] // k_hat.shape[1]
            scale = sm_scale or 1.0 / math.sqrt(qd.shape[-1])
            for b in range(qd.shape[0]):
                n = int(lens[b])
                for h in range(qd.shape[1]):
                    s = scale * (k_hat[b, h // g, :n] @ qd[b, h])
                    p = np.exp(s - s.max())
                    p /= p.sum()
                    kept = p[~np.asarray(skip_mask[b, h, :n], dtype=bool)].sum()
                    res["masked"][b, h] = res["masked"][b, h] / kept if kept > 0 else 0.0
        return res
    monkeypatch.setattr(attention, "decode_attention", bad)
    _fails(P.pin_masked_sum, attention)


@pytest.mark.parametrize("shift", [0, 2])
def test_prefill_causal_limit_off_by_one(monkeypatch, shift):
    """Query j seeing positions up to start + j - 1 (itself excluded) or up to
    start + j + 1 (one token of the future) must fail a pin."""
    def bad(q, k_hat, v_hat, start, sm_scale=None):
        q = np.asarray(q, dtype=np.float64)
        out = np.zeros(q.shape)
        for b in range(q.shape[0]):
            for j in range(q.shape[1]):
                n = max(1, int(start[b]) + j + shift)
                out[b, j] = attention.decode_attention(q[b:b + 1, j], k_hat[b:b + 1], v_hat[b:b + 1], [n],
                                                       sm_scale)["out"][0]
        return out
    monkeypatch.setattr(attention, "prefill_attention", bad)
    _fails(P.pin_prefill, attention)
