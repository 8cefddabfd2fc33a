"""KV vector encoding and decoding: norm, codes, packing, QJL bits, int8 mode.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

Steps, in the order the pages give them:

1. norm separation — [tqai] "TurboQuant的核心创新": the L2 norm is kept
   separately as FP16, only the direction is quantised.  Reading: IEEE
   round-to-nearest-even to fp16, overflow to +inf; the direction is
   x / ||x|| with the exact norm (not the rounded one); a zero vector has
   direction 0.
2. rotation — [inferrs] "核心技术"; see ``oracle.rotation``.
3. per-coordinate Lloyd-Max code — [tqai] "核心创新"; code_i = number of
   boundaries t_j with y_i > t_j (a value on a boundary takes the lower
   index).
4. bit packing ("turbo2/3/4") — [inferrs] "压缩格式对比".  Reading: one
   LSB-first bitstream per vector: bit k of the stream is bit (k mod 8) of
   byte k // 8, code i occupies stream bits [b*i, b*i + b).  3-bit codes
   therefore cross byte boundaries.
5. QJL residual on K (optional) — [google] "第二步：QJL —— 1 bit 清理殘差":
   a 1-bit Johnson-Lindenstrauss sketch of the quantisation residual,
   which removes the inner-product bias.  Reading: r = y - c[code] in the
   rotated unit-vector domain, gamma = ||r|| stored as fp16, z_j = 1 when
   (S r)_j >= 0 else 0 for the m x d Gaussian matrix S of ``oracle.rng``,
   packed LSB-first like the codes.  Reconstruction of the residual is
   gamma * sqrt(pi/2) / m * S^T (2z - 1).
6. int8 boundary-layer mode — [inferrs] "三个反直觉的关键发现" item 3
   (first and last layers kept at q8_0 precision).  Reading: per-vector
   absmax scale = fp16(fp32(absmax) / 127), r = fp32(1 / scale) correctly
   rounded, q_i = round-half-even of the fp32 product x_i * r, clamped to
   [-127, 127]; q = 0 when the scale is 0 or infinite.  These are the IEEE
   fp32 operations the kernel performs, so both sides decide every q_i
   identically.
"""

import math

import numpy as np

from . import rotation


def norm(x):
    """Exact (fp64) L2 norm over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return np.sqrt(np.sum(x * x, axis=-1))


def to_fp16(v):
    """IEEE round-to-nearest-even to binary16 (numpy's conversion), as fp16."""
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float16)


def codes_from_rotated(y, boundaries):
    """code_i = #{j : y_i > t_j}."""
    y = np.asarray(y, dtype=np.float64)
    t = np.asarray(boundaries, dtype=np.float64)
    return np.sum(y[..., None] > t, axis=-1).astype(np.int64)


def pack(codes, bits):
    """Pack integer codes [..., n] (each < 2^bits) into an LSB-first bitstream of
    bytes; a stream that is not a whole number of bytes is padded with zero bits."""
    codes = np.asarray(codes, dtype=np.int64)
    n = codes.shape[-1]
    bitplanes = (codes[..., None] >> np.arange(bits)) & 1
    stream = bitplanes.reshape(codes.shape[:-1] + (n * bits,)).astype(np.uint8)
    return np.packbits(stream, axis=-1, bitorder="little")


def unpack(packed, bits, n):
    """Inverse of ``pack``: bytes [..., n*bits/8] -> codes [..., n]."""
    packed = np.asarray(packed, dtype=np.uint8)
    stream = np.unpackbits(packed, axis=-1, bitorder="little")[..., : n * bits]
    planes = stream.reshape(packed.shape[:-1] + (n, bits)).astype(np.int64)
    return np.sum(planes << np.arange(bits), axis=-1)


def encode_turbo(x, signs, centroids, boundaries, bits, qjl=None):
    """Encode vectors x [..., d].

    Returns a dict with ``norm16`` (fp16), ``rotated`` (fp64 y, for the
    boundary-window parity rule), ``codes`` (int), ``packed`` (uint8) and,
    when ``qjl`` (the m x d matrix S) is given, ``gamma16`` (fp16) and
    ``qjl_packed`` (uint8, m/8 bytes) plus ``projection`` (S r, fp64).
    """
    x = np.asarray(x, dtype=np.float64)
    n = norm(x)
    safe = np.where(n > 0, n, 1.0)
    u = np.where((n > 0)[..., None], x / safe[..., None], 0.0)
    y = rotation.rotate(u, signs)
    codes = codes_from_rotated(y, boundaries)
    out = {"norm16": to_fp16(n), "rotated": y, "codes": codes, "packed": pack(codes, bits)}
    if qjl is not None:
        s = np.asarray(qjl, dtype=np.float64)
        r = y - np.asarray(centroids, dtype=np.float64)[codes]
        proj = r @ s.T
        z = (proj >= 0).astype(np.int64)
        out["gamma16"] = to_fp16(norm(r))
        out["projection"] = proj
        out["residual_norm"] = norm(r)
        out["qjl_bits"] = z
        out["qjl_packed"] = pack(z, 1)
    return out


def dequantize_turbo(codes, norm16, signs, centroids, qjl=None, qjl_bits=None, gamma16=None):
    """x_hat = ||x||_16 * R^-1(c[code] + [QJL] gamma_16 sqrt(pi/2)/m S^T (2z-1))."""
    yhat = np.asarray(centroids, dtype=np.float64)[np.asarray(codes)]
    if qjl is not None:
        s = np.asarray(qjl, dtype=np.float64)
        m = s.shape[0]
        zpm = 2.0 * np.asarray(qjl_bits, dtype=np.float64) - 1.0
        g = np.asarray(gamma16, dtype=np.float64)
        yhat = yhat + (g * math.sqrt(math.pi / 2.0) / m)[..., None] * (zpm @ s)
    return np.asarray(norm16, dtype=np.float64)[..., None] * rotation.unrotate(yhat, signs)


def encode_int8(x):
    """int8 boundary-layer mode; returns (q int64 [..., d], scale16 fp16 [...])."""
    x32 = np.asarray(x, dtype=np.float32)
    absmax = np.max(np.abs(x32), axis=-1)
    with np.errstate(over="ignore"):
        scale16 = (absmax / np.float32(127.0)).astype(np.float32).astype(np.float16)
    scale32 = scale16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        recip = (np.float32(1.0) / scale32).astype(np.float32)
        prod = (x32 * recip[..., None]).astype(np.float32)
    q = np.clip(np.rint(prod), -127, 127)
    q = np.where((scale32 > 0)[..., None] & np.isfinite(scale32)[..., None], q, 0)
    return q.astype(np.int64), scale16


def dequantize_int8(q, scale16):
    """x_hat = scale_16 * q."""
    return np.asarray(scale16, dtype=np.float64)[..., None] * np.asarray(q, dtype=np.float64)
