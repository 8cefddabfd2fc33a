"""Decode attention over dequantised K/V, and the Sparse-V bounds.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

[google] "再看速度" (attention computed from 4-bit TurboQuant keys) and
[inferrs] "Sparse V：速度加成" (attention gating skips the V work of
low-weight positions; it saves compute, not memory).

Per batch entry b and query head h, with kv head h // G (G = Hq / Hkv,
contiguous grouping) and sm_scale defaulting to 1/sqrt(d):

    s_i = sm_scale <q, k_hat_i>,  i < len_b
    p   = softmax(s)
    o   = sum_i p_i v_hat_i

computed in the original (unrotated) domain from the oracle's own
dequantised vectors.  ``attention_rotated`` is the same quantity computed
the way the kernels organise it (rotated query, centroid dot products,
rotated-domain V sum, one inverse rotation); the two agree because the
rotation is orthogonal, and a test checks that they do.

Sparse V.  The pages gate on the softmax weight with threshold 1e-6 but do
not say which weight estimate the gate sees during a one-pass kernel.  The
reading adopted: a position i may be dropped from the numerator for head h
only if p_i < tau (its exact weight), and the denominator always keeps it.
Any skip set M inside E = {i : p_i < tau} is admissible, so the oracle
returns the full output together with the exact per-coordinate interval
that every admissible M lands in:

    o_full - sum_{i in E} max(p_i v_i, 0)  <=  o_M  <=  o_full - sum_{i in E} min(p_i v_i, 0).
"""

import math

import numpy as np

from . import rotation


def _softmax(s):
    m = np.max(s)
    e = np.exp(s - m)
    return e / np.sum(e)


def decode_attention(q, k_hat, v_hat, lens, sm_scale=None, sparse_tau=0.0, skip_mask=None):
    """q [B, Hq, d]; k_hat, v_hat [B, Hkv, L, d]; lens [B].

    Returns dict: ``out`` [B, Hq, d] (no skipping), and when sparse_tau > 0
    also ``lo``/``hi`` (the admissible interval above), ``exact_sparse``
    (skip set = E) and ``skip_fraction`` (|E| / len, averaged).

    ``skip_mask`` (bool [B, Hq, >= max len], optional) is a skip set M per
    (b, h): then ``masked`` [B, Hq, d] is sum_{i not in M} p_i v_i with the
    denominator over every position, ``mask_max_weight`` [B, Hq] the largest
    exact weight p_i among the positions in M (0 when M is empty) and
    ``mask_count`` [B, Hq] the size of M below the length.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv = k_hat.shape[1]
    g = hq // hkv
    scale = 1.0 / math.sqrt(d) if not sm_scale else sm_scale
    out = np.zeros((bsz, hq, d))
    lo = np.zeros_like(out)
    hi = np.zeros_like(out)
    exact = np.zeros_like(out)
    skipped = []
    masked = np.zeros_like(out)
    mask_max = np.zeros((bsz, hq))
    mask_count = np.zeros((bsz, hq), dtype=np.int64)
    for b in range(bsz):
        n = int(lens[b])
        for h in range(hq):
            kv = h // g
            k = np.asarray(k_hat[b, kv, :n], dtype=np.float64)
            v = np.asarray(v_hat[b, kv, :n], dtype=np.float64)
            p = _softmax(scale * (k @ q[b, h]))
            out[b, h] = p @ v
            if skip_mask is not None:
                m = np.asarray(skip_mask[b, h, :n], dtype=bool)
                masked[b, h] = p[~m] @ v[~m]
                mask_max[b, h] = p[m].max() if m.any() else 0.0
                mask_count[b, h] = int(m.sum())
            if sparse_tau > 0:
                e = p < sparse_tau
                contrib = p[e, None] * v[e]
                lo[b, h] = out[b, h] - np.sum(np.maximum(contrib, 0.0), axis=0)
                hi[b, h] = out[b, h] - np.sum(np.minimum(contrib, 0.0), axis=0)
                exact[b, h] = p[~e] @ v[~e]
                skipped.append(np.mean(e))
    res = {"out": out}
    if skip_mask is not None:
        res.update(masked=masked, mask_max_weight=mask_max, mask_count=mask_count)
    if sparse_tau > 0:
        res.update(lo=lo, hi=hi, exact_sparse=exact, skip_fraction=float(np.mean(skipped)))
    return res


def attention_rotated(q, signs, k_yhat, k_norm, v_yhat, v_norm, sm_scale=None):
    """One (b, h) decode step in the rotated domain.

    q [d]; k_yhat, v_yhat [L, d] are the rotated-domain reconstructions
    (centroids, plus the QJL term for K); k_norm, v_norm [L] the stored norms.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if not sm_scale else sm_scale
    q_rot = rotation.rotate(q, signs)
    s = scale * np.asarray(k_norm, dtype=np.float64) * (np.asarray(k_yhat) @ q_rot)
    p = _softmax(s)
    acc = (p * np.asarray(v_norm, dtype=np.float64)) @ np.asarray(v_yhat, dtype=np.float64)
    return rotation.unrotate(acc, signs)


def prefill_attention(q, k_hat, v_hat, start, sm_scale=None):
    """Chunked prefill over a cache that already holds the chunk.

    q [B, C, Hq, d] are the queries of C new tokens of each sequence;
    k_hat, v_hat [B, Hkv, L, d] the reconstructed cache with the chunk at
    positions start[b] .. start[b] + C - 1.  Query j of sequence b attends
    causally to positions 0 .. start[b] + j (itself included), exactly as
    a decode step over start[b] + j + 1 tokens would ([google] table "M5 Max
    128GB 上的實測" and [inferrs] table "性能表现" measure prefill from the
    compressed cache; the pages give no other rule, so the chunk attends to
    its own tokens in compressed form, as the decode step attends to the
    token it appended).  Returns out [B, C, Hq, d].
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, c, hq, d = q.shape
    out = np.zeros((bsz, c, hq, d))
    for b in range(bsz):
        for j in range(c):
            r = decode_attention(q[b:b + 1, j], k_hat[b:b + 1], v_hat[b:b + 1], [int(start[b]) + j + 1], sm_scale)
            out[b, j] = r["out"][0]
    return out

