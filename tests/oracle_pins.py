"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle module it is
given is wrong.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutations.py`` runs them on copies with a planted mistake
(a dropped term, a wrong sign or index, a transposed operand) and checks
that some pin fails.

What pins what (none of them retypes the oracle's own formula):
* SplitMix64: published first outputs from state 0 (golden file).
* signs / QJL matrix: the first signs and the first Box-Muller pair derived
  by hand from the published SplitMix64 words (golden file); sign balance;
  Kolmogorov-Smirnov against scipy's normal CDF.
* rotation: scipy.linalg.hadamard; H H^T = d I in integers; norm
  preservation and exact inversion (page: the transform is orthogonal and
  invertible); closed form of the image of a basis vector.
* codebook: scipy.integrate.quad moments and centroid conditions; the
  uniform-density case d = 3 (textbook uniform quantiser); the 1-bit closed
  form E|X|; Max's 1960 Gaussian table in the d -> infinity limit; the
  pages' distortion factor (golden files); Monte-Carlo distortion through
  the full encode/decode pipeline against the closed-form D.
* packing: an independent big-integer bitstream construction.
* codes: brute-force nearest centroid.
* dequantisation: the decoded vector beats every one-code-moved decoding
  (nearest-neighbour cells through an orthogonal rotation).
* int8: hand-worked cases including round-half-even ties.
* QJL: statistical unbiasedness of the inner-product estimate (the
  property the page gives for the 1-bit residual), and the bias it removes.
* attention: one token, identical keys, zero query, the GQA head mapping,
  and the rotated-domain evaluation used by the kernels.
"""

import math

import numpy as np
import scipy.integrate
import scipy.linalg
import scipy.stats

from conftest import read_golden


# ----------------------------------------------------------------- rng
def pin_splitmix64(rng):
    gold = read_golden("splitmix64_state0.txt")
    outs = rng.splitmix64(0, 3)
    for i in range(3):
        assert outs[i] == int(gold[str(i)][0], 16), (i, hex(outs[i]))


def pin_sign_balance(rng):
    s = rng.rotation_signs(12345, 8192)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(np.mean(s)) < 4.0 / math.sqrt(8192)
    # signs of different seeds are not the same vector
    assert not np.array_equal(rng.rotation_signs(1, 256), rng.rotation_signs(2, 256))


def pin_first_signs(rng):
    """Seed 0: signs from bit 63 of the published SplitMix64 outputs (golden)."""
    gold = read_golden("qjl_first_pair.txt")
    want = np.array([float(x) for x in gold["signs_seed0"]])
    assert np.array_equal(rng.rotation_signs(0, len(want)), want)


def pin_first_qjl_pair(rng):
    """The sketch stream of seed 0x5155414E544A4C00 starts at state 0, so its
    first Box-Muller pair follows by hand from the published words (golden):
    u1 from the first word, cos term first, row-major fill."""
    gold = read_golden("qjl_first_pair.txt")
    seed = int(gold["qjl_seed"][0], 16)
    s = rng.qjl_matrix(seed, 64, 128)
    want = np.array([float(gold["qjl_s00"][0]), float(gold["qjl_s01"][0])]).astype(np.float32)
    assert np.array_equal(s[0, :2], want.astype(np.float64)), (s[0, :2], want)
    assert abs(s[0, 0] - float(gold["qjl_s00"][0])) < 1e-6 and abs(s[0, 1] - float(gold["qjl_s01"][0])) < 1e-6


def pin_qjl_gaussian(rng):
    s = rng.qjl_matrix(7, 64, 128)
    assert s.shape == (64, 128)
    assert np.array_equal(s, s.astype(np.float32).astype(np.float64))
    ks = scipy.stats.kstest(s.ravel(), scipy.stats.norm.cdf)
    assert ks.pvalue > 1e-4, ks
    # rows are not copies of each other (row-major fill of independent pairs)
    assert abs(np.corrcoef(s[0], s[1])[0, 1]) < 0.5


# ------------------------------------------------------------ rotation
def pin_hadamard(rot):
    for k in range(0, 9):
        d = 1 << k
        assert np.array_equal(rot.hadamard(d), scipy.linalg.hadamard(d).astype(np.float64))
        h = rot.hadamard(d).astype(np.int64)
        assert np.array_equal(h @ h.T, d * np.eye(d, dtype=np.int64))


def pin_rotation_orthogonal(rot, rng):
    gen = np.random.default_rng(0)
    for d in (4, 16, 128, 256):
        s = rng.rotation_signs(d, d)
        x = gen.standard_normal((8, d))
        y = rot.rotate(x, s)
        assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14, atol=0)
        assert np.allclose(rot.unrotate(y, s), x, rtol=0, atol=1e-13)
        assert np.allclose(rot.rotate(rot.unrotate(x, s), s), x, rtol=0, atol=1e-13)


def pin_rotation_basis(rot, rng):
    """R(e_j) = s_j H[:, j] / sqrt(d) and R^-1(e_i) = s * H[:, i] / sqrt(d)."""
    for d in (8, 256):
        s = rng.rotation_signs(99, d)
        h = scipy.linalg.hadamard(d).astype(np.float64)
        for j in (0, 1, d // 2 + 3, d - 1):
            e = np.zeros(d)
            e[j] = 1.0
            assert np.allclose(rot.rotate(e, s), s[j] * h[:, j] / math.sqrt(d), atol=1e-15)
            assert np.allclose(rot.unrotate(e, s), s * h[:, j] / math.sqrt(d), atol=1e-15)
    # d = 256: 1/sqrt(d) = 1/16 exactly, so a basis vector maps to exact +-1/16
    s = rng.rotation_signs(3, 256)
    e = np.zeros(256)
    e[5] = 1.0
    assert set(np.abs(rot.rotate(e, s))) == {1.0 / 16.0}


# ------------------------------------------------------------ codebook
def pin_density_moments(cb):
    for d in (3, 4, 8, 128, 256):
        total = scipy.integrate.quad(lambda x: float(cb.density(np.array([x]), d)[0]), -1, 1,
                                     points=[0.0], limit=200, epsabs=1e-14, epsrel=1e-13)[0]
        second = scipy.integrate.quad(lambda x: x * x * float(cb.density(np.array([x]), d)[0]), -1, 1,
                                      points=[0.0], limit=200, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(total - 1.0) < 1e-10, (d, total)
        assert abs(second - 1.0 / d) < 1e-10, (d, second)


def pin_uniform_case(cb):
    """d = 3: f is uniform on [-1, 1]; the Lloyd-Max quantiser is uniform."""
    for bits in (1, 2, 3, 4):
        n = 1 << bits
        c, t = cb.lloyd_max(3, bits)
        want = np.array([-1.0 + (2 * j + 1) / n for j in range(n)])
        assert np.allclose(c, want, atol=1e-12), (bits, c)
        assert np.allclose(t, 0.5 * (want[:-1] + want[1:]), atol=1e-12)


def pin_one_bit_closed_form(cb):
    """b = 1: c = +-E|X| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)); d = 4 gives 4/(3 pi)."""
    for d in (4, 8, 128, 256):
        c, t = cb.lloyd_max(d, 1)
        want = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
        assert abs(c[1] - want) < 1e-12 and abs(c[0] + want) < 1e-12, (d, c, want)
        assert abs(t[0]) < 1e-15
    c, _ = cb.lloyd_max(4, 1)
    assert abs(c[1] - 4.0 / (3.0 * math.pi)) < 1e-12


def pin_centroid_condition(cb):
    """Every centroid is the conditional mean of its cell (scipy quad)."""
    for d, bits in ((128, 2), (128, 3), (128, 4), (256, 3), (16, 4)):
        c, t = cb.lloyd_max(d, bits)
        edges = np.concatenate([[-1.0], t, [1.0]])
        f = lambda x: float(cb.density(np.array([x]), d)[0])
        for j in range(len(c)):
            a, b = edges[j], edges[j + 1]
            mass = scipy.integrate.quad(f, a, b, epsabs=1e-15, epsrel=1e-13, limit=200)[0]
            mom = scipy.integrate.quad(lambda x: x * f(x), a, b, epsabs=1e-16, epsrel=1e-13, limit=200)[0]
            assert abs(mom / mass - c[j]) < 1e-9 * max(1.0, abs(c[j]) * math.sqrt(d)), (d, bits, j)
        assert np.allclose(c, -c[::-1], atol=0)
        assert np.all(np.diff(c) > 0)
        assert np.allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-16)


def pin_gaussian_limit(cb):
    gold = read_golden("gaussian_lloyd_max.txt")
    for bits in (1, 2, 3, 4):
        want = np.array([float(v) for v in gold[str(bits)]])
        g, _ = cb.gaussian_lloyd_max(bits)
        half = g[len(g) // 2:]
        assert np.allclose(half, want, rtol=6e-4, atol=6e-4), (bits, half, want)
        c, _ = cb.lloyd_max(8192, bits)
        scaled = c[len(c) // 2:] * math.sqrt(8192)
        assert np.allclose(scaled, half, rtol=2e-3, atol=2e-3), (bits, scaled, half)


def pin_distortion(cb):
    """D from the closed-form identity equals direct quadrature of the MSE, and
    4^-b <= d D <= 2.72 * 4^-b (the pages' factor of about 2.7)."""
    gold = read_golden("distortion_bound.txt")
    lo, hi = float(gold["lower_factor"][0]), float(gold["upper_factor"][0])
    for d, bits in ((4, 1), (8, 2), (16, 3), (16, 4), (128, 2), (128, 3), (128, 4), (256, 4)):
        c, t = cb.lloyd_max(d, bits)
        dd = cb.distortion(c, t, d)
        edges = np.concatenate([[-1.0], t, [1.0]])
        f = lambda x: float(cb.density(np.array([x]), d)[0])
        direct = sum(scipy.integrate.quad(lambda x: (x - c[j]) ** 2 * f(x), edges[j], edges[j + 1],
                                          epsabs=1e-16, epsrel=1e-12, limit=200)[0]
                     for j in range(len(c)))
        assert abs(direct - dd) < 1e-10 * max(dd, 1e-3), (d, bits, direct, dd)
        ratio = d * dd * 4.0 ** bits
        assert lo <= ratio <= hi, (d, bits, ratio)


# ------------------------------------------------------------ quantise
def pin_pack_bigint(q):
    gen = np.random.default_rng(1)
    for bits in (1, 2, 3, 4):
        for n in (8, 16, 128, 256):
            codes = gen.integers(0, 1 << bits, size=n)
            acc = 0
            for i, c in enumerate(codes):
                acc |= int(c) << (bits * i)
            want = np.frombuffer(acc.to_bytes(n * bits // 8, "little"), dtype=np.uint8)
            got = q.pack(codes[None, :], bits)[0]
            assert np.array_equal(got, want), (bits, n)
            assert np.array_equal(q.unpack(want[None, :], bits, n)[0], codes)


def pin_codes_nearest(q, cb, rng):
    """Codes are the nearest centroid of the rotated unit coordinate."""
    gen = np.random.default_rng(2)
    for bits in (2, 3, 4):
        c, t = cb.lloyd_max(128, bits)
        s = rng.rotation_signs(5, 128)
        x = gen.standard_normal((64, 128)) * np.exp(gen.standard_normal(128))
        enc = q.encode_turbo(x, s, c, t, bits)
        y = enc["rotated"]
        brute = np.argmin(np.abs(y[..., None] - c[None, None, :]), axis=-1)
        assert np.array_equal(enc["codes"], brute)
        # y is the rotation of the unit direction: a unit vector
        assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
        assert np.allclose(enc["norm16"].astype(np.float64), np.linalg.norm(x, axis=-1), rtol=2 ** -11)
    # zero vector: norm 0 and every code is the middle-lower cell 2^(b-1) - 1
    c, t = cb.lloyd_max(128, 3)
    enc = q.encode_turbo(np.zeros((1, 128)), rng.rotation_signs(5, 128), c, t, 3)
    assert float(enc["norm16"][0]) == 0.0
    assert np.all(enc["codes"] == 3)
    # a 3-4-5 vector has norm exactly 5
    v = np.zeros((1, 128))
    v[0, 0], v[0, 1] = 3.0, 4.0
    assert float(q.encode_turbo(v, rng.rotation_signs(5, 128), c, t, 3)["norm16"][0]) == 5.0


def pin_dequant_nearest(q, cb, rng):
    """Decoding inverts the encoder's rotation: with an exactly representable
    norm, the decoded vector is closer to x than any decoding with one code
    moved to a neighbouring cell (Lloyd-Max cells are nearest-neighbour cells
    and the rotation is orthogonal)."""
    gen = np.random.default_rng(3)
    for bits in (2, 3, 4):
        c, t = cb.lloyd_max(128, bits)
        s = rng.rotation_signs(11, 128)
        u = gen.standard_normal((4, 128))
        x = 2.5 * u / np.linalg.norm(u, axis=-1, keepdims=True)
        enc = q.encode_turbo(x, s, c, t, bits)
        assert np.all(enc["norm16"].astype(np.float64) == 2.5)
        best = np.linalg.norm(x - q.dequantize_turbo(enc["codes"], enc["norm16"], s, c), axis=-1)
        for trial in range(24):
            i = int(gen.integers(0, 128))
            moved = enc["codes"].copy()
            step = np.where(moved[:, i] == (1 << bits) - 1, -1, 1)
            moved[:, i] += step
            err = np.linalg.norm(x - q.dequantize_turbo(moved, enc["norm16"], s, c), axis=-1)
            assert np.all(err > best), (bits, i, err, best)


def pin_int8_cases(q):
    x = np.array([[127.0, -63.5, 2.5, 3.5, -2.5, 0.0, 126.5, -127.0]], dtype=np.float32)
    qq, sc = q.encode_int8(x)
    assert float(sc[0]) == 1.0
    assert qq[0].tolist() == [127, -64, 2, 4, -2, 0, 126, -127]
    qq, sc = q.encode_int8(np.zeros((1, 8), dtype=np.float32))
    assert float(sc[0]) == 0.0 and np.all(qq == 0)
    # absmax 254 -> scale 2; 3 / 2 = 1.5 -> 2 (half-even), 5 / 2 = 2.5 -> 2
    qq, sc = q.encode_int8(np.array([[254.0, 3.0, 5.0, -1.0]], dtype=np.float32))
    assert float(sc[0]) == 2.0 and qq[0].tolist() == [127, 2, 2, 0]
    assert np.allclose(q.dequantize_int8(qq, sc), [[254.0, 4.0, 4.0, 0.0]])


def pin_qjl_unbiased(q, cb, rng):
    """The QJL-corrected reconstruction gives unbiased inner products, and the
    codebook-only reconstruction does not (at 2 bits it shrinks them)."""
    d, m, bits, trials = 32, 32, 2, 1500
    c, t = cb.lloyd_max(d, bits)
    gen = np.random.default_rng(4)
    x = gen.standard_normal(d)
    query = x + 0.5 * gen.standard_normal(d)
    truth = float(query @ x)
    with_qjl, without = [], []
    for seed in range(trials):
        s = rng.rotation_signs(1000 + seed, d)
        sk = rng.qjl_matrix(1000 + seed, m, d)
        enc = q.encode_turbo(x[None, :], s, c, t, bits, qjl=sk)
        full = q.dequantize_turbo(enc["codes"], enc["norm16"], s, c, qjl=sk,
                                  qjl_bits=enc["qjl_bits"], gamma16=enc["gamma16"])[0]
        base = q.dequantize_turbo(enc["codes"], enc["norm16"], s, c)[0]
        with_qjl.append(float(query @ full))
        without.append(float(query @ base))
    with_qjl, without = np.array(with_qjl), np.array(without)
    se = np.std(with_qjl) / math.sqrt(trials)
    # fp16 norm and fp16 gamma leave a relative bias below 2^-10
    assert abs(np.mean(with_qjl) - truth) < 4 * se + 2e-3 * abs(truth), (np.mean(with_qjl), truth, se)
    se0 = np.std(without) / math.sqrt(trials)
    assert abs(np.mean(without) - truth) > 4 * se0, (np.mean(without), truth)


def pin_mc_distortion(q, cb, rng):
    """E||u - u_hat||^2 over uniform unit vectors equals d * D (4 sigma)."""
    gen = np.random.default_rng(5)
    for d, bits, n in ((4, 1, 40000), (8, 2, 40000), (16, 4, 40000), (128, 2, 6000), (128, 4, 6000)):
        c, t = cb.lloyd_max(d, bits)
        s = rng.rotation_signs(21, d)
        u = gen.standard_normal((n, d))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        enc = q.encode_turbo(u, s, c, t, bits)
        uhat = q.dequantize_turbo(enc["codes"], enc["norm16"], s, c)
        err = np.sum((u - uhat) ** 2, axis=-1)
        want = d * cb.distortion(c, t, d)
        assert abs(np.mean(err) - want) < 4 * np.std(err) / math.sqrt(n) + 1e-12, (d, bits, np.mean(err), want)


# ------------------------------------------------------------ attention
def pin_attention_special(att):
    gen = np.random.default_rng(6)
    d = 16
    # one token: o = v_0
    k = gen.standard_normal((1, 1, 1, d))
    v = gen.standard_normal((1, 1, 1, d))
    qv = gen.standard_normal((1, 1, d))
    assert np.allclose(att.decode_attention(qv, k, v, [1])["out"][0, 0], v[0, 0, 0], atol=1e-15)
    # identical keys: o = mean(v)
    k = np.repeat(gen.standard_normal((1, 1, 1, d)), 7, axis=2)
    v = gen.standard_normal((1, 1, 7, d))
    assert np.allclose(att.decode_attention(qv, k, v, [7])["out"][0, 0], v[0, 0].mean(axis=0), atol=1e-14)
    # zero query: uniform average, and only the first len_b positions count
    k = gen.standard_normal((1, 1, 9, d))
    v = gen.standard_normal((1, 1, 9, d))
    out = att.decode_attention(np.zeros((1, 1, d)), k, v, [5])["out"][0, 0]
    assert np.allclose(out, v[0, 0, :5].mean(axis=0), atol=1e-14)
    # a dominant key selects its value; scale 1/sqrt(d) is applied (s = 4 vs 0)
    k = np.zeros((1, 1, 2, d))
    k[0, 0, 0, 0] = 4.0 * math.sqrt(d)
    v = np.zeros((1, 1, 2, d))
    v[0, 0, 0, 0], v[0, 0, 1, 0] = 1.0, 0.0
    qv = np.zeros((1, 1, d))
    qv[0, 0, 0] = 1.0
    p0 = math.exp(4.0) / (math.exp(4.0) + 1.0)
    assert abs(att.decode_attention(qv, k, v, [2])["out"][0, 0, 0] - p0) < 1e-14
    # GQA: q head h reads kv head h // G
    k = np.zeros((1, 2, 3, d))
    v = np.stack([np.full((3, d), 1.0), np.full((3, d), 2.0)])[None]
    out = att.decode_attention(gen.standard_normal((1, 4, d)), k, v, [3])["out"][0]
    assert np.allclose(out[:, 0], [1.0, 1.0, 2.0, 2.0])


def pin_sparse_v(att):
    d = 4
    k = np.zeros((1, 1, 3, d))
    k[0, 0, 2, 0] = -100.0 * 2.0  # s_2 = -100 with the 1/sqrt(4) scale
    v = np.array([[[[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 1.0, 0]]]])
    qv = np.array([[[1.0, 0, 0, 0]]])
    r = att.decode_attention(qv, k, v, [3], sparse_tau=1e-6)
    den = 2.0 + math.exp(-100.0)
    assert np.allclose(r["exact_sparse"][0, 0], [1 / den, 1 / den, 0, 0], atol=1e-16)
    assert np.all(r["lo"] <= r["exact_sparse"] + 1e-16) and np.all(r["exact_sparse"] <= r["hi"] + 1e-16)
    assert np.all(r["lo"] <= r["out"] + 1e-16) and np.all(r["out"] <= r["hi"] + 1e-16)
    assert abs(r["skip_fraction"] - 1.0 / 3.0) < 1e-12


def pin_rotated_domain(att, q, cb, rng):
    """The kernels' rotated-domain evaluation equals original-domain attention."""
    gen = np.random.default_rng(7)
    d, n = 128, 50
    ck, tk = cb.lloyd_max(d, 3)
    cv, tv = cb.lloyd_max(d, 2)
    s = rng.rotation_signs(31, d)
    sk = rng.qjl_matrix(31, 64, d)
    kx = gen.standard_normal((n, d)) * 3
    vx = gen.standard_normal((n, d))
    qv = gen.standard_normal(d)
    ek = q.encode_turbo(kx, s, ck, tk, 3, qjl=sk)
    ev = q.encode_turbo(vx, s, cv, tv, 2)
    khat = q.dequantize_turbo(ek["codes"], ek["norm16"], s, ck, qjl=sk, qjl_bits=ek["qjl_bits"], gamma16=ek["gamma16"])
    vhat = q.dequantize_turbo(ev["codes"], ev["norm16"], s, cv)
    ref = att.decode_attention(qv[None, None], khat[None, None], vhat[None, None], [n])["out"][0, 0]
    k_y = ck[ek["codes"]] + (ek["gamma16"].astype(np.float64) * math.sqrt(math.pi / 2) / 64)[:, None] * ((2.0 * ek["qjl_bits"] - 1.0) @ sk)
    got = att.attention_rotated(qv, s, k_y, ek["norm16"], cv[ev["codes"]], ev["norm16"])
    assert np.allclose(got, ref, atol=1e-12, rtol=0)


def pin_masked_sum(att):
    """The sum with a given skip set (reading of [inferrs] "Sparse V：速度加成":
    dropped positions leave the numerator, never the denominator): an empty
    set gives full attention, the set E = {p_i < tau} gives the exact sparse
    sum, the full set gives zero, and a two-token hand case with weights
    3/4, 1/4 (score gap ln 3) dropping the second token gives 3/4 v_0."""
    gen = np.random.default_rng(3)
    q = gen.normal(size=(1, 2, 8))
    k = gen.normal(size=(1, 1, 40, 8)) * 3.0
    v = gen.normal(size=(1, 1, 40, 8))
    none = np.zeros((1, 2, 40), dtype=bool)
    r0 = att.decode_attention(q, k, v, [40], sparse_tau=0.05, skip_mask=none)
    assert np.allclose(r0["masked"], r0["out"], rtol=0, atol=1e-14)
    assert np.all(r0["mask_count"] == 0) and np.all(r0["mask_max_weight"] == 0)
    s = np.einsum("hd,ld->hl", q[0], k[0, 0]) / math.sqrt(8)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    e = (p < 0.05)[None]
    r1 = att.decode_attention(q, k, v, [40], sparse_tau=0.05, skip_mask=e)
    assert np.allclose(r1["masked"], r1["exact_sparse"], rtol=0, atol=1e-14)
    assert np.all(r1["mask_count"] == e.sum(axis=2)) and np.all(r1["mask_max_weight"] < 0.05)
    r2 = att.decode_attention(q, k, v, [40], skip_mask=np.ones((1, 2, 40), dtype=bool))
    assert np.all(r2["masked"] == 0.0)
    # hand case: keys chosen so that the scores differ by ln 3
    d = 4
    qq = np.array([[[2.0, 0.0, 0.0, 0.0]]])
    kk = np.zeros((1, 1, 2, d))
    kk[0, 0, 0, 0] = math.log(3.0)  # scores ln 3 and 0 (sm_scale 1/2)
    vv = np.array([[[[1.0, 2.0, 3.0, 4.0], [5.0, 6.0, 7.0, 8.0]]]])
    r3 = att.decode_attention(qq, kk, vv, [2], skip_mask=np.array([[[False, True]]]))
    assert np.allclose(r3["masked"][0, 0], 0.75 * vv[0, 0, 0], rtol=0, atol=1e-14)
    assert abs(r3["mask_max_weight"][0, 0] - 0.25) < 1e-14


def pin_prefill(att):
    """Chunked prefill: a chunk of one query is one decode step over start + 1
    positions; with identical keys (equal scores) query j's output is the
    plain mean of v_0 .. v_{start+j} (the causal prefix, itself included),
    which fixes the causal limit; with q = 0 the same holds for any keys."""
    gen = np.random.default_rng(5)
    d, hkv, hq, L = 16, 2, 4, 30
    k = gen.normal(size=(1, hkv, L, d))
    v = gen.normal(size=(1, hkv, L, d))
    q = gen.normal(size=(1, 1, hq, d))
    one = att.prefill_attention(q, k, v, [11])
    dec = att.decode_attention(q[:, 0], k, v, [12])["out"]
    assert np.allclose(one[:, 0], dec, rtol=0, atol=1e-14)
    same = np.broadcast_to(k[:, :, :1], k.shape).copy()
    qc = gen.normal(size=(1, 5, hq, d))
    out = att.prefill_attention(qc, same, v, [20])
    for j in range(5):
        for h in range(hq):
            want = v[0, h // (hq // hkv), :20 + j + 1].mean(axis=0)
            assert np.allclose(out[0, j, h], want, rtol=0, atol=1e-12), (j, h)
    zero = att.prefill_attention(np.zeros((1, 3, hq, d)), k, v, [7])
    for j in range(3):
        assert np.allclose(zero[0, j, 0], v[0, 0, :7 + j + 1].mean(axis=0), rtol=0, atol=1e-12)

