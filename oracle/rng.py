"""Random numbers the method draws: rotation signs and the QJL sketch matrix.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

The pages fix no generator ([inferrs] "核心技术" and [fwht] "快速Walsh-Hadamard
变换（FWHT）预处理" name a random-sign Walsh-Hadamard rotation, [google]
"第二步：QJL" a 1-bit Johnson-Lindenstrauss sketch).  The reading adopted
here, and implemented independently by the CUDA library's host code, is:

* stream: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
  number generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, output =
  the published three-step xor-shift/multiply finaliser of the new state;
* rotation sign i (i = 0..d-1) is -1 when bit 63 of output i (state = seed)
  is set, else +1;
* QJL matrix S (m x d, row-major) holds iid N(0,1) entries made by the
  Box-Muller transform (Box & Muller 1958) from consecutive pairs of
  53-bit uniforms of the stream with state = seed XOR 0x5155414E544A4C00;
  pair k fills entries 2k and 2k+1 with r*cos(2*pi*u2) and r*sin(2*pi*u2),
  r = sqrt(-2 ln(1 - u1)); entries are then rounded to fp32.

Pure Python integers are used so that the 64-bit arithmetic is exact.
"""

import math

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
QJL_STREAM_XOR = 0x5155414E544A4C00


def splitmix64(state, count):
    """Return ``count`` consecutive SplitMix64 outputs starting from ``state``."""
    out = []
    s = state & MASK64
    for _ in range(count):
        s = (s + GOLDEN_GAMMA) & MASK64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def rotation_signs(seed, d):
    """Rotation sign vector s in {+1,-1}^d (fp64)."""
    words = splitmix64(seed, d)
    return np.array([-1.0 if (w >> 63) & 1 else 1.0 for w in words], dtype=np.float64)


def qjl_matrix(seed, m, d):
    """Gaussian sketch S (m x d), fp64 array holding fp32-rounded values."""
    n = m * d
    pairs = (n + 1) // 2
    words = splitmix64(seed ^ QJL_STREAM_XOR, 2 * pairs)
    vals = []
    for k in range(pairs):
        u1 = (words[2 * k] >> 11) * 2.0 ** -53
        u2 = (words[2 * k + 1] >> 11) * 2.0 ** -53
        r = math.sqrt(-2.0 * math.log(1.0 - u1))
        vals.append(r * math.cos(2.0 * math.pi * u2))
        vals.append(r * math.sin(2.0 * math.pi * u2))
    s = np.array(vals[:n], dtype=np.float64).astype(np.float32).astype(np.float64)
    return s.reshape(m, d)
