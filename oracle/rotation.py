"""Random-sign Walsh-Hadamard rotation, written as a dense matrix product.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

[inferrs] section "核心技术" (item 2, Walsh-Hadamard rotation before
quantisation) and [fwht] section "2. 快速Walsh-Hadamard变换（FWHT）预处理"
(orthogonal, spreads energy, decorrelates, exactly invertible).  [tqai]
section "TurboQuant的核心创新" describes a Haar rotation instead; the
Walsh-Hadamard reading is the one adopted.

Reading: natural (Sylvester) order H[i, j] = (-1)^popcount(i & j), one sign
layer, normalised by 1/sqrt(d):

    R(x)    = H (s * x) / sqrt(d)
    R^-1(y) = s * (H y) / sqrt(d)

Deliberately no butterfly: an O(d^2) product with the explicit matrix.
"""

import numpy as np


def hadamard(d):
    """Sylvester-order Hadamard matrix of order d (a power of two), fp64."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d)
    anded = i[:, None] & i[None, :]
    parity = np.zeros_like(anded)
    for bit in range(int(d).bit_length()):
        parity ^= (anded >> bit) & 1
    return np.where(parity == 1, -1.0, 1.0)


def rotate(x, signs):
    """R(x) over the last axis of x."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = hadamard(d)
    return ((x * signs) @ h.T) / np.sqrt(d)


def unrotate(y, signs):
    """R^-1(y) over the last axis of y."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    h = hadamard(d)
    return signs * (y @ h.T) / np.sqrt(d)
