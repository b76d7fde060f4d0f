"""Rows whose rotation lands exactly on .5 rounding ties (test input builder).

The rotation of a row x is y = x R with R = I_G (x) H_n (Comfy-Org/comfy-quants
issue, section 1), and H_n = (J - 2I)^{(x)k} / 2^k is symmetric and orthogonal,
so R R = I.  Choosing y first and setting x = y R therefore gives a row whose
rotation is y exactly in real arithmetic.

y is sparse: at most nine nonzeros per group, each an odd multiple of s0 / 2
(the values +-0.5 s0 ... +-6.5 s0) or one +-7 s0 per row, with s0 a power of
two.  Every x entry is then an integer of magnitude <= 9 x 14 = 126 times
s0 / (2 sqrt(n)), so x is exact in bf16 (8 significant bits), and every
intermediate of a radix-4 butterfly evaluation (at most 4^k x 126 units) is
exact in fp32.  The row's absmax is 7 s0, the scale is s0 and y / s0 is an
exact half-integer wherever y is not 0 or +-7 s0: every such code is decided
by the tie rule alone (round half away from zero: 2.5 -> 3, -0.5 -> -1).

Built with numpy here; nothing in this module comes from the oracle or the
CUDA library.
"""
from __future__ import annotations

import numpy as np


def regular_hadamard(n: int) -> np.ndarray:
    """(J - 2I)^{(x)k} / 2^k by repeated numpy.kron, n = 4^k."""
    T = (np.ones((4, 4)) - 2 * np.eye(4)) / 2
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.kron(H, T)
    assert H.shape[0] == n
    return H


def exact_tie_rows(M: int, K: int, group: int, seed: int):
    """(x bf16 bits [M][K], y fp64 [M][K], s0 fp32 [M], codes int8 [M][K]).

    codes is the expected quantisation of y: round half away from zero of
    y / s0, which is exact here."""
    rng = np.random.default_rng(seed)
    H = regular_hadamard(group)
    G = K // group
    y = np.zeros((M, K))
    s0 = np.empty(M)
    for m in range(M):
        s = 2.0 ** int(rng.integers(-6, 3))
        s0[m] = s
        for g in range(G):
            nz = int(rng.integers(0, min(9, group + 1)))
            idx = rng.choice(group, size=nz, replace=False)
            half = rng.integers(0, 7, nz) + 0.5              # 0.5 .. 6.5
            sign = rng.choice([-1.0, 1.0], nz)
            y[m, g * group + idx] = sign * half * s
        j = int(rng.integers(0, K))
        y[m, j] = (7.0 if rng.random() < 0.5 else -7.0) * s
    x = (y.reshape(M, G, group) @ H).reshape(M, K)
    x32 = x.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), x), "x must be exact in fp32"
    bits32 = x32.view(np.uint32)
    assert not (bits32 & 0xFFFF).any(), "x must be exact in bf16"
    x_bits = (bits32 >> 16).astype(np.uint16)
    v = y / s0[:, None]
    codes = (np.sign(v) * np.floor(np.abs(v) + 0.5)).astype(np.int8)
    return x_bits, y, s0.astype(np.float32), codes
