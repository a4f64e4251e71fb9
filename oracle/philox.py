"""Philox4x32-10 and the uniform draws of the Psi-Spec sampler (oracle; test infrastructure).

Philox is the counter-based generator of Salmon, Moraes, Dror & Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), section 3 (the Philox
S-P network): a 4x32-bit counter and a 2x32-bit key; each of the 10 rounds
multiplies words 0 and 2 by two fixed odd constants, swaps and XORs the
high halves with the key, and the key is bumped by two Weyl constants between
rounds. The pages describe no generator; the decode step needs reproducible
uniforms that do not depend on the GPU launch shape, hence this choice.

Counter layout (one draw per word-0 output):
    counter = (index, step mod 2^32, step >> 32, stream), key = (seed mod 2^32, seed >> 32)
    index   = b*k + j (global sequence b, block position j; the bonus uses j = k)
    stream  = 0 draft, 1 accept, 2 residual, 3 bonus
Uniform: u = (x0 >> 8) * 2^-24, in [0, 1 - 2^-24]; exact in fp32 and fp64.
"""
from __future__ import annotations

import numpy as np

MASK32 = 0xFFFFFFFF
# Multipliers and Weyl key increments of Philox4x32 (Salmon et al. 2011, table 2).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
ROUNDS = 10

STREAM_DRAFT = 0
STREAM_ACCEPT = 1
STREAM_RESIDUAL = 2
STREAM_BONUS = 3


def _round(c, k):
    prod0 = PHILOX_M0 * c[0]
    prod1 = PHILOX_M1 * c[2]
    hi0, lo0 = prod0 >> 32, prod0 & MASK32
    hi1, lo1 = prod1 >> 32, prod1 & MASK32
    return [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]


def philox4x32_10(counter, key):
    """Scalar Philox4x32-10 on Python ints: 4 counter words, 2 key words -> 4 words."""
    c = [int(w) & MASK32 for w in counter]
    k = [int(w) & MASK32 for w in key]
    for r in range(ROUNDS):
        if r:
            k = [(k[0] + PHILOX_W0) & MASK32, (k[1] + PHILOX_W1) & MASK32]
        c = _round(c, k)
    return c


def philox4x32_10_np(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 (uint64 lanes hold 32-bit words); returns 4 uint32 arrays."""
    m32 = np.uint64(MASK32)
    c0, c1, c2, c3 = (np.asarray(v, dtype=np.uint64) & m32 for v in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & m32
    k1 = np.asarray(k1, dtype=np.uint64) & m32
    c0, c1, c2, c3, k0, k1 = np.broadcast_arrays(c0, c1, c2, c3, k0, k1)
    k0, k1 = k0.copy(), k1.copy()
    for r in range(ROUNDS):
        if r:
            k0 = (k0 + np.uint64(PHILOX_W0)) & m32
            k1 = (k1 + np.uint64(PHILOX_W1)) & m32
        p0 = np.uint64(PHILOX_M0) * c0      # < 2^64: no wrap
        p1 = np.uint64(PHILOX_M1) * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & m32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & m32)
    return tuple(v.astype(np.uint32) for v in (c0, c1, c2, c3))


def uniform24(x0):
    """u = (x >> 8) * 2^-24 from a 32-bit word (scalar or array), as float64."""
    if isinstance(x0, (int, np.integer)):
        return float(int(x0) >> 8) * 2.0 ** -24
    return (np.asarray(x0, dtype=np.uint64) >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


def draw_word0(seed: int, step: int, stream: int, index):
    """Word 0 of Philox at counter (index, step lo, step hi, stream), key (seed lo, seed hi)."""
    index = np.asarray(index, dtype=np.uint64)
    x0, _, _, _ = philox4x32_10_np(index, step & MASK32, (step >> 32) & MASK32, stream,
                                   seed & MASK32, (seed >> 32) & MASK32)
    return x0


def uniforms(seed: int, step: int, stream: int, index):
    """The sampler's uniforms u in [0,1) for the given counter indices."""
    return uniform24(draw_word0(seed, step, stream, index))


def uniform_scalar(seed: int, step: int, stream: int, index: int) -> float:
    """Scalar form of `uniforms` on the pure-int Philox (for small cases)."""
    x0 = philox4x32_10([index, step & MASK32, (step >> 32) & MASK32, stream],
                       [seed & MASK32, (seed >> 32) & MASK32])[0]
    return uniform24(x0)
