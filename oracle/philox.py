"""Philox4x32-10 and the uniforms drawn by acceptance (oracle side).

Follows the published definition of Philox4x32 (Salmon, Moraes, Dror, Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 3.3): a
128-bit counter (c0, c1, c2, c3) and a 64-bit key (k0, k1); each of the 10
rounds multiplies c0 and c2 by the constants 0xD2511F53 and 0xCD9E8D57 into
64-bit products (hi, lo) and forms

    (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));

the key is bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85) before every
round after the first.  Vectorised over numpy arrays; uint64 holds each
32x32-bit product exactly.

Uniform stream used by the acceptance walk (one independent draw per decision,
so that every node's decision depends on its own draws only):

    key     = (seed mod 2^32, seed >> 32)
    counter = (node, sequence b, (tag << 28) | draw, step mod 2^32)
    u       = ((w0 << 32 | w1) >> 11) * 2^-53          in [0, 1)

tag 1 = accept test of a node's j-th child (draw = j), tag 2 = residual
sample after all children of a node were rejected, tag 3 = the per-node
sample of the deterministic-tree rule.
"""

from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint64(0x9E3779B9)
W1 = np.uint64(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)

TAG_CHILD = 1
TAG_RESIDUAL = 2
TAG_SPECEXEC = 3


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds.  All arguments are integer scalars or
    arrays of values in [0, 2^32); returns four uint64 arrays holding 32-bit
    words."""
    c0, c1, c2, c3, k0, k1 = (np.asarray(x, dtype=np.uint64) & MASK32
                              for x in (c0, c1, c2, c3, k0, k1))
    c0, c1, c2, c3, k0, k1 = np.broadcast_arrays(c0, c1, c2, c3, k0, k1)
    c0, c1, c2, c3 = c0.copy(), c1.copy(), c2.copy(), c3.copy()
    k0, k1 = k0.copy(), k1.copy()
    for r in range(10):
        if r > 0:
            k0 = (k0 + W0) & MASK32
            k1 = (k1 + W1) & MASK32
        p0 = M0 * c0            # < 2^64: exact in uint64
        p1 = M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0), lo1, (hi0 ^ c3 ^ k1), lo0
    return c0, c1, c2, c3


def uniform(seed: int, step: int, b, node, draw, tag):
    """The acceptance uniform for (sequence b, node, draw, tag): float64 in
    [0, 1) built from the top 53 bits of (w0, w1)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    k0 = seed & 0xFFFFFFFF
    k1 = seed >> 32
    draw = np.asarray(draw, dtype=np.uint64)
    tag = np.asarray(tag, dtype=np.uint64)
    c2 = ((tag << np.uint64(28)) | (draw & np.uint64(0x0FFFFFFF))) & MASK32
    w0, w1, _, _ = philox4x32_10(node, b, c2, int(step) & 0xFFFFFFFF, k0, k1)
    bits = ((w0 << np.uint64(32)) | w1) >> np.uint64(11)
    u = bits.astype(np.float64) * (2.0 ** -53)
    return u if np.ndim(u) else float(u)
