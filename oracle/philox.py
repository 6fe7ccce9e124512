"""Counter-based random bits for attention dropout, in plain numpy.

TEST INFRASTRUCTURE ONLY (see attention.py): imported by the oracle, the
tests and nothing on the product path.

The pages pass ``dropout_p`` to flash_attn_func (Flash Attention | Hermes
Skill, Workflow 2, Step 2) but name no random generator, so this library
fixes one that the GPU kernels and this oracle can each compute from a
published definition: Philox4x32 with 10 rounds (Salmon, Moraes, Dror and
Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011, section 4.2).
A round maps the counter (c0, c1, c2, c3) under the key (k0, k1) to

    (hi(M1 * c2) ^ c1 ^ k0,  lo(M1 * c2),  hi(M0 * c0) ^ c3 ^ k1,  lo(M0 * c0))

with M0 = 0xD2511F53, M1 = 0xCD9E8D57 and hi/lo the upper/lower 32 bits of
the 64-bit product; between rounds the key is bumped by the Weyl constants
(0x9E3779B9, 0xBB67AE85).  The same rounds on 64-bit words (Philox4x64-10,
multipliers 0xD2E7470EE14C6C93 / 0xCA5A826395121157, bumps
0x9E3779B97F4A7C15 / 0xBB67AE8584CAA73B) are numpy's ``Philox`` bit
generator, which the tests use to check the round structure written here.

Dropout keep bits (this library's reading; the pages give none): for batch
b, query head h of H, query row i, key j, with a 64-bit seed and a 32-bit
offset (a per-call stream number),

    counter = (j // 8, i, b * H + h, offset),  key = (seed mod 2^32, seed // 2^32)
    u       = 16-bit half (j mod 2) of word (j mod 8) // 2 of Philox4x32-10(counter, key)
              (the low half for even j)
    keep    = u >= round(p * 65536)

so a key is kept with probability 1 - round(p * 65536) / 65536, and kept
probabilities are scaled by 1 / (1 - p).
"""

from __future__ import annotations

import numpy as np

M4x32 = (0xD2511F53, 0xCD9E8D57)
W4x32 = (0x9E3779B9, 0xBB67AE85)
M4x64 = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
W4x64 = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)

__all__ = ["philox4x32", "philox4x64_py", "dropout_threshold", "dropout_keep"]


def philox4x32(counter, key, rounds: int = 10) -> np.ndarray:
    """Philox4x32 on arrays: counter [..., 4], key [..., 2] (broadcast), uint32.
    Returns [..., 4] uint32."""
    c = np.asarray(counter, dtype=np.uint64) & 0xFFFFFFFF
    k = np.asarray(key, dtype=np.uint64) & 0xFFFFFFFF
    c0, c1, c2, c3 = (c[..., i] for i in range(4))
    k0, k1 = k[..., 0], k[..., 1]
    mask = np.uint64(0xFFFFFFFF)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + np.uint64(W4x32[0])) & mask
            k1 = (k1 + np.uint64(W4x32[1])) & mask
        p0 = np.uint64(M4x32[0]) * c0          # < 2^64: exact in uint64
        p1 = np.uint64(M4x32[1]) * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def philox4x64_py(counter, key, rounds: int = 10):
    """Philox4x64 on Python integers (one counter): the same rounds on 64-bit
    words.  Returns a tuple of four ints."""
    mask = (1 << 64) - 1
    c0, c1, c2, c3 = (int(x) & mask for x in counter)
    k0, k1 = (int(x) & mask for x in key)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + W4x64[0]) & mask
            k1 = (k1 + W4x64[1]) & mask
        p0 = M4x64[0] * c0
        p1 = M4x64[1] * c2
        hi0, lo0 = p0 >> 64, p0 & mask
        hi1, lo1 = p1 >> 64, p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def dropout_threshold(p: float) -> int:
    """The 16-bit threshold of a dropout probability p in [0, 1): keys whose
    value is below it are dropped."""
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return int(round(p * 65536.0))


def dropout_keep(seed: int, offset: int, b: int, h: int, H: int, rows, n_k: int, p: float) -> np.ndarray:
    """Boolean [len(rows), n_k]: True where key j is kept for query row i of
    (batch b, query head h); the rule in the module docstring."""
    rows = np.asarray(rows, dtype=np.int64)
    t = dropout_threshold(p)
    j = np.arange(n_k, dtype=np.int64)
    groups = np.arange((n_k + 7) // 8, dtype=np.int64)
    ctr = np.zeros((rows.shape[0], groups.shape[0], 4), dtype=np.uint64)
    ctr[..., 0] = groups[None, :]
    ctr[..., 1] = rows[:, None]
    ctr[..., 2] = b * H + h
    ctr[..., 3] = offset & 0xFFFFFFFF
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    words = philox4x32(ctr, key)                        # [R, G, 4]
    halves = np.stack([words & 0xFFFF, words >> 16], axis=-1).reshape(rows.shape[0], -1)   # [R, 8G]
    u = halves[:, :n_k].astype(np.int64)
    return u >= t
