"""Philox4x32-10 counter-based generator and the round's random-number layout.

Philox4x32-10 is the generator of Salmon, Moraes, Dror and Shaw, "Parallel
random numbers: as easy as 1, 2, 3" (SC'11), section 3: ten rounds of two
32x32->64 multiplications with the constants M0=0xD2511F53, M1=0xCD9E8D57,
the key bumped by the Weyl constants W0=0x9E3779B9, W1=0xBB67AE85 between
rounds.  The pages only say "Philox uniforms"; the counter layout below is
this project's own convention and is documented identically in the C header.

Counter layout (key = (seed lo32, seed hi32), c3 = low 32 bits of offset):
  c0 = (x >> 2) | (request << 18) | (purpose << 28), output word x & 3
  purpose 0  sibling sampling at an expanded node: c1,c2 = 64-bit path id
  purpose 1  acceptance coin of candidate node i:  c1 = i,  x = 0
  purpose 2  bonus race at stop node s:            c1 = s + 1 (root = 0)
Uniform: U = ((w >> 9) + 0.5) * 2^-23, strictly inside (0, 1); 23 random bits so
that U and 1 - U are exact in fp32 as well as fp64.
"""
import numpy as np

M0, M1 = 0xD2511F53, 0xCD9E8D57
W0, W1 = 0x9E3779B9, 0xBB67AE85
_MASK = 0xFFFFFFFF

PURPOSE_SIBLINGS = 0
PURPOSE_COIN = 1
PURPOSE_BONUS = 2


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over uint32-valued arrays; returns 4 uint64 arrays."""
    c = [np.asarray(v, dtype=np.uint64) & _MASK for v in (c0, c1, c2, c3)]
    c0, c1, c2, c3 = np.broadcast_arrays(*c)
    k0 = np.uint64(k0 & _MASK)
    k1 = np.uint64(k1 & _MASK)
    for _ in range(10):
        p0 = np.uint64(M0) * c0
        p1 = np.uint64(M1) * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(_MASK)
        hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(_MASK)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        k0 = np.uint64((int(k0) + W0) & _MASK)
        k1 = np.uint64((int(k1) + W1) & _MASK)
    return c0, c1, c2, c3


def uniform_from_word(w):
    """23-bit uniform strictly inside (0,1), exact in fp32 and fp64."""
    w = np.asarray(w, dtype=np.uint64)
    return ((w >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def _key(seed):
    return seed & _MASK, (seed >> 32) & _MASK


def uniforms(seed, offset, purpose, request, c1, c2, xs):
    """Uniforms for tokens ``xs`` (array) at one (purpose, request, c1, c2)."""
    xs = np.asarray(xs, dtype=np.uint64)
    if np.any(xs >= (1 << 20)):
        raise ValueError("token id beyond the 2^20 counter field")
    if request >= (1 << 10) or purpose >= 16:
        raise ValueError("request or purpose beyond its counter field")
    c0 = (xs >> np.uint64(2)) | np.uint64(request << 18) | np.uint64(purpose << 28)
    out = philox4x32_10(c0, c1 & _MASK, c2 & _MASK, offset & _MASK, *_key(seed))
    lane = (xs & np.uint64(3)).astype(np.int64)
    words = np.stack(out, axis=-1)
    return uniform_from_word(np.take_along_axis(words, lane[..., None], -1)[..., 0])


def path_id(ranks):
    """64-bit id of a tree node from its 0-based sibling ranks, root = ().

    4 bits per level (ranks < 16), depth in bits 60..63 (depth <= 15).
    """
    if len(ranks) > 15:
        raise ValueError("path too deep for the 64-bit id")
    v = 0
    for i, j in enumerate(ranks):
        if not 0 <= j < 16:
            raise ValueError("rank beyond 4 bits")
        v |= j << (4 * i)
    return v | (len(ranks) << 60)
