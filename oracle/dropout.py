"""Counter-based dropout decision for the oracle (test infrastructure only).

The sources make dropout an optional elementwise step on P ("FlashAttention 的第一原则",
section 2 and section 4.1, observation 4) but fix no random-number generator.  The
reading used on both sides of this library is a counter hash, so that the forward and
the backward regenerate the same mask without storing it:

    ctr  = ((b * H + h) * N + i) * N + j            (uint64; i = query row, j = key column)
    z    = seed + (ctr + 1) * 0x9E3779B97F4A7C15     (mod 2^64)
    z    = SplitMix64 output mix of z                 (Steele, Lea & Flood, OOPSLA 2014)
    r    = z >> 32                                    (uint32)
    thr  = min(floor(p * 2^32), 2^32 - 1)             (computed in fp64 from the fp32 p)
    keep = r >= thr

For seed = 0 and ctr = 0, 1, 2 the mixed values are the first three outputs of a
SplitMix64 generator started from state 0; the tests pin them to the published values.
Kept elements are scaled by 1 / (1 - p) (inverted dropout); lse and the row sum use the
undropped P.
"""
import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
MIX1 = np.uint64(0xBF58476D1CE4E5B9)
MIX2 = np.uint64(0x94D049BB133111EB)


def splitmix64_mix(z: np.ndarray) -> np.ndarray:
    """The SplitMix64 output function (xor-shift-multiply, shifts 30, 27, 31)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * MIX1
        z = (z ^ (z >> np.uint64(27))) * MIX2
    return z ^ (z >> np.uint64(31))


def keep_threshold(p: float) -> int:
    """uint32 threshold: an element is kept when its 32-bit draw is >= this value."""
    p32 = float(np.float32(p))
    return int(min(np.floor(p32 * 4294967296.0), 4294967295.0))


def keep_mask(seed: int, b: int, h: int, H: int, N: int, rows, cols, p: float) -> np.ndarray:
    """Boolean keep decisions for query rows ``rows`` x key columns ``cols`` of head (b, h)."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1, 1)
    cols = np.asarray(cols, dtype=np.uint64).reshape(1, -1)
    base = np.uint64((b * H + h) * N)
    with np.errstate(over="ignore"):
        ctr = (base + rows) * np.uint64(N) + cols
        z = np.uint64(seed) + (ctr + np.uint64(1)) * GOLDEN_GAMMA
    r = splitmix64_mix(z) >> np.uint64(32)
    return r >= np.uint64(keep_threshold(p))
