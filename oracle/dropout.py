"""Counter-based dropout decision for the oracle (test infrastructure only).

The sources make dropout an optional elementwise step on P ("FlashAttention 的第一原则",
section 2 and section 4.1, observation 4) but fix no random-number generator.  The
reading used on both sides of this library is a counter hash, so that the forward and
the backward regenerate the same mask without storing it.  One 64-bit draw decides four
consecutive key columns of a query row:

    W    = ceil(N / 4)                                  (draws per query row)
    g    = ((b * H + h) * N + i) * W + j // 4           (uint64; i = query row, j = key column)
    z    = seed + (g + 1) * 0x9E3779B97F4A7C15          (mod 2^64)
    x    = SplitMix64 output mix of z                   (Steele, Lea & Flood, OOPSLA 2014)
    u    = (x >> (16 * (j % 4))) & 0x7FFF                (the 15-bit draw of column j)
    thr  = min(floor(p * 2^15), 2^15 - 1)               (computed in fp64 from the fp32 p)
    keep = u >= thr

So the drop probability is thr / 2^15, p rounded down to a multiple of 2^-15.  For seed = 0
and b = h = i = 0, draw g is output g + 1 of a SplitMix64 generator started from state 0;
the tests pin the keep decisions of columns 0..11 to the published values.  Kept elements
are scaled by 1 / (1 - p) (inverted dropout); lse and the row sum use the undropped P.
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
    """15-bit threshold: an element is kept when its 15-bit draw is >= this value."""
    p32 = float(np.float32(p))
    return int(min(np.floor(p32 * 32768.0), 32767.0))


def keep_mask(seed: int, b: int, h: int, H: int, N: int, rows, cols, p: float) -> np.ndarray:
    """Boolean keep decisions for query rows ``rows`` x key columns ``cols`` of head (b, h)."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1, 1)
    cols = np.asarray(cols, dtype=np.uint64).reshape(1, -1)
    W = np.uint64((N + 3) // 4)
    base = np.uint64((b * H + h) * N)
    with np.errstate(over="ignore"):
        g = (base + rows) * W + (cols >> np.uint64(2))
        z = np.uint64(seed) + (g + np.uint64(1)) * GOLDEN_GAMMA
    x = splitmix64_mix(z)
    u = (x >> (np.uint64(16) * (cols & np.uint64(3)))) & np.uint64(0x7FFF)
    return u >= np.uint64(keep_threshold(p))
