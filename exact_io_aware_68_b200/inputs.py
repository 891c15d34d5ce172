"""Seeded synthetic inputs shared by the tests, the bench and the host-side oracle.

This module draws numbers and rounds them to the storage type; it holds none of the
attention arithmetic.  Recipe (one generator per workload,
``numpy.random.default_rng(seed)``, PCG64):

1. Q, K, V, dO are drawn in that order, each as ``standard_normal((B, H, N, d))`` in
   fp64, then multiplied by the workload's factor.
2. With a key-padding range [lo, hi], ``key_lens = rng.integers(lo, hi + 1, B)``
   (int32) is drawn after dO.
3. bf16 workloads round every element fp64 -> fp32 (round to nearest even) -> bf16
   (round to nearest even, done here on the fp32 bit pattern).  fp32 workloads
   round fp64 -> fp32.

The draws are generated one (b, h) head at a time; a head-sized draw of N*d normals
consumes the generator exactly like the matching slice of one (B, H, N, d) draw, so
the chunking does not change the stream (tests check this).
"""
import numpy as np

from .workloads import Workload


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 with round-to-nearest-even; returns the uint16 bit patterns.

    NaN is not expected from normal draws and is not special-cased.
    """
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + rounding) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to fp64."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def _round(x64: np.ndarray, dtype: str):
    """Return (storage array, exact fp64 value of the stored element)."""
    x32 = x64.astype(np.float32)
    if dtype == "f32":
        return x32, x32.astype(np.float64)
    bits = f32_to_bf16_bits(x32)
    return bits, bf16_bits_to_f64(bits)


def draw_tensor(rng: np.random.Generator, shape, factor: float, dtype: str, exact: bool = True):
    """Draw one (B, H, N, d) tensor head by head; returns (storage, fp64 exact values or None)."""
    B, H, N, d = shape
    store = np.empty(shape, dtype=np.float32 if dtype == "f32" else np.uint16)
    ex = np.empty(shape, dtype=np.float64) if exact else None
    for b in range(B):
        for h in range(H):
            x = rng.standard_normal((N, d))
            if factor != 1.0:
                x = x * factor
            s, e = _round(x, dtype)
            store[b, h] = s
            if exact:
                ex[b, h] = e
    return store, ex


def make_inputs(w: Workload, N: int = None, B: int = None, H: int = None, seed: int = None,
                with_do: bool = True, exact: bool = True):
    """Draw the inputs of a workload (optionally with a smaller N, B or H for parity cases).

    Returns a dict with, for each of q, k, v (and do): ``<name>`` the storage array
    (uint16 bf16 bits or float32) and ``<name>64`` its exact fp64 value; plus
    ``key_lens`` (int32 [B] or None) and the scalar parameters.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    seed = w.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    shape = (B, H, N, w.d)
    out = {"B": B, "H": H, "N": N, "d": w.d, "dtype": w.dtype, "scale": w.scale,
           "causal": w.causal, "dropout_p": w.dropout_p, "seed": seed}
    names = ["q", "k", "v"] + (["do"] if with_do else [])
    for name in names:
        s, e = draw_tensor(rng, shape, w.factor, w.dtype, exact)
        out[name] = s
        out[name + "64"] = e
    if w.key_len_range is not None:
        lo, hi = w.key_len_range
        lo, hi = min(lo, N), min(hi, N)
        out["key_lens"] = rng.integers(lo, hi + 1, B).astype(np.int32)
    else:
        out["key_lens"] = None
    return out


def sampled_rows(seed: int, h: int, N: int, count: int) -> np.ndarray:
    """Query rows checked per head for long contexts: ``default_rng([seed, h]).choice``."""
    rng = np.random.default_rng([seed, h])
    return np.sort(rng.choice(N, size=min(count, N), replace=False))


def make_decode_inputs(B: int, H: int, Nq: int, Nkv: int, d: int, seed: int, key_len_range=None,
                       factor: float = 1.0, exact: bool = True):
    """Inputs of a decode-shaped call: Nq query rows against a cache of Nkv keys per head.

    One generator ``numpy.random.default_rng(seed)``: q [B,H,Nq,d], then k and v [B,H,Nkv,d],
    each standard normal x ``factor`` rounded to bf16 like ``make_inputs``; with a key-length range
    [lo, hi], ``key_lens = rng.integers(lo, hi + 1, B)`` (int32) follows.
    """
    rng = np.random.default_rng(seed)
    out = {"B": B, "H": H, "Nq": Nq, "Nkv": Nkv, "d": d, "scale": 1.0 / float(d) ** 0.5, "seed": seed}
    for name, n in (("q", Nq), ("k", Nkv), ("v", Nkv)):
        s, e = draw_tensor(rng, (B, H, n, d), factor, "bf16", exact)
        out[name] = s
        out[name + "64"] = e
    if key_len_range is not None:
        lo, hi = key_len_range
        out["key_lens"] = rng.integers(lo, hi + 1, B).astype(np.int32)
    else:
        out["key_lens"] = None
    return out
