"""Pins for the fp64 oracle, independent of the oracle's own code (CPU only).

Each pin checks the oracle against something other than itself: a pure-Python brute
force, closed forms, invariants of softmax attention, central finite differences,
torch's fp64 CPU scaled_dot_product_attention, and the published SplitMix64 stream.
A plausible slip anywhere in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong mask direction, dropout scaling applied to lse) fails at
least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.dropout import keep_mask, keep_threshold, splitmix64_mix
from exact_io_aware_68_b200.workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M64 = (1 << 64) - 1


def _rand(shape, seed, factor=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * factor


# ----------------------------------------------------------------------------- brute force
def _bf_keep(seed, b, h, H, N, i, j, p):
    """Pure-Python-int counter hash (pinned below to the published SplitMix64 stream): one draw per
    four key columns, a 15-bit field of its 16-bit lane j % 4 against floor(p 2^15)."""
    g = ((b * H + h) * N + i) * ((N + 3) // 4) + j // 4
    z = (seed + (g + 1) * 0x9E3779B97F4A7C15) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    z ^= z >> 31
    thr = min(math.floor(float(np.float32(p)) * 2.0 ** 15), 2 ** 15 - 1)
    return ((z >> (16 * (j % 4))) & 0x7FFF) >= thr


def _brute_forward(q, k, v, scale, causal, key_lens, p, seed):
    """Triple loop over rows, keys and features; scalar math only."""
    B, H, N, d = q.shape
    dv = v.shape[3]
    O = [[[[0.0] * dv for _ in range(N)] for _ in range(H)] for _ in range(B)]
    L = [[[0.0] * N for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                s = []
                for j in range(N):
                    ok = (not causal or j <= i) and (key_lens is None or j < key_lens[b])
                    if ok:
                        acc = 0.0
                        for c in range(d):
                            acc += float(q[b, h, i, c]) * float(k[b, h, j, c])
                        s.append(acc * scale)
                    else:
                        s.append(None)
                vals = [x for x in s if x is not None]
                if not vals:
                    L[b][h][i] = -math.inf
                    continue
                m = max(vals)
                e = [0.0 if x is None else math.exp(x - m) for x in s]
                tot = sum(e)
                L[b][h][i] = m + math.log(tot)
                for j in range(N):
                    pij = e[j] / tot
                    if p > 0:
                        pij = pij / (1.0 - float(np.float32(p))) if _bf_keep(seed, b, h, H, N, i, j, p) else 0.0
                    for c in range(dv):
                        O[b][h][i][c] += pij * float(v[b, h, j, c])
    return np.array(O), np.array(L)


@pytest.mark.parametrize("N,causal,pad,p", [(1, False, False, 0.0), (3, True, False, 0.0),
                                            (5, False, True, 0.0), (7, True, True, 0.3),
                                            (8, False, False, 0.5), (6, True, False, 0.2)])
def test_brute_force_forward(N, causal, pad, p):
    B, H, d = 2, 2, 4
    q, k, v = (_rand((B, H, N, d), s) for s in (1, 2, 3))
    key_lens = np.array([max(1, N - 2), N], dtype=np.int32) if pad else None
    O, lse = oracle.forward(q, k, v, 0.7, causal, key_lens, p, 1234)
    Ob, lb = _brute_forward(q, k, v, 0.7, causal, key_lens, p, 1234)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- closed forms
def test_single_key_closed_form():
    q, k, v = (_rand((2, 3, 1, 8), s) for s in (4, 5, 6))
    O, lse = oracle.forward(q, k, v, 0.25)
    np.testing.assert_allclose(O, v, atol=1e-14)
    np.testing.assert_allclose(lse, 0.25 * np.einsum("bhnc,bhnc->bhn", q, k), atol=1e-14)
    # with dropout the single element is either kept (x 1/(1-p)) or dropped
    O, lse2 = oracle.forward(q, k, v, 0.25, dropout_p=0.5, seed=9)
    for b in range(2):
        for h in range(3):
            keep = _bf_keep(9, b, h, 3, 1, 0, 0, 0.5)
            np.testing.assert_allclose(O[b, h], v[b, h] * (2.0 if keep else 0.0), atol=1e-14)
    np.testing.assert_allclose(lse2, lse, atol=1e-14)   # lse ignores dropout


@pytest.mark.parametrize("causal,pad", [(False, False), (True, False), (False, True), (True, True)])
def test_zero_query_gives_mean_of_allowed_values(causal, pad):
    B, H, N, d = 2, 2, 9, 4
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 7), _rand((B, H, N, d), 8)
    key_lens = np.array([4, 9], dtype=np.int32) if pad else None
    O, lse = oracle.forward(q, k, v, 0.3, causal, key_lens)
    for b in range(B):
        for i in range(N):
            hi = i + 1 if causal else N
            if pad:
                hi = min(hi, int(key_lens[b]))
            np.testing.assert_allclose(O[b, :, i], v[b, :, :hi].mean(axis=1), atol=1e-14)
            np.testing.assert_allclose(lse[b, :, i], math.log(hi), atol=1e-14)


def test_causal_row_zero():
    q, k, v = (_rand((1, 2, 6, 4), s) for s in (10, 11, 12))
    O, lse = oracle.forward(q, k, v, 0.5, causal=True)
    np.testing.assert_allclose(O[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], 0.5 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-15)


def test_constant_values_give_constant_output():
    q, k = _rand((2, 2, 10, 4), 13), _rand((2, 2, 10, 4), 14)
    c = np.array([1.5, -2.0, 0.25, 3.0])
    v = np.broadcast_to(c, (2, 2, 10, 4)).copy()
    for causal, key_lens in [(False, None), (True, None), (False, np.array([3, 10]))]:
        O, _ = oracle.forward(q, k, v, 0.4, causal, key_lens)
        np.testing.assert_allclose(O, np.broadcast_to(c, O.shape), atol=1e-14)


def test_identity_values_expose_dropped_probabilities():
    """V = I (N <= d): row i of O is row i of P * Z / (1 - p), zero exactly where dropped."""
    B, H, N, d = 1, 2, 6, 8
    q, k = _rand((B, H, N, d), 15), _rand((B, H, N, d), 16)
    v = np.zeros((B, H, N, d))
    v[:, :, np.arange(N), np.arange(N)] = 1.0
    O, _, P, Z = oracle.forward(q, k, v, 0.35, False, None, 0.4, 77, return_p=True)
    np.testing.assert_allclose(O[..., :N], P * Z / (1 - float(np.float32(0.4))), atol=1e-15)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                for j in range(N):
                    assert (O[b, h, i, j] == 0.0) == (not _bf_keep(77, b, h, H, N, i, j, 0.4))


# ----------------------------------------------------------------------------- invariants
def test_probability_rows_sum_to_one():
    q, k, v = (_rand((2, 2, 12, 4), s) for s in (17, 18, 19))
    _, _, P, _ = oracle.forward(q, k, v, 0.5, True, np.array([5, 12]), return_p=True)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-14)
    assert np.all(P >= 0)
    # nothing leaks past a mask
    assert np.all(np.triu(P[0, 0], 1) == 0) and np.all(P[0, :, :, 5:] == 0)


def test_joint_key_value_permutation_invariance():
    q, k, v = (_rand((1, 2, 11, 4), s) for s in (20, 21, 22))
    perm = np.random.default_rng(0).permutation(11)
    O1, l1 = oracle.forward(q, k, v, 0.6)
    O2, l2 = oracle.forward(q, k[:, :, perm], v[:, :, perm], 0.6)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_key_shift_invariance():
    q, k, v = (_rand((1, 2, 9, 4), s) for s in (23, 24, 25))
    u = np.array([0.3, -1.2, 0.7, 2.0])
    O1, l1 = oracle.forward(q, k, v, 0.6, True)
    O2, l2 = oracle.forward(q, k + u, v, 0.6, True)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, 0.6 * q @ u, atol=1e-13)


def test_gradient_sum_identities():
    q, k, v, do = (_rand((2, 2, 10, 4), s) for s in (26, 27, 28, 29))
    for causal in (False, True):
        dq, dk, dv = oracle.backward(q, k, v, do, 0.45, causal, np.array([6, 10]))
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-12)


def test_fully_masked_row():
    q, k, v, do = (_rand((2, 1, 5, 4), s) for s in (30, 31, 32, 33))
    key_lens = np.array([0, 5], dtype=np.int32)
    O, lse = oracle.forward(q, k, v, 0.5, False, key_lens)
    assert np.all(O[0] == 0) and np.all(np.isneginf(lse[0])) and np.all(np.isfinite(lse[1]))
    dq, dk, dv = oracle.backward(q, k, v, do, 0.5, False, key_lens)
    assert np.all(dq[0] == 0) and np.all(dk[0] == 0) and np.all(dv[0] == 0)


# ----------------------------------------------------------------------------- gradients
@pytest.mark.parametrize("causal,pad,p", [(False, False, 0.0), (True, False, 0.0),
                                          (False, True, 0.0), (True, True, 0.25)])
def test_finite_difference_gradients(causal, pad, p):
    B, H, N, d = 1, 2, 7, 3
    q, k, v, do = (_rand((B, H, N, d), s) for s in (34, 35, 36, 37))
    key_lens = np.array([5], dtype=np.int32) if pad else None
    tau, seed, eps = 0.8, 5, 1e-6

    def loss(q_, k_, v_):
        O, _ = oracle.forward(q_, k_, v_, tau, causal, key_lens, p, seed)
        return float((O * do).sum())

    grads = oracle.backward(q, k, v, do, tau, causal, key_lens, p, seed)
    for which, g in enumerate(grads):
        fd = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += eps
            lp = loss(*args)
            args[which][idx] -= 2 * eps
            lm = loss(*args)
            fd[idx] = (lp - lm) / (2 * eps)
        rel = np.linalg.norm(fd - g) / max(np.linalg.norm(g), 1e-30)
        assert rel < 1e-6, (which, rel)


# ----------------------------------------------------------------------------- torch cross-check
@pytest.mark.parametrize("causal,pad", [(False, False), (True, False), (False, True)])
def test_matches_torch_sdpa_fp64(causal, pad):
    B, H, N, d = 2, 3, 33, 16
    q, k, v, do = (_rand((B, H, N, d), s) for s in (38, 39, 40, 41))
    key_lens = np.array([20, 33], dtype=np.int32) if pad else None
    tau = 1 / math.sqrt(d)
    O, _ = oracle.forward(q, k, v, tau, causal, key_lens)
    dq, dk, dv = oracle.backward(q, k, v, do, tau, causal, key_lens)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    mask = None
    if pad:
        mask = torch.zeros(B, 1, N, N, dtype=torch.bool)
        for b in range(B):
            mask[b, :, :, : key_lens[b]] = True
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, is_causal=causal,
                                                              scale=tau)
    to.backward(torch.tensor(do))
    np.testing.assert_allclose(O, to.detach().numpy(), atol=1e-12)
    for mine, theirs in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, theirs.grad.numpy(), atol=1e-11)


# ----------------------------------------------------------------------------- dropout hash
def test_hash_matches_published_splitmix64_stream():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "splitmix64_state0.txt"))
            if ln.strip() and not ln.startswith("#")]
    for ctr, want in rows:
        z = (int(ctr) + 1) * 0x9E3779B97F4A7C15 & M64   # seed 0
        got = int(splitmix64_mix(np.array([z], dtype=np.uint64))[0])
        assert got == int(want, 16)
    # the layout: (b, h, i, j) -> draw g = ((b*H + h)*N + i)*ceil(N/4) + j // 4, lane j % 4; with
    # seed 0, row 0 of head 0 takes draws 0, 1, 2 for columns 0-3, 4-7, 8-11
    H, N = 3, 13
    for p in (0.5, 0.1, 0.9):
        keep = keep_mask(0, 0, 0, H, N, [0], np.arange(12), p)
        thr = math.floor(float(np.float32(p)) * 2 ** 15)
        expect = [((int(w, 16) >> (16 * lane)) & 0x7FFF) >= thr for _, w in rows for lane in range(4)]
        assert list(keep[0]) == expect
    # a worked value: output 1 = 0xe220a8397b1dcdaf has 15-bit lanes 0x4daf, 0x7b1d, 0x2839, 0x6220
    assert [((0xE220A8397B1DCDAF >> (16 * k)) & 0x7FFF) for k in range(4)] == [0x4DAF, 0x7B1D, 0x2839, 0x6220]
    assert list(keep_mask(0, 0, 0, H, N, [0], [0, 1, 2, 3], 0.61)[0]) == [False, True, False, True]
    # draws of the next row start at ceil(N/4) = 4: row 1, column 0 is output 5 of the stream
    assert keep_mask(0, 0, 0, H, N, [1], [0], 0.5)[0, 0] == _bf_keep(0, 0, 0, H, N, 1, 0, 0.5)


def test_threshold_and_rates():
    assert keep_threshold(0.0) == 0
    assert keep_threshold(0.5) == 2 ** 14
    assert keep_threshold(0.1) == 3276            # floor(0.1 * 32768): drop rate 0.09998
    assert keep_threshold(0.9999999) == 2 ** 15 - 1
    w = WORKLOADS["bf16_keypad_dropout_16x16x512x64"]
    p, n, kept = w.dropout_p, 0, 0
    for b in range(w.B):
        for h in range(0, w.H, 4):
            km = keep_mask(w.seed, b, h, w.H, w.N, np.arange(w.N), np.arange(w.N), p)
            kept += int(km.sum())
            n += km.size
    sigma = math.sqrt(n * p * (1 - p))
    assert abs((n - kept) - n * p) < 4 * sigma
    # distinct heads draw distinct masks
    a = keep_mask(3, 0, 0, 16, 64, np.arange(64), np.arange(64), 0.5)
    b_ = keep_mask(3, 0, 1, 16, 64, np.arange(64), np.arange(64), 0.5)
    assert (a != b_).mean() > 0.3


# ----------------------------------------------------------------------------- long-context helpers
def test_row_subset_and_blocked_backward_match_full():
    B, H, N, d = 1, 2, 40, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (42, 43, 44, 45))
    O, lse = oracle.forward(q, k, v, 0.5, True, None, 0.2, 3)
    rows = np.array([0, 7, 39])
    Or, lr = oracle.forward_rows(q, k, v, 0.5, True, None, 0.2, 3, 0, 1, rows)
    np.testing.assert_allclose(Or, O[0, 1, rows], atol=1e-14)
    np.testing.assert_allclose(lr, lse[0, 1, rows], atol=1e-14)
    full = oracle.backward(q, k, v, do, 0.5, True, None, 0.2, 3)
    blk = oracle.backward_head_blocked(q, k, v, do, 0.5, True, None, 0.2, 3, 0, 1, block=16)
    for f, g in zip(full, blk):
        np.testing.assert_allclose(g, f[0, 1], atol=1e-13)


# ----------------------------------------------------------------------------- negative control
def _tiles_without_rescale(q, k, v, scale, tile):
    """Per-tile softmax accumulated with no running max / sum (the flawed sketch)."""
    N = q.shape[0]
    O = np.zeros_like(v)
    for i in range(0, N, tile):
        for j in range(0, N, tile):
            s = q[i:i + tile] @ k[j:j + tile].T * scale
            e = np.exp(s - s.max(1, keepdims=True))
            O[i:i + tile] += (e / e.sum(1, keepdims=True)) @ v[j:j + tile]
    return O


def _tiles_online(q, k, v, scale, tile):
    """Per-tile loop keeping running m and l, rescaling O whenever m grows."""
    N = q.shape[0]
    O = np.zeros_like(v)
    for i in range(0, N, tile):
        m = np.full(min(tile, N - i), -np.inf)
        l = np.zeros_like(m)
        acc = np.zeros((len(m), v.shape[1]))
        for j in range(0, N, tile):
            s = q[i:i + tile] @ k[j:j + tile].T * scale
            m_new = np.maximum(m, s.max(1))
            alpha = np.exp(m - m_new)
            p = np.exp(s - m_new[:, None])
            l = alpha * l + p.sum(1)
            acc = alpha[:, None] * acc + p @ v[j:j + tile]
            m = m_new
        O[i:i + tile] = acc / l[:, None]
    return O


def test_tiling_without_rescale_fails_and_online_softmax_matches():
    N, d = 512, 64
    q, k, v = (_rand((1, 1, N, d), s) for s in (46, 47, 48))
    O, _ = oracle.forward(q, k, v, 1 / 8)
    bad = _tiles_without_rescale(q[0, 0], k[0, 0], v[0, 0], 1 / 8, 256)
    good = _tiles_online(q[0, 0], k[0, 0], v[0, 0], 1 / 8, 256)
    assert np.abs(bad - O[0, 0]).max() > 1e-1
    np.testing.assert_allclose(good, O[0, 0], atol=1e-12)


# ----------------------------------------------------------------------------- decode-shaped forward
def _brute_decode(q, k, v, scale, causal, key_lens):
    """Scalar loops: query i of Nq is the token at position L - Nq + i of a cache of L valid keys."""
    B, H, Nq, d = q.shape
    Nkv, dv = k.shape[2], v.shape[3]
    O = np.zeros((B, H, Nq, dv))
    L_ = np.zeros((B, H, Nq))
    for b in range(B):
        L = Nkv if key_lens is None else int(key_lens[b])
        for h in range(H):
            for i in range(Nq):
                keys = [j for j in range(Nkv) if j < L and (not causal or j <= L - Nq + i)]
                if not keys:
                    L_[b, h, i] = -math.inf
                    continue
                s = {j: sum(float(q[b, h, i, c]) * float(k[b, h, j, c]) for c in range(d)) * scale for j in keys}
                m = max(s.values())
                e = {j: math.exp(x - m) for j, x in s.items()}
                tot = sum(e.values())
                L_[b, h, i] = m + math.log(tot)
                for j in keys:
                    for c in range(dv):
                        O[b, h, i, c] += e[j] / tot * float(v[b, h, j, c])
    return O, L_


@pytest.mark.parametrize("Nq,Nkv,causal,lens", [(1, 7, False, None), (3, 9, True, None), (4, 10, True, [10, 6]),
                                               (2, 6, False, [4, 0]), (5, 5, True, [5, 3])])
def test_decode_brute_force(Nq, Nkv, causal, lens):
    q, k, v = _rand((2, 2, Nq, 4), 60), _rand((2, 2, Nkv, 4), 61), _rand((2, 2, Nkv, 3), 62)
    kl = None if lens is None else np.array(lens, dtype=np.int32)
    O, L = oracle.forward_decode(q, k, v, 0.5, causal, kl)
    Ob, Lb = _brute_decode(q, k, v, 0.5, causal, kl)
    np.testing.assert_allclose(O, Ob, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(L), np.isneginf(Lb))
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], atol=1e-12)


def test_decode_rows_equal_the_last_rows_of_causal_self_attention():
    """The last Nq rows of causal self-attention over N tokens are decode rows against all N keys;
    with key padding to L, they are rows L - Nq .. L - 1 of causal self-attention over the first L."""
    N, Nq, d = 40, 6, 8
    q, k, v = (_rand((1, 2, N, d), s) for s in (63, 64, 65))
    O, L = oracle.forward(q, k, v, 0.3, True)
    Od, Ld = oracle.forward_decode(q[:, :, N - Nq:], k, v, 0.3, True)
    np.testing.assert_allclose(Od, O[:, :, N - Nq:], atol=1e-12)
    np.testing.assert_allclose(Ld, L[:, :, N - Nq:], atol=1e-12)
    Lk = 29
    O2, L2 = oracle.forward(q[:, :, :Lk], k[:, :, :Lk], v[:, :, :Lk], 0.3, True)
    qd = np.zeros((1, 2, Nq, d))
    qd[:] = q[:, :, Lk - Nq:Lk]
    Od2, Ld2 = oracle.forward_decode(qd, k, v, 0.3, True, np.array([Lk], dtype=np.int32))
    np.testing.assert_allclose(Od2, O2[:, :, Lk - Nq:], atol=1e-12)
    np.testing.assert_allclose(Ld2, L2[:, :, Lk - Nq:], atol=1e-12)


def test_decode_square_non_causal_is_self_attention_and_zero_query_is_a_mean():
    N, d = 12, 5
    q, k, v = (_rand((2, 1, N, d), s) for s in (66, 67, 68))
    O, L = oracle.forward(q, k, v, 0.4)
    Od, Ld = oracle.forward_decode(q, k, v, 0.4)
    np.testing.assert_allclose(Od, O, atol=1e-12)
    np.testing.assert_allclose(Ld, L, atol=1e-12)
    # q = 0: uniform weights over the allowed keys (causal: j <= L - Nq + i)
    Nq, Nkv, Lk = 3, 20, 17
    k2, v2 = _rand((1, 1, Nkv, d), 69), _rand((1, 1, Nkv, d), 70)
    Oz, Lz = oracle.forward_decode(np.zeros((1, 1, Nq, d)), k2, v2, 0.4, True, np.array([Lk], dtype=np.int32))
    for i in range(Nq):
        n_allowed = Lk - Nq + i + 1
        np.testing.assert_allclose(Oz[0, 0, i], v2[0, 0, :n_allowed].mean(0), atol=1e-12)
        assert abs(Lz[0, 0, i] - math.log(n_allowed)) < 1e-12
