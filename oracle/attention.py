"""Plain fp64 attention, forward and backward, one (b, h) head at a time (test infrastructure only).

Notation follows the sources: Q, K, V, O are N x d per head; S = tau * Q K^T are the
scaled scores (tau = ``scale``, 1/sqrt(d) by default); P = softmax(S) row by row; the
saved per-row normaliser is lse = m + ln(l) with m the row max and l the row sum of
exp(S - m) ("48 FlashAttention", block "Tiling и online softmax" names m and l, block
"Backward — тоже без N×N" says the backward recomputes from them).

Readings where the sources are silent (each one is listed with the library's design notes):
* masks are additive -inf; causal keeps key j <= query i (top-left aligned); key
  padding keeps j < key_lens[b] and masks keys only;
* a row with no allowed key has O = 0, lse = -inf and zero gradients;
* dropout multiplies P elementwise by keep / (1 - p) after the softmax; l and lse use the
  undropped P; the keep decision is ``oracle.dropout.keep_mask``;
* gradients are the exact derivatives of the forward function above.

Inputs are float64 arrays; bf16 data enters as its exact fp64 value.
"""
import numpy as np

from .dropout import keep_mask


def allowed_mask(rows, N: int, causal: bool, key_len) -> np.ndarray:
    """allowed[i, j] for the given query rows: (not causal or j <= i) and j < key_len.

    "FlashAttention 的第一原则", section 2: masking is an optional elementwise step.
    """
    rows = np.asarray(rows).reshape(-1, 1)
    cols = np.arange(N).reshape(1, -1)
    ok = np.ones((rows.shape[0], N), dtype=bool)
    if causal:
        ok &= cols <= rows
    if key_len is not None:
        ok &= cols < int(key_len)
    return ok


def _softmax_rows(S: np.ndarray):
    """Row softmax of masked scores S (-inf = masked). Returns P, m, l, lse.

    "FlashAttention 的第一原则", section 4.2: the softmax is taken per row and needs the
    whole row; m is subtracted for stability.
    """
    m = S.max(axis=1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    E = np.exp(S - m_safe[:, None])          # exp(-inf) = 0 on masked entries
    l = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(l[:, None] > 0, E / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m_safe + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return P, m, l, lse


def _head_forward(q, k, v, scale, causal, key_len, p, seed, b, h, H, rows):
    """Forward for query ``rows`` of one head: returns O[rows], lse[rows], P, Z (Z=None if p=0).

    Steps in the order matmul -> scale -> mask -> softmax -> dropout -> matmul
    ("FlashAttention 的第一原则", section 3.2; "48 FlashAttention", sdpa block).
    """
    N = k.shape[0]
    S = (q[rows] @ k.T) * scale
    S = np.where(allowed_mask(rows, N, causal, key_len), S, -np.inf)
    P, _, _, lse = _softmax_rows(S)
    if p > 0.0:
        Z = keep_mask(seed, b, h, H, N, rows, np.arange(N), p).astype(np.float64)
        Pt = P * Z / (1.0 - float(np.float32(p)))
    else:
        Z = None
        Pt = P
    O = Pt @ v
    return O, lse, P, Z


def forward(q, k, v, scale, causal=False, key_lens=None, dropout_p=0.0, seed=0, return_p=False):
    """O [B,H,N,d] and lse [B,H,N] (natural log) of exact attention over every row.

    With ``return_p`` also returns P (undropped) [B,H,N,N] and the keep mask Z (or None).
    """
    B, H, N, _ = q.shape
    O = np.zeros(q.shape[:3] + (v.shape[3],))
    lse = np.zeros((B, H, N))
    Ps, Zs = [], []
    rows = np.arange(N)
    for b in range(B):
        kl = None if key_lens is None else int(key_lens[b])
        for h in range(H):
            O[b, h], lse[b, h], P, Z = _head_forward(q[b, h], k[b, h], v[b, h], scale, causal, kl,
                                                     dropout_p, seed, b, h, H, rows)
            if return_p:
                Ps.append(P)
                Zs.append(Z)
    if return_p:
        Pall = np.stack(Ps).reshape(B, H, N, N)
        Zall = None if dropout_p <= 0 else np.stack(Zs).reshape(B, H, N, N)
        return O, lse, Pall, Zall
    return O, lse


def forward_rows(q, k, v, scale, causal, key_lens, dropout_p, seed, b, h, rows):
    """O and lse of head (b, h) for a subset of query rows only (full rows, no tiling).

    Each output row depends only on its own score row, so evaluating the definition on
    a subset of rows is exact; used when N x N does not fit on the host.
    """
    H = q.shape[1]
    kl = None if key_lens is None else int(key_lens[b])
    O, lse, _, _ = _head_forward(q[b, h], k[b, h], v[b, h], scale, causal, kl, dropout_p, seed,
                                 b, h, H, np.asarray(rows))
    return O, lse


def _head_backward_rows(q, k, v, do, scale, causal, key_len, p, seed, b, h, H, rows):
    """Gradient contributions of query ``rows`` of one head.

    Returns dQ[rows] and this block's additive share of dK and dV.  With
    L = sum(dO * O) the chain rule through O = Pt V, Pt = P * Z / (1 - p), P = softmax(S),
    S = tau Q K^T gives:
      dV = Pt^T dO;  dPt = dO V^T;  dP = dPt * Z / (1 - p);  D_i = sum_j P_ij dP_ij;
      dS = P * (dP - D);  dQ = tau dS K;  dK = tau dS^T Q.
    """
    _, _, P, Z = _head_forward(q, k, v, scale, causal, key_len, p, seed, b, h, H, rows)
    keep_scale = 1.0 / (1.0 - float(np.float32(p))) if p > 0.0 else 1.0
    Pt = P if Z is None else P * Z * keep_scale
    dO = do[rows]
    dV = Pt.T @ dO
    dPt = dO @ v.T
    dP = dPt if Z is None else dPt * Z * keep_scale
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q[rows])
    return dQ, dK, dV


def backward(q, k, v, do, scale, causal=False, key_lens=None, dropout_p=0.0, seed=0):
    """dQ, dK, dV [B,H,N,d] of L = sum(dO * O), every head, every row at once."""
    B, H, N, _ = q.shape
    dQ = np.zeros(q.shape)
    dK = np.zeros(k.shape)
    dV = np.zeros(v.shape)
    rows = np.arange(N)
    for b in range(B):
        kl = None if key_lens is None else int(key_lens[b])
        for h in range(H):
            dQ[b, h], dK[b, h], dV[b, h] = _head_backward_rows(
                q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, kl, dropout_p, seed, b, h, H, rows)
    return dQ, dK, dV


def backward_head_blocked(q, k, v, do, scale, causal, key_lens, dropout_p, seed, b, h, block=1024):
    """dQ, dK, dV of one head with the query rows taken ``block`` at a time.

    Every row is still a full-row softmax; dK and dV are the sums of the per-block
    shares (the matmul over query rows split into partial sums).  Used for long contexts.
    """
    H, N = q.shape[1], q.shape[2]
    kl = None if key_lens is None else int(key_lens[b])
    dQ = np.zeros(q.shape[2:])
    dK = np.zeros(k.shape[2:])
    dV = np.zeros(v.shape[2:])
    for r0 in range(0, N, block):
        rows = np.arange(r0, min(N, r0 + block))
        dq, dk, dv = _head_backward_rows(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, kl,
                                         dropout_p, seed, b, h, H, rows)
        dQ[rows] = dq
        dK += dk
        dV += dv
    return dQ, dK, dV


def forward_decode(q, k, v, scale, causal=False, key_lens=None):
    """O [B,H,Nq,d] and lse [B,H,Nq] for Nq new query rows against a cache of Nkv keys per head.

    The decode use of exact attention ("48 FlashAttention", block "Связи": the kernel under vLLM /
    PagedAttention; the operation itself is the one of "FlashAttention 的第一原则", section 2).
    Reading where the page is silent: the cache of sequence b holds L = key_lens[b] valid keys
    (all Nkv when key_lens is None) and query i of Nq is the token at position L - Nq + i, so
    causal keeps key j <= L - Nq + i (self-attention's j <= i in absolute positions) and key
    padding keeps j < L.  A query with no allowed key has O = 0 and lse = -inf.
    """
    B, H, Nq, _ = q.shape
    Nkv = k.shape[2]
    O = np.zeros((B, H, Nq, v.shape[3]))
    lse = np.zeros((B, H, Nq))
    cols = np.arange(Nkv).reshape(1, -1)
    for b in range(B):
        L = Nkv if key_lens is None else int(key_lens[b])
        allowed = np.broadcast_to(cols < L, (Nq, Nkv))
        if causal:
            pos = (L - Nq + np.arange(Nq)).reshape(-1, 1)
            allowed = allowed & (cols <= pos)
        for h in range(H):
            S = (q[b, h] @ k[b, h].T) * scale
            S = np.where(allowed, S, -np.inf)
            P, _, _, lse[b, h] = _softmax_rows(S)
            O[b, h] = P @ v[b, h]
    return O, lse
