"""Independent numpy (fp64) forms of causal linear attention that pin the oracle.

None of these is the oracle's token loop.  Each is a different closed or parallel form
that the pages state to be equal to it, so agreement with the oracle is evidence that
the oracle's loop is right:

* ``masked_quadratic`` -- the ratio-of-sums form with a causal mask, evaluated as dense
  matrices ("Linear Attention and Retentive Networks ...", "The Associative Property and
  Linear Kernel Formulation").
* ``retention_parallel`` -- the parallel retention form with the decay matrix
  D[n, m] = gamma^(n - m) for n >= m (same page, "1. Multi-Scale Decay Formulation" and
  "A. Parallel Representation").
* ``final_state_closed`` -- the final state as one weighted matrix product (the sum
  definitions in "Log-Depth Chunked Linear-Attention Scan", "Mathematical statement",
  with the decay weights of the recurrent retention form).
* ``chunked_scan`` -- chunk summaries, an exclusive Hillis-Steele scan over them with a
  round counter, and the per-chunk combine ("Log-Depth Chunked Linear-Attention Scan",
  "Formulas", "Mathematical statement" and "Implementation notes"; the decay placement
  of "C. Chunkwise Recurrent Representation" on the retention page).

They are slow, dense and meant for tiny inputs only.
"""

from __future__ import annotations

import numpy as np


def psi(x: np.ndarray, feature_map: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    if feature_map == "identity":
        return x.copy()
    # ELU with alpha = 1, plus one: x + 1 above zero, e^x at or below zero.
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def _decay_matrix(T: int, g: float) -> np.ndarray:
    n = np.arange(T)[:, None]
    m = np.arange(T)[None, :]
    D = np.zeros((T, T))
    mask = n >= m
    D[mask] = np.power(g, (n - m)[mask].astype(np.float64))
    return D


def masked_quadratic(q, k, v, feature_map="elu1", normalize=True, eps=0.0):
    """o = ((psiQ psiK^T) * M) V, divided by ((psiQ psiK^T) * M) 1 when normalised."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, H, T, _ = q.shape
    out = np.zeros(v.shape)
    M = np.tril(np.ones((T, T)))
    for b in range(B):
        for h in range(H):
            A = (psi(q[b, h], feature_map) @ psi(k[b, h], feature_map).T) * M
            num = A @ v[b, h]
            if normalize:
                out[b, h] = num / (A.sum(axis=1, keepdims=True) + eps)
            else:
                out[b, h] = num
    return out


def retention_parallel(q, k, v, gammas, feature_map="identity", normalize=False, eps=0.0):
    """o = ((psiQ psiK^T) * D) V with the per-head decay matrix D."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, H, T, _ = q.shape
    out = np.zeros(v.shape)
    for h in range(H):
        D = _decay_matrix(T, float(gammas[h]))
        for b in range(B):
            A = (psi(q[b, h], feature_map) @ psi(k[b, h], feature_map).T) * D
            num = A @ v[b, h]
            out[b, h] = num / (A.sum(axis=1, keepdims=True) + eps) if normalize else num
    return out


def final_state_closed(k, v, gammas=None, feature_map="elu1"):
    """S_T = psiK^T diag(w) V and Z_T = psiK^T w with w_i = gamma^(T - 1 - i)."""
    k, v = (np.asarray(a, dtype=np.float64) for a in (k, v))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv))
    Z = np.zeros((B, H, dk))
    for h in range(H):
        g = 1.0 if gammas is None else float(gammas[h])
        w = np.power(g, (T - 1 - np.arange(T)).astype(np.float64))
        for b in range(B):
            fk = psi(k[b, h], feature_map) * w[:, None]
            S[b, h] = fk.T @ v[b, h]
            Z[b, h] = fk.sum(axis=0)
    return S, Z


def chunked_scan(q, k, v, C, gammas=None, feature_map="elu1", normalize=True, eps=0.0):
    """Chunk summaries, exclusive Hillis-Steele scan, per-chunk combine.

    Chunk c holds tokens [cC, cC + L_c), L_c = C except for a shorter last chunk; the
    positions a padded chunk would hold past T contribute nothing and do not advance the
    decay.  Within a chunk, position j (0-based) gets the summary weight
    Xi_j = gamma^(L_c - 1 - j) and the prefix weight Theta_j = gamma^(j + 1).  The scan
    element is (a, S, Z) with a = gamma^(L_c) and
    (a1, S1, Z1) + (a2, S2, Z2) = (a1 a2, a2 S1 + S2, a2 Z1 + Z2);
    without decay this is the plain sum of the scan page's monoid.

    Returns (out, S_final, Z_final, rounds) where rounds counts the Hillis-Steele rounds
    actually executed (the maximum over heads).
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    NC = -(-T // C)
    out = np.zeros((B, H, T, dv))
    S_fin = np.zeros((B, H, dk, dv))
    Z_fin = np.zeros((B, H, dk))
    max_rounds = 0
    for b in range(B):
        for h in range(H):
            g = 1.0 if gammas is None else float(gammas[h])
            fq = psi(q[b, h], feature_map)
            fk = psi(k[b, h], feature_map)
            V = v[b, h]
            if NC == 0:
                continue
            # Per-chunk local summaries.
            a = np.zeros(NC)
            X = np.zeros((NC, dk, dv))
            Y = np.zeros((NC, dk))
            for c in range(NC):
                s = c * C
                L = min(C, T - s)
                xi = np.power(g, (L - 1 - np.arange(L)).astype(np.float64))
                kw = fk[s:s + L] * xi[:, None]
                X[c] = kw.T @ V[s:s + L]
                Y[c] = kw.sum(axis=0)
                a[c] = g ** L
            # Inclusive Hillis-Steele scan: in round r every element i >= 2^r absorbs
            # element i - 2^r from the previous round.
            rounds = 0
            d = 1
            while d < NC:
                a_n, X_n, Y_n = a.copy(), X.copy(), Y.copy()
                for i in range(d, NC):
                    a_n[i] = a[i - d] * a[i]
                    X_n[i] = a[i] * X[i - d] + X[i]
                    Y_n[i] = a[i] * Y[i - d] + Y[i]
                a, X, Y = a_n, X_n, Y_n
                rounds += 1
                d *= 2
            max_rounds = max(max_rounds, rounds)
            S_fin[b, h] = X[NC - 1]
            Z_fin[b, h] = Y[NC - 1]
            # Exclusive prefixes.
            P = np.zeros((NC, dk, dv))
            ZP = np.zeros((NC, dk))
            P[1:] = X[:-1]
            ZP[1:] = Y[:-1]
            # Per-chunk combine.
            for c in range(NC):
                s = c * C
                L = min(C, T - s)
                theta = np.power(g, (np.arange(L) + 1).astype(np.float64))
                A = (fq[s:s + L] @ fk[s:s + L].T) * _decay_matrix(L, g)
                num = theta[:, None] * (fq[s:s + L] @ P[c]) + A @ V[s:s + L]
                if normalize:
                    den = theta * (fq[s:s + L] @ ZP[c]) + A.sum(axis=1)
                    out[b, h, s:s + L] = num / (den[:, None] + eps)
                else:
                    out[b, h, s:s + L] = num
    return out, S_fin, Z_fin, max_rounds
