"""fp64 chunkwise re-derivation of the Gated DeltaNet layer (forward + backward).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  This is an
independent restatement, in numpy, of the chunkwise-parallel algebra that the
CUDA kernels implement.  It exists to pin that algebra against the
token-by-token recurrence in ``gdn_ref.c`` for any chunk size (the pages name
the chunk-parallel form -- jax-linear-attention 0.1.0, "How it works": a
chunk-parallel op beside the token-by-token reference -- but never print its
equations; the form below is derived from the recurrence).

Per chunk of n <= C tokens, with the state H = S^T (K x V) entering it and the
query pre-multiplied by ``scale``:

  G     = cumsum(g) inside the chunk ;  gam_i = exp(G_i)
  Gam   = exp(G_i - G_j) for i >= j, else 0
  L     = strict_lower( diag(beta) K K^T * Gam )
  A     = (I + L)^-1                      (unit lower triangular)
  W     = A diag(beta * gam) K ;  Ut = A diag(beta) V
  U     = Ut - W H                        (delta-corrected values)
  O     = diag(gam) Q H + lower(Q K^T * Gam) U
  H'    = gam_n H + (diag(e) K)^T U,   e_j = exp(G_n - G_j)

The backward is the reverse-mode of exactly these steps, chunk by chunk in
reverse order.  A triangular solve stands in for the inverse (a library
primitive; the kernels use blocked forward substitution).
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _chunk_terms(q, k, v, g, beta, scale):
    n = k.shape[0]
    Q = scale * q
    G = np.cumsum(g)
    gam = np.exp(G)
    low = np.tril(np.ones((n, n), dtype=bool))
    Gam = np.exp(np.where(low, G[:, None] - G[None, :], -np.inf))
    Lm = np.tril(beta[:, None] * (k @ k.T) * Gam, -1)
    A = solve_triangular(np.eye(n) + Lm, np.eye(n), lower=True, unit_diagonal=True)
    W = A @ ((beta * gam)[:, None] * k)
    Ut = A @ (beta[:, None] * v)
    P = np.tril((Q @ k.T) * Gam)
    e = np.exp(G[-1] - G)
    return dict(Q=Q, G=G, gam=gam, Gam=Gam, L=Lm, A=A, W=W, Ut=Ut, P=P, e=e)


def fwd_unit(q, k, v, g, beta, h0=None, scale=1.0, C=64):
    """One (document, head) unit: q,k (L,K); v (L,V); g, beta (L,).  Returns o (L,V), hT (K,V)."""
    L, K = k.shape
    V = v.shape[1]
    H = np.zeros((K, V)) if h0 is None else np.array(h0, dtype=np.float64)
    o = np.zeros((L, V))
    for t0 in range(0, L, C):
        sl = slice(t0, min(t0 + C, L))
        c = _chunk_terms(q[sl], k[sl], v[sl], g[sl], beta[sl], scale)
        U = c["Ut"] - c["W"] @ H
        o[sl] = c["gam"][:, None] * (c["Q"] @ H) + c["P"] @ U
        H = c["gam"][-1] * H + (c["e"][:, None] * k[sl]).T @ U
    return o, H


def bwd_unit(q, k, v, g, beta, do, h0=None, dhT=None, scale=1.0, C=64):
    """Reverse-mode of ``fwd_unit`` for upstream do (L,V) and dhT (K,V).
    Returns dq, dk, dv (L,.), dg, dbeta (L,), dh0 (K,V)."""
    L, K = k.shape
    V = v.shape[1]
    starts = list(range(0, L, C))
    Hs = []
    H = np.zeros((K, V)) if h0 is None else np.array(h0, dtype=np.float64)
    for t0 in starts:  # states entering each chunk (recomputed, not stored by the forward)
        sl = slice(t0, min(t0 + C, L))
        Hs.append(H)
        c = _chunk_terms(q[sl], k[sl], v[sl], g[sl], beta[sl], scale)
        H = c["gam"][-1] * H + (c["e"][:, None] * k[sl]).T @ (c["Ut"] - c["W"] @ H)
    dq = np.zeros((L, K)); dk = np.zeros((L, K)); dv = np.zeros((L, V))
    dg = np.zeros(L); dbeta = np.zeros(L)
    dH = np.zeros((K, V)) if dhT is None else np.array(dhT, dtype=np.float64)
    for idx in reversed(range(len(starts))):
        t0 = starts[idx]
        sl = slice(t0, min(t0 + C, L))
        H = Hs[idx]
        kc, vc, bc, dO = k[sl], v[sl], beta[sl], do[sl]
        c = _chunk_terms(q[sl], kc, vc, g[sl], bc, scale)
        Q, gam, Gam, A, W, P, e = (c[x] for x in ("Q", "gam", "Gam", "A", "W", "P", "e"))
        U = c["Ut"] - W @ H
        Kd = e[:, None] * kc
        n = kc.shape[0]
        dG = np.zeros(n)
        # H' = gam_n H + Kd^T U
        dU = Kd @ dH + P.T @ dO
        dKd = U @ dH.T
        dHc = gam[-1] * dH
        dkc = e[:, None] * dKd
        de = np.sum(kc * dKd, axis=1)
        dG[-1] += gam[-1] * np.sum(H * dH) + np.sum(e * de)
        dG -= e * de
        # O = diag(gam) Q H + P U
        dOH = dO @ H.T
        dQ = gam[:, None] * dOH
        dHc += (gam[:, None] * Q).T @ dO
        dG += gam * np.sum(Q * dOH, axis=1)
        dP = np.tril(dO @ U.T)
        dS = dP * Gam
        dQ += dS @ kc
        dkc += dS.T @ Q
        dPP = dP * P
        dG += dPP.sum(1) - dPP.sum(0)
        # U = Ut - W H
        dW = -dU @ H.T
        dHc -= W.T @ dU
        # Ut = A diag(beta) V
        dA = dU @ (bc[:, None] * vc).T
        AtdU = A.T @ dU
        dvc = bc[:, None] * AtdU
        dbc = np.sum(vc * AtdU, axis=1)
        # W = A diag(beta gam) K
        bg = bc * gam
        dA += dW @ (bg[:, None] * kc).T
        Z = A.T @ dW
        dkc += bg[:, None] * Z
        kZ = np.sum(kc * Z, axis=1)
        dbc += gam * kZ
        dG += bg * kZ
        # A = (I + L)^-1 ; L = strict_lower(diag(beta) K K^T * Gam)
        dL = np.tril(-A.T @ dA @ A.T, -1)
        dLG = dL * Gam
        dbc += np.sum(dLG * (kc @ kc.T), axis=1)
        dkc += bc[:, None] * (dLG @ kc) + (bc[:, None] * dLG).T @ kc
        dLL = dL * c["L"]
        dG += dLL.sum(1) - dLL.sum(0)
        dq[sl] = scale * dQ
        dk[sl] = dkc
        dv[sl] = dvc
        dbeta[sl] = dbc
        dg[sl] = np.cumsum(dG[::-1])[::-1]
        dH = dHc
    return dq, dk, dv, dg, dbeta, dH

