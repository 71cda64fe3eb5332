"""Float64 chunked form of the gated delta rule, restated from the Muir review.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).  It follows the chunked
kernel the Muir review describes in §2.4 ("Boundary-Pivoted Chunkwise
Kernel"), step by step, in numpy float64, for one head at a time:

1. cumulative log-decay Lambda_t inside each chunk;
2. the decay-relative key/query products, built without any division:
   leaves of at most ``leaf`` tokens use exp(Lambda_t - Lambda_s) (t >= s, a
   non-positive exponent) directly; two adjacent blocks are merged by taking
   the pivot p at the end of the left block and splitting
   Lambda_t - Lambda_s = (Lambda_t - Lambda_p) + (Lambda_p - Lambda_s), both
   parts non-positive, so each scaled operand is a plain matrix product;
3. the inverse of the unit lower-triangular chunk matrix T = I + L_strict by
   divide and conquer: Neumann-series leaves, then block merges
   [[A, 0], [C, D]]^-1 = [[A^-1, 0], [-D^-1 C A^-1, D^-1]];
4. the chunk solve and the inter-chunk state scan.

The unknowns are named after the algebra below (unrolling the token
recurrence inside a chunk from its start state S_0, row-vector convention):

  r_t = k_t Diag(alpha_t) S_{t-1}
  (I + L) R = K_gamma S_0 + M V_hat            => R = W S_0 + U
  O     = (Q_til * gamma) S_0 + Aq V_hat - Bq R
  S_C   = Diag(gamma_C) S_0 + (K*pi_C)^T V_hat - (K_hat*pi_C)^T R

with M_ts = k_t E(t,s) k_s^T, L_ts = k_t E(t,s) k_hat_s^T (t > s),
Aq_ts = q_til_t E(t,s) k_s^T, Bq_ts = q_til_t E(t,s) k_hat_s^T (t >= s),
E(t,s) = Diag(exp(Lambda_t - Lambda_s)), gamma_t = exp(Lambda_t),
pi_C,s = exp(Lambda_C - Lambda_s).  The page writes the solve with the
right-hand side [V_hat, K_hat pi]; the unknowns differ by name only.
"""
from __future__ import annotations

import numpy as np


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def pivot_products(A: np.ndarray, Bm: np.ndarray, lam: np.ndarray, strict: bool,
                   leaf: int = 8) -> np.ndarray:
    """P_ts = sum_i A_ti exp(lam_ti - lam_si) B_si for t > s (strict) or t >= s.

    A: [n, d], Bm: [n, d], lam: [n, d] cumulative log-decay.  Upper part is 0.
    """
    n = A.shape[0]
    P = np.zeros((n, n))

    def rec(lo: int, hi: int) -> None:
        if hi - lo <= leaf:
            for t in range(lo, hi):
                for s in range(lo, t + (0 if strict else 1)):
                    P[t, s] = np.sum(A[t] * np.exp(lam[t] - lam[s]) * Bm[s])
            return
        mid = lo + (hi - lo + 1) // 2
        rec(lo, mid)
        rec(mid, hi)
        p = mid - 1                                            # end of the left block
        right = A[mid:hi] * np.exp(lam[mid:hi] - lam[p])       # exponents <= 0
        left = Bm[lo:mid] * np.exp(lam[p] - lam[lo:mid])       # exponents <= 0
        P[mid:hi, lo:mid] = right @ left.T

    if n:
        rec(0, n)
    return P


def unit_lower_inverse(Tm: np.ndarray, leaf: int = 8) -> np.ndarray:
    """Inverse of a unit lower-triangular matrix by divide and conquer."""
    n = Tm.shape[0]

    def rec(lo: int, hi: int) -> np.ndarray:
        m = hi - lo
        if m <= leaf:
            N = Tm[lo:hi, lo:hi] - np.eye(m)        # strictly lower, N^m = 0
            X = np.eye(m)
            P = np.eye(m)
            for _ in range(1, m):
                P = P @ (-N)
                X = X + P
            return X
        mid = lo + (m + 1) // 2
        Ai = rec(lo, mid)
        Di = rec(mid, hi)
        out = np.zeros((m, m))
        out[: mid - lo, : mid - lo] = Ai
        out[mid - lo:, mid - lo:] = Di
        out[mid - lo:, : mid - lo] = -Di @ Tm[mid:hi, lo:mid] @ Ai
        return out

    return rec(0, n) if n else np.zeros((0, 0))


def chunked_head(q, k, v, b, w, z, g, log_alpha, gamma_stat, S0, chunk: int,
                 eps: float = 1e-6, leaf: int = 8):
    """One head, arrays [T, d] (float64).  Returns y, o_raw [T, dv], S_T."""
    q, k, v, b, w, z, g, la = (np.asarray(x, dtype=np.float64)
                               for x in (q, k, v, b, w, z, g, log_alpha))
    T, dk = q.shape
    dv = v.shape[1]
    gs = np.ones(dk) if gamma_stat is None else np.asarray(gamma_stat, dtype=np.float64)
    qt = q * gs * 2.0 * _sigmoid(z)
    kh = b * k
    vh = w * v
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    O = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        n = sl.stop - sl.start
        lam = np.cumsum(la[sl], axis=0)
        kc, khc, qc, vhc = k[sl], kh[sl], qt[sl], vh[sl]
        M = pivot_products(kc, kc, lam, True, leaf)
        L = pivot_products(kc, khc, lam, True, leaf)
        Aq = pivot_products(qc, kc, lam, False, leaf)
        Bq = pivot_products(qc, khc, lam, False, leaf)
        Ti = unit_lower_inverse(np.eye(n) + L, leaf)
        gam = np.exp(lam)                       # <= 1
        W = Ti @ (kc * gam)
        U = Ti @ (M @ vhc)
        R = W @ S + U
        O[sl] = (qc * gam) @ S + Aq @ vhc - Bq @ R
        pi_c = np.exp(lam[-1] - lam)            # <= 1
        S = gam[-1][:, None] * S + (kc * pi_c).T @ vhc - (khc * pi_c).T @ R
    y = g * O / np.sqrt(np.mean(O * O, axis=1, keepdims=True) + eps)
    return y, O, S
