"""The WY-form chunk solve, written with dense fp64 linear algebra.

Test infrastructure only; see ``oracle/__init__.py``.  Used to pin the
sequential oracle: the CARVE summaries (gist.science, section 3,
"Chunkability Boundary", Theorem 11) state that with erase on the key axis
only, one triangular solve per chunk -- shared by every value row --
reproduces the token recurrence exactly.  This module is that chunk form,
derived by unrolling the recurrence over the tokens t = 1..n of a block:

  Gamma_t   = exp(g_1 + ... + g_t)        (inclusive cumulative decay, per key channel)
  Gamma^-_t = Gamma_{t-1}, Gamma^-_1 = 1   (exclusive)
  gamma     = Gamma_n
  K~ = K (.) Gamma       K^ = K / Gamma       Q~ = Q (.) Gamma^-
  kap^ = (b (.) K) / Gamma
  A    = strict_lower(K~ kap^T)   M   = strict_lower(K~ K^T)
  P_k  = strict_lower(Q~ K^T)     P_kap = strict_lower(Q~ kap^T)
  W    = w (.) V
  E    = (I + A)^{-1} (K~ S^T + M W)               (the WY pseudo-values)
  O    = Q~ S^T + P_k W - P_kap E                  (o_t = S_{t-1} q_t)
  S   <- S Diag(gamma) + W^T K_end - E^T kap_end,  K_end = K^ (.) gamma,
                                                   kap_end = kap^ (.) gamma

The gate b is fixed across a chunk of L tokens (it depends on m_c only), so a
chunk may be solved as several consecutive blocks of ``block`` tokens; the
chunk mean m_{c+1} still averages the L outputs of the whole chunk.

For the other key-axis erase (erase = 1: S_t = S'(I - (b (.) k) k^T) +
w v k^T, the gated key reads the state, the plain key is written) unrolling
gives e_t = S'_t kap_t - w_t v_t and S_t = S'_t - e_t k_t^T, hence one
triangular solve per chunk with the roles of the keys exchanged:

  kap~ = b (.) K (.) Gamma
  A    = strict_lower(kap~ K^T)
  E    = (I + A)^{-1} (kap~ S^T - W)
  O    = Q~ S^T - P_k E
  S   <- (S - E^T K^) Diag(gamma)
"""
import numpy as np


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def chunked_fwd_pair(q, k, v, g, bx, w, u_down, u_up, L, S0=None, m0=None,
                     block=None, erase=0):
    """Same contract as ``ref.fwd_pair``; returns (o, S_T, m_T)."""
    q, k, v, g, bx, w = (np.asarray(a, dtype=np.float64)
                         for a in (q, k, v, g, bx, w))
    T, DK = q.shape
    DV = v.shape[1]
    S = np.zeros((DV, DK)) if S0 is None else np.array(S0, dtype=np.float64)
    m = np.zeros(DV) if m0 is None else np.array(m0, dtype=np.float64)
    o = np.zeros((T, DV))
    block = L if block is None else block
    for t0 in range(0, T, L):
        t1 = min(t0 + L, T)
        p = u_up @ (u_down @ m)                      # U_b m_c, rank r
        for s0 in range(t0, t1, block):
            s1 = min(s0 + block, t1)
            n = s1 - s0
            G = np.cumsum(g[s0:s1], axis=0)         # log Gamma (inclusive)
            Gam = np.exp(G)
            Gam_ex = np.exp(np.vstack([np.zeros((1, DK)), G[:-1]]))
            gam = Gam[-1]
            K, Q = k[s0:s1], q[s0:s1]
            b = _sigmoid(bx[s0:s1] + p[None, :])
            Kt, Kh, Qt = K * Gam, K / Gam, Q * Gam_ex
            W = w[s0:s1, None] * v[s0:s1]
            if erase:
                kap_t = b * K * Gam
                A = np.tril(kap_t @ Kh.T, -1)
                Pk = np.tril(Qt @ Kh.T, -1)
                E = np.linalg.solve(np.eye(n) + A, kap_t @ S.T - W)
                o[s0:s1] = Qt @ S.T - Pk @ E
                S = (S - E.T @ Kh) * gam[None, :]
                continue
            kap_h = b * K / Gam
            A = np.tril(Kt @ kap_h.T, -1)
            M = np.tril(Kt @ Kh.T, -1)
            Pk = np.tril(Qt @ Kh.T, -1)
            Pkap = np.tril(Qt @ kap_h.T, -1)
            E = np.linalg.solve(np.eye(n) + A, Kt @ S.T + M @ W)
            o[s0:s1] = Qt @ S.T + Pk @ W - Pkap @ E
            K_end, kap_end = Kh * gam[None, :], kap_h * gam[None, :]
            S = S * gam[None, :] + W.T @ K_end - E.T @ kap_end
        m = o[t0:t1].sum(axis=0) / L
    return o, S, m
