"""Oracle of the single-token recurrent decode step, fp64 numpy.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module; the product path never does.

Inference advances the CARVE recurrence one token at a time.  The state of
one (sequence, head) pair between tokens is

  S     [DV, DK]  the matrix state S_{t-1}      (CARVE technical summary,
                                                  gist.science, section 1)
  m     [DV]      the content signal m_c of the current chunk: the mean of
                  the previous chunk's outputs  (section 2.1, "Content-Aware
                  Erase via Output Reuse": one chunk stale)
  osum  [DV]      the sum of the current chunk's outputs so far
  pos             tokens already processed (the new token's index)

One step with the new token's q, k, v, g, b_x, w:

  p   = U_up (U_down m)                          low-rank U_b (section 2.1)
  b   = sigmoid(b_x + p)                         erase gate on the key axis
  o   = S q                                      o_t = S_{t-1} q_t
  S'  = S Diag(exp g)                            key-axis decay (section 2.3)
  S   = S' - (S' k)(b * k)^T + w v k^T           erase only on the key axis;
                                                 scalar write gate (2.2)
  osum += o;  at a chunk's last token ((pos + 1) % L == 0):
  m = osum / L, osum = 0                         the next chunk's signal

This is the per-token loop of ``carve_oracle.c`` restated for one token with
the chunk bookkeeping carried explicitly; ``tests/test_decode_oracle.py``
pins it to that file's forward over whole sequences.
"""
import numpy as np


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def decode_step(S, m, osum, pos, q, k, v, g, bx, w, u_down, u_up, L,
                erase=0):
    """One token for one (sequence, head) pair, in fp64.  erase = 1: the
    other key-axis erase, e = S' (b * k) and S = S' - e k^T + w v k^T.

    S [DV, DK], m [DV], osum [DV]; q, k, g, bx [DK]; v [DV]; w scalar;
    u_down [R, DV]; u_up [DK, R].  Returns (o [DV], S, m, osum) after the
    token (new arrays; the inputs are not modified)."""
    S = np.asarray(S, np.float64)
    p = u_up @ (u_down @ m) if u_down.shape[0] > 0 else np.zeros(k.shape)
    b = sigmoid(bx + p)
    o = S @ q
    S1 = S * np.exp(g)[None, :]
    if erase:
        e = S1 @ (b * k)
        S_new = S1 - np.outer(e, k) + w * np.outer(v, k)
    else:
        e = S1 @ k
        S_new = S1 - np.outer(e, b * k) + w * np.outer(v, k)
    osum_new = osum + o
    m_new = np.array(m, np.float64)
    if (pos + 1) % L == 0:
        m_new = osum_new / L
        osum_new = np.zeros_like(osum_new)
    return o, S_new, m_new, osum_new


def decode_steps(S, m, osum, pos0, q, k, v, g, bx, w, u_down, u_up, L,
                 erase=0):
    """T consecutive steps for one pair: q, k, g, bx [T, DK], v [T, DV],
    w [T].  Returns (o [T, DV], S, m, osum)."""
    T = q.shape[0]
    out = np.zeros((T, v.shape[1]))
    for t in range(T):
        out[t], S, m, osum = decode_step(S, m, osum, pos0 + t, q[t], k[t],
                                         v[t], g[t], bx[t], w[t], u_down,
                                         u_up, L, erase)
    return out, S, m, osum
