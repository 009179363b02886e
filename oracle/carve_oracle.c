/*
 * carve_oracle.c -- plain fp64 CPU oracle for the CARVE recurrent core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes, for ONE (sequence, head) pair, token by token, in fp64:
 *
 *   state S in R^{DV x DK}                 (CARVE technical summary, gist.science,
 *                                           section 1 "Problemstellung": fixed-size
 *                                           matrix state S_t in R^{d_v x d_k})
 *   o_t   = S_{t-1} q_t                    (section 2.1: the recurrent output
 *                                           tensor o_t = S_{t-1} q_t)
 *   alpha = exp(g_t)                       (section 2.3: exponential decay gate on
 *                                           the key axis only)
 *   S'    = S_{t-1} Diag(alpha)
 *   kappa = b_t (.) k_t                    (abstract / section 3 "Chunkability
 *                                           Boundary": erase only on the key axis)
 *   S_t   = S' - (S' k_t) kappa^T + w_t v_t k_t^T
 *                                          (section 2.2: one scalar write gate w
 *                                           per head, broadcast over value channels)
 *
 * i.e. S_t = S_{t-1} Diag(exp g_t) (I - k_t (b_t (.) k_t)^T) + w_t v_t k_t^T.
 *
 * Content-aware erase gate (section 2.1 "Content-Aware Erase via Output Reuse"):
 *   m_c     = (1/L) sum of the outputs o_t of chunk c-1   (one chunk stale)
 *   b_{c,t} = sigmoid(bx_t + U_b m_c),   U_b = U_up U_down  (low rank dv -> r -> dk)
 * Chunks are the consecutive groups of L tokens from the start of the
 * sequence.  Chunk 0 sees m = m0 (zero when m0 is NULL: the summary's stated
 * limitation that sequences shorter than two chunks get no content signal).
 * A short last chunk (T % L != 0) is allowed; its mean still divides by L.
 *
 * Layouts (row-major, contiguous, one pair):
 *   q, k, g, bx : [T][DK]      v, o : [T][DV]      w : [T]
 *   u_down      : [R][DV]      u_up : [DK][R]
 *   S0, S_T     : [DV][DK]     m0, m_T : [DV]
 *
 * carve_oracle_bwd is the exact reverse mode of carve_oracle_fwd, written as
 * a sequential reverse walk over tokens (chunk-start states are kept and each
 * chunk is re-run forward to recover the per-token states).
 *
 * The *_erase entry points take the erase form as an argument: 0 is the
 * form above; 1 is the other erase that acts on the key axis only,
 *   S_t = S' (I - (b_t (.) k_t) k_t^T) + w_t v_t k_t^T,  i.e.  e = S' kappa,
 *   S_t = S' - e k_t^T + w_t v_t k_t^T,
 * where the gated key reads the state and the plain key is written (the
 * abstract and section 3 "Chunkability Boundary" require only that the
 * erase act on the key axis; both forms are chunkable).  For a gate b that
 * is the same on every key channel the two forms coincide.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* p = U_up (U_down m): the low-rank content projection of one chunk. */
static void content_projection(int DK, int DV, int R, const double* u_down,
                               const double* u_up, const double* m,
                               double* h /* [R] */, double* p /* [DK] */) {
  for (int r = 0; r < R; ++r) {
    double acc = 0.0;
    for (int v = 0; v < DV; ++v) acc += u_down[(size_t)r * DV + v] * m[v];
    h[r] = acc;
  }
  for (int j = 0; j < DK; ++j) {
    double acc = 0.0;
    for (int r = 0; r < R; ++r) acc += u_up[(size_t)j * R + r] * h[r];
    p[j] = acc;
  }
}

/*
 * One token of the recurrence.  S is updated in place from S_{t-1} to S_t;
 * o (length DV) receives S_{t-1} q.  'e' is DV doubles of scratch.
 */
static void token_step(int DK, int DV, double* S, const double* q,
                       const double* k, const double* vv, const double* g,
                       const double* b, double w, double* o, double* e,
                       double* alpha, int erase) {
  /* o_t = S_{t-1} q_t */
  for (int v = 0; v < DV; ++v) {
    double acc = 0.0;
    for (int j = 0; j < DK; ++j) acc += S[(size_t)v * DK + j] * q[j];
    o[v] = acc;
  }
  /* S' = S_{t-1} Diag(exp g_t) ; e = S' k_t  (erase 1: e = S' (b (.) k_t)) */
  for (int j = 0; j < DK; ++j) alpha[j] = exp(g[j]);
  for (int v = 0; v < DV; ++v) {
    double acc = 0.0;
    for (int j = 0; j < DK; ++j) {
      S[(size_t)v * DK + j] *= alpha[j];
      acc += S[(size_t)v * DK + j] * (erase ? b[j] * k[j] : k[j]);
    }
    e[v] = acc;
  }
  /* S_t = S' - e (b (.) k)^T + w v k^T   (erase 1: S' - e k^T + w v k^T) */
  for (int v = 0; v < DV; ++v)
    for (int j = 0; j < DK; ++j)
      S[(size_t)v * DK + j] +=
          -e[v] * (erase ? k[j] : b[j] * k[j]) + w * vv[v] * k[j];
}

int carve_oracle_fwd_erase(int T, int DK, int DV, int R, int L, int erase,
                           const double* q, const double* k, const double* v,
                           const double* g, const double* bx, const double* w,
                           const double* u_down, const double* u_up,
                           const double* S0, const double* m0,
                           double* o, double* S_T, double* m_T) {
  if (T < 0 || DK <= 0 || DV <= 0 || R < 0 || L <= 0) return 1;
  double* S = (double*)calloc((size_t)DV * DK, sizeof(double));
  double* m = (double*)calloc((size_t)DV, sizeof(double));
  double* msum = (double*)calloc((size_t)DV, sizeof(double));
  double* h = (double*)calloc((size_t)(R > 0 ? R : 1), sizeof(double));
  double* p = (double*)calloc((size_t)DK, sizeof(double));
  double* b = (double*)calloc((size_t)DK, sizeof(double));
  double* e = (double*)calloc((size_t)DV, sizeof(double));
  double* alpha = (double*)calloc((size_t)DK, sizeof(double));
  if (!S || !m || !msum || !h || !p || !b || !e || !alpha) return 2;
  if (S0) memcpy(S, S0, sizeof(double) * (size_t)DV * DK);
  if (m0) memcpy(m, m0, sizeof(double) * (size_t)DV);

  for (int t0 = 0; t0 < T; t0 += L) {
    int t1 = t0 + L < T ? t0 + L : T;
    /* gate of this chunk: b_{c,t} = sigmoid(bx_t + U_up U_down m_c) */
    content_projection(DK, DV, R, u_down, u_up, m, h, p);
    memset(msum, 0, sizeof(double) * (size_t)DV);
    for (int t = t0; t < t1; ++t) {
      for (int j = 0; j < DK; ++j) b[j] = sigmoid(bx[(size_t)t * DK + j] + p[j]);
      token_step(DK, DV, S, q + (size_t)t * DK, k + (size_t)t * DK,
                 v + (size_t)t * DV, g + (size_t)t * DK, b, w[t],
                 o + (size_t)t * DV, e, alpha, erase);
      for (int vv = 0; vv < DV; ++vv) msum[vv] += o[(size_t)t * DV + vv];
    }
    /* m_{c+1} = (1/L) sum over chunk c of o_t */
    for (int vv = 0; vv < DV; ++vv) m[vv] = msum[vv] / (double)L;
  }
  if (S_T) memcpy(S_T, S, sizeof(double) * (size_t)DV * DK);
  if (m_T) memcpy(m_T, m, sizeof(double) * (size_t)DV);
  free(S); free(m); free(msum); free(h); free(p); free(b); free(e);
  free(alpha);
  return 0;
}

int carve_oracle_fwd(int T, int DK, int DV, int R, int L,
                     const double* q, const double* k, const double* v,
                     const double* g, const double* bx, const double* w,
                     const double* u_down, const double* u_up,
                     const double* S0, const double* m0,
                     double* o, double* S_T, double* m_T) {
  return carve_oracle_fwd_erase(T, DK, DV, R, L, 0, q, k, v, g, bx, w, u_down,
                                u_up, S0, m0, o, S_T, m_T);
}

/*
 * Reverse mode of carve_oracle_fwd.
 *   d_o  : [T][DV]  upstream gradient of o
 *   dS_T : [DV][DK] upstream gradient of S_T (NULL = zero)
 *   dm_T : [DV]     upstream gradient of m_T (NULL = zero)
 * Outputs (all overwritten): dq, dk, dg, dbx [T][DK]; dv [T][DV]; dw [T];
 * du_down [R][DV]; du_up [DK][R]; dS0 [DV][DK]; dm0 [DV].
 */
int carve_oracle_bwd_erase(int T, int DK, int DV, int R, int L, int erase,
                           const double* q, const double* k, const double* v,
                           const double* g, const double* bx, const double* w,
                           const double* u_down, const double* u_up,
                           const double* S0, const double* m0,
                           const double* d_o, const double* dS_T,
                           const double* dm_T, double* dq, double* dk,
                           double* dv, double* dg, double* dbx, double* dw,
                           double* du_down, double* du_up, double* dS0,
                           double* dm0) {
  if (T < 0 || DK <= 0 || DV <= 0 || R < 0 || L <= 0) return 1;
  const size_t SZ = (size_t)DV * DK;
  const int NC = (T + L - 1) / L;
  const int RR = R > 0 ? R : 1;
  /* forward pass keeping the state and the gate input at every chunk start */
  double* Sck = (double*)calloc((size_t)(NC > 0 ? NC : 1) * SZ, sizeof(double));
  double* mck = (double*)calloc((size_t)(NC > 0 ? NC : 1) * DV, sizeof(double));
  double* Stok = (double*)calloc((size_t)L * SZ, sizeof(double)); /* S_{t-1} per token */
  double* S = (double*)calloc(SZ, sizeof(double));
  double* Sp = (double*)calloc(SZ, sizeof(double));
  double* dS = (double*)calloc(SZ, sizeof(double));
  double* m = (double*)calloc((size_t)DV, sizeof(double));
  double* msum = (double*)calloc((size_t)DV, sizeof(double));
  double* dm_next = (double*)calloc((size_t)DV, sizeof(double));
  double* h = (double*)calloc((size_t)RR, sizeof(double));
  double* dh = (double*)calloc((size_t)RR, sizeof(double));
  double* p = (double*)calloc((size_t)DK, sizeof(double));
  double* dp = (double*)calloc((size_t)DK, sizeof(double));
  double* b = (double*)calloc((size_t)DK, sizeof(double));
  double* kap = (double*)calloc((size_t)DK, sizeof(double));
  double* dkap = (double*)calloc((size_t)DK, sizeof(double));
  double* alpha = (double*)calloc((size_t)DK, sizeof(double));
  double* e = (double*)calloc((size_t)DV, sizeof(double));
  double* de = (double*)calloc((size_t)DV, sizeof(double));
  double* otmp = (double*)calloc((size_t)DV, sizeof(double));
  double* dot = (double*)calloc((size_t)DV, sizeof(double));
  if (!Sck || !mck || !Stok || !S || !Sp || !dS || !m || !msum || !dm_next ||
      !h || !dh || !p || !dp || !b || !kap || !dkap || !alpha || !e || !de ||
      !otmp || !dot)
    return 2;

  if (S0) memcpy(S, S0, sizeof(double) * SZ);
  if (m0) memcpy(m, m0, sizeof(double) * (size_t)DV);
  for (int c = 0; c < NC; ++c) {
    int t0 = c * L, t1 = t0 + L < T ? t0 + L : T;
    memcpy(Sck + (size_t)c * SZ, S, sizeof(double) * SZ);
    memcpy(mck + (size_t)c * DV, m, sizeof(double) * (size_t)DV);
    content_projection(DK, DV, R, u_down, u_up, m, h, p);
    memset(msum, 0, sizeof(double) * (size_t)DV);
    for (int t = t0; t < t1; ++t) {
      for (int j = 0; j < DK; ++j) b[j] = sigmoid(bx[(size_t)t * DK + j] + p[j]);
      token_step(DK, DV, S, q + (size_t)t * DK, k + (size_t)t * DK,
                 v + (size_t)t * DV, g + (size_t)t * DK, b, w[t], otmp, e,
                 alpha, erase);
      for (int vv = 0; vv < DV; ++vv) msum[vv] += otmp[vv];
    }
    for (int vv = 0; vv < DV; ++vv) m[vv] = msum[vv] / (double)L;
  }

  /* reverse walk */
  if (dS_T) memcpy(dS, dS_T, sizeof(double) * SZ);
  if (dm_T) memcpy(dm_next, dm_T, sizeof(double) * (size_t)DV);
  memset(du_down, 0, sizeof(double) * (size_t)R * DV);
  memset(du_up, 0, sizeof(double) * (size_t)DK * R);
  for (int c = NC - 1; c >= 0; --c) {
    int t0 = c * L, t1 = t0 + L < T ? t0 + L : T;
    const double* mc = mck + (size_t)c * DV;
    content_projection(DK, DV, R, u_down, u_up, mc, h, p);
    /* re-run the chunk forward from its start state, keeping S_{t-1} */
    memcpy(S, Sck + (size_t)c * SZ, sizeof(double) * SZ);
    for (int t = t0; t < t1; ++t) {
      memcpy(Stok + (size_t)(t - t0) * SZ, S, sizeof(double) * SZ);
      for (int j = 0; j < DK; ++j) b[j] = sigmoid(bx[(size_t)t * DK + j] + p[j]);
      token_step(DK, DV, S, q + (size_t)t * DK, k + (size_t)t * DK,
                 v + (size_t)t * DV, g + (size_t)t * DK, b, w[t], otmp, e,
                 alpha, erase);
    }
    memset(dp, 0, sizeof(double) * (size_t)DK);
    for (int t = t1 - 1; t >= t0; --t) {
      const double* St = Stok + (size_t)(t - t0) * SZ; /* S_{t-1} */
      const double* qt = q + (size_t)t * DK;
      const double* kt = k + (size_t)t * DK;
      const double* vt = v + (size_t)t * DV;
      const double* gt = g + (size_t)t * DK;
      const double wt = w[t];
      /* upstream gradient of o_t: direct, plus the share of the next chunk's
         gate input m_{c+1} = (1/L) sum o_t */
      for (int vv = 0; vv < DV; ++vv)
        dot[vv] = d_o[(size_t)t * DV + vv] + dm_next[vv] / (double)L;
      for (int j = 0; j < DK; ++j) {
        b[j] = sigmoid(bx[(size_t)t * DK + j] + p[j]);
        kap[j] = b[j] * kt[j];
        alpha[j] = exp(gt[j]);
      }
      /* recompute S' and e (e = S' k, or S' kappa for erase 1) */
      for (int vv = 0; vv < DV; ++vv) {
        double acc = 0.0;
        for (int j = 0; j < DK; ++j) {
          Sp[(size_t)vv * DK + j] = St[(size_t)vv * DK + j] * alpha[j];
          acc += Sp[(size_t)vv * DK + j] * (erase ? kap[j] : kt[j]);
        }
        e[vv] = acc;
      }
      /* write term  w v k^T */
      double dwt = 0.0;
      for (int vv = 0; vv < DV; ++vv) {
        double dSk = 0.0;
        for (int j = 0; j < DK; ++j) dSk += dS[(size_t)vv * DK + j] * kt[j];
        dwt += vt[vv] * dSk;
        dv[(size_t)t * DV + vv] = wt * dSk;
      }
      dw[t] = dwt;
      for (int j = 0; j < DK; ++j) {
        double acc = 0.0;
        for (int vv = 0; vv < DV; ++vv) acc += dS[(size_t)vv * DK + j] * vt[vv];
        dk[(size_t)t * DK + j] = wt * acc;
      }
      /* erase term  -e x^T with x = kappa (erase 0) or k (erase 1) */
      for (int vv = 0; vv < DV; ++vv) {
        double acc = 0.0;
        for (int j = 0; j < DK; ++j)
          acc += dS[(size_t)vv * DK + j] * (erase ? kt[j] : kap[j]);
        de[vv] = -acc;
      }
      for (int j = 0; j < DK; ++j) {
        double acc = 0.0;
        for (int vv = 0; vv < DV; ++vv) acc += dS[(size_t)vv * DK + j] * e[vv];
        if (erase)
          dk[(size_t)t * DK + j] -= acc;  /* d/dx of -e x^T, x = k */
        else
          dkap[j] = -acc;                 /* x = kappa */
      }
      /* e = S' y, y = k (erase 0) or kappa (erase 1):  dS' = dS + de y^T,
         dy = S'^T de  (dS now holds dS') */
      for (int vv = 0; vv < DV; ++vv)
        for (int j = 0; j < DK; ++j)
          dS[(size_t)vv * DK + j] += de[vv] * (erase ? kap[j] : kt[j]);
      for (int j = 0; j < DK; ++j) {
        double acc = 0.0;
        for (int vv = 0; vv < DV; ++vv) acc += Sp[(size_t)vv * DK + j] * de[vv];
        if (erase)
          dkap[j] = acc;
        else
          dk[(size_t)t * DK + j] += acc;
      }
      /* kappa = b (.) k ; b = sigmoid(bx + p) */
      for (int j = 0; j < DK; ++j) {
        dk[(size_t)t * DK + j] += b[j] * dkap[j];
        double db = kt[j] * dkap[j];
        double dz = db * b[j] * (1.0 - b[j]);
        dbx[(size_t)t * DK + j] = dz;
        dp[j] += dz;
      }
      /* S' = S_{t-1} Diag(alpha) ; alpha = exp(g) */
      for (int j = 0; j < DK; ++j) {
        double acc = 0.0;
        for (int vv = 0; vv < DV; ++vv)
          acc += St[(size_t)vv * DK + j] * dS[(size_t)vv * DK + j];
        dg[(size_t)t * DK + j] = alpha[j] * acc;
      }
      /* o_t = S_{t-1} q_t */
      for (int j = 0; j < DK; ++j) {
        double acc = 0.0;
        for (int vv = 0; vv < DV; ++vv) acc += St[(size_t)vv * DK + j] * dot[vv];
        dq[(size_t)t * DK + j] = acc;
      }
      /* gradient of S_{t-1} */
      for (int vv = 0; vv < DV; ++vv)
        for (int j = 0; j < DK; ++j)
          dS[(size_t)vv * DK + j] = dS[(size_t)vv * DK + j] * alpha[j] + dot[vv] * qt[j];
    }
    /* gate of chunk c:  p = U_up h,  h = U_down m_c */
    for (int r = 0; r < R; ++r) {
      double acc = 0.0;
      for (int j = 0; j < DK; ++j) {
        du_up[(size_t)j * R + r] += dp[j] * h[r];
        acc += u_up[(size_t)j * R + r] * dp[j];
      }
      dh[r] = acc;
    }
    for (int vv = 0; vv < DV; ++vv) {
      double acc = 0.0;
      for (int r = 0; r < R; ++r) {
        du_down[(size_t)r * DV + vv] += dh[r] * mc[vv];
        acc += u_down[(size_t)r * DV + vv] * dh[r];
      }
      dm_next[vv] = acc; /* gradient of m_c, spread over chunk c-1 next */
    }
  }
  memcpy(dS0, dS, sizeof(double) * SZ);
  memcpy(dm0, dm_next, sizeof(double) * (size_t)DV);

  free(Sck); free(mck); free(Stok); free(S); free(Sp); free(dS); free(m);
  free(msum); free(dm_next); free(h); free(dh); free(p); free(dp); free(b);
  free(kap); free(dkap); free(alpha); free(e); free(de); free(otmp); free(dot);
  return 0;
}

int carve_oracle_bwd(int T, int DK, int DV, int R, int L,
                     const double* q, const double* k, const double* v,
                     const double* g, const double* bx, const double* w,
                     const double* u_down, const double* u_up,
                     const double* S0, const double* m0,
                     const double* d_o, const double* dS_T, const double* dm_T,
                     double* dq, double* dk, double* dv, double* dg,
                     double* dbx, double* dw, double* du_down, double* du_up,
                     double* dS0, double* dm0) {
  return carve_oracle_bwd_erase(T, DK, DV, R, L, 0, q, k, v, g, bx, w, u_down,
                                u_up, S0, m0, d_o, dS_T, dm_T, dq, dk, dv, dg,
                                dbx, dw, du_down, du_up, dS0, dm0);
}
