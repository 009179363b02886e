// carve_generic.cu -- the generic CARVE chunk kernels (fp32 CUDA-core math).
//
// One CTA walks the chunks of one (sequence, head) pair in order.  Each
// chunk of L tokens is solved as L / C consecutive blocks of C = min(L, 64)
// tokens with the WY form of the key-axis-gated delta rule (the CARVE
// summaries, gist.science, section 3 "Chunkability Boundary": with the
// erase on the key axis only, one triangular solve per block serves every
// value row).  For a block with start state S (DV x DK):
//
//   Gamma_t = exp(g_1 + .. + g_t)  (per key channel), gamma = Gamma_C
//   K~ = K Gamma, K^ = K / Gamma, Q~ = Q Gamma_{t-1}, kap^ = b K / Gamma
//   A = sl(K~ kap^T), M = sl(K~ K^T), P_k = sl(Q~ K^T), P_kap = sl(Q~ kap^T)
//   T = (I + A)^{-1}, W = w V
//   E = T (K~ S^T + M W)                  WY pseudo-values
//   O = Q~ S^T + P_k W - P_kap E          o_t = S_{t-1} q_t
//   S <- (S + W^T K^ - E^T kap^) Diag(gamma)
// (sl = strictly lower part).  The gate b_{c,t} = sigmoid(bx_t + U_up U_down
// m_c) is fixed per chunk, m_{c+1} is the mean of the chunk's L outputs
// (section 2.1, "Content-Aware Erase via Output Reuse").
//
// This path keeps the block's L x L matrices in shared memory and the
// larger per-block operands in an L2-resident per-pair scratch area of the
// workspace; every product is a plain fp32 FMA loop.  It serves the fp32
// I/O mode, every supported shape, and the backward pass.
#include "carve_internal.cuh"

namespace carve {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }

// out(i, j) = [out(i, j) if accumulate] + alpha * sum_k A(i, k) B(k, j)
// with A(i, k) = A[i*ars + k*acs] and B(k, j) = B[k*brs + j*bcs].
// strict_lower computes only j < i; the rest is set to 0 (or left alone
// when accumulating).
__device__ void mm(float* out, int ldo, const float* A, int ars, int acs,
                   const float* Bm, int brs, int bcs, int M, int N, int K,
                   float alpha, bool accumulate, bool strict_lower) {
  for (int idx = threadIdx.x; idx < M * N; idx += blockDim.x) {
    const int i = idx / N, j = idx - i * N;
    float acc = 0.f;
    const bool live = !strict_lower || j < i;
    if (live) {
      const float* ap = A + (size_t)i * ars;
      const float* bp = Bm + (size_t)j * bcs;
      for (int k = 0; k < K; ++k)
        acc = fmaf(ap[(size_t)k * acs], bp[(size_t)k * brs], acc);
    }
    float* o = out + (size_t)i * ldo + j;
    if (accumulate) {
      if (live) *o += alpha * acc;
    } else {
      *o = alpha * acc;
    }
  }
  __syncthreads();
}

// T = (I + A)^{-1} for strictly-lower A (C x C, row-major), by forward
// substitution; each thread owns one column of T.
__device__ void unit_lower_inverse(float* sT, const float* sA, int C) {
  for (int j = threadIdx.x; j < C; j += blockDim.x) {
    for (int i = 0; i <= j; ++i) sT[i * C + j] = (i == j) ? 1.f : 0.f;
    for (int i = j + 1; i < C; ++i) {
      float acc = 0.f;
      for (int l = j; l < i; ++l) acc = fmaf(sA[i * C + l], sT[l * C + j], acc);
      sT[i * C + j] = -acc;
    }
  }
  __syncthreads();
}

// Index of element (b, t, h, j) of a [B, T, H, D] tensor.
__device__ __forceinline__ size_t bthd(int b, int t, int h, int j, int T,
                                       int H, int D) {
  return (((size_t)b * T + t) * H + h) * D + j;
}

// Gate of one chunk: s_h = U_down m (R), s_p = U_up s_h (DK).
template <typename TIn>
__device__ void content_gate(const TIn* ud, const TIn* uu, const float* s_m,
                             float* s_h, float* s_p, int h, int R, int DK,
                             int DV) {
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float acc = 0.f;
    for (int v = 0; v < DV; ++v)
      acc = fmaf(ldf(ud, ((size_t)h * R + r) * DV + v), s_m[v], acc);
    s_h[r] = acc;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < DK; j += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < R; ++r)
      acc = fmaf(ldf(uu, ((size_t)h * DK + j) * R + r), s_h[r], acc);
    s_p[j] = acc;
  }
  __syncthreads();
}

// Per-token inverse Euclidean norms of q and k over DK for the block's Cb
// tokens (one warp per token), or 1 when the inputs are used as given.
template <typename TIn>
__device__ void token_inv_norms(const TIn* q, const TIn* k, int b, int t0,
                                int T, int h, int H, int Cb, int DK,
                                float* s_qn, float* s_kn, int on) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < Cb; i += blockDim.x >> 5) {
    float sq = 0.f, sk = 0.f;
    if (on)
      for (int j = lane; j < DK; j += 32) {
        const size_t x = bthd(b, t0 + i, h, j, T, H, DK);
        const float qq = ldf(q, x), kk = ldf(k, x);
        sq = fmaf(qq, qq, sq);
        sk = fmaf(kk, kk, sk);
      }
    for (int o = 16; o >= 1; o >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      sk += __shfl_xor_sync(0xffffffffu, sk, o);
    }
    if (lane == 0) {
      s_qn[i] = on ? 1.0f / sqrtf(sq) : 1.f;
      s_kn[i] = on ? 1.0f / sqrtf(sk) : 1.f;
    }
  }
  __syncthreads();
}

// Decay scan and gated operands of one block.  Writes K~, K^, Q~, kap^
// ([C][DK] fp32), optionally log Gamma, and gamma (s_gam), plus W = w V.
template <typename TIn>
__device__ void block_operands(const TIn* q, const TIn* k, const TIn* v,
                               const TIn* g, const TIn* bx, const TIn* w,
                               const float* s_p, int b, int h, int t0, int T,
                               int H, int C, int DK, int DV, float* Kt,
                               float* Kh, float* Qt, float* Kp, float* Gl,
                               float* s_gam, float* s_w, float* W,
                               float dscale, const float* s_qn,
                               const float* s_kn, int erase) {
  for (int j = threadIdx.x; j < DK; j += blockDim.x) {
    float G = 0.f;
    for (int i = 0; i < C; ++i) {
      const size_t x = bthd(b, t0 + i, h, j, T, H, DK);
      const float kk = ldf(k, x) * s_kn[i], qq = ldf(q, x) * s_qn[i];
      const float bb = sigm(ldf(bx, x) + s_p[j]);
      const float Gm = G;
      G += decay_act(ldf(g, x), dscale);
      const float gam = expf(G), igam = expf(-G);
      Kt[i * DK + j] = kk * gam;
      Kh[i * DK + j] = kk * igam;
      Qt[i * DK + j] = qq * expf(Gm);
      // kap^ = b K / Gamma; the other erase form reads with kap~ = b K Gamma
      Kp[i * DK + j] = bb * kk * (erase ? gam : igam);
      if (Gl) Gl[i * DK + j] = G;
    }
    s_gam[j] = expf(G);
  }
  for (int i = threadIdx.x; i < C; i += blockDim.x)
    s_w[i] = ldf(w, ((size_t)b * T + t0 + i) * H + h);
  __syncthreads();
  for (int idx = threadIdx.x; idx < C * DV; idx += blockDim.x) {
    const int i = idx / DV, vv = idx - i * DV;
    W[idx] = s_w[i] * ldf(v, bthd(b, t0 + i, h, vv, T, H, DV));
  }
  __syncthreads();
}

// The four strictly-lower Gram matrices and T of one block (the other
// erase form: A = tril(kap~ K^T) and P_k only).
__device__ void block_grams(const float* Kt, const float* Kh, const float* Qt,
                            const float* Kp, int C, int DK, float* sA,
                            float* sT, float* sM, float* sPk, float* sPq,
                            int erase) {
  if (erase) {
    mm(sA, C, Kp, DK, 1, Kh, 1, DK, C, C, DK, 1.f, false, true);
    mm(sPk, C, Qt, DK, 1, Kh, 1, DK, C, C, DK, 1.f, false, true);
    unit_lower_inverse(sT, sA, C);
    return;
  }
  // X Y^T: A(i, k) = X[i*DK + k], B(k, j) = Y[j*DK + k]
  mm(sA, C, Kt, DK, 1, Kp, 1, DK, C, C, DK, 1.f, false, true);
  mm(sM, C, Kt, DK, 1, Kh, 1, DK, C, C, DK, 1.f, false, true);
  mm(sPk, C, Qt, DK, 1, Kh, 1, DK, C, C, DK, 1.f, false, true);
  mm(sPq, C, Qt, DK, 1, Kp, 1, DK, C, C, DK, 1.f, false, true);
  unit_lower_inverse(sT, sA, C);
}

template <typename TIn>
__global__ void __launch_bounds__(kThreads) fwd_generic_kernel(FwdArgs a) {
  extern __shared__ float smem[];
  const int C = a.C, DK = a.DK, DV = a.DV, R = a.R, H = a.H, T = a.T;
  const int pair = blockIdx.x, b = pair / H, h = pair - b * H;
  const int tid = threadIdx.x, nt = blockDim.x;
  const TIn* q = (const TIn*)a.q;
  const TIn* k = (const TIn*)a.k;
  const TIn* v = (const TIn*)a.v;
  const TIn* g = (const TIn*)a.g;
  const TIn* bx = (const TIn*)a.bx;
  const TIn* w = (const TIn*)a.w;
  const TIn* ud = (const TIn*)a.u_down;
  const TIn* uu = (const TIn*)a.u_up;
  TIn* o = (TIn*)a.o;
  // a training forward of this family: tensor-core records are not written
  if (a.ck_S && pair == 0 && tid == 0) a.hdr->magic = kWsMagic;

  float* sA = smem;
  float* sT = sA + C * C;
  float* sM = sT + C * C;
  float* sPk = sM + C * C;
  float* sPq = sPk + C * C;
  float* s_m = sPq + C * C;   // DV
  float* s_msum = s_m + DV;   // DV
  float* s_h = s_msum + DV;   // kMaxR
  float* s_p = s_h + kMaxR;   // DK
  float* s_gam = s_p + DK;    // DK
  float* s_w = s_gam + DK;    // C
  float* s_qn = s_w + C;      // C: per-token inverse norms of q, k
  float* s_kn = s_qn + C;     // C

  float* Kt = a.scratch + (size_t)pair * a.scratch_per_pair;
  float* Kh = Kt + C * DK;
  float* Qt = Kh + C * DK;
  float* Kp = Qt + C * DK;
  float* W = Kp + C * DK;
  float* Rr = W + C * DV;
  float* E = Rr + C * DV;
  float* O = E + C * DV;
  float* S = O + C * DV;

  const size_t SZ = (size_t)DV * DK;
  for (size_t i = tid; i < SZ; i += nt)
    S[i] = a.S0 ? a.S0[(size_t)pair * SZ + i] : 0.f;
  for (int i = tid; i < DV; i += nt)
    s_m[i] = a.m0 ? a.m0[(size_t)pair * DV + i] : 0.f;
  // this sequence's tokens: B sequences of T tokens, or packed sequences
  // [cu[b], cu[b + 1]) of a T-token tensor; the last block may be partial
  int tok0 = b * T, Tn = T;
  if (a.cu) {
    tok0 = a.cu[b];
    Tn = a.cu[b + 1] - tok0;
    if (tok0 < 0 || Tn < 0 || tok0 > T - Tn) {  // malformed offsets: skip
      if (tid == 0) {
        atomicExch(&a.hdr->status, (uint32_t)CARVE_ERR_INVALID_ARG);
        a.hdr->where = 90;
      }
      tok0 = 0;
      Tn = 0;
    }
  }
  __syncthreads();

  // chunks of L tokens from the sequence's start, solved in blocks of up to
  // C tokens (token addresses below use the packed index tok0 + t)
  for (int t0 = 0; t0 < Tn; t0 += C) {
    const int Cb = min(C, Tn - t0);
    const int c = t0 / a.L, ib = t0 / C;
    if (t0 % a.L == 0) {  // first block of chunk c: its gate
      if (a.ck_m)
        for (int i = tid; i < DV; i += nt)
          a.ck_m[((size_t)pair * a.NC + c) * DV + i] = s_m[i];
      content_gate(ud, uu, s_m, s_h, s_p, h, R, DK, DV);
      for (int i = tid; i < DV; i += nt) s_msum[i] = 0.f;
    }
    {
      const int tt = tok0 + t0;  // packed index of the block's first token
      if (a.ck_S) {
        float* dst = a.ck_S + ((size_t)pair * (a.NB + 1) + ib) * SZ;
        for (size_t i = tid; i < SZ; i += nt) dst[i] = S[i];
      }
      token_inv_norms(q, k, 0, tt, T, h, H, Cb, DK, s_qn, s_kn, a.qknorm);
      block_operands(q, k, v, g, bx, w, s_p, 0, h, tt, T, H, Cb, DK, DV, Kt,
                     Kh, Qt, Kp, (float*)nullptr, s_gam, s_w, W, a.dscale,
                     s_qn, s_kn, a.erase);
      block_grams(Kt, Kh, Qt, Kp, Cb, DK, sA, sT, sM, sPk, sPq, a.erase);
      if (a.erase) {
        // other erase form: R = kap~ S^T - W ; E = T R ; O = Q~ S^T - P_k E
        mm(Rr, DV, Kp, DK, 1, S, 1, DK, Cb, DV, DK, 1.f, false, false);
        for (int idx = tid; idx < Cb * DV; idx += nt) Rr[idx] -= W[idx];
        __syncthreads();
        mm(E, DV, sT, Cb, 1, Rr, DV, 1, Cb, DV, Cb, 1.f, false, false);
        mm(O, DV, Qt, DK, 1, S, 1, DK, Cb, DV, DK, 1.f, false, false);
        mm(O, DV, sPk, Cb, 1, E, DV, 1, Cb, DV, Cb, -1.f, true, false);
      } else {
        // R = K~ S^T + M W ;  E = T R
        mm(Rr, DV, Kt, DK, 1, S, 1, DK, Cb, DV, DK, 1.f, false, false);
        mm(Rr, DV, sM, Cb, 1, W, DV, 1, Cb, DV, Cb, 1.f, true, false);
        mm(E, DV, sT, Cb, 1, Rr, DV, 1, Cb, DV, Cb, 1.f, false, false);
        // O = Q~ S^T + P_k W - P_kap E
        mm(O, DV, Qt, DK, 1, S, 1, DK, Cb, DV, DK, 1.f, false, false);
        mm(O, DV, sPk, Cb, 1, W, DV, 1, Cb, DV, Cb, 1.f, true, false);
        mm(O, DV, sPq, Cb, 1, E, DV, 1, Cb, DV, Cb, -1.f, true, false);
      }
      for (int idx = tid; idx < Cb * DV; idx += nt) {
        const int i = idx / DV, vv = idx - i * DV;
        stf(o, bthd(0, tt + i, h, vv, T, H, DV), O[idx]);
      }
      for (int vv = tid; vv < DV; vv += nt) {
        float acc = 0.f;
        for (int i = 0; i < Cb; ++i) acc += O[i * DV + vv];
        s_msum[vv] += acc;
      }
      // S <- (S + W^T K^ - E^T kap^) Diag(gamma)
      //      (other erase form: S <- (S - E^T K^) Diag(gamma))
      for (size_t idx = tid; idx < SZ; idx += nt) {
        const int vv = (int)(idx / DK), j = (int)(idx - (size_t)vv * DK);
        float acc = S[idx];
        if (a.erase)
          for (int i = 0; i < Cb; ++i)
            acc = fmaf(-E[i * DV + vv], Kh[i * DK + j], acc);
        else
          for (int i = 0; i < Cb; ++i)
            acc = fmaf(W[i * DV + vv], Kh[i * DK + j],
                       fmaf(-E[i * DV + vv], Kp[i * DK + j], acc));
        S[idx] = acc * s_gam[j];
      }
      __syncthreads();
    }
    if ((t0 + Cb) % a.L == 0 || t0 + Cb == Tn) {  // chunk end (or the
      // sequence's end inside a chunk: that partial mean still divides by L)
      for (int i = tid; i < DV; i += nt) s_m[i] = s_msum[i] / (float)a.L;
      __syncthreads();
    }
  }
  if (a.ck_S) {
    float* dst = a.ck_S + ((size_t)pair * (a.NB + 1) + a.NB) * SZ;
    for (size_t i = tid; i < SZ; i += nt) dst[i] = S[i];
  }
  if (a.S_T)
    for (size_t i = tid; i < SZ; i += nt) a.S_T[(size_t)pair * SZ + i] = S[i];
  if (a.m_T)
    for (int i = tid; i < DV; i += nt) a.m_T[(size_t)pair * DV + i] = s_m[i];
}

template <typename TIn>
__global__ void __launch_bounds__(kThreads) bwd_generic_kernel(BwdArgs a) {
  extern __shared__ float smem[];
  const int C = a.C, DK = a.DK, DV = a.DV, R = a.R, H = a.H, T = a.T;
  const int pair = blockIdx.x, b = pair / H, h = pair - b * H;
  const int tid = threadIdx.x, nt = blockDim.x;
  // the fp32 block checkpoints exist only after this family's forward
  if (a.hdr->magic != kWsMagic) {
    if (tid == 0) {
      atomicExch(&a.hdr->status, (uint32_t)CARVE_ERR_WORKSPACE);
      a.hdr->where = 97;
    }
    return;
  }
  const TIn* q = (const TIn*)a.q;
  const TIn* k = (const TIn*)a.k;
  const TIn* v = (const TIn*)a.v;
  const TIn* g = (const TIn*)a.g;
  const TIn* bx = (const TIn*)a.bx;
  const TIn* w = (const TIn*)a.w;
  const TIn* ud = (const TIn*)a.u_down;
  const TIn* uu = (const TIn*)a.u_up;
  const TIn* d_o = (const TIn*)a.d_o;
  TIn* dq = (TIn*)a.dq;
  TIn* dk = (TIn*)a.dk;
  TIn* dv = (TIn*)a.dv;
  TIn* dg = (TIn*)a.dg;
  TIn* dbx = (TIn*)a.dbx;
  TIn* dw = (TIn*)a.dw;

  const int CC = C * C;
  float* sA = smem;
  float* sT = sA + CC;
  float* sM = sT + CC;
  float* sPk = sM + CC;
  float* sPq = sPk + CC;
  float* dA = sPq + CC;
  float* dM = dA + CC;
  float* dPk = dM + CC;
  float* dPq = dPk + CC;
  float* s_dmn = dPq + CC;   // DV: gradient of the mean of the current chunk
  float* s_mc = s_dmn + DV;  // DV
  float* s_h = s_mc + DV;    // kMaxR
  float* s_dh = s_h + kMaxR; // kMaxR
  float* s_p = s_dh + kMaxR; // DK
  float* s_gam = s_p + DK;   // DK
  float* s_dlg = s_gam + DK; // DK
  float* s_dp = s_dlg + DK;  // DK
  float* s_w = s_dp + DK;    // C
  float* s_qn = s_w + C;     // C: per-token inverse norms of q, k
  float* s_kn = s_qn + C;    // C

  float* Kt = a.scratch + (size_t)pair * a.scratch_per_pair;
  float* Kh = Kt + C * DK;
  float* Qt = Kh + C * DK;
  float* Kp = Qt + C * DK;
  float* Gl = Kp + C * DK;
  float* dKt = Gl + C * DK;
  float* dKh = dKt + C * DK;
  float* dKp = dKh + C * DK;
  float* dQt = dKp + C * DK;
  float* W = dQt + C * DK;
  float* Rr = W + C * DV;
  float* E = Rr + C * DV;
  float* dO = E + C * DV;
  float* dE = dO + C * DV;
  float* dR = dE + C * DV;
  float* dW = dR + C * DV;
  float* dS = dW + C * DV;
  float* dSb = dS + (size_t)DV * DK;
  float* Dq = dSb + (size_t)DV * DK;  // gradients of the unit q, k rows
  float* Dk = Dq + C * DK;            // (fused normalisation only)

  float* dUd = a.du + (size_t)pair * ((size_t)R * DV + (size_t)DK * R);
  float* dUu = dUd + (size_t)R * DV;

  const size_t SZ = (size_t)DV * DK;
  for (size_t i = tid; i < SZ; i += nt)
    dS[i] = a.dS_T ? a.dS_T[(size_t)pair * SZ + i] : 0.f;
  for (int i = tid; i < DV; i += nt)
    s_dmn[i] = a.dm_T ? a.dm_T[(size_t)pair * DV + i] : 0.f;
  for (int i = tid; i < R * DV + DK * R; i += nt) dUd[i] = 0.f;
  __syncthreads();

  const int bpc = a.L / C;
  const float invL = 1.0f / (float)a.L;
  for (int c = a.NC - 1; c >= 0; --c) {
    for (int i = tid; i < DV; i += nt)
      s_mc[i] = a.ck_m[((size_t)pair * a.NC + c) * DV + i];
    for (int j = tid; j < DK; j += nt) s_dp[j] = 0.f;
    __syncthreads();
    content_gate(ud, uu, s_mc, s_h, s_p, h, R, DK, DV);
    for (int blk = bpc - 1; blk >= 0; --blk) {
      const int ib = c * bpc + blk, t0 = ib * C;
      const float* S = a.ck_S + ((size_t)pair * (a.NB + 1) + ib) * SZ;
      const float* Sn = S + SZ;  // state at the end of this block
      token_inv_norms(q, k, b, t0, T, h, H, C, DK, s_qn, s_kn, a.qknorm);
      block_operands(q, k, v, g, bx, w, s_p, b, h, t0, T, H, C, DK, DV, Kt,
                     Kh, Qt, Kp, Gl, s_gam, s_w, W, a.dscale, s_qn, s_kn,
                     a.erase);
      block_grams(Kt, Kh, Qt, Kp, C, DK, sA, sT, sM, sPk, sPq, a.erase);
      if (a.erase) {
        mm(Rr, DV, Kp, DK, 1, S, 1, DK, C, DV, DK, 1.f, false, false);
        for (int idx = tid; idx < C * DV; idx += nt) Rr[idx] -= W[idx];
        __syncthreads();
      } else {
        mm(Rr, DV, Kt, DK, 1, S, 1, DK, C, DV, DK, 1.f, false, false);
        mm(Rr, DV, sM, C, 1, W, DV, 1, C, DV, C, 1.f, true, false);
      }
      mm(E, DV, sT, C, 1, Rr, DV, 1, C, DV, C, 1.f, false, false);
      // upstream gradient of O, including this chunk's share of dm_{c+1}
      for (int idx = tid; idx < C * DV; idx += nt) {
        const int i = idx / DV, vv = idx - i * DV;
        dO[idx] = ldf(d_o, bthd(b, t0 + i, h, vv, T, H, DV)) + s_dmn[vv] * invL;
      }
      // dS holds the gradient of the block-end state; dS~ = dS Diag(gamma)
      for (size_t idx = tid; idx < SZ; idx += nt) {
        const int j = (int)(idx % DK);
        dSb[idx] = dS[idx] * s_gam[j];
      }
      for (int j = tid; j < DK; j += nt) {
        float acc = 0.f;
        for (int vv = 0; vv < DV; ++vv)
          acc = fmaf(dS[(size_t)vv * DK + j], Sn[(size_t)vv * DK + j], acc);
        s_dlg[j] = acc;  // gradient of log gamma_j
      }
      __syncthreads();
      if (a.erase) {
        // other erase form (R = kap~ S^T - W, A = tril(kap~ K^T),
        // O = Q~ S^T - P_k E, S_new = (S - E^T K^) Diag(gamma)):
        // dE = -K^ dS~^T - P_k^T dO ;  dR = T^T dE
        mm(dE, DV, Kh, DK, 1, dSb, 1, DK, C, DV, DK, -1.f, false, false);
        mm(dE, DV, sPk, 1, C, dO, DV, 1, C, DV, C, -1.f, true, false);
        mm(dR, DV, sT, 1, C, dE, DV, 1, C, DV, C, 1.f, false, false);
        mm(dA, C, dR, DV, 1, E, 1, DV, C, C, DV, -1.f, false, true);
        mm(dPk, C, dO, DV, 1, E, 1, DV, C, C, DV, -1.f, false, true);
        for (int idx = tid; idx < C * DV; idx += nt) dW[idx] = -dR[idx];
        __syncthreads();
        for (int idx = tid; idx < C * DV; idx += nt) {
          const int i = idx / DV, vv = idx - i * DV;
          stf(dv, bthd(b, t0 + i, h, vv, T, H, DV), s_w[i] * dW[idx]);
        }
        for (int i = tid; i < C; i += nt) {
          float acc = 0.f;
          for (int vv = 0; vv < DV; ++vv)
            acc = fmaf(dW[i * DV + vv], ldf(v, bthd(b, t0 + i, h, vv, T, H, DV)), acc);
          stf(dw, ((size_t)b * T + t0 + i) * H + h, acc);
        }
        for (int idx = tid; idx < C * DK; idx += nt) dKt[idx] = 0.f;
        // dkap~ = dR S + dA K^ ;  dK^ = dA^T kap~ + dP_k^T Q~ - E dS~
        mm(dKp, DK, dR, DV, 1, S, DK, 1, C, DK, DV, 1.f, false, false);
        mm(dKp, DK, dA, C, 1, Kh, DK, 1, C, DK, C, 1.f, true, false);
        mm(dKh, DK, dA, 1, C, Kp, DK, 1, C, DK, C, 1.f, false, false);
        mm(dKh, DK, dPk, 1, C, Qt, DK, 1, C, DK, C, 1.f, true, false);
        mm(dKh, DK, E, DV, 1, dSb, DK, 1, C, DK, DV, -1.f, true, false);
        // dQ~ = dO S + dP_k K^
        mm(dQt, DK, dO, DV, 1, S, DK, 1, C, DK, DV, 1.f, false, false);
        mm(dQt, DK, dPk, C, 1, Kh, DK, 1, C, DK, C, 1.f, true, false);
      } else {
        // dE = -kap^ dS~^T - P_kap^T dO ;  dR = T^T dE
        mm(dE, DV, Kp, DK, 1, dSb, 1, DK, C, DV, DK, -1.f, false, false);
        mm(dE, DV, sPq, 1, C, dO, DV, 1, C, DV, C, -1.f, true, false);
        mm(dR, DV, sT, 1, C, dE, DV, 1, C, DV, C, 1.f, false, false);
        // gradients of the four Gram matrices (strictly lower)
        mm(dA, C, dR, DV, 1, E, 1, DV, C, C, DV, -1.f, false, true);
        mm(dM, C, dR, DV, 1, W, 1, DV, C, C, DV, 1.f, false, true);
        mm(dPk, C, dO, DV, 1, W, 1, DV, C, C, DV, 1.f, false, true);
        mm(dPq, C, dO, DV, 1, E, 1, DV, C, C, DV, -1.f, false, true);
        // dW = K^ dS~^T + P_k^T dO + M^T dR
        mm(dW, DV, Kh, DK, 1, dSb, 1, DK, C, DV, DK, 1.f, false, false);
        mm(dW, DV, sPk, 1, C, dO, DV, 1, C, DV, C, 1.f, true, false);
        mm(dW, DV, sM, 1, C, dR, DV, 1, C, DV, C, 1.f, true, false);
        for (int idx = tid; idx < C * DV; idx += nt) {
          const int i = idx / DV, vv = idx - i * DV;
          stf(dv, bthd(b, t0 + i, h, vv, T, H, DV), s_w[i] * dW[idx]);
        }
        for (int i = tid; i < C; i += nt) {
          float acc = 0.f;
          for (int vv = 0; vv < DV; ++vv)
            acc = fmaf(dW[i * DV + vv], ldf(v, bthd(b, t0 + i, h, vv, T, H, DV)), acc);
          stf(dw, ((size_t)b * T + t0 + i) * H + h, acc);
        }
        // dK~ = dR S + dA kap^ + dM K^
        mm(dKt, DK, dR, DV, 1, S, DK, 1, C, DK, DV, 1.f, false, false);
        mm(dKt, DK, dA, C, 1, Kp, DK, 1, C, DK, C, 1.f, true, false);
        mm(dKt, DK, dM, C, 1, Kh, DK, 1, C, DK, C, 1.f, true, false);
        // dK^ = dM^T K~ + dP_k^T Q~ + W dS~
        mm(dKh, DK, dM, 1, C, Kt, DK, 1, C, DK, C, 1.f, false, false);
        mm(dKh, DK, dPk, 1, C, Qt, DK, 1, C, DK, C, 1.f, true, false);
        mm(dKh, DK, W, DV, 1, dSb, DK, 1, C, DK, DV, 1.f, true, false);
        // dkap^ = dA^T K~ + dP_kap^T Q~ - E dS~
        mm(dKp, DK, dA, 1, C, Kt, DK, 1, C, DK, C, 1.f, false, false);
        mm(dKp, DK, dPq, 1, C, Qt, DK, 1, C, DK, C, 1.f, true, false);
        mm(dKp, DK, E, DV, 1, dSb, DK, 1, C, DK, DV, -1.f, true, false);
        // dQ~ = dO S + dP_k K^ + dP_kap kap^
        mm(dQt, DK, dO, DV, 1, S, DK, 1, C, DK, DV, 1.f, false, false);
        mm(dQt, DK, dPk, C, 1, Kh, DK, 1, C, DK, C, 1.f, true, false);
        mm(dQt, DK, dPq, C, 1, Kp, DK, 1, C, DK, C, 1.f, true, false);
      }
      // gradient of the block-start state: dS~ + dO^T Q~ + dR^T K~
      // (other erase form: dR^T kap~)
      const float* Rk = a.erase ? Kp : Kt;
      for (size_t idx = tid; idx < SZ; idx += nt) {
        const int vv = (int)(idx / DK), j = (int)(idx - (size_t)vv * DK);
        float acc = dSb[idx];
        for (int i = 0; i < C; ++i)
          acc = fmaf(dO[i * DV + vv], Qt[i * DK + j],
                     fmaf(dR[i * DV + vv], Rk[i * DK + j], acc));
        dS[idx] = acc;
      }
      // per key channel: chain rule through Gamma, the gate and the inputs;
      // dg is the reverse cumulative sum of the log-Gamma gradients.
      for (int j = tid; j < DK; j += nt) {
        float acc = 0.f;
        for (int i = C - 1; i >= 0; --i) {
          const size_t x = bthd(b, t0 + i, h, j, T, H, DK);
          const int e = i * DK + j;
          const float G = Gl[e];
          const float Gm = i > 0 ? Gl[e - DK] : 0.f;
          const float gam = expf(G), igam = expf(-G);
          const float kk = ldf(k, x) * s_kn[i];
          const float bb = sigm(ldf(bx, x) + s_p[j]);
          const float gq = dQt[e] * expf(Gm);
          // kap^ = b K / Gamma (kap~ = b K Gamma in the other erase form)
          const float kps = a.erase ? gam : igam;
          const float gk = dKt[e] * gam + dKh[e] * igam + dKp[e] * bb * kps;
          if (a.qknorm) {  // gradients of the unit rows: projected below
            Dq[e] = gq;
            Dk[e] = gk;
          } else {
            stf(dq, x, gq);
            stf(dk, x, gk);
          }
          const float dz = dKp[e] * kk * kps * bb * (1.f - bb);
          stf(dbx, x, dz);
          s_dp[j] += dz;
          float dG = dKt[e] * Kt[e] - dKh[e] * Kh[e] +
                     (a.erase ? dKp[e] : -dKp[e]) * Kp[e];
          if (i == C - 1) dG += s_dlg[j];
          if (i + 1 < C) dG += dQt[e + DK] * Qt[e + DK];
          acc += dG;
          // with raw decay logits, dL/da = dL/dg * (-s sigmoid(a))
          stf(dg, x, a.dscale > 0.f
                         ? acc * -a.dscale * sigm(ldf(g, x))
                         : acc);
        }
      }
      __syncthreads();
      if (a.qknorm) {
        // fused normalisation: x^ = x / |x| per token, so the raw
        // gradient is (dx^ - x^ (x^ . dx^)) / |x| (one warp per token)
        const int warp = tid >> 5, lane = tid & 31;
        for (int i = warp; i < C; i += nt >> 5) {
          float dotq = 0.f, dotk = 0.f;
          for (int j = lane; j < DK; j += 32) {
            const size_t x = bthd(b, t0 + i, h, j, T, H, DK);
            dotq = fmaf(ldf(q, x) * s_qn[i], Dq[i * DK + j], dotq);
            dotk = fmaf(ldf(k, x) * s_kn[i], Dk[i * DK + j], dotk);
          }
          for (int o = 16; o >= 1; o >>= 1) {
            dotq += __shfl_xor_sync(0xffffffffu, dotq, o);
            dotk += __shfl_xor_sync(0xffffffffu, dotk, o);
          }
          for (int j = lane; j < DK; j += 32) {
            const size_t x = bthd(b, t0 + i, h, j, T, H, DK);
            const float qh = ldf(q, x) * s_qn[i], kh = ldf(k, x) * s_kn[i];
            stf(dq, x, (Dq[i * DK + j] - qh * dotq) * s_qn[i]);
            stf(dk, x, (Dk[i * DK + j] - kh * dotk) * s_kn[i]);
          }
        }
        __syncthreads();
      }
    }
    // gate of chunk c: p = U_up h, h = U_down m_c
    for (int idx = tid; idx < DK * R; idx += nt) {
      const int j = idx / R, r = idx - j * R;
      dUu[idx] += s_dp[j] * s_h[r];
    }
    for (int r = tid; r < R; r += nt) {
      float acc = 0.f;
      for (int j = 0; j < DK; ++j)
        acc = fmaf(ldf(uu, ((size_t)h * DK + j) * R + r), s_dp[j], acc);
      s_dh[r] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < R * DV; idx += nt) {
      const int r = idx / DV, vv = idx - r * DV;
      dUd[idx] += s_dh[r] * s_mc[vv];
    }
    for (int vv = tid; vv < DV; vv += nt) {
      float acc = 0.f;
      for (int r = 0; r < R; ++r)
        acc = fmaf(ldf(ud, ((size_t)h * R + r) * DV + vv), s_dh[r], acc);
      s_dmn[vv] = acc;  // gradient of m_c, spread over chunk c-1
    }
    __syncthreads();
  }
  if (a.dS0)
    for (size_t i = tid; i < SZ; i += nt) a.dS0[(size_t)pair * SZ + i] = dS[i];
  if (a.dm0)
    for (int i = tid; i < DV; i += nt) a.dm0[(size_t)pair * DV + i] = s_dmn[i];
}

// du_down[h] = sum_b partial[b, h] (and du_up likewise), fixed order.
__global__ void du_reduce_kernel(const float* __restrict__ part, int B, int H,
                                 int R, int DK, int DV, float* du_down,
                                 float* du_up) {
  const size_t per = (size_t)R * DV + (size_t)DK * R;
  const size_t n = (size_t)H * per;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int h = (int)(idx / per);
    const size_t e = idx - (size_t)h * per;
    float acc = 0.f;
    for (int bb = 0; bb < B; ++bb) acc += part[((size_t)bb * H + h) * per + e];
    if (e < (size_t)R * DV)
      du_down[(size_t)h * R * DV + e] = acc;
    else
      du_up[(size_t)h * DK * R + (e - (size_t)R * DV)] = acc;
  }
}

}  // namespace

size_t generic_fwd_smem_bytes(int C, int DK, int DV) {
  return (size_t)(5 * C * C + 2 * DV + kMaxR + 2 * DK + 3 * C) * sizeof(float);
}
size_t generic_bwd_smem_bytes(int C, int DK, int DV) {
  return (size_t)(9 * C * C + 2 * DV + 2 * kMaxR + 4 * DK + 3 * C) * sizeof(float);
}

cudaError_t launch_fwd_generic(const FwdArgs& a, int dtype, cudaStream_t st) {
  const size_t smem = generic_fwd_smem_bytes(a.C, a.DK, a.DV);
  const int grid = a.B * a.H;
  cudaError_t e;
  if (dtype == CARVE_BF16) {
    e = cudaFuncSetAttribute(fwd_generic_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    fwd_generic_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(fwd_generic_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    fwd_generic_kernel<float><<<grid, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_generic(const BwdArgs& a, int dtype, cudaStream_t st) {
  const size_t smem = generic_bwd_smem_bytes(a.C, a.DK, a.DV);
  const int grid = a.B * a.H;
  cudaError_t e;
  if (dtype == CARVE_BF16) {
    e = cudaFuncSetAttribute(bwd_generic_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_generic_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(bwd_generic_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_generic_kernel<float><<<grid, kThreads, smem, st>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)a.H * ((size_t)a.R * a.DV + (size_t)a.DK * a.R);
  if (n > 0) {
    const int threads = 256;
    int blocks = (int)((n + threads - 1) / threads);
    if (blocks > 4 * 148) blocks = 4 * 148;
    du_reduce_kernel<<<blocks, threads, 0, st>>>(a.du, a.B, a.H, a.R, a.DK,
                                                 a.DV, a.du_down, a.du_up);
  }
  return cudaGetLastError();
}

}  // namespace carve
