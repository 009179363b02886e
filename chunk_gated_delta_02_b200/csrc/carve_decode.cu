// carve_decode.cu -- the single-token recurrent decode step (inference).
//
// One new token per (sequence, head) advances the state the way the token
// form of the recurrence does (CARVE technical summary, gist.science,
// sections 1, 2.1-2.3):
//
//   p  = U_up (U_down m_c)         the chunk's content signal (one chunk stale)
//   b  = sigmoid(b_x + p)          erase gate on the key axis
//   o  = S q                       o_t = S_{t-1} q_t
//   S' = S Diag(exp g)             key-axis decay
//   S  = S' - (S' k)(b k)^T + w v k^T
//   osum += o; at the chunk's last token m_{c+1} = osum / L, osum = 0
//
// Memory-bound: every step reads and writes the fp32 state once.  Each value
// row of S is independent once the key-side vectors (q, exp g, k, b k) are
// known, so a (sequence, head) pair runs as a cluster of kSplit CTAs, each
// owning a quarter of the value rows: every CTA forms the key-side vectors
// and the gate itself (they are small) while its rows of S arrive in shared
// memory by bulk copies (requested first, on the copy engine), then its
// warps take batches of rows, reduce S q and S' k of a batch together by
// shuffles, and write the new rows back.  The gate of every CTA reads all of m_c, which a
// chunk's last token rewrites row by row, so at that token the CTAs of a
// cluster meet once after staging m_c and before any of them can write it.
#include <cuda_bf16.h>

#include "carve_internal.cuh"
#include "sm100_ptx.cuh"

namespace carve {
namespace {

constexpr int kDecThreads = 128;   // 4 warps per CTA
constexpr int kSplit = 4;          // CTAs (a cluster) per (sequence, head)
constexpr int kDecWarps = kDecThreads / 32;
constexpr long long kDecWaitCycles = 1ll << 31;  // a copy wait gives up (~1 s)

__device__ __forceinline__ float allsum(float x) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) x += __shfl_xor_sync(0xffffffffu, x, k);
  return x;
}

// Warp sums of N values at once (N = 8 or 16): lane l ends with the sum over
// the warp of v[l % N] (N - 1 + log2(32 / N) shuffles instead of 5 N).  At
// the step for bit k a lane keeps the half of its values whose index has
// bit k equal to its own lane bit k, adding its partner's copy of them.
template <int N>
__device__ __forceinline__ float reduce_scatter(float* v, int lane) {
#pragma unroll
  for (int k = N / 2; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = up ? v[i] : v[i + k];
      const float keep = up ? v[i + k] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  float x = v[0];
#pragma unroll
  for (int k = N; k < 32; k <<= 1) x += __shfl_xor_sync(0xffffffffu, x, k);
  return x;
}

// 16-byte vector of the I/O dtype -> fp32 (8 bf16 or 4 fp32 elements).
template <typename TIn>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* x) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const float* p, float* x) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
  }
};

// NJ = columns per lane (DK <= 32 NJ)
template <typename TIn, int NJ>
__global__ void __launch_bounds__(kDecThreads)
    decode_kernel(const DecArgs a) {
  extern __shared__ float dsm[];
  const int DK = a.DK, DV = a.DV, R = a.R;
  float* s_q = dsm;             // q            [DK]
  float* s_k = s_q + DK;        // k            [DK]
  float* s_al = s_k + DK;       // exp(g)       [DK]
  float* s_kp = s_al + DK;      // b k          [DK]
  float* s_bx = s_kp + DK;      // b_x          [DK]
  float* s_m = s_bx + DK;       // m_c          [DV]
  float* s_v = s_m + DV;        // v            [DV]
  float* s_h = s_v + DV;        // U_down m_c   [R]
  // the head's U_b factors in the I/O dtype, as stored: U_down [R][DV],
  // U_up [DK][R]
  TIn* s_ud = reinterpret_cast<TIn*>(
      (reinterpret_cast<uintptr_t>(s_h + (R > 0 ? R : 1)) + 15) & ~uintptr_t(15));
  TIn* s_uu = s_ud + R * DV;
  // raw copies of the token's vectors and m_c (16-byte aligned): q, k, g,
  // b_x [DK], v [DV] in the I/O dtype, then m_c [DV] fp32
  TIn* s_raw = s_uu + DK * R;
  float* s_mraw = reinterpret_cast<float*>(s_raw + 4 * DK + DV);
  const int pair = blockIdx.x / kSplit, part = blockIdx.x % kSplit;
  const int bseq = pair / a.H, h = pair - bseq * a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* S = a.S + (size_t)pair * DV * DK;
  // this CTA's value rows rlo .. rlo + nrow - 1 (DV is a multiple of 16,
  // so rq is a multiple of 4 and each CTA's rows start on a 16-byte
  // boundary of the output sums too)
  const int rq = DV / kSplit;
  const int rlo = part * rq, nrow = rq;
  // the CTA's rows of S [nrow][DK] and of the running output sum [nrow],
  // fp32, after m_c
  float* s_S = s_mraw + DV;
  float* s_os = s_S + (size_t)rq * DK;
  float* osum = a.osum + (size_t)pair * DV;

  const TIn* q = static_cast<const TIn*>(a.q) + (size_t)pair * DK;
  const TIn* k = static_cast<const TIn*>(a.k) + (size_t)pair * DK;
  const TIn* g = static_cast<const TIn*>(a.g) + (size_t)pair * DK;
  const TIn* bx = static_cast<const TIn*>(a.bx) + (size_t)pair * DK;
  const TIn* v = static_cast<const TIn*>(a.v) + (size_t)pair * DV;
  float* m = a.m + (size_t)pair * DV;
  TIn* o = static_cast<TIn*>(a.o) + (size_t)pair * DV;
  const float w = ldf(static_cast<const TIn*>(a.w), pair);
  const bool chunk_end = (a.pos[bseq] + 1) % a.L == 0;

  // Everything the CTA reads comes in by bulk copies that thread 0 issues
  // at once (the copy engine, not the load/store pipe the gate uses): the
  // head's U_b factors, the token's vectors and m_c on mbarrier 0, then
  // the CTA's rows of S and of the output sum on mbarrier 1, which land
  // while the gate is formed.  Each barrier completes once (parity 0); a
  // wait gives up after a.wait_cycles (normally kDecWaitCycles), and a CTA
  // whose copies did not land leaves S, m and the sums as they were and
  // writes NaN to its o.
  __shared__ __align__(8) uint64_t s_bar[2];
  if (tid == 0) {
    ptx::mbar_init(&s_bar[0], 1);
    ptx::mbar_init(&s_bar[1], 1);
    ptx::mbar_init_fence();
  }
  __syncthreads();
  // (test only, a.stall: CTA 0 announces its first group's bytes but
  // issues none of its copies, so that group never completes and the wait
  // for it gives up; nothing of it is in flight when the CTA leaves)
  const bool issue0 = !(a.stall && blockIdx.x == 0);
  if (tid == 0) {
    constexpr uint32_t sz = sizeof(TIn);
    ptx::mbar_expect_tx(&s_bar[0], (uint32_t)(R * (DV + DK) + 4 * DK + DV) * sz +
                                       (uint32_t)DV * 4u);
  }
  if (tid == 0 && issue0) {
    constexpr uint32_t sz = sizeof(TIn);
    if (R > 0) {
      ptx::bulk_load(s_ud, static_cast<const TIn*>(a.u_down) + (size_t)h * R * DV,
                     (uint32_t)(R * DV) * sz, &s_bar[0]);
      ptx::bulk_load(s_uu, static_cast<const TIn*>(a.u_up) + (size_t)h * DK * R,
                     (uint32_t)(DK * R) * sz, &s_bar[0]);
    }
    ptx::bulk_load(s_raw, q, (uint32_t)DK * sz, &s_bar[0]);
    ptx::bulk_load(s_raw + DK, k, (uint32_t)DK * sz, &s_bar[0]);
    ptx::bulk_load(s_raw + 2 * DK, g, (uint32_t)DK * sz, &s_bar[0]);
    ptx::bulk_load(s_raw + 3 * DK, bx, (uint32_t)DK * sz, &s_bar[0]);
    ptx::bulk_load(s_raw + 4 * DK, v, (uint32_t)DV * sz, &s_bar[0]);
    ptx::bulk_load(s_mraw, m, (uint32_t)DV * 4u, &s_bar[0]);
  }
  if (tid == 0) {
    ptx::mbar_expect_tx(&s_bar[1], (uint32_t)(nrow * DK + nrow) * 4u);
    ptx::bulk_load(s_S, S + (size_t)rlo * DK, (uint32_t)(nrow * DK) * 4u, &s_bar[1]);
    ptx::bulk_load(s_os, osum + rlo, (uint32_t)nrow * 4u, &s_bar[1]);
  }
  // every thread waits on the barrier itself (measured: faster than one
  // warp waiting while the others sit at the CTA barrier after it)
  auto mwait = [&](uint64_t* bar, long long limit) {
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, 0))
      if (clock64() - t0 > limit) return false;
    return true;
  };
  auto give_up = [&]() {  // after the last cluster barrier only
    // the state copies land before the CTA leaves (on the full limit)
    mwait(&s_bar[1], kDecWaitCycles);
    for (int rl = tid; rl < nrow; rl += kDecThreads) stf(o, rlo + rl, __int_as_float(0x7fc00000));
  };
  const bool bad = __syncthreads_or(!mwait(&s_bar[0], a.wait_cycles));
  if (!bad) {
    for (int j = tid; j < DK; j += kDecThreads) {
      s_q[j] = ldf(s_raw, j);
      s_k[j] = ldf(s_raw + DK, j);
      s_al[j] = ldf(s_raw + 2 * DK, j);
      s_bx[j] = ldf(s_raw + 3 * DK, j);
    }
    for (int i = tid; i < DV; i += kDecThreads) {
      s_v[i] = ldf(s_raw + 4 * DK, i);
      s_m[i] = s_mraw[i];
    }
  }
  __syncthreads();
  // every CTA of the pair has m_c: a chunk's last token may now rewrite it
  // (only that token writes m, and chunk_end is the same for the whole
  // cluster, so the other tokens skip the barrier; every CTA takes it)
  if (chunk_end) ptx::cluster_sync();
  if (bad) {
    give_up();
    return;
  }
  if (a.qknorm) {  // fused normalisation: q / |q|, k / |k| (warp 0 reduces)
    if (warp == 0) {
      float sq = 0.f, sk = 0.f;
      for (int j = lane; j < DK; j += 32) {
        sq = fmaf(s_q[j], s_q[j], sq);
        sk = fmaf(s_k[j], s_k[j], sk);
      }
      sq = allsum(sq);
      sk = allsum(sk);
      if (lane == 0) {  // s_kp is free until the gate below
        s_kp[0] = sq > 0.f ? 1.0f / sqrtf(sq) : 0.f;
        s_kp[1] = sk > 0.f ? 1.0f / sqrtf(sk) : 0.f;
      }
    }
    __syncthreads();
    const float iq = s_kp[0], ik = s_kp[1];
    __syncthreads();  // every thread has read them before the gate rewrites s_kp
    for (int j = tid; j < DK; j += kDecThreads) {
      s_q[j] *= iq;
      s_k[j] *= ik;
    }
  }
  for (int j = tid; j < DK; j += kDecThreads)
    s_al[j] = __expf(decay_act(s_al[j], a.dscale));
  // h = U_down m_c and p = U_up h.  Where a factor's rows are a power of
  // two (<= 32) of 16-byte chunks, a warp instruction reads 32 consecutive
  // chunks (512 contiguous bytes: whole rows side by side, no bank
  // conflict), each lane takes the dot product of its chunk, and the lanes
  // of a row sum by shuffles; otherwise four threads per rank (h) and a
  // thread per key channel (p).  Every lane of a warp takes every pass, so
  // the whole warp meets the shuffles; rows past R (or DK) add nothing.
  constexpr int VN = Vec<TIn>::N;
  auto pow2 = [](int x) { return x >= 1 && x <= 32 && (x & (x - 1)) == 0; };
  const int cpr_d = DV / VN, cpr_u = R / VN;  // 16-byte chunks per row
  if (pow2(cpr_d)) {
    const int sub = lane / cpr_d, ch = lane % cpr_d, rpi = 32 / cpr_d;
    float mv[VN];
#pragma unroll
    for (int e = 0; e < VN; ++e) mv[e] = s_m[ch * VN + e];
    for (int r0 = warp * rpi; r0 < R; r0 += kDecWarps * rpi) {
      const int r = r0 + sub;
      float acc = 0.f;
      if (r < R) {
        float u[VN];
        Vec<TIn>::load(s_ud + (size_t)r * DV + ch * VN, u);
#pragma unroll
        for (int e = 0; e < VN; ++e) acc = fmaf(u[e], mv[e], acc);
      }
      for (int k = 1; k < cpr_d; k <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, k);
      if (ch == 0 && r < R) s_h[r] = acc;
    }
  } else {
    for (int base = 0; base < R; base += kDecThreads / 4) {
      const int r = base + (tid >> 2), q4 = tid & 3;
      float acc = 0.f;
      if (r < R) {  // a contiguous quarter of the row
        const int i0 = q4 * (DV / 4), i1 = i0 + DV / 4;
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
        if ((DV / 4) % VN == 0) {
          for (int i = i0; i < i1; i += VN) {
            float u[VN];
            Vec<TIn>::load(s_ud + (size_t)r * DV + i, u);
#pragma unroll
            for (int e = 0; e < VN; ++e) a4[e & 3] = fmaf(u[e], s_m[i + e], a4[e & 3]);
          }
        } else {
          for (int i = i0; i < i1; ++i) a4[0] = fmaf(ldf(s_ud, r * DV + i), s_m[i], a4[0]);
        }
        acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (q4 == 0 && r < R) s_h[r] = acc;
    }
  }
  __syncthreads();
  // b = sigmoid(b_x + p), b k
  auto gate_j = [&](int j, float p) {
    const float bj = 1.0f / (1.0f + __expf(-(s_bx[j] + p)));
    s_kp[j] = bj * s_k[j];
  };
  if (R % VN == 0 && pow2(cpr_u)) {
    const int sub = lane / cpr_u, ch = lane % cpr_u, rpi = 32 / cpr_u;
    float hv[VN];
#pragma unroll
    for (int e = 0; e < VN; ++e) hv[e] = s_h[ch * VN + e];
    for (int j0 = warp * rpi; j0 < DK; j0 += kDecWarps * rpi) {
      const int j = j0 + sub;
      float acc = 0.f;
      if (j < DK) {
        float u[VN];
        Vec<TIn>::load(s_uu + (size_t)j * R + ch * VN, u);
#pragma unroll
        for (int e = 0; e < VN; ++e) acc = fmaf(u[e], hv[e], acc);
      }
      for (int k = 1; k < cpr_u; k <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, k);
      if (ch == 0 && j < DK) gate_j(j, acc);
    }
  } else {
    for (int j = tid; j < DK; j += kDecThreads) {
      float p4[4] = {0.f, 0.f, 0.f, 0.f};
      if (R % VN == 0) {
        for (int r = 0; r < R; r += VN) {
          float u[VN];
          Vec<TIn>::load(s_uu + (size_t)j * R + r, u);
#pragma unroll
          for (int e = 0; e < VN; ++e) p4[e & 3] = fmaf(u[e], s_h[r + e], p4[e & 3]);
        }
      } else {
        for (int r = 0; r < R; ++r) p4[0] = fmaf(ldf(s_uu, j * R + r), s_h[r], p4[0]);
      }
      gate_j(j, (p4[0] + p4[1]) + (p4[2] + p4[3]));
    }
  }
  __syncthreads();

  // this lane's columns of the key-side vectors
  float qj[NJ], kj[NJ], alj[NJ], kpj[NJ];
#pragma unroll
  for (int c = 0; c < NJ; ++c) {
    const int j = lane + 32 * c;
    const bool in = j < DK;
    qj[c] = in ? s_q[j] : 0.f;
    kj[c] = in ? s_k[j] : 0.f;
    alj[c] = in ? s_al[j] : 0.f;
    kpj[c] = in ? s_kp[j] : 0.f;
  }
  // the key that reads the state and the one the erase writes along:
  // e = S' k, S -= e (b k)^T; the other erase form: e = S' (b k), S -= e k^T
  float erj[NJ], ewj[NJ];
#pragma unroll
  for (int c = 0; c < NJ; ++c) {
    erj[c] = a.erase ? kpj[c] : kj[c];
    ewj[c] = a.erase ? kj[c] : kpj[c];
  }
  const float invL = 1.0f / (float)a.L;
  if (__syncthreads_or(!mwait(&s_bar[1], a.wait_cycles))) {  // the state rows
    give_up();
    return;
  }
  // warp w takes batches of RW consecutive local rows (w RW, then
  // w RW + 4 RW, ...); the batch's 2 RW partial sums (S q and S' k of each
  // row) are reduced together, lane i ending with sum i % (2 RW); lane r
  // writes the per-row scalars of the batch's row r
  constexpr int RW = NJ > 4 ? 4 : 8;
  for (int rl0 = warp * RW; rl0 < nrow; rl0 += kDecWarps * RW) {
    float red[2 * RW];
    float sv[RW][NJ];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int rl = rl0 + r;
      float ov = 0.f, ev = 0.f;
#pragma unroll
      for (int c = 0; c < NJ; ++c) {
        const int j = lane + 32 * c;
        float x = (rl < nrow && j < DK) ? s_S[(size_t)rl * DK + j] : 0.f;
        ov = fmaf(x, qj[c], ov);
        x *= alj[c];  // S' = S Diag(exp g)
        ev = fmaf(x, erj[c], ev);
        sv[r][c] = x;
      }
      red[r] = ov;
      red[RW + r] = ev;
    }
    const float tot = reduce_scatter<2 * RW>(red, lane);
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int rl = rl0 + r;
      const float ev = __shfl_sync(0xffffffffu, tot, RW + r);
      if (rl < nrow) {  // (warp-uniform)
        const int row = rlo + rl;
        const float wv = w * s_v[row];
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
          const int j = lane + 32 * c;
          if (j < DK) S[(size_t)row * DK + j] = fmaf(-ev, ewj[c], fmaf(wv, kj[c], sv[r][c]));
        }
        if (lane == r) {  // tot is S q of row r here
          stf(o, row, tot);
          const float os = s_os[rl] + tot;
          if (chunk_end) {
            m[row] = os * invL;
            osum[row] = 0.f;
          } else {
            osum[row] = os;
          }
        }
      }
    }
  }
}

template <typename TIn, int NJ>
cudaError_t launch_nj(const DecArgs& a, size_t smem, cudaStream_t st) {
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        decode_kernel<TIn, NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * a.H) * kSplit);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<TIn, NJ>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_typed(const DecArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)(5 * a.DK + 2 * a.DV + (a.R > 0 ? a.R : 1)) * 4 +
                      16 + (size_t)a.R * (a.DK + a.DV) * sizeof(TIn) +
                      (size_t)(4 * a.DK + a.DV) * sizeof(TIn) + (size_t)a.DV * 4 +
                      (size_t)(a.DV / kSplit) * (a.DK + 1) * 4;
  if ((long long)a.B * a.H * kSplit > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (a.DK <= 64) return launch_nj<TIn, 2>(a, smem, st);
  if (a.DK <= 128) return launch_nj<TIn, 4>(a, smem, st);
  return launch_nj<TIn, 8>(a, smem, st);
}

}  // namespace

cudaError_t launch_decode(const DecArgs& a, int dtype, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return dtype == CARVE_BF16 ? launch_typed<__nv_bfloat16>(a, st)
                             : launch_typed<float>(a, st);
}

}  // namespace carve
