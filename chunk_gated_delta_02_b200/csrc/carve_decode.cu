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
// known, so one CTA per (sequence, head) forms those vectors and the gate,
// and its warps stream the rows: a warp holds a batch of rows in registers
// (each row read as coalesced 128-byte segments), reduces S q and S' k with
// butterfly shuffles, and writes the new row back.
#include <cuda_bf16.h>

#include "carve_internal.cuh"

namespace carve {
namespace {

constexpr int kDecThreads = 512;   // 16 warps
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kRows = 8;           // value rows a warp holds at once (DK <= 128)

__device__ __forceinline__ float allsum(float x) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) x += __shfl_xor_sync(0xffffffffu, x, k);
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

// Copies n elements (a multiple of the vector width, 16-byte aligned) of
// the I/O dtype into fp32 shared memory with 16-byte loads.
template <typename TIn>
__device__ __forceinline__ void stage(float* dst, const TIn* src, int n) {
  constexpr int N = Vec<TIn>::N;
  for (int i = threadIdx.x * N; i < n; i += kDecThreads * N) {
    float x[N];
    Vec<TIn>::load(src + i, x);
#pragma unroll
    for (int e = 0; e < N; ++e) dst[i + e] = x[e];
  }
}

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
  // the head's U_b factors in the I/O dtype: U_down [R][DV], U_up [DK][R]
  TIn* s_ud = reinterpret_cast<TIn*>(
      (reinterpret_cast<uintptr_t>(s_h + (R > 0 ? R : 1)) + 15) & ~uintptr_t(15));
  TIn* s_uu = s_ud + R * DV;
  const int pair = blockIdx.x;
  const int bseq = pair / a.H, h = pair - bseq * a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* S = a.S + (size_t)pair * DV * DK;
  constexpr int RW = NJ > 4 ? kRows / 2 : kRows;  // rows per batch in registers

  // the first batch of this warp's state rows: requested before anything
  // else, so that the gate below runs while they are in flight
  float sv[RW][NJ];
  float osv = 0.f;  // lane r < RW: the running output sum of row r0 + r
  float* osum = a.osum + (size_t)pair * DV;
  auto load_rows = [&](int r0) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NJ; ++c) {
        const int j = lane + 32 * c;
        sv[r][c] = (r0 + r < DV && j < DK) ? S[(size_t)(r0 + r) * DK + j] : 0.f;
      }
    osv = (lane < RW && r0 + lane < DV) ? osum[r0 + lane] : 0.f;
  };
  load_rows(warp * RW);

  const TIn* q = static_cast<const TIn*>(a.q) + (size_t)pair * DK;
  const TIn* k = static_cast<const TIn*>(a.k) + (size_t)pair * DK;
  const TIn* g = static_cast<const TIn*>(a.g) + (size_t)pair * DK;
  const TIn* bx = static_cast<const TIn*>(a.bx) + (size_t)pair * DK;
  const TIn* v = static_cast<const TIn*>(a.v) + (size_t)pair * DV;
  float* m = a.m + (size_t)pair * DV;
  TIn* o = static_cast<TIn*>(a.o) + (size_t)pair * DV;
  const float w = ldf(static_cast<const TIn*>(a.w), pair);
  const bool chunk_end = (a.pos[bseq] + 1) % a.L == 0;

  // the token's vectors, m_c and the head's U_b factors -> shared memory
  // (16-byte loads; DK, DV and R * DV, DK * R are multiples of 8)
  stage(s_q, q, DK);
  stage(s_k, k, DK);
  stage(s_al, g, DK);
  stage(s_bx, bx, DK);
  stage(s_v, v, DV);
  for (int i = tid * 4; i < DV; i += kDecThreads * 4)
    *reinterpret_cast<float4*>(s_m + i) = *reinterpret_cast<const float4*>(m + i);
  if (R > 0) {  // raw 16-byte copies (R * DV and DK * R bytes are multiples of 16)
    const uint4* ud4 = reinterpret_cast<const uint4*>(
        static_cast<const TIn*>(a.u_down) + (size_t)h * R * DV);
    const uint4* uu4 = reinterpret_cast<const uint4*>(
        static_cast<const TIn*>(a.u_up) + (size_t)h * DK * R);
    const int nd = R * DV * (int)sizeof(TIn) / 16, nu = DK * R * (int)sizeof(TIn) / 16;
    for (int i = tid; i < nd; i += kDecThreads) reinterpret_cast<uint4*>(s_ud)[i] = ud4[i];
    for (int i = tid; i < nu; i += kDecThreads) reinterpret_cast<uint4*>(s_uu)[i] = uu4[i];
  }
  __syncthreads();
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
    s_al[j] = expf(decay_act(s_al[j], a.dscale));
  // h = U_down m_c: one warp per rank
  for (int r = warp; r < R; r += kDecWarps) {
    float acc = 0.f;
    for (int i = lane; i < DV; i += 32) acc = fmaf(ldf(s_ud, r * DV + i), s_m[i], acc);
    acc = allsum(acc);
    if (lane == 0) s_h[r] = acc;
  }
  __syncthreads();
  // p = U_up h (one warp per key channel j, lanes over the rank: rows of
  // U_up read contiguously), b = sigmoid(b_x + p), b k
  for (int j = warp; j < DK; j += kDecWarps) {
    float p = 0.f;
    for (int r = lane; r < R; r += 32) p = fmaf(ldf(s_uu, j * R + r), s_h[r], p);
    p = allsum(p);
    if (lane == 0) {
      const float bj = 1.0f / (1.0f + expf(-(s_bx[j] + p)));
      s_kp[j] = bj * s_k[j];
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
  for (int r0 = warp * RW; r0 < DV; r0 += kDecWarps * RW) {
    if (r0 != warp * RW) load_rows(r0);
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int row = r0 + r;
      float ov = 0.f, ev = 0.f;
#pragma unroll
      for (int c = 0; c < NJ; ++c) {
        ov = fmaf(sv[r][c], qj[c], ov);
        sv[r][c] *= alj[c];  // S' = S Diag(exp g)
        ev = fmaf(sv[r][c], erj[c], ev);
      }
      ov = allsum(ov);
      ev = allsum(ev);
      if (row < DV) {
        const float wv = w * s_v[row];
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
          const int j = lane + 32 * c;
          if (j < DK)
            S[(size_t)row * DK + j] = fmaf(-ev, ewj[c], fmaf(wv, kj[c], sv[r][c]));
        }
        if (lane == r) {  // spread the per-row scalars over the warp's lanes
          stf(o, row, ov);
          const float os = osv + ov;
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

template <typename TIn>
cudaError_t launch_typed(const DecArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)(5 * a.DK + 2 * a.DV + (a.R > 0 ? a.R : 1)) * 4 +
                      16 + (size_t)a.R * (a.DK + a.DV) * sizeof(TIn);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaSuccess;
    if (a.DK <= 64)
      e = cudaFuncSetAttribute(decode_kernel<TIn, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else if (a.DK <= 128)
      e = cudaFuncSetAttribute(decode_kernel<TIn, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
      e = cudaFuncSetAttribute(decode_kernel<TIn, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(a.B * a.H), block(kDecThreads);
  if (a.DK <= 64)
    decode_kernel<TIn, 2><<<grid, block, smem, st>>>(a);
  else if (a.DK <= 128)
    decode_kernel<TIn, 4><<<grid, block, smem, st>>>(a);
  else
    decode_kernel<TIn, 8><<<grid, block, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecArgs& a, int dtype, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return dtype == CARVE_BF16 ? launch_typed<__nv_bfloat16>(a, st)
                             : launch_typed<float>(a, st);
}

}  // namespace carve
