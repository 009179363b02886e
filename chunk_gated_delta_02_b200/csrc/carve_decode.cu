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
// memory by asynchronous copies (requested first, and holding no register
// while in flight), then its warps take a row each in turn, reduce S q and
// S' k with butterfly shuffles, and write the new row back.  The gate of every CTA reads all of m_c, which a
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

  // the head's U_b factors -> shared memory by asynchronous 16-byte copies
  // (R * DV and DK * R elements fill whole 16-byte chunks: DK, DV are
  // multiples of 16), in flight with the state rows; then the token's
  // vectors and m_c
  if (R > 0) {
    const uint8_t* udg = reinterpret_cast<const uint8_t*>(
        static_cast<const TIn*>(a.u_down) + (size_t)h * R * DV);
    const uint8_t* uug = reinterpret_cast<const uint8_t*>(
        static_cast<const TIn*>(a.u_up) + (size_t)h * DK * R);
    const int nd = R * DV * (int)sizeof(TIn) / 16, nu = DK * R * (int)sizeof(TIn) / 16;
    for (int i = tid; i < nd; i += kDecThreads)
      ptx::cp_async16(reinterpret_cast<uint8_t*>(s_ud) + 16 * i, udg + 16 * i);
    for (int i = tid; i < nu; i += kDecThreads)
      ptx::cp_async16(reinterpret_cast<uint8_t*>(s_uu) + 16 * i, uug + 16 * i);
  }
  {  // every 16-byte chunk of the vectors and of m_c in one batch of copies
    const int cv = DK * (int)sizeof(TIn) / 16, cw = DV * (int)sizeof(TIn) / 16;
    const int nc = 4 * cv + cw + DV / 4;
    for (int i = tid; i < nc; i += kDecThreads) {
      const int which = i < 4 * cv ? i / cv : (i < 4 * cv + cw ? 4 : 5);
      const int ci = which < 4 ? i - which * cv : (which == 4 ? i - 4 * cv : i - 4 * cv - cw);
      const void* src = which == 0 ? (const void*)q : which == 1 ? (const void*)k
                      : which == 2 ? (const void*)g : which == 3 ? (const void*)bx
                      : which == 4 ? (const void*)v : (const void*)m;
      uint8_t* dst = which < 5 ? reinterpret_cast<uint8_t*>(s_raw + which * DK)
                               : reinterpret_cast<uint8_t*>(s_mraw);
      ptx::cp_async16(dst + 16 * ci, static_cast<const uint8_t*>(src) + 16 * ci);
    }
    ptx::cp_async_commit();
  }
  {  // then the state rows and their output sums (the newest group): they
     // land while the gate is formed
    const float* Sg = S + (size_t)rlo * DK;
    const int ns = nrow * DK / 4;
    for (int i = tid; i < ns; i += kDecThreads) ptx::cp_async16(s_S + 4 * i, Sg + 4 * i);
    for (int i = tid; i < nrow / 4; i += kDecThreads)
      ptx::cp_async16(s_os + 4 * i, osum + rlo + 4 * i);
    ptx::cp_async_commit();
  }
  ptx::cp_async_wait_but_newest();
  __syncthreads();
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
  __syncthreads();
  // every CTA of the pair has m_c: a chunk's last token may now rewrite it
  // (only that token writes m, and chunk_end is the same for the whole
  // cluster, so the other tokens skip the barrier)
  if (chunk_end) ptx::cluster_sync();
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
  // h = U_down m_c: four threads per rank, each over a quarter of the
  // values (every thread takes every pass, so that the whole warp meets the
  // shuffles; ranks past R add nothing)
  for (int base = 0; base < R; base += kDecThreads / 4) {
    const int r = base + (tid >> 2), q4 = tid & 3;
    float acc = 0.f;
    if (r < R) {  // a contiguous quarter of the row, 16-byte vectors
      constexpr int VN = Vec<TIn>::N;
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
  __syncthreads();
  // p = U_up h (a thread per key channel, its row of U_up read as 16-byte
  // vectors when the row fills whole ones), b = sigmoid(b_x + p), b k
  constexpr int VN = Vec<TIn>::N;
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
    const float p = (p4[0] + p4[1]) + (p4[2] + p4[3]);
    const float bj = 1.0f / (1.0f + expf(-(s_bx[j] + p)));
    s_kp[j] = bj * s_k[j];
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
  ptx::cp_async_wait_all();  // this thread's state copies
  __syncthreads();           // and everyone's
  // warp w takes batches of RW consecutive local rows (w RW, then
  // w RW + 4 RW, ...), a batch unrolled so that its rows' reductions
  // overlap; lane r writes the per-row scalars of the batch's row r
  constexpr int RW = NJ > 4 ? 4 : 8;
  for (int rl0 = warp * RW; rl0 < nrow; rl0 += kDecWarps * RW) {
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int rl = rl0 + r;
      if (rl < nrow) {  // (warp-uniform)
        const int row = rlo + rl;
        float sv[NJ];
        float ov = 0.f, ev = 0.f;
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
          const int j = lane + 32 * c;
          sv[c] = j < DK ? s_S[(size_t)rl * DK + j] : 0.f;
          ov = fmaf(sv[c], qj[c], ov);
          sv[c] *= alj[c];  // S' = S Diag(exp g)
          ev = fmaf(sv[c], erj[c], ev);
        }
        ov = allsum(ov);
        ev = allsum(ev);
        const float wv = w * s_v[row];
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
          const int j = lane + 32 * c;
          if (j < DK) S[(size_t)row * DK + j] = fmaf(-ev, ewj[c], fmaf(wv, kj[c], sv[c]));
        }
        if (lane == r) {
          stf(o, row, ov);
          const float os = s_os[rl] + ov;
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
