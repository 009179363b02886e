// tc_common.cuh -- small device helpers shared by the tensor-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "carve_internal.cuh"
#include "sm100_ptx.cuh"

namespace carve {
namespace tc {

__device__ __forceinline__ float ldbf(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
__device__ __forceinline__ void stbf(uint8_t* p, float x) {
  *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Logistic function with one MUFU op: sigma(x) = 0.5 tanh(x / 2) + 0.5
// (tanh.approx.f32, max error about 2^-11 -- below the bf16 rounding of the
// operands it scales; sigma(-inf) = 0, sigma(+inf) = 1 exactly).
__device__ __forceinline__ float sigm(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(0.5f * x));
  return fmaf(0.5f, y, 0.5f);
}
__device__ __forceinline__ void bar_named(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Arrive on named barrier `id` (n threads in all) without waiting: the
// producer side of a hand-off whose consumers bar_named(id, n).
__device__ __forceinline__ void bar_arrive_named(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// 8 fp32 values -> one 16-byte chunk of bf16 at `p`.
__device__ __forceinline__ void st_chunk(uint8_t* p, const float* x) {
  uint4 u;
  u.x = pack2(x[0], x[1]);
  u.y = pack2(x[2], x[3]);
  u.z = pack2(x[4], x[5]);
  u.w = pack2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// 8 fp32 values -> one 16-byte chunk of fp16 at `p`.
__device__ __forceinline__ void st_chunk_h(uint8_t* p, const float* x) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 hv = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  *reinterpret_cast<uint4*>(p) = u;
}
// 16-byte chunk of fp16 -> 8 fp32 values.
__device__ __forceinline__ void ld_chunk_h(const uint8_t* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* hv = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(hv[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// 16-byte chunk of bf16 -> 8 fp32 values.
__device__ __forceinline__ void ld_chunk(const uint8_t* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Element-wise transform of one block of 64 tokens x 128 key channels (CARVE
// summaries, gist.science, section 2.3: decay on the key axis; section 2.1:
// the content gate b = sigmoid(b_x + U_b m_c)); with dscale > 0 the g tile
// holds raw decay logits a and the log-decay is -dscale softplus(a); token
// rows at or past `nvalid` (the block's length) get log-decay 0:
//   Gamma_t = exp(sum_{u <= t} g_u)   K~ = K Gamma    Q~_t = Q_t Gamma_{t-1}
//   K^ = K / Gamma                    kap^ = b K^     gamma = Gamma_63
// All tiles are 128-byte swizzled 64-column blocks.  `x` holds [K; Q]
// (128 rows per column block; rewritten in place to [K~; Q~]), `graw` raw g
// and `bsm` the gate b itself in fp16 (b lies in (0, 1), where fp16 keeps
// 11 significant bits; 64 rows per column block; formed by other
// warps, which arrive on named barrier `bar_b` of `n_b` threads once it is
// written: the token loop waits there), `kh`, `kp` receive K^ and kap^ (64
// rows per column block, blocks `khs` bytes apart), `s_gam` gamma.  `red`
// is NW * 64 floats of scratch.  Called by NW warps: half of them per column block;
// thread (chunk of 8 channels, group of TPT = 128 / (4 NW) consecutive
// tokens) touches one 16-byte chunk per row, the 8 threads of a
// quarter-warp the 8 chunks of one row (conflict-free under the swizzle).
// The log-decay prefix over the token groups is a shuffle scan inside each
// warp plus the totals of the preceding warps (named barriers bar_id,
// bar_id + 1 for the two column blocks).
// QKN: q and k are first divided by their per-token L2 norms (sums of
// squares over each thread's 8 channels, reduced over the 8 lanes of a
// token and exchanged between the two column blocks through `nrm`, 1 KB,
// across named barrier bar_n of the NW warps); the inverse norms go to
// qn_out as fp16 pairs [t][k, q] (zero rows get 0).
template <int NW, bool ACT = false, bool QKN = false>
__device__ __forceinline__ void transform_block(uint8_t* x, uint8_t* kh,
                                                uint8_t* kp,
                                                const uint8_t* graw,
                                                const uint8_t* bsm,
                                                float* s_gam, float* red,
                                                int bar_id, uint32_t khs,
                                                int bar_b, int n_b,
                                                float dscale, int nvalid,
                                                float* nrm = nullptr,
                                                __half* qn_out = nullptr,
                                                int bar_n = 0) {
  constexpr int WPB = NW / 2;         // warps per column block
  constexpr int TPT = 64 / (4 * WPB); // tokens per thread
  constexpr int NG = 64 / TPT;        // token groups
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = warp / WPB, wq = warp % WPB, ch = lane & 7, t4 = lane >> 3;
  const int tg = wq * 4 + t4;        // tokens TPT tg .. TPT tg + TPT - 1
  const int j0 = blk * 64 + ch * 8;  // channels j0 .. j0 + 7
  auto off64 = [&](int t) {
    return (uint32_t)(blk * 8192 + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  auto off128 = [&](int t) {
    return (uint32_t)(blk * 16384 + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  auto offk = [&](int t) {
    return (uint32_t)(blk * khs + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  float ink[TPT], inq[TPT];
#pragma unroll
  for (int i = 0; i < TPT; ++i) ink[i] = inq[i] = 1.f;
  if constexpr (QKN) {
    float sk[TPT], sq[TPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      const int t = TPT * tg + i;
      float kv[8], qv[8];
      ld_chunk(x + off128(t), kv);
      ld_chunk(x + off128(64 + t), qv);
      sk[i] = sq[i] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sk[i] = fmaf(kv[e], kv[e], sk[i]);
        sq[i] = fmaf(qv[e], qv[e], sq[i]);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
        sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], o);
      }
      if (ch == 0) {
        nrm[(blk * 64 + t) * 2] = sk[i];
        nrm[(blk * 64 + t) * 2 + 1] = sq[i];
      }
    }
    bar_named(bar_n, NW * 32);
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      const int t = TPT * tg + i;
      const float tk = nrm[t * 2] + nrm[(64 + t) * 2];
      const float tq = nrm[t * 2 + 1] + nrm[(64 + t) * 2 + 1];
      ink[i] = tk > 0.f ? 1.0f / sqrtf(tk) : 0.f;
      inq[i] = tq > 0.f ? 1.0f / sqrtf(tq) : 0.f;
      if (blk == 0 && ch == 0) {
        qn_out[t * 2] = __float2half_rn(ink[i]);
        qn_out[t * 2 + 1] = __float2half_rn(inq[i]);
      }
    }
  }
  float gl[TPT][8];  // inclusive log-decay sums inside the token group
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    float gv[8];
    ld_chunk(graw + off64(TPT * tg + i), gv);
    // raw decay logits -> log-decay (ACT: the kernel instance for dscale >
    // 0; rows past the block's nvalid tokens: 0)
    if constexpr (ACT) decay_act8(gv, dscale, TPT * tg + i < nvalid);
#pragma unroll
    for (int e = 0; e < 8; ++e) gl[i][e] = (i ? gl[i - 1][e] : 0.f) + gv[e];
  }
  float ex[8];  // exclusive prefix of the token group
  float wt[8];  // running inclusive sum over the warp's groups
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float tot = gl[TPT - 1][e];
    float incl = tot;
    float v = __shfl_up_sync(0xffffffffu, incl, 8);
    if (t4 >= 1) incl += v;
    v = __shfl_up_sync(0xffffffffu, incl, 16);
    if (t4 >= 2) incl += v;
    ex[e] = incl - tot;
    wt[e] = incl;  // t4 == 3: the warp's total
  }
  if (t4 == 3) {
    *reinterpret_cast<float4*>(red + wq * 128 + j0) =
        make_float4(wt[0], wt[1], wt[2], wt[3]);
    *reinterpret_cast<float4*>(red + wq * 128 + j0 + 4) =
        make_float4(wt[4], wt[5], wt[6], wt[7]);
  }
  bar_named(bar_id + blk, WPB * 32);
  for (int w2 = 0; w2 < wq; ++w2) {
    const float4 a = *reinterpret_cast<const float4*>(red + w2 * 128 + j0);
    const float4 b = *reinterpret_cast<const float4*>(red + w2 * 128 + j0 + 4);
    ex[0] += a.x; ex[1] += a.y; ex[2] += a.z; ex[3] += a.w;
    ex[4] += b.x; ex[5] += b.y; ex[6] += b.z; ex[7] += b.w;
  }
  float gprev[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) gprev[e] = __expf(ex[e]);  // Gamma_{TPT tg - 1}
  bar_named(bar_b, n_b);  // b written
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = TPT * tg + i;
    float kv[8], qv[8], bv[8], o_kt[8], o_qt[8], o_kh[8], o_kp[8];
    ld_chunk(x + off128(t), kv);
    ld_chunk(x + off128(64 + t), qv);
    ld_chunk_h(bsm + off64(t), bv);
    if constexpr (QKN) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kv[e] *= ink[i];
        qv[e] *= inq[i];
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float gam = __expf(ex[e] + gl[i][e]);
      const float igam = __fdividef(1.0f, gam);
      o_kt[e] = kv[e] * gam;
      o_qt[e] = qv[e] * gprev[e];
      o_kh[e] = kv[e] * igam;
      o_kp[e] = bv[e] * o_kh[e];
      gprev[e] = gam;
    }
    st_chunk(x + off128(t), o_kt);
    st_chunk(x + off128(64 + t), o_qt);
    st_chunk(kh + offk(t), o_kh);
    st_chunk(kp + offk(t), o_kp);
  }
  if (tg == NG - 1) {  // gamma = Gamma_63
    *reinterpret_cast<float4*>(s_gam + j0) =
        make_float4(gprev[0], gprev[1], gprev[2], gprev[3]);
    *reinterpret_cast<float4*>(s_gam + j0 + 4) =
        make_float4(gprev[4], gprev[5], gprev[6], gprev[7]);
  }
}

// The key side of transform_block (Gamma, K~, Q~, K^, gamma), without the
// gate: kap^ = b K^ follows from kappa_block once p is known.  Run by warps
// wbase .. wbase + NW - 1.  With khs = 8192, K^ may overwrite the raw g
// tile in place (kh == graw): each thread reads all its g chunks before it
// writes K^ to the same offsets, and no other thread touches them.
template <int NW, bool ACT = false>
__device__ __forceinline__ void transform_keys(uint8_t* x, uint8_t* kh,
                                               const uint8_t* graw,
                                               float* s_gam, float* red,
                                               int bar_id, uint32_t khs,
                                               int wbase, float dscale,
                                               int nvalid, float* nrm) {
  constexpr int WPB = NW / 2;         // warps per column block
  constexpr int TPT = 64 / (4 * WPB); // tokens per thread
  constexpr int NG = 64 / TPT;        // token groups
  const int warp = (threadIdx.x >> 5) - wbase, lane = threadIdx.x & 31;
  const int blk = warp / WPB, wq = warp % WPB, ch = lane & 7, t4 = lane >> 3;
  const int tg = wq * 4 + t4;        // tokens TPT tg .. TPT tg + TPT - 1
  const int j0 = blk * 64 + ch * 8;  // channels j0 .. j0 + 7
  auto off64 = [&](int t) {
    return (uint32_t)(blk * 8192 + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  auto off128 = [&](int t) {
    return (uint32_t)(blk * 16384 + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  auto offk = [&](int t) {
    return (uint32_t)(blk * khs + t * 128 + ((ch ^ (t & 7)) << 4));
  };
  // fused q / k normalisation (nrm != nullptr): per-token inverse norms
  // over the 128 channels.  Each thread sums the squares of its 8 channels
  // of its TPT tokens, the 8 lanes of a token reduce by shuffles, and the
  // two column blocks' warps exchange their halves through nrm
  // ([2 blocks][64 tokens][k, q] floats, 1 KB; it may alias `red`, which
  // the scan below reuses after a second barrier) across named barrier
  // bar_id + 4 of the NW warps.  Zero rows (padding) get 0, not inf.
  float ink[TPT], inq[TPT];
#pragma unroll
  for (int i = 0; i < TPT; ++i) ink[i] = inq[i] = 1.f;
  if (nrm) {
    float sk[TPT], sq[TPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      const int t = TPT * tg + i;
      float kv[8], qv[8];
      ld_chunk(x + off128(t), kv);
      ld_chunk(x + off128(64 + t), qv);
      sk[i] = sq[i] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sk[i] = fmaf(kv[e], kv[e], sk[i]);
        sq[i] = fmaf(qv[e], qv[e], sq[i]);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
        sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], o);
      }
      if (ch == 0) {
        nrm[(blk * 64 + t) * 2] = sk[i];
        nrm[(blk * 64 + t) * 2 + 1] = sq[i];
      }
    }
    bar_named(bar_id + 4, NW * 32);
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
      const int t = TPT * tg + i;
      const float tk = nrm[t * 2] + nrm[(64 + t) * 2];
      const float tq = nrm[t * 2 + 1] + nrm[(64 + t) * 2 + 1];
      ink[i] = tk > 0.f ? 1.0f / sqrtf(tk) : 0.f;
      inq[i] = tq > 0.f ? 1.0f / sqrtf(tq) : 0.f;
    }
    bar_named(bar_id + 4, NW * 32);  // nrm may be the scan buffer `red`
  }
  float gl[TPT][8];  // inclusive log-decay sums inside the token group
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    float gv[8];
    ld_chunk(graw + off64(TPT * tg + i), gv);
    // raw decay logits -> log-decay (ACT: the kernel instance for dscale >
    // 0; rows past the block's nvalid tokens: 0)
    if constexpr (ACT) decay_act8(gv, dscale, TPT * tg + i < nvalid);
#pragma unroll
    for (int e = 0; e < 8; ++e) gl[i][e] = (i ? gl[i - 1][e] : 0.f) + gv[e];
  }
  float ex[8];  // exclusive prefix of the token group
  float wt[8];  // running inclusive sum over the warp's groups
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float tot = gl[TPT - 1][e];
    float incl = tot;
    float v = __shfl_up_sync(0xffffffffu, incl, 8);
    if (t4 >= 1) incl += v;
    v = __shfl_up_sync(0xffffffffu, incl, 16);
    if (t4 >= 2) incl += v;
    ex[e] = incl - tot;
    wt[e] = incl;  // t4 == 3: the warp's total
  }
  if (t4 == 3) {
    *reinterpret_cast<float4*>(red + wq * 128 + j0) =
        make_float4(wt[0], wt[1], wt[2], wt[3]);
    *reinterpret_cast<float4*>(red + wq * 128 + j0 + 4) =
        make_float4(wt[4], wt[5], wt[6], wt[7]);
  }
  bar_named(bar_id + blk, WPB * 32);
  for (int w2 = 0; w2 < wq; ++w2) {
    const float4 a = *reinterpret_cast<const float4*>(red + w2 * 128 + j0);
    const float4 b = *reinterpret_cast<const float4*>(red + w2 * 128 + j0 + 4);
    ex[0] += a.x; ex[1] += a.y; ex[2] += a.z; ex[3] += a.w;
    ex[4] += b.x; ex[5] += b.y; ex[6] += b.z; ex[7] += b.w;
  }
  float gprev[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) gprev[e] = __expf(ex[e]);  // Gamma_{TPT tg - 1}
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = TPT * tg + i;
    float kv[8], qv[8], o_kt[8], o_qt[8], o_kh[8];
    ld_chunk(x + off128(t), kv);
    ld_chunk(x + off128(64 + t), qv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      kv[e] *= ink[i];
      qv[e] *= inq[i];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float gam = __expf(ex[e] + gl[i][e]);
      const float igam = __fdividef(1.0f, gam);
      o_kt[e] = kv[e] * gam;
      o_qt[e] = qv[e] * gprev[e];
      o_kh[e] = kv[e] * igam;
      gprev[e] = gam;
    }
    st_chunk(x + off128(t), o_kt);
    st_chunk(x + off128(64 + t), o_qt);
    st_chunk(kh + offk(t), o_kh);
  }
  if (tg == NG - 1) {  // gamma = Gamma_63
    *reinterpret_cast<float4*>(s_gam + j0) =
        make_float4(gprev[0], gprev[1], gprev[2], gprev[3]);
    *reinterpret_cast<float4*>(s_gam + j0 + 4) =
        make_float4(gprev[4], gprev[5], gprev[6], gprev[7]);
  }
}

// kap^ = sigmoid(b_x + p) K^ for one block, with K^ already in its operand
// slot: `kh` holds K^ in rows 0..63 of each 128-row column block (blocks
// `khs` bytes apart) and kap^ goes to rows 64..127 of the same blocks.
// Thread t_id of n_thr takes 16-byte chunks t_id, t_id + n_thr, ... of the
// first `nrows` token rows of the 64 x 128 tile (the caller keeps the rows
// past them zero); the 8 threads of a quarter-warp take the 8 chunks of one
// row (conflict-free under the swizzle).
__device__ __forceinline__ void kappa_in_place(uint8_t* kh, const uint8_t* braw,
                                               const float* s_p, uint32_t khs,
                                               int t_id, int n_thr, int nrows = 64) {
  for (int c = t_id; c < 16 * nrows; c += n_thr) {
    const int t = c >> 4, blk = (c >> 3) & 1, ch = c & 7;
    const uint32_t sw = (uint32_t)(t * 128 + ((ch ^ (t & 7)) << 4));
    float kv[8], bv[8], o[8];
    ld_chunk(kh + blk * khs + sw, kv);
    ld_chunk(braw + blk * 8192 + sw, bv);
    const float4 p0 = *reinterpret_cast<const float4*>(s_p + blk * 64 + ch * 8);
    const float4 p1 = *reinterpret_cast<const float4*>(s_p + blk * 64 + ch * 8 + 4);
    const float pj[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = sigm(bv[e] + pj[e]) * kv[e];
    st_chunk(kh + blk * khs + 8192 + sw, o);
  }
}

// Sum over the 32 lanes of a warp of v[i] (i < 32): lane l ends with the
// sum of index l in v[0] (31 shuffles).
__device__ __forceinline__ float warp_reduce_scatter32(float* v, int lane) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = up ? v[i] : v[i + k];
      const float keep = up ? v[i + k] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  return v[0];
}

// kap^ = sigmoid(b_x + p) K^ for one block (the gate half of
// transform_block), from the bf16 K^ at `kh_src` (64-row column blocks
// 8192 B apart); K^ is copied to `kh` and kap^ written to `kp` (column blocks
// `khs` apart).  Thread t_id of n_thr takes 16-byte chunks t_id,
// t_id + n_thr, ... of the 64 x 128 tile; the 8 threads of a quarter-warp
// take the 8 chunks of one row (conflict-free under the swizzle).
__device__ __forceinline__ void kappa_block(const uint8_t* kh_src, uint8_t* kh,
                                            uint8_t* kp, const uint8_t* braw,
                                            const float* s_p, uint32_t khs,
                                            int t_id, int n_thr) {
  for (int c = t_id; c < 1024; c += n_thr) {
    const int t = c >> 4, blk = (c >> 3) & 1, ch = c & 7;
    const uint32_t sw = (uint32_t)(t * 128 + ((ch ^ (t & 7)) << 4));
    const uint4 kraw = *reinterpret_cast<const uint4*>(kh_src + blk * 8192 + sw);
    float kv[8], bv[8], o[8];
    ld_chunk(kh_src + blk * 8192 + sw, kv);
    ld_chunk(braw + blk * 8192 + sw, bv);
    const float4 p0 = *reinterpret_cast<const float4*>(s_p + blk * 64 + ch * 8);
    const float4 p1 = *reinterpret_cast<const float4*>(s_p + blk * 64 + ch * 8 + 4);
    const float pj[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = sigm(bv[e] + pj[e]) * kv[e];
    *reinterpret_cast<uint4*>(kh + blk * khs + sw) = kraw;
    st_chunk(kp + blk * khs + sw, o);
  }
}

// Bounded wait on an mbarrier phase: gives up after `spin` cycles
// (kSpinCycles unless a test lowers it).  On expiry: record
// CARVE_ERR_TIMEOUT and the wait site in the workspace header, raise the CTA
// abort flag and return (the caller keeps its barrier sequence; every later
// wait returns at once, and the block loop exits at its next block-wide
// check of the flag, which every thread takes together).
// Returns whether the phase completed.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity,
                                         uint32_t where,
                                         volatile uint32_t* abort_flag,
                                         WsHeader* hdr, long long spin) {
  const long long t0 = clock64();
  while (!*abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > spin) {
      atomicExch(&hdr->status, (uint32_t)CARVE_ERR_TIMEOUT);
      hdr->where = where;
      *abort_flag = 1;
    }
  }
  return false;
}

// Bounded wait that ignores the abort flag: before a CTA that aborted
// exits, its copies and MMAs still in flight are given up to kSpinCycles
// (~1 s) each to land (their shared and tensor memory must outlive them);
// the limit is never lowered.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kSpinCycles) return;
}

}  // namespace tc
}  // namespace carve

namespace carve {
namespace tc {

// Index of element (r, c) of a 64 x 64 fp32 matrix stored row-major with the
// float4 groups of each row XOR-permuted by (r % 8): rows 256 B apart then
// fall in different banks, and float4 groups stay contiguous.
__device__ __forceinline__ int fsw(int r, int c) {
  return r * 64 + (c ^ ((r & 7) << 2));
}

// Index of element (R, c) of the four diagonal 16 x 16 blocks of a 64 x 64
// matrix stored compactly (row R in [0, 64), column c in [0, 16) within the
// block); float4 groups XOR-permuted so that the rows of a warp's fragment
// loads hit distinct banks.
__device__ __forceinline__ int csw(int R, int c) {
  return R * 16 + (c ^ (((R >> 1) & 3) << 2));
}
template <bool CPT>
__device__ __forceinline__ int mx(int R, int C) {
  return CPT ? csw(R, C & 15) : fsw(R, C);
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
// c (16 x 8 fp32 fragment) += a (16 x 8 tf32) * b (8 x 8 tf32), warp-wide.
__device__ __forceinline__ void mma_tf32(float* c, const uint32_t* a,
                                         const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Warp-level 16 x 16 tile product on shared-memory fp32 matrices:
// acc (two 16 x 8 fragments) += X[xr .., xc .. xc + 16 NB) * Y[yr .., yc .. yc + 16).
// XC / YC select the compact (csw) or full (fsw) layout.  All fragments are
// loaded first and every 16-wide K block accumulates into its own registers,
// so the dependent chain is one load, one convert and two MMAs deep.
template <bool XC, bool YC, int NB>
__device__ __forceinline__ void tile_mac(float* acc, const float* X, int xr,
                                         int xc, const float* Y, int yr,
                                         int yc) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float xa[NB][2][4], yb[NB][2][2][2];
#pragma unroll
  for (int kb = 0; kb < NB; ++kb)
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int c = xc + 16 * kb + 8 * kk + t;
      xa[kb][kk][0] = X[mx<XC>(xr + g, c)];
      xa[kb][kk][1] = X[mx<XC>(xr + g + 8, c)];
      xa[kb][kk][2] = X[mx<XC>(xr + g, c + 4)];
      xa[kb][kk][3] = X[mx<XC>(xr + g + 8, c + 4)];
#pragma unroll
      for (int nn = 0; nn < 2; ++nn) {
        const int r = yr + 16 * kb + 8 * kk + t;
        yb[kb][kk][nn][0] = Y[mx<YC>(r, yc + 8 * nn + g)];
        yb[kb][kk][nn][1] = Y[mx<YC>(r + 4, yc + 8 * nn + g)];
      }
    }
  float part[NB][8];
#pragma unroll
  for (int kb = 0; kb < NB; ++kb) {
#pragma unroll
    for (int i = 0; i < 8; ++i) part[kb][i] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = to_tf32(xa[kb][kk][i]);
#pragma unroll
      for (int nn = 0; nn < 2; ++nn) {
        uint32_t b[2] = {to_tf32(yb[kb][kk][nn][0]), to_tf32(yb[kb][kk][nn][1])};
        mma_tf32(part[kb] + 4 * nn, a, b);
      }
    }
  }
#pragma unroll
  for (int kb = 0; kb < NB; ++kb)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += part[kb][i];
}
// acc (two 16 x 8 fragments) <- / -> a 16 x 16 tile of Z at (zr, zc), scaled.
template <bool ZC>
__device__ __forceinline__ void tile_ld(float* acc, const float* Z, int zr,
                                        int zc) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nn = 0; nn < 2; ++nn) {
    acc[4 * nn + 0] = Z[mx<ZC>(zr + g, zc + 8 * nn + 2 * t)];
    acc[4 * nn + 1] = Z[mx<ZC>(zr + g, zc + 8 * nn + 2 * t + 1)];
    acc[4 * nn + 2] = Z[mx<ZC>(zr + g + 8, zc + 8 * nn + 2 * t)];
    acc[4 * nn + 3] = Z[mx<ZC>(zr + g + 8, zc + 8 * nn + 2 * t + 1)];
  }
}
template <bool ZC>
__device__ __forceinline__ void tile_st(float* Z, int zr, int zc,
                                        const float* acc, float s) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nn = 0; nn < 2; ++nn) {
    Z[mx<ZC>(zr + g, zc + 8 * nn + 2 * t)] = s * acc[4 * nn + 0];
    Z[mx<ZC>(zr + g, zc + 8 * nn + 2 * t + 1)] = s * acc[4 * nn + 1];
    Z[mx<ZC>(zr + g + 8, zc + 8 * nn + 2 * t)] = s * acc[4 * nn + 2];
    Z[mx<ZC>(zr + g + 8, zc + 8 * nn + 2 * t + 1)] = s * acc[4 * nn + 3];
  }
}

// T = (I + A)^{-1} for a strictly lower 64 x 64 fp32 matrix A (layout fsw),
// by 16 x 16 blocks.  (1) Diagonal blocks by forward substitution in fp32,
// one thread per column (threads 0..63): t_i = -sum_{k<i} a_ik t_k with the
// row loaded as float4 groups and the terms before k = i - 1 summed ahead of
// t_{i-1}.  (2) Pairs of blocks merge into 32 x 32 blocks,
// T_10 = -T_11 (A_10 T_00), one warp per pair.  (3) The two 32 x 32 blocks
// merge, T_BA = -T_B (A_BA T_A), one warp per 16 x 16 output tile.  (2) and
// (3) run on the warp-level tensor cores (tf32 in, fp32 out; T is rounded to
// bf16 by its users).  Called by warps 0..3 only (128 threads, named barrier
// `bar_id`); the other warps of the CTA are free meanwhile.  T (layout fsw)
// goes to `tf`, which may be `af` (in place: each block of A is read before
// the block of T in its place is written); `ws` is >= 2048 floats of
// scratch.  With nblk < 4 the rows (and columns) past 16 nblk of A are zero,
// so T is I there and block merges reaching only those rows are skipped.
// Ends with that named barrier.
static __device__ __noinline__ void unit_lower_inverse64(const float* af, float* tf,
                                                  float* ws, int bar_id,
                                                  int nblk = 4) {
  const int tid = threadIdx.x, warp = tid >> 5;
  // zero blocks above the diagonal (6 blocks, 3 float4 per thread)
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const int e = tid + 128 * q;          // 0..383
    const int blk = e >> 6, r = (e & 63) >> 2, c4 = (e & 3) << 2;
    const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
    const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
    *reinterpret_cast<float4*>(tf + fsw(16 * bi + r, 16 * bj + c4)) =
        make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // (1) diagonal blocks (every read of A's diagonal blocks precedes the
  // barrier before the stores, so `tf` may be `af`)
  const int o = 16 * (tid >> 4), j = tid & 15;
  float t[16];
  if (tid < 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = 0.f;
      if (i > 0) {
        float a[16];
#pragma unroll
        for (int g = 0; g < (i + 3) / 4; ++g) {
          const float4 v = *reinterpret_cast<const float4*>(af + fsw(o + i, o + 4 * g));
          a[4 * g] = v.x; a[4 * g + 1] = v.y; a[4 * g + 2] = v.z; a[4 * g + 3] = v.w;
        }
        float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < i - 1; ++k) p[k & 3] = fmaf(a[k], t[k], p[k & 3]);
        acc = fmaf(a[i - 1], t[i - 1], (p[0] + p[1]) + (p[2] + p[3]));
      }
      t[i] = i < j ? 0.f : (i == j ? 1.f : -acc);
    }
  }
  bar_named(bar_id, 128);
  if (tid < 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) tf[fsw(o + i, o + j)] = t[i];
  }
  bar_named(bar_id, 128);
  // rows past 16 nblk are zero (padding tokens): T is I there and the
  // merges that only reach those rows are skipped (nblk is uniform)
  if (nblk <= 1) return;
  // (2) T_10 = -T_11 (A_10 T_00) for the block pairs (0, 1) and (2, 3)
  if (warp < 2) {
    const int o0 = 32 * warp, o1 = o0 + 16;
    float acc[8], acc2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = acc2[i] = 0.f;
    tile_mac<false, false, 1>(acc, af, o1, o0, tf, o0, o0);
    __syncwarp();  // A_10 read by every lane before its place takes A_10 T_00
    tile_st<false>(tf, o1, o0, acc, 1.f);
    __syncwarp();
    tile_mac<false, false, 1>(acc2, tf, o1, o1, tf, o1, o0);
    __syncwarp();
    tile_st<false>(tf, o1, o0, acc2, -1.f);
  }
  bar_named(bar_id, 128);
  if (nblk <= 2) return;
  // (3) T_BA = -T_B (A_BA T_A): output tile (I, J), I = 2, 3, J = 0, 1
  const int I = 2 + (warp >> 1), J = warp & 1;
  {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (J == 0)
      tile_mac<false, false, 2>(acc, af, 16 * I, 0, tf, 0, 0);
    else
      tile_mac<false, false, 1>(acc, af, 16 * I, 16, tf, 16, 16);
    tile_st<false>(ws, 16 * (I - 2), 16 * J, acc, 1.f);
  }
  bar_named(bar_id, 128);
  {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (I == 2)
      tile_mac<false, false, 1>(acc, tf, 32, 32, ws, 0, 16 * J);
    else
      tile_mac<false, false, 2>(acc, tf, 48, 32, ws, 0, 16 * J);
    tile_st<false>(tf, 16 * I, 16 * J, acc, -1.f);
  }
  bar_named(bar_id, 128);
}

}  // namespace tc
}  // namespace carve
