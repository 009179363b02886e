// carve_tc_bwd.cu -- tensor-core (tcgen05 / TMEM / TMA) backward of the CARVE
// recurrent core for bf16 inputs, dk = dv = 128, chunks of 64 or 128 tokens.
//
// Exact reverse mode of the chunk form (see carve_tc_fwd.cu).  One CTA
// walks the blocks of one (sequence, head) pair from last to first.  The
// gradient of the block-end state, dS (dv x dk, fp32), lives in tensor
// memory for the whole walk.  Per block the training forward left a record
// (the bf16 state operand S, E^T and T = (I + A)^{-1}, as shared-memory
// images) and the chunk's gate vector p_c; the element-wise transform and
// the Gram matrices are recomputed from the inputs.
//
// Per block, with dO = d_o + dm_{c+1} / L (the gate feedback: the next
// chunk's mean reads these outputs) and dS~ = dS Diag(gamma):
//
//   recompute  M, P_k, P_kap (strictly lower Grams)
//   dE   = -kap^ dS~^T - P_kap^T dO          dR = T^T dE
//   G2   = [dR; dO] [E; W]^T = [[-dA, dM], [-dP_kap, dP_k]]  (strictly lower)
//   dW   = K^ dS~^T + P_k^T dO + M^T dR     -> dv = w dW, dw = rowsum(dW V)
//   [dK~; dQ~]   = [dR; dO] S + G2 [-kap^; K^]
//   [-dkap^; dK^] = G2^T [K~; Q~] + [E; W] dS~
//   dS_prev = dS~ + dR^T K~ + dO^T Q~
//   dlog gamma_j = sum_v dS S_new  (S_new: the fp32 checkpoint of the block end)
//   per key channel: dq, dk, db_x, dg (reverse cumulative sum of the
//   log-Gamma gradients), dp = sum_t db_x  (the gate's logit gradient)
//
// All products are M = 128 tcgen05 MMAs, most in transposed form so that the
// 128 lanes are value rows or key channels.  Shared memory (227 KB) is
// time-shared: raw g / b_x and the bf16 dS~ share one region; the C x C
// gradient G2 reuses the Gram and T buffers once their MMAs retired.  At each
// chunk start the gate gradient (dp, dh = U_up^T dp) is recorded so that a
// second kernel forms dU_up, dU_down in fixed order.
#include <cudaTypedefs.h>

#include "carve_internal.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace carve {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kThreads = 256;
constexpr int kBlk = 64;
constexpr int kDK = 128;
constexpr int kDV = 128;
constexpr int kRMax = 32;

// shared memory map (bytes; the dynamic shared memory base is required to
// be 1024-aligned, which the kernel checks).  Tiles are 128-byte swizzled
// 64-column blocks of `rows` x 128 B, the UMMA canonical layout.
constexpr uint32_t R_X = 0;          // [K~; Q~]                        32 KB
constexpr uint32_t R_KH = 32768;     // K^                              16 KB
constexpr uint32_t R_KP = 49152;     // kap^                            16 KB
constexpr uint32_t R_ET = 65536;     // E^T (forward record)            16 KB
constexpr uint32_t R_W = 81920;      // raw v -> W = w V                16 KB
constexpr uint32_t R_RO = 98304;     // [dE -> dR ; dO]                 32 KB
constexpr uint32_t R_DSB = 131072;   // raw g, b_x | dS~ bf16           32 KB
constexpr uint32_t R_SB = 163840;    // S bf16 (record) | raw g, b_x    32 KB
constexpr uint32_t R_MP = 196608;    // [M; P_k] | G2 cols 0..63        16 KB
constexpr uint32_t R_PQ = 212992;    // P_kap    | G2 cols 64..127 (1/2) 8 KB
constexpr uint32_t R_TT = 221184;    // T (record) | G2 cols 64..127 (2/2) 8 KB
constexpr uint32_t R_SM = 229376;    // small region
constexpr uint32_t SM_P = 0;         // p_j                128 f32
constexpr uint32_t SM_DMN = 512;     // dm fed into dO     128 f32
constexpr uint32_t SM_X = 1024;      // g half sums | dlog gamma | dp   128 f32
constexpr uint32_t SM_GAM = 1536;    // gamma | dg hand-off | dh parts  128 f32
constexpr uint32_t SM_W = 2048;      // w_t                 64 f32
constexpr uint32_t SM_DW = 2304;     // dw sums | dh        64 f32
constexpr uint32_t SM_BAR = 2560;    // 8 mbarriers
constexpr uint32_t SM_TMEM = 2624;
constexpr uint32_t SM_ABORT = 2628;
constexpr uint32_t kSmemBytes = 232448;
static_assert(R_SM + 2688 <= kSmemBytes, "small region");
static_assert(R_PQ == R_MP + 16384 && R_TT == R_PQ + 8192, "G2 blocks");

// TMEM columns
constexpr uint32_t T_DS = 0;     // dS [v][j]
constexpr uint32_t T_G = 128;    // [A|M ; P_kap|P_k] [i][t]  -> [dK~^T | dQ~^T]
constexpr uint32_t T_RE = 256;   // dW^T  -> [-dkap^T | dK^T] (128 cols)
constexpr uint32_t T_DER = 320;  // dE^T -> dR^T
constexpr uint32_t T_G2 = 384;   // raw G2 [r][c]
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t ID_KK64 = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_KM64 = idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_MK64 = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_MK128 = idesc_bf16(128, 128, true, false);
constexpr uint32_t ID_MM64 = idesc_bf16(128, 64, true, true);
constexpr uint32_t ID_MM128 = idesc_bf16(128, 128, true, true);
constexpr uint32_t ID_KK64_NA = idesc_bf16_neg(128, 64, false, false, true, false);
constexpr uint32_t ID_MM64_NA = idesc_bf16_neg(128, 64, true, true, true, false);
constexpr uint32_t ID_MK128_NA = idesc_bf16_neg(128, 128, true, false, true, false);

// Sum over the 32 lanes of a warp of v[i] (i < 32): lane l ends with the
// sum of index l in v[0].  (Reduce-scatter: 31 shuffles.)
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

struct BwdTcArgs {
  BwdArgs a;
  float* gate_rec;  // [B*H][NC][DK + R]: dp | dh per chunk
};

__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const BwdTcArgs args,
                  const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_g,
                  const __grid_constant__ CUtensorMap tm_bx,
                  const __grid_constant__ CUtensorMap tm_do) {
  const BwdArgs& a = args.a;
  extern __shared__ __align__(1024) uint8_t sm[];
  float* s_p = reinterpret_cast<float*>(sm + R_SM + SM_P);
  float* s_dmn = reinterpret_cast<float*>(sm + R_SM + SM_DMN);
  float* s_x = reinterpret_cast<float*>(sm + R_SM + SM_X);
  float* s_gam = reinterpret_cast<float*>(sm + R_SM + SM_GAM);
  float* s_w = reinterpret_cast<float*>(sm + R_SM + SM_W);
  float* s_dw = reinterpret_cast<float*>(sm + R_SM + SM_DW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + R_SM + SM_BAR);
  uint64_t* bar_in = bars + 0;
  uint64_t* bar_gb = bars + 1;
  uint64_t* bar1 = bars + 2;
  uint64_t* bar3 = bars + 4;
  uint64_t* bar4 = bars + 5;
  uint64_t* bar5 = bars + 6;
  uint64_t* bar7 = bars + 7;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + R_SM + SM_TMEM);
  volatile uint32_t* s_abort =
      reinterpret_cast<volatile uint32_t*>(sm + R_SM + SM_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = warp >> 2;
  const int row = (warp & 3) * 32 + lane;
  const int pair = blockIdx.x, b = pair / a.H, h = pair - b * a.H;
  const int T = a.T, H = a.H, R = a.R, NB = a.NB, NC = a.NC;
  const int bpc = a.L / kBlk;
  const size_t SZ = (size_t)kDV * kDK;
  const __nv_bfloat16* w_in = static_cast<const __nv_bfloat16*>(a.w);
  const __nv_bfloat16* ud = static_cast<const __nv_bfloat16*>(a.u_down);
  const __nv_bfloat16* uu = static_cast<const __nv_bfloat16*>(a.u_up);
  __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(a.dq);
  __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(a.dk);
  __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(a.dv);
  __nv_bfloat16* dg = static_cast<__nv_bfloat16*>(a.dg);
  __nv_bfloat16* dbx = static_cast<__nv_bfloat16*>(a.dbx);
  __nv_bfloat16* dw = static_cast<__nv_bfloat16*>(a.dw);
  const int GR = kDK + R;  // floats per gate record and per gate input

  // layout assumption broken, or the workspace was not written by the
  // tensor-core training forward: refuse
  if ((smem_u32(sm) & 1023u) != 0 || a.hdr->magic != kWsMagicTc) {
    if (tid == 0) {
      const bool align = (smem_u32(sm) & 1023u) != 0;
      atomicExch(&a.hdr->status, (uint32_t)(align ? CARVE_ERR_UNSUPPORTED
                                                  : CARVE_ERR_WORKSPACE));
      a.hdr->where = align ? 99 : 98;
    }
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(bars + i, 1);
    *s_abort = 0;
    mbar_init_fence();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
    prefetch_tmap(&tm_bx);
    prefetch_tmap(&tm_do);
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  // U_b factors: threads < 128 hold U_up[h][tid][:], threads >= 128 hold
  // U_down[h][:][tid - 128].
  float ureg[kRMax];
#pragma unroll
  for (int r = 0; r < kRMax; ++r) {
    float x = 0.f;
    if (r < R)
      x = half == 0 ? __bfloat162float(uu[((size_t)h * kDK + tid) * R + r])
                    : __bfloat162float(ud[((size_t)h * R + r) * kDV + row]);
    ureg[r] = x;
  }

  // dS <- dS_T (or 0); dm <- dm_T (or 0)
  {
    const int c0 = half * 64;
    const float* src = a.dS_T ? a.dS_T + (size_t)pair * SZ + (size_t)row * kDK + c0
                              : nullptr;
    float vals[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 x = src ? *reinterpret_cast<const float4*>(src + part * 32 + i)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        vals[i] = x.x; vals[i + 1] = x.y; vals[i + 2] = x.z; vals[i + 3] = x.w;
      }
      tmem_st32(tl + T_DS + c0 + part * 32, vals);
    }
    tmem_st_wait();
  }
  if (tid < 128) s_dmn[tid] = a.dm_T ? a.dm_T[(size_t)pair * kDV + tid] : 0.f;

  auto wait = [&](uint64_t* bar, uint32_t par, uint32_t where) {
    wait_bar(bar, par, where, s_abort, a.hdr);
  };

  float dp_acc = 0.f;   // this thread's share of dp_j for the current chunk
  float vals[32];
  for (int ib = NB - 1, it = 0; ib >= 0; --ib, ++it) {
    const uint32_t par = (uint32_t)(it & 1);
    const int t0 = ib * kBlk;
    const int c = ib / bpc;
    const bool chunk_last = (ib + 1) % bpc == 0;  // first visited block of c
    const bool chunk_first = ib % bpc == 0;       // last visited block of c
    const int tok = b * T + t0;
    float* rec = args.gate_rec + ((size_t)pair * NC + c) * GR;
    const uint8_t* trec = a.tc_rec + ((size_t)pair * NB + ib) * kTcRecBytes;

    // ---- S0: gate of chunk c, p = U_up U_down m_c (forward record)
    if (chunk_last) {
      if (tid < 128) s_p[tid] = a.gin[((size_t)pair * NC + c) * GR + tid];
      dp_acc = 0.f;
    }

    // ---- S1: inputs: TMA of k, q, v, d_o, g, b_x; records S, E^T, T
    if (tid == 0) {
      mbar_expect_tx(bar_in, 6 * 16384 + (uint32_t)kTcRecBytes);
      tma_load_3d(sm + R_X, &tm_k, bar_in, 0, h, tok);
      tma_load_3d(sm + R_X + 16384, &tm_k, bar_in, 64, h, tok);
      tma_load_3d(sm + R_X + 8192, &tm_q, bar_in, 0, h, tok);
      tma_load_3d(sm + R_X + 24576, &tm_q, bar_in, 64, h, tok);
      tma_load_3d(sm + R_W, &tm_v, bar_in, 0, h, tok);
      tma_load_3d(sm + R_W + 8192, &tm_v, bar_in, 64, h, tok);
      tma_load_3d(sm + R_RO + 8192, &tm_do, bar_in, 0, h, tok);
      tma_load_3d(sm + R_RO + 24576, &tm_do, bar_in, 64, h, tok);
      tma_load_3d(sm + R_DSB, &tm_g, bar_in, 0, h, tok);
      tma_load_3d(sm + R_DSB + 8192, &tm_g, bar_in, 64, h, tok);
      tma_load_3d(sm + R_DSB + 16384, &tm_bx, bar_in, 0, h, tok);
      tma_load_3d(sm + R_DSB + 24576, &tm_bx, bar_in, 64, h, tok);
      bulk_load(sm + R_SB, trec + kTcRecS, 32768, bar_in);
      bulk_load(sm + R_ET, trec + kTcRecE, 16384, bar_in);
      bulk_load(sm + R_TT, trec + kTcRecT, 8192, bar_in);
      if (ib > 0) {  // the next block visited: its tiles, record and end state -> L2
        const int tn = tok - kBlk;
#pragma unroll
        for (int x0 = 0; x0 < 128; x0 += 64) {
          tma_prefetch_3d(&tm_k, x0, h, tn);
          tma_prefetch_3d(&tm_q, x0, h, tn);
          tma_prefetch_3d(&tm_v, x0, h, tn);
          tma_prefetch_3d(&tm_do, x0, h, tn);
          tma_prefetch_3d(&tm_g, x0, h, tn);
          tma_prefetch_3d(&tm_bx, x0, h, tn);
        }
        bulk_prefetch_l2(trec - kTcRecBytes, (uint32_t)kTcRecBytes);
        const float* nxt = a.ck_S + ((size_t)pair * (NB + 1) + ib) * SZ;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) bulk_prefetch_l2(nxt + q4 * 4096, 16384);
      }
    }
    if (tid < 64) s_w[tid] = __bfloat162float(w_in[((size_t)tok + tid) * H + h]);
    wait(bar_in, par, 11);
    const int j = tid & 127;
    if (half == 0) {
      float G = 0.f;
#pragma unroll 8
      for (int t = 0; t < 32; ++t) G += ldbf(sm + R_DSB + sw128_off(t, j, 64));
      s_x[j] = G;
    }
    __syncthreads();

    // ---- S2: transform (the half sums in s_x are consumed and zeroed: the
    //      same words accumulate dlog gamma next)
    {
      float G = 0.f;
      if (half) {
        G = s_x[j];
        s_x[j] = 0.f;
      }
      float gprev = half ? __expf(G) : 1.f;
      const float pj = s_p[j];
#pragma unroll 4
      for (int tt = 0; tt < 32; ++tt) {
        const int t = half * 32 + tt;
        const uint32_t oj = sw128_off(t, j, 64);
        const uint32_t ok = sw128_off(t, j, 128);
        const uint32_t oq = sw128_off(64 + t, j, 128);
        const float kk = ldbf(sm + R_X + ok);
        const float qq = ldbf(sm + R_X + oq);
        const float bb = sigm(ldbf(sm + R_DSB + 16384 + oj) + pj);
        G += ldbf(sm + R_DSB + oj);
        const float gam = __expf(G), igam = __fdividef(1.0f, gam);
        stbf(sm + R_X + ok, kk * gam);
        stbf(sm + R_X + oq, qq * gprev);
        const float kh = kk * igam;
        stbf(sm + R_KH + oj, kh);
        stbf(sm + R_KP + oj, bb * kh);
        gprev = gam;
      }
      if (half) s_gam[j] = gprev;
    }
    {
      const float invL = 1.0f / (float)a.L;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cidx = tid + 256 * i;  // 16-byte chunk of a 64 x 128 tile
        const int kb = cidx >> 9, rr = (cidx >> 3) & 63, ch = cidx & 7;
        const uint32_t sub = (uint32_t)((rr >> 3) * 1024 + (rr & 7) * 128 + ch * 16);
        // W = w V in place
        {
          const uint32_t off = (uint32_t)(kb * 8192) + sub;
          const uint4 x = *reinterpret_cast<const uint4*>(sm + R_W + off);
          const float wt = s_w[rr];
          const __nv_bfloat162* xv = reinterpret_cast<const __nv_bfloat162*>(&x);
          uint4 y;
          uint32_t* yv = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xv[e]);
            yv[e] = pack2(f.x * wt, f.y * wt);
          }
          *reinterpret_cast<uint4*>(sm + R_W + off) = y;
        }
        // dO = d_o + dm / L (rows 64.. of RO); logical column of the chunk
        {
          const uint32_t off = (uint32_t)(kb * 16384 + 8192) + sub;
          const uint4 x = *reinterpret_cast<const uint4*>(sm + R_RO + off);
          const int v0 = kb * 64 + ((ch ^ (rr & 7)) << 3);
          const __nv_bfloat162* xv = reinterpret_cast<const __nv_bfloat162*>(&x);
          uint4 y;
          uint32_t* yv = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xv[e]);
            yv[e] = pack2(f.x + s_dmn[v0 + 2 * e] * invL,
                          f.y + s_dmn[v0 + 2 * e + 1] * invL);
          }
          *reinterpret_cast<uint4*>(sm + R_RO + off) = y;
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (*s_abort) break;

    // ---- S3: G = X [kap^ | K^]^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t x0 = smem_u32(sm + R_X), kp0 = smem_u32(sm + R_KP);
      const uint32_t kh0 = smem_u32(sm + R_KH);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        const uint32_t k64 = (ks >> 2) * 8192 + (ks & 3) * 32;
        umma_bf16(tmem + T_G, desc_kmajor_sw128(x0 + kx),
                  desc_kmajor_sw128(kp0 + k64), ID_KK64, ks > 0);
        umma_bf16(tmem + T_G + 64, desc_kmajor_sw128(x0 + kx),
                  desc_kmajor_sw128(kh0 + k64), ID_KK64, ks > 0);
      }
      umma_commit(bar1);
    }

    // ---- S4: dS~ = dS Diag(gamma) (TMEM, and its bf16 operand over the
    //      consumed raw g, b_x) with dlog gamma_j = sum_v dS S_new; then the
    //      strictly lower [M; P_k] (warps 4-7) and P_kap (warps 2-3) operands
    {
      const int c0 = half * 64;
      const float* sn = a.ck_S + ((size_t)pair * (NB + 1) + ib + 1) * SZ +
                        (size_t)row * kDK + c0;
      float prod[64];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tl + T_DS + c0 + part * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(sn + part * 32 + e);
          prod[part * 32 + e] = vals[e] * x.x;
          prod[part * 32 + e + 1] = vals[e + 1] * x.y;
          prod[part * 32 + e + 2] = vals[e + 2] * x.z;
          prod[part * 32 + e + 3] = vals[e + 3] * x.w;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) vals[e] *= s_gam[c0 + part * 32 + e];
        tmem_st32(tl + T_DS + c0 + part * 32, vals);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(sm + R_DSB + sw128_chunk(row, half, part * 4 + c8, 128),
                   vals + c8 * 8);
      }
      float hi[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) hi[i] = prod[32 + i];
      const float s_lo = warp_reduce_scatter32(prod, lane);
      const float s_hi = warp_reduce_scatter32(hi, lane);
      atomicAdd(&s_x[c0 + lane], s_lo);
      atomicAdd(&s_x[c0 + 32 + lane], s_hi);
    }
    wait(bar1, par, 12);
    tc_fence_after();
    const int gi = row, gr = gi < 64 ? gi : gi - 64;
    if (half == 1 || gi >= 64) {
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tl + T_G + (half ? 64 : 0) + part * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (part * 32 + e >= gr) vals[e] = 0.f;
        if (half) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_chunk(sm + R_MP + sw128_chunk(gi, 0, part * 4 + c8, 128),
                     vals + c8 * 8);
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_chunk(sm + R_PQ + sw128_chunk(gr, 0, part * 4 + c8, 64),
                     vals + c8 * 8);
        }
      }
    }
    tmem_st_wait();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) break;

    // ---- S6: dE^T = -dS~ kap^T - dO^T P_kap
    if (tid == 0) {
      tc_fence_after();
      const uint32_t dsb0 = smem_u32(sm + R_DSB), kp0 = smem_u32(sm + R_KP);
      const uint32_t ro0 = smem_u32(sm + R_RO), pq0 = smem_u32(sm + R_PQ);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tmem + T_DER,
                  desc_kmajor_sw128(dsb0 + (ks >> 2) * 16384 + (ks & 3) * 32),
                  desc_kmajor_sw128(kp0 + (ks >> 2) * 8192 + (ks & 3) * 32),
                  ID_KK64_NA, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16(tmem + T_DER,
                  desc_mnmajor_sw128(ro0 + 8192 + ks * 2048, 16384),
                  desc_mnmajor_sw128(pq0 + ks * 2048, 8192), ID_MM64_NA, 1);
      umma_commit(bar3);
    }
    wait(bar3, par, 14);
    tc_fence_after();

    // ---- S7: dE -> RO rows 0..63 (tokens split between the halves);
    //      dR^T = dE^T T
    tmem_ld32(tl + T_DER + half * 32, vals);
#pragma unroll
    for (int e = 0; e < 32; ++e)
      stbf(sm + R_RO + sw128_off(half * 32 + e, row, 128), vals[e]);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), tt0 = smem_u32(sm + R_TT);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16(tmem + T_DER, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(tt0 + ks * 2048, 8192), ID_MM64, ks > 0);
      umma_commit(bar4);
    }
    if (tid < 64) s_dw[tid] = 0.f;
    wait(bar4, par, 15);
    tc_fence_after();

    // ---- S8: dR -> RO rows 0..63
    tmem_ld32(tl + T_DER + half * 32, vals);
#pragma unroll
    for (int e = 0; e < 32; ++e)
      stbf(sm + R_RO + sw128_off(half * 32 + e, row, 128), vals[e]);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) break;

    // ---- S9: G2raw = [dR; dO] [E; W]^T, dW^T, dS += [dR; dO]^T [K~; Q~],
    //      D7^T = S^T [dR; dO]^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), et0 = smem_u32(sm + R_ET);
      const uint32_t w0 = smem_u32(sm + R_W), dsb0 = smem_u32(sm + R_DSB);
      const uint32_t kh0 = smem_u32(sm + R_KH), mp0 = smem_u32(sm + R_MP);
      const uint32_t x0 = smem_u32(sm + R_X), sb0 = smem_u32(sm + R_SB);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        const uint32_t k64 = (ks >> 2) * 8192 + (ks & 3) * 32;
        umma_bf16(tmem + T_G2, desc_kmajor_sw128(ro0 + kx),
                  desc_mnmajor_sw128(et0 + ks * 2048, 16384), ID_KM64, ks > 0);
        umma_bf16(tmem + T_G2 + 64, desc_kmajor_sw128(ro0 + kx),
                  desc_kmajor_sw128(w0 + k64), ID_KK64, ks > 0);
        umma_bf16(tmem + T_RE, desc_kmajor_sw128(dsb0 + kx),
                  desc_kmajor_sw128(kh0 + k64), ID_KK64, ks > 0);
        umma_bf16(tmem + T_G, desc_mnmajor_sw128(sb0 + ks * 2048, 16384),
                  desc_kmajor_sw128(ro0 + kx), ID_MK128, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tmem + T_RE, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(mp0 + ks * 2048, 16384), ID_MM64, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tmem + T_DS, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(x0 + ks * 2048, 16384), ID_MM128, 1);
      umma_commit(bar5);
    }
    wait(bar5, par, 16);
    tc_fence_after();

    // ---- S10: reload raw g, b_x into SB; G2 (masked, bf16); dv, dw
    if (tid == 0 && !*s_abort) {
      mbar_expect_tx(bar_gb, 2 * 16384);
      tma_load_3d(sm + R_SB, &tm_g, bar_gb, 0, h, tok);
      tma_load_3d(sm + R_SB + 8192, &tm_g, bar_gb, 64, h, tok);
      tma_load_3d(sm + R_SB + 16384, &tm_bx, bar_gb, 0, h, tok);
      tma_load_3d(sm + R_SB + 24576, &tm_bx, bar_gb, 64, h, tok);
    }
    if (half == 1) {
      const int rl = row & 63;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        tmem_ld32(tl + T_G2 + q4 * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (((q4 & 1) * 32 + e) >= rl) vals[e] = 0.f;
        uint8_t* blk = sm + ((q4 >> 1) == 0 ? R_MP : R_PQ);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(blk + sw128_chunk(row, 0, (q4 & 1) * 4 + c8, 128), vals + c8 * 8);
      }
      fence_async_smem();
    } else {
      float prod[64];
      __nv_bfloat16* dvrow = dv + (size_t)tok * H * kDV + (size_t)h * kDV + row;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tl + T_RE + part * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int t = part * 32 + e;
          dvrow[(size_t)t * H * kDV] = __float2bfloat16_rn(s_w[t] * vals[e]);
          prod[t] = vals[e] * ldbf(sm + R_W + sw128_off(t, row, 64));
        }
      }
      float hi[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) hi[i] = prod[32 + i];
      const float s_lo = warp_reduce_scatter32(prod, lane);
      const float s_hi = warp_reduce_scatter32(hi, lane);
      atomicAdd(&s_dw[lane], s_lo);
      atomicAdd(&s_dw[32 + lane], s_hi);
    }
    tc_fence_before();
    __syncthreads();
    if (*s_abort) break;
    if (tid < 64) {  // dw_t = sum_v dW V = (sum_v dW W) / w_t
      const float wt = s_w[tid];
      dw[((size_t)tok + tid) * H + h] =
          __float2bfloat16_rn(wt != 0.f ? s_dw[tid] / wt : 0.f);
    }

    // ---- S11: D7^T += [-kap^; K^]^T G2^T ; D8^T = X^T G2 + dS~^T [E; W]^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kp0 = smem_u32(sm + R_KP), kh0 = smem_u32(sm + R_KH);
      const uint32_t mp0 = smem_u32(sm + R_MP), pq0 = smem_u32(sm + R_PQ);
      const uint32_t x0 = smem_u32(sm + R_X), dsb0 = smem_u32(sm + R_DSB);
      const uint32_t et0 = smem_u32(sm + R_ET), w0 = smem_u32(sm + R_W);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a0 = (ks < 4 ? kp0 : kh0) + (ks & 3) * 2048;
        const uint32_t g2 = (ks < 4 ? mp0 : pq0) + (ks & 3) * 32;
        umma_bf16(tmem + T_G, desc_mnmajor_sw128(a0, 8192),
                  desc_kmajor_sw128(g2), ks < 4 ? ID_MK128_NA : ID_MK128, 1);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tmem + T_RE, desc_mnmajor_sw128(x0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(mp0 + ks * 2048, 16384), ID_MM128, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        umma_bf16(tmem + T_RE, desc_mnmajor_sw128(dsb0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(et0 + ks * 2048, 16384), ID_MM64, 1);
        umma_bf16(tmem + T_RE + 64, desc_mnmajor_sw128(dsb0 + ks * 2048, 16384),
                  desc_kmajor_sw128(w0 + (ks >> 2) * 8192 + (ks & 3) * 32),
                  ID_MK64, 1);
      }
      umma_commit(bar7);
    }
    wait(bar7, par, 17);
    wait(bar_gb, par, 18);
    tc_fence_after();

    // ---- S12: per key channel j: dq, dk, db_x, dg, dp.  Pass 1 (ascending
    //      tokens) carries Gamma and forms every per-token gradient and the
    //      log-Gamma gradients dG_t; pass 2 (descending) sums dg_t = sum_{s>=t} dG_s.
    {
      const int jj = row;                 // key channel (TMEM lane)
      const int tb = half == 0 ? 32 : 0;  // token range [tb, tb + 32)
      const float pj = s_p[jj];
      const size_t tstride = (size_t)H * kDK;
      const size_t x0 = ((size_t)tok * H + h) * kDK + jj;
      float Gs = 0.f;                     // log Gamma before the range
      if (half == 0) {
#pragma unroll 8
        for (int t = 0; t < 32; ++t) Gs += ldbf(sm + R_SB + sw128_off(t, jj, 64));
      }
      float G = Gs, gprev = __expf(Gs);
      float dGv[32];
      float qfirst = 0.f;                 // dQ~ Q~ of the range's first token
      float d7k[16], d7q[16], d8p[16], d8h[16];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int tsub = tb + 16 * sub;
        tmem_ld16(tl + T_G + tsub, d7k);
        tmem_ld16(tl + T_G + 64 + tsub, d7q);
        tmem_ld16(tl + T_RE + tsub, d8p);
        tmem_ld16(tl + T_RE + 64 + tsub, d8h);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int tl_ = 16 * sub + e;
          const int t = tb + tl_;
          const uint32_t o64 = sw128_off(t, jj, 64);
          G += ldbf(sm + R_SB + o64);
          const float gam = __expf(G), igam = __fdividef(1.0f, gam);
          const float bb = sigm(ldbf(sm + R_SB + 16384 + o64) + pj);
          const float kt = ldbf(sm + R_X + sw128_off(t, jj, 128));
          const float qt = ldbf(sm + R_X + sw128_off(64 + t, jj, 128));
          const float kh = ldbf(sm + R_KH + o64);
          const float kp = ldbf(sm + R_KP + o64);
          const float dKt = d7k[e], dQt = d7q[e], dKp = -d8p[e], dKh = d8h[e];
          const size_t x = x0 + (size_t)t * tstride;
          dq[x] = __float2bfloat16_rn(dQt * gprev);
          dk[x] = __float2bfloat16_rn(dKt * gam + dKh * igam + dKp * bb * igam);
          const float dz = dKp * kh * bb * (1.f - bb);
          dbx[x] = __float2bfloat16_rn(dz);
          dp_acc += dz;
          const float qp = dQt * qt;        // Q~_t reads Gamma_{t-1}
          dGv[tl_] = dKt * kt - dKh * kh - dKp * kp;
          if (tl_ > 0)
            dGv[tl_ - 1] += qp;
          else
            qfirst = qp;
          gprev = gam;
        }
      }
      if (half == 0) {
        dGv[31] += s_x[jj];                 // t = 63: gradient of log gamma
        float tot = qfirst;                 // dG_31 (lower half) reads Q~_32
#pragma unroll
        for (int i = 0; i < 32; ++i) tot += dGv[i];
        s_gam[jj] = tot;                    // hand-off to the lower half
      }
      __syncthreads();
      float acc = half == 1 ? s_gam[jj] : 0.f;
#pragma unroll
      for (int i = 31; i >= 0; --i) {
        acc += dGv[i];
        dg[x0 + (size_t)(tb + i) * tstride] = __float2bfloat16_rn(acc);
      }
    }

    // ---- S13: gate of chunk c once all its blocks are done
    if (chunk_first) {
      if (half == 0) s_x[row] = dp_acc;
      __syncthreads();
      if (half == 1) {
        const float dpj = s_x[row] + dp_acc;
        s_x[row] = dpj;
        rec[row] = dpj;
      }
      __syncthreads();
      if (half == 0) {  // dh[r] = sum_j U_up[j][r] dp[j]
        float pr[kRMax];
        const float dpj = s_x[tid];
#pragma unroll
        for (int r = 0; r < kRMax; ++r) pr[r] = ureg[r] * dpj;
        const float part = warp_reduce_scatter32(pr, lane);
        s_gam[warp * 32 + lane] = part;
      }
      __syncthreads();
      if (tid < 32) {
        const float dhv = s_gam[tid] + s_gam[32 + tid] + s_gam[64 + tid] + s_gam[96 + tid];
        s_dw[tid] = dhv;
        if (tid < R) rec[kDK + tid] = dhv;
      }
      __syncthreads();
      if (half == 1) {  // dm[v] = sum_r U_down[r][v] dh[r]
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kRMax; ++r) acc = fmaf(ureg[r], s_dw[r], acc);
        s_dmn[row] = acc;
      }
      dp_acc = 0.f;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  // ---- dS0, dm0
  if (!*s_abort) {
    const int c0 = half * 64;
    if (a.dS0) {
      float* dst = a.dS0 + (size_t)pair * SZ + (size_t)row * kDK + c0;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tl + T_DS + c0 + part * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + part * 32 + e) =
              make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
      }
    }
    if (a.dm0 && tid < 128) a.dm0[(size_t)pair * kDV + tid] = s_dmn[tid];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dU_up[h][j][r] = sum_{b,c} dp[b,h,c][j] h[b,h,c][r]
// dU_down[h][r][v] = sum_{b,c} dh[b,h,c][r] m[b,h,c][v]   (fixed order)
// dp, dh come from the backward's gate records, h = U_down m_c from the
// forward's gate inputs, m_c from its checkpoints.
__global__ void du_from_gate_records(const float* __restrict__ rec,
                                     const float* __restrict__ gin,
                                     const float* __restrict__ ck_m, int B,
                                     int H, int NC, int R, int DK, int DV,
                                     float* du_down, float* du_up) {
  const int GR = DK + R;
  const size_t per = (size_t)DK * R + (size_t)R * DV;
  const size_t n = (size_t)H * per;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int h = (int)(idx / per);
    const size_t e = idx - (size_t)h * per;
    float acc = 0.f;
    if (e < (size_t)DK * R) {
      const int jj = (int)(e / R), r = (int)(e % R);
      for (int bb = 0; bb < B; ++bb)
        for (int c = 0; c < NC; ++c) {
          const size_t o = ((size_t)(bb * H + h) * NC + c) * GR;
          acc += rec[o + jj] * gin[o + DK + r];
        }
      du_up[(size_t)h * DK * R + e] = acc;
    } else {
      const size_t e2 = e - (size_t)DK * R;
      const int r = (int)(e2 / DV), v = (int)(e2 % DV);
      for (int bb = 0; bb < B; ++bb)
        for (int c = 0; c < NC; ++c) {
          const size_t o = ((size_t)(bb * H + h) * NC + c);
          acc += rec[o * GR + DK + r] * ck_m[o * DV + v];
        }
      du_down[(size_t)h * R * DV + e2] = acc;
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int D, int H, long long rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlk};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t tc_bwd_gate_record_floats(const carve_shape& s) {
  return (size_t)s.B * s.H * (size_t)(s.T / s.L) * (s.DK + s.R);
}

cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mg, mb, mdo;
  if (!a.tc_rec || !a.gin) return cudaErrorInvalidValue;
  const long long rows = (long long)a.B * a.T;
  if (!make_map(&mq, a.q, kDK, a.H, rows) || !make_map(&mk, a.k, kDK, a.H, rows) ||
      !make_map(&mv, a.v, kDV, a.H, rows) || !make_map(&mg, a.g, kDK, a.H, rows) ||
      !make_map(&mb, a.bx, kDK, a.H, rows) || !make_map(&mdo, a.d_o, kDV, a.H, rows))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(
      bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdTcArgs args{a, a.scratch};  // gate records live in the scratch area
  bwd_tc_kernel<<<a.B * a.H, kThreads, kSmemBytes, st>>>(args, mq, mk, mv, mg,
                                                         mb, mdo);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)a.H * ((size_t)a.DK * a.R + (size_t)a.R * a.DV);
  if (n > 0) {
    int blocks = (int)((n + 255) / 256);
    if (blocks > 4 * 148) blocks = 4 * 148;
    du_from_gate_records<<<blocks, 256, 0, st>>>(a.scratch, a.gin, a.ck_m, a.B,
                                                 a.H, a.NC, a.R, a.DK, a.DV,
                                                 a.du_down, a.du_up);
  }
  return cudaGetLastError();
}

}  // namespace carve
