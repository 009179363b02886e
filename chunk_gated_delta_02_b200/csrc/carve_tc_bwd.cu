// carve_tc_bwd.cu -- tensor-core (tcgen05 / TMEM / TMA) backward of the CARVE
// recurrent core for bf16 inputs, dk = dv = 128, chunks of 64 or 128 tokens.
//
// Exact reverse mode of the chunk form (see carve_tc_fwd.cu).  One CTA
// walks the blocks of one (sequence, head) pair from last to first.  The
// gradient of the block-end state, dS (dv x dk, fp32), lives in tensor
// memory for the whole walk.  Per block the training forward left a record
// (the bf16 state operand S, E and T = (I + A)^{-1}, as shared-memory
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

constexpr int kThreads = 512;
constexpr int kBlk = 64;
constexpr int kDK = 128;
constexpr int kDV = 128;

// shared memory map (bytes; the dynamic shared memory base is required to
// be 1024-aligned, which the kernel checks).  Tiles are 128-byte swizzled
// 64-column blocks of `rows` x 128 B, the UMMA canonical layout.
constexpr uint32_t R_X = 0;          // [K~; Q~]                        32 KB
constexpr uint32_t R_KHP = 32768;    // [K^; kap^] 2 blk x 128 rows     32 KB
constexpr uint32_t R_EW = 65536;     // [E (record); raw v -> W = w V]  32 KB
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
constexpr uint32_t SM_BAR = 2560;    // kNumBars mbarriers
constexpr uint32_t SM_TMEM = 2664;
constexpr uint32_t SM_ABORT = 2668;
constexpr uint32_t SM_QN = 2688;     // fused q / k norm: inverse norms [t][k, q] fp16, 256 B
constexpr uint32_t kSmemBytes = 232448;
static_assert(R_SM + SM_QN + 256 <= kSmemBytes, "small region");
static_assert(R_PQ == R_MP + 16384 && R_TT == R_PQ + 8192, "G2 blocks");

// mbarriers (index into the small region's array)
constexpr int B_IN = 0;    // q, d_o of this block
constexpr int B_GB = 1;    // raw g, b_x again for the epilogue
constexpr int B_1 = 2;     // MMA S3
constexpr int B_SB = 3;    // bf16 state record
constexpr int B_3 = 4;     // MMA S6
constexpr int B_4 = 5;     // MMA S7
constexpr int B_5 = 6;     // MMA S9
constexpr int B_7 = 7;     // MMA S11
constexpr int B_PRE = 8;   // v, g, b_x, E and T records
constexpr int B_7B = 9;    // MMA S11, the D8 half (issued by thread 256)
constexpr int B_5B = 10;   // MMA S9, the dW^T and dS half (issued by thread 256)
constexpr int B_TEST = 11; // test only: the redirected commit of a stalled block
constexpr int B_FIN = 12;  // an aborting CTA: thread 288's MMAs not yet committed
constexpr int kNumBars = 13;
static_assert(SM_BAR + 8 * kNumBars <= SM_TMEM, "mbarriers");

// TMEM columns
constexpr uint32_t T_DS = 0;     // dS [v][j]
constexpr uint32_t T_G = 128;    // [A|M ; P_kap|P_k] [i][t]  -> [dK~^T | dQ~^T]
constexpr uint32_t T_RE = 256;   // dW^T
constexpr uint32_t T_DER = 320;  // dE^T -> dR^T
constexpr uint32_t T_G2 = 384;   // raw G2 [r][c] -> D8 = [-dkap^T | dK^T]
constexpr uint32_t T_D8 = T_G2;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t ID_KK64 = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_KK128 = idesc_bf16(128, 128, false, false);
constexpr uint32_t ID_MK128 = idesc_bf16(128, 128, true, false);
constexpr uint32_t ID_MM64 = idesc_bf16(128, 64, true, true);
constexpr uint32_t ID_MM128 = idesc_bf16(128, 128, true, true);
constexpr uint32_t ID_KK64_NA = idesc_bf16_neg(128, 64, false, false, true, false);
constexpr uint32_t ID_MM64_NA = idesc_bf16_neg(128, 64, true, true, true, false);
constexpr uint32_t ID_MK128_NA = idesc_bf16_neg(128, 128, true, false, true, false);

using tc::warp_reduce_scatter32;

// Sum over the 32 lanes of a warp of v[i] (i < 16): lanes l and l ^ 16 end
// with the sum of index l % 16 in v[0].  (15 + 1 shuffles.)
__device__ __forceinline__ float warp_reduce_scatter16(float* v, int lane) {
#pragma unroll
  for (int k = 8; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = up ? v[i] : v[i + k];
      const float keep = up ? v[i + k] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// Sum over the 32 lanes of a warp of v[i] (i < 8): lanes l, l ^ 8, l ^ 16,
// l ^ 24 end with the sum of index l % 8 in v[0].
__device__ __forceinline__ float warp_reduce_scatter8(float* v, int lane) {
#pragma unroll
  for (int k = 4; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = up ? v[i] : v[i + k];
      const float keep = up ? v[i + k] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  float x = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 8);
  return x + __shfl_xor_sync(0xffffffffu, x, 16);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

struct BwdTcArgs {
  BwdArgs a;
  float* gate_rec;  // [B*H][NC][DK + R]: dp | dh per chunk
};

// 16 warps: warp w serves TMEM lane quadrant qd = w % 4 (value rows or key
// channels 32 qd .. 32 qd + 31) and column group gp = w / 4, so every
// element-wise phase is split four ways along the TMEM columns.
// ACT: the instance for raw decay logits (decay_scale > 0); QKN: the one
// for the fused q / k normalisation.  Instances without them carry none of
// their code.
template <bool ACT, bool QKN>
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
  __half* s_qn = reinterpret_cast<__half*>(sm + R_SM + SM_QN);
  float* s_dmn = reinterpret_cast<float*>(sm + R_SM + SM_DMN);
  float* s_x = reinterpret_cast<float*>(sm + R_SM + SM_X);
  float* s_gam = reinterpret_cast<float*>(sm + R_SM + SM_GAM);
  float* s_w = reinterpret_cast<float*>(sm + R_SM + SM_W);
  float* s_dw = reinterpret_cast<float*>(sm + R_SM + SM_DW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + R_SM + SM_BAR);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + R_SM + SM_TMEM);
  volatile uint32_t* s_abort =
      reinterpret_cast<volatile uint32_t*>(sm + R_SM + SM_ABORT);
  // fp32 scratch of the epilogue and the gate backward (the G2 buffer is
  // free once the last MMA that reads it retired)
  float* s_scr = reinterpret_cast<float*>(sm + R_MP);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, gp = warp >> 2;
  const int row = qd * 32 + lane;
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
    for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
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
  const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);

  // U_b factors as bf16 pairs: U_up[h][row][8 gp .. 8 gp + 7] and
  // U_down[h][8 gp .. 8 gp + 7][row] (zero beyond R)
  uint32_t uup[4], udn[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r0 = 8 * gp + 2 * i;
    float u0 = 0.f, u1 = 0.f, d0 = 0.f, d1 = 0.f;
    if (r0 < R) {
      u0 = __bfloat162float(uu[((size_t)h * kDK + row) * R + r0]);
      d0 = __bfloat162float(ud[((size_t)h * R + r0) * kDV + row]);
    }
    if (r0 + 1 < R) {
      u1 = __bfloat162float(uu[((size_t)h * kDK + row) * R + r0 + 1]);
      d1 = __bfloat162float(ud[((size_t)h * R + r0 + 1) * kDV + row]);
    }
    uup[i] = pack2(u0, u1);
    udn[i] = pack2(d0, d1);
  }

  // dS <- dS_T (or 0); dm <- dm_T (or 0).  dlog gamma_j = sum_v dS S_new
  // of the next block visited: this thread's share (column 32 gp + lane,
  // rows of its quadrant) rides in `dlg_part` until that block's S4; for the
  // last block S_new is the fp32 final state, later ones take the bf16 state
  // record of the block after them.
  float dlg_part = 0.f;
  {
    const int c0 = gp * 32;
    const float* src = a.dS_T ? a.dS_T + (size_t)pair * SZ + (size_t)row * kDK + c0
                              : nullptr;
    const float* sfin = a.ck_S + (size_t)pair * SZ + (size_t)row * kDK + c0;
    float vals[32], prod[32];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 x = src ? *reinterpret_cast<const float4*>(src + i)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 y = *reinterpret_cast<const float4*>(sfin + i);
      vals[i] = x.x; vals[i + 1] = x.y; vals[i + 2] = x.z; vals[i + 3] = x.w;
      prod[i] = x.x * y.x; prod[i + 1] = x.y * y.y;
      prod[i + 2] = x.z * y.z; prod[i + 3] = x.w * y.w;
    }
    tmem_st32(tl + T_DS + c0, vals);
    dlg_part = warp_reduce_scatter32(prod, lane);
    tmem_st_wait();
  }
  if (tid < 128) s_dmn[tid] = a.dm_T ? a.dm_T[(size_t)pair * kDV + tid] : 0.f;

  // Every barrier has at most one phase in flight.  `npar` holds the parity
  // each thread waits for next; the issuing threads also track in `pend`
  // the phases they started (copies issued, MMAs committed) so that an
  // aborting CTA drains them before it exits.
  uint32_t npar = 0, pend = 0;
  bool der_open = false;  // thread 288 issued S4's MMAs, S6 has not committed them
  auto wait = [&](int i, uint32_t where) {
    if (wait_bar(bars + i, (npar >> i) & 1u, where, s_abort, a.hdr, a.spin)) {
      npar ^= 1u << i;
      pend &= ~(1u << i);
    }
  };
  auto mark = [&](int i) { pend |= 1u << i; };
  auto tok_of = [&](int blk) { return b * T + blk * kBlk; };
  const uint8_t* rec0 = a.tc_rec + (size_t)pair * NB * kTcRecBytes;
  // k, q -> X; d_o -> RO rows 64..127
  auto issue_top = [&](int blk) {
    const int tk = tok_of(blk);
    mbar_expect_tx(bars + B_IN, 2 * 16384);
    tma_load_3d(sm + R_X + 8192, &tm_q, bars + B_IN, 0, h, tk);
    tma_load_3d(sm + R_X + 24576, &tm_q, bars + B_IN, 64, h, tk);
    tma_load_3d(sm + R_RO + 8192, &tm_do, bars + B_IN, 0, h, tk);
    tma_load_3d(sm + R_RO + 24576, &tm_do, bars + B_IN, 64, h, tk);
    mark(B_IN);
  };
  // the block's bf16 state operand (forward record) -> SB
  auto issue_sb = [&](int blk) {
    mbar_expect_tx(bars + B_SB, 32768);
    bulk_load(sm + R_SB, rec0 + (size_t)blk * kTcRecBytes + kTcRecS, 32768,
              bars + B_SB);
    mark(B_SB);
  };
  // k -> X rows 0..63; v -> W (rows 64.. of EW); g, b_x -> DSB; records
  // E -> rows 0..63 of EW, T -> TT
  auto issue_pre = [&](int blk) {
    const int tk = tok_of(blk);
    const uint8_t* r = rec0 + (size_t)blk * kTcRecBytes;
    mbar_expect_tx(bars + B_PRE, 5 * 16384 + 8192);
    // k -> rows 0..63 of X: K~ is no longer read once the D7 / D8 MMAs
    // retired (the epilogue takes K~ from K^)
    tma_load_3d(sm + R_X, &tm_k, bars + B_PRE, 0, h, tk);
    tma_load_3d(sm + R_X + 16384, &tm_k, bars + B_PRE, 64, h, tk);
    tma_load_3d(sm + R_EW + 8192, &tm_v, bars + B_PRE, 0, h, tk);
    tma_load_3d(sm + R_EW + 24576, &tm_v, bars + B_PRE, 64, h, tk);
    tma_load_3d(sm + R_DSB, &tm_g, bars + B_PRE, 0, h, tk);
    tma_load_3d(sm + R_DSB + 8192, &tm_g, bars + B_PRE, 64, h, tk);
    tma_load_3d(sm + R_DSB + 16384, &tm_bx, bars + B_PRE, 0, h, tk);
    tma_load_3d(sm + R_DSB + 24576, &tm_bx, bars + B_PRE, 64, h, tk);
    bulk_load(sm + R_EW, r + kTcRecE, 8192, bars + B_PRE);
    bulk_load(sm + R_EW + 16384, r + kTcRecE + 8192, 8192, bars + B_PRE);
    bulk_load(sm + R_TT, r + kTcRecT, 8192, bars + B_PRE);
    mark(B_PRE);
  };
  // raw g, b_x again for the epilogue -> RO
  auto issue_gb = [&](int blk) {
    const int tk = tok_of(blk);
    mbar_expect_tx(bars + B_GB, 2 * 16384);
    tma_load_3d(sm + R_RO, &tm_g, bars + B_GB, 0, h, tk);
    tma_load_3d(sm + R_RO + 8192, &tm_g, bars + B_GB, 64, h, tk);
    tma_load_3d(sm + R_RO + 16384, &tm_bx, bars + B_GB, 0, h, tk);
    tma_load_3d(sm + R_RO + 24576, &tm_bx, bars + B_GB, 64, h, tk);
    mark(B_GB);
  };
  if (tid == 0) {
    issue_top(NB - 1);
    issue_sb(NB - 1);
    issue_pre(NB - 1);
  }

  // w_t of the two token rows a thread of warps 8-15 scales in W = w V,
  // fetched one block ahead into registers (raw bf16 bits: converted only
  // when used, so the loads' latency is not waited for at issue)
  const unsigned short* w_bits = reinterpret_cast<const unsigned short*>(w_in);
  uint32_t w_lo = 0, w_hi = 0;
  if (warp >= 8) {
    const size_t r0 = (size_t)b * T + (NB - 1) * kBlk + ((tid - 256) >> 3);
    w_lo = w_bits[r0 * H + h];
    w_hi = w_bits[(r0 + 32) * H + h];
  }
  bool dm_pending = false;  // s_dmn still to be summed from the last chunk's partials
  float dp_acc = 0.f;   // dp_j share (channel row, this warp's token quarter)
  // p of the last chunk (the first visited); later chunks' p arrive by
  // async copies issued in the previous block's epilogue
  if (tid < 128) s_p[tid] = a.gin[((size_t)pair * NC + NC - 1) * GR + tid];
  for (int ib = NB - 1; ib >= 0; --ib) {
    const int t0 = ib * kBlk;
    const int c = ib / bpc;
    const bool chunk_last = (ib + 1) % bpc == 0;  // first visited block of c
    const bool chunk_first = ib % bpc == 0;       // last visited block of c
    const int tok = b * T + t0;
    float* rec = args.gate_rec + ((size_t)pair * NC + c) * GR;

    // ---- S0: gate of chunk c, p = U_up U_down m_c (forward record,
    //      copied into s_p during the previous block; published by the
    //      barrier at the end of S1)
    if (chunk_last) {
      if (ib < NB - 1 && tid < 32) cp_async_wait_all();
      dp_acc = 0.f;
    }
    if (dm_pending && tid < 128) {  // dm of the chunk after this one (S13)
      const float* s_dmq = reinterpret_cast<const float*>(sm + R_MP) + 2688;
      s_dmn[tid] = (s_dmq[tid] + s_dmq[128 + tid]) + (s_dmq[256 + tid] + s_dmq[384 + tid]);
    }
    dm_pending = false;

    // ---- S1: inputs, all requested during the previous block (q, d_o
    //      in its epilogue).  Block ib - 1's q, d_o tiles -> L2 (and k,
    //      which loads during this block).
    if (tid == 32 && ib > 0) {  // (the rest of block ib - 1 loads a block ahead)
      const int tn = tok - kBlk;
#pragma unroll 1
      for (int x0 = 0; x0 < 128; x0 += 64) {
        tma_prefetch_3d(&tm_k, x0, h, tn);
        tma_prefetch_3d(&tm_q, x0, h, tn);
        tma_prefetch_3d(&tm_do, x0, h, tn);
      }
    }
    wait(B_SB, 10);
    wait(B_PRE, 11);
    wait(B_IN, 12);
    __syncthreads();  // s_p of S0

    // ---- S2: transform (warps 0-7 the key side; warps 8-15 first the gate
    //      b = sigmoid(b_x + p) in fp16 over the raw b_x tile, handed to
    //      warps 0-7 by named barrier 7, then W = w V and dO = d_o + dm / L);
    //      s_x is cleared: it accumulates dlog gamma next
    if (warp < 8) {
      tc::transform_block<8, ACT, QKN>(
          sm + R_X, sm + R_KHP, sm + R_KHP + 8192, sm + R_DSB, sm + R_DSB + 16384,
          s_gam, reinterpret_cast<float*>(sm + R_MP), 3, 16384, 7, kThreads,
          a.dscale, kBlk, reinterpret_cast<float*>(sm + R_MP) + 1024, s_qn, 12);
      if (tid < 128) s_x[tid] = 0.f;
    } else {
      const int u = tid - 256;
      // b: chunk c = u + 256 i of the 64 x 128 tile (row c / 16, column
      // block (c / 8) % 2, 16-byte chunk c % 8; a quarter-warp per row)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = u + 256 * i;
        const int t = c >> 4, kb = (c >> 3) & 1, ch = c & 7;
        const uint32_t off = (uint32_t)(16384 + kb * 8192 + t * 128 + ((ch ^ (t & 7)) << 4));
        float bv[8];
        ld_chunk(sm + R_DSB + off, bv);
        const int j0 = kb * 64 + ch * 8;
        const float4 p0 = *reinterpret_cast<const float4*>(s_p + j0);
        const float4 p1 = *reinterpret_cast<const float4*>(s_p + j0 + 4);
        const float pj[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) bv[e] = sigm(bv[e] + pj[e]);
        tc::st_chunk_h(sm + R_DSB + off, bv);
      }
      bar_arrive_named(7, kThreads);
      const float invL = 1.0f / (float)a.L;
      const int rr = u >> 3, ch = u & 7;  // token rows rr, rr + 32; 16-byte chunk
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rr + 32 * (i & 1), kb = i >> 1;
        const uint32_t sub = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ch * 16);
        // W = w V in place (rows 64.. of EW)
        {
          const uint32_t off = (uint32_t)(kb * 16384 + 8192) + sub;
          const uint4 x = *reinterpret_cast<const uint4*>(sm + R_EW + off);
          const float wt = __uint_as_float(((i & 1) ? w_hi : w_lo) << 16);
          const __nv_bfloat162* xv = reinterpret_cast<const __nv_bfloat162*>(&x);
          uint4 y;
          uint32_t* yv = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xv[e]);
            yv[e] = pack2(f.x * wt, f.y * wt);
          }
          *reinterpret_cast<uint4*>(sm + R_EW + off) = y;
        }
        // dO = d_o + dm / L (rows 64.. of RO); logical column of the chunk
        {
          const uint32_t off = (uint32_t)(kb * 16384 + 8192) + sub;
          const uint4 x = *reinterpret_cast<const uint4*>(sm + R_RO + off);
          const int v0 = kb * 64 + ((ch ^ (r & 7)) << 3);
          const float4 m0 = *reinterpret_cast<const float4*>(s_dmn + v0);
          const float4 m1 = *reinterpret_cast<const float4*>(s_dmn + v0 + 4);
          const float dm8[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
          const __nv_bfloat162* xv = reinterpret_cast<const __nv_bfloat162*>(&x);
          uint4 y;
          uint32_t* yv = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xv[e]);
            yv[e] = pack2(fmaf(dm8[2 * e], invL, f.x), fmaf(dm8[2 * e + 1], invL, f.y));
          }
          *reinterpret_cast<uint4*>(sm + R_RO + off) = y;
        }
      }
      if ((u & 7) == 0) {  // this block's w_t for dv, dw (S11)
        s_w[u >> 3] = __uint_as_float(w_lo << 16);
        s_w[(u >> 3) + 32] = __uint_as_float(w_hi << 16);
      }
      if (ib > 0) {  // the next block's w_t
        const size_t r0 = (size_t)b * T + (ib - 1) * kBlk + ((tid - 256) >> 3);
        w_lo = w_bits[r0 * H + h];
        w_hi = w_bits[(r0 + 32) * H + h];
      }
    }
    fence_async_smem();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads

    // ---- S3: G = X [K^; kap^]^T (one N = 128 product per k-step):
    //      columns 0-63 [M; P_k], 64-127 [A; P_kap]
    if (tid == 0) {
      tc_fence_after();
      const uint32_t x0 = smem_u32(sm + R_X), khp0 = smem_u32(sm + R_KHP);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        umma_bf16(tmem + T_G, desc_kmajor_sw128(x0 + kx),
                  desc_kmajor_sw128(khp0 + kx), ID_KK128, ks > 0);
      }
      // test only: CTA 0 of a chosen block commits to a barrier nobody
      // waits on, so the wait for S3 below runs out (the products still
      // complete and are drained before the CTA exits)
      const int bm = (ib == a.stall_block && blockIdx.x == 0) ? B_TEST : B_1;
      umma_commit(bars + bm);
      mark(bm);
    }

    // ---- S4: dS~ = dS Diag(gamma) (TMEM, and its bf16 operand over the
    //      consumed raw g, b_x), dlog gamma; then the strictly lower
    //      [M; P_k] and P_kap operands
    {
      const int c0 = gp * 32;
      float vals[32];
      tmem_ld32(tl + T_DS + c0, vals);
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 gm = *reinterpret_cast<const float4*>(s_gam + c0 + e);
        vals[e] *= gm.x; vals[e + 1] *= gm.y; vals[e + 2] *= gm.z; vals[e + 3] *= gm.w;
      }
      tmem_st32(tl + T_DS + c0, vals);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        st_chunk(sm + R_DSB + sw128_chunk(row, gp >> 1, (gp & 1) * 4 + c8, 128),
                 vals + c8 * 8);
      atomicAdd(&s_x[c0 + lane], dlg_part);
    }
    // dE^T = -dS~ kap^T needs only dS~ and kap^: issued now, it runs while
    // the Grams are masked; thread 288 issues it (and S6), its warp has no
    // masking to do
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 288 && !*s_abort) {
      tc_fence_after();
      const uint32_t dsb0 = smem_u32(sm + R_DSB), kp0 = smem_u32(sm + R_KHP) + 8192;
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks)
        umma_bf16(tmem + T_DER,
                  desc_kmajor_sw128(dsb0 + (ks >> 2) * 16384 + (ks & 3) * 32),
                  desc_kmajor_sw128(kp0 + (ks >> 2) * 16384 + (ks & 3) * 32),
                  ID_KK64_NA, ks > 0);
      der_open = true;
    }
    wait(B_1, 13);
    tc_fence_after();
    {
      const int gr = row < 64 ? row : row - 64;
      const bool mp = gp < 2;
      if (mp || row >= 64) {
        const int piece = gp & 1;
        float vals[32];
        tmem_ld32(tl + T_G + (mp ? 0 : 64) + piece * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (piece * 32 + e >= gr) vals[e] = 0.f;
        if (mp) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_chunk(sm + R_MP + sw128_chunk(row, 0, piece * 4 + c8, 128),
                     vals + c8 * 8);
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_chunk(sm + R_PQ + sw128_chunk(gr, 0, piece * 4 + c8, 64),
                     vals + c8 * 8);
        }
      }
    }
    tmem_st_wait();
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads

    // ---- S6: dE^T = -dS~ kap^T (issued in S4) - dO^T P_kap
    if (tid == 288) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), pq0 = smem_u32(sm + R_PQ);
#pragma unroll 1
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16(tmem + T_DER,
                  desc_mnmajor_sw128(ro0 + 8192 + ks * 2048, 16384),
                  desc_mnmajor_sw128(pq0 + ks * 2048, 8192), ID_MM64_NA, 1);
      umma_commit(bars + B_3);
      mark(B_3);
      der_open = false;
    }
    wait(B_3, 14);
    tc_fence_after();

    // ---- S7: dE -> RO rows 0..63 (16 tokens per column group);
    //      dR^T = dE^T T
    {
      float vals[16];
      tmem_ld16(tl + T_DER + gp * 16, vals);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        stbf(sm + R_RO + sw128_off(gp * 16 + e, row, 128), vals[e]);
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), tt0 = smem_u32(sm + R_TT);
#pragma unroll 1
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16(tmem + T_DER, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(tt0 + ks * 2048, 8192), ID_MM64, ks > 0);
      umma_commit(bars + B_4);
      mark(B_4);
    }
    if (tid < 64) s_dw[tid] = 0.f;
    wait(B_4, 15);
    tc_fence_after();

    // ---- S8: dR -> RO rows 0..63
    {
      float vals[16];
      tmem_ld16(tl + T_DER + gp * 16, vals);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        stbf(sm + R_RO + sw128_off(gp * 16 + e, row, 128), vals[e]);
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads

    // ---- S9: G2raw = [dR; dO] [E; W]^T, dW^T, dS += [dR; dO]^T [K~; Q~],
    //      D7^T = S^T [dR; dO]^T.  Two issuers with their own commits:
    //      thread 0 G2 and D7 (TMEM columns T_G2, T_G), thread 256 dW^T and
    //      dS (T_RE, T_DS)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), ew0 = smem_u32(sm + R_EW);
      const uint32_t sb0 = smem_u32(sm + R_SB);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        umma_bf16(tmem + T_G2, desc_kmajor_sw128(ro0 + kx),
                  desc_kmajor_sw128(ew0 + kx), ID_KK128, ks > 0);
        umma_bf16(tmem + T_G, desc_mnmajor_sw128(sb0 + ks * 2048, 16384),
                  desc_kmajor_sw128(ro0 + kx), ID_MK128, ks > 0);
      }
      umma_commit(bars + B_5);
      mark(B_5);
    } else if (tid == 256) {
      tc_fence_after();
      const uint32_t ro0 = smem_u32(sm + R_RO), dsb0 = smem_u32(sm + R_DSB);
      const uint32_t kh0 = smem_u32(sm + R_KHP), mp0 = smem_u32(sm + R_MP);
      const uint32_t x0 = smem_u32(sm + R_X);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        umma_bf16(tmem + T_RE, desc_kmajor_sw128(dsb0 + kx),
                  desc_kmajor_sw128(kh0 + kx), ID_KK64, ks > 0);
      }
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        umma_bf16(tmem + T_RE, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(mp0 + ks * 2048, 16384), ID_MM64, 1);
        umma_bf16(tmem + T_DS, desc_mnmajor_sw128(ro0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(x0 + ks * 2048, 16384), ID_MM128, 1);
      }
      umma_commit(bars + B_5B);
      mark(B_5B);
    }
    wait(B_5, 16);
    wait(B_5B, 21);
    tc_fence_after();

    // ---- S10: the epilogue's raw g, b_x -> RO; G2 (masked, bf16; 32
    //      columns per group)
    if (tid == 0 && !*s_abort) issue_gb(ib);
    {
      const int rl = row & 63;
      float vals[32];
      tmem_ld32(tl + T_G2 + gp * 32, vals);
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (((gp & 1) * 32 + e) >= rl) vals[e] = 0.f;
      uint8_t* blk = sm + ((gp >> 1) == 0 ? R_MP : R_PQ);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        st_chunk(blk + sw128_chunk(row, 0, (gp & 1) * 4 + c8, 128), vals + c8 * 8);
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads

    // ---- S11: D7^T += [-kap^; K^]^T G2^T ; D8^T = X^T G2 + dS~^T [E; W]^T
    //      (into the columns G2 left); meanwhile dv, dw (16 tokens per group)
    //      and the dlog gamma share of block ib - 1 (its S_new is this
    //      block's state record, still in SB)
    //      Two issuers, so that neither warp is late for the barrier below
    //      by the whole batch: thread 0 the D7 half, thread 256 the D8 half
    //      (separate accumulators, separate commits).
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kh0 = smem_u32(sm + R_KHP), kp0 = kh0 + 8192;
      const uint32_t mp0 = smem_u32(sm + R_MP), pq0 = smem_u32(sm + R_PQ);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a0 = (ks < 4 ? kp0 : kh0) + (ks & 3) * 2048;
        const uint32_t g2 = (ks < 4 ? mp0 : pq0) + (ks & 3) * 32;
        umma_bf16(tmem + T_G, desc_mnmajor_sw128(a0, 16384),
                  desc_kmajor_sw128(g2), ks < 4 ? ID_MK128_NA : ID_MK128, 1);
      }
      umma_commit(bars + B_7);
      mark(B_7);
    } else if (tid == 256) {
      tc_fence_after();
      const uint32_t mp0 = smem_u32(sm + R_MP);
      const uint32_t x0 = smem_u32(sm + R_X), dsb0 = smem_u32(sm + R_DSB);
      const uint32_t ew0 = smem_u32(sm + R_EW);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        umma_bf16(tmem + T_D8, desc_mnmajor_sw128(x0 + ks * 2048, 16384),
                  desc_mnmajor_sw128(mp0 + ks * 2048, 16384), ID_MM128, ks > 0);
        umma_bf16(tmem + T_D8, desc_mnmajor_sw128(dsb0 + ks * 2048, 16384),
                  desc_kmajor_sw128(ew0 + (ks >> 2) * 16384 + (ks & 3) * 32),
                  ID_MK128, 1);
      }
      umma_commit(bars + B_7B);
      mark(B_7B);
    }
    if (ib > 0) {
      float vals[32];
      tmem_ld32(tl + T_DS + gp * 32, vals);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float sv[8];
        ld_chunk(sm + R_SB + sw128_chunk(row, gp >> 1, (gp & 1) * 4 + c8, 128), sv);
#pragma unroll
        for (int e = 0; e < 8; ++e) vals[8 * c8 + e] *= sv[e];
      }
      dlg_part = warp_reduce_scatter32(vals, lane);
    }
    {
      float dwv[16];
      tmem_ld16(tl + T_RE + gp * 16, dwv);
      __nv_bfloat16* dvrow = dv + ((size_t)tok + gp * 16) * H * kDV +
                             (size_t)h * kDV + row;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int t = gp * 16 + e;
        dvrow[(size_t)e * H * kDV] = __float2bfloat16_rn(s_w[t] * dwv[e]);
        dwv[e] *= ldbf(sm + R_EW + sw128_off(64 + t, row, 128));
      }
      const float sdw = warp_reduce_scatter16(dwv, lane);
      if (lane < 16) atomicAdd(&s_dw[gp * 16 + lane], sdw);
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 64) {  // dw_t = sum_v dW V = (sum_v dW W) / w_t
      const float wt = s_w[tid];
      dw[((size_t)tok + tid) * H + h] =
          __float2bfloat16_rn(wt != 0.f ? s_dw[tid] / wt : 0.f);
    }
    // block ib - 1's state operand -> SB (read above)
    if (tid == 0 && ib > 0 && !*s_abort) issue_sb(ib - 1);
    wait(B_7, 17);
    wait(B_7B, 20);
    // block ib - 1's v, g, b_x, E, T into the buffers S11 released
    if (tid == 0 && ib > 0 && !*s_abort) issue_pre(ib - 1);
    wait(B_GB, 18);
    tc_fence_after();

    // ---- S12: per key channel j = row and token quarter gp: dq, dk, db_x,
    //      dg, dp.  Ascending pass: Gamma from the quarter's log-decay prefix,
    //      every per-token gradient and the log-Gamma gradients dG_t;
    //      descending pass: dg_t = sum_{s >= t} dG_s with the later quarters'
    //      sums exchanged through shared memory.
    {
      const int jj = row;
      const int tb = gp * 16;             // token range [tb, tb + 16)
      float* s_gq = s_scr;                // [4][128] quarter log-decay sums
      float* s_lq = s_scr + 512;          // [4][128] quarter dG sums
      float* s_qf = s_scr + 1024;         // [4][128] dQ~ Q~ of a quarter's first token
      float gv[16];  // the range's log-decays, kept for the ascending pass
      {
        float gsum = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) gv[e] = ldbf(sm + R_RO + sw128_off(tb + e, jj, 64));
        if constexpr (ACT) {  // raw decay logits
          decay_act8(gv, a.dscale, true);
          decay_act8(gv + 8, a.dscale, true);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) gsum += gv[e];
        s_gq[gp * 128 + jj] = gsum;
      }
      __syncthreads();
      float G = 0.f;                      // log Gamma before the range
      for (int g2 = 0; g2 < gp; ++g2) G += s_gq[g2 * 128 + jj];
      const float pj = s_p[jj];
      const size_t tstride = (size_t)H * kDK;
      const size_t x0 = ((size_t)tok * H + h) * kDK + jj;
      float gprev = __expf(G);
      float dGv[16];
      float qfirst = 0.f;
      // Outputs leave as bf16 pairs of neighbouring channels: for each pair
      // of tokens (2u, 2u + 1) the even lane of a lane pair stores token 2u
      // and the odd lane token 2u + 1, each after one shuffle (half the
      // store instructions of one 2-byte store per value).
      const bool odd = (lane & 1) != 0;
      const size_t xp = x0 - (jj & 1);    // element offset of the pair's even channel
      auto st_pair = [&](__nv_bfloat16* base, int t_even, float v_even, float v_odd) {
        const float recv = __shfl_xor_sync(0xffffffffu, odd ? v_even : v_odd, 1);
        const __nv_bfloat162 pr = odd ? __floats2bfloat162_rn(recv, v_odd)
                                      : __floats2bfloat162_rn(v_even, recv);
        *reinterpret_cast<__nv_bfloat162*>(
            base + xp + (size_t)(t_even + (odd ? 1 : 0)) * tstride) = pr;
      };
      float hq = 0.f, hk = 0.f, hz = 0.f;  // the even token's values
      float igprev = 0.f;                   // 1 / Gamma_{t-1} (QKN only)
      if constexpr (QKN) igprev = __expf(-G);
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        float vq8[8], vk8[8], qh8[8], kh8[8];  // QKN: this sub-block's tokens
        float dd[32];  // dK~ | dQ~ | -dkap^ | dK^ of 8 tokens
        const int tsub = tb + 8 * sub;
        tmem_ld8x4(tl + T_G + tsub, tl + T_G + 64 + tsub, tl + T_D8 + tsub,
                   tl + T_D8 + 64 + tsub, dd);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int tl_ = 8 * sub + e;
          const int t = tb + tl_;
          const uint32_t o64 = sw128_off(t, jj, 64);
          G += gv[tl_];
          const float gam = __expf(G), igam = __fdividef(1.0f, gam);
          const float bb = sigm(ldbf(sm + R_RO + 16384 + o64) + pj);
          const float qt = ldbf(sm + R_X + sw128_off(64 + t, jj, 128));
          const float kh = ldbf(sm + R_KHP + sw128_off(t, jj, 128));
          const float kt = kh * gam * gam;  // K~ = K^ Gamma^2
          const float kp = bb * kh;         // kap^ = b K^
          const float dKt = dd[e], dQt = dd[8 + e], dKp = -dd[16 + e], dKh = dd[24 + e];
          const float vq = dQt * gprev;
          const float vk = fmaf(dKt, gam, fmaf(dKp, bb, dKh) * igam);
          const float dz = dKp * kh * bb * (1.f - bb);
          if constexpr (QKN) {
            // the gradients of the unit q^, k^ (q^ = Q~ / Gamma_{t-1},
            // k^ = K^ Gamma_t), projected once the block's dots are known
            vq8[e] = vq;
            vk8[e] = vk;
            qh8[e] = qt * igprev;
            kh8[e] = kh * gam;
          }
          if ((e & 1) == 0) {
            hq = vq; hk = vk; hz = dz;
          } else {
            if constexpr (!QKN) {
              st_pair(dq, t - 1, hq, vq);
              st_pair(dk, t - 1, hk, vk);
            }
            st_pair(dbx, t - 1, hz, dz);
          }
          dp_acc += dz;
          const float qp = dQt * qt;        // Q~_t reads Gamma_{t-1}
          dGv[tl_] = dKt * kt - dKh * kh - dKp * kp;
          if (tl_ > 0)
            dGv[tl_ - 1] += qp;
          else
            qfirst = qp;
          gprev = gam;
          if constexpr (QKN) igprev = igam;
        }
        if constexpr (QKN) {
          // dq = (dq^ - q^ (q^ . dq^)) / |q| and the same for k: the dots
          // over the 128 channels of each token live on the four warps of
          // this token quarter (warps 4 gp .. 4 gp + 3, named barrier 8 + gp)
          float pr[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pr[e] = vq8[e] * qh8[e];
            pr[8 + e] = vk8[e] * kh8[e];
          }
          const float wsum = warp_reduce_scatter16(pr, lane);
          float* s_part = s_scr + 1536;  // [4 quarters][4 warps][16]
          float* s_fin = s_scr + 1792;   // [4 quarters][16]
          if (lane < 16) s_part[(gp * 4 + qd) * 16 + lane] = wsum;
          bar_named(8 + gp, 128);
          if (qd == 0 && lane < 16)
            s_fin[gp * 16 + lane] =
                (s_part[(gp * 4) * 16 + lane] + s_part[(gp * 4 + 1) * 16 + lane]) +
                (s_part[(gp * 4 + 2) * 16 + lane] + s_part[(gp * 4 + 3) * 16 + lane]);
          bar_named(8 + gp, 128);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int t = tsub + e;
            const float ink = __half2float(s_qn[t * 2]), inq = __half2float(s_qn[t * 2 + 1]);
            const float dqr = inq * fmaf(-qh8[e], s_fin[gp * 16 + e], vq8[e]);
            const float dkr = ink * fmaf(-kh8[e], s_fin[gp * 16 + 8 + e], vk8[e]);
            if ((e & 1) == 0) {
              hq = dqr; hk = dkr;
            } else {
              st_pair(dq, t - 1, hq, dqr);
              st_pair(dk, t - 1, hk, dkr);
            }
          }
        }
      }
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) lsum += dGv[i];
      s_lq[gp * 128 + jj] = lsum;
      s_qf[gp * 128 + jj] = qfirst;
      __syncthreads();
      // the ascending pass was the last reader of Q~ (X rows 64..127) and of
      // the raw g, b_x (RO): block ib - 1's q, d_o load from here on
      if (tid == 0 && ib > 0 && !*s_abort) issue_top(ib - 1);
      // s_p was last read above: the next block starts chunk c - 1
      if (chunk_first && ib > 0 && tid < 32) {
        cp_async16(s_p + 4 * tid, a.gin + ((size_t)pair * NC + c - 1) * GR + 4 * tid);
        cp_async_commit();
      }
      // dG_{tb+15} reads the next quarter's first Q~ term (t = 63: the
      // gradient of log gamma); the later quarters' sums seed the suffix
      const float dlg = s_x[jj];
      dGv[15] += gp < 3 ? s_qf[(gp + 1) * 128 + jj] : dlg;
      float acc = 0.f;
      for (int g2 = gp + 1; g2 < 4; ++g2)
        acc += s_lq[g2 * 128 + jj] + (g2 < 3 ? s_qf[(g2 + 1) * 128 + jj] : dlg);
      // with raw decay logits a (decay_scale s > 0) the output is dL/da =
      // dL/dg * s expm1(g / s), formed from the log-decay itself
      if constexpr (ACT) {  // dL/dg -> dL/da needs s expm1(g / s)
#pragma unroll
        for (int i = 0; i < 16; ++i) gv[i] = decay_act_grad(gv[i], a.dscale);
      }
      float hg = 0.f;  // the odd token's suffix sum
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        acc += dGv[i];
        const float out = ACT ? acc * gv[i] : acc;
        if (i & 1)
          hg = out;
        else
          st_pair(dg, tb + i, out, hg);
      }
    }

    // ---- S13: gate of chunk c once all its blocks are done:
    //      dp_j -> dh = U_up^T dp -> dm = U_down^T dh
    if (chunk_first) {
      float* s_dpq = s_scr + 2048;        // [4][128] dp quarter sums
      float* s_dhq = s_scr + 2560;        // [4][32] dh partials (per quadrant)
      float* s_dmq = s_scr + 2688;        // [4][128] dm partials (per group)
      s_dpq[gp * 128 + row] = dp_acc;
      __syncthreads();
      const float dpj = s_dpq[row] + s_dpq[128 + row] + s_dpq[256 + row] +
                        s_dpq[384 + row];
      if (gp == 0) rec[row] = dpj;
      {  // dh[r], r = 8 gp + i: this quadrant's channels
        float pr[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pr[2 * i] = bf_lo(uup[i]) * dpj;
          pr[2 * i + 1] = bf_hi(uup[i]) * dpj;
        }
        const float part = warp_reduce_scatter8(pr, lane);
        if (lane < 8) s_dhq[qd * 32 + gp * 8 + lane] = part;
      }
      __syncthreads();
      // dh[r] = sum of the four quadrants' partials, formed where it is
      // used; dm[v] partial over r = 8 gp .. 8 gp + 7, v = row (summed
      // into s_dmn at the next block's start, after the block barrier)
      auto dh = [&](int r) {
        return (s_dhq[r] + s_dhq[32 + r]) + (s_dhq[64 + r] + s_dhq[96 + r]);
      };
      if (tid < R) rec[kDK + tid] = dh(tid);
      {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc = fmaf(bf_lo(udn[i]), dh(8 * gp + 2 * i), acc);
          acc = fmaf(bf_hi(udn[i]), dh(8 * gp + 2 * i + 1), acc);
        }
        s_dmq[gp * 128 + row] = acc;
      }
      dm_pending = true;
      dp_acc = 0.f;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (tid < 32) cp_async_wait_all();  // (an aborted walk may leave one in flight)
  // ---- dS0, dm0; an aborted CTA first lets its copies and MMAs land
  if (*s_abort) {
    if (tid == 288 && der_open) {  // S4's MMAs were issued, S6 never committed them
      umma_commit(bars + B_FIN);
      mark(B_FIN);
    }
    if (tid == 0 || tid == 256 || tid == 288)  // the threads that start copies and MMAs
      for (int i = 0; i < kNumBars; ++i)
        if ((pend >> i) & 1u) drain_bar(bars + i, (npar >> i) & 1u);
  } else {
    const int c0 = gp * 32;
    if (a.dS0) {
      float* dst = a.dS0 + (size_t)pair * SZ + (size_t)row * kDK + c0;
      float vals[32];
      tmem_ld32(tl + T_DS + c0, vals);
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + e) =
            make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
    }
    if (a.dm0 && tid < 128) {  // chunk 0's dm, from S13's partials
      const float* s_dmq = reinterpret_cast<const float*>(sm + R_MP) + 2688;
      a.dm0[(size_t)pair * kDV + tid] =
          (s_dmq[tid] + s_dmq[128 + tid]) + (s_dmq[256 + tid] + s_dmq[384 + tid]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dU_up[h][j][r] = sum_b sum_c dp[b,h,c][j] h[b,h,c][r]
// dU_down[h][r][v] = sum_b sum_c dh[b,h,c][r] m[b,h,c][v]   (fixed order)
// dp, dh come from the backward's gate records, h = U_down m_c from the
// forward's gate inputs, m_c from its checkpoints.  Stage 1: CTA (pair,
// part) sums the pair's chunks in order for the channel rows 32 part .. + 31
// of dU_up and the value columns 32 part .. + 31 of dU_down, through
// 64-record slabs in shared memory, into the pair's slot of the workspace
// (layout: dU_down [R][DV] then dU_up [DK][R]); stage 2 sums the pairs of a
// head over b in order.  R <= 32.
constexpr int kDuThreads = 256;
constexpr int kDuSlab = 64;
__global__ void __launch_bounds__(kDuThreads)
    du_pair_partials(const float* __restrict__ rec,
                     const float* __restrict__ gin,
                     const float* __restrict__ ck_m, int NC, int R,
                     float* __restrict__ part) {
  __shared__ __align__(16) float s_dp[kDuSlab][32];
  __shared__ __align__(16) float s_hv[kDuSlab][32];
  __shared__ __align__(16) float s_dh[kDuSlab][32];
  __shared__ __align__(16) float s_m[kDuSlab][32];
  const int pair = blockIdx.x, pt = blockIdx.y, t = threadIdx.x;
  const int GR = kDK + R;
  const int hi = t >> 3, lo4 = 4 * (t & 7);
  float up[4] = {0.f, 0.f, 0.f, 0.f}, dn[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < NC; c0 += kDuSlab) {
    for (int idx = t; idx < kDuSlab * 32; idx += kDuThreads) {
      const int c = c0 + (idx >> 5), k = idx & 31;
      float dp = 0.f, hv = 0.f, dh = 0.f, mv = 0.f;
      if (c < NC) {
        const size_t o = (size_t)pair * NC + c;
        dp = rec[o * GR + 32 * pt + k];
        mv = ck_m[o * kDV + 32 * pt + k];
        if (k < R) {
          hv = gin[o * GR + kDK + k];
          dh = rec[o * GR + kDK + k];
        }
      }
      s_dp[idx >> 5][k] = dp;
      s_hv[idx >> 5][k] = hv;
      s_dh[idx >> 5][k] = dh;
      s_m[idx >> 5][k] = mv;
    }
    __syncthreads();
    const int ns = min(kDuSlab, NC - c0);
    for (int n = 0; n < ns; ++n) {
      const float a = s_dp[n][hi], d = s_dh[n][hi];
      const float4 hv = *reinterpret_cast<const float4*>(&s_hv[n][lo4]);
      const float4 mv = *reinterpret_cast<const float4*>(&s_m[n][lo4]);
      up[0] = fmaf(a, hv.x, up[0]); up[1] = fmaf(a, hv.y, up[1]);
      up[2] = fmaf(a, hv.z, up[2]); up[3] = fmaf(a, hv.w, up[3]);
      dn[0] = fmaf(d, mv.x, dn[0]); dn[1] = fmaf(d, mv.y, dn[1]);
      dn[2] = fmaf(d, mv.z, dn[2]); dn[3] = fmaf(d, mv.w, dn[3]);
    }
    __syncthreads();
  }
  float* base = part + (size_t)pair * ((size_t)R * kDV + (size_t)kDK * R);
  const int j = 32 * pt + hi;  // dU_up row; dU_down row is r = hi
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (hi < R) base[(size_t)hi * kDV + 32 * pt + lo4 + k] = dn[k];
    if (lo4 + k < R) base[(size_t)R * kDV + (size_t)j * R + lo4 + k] = up[k];
  }
}

__global__ void du_sum_pairs(const float* __restrict__ part, int B, int H,
                             int R, float* du_down, float* du_up) {
  const size_t per = (size_t)R * kDV + (size_t)kDK * R;
  const size_t n = (size_t)H * per;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int h = (int)(idx / per);
    const size_t e = idx - (size_t)h * per;
    float acc = 0.f;
    for (int bb = 0; bb < B; ++bb) acc += part[((size_t)bb * H + h) * per + e];
    if (e < (size_t)R * kDV)
      du_down[(size_t)h * R * kDV + e] = acc;
    else
      du_up[(size_t)h * kDK * R + (e - (size_t)R * kDV)] = acc;
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
  auto kern = a.dscale > 0.f ? (a.qknorm ? bwd_tc_kernel<true, true> : bwd_tc_kernel<true, false>)
                             : (a.qknorm ? bwd_tc_kernel<false, true> : bwd_tc_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdTcArgs args{a, a.scratch};  // gate records live in the scratch area
  kern<<<a.B * a.H, kThreads, kSmemBytes, st>>>(args, mq, mk, mv, mg, mb, mdo);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.R > 0) {
    du_pair_partials<<<dim3(a.B * a.H, kDK / 32), kDuThreads, 0, st>>>(
        a.scratch, a.gin, a.ck_m, a.NC, a.R, a.du);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t n = (size_t)a.H * ((size_t)a.R * kDV + (size_t)kDK * a.R);
    int blocks = (int)((n + 255) / 256);
    if (blocks > 4 * 148) blocks = 4 * 148;
    du_sum_pairs<<<blocks, 256, 0, st>>>(a.du, a.B, a.H, a.R, a.du_down, a.du_up);
  }
  return cudaGetLastError();
}

}  // namespace carve
