// carve_tc_fwd.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of the CARVE
// recurrent core for bf16 inputs, dk = dv = 128, chunks of 64 or 128 tokens.
//
// One CTA (16 warps) walks one (sequence, head) pair through its blocks of
// C = 64 tokens.  The fp32 state S (dv x dk) lives in tensor memory for the
// whole walk; a bf16 copy in shared memory is the MMA operand.  Per block,
// with the notation of the chunk form (CARVE summaries, gist.science,
// section 3, "Chunkability Boundary": erase on the key axis only, so one
// triangular solve per block serves every value row):
//
//   keys        Gamma = exp(cumsum g), K~ = K Gamma, Q~ = Q Gamma_{t-1},
//               K^ = K / Gamma (section 2.3: key-axis decay)
//   gate        at a chunk's end: p = U_up U_down m_{c+1} (section 2.1)
//   G           kap^ = sigmoid(b_x + p) K^, then both Grams in one product
//               G = [K~; Q~] [K^; kap^]^T -> [M ; P_k | A ; P_kap]
//   D1          S [K~; Q~]^T -> [(K~ S^T)^T | (Q~ S^T)^T];  W = w V
//   MMA 2       D1 += W^T [M; P_k]^T          ->  [R^T | (Q~ S^T + P_k W)^T]
//   solve       T = (I + A)^{-1} by 16 x 16 blocks
//   MMA 3a      E^T = R^T T^T                 (E = T R, the WY pseudo-values)
//   MMA 3b      D1[O] -= E^T P_kap^T          ->  O^T = (Q~ S^T + P_k W - P_kap E)^T
//   MMA 4       S += W^T K^ (issued once W is formed) - E^T kap^ ;
//               S <- S Diag(gamma)
//   output      o_t = row t of O; m_{c+1} = mean of the chunk's o_t
//
// The transposed products put one value row v of S, R, E and O in TMEM lane
// v, so each thread owns a value row: the chunk mean is a per-thread sum.
// Raw input tiles arrive by TMA (128-byte swizzle) into buffers whose layout
// is exactly the UMMA canonical layout, so the element-wise transforms write
// operands at the offsets they read them from (W = w V over the v tile, T
// over A).  Three warp groups run the blocks without a CTA-wide barrier:
// warps 0-3 the chain through the solve and MMAs 3a-4, warps 4-7 MMA 2 and
// the state rescale, warps 8-15 the next block's key side, gate and Grams,
// so that a block's solve starts as soon as its Grams land.  In training
// mode each block's bf16 S operand, E and T go straight from registers to
// the workspace (the backward's records); of the fp32 states only the final
// one is kept.
#include <cudaTypedefs.h>

#include "carve_internal.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace carve {
namespace {

using namespace ptx;
using tc::bar_arrive_named;
using tc::bar_named;
using tc::fsw;
using tc::pack2;
using tc::st_chunk;
using tc::unit_lower_inverse64;

constexpr int kThreads = 512;
constexpr int kBlk = 64;   // rows of a token tile (tokens per block C <= 64)
constexpr int kDK = 128;   // key width
constexpr int kDV = 128;   // value rows per CTA
constexpr int kRMax = 32;  // rank of U_b held in registers

// shared memory map (bytes from a 1024-aligned base); 128-byte swizzled
// tiles are 64-column blocks of `rows` x 128 B.
constexpr uint32_t OFF_X = 0;          // [K~; Q~]   2 blk x 128 rows  32 KB
constexpr uint32_t OFF_KHP = 32768;    // [K^; kap^] 2 blk x 128 rows  32 KB
constexpr uint32_t OFF_PQ = 65536;     // P_kap bf16 64 rows            8 KB
constexpr uint32_t OFF_WS = 73728;     // the inversion's scratch fp32  8 KB
constexpr uint32_t OFF_MY = 81920;     // [M;P_k] then Y, 128 rows     16 KB
constexpr uint32_t OFF_RE = 98304;     // R^T then -E^T, 128 rows      16 KB
constexpr uint32_t OFF_SB = 114688;    // S (bf16)   2 blk x 128 rows  32 KB
constexpr uint32_t OFF_RV = 147456;    // raw v -> W = w V in place    16 KB
constexpr uint32_t OFF_RG = 163840;    // raw g                        16 KB
constexpr uint32_t OFF_RB = 180224;    // raw b_x                      16 KB
constexpr uint32_t OFF_AF = 196608;    // A -> T in place, fp32 64 x 64 16 KB
constexpr uint32_t OFF_SMALL = 212992;
constexpr uint32_t SM_GAM = 0;         // gamma_j (even blocks) 128 f32
constexpr uint32_t SM_P = 512;         // (U_b m)_j          128 f32
constexpr uint32_t SM_HX = 1024;       // the other CTA's half of U_down m, 2 x 32 f32
constexpr uint32_t SM_M = 1280;        // m_v                128 f32
constexpr uint32_t SM_H = 1792;        // U_down m            64 f32
constexpr uint32_t SM_GAM1 = 2048;     // gamma_j (odd blocks)  128 f32
constexpr uint32_t SM_BAR = 2560;      // kNumBars mbarriers
constexpr uint32_t SM_TMEM = 2648;     // TMEM base address
constexpr uint32_t SM_ABORT = 2652;    // abort flag
constexpr uint32_t kSmallBytes = 2688;
constexpr uint32_t OFF_UU = 215808;    // U_up^T bf16 [kRMax][kUuLd]   8.5 KB
constexpr int kUuLd = 128 + 8;         // row pitch: 16 B of padding per row
constexpr uint32_t OFF_RED = OFF_UU + kRMax * kUuLd * 2;  // decay-scan scratch 2 KB
constexpr uint32_t kSmemBytes = OFF_RED + 2048 + 1024;
static_assert(OFF_SMALL + kSmallBytes <= OFF_UU, "shared memory map overlap");
static_assert(kSmemBytes <= 232448, "dynamic shared memory above 227 KB");

// mbarriers (index into the small region's array).  Each is waited once per
// block by every thread of the groups listed (warps 0-3: S, 4-7: R, 8-15: K)
constexpr int B_GB = 0;    // TMA g, b_x (thread 256; K)
constexpr int B_KQ = 1;    // TMA k, q (thread 256; K)
constexpr int B_GK = 2;    // Grams [M; P_k | A; P_kap] (thread 256; S, R, K)
constexpr int B_M2 = 3;    // MMA 2 (thread 128; S, R, K)
constexpr int B_M3 = 4;    // MMA 3a (thread 0; S, and R one block later)
constexpr int B_M4 = 5;    // MMA 3b + 4 (thread 0; S, R, K)
constexpr int B_X = 6;     // dv = 256: the other CTA's half of U_down m arrived
constexpr int B_WK = 7;    // S += W^T K^ (thread 256; S, R, K)
constexpr int B_TEST = 8;  // test only: the redirected commit of a stalled block
constexpr int B_D1 = 9;    // D1 = S [K~; Q~]^T (thread 128; R, K)
constexpr int B_V = 10;    // TMA v (thread 256; K)
constexpr int kNumBars = 11;
static_assert(SM_BAR + 8 * kNumBars <= SM_TMEM, "mbarriers");

// TMEM columns (fp32, lanes = rows)
constexpr uint32_t TM_S = 0;     // state S          [v][j]     128 cols
constexpr uint32_t TM_D1 = 128;  // [R|..] -> [E|O]  [v][n]     128 cols
constexpr uint32_t TM_G = 256;   // [M; P_k | A; P_kap]  [i][t] 128 cols
constexpr uint32_t TM_GM = 256;  //   [M; P_k]                   64 cols
constexpr uint32_t TM_GK = 320;  //   [A; P_kap]                 64 cols
constexpr uint32_t TM_E = 384;   // E = T R (training) [t][v], lanes 0-63  128 cols
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t ID_N64 = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_N128 = idesc_bf16(128, 128, false, false);
constexpr uint32_t ID_AMN = idesc_bf16(128, 128, true, false);
constexpr uint32_t ID_AMN_BMN = idesc_bf16(128, 128, true, true);
constexpr uint32_t ID_N64_NA = idesc_bf16_neg(128, 64, false, false, true, false);
constexpr uint32_t ID_BMN_NA = idesc_bf16_neg(128, 128, false, true, true, false);


// Key side of one block's transform by warps 8-15 (one out-of-line copy of
// the unrolled code serves the prologue and the block loop): K~, Q~ in place
// in X, K^ straight into rows 0..63 of its operand slot in KHP.
template <bool ACT>
static __device__ __noinline__ void keys_w8(uint8_t* x, uint8_t* kh,
                                            const uint8_t* rg, float* gam,
                                            float* red, float dscale,
                                            int nvalid, float* nrm) {
  tc::transform_keys<8, ACT>(x, kh, rg, gam, red, 3, 16384, 8, dscale, nvalid, nrm);
}

// 16 warps in three groups (see the block loop): warp w serves TMEM lane
// quadrant qd = w % 4 (value rows or Gram rows 32 qd .. 32 qd + 31).  Thread
// 0 issues MMAs 3a, 3b, 4; thread 128 D1 and MMA 2; thread 256 the copies,
// S += W^T K^ and the Grams.
// ACT: the instance for raw decay logits (decay_scale > 0); the other one
// has no activation code at all.  SHORT: the instance for blocks shorter
// than 64 tokens (chunks of 16, 32, 48), which forms kap^ for the block's
// rows only; the full-block instance keeps its 64-row loop
template <bool ACT, bool SHORT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_g,
                  const __grid_constant__ CUtensorMap tm_bx,
                  const __grid_constant__ CUtensorMap tm_o) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_gam0 = reinterpret_cast<float*>(sm + OFF_SMALL + SM_GAM);
  float* s_gam1 = reinterpret_cast<float*>(sm + OFF_SMALL + SM_GAM1);
  float* s_red = reinterpret_cast<float*>(sm + OFF_RED);
  float* s_p = reinterpret_cast<float*>(sm + OFF_SMALL + SM_P);
  float* s_m = reinterpret_cast<float*>(sm + OFF_SMALL + SM_M);
  float* s_h = reinterpret_cast<float*>(sm + OFF_SMALL + SM_H);
  float* s_hx = reinterpret_cast<float*>(sm + OFF_SMALL + SM_HX);
  float* s_af = reinterpret_cast<float*>(sm + OFF_AF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_SMALL + SM_BAR);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SMALL + SM_TMEM);
  volatile uint32_t* s_abort =
      reinterpret_cast<volatile uint32_t*>(sm + OFF_SMALL + SM_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, gp = warp >> 2;
  const int row = qd * 32 + lane;             // TMEM lane owned by the thread
  // dv = 256: a cluster of two CTAs per pair, each with 128 value rows (the
  // rows of S evolve independently given the chunk's key-side quantities,
  // which both CTAs form); they exchange their halves of U_down m per chunk
  const bool dv2 = a.DV == 2 * kDV;
  const int vh = dv2 ? (int)(blockIdx.x & 1) : 0;
  const int DVt = a.DV, v0 = kDV * vh;        // tensors' value width; first row here
  const int pair = dv2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int b = pair / a.H, h = pair - b * a.H;
  const int T = a.T, H = a.H, R = a.R;
  // blocks of C = min(L, 64) tokens; with C < 64 (chunks of 16, 32 or 48
  // tokens) the block is a chunk and rows C..63 of every token tile stay
  // zero, which contributes nothing to any product (see below)
  const int C = a.C;
  const int bpc = a.L / C;
  // this sequence's tokens: B sequences of T tokens, or packed sequences
  // [cu[b], cu[b + 1]) of a T-token tensor; a last block may be partial
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
  const int NB = (Tn + C - 1) / C;
  const size_t SZ = (size_t)kDV * kDK;
  const __nv_bfloat16* w_in = static_cast<const __nv_bfloat16*>(a.w);
  const __nv_bfloat16* ud = static_cast<const __nv_bfloat16*>(a.u_down);
  const __nv_bfloat16* uu = static_cast<const __nv_bfloat16*>(a.u_up);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);

  if (tid == 0) {
    if (a.tc_rec && blockIdx.x == 0) a.hdr->magic = kWsMagicTc;
    for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
    *s_abort = 0;
    mbar_init_fence();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
    prefetch_tmap(&tm_bx);
    prefetch_tmap(&tm_o);
  }
  if (C < kBlk) {
    // blocks shorter than the 64-row tiles: every token tile starts zero.
    // The copies only ever write rows 0..C-1; rows C..63 then stay zero
    // through the in-place transform (K~ = K Gamma, Q~, K^ = K / Gamma of a
    // zero row are zero; a zero log-decay leaves gamma = Gamma_{C-1}), so
    // those rows add nothing to the Grams, R, E, O or the state update.
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid; i < 32768 / 16; i += kThreads)
      *reinterpret_cast<uint4*>(sm + OFF_X + 16 * i) = z;
    // [K^; kap^] too: kap^ is formed for rows 0..C-1 only, its other rows
    // stay zero
    for (int i = tid; i < 32768 / 16; i += kThreads)
      *reinterpret_cast<uint4*>(sm + OFF_KHP + 16 * i) = z;
    for (int i = tid; i < 49152 / 16; i += kThreads)
      *reinterpret_cast<uint4*>(sm + OFF_RV + 16 * i) = z;  // RV, RG, RB
    fence_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (dv2) cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);  // lane base

  // Every barrier has at most one phase in flight.  `npar` holds the parity
  // each thread waits for next; the issuing threads also track in `pend`
  // the phases they started (copies issued, MMAs committed) so that an
  // aborting CTA drains them before it exits.
  uint32_t npar = 0, pend = 0;
  auto wait = [&](int i, uint32_t where) {
    if (tc::wait_bar(bars + i, (npar >> i) & 1u, where, s_abort, a.hdr, a.spin)) {
      npar ^= 1u << i;
      pend &= ~(1u << i);
    }
  };
  auto mark = [&](int i) { pend |= 1u << i; };

  // U_b factors: thread u = tid - 256 of warps 8-15 (r = u / 8, part = u % 8)
  // holds U_down[h][r][part + 8 i], i < 16, in registers as bf16 pairs
  // (i = 2 n, 2 n + 1 in ud_p[n]; lanes read consecutive m values); U_up[h]
  // is kept transposed in shared memory (s_uu[r][j], zero for r >= R; rows
  // kUuLd apart so that rows 4 apart fall in different banks).
  uint32_t ud_p[8];
  __nv_bfloat16* s_uu = reinterpret_cast<__nv_bfloat16*>(sm + OFF_UU);
  {
    const int r = (tid & 255) >> 3, part = tid & 7;
    const unsigned short* udr = reinterpret_cast<const unsigned short*>(ud) +
                                ((size_t)h * R + r) * DVt + v0 + part;
#pragma unroll
    for (int n = 0; n < 8; ++n)
      ud_p[n] = (warp >= 8 && r < R)
                    ? (uint32_t)udr[16 * n] | ((uint32_t)udr[16 * n + 8] << 16)
                    : 0u;
    for (int e = tid; e < kRMax * kDK; e += kThreads) {
      const int r2 = e / kDK, jj = e - r2 * kDK;
      s_uu[r2 * kUuLd + jj] = (r2 < R) ? uu[((size_t)h * kDK + jj) * R + r2]
                                       : __float2bfloat16_rn(0.f);
    }
  }

  // content gate of chunk c, on warps 8-15 (u = tid - 256): from m_c in
  // s_m (m_0 set up front, later ones formed at the previous chunk's end),
  // h = U_down m_c, s_p = U_up h.  Training records p_c, h_c and m_c for
  // the backward during the chunk's first block.
  const float invL = 1.0f / (float)a.L;
  // pieces of the chunk mean, in the rows of MY that [M; P_k] leaves once
  // MMA 2 has read it: c_O[128] (row sums of Q~ S^T + P_k W over the
  // block's tokens), eu[128] (E^T u) and u2[2][64] (column sums of P_kap
  // over each half of the tokens)
  float* s_co = reinterpret_cast<float*>(sm + OFF_MY + 8192);
  float* s_eu = s_co + 128;
  float* s_u2 = s_co + 256;
  float* s_eu2 = s_co + 384;  // E^T u over the block's tokens 32..63
  auto gate = [&](int c) {
    const int u = tid - 256;
    bar_named(6, 256);  // s_m visible to all of warps 8-15
    {
      const int r = u >> 3, part = u & 7;
      float acc = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        acc = fmaf(__uint_as_float(ud_p[n] << 16), s_m[part + 16 * n], acc);
        acc = fmaf(__uint_as_float(ud_p[n] & 0xffff0000u), s_m[part + 16 * n + 8], acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (part == 0) s_h[r] = acc;
    }
    bar_named(6, 256);
    const float* hv = s_h;
    if (dv2) {
      // send this CTA's half of h to the other CTA's slot, arrive on its
      // barrier; wait for the other half in our slot and add (double
      // buffered by chunk parity: a slot is rewritten only after its reader
      // arrived on the writer's barrier for the next chunk)
      float* slot = s_hx + 32 * (c & 1);
      if (u == 0) {
        const uint32_t peer = (uint32_t)(vh ^ 1);
        const uint32_t dst = cluster_map(slot, peer);
#pragma unroll 1
        for (int r = 0; r < 32; ++r) st_cluster_f32(dst + 4 * r, s_h[r]);
        mbar_arrive_remote(cluster_map(bars + B_X, peer));
      }
      wait(B_X, 20);
      fence_acquire_cluster();
      if (u < 32) slot[u] += s_h[u];
      bar_named(6, 256);
      hv = slot;
    }
    {  // p_j: two threads per channel j = u / 2, 16 ranks each (rank sets
       // 4 apart, so the pair reads U_up rows in different banks)
      const int jj = u >> 1, rq = u & 1;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = (i & 3) + 8 * (i >> 2) + 4 * rq;
        acc = fmaf(__bfloat162float(s_uu[r * kUuLd + jj]), hv[r], acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      if (rq == 0) s_p[jj] = acc;
    }
    bar_named(6, 256);  // p visible to all of warps 8-15
  };

  // g, b_x tiles of block ib (thread 256)
  auto issue_gb = [&](int ib) {
    const int tok = tok0 + ib * C;
    mbar_expect_tx(bars + B_GB, 2 * 2 * 128 * C);
    tma_load_3d(sm + OFF_RG, &tm_g, bars + B_GB, 0, h, tok);
    tma_load_3d(sm + OFF_RG + 8192, &tm_g, bars + B_GB, 64, h, tok);
    tma_load_3d(sm + OFF_RB, &tm_bx, bars + B_GB, 0, h, tok);
    tma_load_3d(sm + OFF_RB + 8192, &tm_bx, bars + B_GB, 64, h, tok);
    mark(B_GB);
  };
  // v tile of block ib (thread 256), into the buffer W = w V is formed in
  auto issue_v = [&](int ib) {
    const int tok = tok0 + ib * C;
    mbar_expect_tx(bars + B_V, 2 * 128 * C);
    tma_load_3d(sm + OFF_RV, &tm_v, bars + B_V, v0, h, tok);
    tma_load_3d(sm + OFF_RV + 8192, &tm_v, bars + B_V, v0 + 64, h, tok);
    mark(B_V);
  };
  // k, q, g of block ib -> L2 ahead of their loads
  auto prefetch_kqg = [&](int ib) {
    const int tok = tok0 + ib * C;
#pragma unroll 1
    for (int x = 0; x < kDK; x += 64) {
      tma_prefetch_3d(&tm_k, x, h, tok);
      tma_prefetch_3d(&tm_q, x, h, tok);
      tma_prefetch_3d(&tm_g, x, h, tok);
    }
  };
  auto issue_kq = [&](int ib) {
    const int tok = tok0 + ib * C;
    mbar_expect_tx(bars + B_KQ, 2 * 2 * 128 * C);
    tma_load_3d(sm + OFF_X, &tm_k, bars + B_KQ, 0, h, tok);
    tma_load_3d(sm + OFF_X + 16384, &tm_k, bars + B_KQ, 64, h, tok);
    tma_load_3d(sm + OFF_X + 8192, &tm_q, bars + B_KQ, 0, h, tok);
    tma_load_3d(sm + OFF_X + 16384 + 8192, &tm_q, bars + B_KQ, 64, h, tok);
    mark(B_KQ);
  };

  // key side of block nb's transform (warps 8-15): K~, Q~ in place in X,
  // K^ into its operand slot (rows 0..63 of KHP), gamma into its parity's
  // buffer; with the fused normalisation, q and k divided by their norms
  // first (exchanged through the scan buffer)
  auto keys = [&](int nb) {
    wait(B_GB, 1);
    wait(B_KQ, 2);
    const int cb = min(C, Tn - nb * C);  // tokens in block nb
    if (cb < C) {
      // a sequence ending inside the block: rows cb..C-1 of the raw k, q, g
      // tiles hold the next sequence's tokens (or the copies' zero fill
      // past the tensor) -- zeroed, so they add nothing, as in the 64-row
      // tiles of short chunks (the v rows are zeroed where W is formed)
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      const int nrow = C - cb, u = tid - 256;
      for (int i = u; i < nrow * 6 * 8; i += 256) {
        const int r = cb + i / 48, set = (i / 8) % 6, c16 = i & 7;
        // sets: K, Q rows of both column blocks in X; g of both blocks
        uint8_t* base = set < 4 ? sm + OFF_X + (set & 1) * 16384 + (set >> 1) * 8192
                                : sm + OFF_RG + (set & 1) * 8192;
        *reinterpret_cast<uint4*>(base + (r >> 3) * 1024 + (r & 7) * 128 + c16 * 16) = z;
      }
      bar_named(5, 256);
    }
    keys_w8<ACT>(sm + OFF_X, sm + OFF_KHP, sm + OFF_RG, (nb & 1) ? s_gam1 : s_gam0,
            s_red, a.dscale, cb, a.qknorm ? s_red : nullptr);
  };

  // ---- initial state: S0 -> TMEM (fp32) and the bf16 operand copy
  {
    const int c0 = gp * 32;
    const float* s0 = a.S0 ? a.S0 + ((size_t)pair * DVt + v0 + row) * kDK + c0
                           : nullptr;
    float vals[32];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      float4 x = s0 ? *reinterpret_cast<const float4*>(s0 + i)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      vals[i] = x.x; vals[i + 1] = x.y; vals[i + 2] = x.z; vals[i + 3] = x.w;
    }
    tmem_st32(tl + TM_S + c0, vals);
    // block 0's state record is the initial state (those of later blocks
    // are written at the end of the block before)
    uint8_t* rs = (a.tc_rec && NB > 0)
                      ? a.tc_rec + (size_t)pair * NB * kTcRecBytes + kTcRecS
                      : nullptr;
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      const uint32_t off = sw128_chunk(row, gp >> 1, (gp & 1) * 4 + c8, 128);
      st_chunk(sm + OFF_SB + off, vals + c8 * 8);
      if (rs) st_chunk(rs + off, vals + c8 * 8);
    }
    if (NB == 0 && a.S_T) {  // an empty sequence keeps its initial state
      float* st = a.S_T + ((size_t)pair * DVt + v0 + row) * kDK + c0;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(st + e) = make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
    }
  }
  if (tid < 128) s_m[tid] = a.m0 ? a.m0[(size_t)pair * DVt + v0 + tid] : 0.f;
  // thread 128: D1 = S [K~; Q~]^T (the block's state operand and key side)
  auto issue_d1 = [&]() {
    const uint32_t x0 = smem_u32(sm + OFF_X), sb0 = smem_u32(sm + OFF_SB);
#pragma unroll 1
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
      umma_bf16(tmem + TM_D1, desc_kmajor_sw128(sb0 + kx),
                desc_kmajor_sw128(x0 + kx), ID_N128, ks > 0);
    }
    umma_commit(bars + B_D1);
    mark(B_D1);
  };
  // warps 8-15 (thread kid of nthr = 256): kap^ = sigmoid(b_x + p) K^ of
  // block nb next to K^, then (thread 256) both Grams in one product,
  // G = [K~; Q~] [K^; kap^]^T -> [M; P_k | A; P_kap]
  auto kappa_g = [&](int nb, int kid, int nthr) {
    // short blocks: kap^ only for the block's C rows (the rest of its slot
    // was zeroed at entry); full blocks keep the 64-row loop
    tc::kappa_in_place(sm + OFF_KHP, sm + OFF_RB, s_p, 16384, kid, nthr, SHORT ? C : kBlk);
    fence_async_smem();
    bar_named(9, nthr);
    if (tid == 256 && !*s_abort) {
      tc_fence_after();
      const uint32_t x0 = smem_u32(sm + OFF_X), kh0 = smem_u32(sm + OFF_KHP);
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t kx = (ks >> 2) * 16384 + (ks & 3) * 32;
        umma_bf16(tmem + TM_G, desc_kmajor_sw128(x0 + kx),
                  desc_kmajor_sw128(kh0 + kx), ID_N128, ks > 0);
      }
      // test only: CTA 0 commits a chosen block's Grams to a barrier nobody
      // waits on, so that block's waits for them run out (the products
      // still complete and are drained before the CTA exits)
      const int bm = (nb == a.stall_block && blockIdx.x == 0) ? B_TEST : B_GK;
      umma_commit(bars + bm);
      mark(bm);
    }
  };

  if (tid == 256 && NB > 0) {
    issue_gb(0);
    issue_kq(0);
    issue_v(0);
  }
  if (tid == 32 && NB > 1) prefetch_kqg(1);
  tmem_st_wait();
  tc_fence_before();
  __syncthreads();
  // prologue: block 0's key side, chunk 0's gate, kap^ and Grams (warps 8-15)
  if (warp >= 8 && NB > 0) {
    keys(0);
    gate(0);
    kappa_g(0, tid - 256, 256);
  }

  tc_fence_before();
  __syncthreads();

  // w_t of the two token rows a thread of warps 8-15 scales in W = w V,
  // fetched one block ahead into registers (raw bf16 bits: converted only
  // when used, so the loads' latency is not waited for at issue)
  const unsigned short* w_bits = reinterpret_cast<const unsigned short*>(w_in);
  uint32_t w_lo = 0, w_hi = 0;
  if (warp >= 8) {
    const int wr = (tid - 256) >> 3, cb = min(C, Tn);
    const size_t r0 = (size_t)tok0 + wr;
    w_lo = wr < cb ? w_bits[r0 * H + h] : 0u;
    w_hi = wr + 32 < cb ? w_bits[(r0 + 32) * H + h] : 0u;
  }

  // The block loop runs in three warp groups with one CTA-wide barrier per
  // block, at its end:
  //   S (warps 0-3): [A; P_kap] -> A, P_kap; T = (I + A)^{-1}; T -> operand;
  //       MMA 3a; E^T -> operand and E^T u; MMA 3b + 4; the outputs o_t
  //   R (warps 4-7): D1 (once the block's Grams are done, so that they
  //       run first); [M; P_k] -> operand; MMA 2; R^T -> operand and the
  //       chunk-mean pieces; S <- S Diag(gamma), its bf16 operand
  //   K (warps 8-15): W = w V; S += W^T K^; the next block's key side; the
  //       chunk mean and the next chunk's gate; the next kap^ and Grams
  // Hand-offs: mbarriers for the copies and MMAs; named barriers for data
  // one group writes for another within the block (11: R -> S, 12: S, R ->
  // K; the arriving side never waits), each met once per block
  // by every thread of its groups; the end-of-block barrier orders what a
  // block leaves for the next (the rescaled S and its operand, the next key
  // side, O read out of TMEM) before the next block's MMAs read it.  A wait
  // that runs out raises the abort flag and every later wait returns at
  // once; the block still runs to its end (each group meets each of its
  // named barriers exactly once, so none can be met twice before it
  // completes), where one CTA-wide decision ends the walk.
  for (int ib = 0; ib < NB; ++ib) {
    const int t0 = ib * C;
    const bool chunk_end = ((ib + 1) % bpc) == 0 || ib == NB - 1;
    const bool more = ib + 1 < NB;
    float* s_gam = (ib & 1) ? s_gam1 : s_gam0;  // this block's gamma
    const int gr = row < 64 ? row : row - 64;  // token index of Gram row `row`
    // token-axis products: K-steps of 16 over the block's C rows only (the
    // rows past C of every token operand are zero)
    const int nks = C >> 4;

    if (warp < 4) {
      // ================= S: warps 0-3 =================
      uint8_t* rec = a.tc_rec ? a.tc_rec + ((size_t)pair * NB + ib) * kTcRecBytes
                              : nullptr;
      if (tid == 32 && ib + 2 < NB) prefetch_kqg(ib + 2);
      // ---- S1. [A; P_kap] (strictly lower): A -> fp32, P_kap -> bf16
      //      operand (both buffers were last read by this group's own
      //      inversion and by MMA 3b, which it waited for)
      wait(B_GK, 3);
      tc_fence_after();
      {
        float vals[64];  // the whole Gram row in one TMEM load
        tmem_ld64(tl + TM_GK, vals);
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e >= gr) vals[e] = 0.f;
        if (row < 64) {
#pragma unroll
          for (int e = 0; e < 64; e += 4)
            *reinterpret_cast<float4*>(s_af + fsw(row, e)) =
                make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8)
            st_chunk(sm + OFF_PQ + sw128_chunk(gr, 0, c8, 64), vals + c8 * 8);
        }
      }
      bar_named(2, 128);
      // ---- S2. T = (I + A)^{-1} in place
      unit_lower_inverse64(s_af, s_af, reinterpret_cast<float*>(sm + OFF_WS), 2, nks);
      wait(B_M2, 5);  // MMA 2 read [M; P_k]: T takes its rows of MY
      {  // T -> bf16 operand (and the record): a half row per thread
        const int tr = tid & 63, part = tid >> 6;
        float vals[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(s_af + fsw(tr, part * 32 + e));
          vals[e] = x.x; vals[e + 1] = x.y; vals[e + 2] = x.z; vals[e + 3] = x.w;
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(sm + OFF_MY + sw128_chunk(tr, 0, part * 4 + c8, 64), vals + c8 * 8);
      }
      fence_async_smem();
      tc_fence_before();
      bar_named(11, 256);  // R^T and the chunk-mean pieces from warps 4-7
      if (tid == 0 && rec) {  // T record (read before this block ends)
        bulk_store(rec + kTcRecT, sm + OFF_MY, 8192);
        bulk_commit();
      }
      // ---- S3. MMA 3a: E^T = R^T T^T; training also E = T R (lanes 0-63;
      //      the rows of MY past T only feed the unused lanes)
      if (tid == 0 && !*s_abort) {
        tc_fence_after();
        const uint32_t re0 = smem_u32(sm + OFF_RE), my0 = smem_u32(sm + OFF_MY);
#pragma unroll 1
        for (int ks = 0; ks < nks; ++ks) {
          umma_bf16(tmem + TM_D1, desc_kmajor_sw128(re0 + ks * 32),
                    desc_kmajor_sw128(my0 + ks * 32), ID_N64, ks > 0);
          if (rec)
            umma_bf16(tmem + TM_E, desc_kmajor_sw128(my0 + ks * 32),
                      desc_kmajor_sw128(re0 + ks * 32), ID_N128, ks > 0);
        }
        umma_commit(bars + B_M3);
        mark(B_M3);
      }
      wait(B_M3, 7);
      tc_fence_after();
      {  // E^T columns 0..31 -> bf16 operand (negated by the MMAs that use
         // it) and their share of E^T u; warps 4-7 take columns 32..63
        float vals[32];
        tmem_ld32(tl + TM_D1, vals);
        float eu = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) eu = fmaf(vals[e], s_u2[e] + s_u2[64 + e], eu);
        s_eu[row] = eu;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(sm + OFF_RE + sw128_chunk(row, 0, c8, 128), vals + c8 * 8);
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive_named(12, 512);  // E^T u (first half) -> warps 8-15
      bar_named(13, 256);         // -E^T complete (warps 4-7 wrote the rest)
      // ---- S4. MMA 3b: O^T -= E^T P_kap^T; MMA 4: S -= E^T kap^ (after
      //      S += W^T K^)
      wait(B_WK, 11);
      if (tid == 0 && !*s_abort) {
        tc_fence_after();
        const uint32_t kp0 = smem_u32(sm + OFF_KHP) + 8192;
        const uint32_t re0 = smem_u32(sm + OFF_RE), pq0 = smem_u32(sm + OFF_PQ);
#pragma unroll 1
        for (int ks = 0; ks < nks; ++ks) {
          umma_bf16(tmem + TM_D1 + 64, desc_kmajor_sw128(re0 + ks * 32),
                    desc_kmajor_sw128(pq0 + ks * 32), ID_N64_NA, 1);
          umma_bf16(tmem + TM_S, desc_kmajor_sw128(re0 + ks * 32),
                    desc_mnmajor_sw128(kp0 + ks * 2048, 16384), ID_BMN_NA, 1);
        }
        umma_commit(bars + B_M4);
        mark(B_M4);
      }
      wait(B_M4, 8);
      tc_fence_after();
      // ---- S5. outputs o_t (a value row per thread, 64 tokens).  A whole
      //      block goes out as one tile: O [t][v] in bf16 over the dead
      //      P_kap and scratch buffers (the 128-byte-swizzled image of two
      //      64-column boxes), then one tensor store per box; a block cut
      //      short by the sequence's end stores its live tokens directly
      const int nlive_blk = min(C, Tn - t0);
      if (nlive_blk == C) {
        float vals[64];
        tmem_ld64(tl + TM_D1 + 64, vals);
        uint8_t* ot = sm + OFF_PQ;
        // bf16 pairs of neighbouring value rows, one 32-bit store each: for
        // tokens (2u, 2u + 1) the even lane of a lane pair writes token 2u
        // and the odd lane token 2u + 1, after one shuffle (rows past C of
        // a short chunk are zero and stay in the tile unread)
        const bool odd = (lane & 1) != 0;
        const int vrow = row & ~1;
#pragma unroll
        for (int t = 0; t < 64; t += 2) {
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? vals[t] : vals[t + 1], 1);
          const uint32_t w = odd ? pack2(recv, vals[t + 1]) : pack2(vals[t], recv);
          *reinterpret_cast<uint32_t*>(ot + sw128_off(t + (odd ? 1 : 0), vrow, 64)) = w;
        }
        fence_async_smem();
        bar_named(2, 128);
        if (tid == 0) {
          tma_store_3d(&tm_o, ot, v0, h, tok0 + t0);
          tma_store_3d(&tm_o, ot + 8192, v0 + 64, h, tok0 + t0);
          bulk_commit();
        }
      } else {
#pragma unroll 1
        for (int g4 = 0; g4 < 4; ++g4) {  // tokens 16 g4 .. 16 g4 + 15
          float vals[16];
          tmem_ld16(tl + TM_D1 + 64 + g4 * 16, vals);
          // bf16 pairs of neighbouring value rows: for tokens (2u, 2u + 1)
          // the even lane of a lane pair stores token 2u and the odd lane
          // token 2u + 1, after one shuffle
          const bool odd = (lane & 1) != 0;
          __nv_bfloat16* orow = o + ((size_t)tok0 + t0 + g4 * 16 + (odd ? 1 : 0)) * H * DVt +
                                (size_t)h * DVt + v0 + (row & ~1);
          const int nlive = nlive_blk - g4 * 16 - (odd ? 1 : 0);  // this lane's tokens
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float recv = __shfl_xor_sync(0xffffffffu, odd ? vals[e] : vals[e + 1], 1);
            if (e < nlive)
              *reinterpret_cast<__nv_bfloat162*>(orow + (size_t)e * H * DVt) =
                  odd ? __floats2bfloat162_rn(recv, vals[e + 1])
                      : __floats2bfloat162_rn(vals[e], recv);
          }
        }
      }
      tc_fence_before();
      // the tile, T and E copies have read their shared memory before the
      // next block rewrites it
      if (tid == 0) bulk_wait_read_all();
    } else if (warp < 8) {
      // ================= R: warps 4-7 =================
      // ---- R1. D1 = S [K~; Q~]^T, issued after the Grams (the chain's
      //      next step) have run; [M; P_k] (strictly lower) -> bf16 operand
      //      in MY (the previous block's MMA 3a, waited for there, read T);
      //      MMA 2 (after D1, and once W is formed)
      wait(B_GK, 3);
      tc_fence_after();
      if (tid == 128 && !*s_abort) issue_d1();
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        float vals[32];
        tmem_ld32(tl + TM_GM + part * 32, vals);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (part * 32 + e >= gr) vals[e] = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(sm + OFF_MY + sw128_chunk(row, 0, part * 4 + c8, 128),
                   vals + c8 * 8);
      }
      fence_async_smem();
      tc_fence_before();
      bar_named(1, 128);
      wait(B_WK, 12);  // W = w V formed (and S += W^T K^ issued after it)
      wait(B_D1, 15);  // MMA 2 accumulates onto D1
      if (tid == 128 && !*s_abort) {
        tc_fence_after();
        const uint32_t w0 = smem_u32(sm + OFF_RV), my0 = smem_u32(sm + OFF_MY);
#pragma unroll 1
        for (int ks = 0; ks < nks; ++ks)
          umma_bf16(tmem + TM_D1, desc_mnmajor_sw128(w0 + ks * 2048, 8192),
                    desc_kmajor_sw128(my0 + ks * 32), ID_AMN, 1);
        umma_commit(bars + B_M2);
        mark(B_M2);
      }
      wait(B_M2, 4);  // [M; P_k] consumed, R^T complete
      tc_fence_after();
      // ---- R2. R^T -> bf16 operand (RE was read by the previous block's
      //      MMA 3b/4, which this group waited for); the pieces of the chunk
      //      mean: with u_i = sum_t P_kap[t][i], sum_t o_t =
      //      sum_t (Q~ S^T + P_k W)[t] - E^T u
      {
        float co = 0.f;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          float vals[32];
          tmem_ld32(tl + TM_D1 + part * 32, vals);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            st_chunk(sm + OFF_RE + sw128_chunk(row, 0, part * 4 + c8, 128),
                     vals + c8 * 8);
          tmem_ld32(tl + TM_D1 + 64 + part * 32, vals);
#pragma unroll
          for (int e = 0; e < 32; ++e) co += vals[e];
          if (qd >= 2) {  // the P_kap rows (lanes 64..127): half of u each
            tmem_ld32(tl + TM_GK + part * 32, vals);
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (part * 32 + e >= gr) vals[e] = 0.f;  // strictly lower
            s_u2[(qd - 2) * 64 + part * 32 + lane] = tc::warp_reduce_scatter32(vals, lane);
          }
        }
        s_co[row] = co;
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive_named(11, 256);  // R^T, u -> warps 0-3
      wait(B_M3, 17);  // MMA 3a: MY free for the next block; E formed
      tc_fence_after();
      {  // E^T columns 32..63 -> bf16 operand and their share of E^T u
        float vals[32];
        tmem_ld32(tl + TM_D1 + 32, vals);
        float eu = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) eu = fmaf(vals[e], s_u2[32 + e] + s_u2[96 + e], eu);
        s_eu2[row] = eu;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk(sm + OFF_RE + sw128_chunk(row, 0, 4 + c8, 128), vals + c8 * 8);
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive_named(13, 256);  // -E^T second half -> warps 0-3
      bar_arrive_named(12, 512);  // c_O, E^T u (second half) -> warps 8-15
      if (a.tc_rec) {
        // training: E [t][v] (K-major, the backward's operand layout) ->
        // the A buffer (T was read from it before MMA 3a) -> the record
        // (lanes 0-63 of TMEM hold E: warps 4 and 5)
        if (row < 64) {
          tc_fence_after();
#pragma unroll 1
          for (int pc = 0; pc < 4; ++pc) {
            float vals[32];
            tmem_ld32(tl + TM_E + pc * 32, vals);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8)
              st_chunk(sm + OFF_AF + sw128_chunk(row, pc >> 1, (pc & 1) * 4 + c8, 64),
                       vals + c8 * 8);
          }
        }
        fence_async_smem();
        bar_named(1, 128);
        if (tid == 128) {
          bulk_store(a.tc_rec + ((size_t)pair * NB + ib) * kTcRecBytes + kTcRecE,
                     sm + OFF_AF, 16384);
          bulk_commit();
        }
      }
      // ---- R3. S <- S Diag(gamma) (a value row per thread), its bf16
      //      operand (SB was read by this block's D1) and, in training, the
      //      next block's state record; the final state
      wait(B_M4, 18);
      tc_fence_after();
      {
        float* ck = (a.ck_S && !more) ? a.ck_S + (size_t)pair * SZ + (size_t)row * kDK
                                      : nullptr;
        float* st = (a.S_T && !more) ? a.S_T + ((size_t)pair * DVt + v0 + row) * kDK
                                     : nullptr;
#pragma unroll 1
        for (int c0 = 0; c0 < kDK; c0 += 32) {
          float sv[32];
          tmem_ld32(tl + TM_S + c0, sv);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 gm = *reinterpret_cast<const float4*>(s_gam + c0 + e);
            sv[e] *= gm.x; sv[e + 1] *= gm.y; sv[e + 2] *= gm.z; sv[e + 3] *= gm.w;
          }
          tmem_st32(tl + TM_S + c0, sv);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            st_chunk(sm + OFF_SB + sw128_chunk(row, c0 >> 6, ((c0 >> 5) & 1) * 4 + c8, 128),
                     sv + c8 * 8);
          }
          // fp32 checkpoint: the final state only, one slot per pair (the
          // backward of this family reads the bf16 records; the fp32 state
          // ends dlog gamma of the last block)
          if (ck) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(ck + c0 + e) =
                  make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
          }
          if (st) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(st + c0 + e) =
                  make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
          }
        }
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      if (a.tc_rec && more) {  // the next block's state record: the new operand
        bar_named(1, 128);
        if (tid == 128) {
          bulk_store(a.tc_rec + ((size_t)pair * NB + ib + 1) * kTcRecBytes + kTcRecS,
                     sm + OFF_SB, 32768);
          bulk_commit();
        }
      }
      if (tid == 128 && a.tc_rec) bulk_wait_read_all();  // SB, the A buffer are rewritten next block
    } else {
      // ================= K: warps 8-15 =================
      const int u = tid - 256;
      // ---- K1. W = w V in place over the v tile (rows past the block's
      //      tokens: zero); then thread 256 issues S += W^T K^ (warps 4-7
      //      rescaled the state before the previous block ended) and
      //      requests the next g, b_x tiles (g was read by the key
      //      transform, b_x by kap^)
      wait(B_V, 19);
      {
        const int rr = u >> 3, ch = u & 7;  // token rows rr, rr + 32; 16-byte chunk
        const int cb = min(C, Tn - t0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rr + 32 * (i & 1), kb = i >> 1;
          const uint32_t off = (uint32_t)(kb * 8192 + (r >> 3) * 1024 +
                                          (r & 7) * 128 + ch * 16);
          const uint4 x = *reinterpret_cast<const uint4*>(sm + OFF_RV + off);
          const float wt = __uint_as_float(((i & 1) ? w_hi : w_lo) << 16);
          const __nv_bfloat162* xv = reinterpret_cast<const __nv_bfloat162*>(&x);
          uint4 y = make_uint4(0u, 0u, 0u, 0u);
          if (r < cb) {
            uint32_t* yv = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(xv[e]);
              yv[e] = pack2(f.x * wt, f.y * wt);
            }
          }
          *reinterpret_cast<uint4*>(sm + OFF_RV + off) = y;
        }
        if (more) {  // the next block's w_t (0 past the block's tokens)
          const int cn = min(C, Tn - (ib + 1) * C);
          const size_t r0 = (size_t)tok0 + (ib + 1) * C + rr;
          w_lo = rr < cn ? w_bits[r0 * H + h] : 0u;
          w_hi = rr + 32 < cn ? w_bits[(r0 + 32) * H + h] : 0u;
        }
      }
      fence_async_smem();
      bar_named(8, 256);
      if (tid == 256 && !*s_abort) {
        tc_fence_after();
        const uint32_t w0 = smem_u32(sm + OFF_RV), kh0 = smem_u32(sm + OFF_KHP);
#pragma unroll 1
        for (int ks = 0; ks < nks; ++ks)
          umma_bf16(tmem + TM_S, desc_mnmajor_sw128(w0 + ks * 2048, 8192),
                    desc_mnmajor_sw128(kh0 + ks * 2048, 16384), ID_AMN_BMN, 1);
        umma_commit(bars + B_WK);
        mark(B_WK);
        if (more) issue_gb(ib + 1);
      }
      // ---- K2. the next block's key side: X is free once the Grams and
      //      D1 have read it (thread 256 then requests the next k, q tiles
      //      into it), K^'s slot once S += W^T K^ has
      wait(B_GK, 3);
      wait(B_D1, 16);
      if (tid == 256 && more && !*s_abort) issue_kq(ib + 1);
      if (gp == 3 && a.gin && ib % bpc == 0) {
        // warps 12-15: the chunk's gate records for the backward (p_c, h_c,
        // m_c: s_p, s_h, s_m hold them until the chunk's end)
        const int uu3 = tid - 384, c = ib / bpc;
        a.gin[((size_t)pair * a.NC + c) * (kDK + R) + uu3] = s_p[uu3];
        if (uu3 < R) a.gin[((size_t)pair * a.NC + c) * (kDK + R) + kDK + uu3] = s_h[uu3];
        if (a.ck_m) a.ck_m[((size_t)pair * a.NC + c) * kDV + uu3] = s_m[uu3];
      }
      wait(B_WK, 12);
      if (more) keys(ib + 1);
      wait(B_M2, 20);  // MMA 2 read W: its buffer takes the next v tile
      if (tid == 256 && more && !*s_abort) issue_v(ib + 1);
      // ---- K3. the block's sum of o and, at a chunk's end, its mean
      //      m_{c+1} and the next chunk's gate p = U_up U_down m_{c+1}
      bar_named(12, 512);  // c_O (warps 4-7), E^T u (warps 0-3)
      if (u < 128) {
        const float bs = s_co[u] - (s_eu[u] + s_eu2[u]);
        const float acc = (ib % bpc == 0) ? bs : s_m[u] + bs;
        s_m[u] = chunk_end ? acc * invL : acc;
      }
      if (chunk_end && more) gate(ib / bpc + 1);
      // ---- K4. the next block's kap^ (its slot was read by MMA 4), then
      //      the next Grams
      wait(B_M4, 21);
      if (more) kappa_g(ib + 1, tid - 256, 256);
    }
    tc_fence_before();
    if (__syncthreads_or(*s_abort)) break;  // one decision for all threads
    tc_fence_after();
  }
  tc_fence_before();
  __syncthreads();

  if (*s_abort) {
    if (tid == 0 || tid == 128 || tid == 256)  // the threads that start copies and MMAs
      for (int i = 0; i < kNumBars; ++i)
        if ((pend >> i) & 1u) tc::drain_bar(bars + i, (npar >> i) & 1u);
  } else if (a.m_T && tid < 128) {  // the last chunk's mean
    a.m_T[(size_t)pair * DVt + v0 + tid] = s_m[tid];
  }
  if (tid == 0 || tid == 128) bulk_wait_all();  // output tiles and records written
  tc_fence_before();
  __syncthreads();
  // neither CTA of a pair leaves while the other may still write to it
  if (dv2) cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

// [B*T, H, D] bf16 tensor viewed as 3-D (D innermost); boxes of
// 64 x 1 x box_rows (the block's C tokens) with the 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int D, int H, long long rows,
              int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_fwd_supported(const carve_shape& s, bool training) {
  return tc_fwd_shape(s, training);
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mg, mb, mo;
  const long long rows = a.cu ? (long long)a.T : (long long)a.B * a.T;
  const bool dv2 = a.DV == 2 * kDV;
  if (dv2 && (a.ck_S || a.tc_rec)) return cudaErrorInvalidValue;  // inference only
  const int C = a.C;
  if (C < 16 || C > kBlk || C % 16 || (C < kBlk && (a.ck_S || a.tc_rec)))
    return cudaErrorInvalidValue;  // training: blocks of 64 only
  if (!make_map(&mq, a.q, kDK, a.H, rows, C) || !make_map(&mk, a.k, kDK, a.H, rows, C) ||
      !make_map(&mv, a.v, a.DV, a.H, rows, C) || !make_map(&mg, a.g, kDK, a.H, rows, C) ||
      !make_map(&mb, a.bx, kDK, a.H, rows, C) || !make_map(&mo, a.o, a.DV, a.H, rows, C))
    return cudaErrorInvalidValue;
  // instances: the fused decay activation or not, and blocks shorter than
  // 64 tokens (chunks of 16, 32, 48) or not, chosen here
  const bool act = a.dscale > 0.f, sh = C < kBlk;
  auto kern = act ? (sh ? fwd_tc_kernel<true, true> : fwd_tc_kernel<true, false>)
                  : (sh ? fwd_tc_kernel<false, true> : fwd_tc_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  if (!dv2) {
    kern<<<a.B * a.H, kThreads, kSmemBytes, st>>>(a, mq, mk, mv, mg, mb, mo);
    return cudaGetLastError();
  }
  // dv = 256: clusters of two CTAs, one per value half
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.B * a.H);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, mq, mk, mv, mg, mb, mo);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace carve
