// carve_internal.cuh -- shared definitions of libcarve's host and device code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/carve.h"

namespace carve {

constexpr uint32_t kWsMagic = 0xCA7E0001u;
constexpr size_t kHeaderBytes = 256;
constexpr int kMaxR = 64;
constexpr int kMaxBlock = 64;  // tokens per solver block (C = min(L, 64))
// Cycles a device-side wait spins before it records CARVE_ERR_TIMEOUT
// (about 1 s at the B200's clocks).
constexpr long long kSpinCycles = 1LL << 31;

// Device status word at the start of the workspace.
struct WsHeader {
  uint32_t status;   // carve_status written by kernels (sticky)
  uint32_t magic;    // which training forward wrote the checkpoints
  uint32_t where;    // diagnostic: which wait gave up
  uint32_t pad[61];
};
constexpr uint32_t kWsMagicTc = 0xCA7E7C01u;  // tensor-core forward: tc records valid

// Per-block record the tensor-core training forward leaves for the backward:
// shared-memory images (128-byte swizzled UMMA layout of a 1024-aligned
// base) of the bf16 state operand S, of E and of T = (I + A)^{-1}.
constexpr size_t kTcRecS = 0;          // S    [v 128][j 128] bf16  32 KB
constexpr size_t kTcRecE = 32768;      // E    [t 64][v 128]  bf16  16 KB (2 x 8 KB column blocks)
constexpr size_t kTcRecT = 49152;      // T    [t 64][s 64]   bf16   8 KB
constexpr size_t kTcRecBytes = 57344;

// Tensor-core kernels: bf16, DK = DV = 128, L % 64 == 0, R <= 32, T > 0
// (the training forward, whose records this describes, and the backward;
// both with or without the fused per-token q / k normalisation).
inline bool tc_shape(const carve_shape& s) {
  return s.dtype == CARVE_BF16 && s.DK == 128 && s.DV == 128 &&
         s.L % kMaxBlock == 0 && s.R <= 32 && s.T > 0 && !s.erase_form;
}
// The tensor-core forward also runs, without training, DV = 256 (two CTAs
// per pair) and chunks of 16, 32 or 48 tokens (one chunk per block, the
// 64-row tiles zero past the chunk).
inline bool tc_fwd_shape(const carve_shape& s, bool training) {
  if (tc_shape(s)) return true;
  if (training || s.erase_form) return false;
  const bool chunk_ok = s.L % kMaxBlock == 0 || (s.L < kMaxBlock && s.L % 16 == 0);
  return !training && s.dtype == CARVE_BF16 && s.DK == 128 &&
         (s.DV == 128 || s.DV == 256) && chunk_ok && s.R <= 32 && s.T > 0;
}
static_assert(sizeof(WsHeader) == kHeaderBytes, "header size");

// Layout of the workspace (byte offsets, 256-aligned).  `tc` says which
// forward family writes it (the tensor-core one keeps only what its own
// backward reads).
struct WsLayout {
  int C;    // tokens per solver block
  int NB;   // blocks per sequence
  int NC;   // chunks per sequence
  int ck_slots;        // fp32 states kept per pair: NB + 1 (generic), 1 (tc)
  size_t ck_S;         // [B*H][ck_slots][DV][DK] fp32 block-start states
  size_t ck_m;         // [B*H][NC][DV] fp32 chunk gate inputs m_c
  size_t scratch;      // per-pair fp32 scratch (generic kernels; tc: dp | dh)
  size_t scratch_per_pair;  // floats
  size_t du;           // [B*H][R*DV + DK*R] fp32 per-pair U_b gradients
  size_t tc_rec;       // [B*H][NB] tensor-core records (kTcRecBytes each)
  size_t gin;          // [B*H][NC][DK + R] fp32 chunk gate inputs p_c | h_c
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int block_len(int L) { return L < kMaxBlock ? L : kMaxBlock; }

inline size_t generic_fwd_scratch_floats(int C, int DK, int DV) {
  return 4 * (size_t)C * DK + 4 * (size_t)C * DV + (size_t)DV * DK;
}
inline size_t generic_bwd_scratch_floats(int C, int DK, int DV) {
  return 11 * (size_t)C * DK + 7 * (size_t)C * DV + 2 * (size_t)DV * DK;
}

// tc: the tensor-core forward writes this workspace.  It needs no generic
// scratch; in training it keeps the final fp32 state only (its backward
// walks the bf16 state records), the chunk gate inputs, the records, and
// scratch for the backward's per-chunk gate gradients.
inline WsLayout ws_layout(const carve_shape& s, bool training, bool tc) {
  WsLayout w{};
  w.C = block_len(s.L);
  w.NB = s.T / w.C;
  w.NC = s.T / s.L;
  w.ck_slots = tc ? 1 : w.NB + 1;
  const size_t P = (size_t)s.B * s.H;
  const size_t NCc = (size_t)(w.NC > 0 ? w.NC : 1);
  size_t off = kHeaderBytes;
  if (training) {
    w.ck_S = off;
    off = align256(off + P * (size_t)w.ck_slots * s.DV * s.DK * 4);
    w.ck_m = off;
    off = align256(off + P * NCc * s.DV * 4);
  }
  size_t sc = 0;
  if (!tc) {
    sc = generic_fwd_scratch_floats(w.C, s.DK, s.DV);
    if (training) {
      const size_t sb = generic_bwd_scratch_floats(w.C, s.DK, s.DV);
      sc = sc > sb ? sc : sb;
    }
  } else if (training) {
    sc = NCc * (s.DK + s.R);  // the backward's per-chunk gate gradients
  }
  w.scratch_per_pair = sc;
  w.scratch = off;
  off = align256(off + P * sc * 4);
  if (training) {
    w.du = off;
    off = align256(off + P * ((size_t)s.R * s.DV + (size_t)s.DK * s.R) * 4);
    if (tc) {
      w.tc_rec = off;
      off = align256(off + P * (size_t)w.NB * kTcRecBytes);
      w.gin = off;
      off = align256(off + P * NCc * (s.DK + s.R) * 4);
    }
  }
  w.total = off;
  return w;
}

// The decay activation applied to raw logits when decay_scale s > 0:
// g = -s softplus(a), softplus(a) = max(a, 0) + log1p(exp(-|a|)); s == 0
// passes g through.  Its derivative dg/da = -s sigmoid(a) is formed by the
// backward kernels from g itself: sigmoid(a) = 1 - exp(-softplus(a)) =
// -expm1(g / s).
__device__ __forceinline__ float decay_act(float a, float s) {
  return s > 0.f ? -s * (fmaxf(a, 0.f) + log1pf(expf(-fabsf(a)))) : a;
}
__device__ __forceinline__ float decay_act_grad(float g, float s) {
  return s > 0.f ? s * expm1f(g / s) : 1.f;
}
// The same over 8 values passed by value (a row at or past `valid` gets
// log-decay 0), kept out of line: the hot loops call it only under a
// uniform s > 0 branch, so neither its code nor its transcendental
// functions cost anything when the log-decay is given.
struct F8 {
  float x[8];
};
static __device__ __noinline__ F8 decay_act8(F8 v, float s, bool valid) {
#pragma unroll
  for (int e = 0; e < 8; ++e)
    v.x[e] = valid ? -s * (fmaxf(v.x[e], 0.f) + log1pf(expf(-fabsf(v.x[e])))) : 0.f;
  return v;
}
static __device__ __forceinline__ void decay_act8(float* x, float s, bool valid) {
  F8 v;
#pragma unroll
  for (int e = 0; e < 8; ++e) v.x[e] = x[e];
  v = decay_act8(v, s, valid);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = v.x[e];
}

// Element load/store in the I/O dtype, arithmetic in fp32.
__device__ __forceinline__ float ldf(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void stf(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// Arguments of the forward kernels (pointers already validated).
struct FwdArgs {
  int B, T, H, DK, DV, R, L, C, NB, NC;
  const void *q, *k, *v, *g, *bx, *w, *u_down, *u_up;
  const float *S0, *m0;
  void* o;
  float *S_T, *m_T;
  float* ck_S;     // NULL unless training
  float* ck_m;     // NULL unless training
  float* scratch;  // generic kernels only
  size_t scratch_per_pair;
  uint8_t* tc_rec;  // tensor-core records; NULL unless training
  float* gin;       // chunk gate inputs p_c | h_c; NULL unless training
  WsHeader* hdr;
  long long spin;   // cycles a device-side wait spins before it gives up
  int stall_block;  // test only: block whose MMA commit CTA 0 redirects (-1: none)
  float dscale;     // decay activation scale (0: g is the log-decay)
  int qknorm;       // 1: q, k are normalised per token inside the kernels
  int erase;        // 1: the other erase form S' (I - (b k) k^T)
  // packed sequences: B sequences at token offsets cu[b] .. cu[b + 1] of a
  // T-token tensor ([T, H, D] layouts), or NULL: B sequences of T tokens
  const int32_t* cu;
};

struct BwdArgs {
  int B, T, H, DK, DV, R, L, C, NB, NC;
  const void *q, *k, *v, *g, *bx, *w, *u_down, *u_up;
  const void* d_o;
  const float *dS_T, *dm_T;
  const float *ck_S, *ck_m;
  float* scratch;
  size_t scratch_per_pair;
  float* du;  // per-pair partial U_b gradients
  const uint8_t* tc_rec;  // records of the tensor-core forward
  const float* gin;       // its chunk gate inputs p_c | h_c
  void *dq, *dk, *dv, *dg, *dbx, *dw;
  float *du_down, *du_up, *dS0, *dm0;
  WsHeader* hdr;
  long long spin;   // cycles a device-side wait spins before it gives up
  int stall_block;  // test only: block whose MMA commit CTA 0 redirects (-1: none)
  float dscale;     // decay activation scale (0: g is the log-decay)
  int qknorm;       // 1: q, k are normalised per token inside the kernels
  int erase;        // 1: the other erase form S' (I - (b k) k^T)
};

// Arguments of the decode step (one token per (sequence, head)).
struct DecArgs {
  int B, H, DK, DV, R, L;
  const void *q, *k, *v, *g, *bx, *w, *u_down, *u_up;  // [B, H, D] one token
  const int32_t* pos;  // [B] tokens already processed per sequence
  float *S, *m, *osum;  // [B, H, DV, DK], [B, H, DV], [B, H, DV] in/out
  void* o;              // [B, H, DV]
  float dscale;         // decay activation scale (0: g is the log-decay)
  int qknorm;           // 1: q, k are normalised inside the kernel
  int erase;            // 1: the other erase form S' (I - (b k) k^T)
  long long wait_cycles;  // a copy wait gives up after this many cycles
  int stall;            // test only: CTA 0 issues none of its first copies
};
cudaError_t launch_decode(const DecArgs& a, int dtype, cudaStream_t st);

// Host-side checks (carve_api.cu): the supported-shape check of every entry
// point, and the test-only wait limit / stall knobs.
carve_status check_shape(const carve_shape* s);
void test_knobs(long long* spin, int* stall_block);

// Host launchers (carve_generic.cu).
cudaError_t launch_fwd_generic(const FwdArgs& a, int dtype, cudaStream_t st);
cudaError_t launch_bwd_generic(const BwdArgs& a, int dtype, cudaStream_t st);
size_t generic_fwd_smem_bytes(int C, int DK, int DV);

// Tensor-core forward (carve_tc_fwd.cu): see tc_fwd_shape.
bool tc_fwd_supported(const carve_shape& s, bool training);
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t st);

// Tensor-core backward (carve_tc_bwd.cu), same shapes as the forward; it
// reads the tensor-core forward's records.  Its per-chunk gate gradients
// (B*H*NC*(DK + R) floats: dp | dh) live in the scratch area.
size_t tc_bwd_gate_record_floats(const carve_shape& s);
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st);
size_t generic_bwd_smem_bytes(int C, int DK, int DV);

}  // namespace carve
