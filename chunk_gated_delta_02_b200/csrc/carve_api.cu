// carve_api.cu -- the C ABI of libcarve: validation, workspace layout and
// kernel dispatch.  Declared in include/carve.h.
#include <stdlib.h>
#include <string.h>

#include "carve_internal.cuh"

using namespace carve;

namespace carve {

// The supported-shape check every entry point applies first (declared in
// carve_internal.cuh so that the allocation-free entry point shares it).
carve_status check_shape(const carve_shape* s) {
  if (!s) return CARVE_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->T < 0 || s->R < 0 || s->L < 1 ||
      s->DK < 1 || s->DV < 1)
    return CARVE_ERR_INVALID_ARG;
  if (s->dtype != CARVE_BF16 && s->dtype != CARVE_FP32)
    return CARVE_ERR_INVALID_ARG;
  if (!(s->decay_scale >= 0.f) || s->decay_scale > 3.0e38f)  // NaN, < 0, inf
    return CARVE_ERR_INVALID_ARG;
  if (s->qk_l2norm != 0 && s->qk_l2norm != 1) return CARVE_ERR_INVALID_ARG;
  if (s->erase_form != 0 && s->erase_form != 1) return CARVE_ERR_INVALID_ARG;
  if (s->DK % 16 || s->DV % 16 || s->DK > 256 || s->DV > 256)
    return CARVE_ERR_UNSUPPORTED;
  if (s->R > kMaxR) return CARVE_ERR_UNSUPPORTED;
  if (!(s->L <= kMaxBlock || (s->L % kMaxBlock == 0 && s->L <= 256)))
    return CARVE_ERR_UNSUPPORTED;
  // all element indices are computed in 64-bit; grid is B*H CTAs
  if ((long long)s->B * s->H > (1LL << 30)) return CARVE_ERR_UNSUPPORTED;
  const int C = block_len(s->L);
  if (generic_bwd_smem_bytes(C, s->DK, s->DV) > 227 * 1024)
    return CARVE_ERR_UNSUPPORTED;
  return CARVE_OK;
}

// Test-only knobs, read from the environment on every call (unset in
// normal use): CARVE_TEST_WAIT_CYCLES lowers the cycles a device-side wait
// spins before it gives up; CARVE_TEST_STALL_BLOCK makes CTA 0 of the
// tensor-core kernels redirect the MMA commit of that block to a barrier
// nobody waits on, so that a wait runs out and the timeout path runs (in
// the decode step, any value >= 0 makes CTA 0 issue none of its first
// group of copies).
void test_knobs(long long* spin, int* stall_block) {
  *spin = kSpinCycles;
  *stall_block = -1;
  if (const char* e = getenv("CARVE_TEST_WAIT_CYCLES")) {
    const long long v = atoll(e);
    if (v > 0 && v < kSpinCycles) *spin = v;
  }
  if (const char* e = getenv("CARVE_TEST_STALL_BLOCK")) *stall_block = atoi(e);
}

}  // namespace carve

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

// Forward kernel family for a valid shape: the tensor-core kernel where it
// applies, else the generic one.  CARVE_FWD_PATH=generic forces the generic
// kernel (both are GPU kernels; used to cross-check the two paths).
bool use_tc_fwd(const carve_shape& s, bool training) {
  const char* env = getenv("CARVE_FWD_PATH");
  if (env && strcmp(env, "generic") == 0) return false;
  return tc_fwd_supported(s, training);
}
bool opt_ptr_ok(const void* p) { return p == nullptr || aligned16(p); }

// Backward kernel family: tensor-core where the tensor-core forward ran (it
// reads that forward's records); CARVE_BWD_PATH=generic forces the generic
// one, which reads the generic forward's per-block fp32 checkpoints (a
// tensor-core workspace has none and is refused).
bool use_tc_bwd(const carve_shape& s) {
  const char* env = getenv("CARVE_BWD_PATH");
  if (env && strcmp(env, "generic") == 0) return false;
  return use_tc_fwd(s, true);
}

}  // namespace

extern "C" {

size_t carve_workspace_bytes(const carve_shape* shape, int training) {
  if (check_shape(shape) != CARVE_OK) return 0;
  if (training && shape->T % shape->L) return 0;  // training: whole chunks
  return ws_layout(*shape, training != 0, use_tc_fwd(*shape, training != 0))
      .total;
}

const char* carve_status_str(carve_status s) {
  switch (s) {
    case CARVE_OK: return "CARVE_OK";
    case CARVE_ERR_INVALID_ARG: return "CARVE_ERR_INVALID_ARG";
    case CARVE_ERR_UNSUPPORTED: return "CARVE_ERR_UNSUPPORTED";
    case CARVE_ERR_WORKSPACE: return "CARVE_ERR_WORKSPACE";
    case CARVE_ERR_CUDA: return "CARVE_ERR_CUDA";
    case CARVE_ERR_TIMEOUT: return "CARVE_ERR_TIMEOUT";
  }
  return "CARVE_ERR_UNKNOWN";
}

const char* carve_fwd_path(const carve_shape* shape) {
  if (check_shape(shape) != CARVE_OK) return nullptr;
  return use_tc_fwd(*shape, false) ? "tc" : "generic";
}

carve_status carve_chunk_fwd(const carve_shape* shape, const void* q,
                             const void* k, const void* v, const void* g,
                             const void* b_x, const void* w,
                             const void* u_down, const void* u_up,
                             const float* S0, const float* m0, void* o,
                             float* S_T, float* m_T, void* workspace,
                             size_t workspace_bytes, int training,
                             void* stream) {
  carve_status st = check_shape(shape);
  if (st != CARVE_OK) return st;
  const carve_shape& s = *shape;
  if (training && s.T % s.L) return CARVE_ERR_UNSUPPORTED;
  const bool tok = s.T > 0;
  if (tok && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) ||
              !ptr_ok(b_x) || !ptr_ok(w) || !ptr_ok(o)))
    return CARVE_ERR_INVALID_ARG;
  if (s.R > 0 && (!ptr_ok(u_down) || !ptr_ok(u_up)))
    return CARVE_ERR_INVALID_ARG;
  if (!opt_ptr_ok(S0) || !opt_ptr_ok(m0) || !opt_ptr_ok(S_T) ||
      !opt_ptr_ok(m_T))
    return CARVE_ERR_INVALID_ARG;
  const bool tc = use_tc_fwd(s, training != 0);
  const WsLayout L = ws_layout(s, training != 0, tc);
  if (!workspace || !aligned16(workspace)) return CARVE_ERR_WORKSPACE;
  if (workspace_bytes < L.total) return CARVE_ERR_WORKSPACE;

  char* ws = (char*)workspace;
  FwdArgs a{};
  a.B = s.B; a.T = s.T; a.H = s.H; a.DK = s.DK; a.DV = s.DV; a.R = s.R;
  a.L = s.L; a.C = L.C; a.NB = L.NB; a.NC = L.NC;
  a.q = q; a.k = k; a.v = v; a.g = g; a.bx = b_x; a.w = w;
  a.u_down = u_down; a.u_up = u_up; a.S0 = S0; a.m0 = m0;
  a.o = o; a.S_T = S_T; a.m_T = m_T;
  a.ck_S = training ? (float*)(ws + L.ck_S) : nullptr;
  a.ck_m = training ? (float*)(ws + L.ck_m) : nullptr;
  a.scratch = (float*)(ws + L.scratch);
  a.scratch_per_pair = L.scratch_per_pair;
  a.tc_rec = training && L.tc_rec ? (uint8_t*)(ws + L.tc_rec) : nullptr;
  a.gin = training && L.gin ? (float*)(ws + L.gin) : nullptr;
  a.hdr = (WsHeader*)ws;
  a.dscale = s.decay_scale;
  a.qknorm = s.qk_l2norm;
  a.erase = s.erase_form;
  test_knobs(&a.spin, &a.stall_block);
  cudaError_t e = tc ? launch_fwd_tc(a, (cudaStream_t)stream)
                      : launch_fwd_generic(a, s.dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

carve_status carve_chunk_fwd_varlen(
    const carve_shape* shape, const int32_t* cu_seqlens, const void* q,
    const void* k, const void* v, const void* g, const void* b_x,
    const void* w, const void* u_down, const void* u_up, const float* S0,
    const float* m0, void* o, float* S_T, float* m_T, void* workspace,
    size_t workspace_bytes, void* stream) {
  carve_status st = check_shape(shape);
  if (st != CARVE_OK) return st;
  const carve_shape& s = *shape;
  if (!ptr_ok(cu_seqlens)) return CARVE_ERR_INVALID_ARG;
  const bool tok = s.T > 0;
  if (tok && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) ||
              !ptr_ok(b_x) || !ptr_ok(w) || !ptr_ok(o)))
    return CARVE_ERR_INVALID_ARG;
  if (s.R > 0 && (!ptr_ok(u_down) || !ptr_ok(u_up)))
    return CARVE_ERR_INVALID_ARG;
  if (!opt_ptr_ok(S0) || !opt_ptr_ok(m0) || !opt_ptr_ok(S_T) ||
      !opt_ptr_ok(m_T))
    return CARVE_ERR_INVALID_ARG;
  const bool tc = use_tc_fwd(s, false);
  const WsLayout L = ws_layout(s, false, tc);
  if (!workspace || !aligned16(workspace)) return CARVE_ERR_WORKSPACE;
  if (workspace_bytes < L.total) return CARVE_ERR_WORKSPACE;
  char* ws = (char*)workspace;
  FwdArgs a{};
  a.B = s.B; a.T = s.T; a.H = s.H; a.DK = s.DK; a.DV = s.DV; a.R = s.R;
  a.L = s.L; a.C = L.C; a.NB = L.NB; a.NC = L.NC;
  a.q = q; a.k = k; a.v = v; a.g = g; a.bx = b_x; a.w = w;
  a.u_down = u_down; a.u_up = u_up; a.S0 = S0; a.m0 = m0;
  a.o = o; a.S_T = S_T; a.m_T = m_T;
  a.scratch = (float*)(ws + L.scratch);
  a.scratch_per_pair = L.scratch_per_pair;
  a.hdr = (WsHeader*)ws;
  a.dscale = s.decay_scale;
  a.qknorm = s.qk_l2norm;
  a.erase = s.erase_form;
  a.cu = cu_seqlens;
  test_knobs(&a.spin, &a.stall_block);
  cudaError_t e = tc ? launch_fwd_tc(a, (cudaStream_t)stream)
                     : launch_fwd_generic(a, s.dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

carve_status carve_chunk_bwd(const carve_shape* shape, const void* q,
                             const void* k, const void* v, const void* g,
                             const void* b_x, const void* w,
                             const void* u_down, const void* u_up,
                             const void* d_o, const float* dS_T,
                             const float* dm_T, void* workspace,
                             size_t workspace_bytes, void* dq, void* dk,
                             void* dv, void* dg, void* db_x, void* dw,
                             float* du_down, float* du_up, float* dS0,
                             float* dm0, void* stream) {
  carve_status st = check_shape(shape);
  if (st != CARVE_OK) return st;
  const carve_shape& s = *shape;
  if (s.T % s.L) return CARVE_ERR_UNSUPPORTED;  // training: whole chunks
  const bool tok = s.T > 0;
  if (tok && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) ||
              !ptr_ok(b_x) || !ptr_ok(w) || !ptr_ok(d_o) || !ptr_ok(dq) ||
              !ptr_ok(dk) || !ptr_ok(dv) || !ptr_ok(dg) || !ptr_ok(db_x) ||
              !ptr_ok(dw)))
    return CARVE_ERR_INVALID_ARG;
  if (s.R > 0 && (!ptr_ok(u_down) || !ptr_ok(u_up) || !ptr_ok(du_down) ||
                  !ptr_ok(du_up)))
    return CARVE_ERR_INVALID_ARG;
  if (!opt_ptr_ok(dS_T) || !opt_ptr_ok(dm_T) || !opt_ptr_ok(dS0) ||
      !opt_ptr_ok(dm0))
    return CARVE_ERR_INVALID_ARG;
  // the workspace layout of the forward family this backward reads (a
  // tensor-core workspace is too small for the generic backward's layout:
  // that mismatch is refused here)
  const bool tc = use_tc_bwd(s);
  const WsLayout L = ws_layout(s, true, tc);
  if (!workspace || !aligned16(workspace)) return CARVE_ERR_WORKSPACE;
  if (workspace_bytes < L.total) return CARVE_ERR_WORKSPACE;

  char* ws = (char*)workspace;
  BwdArgs a{};
  a.B = s.B; a.T = s.T; a.H = s.H; a.DK = s.DK; a.DV = s.DV; a.R = s.R;
  a.L = s.L; a.C = L.C; a.NB = L.NB; a.NC = L.NC;
  a.q = q; a.k = k; a.v = v; a.g = g; a.bx = b_x; a.w = w;
  a.u_down = u_down; a.u_up = u_up; a.d_o = d_o; a.dS_T = dS_T; a.dm_T = dm_T;
  a.ck_S = (const float*)(ws + L.ck_S);
  a.ck_m = (const float*)(ws + L.ck_m);
  a.scratch = (float*)(ws + L.scratch);
  a.scratch_per_pair = L.scratch_per_pair;
  a.du = (float*)(ws + L.du);
  a.tc_rec = L.tc_rec ? (const uint8_t*)(ws + L.tc_rec) : nullptr;
  a.gin = L.gin ? (const float*)(ws + L.gin) : nullptr;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbx = db_x; a.dw = dw;
  a.du_down = du_down; a.du_up = du_up; a.dS0 = dS0; a.dm0 = dm0;
  a.hdr = (WsHeader*)ws;
  a.dscale = s.decay_scale;
  a.qknorm = s.qk_l2norm;
  a.erase = s.erase_form;
  test_knobs(&a.spin, &a.stall_block);
  cudaError_t e = tc ? launch_bwd_tc(a, (cudaStream_t)stream)
                      : launch_bwd_generic(a, s.dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}

carve_status carve_decode_step(const carve_shape* shape, const void* q,
                               const void* k, const void* v, const void* g,
                               const void* b_x, const void* w,
                               const void* u_down, const void* u_up,
                               const int32_t* pos, float* S, float* m,
                               float* osum, void* o, void* stream) {
  if (!shape) return CARVE_ERR_INVALID_ARG;
  carve_shape s = *shape;
  s.T = 0;  // one token per call: the sequence length plays no part
  carve_status st = check_shape(&s);
  if (st != CARVE_OK) return st;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(b_x) ||
      !ptr_ok(w) || !ptr_ok(pos) || !ptr_ok(S) || !ptr_ok(m) ||
      !ptr_ok(osum) || !ptr_ok(o))
    return CARVE_ERR_INVALID_ARG;
  if (s.R > 0 && (!ptr_ok(u_down) || !ptr_ok(u_up)))
    return CARVE_ERR_INVALID_ARG;
  DecArgs a{};
  a.B = s.B; a.H = s.H; a.DK = s.DK; a.DV = s.DV; a.R = s.R; a.L = s.L;
  a.q = q; a.k = k; a.v = v; a.g = g; a.bx = b_x; a.w = w;
  a.u_down = u_down; a.u_up = u_up; a.pos = pos;
  a.S = S; a.m = m; a.osum = osum; a.o = o;
  a.dscale = s.decay_scale;
  a.qknorm = s.qk_l2norm;
  a.erase = s.erase_form;
  int stall_block = -1;
  test_knobs(&a.wait_cycles, &stall_block);
  a.stall = stall_block >= 0 ? 1 : 0;
  return launch_decode(a, s.dtype, (cudaStream_t)stream) == cudaSuccess
             ? CARVE_OK
             : CARVE_ERR_CUDA;
}

carve_status carve_get_status(const void* workspace, void* stream) {
  if (!workspace) return CARVE_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost,
                      st) != cudaSuccess)
    return CARVE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CARVE_ERR_CUDA;
  return (carve_status)word;
}

carve_status carve_reset_status(void* workspace, void* stream) {
  if (!workspace) return CARVE_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), (cudaStream_t)stream) !=
      cudaSuccess)
    return CARVE_ERR_CUDA;
  return CARVE_OK;
}

}  // extern "C"
