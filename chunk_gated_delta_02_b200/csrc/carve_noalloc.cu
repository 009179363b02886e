// carve_noalloc.cu -- carve_chunk_fwd_noalloc, a forward entry point that
// allocates nothing and takes no workspace.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they
// run the recurrence -- a plugin that a host framework hands only its input
// and output tensors (the framework owns every device allocation), a
// stream-ordered section where cudaMalloc's implicit device-wide
// synchronisation would stall other streams, or a real-time loop that must
// stay inside a fixed memory budget.  Everything else should use
// carve_chunk_fwd with a caller-owned workspace.
//
// How: the generic forward kernel runs with its per-(sequence, head)
// scratch placed in the file-scope device array below instead of a
// workspace.  The array is part of the library's device image, so every
// GPU that loads libcarve holds CARVE_NOALLOC_SCRATCH_BYTES of it until the
// process exits.  Its device address is looked up on every call, with the
// caller's device current (a host-side query that allocates nothing; a
// pointer cached across calls could outlive a device reset).
#include "carve_internal.cuh"

namespace {

using namespace carve;

// Scratch of the allocation-free forward: a 256-byte header (unused status
// word, kept so that the kernel sees the same layout as with a workspace)
// followed by the per-pair scratch of the generic forward kernel.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[CARVE_NOALLOC_SCRATCH_BYTES];

// The array's device address on the current device (host code cannot use
// the symbol itself as a pointer: in host code it names a host-side
// stand-in).  Looked up on every call.
carve_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
    return CARVE_ERR_CUDA;
  *out = p;
  return CARVE_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }
bool opt_ptr_ok(const void* p) { return p == nullptr || aligned16(p); }

}  // namespace

extern "C" carve_status carve_chunk_fwd_noalloc(
    const carve_shape* shape, const void* q, const void* k, const void* v,
    const void* g, const void* b_x, const void* w, const void* u_down,
    const void* u_up, const float* S0, const float* m0, void* o, float* S_T,
    float* m_T, void* stream) {
  // the supported set and status codes of carve_chunk_fwd
  carve_status st = check_shape(shape);
  if (st != CARVE_OK) return st;
  const carve_shape& s = *shape;
  if (s.T > 0 && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) ||
                  !ptr_ok(b_x) || !ptr_ok(w) || !ptr_ok(o)))
    return CARVE_ERR_INVALID_ARG;
  if (s.R > 0 && (!ptr_ok(u_down) || !ptr_ok(u_up)))
    return CARVE_ERR_INVALID_ARG;
  if (!opt_ptr_ok(S0) || !opt_ptr_ok(m0) || !opt_ptr_ok(S_T) ||
      !opt_ptr_ok(m_T))
    return CARVE_ERR_INVALID_ARG;

  const int C = block_len(s.L);
  const size_t per_pair = generic_fwd_scratch_floats(C, s.DK, s.DV);
  const size_t need =
      kHeaderBytes + (size_t)s.B * s.H * per_pair * sizeof(float);
  if (need > CARVE_NOALLOC_SCRATCH_BYTES) return CARVE_ERR_WORKSPACE;

  void* base = nullptr;
  st = scratch_address(&base);
  if (st != CARVE_OK) return st;

  FwdArgs a{};
  a.B = s.B; a.T = s.T; a.H = s.H; a.DK = s.DK; a.DV = s.DV; a.R = s.R;
  a.L = s.L; a.C = C; a.NB = s.T / C; a.NC = s.T / s.L;
  a.q = q; a.k = k; a.v = v; a.g = g; a.bx = b_x; a.w = w;
  a.u_down = u_down; a.u_up = u_up; a.S0 = S0; a.m0 = m0;
  a.o = o; a.S_T = S_T; a.m_T = m_T;
  a.ck_S = nullptr;
  a.ck_m = nullptr;
  a.scratch = (float*)((char*)base + kHeaderBytes);
  a.scratch_per_pair = per_pair;
  a.hdr = (WsHeader*)base;
  a.spin = kSpinCycles;
  a.stall_block = -1;
  a.dscale = s.decay_scale;
  a.qknorm = s.qk_l2norm;
  a.erase = s.erase_form;
  cudaError_t e = launch_fwd_generic(a, s.dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? CARVE_OK : CARVE_ERR_CUDA;
}
