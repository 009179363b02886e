/*
 * carve.h -- C ABI of libcarve, the B200 (sm_100a) implementation of the
 * CARVE chunk-parallel recurrent core.
 *
 * The operation (one state per (sequence b, head h)); the pages' notation:
 *
 *   S_t = S_{t-1} Diag(exp g_t) (I - k_t (b_t (.) k_t)^T) + w_t v_t k_t^T
 *   o_t = S_{t-1} q_t
 *   b_{c,t} = sigmoid(b_x,t + U_b m_c),  U_b = U_up U_down  (rank R)
 *   m_c = (1/L) sum of o_t over chunk c-1 (L tokens); chunk 0 uses m0 (or 0)
 *
 * Sources (CARVE: Content-Aware Recurrent with Value Efficiency for
 * Chunk-Parallel Linear Attention, arXiv 2606.27229, as summarised on
 * gist.science):
 *   state S_t in R^{dv x dk} ............ technical summary section 1
 *   o_t = S_{t-1} q_t, m_c, b_{c,t} ...... section 2.1 (content-aware erase
 *                                          via output reuse)
 *   scalar write gate w per head ......... section 2.2
 *   exponential decay on the key axis .... section 2.3
 *   erase on the key axis only, solved by
 *   one WY triangular solve per chunk .... abstract; section 3 (Theorem 11)
 *   no content signal in chunk 0 ......... section 5 (acknowledged limitation)
 *
 * Conventions for every entry point
 *   - All tensor pointers are caller-owned DEVICE memory on the current
 *     device, contiguous row-major in the layouts given, 16-byte aligned.
 *   - The library never allocates, frees or synchronises (except
 *     carve_get_status); work is enqueued on `stream` (a cudaStream_t; NULL
 *     = legacy default stream) and the call returns immediately.
 *   - Host-side validation failures return a status and enqueue nothing.
 *   - "dtype" tensors are bf16 (CARVE_BF16) or fp32 (CARVE_FP32) as given in
 *     carve_shape.dtype; the state, S0, S_T, m0, m_T and the U_b gradients
 *     are always fp32.  Arithmetic is fp32 with fp32 accumulation.
 */
#ifndef CARVE_H_
#define CARVE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CARVE_OK = 0,
  CARVE_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size        */
  CARVE_ERR_UNSUPPORTED = 2, /* shape outside the supported set (see below) */
  CARVE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
  CARVE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed        */
  CARVE_ERR_TIMEOUT = 5      /* a device-side bounded wait gave up          */
} carve_status;

typedef enum { CARVE_BF16 = 0, CARVE_FP32 = 1 } carve_dtype;

/*
 * Problem shape.  B sequences of T tokens, H heads, key width DK, value
 * width DV, rank R of U_b, chunk length L.
 * Supported: B, H >= 1; T >= 0; DK, DV multiples of 16 in [16, 256];
 * 0 <= R <= 64; L in [1, 64] or a multiple of 64 up to 256.  Training
 * (carve_chunk_fwd with training != 0, carve_chunk_bwd) needs T % L == 0;
 * the forward without training takes any T (the last chunk of a sequence
 * may be short; its mean, returned in m_T, still divides by L).
 * Anything else returns CARVE_ERR_UNSUPPORTED.
 * Kernel families: bf16 with DK = 128, R <= 32, T > 0 runs on the tensor
 * cores for DV = 128 with L a multiple of 64 (forward, training forward and
 * backward), and for the forward without training also with DV = 256 and
 * with L = 16, 32 or 48 (one chunk per 64-row tile); every other shape, and
 * fp32 inputs, on the generic CUDA-core kernels.
 */
typedef struct {
  int32_t B, T, H, DK, DV, R, L;
  int32_t dtype;      /* carve_dtype */
  float decay_scale;  /* 0: g is the log-decay itself (g <= 0);
                       * s > 0: g holds raw decay logits a and the kernels
                       * use g = -s * softplus(a) (the activation fused into
                       * the chunk kernels, CARVE summaries, gist.science,
                       * section 2.3 "Key-Axis Decay und Fusion"); the
                       * backward then returns dL/da in dg.  Negative or
                       * non-finite: CARVE_ERR_INVALID_ARG. */
  int32_t qk_l2norm;  /* 0: q and k are used as given (the workloads pass
                       * unit rows); 1: the kernels divide every token's q
                       * and k by their Euclidean norms over DK themselves
                       * (a fused prologue) and the backward returns the
                       * gradients of the raw q and k.  Other values:
                       * CARVE_ERR_INVALID_ARG. */
  int32_t erase_form; /* 0: S' (I - k (b (.) k)^T) as above; 1: the other
                       * erase that acts on the key axis only,
                       * S' (I - (b (.) k) k^T) (the gated key reads the
                       * state, the plain key is written; both forms are
                       * chunkable, gist.science section 3).  Form 1 runs on
                       * the generic kernels and the decode step.  Other
                       * values: CARVE_ERR_INVALID_ARG. */
} carve_shape;

/*
 * Bytes of device workspace carve_chunk_fwd / carve_chunk_bwd need for this
 * shape.  training != 0 adds what carve_chunk_bwd reads: on the tensor-core
 * path the final fp32 state, the per-chunk gate inputs and the per-block
 * records (bf16 state operand, E and T; 56 KiB per 64-token block); on the
 * generic path the fp32 state at every block start.  Returns 0 for an
 * invalid or unsupported shape.  The workspace starts with a 256-byte
 * header holding the device status word (see carve_get_status).  The size
 * depends on which kernel family runs (carve_fwd_path; the environment
 * override CARVE_FWD_PATH=generic selects the generic one), so query it
 * under the same setting as the calls that use it.
 */
size_t carve_workspace_bytes(const carve_shape* shape, int training);

/*
 * Forward pass over all chunks of all (b, h) pairs.
 *
 *   q, k, g, b_x : [B, T, H, DK] dtype   (g is the log-decay, g <= 0)
 *   v            : [B, T, H, DV] dtype
 *   w            : [B, T, H]     dtype   scalar write gate per token, head
 *   u_down       : [H, R, DV]    dtype   U_b = u_up[h] @ u_down[h]
 *   u_up         : [H, DK, R]    dtype   (may be NULL when R == 0)
 *   S0           : [B, H, DV, DK] fp32, or NULL for zeros
 *   m0           : [B, H, DV]     fp32, or NULL for zeros (the pages' rule:
 *                  chunk 0 gets no content signal); a non-NULL m0 resumes a
 *                  sequence split at a chunk boundary exactly
 *   o            : [B, T, H, DV] dtype   (output, overwritten)
 *   S_T          : [B, H, DV, DK] fp32 final state, or NULL
 *   m_T          : [B, H, DV]     fp32 mean of the last chunk's outputs
 *                  (the next call's m0), or NULL
 *   workspace    : carve_workspace_bytes(shape, training) bytes
 *   training     : nonzero to keep what carve_chunk_bwd needs in workspace
 *
 * Inputs and outputs must not overlap.  Errors: INVALID_ARG, UNSUPPORTED,
 * WORKSPACE, CUDA (launch failure; the stream is left as CUDA left it).
 */
carve_status carve_chunk_fwd(const carve_shape* shape,
                             const void* q, const void* k, const void* v,
                             const void* g, const void* b_x, const void* w,
                             const void* u_down, const void* u_up,
                             const float* S0, const float* m0,
                             void* o, float* S_T, float* m_T,
                             void* workspace, size_t workspace_bytes,
                             int training, void* stream);

/*
 * Forward without training over packed sequences of different lengths
 * (variable-length batches: the chunk-0 rule of the CARVE technical
 * summary, gist.science, section 5 (acknowledged limitation), applies to
 * each sequence from its own start).
 *
 *   shape        : B = number of sequences, T = total packed tokens (any
 *                  T >= 0), the other fields as for carve_chunk_fwd
 *   cu_seqlens   : [B + 1] int32 DEVICE array: sequence b is tokens
 *                  cu_seqlens[b] .. cu_seqlens[b + 1] - 1, with
 *                  0 <= cu_seqlens[b] <= cu_seqlens[b + 1] <= T (checked on
 *                  the device: a violation sets CARVE_ERR_INVALID_ARG in the
 *                  status word and that sequence is skipped)
 *   q, k, g, b_x : [T, H, DK] dtype   packed tokens
 *   v            : [T, H, DV] dtype
 *   w            : [T, H]     dtype
 *   u_down, u_up : as for carve_chunk_fwd
 *   S0, m0       : [B, H, DV, DK], [B, H, DV] fp32 per sequence, or NULL
 *   o            : [T, H, DV] dtype   (tokens of no sequence are left as is)
 *   S_T, m_T     : [B, H, DV, DK], [B, H, DV] fp32 per sequence, or NULL
 *   workspace    : carve_workspace_bytes(shape, 0) bytes
 *
 * Chunks of L tokens start at each sequence's first token; a sequence's last
 * chunk may be short (its mean, m_T, divides by L).  An empty sequence
 * returns S_T = S0 and m_T = m0.  Errors as for carve_chunk_fwd.
 */
carve_status carve_chunk_fwd_varlen(const carve_shape* shape,
                                    const int32_t* cu_seqlens,
                                    const void* q, const void* k,
                                    const void* v, const void* g,
                                    const void* b_x, const void* w,
                                    const void* u_down, const void* u_up,
                                    const float* S0, const float* m0,
                                    void* o, float* S_T, float* m_T,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * Backward pass: exact reverse mode of carve_chunk_fwd (the gradient also
 * flows through the content gate into the previous chunk's outputs).
 *
 *   q ... u_up   : the same inputs given to the training-mode forward
 *   workspace    : the workspace of that forward (training != 0), untouched
 *                  since; it holds the block-start states, the chunk gate
 *                  inputs and S0 / m0, so S0 and m0 are not passed again
 *   d_o          : [B, T, H, DV] dtype upstream gradient of o
 *   dS_T         : [B, H, DV, DK] fp32 upstream gradient of S_T, or NULL (0)
 *   dm_T         : [B, H, DV] fp32 upstream gradient of m_T, or NULL (0)
 *   dq, dk, dg, db_x : [B, T, H, DK] dtype (overwritten)
 *   dv           : [B, T, H, DV] dtype   (overwritten)
 *   dw           : [B, T, H]     dtype   (overwritten)
 *   du_down      : [H, R, DV] fp32 summed over the batch (overwritten)
 *   du_up        : [H, DK, R] fp32 summed over the batch (overwritten)
 *   dS0          : [B, H, DV, DK] fp32 or NULL;  dm0 : [B, H, DV] fp32 or NULL
 *
 * Errors as for carve_chunk_fwd.
 */
carve_status carve_chunk_bwd(const carve_shape* shape,
                             const void* q, const void* k, const void* v,
                             const void* g, const void* b_x, const void* w,
                             const void* u_down, const void* u_up,
                             const void* d_o, const float* dS_T,
                             const float* dm_T,
                             void* workspace, size_t workspace_bytes,
                             void* dq, void* dk, void* dv, void* dg,
                             void* db_x, void* dw,
                             float* du_down, float* du_up,
                             float* dS0, float* dm0, void* stream);

/*
 * Allocation-free forward (no counterpart in the paper; a convenience of
 * this library).  For callers that cannot allocate device memory where they
 * run the recurrence: a plugin whose host framework hands it only input and
 * output tensors, a stream-ordered section where cudaMalloc's implicit
 * device-wide synchronisation would stall other streams, or a real-time
 * loop with a fixed memory budget.
 *
 * Same arguments and results as carve_chunk_fwd with training = 0, minus
 * the workspace: the generic forward kernel keeps its per-(b, h) scratch in
 * a static device array of CARVE_NOALLOC_SCRATCH_BYTES that is part of the
 * library's device image (every GPU that loads libcarve holds it until the
 * process exits).  The call allocates and frees nothing.
 *   - Needs 256 + B*H*(4*C*DK + 4*C*DV + DV*DK)*4 bytes of that array,
 *     C = min(L, 64); a larger shape returns CARVE_ERR_WORKSPACE and
 *     enqueues nothing.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing).  The first call on a
 *     device may also load the library's device code there: make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; the kernel writes every scratch element before reading it, so
 *     nothing has to be cleared between calls.  Calls whose kernels overlap
 *     on the GPU (e.g. on two streams) race on the array: serialise them.
 *   - Always runs the generic CUDA-core kernel, whatever carve_fwd_path says.
 * Errors as for carve_chunk_fwd.
 */
#define CARVE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
carve_status carve_chunk_fwd_noalloc(const carve_shape* shape,
                                     const void* q, const void* k,
                                     const void* v, const void* g,
                                     const void* b_x, const void* w,
                                     const void* u_down, const void* u_up,
                                     const float* S0, const float* m0,
                                     void* o, float* S_T, float* m_T,
                                     void* stream);

/*
 * One recurrent decode step for inference: the token form of the same
 * recurrence, advancing every (sequence, head) by one new token (CARVE
 * technical summary, gist.science, sections 1 and 2.1-2.3; the content
 * signal m_c is the mean of the previous chunk's outputs, section 2.1).
 *
 *   shape        : B, H, DK, DV, R, L and dtype as for carve_chunk_fwd; T is
 *                  ignored (one token)
 *   q, k, g, b_x : [B, H, DK] dtype   the new token (g: log-decay, <= 0)
 *   v            : [B, H, DV] dtype
 *   w            : [B, H]     dtype
 *   u_down, u_up : [H, R, DV], [H, DK, R] dtype (NULL allowed when R == 0)
 *   pos          : [B] int32  tokens of each sequence already processed (the
 *                  new token's index; read only: the caller advances it)
 *   S            : [B, H, DV, DK] fp32 in/out   S_{t-1} -> S_t
 *   m            : [B, H, DV] fp32 in/out       the current chunk's content
 *                  signal m_c (zero for a new sequence, or m_T of a forward);
 *                  replaced by the chunk's mean after its last token
 *   osum         : [B, H, DV] fp32 in/out       sum of the current chunk's
 *                  outputs so far (zero at a chunk boundary); reset to zero
 *                  after the chunk's last token
 *   o            : [B, H, DV] dtype   o_t = S_{t-1} q_t (overwritten)
 *
 * Per pair: p = U_up U_down m, b = sigmoid(b_x + p), o = S q,
 * S' = S Diag(exp g), S = S' - (S' k)(b k)^T + w v k^T, osum += o, and when
 * (pos + 1) % L == 0: m = osum / L, osum = 0.  A sequence processed by
 * carve_chunk_fwd (T a multiple of L, final S_T and m_T) continues here with
 * S = S_T, m = m_T, osum = 0, pos = T.  A cluster of four CTAs per
 * (sequence, head), each owning a quarter of the value rows; no workspace;
 * asynchronous on `stream`.  Errors: INVALID_ARG, UNSUPPORTED, CUDA (launch
 * failure).  With no workspace there is no status word: a CTA whose input
 * copies have not landed after about 1 s (2^31 cycles) leaves its rows of
 * S, m and osum as they were and writes NaN to its rows of o.  The test
 * knobs of carve_get_status apply: CARVE_TEST_WAIT_CYCLES lowers that
 * limit, and CARVE_TEST_STALL_BLOCK (any value >= 0) makes the first CTA
 * (pair 0, rows 0 .. DV/4 - 1) issue none of its first group of copies.
 */
carve_status carve_decode_step(const carve_shape* shape,
                               const void* q, const void* k, const void* v,
                               const void* g, const void* b_x, const void* w,
                               const void* u_down, const void* u_up,
                               const int32_t* pos, float* S, float* m,
                               float* osum, void* o, void* stream);

/*
 * Synchronises `stream`, then reads the device status word that kernels
 * write into the workspace header (CARVE_OK, or CARVE_ERR_TIMEOUT when a
 * bounded device-side wait gave up; the kernel then skipped the rest of its
 * work and left its outputs unspecified; CARVE_ERR_WORKSPACE when a
 * backward was given a workspace the other kernel family wrote).  The word
 * is sticky until carve_reset_status.
 *
 * Every wait of the tensor-core kernels on a copy, an MMA or the partner
 * CTA gives up after about 1 s (2^31 cycles).  Two environment variables
 * exist for tests of that path only: CARVE_TEST_WAIT_CYCLES lowers the
 * limit, and CARVE_TEST_STALL_BLOCK=n makes CTA 0 send the commit of block
 * n's first MMA batch to a barrier nobody waits on, so that its wait runs
 * out (the MMAs still complete and are waited for before the CTA exits).
 */
carve_status carve_get_status(const void* workspace, void* stream);

/* Enqueue a reset of the workspace status word to CARVE_OK on `stream`. */
carve_status carve_reset_status(void* workspace, void* stream);

/* Static, human-readable name of a status code. */
const char* carve_status_str(carve_status status);

/* Name of the kernel family carve_chunk_fwd with training = 0 would use
 * for this shape ("tc" for the tcgen05 path, "generic" otherwise), or NULL
 * if unsupported. */
const char* carve_fwd_path(const carve_shape* shape);

#ifdef __cplusplus
}
#endif

#endif /* CARVE_H_ */
