/*
 * ckda.h -- C ABI of the B200 (sm_100a) Complex KDA (CKDA) recurrence library.
 *
 * The operation (one head of one sequence):
 *
 *   alpha_t = sign_t * exp(g_t)          signed per-channel gate, |alpha| <= 1
 *   S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t     = S_t^T q_t
 *
 * with S in R^{dk x dv} (rows: key channels, columns: value channels),
 * beta_t in [0, 2].  Sources: "openeurollm/complex-kda-1.3B-100B" model card,
 * introduction (signed decay alpha in [-1, 1]; |alpha| carried in log space;
 * the +-1 part carried as a running product folded onto queries and keys so
 * the kernels run the unsigned recurrence); "Complex KDA: Understanding and
 * Enhancing the Expressivity of Kimi Delta Attention", section 2 (Related
 * work, "Linear RNNs": delta-rule transition, KDA's channel-wise gate, WY-based
 * chunk-wise implementations) and section 3 ("CKDA": gate in [-1, 1], beta in
 * [0, 2]).  No output scaling is applied: callers pre-scale q if they want one.
 *
 * Conventions shared by every call
 * --------------------------------
 *  Layout     Activations are [B, T, H, D] contiguous (head-interleaved, the
 *             layout of a [B, T, H*D] projection).  beta is [B, T, H]; g and
 *             sign are [B, T, H, dk]; states are [B, H, dk, dv].  The packed
 *             variable-length call uses B = 1 and cu_seqlens.
 *  Dtypes     io_dtype (CKDA_F32 or CKDA_BF16) applies to q, k, v, beta, o and,
 *             in the backward, to dO, dq, dk, dv and dbeta.  g, dg and every
 *             state (S0, ST, chunk_states, dST, dS0, the decode state) are fp32.
 *             sign is int8 holding +1 or -1 (any other value: undefined
 *             output); a null sign pointer means every sign is +1, i.e.
 *             standard KDA (the same kernels without the sign loads).
 *             g = log|alpha| should be <= 0; the library computes exactly
 *             what it is given, and very negative g (a gate near 0) is
 *             supported.
 *  Shapes     dk, dv in {64, 128}; any T >= 0; the chunk length is 64.
 *  States     Every state crossing this ABI is in the true (signed) frame, so
 *             the final state of a chunked or packed forward can seed a decode
 *             step directly.  The sign folding is internal.
 *  Ownership  All pointers are caller-owned DEVICE memory unless stated.  The
 *             library never allocates, frees or synchronises: all work is
 *             enqueued on `stream`.  Scratch comes from the caller's workspace
 *             `ws` of `ws_bytes` bytes, at least ckda_workspace_size(...);
 *             its contents between calls are unspecified except for the
 *             status word read by ckda_check_device_status.  Calls that share
 *             a workspace must be ordered on the device (same stream).
 *  Alignment  Every tensor pointer must be 16-byte aligned, ws 256-byte
 *             aligned (CKDA_ERR_ALIGNMENT otherwise).
 *  Errors     Each call returns a status.  Argument errors are detected on the
 *             host before anything is enqueued.  Launch failures return
 *             CKDA_ERR_CUDA.  Errors found on the device (a bounded wait that
 *             ran out, malformed cu_seqlens) are recorded in the workspace's
 *             status word; ckda_check_device_status reads it (synchronising
 *             the stream).  Outputs are unspecified after any error.
 */
#ifndef CKDA_H_
#define CKDA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* I/O dtypes */
#define CKDA_F32 0
#define CKDA_BF16 1

/* status codes */
#define CKDA_OK 0
#define CKDA_ERR_INVALID_ARG 1 /* null required pointer, negative size, bad enum  */
#define CKDA_ERR_UNSUPPORTED 2 /* dk or dv outside {64, 128}; B, H or N above 65535;
                                  B*T (total_T) at or above 2^30                   */
#define CKDA_ERR_ALIGNMENT 3   /* a pointer breaks the alignment rule above        */
#define CKDA_ERR_WORKSPACE 4   /* ws null or smaller than ckda_workspace_size()    */
#define CKDA_ERR_CUDA 5        /* a kernel launch or runtime call failed           */
#define CKDA_ERR_TIMEOUT 6     /* device: a bounded wait gave up (kernel returned)  */
#define CKDA_ERR_DEVICE_ARG 7  /* device: malformed cu_seqlens                     */
#define CKDA_ERR_NOALLOC_CAPACITY 8 /* problem too large for the no-alloc scratch  */

/* operations, for ckda_workspace_size */
#define CKDA_OP_CHUNK_FWD 0
#define CKDA_OP_CHUNK_BWD 1
#define CKDA_OP_VARLEN_FWD 2
#define CKDA_OP_VARLEN_BWD 3

#define CKDA_CHUNK 64

/* Workspace bytes an operation needs.  For CKDA_OP_CHUNK_FWD / _BWD pass the
 * batched shape (N ignored); for CKDA_OP_VARLEN_FWD / _BWD pass B = 1,
 * T = total tokens and N = number of sequences.  Returns 0 for invalid
 * arguments. */
size_t ckda_workspace_size(int op, int B, int T, int H, int dk, int dv, int N);

/* Bytes of the "saved" buffer through which ckda_chunk_fwd can hand its
 * per-chunk results (the UT-transform products of every (chunk, head) and
 * the chunk-start states, bf16) to ckda_chunk_bwd, so that the backward
 * recomputes nothing and needs no chunk_states: a memory-for-time trade.
 * Returns 0 for shapes
 * and dtypes that have no saved form (then `saved` is ignored by both calls
 * and the backward recomputes) and for invalid arguments.  The contents are
 * opaque; they are valid for the inputs of the forward that wrote them. */
size_t ckda_saved_size(int B, int T, int H, int dk, int dv, int io_dtype);

/* Chunked forward over B independent sequences of length T.
 *   q, k  [B,T,H,dk] io;  v [B,T,H,dv] io;  g [B,T,H,dk] f32;
 *   sign  [B,T,H,dk] int8;  beta [B,T,H] io
 *   S0    [B,H,dk,dv] f32, nullable (zero initial state)
 *   o     [B,T,H,dv] io (written)
 *   ST    [B,H,dk,dv] f32, nullable: final state
 *   chunk_states [B,H,ceil(T/64),dk,dv] f32, nullable: the state at the start
 *         of every 64-token chunk (true frame); pass it to ckda_chunk_bwd to
 *         skip the backward's forward recomputation.
 *   saved, saved_bytes: nullable; when ckda_saved_size(...) > 0, a 256-byte
 *         aligned buffer of at least that many bytes (CKDA_ERR_WORKSPACE if
 *         smaller) that receives the per-chunk results for ckda_chunk_bwd.
 * The algorithm is the chunk-wise (WY / UT-transform) form the second source
 * names: per 64-token chunk a unit-lower-triangular intra-chunk system is
 * inverted, then a sequential pass carries the state across chunks. */
int ckda_chunk_fwd(int B, int T, int H, int dk, int dv, int io_dtype,
                   const void *q, const void *k, const void *v, const float *g,
                   const int8_t *sign, const void *beta, const float *S0,
                   void *o, float *ST, float *chunk_states, void *saved,
                   size_t saved_bytes, void *ws, size_t ws_bytes,
                   cudaStream_t stream);

/* Gradients of L(o, ST) through ckda_chunk_fwd.
 *   dO    [B,T,H,dv] io: dL/do
 *   dST   [B,H,dk,dv] f32, nullable (zero): dL/dST
 *   chunk_states: nullable; the buffer ckda_chunk_fwd filled for the same
 *         inputs (else the forward chunk states are recomputed in ws)
 *   saved, saved_bytes: nullable; the buffer ckda_chunk_fwd filled for the
 *         same inputs (else the per-chunk results are recomputed in ws).
 *         When given, chunk_states is not read.  Ignored when
 *         ckda_saved_size(...) is 0.
 *   dq, dk_out [B,T,H,dk] io;  dv_out [B,T,H,dv] io;  dg [B,T,H,dk] f32
 *         (dL/d log|alpha|);  dbeta [B,T,H] io;  dS0 [B,H,dk,dv] f32, nullable
 * The sign gets no gradient (piecewise constant); dg is the exact gradient
 * for the g given (the pages defer their gate-floor and backward convention
 * to an appendix that is not in the text). */
int ckda_chunk_bwd(int B, int T, int H, int dk, int dv, int io_dtype,
                   const void *q, const void *k, const void *v, const float *g,
                   const int8_t *sign, const void *beta, const float *S0,
                   const void *dO, const float *dST, const float *chunk_states,
                   const void *saved, size_t saved_bytes, void *dq,
                   void *dk_out, void *dv_out, float *dg, void *dbeta,
                   float *dS0, void *ws, size_t ws_bytes, cudaStream_t stream);

/* One recurrent step of N*H independent states, in place (the model card's
 * "purely recurrent" inference form).
 *   q, k [N,H,dk] io;  v [N,H,dv] io;  g [N,H,dk] f32;  sign [N,H,dk] int8;
 *   beta [N,H] io;  state [N,H,dk,dv] f32 read and written in place (true
 *   frame);  o [N,H,dv] io.  No workspace. */
int ckda_decode_step(int N, int H, int dk, int dv, int io_dtype, const void *q,
                     const void *k, const void *v, const float *g,
                     const int8_t *sign, const void *beta, float *state,
                     void *o, cudaStream_t stream);

/* Up to K recurrent steps per sequence in one pass over its state: batched
 * multi-token decode, and the verify / commit halves of speculative decoding
 * (the model card's "purely recurrent" inference form; each step is the one
 * of ckda_decode_step).  States live in a pool addressed through a slot table
 * (continuous batching: a sequence's state stays in its slot while the batch
 * around it changes).
 *   q, k [N,K,H,dk] io;  v [N,K,H,dv] io;  g [N,K,H,dk] f32;  sign [N,K,H,dk]
 *         int8, nullable (all +1: KDA);  beta [N,K,H] io.  Token t of
 *         sequence n is row (n, t), in order.
 *   n_tokens [N] int32 DEVICE, nullable (all K): steps taken by sequence n;
 *         values are clamped to [0, K].
 *   slots [N] int32 DEVICE, nullable (slot n, needs n_slots >= N): the pool
 *         slot of sequence n; a slot < 0 or >= n_slots skips the sequence
 *         (its o rows are zero and no state is touched).  Two sequences must
 *         not name the same slot when write_state is 1.
 *   state [n_slots,H,dk,dv] f32, the pool (true frame).
 *   write_state: 1 writes the state after the n_tokens steps back into the
 *         slot; 0 leaves the pool untouched (verify: outputs only).
 *   o [N,K,H,dv] io, nullable: rows t >= n_tokens[n] are zero.
 * No workspace. */
int ckda_decode_multi(int N, int K, int H, int dk, int dv, int io_dtype,
                      const void *q, const void *k, const void *v,
                      const float *g, const int8_t *sign, const void *beta,
                      const int32_t *n_tokens, const int32_t *slots, int n_slots,
                      float *state, int write_state, void *o,
                      cudaStream_t stream);

/* ---- token-mixer prologue --------------------------------------------------
 * The recurrence's inputs from the per-token projections of a layer (the
 * model card's architecture: a short convolution of width 4 ahead of the
 * recurrence; the paper's section 3 "CKDA": beta in [0, 2] and a signed gate
 * in [-1, 1] carried as log-magnitude and sign).  The pages leave the gate's
 * parameterisation, floor and backward convention to an appendix they do not
 * contain; this library's reading:
 *   q, k, v = SiLU(y), y[t,c] = sum_j w[c][j] x[t-3+j, c]  (causal depthwise
 *             conv of width 4, tap 3 on the current token, zero history at
 *             each sequence start: every batch row is its own sequence)
 *   q, k   /= sqrt(sum over the head's dk channels of the square + 1e-6)
 *   alpha   = tanh(a);  g = max(log|alpha|, g_floor);  sign = alpha < 0 ? -1 : +1
 *   beta    = 2 sigmoid(b)
 *   xq, xk [B,T,H,dk] io;  xv [B,T,H,dv] io;  wq, wk [H*dk, 4] f32;
 *   wv [H*dv, 4] f32 (row h*d + c holds channel c of head h's four taps);
 *   a [B,T,H,dk] f32 (gate pre-activation);  b [B,T,H] io;
 *   g_floor: finite and <= 0 (e.g. -5), else CKDA_ERR_INVALID_ARG.
 *   cu_seqlens: null (every batch row is one sequence), or [N+1] int32
 *             DEVICE offsets of N documents packed in one row (B = 1, else
 *             CKDA_ERR_INVALID_ARG; 4-byte aligned; N >= 1): the history
 *             restarts at each document's first token, as ckda_varlen_fwd's
 *             recurrence does.  Its offsets are not checked here (the varlen
 *             calls do): malformed ones give unspecified values, never an
 *             access outside the buffers.
 *   Outputs q, k [B,T,H,dk] io;  v [B,T,H,dv] io;  g [B,T,H,dk] f32;
 *   sign [B,T,H,dk] int8;  beta [B,T,H] io: the inputs of ckda_chunk_fwd
 *   (of ckda_varlen_fwd with cu_seqlens).
 * B and H at most 65535.  No workspace. */
int ckda_prologue_fwd(int B, int T, int H, int dk, int dv, int io_dtype,
                      const void *xq, const void *xk, const void *xv,
                      const float *wq, const float *wk, const float *wv,
                      const float *a, const void *b, float g_floor,
                      const int32_t *cu_seqlens, int N, void *q,
                      void *k, void *v, float *g, int8_t *sign, void *beta,
                      cudaStream_t stream);

/* Backward of ckda_prologue_fwd (same inputs, cu_seqlens and N included) from the gradients of its
 * outputs (dq, dk_in [B,T,H,dk] io;  dv_in [B,T,H,dv] io;  dg [B,T,H,dk]
 * f32;  dbeta [B,T,H] io -- what ckda_chunk_bwd returns).  Exact gradients of
 * the formulas above; the sign gets none; where the floor is active g gets
 * none through a.
 *   dxq, dxk [B,T,H,dk] io;  dxv [B,T,H,dv] io;  da [B,T,H,dk] f32;
 *   db [B,T,H] io;  dwq, dwk [H*dk, 4] f32;  dwv [H*dv, 4] f32.
 * dw* are overwritten: cleared on the stream, then summed over the tokens
 * with float atomics (the order of the partial sums is not fixed). */
int ckda_prologue_bwd(int B, int T, int H, int dk, int dv, int io_dtype,
                      const void *xq, const void *xk, const void *xv,
                      const float *wq, const float *wk, const float *wv,
                      const float *a, const void *b, float g_floor,
                      const int32_t *cu_seqlens, int N,
                      const void *dq, const void *dk_in, const void *dv_in,
                      const float *dg, const void *dbeta, void *dxq, void *dxk,
                      void *dxv, float *dwq, float *dwk, float *dwv, float *da,
                      void *db, cudaStream_t stream);

/* Chunked forward over N packed documents (training packs documents back to
 * back; the state restarts at each boundary).
 *   cu_seqlens [N+1] int32 DEVICE: cu[0] = 0, non-decreasing, cu[N] = total_T
 *   max_seqlen: an upper bound on every document's length (1..total_T);
 *         a document longer than it is reported as CKDA_ERR_DEVICE_ARG
 *   q, k [1,total_T,H,dk] ... as ckda_chunk_fwd with B = 1, T = total_T
 *   S0, ST [N,H,dk,dv] f32, nullable: per-document initial / final states
 *   saved, saved_bytes: nullable; when ckda_varlen_saved_size(...) > 0, a
 *         256-byte aligned buffer of at least that many bytes that receives
 *         the per-chunk results for ckda_varlen_bwd (as for ckda_chunk_fwd)
 * Chunks restart at each document start; a document's last chunk may be
 * partial.  Malformed cu_seqlens are detected on the device
 * (CKDA_ERR_DEVICE_ARG via ckda_check_device_status; no output is written). */
int ckda_varlen_fwd(int total_T, int N, const int32_t *cu_seqlens,
                    int max_seqlen, int H, int dk, int dv, int io_dtype,
                    const void *q, const void *k, const void *v, const float *g,
                    const int8_t *sign, const void *beta, const float *S0,
                    void *o, float *ST, void *saved, size_t saved_bytes,
                    void *ws, size_t ws_bytes, cudaStream_t stream);

/* Bytes of the packed forward's saved buffer (0: no saved form for this
 * configuration, or invalid arguments); the packed counterpart of
 * ckda_saved_size. */
size_t ckda_varlen_saved_size(int total_T, int N, int H, int dk, int dv,
                              int io_dtype);

/* Backward of ckda_varlen_fwd: gradients over N packed documents (training
 * on packed documents).  Arguments as ckda_varlen_fwd plus
 *   dO [1,total_T,H,dv] io;  dST [N,H,dk,dv] f32, nullable: per-document
 *   gradient of the final states;  saved, saved_bytes: nullable, the buffer
 *   ckda_varlen_fwd filled for the same inputs (and the same cu_seqlens and
 *   max_seqlen), else the per-chunk results are recomputed in ws;
 *   dq, dk_out [1,total_T,H,dk] io;
 *   dv_out [1,total_T,H,dv] io;  dg [1,total_T,H,dk] f32;  dbeta
 *   [1,total_T,H] io;  dS0 [N,H,dk,dv] f32, nullable.
 * Workspace: ckda_workspace_size(CKDA_OP_VARLEN_BWD, 1, total_T, H, dk, dv,
 * N) bytes.
 * Malformed cu_seqlens are reported as for the forward. */
int ckda_varlen_bwd(int total_T, int N, const int32_t *cu_seqlens,
                    int max_seqlen, int H, int dk, int dv, int io_dtype,
                    const void *q, const void *k, const void *v, const float *g,
                    const int8_t *sign, const void *beta, const float *S0,
                    const void *dO, const float *dST, const void *saved,
                    size_t saved_bytes, void *dq, void *dk_out, void *dv_out,
                    float *dg, void *dbeta, float *dS0, void *ws,
                    size_t ws_bytes, cudaStream_t stream);

/* ---- chunked forward without any allocation --------------------------------
 * The pages have no counterpart to this call; it serves callers that cannot
 * allocate device memory: a plug-in inside a host application that owns every
 * device allocation (a fixed pool or its own allocator, and no workspace to
 * hand over), or a latency-critical path that must not call cudaMalloc, which
 * can synchronise the device and fail at run time.
 *
 * Same arguments, semantics and outputs as ckda_chunk_fwd, minus the
 * workspace: scratch comes from one fixed array of CKDA_NOALLOC_SCRATCH_BYTES
 * that the library holds on every GPU that loads it, until the process exits.
 * Nothing is allocated or freed by the call.
 *  - Capacity: the records, one per (64-token chunk, head) -- 147 968 B
 *    (about 144.5 KiB) at dk = dv = 128, 82 176 B at dk = dv = 64 -- plus
 *    the intra-chunk kernel's fixed scratch (16 CTAs; 4 718 592 B, 4.5 MiB,
 *    at d = 128) must fit: at most 194 chunk-heads at d = 128 (e.g. B=1,
 *    T=4096, H=3, or B=2, T=6208, H=1), 379 at d = 64.  Larger problems
 *    return CKDA_ERR_NOALLOC_CAPACITY; like every argument error, before
 *    anything is enqueued.
 *  - Every pointer must be on the device that is current at the call, and
 *    `stream` must belong to that device (CKDA_ERR_INVALID_ARG otherwise):
 *    the scratch array used is the current device's.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture starts.
 *  - Every call uses the same array, which keeps the previous call's
 *    contents; calls whose work may overlap on the GPU (other streams, other
 *    host threads) race on it and must be serialised by the caller.
 *  - The kernels it runs have no bounded waits and no device-checked inputs:
 *    there is no device-side status to read for this call. */
#define CKDA_NOALLOC_SCRATCH_BYTES (32u << 20)
int ckda_chunk_fwd_noalloc(int B, int T, int H, int dk, int dv, int io_dtype,
                           const void *q, const void *k, const void *v,
                           const float *g, const int8_t *sign, const void *beta,
                           const float *S0, void *o, float *ST,
                           float *chunk_states, cudaStream_t stream);

/* Reads the device-side status recorded in ws by the last call that used it
 * (synchronises `stream`).  Returns CKDA_OK, CKDA_ERR_TIMEOUT,
 * CKDA_ERR_DEVICE_ARG or CKDA_ERR_CUDA. */
int ckda_check_device_status(const void *ws, cudaStream_t stream);

/* Static message for a status code. */
const char *ckda_status_string(int status);

/* Failure-detection self-test (not part of the recurrence).  Clears the
 * status word at the head of `ws` (at least 256 bytes, 256-byte aligned,
 * device memory), then launches one warp whose thread 0 waits, with the
 * library's bounded mbarrier wait limited to `polls` polls (the kernels use
 * 2^20, about 4 s), on a barrier that nothing arrives at.  The wait gives up, records
 * the time-out (status flag bit 0; detail word = site 900) and the kernel
 * returns, leaving the context usable: ckda_check_device_status(ws) then
 * returns CKDA_ERR_TIMEOUT.  Errors: null ws CKDA_ERR_INVALID_ARG, smaller
 * than 256 bytes CKDA_ERR_WORKSPACE, misaligned CKDA_ERR_ALIGNMENT. */
int ckda_selftest_bounded_wait(void *ws, size_t ws_bytes, uint32_t polls,
                               cudaStream_t stream);

/* ---- optional per-kernel timing (host side, off by default) -------------
 * Not part of the recurrence: a measurement aid.  While enabled, every kernel
 * launch of the library is bracketed by a pair of CUDA events recorded on the
 * launch stream.  ckda_profile_collect synchronises those events and folds
 * them into per-kernel totals; ckda_profile_get reads total i (name copied
 * into `name`, at most name_len bytes with the terminator).  The library
 * creates the events lazily (no device memory). */
int ckda_profile_enable(int on); /* returns the previous setting */
int ckda_profile_collect(void);  /* number of kernels with totals, or -status */
int ckda_profile_get(int i, char *name, int name_len, int *count, double *total_ms);
void ckda_profile_reset(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int ckda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CKDA_H_ */
