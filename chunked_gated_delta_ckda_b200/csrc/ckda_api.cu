// ckda_api.cu -- the extern "C" entry points of include/ckda.h: argument
// validation, workspace layout and dispatch to the kernels.  Host only.
#include <cstdint>
#include <cstring>

#include "ckda_internal.cuh"

namespace ckda {

WsLayout ws_layout(int op, int B, int T, int H, int dk, int dv, int N) {
  WsLayout L;
  const bool packed = (op == CKDA_OP_VARLEN_FWD || op == CKDA_OP_VARLEN_BWD);
  int64_t nch;
  int NC = 0;
  if (packed) {
    const int64_t bound = (int64_t)T / C + N;
    nch = bound < T ? bound : T;
  } else {
    NC = (T + C - 1) / C;
    nch = (int64_t)B * NC;
  }
  L.n_chunks_bound = (int)nch;
  size_t off = align256(sizeof(DevStatus));
  if (packed) {
    L.table = off;
    off += align256((size_t)nch * 4 * sizeof(int32_t));
    L.seq_first = off;
    off += align256((size_t)(N + 1) * sizeof(int32_t));
  }
  L.intra_stride = intra_floats(dk, dv);
  L.intra = off;
  off += align256((size_t)nch * H * L.intra_stride * sizeof(float));
  L.fscratch = off;
  off += align256(v1_fwd_scratch_floats(dk, dv) * sizeof(float));
  if (!packed) {
    L.seg = off;
    off += align256(tc_seg_ws_bytes());
  }
  if (op == CKDA_OP_CHUNK_BWD || op == CKDA_OP_VARLEN_BWD) {
    const size_t st = (size_t)(packed ? nch : (int64_t)B * NC) * H * dk * dv * sizeof(float);
    L.states = off;
    off += align256(st);
    L.dsend = off;
    off += align256(st);
    L.du = off;
    off += align256((size_t)nch * H * C * dv * sizeof(float));
    L.scratch = off;
    off += align256(bwd_scratch_floats(dk, dv) * kBwdCtas * sizeof(float));
  }
  L.total = off;
  return L;
}

}  // namespace ckda

using namespace ckda;

namespace {

bool a256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

int check_ws(const void *ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return CKDA_ERR_WORKSPACE;
  if (!a256(ws)) return CKDA_ERR_ALIGNMENT;
  return CKDA_OK;
}

// bytes of the forward-to-backward saved buffer; 0: no saved form
size_t saved_bytes_for(int B, int T, int H, int dk, int dv, int io_dtype);

// The saved buffer, if one is given and the configuration has a saved form;
// null otherwise.  *rc: CKDA_OK or the argument error.
const void *saved_or_null(const void *saved, size_t saved_bytes, int B, int T, int H, int dk, int dv,
                          int io_dtype, int *rc) {
  *rc = CKDA_OK;
  const size_t need = saved_bytes_for(B, T, H, dk, dv, io_dtype);
  if (!saved || need == 0) return nullptr;
  *rc = check_ws(saved, saved_bytes, need);
  return *rc == CKDA_OK ? saved : nullptr;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA; }

// bf16 I/O at dk = dv = 128 runs on the tensor cores; other shapes and fp32
// I/O (whose 1e-4 accuracy target bf16 operands cannot meet) on CUDA cores.
bool use_tensor_cores(int io_dtype, int dk, int dv) {
  return io_dtype == CKDA_BF16 && dk == 128 && dv == 128;
}

// The tensor-core path's per-(chunk, head) records are what the forward can
// save for the backward.
size_t saved_bytes_for(int B, int T, int H, int dk, int dv, int io_dtype) {
  if (!use_tensor_cores(io_dtype, dk, dv)) return 0;
  const int64_t nch = (int64_t)B * ((T + C - 1) / C);
  return (size_t)nch * H * tc_record_bytes();
}

// packed documents: one record per (chunk, head) of the chunk bound
size_t packed_saved_bytes_for(int total_T, int N, int H, int dk, int dv, int io_dtype) {
  if (!use_tensor_cores(io_dtype, dk, dv) || total_T <= 0) return 0;
  return (size_t)ws_layout(CKDA_OP_VARLEN_FWD, 1, total_T, H, dk, dv, N).n_chunks_bound * H * tc_record_bytes();
}

#define CKDA_TRY(expr)                          \
  do {                                          \
    int _rc = (expr);                           \
    if (_rc != CKDA_OK) return _rc;             \
  } while (0)
#define CKDA_CUDA(expr) CKDA_TRY(cuda_status(expr))

}  // namespace

extern "C" {

size_t ckda_workspace_size(int op, int B, int T, int H, int dk, int dv, int N) {
  if (op < CKDA_OP_CHUNK_FWD || op > CKDA_OP_VARLEN_BWD) return 0;
  if (op == CKDA_OP_VARLEN_FWD || op == CKDA_OP_VARLEN_BWD) {
    if (B != 1 || N < 0) return 0;
  }
  if (check_common(B, T, H, dk, dv, CKDA_F32) != CKDA_OK || check_grid(B, H, N) != CKDA_OK) return 0;
  return ws_layout(op, B, T, H, dk, dv, N).total;
}

size_t ckda_saved_size(int B, int T, int H, int dk, int dv, int io_dtype) {
  if (check_common(B, T, H, dk, dv, io_dtype) != CKDA_OK || check_grid(B, H, 0) != CKDA_OK) return 0;
  return saved_bytes_for(B, T, H, dk, dv, io_dtype);
}

size_t ckda_varlen_saved_size(int total_T, int N, int H, int dk, int dv, int io_dtype) {
  if (check_common(1, total_T, H, dk, dv, io_dtype) != CKDA_OK || N < 0 || check_grid(1, H, N) != CKDA_OK)
    return 0;
  return packed_saved_bytes_for(total_T, N, H, dk, dv, io_dtype);
}

int ckda_chunk_fwd(int B, int T, int H, int dk, int dv, int io_dtype, const void *q,
                   const void *k, const void *v, const float *g, const int8_t *sign,
                   const void *beta, const float *S0, void *o, float *ST, float *chunk_states,
                   void *saved, size_t saved_bytes, void *ws, size_t ws_bytes,
                   cudaStream_t stream) {
  CKDA_TRY(check_common(B, T, H, dk, dv, io_dtype));
  CKDA_TRY(check_grid(B, H, 0));
  const bool empty = (int64_t)B * T == 0;
  if (!empty) CKDA_TRY(check_ptrs({q, k, v, g, beta, o}, {sign, S0, ST, chunk_states}));
  else CKDA_TRY(check_ptrs({}, {sign, S0, ST, chunk_states}));
  int rc;
  unsigned char *recs_out = static_cast<unsigned char *>(
      const_cast<void *>(saved_or_null(saved, saved_bytes, B, T, H, dk, dv, io_dtype, &rc)));
  CKDA_TRY(rc);
  const WsLayout L = ws_layout(CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, 0);
  CKDA_TRY(check_ws(ws, ws_bytes, L.total));
  char *w = static_cast<char *>(ws);
  CKDA_CUDA(cudaMemsetAsync(w, 0, sizeof(DevStatus), stream));
  FwdArgs a{};
  a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.sign = sign;
  a.S0 = S0; a.o = o; a.ST = ST; a.chunk_states = chunk_states;
  a.map.T = T;
  a.map.NC = (T + C - 1) / C;
  a.map.n_seq = B;
  a.map.n_chunks_bound = L.n_chunks_bound;
  a.intra = reinterpret_cast<float *>(w + L.intra);
  a.status = reinterpret_cast<DevStatus *>(w);
  const bool bf16 = io_dtype == CKDA_BF16;
  if (use_tensor_cores(io_dtype, dk, dv)) {
    // with a saved buffer the state pass also stores each chunk-start state there
    CKDA_CUDA(tc_forward(a, recs_out ? recs_out : reinterpret_cast<unsigned char *>(w + L.intra),
                         reinterpret_cast<float *>(w + L.fscratch), true, chunk_states, stream,
                         /*state_pass=*/true, /*intra_pass=*/true, /*state_tiles=*/recs_out != nullptr,
                         reinterpret_cast<float *>(w + L.seg)));
    return CKDA_OK;
  }
  CKDA_CUDA(v1_intra(a, bf16, reinterpret_cast<float *>(w + L.fscratch), stream));
  CKDA_CUDA(v1_state_fwd(a, bf16, true, chunk_states, stream));
  return CKDA_OK;
}

int ckda_chunk_bwd(int B, int T, int H, int dk, int dv, int io_dtype, const void *q,
                   const void *k, const void *v, const float *g, const int8_t *sign,
                   const void *beta, const float *S0, const void *dO, const float *dST,
                   const float *chunk_states, const void *saved, size_t saved_bytes, void *dq,
                   void *dk_out, void *dv_out, float *dg, void *dbeta, float *dS0, void *ws,
                   size_t ws_bytes, cudaStream_t stream) {
  CKDA_TRY(check_common(B, T, H, dk, dv, io_dtype));
  CKDA_TRY(check_grid(B, H, 0));
  const bool empty = (int64_t)B * T == 0;
  if (!empty)
    CKDA_TRY(check_ptrs({q, k, v, g, beta, dO, dq, dk_out, dv_out, dg, dbeta},
                        {sign, S0, dST, chunk_states, dS0}));
  else
    CKDA_TRY(check_ptrs({}, {S0, dST, chunk_states, dS0}));
  int rc;
  const unsigned char *recs_in = static_cast<const unsigned char *>(
      saved_or_null(saved, saved_bytes, B, T, H, dk, dv, io_dtype, &rc));
  CKDA_TRY(rc);
  const WsLayout L = ws_layout(CKDA_OP_CHUNK_BWD, B, T, H, dk, dv, 0);
  CKDA_TRY(check_ws(ws, ws_bytes, L.total));
  char *w = static_cast<char *>(ws);
  CKDA_CUDA(cudaMemsetAsync(w, 0, sizeof(DevStatus), stream));
  const bool bf16 = io_dtype == CKDA_BF16;
  const bool tcp = use_tensor_cores(io_dtype, dk, dv);
  FwdArgs f{};
  f.B = B; f.T = T; f.H = H; f.dk = dk; f.dv = dv;
  f.q = q; f.k = k; f.v = v; f.beta = beta; f.g = g; f.sign = sign; f.S0 = S0;
  f.map.T = T;
  f.map.NC = (T + C - 1) / C;
  f.map.n_seq = B;
  f.map.n_chunks_bound = L.n_chunks_bound;
  f.intra = reinterpret_cast<float *>(w + L.intra);
  f.status = reinterpret_cast<DevStatus *>(w);
  const float *states = chunk_states;
  const unsigned char *recs =
      recs_in ? recs_in : reinterpret_cast<const unsigned char *>(w + L.intra);
  if (tcp && !recs_in) {
    // no saved buffer: recompute the records here.  Their chunk-start state
    // tiles come from the caller's fp32 chunk states when given, else from a
    // recomputed state pass.
    unsigned char *rw = const_cast<unsigned char *>(recs);
    CKDA_CUDA(tc_forward(f, rw, reinterpret_cast<float *>(w + L.fscratch), false, nullptr, stream,
                         /*state_pass=*/states == nullptr, /*intra_pass=*/true, /*state_tiles=*/true,
                         reinterpret_cast<float *>(w + L.seg)));
    if (states) CKDA_CUDA(tc_state_tiles(states, rw, B, H, f.map.NC, stream));
  } else if (!tcp) {
    CKDA_CUDA(v1_intra(f, bf16, reinterpret_cast<float *>(w + L.fscratch), stream));
    if (!states) {
      float *st = reinterpret_cast<float *>(w + L.states);
      CKDA_CUDA(v1_state_fwd(f, bf16, false, st, stream));
      states = st;
    }
  }
  BwdArgs a{};
  a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.dO = dO; a.g = g; a.sign = sign;
  a.S0 = S0; a.dST = dST; a.states = states;
  a.dq = dq; a.dkg = dk_out; a.dvg = dv_out; a.dbeta = dbeta; a.dg = dg; a.dS0 = dS0;
  a.map = f.map;
  a.intra = f.intra;
  a.dsend = reinterpret_cast<float *>(w + L.dsend);
  a.du = reinterpret_cast<float *>(w + L.du);
  a.scratch = reinterpret_cast<float *>(w + L.scratch);
  a.status = f.status;
  if (tcp) {
    CKDA_CUDA(tc_backward(a, recs, reinterpret_cast<unsigned char *>(w + L.dsend),
                          reinterpret_cast<unsigned char *>(w + L.du),
                          reinterpret_cast<float *>(w + L.fscratch), stream,
                          reinterpret_cast<float *>(w + L.seg)));
    return CKDA_OK;
  }
  CKDA_CUDA(v1_backward(a, bf16, stream));
  return CKDA_OK;
}

int ckda_decode_step(int N, int H, int dk, int dv, int io_dtype, const void *q, const void *k,
                     const void *v, const float *g, const int8_t *sign, const void *beta,
                     float *state, void *o, cudaStream_t stream) {
  CKDA_TRY(check_common(N, 1, H, dk, dv, io_dtype));
  if ((int64_t)N * H > INT32_MAX / 4) return CKDA_ERR_UNSUPPORTED;  // one CTA per (n, h)
  if (N == 0) return CKDA_OK;
  CKDA_TRY(check_ptrs({q, k, v, g, beta, state, o}, {sign}));
  return cuda_status(decode_step(N, H, dk, dv, io_dtype == CKDA_BF16, q, k, v, g, sign, beta,
                                 state, o, stream));
}

int ckda_decode_multi(int N, int K, int H, int dk, int dv, int io_dtype, const void *q, const void *k,
                      const void *v, const float *g, const int8_t *sign, const void *beta,
                      const int32_t *n_tokens, const int32_t *slots, int n_slots, float *state,
                      int write_state, void *o, cudaStream_t stream) {
  CKDA_TRY(check_common(N, K, H, dk, dv, io_dtype));
  if ((int64_t)N * H > INT32_MAX / 4) return CKDA_ERR_UNSUPPORTED;  // up to 4 CTAs per (n, h)
  if (n_slots < 0 || (write_state != 0 && write_state != 1)) return CKDA_ERR_INVALID_ARG;
  if (!slots && n_slots < N) return CKDA_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return CKDA_OK;
  CKDA_TRY(check_ptrs({q, k, v, g, beta, state}, {sign, o}));
  if ((reinterpret_cast<uintptr_t>(n_tokens) & 3u) != 0 || (reinterpret_cast<uintptr_t>(slots) & 3u) != 0)
    return CKDA_ERR_ALIGNMENT;
  return cuda_status(decode_multi(N, K, H, dk, dv, io_dtype == CKDA_BF16, q, k, v, g, sign, beta, n_tokens,
                                  slots, n_slots, state, write_state == 1, o, stream));
}

static int prologue_common(int B, int T, int H, int dk, int dv, int io_dtype, float g_floor,
                           const int32_t *cu_seqlens, int N) {
  CKDA_TRY(check_common(B, T, H, dk, dv, io_dtype));
  if (!(g_floor <= 0.f) || !isfinite(g_floor)) return CKDA_ERR_INVALID_ARG;
  if (cu_seqlens) {
    if (B != 1 || N < 1) return CKDA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return CKDA_ERR_ALIGNMENT;
  }
  return check_grid(B, H, 0);
}

int ckda_prologue_fwd(int B, int T, int H, int dk, int dv, int io_dtype, const void *xq, const void *xk,
                      const void *xv, const float *wq, const float *wk, const float *wv, const float *a,
                      const void *b, float g_floor, const int32_t *cu_seqlens, int N, void *q, void *k,
                      void *v, float *g, int8_t *sign, void *beta, cudaStream_t stream) {
  CKDA_TRY(prologue_common(B, T, H, dk, dv, io_dtype, g_floor, cu_seqlens, N));
  if ((int64_t)B * T == 0) return CKDA_OK;
  CKDA_TRY(check_ptrs({xq, xk, xv, wq, wk, wv, a, b, q, k, v, g, sign, beta}, {}));
  PrologueLaunch p{};
  p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.bf16 = io_dtype == CKDA_BF16; p.backward = false;
  p.g_floor = g_floor;
  p.xq = xq; p.xk = xk; p.xv = xv; p.b = b; p.wq = wq; p.wk = wk; p.wv = wv; p.a = a;
  p.q = q; p.k = k; p.v = v; p.g = g; p.sign = sign; p.beta = beta;
  p.cu = cu_seqlens; p.N = N;
  return cuda_status(prologue(p, stream));
}

int ckda_prologue_bwd(int B, int T, int H, int dk, int dv, int io_dtype, const void *xq, const void *xk,
                      const void *xv, const float *wq, const float *wk, const float *wv, const float *a,
                      const void *b, float g_floor, const int32_t *cu_seqlens, int N, const void *dq,
                      const void *dk_in, const void *dv_in, const float *dg, const void *dbeta, void *dxq,
                      void *dxk, void *dxv, float *dwq, float *dwk, float *dwv, float *da, void *db,
                      cudaStream_t stream) {
  CKDA_TRY(prologue_common(B, T, H, dk, dv, io_dtype, g_floor, cu_seqlens, N));
  CKDA_TRY(check_ptrs({wq, wk, wv, dwq, dwk, dwv}, {}));
  if ((int64_t)B * T > 0)
    CKDA_TRY(check_ptrs({xq, xk, xv, a, b, dq, dk_in, dv_in, dg, dbeta, dxq, dxk, dxv, da, db}, {}));
  // the taps' gradients are sums over every token: cleared here, accumulated by the kernel
  CKDA_CUDA(cudaMemsetAsync(dwq, 0, (size_t)H * dk * 4 * sizeof(float), stream));
  CKDA_CUDA(cudaMemsetAsync(dwk, 0, (size_t)H * dk * 4 * sizeof(float), stream));
  CKDA_CUDA(cudaMemsetAsync(dwv, 0, (size_t)H * dv * 4 * sizeof(float), stream));
  if ((int64_t)B * T == 0) return CKDA_OK;
  PrologueLaunch p{};
  p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.bf16 = io_dtype == CKDA_BF16; p.backward = true;
  p.g_floor = g_floor;
  p.xq = xq; p.xk = xk; p.xv = xv; p.b = b; p.wq = wq; p.wk = wk; p.wv = wv; p.a = a;
  p.dq = dq; p.dk_in = dk_in; p.dv_in = dv_in; p.dg = dg; p.dbeta = dbeta;
  p.dxq = dxq; p.dxk = dxk; p.dxv = dxv; p.db = db; p.dwq = dwq; p.dwk = dwk; p.dwv = dwv; p.da = da;
  p.cu = cu_seqlens; p.N = N;
  return cuda_status(prologue(p, stream));
}

int ckda_varlen_fwd(int total_T, int N, const int32_t *cu_seqlens, int max_seqlen, int H,
                    int dk, int dv, int io_dtype, const void *q, const void *k, const void *v,
                    const float *g, const int8_t *sign, const void *beta, const float *S0,
                    void *o, float *ST, void *saved, size_t saved_bytes, void *ws, size_t ws_bytes,
                    cudaStream_t stream) {
  CKDA_TRY(check_common(1, total_T, H, dk, dv, io_dtype));
  if (N < 0) return CKDA_ERR_INVALID_ARG;
  CKDA_TRY(check_grid(1, H, N));
  if (N == 0) return total_T == 0 ? CKDA_OK : CKDA_ERR_INVALID_ARG;
  if (!cu_seqlens) return CKDA_ERR_INVALID_ARG;
  if (total_T > 0 && (max_seqlen < 1 || max_seqlen > total_T)) return CKDA_ERR_INVALID_ARG;
  if (total_T > 0) CKDA_TRY(check_ptrs({q, k, v, g, beta, o}, {sign, S0, ST}));
  else CKDA_TRY(check_ptrs({}, {sign, S0, ST}));
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return CKDA_ERR_ALIGNMENT;
  unsigned char *recs_out = nullptr;  // the records for ckda_varlen_bwd, if asked for
  {
    const size_t need = packed_saved_bytes_for(total_T, N, H, dk, dv, io_dtype);
    if (saved && need > 0) {
      CKDA_TRY(check_ws(saved, saved_bytes, need));
      recs_out = static_cast<unsigned char *>(saved);
    }
  }
  const WsLayout L = ws_layout(CKDA_OP_VARLEN_FWD, 1, total_T, H, dk, dv, N);
  CKDA_TRY(check_ws(ws, ws_bytes, L.total));
  char *w = static_cast<char *>(ws);
  CKDA_CUDA(cudaMemsetAsync(w, 0, sizeof(DevStatus), stream));
  FwdArgs a{};
  a.B = 1; a.T = total_T; a.H = H; a.dk = dk; a.dv = dv;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.sign = sign;
  a.S0 = S0; a.o = o; a.ST = ST; a.chunk_states = nullptr;
  a.map.table = reinterpret_cast<const int32_t *>(w + L.table);
  a.map.seq_first = reinterpret_cast<const int32_t *>(w + L.seq_first);
  a.map.status = reinterpret_cast<const DevStatus *>(w);
  a.map.T = total_T;
  a.map.NC = 0;
  a.map.n_seq = N;
  a.map.n_chunks_bound = L.n_chunks_bound;
  a.intra = reinterpret_cast<float *>(w + L.intra);
  a.status = reinterpret_cast<DevStatus *>(w);
  CKDA_CUDA(build_chunk_table(cu_seqlens, N, total_T, total_T > 0 ? max_seqlen : 0,
                              L.n_chunks_bound, reinterpret_cast<int32_t *>(w + L.table),
                              reinterpret_cast<int32_t *>(w + L.seq_first),
                              reinterpret_cast<DevStatus *>(w), stream));
  const bool bf16 = io_dtype == CKDA_BF16;
  if (use_tensor_cores(io_dtype, dk, dv)) {
    CKDA_CUDA(tc_forward(a, recs_out ? recs_out : reinterpret_cast<unsigned char *>(w + L.intra),
                         reinterpret_cast<float *>(w + L.fscratch), true, nullptr, stream,
                         /*state_pass=*/true, /*intra_pass=*/true, /*state_tiles=*/recs_out != nullptr));
    return CKDA_OK;
  }
  CKDA_CUDA(v1_intra(a, bf16, reinterpret_cast<float *>(w + L.fscratch), stream));
  CKDA_CUDA(v1_state_fwd(a, bf16, true, nullptr, stream));
  return CKDA_OK;
}

int ckda_varlen_bwd(int total_T, int N, const int32_t *cu_seqlens, int max_seqlen, int H, int dk, int dv,
                    int io_dtype, const void *q, const void *k, const void *v, const float *g,
                    const int8_t *sign, const void *beta, const float *S0, const void *dO, const float *dST,
                    const void *saved, size_t saved_bytes, void *dq, void *dk_out, void *dv_out, float *dg,
                    void *dbeta, float *dS0, void *ws, size_t ws_bytes, cudaStream_t stream) {
  CKDA_TRY(check_common(1, total_T, H, dk, dv, io_dtype));
  if (N < 0) return CKDA_ERR_INVALID_ARG;
  CKDA_TRY(check_grid(1, H, N));
  if (N == 0) return total_T == 0 ? CKDA_OK : CKDA_ERR_INVALID_ARG;
  if (!cu_seqlens) return CKDA_ERR_INVALID_ARG;
  if (total_T > 0 && (max_seqlen < 1 || max_seqlen > total_T)) return CKDA_ERR_INVALID_ARG;
  if (total_T > 0)
    CKDA_TRY(check_ptrs({q, k, v, g, beta, dO, dq, dk_out, dv_out, dg, dbeta}, {sign, S0, dST, dS0}));
  else
    CKDA_TRY(check_ptrs({}, {sign, S0, dST, dS0}));
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return CKDA_ERR_ALIGNMENT;
  const unsigned char *recs_in = nullptr;  // the forward's records, if handed over
  {
    const size_t need = packed_saved_bytes_for(total_T, N, H, dk, dv, io_dtype);
    if (saved && need > 0) {
      CKDA_TRY(check_ws(saved, saved_bytes, need));
      recs_in = static_cast<const unsigned char *>(saved);
    }
  }
  const WsLayout L = ws_layout(CKDA_OP_VARLEN_BWD, 1, total_T, H, dk, dv, N);
  CKDA_TRY(check_ws(ws, ws_bytes, L.total));
  char *w = static_cast<char *>(ws);
  CKDA_CUDA(cudaMemsetAsync(w, 0, sizeof(DevStatus), stream));
  FwdArgs f{};
  f.B = 1; f.T = total_T; f.H = H; f.dk = dk; f.dv = dv;
  f.q = q; f.k = k; f.v = v; f.beta = beta; f.g = g; f.sign = sign; f.S0 = S0;
  f.map.table = reinterpret_cast<const int32_t *>(w + L.table);
  f.map.seq_first = reinterpret_cast<const int32_t *>(w + L.seq_first);
  f.map.status = reinterpret_cast<const DevStatus *>(w);
  f.map.T = total_T;
  f.map.NC = 0;
  f.map.n_seq = N;
  f.map.n_chunks_bound = L.n_chunks_bound;
  f.intra = reinterpret_cast<float *>(w + L.intra);
  f.status = reinterpret_cast<DevStatus *>(w);
  CKDA_CUDA(build_chunk_table(cu_seqlens, N, total_T, total_T > 0 ? max_seqlen : 0, L.n_chunks_bound,
                              reinterpret_cast<int32_t *>(w + L.table), reinterpret_cast<int32_t *>(w + L.seq_first),
                              reinterpret_cast<DevStatus *>(w), stream));
  const bool bf16 = io_dtype == CKDA_BF16;
  const bool tcp = use_tensor_cores(io_dtype, dk, dv);
  const float *states = nullptr;
  const unsigned char *recs = recs_in ? recs_in : reinterpret_cast<const unsigned char *>(w + L.intra);
  if (tcp && !recs_in) {  // records with their bf16 chunk-start states, recomputed
    CKDA_CUDA(tc_forward(f, const_cast<unsigned char *>(recs), reinterpret_cast<float *>(w + L.fscratch), false,
                         nullptr, stream, /*state_pass=*/true, /*intra_pass=*/true, /*state_tiles=*/true, nullptr));
  } else if (!tcp) {
    CKDA_CUDA(v1_intra(f, bf16, reinterpret_cast<float *>(w + L.fscratch), stream));
    float *st = reinterpret_cast<float *>(w + L.states);
    CKDA_CUDA(v1_state_fwd(f, bf16, false, st, stream));
    states = st;
  }
  BwdArgs a{};
  a.B = 1; a.T = total_T; a.H = H; a.dk = dk; a.dv = dv;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.dO = dO; a.g = g; a.sign = sign;
  a.S0 = S0; a.dST = dST; a.states = states;
  a.dq = dq; a.dkg = dk_out; a.dvg = dv_out; a.dbeta = dbeta; a.dg = dg; a.dS0 = dS0;
  a.map = f.map;
  a.intra = f.intra;
  a.dsend = reinterpret_cast<float *>(w + L.dsend);
  a.du = reinterpret_cast<float *>(w + L.du);
  a.scratch = reinterpret_cast<float *>(w + L.scratch);
  a.status = f.status;
  if (tcp) {
    CKDA_CUDA(tc_backward(a, recs, reinterpret_cast<unsigned char *>(w + L.dsend),
                          reinterpret_cast<unsigned char *>(w + L.du),
                          reinterpret_cast<float *>(w + L.fscratch), stream, nullptr));
    return CKDA_OK;
  }
  CKDA_CUDA(v1_backward(a, bf16, stream));
  return CKDA_OK;
}

int ckda_check_device_status(const void *ws, cudaStream_t stream) {
  if (!ws) return CKDA_ERR_INVALID_ARG;
  DevStatus st;
  if (cudaMemcpyAsync(&st, ws, sizeof(st), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return CKDA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return CKDA_ERR_CUDA;
  if (st.flags & kFlagTimeout) return CKDA_ERR_TIMEOUT;
  if (st.flags & kFlagBadSeqlens) return CKDA_ERR_DEVICE_ARG;
  return CKDA_OK;
}

const char *ckda_status_string(int status) {
  switch (status) {
    case CKDA_OK: return "ok";
    case CKDA_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad enum)";
    case CKDA_ERR_UNSUPPORTED:
      return "unsupported shape (dk, dv in {64, 128}; B, H, N at most 65535; B*T below 2^30)";
    case CKDA_ERR_ALIGNMENT: return "misaligned pointer (tensors 16-byte, workspace 256-byte)";
    case CKDA_ERR_WORKSPACE: return "workspace missing or smaller than ckda_workspace_size()";
    case CKDA_ERR_CUDA: return "CUDA launch or runtime error";
    case CKDA_ERR_TIMEOUT: return "a bounded device wait gave up";
    case CKDA_ERR_DEVICE_ARG: return "malformed cu_seqlens (found on the device)";
    case CKDA_ERR_NOALLOC_CAPACITY:
      return "problem does not fit the fixed scratch of ckda_chunk_fwd_noalloc";
    default: return "unknown status";
  }
}

int ckda_version(void) { return 100; }

}  // extern "C"
