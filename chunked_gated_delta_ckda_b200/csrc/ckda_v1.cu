// ckda_v1.cu -- chunked CKDA forward and backward on CUDA cores, fp32 math.
//
// This is the fp32-I/O path of the library (and the reference GPU path for
// the tensor-core kernels).  It follows the chunk-wise WY / UT-transform form
// ("Complex KDA: Understanding and Enhancing the Expressivity of Kimi Delta
// Attention", section 2, "Linear RNNs": KDA and Gated DeltaNet "retain
// diagonal-plus-rank-one transitions and efficient WY-based chunk-wise
// implementations") with the sign of the gate folded onto keys and queries
// ("openeurollm/complex-kda-1.3B-100B" model card, introduction).
//
// Per 64-token chunk, with start state S kept in the true (signed) frame:
//   Gam_r = sum_{s<=r} g_s, p_r = prod_{s<=r} sign_s      (chunk-local)
//   k' = p k, q' = p q
//   A   = strict_tril(sum_c k'_rc k'_sc e^{Gam_rc - Gam_sc})
//   A_q = tril(sum_c q'_rc k'_sc e^{Gam_rc - Gam_sc})
//   T = (I + Diag(beta) A)^{-1} Diag(beta); W = T (k' e^Gam); U0 = T V
//   U = U0 - W S;  O = (q' e^Gam) S + A_q U
//   S <- Diag(p_C e^{Gam_C}) S + Khat^T U,  Khat_s = p_C k'_s e^{Gam_C - Gam_s}
// The pages' running sign product P_t equals P_{chunk start} * p_t; the start
// factor cancels because the state is kept in the true frame between chunks.
//
// Pairwise decays e^{Gam_r - Gam_s} are factored through a reference row m of
// the chunk (e^{Gam_r - Gam_m} e^{Gam_m - Gam_s}) when every |Gam_r - Gam_m|
// <= kTau, so the pair sums become plain matrix products; otherwise (very
// strong decay inside one chunk) they are summed exactly per pair.
//
// Kernels:
//   intra (per chunk, head; parallel) -> W, U0, QG, Khat, A_q, d in workspace
//   state_fwd (per sequence, head, dv slice; sequential over chunks) -> o, S
//   state_bwd (per sequence, head, dv slice; reverse over chunks) -> dU, dS
//   grad (per chunk, head; parallel) -> dq, dk, dv, dbeta, dg
#include <cmath>

#include "ckda_internal.cuh"

namespace ckda {
namespace {

constexpr int NT = 256;
constexpr float kTau = 40.f;  // bound on |Gam_r - Gam_m| for the factored path
constexpr int kRefRow = 31;   // reference row m of the factored path
constexpr int DVS = 32;       // dv columns per CTA in the state passes

// Block-wide C(i,j) = alpha * sum_k A(i,k) B(k,j) (+ C(i,j) if acc), with
// A(i,k) = A[i*ar + k*ac], B(k,j) = B[k*br + j*bc], C(i,j) = C[i*cr + j*cc].
__device__ void bmm(float *Cm, int cr, int cc, const float *A, int ar, int ac,
                    const float *B, int br, int bc, int m, int n, int kd, float alpha,
                    bool acc) {
  for (int idx = threadIdx.x; idx < m * n; idx += blockDim.x) {
    const int i = idx / n, j = idx % n;
    float s = 0.f;
    for (int k = 0; k < kd; ++k) s += A[i * ar + k * ac] * B[k * br + j * bc];
    float *c = Cm + i * cr + j * cc;
    *c = acc ? *c + alpha * s : alpha * s;
  }
}

struct ChunkBufs {
  // global scratch, [C][dk] unless noted
  float *kp, *qp, *Gam, *P, *V /*[C][dv]*/, *Kl, *Kr, *Ql, *KG;
  // outputs of the intra step (global)
  float *QG, *Khat, *W, *U0 /*[C][dv]*/, *d /*[dk]*/;
  // shared
  float *A, *Aq, *M, *T, *bet, *pC, *GamC, *Gm;
  int *flag;
};

// Load one chunk (rows >= len are padding: k = q = v = 0, g = 0, sign = +1,
// beta = 0, which leaves every chunk quantity exact), the chunk-local
// log-magnitude cumsum and sign product, and the folded keys / queries.
template <typename IO>
__device__ void load_chunk(const IO *q, const IO *k, const IO *v, const float *g,
                           const int8_t *sign, const IO *beta, int64_t tok0, int len, int h,
                           int H, int dk, int dv, const ChunkBufs &b) {
  for (int idx = threadIdx.x; idx < C * dv; idx += blockDim.x) {
    const int r = idx / dv, c = idx % dv;
    b.V[idx] = r < len ? ld_io(v, ((size_t)(tok0 + r) * H + h) * dv + c) : 0.f;
  }
  for (int r = threadIdx.x; r < C; r += blockDim.x)
    b.bet[r] = r < len ? ld_io(beta, (size_t)(tok0 + r) * H + h) : 0.f;
  for (int c = threadIdx.x; c < dk; c += blockDim.x) {
    float G = 0.f, Pp = 1.f;
    for (int r = 0; r < C; ++r) {
      float kv = 0.f, qv = 0.f;
      if (r < len) {
        const size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
        G += g[off];
        if (sign && sign[off] < 0) Pp = -Pp;  // no sign tensor: all +1 (KDA)
        kv = ld_io(k, off);
        qv = ld_io(q, off);
      }
      b.kp[r * dk + c] = Pp * kv;
      b.qp[r * dk + c] = Pp * qv;
      b.Gam[r * dk + c] = G;
      b.P[r * dk + c] = Pp;
    }
    b.pC[c] = Pp;
    b.GamC[c] = G;
  }
}

// M = (I + Diag(bet) A)^{-1} for strictly-lower A (C x C, shared memory),
// column-wise forward substitution, 4 lanes per column (needs 256 threads).
__device__ void unit_lower_inverse(float *M, const float *A, const float *bet) {
  const int j = threadIdx.x >> 2, part = threadIdx.x & 3;
  for (int i = part; i < C; i += 4) M[i * C + j] = (i == j) ? 1.f : 0.f;
  __syncwarp();
  for (int i = 1; i < C; ++i) {
    float s = 0.f;
    if (i > j)
      for (int kk = j + part; kk < i; kk += 4) s += A[i * C + kk] * M[kk * C + j];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && i > j) M[i * C + j] = -bet[i] * s;
    __syncwarp();
  }
}

// Everything of one chunk that does not depend on the state.  Returns
// whether the factored (reference-row) path was used.
template <typename IO>
__device__ bool intra_core(const IO *q, const IO *k, const IO *v, const float *g,
                           const int8_t *sign, const IO *beta, int64_t tok0, int len, int h,
                           int H, int dk, int dv, const ChunkBufs &b) {
  load_chunk<IO>(q, k, v, g, sign, beta, tok0, len, h, H, dk, dv, b);
  if (threadIdx.x == 0) *b.flag = 0;
  __syncthreads();
  for (int c = threadIdx.x; c < dk; c += blockDim.x) b.Gm[c] = b.Gam[kRefRow * dk + c];
  __syncthreads();
  int bad = 0;
  for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
    const float dlt = fabsf(b.Gam[idx] - b.Gm[idx % dk]);
    if (!(dlt <= kTau)) bad = 1;
  }
  if (bad) atomicOr(b.flag, 1);
  __syncthreads();
  const bool fast = (*b.flag == 0);
  if (fast) {
    for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
      const float x = b.Gam[idx] - b.Gm[idx % dk];
      const float el = expf(x), er = expf(-x);
      b.Kl[idx] = b.kp[idx] * el;
      b.Kr[idx] = b.kp[idx] * er;
      b.Ql[idx] = b.qp[idx] * el;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
      const int r = idx / C, s = idx % C;
      float a = 0.f, aq = 0.f;
      if (s <= r)
        for (int c = 0; c < dk; ++c) {
          const float kr = b.Kr[s * dk + c];
          a += b.Kl[r * dk + c] * kr;
          aq += b.Ql[r * dk + c] * kr;
        }
      b.A[idx] = s < r ? a : 0.f;
      b.Aq[idx] = s <= r ? aq : 0.f;
    }
  } else {
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
      const int r = idx / C, s = idx % C;
      float a = 0.f, aq = 0.f;
      if (s <= r)
        for (int c = 0; c < dk; ++c) {
          const float e = expf(b.Gam[r * dk + c] - b.Gam[s * dk + c]);
          const float ks = b.kp[s * dk + c] * e;
          a += b.kp[r * dk + c] * ks;
          aq += b.qp[r * dk + c] * ks;
        }
      b.A[idx] = s < r ? a : 0.f;
      b.Aq[idx] = s <= r ? aq : 0.f;
    }
  }
  __syncthreads();
  unit_lower_inverse(b.M, b.A, b.bet);
  __syncthreads();
  for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) b.T[idx] = b.M[idx] * b.bet[idx % C];
  for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
    const int c = idx % dk;
    const float gm = b.Gam[idx];
    const float e = expf(gm);
    b.KG[idx] = b.kp[idx] * e;
    b.QG[idx] = b.qp[idx] * e;
    b.Khat[idx] = b.pC[c] * b.kp[idx] * expf(b.GamC[c] - gm);
  }
  for (int c = threadIdx.x; c < dk; c += blockDim.x) b.d[c] = b.pC[c] * expf(b.GamC[c]);
  __syncthreads();
  bmm(b.W, dk, 1, b.T, C, 1, b.KG, dk, 1, C, dk, C, 1.f, false);
  bmm(b.U0, dv, 1, b.T, C, 1, b.V, dv, 1, C, dv, C, 1.f, false);
  __syncthreads();
  return fast;
}

// shared-memory floats used by intra_core's shared buffers (+ extra C x C)
__host__ __device__ constexpr int intra_smem_floats(int extra_cc) {
  return (4 + extra_cc) * C * C + C + 4 * 128;
}

__device__ void carve_shared(float *sm, ChunkBufs &b) {
  b.A = sm;
  b.Aq = b.A + C * C;
  b.M = b.Aq + C * C;
  b.T = b.M + C * C;
  b.bet = b.T + C * C;
  b.pC = b.bet + C;
  b.GamC = b.pC + 128;
  b.Gm = b.GamC + 128;
}

// ---------------------------------------------------------------------------
// forward, intra-chunk step
// ---------------------------------------------------------------------------
__host__ __device__ inline size_t fwd_scratch_floats(int dk, int dv) {
  return (size_t)C * dk * 8 + (size_t)C * dv;
}

template <typename IO>
__global__ void __launch_bounds__(NT) intra_fwd_kernel(FwdArgs a, float *scratch) {
  extern __shared__ float sm[];
  __shared__ int flag;
  const int dk = a.dk, dv = a.dv, H = a.H;
  ChunkBufs b;
  carve_shared(sm, b);
  b.flag = &flag;
  float *scr = scratch + (size_t)blockIdx.x * fwd_scratch_floats(dk, dv);
  b.kp = scr;
  b.qp = b.kp + C * dk;
  b.Gam = b.qp + C * dk;
  b.P = b.Gam + C * dk;
  b.Kl = b.P + C * dk;
  b.Kr = b.Kl + C * dk;
  b.Ql = b.Kr + C * dk;
  b.KG = b.Ql + C * dk;
  b.V = b.KG + C * dk;
  const int nitems = a.map.n_chunks() * H;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int cid = item / H, h = item % H;
    int seq, len, j;
    int64_t tok0;
    a.map.info(cid, seq, tok0, len, j);
    IntraPtrs o = intra_ptrs(a.intra + (size_t)item * intra_floats(dk, dv), dk, dv);
    b.QG = o.QG;
    b.Khat = o.Khat;
    b.W = o.W;
    b.U0 = o.U0;
    b.d = o.d;
    intra_core<IO>((const IO *)a.q, (const IO *)a.k, (const IO *)a.v, a.g, a.sign,
                   (const IO *)a.beta, tok0, len, h, H, dk, dv, b);
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) o.Aq[idx] = b.Aq[idx];
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// forward, sequential state pass
// ---------------------------------------------------------------------------
template <typename IO>
__global__ void __launch_bounds__(NT) state_fwd_kernel(FwdArgs a, bool write_o,
                                                       float *states_out) {
  extern __shared__ float sm[];
  const int dk = a.dk, dv = a.dv, H = a.H;
  const int sl = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  const int c0 = sl * DVS;
  float *S = sm;            // [dk][DVS]
  float *U = S + dk * DVS;  // [C][DVS]
  const size_t sbase = ((size_t)seq * H + h) * dk * dv;
  for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x) {
    const int c = idx / DVS, jj = idx % DVS;
    S[idx] = a.S0 ? a.S0[sbase + (size_t)c * dv + c0 + jj] : 0.f;
  }
  __syncthreads();
  int first;
  const int nc = a.map.seq_chunks(seq, first);
  IO *o = (IO *)a.o;
  for (int jc = 0; jc < nc; ++jc) {
    const int cid = first + jc;
    int sq, len, jl;
    int64_t tok0;
    a.map.info(cid, sq, tok0, len, jl);
    const IntraPtrs in = intra_ptrs(a.intra + ((size_t)cid * H + h) * intra_floats(dk, dv), dk, dv);
    if (states_out) {
      float *dst = states_out + a.map.state_slot(seq, h, H, jc, cid) * dk * dv;
      for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x)
        dst[(size_t)(idx / DVS) * dv + c0 + idx % DVS] = S[idx];
    }
    for (int idx = threadIdx.x; idx < C * DVS; idx += blockDim.x) {
      const int r = idx / DVS, jj = idx % DVS;
      float s = in.U0[r * dv + c0 + jj];
      for (int c = 0; c < dk; ++c) s -= in.W[r * dk + c] * S[c * DVS + jj];
      U[idx] = s;
    }
    __syncthreads();
    if (write_o)
      for (int idx = threadIdx.x; idx < C * DVS; idx += blockDim.x) {
        const int r = idx / DVS, jj = idx % DVS;
        if (r >= len) continue;
        float s = 0.f;
        for (int c = 0; c < dk; ++c) s += in.QG[r * dk + c] * S[c * DVS + jj];
        for (int t = 0; t <= r; ++t) s += in.Aq[r * C + t] * U[t * DVS + jj];
        st_io(o, ((size_t)(tok0 + r) * H + h) * dv + c0 + jj, s);
      }
    __syncthreads();
    for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x) {
      const int c = idx / DVS, jj = idx % DVS;
      float s = in.d[c] * S[idx];
      for (int r = 0; r < C; ++r) s += in.Khat[r * dk + c] * U[r * DVS + jj];
      S[idx] = s;
    }
    __syncthreads();
  }
  if (a.ST)
    for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x)
      a.ST[sbase + (size_t)(idx / DVS) * dv + c0 + idx % DVS] = S[idx];
}

// ---------------------------------------------------------------------------
// backward, reverse state pass
// ---------------------------------------------------------------------------
template <typename IO>
__global__ void __launch_bounds__(NT) state_bwd_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const int dk = a.dk, dv = a.dv, H = a.H;
  const int sl = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  const int c0 = sl * DVS;
  float *dS = sm;              // [dk][DVS]
  float *dOs = dS + dk * DVS;  // [C][DVS]
  float *dU = dOs + C * DVS;   // [C][DVS]
  const size_t sbase = ((size_t)seq * H + h) * dk * dv;
  for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x)
    dS[idx] = a.dST ? a.dST[sbase + (size_t)(idx / DVS) * dv + c0 + idx % DVS] : 0.f;
  __syncthreads();
  int first;
  const int nc = a.map.seq_chunks(seq, first);
  const IO *dO = (const IO *)a.dO;
  for (int jc = nc - 1; jc >= 0; --jc) {
    const int cid = first + jc;
    int sq, len, jl;
    int64_t tok0;
    a.map.info(cid, sq, tok0, len, jl);
    const IntraPtrs in = intra_ptrs(a.intra + ((size_t)cid * H + h) * intra_floats(dk, dv), dk, dv);
    float *dst = a.dsend + a.map.state_slot(seq, h, H, jc, cid) * dk * dv;
    for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x)
      dst[(size_t)(idx / DVS) * dv + c0 + idx % DVS] = dS[idx];
    for (int idx = threadIdx.x; idx < C * DVS; idx += blockDim.x) {
      const int r = idx / DVS, jj = idx % DVS;
      dOs[idx] = r < len ? ld_io(dO, ((size_t)(tok0 + r) * H + h) * dv + c0 + jj) : 0.f;
    }
    __syncthreads();
    float *duw = a.du + ((size_t)cid * H + h) * C * dv;
    for (int idx = threadIdx.x; idx < C * DVS; idx += blockDim.x) {
      const int r = idx / DVS, jj = idx % DVS;
      float s = 0.f;
      for (int t = r; t < C; ++t) s += in.Aq[t * C + r] * dOs[t * DVS + jj];
      for (int c = 0; c < dk; ++c) s += in.Khat[r * dk + c] * dS[c * DVS + jj];
      dU[idx] = s;
      duw[(size_t)r * dv + c0 + jj] = s;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x) {
      const int c = idx / DVS, jj = idx % DVS;
      float s = in.d[c] * dS[idx];
      for (int r = 0; r < C; ++r)
        s += in.QG[r * dk + c] * dOs[r * DVS + jj] - in.W[r * dk + c] * dU[r * DVS + jj];
      dS[idx] = s;
    }
    __syncthreads();
  }
  if (a.dS0)
    for (int idx = threadIdx.x; idx < dk * DVS; idx += blockDim.x)
      a.dS0[sbase + (size_t)(idx / DVS) * dv + c0 + idx % DVS] = dS[idx];
}

// ---------------------------------------------------------------------------
// backward, per-chunk gradients
// ---------------------------------------------------------------------------
template <typename IO>
__global__ void __launch_bounds__(NT) grad_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  __shared__ int flag;
  const int dk = a.dk, dv = a.dv, H = a.H;
  ChunkBufs b;
  carve_shared(sm, b);
  b.flag = &flag;
  float *dAq = b.Gm + 128;  // [C][C] each
  float *dT = dAq + C * C;
  float *dM = dT + C * C;
  float *dA = dM + C * C;
  float *tmp = dA + C * C;
  float *dbet = tmp + C * C;  // [C]
  float *scr = a.scratch + (size_t)blockIdx.x * bwd_scratch_floats(dk, dv);
  const int CK = C * dk, CV = C * dv;
  b.kp = scr;
  b.qp = b.kp + CK;
  b.Gam = b.qp + CK;
  b.P = b.Gam + CK;
  b.Kl = b.P + CK;
  b.Kr = b.Kl + CK;
  b.Ql = b.Kr + CK;
  b.KG = b.Ql + CK;
  b.QG = b.KG + CK;
  b.Khat = b.QG + CK;
  b.W = b.Khat + CK;
  float *dQG = b.W + CK;
  float *dKhat = dQG + CK;
  float *dW = dKhat + CK;
  float *dKG = dW + CK;
  float *X1 = dKG + CK;
  float *X2 = X1 + CK;
  float *Y1 = X2 + CK;
  float *dkp = Y1 + CK;
  float *dqp = dkp + CK;
  float *dGam = dqp + CK;
  b.V = dGam + CK;
  b.U0 = b.V + CV;
  float *U = b.U0 + CV;
  float *dOs = U + CV;
  float *dUs = dOs + CV;
  float *dVv = dUs + CV;
  b.d = dVv + CV;
  float *dd = b.d + dk;

  const IO *q = (const IO *)a.q, *k = (const IO *)a.k, *v = (const IO *)a.v;
  const IO *beta = (const IO *)a.beta, *dO = (const IO *)a.dO;
  const int nitems = a.map.n_chunks() * H;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int cid = item / H, h = item % H;
    int seq, len, jl;
    int64_t tok0;
    a.map.info(cid, seq, tok0, len, jl);
    const bool fast = intra_core<IO>(q, k, v, a.g, a.sign, beta, tok0, len, h, H, dk, dv, b);
    const size_t sidx = a.map.state_slot(seq, h, H, jl, cid) * dk * dv;
    const float *Sc = a.states + sidx;
    const float *dS1 = a.dsend + sidx;
    const float *duw = a.du + ((size_t)cid * H + h) * C * dv;
    for (int idx = threadIdx.x; idx < CV; idx += blockDim.x) {
      const int r = idx / dv, c = idx % dv;
      dOs[idx] = r < len ? ld_io(dO, ((size_t)(tok0 + r) * H + h) * dv + c) : 0.f;
      dUs[idx] = duw[idx];
      U[idx] = b.U0[idx];
    }
    for (int c = threadIdx.x; c < dk; c += blockDim.x) {
      float s = 0.f;
      for (int jv = 0; jv < dv; ++jv) s += Sc[(size_t)c * dv + jv] * dS1[(size_t)c * dv + jv];
      dd[c] = s;
    }
    __syncthreads();
    // U = U0 - W Sc
    bmm(U, dv, 1, b.W, dk, 1, Sc, dv, 1, C, dv, dk, -1.f, true);
    // dQG = dO Sc^T ; dW = -dU Sc^T
    bmm(dQG, dk, 1, dOs, dv, 1, Sc, 1, dv, C, dk, dv, 1.f, false);
    bmm(dW, dk, 1, dUs, dv, 1, Sc, 1, dv, C, dk, dv, -1.f, false);
    __syncthreads();
    // dKhat = U dS1^T ; dAq = tril(dO U^T)
    bmm(dKhat, dk, 1, U, dv, 1, dS1, 1, dv, C, dk, dv, 1.f, false);
    bmm(dAq, C, 1, dOs, dv, 1, U, 1, dv, C, C, dv, 1.f, false);
    // dV = T^T dU ; dKG = T^T dW
    bmm(dVv, dv, 1, b.T, 1, C, dUs, dv, 1, C, dv, C, 1.f, false);
    bmm(dKG, dk, 1, b.T, 1, C, dW, dk, 1, C, dk, C, 1.f, false);
    // dT = dU V^T + dW KG^T
    bmm(dT, C, 1, dUs, dv, 1, b.V, 1, dv, C, C, dv, 1.f, false);
    __syncthreads();
    bmm(dT, C, 1, dW, dk, 1, b.KG, 1, dk, C, C, dk, 1.f, true);
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
      const int i = idx / C, j = idx % C;
      if (j > i) { dT[idx] = 0.f; dAq[idx] = 0.f; }
      dM[idx] = dT[idx] * b.bet[j];
    }
    __syncthreads();
    for (int j = threadIdx.x; j < C; j += blockDim.x) {
      float s = 0.f;
      for (int i = j; i < C; ++i) s += dT[i * C + j] * b.M[i * C + j];
      dbet[j] = s;
    }
    // tmp = dM M^T ; dL = -M^T tmp -> dA = Diag(bet) strict_lower(dL)
    bmm(tmp, C, 1, dM, C, 1, b.M, 1, C, C, C, C, 1.f, false);
    __syncthreads();
    bmm(dA, C, 1, b.M, 1, C, tmp, C, 1, C, C, C, -1.f, false);
    __syncthreads();
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
      float s = 0.f;
      for (int j = 0; j < i; ++j) s += dA[i * C + j] * b.A[i * C + j];
      dbet[i] += s;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
      const int i = idx / C, j = idx % C;
      dA[idx] = j < i ? dA[idx] * b.bet[i] : 0.f;
    }
    __syncthreads();
    // pairwise terms: X1 = (dA . K~)_left, X2 = (dAq . K~)_left, Y1 = right
    if (fast) {
      bmm(X1, dk, 1, dA, C, 1, b.Kr, dk, 1, C, dk, C, 1.f, false);
      bmm(X2, dk, 1, dAq, C, 1, b.Kr, dk, 1, C, dk, C, 1.f, false);
      bmm(Y1, dk, 1, dA, 1, C, b.Kl, dk, 1, C, dk, C, 1.f, false);
      __syncthreads();
      bmm(Y1, dk, 1, dAq, 1, C, b.Ql, dk, 1, C, dk, C, 1.f, true);
      __syncthreads();
      for (int idx = threadIdx.x; idx < CK; idx += blockDim.x) {
        const float x = b.Gam[idx] - b.Gm[idx % dk];
        X1[idx] *= expf(x);
        X2[idx] *= expf(x);
        Y1[idx] *= expf(-x);
      }
    } else {
      for (int idx = threadIdx.x; idx < CK; idx += blockDim.x) {
        const int r = idx / dk, c = idx % dk;
        const float gr = b.Gam[idx];
        float x1 = 0.f, x2 = 0.f, y1 = 0.f;
        for (int s = 0; s <= r; ++s) {
          const float e = expf(gr - b.Gam[s * dk + c]) * b.kp[s * dk + c];
          x1 += dA[r * C + s] * e;
          x2 += dAq[r * C + s] * e;
        }
        for (int t = r; t < C; ++t) {
          const float e = expf(b.Gam[t * dk + c] - gr);
          y1 += (dA[t * C + r] * b.kp[t * dk + c] + dAq[t * C + r] * b.qp[t * dk + c]) * e;
        }
        X1[idx] = x1;
        X2[idx] = x2;
        Y1[idx] = y1;
      }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < CK; idx += blockDim.x) {
      const int c = idx % dk;
      const float gm = b.Gam[idx];
      const float E = expf(gm);
      float dkv = X1[idx] + Y1[idx];
      float dqv = X2[idx];
      float dG = b.kp[idx] * X1[idx] + b.qp[idx] * X2[idx] - b.kp[idx] * Y1[idx];
      dkv += dKG[idx] * E;
      dG += dKG[idx] * b.KG[idx];
      dqv += dQG[idx] * E;
      dG += dQG[idx] * b.QG[idx];
      dkv += b.pC[c] * dKhat[idx] * expf(b.GamC[c] - gm);
      dG -= dKhat[idx] * b.Khat[idx];
      dkp[idx] = dkv;
      dqp[idx] = dqv;
      dGam[idx] = dG;
    }
    __syncthreads();
    IO *dqo = (IO *)a.dq, *dko = (IO *)a.dkg, *dvo = (IO *)a.dvg, *dbo = (IO *)a.dbeta;
    for (int c = threadIdx.x; c < dk; c += blockDim.x) {
      float gC = dd[c] * b.d[c];
      for (int r = 0; r < C; ++r) gC += dKhat[r * dk + c] * b.Khat[r * dk + c];
      float acc = gC;
      for (int r = C - 1; r >= 0; --r) {
        acc += dGam[r * dk + c];
        if (r < len) {
          const size_t off = ((size_t)(tok0 + r) * H + h) * dk + c;
          a.dg[off] = acc;
          st_io(dqo, off, b.P[r * dk + c] * dqp[r * dk + c]);
          st_io(dko, off, b.P[r * dk + c] * dkp[r * dk + c]);
        }
      }
    }
    for (int idx = threadIdx.x; idx < CV; idx += blockDim.x) {
      const int r = idx / dv, c = idx % dv;
      if (r < len) st_io(dvo, ((size_t)(tok0 + r) * H + h) * dv + c, dVv[idx]);
    }
    for (int r = threadIdx.x; r < len; r += blockDim.x) st_io(dbo, (size_t)(tok0 + r) * H + h, dbet[r]);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// packed-sequence chunk table
// ---------------------------------------------------------------------------
__global__ void chunk_table_kernel(const int32_t *cu, int N, int total_T, int max_seqlen,
                                   int n_chunks_bound, int32_t *table, int32_t *seq_first,
                                   DevStatus *st) {
  // one block; sequential prefix over documents in strides of blockDim
  __shared__ int s_off[1024];
  __shared__ int s_base;
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    s_base = 0;
    s_bad = (cu[0] != 0 || cu[N] != total_T) ? 1 : 0;
  }
  __syncthreads();
  for (int i0 = 0; i0 < N; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    int nc = 0;
    if (i < N) {
      const int len = cu[i + 1] - cu[i];
      if (len < 0 || len > max_seqlen) atomicOr(&s_bad, 1);
      nc = len > 0 ? (len + C - 1) / C : 0;
    }
    s_off[threadIdx.x] = nc;
    __syncthreads();
    for (int d = 1; d < blockDim.x; d <<= 1) {  // inclusive scan
      const int x = threadIdx.x >= d ? s_off[threadIdx.x - d] : 0;
      __syncthreads();
      s_off[threadIdx.x] += x;
      __syncthreads();
    }
    const int excl = s_base + s_off[threadIdx.x] - nc;
    if (i < N) {
      seq_first[i] = excl;
      if (!s_bad && excl + nc <= n_chunks_bound) {
        const int len = cu[i + 1] - cu[i];
        for (int j = 0; j < nc; ++j) {
          int32_t *e = table + 4 * (size_t)(excl + j);
          e[0] = i;
          e[1] = cu[i] + j * C;
          e[2] = min(C, len - j * C);
          e[3] = j;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_base = excl + nc;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (s_base > n_chunks_bound) s_bad = 1;
    seq_first[N] = s_base;
    if (s_bad) {
      st->flags |= kFlagBadSeqlens;
      st->n_chunks = 0;
      for (int i = 0; i <= N; ++i) seq_first[i] = 0;  // every document: no chunks
    } else {
      st->n_chunks = s_base;
    }
  }
}

}  // namespace

cudaError_t build_chunk_table(const int32_t *cu, int N, int total_T, int max_seqlen,
                              int n_chunks_bound, int32_t *table, int32_t *seq_first,
                              DevStatus *status, cudaStream_t s) {
  chunk_table_kernel<<<1, 1024, 0, s>>>(cu, N, total_T, max_seqlen, n_chunks_bound, table,
                                        seq_first, status);
  return cudaGetLastError();
}

namespace {
template <typename IO>
cudaError_t launch_intra(const FwdArgs &a, float *scratch, cudaStream_t s) {
  const size_t sm_intra = intra_smem_floats(0) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(intra_fwd_kernel<IO>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_intra);
  if (e != cudaSuccess) return e;
  ProfScope prof("v1_intra", s);
  intra_fwd_kernel<IO><<<kBwdCtas, NT, sm_intra, s>>>(a, scratch);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_state_fwd(const FwdArgs &a, bool write_o, float *states_out, cudaStream_t s) {
  if (a.map.n_seq == 0) return cudaSuccess;
  const size_t sm_state = (size_t)(a.dk + C) * DVS * sizeof(float);
  dim3 grid(a.dv / DVS, a.H, a.map.n_seq);
  ProfScope prof(write_o ? "v1_state_fwd" : "v1_state_fwd_recompute", s);
  state_fwd_kernel<IO><<<grid, NT, sm_state, s>>>(a, write_o, states_out);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_backward(const BwdArgs &a, cudaStream_t s) {
  const size_t sm_state = (size_t)(a.dk + 2 * C) * DVS * sizeof(float);
  dim3 grid(a.dv / DVS, a.H, a.map.n_seq);
  cudaError_t e;
  {
    ProfScope prof("v1_state_bwd", s);
    state_bwd_kernel<IO><<<grid, NT, sm_state, s>>>(a);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  const size_t sm_grad = (intra_smem_floats(5) + C) * sizeof(float);
  e = cudaFuncSetAttribute(grad_kernel<IO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sm_grad);
  if (e != cudaSuccess) return e;
  ProfScope prof("v1_grad", s);
  grad_kernel<IO><<<kBwdCtas, NT, sm_grad, s>>>(a);
  return cudaGetLastError();
}
}  // namespace

size_t v1_fwd_scratch_floats(int dk, int dv) { return fwd_scratch_floats(dk, dv) * kBwdCtas; }

// Same intra-chunk kernel on a caller-chosen number of persistent CTAs (each
// needs fwd_scratch_floats(dk, dv) floats of scratch); used by the entry
// point that runs out of a fixed static scratch area.
cudaError_t v1_intra_on_ctas(const FwdArgs &a, bool bf16, float *scratch, int ctas,
                             cudaStream_t s) {
  const size_t sm_intra = intra_smem_floats(0) * sizeof(float);
  if (bf16) {
    cudaError_t e = cudaFuncSetAttribute(intra_fwd_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm_intra);
    if (e != cudaSuccess) return e;
    ProfScope prof("v1_intra", s);
    intra_fwd_kernel<__nv_bfloat16><<<ctas, NT, sm_intra, s>>>(a, scratch);
  } else {
    cudaError_t e = cudaFuncSetAttribute(intra_fwd_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm_intra);
    if (e != cudaSuccess) return e;
    ProfScope prof("v1_intra", s);
    intra_fwd_kernel<float><<<ctas, NT, sm_intra, s>>>(a, scratch);
  }
  return cudaGetLastError();
}

size_t v1_fwd_scratch_floats_per_cta(int dk, int dv) { return fwd_scratch_floats(dk, dv); }

cudaError_t v1_intra(const FwdArgs &a, bool bf16, float *scratch, cudaStream_t s) {
  return bf16 ? launch_intra<__nv_bfloat16>(a, scratch, s) : launch_intra<float>(a, scratch, s);
}

cudaError_t v1_state_fwd(const FwdArgs &a, bool bf16, bool write_o, float *states_out,
                         cudaStream_t s) {
  return bf16 ? launch_state_fwd<__nv_bfloat16>(a, write_o, states_out, s)
              : launch_state_fwd<float>(a, write_o, states_out, s);
}

cudaError_t v1_backward(const BwdArgs &a, bool bf16, cudaStream_t s) {
  if (a.map.n_seq == 0) return cudaSuccess;
  return bf16 ? launch_backward<__nv_bfloat16>(a, s) : launch_backward<float>(a, s);
}

}  // namespace ckda
