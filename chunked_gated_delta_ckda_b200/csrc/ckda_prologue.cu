// ckda_prologue.cu -- the token-mixer prologue ahead of the recurrence, and
// its backward.
//
// From the per-token projections to the recurrence's inputs
// ("openeurollm/complex-kda-1.3B-100B" model card, architecture: short
// convolution of width 4; "Complex KDA: ..." paper text, section 3 "CKDA":
// beta in [0, 2], a signed gate in [-1, 1] carried as log-magnitude and sign).
// The gate's exact parameterisation and its floor live in an appendix the
// pages do not contain; these are the readings, stated once in ckda.h:
//   q, k, v = SiLU(causal depthwise conv of width 4), zero history per sequence
//             (per document when documents are packed in one row)
//   q, k   /= sqrt(sum over the head's channels of the square + 1e-6)
//   alpha   = tanh(a):  g = max(log|alpha|, g_floor),  sign = alpha < 0 ? -1 : +1
//   beta    = 2 sigmoid(b)
//
// One CTA of 128 threads per (64-token run, head, sequence); thread c owns
// channel c of q, k, the gate (c < dk) and v (c < dv) and walks the run's
// tokens in order with the convolution window (the three previous inputs) in
// registers, so every input element is read once (plus a three-token halo).
// The L2 norms need reductions over the head's channels: batched over 8
// tokens (forward) or 4 (backward) per barrier, so each batch's loads are in
// flight together.  Its roof is HBM; as measured it is bound by instruction
// issue (about a third of the HBM roof backward, under half forward).
#include "ckda_internal.cuh"

namespace ckda {
namespace {

constexpr int kPrThreads = 128;
constexpr int kPrTok = 64;  // tokens per CTA
constexpr float kNormEps = 1e-6f;

struct PrologueArgs {
  int B, T, H, dk, dv;
  float g_floor;
  const void *xq, *xk, *xv, *b;
  const float *wq, *wk, *wv, *a;
  void *q, *k, *v, *beta;  // forward outputs
  float *g;
  int8_t *sign;
  const void *dq, *dk_in, *dv_in, *dbeta;  // backward inputs
  const float *dg;
  void *dxq, *dxk, *dxv, *db;  // backward outputs
  float *dwq, *dwk, *dwv, *da;
  const int32_t *cu;  // packed documents: [N + 1] offsets (null: every batch row is a sequence)
  int N;
};

// First token of the document of each token t0 - 3 + e, e < n (0 when every
// batch row is its own sequence): the convolution's history stops there.
__device__ __forceinline__ void doc_starts(const PrologueArgs &a, int t0, int n, int *s_ds) {
  for (int e = threadIdx.x; e < n; e += kPrThreads) {
    const int t = t0 - 3 + e;
    int start = 0;
    if (a.cu && t >= 0 && t < a.T) {  // the last i with cu[i] <= t
      int lo = 0, hi = a.N;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cu[mid] <= t) lo = mid; else hi = mid - 1;
      }
      start = a.cu[lo];
    }
    s_ds[e] = start;
  }
}

// sigmoid with the fast exponential and division (a few ulp; 0 for y below
// about -88, where the exponential overflows)
__device__ __forceinline__ float sigm(float y) { return __fdividef(1.f, 1.f + __expf(-y)); }

// tanh from the fast exponential, written from the identities
//   tanh|x| = (1 - e) / (1 + e),  e = exp(-2|x|)          (|x| >= 0.05)
//   tanh x  = x - x^3/3 + 2 x^5/15 - ...  (Taylor series)  (|x| <  0.05, where
//             1 - e would cancel; the first omitted term, 17 x^7/315, is
//             below 1e-9 of the value there)
// both evaluated (no divergence), the sign restored at the end
__device__ __forceinline__ float tanh_fast(float x) {
  const float t = fabsf(x), t2 = t * t;
  const float e = __expf(-2.f * t);
  const float big = __fdividef(1.f - e, 1.f + e);
  const float small = t * (1.f - t2 * (1.f / 3.f) + t2 * t2 * (2.f / 15.f));
  return copysignf(t < 0.05f ? small : big, x);
}

// Sums of 16 values over the CTA's 128 threads; every thread gets all 16
// totals.  In the warp, a halving exchange (8 + 4 + 2 + 1 + 1 shuffles)
// leaves lane pair (2m, 2m + 1) with the warp total of value
// 8 b4 + 4 b3 + 2 b2 + b1 (the lane's bits); the four warps' totals meet in
// shared memory (buffer `par`, alternating between calls: one barrier).
__device__ __forceinline__ void block_sum16(float (&x)[16], float (*red)[kPrThreads / 32][16], int par) {
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
  float p8[8], p4[4], p2[2];
#pragma unroll
  for (int i = 0; i < 8; ++i) p8[i] = (b4 ? x[i + 8] : x[i]) + __shfl_xor_sync(FULL, b4 ? x[i] : x[i + 8], 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) p4[i] = (b3 ? p8[i + 4] : p8[i]) + __shfl_xor_sync(FULL, b3 ? p8[i] : p8[i + 4], 8);
#pragma unroll
  for (int i = 0; i < 2; ++i) p2[i] = (b2 ? p4[i + 2] : p4[i]) + __shfl_xor_sync(FULL, b2 ? p4[i] : p4[i + 2], 4);
  float t = (b1 ? p2[1] : p2[0]) + __shfl_xor_sync(FULL, b1 ? p2[0] : p2[1], 2);
  t += __shfl_xor_sync(FULL, t, 1);
  if (!(lane & 1)) red[par][w][(b4 ? 8 : 0) + (b3 ? 4 : 0) + (b2 ? 2 : 0) + (b1 ? 1 : 0)] = t;
  __syncthreads();
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int ww = 0; ww < kPrThreads / 32; ++ww) {
      const float4 r = reinterpret_cast<const float4 *>(red[par][ww])[q4];
      acc.x += r.x; acc.y += r.y; acc.z += r.z; acc.w += r.w;
    }
    x[4 * q4] = acc.x; x[4 * q4 + 1] = acc.y; x[4 * q4 + 2] = acc.z; x[4 * q4 + 3] = acc.w;
  }
}

// Forward: 8 tokens per reduction (q and k sums of squares).
constexpr int kFwdG = 8;
// PACKED: documents packed in one row (a.cu); otherwise the masks are not compiled.
template <typename IO, int DK, int DV, bool PACKED>
__global__ void __launch_bounds__(kPrThreads, 6) prologue_fwd_kernel(const PrologueArgs a) {
  __shared__ __align__(16) float red[2][kPrThreads / 32][16];
  __shared__ int s_ds[PACKED ? kPrTok + 8 : 1];
  const int c = threadIdx.x, h = blockIdx.y, sq = blockIdx.z;
  const int T = a.T, H = a.H;
  constexpr int dk = DK, dv = DV;
  const int t0 = blockIdx.x * kPrTok, t1 = min(t0 + kPrTok, T);
  const bool kc = DK == kPrThreads || c < DK, vc = DV == kPrThreads || c < DV;  // (compile-time true at 128)
  const IO *xq = (const IO *)a.xq, *xk = (const IO *)a.xk, *xv = (const IO *)a.xv;
  if constexpr (PACKED) {
    doc_starts(a, t0, kPrTok + 3, s_ds);
    __syncthreads();
  }
  float wq[4], wk[4], wv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    wq[j] = kc ? a.wq[((size_t)h * dk + c) * 4 + j] : 0.f;
    wk[j] = kc ? a.wk[((size_t)h * dk + c) * 4 + j] : 0.f;
    wv[j] = vc ? a.wv[((size_t)h * dv + c) * 4 + j] : 0.f;
  }
  // the window: inputs of tokens t - 3, t - 2, t - 1 (zero before the sequence)
  float hq[3], hk[3], hv[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int t = t0 - 3 + i;
    const size_t row = ((size_t)sq * T + (t < 0 ? 0 : t)) * H + h;
    hq[i] = (t >= 0 && kc) ? ld_io(xq, row * dk + c) : 0.f;
    hk[i] = (t >= 0 && kc) ? ld_io(xk, row * dk + c) : 0.f;
    hv[i] = (t >= 0 && vc) ? ld_io(xv, row * dv + c) : 0.f;
  }
  int par = 0;
  for (int tb = t0; tb < t1; tb += kFwdG, par ^= 1) {
    float nq[kFwdG], nk[kFwdG], s[16];
    // every load of the batch first (the stores below could alias them, which
    // would otherwise keep each token's loads behind the previous token's work)
    float lq[kFwdG], lk[kFwdG], lv[kFwdG], la[kFwdG];
#pragma unroll
    for (int i = 0; i < kFwdG; ++i) {
      const int t = tb + i;
      const bool live = t < t1;
      const size_t row = ((size_t)sq * T + (live ? t : tb)) * H + h;
      lq[i] = (live && kc) ? ld_io(xq, row * dk + c) : 0.f;
      lk[i] = (live && kc) ? ld_io(xk, row * dk + c) : 0.f;
      lv[i] = (live && vc) ? ld_io(xv, row * dv + c) : 0.f;
      la[i] = (live && kc) ? a.a[row * dk + c] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kFwdG; ++i) {
      const int t = tb + i;
      const bool live = t < t1;
      const size_t row = ((size_t)sq * T + (live ? t : tb)) * H + h;
      const float xqt = lq[i], xkt = lk[i], xvt = lv[i];
      // history of token t stops at its document's first token
      const int ds = PACKED ? s_ds[(live ? t : tb) - t0 + 3] : 0;
      const float m3 = !PACKED || t - 3 >= ds ? 1.f : 0.f, m2 = !PACKED || t - 2 >= ds ? 1.f : 0.f,
                  m1 = !PACKED || t - 1 >= ds ? 1.f : 0.f;
      const float yq = wq[0] * m3 * hq[0] + wq[1] * m2 * hq[1] + wq[2] * m1 * hq[2] + wq[3] * xqt;
      const float yk = wk[0] * m3 * hk[0] + wk[1] * m2 * hk[1] + wk[2] * m1 * hk[2] + wk[3] * xkt;
      const float yv = wv[0] * m3 * hv[0] + wv[1] * m2 * hv[1] + wv[2] * m1 * hv[2] + wv[3] * xvt;
      hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xqt;
      hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xkt;
      hv[0] = hv[1]; hv[1] = hv[2]; hv[2] = xvt;
      nq[i] = yq * sigm(yq);
      nk[i] = yk * sigm(yk);
      s[2 * i] = nq[i] * nq[i];
      s[2 * i + 1] = nk[i] * nk[i];
      if (live && vc) st_io((IO *)a.v, row * dv + c, yv * sigm(yv));
      if (live && kc) {
        const float al = tanh_fast(la[i]);
        a.g[row * dk + c] = fmaxf(__logf(fabsf(al)), a.g_floor);
        a.sign[row * dk + c] = al < 0.f ? -1 : 1;
      }
    }
    block_sum16(s, red, par);
#pragma unroll
    for (int i = 0; i < kFwdG; ++i) {
      const int t = tb + i;
      if (t < t1 && kc) {
        const size_t row = ((size_t)sq * T + t) * H + h;
        st_io((IO *)a.q, row * dk + c, nq[i] * rsqrtf(s[2 * i] + kNormEps));
        st_io((IO *)a.k, row * dk + c, nk[i] * rsqrtf(s[2 * i + 1] + kNormEps));
      }
    }
  }
  if (c < kPrTok && t0 + c < T) {
    const size_t row = ((size_t)sq * T + t0 + c) * H + h;
    st_io((IO *)a.beta, row, 2.f * sigm(ld_io((const IO *)a.b, row)));
  }
}

// Backward: 4 tokens per reduction (|n|^2 and n . dn for q and k); the run's
// tokens plus a three-token halo (dx of token s needs dy of s .. s + 3).
constexpr int kBwdG = 4;
template <typename IO, int DK, int DV, bool PACKED>
__global__ void __launch_bounds__(kPrThreads, 4) prologue_bwd_kernel(const PrologueArgs a) {
  __shared__ __align__(16) float red[2][kPrThreads / 32][16];
  __shared__ int s_ds[PACKED ? kPrTok + 8 : 1];
  const int c = threadIdx.x, h = blockIdx.y, sq = blockIdx.z;
  const int T = a.T, H = a.H;
  constexpr int dk = DK, dv = DV;
  const int t0 = blockIdx.x * kPrTok, t1 = min(t0 + kPrTok, T);
  const int tend = min(t0 + kPrTok + 3, T);
  if constexpr (PACKED) {
    doc_starts(a, t0, kPrTok + 6, s_ds);
    __syncthreads();
  }
  // first token of t's document, t in [t0 - 3, t0 + kPrTok + 3) (0 unpacked)
  auto ds_of = [&](int t) { return PACKED ? s_ds[t - t0 + 3] : 0; };
  const bool kc = DK == kPrThreads || c < DK, vc = DV == kPrThreads || c < DV;  // (compile-time true at 128)
  const IO *xq = (const IO *)a.xq, *xk = (const IO *)a.xk, *xv = (const IO *)a.xv;
  const IO *gq = (const IO *)a.dq, *gk = (const IO *)a.dk_in, *gv = (const IO *)a.dv_in;
  float wq[4], wk[4], wv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    wq[j] = kc ? a.wq[((size_t)h * dk + c) * 4 + j] : 0.f;
    wk[j] = kc ? a.wk[((size_t)h * dk + c) * 4 + j] : 0.f;
    wv[j] = vc ? a.wv[((size_t)h * dv + c) * 4 + j] : 0.f;
  }
  float hq[3], hk[3], hv[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int t = t0 - 3 + i;
    const size_t row = ((size_t)sq * T + (t < 0 ? 0 : t)) * H + h;
    hq[i] = (t >= 0 && kc) ? ld_io(xq, row * dk + c) : 0.f;
    hk[i] = (t >= 0 && kc) ? ld_io(xk, row * dk + c) : 0.f;
    hv[i] = (t >= 0 && vc) ? ld_io(xv, row * dv + c) : 0.f;
  }
  // dL/dy of tokens t - 3, t - 2, t - 1; the conv taps' gradient sums
  float eq[3] = {0.f, 0.f, 0.f}, ek[3] = {0.f, 0.f, 0.f}, ev[3] = {0.f, 0.f, 0.f};
  float sq4[4] = {0.f, 0.f, 0.f, 0.f}, sk4[4] = {0.f, 0.f, 0.f, 0.f}, sv4[4] = {0.f, 0.f, 0.f, 0.f};
  int par = 0;
  for (int tb = t0; tb < t1 + 3; tb += kBwdG, par ^= 1) {
    // inputs of the batch's tokens (zero past tend), their conv windows kept for the taps' sums
    float xwq[kBwdG + 3], xwk[kBwdG + 3], xwv[kBwdG + 3];
    xwq[0] = hq[0]; xwq[1] = hq[1]; xwq[2] = hq[2];
    xwk[0] = hk[0]; xwk[1] = hk[1]; xwk[2] = hk[2];
    xwv[0] = hv[0]; xwv[1] = hv[1]; xwv[2] = hv[2];
    float yq[kBwdG], yk[kBwdG], pq[kBwdG], pk[kBwdG], dqt[kBwdG], dkt[kBwdG], dyv[kBwdG], s[16];
    // every load of the batch first (see the forward)
    float ldv[kBwdG], la[kBwdG], lg[kBwdG];
#pragma unroll
    for (int i = 0; i < kBwdG; ++i) {
      const int t = tb + i;
      const bool live = t < tend, own = live && t < t1 && kc;
      const size_t row = ((size_t)sq * T + (live ? t : t0)) * H + h;
      xwq[3 + i] = (live && kc) ? ld_io(xq, row * dk + c) : 0.f;
      xwk[3 + i] = (live && kc) ? ld_io(xk, row * dk + c) : 0.f;
      xwv[3 + i] = (live && vc) ? ld_io(xv, row * dv + c) : 0.f;
      dqt[i] = (live && kc) ? ld_io(gq, row * dk + c) : 0.f;
      dkt[i] = (live && kc) ? ld_io(gk, row * dk + c) : 0.f;
      ldv[i] = (live && vc) ? ld_io(gv, row * dv + c) : 0.f;
      la[i] = own ? a.a[row * dk + c] : 0.f;
      lg[i] = own ? a.dg[row * dk + c] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kBwdG; ++i) {
      const int t = tb + i;
      const bool live = t < tend;
      const size_t row = ((size_t)sq * T + (live ? t : t0)) * H + h;
      const float xqt = xwq[3 + i], xkt = xwk[3 + i], xvt = xwv[3 + i];
      const float dvt = ldv[i];
      const int ds = live ? ds_of(t) : 0;
      const float m3 = !PACKED || t - 3 >= ds ? 1.f : 0.f, m2 = !PACKED || t - 2 >= ds ? 1.f : 0.f,
                  m1 = !PACKED || t - 1 >= ds ? 1.f : 0.f;
      yq[i] = wq[0] * m3 * xwq[i] + wq[1] * m2 * xwq[i + 1] + wq[2] * m1 * xwq[i + 2] + wq[3] * xqt;
      yk[i] = wk[0] * m3 * xwk[i] + wk[1] * m2 * xwk[i + 1] + wk[2] * m1 * xwk[i + 2] + wk[3] * xkt;
      const float yv = wv[0] * m3 * xwv[i] + wv[1] * m2 * xwv[i + 1] + wv[2] * m1 * xwv[i + 2] + wv[3] * xvt;
      pq[i] = sigm(yq[i]);
      pk[i] = sigm(yk[i]);
      const float pv = sigm(yv);
      dyv[i] = live ? dvt * (pv * (1.f + yv * (1.f - pv))) : 0.f;
      const float nq = yq[i] * pq[i], nk = yk[i] * pk[i];
      s[4 * i] = nq * nq;
      s[4 * i + 1] = nk * nk;
      s[4 * i + 2] = nq * dqt[i];
      s[4 * i + 3] = nk * dkt[i];
      if (live && t < t1 && kc) {  // gate: the floor's clamp passes no gradient
        const float al = tanh_fast(la[i]);
        const bool open = __logf(fabsf(al)) > a.g_floor;
        a.da[row * dk + c] = open ? __fdividef(lg[i] * (1.f - al * al), al) : 0.f;
      }
    }
    block_sum16(s, red, par);
#pragma unroll
    for (int i = 0; i < kBwdG; ++i) {
      const int t = tb + i;
      const bool live = t < tend;
      // q = n r, r = (|n|^2 + eps)^(-1/2):  dn = r dq - r^3 (n . dq) n;  SiLU' = p (1 + y (1 - p))
      const float rq = rsqrtf(s[4 * i] + kNormEps), rk = rsqrtf(s[4 * i + 1] + kNormEps);
      const float nq = yq[i] * pq[i], nk = yk[i] * pk[i];
      const float dyq = live ? (rq * dqt[i] - rq * rq * rq * s[4 * i + 2] * nq) * (pq[i] * (1.f + yq[i] * (1.f - pq[i]))) : 0.f;
      const float dyk = live ? (rk * dkt[i] - rk * rk * rk * s[4 * i + 3] * nk) * (pk[i] * (1.f + yk[i] * (1.f - pk[i]))) : 0.f;
      const int so = t - 3;  // dx of token t - 3 is complete
      if (so >= t0 && so < t1) {
        // token so + k reads x_so only inside so's document (so >= its first token)
        const float n1 = !PACKED || so >= ds_of(so + 1) ? 1.f : 0.f;
        const float n2 = !PACKED || so >= ds_of(so + 2) ? 1.f : 0.f;
        const float n3 = !PACKED || (t < T && so >= ds_of(t)) ? 1.f : 0.f;
        const size_t row = ((size_t)sq * T + so) * H + h;
        if (kc) {
          st_io((IO *)a.dxq, row * dk + c,
                wq[3] * eq[0] + wq[2] * n1 * eq[1] + wq[1] * n2 * eq[2] + wq[0] * n3 * dyq);
          st_io((IO *)a.dxk, row * dk + c,
                wk[3] * ek[0] + wk[2] * n1 * ek[1] + wk[1] * n2 * ek[2] + wk[0] * n3 * dyk);
        }
        if (vc)
          st_io((IO *)a.dxv, row * dv + c,
                wv[3] * ev[0] + wv[2] * n1 * ev[1] + wv[1] * n2 * ev[2] + wv[0] * n3 * dyv[i]);
      }
      if (t < t1) {  // the taps' sums over this run's tokens: dy_t x_{t-3+j} (inside t's document)
        const int ds = ds_of(t);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float mj = (!PACKED || j == 3 || t - 3 + j >= ds) ? 1.f : 0.f;
          sq4[j] += mj * dyq * xwq[i + j];
          sk4[j] += mj * dyk * xwk[i + j];
          sv4[j] += mj * dyv[i] * xwv[i + j];
        }
      }
      eq[0] = eq[1]; eq[1] = eq[2]; eq[2] = dyq;
      ek[0] = ek[1]; ek[1] = ek[2]; ek[2] = dyk;
      ev[0] = ev[1]; ev[1] = ev[2]; ev[2] = dyv[i];
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      hq[i] = xwq[kBwdG + i];
      hk[i] = xwk[kBwdG + i];
      hv[i] = xwv[kBwdG + i];
    }
  }
  // the taps' gradients: this run's sums (order of the runs' additions is not fixed)
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (kc) {
      atomicAdd(&a.dwq[((size_t)h * dk + c) * 4 + j], sq4[j]);
      atomicAdd(&a.dwk[((size_t)h * dk + c) * 4 + j], sk4[j]);
    }
    if (vc) atomicAdd(&a.dwv[((size_t)h * dv + c) * 4 + j], sv4[j]);
  }
  if (c < kPrTok && t0 + c < T) {
    const size_t row = ((size_t)sq * T + t0 + c) * H + h;
    const float bt = 2.f * sigm(ld_io((const IO *)a.b, row));
    st_io((IO *)a.db, row, ld_io((const IO *)a.dbeta, row) * bt * (1.f - 0.5f * bt));
  }
}

}  // namespace

cudaError_t prologue(const PrologueLaunch &p, cudaStream_t s) {
  PrologueArgs a{};
  a.B = p.B; a.T = p.T; a.H = p.H; a.dk = p.dk; a.dv = p.dv; a.g_floor = p.g_floor;
  a.xq = p.xq; a.xk = p.xk; a.xv = p.xv; a.b = p.b;
  a.wq = p.wq; a.wk = p.wk; a.wv = p.wv; a.a = p.a;
  a.q = p.q; a.k = p.k; a.v = p.v; a.beta = p.beta; a.g = p.g; a.sign = p.sign;
  a.dq = p.dq; a.dk_in = p.dk_in; a.dv_in = p.dv_in; a.dbeta = p.dbeta; a.dg = p.dg;
  a.dxq = p.dxq; a.dxk = p.dxk; a.dxv = p.dxv; a.db = p.db;
  a.dwq = p.dwq; a.dwk = p.dwk; a.dwv = p.dwv; a.da = p.da;
  a.cu = p.cu; a.N = p.N;
  if ((size_t)p.B * p.T * p.H == 0) return cudaSuccess;
  const dim3 grid((p.T + kPrTok - 1) / kPrTok, p.H, p.B);
  ProfScope prof(p.backward ? "prologue_bwd" : "prologue_fwd", s);
#define CKDA_PRO_LAUNCH(IO, K, V)                                                   \
  do {                                                                              \
    if (p.backward) {                                                               \
      if (a.cu) prologue_bwd_kernel<IO, K, V, true><<<grid, kPrThreads, 0, s>>>(a); \
      else prologue_bwd_kernel<IO, K, V, false><<<grid, kPrThreads, 0, s>>>(a);     \
    } else {                                                                        \
      if (a.cu) prologue_fwd_kernel<IO, K, V, true><<<grid, kPrThreads, 0, s>>>(a); \
      else prologue_fwd_kernel<IO, K, V, false><<<grid, kPrThreads, 0, s>>>(a);     \
    }                                                                               \
  } while (0)
#define CKDA_PRO_DIMS(IO)                                   \
  do {                                                      \
    if (p.dk == 128 && p.dv == 128) CKDA_PRO_LAUNCH(IO, 128, 128); \
    else if (p.dk == 128) CKDA_PRO_LAUNCH(IO, 128, 64);    \
    else if (p.dv == 128) CKDA_PRO_LAUNCH(IO, 64, 128);    \
    else CKDA_PRO_LAUNCH(IO, 64, 64);                      \
  } while (0)
  if (p.bf16) CKDA_PRO_DIMS(__nv_bfloat16);
  else CKDA_PRO_DIMS(float);
#undef CKDA_PRO_DIMS
#undef CKDA_PRO_LAUNCH
  return cudaGetLastError();
}

}  // namespace ckda
