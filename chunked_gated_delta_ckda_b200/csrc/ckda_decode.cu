// ckda_decode.cu -- one recurrent CKDA step for many independent states.
//
// Per (sequence n, head h), with the signed gate applied directly
// ("openeurollm/complex-kda-1.3B-100B" model card: a purely recurrent model,
// alpha in [-1, 1], |alpha| in log space):
//   alpha = sign * exp(g)
//   X = Diag(alpha) S,  u = X^T k,  w = v - u
//   S <- X + beta k w^T                     (= (I - beta k k^T) Diag(alpha) S + beta k v^T)
//   o  = S^T q = X^T q + beta (k.q) w
//
// The state (dk x dv fp32, 64 KiB at 128 x 128) is read once and written
// once: each thread keeps its rows x float4 columns in registers between the
// two reductions (over dk, through shared memory) and the rank-one update.
// A warp reads 32 consecutive float4 of a row: fully coalesced 128-bit
// accesses.  The step is HBM-bound (about 1 flop per byte).
#include "ckda_internal.cuh"

namespace ckda {
namespace {

constexpr int kDecThreads = 256;

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const IO *__restrict__ q,
                                                             const IO *__restrict__ k,
                                                             const IO *__restrict__ v,
                                                             const float *__restrict__ g,
                                                             const int8_t *__restrict__ sign,
                                                             const IO *__restrict__ beta,
                                                             float *__restrict__ state,
                                                             IO *__restrict__ o) {
  constexpr int CG = DV / 4;            // float4 column groups per row
  constexpr int RG = kDecThreads / CG;  // row groups
  constexpr int RPT = DK / RG;          // rows per thread
  static_assert(RPT * RG == DK, "row split");
  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ __align__(16) float s_w[DV];
  __shared__ float4 s_u[RG][CG], s_o[RG][CG];
  __shared__ float s_kq[kDecThreads / 32];
  const size_t nh = blockIdx.x;
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;

  float4 *S4 = reinterpret_cast<float4 *>(state + nh * DK * DV);
  float4 x[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) x[r] = S4[(size_t)(rg * RPT + r) * CG + cg];

  float kq = 0.f;
  for (int i = tid; i < DK; i += kDecThreads) {
    const float kk = ld_io(k, nh * DK + i), qq = ld_io(q, nh * DK + i);
    s_k[i] = kk;
    s_q[i] = qq;
    const float a = expf(g[nh * DK + i]);
    s_a[i] = (sign && sign[nh * DK + i] < 0) ? -a : a;  // no sign tensor: all +1 (KDA)
    kq += kk * qq;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  if ((tid & 31) == 0) s_kq[tid >> 5] = kq;
  __syncthreads();

  float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), po = pu;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg * RPT + r;
    const float a = s_a[i], kk = s_k[i], qq = s_q[i];
    x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
    pu.x += kk * x[r].x; pu.y += kk * x[r].y; pu.z += kk * x[r].z; pu.w += kk * x[r].w;
    po.x += qq * x[r].x; po.y += qq * x[r].y; po.z += qq * x[r].z; po.w += qq * x[r].w;
  }
  s_u[rg][cg] = pu;
  s_o[rg][cg] = po;
  __syncthreads();

  const float bt = ld_io(beta, nh);
  if (tid < DV) {
    float kqs = 0.f;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) kqs += s_kq[w];
    const int c4 = tid >> 2, e = tid & 3;
    float u = 0.f, oo = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      u += reinterpret_cast<const float *>(&s_u[r][c4])[e];
      oo += reinterpret_cast<const float *>(&s_o[r][c4])[e];
    }
    const float w = ld_io(v, nh * DV + tid) - u;
    s_w[tid] = w;
    st_io(o, nh * DV + tid, oo + bt * kqs * w);
  }
  __syncthreads();

  const float4 w4 = reinterpret_cast<const float4 *>(s_w)[cg];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const float bk = bt * s_k[rg * RPT + r];
    float4 y = x[r];
    y.x += bk * w4.x; y.y += bk * w4.y; y.z += bk * w4.z; y.w += bk * w4.w;
    S4[(size_t)(rg * RPT + r) * CG + cg] = y;
  }
}

template <typename IO, int DK, int DV>
cudaError_t launch(int NH, const void *q, const void *k, const void *v, const float *g,
                   const int8_t *sign, const void *beta, float *state, void *o, cudaStream_t s) {
  ProfScope prof("decode", s);
  decode_kernel<IO, DK, DV><<<NH, kDecThreads, 0, s>>>(
      (const IO *)q, (const IO *)k, (const IO *)v, g, sign, (const IO *)beta, state, (IO *)o);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t dispatch(int NH, int dk, int dv, const void *q, const void *k, const void *v,
                     const float *g, const int8_t *sign, const void *beta, float *state,
                     void *o, cudaStream_t s) {
  if (dk == 128 && dv == 128) return launch<IO, 128, 128>(NH, q, k, v, g, sign, beta, state, o, s);
  if (dk == 128 && dv == 64) return launch<IO, 128, 64>(NH, q, k, v, g, sign, beta, state, o, s);
  if (dk == 64 && dv == 128) return launch<IO, 64, 128>(NH, q, k, v, g, sign, beta, state, o, s);
  return launch<IO, 64, 64>(NH, q, k, v, g, sign, beta, state, o, s);
}

// ---------------------------------------------------------------------------
// Several steps per sequence with its state kept in registers: batched
// multi-token decode and speculative verify / commit, states in a slot pool.
// A CTA takes one (sequence, head) and a slice of 32 value columns (the
// columns of S evolve independently: w, o and the rank-one update are per
// column; only the reductions over dk and k.q span the whole key axis).  It
// reads its dk x 32 slice of the state once, runs the steps, and writes the
// slice back once.  Thread (row group rg, column group cg) holds rows
// [RPT rg, RPT rg + RPT) x columns [4 cg, 4 cg + 4) as float4s; the
// arithmetic on them is packed two-lane fp32 (f32x2: one instruction per two
// products).  Token t + 1's inputs are loaded while token t runs; the
// per-channel values are double-buffered in shared memory, so three barriers
// per token suffice.
// ---------------------------------------------------------------------------
constexpr int kMdThreads = 128;
constexpr int kMdSlice = 32;  // value columns per CTA

struct MultiArgs {
  int N, K, H, dv, n_slots, write_state;
  const void *q, *k, *v, *beta;
  const float *g;
  const int8_t *sign;
  const int32_t *n_tokens, *slots;
  float *state;
  void *o;
};

typedef unsigned long long u64;
__device__ __forceinline__ u64 f2(float lo, float hi) {
  return (u64)__float_as_uint(lo) | ((u64)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float lo2(u64 x) { return __uint_as_float((uint32_t)x); }
__device__ __forceinline__ float hi2(u64 x) { return __uint_as_float((uint32_t)(x >> 32)); }

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kMdThreads, 8) decode_multi_kernel(const MultiArgs a) {
  constexpr int CG = kMdSlice / 4;     // float4 column groups of the slice
  constexpr int RG = kMdThreads / CG;  // row groups
  constexpr int RPT = DK / RG;         // rows per thread (8 or 4)
  constexpr int slices = DV / kMdSlice;
  static_assert(RPT * RG == DK && DK <= kMdThreads && RPT % 4 == 0, "row split");
  __shared__ __align__(16) float s_k[2][DK], s_q[2][DK], s_a[2][DK];
  __shared__ __align__(16) float s_u[RG][kMdSlice + 16], s_o[RG][kMdSlice + 16];  // rows 16 banks apart
  __shared__ __align__(16) float s_w[kMdSlice];
  __shared__ float s_kq[kMdThreads / 32];
  const int K = a.K, H = a.H;
  const size_t bx = blockIdx.x;
  const int sl = (int)(bx % slices), h = (int)((bx / slices) % H);
  const size_t n = bx / ((size_t)slices * H);
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG, lane = tid & 31;
  const int col0 = sl * kMdSlice;
  const IO *q = (const IO *)a.q, *k = (const IO *)a.k, *v = (const IO *)a.v, *beta = (const IO *)a.beta;
  IO *o = (IO *)a.o;

  int nt = a.n_tokens ? a.n_tokens[n] : K;
  nt = nt < 0 ? 0 : (nt > K ? K : nt);
  const int slot = a.slots ? a.slots[n] : (int)n;
  const bool skip = slot < 0 || slot >= a.n_slots;
  if (o)  // rows that no step fills
    for (int t = skip ? 0 : nt; t < K; ++t)
      if (tid < kMdSlice) st_io(o, ((n * K + t) * H + h) * DV + col0 + tid, 0.f);
  if (skip || nt == 0) return;

  float4 *S4 = reinterpret_cast<float4 *>(a.state + ((size_t)slot * H + h) * DK * DV + col0) + cg;
  u64 xl[RPT], xh[RPT];  // columns (4 cg, 4 cg + 1) and (4 cg + 2, 4 cg + 3) of each row
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const float4 t4 = S4[(size_t)(rg * RPT + r) * (DV / 4)];
    xl[r] = f2(t4.x, t4.y);
    xh[r] = f2(t4.z, t4.w);
  }

  // token inputs in registers: channel tid (key side), column col0 + tid / 2 (value side)
  float nk = 0.f, nq = 0.f, ng = 0.f, nv = 0.f, nb = 0.f;
  int ns = 1;
  auto fetch = [&](int t) {
    const size_t row = (n * K + t) * H + h;
    if (tid < DK) {
      nk = ld_io(k, row * DK + tid);
      nq = ld_io(q, row * DK + tid);
      ng = a.g[row * DK + tid];
      ns = a.sign ? a.sign[row * DK + tid] : 1;  // no sign tensor: all +1 (KDA)
    }
    if (tid < 2 * kMdSlice) nv = ld_io(v, row * DV + col0 + (tid >> 1));
    nb = ld_io(beta, row);
  };
  fetch(0);
  for (int t = 0; t < nt; ++t) {
    const int b = t & 1;
    const float ck = nk, cq = nq, cgt = ng, cv = nv, bt = nb;
    const int cs = ns;
    if (t + 1 < nt) fetch(t + 1);
    float kq = 0.f;
    if (tid < DK) {
      s_k[b][tid] = ck;
      s_q[b][tid] = cq;
      const float al = expf(cgt);
      s_a[b][tid] = cs < 0 ? -al : al;
      kq = ck * cq;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    if (lane == 0) s_kq[tid >> 5] = kq;
    __syncthreads();
    // X = Diag(alpha) S (in place); partial X^T k and X^T q over this thread's rows
    u64 ul = 0, uh = 0, ol = 0, oh = 0;
#pragma unroll
    for (int r4 = 0; r4 < RPT / 4; ++r4) {
      const int i0 = rg * RPT + 4 * r4;
      const float4 a4 = *reinterpret_cast<const float4 *>(&s_a[b][i0]);
      const float4 k4 = *reinterpret_cast<const float4 *>(&s_k[b][i0]);
      const float4 q4 = *reinterpret_cast<const float4 *>(&s_q[b][i0]);
      const float aa[4] = {a4.x, a4.y, a4.z, a4.w}, kk[4] = {k4.x, k4.y, k4.z, k4.w};
      const float qq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * r4 + i;
        const u64 al = f2(aa[i], aa[i]), k2 = f2(kk[i], kk[i]), q2 = f2(qq[i], qq[i]);
        xl[r] = mul2(xl[r], al);
        xh[r] = mul2(xh[r], al);
        ul = fma2(k2, xl[r], ul);
        uh = fma2(k2, xh[r], uh);
        ol = fma2(q2, xl[r], ol);
        oh = fma2(q2, xh[r], oh);
      }
    }
    *reinterpret_cast<float4 *>(&s_u[rg][4 * cg]) = make_float4(lo2(ul), hi2(ul), lo2(uh), hi2(uh));
    *reinterpret_cast<float4 *>(&s_o[rg][4 * cg]) = make_float4(lo2(ol), hi2(ol), lo2(oh), hi2(oh));
    __syncthreads();
    // column c = tid / 2 summed by a lane pair (even / odd row groups)
    if (tid < 2 * kMdSlice) {
      const int c = tid >> 1, par = tid & 1;
      float u0 = 0.f, u1 = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
      for (int r = par; r < RG; r += 4) {
        u0 += s_u[r][c];
        o0 += s_o[r][c];
        u1 += s_u[r + 2][c];
        o1 += s_o[r + 2][c];
      }
      float u = u0 + u1, oo = o0 + o1;
      u += __shfl_xor_sync(0xffffffffu, u, 1);
      oo += __shfl_xor_sync(0xffffffffu, oo, 1);
      if (!par) {
        float kqs = 0.f;
#pragma unroll
        for (int w = 0; w < kMdThreads / 32; ++w) kqs += s_kq[w];
        const float w = cv - u;
        s_w[c] = w;
        if (o) st_io(o, ((n * K + t) * H + h) * DV + col0 + c, oo + bt * kqs * w);
      }
    }
    __syncthreads();
    // S <- X + (beta k) w^T
    const float4 w4 = reinterpret_cast<const float4 *>(s_w)[cg];
    const u64 wl = f2(w4.x, w4.y), wh = f2(w4.z, w4.w);
#pragma unroll
    for (int r4 = 0; r4 < RPT / 4; ++r4) {
      const float4 k4 = *reinterpret_cast<const float4 *>(&s_k[b][rg * RPT + 4 * r4]);
      const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * r4 + i;
        const u64 bk = f2(bt * kk[i], bt * kk[i]);
        xl[r] = fma2(bk, wl, xl[r]);
        xh[r] = fma2(bk, wh, xh[r]);
      }
    }
  }
  if (a.write_state) {
#pragma unroll
    for (int r = 0; r < RPT; ++r)
      S4[(size_t)(rg * RPT + r) * (DV / 4)] = make_float4(lo2(xl[r]), hi2(xl[r]), lo2(xh[r]), hi2(xh[r]));
  }
}

template <typename IO>
cudaError_t launch_multi(const MultiArgs &m, int dk, cudaStream_t s) {
  const unsigned ctas = (unsigned)((size_t)m.N * m.H * (m.dv / kMdSlice));
  ProfScope prof("decode_multi", s);
  if (dk == 128 && m.dv == 128) decode_multi_kernel<IO, 128, 128><<<ctas, kMdThreads, 0, s>>>(m);
  else if (dk == 128) decode_multi_kernel<IO, 128, 64><<<ctas, kMdThreads, 0, s>>>(m);
  else if (m.dv == 128) decode_multi_kernel<IO, 64, 128><<<ctas, kMdThreads, 0, s>>>(m);
  else decode_multi_kernel<IO, 64, 64><<<ctas, kMdThreads, 0, s>>>(m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t decode_multi(int N, int K, int H, int dk, int dv, bool bf16, const void *q, const void *k,
                         const void *v, const float *g, const int8_t *sign, const void *beta,
                         const int32_t *n_tokens, const int32_t *slots, int n_slots, float *state,
                         bool write_state, void *o, cudaStream_t s) {
  if ((size_t)N * H == 0 || K == 0) return cudaSuccess;
  if ((size_t)N * H * (dv / kMdSlice) > 0x7fffffffu) return cudaErrorInvalidConfiguration;
  MultiArgs m{};
  m.N = N; m.K = K; m.H = H; m.dv = dv; m.n_slots = n_slots; m.write_state = write_state ? 1 : 0;
  m.q = q; m.k = k; m.v = v; m.beta = beta; m.g = g; m.sign = sign;
  m.n_tokens = n_tokens; m.slots = slots; m.state = state; m.o = o;
  return bf16 ? launch_multi<__nv_bfloat16>(m, dk, s) : launch_multi<float>(m, dk, s);
}

cudaError_t decode_step(int N, int H, int dk, int dv, bool bf16, const void *q, const void *k,
                        const void *v, const float *g, const int8_t *sign, const void *beta,
                        float *state, void *o, cudaStream_t s) {
  const int NH = N * H;
  if (NH == 0) return cudaSuccess;
  return bf16 ? dispatch<__nv_bfloat16>(NH, dk, dv, q, k, v, g, sign, beta, state, o, s)
              : dispatch<float>(NH, dk, dv, q, k, v, g, sign, beta, state, o, s);
}

}  // namespace ckda
