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

}  // namespace

cudaError_t decode_step(int N, int H, int dk, int dv, bool bf16, const void *q, const void *k,
                        const void *v, const float *g, const int8_t *sign, const void *beta,
                        float *state, void *o, cudaStream_t s) {
  const int NH = N * H;
  if (NH == 0) return cudaSuccess;
  return bf16 ? dispatch<__nv_bfloat16>(NH, dk, dv, q, k, v, g, sign, beta, state, o, s)
              : dispatch<float>(NH, dk, dv, q, k, v, g, sign, beta, state, o, s);
}

}  // namespace ckda
