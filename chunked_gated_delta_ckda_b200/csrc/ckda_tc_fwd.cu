// ckda_tc_fwd.cu -- chunked CKDA forward on 5th-generation tensor cores
// (tcgen05, TMEM accumulators), bf16 I/O, dk = dv = 128.
//
// Same algorithm as the CUDA-core path (chunk-wise WY / UT form with the
// gate sign folded per chunk; "Complex KDA: Understanding and Enhancing the
// Expressivity of Kimi Delta Attention", section 2, and the
// "openeurollm/complex-kda-1.3B-100B" model card introduction), split in two
// kernels:
//
//  tc_intra_kernel  (persistent, 2 CTAs / SM, one (chunk, head) at a time)
//    prep on CUDA cores: chunk-local cumsum Gam and sign product p, the
//      factored operands Q~ = q' e^{Gam-Gam_m}, K~l = k' e^{Gam-Gam_m},
//      K~r = k' e^{Gam_m-Gam}, KG = k' e^Gam, QG = q' e^Gam,
//      Khat = p_C k' e^{Gam_C-Gam}, d = p_C e^{Gam_C}
//    MMA1  [A_q ; A] = [Q~ ; K~l] K~r^T           (M=128, N=64, K=128)
//    triangular inverse M = (I + Diag(beta) A)^{-1}, 16x16 blocks, fp32
//    MMA2  W^T = KG^T T^T, U0^T = V^T T^T          (M=128, N=64, K=64 each)
//    -> one record per (chunk, head), written in the shared-memory image
//       the state kernel consumes (128-byte-swizzled operand tiles).
//
//  tc_state_kernel  (one CTA per (sequence, head), sequential over chunks)
//    the state is kept transposed, S^T (lanes = value channel), fp32 in TMEM;
//    records arrive by one bulk async copy each, double-buffered.
//    MMA3  [(W S)^T | (QG S)^T] = S^T [W^T | QG^T]  (M=128, N=128, K=128)
//    U^T = U0^T - (W S)^T                           (CUDA cores, -> bf16 tile)
//    MMA4  O^T += U^T A_q^T                         (M=128, N=64,  K=64)
//    MMA5  S^T += U^T Khat                          (M=128, N=128, K=64)
//    S^T <- Diag(d_next) S^T and its bf16 copy for the next MMA3.
//
// Chunks whose decay is too strong for the factored operands (any
// |Gam_r - Gam_m| > kTau) compute A and A_q exactly per pair on CUDA cores.
#include <cmath>

#include "ckda_tc.cuh"

namespace ckda {
namespace {

using namespace tc;

constexpr uint32_t REC_PAD = 74752;  // record slot in shared memory (73 x 1024)
static_assert(REC_STATE <= REC_PAD, "the state pass's part of a record fits its slot");

// ===========================================================================
// intra-chunk kernel
// ===========================================================================
constexpr int kIntraThreads = 256;
// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t I_A1 = 0;          // [Q~; K~l]  K-major 128 x 128      32 KiB
constexpr uint32_t I_B1 = 32768;      // K~r        K-major  64 x 128      16 KiB
constexpr uint32_t I_KG = 49152;      // KG         MN-major A (K=64, M=128) 16 KiB
constexpr uint32_t I_V = 65536;       // V          MN-major A (K=64, M=128) 16 KiB
constexpr uint32_t I_T = 81920;       // T          K-major 64 x 64         8 KiB
constexpr uint32_t I_QGS = 90112;     // QG^T staging, MN-major [c][r] 128 x 64 (the record's R1 upper half)
constexpr uint32_t I_MISC = I_QGS + 16384;  // small arrays
constexpr uint32_t I_XS = 43008;      // inverse scratch 3 x 16 x 16 fp32 (in B1, dead after MMA1)
constexpr uint32_t I_NF = 0;          // fp32 N [64][65]  (reuses A1 after MMA1)
constexpr uint32_t I_MF = 16640;      // fp32 M [64][65]  (reuses A1/B1 after MMA1)
// record tiles staged in shared memory and written out by bulk copies
constexpr uint32_t I_AQS = 34816;     // A_q, K-major [r][s] 64 x 64 (in B1, free after MMA1)
constexpr uint32_t I_WS = I_KG;       // W^T, MN-major [c][r]  (KG, free after MMA2)
constexpr uint32_t I_US = I_V;        // U0^T, K-major [v][s]   (V, free after MMA2)
constexpr int LDF = 65;

struct IntraMisc {
  uint64_t mbar1, mbar2, mfin, mld;
  uint32_t tmem;
  int flag;
  float beta[64];
  PrepTot tot;
};
static_assert(I_XS >= I_AQS + 8192 && I_XS + 3 * 16 * 16 * 4 <= I_KG, "inverse scratch in the dead part of B1");

struct TcArgs {
  RowMaps rm;           // q, k, v, g, sign (intra-chunk kernel)
  FwdArgs f;
  unsigned char *recs;  // (chunk, head) records
  float *fb;            // per-CTA fallback scratch: Gam, k', q' (3 x 64 x 128 fp32)
  float *states_out;    // chunk-start states (batched only) or null
  bool write_o;
  bool state_tiles;     // the state pass also stores each chunk-start state (bf16) in its record
  // segment mode (long sequences, few of them): the chunks of a sequence are
  // split into seg_count segments of seg_len chunks; blockIdx.y = seq *
  // seg_count + segment in the segment kernels and the state pass
  int seg_len, seg_count;
  float *seg_M, *seg_b;  // per segment: its affine map S -> M S + b (fp32 [128][128] each)
  float *seg_S0;         // per segment: its start state (fp32 [128][128])
  bool seg_M_rows;       // the map kernel writes M itself ([c][j]) instead of M^T ([j][c])
  bool seg_reverse;      // the scan runs from the last segment down (adjoint states)
  const float *seg_X0;   // the scan's first state (null: zero)
};

__global__ void __launch_bounds__(kIntraThreads, 2) tc_intra_kernel(const __grid_constant__ TcArgs ta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  IntraMisc &ms = *reinterpret_cast<IntraMisc *>(sm + I_MISC);
  const FwdArgs &a = ta.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const __nv_bfloat16 *beta = (const __nv_bfloat16 *)a.beta;

  if (tid == 0) {
    mbar_init(&ms.mbar1, 1);
    mbar_init(&ms.mbar2, 2);  // W^T and U0^T are issued by two threads
    mbar_init(&ms.mfin, 2);
    mbar_init(&ms.mld, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem;
  const uint32_t sA1 = smem_u32(sm + I_A1), sB1 = smem_u32(sm + I_B1);
  const uint32_t sKG = smem_u32(sm + I_KG), sV = smem_u32(sm + I_V), sT = smem_u32(sm + I_T);
  float *Nf = reinterpret_cast<float *>(sm + I_NF);
  float *Mf = reinterpret_cast<float *>(sm + I_MF);
  float *fb = ta.fb + (size_t)blockIdx.x * 3 * 64 * D;

  const int nitems = a.map.n_chunks() * H;
  uint32_t it = 0;
  bool abort = false;
  for (int item = blockIdx.x; item < nitems && !abort; item += gridDim.x, ++it) {
    const int cid = item / H, h = item % H;
    int seq, len, jl;
    int64_t tok0;
    a.map.info(cid, seq, tok0, len, jl);
    unsigned char *rec = ta.recs + (size_t)item * REC;

    // ---------------- loads: one TMA box per 64-row tile, one barrier ----------------
    // q, k staged in the A1 region, g in B1 + KG, sign in T (each consumed by
    // the prep before those tiles are written); V straight into its operand
    // tile (MN-major A, K = token j, M = value channel: the box layout).
    // (issued from lane 0 of four warps; warp 0 posts the byte count with its
    // arrive, so the phase cannot complete before every copy has landed)
    if (lane == 0 && warp < 4) {
      fence_async_smem();  // earlier generic accesses of these regions come first
      const int t = (int)tok0;
      if (warp == 0) {
        mbar_arrive_expect_tx(&ms.mld, kRowBytesQK + kRowBytesG + (a.sign ? kRowBytesSign : 0) + 16384);
        tma_rows(sm + I_A1 + kStageQ, &ta.rm.q, 0, h, t, &ms.mld);
        tma_rows(sm + I_A1 + kStageQ + 8192, &ta.rm.q, 64, h, t, &ms.mld);
      } else if (warp == 1) {
        tma_rows(sm + I_A1 + kStageK, &ta.rm.k, 0, h, t, &ms.mld);
        tma_rows(sm + I_A1 + kStageK + 8192, &ta.rm.k, 64, h, t, &ms.mld);
      } else if (warp == 2) {
        tma_rows(sm + I_B1, &ta.rm.g, 0, h, t, &ms.mld);
        if (a.sign) tma_rows(sm + I_T, &ta.rm.sign, 0, h, t, &ms.mld);
      } else {
        tma_rows(sm + I_V, &ta.rm.v, 0, h, t, &ms.mld);
        tma_rows(sm + I_V + 8192, &ta.rm.v, 64, h, t, &ms.mld);
      }
    }
    if (tid < 64) ms.beta[tid] = tid < len ? __bfloat162float(beta[(size_t)(tok0 + tid) * H + h]) : 0.f;
    {
      const bool ok = mbar_wait_ool(&ms.mld, it & 1, a.status, 100);
      if (__syncthreads_or(!ok)) { abort = true; break; }
    }
    // ---------------- prep: row-group layout (rows 8w.., channels 4l..) ----------------
    Prep P;
    prep_load_smem(sm + I_A1, reinterpret_cast<const float *>(sm + I_B1), a.sign ? sm + I_T : nullptr, len, warp,
                   lane, P, ms.tot);
    if (len < 64) zero_tail_rows(sm + I_V, 8192, len, tid, kIntraThreads);  // V rows past the chunk
    __syncthreads();
    prep_carry(warp, lane, P, ms.tot);
    int bad = 0;
#pragma unroll
    for (int rr = 0; rr < 8; ++rr)
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (!(fabsf(P.G[rr][m] - P.Gm[m]) <= kTau)) bad = 1;
    const bool fast = !__syncthreads_or(bad);
    float eGm[4], eCm[4], pCs[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      eGm[m] = fast_exp(P.Gm[m]);
      eCm[m] = fast_exp(P.GC[m] - P.Gm[m]);
      pCs[m] = ((P.pC >> m) & 1u) ? -1.f : 1.f;
    }
    if (warp == 0)
      *reinterpret_cast<float4 *>(rec + R5 + 16 * lane) =
          make_float4(pCs[0] * fast_exp(P.GC[0]), pCs[1] * fast_exp(P.GC[1]), pCs[2] * fast_exp(P.GC[2]),
                      pCs[3] * fast_exp(P.GC[3]));

    // ---------------- operand tiles and record tiles ----------------
    {
      float qg[8][4], kh[8][4];
      if (fast) {
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * warp + rr;
          float ql[4], kl[4], kr[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float p = prep_p(P, rr, m);
            const float kp = p * prep_k(P, rr, m), qp = p * prep_q(P, rr, m);
            const float el = fast_exp(P.G[rr][m] - P.Gm[m]);
            const float er = rcp_approx(el);
            ql[m] = qp * el;
            kl[m] = kp * el;
            kr[m] = kp * er;
            qg[rr][m] = ql[m] * eGm[m];
            kh[rr][m] = pCs[m] * kr[m] * eCm[m];
          }
          st_bf16x4(sm + I_A1, kmaj_off(r, 4 * lane, 128), ql[0], ql[1], ql[2], ql[3]);
          st_bf16x4(sm + I_A1, kmaj_off(64 + r, 4 * lane, 128), kl[0], kl[1], kl[2], kl[3]);
          st_bf16x4(sm + I_B1, kmaj_off(r, 4 * lane, 64), kr[0], kr[1], kr[2], kr[3]);
          st_bf16x4(sm + I_KG, mnmaj_off(r, 4 * lane, 64), kl[0] * eGm[0], kl[1] * eGm[1], kl[2] * eGm[2],
                    kl[3] * eGm[3]);
        }
      } else {
        // exact path: keep Gam, k', q' for the per-pair sums; KG, QG, Khat directly
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = 8 * warp + rr;
          float kp4[4], qp4[4], g4[4], kg4[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float p = prep_p(P, rr, m);
            kp4[m] = p * prep_k(P, rr, m);
            qp4[m] = p * prep_q(P, rr, m);
            g4[m] = P.G[rr][m];
            const float E = fast_exp(g4[m]);
            kg4[m] = kp4[m] * E;
            qg[rr][m] = qp4[m] * E;
            kh[rr][m] = pCs[m] * kp4[m] * fast_exp(P.GC[m] - g4[m]);
          }
          *reinterpret_cast<float4 *>(fb + r * D + 4 * lane) = make_float4(g4[0], g4[1], g4[2], g4[3]);
          *reinterpret_cast<float4 *>(fb + 64 * D + r * D + 4 * lane) = make_float4(kp4[0], kp4[1], kp4[2], kp4[3]);
          *reinterpret_cast<float4 *>(fb + 128 * D + r * D + 4 * lane) = make_float4(qp4[0], qp4[1], qp4[2], qp4[3]);
          st_bf16x4(sm + I_KG, mnmaj_off(r, 4 * lane, 64), kg4[0], kg4[1], kg4[2], kg4[3]);
        }
      }
      // QG^T (N index 64 + r) and Khat^T (K index r) of each channel: one 16-byte chunk
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cch = 4 * lane + m;
        *reinterpret_cast<uint4 *>(sm + I_QGS + mnmaj_off(cch, 8 * warp, 128)) =
            make_uint4(pack_bf16(qg[0][m], qg[1][m]), pack_bf16(qg[2][m], qg[3][m]),
                       pack_bf16(qg[4][m], qg[5][m]), pack_bf16(qg[6][m], qg[7][m]));
        *reinterpret_cast<uint4 *>(rec + R4 + kmaj_off(cch, 8 * warp, 128)) =
            make_uint4(pack_bf16(kh[0][m], kh[1][m]), pack_bf16(kh[2][m], kh[3][m]),
                       pack_bf16(kh[4][m], kh[5][m]), pack_bf16(kh[6][m], kh[7][m]));
      }
    }
    fence_async_smem();
    __syncthreads();

    // ---------------- A_q and N = Diag(beta) A ----------------
    if (fast) {
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = sdesc_off(sdesc(sA1, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32);
          const uint64_t bd = sdesc_off(sdesc(sB1, 16, 1024), (kk >> 2) * 8192 + (kk & 3) * 32);
          mma_bf16(tmem, ad, bd, id, kk > 0);
        }
        mma_commit(&ms.mbar1);
        bulk_s2g(rec + R1 + 16384, sm + I_QGS, 16384);  // the staged QG^T half of the record
        bulk_commit();
      }
      bool ok = true;
      if (tid == 0) ok = mbar_wait_ool(&ms.mbar1, it & 1, a.status, 101);
      if (__syncthreads_or(!ok)) { abort = true; break; }
      tc_fence_after();
      const int qd = warp & 3, ch = warp >> 2;
      const int L = 32 * qd + lane;
      float x[16], y[16];
      tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + 32 * ch, x);
      tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + 32 * ch + 16, y);
      tmem_wait_ld();
      if (L < 64) {
        const int r = L;
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int s0 = 32 * ch + 2 * j;
          const float v0 = (j < 8 ? x[2 * j] : y[2 * j - 16]);
          const float v1 = (j < 8 ? x[2 * j + 1] : y[2 * j + 1 - 16]);
          pk[j] = pack_bf16(s0 <= r ? v0 : 0.f, s0 + 1 <= r ? v1 : 0.f);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4 *>(sm + I_AQS + kmaj_off(r, 32 * ch + 8 * m, 64)) =
              make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();  // all TMEM reads of MMA1's accumulator done before A1 is reused
      if (tid == 0) {
        bulk_s2g(rec + R3, sm + I_AQS, 8192);
        bulk_commit();
      }
      if (L >= 64) {
        const int r = L - 64;
        const float br = ms.beta[r];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int s = 32 * ch + j;
          const float val = j < 16 ? x[j] : y[j - 16];
          Nf[r * LDF + s] = s < r ? br * val : 0.f;
        }
      }
    } else {
      if (tid == 0) {
        bulk_s2g(rec + R1 + 16384, sm + I_QGS, 16384);  // the staged QG^T half of the record
        bulk_commit();
      }
      // exact per-pair sums (fallback scratch is per CTA, global)
      for (int e = tid; e < 64 * 64; e += kIntraThreads) {
        const int r = e >> 6, s = e & 63;
        float aa = 0.f, aq = 0.f;
        if (s <= r)
          for (int cc = 0; cc < D; ++cc) {
            const float ex = expf(fb[r * D + cc] - fb[s * D + cc]);
            const float ks = fb[64 * D + s * D + cc] * ex;
            aa += fb[64 * D + r * D + cc] * ks;
            aq += fb[128 * D + r * D + cc] * ks;
          }
        Nf[r * LDF + s] = s < r ? ms.beta[r] * aa : 0.f;
        st_bf16(sm + I_AQS, kmaj_off(r, s, 64), s <= r ? aq : 0.f);
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        bulk_s2g(rec + R3, sm + I_AQS, 8192);
        bulk_commit();
      }
    }
    __syncthreads();

    // ---------------- M = (I + N)^{-1}, 16 x 16 blocks ----------------
    inverse64(Mf, Nf, reinterpret_cast<float(*)[16][16]>(sm + I_XS));
    // T = M Diag(beta) -> bf16 K-major B tile [r][j]
    {
      const int r = tid >> 2, j0 = (tid & 3) * 16;
      uint32_t pk[8];
#pragma unroll
      for (int m = 0; m < 8; ++m)
        pk[m] = pack_bf16(Mf[r * LDF + j0 + 2 * m] * ms.beta[j0 + 2 * m],
                          Mf[r * LDF + j0 + 2 * m + 1] * ms.beta[j0 + 2 * m + 1]);
      *reinterpret_cast<uint4 *>(sm + I_T + kmaj_off(r, j0, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4 *>(sm + I_T + kmaj_off(r, j0 + 8, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {  // M and T go to the record too: the backward starts from them
      bulk_s2g(rec + R6, Mf, 64 * LDF * 4);
      bulk_s2g(rec + R8, sm + I_T, 8192);
      bulk_commit();
    }

    // ---------------- W^T = KG^T T^T, U0^T = V^T T^T ----------------
    if (tid == 0 || tid == 32) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, true, false);
      const uint32_t dst = tid == 0 ? 64 : 128;
      const uint64_t ad = tid == 0 ? sdesc(sKG, 8192, 1024) : sdesc(sV, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + dst, sdesc_off(ad, kk * 2048), sdesc_off(sdesc(sT, 16, 1024), kk * 32), id, kk > 0);
      mma_commit(&ms.mbar2);
    }
    {
      bool ok = true;
      if (tid == 0) ok = mbar_wait_ool(&ms.mbar2, it & 1, a.status, 102);
      if (__syncthreads_or(!ok)) { abort = true; break; }
    }
    tc_fence_after();
    {
      const int qd = warp & 3, ch = warp >> 2;
      const int L = 32 * qd + lane;  // c for W^T, v for U0^T
      const uint32_t lanebase = tmem + ((uint32_t)(32 * qd) << 16);
      float x[16], y[16];
      tmem_ld16(lanebase + 64 + 32 * ch, x);
      tmem_ld16(lanebase + 64 + 32 * ch + 16, y);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[8 + j] = pack_bf16(y[2 * j], y[2 * j + 1]);
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<uint4 *>(sm + I_WS + mnmaj_off(L, 32 * ch + 8 * m, 128)) =
            make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
      tmem_ld16(lanebase + 128 + 32 * ch, x);
      tmem_ld16(lanebase + 128 + 32 * ch + 16, y);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[8 + j] = pack_bf16(y[2 * j], y[2 * j + 1]);
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<uint4 *>(sm + I_US + kmaj_off(L, 32 * ch + 8 * m, 128)) =
            make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      // W^T and U0^T out; every staged tile has left shared memory before the
      // next item's loads land there
      bulk_s2g(rec + R1, sm + I_WS, 16384);
      bulk_s2g(rec + R2, sm + I_US, 16384);
      bulk_commit();
      bulk_wait_read_all();
    }
    __syncthreads();
  }
  if (tid == 0) bulk_wait_all();  // every record tile written before the kernel ends
  // wind down: make sure no MMA is still writing TMEM before freeing it
  if (abort && tid == 32) mma_commit(&ms.mfin);
  if (abort && tid == 0) {
    mma_commit(&ms.mfin);
    mbar_wait_ool(&ms.mfin, 0, a.status, 109);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ===========================================================================
// sequential state kernel
// ===========================================================================
constexpr int kStateThreads = 512;   // two warp groups of 256 (two warps per TMEM lane quadrant each)
constexpr int kGroup = 256;
constexpr int kTileStorer = 64;      // group A thread that issues the state tiles' bulk stores
constexpr uint32_t S_REC0 = 0;
constexpr uint32_t S_REC1 = REC_PAD;
constexpr uint32_t S_TS = 2 * REC_PAD;          // S^T bf16, K-major [v][c] 128 x 128
constexpr uint32_t S_TU = S_TS + 32768;         // U^T bf16, K-major [v][s] 128 x 64
constexpr uint32_t S_OST = S_TU + 16384;        // output rows of a chunk, bf16 [64][128] (group B's staging)
constexpr uint32_t S_MISC = S_OST + 16384;

struct StateMisc {
  uint64_t mrec[2], m3, m4, mfin, sready, sdone;
  uint32_t tmem;
};

// TMEM columns: S^T [0,128); per chunk parity p the MMA3/4 accumulator
// [(W S)^T | O^T] at 128 + 128 p.
//
// Two warp groups.  Group A (warps 0-7) runs the chain that carries the
// state: U^T from MMA3, MMA4/5, the bf16 copy of the new state, the next
// MMA3.  Group B (warps 8-15) takes what is off that chain: it writes the
// chunk states out, scales S^T by the next chunk's decay in TMEM (needed only
// by the next MMA5) and writes the chunk's output rows.  They hand off through
// two mbarriers, one arrive per warp: sready (A: S_{j+1} and O_j are in TMEM)
// and sdone (B: S^T is scaled and O_j has been read).
__global__ void __launch_bounds__(kStateThreads, 1) tc_state_kernel(TcArgs ta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  StateMisc &ms = *reinterpret_cast<StateMisc *>(sm + S_MISC);
  const FwdArgs &a = ta.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool grpA = tid < kGroup;
  const int gt = tid & (kGroup - 1);
  const int qd = warp & 3, ch = (warp >> 2) & 1;
  const int h = blockIdx.x, H = a.H;
  const int v = 32 * qd + lane;  // value channel = TMEM lane
  __nv_bfloat16 *o = (__nv_bfloat16 *)a.o;

  // this CTA's chunks: a whole sequence, or one segment of it (whose start
  // state comes from the segment scan; only the last segment has the final state)
  int seq = blockIdx.y, j0 = 0;
  int first;
  int nc = 0;
  const float *S0p;
  bool last_seg = true;
  if (ta.seg_len > 0) {
    seq = blockIdx.y / ta.seg_count;
    const int sg = blockIdx.y % ta.seg_count;
    nc = a.map.seq_chunks(seq, first);
    j0 = sg * ta.seg_len;
    nc = nc - j0 < ta.seg_len ? nc - j0 : ta.seg_len;
    if (nc < 0) nc = 0;
    first += j0;
    S0p = ta.seg_S0 + ((size_t)blockIdx.y * H + h) * D * D;
    last_seg = sg == ta.seg_count - 1;
  } else {
    nc = a.map.seq_chunks(seq, first);
    S0p = a.S0 ? a.S0 + ((size_t)seq * H + h) * D * D : nullptr;
  }
  float *STp = (a.ST && last_seg) ? a.ST + ((size_t)seq * H + h) * D * D : nullptr;
  const int NCb = a.map.NC;

  if (tid == 0) {
    mbar_init(&ms.mrec[0], 1);
    mbar_init(&ms.mrec[1], 1);
    mbar_init(&ms.m3, 1);
    mbar_init(&ms.m4, 2);  // MMA4 and MMA5 are issued by two threads
    mbar_init(&ms.mfin, 2);
    mbar_init(&ms.sready, kGroup / 32);
    mbar_init(&ms.sdone, kGroup / 32);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem;
  const uint32_t lanebase = tmem + ((uint32_t)(32 * qd) << 16);
  unsigned char *recbuf[2] = {sm + S_REC0, sm + S_REC1};
  auto record = [&](int j) -> const unsigned char * {
    return ta.recs + ((size_t)(first + j) * H + h) * REC;
  };
  auto issue_mma3 = [&](int j) {  // by a whole warp
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, 128, false, true);
    const uint32_t sS = smem_u32(sm + S_TS), sR = smem_u32(sm + (j & 1) * S_REC1 + R1);
    const uint64_t dA = sdesc(sS, 16, 1024), dB = sdesc(sR, 16384, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_warp(tmem + 128 + 128 * (j & 1), sdesc_off(dA, (kk >> 2) * 16384 + (kk & 3) * 32),
                    sdesc_off(dB, kk * 2048), id, kk > 0);
    mma_commit_warp(&ms.m3);
  };
  if (tid == 0) {
    for (int j = 0; j < 2 && j < nc; ++j) {
      mbar_arrive_expect_tx(&ms.mrec[j], REC_STATE);
      bulk_g2s(recbuf[j], record(j), REC_STATE, &ms.mrec[j]);
    }
  }
  bool abort = false;
  // initial state (group A): S^T row v = column v of S0; bf16 copy and Diag(d_0)-scaled fp32
  {
    bool ok = true;
    if (grpA && nc > 0) ok = mbar_wait(&ms.mrec[0], 0, a.status, 201);
    if (__syncthreads_or(!ok)) abort = true;
    if (!abort && grpA) {
      const float *d0 = reinterpret_cast<const float *>(recbuf[0] + R5);
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
        float sv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[i] = S0p ? S0p[(size_t)(c0 + i) * D + v] : 0.f;
        if (nc == 0) {
          if (STp)
            for (int i = 0; i < 16; ++i) STp[(size_t)(c0 + i) * D + v] = sv[i];
          continue;
        }
        if (ta.states_out)
          for (int i = 0; i < 16; ++i)
            ta.states_out[(((size_t)seq * H + h) * NCb + j0) * D * D + (size_t)(c0 + i) * D + v] = sv[i];
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(sv[2 * m], sv[2 * m + 1]);
        *reinterpret_cast<uint4 *>(sm + S_TS + kmaj_off(v, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4 *>(sm + S_TS + kmaj_off(v, c0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[i] *= d0[c0 + i];
        tmem_st16(lanebase + c0, sv);
      }
      tmem_wait_st();
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (!abort && warp == 0 && nc > 0) issue_mma3(0);
  if (!abort && tid == kTileStorer && nc > 0 && ta.state_tiles) {  // S_0 for the backward
    bulk_s2g(const_cast<unsigned char *>(record(0)) + R7, sm + S_TS, 32768);
    bulk_commit();
  }

  if (grpA) {
    // one thread polls, the group meets at its own barrier (id 1)
    auto wait_a = [&](uint64_t *bar, uint32_t phase, uint32_t site, bool ok_in) -> bool {
      bool ok = ok_in;
      if (gt == 0 && ok) ok = mbar_wait(bar, phase, a.status, site);
      return !group_sync_or(1, kGroup, !ok);
    };
    for (int j = 0; j < nc && !abort; ++j) {
      const int buf = j & 1;
      unsigned char *rec = recbuf[buf];
      const uint32_t acc = 128 + 128 * buf;  // [(W S)^T | O^T] of this chunk
      if (!wait_a(&ms.m3, j & 1, 203, true)) { abort = true; break; }
      tc_fence_after();
      // U^T = U0^T - (W S)^T  -> bf16 K-major tile [v][s]; this thread: s in [32 ch, 32 ch + 32)
      for (int s0 = 32 * ch; s0 < 32 * ch + 32; s0 += 16) {
        float w[16];
        tmem_ld16(lanebase + acc + s0, w);
        tmem_wait_ld();
        const uint4 u0a = *reinterpret_cast<const uint4 *>(rec + R2 + kmaj_off(v, s0, 128));
        const uint4 u0b = *reinterpret_cast<const uint4 *>(rec + R2 + kmaj_off(v, s0 + 8, 128));
        const __nv_bfloat16 *ua = reinterpret_cast<const __nv_bfloat16 *>(&u0a);
        const __nv_bfloat16 *ub = reinterpret_cast<const __nv_bfloat16 *>(&u0b);
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          pk[m] = pack_bf16(__bfloat162float(ua[2 * m]) - w[2 * m], __bfloat162float(ua[2 * m + 1]) - w[2 * m + 1]);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          pk[4 + m] = pack_bf16(__bfloat162float(ub[2 * m]) - w[8 + 2 * m],
                                __bfloat162float(ub[2 * m + 1]) - w[8 + 2 * m + 1]);
        *reinterpret_cast<uint4 *>(sm + S_TU + kmaj_off(v, s0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4 *>(sm + S_TU + kmaj_off(v, s0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_async_smem();
      tc_fence_before();
      group_sync(1, kGroup);
      // MMA4: O^T += U^T A_q^T (warp 1, at once); MMA5: S^T += U^T Khat (warp 0,
      // once group B has scaled S^T); each issued by one elected lane of its warp
      bool ok = true;
      if (warp == 1) {
        tc_fence_after();
        const uint32_t id4 = idesc_bf16(128, 64, false, false);
        const uint64_t dA = sdesc(smem_u32(sm + S_TU), 16, 1024), dB = sdesc(smem_u32(rec + R3), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_warp(tmem + acc + 64, sdesc_off(dA, kk * 32), sdesc_off(dB, kk * 32), id4, true);
        mma_commit_warp(&ms.m4);
      }
      if (warp == 0) {
        if (j > 0) ok = mbar_wait(&ms.sdone, (j - 1) & 1, a.status, 206);
        ok = __all_sync(0xffffffffu, ok);  // (the same lane issues and commits)
        if (ok) {
          tc_fence_after();
          const uint32_t id5 = idesc_bf16(128, 128, false, false);
          const uint64_t dA = sdesc(smem_u32(sm + S_TU), 16, 1024), dB = sdesc(smem_u32(rec + R4), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16_warp(tmem + 0, sdesc_off(dA, kk * 32), sdesc_off(dB, kk * 32), id5, true);
        }
        mma_commit_warp(&ms.m4);  // also on failure: the other arrival must not wait on a missing one
      }
      if (tid == kTileStorer) bulk_wait_read_all();  // the last state tile has left S_TS
      if (!wait_a(&ms.m4, j & 1, 204, ok)) { abort = true; break; }
      tc_fence_after();
      // the record buffer is free again: fetch chunk j + 2 into it
      if (gt == 0 && j + 2 < nc) {
        mbar_arrive_expect_tx(&ms.mrec[buf], REC_STATE);
        bulk_g2s(rec, record(j + 2), REC_STATE, &ms.mrec[buf]);
      }
      if (j + 1 < nc) {
        // bf16 copy of S_{j+1} for the next MMA3 (columns c in [64 ch, 64 ch + 64))
        for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
          float sv[16];
          tmem_ld16(lanebase + c0, sv);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(sv[2 * m], sv[2 * m + 1]);
          *reinterpret_cast<uint4 *>(sm + S_TS + kmaj_off(v, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4 *>(sm + S_TS + kmaj_off(v, c0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        fence_async_smem();
      }
      // S_{j+1} and O_j are in TMEM, and this warp has read S_{j+1}: hand them
      // to group B (which scales S^T in place) before the next MMA3 is issued
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.sready);
      if (j + 1 < nc) {
        if (!wait_a(&ms.mrec[buf ^ 1], ((j + 1) >> 1) & 1, 205, true)) { abort = true; break; }
        if (warp == 0) issue_mma3(j + 1);
        if (tid == kTileStorer && ta.state_tiles) {  // S_{j+1} for the backward (off the MMA issuer)
          bulk_s2g(const_cast<unsigned char *>(record(j + 1)) + R7, sm + S_TS, 32768);
          bulk_commit();
        }
      }
    }
  } else {
    for (int j = 0; j < nc && !abort; ++j) {
      const int buf = j & 1;
      const uint32_t acc = 128 + 128 * buf;
      int sq, len, jl;
      int64_t tok0;
      a.map.info(first + j, sq, tok0, len, jl);
      const bool last = (j + 1 == nc);
      bool ok = mbar_wait(&ms.sready, j & 1, a.status, 207);
      if (ok && !last) ok = mbar_wait(&ms.mrec[buf ^ 1], ((j + 1) >> 1) & 1, a.status, 208);
      if (group_sync_or(2, kGroup, !ok)) { abort = true; break; }
      tc_fence_after();
      // output rows of this chunk, rows [32 ch, 32 ch + 32): read now (MMA3 of
      // chunk j + 2 reuses these columns once sdone is signalled), stored below
      float ov[16], ow[16];
      if (ta.write_o) {
        tmem_ld16(lanebase + acc + 64 + 32 * ch, ov);
        tmem_ld16(lanebase + acc + 64 + 32 * ch + 16, ow);
      }
      // S_{j+1}: chunk state out (or the final state), then Diag(d_{j+1}) S^T in place
      const float *dn = last ? nullptr : reinterpret_cast<const float *>(recbuf[buf ^ 1] + R5);
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
        float sv[16];
        tmem_ld16(lanebase + c0, sv);
        tmem_wait_ld();
        if (last) {
          if (STp)
            for (int i = 0; i < 16; ++i) STp[(size_t)(c0 + i) * D + v] = sv[i];
          continue;
        }
        if (ta.states_out)
          for (int i = 0; i < 16; ++i)
            ta.states_out[(((size_t)seq * H + h) * NCb + j0 + j + 1) * D * D + (size_t)(c0 + i) * D + v] = sv[i];
#pragma unroll
        for (int i = 0; i < 16; ++i) sv[i] *= dn[c0 + i];
        tmem_st16(lanebase + c0, sv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.sdone);
      if (ta.write_o) {
        // rows through shared memory ([row][channel], this thread's column v),
        // then out in 16-byte pieces: a warp writes two whole 256-byte rows per
        // store instead of 64 bytes of one
        unsigned char *ost = sm + S_OST;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          *reinterpret_cast<__nv_bfloat16 *>(ost + (uint32_t)((32 * ch + i) * D + v) * 2) =
              __float2bfloat16_rn(i < 16 ? ov[i] : ow[i - 16]);
        group_sync(2, kGroup);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int idx = gt + kGroup * k, row = idx >> 4, piece = idx & 15;
          if (row < len)
            *reinterpret_cast<uint4 *>(o + ((size_t)(tok0 + row) * H + h) * D + 8 * piece) =
                *reinterpret_cast<const uint4 *>(ost + row * 256 + 16 * piece);
        }
      }
    }
  }
  if (tid == kTileStorer) bulk_wait_all();  // every state tile written before the kernel ends
  __syncthreads();
  // wind down: the MMAs of warps 0 and 1 (issued by their elected lanes) done
  if (abort && warp == 1) mma_commit_warp(&ms.mfin);
  if (abort && warp == 0) {
    mma_commit_warp(&ms.mfin);
    mbar_wait(&ms.mfin, 0, a.status, 209);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ===========================================================================
// segment scan for long sequences (few (sequence, head) pairs, many chunks)
// ===========================================================================
// A chunk maps the state affinely: S' = A S + B with A = Diag(d) - Khat^T W
// and B = Khat^T U0.  The chunks of a sequence are split into segments:
// (1) tc_segmap_kernel composes each segment's map S -> M S + b in parallel,
//     by running the chunk recurrence on the state [I | 0] (dk x (dk + dv));
// (2) tc_segscan_kernel walks the segments in order (fp32) for their start
//     states;
// (3) the state pass runs every segment from its start state, in parallel.
constexpr int kSegThreads = 256;
constexpr uint32_t SG_RSZ = 50176;                 // compact record slot: W^T | U0^T | Khat^T, d
constexpr uint32_t SG_W = 0, SG_U0 = 16384, SG_KH = 32768, SG_D = 49152;
constexpr uint32_t SG_R0 = 0, SG_R1 = SG_RSZ;
constexpr uint32_t SG_S1 = 2 * SG_RSZ;             // bf16 M^T part, K-major [j][c] 128 x 128
constexpr uint32_t SG_S2 = SG_S1 + 32768;          // bf16 b^T part, K-major [v][c]
constexpr uint32_t SG_U1 = SG_S2 + 32768;          // bf16 U^T of the M part, K-major [j][s]
constexpr uint32_t SG_U2 = SG_U1 + 16384;          // bf16 U^T of the b part
constexpr uint32_t SG_MISC = SG_U2 + 16384;

struct SegMisc {
  uint64_t mrec[2], ma, mb, mfin;
  uint32_t tmem;
};

// TMEM: M^T [0,128), b^T [128,256), (W M)^T [256,320), (W b)^T [320,384).
__global__ void __launch_bounds__(kSegThreads, 1) tc_segmap_kernel(TcArgs ta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  SegMisc &ms = *reinterpret_cast<SegMisc *>(sm + SG_MISC);
  const FwdArgs &a = ta.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, ch = warp >> 2;
  const int h = blockIdx.x, H = a.H;
  const int seq = blockIdx.y / ta.seg_count, sg = blockIdx.y % ta.seg_count;
  const int j = 32 * qd + lane;  // TMEM lane: input index of the map
  int first;
  int nc = a.map.seq_chunks(seq, first);
  const int j0 = sg * ta.seg_len;
  nc = nc - j0 < ta.seg_len ? nc - j0 : ta.seg_len;
  if (nc < 0) nc = 0;
  first += j0;

  if (tid == 0) {
    mbar_init(&ms.mrec[0], 1);
    mbar_init(&ms.mrec[1], 1);
    mbar_init(&ms.ma, 1);
    mbar_init(&ms.mb, 1);
    mbar_init(&ms.mfin, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&ms.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem;
  const uint32_t lanebase = tmem + ((uint32_t)(32 * qd) << 16);
  unsigned char *rb[2] = {sm + SG_R0, sm + SG_R1};
  auto fetch = [&](int i) {  // record of the segment's chunk i into slot i & 1
    const unsigned char *src = ta.recs + ((size_t)(first + i) * H + h) * REC;
    unsigned char *dst = rb[i & 1];
    mbar_arrive_expect_tx(&ms.mrec[i & 1], 16384 + 16384 + 16896);
    bulk_g2s(dst + SG_W, src + R1, 16384, &ms.mrec[i & 1]);
    bulk_g2s(dst + SG_U0, src + R2, 16384, &ms.mrec[i & 1]);
    bulk_g2s(dst + SG_KH, src + R4, 16896, &ms.mrec[i & 1]);  // Khat^T and d
  };
  if (tid == 0) {
    for (int i = 0; i < 2 && i < nc; ++i) fetch(i);
  }
  // start: M^T = I, b^T = 0 (fp32 in TMEM, bf16 operand copies); columns [64 ch, 64 ch + 64)
  for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
    float e[16], z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      e[i] = (c0 + i == j) ? 1.f : 0.f;
      z[i] = 0.f;
    }
    tmem_st16(lanebase + c0, e);
    tmem_st16(lanebase + 128 + c0, z);
    uint32_t pk[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(e[2 * m], e[2 * m + 1]);
    *reinterpret_cast<uint4 *>(sm + SG_S1 + kmaj_off(j, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4 *>(sm + SG_S1 + kmaj_off(j, c0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    *reinterpret_cast<uint4 *>(sm + SG_S2 + kmaj_off(j, c0, 128)) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(sm + SG_S2 + kmaj_off(j, c0 + 8, 128)) = make_uint4(0, 0, 0, 0);
  }
  tmem_wait_st();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();

  bool abort = false;
  for (int i = 0; i < nc && !abort; ++i) {
    unsigned char *rec = rb[i & 1];
    {
      bool ok = true;
      if (tid == 0) ok = mbar_wait_ool(&ms.mrec[i & 1], (i >> 1) & 1, a.status, 221);
      if (__syncthreads_or(!ok)) { abort = true; break; }
    }
    // (W X)^T = X^T W^T for both parts (N = 64, K = c)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, false, true);
      const uint64_t bw = sdesc(smem_u32(rec + SG_W), 16384, 1024);
      const uint64_t a1 = sdesc(smem_u32(sm + SG_S1), 16, 1024), a2 = sdesc(smem_u32(sm + SG_S2), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16(tmem + 256, sdesc_off(a1, ko), sdesc_off(bw, kk * 2048), id, kk > 0);
        mma_bf16(tmem + 320, sdesc_off(a2, ko), sdesc_off(bw, kk * 2048), id, kk > 0);
      }
      mma_commit(&ms.ma);
    }
    {
      bool ok = true;
      if (tid == 0) ok = mbar_wait_ool(&ms.ma, i & 1, a.status, 222);
      if (__syncthreads_or(!ok)) { abort = true; break; }
    }
    tc_fence_after();
    // U^T = -(W M)^T and U0^T - (W b)^T -> bf16 tiles; columns s in [32 ch, 32 ch + 32)
    for (int s0 = 32 * ch; s0 < 32 * ch + 32; s0 += 16) {
      float w1[16], w2[16];
      tmem_ld16(lanebase + 256 + s0, w1);
      tmem_ld16(lanebase + 320 + s0, w2);
      tmem_wait_ld();
      const uint4 ua = *reinterpret_cast<const uint4 *>(rec + SG_U0 + kmaj_off(j, s0, 128));
      const uint4 ub = *reinterpret_cast<const uint4 *>(rec + SG_U0 + kmaj_off(j, s0 + 8, 128));
      const uint32_t u0[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
      uint32_t p1[8], p2[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        p1[m] = pack_bf16(-w1[2 * m], -w1[2 * m + 1]);
        p2[m] = pack_bf16(bf_lo(u0[m]) - w2[2 * m], bf_hi(u0[m]) - w2[2 * m + 1]);
      }
      *reinterpret_cast<uint4 *>(sm + SG_U1 + kmaj_off(j, s0, 128)) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
      *reinterpret_cast<uint4 *>(sm + SG_U1 + kmaj_off(j, s0 + 8, 128)) = make_uint4(p1[4], p1[5], p1[6], p1[7]);
      *reinterpret_cast<uint4 *>(sm + SG_U2 + kmaj_off(j, s0, 128)) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
      *reinterpret_cast<uint4 *>(sm + SG_U2 + kmaj_off(j, s0 + 8, 128)) = make_uint4(p2[4], p2[5], p2[6], p2[7]);
    }
    // X^T <- X^T Diag(d) in TMEM (both parts); columns c in [64 ch, 64 ch + 64)
    {
      const float *dj = reinterpret_cast<const float *>(rec + SG_D);
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
        float x1[16], x2[16];
        tmem_ld16(lanebase + c0, x1);
        tmem_ld16(lanebase + 128 + c0, x2);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          x1[m] *= dj[c0 + m];
          x2[m] *= dj[c0 + m];
        }
        tmem_st16(lanebase + c0, x1);
        tmem_st16(lanebase + 128 + c0, x2);
      }
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // X^T += U^T Khat (N = 128 over c, K = s)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 128, false, false);
      const uint64_t bk = sdesc(smem_u32(rec + SG_KH), 16, 1024);
      const uint64_t u1 = sdesc(smem_u32(sm + SG_U1), 16, 1024), u2 = sdesc(smem_u32(sm + SG_U2), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_bf16(tmem + 0, sdesc_off(u1, kk * 32), sdesc_off(bk, kk * 32), id, true);
        mma_bf16(tmem + 128, sdesc_off(u2, kk * 32), sdesc_off(bk, kk * 32), id, true);
      }
      mma_commit(&ms.mb);
    }
    {
      bool ok = true;
      if (tid == 0) ok = mbar_wait_ool(&ms.mb, i & 1, a.status, 223);
      if (__syncthreads_or(!ok)) { abort = true; break; }
    }
    tc_fence_after();
    if (tid == 0 && i + 2 < nc) fetch(i + 2);  // this slot's record is consumed
    if (i + 1 < nc) {  // bf16 operand copies of the new M^T, b^T
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
        float x1[16], x2[16];
        tmem_ld16(lanebase + c0, x1);
        tmem_ld16(lanebase + 128 + c0, x2);
        tmem_wait_ld();
        uint32_t p1[8], p2[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          p1[m] = pack_bf16(x1[2 * m], x1[2 * m + 1]);
          p2[m] = pack_bf16(x2[2 * m], x2[2 * m + 1]);
        }
        *reinterpret_cast<uint4 *>(sm + SG_S1 + kmaj_off(j, c0, 128)) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
        *reinterpret_cast<uint4 *>(sm + SG_S1 + kmaj_off(j, c0 + 8, 128)) = make_uint4(p1[4], p1[5], p1[6], p1[7]);
        *reinterpret_cast<uint4 *>(sm + SG_S2 + kmaj_off(j, c0, 128)) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
        *reinterpret_cast<uint4 *>(sm + SG_S2 + kmaj_off(j, c0 + 8, 128)) = make_uint4(p2[4], p2[5], p2[6], p2[7]);
      }
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
  }
  if (!abort) {  // the map, fp32: M^T [j][c] as held, b[c][v] = b^T[v][c] (row-major)
    float *Mo = ta.seg_M + ((size_t)blockIdx.y * H + h) * D * D;
    float *bo = ta.seg_b + ((size_t)blockIdx.y * H + h) * D * D;
    for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
      float x1[16], x2[16];
      tmem_ld16(lanebase + c0, x1);
      tmem_ld16(lanebase + 128 + c0, x2);
      tmem_wait_ld();
      if (ta.seg_M_rows) {  // M[c][j]: a warp writes 32 consecutive j of each row c
#pragma unroll
        for (int m = 0; m < 16; ++m) Mo[(size_t)(c0 + m) * D + j] = x1[m];
      } else {
        float4 *mrow = reinterpret_cast<float4 *>(Mo + (size_t)j * D + c0);
#pragma unroll
        for (int m = 0; m < 4; ++m) mrow[m] = make_float4(x1[4 * m], x1[4 * m + 1], x1[4 * m + 2], x1[4 * m + 3]);
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) bo[(size_t)(c0 + m) * D + j] = x2[m];
    }
  }
  if (abort && tid == 0) {
    mma_commit(&ms.mfin);
    mbar_wait(&ms.mfin, 0, a.status, 229);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// The segments of one (sequence, head) in order, fp32 on CUDA cores:
// start(0) = S0 (or 0), start(g + 1) = M_g start(g) + b_g; or, reversed (the
// backward's adjoint states, with the maps' rows M_g^T and the adjoint
// offsets e_g): end(G - 1) = dS_T (or 0), end(g - 1) = M_g^T end(g) + e_g.
// The kernel reads a table T_g (M_g^T for the forward, M_g for the reverse)
// and forms out[c][v] = sum_k T_g[k][c] X[k][v] + b_g[c][v].  The value columns
// are independent, so a CTA takes a slice of VC of them (blockIdx.z); a
// thread holds a 4 x (VC / 8) block of the slice in registers.  M_g^T
// (64 KB) is double-buffered in shared memory by bulk copies.
constexpr int kScanThreads = 256;
template <int VC>
__global__ void __launch_bounds__(kScanThreads, 1) tc_segscan_kernel(TcArgs ta) {
  constexpr int NV = VC / 8;  // columns per thread
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
  float *Mt = reinterpret_cast<float *>(sm);         // [2][128][128] M_g^T
  float *Ss = Mt + 2 * D * D;                         // [128][VC] current start state, this slice
  uint64_t *mfull = reinterpret_cast<uint64_t *>(Ss + D * VC);
  const FwdArgs &a = ta.f;
  const int tid = threadIdx.x, h = blockIdx.x, seq = blockIdx.y, H = a.H, G = ta.seg_count;
  const int tv = tid & 7, tc = tid >> 3;
  const int c0 = 4 * tc, vl = NV * tv, vg = VC * blockIdx.z + vl;  // rows c0..c0+3; local/global column
  if (tid == 0) {
    mbar_init(&mfull[0], 1);
    mbar_init(&mfull[1], 1);
    mbar_fence_init();
  }
  __syncthreads();
  // step i handles segment g(i): i in order, or from the last one down
  auto seg_of = [&](int i) { return ta.seg_reverse ? G - 1 - i : i; };
  auto fetch = [&](int i) {  // the table of step i into buffer i & 1
    const size_t sidx = ((size_t)(seq * G + seg_of(i)) * H + h) * D * D;
    mbar_arrive_expect_tx(&mfull[i & 1], D * D * 4);
    bulk_g2s(Mt + (i & 1) * D * D, ta.seg_M + sidx, D * D * 4, &mfull[i & 1]);
  };
  if (tid == 0 && G > 1) fetch(0);
  float st[4][NV];
  const float *S0 = ta.seg_X0 ? ta.seg_X0 + ((size_t)seq * H + h) * D * D : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < NV; ++k) st[i][k] = S0 ? S0[(size_t)(c0 + i) * D + vg + k] : 0.f;
  for (int g = 0; g < G; ++g) {  // (g counts steps; the segment is seg_of(g))
    const size_t sidx = ((size_t)(seq * G + seg_of(g)) * H + h) * D * D;
    float *out = ta.seg_S0 + sidx;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < NV; ++k) out[(size_t)(c0 + i) * D + vg + k] = st[i][k];
    if (g + 1 == G) break;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < NV; ++k) Ss[(c0 + i) * VC + vl + k] = st[i][k];
    if (tid == 0 && g + 1 < G - 1) fetch(g + 1);  // its buffer was released by the last step's barrier
    const float *bg = ta.seg_b + sidx;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < NV; ++k) st[i][k] = bg[(size_t)(c0 + i) * D + vg + k];
    bool ok = true;
    if (tid == 0) ok = mbar_wait_ool(&mfull[g & 1], (g >> 1) & 1, a.status, 231);
    if (__syncthreads_or(!ok)) {  // gave up: let the copy into the other buffer land first
      if (tid == 0 && g + 1 < G - 1) mbar_wait_ool(&mfull[(g + 1) & 1], ((g + 1) >> 1) & 1, a.status, 232);
      return;
    }
    const float *Mb = Mt + (g & 1) * D * D;
#pragma unroll 4
    for (int jj = 0; jj < D; ++jj) {
      const float4 m = *reinterpret_cast<const float4 *>(Mb + jj * D + c0);
      float sv[NV];
      if constexpr (NV == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(Ss + jj * VC + vl);
        sv[0] = x.x; sv[1] = x.y; sv[2] = x.z; sv[3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2 *>(Ss + jj * VC + vl);
        sv[0] = x.x; sv[1] = x.y;
      }
      const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < NV; ++k) st[i][k] = fmaf(mv[i], sv[k], st[i][k]);
    }
    __syncthreads();  // every read of Ss and of this M buffer is done
  }
}

int g_num_sms = 0;

}  // namespace

size_t tc_fwd_fallback_floats(int ctas) { return (size_t)ctas * 3 * 64 * D; }

int tc_intra_ctas() {
  if (g_num_sms == 0) {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms = n > 0 ? n : 148;
  }
  const int want = 2 * g_num_sms;
  return want < kBwdCtas ? want : kBwdCtas;
}

size_t tc_record_bytes() { return REC; }

// The segment kernels' launches (the segment fields of ta are set).
static cudaError_t launch_segmap(const TcArgs &ta, cudaStream_t s) {
  const size_t sm_map = SG_MISC + sizeof(SegMisc) + 1024;
  cudaError_t e = cudaFuncSetAttribute(tc_segmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_map);
  if (e != cudaSuccess) return e;
  ProfScope prof("tc_segmap", s);
  tc_segmap_kernel<<<dim3(ta.f.H, ta.f.B * ta.seg_count), kSegThreads, sm_map, s>>>(ta);
  return cudaGetLastError();
}
static cudaError_t launch_segscan(const TcArgs &ta, cudaStream_t s) {
  // value-column slices of the scan: 8 (16 columns) while the CTAs fit on the SMs, else 4
  const int split = 8 * ta.f.B * ta.f.H <= g_num_sms ? 8 : 4;
  const size_t sm_scan = 128 + (2 * D * D + D * (D / split)) * sizeof(float) + 2 * sizeof(uint64_t);
  auto scan = split == 8 ? tc_segscan_kernel<16> : tc_segscan_kernel<32>;
  cudaError_t e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_scan);
  if (e != cudaSuccess) return e;
  ProfScope prof("tc_segscan", s);
  scan<<<dim3(ta.f.H, ta.f.B, split), kScanThreads, sm_scan, s>>>(ta);
  return cudaGetLastError();
}

// Forward on tensor cores.  recs: n_chunks_bound * H records of REC bytes;
// fb: tc_fwd_fallback_floats(tc_intra_ctas()) floats.  intra_pass = false
// reuses records an earlier call wrote for the same inputs.
// Segments per sequence for the segment scan: only for batched calls whose
// (sequence, head) pairs fill at most half the SMs and whose sequences are
// long (>= 32 chunks); at least 16 chunks per segment, at most one wave of
// CTAs, and only where the estimate below says it pays.  0: run the plain
// sequential state pass.
int tc_seg_count(int B, int H, int NC) {
  (void)tc_intra_ctas();  // SM count
  const int sms = g_num_sms > 0 ? g_num_sms : 148;
  const int pairs = B * H;
  if (pairs <= 0 || 2 * pairs > sms || NC < 32) return 0;
  int G = sms / pairs;
  if (G > NC / 16) G = NC / 16;
  if (G < 2) return 0;
  const int L = (NC + G - 1) / G;
  G = (NC + L - 1) / L;
  // the maps and the segments' state passes each take about L chunk steps,
  // the scan about one per segment: keep it only where that beats NC steps
  if (2 * L + G + 4 > NC) return 0;
  return G;
}
size_t tc_seg_ws_bytes() {
  (void)tc_intra_ctas();  // SM count
  return (size_t)3 * (g_num_sms > 0 ? g_num_sms : 148) * D * D * sizeof(float);
}

cudaError_t tc_forward(const FwdArgs &f, unsigned char *recs, float *fb, bool write_o,
                       float *states_out, cudaStream_t s, bool state_pass, bool intra_pass,
                       bool state_tiles, float *seg_ws) {
  TcArgs ta{};
  ta.f = f;
  ta.recs = recs;
  ta.fb = fb;
  ta.states_out = states_out;
  ta.write_o = write_o;
  ta.state_tiles = state_tiles;
  const size_t sm_intra = I_MISC + sizeof(IntraMisc) + 1024;
  const size_t sm_state = S_MISC + sizeof(StateMisc) + 1024;
  cudaError_t e = cudaFuncSetAttribute(tc_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm_intra);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_state);
  if (e != cudaSuccess) return e;
  if (intra_pass) {
    e = make_row_maps(ta.rm, f.q, f.k, f.v, nullptr, f.g, f.sign, (int64_t)f.B * f.T, f.H);
    if (e != cudaSuccess) return e;
    ProfScope prof("tc_intra", s);
    tc_intra_kernel<<<tc_intra_ctas(), kIntraThreads, sm_intra, s>>>(ta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (state_pass && f.map.n_seq > 0) {
    const int G = (seg_ws && !f.map.table) ? tc_seg_count(f.B, f.H, f.map.NC) : 0;
    if (G >= 2) {  // long sequences: segment maps, their scan, then every segment at once
      ta.seg_count = G;
      ta.seg_len = (f.map.NC + G - 1) / G;
      const size_t per = (size_t)f.B * G * f.H * D * D;
      ta.seg_M = seg_ws;
      ta.seg_b = seg_ws + per;
      ta.seg_S0 = seg_ws + 2 * per;
      ta.seg_X0 = f.S0;
      if ((e = launch_segmap(ta, s)) != cudaSuccess) return e;
      if ((e = launch_segscan(ta, s)) != cudaSuccess) return e;
      ProfScope prof(write_o ? "tc_state_fwd" : "tc_state_fwd_recompute", s);
      tc_state_kernel<<<dim3(f.H, f.B * G), kStateThreads, sm_state, s>>>(ta);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      return cudaSuccess;
    }
    ProfScope prof(write_o ? "tc_state_fwd" : "tc_state_fwd_recompute", s);
    tc_state_kernel<<<dim3(f.H, f.map.n_seq), kStateThreads, sm_state, s>>>(ta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Segments of the long-sequence backward: the same split as the forward's
// (tc_seg_count) but only where three passes of L chunks (the maps, the
// reverse pass from zero, the reverse pass from the scanned states) and the
// scan beat one pass of NC chunks.
int tc_seg_count_bwd(int B, int H, int NC) {
  const int G = tc_seg_count(B, H, NC);
  if (G < 2) return 0;
  const int L = (NC + G - 1) / G;
  return 3 * L + G + 8 < NC ? G : 0;
}

cudaError_t tc_seg_maps_rows(const FwdArgs &f, const unsigned char *recs, int G, float *seg_M, float *seg_b,
                             cudaStream_t s) {
  TcArgs ta{};
  ta.f = f;
  ta.recs = const_cast<unsigned char *>(recs);
  ta.seg_count = G;
  ta.seg_len = (f.map.NC + G - 1) / G;
  ta.seg_M = seg_M;
  ta.seg_b = seg_b;
  ta.seg_M_rows = true;
  return launch_segmap(ta, s);
}

cudaError_t tc_seg_scan_reverse(const FwdArgs &f, int G, const float *seg_M, const float *seg_e, const float *X0,
                                float *seg_ends, cudaStream_t s) {
  TcArgs ta{};
  ta.f = f;
  ta.seg_count = G;
  ta.seg_len = (f.map.NC + G - 1) / G;
  ta.seg_M = const_cast<float *>(seg_M);
  ta.seg_b = const_cast<float *>(seg_e);
  ta.seg_S0 = seg_ends;
  ta.seg_reverse = true;
  ta.seg_X0 = X0;
  return launch_segscan(ta, s);
}

}  // namespace ckda
