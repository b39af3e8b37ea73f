// ckda_tc_bwd.cu -- chunked CKDA backward on tcgen05 tensor cores (bf16 I/O,
// dk = dv = 128).  Reverse mode of the chunk-wise WY / UT form ("Complex KDA:
// Understanding and Enhancing the Expressivity of Kimi Delta Attention",
// section 2, "Linear RNNs"; sign folding per the "openeurollm/
// complex-kda-1.3B-100B" model card introduction), derived by hand:
//
//   reverse state pass (per sequence and head, chunks in reverse):
//     dU    = A_q^T dO + Khat dS_{c+1}
//     dS_c  = Diag(d) dS_{c+1} + QG^T dO - W^T dU
//   per-chunk gradients (parallel over chunks):
//     U = U0 - W S_c;  dQG = dO S_c^T;  dW = -dU S_c^T;  dKhat = U dS_{c+1}^T
//     dd = rowsum(S_c . dS_{c+1});  dA_q = tril(dO U^T);  dT = tril(dU V^T + dW KG^T)
//     dV = T^T dU;  dKG = T^T dW;  dM = dT Diag(beta);  dL = -M^T dM M^T
//     dA = Diag(beta) strict_tril(dL);  dbeta from dT.M and dL.A
//     pair terms through the reference row: X1 = dA K~r, X2 = dA_q K~r,
//     Y1 = dA^T K~l + dA_q^T Q~, then the exponential factors, a reverse
//     in-chunk cumsum for dg, and the sign unfold of dq, dk.
//
// Kernels: tc_state_bwd_kernel (reverse pass; state gradient kept transposed
// in TMEM, lanes = value channel) writes per chunk the dL/dS_{c+1} and dU
// tiles; tc_grad_kernel (persistent, one CTA per SM) does everything else.
#include <cmath>
#include <type_traits>

#include "ckda_tc.cuh"

namespace ckda {
namespace {

using namespace tc;

// bytes of the per-(chunk, head) tiles the reverse pass hands to the gradient kernel
constexpr uint32_t DS_TILE = 32768;  // dL/dS_{c+1}, transposed: bf16 K-major [v][c], 128 rows
constexpr uint32_t DU_TILE = 16384;  // dU: bf16 K-major [i][v], 64 rows

struct BwdTcArgs {
  RowMaps rm;                 // q, k, v, dO, g, sign (gradient kernel)
  BwdArgs b;
  const unsigned char *recs;  // intra-chunk records (forward layout)
  unsigned char *dS_tiles;    // [n_chunks][H] DS_TILE
  unsigned char *dU_tiles;    // [n_chunks][H] DU_TILE
  float *fb;                  // per-CTA fallback scratch (3 x 64 x 128 fp32)
  // segment mode of the reverse pass (long sequences): blockIdx.y = seq *
  // seg_count + segment, each CTA walks one segment of seg_len chunks
  int seg_len, seg_count;
  const float *seg_in;  // adjoint state at each segment's end, fp32 [128][128] (null: zero)
  float *seg_out;       // adjoint state at each segment's start (null: dS0 for the first segment)
  bool no_tiles;        // provisional pass: no dS / dU tiles
};

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float (&v)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(__float_as_uint(v[0])),
               "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3]))
               : "memory");
}
// one 32-bit column per lane (the whole warp executes it)
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
}

// ===========================================================================
// reverse state pass
// ===========================================================================
constexpr int kSbThreads = 512;  // two warp groups of 256 (two warps per TMEM lane quadrant each)
constexpr int kSbGroup = 256;
constexpr int kSbCopier = 64;  // group A thread that issues the first dS snapshot (the others: group B)
constexpr uint32_t RB_SIZE = 58368;            // compact record: R1 | R3 | R4 | R5
constexpr uint32_t RB_R1 = 0, RB_R3 = 32768, RB_R4 = 40960, RB_R5 = 57344;
constexpr uint32_t SB_RB0 = 0, SB_RB1 = RB_SIZE;
constexpr uint32_t SB_O0 = 2 * RB_SIZE;        // dO tile K-major [r][v], 64 rows (16 KiB)
constexpr uint32_t SB_O1 = SB_O0 + 16384;
constexpr uint32_t SB_DS = SB_O1 + 16384;      // dS^T bf16 K-major [v][c], 128 rows
constexpr uint32_t SB_DU = SB_DS + 32768;      // dU^T bf16 K-major [v][s], 128 rows x 64
constexpr uint32_t SB_DUG = SB_DU + 16384;     // dU bf16 K-major [s][v] 64 rows: the dU tile out
constexpr uint32_t SB_MISC = SB_DUG + 16384;

struct SbMisc {
  uint64_t mrec[2], mdo[2], mu, ms, mfin, dsready, scaled, dudone;
  uint32_t tmem;
};

// TMEM: dS^T fp32 [0,128) (lanes = value channel); dU^T of step s at
// 128 + 64 (s & 1).
//
// Two warp groups.  Group A (warps 0-7) carries the reverse recurrence: the
// dU MMA, the bf16 dU^T operand, the dS MMA, the bf16 dS^T operand (and the
// dL/dS snapshot by bulk store).  Group B (warps 8-15) does what the next
// MMA only needs done in time: dS^T <- dS^T Diag(d_j) in TMEM before the dS
// MMA of step s, and the dU tile out (staged transposed, bulk stored).
// Hand-offs (one arrive per warp): dsready (A: dS^T has been read), scaled
// (B: dS^T is scaled), dudone (B: the dU^T buffer has been read).
__global__ void __launch_bounds__(kSbThreads, 1) tc_state_bwd_kernel(const __grid_constant__ BwdTcArgs ta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  SbMisc &ms = *reinterpret_cast<SbMisc *>(sm + SB_MISC);
  const BwdArgs &a = ta.b;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool grpA = tid < kSbGroup;
  const int gt = tid & (kSbGroup - 1);
  const int qd = warp & 3, ch = (warp >> 2) & 1;
  const int h = blockIdx.x, H = a.H;
  const int v = 32 * qd + lane;
  const __nv_bfloat16 *dO = (const __nv_bfloat16 *)a.dO;
  // this CTA's chunks: a whole sequence, or one segment of it; the adjoint
  // state it starts from (the range's end) and where the range's start state goes
  int seq = blockIdx.y, first, nc;
  const float *X0;
  float *Xout;
  if (ta.seg_len > 0) {
    seq = blockIdx.y / ta.seg_count;
    const int sg = blockIdx.y % ta.seg_count, j0 = sg * ta.seg_len;
    nc = a.map.seq_chunks(seq, first);
    nc = nc - j0 < ta.seg_len ? nc - j0 : ta.seg_len;
    if (nc < 0) nc = 0;
    first += j0;
    const size_t own = ((size_t)blockIdx.y * H + h) * D * D;
    X0 = ta.seg_in ? ta.seg_in + own : nullptr;
    Xout = ta.seg_out ? ta.seg_out + own : ((sg == 0 && a.dS0) ? a.dS0 + ((size_t)seq * H + h) * D * D : nullptr);
  } else {
    nc = a.map.seq_chunks(seq, first);
    X0 = a.dST ? a.dST + ((size_t)seq * H + h) * D * D : nullptr;
    Xout = a.dS0 ? a.dS0 + ((size_t)seq * H + h) * D * D : nullptr;
  }

  if (tid == 0) {
    mbar_init(&ms.mrec[0], 1);
    mbar_init(&ms.mrec[1], 1);
    mbar_init(&ms.mdo[0], 1);
    mbar_init(&ms.mdo[1], 1);
    mbar_init(&ms.mu, 1);
    mbar_init(&ms.ms, 1);
    mbar_init(&ms.mfin, 1);
    mbar_init(&ms.dsready, kSbGroup / 32);
    mbar_init(&ms.scaled, kSbGroup / 32);
    mbar_init(&ms.dudone, kSbGroup / 32);
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
  const uint32_t lanebase = tmem + ((uint32_t)(32 * qd) << 16);
  unsigned char *rb[2] = {sm + SB_RB0, sm + SB_RB1};
  unsigned char *ob[2] = {sm + SB_O0, sm + SB_O1};

  // step s handles chunk j = nc - 1 - s
  auto issue_record = [&](int s) {
    const int j = nc - 1 - s;
    const unsigned char *src = ta.recs + ((size_t)(first + j) * H + h) * REC;
    unsigned char *dst = rb[s & 1];
    mbar_arrive_expect_tx(&ms.mrec[s & 1], 32768 + 25088);
    bulk_g2s(dst + RB_R1, src + R1, 32768, &ms.mrec[s & 1]);
    bulk_g2s(dst + RB_R3, src + R3, 25088, &ms.mrec[s & 1]);
  };
  // dO rows of step s (two TMA boxes, K-major SW128 64 x 128) into buffer s & 1,
  // issued by group B's first thread once that buffer's last readers (the
  // MMAs of step s - 2) are done; a partial chunk's rows past its end are
  // zeroed by group A before use
  auto chunk_len = [&](int s) {
    int sq, len, jl;
    int64_t tok0;
    a.map.info(first + nc - 1 - s, sq, tok0, len, jl);
    return len;
  };
  auto issue_dO = [&](int s) {
    int sq, len, jl;
    int64_t tok0;
    a.map.info(first + nc - 1 - s, sq, tok0, len, jl);
    unsigned char *dst = ob[s & 1];
    mbar_arrive_expect_tx(&ms.mdo[s & 1], 16384);
    tma_rows(dst, &ta.rm.dO, 0, h, (int)tok0, &ms.mdo[s & 1]);
    tma_rows(dst + 8192, &ta.rm.dO, 64, h, (int)tok0, &ms.mdo[s & 1]);
  };
  // dL/dS_{c+1} snapshot of chunk j: the bf16 dS^T operand tile as it stands
  // (one bulk store by group A's first thread, after the tile's writers have synchronised)
  auto snapshot = [&](int j) {
    if (ta.no_tiles) return;
    bulk_s2g(ta.dS_tiles + ((size_t)(first + j) * H + h) * DS_TILE, sm + SB_DS, DS_TILE);
    bulk_commit();
  };

  if (tid == 0 && nc > 0) {
    issue_record(0);
    if (nc > 1) issue_record(1);
  }
  if (tid == kSbGroup && nc > 0) issue_dO(0);
  if (grpA) {
    // dS_T (true frame) -> dS^T rows; bf16 copy for the MMA, fp32 in TMEM
    for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
      float sv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) sv[i] = X0 ? X0[(size_t)(c0 + i) * D + v] : 0.f;
      if (nc == 0) {
        if (Xout)
          for (int i = 0; i < 16; ++i) Xout[(size_t)(c0 + i) * D + v] = sv[i];
        continue;
      }
      uint32_t pk[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(sv[2 * m], sv[2 * m + 1]);
      *reinterpret_cast<uint4 *>(sm + SB_DS + kmaj_off(v, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4 *>(sm + SB_DS + kmaj_off(v, c0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      tmem_st16(lanebase + c0, sv);
    }
    tmem_wait_st();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == kSbCopier && nc > 0) snapshot(nc - 1);
  if (grpA && nc > 0) {  // dS^T is in place: group B may scale it for step 0
    __syncwarp();
    if (lane == 0) mbar_arrive(&ms.dsready);
  }

  bool abort = false;
  int n_do = (tid == kSbGroup && nc > 0) ? 1 : 0;  // dO loads issued (group B's first thread)
  if (grpA) {
    auto wait_a = [&](uint64_t *bar, uint32_t phase, uint32_t site, bool ok_in) -> bool {
      bool ok = ok_in;
      if (gt == 0 && ok) ok = mbar_wait(bar, phase, a.status, site);
      return !group_sync_or(1, kSbGroup, !ok);
    };
    for (int s = 0; s < nc && !abort; ++s) {
      const int j = nc - 1 - s;
      const int b = s & 1;
      unsigned char *rec = rb[b];
      unsigned char *ot = ob[b];
      const uint32_t du = 128 + 64 * b;  // dU^T buffer of this step
      const int len_s = chunk_len(s);
      if (len_s < 64) {  // this step's dO: rows past the chunk are zeros, not the next tokens' rows
        const bool okd = mbar_wait(&ms.mdo[b], (s >> 1) & 1, a.status, 310);
        if (group_sync_or(1, kSbGroup, !okd)) { abort = true; break; }
        zero_tail_rows(ot, 8192, len_s, gt, kSbGroup);
        fence_async_smem();
      }
      if (!wait_a(&ms.mrec[b], (s >> 1) & 1, 301, true)) { abort = true; break; }
      // dU^T = dO^T A_q + dS1^T Khat^T
      bool ok = true;
      if (warp == 0) {  // the whole warp; one elected lane issues
        // group B has read the dU^T of step s - 1 (waiting for that completion
        // rather than the one for step s - 2, whose buffer this step reuses,
        // keeps the parity wait unambiguous: B cannot run two steps ahead)
        if (s >= 1) ok = mbar_wait(&ms.dudone, (s - 1) & 1, a.status, 304);
        if (ok && len_s == 64) ok = mbar_wait(&ms.mdo[b], (s >> 1) & 1, a.status, 310);  // this step's dO
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          const uint32_t sO = smem_u32(ot), sRec = smem_u32(rec), sDS = smem_u32(sm + SB_DS);
          const uint32_t id1 = idesc_bf16(128, 64, true, true);
          const uint32_t id2 = idesc_bf16(128, 64, false, true);
          const uint64_t dO_ = sdesc(sO, 8192, 1024), dAq = sdesc(sRec + RB_R3, 8192, 1024);
          const uint64_t dDS = sdesc(sDS, 16, 1024), dKh = sdesc(sRec + RB_R4, 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_warp(tmem + du, sdesc_off(dO_, kk * 2048), sdesc_off(dAq, kk * 2048), id1, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_warp(tmem + du, sdesc_off(dDS, (kk >> 2) * 16384 + (kk & 3) * 32), sdesc_off(dKh, kk * 2048), id2, true);
          mma_commit_warp(&ms.mu);
        }
      }
      if (!wait_a(&ms.mu, s & 1, 302, ok)) { abort = true; break; }
      tc_fence_after();
      // dU^T -> bf16 operand tile (group B writes the dU tile out)
      for (int s0 = 32 * ch; s0 < 32 * ch + 32; s0 += 16) {
        float w[16];
        tmem_ld16(lanebase + du + s0, w);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(w[2 * m], w[2 * m + 1]);
        *reinterpret_cast<uint4 *>(sm + SB_DU + kmaj_off(v, s0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4 *>(sm + SB_DU + kmaj_off(v, s0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_async_smem();
      tc_fence_before();
      group_sync(1, kSbGroup);
      // dS^T += dO^T QG - dU^T W  (dS^T scaled by group B first)
      ok = true;
      if (warp == 0) {
        ok = mbar_wait(&ms.scaled, s & 1, a.status, 305);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          const uint32_t sO = smem_u32(ot), sRec = smem_u32(rec), sDU = smem_u32(sm + SB_DU);
          const uint32_t id1 = idesc_bf16(128, 128, true, false);
          const uint32_t id2 = idesc_bf16(128, 128, false, false) | (1u << 13);  // negate A
          const uint64_t dO_ = sdesc(sO, 8192, 1024), dQG = sdesc(sRec + RB_R1 + 16384, 16, 1024);
          const uint64_t dDU = sdesc(sDU, 16, 1024), dW = sdesc(sRec + RB_R1, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16_warp(tmem, sdesc_off(dO_, kk * 2048), sdesc_off(dQG, kk * 32), id1, true);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_bf16_warp(tmem, sdesc_off(dDU, kk * 32), sdesc_off(dW, kk * 32), id2, true);
          mma_commit_warp(&ms.ms);
        }
      }
      if (tid == kSbCopier) bulk_wait_read_all();  // the last snapshot has left the dS^T tile
      if (!wait_a(&ms.ms, s & 1, 303, ok)) { abort = true; break; }
      tc_fence_after();
      // dS at the start of chunk j: next step's operand, snapshot of chunk j-1, or dS0
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
        float sv[16];
        tmem_ld16(lanebase + c0, sv);
        tmem_wait_ld();
        if (j == 0) {
          if (Xout)
            for (int i = 0; i < 16; ++i) Xout[(size_t)(c0 + i) * D + v] = sv[i];
          continue;
        }
        uint32_t pk[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) pk[m] = pack_bf16(sv[2 * m], sv[2 * m + 1]);
        *reinterpret_cast<uint4 *>(sm + SB_DS + kmaj_off(v, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4 *>(sm + SB_DS + kmaj_off(v, c0 + 8, 128)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      fence_async_smem();
      tc_fence_before();
      if (j > 0) {  // dS^T has been read: group B may scale it for the next step
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms.dsready);
      }
      group_sync(1, kSbGroup);
    }
  } else {
    for (int s = 0; s < nc && !abort; ++s) {
      const int b = s & 1;
      const uint32_t du = 128 + 64 * b;
      // dS^T <- dS^T Diag(d_j) once group A has read it
      bool ok = mbar_wait(&ms.dsready, s & 1, a.status, 306);
      if (ok) ok = mbar_wait(&ms.mrec[b], (s >> 1) & 1, a.status, 307);
      if (group_sync_or(2, kSbGroup, !ok)) { abort = true; break; }
      // the MMAs of step s - 1 are done (dsready): the next step's dO into their
      // buffer, the next record but one into the slot of step s - 1, and the
      // dL/dS snapshot of the tile group A has just written (the chain's copies,
      // issued off the chain)
      if (gt == 0) {
        if (s + 1 < nc) {
          issue_dO(s + 1);
          ++n_do;
        }
        if (s >= 1 && s + 1 < nc) issue_record(s + 1);
        if (s >= 1) snapshot(nc - 1 - s);
      }
      tc_fence_after();
      {
        const float *dj = reinterpret_cast<const float *>(rb[b] + RB_R5);
        for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 16) {
          float sv[16];
          tmem_ld16(lanebase + c0, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[i] *= dj[c0 + i];
          tmem_st16(lanebase + c0, sv);
        }
        tmem_wait_st();
      }
      if (gt == 0) bulk_wait_read_all();  // the snapshot has left the dS^T tile (group A rewrites it after scaled)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.scaled);
      // the dU tile of this chunk, staged transposed ([s][v]) and bulk stored
      ok = mbar_wait(&ms.mu, s & 1, a.status, 308);
      if (gt == 0) bulk_wait_read_all();  // the previous dU tile has left the staging tile
      if (group_sync_or(2, kSbGroup, !ok)) { abort = true; break; }
      tc_fence_after();
      for (int s0 = 32 * ch; s0 < 32 * ch + 32; s0 += 16) {
        float w[16];
        tmem_ld16(lanebase + du + s0, w);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) st_bf16(sm + SB_DUG, kmaj_off(s0 + i, v, 64), w[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.dudone);
      fence_async_smem();
      group_sync(2, kSbGroup);
      if (gt == 0 && !ta.no_tiles) {
        const int j = nc - 1 - s;
        bulk_s2g(ta.dU_tiles + ((size_t)(first + j) * H + h) * DU_TILE, sm + SB_DUG, DU_TILE);
        bulk_commit();
      }
    }
  }
  if (gt == 0 || tid == kSbCopier) bulk_wait_all();  // every tile written before the kernel ends
  // dO rows still landing (after an abort) finish before the CTA leaves: the
  // last load into each buffer (at most one per buffer is outstanding)
  if (tid == kSbGroup)
    for (int k = n_do > 2 ? n_do - 2 : 0; k < n_do; ++k) mbar_wait(&ms.mdo[k & 1], (k >> 1) & 1, a.status, 311);
  __syncthreads();
  if (abort && warp == 0) {  // the MMAs of warp 0 (issued by its elected lane) done
    mma_commit_warp(&ms.mfin);
    mbar_wait(&ms.mfin, 0, a.status, 309);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ===========================================================================
// per-chunk gradient kernel
// ===========================================================================
constexpr int kGThreads = 512;  // 16 warps: four per TMEM lane quadrant
constexpr uint32_t G_A1 = 0;          // [Q~; K~l] K-major 128 x 128
constexpr uint32_t G_B1 = 32768;      // K~r K-major 64 x 128
constexpr uint32_t G_KG = 49152;      // g staging (with B1); later dM M^T parts
constexpr uint32_t G_UV = 65536;      // [U; V] K-major 128 x 128
constexpr uint32_t G_TT = 98304;      // T K-major [r][j] 64 x 64
constexpr uint32_t G_OU = 106496;     // [dO; dU] K-major 128 x 128
constexpr uint32_t G_SC = 139264;     // S_c^T bf16 K-major [v][c]; later dW in rows 64..127
constexpr uint32_t G_WN = 172032;     // W tile | dS1 tile | [dA; dAq] + dT fp32
constexpr uint32_t G_DT = G_WN + 16384;
constexpr uint32_t G_MF = 205824;     // M fp32 [64][65]
constexpr uint32_t G_MISC = 222464;
constexpr int LDF = 65;
// bf16 hi / lo parts for the dL = -M^T dM M^T products, in tiles idle by then
constexpr uint32_t G_DMH = G_UV, G_DML = G_UV + 8192;           // dM, K-major [i][j]
constexpr uint32_t G_MH = G_UV + 16384, G_ML = G_UV + 24576;    // M, K-major [i][a]
constexpr uint32_t G_TH = G_KG, G_TL = G_KG + 8192;             // dM M^T, K-major [i][k]
// final epilogue scratch in the idle [U; V] tile (rows 0..63 of block 0;
// the next item's V lands in rows 64..): per-quarter sums
constexpr uint32_t G_FSUM = G_UV;               // float [2][4][128]
constexpr uint32_t W_TILE = 16384;              // W^T half of the record's R1 tile
constexpr uint32_t S_TILE = 32768;              // the record's S_c^T (bf16 K-major [v][c])
constexpr uint32_t M_BYTES = 64 * LDF * 4;      // the record's M
constexpr uint32_t T_TILE = 8192;               // the record's T
constexpr uint32_t G_SGN = G_DT;                // sign rows of the next item (dT is dead by then)
static_assert(M_BYTES == R7 - R6 && S_TILE == R8 - R7 && T_TILE == REC - R8, "record layout");

struct GMisc {
  uint64_t bar[7], mdu, mds, mfin, mrec, mld;
  uint32_t tmem;
  int pad;
  float beta[64], dbc[64], dbr[4][64];
  float qt[4][128];    // per-quarter totals of g (prep)
  uint8_t qp[4][128];  // per-quarter sign parities (prep)
  float ddp[8][128];  // partial diag(S_c dS1^T) per eighth of the value channels
};

// Completion of MMAs (or of a copy only MMAs consume): one thread polls the
// mbarrier, the others wait at the CTA barrier (no spinning issue slots).
__device__ __forceinline__ bool wait_one(uint64_t *bar, uint32_t phase, DevStatus *st, uint32_t site) {
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait_ool(bar, phase, st, site);
  return !__syncthreads_or(!ok);
}
// Completion of a copy whose data every thread reads: every thread observes it.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t phase, DevStatus *st, uint32_t site) {
  const bool ok = mbar_wait_ool(bar, phase, st, site);
  return !__syncthreads_or(!ok);
}

// Prep in the channel layout: thread (c = tid & 127, cq = tid >> 7) owns key
// channel c -- the TMEM lane its warp reads -- for chunk rows 16 cq .. 16 cq + 15,
// so the prep values meet the accumulators of the final epilogue in registers.
struct PrepC {
  float G[16];      // chunk-local inclusive cumsum of g (after the carry)
  uint32_t kq[16];  // raw bf16 k (low half) and q (high half)
  uint32_t pre;     // bit i: sign product of row 16 cq + i is negative
  float Gm, GC;     // Gam at the reference row 31 and at the chunk end
  uint32_t pC;      // the chunk's sign product is negative
};
// Reads the staged rows (q, k K-major SW128 tiles, g fp32 [64][128], sign
// int8 [64][128]), scans the 16 rows, writes the quarter totals.
__device__ __forceinline__ void prepc_load(const unsigned char *sqk, const float *sg, const uint8_t *ss, int len,
                                           int c, int cq, PrepC &P, float *qt, uint8_t *qp) {
  float acc = 0.f;
  uint32_t par = 0, pre = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = 16 * cq + i;
    const bool valid = r < len;
    const float g = sg[r * D + c];
    const int8_t sgn = ss ? (int8_t)ss[r * D + c] : (int8_t)1;
    const uint32_t off = kmaj_off(r, c, 64);
    const uint32_t kb = *reinterpret_cast<const uint16_t *>(sqk + kStageK + off);
    const uint32_t qb = *reinterpret_cast<const uint16_t *>(sqk + kStageQ + off);
    P.kq[i] = valid ? (kb | (qb << 16)) : 0u;
    acc += valid ? g : 0.f;
    P.G[i] = acc;
    par ^= (valid && sgn < 0) ? 1u : 0u;
    pre |= par << i;
  }
  P.pre = pre;
  qt[cq * D + c] = acc;
  qp[cq * D + c] = (uint8_t)par;
}
// After a barrier: carry of the earlier quarters, reference row 31, chunk totals.
__device__ __forceinline__ void prepc_carry(int c, int cq, PrepC &P, const float *qt, const uint8_t *qp) {
  float cg = 0.f, gm = 0.f, gc = 0.f;
  uint32_t cp = 0, pc = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float t = qt[q * D + c];
    const uint32_t b = qp[q * D + c];
    if (q < cq) { cg += t; cp ^= b; }
    if (q <= 1) gm += t;
    gc += t;
    pc ^= b;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) P.G[i] += cg;
  if (cp) P.pre ^= 0xffffu;
  P.Gm = gm;
  P.GC = gc;
  P.pC = pc;
}

__global__ void __launch_bounds__(kGThreads, 1) tc_grad_kernel(const __grid_constant__ BwdTcArgs ta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  GMisc &ms = *reinterpret_cast<GMisc *>(sm + G_MISC);
  const BwdArgs &a = ta.b;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const __nv_bfloat16 *beta = (const __nv_bfloat16 *)a.beta;
  __nv_bfloat16 *dq = (__nv_bfloat16 *)a.dq, *dk = (__nv_bfloat16 *)a.dkg;
  __nv_bfloat16 *dv = (__nv_bfloat16 *)a.dvg, *dbeta = (__nv_bfloat16 *)a.dbeta;

  if (tid == 0) {
    // MMA groups that do not share an accumulator are issued by lane 0 of up
    // to three warps (a tcgen05.mma takes tens of ns to issue): each such
    // barrier counts one commit per issuing thread
    const uint32_t issuers[7] = {1, 1, 2, 3, 2, 2, 1};  // (bar[6] is unused)
    for (int i = 0; i < 7; ++i) mbar_init(&ms.bar[i], issuers[i]);
    mbar_init(&ms.mdu, 1);
    mbar_init(&ms.mds, 1);
    mbar_init(&ms.mfin, 3);
    mbar_init(&ms.mrec, 1);
    mbar_init(&ms.mld, 1);
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
  const uint32_t sA1 = smem_u32(sm + G_A1), sB1 = smem_u32(sm + G_B1);
  const uint32_t sUV = smem_u32(sm + G_UV), sTT = smem_u32(sm + G_TT), sOU = smem_u32(sm + G_OU);
  const uint32_t sSC = smem_u32(sm + G_SC), sWN = smem_u32(sm + G_WN);
  float *dTf = reinterpret_cast<float *>(sm + G_DT);
  float *Mf = reinterpret_cast<float *>(sm + G_MF);
  float *fb = ta.fb + (size_t)blockIdx.x * 3 * 64 * D;

  // TMEM-facing mapping: lane quadrant qd of the accumulator rows, column
  // quarter cq; c = 32 qd + lane is the accumulator row (channel) of this
  // thread, and the key channel of its prep (rows 16 cq .. 16 cq + 15)
  const int qd = warp & 3, cq = warp >> 2;
  const int c = tid & 127;
  const uint32_t lanebase = tmem + ((uint32_t)(32 * qd) << 16);
  const int nitems = a.map.n_chunks() * H;

  // Every load of one item: the reverse pass's dU tile, the forward's W tile,
  // M, S_c^T and T, and the row tensors (q, k staged in A1, g in B1 + KG, sign
  // in the dT scratch -- the prep consumes them before those regions are
  // written -- V into rows 64.. of [U; V] and dO into rows 0..63 of [dO; dU],
  // K-major SW128 boxes).  Issued in stages as the previous item's last
  // readers of these regions finish.
  // thread 0's count of issued load sets (each completes mld, mrec and mdu
  // once) and of the completions it has seen: an abort drains the rest
  uint32_t n_issued = 0, n_mld = 0, n_mrec = 0, n_mdu = 0;
  // The next item's copies go out in five stages, each as soon as the regions
  // it fills are no longer read by the current item, so that the loads spread
  // over the item instead of piling up at its end:
  //   0 (after the third MMA group): dU and dO into [dO; dU]; the dS tile into L2
  //   1 (after the fourth):          S_c^T into the S tile, the record's T into T
  //   2 (after the dM M^T products): M
  //   3 (after dL):                  V into rows 64.. of [U; V]
  //   4 (after X, Y):                q, k into A1, g into B1 + KG, the W tile, sign
  //                                  into the dT scratch (dead by then)
  // One copy per warp (lane 0) within a stage.  The three byte counts of the
  // set are posted by thread 0 once the current item's phases of mld, mrec and
  // mdu have completed; a transiently negative transaction count is allowed
  // (a phase also needs that arrive).  `staged` counts the stages issued for
  // the pending set; a wind-down issues the rest first, so that every phase
  // it waits for completes.
  bool posted = false;
  int staged = 0, pending_item = -1;
  auto post_bytes = [&]() {
    mbar_arrive_expect_tx(&ms.mdu, DU_TILE);
    mbar_arrive_expect_tx(&ms.mrec, W_TILE + M_BYTES + S_TILE + T_TILE);
    mbar_arrive_expect_tx(&ms.mld, kRowBytesQK + kRowBytesG + (a.sign ? kRowBytesSign : 0) + 2 * 16384);
  };
  // copy `w` of stage `st` for item itm (w < number of copies of the stage)
  auto stage_copy = [&](int st, int w, int itm) {
    int sq_, len_, jl_;
    int64_t tk_;
    a.map.info(itm / H, sq_, tk_, len_, jl_);
    const int hh = itm % H, t = (int)tk_;
    const unsigned char *gdU = ta.dU_tiles + (size_t)itm * DU_TILE;
    const unsigned char *rec = ta.recs + (size_t)itm * REC;
    fence_async_smem();  // earlier generic accesses of the destinations come first
    if (st == 0) {
      if (w == 0) bulk_g2s(sm + G_OU + 8192, gdU, 8192, &ms.mdu);
      else if (w == 1) bulk_g2s(sm + G_OU + 16384 + 8192, gdU + 8192, 8192, &ms.mdu);
      else if (w == 2) tma_rows(sm + G_OU, &ta.rm.dO, 0, hh, t, &ms.mld);
      else if (w == 3) tma_rows(sm + G_OU + 16384, &ta.rm.dO, 64, hh, t, &ms.mld);
      else prefetch_l2(ta.dS_tiles + (size_t)itm * DS_TILE, DS_TILE);  // copied in mid-item
    } else if (st == 1) {
      if (w == 0) bulk_g2s(sm + G_SC, rec + R7, S_TILE, &ms.mrec);
      else bulk_g2s(sm + G_TT, rec + R8, T_TILE, &ms.mrec);
    } else if (st == 2) {
      bulk_g2s(sm + G_MF, rec + R6, M_BYTES, &ms.mrec);
    } else if (st == 3) {
      tma_rows(sm + G_UV + 8192 + 8192 * w * 2, &ta.rm.v, 64 * w, hh, t, &ms.mld);
    } else {
      if (w == 0) bulk_g2s(sm + G_WN, rec + R1, W_TILE, &ms.mrec);
      else if (w <= 2) tma_rows(sm + G_A1 + kStageQ + 8192 * (w - 1), &ta.rm.q, 64 * (w - 1), hh, t, &ms.mld);
      else if (w <= 4) tma_rows(sm + G_A1 + kStageK + 8192 * (w - 3), &ta.rm.k, 64 * (w - 3), hh, t, &ms.mld);
      else if (w == 5) tma_rows(sm + G_B1, &ta.rm.g, 0, hh, t, &ms.mld);
      else if (a.sign) tma_rows(sm + G_SGN, &ta.rm.sign, 0, hh, t, &ms.mld);
    }
  };
  constexpr int kStageCopies[5] = {5, 2, 1, 2, 7};
  // stage st of the next item's set, issued by lane 0 of the first warps
  auto issue_stage = [&](int st, int itm) {
    if (tid == 0 && st == 0 && !posted) {  // (the first item: counts not posted yet)
      post_bytes();
      posted = true;
      pending_item = itm;
    }
    if (lane == 0 && warp < kStageCopies[st]) stage_copy(st, warp, itm);
    staged = st + 1;
    if (st == 4) {
      if (tid == 0) ++n_issued;
      posted = false;
      staged = 0;
    }
  };
  auto issue_loads = [&](int itm) {  // every stage at once (the first item)
    for (int st = 0; st < 5; ++st) issue_stage(st, itm);
  };

  uint32_t it = 0;
  bool abort = false;
  for (int item = blockIdx.x; item < nitems && !abort; item += gridDim.x, ++it) {
    const uint32_t ph = it & 1;
    const int cid = item / H, h = item % H;
    const int next_item = item + (int)gridDim.x;
    const bool has_next = next_item < nitems;
    int seq, len, jl;
    int64_t tok0;
    a.map.info(cid, seq, tok0, len, jl);
    const unsigned char *gdS = ta.dS_tiles + (size_t)item * DS_TILE;

    // ---------------- loads ----------------
    if (it == 0) issue_loads(item);  // later items: during the previous one
    // beta rows: loaded here for the first item, during the previous item's
    // final epilogue for the others
    if (it == 0 && tid < 64) ms.beta[tid] = tid < len ? __bfloat162float(beta[(size_t)(tok0 + tid) * H + h]) : 0.f;
    if (!wait_all(&ms.mld, ph, a.status, 400)) { abort = true; break; }
    ++n_mld;
    PrepC P;
    prepc_load(sm + G_A1, reinterpret_cast<const float *>(sm + G_B1), a.sign ? sm + G_SGN : nullptr, len, c, cq,
               P, &ms.qt[0][0], &ms.qp[0][0]);
    if (len < 64) {  // V and dO rows past the chunk
      zero_tail_rows(sm + G_UV + 8192, 16384, len, tid, kGThreads);
      zero_tail_rows(sm + G_OU, 16384, len, tid, kGThreads);
    }
    __syncthreads();
    prepc_carry(c, cq, P, &ms.qt[0][0], &ms.qp[0][0]);
    int bad = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (!(fabsf(P.G[i] - P.Gm) <= kTau)) bad = 1;
    const bool fast = !__syncthreads_or(bad);

    // ---------------- operand tiles ----------------
    // the stores of a warp cover 32 consecutive channels of one row
    if (fast) {
      const float eGm = fast_exp(P.Gm);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * cq + i;
        const float p = ((P.pre >> i) & 1u) ? -1.f : 1.f;
        const float kp = p * bf_lo(P.kq[i]), qp = p * bf_hi(P.kq[i]);
        const float el = fast_exp(P.G[i] - P.Gm), er = rcp_approx(el);
        st_bf16(sm + G_A1, kmaj_off(r, c, 128), qp * el);
        st_bf16(sm + G_A1, kmaj_off(64 + r, c, 128), kp * el);
        st_bf16(sm + G_B1, kmaj_off(r, c, 64), kp * er);
      }
    } else {
      // (unrolled: the prep arrays must stay in registers, which a runtime
      // index into them would prevent)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * cq + i;
        const float p = ((P.pre >> i) & 1u) ? -1.f : 1.f;
        const float kp = p * bf_lo(P.kq[i]), qp = p * bf_hi(P.kq[i]);
        fb[r * D + c] = P.G[i];
        fb[64 * D + r * D + c] = kp;
        fb[128 * D + r * D + c] = qp;
        st_bf16(sm + G_A1, kmaj_off(64 + r, c, 128), kp * fast_exp(P.G[i]));  // KG itself (A1 is idle here)
      }
    }
    fence_async_smem();  // (the wait below is the barrier before the MMAs read the tiles)

    // ---------------- the record's tiles (W, M, S_c^T, T = M Diag(beta)) ----------------
    if (!wait_all(&ms.mrec, ph, a.status, 401)) { abort = true; break; }
    ++n_mrec;

    // ---------------- A (kept in TMEM for dbeta), U^T = V^T T^T - (W S)^T ----------------
    if (tid == 32) {  // A, by a second thread (its commit is part of this phase)
      tc_fence_after();
      if (fast) {
        const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem, sdesc_off(sdesc(sA1, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32),
                   sdesc_off(sdesc(sB1, 16, 1024), (kk >> 2) * 8192 + (kk & 3) * 32), id, kk > 0);
      }
      mma_commit(&ms.bar[2]);
    }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idu = idesc_bf16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 128, sdesc_off(sdesc(sUV + 8192, 16384, 1024), kk * 2048), sdesc_off(sdesc(sTT, 16, 1024), kk * 32), idu,
                 kk > 0);
      const uint32_t idw = idesc_bf16(128, 64, false, true) | (1u << 13);  // negate A: subtract
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + 128, sdesc_off(sdesc(sSC, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32),
                 sdesc_off(sdesc(sWN, 16384, 1024), kk * 2048), idw, true);
      mma_commit(&ms.bar[2]);
    }
    if (!wait_one(&ms.bar[2], ph, a.status, 403)) { abort = true; break; }
    tc_fence_after();
    if (tid == 0) {  // the W tile is dead: bring dL/dS_{c+1} into its place
      mbar_arrive_expect_tx(&ms.mds, DS_TILE);
      bulk_g2s(sm + G_WN, gdS, DS_TILE, &ms.mds);
    }
    {  // U rows s (K-major [s][v]) of the [U; V] tile: lane = v, columns 16 cq ..
      float u[16];
      tmem_ld16(lanebase + 128 + 16 * cq, u);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) st_bf16(sm + G_UV, kmaj_off(16 * cq + i, c, 128), u[i]);
    }
    if (!wait_one(&ms.mdu, ph, a.status, 405)) { abort = true; break; }
    ++n_mdu;
    // the item's phases of mld, mrec and mdu are complete: post the next set's counts
    if (tid == 0 && has_next) {
      post_bytes();
      posted = true;
      pending_item = next_item;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- [dQG^T | S dU^T], dV^T, D7 part 1; then dKhat^T ----------------
    // (three independent groups, three issuing threads; dKhat^T, the one product
    // that needs the reverse pass's dS tile, is issued once that tile is in)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id1 = idesc_bf16(128, 128, true, false);  // S_c read MN-major (K = v)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + 256, sdesc_off(sdesc(sSC, 16384, 1024), kk * 2048),
                 sdesc_off(sdesc(sOU, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32), id1, kk > 0);
      mma_commit(&ms.bar[3]);
    } else if (tid == 32) {
      tc_fence_after();
      // dV^T = dU^T T^T (T and dU are in place)
      const uint32_t idT = idesc_bf16(128, 64, true, true);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 448, sdesc_off(sdesc(sOU + 8192, 16384, 1024), kk * 2048),
                 sdesc_off(sdesc(sTT, 8192, 1024), kk * 2048), idT, kk > 0);
      // (its commit follows dKhat^T below: one arrival per issuing thread)
    } else if (tid == 64) {
      tc_fence_after();
      // D7, first part: [dO; dU][U; V]^T (needs neither dW nor the epilogue below)
      const uint32_t id3 = idesc_bf16(128, 128, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16(tmem + 128, sdesc_off(sdesc(sOU, 16, 1024), ko), sdesc_off(sdesc(sUV, 16, 1024), ko), id3, kk > 0);
      }
      mma_commit(&ms.bar[3]);
    }
    // the dS_{c+1} tile is in place (every thread reads it): dKhat^T = dS1^T U^T
    // on the tensor cores, and meanwhile dd = diag(S_c dS1^T) on the CUDA cores
    if (!wait_all(&ms.mds, ph, a.status, 404)) { abort = true; break; }
    if (tid == 32) {
      tc_fence_after();
      const uint32_t id2 = idesc_bf16(128, 64, true, false);  // dS1 read MN-major (K = v)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + 384, sdesc_off(sdesc(sWN, 16384, 1024), kk * 2048),
                 sdesc_off(sdesc(sUV, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32), id2, kk > 0);
      mma_commit(&ms.bar[3]);
    }
    {  // dd[c] = sum over v of S_c[c][v] dS1[c][v] (both tiles K-major [v][c]): this
      // thread takes channels 2 cp, 2 cp + 1 (one 32-bit word per row) over an
      // eighth of the v; the eighths are summed in the epilogue
      const int cp = tid & 63, vg = tid >> 6;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
      for (int v = 16 * vg; v < 16 * vg + 16; ++v) {
        const uint32_t off = kmaj_off(v, 2 * cp, 128);
        const float2 sv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + G_SC + off));
        const float2 dv2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + G_WN + off));
        a0 = fmaf(sv.x, dv2.x, a0);
        a1 = fmaf(sv.y, dv2.y, a1);
      }
      *reinterpret_cast<float2 *>(&ms.ddp[vg][2 * cp]) = make_float2(a0, a1);
    }
    if (!wait_one(&ms.bar[3], ph, a.status, 406)) { abort = true; break; }
    tc_fence_after();
    if (has_next) issue_stage(0, next_item);
    {  // dW = -dU S_c^T -> rows 64..127 of the S_c tile (K-major [i][c]); S_c is dead.
      // Fast path: stored as dW Diag(e^{Gam_m}) (channel c scaled by e^{Gam_m,c}),
      // so that KG = K~l Diag(e^{Gam_m}) is never formed: dW KG^T = (dW Diag(e^{Gam_m})) K~l^T,
      // and dKG comes out scaled by e^{Gam_m} too (the epilogue uses el for E there)
      const float sc = fast ? -fast_exp(P.Gm) : -1.f;
      float w[16];
      tmem_ld16(lanebase + 320 + 16 * cq, w);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) st_bf16(sm + G_SC, kmaj_off(64 + 16 * cq + i, c, 128), sc * w[i]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- D7 = [dO; dU][U; V]^T + [.; dW] KG^T (second part), dKG^T ----------------
    // (KG^T read as the K~l rows 64..127 of A1 -- KG itself on the exact path --
    // against the scaled dW)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id2 = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + 192, sdesc_off(sdesc(sSC, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32),
                 sdesc_off(sdesc(sA1 + 8192, 16, 1024), (kk >> 2) * 16384 + (kk & 3) * 32), id2, true);
      mma_commit(&ms.bar[4]);
    } else if (tid == 32) {
      tc_fence_after();
      // dKG^T = dW^T T^T (dW just written)
      const uint32_t idT = idesc_bf16(128, 64, true, true);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 64, sdesc_off(sdesc(sSC + 8192, 16384, 1024), kk * 2048), sdesc_off(sdesc(sTT, 8192, 1024), kk * 2048), idT,
                 kk > 0);
      mma_commit(&ms.bar[4]);
    }
    if (!wait_one(&ms.bar[4], ph, a.status, 407)) { abort = true; break; }
    tc_fence_after();
    if (has_next) issue_stage(1, next_item);
    {
      float x[16];
      if (qd < 2) {  // dA_q rows -> bf16 rows 64..127 of the [dA; dA_q] tile; M rows as hi / lo
        const int r = c;
        tmem_ld16(lanebase + 128 + 16 * cq, x);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int s0 = 16 * cq + 2 * jj;
          pk[jj] = pack_bf16(s0 <= r ? x[2 * jj] : 0.f, s0 + 1 <= r ? x[2 * jj + 1] : 0.f);
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
          *reinterpret_cast<uint4 *>(sm + G_WN + kmaj_off(64 + r, 16 * cq + 8 * m, 128)) =
              make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int a0 = 16 * cq + 8 * m;
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) split_bf16x2(Mf[r * LDF + a0 + 2 * e], Mf[r * LDF + a0 + 2 * e + 1], hi[e], lo[e]);
          *reinterpret_cast<uint4 *>(sm + G_MH + kmaj_off(r, a0, 64)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(sm + G_ML + kmaj_off(r, a0, 64)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      } else {  // dT rows (masked j <= i) -> fp32, and dM = dT Diag(beta) as bf16 hi + lo parts
        const int i = c - 64;
        tmem_ld16(lanebase + 192 + 16 * cq, x);
        tmem_wait_ld();
        float dm[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = 16 * cq + jj;
          const float val = j <= i ? x[jj] : 0.f;
          dTf[i * LDF + j] = val;
          dm[jj] = val * ms.beta[j];
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) split_bf16x2(dm[8 * m + 2 * e], dm[8 * m + 2 * e + 1], hi[e], lo[e]);
          *reinterpret_cast<uint4 *>(sm + G_DMH + kmaj_off(i, 16 * cq + 8 * m, 64)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(sm + G_DML + kmaj_off(i, 16 * cq + 8 * m, 64)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // tmp = dM M^T on the tensor cores, in three bf16 products of the hi / lo parts
    // (dM_hi M_hi^T + dM_hi M_lo^T + dM_lo M_hi^T, fp32 accumulate: ~16 significant
    // bits).  A has 64 meaningful rows; its other 64 (the next tile) fill TMEM
    // lanes 64..127, which nothing reads.
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint32_t pa = smem_u32(sm + (p == 2 ? G_DML : G_DMH)), pb = smem_u32(sm + (p == 1 ? G_ML : G_MH));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 128, sdesc_off(sdesc(pa, 16, 1024), kk * 32), sdesc_off(sdesc(pb, 16, 1024), kk * 32), id, p > 0 || kk > 0);
      }
      mma_commit(&ms.bar[0]);
    }
    // dbeta (column part): sum_i dT[i][j] M[i][j], eight lanes per column
    {
      const int j = tid >> 3, part = tid & 7;
      float s = 0.f;
      for (int i = j + part; i < 64; i += 8) s += dTf[i * LDF + j] * Mf[i * LDF + j];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (part == 0) ms.dbc[j] = s;
    }
    if (!wait_one(&ms.bar[0], ph, a.status, 410)) { abort = true; break; }
    tc_fence_after();
    if (has_next) issue_stage(2, next_item);  // (M was last read by the dbeta column sums above)
    if (qd < 2) {  // tmp rows i (lanes 0..63) -> bf16 hi + lo tiles, K-major [i][k]
      const int i = c;
      float x[16];
      tmem_ld16(lanebase + 128 + 16 * cq, x);
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split_bf16x2(x[8 * m + 2 * e], x[8 * m + 2 * e + 1], hi[e], lo[e]);
        *reinterpret_cast<uint4 *>(sm + G_TH + kmaj_off(i, 16 * cq + 8 * m, 64)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(sm + G_TL + kmaj_off(i, 16 * cq + 8 * m, 64)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // dL = -M^T tmp, same three-product split: A = M^T is the M tile read
    // MN-major (K = i), B = tmp read MN-major (K = i, N = k); negated A
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, true, true) | (1u << 13);
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint32_t pa = smem_u32(sm + (p == 2 ? G_ML : G_MH)), pb = smem_u32(sm + (p == 1 ? G_TL : G_TH));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 192, sdesc_off(sdesc(pa, 8192, 1024), kk * 2048), sdesc_off(sdesc(pb, 8192, 1024), kk * 2048), id,
                   p > 0 || kk > 0);
      }
      mma_commit(&ms.bar[1]);
    }
    if (!wait_one(&ms.bar[1], ph, a.status, 411)) { abort = true; break; }
    tc_fence_after();
    if (has_next) issue_stage(3, next_item);
    // dN = strict_lower(dL) -> fp32 (for the dbeta row part) and
    // dA = Diag(beta) dN -> bf16 rows 0..63 of the [dA; dA_q] tile
    if (qd < 2) {
      const int r = c;
      float x[16];
      tmem_ld16(lanebase + 192 + 16 * cq, x);
      tmem_wait_ld();
      const float br = ms.beta[r];
      uint32_t pk[8];
#pragma unroll
      for (int jj = 0; jj < 16; jj += 2) {
        const int k0 = 16 * cq + jj;
        const float v0 = k0 < r ? x[jj] : 0.f;
        const float v1 = k0 + 1 < r ? x[jj + 1] : 0.f;
        dTf[r * LDF + k0] = v0;  // row stride 65: scalar stores
        dTf[r * LDF + k0 + 1] = v1;
        pk[jj >> 1] = pack_bf16(br * v0, br * v1);
      }
#pragma unroll
      for (int m = 0; m < 2; ++m)
        *reinterpret_cast<uint4 *>(sm + G_WN + kmaj_off(r, 16 * cq + 8 * m, 128)) =
            make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
    }
    __syncthreads();
    // dbeta (row part): sum_{j < r} dN[r][j] A[r][j]
    if (fast) {
      if (qd >= 2) {
        const int r = c - 64;
        float x[16];
        tmem_ld16(lanebase + 16 * cq, x);
        tmem_wait_ld();
        float s = 0.f;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = 16 * cq + jj;
          if (j < r) s += dTf[r * LDF + j] * x[jj];
        }
        ms.dbr[cq][r] = s;
      }
    } else if (tid < 256) {
      // exact path: recompute the needed A entries from the fallback scratch
      const int r = tid & 63, qq = tid >> 6;
      float s = 0.f;
      for (int j = 16 * qq; j < 16 * qq + 16; ++j) {
        if (j >= r) break;
        float aa = 0.f;
        for (int cc = 0; cc < D; ++cc)
          aa += fb[64 * D + r * D + cc] * fb[64 * D + j * D + cc] * expf(fb[r * D + cc] - fb[j * D + cc]);
        s += dTf[r * LDF + j] * aa;
      }
      ms.dbr[qq][r] = s;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- X^T, Y^T (dV^T and dKG^T were issued earlier) ----------------
    if (tid == 0) {
      tc_fence_after();
      if (fast) {
        const uint32_t idX = idesc_bf16(128, 128, true, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 128, sdesc_off(sdesc(sB1, 8192, 1024), kk * 2048), sdesc_off(sdesc(sWN, 16, 1024), kk * 32), idX, kk > 0);
      }
      mma_commit(&ms.bar[5]);
    } else if (tid == 32) {
      tc_fence_after();
      if (fast) {
        const uint32_t idY = idesc_bf16(128, 64, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 320, sdesc_off(sdesc(sA1 + 8192, 16384, 1024), kk * 2048), sdesc_off(sdesc(sWN, 8192, 1024), kk * 2048),
                   idY, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + 320, sdesc_off(sdesc(sA1, 16384, 1024), kk * 2048), sdesc_off(sdesc(sWN + 8192, 8192, 1024), kk * 2048),
                   idY, true);
      }
      mma_commit(&ms.bar[5]);
    }
    if (!fast) {
      // exact pair terms into the TMEM columns the fast path fills:
      // X1 (128 + r), X2 (192 + r), Y1 (320 + r) of lane c, rows 16 cq ..
      const float *Gc = fb, *kpc = fb + 64 * D, *qpc = fb + 128 * D;
      auto dAv = [&](int r, int s) {  // dA (rows 0..63) / dA_q (rows 64..127) from the bf16 tile
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + G_WN + kmaj_off(r, s, 128)));
      };
      // one column per row into TMEM (no register arrays: this rare path must
      // not raise the register pressure of the common one)
#pragma unroll 1
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * cq + i;
        const float gr = Gc[r * D + c];
        float a1 = 0.f, a2 = 0.f, b1 = 0.f;
        for (int s = 0; s <= r; ++s) {
          const float e = expf(gr - Gc[s * D + c]) * kpc[s * D + c];
          a1 += dAv(r, s) * e;
          a2 += dAv(64 + r, s) * e;
        }
        for (int t = r; t < 64; ++t) {
          const float e = expf(Gc[t * D + c] - gr);
          b1 += (dAv(t, r) * kpc[t * D + c] + dAv(64 + t, r) * qpc[t * D + c]) * e;
        }
        tmem_st1(lanebase + 128 + r, a1);
        tmem_st1(lanebase + 192 + r, a2);
        tmem_st1(lanebase + 320 + r, b1);
      }
      tmem_wait_st();
    }
    if (!wait_one(&ms.bar[5], ph, a.status, 408)) { abort = true; break; }
    tc_fence_after();
    // every shared-memory tile is idle now: the next item's loads overlap the
    // final epilogue (TMEM, registers and the quarter sums only)
    if (has_next) issue_stage(4, next_item);

    // ---------------- final elementwise gradients ----------------
    // thread (c, cq): rows 16 cq .. 16 cq + 15 of key channel c, prep values
    // and accumulators both at hand; dL/dGam stays in registers
    {
      float *qsum = reinterpret_cast<float *>(sm + G_FSUM);  // [2][4][128]
      const float pCs = P.pC ? -1.f : 1.f;
      const float eGm = fast_exp(P.Gm), eCm = fast_exp(P.GC - P.Gm);
      const float dC = pCs * fast_exp(P.GC);
      const size_t rstride = (size_t)H * D;
      // the next item's beta, requested now and stored after the loop below
      float beta_next = 0.f;
      const int nxt = item + gridDim.x;
      if (tid < 64 && nxt < nitems) {
        int sq_, len_, jl_;
        int64_t tk_;
        a.map.info(nxt / H, sq_, tk_, len_, jl_);
        if (tid < len_) beta_next = __bfloat162float(beta[(size_t)(tk_ + tid) * H + nxt % H]);
      }
      float gcp = 0.f, part = 0.f;
      // fast path: the pair terms carry the reference-row scaling; exact path:
      // they are final, and the factors come straight from Gam
      auto rows = [&](auto fast_c) {
        constexpr bool kFast = decltype(fast_c)::value;
#pragma unroll
      // four batches of four rows: seven 4-column loads per batch keep the
      // accumulators of one batch and the prep values within the registers
      for (int b4 = 0; b4 < 4; ++b4) {
        const int r0 = 16 * cq + 4 * b4;
        float X1[4], X2[4], Y1[4], dQG[4], dKG[4], dKh[4], dVv[4];
        tmem_ld4(lanebase + 128 + r0, X1);
        tmem_ld4(lanebase + 192 + r0, X2);
        tmem_ld4(lanebase + 320 + r0, Y1);
        tmem_ld4(lanebase + 256 + r0, dQG);
        tmem_ld4(lanebase + 64 + r0, dKG);
        tmem_ld4(lanebase + 384 + r0, dKh);
        tmem_ld4(lanebase + 448 + r0, dVv);
        tmem_wait_ld();
        const size_t off0 = ((size_t)(tok0 + r0) * H + h) * D + c;
        float dg4[4];  // dL/dGam of the batch's rows: parked in TMEM columns [0, 64) (A is dead)
        // two rows at a time in packed fp32x2 arithmetic (sm_100 FFMA2 / FMUL2)
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
          const int ii = 4 * b4 + i, r = r0 + i;
          const float2 p2 = make_float2(((P.pre >> ii) & 1u) ? -1.f : 1.f, ((P.pre >> (ii + 1)) & 1u) ? -1.f : 1.f);
          const float2 kp = __fmul2_rn(p2, make_float2(bf_lo(P.kq[ii]), bf_lo(P.kq[ii + 1])));
          const float2 qp = __fmul2_rn(p2, make_float2(bf_hi(P.kq[ii]), bf_hi(P.kq[ii + 1])));
          float2 el, er, E, eC;
          if (kFast) {
            el = make_float2(fast_exp(P.G[ii] - P.Gm), fast_exp(P.G[ii + 1] - P.Gm));
            er = make_float2(rcp_approx(el.x), rcp_approx(el.y));
            E = __fmul2_rn(el, make_float2(eGm, eGm));
            eC = __fmul2_rn(er, make_float2(eCm, eCm));
          } else {
            el = er = make_float2(1.f, 1.f);
            E = make_float2(fast_exp(P.G[ii]), fast_exp(P.G[ii + 1]));
            eC = make_float2(fast_exp(P.GC - P.G[ii]), fast_exp(P.GC - P.G[ii + 1]));
          }
          const float2 x1 = __fmul2_rn(el, make_float2(X1[i], X1[i + 1]));
          const float2 x2 = __fmul2_rn(el, make_float2(X2[i], X2[i + 1]));
          const float2 y1 = __fmul2_rn(er, make_float2(Y1[i], Y1[i + 1]));
          const float2 dKG2 = make_float2(dKG[i], dKG[i + 1]), dQG2 = make_float2(dQG[i], dQG[i + 1]);
          const float2 dKh2 = make_float2(dKh[i], dKh[i + 1]);
          const float2 Kh = __fmul2_rn(__fmul2_rn(make_float2(pCs, pCs), kp), eC);   // Khat
          const float2 khd = __fmul2_rn(dKh2, Kh);                                     // dKhat . Khat
          // dk' = x1 + y1 + dKG E + pC dKhat eC;  dq' = x2 + dQG E (on the fast
          // path the dKG accumulator already carries e^{Gam_m}: its factor is el)
          const float2 EK = kFast ? el : E;
          const float2 dkp = __ffma2_rn(make_float2(pCs, pCs), __fmul2_rn(dKh2, eC), __ffma2_rn(dKG2, EK, __fadd2_rn(x1, y1)));
          const float2 dqp = __ffma2_rn(dQG2, E, x2);
          // dL/dGam: k' x1 + q' x2 - k' y1 + dKG KG + dQG QG - dKhat Khat
          float2 dgv = __fmul2_rn(kp, __fadd2_rn(x1, make_float2(-y1.x, -y1.y)));
          dgv = __ffma2_rn(qp, x2, dgv);
          dgv = __ffma2_rn(__fmul2_rn(dKG2, kp), EK, dgv);
          dgv = __ffma2_rn(__fmul2_rn(dQG2, qp), E, dgv);
          dgv = __fadd2_rn(dgv, make_float2(-khd.x, -khd.y));
          dg4[i] = dgv.x;
          dg4[i + 1] = dgv.y;
          part += dgv.x + dgv.y;
          gcp += khd.x + khd.y;
          const float2 oq = __fmul2_rn(p2, dqp), ok = __fmul2_rn(p2, dkp);
          const __nv_bfloat162 bq = __floats2bfloat162_rn(oq.x, oq.y), bk = __floats2bfloat162_rn(ok.x, ok.y);
          const __nv_bfloat162 bv = __floats2bfloat162_rn(dVv[i], dVv[i + 1]);  // lane c is value channel c here
          // lanes 2k, 2k + 1 (channels c, c ^ 1) swap halves: the even lane
          // then holds row r of both channels, the odd one row r + 1, and one
          // 4-byte store per lane writes two rows per warp instruction
          const uint32_t pq = bf162_bits(bq), pk = bf162_bits(bk), pv = bf162_bits(bv);
          const uint32_t xq = __shfl_xor_sync(0xffffffffu, pq, 1), xk = __shfl_xor_sync(0xffffffffu, pk, 1);
          const uint32_t xv = __shfl_xor_sync(0xffffffffu, pv, 1);
          const bool odd = lane & 1;
          const size_t off = off0 + i * rstride + (odd ? rstride - 1 : 0);  // (row r + 1, channel c - 1) on odd lanes
          if ((odd ? r + 1 : r) < len) {
            *reinterpret_cast<uint32_t *>(dq + off) = odd ? __byte_perm(xq, pq, 0x7632) : __byte_perm(pq, xq, 0x5410);
            *reinterpret_cast<uint32_t *>(dk + off) = odd ? __byte_perm(xk, pk, 0x7632) : __byte_perm(pk, xk, 0x5410);
            *reinterpret_cast<uint32_t *>(dv + off) = odd ? __byte_perm(xv, pv, 0x7632) : __byte_perm(pv, xv, 0x5410);
          }
        }
        tmem_st4(lanebase + 16 * cq + 4 * b4, dg4);
      }
      };
      if (fast) rows(std::true_type{});
      else rows(std::false_type{});
      if (tid < 64) ms.beta[tid] = beta_next;  // this item's beta is no longer read
      // reverse in-chunk cumsum of dL/dGam (plus the chunk-end terms) -> dg;
      // the four quarters at once: each starts from the totals of the later ones
      qsum[cq * D + c] = gcp;
      qsum[4 * D + cq * D + c] = part;
      __syncthreads();
      float gC = 0.f, later = 0.f;
      float ddc = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ddc += ms.ddp[e][c];
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        gC += qsum[q2 * D + c];
        if (q2 > cq) later += qsum[4 * D + q2 * D + c];
      }
      float acc = gC + ddc * dC + later;
      float dgs[16];
      tmem_wait_st();
      tmem_ld16(lanebase + 16 * cq, dgs);
      tmem_wait_ld();
#pragma unroll
      for (int ii = 15; ii >= 0; --ii) {
        acc += dgs[ii];
        dgs[ii] = acc;
      }
      // the same pairing as above, 8 bytes per lane: rows 2m (even lanes) and
      // 2m + 1 (odd lanes) of channels c & ~1, c | 1
      {
        const bool odd = lane & 1;
        const size_t base = ((size_t)(tok0 + 16 * cq) * H + h) * D + (c & ~1);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float x = __shfl_xor_sync(0xffffffffu, odd ? dgs[2 * m] : dgs[2 * m + 1], 1);
          const int r = 16 * cq + 2 * m + (odd ? 1 : 0);
          if (r < len)
            *reinterpret_cast<float2 *>(a.dg + base + (size_t)(2 * m + (odd ? 1 : 0)) * H * D) =
                odd ? make_float2(x, dgs[2 * m + 1]) : make_float2(dgs[2 * m], x);
        }
      }
      if (tid < 64 && tid < len)
        dbeta[(size_t)(tok0 + tid) * H + h] = __float2bfloat16_rn(
            ms.dbc[tid] + ms.dbr[0][tid] + ms.dbr[1][tid] + ms.dbr[2][tid] + ms.dbr[3][tid]);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (abort && (tid == 32 || tid == 64)) mma_commit(&ms.mfin);
  if (abort && tid == 0) {
    mma_commit(&ms.mfin);
    mbar_wait(&ms.mfin, 0, a.status, 409);
    // a set whose counts are posted: issue the copies not issued yet, so that
    // its phases complete, then count it
    if (posted) {
      for (int st = staged; st < 5; ++st)
        for (int w = 0; w < kStageCopies[st]; ++w) stage_copy(st, w, pending_item);
      ++n_issued;
    }
    // copies still landing in shared memory finish before the CTA leaves
    for (; n_mld < n_issued; ++n_mld) mbar_wait(&ms.mld, n_mld & 1, a.status, 413);
    for (; n_mrec < n_issued; ++n_mrec) mbar_wait(&ms.mrec, n_mrec & 1, a.status, 414);
    for (; n_mdu < n_issued; ++n_mdu) mbar_wait(&ms.mdu, n_mdu & 1, a.status, 415);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// bf16 S^T tile (K-major [v][c], 128-byte swizzle) of one fp32 chunk state
// [c][v] per CTA: the record field the gradient kernel reads, for callers
// that hand over fp32 chunk states instead of the forward's saved buffer.
__global__ void __launch_bounds__(256) tc_state_tiles_kernel(const float *cs, unsigned char *recs, int H,
                                                             int NC) {
  const int item = blockIdx.x;  // (sequence * NC + chunk) * H + head
  const int h = item % H, cid = item / H, b = cid / NC, j = cid % NC;
  const float *src = cs + (((size_t)b * H + h) * NC + j) * D * D;
  unsigned char *dst = recs + (size_t)item * REC + R7;
  const int v = threadIdx.x & 127, half = threadIdx.x >> 7;
#pragma unroll 2
  for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 8) {
    uint32_t pk[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) pk[m] = pack_bf16(src[(size_t)(c0 + 2 * m) * D + v], src[(size_t)(c0 + 2 * m + 1) * D + v]);
    *reinterpret_cast<uint4 *>(dst + kmaj_off(v, c0, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

int g_sms = 0;
int num_sms() {
  if (g_sms == 0) {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms = n > 0 ? n : 148;
  }
  return g_sms;
}

}  // namespace

// Backward on tensor cores.  recs: records of tc_forward's intra kernel for
// these inputs; dS_tiles / dU_tiles: n_chunks * H tiles of 32 KiB / 16 KiB.
cudaError_t tc_backward(const BwdArgs &b, const unsigned char *recs, unsigned char *dS_tiles,
                        unsigned char *dU_tiles, float *fb, cudaStream_t s, float *seg_ws) {
  BwdTcArgs ta{};
  ta.b = b;
  ta.recs = recs;
  ta.dS_tiles = dS_tiles;
  ta.dU_tiles = dU_tiles;
  ta.fb = fb;
  const size_t sm_sb = SB_MISC + sizeof(SbMisc) + 1024;
  const size_t sm_g = G_MISC + sizeof(GMisc) + 1024;
  cudaError_t e = cudaFuncSetAttribute(tc_state_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm_sb);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tc_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_g);
  if (e != cudaSuccess) return e;
  if (b.map.n_seq == 0) return cudaSuccess;
  // the row tensors' TMA maps (dO for the reverse pass; all of them for the gradient kernel)
  e = make_row_maps(ta.rm, b.q, b.k, b.v, b.dO, b.g, b.sign, (int64_t)b.B * b.T, b.H);
  if (e != cudaSuccess) return e;
  const int G = (seg_ws && !b.map.table) ? tc_seg_count_bwd(b.B, b.H, b.map.NC) : 0;
  if (G >= 2) {
    // long sequences: dS at a segment's start = M_g^T (dS at its end) + e_g, with
    // M_g the forward map of the segment's chunks and e_g the reverse pass from
    // zero; the segments' maps, their provisional passes, the reverse scan, then
    // every segment's pass from its true end state
    FwdArgs f{};
    f.B = b.B; f.T = b.T; f.H = b.H; f.dk = b.dk; f.dv = b.dv;
    f.map = b.map;
    f.status = b.status;
    const size_t per = (size_t)b.B * G * b.H * D * D;
    float *segM = seg_ws, *sege = seg_ws + per, *segE = seg_ws + 2 * per;
    if ((e = tc_seg_maps_rows(f, recs, G, segM, sege, s)) != cudaSuccess) return e;
    ta.seg_count = G;
    ta.seg_len = (b.map.NC + G - 1) / G;
    ta.seg_in = nullptr;
    ta.seg_out = sege;
    ta.no_tiles = true;
    {
      ProfScope prof("tc_state_bwd_provisional", s);
      tc_state_bwd_kernel<<<dim3(b.H, b.B * G), kSbThreads, sm_sb, s>>>(ta);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = tc_seg_scan_reverse(f, G, segM, sege, b.dST, segE, s)) != cudaSuccess) return e;
    ta.seg_in = segE;
    ta.seg_out = nullptr;
    ta.no_tiles = false;
    ProfScope prof("tc_state_bwd", s);
    tc_state_bwd_kernel<<<dim3(b.H, b.B * G), kSbThreads, sm_sb, s>>>(ta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ta.seg_len = 0;
  } else {
    ProfScope prof("tc_state_bwd", s);
    tc_state_bwd_kernel<<<dim3(b.H, b.map.n_seq), kSbThreads, sm_sb, s>>>(ta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    ProfScope prof("tc_grad", s);
    tc_grad_kernel<<<num_sms(), kGThreads, sm_g, s>>>(ta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t tc_state_tiles(const float *chunk_states, unsigned char *recs, int B, int H, int NC,
                           cudaStream_t s) {
  const int64_t items = (int64_t)B * NC * H;
  if (items == 0) return cudaSuccess;
  ProfScope prof("tc_state_tiles", s);
  tc_state_tiles_kernel<<<(unsigned)items, 256, 0, s>>>(chunk_states, recs, H, NC);
  return cudaGetLastError();
}

size_t tc_bwd_smem_bytes() { return G_MISC + sizeof(GMisc) + 1024; }
static_assert(G_MISC + sizeof(GMisc) + 1024 <= 232448, "gradient kernel shared memory");

}  // namespace ckda
