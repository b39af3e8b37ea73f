// ckda_tc.cuh -- sm_100a building blocks: tcgen05 (5th-generation tensor core
// MMA with TMEM accumulators), shared-memory matrix descriptors, mbarriers
// with bounded waits, bulk async copies.  Inline PTX only (PTX ISA forms).
#pragma once

#include <cuda.h>  // CUtensorMap (a plain 128-byte descriptor type)
#include <cuda_bf16.h>
#include <stdint.h>

#include "ckda_internal.cuh"

namespace ckda {
namespace tc {

// Tensor maps of the per-token row tensors, viewed as [tokens][H][128]: each
// TMA box is 64 tokens x one head x 64 channels (bf16, 128-byte swizzle: the
// K-major SW128 tile layout) or 128 channels (g fp32, sign int8; plain rows).
// Rows past the last token read as zeros.  Without a sign tensor (standard
// KDA, every sign +1) the sign map stays empty and is never used.
struct RowMaps {
  CUtensorMap q, k, v, dO, g, sign;
};
// host: encode the maps for ntok tokens of H heads (dO may be null)
cudaError_t make_row_maps(RowMaps &m, const void *q, const void *k, const void *v, const void *dO,
                          const float *g, const int8_t *sign, int64_t ntok, int H);

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after `limit` polls, records the failure in the
// device status word and returns false (the caller then winds down).  A poll
// that finds the phase incomplete suspends the thread for about 4 us on B200
// (measured), so the default gives up after about 4 s; every wait of these
// kernels completes within microseconds.
constexpr uint32_t kWaitPolls = 1u << 20;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase, DevStatus *st,
                                          uint32_t site, uint32_t limit = kWaitPolls) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, phase)) return true;
  if (st) {
    atomicOr(&st->flags, kFlagTimeout);
    atomicCAS(&st->detail, 0u, site);
  }
  return false;
}
// Plain arrive (release): for hand-offs between warp groups of one CTA.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Barrier over `nthreads` threads (a warp group) with id `id` (1..15), and
// its OR-reduction form: every thread of the group gets the OR of `v`.
__device__ __forceinline__ void group_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ bool group_sync_or(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
// The same wait out of line, for kernels that wait at many sites: one copy
// of the loop keeps their instruction footprint small (the latency-bound
// state passes keep the inline form).
static __device__ __noinline__ bool mbar_wait_ool(uint64_t *bar, uint32_t phase, DevStatus *st, uint32_t site) {
  return mbar_wait(bar, phase, st, site);
}

// ---------------------------------------------------------------------------
// bulk async copy global -> shared (1-D, 16-byte aligned, size % 16 == 0)
// ---------------------------------------------------------------------------
// Bulk async copy shared -> global (1-D, both 16-byte aligned, size % 16 ==
// 0), tracked by the issuing thread's bulk groups: commit, then wait until
// the source may be overwritten (.read) or the data is written.
__device__ __forceinline__ void bulk_s2g(void *gmem_dst, const void *smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
// L2 prefetch of a 16-byte aligned range (size % 16 == 0), fire and forget.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One TMA box of a RowMaps tensor: channels c0.., head h, tokens tok..tok+63.
// c0 * element size is a multiple of 16 bytes (0 or 64 channels of bf16).
__device__ __forceinline__ void tma_rows(void *smem_dst, const CUtensorMap *map, int c0, int h, int tok,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(h), "r"(tok), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// fences
// ---------------------------------------------------------------------------
// generic-proxy shared-memory writes -> visible to the async proxy (MMA, bulk copies)
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMEM allocation (one full warp executes these)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ---------------------------------------------------------------------------
// TMEM <-> registers (32 lanes x 32-bit; warp w of a warpgroup sees lanes
// 32*(w%4) .. +31; taddr = (lane << 16) | column)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// shared-memory matrix descriptors, 128-byte swizzle
//
// K-major tile: rows of 64 bf16 (128 B); 8-row groups of 1024 B at stride
//   SBO; a K range wider than 64 continues in another 64-column block.
// MN-major tile: for each K index a row of 64 MN-contiguous bf16 (128 B);
//   8 K-rows form a 1024 B atom; atoms along K at stride SBO, along MN at
//   stride LBO.
// In both, the 16-byte chunk index within a 128 B row is XORed with the
// row's index within its 8-row group (bits [4,7) ^= bits [7,10) of the
// address), so tiles start at 1024-byte aligned addresses.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;  // 128-byte swizzle
  return d;
}

// The same descriptor for the tile `byte_off` bytes further on (a multiple of
// 16): only the 14-bit start-address field moves, and shared-memory
// addresses stay below 2^18, so the add never carries out of it.  Lets one
// thread issue a run of MMAs with one add per operand instead of rebuilding
// each 64-bit descriptor.
__device__ __forceinline__ uint64_t sdesc_off(uint64_t d, uint32_t byte_off) { return d + (byte_off >> 4); }

// byte offset of element (row, col) inside a K-major SW128 tile whose rows
// are `rows` long groups of 64 columns (col may exceed 63: next 64-col block)
__host__ __device__ __forceinline__ uint32_t kmaj_off(int row, int col, int rows) {
  const int blk = col >> 6, c = col & 63;
  return (uint32_t)(blk * rows * 128 + row * 128 + ((((c >> 3) ^ (row & 7)) << 4) | ((c & 7) << 1)));
}
// byte offset of element (k, mn) inside an MN-major SW128 tile with `kdim`
// rows along K (SBO = 1024, LBO = kdim * 128)
__host__ __device__ __forceinline__ uint32_t mnmaj_off(int k, int mn, int kdim) {
  const int blk = mn >> 6, c = mn & 63;
  return (uint32_t)(blk * kdim * 128 + k * 128 + ((((c >> 3) ^ (k & 7)) << 4) | ((c & 7) << 1)));
}

// Instruction descriptor, kind::f16, bf16 x bf16 -> fp32.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                      // D fp32
         | (1u << 7)                    // A bf16
         | (1u << 10)                   // B bf16
         | ((a_mn ? 1u : 0u) << 15)     // A major
         | ((b_mn ? 1u : 0u) << 16)     // B major
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// The same, executed by a whole warp: one lane (elect.sync) issues it.
__device__ __forceinline__ void mma_bf16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// bf16 pair packing
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
// the 32 bits of a bf16 pair
__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): a pair of bf16 values
// that carries ~16 significant bits into a tensor-core product
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = pack_bf16(a - hf.x, b - hf.y);
}

// ---------------------------------------------------------------------------
// per (chunk, head) record of the intra-chunk kernel (bf16 I/O, dk = dv = 128),
// laid out as the shared-memory image its consumers read (tiles 1024-aligned)
// ---------------------------------------------------------------------------
constexpr int D = 128;
constexpr float kTau = 40.f;  // bound on |Gam_r - Gam_m| for the factored operands
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t R1 = 0;       // [W^T | QG^T]: MN-major B tile, K = c (128), N = r' (128)
constexpr uint32_t R2 = 32768;   // U0^T: K-major tile [v][s] (128 x 64)
constexpr uint32_t R3 = 49152;   // A_q: K-major tile [r][s] (64 x 64)
constexpr uint32_t R4 = 57344;   // Khat^T: K-major tile [c][s] (128 x 64)
constexpr uint32_t R5 = 73728;   // d[128] fp32
constexpr uint32_t R6 = 74240;   // M = (I + Diag(beta) A)^{-1}: fp32 [64][65] (row stride 65)
constexpr uint32_t R7 = 90880;   // S_c^T bf16, K-major [v][c] 128 x 128: the chunk-start state
                                 // (written by the state pass, read by the backward)
constexpr uint32_t R8 = 123648;  // T = M Diag(beta) bf16, K-major [r][j] 64 x 64 (read by the backward)
constexpr uint32_t REC_STATE = R6;  // R1 .. R5: the part the sequential state passes read
constexpr uint32_t REC = 131840;    // bytes per (chunk, head) record

// 2^x and 1/x with one MUFU instruction each (PTX ex2.approx / rcp.approx);
// their relative error (~2^-22) is far below the bf16 operand rounding.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fast_exp(float x) { return ex2_approx(x * kLog2e); }

__device__ __forceinline__ void st_bf16(unsigned char *base, uint32_t off, float x) {
  *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// Chunk preprocessing in the "row-group" thread layout (256 threads):
// warp w owns chunk rows 8w .. 8w+7, lane l owns key channels 4l .. 4l+3.
// Each warp reads whole 128-channel rows of the staged (TMA-loaded) tiles.
// ---------------------------------------------------------------------------
// per-group totals exchanged through shared memory (G is accessed as float4)
struct alignas(16) PrepTot {
  float G[8][128];
  uint8_t P[8][128];
};

struct Prep {
  float G[8][4];     // chunk-local inclusive cumsum of g (after the carry)
  uint32_t k2[8][2]; // raw bf16 k, two channels per word
  uint32_t q2[8][2];
  uint32_t pre;      // bit 4*rr+m: sign product of row 8w+rr, channel 4l+m is negative
  float Gm[4], GC[4];
  uint32_t pC;       // bit m: chunk sign product of channel 4l+m is negative
};

// Staged rows of one chunk-head in shared memory (TMA boxes, see RowMaps):
// q and k as K-major SW128 tiles of 64 rows (two 64-channel blocks), g as
// fp32 [64][128], sign as int8 [64][128] (null: no sign tensor, all +1).
// Rows past the chunk's length hold other tokens or zeros; they are masked
// here.
constexpr uint32_t kStageQ = 0, kStageK = 16384;  // offsets inside the q|k staging region
constexpr uint32_t kRowBytesQK = 2 * 16384, kRowBytesG = 32768, kRowBytesSign = 8192;

// Reads the 8 x 4 block of this thread, local scans, writes the group totals.
__device__ __forceinline__ void prep_load_smem(const unsigned char *sqk, const float *sg, const uint8_t *ss,
                                               int len, int w, int l, Prep &P, PrepTot &tot) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t par = 0, pre = 0;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int r = 8 * w + rr;
    const bool valid = r < len;
    const float4 gv = *reinterpret_cast<const float4 *>(sg + r * D + 4 * l);
    const uint32_t sgn = ss ? *reinterpret_cast<const uint32_t *>(ss + r * D + 4 * l) : 0u;
    const uint32_t off = kmaj_off(r, 4 * l, 64);
    const uint2 kv = *reinterpret_cast<const uint2 *>(sqk + kStageK + off);
    const uint2 qv = *reinterpret_cast<const uint2 *>(sqk + kStageQ + off);
    P.k2[rr][0] = valid ? kv.x : 0u;
    P.k2[rr][1] = valid ? kv.y : 0u;
    P.q2[rr][0] = valid ? qv.x : 0u;
    P.q2[rr][1] = valid ? qv.y : 0u;
    const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      acc[m] += valid ? gg[m] : 0.f;
      P.G[rr][m] = acc[m];
      const bool neg = valid && (int8_t)((sgn >> (8 * m)) & 0xffu) < 0;
      par ^= (neg ? 1u : 0u) << m;
    }
    pre |= par << (4 * rr);
  }
  P.pre = pre;
  *reinterpret_cast<float4 *>(&tot.G[w][4 * l]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
#pragma unroll
  for (int m = 0; m < 4; ++m) tot.P[w][4 * l + m] = (uint8_t)((par >> m) & 1u);
}

// Zero rows len..63 of a 64-row, 128-channel K-major SW128 tile (two 8 KiB
// blocks at `base` and `base + block_stride`): whole 128-byte rows, so the
// swizzle does not matter.
__device__ __forceinline__ void zero_tail_rows(unsigned char *base, uint32_t block_stride, int len, int tid,
                                               int nthreads) {
  for (int e = tid; e < (64 - len) * 16; e += nthreads) {
    const int r = len + (e >> 4), ch = e & 15;
    *reinterpret_cast<uint4 *>(base + (ch >> 3) * block_stride + r * 128 + (ch & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
}

// After a barrier: add the carry of the earlier row groups; reference row 31
// and chunk totals per channel.
__device__ __forceinline__ void prep_carry(int w, int l, Prep &P, const PrepTot &tot) {
  float cg[4] = {0.f, 0.f, 0.f, 0.f}, gm[4] = {0.f, 0.f, 0.f, 0.f}, gc[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t cp = 0, pc = 0;
#pragma unroll
  for (int ww = 0; ww < 8; ++ww) {
    const float4 t = *reinterpret_cast<const float4 *>(&tot.G[ww][4 * l]);
    const float tt[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t pb = tot.P[ww][4 * l + m];
      if (ww < w) { cg[m] += tt[m]; cp ^= pb << m; }
      if (ww <= 3) gm[m] += tt[m];
      gc[m] += tt[m];
      pc ^= pb << m;
    }
  }
#pragma unroll
  for (int rr = 0; rr < 8; ++rr)
#pragma unroll
    for (int m = 0; m < 4; ++m) P.G[rr][m] += cg[m];
  uint32_t rep = 0;  // replicate the 4-bit carry parity over the 8 rows
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) rep |= cp << (4 * rr);
  P.pre ^= rep;
#pragma unroll
  for (int m = 0; m < 4; ++m) { P.Gm[m] = gm[m]; P.GC[m] = gc[m]; }
  P.pC = pc;
}

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
// raw k (q) of row rr, channel m of this thread
__device__ __forceinline__ float prep_k(const Prep &P, int rr, int m) {
  const uint32_t w2 = P.k2[rr][m >> 1];
  return (m & 1) ? bf_hi(w2) : bf_lo(w2);
}
__device__ __forceinline__ float prep_q(const Prep &P, int rr, int m) {
  const uint32_t w2 = P.q2[rr][m >> 1];
  return (m & 1) ? bf_hi(w2) : bf_lo(w2);
}
__device__ __forceinline__ float prep_p(const Prep &P, int rr, int m) {
  return ((P.pre >> (4 * rr + m)) & 1u) ? -1.f : 1.f;
}
// 4 consecutive bf16 (8 bytes) of a row of a 128-byte-swizzled tile
__device__ __forceinline__ void st_bf16x4(unsigned char *base, uint32_t off, float a, float b, float c,
                                          float d) {
  *reinterpret_cast<uint2 *>(base + off) = make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}

// ---------------------------------------------------------------------------
// M = (I + N)^{-1} for strictly lower N (fp32, row stride LDF), 64 x 64, by
// 16 x 16 blocks, 256 threads: diagonal blocks by forward substitution (one
// column per thread), then the block diagonals d = 1, 2, 3:
//   M_IJ = -M_II sum_{K=J}^{I-1} N_IK M_KJ,
// two passes per diagonal (the inner sum into Xs, then the product with
// M_II), each output block in 2 x 2 register tiles.
// Every entry on or below the diagonal is written; the strictly upper 16x16
// blocks are zeroed (the diagonal blocks carry their own zeros).
// ---------------------------------------------------------------------------
constexpr int kLdf = 65;
__device__ __forceinline__ void inverse64(float *Mf, const float *Nf, float (*Xs)[16][16]) {
  const int tid = threadIdx.x;
  if (tid < 64) {
    const int bI = tid >> 4, j = tid & 15, o = 16 * bI;
    float xc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float s = 0.f;
#pragma unroll
      for (int kk = 0; kk < i; ++kk) s += Nf[(o + i) * kLdf + o + kk] * xc[kk];
      xc[i] = (i == j) ? 1.f : (i < j ? 0.f : -s);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Mf[(o + i) * kLdf + o + j] = xc[i];
  } else {
    // strictly upper blocks (I < J): 6 blocks of 256
    for (int e = tid - 64; e < 6 * 256; e += 192) {
      const int b = e >> 8, aa = (e >> 4) & 15, bb = e & 15;
      const int I = b < 3 ? 0 : (b < 5 ? 1 : 2);
      const int J = b < 3 ? b + 1 : (b < 5 ? b - 1 : 3);
      Mf[(16 * I + aa) * kLdf + 16 * J + bb] = 0.f;
    }
  }
  __syncthreads();
  // each thread a 2 x 2 block of outputs (rows aa, aa + 1, columns bb, bb + 1):
  // two loads of N and two of M feed four products
#pragma unroll 1
  for (int d = 1; d < 4; ++d) {
    const int nb = 4 - d;
    for (int e = tid; e < nb * 64; e += 256) {
      const int J = e >> 6, I = J + d, aa = ((e >> 3) & 7) * 2, bb = (e & 7) * 2;
      float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
      for (int K = J; K < I; ++K) {
        const float *n0 = Nf + (16 * I + aa) * kLdf + 16 * K, *n1 = n0 + kLdf;
        const float *mc = Mf + (16 * K) * kLdf + 16 * J + bb;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float a0 = n0[t], a1 = n1[t], b0 = mc[t * kLdf], b1 = mc[t * kLdf + 1];
          s00 += a0 * b0; s01 += a0 * b1; s10 += a1 * b0; s11 += a1 * b1;
        }
      }
      Xs[J][aa][bb] = s00; Xs[J][aa][bb + 1] = s01;
      Xs[J][aa + 1][bb] = s10; Xs[J][aa + 1][bb + 1] = s11;
    }
    __syncthreads();
    for (int e = tid; e < nb * 64; e += 256) {
      const int J = e >> 6, I = J + d, aa = ((e >> 3) & 7) * 2, bb = (e & 7) * 2;
      const float *m0 = Mf + (16 * I + aa) * kLdf + 16 * I, *m1 = m0 + kLdf;
      float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float a0 = m0[t], a1 = m1[t], b0 = Xs[J][t][bb], b1 = Xs[J][t][bb + 1];
        s00 += a0 * b0; s01 += a0 * b1; s10 += a1 * b0; s11 += a1 * b1;
      }
      float *o0 = Mf + (16 * I + aa) * kLdf + 16 * J + bb, *o1 = o0 + kLdf;
      o0[0] = -s00; o0[1] = -s01; o1[0] = -s10; o1[1] = -s11;
    }
    __syncthreads();
  }
}

}  // namespace tc
}  // namespace ckda
