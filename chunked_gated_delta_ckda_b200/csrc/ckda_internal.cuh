// ckda_internal.cuh -- shared definitions of the CKDA CUDA library (not part
// of the ABI): parameter blocks, workspace layout, I/O conversions, chunk map.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>

#include "ckda.h"

namespace ckda {

constexpr int C = CKDA_CHUNK;  // chunk length (tokens)

// --------------------------------------------------------------------------
// I/O element conversions
// --------------------------------------------------------------------------
__device__ __forceinline__ float ld_io(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_io(const __nv_bfloat16 *p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_io(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_io(__nv_bfloat16 *p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// --------------------------------------------------------------------------
// Device status word (first bytes of every workspace)
// --------------------------------------------------------------------------
struct DevStatus {
  uint32_t flags;    // bit 0: bounded wait gave up; bit 1: malformed cu_seqlens
  uint32_t detail;   // first failing site / document index
  int32_t n_chunks;  // packed call: number of chunks actually present
  int32_t pad[61];
};
static_assert(sizeof(DevStatus) == 256, "status block is 256 bytes");
constexpr uint32_t kFlagTimeout = 1u;
constexpr uint32_t kFlagBadSeqlens = 2u;

// --------------------------------------------------------------------------
// Chunk map: global chunk id -> (sequence, first token, length)
//   batched: sequence b = cid / NC, chunk j = cid % NC (no table)
//   packed : table built on the device from cu_seqlens
// --------------------------------------------------------------------------
struct ChunkMap {
  const int32_t *table;      // packed: [n_chunks_bound][4] = seq, tok0, len, j
  const int32_t *seq_first;  // packed: [N+1] first chunk id of each sequence
  const DevStatus *status;   // packed: n_chunks, flags
  int T;                     // batched: tokens per sequence
  int NC;                    // batched: chunks per sequence
  int n_seq;                 // B (batched) or N (packed)
  int n_chunks_bound;        // grid bound on chunk ids

  __device__ __forceinline__ bool packed() const { return table != nullptr; }
  __device__ __forceinline__ int n_chunks() const {
    return packed() ? status->n_chunks : n_seq * NC;
  }
  __device__ __forceinline__ void info(int cid, int &seq, int64_t &tok0, int &len,
                                       int &j) const {
    if (packed()) {
      const int32_t *e = table + 4 * (size_t)cid;
      seq = e[0];
      tok0 = e[1];
      len = e[2];
      j = e[3];
    } else {
      seq = cid / NC;
      j = cid % NC;
      tok0 = (int64_t)seq * T + (int64_t)j * C;
      int rem = T - j * C;
      len = rem < C ? rem : C;
    }
  }
  // slot of a per-(chunk, head) state in a chunk-state buffer: [B][H][NC]
  // (batched: the layout callers see) or [chunk id][H] (packed)
  __device__ __forceinline__ size_t state_slot(int seq, int h, int H, int j, int cid) const {
    return packed() ? (size_t)cid * H + h : ((size_t)seq * H + h) * NC + j;
  }
  __device__ __forceinline__ int seq_chunks(int seq, int &first) const {
    if (packed()) {
      first = seq_first[seq];
      return seq_first[seq + 1] - first;
    }
    first = seq * NC;
    return NC;
  }
};

// --------------------------------------------------------------------------
// Workspace layout
// --------------------------------------------------------------------------
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct WsLayout {
  size_t status = 0;     // DevStatus
  size_t table = 0;      // packed chunk table
  size_t seq_first = 0;  // packed per-sequence first chunk
  size_t intra = 0;      // per (chunk, head): W, U0, QG, Khat, Aq, d  (fp32)
  size_t states = 0;     // bwd: chunk-start states  [B,H,NC,dk,dv]
  size_t dsend = 0;      // bwd: dL/dS at each chunk end [B,H,NC,dk,dv]
  size_t du = 0;         // bwd: dL/dU per (chunk, head) [C, dv]
  size_t fscratch = 0;   // per-CTA scratch of the intra-chunk kernel
  size_t scratch = 0;    // bwd: per-CTA scratch of the per-chunk gradient kernel
  size_t seg = 0;        // segment maps, their scan (long sequences; tensor-core path)
  size_t total = 0;
  size_t intra_stride = 0;  // floats per (chunk, head)
  int n_chunks_bound = 0;
  int bwd_ctas = 0;
};

// floats of one (chunk, head) intra record
__host__ __device__ inline size_t intra_floats(int dk, int dv) {
  return (size_t)C * dk * 3 + (size_t)C * dv + (size_t)C * C + dk;
}
struct IntraPtrs {
  float *W, *U0, *QG, *Khat, *Aq, *d;
};
__host__ __device__ inline IntraPtrs intra_ptrs(float *base, int dk, int dv) {
  IntraPtrs p;
  p.W = base;
  p.QG = p.W + C * dk;
  p.Khat = p.QG + C * dk;
  p.U0 = p.Khat + C * dk;
  p.Aq = p.U0 + C * dv;
  p.d = p.Aq + C * C;
  return p;
}

// floats of the backward per-CTA scratch
__host__ __device__ inline size_t bwd_scratch_floats(int dk, int dv) {
  return (size_t)C * dk * 21 + (size_t)C * dv * 6 + 2 * dk;
}
constexpr int kBwdCtas = 296;  // persistent CTAs of the per-chunk gradient kernel

WsLayout ws_layout(int op, int B, int T, int H, int dk, int dv, int N);

// --------------------------------------------------------------------------
// Host-side argument checks shared by the entry points (run before anything
// is enqueued)
// --------------------------------------------------------------------------
inline bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sizes, dtype code and head dimensions
inline int check_common(int B, int T, int H, int dk, int dv, int io_dtype) {
  if (B < 0 || T < 0 || H < 1) return CKDA_ERR_INVALID_ARG;
  if (io_dtype != CKDA_F32 && io_dtype != CKDA_BF16) return CKDA_ERR_INVALID_ARG;
  if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return CKDA_ERR_UNSUPPORTED;
  // index arithmetic is 64-bit; chunk ids and token offsets are 32-bit
  if ((int64_t)B * T > INT32_MAX / 2) return CKDA_ERR_UNSUPPORTED;
  return CKDA_OK;
}

// sequences (B or N) and heads index grid dimensions limited to 65535
inline int check_grid(int B, int H, int N) {
  if (B > 65535 || H > 65535 || N > 65535) return CKDA_ERR_UNSUPPORTED;
  return CKDA_OK;
}

// required pointers non-null and 16-byte aligned; optional ones aligned when given
inline int check_ptrs(std::initializer_list<const void *> required,
                      std::initializer_list<const void *> optional) {
  for (const void *p : required)
    if (!p) return CKDA_ERR_INVALID_ARG;
  for (const void *p : required)
    if (!a16(p)) return CKDA_ERR_ALIGNMENT;
  for (const void *p : optional)
    if (p && !a16(p)) return CKDA_ERR_ALIGNMENT;
  return CKDA_OK;
}

// --------------------------------------------------------------------------
// Parameter blocks
// --------------------------------------------------------------------------
struct FwdArgs {
  int B, T, H, dk, dv;
  const void *q, *k, *v, *beta;
  const float *g;
  const int8_t *sign;
  const float *S0;
  void *o;
  float *ST;
  float *chunk_states;  // batched only
  ChunkMap map;
  float *intra;
  DevStatus *status;
};

struct BwdArgs {
  int B, T, H, dk, dv;
  const void *q, *k, *v, *beta, *dO;
  const float *g;
  const int8_t *sign;
  const float *S0, *dST;
  const float *states;  // chunk-start states [B,H,NC,dk,dv]
  void *dq, *dkg, *dvg, *dbeta;  // gradients of q, k, v, beta
  float *dg, *dS0;
  ChunkMap map;
  float *intra, *dsend, *du, *scratch;
  DevStatus *status;
};

// Optional per-kernel timing (ckda_profile_enable): records a CUDA event pair
// on the launch stream around the launches made while the scope lives.
class ProfScope {
 public:
  ProfScope(const char *name, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope &) = delete;
  ProfScope &operator=(const ProfScope &) = delete;

 private:
  int idx_;
  cudaStream_t s_;
};

// launchers (return cudaError_t of the launches)
cudaError_t build_chunk_table(const int32_t *cu, int N, int total_T, int max_seqlen,
                              int n_chunks_bound, int32_t *table, int32_t *seq_first,
                              DevStatus *status, cudaStream_t s);
size_t v1_fwd_scratch_floats(int dk, int dv);
cudaError_t v1_intra(const FwdArgs &a, bool bf16, float *scratch, cudaStream_t s);
size_t v1_fwd_scratch_floats_per_cta(int dk, int dv);
cudaError_t v1_intra_on_ctas(const FwdArgs &a, bool bf16, float *scratch, int ctas,
                             cudaStream_t s);
cudaError_t v1_state_fwd(const FwdArgs &a, bool bf16, bool write_o, float *states_out,
                         cudaStream_t s);
cudaError_t v1_backward(const BwdArgs &a, bool bf16, cudaStream_t s);
size_t tc_fwd_fallback_floats(int ctas);
int tc_intra_ctas();
size_t tc_record_bytes();
cudaError_t tc_forward(const FwdArgs &f, unsigned char *recs, float *fb, bool write_o,
                       float *states_out, cudaStream_t s, bool state_pass = true,
                       bool intra_pass = true, bool state_tiles = false, float *seg_ws = nullptr);
int tc_seg_count(int B, int H, int NC);  // segments per sequence of the long-sequence scan (0: off)
size_t tc_seg_ws_bytes();                // workspace of the long-sequence scan
int tc_seg_count_bwd(int B, int H, int NC);  // segments of the long-sequence backward (0: off)
// the segments' maps M_g as rows [c][j] (and their offsets) from the records
cudaError_t tc_seg_maps_rows(const FwdArgs &f, const unsigned char *recs, int G, float *seg_M, float *seg_b,
                             cudaStream_t s);
// adjoint states at each segment's end, from the last segment down:
// end(G-1) = X0 (or 0), end(g-1) = M_g^T end(g) + e_g
cudaError_t tc_seg_scan_reverse(const FwdArgs &f, int G, const float *seg_M, const float *seg_e, const float *X0,
                                float *seg_ends, cudaStream_t s);
// bf16 chunk-start state tiles of the records from fp32 chunk states [B,H,NC,128,128]
cudaError_t tc_state_tiles(const float *chunk_states, unsigned char *recs, int B, int H, int NC,
                           cudaStream_t s);
cudaError_t tc_backward(const BwdArgs &b, const unsigned char *recs, unsigned char *dS_tiles,
                        unsigned char *dU_tiles, float *fb, cudaStream_t s, float *seg_ws = nullptr);
cudaError_t decode_step(int N, int H, int dk, int dv, bool bf16, const void *q,
                        const void *k, const void *v, const float *g, const int8_t *sign,
                        const void *beta, float *state, void *o, cudaStream_t s);
cudaError_t decode_multi(int N, int K, int H, int dk, int dv, bool bf16, const void *q, const void *k,
                         const void *v, const float *g, const int8_t *sign, const void *beta,
                         const int32_t *n_tokens, const int32_t *slots, int n_slots, float *state,
                         bool write_state, void *o, cudaStream_t s);

// token-mixer prologue (forward, or backward when `backward`)
struct PrologueLaunch {
  int B, T, H, dk, dv;
  bool bf16, backward;
  float g_floor;
  const void *xq, *xk, *xv, *b;
  const float *wq, *wk, *wv, *a;
  void *q, *k, *v, *beta;
  float *g;
  int8_t *sign;
  const void *dq, *dk_in, *dv_in, *dbeta;
  const float *dg;
  void *dxq, *dxk, *dxv, *db;
  float *dwq, *dwk, *dwv, *da;
  const int32_t *cu;  // packed documents (null: batch rows)
  int N;
};
cudaError_t prologue(const PrologueLaunch &p, cudaStream_t s);

}  // namespace ckda
