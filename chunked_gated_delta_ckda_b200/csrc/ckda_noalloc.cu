// ckda_noalloc.cu -- ckda_chunk_fwd_noalloc: the chunked forward run out of a
// fixed scratch area that the library itself owns, for callers that cannot
// allocate device memory.
//
// Who needs this: code that lives inside a host application which owns every
// device allocation (a fixed memory pool or its own allocator, with no way
// for a plug-in to obtain a workspace buffer), and code on latency-critical
// paths that must not call cudaMalloc because it can synchronise the device
// and fail at run time.  Such callers still pass their inputs and outputs;
// the scratch comes from the array below instead of a workspace argument.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library holds CKDA_NOALLOC_SCRATCH_BYTES of device memory for it until the
// process exits.  Host code cannot use the array's name as a device address
// (on the host it names a stand-in object), so the address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call made on that device; make that first call before any stream
// capture begins.  All calls share the one array and it keeps the previous
// call's contents: calls whose work overlaps on the GPU (different streams,
// or different host threads) race on it and must be serialised by the caller.
#include <mutex>

#include "ckda_internal.cuh"

namespace {

// The scratch itself.  Device code in this file could name it directly; the
// launches below receive its device address instead.
static __device__ __align__(256) unsigned char g_scratch[CKDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr int kNoAllocCtas = 16;  // persistent CTAs of the intra-chunk kernel here

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once).
int scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CKDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CKDA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return CKDA_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return CKDA_OK;
}

}  // namespace

using namespace ckda;

#define NOALLOC_TRY(expr)              \
  do {                                 \
    const int _rc = (expr);            \
    if (_rc != CKDA_OK) return _rc;    \
  } while (0)

extern "C" int ckda_chunk_fwd_noalloc(int B, int T, int H, int dk, int dv, int io_dtype,
                                      const void *q, const void *k, const void *v,
                                      const float *g, const int8_t *sign, const void *beta,
                                      const float *S0, void *o, float *ST,
                                      float *chunk_states, cudaStream_t stream) {
  // the same argument checks as ckda_chunk_fwd, before any size is derived
  NOALLOC_TRY(check_common(B, T, H, dk, dv, io_dtype));
  NOALLOC_TRY(check_grid(B, H, 0));
  if ((int64_t)B * T > 0) NOALLOC_TRY(check_ptrs({q, k, v, g, beta, o}, {sign, S0, ST, chunk_states}));
  else NOALLOC_TRY(check_ptrs({}, {sign, S0, ST, chunk_states}));
  // capacity: per-CTA intra scratch, one record per (chunk, head).  The kernels
  // this call runs have no bounded waits and no device-checked inputs, so it
  // keeps no device status block.
  const int NC = (T + C - 1) / C;
  const size_t slabs = align256(v1_fwd_scratch_floats_per_cta(dk, dv) * kNoAllocCtas * sizeof(float));
  const size_t records = align256((size_t)B * NC * H * intra_floats(dk, dv) * sizeof(float));
  if (slabs + records > (size_t)CKDA_NOALLOC_SCRATCH_BYTES) return CKDA_ERR_NOALLOC_CAPACITY;
  // the scratch address is that of the current device: the stream must belong to it
  int dev = -1, sdev = -2;
  if (cudaGetDevice(&dev) != cudaSuccess) return CKDA_ERR_CUDA;
  if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) return CKDA_ERR_INVALID_ARG;
  if (sdev != dev) return CKDA_ERR_INVALID_ARG;

  void *base = nullptr;
  NOALLOC_TRY(scratch_address(&base));
  char *w = static_cast<char *>(base);
  FwdArgs a{};
  a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.g = g; a.sign = sign;
  a.S0 = S0; a.o = o; a.ST = ST; a.chunk_states = chunk_states;
  a.map.T = T;
  a.map.NC = NC;
  a.map.n_seq = B;
  a.map.n_chunks_bound = B * NC;
  a.status = nullptr;
  float *slab = reinterpret_cast<float *>(w);
  a.intra = reinterpret_cast<float *>(w + slabs);
  const bool bf16 = io_dtype == CKDA_BF16;
  if (v1_intra_on_ctas(a, bf16, slab, kNoAllocCtas, stream) != cudaSuccess) return CKDA_ERR_CUDA;
  if (v1_state_fwd(a, bf16, true, chunk_states, stream) != cudaSuccess) return CKDA_ERR_CUDA;
  return CKDA_OK;
}
