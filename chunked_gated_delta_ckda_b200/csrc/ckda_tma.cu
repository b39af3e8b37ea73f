// ckda_tma.cu -- host side of the tensor-memory-accelerator (TMA) loads:
// encodes the tensor maps of the per-token row tensors.  The driver's
// encoder is reached through the runtime's entry-point query, so the library
// needs no link-time dependency on the driver library.
#include <cudaTypedefs.h>

#include <mutex>

#include "ckda_tc.cuh"

namespace ckda {
namespace tc {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [ntok][H][128] elements of `esize` bytes; box = box_c channels x 1 head x 64 tokens
cudaError_t encode(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int64_t ntok, int H,
                   int box_c, bool swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)ntok};
  const cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize};
  const cuuint32_t box[3] = {(cuuint32_t)box_c, 1u, 64u};
  const cuuint32_t estride[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t make_row_maps(RowMaps &m, const void *q, const void *k, const void *v, const void *dO,
                          const float *g, const int8_t *sign, int64_t ntok, int H) {
  m = RowMaps{};
  if (ntok <= 0) return cudaSuccess;  // nothing will be loaded
  cudaError_t e;
  if ((e = encode(&m.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ntok, H, 64, true)) != cudaSuccess) return e;
  if ((e = encode(&m.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ntok, H, 64, true)) != cudaSuccess) return e;
  if ((e = encode(&m.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ntok, H, 64, true)) != cudaSuccess) return e;
  if (dO && (e = encode(&m.dO, dO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ntok, H, 64, true)) != cudaSuccess)
    return e;
  if ((e = encode(&m.g, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ntok, H, D, false)) != cudaSuccess) return e;
  if (!sign) return cudaSuccess;  // all +1: no sign rows to load
  return encode(&m.sign, sign, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ntok, H, D, false);
}

}  // namespace tc
}  // namespace ckda
