// TMA tensor-map encoding shared by the kernels' host launchers.
#include <cstdio>
#include <mutex>

#include "internal.cuh"

namespace fp {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver function, looked up once through the runtime (no link against libcuda).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

bool encode_tiled(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled lookup", 0, "driver entry point not found");
    return false;
  }
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, type, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[200];
    int n = snprintf(buf, sizeof(buf), "rank %d dims", rank);
    for (int d = 0; d < rank && n > 0 && n < (int)sizeof(buf); ++d)
      n += snprintf(buf + n, sizeof(buf) - n, " %llu", (unsigned long long)dims[d]);
    for (int d = 0; d < rank && n > 0 && n < (int)sizeof(buf); ++d)
      n += snprintf(buf + n, sizeof(buf) - n, "%s%u", d ? "," : " box ", box[d]);
    set_last_error("cuTensorMapEncodeTiled", (int)r, buf);
    return false;
  }
  return true;
}

}  // namespace fp
