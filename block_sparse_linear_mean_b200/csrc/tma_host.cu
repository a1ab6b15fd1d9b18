// Host-side TMA descriptor encoding (driver entry point looked up through the
// runtime, so the library never links the driver directly), and the SM count
// that sizes the persistent grids.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.h"

namespace sla {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool tma_available() { return encode_fn() != nullptr; }

// Unique id of the calling thread's current CUDA context (never reused in a
// process, unlike the context handle), through the driver entry points.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    looked_up = true;
  }
  CUcontext c = nullptr;
  if (!get_ctx || !get_id || get_ctx(&c) != CUDA_SUCCESS || !c) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

// SMs of the current device (persistent kernels launch one CTA per SM, or a
// fixed number per SM); 148 if the query fails.
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// Tensor of rank 2 or 3 (dims[0] innermost, strides in bytes for dims
// 1..rank-1), 128-byte swizzle, out-of-range elements read as zero.
static bool encode_map(CUtensorMapDataType type, void* map, const void* ptr, int rank,
                       const uint64_t* dims, const uint64_t* strides, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn || rank < 2 || rank > 3) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides[i];
  CUresult r = fn(static_cast<CUtensorMap*>(map), type, rank,
                  const_cast<void*>(ptr), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_bf16_map(void* map, const void* ptr, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box) {
  return encode_map(CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, map, ptr, rank, dims, strides, box);
}

// Same for an fp32 tensor.
bool encode_f32_map(void* map, const void* ptr, int rank, const uint64_t* dims,
                    const uint64_t* strides, const uint32_t* box) {
  return encode_map(CU_TENSOR_MAP_DATA_TYPE_FLOAT32, map, ptr, rank, dims, strides, box);
}

}  // namespace sla
