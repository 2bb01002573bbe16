// Host-side helpers: error strings, launch checks, TMA descriptor encoding
// through the driver entry point (no link-time dependency on libcuda).
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"

namespace ispa {

static thread_local char g_last_error[512] = "";

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

ispa_status_t invalid(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return ISPA_ERR_INVALID_ARG;
}

ispa_status_t unsupported(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return ISPA_ERR_UNSUPPORTED;
}

ispa_status_t check_launch(const char* kernel_name) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("launch of %s failed: %s", kernel_name, cudaGetErrorString(e));
    return ISPA_ERR_CUDA;
  }
  return ISPA_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_map_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                        uint32_t box_inner, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled failed (%d): inner=%llu rows=%llu row_bytes=%llu box=%ux%u", (int)r,
                   (unsigned long long)inner, (unsigned long long)rows, (unsigned long long)row_bytes, box_inner,
                   box_rows);
    return false;
  }
  return true;
}

bool encode_map_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled (8-bit) failed (%d): inner=%llu rows=%llu row_bytes=%llu box=%ux%u",
                   (int)r, (unsigned long long)inner, (unsigned long long)rows, (unsigned long long)row_bytes,
                   box_inner, box_rows);
    return false;
  }
  return true;
}

bool encode_map_out_2d(CUtensorMap* map, const void* base, bool f32, uint64_t inner, uint64_t rows,
                       uint64_t row_bytes) {
  auto fn = get_encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled (output) failed (%d): inner=%llu rows=%llu row_bytes=%llu", (int)r,
                   (unsigned long long)inner, (unsigned long long)rows, (unsigned long long)row_bytes);
    return false;
  }
  return true;
}

ispa_status_t set_smem(const void* kernel, int bytes) {
  // The attribute is per device; set it once per (kernel, device) so later
  // calls (including calls made while a stream is being captured) skip it.
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kernel, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return ISPA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(%d bytes of shared memory): %s", bytes, cudaGetErrorString(e));
    return ISPA_ERR_CUDA;
  }
  done[key] = bytes;
  return ISPA_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace ispa

extern "C" const char* ispa_last_error(void) { return ispa::g_last_error; }

extern "C" const char* ispa_status_string(ispa_status_t s) {
  switch (s) {
    case ISPA_OK: return "ok";
    case ISPA_ERR_INVALID_ARG: return "invalid argument";
    case ISPA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ISPA_ERR_CUDA: return "CUDA error";
    case ISPA_ERR_NOT_SPD: return "matrix not positive definite";
    case ISPA_ERR_TIMEOUT: return "device wait timed out";
    case ISPA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

extern "C" int32_t ispa_version(void) { return 100; }
