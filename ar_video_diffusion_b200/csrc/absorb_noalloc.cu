// ispa_absorb_solve_noalloc: the absorb solve with its scratch memory held in
// a fixed device array that the library owns, for callers that cannot
// allocate device memory themselves.
//
// Who needs it: code that runs where cudaMalloc is off limits or unavailable
// -- inside a host callback or a custom allocator hook, in a process whose
// memory is budgeted up front by a serving runtime, or in a plugin that is
// handed device pointers for its inputs and outputs but no allocator.  The
// caller still supplies G, R, W and the outputs; only the working matrices of
// the solve come from the array below.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library reserves kNoAllocBytes of device memory for it until the process
// exits.  Its size bounds d_model at kNoAllocMaxD.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"

namespace ispa {

size_t absorb_compact_workspace_bytes(int64_t D);
ispa_status_t absorb_solve_compact(const float* G, const float* R, const void* W, ispa_dtype_t w_dt, int64_t D,
                                   double lam_abs, double lam_rel, float* dW, void* w_new, void* workspace,
                                   int32_t* status, cudaStream_t st);

constexpr int64_t kNoAllocMaxD = 2048;
constexpr size_t kNoAllocBytes = (size_t)(4 * kNoAllocMaxD * kNoAllocMaxD + 256 * kNoAllocMaxD + 256);

// Scratch of the no-allocation solve.  In host code this name is only a
// host-side stand-in: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_absorb_scratch[kNoAllocBytes];

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::mutex g_mu;
// (context id, device address of g_absorb_scratch in that context).  The id
// that cuCtxGetId returns is unique for the life of the process, so a context
// that replaced a destroyed one (after cudaDeviceReset, say) never finds the
// address the old context had.
std::vector<std::pair<unsigned long long, void*>> g_scratch_by_ctx;

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context; 0 when there is none yet.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  *id = 0;
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  return !ctx || get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_absorb_scratch in the current device's context.  The
// lookup runs once per context, with that context current (on the first call
// a context sees); later calls find the cached address.
ispa_status_t scratch_for_current_device(void** out) {
  unsigned long long id = 0;
  if (!current_context_id(&id)) {
    set_last_error("cuCtxGetCurrent / cuCtxGetId are not available from the driver");
    return ISPA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (id != 0) {
    for (const auto& e : g_scratch_by_ctx)
      if (e.first == id) {
        *out = e.second;
        return ISPA_OK;
      }
  }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_absorb_scratch);
  if (e != cudaSuccess || !p) {
    set_last_error("cudaGetSymbolAddress of the absorb scratch failed: %s", cudaGetErrorString(e));
    return ISPA_ERR_CUDA;
  }
  if (id == 0 && !current_context_id(&id)) {  // the lookup made the runtime's context current
    set_last_error("cuCtxGetId failed");
    return ISPA_ERR_CUDA;
  }
  if (id != 0) g_scratch_by_ctx.emplace_back(id, p);
  *out = p;
  return ISPA_OK;
}
}  // namespace

}  // namespace ispa

extern "C" ispa_status_t ispa_absorb_solve_noalloc(const float* G, const float* R, const void* W, ispa_dtype_t w_dt,
                                                   int64_t d_model, double lambda_abs, double lambda_rel,
                                                   float* delta_w, void* w_new, int32_t* dev_status, void* stream) {
  using namespace ispa;
  if (w_dt != ISPA_DT_BF16 && w_dt != ISPA_DT_F32) return unsupported("unknown dtype %d", (int)w_dt);
  if (!G || !R || !W || !delta_w) return invalid("required pointer is NULL");
  if (d_model <= 0 || d_model % 64) return unsupported("d_model must be a positive multiple of 64");
  if (d_model > kNoAllocMaxD)
    return unsupported("ispa_absorb_solve_noalloc supports d_model <= %lld (got %lld); use ispa_absorb_solve "
                       "with a caller-provided workspace",
                       (long long)kNoAllocMaxD, (long long)d_model);
  if (!(lambda_abs >= 0.0) || !(lambda_rel >= 0.0) || !std::isfinite(lambda_abs) || !std::isfinite(lambda_rel))
    return invalid("lambda_abs and lambda_rel must be finite and >= 0");
  for (const void* p : {(const void*)G, (const void*)R, W, (const void*)delta_w, (const void*)w_new})
    if (p && !aligned16(p)) return invalid("matrices must be 16-byte aligned");
  if (absorb_compact_workspace_bytes(d_model) > kNoAllocBytes) return unsupported("scratch too small for d_model");
  void* scratch = nullptr;
  ispa_status_t st = scratch_for_current_device(&scratch);
  if (st != ISPA_OK) return st;
  // The compact form of the solve (working matrices 4 d^2 + 256 d + 256
  // bytes) keeps the array small.  Every working matrix of it is written
  // before it is read, so the stale contents left by an earlier call need no
  // clearing.
  return absorb_solve_compact(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new, scratch, dev_status,
                              static_cast<cudaStream_t>(stream));
}
