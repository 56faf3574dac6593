// kl_noalloc.cu -- kl_ln_modulate_quantize_nvfp4_static: the fused
// LayerNorm + adaLN + NVFP4 encoder for callers that cannot hand this library
// any device memory for scratch.
//
// Who needs it: a host that owns and plans all device memory up front (for
// example an inference server that reserves the whole device pool at start-up
// and forbids later allocations, or a plugin interface that passes only
// input/output buffers) cannot call cudaMalloc for us and has no workspace to
// lend.  This entry point keeps its scratch -- one amax word and the per-row
// LayerNorm statistics -- in a fixed array compiled into the library.
//
// Cost: every GPU that loads the library keeps KL_STATIC_SCRATCH_BYTES of
// device memory for that array until the process exits.
#include <mutex>

#include "../../include/klein.h"
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

constexpr int64_t kStaticScratchRows = KL_STATIC_SCRATCH_MAX_ROWS;
constexpr size_t kStaticScratchBytes = 256 + (size_t)kStaticScratchRows * sizeof(float2);

// The scratch itself.  In host code this name is only a host-side handle for
// the device symbol, never a device address: the address is looked up with
// cudaGetSymbolAddress once per device (below) and passed to the kernels.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's device address belongs to the device's current context: a
// cudaDeviceReset (or any teardown of the primary context) makes a new
// context in which the array lives elsewhere.  So the address is cached per
// device together with the id of the context it was resolved in, and
// resolved again when that id changes.
struct StaticScratchSlot {
  unsigned long long ctx_id;
  void* ptr;
};
static StaticScratchSlot g_static_scratch_slot[kMaxDevices];
static std::mutex g_static_scratch_mu;

typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);

// id of the calling thread's current context (0 if there is none yet)
static unsigned long long current_ctx_id() {
  static PFN_ctx_get_current get_current = nullptr;
  static PFN_ctx_get_id get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctx_get_current>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctx_get_id>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Set-up on the current device (first call, and again after the device's
// context was replaced): resolve the array's device address with the device
// current.  cudaGetSymbolAddress also makes the primary context current if
// no context is yet, so the context id is read after it.
static kl_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(g_last_err, sizeof(g_last_err), "kl_ln_modulate_quantize_nvfp4_static: device index %d >= %d", dev,
             kMaxDevices);
    return KL_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  StaticScratchSlot& slot = g_static_scratch_slot[dev];
  const unsigned long long id = current_ctx_id();
  if (!slot.ptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    slot.ptr = p;
    slot.ctx_id = current_ctx_id();
  }
  *out = slot.ptr;
  return KL_OK;
}

}  // namespace kl

extern "C" kl_status kl_ln_modulate_quantize_nvfp4_static(const void* x, int64_t rows, int64_t cols,
                                                          const void* shift, const void* scale, void* codes,
                                                          void* scales, float* global_scale, void* m_out,
                                                          void* stream) {
  using namespace kl;
  if (!x || !shift || !scale || !codes || !scales || !global_scale) return KL_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 || cols > 8192) return KL_ERR_UNSUPPORTED_SHAPE;
  if (rows > kStaticScratchRows) {
    snprintf(g_last_err, sizeof(g_last_err),
             "kl_ln_modulate_quantize_nvfp4_static: %lld rows exceed the static scratch capacity of %lld rows",
             (long long)rows, (long long)kStaticScratchRows);
    return KL_ERR_WORKSPACE;
  }
  if (!aligned(x, 16) || !aligned(shift, 16) || !aligned(scale, 16) || !aligned(codes, 8) ||
      (m_out && !aligned(m_out, 16)))
    return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  void* base = nullptr;
  if ((st = static_scratch(&base)) != KL_OK) return st;
  uint8_t* ws = reinterpret_cast<uint8_t*>(base);
  // the amax word is zeroed on the stream inside the launcher before use; the
  // statistics rows are fully rewritten before they are read
  cudaError_t e = launch_ln_modulate_quantize(x, rows, cols, shift, scale, codes, scales, global_scale, m_out,
                                              reinterpret_cast<float2*>(ws + 256), reinterpret_cast<float*>(ws),
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}
