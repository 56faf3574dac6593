// kl_api.cu -- the extern "C" boundary of libklein.so: argument validation,
// tensor-map construction, and the joint-block driver that orders the kernels
// on the caller's stream with a caller-provided workspace.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/klein.h"
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

static thread_local char g_last_err[256] = "";

static kl_status cuda_fail(cudaError_t e) {
  snprintf(g_last_err, sizeof(g_last_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return KL_ERR_CUDA;
}

constexpr int kMaxDevices = 64;
static int g_sms[kMaxDevices];
static int g_arch_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other

int device_sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return kNumSMs;
  if (g_sms[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = n > 0 ? n : kNumSMs;
  }
  return g_sms[dev];
}

static kl_status check_arch() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const bool cached = dev >= 0 && dev < kMaxDevices;  // devices past the cache are asked every time
  if (!cached || g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    const int ok = (major == 10 && minor == 0) ? 1 : -1;
    if (!cached) return ok == 1 ? KL_OK : KL_ERR_ARCH;
    g_arch_ok[dev] = ok;
  }
  return g_arch_ok[dev] == 1 ? KL_OK : KL_ERR_ARCH;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = swizzle_bytes == 64    ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : swizzle_bytes == 0   ? CU_TENSOR_MAP_SWIZZLE_NONE
                                                        : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return false;
  }
  return true;
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                  const uint64_t strides_bytes[2], const uint32_t box[3]) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled (3D) failed (%d)", (int)r);
    return false;
  }
  return true;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
static inline int64_t pad128(int64_t r) { return (r + 127) / 128 * 128; }
static inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace kl

using namespace kl;

extern "C" {

const char* kl_status_string(kl_status s) {
  switch (s) {
    case KL_OK: return "KL_OK";
    case KL_ERR_INVALID_ARG: return "KL_ERR_INVALID_ARG";
    case KL_ERR_UNSUPPORTED_SHAPE: return "KL_ERR_UNSUPPORTED_SHAPE";
    case KL_ERR_MISALIGNED: return "KL_ERR_MISALIGNED";
    case KL_ERR_WORKSPACE: return "KL_ERR_WORKSPACE";
    case KL_ERR_CUDA: return "KL_ERR_CUDA";
    case KL_ERR_DEVICE_TIMEOUT: return "KL_ERR_DEVICE_TIMEOUT";
    case KL_ERR_ARCH: return "KL_ERR_ARCH";
    case KL_ERR_NONFINITE: return "KL_ERR_NONFINITE";
    default: return "KL_ERR_UNKNOWN";
  }
}

const char* kl_last_cuda_error(void) { return g_last_err; }

int kl_version(void) { return 100; }

kl_status kl_device_status(int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int w = 0;
  e = cudaMemcpyFromSymbol(&w, g_device_status, sizeof(w));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_device_status, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (w & KL_DEVERR_TIMEOUT) return KL_ERR_DEVICE_TIMEOUT;
  if (w & KL_DEVERR_NONFINITE) return KL_ERR_NONFINITE;
  return KL_OK;
}

size_t kl_nvfp4_scales_bytes(int64_t rows, int64_t cols, int layout) {
  if (rows < 0 || cols < 0) return 0;
  return (size_t)(layout == KL_SCALE_MMA ? pad128(rows) : rows) * (size_t)(cols / 16);
}

size_t kl_quantize_workspace_size(void) { return 256; }

kl_status kl_quantize_nvfp4(const void* x, int64_t rows, int64_t cols, void* codes, void* scales,
                            float* global_scale, int flags, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !codes || !scales || !global_scale) return KL_ERR_INVALID_ARG;
  if (flags & ~(KL_SCALE_MMA | KL_GLOBAL_SCALE_GIVEN | KL_ROWS_SWIGLU_INTERLEAVE | KL_AMAX_GIVEN))
    return KL_ERR_INVALID_ARG;
  if ((flags & KL_GLOBAL_SCALE_GIVEN) && (flags & KL_AMAX_GIVEN)) return KL_ERR_INVALID_ARG;
  if (rows < 1 || cols < 16 || cols % 16) return KL_ERR_UNSUPPORTED_SHAPE;
  if ((flags & KL_SCALE_MMA) && cols % 64) return KL_ERR_UNSUPPORTED_SHAPE;
  if ((flags & KL_ROWS_SWIGLU_INTERLEAVE) && rows % 128) return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(codes, 8) || !aligned(global_scale, 4)) return KL_ERR_MISALIGNED;
  const bool given = flags & KL_GLOBAL_SCALE_GIVEN;
  if (!given && (!workspace || ws_bytes < kl_quantize_workspace_size())) return KL_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 16)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* amax = reinterpret_cast<float*>(workspace);
  cudaError_t e = cudaSuccess;
  if (!given && !(flags & KL_AMAX_GIVEN)) e = launch_amax_bf16(x, rows * cols, amax, s);
  if (e == cudaSuccess) {
    const int mode = ((flags & KL_SCALE_MMA) ? 1 : 0) | (given ? 2 : 0) | ((flags & KL_ROWS_SWIGLU_INTERLEAVE) ? 4 : 0);
    e = launch_quantize(x, rows, cols, codes, scales, global_scale, amax, mode, s);
  }
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

kl_status kl_amax_bf16(const void* x, int64_t n, float* amax_out, void* stream) {
  if (!x || !amax_out) return KL_ERR_INVALID_ARG;
  if (n < 8 || n % 8) return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(amax_out, 4)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_amax_bf16(x, n, amax_out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

kl_status kl_ln_modulate_bf16(const void* x, int64_t rows, int64_t cols, const void* shift, const void* scale,
                              void* m_out, float* amax_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !shift || !scale || !m_out || !amax_out) return KL_ERR_INVALID_ARG;
  const int64_t w = cols / 256;  // the row kernel's widths
  if (rows < 1 || cols % 256 || !(w == 1 || w == 2 || w == 4 || w == 8 || w == 12 || w == 16))
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(shift, 16) || !aligned(scale, 16) || !aligned(m_out, 16) || !aligned(amax_out, 4))
    return KL_ERR_MISALIGNED;
  if (!workspace || ws_bytes < kl_ln_workspace_size(rows)) return KL_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_ln_modulate_m(x, rows, cols, shift, scale, m_out,
                                       reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(workspace) + 256),
                                       amax_out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

size_t kl_ln_workspace_size(int64_t rows) { return 256 + up256((size_t)(rows > 0 ? rows : 0) * sizeof(float2)); }

kl_status kl_ln_modulate_quantize_nvfp4(const void* x, int64_t rows, int64_t cols, const void* shift,
                                        const void* scale, void* codes, void* scales, float* global_scale,
                                        void* m_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !shift || !scale || !codes || !scales || !global_scale) return KL_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 || cols > 8192) return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(shift, 16) || !aligned(scale, 16) || !aligned(codes, 8) ||
      (m_out && !aligned(m_out, 16)))
    return KL_ERR_MISALIGNED;
  if (!workspace || ws_bytes < kl_ln_workspace_size(rows)) return KL_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  cudaError_t e = launch_ln_modulate_quantize(x, rows, cols, shift, scale, codes, scales, global_scale, m_out,
                                              reinterpret_cast<float2*>(ws + 256), reinterpret_cast<float*>(ws),
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

static kl_status check_operand(const kl_nvfp4_tensor* t) {
  if (!t || !t->codes || !t->scales || !t->global_scale) return KL_ERR_INVALID_ARG;
  if (!aligned(t->codes, 16) || !aligned(t->scales, 16) || !aligned(t->global_scale, 4)) return KL_ERR_MISALIGNED;
  return KL_OK;
}

kl_status kl_gemm_nvfp4_fused(const kl_nvfp4_tensor* A, const kl_nvfp4_tensor* W, int64_t M, int64_t N, int64_t K,
                              const kl_epilogue* epi, void* stream) {
  kl_status st = check_operand(A);
  if (st == KL_OK) st = check_operand(W);
  if (st != KL_OK) return st;
  if (!epi || !epi->out) return KL_ERR_INVALID_ARG;
  if (M < 1 || N < 128 || K < 64 || N % 128 || K % 64 || M > (int64_t)1 << 31 || N > (int64_t)1 << 30)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(epi->out, 16)) return KL_ERR_MISALIGNED;
  switch (epi->kind) {
    case KL_EPI_NONE:
      if (epi->out_dtype != KL_OUT_BF16 && epi->out_dtype != KL_OUT_F32) return KL_ERR_INVALID_ARG;
      break;
    case KL_EPI_QKV_ROPE:
      if (!epi->rope_cs || !epi->amax_out) return KL_ERR_INVALID_ARG;
      if (N % 384 || N / 3 / 128 > 64) return KL_ERR_UNSUPPORTED_SHAPE;
      if (!aligned(epi->rope_cs, 32)) return KL_ERR_MISALIGNED;  // 32-byte table loads
      break;
    case KL_EPI_SWIGLU:
      if (!epi->amax_out) return KL_ERR_INVALID_ARG;
      break;
    case KL_EPI_GATED_RESIDUAL:
      if (!epi->gate || !epi->residual) return KL_ERR_INVALID_ARG;
      if (!aligned(epi->gate, 16) || !aligned(epi->residual, 16)) return KL_ERR_MISALIGNED;
      break;
    default:
      return KL_ERR_INVALID_ARG;
  }
  if (epi->kind != KL_EPI_NONE && epi->out_dtype != KL_OUT_BF16) return KL_ERR_INVALID_ARG;
  st = check_arch();
  if (st != KL_OK) return st;
  GemmArgs g{};
  g.a_codes = A->codes;
  g.a_scales = A->scales;
  g.a_gs = A->global_scale;
  g.w_codes = W->codes;
  g.w_scales = W->scales;
  g.w_gs = W->global_scale;
  g.M = M;
  g.N = N;
  g.K = K;
  g.epi = epi->kind;
  g.out_f32 = epi->out_dtype == KL_OUT_F32;
  g.out = epi->out;
  g.rope_cs = epi->rope_cs;
  g.gate = epi->gate;
  g.residual = epi->residual;
  g.amax = epi->amax_out;
  static const int kTileBn[5] = {0, 128, 256, 384, 512};
  if (epi->tile < KL_TILE_AUTO || epi->tile > KL_TILE_2SM_256x256) return KL_ERR_INVALID_ARG;
  if ((epi->tile == KL_TILE_1CTA_128x256 || epi->tile == KL_TILE_2SM_256x256) && N % 256) return KL_ERR_UNSUPPORTED_SHAPE;
  g.force_bn = kTileBn[epi->tile];
  cudaError_t e = launch_gemm_nvfp4(g, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

int64_t kl_layout_tokens(const kl_token_layout* L) {
  if (!L || L->n_text < 0 || L->grid_h < 0 || L->grid_w < 0 || L->n_ref < 0) return -1;
  return L->n_text + (1 + L->n_ref) * L->grid_h * L->grid_w;
}

kl_status kl_rope_table(const kl_token_layout* L, float theta, float* cs_out, void* stream) {
  if (!L || !cs_out || !(theta > 1.0f)) return KL_ERR_INVALID_ARG;
  const int64_t T = kl_layout_tokens(L);
  if (T < 1) return KL_ERR_UNSUPPORTED_SHAPE;
  if ((L->grid_h == 0 || L->grid_w == 0) && T > L->n_text) return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(cs_out, 16)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_rope_table(L->n_text, L->grid_h, L->grid_w, L->n_ref, (double)theta, cs_out,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

kl_status kl_cast_fp8_per_head(const void* x, int64_t T, int64_t ncols, int64_t ld, const float* amax, void* out,
                               float* scales_out, void* stream) {
  if (!x || !amax || !out || !scales_out) return KL_ERR_INVALID_ARG;
  if (T < 1 || ncols < 128 || ncols % 128 || ncols / 128 > 256 || ld < ncols || ld % 16)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x, 16) || !aligned(out, 16)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_fp8_cast(x, T, ncols, ld, amax, out, scales_out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

kl_status kl_joint_attention_fp8(const void* q, const void* k, const void* v, int64_t ld, const float* sq,
                                 const float* sk, const float* sv, int64_t T, int64_t H, int64_t head_dim,
                                 int precision, void* out, float* amax_out, void* stream) {
  if (!q || !k || !v || !out) return KL_ERR_INVALID_ARG;
  if (precision != KL_ATTN_FP8 && precision != KL_ATTN_BF16) return KL_ERR_INVALID_ARG;
  if (precision == KL_ATTN_FP8 && (!sq || !sk || !sv)) return KL_ERR_INVALID_ARG;
  if (head_dim != 128 || T < 1 || H < 1 || H > 65535 || T > (int64_t)1 << 31 || ld < H * 128 || ld % 64)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  AttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.ld = ld;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.T = T;
  a.H = H;
  a.fp8 = precision == KL_ATTN_FP8;
  a.out = out;
  a.amax = amax_out;
  cudaError_t e = launch_attention(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

size_t kl_sol_list_ints(int64_t T, int64_t H, int precision) {
  if (T < 1 || H < 1 || (precision != KL_ATTN_FP8 && precision != KL_ATTN_BF16)) return 0;
  return sol_list_ints(T, H, precision == KL_ATTN_FP8);
}

size_t kl_sol_workspace_size(int64_t T, int64_t H, int precision) {
  if (T < 1 || H < 1 || (precision != KL_ATTN_FP8 && precision != KL_ATTN_BF16)) return 0;
  return sol_workspace_bytes(T, H, precision == KL_ATTN_FP8);
}

kl_status kl_sol_select(const void* q, const void* k, int64_t ld, const float* sq, const float* sk, int64_t T,
                        int64_t H, int precision, float tau, int* kv_list, void* workspace, size_t ws_bytes,
                        void* stream) {
  if (!q || !k || !kv_list) return KL_ERR_INVALID_ARG;
  if (precision != KL_ATTN_FP8 && precision != KL_ATTN_BF16) return KL_ERR_INVALID_ARG;
  if (precision == KL_ATTN_FP8 && (!sq || !sk)) return KL_ERR_INVALID_ARG;
  if (!(tau >= 0.f)) return KL_ERR_INVALID_ARG;  // also rejects NaN
  if (T < 1 || H < 1 || H > 65535 || ld < H * 128 || ld % 64 || (T + 127) / 128 > 48 * 1024)
    return KL_ERR_UNSUPPORTED_SHAPE;
  const bool fp8 = precision == KL_ATTN_FP8;
  if (!workspace || ws_bytes < sol_workspace_bytes(T, H, fp8)) return KL_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(kv_list, 4) || !aligned(workspace, 16)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_sol_select(q, k, ld, sq, sk, T, H, fp8, tau, kv_list, workspace,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

kl_status kl_joint_attention_sparse(const void* q, const void* k, const void* v, int64_t ld, const float* sq,
                                    const float* sk, const float* sv, int64_t T, int64_t H, int64_t head_dim,
                                    int precision, const int* kv_list, void* out, float* amax_out, void* stream) {
  if (!q || !k || !v || !out || !kv_list) return KL_ERR_INVALID_ARG;
  if (precision != KL_ATTN_FP8 && precision != KL_ATTN_BF16) return KL_ERR_INVALID_ARG;
  if (precision == KL_ATTN_FP8 && (!sq || !sk || !sv)) return KL_ERR_INVALID_ARG;
  if (head_dim != 128 || T < 1 || H < 1 || H > 65535 || T > (int64_t)1 << 31 || ld < H * 128 || ld % 64)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(kv_list, 4))
    return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  AttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.ld = ld;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.T = T;
  a.H = H;
  a.fp8 = precision == KL_ATTN_FP8;
  a.out = out;
  a.amax = amax_out;
  a.kv_list = kv_list;
  cudaError_t e = launch_attention(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

// ------------------------------------------------------------ VC-Attention
size_t kl_vc_workspace_size(int64_t T, int64_t H) {
  if (T < 1 || H < 1) return 0;
  return vc_select_workspace_bytes(T, H);
}

kl_status kl_vc_select(const void* q, const void* k, int64_t ld, int64_t T, int64_t H, float budget, int* list_fp8,
                       int* list_bf16, void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !list_fp8 || !list_bf16) return KL_ERR_INVALID_ARG;
  if (!(budget >= 0.f && budget <= 1.f)) return KL_ERR_INVALID_ARG;  // also rejects NaN
  if (T < 1 || H < 1 || H > 65535 || ld < H * 128 || ld % 64 || (T + 127) / 128 > 12 * 1024)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || ws_bytes < kl_vc_workspace_size(T, H)) return KL_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(list_fp8, 4) || !aligned(list_bf16, 4) ||
      !aligned(workspace, 256))
    return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  cudaError_t e = launch_vc_select(q, k, ld, T, H, budget, list_fp8, list_bf16, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

// [ml8: float2 T*H][ml16: float2 T*H][o16: fp32 T*H*128]
size_t kl_vc_attention_workspace_size(int64_t T, int64_t H) {
  if (T < 1 || H < 1) return 0;
  const int64_t nqb16 = (T + 127) / 128;
  return 2 * up256((size_t)T * H * sizeof(float2)) + up256((size_t)T * H * 128 * sizeof(float)) +
         up256((size_t)(H * nqb16 + 1) * sizeof(int));
}

static cudaError_t vc_attention(const AttnArgs& a8, const void* q, const void* k, const void* v, int64_t ld,
                                const int* list16, uint8_t* ws, cudaStream_t s) {
  const int64_t T = a8.T, H = a8.H;
  float2* ml8 = reinterpret_cast<float2*>(ws);
  float2* ml16 = reinterpret_cast<float2*>(ws + up256((size_t)T * H * sizeof(float2)));
  float* o16 = reinterpret_cast<float*>(ws + 2 * up256((size_t)T * H * sizeof(float2)));
  int* work = reinterpret_cast<int*>(ws + 2 * up256((size_t)T * H * sizeof(float2)) +
                                     up256((size_t)T * H * 128 * sizeof(float)));
  const int nqb16 = (int)((T + 127) / 128), nkt = (int)((T + 127) / 128);
  int* work_count = work + H * nqb16;
  AttnArgs f = a8;  // the FP8 pass over the tiles that are not repaired
  f.amax = nullptr;
  f.ml_out = ml8;
  f.empty_ok = 1;
  cudaError_t e = launch_attention(f, s);
  if (e != cudaSuccess) return e;
  // the BF16 pass over the repaired tiles runs only the (head, 128-row
  // block) items that have some: rows of the others keep l = 0 in ml16, which
  // the merge reads as "no repaired part"
  if ((e = cudaMemsetAsync(ml16, 0, (size_t)T * H * sizeof(float2), s)) != cudaSuccess) return e;
  if ((e = launch_list_work(list16, H, nqb16, nkt, work, work_count, s)) != cudaSuccess) return e;
  AttnArgs b{};
  b.q = q;
  b.k = k;
  b.v = v;
  b.ld = ld;
  b.T = T;
  b.H = H;
  b.fp8 = 0;
  b.out = a8.out;
  b.kv_list = list16;
  b.ml_out = ml16;
  b.o32 = o16;
  b.empty_ok = 1;
  b.work = work;
  b.work_count = work_count;
  if ((e = launch_attention(b, s)) != cudaSuccess) return e;
  if ((e = launch_vc_merge(a8.out, o16, ml8, ml16, T, H, s)) != cudaSuccess) return e;
  if (!a8.amax) return cudaSuccess;
  // max |O| of the merged output, max-accumulated into amax
  return launch_pdl(amax_bf16_kernel, dim3(grid_for(T * H * 16, 256)), dim3(256), 0, s,
                    reinterpret_cast<const uint4*>(a8.out), T * H * 16, a8.amax);
}

kl_status kl_joint_attention_vc(const void* q8, const void* k8, const void* v8, int64_t ld8, const float* sq,
                                const float* sk, const float* sv, const void* q, const void* k, const void* v,
                                int64_t ld, int64_t T, int64_t H, int64_t head_dim, const int* list_fp8,
                                const int* list_bf16, void* out, float* amax_out, void* workspace, size_t ws_bytes,
                                void* stream) {
  if (!q8 || !k8 || !v8 || !sq || !sk || !sv || !q || !k || !v || !list_fp8 || !list_bf16 || !out)
    return KL_ERR_INVALID_ARG;
  if (head_dim != 128 || T < 1 || H < 1 || H > 65535 || T > (int64_t)1 << 31 || ld8 < H * 128 || ld8 % 64 ||
      ld < H * 128 || ld % 64)
    return KL_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || ws_bytes < kl_vc_attention_workspace_size(T, H)) return KL_ERR_WORKSPACE;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(q, 16) || !aligned(k, 16) ||
      !aligned(v, 16) || !aligned(out, 16) || !aligned(list_fp8, 4) || !aligned(list_bf16, 4) ||
      !aligned(workspace, 256) || (amax_out && !aligned(amax_out, 4)))
    return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  AttnArgs a{};
  a.q = q8;
  a.k = k8;
  a.v = v8;
  a.ld = ld8;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.T = T;
  a.H = H;
  a.fp8 = 1;
  a.out = out;
  a.amax = amax_out;
  a.kv_list = list_fp8;
  cudaError_t e = vc_attention(a, q, k, v, ld, list_bf16, reinterpret_cast<uint8_t*>(workspace),
                               reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

// ------------------------------------------------------------ block driver
// Workspace layout (each piece 256-byte aligned):
//   words  : amax[0..3] (O at 1, h at 3), gs[4..7], qkv amax [3H], fp8 scales [3H],
//            LN1 and LN2 amax words [2 + 2]
//   stats  : float2 [T]                       LayerNorm mean / rstd
//   acodes : uint8 [T, D/2], ascales [Tp, D/16]   NVFP4 A operand (m1, then O, then m2)
//   qkv    : bf16 [T, 3D]
//   qkv8   : e4m3 [T, 3D]                     (FP8 attention only)
//   o      : bf16 [T, D]
//   x1     : bf16 [T, D]
//   h      : bf16 [T, F]
//   hcodes : uint8 [T, F/2], hscales [Tp, F/16]
struct BlockWs {
  float* words;
  float2* stats;
  uint8_t *acodes, *ascales, *qkv8, *hcodes, *hscales;
  uint16_t *qkv, *o, *x1, *h;
  void* sol_ws;   // Sol-Attention block means
  int* sol_list;  // Sol-Attention key-tile lists
  void* vc_ws;    // VC-Attention: shares and marks, the two tile lists, the partial results
  int *vc_list8, *vc_list16;
  uint8_t* vc_att;
  size_t total;
};
static BlockWs block_ws_layout(uint8_t* base, int64_t T, int64_t D, int64_t H, int64_t F, int prec) {
  BlockWs w{};
  const int64_t Tp = pad128(T);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += up256(bytes);
    return p;
  };
  w.words = reinterpret_cast<float*>(take((12 + 6 * (size_t)H) * sizeof(float)));
  w.stats = reinterpret_cast<float2*>(take((size_t)T * sizeof(float2)));
  w.acodes = take((size_t)T * D / 2);
  w.ascales = take((size_t)Tp * D / 16);
  w.qkv = reinterpret_cast<uint16_t*>(take((size_t)T * 3 * D * 2));
  w.qkv8 = prec == KL_ATTN_FP8 ? take((size_t)T * 3 * D) : nullptr;
  w.o = reinterpret_cast<uint16_t*>(take((size_t)T * D * 2));
  w.x1 = reinterpret_cast<uint16_t*>(take((size_t)T * D * 2));
  w.h = reinterpret_cast<uint16_t*>(take((size_t)T * F * 2));
  w.hcodes = take((size_t)T * F / 2);
  w.hscales = take((size_t)Tp * F / 16);
  w.sol_ws = take(sol_workspace_bytes(T, H, prec == KL_ATTN_FP8));
  w.sol_list = reinterpret_cast<int*>(take(sol_list_ints(T, H, prec == KL_ATTN_FP8) * sizeof(int)));
  if (prec == KL_ATTN_FP8) {
    w.vc_ws = take(vc_select_workspace_bytes(T, H));
    w.vc_list8 = reinterpret_cast<int*>(take(sol_list_ints(T, H, true) * sizeof(int)));
    w.vc_list16 = reinterpret_cast<int*>(take(sol_list_ints(T, H, false) * sizeof(int)));
    w.vc_att = take(kl_vc_attention_workspace_size(T, H));
  }
  w.total = off;
  return w;
}

size_t kl_block_workspace_size(int64_t T, int64_t D, int64_t H, int64_t F, int prec) {
  if (T < 1 || D < 1 || H < 1 || F < 1) return 0;
  return block_ws_layout(nullptr, T, D, H, F, prec).total;
}

kl_status kl_joint_block_forward(const kl_block_weights* w, const kl_block_io* io, void* workspace,
                                 size_t ws_bytes, void* stream) {
  if (!w || !io || !io->x || !io->rope_cs || !io->out) return KL_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!io->mod[i] || !aligned(io->mod[i], 16)) return io->mod[i] ? KL_ERR_MISALIGNED : KL_ERR_INVALID_ARG;
  const int64_t T = io->T, D = io->D, H = io->H, F = io->F;
  if (io->attn_precision != KL_ATTN_FP8 && io->attn_precision != KL_ATTN_BF16) return KL_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || H > 64 || D != 128 * H || F < 128 || F % 128 || D > 8192) return KL_ERR_UNSUPPORTED_SHAPE;
  if (io->out == io->x) return KL_ERR_INVALID_ARG;
  if (!(io->vc_budget >= 0.f && io->vc_budget <= 1.f)) return KL_ERR_INVALID_ARG;  // also rejects NaN
  if (io->vc_budget > 0.f && (io->attn_precision != KL_ATTN_FP8 || io->sol_tau > 0.f)) return KL_ERR_INVALID_ARG;
  kl_status st = KL_OK;
  const kl_nvfp4_tensor* ops[4] = {&w->wqkv, &w->wo, &w->w1, &w->w2};
  for (auto* t : ops)
    if ((st = check_operand(t)) != KL_OK) return st;
  if (!aligned(io->x, 16) || !aligned(io->out, 16) || !aligned(io->rope_cs, 32)) return KL_ERR_MISALIGNED;
  const size_t need = kl_block_workspace_size(T, D, H, F, io->attn_precision);
  if (!workspace || ws_bytes < need) return KL_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KL_ERR_MISALIGNED;
  if ((st = check_arch()) != KL_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  BlockWs ws = block_ws_layout(reinterpret_cast<uint8_t*>(workspace), T, D, H, F, io->attn_precision);
  float* amax = ws.words;          // [1] O, [3] h (LN amaxes live in ln1 / ln2)
  float* gs = ws.words + 4;        // [0] m1, [1] O, [2] m2, [3] h
  float* amax_qkv = ws.words + 8;  // [3H]
  float* sc8 = amax_qkv + 3 * H;   // [3H]
  float* ln1 = sc8 + 3 * H;        // LN1 amax
  float* ln2 = ln1 + 2;            // LN2 amax
  cudaError_t e = cudaMemsetAsync(ws.words, 0, (12 + 6 * H) * sizeof(float), s);
#define KL_TRY(x)                      \
  do {                                 \
    if (e == cudaSuccess) e = (x);     \
  } while (0)
  auto mark = [&](int stage) {
    if (io->stage_events && e == cudaSuccess)
      e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(io->stage_events[stage]), s);
  };
  mark(0);
  // 1. m1 = bf16(LN(x)(1+scale1)+shift1) -> NVFP4
  // (m1 goes through the attention-output buffer, free until step 4)
  if (D % 256 == 0 && D <= 4096)
    KL_TRY(launch_ln_modulate_quantize_via_m(io->x, T, D, io->mod[0], io->mod[1], ws.acodes, ws.ascales, &gs[0],
                                             ws.o, ws.stats, ln1, s));
  else
    KL_TRY(launch_ln_modulate_quantize(io->x, T, D, io->mod[0], io->mod[1], ws.acodes, ws.ascales, &gs[0], nullptr,
                                       ws.stats, ln1, s, /*amax_zeroed=*/true));
  mark(1);
  // 2. qkv = m1 Wqkv^T with RoPE on q, k and per-head amax
  GemmArgs g{};
  g.a_codes = ws.acodes;
  g.a_scales = ws.ascales;
  g.a_gs = &gs[0];
  g.w_codes = w->wqkv.codes;
  g.w_scales = w->wqkv.scales;
  g.w_gs = w->wqkv.global_scale;
  g.M = T;
  g.N = 3 * D;
  g.K = D;
  g.epi = KL_EPI_QKV_ROPE;
  g.out = ws.qkv;
  g.rope_cs = io->rope_cs;
  g.amax = amax_qkv;
  KL_TRY(launch_gemm_nvfp4(g, s));
  // 3-4. (FP8 cast) and joint attention -> O bf16 + amax
  AttnArgs a{};
  a.T = T;
  a.H = H;
  a.ld = 3 * D;
  a.out = ws.o;
  a.amax = &amax[1];
  mark(2);
  if (io->attn_precision == KL_ATTN_FP8) {
    KL_TRY(launch_fp8_cast(ws.qkv, T, 3 * D, 3 * D, amax_qkv, ws.qkv8, sc8, s));
    a.fp8 = 1;
    a.q = ws.qkv8;
    a.k = ws.qkv8 + D;
    a.v = ws.qkv8 + 2 * D;
    a.sq = sc8;
    a.sk = sc8 + H;
    a.sv = sc8 + 2 * H;
  } else {
    a.fp8 = 0;
    a.q = ws.qkv;
    a.k = ws.qkv + D;
    a.v = ws.qkv + 2 * D;
  }
  mark(3);
  if (io->sol_tau > 0.f) {  // Sol-Attention: the key tiles each query block visits
    KL_TRY(launch_sol_select(a.q, a.k, a.ld, a.sq, a.sk, T, H, a.fp8 != 0, io->sol_tau, ws.sol_list, ws.sol_ws, s));
    a.kv_list = ws.sol_list;
  }
  if (io->vc_budget > 0.f) {  // VC-Attention: repaired tile pairs from the bf16 q, k, v
    KL_TRY(launch_vc_select(ws.qkv, ws.qkv + D, 3 * D, T, H, io->vc_budget, ws.vc_list8, ws.vc_list16, ws.vc_ws, s));
    a.kv_list = ws.vc_list8;
    KL_TRY(vc_attention(a, ws.qkv, ws.qkv + D, ws.qkv + 2 * D, 3 * D, ws.vc_list16, ws.vc_att, s));
  } else {
    KL_TRY(launch_attention(a, s));
  }
  mark(4);
  // 5. O -> NVFP4 (gs from the attention amax)
  KL_TRY(launch_quantize(ws.o, T, D, ws.acodes, ws.ascales, &gs[1], &amax[1], 1, s));
  mark(5);
  // 6. x1 = bf16(x + gate1 * O Wo^T)
  g = GemmArgs{};
  g.a_codes = ws.acodes;
  g.a_scales = ws.ascales;
  g.a_gs = &gs[1];
  g.w_codes = w->wo.codes;
  g.w_scales = w->wo.scales;
  g.w_gs = w->wo.global_scale;
  g.M = T;
  g.N = D;
  g.K = D;
  g.epi = KL_EPI_GATED_RESIDUAL;
  g.out = ws.x1;
  g.gate = io->mod[2];
  g.residual = io->x;
  KL_TRY(launch_gemm_nvfp4(g, s));
  mark(6);
  // 7. m2 = bf16(LN(x1)(1+scale2)+shift2) -> NVFP4
  // (m2 goes through the attention-output buffer, free again after step 5)
  if (D % 256 == 0 && D <= 4096)
    KL_TRY(launch_ln_modulate_quantize_via_m(ws.x1, T, D, io->mod[3], io->mod[4], ws.acodes, ws.ascales, &gs[2],
                                             ws.o, ws.stats, ln2, s));
  else
    KL_TRY(launch_ln_modulate_quantize(ws.x1, T, D, io->mod[3], io->mod[4], ws.acodes, ws.ascales, &gs[2], nullptr,
                                       ws.stats, ln2, s, /*amax_zeroed=*/true));
  mark(7);
  // 8. h = bf16(silu(g) u), [g u] = m2 W1^T, + amax
  g = GemmArgs{};
  g.a_codes = ws.acodes;
  g.a_scales = ws.ascales;
  g.a_gs = &gs[2];
  g.w_codes = w->w1.codes;
  g.w_scales = w->w1.scales;
  g.w_gs = w->w1.global_scale;
  g.M = T;
  g.N = 2 * F;
  g.K = D;
  g.epi = KL_EPI_SWIGLU;
  g.out = ws.h;
  g.amax = &amax[3];
  KL_TRY(launch_gemm_nvfp4(g, s));
  mark(8);
  // 9. h -> NVFP4
  KL_TRY(launch_quantize(ws.h, T, F, ws.hcodes, ws.hscales, &gs[3], &amax[3], 1, s));
  mark(9);
  // 10. out = bf16(x1 + gate2 * h W2^T)
  g = GemmArgs{};
  g.a_codes = ws.hcodes;
  g.a_scales = ws.hscales;
  g.a_gs = &gs[3];
  g.w_codes = w->w2.codes;
  g.w_scales = w->w2.scales;
  g.w_gs = w->w2.global_scale;
  g.M = T;
  g.N = D;
  g.K = F;
  g.epi = KL_EPI_GATED_RESIDUAL;
  g.out = io->out;
  g.gate = io->mod[5];
  g.residual = ws.x1;
  KL_TRY(launch_gemm_nvfp4(g, s));
  mark(KL_BLOCK_STAGES);
#undef KL_TRY
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

// The block on host buffers: [block workspace][x][out][6 modulation vectors],
// each piece 256-byte aligned.
size_t kl_block_host_workspace_size(int64_t T, int64_t D, int64_t H, int64_t F, int prec) {
  const size_t ws = kl_block_workspace_size(T, D, H, F, prec);
  if (ws == 0) return 0;
  return up256(ws) + 2 * up256((size_t)T * D * 2) + up256((size_t)6 * D * 2);
}

kl_status kl_joint_block_forward_host(const kl_block_weights* w, const kl_block_io* io, void* workspace,
                                      size_t ws_bytes, void* stream) {
  if (!w || !io || !io->x || !io->rope_cs || !io->out) return KL_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!io->mod[i]) return KL_ERR_INVALID_ARG;
  const int64_t T = io->T, D = io->D, H = io->H, F = io->F;
  if (io->attn_precision != KL_ATTN_FP8 && io->attn_precision != KL_ATTN_BF16) return KL_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || H > 64 || D != 128 * H || F < 128 || F % 128 || D > 8192) return KL_ERR_UNSUPPORTED_SHAPE;
  const size_t need = kl_block_host_workspace_size(T, D, H, F, io->attn_precision);
  if (!workspace || ws_bytes < need) return KL_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  const size_t ws_block = up256(kl_block_workspace_size(T, D, H, F, io->attn_precision));
  const size_t act = (size_t)T * D * 2;
  uint8_t* x_dev = base + ws_block;
  uint8_t* out_dev = x_dev + up256(act);
  uint8_t* mod_dev = out_dev + up256(act);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(x_dev, io->x, act, cudaMemcpyHostToDevice, s);
  kl_block_io dio = *io;
  dio.x = x_dev;
  dio.out = out_dev;
  for (int i = 0; i < 6 && e == cudaSuccess; ++i) {
    e = cudaMemcpyAsync(mod_dev + (size_t)i * D * 2, io->mod[i], (size_t)D * 2, cudaMemcpyHostToDevice, s);
    dio.mod[i] = mod_dev + (size_t)i * D * 2;
  }
  if (e != cudaSuccess) return cuda_fail(e);
  st = kl_joint_block_forward(w, &dio, workspace, ws_block, stream);
  if (st != KL_OK) return st;
  e = cudaMemcpyAsync(io->out, out_dev, act, cudaMemcpyDeviceToHost, s);
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

}  // extern "C"
