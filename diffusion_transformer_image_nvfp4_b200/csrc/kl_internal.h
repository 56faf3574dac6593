// kl_internal.h -- host-side launchers shared by the libklein translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kl {

constexpr int kNumSMs = 148;  // B200; only caps grid-stride grids (persistent kernels query the device)

int device_sm_count();  // cached per process

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger
// in kl_common.cuh); every library kernel waits before its first global access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// HBM-bound kernels (kl_quant.cu)
cudaError_t launch_amax_bf16(const void* x, int64_t n, float* amax, cudaStream_t s);
cudaError_t launch_quantize(const void* x, int64_t rows, int64_t cols, void* codes, void* scales, float* gs_io,
                            const float* amax, int mode, cudaStream_t s);
cudaError_t launch_ln_modulate_quantize(const void* x, int64_t rows, int64_t cols, const void* shift,
                                        const void* scale, void* codes, void* scales, float* gs_out,
                                        void* m_out, float2* stats, float* amax, cudaStream_t s,
                                        bool amax_zeroed = false);  // true: the caller zeroed amax[0] on s
cudaError_t launch_ln_modulate_quantize_via_m(const void* x, int64_t rows, int64_t cols, const void* shift,
                                             const void* scale, void* codes, void* scales, float* gs_out,
                                             void* m_buf, float2* stats, float* amax, cudaStream_t s);
cudaError_t launch_ln_modulate_m(const void* x, int64_t rows, int64_t cols, const void* shift, const void* scale,
                                 void* m_buf, float2* stats, float* amax, cudaStream_t s);
cudaError_t launch_fp8_cast(const void* x, int64_t T, int64_t ncols, int64_t ld, const float* amax, void* out,
                            float* scales_out, cudaStream_t s);
cudaError_t launch_rope_table(int64_t n_text, int64_t gh, int64_t gw, int64_t n_ref, double theta, float* cs,
                              cudaStream_t s);

// tcgen05 NVFP4 GEMM (kl_gemm.cu)
struct GemmArgs {
  const void* a_codes;
  const void* a_scales;
  const float* a_gs;
  const void* w_codes;
  const void* w_scales;
  const float* w_gs;
  int64_t M, N, K;
  int epi;        // KL_EPI_*
  int out_f32;    // KL_EPI_NONE only
  void* out;
  const float* rope_cs;
  const void* gate;
  const void* residual;
  float* amax;
  int force_bn;   // 0 = heuristic; 128 / 256 one-CTA tiles, 384 / 512 2-SM pair tiles 256 x 128 / 256 x 256
};
cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s);

// tcgen05 flash attention (kl_attn.cu)
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t ld;  // row stride in elements
  const float* sq;
  const float* sk;
  const float* sv;
  int64_t T, H;
  int fp8;
  void* out;   // bf16 [T, H*128]
  float* amax; // nullable
  const int* kv_list = nullptr;  // nullable: Sol-Attention key-tile lists (kl_sol_select layout)
  float2* ml_out = nullptr;      // nullable: per (row, head) reference maximum m and mass l (partial results)
  float* o32 = nullptr;          // nullable: fp32 output instead of out (partial results)
  int empty_ok = 0;              // kv_list counts of 0 allowed (the CTA writes only ml_out)
  const int* work = nullptr;     // nullable: only the (head, query block) items listed here, as
  const int* work_count = nullptr;  //   h * n_qblocks + qblk, *work_count of them (CTAs past it exit)
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);
// the (head, query block) items whose key-tile list is not empty, ascending
// (h * nqb + b), and their count: one CTA, a block scan (kl_vc.cu)
cudaError_t launch_list_work(const int* list, int64_t H, int nqb, int nkt, int* work, int* count, cudaStream_t s);

// Sol-Attention key-tile selection (kl_sparse.cu)
int sol_query_rows(bool fp8);  // rows of one attention query block: 256 (FP8) / 128 (BF16)
size_t sol_list_ints(int64_t T, int64_t H, bool fp8);
size_t sol_workspace_bytes(int64_t T, int64_t H, bool fp8);
cudaError_t launch_sol_select(const void* q, const void* k, int64_t ld, const float* sq, const float* sk, int64_t T,
                              int64_t H, bool fp8, float tau, int* list, void* ws, cudaStream_t s);

// VC-Attention repair (kl_vc.cu)
size_t vc_select_workspace_bytes(int64_t T, int64_t H);
int64_t vc_repair_count(int64_t T, float budget);  // repaired pairs per head
cudaError_t launch_vc_select(const void* q, const void* k, int64_t ld, int64_t T, int64_t H, float budget,
                             int* list8, int* list16, void* ws, cudaStream_t s);
cudaError_t launch_vc_merge(void* out, const float* o16, const float2* ml8, const float2* ml16, int64_t T,
                            int64_t H, cudaStream_t s);

// tensor maps (kl_api.cu)
// 2D tensor map, box_inner x box_outer elements; swizzle_bytes 128, 64 or 0 (none)
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes = 128);
// 3D tensor map without swizzle: dims / box innermost first, strides of dims 1 and 2 in bytes
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                  const uint64_t strides_bytes[2], const uint32_t box[3]);

}  // namespace kl
