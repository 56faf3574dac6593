// kl_dit.cu -- one Euler step of a synthetic FLUX-3-Image-Klein-style DiT on
// the block kernels: patchify the latent, NVFP4 input projection, per-mode
// blocks on the text and image streams, joint blocks on the concatenated
// sequence, final LayerNorm + adaLN + NVFP4, output projection to the
// velocity per patch, and the Euler update latent += dt * v.
//
// Structure ([P2] "FLUX.3 Image Klein Brings 2-Second AI Image Generation to
// Diffusers", Summary: 5 blocks per mode, then 28 joint blocks; [P4] "Welcome
// FLUX.3 Image Klein in Diffusers", The VAE and Tokenization: 2x2 patches of
// the latent; Two-Stage Processing: each stream in its own blocks first).  The
// pages give no layer-level detail beyond that; the readings (patch feature
// order, no biases, text conditioning copied in each step, final adaLN with a
// shift/scale pair) are the plainest ones and are stated with the entry point.
#include "kl_common.cuh"
#include "kl_internal.h"
#include "../../include/klein.h"

namespace kl {

// latent fp32 [2 gh, 2 gw, C] -> patches bf16 [gh * gw, 4 C]: token
// t = (y / 2) * gw + x / 2, feature k = 4 c + 2 (y % 2) + (x % 2)
__global__ void __launch_bounds__(256) patchify_kernel(const float* __restrict__ latent, int64_t gh, int64_t gw,
                                                       int64_t C, uint16_t* __restrict__ patches) {
  pdl_wait();
  pdl_trigger();
  const int64_t K = 4 * C, n = gh * gw * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / K, k = i - t * K;
    const int64_t c = k >> 2, dy = (k >> 1) & 1, dx = k & 1;
    const int64_t y = (t / gw) * 2 + dy, x = (t % gw) * 2 + dx;
    patches[i] = (uint16_t)f32_to_bf16_bits(latent[(y * 2 * gw + x) * C + c]);
  }
}

// latent[y][x][c] = fl(latent + fl(dt * v[t][k])) with the same (t, k) map
__global__ void __launch_bounds__(256) euler_unpatchify_kernel(float* __restrict__ latent,
                                                               const float* __restrict__ v, int64_t gh, int64_t gw,
                                                               int64_t C, float dt) {
  pdl_wait();
  pdl_trigger();
  const int64_t W = 2 * gw, n = 2 * gh * W * C;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % C, yx = i / C, y = yx / W, x = yx - y * W;
    const int64_t t = (y >> 1) * gw + (x >> 1), k = 4 * c + 2 * (y & 1) + (x & 1);
    latent[i] = __fadd_rn(latent[i], __fmul_rn(dt, v[t * 4 * C + k]));
  }
}

static int grid_256(int64_t n) {
  int64_t g = (n + 255) / 256;
  const int64_t cap = (int64_t)kNumSMs * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

struct DitWs {
  uint16_t *tok_a, *tok_b, *patch;
  uint8_t *pcodes, *pscales, *fcodes, *fscales;
  float *words, *v;  // words: [0] patch amax, [1] patch gs, [2..3] final LN amax, [4] final gs
  float2* stats;
  uint8_t* block_ws;
  size_t block_ws_bytes, total;
};

static inline size_t up256d(size_t b) { return (b + 255) & ~size_t(255); }

static DitWs dit_ws_layout(uint8_t* base, const kl_dit_shape& s) {
  const int64_t Ti = s.grid_h * s.grid_w, T = s.n_text + Ti, K = 4 * s.channels;
  DitWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += up256d(bytes);
    return p;
  };
  w.words = reinterpret_cast<float*>(take(64));
  w.tok_a = reinterpret_cast<uint16_t*>(take((size_t)T * s.D * 2));
  w.tok_b = reinterpret_cast<uint16_t*>(take((size_t)T * s.D * 2));
  w.patch = reinterpret_cast<uint16_t*>(take((size_t)Ti * K * 2));
  w.pcodes = take((size_t)Ti * K / 2);
  w.pscales = take(kl_nvfp4_scales_bytes(Ti, K, KL_SCALE_MMA));
  w.fcodes = take((size_t)Ti * s.D / 2);
  w.fscales = take(kl_nvfp4_scales_bytes(Ti, s.D, KL_SCALE_MMA));
  w.stats = reinterpret_cast<float2*>(take((size_t)Ti * sizeof(float2)));
  w.v = reinterpret_cast<float*>(take((size_t)Ti * K * 4));
  w.block_ws_bytes = kl_block_workspace_size(T, s.D, s.H, s.F, s.attn_precision);
  w.block_ws = take(w.block_ws_bytes);
  w.total = off;
  return w;
}

static bool dit_shape_ok(const kl_dit_shape& s) {
  return s.n_text >= 1 && s.grid_h >= 1 && s.grid_w >= 1 && s.channels >= 1 && (4 * s.channels) % 128 == 0 &&
         s.H >= 1 && s.H <= 64 && s.D == 128 * s.H && s.F >= 128 && s.F % 128 == 0 && s.n_mode_blocks >= 0 &&
         s.n_joint_blocks >= 0 && (s.attn_precision == KL_ATTN_FP8 || s.attn_precision == KL_ATTN_BF16);
}

}  // namespace kl

using namespace kl;

extern "C" {

size_t kl_dit_workspace_size(const kl_dit_shape* shape) {
  if (!shape || !dit_shape_ok(*shape)) return 0;
  return dit_ws_layout(nullptr, *shape).total;
}

kl_status kl_dit_step(const kl_dit_shape* shape, const kl_dit_weights* w, const kl_dit_step_io* io, void* workspace,
                      size_t ws_bytes, void* stream) {
  if (!shape || !w || !io || !io->latent || !io->text || !io->mod_final || !io->rope_text || !io->rope_image ||
      !io->rope_joint)
    return KL_ERR_INVALID_ARG;
  const kl_dit_shape s = *shape;
  if (!dit_shape_ok(s)) return KL_ERR_UNSUPPORTED_SHAPE;
  if ((s.n_mode_blocks > 0 && (!w->mode_text || !w->mode_image || !io->mod_mode)) ||
      (s.n_joint_blocks > 0 && (!w->joint || !io->mod_joint)))
    return KL_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < kl_dit_workspace_size(&s)) return KL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return KL_ERR_MISALIGNED;
  const int64_t Ti = s.grid_h * s.grid_w, T = s.n_text + Ti, K = 4 * s.channels, D = s.D;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DitWs ws = dit_ws_layout(reinterpret_cast<uint8_t*>(workspace), s);
  const uint16_t* mod_mode = reinterpret_cast<const uint16_t*>(io->mod_mode);
  const uint16_t* mod_joint = reinterpret_cast<const uint16_t*>(io->mod_joint);
  const uint16_t* mod_final = reinterpret_cast<const uint16_t*>(io->mod_final);
  kl_status r = KL_OK;
  cudaError_t e = cudaMemsetAsync(ws.words, 0, 64, st);
  if (e != cudaSuccess) return cuda_fail(e);

  // 1. patches of the latent -> NVFP4 -> image tokens (rows n_text.. of tok_a)
  e = launch_pdl(patchify_kernel, dim3(grid_256(Ti * K)), dim3(256), 0, st, (const float*)io->latent, s.grid_h,
                 s.grid_w, s.channels, ws.patch);
  if (e == cudaSuccess) e = launch_amax_bf16(ws.patch, Ti * K, &ws.words[0], st);
  if (e == cudaSuccess) e = launch_quantize(ws.patch, Ti, K, ws.pcodes, ws.pscales, &ws.words[1], &ws.words[0], 1, st);
  if (e != cudaSuccess) return cuda_fail(e);
  {
    kl_nvfp4_tensor A{ws.pcodes, ws.pscales, &ws.words[1]};
    kl_epilogue epi{};
    epi.kind = KL_EPI_NONE;
    epi.out_dtype = KL_OUT_BF16;
    epi.out = ws.tok_a + s.n_text * D;
    if ((r = kl_gemm_nvfp4_fused(&A, &w->w_in, Ti, D, K, &epi, stream)) != KL_OK) return r;
  }
  // 2. the text conditioning (rows 0..n_text of tok_a)
  e = cudaMemcpyAsync(ws.tok_a, io->text, (size_t)s.n_text * D * 2, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e);

  // 3. per-mode blocks: each stream attends within itself, its own weights
  uint16_t *cur = ws.tok_a, *nxt = ws.tok_b;
  auto block = [&](const kl_block_weights* bw, const uint16_t* in, uint16_t* out, int64_t Tb, const uint16_t* mod6,
                   const float* rope) {
    kl_block_io b{};
    b.x = in;
    for (int i = 0; i < 6; ++i) b.mod[i] = mod6 + i * D;
    b.rope_cs = rope;
    b.T = Tb;
    b.D = D;
    b.H = s.H;
    b.F = s.F;
    b.attn_precision = s.attn_precision;
    b.out = out;
    return kl_joint_block_forward(bw, &b, ws.block_ws, ws.block_ws_bytes, stream);
  };
  for (int i = 0; i < s.n_mode_blocks; ++i) {
    const uint16_t* m = mod_mode + (size_t)i * 2 * 6 * D;
    if ((r = block(&w->mode_text[i], cur, nxt, s.n_text, m, io->rope_text)) != KL_OK) return r;
    if ((r = block(&w->mode_image[i], cur + s.n_text * D, nxt + s.n_text * D, Ti, m + 6 * D, io->rope_image)) !=
        KL_OK)
      return r;
    uint16_t* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  // 4. joint blocks over [text; image]
  for (int i = 0; i < s.n_joint_blocks; ++i) {
    if ((r = block(&w->joint[i], cur, nxt, T, mod_joint + (size_t)i * 6 * D, io->rope_joint)) != KL_OK) return r;
    uint16_t* tmp = cur;
    cur = nxt;
    nxt = tmp;
  }
  // 5. final LayerNorm + adaLN (shift, scale) of the image tokens -> NVFP4 ->
  //    velocity per patch (fp32) -> latent += dt * v
  e = launch_ln_modulate_quantize(cur + s.n_text * D, Ti, D, mod_final, mod_final + D, ws.fcodes, ws.fscales,
                                  &ws.words[4], nullptr, ws.stats, &ws.words[2], st, /*amax_zeroed=*/true);
  if (e != cudaSuccess) return cuda_fail(e);
  {
    kl_nvfp4_tensor A{ws.fcodes, ws.fscales, &ws.words[4]};
    kl_epilogue epi{};
    epi.kind = KL_EPI_NONE;
    epi.out_dtype = KL_OUT_F32;
    epi.out = ws.v;
    if ((r = kl_gemm_nvfp4_fused(&A, &w->w_out, Ti, K, D, &epi, stream)) != KL_OK) return r;
  }
  e = launch_pdl(euler_unpatchify_kernel, dim3(grid_256(Ti * K)), dim3(256), 0, st, io->latent, (const float*)ws.v,
                 s.grid_h, s.grid_w, s.channels, io->dt);
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}

}  // extern "C"
