// kl_sparse.cu -- Sol-Attention key-tile selection ([P1] "Optimizing FLUX 3
// Image Klein inference on NVIDIA Blackwell GPUs", How it works: sparse
// attention leaves out less important token pairs by a sparsity threshold;
// What you can do: the tau parameter and a number of initial dense steps).
//
// Pairs are skipped a whole tensor-core tile at a time: the query block one
// attention CTA owns (256 rows with FP8 inputs, 128 with BF16) against a key
// tile of 128 keys.  A pair's importance is estimated from block means,
// s_hat = c * (qbar . kbar) in the kernel's log2 score units (c =
// log2(e)/sqrt(128), times sq*sk for E4M3 inputs, whose unscaled values are
// pooled); a key tile is kept when s_hat >= max_j s_hat_j - tau, so its
// estimated weight is at least 2^-tau of the strongest tile's, which is always
// kept.  The lists feed attn_kernel's kv_list: per (head, query block)
// [count, ascending tile indices], n_kv + 1 ints.
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

// block means: CTA (block b, head h), 8 warps.  A lane loads 16 bytes (16
// E4M3 / 8 BF16 dimensions) of one row, so one warp load covers 4 (FP8) / 2
// (BF16) rows of the head's 128 columns; warp w takes row groups w, w + 8, ...
// with all of its loads in flight together (a query block is 8 groups per
// warp).  Lanes holding the same dimensions are summed by shuffles, then the
// warps' partial sums in warp order in shared memory.  Blocks [0, nqb) pool
// query rows (q_rows each), [nqb, nqb + nkt) key rows (128 each), the last of
// each over its valid rows only.
template <bool FP8>
__global__ void __launch_bounds__(256) sol_pool_kernel(const void* __restrict__ q, const void* __restrict__ k,
                                                       int64_t ld, int64_t T, int q_rows, int nqb, int nkt,
                                                       float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int ELEM = FP8 ? 1 : 2;
  constexpr int DPL = 16 / ELEM;          // dimensions per lane
  constexpr int LPR = 128 / DPL;          // lanes per row
  constexpr int RPG = 32 / LPR;           // rows per warp load
  pdl_wait();
  pdl_trigger();
  __shared__ float part[8][128];
  const int h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool is_q = (int)blockIdx.x < nqb;
  const int b = is_q ? blockIdx.x : blockIdx.x - nqb;
  const int rows = is_q ? q_rows : 128;
  const int64_t r0 = (int64_t)b * rows;
  const int64_t r1 = r0 + rows < T ? r0 + rows : T;
  const int sub = lane / LPR, dim0 = (lane % LPR) * DPL;
  const uint8_t* x = reinterpret_cast<const uint8_t*>(is_q ? q : k) + ((int64_t)h * 128 + dim0) * ELEM;
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  const int groups = (rows + RPG - 1) / RPG;
  for (int g0 = 0; g0 < groups; g0 += 64) {  // one pass covers a whole block here (<= 64 groups)
    uint4 buf[8];  // all eight loads first, then the sums (zeros past the end add nothing)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = g0 + warp + 8 * i;
      const int64_t r = r0 + (int64_t)g * RPG + sub;
      buf[i] = (g < groups && r < r1) ? *reinterpret_cast<const uint4*>(x + r * ld * ELEM) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t ww[4] = {buf[i].x, buf[i].y, buf[i].z, buf[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (FP8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[4 * j + e] += e4m3_to_f32(ww[j] >> (8 * e));
        } else {
          acc[2 * j] += bf16lo_f32(ww[j]);
          acc[2 * j + 1] += bf16hi_f32(ww[j]);
        }
      }
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (sub == 0)
#pragma unroll
    for (int i = 0; i < DPL; ++i) part[warp][dim0 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < 128) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += part[w][threadIdx.x];
    const float mean = sum / (float)(r1 - r0);
    if (is_q)
      qbar[((int64_t)h * nqb + b) * 128 + threadIdx.x] = mean;
    else
      kbar[((int64_t)h * nkt + b) * 128 + threadIdx.x] = mean;
  }
}

// CTA (query block b, head h), 8 warps: s_hat for every key tile (a warp per
// tile, 4 dimensions per lane), the maximum, then the kept tiles in ascending
// order (thread 0).  Non-finite estimates keep every tile.
__global__ void __launch_bounds__(256) sol_select_kernel(const float* __restrict__ qbar,
                                                         const float* __restrict__ kbar, int nqb, int nkt,
                                                         const float* __restrict__ sq, const float* __restrict__ sk,
                                                         float c0, float tau, int* __restrict__ list) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float s_hat[];  // nkt
  __shared__ float qs[128];
  __shared__ float red[8];
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 128) qs[threadIdx.x] = qbar[((int64_t)h * nqb + b) * 128 + threadIdx.x];
  __syncthreads();
  const float c = sq ? c0 * __ldg(sq + h) * __ldg(sk + h) : c0;
  float mx = -INFINITY;
  for (int j = warp; j < nkt; j += 8) {
    const float4 kv = reinterpret_cast<const float4*>(kbar + ((int64_t)h * nkt + j) * 128)[lane];
    float dot = qs[4 * lane] * kv.x;
    dot = fmaf(qs[4 * lane + 1], kv.y, dot);
    dot = fmaf(qs[4 * lane + 2], kv.z, dot);
    dot = fmaf(qs[4 * lane + 3], kv.w, dot);
    const float sh = warp_sum(dot) * c;
    if (lane == 0) s_hat[j] = sh;
    mx = fmaxf(mx, sh);
  }
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    int* L = list + ((int64_t)h * nqb + b) * (nkt + 1);
    int cnt = 0;
    if (isfinite(m)) {
      const float thr = m - tau;
      for (int j = 0; j < nkt; ++j)
        if (s_hat[j] >= thr) L[1 + cnt++] = j;
    }
    if (cnt == 0)
      for (int j = 0; j < nkt; ++j) L[1 + cnt++] = j;
    L[0] = cnt;
  }
}

int sol_query_rows(bool fp8) { return fp8 ? 256 : 128; }

size_t sol_list_ints(int64_t T, int64_t H, bool fp8) {
  const int64_t qr = sol_query_rows(fp8), nqb = (T + qr - 1) / qr, nkt = (T + 127) / 128;
  return (size_t)(H * nqb * (nkt + 1));
}

size_t sol_workspace_bytes(int64_t T, int64_t H, bool fp8) {
  const int64_t qr = sol_query_rows(fp8), nqb = (T + qr - 1) / qr, nkt = (T + 127) / 128;
  return (size_t)(H * (nqb + nkt) * 128 * sizeof(float));
}

cudaError_t launch_sol_select(const void* q, const void* k, int64_t ld, const float* sq, const float* sk, int64_t T,
                              int64_t H, bool fp8, float tau, int* list, void* ws, cudaStream_t s) {
  const int qr = sol_query_rows(fp8);
  const int nqb = (int)((T + qr - 1) / qr), nkt = (int)((T + 127) / 128);
  float* qbar = reinterpret_cast<float*>(ws);
  float* kbar = qbar + (int64_t)H * nqb * 128;
  const dim3 pool_grid((unsigned)(nqb + nkt), (unsigned)H);
  cudaError_t e = fp8 ? launch_pdl(sol_pool_kernel<true>, pool_grid, dim3(256), 0, s, q, k, ld, T, qr, nqb, nkt, qbar,
                                   kbar)
                      : launch_pdl(sol_pool_kernel<false>, pool_grid, dim3(256), 0, s, q, k, ld, T, qr, nqb, nkt,
                                   qbar, kbar);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)nkt * sizeof(float);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(sol_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(sol_select_kernel, dim3((unsigned)nqb, (unsigned)H), dim3(256), smem, s, (const float*)qbar,
                    (const float*)kbar, nqb, nkt, fp8 ? sq : nullptr, fp8 ? sk : nullptr,
                    1.4426950408889634f / sqrtf(128.0f), tau, list);
}

}  // namespace kl
