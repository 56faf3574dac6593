// kl_vc.cu -- VC-Attention repair of FP8 attention ([P1] "Optimizing FLUX 3
// Image Klein inference on NVIDIA Blackwell GPUs", How it works: VC-Attention
// adds a repair budget that corrects the quantization errors of FP8
// attention; Key details: a repair budget of 0.005).
//
// Reading (the pages give no more): the unit of repair is the FP8 attention's
// tile pair, a query block of 256 rows against a key tile of 128 keys, per
// head.  A budget b repairs R = floor(b * n_qb * n_kt) of a head's pairs:
// those with the largest estimated share of their query block's attention,
// w(b, j) = 2^(s_hat(b, j) - max) / sum_j' 2^(s_hat(b, j') - max), s_hat =
// (qbar . kbar) log2(e)/sqrt(128) from block means of the bf16 q and k; equal
// shares go to the lower (b, j) in row-major order.  A repaired pair is
// computed from the bf16 q, k, v: the FP8 kernel visits each query block's
// other tiles, the BF16 kernel its repaired tiles, each leaving per row its
// reference maximum m and mass l, and the two parts are merged exactly:
// O = (O_8 l_8 2^(m_8 - M) + O_16 l_16 2^(m_16 - M)) / (l_8 2^(m_8 - M) +
// l_16 2^(m_16 - M)), M = max(m_8, m_16).
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

constexpr int kVcRows = 256;  // query rows per repair unit (the FP8 attention CTA)

// shares w[h][b][j] of key tile j in query block b's attention: CTA (b, h), a
// warp per key tile for the dots, then max, exp2 and the normalisation.
__global__ void __launch_bounds__(256) vc_share_kernel(const float* __restrict__ qbar,
                                                       const float* __restrict__ kbar, int nqb, int nkt, float c,
                                                       float* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float s_hat[];  // nkt
  __shared__ float qs[128];
  __shared__ float red[8];
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 128) qs[threadIdx.x] = qbar[((int64_t)h * nqb + b) * 128 + threadIdx.x];
  __syncthreads();
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
  mx = red[0];
  for (int i = 1; i < 8; ++i) mx = fmaxf(mx, red[i]);
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < nkt; j += blockDim.x) {
    const float e = exp2f(s_hat[j] - mx);
    s_hat[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < 8; ++i) tot += red[i];  // fixed order
  float* wo = w + ((int64_t)h * nqb + b) * nkt;
  for (int j = threadIdx.x; j < nkt; j += blockDim.x) wo[j] = s_hat[j] / tot;
}

// Per head (CTA of 1024 threads): the R largest shares.  The R-th largest
// value is found by a radix select over the fp32 bit patterns (non-negative,
// so they order like the values), 8 bits at a time from the top; then every
// share above it is repaired, and of the shares equal to it the first ones
// in index order, up to R.  mark[h][b][j] = 1 for a repaired pair.
// SMEM: the head's n shares are held in shared memory (read from global
// once); otherwise every pass reads them from global memory.  The bin holding
// the R-th value is found by warp 0 (8 bins per lane, suffix sums by
// shuffles), the index order of equal shares by a two-level shuffle scan.
template <bool SMEM>
__global__ void __launch_bounds__(1024) vc_topk_kernel(const float* __restrict__ w, int n, int R,
                                                       uint8_t* __restrict__ mark) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t sv[];  // SMEM: n share bit patterns
  __shared__ unsigned int hist[256];
  __shared__ unsigned int sel[3];  // prefix bits, prefix mask, count still to place above the prefix
  __shared__ int wsum[32];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t* wb = reinterpret_cast<const uint32_t*>(w) + (int64_t)h * n;
  uint8_t* mk = mark + (int64_t)h * n;
  auto val = [&](int i) -> uint32_t { return SMEM ? sv[i] : __ldg(wb + i); };
  for (int i = tid; i < n; i += blockDim.x) {
    mk[i] = 0;
    if (SMEM) sv[i] = __ldg(wb + i);
  }
  if (R <= 0) return;
  if (R >= n) {
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) mk[i] = 1;
    return;
  }
  if (tid == 0) {
    sel[0] = 0u;
    sel[1] = 0u;
    sel[2] = (unsigned)R;
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    const uint32_t pre = sel[0], pmask = sel[1];
    for (int i = tid; i < n; i += blockDim.x) {
      const uint32_t v = val(i);
      if ((v & pmask) == pre) atomicAdd(&hist[(v >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l (descending); count at or above
      // each of its bins = the sums of the lanes before it + its own prefix
      unsigned int c[8], tot = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * lane - q];
        tot += c[q];
      }
      unsigned int before = tot;  // inclusive scan of the lane totals, then exclusive
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned int t = __shfl_up_sync(0xffffffffu, before, off);
        if (lane >= off) before += t;
      }
      before -= tot;
      const unsigned int need = sel[2];
      // the lane whose bins reach need: before < need <= before + tot
      const bool mine = before < need && need <= before + tot;
      const unsigned int who = __ballot_sync(0xffffffffu, mine);
      if (mine && lane == __ffs(who) - 1) {
        unsigned int acc = before;
        int d = 255 - 8 * lane;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (acc + c[q] >= need) {
            d = 255 - 8 * lane - q;
            break;
          }
          acc += c[q];
        }
        sel[0] = pre | ((uint32_t)d << shift);
        sel[1] = pmask | (255u << shift);
        sel[2] = need - acc;
      }
    }
    __syncthreads();
  }
  const uint32_t theta = sel[0];
  const unsigned int eq_take = sel[2];  // shares equal to theta that are repaired
  // above theta: repaired; equal: the first eq_take in index order (each
  // thread a contiguous chunk of indices, counts scanned across the block)
  const int chunk = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = tid * chunk, i1 = min(n, i0 + chunk);
  int eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t v = val(i);
    if (v > theta) mk[i] = 1;
    eq += v == theta;
  }
  int incl = eq;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    int xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, off);
      if (lane >= off) xi += t;
    }
    wsum[lane] = xi - x;  // equal shares in the warps before
  }
  __syncthreads();
  int before = wsum[warp] + incl - eq;  // equal shares at lower indices
  for (int i = i0; i < i1; ++i) {
    if (val(i) == theta) {
      if ((unsigned)before < eq_take) mk[i] = 1;
      ++before;
    }
  }
}

// CTA (256-row block b, head h): the FP8 list (the block's tiles that are not
// repaired) and the BF16 lists of its two 128-row halves (the repaired ones),
// ascending, in the kl_sol_select list layout.
__global__ void vc_lists_kernel(const uint8_t* __restrict__ mark, int nqb, int nqb16, int nkt,
                                int* __restrict__ list8, int* __restrict__ list16) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0) return;
  const int b = blockIdx.x, h = blockIdx.y;
  const uint8_t* mk = mark + ((int64_t)h * nqb + b) * nkt;
  int* L8 = list8 + ((int64_t)h * nqb + b) * (nkt + 1);
  int* L16a = list16 + ((int64_t)h * nqb16 + 2 * b) * (nkt + 1);
  int* L16b = 2 * b + 1 < nqb16 ? L16a + (nkt + 1) : nullptr;
  int c8 = 0, c16 = 0;
  for (int j = 0; j < nkt; ++j) {
    if (mk[j]) {
      L16a[1 + c16] = j;
      if (L16b) L16b[1 + c16] = j;
      ++c16;
    } else {
      L8[1 + c8++] = j;
    }
  }
  L8[0] = c8;
  L16a[0] = c16;
  if (L16b) L16b[0] = c16;
}

// O = merge of the FP8 part (bf16 O in out, (m, l) in ml8) and the repaired
// part (fp32 O in o16, (m, l) in ml16), in place; rows whose repaired part is
// empty keep the FP8 result.  8 elements of one (row, head) per thread.
__global__ void __launch_bounds__(256) vc_merge_kernel(uint16_t* __restrict__ out, const float* __restrict__ o16,
                                                       const float2* __restrict__ ml8,
                                                       const float2* __restrict__ ml16, int64_t T, int H) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = T * H * 16;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rh = i >> 4;  // row * H + head
    const float2 b = ml16[rh];
    if (!(b.y > 0.f)) continue;
    const float2 a = ml8[rh];
    const float M = fmaxf(a.x, b.x);
    const float wa = a.y > 0.f ? a.y * exp2f(a.x - M) : 0.f;
    const float wb = b.y * exp2f(b.x - M);
    const float inv = 1.0f / (wa + wb);
    const int64_t e = rh * 128 + (i & 15) * 8;  // element offset in the [T, H*128] row-major outputs
    const uint4 av = *reinterpret_cast<const uint4*>(out + e);
    const float4 b0 = reinterpret_cast<const float4*>(o16 + e)[0];
    const float4 b1 = reinterpret_cast<const float4*>(o16 + e)[1];
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    uint32_t r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // a query block whose every tile was repaired has no FP8 part (wa = 0,
      // and out holds no result for it)
      const float alo = wa > 0.f ? bf16lo_f32(aw[k]) * wa : 0.f, ahi = wa > 0.f ? bf16hi_f32(aw[k]) * wa : 0.f;
      r[k] = pack_bf16x2((alo + bv[2 * k] * wb) * inv, (ahi + bv[2 * k + 1] * wb) * inv);
    }
    *reinterpret_cast<uint4*>(out + e) = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// The (head, query block) items with a non-empty key-tile list, ascending:
// one CTA of 1024 threads, each a contiguous chunk of items, a two-level
// shuffle scan of the counts for the output positions.
__global__ void __launch_bounds__(1024) list_work_kernel(const int* __restrict__ list, int nitems, int stride,
                                                         int* __restrict__ work, int* __restrict__ count) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = (nitems + blockDim.x - 1) / blockDim.x;
  const int i0 = tid * chunk, i1 = min(nitems, i0 + chunk);
  int c = 0;
  for (int i = i0; i < i1; ++i) c += __ldg(list + (int64_t)i * stride) > 0;
  int incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int x = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
    int xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, off);
      if (lane >= off) xi += t;
    }
    wsum[lane] = xi - x;
    if (lane == 31) *count = xi;
  }
  __syncthreads();
  int pos = wsum[warp] + incl - c;
  for (int i = i0; i < i1; ++i)
    if (__ldg(list + (int64_t)i * stride) > 0) work[pos++] = i;
}

// ------------------------------------------------------------ host side
struct VcWs {
  float *qbar, *kbar, *w;
  uint8_t* mark;
  size_t total;
};
static VcWs vc_ws_layout(uint8_t* base, int64_t T, int64_t H) {
  const int64_t nqb = (T + kVcRows - 1) / kVcRows, nkt = (T + 127) / 128;
  VcWs v{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~size_t(255);
    return p;
  };
  v.qbar = reinterpret_cast<float*>(take((size_t)H * nqb * 128 * sizeof(float)));
  v.kbar = reinterpret_cast<float*>(take((size_t)H * nkt * 128 * sizeof(float)));
  v.w = reinterpret_cast<float*>(take((size_t)H * nqb * nkt * sizeof(float)));
  v.mark = take((size_t)H * nqb * nkt);
  v.total = off;
  return v;
}

size_t vc_select_workspace_bytes(int64_t T, int64_t H) { return vc_ws_layout(nullptr, T, H).total; }

int64_t vc_repair_count(int64_t T, float budget) {
  const int64_t nqb = (T + kVcRows - 1) / kVcRows, nkt = (T + 127) / 128;
  const double r = std::floor((double)budget * (double)(nqb * nkt));
  return r < 0 ? 0 : (int64_t)r;
}

cudaError_t launch_vc_select(const void* q, const void* k, int64_t ld, int64_t T, int64_t H, float budget,
                             int* list8, int* list16, void* ws, cudaStream_t s) {
  const int nqb = (int)((T + kVcRows - 1) / kVcRows), nqb16 = (int)((T + 127) / 128), nkt = (int)((T + 127) / 128);
  VcWs v = vc_ws_layout(reinterpret_cast<uint8_t*>(ws), T, H);
  cudaError_t e = launch_pdl(sol_pool_kernel<false>, dim3((unsigned)(nqb + nkt), (unsigned)H), dim3(256), 0, s, q, k,
                             ld, T, kVcRows, nqb, nkt, v.qbar, v.kbar);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)nkt * sizeof(float);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(vc_share_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(vc_share_kernel, dim3((unsigned)nqb, (unsigned)H), dim3(256), smem, s, (const float*)v.qbar,
                 (const float*)v.kbar, nqb, nkt, 1.4426950408889634f / sqrtf(128.0f), v.w);
  if (e != cudaSuccess) return e;
  const int64_t R = vc_repair_count(T, budget);
  const int n = nqb * nkt;
  const size_t tsm = (size_t)n * sizeof(uint32_t);
  if (tsm <= 160 * 1024) {
    if (tsm > 48 * 1024) {
      e = cudaFuncSetAttribute(vc_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
      if (e != cudaSuccess) return e;
    }
    e = launch_pdl(vc_topk_kernel<true>, dim3((unsigned)H), dim3(1024), tsm, s, (const float*)v.w, n, (int)R, v.mark);
  } else {
    e = launch_pdl(vc_topk_kernel<false>, dim3((unsigned)H), dim3(1024), 0, s, (const float*)v.w, n, (int)R, v.mark);
  }
  if (e != cudaSuccess) return e;
  return launch_pdl(vc_lists_kernel, dim3((unsigned)nqb, (unsigned)H), dim3(32), 0, s, (const uint8_t*)v.mark, nqb,
                    nqb16, nkt, list8, list16);
}

cudaError_t launch_list_work(const int* list, int64_t H, int nqb, int nkt, int* work, int* count, cudaStream_t s) {
  return launch_pdl(list_work_kernel, dim3(1), dim3(1024), 0, s, list, (int)(H * nqb), nkt + 1, work, count);
}

cudaError_t launch_vc_merge(void* out, const float* o16, const float2* ml8, const float2* ml16, int64_t T,
                            int64_t H, cudaStream_t s) {
  int64_t g = (T * H * 16 + 255) / 256;
  if (g > (int64_t)kNumSMs * 16) g = (int64_t)kNumSMs * 16;
  return launch_pdl(vc_merge_kernel, dim3((unsigned)g), dim3(256), 0, s, reinterpret_cast<uint16_t*>(out), o16, ml8,
                    ml16, T, (int)H);
}

}  // namespace kl
