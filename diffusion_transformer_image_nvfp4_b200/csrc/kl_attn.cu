// kl_attn.cu -- flash-style joint attention on tcgen05 tensor cores, FP8
// (E4M3, per-head scales) or BF16 inputs, fp32 accumulation in TMEM.
//
// Joint attention: every text, noisy-image and reference token attends to all
// tokens of the concatenated sequence ([P4] "Welcome FLUX.3 Image Klein in
// Diffusers", Two-Stage Processing; [P2] "FLUX.3 Image Klein Brings 2-Second AI
// Image Generation to Diffusers", Summary).  FP8 Q/K/V: [P1] "Optimizing FLUX 3
// Image Klein inference on NVIDIA Blackwell GPUs", How it works ("Quantized
// attention uses FP8 precision for query, key, and value").
//
// One CTA = one 128-query tile of one head (192 threads, one CTA per SM):
//  * warp 0 lane 0 -- TMA: the Q tile once, then K and V tiles of 128 keys
//    into a 4-stage (FP8) / 2-stage (BF16) ring, 128-byte swizzle;
//  * warp 1 lane 0 -- MMA: S_j = Q K_j^T into one of two TMEM score buffers,
//    then O_j = P_j V_j into one of two TMEM output buffers (V read MN-major
//    straight from its row-major tile); the score MMA of tile j+1 is issued
//    before the P.V MMA of tile j so the tensor core works while the softmax
//    warps exponentiate;
//  * warps 2-5 -- softmax (thread = query row): row max over S_j (pass 1),
//    p = 2^(s*c - m) (pass 2), P written to smem in the MMA's K-major swizzled
//    layout (FP8: p*256 rounded to E4M3), running row sum l from the unrounded
//    p; O_j is folded into a register accumulator O = O*2^(m_old-m_new) + O_j.
//    Output O / l (times s_v/256 in FP8 mode) as bf16, plus a tensor amax.
// TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

struct AttnParams {
  int64_t T;
  int H;
  int n_kv;
  float c_log2;        // BF16: log2(e)/sqrt(128); FP8: times sq*sk (per head, applied in kernel)
  const float* sq;
  const float* sk;
  const float* sv;
  uint16_t* out;
  float* amax;
};

template <bool FP8>
struct AttnCfg {
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int TILE = 128 * 128 * ELEM;  // Q, K, V or P tile bytes
  static constexpr int NS = FP8 ? 4 : 2;
  static constexpr int KSTEPS = FP8 ? 4 : 8;     // MMA K = 32 (e4m3) or 16 (bf16)
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = TILE;
  static constexpr int P_OFF = KV_OFF + NS * 2 * TILE;
  static constexpr int BAR_OFF = P_OFF + 2 * TILE;
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
  static_assert(SMEM_BYTES <= 232448, "smem budget");
};

// K-major SW128 descriptor of MMA step kk inside a [128 rows x 128 elems] tile
template <bool FP8>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
  const uint32_t off = FP8 ? (uint32_t)kk * 32u : (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
  return smem_desc(base + off, 16, 1024, kLayoutSw128);
}
// MN-major SW128 descriptor of MMA step kk of a V tile [128 keys x 128 dims]
template <bool FP8>
__device__ __forceinline__ uint64_t vdesc(uint32_t base, int kk) {
  const uint32_t rows_per_step = FP8 ? 32u : 16u;
  return smem_desc(base + (uint32_t)kk * rows_per_step * 128u, 16384, 1024, kLayoutSw128);
}

template <bool FP8>
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  tma_load_2d(dst, map, x, y, bar);
  if (!FP8) tma_load_2d(dst + 16384, map, x + 64, y, bar);
}

template <bool FP8>
__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const AttnParams p) {
  using C = AttnCfg<FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + C::NS;
  uint64_t* s_full = kv_empty + C::NS;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 2;
  uint64_t* o_full = p_empty + 2;
  uint64_t* o_empty = o_full + 2;
  uint64_t* drain = o_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y;
  const int n = p.n_kv;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_empty[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* kv_smem = smem + C::KV_OFF;
  uint8_t* p_smem = smem + C::P_OFF;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      mbar_arrive_expect_tx(q_full, C::TILE);
      tma_tile<FP8>(q_smem, &tq, h * 128, qt * 128, q_full);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int s = j % C::NS;
        if (!mbar_wait(&kv_empty[s], ((uint32_t)(j / C::NS) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* ks = kv_smem + s * 2 * C::TILE;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::TILE);
        tma_tile<FP8>(ks, &tk, h * 128, j * 128, &kv_full[s]);
        tma_tile<FP8>(ks + C::TILE, &tv, h * 128, j * 128, &kv_full[s]);
        ++issued;
      }
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort);
      if (!ok) {
        const int first = issued > C::NS ? issued - C::NS : 0;
        for (int i = first; i < issued; ++i) {
          volatile int na = 0;
          mbar_wait(&kv_full[i % C::NS], (uint32_t)(i / C::NS) & 1u, &na);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA
      const uint32_t id_qk = FP8 ? idesc_e4m3(128, 128, 0) : idesc_bf16(128, 128, 0);
      const uint32_t id_pv = FP8 ? idesc_e4m3(128, 128, 1) : idesc_bf16(128, 128, 1);
      const uint32_t q_addr = smem_u32(q_smem);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int s = j % C::NS, b = j & 1;
          if (!mbar_wait(&kv_full[s], (uint32_t)(j / C::NS) & 1u, abort_flag) ||
              !mbar_wait(&s_empty[b], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(kv_smem + s * 2 * C::TILE);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint64_t ad = kmajor_desc<FP8>(q_addr, kk), bd = kmajor_desc<FP8>(k_addr, kk);
            if (FP8)
              mma_f8(tmem + b * 128, ad, bd, id_qk, kk > 0);
            else
              mma_f16(tmem + b * 128, ad, bd, id_qk, kk > 0);
          }
          tc_commit(&s_full[b]);
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj % C::NS, b = jj & 1;
          const uint32_t ph = (uint32_t)(jj >> 1) & 1u;
          if (!mbar_wait(&p_full[b], ph, abort_flag) || !mbar_wait(&o_empty[b], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t p_addr = smem_u32(p_smem + b * C::TILE);
          const uint32_t v_addr = smem_u32(kv_smem + s * 2 * C::TILE + C::TILE);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint64_t ad = kmajor_desc<FP8>(p_addr, kk), bd = vdesc<FP8>(v_addr, kk);
            if (FP8)
              mma_f8(tmem + 256 + b * 128, ad, bd, id_pv, kk > 0);
            else
              mma_f16(tmem + 256 + b * 128, ad, bd, id_pv, kk > 0);
          }
          tc_commit(&o_full[b]);
          tc_commit(&p_empty[b]);
          tc_commit(&kv_empty[s]);
        }
      }
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row inside the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    float c = p.c_log2;
    if (FP8) c *= __ldg(p.sq + h) * __ldg(p.sk + h);
    float o[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, alpha_prev = 0.f;
    bool ok = true;

    auto combine = [&](int i, float a) -> bool {
      const int b = i & 1;
      if (!mbar_wait(&o_full[b], (uint32_t)(i >> 1) & 1u, abort_flag)) return false;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(lane_base + 256 + b * 128 + cc * 32, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) o[cc * 32 + t] = fmaf(o[cc * 32 + t], a, v[t]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[b]);
      return true;
    };

    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      const uint32_t ph = (uint32_t)(j >> 1) & 1u;
      if (!mbar_wait(&s_full[b], ph, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t rem = p.T - (int64_t)j * 128;
      const int valid = rem < 128 ? (int)rem : 128;
      float mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(lane_base + b * 128 + cc * 32, v);
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (cc * 32 + t < valid) mx = fmaxf(mx, v[t]);
      }
      const float m_new = fmaxf(m, mx * c);
      const float alpha = ex2_approx(m - m_new);
      if (!mbar_wait(&p_empty[b], ph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* prow = p_smem + b * C::TILE + r * 128;
      float rowsum = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(lane_base + b * 128 + cc * 32, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float pv = (cc * 32 + t < valid) ? ex2_approx(fmaf(v[t], c, -m_new)) : 0.f;
          rowsum += pv;
          v[t] = pv;
        }
        if (FP8) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float* x = v + hh * 16 + q * 4;
              w[q] = f32x2_to_e4m3x2(x[0] * 256.f, x[1] * 256.f) | (f32x2_to_e4m3x2(x[2] * 256.f, x[3] * 256.f) << 16);
            }
            const int chunk = cc * 2 + hh;
            *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float* x = v + q * 8;
            const uint4 w = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                       pack_bf16x2(x[6], x[7]));
            const int chunk = (cc & 1) * 4 + q;
            *reinterpret_cast<uint4*>(prow + (cc >> 1) * 16384 + ((chunk ^ (r & 7)) << 4)) = w;
          }
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_empty[b]);
        mbar_arrive(&p_full[b]);
      }
      l = fmaf(l, alpha, rowsum);
      if (j >= 1 && !combine(j - 1, alpha_prev)) {
        ok = false;
        break;
      }
      alpha_prev = alpha;
      m = m_new;
    }
    if (ok) ok = combine(n - 1, alpha_prev);
    // epilogue: O / l, bf16, tensor amax
    const int64_t row = (int64_t)qt * 128 + r;
    const bool valid_row = ok && row < p.T;
    float scale = 1.0f / l;
    if (FP8) scale *= __ldg(p.sv + h) * (1.0f / 256.0f);
    float amax = 0.f;
    uint4* dst = reinterpret_cast<uint4*>(p.out + row * (int64_t)p.H * 128 + h * 128);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      float x[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        x[t] = bf16_bits_to_f32(f32_to_bf16_bits(o[q * 8 + t] * scale));
        amax = fmaxf(amax, fabsf(x[t]));
      }
      if (valid_row)
        dst[q] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                            pack_bf16x2(x[6], x[7]));
    }
    if (p.amax) {
      amax = warp_max(valid_row ? amax : 0.f);
      if (lane == 0) atomic_max_nonneg(p.amax, amax);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool FP8>
static cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<FP8>;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t box_inner = FP8 ? 128 : 64;
  const uint64_t cols = (uint64_t)a.H * 128, stride = (uint64_t)a.ld * C::ELEM;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_2d(&tq, dt, a.q, cols, (uint64_t)a.T, stride, box_inner, 128) ||
      !make_tmap_2d(&tk, dt, a.k, cols, (uint64_t)a.T, stride, box_inner, 128) ||
      !make_tmap_2d(&tv, dt, a.v, cols, (uint64_t)a.T, stride, box_inner, 128))
    return cudaErrorInvalidValue;
  AttnParams p;
  p.T = a.T;
  p.H = (int)a.H;
  p.n_kv = (int)((a.T + 127) / 128);
  p.c_log2 = 1.4426950408889634f / sqrtf(128.0f);
  p.sq = a.sq;
  p.sk = a.sk;
  p.sv = a.sv;
  p.out = reinterpret_cast<uint16_t*>(a.out);
  p.amax = a.amax;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.n_kv, (unsigned)a.H);
  attn_kernel<FP8><<<grid, 192, C::SMEM_BYTES, s>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  return a.fp8 ? launch_t<true>(a, s) : launch_t<false>(a, s);
}

}  // namespace kl
