// kl_gemm.cu -- NVFP4 block-scaled GEMM on 5th-generation tensor cores
// (tcgen05.mma kind::mxf4nvf4, 16-element UE4M3 block scales), with the fused
// epilogues of the joint block: RoPE + per-head amax on the QKV projection,
// SwiGLU + amax on the MLP up projection, adaLN-gated residual on the output
// and MLP down projections.
//
// [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs",
// How it works: NVFP4 weights and activations feed optimised GEMM kernels that
// fuse SwiGLU activations and rotary position embeddings.  The page names
// those kernels (PrimsTS) but gives no design; this one is written for B200:
//
//  * persistent grid (one 352-thread CTA per SM), 128 x BN output tiles,
//    BN = 256 (one TMEM accumulator) or 128 (two, so the epilogue of tile i
//    overlaps the main loop of tile i+1);
//  * warp 0 lane 0: TMA producer.  A [128 x 256] and W [BN x 256] FP4 tiles
//    (128 bytes per row, 128-byte swizzle) by cp.async.bulk.tensor; the block
//    scales for those tiles, already stored in the MMA scale layout, by
//    cp.async.bulk (contiguous 512-byte atoms);
//  * warp 10 lane 0: scale copier.  Per 64-wide K step, tcgen05.cp of the A
//    and W scale atoms into the stage's own TMEM scale buffer, ahead of the
//    MMA issuer (tcgen05.commit -> sf_ready);
//  * warp 1 lane 0: MMA issuer.  One 128 x BN x 64 block-scaled MMA per K
//    step into the TMEM accumulator; tcgen05.commit releases smem stages and
//    publishes finished tiles;
//  * warps 2-9: epilogue (thread = row, two warps per 32-lane TMEM group,
//    one per half of the tile's columns).  The whole accumulator is drained
//    to registers with tcgen05.ld and released before the math, so scaling by
//    gA*gW, the fused epilogue and the stores overlap the next tile's MMAs.
// Smem ring: 4 (BN 256) or 6 (BN 128) stages of ~54 / 36 KB.
#include "kl_common.cuh"
#include "kl_internal.h"
#include "../../include/klein.h"

namespace kl {

struct GemmParams {
  int64_t M, N, K;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* gsa;
  const float* gsw;
  int epi, out_f32;
  void* out;
  const float2* rope_cs;
  const uint16_t* gate;
  const uint16_t* residual;
  float* amax;
  int num_m, num_tiles, num_kt, kbn;  // kbn = K / 64
};

// BN: output tile width (256 or 128).  KS: 64-wide K steps per smem stage
// (4 -> 128-byte operand rows, 128-byte swizzle; 2 -> 64-byte rows, 64-byte
// swizzle and twice the stages for the same bytes in flight).
template <int BN, int KS = 4>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int ROWB = KS * 32;               // operand bytes per row per stage
  static constexpr int A_BYTES = BM * ROWB;
  static constexpr int B_BYTES = BN * ROWB;
  static constexpr int SFA_BYTES = KS * 512;
  static constexpr int SFB_BYTES = (BN / 128) * KS * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = (220 * 1024) / STAGE_BYTES;
  static constexpr int ACC = BN == 256 ? 1 : 2;
  static constexpr uint32_t LAYOUT = KS == 4 ? 2u : 4u;   // smem descriptor swizzle: 128 B or 64 B
  static constexpr uint32_t SBO = 8 * ROWB;               // bytes between 8-row groups
  // block scales: one TMEM buffer per smem stage (SFA 4*KS columns, SFB
  // KS*4*BN/128), so the scale copy of a K tile never waits for the MMAs of
  // an earlier K tile to finish reading the previous scales
  static constexpr uint32_t SF_COLS = 4 * KS + KS * 4 * (BN / 128);
  static constexpr uint32_t SF_BASE = ACC * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 512;
  static_assert(SF_BASE + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "smem budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
};

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void load_bf16x32(const uint16_t* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = __ldg(s + q);
    uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * q + 2 * j] = bf16_bits_to_f32(u[j] & 0xFFFFu);
      v[8 * q + 2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
    }
  }
}
// round to bf16 in place (the stored value), returning max |.|
__device__ __forceinline__ float round_bf16x32(float (&v)[32]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = bf16_bits_to_f32(f32_to_bf16_bits(v[i]));
    m = fmaxf(m, fabsf(v[i]));
  }
  return m;
}

template <int BN, int KS>
__global__ void __launch_bounds__(352, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const GemmParams p) {
  using C = GemmCfg<BN, KS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + C::ACC;
  uint64_t* sf_ready = tempty + C::ACC;   // STAGES: scales of the stage are in TMEM
  uint64_t* drain = sf_ready + C::STAGES;  // 2: MMA issuer, scale copier
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    for (int a = 0; a < C::ACC; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int mb = tile % p.num_m, nb = tile / p.num_m;
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          uint8_t* ssfa = sb + C::B_BYTES;
          uint8_t* ssfb = ssfa + C::SFA_BYTES;
          const int nk = min(KS, p.kbn - kt * KS);
          const uint32_t sf_bytes = (uint32_t)nk * 512u;
          mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + sf_bytes * (1 + BN / 128));
          tma_load_2d(sa, &tmap_a, kt * C::ROWB, mb * 128, &full[stage]);
          tma_load_2d(sb, &tmap_b, kt * C::ROWB, nb * BN, &full[stage]);
          bulk_load(ssfa, p.sfa + ((int64_t)mb * p.kbn + kt * KS) * 512, sf_bytes, &full[stage]);
#pragma unroll
          for (int j = 0; j < BN / 128; ++j)
            bulk_load(ssfb + j * KS * 512, p.sfb + ((int64_t)(nb * (BN / 128) + j) * p.kbn + kt * KS) * 512,
                      sf_bytes, &full[stage]);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA can exit
        const int64_t first = issued > C::STAGES ? issued - C::STAGES : 0;
        for (int64_t i = first; i < issued; ++i) {
          volatile int no_abort = 0;
          mbar_wait(&full[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), &no_abort);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_nvf4(128, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kt = 0; kt < p.num_kt; ++kt) {
          // the operand tiles have landed and the scale-copy warp has moved
          // this stage's block scales into the stage's TMEM scale buffer
          if (!mbar_wait(&full[stage], phase, abort_flag) || !mbar_wait(&sf_ready[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = smem + stage * C::STAGE_BYTES;
          const uint8_t* sb = sa + C::A_BYTES;
          const int nk = min(KS, p.kbn - kt * KS);
          const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4 * KS;
          for (int kk = 0; kk < nk; ++kk) {
            const uint64_t ad = smem_desc(smem_u32(sa + kk * 32), 16, C::SBO, C::LAYOUT);
            const uint64_t bd = smem_desc(smem_u32(sb + kk * 32), 16, C::SBO, C::LAYOUT);
            mma_nvf4(d_tmem, ad, bd, idesc, sfa_t + kk * 4, sfb_t + kk * (BN / 32), (kt | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == C::ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // every MMA issued by this thread has completed before TMEM is freed
      tc_commit(&drain[0]);
      volatile int no_abort = 0;
      mbar_wait(&drain[0], 0, &no_abort);
    }
  } else if (warp == 10) {
    // -------------------------------------------------------- scale copier
    // Moves each stage's block scales from smem into that stage's TMEM scale
    // buffer as soon as the stage lands, ahead of the MMA issuer, so the MMA
    // thread issues only MMAs.  A stage (and its scale buffer) is refilled
    // only after the MMAs that read it have completed (empty -> producer ->
    // full), so the copies never overwrite scales still in use.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* ssfa = smem + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
          const uint8_t* ssfb = ssfa + C::SFA_BYTES;
          const int nk = min(KS, p.kbn - kt * KS);
          const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4 * KS;
          for (int kk = 0; kk < nk; ++kk) {
            tmem_cp_32x128b_x4(sfa_t + kk * 4, smem_desc(smem_u32(ssfa + kk * 512), 0, 128, kLayoutNone));
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tmem_cp_32x128b_x4(sfb_t + kk * (BN / 32) + j * 4,
                                 smem_desc(smem_u32(ssfb + j * KS * 512 + kk * 512), 0, 128, kLayoutNone));
          }
          tc_commit(&sf_ready[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      tc_commit(&drain[1]);
      volatile int no_abort = 0;
      mbar_wait(&drain[1], 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // 8 warps: warp w reads TMEM lanes 32*(w%4).. (its rows) and one half of
    // the tile's columns.  Each tile is first drained into registers and the
    // accumulator released at once, so the math and stores below overlap the
    // next tile's MMAs.
    constexpr int HALF = BN / 2;        // accumulator columns per thread
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = quad * 32 + lane;
    const float alpha = __fmul_rn(__ldg(p.gsa), __ldg(p.gsw));
    const int64_t D = p.N / 3;           // QKV only
    const int H = (int)(D >> 7);
    int acc = 0;
    uint32_t acc_phase = 0;
    float v[HALF];
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      if (!warp_wait(&tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int64_t row = (int64_t)mb * 128 + row_in_tile;
      const bool valid = row < p.M;
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      const int64_t n0 = (int64_t)nb * BN;
      if constexpr (BN == 256) {
        // columns [128*half, 128*half + 128): for SwiGLU that is exactly one
        // 64-gate + 64-up row group, already in the order used below
        tmem_ld128(tbase + half * 128, v);
      } else if (p.epi == KL_EPI_SWIGLU) {
        // this thread's outputs o in [half*BN/4, (half+1)*BN/4): gate column
        // (o/64)*128 + o%64 of the tile, up column = gate column + 64
#pragma unroll
        for (int c = 0; c < BN / 4; c += 32) {
          const int o0 = half * (BN / 4) + c;
          const int gcol = (o0 >> 6) * 128 + (o0 & 63);
          tmem_ld32(tbase + gcol, *reinterpret_cast<float(*)[32]>(v + c));
          tmem_ld32(tbase + gcol + 64, *reinterpret_cast<float(*)[32]>(v + BN / 4 + c));
        }
      } else {
#pragma unroll
        for (int c = 0; c < HALF; c += 32) tmem_ld32(tbase + half * HALF + c, *reinterpret_cast<float(*)[32]>(v + c));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == C::ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
#pragma unroll
      for (int i = 0; i < HALF; ++i) v[i] *= alpha;

      if (p.epi == KL_EPI_SWIGLU) {
        const int64_t F = p.N >> 1;
        float amax = 0.f;
#pragma unroll
        for (int c = 0; c < BN / 4; c += 32) {
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            // silu(g) * u with the fast exp / divide intrinsics (relative
            // error ~1e-6, far below the bf16 rounding of h); the argument
            // is clamped so the denominator stays finite
            const float gg = v[c + i], uu = v[BN / 4 + c + i];
            h[i] = __fdividef(gg, 1.0f + __expf(fminf(-gg, 80.0f))) * uu;
          }
          amax = fmaxf(amax, round_bf16x32(h));
          if (valid) store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * F + (n0 >> 1) + half * (BN / 4) + c, h);
        }
        amax = warp_max(valid ? amax : 0.f);
        if (lane == 0) atomic_max_nonneg(p.amax, amax);
      } else {
#pragma unroll
        for (int c = 0; c < HALF; c += 32) {
          float* w = v + c;
          const int64_t n = n0 + half * HALF + c;
          if (p.epi == KL_EPI_NONE) {
            if (valid) {
              if (p.out_f32) {
                float4* d = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + row * p.N + n);
#pragma unroll
                for (int q = 0; q < 8; ++q) d[q] = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
              } else {
                store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * p.N + n, *reinterpret_cast<float(*)[32]>(w));
              }
            }
          } else if (p.epi == KL_EPI_GATED_RESIDUAL) {
            if (valid) {
              float gt[32], rs[32];
              load_bf16x32(p.gate + n, gt);
              load_bf16x32(p.residual + row * p.N + n, rs);
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = __fmaf_rn(gt[i], w[i], rs[i]);
              store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * p.N + n, *reinterpret_cast<float(*)[32]>(w));
            }
          } else {  // KL_EPI_QKV_ROPE
            const int region = (int)(n / D);
            const int64_t cc = n - (int64_t)region * D;
            const int head = (int)(cc >> 7);
            if (region < 2) {
              const int j0 = (int)((cc & 127) >> 1);
              const float4* cs = reinterpret_cast<const float4*>(p.rope_cs + (valid ? row : 0) * 64 + j0);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 t = __ldg(cs + q);  // (c, s) of two consecutive pairs
                const float a0 = w[4 * q], b0 = w[4 * q + 1], a1 = w[4 * q + 2], b1 = w[4 * q + 3];
                w[4 * q] = a0 * t.x - b0 * t.y;
                w[4 * q + 1] = a0 * t.y + b0 * t.x;
                w[4 * q + 2] = a1 * t.z - b1 * t.w;
                w[4 * q + 3] = a1 * t.w + b1 * t.z;
              }
            }
            float amax = round_bf16x32(*reinterpret_cast<float(*)[32]>(w));
            if (valid) store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * p.N + n, *reinterpret_cast<float(*)[32]>(w));
            amax = warp_max(valid ? amax : 0.f);
            if (lane == 0) atomic_max_nonneg(p.amax + region * H + head, amax);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int KS>
static cudaError_t launch_bn(const GemmArgs& a, cudaStream_t s) {
  using C = GemmCfg<BN, KS>;
  CUtensorMap ta, tb;
  const int swz = KS == 4 ? 128 : 64;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, (uint64_t)(a.K / 2), (uint64_t)a.M,
                    (uint64_t)(a.K / 2), C::ROWB, 128, swz))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, (uint64_t)(a.K / 2), (uint64_t)a.N,
                    (uint64_t)(a.K / 2), C::ROWB, BN, swz))
    return cudaErrorInvalidValue;
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.sfa = reinterpret_cast<const uint8_t*>(a.a_scales);
  p.sfb = reinterpret_cast<const uint8_t*>(a.w_scales);
  p.gsa = a.a_gs;
  p.gsw = a.w_gs;
  p.epi = a.epi;
  p.out_f32 = a.out_f32;
  p.out = a.out;
  p.rope_cs = reinterpret_cast<const float2*>(a.rope_cs);
  p.gate = reinterpret_cast<const uint16_t*>(a.gate);
  p.residual = reinterpret_cast<const uint16_t*>(a.residual);
  p.amax = a.amax;
  p.num_m = (int)((a.M + 127) / 128);
  p.num_tiles = p.num_m * (int)(a.N / BN);
  p.kbn = (int)(a.K / 64);
  p.num_kt = (p.kbn + KS - 1) / KS;
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<BN, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < device_sm_count() ? p.num_tiles : device_sm_count();
  gemm_nvfp4_kernel<BN, KS><<<grid, 352, C::SMEM_BYTES, s>>>(ta, tb, p);
  return cudaGetLastError();
}

#ifndef KL_GEMM_KSTEPS
#define KL_GEMM_KSTEPS 4
#endif

cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s) {
  int bn = a.force_bn;
  if (bn == 0) bn = (a.N % 256 == 0) ? 256 : 128;
  if (bn == 256 && a.N % 256 != 0) return cudaErrorInvalidValue;
  return bn == 256 ? launch_bn<256, KL_GEMM_KSTEPS>(a, s) : launch_bn<128, KL_GEMM_KSTEPS>(a, s);
}

}  // namespace kl
