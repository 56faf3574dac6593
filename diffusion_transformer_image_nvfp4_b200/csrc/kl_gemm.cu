// kl_gemm.cu -- NVFP4 block-scaled GEMM on 5th-generation tensor cores
// (tcgen05.mma kind::mxf4nvf4, 16-element UE4M3 block scales), with the fused
// epilogues of the joint block: RoPE + per-head amax on the QKV projection,
// SwiGLU + amax on the MLP up projection, adaLN-gated residual on the output
// and MLP down projections.
//
// [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs",
// How it works: the projections run NVFP4 x NVFP4 in GEMM kernels that also
// apply the SwiGLU gate and the rotary embedding in place.  The page names
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
// The 2-SM pair kernel further down (the one large GEMMs use) keeps these
// roles with cta_group::2 MMAs; its scale copies are issued by the MMA warp,
// and for a gated epilogue with K <= 4096 its warp 10 stages each tile's
// residual rows in shared memory instead (see the comments there).
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
  int res_prefetch;                   // 2-SM kernel: L2 prefetch of each tile's residual rows
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

// 32 bf16 (64 bytes) of one row.  Each thread of a warp writes a different
// row, so one store instruction touches 32 rows: 32-byte stores (dst 32-byte
// aligned) fill whole L2 sectors and halve the store instructions.
__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&v)[32]) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  if ((reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 16 * h), "r"(w[8 * h]),
                   "r"(w[8 * h + 1]), "r"(w[8 * h + 2]), "r"(w[8 * h + 3]), "r"(w[8 * h + 4]), "r"(w[8 * h + 5]),
                   "r"(w[8 * h + 6]), "r"(w[8 * h + 7])
                   : "memory");
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}
__device__ __forceinline__ void load_bf16x32(const uint16_t* src, float (&v)[32]) {
  uint32_t u[16];
  if ((reinterpret_cast<uintptr_t>(src) & 31) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(u[8 * h]), "=r"(u[8 * h + 1]), "=r"(u[8 * h + 2]), "=r"(u[8 * h + 3]), "=r"(u[8 * h + 4]),
                     "=r"(u[8 * h + 5]), "=r"(u[8 * h + 6]), "=r"(u[8 * h + 7])
                   : "l"(src + 16 * h));
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = __ldg(s + q);
      u[4 * q] = w.x;
      u[4 * q + 1] = w.y;
      u[4 * q + 2] = w.z;
      u[4 * q + 3] = w.w;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v[2 * j] = bf16_bits_to_f32(u[j] & 0xFFFFu);
    v[2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
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

// Fused epilogue of one thread's accumulator slice: v holds BN/2 fp32
// columns of one output row (SwiGLU: BN/4 gate then BN/4 up columns), already
// drained from TMEM.  row / valid: the output row and whether it is < M; n0:
// first column of the tile; half: which half of the tile's columns.
template <int BN>
__device__ __forceinline__ void epilogue_apply(const GemmParams& p, float (&v)[BN / 2], float alpha, int64_t row,
                                               bool valid, int64_t n0, int half, int lane) {
  constexpr int HALF = BN / 2;
  const int64_t D = p.N / 3;  // QKV only
  const int H = (int)(D >> 7);
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
  } else if (BN == 256 && p.epi == KL_EPI_QKV_ROPE) {
    // two heads per tile (columns n0.. and n0 + 128..), each in its own
    // region (q, k or v); this thread holds the columns of pairs
    // [32*half, 32*half + 32) of both: v[0..63] head A, v[64..127] head B
    int region[2], head[2];
    float hmax[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int64_t ne = n0 + e * 128;
      region[e] = (int)(ne / D);
      head[e] = (int)((ne - (int64_t)region[e] * D) >> 7);
    }
    const bool rope = region[0] < 2 || region[1] < 2;
    // table: groups of 4 pairs per token ([16][M][4] of (c, s)); pair
    // 32*half + c/2 + 4*g4 + u of chunk c is group 8*half + c/8 + g4
    const float* cs =
        reinterpret_cast<const float*>(p.rope_cs) + ((int64_t)(8 * half) * p.M + (valid ? row : 0)) * 8;
#pragma unroll
    for (int c = 0; c < 64; c += 32) {
      if (rope) {
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          float t[8];
          // (not volatile: a read-only load the compiler may schedule early)
          asm("ld.global.nc.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
              : "=f"(t[0]), "=f"(t[1]), "=f"(t[2]), "=f"(t[3]), "=f"(t[4]), "=f"(t[5]), "=f"(t[6]), "=f"(t[7])
              : "l"(cs + ((int64_t)(c >> 3) + g4) * p.M * 8));
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (region[e] < 2) {
              float* w = v + e * 64 + c + 8 * g4;
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float a0 = w[2 * u], b0 = w[2 * u + 1];
                w[2 * u] = a0 * t[2 * u] - b0 * t[2 * u + 1];
                w[2 * u + 1] = a0 * t[2 * u + 1] + b0 * t[2 * u];
              }
            }
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float* w = v + e * 64 + c;
        hmax[e] = fmaxf(hmax[e], round_bf16x32(*reinterpret_cast<float(*)[32]>(w)));
        if (valid)
          store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * p.N + n0 + e * 128 + 64 * half + c,
                        *reinterpret_cast<float(*)[32]>(w));
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float m = warp_max(valid ? hmax[e] : 0.f);
      if (lane == 0) atomic_max_nonneg(p.amax + region[e] * H + head[e], m);
    }
  } else {
    // QKV: a thread's HALF (<= 128) columns lie in one head of one region
    // (heads are 128 columns, n0 + half*HALF is a multiple of HALF)
    float qkv_amax = 0.f;
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
        if (region < 2) {
          // the table holds groups of 4 pairs per token ([16][M][4] of (c, s)):
          // one 32-byte load gives a thread its row's 4 pairs, and the 32 lanes
          // (32 consecutive rows) read 1 KB contiguous per load
          const int j0 = (int)((cc & 127) >> 1);  // multiple of 16
          const float* cs = reinterpret_cast<const float*>(p.rope_cs) + ((int64_t)(j0 >> 2) * p.M + (valid ? row : 0)) * 8;
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            float t[8];
            // (not volatile: a read-only load the compiler may schedule early)
            asm("ld.global.nc.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                : "=f"(t[0]), "=f"(t[1]), "=f"(t[2]), "=f"(t[3]), "=f"(t[4]), "=f"(t[5]), "=f"(t[6]), "=f"(t[7])
                : "l"(cs + (int64_t)g4 * p.M * 8));
#pragma unroll
            for (int u = 0; u < 4; ++u) {  // pair j0 + 4*g4 + u
              const int q = 4 * g4 + u;
              const float a0 = w[2 * q], b0 = w[2 * q + 1];
              w[2 * q] = a0 * t[2 * u] - b0 * t[2 * u + 1];
              w[2 * q + 1] = a0 * t[2 * u + 1] + b0 * t[2 * u];
            }
          }
        }
        qkv_amax = fmaxf(qkv_amax, round_bf16x32(*reinterpret_cast<float(*)[32]>(w)));
        if (valid) store_bf16x32(reinterpret_cast<uint16_t*>(p.out) + row * p.N + n, *reinterpret_cast<float(*)[32]>(w));
      }
    }
    if (p.epi == KL_EPI_QKV_ROPE) {
      const int64_t nq = n0 + half * HALF;
      const int region = (int)(nq / D);
      const int head = (int)((nq - (int64_t)region * D) >> 7);
      qkv_amax = warp_max(valid ? qkv_amax : 0.f);
      if (lane == 0) atomic_max_nonneg(p.amax + region * H + head, qkv_amax);
    }
  }

}

// The gated-residual epilogue with the tile's residual rows already in
// shared memory, brought in by TMA during the main loop as 4 boxes of 64
// columns x 128 rows (bf16, 128-byte swizzle: the 16-byte chunk k of row r
// sits at chunk k ^ (r & 7), so the 32 rows a warp reads at one column offset
// hit 8 different chunk positions).  BN 256 tiles, 8 epilogue warps, half =
// which 128 columns.
__device__ __forceinline__ void epilogue_apply_smem(const GemmParams& p, float (&v)[128], float alpha, int64_t row,
                                                    bool valid, int64_t n0, int half, int r, const uint8_t* es) {
  if (!valid) return;
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] *= alpha;
  uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) + row * p.N + n0 + half * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint8_t* box = es + (2 * half + (c >> 1)) * 16384 + r * 128;
    uint32_t rw[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 q = *reinterpret_cast<const uint4*>(box + ((((c & 1) * 4 + u) ^ (r & 7)) << 4));
      rw[4 * u] = q.x;
      rw[4 * u + 1] = q.y;
      rw[4 * u + 2] = q.z;
      rw[4 * u + 3] = q.w;
    }
    float gt[32];
    load_bf16x32(p.gate + n0 + half * 128 + c * 32, gt);  // the same 64 bytes for every row: L1 hits
    float* w = v + c * 32;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      w[2 * j] = __fmaf_rn(gt[2 * j], w[2 * j], bf16_bits_to_f32(rw[j] & 0xFFFFu));
      w[2 * j + 1] = __fmaf_rn(gt[2 * j + 1], w[2 * j + 1], bf16_bits_to_f32(rw[j] >> 16));
    }
    store_bf16x32(dst + c * 32, *reinterpret_cast<float(*)[32]>(w));
  }
}

// Drains one thread's slice of a 128 x BN accumulator (its TMEM lane group
// at tbase) into registers: the BN/2 columns of tile half `half`, or for
// SwiGLU the BN/4 gate and BN/4 up columns of the outputs that half owns.
template <int BN>
__device__ __forceinline__ void epilogue_drain(const GemmParams& p, uint32_t tbase, int half, float (&v)[BN / 2]) {
  constexpr int HALF = BN / 2;
  if constexpr (BN == 256) {
    if (p.epi == KL_EPI_QKV_ROPE) {
      // the tile holds two heads: this thread takes rotation pairs
      // [32*half, 32*half + 32) of both (columns 64*half.. and 128 + 64*half..),
      // so the RoPE table entries it loads serve both heads
      tmem_ld64(tbase + half * 64, *reinterpret_cast<float(*)[64]>(v));
      tmem_ld64(tbase + 128 + half * 64, *reinterpret_cast<float(*)[64]>(v + 64));
    } else {
      // columns [128*half, 128*half + 128): for SwiGLU that is exactly one
      // 64-gate + 64-up row group, already in the order used by the epilogue
      tmem_ld128(tbase + half * 128, v);
    }
  } else {
    if (p.epi == KL_EPI_SWIGLU) {
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
  }
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
  pdl_wait();  // no global memory before the previous kernel of the stream is done
  pdl_trigger();

  // Shared-memory descriptors of stage 0; a stage or K-step offset is added
  // in 16-byte units to the start-address field (no carry: smem < 256 KB).
  const uint64_t desc_a0 = smem_desc(smem_u32(smem), 16, C::SBO, C::LAYOUT);
  const uint64_t desc_b0 = smem_desc(smem_u32(smem + C::A_BYTES), 16, C::SBO, C::LAYOUT);
  const uint64_t desc_sf0 = smem_desc(smem_u32(smem + C::A_BYTES + C::B_BYTES), 0, 128, kLayoutNone);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int mb = tile % p.num_m, nb = tile / p.num_m;
      const uint8_t* sfa_src = p.sfa + (int64_t)mb * p.kbn * 512;
      const uint8_t* sfb_src = p.sfb + (int64_t)nb * (BN / 128) * p.kbn * 512;
      for (int kt = 0; kt < p.num_kt; ++kt) {
        if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          uint8_t* ssfa = sb + C::B_BYTES;
          uint8_t* ssfb = ssfa + C::SFA_BYTES;
          const int nk = min(KS, p.kbn - kt * KS);
          const uint32_t sf_bytes = (uint32_t)nk * 512u;
          mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + sf_bytes * (1 + BN / 128));
          tma_load_2d(sa, &tmap_a, kt * C::ROWB, mb * 128, &full[stage]);
          tma_load_2d(sb, &tmap_b, kt * C::ROWB, nb * BN, &full[stage]);
          bulk_load(ssfa, sfa_src + kt * (KS * 512), sf_bytes, &full[stage]);
#pragma unroll
          for (int j = 0; j < BN / 128; ++j)
            bulk_load(ssfb + j * KS * 512, sfb_src + (int64_t)j * p.kbn * 512 + kt * (KS * 512), sf_bytes,
                      &full[stage]);
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // let every load already issued land before the CTA can exit
      const int64_t first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (int64_t i = first; i < issued; ++i) {
        volatile int no_abort = 0;
        mbar_wait(&full[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), &no_abort);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_nvf4(128, BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      if (!warp_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
      for (int kt = 0; kt < p.num_kt; ++kt) {
        // the operand tiles have landed and the scale-copy warp has moved
        // this stage's block scales into the stage's TMEM scale buffer
        if (!warp_wait(&full[stage], phase, abort_flag) || !warp_wait(&sf_ready[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const int nk = min(KS, p.kbn - kt * KS);
          const uint64_t soff = (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4 * KS;
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            if (kk < nk)
              mma_nvf4(d_tmem, desc_a0 + soff + (uint64_t)(kk * 2), desc_b0 + soff + (uint64_t)(kk * 2), idesc,
                       sfa_t + kk * 4, sfb_t + kk * (BN / 32), (kt | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == C::ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // every MMA issued by this warp has completed before TMEM is freed
    if (elect_one()) tc_commit(&drain[0]);
    __syncwarp();
    volatile int no_abort = 0;
    warp_wait(&drain[0], 0, &no_abort);
  } else if (warp == 10) {
    // -------------------------------------------------------- scale copier
    // Moves each stage's block scales from smem into that stage's TMEM scale
    // buffer as soon as the stage lands, ahead of the MMA issuer, so the MMA
    // warp issues only MMAs.  A stage (and its scale buffer) is refilled
    // only after the MMAs that read it have completed (empty -> producer ->
    // full), so the copies never overwrite scales still in use.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < p.num_kt; ++kt) {
        if (!warp_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const int nk = min(KS, p.kbn - kt * KS);
          const uint64_t soff = (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + 4 * KS;
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            if (kk < nk) {
              tmem_cp_32x128b_x4(sfa_t + kk * 4, desc_sf0 + soff + (uint64_t)(kk * 32));
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tmem_cp_32x128b_x4(sfb_t + kk * (BN / 32) + j * 4,
                                   desc_sf0 + soff + (uint64_t)((C::SFA_BYTES + j * KS * 512 + kk * 512) >> 4));
            }
          }
          tc_commit(&sf_ready[stage]);
        }
        __syncwarp();
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (elect_one()) tc_commit(&drain[1]);
    __syncwarp();
    volatile int no_abort = 0;
    warp_wait(&drain[1], 0, &no_abort);
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
      epilogue_drain<BN>(p, tbase, half, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == C::ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
      epilogue_apply<BN>(p, v, alpha, row, valid, n0, half, lane);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------------- 2-SM
// A CTA pair (cluster of 2) computes a 256 x BN output tile with
// tcgen05.mma.cta_group::2 (M = 256 across the pair): each CTA holds 128 rows
// of A, its BN/2-row half of the W rows, its 128 x BN fp32 accumulator in
// TMEM, and in smem the block scales of its A rows (SFA) and of all BN W rows
// (SFB).  One MMA instruction covers 256 x BN x 64 and one scale copy fills
// both CTAs' TMEM, so per FLOP the pair issues half the instructions of two
// single-CTA tiles, and each CTA loads half of W per stage (38 KB stages at
// BN 256: 5 in flight).  BN 256: one accumulator (256 + 5 x 48 scale columns
// of TMEM); BN 128: two (2 x 128 + 7 x 32), so the epilogue of one tile
// overlaps the MMAs of the next.
//
// Roles (whole warps; one elected lane issues): warp 0 of both CTAs loads its
// operand tiles and scales with cta_group::2 tensor copies that signal the
// leader's stage barrier; warp 1 of the leader issues the scale copies into
// TMEM (tcgen05.cp.cta_group::2) and the MMAs, multicasting its commits to
// both CTAs' stage-empty and accumulator-full barriers; warps 2-9 of both
// CTAs drain their accumulator and arrive on the leader's accumulator-empty
// barrier.  Warp 10: with a staged gated epilogue (ESM) it loads each tile's
// residual rows into shared memory one tile ahead; built with
// KL_SF_IN_MMA=0 it copies the scales instead of warp 1.
#ifndef KL_SF_IN_MMA
#define KL_SF_IN_MMA 1
#endif

// ESM: the gated epilogue's residual rows are staged in shared memory (64 KB,
// loaded by warp 10 during the main loop; one K stage fewer).
template <int BN, bool ESM = false>
struct Gemm2Cfg {
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_BYTES = (BN / 2) * 128;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = ESM ? 4 : (196 * 1024) / STAGE_BYTES;
  static constexpr int EPI_BYTES = ESM ? 65536 : 0;
  static constexpr int ACC = BN == 256 ? 1 : 2;
  static constexpr uint32_t ACC_COLS = BN;
  static constexpr uint32_t SF_COLS = 16 + 16 * (BN / 128);
  static constexpr uint32_t SF_BASE = ACC * ACC_COLS;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 512;
  static_assert(SF_BASE + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "smem budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(!ESM || BN == 256, "staged epilogue: 256-column tiles");
  static_assert(!ESM || KL_SF_IN_MMA, "the staged rows' loader is the scale-copier warp");
};

template <int BN, bool ESM>
__global__ void __launch_bounds__(352, 1)
    gemm_nvfp4_2sm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                          const __grid_constant__ CUtensorMap tmap_res, const GemmParams p) {
  using C = Gemm2Cfg<BN, ESM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + C::STAGES * C::STAGE_BYTES;  // ESM: 64 KB, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::EPI_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_ready = empty + C::STAGES;
  uint64_t* tfull = sf_ready + C::STAGES;  // ACC
  uint64_t* tempty = tfull + C::ACC;       // ACC (leader: 16 arrivals each)
  uint64_t* drain = tempty + C::ACC;       // 2
  uint64_t* epi_full = drain + 2;          // ESM: this CTA's staged rows landed
  uint64_t* epi_empty = epi_full + 1;      // ESM: its 8 epilogue warps are done with them
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epi_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    for (int a = 0; a < C::ACC; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(epi_full, 1);
    mbar_init(epi_empty, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    if (p.res_prefetch || ESM) prefetch_tmap(&tmap_res);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();  // no global memory before the previous kernel of the stream is done
  pdl_trigger();
  const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
  const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
  const int num_m2 = (int)((p.M + 255) / 256);
  const int num_tiles = num_m2 * (int)(p.N / BN);
  // stage-0 descriptors; offsets are added in 16-byte units
  const uint64_t desc_a0 = smem_desc(smem_u32(smem), 16, 1024, kLayoutSw128);
  const uint64_t desc_b0 = smem_desc(smem_u32(smem + C::A_BYTES), 16, 1024, kLayoutSw128);
  const uint64_t desc_sf0 = smem_desc(smem_u32(smem + C::A_BYTES + C::B_BYTES), 0, 128, kLayoutNone);

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
      const int mb2 = tile % num_m2, nb = tile / num_m2;
      for (int kt = 0; kt < p.num_kt; ++kt) {
        if (!warp_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          uint8_t* ssfa = sb + C::B_BYTES;
          uint8_t* ssfb = ssfa + C::SFA_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const uint32_t fb = full_leader + (uint32_t)stage * 8u;
          tma_load_2d_pair(sa, &tmap_a, kt * 128, mb2 * 256 + (int)rank * 128, fb);
          tma_load_2d_pair(sb, &tmap_b, kt * 128, nb * BN + (int)rank * (BN / 2), fb);
          tma_load_2d_pair(ssfa, &tmap_sfa, 0, (mb2 * 2 + (int)rank) * p.kbn + kt * 4, fb);
          tma_load_3d_pair(ssfb, &tmap_sfb, 0, kt * 4, nb * (BN / 128), fb);
          // the epilogue of this tile reads its residual rows: bring them
          // into L2 now, a whole main loop ahead, instead of in the burst in
          // which every SM's epilogue reads at once
          if (!ESM && kt == 0 && p.res_prefetch) tma_prefetch_2d(&tmap_res, nb * BN, mb2 * 256 + (int)rank * 128);
        }
        __syncwarp();
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- MMA issuer (leader)
    if (leader) {
      constexpr uint32_t idesc = idesc_nvf4(256, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        if (!warp_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)acc * C::ACC_COLS;
        for (int kt = 0; kt < p.num_kt; ++kt) {
#if KL_SF_IN_MMA
          if (!warp_wait(&full[stage], phase, abort_flag)) {
#else
          if (!warp_wait(&full[stage], phase, abort_flag) || !warp_wait(&sf_ready[stage], phase, abort_flag)) {
#endif
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const int nk = min(4, p.kbn - kt * 4);
            const uint64_t soff = (uint64_t)((stage * C::STAGE_BYTES) >> 4);
            const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
            const uint32_t sfb_t = sfa_t + 16;
#if KL_SF_IN_MMA
            // scale copies ahead of the MMAs that read them: tcgen05.cp then
            // tcgen05.mma from one thread execute in issue order
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nk) {
                tmem_cp_32x128b_x4_pair(sfa_t + kk * 4, desc_sf0 + soff + (uint64_t)(kk * 32));
#pragma unroll
                for (int j = 0; j < BN / 128; ++j)
                  tmem_cp_32x128b_x4_pair(sfb_t + kk * (BN / 32) + j * 4,
                                          desc_sf0 + soff + (uint64_t)((C::SFA_BYTES + j * 2048 + kk * 512) >> 4));
              }
            }
#endif
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nk)
                mma_nvf4_pair(d_tmem, desc_a0 + soff + (uint64_t)(kk * 2), desc_b0 + soff + (uint64_t)(kk * 2), idesc,
                              sfa_t + kk * 4, sfb_t + kk * (BN / 32), (kt | kk) != 0 ? 1u : 0u);
            }
            tc_commit_pair_mc(&empty[stage], 3);
          }
          __syncwarp();
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair_mc(&tfull[acc], 3);
        __syncwarp();
        if (++acc == C::ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (elect_one()) tc_commit_pair(&drain[0]);
      __syncwarp();
      volatile int no_abort = 0;
      warp_wait(&drain[0], 0, &no_abort);
    }
  } else if (warp == 10) {
    if (ESM) {
      // ------------------------------- residual rows loader (both CTAs)
      // one tile ahead of the epilogue: once its warps are done with the
      // previous tile's rows, this CTA's 128 residual rows of the next tile
      int it = 0;
      for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
        const int mb2 = tile % num_m2, nb = tile / num_m2;
        if (!warp_wait(epi_empty, ((uint32_t)it & 1u) ^ 1u, abort_flag)) break;
        if (elect_one()) {
          const int y = mb2 * 256 + (int)rank * 128;
          mbar_arrive_expect_tx(epi_full, 65536);
#pragma unroll
          for (int b = 0; b < 4; ++b) tma_load_2d(epi_smem + b * 16384, &tmap_res, nb * BN + 64 * b, y, epi_full);
        }
        __syncwarp();
      }
    } else if (leader && !KL_SF_IN_MMA) {
      // ---------------------------------------------- scale copier (leader)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!warp_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const int nk = min(4, p.kbn - kt * 4);
            const uint64_t soff = (uint64_t)((stage * C::STAGE_BYTES) >> 4);
            const uint32_t sfa_t = tmem + C::SF_BASE + (uint32_t)stage * C::SF_COLS;
            const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nk) {
                tmem_cp_32x128b_x4_pair(sfa_t + kk * 4, desc_sf0 + soff + (uint64_t)(kk * 32));
#pragma unroll
                for (int j = 0; j < BN / 128; ++j)
                  tmem_cp_32x128b_x4_pair(sfb_t + kk * (BN / 32) + j * 4,
                                          desc_sf0 + soff + (uint64_t)((C::SFA_BYTES + j * 2048 + kk * 512) >> 4));
              }
            }
            tc_commit_pair(&sf_ready[stage]);
          }
          __syncwarp();
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (elect_one()) tc_commit_pair(&drain[1]);
      __syncwarp();
      volatile int no_abort = 0;
      warp_wait(&drain[1], 0, &no_abort);
    }
  } else {
    // ---------------------------------------------- epilogue (both CTAs)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = quad * 32 + lane;
    const float alpha = __fmul_rn(__ldg(p.gsa), __ldg(p.gsw));
    int acc = 0;
    uint32_t acc_phase = 0;
    float v[BN / 2];
    int it = 0;  // ESM: tiles done (phase of the staged rows)
    for (int tile = pair; tile < num_tiles; tile += npairs) {
      const int mb2 = tile % num_m2, nb = tile / num_m2;
      if (!warp_wait(&tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)acc * C::ACC_COLS;
      epilogue_drain<BN>(p, tb, half, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + (uint32_t)acc * 8u);
      if (++acc == C::ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
      const int64_t row = (int64_t)mb2 * 256 + rank * 128 + row_in_tile;
      if constexpr (ESM) {
        if (!warp_wait(epi_full, (uint32_t)it & 1u, abort_flag)) break;
        epilogue_apply_smem(p, v, alpha, row, row < p.M, (int64_t)nb * BN, half, row_in_tile, epi_smem);
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_empty);
        ++it;
      } else {
        epilogue_apply<BN>(p, v, alpha, row, row < p.M, (int64_t)nb * BN, half, lane);
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while its pair may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

template <int BN, bool ESM>
static cudaError_t launch_2sm(const GemmArgs& a, cudaStream_t s, const CUtensorMap* t_epi) {
  using C = Gemm2Cfg<BN, ESM>;
  CUtensorMap ta, tb, tsa, tsb;
  const uint64_t kbn = (uint64_t)(a.K / 64);
  // block scales: SFA as rows of one 512-byte atom (128 x uint32), 4 atoms
  // (one K stage) per box; SFB as (atom, K block, 128-row block of W), a box
  // of 4 K blocks x BN/128 row blocks
  const uint64_t sfb_dims[3] = {128, kbn, (uint64_t)(a.N / 128)};
  const uint64_t sfb_strides[2] = {512, kbn * 512};
  const uint32_t sfb_box[3] = {128, 4, (uint32_t)(BN / 128)};
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, (uint64_t)(a.K / 2), (uint64_t)a.M,
                    (uint64_t)(a.K / 2), 128, 128, 128) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, (uint64_t)(a.K / 2), (uint64_t)a.N,
                    (uint64_t)(a.K / 2), 128, BN / 2, 128) ||
      !make_tmap_2d(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.a_scales, 128, (uint64_t)((a.M + 127) / 128) * kbn, 512,
                    128, 4, 0) ||
      !make_tmap_3d(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.w_scales, sfb_dims, sfb_strides, sfb_box))
    return cudaErrorInvalidValue;
  // ESM: the staged epilogue rows' map (t_epi); otherwise the residual rows
  // of a tile half (BN x 128 bf16) for the L2 prefetch, skipped when the
  // pointer does not suit a tensor map
  CUtensorMap tr = ESM ? *t_epi : ta;
  int res_prefetch = 0;
  if (!ESM && a.epi == KL_EPI_GATED_RESIDUAL && (reinterpret_cast<uintptr_t>(a.residual) & 15) == 0 &&
      make_tmap_2d(&tr, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.residual, (uint64_t)a.N, (uint64_t)a.M,
                   (uint64_t)a.N * 2, BN, 128, 0))
    res_prefetch = 1;
  GemmParams p;
  p.res_prefetch = res_prefetch;
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
  p.num_m = (int)((a.M + 255) / 256);
  p.num_tiles = p.num_m * (int)(a.N / BN);
  p.kbn = (int)kbn;
  p.num_kt = (p.kbn + 3) / 4;
  cudaError_t e =
      cudaFuncSetAttribute(gemm_nvfp4_2sm_kernel<BN, ESM>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int pairs_max = device_sm_count() / 2;
  const int pairs = p.num_tiles < pairs_max ? p.num_tiles : pairs_max;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(352);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_2sm_kernel<BN, ESM>, ta, tb, tsa, tsb, tr, p);
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
  p.res_prefetch = 0;
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
  return launch_pdl(gemm_nvfp4_kernel<BN, KS>, dim3(grid), dim3(352), C::SMEM_BYTES, s, ta, tb, p);
}

#ifndef KL_GEMM_KSTEPS
#define KL_GEMM_KSTEPS 4
#endif

// Tile choice: 2-SM 256 x BN pair tiles when M > 128 (BN = 256 when
// N % 256 == 0, else 128); otherwise one-CTA 128 x 256 or 128 x 128 tiles.
// force_bn: 0 automatic, 512 / 384 pair tiles of width 256 / 128, 256 / 128
// one-CTA tiles.
cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s) {
  int bn = a.force_bn;
  if (bn == 0) bn = a.M > 128 ? ((a.N % 256 == 0) ? 512 : 384) : ((a.N % 256 == 0) ? 256 : 128);
  if ((bn == 256 || bn == 512) && a.N % 256 != 0) return cudaErrorInvalidValue;
  if (bn == 512) {
    // Staged epilogue rows (shared memory filled by TMA during the main loop,
    // one K stage fewer): measured a gain only for the gated residual with a
    // short K (the out-projection, K = 3,072: 59.4 -> 55.3 us at 8,704 rows);
    // with K = 9,216 the lost stage costs more (60 -> 65 us), and the QKV
    // RoPE table staged the same way was slower too (74 -> 77 us), so those
    // keep the L2-prefetch / register epilogue.  Used when the pointer suits
    // a tensor map.
    CUtensorMap te;
    bool esm = false;
    if (a.epi == KL_EPI_GATED_RESIDUAL && a.K <= 4096 && a.residual &&
        (reinterpret_cast<uintptr_t>(a.residual) & 15) == 0)
      esm = make_tmap_2d(&te, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.residual, (uint64_t)a.N, (uint64_t)a.M,
                         (uint64_t)a.N * 2, 64, 128, 128);
    return esm ? launch_2sm<256, true>(a, s, &te) : launch_2sm<256, false>(a, s, nullptr);
  }
  if (bn == 384) return launch_2sm<128, false>(a, s, nullptr);
  return bn == 256 ? launch_bn<256, KL_GEMM_KSTEPS>(a, s) : launch_bn<128, KL_GEMM_KSTEPS>(a, s);
}

}  // namespace kl
