// kl_quant.cu -- the HBM-bound kernels of the block: per-tensor amax, the
// NVFP4 quantiser, fused LayerNorm + adaLN modulation + NVFP4 quantiser, the
// per-head FP8 cast of Q/K/V, and the RoPE cos/sin table.
//
// NVFP4 reading (the NVFP4 variant of "Optimizing FLUX 3 Image Klein inference
// on NVIDIA Blackwell GPUs", How it works; the page names the format but not
// its encoding): E2M1 codes, one unsigned E4M3 scale per 16 elements, fp32
// decode global scale gs = amax/2688.  Every step is one IEEE fp32 operation
// with round-to-nearest-even (explicit __f*_rn intrinsics, so no FMA
// contraction and no approximate reciprocal can change a code), then the
// hardware cvt.rn.satfinite conversions to E4M3 / E2M1.
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

constexpr float kGsDivisor = 2688.0f;  // 6 * 448

// ------------------------------------------------------------------ amax
// max |x| over n bf16 values (n % 8 == 0, 16-byte aligned) into *amax (which
// the launcher zeroes first).  Non-finite input sets KL_DEVERR_NONFINITE.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint4* __restrict__ x, int64_t n8,
                                                        float* __restrict__ amax) {
  pdl_wait();
  pdl_trigger();
  float m = 0.f;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    uint4 v = __ldg(x + i);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
      bad |= (lo >= 0x7F80u) | (hi >= 0x7F80u);
      m = fmaxf(m, fmaxf(__uint_as_float(lo << 16), __uint_as_float(hi << 16)));
    }
  }
  m = warp_max(m);
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = m;
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(KL_DEVERR_NONFINITE);
  __syncthreads();
  if (warp == 0) {
    m = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    m = warp_max(m);
    if (lane == 0) atomic_max_nonneg(amax, m);
  }
}

// --------------------------------------------------------- block encoder
struct GsParams {
  float gs, inv;  // decode global scale and 1/(6 gs)
};
__device__ __forceinline__ GsParams gs_from_amax(float amax) {
  GsParams p;
  p.gs = amax == 0.f ? 1.0f : __fdiv_rn(amax, kGsDivisor);
  p.inv = __fdiv_rn(1.0f, __fmul_rn(6.0f, p.gs));
  return p;
}
__device__ __forceinline__ GsParams gs_given(float gs) {
  GsParams p;
  p.gs = gs;
  p.inv = __fdiv_rn(1.0f, __fmul_rn(6.0f, gs));
  return p;
}

// 1/S for every scale byte sb (S = e4m3(sb) * gs; 0 when S is 0), computed
// once per CTA: the same IEEE fp32 multiply and division the encoder would
// otherwise do per 16-element block, so the codes are unchanged.  sb never
// exceeds 0x7E (448) after the satfinite conversion.
__device__ __forceinline__ void fill_rcp_table(float* tab, const GsParams& g) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    const float S = __fmul_rn(e4m3_to_f32((uint32_t)i), g.gs);
    tab[i] = S == 0.f ? 0.f : __fdiv_rn(1.0f, S);
  }
}

// y = v * r for eight floats (packed fp32x2 multiplies, RNE) -> eight e2m1
__device__ __forceinline__ uint32_t scale_to_e2m1x8(const float* v, float r) {
  const uint64_t r2 = pack_f32x2(r, r);
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) unpack_f32x2(mul_f32x2(pack_f32x2(v[i], v[i + 1]), r2), y[i], y[i + 1]);
  return f32x8_to_e2m1x8(y);
}

// Encode 16 values: returns the scale byte, writes 8 packed code bytes.
__device__ __forceinline__ uint32_t encode_block16(const float (&v)[16], const GsParams& g, const float* rtab,
                                                   uint2& packed) {
  float amax_b = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
  const uint32_t sb = amax_b > 0.f ? f32_to_e4m3(__fmul_rn(amax_b, g.inv)) : 0u;
  const float r = rtab[sb];
  if (r == 0.f) {
    packed = make_uint2(0u, 0u);
    return sb;
  }
  packed.x = scale_to_e2m1x8(v, r);
  packed.y = scale_to_e2m1x8(v + 8, r);
  return sb;
}

__device__ __forceinline__ int64_t mma_scale_offset(int64_t row, int64_t kb, int64_t cols) {
  const int64_t rb = row >> 7, r = row & 127;
  return ((rb * (cols >> 6) + (kb >> 2)) << 9) + ((r & 31) << 4) + ((r >> 5) << 2) + (kb & 3);
}

__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&v)[16]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}

// floor(b / d) for a per-launch divisor d as the high word of b * r,
// r = ceil(2^64 / d) (host: rcp64): with r = 2^64/d + e, 0 <= e < 1, the
// product overshoots b/d by b*e/2^64 < 1/d for every b < 2^64/d, which never
// reaches the next integer -- exact, without a 64-bit division per element.
// d = 1 wraps r to 0, which div_rcp reads as "no division".
__host__ __device__ __forceinline__ uint64_t rcp64(uint64_t d) { return ~0ull / d + 1; }
__device__ __forceinline__ int64_t div_rcp(int64_t b, uint64_t r) {
  return r ? (int64_t)__umul64hi((uint64_t)b, r) : b;
}

__device__ __forceinline__ int64_t swiglu_src_row(int64_t r, int64_t rows) {
  const int64_t g = r >> 7, i = r & 127;
  return i < 64 ? (g << 6) + i : (rows >> 1) + (g << 6) + (i - 64);
}

// One thread per 16-element block.  mode bits: 1 = MMA scale layout,
// 2 = gs given (read *gs_io), 4 = SwiGLU row interleave.
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                       int64_t cols, int64_t rows_padded,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                       float* __restrict__ gs_io, const float* __restrict__ amax,
                                                       uint64_t kbn_rcp, int mode) {
  pdl_wait();
  pdl_trigger();
  const bool mma = mode & 1, given = mode & 2, perm = mode & 4;
  const GsParams g = given ? gs_given(*gs_io) : gs_from_amax(*amax);
  __shared__ float rtab[128];
  fill_rcp_table(rtab, g);
  __syncthreads();
  const int64_t kbn = cols >> 4;
  const int64_t total = rows_padded * kbn;
  if (!given && blockIdx.x == 0 && threadIdx.x == 0) *gs_io = g.gs;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < total; b += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = div_rcp(b, kbn_rcp), kb = b - row * kbn;
    const int64_t soff = mma ? mma_scale_offset(row, kb, cols) : row * kbn + kb;
    if (row >= rows) {  // padding rows of the MMA layout
      scales[soff] = 0;
      continue;
    }
    const int64_t src = perm ? swiglu_src_row(row, rows) : row;
    float v[16];
    load16_bf16(x + src * cols + (kb << 4), v);
    uint2 pk;
    const uint32_t sb = encode_block16(v, g, rtab, pk);
    *reinterpret_cast<uint2*>(codes + row * (cols >> 1) + (kb << 3)) = pk;
    scales[soff] = (uint8_t)sb;
  }
}

// ---------------------------------------------- LayerNorm + adaLN modulate
// m = bf16( ((x - mean) * rstd) * (1 + scale) + shift ), each step rounded.
__device__ __forceinline__ float ln_mod_value(float xv, float mean, float rstd, float onep, float shift) {
  const float y = __fmul_rn(__fsub_rn(xv, mean), rstd);
  return bf16_bits_to_f32(f32_to_bf16_bits(__fmaf_rn(y, onep, shift)));
}

// One warp per row: mean and rstd (fp32, two passes), then amax of m.
__global__ void __launch_bounds__(256) ln_stats_amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            int64_t cols, const uint16_t* __restrict__ shift,
                                                            const uint16_t* __restrict__ scale,
                                                            float2* __restrict__ stats, float* __restrict__ amax) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x >> 5) + warp;
  float m = 0.f;
  if (row < rows) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * cols);
    const int n8 = (int)(cols >> 3);
    float s = 0.f;
    for (int i = lane; i < n8; i += 32) {
      uint4 v = __ldg(xr + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) s += bf16_bits_to_f32(w[j] & 0xFFFFu) + bf16_bits_to_f32(w[j] >> 16);
    }
    const float mean = __fdiv_rn(warp_sum(s), (float)cols);
    float ss = 0.f;
    for (int i = lane; i < n8; i += 32) {
      uint4 v = __ldg(xr + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float a = bf16_bits_to_f32(w[j] & 0xFFFFu) - mean, b = bf16_bits_to_f32(w[j] >> 16) - mean;
        ss += a * a + b * b;
      }
    }
    const float var = __fdiv_rn(warp_sum(ss), (float)cols);
    const float rstd = __frsqrt_rn(__fadd_rn(var, 1e-6f));
    if (lane == 0) stats[row] = make_float2(mean, rstd);
    const uint4* shr = reinterpret_cast<const uint4*>(shift);
    const uint4* scr = reinterpret_cast<const uint4*>(scale);
    for (int i = lane; i < n8; i += 32) {
      uint4 v = __ldg(xr + i), sh = __ldg(shr + i), sc = __ldg(scr + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w}, a[4] = {sh.x, sh.y, sh.z, sh.w}, c[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t sft = h ? 16 : 0;
          const float xv = bf16_bits_to_f32((w[j] >> sft) & 0xFFFFu);
          const float onep = __fadd_rn(1.0f, bf16_bits_to_f32((c[j] >> sft) & 0xFFFFu));
          const float mv = ln_mod_value(xv, mean, rstd, onep, bf16_bits_to_f32((a[j] >> sft) & 0xFFFFu));
          m = fmaxf(m, fabsf(mv));
        }
      }
    }
  }
  m = warp_max(m);
  if (lane == 0 && row < rows) atomic_max_nonneg(amax, m);
}

// One thread per 16-element block: recompute m and encode it (MMA layout).
__global__ void __launch_bounds__(256) ln_quant_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                                                       int64_t rows_padded, const uint16_t* __restrict__ shift,
                                                       const uint16_t* __restrict__ scale,
                                                       const float2* __restrict__ stats,
                                                       const float* __restrict__ amax, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales, float* __restrict__ gs_out,
                                                       uint16_t* __restrict__ m_out) {
  pdl_wait();
  pdl_trigger();
  const GsParams g = gs_from_amax(*amax);
  __shared__ float rtab[128];
  fill_rcp_table(rtab, g);
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) *gs_out = g.gs;
  const int64_t kbn = cols >> 4;
  const int64_t total = rows_padded * kbn;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < total; b += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = b / kbn, kb = b - row * kbn;
    const int64_t soff = mma_scale_offset(row, kb, cols);
    if (row >= rows) {
      scales[soff] = 0;
      continue;
    }
    const float2 st = stats[row];
    float xv[16], sh[16], sc[16], v[16];
    load16_bf16(x + row * cols + (kb << 4), xv);
    load16_bf16(shift + (kb << 4), sh);
    load16_bf16(scale + (kb << 4), sc);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = ln_mod_value(xv[i], st.x, st.y, __fadd_rn(1.0f, sc[i]), sh[i]);
    if (m_out) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      uint4* dst = reinterpret_cast<uint4*>(m_out + row * cols + (kb << 4));
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    uint2 pk;
    const uint32_t sb = encode_block16(v, g, rtab, pk);
    *reinterpret_cast<uint2*>(codes + row * (cols >> 1) + (kb << 3)) = pk;
    scales[soff] = (uint8_t)sb;
  }
}

// m of the 8 elements of one 16-byte chunk (4 words of bf16 pairs each for
// x, shift, scale): packed fp32x2 RNE steps, the same operations as
// ln_mod_value (x - mean, * rstd, fma with 1 + scale and shift), then one
// bf16x2 conversion per pair.  Returns the 4 words of bf16 m.
__device__ __forceinline__ uint4 ln_mod_chunk(const uint4& xv, const uint4& sh, const uint4& sc, uint64_t negmean2,
                                              uint64_t rstd2) {
  const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w}, a[4] = {sh.x, sh.y, sh.z, sh.w}, b[4] = {sc.x, sc.y, sc.z, sc.w};
  const uint64_t one2 = pack_f32x2(1.0f, 1.0f);
  uint32_t m[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint64_t y = mul_f32x2(add_f32x2(bf16x2_to_f32x2(w[j]), negmean2), rstd2);
    const uint64_t onep = add_f32x2(one2, bf16x2_to_f32x2(b[j]));
    float lo, hi;
    unpack_f32x2(fma_f32x2(y, onep, bf16x2_to_f32x2(a[j])), lo, hi);
    m[j] = pack_bf16x2(lo, hi);
  }
  return make_uint4(m[0], m[1], m[2], m[3]);
}

// ------------------------- LayerNorm + modulate, warp per row, NCH chunks
// Lane l holds elements [(c*32 + l)*8, +8) of chunk c, c < NCH = cols/256;
// all NCH 16-byte loads of a row are issued before any arithmetic.
// Statistics pass: mean, rstd (the same fp32 operation sequence as
// ln_stats_amax_kernel) and the amax of m, from registers.
template <int NCH>
__global__ void __launch_bounds__(256, 2) ln_stats_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            const uint16_t* __restrict__ shift,
                                                            const uint16_t* __restrict__ scale,
                                                            float2* __restrict__ stats, float* __restrict__ amax,
                                                            uint16_t* __restrict__ m_out) {
  pdl_wait();
  pdl_trigger();
  constexpr int64_t cols = NCH * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  uint32_t amax_w = 0u;
  if (row < rows) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * cols);
    uint4 xv[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) xv[c] = __ldg(xr + c * 32 + lane);
    // sums in two packed fp32 chains per lane (a fixed order, so the same
    // row always gives the same statistics)
    uint64_t s2[2] = {0ull, 0ull};
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const uint32_t w[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) s2[j & 1] = add_f32x2(s2[j & 1], bf16x2_to_f32x2(w[j]));
    }
    float s0, s1, s2a, s3;
    unpack_f32x2(s2[0], s0, s1);
    unpack_f32x2(s2[1], s2a, s3);
    const float mean = __fdiv_rn(warp_sum((s0 + s1) + (s2a + s3)), (float)cols);
    const uint64_t negmean2 = pack_f32x2(-mean, -mean);
    uint64_t q2[2] = {0ull, 0ull};
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const uint32_t w[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t d = add_f32x2(bf16x2_to_f32x2(w[j]), negmean2);
        q2[j & 1] = fma_f32x2(d, d, q2[j & 1]);
      }
    }
    unpack_f32x2(q2[0], s0, s1);
    unpack_f32x2(q2[1], s2a, s3);
    const float rstd = __frsqrt_rn(__fadd_rn(__fdiv_rn(warp_sum((s0 + s1) + (s2a + s3)), (float)cols), 1e-6f));
    if (lane == 0) stats[row] = make_float2(mean, rstd);
    const uint64_t rstd2 = pack_f32x2(rstd, rstd);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const uint4 sh = __ldg(reinterpret_cast<const uint4*>(shift) + c * 32 + lane);
      const uint4 sc = __ldg(reinterpret_cast<const uint4*>(scale) + c * 32 + lane);
      const uint4 m = ln_mod_chunk(xv[c], sh, sc, negmean2, rstd2);
      if (m_out) reinterpret_cast<uint4*>(m_out + row * cols)[c * 32 + lane] = m;
      amax_w = bf16x2_absmax(bf16x2_absmax(amax_w, m.x), m.y);
      amax_w = bf16x2_absmax(bf16x2_absmax(amax_w, m.z), m.w);
    }
  }
  // one atomic per CTA (not per row): the 8 warps' maxima meet in shared memory
  __shared__ float red[8];
  const float lmax = warp_max(bf16x2_hmax_f32(amax_w));
  if (lane == 0) red[warp] = lmax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    atomic_max_nonneg(amax, m);
  }
}

// Encode pass: recompute m from x (an L2 re-read) and the stored statistics,
// 16-element blocks = the 8 elements of lanes 2k and 2k+1 of one chunk.
template <int NCH>
__global__ void __launch_bounds__(256) ln_quant_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            int64_t rows_padded, const uint16_t* __restrict__ shift,
                                                            const uint16_t* __restrict__ scale,
                                                            const float2* __restrict__ stats,
                                                            const float* __restrict__ amax,
                                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                            float* __restrict__ gs_out, uint16_t* __restrict__ m_out) {
  pdl_wait();
  pdl_trigger();
  constexpr int64_t cols = NCH * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  const GsParams g = gs_from_amax(*amax);
  __shared__ float rtab[128];
  fill_rcp_table(rtab, g);
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) *gs_out = g.gs;
  if (row >= rows_padded) return;
  if (row >= rows) {  // padding rows of the MMA scale layout
    for (int64_t kb = lane; kb < (cols >> 4); kb += 32) scales[mma_scale_offset(row, kb, cols)] = 0;
    return;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * cols);
  uint4 xv[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) xv[c] = __ldg(xr + c * 32 + lane);
  const float2 st = stats[row];
  const uint64_t negmean2 = pack_f32x2(-st.x, -st.x), rstd2 = pack_f32x2(st.y, st.y);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int64_t col = ((int64_t)c * 32 + lane) * 8;
    const uint4 sh = __ldg(reinterpret_cast<const uint4*>(shift) + c * 32 + lane);
    const uint4 sc = __ldg(reinterpret_cast<const uint4*>(scale) + c * 32 + lane);
    const uint4 m = ln_mod_chunk(xv[c], sh, sc, negmean2, rstd2);
    if (m_out) *reinterpret_cast<uint4*>(m_out + row * cols + col) = m;
    // 16-element block = this lane's 8 values and its neighbour's
    const float a8 = bf16x2_hmax_f32(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(0u, m.x), m.y), m.z), m.w));
    const float amax_b = fmaxf(a8, __shfl_xor_sync(0xffffffffu, a8, 1));
    const uint32_t sb = amax_b > 0.f ? f32_to_e4m3(__fmul_rn(amax_b, g.inv)) : 0u;
    const float rr = rtab[sb];
    uint32_t code = 0u;
    if (rr != 0.f) {
      const float v[8] = {bf16lo_f32(m.x), bf16hi_f32(m.x), bf16lo_f32(m.y), bf16hi_f32(m.y),
                          bf16lo_f32(m.z), bf16hi_f32(m.z), bf16lo_f32(m.w), bf16hi_f32(m.w)};
      code = scale_to_e2m1x8(v, rr);
    }
    *reinterpret_cast<uint32_t*>(codes + row * (cols >> 1) + (col >> 1)) = code;
    // the chunk's 16 scale bytes (lanes 0, 2, .., 30) are 4 words of the MMA
    // layout: scale kb = c*16 + lane/2 sits at byte (kb & 3) of its word
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sb, 2);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sb, 4);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sb, 6);
    if ((lane & 7) == 0)
      *reinterpret_cast<uint32_t*>(scales + mma_scale_offset(row, col >> 4, cols)) =
          sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

template <int NCH>
static cudaError_t launch_ln_rows(const void* x, int64_t rows, const void* shift, const void* scale, void* codes,
                                  void* scales, float* gs_out, void* m_out, float2* stats, float* amax,
                                  cudaStream_t s) {
  const uint16_t* xp = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* shp = reinterpret_cast<const uint16_t*>(shift);
  const uint16_t* scp = reinterpret_cast<const uint16_t*>(scale);
  cudaError_t e = launch_pdl(ln_stats_rows_kernel<NCH>, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, s, xp, rows,
                             shp, scp, stats, amax, (uint16_t*)nullptr);
  if (e != cudaSuccess) return e;
  const int64_t rows_padded = ((rows + 127) / 128) * 128;
  return launch_pdl(ln_quant_rows_kernel<NCH>, dim3((unsigned)((rows_padded + 7) / 8)), dim3(256), 0, s, xp, rows,
                    rows_padded, shp, scp, stats, (const float*)amax, reinterpret_cast<uint8_t*>(codes),
                    reinterpret_cast<uint8_t*>(scales), gs_out, reinterpret_cast<uint16_t*>(m_out));
}

// ------------------------------------------------------------ FP8 cast
constexpr int kFp8MaxHeads = 512;  // ncols / 128 (the launcher checks)
// 16 elements per thread (inside one 128-wide head).
__global__ void __launch_bounds__(256) fp8_cast_kernel(const uint16_t* __restrict__ x, int64_t T, int64_t ncols,
                                                       int64_t ld, const float* __restrict__ amax,
                                                       uint8_t* __restrict__ out, float* __restrict__ scales_out,
                                                       uint64_t n16_rcp) {
  pdl_wait();
  pdl_trigger();
  const int64_t n16 = ncols >> 4;
  const int64_t total = T * n16;
  const int64_t nheads = ncols >> 7;
  if (blockIdx.x == 0) {
    for (int hh = threadIdx.x; hh < nheads; hh += blockDim.x) {
      const float a = amax[hh];
      scales_out[hh] = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
    }
  }
  // 448/amax per head (the same IEEE division, once per CTA and head)
  __shared__ float inv_tab[kFp8MaxHeads];
  for (int hh = threadIdx.x; hh < nheads; hh += blockDim.x) {
    const float a = amax[hh];
    inv_tab[hh] = a > 0.f ? __fdiv_rn(448.0f, a) : 1.0f;
  }
  __syncthreads();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = div_rcp(i, n16_rcp), c = (i - t * n16) << 4;
    const float inv = inv_tab[c >> 7];
    float v[16];
    load16_bf16(x + t * ld + c, v);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = f32x2_to_e4m3x2(__fmul_rn(v[4 * j], inv), __fmul_rn(v[4 * j + 1], inv)) |
             (f32x2_to_e4m3x2(__fmul_rn(v[4 * j + 2], inv), __fmul_rn(v[4 * j + 3], inv)) << 16);
    *reinterpret_cast<uint4*>(out + t * ld + c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------ RoPE table
__global__ void rope_table_kernel(int64_t n_text, int64_t gh, int64_t gw, int64_t n_ref, double theta,
                                  float2* __restrict__ cs) {
  pdl_wait();
  pdl_trigger();
  // grouped pair-major: the (c, s) of pair j of token t at
  // cs[(j/4 * T + t) * 4 + j%4]; thread i = (j/4 * T + t) * 4 + j%4
  const int64_t T = n_text + (1 + n_ref) * gh * gw;
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= T * 64) return;
  const int64_t gt = i >> 2;
  const int g = (int)(gt / T);
  const int64_t t = gt - (int64_t)g * T;
  const int j = g * 4 + (int)(i & 3);
  double phi;
  if (t < n_text) {
    phi = (double)t * pow(theta, -2.0 * j / 128.0);
  } else {
    const int64_t s = t - n_text, img = gh * gw;
    const int64_t f = s / img, rc = s - f * img, r = rc / gw, c = rc - r * gw;
    if (j < 16)
      phi = (double)f * pow(theta, -2.0 * j / 32.0);
    else if (j < 40)
      phi = (double)r * pow(theta, -2.0 * (j - 16) / 48.0);
    else
      phi = (double)c * pow(theta, -2.0 * (j - 40) / 48.0);
  }
  cs[i] = make_float2((float)cos(phi), (float)sin(phi));
}

// --------------------------------------------------------------- launchers
static int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)kNumSMs * 16;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_amax_bf16(const void* x, int64_t n, float* amax, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  return launch_pdl(amax_bf16_kernel, dim3(grid_for(n / 8, 256)), dim3(256), 0, s, reinterpret_cast<const uint4*>(x),
                    n / 8, amax);
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t cols, void* codes, void* scales, float* gs_io,
                            const float* amax, int mode, cudaStream_t s) {
  const int64_t rows_padded = (mode & 1) ? ((rows + 127) / 128) * 128 : rows;
  return launch_pdl(quantize_kernel, dim3(grid_for(rows_padded * (cols / 16), 256)), dim3(256), 0, s,
                    reinterpret_cast<const uint16_t*>(x), rows, cols, rows_padded, reinterpret_cast<uint8_t*>(codes),
                    reinterpret_cast<uint8_t*>(scales), gs_io, amax, rcp64((uint64_t)(cols / 16)), mode);
}

cudaError_t launch_ln_modulate_quantize(const void* x, int64_t rows, int64_t cols, const void* shift,
                                        const void* scale, void* codes, void* scales, float* gs_out,
                                        void* m_out, float2* stats, float* amax, cudaStream_t s, bool amax_zeroed) {
  cudaError_t e = amax_zeroed ? cudaSuccess : cudaMemsetAsync(amax, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  if (cols % 256 == 0) {
    switch (cols / 256) {
      case 1: return launch_ln_rows<1>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      case 2: return launch_ln_rows<2>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      case 4: return launch_ln_rows<4>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      case 8: return launch_ln_rows<8>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      case 12: return launch_ln_rows<12>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      case 16: return launch_ln_rows<16>(x, rows, shift, scale, codes, scales, gs_out, m_out, stats, amax, s);
      default: break;
    }
  }
  // generic widths: row loop per lane, then one thread per 16-element block
  const int64_t blocks = (rows + 7) / 8;
  e = launch_pdl(ln_stats_amax_kernel, dim3((unsigned)blocks), dim3(256), 0, s, reinterpret_cast<const uint16_t*>(x),
                 rows, cols, reinterpret_cast<const uint16_t*>(shift), reinterpret_cast<const uint16_t*>(scale), stats,
                 amax);
  if (e != cudaSuccess) return e;
  const int64_t rows_padded = ((rows + 127) / 128) * 128;
  return launch_pdl(ln_quant_kernel, dim3(grid_for(rows_padded * (cols / 16), 256)), dim3(256), 0, s,
                    reinterpret_cast<const uint16_t*>(x), rows, cols, rows_padded,
                    reinterpret_cast<const uint16_t*>(shift), reinterpret_cast<const uint16_t*>(scale),
                    (const float2*)stats, (const float*)amax, reinterpret_cast<uint8_t*>(codes),
                    reinterpret_cast<uint8_t*>(scales), gs_out, reinterpret_cast<uint16_t*>(m_out));
}

// LN + adaLN + NVFP4 as two passes over a materialised m: the statistics
// pass also stores m (bf16, rows x cols into m_buf), then the standalone
// quantiser encodes m with gs from the same amax -- the codes the fused
// encoder would produce (it encodes the same bf16 m), from a kernel with one
// thread per 16-element block.  Widths cols = 256 * {1, 2, 4, 8, 12, 16};
// returns cudaErrorInvalidValue for others.  amax[0] must be zero on s.
cudaError_t launch_ln_modulate_quantize_via_m(const void* x, int64_t rows, int64_t cols, const void* shift,
                                             const void* scale, void* codes, void* scales, float* gs_out,
                                             void* m_buf, float2* stats, float* amax, cudaStream_t s) {
  if (cols % 256) return cudaErrorInvalidValue;
  const uint16_t* xp = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* shp = reinterpret_cast<const uint16_t*>(shift);
  const uint16_t* scp = reinterpret_cast<const uint16_t*>(scale);
  uint16_t* mp = reinterpret_cast<uint16_t*>(m_buf);
  const dim3 grid((unsigned)((rows + 7) / 8)), block(256);
  cudaError_t e;
  switch (cols / 256) {
    case 1: e = launch_pdl(ln_stats_rows_kernel<1>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    case 2: e = launch_pdl(ln_stats_rows_kernel<2>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    case 4: e = launch_pdl(ln_stats_rows_kernel<4>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    case 8: e = launch_pdl(ln_stats_rows_kernel<8>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    case 12: e = launch_pdl(ln_stats_rows_kernel<12>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    case 16: e = launch_pdl(ln_stats_rows_kernel<16>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_quantize(m_buf, rows, cols, codes, scales, gs_out, amax, 1, s);
}

// the first half of launch_ln_modulate_quantize_via_m: m (bf16) and max|m|
// max-accumulated into amax (the caller zero-fills it)
cudaError_t launch_ln_modulate_m(const void* x, int64_t rows, int64_t cols, const void* shift, const void* scale,
                                 void* m_buf, float2* stats, float* amax, cudaStream_t s) {
  if (cols % 256) return cudaErrorInvalidValue;
  const uint16_t* xp = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* shp = reinterpret_cast<const uint16_t*>(shift);
  const uint16_t* scp = reinterpret_cast<const uint16_t*>(scale);
  uint16_t* mp = reinterpret_cast<uint16_t*>(m_buf);
  const dim3 grid((unsigned)((rows + 7) / 8)), block(256);
  switch (cols / 256) {
    case 1: return launch_pdl(ln_stats_rows_kernel<1>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    case 2: return launch_pdl(ln_stats_rows_kernel<2>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    case 4: return launch_pdl(ln_stats_rows_kernel<4>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    case 8: return launch_pdl(ln_stats_rows_kernel<8>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    case 12: return launch_pdl(ln_stats_rows_kernel<12>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    case 16: return launch_pdl(ln_stats_rows_kernel<16>, grid, block, 0, s, xp, rows, shp, scp, stats, amax, mp);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fp8_cast(const void* x, int64_t T, int64_t ncols, int64_t ld, const float* amax, void* out,
                            float* scales_out, cudaStream_t s) {
  if (ncols / 128 > kFp8MaxHeads) return cudaErrorInvalidValue;
  return launch_pdl(fp8_cast_kernel, dim3(grid_for(T * (ncols / 16), 256)), dim3(256), 0, s,
                    reinterpret_cast<const uint16_t*>(x), T, ncols, ld, amax, reinterpret_cast<uint8_t*>(out),
                    scales_out, rcp64((uint64_t)(ncols / 16)));
}

cudaError_t launch_rope_table(int64_t n_text, int64_t gh, int64_t gw, int64_t n_ref, double theta, float* cs,
                              cudaStream_t s) {
  const int64_t T = n_text + (1 + n_ref) * gh * gw;
  const int64_t n = T * 64;
  return launch_pdl(rope_table_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, n_text, gh, gw, n_ref,
                    theta, reinterpret_cast<float2*>(cs));
}

}  // namespace kl
