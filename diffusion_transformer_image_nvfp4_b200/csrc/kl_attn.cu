// kl_attn.cu -- flash-style joint attention on tcgen05 tensor cores, FP8
// (E4M3, per-head scales) or BF16 inputs, fp32 accumulation in TMEM.
//
// Joint attention: every text, noisy-image and reference token attends to all
// tokens of the concatenated sequence ([P4] "Welcome FLUX.3 Image Klein in
// Diffusers", Two-Stage Processing; [P2] "FLUX.3 Image Klein Brings 2-Second AI
// Image Generation to Diffusers", Summary).  FP8 Q/K/V: [P1] "Optimizing FLUX 3
// Image Klein inference on NVIDIA Blackwell GPUs", How it works: the quantized
// attention takes its query, key and value in FP8.
//
// One CTA = QT query tiles of 128 rows of one head (FP8: QT = 2, BF16: 1):
//  * warp 0 lane 0 -- TMA: the Q tiles once, then K and V tiles of 128 keys
//    into a ring (FP8: 3 stages, BF16: 2), 128-byte swizzle;
//  * warp 1 lane 0 -- MMA: per key tile j and query tile t, S_t = Q_t K_j^T
//    into TMEM; then O_t += P_t V_{j-1} (V read MN-major straight from its
//    row-major tile) for the previous key tile, so the tensor core computes
//    the next scores while the softmax warps exponentiate;
//  * 8 softmax warps per query tile: two per 32-row TMEM lane group, each
//    thread owning one query row and 64 of the 128 score columns (four
//    softmax warps per SM sub-partition hide the exponent and conversion
//    latencies).  Both halves of a row reduce the row maximum over all 128
//    scores (the other half's columns are read from TMEM for that only), so
//    they take the same decisions without exchanging anything; the running
//    maximum m is only moved (and O, l rescaled in place -- O in TMEM after
//    the previous P.V has landed) when a tile's maximum exceeds m by more
//    than TAU (log2 units), so p = 2^(s*c - m) <= 2^TAU; p * P_SCALE is
//    rounded to E4M3 (BF16: bf16) and written to a double-buffered smem P
//    tile in the MMA's K-major swizzled layout; each half sums its unrounded
//    p * P_SCALE, and the halves' sums are added once at the end.
//    Finally O = O_tmem / l (FP8: times s_v), bf16, and a tensor amax.
// TMEM per query tile: S [128 cols] + O [128 cols].
//
// Sol-Attention ([P1] How it works: less important token pairs are skipped
// by a sparsity threshold): with a key-tile list (kl_sol_select) each CTA
// visits only the key tiles listed for its query block, in ascending order;
// every role counts its iterations the same way, so the ring and barrier
// phases are those of a dense run over fewer tiles.
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

struct AttnParams {
  int64_t T;
  int H;
  int n_kv;
  float c_log2;  // log2(e)/sqrt(128); FP8: times sq*sk (per head, in the kernel)
  const float* sq;
  const float* sk;
  const float* sv;
  uint16_t* out;
  float* amax;
  const int* kv_list;  // nullable: per (head, query block) [count, tile indices...], n_kv + 1 ints
  // partial results (VC-Attention repair): all nullable / 0 by default
  float2* ml_out;      // [T, H]: per row the reference maximum m and the mass l (sum 2^(t-m) of the visited keys)
  float* o32;          // [T, H*128] fp32: O written here (normalised, FP8: times s_v) instead of bf16 to out
  int empty_ok;        // a list count of 0 is allowed: the CTA only writes ml_out = (-inf, 0) for its rows
  const int* work;     // nullable: CTA i takes item work[i] = h * gridDim.x + qblk if i < *work_count, else exits
  const int* work_count;
};

template <bool FP8>
struct AttnCfg {
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int QT = FP8 ? 2 : 1;           // query tiles per CTA
  static constexpr int TILE = 128 * 128 * ELEM;    // Q, K, V or P tile bytes
  static constexpr int NS = FP8 ? 3 : 2;           // K/V ring stages
  static constexpr int KSTEPS = FP8 ? 4 : 8;       // MMA K = 32 (e4m3) or 16 (bf16)
  static constexpr float TAU = FP8 ? 4.0f : 8.0f;  // lazy-rescale threshold, log2 units
  static constexpr float P_SCALE = FP8 ? 16.0f : 1.0f;  // p * P_SCALE <= 2^(TAU+4) <= 448
  static constexpr float LOG2_P_SCALE = FP8 ? 4.0f : 0.0f;
  static constexpr int SPLIT = 2;                  // softmax warps per 32 query rows
  static constexpr int COLS = 128 / SPLIT;         // score / output columns per softmax thread
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = QT * TILE;
  static constexpr int P_OFF = KV_OFF + NS * 2 * TILE;
  static constexpr int BAR_OFF = P_OFF + QT * 2 * TILE;
  static constexpr int L_OFF = BAR_OFF + 512;      // partial row sums, QT x SPLIT x 128 fp32
  static constexpr int SOFTMAX_THREADS = QT * 128 * SPLIT;
  static constexpr int PV_WARP = 2 + SOFTMAX_THREADS / 32;  // after the softmax warps
  static constexpr int THREADS = 64 + SOFTMAX_THREADS + 32;
  static constexpr uint32_t TMEM_COLS = QT * 256;
  static constexpr int SMEM_BYTES = L_OFF + QT * SPLIT * 128 * 4 + 1024;
  static_assert(SMEM_BYTES <= 232448, "smem budget");
};

// entry j of a key-tile list, clamped to the tiles that exist
__device__ __forceinline__ int tile_index(const int* list, int j, int n_kv) {
  const int t = __ldg(list + 1 + j);
  return t < 0 ? 0 : (t >= n_kv ? n_kv - 1 : t);
}

template <bool FP8>
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  tma_load_2d(dst, map, x, y, bar);
  if (!FP8) tma_load_2d(dst + 16384, map, x + 64, y, bar);
}

template <bool FP8, bool SPARSE>
__global__ void __launch_bounds__(AttnCfg<FP8>::THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const AttnParams p) {
  using C = AttnCfg<FP8>;
  constexpr int QT = C::QT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;                    // 1
  uint64_t* kv_full = q_full + 1;             // NS
  uint64_t* kv_empty = kv_full + C::NS;       // NS
  uint64_t* s_full = kv_empty + C::NS;        // QT
  uint64_t* s_empty = s_full + QT;            // QT
  uint64_t* p_full = s_empty + QT;            // QT x 2
  uint64_t* p_empty = p_full + 2 * QT;        // QT x 2
  uint64_t* o_done = p_empty + 2 * QT;        // QT: one phase per P.V
  uint64_t* o_last = o_done + QT;             // QT: the last P.V only
  uint64_t* drain = o_last + QT;              // 2: S issuer, P.V issuer
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int qblk = blockIdx.x, h = blockIdx.y;
  if (SPARSE && p.work) {
    // a compacted work list: the items are known only once the previous
    // kernel is done, and a CTA past the count leaves before any setup
    pdl_wait();
    const int i = blockIdx.y * gridDim.x + blockIdx.x;
    if (i >= __ldg(p.work_count)) return;
    const int item = __ldg(p.work + i);
    qblk = item % gridDim.x;
    h = item / gridDim.x;
  }
  // dense: key tiles 0..n_kv-1; sparse: the listed ones (read after pdl_wait)
  const int* kv_tiles = SPARSE ? p.kv_list + ((int64_t)h * gridDim.x + qblk) * (p.n_kv + 1) : nullptr;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);  // K read by the S issuer, V by the P.V issuer
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_empty[t], 4 * C::SPLIT);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_last[t], 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&p_full[2 * t + b], 4 * C::SPLIT);
        mbar_init(&p_empty[2 * t + b], 1);
      }
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
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
  int n = p.n_kv;
  if constexpr (SPARSE) {
    n = __ldg(kv_tiles);
    // at least one tile (the last P.V signals the epilogue), unless empty lists are allowed
    const int lo = p.empty_ok ? 0 : 1;
    n = n < lo ? lo : (n > p.n_kv ? p.n_kv : n);
  }
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* kv_smem = smem + C::KV_OFF;
  uint8_t* p_smem = smem + C::P_OFF;

  if (warp == 0) {
    // -------------------------------------------------------------- TMA
    // the whole warp runs the loop; one elected lane issues
    if (elect_one()) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      mbar_arrive_expect_tx(q_full, QT * C::TILE);
      for (int t = 0; t < QT; ++t) tma_tile<FP8>(q_smem + t * C::TILE, &tq, h * 128, (qblk * QT + t) * 128, q_full);
    }
    __syncwarp();
    int issued = 0;
    bool ok = true;
    int jt_next = SPARSE ? tile_index(kv_tiles, 0, p.n_kv) : 0;  // list entries are read one tile ahead
    for (int j = 0; j < n; ++j) {
      const int jt = SPARSE ? jt_next : j;
      if (SPARSE && j + 1 < n) jt_next = tile_index(kv_tiles, j + 1, p.n_kv);
      const int s = j % C::NS;
      if (!warp_wait(&kv_empty[s], ((uint32_t)(j / C::NS) & 1u) ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      if (elect_one()) {
        uint8_t* ks = kv_smem + s * 2 * C::TILE;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::TILE);
        tma_tile<FP8>(ks, &tk, h * 128, jt * 128, &kv_full[s]);
        tma_tile<FP8>(ks + C::TILE, &tv, h * 128, jt * 128, &kv_full[s]);
      }
      __syncwarp();
      ++issued;
    }
    if (lane == 0) {
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
  } else if (warp == 1 || warp == C::PV_WARP) {
    // ------------------------------------------------------- MMA issuers
    // Two warps issue to the tensor core: warp 1 the scores S_t(j) = Q_t K_j^T
    // (waiting only for K_j and for the softmax to have read S_t(j-1)), the
    // P.V warp O_t += P_t(j) V_j (waiting for P_t(j)).  The scores of the
    // next key tile therefore never queue behind a P.V that waits for the
    // softmax.  Each warp commits its own barriers; a K/V stage is released
    // by one arrival from each.  One elected lane issues; smem descriptors are
    // built once and advanced by offsets (16-byte units).
    const bool s_issuer = warp == 1;
    constexpr uint32_t id_qk = FP8 ? idesc_e4m3(128, 128, 0) : idesc_bf16(128, 128, 0);
    constexpr uint32_t id_pv = FP8 ? idesc_e4m3(128, 128, 1) : idesc_bf16(128, 128, 1);
    constexpr uint64_t TILE16 = (uint64_t)(C::TILE >> 4);
    const uint64_t q_desc0 = smem_desc(smem_u32(q_smem), 16, 1024, kLayoutSw128);
    const uint64_t k_desc0 = smem_desc(smem_u32(kv_smem), 16, 1024, kLayoutSw128);
    const uint64_t v_desc0 = smem_desc(smem_u32(kv_smem + C::TILE), 16384, 1024, kLayoutSw128);
    const uint64_t p_desc0 = smem_desc(smem_u32(p_smem), 16, 1024, kLayoutSw128);
    bool ok = !s_issuer || warp_wait(q_full, 0, abort_flag);
    for (int j = 0; ok && j < n; ++j) {
      const int s = j % C::NS, b = j & 1;
      if (!warp_wait(&kv_full[s], (uint32_t)(j / C::NS) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      for (int t = 0; t < QT && ok; ++t) {
        if (s_issuer) {
          if (!warp_wait(&s_empty[t], ((uint32_t)j & 1u) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const uint64_t q_desc = q_desc0 + (uint64_t)t * TILE16;
            const uint64_t k_desc = k_desc0 + (uint64_t)(2 * s) * TILE16;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              // K-major step kk: FP8 32 bytes, BF16 16 elements (64-element halves 16 KB apart)
              const uint64_t off = FP8 ? (uint64_t)(kk * 2) : (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
              if (FP8)
                mma_f8(tmem + t * 256, q_desc + off, k_desc + off, id_qk, kk > 0);
              else
                mma_f16(tmem + t * 256, q_desc + off, k_desc + off, id_qk, kk > 0);
            }
            tc_commit(&s_full[t]);
          }
          __syncwarp();
        } else {
          if (!warp_wait(&p_full[2 * t + b], (uint32_t)(j >> 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const uint64_t p_desc = p_desc0 + (uint64_t)(2 * t + b) * TILE16;
            const uint64_t v_desc = v_desc0 + (uint64_t)(2 * s) * TILE16;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const uint64_t off = FP8 ? (uint64_t)(kk * 2) : (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
              // MN-major V: step kk covers keys [kk*R, kk*R + R), R = 32 (FP8) / 16 (BF16) rows of 128 B
              const uint64_t voff = (uint64_t)(kk * (FP8 ? 32 : 16) * 8);
              if (FP8)
                mma_f8(tmem + t * 256 + 128, p_desc + off, v_desc + voff, id_pv, (j | kk) != 0);
              else
                mma_f16(tmem + t * 256 + 128, p_desc + off, v_desc + voff, id_pv, (j | kk) != 0);
            }
            tc_commit(&o_done[t]);
            tc_commit(&p_empty[2 * t + b]);
            if (j == n - 1) tc_commit(&o_last[t]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      // this warp's reads of stage s (K or V of tile j) are done once its
      // MMAs so far have completed
      if (elect_one()) tc_commit(&kv_empty[s]);
      __syncwarp();
    }
    uint64_t* my_drain = &drain[s_issuer ? 0 : 1];
    if (elect_one()) tc_commit(my_drain);
    __syncwarp();
    volatile int no_abort = 0;
    warp_wait(my_drain, 0, &no_abort);
  } else {
    // ------------------------------------------------------------ softmax
    constexpr int COLS = C::COLS;
    const int g = (warp - 2) >> 2;        // 4 consecutive warps cover the 4 lane groups
    const int t = g / C::SPLIT;           // query tile of this warp
    const int part = g % C::SPLIT;        // its score / output columns [part*COLS, +COLS)
    const int quad = warp & 3;            // TMEM lane group this warp may access
    const int r = quad * 32 + lane;       // query row inside the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(t * 256);
    const uint32_t s_tmem = lane_base, o_tmem = lane_base + 128 + (uint32_t)(part * COLS);
    float c = p.c_log2;
    if (FP8) c *= __ldg(p.sq + h) * __ldg(p.sk + h);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int jt_next = SPARSE ? tile_index(kv_tiles, 0, p.n_kv) : 0;  // list entries are read one tile ahead
    for (int j = 0; j < n; ++j) {
      const int jt = SPARSE ? jt_next : j;
      if (SPARSE && j + 1 < n) jt_next = tile_index(kv_tiles, j + 1, p.n_kv);
      if (!warp_wait(&s_full[t], (uint32_t)j & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t rem = p.T - (int64_t)jt * 128;
      float sc[COLS];
      float mk[8];
      // row maximum over all 128 scores: first the other half's columns
      // (read for the maximum only), then this thread's own, kept in sc
#pragma unroll
      for (int k = 0; k < 8; ++k) mk[k] = -INFINITY;
#pragma unroll
      for (int pass = C::SPLIT == 2 ? 0 : 1; pass < 2; ++pass) {
        const int col0 = pass == 0 ? (1 - part) * COLS : part * COLS;
        if constexpr (COLS == 128)
          tmem_ld128(s_tmem + col0, sc);
        else
          tmem_ld64(s_tmem + col0, sc);
        if (rem < 128) {
#pragma unroll
          for (int i = 0; i < COLS; ++i)
            if (col0 + i >= rem) sc[i] = -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < COLS; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mk[k] = max3f(mk[k], sc[i + 2 * k], sc[i + 2 * k + 1]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[t]);
      float mx = max3f(max3f(mk[0], mk[1], mk[2]), max3f(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7])) * c;
      // this P buffer was last read by P.V of key tile j-2: once it is free,
      // every P.V up to j-2 has landed
      const int b = j & 1;
      if (!warp_wait(&p_empty[2 * t + b], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const bool move = mx > m + C::TAU;
      if (__any_sync(0xffffffffu, move)) {
        // move the reference maximum of the rows that need it and rescale
        // their O columns (in TMEM, after P.V of tile j-1 has landed) and l
        // by 2^(m_old - m_new).  TMEM loads/stores are warp-wide, so the
        // whole warp takes this path; rows that do not move use a factor of 1.
        const float alpha = move ? ex2_approx(m - mx) : 1.0f;
        if (j > 0) {
          if (!warp_wait(&o_done[t], (uint32_t)(j - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < COLS / 32; ++cc) {
            float o[32];
            tmem_ld32(o_tmem + cc * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(o_tmem + cc * 32, o);
          }
          tc_fence_before();
        }
        l *= alpha;
        if (move) m = mx;
      }
      uint8_t* prow = p_smem + (2 * t + b) * C::TILE + r * 128;
      // p * P_SCALE = 2^(s*c - (m - log2 P_SCALE)); packed fp32x2 FMAs, and
      // the row sum (of the scaled p) in 4 independent packed chains
      const uint64_t c2 = pack_f32x2(c, c);
      const float mb = -(m - C::LOG2_P_SCALE);
      const uint64_t mb2 = pack_f32x2(mb, mb);
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int i = 0; i < COLS; i += 2) {
        const uint64_t x2 = fma_f32x2(pack_f32x2(sc[i], sc[i + 1]), c2, mb2);
        float lo, hi;
        unpack_f32x2(x2, lo, hi);
        sc[i] = ex2_approx(lo);
        sc[i + 1] = ex2_approx(hi);
        acc2[(i >> 1) & 3] = add_f32x2(acc2[(i >> 1) & 3], pack_f32x2(sc[i], sc[i + 1]));
      }
      float a0, a1, b0, b1;
      unpack_f32x2(add_f32x2(acc2[0], acc2[1]), a0, a1);
      unpack_f32x2(add_f32x2(acc2[2], acc2[3]), b0, b1);
      const float rowsum = (a0 + a1) + (b0 + b1);
      if (FP8) {
        // this thread's COLS bytes of the 128-byte P row: 16-byte chunks
        // part*COLS/16 .., stored at chunk ^ (r & 7) (128-byte swizzle)
#pragma unroll
        for (int chunk = 0; chunk < COLS / 16; ++chunk) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float* x = sc + chunk * 16 + q * 4;
            w[q] = f32x2_to_e4m3x2(x[0], x[1]) | (f32x2_to_e4m3x2(x[2], x[3]) << 16);
          }
          const int gc = part * (COLS / 16) + chunk;
          *reinterpret_cast<uint4*>(prow + ((gc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
        // bf16 P row: two 16 KB halves of 64 elements; 16-byte chunk gc
#pragma unroll
        for (int chunk = 0; chunk < COLS / 8; ++chunk) {
          const float* x = sc + chunk * 8;
          const uint4 w = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                     pack_bf16x2(x[6], x[7]));
          const int gc = part * (COLS / 8) + chunk;
          *reinterpret_cast<uint4*>(prow + (gc >> 3) * 16384 + (((gc & 7) ^ (r & 7)) << 4)) = w;
        }
      }
      l += rowsum;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[2 * t + b]);
    }
    // the row sum is the sum of the halves' partial sums; every softmax
    // thread reaches this barrier (also after a failed wait)
    float* lsm = reinterpret_cast<float*>(smem + C::L_OFF);
    lsm[(t * C::SPLIT + part) * 128 + r] = l;
    asm volatile("bar.sync 1, %0;" ::"n"(C::SOFTMAX_THREADS) : "memory");
    float lsum = 0.f;
#pragma unroll
    for (int q = 0; q < C::SPLIT; ++q) lsum += lsm[(t * C::SPLIT + q) * 128 + r];
    // epilogue: O / l (FP8: times s_v), bf16 (or fp32), tensor amax
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n > 0) ok = warp_wait(&o_last[t], 0, abort_flag);
    const int64_t row = ((int64_t)qblk * QT + t) * 128 + r;
    const bool valid_row = ok && n > 0 && row < p.T;
    if (p.ml_out && part == 0 && ok && row < p.T)  // the mass of the visited keys: lsum / P_SCALE * 2^m
      p.ml_out[row * p.H + h] = n > 0 ? make_float2(m, lsum * (1.0f / C::P_SCALE)) : make_float2(-INFINITY, 0.f);
    float scale = 1.0f / lsum;  // l sums p * P_SCALE, so this also undoes P_SCALE
    if (FP8) scale *= __ldg(p.sv + h);
    float amax = 0.f;
    if (ok && n > 0 && p.o32) {
      tc_fence_after();
      float4* dst = reinterpret_cast<float4*>(p.o32 + row * (int64_t)p.H * 128 + h * 128 + part * COLS);
#pragma unroll 1
      for (int cc = 0; cc < COLS / 32; ++cc) {
        float o[32];
        tmem_ld32(o_tmem + cc * 32, o);
        if (valid_row)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[cc * 8 + q] = make_float4(o[4 * q] * scale, o[4 * q + 1] * scale, o[4 * q + 2] * scale,
                                          o[4 * q + 3] * scale);
      }
    } else if (ok && n > 0) {
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * (int64_t)p.H * 128 + h * 128 + part * COLS);
#pragma unroll 1
      for (int cc = 0; cc < COLS / 32; ++cc) {
        float o[32];
        tmem_ld32(o_tmem + cc * 32, o);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i] = bf16_bits_to_f32(f32_to_bf16_bits(o[q * 8 + i] * scale));
            amax = fmaxf(amax, fabsf(x[i]));
          }
          if (valid_row)
            dst[cc * 4 + q] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                         pack_bf16x2(x[6], x[7]));
        }
      }
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
    tmem_dealloc(tmem, C::TMEM_COLS);
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
  p.kv_list = a.kv_list;
  p.ml_out = a.ml_out;
  p.o32 = a.o32;
  p.empty_ok = a.empty_ok;
  p.work = a.work;
  p.work_count = a.work_count;
  if (a.work && !a.kv_list) return cudaErrorInvalidValue;
  const int qblocks = (int)((a.T + 128 * C::QT - 1) / (128 * C::QT));
  dim3 grid((unsigned)qblocks, (unsigned)a.H);
  auto kern = a.kv_list ? attn_kernel<FP8, true> : attn_kernel<FP8, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM_BYTES, s, tq, tk, tv, p);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  return a.fp8 ? launch_t<true>(a, s) : launch_t<false>(a, s);
}

}  // namespace kl
