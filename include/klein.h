/*
 * klein.h -- C ABI of libklein.so: the forward pass of one FLUX-3-Image-Klein-
 * style joint transformer block on NVIDIA B200 (sm_100a), built from NVFP4
 * block-scaled GEMMs (tcgen05, TMEM accumulators) with fused RoPE / SwiGLU /
 * gated-residual epilogues and a flash-style FP8 (or BF16) joint attention.
 *
 * Sources (page titles and sections):
 *  [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs",
 *       How it works: NVFP4 weights and activations; GEMM kernels with the
 *       SwiGLU gate and the rotary embedding folded in; attention on FP8 Q/K/V.
 *  [P2] "FLUX.3 Image Klein Brings 2-Second AI Image Generation to Diffusers",
 *       Summary: 28 joint blocks run over one sequence of text, target-image
 *       and reference-image tokens; each 1024x1024 reference brings another
 *       4,096 tokens.
 *  [P4] "Welcome FLUX.3 Image Klein in Diffusers", Architecture and Technical
 *       Deep Dive: 64x64 = 4,096 tokens per 1024x1024 image; 3072-wide
 *       transformer; joint blocks attend over the concatenated streams.
 * The pages do not define the NVFP4 encoding or the block's wiring; the
 * readings implemented here are stated at each entry point.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  Nothing on
 *    this path allocates or frees device memory; scratch comes from a caller
 *    workspace whose size a *_workspace_size call returns.
 *  - Every call is asynchronous on the given CUDA stream (cudaStream_t passed
 *    as void*; NULL = legacy default stream) and returns a kl_status.  Host-side
 *    argument checks return an error before anything is enqueued.  Device-side
 *    conditions (a bounded wait that expired, a non-finite input) are recorded
 *    in a per-device status word that kl_device_status() reads.
 *  - Shapes are int64_t, row-major, rows x columns.  bf16 tensors are passed
 *    as uint16_t bit patterns.  Pointers must be 16-byte aligned (128-byte
 *    aligned for operands read by TMA: NVFP4 codes, FP8/bf16 Q/K/V).
 *  - No C++ exception crosses this ABI.
 */
#ifndef KLEIN_H
#define KLEIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int kl_status;
#define KL_OK 0
#define KL_ERR_INVALID_ARG 1       /* null pointer, bad enum, bad stride */
#define KL_ERR_UNSUPPORTED_SHAPE 2 /* a dimension this library does not tile */
#define KL_ERR_MISALIGNED 3        /* pointer alignment rule broken */
#define KL_ERR_WORKSPACE 4         /* workspace missing or too small */
#define KL_ERR_CUDA 5              /* a CUDA runtime/driver call failed */
#define KL_ERR_DEVICE_TIMEOUT 6    /* a bounded device wait expired (device status) */
#define KL_ERR_ARCH 7              /* current device is not sm_100 */
#define KL_ERR_NONFINITE 8         /* NaN/Inf met by an amax pass (device status) */

/* Human-readable name of a status code (static string). */
const char* kl_status_string(kl_status s);
/* Text of the last CUDA error seen by this library on this thread ("" if none). */
const char* kl_last_cuda_error(void);
/* Library version, major*10000 + minor*100 + patch. */
int kl_version(void);

/*
 * Device status word of the current device.  Synchronises the device, then
 * returns KL_OK, KL_ERR_DEVICE_TIMEOUT or KL_ERR_NONFINITE (the first recorded
 * condition, timeouts first).  If `clear` is non-zero the word is reset to 0.
 * Kernels never trap: an expired wait sets the word and the kernel returns.
 */
kl_status kl_device_status(int clear);

/*
 * kl_selftest_wait_timeout -- exercises the failure path every kernel shares:
 * one warp waits on an mbarrier that nothing ever arrives on, with the
 * library's bounded wait given limit_ns (1 us .. 1 s) instead of its usual
 * 2 s.  The wait runs out, the kernel records KL_ERR_DEVICE_TIMEOUT in the
 * device status word (read it with kl_device_status) and returns; nothing
 * traps and the context stays usable.  waited_out (device int, nullable)
 * receives 0 when the wait gave up, 1 if it had completed.  Asynchronous on
 * stream; KL_ERR_INVALID_ARG for a limit outside the range.
 */
kl_status kl_selftest_wait_timeout(uint64_t limit_ns, int* waited_out, void* stream);

/* ------------------------------------------------------------------------
 * NVFP4 tensors
 *
 * Reading of NVFP4 ([P1] How it works names the format, not the encoding):
 * E2M1 element codes, one unsigned E4M3 decode scale per 16 consecutive
 * elements of a row, one fp32 per-tensor decode scale gs; decoded value =
 * e2m1(code) * e4m3(scale) * gs.  Codes: uint8 [R, C/2], element 2i in the
 * low nibble of byte i.  Scales ("scale layouts"):
 *   KL_SCALE_LINEAR : uint8 [R, C/16] row-major;
 *   KL_SCALE_MMA    : the tcgen05 block-scale layout, padded to
 *                     ceil(R/128)*128 rows: 512-byte atoms, one per
 *                     (128-row block rb, 64-column block kb), atom index
 *                     rb*(C/64) + kb, byte (r%32)*16 + ((r/32)%4)*4 + (c/16)%4
 *                     inside the atom.  Padding rows hold scale 0.
 * ---------------------------------------------------------------------- */
#define KL_SCALE_LINEAR 0
#define KL_SCALE_MMA 1
#define KL_GLOBAL_SCALE_GIVEN 2    /* use *global_scale as gs instead of amax/2688 */
#define KL_ROWS_SWIGLU_INTERLEAVE 4/* output row r reads input row perm(r), see below */
#define KL_AMAX_GIVEN 8            /* kl_quantize_nvfp4: the workspace's first fp32 word already
                                      holds amax_t (e.g. a max all-reduced over ranks); the amax
                                      pass is skipped and gs = amax_t/2688 as usual */

/* Bytes of the scale array for an [R, C] NVFP4 tensor in the given layout. */
size_t kl_nvfp4_scales_bytes(int64_t rows, int64_t cols, int layout);

/* Workspace bytes kl_quantize_nvfp4 needs (an amax word). */
size_t kl_quantize_workspace_size(void);

/*
 * kl_quantize_nvfp4 -- NVFP4-encode a bf16 tensor x [rows, cols].
 * cols % 16 == 0 (% 64 for KL_SCALE_MMA).  Steps, each an IEEE fp32 operation
 * rounded to nearest even: amax_t = max|x|; gs = amax_t/2688 (1 if amax_t==0)
 * unless KL_GLOBAL_SCALE_GIVEN; inv = 1/(6*gs); per 16-block
 * sb = e4m3_rne_satfinite(amax_b*inv) (0 if amax_b==0); S = e4m3(sb)*gs;
 * code_i = e2m1_rne_satfinite(x_i * (1/S)) (all 0 if S==0).
 * Output: codes [rows, cols/2]; scales (layout from flags); *global_scale = gs
 * (device fp32; read instead of written with KL_GLOBAL_SCALE_GIVEN).
 * KL_AMAX_GIVEN (not with KL_GLOBAL_SCALE_GIVEN): amax_t is read from the
 *   workspace's first fp32 word instead of computed from x.
 * KL_ROWS_SWIGLU_INTERLEAVE (rows % 128 == 0): output row r holds input row
 *   (r/128)*64 + (r%128)       if r%128 < 64   (gate half, rows [0, rows/2))
 *   rows/2 + (r/128)*64 + r%64 otherwise        (up half, rows [rows/2, rows))
 * i.e. each 128-row group is 64 gate rows followed by the matching 64 up rows,
 * the layout the SwiGLU GEMM epilogue expects for W1.
 * workspace: >= kl_quantize_workspace_size() bytes, 16-byte aligned.
 * Non-finite input is undefined; the amax pass records KL_ERR_NONFINITE.
 */
kl_status kl_quantize_nvfp4(const void* x_bf16, int64_t rows, int64_t cols,
                            void* codes, void* scales, float* global_scale, int flags,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * kl_ln_modulate_quantize_nvfp4 -- fused LayerNorm + adaLN modulation +
 * NVFP4 encode of x [rows, cols] bf16 (the pre-attention and pre-MLP step of
 * the block).  Reading ([P1]/[P2] do not define the wiring): LN over cols
 * with biased variance and eps 1e-6, no affine;
 * m = bf16(LN(x) * (1 + scale) + shift) with shift/scale bf16 [cols] shared by
 * all rows; then the kl_quantize_nvfp4 encoding of m (dynamic gs from amax of
 * m, scales in KL_SCALE_MMA layout).  m_out (nullable) receives m as bf16
 * [rows, cols] (a debug export).  cols % 64 == 0, cols <= 8192.
 * workspace: >= kl_ln_workspace_size(rows).
 */
size_t kl_ln_workspace_size(int64_t rows);
kl_status kl_ln_modulate_quantize_nvfp4(const void* x_bf16, int64_t rows, int64_t cols,
                                        const void* shift_bf16, const void* scale_bf16,
                                        void* codes, void* scales, float* global_scale,
                                        void* m_out_bf16, void* workspace, size_t ws_bytes,
                                        void* stream);

/*
 * Pieces for sequence-parallel callers, whose per-tensor scales must come
 * from a maximum over all ranks' tokens (a max all-reduce between the pieces):
 * kl_amax_bf16 -- *amax_out = max|x| over n bf16 values (n % 8 == 0, x 16-byte
 *   aligned); the word is overwritten.
 * kl_ln_modulate_bf16 -- the first half of the block's LayerNorm step:
 *   m = bf16(LN(x) * (1 + scale) + shift) as kl_ln_modulate_quantize_nvfp4
 *   defines it, written to m_out [rows, cols], and max|m| max-accumulated into
 *   *amax_out (caller zero-fills).  cols / 256 in {1, 2, 4, 8, 12, 16} (the
 *   widths the block computes m this way).  Encoding m with
 *   kl_quantize_nvfp4(KL_SCALE_MMA | KL_AMAX_GIVEN) and the global amax gives
 *   the block's operand bit for bit.  workspace: >= kl_ln_workspace_size(rows),
 *   256-byte aligned (row statistics).
 */
kl_status kl_amax_bf16(const void* x_bf16, int64_t n, float* amax_out, void* stream);
kl_status kl_ln_modulate_bf16(const void* x_bf16, int64_t rows, int64_t cols, const void* shift_bf16,
                              const void* scale_bf16, void* m_out_bf16, float* amax_out, void* workspace,
                              size_t ws_bytes, void* stream);

/*
 * kl_ln_modulate_quantize_nvfp4_static -- the same computation, arguments and
 * outputs as kl_ln_modulate_quantize_nvfp4, without the workspace.  The pages
 * have no counterpart: this exists for callers that cannot give the library
 * any device memory, e.g. a host that plans and owns the whole device pool up
 * front and forbids allocations after start-up, or a plugin interface that
 * passes only input and output buffers.  The call allocates nothing (no
 * cudaMalloc / cudaFree, no allocating library routine).
 *  - Scratch (one amax word + 8 bytes of LayerNorm statistics per row) lives
 *    in a fixed device array compiled into the library:
 *    256 + 8 * KL_STATIC_SCRATCH_MAX_ROWS bytes (= 262,400), held on every GPU
 *    that loads the library until the process exits.
 *  - rows > KL_STATIC_SCRATCH_MAX_ROWS is rejected with KL_ERR_WORKSPACE
 *    (kl_last_cuda_error() names the limit) before anything is enqueued.
 *  - The first call on a device looks up that array's device address
 *    (cudaGetSymbolAddress) with the device current; make that first call
 *    before any stream capture.  The address is kept per device with the id
 *    of the context it belongs to and looked up again when the device's
 *    context has been replaced (e.g. after cudaDeviceReset), so such a call
 *    is again a first call.
 *  - All calls share the one array and it keeps the last call's contents;
 *    each call zeroes the amax word on its stream before use.  Calls that
 *    overlap on the same GPU (e.g. issued on two streams) race on it:
 *    serialise them.  Each device has its own copy of the array.
 */
#define KL_STATIC_SCRATCH_MAX_ROWS 32768
kl_status kl_ln_modulate_quantize_nvfp4_static(const void* x_bf16, int64_t rows, int64_t cols,
                                               const void* shift_bf16, const void* scale_bf16,
                                               void* codes, void* scales, float* global_scale,
                                               void* m_out_bf16, void* stream);

/* An NVFP4 GEMM operand: codes [R, K/2], scales in KL_SCALE_MMA layout,
 * global decode scale (device fp32). */
typedef struct kl_nvfp4_tensor {
  const void* codes;
  const void* scales;
  const float* global_scale;
} kl_nvfp4_tensor;

/* GEMM epilogues */
#define KL_EPI_NONE 0            /* out[m,n] = acc (bf16 or fp32)                   */
#define KL_EPI_QKV_ROPE 1        /* q|k|v split, RoPE on q and k, per-head amax     */
#define KL_EPI_SWIGLU 2          /* h = silu(gate)*up over interleaved rows, amax   */
#define KL_EPI_GATED_RESIDUAL 3  /* out = residual + gate[n] * acc                  */

#define KL_OUT_BF16 0
#define KL_OUT_F32 1

typedef struct kl_epilogue {
  int kind;               /* KL_EPI_* */
  int out_dtype;          /* KL_OUT_BF16 (all kinds) or KL_OUT_F32 (KL_EPI_NONE only) */
  void* out;              /* NONE/GATED_RESIDUAL/QKV_ROPE: [M, N]; SWIGLU: [M, N/2]; row-major */
  const float* rope_cs;   /* QKV_ROPE: fp32 (cos, sin) table in the kl_rope_table layout, M tokens, 32-byte aligned */
  const void* gate;       /* GATED_RESIDUAL: bf16 [N] */
  const void* residual;   /* GATED_RESIDUAL: bf16 [M, N] (may alias nothing else written) */
  float* amax_out;        /* QKV_ROPE: [3*N/384] per (q|k|v, head) max|out|; SWIGLU: [1].
                             Max-accumulated as non-negative floats: caller zero-fills. */
  int tile;               /* KL_TILE_AUTO (0), or a forced output-tile variant (tests, tuning) */
} kl_epilogue;

/* Output-tile variants of kl_gemm_nvfp4_fused.  AUTO: 2-SM pair tiles of
 * 256 x 256 (N % 256 == 0) or 256 x 128 when M > 128, else one-CTA 128 x 256
 * (N % 256 == 0) or 128 x 128.  Every variant computes the same sums in the
 * same K order per output, so all give bit-identical results.  A 256-wide
 * variant with N % 256 != 0 returns KL_ERR_UNSUPPORTED_SHAPE. */
#define KL_TILE_AUTO 0
#define KL_TILE_1CTA_128x128 1
#define KL_TILE_1CTA_128x256 2
#define KL_TILE_2SM_256x128 3
#define KL_TILE_2SM_256x256 4

/*
 * kl_gemm_nvfp4_fused -- C[M,N] = gA*gW * sum_k dec(A)[m,k] * dec(W)[n,k]
 * (both operands K-major, "y = x W^T") on tcgen05 block-scaled FP4 tensor
 * cores, followed by the epilogue:
 *  NONE           out = C.
 *  QKV_ROPE       N = 3*D, D = 128*H.  Columns [0,D) are q, [D,2D) k, [2D,3D)
 *                 v; head h = columns [128h, 128h+128) of each.  q and k pairs
 *                 (2j, 2j+1) are rotated (a,b) -> (a c - b s, a s + b c) with
 *                 (c, s) = rope_cs[j/4, m, j%4]; out is bf16 [M, 3D]; amax_out[r*H+h]
 *                 receives the max |bf16 value| of region r (q,k,v), head h.
 *  SWIGLU         W holds 2F rows in the KL_ROWS_SWIGLU_INTERLEAVE order (each
 *                 128-row group: 64 gate rows then the matching 64 up rows);
 *                 out[m, f] = bf16(silu(g) * u), silu(g) = g / (1 + e^-g),
 *                 out is [M, F], F = N/2; amax_out[0] = max |out|.
 *  GATED_RESIDUAL out = bf16(residual + gate[n] * C).
 * Shapes: K % 64 == 0; N % 128 == 0 (N % 384 for QKV, % 256 for SWIGLU); any M >= 1.
 * ([P1] How it works: "kernels fuse ... SwiGLU activations and rotary position
 * embeddings"; the gated residual is the adaLN reading above.)
 */
kl_status kl_gemm_nvfp4_fused(const kl_nvfp4_tensor* A, const kl_nvfp4_tensor* W,
                              int64_t M, int64_t N, int64_t K, const kl_epilogue* epi,
                              void* stream);

/*
 * kl_rope_table -- fp32 (cos, sin) table [16, T, 4, 2] (groups of 4 pairs,
 * token within group: pair j of token t at cs_out[2*((j/4*T + t)*4 + j%4)];
 * 32-byte aligned rows of 4 pairs, so a consumer thread holding one token
 * reads 4 pairs with one 32-byte load) for the joint sequence
 * [text (n_text); noisy image (grid_h x grid_w, row-major); n_ref references
 * on grids of the same size].  Reading (RoPE theta 10000 on head dim 128,
 * interleaved pairs): text token i turns pair j by i*theta^(-2j/128); an
 * image-family token at (f, r, c) -- f = 0 for the noisy image, f = k for
 * reference k -- turns pairs [0,16) by f*theta^(-2u/32), [16,40) by
 * r*theta^(-2u/48), [40,64) by c*theta^(-2u/48) (u = pair index inside the
 * section).  Angles and cos/sin are evaluated in fp64 on the device and
 * rounded to fp32.  [P4] The VAE and Tokenization gives the 64x64 grid.
 */
typedef struct kl_token_layout {
  int64_t n_text;
  int64_t grid_h;
  int64_t grid_w;
  int64_t n_ref;
} kl_token_layout;
int64_t kl_layout_tokens(const kl_token_layout* layout);
kl_status kl_rope_table(const kl_token_layout* layout, float theta, float* cs_out, void* stream);

/*
 * kl_cast_fp8_per_head -- x bf16 [T, ncols] (row stride ld elements), cols in
 * heads of 128: s[h] = amax[h]/448 (1 if amax[h]==0) and
 * out[t, c] = e4m3_rne_satfinite(x[t,c] * (448/amax[h])), out row stride ld.
 * amax: fp32 [ncols/128] (e.g. the QKV epilogue's amax_out); scales_out: fp32
 * [ncols/128] decode scales.  ([P1] How it works: FP8 query/key/value.)
 */
kl_status kl_cast_fp8_per_head(const void* x_bf16, int64_t T, int64_t ncols, int64_t ld,
                               const float* amax, void* out_e4m3, float* scales_out,
                               void* stream);

/*
 * kl_joint_attention_fp8 -- O = softmax(Q K^T / sqrt(128)) V per head over all
 * T tokens (joint, unmasked: [P4] Two-Stage Processing; [P2] Summary).
 * q, k, v: [T, H, 128] with row stride ld elements (e.g. the three column
 * blocks of one [T, 3*H*128] buffer with ld = 3*H*128).
 *  KL_ATTN_FP8  : E4M3 inputs with per-head decode scales scale_q/k/v [H];
 *                 S = (q8.k8) * sq*sk.  Keys are taken in tiles of 128; per
 *                 query row a reference maximum m (log2 units) moves only when
 *                 a tile's maximum exceeds it by more than 4, and then the
 *                 partial output and row sum are rescaled, so p = 2^(s - m) <=
 *                 16; p * 16 is rounded to E4M3 and fed to the P.V MMA; the row
 *                 sum l uses the unrounded p; O = (P8.V8) * sv / (16 * l).
 *  KL_ATTN_BF16 : bf16 inputs, scales ignored (may be NULL); the same scheme
 *                 with threshold 8 and P rounded to bf16 (no extra scale).
 * out: bf16 [T, H*128] (row stride H*128).  amax_out (nullable): max|out| is
 * max-accumulated into it (caller zero-fills).  head_dim must be 128;
 * ld % 64 == 0.
 */
#define KL_ATTN_FP8 0
#define KL_ATTN_BF16 1
kl_status kl_joint_attention_fp8(const void* q, const void* k, const void* v, int64_t ld,
                                 const float* scale_q, const float* scale_k, const float* scale_v,
                                 int64_t T, int64_t H, int64_t head_dim, int precision,
                                 void* out_bf16, float* amax_out, void* stream);

/*
 * Sol-Attention ([P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA
 * Blackwell GPUs", How it works: sparse attention leaves out less important
 * token pairs by a sparsity threshold; What you can do: tau and a number of
 * initial dense denoising steps).  Readings (the pages give no more): pairs
 * are skipped one tensor-core tile at a time -- a query block (256 rows with
 * KL_ATTN_FP8, 128 with KL_ATTN_BF16: the rows one attention CTA owns)
 * against a key tile of 128 keys.  The estimate is
 *   s_hat = c * (qbar . kbar),
 * with qbar / kbar the means of the block's query rows / the tile's key rows
 * (valid rows only at a ragged end; for KL_ATTN_FP8 the unscaled E4M3 values)
 * and c = log2(e)/sqrt(128) (times sq[h]*sk[h] for KL_ATTN_FP8).  A tile is
 * kept when s_hat >= max over tiles - tau (the strongest is always kept;
 * tau = +inf keeps all).  Means and dots are fp32; the decision compares in
 * fp32, so estimates within a few fp32 ulps of the threshold may go either way.
 *
 * kl_sol_select: q, k as for kl_joint_attention_fp8 (row stride ld, a
 * multiple of 64; q and k 16-byte aligned).
 * kv_list (device, int32, kl_sol_list_ints(T, H, precision) entries): per head
 * h and query block b, at offset (h * n_qb + b) * (n_kt + 1) with n_qb =
 * ceil(T / rows_per_block), n_kt = ceil(T / 128): the count, then the kept
 * tile indices in ascending order.  workspace: >= kl_sol_workspace_size bytes,
 * 16-byte aligned (the block means).  tau >= 0 (NaN is rejected).
 *
 * kl_joint_attention_sparse: kl_joint_attention_fp8 where each query block
 * visits only the key tiles of its kv_list entry, in the given (ascending)
 * order, with the same steps; a count outside [1, n_kt] is clamped into it
 * and tile indices into [0, n_kt).  A list with every tile gives the dense
 * result bit for bit.
 */
size_t kl_sol_list_ints(int64_t T, int64_t H, int precision);
size_t kl_sol_workspace_size(int64_t T, int64_t H, int precision);
kl_status kl_sol_select(const void* q, const void* k, int64_t ld, const float* scale_q, const float* scale_k,
                        int64_t T, int64_t H, int precision, float tau, int* kv_list, void* workspace,
                        size_t ws_bytes, void* stream);
kl_status kl_joint_attention_sparse(const void* q, const void* k, const void* v, int64_t ld, const float* scale_q,
                                    const float* scale_k, const float* scale_v, int64_t T, int64_t H,
                                    int64_t head_dim, int precision, const int* kv_list, void* out,
                                    float* amax_out, void* stream);

/*
 * VC-Attention repair ([P1] "Optimizing FLUX 3 Image Klein inference on
 * NVIDIA Blackwell GPUs", How it works: VC-Attention adds a repair budget that
 * corrects the quantization errors of FP8 attention; Key details: a repair
 * budget of 0.005).  Readings (the pages give no more): the unit of repair is
 * the FP8 attention's tile pair, a query block of 256 rows against a key tile
 * of 128 keys, per head; budget b repairs R = floor(b * n_qb * n_kt) of a
 * head's n_qb * n_kt pairs (n_qb = ceil(T/256), n_kt = ceil(T/128)): those
 * with the largest estimated share of their query block's attention,
 *   w(b, j) = 2^(s_hat(b,j) - max_j') / sum_j' 2^(s_hat(b,j') - max_j'),
 *   s_hat = (qbar . kbar) * log2(e)/sqrt(128),
 * qbar / kbar the means of the block's bf16 query rows / the tile's bf16 key
 * rows (valid rows only); equal shares go to the lower (b, j) in row-major
 * order.  Shares are fp32, so pairs whose shares lie within fp32 rounding of
 * the R-th largest may go either way.  A repaired pair is computed from the
 * bf16 q, k, v: the query block's output is the exact merge of the FP8
 * attention over its other tiles and the BF16 attention over its repaired
 * tiles, O = (O_8 W_8 + O_16 W_16) / (W_8 + W_16), W the softmax mass of
 * each part.
 *
 * kl_vc_select: q, k bf16 [T, H, 128] (row stride ld, a multiple of 64;
 * 16-byte aligned), budget in [0, 1].  list_fp8 (kl_sol_list_ints(T, H,
 * KL_ATTN_FP8) ints): per (head, 256-row block) the tiles that are not
 * repaired; list_bf16 (kl_sol_list_ints(T, H, KL_ATTN_BF16) ints): per (head,
 * 128-row block) the repaired tiles of its 256-row block; both ascending, in
 * the kl_sol_select layout, counts may be 0.  workspace >=
 * kl_vc_workspace_size(T, H) bytes, 256-byte aligned.
 *
 * kl_joint_attention_vc: q8, k8, v8 E4M3 (row stride ld8) with scales sq, sk,
 * sv as for kl_joint_attention_fp8, and q, k, v their bf16 values (row stride
 * ld); the two lists from kl_vc_select.  out bf16 [T, H*128]; amax_out
 * (nullable) max-accumulates max|out| (caller zero-fills).  workspace >=
 * kl_vc_attention_workspace_size(T, H) bytes, 256-byte aligned (per row and
 * head the reference maximum and mass of both parts, the BF16 part's fp32
 * output, and the list of (head, 128-row block) items with repaired tiles:
 * the BF16 pass runs only those).  With budget 0 the result is
 * kl_joint_attention_fp8's bit for bit.
 */
size_t kl_vc_workspace_size(int64_t T, int64_t H);
kl_status kl_vc_select(const void* q, const void* k, int64_t ld, int64_t T, int64_t H, float budget, int* list_fp8,
                       int* list_bf16, void* workspace, size_t ws_bytes, void* stream);
size_t kl_vc_attention_workspace_size(int64_t T, int64_t H);
kl_status kl_joint_attention_vc(const void* q8, const void* k8, const void* v8, int64_t ld8, const float* scale_q,
                                const float* scale_k, const float* scale_v, const void* q, const void* k,
                                const void* v, int64_t ld, int64_t T, int64_t H, int64_t head_dim,
                                const int* list_fp8, const int* list_bf16, void* out, float* amax_out,
                                void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The joint block
 * ---------------------------------------------------------------------- */
typedef struct kl_block_weights {
  kl_nvfp4_tensor wqkv; /* [3D, D]  rows: q (D), k (D), v (D)                      */
  kl_nvfp4_tensor wo;   /* [D, D]                                                  */
  kl_nvfp4_tensor w1;   /* [2F, D] in KL_ROWS_SWIGLU_INTERLEAVE order (gate, up)   */
  kl_nvfp4_tensor w2;   /* [D, F]                                                  */
} kl_block_weights;

typedef struct kl_block_io {
  const void* x;        /* bf16 [T, D] input residual stream                       */
  const void* mod[6];   /* bf16 [D] each: shift1, scale1, gate1, shift2, scale2, gate2 */
  const float* rope_cs; /* fp32 [16, T, 4, 2] from kl_rope_table                    */
  int64_t T, D, H, F;
  int attn_precision;   /* KL_ATTN_FP8 or KL_ATTN_BF16                             */
  void* out;            /* bf16 [T, D] block output (must not alias x)             */
  void* const* stage_events; /* optional (NULL): KL_BLOCK_STAGES+1 cudaEvent_t handles
                                owned by the caller; events[i] is recorded on the
                                stream before stage i, events[KL_BLOCK_STAGES] after
                                the last stage (per-kernel device timing)            */
  float sol_tau;        /* Sol-Attention threshold (log2 units): 0 (default) = dense
                           attention; > 0 = each query block visits only the key
                           tiles kl_sol_select keeps at this tau (selection runs
                           inside the attention stage)                          */
  float vc_budget;      /* VC-Attention repair budget in [0, 1]: 0 (default) = off;
                           > 0 = FP8 attention only (not with sol_tau), the pairs
                           kl_vc_select picks are computed from the bf16 q, k, v */
} kl_block_io;

/* Stages of kl_joint_block_forward, in launch order (stage_events index). */
#define KL_STAGE_LN1 0         /* LayerNorm1 + modulate + NVFP4 (2 kernels)       */
#define KL_STAGE_QKV 1         /* QKV GEMM + RoPE epilogue                        */
#define KL_STAGE_FP8_CAST 2    /* per-head E4M3 cast (FP8 attention only)         */
#define KL_STAGE_ATTN 3        /* joint attention                                 */
#define KL_STAGE_QUANT_O 4     /* NVFP4 of O                                      */
#define KL_STAGE_OUT 5         /* output-projection GEMM + gated residual         */
#define KL_STAGE_LN2 6         /* LayerNorm2 + modulate + NVFP4 (2 kernels)       */
#define KL_STAGE_MLP_UP 7      /* MLP-up GEMM + SwiGLU epilogue                   */
#define KL_STAGE_QUANT_H 8     /* NVFP4 of h                                      */
#define KL_STAGE_MLP_DOWN 9    /* MLP-down GEMM + gated residual                  */
#define KL_BLOCK_STAGES 10

size_t kl_block_workspace_size(int64_t T, int64_t D, int64_t H, int64_t F, int attn_precision);

/*
 * kl_joint_block_forward -- one joint transformer block ([P2] Summary; [P4]
 * Two-Stage Processing), plain reading of the wiring:
 *   m1  = bf16(LN(x)*(1+scale1)+shift1)            -> NVFP4 (dynamic gs)
 *   qkv = m1 . Wqkv^T, RoPE on q,k, bf16            (QKV_ROPE epilogue)
 *   [FP8: per-head E4M3 cast of q, k, v]
 *   O   = joint attention over all T tokens, bf16   -> NVFP4
 *   x1  = bf16(x + gate1 * (O . Wo^T))              (GATED_RESIDUAL)
 *   m2  = bf16(LN(x1)*(1+scale2)+shift2)            -> NVFP4
 *   h   = bf16(silu(g)*u), [g u] = m2 . W1^T        (SWIGLU) -> NVFP4
 *   out = bf16(x1 + gate2 * (h . W2^T))             (GATED_RESIDUAL)
 * D = 128*H (H <= 64); F % 128 == 0; T >= 1.
 * workspace: >= kl_block_workspace_size(...), 256-byte aligned.
 */
kl_status kl_joint_block_forward(const kl_block_weights* w, const kl_block_io* io,
                                 void* workspace, size_t ws_bytes, void* stream);

/*
 * kl_joint_block_forward_host -- kl_joint_block_forward for a caller whose
 * activations live in host memory: io->x, io->mod[0..5] and io->out are HOST
 * pointers (page-locked memory keeps the copies asynchronous; pageable
 * memory makes them block the calling thread); the weights, io->rope_cs and
 * the workspace are device memory as above.  On the stream: x and the six
 * modulation vectors are copied into the workspace, the block runs there,
 * and the output is copied back to io->out.  The host buffers must stay
 * valid, and io->out unread, until the stream has reached the end of the
 * call.  workspace: >= kl_block_host_workspace_size(...) bytes, 256-byte
 * aligned (the block's workspace followed by x, out and the modulation
 * vectors).
 */
size_t kl_block_host_workspace_size(int64_t T, int64_t D, int64_t H, int64_t F, int attn_precision);
kl_status kl_joint_block_forward_host(const kl_block_weights* w, const kl_block_io* io,
                                      void* workspace, size_t ws_bytes, void* stream);

/*
 * kl_dit_step -- one Euler step of a synthetic DiT on the block above ([P2]
 * Summary: per-mode blocks for each stream, then joint blocks; [P4] The VAE
 * and Tokenization: 2x2 latent patches; Two-Stage Processing).  Readings
 * (the pages stop at the block structure):
 *   patches p[t][k] = bf16(latent[y][x][c]), t = (y/2)*grid_w + x/2,
 *     k = 4c + 2(y%2) + (x%2)                       (no bias, no norm)
 *   image tokens = NVFP4(p) . w_in^T (bf16); the text conditioning [n_text, D]
 *     is copied in front of them each step: sequence [text; image]
 *   per-mode block i: the block on the text rows alone (mode_text[i], text
 *     RoPE layout) and on the image rows alone (mode_image[i], image layout)
 *   joint block i: the block on the whole sequence (joint layout)
 *   v = NVFP4(bf16(LN(img)*(1+scale_f)+shift_f)) . w_out^T   (fp32 [Ti, 4C])
 *   latent[y][x][c] = fl(latent + fl(dt * v[t][k]))  (Euler, same (t, k) map)
 * Shapes: latent fp32 [2*grid_h, 2*grid_w, channels], 4*channels % 128 == 0;
 * D = 128*H; the block constraints.  mode_text / mode_image / joint are host
 * arrays (n_mode_blocks / n_joint_blocks entries) of device weights.  Every
 * pointer in kl_dit_step_io is a device pointer; rope_* come from
 * kl_rope_table for the layouts (n_text,0,0,0), (0,grid_h,grid_w,0),
 * (n_text,grid_h,grid_w,0).  workspace >= kl_dit_workspace_size, 256-byte
 * aligned.  The call is capturable in a CUDA graph (no host sync).
 */
typedef struct kl_dit_shape {
  int64_t n_text, grid_h, grid_w, channels;
  int64_t D, H, F;
  int n_mode_blocks, n_joint_blocks;
  int attn_precision; /* KL_ATTN_FP8 or KL_ATTN_BF16 */
} kl_dit_shape;

typedef struct kl_dit_weights {
  kl_nvfp4_tensor w_in;               /* [D, 4*channels] */
  const kl_block_weights* mode_text;  /* host array [n_mode_blocks] */
  const kl_block_weights* mode_image; /* host array [n_mode_blocks] */
  const kl_block_weights* joint;      /* host array [n_joint_blocks] */
  kl_nvfp4_tensor w_out;              /* [4*channels, D] */
} kl_dit_weights;

typedef struct kl_dit_step_io {
  float* latent;           /* fp32 [2*grid_h, 2*grid_w, channels], updated in place */
  const void* text;        /* bf16 [n_text, D] */
  const void* mod_mode;    /* bf16 [n_mode_blocks][2 (text, image)][6][D] (block order of kl_block_io.mod) */
  const void* mod_joint;   /* bf16 [n_joint_blocks][6][D] */
  const void* mod_final;   /* bf16 [2][D]: shift_f, scale_f */
  const float* rope_text;
  const float* rope_image;
  const float* rope_joint;
  float dt;                /* t_{i+1} - t_i */
  float sol_tau;           /* kl_block_io.sol_tau for every block of the step (0: dense;
                              a caller keeps the first steps dense by passing 0) */
} kl_dit_step_io;

size_t kl_dit_workspace_size(const kl_dit_shape* shape);

/*
 * kl_dit_workspace_views -- where, inside kl_dit_step's workspace, the step
 * leaves its intermediates, as byte offsets from the workspace start (for
 * inspection and stage-by-stage tests; no device work).  Valid after a
 * kl_dit_step call (not kl_dit_step_cached) until the next call that uses
 * the workspace:
 *   tokens       bf16 [T, D]: the sequence after the last block (the head's input)
 *   head_codes   NVFP4 codes [grid_h*grid_w, D/2] of the head's
 *                bf16(LN(image rows)*(1+scale_f)+shift_f)
 *   head_scales  their scales, KL_SCALE_MMA layout
 *   head_gs      their fp32 global scale
 *   velocity     fp32 [grid_h*grid_w, 4*channels]: v before the Euler update
 */
typedef struct kl_dit_views {
  size_t tokens, head_codes, head_scales, head_gs, velocity;
} kl_dit_views;
kl_status kl_dit_workspace_views(const kl_dit_shape* shape, kl_dit_views* out);

kl_status kl_dit_step(const kl_dit_shape* shape, const kl_dit_weights* w, const kl_dit_step_io* io,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * kl_dit_step_cached -- kl_dit_step with Cache-DiT step caching ([P1]
 * "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs", How it
 * works: a residual difference between denoising steps is watched and, under
 * a threshold, cached transformer outputs are reused; What you can do:
 * residual_diff_threshold 0.24).  Readings (the pages give no more):
 *   block 0 of the stack (the first per-mode pair, else the first joint
 *     block) is the probe and runs every step: F = its output, r = F - its
 *     input (fp32 of the bf16 tokens, all T = n_text + grid_h*grid_w rows);
 *   diff = sum|r - r_ref| / sum|r_ref| (0/0 -> 0, x/0 -> +inf), r_ref being
 *     the probe residual of the last step that ran every block; no
 *     reference yet (first step after kl_dit_cache_reset) -> diff = +inf;
 *   hit = diff < threshold: blocks 1.. are skipped and the final tokens are
 *     bf16(F + R); miss: blocks 1.. run, R = final - F (fp32) and r_ref = r;
 *   the head (final LN, adaLN, w_out, Euler update) runs either way.
 * The sums are fp32 per thread and fp64 across thread blocks (their order is
 * not fixed, so diff may vary in its last bits between runs); the decision
 * compares diff in fp64.
 *
 * cache: a caller-owned device buffer of kl_dit_cache_size(shape) bytes,
 * 256-byte aligned, holding a kl_dit_cache_header at offset 0 followed by
 * F bf16 [T, D], r_cur fp32 [T, D], r_ref fp32 [T, D], R fp32 [T, D], each at
 * the next 256-byte boundary.  Call kl_dit_cache_reset(cache, stream) before
 * the first step of every generation (it also creates, outside any graph
 * capture, the side stream used below).  The header can be read back (e.g.
 * with cudaMemcpy) after a step: diff, hit, and hits / steps since the reset.
 *
 * Outside stream capture the call synchronises the stream once, to read the
 * decision on the host.  Under capture (a CUDA graph) it does not: a one-
 * thread kernel takes the decision on the device and sets the condition of a
 * conditional (IF) graph node whose body, captured on a side stream, holds
 * blocks 1..; a skipped step then costs the probe block, the head and three
 * small kernels.  Errors: as kl_dit_step; KL_ERR_UNSUPPORTED_SHAPE without any
 * block; KL_ERR_WORKSPACE if cache_bytes is too small.
 */
typedef struct kl_dit_cache_header {
  double num, den; /* sums of the step in flight (zero between steps) */
  float diff;      /* residual difference of the last step (+inf: no reference) */
  int hit;         /* 1: the last step reused the cache */
  int has_ref;     /* 1: a reference step exists */
  int hits;        /* hits since the last reset */
  int steps;       /* steps since the last reset */
} kl_dit_cache_header;

size_t kl_dit_cache_size(const kl_dit_shape* shape); /* 0: bad shape or no block */
kl_status kl_dit_cache_reset(void* cache, void* stream);
kl_status kl_dit_step_cached(const kl_dit_shape* shape, const kl_dit_weights* w, const kl_dit_step_io* io,
                             float threshold, void* cache, size_t cache_bytes, void* workspace, size_t ws_bytes,
                             void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KLEIN_H */
