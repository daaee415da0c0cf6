/*
 * wf.h -- C ABI of libwf.so: the wave-round hot path of Wave Forcing on B200.
 *
 * Source of the operations: "Wave Forcing: Towards Speed-of-Light Streaming
 * Video Generation" (abstract): one concurrent forward round ("wave") runs S
 * chunks at staggered denoising steps plus one cache-refresh chunk; chunk-wise
 * causal attention lets each chunk read earlier, cleaner chunks (including
 * ones whose denoising is not finished) and the rolling history cache; Wave
 * Parallelism delivers each layer's K/V early.  The airadar.tv summary
 * ("usage") fixes the wave sizes (--rf-step 4 --wp-size 5, --rf-step 5
 * --wp-size 6) and 3-latent-frame chunks.
 *
 * Notation.  L = tokens per chunk, W = chunks in the wave (denoising chunks +
 * the refresh chunk, refresh chunk = wave chunk 0, the oldest), Hh = history
 * chunks, H = heads, D = head_dim, T = W*L, R = Hh + W ring slots.  In round r
 * wave chunk c is absolute chunk r + c; the history is the h = min(Hh, r)
 * chunks r-h .. r-1.  Absolute chunk g lives in ring slot g mod R.
 *
 * Layouts (all row-major, bf16 = 16-bit bfloat16 bit patterns):
 *   q, k, v, q_out, o     [T][H][D]  token-major, as a QKV projection emits
 *   k_cache, v_cache      [R][L][H][D]
 *   pos_thw               [T][3] int32 (t, h, w) or NULL (derived, see below)
 *   gamma_q, gamma_k      [H][D] float32
 *   lse                   [H][T] float32 natural-log sum-exp, or NULL
 *
 * Ownership.  The caller owns every buffer and stream.  The library owns the
 * plan (host memory plus a few bytes of device memory on the device that was
 * current at wf_plan, freed by wf_plan_destroy).  The two hot calls allocate
 * nothing, never synchronise the host and use only the stream they are given
 * (NULL = the legacy default stream).  They are asynchronous: errors raised on
 * the device are reported by wf_sync_status.  Hot calls of one plan must not
 * run concurrently on the GPU (the plan's device words are shared).
 *
 * Errors.  Every entry point returns a wf_status (0 = WF_OK) or a value that
 * documents its own failure value.  Nothing aborts the process, nothing traps
 * on the device; a device-side wait that runs past its limit ends the kernel
 * with WF_ERR_TIMEOUT recorded in the plan.
 */
#ifndef WF_H_
#define WF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WF_API __attribute__((visibility("default")))
#else
#define WF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum wf_status {
    WF_OK = 0,
    WF_ERR_INVALID_ARG = 1,   /* a size, pointer or alignment check failed        */
    WF_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. head_dim not 64/128)    */
    WF_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed       */
    WF_ERR_TIMEOUT = 4,       /* a bounded device wait expired (kernel stopped)    */
    WF_ERR_NO_DEVICE = 5,     /* the plan has no device state (no GPU at wf_plan)  */
    WF_ERR_DEVICE = 6,        /* the device is not an sm_100 (B200-class) part     */
    WF_ERR_BOUNDS = 7         /* a bounds check of the WF_CHECK debug build failed */
} wf_status;

typedef struct wf_plan_s *wf_plan_t;

/* Build a plan for one layer's wave round.
 * Passage: "Wave Forcing" abstract -- a wave is S chunks at staggered denoising
 * steps plus one cache-refresh chunk (W = S + 1), with a rolling history; the
 * airadar.tv summary, usage section, gives the sizes (--rf-step 4 --wp-size 5:
 * W = 5; 3-latent-frame chunks).
 * chunk_tokens L >= 1, n_wave_chunks W >= 1, n_hist_chunks Hh >= 0, heads H >= 1,
 * head_dim D in {64, 128}; T*H*D must fit in 2^31 elements per tensor.
 * Host work only, plus a 256-byte device allocation (status word and the
 * attention scheduler's counter) on the current device.  If no CUDA device is
 * present the plan is still created for the host-side queries and the hot
 * calls return WF_ERR_NO_DEVICE.  RoPE defaults: no grid set (pos_thw must be
 * passed), split dt = D - 4*(D/6), dh = dw = 2*(D/6), theta = 10000;
 * RMSNorm eps = 1e-6.  *out is NULL on failure. */
WF_API int wf_plan(int chunk_tokens, int n_wave_chunks, int n_hist_chunks, int heads,
            int head_dim, wf_plan_t *out);

/* Latent geometry of a chunk for derived positions: L must equal
 * frames_per_chunk * grid_h * grid_w.  Token n = c*L + f*grid_h*grid_w + y*grid_w + x
 * of round r gets (t, h, w) = ((r + c)*frames_per_chunk + f, y, x).  theta > 0. */
WF_API int wf_plan_set_rope(wf_plan_t plan, int frames_per_chunk, int grid_h, int grid_w,
                     double theta);

/* Channel widths of the t/h/w RoPE blocks (each even, sum = D). */
WF_API int wf_plan_set_rope_split(wf_plan_t plan, int d_t, int d_h, int d_w);

/* RMSNorm epsilon (>= 0). */
WF_API int wf_plan_set_norm_eps(wf_plan_t plan, double eps);

/* Device-wait limit in SM clock cycles for the attention and GEMM kernels
 * (0 = default, about two seconds).  Exposed so that tests can make a wait
 * expire quickly. */
WF_API int wf_plan_set_wait_limit(wf_plan_t plan, unsigned long long cycles);

/* Test hook for failure detection, off by default.  With on != 0 the attention
 * kernel's producer withholds the first Q-tile copy of every CTA (with the
 * pair kernel: of every cluster's leader CTA), so the MMA
 * warp's wait for it cannot complete: the bounded wait expires, the kernel
 * stops cleanly (copies and MMAs in flight drained, TMEM freed) and
 * wf_sync_status returns WF_ERR_TIMEOUT.  Nothing faults or traps; the
 * context stays usable.  Pair it with a short wf_plan_set_wait_limit.  The
 * GEMM calls (wf_linear, wf_qkv_proj_norm_rope_append) honour the same hook:
 * no CTA issues, and the leader does not arm, the copies of the first K slice,
 * so the MMA's wait for it expires the same way. */
WF_API int wf_plan_set_withhold_q(wf_plan_t plan, int on);

/* Attention kernel variant.  Both compute the same result (within the
 * attention tolerance; they accumulate in different orders):
 *   WF_ATTN_SINGLE  one CTA per SM, two 128-row query tiles per work unit,
 *                   units taken from a global counter (head_dim 64 and 128);
 *   WF_ATTN_PAIR    clusters of two CTAs on two SMs sharing 256-row tensor-core
 *                   MMAs (tcgen05 cta_group::2), S double-buffered in tensor
 *                   memory, a static longest-first unit order (head_dim 128 only);
 *   WF_ATTN_AUTO    the default: SINGLE, the faster of the two on B200 at every
 *                   shape measured (the Wan 1.3B / 14B wave rounds).
 * Returns WF_ERR_UNSUPPORTED for PAIR with head_dim 64, WF_ERR_INVALID_ARG for
 * an unknown value. */
#define WF_ATTN_AUTO 0
#define WF_ATTN_SINGLE 1
#define WF_ATTN_PAIR 2
WF_API int wf_plan_set_attn_kernel(wf_plan_t plan, int kind);

/* Order of the attention's work units (single-CTA kernel, bf16 and FP8 Q.K^T).
 * A unit is (wave chunk c, head h, pair of 128-row query tiles); it reads the
 * key/value chunks that chunk-wise causal attention ("Wave Forcing", abstract)
 * lets chunk c see: the valid history chunks and wave chunks 0..c of head h.
 * The same key chunk is read by the units of every wave chunk at or after it,
 * so the kernel takes the heads in blocks: all units of one block of heads,
 * longest first inside the block, then the next block.
 *
 * wf_plan_set_head_block sets the heads per block, 1..heads; 0 (the default)
 * lets each call choose with wf_attn_head_block.  Outputs are bit-identical
 * for every value: each unit computes the same rows in the same order, only
 * the order of the units changes.  WF_ERR_INVALID_ARG outside 0..heads or for
 * a NULL plan. */
WF_API int wf_plan_set_head_block(wf_plan_t plan, int heads);

/* Heads per block that round `round`'s attention call uses (fp8_keys != 0: the
 * FP8 Q.K^T call, whose keys are 1 byte).  -1 for a NULL plan or round < 0. */
WF_API int wf_plan_head_block(wf_plan_t plan, long round, int fp8_keys);

/* The choice itself (host arithmetic only).  A block's visible keys and values,
 * (h_valid + n_wave_chunks) * chunk_tokens * head_dim * (key_bytes + 2) bytes
 * per head, are kept within half of l2_bytes, so that the units reading a key
 * tile after the first find it in L2; that caps the count at g_max (at least
 * 1, at most heads; heads when l2_bytes <= 0).  Among 1..g_max the count whose
 * schedule ends first is returned, each count played through the kernel's
 * dynamic schedule over n_ctas CTAs (a unit costs its key tiles, 0.93 of that
 * with a single query tile, plus 3 tiles of set-up; ties go to the larger
 * count).  g_max is returned without that comparison when n_ctas is outside
 * 1..1024 or the comparison would take over 4M unit steps.  Returns -1 for
 * sizes that are not positive (h_valid < 0, key_bytes not 1 or 2). */
WF_API int wf_attn_head_block(int heads, int n_wave_chunks, int h_valid, int chunk_tokens,
                              int head_dim, int key_bytes, long long l2_bytes, int n_ctas);

WF_API void wf_plan_destroy(wf_plan_t plan);

/* Bytes of ONE ring (K or V): R * L * H * D * 2.  0 for a NULL plan. */
WF_API size_t wf_cache_bytes(wf_plan_t plan);

/* Useful attention FLOPs of round r: 4*H*D*L^2 * sum_c (min(Hh, r) + c + 1),
 * counting the key chunks that chunk-wise causal attention ("Wave Forcing"
 * abstract) lets wave chunk c see: the valid history plus wave chunks 0..c;
 * i.e. QK^T and PV over visible, unpadded pairs.  -1 for a NULL plan. */
WF_API double wf_useful_flops(wf_plan_t plan, long round);

/* Fused per-head RMSNorm(q, k) * gamma, 3D RoPE, and ring append.
 * Passage: "Wave Forcing" abstract and the airadar.tv summary's mechanism
 * paragraph -- each layer's K/V is handed to the later chunks early (Wave
 * Parallelism); on one GPU that hand-over is this write into the ring the
 * attention reads.  The per-head norm and (t,h,w) RoPE are those of the Wan2.1
 * DiT the pages run (their formulas are not printed; plain definitions here).
 * For every wave token n (chunk c = n / L) and head h:
 *   q_out[n,h] = bf16(RoPE(pos[n], RMSNorm(q[n,h]) * gamma_q[h]))
 *   k_cache[(r+c) mod R, n mod L, h] = bf16(RoPE(pos[n], RMSNorm(k[n,h]) * gamma_k[h]))
 *   v_cache[(r+c) mod R, n mod L, h] = v[n,h]          (bit-exact copy)
 * fp32 arithmetic, one round-to-nearest-even to bf16.  round >= 0.  All
 * pointers are device pointers, 16-byte aligned; pos_thw may be NULL when
 * wf_plan_set_rope set the geometry.  q_out may alias q; nothing else may
 * overlap.  One kernel launch on `stream` (a cudaStream_t). */
WF_API int wf_qk_norm_rope_append(wf_plan_t plan, long round,
                           const void *q, const void *k, const void *v,
                           const int32_t *pos_thw,
                           const float *gamma_q, const float *gamma_k,
                           void *q_out, void *k_cache, void *v_cache,
                           void *stream);

/* Chunk-causal attention of round r.
 * Passage: "Wave Forcing" abstract -- chunk-wise causal attention: a chunk attends
 * to the history cache and to the earlier (cleaner) chunks of the wave even while
 * those are still being denoised, and bidirectionally inside itself.
 * For query token n of wave chunk c, head h:
 *   O[n,h] = softmax_j(q_out[n,h] . K_j / sqrt(D)) V_j
 * over every token j of the min(Hh, r) history chunks and of wave chunks 0..c
 * (bidirectional inside a chunk), read from the ring slots written by
 * wf_qk_norm_rope_append.  bf16 tensor-core products, fp32 accumulation and
 * softmax, one rounding of O to bf16.  lse (optional) gets the natural-log
 * sum-exp per (h, n).  Device pointers, 16-byte aligned; o must not overlap the
 * inputs.  One persistent kernel launch (plus a 4-byte memset of the scheduler
 * counter) on `stream`. */
WF_API int wf_chunk_causal_attn(wf_plan_t plan, long round,
                         const void *q_out, const void *k_cache, const void *v_cache,
                         void *o, float *lse, void *stream);

/* ---- FP8 (E4M3) Q.K^T variant --------------------------------------------
 * The quantized-attention counterpart ("Wave Forcing" abstract: the systems run
 * on SageAttention with W8A8 backends): Q and K enter the score MMA as 8-bit
 * E4M3 codes with fp32 scales, P.V stays bf16.  The quantization rule is exact:
 * for a group x, amax = max|x|, scale = amax / 448 (IEEE fp32 division; 1 for
 * amax = 0), code = E4M3(x / scale) with the fp32 quotient rounded to nearest,
 * ties to even, saturating at +-448.  Groups: one (token, head) row of q_out;
 * one 128-row key tile of one chunk and head of K.  The codes use the layouts of
 * their bf16 sources with one byte per element. */

/* Quantize q_out [T,H,D] -> q8 [T,H,D] (E4M3 codes) and q_scale [H,T] (fp32),
 * one scale per (token, head).  Device pointers: q_out and q8 16-byte aligned,
 * q_scale 4-byte aligned.  One kernel launch on `stream`. */
WF_API int wf_quantize_q_fp8(wf_plan_t plan, const void *q_out, void *q8, float *q_scale,
                             void *stream);

/* wf_qk_norm_rope_append with the row quantization of wf_quantize_q_fp8 fused
 * into the same pass: q8 [T,H,D] E4M3 codes and q_scale [H,T] are exactly what
 * wf_quantize_q_fp8 writes for the bf16 q_out this call computes (same rule,
 * same bits), and K'/V go to the ring as in wf_qk_norm_rope_append.  q_out may
 * be NULL (the FP8 attention reads only q8), which saves its write.  Device
 * pointers: q, k, v, q_out, q8 and the caches 16-byte aligned, q_scale 4-byte
 * aligned.  One kernel launch on `stream`; per element it reads q, k, v and
 * writes K', V and one code byte (plus q_out when given). */
WF_API int wf_qk_norm_rope_append_fp8q(wf_plan_t plan, long round,
                                       const void *q, const void *k, const void *v,
                                       const int32_t *pos_thw,
                                       const float *gamma_q, const float *gamma_k,
                                       void *q_out, void *q8, float *q_scale,
                                       void *k_cache, void *v_cache, void *stream);

/* Quantize the K of absolute chunks first_chunk .. first_chunk+n_chunks-1, read
 * from k_cache [R,L,H,D] bf16 at slots (chunk mod R), into k8_cache [R,L,H,D]
 * (E4M3 codes, same slots) and k_scale [R, ceil(L/128), H] (fp32), one scale
 * per (slot, 128-row key tile, head).  After wf_qk_norm_rope_append(round) the
 * wave's chunks are first_chunk = round, n_chunks = W; history chunks are
 * quantized once, when they were appended.  0 <= n_chunks <= R, first_chunk >= 0.
 * Device pointers as above.  One kernel launch on `stream`. */
WF_API int wf_quantize_k_fp8(wf_plan_t plan, long first_chunk, int n_chunks,
                             const void *k_cache, void *k8_cache, float *k_scale,
                             void *stream);

/* Chunk-causal attention of round r as wf_chunk_causal_attn, with scores
 * s = (q8 . k8) * q_scale * k_scale / sqrt(D) from an E4M3 tensor-core product
 * (fp32 accumulation) and bf16 P.V.  head_dim 128 only (WF_ERR_UNSUPPORTED
 * otherwise).  q8/k8_cache as written by the two calls above; v_cache is the
 * bf16 ring.  Device pointers (codes and v 16-byte aligned, scales 4-byte
 * aligned); o must not overlap the inputs.  One persistent kernel launch (plus
 * a 4-byte memset of the scheduler counter) on `stream`. */
WF_API int wf_chunk_causal_attn_fp8qk(wf_plan_t plan, long round, const void *q8,
                                      const float *q_scale, const void *k8_cache,
                                      const float *k_scale, const void *v_cache, void *o,
                                      float *lse, void *stream);

/* ---- The DiT block around the wave round ---------------------------------
 * "Wave Forcing" (abstract) runs every wave chunk through the layers of
 * Wan2.1-T2V-1.3B in one forward pass.  Around the chunk-causal attention a DiT
 * block holds dense projections (QKV, output, two feed-forward layers) and the
 * adaLN-modulated LayerNorms before the attention and the feed-forward.  The
 * pages print no formula for these layers; the definitions below are the plain
 * ones.  Every chunk of a wave sits at its own denoising step, so modulation
 * rows are per chunk: row n uses row n / rows_per_group of a modulation table.
 *
 * GEMMs are bf16 tensor-core products with fp32 accumulation, computed as
 * y = x W^T with x [M][K] and W [N][K] (a linear layer's weight, out x in),
 * both row-major bf16; the epilogue works in fp32 and rounds once to bf16.
 * Each GEMM is one persistent kernel launch on `stream` (clusters of two CTAs).
 * They use the plan only for its device status word and wait limit; calls on
 * one plan must not run concurrently on the GPU. */

enum {
    WF_EPI_STORE = 0,            /* y = x W^T + bias                                   */
    WF_EPI_GELU_TANH = 1,        /* y = gelu(x W^T + bias), tanh form of GELU          */
    WF_EPI_GATED_RESIDUAL = 2    /* y = resid + gate[n / rows_per_group] * (x W^T + bias) */
};

/* A linear layer with a fused epilogue.  M >= 0 rows, N >= 32 and N % 32 == 0
 * outputs, K >= 8 and K % 8 == 0 inputs.  x [M][K], w [N][K], y [M][N], resid
 * [M][N]: bf16 device pointers, 16-byte aligned; bias [N] fp32 or NULL; gate [G][N]
 * fp32 with G >= ceil(M / rows_per_group) (gated residual only; NULL otherwise).
 * y must not overlap x or w (it may be resid).  M = 0 is a no-op that reads no
 * pointer (they may be NULL).  Returns WF_ERR_INVALID_ARG on a bad size,
 * epilogue, pointer or alignment. */
WF_API int wf_linear(wf_plan_t plan, int M, int N, int K, const void *x, const void *w,
                     const float *bias, int epilogue, const float *gate, const void *resid,
                     int rows_per_group, void *y, void *stream);

/* The QKV projection of the wave with wf_qk_norm_rope_append fused into its
 * epilogue: y = x W_qkv^T + b_qkv ([T][3*H*D], q | k | v, each head-major), then
 * per head the RMSNorm (gain gamma) and 3D RoPE of q and k, computed on the fp32
 * accumulator (no rounding before the norm), and one rounding to bf16 each.  q
 * goes to q_out [T][H][D]; k and v of wave chunk c go to ring slot (round + c)
 * mod R of k_cache / v_cache, exactly where wf_qk_norm_rope_append writes them.
 * x [T][hidden] and w_qkv [3*H*D][hidden] bf16 (hidden % 8 == 0), b_qkv [3*H*D]
 * fp32 or NULL, gammas [H][D] fp32; device pointers, 16-byte aligned.  Positions
 * are derived from the plan's grid (wf_plan_set_rope is required;
 * WF_ERR_INVALID_ARG without it).  H*D must be a multiple of 128, and the
 * rotation tables (W*F*dt/2 + grid_h*dh/2 + grid_w*dw/2 entries) must fit 3072
 * entries; WF_ERR_UNSUPPORTED otherwise.  One kernel launch on `stream`. */
WF_API int wf_qkv_proj_norm_rope_append(wf_plan_t plan, long round, int hidden, const void *x,
                                        const void *w_qkv, const float *b_qkv,
                                        const float *gamma_q, const float *gamma_k, void *q_out,
                                        void *k_cache, void *v_cache, void *stream);

/* LayerNorm over the last axis without a learned affine (eps 1e-6), then the
 * adaLN modulation y = x_hat * (1 + scale[g]) + shift[g], g = n / rows_per_group.
 * x, y [M][C] bf16; shift, scale [G][C] fp32; device pointers, 16-byte aligned;
 * C % 8 == 0 and C <= 6144 (WF_ERR_UNSUPPORTED above).  y may equal x.  fp32
 * arithmetic, one rounding to bf16.  One kernel launch on `stream`. */
WF_API int wf_layer_norm_modulate(wf_plan_t plan, int M, int C, const void *x, const float *shift,
                                  const float *scale, int rows_per_group, void *y, void *stream);

/* ---- The streaming VAE-decode stage -------------------------------------
 * "Wave Forcing" (abstract) lists pipelined VAE decoding as one part of its
 * runtime; the airadar.tv summary (usage section) takes the VAE from the Wan2.1
 * base model, splits its decode into 2 or 3 pipeline stages (--vae-stages) and
 * decodes 399 latent frames into 1593 video frames.  The pages print no layer
 * of the decoder; these calls are the plain definitions of a causal 3D-conv
 * decoder stage.  Activations are channels-last [T][H][W][C] bf16.  A video is
 * decoded chunk by chunk: a convolution of chunk i reads, before its first
 * frame, the last two frames of the same convolution's input in chunk i - 1,
 * so streaming the chunks gives exactly the convolution of the whole video and
 * the decode of one chunk can run while the next chunk is generated. */

/* Causal 3x3x3 convolution of one chunk:
 *   y[t,i,j,o] = bias[o] + sum over dt, dy, dx in 0..2 and c of
 *                w[o][dt][dy][dx][c] * X(t+dt-2, i+dy-1, j+dx-1, c)  (+ resid[t,i,j,o])
 * where X(tau, ...) is x for tau >= 0, x_hist[tau + 2] for tau < 0 (x_hist: the
 * previous chunk's last two input frames [2][H][W][Cin], or NULL at the start
 * of the video, which reads zeros), and zero outside the H x W frame.
 * x [T][H][W][Cin], w [Cout][3][3][3][Cin], resid and y [T][H][W][Cout]: bf16
 * device pointers, 16-byte aligned; bias [Cout] fp32 or NULL; resid may be NULL
 * and may equal y; y must not overlap x, x_hist or w.  Cin % 8 == 0, Cout % 32
 * == 0, T*H*W < 2^31.  bf16 tensor-core products (an implicit GEMM: K = 27 taps
 * x Cin) with fp32 accumulation, one rounding to bf16.  One persistent kernel
 * launch on `stream` (clusters of two CTAs). */
WF_API int wf_causal_conv3d(wf_plan_t plan, int T, int H, int W, int Cin, int Cout,
                            const void *x, const void *x_hist, const void *w,
                            const float *bias, const void *resid, void *y, void *stream);

/* Per pixel (row of C channels): y = x / sqrt(mean_c x^2 + 1e-6) * gamma, then
 * y * sigmoid(y) (SiLU).  x, y [M][C] bf16, gamma [C] fp32; device pointers,
 * 16-byte aligned; C % 8 == 0 and C <= 512 (WF_ERR_UNSUPPORTED above).  y may
 * equal x.  fp32 arithmetic, one rounding to bf16.  One kernel launch. */
WF_API int wf_rms_norm_silu(wf_plan_t plan, int M, int C, const void *x, const float *gamma,
                            void *y, void *stream);

/* Wait for `stream`, then read and clear the plan's device status word.
 * Returns WF_OK, WF_ERR_TIMEOUT (a bounded device wait expired), WF_ERR_BOUNDS
 * (only in the debug build libwf_check.so, compiled with -DWF_CHECK: a computed
 * index fell outside its tensor; the access was skipped) or WF_ERR_CUDA. */
WF_API int wf_sync_status(wf_plan_t plan, void *stream);

/* The key chunks the attention kernel visits in round r, in visiting order:
 * for each wave chunk c, for each visible chunk (oldest first), the quadruple
 * (c, logical index b, absolute chunk id, ring slot).  Writes at most cap
 * quadruples (4*cap int32) and returns the number needed, or -1 on bad input.
 * The kernel computes slots with the same function. */
WF_API int wf_plan_debug_ranges(wf_plan_t plan, long round, int32_t *out, int cap);

WF_API const char *wf_status_string(int status);

/* Chunk-causal attention of round r without a plan, for callers that must not
 * allocate device memory (for example a serving loop whose device memory is
 * owned by a framework's caching allocator or reserved up front, where a
 * direct cudaMalloc would break that accounting or stall the device).  The
 * paper has no counterpart: this is an interface choice of this library.
 * Same computation, layouts, alignment rules and shape limits as wf_plan +
 * wf_chunk_causal_attn; the shape is passed directly.  Instead of the plan's
 * device block the kernel's scratch (status word, timeout site, work counter)
 * lives in a 256-byte block compiled into the library, present on every GPU
 * that loads it until the process exits; no cudaMalloc, cudaFree or
 * allocating library call is made.  The first call on a device (and the first
 * after that device's context was created again, e.g. after cudaDeviceReset)
 * looks up that block's device address (cudaGetSymbolAddress); make that first
 * call before any stream capture.  All calls on a device share the block: each
 * clears what must start at zero on its own stream, and calls that overlap on
 * the GPU race on it.  A device-side timeout is recorded in the block; the
 * call itself returns before the kernel runs (WF_OK, o then partly written),
 * and wf_noalloc_sync_status below reads the recorded status back.  Returns WF_OK, WF_ERR_INVALID_ARG / WF_ERR_UNSUPPORTED for shapes or
 * pointers the plan API would reject, WF_ERR_NO_DEVICE, WF_ERR_DEVICE or
 * WF_ERR_CUDA. */
WF_API int wf_chunk_causal_attn_noalloc(int chunk_tokens, int n_wave_chunks, int n_hist_chunks,
                                        int heads, int head_dim, long round,
                                        const void *q_out, const void *k_cache,
                                        const void *v_cache, void *o, float *lse, void *stream);

/* Test hook of the entry point above: sets every 32-bit word of the current
 * device's scratch block to `word` (synchronously), the state a call whose
 * bounded wait ran out leaves behind (status and timeout site set, the work
 * counter past the last unit), so that a test can check that the next call
 * starts clean.  It copies into the library's own block and allocates
 * nothing.  Must not run while a call is in flight.  WF_OK, WF_ERR_NO_DEVICE,
 * WF_ERR_CUDA. */
WF_API int wf_noalloc_debug_fill_scratch(unsigned int word);

/* Wait for `stream`, then read the status the attention kernel recorded in the
 * current device's scratch block: WF_ERR_TIMEOUT (a bounded device wait ran
 * out; that call's o is partly written), WF_ERR_BOUNDS (a bounds check of the
 * checked build failed), else WF_OK.  Copies two words to host memory and
 * allocates nothing; clears nothing (the next call does).  The block is shared
 * by every call on the device, so the answer covers the calls since the last
 * one started.  WF_ERR_NO_DEVICE / WF_ERR_CUDA on a device error. */
WF_API int wf_noalloc_sync_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* WF_H_ */
