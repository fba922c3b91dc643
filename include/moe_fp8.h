/*
 * moe_fp8.h -- C ABI of the B200 (sm_100a) FP8 DeepSeekMoE layer forward.
 *
 * The operations follow the DeepSeek-V3 pages:
 *  [P4] "DeepSeek-V3 Technischer Bericht" (xyznot.com/de): "Kernideen", FP8
 *       bullet (E4M3 for all tensors, 1x128 activation tiles, 128x128 weight
 *       blocks, FP32 promotion every N_c = 128 accumulation steps); "Methode"
 *       section 2 "DeepSeekMoE mit Auxiliary-Loss-Free Balancing" (layer
 *       output equation, sigmoid affinity, biased top-K_r gating, gate
 *       normalisation, per-step bias update with gamma = 0.001).
 *  [P1] "DeepSeek-V3 技術報告書：MLAと極小スパースMoEがもたらす超低コストフロンティアモデル"
 *       (singularity-lens.com), formula paragraph: S = max|X| / 448,
 *       X_FP8 = clip(round(X / S), -448, 448); b_i += gamma*sign(mean - f_i).
 *  [P2] "DeepSeek-V3 Technical Report" slides (slideify.app), "FP8
 *       Quantization Logic": 1x128 tiles, 128x128 blocks.
 *  [P3] "DeepSeek-V3 MoE 2024" glossary (jisaku.com): 256 routed experts +
 *       1 shared expert, top-8 per token.
 *
 * Conventions for every entry point
 *  - Pointers named *_dev are device pointers (cudaMalloc'd or from a
 *    framework allocator) owned by the caller; the library keeps no reference
 *    after the call returns (the one exception: the event handles given to
 *    moe_profile_events, kept until the hook is turned off) and allocates no
 *    device memory (moe_route_noalloc's fixed scratch is a static array of
 *    the library image).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; no entry point synchronises the stream except
 *    moe_check_device_error.
 *  - Arguments are validated on the host before anything is enqueued; an
 *    invalid call returns a negative status and enqueues nothing.
 *  - bf16 tensors are passed as raw 16-bit words (const void*), E4M3 codes as
 *    uint8_t (OCP E4M3FN bit patterns), scales as IEEE float.
 *  - Matrices are row-major; "K-contiguous" means the contraction index is
 *    the fastest-varying one.
 *  - Dimensions that the fine-grained scaling tiles (hidden, intermediate,
 *    GEMM N and K) must be multiples of 128, else MOE_ERR_UNSUPPORTED_SHAPE.
 *  - err_flag_dev is an int32 in device memory that kernels set (bitwise OR of
 *    MOE_DEVERR_* codes) when a bounded wait gives up; the caller zeroes it
 *    and reads it after synchronising (moe_check_device_error).  Kernels
 *    never trap or spin forever.
 *  - No C++ exception crosses this boundary.
 */
#ifndef MOE_FP8_H
#define MOE_FP8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,        /* null pointer, bad size, misaligned pointer */
    MOE_ERR_UNSUPPORTED_SHAPE = -2,  /* a tiled dimension is not a multiple of 128, or too large */
    MOE_ERR_WORKSPACE_TOO_SMALL = -3,
    MOE_ERR_CUDA = -4,               /* a CUDA runtime call failed (launch, attribute, ...) */
    MOE_ERR_TIMEOUT = -5,            /* a device-side bounded wait gave up (see err_flag) */
    MOE_ERR_NOT_IMPLEMENTED = -6,
    MOE_ERR_NO_DEVICE = -7,          /* no sm_100 device current */
    MOE_ERR_DEVICE = -8              /* err_flag holds a non-timeout device error */
};

/* bits that kernels OR into *err_flag_dev */
enum {
    MOE_DEVERR_TIMEOUT = 1,          /* an mbarrier wait exceeded its time limit */
    MOE_DEVERR_BAD_INDEX = 2         /* a routed expert index outside [0, n_routed) was seen */
};

/* Output element types for moe_forward. */
enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_F32 = 1 };

/* Human-readable text for a status code (static storage). */
MOE_API const char *moe_status_string(int status);

/* ABI version (major*100 + minor). */
MOE_API int moe_abi_version(void);

/* ----------------------------------------------------------- layer shape */
/* Shape of one DeepSeekMoE layer ([P4] Methode 2; [P3]).
 *   hidden      H, multiple of 128, at most 32768 (7168 in DeepSeek-V3)
 *   inter       I, expert SwiGLU intermediate size, multiple of 128, at
 *               most 32768 (2048)
 *   n_routed    N_r routed experts, 1..256 (256)
 *   top_k       K_r experts per token, 1..min(N_r, 16) (8)
 *   n_shared    N_s always-active experts, 0 or 1 (1)
 *   n_groups    group-limited routing: 0 = off, else number of equal
 *               contiguous expert groups (divides N_r, <= 32, at least two
 *               experts per group: a group's score is the sum of its two
 *               best biased scores)
 *   topk_groups groups kept per token when n_groups > 0 (1..n_groups)
 *   route_scale factor applied to the normalised gates (1.0 = the pages')
 *   scale_mode  MOE_SCALE_AMAX (0, the pages' S = amax / 448, the default of
 *               a zero-initialised config) or MOE_SCALE_POW2 (1: power-of-two
 *               scales, see fp8_quant_1x128_pow2; moe_forward then runs the
 *               expert GEMMs with the scales applied by the tensor core, and
 *               the weights must have been quantized with the _pow2
 *               quantizer) */
#define MOE_SCALE_AMAX 0
#define MOE_SCALE_POW2 1
typedef struct {
    int32_t hidden;
    int32_t inter;
    int32_t n_routed;
    int32_t top_k;
    int32_t n_shared;
    int32_t n_groups;
    int32_t topk_groups;
    float route_scale;
    int32_t scale_mode;
} moe_config;

/* Quantized layer weights, all device pointers, experts stacked routed
 * first (0..N_r-1) then shared (N_r..N_r+N_s-1); E = N_r + N_s.
 *   w13_dev   E4M3 [E, 2I, H]: rows 0..I-1 of each expert are the gate
 *             projection W1, rows I..2I-1 the up projection W3 (K = H
 *             contiguous)
 *   s13_dev   float [E, 2I/128, H/128] 128x128 block scales of w13
 *   w2_dev    E4M3 [E, H, I] down projection (K = I contiguous)
 *   s2_dev    float [E, H/128, I/128]
 *   wr_dev    bf16 [N_r, H] router centroids e_i
 * The E4M3 and bf16 pointers must be 16-byte aligned, the scale pointers
 * 4-byte aligned. */
typedef struct {
    const uint8_t *w13_dev;
    const float *s13_dev;
    const uint8_t *w2_dev;
    const float *s2_dev;
    const void *wr_dev;
} moe_weights;

/* ------------------------------------------------------------ quantizers */
/* 1x128 activation quantization ([P4] Kernideen; [P1] formula; [P2]).
 * For each row r and each group g of 128 consecutive columns:
 *   amax = max |x[r, 128g .. 128g+127]|, S = amax / 448 (FP32, IEEE),
 *   q[r, c] = E4M3_RNE_satfinite(x[r, c] / S) (IEEE FP32 quotient),
 *   scales[r, g] = S;  amax == 0 gives S = 0 and codes 0x00.
 *   x_dev       bf16 [rows, ld_x] (16-byte aligned, ld_x % 8 == 0, ld_x >= cols)
 *   q_dev       E4M3 [rows, cols], dense (16-byte aligned)
 *   scales_dev  float [rows, cols/128], dense
 * rows >= 0 (0 enqueues nothing), cols % 128 == 0. */
MOE_API int fp8_quant_1x128(const void *x_dev, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *q_dev,
                    float *scales_dev, void *stream);

/* 128x128 weight-block quantization (same rule per 128x128 block; setup
 * step, not part of the timed layer).
 *   w_dev       bf16 [n, k] dense, n % 128 == 0, k % 128 == 0
 *   q_dev       E4M3 [n, k];  scales_dev float [n/128, k/128] */
MOE_API int fp8_quant_128x128(const void *w_dev, int64_t n, int64_t k, uint8_t *q_dev, float *scales_dev,
                      void *stream);

/* The same two quantizers with power-of-two scales (not on the pages: the
 * variant whose scales a block-scaled tensor-core MMA applies itself, as
 * 8-bit exponent codes): S = 2^e with e the smallest integer for which
 * amax <= 448 * 2^e, held at 2^-127 or above; amax == 0 gives S = 0.  x / S
 * is then an exact scaling and q = E4M3_RNE_satfinite(x / S).  Arguments,
 * layouts and errors as above. */
MOE_API int fp8_quant_1x128_pow2(const void *x_dev, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *q_dev,
                         float *scales_dev, void *stream);
MOE_API int fp8_quant_128x128_pow2(const void *w_dev, int64_t n, int64_t k, uint8_t *q_dev, float *scales_dev,
                           void *stream);

/* ---------------------------------------------------------------- GEMM */
/* Fine-grained block-scaled FP8 GEMM ([P4] Kernideen):
 *   C[m, n] = sum_kb sA[m, kb] * sB[n/128, kb] * sum_{k in kb} A[m, k] B[n, k]
 * where each 128-long partial is formed on the tensor cores and promoted
 * (scaled and added) into an FP32 accumulator -- promotion every N_c = 128.
 *   A_dev   E4M3 [M, K] K-contiguous;  sA_dev float [M, K/128]
 *   B_dev   E4M3 [N, K] K-contiguous (the weight, "Linear" layout);
 *   sB_dev  float [N/128, K/128]
 *   C_dev   bf16 [M, N] (RNE of the FP32 accumulator)
 * M >= 0 (0 enqueues nothing), N % 128 == 0, K % 128 == 0, K <= 32768;
 * A_dev, B_dev, C_dev 16-byte aligned, sA_dev, sB_dev, err_flag_dev 4-byte
 * aligned. */
MOE_API int fp8_blockscaled_gemm(const uint8_t *A_dev, const float *sA_dev, const uint8_t *B_dev,
                         const float *sB_dev, void *C_dev, int64_t M, int64_t N, int64_t K,
                         int32_t *err_flag_dev, void *stream);

/* -------------------------------------------------------------- routing */
/* Router ([P4] Methode 2): s[t, i] = sigmoid(x_t . e_i) (bf16 inputs, FP32
 * accumulation on the tensor cores); the K_r experts with the largest
 * s[t, i] + bias[i] are selected (ties: lower index; if n_groups > 0 only
 * experts of the topk_groups groups with the largest sum of their two best
 * s + bias are eligible); gate[t, k] = route_scale * s[t, idx[t, k]] /
 * sum_k' s[t, idx[t, k']].  idx lists the selection in descending s + bias.
 *   x_dev      bf16 [T, H] (16-byte aligned)
 *   wr_dev     bf16 [N_r, H]
 *   bias_dev   float [N_r]
 *   idx_dev    int32 [T, K_r];  gate_dev float [T, K_r]
 *   counts_dev int32 [N_r]: per-expert number of selections (overwritten)
 *   ws_dev     scratch of moe_route_workspace_size() bytes (256-byte aligned) */
MOE_API size_t moe_route_workspace_size(const moe_config *cfg, int64_t T);
MOE_API int moe_route(const moe_config *cfg, const void *x_dev, const void *wr_dev, const float *bias_dev,
              int64_t T, int32_t *idx_dev, float *gate_dev, int32_t *counts_dev, void *ws_dev,
              size_t ws_bytes, int32_t *err_flag_dev, void *stream);

/* Allocation-free variant of moe_route (the pages have no counterpart: this
 * is an interface convenience).  Some callers cannot call cudaMalloc or hand
 * the library a scratch buffer -- e.g. a host that owns every byte of device
 * memory through its own planner, or a latency-critical path where an
 * allocation's implicit device synchronisation is not acceptable.  This entry
 * point takes the same inputs and outputs as moe_route but keeps the router's
 * FP32 logit partials in a fixed scratch array inside the library
 * (MOE_ROUTE_NOALLOC_SCRATCH_BYTES = 16 MiB on every GPU that loads the
 * library, held until the process exits) and allocates nothing.
 *   - Limit: the partials moe_route would keep in its workspace must fit,
 *     i.e. moe_route_workspace_size(cfg, T) - 256 <= 16 MiB (for
 *     n_routed = 256 on a 148-SM device every T <= 16384 fits); larger
 *     calls return
 *     MOE_ERR_WORKSPACE_TOO_SMALL and enqueue nothing.
 *   - Every call looks up the scratch's device address in the current
 *     device's context (cudaGetSymbolAddress, which allocates nothing), so
 *     the address stays right after a context is torn down and created
 *     again.  The first call on a device may load the library's device code
 *     into that context: make it before any stream capture.
 *   - Every call shares the one scratch and it keeps the last call's
 *     contents (each call overwrites every partial it reads, so nothing has
 *     to start at zero); calls whose execution overlaps on the GPU race on
 *     it, so serialise them (one stream, or events).
 * Arguments, outputs and error behaviour are otherwise those of moe_route. */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (16u << 20)
MOE_API int moe_route_noalloc(const moe_config *cfg, const void *x_dev, const void *wr_dev,
                              const float *bias_dev, int64_t T, int32_t *idx_dev, float *gate_dev,
                              int32_t *counts_dev, int32_t *err_flag_dev, void *stream);

/* ------------------------------------------------------------ full layer */
/* One DeepSeekMoE layer forward ([P4] Methode 2):
 *   out[t] = u_t + sum_{shared} FFN_s(u_t) + sum_k gate[t, k] FFN_{idx[t,k]}(u_t)
 * with FFN(u) = W2 (silu(W1 u) * (W3 u)), every projection an FP8 block-scaled
 * GEMM: u quantized 1x128 (fp8_quant_1x128), routed as moe_route, rows
 * grouped per expert (stable: token order, then slot), h = silu(G) * U in FP32
 * re-quantized 1x128 along I before the down projection, the down-projection
 * output scaled by the gate (FP32), then summed per token in FP32 in a fixed
 * order (residual, shared expert, slots 0..K_r-1) and written as out_dtype.
 *   x_dev        bf16 [T, H]
 *   out_dev      [T, H] of MOE_DTYPE_BF16 (RNE) or MOE_DTYPE_F32
 *   idx_out_dev  nullable int32 [T, K_r]: routing decision
 *   counts_out_dev nullable int32 [N_r]: per-expert load (input of moe_bias_update)
 *   ws_dev       scratch of moe_workspace_size() bytes, 256-byte aligned; its
 *                layout is reported by moe_workspace_layout (for inspection)
 * T >= 0 (0 enqueues nothing). */
MOE_API size_t moe_workspace_size(const moe_config *cfg, int64_t T);
MOE_API int moe_forward(const moe_config *cfg, const moe_weights *w, const float *bias_dev, const void *x_dev,
                int64_t T, void *out_dev, int32_t out_dtype, int32_t *idx_out_dev,
                int32_t *counts_out_dev, void *ws_dev, size_t ws_bytes, int32_t *err_flag_dev,
                void *stream);

/* Byte offsets of the intermediates inside moe_forward's workspace, for
 * tests and profiling (all 256-byte aligned).  Rows: R = T*K_r routed rows in
 * expert-contiguous order, then T*N_s shared-expert rows in token order.
 * Each entry is {offset, bytes}. */
typedef struct {
    size_t xq[2];       /* E4M3 [T, H]       1x128-quantized input            */
    size_t xs[2];       /* float [T, H/128]                                    */
    size_t idx[2];      /* int32 [T, K_r]                                      */
    size_t gate[2];     /* float [T, K_r]                                      */
    size_t counts[2];   /* int32 [N_r]                                         */
    size_t offsets[2];  /* int32 [N_r + 1]  first row of each expert           */
    size_t pos[2];      /* int32 [T, K_r]   row of (t, k) in expert order      */
    size_t ap[2];       /* E4M3 [R, H]      expert-contiguous copy of xq rows  */
    size_t as[2];       /* float [H/128, P] scales of every row, transposed;
                           P = R + T rounded up to a multiple of 4          */
    size_t row_gate[2]; /* float [R + T*N_s] gate of each row (1 for shared)   */
    size_t row_src[2];  /* int32 [R]        token of each routed row           */
    size_t hq[2];       /* E4M3 [R + T*N_s, I] re-quantized SwiGLU output      */
    size_t hs[2];       /* float [I/128, P] its scales, transposed             */
    size_t y[2];        /* float [R + T*N_s, H] gate-scaled expert outputs     */
    size_t meta[2];     /* int32 [4]: number of chunks, routed rows            */
    size_t logits[2];   /* float [S, T, N_r] router logit partials (S K-splits) */
    size_t blk_hist[2]; /* int32 [ceil(T/128), N_r] per-block expert counts    */
    size_t blk_base[2]; /* int32 [ceil(T/128), N_r] per-block first rows       */
    size_t chunks[2];   /* int32x4 per chunk: {expert | input flag << 16,
                           activation row, output row, rows <= 128 (single
                           CTAs) or <= 256 (CTA pairs)}                        */
    size_t total;
} moe_ws_layout;
MOE_API int moe_workspace_layout(const moe_config *cfg, int64_t T, moe_ws_layout *layout);

/* Measurement hook: when set (n_events >= MOE_PROFILE_EVENTS), every later
 * moe_forward on this host thread records events[i] (caller-created
 * cudaEvent_t handles) on its stream at the stage boundaries below, so
 * per-stage device time can be read with cudaEventElapsedTime.  Pass NULL/0
 * to turn it off.  Events are recorded, never created or destroyed, by the
 * library; recording adds no kernel launches.  The caller keeps the events
 * alive while the hook is set (turn it off before destroying them: a
 * destroyed event makes the next moe_forward return MOE_ERR_CUDA).
 *   0 start | 1 after quantize | 2 after routing | 3 after grouping (hist,
 *   work lists, row copies) | 4 after gate/up GEMM (+SwiGLU, requant) |
 *   5 after down GEMM | 6 after combine */
enum { MOE_PROFILE_EVENTS = 7 };
/* With n_events >= MOE_PROFILE_EVENTS + MOE_PROFILE_BWD_EVENTS, every later
 * moe_backward also records events[MOE_PROFILE_EVENTS + i] at:
 *   0 start | 1 after G, U recomputed | 2 after the dout quantization and
 *   the dh GEMM | 3 after the SwiGLU backward | 4 after the dx-rows GEMM |
 *   5 after the dx combine | 6 after the weight-gradient tiles and the
 *   128x1 quantizations | 7 after the dW2 GEMM | 8 after the dW13 GEMM */
enum { MOE_PROFILE_BWD_EVENTS = 9 };
MOE_API int moe_profile_events(void *const *events, int32_t n_events);

/* ------------------------------------------------------------ backward */
/* Backward of the layer's expert FFNs with the routing held fixed ([P4]
 * Kernideen, FP8 bullet: "E4M3 for all tensors"; the tile orientation is a
 * reading, the DeepSeek-V3 technical report's: each GEMM input quantized
 * along that GEMM's contraction).  For out_t = u_t + FFN_s(u_t) +
 * sum_k g_{t,k} FFN_{e_{t,k}}(u_t) and a gradient dout of out:
 *   every expert row p (token t, gate g; g = 1 for the shared expert)
 *   receives dY_p = g * dout_t, and the gate is kept out of every
 *   quantized tile of dY: a 1x128 tile of g * dout has the codes of dout's
 *   tile (g cancels in the quotient), so
 *   G, U recomputed (the forward's gate/up GEMM, FP32 results);
 *   dh = g (dout_t W2)  (dout 1x128 along H, W2's blocks transposed; g
 *                        times the FP32 result)
 *   dG = dh U silu'(G), dU = dh silu(G), h = silu(G) U       (FP32)
 *   dx_p = dG W1 + dU W3  (dG, dU 1x128 along I, W1/W3's blocks transposed)
 *   dx_t = dout_t + sum over the token's rows of dx_p         (FP32)
 *   dW2_e = dout_e^T (g h)_e (= dY_e^T h_e), dW13_e = [dG | dU]_e^T x_e
 *   over expert e's tokens (both operands 128x1 along tokens: one scale per
 *   channel per 128 tokens, a ragged last tile shorter; every GEMM promotes
 *   each 128-long partial into FP32).
 * The gates' own gradient (router backward) is not part of this.
 *
 * moe_transpose_weights (set-up): the dgrad GEMMs' weights, each expert's
 * codes and 128x128 block scales transposed:
 *   w13t_dev E4M3 [E, H, 2I], s13t_dev float [E, H/128, 2I/128]
 *   w2t_dev  E4M3 [E, I, H],  s2t_dev  float [E, I/128, H/128]
 * moe_backward: call after the moe_forward of the same batch, same cfg and T,
 * passing that forward's workspace (fwd_ws_dev), whose routing and grouping
 * it reuses.
 *   x_dev     bf16 [T, H] the forward's input;  dout_dev bf16 [T, H]
 *   dx_dev    float [T, H]
 *   dW13_dev  float [E, 2I, H] (rows 0..I-1 gate W1, I..2I-1 up W3)
 *   dW2_dev   float [E, H, I]  (an expert no token selected gets zeros)
 *   ws_dev    moe_backward_workspace_size() bytes, 256-byte aligned
 * T >= 1; only scale_mode MOE_SCALE_AMAX (else MOE_ERR_NOT_IMPLEMENTED). */
MOE_API int moe_transpose_weights(const moe_config *cfg, const moe_weights *w, uint8_t *w13t_dev, float *s13t_dev,
                                  uint8_t *w2t_dev, float *s2t_dev, void *stream);
MOE_API size_t moe_backward_workspace_size(const moe_config *cfg, int64_t T);
/* Byte offsets {offset, bytes} of the backward's intermediates inside its
 * workspace (for tests and inspection), rows in the forward's row order
 * (RS = T*K_r + T*N_s): gu float [RS, 2I] (G then U), dh float [RS, I] (with
 * the gate), gh float [RS, I] (the row's gate times h),
 * dgu float [RS, 2I] (dG then dU), dx_rows float [RS, H], seg int32 [E + 1]
 * (each expert's token segment of the weight-gradient operands, P columns). */
typedef struct {
    size_t gu[2], dh[2], gh[2], dgu[2], dx_rows[2], seg[2];
    int64_t P;
    size_t total;
} moe_bwd_layout;
MOE_API int moe_backward_workspace_layout(const moe_config *cfg, int64_t T, moe_bwd_layout *layout);
MOE_API int moe_backward(const moe_config *cfg, const moe_weights *w, const uint8_t *w13t_dev,
                         const float *s13t_dev, const uint8_t *w2t_dev, const float *s2t_dev, const void *x_dev,
                         const void *dout_dev, int64_t T, float *dx_dev, float *dW13_dev, float *dW2_dev,
                         const void *fwd_ws_dev, size_t fwd_ws_bytes, void *ws_dev, size_t ws_bytes,
                         int32_t *err_flag_dev, void *stream);

/* ------------------------------------------------- expert parallelism */
/* The layer with its routed experts spread over W ranks (one GPU each), as
 * the DeepSeek-V3 pages run it: tokens travel to the GPUs of their experts
 * and the expert outputs travel back by all-to-all exchanges ([P4] "Problem
 * und Motivation" item 2 and "Kernideen", DualPipe bullet).  Rank d owns the
 * routed experts [d*N_r/W, (d+1)*N_r/W) (N_r % W == 0); every rank holds the
 * router, the shared expert and its own tokens.  The exchanges themselves are
 * the caller's collectives (e.g. NCCL all-to-all over NVLink); these calls
 * are the compute on either side of them.  One rank's forward:
 *   1. fp8_quant_1x128 and moe_route on its tokens (xq, xs, idx, gate);
 *   2. moe_ep_dispatch: packed rows per destination (send buffer), the row
 *      counts and offsets per destination, each token's row per destination;
 *   3. exchange: rows r -> d (all-to-all, send_counts rows of
 *      moe_ep_row_bytes each);
 *   4. moe_ep_experts on the received rows with this rank's experts: the
 *      gate-weighted sum over each row's slots whose experts live here
 *      (bf16 partial sums, one per received row);
 *   5. exchange back: the partial sums d -> r (the reverse all-to-all);
 *   6. moe_ep_experts on self_rows with the shared expert's weights
 *      (n_routed = 1, gate 1) gives y_shared; moe_ep_combine adds u_t,
 *      y_shared and the returned partial sums (destinations in ascending
 *      order) in FP32.
 * Packed row (moe_ep_row_bytes bytes, a multiple of 16): the token's H E4M3
 * codes, its H/128 FP32 scales, K_r int32 local expert ids (-1: the slot's
 * expert lives elsewhere) and K_r FP32 gates (0 where -1).
 * The result equals moe_forward's up to the order of the FP32 additions and
 * the bf16 rounding of the partial sums. */
MOE_API int64_t moe_ep_row_bytes(const moe_config *cfg);

/* Dispatch of one rank's T routed tokens (step 2).
 *   cfg           the whole layer's shape (n_routed = all routed experts)
 *   world         W, 1..64, dividing n_routed
 *   xq_dev, xs_dev the tokens quantized 1x128 (E4M3 [T, H], float [T, H/128])
 *   idx_dev, gate_dev routing decision [T, K_r] (moe_route's outputs)
 *   send_rows_dev packed rows [send_cap_rows, moe_ep_row_bytes], grouped by
 *                 destination (rank order), token order within a
 *                 destination; send_cap_rows >= T * min(W, K_r)
 *   send_counts_dev int32 [W]: rows for each destination (device; copy it
 *                 to the host to size the exchange)
 *   send_offsets_dev int32 [W + 1]: first row of each destination, total
 *   row_of_dev    int32 [T, W]: row of token t for destination d, or -1
 *   self_rows_dev nullable [T, moe_ep_row_bytes]: every token packed for the
 *                 shared expert (slot 0 = expert 0, gate 1)
 *   ws_dev        moe_ep_dispatch_workspace_size() bytes, 256-byte aligned
 * err_flag_dev gets MOE_DEVERR_BAD_INDEX for an expert index out of range. */
MOE_API size_t moe_ep_dispatch_workspace_size(const moe_config *cfg, int32_t world, int64_t T);
MOE_API int moe_ep_dispatch(const moe_config *cfg, int32_t world, const uint8_t *xq_dev, const float *xs_dev,
                            const int32_t *idx_dev, const float *gate_dev, int64_t T, uint8_t *send_rows_dev,
                            int64_t send_cap_rows, int32_t *send_counts_dev, int32_t *send_offsets_dev,
                            int32_t *row_of_dev, uint8_t *self_rows_dev, void *ws_dev, size_t ws_bytes,
                            int32_t *err_flag_dev, void *stream);

/* The experts of one rank over received packed rows (steps 4 and 6).
 *   cfg_local     n_routed = the rank's experts (N_r / W, or 1 for the
 *                 shared expert), top_k = the layer's K_r (the slots of a
 *                 packed row; it may exceed n_routed), n_shared = 0,
 *                 n_groups = 0, other fields as the layer's
 *   w_local       those experts' weights (layout of moe_weights; wr_dev unused)
 *   rows_dev      n_rows packed rows, row_bytes = moe_ep_row_bytes(cfg_local)
 *   partial_out_dev bf16 [n_rows, H]: per row, the sum over its slots of
 *                 gate * FFN_expert(row) in FP32 (slot order), rounded to bf16
 *   ws_dev        moe_ep_experts_workspace_size() bytes, 256-byte aligned */
MOE_API size_t moe_ep_experts_workspace_size(const moe_config *cfg_local, int64_t n_rows);
MOE_API int moe_ep_experts(const moe_config *cfg_local, const moe_weights *w_local, const uint8_t *rows_dev,
                           int64_t n_rows, int64_t row_bytes, void *partial_out_dev, void *ws_dev, size_t ws_bytes,
                           int32_t *err_flag_dev, void *stream);

/* Combine on the sending rank (step 6): out[t] = u_t + y_shared[t] (if given)
 * + sum over d = 0..W-1 with row_of[t, d] >= 0 of back[row_of[t, d]], in FP32,
 * written as out_dtype.
 *   x_dev         bf16 [T, H] (the layer input u_t)
 *   row_of_dev    moe_ep_dispatch's int32 [T, W]
 *   back_dev      bf16 [send rows, H]: the partial sums returned by the
 *                 destinations, in the send buffer's row order
 *   y_shared_dev  nullable bf16 [T, H] */
MOE_API int moe_ep_combine(const moe_config *cfg, int32_t world, const void *x_dev, int64_t T,
                           const int32_t *row_of_dev, const void *back_dev, const void *y_shared_dev, void *out_dev,
                           int32_t out_dtype, void *stream);

/* Kernel choice of the grouped expert GEMMs in the default scale mode
 * (process-wide; a tuning and testing switch, the arithmetic is the same):
 *   MOE_GEMM_AUTO   (default) the measured-fastest choice: single CTAs
 *   MOE_GEMM_SINGLE one CTA per tile: <= 128 rows of one expert per pass over
 *                   a weight-block pair
 *   MOE_GEMM_PAIR   a pair of CTAs on two SMs per tile (<= 256 rows per
 *                   weight pass, one tcgen05.mma.cta_group::2 per K step)
 *                   when the down projection's 128-row weight blocks pair up
 *                   (hidden a multiple of 256), else single CTAs
 *   MOE_GEMM_TALL   tall tiles: up to 256 rows of an expert x 64 gate + 64 up
 *                   channels (or 128 output channels) per CTA, so an expert
 *                   of up to 256 rows streams each weight tile once; clusters
 *                   of two exchange the requantization amax (hidden a
 *                   multiple of 256, else single CTAs)
 * Returns MOE_ERR_INVALID_ARG for any other value.  Takes effect for the
 * next moe_forward on any thread; not synchronised with calls in flight. */
enum { MOE_GEMM_AUTO = 0, MOE_GEMM_SINGLE = 1, MOE_GEMM_PAIR = 2, MOE_GEMM_BLOCK_SCALED = 3, MOE_GEMM_TALL = 4 };
MOE_API int moe_set_gemm_variant(int32_t variant);
/* The grouped-GEMM kernel the next moe_forward of T tokens under cfg runs
 * with the current variant setting: MOE_GEMM_SINGLE, MOE_GEMM_PAIR, or
 * MOE_GEMM_BLOCK_SCALED (scale_mode MOE_SCALE_POW2: the tensor core applies
 * the power-of-two scales), or a (negative) error status for an invalid
 * cfg or T.  Host-only; no device work. */
MOE_API int moe_gemm_kernel_for(const moe_config *cfg, int64_t T);

/* --------------------------------------------------------- bias update */
/* Auxiliary-loss-free balancing step ([P4] Methode 2; [P1]): with
 * mean = total_assignments / n_routed, bias[i] -= gamma if counts[i] > mean,
 * bias[i] += gamma if counts[i] < mean, unchanged if equal (FP32, in place).
 *   bias_dev float [n_routed];  counts_dev int32 [n_routed] */
MOE_API int moe_bias_update(float *bias_dev, const int32_t *counts_dev, int32_t n_routed,
                    int64_t total_assignments, float gamma, void *stream);

/* Sequence-wise balance loss of the batch the last moe_forward routed ([P4]
 * Methode 2 names this complementary loss and its weight alpha = 0.0001 but
 * prints no formula; the form is the DeepSeek-V3 technical report's).  For
 * each run of seq_len consecutive tokens (L = seq_len):
 *   f_i  = N_r / (K_r L) * (tokens of the run that select expert i)
 *   P_i  = (1/L) * sum_t s_{i,t} / sum_j s_{j,t}   (s: sigmoid affinities)
 *   loss = alpha * sum_i f_i P_i                    (FP32)
 * It reads the router's logit partials and routing decision that moe_forward
 * leaves in its workspace, so call it on the same stream, after that
 * moe_forward, with the same cfg, T and workspace.  A metric of the routing:
 * nothing in the forward pass depends on it.
 *   T            tokens of that forward; a multiple of seq_len (else
 *                MOE_ERR_INVALID_ARG); T == 0 enqueues nothing
 *   ws_dev       that forward's workspace (256-byte aligned, ws_bytes >=
 *                moe_workspace_size(cfg, T))
 *   loss_dev     float [T / seq_len], 4-byte aligned
 *   err_flag_dev gets MOE_DEVERR_BAD_INDEX if a routed index is out of range */
MOE_API int moe_seq_balance_loss(const moe_config *cfg, int64_t T, int64_t seq_len, float alpha,
                                 const void *ws_dev, size_t ws_bytes, float *loss_dev, int32_t *err_flag_dev,
                                 void *stream);

/* ------------------------------------------------------------ errors */
/* Synchronises `stream`, copies *err_flag_dev to *host_value (nullable) and
 * returns MOE_OK if it is 0, MOE_ERR_TIMEOUT if the timeout bit is set, else
 * MOE_ERR_DEVICE.  Does not clear the flag. */
MOE_API int moe_check_device_error(const int32_t *err_flag_dev, int32_t *host_value, void *stream);

/* Failure-detection self test: launches one block whose thread waits on an
 * mbarrier that nothing arrives on, with a wait limit of limit_us
 * microseconds (1..10^6).  The wait gives up, sets MOE_DEVERR_TIMEOUT in
 * *err_flag_dev and the kernel returns; the context stays usable. */
MOE_API int moe_selftest_wait_timeout(int32_t *err_flag_dev, int64_t limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FP8_H */
