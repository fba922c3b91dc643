// kernels.h -- host-side launchers of the libmoefp8 kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace moe {

// Raise a kernel's dynamic shared-memory limit once per device: the attribute
// belongs to the current device's context, so a process that drives several
// GPUs sets it on each.  `done` keeps one bit per device ordinal (< 64;
// higher ordinals set it on every call).
template <typename Fn>
inline cudaError_t smem_attr_once(Fn *fn, int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// One unit of work of the grouped block-scaled GEMM, decoded on the device
// from a chunk (<= 128 activation rows of one expert) and a weight-block pair.
struct GemmTile {
  int32_t w_row0;   // first row of weight block A in the weight tensor
  int32_t w_row1;   // first row of weight block B, or -1
  int32_t a_row;    // first activation row (in the tensor map the tile reads)
  int32_t n;        // activation rows in this tile, 1..128 (one CTA) or 1..256 (a CTA pair)
  int32_t out_row;  // first output row (also the column of the transposed scales)
  int32_t out_col;  // first output column of block A's outputs
  int32_t from1;    // activations come from the second tensor map
  int32_t group;    // chunks of this tile's expert (their tiles of one weight block run side by side)
};

// Chunk table entry (int4), written by build_chunks_kernel:
//   x = expert | from1 << 16 | (index of the chunk among its expert's) << 17
//   y = first activation row, z = first output row,
//   w = rows | (chunks of the expert) << 16
// Field accessors shared by every kernel that reads the table.
__host__ __device__ inline int chunk_expert(const int4 &c) { return c.x & 0xFFFF; }
__host__ __device__ inline int chunk_from1(const int4 &c) { return (c.x >> 16) & 1; }
__host__ __device__ inline int chunk_pos(const int4 &c) { return (c.x >> 17) & 0x7FFF; }
__host__ __device__ inline int chunk_rows_of(const int4 &c) { return c.w & 0xFFFF; }
__host__ __device__ inline int chunk_group(const int4 &c) { return (c.w >> 16) & 0x7FFF; }

enum EpiKind : int { EPI_SWIGLU_Q = 0, EPI_GATE_F32 = 1, EPI_BF16 = 2, EPI_F32 = 3 };

struct GemmLaunch {
  // tensor operands
  const uint8_t *w;       // weights [w_rows, K]
  int64_t w_rows;
  const uint8_t *a0;      // activations [a0_rows, K]
  int64_t a0_rows;
  const uint8_t *a1;      // second activation tensor (may equal a0)
  int64_t a1_rows;
  int64_t a1_ld;          // bytes between a1 rows (0: K); a multiple of 16
  int64_t K;
  const float *sw;        // weight scales [w_rows/128, K/128]
  const float *sa0;       // activation scales [a0_rows, K/128]
  const float *sa1;
  // work: a chunk table (chunks != null, count at n_chunks[0]) or the dense
  // grid of a plain GEMM (dense_M rows); nb weight-block pairs per chunk
  const int4 *chunks;
  const int32_t *n_chunks;
  int max_chunks;          // host-side upper bound (grid sizing)
  int chunk_rows;          // most rows per chunk: 128 (one CTA per tile) or 256 (a CTA pair per tile)
  int64_t dense_M;
  int nb;                  // weight-block pairs per chunk
  int gate_up;             // pair block j with block j + half (SwiGLU) instead of 2j, 2j+1
  int a_is_out_row;        // activation row = the chunk's output row (input is a previous GEMM's output)
  int64_t half;            // I for the gate/up GEMM
  int64_t rows_per_expert; // weight rows per expert (2I, H, or N for the dense GEMM)
  int sa_transposed;       // activation scales stored [K/128][sa_ld] (column = out_row)
  int64_t sa_ld;
  // epilogue
  int epi;
  void *out;
  int64_t ldo;
  int64_t out_rows;       // rows of `out` (bounds check)
  int64_t out_cols;       // output columns addressable per row (bounds check)
  float *out_scale;       // EPI_SWIGLU_Q: transposed scales [I/128][ld_os], column = row
  int64_t ld_os;
  const float *row_gate;
  int32_t *err;
  uint64_t wait_limit_ns;
};

// pow2: power-of-two scales (pow2_scale) instead of S = amax / 448
cudaError_t launch_quant_1x128(const void *x, int64_t rows, int64_t cols, int64_t ldx, uint8_t *q, float *s,
                               cudaStream_t st, bool pow2 = false);
cudaError_t launch_quant_128x128(const void *w, int64_t n, int64_t k, uint8_t *q, float *s, cudaStream_t st,
                                 bool pow2 = false);

int router_ksplit(int64_t T, int Nr, int H);
// capacity of the fixed router scratch used by moe_route_noalloc (floats)
constexpr size_t kRouteNoAllocScratchFloats = size_t(4) << 20;
cudaError_t route_static_scratch(float **ptr);
cudaError_t launch_router_logits(const void *x, const void *wr, int64_t T, int Nr, int H, float *partial,
                                 int32_t *err, uint64_t limit_ns, cudaStream_t st);
cudaError_t launch_router_topk(const float *partial, int n_ks, int64_t T, int Nr, int Kr, int n_groups,
                               int topk_groups, float route_scale, const float *bias, int32_t *idx, float *gate,
                               int32_t *counts, cudaStream_t st);

// Sequence-wise balance loss of each run of seq_len tokens (T % seq_len == 0)
// from the router's logit partials and routing decision.
cudaError_t launch_seq_balance(const float *partial, int n_ks, int64_t T, int Nr, const int32_t *idx, int Kr,
                               int64_t seq_len, float alpha, float *loss, int32_t *err, cudaStream_t st);

cudaError_t launch_hist(const int32_t *idx, int64_t T, int Kr, int Nr, int allow_empty, int32_t *blk_hist,
                        int32_t *err, cudaStream_t st);
cudaError_t launch_build_chunks(const int32_t *blk_hist, int64_t T, int Kr, int Nr, int Ns, int chunk_rows,
                                int32_t *counts, int32_t *offsets, int32_t *blk_base, int4 *chunks, int32_t *meta,
                                int32_t *counts_out, cudaStream_t st);
cudaError_t launch_rank(const int32_t *idx, const float *gate, int64_t T, int Kr, int Nr, int Ns,
                        const int32_t *blk_base, float *row_gate, int32_t *row_src, int32_t *pos, cudaStream_t st);
cudaError_t launch_copy_rows(const uint8_t *xq, int64_t xq_ld, const float *xs, const int32_t *row_src, int64_t R,
                             int64_t T, int Ns, int H, uint8_t *ap, float *as_t, int64_t ld, cudaStream_t st);
// Row pitch of the transposed scale tables [K/128][pitch]: R + T rounded up to
// 4 floats (16-byte aligned rows for bulk copies); the tables carry
// kScaleSlack floats after their last row so a 260-float copy stays in bounds.
inline int64_t scale_pitch(int64_t R, int64_t T) { return (R + T + 3) / 4 * 4; }
constexpr int64_t kScaleSlack = 264;

cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t st);
// The same GEMM on CTA pairs (clusters of two): chunk_rows = 256, one
// tcgen05.mma.cta_group::2 per 32-long K step over both CTAs' tiles; the
// weight-block count per expert must be even (always true for gate/up).
cudaError_t launch_gemm_pair(const GemmLaunch &g, cudaStream_t st);
// Tall tiles (gemm_tall.cu): up to 256 rows per weight pass on one CTA,
// clusters of two for the 1x128 requantization; chunk_rows 256, transposed
// activation scales, EPI_SWIGLU_Q / EPI_GATE_F32 / EPI_F32; gate/up: nb = I/128,
// down: nb = H/256.
cudaError_t launch_gemm_tall(const GemmLaunch &g, cudaStream_t st);
// The same grouped GEMM with power-of-two scales applied by the tensor core
// (block-scaled MMA); transposed activation scales, EPI_SWIGLU_Q (with
// power-of-two requantization) or EPI_GATE_F32 only.
cudaError_t launch_gemm_mx(const GemmLaunch &g, cudaStream_t st);

// out[t] = x[t] (when x is not null) + y[R + t] (when Ns) + sum_k y[pos[t, k]]
// (pos >= 0), FP32 in that order, written as FP32 or bf16 (RNE)
// (y rows bf16, or FP32 when y_f32)
cudaError_t launch_combine(const void *x, const void *y, const int32_t *pos, int64_t T, int H, int Kr,
                           int64_t R, int Ns, void *out, int out_f32, cudaStream_t st, bool y_f32 = false);
// Expert parallelism (ep.cu): dispatch of one rank's routed tokens into a
// send buffer ordered by destination, the receiving side's unpacking of the
// packed rows, and the sending side's combine of the returned partial sums.
cudaError_t launch_ep_dispatch(const uint8_t *xq, const float *xs, const int32_t *idx, const float *gate, int64_t T,
                               int H, int Kr, int Nr, int W, int32_t *blk_cnt, int32_t *blk_base,
                               int32_t *send_counts, int32_t *send_off, int32_t *row_of, uint8_t *send,
                               int64_t row_bytes, uint8_t *self_rows, int32_t *err, cudaStream_t st);
cudaError_t launch_ep_unpack(const uint8_t *rows, int64_t n, int64_t row_bytes, int H, int Kr, int n_local,
                             int32_t *idx, float *gate, float *xs, int32_t *err, cudaStream_t st);
cudaError_t launch_ep_combine(const void *x, const void *y_sh, const void *back, const int32_t *row_of, int64_t T,
                              int W, int H, void *out, int out_f32, cudaStream_t st);

// Backward of the expert FFNs (backward.cu, gemm_wgrad.cu).
cudaError_t launch_transpose_blocks(const uint8_t *q, const float *s, int64_t n, int64_t k, int64_t batch,
                                    uint8_t *qt, float *st, cudaStream_t stream);
cudaError_t launch_dout_quant(const void *dout, const int32_t *row_src, int64_t R, int64_t RS, int H, uint8_t *q,
                              float *s_t, int64_t ld, cudaStream_t st);
cudaError_t launch_swiglu_bwd(const float *GU, const float *dh, const float *row_gate, int64_t RS, int I, float *h,
                              float *dGU, uint8_t *q, float *s_t, int64_t ld, cudaStream_t st);
cudaError_t launch_wgrad_tiles(const int32_t *offsets, int Nr, int Ns, int64_t R, int64_t T, int32_t *seg,
                               int4 *tiles, int32_t *meta, cudaStream_t st);
// src: 0 = FP32 rows (f32rows, f32_ld floats apart), 1 = bf16 [T, C] rows
// gathered by the row's token (row_src for p < R, p - R after)
cudaError_t launch_colquant(int src, const int4 *tiles, const int32_t *meta, int max_tiles, const float *f32rows,
                            int64_t f32_ld, const void *bf16rows, const int32_t *row_src, int64_t R, int C,
                            uint8_t *out, int64_t out_ld, float *s_t, cudaStream_t st);

// Weight-gradient GEMM: dW[e] = A_e^T B_e over each expert's token segment.
struct WgradLaunch {
  const uint8_t *a_t;    // E4M3 [C_out, P] (tokens contiguous)
  const uint8_t *b_t;    // E4M3 [C_in, P]
  const float *sa_t;     // [P/128][C_out]
  const float *sb_t;     // [P/128][C_in]
  const int32_t *seg;    // [E + 1] segment starts (multiples of 128), seg[E] <= P
  int E;
  int64_t C_out, C_in, P;
  float *out;            // FP32 [E, C_out, C_in]
  int32_t *err;
  uint64_t wait_limit_ns;
};
cudaError_t launch_gemm_wgrad(const WgradLaunch &g, cudaStream_t st);

cudaError_t launch_bias_update(float *bias, const int32_t *counts, int Nr, int64_t total, float gamma,
                               cudaStream_t st);
cudaError_t launch_wait_selftest(int32_t *err, uint64_t limit_ns, cudaStream_t st);

// weight-block pairs (tiles) per chunk of activations in each grouped GEMM
__host__ __device__ inline int gemm1_blocks(int I) { return I / 128; }
__host__ __device__ inline int gemm2_blocks(int H) { return (H / 128 + 1) / 2; }
// upper bound on chunks of <= 128 rows over all experts
inline int64_t max_chunks(int64_t T, int Kr, int Nr, int Ns) {
  return (T * Kr) / 128 + Nr + 1 + (Ns ? (T + 127) / 128 : 0);
}

}  // namespace moe
