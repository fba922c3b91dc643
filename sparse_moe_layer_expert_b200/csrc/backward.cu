// backward.cu -- the FP8 backward of the layer's expert FFNs (routing held
// fixed): the elementwise and quantization kernels around the grouped GEMMs.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Kernideen, FP8 bullet:
// E4M3 for all tensors, fine-grained scales, FP32 accumulation promoted per
// 128-long block.  The pages give no backward tile orientation; the one used
// is the DeepSeek-V3 technical report's: every GEMM input quantized along
// that GEMM's contraction -- the data gradients (dgrad) take the incoming
// gradient as 1x128 tiles along its row and the weights as the forward's
// 128x128 blocks transposed; the weight gradients (wgrad) take both operands
// as 128x1 tiles along tokens (a ragged last tile holds fewer).
//
// With the forward's row order (routed rows per expert in token order, then
// the shared expert's rows), one layer-output gradient dout [T, H] and the
// row gates g_p (1 for the shared expert), row p's output gradient is
// dY[p] = g_p dout[token(p)].  The gate is kept out of every quantized tile
// of dY: a 1x128 tile of g D has the codes of D's tile (g cancels in the
// quotient), so the dgrad quantizes dout and scales its FP32 result by g;
// the wgrad carries g on h (dY^T h = dout^T (g h)).
//   G, U   = the forward's gate/up GEMM, FP32          (grouped GEMM, EPI_F32)
//   dh     = g (dout W2)  (dout 1x128 along H)   (grouped GEMM, EPI_GATE_F32)
//   h      = silu(G) U,   dG = dh U silu'(G),   dU = dh silu(G)   (FP32)
//   dx_p   = dG W1 + dU W3  (dG|dU 1x128 along I)     (grouped GEMM, FP32)
//   dx_t   = dout_t + sum over the token's rows of dx_p   (the combine)
//   dW2_e  = dout_e^T (g h)_e,  dW13_e = [dG|dU]_e^T x_e  (128x1 along
//                                                   tokens; gemm_wgrad.cu)
//
// Kernels here:
//   transpose_blocks_kernel  E4M3 [n, k] with [n/128, k/128] block scales ->
//                            the transpose [k, n] and [k/128, n/128] (set-up
//                            of the dgrad weights)
//   dout_quant_kernel        dout rows in the forward's row order, 1x128
//                            along H -> codes + transposed scale table (the
//                            dgrad GEMM's A operand)
//   swiglu_bwd_kernel        g h, dG, dU from G, U, dh; dG|dU 1x128 along I
//   wgrad_tiles_kernel       per expert: its padded token segment and its
//                            128-token tiles
//   colquant_kernel          128x1 tiles along an expert's tokens, stored
//                            transposed (channel-major: K-major for wgrad)
#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------- transpose
// One CTA per 128x128 block: codes through shared memory, the block's scale
// moved to its transposed place.
__global__ void __launch_bounds__(256) transpose_blocks_kernel(const uint8_t *__restrict__ q,
                                                                const float *__restrict__ s, int64_t n, int64_t k,
                                                                uint8_t *__restrict__ qt, float *__restrict__ st) {
  __shared__ uint8_t tile[128][129];
  const int64_t nk = k / 128, nn = n / 128;
  const int64_t batch = blockIdx.y;
  const int64_t bi = blockIdx.x / nk, bj = blockIdx.x - (blockIdx.x / nk) * nk;
  const uint8_t *src = q + batch * n * k;
  uint8_t *dst = qt + batch * n * k;
  for (int i = threadIdx.x; i < 128 * 128; i += blockDim.x) {
    const int r = i >> 7, c = i & 127;
    tile[r][c] = src[(bi * 128 + r) * k + bj * 128 + c];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 128 * 128; i += blockDim.x) {
    const int r = i >> 7, c = i & 127;  // row r of the transposed block = column r of the block
    dst[(bj * 128 + r) * n + bi * 128 + c] = tile[c][r];
  }
  if (threadIdx.x == 0) st[batch * nn * nk + bj * nn + bi] = s[batch * nn * nk + bi * nk + bj];
}

// --------------------------------------------------------------- helpers
// 16 lanes hold a 128-long group, 8 values each: amax over the group, S, the
// codes (the correctly rounded quotient x / S, E4M3 RNE satfinite, as the
// forward quantizer).
__device__ __forceinline__ float group_scale16(const float (&f)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  return amax / 448.0f;
}

// The correctly rounded quotient v / S of values sharing one divisor: through
// the reciprocal y = RN(1/S) plus one residual correction (div_by_recip,
// common.cuh) for S >= 2^-100, by the division itself below that.
__device__ __forceinline__ float quot(float v, float S, float y) {
  return S >= 0x1p-100f ? div_by_recip(v, S, y) : v / S;
}

__device__ __forceinline__ uint2 codes8_div(const float (&f)[8], float S) {
  uint32_t lo = 0, hi = 0;
  if (S != 0.0f) {
    const float y = __frcp_rn(S);
#pragma unroll
    for (int i = 0; i < 4; ++i) lo |= static_cast<uint32_t>(e4m3_rn_sat(quot(f[i], S, y))) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) hi |= static_cast<uint32_t>(e4m3_rn_sat(quot(f[4 + i], S, y))) << (8 * i);
  }
  return make_uint2(lo, hi);
}

// ------------------------------------------------------------ dout rows
// Row p of the forward's row order: token t = row_src[p] (routed, p < R) or
// p - R (shared); dout[t] quantized 1x128 along H: codes [RS, H], scales
// into the transposed table [H/128][ld].
__global__ void __launch_bounds__(256) dout_quant_kernel(const uint16_t *__restrict__ dout,
                                                          const int32_t *__restrict__ row_src, int64_t R,
                                                          int64_t RS, int H, uint8_t *__restrict__ q,
                                                          float *__restrict__ s_t, int64_t ld) {
  const int64_t groups = H / 128;
  const int64_t gid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int sub = threadIdx.x & 15;
  const bool valid = gid < RS * groups;
  const int64_t p = valid ? gid / groups : 0;
  const int64_t g = valid ? gid - p * groups : 0;
  float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (valid) {
    const int64_t t = p < R ? row_src[p] : p - R;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(dout + t * H + g * 128 + sub * 8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  const float S = group_scale16(f);
  if (valid) {
    *reinterpret_cast<uint2 *>(q + p * H + g * 128 + sub * 8) = codes8_div(f, S);
    if (sub == 0) s_t[g * ld + p] = S;
  }
}

// --------------------------------------------------------- SwiGLU backward
// Per row p and 128-channel group j of I (one warp: 4 channels per lane),
// with dh already carrying the row's gate g:
//   sig = 1/(1+exp(-G)), silu = G sig, h = silu U,
//   dG = dh U sig (1 + G (1 - sig)), dU = dh silu          (FP32)
// Writes gh = g h [RS, I] (the dW2 operand) and dGU [RS, 2I] (dG at column
// c, dU at I + c) in FP32, and dG | dU quantized 1x128 along I: codes
// [RS, 2I], scales into the transposed table [2I/128][ld].
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const float *__restrict__ GU, const float *__restrict__ dh,
                                                          const float *__restrict__ row_gate, int64_t RS, int I,
                                                          float *__restrict__ h,
                                                          float *__restrict__ dGU, uint8_t *__restrict__ q,
                                                          float *__restrict__ s_t, int64_t ld) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t groups = I / 128;
  if (wid >= RS * groups) return;
  const int64_t p = wid / groups, j = wid - (wid / groups) * groups;
  const int64_t c = j * 128 + lane * 4;
  const float4 G4 = *reinterpret_cast<const float4 *>(GU + p * 2 * I + c);
  const float4 U4 = *reinterpret_cast<const float4 *>(GU + p * 2 * I + I + c);
  const float4 D4 = *reinterpret_cast<const float4 *>(dh + p * I + c);
  const float G[4] = {G4.x, G4.y, G4.z, G4.w}, U[4] = {U4.x, U4.y, U4.z, U4.w}, D[4] = {D4.x, D4.y, D4.z, D4.w};
  const float gt = __ldg(row_gate + p);
  float hv[4], dg[4], du[4];
  float ag = 0.0f, au = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float sig = 1.0f / (1.0f + expf(-G[i]));
    const float silu = G[i] * sig;
    hv[i] = gt * (silu * U[i]);
    dg[i] = D[i] * U[i] * sig * (1.0f + G[i] * (1.0f - sig));
    du[i] = D[i] * silu;
    ag = fmaxf(ag, fabsf(dg[i]));
    au = fmaxf(au, fabsf(du[i]));
  }
  *reinterpret_cast<float4 *>(h + p * I + c) = make_float4(hv[0], hv[1], hv[2], hv[3]);
  *reinterpret_cast<float4 *>(dGU + p * 2 * I + c) = make_float4(dg[0], dg[1], dg[2], dg[3]);
  *reinterpret_cast<float4 *>(dGU + p * 2 * I + I + c) = make_float4(du[0], du[1], du[2], du[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ag = fmaxf(ag, __shfl_xor_sync(0xffffffffu, ag, o));
    au = fmaxf(au, __shfl_xor_sync(0xffffffffu, au, o));
  }
  const float Sg = ag / 448.0f, Su = au / 448.0f;
  uint32_t wg = 0, wu = 0;
  if (Sg != 0.0f) {
    const float y = __frcp_rn(Sg);
#pragma unroll
    for (int i = 0; i < 4; ++i) wg |= static_cast<uint32_t>(e4m3_rn_sat(quot(dg[i], Sg, y))) << (8 * i);
  }
  if (Su != 0.0f) {
    const float y = __frcp_rn(Su);
#pragma unroll
    for (int i = 0; i < 4; ++i) wu |= static_cast<uint32_t>(e4m3_rn_sat(quot(du[i], Su, y))) << (8 * i);
  }
  *reinterpret_cast<uint32_t *>(q + p * 2 * I + c) = wg;
  *reinterpret_cast<uint32_t *>(q + p * 2 * I + I + c) = wu;
  if (lane == 0) {
    s_t[j * ld + p] = Sg;
    s_t[(groups + j) * ld + p] = Su;
  }
}

// ------------------------------------------------- wgrad token segments
// One thread per expert (routed 0..Nr-1, then the shared expert at Nr):
// rows [first, first + count) of the forward's row order, its token segment
// padded to a multiple of 128 at seg[e] (exclusive scan), and one tile entry
// per 128 tokens: {expert, first row, rows (<= 128), segment column}.
// meta[0] = number of tiles, seg[E] = total padded columns.
__global__ void __launch_bounds__(512) wgrad_tiles_kernel(const int32_t *__restrict__ offsets, int Nr, int Ns,
                                                           int64_t R, int64_t T, int32_t *__restrict__ seg,
                                                           int4 *__restrict__ tiles, int32_t *__restrict__ meta) {
  __shared__ int s_pad[512], s_nt[512];
  const int e = threadIdx.x;
  const int E = Nr + Ns;
  int first = 0, cnt = 0;
  if (e < Nr) {
    first = offsets[e];
    cnt = offsets[e + 1] - offsets[e];
  } else if (e < E) {
    first = static_cast<int>(R);
    cnt = static_cast<int>(T);
  }
  const int nt = (cnt + 127) / 128;
  s_pad[e] = e < E ? nt * 128 : 0;
  s_nt[e] = e < E ? nt : 0;
  __syncthreads();
  if (e == 0) {  // exclusive scans (E <= 257)
    int run = 0, runt = 0;
    for (int i = 0; i < E; ++i) {
      const int a = s_pad[i], b = s_nt[i];
      s_pad[i] = run;
      s_nt[i] = runt;
      run += a;
      runt += b;
    }
    seg[E] = run;
    meta[0] = runt;
  }
  __syncthreads();
  if (e < E) {
    seg[e] = s_pad[e];
    for (int i = 0; i < nt; ++i) {
      const int n = cnt - 128 * i < 128 ? cnt - 128 * i : 128;
      tiles[s_nt[e] + i] = make_int4(e, first + 128 * i, n, s_pad[e] + 128 * i);
    }
  }
}

// ------------------------------------------------ 128x1 tiles, transposed
// Grid: (tile, 64-channel block).  The tile's rows (tokens) of 64 channels
// are read in FP32 (from an FP32 row matrix, or a bf16 [T, C] matrix gathered
// by the row's token: dout, the layer input), each channel's amax over
// the tile's rows gives its scale, and the codes are written channel-major:
// out[c][col0 + r] (K-major along tokens for the wgrad GEMM); scales to
// s_t[(col0 / 128)][c].  Padding rows (beyond the tile's rows) are zero.
enum ColSrc : int { COL_F32 = 0, COL_TOKEN = 1 };
constexpr int kColCh = 64;

template <int SRC>
__global__ void __launch_bounds__(256) colquant_kernel(const int4 *__restrict__ tiles, const int32_t *__restrict__ meta,
                                                        int max_tiles, const float *__restrict__ f32rows,
                                                        int64_t f32_ld, const uint16_t *__restrict__ bf16rows,
                                                        const int32_t *__restrict__ row_src, int64_t R, int C,
                                                        uint8_t *__restrict__ out, int64_t out_ld,
                                                        float *__restrict__ s_t) {
  __shared__ float vals[128][kColCh + 1];
  __shared__ float part[4][kColCh];
  __shared__ __align__(16) uint8_t codes[kColCh][128 + 16];
  int ntiles = meta[0];
  if (ntiles > max_tiles) ntiles = max_tiles;
  const int tix = blockIdx.x;
  if (tix >= ntiles) return;
  const int4 tl = tiles[tix];
  const int first = tl.y, nrows = tl.z, col0 = tl.w;
  const int64_t c0 = static_cast<int64_t>(blockIdx.y) * kColCh;
  const int tid = threadIdx.x;
  for (int i = tid; i < 128 * (kColCh / 4); i += blockDim.x) {
    const int r = i / (kColCh / 4), c4 = (i % (kColCh / 4)) * 4;  // row, first of 4 channels
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < nrows) {
      const int64_t p = first + r;
      if (SRC == COL_F32) {
        const float4 a = *reinterpret_cast<const float4 *>(f32rows + p * f32_ld + c0 + c4);
        v[0] = a.x;
        v[1] = a.y;
        v[2] = a.z;
        v[3] = a.w;
      } else {
        const int64_t t = p < R ? row_src[p] : p - R;
        const uint2 b = *reinterpret_cast<const uint2 *>(bf16rows + t * C + c0 + c4);
        v[0] = __uint_as_float(b.x << 16);
        v[1] = __uint_as_float(b.x & 0xFFFF0000u);
        v[2] = __uint_as_float(b.y << 16);
        v[3] = __uint_as_float(b.y & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) vals[r][c4 + k] = v[k];
  }
  __syncthreads();
  // per channel amax over the 128 rows: 4 threads per channel, 32 rows each
  const int c = tid & (kColCh - 1), quarter = tid / kColCh;
  {
    float a = 0.0f;
    for (int r = quarter * 32; r < quarter * 32 + 32; ++r) a = fmaxf(a, fabsf(vals[r][c]));
    part[quarter][c] = a;
  }
  __syncthreads();
  {
    const float S = fmaxf(fmaxf(part[0][c], part[1][c]), fmaxf(part[2][c], part[3][c])) / 448.0f;
    const float y = S != 0.0f ? __frcp_rn(S) : 0.0f;
    // 32 codes of this channel as two 16-byte words, converted in pairs
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r0 = quarter * 32 + 16 * h;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (S != 0.0f) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = r0 + 4 * k;
          const uint32_t lo = e4m3x2_rn_sat(quot(vals[r][c], S, y), quot(vals[r + 1][c], S, y));
          const uint32_t hi = e4m3x2_rn_sat(quot(vals[r + 2][c], S, y), quot(vals[r + 3][c], S, y));
          w[k] = lo | (hi << 16);
        }
      }
      *reinterpret_cast<uint4 *>(&codes[c][r0]) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (quarter == 0) s_t[static_cast<int64_t>(col0 / 128) * C + c0 + c] = S;
  }
  __syncthreads();
  // store: channel c's 128 tokens are 128 contiguous bytes of out row c0 + c
  for (int i = tid; i < kColCh * 8; i += blockDim.x) {
    const int cc = i >> 3, v = i & 7;
    const uint4 w = *reinterpret_cast<const uint4 *>(&codes[cc][v * 16]);
    *reinterpret_cast<uint4 *>(out + (c0 + cc) * out_ld + col0 + v * 16) = w;
  }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_transpose_blocks(const uint8_t *q, const float *s, int64_t n, int64_t k, int64_t batch,
                                    uint8_t *qt, float *st, cudaStream_t stream) {
  const int64_t blocks = (n / 128) * (k / 128);
  if (blocks == 0 || batch == 0) return cudaSuccess;
  transpose_blocks_kernel<<<dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(batch)), 256, 0, stream>>>(
      q, s, n, k, qt, st);
  return cudaGetLastError();
}

cudaError_t launch_dout_quant(const void *dout, const int32_t *row_src, int64_t R, int64_t RS, int H, uint8_t *q,
                              float *s_t, int64_t ld, cudaStream_t st) {
  const int64_t groups = RS * (H / 128);
  if (groups == 0) return cudaSuccess;
  const int64_t blocks = (groups * 16 + 255) / 256;
  dout_quant_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<const uint16_t *>(dout), row_src, R,
                                                                    RS, H, q, s_t, ld);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_bwd(const float *GU, const float *dh, const float *row_gate, int64_t RS, int I, float *h,
                              float *dGU, uint8_t *q, float *s_t, int64_t ld, cudaStream_t st) {
  const int64_t warps = RS * (I / 128);
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + 7) / 8;
  swiglu_bwd_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(GU, dh, row_gate, RS, I, h, dGU, q, s_t, ld);
  return cudaGetLastError();
}

cudaError_t launch_wgrad_tiles(const int32_t *offsets, int Nr, int Ns, int64_t R, int64_t T, int32_t *seg,
                               int4 *tiles, int32_t *meta, cudaStream_t st) {
  wgrad_tiles_kernel<<<1, 512, 0, st>>>(offsets, Nr, Ns, R, T, seg, tiles, meta);
  return cudaGetLastError();
}

cudaError_t launch_colquant(int src, const int4 *tiles, const int32_t *meta, int max_tiles, const float *f32rows,
                            int64_t f32_ld, const void *bf16rows, const int32_t *row_src, int64_t R, int C,
                            uint8_t *out, int64_t out_ld, float *s_t, cudaStream_t st) {
  if (max_tiles <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(max_tiles), static_cast<unsigned>(C / kColCh));
  const auto *b = static_cast<const uint16_t *>(bf16rows);
  if (src == COL_F32)
    colquant_kernel<COL_F32><<<grid, 256, 0, st>>>(tiles, meta, max_tiles, f32rows, f32_ld, b, row_src, R, C, out,
                                                    out_ld, s_t);
  else
    colquant_kernel<COL_TOKEN><<<grid, 256, 0, st>>>(tiles, meta, max_tiles, f32rows, f32_ld, b, row_src, R, C, out,
                                                      out_ld, s_t);
  return cudaGetLastError();
}

}  // namespace moe
