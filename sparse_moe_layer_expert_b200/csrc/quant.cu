// quant.cu -- fine-grained FP8 (E4M3) quantizers.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Kernideen, FP8 bullet:
// E4M3 for all tensors, 1x128 tiles for activations, 128x128 blocks for
// weights.  "DeepSeek-V3 技術報告書" (singularity-lens.com), formula
// paragraph: S = max|X| / 448 and X_FP8 = clip(round(X / S), -448, 448).
// The quotient X / S is the IEEE FP32 correctly rounded one (this file is
// compiled without fast-math) and the cast rounds to nearest even, saturating
// at +-448.
// POW2 = true: the power-of-two scale variant (pow2_scale in common.cuh),
// for which X / S is an exact scaling.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Codes of 8 values sharing the scale S.  The quotients x / S are the IEEE
// correctly rounded ones: for S well inside the normal range through the
// reciprocal plus one residual correction (div_by_recip, common.cuh), which
// gives the same correctly rounded result as the division; for tiny S by the
// division itself.
__device__ __forceinline__ uint2 codes8(const float (&f)[8], float S) {
  uint32_t lo = 0, hi = 0;
  if (S >= 0x1p-100f) {
    const float y = __frcp_rn(S);
    lo = e4m3x2_rn_sat(div_by_recip(f[0], S, y), div_by_recip(f[1], S, y)) |
         (e4m3x2_rn_sat(div_by_recip(f[2], S, y), div_by_recip(f[3], S, y)) << 16);
    hi = e4m3x2_rn_sat(div_by_recip(f[4], S, y), div_by_recip(f[5], S, y)) |
         (e4m3x2_rn_sat(div_by_recip(f[6], S, y), div_by_recip(f[7], S, y)) << 16);
  } else if (S != 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) lo |= static_cast<uint32_t>(e4m3_rn_sat(f[i] / S)) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) hi |= static_cast<uint32_t>(e4m3_rn_sat(f[4 + i] / S)) << (8 * i);
  }
  return make_uint2(lo, hi);
}

// 1x128 tiles: 16 lanes per tile, 8 bf16 (one 16-byte load) per lane; each
// 16-lane set takes 2 consecutive tiles, all loads issued first.
template <bool POW2>
__global__ void __launch_bounds__(256) quant_1x128_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                           int64_t cols, int64_t ldx, uint8_t *__restrict__ q,
                                                           float *__restrict__ s) {
  constexpr int G = 2;
  const int64_t gpr = cols / 128;
  const int64_t total = rows * gpr;
  const int64_t gid0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4) * G;
  const int sub = threadIdx.x & 15;
  int64_t r = gid0 / gpr;
  int64_t g = gid0 - r * gpr;
  int64_t rr[G], gg[G];
  uint4 v[G];
#pragma unroll
  for (int k = 0; k < G; ++k) {
    rr[k] = r;
    gg[k] = g;
    v[k] = make_uint4(0, 0, 0, 0);
    if (gid0 + k < total) v[k] = __ldg(reinterpret_cast<const uint4 *>(x + r * ldx + g * 128 + sub * 8));
    if (++g == gpr) {
      g = 0;
      ++r;
    }
  }
#pragma unroll
  for (int k = 0; k < G; ++k) {
    float f[8];
    bf16x8_to_f32(v[k], f);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float S = POW2 ? pow2_scale(amax) : amax / 448.0f;
    if (gid0 + k < total) {
      *reinterpret_cast<uint2 *>(q + rr[k] * cols + gg[k] * 128 + sub * 8) = codes8(f, S);
      if (sub == 0) s[rr[k] * gpr + gg[k]] = S;
    }
  }
}

// 128x128 blocks: one CTA of 256 threads per block, 8 x 16-byte chunks each.
template <bool POW2>
__global__ void __launch_bounds__(256) quant_128x128_kernel(const __nv_bfloat16 *__restrict__ w, int64_t n,
                                                             int64_t k, uint8_t *__restrict__ q,
                                                             float *__restrict__ s) {
  __shared__ float red[8];
  const int64_t kb = k / 128;
  const int64_t bi = blockIdx.x / kb, bj = blockIdx.x - (blockIdx.x / kb) * kb;
  const int tid = threadIdx.x;
  float f[8][8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * 256 + tid;  // chunk of 8 elements: 16 chunks per row
    const int row = c >> 4, cc = c & 15;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(w + (bi * 128 + row) * k + bj * 128 + cc * 8));
    bf16x8_to_f32(v, f[i]);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[i][j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float S = POW2 ? pow2_scale(amax) : amax / 448.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * 256 + tid;
    const int row = c >> 4, cc = c & 15;
    *reinterpret_cast<uint2 *>(q + (bi * 128 + row) * k + bj * 128 + cc * 8) = codes8(f[i], S);
  }
  if (tid == 0) s[bi * kb + bj] = S;
}

cudaError_t launch_quant_1x128(const void *x, int64_t rows, int64_t cols, int64_t ldx, uint8_t *q, float *s,
                               cudaStream_t st, bool pow2) {
  const int64_t groups = rows * (cols / 128);
  if (groups == 0) return cudaSuccess;
  const int64_t threads = (groups + 1) / 2 * 16;  // 16 lanes per pair of tiles
  const int64_t blocks = (threads + 255) / 256;
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  if (pow2)
    quant_1x128_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(xb, rows, cols, ldx, q, s);
  else
    quant_1x128_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(xb, rows, cols, ldx, q, s);
  return cudaGetLastError();
}

cudaError_t launch_quant_128x128(const void *w, int64_t n, int64_t k, uint8_t *q, float *s, cudaStream_t st,
                                 bool pow2) {
  const int64_t blocks = (n / 128) * (k / 128);
  if (blocks == 0) return cudaSuccess;
  const auto *wb = static_cast<const __nv_bfloat16 *>(w);
  if (pow2)
    quant_128x128_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(wb, n, k, q, s);
  else
    quant_128x128_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(wb, n, k, q, s);
  return cudaGetLastError();
}

}  // namespace moe
