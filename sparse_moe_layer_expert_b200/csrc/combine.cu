// combine.cu -- layer output, bias update and the bounded-wait self test.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Methode section 2:
//   h'_t = u_t + sum_{i<=N_s} FFN^(s)_i(u_t) + sum_{i<=N_r} g_{i,t} FFN^(r)_i(u_t).
// The routed outputs arrive already multiplied by their gate (down-projection
// epilogue), so the combine is a plain FP32 sum per token in a fixed order:
// residual, shared expert, then the K_r slots in selection order.
//
// Bias update (same section): an overloaded expert gets b_i -= gamma, an
// underloaded one b_i += gamma, once per step.
#include "common.cuh"
#include "kernels.h"

namespace moe {

template <bool OUT_F32>
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ y,
                                                       const int32_t *__restrict__ pos, int H, int Kr, int64_t R,
                                                       int Ns, void *__restrict__ out) {
  const int64_t t = blockIdx.x;
  int p[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) p[k] = (k < Kr) ? pos[t * Kr + k] : 0;
  const int hv = H / 4;
  const uint2 *xr = reinterpret_cast<const uint2 *>(x + t * H);
  const float4 *ysh = reinterpret_cast<const float4 *>(y + (R + t) * H);
  for (int v = threadIdx.x; v < hv; v += blockDim.x) {
    const uint2 xv = __ldg(xr + v);
    float4 acc;
    acc.x = __uint_as_float(xv.x << 16);
    acc.y = __uint_as_float(xv.x & 0xFFFF0000u);
    acc.z = __uint_as_float(xv.y << 16);
    acc.w = __uint_as_float(xv.y & 0xFFFF0000u);
    if (Ns) {
      const float4 s = __ldg(ysh + v);
      acc.x += s.x;
      acc.y += s.y;
      acc.z += s.z;
      acc.w += s.w;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < Kr && p[k] >= 0) {
        const float4 s = __ldg(reinterpret_cast<const float4 *>(y + static_cast<int64_t>(p[k]) * H) + v);
        acc.x += s.x;
        acc.y += s.y;
        acc.z += s.z;
        acc.w += s.w;
      }
    }
    if (OUT_F32) {
      reinterpret_cast<float4 *>(static_cast<float *>(out) + t * H)[v] = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 o;
      o.x = *reinterpret_cast<uint32_t *>(&lo);
      o.y = *reinterpret_cast<uint32_t *>(&hi);
      reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + t * H)[v] = o;
    }
  }
}

__global__ void bias_update_kernel(float *bias, const int32_t *counts, int Nr, int64_t total, float gamma) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= Nr) return;
  // compare load_i with the mean total/Nr exactly, in integers
  const int64_t d = static_cast<int64_t>(counts[i]) * Nr - total;
  if (d > 0)
    bias[i] = bias[i] - gamma;
  else if (d < 0)
    bias[i] = bias[i] + gamma;
}

// One thread waits on an mbarrier that nothing arrives on; the bounded wait
// must give up, set MOE_DEVERR_TIMEOUT and let the kernel return.
__global__ void wait_selftest_kernel(int32_t *err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, err, limit_ns};
    mbar_wait(&bar, 0, ctl);
  }
}

cudaError_t launch_combine(const void *x, const float *y, const int32_t *pos, int64_t T, int H, int Kr, int64_t R,
                           int Ns, void *out, int out_f32, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (out_f32)
    combine_kernel<true><<<static_cast<unsigned>(T), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), y, pos,
                                                                    H, Kr, R, Ns, out);
  else
    combine_kernel<false><<<static_cast<unsigned>(T), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), y, pos,
                                                                     H, Kr, R, Ns, out);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(float *bias, const int32_t *counts, int Nr, int64_t total, float gamma,
                               cudaStream_t st) {
  bias_update_kernel<<<(Nr + 255) / 256, 256, 0, st>>>(bias, counts, Nr, total, gamma);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int32_t *err, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
