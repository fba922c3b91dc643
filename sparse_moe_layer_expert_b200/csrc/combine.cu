// combine.cu -- layer output, bias update and the bounded-wait self test.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Methode section 2:
//   h'_t = u_t + sum_{i<=N_s} FFN^(s)_i(u_t) + sum_{i<=N_r} g_{i,t} FFN^(r)_i(u_t).
// The routed outputs arrive already multiplied by their gate (down-projection
// epilogue, stored as bf16), so the combine is a plain FP32 sum per token in a
// fixed order: residual, shared expert, then the K_r slots in selection order.
//
// Bias update (same section): an overloaded expert gets b_i -= gamma, an
// underloaded one b_i += gamma, once per step.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// bf16 x 8 (one 16-byte word) added to eight FP32 accumulators
__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 &v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// eight FP32 values (two 16-byte words) added to eight FP32 accumulators
__device__ __forceinline__ void add_f32x8(float (&acc)[8], const float4 *p) {
  const float4 a = __ldg(p), b = __ldg(p + 1);
  acc[0] += a.x;
  acc[1] += a.y;
  acc[2] += a.z;
  acc[3] += a.w;
  acc[4] += b.x;
  acc[5] += b.y;
  acc[6] += b.z;
  acc[7] += b.w;
}

// One CTA per token, 8 channels (16-byte loads of x and of every y row) per
// thread and step.  y rows are bf16 (the gate-scaled output of each routed
// expert, the shared expert's at row R + t), or FP32 when Y_F32.
template <bool OUT_F32, bool Y_F32>
__global__ void __launch_bounds__(128) combine_kernel(const __nv_bfloat16 *__restrict__ x, const void *__restrict__ yv,
                                                       const int32_t *__restrict__ pos, int H, int Kr, int64_t R,
                                                       int Ns, void *__restrict__ out) {
  const __nv_bfloat16 *y = static_cast<const __nv_bfloat16 *>(yv);
  const float *yf = static_cast<const float *>(yv);
  const int64_t t = blockIdx.x;
  int p[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) p[k] = (k < Kr) ? pos[t * Kr + k] : -1;
  const int hv = H / 8;
  const uint4 *xr = x ? reinterpret_cast<const uint4 *>(x + t * H) : nullptr;
  for (int v = threadIdx.x; v < hv; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (xr) add_bf16x8(acc, __ldg(xr + v));  // residual u_t
    auto add_row = [&](int64_t row) {
      if (Y_F32)
        add_f32x8(acc, reinterpret_cast<const float4 *>(yf + row * H) + 2 * v);
      else
        add_bf16x8(acc, __ldg(reinterpret_cast<const uint4 *>(y + row * H) + v));
    };
    if (Ns) add_row(R + t);
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (k < Kr && p[k] >= 0) add_row(p[k]);
    if (OUT_F32) {
      float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + t * H) + 2 * v;
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&b2);
      }
      reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + t * H)[v] = make_uint4(w[0], w[1], w[2], w[3]);
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

cudaError_t launch_combine(const void *x, const void *y, const int32_t *pos, int64_t T, int H, int Kr, int64_t R,
                           int Ns, void *out, int out_f32, cudaStream_t st, bool y_f32) {
  if (T == 0) return cudaSuccess;
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  const dim3 grid(static_cast<unsigned>(T));
  if (y_f32) {
    if (out_f32)
      combine_kernel<true, true><<<grid, 128, 0, st>>>(xb, y, pos, H, Kr, R, Ns, out);
    else
      combine_kernel<false, true><<<grid, 128, 0, st>>>(xb, y, pos, H, Kr, R, Ns, out);
  } else {
    if (out_f32)
      combine_kernel<true, false><<<grid, 128, 0, st>>>(xb, y, pos, H, Kr, R, Ns, out);
    else
      combine_kernel<false, false><<<grid, 128, 0, st>>>(xb, y, pos, H, Kr, R, Ns, out);
  }
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
