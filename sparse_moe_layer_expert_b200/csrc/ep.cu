// ep.cu -- dispatch and combine of the expert-parallel layer.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), "Problem und
// Motivation" item 2 and "Kernideen" (DualPipe bullet): the routed experts of
// a layer live on different GPUs; tokens travel to the GPUs of their experts
// and the expert outputs travel back, by all-to-all exchanges.  With W ranks,
// rank d owns the routed experts [d*N_r/W, (d+1)*N_r/W).  A token is sent to
// a rank once, whatever the number of its experts there; the packed row
// carries, for each of the token's K_r slots, the local index of the expert
// on that rank (or -1) and the gate:
//
//   [0, H)                     E4M3 codes of the token (1x128 quantized)
//   [H, H + 4 H/128)           its FP32 scales
//   [.., + 4 K_r)              int32 local expert per slot, -1 = elsewhere
//   [.., + 4 K_r)              FP32 gate per slot (0 where -1)
//   padded to a multiple of 16 bytes
//
// Kernels (all on the sending or receiving rank's own memory; the exchange
// itself is the caller's collective):
//   ep_count_kernel    per block of 256 tokens, rows per destination
//   ep_scan_kernel     one CTA: send counts, offsets, per-block bases
//   ep_rows_kernel     per block: each token's row in the send buffer per
//                      destination (token order within a destination)
//   ep_pack_kernel     one warp per token: packed rows into the send buffer
//                      (and, optionally, every token's row for the shared
//                      expert: slot 0 = expert 0, gate 1)
//   ep_unpack_kernel   receiving side: slots, gates and scales of the rows
//   ep_combine_kernel  sending side: out_t = u_t + shared + sum over the
//                      destinations (ascending) of the returned partial sums
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int kEpBlock = 256;

__device__ __forceinline__ uint64_t dest_mask(const int32_t *__restrict__ idx, int64_t t, int Kr, int per, int W,
                                              bool &bad) {
  uint64_t m = 0;
  for (int k = 0; k < Kr; ++k) {
    const int e = idx[t * Kr + k];
    const int d = e / per;
    if (e < 0 || d >= W)
      bad = true;
    else
      m |= uint64_t(1) << d;
  }
  return m;
}
}  // namespace

__global__ void __launch_bounds__(kEpBlock) ep_count_kernel(const int32_t *__restrict__ idx, int64_t T, int Kr,
                                                             int per, int W, int32_t *__restrict__ blk_cnt,
                                                             int32_t *__restrict__ err) {
  __shared__ int cnt[64];
  for (int d = threadIdx.x; d < W; d += blockDim.x) cnt[d] = 0;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kEpBlock + threadIdx.x;
  bool bad = false;
  if (t < T) {
    uint64_t m = dest_mask(idx, t, Kr, per, W, bad);
    while (m) {
      const int d = __ffsll(static_cast<long long>(m)) - 1;
      m &= m - 1;
      atomicAdd(&cnt[d], 1);
    }
  }
  if (bad && err) atomicOr(err, MOE_DEVERR_BAD_INDEX);
  __syncthreads();
  for (int d = threadIdx.x; d < W; d += blockDim.x) blk_cnt[static_cast<int64_t>(blockIdx.x) * W + d] = cnt[d];
}

// Thread d: the blocks' counts for destination d in block order -> per-block
// bases; totals -> send counts; exclusive scan over destinations -> offsets.
__global__ void ep_scan_kernel(const int32_t *__restrict__ blk_cnt, int nblk, int W, int32_t *__restrict__ blk_base,
                               int32_t *__restrict__ send_counts, int32_t *__restrict__ send_off) {
  __shared__ int tot[64];
  const int d = threadIdx.x;
  if (d < W) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      blk_base[static_cast<int64_t>(b) * W + d] = run;
      run += blk_cnt[static_cast<int64_t>(b) * W + d];
    }
    tot[d] = run;
    send_counts[d] = run;
  }
  __syncthreads();
  if (d == 0) {
    int run = 0;
    for (int j = 0; j < W; ++j) {
      send_off[j] = run;
      run += tot[j];
    }
    send_off[W] = run;
  }
}

// One token per thread; for each destination the token's rank among the
// block's tokens sending there (warp ballots, then the warps' totals).
__global__ void __launch_bounds__(kEpBlock) ep_rows_kernel(const int32_t *__restrict__ idx, int64_t T, int Kr,
                                                            int per, int W, const int32_t *__restrict__ blk_base,
                                                            const int32_t *__restrict__ send_off,
                                                            int32_t *__restrict__ row_of) {
  __shared__ int wsum[kEpBlock / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kEpBlock + threadIdx.x;
  bool bad = false;
  const uint64_t m = t < T ? dest_mask(idx, t, Kr, per, W, bad) : 0;
  for (int d = 0; d < W; ++d) {
    const bool hit = (m >> d) & 1;
    const uint32_t bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    before += __popc(bal & ((1u << lane) - 1u));
    if (t < T)
      row_of[t * W + d] = hit ? send_off[d] + blk_base[static_cast<int64_t>(blockIdx.x) * W + d] + before : -1;
    __syncthreads();  // wsum is reused by the next destination
  }
}

// One warp per token: its packed row for every destination it goes to, and
// (self_rows) its row for the shared expert.
__global__ void __launch_bounds__(256) ep_pack_kernel(const uint8_t *__restrict__ xq, const float *__restrict__ xs,
                                                       const int32_t *__restrict__ idx, const float *__restrict__ gate,
                                                       int64_t T, int H, int Kr, int per, int W,
                                                       const int32_t *__restrict__ row_of, uint8_t *__restrict__ send,
                                                       int64_t row_bytes, uint8_t *__restrict__ self_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int hv = H / 16, nkb = H / 128;
  const uint4 *src = reinterpret_cast<const uint4 *>(xq + t * H);
  const int64_t off_s = H, off_i = H + 4 * nkb, off_g = off_i + 4 * Kr;
  for (int d = 0; d < W + (self_rows ? 1 : 0); ++d) {
    uint8_t *row;
    if (d < W) {
      const int r = row_of[t * W + d];
      if (r < 0) continue;
      row = send + static_cast<int64_t>(r) * row_bytes;
    } else {
      row = self_rows + t * row_bytes;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(row);
    for (int i = lane; i < hv; i += 32) dst[i] = __ldg(src + i);
    float *ds = reinterpret_cast<float *>(row + off_s);
    for (int i = lane; i < nkb; i += 32) ds[i] = __ldg(xs + t * nkb + i);
    int32_t *di = reinterpret_cast<int32_t *>(row + off_i);
    float *dg = reinterpret_cast<float *>(row + off_g);
    for (int k = lane; k < Kr; k += 32) {
      if (d < W) {
        const int e = idx[t * Kr + k];
        const bool here = e >= 0 && e / per == d;
        di[k] = here ? e - d * per : -1;
        dg[k] = here ? gate[t * Kr + k] : 0.0f;
      } else {  // the shared expert: one slot, gate 1
        di[k] = k == 0 ? 0 : -1;
        dg[k] = k == 0 ? 1.0f : 0.0f;
      }
    }
  }
}

// One warp per received row: slots, gates and scales into dense arrays.
__global__ void __launch_bounds__(256) ep_unpack_kernel(const uint8_t *__restrict__ rows, int64_t n, int64_t row_bytes,
                                                         int H, int Kr, int n_local, int32_t *__restrict__ idx,
                                                         float *__restrict__ gate, float *__restrict__ xs,
                                                         int32_t *__restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (i >= n) return;
  const int nkb = H / 128;
  const uint8_t *row = rows + i * row_bytes;
  const float *ss = reinterpret_cast<const float *>(row + H);
  const int32_t *si = reinterpret_cast<const int32_t *>(row + H + 4 * nkb);
  const float *sg = reinterpret_cast<const float *>(row + H + 4 * nkb + 4 * Kr);
  for (int j = lane; j < nkb; j += 32) xs[i * nkb + j] = ss[j];
  bool bad = false;
  for (int k = lane; k < Kr; k += 32) {
    int e = si[k];
    if (e < -1 || e >= n_local) {
      bad = true;
      e = -1;
    }
    idx[i * Kr + k] = e;
    gate[i * Kr + k] = e >= 0 ? sg[k] : 0.0f;
  }
  if (bad && err) atomicOr(err, MOE_DEVERR_BAD_INDEX);
}

// One CTA per token, 8 channels (16-byte words) per thread and step:
// out_t = u_t + y_shared[t] + sum_{d ascending} back[row_of[t, d]], in FP32.
template <bool OUT_F32>
__global__ void __launch_bounds__(128) ep_combine_kernel(const __nv_bfloat16 *__restrict__ x,
                                                          const __nv_bfloat16 *__restrict__ y_sh,
                                                          const __nv_bfloat16 *__restrict__ back,
                                                          const int32_t *__restrict__ row_of, int W, int H,
                                                          void *__restrict__ out) {
  const int64_t t = blockIdx.x;
  const int hv = H / 8;
  for (int v = threadIdx.x; v < hv; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    auto add = [&](const __nv_bfloat16 *rowp) {
      const uint4 w4 = __ldg(reinterpret_cast<const uint4 *>(rowp) + v);
      const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
      }
    };
    add(x + t * H);
    if (y_sh) add(y_sh + t * H);
    for (int d = 0; d < W; ++d) {
      const int r = row_of[t * W + d];
      if (r >= 0) add(back + static_cast<int64_t>(r) * H);
    }
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

cudaError_t launch_ep_dispatch(const uint8_t *xq, const float *xs, const int32_t *idx, const float *gate, int64_t T,
                               int H, int Kr, int Nr, int W, int32_t *blk_cnt, int32_t *blk_base,
                               int32_t *send_counts, int32_t *send_off, int32_t *row_of, uint8_t *send,
                               int64_t row_bytes, uint8_t *self_rows, int32_t *err, cudaStream_t st) {
  const int per = Nr / W;
  const int nblk = static_cast<int>((T + kEpBlock - 1) / kEpBlock);
  if (nblk > 0) {
    ep_count_kernel<<<nblk, kEpBlock, 0, st>>>(idx, T, Kr, per, W, blk_cnt, err);
    if (const cudaError_t e = cudaGetLastError()) return e;
  }
  ep_scan_kernel<<<1, 64, 0, st>>>(blk_cnt, nblk, W, blk_base, send_counts, send_off);
  if (const cudaError_t e = cudaGetLastError()) return e;
  if (nblk == 0) return cudaSuccess;
  ep_rows_kernel<<<nblk, kEpBlock, 0, st>>>(idx, T, Kr, per, W, blk_base, send_off, row_of);
  if (const cudaError_t e = cudaGetLastError()) return e;
  const int64_t blocks = (T + 7) / 8;
  ep_pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(xq, xs, idx, gate, T, H, Kr, per, W, row_of, send,
                                                                 row_bytes, self_rows);
  return cudaGetLastError();
}

cudaError_t launch_ep_unpack(const uint8_t *rows, int64_t n, int64_t row_bytes, int H, int Kr, int n_local,
                             int32_t *idx, float *gate, float *xs, int32_t *err, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 7) / 8;
  ep_unpack_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(rows, n, row_bytes, H, Kr, n_local, idx, gate, xs,
                                                                   err);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const void *x, const void *y_sh, const void *back, const int32_t *row_of, int64_t T,
                              int W, int H, void *out, int out_f32, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  const auto *yb = static_cast<const __nv_bfloat16 *>(y_sh);
  const auto *bb = static_cast<const __nv_bfloat16 *>(back);
  if (out_f32)
    ep_combine_kernel<true><<<static_cast<unsigned>(T), 128, 0, st>>>(xb, yb, bb, row_of, W, H, out);
  else
    ep_combine_kernel<false><<<static_cast<unsigned>(T), 128, 0, st>>>(xb, yb, bb, row_of, W, H, out);
  return cudaGetLastError();
}

}  // namespace moe
