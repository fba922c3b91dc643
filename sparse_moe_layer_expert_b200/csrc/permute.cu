// permute.cu -- expert-contiguous grouping of the routed (token, slot) pairs.
//
// The routed experts of the DeepSeekMoE layer ("DeepSeek-V3 Technischer
// Bericht", Methode section 2) each see only the tokens that selected them.
// To run every expert as one GEMM over contiguous rows, the FP8 rows of the
// quantized input are copied into expert order with a stable counting sort:
// rows of expert e occupy [offsets[e], offsets[e+1]), in token order, then
// slot order.  All of it runs on the device; the host never learns the
// per-expert counts.
//
//  hist_kernel        per 128-token block, per-expert counts
//  build_tiles_kernel one CTA: totals, exclusive scans, per-block bases, and
//                     the work lists of both grouped GEMMs
//  scatter_kernel     per 128-token block: stable ranks (warp match), then
//                     row copies (16-byte vectors) and per-row gate values
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kTokBlock = 128;

__global__ void __launch_bounds__(256) hist_kernel(const int32_t *__restrict__ idx, int64_t T, int Kr, int Nr,
                                                    int32_t *__restrict__ blk_hist, int32_t *__restrict__ err) {
  __shared__ int h[256];
  for (int e = threadIdx.x; e < Nr; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTokBlock;
  const int64_t nt = (T - t0) < kTokBlock ? (T - t0) : kTokBlock;
  const int na = static_cast<int>(nt) * Kr;
  bool bad = false;
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    const int e = idx[t0 * Kr + a];
    if (e >= 0 && e < Nr)
      atomicAdd(&h[e], 1);
    else
      bad = true;
  }
  if (bad && err) atomicOr(err, MOE_DEVERR_BAD_INDEX);
  __syncthreads();
  for (int e = threadIdx.x; e < Nr; e += blockDim.x) blk_hist[static_cast<int64_t>(blockIdx.x) * Nr + e] = h[e];
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 256).
__device__ int block_excl_scan(int v, int *total) {
  __shared__ int warp_sums[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  int base = 0, all = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) base += warp_sums[w];
    all += warp_sums[w];
  }
  __syncthreads();
  *total = all;
  return base + x - v;
}

__global__ void __launch_bounds__(256) build_tiles_kernel(const int32_t *__restrict__ blk_hist, int64_t T, int Kr,
                                                           int Nr, int Ns, int H, int I, int32_t *counts,
                                                           int32_t *offsets, int32_t *blk_base, GemmTile *tiles1,
                                                           GemmTile *tiles2, int32_t *ntiles, int32_t *counts_out) {
  const int e = threadIdx.x;
  const int nblk = static_cast<int>((T + kTokBlock - 1) / kTokBlock);
  const int64_t R = T * Kr;
  int cnt = 0;
  if (e < Nr)
    for (int b = 0; b < nblk; ++b) cnt += blk_hist[static_cast<int64_t>(b) * Nr + e];
  int total_rows;
  const int off = block_excl_scan(cnt, &total_rows);
  const int nch = (cnt + 127) / 128;
  int total_chunks;
  const int cbase = block_excl_scan(nch, &total_chunks);
  if (e < Nr) {
    counts[e] = cnt;
    if (counts_out) counts_out[e] = cnt;
    offsets[e] = off;
    if (e == Nr - 1) offsets[Nr] = off + cnt;
    int run = off;
    for (int b = 0; b < nblk; ++b) {
      blk_base[static_cast<int64_t>(b) * Nr + e] = run;
      run += blk_hist[static_cast<int64_t>(b) * Nr + e];
    }
  }
  const int nb1 = gemm1_blocks(I), nb2 = gemm2_blocks(H);
  const int hb = H / 128, ib = I / 128;
  const int sh_chunks = Ns ? static_cast<int>((T + 127) / 128) : 0;
  // shared-expert tiles first (full 128-row chunks, largest work first)
  for (int i = threadIdx.x; i < sh_chunks * nb1; i += blockDim.x) {
    const int c = i / nb1, rb = i % nb1;
    const int es = Nr;  // shared expert index
    const int n = static_cast<int>((T - c * 128) < 128 ? (T - c * 128) : 128);
    GemmTile t;
    t.w_row0 = es * 2 * I + rb * 128;
    t.w_row1 = es * 2 * I + I + rb * 128;
    t.sw0 = es * (2 * ib) + rb;
    t.sw1 = es * (2 * ib) + ib + rb;
    t.a_row = c * 128;
    t.n = n;
    t.out_row = static_cast<int32_t>(R) + c * 128;
    t.out_col = (rb * 128) | kTileFromMap1;
    tiles1[rb * sh_chunks + c] = t;
  }
  for (int i = threadIdx.x; i < sh_chunks * nb2; i += blockDim.x) {
    const int c = i / nb2, p = i % nb2;
    const int es = Nr;
    const int n = static_cast<int>((T - c * 128) < 128 ? (T - c * 128) : 128);
    GemmTile t;
    t.w_row0 = es * H + (2 * p) * 128;
    t.w_row1 = (2 * p + 1 < hb) ? es * H + (2 * p + 1) * 128 : -1;
    t.sw0 = es * hb + 2 * p;
    t.sw1 = es * hb + 2 * p + 1;
    t.a_row = static_cast<int32_t>(R) + c * 128;
    t.n = n;
    t.out_row = t.a_row;
    t.out_col = 2 * p * 128;
    tiles2[p * sh_chunks + c] = t;
  }
  if (e < Nr && nch > 0) {
    const int sz = (cnt + nch - 1) / nch;  // <= 128
    const int64_t base1 = static_cast<int64_t>(sh_chunks) * nb1 + static_cast<int64_t>(cbase) * nb1;
    const int64_t base2 = static_cast<int64_t>(sh_chunks) * nb2 + static_cast<int64_t>(cbase) * nb2;
    for (int rb = 0; rb < nb1; ++rb) {
      for (int c = 0; c < nch; ++c) {
        GemmTile t;
        t.w_row0 = e * 2 * I + rb * 128;
        t.w_row1 = e * 2 * I + I + rb * 128;
        t.sw0 = e * (2 * ib) + rb;
        t.sw1 = e * (2 * ib) + ib + rb;
        t.a_row = off + c * sz;
        t.n = (cnt - c * sz) < sz ? (cnt - c * sz) : sz;
        t.out_row = t.a_row;
        t.out_col = rb * 128;
        tiles1[base1 + rb * nch + c] = t;
      }
    }
    for (int p = 0; p < nb2; ++p) {
      for (int c = 0; c < nch; ++c) {
        GemmTile t;
        t.w_row0 = e * H + (2 * p) * 128;
        t.w_row1 = (2 * p + 1 < hb) ? e * H + (2 * p + 1) * 128 : -1;
        t.sw0 = e * hb + 2 * p;
        t.sw1 = e * hb + 2 * p + 1;
        t.a_row = off + c * sz;
        t.n = (cnt - c * sz) < sz ? (cnt - c * sz) : sz;
        t.out_row = t.a_row;
        t.out_col = 2 * p * 128;
        tiles2[base2 + p * nch + c] = t;
      }
    }
  }
  if (threadIdx.x == 0) {
    ntiles[0] = (sh_chunks + total_chunks) * nb1;
    ntiles[1] = (sh_chunks + total_chunks) * nb2;
    ntiles[2] = total_rows;
    ntiles[3] = total_chunks;
  }
}

__global__ void __launch_bounds__(256) scatter_kernel(const int32_t *__restrict__ idx, const float *__restrict__ gate,
                                                       const uint8_t *__restrict__ xq, const float *__restrict__ xs,
                                                       int64_t T, int Kr, int Nr, int Ns, int H,
                                                       const int32_t *__restrict__ blk_base, uint8_t *__restrict__ ap,
                                                       float *__restrict__ as, float *__restrict__ row_gate,
                                                       int32_t *__restrict__ pos) {
  __shared__ int s_cnt[256];
  __shared__ int s_pos[kTokBlock * 16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(b) * kTokBlock;
  const int nt = static_cast<int>((T - t0) < kTokBlock ? (T - t0) : kTokBlock);
  const int na = nt * Kr;
  const int64_t R = T * Kr;
  for (int e = threadIdx.x; e < Nr; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  if (warp == 0) {
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < na; base += 32) {
      const int a = base + lane;
      const bool valid = a < na;
      int e = valid ? idx[t0 * Kr + a] : -1;
      if (e < 0 || e >= Nr) e = -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & lt_mask);
      const int prior = (e >= 0) ? s_cnt[e] : 0;
      __syncwarp();
      if (e >= 0 && rank == 0) s_cnt[e] = prior + __popc(peers);
      __syncwarp();
      if (valid) s_pos[a] = (e >= 0) ? blk_base[static_cast<int64_t>(b) * Nr + e] + prior + rank : -1;
    }
  }
  __syncthreads();
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    const int p = s_pos[a];
    pos[t0 * Kr + a] = p;
    if (p >= 0) row_gate[p] = gate[t0 * Kr + a];
  }
  if (Ns)
    for (int i = threadIdx.x; i < nt; i += blockDim.x) row_gate[R + t0 + i] = 1.0f;
  const int hv = H / 16, hs = H / 128;
  for (int a = warp; a < na; a += blockDim.x / 32) {
    const int p = s_pos[a];
    if (p < 0) continue;
    const int64_t t = t0 + a / Kr;
    const uint4 *src = reinterpret_cast<const uint4 *>(xq + t * H);
    uint4 *dst = reinterpret_cast<uint4 *>(ap + static_cast<int64_t>(p) * H);
    for (int i = lane; i < hv; i += 32) dst[i] = __ldg(src + i);
    for (int i = lane; i < hs; i += 32) as[static_cast<int64_t>(p) * hs + i] = __ldg(xs + t * hs + i);
  }
}

cudaError_t launch_hist(const int32_t *idx, int64_t T, int Kr, int Nr, int32_t *blk_hist, int32_t *err,
                        cudaStream_t st) {
  const int64_t nblk = (T + kTokBlock - 1) / kTokBlock;
  if (nblk == 0) return cudaSuccess;
  hist_kernel<<<static_cast<unsigned>(nblk), 256, 0, st>>>(idx, T, Kr, Nr, blk_hist, err);
  return cudaGetLastError();
}

cudaError_t launch_build_tiles(const int32_t *blk_hist, int64_t T, int Kr, int Nr, int Ns, int H, int I,
                               int32_t *counts, int32_t *offsets, int32_t *blk_base, GemmTile *tiles1,
                               GemmTile *tiles2, int32_t *ntiles, int32_t *counts_out, cudaStream_t st) {
  build_tiles_kernel<<<1, 256, 0, st>>>(blk_hist, T, Kr, Nr, Ns, H, I, counts, offsets, blk_base, tiles1, tiles2,
                                        ntiles, counts_out);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const int32_t *idx, const float *gate, const uint8_t *xq, const float *xs, int64_t T,
                           int Kr, int Nr, int Ns, int H, const int32_t *blk_base, uint8_t *ap, float *as,
                           float *row_gate, int32_t *pos, cudaStream_t st) {
  const int64_t nblk = (T + kTokBlock - 1) / kTokBlock;
  if (nblk == 0) return cudaSuccess;
  scatter_kernel<<<static_cast<unsigned>(nblk), 256, 0, st>>>(idx, gate, xq, xs, T, Kr, Nr, Ns, H, blk_base, ap,
                                                               as, row_gate, pos);
  return cudaGetLastError();
}

}  // namespace moe
