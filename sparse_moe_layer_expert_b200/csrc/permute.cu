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
//  hist_kernel         per 128-token block, per-expert counts
//  build_chunks_kernel one CTA: totals, exclusive scans, per-block bases and
//                      the chunk table (<= 128 or <= 256 rows of one expert
//                      per chunk, for one CTA or a CTA pair per tile) from
//                      which both grouped GEMMs derive their tiles
//  rank_kernel         per 128-token block: stable ranks (warp matches over
//                      8 ranges of the block) -> row of every (token, slot),
//                      per-row gate and source
//  copy_rows_kernel    one warp per row: FP8 row copy (16-byte vectors, eight
//                      loads in flight per lane) and, per CTA of 8 rows, the
//                      rows' scales into the transposed scale table as 8
//                      consecutive floats per K block
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kTokBlock = 128;

// idx entries of -1 mean "no expert in this slot" when allow_empty is set
// (rows received by an expert-parallel rank list only the slots whose expert
// lives there); any other value outside [0, Nr) is reported.
__global__ void __launch_bounds__(256) hist_kernel(const int32_t *__restrict__ idx, int64_t T, int Kr, int Nr,
                                                    int allow_empty, int32_t *__restrict__ blk_hist,
                                                    int32_t *__restrict__ err) {
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
    else if (!(allow_empty && e == -1))
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

// Chunk table entry: {expert | from_input << 16, activation row, output row, rows}.
__global__ void __launch_bounds__(256) build_chunks_kernel(const int32_t *__restrict__ blk_hist, int64_t T, int Kr,
                                                            int Nr, int Ns, int chunk_rows, int32_t *counts,
                                                            int32_t *offsets, int32_t *blk_base, int4 *chunks,
                                                            int32_t *meta, int32_t *counts_out) {
  const int e = threadIdx.x;
  const int nblk = static_cast<int>((T + kTokBlock - 1) / kTokBlock);
  const int64_t R = T * Kr;
  int cnt = 0;
  if (e < Nr)
    for (int b = 0; b < nblk; ++b) cnt += blk_hist[static_cast<int64_t>(b) * Nr + e];
  int total_rows;
  const int off = block_excl_scan(cnt, &total_rows);
  const int nch = (cnt + chunk_rows - 1) / chunk_rows;
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
  // shared-expert chunks first (full chunks: largest work first)
  const int sh_chunks = Ns ? static_cast<int>((T + chunk_rows - 1) / chunk_rows) : 0;
  for (int c = threadIdx.x; c < sh_chunks; c += blockDim.x) {
    const int64_t r0 = static_cast<int64_t>(c) * chunk_rows;
    const int n = static_cast<int>((T - r0) < chunk_rows ? (T - r0) : chunk_rows);
    chunks[c] = make_int4(Nr | (1 << 16) | (c << 17), static_cast<int>(r0), static_cast<int>(R + r0),
                          n | (sh_chunks << 16));
  }
  if (e < Nr && nch > 0) {
    const int sz = (cnt + nch - 1) / nch;  // <= chunk_rows: rows split evenly over the chunks
    for (int c = 0; c < nch; ++c) {
      const int r0 = off + c * sz;
      const int n = (cnt - c * sz) < sz ? (cnt - c * sz) : sz;
      chunks[sh_chunks + cbase + c] = make_int4(e | (c << 17), r0, r0, n | (nch << 16));
    }
  }
  if (threadIdx.x == 0) {
    meta[0] = sh_chunks + total_chunks;
    meta[1] = total_rows;
  }
}

// Stable ranks of one 128-token block's assignments.  The block's A = nt*K_r
// assignments (row-major (token, slot) order) are cut into 8 contiguous
// ranges, one per warp: pass 1 counts each expert per range, the per-expert
// counts of the earlier ranges give each range its starting rank, and pass 2
// ranks within the range with warp matches -- the order is the same as one
// sequential walk over the block, with an eighth of its dependent steps.
__global__ void __launch_bounds__(256) rank_kernel(const int32_t *__restrict__ idx, const float *__restrict__ gate,
                                                    int64_t T, int Kr, int Nr, int Ns,
                                                    const int32_t *__restrict__ blk_base,
                                                    float *__restrict__ row_gate, int32_t *__restrict__ row_src,
                                                    int32_t *__restrict__ pos) {
  constexpr int W = 8;
  __shared__ int s_cnt[W][256];   // pass 1: per range counts; then per range running ranks
  __shared__ int s_pos[kTokBlock * 16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(b) * kTokBlock;
  const int nt = static_cast<int>((T - t0) < kTokBlock ? (T - t0) : kTokBlock);
  const int na = nt * Kr;
  const int64_t R = T * Kr;
  const int per = (na + W - 1) / W;
  const int a0 = warp * per, a1 = (a0 + per) < na ? (a0 + per) : na;
  for (int i = threadIdx.x; i < W * 256; i += blockDim.x) (&s_cnt[0][0])[i] = 0;
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  // pass 1: counts per expert in this warp's range
  for (int base = a0; base < a1; base += 32) {
    const int a = base + lane;
    int e = a < a1 ? idx[t0 * Kr + a] : -1;
    if (e < 0 || e >= Nr) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && __popc(peers & lt_mask) == 0) s_cnt[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over the ranges, per expert, plus the block's base row
  for (int e = threadIdx.x; e < Nr; e += blockDim.x) {
    int run = blk_base[static_cast<int64_t>(b) * Nr + e];
    for (int w = 0; w < W; ++w) {
      const int c = s_cnt[w][e];
      s_cnt[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 2: ranks inside the range
  for (int base = a0; base < a1; base += 32) {
    const int a = base + lane;
    const bool valid = a < a1;
    int e = valid ? idx[t0 * Kr + a] : -1;
    if (e < 0 || e >= Nr) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    const int prior = (e >= 0) ? s_cnt[warp][e] : 0;
    __syncwarp();
    if (e >= 0 && rank == 0) s_cnt[warp][e] = prior + __popc(peers);
    __syncwarp();
    if (valid) s_pos[a] = (e >= 0) ? prior + rank : -1;
  }
  __syncthreads();
  for (int a = threadIdx.x; a < na; a += blockDim.x) {
    const int p = s_pos[a];
    pos[t0 * Kr + a] = p;
    if (p >= 0) {
      row_gate[p] = gate[t0 * Kr + a];
      row_src[p] = static_cast<int32_t>(t0 + a / Kr);
    }
  }
  if (Ns)
    for (int i = threadIdx.x; i < nt; i += blockDim.x) row_gate[R + t0 + i] = 1.0f;
}

// Rows [0, R): routed rows, copied from the quantized input row row_src[p]
// (xq rows xq_ld bytes apart, 16-byte aligned);
// rows [R, R + T): the shared expert's rows (token p - R), scales only (the
// gate/up GEMM reads their codes from the quantized input directly).
// Scales go to the transposed table as_t[kb * ld + p].
__global__ void __launch_bounds__(256) copy_rows_kernel(const uint8_t *__restrict__ xq, int64_t xq_ld,
                                                         const float *__restrict__ xs,
                                                         const int32_t *__restrict__ row_src, int64_t R, int64_t T,
                                                         int Ns, int H, uint8_t *__restrict__ ap,
                                                         float *__restrict__ as_t, int64_t ld) {
  constexpr int U = 8;        // 16-byte loads in flight per lane
  constexpr int KC = 32;      // K blocks of scales staged per pass
  __shared__ float sc[8][KC + 1];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * 8;
  const int64_t p = p0 + w;
  const int64_t rows = R + (Ns ? T : 0);
  const int hv = H / 16, kb = H / 128;
  int64_t t = -1;
  if (p < rows) {
    if (p < R) {
      t = row_src[p];
      if (t < 0 || t >= T) t = -1;
    } else {
      t = p - R;
    }
  }
  if (t >= 0 && p < R) {
    const uint4 *s = reinterpret_cast<const uint4 *>(xq + t * xq_ld);
    uint4 *d = reinterpret_cast<uint4 *>(ap + p * H);
    for (int base = 0; base < hv; base += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * 32 + lane;
        if (i < hv) v[u] = __ldg(s + i);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * 32 + lane;
        if (i < hv) d[i] = v[u];
      }
    }
  }
  // scales: the block's 8 rows go to as_t[k * ld + p0 .. p0 + 7], written
  // as 8 consecutive floats per K block
  for (int k0 = 0; k0 < kb; k0 += KC) {
    const int nk = kb - k0 < KC ? kb - k0 : KC;
    if (lane < nk) sc[w][lane] = t >= 0 ? __ldg(xs + t * kb + k0 + lane) : 0.0f;
    __syncthreads();
    const int j = threadIdx.x & 7, k = threadIdx.x >> 3;
    const int64_t pj = p0 + j;
    if (k < nk && pj < rows) {
      const bool live = pj >= R || (row_src[pj] >= 0 && row_src[pj] < T);
      if (live) as_t[static_cast<int64_t>(k0 + k) * ld + pj] = sc[j][k];
    }
    __syncthreads();
  }
}

cudaError_t launch_hist(const int32_t *idx, int64_t T, int Kr, int Nr, int allow_empty, int32_t *blk_hist,
                        int32_t *err, cudaStream_t st) {
  const int64_t nblk = (T + kTokBlock - 1) / kTokBlock;
  if (nblk == 0) return cudaSuccess;
  hist_kernel<<<static_cast<unsigned>(nblk), 256, 0, st>>>(idx, T, Kr, Nr, allow_empty, blk_hist, err);
  return cudaGetLastError();
}

cudaError_t launch_build_chunks(const int32_t *blk_hist, int64_t T, int Kr, int Nr, int Ns, int chunk_rows,
                                int32_t *counts, int32_t *offsets, int32_t *blk_base, int4 *chunks, int32_t *meta,
                                int32_t *counts_out, cudaStream_t st) {
  build_chunks_kernel<<<1, 256, 0, st>>>(blk_hist, T, Kr, Nr, Ns, chunk_rows, counts, offsets, blk_base, chunks,
                                         meta, counts_out);
  return cudaGetLastError();
}

cudaError_t launch_rank(const int32_t *idx, const float *gate, int64_t T, int Kr, int Nr, int Ns,
                        const int32_t *blk_base, float *row_gate, int32_t *row_src, int32_t *pos, cudaStream_t st) {
  const int64_t nblk = (T + kTokBlock - 1) / kTokBlock;
  if (nblk == 0) return cudaSuccess;
  rank_kernel<<<static_cast<unsigned>(nblk), 256, 0, st>>>(idx, gate, T, Kr, Nr, Ns, blk_base, row_gate, row_src,
                                                            pos);
  return cudaGetLastError();
}

cudaError_t launch_copy_rows(const uint8_t *xq, int64_t xq_ld, const float *xs, const int32_t *row_src, int64_t R,
                             int64_t T, int Ns, int H, uint8_t *ap, float *as_t, int64_t ld, cudaStream_t st) {
  const int64_t rows = R + (Ns ? T : 0);
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + 7) / 8;
  copy_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(xq, xq_ld, xs, row_src, R, T, Ns, H, ap, as_t,
                                                                   ld);
  return cudaGetLastError();
}

}  // namespace moe
