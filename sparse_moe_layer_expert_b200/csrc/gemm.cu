// gemm.cu -- grouped, fine-grained block-scaled FP8 GEMM for sm_100a.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Kernideen, FP8 bullet:
// E4M3 operands, 1x128 scales on activations, 128x128 scales on weights, and
// the partial sums promoted to FP32 every N_c = 128 accumulation steps.  The
// pages do this on Hopper by copying the tensor-core partials into CUDA-core
// registers; here the same arithmetic is laid out for Blackwell:
//
//   * tile = up to 128 activation rows (one expert's rows, padded to the MMA's
//     M = 128) x a pair of 128-row weight blocks (N = 256: for the gate/up
//     projection the gate block and the up block of the same 128 channels);
//   * one 128-long K block per pipeline stage: TMA brings the 128x128 byte
//     activation tile and the two weight tiles into shared memory (128-byte
//     swizzle, K-major) -- the weights stream from HBM once per tile;
//   * one thread issues tcgen05.mma kind::f8f6f4 (M = 128, N = 256,
//     K = 4 x 32) into a TMEM partial that starts from zero for every K
//     block -- the tensor core only ever sums 128 products;
//   * 256 promotion threads (two warpgroups) each own one activation row and
//     64 columns of each weight block: they read the partial with tcgen05.ld
//     and fold it into FP32 register accumulators with FMA by the scalar
//     sA[row, kb] * sW[block, kb] (one scale per thread per block and K
//     block, so promotion needs no per-element scale loads);
//   * TMEM holds two partial buffers (2 x 256 columns), so the tensor core
//     fills one while the promotion threads drain the other.
//
// Epilogues (after the last K block of a tile), one row per thread:
//   EPI_SWIGLU_Q  block A = gate, block B = up: h = silu(G) * U in FP32, then
//                 the 1x128 requantization of h over the tile's 128 channels
//                 (amax of the row's two 64-channel halves exchanged between
//                 the warpgroups, S = amax / 448, E4M3 RNE), 64 codes per
//                 thread stored as 16-byte vectors -> hq, scale -> hs
//   EPI_GATE_F32  y = acc * gate[row] as FP32 (down projection)
//   EPI_BF16      C = bf16(acc) (plain GEMM)
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warp 2 scale producer, warp 3 idle, warps 4..11 promotion +
// epilogue (two warpgroups).  Every wait is bounded (see common.cuh) so a
// fault upstream ends the kernel with MOE_DEVERR_TIMEOUT instead of a hang.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int G_STAGES = 4;
constexpr int G_SSLOTS = 8;
constexpr int G_AB = 128 * 128;           // activation tile: 128 rows x 128 bytes
constexpr int G_WB = 128 * 128;           // one 128x128 weight tile (bytes)
constexpr int G_STAGE = G_AB + 2 * G_WB;  // 48 KB
constexpr int G_THREADS = 384;
// Scale slot (floats): [0, 132) activation scales of the tile's rows, starting
// at row offset out_row & 3 (a bulk copy starts on a 16-byte boundary);
// [132] and [133] the two weight-block scales.
constexpr int G_RING = 136;
constexpr int G_SA_SPAN = 132;            // activation scales copied per K block
constexpr int G_AMAX = 2 * 128;           // floats, SwiGLU amax exchange (per warpgroup, per row)
constexpr int G_KBMAX = 256;              // K/128 up to 256 (K <= 32768)
constexpr int G_WSC = 2 * 2 * G_KBMAX;    // floats: weight-scale rows of 2 tiles x 2 blocks
constexpr int G_OPITCH = 20;              // floats per row of an output transpose buffer (16 + pad)
constexpr int G_OUTX = 8 * 32 * G_OPITCH; // floats: one 32-row x 16-float buffer per promotion warp
constexpr int G_SMEM =
    1024 + G_STAGES * G_STAGE + G_SSLOTS * G_RING * 4 + G_AMAX * 4 + G_WSC * 4 + G_OUTX * 4 + 256;
static_assert(G_SMEM <= 232448, "shared memory budget");

struct GemmArgs {
  const int4 *chunks;        // chunk table, or null for the dense grid
  const int32_t *n_chunks;   // device count of chunks
  int max_chunks;
  int dense_chunks;
  int64_t dense_M;
  int nb;                    // weight-block pairs per chunk
  int gate_up;
  int a_is_out_row;          // activations are the rows of the previous GEMM's output
  int64_t half;
  int64_t rows_per_expert;
  const float *sw;
  const float *sa0;
  const float *sa1;
  int sa_transposed;         // [K/128][sa_ld] tables, sa_ld % 4 == 0, 132 floats of slack
  int64_t sa_ld;
  int KB;
  void *out;
  int64_t ldo;
  float *out_scale;
  int64_t ld_os;
  const float *row_gate;
  int32_t *err;
  uint64_t limit_ns;
  // bounds every tile is checked against before any access
  int64_t w_rows, a_rows0, a_rows1, out_rows, out_cols;
};

struct GemmBars {
  uint64_t full[G_STAGES];
  uint64_t empty[G_STAGES];
  uint64_t sfull[G_SSLOTS];
  uint64_t sempty[G_SSLOTS];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};

// Tile t = (chunk t / nb, weight-block pair t % nb).
__device__ __forceinline__ GemmTile get_tile(const GemmArgs &a, int t) {
  const int c = t / a.nb, rb = t - (t / a.nb) * a.nb;
  GemmTile d;
  int e;
  if (a.chunks) {
    const int4 ch = a.chunks[c];
    e = ch.x & 0xFFFF;
    d.from1 = (ch.x >> 16) & 1;
    d.a_row = ch.y;
    d.out_row = ch.z;
    d.n = ch.w;
  } else {
    e = 0;
    d.from1 = 0;
    d.a_row = c * 128;
    const int64_t rem = a.dense_M - static_cast<int64_t>(c) * 128;
    d.n = rem < 128 ? static_cast<int32_t>(rem) : 128;
    d.out_row = d.a_row;
  }
  if (a.a_is_out_row) {
    d.a_row = d.out_row;
    d.from1 = 0;
  }
  const int64_t base = static_cast<int64_t>(e) * a.rows_per_expert;
  if (a.gate_up) {
    d.w_row0 = static_cast<int32_t>(base + rb * 128);
    d.w_row1 = static_cast<int32_t>(base + a.half + rb * 128);
    d.out_col = rb * 128;
  } else {
    d.w_row0 = static_cast<int32_t>(base + 2 * rb * 128);
    d.w_row1 = (static_cast<int64_t>(2 * rb + 1) * 128 < a.rows_per_expert) ? d.w_row0 + 128 : -1;
    d.out_col = 2 * rb * 128;
  }
  d.pad = 0;
  return d;
}

// A tile whose fields would read or write outside the operands is skipped by
// every role alike (and reported), so a corrupt chunk table cannot fault.
__device__ __forceinline__ bool tile_ok(const GemmArgs &a, const GemmTile &d) {
  const int64_t arows = d.from1 ? a.a_rows1 : a.a_rows0;
  const bool two = d.w_row1 >= 0;
  return d.n >= 1 && d.n <= 128 && d.a_row >= 0 && d.a_row + d.n <= arows && d.out_row >= 0 &&
         d.out_row + d.n <= a.out_rows && d.w_row0 >= 0 && d.w_row0 + 128 <= a.w_rows &&
         (!two || d.w_row1 + 128 <= a.w_rows) && d.out_col >= 0 && d.out_col + (two ? 256 : 128) <= a.out_cols &&
         (!a.sa_transposed || d.out_row + d.n <= a.sa_ld) && a.KB <= G_KBMAX;
}
}  // namespace

template <int EPI>
__global__ void __launch_bounds__(G_THREADS, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_a0,
                    const __grid_constant__ CUtensorMap map_a1, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *sring = reinterpret_cast<float *>(smem + G_STAGES * G_STAGE);
  float *amax_x = sring + G_SSLOTS * G_RING;
  float *wsc = amax_x + G_AMAX;
  float *outx = wsc + G_WSC;
  GemmBars *bars = reinterpret_cast<GemmBars *>(outx + G_OUTX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < G_STAGES; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < G_SSLOTS; ++i) {
      mbar_init(&bars->sfull[i], 2);  // the bulk copy's expect_tx arrival + the weight scales
      mbar_init(&bars->sempty[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->tfull[i], 1);
      mbar_init(&bars->tempty[i], 8);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&map_w);
    tma_prefetch_map(&map_a0);
    tma_prefetch_map(&map_a1);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abortp = &bars->abort_flag;
  const WaitCtl ctl{abortp, args.err, args.limit_ns};
  int nchunks = args.chunks ? args.n_chunks[0] : args.dense_chunks;
  if (nchunks > args.max_chunks || nchunks < 0) {
    if (threadIdx.x == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
    nchunks = nchunks < 0 ? 0 : args.max_chunks;
  }
  const int ntiles = nchunks * args.nb;
  const int KB = args.KB;

  // Register split: warps 0..3 (producer, MMA, scales) keep 72 registers,
  // the two promotion warpgroups get 216; 128*72 + 256*216 = 384*168, the
  // allocation the CTA is launched with.  Each role's code sits inside the
  // branch that resizes its registers so ptxas allocates it at that size.
  if (warp < 4) {
    setmaxnreg_dec<72>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_a = policy_evict_last();
        uint32_t it = 0;
        bool stop = false;
        GemmTile tn = get_tile(args, blockIdx.x < ntiles ? blockIdx.x : 0);  // next tile, loaded one tile ahead
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const GemmTile td = tn;
          if (tile + gridDim.x < ntiles) tn = get_tile(args, tile + gridDim.x);
          if (!tile_ok(args, td)) continue;
          const CUtensorMap *amap = td.from1 ? &map_a1 : &map_a0;
          const bool two = td.w_row1 >= 0;
          const uint32_t bytes = G_AB + (two ? 2 : 1) * G_WB;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % G_STAGES;
            if (!mbar_wait(&bars->empty[s], ((it / G_STAGES) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * G_STAGE;
            mbar_arrive_expect_tx(&bars->full[s], bytes);
            const int x = kb * 128;
            tma_load_2d_hint(st, amap, &bars->full[s], x, td.a_row, pol_a);
            tma_load_2d_hint(st + G_AB, &map_w, &bars->full[s], x, td.w_row0, pol_w);
            if (two) tma_load_2d_hint(st + G_AB + G_WB, &map_w, &bars->full[s], x, td.w_row1, pol_w);
          }
        }
        // let copies still in flight land before the CTA can exit
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < G_STAGES ? it : G_STAGES;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->full[j % G_STAGES], (j / G_STAGES) & 1, drain);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0;
        bool stop = false;
        GemmTile tn = get_tile(args, blockIdx.x < ntiles ? blockIdx.x : 0);  // next tile, loaded one tile ahead
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const GemmTile td = tn;
          if (tile + gridDim.x < ntiles) tn = get_tile(args, tile + gridDim.x);
          if (!tile_ok(args, td)) continue;
          const bool two = td.w_row1 >= 0;
          // D[128 activation rows, 256 (or 128) weight rows]
          const uint32_t idesc = idesc_e4m3_f32(128, two ? 256 : 128);
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % G_STAGES;
            const uint32_t buf = it & 1;
            if (!mbar_wait2(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, &bars->full[s], (it / G_STAGES) & 1, ctl)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(stages + s * G_STAGE);
            const uint64_t da = sw128_kmajor_desc(base);
            const uint64_t dw = sw128_kmajor_desc(base + G_AB);
            const uint32_t d0 = tmem + buf * 256;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // +32 bytes along K inside the 128-byte swizzled row = +2 in the
              // descriptor's 16-byte address units
              umma_f8(d0, da + 2 * k, dw + 2 * k, idesc, k > 0 ? 1u : 0u);
            }
            umma_commit(&bars->empty[s]);
            umma_commit(&bars->tfull[buf]);
          }
        }
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        umma_commit(&bars->teardown);
        mbar_wait(&bars->teardown, 0, drain);
      }
    } else if (warp == 2) {
      // -------------------------------------------------------- scale producer
      // Fills one promotion-ring slot per K block: the K block's activation
      // scales of the tile's rows (one bulk copy from the transposed table,
      // completing on the slot's barrier) and the two weight-block scales
      // (from the tile's weight-scale rows, staged in shared memory once per
      // tile).  The ring runs up to G_SSLOTS K blocks ahead of promotion.
      uint32_t it = 0;
      int par = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
        if (*abortp) break;
        const GemmTile td = get_tile(args, tile);
        if (!tile_ok(args, td)) {
          if (lane == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
          continue;
        }
        const bool two = td.w_row1 >= 0;
        float *wA = wsc + par * (2 * G_KBMAX), *wB = wA + G_KBMAX;
        par ^= 1;
        {
          const float *swa = args.sw + static_cast<int64_t>(td.w_row0 / 128) * KB;
          const float *swb = args.sw + static_cast<int64_t>((two ? td.w_row1 : td.w_row0) / 128) * KB;
          for (int i = lane; i < KB; i += 32) {
            wA[i] = __ldg(swa + i);
            wB[i] = two ? __ldg(swb + i) : 0.0f;
          }
          __syncwarp();
        }
        const float *sa = td.from1 ? args.sa1 : args.sa0;
        const int off = args.sa_transposed ? (td.out_row & 3) : 0;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int slot = it % G_SSLOTS;
          if (!mbar_wait(&bars->sempty[slot], ((it / G_SSLOTS) & 1) ^ 1, ctl)) {
            stop = true;
            break;
          }
          float *rs = sring + slot * G_RING;
          if (args.sa_transposed) {
            if (lane == 0) {
              mbar_arrive_expect_tx(&bars->sfull[slot], G_SA_SPAN * 4);
              bulk_load(rs, sa + static_cast<int64_t>(kb) * args.sa_ld + (td.out_row - off), G_SA_SPAN * 4,
                        &bars->sfull[slot]);
            }
          } else {
            // row-major scales [rows, K/128] (plain GEMM): strided loads
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = lane + 32 * i;
              rs[j] = (j < td.n) ? __ldg(sa + static_cast<int64_t>(td.a_row + j) * KB + kb) : 0.0f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sfull[slot]);
          }
          if (lane == 0) {
            rs[132] = wA[kb];
            rs[133] = wB[kb];
            mbar_arrive(&bars->sfull[slot]);
          }
        }
      }
    }
  } else {
    setmaxnreg_inc<216>();
    // ------------------------------------------------- promotion + epilogue
    const int wg = (warp - 4) >> 2;  // which 64 columns of each weight block
    const int q = warp & 3;          // TMEM lane quarter
    const int r = q * 32 + lane;     // activation row of this thread inside the tile
    float *amx = amax_x;             // [2 warpgroups][128 rows]
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (named_bar_or(1, 256, *abortp != 0)) break;
      const GemmTile td = get_tile(args, tile);
      if (!tile_ok(args, td)) continue;
      const bool two = td.w_row1 >= 0;
      const int soff = args.sa_transposed ? (td.out_row & 3) : 0;  // row offset inside a scale slot
      // a warp whose 32 rows are all padding (short chunks) skips its TMEM
      // reads and FMAs; it still takes every wait and arrival of the ring
      const bool live = q * 32 < td.n;
      float acc0[64], acc1[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t buf = it & 1;
        const int slot = it % G_SSLOTS;
        const bool ok = mbar_wait2(&bars->tfull[buf], (it >> 1) & 1, &bars->sfull[slot], (it / G_SSLOTS) & 1, ctl);
        if (ok && live) {
          tc_fence_after();
          const float *rs = sring + slot * G_RING;
          const float sx = rs[r + soff];
          const float ca = sx * rs[132];  // promotion scale of block A for this row
          const float cb = sx * rs[133];  // and of block B
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + wg * 64;
          uint32_t p[64];
          tmem_ld64(ta, p);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_scalar(acc0[j], acc0[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), ca);
          if (two) {
            tmem_ld64(ta + 128, p);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 64; j += 2)
              ffma2_scalar(acc1[j], acc1[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), cb);
          }
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->tempty[buf]);
          mbar_arrive(&bars->sempty[slot]);
        }
      }

      const bool valid = r < td.n;
      const int64_t orow = static_cast<int64_t>(td.out_row) + r;
      const int c0 = td.out_col + wg * 64;  // first output column of this thread (block A)
      if constexpr (EPI == EPI_SWIGLU_Q) {
        // h = silu(G) * U in FP32 for this row's 64 channels (fast exp and
        // divide: a few ulp, far inside the layer's tolerance)
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float g = acc0[j];
          acc0[j] = __fdividef(g, 1.0f + __expf(-g)) * acc1[j];
          amax = fmaxf(amax, fabsf(acc0[j]));
        }
        // amax over the tile's 128 channels = this warpgroup's 64 + the other's
        amx[wg * 128 + r] = amax;
        named_bar_sync(1, 256);
        amax = fmaxf(amx[r], amx[128 + r]);
        const float S = amax / 448.0f;
        if (valid) {
          uint8_t *hq = static_cast<uint8_t *>(args.out) + orow * args.ldo + c0;
          uint4 *hq4 = reinterpret_cast<uint4 *>(hq);
          if (S != 0.0f) {
            // quotients h / S share the divisor: correctly rounded through the
            // reciprocal plus one residual correction
            const float y = __frcp_rn(S);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int j = v * 16 + k * 4;
                const uint32_t lo = e4m3x2_rn_sat(div_by_recip(acc0[j], S, y), div_by_recip(acc0[j + 1], S, y));
                const uint32_t hi =
                    e4m3x2_rn_sat(div_by_recip(acc0[j + 2], S, y), div_by_recip(acc0[j + 3], S, y));
                w[k] = lo | (hi << 16);
              }
              hq4[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v) hq4[v] = make_uint4(0, 0, 0, 0);
          }
          if (wg == 0) args.out_scale[static_cast<int64_t>(td.out_col / 128) * args.ld_os + orow] = S;
        }
        named_bar_sync(1, 256);  // amx is reused by the next tile
      } else {
        // Rows are written through a per-warp 32 x 16-float transpose buffer
        // so that each 16-byte store instruction covers 8 rows x 64
        // contiguous bytes instead of 32 scattered rows.
        float *xb = outx + (warp - 4) * (32 * G_OPITCH);
        const int rbase = q * 32;  // this warp's first row in the tile
        const float g = (EPI == EPI_GATE_F32 && valid) ? __ldg(args.row_gate + orow) : 1.0f;
        auto emit = [&](const float(&acc)[64], int b) {
#pragma unroll
          for (int piece = 0; piece < (EPI == EPI_GATE_F32 ? 4 : 2); ++piece) {
            // stage: this thread's 16 floats (or 32 bf16) of the piece, row = lane
            float4 *dst = reinterpret_cast<float4 *>(xb + lane * G_OPITCH);
            if constexpr (EPI == EPI_GATE_F32) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int j = piece * 16 + 4 * v;
                dst[v] = make_float4(acc[j] * g, acc[j + 1] * g, acc[j + 2] * g, acc[j + 3] * g);
              }
            } else {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                float f[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int j = piece * 32 + 8 * v + 2 * k;
                  const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[j], acc[j + 1]);
                  f[k] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&b2));
                }
                dst[v] = make_float4(f[0], f[1], f[2], f[3]);
              }
            }
            __syncwarp();
            // drain: lane L stores 16 bytes of row (L / 4 + 8 s), chunk L % 4
#pragma unroll
            for (int sgrp = 0; sgrp < 4; ++sgrp) {
              const int rr = lane / 4 + 8 * sgrp;  // row within the warp's 32
              if (rbase + rr < td.n) {
                const float4 val = reinterpret_cast<const float4 *>(xb + rr * G_OPITCH)[lane & 3];
                const int64_t grow = static_cast<int64_t>(td.out_row) + rbase + rr;
                if constexpr (EPI == EPI_GATE_F32) {
                  float *yrow = static_cast<float *>(args.out) + grow * args.ldo + c0 + 128 * b + piece * 16;
                  reinterpret_cast<float4 *>(yrow)[lane & 3] = val;
                } else {
                  __nv_bfloat16 *crow =
                      static_cast<__nv_bfloat16 *>(args.out) + grow * args.ldo + c0 + 128 * b + piece * 32;
                  reinterpret_cast<float4 *>(crow)[lane & 3] = val;
                }
              }
            }
            __syncwarp();
          }
        };
        emit(acc0, 0);
        if (two) emit(acc1, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int EPI>
static cudaError_t launch_epi(const CUtensorMap &mw, const CUtensorMap &m0, const CUtensorMap &m1,
                              const GemmArgs &a, int grid, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e =
        cudaFuncSetAttribute(gemm_fp8_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  gemm_fp8_kernel<EPI><<<grid, G_THREADS, G_SMEM, st>>>(mw, m0, m1, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t st) {
  if (g.max_chunks <= 0 || g.nb <= 0) return cudaSuccess;
  CUtensorMap mw, m0, m1;
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, K, g.w_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a0, K, g.a0_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a1, K, g.a1_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.chunks = g.chunks;
  a.n_chunks = g.n_chunks;
  a.max_chunks = g.max_chunks;
  a.dense_M = g.dense_M;
  a.dense_chunks = g.chunks ? 0 : static_cast<int>((g.dense_M + 127) / 128);
  a.nb = g.nb;
  a.gate_up = g.gate_up;
  a.a_is_out_row = g.a_is_out_row;
  a.half = g.half;
  a.rows_per_expert = g.rows_per_expert;
  a.sw = g.sw;
  a.sa0 = g.sa0;
  a.sa1 = g.sa1;
  a.sa_transposed = g.sa_transposed;
  a.sa_ld = g.sa_ld;
  a.KB = static_cast<int>(g.K / 128);
  a.out = g.out;
  a.ldo = g.ldo;
  a.out_scale = g.out_scale;
  a.ld_os = g.ld_os;
  a.row_gate = g.row_gate;
  a.err = g.err;
  a.limit_ns = g.wait_limit_ns;
  a.w_rows = g.w_rows;
  a.a_rows0 = g.a0_rows;
  a.a_rows1 = g.a1_rows;
  a.out_rows = g.out_rows;
  a.out_cols = g.out_cols;
  const int sms = moe_host::sm_count();
  const int64_t max_tiles = static_cast<int64_t>(g.max_chunks) * g.nb;
  const int grid = static_cast<int>(max_tiles < sms ? max_tiles : sms);
  switch (g.epi) {
    case EPI_SWIGLU_Q: return launch_epi<EPI_SWIGLU_Q>(mw, m0, m1, a, grid, st);
    case EPI_GATE_F32: return launch_epi<EPI_GATE_F32>(mw, m0, m1, a, grid, st);
    default: return launch_epi<EPI_BF16>(mw, m0, m1, a, grid, st);
  }
}

}  // namespace moe
