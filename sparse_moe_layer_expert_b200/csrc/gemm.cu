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
// Epilogues (after the last K block of a tile, one row per thread; shared
// with the block-scaled kernel in gemm_tiles.cuh):
//   EPI_SWIGLU_Q  block A = gate, block B = up: h = silu(G) * U in FP32, then
//                 the 1x128 requantization of h over the tile's 128 channels
//                 (amax of the row's two 64-channel halves exchanged between
//                 the warpgroups, S = amax / 448, E4M3 RNE), 64 codes per
//                 thread stored as 16-byte vectors -> hq, scale -> hs
//   EPI_GATE_F32  y = acc * gate[row] in FP32 (down projection)
//   EPI_BF16      C = bf16(acc) (plain GEMM)
//   EPI_F32       C = acc in FP32 (the backward's recomputed G, U and dh)
//
// Rows over TMEM lanes: the MMA issuer (warp 1) shares sub-partition 1 with
// the promotion warps of TMEM lanes 32..63, which its instruction issue
// slows; so the tile's last 32 rows (often padding in a short chunk, whose
// warps then skip their reads) go to lanes 32..63: tile rows 0-31 / 32-63 /
// 64-95 / 96-127 sit in lanes 0-31 / 64-95 / 96-127 / 32-63.  The
// activation tile is loaded as four 32-row TMA boxes into those places (the
// boxes the chunk has no rows in from past the tensor's last row: zeros).
//
// FP32 outputs (EPI_GATE_F32, EPI_F32) leave through TMA stores, warp by
// warp: each promotion warp puts its 32 rows x 64 columns of a 128 x 128
// block into its own 8 KB of shared memory as two boxes of 32 rows x 32
// columns (128-byte swizzle) and its lane 0 stores them; the rows of a
// tile's last, partial quarter (rows beyond belong to the next chunk) are
// stored by their threads.  No barrier joins the warps at the end of a tile,
// so one warp's epilogue does not hold up the others, and the stores drain
// while the next tile's K blocks run (a down-projection tile has only I/128
// K blocks for 128 x 256 FP32 outputs).  Those two epilogues run with three
// operand stages, which leaves room for the 64 KB of staging.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warp 2 scale producer, warp 3 idle, warps 4..11 promotion +
// epilogue (two warpgroups).  Every wait is bounded (see common.cuh) so a
// fault upstream ends the kernel with MOE_DEVERR_TIMEOUT instead of a hang.
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

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
constexpr int G_WSC = 2 * 2 * G_KBMAX;    // floats: weight-scale rows of 2 tiles x 2 blocks
constexpr int G_OUTX = 8 * 32 * G_OPITCH; // floats: one 32-row x 16-float buffer per promotion warp
constexpr int G_OBOX = 32 * 128;          // one staged output box: 32 rows x 32 FP32 columns (bytes)
constexpr int G_ABOX = 32 * 128;          // one 32-row activation box
// TMEM lane quarter of tile-row quarter qa, and the tile-row quarter of lane quarter q
__host__ __device__ constexpr int lane_q_of_rows(int qa) { return qa == 0 ? 0 : (qa == 3 ? 1 : qa + 1); }
__host__ __device__ constexpr int rows_q_of_lane(int q) { return q == 0 ? 0 : (q == 1 ? 3 : q - 1); }
static_assert(rows_q_of_lane(lane_q_of_rows(0)) == 0 && rows_q_of_lane(lane_q_of_rows(1)) == 1 &&
                  rows_q_of_lane(lane_q_of_rows(2)) == 2 && rows_q_of_lane(lane_q_of_rows(3)) == 3,
              "row quarters and lane quarters are inverse maps");
constexpr int G_OBLK = 16 * G_OBOX;       // a 128 x 128 FP32 block: 4 row quarters x 4 column boxes

// Shared-memory plan per epilogue: FP32 outputs through TMA stores take three
// operand stages and one staged block; the others four stages and the
// per-warp transpose buffers.
template <int EPI>
struct GLayout {
  static constexpr bool kTma = EPI == EPI_GATE_F32 || EPI == EPI_F32;
  static constexpr int kStages = kTma ? 3 : 4;
  static constexpr int kOut = kTma ? G_OBLK : G_OUTX * 4;  // bytes, directly after the stages (1024-aligned)
  static constexpr int kSmem =
      1024 + kStages * G_STAGE + kOut + G_SSLOTS * G_RING * 4 + G_AMAX * 4 + G_WSC * 4 + 256;
  static_assert(kSmem <= 232448, "shared memory budget");
};

// This warp's 32 rows x 64 columns of a 128 x 128 FP32 block, times gate,
// into its 8 KB of staging as two boxes of 32 rows x 32 columns, each row's
// 128 bytes as 16-byte chunks at j ^ (lane & 7) (the tensor map's 128-byte
// swizzle).  Lane 0 first waits until its previous stores have read the area.
__device__ __forceinline__ void stage_rows_warp(const float (&acc)[64], float gate, uint8_t *wstage, int lane) {
  if (lane == 0) bulk_wait_read();
  __syncwarp();
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint8_t *box = wstage + b * G_OBOX + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = b * 32 + j * 4;
      *reinterpret_cast<float4 *>(box + ((j ^ (lane & 7)) << 4)) =
          make_float4(acc[c] * gate, acc[c + 1] * gate, acc[c + 2] * gate, acc[c + 3] * gate);
    }
  }
}

// Store this warp's part of one 128 x 128 FP32 block of a tile: rows
// 32 q .. 32 q + 31 (this thread: row 32 q + lane) and columns 64 wg .. +63
// of the block, at output (row0, col0).  A warp whose 32 rows all lie inside
// the tile's n rows stages them and its lane 0 stores the two boxes with TMA.
// A warp of the tile's last, partial quarter (rows beyond n belong to the
// next chunk) stages them too and then writes each of its m rows with one
// warp-wide access (8 bytes per lane, the row's 256 bytes contiguous).  No
// thread waits for another warp: the eight promotion warps leave a tile
// independently.
__device__ __forceinline__ void store_rows_warp(const float (&acc)[64], float gate, uint8_t *wstage,
                                                const CUtensorMap *map, float *out, int64_t ldo, int64_t row0,
                                                int col0, int n, int wg, int q, int lane) {  // q: row quarter
  const int m = n - 32 * q;  // rows of this quarter inside the tile
  if (m <= 0) return;
  stage_rows_warp(acc, gate, wstage, lane);
  if (m >= 32) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int32_t y0 = static_cast<int32_t>(row0 + 32 * q);
      tma_store_2d(map, wstage, col0 + 64 * wg, y0);
      tma_store_2d(map, wstage + G_OBOX, col0 + 64 * wg + 32, y0);
      bulk_commit();
    }
  } else {
    __syncwarp();
    // lane l holds columns 2l, 2l + 1: box l / 16, chunk (l % 16) / 2, half l % 2
    const uint8_t *src = wstage + (lane >> 4) * G_OBOX + (lane & 1) * 8;
    const int ch = (lane & 15) >> 1;
    float *dst = out + (row0 + 32 * q) * ldo + col0 + wg * 64 + 2 * lane;
    for (int i = 0; i < m; ++i)
      *reinterpret_cast<float2 *>(dst + i * ldo) =
          *reinterpret_cast<const float2 *>(src + i * 128 + ((ch ^ (i & 7)) << 4));
  }
}

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

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(G_THREADS, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_a0,
                    const __grid_constant__ CUtensorMap map_a1, const __grid_constant__ CUtensorMap map_out,
                    const GemmArgs args) {
  using L = GLayout<EPI>;
  constexpr int NST = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *ostage = smem + NST * G_STAGE;  // staged FP32 block, or the per-warp transpose buffers
  float *outx = reinterpret_cast<float *>(ostage);
  float *sring = reinterpret_cast<float *>(ostage + L::kOut);
  float *amax_x = sring + G_SSLOTS * G_RING;
  float *wsc = amax_x + G_AMAX;
  GemmBars *bars = reinterpret_cast<GemmBars *>(wsc + G_WSC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
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
        // weights: evict-first when one pass reads them, normal when the
        // other chunks of the expert read the same tiles right after
        const uint64_t pol_w1 = policy_evict_first();
        const uint64_t pol_wk = policy_evict_normal();
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
          const int nbox = (td.n + 31) / 32;  // activation boxes holding the chunk's rows (1..4)
          const uint32_t bytes = 4 * G_ABOX + (two ? 2 : 1) * G_WB;
          // the quarters without rows get a box from past the map's last row,
          // which TMA fills with zeros: the MMA then multiplies zeros there
          // instead of a stale stage's codes (the same result for the rows
          // that are kept, at a lower tensor-core power under the power cap)
          const int zrow = static_cast<int>(td.from1 ? args.a_rows1 : args.a_rows0);
          const uint64_t pol_w = td.group > 1 ? pol_wk : pol_w1;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % NST;
            if (!mbar_wait(&bars->empty[s], ((it / NST) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * G_STAGE;
            mbar_arrive_expect_tx(&bars->full[s], bytes);
            const int x = kb * 128;
            for (int b = 0; b < 4; ++b)
              tma_load_2d_hint(st + lane_q_of_rows(b) * G_ABOX, amap, &bars->full[s], x,
                               b < nbox ? td.a_row + 32 * b : zrow, pol_a);
            tma_load_2d_hint(st + G_AB, &map_w, &bars->full[s], x, td.w_row0, pol_w);
            if (two) tma_load_2d_hint(st + G_AB + G_WB, &map_w, &bars->full[s], x, td.w_row1, pol_w);
          }
        }
        // let copies still in flight land before the CTA can exit
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < NST ? it : NST;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->full[j % NST], (j / NST) & 1, drain);
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
            const int s = it % NST;
            const uint32_t buf = it & 1;
            if (!mbar_wait2(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, &bars->full[s], (it / NST) & 1, ctl)) {
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
    const int rq = rows_q_of_lane(q);  // the tile rows those lanes hold
    const int r = rq * 32 + lane;    // activation row of this thread inside the tile
    float *amx = amax_x;             // [2 warpgroups][128 rows]
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      // the SwiGLU epilogue exchanges amax between the warpgroups, so they
      // stop together; the FP32 epilogues have no cross-warp step
      if (L::kTma ? (*abortp != 0) : named_bar_or(1, 256, *abortp != 0)) break;
      const GemmTile td = get_tile(args, tile);
      if (!tile_ok(args, td)) continue;
      const bool two = td.w_row1 >= 0;
      const int soff = args.sa_transposed ? (td.out_row & 3) : 0;  // row offset inside a scale slot
      // a warp whose 32 rows are all padding (short chunks) skips its TMEM
      // reads and FMAs; it still takes every wait and arrival of the ring
      const bool live = rq * 32 < td.n;
      // the row's gate (down projection), loaded before the K loop so its
      // latency is not part of the epilogue
      const float gt = (EPI == EPI_GATE_F32 && r < td.n) ? __ldg(args.row_gate + td.out_row + r) : 1.0f;
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

      if constexpr (L::kTma) {
        // FP32 rows through TMA stores: block A at out_col + 64 wg, block B
        // at +128 (down projection) or +half (a gate/up pair)
        const int64_t cB = args.gate_up ? args.half : 128;
        float *outp = static_cast<float *>(args.out);
        uint8_t *wstage = ostage + (warp - 4) * 2 * G_OBOX;  // this warp's two boxes
        store_rows_warp(acc0, gt, wstage, &map_out, outp, args.ldo, td.out_row, td.out_col, td.n, wg, rq, lane);
        if (two)
          store_rows_warp(acc1, gt, wstage, &map_out, outp, args.ldo, td.out_row, static_cast<int>(td.out_col + cB),
                          td.n, wg, rq, lane);
      } else {
        tile_epilogue<EPI, false>(args, td, acc0, acc1, two, warp, lane, amx, outx, rq);
      }
    }
    // the staging area stays valid until each warp's last stores have read it
    if (L::kTma && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int EPI>
static cudaError_t launch_epi(const CUtensorMap &mw, const CUtensorMap &m0, const CUtensorMap &m1,
                              const CUtensorMap &mo, const GemmArgs &a, int grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_fp8_kernel<EPI>, GLayout<EPI>::kSmem, attr_done)) return e;
  gemm_fp8_kernel<EPI><<<grid, G_THREADS, GLayout<EPI>::kSmem, st>>>(mw, m0, m1, mo, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t st) {
  if (g.max_chunks <= 0 || g.nb <= 0) return cudaSuccess;
  CUtensorMap mw, m0, m1;
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, K, g.w_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  // activations in 32-row boxes (placed in the lane quarters above)
  if (moe_host::encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a0, K, g.a0_rows, K, 128, 32) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a1, K, g.a1_rows,
                               g.a1_ld ? static_cast<uint64_t>(g.a1_ld) : K, 128, 32) != 0)
    return cudaErrorInvalidValue;
  // FP32 outputs: [out_rows, ldo] in 32 x 32 boxes for the TMA-store epilogue
  // (the other epilogues get a copy of the weight map, never used)
  CUtensorMap mo = mw;
  if (g.epi == EPI_GATE_F32 || g.epi == EPI_F32) {
    if ((g.ldo * 4) % 16 != 0 || g.out_rows <= 0 ||
        moe_host::encode_tmap_2d(&mo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.out, static_cast<uint64_t>(g.ldo),
                                 static_cast<uint64_t>(g.out_rows), static_cast<uint64_t>(g.ldo) * 4, 32, 32) != 0)
      return cudaErrorInvalidValue;
  }
  GemmArgs a = make_args(g);
  const int sms = moe_host::sm_count();
  const int64_t max_tiles = static_cast<int64_t>(g.max_chunks) * g.nb;
  const int grid = static_cast<int>(max_tiles < sms ? max_tiles : sms);
  switch (g.epi) {
    case EPI_SWIGLU_Q: return launch_epi<EPI_SWIGLU_Q>(mw, m0, m1, mo, a, grid, st);
    case EPI_GATE_F32: return launch_epi<EPI_GATE_F32>(mw, m0, m1, mo, a, grid, st);
    case EPI_F32: return launch_epi<EPI_F32>(mw, m0, m1, mo, a, grid, st);
    default: return launch_epi<EPI_BF16>(mw, m0, m1, mo, a, grid, st);
  }
}

}  // namespace moe
