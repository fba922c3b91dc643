// gemm.cu -- grouped, fine-grained block-scaled FP8 GEMM for sm_100a.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Kernideen, FP8 bullet:
// E4M3 operands, 1x128 scales on activations, 128x128 scales on weights, and
// the partial sums promoted to FP32 every N_c = 128 accumulation steps.  The
// pages do this on Hopper by copying the tensor-core partials into CUDA-core
// registers; here the same arithmetic is laid out for Blackwell:
//
//   * one 128-long K block per pipeline stage: TMA brings a 128x128 tile of
//     each of two weight blocks (A, B) and up to 128 activation rows into
//     shared memory (128-byte swizzle, K-major);
//   * one thread issues tcgen05.mma kind::f8f6f4 (M = 128 weight rows,
//     N = activation rows rounded up to 16, K = 4 x 32) into a TMEM partial
//     that starts from zero for every K block -- the tensor core only ever
//     sums 128 products;
//   * 256 promotion threads (two warpgroups, one per half of the activation
//     columns) read each partial with tcgen05.ld and fold it into FP32
//     register accumulators with FMA by the combined scale sA[row, kb] *
//     sW[block, kb] (precomputed per K block by a scale warp);
//   * TMEM holds two partial buffers (2 x 256 columns), so the tensor core
//     fills one while the promotion threads drain the other.
//
// The weight block is the MMA's M operand ("swap AB"): the weights stream
// from HBM exactly once per tile, the ragged number of activation rows per
// expert only sets the MMA's N (multiple of 16) -- no padding to 128 rows.
//
// Epilogues (after the last K block of a tile):
//   EPI_SWIGLU_Q  block A = gate rows, block B = up rows of the same 128
//                 intermediate channels: h = silu(G) * U in FP32, then the
//                 1x128 requantization of h (amax over the 128 channels of the
//                 tile, S = amax / 448, E4M3 RNE) -> hq, hs
//   EPI_GATE_F32  y = acc * gate[row] as FP32 (down projection)
//   EPI_BF16      C = bf16(acc) (plain GEMM)
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warp 2 scale producer, warp 3 idle, warps 4..11 promotion +
// epilogue (two warpgroups).  Every wait is bounded (see common.cuh) so a fault upstream
// ends the kernel with MOE_DEVERR_TIMEOUT instead of a hang.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int G_STAGES = 4;
constexpr int G_SSLOTS = 8;
constexpr int G_WB = 128 * 128;           // one 128x128 weight tile (bytes)
constexpr int G_XB = 128 * 128;           // up to 128 activation rows x 128 bytes
constexpr int G_STAGE = 2 * G_WB + G_XB;  // 48 KB
constexpr int G_XBOX = 16;                // activation rows per TMA box
constexpr int G_THREADS = 384;
constexpr int G_RING = 256;               // floats per scale slot (A: 128, B: 128)
constexpr int G_AMAX = 2 * 4 * 64;        // floats, SwiGLU amax exchange
constexpr int G_SMEM = 1024 + G_STAGES * G_STAGE + G_SSLOTS * G_RING * 4 + G_AMAX * 4 + 256;

struct GemmArgs {
  const GemmTile *tiles;
  const int32_t *n_tiles;
  int tile_slot;
  int dense_ntiles;
  int dense_pairs;
  int dense_wblocks;
  int64_t dense_M;
  const float *sw;
  const float *sa0;
  const float *sa1;
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
  int max_tiles;
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

__device__ __forceinline__ GemmTile get_tile(const GemmArgs &a, int t) {
  if (a.tiles) return a.tiles[t];
  GemmTile d;
  const int np = t % a.dense_pairs, mc = t / a.dense_pairs;
  d.w_row0 = np * 256;
  d.w_row1 = (2 * np + 1 < a.dense_wblocks) ? np * 256 + 128 : -1;
  d.sw0 = 2 * np;
  d.sw1 = 2 * np + 1;
  d.a_row = mc * 128;
  const int64_t rem = a.dense_M - static_cast<int64_t>(mc) * 128;
  d.n = rem < 128 ? static_cast<int32_t>(rem) : 128;
  d.out_row = d.a_row;
  d.out_col = np * 256;
  return d;
}

// A tile whose fields would read or write outside the operands is skipped by
// every role alike (and reported), so a corrupt work list cannot fault.
__device__ __forceinline__ bool tile_ok(const GemmArgs &a, const GemmTile &d) {
  const int64_t arows = (d.out_col & kTileFromMap1) ? a.a_rows1 : a.a_rows0;
  const int64_t col0 = d.out_col & 0xFFFFFF;
  const bool two = d.w_row1 >= 0;
  return d.n >= 1 && d.n <= 128 && d.a_row >= 0 && d.a_row + d.n <= arows && d.out_row >= 0 &&
         d.out_row + d.n <= a.out_rows && d.w_row0 >= 0 && d.w_row0 + 128 <= a.w_rows &&
         (!two || d.w_row1 + 128 <= a.w_rows) && d.sw0 >= 0 && static_cast<int64_t>(d.sw0) * 128 < a.w_rows &&
         (!two || (d.sw1 >= 0 && static_cast<int64_t>(d.sw1) * 128 < a.w_rows)) && col0 >= 0 &&
         col0 + (two ? 256 : 128) <= a.out_cols;
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
  GemmBars *bars = reinterpret_cast<GemmBars *>(amax_x + G_AMAX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < G_STAGES; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < G_SSLOTS; ++i) {
      mbar_init(&bars->sfull[i], 1);
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
  int ntiles = args.tiles ? args.n_tiles[args.tile_slot] : args.dense_ntiles;
  if (ntiles > args.max_tiles) {
    if (threadIdx.x == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
    ntiles = args.max_tiles;
  }
  const int KB = args.KB;

  // Register split: warps 0..3 (producer, MMA, scales) keep 56 registers,
  // the two promotion warpgroups get 224; 128*56 + 256*224 = 384*168, the
  // allocation the CTA is launched with.  Each role's code sits inside the
  // branch that resizes its registers so ptxas allocates it at that size.
  if (warp < 4) {
    setmaxnreg_dec<56>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      uint32_t it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
        if (*abortp) break;
        const GemmTile td = get_tile(args, tile);
        if (!tile_ok(args, td)) continue;
        const CUtensorMap *amap = (td.out_col & kTileFromMap1) ? &map_a1 : &map_a0;
        const bool two = td.w_row1 >= 0;
        const int nbox = (td.n + G_XBOX - 1) / G_XBOX;
        const uint32_t bytes = (two ? 2 : 1) * G_WB + nbox * (G_XBOX * 128);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % G_STAGES;
          if (!mbar_wait(&bars->empty[s], ((it / G_STAGES) & 1) ^ 1, ctl)) {
            stop = true;
            break;
          }
          uint8_t *st = stages + s * G_STAGE;
          mbar_arrive_expect_tx(&bars->full[s], bytes);
          const int x = kb * 128;
          tma_load_2d_hint(st, &map_w, &bars->full[s], x, td.w_row0, pol_w);
          if (two) tma_load_2d_hint(st + G_WB, &map_w, &bars->full[s], x, td.w_row1, pol_w);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_hint(st + 2 * G_WB + b * (G_XBOX * 128), amap, &bars->full[s], x, td.a_row + b * G_XBOX,
                             pol_a);
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
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
        if (*abortp) break;
        const GemmTile td = get_tile(args, tile);
        if (!tile_ok(args, td)) continue;
        const bool two = td.w_row1 >= 0;
        const int nm = (td.n + 15) & ~15;
        const uint32_t idesc = idesc_e4m3_f32(128, nm);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % G_STAGES;
          const uint32_t buf = it & 1;
          if (!mbar_wait(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, ctl) ||
              !mbar_wait(&bars->full[s], (it / G_STAGES) & 1, ctl)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(stages + s * G_STAGE);
          const uint64_t da = sw128_kmajor_desc(base);
          const uint64_t db = sw128_kmajor_desc(base + G_WB);
          const uint64_t dx = sw128_kmajor_desc(base + 2 * G_WB);
          const uint32_t d0 = tmem + buf * 256;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // +32 bytes along K inside the 128-byte swizzled row = +2 in the
            // descriptor's 16-byte address units
            umma_f8(d0, da + 2 * k, dx + 2 * k, idesc, k > 0 ? 1u : 0u);
            if (two) umma_f8(d0 + 128, db + 2 * k, dx + 2 * k, idesc, k > 0 ? 1u : 0u);
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
    // ---------------------------------------------------------- scale producer
    uint32_t it = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
      if (*abortp) break;
      const GemmTile td = get_tile(args, tile);
      if (!tile_ok(args, td)) {
        if (lane == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
        continue;
      }
      const bool two = td.w_row1 >= 0;
      const float *sa = (td.out_col & kTileFromMap1) ? args.sa1 : args.sa0;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int slot = it % G_SSLOTS;
        if (!mbar_wait(&bars->sempty[slot], ((it / G_SSLOTS) & 1) ^ 1, ctl)) {
          stop = true;
          break;
        }
        const float wa = __ldg(args.sw + static_cast<int64_t>(td.sw0) * KB + kb);
        const float wb = two ? __ldg(args.sw + static_cast<int64_t>(td.sw1) * KB + kb) : 0.0f;
        float *cs = sring + slot * G_RING;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = lane + 32 * i;
          const float sx = (j < td.n) ? __ldg(sa + static_cast<int64_t>(td.a_row + j) * KB + kb) : 0.0f;
          cs[j] = sx * wa;
          cs[128 + j] = sx * wb;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->sfull[slot]);
      }
    }
  }
  } else {
    setmaxnreg_inc<224>();
    // ------------------------------------------------- promotion + epilogue
    const int wg = (warp - 4) >> 2;  // which half of the activation columns
    const int q = warp & 3;          // TMEM lane quarter
    const int row = q * 32 + lane;   // row inside a 128-row weight block
    const uint32_t bar_id = 1 + wg;
    float *amx = amax_x + wg * 4 * 64;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (named_bar_or(bar_id, 128, *abortp != 0)) break;
      const GemmTile td = get_tile(args, tile);
      if (!tile_ok(args, td)) continue;
      const bool two = td.w_row1 >= 0;
      int ncols = td.n - wg * 64;
      ncols = ncols < 0 ? 0 : (ncols > 64 ? 64 : ncols);
      float acc0[64], acc1[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t buf = it & 1;
        const int slot = it % G_SSLOTS;
        const bool ok = mbar_wait(&bars->tfull[buf], (it >> 1) & 1, ctl) &&
                        mbar_wait(&bars->sfull[slot], (it / G_SSLOTS) & 1, ctl);
        if (ok) {
          tc_fence_after();
          const float *cs = sring + slot * G_RING + wg * 64;
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + wg * 64;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (c * 32 < ncols) {
              uint32_t r[32];
              tmem_ld32(ta + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j)
                acc0[c * 32 + j] = fmaf(__uint_as_float(r[j]), cs[c * 32 + j], acc0[c * 32 + j]);
              if (two) {
                tmem_ld32(ta + 128 + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  acc1[c * 32 + j] = fmaf(__uint_as_float(r[j]), cs[128 + c * 32 + j], acc1[c * 32 + j]);
              }
            }
          }
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->tempty[buf]);
          mbar_arrive(&bars->sempty[slot]);
        }
      }

      const int col0 = td.out_col & 0xFFFFFF;
      if constexpr (EPI == EPI_SWIGLU_Q) {
        // h = silu(G) * U, FP32
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float g = acc0[j];
          acc0[j] = (g / (1.0f + expf(-g))) * acc1[j];
        }
        // per token: amax over the 128 channels = 4 warps x 32 lanes
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(acc0[j])));
          if (lane == (j & 31)) amx[q * 64 + j] = __uint_as_float(m);
        }
        named_bar_sync(bar_id, 128);
        uint8_t *hq = static_cast<uint8_t *>(args.out);
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < ncols) {
            const float a = fmaxf(fmaxf(amx[j], amx[64 + j]), fmaxf(amx[128 + j], amx[192 + j]));
            const float S = a / 448.0f;
            const uint8_t code = (S != 0.0f) ? e4m3_rn_sat(acc0[j] / S) : static_cast<uint8_t>(0);
            const int64_t orow = static_cast<int64_t>(td.out_row) + wg * 64 + j;
            hq[orow * args.ldo + col0 + row] = code;
            if (q == 0 && lane == (j & 31)) args.out_scale[orow * args.ld_os + col0 / 128] = S;
          }
        }
        named_bar_sync(bar_id, 128);
      } else if constexpr (EPI == EPI_GATE_F32) {
        float *y = static_cast<float *>(args.out);
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < ncols) {
            const int64_t orow = static_cast<int64_t>(td.out_row) + wg * 64 + j;
            const float g = __ldg(args.row_gate + orow);
            y[orow * args.ldo + col0 + row] = acc0[j] * g;
            if (two) y[orow * args.ldo + col0 + 128 + row] = acc1[j] * g;
          }
        }
      } else {
        __nv_bfloat16 *Cm = static_cast<__nv_bfloat16 *>(args.out);
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < ncols) {
            const int64_t orow = static_cast<int64_t>(td.out_row) + wg * 64 + j;
            Cm[orow * args.ldo + col0 + row] = __float2bfloat16_rn(acc0[j]);
            if (two) Cm[orow * args.ldo + col0 + 128 + row] = __float2bfloat16_rn(acc1[j]);
          }
        }
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
  if (g.max_tiles <= 0) return cudaSuccess;
  CUtensorMap mw, m0, m1;
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, K, g.w_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a0, K, g.a0_rows, K, 128, G_XBOX) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a1, K, g.a1_rows, K, 128, G_XBOX) != 0)
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.tiles = g.tiles;
  a.n_tiles = g.n_tiles;
  a.tile_slot = g.tile_slot;
  a.dense_wblocks = static_cast<int>(g.w_rows / 128);
  a.dense_pairs = (a.dense_wblocks + 1) / 2;
  a.dense_M = g.dense_M;
  a.dense_ntiles = g.tiles ? 0 : static_cast<int>(((g.dense_M + 127) / 128) * a.dense_pairs);
  a.sw = g.sw;
  a.sa0 = g.sa0;
  a.sa1 = g.sa1;
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
  a.max_tiles = g.max_tiles;
  const int sms = moe_host::sm_count();
  const int grid = g.max_tiles < sms ? g.max_tiles : sms;
  switch (g.epi) {
    case EPI_SWIGLU_Q: return launch_epi<EPI_SWIGLU_Q>(mw, m0, m1, a, grid, st);
    case EPI_GATE_F32: return launch_epi<EPI_GATE_F32>(mw, m0, m1, a, grid, st);
    default: return launch_epi<EPI_BF16>(mw, m0, m1, a, grid, st);
  }
}

}  // namespace moe
