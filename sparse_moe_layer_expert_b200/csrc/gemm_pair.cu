// gemm_pair.cu -- the grouped, fine-grained block-scaled FP8 GEMM on CTA pairs.
//
// Same arithmetic as gemm.cu ("DeepSeek-V3 Technischer Bericht",
// xyznot.com/de, Kernideen, FP8 bullet: E4M3 operands, 1x128 activation
// scales, 128x128 weight-block scales, each 128-long partial promoted into
// FP32 with its two scales), laid out on the two SMs of a cluster of two CTAs
// so that one pass over a weight tile serves up to 256 activation rows:
//
//   * tile = up to 256 rows of one expert x a pair of 128-row weight blocks
//     (gate block j and up block j of the same 128 channels, or two adjacent
//     blocks of the down projection); the even CTA of the pair holds rows
//     0..127 and weight block A, the odd CTA rows 128..255 and weight block B;
//   * one tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32; four per 128-K
//     block), issued by the even CTA, reads both CTAs' shared memory and
//     leaves in each CTA's TMEM its own 128 rows x all 256 columns -- so each
//     CTA holds the gate and the up partials of its rows, and every SwiGLU /
//     requantization epilogue stays inside one CTA;
//   * per stage each CTA loads 32 KB (its activation tile and its weight
//     tile) instead of 48 KB on a single CTA, so six stages fit, and a chunk of
//     129..256 rows streams its weights once instead of twice;
//   * promotion as in gemm.cu: the partial of every K block starts from zero
//     in one of two TMEM buffers; 256 promotion threads per CTA fold it into
//     FP32 registers with sA[row, kb] * sW[block, kb].
//
// Synchronisation of the pair: both CTAs' TMA loads count on the even CTA's
// stage barrier (each CTA announces its own bytes); the even CTA's commits
// arrive on the stage-free and partial-ready barriers of both CTAs; the odd
// CTA's promotion warps report a drained TMEM buffer to the even CTA's
// barrier.  Every wait is bounded (common.cuh).
//
// Warp roles (384 threads per CTA): warp 0 TMA producer, warp 1 TMEM owner
// (and, in the even CTA, MMA issuer), warp 2 scale producer, warp 3 idle,
// warps 4..11 promotion + epilogue.
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

namespace {
constexpr int P_STAGES = 6;
constexpr int P_AB = 128 * 128;           // this CTA's 128 activation rows x 128 bytes
constexpr int P_WB = 128 * 128;           // this CTA's 128x128 weight tile
constexpr int P_STAGE = P_AB + P_WB;      // 32 KB
constexpr int P_THREADS = 384;
constexpr int P_SSLOTS = 8;
constexpr int P_RING = 136;               // floats per scale slot (as gemm.cu)
constexpr int P_SA_SPAN = 132;
constexpr int P_AMAX = 2 * 128;
constexpr int P_WSC = 2 * 2 * G_KBMAX;
constexpr int P_OUTX = 8 * 32 * G_OPITCH;
constexpr int P_BARS = 512;
constexpr int P_SMEM =
    1024 + P_STAGES * P_STAGE + P_SSLOTS * P_RING * 4 + P_AMAX * 4 + P_WSC * 4 + P_OUTX * 4 + P_BARS;
static_assert(P_SMEM <= 232448, "shared memory budget");

struct PairBars {
  uint64_t full[P_STAGES];    // even CTA: a stage's operands of both CTAs have landed (2 arrivals + bytes)
  uint64_t empty[P_STAGES];   // each CTA: the pair MMAs have read the stage
  uint64_t sfull[P_SSLOTS];
  uint64_t sempty[P_SSLOTS];
  uint64_t tfull[2];          // each CTA: a K block's partial is in this CTA's TMEM
  uint64_t tempty[2];         // even CTA: both CTAs' promotion warps have read the buffer (16 arrivals)
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PairBars) <= P_BARS, "barrier block");

// The rows of a pair tile that CTA `rank` holds.
__device__ __forceinline__ GemmTile sub_tile(const GemmTile &d, int rank) {
  GemmTile s = d;
  const int lo = 128 * rank;
  s.n = d.n > lo ? (d.n - lo < 128 ? d.n - lo : 128) : 0;
  s.a_row = d.a_row + lo;
  s.out_row = d.out_row + lo;
  return s;
}

// This CTA's rank in its pair, the pair's index and the number of pairs
// (read from special registers where used, so that no register holds them
// across the long loops).
__device__ __forceinline__ int pair_rank() { return static_cast<int>(cluster_ctarank()); }
__device__ __forceinline__ int pair_id() { return static_cast<int>(blockIdx.x >> 1); }
__device__ __forceinline__ int pair_count() { return static_cast<int>(gridDim.x >> 1); }

// A pair tile always has two weight blocks (the host takes this kernel only
// when the weight-block count is even).
__device__ __forceinline__ bool pair_tile_ok(const GemmArgs &a, const GemmTile &d) {
  return d.w_row1 >= 0 && tile_ok(a, d);
}
}  // namespace

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_a0,
                     const __grid_constant__ CUtensorMap map_a1, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *sring = reinterpret_cast<float *>(smem + P_STAGES * P_STAGE);
  float *amax_x = sring + P_SSLOTS * P_RING;
  float *wsc = amax_x + P_AMAX;
  float *outx = wsc + P_WSC;
  PairBars *bars = reinterpret_cast<PairBars *>(outx + P_OUTX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < P_STAGES; ++i) {
      mbar_init(&bars->full[i], 2);  // each CTA's producer announces its bytes
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < P_SSLOTS; ++i) {
      mbar_init(&bars->sfull[i], 2);
      mbar_init(&bars->sempty[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->tfull[i], 1);
      mbar_init(&bars->tempty[i], 16);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&map_w);
    tma_prefetch_map(&map_a0);
    tma_prefetch_map(&map_a1);
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars->tmem_base, 512);
    tmem_relinquish_pair();
  }
  // the peer's arrivals and copies may target this CTA's barriers only once
  // they are initialised: a cluster-wide barrier before any role starts
  tc_fence_before();
  cluster_sync_all();
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

  // Register split as in gemm.cu: 72 for warps 0..3, 216 for the promotion
  // warpgroups (128*72 + 256*216 = 384*168, the launch allocation).
  if (warp < 4) {
    setmaxnreg_dec<72>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint64_t pol_w1 = policy_evict_first();  // one pass reads the weight tile
        const uint64_t pol_wk = policy_evict_normal(); // the expert's other chunks read it next
        const uint64_t pol_a = policy_evict_last();
        uint32_t it = 0;
        bool stop = false;
        for (int tile = pair_id(); tile < ntiles && !stop; tile += pair_count()) {
          if (*abortp) break;
          const GemmTile td = get_tile(args, tile);
          if (!pair_tile_ok(args, td)) continue;
          const GemmTile sd = sub_tile(td, pair_rank());
          const CUtensorMap *amap = td.from1 ? &map_a1 : &map_a0;
          const int32_t w_row = pair_rank() == 0 ? td.w_row0 : td.w_row1;
          const uint32_t bytes = P_WB + (sd.n > 0 ? P_AB : 0);
          const uint64_t pol_w = td.group > 1 ? pol_wk : pol_w1;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % P_STAGES;
            if (!mbar_wait(&bars->empty[s], ((it / P_STAGES) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * P_STAGE;
            const uint32_t fbar = mapa_shared(smem_u32(&bars->full[s]), 0);
            mbar_arrive_expect_tx_cluster(fbar, bytes);
            const int x = kb * 128;
            if (sd.n > 0) tma_load_2d_pair(st, amap, fbar, x, sd.a_row, pol_a);
            tma_load_2d_pair(st + P_AB, &map_w, fbar, x, w_row, pol_w);
          }
        }
        // the stages still in flight are read by the pair MMAs before this
        // CTA may exit: wait until they are released
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < P_STAGES ? it : P_STAGES;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->empty[j % P_STAGES], (j / P_STAGES) & 1, drain);
      }
    } else if (warp == 1) {
      // ------------------------------------------------- MMA issuer (even CTA)
      if (lane == 0 && pair_rank() == 0) {
        uint32_t it = 0;
        bool stop = false;
        // D[256 rows of the pair, 256 weight rows]: M = 256 over the two CTAs
        const uint32_t idesc = idesc_e4m3_f32(256, 256);
        for (int tile = pair_id(); tile < ntiles && !stop; tile += pair_count()) {
          if (*abortp) break;
          const GemmTile td = get_tile(args, tile);
          if (!pair_tile_ok(args, td)) continue;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % P_STAGES;
            const uint32_t buf = it & 1;
            if (!mbar_wait2(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, &bars->full[s], (it / P_STAGES) & 1, ctl)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(stages + s * P_STAGE);
            const uint64_t da = sw128_kmajor_desc(base);
            const uint64_t dw = sw128_kmajor_desc(base + P_AB);
            const uint32_t d0 = tmem + buf * 256;
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f8_pair(d0, da + 2 * k, dw + 2 * k, idesc, k > 0 ? 1u : 0u);
            umma_commit_pair(&bars->empty[s], 0x3);
            umma_commit_pair(&bars->tfull[buf], 0x3);
          }
        }
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        umma_commit_pair(&bars->teardown, 0x1);
        mbar_wait(&bars->teardown, 0, drain);
      }
    } else if (warp == 2) {
      // -------------------------------------------------------- scale producer
      // One promotion-ring slot per K block: the K block's activation scales
      // of this CTA's rows (one bulk copy from the transposed table) and the
      // two weight-block scales (both CTAs hold both blocks' partials).
      uint32_t it = 0;
      int par = 0;
      bool stop = false;
      for (int tile = pair_id(); tile < ntiles && !stop; tile += pair_count()) {
        if (*abortp) break;
        const GemmTile td = get_tile(args, tile);
        if (!pair_tile_ok(args, td)) {
          if (lane == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
          continue;
        }
        const GemmTile sd = sub_tile(td, pair_rank());
        float *wA = wsc + par * (2 * G_KBMAX), *wB = wA + G_KBMAX;
        par ^= 1;
        {
          const float *swa = args.sw + static_cast<int64_t>(td.w_row0 / 128) * KB;
          const float *swb = args.sw + static_cast<int64_t>(td.w_row1 / 128) * KB;
          for (int i = lane; i < KB; i += 32) {
            wA[i] = __ldg(swa + i);
            wB[i] = __ldg(swb + i);
          }
          __syncwarp();
        }
        const float *sa = td.from1 ? args.sa1 : args.sa0;
        const int off = args.sa_transposed ? (sd.out_row & 3) : 0;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int slot = it % P_SSLOTS;
          if (!mbar_wait(&bars->sempty[slot], ((it / P_SSLOTS) & 1) ^ 1, ctl)) {
            stop = true;
            break;
          }
          float *rs = sring + slot * P_RING;
          if (args.sa_transposed) {
            if (lane == 0) {
              if (sd.n > 0) {
                mbar_arrive_expect_tx(&bars->sfull[slot], P_SA_SPAN * 4);
                bulk_load(rs, sa + static_cast<int64_t>(kb) * args.sa_ld + (sd.out_row - off), P_SA_SPAN * 4,
                          &bars->sfull[slot]);
              } else {
                mbar_arrive(&bars->sfull[slot]);  // no rows here: nothing to load
              }
            }
          } else {
            // row-major scales [rows, K/128] (plain GEMM): strided loads
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = lane + 32 * i;
              rs[j] = (j < sd.n) ? __ldg(sa + static_cast<int64_t>(sd.a_row + j) * KB + kb) : 0.0f;
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
    const int wg = (warp - 4) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    float *amx = amax_x;
    uint32_t it = 0;
    for (int tile = pair_id(); tile < ntiles; tile += pair_count()) {
      if (named_bar_or(1, 256, *abortp != 0)) break;
      const GemmTile td = get_tile(args, tile);
      if (!pair_tile_ok(args, td)) continue;
      const GemmTile sd = sub_tile(td, pair_rank());
      const int soff = args.sa_transposed ? (sd.out_row & 3) : 0;
      const bool live = q * 32 < sd.n;
      float acc0[64], acc1[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t buf = it & 1;
        const int slot = it % P_SSLOTS;
        const bool ok = mbar_wait2(&bars->tfull[buf], (it >> 1) & 1, &bars->sfull[slot], (it / P_SSLOTS) & 1, ctl);
        if (ok && live) {
          tc_fence_after();
          const float *rs = sring + slot * P_RING;
          const float sx = rs[r + soff];
          const float ca = sx * rs[132];
          const float cb = sx * rs[133];
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + wg * 64;
          uint32_t p[64];
          tmem_ld64(ta, p);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_scalar(acc0[j], acc0[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), ca);
          tmem_ld64(ta + 128, p);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_scalar(acc1[j], acc1[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), cb);
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          // to the even CTA, which issues the next MMAs into this buffer
          mbar_arrive_cluster(mapa_shared(smem_u32(&bars->tempty[buf]), 0));
          mbar_arrive(&bars->sempty[slot]);
        }
      }
      if (sd.n > 0) tile_epilogue<EPI, false>(args, sd, acc0, acc1, true, warp, lane, amx, outx, warp & 3);
    }
  }

  // neither CTA may leave (or free TMEM) while the other still works with
  // its shared memory, barriers or TMEM
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

namespace {
// Clusters of two that fit on the device at once (queried once per device).
template <int EPI>
std::atomic<int> *attr_done_clusters() {
  static std::atomic<int> n[64];
  return n;
}

template <typename Fn>
int64_t resident_pairs(Fn *fn, int smem, std::atomic<int> *cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_acquire);
    if (c > 0) return c;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(P_THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = moe_host::sm_count() / 2;
  }
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_release);
  return n;
}

template <int EPI>
cudaError_t launch_pair_epi(const CUtensorMap &mw, const CUtensorMap &m0, const CUtensorMap &m1, const GemmArgs &a,
                            int64_t max_tiles, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_pair_kernel<EPI>, P_SMEM, attr_done)) return e;
  // as many pairs as can be resident at once (persistent), fewer when there
  // are fewer tiles
  const int64_t pairs = resident_pairs(gemm_pair_kernel<EPI>, P_SMEM, attr_done_clusters<EPI>());
  if (pairs <= 0) return cudaErrorLaunchOutOfResources;
  const int64_t ncl = max_tiles < pairs ? max_tiles : pairs;
  gemm_pair_kernel<EPI><<<static_cast<unsigned>(2 * ncl), P_THREADS, P_SMEM, st>>>(mw, m0, m1, a);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_gemm_pair(const GemmLaunch &g, cudaStream_t st) {
  if (g.max_chunks <= 0 || g.nb <= 0) return cudaSuccess;
  if (g.chunk_rows != 256) return cudaErrorInvalidValue;
  // every tile must have two weight blocks (gate/up tiles always do)
  if (!g.gate_up && (g.rows_per_expert / 128) % 2 != 0) return cudaErrorInvalidValue;
  CUtensorMap mw, m0, m1;
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, K, g.w_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a0, K, g.a0_rows, K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a1, K, g.a1_rows,
                               g.a1_ld ? static_cast<uint64_t>(g.a1_ld) : K, 128, 128) != 0)
    return cudaErrorInvalidValue;
  const GemmArgs a = make_args(g);
  const int64_t max_tiles = static_cast<int64_t>(g.max_chunks) * g.nb;
  switch (g.epi) {
    case EPI_SWIGLU_Q: return launch_pair_epi<EPI_SWIGLU_Q>(mw, m0, m1, a, max_tiles, st);
    case EPI_GATE_F32: return launch_pair_epi<EPI_GATE_F32>(mw, m0, m1, a, max_tiles, st);
    default: return launch_pair_epi<EPI_BF16>(mw, m0, m1, a, max_tiles, st);
  }
}

}  // namespace moe
