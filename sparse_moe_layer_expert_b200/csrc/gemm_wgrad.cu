// gemm_wgrad.cu -- weight gradients of the expert FFNs: a grouped FP8 GEMM
// that contracts over each expert's tokens.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Kernideen, FP8 bullet:
// E4M3 for all tensors with FP32 promotion every 128 accumulation steps.  For
// the weight gradient dW_e = Grad_e^T Act_e of expert e (dW2 = dY^T h,
// dW13 = [dG|dU]^T x) the contraction runs over the expert's tokens, so both
// operands carry 128x1 tiles along tokens (one scale per channel per 128
// tokens; the technical report's reading, as the backward oracle): the
// promoted partial of K block kb is sA[m, kb] * sB[n, kb] * P_kb[m, n] -- a
// scale per output row AND per output column, unlike the forward's per-row
// times per-block scalar.
//
// Operands (written by colquant_kernel, backward.cu): Grad^T [C_out, P] and
// Act^T [C_in, P] E4M3, K-major (tokens contiguous), each expert's tokens a
// segment [seg[e], seg[e+1]) padded to a multiple of 128 with zero codes;
// scales transposed [P/128][C_out] and [P/128][C_in].
//
// Tile = (expert e, 128 output rows, 2 x 128 output columns), the K loop over
// the expert's segment only (an unused expert's tile has no K block and
// writes zeros).  The pipeline is gemm.cu's: 4-stage TMA ring, one thread
// issuing tcgen05.mma kind::f8f6f4 (M = 128, N = 256, K = 32) into one of two
// TMEM partials per K block, two promotion warpgroups folding the partial into
// FP32 registers, here with a per-column multiplier sB[n] * sA[m] (packed
// two-multiplier FMAs), and FP32 stores of the tile.  Every wait is bounded.
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

namespace {
constexpr int W_STAGES = 4;
constexpr int W_AB = 128 * 128;
constexpr int W_BB = 128 * 128;
constexpr int W_STAGE = W_AB + 2 * W_BB;
constexpr int W_THREADS = 384;
constexpr int W_SSLOTS = 6;
constexpr int W_RING = 128 + 256;  // floats per slot: row scales, then column scales
constexpr int W_OUTX = 8 * 32 * G_OPITCH;
constexpr int W_SMEM = 1024 + W_STAGES * W_STAGE + W_SSLOTS * W_RING * 4 + W_OUTX * 4 + 256;
static_assert(W_SMEM <= 232448, "shared memory budget");

struct WgArgs {
  int E, MB, NB;             // experts, 128-row blocks of C_out, 256-column pairs of C_in
  int C_out, C_in;
  int P_blocks;              // K blocks of the operand tables (bounds every segment)
  const int32_t *seg;        // [E + 1] padded token segments (multiples of 128)
  const float *sA_t;         // [P/128][C_out]
  const float *sB_t;         // [P/128][C_in]
  GemmArgs epi;              // output (FP32 [E * C_out, C_in]) for the shared epilogue
  int32_t *err;
  uint64_t limit_ns;
};

struct WgBars {
  uint64_t full[W_STAGES];
  uint64_t empty[W_STAGES];
  uint64_t sfull[W_SSLOTS];
  uint64_t sempty[W_SSLOTS];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};

struct WgTile {
  int e, mb, nb, kb0, nkb;
  bool two;
};

__device__ __forceinline__ WgTile wg_tile(const WgArgs &a, int t) {
  WgTile d;
  const int per = a.MB * a.NB;
  d.e = t / per;
  const int rem = t - d.e * per;
  d.mb = rem / a.NB;
  d.nb = rem - d.mb * a.NB;
  const int s0 = a.seg[d.e], s1 = a.seg[d.e + 1];
  d.kb0 = s0 >> 7;
  d.nkb = (s1 - s0) >> 7;
  // a malformed segment computes nothing (the tile writes zeros)
  if (d.nkb < 0 || (s0 & 127) || (s1 & 127) || s0 < 0 || d.kb0 + d.nkb > a.P_blocks) d.nkb = 0;
  d.two = d.nb * 256 + 128 < a.C_in;
  return d;
}
}  // namespace

__global__ void __launch_bounds__(W_THREADS, 1)
    gemm_wgrad_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const WgArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *sring = reinterpret_cast<float *>(smem + W_STAGES * W_STAGE);
  float *outx = sring + W_SSLOTS * W_RING;
  WgBars *bars = reinterpret_cast<WgBars *>(outx + W_OUTX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < W_STAGES; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < W_SSLOTS; ++i) {
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
    tma_prefetch_map(&map_a);
    tma_prefetch_map(&map_b);
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
  const int ntiles = args.E * args.MB * args.NB;

  if (warp < 4) {
    setmaxnreg_dec<72>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint64_t pol = policy_evict_first();
        uint32_t it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const WgTile td = wg_tile(args, tile);
          const uint32_t bytes = W_AB + (td.two ? 2 : 1) * W_BB;
          for (int i = 0; i < td.nkb; ++i, ++it) {
            const int s = it % W_STAGES;
            if (!mbar_wait(&bars->empty[s], ((it / W_STAGES) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * W_STAGE;
            mbar_arrive_expect_tx(&bars->full[s], bytes);
            const int x = (td.kb0 + i) * 128;
            tma_load_2d_hint(st, &map_a, &bars->full[s], x, td.mb * 128, pol);
            tma_load_2d_hint(st + W_AB, &map_b, &bars->full[s], x, td.nb * 256, pol);
            if (td.two) tma_load_2d_hint(st + W_AB + W_BB, &map_b, &bars->full[s], x, td.nb * 256 + 128, pol);
          }
        }
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < W_STAGES ? it : W_STAGES;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->full[j % W_STAGES], (j / W_STAGES) & 1, drain);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const WgTile td = wg_tile(args, tile);
          const uint32_t idesc = idesc_e4m3_f32(128, td.two ? 256 : 128);
          for (int i = 0; i < td.nkb; ++i, ++it) {
            const int s = it % W_STAGES;
            const uint32_t buf = it & 1;
            if (!mbar_wait2(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, &bars->full[s], (it / W_STAGES) & 1, ctl)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(stages + s * W_STAGE);
            const uint64_t da = sw128_kmajor_desc(base);
            const uint64_t db = sw128_kmajor_desc(base + W_AB);
            const uint32_t d0 = tmem + buf * 256;
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f8(d0, da + 2 * k, db + 2 * k, idesc, k > 0 ? 1u : 0u);
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
      // Per K block: the tile's 128 row scales and 256 (or 128) column scales,
      // two bulk copies from the transposed tables.
      uint32_t it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
        if (*abortp) break;
        const WgTile td = wg_tile(args, tile);
        const uint32_t nb_bytes = (td.two ? 256 : 128) * 4;
        for (int i = 0; i < td.nkb; ++i, ++it) {
          const int slot = it % W_SSLOTS;
          if (!mbar_wait(&bars->sempty[slot], ((it / W_SSLOTS) & 1) ^ 1, ctl)) {
            stop = true;
            break;
          }
          if (lane == 0) {
            float *rs = sring + slot * W_RING;
            const int64_t kb = td.kb0 + i;
            mbar_arrive_expect_tx(&bars->sfull[slot], 128 * 4 + nb_bytes);
            bulk_load(rs, args.sA_t + kb * args.C_out + td.mb * 128, 128 * 4, &bars->sfull[slot]);
            bulk_load(rs + 128, args.sB_t + kb * args.C_in + td.nb * 256, nb_bytes, &bars->sfull[slot]);
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
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (named_bar_or(1, 256, *abortp != 0)) break;
      const WgTile td = wg_tile(args, tile);
      float acc0[64], acc1[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      for (int i = 0; i < td.nkb; ++i, ++it) {
        const uint32_t buf = it & 1;
        const int slot = it % W_SSLOTS;
        const bool ok = mbar_wait2(&bars->tfull[buf], (it >> 1) & 1, &bars->sfull[slot], (it / W_SSLOTS) & 1, ctl);
        if (ok) {
          tc_fence_after();
          const float *rs = sring + slot * W_RING;
          const float sa = rs[r];
          const float *sb = rs + 128 + wg * 64;  // this thread's 64 columns of block A (block B at +128)
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + wg * 64;
          uint32_t p[64];
          tmem_ld64(ta, p);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_vec(acc0[j], acc0[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), sa * sb[j],
                      sa * sb[j + 1]);
          if (td.two) {
            tmem_ld64(ta + 128, p);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 64; j += 2)
              ffma2_vec(acc1[j], acc1[j + 1], __uint_as_float(p[j]), __uint_as_float(p[j + 1]), sa * sb[128 + j],
                        sa * sb[128 + j + 1]);
          }
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->tempty[buf]);
          mbar_arrive(&bars->sempty[slot]);
        }
      }
      GemmTile ot;
      ot.w_row0 = 0;
      ot.w_row1 = td.two ? 128 : -1;
      ot.a_row = 0;
      ot.n = 128;
      ot.out_row = td.e * args.C_out + td.mb * 128;
      ot.out_col = td.nb * 256;
      ot.from1 = 0;
      ot.group = 1;
      tile_epilogue<EPI_F32, false>(args.epi, ot, acc0, acc1, td.two, warp, lane, nullptr, outx);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

cudaError_t launch_gemm_wgrad(const WgradLaunch &g, cudaStream_t st) {
  const int MB = static_cast<int>(g.C_out / 128), NB = static_cast<int>((g.C_in / 128 + 1) / 2);
  const int64_t ntiles = static_cast<int64_t>(g.E) * MB * NB;
  if (ntiles == 0) return cudaSuccess;
  if (ntiles > INT32_MAX) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (moe_host::encode_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a_t, g.P, g.C_out, g.P, 128, 128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b_t, g.P, g.C_in, g.P, 128, 128) != 0)
    return cudaErrorInvalidValue;
  WgArgs a{};
  a.E = g.E;
  a.MB = MB;
  a.NB = NB;
  a.C_out = static_cast<int>(g.C_out);
  a.C_in = static_cast<int>(g.C_in);
  a.P_blocks = static_cast<int>(g.P / 128);
  a.seg = g.seg;
  a.sA_t = g.sa_t;
  a.sB_t = g.sb_t;
  a.epi = GemmArgs{};
  a.epi.out = g.out;
  a.epi.ldo = g.C_in;
  a.epi.gate_up = 0;
  a.err = g.err;
  a.limit_ns = g.wait_limit_ns;
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_wgrad_kernel, W_SMEM, attr_done)) return e;
  const int sms = moe_host::sm_count();
  const int grid = static_cast<int>(ntiles < sms ? ntiles : sms);
  gemm_wgrad_kernel<<<grid, W_THREADS, W_SMEM, st>>>(ma, mb, a);
  return cudaGetLastError();
}

}  // namespace moe
