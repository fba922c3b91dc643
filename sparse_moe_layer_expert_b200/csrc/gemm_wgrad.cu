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
// two-multiplier FMAs).  A tile has only as many K blocks as its expert has
// 128-token tiles (one or two at prefill) but writes 128 x 256 FP32 outputs,
// so the output stream sets the pace: the promotion threads put each 128 x
// 128 block into shared memory as four 32-column boxes (128-byte swizzle) in
// a ring of box slots, and one of them hands each box to a TMA store; the
// stores drain to HBM while the next tile's K blocks are computed.  (The
// ring holds one block next to three operand stages; fewer operand stages
// for a deeper ring measured slower.)  Every wait is bounded.
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

namespace {
constexpr int W_STAGES = 3;
constexpr int W_AB = 128 * 128;
constexpr int W_BB = 128 * 128;
constexpr int W_STAGE = W_AB + 2 * W_BB;
constexpr int W_THREADS = 384;
constexpr int W_SSLOTS = 6;
constexpr int W_RING = 128 + 256;  // floats per slot: row scales, then column scales
constexpr int W_OBOX = 128 * 128;                // one 32-column FP32 box of 128 rows (bytes)
constexpr int W_OSLOTS = 4;                       // box slots of the output ring (one 128 x 128 block)
constexpr int W_OUT = W_OSLOTS * W_OBOX;
constexpr int W_SMEM = 1024 + W_STAGES * W_STAGE + W_OUT + W_SSLOTS * W_RING * 4 + 256;
static_assert(W_SMEM <= 232448, "shared memory budget");

struct WgArgs {
  int E, MB, NB;             // experts, 128-row blocks of C_out, 256-column pairs of C_in
  int C_out, C_in;
  int P_blocks;              // K blocks of the operand tables (bounds every segment)
  const int32_t *seg;        // [E + 1] padded token segments (multiples of 128)
  const float *sA_t;         // [P/128][C_out]
  const float *sB_t;         // [P/128][C_in]
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

// One 128 x 128 FP32 output block (this thread: row r, columns 64 wg .. +63
// of the block, in acc) through shared memory to TMA stores: four boxes of
// 32 columns x 128 rows (box k of the block in ring slot (nbox + k) %
// W_OSLOTS), each row's 128 bytes in 16-byte chunks swizzled by the row
// (chunk j at j ^ (r & 7)), as the tensor map's 128-byte swizzle expects; one
// bulk group per box.  Before four slots are rewritten the issuing thread
// waits until at most W_OSLOTS - 4 of its groups are still reading (the boxes
// that last used those slots are done); all 256 promotion threads meet at
// named barrier 2.
__device__ __forceinline__ void store_block(const float (&acc)[64], uint8_t *ostage, const CUtensorMap *map,
                                            int col0, int row0, int wg, int r, bool issuer, uint32_t &nbox) {
  static_assert(W_OSLOTS >= 4 && W_OSLOTS <= 7, "ring of 4..7 box slots");
  if (issuer) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(W_OSLOTS - 4) : "memory");
  named_bar_sync(2, 256);
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint8_t *box = ostage + ((nbox + wg * 2 + b) % W_OSLOTS) * W_OBOX + r * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = b * 32 + j * 4;
      *reinterpret_cast<float4 *>(box + ((j ^ (r & 7)) << 4)) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
    }
  }
  fence_proxy_async_smem();
  named_bar_sync(2, 256);
  if (issuer) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      tma_store_2d(map, ostage + ((nbox + b) % W_OSLOTS) * W_OBOX, col0 + 32 * b, row0);
      bulk_commit();
    }
  }
  nbox += 4;
}

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
                      const __grid_constant__ CUtensorMap map_out, const WgArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *ostage = smem + W_STAGES * W_STAGE;  // 1024-aligned: the boxes use the 128-byte swizzle
  float *sring = reinterpret_cast<float *>(ostage + W_OUT);
  WgBars *bars = reinterpret_cast<WgBars *>(sring + W_SSLOTS * W_RING);

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
    uint32_t it = 0, nbox = 0;
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
      // the tile's output: block A (columns nb*256 ..), then block B (+128)
      const int orow = td.e * args.C_out + td.mb * 128;
      store_block(acc0, ostage, &map_out, td.nb * 256, orow, wg, r, warp == 4 && lane == 0, nbox);
      if (td.two) store_block(acc1, ostage, &map_out, td.nb * 256 + 128, orow, wg, r, warp == 4 && lane == 0, nbox);
    }
    // the shared-memory source of the last stores stays valid until they are done
    if (warp == 4 && lane == 0) bulk_wait_all();
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
  CUtensorMap mo;  // the FP32 output [E * C_out, C_in], 32-column x 128-row boxes
  if (moe_host::encode_tmap_2d(&mo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.out, g.C_in,
                               static_cast<uint64_t>(g.E) * g.C_out, g.C_in * 4, 32, 128) != 0)
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
  a.err = g.err;
  a.limit_ns = g.wait_limit_ns;
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_wgrad_kernel, W_SMEM, attr_done)) return e;
  const int sms = moe_host::sm_count();
  const int grid = static_cast<int>(ntiles < sms ? ntiles : sms);
  gemm_wgrad_kernel<<<grid, W_THREADS, W_SMEM, st>>>(ma, mb, mo, a);
  return cudaGetLastError();
}

}  // namespace moe
