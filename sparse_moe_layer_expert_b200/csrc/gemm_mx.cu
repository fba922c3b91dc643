// gemm_mx.cu -- grouped FP8 GEMM with power-of-two block scales applied by
// the tensor core (tcgen05.mma kind::mxf8f6f4.block_scale).
//
// The fine-grained scaling of "DeepSeek-V3 Technischer Bericht"
// (xyznot.com/de), Kernideen, FP8 bullet -- E4M3 operands, one scale per 1x128
// activation tile and per 128x128 weight block -- with the scales restricted
// to powers of two (pow2_scale in common.cuh; the pages' S = amax/448 is the
// default path in gemm.cu).  A power-of-two scale is an 8-bit exponent code,
// which the block-scaled MMA applies to each 32-long K slice of both operands
// itself, so the tile's partial sums never leave TMEM: one accumulator per
// tile gathers all K blocks and is read once, by the epilogue.  The exact
// result is the same sum of scaled 128-long partials sA * sW * P_kb as on the
// promotion path; here the tensor core scales each 32-long slice and adds
// the whole K range in FP32, so only the rounding of the additions differs.
//
//   * tiles, chunk table, bounds checks and epilogues as gemm.cu (shared in
//     gemm_tiles.cuh): <= 128 activation rows of one expert (M = 128) x a pair
//     of 128-row weight blocks (N = 256);
//   * 4-stage TMA ring; each stage also holds the K block's scale factors in
//     the layout tcgen05.cp expects: one 512-byte atom for the 128 activation
//     rows and one per 128-row weight block (byte (row % 32) * 16 +
//     (row / 32) * 4 + slice, the code repeated for the four 32-long slices
//     of the 128-long K block);
//   * warp 2 builds those atoms from the FP32 scale tables (the code is the
//     float's exponent byte); its loads run up to 7 K blocks ahead through a
//     small cp.async ring in shared memory (their latency under load is as
//     long as the operand loads', so a shallow look-ahead stalls the ring);
//   * warp 1's lane 0 copies the atoms into TMEM (tcgen05.cp 32x128b.warpx4;
//     two sets of 12 columns from column 256, alternate K blocks) and issues
//     the four block-scaled MMAs of the K block, slice k reading byte k;
//   * TMEM: accumulator columns 0..255 + the scale-factor columns; the
//     epilogue warps copy the accumulator to registers, hand TMEM back to the
//     tensor core (which starts the next tile) and then run the epilogue.
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

namespace {
constexpr int X_STAGES = 4;
constexpr int X_AB = 128 * 128;                 // activation tile: 128 rows x 128 bytes
constexpr int X_WB = 128 * 128;                 // one 128x128 weight tile
constexpr int X_SF = X_AB + 2 * X_WB;           // scale-factor atoms: A at +0, weight blocks at +512, +1024
constexpr int X_STAGE = X_SF + 2048;            // 50 KB: keeps every stage 1024-byte aligned
constexpr int X_THREADS = 384;
constexpr int X_AMAX = 2 * 128;
constexpr int X_OUTX = 8 * 32 * G_OPITCH;
constexpr int X_SR = 8;                         // K blocks of scales the builder keeps in flight
constexpr int X_SRING = 136;                    // floats per ring slot: 128 row scales, 2 block scales
constexpr int X_SMEM = 1024 + X_STAGES * X_STAGE + X_AMAX * 4 + X_OUTX * 4 + X_SR * X_SRING * 4 + 256;
static_assert(X_SMEM <= 232448, "shared memory budget");
static_assert(X_STAGE % 1024 == 0, "stage alignment");
// TMEM columns of the scale factors, two sets used by alternate K blocks (a
// copy into one set does not wait for MMAs still reading the other): A at
// +0, the two weight blocks at +4 and +8.
constexpr uint32_t X_TSF = 256;
constexpr uint32_t X_TSF_SET = 16;

struct XBars {
  uint64_t full[X_STAGES];   // TMA bytes + the scale-factor atoms
  uint64_t empty[X_STAGES];
  uint64_t acc_full;         // the tile's accumulator is complete
  uint64_t acc_empty;        // the epilogue has copied it out
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};

// K-major shared-memory descriptor without swizzle for a tcgen05.cp source:
// 16-byte rows, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (1ull << 46);
}

__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint32_t saddr) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sf_atom_desc(saddr))
               : "memory");
}

// Instruction descriptor of the block-scaled MMA: E4M3 x E4M3 -> FP32,
// K-major operands, 8-bit exponent scale factors, scale byte `slice` of A's
// and B's scale-factor words.
__device__ __forceinline__ uint32_t idesc_mx(uint32_t M, uint32_t N, uint32_t slice) {
  return (slice << 4) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) | (slice << 29);
}

__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// The 8-bit scale-factor code of a power-of-two scale, repeated in all four
// bytes of a word (one byte per 32-long slice of the 128-long K block).
__device__ __forceinline__ uint32_t sf_word(float S) { return ((__float_as_uint(S) >> 23) & 0xFFu) * 0x01010101u; }

// Next tile of this CTA's walk that passes the bounds check (all roles skip
// the same tiles), or ntiles.
__device__ __forceinline__ int next_valid_tile(const GemmArgs &a, int t, int ntiles) {
  while (t < ntiles && !tile_ok(a, get_tile(a, t))) t += gridDim.x;
  return t;
}
}  // namespace

template <int EPI>
__global__ void __launch_bounds__(X_THREADS, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_a0,
                   const __grid_constant__ CUtensorMap map_a1, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *amax_x = reinterpret_cast<float *>(smem + X_STAGES * X_STAGE);
  float *outx = amax_x + X_AMAX;
  float *sring = outx + X_OUTX;  // the scale-factor builder's load ring
  XBars *bars = reinterpret_cast<XBars *>(sring + X_SR * X_SRING);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < X_STAGES; ++i) {
      mbar_init(&bars->full[i], 2);  // the TMA's expect_tx arrival + the scale-factor atoms
      mbar_init(&bars->empty[i], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 8);
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

  // Register split as in gemm.cu: 56 for warps 0..3, 224 for the epilogue
  // warpgroups (128*56 + 256*224 = 384*168, the launch allocation).
  if (warp < 4) {
    setmaxnreg_dec<56>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0) {
        const uint64_t pol_w1 = policy_evict_first();  // one pass reads the weight tile
        const uint64_t pol_wk = policy_evict_normal(); // the expert's other chunks read it next
        const uint64_t pol_a = policy_evict_last();
        uint32_t it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const GemmTile td = get_tile(args, tile);
          if (!tile_ok(args, td)) continue;
          const CUtensorMap *amap = td.from1 ? &map_a1 : &map_a0;
          const bool two = td.w_row1 >= 0;
          const uint32_t bytes = X_AB + (two ? 2 : 1) * X_WB;
          const uint64_t pol_w = td.group > 1 ? pol_wk : pol_w1;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % X_STAGES;
            if (!mbar_wait(&bars->empty[s], ((it / X_STAGES) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * X_STAGE;
            mbar_arrive_expect_tx(&bars->full[s], bytes);
            const int x = kb * 128;
            tma_load_2d_hint(st, amap, &bars->full[s], x, td.a_row, pol_a);
            tma_load_2d_hint(st + X_AB, &map_w, &bars->full[s], x, td.w_row0, pol_w);
            if (two) tma_load_2d_hint(st + X_AB + X_WB, &map_w, &bars->full[s], x, td.w_row1, pol_w);
          }
        }
        // let copies still in flight land before the CTA can exit
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < X_STAGES ? it : X_STAGES;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->full[j % X_STAGES], (j / X_STAGES) & 1, drain);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0, tcount = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
          if (*abortp) break;
          const GemmTile td = get_tile(args, tile);
          if (!tile_ok(args, td)) continue;
          const bool two = td.w_row1 >= 0;
          const uint32_t N = two ? 256 : 128;
          // the epilogue has copied the previous tile's accumulator out
          if (!mbar_wait(&bars->acc_empty, (tcount & 1) ^ 1, ctl)) break;
          tc_fence_after();
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % X_STAGES;
            if (!mbar_wait(&bars->full[s], (it / X_STAGES) & 1, ctl)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(stages + s * X_STAGE);
            // scale factors of this K block into TMEM (ordered before the MMAs
            // that read them)
            const uint32_t t_sfa = tmem + X_TSF + (it & 1) * X_TSF_SET, t_sfb = t_sfa + 4;
            tmem_cp_atom(t_sfa, base + X_SF);
            tmem_cp_atom(t_sfb, base + X_SF + 512);
            if (two) tmem_cp_atom(t_sfb + 4, base + X_SF + 1024);
            const uint64_t da = sw128_kmajor_desc(base);
            const uint64_t dw = sw128_kmajor_desc(base + X_AB);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // slice k: +32 bytes along K (+2 in the descriptor's 16-byte
              // units); its scale factors are byte k of each TMEM word
              const uint32_t sel = static_cast<uint32_t>(k) << 30;
              umma_mx(tmem, da + 2 * k, dw + 2 * k, idesc_mx(128, N, k), (kb > 0 || k > 0) ? 1u : 0u,
                      t_sfa | sel, t_sfb | sel);
            }
            umma_commit(&bars->empty[s]);
          }
          if (stop) break;
          umma_commit(&bars->acc_full);
          ++tcount;
        }
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        umma_commit(&bars->teardown);
        mbar_wait(&bars->teardown, 0, drain);
      }
    } else if (warp == 2) {
      // ------------------------------------------------ scale-factor builder
      // Per K block: the activation atom from the transposed scale table
      // [K/128][sa_ld] (column = output row; the tile's 128 rows, padding rows
      // included, stay inside the table and its slack) and one atom per weight
      // block (its single scale in all 128 rows).  Lane l owns rows l, l+32,
      // l+64, l+96, i.e. the 16-byte group l of each atom.  The scales come
      // through a ring of X_SR slots filled by cp.async, one commit group per
      // K block, X_SR - 1 K blocks ahead of the atoms being written.
      struct Pos {
        int t, kb;
        GemmTile d;  // descriptor of tile t, read once per tile
      };
      auto seek = [&](Pos &p, int t) {  // first valid tile from t
        p.t = next_valid_tile(args, t, ntiles);
        p.kb = 0;
        if (p.t < ntiles) p.d = get_tile(args, p.t);
      };
      auto advance = [&](Pos &p) {
        if (++p.kb == KB) seek(p, p.t + gridDim.x);
      };
      auto issue = [&](const Pos &p, int slot) {
        float *dst = sring + slot * X_SRING;
        const float *col =
            (p.d.from1 ? args.sa1 : args.sa0) + static_cast<int64_t>(p.kb) * args.sa_ld + p.d.out_row;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async4(dst + lane + 32 * i, col + lane + 32 * i);
        if (lane == 0) {
          cp_async4(dst + 128, args.sw + static_cast<int64_t>(p.d.w_row0 >> 7) * KB + p.kb);
          if (p.d.w_row1 >= 0) cp_async4(dst + 129, args.sw + static_cast<int64_t>(p.d.w_row1 >> 7) * KB + p.kb);
        }
      };
      Pos p;  // the next K block to load
      seek(p, blockIdx.x);
      int loaded = 0;
      for (int j = 0; j < X_SR - 1; ++j) {
        if (p.t < ntiles) {
          issue(p, j);
          advance(p);
          ++loaded;
        }
        cp_async_commit();  // one group per K block (empty past the end)
      }
      for (int it = 0; it < loaded; ++it) {
        if (*abortp) break;
        if (p.t < ntiles) {
          issue(p, (it + X_SR - 1) % X_SR);  // the slot K block it - 1 has left
          advance(p);
          ++loaded;
        }
        cp_async_commit();
        cp_async_wait<X_SR - 1>();  // K block it's group has landed (this lane's part) ...
        __syncwarp();               // ... and every lane's
        const int s = it % X_STAGES;
        if (!mbar_wait(&bars->empty[s], ((it / X_STAGES) & 1) ^ 1, ctl)) break;
        const float *v = sring + (it % X_SR) * X_SRING;
        uint8_t *sf = stages + s * X_STAGE + X_SF;
        reinterpret_cast<uint4 *>(sf)[lane] =
            make_uint4(sf_word(v[lane]), sf_word(v[lane + 32]), sf_word(v[lane + 64]), sf_word(v[lane + 96]));
        const uint32_t wa = sf_word(v[128]), wb = sf_word(v[129]);
        reinterpret_cast<uint4 *>(sf + 512)[lane] = make_uint4(wa, wa, wa, wa);
        reinterpret_cast<uint4 *>(sf + 1024)[lane] = make_uint4(wb, wb, wb, wb);
        fence_proxy_async_smem();  // generic writes -> the tensor core's copy
        __syncwarp();              // (also: every lane has read slot it before it is refilled)
        if (lane == 0) mbar_arrive(&bars->full[s]);
      }
      cp_async_wait<0>();  // nothing may land in shared memory after the CTA ends
    }
  } else {
    setmaxnreg_inc<224>();
    // ---------------------------------------------------------- epilogue
    const int wg = (warp - 4) >> 2;
    const int q = warp & 3;
    float *amx = amax_x;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (named_bar_or(1, 256, *abortp != 0)) break;
      const GemmTile td = get_tile(args, tile);
      if (!tile_ok(args, td)) continue;
      const bool two = td.w_row1 >= 0;
      const bool live = q * 32 < td.n;  // a warp whose rows are all padding reads nothing
      float acc0[64], acc1[64];
      const bool ok = mbar_wait(&bars->acc_full, tcount & 1, ctl);
      if (ok && live) {
        tc_fence_after();
        const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + wg * 64;
        uint32_t p[64];
        tmem_ld64(ta, p);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 64; ++j) acc0[j] = __uint_as_float(p[j]);
        if (two) {
          tmem_ld64(ta + 128, p);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; ++j) acc1[j] = __uint_as_float(p[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) acc1[j] = 0.0f;
        }
        tc_fence_before();
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          acc0[j] = 0.0f;
          acc1[j] = 0.0f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);  // TMEM goes back to the tensor core
      ++tcount;
      tile_epilogue<EPI, true>(args, td, acc0, acc1, two, warp, lane, amx, outx, warp & 3);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int EPI>
static cudaError_t launch_mx(const CUtensorMap &mw, const CUtensorMap &m0, const CUtensorMap &m1,
                             const GemmArgs &a, int grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_mx_kernel<EPI>, X_SMEM, attr_done)) return e;
  gemm_mx_kernel<EPI><<<grid, X_THREADS, X_SMEM, st>>>(mw, m0, m1, a);
  return cudaGetLastError();
}

// Same work description as launch_gemm; the scales must be powers of two and
// the activation scales stored transposed (the layer's tables).
cudaError_t launch_gemm_mx(const GemmLaunch &g, cudaStream_t st) {
  if (g.max_chunks <= 0 || g.nb <= 0) return cudaSuccess;
  if (!g.sa_transposed || !g.chunks || (g.epi != EPI_SWIGLU_Q && g.epi != EPI_GATE_F32))
    return cudaErrorInvalidValue;
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
  const int sms = moe_host::sm_count();
  const int64_t max_tiles = static_cast<int64_t>(g.max_chunks) * g.nb;
  const int grid = static_cast<int>(max_tiles < sms ? max_tiles : sms);
  return g.epi == EPI_SWIGLU_Q ? launch_mx<EPI_SWIGLU_Q>(mw, m0, m1, a, grid, st)
                               : launch_mx<EPI_GATE_F32>(mw, m0, m1, a, grid, st);
}

}  // namespace moe
