// gemm_tall.cu -- the grouped, fine-grained block-scaled FP8 GEMM on tall
// tiles: up to 256 rows of one expert per pass over a weight tile.
//
// Same arithmetic as gemm.cu ("DeepSeek-V3 Technischer Bericht",
// xyznot.com/de, Kernideen, FP8 bullet: E4M3 operands, 1x128 activation
// scales, 128x128 weight-block scales, each 128-long partial promoted into
// FP32 with its two scales).  What changes is the tile's shape:
//
//   * tile = up to 256 activation rows (one expert's chunk) x 128 weight rows:
//     for the gate/up projection the 64 gate rows and the 64 up rows of one
//     half of a 128-channel block, for the down projection 128 output
//     channels.  Where gemm.cu cuts an expert at 128 rows and streams its
//     weights once per cut, a chunk here holds up to 256 rows: an expert of
//     129..256 rows reads each weight tile once;
//   * two CTAs form a cluster and take the two halves of the same (chunk,
//     block): the two 64-channel halves of a 128-channel block of h, whose
//     1x128 requantization needs the amax over both halves (exchanged through
//     distributed shared memory once per tile), or two adjacent 128-channel
//     blocks of the down projection;
//   * per 128-K block the stage holds the chunk's rows (32-row TMA boxes, as
//     many as the chunk has: the bytes loaded follow the rows present) and
//     the 128 weight rows (two 64-row boxes); one thread issues four
//     tcgen05.mma (M = 128, N = 128, K = 32) for rows 0..127 and, when the
//     chunk has more than 128 rows, four more for rows 128..255, into a TMEM
//     partial that starts from zero for every K block;
//   * promotion warpgroup g owns rows 128 g .. 128 g + 127: each thread one
//     row, 64 columns of each of the two 64-wide halves of the partial
//     (gate | up, or the two 64-channel halves of a down block), folded into
//     FP32 registers with sA[row, kb] * sW[block, kb]; a warp whose rows are
//     all beyond the chunk skips its reads;
//   * TMEM holds two partial buffers of 256 columns (rows 0..127 in columns
//     0..127, rows 128..255 in 128..255), so the tensor core fills one while
//     the promotion threads drain the other.
//
// Epilogues (one row per thread):
//   EPI_SWIGLU_Q  h = silu(G) U in FP32 for the thread's 64 channels; the
//                 row's amax over them goes to the other CTA of the cluster
//                 (and its amax comes back): S = amax over the 128 channels
//                 / 448, E4M3 RNE codes (64 per thread, 16-byte stores) ->
//                 hq; the even CTA writes the scale -> hs
//   EPI_GATE_F32  y = acc * gate[row] in FP32 (down projection)
//   EPI_F32       C = acc in FP32
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warp 2 scale producer, warp 3 idle, warps 4..11 promotion +
// epilogue.  Every wait is bounded (common.cuh).
#include "common.cuh"
#include "gemm_tiles.cuh"
#include "kernels.h"

namespace moe {

using namespace gemm_detail;

namespace {
constexpr int T_STAGES = 4;
constexpr int T_SSLOTS = 6;
constexpr int T_AB = 256 * 128;           // up to 256 activation rows x 128 bytes
constexpr int T_ABOX = 32 * 128;          // one 32-row activation box
constexpr int T_WB = 128 * 128;           // 128 weight rows (two 64-row boxes)
constexpr int T_WBOX = 64 * 128;          // one 64-row weight box
constexpr int T_STAGE = T_AB + T_WB;      // 48 KB
constexpr int T_THREADS = 384;
// Scale slot (floats): [0, 260) activation scales of the tile's rows from row
// offset out_row & 3 (a bulk copy starts on a 16-byte boundary); [260] and
// [261] the weight-block scales of the two 64-wide halves.
constexpr int T_RING = 264;
constexpr int T_SA_SPAN = 260;
constexpr int T_XAMAX = 2 * 256;          // floats: the other CTA's row amax, by tile parity
constexpr int T_WSC = 2 * 2 * G_KBMAX;    // floats: weight-scale rows of 2 tiles x 2 halves
constexpr int T_OUTX = 8 * 32 * G_OPITCH; // floats: one 32-row x 16-float buffer per promotion warp
constexpr int T_BARS = 256;
constexpr int T_SMEM =
    1024 + T_STAGES * T_STAGE + T_SSLOTS * T_RING * 4 + T_XAMAX * 4 + T_WSC * 4 + T_OUTX * 4 + T_BARS;
static_assert(T_SMEM <= 232448, "shared memory budget");
static_assert(T_SA_SPAN <= kScaleSlack, "the scale tables' slack covers one slot's copy past the last row");

struct TallBars {
  uint64_t full[T_STAGES];
  uint64_t empty[T_STAGES];
  uint64_t sfull[T_SSLOTS];
  uint64_t sempty[T_SSLOTS];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t xfull[2];   // the other CTA's row amax of a tile has arrived (256 arrivals)
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(TallBars) <= T_BARS, "barrier block");

// One half (cluster rank `half`) of pair tile p = (chunk p / nb, block j = p % nb).
struct TallTile {
  int32_t w_row0, w_row1;  // the two 64-row weight boxes
  int32_t a_row, n, out_row, out_col, from1;
  int32_t sw_row0, sw_row1;  // weight-scale rows of the two halves
  int32_t blk;             // gate/up: the 128-channel block j (row of the h scale table)
  int32_t group;           // chunks of the expert
};

// (pair tiles of an expert's chunks run block by block, as in gemm_tiles.cuh)
__device__ __forceinline__ TallTile tall_tile(const GemmArgs &a, int p, int half) {
  int c, j;
  int4 ch = make_int4(0, 0, 0, 0);
  tile_coords(a, p, c, j, ch);
  TallTile d;
  int e;
  if (a.chunks) {
    e = chunk_expert(ch);
    d.from1 = chunk_from1(ch);
    d.a_row = ch.y;
    d.out_row = ch.z;
    d.n = chunk_rows_of(ch);
    d.group = chunk_group(ch);
  } else {
    e = 0;
    d.from1 = 0;
    d.a_row = c * a.chunk_rows;
    const int64_t rem = a.dense_M - static_cast<int64_t>(c) * a.chunk_rows;
    d.n = rem < a.chunk_rows ? static_cast<int32_t>(rem) : a.chunk_rows;
    d.out_row = d.a_row;
    d.group = 1;
  }
  if (a.a_is_out_row) {
    d.a_row = d.out_row;
    d.from1 = 0;
  }
  const int64_t base = static_cast<int64_t>(e) * a.rows_per_expert;
  if (a.gate_up) {
    // gate rows and up rows of channels j*128 + half*64 .. +63
    d.w_row0 = static_cast<int32_t>(base + j * 128 + half * 64);
    d.w_row1 = static_cast<int32_t>(base + a.half + j * 128 + half * 64);
    d.sw_row0 = static_cast<int32_t>((base + j * 128) / 128);
    d.sw_row1 = static_cast<int32_t>((base + a.half + j * 128) / 128);
    d.out_col = j * 128 + half * 64;
  } else {
    // output channels j*256 + half*128 .. +127: one 128-row weight block
    d.w_row0 = static_cast<int32_t>(base + j * 256 + half * 128);
    d.w_row1 = d.w_row0 + 64;
    d.sw_row0 = d.w_row0 / 128;
    d.sw_row1 = d.sw_row0;
    d.out_col = j * 256 + half * 128;
  }
  d.blk = j;
  return d;
}

// Bounds of a tile, checked for the odd half (whose rows and columns are the
// larger ones) so that both CTAs of a cluster take the same decision.
__device__ __forceinline__ bool tall_ok(const GemmArgs &a, int p) {
  const TallTile d = tall_tile(a, p, 1);
  const int64_t arows = d.from1 ? a.a_rows1 : a.a_rows0;
  const int ncols = a.gate_up ? 64 : 128;  // output columns of one half
  return d.n >= 1 && d.n <= 256 && d.a_row >= 0 && d.a_row + d.n <= arows && d.out_row >= 0 &&
         d.out_row + d.n <= a.out_rows && d.w_row0 >= 64 && d.w_row0 + 64 <= a.w_rows &&
         d.w_row1 + 64 <= a.w_rows && d.out_col >= ncols && d.out_col + ncols <= a.out_cols &&
         d.out_row + d.n <= a.sa_ld && a.sa_transposed && a.KB <= G_KBMAX &&
         (a.gate_up ? (a.out_scale != nullptr) : true);
}

// Distributed-shared-memory exchange of the SwiGLU row amax (once per tile).
__device__ __forceinline__ void st_cluster_f32(uint32_t caddr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr), "f"(v) : "memory");
}
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_acq_cluster(uint64_t *bar, uint32_t parity, const WaitCtl &ctl) {
  if (mbar_try_wait_acq_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if (*ctl.abort) return false;
    if (global_timer_ns() - t0 > ctl.limit_ns) {
      *ctl.abort = 1;
      if (ctl.err) atomicOr(ctl.err, MOE_DEVERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ int tall_half() { return static_cast<int>(cluster_ctarank()); }
__device__ __forceinline__ int tall_cluster() { return static_cast<int>(blockIdx.x >> 1); }
__device__ __forceinline__ int tall_clusters() { return static_cast<int>(gridDim.x >> 1); }
}  // namespace

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(T_THREADS, 1)
    gemm_tall_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_a0,
                     const __grid_constant__ CUtensorMap map_a1, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *sring = reinterpret_cast<float *>(smem + T_STAGES * T_STAGE);
  float *xamax = sring + T_SSLOTS * T_RING;
  float *wsc = xamax + T_XAMAX;
  float *outx = wsc + T_WSC;
  TallBars *bars = reinterpret_cast<TallBars *>(outx + T_OUTX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < T_STAGES; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < T_SSLOTS; ++i) {
      mbar_init(&bars->sfull[i], 2);  // the bulk copy's expect_tx arrival + the weight scales
      mbar_init(&bars->sempty[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->tfull[i], 1);
      mbar_init(&bars->tempty[i], 8);
      mbar_init(&bars->xfull[i], 256);
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
  // the other CTA's amax arrivals may target this CTA's barriers only once
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
  const int npairs = nchunks * args.nb;
  const int KB = args.KB;

  // Register split as in gemm.cu: warps 0..3 keep 72 registers, the two
  // promotion warpgroups get 216 (128*72 + 256*216 = 384*168).
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
        for (int p = tall_cluster(); p < npairs && !stop; p += tall_clusters()) {
          if (*abortp) break;
          if (!tall_ok(args, p)) continue;
          const TallTile td = tall_tile(args, p, tall_half());
          const CUtensorMap *amap = td.from1 ? &map_a1 : &map_a0;
          const int nbox = (td.n + 31) / 32;
          const uint32_t bytes = T_WB + nbox * T_ABOX;
          const uint64_t pol_w = td.group > 1 ? pol_wk : pol_w1;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % T_STAGES;
            if (!mbar_wait(&bars->empty[s], ((it / T_STAGES) & 1) ^ 1, ctl)) {
              stop = true;
              break;
            }
            uint8_t *st = stages + s * T_STAGE;
            mbar_arrive_expect_tx(&bars->full[s], bytes);
            const int x = kb * 128;
            tma_load_2d_hint(st + T_AB, &map_w, &bars->full[s], x, td.w_row0, pol_w);
            tma_load_2d_hint(st + T_AB + T_WBOX, &map_w, &bars->full[s], x, td.w_row1, pol_w);
            for (int b = 0; b < nbox; ++b)
              tma_load_2d_hint(st + b * T_ABOX, amap, &bars->full[s], x, td.a_row + 32 * b, pol_a);
          }
        }
        // let copies still in flight land before the CTA can exit
        int quiet = 0;
        const WaitCtl drain{&quiet, nullptr, 100000000ull};
        const uint32_t n_inflight = it < T_STAGES ? it : T_STAGES;
        for (uint32_t j = it - n_inflight; j < it; ++j)
          mbar_wait(&bars->full[j % T_STAGES], (j / T_STAGES) & 1, drain);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0;
        bool stop = false;
        const uint32_t idesc = idesc_e4m3_f32(128, 128);
        for (int p = tall_cluster(); p < npairs && !stop; p += tall_clusters()) {
          if (*abortp) break;
          if (!tall_ok(args, p)) continue;
          const TallTile td = tall_tile(args, p, tall_half());
          const bool lower = td.n > 128;  // rows 128..255 present
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % T_STAGES;
            const uint32_t buf = it & 1;
            if (!mbar_wait2(&bars->tempty[buf], ((it >> 1) & 1) ^ 1, &bars->full[s], (it / T_STAGES) & 1, ctl)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(stages + s * T_STAGE);
            const uint64_t da0 = sw128_kmajor_desc(base);
            const uint64_t dw = sw128_kmajor_desc(base + T_AB);
            const uint32_t d0 = tmem + buf * 256;
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_f8(d0, da0 + 2 * k, dw + 2 * k, idesc, k > 0 ? 1u : 0u);
            if (lower) {
              // rows 128..255 start 16 KB (sixteen 8-row swizzle atoms) into the stage
              const uint64_t da1 = sw128_kmajor_desc(base + 128 * 128);
#pragma unroll
              for (int k = 0; k < 4; ++k) umma_f8(d0 + 128, da1 + 2 * k, dw + 2 * k, idesc, k > 0 ? 1u : 0u);
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
      // One promotion-ring slot per K block: the K block's activation scales
      // of the tile's rows (one bulk copy from the transposed table) and the
      // weight-block scales of the two halves (staged once per tile).
      uint32_t it = 0;
      int par = 0;
      bool stop = false;
      for (int p = tall_cluster(); p < npairs && !stop; p += tall_clusters()) {
        if (*abortp) break;
        if (!tall_ok(args, p)) {
          if (lane == 0 && args.err) atomicOr(args.err, MOE_DEVERR_BAD_INDEX);
          continue;
        }
        const TallTile td = tall_tile(args, p, tall_half());
        float *wA = wsc + par * (2 * G_KBMAX), *wB = wA + G_KBMAX;
        par ^= 1;
        {
          const float *swa = args.sw + static_cast<int64_t>(td.sw_row0) * KB;
          const float *swb = args.sw + static_cast<int64_t>(td.sw_row1) * KB;
          for (int i = lane; i < KB; i += 32) {
            wA[i] = __ldg(swa + i);
            wB[i] = __ldg(swb + i);
          }
          __syncwarp();
        }
        const float *sa = td.from1 ? args.sa1 : args.sa0;
        const int off = td.out_row & 3;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int slot = it % T_SSLOTS;
          if (!mbar_wait(&bars->sempty[slot], ((it / T_SSLOTS) & 1) ^ 1, ctl)) {
            stop = true;
            break;
          }
          float *rs = sring + slot * T_RING;
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars->sfull[slot], T_SA_SPAN * 4);
            bulk_load(rs, sa + static_cast<int64_t>(kb) * args.sa_ld + (td.out_row - off), T_SA_SPAN * 4,
                      &bars->sfull[slot]);
            rs[260] = wA[kb];
            rs[261] = wB[kb];
            mbar_arrive(&bars->sfull[slot]);
          }
        }
      }
    }
  } else {
    setmaxnreg_inc<216>();
    // ------------------------------------------------- promotion + epilogue
    const int g = (warp - 4) >> 2;     // rows 128 g .. 128 g + 127
    const int q = warp & 3;            // TMEM lane quarter
    const int r = g * 128 + q * 32 + lane;
    uint32_t it = 0, ntile = 0;
    for (int p = tall_cluster(); p < npairs; p += tall_clusters()) {
      if (named_bar_or(1, 256, *abortp != 0)) break;
      if (!tall_ok(args, p)) continue;
      const TallTile td = tall_tile(args, p, tall_half());
      const int soff = td.out_row & 3;
      const bool live = g * 128 + q * 32 < td.n;
      float acc0[64], acc1[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        acc0[j] = 0.0f;
        acc1[j] = 0.0f;
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t buf = it & 1;
        const int slot = it % T_SSLOTS;
        const bool ok = mbar_wait2(&bars->tfull[buf], (it >> 1) & 1, &bars->sfull[slot], (it / T_SSLOTS) & 1, ctl);
        if (ok && live) {
          tc_fence_after();
          const float *rs = sring + slot * T_RING;
          const float sx = rs[r + soff];
          const float ca = sx * rs[260];
          const float cb = sx * rs[261];
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + g * 128;
          uint32_t pr[64];
          tmem_ld64(ta, pr);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_scalar(acc0[j], acc0[j + 1], __uint_as_float(pr[j]), __uint_as_float(pr[j + 1]), ca);
          tmem_ld64(ta + 64, pr);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 64; j += 2)
            ffma2_scalar(acc1[j], acc1[j + 1], __uint_as_float(pr[j]), __uint_as_float(pr[j + 1]), cb);
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
      if constexpr (EPI == EPI_SWIGLU_Q) {
        // h = silu(G) * U for this row's 64 channels (fast exp and divide:
        // a few ulp, far inside the layer's tolerance)
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float gv = acc0[j];
          acc0[j] = __fdividef(gv, 1.0f + __expf(-gv)) * acc1[j];
          amax = fmaxf(amax, fabsf(acc0[j]));
        }
        // the row's amax over the other 64 channels of the 128-channel
        // tile lives in the other CTA: each thread hands its amax over and
        // takes the other's (double-buffered by tile parity)
        const int tp = static_cast<int>(ntile & 1);
        const uint32_t other = static_cast<uint32_t>(tall_half() ^ 1);
        st_cluster_f32(mapa_shared(smem_u32(xamax + tp * 256 + r), other), valid ? amax : 0.0f);
        mbar_arrive_release_cluster(mapa_shared(smem_u32(&bars->xfull[tp]), other));
        if (mbar_wait_acq_cluster(&bars->xfull[tp], (ntile >> 1) & 1, ctl)) amax = fmaxf(amax, xamax[tp * 256 + r]);
        const float S = amax / 448.0f;
        if (valid) {
          uint8_t *hq = static_cast<uint8_t *>(args.out) + orow * args.ldo + td.out_col;
          uint4 *hq4 = reinterpret_cast<uint4 *>(hq);
          if (S != 0.0f) {
            // quotients h / S share the divisor: correctly rounded through
            // the reciprocal plus one residual correction
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
          if (tall_half() == 0) args.out_scale[static_cast<int64_t>(td.blk) * args.ld_os + orow] = S;
        }
      } else {
        // FP32 rows (times the row's gate for EPI_GATE_F32), written through a
        // per-warp 32 x 16-float transpose buffer: each 16-byte store covers
        // 8 rows x 64 contiguous bytes instead of 32 scattered rows
        float *xb = outx + (warp - 4) * (32 * G_OPITCH);
        const int rbase = g * 128 + q * 32;  // this warp's first row in the tile
        const float gt = (EPI == EPI_GATE_F32 && valid) ? __ldg(args.row_gate + orow) : 1.0f;
        auto emit = [&](const float(&acc)[64], int64_t cbase) {
#pragma unroll
          for (int piece = 0; piece < 4; ++piece) {
            float4 *dst = reinterpret_cast<float4 *>(xb + lane * G_OPITCH);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int j = piece * 16 + 4 * v;
              dst[v] = make_float4(acc[j] * gt, acc[j + 1] * gt, acc[j + 2] * gt, acc[j + 3] * gt);
            }
            __syncwarp();
#pragma unroll
            for (int sgrp = 0; sgrp < 4; ++sgrp) {
              const int rr = lane / 4 + 8 * sgrp;
              if (rbase + rr < td.n) {
                const float4 val = reinterpret_cast<const float4 *>(xb + rr * G_OPITCH)[lane & 3];
                const int64_t grow = static_cast<int64_t>(td.out_row) + rbase + rr;
                float *crow = static_cast<float *>(args.out) + grow * args.ldo + cbase + piece * 16;
                reinterpret_cast<float4 *>(crow)[lane & 3] = val;
              }
            }
            __syncwarp();
          }
        };
        emit(acc0, td.out_col);
        emit(acc1, td.out_col + 64);
      }
      ++ntile;
    }
  }

  // neither CTA may leave while the other can still write its amax buffer
  // or arrive on its barriers
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

namespace {
template <int EPI>
std::atomic<int> *tall_cluster_cache() {
  static std::atomic<int> n[64];
  return n;
}

// Clusters of two that can be resident at once (queried once per device).
template <typename Fn>
int64_t resident_clusters(Fn *fn, std::atomic<int> *cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_acquire);
    if (c > 0) return c;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(T_THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(T_SMEM);
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
cudaError_t launch_tall_epi(const CUtensorMap &mw, const CUtensorMap &m0, const CUtensorMap &m1, const GemmArgs &a,
                            int64_t max_pairs, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(gemm_tall_kernel<EPI>, T_SMEM, attr_done)) return e;
  const int64_t clusters = resident_clusters(gemm_tall_kernel<EPI>, tall_cluster_cache<EPI>());
  if (clusters <= 0) return cudaErrorLaunchOutOfResources;
  const int64_t ncl = max_pairs < clusters ? max_pairs : clusters;
  gemm_tall_kernel<EPI><<<static_cast<unsigned>(2 * ncl), T_THREADS, T_SMEM, st>>>(mw, m0, m1, a);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_gemm_tall(const GemmLaunch &g, cudaStream_t st) {
  if (g.max_chunks <= 0 || g.nb <= 0) return cudaSuccess;
  if (g.chunk_rows != 256 || !g.sa_transposed) return cudaErrorInvalidValue;
  if (g.epi != EPI_SWIGLU_Q && g.epi != EPI_GATE_F32 && g.epi != EPI_F32) return cudaErrorInvalidValue;
  // gate/up: blocks of 128 channels (gate_up, nb = I / 128); down: pairs of
  // 128-channel output blocks (nb = H / 256)
  if (g.gate_up ? (g.half % 128 != 0 || g.nb * 128 != g.half)
                : (g.rows_per_expert % 256 != 0 || g.nb * 256 != g.rows_per_expert))
    return cudaErrorInvalidValue;
  CUtensorMap mw, m0, m1;
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, K, g.w_rows, K, 128, 64) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m0, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a0, K, g.a0_rows, K, 128, 32) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&m1, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a1, K, g.a1_rows,
                               g.a1_ld ? static_cast<uint64_t>(g.a1_ld) : K, 128, 32) != 0)
    return cudaErrorInvalidValue;
  const GemmArgs a = make_args(g);
  const int64_t max_pairs = static_cast<int64_t>(g.max_chunks) * g.nb;
  switch (g.epi) {
    case EPI_SWIGLU_Q: return launch_tall_epi<EPI_SWIGLU_Q>(mw, m0, m1, a, max_pairs, st);
    case EPI_GATE_F32: return launch_tall_epi<EPI_GATE_F32>(mw, m0, m1, a, max_pairs, st);
    default: return launch_tall_epi<EPI_F32>(mw, m0, m1, a, max_pairs, st);
  }
}

}  // namespace moe
