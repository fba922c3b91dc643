// gemm_tiles.cuh -- work decomposition shared by the grouped FP8 GEMM kernels
// (gemm.cu: FP32 scales promoted per 128-K block; gemm_mx.cu: power-of-two
// scales applied by the tensor core).  Internal to the library.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace gemm_detail {

constexpr int G_KBMAX = 256;  // K/128 up to 256 (K <= 32768)

struct GemmArgs {
  const int4 *chunks;        // chunk table, or null for the dense grid
  const int32_t *n_chunks;   // device count of chunks
  int max_chunks;
  int chunk_rows;            // most activation rows per chunk: 128 (one CTA) or 256 (a CTA pair)
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

// Tile order.  Tiles t in [c0 nb, (c0 + k) nb) belong to the k chunks
// c0 .. c0 + k - 1 of one expert; inside that range they run weight block by
// weight block (t = c0 nb + rb k + i: chunk c0 + i, block rb), so the k tiles
// that read the same weight tile are neighbours in the persistent walk and
// run side by side: the weight tile comes from HBM once and from L2 for the
// other k - 1.  An expert of one chunk keeps (chunk, block) = (t / nb, t % nb).
__device__ __forceinline__ void tile_coords(const GemmArgs &a, int t, int &c, int &rb, int4 &ch) {
  c = t / a.nb;
  rb = t - c * a.nb;
  if (!a.chunks) return;
  ch = a.chunks[c];
  const int k = chunk_group(ch);
  if (k > 1) {
    // (a table that does not describe a group keeps the plain order; every
    // entry read stays inside the table's max_chunks entries)
    const int c0 = c - chunk_pos(ch);
    const int local = t - c0 * a.nb;
    if (c0 >= 0 && c0 + k <= a.max_chunks && local >= 0 && local < k * a.nb) {
      rb = local / k;
      c = c0 + (local - rb * k);
      ch = a.chunks[c];
    }
  }
}

__device__ __forceinline__ GemmTile get_tile(const GemmArgs &a, int t) {
  int c, rb;
  int4 ch = make_int4(0, 0, 0, 0);
  tile_coords(a, t, c, rb, ch);
  GemmTile d;
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
    d.w_row0 = static_cast<int32_t>(base + rb * 128);
    d.w_row1 = static_cast<int32_t>(base + a.half + rb * 128);
    d.out_col = rb * 128;
  } else {
    d.w_row0 = static_cast<int32_t>(base + 2 * rb * 128);
    d.w_row1 = (static_cast<int64_t>(2 * rb + 1) * 128 < a.rows_per_expert) ? d.w_row0 + 128 : -1;
    d.out_col = 2 * rb * 128;
  }
  return d;
}

// A tile whose fields would read or write outside the operands is skipped by
// every role alike (and reported), so a corrupt chunk table cannot fault.
__device__ __forceinline__ bool tile_ok(const GemmArgs &a, const GemmTile &d) {
  const int64_t arows = d.from1 ? a.a_rows1 : a.a_rows0;
  const bool two = d.w_row1 >= 0;
  return d.n >= 1 && d.n <= a.chunk_rows && d.a_row >= 0 && d.a_row + d.n <= arows && d.out_row >= 0 &&
         d.out_row + d.n <= a.out_rows && d.w_row0 >= 0 && d.w_row0 + 128 <= a.w_rows &&
         (!two || d.w_row1 + 128 <= a.w_rows) && d.out_col >= 0 && d.out_col + (two ? 256 : 128) <= a.out_cols &&
         (!a.sa_transposed || d.out_row + d.n <= a.sa_ld) && a.KB <= G_KBMAX;
}

// Epilogue of one tile for the thread owning activation row r (lane quarter
// q = warp & 3 of warpgroup wg = (warp - 4) / 4) and 64 columns of each
// weight block, after the tile's accumulators are in acc0 / acc1:
//   EPI_SWIGLU_Q  block A = gate, block B = up: h = silu(G) * U in FP32, then
//                 the 1x128 requantization of h over the tile's 128 channels
//                 (amax of the row's two 64-channel halves exchanged between
//                 the warpgroups through amx; S = amax / 448, or the power-of-
//                 two scale when POW2; E4M3 RNE), 64 codes per thread stored
//                 as 16-byte vectors -> hq, scale -> hs
//   EPI_GATE_F32  y = acc * gate[row] in FP32 (down projection)
//   EPI_BF16      C = bf16(acc) (plain GEMM)
//   EPI_F32       C = acc in FP32 (block B at +128 columns, or at +half for a
//                 gate/up pair)
// Both warpgroups take the named barrier 1 (256 threads) twice per tile in
// EPI_SWIGLU_Q.
constexpr int G_OPITCH = 20;  // floats per row of an output transpose buffer (16 + pad)

template <int EPI, bool POW2>
// rq: the tile-row quarter whose rows the thread's TMEM lane quarter holds
// (the lane quarter itself unless the kernel permutes rows over lanes).
__device__ __forceinline__ void tile_epilogue(const GemmArgs &args, const GemmTile &td, float (&acc0)[64],
                                              float (&acc1)[64], bool two, int warp, int lane, float *amx,
                                              float *outx, int rq) {
  const int wg = (warp - 4) >> 2;
  const int q = rq;
  const int r = q * 32 + lane;
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
    const float S = POW2 ? pow2_scale(amax) : amax / 448.0f;
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
  } else if constexpr (EPI == EPI_F32 || EPI == EPI_GATE_F32) {
    // FP32 results of both blocks (times the row's gate for EPI_GATE_F32);
    // block B's columns follow block A's (+128), or start at +half when the
    // pair is gate block j / up block j
    float *xb = outx + (warp - 4) * (32 * G_OPITCH);
    const int rbase = q * 32;
    const int64_t cB = args.gate_up ? args.half : 128;
    const float g = (EPI == EPI_GATE_F32 && valid) ? __ldg(args.row_gate + orow) : 1.0f;
    auto emit = [&](const float(&acc)[64], int64_t cbase) {
#pragma unroll
      for (int piece = 0; piece < 4; ++piece) {
        float4 *dst = reinterpret_cast<float4 *>(xb + lane * G_OPITCH);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int j = piece * 16 + 4 * v;
          dst[v] = make_float4(acc[j] * g, acc[j + 1] * g, acc[j + 2] * g, acc[j + 3] * g);
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
    emit(acc0, c0);
    if (two) emit(acc1, c0 + cB);
  } else {
    // Rows are written through a per-warp 32 x 16-float transpose buffer
    // so that each 16-byte store instruction covers 8 rows x 64
    // contiguous bytes instead of 32 scattered rows.
    float *xb = outx + (warp - 4) * (32 * G_OPITCH);
    const int rbase = q * 32;  // this warp's first row in the tile
    auto emit = [&](const float(&acc)[64], int b) {
#pragma unroll
      for (int piece = 0; piece < 2; ++piece) {
        // stage: this thread's 32 bf16 of the piece, row = lane
        float4 *dst = reinterpret_cast<float4 *>(xb + lane * G_OPITCH);
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
        __syncwarp();
        // drain: lane L stores 16 bytes of row (L / 4 + 8 s), chunk L % 4
#pragma unroll
        for (int sgrp = 0; sgrp < 4; ++sgrp) {
          const int rr = lane / 4 + 8 * sgrp;  // row within the warp's 32
          if (rbase + rr < td.n) {
            const float4 val = reinterpret_cast<const float4 *>(xb + rr * G_OPITCH)[lane & 3];
            const int64_t grow = static_cast<int64_t>(td.out_row) + rbase + rr;
            __nv_bfloat16 *crow =
                static_cast<__nv_bfloat16 *>(args.out) + grow * args.ldo + c0 + 128 * b + piece * 32;
            reinterpret_cast<float4 *>(crow)[lane & 3] = val;
          }
        }
        __syncwarp();
      }
    };
    emit(acc0, 0);
    if (two) emit(acc1, 1);
  }
}

// Kernel arguments of one launch from the host-side description.
inline GemmArgs make_args(const GemmLaunch &g) {
  GemmArgs a;
  a.chunks = g.chunks;
  a.n_chunks = g.n_chunks;
  a.max_chunks = g.max_chunks;
  a.dense_M = g.dense_M;
  a.chunk_rows = g.chunk_rows == 256 ? 256 : 128;
  a.dense_chunks = g.chunks ? 0 : static_cast<int>((g.dense_M + a.chunk_rows - 1) / a.chunk_rows);
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
  return a;
}

}  // namespace gemm_detail
}  // namespace moe
