// router.cu -- sigmoid-affinity routing with a selection-only bias.
//
// "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), Methode section 2:
// s_{i,t} = Sigmoid(u_t^T e_i); expert i is chosen for token t when
// s_{i,t} + b_i is among the K_r largest of {s_{j,t} + b_j}; the gate of a
// chosen expert is s_{i,t} normalised over the chosen set.
//
// Three kernels:
//  1. router_logits_kernel: z = x . e_i for all (token, expert) on the
//     tensor cores (tcgen05 kind::f16, bf16 operands, FP32 accumulation in
//     TMEM), split over K so that enough CTAs run; each split writes its own
//     FP32 partial, summed in a fixed order by kernel 2 (deterministic).
//  2. router_topk_kernel: one warp per token; each lane holds the experts
//     lane, lane+32, ... in registers; sigmoid, bias, optional group
//     pre-selection and K_r rounds of warp-wide argmax.
//  3. seq_balance_kernel: the sequence-wise balance loss of a routed batch
//     (a metric of the routing, outside the layer step).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int R_STAGES = 6;
constexpr int R_TILE_BYTES = 128 * 128;  // 128 rows x 64 bf16
constexpr int R_STAGE_BYTES = 2 * R_TILE_BYTES;
constexpr int R_THREADS = 192;           // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int R_SMEM = R_STAGES * R_STAGE_BYTES + 1024 + 256;

struct RouterArgs {
  int64_t T;
  int Nr, n_eb, n_tb, n_ks, kb_total;
  float *partial;  // [n_ks, T, Nr]
  int32_t *err;
  uint64_t limit_ns;
};
}  // namespace

__global__ void __launch_bounds__(R_THREADS, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                         const RouterArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + R_STAGES * R_STAGE_BYTES);
  uint64_t *empty = full + R_STAGES;
  uint64_t *tfull = empty + R_STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *teardown = tempty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(teardown + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < R_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&map_w);
    tma_prefetch_map(&map_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl ctl{abort_flag, args.err, args.limit_ns};
  const int n_tiles = args.n_eb * args.n_tb * args.n_ks;

  auto tile_coords = [&](int tile, int &eb, int &tb, int &ks, int &kb0, int &kb1) {
    eb = tile % args.n_eb;
    const int r = tile / args.n_eb;
    tb = r % args.n_tb;
    ks = r / args.n_tb;
    kb0 = (ks * args.kb_total) / args.n_ks;
    kb1 = ((ks + 1) * args.kb_total) / args.n_ks;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      const uint64_t pol = policy_evict_last();
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        int eb, tb, ks, kb0, kb1;
        tile_coords(tile, eb, tb, ks, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % R_STAGES;
          if (!mbar_wait(&empty[s], ((it / R_STAGES) & 1) ^ 1, ctl)) break;
          uint8_t *st = smem + s * R_STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], R_STAGE_BYTES);
          tma_load_2d_hint(st, &map_w, &full[s], kb * 64, eb * 128, pol);
          tma_load_2d_hint(st + R_TILE_BYTES, &map_x, &full[s], kb * 64, tb * 128, pol);
        }
      }
      // let copies still in flight land before the CTA can exit
      int quiet = 0;
      const WaitCtl drain{&quiet, nullptr, 100000000ull};
      const uint32_t n_inflight = it < R_STAGES ? it : R_STAGES;
      for (uint32_t j = it - n_inflight; j < it; ++j) mbar_wait(&full[j % R_STAGES], (j / R_STAGES) & 1, drain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      const uint32_t idesc = idesc_bf16_f32(128, 128);
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x, ++tc) {
        int eb, tb, ks, kb0, kb1;
        tile_coords(tile, eb, tb, ks, kb0, kb1);
        const uint32_t buf = tc & 1;
        if (!mbar_wait(&tempty[buf], ((tc >> 1) & 1) ^ 1, ctl)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * 128;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % R_STAGES;
          if (!mbar_wait(&full[s], (it / R_STAGES) & 1, ctl)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * R_STAGE_BYTES);
          const uint64_t da = sw128_kmajor_desc(a_addr), db = sw128_kmajor_desc(a_addr + R_TILE_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_bf16(d, da + 2 * k, db + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        umma_commit(&tfull[buf]);
      }
      int quiet = 0;
      const WaitCtl drain{&quiet, nullptr, 100000000ull};
      umma_commit(teardown);
      mbar_wait(teardown, 0, drain);
    }
  } else {
    // epilogue: warps 2..5 -> TMEM lane quarters 2,3,0,1
    const int q = warp & 3;
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      int eb, tb, ks, kb0, kb1;
      tile_coords(tile, eb, tb, ks, kb0, kb1);
      const uint32_t buf = tc & 1;
      const bool ok = mbar_wait(&tfull[buf], (tc >> 1) & 1, ctl);
      if (!ok) break;
      tc_fence_after();
      const int e = eb * 128 + q * 32 + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 128;
      float *dst = args.partial + (static_cast<int64_t>(ks) * args.T) * args.Nr;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait();
        if (e < args.Nr) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int64_t t = static_cast<int64_t>(tb) * 128 + c * 32 + j;
            if (t < args.T) dst[t * args.Nr + e] = __uint_as_float(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ----------------------------------------------------------------- top-k
namespace {
constexpr int EPL = 8;  // experts per lane (N_r <= 256)

// s_{e,t} from the router's logit partials: the K splits are added in split
// order, then the sigmoid.  Every kernel that needs the affinities computes
// them here, so they agree bit for bit.
__device__ __forceinline__ float affinity(const float *__restrict__ partial, int n_ks, int64_t T, int Nr,
                                          int64_t t, int e) {
  float z = 0.0f;
  for (int k = 0; k < n_ks; ++k) z += partial[(static_cast<int64_t>(k) * T + t) * Nr + e];
  return 1.0f / (1.0f + expf(-z));
}

// Unsigned key with the order of the floats (-0 taken as +0), and back.
__device__ __forceinline__ uint32_t ord_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_val(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Largest v over the warp, ties to the smallest index i: two warp-wide
// reductions (the largest key, then the smallest index holding it).
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
  const uint32_t k = ord_key(v);
  const uint32_t best = __reduce_max_sync(0xffffffffu, k);
  const uint32_t bi = __reduce_min_sync(0xffffffffu, k == best ? static_cast<uint32_t>(i) : 0xffffffffu);
  v = ord_val(best);
  i = static_cast<int>(bi);
}
}  // namespace

__global__ void __launch_bounds__(256) router_topk_kernel(const float *__restrict__ partial, int n_ks, int64_t T,
                                                           int Nr, int Kr, int n_groups, int topk_groups,
                                                           float route_scale, const float *__restrict__ bias,
                                                           int32_t *__restrict__ idx, float *__restrict__ gate,
                                                           int32_t *__restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float s[EPL], c[EPL];
  bool ok[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    ok[i] = e < Nr;
    s[i] = 0.0f;
    c[i] = -INFINITY;
    if (ok[i]) {
      s[i] = affinity(partial, n_ks, T, Nr, t, e);
      c[i] = s[i] + bias[e];
    }
  }
  if (n_groups > 0) {
    // group g = experts [g*gs, (g+1)*gs); score = sum of its two largest c
    const int gs = Nr / n_groups;
    int grp[EPL];  // the group of each of this lane's experts, divided once
#pragma unroll
    for (int i = 0; i < EPL; ++i) grp[i] = (lane + 32 * i) / gs;
    float my_score = -INFINITY;  // lane g holds the score of group g
    if (gs == 32) {
      // lane l's expert i is expert 32 i + l, in group i: the top two of each
      // group over the lanes, all groups' butterflies side by side
      float b1[EPL], b2[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        b1[i] = ok[i] ? c[i] : -INFINITY;
        b2[i] = -INFINITY;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const float o1 = __shfl_xor_sync(0xffffffffu, b1[i], o);
          const float o2 = __shfl_xor_sync(0xffffffffu, b2[i], o);
          if (b1[i] >= o1) {
            b2[i] = fmaxf(b2[i], o1);
          } else {
            b2[i] = fmaxf(o2, b1[i]);
            b1[i] = o1;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane == i && i < n_groups) my_score = b1[i] + b2[i];
    }
    for (int g = 0; g < n_groups && gs != 32; ++g) {
      float b1 = -INFINITY, b2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if (ok[i] && grp[i] == g) {
          if (c[i] > b1) {
            b2 = b1;
            b1 = c[i];
          } else if (c[i] > b2) {
            b2 = c[i];
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, b1, o);
        const float o2 = __shfl_xor_sync(0xffffffffu, b2, o);
        if (b1 >= o1) {
          b2 = fmaxf(b2, o1);
        } else {
          b2 = fmaxf(o2, b1);
          b1 = o1;
        }
      }
      if (lane == g) my_score = b1 + b2;
    }
    uint32_t keep = 0;
    for (int r = 0; r < topk_groups; ++r) {
      float v = (keep >> lane) & 1u ? -INFINITY : my_score;
      int gi = lane < n_groups && !((keep >> lane) & 1u) ? lane : 0x7fffffff;
      if (lane >= n_groups) v = -INFINITY;
      warp_argmax(v, gi);
      keep |= 1u << gi;
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (ok[i] && !((keep >> grp[i]) & 1u)) ok[i] = false;
  }
  int sel_e = -1;   // lane r keeps the r-th choice
  float sel_s = 0.0f;
  float ssum = 0.0f;
  for (int r = 0; r < Kr; ++r) {
    float v = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (ok[i] && (c[i] > v || (c[i] == v && e < bi))) {
        v = c[i];
        bi = e;
      }
    }
    warp_argmax(v, bi);
    // owner lane fetches s of the winner and removes it
    float sw = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e == bi) {
        sw = s[i];
        ok[i] = false;
      }
    }
    sw = __shfl_sync(0xffffffffu, sw, bi & 31);
    ssum += sw;
    if (lane == r) {
      sel_e = bi;
      sel_s = sw;
    }
  }
  if (lane < Kr) {
    idx[t * Kr + lane] = sel_e;
    gate[t * Kr + lane] = route_scale * (sel_s / ssum);
    if (counts && sel_e >= 0 && sel_e < Nr) atomicAdd(&counts[sel_e], 1);
  }
}

// ------------------------------------------------ sequence-wise balance loss
// One CTA per sequence of L tokens (the complementary loss of "DeepSeek-V3
// Technischer Bericht", Methode section 2, in the technical report's form):
//   loss = alpha * sum_i f_i P_i,  f_i = N_r / (K_r L) * picks_i,
//   P_i = (1/L) sum_t s_{i,t} / sum_j s_{j,t}.
// Warp w takes tokens w, w + BL_WARPS, ... of the sequence; lane l keeps, for
// the experts l, l+32, ..., the running sums of the normalised affinities and
// of the picks.  The warps' sums are then added in warp order and the
// experts' terms in expert order, so the result does not depend on the
// schedule.  Reads the partials once: HBM-bound, a metric outside the step.
constexpr int BL_WARPS = 16;

__global__ void __launch_bounds__(BL_WARPS * 32)
    seq_balance_kernel(const float *__restrict__ partial, int n_ks, int64_t T, int Nr,
                       const int32_t *__restrict__ idx, int Kr, int64_t seq_len, float alpha,
                       float *__restrict__ loss, int32_t *err) {
  __shared__ float p_sh[BL_WARPS][EPL * 32];
  __shared__ int c_sh[BL_WARPS][EPL * 32];
  __shared__ float term[EPL * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * seq_len;
  float acc[EPL];
  int cnt[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    acc[i] = 0.0f;
    cnt[i] = 0;
  }
  bool bad = false;
  for (int64_t t = t0 + warp; t < t0 + seq_len; t += BL_WARPS) {
    float s[EPL];
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      s[i] = e < Nr ? affinity(partial, n_ks, T, Nr, t, e) : 0.0f;
      sum += s[i];
    }
    // butterfly: every lane ends with the same total
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] += s[i] / sum;
    for (int k = 0; k < Kr; ++k) {
      const int e = idx[t * Kr + k];
      if (e < 0 || e >= Nr) {
        bad = true;
        continue;
      }
      if ((e & 31) == lane) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) cnt[i] += (i == (e >> 5)) ? 1 : 0;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    p_sh[warp][lane + 32 * i] = acc[i];
    c_sh[warp][lane + 32 * i] = cnt[i];
  }
  if (bad && lane == 0 && err) atomicOr(err, MOE_DEVERR_BAD_INDEX);
  __syncthreads();
  if (threadIdx.x < EPL * 32) {
    const int e = threadIdx.x;
    float p = 0.0f;
    int c = 0;
    for (int w = 0; w < BL_WARPS; ++w) {
      p += p_sh[w][e];
      c += c_sh[w][e];
    }
    term[e] = e < Nr ? static_cast<float>(c) * p : 0.0f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.0f;
    for (int e = 0; e < Nr; ++e) tot += term[e];
    const float L = static_cast<float>(seq_len);
    // sum_i f_i P_i = N_r / (K_r L) * sum_i picks_i * (sum_t s'_{i,t}) / L
    loss[blockIdx.x] = alpha * (static_cast<float>(Nr) / (static_cast<float>(Kr) * L)) * (tot / L);
  }
}

cudaError_t launch_seq_balance(const float *partial, int n_ks, int64_t T, int Nr, const int32_t *idx, int Kr,
                               int64_t seq_len, float alpha, float *loss, int32_t *err, cudaStream_t st) {
  if (T == 0 || seq_len <= 0) return cudaSuccess;
  const int64_t n_seq = T / seq_len;
  seq_balance_kernel<<<static_cast<unsigned>(n_seq), BL_WARPS * 32, 0, st>>>(partial, n_ks, T, Nr, idx, Kr,
                                                                             seq_len, alpha, loss, err);
  return cudaGetLastError();
}

// ------------------------------------------------ fixed scratch (no allocation)
// Scratch of moe_route_noalloc: the router's FP32 logit partials live in this
// file-scope array instead of a caller buffer.  Every GPU that loads the
// library holds it (16 MiB) until the process exits, and all calls share it.
static __device__ __align__(256) float g_route_scratch[kRouteNoAllocScratchFloats];

// Device address of g_route_scratch in the current device's context, looked
// up on every call (cudaGetSymbolAddress allocates nothing and is cheap), so
// a context torn down and created again (cudaDeviceReset) never leaves a
// stale address behind.  Host code must never pass the array's host-side
// name itself.
cudaError_t route_static_scratch(float **ptr) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
  if (e != cudaSuccess) return e;
  *ptr = static_cast<float *>(p);
  return cudaSuccess;
}

int router_ksplit(int64_t T, int Nr, int H) {
  const int64_t base = ((T + 127) / 128) * ((Nr + 127) / 128);
  const int kb_total = H / 64;
  if (base <= 0) return 1;
  // as many K splits as fit the SMs in one wave: a second, partial wave
  // would add a whole split's time for a few CTAs
  const int64_t sms = moe_host::sm_count();
  int64_t ks = sms / base;
  if (ks > 16) ks = 16;
  if (ks > kb_total) ks = kb_total;
  if (ks < 1) ks = 1;
  return static_cast<int>(ks);
}

cudaError_t launch_router_logits(const void *x, const void *wr, int64_t T, int Nr, int H, float *partial,
                                 int32_t *err, uint64_t limit_ns, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  CUtensorMap mw, mx;
  if (moe_host::encode_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wr, H, Nr, static_cast<uint64_t>(H) * 2, 64,
                               128) != 0)
    return cudaErrorInvalidValue;
  if (moe_host::encode_tmap_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, T, static_cast<uint64_t>(H) * 2, 64,
                               128) != 0)
    return cudaErrorInvalidValue;
  RouterArgs a;
  a.T = T;
  a.Nr = Nr;
  a.n_eb = (Nr + 127) / 128;
  a.n_tb = static_cast<int>((T + 127) / 128);
  a.n_ks = router_ksplit(T, Nr, H);
  a.kb_total = H / 64;
  a.partial = partial;
  a.err = err;
  a.limit_ns = limit_ns;
  static std::atomic<uint64_t> attr_done{0};
  if (const cudaError_t e = smem_attr_once(router_logits_kernel, R_SMEM, attr_done)) return e;
  const int tiles = a.n_eb * a.n_tb * a.n_ks;
  const int grid = tiles < moe_host::sm_count() ? tiles : moe_host::sm_count();
  router_logits_kernel<<<grid, R_THREADS, R_SMEM, st>>>(mw, mx, a);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const float *partial, int n_ks, int64_t T, int Nr, int Kr, int n_groups,
                               int topk_groups, float route_scale, const float *bias, int32_t *idx, float *gate,
                               int32_t *counts, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t blocks = (T + 7) / 8;
  router_topk_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(partial, n_ks, T, Nr, Kr, n_groups,
                                                                     topk_groups, route_scale, bias, idx, gate,
                                                                     counts);
  return cudaGetLastError();
}

}  // namespace moe
