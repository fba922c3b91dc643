// api.cu -- the extern "C" entry points of libmoefp8 (declared in
// include/moe_fp8.h): argument validation, workspace carving, tensor-map
// encoding and the launch sequence of the layer forward.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace moe_host {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void resolve_encode() {
  cudaDriverEntryPointQueryResult q;
  void *fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
int g_major[kMaxDevices] = {0};
}  // namespace

int encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, resolve_encode);
  if (!g_encode) return -1;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

static int device_info(int *sms, int *major) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  if (g_sms[dev] == 0) {
    int s = 0, m = 0;
    if (cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&m, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
    g_major[dev] = m;
    g_sms[dev] = s;
  }
  *sms = g_sms[dev];
  *major = g_major[dev];
  return 0;
}

int sm_count() {
  int s = 0, m = 0;
  if (device_info(&s, &m) != 0) return 148;
  return s;
}

}  // namespace moe_host

namespace {


inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Longest contraction the GEMM kernels take: each tile keeps the scales of up
// to 256 K blocks of 128.
constexpr int64_t kMaxK = 256 * 128;

int check_device() {
  int sms = 0, major = 0;
  if (moe_host::device_info(&sms, &major) != 0) return MOE_ERR_NO_DEVICE;
  if (major != 10) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

// NVTX ranges (host side, header-only NVTX3: inert unless a profiler is
// attached) around each public call and the stages of the layer, so that a
// timeline tool can attribute launches to them.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

int check_cfg(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_routed <= 0 || c->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 || c->inter % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->hidden > kMaxK || c->inter > kMaxK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_routed > 256 || c->top_k > 16 || c->top_k > c->n_routed) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_shared < 0 || c->n_shared > 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_groups < 0) return MOE_ERR_INVALID_ARG;
  if (c->n_groups > 0) {
    if (c->n_groups > 32 || c->n_routed % c->n_groups) return MOE_ERR_UNSUPPORTED_SHAPE;
    // a group's score is the sum of its two best biased scores: it needs two
    // experts per group
    if (c->n_routed / c->n_groups < 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(c->topk_groups) * (c->n_routed / c->n_groups) < c->top_k) return MOE_ERR_INVALID_ARG;
  }
  if (!(c->route_scale == c->route_scale)) return MOE_ERR_INVALID_ARG;
  if (c->scale_mode != MOE_SCALE_AMAX && c->scale_mode != MOE_SCALE_POW2) return MOE_ERR_INVALID_ARG;
  // weight rows must be addressable by 32-bit TMA coordinates
  const int64_t E = static_cast<int64_t>(c->n_routed) + c->n_shared;
  if (E * 2 * c->inter > INT32_MAX || E * c->hidden > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// The expert side of expert parallelism: top_k counts the slots of a packed
// row, which may exceed the rank's own experts (a slot whose expert lives
// elsewhere is -1); no routing groups, no shared expert.
int check_cfg_local(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > 16 || c->n_routed < 1) return c->top_k > 16 ? MOE_ERR_UNSUPPORTED_SHAPE : MOE_ERR_INVALID_ARG;
  if (c->n_shared != 0 || c->n_groups != 0) return MOE_ERR_INVALID_ARG;
  moe_config t = *c;
  t.top_k = 1;  // the rest of the checks as for a layer
  return check_cfg(&t);
}

constexpr int64_t kMaxTokens = 1 << 20;

// The grouped GEMMs of the default scale mode run on single CTAs (<= 128 rows
// of an expert per weight pass) or on CTA pairs (<= 256 rows), the latter only
// when the down projection's weight blocks pair up (H a multiple of 256).
// MOE_GEMM_AUTO takes pairs when the routed experts average at least 256 rows
// (T * K_r >= 256 * N_r): then most experts fill pair tiles and each weight
// block is read half as often; below that, half-empty pair tiles cost more
// than the saved weight reads (measured at V3 sizes: 128 rows per expert is
// faster on single CTAs, 512 on pairs).
std::atomic<int> g_gemm_variant{MOE_GEMM_AUTO};

// The grouped-GEMM kernel of a forward of T tokens (MOE_GEMM_SINGLE, _PAIR,
// _TALL or _BLOCK_SCALED).  Pairs and tall tiles need the down projection's
// 128-row weight blocks to pair up (H a multiple of 256).  MOE_GEMM_AUTO takes
// single CTAs: with the tiles of an expert's chunks run side by side (one HBM
// read of each weight tile), they were the fastest at every V3 size measured
// (decode 64, prefill 4096 and skewed 16384 tokens).
int gemm_kernel_for(const moe_config *c, int64_t T) {
  (void)T;
  if (c->scale_mode == MOE_SCALE_POW2) return MOE_GEMM_BLOCK_SCALED;
  if ((c->hidden / 128) % 2 != 0) return MOE_GEMM_SINGLE;
  const int v = g_gemm_variant.load(std::memory_order_relaxed);
  if (v == MOE_GEMM_PAIR || v == MOE_GEMM_TALL) return v;
  return MOE_GEMM_SINGLE;
}

struct Carve {
  size_t off = 0;
  void take(size_t (&slot)[2], size_t bytes) {
    off = (off + 255) & ~size_t(255);
    slot[0] = off;
    slot[1] = bytes;
    off += bytes;
  }
};

void make_layout(const moe_config *c, int64_t T, moe_ws_layout *L) {
  const int64_t H = c->hidden, I = c->inter, Nr = c->n_routed, Kr = c->top_k, Ns = c->n_shared;
  const int64_t R = T * Kr, RS = R + T * Ns;
  const int64_t nblk = (T + 127) / 128;
  const int64_t ks = moe::router_ksplit(T, static_cast<int>(Nr), static_cast<int>(H));
  const int64_t chunks = moe::max_chunks(T, static_cast<int>(Kr), static_cast<int>(Nr), static_cast<int>(Ns));
  Carve cv;
  cv.take(L->xq, T * H);
  cv.take(L->xs, T * (H / 128) * 4);
  cv.take(L->idx, T * Kr * 4);
  cv.take(L->gate, T * Kr * 4);
  cv.take(L->counts, Nr * 4);
  cv.take(L->offsets, (Nr + 1) * 4);
  cv.take(L->pos, T * Kr * 4);
  cv.take(L->ap, R * H);
  const int64_t pitch = moe::scale_pitch(R, T);
  cv.take(L->as, ((H / 128) * pitch + moe::kScaleSlack) * 4);
  cv.take(L->row_gate, RS * 4);
  cv.take(L->row_src, R * 4);
  cv.take(L->hq, RS * I);
  cv.take(L->hs, ((I / 128) * pitch + moe::kScaleSlack) * 4);
  cv.take(L->y, RS * H * 4);
  cv.take(L->meta, 4 * 4);
  cv.take(L->logits, ks * T * Nr * 4);
  cv.take(L->blk_hist, nblk * Nr * 4);
  cv.take(L->blk_base, nblk * Nr * 4);
  cv.take(L->chunks, chunks * 16);
  L->total = (cv.off + 255) & ~size_t(255);
}

thread_local cudaEvent_t g_prof_events[MOE_PROFILE_EVENTS + MOE_PROFILE_BWD_EVENTS];
thread_local bool g_prof_on = false;
thread_local bool g_prof_bwd_on = false;

inline cudaError_t prof_mark_bwd(int i, cudaStream_t st) {
  return g_prof_bwd_on ? cudaEventRecord(g_prof_events[MOE_PROFILE_EVENTS + i], st) : cudaSuccess;
}
inline cudaError_t prof_mark(int i, cudaStream_t st) {
  return g_prof_on ? cudaEventRecord(g_prof_events[i], st) : cudaSuccess;
}

template <typename P>
inline P at(void *ws, const size_t (&slot)[2]) {
  return reinterpret_cast<P>(static_cast<uint8_t *>(ws) + slot[0]);
}

}  // namespace

extern "C" {

const char *moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (tiled dimensions must be multiples of 128)";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_NOT_IMPLEMENTED: return "not implemented";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device is current";
    case MOE_ERR_DEVICE: return "device reported an error";
    default: return "unknown status";
  }
}

int moe_abi_version(void) { return 104; }

int moe_set_gemm_variant(int32_t variant) {
  if (variant != MOE_GEMM_AUTO && variant != MOE_GEMM_SINGLE && variant != MOE_GEMM_PAIR && variant != MOE_GEMM_TALL)
    return MOE_ERR_INVALID_ARG;
  g_gemm_variant.store(variant, std::memory_order_relaxed);
  return MOE_OK;
}

int moe_gemm_kernel_for(const moe_config *cfg, int64_t T) {
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  return gemm_kernel_for(cfg, T);
}

static int quant_1x128(const void *x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *q, float *scales,
                       void *stream, bool pow2) {
  if (rows < 0 || cols <= 0 || ld_x < cols || (ld_x % 8) != 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3))
    return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  return cuda_status(
      moe::launch_quant_1x128(x, rows, cols, ld_x, q, scales, static_cast<cudaStream_t>(stream), pow2));
}

int fp8_quant_1x128(const void *x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *q, float *scales,
                    void *stream) {
  return quant_1x128(x, rows, cols, ld_x, q, scales, stream, false);
}

int fp8_quant_1x128_pow2(const void *x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *q, float *scales,
                         void *stream) {
  return quant_1x128(x, rows, cols, ld_x, q, scales, stream, true);
}

static int quant_128x128(const void *w, int64_t n, int64_t k, uint8_t *q, float *scales, void *stream,
                         bool pow2) {
  if (n < 0 || k < 0) return MOE_ERR_INVALID_ARG;
  if (n % 128 || k % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (n == 0 || k == 0) return MOE_OK;
  if (!w || !q || !scales || !aligned16(w) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3))
    return MOE_ERR_INVALID_ARG;
  if ((n / 128) * (k / 128) > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (const int d = check_device()) return d;
  return cuda_status(moe::launch_quant_128x128(w, n, k, q, scales, static_cast<cudaStream_t>(stream), pow2));
}

int fp8_quant_128x128(const void *w, int64_t n, int64_t k, uint8_t *q, float *scales, void *stream) {
  return quant_128x128(w, n, k, q, scales, stream, false);
}

int fp8_quant_128x128_pow2(const void *w, int64_t n, int64_t k, uint8_t *q, float *scales, void *stream) {
  return quant_128x128(w, n, k, q, scales, stream, true);
}

int fp8_blockscaled_gemm(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB, void *C, int64_t M,
                         int64_t N, int64_t K, int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("fp8_blockscaled_gemm");
  if (M < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (N % 128 || K % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return MOE_OK;
  if (M > INT32_MAX - 256 || N > INT32_MAX - 256 || K > kMaxK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!A || !sA || !B || !sB || !C || !err_flag) return MOE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || !aligned4(sA) || !aligned4(sB) || !aligned4(err_flag))
    return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  moe::GemmLaunch g{};
  g.w = B;
  g.w_rows = N;
  g.a0 = A;
  g.a0_rows = M;
  g.a1 = A;
  g.a1_rows = M;
  g.K = K;
  g.sw = sB;
  g.sa0 = sA;
  g.sa1 = sA;
  g.sa_transposed = 0;
  g.chunks = nullptr;
  g.n_chunks = nullptr;
  g.dense_M = M;
  g.max_chunks = static_cast<int>((M + 127) / 128);
  g.chunk_rows = 128;
  g.nb = static_cast<int>((N / 128 + 1) / 2);
  g.gate_up = 0;
  g.rows_per_expert = N;
  g.epi = moe::EPI_BF16;
  g.out = C;
  g.ldo = N;
  g.out_rows = M;
  g.out_cols = N;
  g.err = err_flag;
  g.wait_limit_ns = moe::kDefaultWaitLimitNs;
  return cuda_status(moe::launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

size_t moe_route_workspace_size(const moe_config *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0 || T > kMaxTokens) return 0;
  const int64_t ks = moe::router_ksplit(T, cfg->n_routed, cfg->hidden);
  return static_cast<size_t>(ks * T * cfg->n_routed * 4 + 256);
}

int moe_route(const moe_config *cfg, const void *x, const void *wr, const float *bias, int64_t T, int32_t *idx,
              float *gate, int32_t *counts, void *ws, size_t ws_bytes, int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("moe_route");
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (!counts) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (const int d = check_device()) return d;
    return cuda_status(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_routed, st));
  }
  if (!x || !wr || !bias || !idx || !gate || !ws || !err_flag) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wr) || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOE_ERR_INVALID_ARG;
  if (!aligned4(bias) || !aligned4(idx) || !aligned4(gate) || !aligned4(counts) || !aligned4(err_flag))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_route_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  float *partial = static_cast<float *>(ws);
  const int ks = moe::router_ksplit(T, cfg->n_routed, cfg->hidden);
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_routed, st);
  if (e == cudaSuccess)
    e = moe::launch_router_logits(x, wr, T, cfg->n_routed, cfg->hidden, partial, err_flag,
                                  moe::kDefaultWaitLimitNs, st);
  if (e == cudaSuccess)
    e = moe::launch_router_topk(partial, ks, T, cfg->n_routed, cfg->top_k, cfg->n_groups, cfg->topk_groups,
                                cfg->route_scale, bias, idx, gate, counts, st);
  return cuda_status(e);
}

int moe_route_noalloc(const moe_config *cfg, const void *x, const void *wr, const float *bias, int64_t T,
                      int32_t *idx, float *gate, int32_t *counts, int32_t *err_flag, void *stream) {
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (!counts) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (const int d = check_device()) return d;
    return cuda_status(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_routed, st));
  }
  if (!x || !wr || !bias || !idx || !gate || !err_flag) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wr)) return MOE_ERR_INVALID_ARG;
  if (!aligned4(bias) || !aligned4(idx) || !aligned4(gate) || !aligned4(counts) || !aligned4(err_flag))
    return MOE_ERR_INVALID_ARG;
  const int ks = moe::router_ksplit(T, cfg->n_routed, cfg->hidden);
  if (static_cast<size_t>(ks) * static_cast<size_t>(T) * cfg->n_routed > moe::kRouteNoAllocScratchFloats)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  float *partial = nullptr;
  cudaError_t e = moe::route_static_scratch(&partial);
  if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_routed, st);
  if (e == cudaSuccess)
    e = moe::launch_router_logits(x, wr, T, cfg->n_routed, cfg->hidden, partial, err_flag,
                                  moe::kDefaultWaitLimitNs, st);
  if (e == cudaSuccess)
    e = moe::launch_router_topk(partial, ks, T, cfg->n_routed, cfg->top_k, cfg->n_groups, cfg->topk_groups,
                                cfg->route_scale, bias, idx, gate, counts, st);
  return cuda_status(e);
}

size_t moe_workspace_size(const moe_config *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0 || T > kMaxTokens) return 0;
  moe_ws_layout L;
  make_layout(cfg, T, &L);
  return L.total;
}

int moe_workspace_layout(const moe_config *cfg, int64_t T, moe_ws_layout *layout) {
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens || !layout) return MOE_ERR_INVALID_ARG;
  make_layout(cfg, T, layout);
  return MOE_OK;
}

// Grouping, both grouped GEMMs and the combine of one forward, from rows
// already quantized (xq rows xq_ld bytes apart, xs [T, H/128] contiguous) and
// routed (idx, gate [T, K_r]; with allow_empty, -1 marks an unused slot).
// out[t] = x_resid[t] (if given) + shared expert (if N_s) + sum_k g y.
struct ExpertPath {
  const moe_config *cfg;
  const moe_weights *w;
  int64_t T;
  const uint8_t *xq;
  int64_t xq_ld;
  const float *xs;
  const int32_t *idx;
  const float *gate;
  int allow_empty;
  const void *x_resid;
  void *out;
  int out_f32;
  int32_t *counts_out;
  const moe_ws_layout *L;
  void *ws;
  int32_t *err;
  cudaStream_t st;
};

static cudaError_t run_expert_path(const ExpertPath &P) {
  const moe_config *cfg = P.cfg;
  const moe_weights *w = P.w;
  const moe_ws_layout &L = *P.L;
  void *ws = P.ws;
  cudaStream_t st = P.st;
  int32_t *err_flag = P.err;
  const int64_t T = P.T;
  const int H = cfg->hidden, I = cfg->inter, Nr = cfg->n_routed, Kr = cfg->top_k, Ns = cfg->n_shared;
  const int64_t R = T * Kr, RS = R + T * Ns;
  const int64_t E = static_cast<int64_t>(Nr) + Ns;
  int32_t *counts = at<int32_t *>(ws, L.counts);
  int32_t *offsets = at<int32_t *>(ws, L.offsets);
  int32_t *pos = at<int32_t *>(ws, L.pos);
  uint8_t *ap = at<uint8_t *>(ws, L.ap);
  float *as_t = at<float *>(ws, L.as);
  float *row_gate = at<float *>(ws, L.row_gate);
  int32_t *row_src = at<int32_t *>(ws, L.row_src);
  uint8_t *hq = at<uint8_t *>(ws, L.hq);
  float *hs_t = at<float *>(ws, L.hs);
  float *y = at<float *>(ws, L.y);
  int32_t *meta = at<int32_t *>(ws, L.meta);
  int32_t *blk_hist = at<int32_t *>(ws, L.blk_hist);
  int32_t *blk_base = at<int32_t *>(ws, L.blk_base);
  int4 *chunks = at<int4 *>(ws, L.chunks);
  const int64_t max_chunks = moe::max_chunks(T, Kr, Nr, Ns);
  const int kern = gemm_kernel_for(cfg, T);
  const bool pow2 = kern == MOE_GEMM_BLOCK_SCALED;
  const bool pair = kern == MOE_GEMM_PAIR;
  const bool tall = kern == MOE_GEMM_TALL;
  const int chunk_rows = pair || tall ? 256 : 128;

  cudaError_t e = moe::launch_hist(P.idx, T, Kr, Nr, P.allow_empty, blk_hist, err_flag, st);
  if (e == cudaSuccess)
    e = moe::launch_build_chunks(blk_hist, T, Kr, Nr, Ns, chunk_rows, counts, offsets, blk_base, chunks, meta,
                                 P.counts_out, st);
  if (e == cudaSuccess) e = moe::launch_rank(P.idx, P.gate, T, Kr, Nr, Ns, blk_base, row_gate, row_src, pos, st);
  const int64_t pitch = moe::scale_pitch(R, T);
  if (e == cudaSuccess) e = moe::launch_copy_rows(P.xq, P.xq_ld, P.xs, row_src, R, T, Ns, H, ap, as_t, pitch, st);
  if (e == cudaSuccess) e = prof_mark(3, st);
  if (e == cudaSuccess) {
    const NvtxRange nvtx_stage("gemm_gate_up");
    // gate/up projection + SwiGLU + 1x128 requantization
    moe::GemmLaunch g{};
    g.w = w->w13_dev;
    g.w_rows = E * 2 * I;
    g.a0 = ap;
    g.a0_rows = R;
    g.a1 = Ns ? P.xq : ap;  // the shared expert's rows are the quantized input itself
    g.a1_rows = Ns ? T : R;
    g.a1_ld = Ns ? P.xq_ld : H;
    g.K = H;
    g.sw = w->s13_dev;
    g.sa0 = as_t;
    g.sa1 = as_t;
    g.sa_transposed = 1;
    g.sa_ld = pitch;
    g.chunks = chunks;
    g.n_chunks = meta;
    g.max_chunks = static_cast<int>(max_chunks);
    g.chunk_rows = chunk_rows;
    g.nb = moe::gemm1_blocks(I);
    g.gate_up = 1;
    g.half = I;
    g.rows_per_expert = 2 * static_cast<int64_t>(I);
    g.epi = moe::EPI_SWIGLU_Q;
    g.out = hq;
    g.ldo = I;
    g.out_rows = RS;
    g.out_cols = 2 * I;  // block B (up) shares block A's output columns
    g.out_scale = hs_t;
    g.ld_os = pitch;
    g.err = err_flag;
    g.wait_limit_ns = moe::kDefaultWaitLimitNs;
    e = pow2   ? moe::launch_gemm_mx(g, st)
        : pair ? moe::launch_gemm_pair(g, st)
        : tall ? moe::launch_gemm_tall(g, st)
               : moe::launch_gemm(g, st);
  }
  if (e == cudaSuccess) e = prof_mark(4, st);
  if (e == cudaSuccess) {
    const NvtxRange nvtx_stage("gemm_down");
    // down projection, scaled by the gate of each row
    moe::GemmLaunch g{};
    g.w = w->w2_dev;
    g.w_rows = E * H;
    g.a0 = hq;
    g.a0_rows = RS;
    g.a1 = hq;
    g.a1_rows = RS;
    g.K = I;
    g.sw = w->s2_dev;
    g.sa0 = hs_t;
    g.sa1 = hs_t;
    g.sa_transposed = 1;
    g.sa_ld = pitch;
    g.chunks = chunks;
    g.n_chunks = meta;
    g.max_chunks = static_cast<int>(max_chunks);
    g.chunk_rows = chunk_rows;
    g.nb = tall ? H / 256 : moe::gemm2_blocks(H);
    g.gate_up = 0;
    g.a_is_out_row = 1;
    g.rows_per_expert = H;
    g.epi = moe::EPI_GATE_F32;
    g.out = y;
    g.ldo = H;
    g.out_rows = RS;
    g.out_cols = H;
    g.row_gate = row_gate;
    g.err = err_flag;
    g.wait_limit_ns = moe::kDefaultWaitLimitNs;
    e = pow2   ? moe::launch_gemm_mx(g, st)
        : pair ? moe::launch_gemm_pair(g, st)
        : tall ? moe::launch_gemm_tall(g, st)
               : moe::launch_gemm(g, st);
  }
  if (e == cudaSuccess) e = prof_mark(5, st);
  if (e == cudaSuccess) e = moe::launch_combine(P.x_resid, y, pos, T, H, Kr, R, Ns, P.out, P.out_f32, st, true);
  if (e == cudaSuccess) e = prof_mark(6, st);
  return e;
}

int moe_forward(const moe_config *cfg, const moe_weights *w, const float *bias, const void *x, int64_t T, void *out,
                int32_t out_dtype, int32_t *idx_out, int32_t *counts_out, void *ws, size_t ws_bytes,
                int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("moe_forward");
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_DTYPE_BF16 && out_dtype != MOE_DTYPE_F32) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (counts_out) {
      if (const int d = check_device()) return d;
      return cuda_status(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * cfg->n_routed, st));
    }
    return MOE_OK;
  }
  if (!w || !bias || !x || !out || !ws || !err_flag) return MOE_ERR_INVALID_ARG;
  if (!w->w13_dev || !w->s13_dev || !w->w2_dev || !w->s2_dev || !w->wr_dev) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned16(w->w13_dev) || !aligned16(w->w2_dev) || !aligned16(w->wr_dev) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  if (!aligned4(w->s13_dev) || !aligned4(w->s2_dev) || !aligned4(bias) || !aligned4(err_flag) ||
      !aligned4(idx_out) || !aligned4(counts_out))
    return MOE_ERR_INVALID_ARG;
  moe_ws_layout L;
  make_layout(cfg, T, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;

  const int H = cfg->hidden, Nr = cfg->n_routed, Kr = cfg->top_k;
  uint8_t *xq = at<uint8_t *>(ws, L.xq);
  float *xs = at<float *>(ws, L.xs);
  int32_t *idx = at<int32_t *>(ws, L.idx);
  float *gate = at<float *>(ws, L.gate);
  float *logits = at<float *>(ws, L.logits);
  const int ks = moe::router_ksplit(T, Nr, H);

  cudaError_t e = prof_mark(0, st);
  const bool pow2 = cfg->scale_mode == MOE_SCALE_POW2;
  if (e == cudaSuccess) e = moe::launch_quant_1x128(x, T, H, H, xq, xs, st, pow2);
  if (e == cudaSuccess) e = prof_mark(1, st);
  if (e == cudaSuccess)
    e = moe::launch_router_logits(x, w->wr_dev, T, Nr, H, logits, err_flag, moe::kDefaultWaitLimitNs, st);
  if (e == cudaSuccess)
    e = moe::launch_router_topk(logits, ks, T, Nr, Kr, cfg->n_groups, cfg->topk_groups, cfg->route_scale, bias,
                                idx, gate, nullptr, st);
  if (e == cudaSuccess) e = prof_mark(2, st);
  if (e == cudaSuccess) {
    ExpertPath P{};
    P.cfg = cfg;
    P.w = w;
    P.T = T;
    P.xq = xq;
    P.xq_ld = H;
    P.xs = xs;
    P.idx = idx;
    P.gate = gate;
    P.allow_empty = 0;
    P.x_resid = x;
    P.out = out;
    P.out_f32 = out_dtype == MOE_DTYPE_F32;
    P.counts_out = counts_out;
    P.L = &L;
    P.ws = ws;
    P.err = err_flag;
    P.st = st;
    e = run_expert_path(P);
  }
  if (e == cudaSuccess && idx_out)
    e = cudaMemcpyAsync(idx_out, idx, sizeof(int32_t) * T * Kr, cudaMemcpyDeviceToDevice, st);
  return cuda_status(e);
}

// ------------------------------------------------------ expert parallelism
int64_t moe_ep_row_bytes(const moe_config *cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  const int64_t H = cfg->hidden, Kr = cfg->top_k;
  return (H + 4 * (H / 128) + 8 * Kr + 15) / 16 * 16;
}

static void ep_dispatch_layout(int32_t world, int64_t T, size_t *cnt_off, size_t *base_off, size_t *total) {
  const int64_t nblk = (T + 255) / 256;
  Carve cv;
  size_t a[2], b[2];
  cv.take(a, static_cast<size_t>(nblk) * world * 4);
  cv.take(b, static_cast<size_t>(nblk) * world * 4);
  *cnt_off = a[0];
  *base_off = b[0];
  *total = (cv.off + 255) & ~size_t(255);
}

size_t moe_ep_dispatch_workspace_size(const moe_config *cfg, int32_t world, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || world < 1 || world > 64 || cfg->n_routed % world || T < 0 || T > kMaxTokens)
    return 0;
  size_t c, b, tot;
  ep_dispatch_layout(world, T, &c, &b, &tot);
  return tot < 256 ? 256 : tot;
}

int moe_ep_dispatch(const moe_config *cfg, int32_t world, const uint8_t *xq, const float *xs, const int32_t *idx,
                    const float *gate, int64_t T, uint8_t *send_rows, int64_t send_cap_rows, int32_t *send_counts,
                    int32_t *send_offsets, int32_t *row_of, uint8_t *self_rows, void *ws, size_t ws_bytes,
                    int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("moe_ep_dispatch");
  if (const int c = check_cfg(cfg)) return c;
  if (world < 1 || world > 64 || cfg->n_routed % world) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  const int64_t Kr = cfg->top_k;
  if (send_cap_rows < T * (world < Kr ? world : Kr)) return MOE_ERR_INVALID_ARG;
  if (!send_counts || !send_offsets || !ws || !err_flag) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!xq || !xs || !idx || !gate || !send_rows || !row_of)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(send_rows) || !aligned16(self_rows) || !aligned4(xs) || !aligned4(idx) ||
      !aligned4(gate) || !aligned4(send_counts) || !aligned4(send_offsets) || !aligned4(row_of) ||
      !aligned4(err_flag) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_ep_dispatch_workspace_size(cfg, world, T)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  size_t c_off, b_off, tot;
  ep_dispatch_layout(world, T, &c_off, &b_off, &tot);
  auto *w8 = static_cast<uint8_t *>(ws);
  return cuda_status(moe::launch_ep_dispatch(
      xq, xs, idx, gate, T, cfg->hidden, cfg->top_k, cfg->n_routed, world, reinterpret_cast<int32_t *>(w8 + c_off),
      reinterpret_cast<int32_t *>(w8 + b_off), send_counts, send_offsets, row_of, send_rows, moe_ep_row_bytes(cfg),
      self_rows, err_flag, static_cast<cudaStream_t>(stream)));
}

size_t moe_ep_experts_workspace_size(const moe_config *cfg_local, int64_t n_rows) {
  if (check_cfg_local(cfg_local) != MOE_OK || n_rows < 0 || n_rows > kMaxTokens) return 0;
  moe_ws_layout L;
  make_layout(cfg_local, n_rows, &L);
  return L.total < 256 ? 256 : L.total;
}

int moe_ep_experts(const moe_config *cfg_local, const moe_weights *w_local, const uint8_t *rows, int64_t n_rows,
                   int64_t row_bytes, void *partial_out, void *ws, size_t ws_bytes, int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("moe_ep_experts");
  if (const int c = check_cfg_local(cfg_local)) return c;
  if (n_rows < 0 || n_rows > kMaxTokens) return MOE_ERR_INVALID_ARG;
  const int64_t H = cfg_local->hidden, Kr = cfg_local->top_k;
  if (row_bytes != (H + 4 * (H / 128) + 8 * Kr + 15) / 16 * 16) return MOE_ERR_INVALID_ARG;
  if (n_rows == 0) return MOE_OK;
  if (!w_local || !rows || !partial_out || !ws || !err_flag) return MOE_ERR_INVALID_ARG;
  if (!w_local->w13_dev || !w_local->s13_dev || !w_local->w2_dev || !w_local->s2_dev) return MOE_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(partial_out) || !aligned16(w_local->w13_dev) || !aligned16(w_local->w2_dev) ||
      !aligned4(w_local->s13_dev) || !aligned4(w_local->s2_dev) || !aligned4(err_flag) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  moe_ws_layout L;
  make_layout(cfg_local, n_rows, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t *idx = at<int32_t *>(ws, L.idx);
  float *gate = at<float *>(ws, L.gate);
  float *xs = at<float *>(ws, L.xs);
  cudaError_t e = moe::launch_ep_unpack(rows, n_rows, row_bytes, cfg_local->hidden, cfg_local->top_k,
                                        cfg_local->n_routed, idx, gate, xs, err_flag, st);
  if (e == cudaSuccess) {
    ExpertPath P{};
    P.cfg = cfg_local;
    P.w = w_local;
    P.T = n_rows;
    P.xq = rows;
    P.xq_ld = row_bytes;
    P.xs = xs;
    P.idx = idx;
    P.gate = gate;
    P.allow_empty = 1;
    P.x_resid = nullptr;
    P.out = partial_out;
    P.out_f32 = 0;
    P.counts_out = nullptr;
    P.L = &L;
    P.ws = ws;
    P.err = err_flag;
    P.st = st;
    e = run_expert_path(P);
  }
  return cuda_status(e);
}

int moe_ep_combine(const moe_config *cfg, int32_t world, const void *x, int64_t T, const int32_t *row_of,
                   const void *back, const void *y_shared, void *out, int32_t out_dtype, void *stream) {
  const NvtxRange nvtx_call("moe_ep_combine");
  if (const int c = check_cfg(cfg)) return c;
  if (world < 1 || world > 64 || T < 0 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_DTYPE_BF16 && out_dtype != MOE_DTYPE_F32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !row_of || !back || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(back) || !aligned16(y_shared) || !aligned16(out) || !aligned4(row_of))
    return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  return cuda_status(moe::launch_ep_combine(x, y_shared, back, row_of, T, world, cfg->hidden, out,
                                            out_dtype == MOE_DTYPE_F32, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ backward
namespace {
struct BwdLayout {
  size_t gu[2], dyq[2], dys[2], dh[2], gh[2], dgu[2], dguq[2], dgus[2], dxr[2];
  size_t counts[2], offsets[2], blk_base[2], chunks[2], meta[2];
  size_t seg[2], tiles[2], tmeta[2];
  size_t dyt[2], sdy[2], ht[2], sh[2], dgut[2], sdgu[2], xt[2], sx[2];
  int64_t P, max_tiles;
  size_t total;
};

void make_bwd_layout(const moe_config *c, int64_t T, BwdLayout *B) {
  const int64_t H = c->hidden, I = c->inter, Nr = c->n_routed, Kr = c->top_k, Ns = c->n_shared;
  const int64_t R = T * Kr, RS = R + T * Ns, E = Nr + Ns;
  const int64_t pitch = moe::scale_pitch(R, T);
  const int64_t nblk = (T + 127) / 128;
  B->P = (RS + 128 * E + 127) / 128 * 128;
  B->max_tiles = RS / 128 + E;
  Carve cv;
  cv.take(B->gu, RS * 2 * I * 4);
  cv.take(B->dyq, RS * H);
  cv.take(B->dys, ((H / 128) * pitch + moe::kScaleSlack) * 4);
  cv.take(B->dh, RS * I * 4);
  cv.take(B->gh, RS * I * 4);
  cv.take(B->dgu, RS * 2 * I * 4);
  cv.take(B->dguq, RS * 2 * I);
  cv.take(B->dgus, ((2 * I / 128) * pitch + moe::kScaleSlack) * 4);
  cv.take(B->dxr, RS * H * 4);
  cv.take(B->counts, Nr * 4);
  cv.take(B->offsets, (Nr + 1) * 4);
  cv.take(B->blk_base, nblk * Nr * 4);
  cv.take(B->chunks, moe::max_chunks(T, static_cast<int>(Kr), static_cast<int>(Nr), static_cast<int>(Ns)) * 16);
  cv.take(B->meta, 4 * 4);
  cv.take(B->seg, (E + 1) * 4);
  cv.take(B->tiles, B->max_tiles * 16);
  cv.take(B->tmeta, 4 * 4);
  cv.take(B->dyt, H * B->P);
  cv.take(B->sdy, (B->P / 128) * H * 4);
  cv.take(B->ht, I * B->P);
  cv.take(B->sh, (B->P / 128) * I * 4);
  cv.take(B->dgut, 2 * I * B->P);
  cv.take(B->sdgu, (B->P / 128) * 2 * I * 4);
  cv.take(B->xt, H * B->P);
  cv.take(B->sx, (B->P / 128) * H * 4);
  B->total = (cv.off + 255) & ~size_t(255);
}
}  // namespace

int moe_transpose_weights(const moe_config *cfg, const moe_weights *w, uint8_t *w13t, float *s13t, uint8_t *w2t,
                          float *s2t, void *stream) {
  if (const int c = check_cfg(cfg)) return c;
  if (!w || !w->w13_dev || !w->s13_dev || !w->w2_dev || !w->s2_dev || !w13t || !s13t || !w2t || !s2t)
    return MOE_ERR_INVALID_ARG;
  if (!aligned4(w->s13_dev) || !aligned4(w->s2_dev) || !aligned4(s13t) || !aligned4(s2t)) return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  const int64_t E = static_cast<int64_t>(cfg->n_routed) + cfg->n_shared, H = cfg->hidden, I = cfg->inter;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = moe::launch_transpose_blocks(w->w13_dev, w->s13_dev, 2 * I, H, E, w13t, s13t, st);
  if (e == cudaSuccess) e = moe::launch_transpose_blocks(w->w2_dev, w->s2_dev, H, I, E, w2t, s2t, st);
  return cuda_status(e);
}

int moe_backward_workspace_layout(const moe_config *cfg, int64_t T, moe_bwd_layout *out) {
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens || !out) return MOE_ERR_INVALID_ARG;
  BwdLayout B;
  make_bwd_layout(cfg, T, &B);
  auto cp = [](size_t (&d)[2], const size_t (&s_)[2]) {
    d[0] = s_[0];
    d[1] = s_[1];
  };
  cp(out->gu, B.gu);
  cp(out->dh, B.dh);
  cp(out->gh, B.gh);
  cp(out->dgu, B.dgu);
  cp(out->dx_rows, B.dxr);
  cp(out->seg, B.seg);
  out->P = B.P;
  out->total = B.total;
  return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_config *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0 || T > kMaxTokens) return 0;
  BwdLayout B;
  make_bwd_layout(cfg, T, &B);
  return B.total;
}

int moe_backward(const moe_config *cfg, const moe_weights *w, const uint8_t *w13t, const float *s13t,
                 const uint8_t *w2t, const float *s2t, const void *x, const void *dout, int64_t T, float *dx,
                 float *dW13, float *dW2, const void *fwd_ws, size_t fwd_ws_bytes, void *ws, size_t ws_bytes,
                 int32_t *err_flag, void *stream) {
  const NvtxRange nvtx_call("moe_backward");
  if (const int c = check_cfg(cfg)) return c;
  if (cfg->scale_mode != MOE_SCALE_AMAX) return MOE_ERR_NOT_IMPLEMENTED;
  if (T < 1 || T > kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (!w || !w->w13_dev || !w->s13_dev || !w->w2_dev || !w->s2_dev || !w13t || !s13t || !w2t || !s2t || !x ||
      !dout || !dx || !dW13 || !dW2 || !fwd_ws || !ws || !err_flag)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dout) || !aligned16(dx) || !aligned16(dW13) || !aligned16(dW2) ||
      !aligned16(w13t) || !aligned16(w2t) || !aligned4(s13t) || !aligned4(s2t) || !aligned4(err_flag) ||
      (reinterpret_cast<uintptr_t>(ws) & 255) || (reinterpret_cast<uintptr_t>(fwd_ws) & 255))
    return MOE_ERR_INVALID_ARG;
  moe_ws_layout L;
  make_layout(cfg, T, &L);
  if (fwd_ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  BwdLayout B;
  make_bwd_layout(cfg, T, &B);
  if (ws_bytes < B.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void *fws = const_cast<void *>(fwd_ws);
  const int H = cfg->hidden, I = cfg->inter, Nr = cfg->n_routed, Kr = cfg->top_k, Ns = cfg->n_shared;
  const int64_t R = T * Kr, RS = R + T * Ns, E = static_cast<int64_t>(Nr) + Ns;
  const int64_t pitch = moe::scale_pitch(R, T);
  // the forward's intermediates this backward reads
  const uint8_t *xq = at<uint8_t *>(fws, L.xq);
  const uint8_t *ap = at<uint8_t *>(fws, L.ap);
  const float *as_t = at<float *>(fws, L.as);
  const int32_t *pos = at<int32_t *>(fws, L.pos);
  const int32_t *row_src = at<int32_t *>(fws, L.row_src);
  const float *row_gate = at<float *>(fws, L.row_gate);
  const int32_t *blk_hist = at<int32_t *>(fws, L.blk_hist);
  // this backward's own buffers
  float *GU = at<float *>(ws, B.gu);
  uint8_t *dyq = at<uint8_t *>(ws, B.dyq);
  float *dys = at<float *>(ws, B.dys);
  float *dh = at<float *>(ws, B.dh);
  float *ghbuf = at<float *>(ws, B.gh);
  float *dGU = at<float *>(ws, B.dgu);
  uint8_t *dGUq = at<uint8_t *>(ws, B.dguq);
  float *dGUs = at<float *>(ws, B.dgus);
  float *dxr = at<float *>(ws, B.dxr);
  int32_t *counts = at<int32_t *>(ws, B.counts);
  int32_t *offsets = at<int32_t *>(ws, B.offsets);
  int32_t *blk_base = at<int32_t *>(ws, B.blk_base);
  int4 *chunks = at<int4 *>(ws, B.chunks);
  int32_t *meta = at<int32_t *>(ws, B.meta);
  int32_t *seg = at<int32_t *>(ws, B.seg);
  int4 *tiles = at<int4 *>(ws, B.tiles);
  int32_t *tmeta = at<int32_t *>(ws, B.tmeta);
  const int64_t max_chunks = moe::max_chunks(T, Kr, Nr, Ns);

  // 128-row chunks of the forward's expert grouping (the single-CTA GEMM)
  cudaError_t e = prof_mark_bwd(0, st);
  if (e == cudaSuccess)
    e = moe::launch_build_chunks(blk_hist, T, Kr, Nr, Ns, 128, counts, offsets, blk_base, chunks, meta,
                                           nullptr, st);
  auto base_gemm = [&](moe::GemmLaunch &g) {
    g.chunks = chunks;
    g.n_chunks = meta;
    g.max_chunks = static_cast<int>(max_chunks);
    g.chunk_rows = 128;
    g.sa_transposed = 1;
    g.sa_ld = pitch;
    g.err = err_flag;
    g.wait_limit_ns = moe::kDefaultWaitLimitNs;
  };
  if (e == cudaSuccess) {
    // G, U again: the forward's gate/up GEMM with FP32 outputs
    moe::GemmLaunch g{};
    base_gemm(g);
    g.w = w->w13_dev;
    g.w_rows = E * 2 * I;
    g.a0 = ap;
    g.a0_rows = R;
    g.a1 = Ns ? xq : ap;
    g.a1_rows = Ns ? T : R;
    g.K = H;
    g.sw = w->s13_dev;
    g.sa0 = as_t;
    g.sa1 = as_t;
    g.nb = moe::gemm1_blocks(I);
    g.gate_up = 1;
    g.half = I;
    g.rows_per_expert = 2 * static_cast<int64_t>(I);
    g.epi = moe::EPI_F32;
    g.out = GU;
    g.ldo = 2 * I;
    g.out_rows = RS;
    g.out_cols = 2 * I;
    e = moe::launch_gemm(g, st);
  }
  if (e == cudaSuccess) e = prof_mark_bwd(1, st);
  if (e == cudaSuccess) e = moe::launch_dout_quant(dout, row_src, R, RS, H, dyq, dys, pitch, st);
  if (e == cudaSuccess) {
    // dh = g (dout W2): K = H against W2^T [E, I, H], the row's gate in the
    // FP32 epilogue
    moe::GemmLaunch g{};
    base_gemm(g);
    g.w = w2t;
    g.w_rows = E * I;
    g.a0 = dyq;
    g.a0_rows = RS;
    g.a1 = dyq;
    g.a1_rows = RS;
    g.K = H;
    g.sw = s2t;
    g.sa0 = dys;
    g.sa1 = dys;
    g.nb = moe::gemm2_blocks(I);
    g.gate_up = 0;
    g.a_is_out_row = 1;
    g.rows_per_expert = I;
    g.epi = moe::EPI_GATE_F32;
    g.row_gate = row_gate;
    g.out = dh;
    g.ldo = I;
    g.out_rows = RS;
    g.out_cols = I;
    e = moe::launch_gemm(g, st);
  }
  if (e == cudaSuccess) e = prof_mark_bwd(2, st);
  if (e == cudaSuccess) e = moe::launch_swiglu_bwd(GU, dh, row_gate, RS, I, ghbuf, dGU, dGUq, dGUs, pitch, st);
  if (e == cudaSuccess) e = prof_mark_bwd(3, st);
  if (e == cudaSuccess) {
    // dx rows = [dG|dU] [W1; W3] (FP32): K = 2I against W13^T [E, H, 2I]
    moe::GemmLaunch g{};
    base_gemm(g);
    g.w = w13t;
    g.w_rows = E * H;
    g.a0 = dGUq;
    g.a0_rows = RS;
    g.a1 = dGUq;
    g.a1_rows = RS;
    g.K = 2 * I;
    g.sw = s13t;
    g.sa0 = dGUs;
    g.sa1 = dGUs;
    g.nb = moe::gemm2_blocks(H);
    g.gate_up = 0;
    g.a_is_out_row = 1;
    g.rows_per_expert = H;
    g.epi = moe::EPI_F32;
    g.out = dxr;
    g.ldo = H;
    g.out_rows = RS;
    g.out_cols = H;
    e = moe::launch_gemm(g, st);
  }
  // dx_t = dout_t + the token's rows (shared, then its slots), FP32
  if (e == cudaSuccess) e = prof_mark_bwd(4, st);
  if (e == cudaSuccess) e = moe::launch_combine(dout, dxr, pos, T, H, Kr, R, Ns, dx, 1, st, true);
  if (e == cudaSuccess) e = prof_mark_bwd(5, st);
  // weight gradients: 128-token tiles of every expert, operands transposed
  if (e == cudaSuccess) e = moe::launch_wgrad_tiles(offsets, Nr, Ns, R, T, seg, tiles, tmeta, st);
  const int mt = static_cast<int>(B.max_tiles);
  if (e == cudaSuccess)
    e = moe::launch_colquant(1, tiles, tmeta, mt, nullptr, 0, dout, row_src, R, H, at<uint8_t *>(ws, B.dyt), B.P,
                             at<float *>(ws, B.sdy), st);
  if (e == cudaSuccess)
    e = moe::launch_colquant(0, tiles, tmeta, mt, ghbuf, I, nullptr, row_src, R, I, at<uint8_t *>(ws, B.ht), B.P,
                             at<float *>(ws, B.sh), st);
  if (e == cudaSuccess)
    e = moe::launch_colquant(0, tiles, tmeta, mt, dGU, 2 * I, nullptr, row_src, R, 2 * I,
                             at<uint8_t *>(ws, B.dgut), B.P, at<float *>(ws, B.sdgu), st);
  if (e == cudaSuccess)
    e = moe::launch_colquant(1, tiles, tmeta, mt, nullptr, 0, x, row_src, R, H, at<uint8_t *>(ws, B.xt), B.P,
                             at<float *>(ws, B.sx), st);
  if (e == cudaSuccess) e = prof_mark_bwd(6, st);
  if (e == cudaSuccess) {
    moe::WgradLaunch g{};
    g.a_t = at<uint8_t *>(ws, B.dyt);
    g.b_t = at<uint8_t *>(ws, B.ht);
    g.sa_t = at<float *>(ws, B.sdy);
    g.sb_t = at<float *>(ws, B.sh);
    g.seg = seg;
    g.E = static_cast<int>(E);
    g.C_out = H;
    g.C_in = I;
    g.P = B.P;
    g.out = dW2;
    g.err = err_flag;
    g.wait_limit_ns = moe::kDefaultWaitLimitNs;
    e = moe::launch_gemm_wgrad(g, st);
  }
  if (e == cudaSuccess) e = prof_mark_bwd(7, st);
  if (e == cudaSuccess) {
    moe::WgradLaunch g{};
    g.a_t = at<uint8_t *>(ws, B.dgut);
    g.b_t = at<uint8_t *>(ws, B.xt);
    g.sa_t = at<float *>(ws, B.sdgu);
    g.sb_t = at<float *>(ws, B.sx);
    g.seg = seg;
    g.E = static_cast<int>(E);
    g.C_out = 2 * I;
    g.C_in = H;
    g.P = B.P;
    g.out = dW13;
    g.err = err_flag;
    g.wait_limit_ns = moe::kDefaultWaitLimitNs;
    e = moe::launch_gemm_wgrad(g, st);
  }
  if (e == cudaSuccess) e = prof_mark_bwd(8, st);
  return cuda_status(e);
}

int moe_seq_balance_loss(const moe_config *cfg, int64_t T, int64_t seq_len, float alpha, const void *ws,
                         size_t ws_bytes, float *loss, int32_t *err_flag, void *stream) {
  if (const int c = check_cfg(cfg)) return c;
  if (T < 0 || T > kMaxTokens || seq_len < 1 || !(alpha == alpha)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (T % seq_len) return MOE_ERR_INVALID_ARG;
  if (!ws || !loss || !err_flag || (reinterpret_cast<uintptr_t>(ws) & 255) || !aligned4(loss) ||
      !aligned4(err_flag))
    return MOE_ERR_INVALID_ARG;
  moe_ws_layout L;
  make_layout(cfg, T, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (const int d = check_device()) return d;
  void *w = const_cast<void *>(ws);
  const int ks = moe::router_ksplit(T, cfg->n_routed, cfg->hidden);
  return cuda_status(moe::launch_seq_balance(at<const float *>(w, L.logits), ks, T, cfg->n_routed,
                                             at<const int32_t *>(w, L.idx), cfg->top_k, seq_len, alpha, loss,
                                             err_flag, static_cast<cudaStream_t>(stream)));
}

int moe_profile_events(void *const *events, int32_t n_events) {
  if (!events || n_events <= 0) {
    g_prof_on = false;
    g_prof_bwd_on = false;
    return MOE_OK;
  }
  if (n_events < MOE_PROFILE_EVENTS) return MOE_ERR_INVALID_ARG;
  const int n = n_events >= MOE_PROFILE_EVENTS + MOE_PROFILE_BWD_EVENTS ? MOE_PROFILE_EVENTS + MOE_PROFILE_BWD_EVENTS
                                                                       : MOE_PROFILE_EVENTS;
  for (int i = 0; i < n; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) g_prof_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_prof_on = true;
  g_prof_bwd_on = n > MOE_PROFILE_EVENTS;
  return MOE_OK;
}

int moe_bias_update(float *bias, const int32_t *counts, int32_t n_routed, int64_t total, float gamma,
                    void *stream) {
  if (!bias || !counts || n_routed <= 0 || total < 0 || !aligned4(bias) || !aligned4(counts))
    return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  return cuda_status(moe::launch_bias_update(bias, counts, n_routed, total, gamma, static_cast<cudaStream_t>(stream)));
}

int moe_check_device_error(const int32_t *err_flag, int32_t *host_value, void *stream) {
  if (!err_flag) return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  int32_t v = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&v, err_flag, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (host_value) *host_value = v;
  if (v == 0) return MOE_OK;
  return (v & MOE_DEVERR_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE;
}

int moe_selftest_wait_timeout(int32_t *err_flag, int64_t limit_us, void *stream) {
  if (!err_flag || limit_us < 1 || limit_us > 1000000) return MOE_ERR_INVALID_ARG;
  if (const int d = check_device()) return d;
  return cuda_status(
      moe::launch_wait_selftest(err_flag, static_cast<uint64_t>(limit_us) * 1000ull, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
