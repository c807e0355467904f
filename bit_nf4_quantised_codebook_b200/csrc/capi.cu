// capi.cu — the extern "C" boundary: argument validation, workspace layout,
// tensor maps, and dispatch to the quantiser and the linear-layer launches.
// Nothing here allocates device memory or synchronises the caller's stream.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>
#include "internal.h"
#include "linear_plan.h"
#include "nf4_decode.cuh"

namespace qlora {
namespace {

struct Globals {
  float levels[16];
  float thresholds[15];
  unsigned long long timeout_ns = 2000000000ull;  // 2 s per pipeline wait
};

Globals &globals() {
  static Globals g;
  static std::once_flag once;
  std::call_once(once, [] {
    build_codebook_f32(g.levels, g.thresholds);
    if (const char *env = std::getenv("QLORA_WAIT_TIMEOUT_MS")) {
      const long long ms = std::atoll(env);
      if (ms > 0) g.timeout_ns = static_cast<unsigned long long>(ms) * 1000000ull;
    }
  });
  return g;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


SplitPlan choose(int64_t tiles, int64_t k_total, int target_ctas, int min_iters) {
  SplitPlan sp;
  sp.k_iters_total = static_cast<int>(k_total);
  int64_t s = std::max<int64_t>(1, target_ctas / std::max<int64_t>(1, tiles));
  s = std::min<int64_t>(s, std::max<int64_t>(1, k_total / std::max(1, min_iters)));
  const int64_t kps = (k_total + s - 1) / s;
  sp.k_iters = static_cast<int>(kps);
  sp.splits = static_cast<int>((k_total + kps - 1) / kps);
  return sp;
}

// K splits of a skinny product, run as one cluster per output tile: a power of
// two up to 8 (the portable cluster size), at least two K steps per split.
SplitPlan choose_cluster(int64_t tiles, int64_t k_total, int target_ctas) {
  SplitPlan sp;
  sp.k_iters_total = static_cast<int>(k_total);
  int s = 1;
  while (s < 8 && tiles * s * 2 <= target_ctas && k_total >= 4 * s) s *= 2;
  sp.splits = s;
  sp.k_iters = static_cast<int>((k_total + s - 1) / s);
  return sp;
}

// K splits of the small-M forward (one cluster of S <= 8 CTAs per 128 W rows).
// The decode's integer work sets the time, and an SM decodes at about the same
// rate with one or two resident CTAs, so the cost is the weight blocks of the
// busiest SM: ceil(tiles·S / SMs) CTAs of kps blocks each.  Clusters of more than
// 4 CTAs measured slower (co-scheduling and the 8-way reduction) and are used only
// where K needs them.  Ties go to more splits (two CTAs per SM hide more latency
// than one: 8192² at 64 tokens ran 34.9 µs with 4 splits, 36.1 µs with 2).
SplitPlan choose_small(int64_t N, int64_t k_total, int num_sms) {
  SplitPlan best;
  best.k_iters_total = static_cast<int>(k_total);
  const int64_t tiles = (N + 127) / 128, sms = num_sms > 0 ? num_sms : 1;
  int64_t best_cost = -1;
  for (int pass = 0; pass < 2 && best_cost < 0; ++pass) {
    for (int s = 1; s <= (pass == 0 ? 4 : 8); ++s) {
      int64_t kps = (k_total + s - 1) / s;
      if (k_total % 4 == 0) kps = (kps + 3) / 4 * 4;  // splits start on 4-byte boundaries of a constants row
      if (kps > kSmallMaxKIters) continue;
      if (s > 1 && (s - 1) * kps >= k_total) continue;  // a split would have no work
      const int64_t cost = (tiles * s + sms - 1) / sms * kps;
      if (best_cost < 0 || cost <= best_cost) {
        best_cost = cost;
        best.splits = s;
        best.k_iters = static_cast<int>(kps);
      }
    }
  }
  return best;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

bool device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status check_weight(const qlora_nf4_weight *w) {
  if (!w || !w->codes || !w->c2q || !w->c1 || !w->mean) return QLORA_ERR_INVALID_ARG;
  if (w->N < 1 || w->K < 64) return QLORA_ERR_INVALID_ARG;
  if (w->K % 64 != 0 || w->N > (1ll << 30) || w->K > (1ll << 30) || w->N * w->K > (1ll << 40))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w->codes) || !aligned16(w->c2q) || !aligned16(w->c1) || !aligned16(w->mean))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

qlora_status check_linear(const qlora_nf4_weight *w, int64_t M, int r) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  if (M < 1 || r < 1) return QLORA_ERR_INVALID_ARG;
  if (r % 8 != 0 || r > 256 || w->N % 8 != 0 || M > (1ll << 30)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

std::atomic<uint64_t> g_launches{0};
TimingHooks g_hooks;

}  // namespace

thread_local int t_last_cuda_error = 0;

qlora_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QLORA_OK;
  t_last_cuda_error = static_cast<int>(e);
  return QLORA_ERR_CUDA;
}

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
const TimingHooks &timing_hooks() { return g_hooks; }

LinearPlan make_plan(int op, int64_t M, int64_t N, int64_t K, int r, int num_sms) {
  LinearPlan pl;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  if (op == QLORA_OP_QUANTIZE || op == QLORA_OP_MERGE) {
    const int64_t nb = N * K / 64;
    const int64_t ng = (nb + 255) / 256;
    int64_t size = 1;
    while (size < ng) size *= 2;
    pl.gsum_size = size;
    pl.off_absmax = take(static_cast<size_t>(nb) * 4);
    pl.off_gsum = take(static_cast<size_t>(size) * 8);
    pl.bytes = off;
    return pl;
  }
  pl.rpad = r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : r <= 128 ? 128 : 256;
  const int64_t mt = (M + 127) / 128;
  pl.sp_t = choose_cluster(mt, K / 64, 2 * num_sms);
  pl.off_sT = take(static_cast<size_t>(M) * r * 2);
  if (op == QLORA_OP_FORWARD) {
    if (M <= kSmallMaxTokens && K / 64 <= 8 * kSmallMaxKIters) {
      pl.small_main = true;
      pl.sp_main = choose_small(N, K / 64, num_sms);
      pl.bytes = off;
      return pl;
    }
    pl.pair_main = M > 128;
    pl.sp_main = choose((pl.pair_main ? 2 * ((M + 511) / 512) : mt) * ((N + 255) / 256), K / 64, num_sms, 4);
    if (pl.sp_main.splits > 1) pl.off_main_part = take(static_cast<size_t>(pl.sp_main.splits) * M * N * 4);
  } else {
    pl.sp_u = choose_cluster(mt, (N + 63) / 64, 2 * num_sms);
    pl.pair_dx = M > 128;
    pl.sp_dx = choose((pl.pair_dx ? 2 * ((M + 511) / 512) : mt) * ((K + 255) / 256), (N + 63) / 64, num_sms, 4);
    pl.sp_da = choose_cluster((K + 127) / 128, (M + 63) / 64, 2 * num_sms);
    pl.sp_db = choose_cluster((N + 127) / 128, (M + 63) / 64, 2 * num_sms);
    pl.off_sU = take(static_cast<size_t>(M) * r * 2);
    if (pl.sp_dx.splits > 1) pl.off_main_part = take(static_cast<size_t>(pl.sp_dx.splits) * M * K * 4);
  }
  pl.bytes = off;
  return pl;
}

bool map_bf16_kmajor(CUtensorMap *m, const void *ptr, int64_t inner, int64_t outer, int box_rows) {
  return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, inner, outer, inner * 2, 64, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}
bool map_bf16_mn(CUtensorMap *m, const void *ptr, int64_t inner, int64_t outer) {
  return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, inner, outer, inner * 2, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}
bool map_codes(CUtensorMap *m, const void *codes, int64_t N, int64_t K, int box_bytes, int box_rows,
               int swizzle_bytes) {
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  return encode_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, box_bytes, box_rows, sw);
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char *qlora_last_cuda_error(int *code) {
  if (code) *code = t_last_cuda_error;
  return t_last_cuda_error ? cudaGetErrorString(static_cast<cudaError_t>(t_last_cuda_error)) : "no error";
}

const char *qlora_status_string(qlora_status st) {
  switch (st) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QLORA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_NO_DEVICE: return "current device is not sm_100";
    case QLORA_ERR_TOO_LARGE: return "weight larger than the static scratch of qlora_quantize_noalloc (N*K <= 2^26)";
  }
  return "unknown status";
}

qlora_status qlora_build_codebook(float levels[16], float thresholds[15]) {
  build_codebook_f32(levels, thresholds);
  return QLORA_OK;
}

qlora_status qlora_nf4_sizes(int64_t N, int64_t K, size_t *codes_bytes, size_t *c2q_bytes, size_t *c1_bytes) {
  if (N < 1 || K < 64) return QLORA_ERR_INVALID_ARG;
  if (K % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t nb = N * K / 64;
  if (codes_bytes) *codes_bytes = static_cast<size_t>(N * K / 2);
  if (c2q_bytes) *c2q_bytes = static_cast<size_t>(nb);
  if (c1_bytes) *c1_bytes = static_cast<size_t>((nb + 255) / 256) * 4;
  return QLORA_OK;
}

qlora_status qlora_workspace_size(int op, int64_t M, int64_t N, int64_t K, int r, size_t *bytes) {
  if (!bytes || N < 1 || K < 64) return QLORA_ERR_INVALID_ARG;
  if (K % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (op < QLORA_OP_QUANTIZE || op > QLORA_OP_MERGE) return QLORA_ERR_INVALID_ARG;
  if (op == QLORA_OP_FORWARD || op == QLORA_OP_BACKWARD) {
    if (M < 1 || r < 1) return QLORA_ERR_INVALID_ARG;
    if (r % 8 != 0 || r > 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  }
  *bytes = make_plan(op, M, N, K, r, device_sms()).bytes;
  return QLORA_OK;
}

qlora_status qlora_quantize(const uint16_t *W, const qlora_nf4_weight *out, void *ws, size_t ws_bytes, int *dev_err,
                            void *stream) {
  if (!W) return QLORA_ERR_INVALID_ARG;
  qlora_status st = check_weight(out);
  if (st != QLORA_OK) return st;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const LinearPlan pl = make_plan(QLORA_OP_QUANTIZE, 0, out->N, out->K, 0, device_sms());
  if (!ws || ws_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  Globals &g = globals();
  Nf4Thresholds thr;
  std::memcpy(thr.t, g.thresholds, sizeof(thr.t));
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const int64_t nb = out->N * out->K / 64;
  cudaError_t e = launch_quantize(W, nb, out->codes, out->c2q, out->c1, out->mean,
                                  reinterpret_cast<float *>(w8 + pl.off_absmax),
                                  reinterpret_cast<double *>(w8 + pl.off_gsum), pl.gsum_size, thr, dev_err,
                                  static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

qlora_status qlora_dequantize(const qlora_nf4_weight *w, uint16_t *W_out, void *stream) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  Globals &g = globals();
  Nf4Levels lv;
  std::memcpy(lv.q, g.levels, sizeof(lv.q));
  cudaError_t e = launch_dequantize(w->codes, w->c2q, w->c1, w->mean, w->N * w->K / 64, lv, W_out,
                                    static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

// True when [a, a+na) and [b, b+nb) share a byte.
static bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

qlora_status qlora_merge_requantize(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const qlora_nf4_weight *out, uint16_t *W_merged, void *ws, size_t ws_bytes,
                                    int *dev_err, void *stream) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  if ((st = check_weight(out)) != QLORA_OK) return st;
  if (!A || !B || out->N != w->N || out->K != w->K || r < 1) return QLORA_ERR_INVALID_ARG;
  if (r % 8 != 0 || r > 256 || w->N % 8 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(A) || !aligned16(B) || (W_merged && !aligned16(W_merged))) return QLORA_ERR_MISALIGNED;
  const int64_t nb = w->N * w->K / 64;
  const size_t in_sz[4] = {static_cast<size_t>(w->N * w->K / 2), static_cast<size_t>(nb),
                           static_cast<size_t>((nb + 255) / 256) * 4, 4};
  const void *in_p[4] = {w->codes, w->c2q, w->c1, w->mean};
  const void *out_p[4] = {out->codes, out->c2q, out->c1, out->mean};
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 4; ++j)
      if (!(i == j && in_p[i] == out_p[j]) && overlap(in_p[i], in_sz[i], out_p[j], in_sz[j]))
        return QLORA_ERR_INVALID_ARG;
  if (W_merged)
    for (int i = 0; i < 4; ++i)
      if (overlap(W_merged, static_cast<size_t>(w->N * w->K) * 2, in_p[i], in_sz[i]) ||
          overlap(W_merged, static_cast<size_t>(w->N * w->K) * 2, out_p[i], in_sz[i]))
        return QLORA_ERR_INVALID_ARG;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const LinearPlan pl = make_plan(QLORA_OP_MERGE, 0, w->N, w->K, r, device_sms());
  if (!ws || ws_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  Globals &g = globals();
  Nf4Levels lv;
  std::memcpy(lv.q, g.levels, sizeof(lv.q));
  Nf4Thresholds thr;
  std::memcpy(thr.t, g.thresholds, sizeof(thr.t));
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const cudaError_t e = launch_merge_requantize(*w, A, B, r, s, *out, W_merged,
                                                reinterpret_cast<float *>(w8 + pl.off_absmax),
                                                reinterpret_cast<double *>(w8 + pl.off_gsum), pl.gsum_size, lv, thr,
                                                dev_err, g.timeout_ns, static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

// ---------------------------------------------------------------- format variants
static qlora_status check_format(const qlora_format *f) {
  if (!f || f->codebook < QLORA_CB_NF4 || f->codebook > QLORA_CB_FP4_E3M0 || f->dq < QLORA_DQ_NONE ||
      f->dq > QLORA_DQ_INT8)
    return QLORA_ERR_INVALID_ARG;
  if (f->block != 32 && f->block != 64 && f->block != 128 && f->block != 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

static qlora_status check_format_shape(const qlora_format *f, int64_t N, int64_t K) {
  qlora_status st = check_format(f);
  if (st != QLORA_OK) return st;
  if (N < 1 || K < 1) return QLORA_ERR_INVALID_ARG;
  if (K % f->block != 0 || N > (1ll << 30) || K > (1ll << 30) || N * K > (1ll << 40))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

static qlora_status check_qweight(const qlora_qweight *w) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  qlora_status st = check_format_shape(&w->fmt, w->N, w->K);
  if (st != QLORA_OK) return st;
  if (!w->codes || !w->consts || (w->fmt.dq != QLORA_DQ_NONE && (!w->c1 || !w->mean))) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(w->codes) || !aligned16(w->consts) || (w->c1 && !aligned16(w->c1)) ||
      (w->mean && !aligned16(w->mean)))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Workspace of the format quantiser: float32 absmax per block, then the
// power-of-two padded float64 group sums.
static void format_ws_layout(int64_t nb, size_t *off_gsum, int64_t *gsum_size, size_t *bytes) {
  const int64_t ng = (nb + 255) / 256;
  int64_t size = 1;
  while (size < ng) size *= 2;
  *off_gsum = align256(static_cast<size_t>(nb) * 4);
  *gsum_size = size;
  *bytes = align256(*off_gsum + static_cast<size_t>(size) * 8);
}

qlora_status qlora_format_codebook(int codebook, float levels[16], float thresholds[15]) {
  return build_format_codebook_f32(codebook, levels, thresholds) ? QLORA_OK : QLORA_ERR_INVALID_ARG;
}

qlora_status qlora_format_sizes(const qlora_format *fmt, int64_t N, int64_t K, size_t *codes_bytes,
                                size_t *consts_bytes, size_t *c1_bytes) {
  qlora_status st = check_format_shape(fmt, N, K);
  if (st != QLORA_OK) return st;
  const int64_t nb = N * K / fmt->block;
  if (codes_bytes) *codes_bytes = static_cast<size_t>(N * K / 2);
  if (consts_bytes) *consts_bytes = static_cast<size_t>(nb) * (fmt->dq == QLORA_DQ_NONE ? 4 : 1);
  if (c1_bytes) *c1_bytes = fmt->dq == QLORA_DQ_NONE ? 0 : static_cast<size_t>((nb + 255) / 256) * 4;
  return QLORA_OK;
}

qlora_status qlora_format_workspace_size(const qlora_format *fmt, int64_t N, int64_t K, size_t *bytes) {
  if (!bytes) return QLORA_ERR_INVALID_ARG;
  qlora_status st = check_format_shape(fmt, N, K);
  if (st != QLORA_OK) return st;
  size_t off;
  int64_t size;
  format_ws_layout(N * K / fmt->block, &off, &size, bytes);
  return QLORA_OK;
}

qlora_status qlora_quantize_format(const uint16_t *W, const qlora_qweight *w, void *ws, size_t ws_bytes,
                                   int *dev_err, void *stream) {
  if (!W) return QLORA_ERR_INVALID_ARG;
  qlora_status st = check_qweight(w);
  if (st != QLORA_OK) return st;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  size_t off_gsum, need;
  int64_t gsum_size;
  format_ws_layout(w->N * w->K / w->fmt.block, &off_gsum, &gsum_size, &need);
  if (!ws || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  float levels[16], thr[15];
  build_format_codebook_f32(w->fmt.codebook, levels, thr);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const cudaError_t e = launch_quantize_format(W, *w, levels, thr, reinterpret_cast<float *>(w8),
                                               reinterpret_cast<double *>(w8 + off_gsum), gsum_size, dev_err,
                                               static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

qlora_status qlora_dequantize_format(const qlora_qweight *w, uint16_t *W_out, void *stream) {
  qlora_status st = check_qweight(w);
  if (st != QLORA_OK) return st;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  float levels[16];
  build_format_codebook_f32(w->fmt.codebook, levels, nullptr);
  const cudaError_t e = launch_dequantize_format(*w, levels, W_out, static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

qlora_status qlora_quant_error(const uint16_t *W, const uint16_t *W_hat, int64_t n, double *stats, void *stream) {
  if (!W || !W_hat || !stats || n < 1) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(W_hat) || (reinterpret_cast<uintptr_t>(stats) & 7u) != 0)
    return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const cudaError_t e = launch_quant_error(W, W_hat, n, stats, device_sms(), static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

static LaunchCtx make_ctx(int *dev_err, void *stream) {
  Globals &g = globals();
  LaunchCtx c;
  c.stream = static_cast<cudaStream_t>(stream);
  c.dev_err = dev_err;
  c.timeout_ns = g.timeout_ns;
  std::memcpy(c.levels.q, g.levels, sizeof(c.levels.q));
  return c;
}

qlora_status qlora_linear_forward(const qlora_nf4_weight *w, const uint16_t *X, int64_t M, const uint16_t *A,
                                  const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *T_save, void *ws,
                                  size_t ws_bytes, int *dev_err, void *stream) {
  qlora_status st = check_linear(w, M, r);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || (T_save && !aligned16(T_save)))
    return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const LinearPlan pl = make_plan(QLORA_OP_FORWARD, M, w->N, w->K, r, device_sms());
  if (!ws || ws_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  cudaError_t e = run_forward(make_ctx(dev_err, stream), *w, X, M, A, B, r, s, Y, T_save, pl,
                              static_cast<uint8_t *>(ws));
  return cuda_status(e);
}

qlora_status qlora_linear_backward(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY, int64_t M,
                                   const uint16_t *A, const uint16_t *B, int r, float s, const uint16_t *T_saved,
                                   uint16_t *dX, float *dA, float *dB, void *ws, size_t ws_bytes, int *dev_err,
                                   void *stream) {
  qlora_status st = check_linear(w, M, r);
  if (st != QLORA_OK) return st;
  if (!X || !dY || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB) ||
      (dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved)))
    return QLORA_ERR_MISALIGNED;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const LinearPlan pl = make_plan(QLORA_OP_BACKWARD, M, w->N, w->K, r, device_sms());
  if (!ws || ws_bytes < pl.bytes) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  cudaError_t e = run_backward(make_ctx(dev_err, stream), *w, X, dY, M, A, B, r, s, T_saved, dX, dA, dB, pl,
                               static_cast<uint8_t *>(ws));
  return cuda_status(e);
}

uint64_t qlora_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

qlora_status qlora_adamw_step(const qlora_adamw_tensor *tensors, int count, float lr, float beta1, float beta2,
                              float eps, float weight_decay, int64_t step, void *stream) {
  if (!tensors || count < 1 || count > QLORA_ADAMW_MAX_TENSORS || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!(lr >= 0.f) || !(weight_decay >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) ||
      !(eps > 0.f))
    return QLORA_ERR_INVALID_ARG;
  for (int k = 0; k < count; ++k) {
    const qlora_adamw_tensor &t = tensors[k];
    if (!t.param || !t.grad || !t.m || !t.v || t.n < 1) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(t.param) || !aligned16(t.grad) || !aligned16(t.m) || !aligned16(t.v) ||
        (t.param_bf16 && !aligned16(t.param_bf16)))
      return QLORA_ERR_MISALIGNED;
  }
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  const double bc1 = 1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step));
  if (!(bc1 > 0.0) || !(bc2 > 0.0)) return QLORA_ERR_INVALID_ARG;
  cudaError_t e = launch_adamw(tensors, count, lr, beta1, beta2, eps, weight_decay, static_cast<double>(lr) / bc1,
                               std::sqrt(bc2), device_sms(), static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

qlora_status qlora_selftest_bounded_wait(unsigned timeout_us, int *dev_err, int *gave_up, void *stream) {
  if (!dev_err || timeout_us == 0 || timeout_us > 10000000u) return QLORA_ERR_INVALID_ARG;
  if (!device_ok()) return QLORA_ERR_NO_DEVICE;
  cudaError_t e = launch_selftest_wait(static_cast<unsigned long long>(timeout_us) * 1000ull, dev_err, gave_up,
                                       static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

qlora_status qlora_set_timing_events(void *fwd_begin, void *fwd_end, void *bwd_begin, void *bwd_end) {
  g_hooks.fwd_begin = static_cast<cudaEvent_t>(fwd_begin);
  g_hooks.fwd_end = static_cast<cudaEvent_t>(fwd_end);
  g_hooks.bwd_begin = static_cast<cudaEvent_t>(bwd_begin);
  g_hooks.bwd_end = static_cast<cudaEvent_t>(bwd_end);
  return QLORA_OK;
}

}  // extern "C"
