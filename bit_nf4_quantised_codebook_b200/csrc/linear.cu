// linear.cu — QLoRA linear forward / backward launch plans on top of the
// tcgen05 GEMM template, plus the split-reduction finalize kernels.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §The QLoRA layer, end to end (forward/backward listing), with W stored
// [N, K], A = L1 [K, r], B = L2 [r, N]:
//   forward : T = X·A;  sT = bf16(s·T);  Y = X·W_hatᵀ + sT·B
//   backward: U = dY·Bᵀ; sU = bf16(s·U);  dX = dY·W_hat + sU·Aᵀ;
//             dA = Xᵀ·sU;  dB = sTᵀ·dY
// The two big products run in the dequant GEMM (W_hat built in shared memory,
// never in HBM), with the LoRA product appended as extra K steps into the same
// TMEM accumulator.  The four skinny products (output width r) run in the same
// GEMM template with both operands streamed by TMA and the long reduction split
// across the CTAs of a thread-block cluster, summed in rank order through
// distributed shared memory (no partial buffers, no extra launch).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_smallm.cuh"
#include "internal.h"
#include "launch.cuh"
#include "linear_plan.h"

namespace qlora {

// ---------------------------------------------------------------- kernel configurations
using CfgFwd = GemmCfg<256, 4, false, B_DQ_K, LORA_B2_MN, OUT_BF16>;
using CfgFwdSplit = GemmCfg<256, 4, false, B_DQ_K, LORA_B2_MN, OUT_F32>;
using CfgBwd = GemmCfg<256, 4, false, B_DQ_MN, LORA_B2_K, OUT_BF16>;
using CfgBwdSplit = GemmCfg<256, 4, false, B_DQ_MN, LORA_B2_K, OUT_F32>;
// skinny: output width r_pad (16..256); K splits reduced inside a cluster
template <int BN>
using CfgT = GemmCfg<BN, 4, false, B_TMA_MN, LORA_NONE, OUT_RED_BF16>;  // s·X·A   (X K-major, Aᵀ MN-major)
template <int BN>
using CfgU = GemmCfg<BN, 4, false, B_TMA_K, LORA_NONE, OUT_RED_BF16>;   // s·dY·Bᵀ (B K-major)
template <int BN>
using CfgDA = GemmCfg<BN, 4, true, B_TMA_MN, LORA_NONE, OUT_RED_F32>;   // Xᵀ·sU   (both MN-major)
template <int BN>
using CfgDB = GemmCfg<BN, 4, true, B_TMA_MN, LORA_NONE, OUT_RED_F32_T>; // (dYᵀ·sT)ᵀ written as dB

template <class C>
static cudaError_t prepare() {
  static std::atomic<uint64_t> done{0};
  return smem_attr_once(reinterpret_cast<const void *>(gemm_kernel<C>), C::SMEM_BYTES, done);
}

template <class C>
static cudaError_t launch(dim3 grid, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  cudaError_t e = prepare<C>();
  if (e != cudaSuccess) return e;
  return launch_k_ordered(gemm_kernel<C>, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, st, 1, m.a, m.b, m.a2, m.b2,
                          p);
}

// Launch with clusters of 1 x 1 x cz CTAs (the K splits of one output tile).
template <class C>
static cudaError_t launch_cluster(dim3 grid, int cz, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  cudaError_t e = prepare<C>();
  if (e != cudaSuccess) return e;
  return launch_k_ordered(gemm_kernel<C>, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, st, static_cast<unsigned>(cz), m.a,
                  m.b, m.a2, m.b2, p);
}

using PairFwd = PairCfg<4, B_DQ_K, LORA_B2_MN, OUT_BF16, 2>;
using PairFwdSplit = PairCfg<4, B_DQ_K, LORA_B2_MN, OUT_F32, 2>;
using PairBwd = PairCfg<4, B_DQ_MN, LORA_B2_K, OUT_BF16, 2>;
using PairBwdSplit = PairCfg<4, B_DQ_MN, LORA_B2_K, OUT_F32, 2>;
constexpr int kPairTokens = 2 * 128 * 2;  // tokens per CTA pair (2 CTAs x MSUB x 128)

template <class C>
static cudaError_t launch_pair(dim3 grid, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = smem_attr_once(reinterpret_cast<const void *>(gemm_pair_kernel<C>), C::SMEM_BYTES, prepared);
  if (e != cudaSuccess) return e;
  return launch_k_ordered(gemm_pair_kernel<C>, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, st, 1, m.a, m.b, m.a2,
                          m.b2, p);
}

// ---------------------------------------------------------------- finalize kernels
// out[row, c] = cvt(scale * sum_s part[s][row][c]), c < cols, sequential over s.
__global__ void k_finalize_bf16(const float *__restrict__ part, int splits, int64_t split_stride, int64_t rows,
                                int cols, int ldp, float scale, uint16_t *__restrict__ out, int64_t ldo) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nvec = rows * (cols / 4);
  if (idx >= nvec) return;
  const int64_t row = idx / (cols / 4);
  const int c = static_cast<int>(idx % (cols / 4)) * 4;
  float4 acc = *reinterpret_cast<const float4 *>(part + row * ldp + c);
  for (int s = 1; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4 *>(part + s * split_stride + row * ldp + c);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * scale, acc.y * scale);
  pk.y = pack_bf16x2(acc.z * scale, acc.w * scale);
  *reinterpret_cast<uint2 *>(out + row * ldo + c) = pk;
}

static cudaError_t finalize_bf16(const float *part, int splits, int64_t split_stride, int64_t rows, int cols,
                                 int ldp, float scale, uint16_t *out, int64_t ldo, cudaStream_t st) {
  const int64_t n = rows * (cols / 4);
  const int64_t grid = (n + 255) / 256;
  return launch_k(k_finalize_bf16, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, 1,
                  static_cast<const float *>(part), splits, split_stride, rows, cols, ldp, scale, out, ldo);
}
// ---------------------------------------------------------------- skinny GEMM dispatch over r buckets
enum SkinnyKind { SK_T = 0, SK_U = 1, SK_DA = 2, SK_DB = 3 };

template <template <int> class CF>
static cudaError_t launch_bucket(int rpad, dim3 grid, int cz, const TmaMaps &m, const GemmParams &p,
                                 cudaStream_t st) {
  switch (rpad) {
    case 16: return launch_cluster<CF<16>>(grid, cz, m, p, st);
    case 32: return launch_cluster<CF<32>>(grid, cz, m, p, st);
    case 64: return launch_cluster<CF<64>>(grid, cz, m, p, st);
    case 128: return launch_cluster<CF<128>>(grid, cz, m, p, st);
    case 256: return launch_cluster<CF<256>>(grid, cz, m, p, st);
    default: return cudaErrorInvalidValue;
  }
}

static GemmParams base_params(const LaunchCtx &c) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.dev_err = c.dev_err;
  p.timeout_ns = c.timeout_ns;
  p.lv = c.levels;
  p.k_shr16 = 1u << 16;
  p.k_shr1 = 1u << 31;
  p.cluster = 1;
  p.scale = 1.0f;
  return p;
}

// Skinny product: D[rows x r] = scale · sum over the reduction of Aop·Bopᵀ, the
// reduction split over the sp.splits CTAs of one cluster and summed in-cluster.
// Writes out[row][c] (ld_out) or, for SK_DB, out[c][row].
static cudaError_t run_skinny(SkinnyKind kind, const LaunchCtx &c, const SplitPlan &sp, int rpad, int r, int rows,
                              float scale, const TmaMaps &maps, void *out, int64_t ld_out, bool trigger = false) {
  GemmParams p = base_params(c);
  p.trigger_dependents = trigger ? 1 : 0;
  p.rows = rows;
  p.cols = rpad;
  p.k_iters = sp.k_iters;
  p.k_iters_total = sp.k_iters_total;
  p.out = out;
  p.ld_out = ld_out;
  p.cluster = sp.splits;
  p.red_cols = r;
  p.scale = scale;
  dim3 grid(static_cast<unsigned>((rows + 127) / 128), 1, static_cast<unsigned>(sp.splits));
  switch (kind) {
    case SK_T: return launch_bucket<CfgT>(rpad, grid, sp.splits, maps, p, c.stream);
    case SK_U: return launch_bucket<CfgU>(rpad, grid, sp.splits, maps, p, c.stream);
    case SK_DA: return launch_bucket<CfgDA>(rpad, grid, sp.splits, maps, p, c.stream);
    default: return launch_bucket<CfgDB>(rpad, grid, sp.splits, maps, p, c.stream);
  }
}

// ---------------------------------------------------------------- fused dequant GEMM
#ifndef QLORA_RASTER_GROUP
#define QLORA_RASTER_GROUP 4
#endif
// Token-pair tiles per raster group of the CTA-pair kernel (0: the launch
// grid's order).  The 74 CTA pairs resident at a time then cover about 4 token
// tiles x 18 W tiles: a wave reads 4 activation tiles (1 KiB per reduction
// index each) and 18 W tiles (about 133 bytes per reduction index each) from
// DRAM, close to the minimum of 1024·a + 133·b over a·b = 74 (a ≈ 3); the
// grid's own order (all 16 token tiles of M = 8192 with 4-5 W tiles) reads
// about 2.6 times as much.  Consecutive waves of a group share its activation
// tiles, which L2 keeps when they fit.
constexpr int kRasterGroup = QLORA_RASTER_GROUP;

// fwd: D[M x N] = X·W_hatᵀ + sT·B       (W-side operand K-major: rows of W)
// bwd: D[M x K] = dY·W_hat + sU·Aᵀ      (W-side operand MN-major: columns of W)
// `pair` selects the CTA-pair kernel (256-token tiles); otherwise one CTA per
// 128-token tile.  With sp.splits > 1 the K range is split and float32 partials
// go to `part` before a fixed-order reduction.
static cudaError_t run_fused(bool fwd, const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *act, int64_t M,
                             const uint16_t *lora_a, const uint16_t *lora_b, int r, uint16_t *out, bool pair,
                             const SplitPlan &sp, float *part, cudaEvent_t ev0, cudaEvent_t ev1) {
  cudaError_t e;
  const int N = static_cast<int>(w.N), K = static_cast<int>(w.K);
  const int n_out = fwd ? N : K;
  const int red = fwd ? K : N;
  TmaMaps m;
  bool ok = map_bf16_kmajor(&m.a, act, red, M, 128) && map_bf16_kmajor(&m.a2, lora_a, r, M, 128);
  if (fwd) {
    ok = ok && map_codes(&m.b, w.codes, N, K, 32, pair ? 128 : 256, 0) && map_bf16_mn(&m.b2, lora_b, N, r);
  } else {
    ok = ok && (pair ? map_codes(&m.b, w.codes, N, K, 64, 64, 64) : map_codes(&m.b, w.codes, N, K, 128, 64, 0)) &&
         map_bf16_kmajor(&m.b2, lora_b, r, K, pair ? 128 : 256);
  }
  if (!ok) return cudaErrorInvalidValue;
  GemmParams p = base_params(c);
  p.rows = static_cast<int>(M);
  p.cols = n_out;
  p.k_iters = sp.k_iters;
  p.k_iters_total = sp.k_iters_total;
  p.lora_r = r;
  p.c2q = w.c2q;
  p.c1 = w.c1;
  p.mean = w.mean;
  p.w_rows = N;
  p.w_kblocks = K / 64;
  p.ld_out = n_out;
  const bool split = sp.splits > 1;
  p.out = split ? static_cast<void *>(part) : static_cast<void *>(out);
  p.split_stride = M * n_out;
  const unsigned gx = pair ? static_cast<unsigned>(2 * ((M + kPairTokens - 1) / kPairTokens))
                           : static_cast<unsigned>((M + 127) / 128);
  if (pair && kRasterGroup > 0) {
    const int tmp = static_cast<int>(gx / 2);
    p.raster_gm = kRasterGroup < tmp ? kRasterGroup : tmp;
  }
  dim3 grid(gx, static_cast<unsigned>((n_out + 255) / 256), static_cast<unsigned>(sp.splits));
  if (ev0) cudaEventRecord(ev0, c.stream);
  if (pair) {
    if (fwd) e = split ? launch_pair<PairFwdSplit>(grid, m, p, c.stream) : launch_pair<PairFwd>(grid, m, p, c.stream);
    else e = split ? launch_pair<PairBwdSplit>(grid, m, p, c.stream) : launch_pair<PairBwd>(grid, m, p, c.stream);
  } else {
    if (fwd) e = split ? launch<CfgFwdSplit>(grid, m, p, c.stream) : launch<CfgFwd>(grid, m, p, c.stream);
    else e = split ? launch<CfgBwdSplit>(grid, m, p, c.stream) : launch<CfgBwd>(grid, m, p, c.stream);
  }
  if (e != cudaSuccess) return e;
  if (ev1) cudaEventRecord(ev1, c.stream);
  if (split) return finalize_bf16(part, sp.splits, M * n_out, M, n_out, n_out, 1.0f, out, n_out, c.stream);
  return cudaSuccess;
}

// ---------------------------------------------------------------- small-M forward
#ifndef QLORA_SMALL_GROUPS
#define QLORA_SMALL_GROUPS 2
#endif
constexpr int kSmallGroups = QLORA_SMALL_GROUPS;  // dequant groups of 4 warps per CTA

template <class C>
static cudaError_t launch_small(dim3 grid, int cz, const TmaMaps &m, const SmallParams &p, cudaStream_t st) {
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = smem_attr_once(reinterpret_cast<const void *>(gemm_smallm_kernel<C>), C::SMEM_BYTES, prepared);
  if (e != cudaSuccess) return e;
  return launch_k(gemm_smallm_kernel<C>, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, st, static_cast<unsigned>(cz),
                  m.a, m.b, m.a2, m.b2, p);
}

// Y = X·W_hatᵀ + sT·B for M <= 64 tokens: W rows on the MMA M side, tokens on N.
static cudaError_t run_small_forward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, int64_t M,
                                     const uint16_t *sT, const uint16_t *B, int r, uint16_t *Y, const SplitPlan &sp,
                                     cudaEvent_t ev0, cudaEvent_t ev1) {
  const int N = static_cast<int>(w.N), K = static_cast<int>(w.K);
  const int nt = static_cast<int>((M + 15) / 16) * 16;
  TmaMaps m;  // a = X, b = codes, a2 = sT, b2 = B
  const int crow = nt == 64 ? 32 : 64;  // code bytes per W row and pipeline step (SmallCfg::C_ROW)
  static_assert(SmallCfg<64, kSmallGroups>::C_ROW == 32 && SmallCfg<48, kSmallGroups>::C_ROW == 64, "code box");
  if (!map_bf16_kmajor(&m.a, X, K, M, nt) || !map_codes(&m.b, w.codes, N, K, crow, 128, crow) ||
      !map_bf16_kmajor(&m.a2, sT, r, M, nt) || !map_bf16_mn(&m.b2, B, N, r))
    return cudaErrorInvalidValue;
  SmallParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = static_cast<int>(M);
  p.N = N;
  p.k_iters = sp.k_iters;
  p.k_iters_total = sp.k_iters_total;
  p.splits = sp.splits;
  int words = (sp.k_iters + 3) / 4;
  if (words % 2 == 0) ++words;  // odd word stride: 32 consecutive rows hit 32 banks
  p.q8_stride = 4 * words;
  p.q8_words = (sp.k_iters_total % 4 == 0 && sp.k_iters % 4 == 0) ? 1 : 0;
  p.lora_r = r;
  p.c2q = w.c2q;
  p.c1 = w.c1;
  p.mean = w.mean;
  p.lv = c.levels;
  p.k_shr16 = 1u << 16;
  p.k_shr1 = 1u << 31;
  p.Y = Y;
  p.dev_err = c.dev_err;
  p.timeout_ns = c.timeout_ns;
  const dim3 grid(static_cast<unsigned>((N + 127) / 128), 1, static_cast<unsigned>(sp.splits));
  if (ev0) cudaEventRecord(ev0, c.stream);
  cudaError_t e;
  switch (nt) {
    case 16: e = launch_small<SmallCfg<16, kSmallGroups>>(grid, sp.splits, m, p, c.stream); break;
    case 32: e = launch_small<SmallCfg<32, kSmallGroups>>(grid, sp.splits, m, p, c.stream); break;
    case 48: e = launch_small<SmallCfg<48, kSmallGroups>>(grid, sp.splits, m, p, c.stream); break;
    case 64: e = launch_small<SmallCfg<64, kSmallGroups>>(grid, sp.splits, m, p, c.stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if (ev1) cudaEventRecord(ev1, c.stream);
  return cudaSuccess;
}

// ---------------------------------------------------------------- forward
// sT = bf16(s·X·A)  (A-op X [M,K] K-major; B-op Aᵀ: A [K,r] read MN-major)
static cudaError_t run_t(const LaunchCtx &c, const uint16_t *X, int64_t M, int K, const uint16_t *A, int r, float s,
                         uint16_t *sT, const LinearPlan &pl, bool trigger) {
  TmaMaps m;
  if (!map_bf16_kmajor(&m.a, X, K, M, 128) || !map_bf16_mn(&m.b, A, r, K)) return cudaErrorInvalidValue;
  m.a2 = m.a;
  m.b2 = m.b;
  return run_skinny(SK_T, c, pl.sp_t, pl.rpad, r, static_cast<int>(M), s, m, sT, r, trigger);
}

cudaError_t run_forward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, int64_t M,
                        const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *T_save,
                        const LinearPlan &pl, uint8_t *ws) {
  cudaError_t e;
  const int K = static_cast<int>(w.K);
  uint16_t *sT = T_save ? T_save : reinterpret_cast<uint16_t *>(ws + pl.off_sT);
  // the small-M forward that follows overlaps this grid's tail; the CTA-pair GEMM does not (gemm.cuh)
  if ((e = run_t(c, X, M, K, A, r, s, sT, pl, pl.small_main)) != cudaSuccess) return e;
  // Y = X·W_hatᵀ + sT·B
  const TimingHooks &hk = timing_hooks();
  if (pl.small_main) return run_small_forward(c, w, X, M, sT, B, r, Y, pl.sp_main, hk.fwd_begin, hk.fwd_end);
  float *part = reinterpret_cast<float *>(ws + pl.off_main_part);
  return run_fused(true, c, w, X, M, sT, B, r, Y, pl.pair_main, pl.sp_main, part, hk.fwd_begin, hk.fwd_end);
}

// ---------------------------------------------------------------- backward
cudaError_t run_backward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, const uint16_t *dY,
                         int64_t M, const uint16_t *A, const uint16_t *B, int r, float s, const uint16_t *T_saved,
                         uint16_t *dX, float *dA, float *dB, const LinearPlan &pl, uint8_t *ws) {
  cudaError_t e;
  const int N = static_cast<int>(w.N), K = static_cast<int>(w.K);
  const uint16_t *sT = T_saved;
  if (!sT) {  // recompute bf16(s·X·A)
    uint16_t *sT_ws = reinterpret_cast<uint16_t *>(ws + pl.off_sT);
    if ((e = run_t(c, X, M, K, A, r, s, sT_ws, pl, false)) != cudaSuccess) return e;
    sT = sT_ws;
  }
  uint16_t *sU = reinterpret_cast<uint16_t *>(ws + pl.off_sU);
  // sU = bf16(s·dY·Bᵀ)  (A-op dY [M,N] K-major; B-op B [r,N] K-major)
  {
    TmaMaps m;
    if (!map_bf16_kmajor(&m.a, dY, N, M, 128) || !map_bf16_kmajor(&m.b, B, N, r, pl.rpad))
      return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_U, c, pl.sp_u, pl.rpad, r, static_cast<int>(M), s, m, sU, r)) != cudaSuccess) return e;
  }
  // dX = dY·W_hat + sU·Aᵀ
  if (dX) {
    const TimingHooks &hk = timing_hooks();
    float *part = reinterpret_cast<float *>(ws + pl.off_main_part);
    if ((e = run_fused(false, c, w, dY, M, sU, A, r, dX, pl.pair_dx, pl.sp_dx, part, hk.bwd_begin, hk.bwd_end)) !=
        cudaSuccess)
      return e;
  }
  // dA = Xᵀ·sU : D[K x r] (A-op Xᵀ: X [M,K] MN-major; B-op sUᵀ: sU [M,r] MN-major)
  {
    TmaMaps m;
    if (!map_bf16_mn(&m.a, X, K, M) || !map_bf16_mn(&m.b, sU, r, M)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_DA, c, pl.sp_da, pl.rpad, r, K, 1.0f, m, dA, r)) != cudaSuccess) return e;
  }
  // dB = sTᵀ·dY : D[N x r] = dYᵀ·sT, written transposed into dB [r, N]
  {
    TmaMaps m;
    if (!map_bf16_mn(&m.a, dY, N, M) || !map_bf16_mn(&m.b, sT, r, M)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_DB, c, pl.sp_db, pl.rpad, r, N, 1.0f, m, dB, N)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qlora
