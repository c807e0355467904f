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
// across CTAs; partial sums are reduced in a fixed order by finalize kernels.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "internal.h"
#include "linear_plan.h"

namespace qlora {

// ---------------------------------------------------------------- kernel configurations
using CfgFwd = GemmCfg<256, 4, false, B_DQ_K, LORA_B2_MN, OUT_BF16>;
using CfgFwdSplit = GemmCfg<256, 4, false, B_DQ_K, LORA_B2_MN, OUT_F32>;
using CfgBwd = GemmCfg<256, 4, false, B_DQ_MN, LORA_B2_K, OUT_BF16>;
using CfgBwdSplit = GemmCfg<256, 4, false, B_DQ_MN, LORA_B2_K, OUT_F32>;
// skinny: output width r_pad (16..256); instantiated for the r buckets below
template <int BN>
using CfgT = GemmCfg<BN, 4, false, B_TMA_MN, LORA_NONE, OUT_F32>;  // X·A        (A-op X K-major, B-op Aᵀ MN-major)
template <int BN>
using CfgU = GemmCfg<BN, 4, false, B_TMA_K, LORA_NONE, OUT_F32>;   // dY·Bᵀ      (B-op B K-major)
template <int BN>
using CfgW = GemmCfg<BN, 4, true, B_TMA_MN, LORA_NONE, OUT_F32>;   // Xᵀ·sU, dYᵀ·sT (both MN-major)

template <class C>
static cudaError_t prepare() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e == cudaSuccess) done = true;
  return e;
}

template <class C>
static cudaError_t launch(dim3 grid, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  cudaError_t e = prepare<C>();
  if (e != cudaSuccess) return e;
  gemm_kernel<C><<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(m.a, m.b, m.a2, m.b2, p);
  count_launches(1);
  return cudaGetLastError();
}

using PairFwd = PairCfg<4, B_DQ_K, LORA_B2_MN, OUT_BF16, 2>;
using PairFwdSplit = PairCfg<4, B_DQ_K, LORA_B2_MN, OUT_F32, 2>;
using PairBwd = PairCfg<4, B_DQ_MN, LORA_B2_K, OUT_BF16, 2>;
using PairBwdSplit = PairCfg<4, B_DQ_MN, LORA_B2_K, OUT_F32, 2>;
constexpr int kPairTokens = 2 * 128 * 2;  // tokens per CTA pair (2 CTAs x MSUB x 128)

template <class C>
static cudaError_t launch_pair(dim3 grid, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  static bool prepared = false;
  if (!prepared) {
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    prepared = true;
  }
  gemm_pair_kernel<C><<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(m.a, m.b, m.a2, m.b2, p);
  count_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- finalize kernels
// out[row, c] = cvt(scale * sum_s part[s][row][c]), c < cols, sequential over s.
__global__ void k_finalize_bf16(const float *__restrict__ part, int splits, int64_t split_stride, int64_t rows,
                                int cols, int ldp, float scale, uint16_t *__restrict__ out, int64_t ldo) {
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

__global__ void k_finalize_f32(const float *__restrict__ part, int splits, int64_t split_stride, int64_t rows,
                               int cols, int ldp, float scale, float *__restrict__ out, int64_t ldo) {
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
  acc.x *= scale;
  acc.y *= scale;
  acc.z *= scale;
  acc.w *= scale;
  *reinterpret_cast<float4 *>(out + row * ldo + c) = acc;
}

// out[c, row] = scale * sum_s part[s][row][c]   (transposing finalize, 32x32 tiles)
__global__ void k_finalize_f32_t(const float *__restrict__ part, int splits, int64_t split_stride, int64_t rows,
                                 int cols, int ldp, float scale, float *__restrict__ out, int64_t ldo) {
  __shared__ float tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int c0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t row = r0 + i;
    const int c = c0 + threadIdx.x;
    float acc = 0.f;
    if (row < rows && c < cols) {
      acc = part[row * ldp + c];
      for (int s = 1; s < splits; ++s) acc += part[s * split_stride + row * ldp + c];
    }
    tile[i][threadIdx.x] = acc * scale;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i;
    const int64_t row = r0 + threadIdx.x;
    if (row < rows && c < cols) out[static_cast<int64_t>(c) * ldo + row] = tile[threadIdx.x][i];
  }
}

static cudaError_t finalize_bf16(const float *part, int splits, int64_t split_stride, int64_t rows, int cols,
                                 int ldp, float scale, uint16_t *out, int64_t ldo, cudaStream_t st) {
  const int64_t n = rows * (cols / 4);
  const int64_t grid = (n + 255) / 256;
  k_finalize_bf16<<<static_cast<unsigned>(grid), 256, 0, st>>>(part, splits, split_stride, rows, cols, ldp, scale,
                                                                 out, ldo);
  count_launches(1);
  return cudaGetLastError();
}
static cudaError_t finalize_f32(const float *part, int splits, int64_t split_stride, int64_t rows, int cols, int ldp,
                                float scale, float *out, int64_t ldo, cudaStream_t st) {
  const int64_t n = rows * (cols / 4);
  const int64_t grid = (n + 255) / 256;
  k_finalize_f32<<<static_cast<unsigned>(grid), 256, 0, st>>>(part, splits, split_stride, rows, cols, ldp, scale, out,
                                                                ldo);
  count_launches(1);
  return cudaGetLastError();
}
static cudaError_t finalize_f32_t(const float *part, int splits, int64_t split_stride, int64_t rows, int cols,
                                  int ldp, float scale, float *out, int64_t ldo, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((rows + 31) / 32), static_cast<unsigned>((cols + 31) / 32));
  k_finalize_f32_t<<<grid, dim3(32, 8), 0, st>>>(part, splits, split_stride, rows, cols, ldp, scale, out, ldo);
  count_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- skinny GEMM dispatch over r buckets
enum SkinnyKind { SK_T = 0, SK_U = 1, SK_W = 2 };

template <template <int> class CF>
static cudaError_t launch_bucket(int rpad, dim3 grid, const TmaMaps &m, const GemmParams &p, cudaStream_t st) {
  switch (rpad) {
    case 16: return launch<CF<16>>(grid, m, p, st);
    case 32: return launch<CF<32>>(grid, m, p, st);
    case 64: return launch<CF<64>>(grid, m, p, st);
    case 128: return launch<CF<128>>(grid, m, p, st);
    case 256: return launch<CF<256>>(grid, m, p, st);
    default: return cudaErrorInvalidValue;
  }
}

static cudaError_t launch_skinny(SkinnyKind kind, int rpad, dim3 grid, const TmaMaps &m, const GemmParams &p,
                                 cudaStream_t st) {
  switch (kind) {
    case SK_T: return launch_bucket<CfgT>(rpad, grid, m, p, st);
    case SK_U: return launch_bucket<CfgU>(rpad, grid, m, p, st);
    default: return launch_bucket<CfgW>(rpad, grid, m, p, st);
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
  return p;
}

// Skinny product: D[rows x rpad] = sum over `red` (split) of Aop·Bopᵀ, written as
// float32 partials [splits][rows][rpad] into `part`.
static cudaError_t run_skinny(SkinnyKind kind, const LaunchCtx &c, const SplitPlan &sp, int rpad, int rows,
                              const TmaMaps &maps, float *part) {
  GemmParams p = base_params(c);
  p.rows = rows;
  p.cols = rpad;
  p.k_iters = sp.k_iters;
  p.k_iters_total = sp.k_iters_total;
  p.out = part;
  p.ld_out = rpad;
  p.split_stride = static_cast<int64_t>(rows) * rpad;
  dim3 grid(static_cast<unsigned>((rows + 127) / 128), 1, static_cast<unsigned>(sp.splits));
  return launch_skinny(kind, rpad, grid, maps, p, c.stream);
}

// ---------------------------------------------------------------- fused dequant GEMM
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
    ok = ok && map_codes(&m.b, w.codes, N, K, 32, pair ? 128 : 256, false) && map_bf16_mn(&m.b2, lora_b, N, r);
  } else {
    ok = ok && (pair ? map_codes(&m.b, w.codes, N, K, 64, 64, true) : map_codes(&m.b, w.codes, N, K, 128, 64, false)) &&
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

// ---------------------------------------------------------------- forward
cudaError_t run_forward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, int64_t M,
                        const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *T_save,
                        const LinearPlan &pl, uint8_t *ws) {
  cudaError_t e;
  const int N = static_cast<int>(w.N), K = static_cast<int>(w.K);
  float *t_part = reinterpret_cast<float *>(ws + pl.off_t_part);
  uint16_t *sT = T_save ? T_save : reinterpret_cast<uint16_t *>(ws + pl.off_sT);
  // T = X·A  (A-op X [M,K] K-major; B-op Aᵀ: A [K,r] read MN-major)
  {
    TmaMaps m;
    if (!map_bf16_kmajor(&m.a, X, K, M, 128) || !map_bf16_mn(&m.b, A, r, K)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_T, c, pl.sp_t, pl.rpad, static_cast<int>(M), m, t_part)) != cudaSuccess) return e;
    if ((e = finalize_bf16(t_part, pl.sp_t.splits, M * pl.rpad, M, r, pl.rpad, s, sT, r, c.stream)) != cudaSuccess)
      return e;
  }
  // Y = X·W_hatᵀ + sT·B
  {
    const TimingHooks &hk = timing_hooks();
    float *part = reinterpret_cast<float *>(ws + pl.off_main_part);
    if ((e = run_fused(true, c, w, X, M, sT, B, r, Y, pl.pair_main, pl.sp_main, part, hk.fwd_begin, hk.fwd_end)) !=
        cudaSuccess)
      return e;
  }
  return cudaSuccess;
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
    float *t_part = reinterpret_cast<float *>(ws + pl.off_t_part);
    TmaMaps m;
    if (!map_bf16_kmajor(&m.a, X, K, M, 128) || !map_bf16_mn(&m.b, A, r, K)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_T, c, pl.sp_t, pl.rpad, static_cast<int>(M), m, t_part)) != cudaSuccess) return e;
    if ((e = finalize_bf16(t_part, pl.sp_t.splits, M * pl.rpad, M, r, pl.rpad, s, sT_ws, r, c.stream)) !=
        cudaSuccess)
      return e;
    sT = sT_ws;
  }
  uint16_t *sU = reinterpret_cast<uint16_t *>(ws + pl.off_sU);
  // U = dY·Bᵀ  (A-op dY [M,N] K-major; B-op B [r,N] K-major)
  {
    float *u_part = reinterpret_cast<float *>(ws + pl.off_u_part);
    TmaMaps m;
    if (!map_bf16_kmajor(&m.a, dY, N, M, 128) || !map_bf16_kmajor(&m.b, B, N, r, pl.rpad))
      return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_U, c, pl.sp_u, pl.rpad, static_cast<int>(M), m, u_part)) != cudaSuccess) return e;
    if ((e = finalize_bf16(u_part, pl.sp_u.splits, M * pl.rpad, M, r, pl.rpad, s, sU, r, c.stream)) != cudaSuccess)
      return e;
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
    float *part = reinterpret_cast<float *>(ws + pl.off_da_part);
    TmaMaps m;
    if (!map_bf16_mn(&m.a, X, K, M) || !map_bf16_mn(&m.b, sU, r, M)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_W, c, pl.sp_da, pl.rpad, K, m, part)) != cudaSuccess) return e;
    if ((e = finalize_f32(part, pl.sp_da.splits, static_cast<int64_t>(K) * pl.rpad, K, r, pl.rpad, 1.0f, dA, r,
                          c.stream)) != cudaSuccess)
      return e;
  }
  // dB = sTᵀ·dY : computed as D[N x r] = dYᵀ·sT, then transposed by the finalize
  {
    float *part = reinterpret_cast<float *>(ws + pl.off_db_part);
    TmaMaps m;
    if (!map_bf16_mn(&m.a, dY, N, M) || !map_bf16_mn(&m.b, sT, r, M)) return cudaErrorInvalidValue;
    m.a2 = m.a;
    m.b2 = m.b;
    if ((e = run_skinny(SK_W, c, pl.sp_db, pl.rpad, N, m, part)) != cudaSuccess) return e;
    if ((e = finalize_f32_t(part, pl.sp_db.splits, static_cast<int64_t>(N) * pl.rpad, N, r, pl.rpad, 1.0f, dB, N,
                            c.stream)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace qlora
