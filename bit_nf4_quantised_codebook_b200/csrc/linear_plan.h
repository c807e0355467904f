// linear_plan.h — launch planning (split counts, workspace layout) and TMA
// tensor-map construction shared by the C ABI and the launch code.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "internal.h"
#include "nf4_decode.cuh"

namespace qlora {

struct TmaMaps {
  CUtensorMap a, b, a2, b2;
};

struct LaunchCtx {
  cudaStream_t stream;
  int *dev_err;
  unsigned long long timeout_ns;
  Nf4Levels levels;
};

// Forward at M <= kSmallMaxTokens runs the swapped-orientation kernel
// (gemm_smallm.cuh): K splits of at most kSmallMaxKIters steps, at most 8 per
// cluster, so K <= 8 · 64 · kSmallMaxKIters.
constexpr int kSmallMaxTokens = 64;
constexpr int kSmallMaxKIters = 64;

struct SplitPlan {
  int splits = 1;
  int k_iters = 0;        // stages per split
  int k_iters_total = 0;  // stages in total
};

struct LinearPlan {
  int rpad = 16;
  SplitPlan sp_t, sp_u, sp_main, sp_dx, sp_da, sp_db;
  bool pair_main = false, pair_dx = false;  // CTA-pair kernel for the fused GEMMs
  bool small_main = false;                  // forward through the small-M kernel (sp_main = its splits)
  size_t off_sT = 0, off_sU = 0, off_main_part = 0;
  size_t off_absmax = 0, off_gsum = 0;
  int64_t gsum_size = 0;
  size_t bytes = 0;
};

// op = QLORA_OP_*; num_sms = multiprocessors of the device the work runs on.
LinearPlan make_plan(int op, int64_t M, int64_t N, int64_t K, int r, int num_sms);

// bf16 [outer, inner] row-major, read K-major: box {64, box_rows}, 128-byte swizzle.
bool map_bf16_kmajor(CUtensorMap *m, const void *ptr, int64_t inner, int64_t outer, int box_rows);
// bf16 [outer, inner] row-major, read MN-major (inner = MN): box {64, 64}, 128-byte swizzle.
bool map_bf16_mn(CUtensorMap *m, const void *ptr, int64_t inner, int64_t outer);
// packed codes of an N x K weight, uint8 [N, K/2]: box {box_bytes, box_rows}; swizzle_bytes 0 (none), 32, 64
// or 128.
bool map_codes(CUtensorMap *m, const void *codes, int64_t N, int64_t K, int box_bytes, int box_rows,
               int swizzle_bytes);

cudaError_t run_forward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, int64_t M,
                        const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *T_save,
                        const LinearPlan &pl, uint8_t *ws);
cudaError_t run_backward(const LaunchCtx &c, const qlora_nf4_weight &w, const uint16_t *X, const uint16_t *dY,
                         int64_t M, const uint16_t *A, const uint16_t *B, int r, float s, const uint16_t *T_saved,
                         uint16_t *dX, float *dA, float *dB, const LinearPlan &pl, uint8_t *ws);

}  // namespace qlora
