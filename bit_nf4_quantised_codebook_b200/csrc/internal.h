// internal.h — declarations shared by the library's translation units.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "../../include/qlora_nf4.h"

namespace qlora {

struct Nf4Levels;  // nf4_decode.cuh

struct Nf4Thresholds {
  float t[15];
};

// Process-wide diagnostics (capi.cu).
void count_launches(int n);
// QLORA_OK for cudaSuccess; otherwise records `e` as this host thread's last CUDA
// failure (qlora_last_cuda_error) and returns QLORA_ERR_CUDA.
qlora_status cuda_status(cudaError_t e);
struct TimingHooks {
  cudaEvent_t fwd_begin = nullptr, fwd_end = nullptr, bwd_begin = nullptr, bwd_end = nullptr;
};
const TimingHooks &timing_hooks();

// Host code-book construction (codebook.cpp).
void build_codebook_f64(double levels[16]);
void build_codebook_f32(float levels[16], float thresholds[15]);
void thresholds_f32(const float levels[16], float thresholds[15]);
bool build_format_codebook_f32(int codebook, float levels[16], float thresholds[15]);

cudaError_t launch_quantize(const uint16_t *W, int64_t nb, uint8_t *codes, uint8_t *c2q, float *c1, float *mean,
                            float *ws_absmax, double *ws_gsum, int64_t gsum_size, const Nf4Thresholds &thr,
                            int *dev_err, cudaStream_t st);
// The second quantisation from block constants already in ws_absmax: group
// sums (launch_group_sums, when the caller has not formed them), the fixed-order
// mean, then the E4M3 codes and group scales.
cudaError_t launch_group_sums(const float *ws_absmax, int64_t nb, double *ws_gsum, cudaStream_t st);
cudaError_t launch_mean_tree(double *ws_gsum, int64_t nb, int64_t gsum_size, float *mean, cudaStream_t st);
cudaError_t launch_mean_and_double_quant(const float *ws_absmax, int64_t nb, double *ws_gsum, int64_t gsum_size,
                                         float *mean, uint8_t *c2q, float *c1, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *c2q, const float *c1, const float *mean,
                              int64_t nb, const Nf4Levels &lv, uint16_t *out, cudaStream_t st);
// merge.cu
size_t merge_smem_bytes(int r);
cudaError_t launch_merge_requantize(const qlora_nf4_weight &w, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const qlora_nf4_weight &out, uint16_t *w_merged, float *ws_absmax,
                                    double *ws_gsum, int64_t gsum_size, const Nf4Levels &lv,
                                    const Nf4Thresholds &thr, int *dev_err, unsigned long long timeout_ns,
                                    cudaStream_t st);
// formats.cu
cudaError_t launch_quantize_format(const uint16_t *W, const qlora_qweight &w, const float levels[16],
                                   const float thresholds[15], float *ws_absmax, double *ws_gsum, int64_t gsum_size,
                                   int *dev_err, cudaStream_t st);
cudaError_t launch_dequantize_format(const qlora_qweight &w, const float levels[16], uint16_t *out, cudaStream_t st);
cudaError_t launch_quant_error(const uint16_t *W, const uint16_t *W_hat, int64_t n, double *stats, int num_sms,
                               cudaStream_t st);
cudaError_t launch_double_quant_int8(const float *ws_absmax, int64_t nb, const float *mean, int8_t *c2q, float *c1,
                                     cudaStream_t st);
// adamw.cu
using AdamwTensor = qlora_adamw_tensor;
constexpr int kAdamwMaxTensors = QLORA_ADAMW_MAX_TENSORS;
cudaError_t launch_adamw(const AdamwTensor *t, int count, float lr, float b1, float b2, float eps, float wd,
                         double step_size, double bc2_sqrt, int num_sms, cudaStream_t st);
// selftest.cu
cudaError_t launch_selftest_wait(unsigned long long timeout_ns, int *dev_err, int *gave_up, cudaStream_t st);

}  // namespace qlora
