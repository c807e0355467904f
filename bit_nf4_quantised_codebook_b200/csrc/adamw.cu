// adamw.cu — the adapter optimiser step: AdamW over up to 16 float32 tensors
// (the LoRA factors A and B) in one launch.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §Where finetuning memory goes (Adam's running mean and variance, 32-bit, per
// trained weight) and §The QLoRA layer, end to end (only the adapters carry a
// gradient and optimiser state); AdamW as published by Loshchilov and Hutter,
// in PyTorch's arrangement.  Per element, at step t:
//   p <- p·(1 - lr·wd);  m <- m + (1 - b1)(g - m);  v <- b2·v + (1 - b2)·g²;
//   p <- p - step_size · m / (sqrt(v) / bc2_sqrt + eps),
// step_size = lr / (1 - b1^t), bc2_sqrt = sqrt(1 - b2^t) (host, float64).
// Optionally writes the bfloat16 copy of p that the linear layer reads.
//
// HBM-bound streaming kernel: 16-byte loads and stores, grid-stride over the
// concatenated elements of all tensors (16 + 12 (+2) bytes per element).
#include <cstdint>
#include <cuda_runtime.h>
#include "internal.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace qlora {

struct AdamwArgs {
  AdamwTensor t[kAdamwMaxTensors];
  int64_t start[kAdamwMaxTensors + 1];  // prefix sums of the element counts (in units of 4)
  int count;
  float lr, b1, b2, eps, wd, step_size, bc2_sqrt;
};

__device__ __forceinline__ void adamw_one(float &p, float g, float &m, float &v, const AdamwArgs &a) {
  p = p * (1.0f - a.lr * a.wd);
  m = __fmaf_rn(1.0f - a.b1, g - m, m);
  v = __fmaf_rn(a.b2, v, (1.0f - a.b2) * g * g);
  const float denom = __fsqrt_rn(v) / a.bc2_sqrt + a.eps;
  p = p - a.step_size * (m / denom);
}

__global__ void __launch_bounds__(256) k_adamw(const __grid_constant__ AdamwArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t total4 = a.start[a.count];
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int k = 0;
    while (k + 1 < a.count && i >= a.start[k + 1]) ++k;
    const AdamwTensor &t = a.t[k];
    const int64_t e = (i - a.start[k]) * 4;  // first element of this quad
    if (e + 4 <= t.n) {
      float4 p = *reinterpret_cast<const float4 *>(t.param + e);
      const float4 g = *reinterpret_cast<const float4 *>(t.grad + e);
      float4 m = *reinterpret_cast<const float4 *>(t.m + e);
      float4 v = *reinterpret_cast<const float4 *>(t.v + e);
      adamw_one(p.x, g.x, m.x, v.x, a);
      adamw_one(p.y, g.y, m.y, v.y, a);
      adamw_one(p.z, g.z, m.z, v.z, a);
      adamw_one(p.w, g.w, m.w, v.w, a);
      *reinterpret_cast<float4 *>(t.param + e) = p;
      *reinterpret_cast<float4 *>(t.m + e) = m;
      *reinterpret_cast<float4 *>(t.v + e) = v;
      if (t.param_bf16) {
        uint2 pk;
        pk.x = pack_bf16x2(p.x, p.y);
        pk.y = pack_bf16x2(p.z, p.w);
        *reinterpret_cast<uint2 *>(t.param_bf16 + e) = pk;
      }
    } else {
      for (int64_t j = e; j < t.n; ++j) {  // ragged tail of this tensor
        float p = t.param[j], m = t.m[j], v = t.v[j];
        adamw_one(p, t.grad[j], m, v, a);
        t.param[j] = p;
        t.m[j] = m;
        t.v[j] = v;
        if (t.param_bf16) t.param_bf16[j] = static_cast<uint16_t>(pack_bf16x2(p, 0.f) & 0xFFFFu);
      }
    }
  }
}

cudaError_t launch_adamw(const AdamwTensor *t, int count, float lr, float b1, float b2, float eps, float wd,
                         double step_size, double bc2_sqrt, int num_sms, cudaStream_t st) {
  AdamwArgs a;
  a.count = count;
  a.start[0] = 0;
  for (int k = 0; k < count; ++k) {
    a.t[k] = t[k];
    a.start[k + 1] = a.start[k] + (t[k].n + 3) / 4;
  }
  for (int k = count; k < kAdamwMaxTensors; ++k) {
    a.t[k] = AdamwTensor{};
    a.start[k + 1] = a.start[count];
  }
  a.lr = lr;
  a.b1 = b1;
  a.b2 = b2;
  a.eps = eps;
  a.wd = wd;
  a.step_size = static_cast<float>(step_size);
  a.bc2_sqrt = static_cast<float>(bc2_sqrt);
  const int64_t total4 = a.start[count];
  int64_t grid = (total4 + 255) / 256;
  const int64_t cap = 4 * static_cast<int64_t>(num_sms);
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  return launch_k(k_adamw, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, 1, a);
}

}  // namespace qlora
