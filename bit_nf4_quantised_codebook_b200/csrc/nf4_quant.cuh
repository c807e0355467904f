// nf4_quant.cuh — exact normalisation and nearest-level code of one weight.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §Quantize in blocks / §NormalFloat: each weight is divided by its block's
// absmax and mapped to the nearest NF4 level.  The library defines
//   x_hat = float32(w / absmax)   (IEEE division, round to nearest even)
//   code  = #{ i : x_hat >= t_i }  (t_i = smallest float32 above midpoint i)
// and must reproduce both exactly.  Two cheaper, exact, steps:
//
// Quotient.  With y = RN(1/a) and q = RN(x·y), the residual r = x - a·q is
// exact as one fused multiply-add, and RN(q + r·y) = RN(x/a) (Markstein's
// correction theorem for a reciprocal within half an ulp and a quotient within
// one ulp; P. Markstein, IBM J. Res. Dev. 34(1), 1990).  Per block the
// reciprocal is computed once; each element then costs one multiply and two
// fused multiply-adds.  tests/test_gpu_quotient.py checks the result against
// CUDA's own correctly rounded division for every pair of bfloat16 inputs with
// |x| <= a that the quantiser can meet.
//
// Code.  x_hat lies in [-1, 1].  Cut that range into 64 buckets of width 1/32;
// widen each by a margin far above any rounding error of the bucket index
// computation and far below the smallest gap between two thresholds (0.0796).
// Each widened bucket then holds at most one threshold, so
//   code = base[b] + (x_hat >= thr[b]),
// with base[b] = thresholds below the widened bucket and thr[b] the one inside
// it (+inf if none).  The 64-entry table is built per CTA from the thresholds.
#pragma once
#include <cstdint>

namespace qlora {

constexpr int kBuckets = 64;
constexpr float kBucketScale = 32.0f;          // buckets per unit of x_hat
constexpr float kBucketMargin = 1.0f / 1024;   // widening on each side

struct __align__(8) CodeBucket {  // 8-byte aligned: one 64-bit shared-memory load per lookup
  int base;
  float thr;
};

// RN(x / a) for finite x, a > 0 with |x| <= a, given ra = RN(1/a).
__device__ __forceinline__ float quotient_rn(float x, float a, float ra) {
  const float q = __fmul_rn(x, ra);
  const float r = __fmaf_rn(-q, a, x);
  return __fmaf_rn(r, ra, q);
}

// Fill bucket b (0..63) from the 15 thresholds.
__device__ __forceinline__ CodeBucket make_bucket(int b, const float (&t)[15]) {
  const float lo = static_cast<float>(b) / kBucketScale - 1.0f - kBucketMargin;
  const float hi = static_cast<float>(b + 1) / kBucketScale - 1.0f + kBucketMargin;
  CodeBucket e;
  e.base = 0;
  e.thr = __int_as_float(0x7F800000);  // +inf
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    if (t[i] < lo) e.base += 1;
    else if (t[i] <= hi) e.thr = t[i];
  }
  return e;
}

__device__ __forceinline__ uint32_t bucket_code(float xh, const CodeBucket *tab) {
  int b = __float2int_rd(__fmaf_rn(xh, kBucketScale, kBucketScale));
  b = min(max(b, 0), kBuckets - 1);
  const CodeBucket e = tab[b];
  return static_cast<uint32_t>(e.base + (xh >= e.thr ? 1 : 0));
}

// Nearest level by counting thresholds (15 compares); for the rare blocks
// whose absmax is too small for the reciprocal path.
template <typename Thresholds>
__device__ __forceinline__ uint32_t nf4_code(float xh, const Thresholds &t) {
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) c += (xh >= t.t[i]) ? 1u : 0u;
  return c;
}

// Blocks whose absmax is at least this use the reciprocal + corrected-quotient
// path (exact there: see quotient_rn); smaller ones divide directly.
constexpr float kFastQuotientMinAbsmax = 7.888609052210118e-31f;  // 2^-100

// Centred buckets, for an index computed without a float-to-int conversion:
// v = x_hat * 32 + 32 + 2^23, one fused multiply-add rounded to nearest, holds
// round(x_hat * 32 + 32) in its low mantissa bits (0 .. 64 for x_hat in
// [-1, 1]).  Bucket b therefore covers x_hat in [(b - 1/2)/32 - 1,
// (b + 1/2)/32 - 1], widened by the same margin on each side, which again holds
// at most one threshold (width 1/32 + 2/1024 < 0.0796).  65 buckets.
constexpr int kCentredBuckets = 65;
constexpr float kCentredMagic = 8388608.0f + 32.0f;  // 2^23 + 32: exact in float32
constexpr int kCentredMagicBits = 0x4B000020;        // its bit pattern

__device__ __forceinline__ CodeBucket make_bucket_centred(int b, const float (&t)[15]) {
  const float lo = (static_cast<float>(b) - 0.5f) / kBucketScale - 1.0f - kBucketMargin;
  const float hi = (static_cast<float>(b) + 0.5f) / kBucketScale - 1.0f + kBucketMargin;
  CodeBucket e;
  e.base = 0;
  e.thr = __int_as_float(0x7F800000);  // +inf
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    if (t[i] < lo) e.base += 1;
    else if (t[i] <= hi) e.thr = t[i];
  }
  return e;
}

// Code of x_hat in [-1, 1] from a centred table replicated once per lane
// ([bucket][lane], so 32 lanes with arbitrary buckets never share a bank).
__device__ __forceinline__ uint32_t lane_centred_code(float xh, const CodeBucket (*tab)[32], int lane) {
  const int b = __float_as_int(__fmaf_rn(xh, kBucketScale, kCentredMagic)) - (kCentredMagicBits - 32);
  const CodeBucket e = tab[b][lane];
  return static_cast<uint32_t>(e.base + (xh >= e.thr ? 1 : 0));
}

// Same lookup in a table replicated once per lane ([bucket][lane]), so that 32
// lanes looking up arbitrary buckets never share a bank.
__device__ __forceinline__ uint32_t lane_bucket_code(float xh, const CodeBucket (*tab)[32], int lane) {
  int b = __float2int_rd(__fmaf_rn(xh, kBucketScale, kBucketScale));
  b = min(max(b, 0), kBuckets - 1);
  const CodeBucket e = tab[b][lane];
  return static_cast<uint32_t>(e.base + (xh >= e.thr ? 1 : 0));
}

}  // namespace qlora
