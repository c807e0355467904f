// formats.cu — the quantiser and dequantiser for the storage-format variants
// (other 4-bit code books, blocks of 32..256, block constants kept as float32,
// E4M3 or int8), and the error statistics of a round trip.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai):
//   §Quantize in blocks  — absmax blocks; the int8 absmax grid (scale 127/absmax);
//   §NormalFloat         — NF4 set against the uniform Int4 grid;
//   §Double quantization — constants in 8 bits, groups of 256, mean subtracted;
//   §It matches 16-bit finetuning — NF4 + DQ against "4-bit float variants".
// "QLoRA Review" (tildalice.io), §What Would Trip You Up in Practice: smaller
// blocks are more precise and cost more.
//
// k_quant_format<BLOCK>: each thread codes 8 consecutive weights (one 16-byte
// load); the BLOCK/8 threads of a block are consecutive lanes of one warp and
// find its absmax with xor-shuffles.  x = float32(w / absmax) exactly as in the
// main quantiser (corrected quotient, nf4_quant.cuh); the code is the count of
// thresholds at or below x, found by a 4-step binary search over the 15
// thresholds in shared memory (any sorted table works, unlike the bucket
// table of the NF4 kernel, which needs thresholds at least 1/32 apart).
// The second quantisation reuses quantize.cu's group sums and mean; the int8
// variant of the E4M3 step is k_double_quant_int8 here.
#include <cstdint>
#include <cuda_runtime.h>
#include "internal.h"
#include "launch.cuh"
#include "nf4_decode.cuh"
#include "nf4_quant.cuh"
#include "ptx.cuh"

namespace qlora {
namespace {

struct Table16 {
  float v[16];
};
struct Table15 {
  float v[15];
};

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// #{i : x >= t[i]} for ascending t[0..14].
__device__ __forceinline__ uint32_t count_thresholds(float x, const float *t) {
  uint32_t c = x >= t[7] ? 8u : 0u;
  c += x >= t[c + 3] ? 4u : 0u;
  c += x >= t[c + 1] ? 2u : 0u;
  c += x >= t[c] ? 1u : 0u;
  return c;
}

template <int BLOCK>
__global__ void __launch_bounds__(256) k_quant_format(const uint16_t *__restrict__ W, int64_t n8,
                                                       uint8_t *__restrict__ codes, float *__restrict__ absmax,
                                                       Table15 thr, int *dev_err) {
  constexpr int T = BLOCK / 8;  // threads per block
  static_assert(T >= 4 && T <= 32 && (T & (T - 1)) == 0, "block of 32..256");
  __shared__ float s_thr[15];
  if (threadIdx.x < 15) s_thr[threadIdx.x] = thr.v[threadIdx.x];
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  bool bad = false;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32) * 32; base < n8;
       base += warps * 32) {
    const int64_t u = base + lane;  // this thread's 8 weights: 8u .. 8u+7
    const bool valid = u < n8;      // n8 is a multiple of T: whole blocks are valid or not
    const uint4 raw = valid ? ld_nc_v4(W + u * 8) : make_uint4(0, 0, 0, 0);
    const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
    float x[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(wd[i] << 16);
      x[2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = fabsf(x[i]);
      bad |= !(a <= 3.402823466e38f);
      amax = fmaxf(amax, a);
    }
#pragma unroll
    for (int o = 1; o < T; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    float xh[8];
    if (amax >= kFastQuotientMinAbsmax) {
      const float ra = __frcp_rn(amax);
#pragma unroll
      for (int i = 0; i < 8; ++i) xh[i] = quotient_rn(x[i], amax, ra);
    } else if (amax > 0.f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) xh[i] = __fdiv_rn(x[i], amax);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) xh[i] = 0.f;  // all-zero block: the first zero level
    }
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t hi = count_thresholds(xh[2 * i], s_thr), lo = count_thresholds(xh[2 * i + 1], s_thr);
      packed |= ((hi << 4) | lo) << (8 * i);
    }
    if (valid) {
      reinterpret_cast<uint32_t *>(codes)[u] = packed;
      if ((lane & (T - 1)) == 0) absmax[u / T] = amax;
    }
  }
  if (bad && dev_err) atomicOr(dev_err, QLORA_DEVERR_NONFINITE);
}

// Int8 absmax grid of the mean-centred constants, one CTA per group of 256 blocks.
__global__ void __launch_bounds__(256) k_double_quant_int8(const float *__restrict__ absmax, int64_t nb,
                                                            const float *__restrict__ mean, int8_t *__restrict__ c2q,
                                                            float *__restrict__ c1) {
  __shared__ float s_red[8];
  pdl_wait();
  pdl_launch_dependents();
  const int64_t g = blockIdx.x;
  const int64_t b = g * 256 + threadIdx.x;
  const bool valid = b < nb;
  const float mu = *mean;
  const float dev = valid ? __fsub_rn(absmax[b], mu) : 0.f;
  float a = fabsf(dev);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = a;
  __syncthreads();
  float amax = s_red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, s_red[i]);
  const float sg = __fdiv_rn(amax, 127.0f);
  int e = 0;
  if (sg != 0.f) e = min(127, max(-127, __float2int_rn(__fdiv_rn(dev, sg))));
  if (valid) c2q[b] = static_cast<int8_t>(e);
  if (threadIdx.x == 0) c1[g] = sg;
}

template <int BLOCK>
__global__ void __launch_bounds__(256) k_dequant_format(const uint8_t *__restrict__ codes,
                                                         const void *__restrict__ consts, const float *__restrict__ c1,
                                                         const float *__restrict__ mean, int dq, int64_t n8,
                                                         Nf4Levels lv, uint16_t *__restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n8; u += stride) {
    const int64_t b = u / (BLOCK / 8);
    float ch;
    if (dq == QLORA_DQ_NONE) {
      ch = static_cast<const float *>(consts)[b];
    } else {
      const uint32_t e = static_cast<const uint8_t *>(consts)[b];
      const float sg = c1[b >> 8], mu = *mean;
      ch = dq == QLORA_DQ_E4M3 ? reconstruct_c2(e, sg, mu)
                               : __fmaf_rn(static_cast<float>(static_cast<int8_t>(e)), sg, mu);
    }
    const BlockLut lut = make_lut(ch, lv);
    uint32_t o[4];
    decode8(reinterpret_cast<const uint32_t *>(codes)[u], lut, o);
    reinterpret_cast<uint4 *>(out)[u] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__global__ void k_stats_init(double *stats) {
  pdl_wait();
  pdl_launch_dependents();
  stats[0] = 0.0;
  stats[1] = 0.0;
  stats[2] = 0.0;
}

__global__ void __launch_bounds__(256) k_quant_error(const uint16_t *__restrict__ W, const uint16_t *__restrict__ Wh,
                                                      int64_t n, double *stats) {
  __shared__ double s_part[3][8];
  pdl_wait();
  pdl_launch_dependents();
  double se = 0.0, sw = 0.0, mx = 0.0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const double w = static_cast<double>(__uint_as_float(static_cast<uint32_t>(W[i]) << 16));
    const double h = static_cast<double>(__uint_as_float(static_cast<uint32_t>(Wh[i]) << 16));
    const double d = w - h;  // exact: two bfloat16 values
    se = fma(d, d, se);
    sw = fma(w, w, sw);
    mx = fmax(mx, fabs(d));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    se += __shfl_xor_sync(0xFFFFFFFFu, se, o);
    sw += __shfl_xor_sync(0xFFFFFFFFu, sw, o);
    mx = fmax(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    s_part[0][warp] = se;
    s_part[1][warp] = sw;
    s_part[2][warp] = mx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) {
      se += s_part[0][i];
      sw += s_part[1][i];
      mx = fmax(mx, s_part[2][i]);
    }
    atomicAdd(stats, se);
    atomicAdd(stats + 1, sw);
    // non-negative doubles order like their bit patterns
    atomicMax(reinterpret_cast<unsigned long long *>(stats + 2), static_cast<unsigned long long>(__double_as_longlong(mx)));
  }
}

template <int BLOCK>
cudaError_t quant_launch(const uint16_t *W, int64_t n8, uint8_t *codes, float *absmax, const Table15 &thr,
                         int *dev_err, cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n8 + 255) / 256;
  const int64_t grid = want < 8 * static_cast<int64_t>(sms) ? want : 8 * static_cast<int64_t>(sms);
  return launch_k(k_quant_format<BLOCK>, dim3(static_cast<unsigned>(grid > 0 ? grid : 1)), dim3(256), 0, st, 1, W,
                  n8, codes, absmax, thr, dev_err);
}

template <int BLOCK>
cudaError_t dequant_launch(const qlora_qweight &w, int64_t n8, const Nf4Levels &lv, uint16_t *out, cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n8 + 255) / 256;
  const int64_t grid = want < 8 * static_cast<int64_t>(sms) ? want : 8 * static_cast<int64_t>(sms);
  return launch_k(k_dequant_format<BLOCK>, dim3(static_cast<unsigned>(grid > 0 ? grid : 1)), dim3(256), 0, st, 1,
                  static_cast<const uint8_t *>(w.codes), static_cast<const void *>(w.consts),
                  static_cast<const float *>(w.c1), static_cast<const float *>(w.mean), w.fmt.dq, n8, lv, out);
}

}  // namespace

cudaError_t launch_double_quant_int8(const float *ws_absmax, int64_t nb, const float *mean, int8_t *c2q, float *c1,
                                     cudaStream_t st) {
  const int64_t ng = (nb + 255) / 256;
  return launch_k(k_double_quant_int8, dim3(static_cast<unsigned>(ng)), dim3(256), 0, st, 1, ws_absmax, nb, mean,
                  c2q, c1);
}

cudaError_t launch_quantize_format(const uint16_t *W, const qlora_qweight &w, const float levels[16],
                                   const float thresholds[15], float *ws_absmax, double *ws_gsum, int64_t gsum_size,
                                   int *dev_err, cudaStream_t st) {
  (void)levels;
  Table15 thr;
  for (int i = 0; i < 15; ++i) thr.v[i] = thresholds[i];
  const int64_t n8 = w.N * w.K / 8;
  const int64_t nb = w.N * w.K / w.fmt.block;
  // DQ_NONE: the absmax values are the stored constants
  float *amax = w.fmt.dq == QLORA_DQ_NONE ? static_cast<float *>(w.consts) : ws_absmax;
  cudaError_t e;
  switch (w.fmt.block) {
    case 32: e = quant_launch<32>(W, n8, w.codes, amax, thr, dev_err, st); break;
    case 64: e = quant_launch<64>(W, n8, w.codes, amax, thr, dev_err, st); break;
    case 128: e = quant_launch<128>(W, n8, w.codes, amax, thr, dev_err, st); break;
    case 256: e = quant_launch<256>(W, n8, w.codes, amax, thr, dev_err, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || w.fmt.dq == QLORA_DQ_NONE) return e;
  if ((e = launch_group_sums(ws_absmax, nb, ws_gsum, st)) != cudaSuccess) return e;
  if (w.fmt.dq == QLORA_DQ_E4M3)
    return launch_mean_and_double_quant(ws_absmax, nb, ws_gsum, gsum_size, w.mean, static_cast<uint8_t *>(w.consts),
                                        w.c1, st);
  if ((e = launch_mean_tree(ws_gsum, nb, gsum_size, w.mean, st)) != cudaSuccess) return e;
  return launch_double_quant_int8(ws_absmax, nb, w.mean, static_cast<int8_t *>(w.consts), w.c1, st);
}

cudaError_t launch_dequantize_format(const qlora_qweight &w, const float levels[16], uint16_t *out, cudaStream_t st) {
  Nf4Levels lv;
  for (int i = 0; i < 16; ++i) lv.q[i] = levels[i];
  const int64_t n8 = w.N * w.K / 8;
  switch (w.fmt.block) {
    case 32: return dequant_launch<32>(w, n8, lv, out, st);
    case 64: return dequant_launch<64>(w, n8, lv, out, st);
    case 128: return dequant_launch<128>(w, n8, lv, out, st);
    case 256: return dequant_launch<256>(w, n8, lv, out, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quant_error(const uint16_t *W, const uint16_t *W_hat, int64_t n, double *stats, int num_sms,
                               cudaStream_t st) {
  cudaError_t e = launch_k(k_stats_init, dim3(1), dim3(1), 0, st, 1, stats);
  if (e != cudaSuccess) return e;
  const int64_t want = (n + 255) / 256;
  const int64_t grid = want < 4 * static_cast<int64_t>(num_sms) ? want : 4 * static_cast<int64_t>(num_sms);
  return launch_k(k_quant_error, dim3(static_cast<unsigned>(grid > 0 ? grid : 1)), dim3(256), 0, st, 1, W, W_hat, n,
                  stats);
}

}  // namespace qlora
