// quantize.cu — blockwise NF4 quantiser with double quantisation, and the
// standalone double-dequantiser.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai):
//   §Quantize in blocks  — flatten, cut into 64-element blocks, absmax per block;
//   §NormalFloat         — each normalised weight goes to the nearest NF4 level;
//   §Double quantization — block constants, mean-centred, become 8-bit floats in
//                          groups of 256 with one float32 scale per group.
//
// Three launches, all HBM-streaming and deterministic:
//   k_quant_blocks : CTAs walk the groups of 256 blocks, prefetching the next
//                    group while coding the current one.  8 threads per block,
//                    one 16-byte load each; absmax by 3 xor-shuffles; exact
//                    quotient and code via nf4_quant.cuh; nibble packing;
//                    per-group float64 pairwise tree of the absmax values.
//   k_mean_tree    : one CTA, power-of-two pairwise tree over the group sums.
//   k_double_quant : one CTA per group: centred constants, group absmax, S_g,
//                    E4M3 codes (round to nearest even, saturating).
#include <cstdint>
#include <cuda_runtime.h>
#include "internal.h"
#include "nf4_decode.cuh"
#include "nf4_quant.cuh"
#include "launch.cuh"

namespace qlora {

__device__ __forceinline__ uint32_t e4m3_from_f32_satfinite(float x) {
  uint16_t two;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(x), "f"(x));
  return two & 0xFFu;
}


// Streaming 16-byte load that does not keep the line in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Sum of s[0..255] by the pairwise tree (h = 128, 64, ..., 1: s[i] += s[i+h]);
// called by all 256 threads, the sum is returned in thread 0.  Both the
// quantiser and the group-sum pass of the adapter merge use it, so the block
// constants of a group are always added in this one order.
__device__ __forceinline__ double tree_sum256(double *s) {
  __syncthreads();
  const int t = threadIdx.x;
  for (int h = 128; h >= 32; h >>= 1) {
    if (t < h) s[t] = __dadd_rn(s[t], s[t + h]);
    __syncthreads();
  }
  double v = 0.0;
  if (t < 32) {
    v = s[t];
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) {
      const double o = __shfl_down_sync(0xFFFFFFFFu, v, h);
      if (t < h) v = __dadd_rn(v, o);
    }
  }
  return v;
}

// 1-D bulk copy (TMA, no tensor map) of `bytes` (a multiple of 16, both addresses
// 16-byte aligned) from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

constexpr unsigned long long kQuantWaitNs = 2000000000ull;  // bound on a wait for a group's bytes (2 s)
constexpr int kQThreads = 1024;                   // 32 warps; 8 threads per 64-element block
constexpr int kQStages = 4;                       // groups in the shared-memory ring
constexpr int kQGroupBytes = 256 * 64 * 2;        // one group of 256 blocks of bfloat16: 32 KiB
constexpr int kQTabBytes = kCentredBuckets * 32 * static_cast<int>(sizeof(CodeBucket));
constexpr int kQSmemBytes = kQStages * kQGroupBytes + kQTabBytes + 2 * 256 * 8 + kQStages * 8 + 128;

// One CTA of 1024 threads per SM walks groups g = blockIdx.x, blockIdx.x +
// gridDim.x, ...  Each group's 32 KiB of bfloat16 weights arrive in a 4-deep
// shared-memory ring by one bulk copy, issued three groups ahead, so HBM reads
// never wait on the arithmetic.  Eight threads share a block: 16-byte chunk each, absmax by three
// xor-shuffles, exact quotient and code (nf4_quant.cuh), nibble packing.  The
// group's 256 absmax values are summed by one warp in the pairwise-tree order
// (a[i] += a[i + h] for h = 128 .. 1) while the other warps start the next group.
__global__ void __launch_bounds__(kQThreads, 1) k_quant_blocks(const uint16_t *__restrict__ W, int64_t nb,
                                                                uint8_t *__restrict__ codes,
                                                                float *__restrict__ absmax, double *__restrict__ gsum,
                                                                Nf4Thresholds thr, int *dev_err,
                                                                unsigned long long timeout_ns) {
  extern __shared__ __align__(128) uint8_t q_smem[];
  uint8_t *ring = q_smem;
  CodeBucket(*tab)[32] = reinterpret_cast<CodeBucket(*)[32]>(q_smem + kQStages * kQGroupBytes);
  double *s_amax = reinterpret_cast<double *>(q_smem + kQStages * kQGroupBytes + kQTabBytes);  // [2][256]
  uint64_t *full = reinterpret_cast<uint64_t *>(s_amax + 2 * 256);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(full + kQStages);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int part = tid & 7;  // 8-element chunk of the block
  const int64_t ng = (nb + 255) / 256;
  for (int i = tid; i < kCentredBuckets * 32; i += kQThreads) tab[i >> 5][i & 31] = make_bucket_centred(i >> 5, thr.t);
  if (tid == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  auto issue = [&](int64_t g, int s) {
    const int64_t blocks = nb - g * 256 < 256 ? nb - g * 256 : 256;
    const uint32_t bytes = static_cast<uint32_t>(blocks) * 128;
    mbar_arrive_expect_tx(&full[s], bytes);
    bulk_load(ring + s * kQGroupBytes, W + g * 256 * 64, bytes, &full[s]);
  };
  int issued = 0;  // groups issued (thread 0), group k of this CTA into stage k % kQStages
  if (tid == 0)
    for (int k = 0; k < kQStages - 1; ++k) {
      const int64_t g = blockIdx.x + static_cast<int64_t>(k) * gridDim.x;
      if (g < ng) {
        issue(g, k);
        ++issued;
      }
    }
  bool bad = false;
  int it = 0;
  for (int64_t g = blockIdx.x; g < ng; g += gridDim.x, ++it) {
    const int s = it % kQStages;
    if (tid == 0) {  // the stage freed at the end of the previous group takes the group three ahead
      const int64_t g2 = g + static_cast<int64_t>(kQStages - 1) * gridDim.x;
      if (g2 < ng) {
        issue(g2, (it + kQStages - 1) % kQStages);
        ++issued;
      }
    }
    const bool ok = mbar_wait_bounded(&full[s], (it / kQStages) & 1, abort_flag, dev_err, timeout_ns);
    if (__syncthreads_or(!ok)) break;
    const uint8_t *st = ring + s * kQGroupBytes;
    double *sa = s_amax + (it & 1) * 256;
#pragma unroll
    for (int pass = 0; pass < 256 * 8 / kQThreads; ++pass) {
      const int lb = pass * (kQThreads / 8) + (tid >> 3);  // block within the group
      const int64_t b = g * 256 + lb;
      const bool valid = b < nb;
      uint32_t u[4] = {0, 0, 0, 0};
      if (valid) ld_shared_v4(smem_u32(st + lb * 128 + part * 16), u[0], u[1], u[2], u[3]);
      float x[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
      // absmax on the bit patterns: with the sign cleared, bfloat16 magnitudes
      // order like unsigned integers, two per 16x2 max; a block maximum at or
      // above 0x7F80 (the infinity pattern) means an infinity or NaN in the block
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) m2 = __vmaxu2(m2, u[i] & 0x7FFF7FFFu);
      uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);
      mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
      mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 2));
      mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 4));
      const float amax = __uint_as_float(mb << 16);
      uint32_t packed = 0x77777777u;  // all-zero block: every code is the zero level
      if (mb >= 0x7F80u) {
        bad = true;  // reported; the block keeps the zero-level codes (the bucket index needs |x_hat| <= 1)
      } else if (amax >= kFastQuotientMinAbsmax) {
        const float ra = __frcp_rn(amax);
        packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t hi = lane_centred_code(quotient_rn(x[2 * i], amax, ra), tab, lane);
          const uint32_t lo = lane_centred_code(quotient_rn(x[2 * i + 1], amax, ra), tab, lane);
          packed += (lo + (hi << 4)) << (8 * i);  // disjoint nibbles: + is |
        }
      } else if (amax > 0.f) {
        packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t hi = nf4_code(__fdiv_rn(x[2 * i], amax), thr);
          const uint32_t lo = nf4_code(__fdiv_rn(x[2 * i + 1], amax), thr);
          packed += (lo + (hi << 4)) << (8 * i);
        }
      }
      if (valid) {
        reinterpret_cast<uint32_t *>(codes + b * 32)[part] = packed;
        if (part == 0) absmax[b] = amax;
      }
      if (part == 0) sa[lb] = valid ? static_cast<double>(amax) : 0.0;
    }
    __syncthreads();  // the stage is free again; the group's absmax values are in sa
    if (tid < 32) {
      // pairwise tree over the 256 (zero-padded) block constants: lane l holds
      // a[l + 32j]; h = 128, 64, 32 in registers, then h = 16 .. 1 across lanes
      double v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = sa[lane + 32 * j];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __dadd_rn(v[j], v[j + 4]);
#pragma unroll
      for (int j = 0; j < 2; ++j) v[j] = __dadd_rn(v[j], v[j + 2]);
      double a = __dadd_rn(v[0], v[1]);
#pragma unroll
      for (int h = 16; h >= 1; h >>= 1) {
        const double o = __shfl_down_sync(0xFFFFFFFFu, a, h);
        if (lane < h) a = __dadd_rn(a, o);
      }
      if (lane == 0) gsum[g] = a;
    }
  }
  // groups issued but never consumed (only after an abort) land before the CTA exits
  if (tid == 0)
    for (int k = it; k < issued; ++k) {
      int dummy = 0;
      mbar_wait_bounded(&full[k % kQStages], (k / kQStages) & 1, &dummy, nullptr, kQuantWaitNs);
    }
  if (bad && dev_err) atomicOr(dev_err, QLORA_DEVERR_NONFINITE);
}

// Group sums of float32 block constants that are already in memory (the
// adapter merge writes them): one CTA per group, the same tree as above.
__global__ void __launch_bounds__(256) k_group_sums(const float *__restrict__ absmax, int64_t nb,
                                                     double *__restrict__ gsum) {
  __shared__ double s_sum[256];
  pdl_wait();
  pdl_launch_dependents();
  const int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  s_sum[threadIdx.x] = b < nb ? static_cast<double>(absmax[b]) : 0.0;
  const double gs = tree_sum256(s_sum);
  if (threadIdx.x == 0) gsum[blockIdx.x] = gs;
}

// Pairwise tree over the power-of-two padded group sums: for h = size/2, ..., 1
// every a[i] (i < h) becomes a[i] + a[i+h].  Levels with h >= 1024 run in global
// memory, h = 512..32 in shared memory, h = 16..1 as warp shuffles — the same
// additions in the same order at every level.
__global__ void __launch_bounds__(1024) k_mean_tree(double *__restrict__ a, int64_t ng, int64_t size, int64_t nb,
                                                     float *__restrict__ mean) {
  __shared__ double s[1024];
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t i = ng + threadIdx.x; i < size; i += blockDim.x) a[i] = 0.0;
  __syncthreads();
  int64_t h = size / 2;
  for (; h >= 1024; h /= 2) {
    for (int64_t i = threadIdx.x; i < h; i += blockDim.x) a[i] = __dadd_rn(a[i], a[i + h]);
    __syncthreads();
  }
  // now at most 2*min(size,1024) live values remain: a[0 .. 2h)
  const int t = threadIdx.x;
  const int live = static_cast<int>(size < 1024 ? size : 1024);
  s[t] = t < live ? a[t] : 0.0;
  __syncthreads();
  for (int hh = live / 2; hh >= 32; hh /= 2) {
    if (t < hh) s[t] = __dadd_rn(s[t], s[t + hh]);
    __syncthreads();
  }
  if (t < 32) {
    double v = s[t];
    for (int hh = (live < 32 ? live / 2 : 16); hh >= 1; hh /= 2) {
      const double o = __shfl_down_sync(0xFFFFFFFFu, v, hh);
      if (t < hh) v = __dadd_rn(v, o);
    }
    if (t == 0) *mean = __double2float_rn(__ddiv_rn(v, static_cast<double>(nb)));
  }
}

__global__ void __launch_bounds__(256) k_double_quant(const float *__restrict__ absmax, int64_t nb,
                                                       const float *__restrict__ mean, uint8_t *__restrict__ c2q,
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
  const float sg = __fdiv_rn(amax, 448.0f);
  uint32_t e = 0;
  if (sg != 0.f) e = e4m3_from_f32_satfinite(__fdiv_rn(dev, sg));
  if (valid) c2q[b] = static_cast<uint8_t>(e);
  if (threadIdx.x == 0) c1[g] = sg;
}

__global__ void __launch_bounds__(256) k_dequant(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ c2q,
                                                  const float *__restrict__ c1, const float *__restrict__ mean,
                                                  int64_t nb, Nf4Levels lv, uint16_t *__restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const float c2h = reconstruct_c2(c2q[b], c1[b >> 8], *mean);
  const BlockLut lut = make_lut(c2h, lv);
  const uint4 *cp = reinterpret_cast<const uint4 *>(codes + b * 32);
  const uint4 q0 = __ldg(cp), q1 = __ldg(cp + 1);
  const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  uint4 *op = reinterpret_cast<uint4 *>(out + b * 64);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t o[4];
    decode8(w[c], lut, o);
    op[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------- host launchers
cudaError_t launch_quantize(const uint16_t *W, int64_t nb, uint8_t *codes, uint8_t *c2q, float *c1, float *mean,
                            float *ws_absmax, double *ws_gsum, int64_t gsum_size, const Nf4Thresholds &thr,
                            int *dev_err, cudaStream_t st) {
  const int64_t ng = (nb + 255) / 256;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = ng < static_cast<int64_t>(sms) ? ng : static_cast<int64_t>(sms);
  static std::atomic<uint64_t> prepared{0};
  cudaError_t e = smem_attr_once(reinterpret_cast<const void *>(k_quant_blocks), kQSmemBytes, prepared);
  if (e != cudaSuccess) return e;
  e = launch_k(k_quant_blocks, dim3(static_cast<unsigned>(grid)), dim3(kQThreads), kQSmemBytes, st, 1, W, nb, codes,
               ws_absmax, ws_gsum, thr, dev_err, kQuantWaitNs);
  if (e != cudaSuccess) return e;
  return launch_mean_and_double_quant(ws_absmax, nb, ws_gsum, gsum_size, mean, c2q, c1, st);
}

cudaError_t launch_mean_tree(double *ws_gsum, int64_t nb, int64_t gsum_size, float *mean, cudaStream_t st) {
  const int64_t ng = (nb + 255) / 256;
  return launch_k(k_mean_tree, dim3(1), dim3(1024), 0, st, 1, ws_gsum, ng, gsum_size, nb, mean);
}

cudaError_t launch_mean_and_double_quant(const float *ws_absmax, int64_t nb, double *ws_gsum, int64_t gsum_size,
                                         float *mean, uint8_t *c2q, float *c1, cudaStream_t st) {
  const int64_t ng = (nb + 255) / 256;
  cudaError_t e = launch_mean_tree(ws_gsum, nb, gsum_size, mean, st);
  if (e != cudaSuccess) return e;
  return launch_k(k_double_quant, dim3(static_cast<unsigned>(ng)), dim3(256), 0, st, 1, ws_absmax, nb,
                  static_cast<const float *>(mean), c2q, c1);
}

cudaError_t launch_group_sums(const float *ws_absmax, int64_t nb, double *ws_gsum, cudaStream_t st) {
  const int64_t ng = (nb + 255) / 256;
  return launch_k(k_group_sums, dim3(static_cast<unsigned>(ng)), dim3(256), 0, st, 1, ws_absmax, nb, ws_gsum);
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *c2q, const float *c1, const float *mean,
                              int64_t nb, const Nf4Levels &lv, uint16_t *out, cudaStream_t st) {
  const int64_t grid = (nb + 255) / 256;
  return launch_k(k_dequant, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, 1, codes, c2q, c1, mean, nb, lv,
                  out);
}

}  // namespace qlora
