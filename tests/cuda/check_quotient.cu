// Exhaustive check of the quantiser's fast quotient and bucket code against
// CUDA's correctly rounded division and a plain count of thresholds.
//
// Domain: every positive normal bfloat16 a >= 2^-100 (the quantiser's fast-path
// range for the block absmax) and every finite bfloat16 x with |x| <= a.
// For each pair:
//   ref  = __fdiv_rn(x, a);            code_ref  = #{i : ref >= t_i}
//   fast = quotient_rn(x, a, RN(1/a));  code_fast = bucket_code(fast, table)
//                                       code_centred = lane_centred_code(fast, centred table)
// Counts pairs whose codes differ (must be 0, for both tables) and pairs with
// |ref| >= 1/32 (every threshold is at least 0.0398 in magnitude, so only those
// can decide a code) whose quotients differ in any bit (must be 0).
//
// usage: check_quotient t0 .. t14   (thresholds as float32 hex bit patterns)
#include <cstdio>
#include <cstdlib>
#include <cuda_runtime.h>
#include "nf4_quant.cuh"

using namespace qlora;

struct Thr {
  float t[15];
};

__global__ void check(Thr thr, unsigned long long *bad_code, unsigned long long *bad_q, unsigned long long *pairs,
                      unsigned long long *bad_centred) {
  __shared__ CodeBucket tab[kBuckets];
  __shared__ CodeBucket ctab[kCentredBuckets][32];
  if (threadIdx.x < kBuckets) tab[threadIdx.x] = make_bucket(threadIdx.x, thr.t);
  for (int i = threadIdx.x; i < kCentredBuckets * 32; i += blockDim.x)
    ctab[i >> 5][i & 31] = make_bucket_centred(i >> 5, thr.t);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  unsigned long long n_centred = 0;
  const uint32_t a_bits = 0x0D80u + blockIdx.x;  // 2^-100 upwards
  const float a = __uint_as_float(a_bits << 16);
  const float ra = __frcp_rn(a);
  unsigned long long n_code = 0, n_q = 0, n = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    const float x = __uint_as_float(xb << 16);
    if (!(fabsf(x) <= a)) continue;  // also skips NaN
    const float ref = __fdiv_rn(x, a);
    const float fast = quotient_rn(x, a, ra);
    uint32_t cref = 0;
    for (int i = 0; i < 15; ++i) cref += ref >= thr.t[i] ? 1u : 0u;
    const uint32_t cfast = bucket_code(fast, tab);
    const uint32_t ccent = lane_centred_code(fast, ctab, lane);
    n += 1;
    n_code += cref != cfast;
    n_centred += cref != ccent;
    n_q += (fabsf(ref) >= 0.03125f) && (__float_as_uint(ref) != __float_as_uint(fast));
  }
  atomicAdd(bad_code, n_code);
  atomicAdd(bad_q, n_q);
  atomicAdd(pairs, n);
  atomicAdd(bad_centred, n_centred);
}

int main(int argc, char **argv) {
  if (argc != 16) {
    fprintf(stderr, "need 15 thresholds\n");
    return 2;
  }
  Thr thr;
  for (int i = 0; i < 15; ++i) {
    const unsigned v = static_cast<unsigned>(strtoul(argv[1 + i], nullptr, 16));
    memcpy(&thr.t[i], &v, 4);
  }
  unsigned long long *d = nullptr;
  if (cudaMalloc(&d, 4 * sizeof(unsigned long long)) != cudaSuccess) return 3;
  cudaMemset(d, 0, 4 * sizeof(unsigned long long));
  const unsigned n_a = 0x7F7Fu - 0x0D80u + 1;  // up to the largest finite bfloat16
  check<<<n_a, 256>>>(thr, d, d + 1, d + 2, d + 3);
  unsigned long long h[4] = {0, 0, 0, 0};
  const cudaError_t e = cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    fprintf(stderr, "cuda error %s\n", cudaGetErrorString(e));
    return 4;
  }
  printf("pairs=%llu bad_code=%llu bad_quotient=%llu bad_centred=%llu\n", h[2], h[0], h[1], h[3]);
  cudaFree(d);
  return 0;
}
