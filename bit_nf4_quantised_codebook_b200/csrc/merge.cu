// merge.cu — merge a trained adapter into the NF4 base weight and requantise.
//
// "QLoRA: quantising the part you are not training" (addaly.com), §What it
// costs: an adapter trained against the quantised base can be merged into it,
// at the price of requantising the merged weight.  The weight the adapter adds
// follows from the layer of "QLoRA: Efficient Finetuning of Quantized LLMs"
// (intuitivepapers.ai), §The QLoRA layer, end to end (Y = X·Ŵᵀ + s·(X·A)·B):
//     W_eff[n, k] = bf16_rn( fmaf(s, sum_j A[k, j]·B[j, n], ŵ[n, k]) ),
// and W_eff is quantised exactly as the quantiser does it (64-element absmax
// blocks, NF4 codes, then the double quantisation of the block constants).
//
// k_merge_quant, one CTA of 128 threads per 128 (W rows n) x 128 (columns k) tile:
//   - thread 0 loads the tile's slices of B (MN-major: n contiguous) and A
//     (K-major: j contiguous) by TMA, then issues rpad/16 tcgen05 MMAs
//     (M = 128 rows n, N = 128 columns k, K = 16) into a 128-column TMEM
//     accumulator: sum_j B[j, n]·A[k, j] in float32 (rpad = r rounded up to 16;
//     rows of B and columns of A beyond r arrive as zeros);
//   - meanwhile each thread loads the old codes and block constants of its
//     row's two 64-element blocks (thread = TMEM lane = W row);
//   - each thread then reads its row's accumulator columns 32 at a time,
//     decodes ŵ with the block's lookup table, forms the merged bfloat16 values
//     and codes the block: absmax, exact quotient, nearest level by the bucket
//     table, nibble packing — the quantiser's own steps (nf4_quant.cuh).
// The float32 absmax of every block goes to the workspace; the group sums, the
// fixed-order mean and the E4M3 codes follow in quantize.cu's kernels.
//
// In place: out may be the input weight itself.  Each thread reads the codes
// and constants of its blocks before it writes codes, and the constants are
// rewritten only by the later kernels, which wait for this one to finish.
//
// Every wait is bounded: on timeout the CTA raises QLORA_DEVERR_TIMEOUT, skips
// its epilogue, drains the copies and MMAs it issued, frees TMEM and exits.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "internal.h"
#include "launch.cuh"
#include "linear_plan.h"
#include "nf4_decode.cuh"
#include "nf4_quant.cuh"
#include "ptx.cuh"

namespace qlora {
namespace {

constexpr int kTile = 128;                     // rows n and columns k per CTA
constexpr uint32_t kChunkBytes = 16384;        // one 64-wide slice of r: 128 rows x 128 B
constexpr uint32_t kTabBytes = kBuckets * 32 * sizeof(CodeBucket);
constexpr unsigned long long kMergeDrainNs = 1000000000ull;
constexpr uint32_t kIdesc = idesc_bf16(kTile, kTile, true, false);  // A operand (B's slice) MN-major
static_assert(kTabBytes == 16384, "bucket table is 16 KiB");

struct MergeArgs {
  const uint8_t *codes_in;
  const uint8_t *c2q_in;
  const float *c1_in;
  const float *mean_in;
  uint8_t *codes_out;
  float *absmax;       // workspace, one float per block
  uint16_t *w_merged;  // optional N x K bfloat16
  int64_t N, K;
  int nch;     // 64-wide slices of r
  int ksteps;  // MMAs of K = 16
  float s;
  Nf4Levels lv;
  Nf4Thresholds thr;
  int *dev_err;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ uint4 ld_v4(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

__global__ void __launch_bounds__(128) k_merge_quant(const __grid_constant__ CUtensorMap map_b,
                                                      const __grid_constant__ CUtensorMap map_a,
                                                      const __grid_constant__ MergeArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sB = smem;                               // nch x (two 64-row halves of n, 8 KiB each)
  uint8_t *sA = smem + p.nch * kChunkBytes;         // nch x 128 rows k x 128 B
  CodeBucket(*s_tab)[32] = reinterpret_cast<CodeBucket(*)[32]>(smem + 2 * p.nch * kChunkBytes);
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles_k = (p.K + kTile - 1) / kTile;
  const int64_t n0 = (static_cast<int64_t>(blockIdx.x) / tiles_k) * kTile;
  const int64_t k0 = (static_cast<int64_t>(blockIdx.x) % tiles_k) * kTile;

  if (warp == 0) {
    tmem_alloc(&tmem_slot, kTile);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    mbar_init(&tma_bar, 1);
    mbar_init(&mma_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_a);
  }
  for (int i = threadIdx.x; i < kBuckets * 32; i += blockDim.x) s_tab[i >> 5][i & 31] = make_bucket(i >> 5, p.thr.t);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  pdl_wait();
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&tma_bar, static_cast<uint32_t>(p.nch) * 2 * kChunkBytes);
    for (int c = 0; c < p.nch; ++c) {
      tma_load_2d(sB + c * kChunkBytes, &map_b, &tma_bar, static_cast<int>(n0), 64 * c);
      tma_load_2d(sB + c * kChunkBytes + kChunkBytes / 2, &map_b, &tma_bar, static_cast<int>(n0) + 64, 64 * c);
      tma_load_2d(sA + c * kChunkBytes, &map_a, &tma_bar, 64 * c, static_cast<int>(k0));
    }
  }

  // The old codes and constants of this thread's two blocks (row n, 64-column blocks kb0, kb0 + 1).
  const int64_t n = n0 + 32 * warp + lane;
  const int64_t kblocks = p.K / 64;
  const int64_t kb0 = k0 / 64;
  bool valid[2];
  uint32_t words[2][8];
  float c2h[2];
  const float mu = *p.mean_in;
#pragma unroll
  for (int bb = 0; bb < 2; ++bb) {
    valid[bb] = n < p.N && kb0 + bb < kblocks;
    c2h[bb] = 0.f;
    if (valid[bb]) {
      const int64_t b = n * kblocks + kb0 + bb;
      const uint4 q0 = ld_v4(p.codes_in + b * 32), q1 = ld_v4(p.codes_in + b * 32 + 16);
      words[bb][0] = q0.x, words[bb][1] = q0.y, words[bb][2] = q0.z, words[bb][3] = q0.w;
      words[bb][4] = q1.x, words[bb][5] = q1.y, words[bb][6] = q1.z, words[bb][7] = q1.w;
      c2h[bb] = reconstruct_c2(p.c2q_in[b], p.c1_in[b >> 8], mu);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) words[bb][i] = 0x77777777u;
    }
  }

  bool issued = false, mma_issued = false;
  if (threadIdx.x == 0) {
    issued = true;
    if (mbar_wait_bounded(&tma_bar, 0, &abort_flag, p.dev_err, p.timeout_ns)) {
      tc_fence_after();
      const uint32_t a_base = smem_u32(sB), b_base = smem_u32(sA);
      for (int kk = 0; kk < p.ksteps; ++kk) {
        const uint32_t off = static_cast<uint32_t>(kk >> 2) * kChunkBytes;
        const uint64_t ad = smem_desc_sw128(a_base + off + (kk & 3) * 2048, kChunkBytes / 2, 1024);
        const uint64_t bd = smem_desc_sw128(b_base + off + (kk & 3) * 32, 16, 1024);
        mma_bf16_ss(tmem, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(&mma_bar);
      mma_issued = true;
    }
  }

  bool ok = mbar_wait_bounded(&mma_bar, 0, &abort_flag, p.dev_err, p.timeout_ns);
  ok = __all_sync(0xFFFFFFFFu, ok);  // the accumulator loads below are warp-wide
  tc_fence_after();
  bool bad = false;
  if (ok) {
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
      const BlockLut lut = make_lut(c2h[bb], p.lv);
      uint32_t merged[32];  // bf16x2 words of W_eff, element 2i in the low half of word i
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t acc[32];
        tmem_ld32(trow + 64 * bb + 32 * half, acc);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[4];
          decode8(words[bb][4 * half + c], lut, o);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = 8 * c + 2 * q;  // element within this half
            const float w0 = __uint_as_float(o[q] << 16), w1 = __uint_as_float(o[q] & 0xFFFF0000u);
            const float m0 = __fmaf_rn(p.s, __uint_as_float(acc[e]), w0);
            const float m1 = __fmaf_rn(p.s, __uint_as_float(acc[e + 1]), w1);
            merged[16 * half + 4 * c + q] = pack_bf16x2(m0, m1);
          }
        }
      }
      if (!valid[bb]) continue;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float a0 = fabsf(__uint_as_float(merged[i] << 16)), a1 = fabsf(__uint_as_float(merged[i] & 0xFFFF0000u));
        bad |= !(a0 <= 3.402823466e38f) || !(a1 <= 3.402823466e38f);  // Inf or NaN (fmaxf would drop a NaN)
        amax = fmaxf(amax, fmaxf(a0, a1));
      }
      uint32_t packed[8];
      if (amax >= kFastQuotientMinAbsmax) {
        const float ra = __frcp_rn(amax);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t u = merged[4 * c + i];
            const uint32_t hi = lane_bucket_code(quotient_rn(__uint_as_float(u << 16), amax, ra), s_tab, lane);
            const uint32_t lo = lane_bucket_code(quotient_rn(__uint_as_float(u & 0xFFFF0000u), amax, ra), s_tab, lane);
            pk |= ((hi << 4) | lo) << (8 * i);
          }
          packed[c] = pk;
        }
      } else if (amax > 0.f) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t u = merged[4 * c + i];
            const uint32_t hi = nf4_code(__fdiv_rn(__uint_as_float(u << 16), amax), p.thr);
            const uint32_t lo = nf4_code(__fdiv_rn(__uint_as_float(u & 0xFFFF0000u), amax), p.thr);
            pk |= ((hi << 4) | lo) << (8 * i);
          }
          packed[c] = pk;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) packed[c] = 0x77777777u;  // all-zero block: the zero level
      }
      const int64_t b = n * kblocks + kb0 + bb;
      uint4 *cp = reinterpret_cast<uint4 *>(p.codes_out + b * 32);
      cp[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      cp[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      p.absmax[b] = amax;
      if (p.w_merged) {
        uint4 *wp = reinterpret_cast<uint4 *>(p.w_merged + n * p.K + (kb0 + bb) * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          wp[i] = make_uint4(merged[4 * i], merged[4 * i + 1], merged[4 * i + 2], merged[4 * i + 3]);
      }
    }
  }
  if (bad && p.dev_err) atomicOr(p.dev_err, QLORA_DEVERR_NONFINITE);

  if (issued && abort_flag) {
    // a wait gave up: the copies (and MMAs) issued must land before TMEM and shared memory go away
    int dummy = 0;
    mbar_wait_bounded(&tma_bar, 0, &dummy, nullptr, kMergeDrainNs);
    if (mma_issued) mbar_wait_bounded(&mma_bar, 0, &dummy, nullptr, kMergeDrainNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTile);
  }
}

}  // namespace

size_t merge_smem_bytes(int r) {
  const int nch = (r + 63) / 64;
  return 2 * static_cast<size_t>(nch) * kChunkBytes + kTabBytes + 1024;
}

cudaError_t launch_merge_requantize(const qlora_nf4_weight &w, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const qlora_nf4_weight &out, uint16_t *w_merged, float *ws_absmax,
                                    double *ws_gsum, int64_t gsum_size, const Nf4Levels &lv,
                                    const Nf4Thresholds &thr, int *dev_err, unsigned long long timeout_ns,
                                    cudaStream_t st) {
  CUtensorMap mb, ma;
  // B [r, N] read MN-major (box 64 n x 64 j); A [K, r] read K-major (box 64 j x 128 k)
  if (!map_bf16_mn(&mb, B, w.N, r) || !map_bf16_kmajor(&ma, A, r, w.K, kTile)) return cudaErrorInvalidValue;
  MergeArgs a;
  a.codes_in = w.codes;
  a.c2q_in = w.c2q;
  a.c1_in = w.c1;
  a.mean_in = w.mean;
  a.codes_out = out.codes;
  a.absmax = ws_absmax;
  a.w_merged = w_merged;
  a.N = w.N;
  a.K = w.K;
  a.nch = (r + 63) / 64;
  a.ksteps = (r + 15) / 16;
  a.s = s;
  a.lv = lv;
  a.thr = thr;
  a.dev_err = dev_err;
  a.timeout_ns = timeout_ns;
  const size_t smem = merge_smem_bytes(r);
  // At most 4 CTAs fit on an SM by shared memory (>= 48 KiB each), so their
  // 128-column TMEM allocations (512 columns per SM) never wait on one another.
  static_assert(2 * kChunkBytes + kTabBytes >= 48 * 1024, "at most 4 CTAs per SM");
  cudaError_t e = cudaFuncSetAttribute(k_merge_quant, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((w.N + kTile - 1) / kTile) * ((w.K + kTile - 1) / kTile);
  if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const TimingHooks &hk = timing_hooks();
  if (hk.fwd_begin) cudaEventRecord(hk.fwd_begin, st);
  e = launch_k(k_merge_quant, dim3(static_cast<unsigned>(tiles)), dim3(128), smem, st, 1, mb, ma, a);
  if (e != cudaSuccess) return e;
  if (hk.fwd_end) cudaEventRecord(hk.fwd_end, st);
  const int64_t nb = w.N * w.K / 64;
  e = launch_group_sums(ws_absmax, nb, ws_gsum, st);
  if (e != cudaSuccess) return e;
  return launch_mean_and_double_quant(ws_absmax, nb, ws_gsum, gsum_size, out.mean, out.c2q, out.c1, st);
}

}  // namespace qlora
