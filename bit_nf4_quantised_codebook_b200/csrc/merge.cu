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
// k_merge_quant: persistent CTAs of 128 threads; a tile is 128 rows n x 64
// columns k (one 64-weight block per row), so thread = TMEM lane = W row = one block:
//   - thread 0 loads the tile's slices of B (MN-major: n contiguous) and A
//     (K-major: j contiguous) by TMA, then issues rpad/16 tcgen05 MMAs
//     (M = 128 rows n, N = 64 columns k, K = 16) into a 64-column TMEM
//     accumulator: sum_j B[j, n]·A[k, j] in float32 (rpad = r rounded up to 16;
//     rows of B and columns of A beyond r arrive as zeros);
//   - as soon as those MMAs complete it loads the next tile's slices into the
//     same shared memory, and every thread loads the old codes and block
//     constant of its next block, so both are in flight during the epilogue;
//   - the epilogue reads the row's accumulator 32 columns at a time, decodes ŵ
//     with the block's lookup table, forms the merged bfloat16 values and codes
//     the block: absmax, exact quotient, nearest level by the bucket table,
//     nibble packing — the quantiser's own steps (nf4_quant.cuh).
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

constexpr int kRows = 128;                     // rows n per tile (MMA M)
constexpr int kCols = 64;                      // columns k per tile (MMA N): one block per row
constexpr uint32_t kBSlice = 16384;            // B: 64 of r x 128 rows n (two 64-wide boxes)
constexpr uint32_t kASlice = 8192;             // A: 64 rows k x 64 of r
constexpr uint32_t kTabBytes = kBuckets * 32 * sizeof(CodeBucket);
constexpr unsigned long long kMergeDrainNs = 1000000000ull;
constexpr uint32_t kIdesc = idesc_bf16(kRows, kCols, true, false);  // A operand (B's slice) MN-major
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

// The old codes and block constant of one block (row n, 64-column block kb).
struct BlockIn {
  uint32_t words[8];
  float c2h;
  bool valid;
};

__device__ __forceinline__ void load_block(const MergeArgs &p, int64_t tile, int64_t tiles, int row, float mu,
                                           BlockIn &in) {
  const int64_t kblocks = p.K / kCols;
  const int64_t n = (tile / kblocks) * kRows + row;
  in.valid = tile < tiles && n < p.N;
  in.c2h = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) in.words[i] = 0x77777777u;
  if (in.valid) {
    const int64_t b = n * kblocks + tile % kblocks;
    const uint4 q0 = ld_v4(p.codes_in + b * 32), q1 = ld_v4(p.codes_in + b * 32 + 16);
    in.words[0] = q0.x, in.words[1] = q0.y, in.words[2] = q0.z, in.words[3] = q0.w;
    in.words[4] = q1.x, in.words[5] = q1.y, in.words[6] = q1.z, in.words[7] = q1.w;
    in.c2h = reconstruct_c2(p.c2q_in[b], p.c1_in[b >> 8], mu);
  }
}

__global__ void __launch_bounds__(128, 4) k_merge_quant(const __grid_constant__ CUtensorMap map_b,
                                                         const __grid_constant__ CUtensorMap map_a,
                                                         const __grid_constant__ MergeArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sB = smem;                          // nch x (two 64-row halves of n, 8 KiB each)
  uint8_t *sA = smem + p.nch * kBSlice;        // nch x 64 rows k x 128 B
  CodeBucket(*s_tab)[32] = reinterpret_cast<CodeBucket(*)[32]>(smem + p.nch * (kBSlice + kASlice));
  __shared__ CodeBucket s_bucket[kBuckets];
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = 32 * warp + lane;
  const int64_t kblocks = p.K / kCols;
  const int64_t tiles = ((p.N + kRows - 1) / kRows) * kblocks;

  if (warp == 0) {
    tmem_alloc(&tmem_slot, kCols);
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
  // bucket table: 64 entries, then one copy per lane (conflict-free lookups)
  if (threadIdx.x < kBuckets) s_bucket[threadIdx.x] = make_bucket(threadIdx.x, p.thr.t);
  __syncthreads();
  for (int i = threadIdx.x; i < kBuckets * 32; i += blockDim.x) s_tab[i >> 5][i & 31] = s_bucket[i >> 5];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * warp) << 16);

  pdl_wait();
  pdl_launch_dependents();

  auto issue_loads = [&](int64_t tile) {
    const int n0 = static_cast<int>((tile / kblocks) * kRows), k0 = static_cast<int>((tile % kblocks) * kCols);
    mbar_arrive_expect_tx(&tma_bar, static_cast<uint32_t>(p.nch) * (kBSlice + kASlice));
    for (int c = 0; c < p.nch; ++c) {
      tma_load_2d(sB + c * kBSlice, &map_b, &tma_bar, n0, 64 * c);
      tma_load_2d(sB + c * kBSlice + kBSlice / 2, &map_b, &tma_bar, n0 + 64, 64 * c);
      tma_load_2d(sA + c * kASlice, &map_a, &tma_bar, 64 * c, k0);
    }
  };

  const float mu = *p.mean_in;
  int64_t tile = blockIdx.x;
  int pending_tma = -1, pending_mma = -1;  // (thread 0) parity of an issued, not yet awaited, phase
  if (threadIdx.x == 0 && tile < tiles) {
    issue_loads(tile);
    pending_tma = 0;
  }
  BlockIn cur;
  load_block(p, tile, tiles, row, mu, cur);
  bool bad = false;
  for (uint32_t it = 0; tile < tiles; tile += gridDim.x, ++it) {
    const uint32_t ph = it & 1;
    if (threadIdx.x == 0 && mbar_wait_bounded(&tma_bar, ph, &abort_flag, p.dev_err, p.timeout_ns)) {
      pending_tma = -1;
      tc_fence_after();
      const uint32_t a_base = smem_u32(sB), b_base = smem_u32(sA);
      for (int kk = 0; kk < p.ksteps; ++kk) {
        const uint64_t ad = smem_desc_sw128(a_base + (kk >> 2) * kBSlice + (kk & 3) * 2048, kBSlice / 2, 1024);
        const uint64_t bd = smem_desc_sw128(b_base + (kk >> 2) * kASlice + (kk & 3) * 32, 16, 1024);
        mma_bf16_ss(tmem, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(&mma_bar);
      pending_mma = static_cast<int>(ph);
    }
    const bool ok = mbar_wait_bounded(&mma_bar, ph, &abort_flag, p.dev_err, p.timeout_ns);
    if (__syncthreads_or(!ok)) break;  // the same decision in every thread
    tc_fence_after();
    const int64_t next = tile + gridDim.x;
    if (threadIdx.x == 0) {
      pending_mma = -1;
      if (next < tiles) {  // the MMAs are done with the shared slices: refill them now
        issue_loads(next);
        pending_tma = static_cast<int>((it + 1) & 1);
      }
    }
    BlockIn nxt;
    load_block(p, next, tiles, row, mu, nxt);

    const BlockLut lut = make_lut(cur.c2h, p.lv);
    uint32_t merged[32];  // bf16x2 words of W_eff, element 2i in the low half of word i
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t acc[32];
      tmem_ld32(trow + 32 * half, acc);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[4];
        decode8(cur.words[4 * half + c], lut, o);
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
    tc_fence_before();
    if (cur.valid) {
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
      const int64_t n = (tile / kblocks) * kRows + row, kb = tile % kblocks;
      const int64_t b = n * kblocks + kb;
      uint4 *cp = reinterpret_cast<uint4 *>(p.codes_out + b * 32);
      cp[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      cp[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      p.absmax[b] = amax;
      if (p.w_merged) {
        uint4 *wp = reinterpret_cast<uint4 *>(p.w_merged + n * p.K + kb * kCols);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          wp[i] = make_uint4(merged[4 * i], merged[4 * i + 1], merged[4 * i + 2], merged[4 * i + 3]);
      }
    }
    __syncthreads();  // every row has read the accumulator: the next MMAs may overwrite it
    tc_fence_after();
    cur = nxt;
  }
  if (bad && p.dev_err) atomicOr(p.dev_err, QLORA_DEVERR_NONFINITE);

  if (threadIdx.x == 0 && (pending_tma >= 0 || pending_mma >= 0)) {
    // a wait gave up: what was issued must land before TMEM and shared memory go away
    int dummy = 0;
    if (pending_tma >= 0) mbar_wait_bounded(&tma_bar, static_cast<uint32_t>(pending_tma), &dummy, nullptr, kMergeDrainNs);
    if (pending_mma >= 0) mbar_wait_bounded(&mma_bar, static_cast<uint32_t>(pending_mma), &dummy, nullptr, kMergeDrainNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace

size_t merge_smem_bytes(int r) {
  const int nch = (r + 63) / 64;
  return static_cast<size_t>(nch) * (kBSlice + kASlice) + kTabBytes + 1024;
}

cudaError_t launch_merge_requantize(const qlora_nf4_weight &w, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const qlora_nf4_weight &out, uint16_t *w_merged, float *ws_absmax,
                                    double *ws_gsum, int64_t gsum_size, const Nf4Levels &lv,
                                    const Nf4Thresholds &thr, int *dev_err, unsigned long long timeout_ns,
                                    cudaStream_t st) {
  CUtensorMap mb, ma;
  // B [r, N] read MN-major (box 64 n x 64 j); A [K, r] read K-major (box 64 j x 64 k)
  if (!map_bf16_mn(&mb, B, w.N, r) || !map_bf16_kmajor(&ma, A, r, w.K, kCols)) return cudaErrorInvalidValue;
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
  // At most 5 CTAs fit on an SM by shared memory (>= 40 KiB each), so their
  // 64-column TMEM allocations (512 columns per SM) never wait on one another.
  static_assert(kBSlice + kASlice + kTabBytes >= 40 * 1024, "at most 5 CTAs per SM");
  cudaError_t e = cudaFuncSetAttribute(k_merge_quant, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // Several CTAs per SM need the largest shared-memory share of the on-chip memory;
  // without this hint the driver may configure room for only one.
  e = cudaFuncSetAttribute(k_merge_quant, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // CTAs resident per SM, from registers, shared memory and TMEM columns.
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, k_merge_quant)) != cudaSuccess) return e;
  int dev = 0, sms = 148, smem_sm = 0, reserved = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
  const int by_regs = regs_warp > 0 ? 65536 / (regs_warp * 4) : 1;
  const int by_smem = static_cast<int>(smem_sm / (smem + fa.sharedSizeBytes + reserved));
  int per_sm = by_regs < by_smem ? by_regs : by_smem;
  if (per_sm > 512 / kCols) per_sm = 512 / kCols;
  if (per_sm < 1) per_sm = 1;
  const int64_t tiles = ((w.N + kRows - 1) / kRows) * (w.K / kCols);
  const int64_t slots = static_cast<int64_t>(per_sm) * sms;
  const int64_t grid = tiles < slots ? tiles : slots;
  const TimingHooks &hk = timing_hooks();
  if (hk.fwd_begin) cudaEventRecord(hk.fwd_begin, st);
  e = launch_k(k_merge_quant, dim3(static_cast<unsigned>(grid)), dim3(128), smem, st, 1, mb, ma, a);
  if (e != cudaSuccess) return e;
  if (hk.fwd_end) cudaEventRecord(hk.fwd_end, st);
  const int64_t nb = w.N * w.K / 64;
  e = launch_group_sums(ws_absmax, nb, ws_gsum, st);
  if (e != cudaSuccess) return e;
  return launch_mean_and_double_quant(ws_absmax, nb, ws_gsum, gsum_size, out.mean, out.c2q, out.c1, st);
}

}  // namespace qlora
