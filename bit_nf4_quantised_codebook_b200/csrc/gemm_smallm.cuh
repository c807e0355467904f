// gemm_smallm.cuh — forward dequant GEMM for decode-sized batches (M <= 64),
// with the dequantised weight as the TMEM operand of the MMA.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §The QLoRA layer, end to end: Y = X·W_hatᵀ + sT·B with sT = bf16(s·X·A).
// Computed transposed per CTA:
//   Yᵀ[128 W rows x NT tokens] = W_hat[128 x K] · Xᵀ  +  Bᵀ[128 x r] · sTᵀ
// W rows sit on the MMA M side (128 per CTA) and the tokens on the N side
// (NT = M rounded up to 16, at most 64), so at this size neither MMA work nor
// activation traffic is spent on padding and the kernel streams the 4-bit
// weight once.  Each dequant thread owns one W row, which is its TMEM lane: per
// K step it expands that row's 64-element block with byte permutes
// (nf4_decode.cuh) and writes the 32 packed bf16 pairs into the step's TMEM A
// stage with one tcgen05.st — no shared-memory round trip, no proxy fence.
// The activation tile (K-major, 128-byte swizzle) is the MMA's B operand from
// shared memory; the accumulator lives in TMEM.
//
// K is split across the S CTAs of a 1 x 1 x S cluster (S <= 8).  Rank 0 also
// runs the adapter product Bᵀ·sTᵀ as extra K steps on the tensor cores (both
// operands by TMA: B read MN-major, sT K-major).  Every CTA parks its float32
// partial in shared memory; after a cluster barrier each rank sums the S
// partials of its share of the 128 columns in rank order through distributed
// shared memory and writes bf16 Y.
//
// Programmatic dependent launch: the kernel launched just before this one
// writes sT; everything else it reads (X, the stored weight, B) was written
// further back and is complete when this grid starts (launch.cuh).  So only
// rank 0's producer waits on the predecessor, right before loading sT, and the
// main loop overlaps the predecessor's tail.
//
// Roles (352 threads, 2 CTAs per SM): warp 0 TMA producer, warp 1 TMEM
// allocator and MMA issuer of dequant group 0, warps 2..9 two dequant groups of
// 4 warps (one warp per TMEM lane quadrant) taking alternate K steps, warp 10
// the MMA issuer of group 1.  Each issuer accumulates its group's steps in its
// own TMEM accumulator (two MMA streams per CTA; a single issuing thread paces
// the MMAs of 128 x NT x 16 well below the tensor pipe's rate), and the two are
// added when the partial is parked.  The E4M3 block constants
// and fp32 group scales of the CTA's weight slice are staged in shared memory
// once, by the dequant threads, with coalesced loads.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "gemm.cuh"
#include "linear_plan.h"

namespace qlora {

constexpr int kSmallC1Max = 260;
// Pipeline waits sleep in the barrier (up to this long per poll) instead of
// spinning, so waiting warps leave the issue slots and the integer pipe to the
// decoding ones.
constexpr uint32_t kSmallWaitHintNs = 1000;     // group scales a CTA can touch: (127·512 + 64)/256 + 2, rounded up

template <int NT_, int GROUPS_>
struct SmallCfg {
  static constexpr int NT = NT_;          // tokens on the MMA N side (multiple of 16, <= 64)
  static constexpr int GROUPS = GROUPS_;  // dequant groups of 4 warps
  static constexpr int KB = NT == 64 ? 1 : 2;  // 64-element K blocks per pipeline step
  static constexpr int X_BYTES = NT * 128;       // one block's activation tile: NT rows x 64 bf16, 128-byte swizzle
  static constexpr int C_ROW = 32 * KB;          // bytes of packed codes per W row and step
  static constexpr int C_BYTES = 128 * C_ROW;    // swizzled with the C_ROW-byte TMA swizzle
  static constexpr int STAGE_BYTES = KB * X_BYTES + C_BYTES;
  static constexpr int ACC_COLS = NT < 32 ? 32 : NT;
  static constexpr int TMEM_COLS = 256;
  static constexpr int NACC = 2;                 // one accumulator per dequant group and its MMA issuer
  static constexpr int TSLOTS_FIT = (TMEM_COLS - NACC * ACC_COLS) / (32 * KB);
  static constexpr int TSLOTS = TSLOTS_FIT < 6 / KB ? TSLOTS_FIT : 6 / KB;  // TMEM A slots (KB x 32 columns each)
  // Shared-memory ring: an even number of stages, so that with two dequant groups taking
  // alternate steps every stage belongs to one group, and each full-barrier phase is
  // awaited in order by a single consumer (a parity wait only tells apart the phase it
  // waits for and the one before it).
  static constexpr int STAGES = STAGE_BYTES <= 12288 ? 6 : 4;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int LA_BYTES = 16384;    // Bᵀ tile: 128 W rows x 64 adapter columns, MN-major
  static constexpr int LX_BYTES = X_BYTES;  // sT tile: NT tokens x 64 adapter columns, K-major
  static constexpr int Q8_STRIDE_MAX = kSmallMaxKIters + 4;
  static constexpr int OFF_LA = RING_BYTES;
  static constexpr int OFF_LX = OFF_LA + LA_BYTES;
  static constexpr int OFF_Q8 = OFF_LX + LX_BYTES;
  static constexpr int OFF_C1 = OFF_Q8 + 128 * Q8_STRIDE_MAX;
  static constexpr int OFF_BAR = (OFF_C1 + kSmallC1Max * 4 + 7) & ~7;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr int PSTRIDE = 128 + 4;  // floats per token row of the parked partial
  static constexpr int P_BYTES = NT * PSTRIDE * 4;
  static constexpr int DQ_THREADS = 128 * GROUPS;
  static constexpr int ISSUER1_WARP = 2 + 4 * GROUPS;  // the second MMA issuer, after the dequant warps
  static constexpr int NUM_THREADS = 64 + DQ_THREADS + 32;
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 64, "token tile");
  static_assert(NACC * ACC_COLS + TSLOTS * 32 * KB <= TMEM_COLS, "TMEM budget");
  static_assert(GROUPS == NACC, "each dequant group has its own issuer and accumulator");
  static_assert(STAGES >= TSLOTS, "a slot's barrier phase is never overtaken before its waiter checks it");
  static_assert(STAGE_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(P_BYTES <= RING_BYTES, "the partial is parked in the drained ring");
  static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");
  static_assert(GROUPS <= TSLOTS, "each group's next slot is at most one lap ahead");
  static_assert(STAGES % GROUPS == 0, "every ring stage belongs to one dequant group");
};

struct SmallParams {
  int M;              // tokens (<= NT)
  int N;              // W rows = output columns
  int k_iters;        // K steps per split
  int k_iters_total;  // K / 64
  int splits;         // cluster size along z
  int q8_stride;      // bytes per row of the staged block constants (4 · odd)
  int q8_words;       // 1: stage the constants as 4-byte words (K/64 and k_iters multiples of 4)
  int lora_r;         // adapter rank (multiple of 8, <= 256)
  const uint8_t *c2q;
  const float *c1;
  const float *mean;
  Nf4Levels lv;
  uint32_t k_shr16, k_shr1;
  uint16_t *Y;  // bf16 [M, N]
  int *dev_err;
  unsigned long long timeout_ns;
};

// maps: x = X [M, K] box {64, NT}; codes = [N, K/2] box {64, 128}, 64-byte swizzle;
// st = sT [M, r] box {64, NT}; b = B [r, N] read MN-major, box {64, 64}.
template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 2)
    gemm_smallm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
                       const __grid_constant__ CUtensorMap map_st, const __grid_constant__ CUtensorMap map_b,
                       const SmallParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *full = bars;               // activation + code tiles landed
  uint64_t *empty = full + C::STAGES;  // the step's MMAs done: smem stage and TMEM A stage free
  uint64_t *ready = empty + C::STAGES; // a dequant group wrote the TMEM A stage (4 warp arrivals)
  uint64_t *lfull = ready + C::STAGES; // adapter tiles landed
  uint64_t *lempty = lfull + 1;        // adapter MMAs done
  uint64_t *acc_full = lempty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *q8s = smem + C::OFF_Q8;
  float *c1s = reinterpret_cast<float *>(smem + C::OFF_C1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128;
  const int kbt = p.k_iters_total;
  const int kb_begin = blockIdx.z * p.k_iters;
  int n_main = kbt - kb_begin;
  if (n_main > p.k_iters) n_main = p.k_iters;
  if (n_main < 0) n_main = 0;
  const int n_ss = (n_main + C::KB - 1) / C::KB;  // pipeline steps of KB blocks
  const bool lora = blockIdx.z == 0 && p.lora_r > 0;
  const int n_lora = lora ? (p.lora_r + 63) / 64 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 4);
    }
    mbar_init(lfull, 1);
    mbar_init(lempty, 1);
    mbar_init(acc_full, C::NACC);  // one commit per issuer
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_codes);
    if (lora) {
      tma_prefetch_desc(&map_st);
      tma_prefetch_desc(&map_b);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < n_ss; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait_bounded_sleep(&empty[s], ph ^ 1, abort_flag, p.dev_err, p.timeout_ns, kSmallWaitHintNs)) break;
        uint8_t *st = smem + s * C::STAGE_BYTES;
        const int kb = kb_begin + j * C::KB;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
#pragma unroll
        for (int b = 0; b < C::KB; ++b) tma_load_2d(st + b * C::X_BYTES, &map_x, &full[s], (kb + b) * 64, 0);
        tma_load_2d(st + C::KB * C::X_BYTES, &map_codes, &full[s], kb * 32, n0);
        issued = j + 1;
      }
      int lissued = 0;
      if (lora && issued == n_ss) {
        pdl_wait();  // sT is the predecessor's output
        for (int c = 0; c < n_lora; ++c) {
          if (!mbar_wait_bounded(lempty, (c & 1) ^ 1, abort_flag, p.dev_err, p.timeout_ns)) break;
          mbar_arrive_expect_tx(lfull, C::LA_BYTES + C::LX_BYTES);
          tma_load_2d(smem + C::OFF_LA, &map_b, lfull, n0, c * 64);
          tma_load_2d(smem + C::OFF_LA + 8192, &map_b, lfull, n0 + 64, c * 64);
          tma_load_2d(smem + C::OFF_LX, &map_st, lfull, c * 64, 0);
          lissued = c + 1;
        }
      }
      // drain: every issued load lands before the CTA may exit
      for (int it = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; it < issued; ++it) {
        int dummy = 0;
        mbar_wait_bounded(&full[it % C::STAGES], (it / C::STAGES) & 1, &dummy, nullptr, kDrainNs);
      }
      if (lissued > 0) {
        int dummy = 0;
        mbar_wait_bounded(lfull, (lissued - 1) & 1, &dummy, nullptr, kDrainNs);
      }
    }
  } else if (warp == 1 || warp == C::ISSUER1_WARP) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer g (warp 1: g = 0, the last warp: g = 1) takes the steps of dequant group g
    // (j = g, g + 2, ...) into its own accumulator, so two MMA streams per CTA are in
    // flight; issuer 0 then adds the adapter product to its accumulator.
    if (lane == 0) {
      const int g = warp == 1 ? 0 : 1;
      const uint32_t acc_t = tmem_base + g * C::ACC_COLS;
      constexpr uint32_t idesc_main = idesc_bf16(128, C::NT, false, false);
      constexpr uint32_t idesc_lora = idesc_bf16(128, C::NT, true, false);
      bool ok = true;
      // descriptors advance by constant steps: +2 per 16-element K step (32 bytes >> 4),
      // +X_BYTES >> 4 per block, +STAGE_BYTES >> 4 per ring stage
      const uint64_t desc0 = smem_desc_sw128(smem_base, 16, 1024);
      uint32_t acc = 0;  // the first MMA overwrites the accumulator
      for (int j = g; j < n_ss; j += C::NACC) {
        const int s = j % C::STAGES;
        if (!mbar_wait_bounded_sleep(&ready[s], (j / C::STAGES) & 1, abort_flag, p.dev_err, p.timeout_ns,
                                     kSmallWaitHintNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bd = desc0 + static_cast<uint64_t>((s * C::STAGE_BYTES) >> 4);
        const uint32_t a_tmem = tmem_base + C::NACC * C::ACC_COLS + (j % C::TSLOTS) * 32 * C::KB;
        const bool two = n_main - j * C::KB >= 2;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16_ts(acc_t, a_tmem + kk * 8, bd + 2 * kk, idesc_main, acc);
          acc = 1;
        }
        if (C::KB == 2 && two) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(acc_t, a_tmem + 32 + kk * 8, bd + (C::X_BYTES >> 4) + 2 * kk, idesc_main, 1u);
        }
        mma_commit(&empty[s]);
      }
      bool first = acc == 0;
      for (int c = 0; g == 0 && ok && c < n_lora; ++c) {
        if (!mbar_wait_bounded(lfull, c & 1, abort_flag, p.dev_err, p.timeout_ns)) break;
        tc_fence_after();
        const int rem = p.lora_r - c * 64;
        const int ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
        const uint32_t a_base = smem_base + C::OFF_LA;
        const uint32_t b_base = smem_base + C::OFF_LX;
        for (int kk = 0; kk < ksteps; ++kk) {
          mma_bf16_ss(acc_t, smem_desc_sw128(a_base + kk * 2048, 8192, 1024),
                      smem_desc_sw128(b_base + kk * 32, 16, 1024), idesc_lora, first ? 0u : 1u);
          first = false;
        }
        mma_commit(lempty);
      }
      mma_commit(acc_full);  // tracks completion of everything this issuer issued
    }
  } else {
    // ------------------------------------------------------------ dequant groups (warps 2..9)
    const int t = threadIdx.x - 64;  // 0 .. DQ_THREADS-1
    const int g = t >> 7;
    const int q = warp & 3;         // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;  // W row within the tile = TMEM lane
    const int qs = p.q8_stride;
    // stage the block constants [128 rows x n_main] and the group scales they use
    const int64_t gfirst = (static_cast<int64_t>(n0) * kbt + kb_begin) >> 8;
    {
      const int nm = n_main > 0 ? n_main : 1;
      // group scales first (independent of the constants below, so both loads are in flight together)
      const int rlast = (n0 + 127 < p.N ? n0 + 127 : p.N - 1);
      const int64_t glast = (static_cast<int64_t>(rlast) * kbt + kb_begin + nm - 1) >> 8;
      float c1v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int64_t gi = gfirst + t + C::DQ_THREADS * u;
        c1v[u] = (gi <= glast && gi - gfirst < kSmallC1Max) ? __ldg(p.c1 + gi) : 0.f;
      }
      if (p.q8_words) {
        // 4-byte words (rows of kbt bytes, splits of k_iters bytes, both multiples of 4);
        // 8 independent loads per batch so their latencies overlap
        const int wpr = (nm + 3) >> 2;  // words per row
        for (int base = t; base < 128 * wpr; base += C::DQ_THREADS * 8) {
          uint32_t e[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + C::DQ_THREADS * u;
            const int r = i / wpr, k = (i - r * wpr) * 4;
            e[u] = 0;
            if (i < 128 * wpr && n0 + r < p.N && k < n_main)
              e[u] = __ldg(reinterpret_cast<const uint32_t *>(p.c2q + static_cast<int64_t>(n0 + r) * kbt + kb_begin + k));
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + C::DQ_THREADS * u;
            const int r = i / wpr, k = (i - r * wpr) * 4;
            if (i < 128 * wpr) *reinterpret_cast<uint32_t *>(q8s + r * qs + k) = e[u];
          }
        }
      } else {
        for (int base = t; base < 128 * nm; base += C::DQ_THREADS * 8) {
          uint8_t e[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + C::DQ_THREADS * u;
            const int r = i / nm, k = i - r * nm;
            e[u] = 0;
            if (i < 128 * nm && n0 + r < p.N && k < n_main)
              e[u] = __ldg(p.c2q + static_cast<int64_t>(n0 + r) * kbt + kb_begin + k);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + C::DQ_THREADS * u;
            const int r = i / nm, k = i - r * nm;
            if (i < 128 * nm) q8s[r * qs + k] = e[u];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (t + C::DQ_THREADS * u < kSmallC1Max) c1s[t + C::DQ_THREADS * u] = c1v[u];
    }
    named_barrier(1, 128 * C::GROUPS);
    const float mu = *p.mean;
    // codes tile, C_ROW-byte rows with the C_ROW-byte TMA swizzle: 16-byte chunk c of row i
    // sits at chunk c ^ ((i >> 1) & 3) (64-byte rows) or c ^ ((i >> 2) & 1) (32-byte rows), so
    // the 8 lanes of one shared-memory phase (rows i..i+7) cover all 32 banks
    const uint32_t sw = C::KB == 2 ? (row >> 1) & 3 : (row >> 2) & 1;
    const uint32_t c_row = smem_base + C::KB * C::X_BYTES + row * C::C_ROW;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::NACC * C::ACC_COLS;
    // block index of (row, block i) relative to the first staged group scale
    const int rb = static_cast<int>(static_cast<int64_t>(n0 + row) * kbt + kb_begin - (gfirst << 8));
    const uint8_t *q8row = q8s + row * qs;
    for (int j = g; j < n_ss; j += C::GROUPS) {
      const int s = j % C::STAGES;
      const uint32_t ph = (j / C::STAGES) & 1;
      const uint32_t slot = t_row + (j % C::TSLOTS) * 32 * C::KB;
      const int nb = n_main - j * C::KB < C::KB ? n_main - j * C::KB : C::KB;
      const bool okf = mbar_wait_bounded_sleep(&full[s], ph, abort_flag, p.dev_err, p.timeout_ns, kSmallWaitHintNs);
      if (!__all_sync(0xFFFFFFFFu, okf)) break;
      if (j >= C::TSLOTS) {
        // the MMAs that last read this TMEM slot (step j - TSLOTS) are complete
        const int jp = j - C::TSLOTS;
        const bool oke =
            mbar_wait_bounded_sleep(&empty[jp % C::STAGES], (jp / C::STAGES) & 1, abort_flag, p.dev_err, p.timeout_ns,
                                    kSmallWaitHintNs);
        if (!__all_sync(0xFFFFFFFFu, oke)) break;
      }
      tc_fence_after();
      const uint32_t cs = c_row + s * C::STAGE_BYTES;
      for (int b = 0; b < nb; ++b) {
        const int i = j * C::KB + b;
        const float c2h = reconstruct_c2(q8row[i], c1s[(rb + i) >> 8], mu);
        const BlockLut lut = make_lut(c2h, p.lv);
        uint32_t w[8];
        ld_shared_v4(cs + (((2 * b) ^ sw) << 4), w[0], w[1], w[2], w[3]);
        ld_shared_v4(cs + (((2 * b + 1) ^ sw) << 4), w[4], w[5], w[6], w[7]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[4];
            decode8(w[4 * h + c], lut, o, p.k_shr16, p.k_shr1);
            v[4 * c + 0] = o[0];
            v[4 * c + 1] = o[1];
            v[4 * c + 2] = o[2];
            v[4 * c + 3] = o[3];
          }
          tmem_st16(slot + b * 32 + h * 16, v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);
    }
    // ------------------------------------------------------------ park the float32 partial (group 0)
    if (g == 0) {
      const bool got = mbar_wait_bounded(acc_full, 0, abort_flag, p.dev_err, p.timeout_ns);
      if (__all_sync(0xFFFFFFFFu, got) && !*abort_flag) {
        tc_fence_after();
        float *P = reinterpret_cast<float *>(smem);
        // accumulator 0 holds steps 0, 2, ... and the adapter product; accumulator 1 steps 1, 3, ...
        const bool w0 = n_ss >= 1 || n_lora > 0, w1 = n_ss >= 2;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int c0 = 0; c0 < C::NT; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < C::NT) P[(c0 + j) * C::PSTRIDE + row] = w0 ? __uint_as_float(v[j]) : 0.f;
          if (w1) {
            tmem_ld32(lane_base + C::ACC_COLS + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < C::NT) P[(c0 + j) * C::PSTRIDE + row] += __uint_as_float(v[j]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ in-cluster split reduction
  tc_fence_before();
  cluster_sync();  // every CTA's partial is parked
  pdl_wait();
  pdl_launch_dependents();
  {
    const int S = p.splits;
    const int j = static_cast<int>(cluster_ctarank());
    const int c_lo = (j * 32 / S) * 4;  // this rank's columns [c_lo, c_hi) of the tile
    const int c_hi = ((j + 1) * 32 / S) * 4;
    const int nc4 = (c_hi - c_lo) >> 2;
    for (int v = threadIdx.x; v < p.M * nc4; v += C::NUM_THREADS) {
      const int tok = v / nc4;
      const int c = c_lo + 4 * (v - tok * nc4);
      const int n = n0 + c;
      const uint32_t off = smem_base + static_cast<uint32_t>(tok * C::PSTRIDE + c) * 4;
      float4 part[8];
#pragma unroll
      for (int qr = 0; qr < 8; ++qr)
        if (qr < S) part[qr] = ld_shared_cluster_v4(mapa_shared(off, static_cast<uint32_t>(qr)));
      float4 acc = part[0];
#pragma unroll
      for (int qr = 1; qr < 8; ++qr)
        if (qr < S) {
          acc.x += part[qr].x;
          acc.y += part[qr].y;
          acc.z += part[qr].z;
          acc.w += part[qr].w;
        }
      if (n < p.N) {
        uint2 pk;
        pk.x = pack_bf16x2(acc.x, acc.y);
        pk.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2 *>(p.Y + static_cast<int64_t>(tok) * p.N + n) = pk;
      }
    }
  }
  cluster_sync();  // no CTA leaves while a peer may still read its partial

  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && *abort_flag) {
      int dummy = 0;
      mbar_wait_bounded(acc_full, 0, &dummy, nullptr, kDrainNs);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
