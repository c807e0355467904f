// gemm_pair.cuh — the fused dequant GEMM on a CTA pair (cluster of 2, tcgen05
// cta_group::2): one (256·MSUB) x 256 output tile per pair.
//
//   D[256·MSUB tokens x 256] = sum_k Aop · W_hat-sideᵀ  (+ LoRA tail)
//
// Each CTA of the pair stages its own 128·MSUB token rows of the activation
// (TMA) and dequantises its own 128 rows of the W-side operand; the leader CTA
// issues the pair MMA, which reads both CTAs' shared memory at the same offsets
// and writes each CTA's 128 x 256 accumulator slice into that CTA's TMEM.  With
// MSUB = 2 every dequantised W tile feeds two such MMAs (two accumulators, all
// 512 TMEM columns).  Against a one-CTA 128 x 256 tile this cuts the
// dequantisation work per flop by 2·MSUB and the W-side operand bytes each SM
// stages by 2.
//
// Three rings per CTA, so that the two latencies of a stage — the activation
// TMA and the dequantisation — run side by side instead of one after the other:
//   codes ring (CSTAGES slots, 4 KiB)  packed codes of the CTA's 128 W rows for
//                                      one 64-deep K step; filled ahead by the
//                                      code producer, freed by the dequant group
//                                      right after it has read them;
//   A slots  (STAGES, 16 KiB·MSUB)     activation tiles, TMA;
//   B slots  (STAGES, 16 KiB)          the dequantised W-side tiles.
// A and B slot s are freed together by the pair MMA's multicast commit.
//
// Roles per CTA (608 threads):
//   warp 0      A producer: activation tiles (or the LoRA tiles) into A/B slots.
//   warp 1      TMEM allocation (pair); in the leader, the MMA issuer: waits
//               ready[s] (8 warp arrivals: 4 per CTA), issues the pair MMAs,
//               commits empty[s] to both CTAs (multicast).
//   warps 2..17 four dequant groups of 4 warps; group g owns every 4th K step:
//               codes in (cfull), codes slot released (cempty), B slot free
//               (empty), expand 128 rows x 64 codes to bf16 in the swizzled
//               UMMA layout, fence to the async proxy, wait for the A tile of
//               the same step (afull), arrive on the leader's ready[s].  The
//               block constants of a group's next step are fetched one step
//               ahead.  All 16 then run the epilogue.
//   warp 18     code producer (one lane).
// Shared-memory bank use: K-major code rows are read in an order that gives
// the 8 threads of each 128-bit phase distinct banks; MN-major code tiles are
// staged with the TMA 64-byte swizzle for the same reason.
#pragma once
#include <cstdint>
#include <cuda.h>
#include "gemm.cuh"

namespace qlora {

template <int STAGES_, int BMODE_, int LORA_, int OUT_, int MSUB_>
struct PairCfg {
  static constexpr int STAGES = STAGES_;       // A/B slots
  static constexpr int CSTAGES = 2 * STAGES_;  // code slots
  static constexpr int MSUB = MSUB_;  // 128-token sub-tiles per CTA sharing one dequantised W tile
  static constexpr int BMODE = BMODE_;
  static constexpr int LORA = LORA_;
  static constexpr int OUT = OUT_;
  static constexpr int BN = 256;  // pair N
  static constexpr bool B_MN = BMODE == B_DQ_MN;
  static constexpr int A_BYTES = MSUB * 128 * 64 * 2;
  static constexpr int B_BYTES = 128 * 64 * 2;
  static constexpr int C_BYTES = 4096;
  static constexpr int DQ_GROUPS = 4;  // groups of 4 warps, one per A/B slot
  static constexpr int CODE_WARP = 2 + 4 * DQ_GROUPS;
  static constexpr int NUM_THREADS = 32 * (CODE_WARP + 1);
  static constexpr int TMEM_COLS = 256 * MSUB;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_C + CSTAGES * C_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static_assert(BMODE == B_DQ_K || BMODE == B_DQ_MN, "pair kernel dequantises its W-side operand");
  static_assert(STAGES == DQ_GROUPS, "each dequant group owns one A/B slot");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0 && C_BYTES % 1024 == 0, "1 KiB swizzle atoms");
  static_assert((3 * STAGES + 2 * CSTAGES + 1) * 8 + 8 <= 256, "barrier area");
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::NUM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_codes,
                     const __grid_constant__ CUtensorMap map_a2, const __grid_constant__ CUtensorMap map_b2,
                     const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *afull = bars;                    // A (and LoRA B) tile landed, local
  uint64_t *empty = afull + C::STAGES;       // pair MMAs done with A/B slot (multicast commit)
  uint64_t *ready = empty + C::STAGES;       // leader: both CTAs' slot s staged (8 warp arrivals)
  uint64_t *cfull = ready + C::STAGES;       // code slot landed, local
  uint64_t *cempty = cfull + C::CSTAGES;     // code slot read by its dequant group (4 warps)
  uint64_t *acc_full = cempty + C::CSTAGES;  // all pair MMAs of the tile done (multicast commit)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // the pair's tile (tm: token-pair tile, tn: W-side tile); both CTAs of a pair
  // compute the same indices from the pair's position in the launch order
  int tm = static_cast<int>(blockIdx.x >> 1), tn = static_cast<int>(blockIdx.y);
  if (p.raster_gm > 0) {
    const int tmp = static_cast<int>(gridDim.x >> 1), tnn = static_cast<int>(gridDim.y);
    const int pidx = tn * tmp + tm;                      // launch order: x fastest
    const int group = pidx / (p.raster_gm * tnn);
    const int within = pidx - group * p.raster_gm * tnn;
    const int rows = tmp - group * p.raster_gm < p.raster_gm ? tmp - group * p.raster_gm : p.raster_gm;
    tm = group * p.raster_gm + within % rows;
    tn = within / rows;
  }
  const int m0 = (2 * tm + static_cast<int>(rank)) * 128 * C::MSUB;  // this CTA's token rows
  const int n0 = tn * C::BN;                                          // the pair's W-side tile
  const int nh0 = n0 + 128 * static_cast<int>(rank);  // this CTA's half of it
  const int split = blockIdx.z;
  const int kb_begin = split * p.k_iters;
  int n_main = p.k_iters_total - kb_begin;
  if (n_main > p.k_iters) n_main = p.k_iters;
  const int n_lora = (C::LORA != LORA_NONE && split == 0) ? (p.lora_r + 63) / 64 : 0;
  const int n_total = n_main + n_lora;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 8);
    }
    for (int s = 0; s < C::CSTAGES; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 4);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_codes);
    if (C::LORA != LORA_NONE) {
      tma_prefetch_desc(&map_a2);
      tma_prefetch_desc(&map_b2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  pdl_wait();  // inputs of this grid were written by earlier grids of the stream
  // No early trigger either: the grid after this one starts when it has finished
  // (see gemm.cuh on run-to-run differences seen with early triggers around this kernel).

  if (warp == 0) {
    // ------------------------------------------------------------ A producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_total; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait_cluster_bounded(&empty[s], ph ^ 1, abort_flag, p.dev_err, p.timeout_ns)) break;
        uint8_t *sa = smem + s * C::A_BYTES;
        uint8_t *sb = smem + C::OFF_B + s * C::B_BYTES;
        if (it < n_main) {
          const int k0 = (kb_begin + it) * 64;
          mbar_arrive_expect_tx(&afull[s], C::A_BYTES);
#pragma unroll
          for (int i = 0; i < C::MSUB; ++i) tma_load_2d(sa + i * 16384, &map_a, &afull[s], k0, m0 + 128 * i);
        } else {
          const int r0 = (it - n_main) * 64;
          mbar_arrive_expect_tx(&afull[s], C::A_BYTES + C::B_BYTES);
#pragma unroll
          for (int i = 0; i < C::MSUB; ++i) tma_load_2d(sa + i * 16384, &map_a2, &afull[s], r0, m0 + 128 * i);
          if (C::LORA == LORA_B2_MN) {
            tma_load_2d(sb, &map_b2, &afull[s], nh0, r0);
            tma_load_2d(sb + 8192, &map_b2, &afull[s], nh0 + 64, r0);
          } else {
            tma_load_2d(sb, &map_b2, &afull[s], r0, nh0);
          }
        }
        issued = it + 1;
      }
      for (int it = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; it < issued; ++it) {
        int dummy = 0;
        mbar_wait_bounded(&afull[it % C::STAGES], (it / C::STAGES) & 1, &dummy, nullptr, kDrainNs);
      }
    }
  } else if (warp == C::CODE_WARP) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_main; ++it) {
        const int cs = it % C::CSTAGES;
        const uint32_t ph = (it / C::CSTAGES) & 1;
        if (!mbar_wait_bounded(&cempty[cs], ph ^ 1, abort_flag, p.dev_err, p.timeout_ns)) break;
        uint8_t *sc = smem + C::OFF_C + cs * C::C_BYTES;
        const int k0 = (kb_begin + it) * 64;
        mbar_arrive_expect_tx(&cfull[cs], C::C_BYTES);
        if (C::BMODE == B_DQ_K)
          tma_load_2d(sc, &map_codes, &cfull[cs], k0 / 2, nh0);  // [128 W rows x 32 B]
        else
          tma_load_2d(sc, &map_codes, &cfull[cs], nh0 / 2, k0);  // [64 W rows x 64 B], 64-B swizzle
        issued = it + 1;
      }
      for (int it = issued - C::CSTAGES < 0 ? 0 : issued - C::CSTAGES; it < issued; ++it) {
        int dummy = 0;
        mbar_wait_bounded(&cfull[it % C::CSTAGES], (it / C::CSTAGES) & 1, &dummy, nullptr, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc_main = idesc_bf16(256, 256, false, C::B_MN);
      constexpr uint32_t idesc_lora = idesc_bf16(256, 256, false, C::LORA == LORA_B2_MN);
      for (int it = 0; it < n_total; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        const bool main = it < n_main;
        if (!mbar_wait_cluster_bounded(&ready[s], ph, abort_flag, p.dev_err, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t a_base = smem_base + s * C::A_BYTES;
        const uint32_t b_base = smem_base + C::OFF_B + s * C::B_BYTES;
        int ksteps = 4;
        if (!main) {
          const int rem = p.lora_r - (it - n_main) * 64;
          ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
        }
        const bool b_mn = main ? C::B_MN : (C::LORA == LORA_B2_MN);
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint64_t bd = b_mn ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b_base + kk * 32, 16, 1024);
#pragma unroll
          for (int i = 0; i < C::MSUB; ++i) {
            const uint64_t ad = smem_desc_sw128(a_base + i * 16384 + kk * 32, 16, 1024);
            mma_bf16_ss_pair(tmem_acc + 256 * i, ad, bd, main ? idesc_main : idesc_lora,
                             (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit_pair_mc(&empty[s], 3);
      }
      mma_commit_pair_mc(acc_full, 3);
    }
  } else {
    // ------------------------------------------------------------ dequant groups (warps 2..17)
    const int g = (warp - 2) >> 2;                    // dequant group = A/B slot
    const int t = ((warp - 2) & 3) * 32 + lane;       // 0..127
    const float mu = *p.mean;
    const uint32_t ready_leader = mapa_shared(smem_u32(&ready[0]), 0);
    // block constant of this thread's (row, block) at step `it` (raw E4M3 byte + group scale)
    auto fetch = [&](int it, uint32_t &e, float &sg) {
      e = 0;
      sg = 0.f;
      if (it >= n_main) return;
      const int kb = kb_begin + it;
      int wrow, wblk;
      if (C::BMODE == B_DQ_K) {
        wrow = nh0 + t;
        wblk = kb;
      } else {
        wrow = kb * 64 + (t & 63);
        wblk = nh0 / 64 + (t >> 6);
      }
      if (wrow < p.w_rows && wblk < p.w_kblocks) {
        const int64_t b = static_cast<int64_t>(wrow) * p.w_kblocks + wblk;
        e = __ldg(p.c2q + b);
        sg = __ldg(p.c1 + (b >> 8));
      }
    };
    uint32_t e_cur;
    float s_cur;
    fetch(g, e_cur, s_cur);
    for (int it = g; it < n_total; it += C::DQ_GROUPS) {
      const int s = it % C::STAGES;
      const uint32_t ph = (it / C::STAGES) & 1;
      const bool main = it < n_main;
      uint32_t e_nxt;
      float s_nxt;
      fetch(it + C::DQ_GROUPS, e_nxt, s_nxt);
      const float c2h = main ? reconstruct_c2(e_cur, s_cur, mu) : 0.f;
      e_cur = e_nxt;
      s_cur = s_nxt;
      if (main) {
        // codes of this step: read them into registers and release the code slot at once
        const int cs = it % C::CSTAGES;
        const uint32_t cph = (it / C::CSTAGES) & 1;
        bool ok = mbar_wait_bounded(&cfull[cs], cph, abort_flag, p.dev_err, p.timeout_ns);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        const uint32_t cbase = smem_base + C::OFF_C + cs * C::C_BYTES;
        uint32_t w[8];
        uint32_t obase;
        int swz;
        if (C::BMODE == B_DQ_K) {
          // row t: 32 bytes; threads 4..7 of each 8-thread phase read the upper half first
          const uint32_t first = ((t >> 2) & 1) << 4;
          uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
          ld_shared_v4(cbase + t * 32 + first, a0, a1, a2, a3);
          ld_shared_v4(cbase + t * 32 + (16 - first), b0, b1, b2, b3);
          const bool sw = first != 0;
          w[0] = sw ? b0 : a0; w[1] = sw ? b1 : a1; w[2] = sw ? b2 : a2; w[3] = sw ? b3 : a3;
          w[4] = sw ? a0 : b0; w[5] = sw ? a1 : b1; w[6] = sw ? a2 : b2; w[7] = sw ? a3 : b3;
          obase = smem_base + C::OFF_B + s * C::B_BYTES + t * 128;
          swz = t & 7;
        } else {
          const int r = t & 63, j = t >> 6;
          const uint32_t x = (r >> 1) & 3;  // 64-byte TMA swizzle of the code tile
          ld_shared_v4(cbase + r * 64 + ((((2 * j) ^ x) & 3) << 4), w[0], w[1], w[2], w[3]);
          ld_shared_v4(cbase + r * 64 + ((((2 * j + 1) ^ x) & 3) << 4), w[4], w[5], w[6], w[7]);
          obase = smem_base + C::OFF_B + s * C::B_BYTES + j * 8192 + r * 128;
          swz = r & 7;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[cs]);
        // the B slot is free once the pair MMAs of the previous round finished with it
        ok = mbar_wait_cluster_bounded(&empty[s], ph ^ 1, abort_flag, p.dev_err, p.timeout_ns);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        const BlockLut lut = make_lut(c2h, p.lv);
        const uint32_t sbase = obase | (static_cast<uint32_t>(swz) << 4);  // obase is 128-byte aligned
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          decode8(w[c], lut, o, p.k_shr16, p.k_shr1);
          st_shared_v4(sbase ^ (static_cast<uint32_t>(c) << 4), o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
      }
      // the activation tile (or the LoRA tiles) of this step must have landed too
      const bool okA = mbar_wait_bounded(&afull[s], ph, abort_flag, p.dev_err, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, okA)) break;
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ready_leader + s * 8);
    }
    // ------------------------------------------------------------ epilogue (all dequant warps)
    // warp w reads TMEM lane quadrant (w & 3) and a 64-column slice ((w - 2) >> 2) of
    // every 256-column accumulator.
    {
      const bool got = mbar_wait_cluster_bounded(acc_full, 0, abort_flag, p.dev_err, p.timeout_ns);
      if (__all_sync(0xFFFFFFFFu, got) && !*abort_flag) {
        tc_fence_after();
        const int q = warp & 3;
        const int cg = (warp - 2) >> 2;
#pragma unroll 1
        for (int i = 0; i < C::MSUB; ++i) {
          const int row = m0 + 128 * i + q * 32 + lane;
#pragma unroll 1
          for (int c0 = cg * 64; c0 < cg * 64 + 64; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + 256 * i + c0, v);
            tmem_ld_wait();
            const int col = n0 + c0;
            if (row < p.rows && col < p.cols) {
              if (C::OUT == OUT_BF16) {
                uint16_t *o = reinterpret_cast<uint16_t *>(p.out) + static_cast<int64_t>(row) * p.ld_out + col;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                  if (col + 8 * gq + 8 <= p.cols) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(v[8 * gq + 0]), __uint_as_float(v[8 * gq + 1]));
                    pk.y = pack_bf16x2(__uint_as_float(v[8 * gq + 2]), __uint_as_float(v[8 * gq + 3]));
                    pk.z = pack_bf16x2(__uint_as_float(v[8 * gq + 4]), __uint_as_float(v[8 * gq + 5]));
                    pk.w = pack_bf16x2(__uint_as_float(v[8 * gq + 6]), __uint_as_float(v[8 * gq + 7]));
                    *reinterpret_cast<uint4 *>(o + 8 * gq) = pk;
                  }
                }
              } else {
                float *o = reinterpret_cast<float *>(p.out) + static_cast<int64_t>(split) * p.split_stride +
                           static_cast<int64_t>(row) * p.ld_out + col;
#pragma unroll
                for (int gq = 0; gq < 8; ++gq) {
                  if (col + 4 * gq + 4 <= p.cols)
                    *reinterpret_cast<float4 *>(o + 4 * gq) =
                        make_float4(__uint_as_float(v[4 * gq]), __uint_as_float(v[4 * gq + 1]),
                                    __uint_as_float(v[4 * gq + 2]), __uint_as_float(v[4 * gq + 3]));
                }
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1 && leader && lane == 0 && *abort_flag) {
    int dummy = 0;  // no pair MMA may still be running when TMEM is released
    mbar_wait_cluster_bounded(acc_full, 0, &dummy, nullptr, kDrainNs);
  }
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_acc, C::TMEM_COLS);
  }
}

}  // namespace qlora
