// gemm.cuh — warp-specialised tcgen05 GEMM for sm_100a, with an optional
// on-the-fly NF4 double-dequantised operand and an optional LoRA tail.
//
//   D[128 x BN] (TMEM, f32) = sum_k  Aop[128 x k] · Bop[BN x k]ᵀ
//                           (+ sum_r A2[128 x r] · B2[BN x r]ᵀ   LoRA tail)
//
// Roles (one CTA = one 128 x BN output tile of one K split):
//   warp 0      TMA producer: activation tiles (and the packed NF4 code tiles,
//               or the second bf16 operand) into a STAGES-deep smem ring.
//   warp 1      TMEM allocator and MMA issuer (one elected thread issues
//               tcgen05.mma, commits each stage back to the producer).
//   warps 2..9  (dequant variants only) expand code tiles to bf16 directly in
//               the 128-byte-swizzled UMMA layout, one 64-element block per
//               thread per stage; W_hat never reaches HBM.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, convert, store.
//
// Operand tiles in smem are canonical SWIZZLE_128B layouts:
//   K-major  [rows x 64]: row i at i*128 B, 16-B chunk c stored at chunk c^(i&7);
//                         8-row groups 1024 B apart (SBO); K step of 16 = +32 B.
//   MN-major [64 k-rows x 64·j]: MN blocks of 64 elements 8 KiB apart (LBO),
//                         8-k-row groups 1024 B apart (SBO); K step of 16 = +2 KiB.
// Every wait is bounded (globaltimer); on timeout the kernel raises an abort
// flag, records QLORA_DEVERR_TIMEOUT, drains what it issued and exits cleanly.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "nf4_decode.cuh"
#include "ptx.cuh"

namespace qlora {

enum BMode : int { B_TMA_K = 0, B_TMA_MN = 1, B_DQ_K = 2, B_DQ_MN = 3 };
enum LoraMode : int { LORA_NONE = 0, LORA_B2_MN = 1, LORA_B2_K = 2 };
// OUT_BF16 / OUT_F32: the tile is written as is (OUT_F32 into split partials).
// OUT_RED_*: the K splits of a tile run as one thread-block cluster (1 x 1 x S);
// each CTA parks its float32 partial in shared memory and the cluster sums the
// S partials in rank order through distributed shared memory, scales by
// p.scale and writes the final tile: bf16 [row][col], float32 [row][col], or
// float32 transposed [col][row].
enum OutMode : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_RED_BF16 = 2, OUT_RED_F32 = 3, OUT_RED_F32_T = 4 };

// Bound on the waits that drain in-flight copies and MMAs before exit (independent of
// the configurable pipeline-wait bound, so a short bound never abandons a copy in flight).
constexpr unsigned long long kDrainNs = 1000000000ull;

struct GemmParams {
  int rows;            // valid rows of the MMA-M side
  int cols;            // valid columns of the MMA-N side
  int k_iters;         // main-loop stages (64 reduction elements each) per split
  int k_iters_total;   // main-loop stages over all splits
  int lora_r;          // LoRA rank (0 = none); tail handled by split 0 only
  // NF4 weight (dequant variants): W is [w_rows, 64*w_kblocks]
  const uint8_t *c2q;
  const float *c1;
  const float *mean;
  int w_rows;
  int w_kblocks;
  Nf4Levels lv;
  // output
  void *out;
  int64_t ld_out;        // elements
  int64_t split_stride;  // elements between split partials (OUT_F32)
  int *dev_err;
  unsigned long long timeout_ns;
  uint32_t k_shr16;  // 2^16 (a right shift by 16 done as a high-half multiply)
  uint32_t k_shr1;   // 2^31 (a right shift by 1 likewise)
  // OUT_RED_* only
  int cluster;       // K splits = CTAs per cluster along z (1, 2, 4 or 8)
  int red_cols;      // valid output columns (<= BN)
  float scale;       // applied to the reduced sum
  // CTA-pair kernel only: tile order.  0 = the launch grid's order (token tiles
  // fastest); g > 0 = groups of g token-pair tiles, all W-side tiles of a group
  // before the next group, so that the activation tiles the resident CTAs share
  // stay in L2 while the W tiles stream past them.
  int raster_gm;
  // gemm_kernel only: 1 = let the next grid start early (programmatic launch);
  // set only where the small-M forward follows.
  int trigger_dependents;
};

template <int BN_, int STAGES_, bool A_MN_, int BMODE_, int LORA_, int OUT_>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr bool A_MN = A_MN_;
  static constexpr int BMODE = BMODE_;
  static constexpr int LORA = LORA_;
  static constexpr int OUT = OUT_;
  static constexpr bool DQ = BMODE == B_DQ_K || BMODE == B_DQ_MN;
  static constexpr bool B_MN = BMODE == B_TMA_MN || BMODE == B_DQ_MN;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_ROWS = (B_MN || LORA == LORA_B2_MN) ? (BN < 64 ? 64 : BN) : BN;
  static constexpr int B_BYTES = B_ROWS * 64 * 2;
  static constexpr int C_BYTES = DQ ? 8192 : 0;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  static constexpr int NUM_DQ_WARPS = DQ ? 8 : 0;
  static constexpr int NUM_THREADS = 64 + (DQ ? 256 : 128);
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr bool RED = OUT >= OUT_RED_BF16;
  static constexpr int PSTRIDE = BN + 4;  // floats per row of the parked partial (conflict-free rows)
  static_assert(!RED || 128 * PSTRIDE * 4 <= STAGES * STAGE_BYTES, "partial must fit in the pipeline smem");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N");
  static_assert(!DQ || BN == 256, "dequant tiles are 256 wide");
  static_assert(STAGE_BYTES % 1024 == 0, "swizzle atoms need 1 KiB alignment");
  static_assert((3 * STAGES + 2) * 8 <= BAR_BYTES, "barriers, TMEM slot and abort flag fit");
};

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_a2, const __grid_constant__ CUtensorMap map_b2,
                const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t *full = bars;                      // TMA landed (tx bytes)
  uint64_t *empty = bars + C::STAGES;         // MMA finished reading the stage
  uint64_t *bfull = bars + 2 * C::STAGES;     // dequant warps wrote the W operand
  uint64_t *acc_full = bars + 3 * C::STAGES;  // all MMAs of the tile done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * C::STAGES + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * C::BN;
  const int split = blockIdx.z;
  const int kb_begin = split * p.k_iters;
  int n_main = p.k_iters_total - kb_begin;
  if (n_main > p.k_iters) n_main = p.k_iters;
  const int n_lora = (C::LORA != LORA_NONE && split == 0) ? (p.lora_r + 63) / 64 : 0;
  const int n_total = n_main + n_lora;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&bfull[s], C::NUM_DQ_WARPS > 0 ? C::NUM_DQ_WARPS : 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    if (C::LORA != LORA_NONE) {
      tma_prefetch_desc(&map_a2);
      tma_prefetch_desc(&map_b2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  pdl_wait();  // inputs of this grid were written by earlier grids of the stream
  // Early trigger only where the small-M forward follows.  Elsewhere the next grid
  // (above all the CTA-pair GEMM after s·X·A or s·dY·Bᵀ) becomes resident only when
  // this one has finished: with the trigger, the CTA-pair GEMM produced run-to-run
  // different outputs (one output column of a 512-token tile, in a few launches per
  // hundred) although every one of its CTAs waits for this grid before touching
  // memory; without it, and with programmatic launch switched off altogether,
  // thousands of repeated calls of the LLaMA-7B layer's linears were
  // bit-identical.  The small-M kernel after an
  // early trigger was bit-identical in the same test and gains the overlap (its
  // forward is 27 instead of 36 µs for 8192 x 8192 at 16 tokens).
  if (p.trigger_dependents) pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_total; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, p.dev_err, p.timeout_ns)) break;
        uint8_t *sa = smem + s * C::STAGE_BYTES;
        uint8_t *sb = sa + C::A_BYTES;
        uint8_t *sc = sb + C::B_BYTES;
        if (it < n_main) {
          const int k0 = (kb_begin + it) * 64;
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + (C::DQ ? C::C_BYTES : C::B_BYTES));
          if (C::A_MN) {
            tma_load_2d(sa, &map_a, &full[s], m0, k0);
            tma_load_2d(sa + 8192, &map_a, &full[s], m0 + 64, k0);
          } else {
            tma_load_2d(sa, &map_a, &full[s], k0, m0);
          }
          if (C::BMODE == B_DQ_K) {
            tma_load_2d(sc, &map_b, &full[s], k0 / 2, n0);  // codes [256 rows x 32 B]
          } else if (C::BMODE == B_DQ_MN) {
            tma_load_2d(sc, &map_b, &full[s], n0 / 2, k0);  // codes [64 rows x 128 B]
          } else if (C::B_MN) {
#pragma unroll
            for (int j = 0; j < C::B_ROWS / 64; ++j) tma_load_2d(sb + j * 8192, &map_b, &full[s], n0 + 64 * j, k0);
          } else {
            tma_load_2d(sb, &map_b, &full[s], k0, n0);
          }
        } else {
          const int r0 = (it - n_main) * 64;
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
          tma_load_2d(sa, &map_a2, &full[s], r0, m0);
          if (C::LORA == LORA_B2_MN) {
#pragma unroll
            for (int j = 0; j < C::B_ROWS / 64; ++j) tma_load_2d(sb + j * 8192, &map_b2, &full[s], n0 + 64 * j, r0);
          } else {
            tma_load_2d(sb, &map_b2, &full[s], r0, n0);
          }
        }
        issued = it + 1;
      }
      // drain: every issued load must land before the CTA may exit
      for (int it = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; it < issued; ++it) {
        int dummy = 0;
        mbar_wait_bounded(&full[it % C::STAGES], (it / C::STAGES) & 1, &dummy, nullptr, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = idesc_bf16(128, C::BN, C::A_MN, C::B_MN);
      constexpr uint32_t idesc_lora = idesc_bf16(128, C::BN, false, C::LORA == LORA_B2_MN);
      for (int it = 0; it < n_total; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        const bool main = it < n_main;
        if (!mbar_wait_bounded(&full[s], ph, abort_flag, p.dev_err, p.timeout_ns)) break;
        if (C::DQ && main)
          if (!mbar_wait_bounded(&bfull[s], ph, abort_flag, p.dev_err, p.timeout_ns)) break;
        tc_fence_after();
        const uint32_t a_base = smem_base + s * C::STAGE_BYTES;
        const uint32_t b_base = a_base + C::A_BYTES;
        int ksteps = 4;
        if (!main) {
          const int rem = p.lora_r - (it - n_main) * 64;
          ksteps = rem >= 64 ? 4 : (rem + 15) / 16;
        }
        const bool a_mn = main && C::A_MN;
        const bool b_mn = main ? C::B_MN : (C::LORA == LORA_B2_MN);
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint64_t ad = a_mn ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bd = b_mn ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b_base + kk * 32, 16, 1024);
          mma_bf16_ss(tmem_acc, ad, bd, main ? idesc_main : idesc_lora, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);  // also tracks completion of everything issued above
    }
  } else {
    // ------------------------------------------------------------ dequant producers
    if (C::DQ) {
      const int t = threadIdx.x - 64;  // 0..255
      const float mu = *p.mean;
      for (int it = 0; it < n_main; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        const int kb = kb_begin + it;  // 64-element reduction chunk of this stage
        int wrow, wblk, crow_off, out_off;
        if (C::BMODE == B_DQ_K) {
          wrow = n0 + t;  // W row = MMA-N row; reduction along W's K
          wblk = kb;
          crow_off = t * 32;
          out_off = t * 128;
        } else {
          const int r = t >> 2, j = t & 3;  // W row kb*64+r (reduction), k-block of the 256-wide MMA-N tile
          wrow = kb * 64 + r;
          wblk = n0 / 64 + j;
          crow_off = r * 128 + j * 32;
          out_off = j * 8192 + r * 128;
        }
        const int swz = C::BMODE == B_DQ_K ? (t & 7) : ((t >> 2) & 7);
        float c2h = 0.f;
        if (wrow < p.w_rows && wblk < p.w_kblocks) {
          const int64_t b = static_cast<int64_t>(wrow) * p.w_kblocks + wblk;
          c2h = reconstruct_c2(__ldg(p.c2q + b), __ldg(p.c1 + (b >> 8)), mu);
        }
        const bool ok = mbar_wait_bounded(&full[s], ph, abort_flag, p.dev_err, p.timeout_ns);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        const uint32_t cbase = smem_base + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES + crow_off;
        uint32_t w[8];
        ld_shared_v4(cbase, w[0], w[1], w[2], w[3]);
        ld_shared_v4(cbase + 16, w[4], w[5], w[6], w[7]);
        const BlockLut lut = make_lut(c2h, p.lv);
        const uint32_t obase = smem_base + s * C::STAGE_BYTES + C::A_BYTES + out_off;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          decode8(w[c], lut, o);
          st_shared_v4(obase + ((c ^ swz) << 4), o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull[s]);
      }
    }
    // ------------------------------------------------------------ epilogue (warps 2..5)
    if (C::RED && warp < 6) {
      // park this CTA's float32 partial (row = TMEM lane) in shared memory
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(acc_full, 0, abort_flag, p.dev_err, p.timeout_ns);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (ok && !*abort_flag) {
        __syncwarp();
        tc_fence_after();
        const int q = warp & 3;
        const int row = q * 32 + lane;
        float *prow = reinterpret_cast<float *>(smem) + row * C::PSTRIDE;
        for (int c0 = 0; c0 < C::BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
          tmem_ld_wait();
          const int ncol = C::BN - c0 < 32 ? C::BN - c0 : 32;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            if (4 * g < ncol) {
              float4 f = n_total > 0 ? make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                                   __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
              *reinterpret_cast<float4 *>(prow + c0 + 4 * g) = f;
            }
          }
        }
      }
    }
    if (!C::RED && warp < 6) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(acc_full, 0, abort_flag, p.dev_err, p.timeout_ns);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (ok && !*abort_flag) {
        __syncwarp();
        tc_fence_after();
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = m0 + q * 32 + lane;
        for (int c0 = 0; c0 < C::BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
          tmem_ld_wait();
          const int col = n0 + c0;
          if (row < p.rows && col < p.cols) {
            if (C::OUT == OUT_BF16) {
              uint16_t *o = reinterpret_cast<uint16_t *>(p.out) + static_cast<int64_t>(row) * p.ld_out + col;
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                if (col + 8 * g + 8 <= p.cols) {
                  uint4 pk;
                  pk.x = pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1]));
                  pk.y = pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3]));
                  pk.z = pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5]));
                  pk.w = pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7]));
                  *reinterpret_cast<uint4 *>(o + 8 * g) = pk;
                }
              }
            } else {
              float *o = reinterpret_cast<float *>(p.out) + static_cast<int64_t>(split) * p.split_stride +
                         static_cast<int64_t>(row) * p.ld_out + col;
#pragma unroll
              for (int g = 0; g < 8; ++g) {
                if (col + 4 * g + 4 <= p.cols)
                  *reinterpret_cast<float4 *>(o + 4 * g) =
                      make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                  __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
              }
            }
          }
        }
      }
    }
  }

  if (C::RED) {
    // ------------------------------------------------------------ in-cluster split reduction
    cluster_sync();  // every CTA's partial is parked
    const int S = p.cluster;
    const int j = static_cast<int>(cluster_ctarank());
    const int R = 128 / S;  // rows this CTA finishes
    const uint32_t pbase = smem_base + static_cast<uint32_t>(j * R) * C::PSTRIDE * 4;
    const int ncol4 = (p.red_cols + 3) / 4;  // red_cols is a multiple of 8
    const int nval = R * ncol4;
    for (int v = threadIdx.x; v < nval; v += C::NUM_THREADS) {
      int row, c4;
      if (C::OUT == OUT_RED_F32_T) {  // consecutive threads -> consecutive rows (coalesced transposed writes)
        row = v % R;
        c4 = v / R;
      } else {  // consecutive threads -> consecutive columns
        row = v / ncol4;
        c4 = v % ncol4;
      }
      const uint32_t off = pbase + static_cast<uint32_t>(row * C::PSTRIDE + 4 * c4) * 4;
      float4 part[8];
#pragma unroll
      for (int qr = 0; qr < 8; ++qr)
        if (qr < S) part[qr] = ld_shared_cluster_v4(mapa_shared(off, static_cast<uint32_t>(qr)));
      float4 acc = part[0];
#pragma unroll
      for (int qr = 1; qr < 8; ++qr) {
        if (qr < S) {
          acc.x += part[qr].x;
          acc.y += part[qr].y;
          acc.z += part[qr].z;
          acc.w += part[qr].w;
        }
      }
      acc.x *= p.scale;
      acc.y *= p.scale;
      acc.z *= p.scale;
      acc.w *= p.scale;
      const int grow = m0 + j * R + row;
      const int col = 4 * c4;
      if (grow < p.rows) {
        if (C::OUT == OUT_RED_BF16) {
          uint2 pk;
          pk.x = pack_bf16x2(acc.x, acc.y);
          pk.y = pack_bf16x2(acc.z, acc.w);
          *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.out) + static_cast<int64_t>(grow) * p.ld_out + col) = pk;
        } else if (C::OUT == OUT_RED_F32) {
          *reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + static_cast<int64_t>(grow) * p.ld_out + col) = acc;
        } else {
          float *o = reinterpret_cast<float *>(p.out);
          o[static_cast<int64_t>(col + 0) * p.ld_out + grow] = acc.x;
          o[static_cast<int64_t>(col + 1) * p.ld_out + grow] = acc.y;
          o[static_cast<int64_t>(col + 2) * p.ld_out + grow] = acc.z;
          o[static_cast<int64_t>(col + 3) * p.ld_out + grow] = acc.w;
        }
      }
    }
    cluster_sync();  // no CTA leaves while a peer may still read its partial
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && *abort_flag) {
      // make sure no MMA is still writing TMEM before it is released
      int dummy = 0;
      mbar_wait_bounded(acc_full, 0, &dummy, nullptr, kDrainNs);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_acc, C::TMEM_COLS);
  }
}

}  // namespace qlora
