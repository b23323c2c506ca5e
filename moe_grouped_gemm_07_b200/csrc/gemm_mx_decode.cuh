// gemm_mx_decode.cuh -- block-scaled GEMM for small M (M <= 128, decode) with
// power-of-two (UE8M0) scales applied by the tensor core, sm_100a.
//
// The small-M counterpart of gemm_mx.cuh, for weights in E4M3 (UE8M0 scale
// per 128x128 block) or E2M1 (W4: UE8M0 scale per 1x32 K-strip of a row):
//   D[m][n] = C[m][n] + sum_kb sa(m, kb) * sum_{32-strips j of kb} sw(n, j) *
//             sum_{k in j} X[m][k] * W[n][k]
// arranged as gemm_decode.cuh arranges the promotion path for the
// memory-bound regime:
//
//   * swap-AB: 128 weight rows fill the MMA's M, the tokens its N (BNP);
//   * split-K over a thread-block cluster of `splits` CTAs per 128-row
//     weight tile, each CTA streaming its own K-block range, and the partial
//     tiles summed through distributed shared memory in rank order
//     (splitk_reduce_store);
//   * no promotion pass: each K-block's four block-scaled MMAs
//     (tcgen05.mma kind::mxf8f6f4.block_scale) accumulate into one TMEM
//     accumulator across the CTA's whole K range, so the 8 epilogue warps read
//     it once.
//
// Scales: each ring stage carries, beside its W and X tiles, the two 512-byte
// packed scale units the stage's K-block needs -- W's unit for its 128 rows
// (the K-block's own unit when W4, byte j = strip j; the unit of its group of
// 4 K-blocks otherwise, byte kb % 4) and X's unit for the tokens (byte
// kb % 4) -- loaded by bulk copy on the stage's barrier. The MMA warp copies
// them into one of 4 rotating TMEM scale slots (tcgen05.cp), waiting first for
// the MMAs that last read that slot.
//
// W4: the weight tile is loaded with the 4-bit TMA type, which spreads each 8
// packed bytes over a 16-byte shared-memory cell (the layout kind::mxf8f6f4
// reads 4-bit operands in): the same footprint as an E4M3 tile, half the
// bytes moved.
//
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer
// (converged warps, lane 0 issuing), warps 2..9 epilogue (TMEM lane quadrant
// w % 4, token half (w - 2) / 4). All waits are bounded; both cluster
// barriers are reached on every path.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_decode.cuh"
#include "ptx.cuh"

namespace dg {

struct MxDecodeArgs {
  int M, N, K;
  int KB;               // K / 128
  int splits;           // CTAs per cluster along K
  int rb_w;             // ceil(N / 128): 128-row units of W's packed scales
  const int32_t* sfx;   // X (tokens) packed scales [ceil(K/512)][1][32][4]
  const int32_t* sfw;   // W packed scales: W4 [K/128][rb_w][32][4], else [ceil(K/512)][rb_w][32][4]
  const void* C;        // [M][N] bf16 or null
  void* D;              // [M][N] bf16
  unsigned long long timeout_ns;
  int drop_arrive;
};

template <int BNP_, int MINB_, bool W4_>
struct MxDecodeCfg {
  static constexpr int BNP = BNP_;
  static constexpr int MINB = MINB_;
  static constexpr bool W4 = W4_;
  static constexpr int BK = 128;
  static constexpr int W_BYTES = 128 * BK;                    // shared-memory footprint
  static constexpr int W_TX = W4 ? W_BYTES / 2 : W_BYTES;     // bytes the W load delivers
  static constexpr int X_BYTES = BNP * BK;
  static constexpr int SF_BYTES = 1024;                       // W unit + X unit
  static constexpr int RING = MINB == 2 ? 100 * 1024 : 192 * 1024;
  static constexpr int STAGES_RAW = RING / (W_BYTES + X_BYTES + SF_BYTES);
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int SF_SLOTS = 4, SF_SLOT_COLS = 8;        // W cols +0..3, X cols +4..7
  static constexpr int TMEM_NEED = BNP + SF_SLOTS * SF_SLOT_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : 256;
  static constexpr int EC = BNP / 2;                          // accumulator columns per thread
  static constexpr int CH = EC < 32 ? EC : 32;                // columns per tcgen05.ld
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
  static constexpr int OFF_SF = OFF_X + STAGES * X_BYTES;
  static constexpr int OFF_BAR = OFF_SF + STAGES * SF_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + SF_SLOTS + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // split-K receive slots overlay the ring (see splitk_reduce_store)
  static constexpr int RECV_PITCH = BNP + 4;
  static constexpr int RECV_ROWS = 168;
  static_assert(RECV_ROWS * RECV_PITCH * 4 <= OFF_BAR, "receive slots fit the ring");
  static_assert(BNP == 16 || BNP == 32 || BNP == 64 || BNP == 128, "BNP");
  static_assert(OFF_X % 1024 == 0 && X_BYTES % 1024 == 0 && OFF_SF % 1024 == 0, "alignment");
  static_assert(TMEM_NEED <= TMEM_COLS && TMEM_COLS * MINB <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= (MINB == 2 ? 113 : 227) * 1024, "MINB CTAs per SM");
};

template <int BNP, int MINB, bool W4>
__global__ void __launch_bounds__(320, MINB)
    gemm_mx_decode_kernel(const __grid_constant__ CUtensorMap tm_w,   // [N][K] e4m3 / [N][K/2] e2m1
                          const __grid_constant__ CUtensorMap tm_x,   // [M][K] e4m3
                          const __grid_constant__ MxDecodeArgs args) {
  using Cfg = MxDecodeCfg<BNP, MINB, W4>;
  constexpr int S = Cfg::STAGES;
  constexpr int NSL = Cfg::SF_SLOTS;
  constexpr int EC = Cfg::EC;
  constexpr int CH = Cfg::CH;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sW = smem + Cfg::OFF_W;
  uint8_t* sX = smem + Cfg::OFF_X;
  uint8_t* sSF = smem + Cfg::OFF_SF;
  float* recv = reinterpret_cast<float*>(smem);  // receive slots, after the main loop
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* slot_done = bars + 2 * S;
  uint64_t* tfull = bars + 2 * S + NSL;
  uint64_t* mma_done = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

  const uint32_t warp = warp_id_uniform();
  const uint32_t lane = lane_id();
  const uint64_t tmo = args.timeout_ns;
  const uint32_t rank = cluster_ctarank();
  const int splits = args.splits;
  const int n_tile = blockIdx.y;
  const int n0 = n_tile * 128;
  const int kb_begin = static_cast<int>((static_cast<long long>(rank) * args.KB) / splits);
  const int kb_end = static_cast<int>((static_cast<long long>(rank + 1) * args.KB) / splits);
  const int nkb = kb_end - kb_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NSL; ++i) mbar_init(&slot_done[i], 1);
    mbar_init(tfull, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the first weight tiles go to L2 while the previous kernel finishes
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < S && j < nkb; ++j) tma_prefetch_l2(&tm_w, (kb_begin + j) * Cfg::BK, n0);
  }
  pdl_wait();  // inputs may come from the previous launch on the stream

  float acc[EC];
#pragma unroll
  for (int j = 0; j < EC; ++j) acc[j] = 0.0f;

  if (warp == 0) {
    // ======================= TMA producer (converged warp, lane 0 issues) ===
    int it = 0;
    int dropped = -1;
    for (; it < nkb; ++it) {
      const int s = it % S;
      bool ok = mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int kb = kb_begin + it;
      if (args.drop_arrive && it == 0) {
        dropped = 0;  // test hook: never arm stage 0
      } else if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], Cfg::W_TX + Cfg::X_BYTES + Cfg::SF_BYTES);
        tma_load_2d(sW + s * Cfg::W_BYTES, &tm_w, &full[s], kb * Cfg::BK, n0);
        tma_load_2d(sX + s * Cfg::X_BYTES, &tm_x, &full[s], kb * Cfg::BK, 0);
        const long long wunit = W4 ? static_cast<long long>(kb) * args.rb_w + n_tile
                                   : static_cast<long long>(kb >> 2) * args.rb_w + n_tile;
        bulk_load(sSF + s * Cfg::SF_BYTES, args.sfw + wunit * 128, 512, &full[s]);
        bulk_load(sSF + s * Cfg::SF_BYTES + 512, args.sfx + static_cast<long long>(kb >> 2) * 128,
                  512, &full[s]);
      }
      __syncwarp();
    }
    // bounded wait for every copy still in flight
    for (int j = (it > S ? it - S : 0); j < it; ++j) {
      if (j == dropped) continue;
      volatile int never = 0;
      mbar_wait(&full[j % S], (j / S) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer (converged warp, lane 0 issues) =====
    for (int it = 0; it < nkb; ++it) {
      const int s = it % S;
      const int slot = it % NSL;
      // the MMAs that last read this TMEM scale slot have finished
      bool ok = mbar_wait(&slot_done[slot], ((it / NSL) & 1) ^ 1, abort_flag, tmo,
                          SITE_MMA_TMEM_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      ok = mbar_wait(&full[s], (it / S) & 1, abort_flag, tmo, SITE_MMA_FULL);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (lane == 0) {
        const int kb = kb_begin + it;
        const uint32_t sf_src = smem_addr(sSF + s * Cfg::SF_BYTES);
        const uint32_t sf_w = tmem_base + BNP + slot * Cfg::SF_SLOT_COLS;
        tmem_cp_32x128b_x4(sf_w, smem_desc_noswz(sf_src, 128));            // W rows 0..127
        tmem_cp_32x128b_x4(sf_w + 4, smem_desc_noswz(sf_src + 512, 128));  // tokens 0..127
        const uint32_t w_base = smem_addr(sW + s * Cfg::W_BYTES);
        const uint32_t x_base = smem_addr(sX + s * Cfg::X_BYTES);
        const uint32_t q4 = static_cast<uint32_t>(kb & 3);
#pragma unroll
        for (int k = 0; k < Cfg::BK / 32; ++k) {
          const uint32_t idesc =
              W4 ? idesc_mx_f8f6f4(128, BNP, static_cast<uint32_t>(k), q4, 5u, 0u)
                 : idesc_mx_f8f6f4(128, BNP, q4, q4, 0u, 0u);
          mma_mxf8f6f4(tmem_base, smem_desc_sw128(w_base + k * 32, 16, 1024),
                       smem_desc_sw128(x_base + k * 32, 16, 1024), idesc, sf_w, sf_w + 4,
                       (it > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&slot_done[slot]);
        if (it == nkb - 1) mma_commit(tfull);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(mma_done);
    __syncwarp();
    volatile int never = 0;
    mbar_wait(mma_done, 0, &never, tmo, SITE_TEARDOWN_MMA);
    __syncwarp();
  } else if (nkb > 0) {
    // ======================= epilogue (8 warps): read the accumulator ======
    const uint32_t q = warp & 3;
    const uint32_t h = (warp - 2) >> 2;
    bool ok = mbar_wait(tfull, 0, abort_flag, tmo, SITE_EPI_TMEM_FULL);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const uint32_t t_lane = tmem_base + ((q * 32) << 16) + h * EC;
      uint32_t r[EC / CH][CH];
#pragma unroll
      for (int c = 0; c < EC / CH; ++c) tmem_ld_32x32b<CH>(t_lane + c * CH, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < EC / CH; ++c)
#pragma unroll
        for (int i = 0; i < CH; ++i) acc[c * CH + i] = __uint_as_float(r[c][i]);
    }
  }

  // ---------------------------------------------------------- split-K reduction
  tc_fence_before();
  pdl_trigger();
  splitk_reduce_store<BNP, EC, Cfg::RECV_PITCH>(acc, recv, rank, splits, warp, lane, n0, args.M,
                                                args.N, args.C, args.D);
  // no peer touches this CTA's shared memory after the second barrier

  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace dg
