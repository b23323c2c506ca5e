// gemm_mx.cuh -- dense FP8 NT GEMM with power-of-two (UE8M0) fine-grained
// scales applied by the tensor core itself (tcgen05.mma kind::mxf8f6f4
// .block_scale), sm_100a.
//
// Same operation as gemm.cuh's dense path, D = C + A @ B.T with one scale per
// 1x128 K-strip of A and per 128x128 block of B, for the case where every
// scale is a power of two (UE8M0 bytes). Then sfa * sfb * P_kb can be formed
// inside the MMA: the scale of each 32-wide K slice multiplies that slice's
// products before they are accumulated, so the accumulator stays in TMEM
// across all K-blocks of a tile and no per-K-block promotion pass is needed.
// (The pages' promotion exists because Hopper's FP8 accumulator is imprecise;
// this path measures what the B200 tensor core's own accumulation gives.)
//
// The FP4B instantiation is the FP8 x FP4 GEMM: B in E2M1 with one UE8M0
// scale per 1x32 K-strip of each row (see MxCfgT for its tile and scale
// layout); A keeps E4M3 with 1x128 power-of-two scales.
//
// Packed scale layout (written by the UE8M0 quantiser): for an operand with
// R rows (M for A, N for B) and K columns,
//   packed[q][rb][i][j]  (int32, q < ceil(K/512), rb < ceil(R/128), i < 32, j < 4)
// holds in byte b the UE8M0 scale (biased exponent, 2^(byte-127)) of row
// 128 rb + 32 j + i for K-block 4 q + b. Every (q, rb) unit is 512 contiguous
// bytes whose 16-byte row i is exactly what tcgen05.cp.32x128b.warpx4 puts in
// TMEM lane i of four consecutive columns -- the layout the MMA reads scale
// factors in (row r at lane r % 32, column r / 32, byte = scale id) -- so the
// scales go global -> shared (one bulk copy) -> TMEM with no rearranging.
//
// CTA = 320 threads, one per SM, persistent over 128 x 256 tiles:
//   warp 0      producer: A/B tiles by TMA into a 4-stage ring; per group of
//               4 K-blocks, the tile's scale units (512 B of A, 1 KB of B) by
//               bulk copy into a 4-slot ring (converged warp, lane 0 issues)
//   warp 1      TMEM owner + MMA issuer: per scale group, tcgen05.cp of the
//               scale units into one of 4 TMEM scale slots; per K-block,
//               4 x (M=128, N=256, K=32) block-scaled MMAs accumulating into
//               the tile's TMEM accumulator (columns 0..255)
//   warps 2..9  epilogue: after the tile's last K-block, read the
//               accumulator (lane quadrant w % 4, column half (w - 2) / 4),
//               release it, add C, round to BF16, store through TMA.
// All waits are bounded as in gemm.cuh.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace dg {

struct MxArgs {
  int M, N, K;
  int num_m_blocks, num_n_blocks, total_tiles;
  int rb_a, rb_b;         // 128-row units of the packed scales: ceil(M/128), ceil(N/128)
  const int32_t* sfa;     // packed A scales [ceil(K/512)][rb_a][32][4]
  const int32_t* sfb;     // packed B scales [ceil(K/512)][rb_b][32][4]
  const void* C;          // [M][N] bf16 or null
  void* D;                // [M][N] bf16
  unsigned long long timeout_ns;
  int drop_arrive;
};

// FP4B: B is E2M1 (FP8 x FP4). Its tile occupies the same shared memory as
// an E4M3 tile -- the 4-bit TMA load leaves every 8 bytes of packed codes in
// a 16-byte cell, the layout kind::mxf8f6f4 reads 4-bit operands in -- but
// only the packed bytes are transferred, and its scales come per 32-wide
// K-strip: one 512-byte unit per (K-block, 128 rows), byte b = strip b.
template <bool FP4B>
struct MxCfgT {
  static constexpr int BM = 128, BN = 256, BK = 128;
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK;
  static constexpr int B_TX = FP4B ? B_BYTES / 2 : B_BYTES;  // bytes the B load delivers
  static constexpr int SF_STAGES = FP4B ? 3 : 4;
  // per group of 4 K-blocks: A one unit; B two units (rows 0..127, 128..255),
  // per K-block when FP4B
  static constexpr int SFA_BYTES = 512, SFB_BYTES = FP4B ? 4 * 1024 : 1024;
  static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int TM_SF = 256;        // first TMEM column of the scale slots
  static constexpr int SF_SLOTS = 4;       // TMEM scale slots (one group of 4 K-blocks each)
  // columns per slot: A 0..3, B 4..11 (FP4B: K-block j of the group 4+8j..11+8j)
  static constexpr int SF_SLOT_COLS = FP4B ? 48 : 16;
  static constexpr int TMEM_COLS = 512;
  static constexpr int GROUP_M = 16;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_STAGE = ((OFF_SF + SF_STAGES * SF_BYTES + 1023) / 1024) * 1024;
  static constexpr int STAGE_BYTES_PER_WARP = 32 * 64;  // 32 rows x 32 bf16, 64B-swizzled
  static constexpr int OFF_BAR = OFF_STAGE + 8 * STAGE_BYTES_PER_WARP;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * SF_STAGES + SF_SLOTS + 3;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_B % 1024 == 0 && OFF_SF % 128 == 0 && OFF_STAGE % 1024 == 0, "alignment");
  static_assert(TM_SF + SF_SLOTS * SF_SLOT_COLS <= TMEM_COLS, "TMEM budget");
};
using MxCfg = MxCfgT<false>;

template <int BN>
__device__ __forceinline__ void mx_tile(int t, const MxArgs& a, int& m0, int& n0) {
  const int group_tiles = MxCfg::GROUP_M * a.num_n_blocks;
  const int grp = t / group_tiles;
  const int first_m = grp * MxCfg::GROUP_M;
  const int gm = min(a.num_m_blocks - first_m, MxCfg::GROUP_M);
  const int local = t - grp * group_tiles;
  m0 = (first_m + local % gm) * MxCfg::BM;
  n0 = (local / gm) * BN;
}

template <bool FP4B>
__global__ void __launch_bounds__(320, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ MxArgs args) {
  using Cfg = MxCfgT<FP4B>;
  constexpr int S = Cfg::STAGES;
  constexpr int SFS = Cfg::SF_STAGES;
  constexpr int BN = Cfg::BN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem + Cfg::OFF_A;
  uint8_t* sB = smem + Cfg::OFF_B;
  uint8_t* sSF = smem + Cfg::OFF_SF;
  uint8_t* sStage = smem + Cfg::OFF_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* sf_full = bars + 2 * S;
  uint64_t* sf_empty = bars + 2 * S + SFS;
  uint64_t* slot_done = bars + 2 * S + 2 * SFS;
  uint64_t* tfull = bars + 2 * S + 2 * SFS + Cfg::SF_SLOTS;
  uint64_t* tempty = tfull + 1;
  uint64_t* mma_done = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

  const uint32_t warp = warp_id_uniform();
  const uint32_t lane = lane_id();
  const uint64_t tmo = args.timeout_ns;
  const int nkb = args.K / Cfg::BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < SFS; ++i) {
      mbar_init(&sf_full[i], 1);
      mbar_init(&sf_empty[i], 1);
    }
    for (int i = 0; i < Cfg::SF_SLOTS; ++i) mbar_init(&slot_done[i], 1);
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_d);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // inputs may come from the previous launch on the stream

  if (warp == 0) {
    // ======================= producer (converged warp, lane 0 issues) ======
    uint32_t it = 0, git = 0;
    int dropped = -1;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x) {
      int m0, n0;
      mx_tile<BN>(t, args, m0, n0);
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        if ((kb & 3) == 0) {
          const uint32_t gs = git % SFS;
          bool ok = mbar_wait(&sf_empty[gs], ((git / SFS) & 1) ^ 1, abort_flag, tmo,
                              SITE_PRODUCER_SCALE_EMPTY);
          if (!__all_sync(0xffffffffu, ok)) goto producer_done;
          if (lane == 0) {
            const int q = kb >> 2;
            const int rba = m0 >> 7, rbb = n0 >> 7;
            const uint32_t bbytes = rbb + 1 < args.rb_b ? 1024u : 512u;  // B units of this tile
            uint8_t* dst = sSF + gs * Cfg::SF_BYTES;
            if constexpr (FP4B) {
              const int nk = min(4, nkb - kb);  // K-blocks in this group
              mbar_arrive_expect_tx(&sf_full[gs], Cfg::SFA_BYTES + nk * bbytes);
              bulk_load(dst, args.sfa + (static_cast<long long>(q) * args.rb_a + rba) * 128,
                        Cfg::SFA_BYTES, &sf_full[gs]);
              for (int j = 0; j < nk; ++j)
                bulk_load(dst + Cfg::SFA_BYTES + j * 1024,
                          args.sfb + (static_cast<long long>(kb + j) * args.rb_b + rbb) * 128,
                          bbytes, &sf_full[gs]);
            } else {
              mbar_arrive_expect_tx(&sf_full[gs], Cfg::SFA_BYTES + bbytes);
              bulk_load(dst, args.sfa + (static_cast<long long>(q) * args.rb_a + rba) * 128,
                        Cfg::SFA_BYTES, &sf_full[gs]);
              bulk_load(dst + Cfg::SFA_BYTES,
                        args.sfb + (static_cast<long long>(q) * args.rb_b + rbb) * 128, bbytes,
                        &sf_full[gs]);
            }
          }
          ++git;
        }
        const uint32_t s = it % S;
        bool ok = mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER_EMPTY);
        if (!__all_sync(0xffffffffu, ok)) goto producer_done;
        if (args.drop_arrive && it == 0) {
          dropped = 0;  // test hook: never arm stage 0
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + Cfg::B_TX);
          tma_load_2d(sA + s * Cfg::A_BYTES, &tm_a, &full[s], kb * Cfg::BK, m0);
          tma_load_2d(sB + s * Cfg::B_BYTES, &tm_b, &full[s], kb * Cfg::BK, n0);
        }
        __syncwarp();
      }
    }
  producer_done:
    __syncwarp();
    // bounded wait for every copy still in flight
    for (uint32_t j = (it > S ? it - S : 0); j < it; ++j) {
      if (static_cast<int>(j) == dropped) continue;
      volatile int never = 0;
      mbar_wait(&full[j % S], (j / S) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    for (uint32_t j = (git > SFS ? git - SFS : 0); j < git; ++j) {
      volatile int never = 0;
      mbar_wait(&sf_full[j % SFS], (j / SFS) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer (converged warp, lane 0 issues) ====
    uint32_t it = 0, git = 0, tile_it = 0;
    uint32_t slot = 0;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x, ++tile_it) {
      // the epilogue has read the previous tile's accumulator
      bool ok = mbar_wait(tempty, (tile_it & 1) ^ 1, abort_flag, tmo, SITE_MMA_TMEM_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
      tc_fence_after();
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        if ((kb & 3) == 0) {
          const uint32_t gs = git % SFS;
          slot = git % Cfg::SF_SLOTS;
          ok = mbar_wait(&sf_full[gs], (git / SFS) & 1, abort_flag, tmo, SITE_EPI_SCALE_FULL);
          if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
          // the MMAs of the group that last used this TMEM slot have finished
          ok = mbar_wait(&slot_done[slot], ((git / Cfg::SF_SLOTS) & 1) ^ 1, abort_flag, tmo,
                         SITE_MMA_TMEM_EMPTY);
          if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t src = smem_addr(sSF + gs * Cfg::SF_BYTES);
            const uint32_t dst = tmem_base + Cfg::TM_SF + slot * Cfg::SF_SLOT_COLS;
            tmem_cp_32x128b_x4(dst, smem_desc_noswz(src, 128));                  // A rows 0..127
            if constexpr (FP4B) {
              const int nk = min(4, nkb - kb);
              for (int j = 0; j < nk; ++j) {  // B, K-block kb + j
                const uint32_t sj = src + Cfg::SFA_BYTES + j * 1024;
                tmem_cp_32x128b_x4(dst + 4 + 8 * j, smem_desc_noswz(sj, 128));        // rows 0..127
                tmem_cp_32x128b_x4(dst + 8 + 8 * j, smem_desc_noswz(sj + 512, 128));  // 128..255
              }
            } else {
              tmem_cp_32x128b_x4(dst + 4, smem_desc_noswz(src + 512, 128));     // B rows 0..127
              tmem_cp_32x128b_x4(dst + 8, smem_desc_noswz(src + 1024, 128));    // B rows 128..255
            }
            mma_commit(&sf_empty[gs]);  // the scale stage is free once the copies are done
          }
          __syncwarp();
          ++git;
        }
        const uint32_t s = it % S;
        ok = mbar_wait(&full[s], (it / S) & 1, abort_flag, tmo, SITE_MMA_FULL);
        if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_addr(sA + s * Cfg::A_BYTES);
          const uint32_t b_base = smem_addr(sB + s * Cfg::B_BYTES);
          const uint32_t sid = static_cast<uint32_t>(kb & 3);
          const uint32_t sfa_t = tmem_base + Cfg::TM_SF + slot * Cfg::SF_SLOT_COLS;
          if constexpr (FP4B) {
            // A: byte kb % 4 (one scale per K-block); B: the K-block's own
            // unit, byte k = the 32-wide strip this MMA covers
            const uint32_t sfb_t = sfa_t + 4 + 8 * sid;
#pragma unroll
            for (int k = 0; k < Cfg::BK / 32; ++k)
              mma_mxf8f6f4(tmem_base, smem_desc_sw128(a_base + k * 32, 16, 1024),
                           smem_desc_sw128(b_base + k * 32, 16, 1024),
                           idesc_mx_e4m3_e2m1(Cfg::BM, BN, sid, static_cast<uint32_t>(k)), sfa_t,
                           sfb_t, (kb > 0 || k > 0) ? 1u : 0u);
          } else {
            const uint32_t idesc = idesc_mx_e4m3(Cfg::BM, BN, sid, sid);
#pragma unroll
            for (int k = 0; k < Cfg::BK / 32; ++k)
              mma_mxf8f6f4(tmem_base, smem_desc_sw128(a_base + k * 32, 16, 1024),
                           smem_desc_sw128(b_base + k * 32, 16, 1024), idesc, sfa_t, sfa_t + 4,
                           (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          if ((kb & 3) == 3 || kb == nkb - 1) mma_commit(&slot_done[slot]);
          if (kb == nkb - 1) mma_commit(tfull);
        }
        __syncwarp();
      }
    }
  mma_done_label:
    if (lane == 0) mma_commit(mma_done);
    __syncwarp();
    {
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, tmo, SITE_TEARDOWN_MMA);
    }
    __syncwarp();
  } else {
    // ======================= epilogue (8 warps) =============================
    const uint32_t q = warp & 3;         // TMEM lane quadrant
    const uint32_t h = (warp - 2) >> 2;  // column half
    const int r_in_tile = static_cast<int>(q * 32 + lane);
    const uint32_t t_lane = tmem_base + ((q * 32) << 16) + h * 128;
    uint32_t tile_it = 0;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x, ++tile_it) {
      int m0, n0;
      mx_tile<BN>(t, args, m0, n0);
      bool ok = mbar_wait(tfull, tile_it & 1, abort_flag, tmo, SITE_EPI_TMEM_FULL);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_lane + c * 32, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);  // the next tile's MMAs may overwrite it

      const long long orow = static_cast<long long>(m0) + r_in_tile;
      const bool clipped = orow >= args.M;
      const int col0 = n0 + static_cast<int>(h) * 128;
      uint8_t* stg = sStage + (warp - 2) * Cfg::STAGE_BYTES_PER_WARP;
      const int swz = static_cast<int>((lane >> 1) & 3);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = col0 + c * 32;
        if (n >= args.N) break;
        if (lane == 0) bulk_wait_read0();  // previous chunk has left the staging buffer
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[c][j * 8 + i]);
          if (args.C && !clipped && n + j * 8 < args.N) {
            const uint4 c4 = *reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(args.C) + orow * args.N + n + j * 8);
            v[0] += bf16_lo(c4.x); v[1] += bf16_hi(c4.x);
            v[2] += bf16_lo(c4.y); v[3] += bf16_hi(c4.y);
            v[4] += bf16_lo(c4.z); v[5] += bf16_hi(c4.z);
            v[6] += bf16_lo(c4.w); v[7] += bf16_hi(c4.w);
          }
          uint4 o;
          o.x = pack_bf16x2(v[0], v[1]);
          o.y = pack_bf16x2(v[2], v[3]);
          o.z = pack_bf16x2(v[4], v[5]);
          o.w = pack_bf16x2(v[6], v[7]);
          *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ swz) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_d, stg, n, m0 + static_cast<int>(q) * 32);  // rows past M are clipped
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();  // every TMA store of this warp has completed
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace dg
