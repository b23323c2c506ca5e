// gemm_decode.cuh -- FP8 fine-grained-scaled GEMM for small M (M <= 128,
// decode), sm_100a. Same operation and promotion rule as gemm.cuh:
//   D[m][n] = C[m][n] + sum_kb sfa[kb][m] * sfb[n/128][kb] * P_kb[m][n]
// but arranged for the memory-bound regime (the DeepGEMM launch article notes
// decode shapes are bandwidth-bound; the blog "从矩阵乘法为什么这么慢说起" §2.2,
// §5.1 describes thin shapes starving the tensor cores):
//
//   * swap-AB: the 128 weight rows of an N-tile fill the MMA's M = 128 lanes
//     and the tokens become the MMA's N (BNP = 16..128 columns), so one
//     128-row weight block -- and therefore one sfb value per K-block --
//     covers the whole tile;
//   * split-K across a thread-block cluster: the `splits` CTAs of a cluster
//     share one N-tile and each streams its own slice of K-blocks, so
//     n_tiles x splits CTAs keep HBM busy even when N/128 is small;
//   * the partial tiles are reduced through distributed shared memory: CTA r
//     owns units [16r/splits, 16(r+1)/splits) of the tile's sixteen 8-row
//     units (splits <= 8, any count); after a cluster
//     barrier (every ring is free) each CTA pushes, with remote stores, the
//     rows of its FP32 partial that CTA o owns into o's receive slot for
//     rank r; after a second barrier each CTA sums its units over the slots in
//     rank order (deterministic) from its own shared memory, adds C and
//     stores BF16. Remote stores need no round trip; remote loads, which an
//     owner pulling the partials would issue, are latency-bound.
//
// Roles per CTA (320 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// tcgen05.mma issuer (both run their loops as converged warps, lane 0
// issuing), warps 2..9 promotion (TMEM lane quadrant w % 4, column half
// (w - 2) / 4). The MMA runs up to NACC - 1 K-blocks ahead of the promotion
// (NACC accumulator buffers of BNP columns). All waits are bounded (see
// ptx.cuh); both cluster barriers are reached unconditionally, also after a
// timeout. With a single split the launch has no cluster and CTA barriers
// replace them.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace dg {

struct DecodeArgs {
  int M, N, K;
  int KB;       // K / 128
  int splits;   // CTAs per cluster along K
  const float* sfb;  // [ceil(N/128)][KB]
  const void* C;     // [M][N] bf16 or null
  void* D;           // [M][N] bf16
  unsigned long long timeout_ns;
  int drop_arrive;
};

// MINB = CTAs per SM the configuration is built for: 2 (a CTA gets half of
// shared memory, registers and TMEM) or 1 (the whole SM: every promotion
// thread loads all its accumulator columns in one TMEM round trip, and twice
// the accumulator buffers).
template <int BNP_, int MINB_>
struct DecodeCfg {
  static constexpr int BNP = BNP_;              // token columns (MMA N)
  static constexpr int MINB = MINB_;
  static constexpr int BK = 128;
  static constexpr int W_BYTES = 128 * BK;      // weight tile (MMA A operand)
  static constexpr int X_BYTES = BNP * BK;      // token tile (MMA B operand)
  static constexpr int RING = MINB == 2 ? 96 * 1024 : 192 * 1024;
  static constexpr int STAGES_RAW = RING / (W_BYTES + X_BYTES);
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int SS = 8;                  // sfa slots
  // a TMA destination in shared memory must be 128-byte aligned, so each
  // slot holds at least 32 floats even when BNP = 16
  static constexpr int SLOT_FLOATS = BNP < 32 ? 32 : BNP;
  static constexpr int EC = BNP / 2;            // accumulator columns per promotion thread
  // columns per tcgen05.ld; with one CTA per SM all EC columns are in flight
  // before a single wait, with two the loads go one 16-column chunk at a time
  static constexpr int CH = MINB == 1 ? (EC < 32 ? EC : 32) : (EC < 16 ? EC : 16);
  static constexpr bool ALL_IN_FLIGHT = MINB == 1;
  // accumulator buffers in this CTA's share of TMEM
  static constexpr int NACC = (512 / MINB) / BNP > 8 ? 8 : (512 / MINB) / BNP;
  static constexpr int TMEM_COLS = NACC * BNP;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
  static constexpr int OFF_SCALE = OFF_X + STAGES * X_BYTES;
  static constexpr int OFF_BAR = OFF_SCALE + SS * SLOT_FLOATS * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 2 * SS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // receive slots of the split-K reduction, overlaying the ring:
  // [src rank][owned unit (< ceil(16/splits))][row in unit (8)][RECV_PITCH]
  // floats, tokens along the row; at most 168 rows (splits = 7: 7 x 3 x 8).
  // The pitch is padded by 4 floats so that consecutive rows start in
  // different banks.
  static constexpr int MAX_SPLITS = 8;
  static constexpr int RECV_PITCH = BNP + 4;
  static constexpr int RECV_ROWS = 168;
  static constexpr int RECV_BYTES = RECV_ROWS * RECV_PITCH * 4;
  static_assert(RECV_BYTES <= STAGES * (W_BYTES + X_BYTES), "receive slots fit the ring");
  static_assert((NACC & (NACC - 1)) == 0 && TMEM_COLS >= 32 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                "TMEM allocation is a power of two >= 32 columns");
  static_assert(BNP == 16 || BNP == 32 || BNP == 64 || BNP == 128, "BNP");
  static_assert(OFF_SCALE % 1024 == 0 && (SLOT_FLOATS * 4) % 128 == 0, "TMA smem alignment");
  static_assert(OFF_X % 1024 == 0 && X_BYTES % 1024 == 0, "SW128 tiles are 1024-byte aligned");
  static_assert(SMEM_BYTES <= (MINB == 2 ? 113 : 227) * 1024, "MINB CTAs per SM");
};

// Split-K reduction of a cluster's partial 128 x BNP tiles (swap-AB decode
// kernels): CTA `rank` of `splits` owns the 8-row units [16 rank / splits,
// 16 (rank + 1) / splits) of the tile. After a cluster barrier (every ring is
// free) each of warps 2..9 -- thread (q, h, lane) holding tile row
// 32 q + lane, tokens [h EC, h EC + EC) in acc -- pushes its row into the
// owner's receive slot for this rank with remote stores; after a second
// barrier each CTA sums its units over the slots in rank order
// (deterministic), adds C and stores BF16 rows of D (tokens m < M, weight rows
// n < N). With one split the barriers are CTA barriers and the slots local.
// `recv` is this CTA's shared memory (the ring, free by then).
template <int BNP, int EC, int RECV_PITCH>
__device__ __forceinline__ void splitk_reduce_store(const float (&acc)[EC], float* recv,
                                                    uint32_t rank, int splits, uint32_t warp,
                                                    uint32_t lane, int n0, int M, int N,
                                                    const void* C, void* D) {
  const uint32_t q = warp & 3;
  const uint32_t h = (warp - 2) >> 2;
  if (splits > 1) cluster_sync_all(); else __syncthreads();
  // rank o owns units [16o/splits, 16(o+1)/splits); a slot holds UMAX units
  const int UMAX = (16 + splits - 1) / splits;
  if (warp >= 2) {
    // push: this thread holds row n_local of the tile for tokens [h*EC, h*EC+EC)
    const int n_local = static_cast<int>(q * 32 + lane);
    const int unit = n_local >> 3;
    const int owner = (splits * (unit + 1) + 15) / 16 - 1;  // largest o with 16o/splits <= unit
    const int owner_lo = (owner * 16) / splits;
    const int slot_row = ((static_cast<int>(rank) * UMAX + (unit - owner_lo)) << 3) + (n_local & 7);
    float* dst = recv + slot_row * RECV_PITCH + h * EC;
    if (splits == 1) {
#pragma unroll
      for (int j = 0; j < EC; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    } else {
      const uint32_t remote = dsmem_addr(smem_addr(dst), static_cast<uint32_t>(owner));
#pragma unroll
      for (int j = 0; j < EC; j += 4)
        st_dsmem_f32x4(remote + j * 4, acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
  }
  if (splits > 1) cluster_sync_all(); else __syncthreads();
  {
    // this CTA owns units [lo, hi); item = (unit uu, token m), token fastest
    // so that a warp reads consecutive floats of a slot row
    const int lo = (static_cast<int>(rank) * 16) / splits;
    const int hi = ((static_cast<int>(rank) + 1) * 16) / splits;
    const int items = BNP * (hi - lo);
    for (int itm = threadIdx.x; itm < items; itm += blockDim.x) {
      const int uu = itm / BNP;
      const int m = itm - uu * BNP;
      const int gn = n0 + ((lo + uu) << 3);
      if (m >= M || gn >= N) continue;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int src = 0; src < splits; ++src) {  // rank order: deterministic
        const float* p = recv + ((src * UMAX + uu) << 3) * RECV_PITCH + m;
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8) v[r8] += p[r8 * RECV_PITCH];
      }
      const long long o = static_cast<long long>(m) * N + gn;
      if (C) {
        const uint4 c4 = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(C) + o);
        v[0] += bf16_lo(c4.x); v[1] += bf16_hi(c4.x);
        v[2] += bf16_lo(c4.y); v[3] += bf16_hi(c4.y);
        v[4] += bf16_lo(c4.z); v[5] += bf16_hi(c4.z);
        v[6] += bf16_lo(c4.w); v[7] += bf16_hi(c4.w);
      }
      uint4 out;
      out.x = pack_bf16x2(v[0], v[1]);
      out.y = pack_bf16x2(v[2], v[3]);
      out.z = pack_bf16x2(v[4], v[5]);
      out.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(D) + o) = out;
    }
  }
}

template <int BNP, int MINB>
__global__ void __launch_bounds__(320, MINB)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tm_w,    // B: [N][K] e4m3
                       const __grid_constant__ CUtensorMap tm_x,    // A: [M][K] e4m3
                       const __grid_constant__ CUtensorMap tm_sfa,  // sfa: [KB][ld] f32
                       const __grid_constant__ DecodeArgs args) {
  using Cfg = DecodeCfg<BNP, MINB>;
  constexpr int S = Cfg::STAGES;
  constexpr int SS = Cfg::SS;
  constexpr int EC = Cfg::EC;
  constexpr int CH = Cfg::CH;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sW = smem + Cfg::OFF_W;
  uint8_t* sX = smem + Cfg::OFF_X;
  float* sScale = reinterpret_cast<float*>(smem + Cfg::OFF_SCALE);
  float* recv = reinterpret_cast<float*>(smem);  // receive slots, after the main loop
  constexpr int NA = Cfg::NACC;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + NA;
  uint64_t* sfull = bars + 2 * S + 2 * NA;
  uint64_t* sempty = bars + 2 * S + 2 * NA + SS;
  uint64_t* mma_done = bars + 2 * S + 2 * NA + 2 * SS;
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
    for (int i = 0; i < NA; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    for (int i = 0; i < SS; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 8);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_sfa);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The first weight tiles of this CTA go to L2 while the previous kernel on
  // the stream (typically the activation quantiser) finishes: their DRAM
  // latency leaves the critical path. Only a prefetch happens before the wait.
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < S && j < nkb; ++j) tma_prefetch_l2(&tm_w, (kb_begin + j) * Cfg::BK, n0);
  }
  pdl_wait();  // inputs may come from the previous launch on the stream

  float acc[EC];
#pragma unroll
  for (int j = 0; j < EC; ++j) acc[j] = 0.0f;
  const uint32_t q = warp & 3;
  const uint32_t h = (warp - 2) >> 2;

  if (warp == 0) {
    // ======================= TMA producer (converged warp, lane 0 issues) ===
    int it = 0;
    int dropped = -1;
    for (; it < nkb; ++it) {
      const int s = it % S;
      const int ss = it % SS;
      bool ok = mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      ok = mbar_wait(&sempty[ss], ((it / SS) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER_SCALE_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int kb = kb_begin + it;
      if (args.drop_arrive && it == 0) {
        dropped = 0;  // test hook: never arm stage 0
      } else if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], Cfg::W_BYTES + Cfg::X_BYTES);
        tma_load_2d(sW + s * Cfg::W_BYTES, &tm_w, &full[s], kb * Cfg::BK, n0);
        tma_load_2d(sX + s * Cfg::X_BYTES, &tm_x, &full[s], kb * Cfg::BK, 0);
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&sfull[ss], BNP * 4);
        tma_load_2d(sScale + ss * Cfg::SLOT_FLOATS, &tm_sfa, &sfull[ss], 0, kb);
      }
      __syncwarp();
    }
    // bounded wait for every copy still in flight
    for (int j = (it > S ? it - S : 0); j < it; ++j) {
      if (j == dropped) continue;
      volatile int never = 0;
      mbar_wait(&full[j % S], (j / S) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    for (int j = (it > SS ? it - SS : 0); j < it; ++j) {
      volatile int never = 0;
      mbar_wait(&sfull[j % SS], (j / SS) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= MMA issuer (converged warp, lane 0 issues) =====
    constexpr uint32_t idesc = idesc_e4m3_f32(128, BNP, 0, 0);
    for (int it = 0; it < nkb; ++it) {
      const uint32_t b = static_cast<uint32_t>(it) % NA;
      bool ok = mbar_wait(&tempty[b], ((it / NA) & 1) ^ 1, abort_flag, tmo, SITE_MMA_TMEM_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int s = it % S;
      ok = mbar_wait(&full[s], (it / S) & 1, abort_flag, tmo, SITE_MMA_FULL);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t w_base = smem_addr(sW + s * Cfg::W_BYTES);
        const uint32_t x_base = smem_addr(sX + s * Cfg::X_BYTES);
#pragma unroll
        for (int k = 0; k < Cfg::BK / 32; ++k)
          mma_f8f6f4(tmem_base + b * BNP, smem_desc_sw128(w_base + k * 32, 16, 1024),
                     smem_desc_sw128(x_base + k * 32, 16, 1024), idesc, k > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&tfull[b]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(mma_done);
    __syncwarp();
    volatile int never = 0;
    mbar_wait(mma_done, 0, &never, tmo, SITE_TEARDOWN_MMA);
    __syncwarp();
  } else {
    // ======================= promotion (8 warps) =======================
    const uint32_t t_lane = tmem_base + ((q * 32) << 16);
    const float* pb = args.sfb + static_cast<long long>(n_tile) * args.KB + kb_begin;
    // sfb prefetch ring of 4 K-blocks, loop unrolled by 4 (slot u refilled in place)
    float sbr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (u < nkb) sbr[u] = __ldg(pb + u);
    for (int it0 = 0; it0 < nkb; it0 += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = it0 + u;
        if (it >= nkb) break;
        const uint32_t b = static_cast<uint32_t>(it) % NA;
        bool ok = mbar_wait(&tfull[b], (it / NA) & 1, abort_flag, tmo, SITE_EPI_TMEM_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) goto promo_done;
        const int ss = it % SS;
        bool ok2 = mbar_wait(&sfull[ss], (it / SS) & 1, abort_flag, tmo, SITE_EPI_SCALE_FULL);
        ok2 = __all_sync(0xffffffffu, ok2);
        if (!ok2) goto promo_done;
        tc_fence_after();
        const float sb = sbr[u];
        if (it + 4 < nkb) sbr[u] = __ldg(pb + it + 4);
        const float* sa = sScale + ss * Cfg::SLOT_FLOATS + h * EC;
        auto fma_chunk = [&](int c, const uint32_t (&r)[CH]) {
#pragma unroll
          for (int i = 0; i < CH; i += 4) {
            const float4 s4 = *reinterpret_cast<const float4*>(sa + c * CH + i);
            float t0, t1, t2, t3;
            mul2(t0, t1, s4.x, s4.y, sb, sb);
            mul2(t2, t3, s4.z, s4.w, sb, sb);
            fma2(acc[c * CH + i], acc[c * CH + i + 1], t0, t1, __uint_as_float(r[i]),
                 __uint_as_float(r[i + 1]));
            fma2(acc[c * CH + i + 2], acc[c * CH + i + 3], t2, t3, __uint_as_float(r[i + 2]),
                 __uint_as_float(r[i + 3]));
          }
        };
        auto release_tmem = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        };
        if constexpr (Cfg::ALL_IN_FLIGHT) {
          uint32_t r[EC / CH][CH];
#pragma unroll
          for (int c = 0; c < EC / CH; ++c)
            tmem_ld_32x32b<CH>(t_lane + b * BNP + h * EC + c * CH, r[c]);
          tmem_ld_wait();
          release_tmem();
#pragma unroll
          for (int c = 0; c < EC / CH; ++c) fma_chunk(c, r[c]);
        } else {
#pragma unroll
          for (int c = 0; c < EC / CH; ++c) {
            uint32_t r[CH];
            tmem_ld_32x32b<CH>(t_lane + b * BNP + h * EC + c * CH, r);
            tmem_ld_wait();
            if (c == EC / CH - 1) release_tmem();
            fma_chunk(c, r);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[ss]);
      }
    }
  promo_done:;
  }

  // ---------------------------------------------------------- split-K reduction
  // Every role is done and every copy / MMA has landed, so this CTA's ring is
  // free; the first barrier (inside) makes that true for every CTA of the cluster.
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
