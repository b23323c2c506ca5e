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
//   * each CTA asks L2 for its whole weight slice (a window of `pf` K-blocks
//     ahead, 8 K-blocks per prefetch instruction) before anything else, so
//     the slice's DRAM reads are all in flight while the CTA sets up and
//     while the previous launch finishes; the TMA loads then mostly hit L2;
//   * more than BNP tokens are cut into token tiles of BNP (a grid
//     dimension); the tiles of one N-tile run side by side, so the weight
//     tile comes from DRAM once;
//   * the partial tiles are reduced by token rows: CTA r owns tokens
//     [r R, r R + R) of its token tile, R = ceil(min(M, BNP) / splits). Each CTA writes its FP32 partial
//     to its own shared memory token-major, then one thread bulk-copies the
//     rows every other CTA owns into that CTA's receive slot for this rank
//     (cp.async.bulk shared::cta -> shared::cluster), completing bytes on the
//     owner's mbarrier; the owner sums the slices in rank order
//     (deterministic), adds C and stores whole BF16 rows of D. The receive
//     slots are dedicated, so no cluster barrier waits for the slowest CTA's
//     main loop; one split cluster barrier (arrive after barrier init, wait
//     before the copies) makes the owners' mbarriers visible to the peers.
//
// Roles per CTA (320 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// tcgen05.mma issuer (both run their loops as converged warps, lane 0
// issuing), warps 2..9 promotion (TMEM lane quadrant w % 4, column half
// (w - 2) / 4). The MMA runs up to NACC - 1 K-blocks ahead of the promotion
// (NACC accumulator buffers of BNP columns). sfa comes in chunks of 16
// K-blocks (one TMA box per chunk, two chunk slots). All waits are bounded
// (see ptx.cuh); the cluster barrier and the copies are reached
// unconditionally, also after a timeout, and a CTA that timed out stores
// nothing.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace dg {

struct DecodeArgs {
  int M, N, K;
  int KB;        // K / 128
  int splits;    // CTAs per cluster along K
  int stages;    // depth of the W/X ring (2..DecodeCfg::MAX_STAGES)
  int kg;        // K-blocks per ring stage (1, 2 or 4): one TMA box each for W and X
  int rows_per_owner;  // R = ceil(min(M, BNP) / splits): token rows reduced by each CTA
  uint32_t off_x, off_sfa, off_recv, off_bar;  // shared-memory layout (bytes)
  const float* sfb;  // [ceil(N/128)][KB]
  const void* C;     // [M][N] bf16 or null
  void* D;           // [M][N] bf16
  unsigned long long timeout_ns;
  int drop_arrive;
  int pf;        // weight K-blocks kept requested into L2 ahead of the TMA loads
};

// MINB = CTAs per SM the configuration is built for: 2 (a CTA gets half of
// shared memory, registers and TMEM, and a CTA of the next launch can sit
// beside it) or 1 (the whole SM: every promotion thread loads all its
// accumulator columns in one TMEM round trip, and twice the accumulator
// buffers). A ring stage holds kg consecutive K-blocks of W and of X, each
// moved by one 3-D TMA box (a CTA's TMA throughput grows with the box size).
// The ring depth, kg and the offsets of the other regions are chosen on the
// host per launch (decode_layout in the launcher): ring [stages][kg] W tiles
// then [stages][kg] X tiles, the two sfa chunk slots, the receive slots
// ((splits - 1) x R token rows of 128 floats), then the barriers.
// PAIR: two CTAs of the cluster (ranks 2i, 2i + 1) form a tcgen05 CTA pair
// over two neighbouring N-tiles: one M = 256 MMA, issued by the even rank,
// whose token operand is split between the two CTAs (each loads BNP / 2
// token rows) while each keeps its own 128 weight rows and its own 128 x BNP
// accumulator. A CTA then moves 16 KB of weights + BNP / 2 x 128 bytes of
// tokens per K-block instead of 16 KB + BNP x 128.
template <int BNP_, int MINB_, bool PAIR_ = false>
struct DecodeCfg {
  static constexpr int BNP = BNP_;              // token columns (MMA N)
  static constexpr int MINB = MINB_;
  static constexpr bool PAIR = PAIR_;
  static constexpr int BK = 128;
  static constexpr int W_BYTES = 128 * BK;      // weight tile (MMA A operand)
  static constexpr int X_BYTES = (PAIR ? BNP / 2 : BNP) * BK;  // this CTA's token rows (MMA B)
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int MAX_STAGES = 8;
  static constexpr int SCH = 16;                // K-blocks per sfa chunk
  static constexpr int SFA_CHUNK_BYTES = SCH * BNP * 4;
  static constexpr int PF_BOX = 8;              // K-blocks per L2 prefetch instruction
  static constexpr int EC = BNP / 2;            // accumulator columns per promotion thread
  // columns per tcgen05.ld; with one CTA per SM all EC columns are in flight
  // before a single wait, with two the loads go one 16-column chunk at a time
  static constexpr int CH = MINB == 1 ? (EC < 32 ? EC : 32) : (EC < 16 ? EC : 16);
  static constexpr bool ALL_IN_FLIGHT = MINB == 1;
  // accumulator buffers in this CTA's share of TMEM
  static constexpr int NACC = (512 / MINB) / BNP > 8 ? 8 : (512 / MINB) / BNP;
  static constexpr int TMEM_COLS = NACC * BNP;
  // barriers: full[8] empty[8] tfull[NACC] tempty[NACC] sfull[2] sempty[2]
  // mma_done recv; then the TMEM base address and the abort flag
  static constexpr int NUM_BARS = 2 * MAX_STAGES + 2 * NACC + 4 + 2;
  static constexpr int BAR_BYTES = NUM_BARS * 8 + 16;
  static constexpr int STAGE_OUT_BYTES = BNP * 128 * 4;  // token-major FP32 partial
  static constexpr int SMEM_BUDGET = MINB == 2 ? 113 * 1024 : 227 * 1024;
  static_assert((NACC & (NACC - 1)) == 0 && TMEM_COLS >= 32 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                "TMEM allocation is a power of two >= 32 columns");
  static_assert(BNP == 16 || BNP == 32 || BNP == 64 || BNP == 128, "BNP");
  static_assert(X_BYTES % 1024 == 0, "SW128 tiles are 1024-byte aligned");
  static_assert(!PAIR || (BNP == 128 && MINB == 1), "CTA pairs: 128-token tiles, one CTA per SM");
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

template <int BNP, int MINB, bool PAIR = false>
__global__ void __launch_bounds__(320, MINB)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tm_w,    // B as [KB][N][128], kg-deep boxes
                       const __grid_constant__ CUtensorMap tm_wpf,  // B as [KB][N][128], L2 prefetch
                       const __grid_constant__ CUtensorMap tm_x,    // A as [KB][M][128], kg-deep boxes
                       const __grid_constant__ CUtensorMap tm_sfa,  // sfa: [KB][ld] f32, 16-row boxes
                       const __grid_constant__ DecodeArgs args) {
  using Cfg = DecodeCfg<BNP, MINB, PAIR>;
  constexpr int NA = Cfg::NACC;
  constexpr int EC = Cfg::EC;
  constexpr int CH = Cfg::CH;
  constexpr int SCH = Cfg::SCH;
  constexpr int MS = Cfg::MAX_STAGES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = smem + args.off_x;
  float* sSfa = reinterpret_cast<float*>(smem + args.off_sfa);
  float* recv = reinterpret_cast<float*>(smem + args.off_recv);
  float* stage_out = reinterpret_cast<float*>(smem);  // over the ring, after the main loop
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + args.off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + MS;
  uint64_t* tfull = bars + 2 * MS;
  uint64_t* tempty = tfull + NA;
  uint64_t* sfull = tempty + NA;
  uint64_t* sempty = sfull + 2;
  uint64_t* mma_done = sempty + 2;
  uint64_t* rbar = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id_uniform();
  const uint32_t lane = lane_id();
  const uint64_t tmo = args.timeout_ns;
  // cluster = splits CTAs (x 2 with CTA pairs): `rank` is this CTA's part of
  // the K range; with pairs, `pc` its place in the pair (0 issues the MMAs)
  const uint32_t crank = cluster_ctarank();
  const uint32_t pc = PAIR ? (crank & 1u) : 0u;
  const uint32_t rank = PAIR ? (crank >> 1) : crank;
  const uint32_t leader_rank = crank & ~1u;
  const bool leader = !PAIR || pc == 0;
  const int splits = args.splits;
  const int S = args.stages;
  const int KG = args.kg;
  // grid (splits, token tiles, N-tiles): this CTA's tokens are
  // [m0, m0 + Mloc) -- more than BNP tokens are cut into token tiles that
  // share each weight tile (read from DRAM once, the second time from L2:
  // the tiles of one N-tile are neighbours in launch order)
  const int m0 = static_cast<int>(blockIdx.y) * BNP;
  const int Mloc = min(BNP, args.M - m0);
  const int n_tile = PAIR ? static_cast<int>(blockIdx.z) * 2 + static_cast<int>(pc)
                          : static_cast<int>(blockIdx.z);
  const int n0 = n_tile * 128;  // with pairs and an odd tile count, may lie past N
  const int kb_begin = static_cast<int>((static_cast<long long>(rank) * args.KB) / splits);
  const int kb_end = static_cast<int>((static_cast<long long>(rank + 1) * args.KB) / splits);
  const int nkb = kb_end - kb_begin;
  const int R = args.rows_per_owner;
  const int m_lo = min(Mloc, static_cast<int>(rank) * R);
  const int m_hi = min(Mloc, m_lo + R);

  if (warp == 0) {
    // The weight slice goes to L2 before anything else (an L2 prefetch reads
    // nothing into the kernel, so it may precede the PDL wait).
    const int pf0 = min(args.pf, nkb);
    for (int j = static_cast<int>(lane) * Cfg::PF_BOX; j < pf0; j += 32 * Cfg::PF_BOX)
      tma_prefetch_l2_3d(&tm_wpf, 0, n0, kb_begin + j);
    // lane i initialises barrier i (tempty / sempty count the 8 promotion warps)
    for (int i = static_cast<int>(lane); i < Cfg::NUM_BARS; i += 32) {
      const bool tmem_rel = i >= 2 * MS + NA && i < 2 * MS + 2 * NA;  // pairs: both CTAs' warps
      const bool by_warps = tmem_rel || i == 2 * MS + 2 * NA + 2 || i == 2 * MS + 2 * NA + 3;
      mbar_init(&bars[i], tmem_rel && PAIR ? 16u : by_warps ? 8u : 1u);
    }
    fence_mbarrier_init();
    __syncwarp();
    if (lane == 0) {
      *abort_flag = 0;
      // this CTA receives (splits - 1) slices of its token rows
      if (splits > 1) mbar_arrive_expect_tx(rbar, static_cast<uint32_t>((splits - 1) * (m_hi - m_lo) * 512));
      tma_prefetch_desc(&tm_w);
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_sfa);
    }
  } else if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  // pairs: the partner's copies and TMEM releases signal the even CTA's
  // barriers from the first K-block on, so the whole cluster syncs here;
  // otherwise a split arrive here, matched by cluster_wait() before the
  // split-K copies
  if (!PAIR && splits > 1) cluster_arrive_relaxed();
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next launch on the stream may start (its prologue and weight
  // prefetch) once every CTA of this grid has passed here; its PDL wait
  // still waits for this grid to complete.
  pdl_trigger();
  pdl_wait();  // inputs may come from the previous launch on the stream

  float acc[EC];
#pragma unroll
  for (int j = 0; j < EC; ++j) acc[j] = 0.0f;
  const uint32_t q = warp & 3;
  const uint32_t h = (warp - 2) >> 2;

  if (warp == 0) {
    // ======================= TMA producer (converged warp, lane 0 issues) ===
    // stage i holds K-blocks [i kg, i kg + kg) of this CTA's range (the last
    // stage's box may run past it: those K-blocks are loaded, not used)
    const int nst = (nkb + KG - 1) / KG;
    int i = 0;
    int s = 0;
    uint32_t ph = 0;
    int nchunks = 0;  // sfa chunks loaded
    bool dropped = false;
    for (; i < nst; ++i) {
      const int it = i * KG;
      const int kb = kb_begin + it;
      if (it % SCH == 0) {  // kg divides SCH: a stage never straddles two chunks
        const int c = (it / SCH) & 1;
        bool ok = mbar_wait(&sempty[c], ((it / (2 * SCH)) & 1) ^ 1, abort_flag, tmo,
                            SITE_PRODUCER_SCALE_EMPTY);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) mbar_arrive_expect_tx(&sfull[c], Cfg::SFA_CHUNK_BYTES);
        __syncwarp();
        if (lane == 2) tma_load_2d(sSfa + c * (SCH * BNP), &tm_sfa, &sfull[c], m0, kb);
        ++nchunks;
      }
      bool ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, tmo, SITE_PRODUCER_EMPTY);
      if (!__all_sync(0xffffffffu, ok)) break;
      // One thread's TMA copies are processed one after another (about 60
      // GB/s per thread with 16 KB boxes on B200), copies of different lanes
      // side by side: lane 0 arms the stage and loads W, lane 1 loads X,
      // lane 3 keeps the L2 prefetch window `pf` K-blocks ahead.
      if (args.drop_arrive && i == 0) {
        dropped = true;  // test hook: never arm stage 0
      } else if constexpr (PAIR) {
        // both CTAs' copies complete on the even CTA's barrier, armed there
        if (lane == 0 && leader)
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(2 * KG * Cfg::STAGE_BYTES));
        __syncwarp();
        const uint32_t fb = dsmem_addr(smem_addr(&full[s]), leader_rank);
        if (lane == 0) tma_load_3d_pair(sW + s * KG * Cfg::W_BYTES, &tm_w, fb, 0, n0, kb);
        if (lane == 1)
          tma_load_3d_pair(sX + s * KG * Cfg::X_BYTES, &tm_x, fb, 0,
                           m0 + static_cast<int>(pc) * (BNP / 2), kb);
      } else {
        if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(KG * Cfg::STAGE_BYTES));
        __syncwarp();
        if (lane == 0) tma_load_3d(sW + s * KG * Cfg::W_BYTES, &tm_w, &full[s], 0, n0, kb);
        if (lane == 1) tma_load_3d(sX + s * KG * Cfg::X_BYTES, &tm_x, &full[s], 0, m0, kb);
      }
      if (lane == 3) {
        const int lo = it + args.pf;
        for (int j = (lo + Cfg::PF_BOX - 1) / Cfg::PF_BOX * Cfg::PF_BOX; j < lo + KG && j < nkb;
             j += Cfg::PF_BOX)
          tma_prefetch_l2_3d(&tm_wpf, 0, n0, kb_begin + j);
      }
      __syncwarp();
      if (++s == S) {
        s = 0;
        ph ^= 1;
      }
    }
    // bounded wait for every copy still in flight: the last min(i, S) stages
    // and the last two sfa chunks (earlier ones were consumed before their
    // slot was reloaded)
    {
      volatile int never = 0;
      // (pairs: the even CTA's barriers count both CTAs' copies; the odd
      // CTA leaves only after the closing cluster barrier)
      for (int j = (i > S ? i - S : 0); j < i && leader; ++j) {
        if (dropped && j == 0) continue;
        mbar_wait(&full[j % S], (j / S) & 1, &never, tmo, SITE_TEARDOWN_TMA);
      }
      for (int ci = (nchunks > 2 ? nchunks - 2 : 0); ci < nchunks; ++ci)
        mbar_wait(&sfull[ci & 1], (ci >> 1) & 1, &never, tmo, SITE_TEARDOWN_TMA);
    }
    __syncwarp();
  } else if (warp == 1 && leader) {
    // ======================= MMA issuer (converged warp, lane 0 issues) =====
    constexpr uint32_t idesc = idesc_e4m3_f32(PAIR ? 256 : 128, BNP, 0, 0);
    const uint16_t pair_mask = static_cast<uint16_t>(3u << leader_rank);
    const int nst = (nkb + KG - 1) / KG;
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nst; ++i) {
      bool ok = mbar_wait(&full[s], ph, abort_flag, tmo, SITE_MMA_FULL);
      if (!__all_sync(0xffffffffu, ok)) break;
      for (int j = 0; j < KG && i * KG + j < nkb; ++j) {
        const int it = i * KG + j;
        const uint32_t b = static_cast<uint32_t>(it) % NA;
        ok = mbar_wait(&tempty[b], ((it / NA) & 1) ^ 1, abort_flag, tmo, SITE_MMA_TMEM_EMPTY);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t w_base = smem_addr(sW + (s * KG + j) * Cfg::W_BYTES);
          const uint32_t x_base = smem_addr(sX + (s * KG + j) * Cfg::X_BYTES);
#pragma unroll
          for (int k = 0; k < Cfg::BK / 32; ++k) {
            const uint64_t dw = smem_desc_sw128(w_base + k * 32, 16, 1024);
            const uint64_t dx = smem_desc_sw128(x_base + k * 32, 16, 1024);
            if constexpr (PAIR)
              mma_f8f6f4_pair(tmem_base + b * BNP, dw, dx, idesc, k > 0 ? 1u : 0u);
            else
              mma_f8f6f4(tmem_base + b * BNP, dw, dx, idesc, k > 0 ? 1u : 0u);
          }
          if constexpr (PAIR)
            mma_commit_pair_mc(&tfull[b], pair_mask);  // both accumulators are ready
          else
            mma_commit(&tfull[b]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        if constexpr (PAIR)
          mma_commit_pair_mc(&empty[s], pair_mask);  // frees the stage in both CTAs
        else
          mma_commit(&empty[s]);
      }
      __syncwarp();
      if (++s == S) {
        s = 0;
        ph ^= 1;
      }
    }
    if (lane == 0) {
      if constexpr (PAIR)
        mma_commit_pair_mc(mma_done, static_cast<uint16_t>(1u << crank));
      else
        mma_commit(mma_done);
    }
    __syncwarp();
    volatile int never = 0;
    mbar_wait(mma_done, 0, &never, tmo, SITE_TEARDOWN_MMA);
    __syncwarp();
  } else if (warp >= 2) {
    // ======================= promotion (8 warps) =======================
    const uint32_t t_lane = tmem_base + ((q * 32) << 16);
    const float* pb = args.sfb + static_cast<long long>(n_tile) * args.KB + kb_begin;
    const bool n_in = n0 < args.N;  // a pair's odd CTA past the last N-tile reads no sfb
    // sfb prefetch ring of 4 K-blocks, loop unrolled by 4 (slot u refilled in place)
    float sbr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (u < nkb && n_in) sbr[u] = __ldg(pb + u);
    for (int it0 = 0; it0 < nkb; it0 += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = it0 + u;
        if (it >= nkb) break;
        const uint32_t b = static_cast<uint32_t>(it) % NA;
        const int c = (it / SCH) & 1;
        bool ok = mbar_wait(&tfull[b], (it / NA) & 1, abort_flag, tmo, SITE_EPI_TMEM_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) goto promo_done;
        if (it % SCH == 0) {
          bool ok2 = mbar_wait(&sfull[c], (it / (2 * SCH)) & 1, abort_flag, tmo,
                               SITE_EPI_SCALE_FULL);
          ok2 = __all_sync(0xffffffffu, ok2);
          if (!ok2) goto promo_done;
        }
        tc_fence_after();
        const float sb = sbr[u];
        if (it + 4 < nkb && n_in) sbr[u] = __ldg(pb + it + 4);
        const float* sa = sSfa + c * (SCH * BNP) + (it % SCH) * BNP + h * EC;
        auto fma_chunk = [&](int cc, const uint32_t (&r)[CH]) {
#pragma unroll
          for (int i = 0; i < CH; i += 4) {
            const float4 s4 = *reinterpret_cast<const float4*>(sa + cc * CH + i);
            float t0, t1, t2, t3;
            mul2(t0, t1, s4.x, s4.y, sb, sb);
            mul2(t2, t3, s4.z, s4.w, sb, sb);
            fma2(acc[cc * CH + i], acc[cc * CH + i + 1], t0, t1, __uint_as_float(r[i]),
                 __uint_as_float(r[i + 1]));
            fma2(acc[cc * CH + i + 2], acc[cc * CH + i + 3], t2, t3, __uint_as_float(r[i + 2]),
                 __uint_as_float(r[i + 3]));
          }
        };
        auto release_tmem = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR)
              mbar_arrive_cluster(dsmem_addr(smem_addr(&tempty[b]), leader_rank));
            else
              mbar_arrive(&tempty[b]);
          }
        };
        if constexpr (Cfg::ALL_IN_FLIGHT) {
          uint32_t r[EC / CH][CH];
#pragma unroll
          for (int cc = 0; cc < EC / CH; ++cc)
            tmem_ld_32x32b<CH>(t_lane + b * BNP + h * EC + cc * CH, r[cc]);
          tmem_ld_wait();
          release_tmem();
#pragma unroll
          for (int cc = 0; cc < EC / CH; ++cc) fma_chunk(cc, r[cc]);
        } else {
#pragma unroll
          for (int cc = 0; cc < EC / CH; ++cc) {
            uint32_t r[CH];
            tmem_ld_32x32b<CH>(t_lane + b * BNP + h * EC + cc * CH, r);
            tmem_ld_wait();
            if (cc == EC / CH - 1) release_tmem();
            fma_chunk(cc, r);
          }
        }
        if (it % SCH == SCH - 1 || it == nkb - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&sempty[c]);
        }
      }
    }
  promo_done:;
  }

  // ---------------------------------------------------------- split-K reduction
  // Every role is done and every copy / MMA of this CTA has landed, so its
  // ring is free: the FP32 partial goes there token-major ([token][128 rows]).
  tc_fence_before();
  __syncthreads();
  if (warp >= 2) {
    float* col = stage_out + h * EC * 128 + q * 32 + lane;
#pragma unroll
    for (int j = 0; j < EC; ++j) col[j * 128] = acc[j];
    fence_proxy_async_smem();  // the bulk copies below read it through the async proxy
  }
  __syncthreads();
  if (splits > 1) {
    if (!PAIR) cluster_wait();  // every owner's receive barrier is initialised
    if (threadIdx.x == 0) {
      for (int o = 0; o < splits; ++o) {
        if (o == static_cast<int>(rank)) continue;
        const int lo = min(Mloc, o * R);
        const int hi = min(Mloc, lo + R);
        if (hi <= lo) continue;
        const int slot = static_cast<int>(rank) < o ? static_cast<int>(rank) : static_cast<int>(rank) - 1;
        // the owner is the CTA at the same place in its pair
        const uint32_t orank = PAIR ? static_cast<uint32_t>(2 * o) + pc : static_cast<uint32_t>(o);
        const uint32_t dst = dsmem_addr(smem_addr(recv + slot * R * 128), orank);
        const uint32_t mb = dsmem_addr(smem_addr(rbar), orank);
        bulk_copy_to_cluster(dst, stage_out + lo * 128, static_cast<uint32_t>((hi - lo) * 512), mb);
      }
    }
  }
  bool ok = true;
  if (splits > 1 && m_hi > m_lo) {
    volatile int never = 0;
    ok = mbar_wait(rbar, 0, &never, tmo, SITE_SPLITK_RECV);
  }
  // The copies complete only on the owners' barriers, so a CTA's staged
  // partial must stay until every owner has seen its receive slots complete:
  // each CTA arrives once its own have (or it receives nothing) and waits for
  // the whole cluster before it exits.
  if (splits > 1 && !PAIR) cluster_arrive_relaxed();
  if (ok && !*abort_flag) {
    // this CTA's token rows: item = (token m, 8 weight rows), weight rows fastest
    const int items = (m_hi - m_lo) * 16;
    for (int itm = threadIdx.x; itm < items; itm += blockDim.x) {
      const int m = m_lo + (itm >> 4);
      const int c8 = (itm & 15) << 3;
      const int gn = n0 + c8;
      if (gn >= args.N) continue;  // N % 8 == 0: a group of 8 is wholly in or out
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int src = 0; src < splits; ++src) {  // rank order: deterministic
        const float* p;
        if (src == static_cast<int>(rank)) {
          p = stage_out + m * 128 + c8;
        } else {
          const int slot = src < static_cast<int>(rank) ? src : src - 1;
          p = recv + (slot * R + (m - m_lo)) * 128 + c8;
        }
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
        v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
      }
      const long long o = static_cast<long long>(m0 + m) * args.N + gn;
      if (args.C) {
        const uint4 c4 = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(args.C) + o);
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
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.D) + o) = out;
    }
  }
  if constexpr (PAIR) {
    // the even CTA's MMAs wrote this CTA's TMEM and read its shared memory:
    // neither is released before the whole cluster is here
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
  } else {
    if (splits > 1) cluster_wait();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
  }
}

}  // namespace dg
