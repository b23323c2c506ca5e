// gemm.cuh -- persistent, warp-specialised FP8 GEMM with per-K-block FP32
// promotion for sm_100a (B200).
//
// Operation (DeepGEMM README summary, section "GEMMインターフェースとレイアウト制約"):
//   D = C + A @ B.T, E4M3 operands, FP32 scales per 1x128 strip of A and per
//   128x128 block of B (or per column for the K-grouped TN variant).
// Promotion (picoinsstore DeepGEMM article, paragraph 2): the tensor core's
// partial sum over each 128-wide K-block is NOT carried across K-blocks;
// it is read out of TMEM and accumulated in FP32 registers with the scales
// applied: acc += sfa * sfb * P_kb.
//
// CTA = 320 threads, one CTA per SM, persistent over output tiles:
//   warp 0      TMA producer: A/B tiles (128B-swizzled) into an S-stage ring,
//               and the per-K-block scales into a ring of their own (the
//               tile's 128 sfa values by bulk copy; for K-grouped, the sfa
//               and sfb vectors by TMA); the warp runs the loop, lane 0 issues.
//   warp 1      TMEM allocator + tcgen05.mma issuer (lane 0 of the converged
//               warp): for each
//               K-block, 4 x (M=128, N=BN, K=32) MMAs into one of 512/BN TMEM
//               accumulator buffers (all 512 columns), reset per K-block.
//   warps 2..9  promotion / epilogue: warp w reads TMEM lane quadrant (w % 4)
//               and column half ((w - 2) / 4); acc += s * P in registers
//               (NT: s = sfa from the scale ring x sfb read one K-block
//               ahead, or from a box of sfb in the same ring); at tile end
//               adds C, converts and stores D.
// The MMA runs up to 512/BN - 1 K-blocks ahead of the promotion (2 buffers at
// BN=256, 4 at BN=128); the producer runs up to S K-blocks ahead.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dg {

// MODE_PAIR is the dense GEMM on CTA pairs: a 2-CTA cluster computes a
// 256 x BN tile with tcgen05 cta_group::2 MMAs (each CTA holds 128 rows of A,
// half of the B tile and the accumulator of its 128 rows): the same operand
// traffic per SM as a 128 x 2BN single-CTA tile with half the accumulator.
// MODE_NN / MODE_TN / MODE_TT are the dense GEMM with the other operand
// layouts, named as NT is: the first letter for A ([M][K] = N, [K][M] = T),
// the second for B ([N][K] = T, as in D = A @ B.T; [K][N] = N). NN takes B as
// [K][N], TN takes A as [K][M] and B as [K][N], TT takes A as [K][M].
enum GemmMode : int {
  MODE_DENSE = 0, MODE_CONTIG = 1, MODE_MASKED = 2, MODE_KGROUPED = 3, MODE_PAIR = 4,
  MODE_NN = 5, MODE_TN = 6, MODE_TT = 7,
  // dense tiles split along K over a cluster of `split` CTAs, whose FP32
  // partials are summed through distributed shared memory (a dense launch's
  // partial last wave, or every tile of a launch with few rows), for each
  // operand layout: NT, NN, TN, TT
  MODE_SPLITK = 8, MODE_SPLITK_NN = 9, MODE_SPLITK_TN = 10, MODE_SPLITK_TT = 11,
  // dense NT for short K: a 3-stage ring and a whole-tile output staging (each
  // warp writes all its chunks, fences once and issues its stores together)
  MODE_DENSE_WIDE = 12,
  // the masked launch's partial last wave (its size known only on the
  // device), each tile split along K over a cluster
  MODE_SPLITK_MASKED = 13
};

// Split-K modes (tiles cut along K over a cluster), by layout: 8..11.
__host__ __device__ constexpr bool is_splitk(int mode) {
  return (mode >= MODE_SPLITK && mode <= MODE_SPLITK_TT) || mode == MODE_SPLITK_MASKED;
}
__host__ __device__ constexpr bool is_masked(int mode) {
  return mode == MODE_MASKED || mode == MODE_SPLITK_MASKED;
}
static_assert(!is_splitk(MODE_DENSE_WIDE) && !is_splitk(MODE_TT) && is_splitk(MODE_SPLITK_NN),
              "split-K mode range");

// The operand layout of a mode (a split-K mode has the layout of its dense mode).
constexpr int layout_of(int mode) {
  return mode == MODE_SPLITK || mode == MODE_DENSE_WIDE || mode == MODE_SPLITK_MASKED ? MODE_DENSE
         : mode == MODE_SPLITK_NN ? MODE_NN
         : mode == MODE_SPLITK_TN ? MODE_TN
         : mode == MODE_SPLITK_TT ? MODE_TT
                                  : mode;
}

constexpr int kMaxKGroups = 256;
constexpr int kMaxMaskedGroups = 1024;

struct GemmArgs {
  int M, N, K;     // dense: M; contiguous: Mt; masked: max_m; K-grouped: M (K unused)
  int G;
  int num_m_blocks, num_n_blocks;
  int total_tiles;  // host-known tile count (masked: upper bound, recomputed on device)
  const float* sfa;
  int ld_sfa;
  const float* sfb;
  const int32_t* m_indices;
  const int32_t* masked_m;
  const void* C;
  void* D;
  long long d_rows;  // rows of D viewed as [d_rows][N] (the store tensor map's outer extent)
  unsigned long long timeout_ns;
  int drop_arrive;
  int kb_off[kMaxKGroups + 1];  // K-grouped, host sizes: prefix sums of K-blocks per group
  const int32_t* ks_dev;        // K-grouped, device sizes: [G] K per group (else null)
  int kb_cap;                   // K-grouped, device sizes: K-blocks the operands hold
  int split_tile0, split;       // MODE_SPLITK: first tail tile, CTAs per tile
  // masked: split the partial last wave over clusters of tail_k CTAs (0: no)
  // when its R = T mod grid1 tiles fit in tail_clusters clusters; the
  // full-wave launch then stops at T - R and MODE_SPLITK_MASKED does the rest
  int tail_k, tail_clusters, grid1;
  int sfb_tma;                  // NT: sfb comes through the scale ring (tm_sfb), else __ldg
};

template <int MODE, int BN_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int BK = 128;  // FP8 elements (= bytes) per K-block
  static constexpr bool PAIR = MODE == MODE_PAIR;
  // ring depth from the stage size (A + this CTA's B): 48 KB -> 4, 32 KB -> 6, 24 KB -> 8
  static constexpr bool WIDE = MODE == MODE_DENSE_WIDE;
  static constexpr int STAGES = PAIR ? (BN == 256 ? 6 : 8) : WIDE ? 3 : (BN == 256 ? 4 : 6);
  static constexpr int SCALE_SLOTS = 8;  // K-grouped only
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * BK;  // this CTA's part of the B tile
  static constexpr int SCALE_BYTES = (BM + BN) * 4;
  static constexpr int THREADS = 320;
  static constexpr int NACC = 512 / BN;  // TMEM accumulator buffers (all 512 columns)
  static constexpr int TMEM_COLS = NACC * BN;
  static constexpr int EPI_COLS = BN / 2;  // accumulator columns per promotion thread

  static constexpr int GROUP_M = 16;       // tile rasterisation group (L2 reuse)
  static constexpr bool KG = MODE == MODE_KGROUPED;
  // operands stored MN-major (K-outer) in global and shared memory
  static constexpr int LAYOUT = layout_of(MODE);
  static constexpr bool A_MN = KG || LAYOUT == MODE_TN || LAYOUT == MODE_TT;
  static constexpr bool B_MN = KG || LAYOUT == MODE_NN || LAYOUT == MODE_TN;
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SCALE = OFF_B + STAGES * B_BYTES;
  // NT modes: a ring of SCALE_SLOTS K-blocks of sfa for the tile's BM rows,
  // filled by the producer's bulk copies, each slot followed (at a 128-byte
  // boundary) by a 2 x 4 box of sfb: the two column halves' 128-column
  // blocks x the four K-blocks around this one, loaded by TMA (when the sfb
  // rows are a multiple of 16 bytes long; otherwise the promotion warps read
  // sfb themselves)
  static constexpr int NT_SLOT_FLOATS = BM + 32;
  static constexpr int NT_SCALE_BYTES = NT_SLOT_FLOATS * 4;
  static constexpr int SFB_BOX_BYTES = 2 * 4 * 4;
  static constexpr int OFF_STAGE =
      ((OFF_SCALE + SCALE_SLOTS * (KG ? SCALE_BYTES : NT_SCALE_BYTES) + 1023) / 1024) * 1024;
  // output staging for the TMA-store epilogue: one 32-row x 64-byte chunk
  // (32 bf16 or 16 fp32 columns) per promotion warp, 64-byte swizzled
  static constexpr int STAGE_BYTES_PER_WARP = 32 * 64 * (WIDE ? BN / 64 : 1);
  static constexpr int STORE_COLS = KG ? 16 : 32;
  static constexpr int OFF_BAR = OFF_STAGE + 8 * STAGE_BYTES_PER_WARP;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 2 * SCALE_SLOTS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;       // tmem slot, abort flag
  static constexpr int OFF_PREFIX = OFF_MISC + 16;              // masked: prefix + counts
  static constexpr int PREFIX_BYTES = is_masked(MODE)         ? (2 * kMaxMaskedGroups + 1) * 4
                                      : MODE == MODE_KGROUPED ? (kMaxKGroups + 1) * 4
                                                              : 0;
  static constexpr int SMEM_BYTES = OFF_PREFIX + PREFIX_BYTES + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  // TMA destinations: 128-byte aligned; 128B-swizzled tiles 1024-byte aligned
  static_assert(OFF_B % 1024 == 0 && A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tiles");
  static_assert(OFF_SCALE % 128 == 0 && SCALE_BYTES % 128 == 0 && (BM * 4) % 128 == 0, "scales");
  static_assert(OFF_STAGE % 1024 == 0, "swizzled staging");
  static_assert(BN == 128 || BN == 256, "BN");
};

struct Tile {
  int valid;
  int g;
  int m0;        // first row of the tile in its group's row space
  int n0;        // first column
  int a_row;     // NT: TMA row (y) of A; K-grouped: TMA x of A (= m0)
  int b_row;     // NT: TMA row (y) of B; K-grouped: TMA x of B (= n0)
  int kb0, nkb;  // K-blocks [kb0, kb0 + nkb) along the K axis of the operands
  int rows;      // rows of this tile that may be written (before per-row checks)
  long long out_row0;  // row of D holding tile row 0
};

// Tile t -> coordinates. Every role calls this with identical inputs, so all
// roles walk the same tile sequence.
template <int MODE, int BN>
__device__ __forceinline__ Tile decode_tile(int t, const GemmArgs& a, const int* prefix,
                                            const int* mm_clamped, int rank = 0) {
  using Cfg = GemmCfg<MODE, BN>;
  Tile tl;
  tl.valid = 1;
  tl.kb0 = 0;
  tl.nkb = a.K / Cfg::BK;
  if constexpr (MODE == MODE_PAIR) {
    // pair tile (256 rows x BN): CTA `rank` of the pair owns rows [128 rank, +128)
    const int group_tiles = Cfg::GROUP_M * a.num_n_blocks;
    const int grp = t / group_tiles;
    const int first_m = grp * Cfg::GROUP_M;
    const int gm = min(a.num_m_blocks - first_m, Cfg::GROUP_M);
    const int local = t - grp * group_tiles;
    const int mb = first_m + local % gm;
    const int nb = local / gm;
    tl.g = 0;
    tl.m0 = mb * 256 + rank * 128;
    tl.n0 = nb * BN;
    tl.a_row = tl.m0;
    tl.b_row = tl.n0 + rank * (BN / 2);
    tl.rows = min(Cfg::BM, a.M - tl.m0);  // may be <= 0 for the second CTA
    tl.out_row0 = tl.m0;
  } else if constexpr (MODE == MODE_DENSE || MODE == MODE_DENSE_WIDE || MODE == MODE_CONTIG ||
                       (MODE >= MODE_NN && MODE <= MODE_TT)) {
    const int group_tiles = Cfg::GROUP_M * a.num_n_blocks;
    const int grp = t / group_tiles;
    const int first_m = grp * Cfg::GROUP_M;
    const int gm = min(a.num_m_blocks - first_m, Cfg::GROUP_M);
    const int local = t - grp * group_tiles;
    const int mb = first_m + local % gm;
    const int nb = local / gm;
    tl.m0 = mb * Cfg::BM;
    tl.n0 = nb * BN;
    tl.a_row = tl.m0;
    tl.out_row0 = tl.m0;
    if constexpr (MODE != MODE_CONTIG) {
      tl.g = 0;
      tl.b_row = tl.n0;
      tl.rows = min(Cfg::BM, a.M - tl.m0);
    } else {
      const int g = __ldg(a.m_indices + tl.m0);
      tl.g = g;
      tl.valid = (g >= 0 && g < a.G);
      tl.b_row = g * a.N + tl.n0;
      tl.rows = Cfg::BM;
    }
  } else if constexpr (is_splitk(MODE) && MODE != MODE_SPLITK_MASKED) {
    // tile split_tile0 + t of the dense rasterisation; CTA `rank` of the
    // cluster takes K-blocks [rank * KB / split, (rank + 1) * KB / split)
    const int tt = a.split_tile0 + t;
    const int group_tiles = Cfg::GROUP_M * a.num_n_blocks;
    const int grp = tt / group_tiles;
    const int first_m = grp * Cfg::GROUP_M;
    const int gm = min(a.num_m_blocks - first_m, Cfg::GROUP_M);
    const int local = tt - grp * group_tiles;
    tl.g = 0;
    tl.m0 = (first_m + local % gm) * Cfg::BM;
    tl.n0 = (local / gm) * BN;
    tl.a_row = tl.m0;
    tl.b_row = tl.n0;
    tl.out_row0 = tl.m0;
    tl.rows = min(Cfg::BM, a.M - tl.m0);
    const int KB = a.K / Cfg::BK;
    tl.kb0 = (rank * KB) / a.split;
    tl.nkb = ((rank + 1) * KB) / a.split - tl.kb0;
  } else if constexpr (is_masked(MODE)) {
    // largest g with prefix[g] <= t
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int cnt = (prefix[g + 1] - prefix[g]) / a.num_n_blocks;  // m-blocks of group g
    const int local = t - prefix[g];
    const int mb = local % cnt;
    const int nb = local / cnt;
    tl.g = g;
    tl.m0 = mb * Cfg::BM;
    tl.n0 = nb * BN;
    tl.a_row = g * a.M + tl.m0;
    tl.b_row = g * a.N + tl.n0;
    tl.rows = min(Cfg::BM, mm_clamped[g] - tl.m0);
    tl.out_row0 = static_cast<long long>(g) * a.M + tl.m0;
    if constexpr (MODE == MODE_SPLITK_MASKED) {  // CTA `rank` of the cluster: its part of K
      const int KB = a.K / Cfg::BK;
      tl.kb0 = (rank * KB) / a.split;
      tl.nkb = ((rank + 1) * KB) / a.split - tl.kb0;
    }
  } else {  // K-grouped
    const int per_g = a.num_m_blocks * a.num_n_blocks;
    const int g = t / per_g;
    const int local = t - g * per_g;
    const int group_tiles = Cfg::GROUP_M * a.num_n_blocks;
    const int grp = local / group_tiles;
    const int first_m = grp * Cfg::GROUP_M;
    const int gm = min(a.num_m_blocks - first_m, Cfg::GROUP_M);
    const int l2 = local - grp * group_tiles;
    const int mb = first_m + l2 % gm;
    const int nb = l2 / gm;
    tl.g = g;
    tl.m0 = mb * Cfg::BM;
    tl.n0 = nb * BN;
    tl.a_row = tl.m0;
    tl.b_row = tl.n0;
    tl.kb0 = prefix[g];
    tl.nkb = prefix[g + 1] - prefix[g];
    tl.rows = min(Cfg::BM, a.M - tl.m0);
    tl.out_row0 = static_cast<long long>(g) * a.M + tl.m0;
  }
  return tl;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Site codes reported with DG_ERR_TIMEOUT.
enum : unsigned int {
  SITE_PRODUCER_EMPTY = 1,
  SITE_PRODUCER_SCALE_EMPTY = 2,
  SITE_MMA_TMEM_EMPTY = 3,
  SITE_MMA_FULL = 4,
  SITE_EPI_TMEM_FULL = 5,
  SITE_EPI_SCALE_FULL = 6,
  SITE_TEARDOWN_TMA = 7,
  SITE_TEARDOWN_MMA = 8,
  SITE_K_SIZES = 9,  // device-side K-group sizes were invalid (DG_ERR_INVALID_ARG)
  SITE_SPLITK_RECV = 10,  // a split-K owner waited for its peers' partial sums
};

template <int MODE, int BN>
__global__ void __launch_bounds__(320, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_sfa,
                    const __grid_constant__ CUtensorMap tm_sfb,
                    const __grid_constant__ CUtensorMap tm_d,
                    const __grid_constant__ GemmArgs args) {
  using Cfg = GemmCfg<MODE, BN>;
  constexpr int S = Cfg::STAGES;
  constexpr int SS = Cfg::SCALE_SLOTS;
  constexpr int EC = Cfg::EPI_COLS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem + Cfg::OFF_A;
  uint8_t* sB = smem + Cfg::OFF_B;
  float* sScale = reinterpret_cast<float*>(smem + Cfg::OFF_SCALE);
  uint8_t* sStage = smem + Cfg::OFF_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  constexpr int NA = Cfg::NACC;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + NA;
  uint64_t* sfull = bars + 2 * S + 2 * NA;
  uint64_t* sempty = bars + 2 * S + 2 * NA + SS;
  uint64_t* mma_done = bars + 2 * S + 2 * NA + 2 * SS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
  int* prefix = reinterpret_cast<int*>(smem + Cfg::OFF_PREFIX);
  int* mm_clamped = prefix + kMaxMaskedGroups + 1;

  const uint32_t warp = warp_id_uniform();
  const uint32_t lane = lane_id();
  const uint64_t tmo = args.timeout_ns;
  constexpr bool PAIR = Cfg::PAIR;
  constexpr bool SPLITK = is_splitk(MODE);
  // pair: 0 = leader of the pair; split-K tail: the part of the K range
  const uint32_t rank = (PAIR || SPLITK) ? cluster_ctarank() : 0u;
  const bool leader = !PAIR || rank == 0;
  const int cta_step = PAIR     ? static_cast<int>(gridDim.x >> 1)
                       : SPLITK ? static_cast<int>(gridDim.x) / args.split
                                : static_cast<int>(gridDim.x);
  const int cta_first = PAIR     ? static_cast<int>(blockIdx.x >> 1)
                        : SPLITK ? static_cast<int>(blockIdx.x) / args.split
                                 : static_cast<int>(blockIdx.x);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], PAIR ? 16 : 8);  // pair: promotion warps of both CTAs
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
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if constexpr (Cfg::KG) {
      tma_prefetch_desc(&tm_sfa);
      tma_prefetch_desc(&tm_sfb);
    } else if (args.sfb_tma) {
      tma_prefetch_desc(&tm_sfb);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // inputs may come from the previous launch on the stream: wait for it
  // (everything above touched only shared memory, TMEM and kernel params)
  pdl_wait();
  int total_tiles = args.total_tiles;
  int tail0 = 0;  // MODE_SPLITK_MASKED: tile index of its first tile
  if constexpr (is_masked(MODE)) {
    if (warp == 2) {
      int carry = 0;
      for (int base = 0; base < args.G; base += 32) {
        const int g = base + lane;
        int mm = 0, v = 0;
        if (g < args.G) {
          mm = min(max(__ldg(args.masked_m + g), 0), args.M);
          v = ((mm + Cfg::BM - 1) / Cfg::BM) * args.num_n_blocks;
          mm_clamped[g] = mm;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= static_cast<uint32_t>(o)) v += y;
        }
        if (g < args.G) prefix[g + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) prefix[0] = 0;
    }
  }
  if constexpr (MODE == MODE_KGROUPED) {
    // K-block ranges of the groups in shared memory: from the host's prefix
    // sums, or built here from per-group K sizes in device memory (written
    // by an earlier kernel, hence after pdl_wait). A size that is negative
    // or not a multiple of 128 counts as 0, and the running total is clamped
    // to the K-blocks the operands hold; either records DG_ERR_INVALID_ARG
    // with site SITE_K_SIZES in the error word.
    if (warp == 2) {
      if (args.ks_dev == nullptr) {
        for (int g = lane; g <= args.G; g += 32) prefix[g] = args.kb_off[g];
      } else {
        int carry = 0;
        bool bad = false;
        for (int base = 0; base < args.G; base += 32) {
          const int g = base + lane;
          int v = 0;
          if (g < args.G) {
            const int k = __ldg(args.ks_dev + g);
            if (k >= 0 && (k & 127) == 0) v = k >> 7; else bad = true;
            if (v > args.kb_cap) { v = args.kb_cap; bad = true; }
          }
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= static_cast<uint32_t>(o)) v += y;
          }
          // kb_cap < 2^24, so v < 2^29 and carry + v fits in 32 bits
          if (g < args.G) {
            const int p = carry + v;
            if (p > args.kb_cap) bad = true;
            prefix[g + 1] = min(p, args.kb_cap);
          }
          carry = min(carry + __shfl_sync(0xffffffffu, v, 31), args.kb_cap);
        }
        if (lane == 0) prefix[0] = 0;
        if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(1u, SITE_K_SIZES);
      }
    }
    __syncthreads();
  }
  if constexpr (is_masked(MODE)) {
    __syncthreads();
    total_tiles = prefix[args.G];
    // the same decision in both launches (same counts, same parameters)
    const int R = args.tail_k > 1 ? total_tiles % args.grid1 : 0;
    const bool split = R > 0 && R <= args.tail_clusters;
    if constexpr (MODE == MODE_MASKED) {
      if (split) total_tiles -= R;
    } else {
      tail0 = total_tiles - R;
      total_tiles = split ? R : 0;
    }
  }

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    // ======================= TMA producer ====================================
    // The whole warp runs the loop and waits (converged, as in the MMA
    // issuer); lane 0 arms the barriers and issues the copies.
    {
      uint32_t it = 0, sit = 0;
      int dropped = -1;
      for (int t = cta_first; t < total_tiles; t += cta_step) {
        const Tile tl = decode_tile<MODE, BN>(t + tail0, args, prefix, mm_clamped, rank);
        if (!tl.valid) continue;
        for (int kb = 0; kb < tl.nkb; ++kb, ++it) {
          const uint32_t s = it % S;
          bool ok = mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER_EMPTY);
          if (!__all_sync(0xffffffffu, ok)) goto producer_done;
          {
            // take the scale slot before arming anything, so an abort here
            // leaves no uncounted copy in flight
            const uint32_t ss = sit % SS;
            ok = mbar_wait(&sempty[ss], ((sit / SS) & 1) ^ 1, abort_flag, tmo,
                           SITE_PRODUCER_SCALE_EMPTY);
            if (!__all_sync(0xffffffffu, ok)) goto producer_done;
          }
          // One thread's TMA copies are processed one after another (about
          // 60 GB/s per thread with 16 KB boxes on B200); copies issued by
          // different lanes proceed side by side. So lane 0 arms the
          // barrier, then lane 0 loads A and lanes 1..BN/128 the B tile's
          // 128-row boxes, in parallel.
          if (args.drop_arrive && it == 0) {  // test hook: never arm stage 0
            dropped = 0;
          } else {
            if constexpr (PAIR) {
              // the leader's barrier counts the bytes of both CTAs' loads
              if (lane == 0 && leader)
                mbar_arrive_expect_tx(&full[s], 2 * (Cfg::A_BYTES + Cfg::B_BYTES));
              __syncwarp();
              const uint32_t fb = dsmem_addr(smem_addr(&full[s]), 0);
              const int kk = kb * Cfg::BK;
              if (lane == 0) tma_load_2d_pair(sA + s * Cfg::A_BYTES, &tm_a, fb, kk, tl.a_row);
              if (lane == 1) tma_load_2d_pair(sB + s * Cfg::B_BYTES, &tm_b, fb, kk, tl.b_row);
            } else {
              if (lane == 0) mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + Cfg::B_BYTES);
              __syncwarp();
              const int kk = (tl.kb0 + kb) * Cfg::BK;
              // MN-major operands: 128-element-wide boxes of BK K-rows (x = MN)
              if (lane == 0) {
                if constexpr (Cfg::A_MN)
                  tma_load_2d(sA + s * Cfg::A_BYTES, &tm_a, &full[s], tl.a_row, kk);
                else
                  tma_load_2d(sA + s * Cfg::A_BYTES, &tm_a, &full[s], kk, tl.a_row);
              }
              if constexpr (Cfg::B_MN) {
                if (lane >= 1 && lane <= BN / 128) {
                  const int h = static_cast<int>(lane) - 1;
                  tma_load_2d(sB + s * Cfg::B_BYTES + h * 128 * Cfg::BK, &tm_b, &full[s],
                              tl.b_row + h * 128, kk);
                }
              } else {
                // B in 128-row boxes, one lane each (the map's box is 128 rows)
                if (lane >= 1 && lane <= BN / 128) {
                  const int h = static_cast<int>(lane) - 1;
                  tma_load_2d(sB + s * Cfg::B_BYTES + h * 128 * Cfg::BK, &tm_b, &full[s], kk,
                              tl.b_row + h * 128);
                }
              }
            }
          }
          if constexpr (Cfg::KG) {
            const uint32_t ss = sit % SS;
            if (lane == 0) mbar_arrive_expect_tx(&sfull[ss], Cfg::SCALE_BYTES);
            __syncwarp();
            float* slot = sScale + ss * (Cfg::BM + BN);
            if (lane == 3) tma_load_2d(slot, &tm_sfa, &sfull[ss], tl.m0, tl.kb0 + kb);
            if (lane == 4) tma_load_2d(slot + Cfg::BM, &tm_sfb, &sfull[ss], tl.n0, tl.kb0 + kb);
          } else {
            // sfa of the tile's rows for this K-block: BM contiguous floats of
            // the MN-major [K/128][ld] layout ([G][K/128][ld] when masked),
            // cut at ld so the copy stays inside the tensor (ld % 4 == 0, so
            // the size is a multiple of 16 bytes); rows the copy leaves out
            // lie past M and get zero scales in the promotion
            const uint32_t ss = sit % SS;
            const int nrows = min(Cfg::BM, args.ld_sfa - tl.m0);
            const uint32_t bytes = nrows > 0 ? static_cast<uint32_t>(nrows) * 4u : 0u;
            const bool sfb_box = !Cfg::B_MN && args.sfb_tma;
            if (lane == 0)
              mbar_arrive_expect_tx(&sfull[ss], bytes + (sfb_box ? Cfg::SFB_BOX_BYTES : 0u));
            __syncwarp();
            float* slot = sScale + ss * Cfg::NT_SLOT_FLOATS;
            if (lane == 3 && bytes > 0) {
              long long off = static_cast<long long>(tl.kb0 + kb) * args.ld_sfa + tl.m0;
              if constexpr (is_masked(MODE))
                off += static_cast<long long>(tl.g) * (args.K / Cfg::BK) * args.ld_sfa;
              bulk_load(slot, args.sfa + off, bytes, &sfull[ss]);
            }
            if (lane == 4 && sfb_box) {
              // sfb viewed as [G * ceil(N/128)][K/128]: rows of the tile's two
              // column halves, the 4 K-blocks whose group holds this one
              const int row = tl.g * ((args.N + 127) / 128) + tl.n0 / 128;
              tma_load_2d(slot + Cfg::BM, &tm_sfb, &sfull[ss], (tl.kb0 + kb) & ~3, row);
            }
          }
          ++sit;
          __syncwarp();
        }
      }
    producer_done:
      __syncwarp();
      // Wait (bounded, regardless of abort) for every copy still in flight:
      // the last min(it, S) stages and min(sit, SS) scale slots.
      // (pair: the leader's barriers count both CTAs' copies; the follower
      // leaves only after the leader, at the closing cluster barrier)
      for (uint32_t j = (it > S ? it - S : 0); j < it && leader; ++j) {
        if (static_cast<int>(j) == dropped) continue;
        volatile int never = 0;
        mbar_wait(&full[j % S], (j / S) & 1, &never, tmo, SITE_TEARDOWN_TMA);
      }
      for (uint32_t j = (sit > SS ? sit - SS : 0); j < sit; ++j) {
        volatile int never = 0;
        mbar_wait(&sfull[j % SS], (j / SS) & 1, &never, tmo, SITE_TEARDOWN_TMA);
      }
    }
    __syncwarp();
    if constexpr (SPLITK) {  // the promotion warps' two cluster barriers
      cluster_sync_all();
      cluster_sync_all();
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ======================================
    // The whole warp runs the loop and waits; lane 0 issues the MMAs and
    // commits. Keeping the issuing thread converged with its warp matters on
    // sm_100a: bookkeeping run by a lone diverged thread between MMA groups
    // measurably stalls the tensor pipe (about 20% per K-block here), the
    // same work in a converged warp does not.
    if (leader) {
      constexpr uint32_t idesc =
          idesc_e4m3_f32(PAIR ? 2 * Cfg::BM : Cfg::BM, BN, Cfg::A_MN ? 1 : 0, Cfg::B_MN ? 1 : 0);
      uint32_t s = 0, full_ph = 0, b = 0, tmem_ph = 0;
      for (int t = cta_first; t < total_tiles; t += cta_step) {
        const Tile tl = decode_tile<MODE, BN>(t + tail0, args, prefix, mm_clamped, rank);
        if (!tl.valid) continue;
        for (int kb = 0; kb < tl.nkb; ++kb) {
          bool ok = mbar_wait(&tempty[b], tmem_ph ^ 1, abort_flag, tmo, SITE_MMA_TMEM_EMPTY);
          if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
          tc_fence_after();
          ok = mbar_wait(&full[s], full_ph, abort_flag, tmo, SITE_MMA_FULL);
          if (!__all_sync(0xffffffffu, ok)) goto mma_done_label;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_base = smem_addr(sA + s * Cfg::A_BYTES);
            const uint32_t b_base = smem_addr(sB + s * Cfg::B_BYTES);
            const uint32_t d_tmem = tmem_base + b * BN;
#pragma unroll
            for (int k = 0; k < Cfg::BK / 32; ++k) {
              // MN-major: 32 K-rows of 128 bytes per MMA; MN atoms 16 KB apart.
              // K-major: 32 bytes of K per MMA inside the 128-byte swizzle row.
              const uint64_t da = Cfg::A_MN
                                      ? smem_desc_sw128(a_base + k * 32 * 128, 128 * Cfg::BK, 1024)
                                      : smem_desc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t db = Cfg::B_MN
                                      ? smem_desc_sw128(b_base + k * 32 * 128, 128 * Cfg::BK, 1024)
                                      : smem_desc_sw128(b_base + k * 32, 16, 1024);
              if constexpr (PAIR)
                mma_f8f6f4_pair(d_tmem, da, db, idesc, k > 0 ? 1u : 0u);
              else
                mma_f8f6f4(d_tmem, da, db, idesc, k > 0 ? 1u : 0u);
            }
            if constexpr (PAIR) {
              mma_commit_pair_mc(&empty[s], 0x3);  // frees the stage in both CTAs
              mma_commit_pair_mc(&tfull[b], 0x3);  // both accumulators are ready
            } else {
              mma_commit(&empty[s]);
              mma_commit(&tfull[b]);
            }
          }
          __syncwarp();
          if (++s == S) { s = 0; full_ph ^= 1; }
          if (++b == NA) { b = 0; tmem_ph ^= 1; }
        }
      }
    mma_done_label:
      if (lane == 0) {
        if constexpr (PAIR)
          mma_commit_pair_mc(mma_done, 0x1);
        else
          mma_commit(mma_done);
      }
      __syncwarp();
      {
        volatile int never = 0;
        mbar_wait(mma_done, 0, &never, tmo, SITE_TEARDOWN_MMA);
      }
    }
    __syncwarp();
    if constexpr (SPLITK) {  // the promotion warps' two cluster barriers
      cluster_sync_all();
      cluster_sync_all();
    }
  } else {
    // ======================= promotion + epilogue (8 warps) =================
    const uint32_t q = warp & 3;              // TMEM lane quadrant
    const uint32_t h = (warp - 2) >> 2;       // column half
    const int r_in_tile = static_cast<int>(q * 32 + lane);
    const uint32_t t_lane = tmem_base + ((q * 32) << 16);
    uint32_t acc_it = 0, sit = 0;
    bool cluster_synced = false;  // split-K tail: both cluster barriers passed
    const int KBn = args.K / Cfg::BK;  // NT: K-blocks per row of sfb
    const int nbN = (args.N + 127) / 128;
    for (int t = cta_first; t < total_tiles; t += cta_step) {
      const Tile tl = decode_tile<MODE, BN>(t + tail0, args, prefix, mm_clamped, rank);
      if (!tl.valid) continue;
      float acc[EC];
#pragma unroll
      for (int j = 0; j < EC; ++j) acc[j] = 0.0f;

      // NT scales: sfa of the tile's rows arrives per K-block in the shared
      // ring the producer fills; sfb (one value per K-block for this warp's
      // column half, consecutive floats unless B is stored [K][N]) is read
      // here, one K-block ahead.
      // (rows past M and column halves past N get zero scales; they are
      // never stored, and their scale rows may not exist)
      int pb = 0;  // offset of this column half's first sfb value (sfb < 2^31 floats)
      bool row_in = false, half_in = false;
      float sb_next = 0.f;
      auto sfb_at = [&](int kb) {
        if constexpr (Cfg::B_MN) return __ldg(args.sfb + pb + kb * nbN);
        else return __ldg(args.sfb + pb + kb);
      };
      if constexpr (!Cfg::KG) {
        row_in = tl.m0 + r_in_tile < args.M;
        const int col_first = tl.n0 + static_cast<int>(h) * EC;
        half_in = col_first < args.N;
        // sfb is [G][ceil(N/128)][K/128], or [K/128][ceil(N/128)] for B stored [K][N]
        pb = Cfg::B_MN ? col_first / 128 : (tl.g * nbN + col_first / 128) * KBn;
        if constexpr (SPLITK) pb += Cfg::B_MN ? tl.kb0 * nbN : tl.kb0;  // part starts at kb0
        if (half_in && tl.nkb > 0 && (Cfg::B_MN || !args.sfb_tma)) sb_next = sfb_at(0);
      }

      for (int kb = 0; kb < tl.nkb; ++kb) {
        const uint32_t b = acc_it % NA;
        bool ok = mbar_wait(&tfull[b], (acc_it / NA) & 1, abort_flag, tmo, SITE_EPI_TMEM_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) goto epi_done;
        tc_fence_after();
        if constexpr (!Cfg::KG) {
          const uint32_t ss = sit % SS;
          bool ok2 = mbar_wait(&sfull[ss], (sit / SS) & 1, abort_flag, tmo, SITE_EPI_SCALE_FULL);
          ok2 = __all_sync(0xffffffffu, ok2);
          if (!ok2) goto epi_done;
          const float* slot = sScale + ss * Cfg::NT_SLOT_FLOATS;
          const float sa = row_in ? slot[r_in_tile] : 0.f;
          float sb = sb_next;
          if (!Cfg::B_MN && args.sfb_tma)  // this half's 128-column block (both halves of a 128-wide tile share one)
            sb = half_in ? slot[Cfg::BM + (h * EC / 128) * 4 + ((tl.kb0 + kb) & 3)] : 0.f;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sempty[ss]);  // the slot may be refilled
          ++sit;
          const float sc = sa * sb;
          if (Cfg::B_MN || !args.sfb_tma)
            sb_next = (half_in && kb + 1 < tl.nkb) ? sfb_at(kb + 1) : 0.f;
          auto release_tmem = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (PAIR)
                mbar_arrive_cluster(dsmem_addr(smem_addr(&tempty[b]), 0));
              else
                mbar_arrive(&tempty[b]);
            }
          };
          if constexpr (EC <= 64) {
            // all chunks of this thread's columns in flight, one wait
            uint32_t r[EC / 32][32];
#pragma unroll
            for (int c = 0; c < EC / 32; ++c)
              tmem_ld_32x32b_x32(t_lane + b * BN + h * EC + c * 32, r[c]);
            tmem_ld_wait();
            release_tmem();
#pragma unroll
            for (int c = 0; c < EC / 32; ++c)
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                fma2(acc[c * 32 + i], acc[c * 32 + i + 1], sc, sc, __uint_as_float(r[c][i]),
                     __uint_as_float(r[c][i + 1]));
          } else {
            // 128 accumulator registers leave room for one chunk at a time
#pragma unroll
            for (int c = 0; c < EC / 32; ++c) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(t_lane + b * BN + h * EC + c * 32, r);
              tmem_ld_wait();
              if (c == EC / 32 - 1) release_tmem();
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                fma2(acc[c * 32 + i], acc[c * 32 + i + 1], sc, sc, __uint_as_float(r[i]),
                     __uint_as_float(r[i + 1]));
            }
          }
        } else {
          const uint32_t ss = sit % SS;
          bool ok2 = mbar_wait(&sfull[ss], (sit / SS) & 1, abort_flag, tmo, SITE_EPI_SCALE_FULL);
          ok2 = __all_sync(0xffffffffu, ok2);
          if (!ok2) goto epi_done;
          const float* slot = sScale + ss * (Cfg::BM + BN);
          const float sav = slot[r_in_tile];
          const float* sbv = slot + Cfg::BM + h * EC;
          // 16-column TMEM loads (fewer live registers), two buffers: the
          // next chunk's load is in flight while this chunk is scaled
          constexpr int KC = 16;
          uint32_t r[2][KC];
          tmem_ld_32x32b<KC>(t_lane + b * BN + h * EC, r[0]);
          tmem_ld_wait_regs(r[0]);
#pragma unroll
          for (int c = 0; c < EC / KC; ++c) {
            if (c + 1 < EC / KC) {
              tmem_ld_32x32b<KC>(t_lane + b * BN + h * EC + (c + 1) * KC, r[(c + 1) & 1]);
            } else {  // every load of this buffer has completed
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[b]);
            }
            const uint32_t(&rc)[KC] = r[c & 1];
#pragma unroll
            for (int i = 0; i < KC; i += 4) {
              // acc += sav * (sb * P): the column-scaled products reuse P's registers
              const float4 sb4 = *reinterpret_cast<const float4*>(sbv + c * KC + i);
              float u0, u1, u2, u3;
              mul2(u0, u1, sb4.x, sb4.y, __uint_as_float(rc[i]), __uint_as_float(rc[i + 1]));
              mul2(u2, u3, sb4.z, sb4.w, __uint_as_float(rc[i + 2]), __uint_as_float(rc[i + 3]));
              fma2(acc[c * KC + i], acc[c * KC + i + 1], sav, sav, u0, u1);
              fma2(acc[c * KC + i + 2], acc[c * KC + i + 3], sav, sav, u2, u3);
            }
            if (c + 1 < EC / KC) tmem_ld_wait_regs(r[(c + 1) & 1]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sempty[ss]);
          ++sit;
        }
        ++acc_it;
      }

      // ------------------------------------------------ split-K tail
      if constexpr (SPLITK) {
        // 1. every CTA of the cluster has finished its K range, so every
        //    ring is free; 2. push the rows each part owns, [own r, own r +
        //    own), into that part's ring as [src rank][own rows][256 cols];
        // 3. after the second barrier, sum the owned rows over the parts in
        //    rank order (deterministic), add C, store BF16.
        cluster_sync_all();
        const int sp = args.split, own = 128 / sp;
        const int owner = r_in_tile / own;
        const uint32_t slot = smem_addr(smem) +
            static_cast<uint32_t>(((static_cast<int>(rank) * own + (r_in_tile - owner * own)) * 256 +
                                   static_cast<int>(h) * EC) * 4);
        const uint32_t remote = dsmem_addr(slot, static_cast<uint32_t>(owner));
#pragma unroll
        for (int j = 0; j < EC; j += 4)
          st_dsmem_f32x4(remote + j * 4, acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        cluster_sync_all();
        cluster_synced = true;
        const float* recv = reinterpret_cast<const float*>(smem);
        const int tid = static_cast<int>(warp - 2) * 32 + static_cast<int>(lane);
        for (int idx = tid; idx < own * (BN / 4); idx += 256) {
          const int row = idx / (BN / 4), col = (idx % (BN / 4)) * 4;
          const int trow = static_cast<int>(rank) * own + row;
          const int gcol = tl.n0 + col;
          if (trow >= tl.rows || gcol >= args.N) continue;
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int src = 0; src < sp; ++src) {
            const float4 p = *reinterpret_cast<const float4*>(recv + (src * own + row) * 256 + col);
            v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
          }
          const long long o = (tl.out_row0 + trow) * args.N + gcol;  // N % 8 == 0
          if (args.C) {
            const uint2 c2 =
                *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(args.C) + o);
            v.x += bf16_lo(c2.x); v.y += bf16_hi(c2.x);
            v.z += bf16_lo(c2.y); v.w += bf16_hi(c2.y);
          }
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(args.D) + o) =
              make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
        }
        continue;
      }

      // ------------------------------------------------ tile epilogue
      // A warp whose 32 rows may all be written (or lie past the end of D,
      // where the store clips them) stages 32-column chunks in shared memory
      // and stores them with TMA; a warp holding rows that must stay untouched
      // (masked rows, padding rows, another group's rows) stores directly.
      {
        bool write = r_in_tile < tl.rows;
        const long long orow = tl.out_row0 + r_in_tile;
        if constexpr (MODE == MODE_CONTIG) {
          if (write) write = __ldg(args.m_indices + orow) == tl.g;
        }
        const bool clipped = orow >= args.d_rows;
        const int col0 = tl.n0 + static_cast<int>(h) * EC;
        const bool use_tma = __all_sync(0xffffffffu, write || clipped);
        if (tl.rows <= 0) {
          // pair: this CTA's half of the tile lies entirely past M
        } else if (use_tma) {
          constexpr int CW = Cfg::STORE_COLS;
          uint8_t* stg = sStage + (warp - 2) * Cfg::STAGE_BYTES_PER_WARP;
          uint8_t* const stg0 = stg;
          const int swz = static_cast<int>((lane >> 1) & 3);  // 64-byte swizzle of row `lane`
          if constexpr (Cfg::WIDE) {  // the previous tile's stores have left the staging
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < EC / CW; ++c) {
            const int n = col0 + c * CW;
            if (n >= args.N) break;
            if constexpr (Cfg::WIDE) {
              stg = sStage + (warp - 2) * Cfg::STAGE_BYTES_PER_WARP + c * 32 * 64;
            } else {
              if (lane == 0) bulk_wait_read0();  // previous chunk has left the staging buffer
              __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 o;
              if constexpr (Cfg::KG) {
                float v0 = acc[c * CW + j * 4 + 0], v1 = acc[c * CW + j * 4 + 1];
                float v2 = acc[c * CW + j * 4 + 2], v3 = acc[c * CW + j * 4 + 3];
                if (args.C && !clipped && n + j * 4 < args.N) {
                  const float4 c4 = *reinterpret_cast<const float4*>(
                      static_cast<const float*>(args.C) + orow * args.N + n + j * 4);
                  v0 += c4.x; v1 += c4.y; v2 += c4.z; v3 += c4.w;
                }
                o = make_uint4(__float_as_uint(v0), __float_as_uint(v1), __float_as_uint(v2),
                               __float_as_uint(v3));
              } else {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = acc[c * CW + j * 8 + i];
                if (args.C && !clipped && n + j * 8 < args.N) {
                  const uint4 c4 = *reinterpret_cast<const uint4*>(
                      static_cast<const __nv_bfloat16*>(args.C) + orow * args.N + n + j * 8);
                  v[0] += bf16_lo(c4.x); v[1] += bf16_hi(c4.x);
                  v[2] += bf16_lo(c4.y); v[3] += bf16_hi(c4.y);
                  v[4] += bf16_lo(c4.z); v[5] += bf16_hi(c4.z);
                  v[6] += bf16_lo(c4.w); v[7] += bf16_hi(c4.w);
                }
                o.x = pack_bf16x2(v[0], v[1]);
                o.y = pack_bf16x2(v[2], v[3]);
                o.z = pack_bf16x2(v[4], v[5]);
                o.w = pack_bf16x2(v[6], v[7]);
              }
              *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ swz) << 4)) = o;
            }
            if constexpr (!Cfg::WIDE) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tm_d, stg, n, static_cast<int>(tl.out_row0 + q * 32));
                bulk_commit();
              }
            }
          }
          if constexpr (Cfg::WIDE) {  // one fence, then every chunk's store
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
              for (int c = 0; c < EC / CW; ++c) {
                const int n = col0 + c * CW;
                if (n >= args.N) break;
                tma_store_2d(&tm_d, stg0 + c * 32 * 64, n, static_cast<int>(tl.out_row0 + q * 32));
              }
              bulk_commit();
            }
          }
        } else if (write) {
          if constexpr (Cfg::KG) {
            float* drow = static_cast<float*>(args.D) + orow * args.N;
            const float* crow = args.C ? static_cast<const float*>(args.C) + orow * args.N : nullptr;
#pragma unroll
            for (int j = 0; j < EC; j += 4) {
              const int n = col0 + j;
              if (n < args.N) {
                float4 v = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
                if (crow) {
                  const float4 c4 = *reinterpret_cast<const float4*>(crow + n);
                  v.x += c4.x; v.y += c4.y; v.z += c4.z; v.w += c4.w;
                }
                *reinterpret_cast<float4*>(drow + n) = v;
              }
            }
          } else {
            __nv_bfloat16* drow = static_cast<__nv_bfloat16*>(args.D) + orow * args.N;
            const __nv_bfloat16* crow =
                args.C ? static_cast<const __nv_bfloat16*>(args.C) + orow * args.N : nullptr;
#pragma unroll
            for (int j = 0; j < EC; j += 8) {
              const int n = col0 + j;
              if (n < args.N) {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = acc[j + i];
                if (crow) {
                  const uint4 c4 = *reinterpret_cast<const uint4*>(crow + n);
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
                *reinterpret_cast<uint4*>(drow + n) = o;
              }
            }
          }
        }
      }
    }
  epi_done:
    if constexpr (SPLITK) {  // reach both cluster barriers on every path
      if (!cluster_synced) {
        cluster_sync_all();
        cluster_synced = true;
        cluster_sync_all();
      }
    }
    if (lane == 0) bulk_wait0();  // every TMA store of this warp has completed
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  pdl_trigger();
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // the leader's MMAs into both CTAs' TMEM are done
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace dg
