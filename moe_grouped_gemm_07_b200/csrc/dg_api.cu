// dg_api.cu -- host side of libdg.so: argument validation, the per-shape
// planner (tile width, grid size), TMA tensor-map encoding and kernel launch
// for every entry point declared in include/dg.h. All device code of the
// library is compiled in this one translation unit.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dg.h"
#include "gemm.cuh"
#include "gemm_mx.cuh"
#include "gemm_mx_decode.cuh"
#include "gemm_decode.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

using dg::GemmArgs;

constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms_cap{0};
std::atomic<unsigned long long> g_timeout_ns{0};
std::atomic<int> g_drop_next{0};
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_pdl{1};

// Launches `kern` on `st`, with programmatic dependent launch when enabled
// (dg_set_pdl) and with a 1-D cluster of `cluster` CTAs when cluster > 1.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (g_pdl.load()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int g_sm_count[kMaxDevices];
std::once_flag g_sm_once[kMaxDevices];

bool print_configs() {
  static const bool on = [] {
    const char* e = std::getenv("DG_PRINT_CONFIGS");
    return e && e[0] && e[0] != '0';
  }();
  return on;
}

dg_status cuda_fail(cudaError_t e, const char* what) {
  if (print_configs()) std::fprintf(stderr, "[dg] %s: %s\n", what, cudaGetErrorString(e));
  return DG_ERR_CUDA;
}

dg_status device_sms(int* dev, int* sms) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) return DG_ERR_CUDA;
  std::call_once(g_sm_once[*dev], [d = *dev] {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sm_count[d] = n;
  });
  int n = g_sm_count[*dev];
  if (n <= 0) return DG_ERR_CUDA;
  const int cap = g_num_sms_cap.load();
  *sms = (cap > 0 && cap < n) ? cap : n;
  return DG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

unsigned long long timeout_ns() {
  const unsigned long long t = g_timeout_ns.load();
  return t ? t : 2000000000ull;
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D row-major tensor: `inner` contiguous elements per row, `outer` rows,
// row pitch `pitch_bytes`; box {box_inner, box_outer}.
dg_status make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
                      uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return DG_ERR_CUDA;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (print_configs()) std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed: %d\n", (int)r);
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// 3-D tensor: dims {d0, d1, d2} (d0 contiguous), byte strides of dims 1 and
// 2, box {b0, b1, b2}. A [rows][K] operand viewed as [K/128][rows][128] this
// way lets one box carry several K-blocks of a tile, each landing as the
// [rows][128] tile a 2-D box would give.
dg_status make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0,
                      uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                      uint32_t b1, uint32_t b2,
                      CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return DG_ERR_CUDA;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (print_configs()) std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled (3-D) failed: %d\n", (int)r);
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// ---------------------------------------------------------------- launches
template <int MODE, int BN>
dg_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                      const CUtensorMap& tsb, const CUtensorMap& td, const GemmArgs& args,
                      int grid, cudaStream_t st, int dev, int cluster = 1) {
  using Cfg = dg::GemmCfg<MODE, BN>;
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  auto kern = dg::gemm_fp8_kernel<MODE, BN>;
  std::call_once(once[dev], [&] {
    attr_err[dev] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");
  cudaError_t e = launch(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, st, cluster, ta,
                         tb, tsa, tsb, td, args);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

int take_drop_flag() { return g_drop_next.exchange(0); }

// Tile width (DG_FORCE_BN=128|256 overrides it, for tuning): 256 columns
// unless that leaves the GPU with clearly fewer
// waves' worth of work than 128-column tiles (a 128-wide tile costs about half
// of a 256-wide one, with ~15% lower per-tile efficiency).
int choose_bn(long long m_blocks, int N, int sms) {
  static const int forced = [] {
    const char* e = std::getenv("DG_FORCE_BN");
    return e ? std::atoi(e) : 0;
  }();
  if (forced == 128 || forced == 256) return forced;
  const long long t256 = m_blocks * ((N + 255) / 256);
  const long long t128 = m_blocks * ((N + 127) / 128);
  const double c256 = 2.0 * static_cast<double>((t256 + sms - 1) / sms);
  const double c128 = 1.15 * static_cast<double>((t128 + sms - 1) / sms);
  return c128 < c256 ? 128 : 256;
}

// D = C (or 0) for K == 0 / all-empty K-grouped problems.
template <typename T>
__global__ void copy_or_zero_kernel(const T* __restrict__ c, T* __restrict__ d, long long n) {
  dg::pdl_wait();
  dg::pdl_trigger();
  for (long long i = blockIdx.x * 1ll * blockDim.x + threadIdx.x; i < n;
       i += 1ll * gridDim.x * blockDim.x)
    d[i] = c ? c[i] : T(0);
}

template <typename T>
dg_status copy_or_zero(const void* c, void* d, long long n, int sms, cudaStream_t st) {
  if (n <= 0) return DG_OK;
  if (c == d) return DG_OK;
  const int grid = static_cast<int>(std::min<long long>((n + 255) / 256, 8ll * sms));
  cudaError_t e = launch(copy_or_zero_kernel<T>, dim3(grid), dim3(256), 0, st, 1,
                         static_cast<const T*>(c), static_cast<T*>(d), n);
  if (e != cudaSuccess) return cuda_fail(e, "copy launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

struct Bf16Raw {
  uint16_t v;
  __host__ __device__ Bf16Raw() : v(0) {}
  __host__ __device__ explicit Bf16Raw(int) : v(0) {}
};

// Shared NT launcher for dense / contiguous / masked.
// M <= 128 on 128 x 256 tiles, each split along K over a cluster when the
// tiles leave SMs idle, instead of the swap-AB decode kernel:
// DG_SMALL_M_TILES=1 always, =0 never, unset: the cost model in
// dispatch_decode decides for 65..128 tokens (read on every call).
int small_m_tiles_env() {
  const char* e = std::getenv("DG_SMALL_M_TILES");
  return e ? (e[0] == '1' ? 1 : 0) : -1;
}

// Dense NT tiles with few K-blocks spend much of each tile in the epilogue:
// up to 12 K-blocks run the 3-stage, whole-tile-staging kernel
// (MODE_DENSE_WIDE). DG_WIDE_EPI=0|1 forces it off or on (read on every call).
bool wide_epilogue(int KB) {
  if (const char* e = std::getenv("DG_WIDE_EPI")) return e[0] == '1';
  return KB <= 12;
}

// Split-K tail of a dense launch (MODE_SPLITK): DG_TAIL_SPLIT=0 turns it off.
bool tail_split_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DG_TAIL_SPLIT");
    return !(e && e[0] == '0');
  }();
  return on;
}

// With R = tiles % grid tiles left for a partial last wave, split each over k
// CTAs (k a power of two, at most 8, R * k <= grid, at least 4 K-blocks per
// part). The second launch, its prologue and the cluster exchange cost about
// as much as 40 K-blocks of a tile (measured on B200: splits that save fewer
// ran slower), so a split must save at least that: KB - KB / k >= 40.
// Returns k (1 = no split).
int tail_split_for(long long tiles, int grid, int KB) {
  if (tiles <= grid) return 1;
  const long long R = tiles % grid;
  if (R == 0) return 1;
  int k = 1;
  while (k < 8 && R * (2 * k) <= grid && KB / (2 * k) >= 4) k *= 2;
  return KB - KB / k >= 40 ? k : 1;
}

// The occupancy probes below may leave an error of their own in the
// runtime's last-error slot, which they clear. So that this never swallows an
// error of the caller's earlier asynchronous work, a probe runs only when no
// error is pending (otherwise it reports "unknown" and caches nothing, and
// the caller's error stays pending for its own check).
bool no_pending_error() { return cudaPeekAtLastError() == cudaSuccess; }

// How many k-CTA clusters of the split-K kernel the device runs at once
// (cached per device and k; 0 on error).
template <int SMODE = dg::MODE_SPLITK>
int splitk_clusters(int dev, int k) {
  using Cfg = dg::GemmCfg<SMODE, 256>;
  static std::mutex mu;
  static int cache[kMaxDevices][9];
  static bool done[kMaxDevices][9];
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev][k]) {
    if (!no_pending_error()) return 0;
    done[dev][k] = true;
    cache[dev][k] = 0;
    auto kern = dg::gemm_fp8_kernel<SMODE, 256>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(k, 1, 1);
      cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
      cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = k;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess) cache[dev][k] = n;
    }
    cudaGetLastError();
  }
  return cache[dev][k];
}

// One wave of 128 x 256 tiles (few rows): every tile split along K over a
// cluster of k CTAs, k the largest power of two <= 8 whose clusters all fit
// at once with at least 4 K-blocks per part.
int whole_split_k(long long tiles, int KB, int sms, int dev) {
  int k = 1;
  while (k < 8 && tiles * (2 * k) <= sms && KB / (2 * k) >= 4 && splitk_clusters(dev, 2 * k) >= tiles)
    k *= 2;
  return k;
}

// NT scale ring: sfb viewed as [G * ceil(N/128)][K/128] FP32 with 4 x 2
// boxes (four K-blocks of two 128-column blocks), when its rows are a
// multiple of 16 bytes long (K/128 % 4 == 0); otherwise the kernel reads sfb
// with plain loads. Sets args->sfb_tma accordingly.
void make_sfb_box_map(CUtensorMap* m, const float* sfb, int N, int K, int G, GemmArgs* args) {
  const int kbn = K / 128;
  const int nbn = (N + 127) / 128;
  args->sfb_tma = 0;
  if (kbn % 4 != 0) return;
  if (make_map_2d(m, sfb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, kbn, static_cast<uint64_t>(G) * nbn,
                  4ull * kbn, 4, 2, CU_TENSOR_MAP_SWIZZLE_NONE) == DG_OK)
    args->sfb_tma = 1;
}

template <int MODE>
dg_status run_nt(const void* A, const float* sfa, int ld_sfa, const void* B, const float* sfb,
                 const int32_t* m_indices, const int32_t* masked_m, const void* C, void* D,
                 int rows_total, int M_logical, int N, int K, int G, long long m_blocks_bound,
                 long long tiles_if_known, cudaStream_t st, const char* name,
                 long long m_blocks_plan = -1, bool whole_split = false) {
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  // the tile width is planned for the expected number of 128-row blocks
  // (masked: the caller's expected_m hint), the launch for the bound
  const int bn =
      whole_split ? 256 : choose_bn(m_blocks_plan > 0 ? m_blocks_plan : m_blocks_bound, N, sms);
  CUtensorMap ta, tb, dummy;
  std::memset(&dummy, 0, sizeof dummy);
  s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, rows_total, K, 128, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  // B in 128-row boxes: the kernel loads a BN-row tile as BN/128 boxes from
  // separate producer lanes
  s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, static_cast<uint64_t>(G) * N, K, 128,
                  128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  // D as [rows_total][N] bf16; 32x32 boxes, 64-byte swizzle (TMA-store epilogue)
  CUtensorMap td;
  s = make_map_2d(&td, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, rows_total, 2ull * N, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B);
  if (s != DG_OK) return s;
  GemmArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M_logical;
  args.N = N;
  args.K = K;
  args.G = G;
  args.d_rows = rows_total;
  args.num_m_blocks = static_cast<int>((MODE == dg::MODE_MASKED) ? (M_logical + 127) / 128
                                                                  : (rows_total + 127) / 128);
  args.num_n_blocks = (N + bn - 1) / bn;
  const long long tiles = tiles_if_known >= 0
                              ? tiles_if_known * args.num_n_blocks
                              : m_blocks_bound * args.num_n_blocks;
  args.total_tiles = static_cast<int>(tiles);
  args.sfa = sfa;
  args.ld_sfa = ld_sfa;
  args.sfb = sfb;
  args.m_indices = m_indices;
  args.masked_m = masked_m;
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  CUtensorMap tsb = dummy;
  make_sfb_box_map(&tsb, sfb, N, K, G, &args);
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(sms, tiles)));
  // Dense: a partial last wave of R tiles runs as a second launch that
  // splits each tile along K over a cluster of k CTAs (MODE_SPLITK); the
  // first launch takes the full waves. Both are ordered on the stream.
  int split = 1;
  const long long R = tiles > grid ? tiles % grid : 0;
  if (MODE == dg::MODE_DENSE && bn == 256 && whole_split && tiles <= grid) {
    const int k = whole_split_k(tiles, K / 128, sms, dev);
    if (print_configs())
      std::fprintf(stderr, "[dg] %s M=%d N=%d K=%d: BM=128 BN=256 tiles=%lld split %d\n", name,
                   M_logical, N, K, tiles, k);
    if (k > 1) {
      args.split_tile0 = 0;
      args.split = k;
      args.drop_arrive = 0;
      return launch_gemm<dg::MODE_SPLITK, 256>(ta, tb, dummy, tsb, td, args,
                                               static_cast<int>(tiles) * k, st, dev, k);
    }
    return launch_gemm<MODE, 256>(ta, tb, dummy, tsb, td, args, static_cast<int>(tiles), st, dev);
  }
  if (MODE == dg::MODE_DENSE && bn == 256 && tail_split_enabled()) {
    split = tail_split_for(tiles, grid, K / 128);
    if (split > 1 && splitk_clusters(dev, split) < R) split = 1;  // not all at once
  }
  if (print_configs())
    std::fprintf(stderr,
                 "[dg] %s M=%d N=%d K=%d G=%d: BM=128 BN=%d tiles=%lld grid=%d tail split %dx%lld\n",
                 name, M_logical, N, K, G, bn, tiles, grid, split, split > 1 ? R : 0ll);
  if (split > 1) {
    GemmArgs tail = args;
    args.total_tiles = static_cast<int>(tiles - R);
    dg_status s2 = launch_gemm<MODE, 256>(ta, tb, dummy, tsb, td, args, grid, st, dev);
    if (s2 != DG_OK) return s2;
    tail.total_tiles = static_cast<int>(R);
    tail.split_tile0 = static_cast<int>(tiles - R);
    tail.split = split;
    tail.drop_arrive = 0;
    return launch_gemm<dg::MODE_SPLITK, 256>(ta, tb, dummy, tsb, td, tail,
                                             static_cast<int>(R) * split, st, dev, split);
  }
  if (MODE == dg::MODE_DENSE && bn == 256 && wide_epilogue(K / 128)) {
    if (print_configs()) std::fprintf(stderr, "[dg] %s: wide epilogue (3 stages)\n", name);
    return launch_gemm<dg::MODE_DENSE_WIDE, 256>(ta, tb, dummy, tsb, td, args, grid, st, dev);
  }
  if (MODE == dg::MODE_MASKED && bn == 256 && tail_split_enabled()) {
    // The tile count T is known only on the device. A second launch of
    // clusters of k CTAs takes the partial last wave (R = T mod grid tiles,
    // each split along K) when R fits in its clusters; both launches work
    // out R from the counts, the full-wave launch stops at T - R. Planned
    // when a split saves at least 16 K-blocks of a tile.
    const int KB = K / 128;
    int k = 0;
    for (int c = 4; c >= 2 && k == 0; c /= 2)
      if (KB - KB / c >= 16 && KB / c >= 4) k = c;
    int clusters = k ? std::min(splitk_clusters<dg::MODE_SPLITK_MASKED>(dev, k), grid / k) : 0;
    if (print_configs())
      std::fprintf(stderr, "[dg] %s: masked tail split %d x up to %d clusters\n", name, k, clusters);
    if (k > 1 && clusters > 0) {
      args.tail_k = k;
      args.tail_clusters = clusters;
      args.grid1 = grid;
      dg_status s1 = launch_gemm<MODE, 256>(ta, tb, dummy, tsb, td, args, grid, st, dev);
      if (s1 != DG_OK) return s1;
      GemmArgs tail = args;
      tail.split = k;
      tail.drop_arrive = 0;
      return launch_gemm<dg::MODE_SPLITK_MASKED, 256>(ta, tb, dummy, tsb, td, tail, clusters * k, st,
                                                      dev, k);
    }
  }
  if (bn == 256) return launch_gemm<MODE, 256>(ta, tb, dummy, tsb, td, args, grid, st, dev);
  return launch_gemm<MODE, 128>(ta, tb, dummy, tsb, td, args, grid, st, dev);
}

// Dense GEMM with A and/or B stored MN-major (NN, TN, TT); 128 x 256 tiles.
template <int MODE>
dg_status run_layout(const void* A, const float* sfa, int ld_sfa, const void* B, const float* sfb,
                     const void* C, void* D, int M, int N, int K, cudaStream_t st,
                     const char* name) {
  using Cfg = dg::GemmCfg<MODE, 256>;
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  CUtensorMap ta, tb, td, dummy;
  std::memset(&dummy, 0, sizeof dummy);
  if (Cfg::A_MN)  // A stored [K][M]: 128 x 128 boxes, x along M
    s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, M, K, M, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  else
    s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  if (Cfg::B_MN)  // B stored [K][N]: two 128 x 128 boxes per tile, x along N
    s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, N, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  else
    s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  s = make_map_2d(&td, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, 2ull * N, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B);
  if (s != DG_OK) return s;
  GemmArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.d_rows = M;
  args.num_m_blocks = (M + 127) / 128;
  args.num_n_blocks = (N + 255) / 256;
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  if (tiles > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
  args.total_tiles = static_cast<int>(tiles);
  args.sfa = sfa;
  args.ld_sfa = ld_sfa;
  args.sfb = sfb;
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  CUtensorMap tsb = dummy;
  if (MODE == dg::MODE_TT) make_sfb_box_map(&tsb, sfb, N, K, 1, &args);  // B stored [N][K]
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(sms, tiles)));
  // Split-K as for NT: with one wave of tiles (few rows) every tile is split
  // along K over a cluster when that saves more K-blocks per CTA than the
  // exchange costs (~10 K-blocks on B200); otherwise a partial last wave runs
  // as a second, split launch.
  constexpr int SPLIT_MODE = MODE == dg::MODE_NN   ? dg::MODE_SPLITK_NN
                             : MODE == dg::MODE_TN ? dg::MODE_SPLITK_TN
                                                   : dg::MODE_SPLITK_TT;
  const int KB = K / 128;
  int k = 1;
  long long first = tiles;  // tiles of the unsplit launch
  if (tail_split_enabled()) {
    if (tiles <= grid) {
      k = whole_split_k(tiles, KB, sms, dev);
      if (KB - (KB + k - 1) / k < 10) k = 1;
      if (k > 1) first = 0;
    } else if (tiles % grid != 0) {
      k = tail_split_for(tiles, grid, KB);
      if (k > 1 && splitk_clusters(dev, k) < tiles % grid) k = 1;
      if (k > 1) first = tiles - tiles % grid;
    }
  }
  if (print_configs())
    std::fprintf(stderr, "[dg] %s M=%d N=%d K=%d: BM=128 BN=256 tiles=%lld grid=%d split %dx%lld\n",
                 name, M, N, K, tiles, grid, k, k > 1 ? tiles - first : 0ll);
  if (first > 0) {
    GemmArgs full = args;
    full.total_tiles = static_cast<int>(first);
    dg_status s1 = launch_gemm<MODE, 256>(ta, tb, dummy, tsb, td, full,
                                          static_cast<int>(std::min<long long>(grid, first)), st, dev);
    if (s1 != DG_OK || k == 1) return s1;
  }
  args.total_tiles = static_cast<int>(tiles - first);
  args.split_tile0 = static_cast<int>(first);
  args.split = k;
  args.drop_arrive = 0;
  return launch_gemm<SPLIT_MODE, 256>(ta, tb, dummy, tsb, td, args,
                                      static_cast<int>(tiles - first) * k, st, dev, k);
}

// Shared argument checks of the dense entry points. a_mn / b_mn: the operand
// is stored MN-major, so its rows of M (N) bytes must be 16-byte multiples.
dg_status check_dense(const void* A, const void* sfa, const void* B, const void* sfb, const void* C,
                      void* D, int M, int N, int K, bool a_mn, bool b_mn) {
  if (M < 0 || N < 0 || K < 0) return DG_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if ((a_mn && M % 16 != 0) || (b_mn && N % 16 != 0)) return DG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return DG_OK;
  if (!D) return DG_ERR_INVALID_ARG;
  if (!aligned16(D) || (C && !aligned16(C))) return DG_ERR_MISALIGNED;
  if (K == 0) return DG_OK;
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb))
    return DG_ERR_MISALIGNED;
  return DG_OK;
}

template <int MODE>
dg_status dense_layout_entry(const void* A, const float* sfa, const void* B, const float* sfb,
                             const void* C, void* D, int M, int N, int K, void* stream,
                             const char* name) {
  using Cfg = dg::GemmCfg<MODE, 256>;
  dg_status s = check_dense(A, sfa, B, sfb, C, D, M, N, K, Cfg::A_MN, Cfg::B_MN);
  if (s != DG_OK || M == 0 || N == 0) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {
    int dev = 0, sms = 0;
    if ((s = device_sms(&dev, &sms)) != DG_OK) return s;
    return copy_or_zero<Bf16Raw>(C, D, static_cast<long long>(M) * N, sms, st);
  }
  // sfa: [K/128][align4(M)] for A stored [M][K], [K/128][M] for A stored [K][M]
  const int ld = Cfg::A_MN ? M : (M + 3) / 4 * 4;
  return run_layout<MODE>(A, sfa, ld, B, sfb, C, D, M, N, K, st, name);
}

// ---------------------------------------------------------------- CTA pairs
// Dense GEMM with M > 128 on CTA pairs (256 x BN tiles, cta_group::2 MMAs;
// each CTA loads half of the B tile). Opt-in with DG_PAIR=1: measured on B200
// it runs at the speed of the single-CTA kernel (the per-SM operand bytes
// halve for B, but the shared L2-to-SM path stays the limit), so the
// single-CTA kernel remains the default.
bool use_pairs() {
  static const bool on = [] {
    const char* e = std::getenv("DG_PAIR");
    return e && e[0] == '1';
  }();
  return on;
}

// Columns of a pair tile: 256, or 128 with DG_PAIR_BN=128.
int pair_bn() {
  static const int bn = [] {
    const char* e = std::getenv("DG_PAIR_BN");
    return (e && std::atoi(e) == 128) ? 128 : 256;
  }();
  return bn;
}

dg_status run_pair(const void* A, const float* sfa, int ld_sfa, const void* B, const float* sfb,
                   const void* C, void* D, int M, int N, int K, cudaStream_t st) {
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  CUtensorMap ta, tb, td, dummy;
  std::memset(&dummy, 0, sizeof dummy);
  if ((s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  // pair tiles are 256 x bn; each CTA of a pair loads half (bn/2 rows) of B
  const int bn = pair_bn();
  if ((s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 128, bn / 2,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if ((s = make_map_2d(&td, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, 2ull * N, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_64B)) != DG_OK)
    return s;
  GemmArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.num_m_blocks = (M + 255) / 256;
  args.num_n_blocks = (N + bn - 1) / bn;
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  args.total_tiles = static_cast<int>(tiles);
  args.sfa = sfa;
  args.ld_sfa = ld_sfa;
  args.sfb = sfb;
  args.C = C;
  args.D = D;
  args.d_rows = M;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  CUtensorMap tsb = dummy;
  make_sfb_box_map(&tsb, sfb, N, K, 1, &args);
  const int pairs = static_cast<int>(std::max<long long>(1, std::min<long long>(sms / 2, tiles)));
  if (print_configs())
    std::fprintf(stderr,
                 "[dg] fp8_gemm_nt pairs M=%d N=%d K=%d: 256x%d tiles=%lld on %d CTA pairs\n", M,
                 N, K, bn, tiles, pairs);
  if (bn == 256)
    return launch_gemm<dg::MODE_PAIR, 256>(ta, tb, dummy, tsb, td, args, 2 * pairs, st, dev, 2);
  return launch_gemm<dg::MODE_PAIR, 128>(ta, tb, dummy, tsb, td, args, 2 * pairs, st, dev, 2);
}

// ---------------------------------------------------------------- decode path
// Largest cluster size (1..16) that the device can co-schedule for this
// kernel (above 8 only where non-portable cluster sizes are allowed); cached
// per device and instantiation.
// Largest cluster size (<= 16, or 8 without non-portable sizes) of which
// enough co-resident clusters fit to fill most of the GPU; 0 on failure.
int probe_max_cluster(const void* kern, int smem) {
  if (!no_pending_error()) return -1;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 0;
  const bool nonportable =
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  cudaGetLastError();
  for (int c = nonportable ? 16 : 8; c >= 1; --c) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c, 1, 1);
    cfg.blockDim = dim3(320, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n * c >= 64) return c;
    cudaGetLastError();
  }
  return 0;
}

// Caches a probe's answer per device unless the probe could not run (-1: an
// earlier error was pending).
template <typename Probe>
int cached_probe(std::mutex& mu, int (&best)[kMaxDevices], bool (&done)[kMaxDevices], int dev,
                 Probe probe) {
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    const int r = probe();
    if (r < 0) return r;
    best[dev] = r;
    done[dev] = true;
  }
  return best[dev];
}

template <int BNP, int MINB, bool PAIR = false>
int max_cluster(int dev) {
  static std::mutex mu;
  static int best[kMaxDevices];
  static bool done[kMaxDevices];
  return cached_probe(mu, best, done, dev, [] {
    return probe_max_cluster(
        reinterpret_cast<const void*>(dg::gemm_decode_kernel<BNP, MINB, PAIR>),
        dg::DecodeCfg<BNP, MINB, PAIR>::SMEM_BUDGET);
  });
}

template <int BNP, int MINB, bool W4>
int max_cluster_mx(int dev) {
  static std::mutex mu;
  static int best[kMaxDevices];
  static bool done[kMaxDevices];
  return cached_probe(mu, best, done, dev, [] {
    return probe_max_cluster(
        reinterpret_cast<const void*>(dg::gemm_mx_decode_kernel<BNP, MINB, W4>),
        dg::MxDecodeCfg<BNP, MINB, W4>::SMEM_BYTES);
  });
}

// Decode plan: CTAs per SM (MINB) and split count, from a sweep of both
// configurations x 1..8 splits x 1/2/4 K-blocks per stage over the decode
// shapes on B200, timed back to back. Tokens up to 64 take the half-SM
// configuration (two CTAs per SM; a CTA of the next launch can also sit
// beside one of this launch and prefetch its weights early) with about 256
// CTAs; 128-token tiles need the whole SM, about 128 CTAs. A CTA streams at
// most ~85 GB/s through TMA, so the grid must be wide; more splits than that
// lose to their exchange. At most 8 splits (the portable cluster size and the
// co-schedulable cluster size) and at least 2 K-blocks per split.
struct DecodePlan {
  int minb, splits;
};

// Weight K-blocks each decode CTA keeps requested into L2 ahead of its TMA
// loads, a multiple of 8 (DG_DECODE_PF overrides, read on every call).
int decode_prefetch_kblocks() {
  int pf = 64;
  if (const char* e = std::getenv("DG_DECODE_PF")) {
    const int f = std::atoi(e);
    if (f >= 0) pf = f;
  }
  return (pf + 7) / 8 * 8;
}

// How many clusters of `s` CTAs of this decode configuration, with `smem`
// bytes of shared memory each, the device runs at once (cached per device,
// configuration, s and smem; 0 on error). A cluster lives inside one GPC, so
// e.g. clusters of 7 one-CTA-per-SM CTAs leave SMs of every GPC idle and
// fewer of them fit than SMs / 7.
template <int BNP, int MINB, bool PAIR = false>
int decode_cluster_capacity(int dev, int s, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  if (s < 1 || s > 8) return 0;
  const auto key = std::make_tuple(dev, s, smem);
  const int cs = PAIR ? 2 * s : s;  // CTAs per cluster
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  if (!no_pending_error()) return 0;
  int cap = 0;
  const void* kern = reinterpret_cast<const void*>(dg::gemm_decode_kernel<BNP, MINB, PAIR>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           dg::DecodeCfg<BNP, MINB, PAIR>::SMEM_BUDGET) == cudaSuccess) {
    if (cs > 1) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(320, 1, 1);
      cfg.dynamicSmemBytes = static_cast<size_t>(smem);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess) cap = n;
    } else {
      int per_sm = 0, sms = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 320, smem) == cudaSuccess &&
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        cap = per_sm * sms;
    }
  }
  cudaGetLastError();  // only the queries' own errors can be pending here
  cache[key] = cap;
  return cap;
}

DecodePlan plan_decode(int bnp, int m_tiles, int n_tiles, int KB, int sms, int cap1, int cap2) {
  auto clampi = [](int v, int lo, int hi) { return std::max(lo, std::min(v, hi)); };
  const int minb = bnp <= 64 ? 2 : 1;
  const int cap = minb == 1 ? cap1 : cap2;
  const int target = (minb == 2 ? 256 : 128) * sms / 148;
  const int splits =
      clampi(target / (n_tiles * m_tiles), 1, std::min(std::min(8, cap), std::max(1, KB / 2)));
  return {minb, splits};
}

// Plan of the block-scaled decode kernel (gemm_mx_decode.cuh), from a sweep
// of both configurations x 1..8 splits over the decode shapes on B200: more
// than 4-5 splits lose (each CTA keeps too few K-blocks and its cluster-barrier
// reduction grows); with at least one tile per SM a single split on two CTAs
// per SM is best; M > 64 prefers one CTA per SM, M <= 64 two.
DecodePlan plan_mx_decode(int M, int n_tiles, int KB, int sms, int cap1, int cap2) {
  auto clampi = [](int v, int lo, int hi) { return std::max(lo, std::min(v, hi)); };
  if (n_tiles >= sms) return {2, 1};
  if (M > 64) return {1, clampi(std::min(sms / n_tiles, KB / 2), 1, std::min(5, cap1))};
  return {2, clampi(std::min(2 * sms / n_tiles, KB / 2), 1, std::min(4, cap2))};
}

// Shared-memory layout of one decode launch: the deepest W/X ring (2..8
// stages) that fits beside the sfa chunk slots, the split-K receive slots and
// the barriers in the configuration's share of the SM. False if it does not fit.
template <int BNP, int MINB, bool PAIR = false>
bool decode_layout(int M, int splits, int kg, dg::DecodeArgs* a, int* smem_bytes) {
  using Cfg = dg::DecodeCfg<BNP, MINB, PAIR>;
  const int R = (M + splits - 1) / splits;
  const int recv = splits > 1 ? (splits - 1) * R * 512 : 0;
  const int sfa = 2 * Cfg::SFA_CHUNK_BYTES;
  const int fixed = sfa + recv + Cfg::BAR_BYTES + 1024;  // + alignment slack of the base
  const int stage = kg * Cfg::STAGE_BYTES;
  int stages = (Cfg::SMEM_BUDGET - fixed) / stage;
  stages = std::min(stages, Cfg::MAX_STAGES);
  if (stages < 2 || stages * stage < Cfg::STAGE_OUT_BYTES) return false;
  a->stages = stages;
  a->kg = kg;
  a->rows_per_owner = R;
  a->off_x = static_cast<uint32_t>(stages * kg * Cfg::W_BYTES);
  a->off_sfa = static_cast<uint32_t>(stages * stage);
  a->off_recv = a->off_sfa + static_cast<uint32_t>(sfa);
  a->off_bar = a->off_recv + static_cast<uint32_t>(recv);
  *smem_bytes = static_cast<int>(a->off_bar) + Cfg::BAR_BYTES + 1024;
  return *smem_bytes <= Cfg::SMEM_BUDGET;
}

// Lowers `splits` until every cluster of the launch (with its shared-memory
// layout) is resident at once.
template <int BNP, int MINB, bool PAIR = false>
int fit_splits(int dev, int M, int clusters, int splits) {
  for (; splits > 1; --splits) {
    dg::DecodeArgs a;
    int smem = 0;
    bool fits = false;
    for (int kg = 4; kg >= 1 && !fits; kg /= 2)
      fits = decode_layout<BNP, MINB, PAIR>(std::min(M, BNP), splits, kg, &a, &smem);
    if (fits && decode_cluster_capacity<BNP, MINB, PAIR>(dev, splits, smem) >= clusters) break;
  }
  return splits;
}

template <int BNP, int MINB, bool PAIR = false>
dg_status run_decode(const void* A, const float* sfa, const void* B, const float* sfb,
                     const void* C, void* D, int M, int N, int K, int splits, cudaStream_t st) {
  using Cfg = dg::DecodeCfg<BNP, MINB, PAIR>;
  const int KB = K / 128;
  const int n_tiles = (N + 127) / 128;
  const int m_tiles = (M + BNP - 1) / BNP;
  const int ld = (M + 3) / 4 * 4;
  const int Mt = std::min(M, BNP);  // tokens of the largest token tile
  dg::DecodeArgs args;
  std::memset(&args, 0, sizeof args);
  int smem = 0;
  // K-blocks per ring stage: the deepest box (4, 2, 1) that still leaves a
  // ring of two stages; DG_DECODE_KG=1|2|4 forces it (read on every call)
  int kg = 0;
  if (const char* e = std::getenv("DG_DECODE_KG")) {
    const int f = std::atoi(e);
    if (f == 1 || f == 2 || f == 4) kg = f;
  }
  bool fits = false;
  if (kg) {
    fits = decode_layout<BNP, MINB, PAIR>(Mt, splits, kg, &args, &smem);
  } else {
    for (kg = 4; kg >= 1 && !fits; kg /= 2)
      fits = decode_layout<BNP, MINB, PAIR>(Mt, splits, kg, &args, &smem);
  }
  if (!fits) return DG_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap tw, twpf, tx, tsa;
  dg_status s;
  // weights and tokens viewed as [KB][rows][128]: one box = kg K-blocks of a tile
  if ((s = make_map_3d(&tw, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, N, KB, K, 128, 128, 128,
                       static_cast<uint32_t>(args.kg), CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if ((s = make_map_3d(&twpf, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, N, KB, K, 128, 128, 128,
                       Cfg::PF_BOX)) != DG_OK)
    return s;
  // tokens: BNP rows per box, or the half a CTA of a pair holds
  if ((s = make_map_3d(&tx, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, M, KB, K, 128, 128,
                       PAIR ? BNP / 2 : BNP, static_cast<uint32_t>(args.kg),
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if ((s = make_map_2d(&tsa, sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ld, KB, 4ull * ld, BNP,
                       Cfg::SCH, CU_TENSOR_MAP_SWIZZLE_NONE)) != DG_OK)
    return s;
  args.M = M;
  args.N = N;
  args.K = K;
  args.KB = KB;
  args.splits = splits;
  args.sfb = sfb;
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  args.pf = decode_prefetch_kblocks();
  if (print_configs())
    std::fprintf(stderr,
                 "[dg] fp8_gemm_nt decode M=%d N=%d K=%d: swap-AB BNP=%d (%d CTA/SM)%s, n_tiles=%d x "
                 "token tiles %d x split-K %d (cluster), %d CTAs, %d stages x %d K-blocks, %d B smem\n",
                 M, N, K, BNP, MINB, PAIR ? " CTA pairs" : "", n_tiles, m_tiles, splits,
                 (PAIR ? (n_tiles + 1) / 2 * 2 : n_tiles) * m_tiles * splits, args.stages, args.kg,
                 smem);
  const int cs = PAIR ? 2 * splits : splits;
  cudaError_t e = launch(dg::gemm_decode_kernel<BNP, MINB, PAIR>,
                         dim3(cs, m_tiles, PAIR ? (n_tiles + 1) / 2 : n_tiles), dim3(320),
                         static_cast<size_t>(smem), st, cs, tw, twpf, tx, tsa, args);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

dg_status dispatch_decode(const void* A, const float* sfa, const void* B, const float* sfb,
                          const void* C, void* D, int M, int N, int K, int sms, int dev,
                          cudaStream_t st) {
  const int KB = K / 128;
  const int n_tiles = (N + 127) / 128;
  // token tile: up to 64 tokens in one tile of the half-SM configuration,
  // 65..128 tokens in one 128-token tile on the whole SM. DG_DECODE_BNP=64
  // cuts 65..128 tokens into two 64-token tiles instead (measured slower on
  // B200: the second token tile re-reads every weight tile through L2); read
  // on every call
  int bnp = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  if (M > 64)
    if (const char* e = std::getenv("DG_DECODE_BNP"))
      if (std::atoi(e) == 64) bnp = 64;
  const int m_tiles = (M + bnp - 1) / bnp;
  int cap1 = 0, cap2 = 0;  // co-schedulable cluster sizes of the two configurations
  switch (bnp) {
    case 16: cap1 = max_cluster<16, 1>(dev); cap2 = max_cluster<16, 2>(dev); break;
    case 32: cap1 = max_cluster<32, 1>(dev); cap2 = max_cluster<32, 2>(dev); break;
    case 64: cap1 = max_cluster<64, 1>(dev); cap2 = max_cluster<64, 2>(dev); break;
    default: cap1 = max_cluster<128, 1>(dev); break;
  }
  if (cap1 <= 0 || (bnp < 128 && cap2 <= 0)) return DG_ERR_CUDA;
  // 128-token tiles on CTA pairs (DG_DECODE_PAIR=0|1; read on every call)
  bool pair = false;
  if (bnp == 128)
    if (const char* e = std::getenv("DG_DECODE_PAIR")) pair = std::atoi(e) != 0;
  if (pair) {
    const int pc = max_cluster<128, 1, true>(dev);
    if (pc < 2) return DG_ERR_CUDA;
    cap1 = pc / 2;  // split count of a cluster of pairs
  }
  DecodePlan p = plan_decode(bnp, m_tiles, n_tiles, KB, sms, cap1, cap2);
  // DG_DECODE_MINB=1|2 and DG_DECODE_SPLITS=s force the plan (comparisons;
  // splits clamped to the cluster limit and to one K-block per split; 128
  // tokens always take the whole SM); read on every call
  if (const char* e = std::getenv("DG_DECODE_MINB")) {
    const int f = std::atoi(e);
    if (f == 1 || f == 2) p.minb = f;
  }
  if (bnp == 128) p.minb = 1;
  const int cap = p.minb == 1 ? cap1 : cap2;
  p.splits = std::max(1, std::min(p.splits, std::min(cap, 8)));
  if (const char* e = std::getenv("DG_DECODE_SPLITS")) {
    const int f = std::atoi(e);
    if (f >= 1) p.splits = std::max(1, std::min(std::min(f, std::min(cap, 8)), KB));
  }
  // with one CTA per SM a cluster needs `splits` whole SMs of one GPC, and
  // some sizes (e.g. 7) leave SMs of every GPC idle: lower the split count
  // until all clusters are resident at once (two CTAs per SM pack freely)
  const bool fit = std::getenv("DG_DECODE_SPLITS") == nullptr && p.minb == 1;
  const int clusters = (pair ? (n_tiles + 1) / 2 : n_tiles) * m_tiles;
  // 65..128 tokens: the swap-AB kernel computes 128 weight rows per CTA and
  // K-block, the 128 x 256 tile kernel 256 (its MMA's M side holds the
  // tokens), at about the same per-K-block cadence; the tile kernel has the
  // larger fixed cost, more so with a split-K exchange. Estimates in us,
  // fitted to B200 timings of back-to-back launches of the decode shapes
  // (within ~10%): decode 5.0 + 0.58 x waves x K-blocks per CTA; tiles, per
  // wave, 8.5 + 0.58 x (K-blocks per part - 4) + 5.6 with a split. Forced
  // decode plans keep the decode kernel.
  if (bnp == 128 && !pair && small_m_tiles_env() != 0 && std::getenv("DG_DECODE_SPLITS") == nullptr &&
      std::getenv("DG_DECODE_MINB") == nullptr) {
    const int dsplits = fit ? fit_splits<128, 1>(dev, M, clusters, p.splits) : p.splits;
    const long long dctas = static_cast<long long>(clusters) * dsplits;
    const double t_dec =
        5.0 + 0.58 * static_cast<double>((dctas + sms - 1) / sms) * ((KB + dsplits - 1) / dsplits);
    const long long tiles = (N + 255) / 256;
    const int k = tiles <= sms ? whole_split_k(tiles, KB, sms, dev) : 1;
    const int kb_part = (KB + k - 1) / k;
    const double t_tiles = static_cast<double>((tiles + sms - 1) / sms) *
                           (8.5 + 0.58 * std::max(0, kb_part - 4) + (k > 1 ? 5.6 : 0.0));
    if (t_tiles < t_dec)
      return run_nt<dg::MODE_DENSE>(A, sfa, (M + 3) / 4 * 4, B, sfb, nullptr, nullptr, C, D, M, M,
                                    N, K, 1, 1, 1, st, "fp8_gemm_nt", -1, true);
  }
  if (pair)
    return run_decode<128, 1, true>(A, sfa, B, sfb, C, D, M, N, K,
                                    fit ? fit_splits<128, 1, true>(dev, M, clusters, p.splits)
                                        : p.splits,
                                    st);
#define DG_RUN_DECODE(BNP_, MINB_)                                                         \
  return run_decode<BNP_, MINB_>(A, sfa, B, sfb, C, D, M, N, K,                            \
                                 fit ? fit_splits<BNP_, MINB_>(dev, M, clusters, p.splits) : p.splits, st)
  switch (bnp) {
    case 16:
      if (p.minb == 1) DG_RUN_DECODE(16, 1);
      DG_RUN_DECODE(16, 2);
    case 32:
      if (p.minb == 1) DG_RUN_DECODE(32, 1);
      DG_RUN_DECODE(32, 2);
    case 64:
      if (p.minb == 1) DG_RUN_DECODE(64, 1);
      DG_RUN_DECODE(64, 2);
    default:
      DG_RUN_DECODE(128, 1);
  }
#undef DG_RUN_DECODE
}

// Block-scaled small-M launcher (swap-AB, cluster split-K; W4: E2M1 weights).
template <int BNP, int MINB, bool W4>
dg_status run_mx_decode(const void* X, const int32_t* sfx, const void* W, const int32_t* sfw,
                        const void* C, void* D, int M, int N, int K, int splits, cudaStream_t st) {
  using Cfg = dg::MxDecodeCfg<BNP, MINB, W4>;
  const int n_tiles = (N + 127) / 128;
  CUtensorMap tw, tx;
  dg_status s;
  if (W4)
    s = make_map_2d(&tw, W, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, K, N, K / 2, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  else
    s = make_map_2d(&tw, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  if ((s = make_map_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, BNP,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  dg::MxDecodeArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M;
  args.N = N;
  args.K = K;
  args.KB = K / 128;
  args.splits = splits;
  args.rb_w = n_tiles;
  args.sfx = sfx;
  args.sfw = sfw;
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  if (print_configs())
    std::fprintf(stderr,
                 "[dg] %s decode M=%d N=%d K=%d: block-scaled swap-AB BNP=%d (%d CTA/SM), "
                 "n_tiles=%d x split-K %d (cluster), %d stages\n",
                 W4 ? "fp8_fp4_gemm_nt" : "fp8_gemm_nt_ue8m0", M, N, K, BNP, MINB, n_tiles, splits,
                 Cfg::STAGES);
  cudaError_t e = launch(dg::gemm_mx_decode_kernel<BNP, MINB, W4>, dim3(splits, n_tiles, 1),
                         dim3(320), Cfg::SMEM_BYTES, st, splits, tw, tx, args);
  if (e != cudaSuccess) return cuda_fail(e, "block-scaled decode launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

// M <= 128 on the block-scaled path: the decode plan of the promotion path
// (CTAs per SM, split count), DG_DECODE_MINB / DG_DECODE_SPLITS honoured.
template <bool W4>
dg_status dispatch_mx_decode(const void* X, const int32_t* sfx, const void* W,
                             const int32_t* sfw, const void* C, void* D, int M, int N, int K,
                             cudaStream_t st) {
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  const int KB = K / 128;
  const int n_tiles = (N + 127) / 128;
  const int bnp = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  int cap1 = 0, cap2 = 0;
  switch (bnp) {
    case 16: cap1 = max_cluster_mx<16, 1, W4>(dev); cap2 = max_cluster_mx<16, 2, W4>(dev); break;
    case 32: cap1 = max_cluster_mx<32, 1, W4>(dev); cap2 = max_cluster_mx<32, 2, W4>(dev); break;
    case 64: cap1 = max_cluster_mx<64, 1, W4>(dev); cap2 = max_cluster_mx<64, 2, W4>(dev); break;
    default: cap1 = max_cluster_mx<128, 1, W4>(dev); cap2 = max_cluster_mx<128, 2, W4>(dev); break;
  }
  if (cap1 <= 0 || cap2 <= 0) return DG_ERR_CUDA;
  DecodePlan p = plan_mx_decode(M, n_tiles, KB, sms, cap1, cap2);
  if (W4 && n_tiles < sms) {
    // E2M1 weights (from a sweep of both configurations x 1..8 splits over
    // the decode shapes): two CTAs per SM at every M, and a split keeps at
    // least 8 K-blocks -- half the weight bytes per K-block leave a split with
    // fewer K-blocks too little to stream.
    p.minb = 2;
    p.splits = std::max(1, std::min(std::min(2 * sms / n_tiles, KB / 8), std::min(4, cap2)));
  }
  if (const char* e = std::getenv("DG_DECODE_MINB")) {
    const int f = std::atoi(e);
    if (f == 1 || f == 2) p.minb = f;
  }
  const int cap = p.minb == 1 ? cap1 : cap2;
  p.splits = std::min(p.splits, std::min(cap, 8));
  if (const char* e = std::getenv("DG_DECODE_SPLITS")) {
    const int f = std::atoi(e);
    if (f >= 1) p.splits = std::max(1, std::min(std::min(f, std::min(cap, 8)), KB));
  }
#define DG_RUN_MX_DECODE(BNP_)                                                                  \
  return p.minb == 1                                                                            \
             ? run_mx_decode<BNP_, 1, W4>(X, sfx, W, sfw, C, D, M, N, K, p.splits, st)       \
             : run_mx_decode<BNP_, 2, W4>(X, sfx, W, sfw, C, D, M, N, K, p.splits, st)
  switch (bnp) {
    case 16: DG_RUN_MX_DECODE(16);
    case 32: DG_RUN_MX_DECODE(32);
    case 64: DG_RUN_MX_DECODE(64);
    default: DG_RUN_MX_DECODE(128);
  }
#undef DG_RUN_MX_DECODE
}

// K-grouped TN launcher. Sizes come either from the host (`ks`, sumK their
// total) or from device memory (`ks_dev`, sumK = the K rows the operands
// hold); the kernel builds the per-group K-block ranges itself in the latter
// case.
dg_status run_k_grouped(const void* A, const float* sfa, const void* B, const float* sfb,
                        const int* ks, const int32_t* ks_dev, long long sumK, const float* C,
                        float* D, int G, int M, int N, void* stream) {
  if (M == 0 || N == 0) return DG_OK;
  if (!D) return DG_ERR_INVALID_ARG;
  if (!aligned16(D) || (C && !aligned16(C))) return DG_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sumK == 0) return copy_or_zero<float>(C, D, static_cast<long long>(G) * M * N, sms, st);
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb))
    return DG_ERR_MISALIGNED;
  const int mb = (M + 127) / 128;
  const int bn = choose_bn(static_cast<long long>(G) * mb, N, sms);
  const uint64_t sumKB = static_cast<uint64_t>(sumK / 128);
  CUtensorMap ta, tb, tsa, tsb;
  if ((s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, M, sumK, M, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if ((s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, sumK, N, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if ((s = make_map_2d(&tsa, sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, sumKB, 4ull * M, 128, 1,
                       CU_TENSOR_MAP_SWIZZLE_NONE)) != DG_OK)
    return s;
  if ((s = make_map_2d(&tsb, sfb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, sumKB, 4ull * N, bn, 1,
                       CU_TENSOR_MAP_SWIZZLE_NONE)) != DG_OK)
    return s;
  CUtensorMap td;  // D as [G*M][N] fp32; 16x32 boxes, 64-byte swizzle
  if ((s = make_map_2d(&td, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, static_cast<uint64_t>(G) * M,
                       4ull * N, 16, 32, CU_TENSOR_MAP_SWIZZLE_64B)) != DG_OK)
    return s;
  GemmArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M;
  args.N = N;
  args.K = 0;
  args.G = G;
  args.d_rows = static_cast<long long>(G) * M;
  args.num_m_blocks = mb;
  args.num_n_blocks = (N + bn - 1) / bn;
  const long long tiles = static_cast<long long>(G) * mb * args.num_n_blocks;
  args.total_tiles = static_cast<int>(tiles);
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  if (ks) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      args.kb_off[g] = acc;
      acc += ks[g] / 128;
    }
    args.kb_off[G] = acc;
  } else {
    args.ks_dev = ks_dev;
    args.kb_cap = static_cast<int>(sumKB);
  }
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(sms, tiles)));
  if (print_configs())
    std::fprintf(stderr,
                 "[dg] k_grouped_fp8_gemm_tn M=%d N=%d %s=%lld G=%d: BN=%d tiles=%lld grid=%d\n",
                 M, N, ks ? "sumK" : "K capacity (sizes on device)", sumK, G, bn, tiles, grid);
  if (bn == 256)
    return launch_gemm<dg::MODE_KGROUPED, 256>(ta, tb, tsa, tsb, td, args, grid, st, dev);
  return launch_gemm<dg::MODE_KGROUPED, 128>(ta, tb, tsa, tsb, td, args, grid, st, dev);
}

// UE8M0 block-scaled dense GEMM launcher (one CTA per SM, persistent).
// FP4B: B is packed E2M1 [N][K/2], loaded by the 4-bit TMA type that spreads
// each 8 packed bytes over a 16-byte shared-memory cell.
template <bool FP4B>
dg_status run_mx(const void* A, const int32_t* sfa, const void* B, const int32_t* sfb,
                 const void* C, void* D, int M, int N, int K, cudaStream_t st) {
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  using Cfg = dg::MxCfgT<FP4B>;
  CUtensorMap ta, tb, td;
  if ((s = make_map_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
    return s;
  if (FP4B)
    s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, K, N, K / 2, 128, Cfg::BN,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  else
    s = make_map_2d(&tb, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, 128, Cfg::BN,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != DG_OK) return s;
  if ((s = make_map_2d(&td, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, 2ull * N, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_64B)) != DG_OK)
    return s;
  dg::MxArgs args;
  std::memset(&args, 0, sizeof args);
  args.M = M;
  args.N = N;
  args.K = K;
  args.num_m_blocks = (M + 127) / 128;
  args.num_n_blocks = (N + Cfg::BN - 1) / Cfg::BN;
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  if (tiles > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
  args.total_tiles = static_cast<int>(tiles);
  args.rb_a = (M + 127) / 128;
  args.rb_b = (N + 127) / 128;
  args.sfa = sfa;
  args.sfb = sfb;
  args.C = C;
  args.D = D;
  args.timeout_ns = timeout_ns();
  args.drop_arrive = take_drop_flag();
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(sms, tiles)));
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(dg::gemm_mx_kernel<FP4B>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err[dev] != cudaSuccess) return cuda_fail(attr_err[dev], "cudaFuncSetAttribute");
  if (print_configs())
    std::fprintf(stderr, "[dg] %s M=%d N=%d K=%d: 128x256 block-scaled tiles=%lld grid=%d\n",
                 FP4B ? "fp8_fp4_gemm_nt" : "fp8_gemm_nt_ue8m0", M, N, K, tiles, grid);
  cudaError_t e = launch(dg::gemm_mx_kernel<FP4B>, dim3(grid), dim3(320), Cfg::SMEM_BYTES, st, 1,
                         ta, tb, td, args);
  if (e != cudaSuccess) return cuda_fail(e, "mx gemm launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

}  // namespace

// =============================================================== C ABI
extern "C" {

const char* dg_status_string(dg_status s) {
  switch (s) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED_SHAPE: return "DG_ERR_UNSUPPORTED_SHAPE";
    case DG_ERR_MISALIGNED: return "DG_ERR_MISALIGNED";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
  }
  return "DG_ERR_UNKNOWN";
}

int dg_get_mk_alignment_for_contiguous_layout(void) { return 128; }

int dg_get_tma_aligned_size(int mn, int elem_bytes) {
  if (mn < 0 || elem_bytes <= 0 || 16 % elem_bytes != 0) return -1;
  const int a = 16 / elem_bytes;
  return (mn + a - 1) / a * a;
}

void dg_set_num_sms(int n) { g_num_sms_cap.store(n > 0 ? n : 0); }

int dg_get_num_sms(void) {
  int dev = 0, sms = 0;
  if (device_sms(&dev, &sms) != DG_OK) return g_num_sms_cap.load();
  return sms;
}

void dg_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns); }

void dg_set_pdl(int enable) { g_pdl.store(enable ? 1 : 0); }

int dg_get_pdl(void) { return g_pdl.load(); }

void dg_debug_drop_next_arrive(int enable) { g_drop_next.store(enable ? 1 : 0); }

uint64_t dg_get_launch_count(void) { return g_launches.load(); }

dg_status dg_get_last_device_error(void* stream, int* site) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int w[2] = {0, 0};
  e = cudaMemcpyFromSymbol(w, dg::g_error_word, sizeof w);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  const unsigned int z[2] = {0, 0};
  e = cudaMemcpyToSymbol(dg::g_error_word, z, sizeof z);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  if (site) *site = static_cast<int>(w[1]);
  if (w[0] == 0) return DG_OK;
  if (w[0] == static_cast<unsigned int>(DG_ERR_TIMEOUT)) return DG_ERR_TIMEOUT;
  if (w[0] == static_cast<unsigned int>(DG_ERR_INVALID_ARG)) return DG_ERR_INVALID_ARG;
  return DG_ERR_CUDA;
}

dg_status dg_quantize_fp8(const void* x, int in_dtype, int batch, int rows, int cols, int mode,
                          void* codes, float* scales, int ld_scales, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return DG_ERR_INVALID_ARG;
  if (in_dtype != DG_IN_F32 && in_dtype != DG_IN_BF16) return DG_ERR_INVALID_ARG;
  if (mode < DG_QUANT_ROW_1x128 || mode > DG_QUANT_COL_128x1) return DG_ERR_INVALID_ARG;
  if (mode == DG_QUANT_ROW_1x128) {
    if (cols % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  } else if (mode == DG_QUANT_BLOCK_128x128) {
    if (cols % 4 != 0) return DG_ERR_UNSUPPORTED_SHAPE;  // a lane's 4 columns
  } else {
    if (rows % 128 != 0 || cols % 4 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  }
  if (mode == DG_QUANT_ROW_1x128 && (ld_scales < rows || ld_scales % 4 != 0))
    return DG_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * rows * cols == 0) return DG_OK;
  if (!x || !codes || !scales) return DG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return DG_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* q = static_cast<uint8_t*>(codes);
  const bool bf = in_dtype == DG_IN_BF16;
  cudaError_t e = cudaSuccess;
  if (mode == DG_QUANT_ROW_1x128) {
    const long long strips = static_cast<long long>(batch) * rows * (cols / 128);
    if (strips >= 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
    const int grid = static_cast<int>(std::min<long long>((strips + 31) / 32, 8ll * sms));
    uint8_t* none = nullptr;
    e = bf ? launch(dg::quant_row_kernel<true>, dim3(grid), dim3(256), 0, st, 1, x, batch, rows,
                    cols, q, scales, ld_scales, none)
           : launch(dg::quant_row_kernel<false>, dim3(grid), dim3(256), 0, st, 1, x, batch, rows,
                    cols, q, scales, ld_scales, none);
  } else if (mode == DG_QUANT_BLOCK_128x128) {
    const long long blocks =
        static_cast<long long>(batch) * ((rows + 127) / 128) * ((cols + 127) / 128);
    if (blocks > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
    uint8_t* none = nullptr;
    e = bf ? launch(dg::quant_block_kernel<true>, dim3(static_cast<int>(blocks)), dim3(256), 0, st,
                    1, x, batch, rows, cols, q, scales, none)
           : launch(dg::quant_block_kernel<false>, dim3(static_cast<int>(blocks)), dim3(256), 0, st,
                    1, x, batch, rows, cols, q, scales, none);
  } else {
    const long long blocks = static_cast<long long>(batch) * (rows / 128) * ((cols + 63) / 64);
    if (blocks > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
    e = bf ? launch(dg::quant_col_kernel<true>, dim3(static_cast<int>(blocks)), dim3(256), 0, st, 1,
                    x, batch, rows, cols, q, scales)
           : launch(dg::quant_col_kernel<false>, dim3(static_cast<int>(blocks)), dim3(256), 0, st, 1,
                    x, batch, rows, cols, q, scales);
  }
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

dg_status dg_quantize_fp8_ue8m0(const void* x, int in_dtype, int rows, int cols, int mode,
                                void* codes, float* scales, int ld_scales, int32_t* packed,
                                void* stream) {
  if (rows < 0 || cols < 0) return DG_ERR_INVALID_ARG;
  if (in_dtype != DG_IN_F32 && in_dtype != DG_IN_BF16) return DG_ERR_INVALID_ARG;
  if (mode != DG_QUANT_ROW_1x128 && mode != DG_QUANT_BLOCK_128x128) return DG_ERR_INVALID_ARG;
  if (cols % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (mode == DG_QUANT_ROW_1x128 && scales && (ld_scales < rows || ld_scales % 4 != 0))
    return DG_ERR_INVALID_ARG;
  if (static_cast<long long>(rows) * cols == 0) return DG_OK;
  if (!x || !codes || !packed) return DG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(packed) || (scales && !aligned16(scales)))
    return DG_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* q = static_cast<uint8_t*>(codes);
  uint8_t* pk = reinterpret_cast<uint8_t*>(packed);
  const bool bf = in_dtype == DG_IN_BF16;
  cudaError_t e;
  if (mode == DG_QUANT_ROW_1x128) {
    const long long strips = static_cast<long long>(rows) * (cols / 128);
    if (strips >= 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
    const int grid = static_cast<int>(std::min<long long>((strips + 31) / 32, 8ll * sms));
    e = bf ? launch(dg::quant_row_kernel<true, true>, dim3(grid), dim3(256), 0, st, 1, x, 1, rows,
                    cols, q, scales, ld_scales, pk)
           : launch(dg::quant_row_kernel<false, true>, dim3(grid), dim3(256), 0, st, 1, x, 1, rows,
                    cols, q, scales, ld_scales, pk);
  } else {
    const long long blocks = static_cast<long long>((rows + 127) / 128) * (cols / 128);
    if (blocks > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
    e = bf ? launch(dg::quant_block_kernel<true, true>, dim3(static_cast<int>(blocks)), dim3(256),
                    0, st, 1, x, 1, rows, cols, q, scales, pk)
           : launch(dg::quant_block_kernel<false, true>, dim3(static_cast<int>(blocks)), dim3(256),
                    0, st, 1, x, 1, rows, cols, q, scales, pk);
  }
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

dg_status dg_fp8_gemm_nt_ue8m0(const void* A, const int32_t* sfa, const void* B,
                               const int32_t* sfb, const void* C, void* D, int M, int N, int K,
                               void* stream) {
  if (M < 0 || N < 0 || K < 0) return DG_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return DG_OK;
  if (!D) return DG_ERR_INVALID_ARG;
  if (!aligned16(D) || (C && !aligned16(C))) return DG_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {
    int dev = 0, sms = 0;
    dg_status s = device_sms(&dev, &sms);
    if (s != DG_OK) return s;
    return copy_or_zero<Bf16Raw>(C, D, static_cast<long long>(M) * N, sms, st);
  }
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb))
    return DG_ERR_MISALIGNED;
  if (M <= 128) return dispatch_mx_decode<false>(A, sfa, B, sfb, C, D, M, N, K, st);
  return run_mx<false>(A, sfa, B, sfb, C, D, M, N, K, st);
}

dg_status dg_quantize_fp4_e2m1(const void* x, int in_dtype, int rows, int cols, void* codes,
                               float* scales, int32_t* packed, void* stream) {
  if (rows < 0 || cols < 0) return DG_ERR_INVALID_ARG;
  if (in_dtype != DG_IN_F32 && in_dtype != DG_IN_BF16) return DG_ERR_INVALID_ARG;
  if (cols % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(rows) * cols == 0) return DG_OK;
  if (!x || !codes || !packed) return DG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(packed) || (scales && !aligned16(scales)))
    return DG_ERR_MISALIGNED;
  const long long strips = static_cast<long long>(rows) * (cols / 128);
  if (strips >= 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
  int dev = 0, sms = 0;
  dg_status s = device_sms(&dev, &sms);
  if (s != DG_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* q = static_cast<uint8_t*>(codes);
  uint8_t* pk = reinterpret_cast<uint8_t*>(packed);
  const int grid = static_cast<int>(std::min<long long>((strips + 63) / 64, 8ll * sms));
  cudaError_t e =
      in_dtype == DG_IN_BF16
          ? launch(dg::quant_fp4_kernel<true>, dim3(grid), dim3(256), 0, st, 1, x, rows, cols, q,
                   scales, pk)
          : launch(dg::quant_fp4_kernel<false>, dim3(grid), dim3(256), 0, st, 1, x, rows, cols, q,
                   scales, pk);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  g_launches.fetch_add(1);
  return DG_OK;
}

dg_status dg_fp8_fp4_gemm_nt(const void* A, const int32_t* sfa, const void* B,
                             const int32_t* sfb, const void* C, void* D, int M, int N, int K,
                             void* stream) {
  if (M < 0 || N < 0 || K < 0) return DG_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return DG_OK;
  if (!D) return DG_ERR_INVALID_ARG;
  if (!aligned16(D) || (C && !aligned16(C))) return DG_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {
    int dev = 0, sms = 0;
    dg_status s = device_sms(&dev, &sms);
    if (s != DG_OK) return s;
    return copy_or_zero<Bf16Raw>(C, D, static_cast<long long>(M) * N, sms, st);
  }
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || reinterpret_cast<uintptr_t>(B) % 32 != 0 || !aligned16(sfa) ||
      !aligned16(sfb))
    return DG_ERR_MISALIGNED;
  if (M <= 128) return dispatch_mx_decode<true>(A, sfa, B, sfb, C, D, M, N, K, st);
  return run_mx<true>(A, sfa, B, sfb, C, D, M, N, K, st);
}

dg_status dg_fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream) {
  if (M < 0 || N < 0 || K < 0) return DG_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return DG_OK;
  if (!D) return DG_ERR_INVALID_ARG;
  if (!aligned16(D) || (C && !aligned16(C))) return DG_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (K == 0) {
    int dev = 0, sms = 0;
    dg_status s = device_sms(&dev, &sms);
    if (s != DG_OK) return s;
    return copy_or_zero<Bf16Raw>(C, D, static_cast<long long>(M) * N, sms, st);
  }
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb))
    return DG_ERR_MISALIGNED;
  const int ld = (M + 3) / 4 * 4;
  const long long mb = (M + 127) / 128;
  if (M <= 128) {
    if (small_m_tiles_env() == 1)
      return run_nt<dg::MODE_DENSE>(A, sfa, ld, B, sfb, nullptr, nullptr, C, D, M, M, N, K, 1, mb,
                                    mb, st, "fp8_gemm_nt", -1, true);
    int dev = 0, sms = 0;
    dg_status s = device_sms(&dev, &sms);
    if (s != DG_OK) return s;
    return dispatch_decode(A, sfa, B, sfb, C, D, M, N, K, sms, dev, st);
  }
  if (use_pairs()) return run_pair(A, sfa, ld, B, sfb, C, D, M, N, K, st);
  return run_nt<dg::MODE_DENSE>(A, sfa, ld, B, sfb, nullptr, nullptr, C, D, M, M, N, K, 1, mb, mb,
                                st, "fp8_gemm_nt");
}

dg_status dg_fp8_gemm_nn(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream) {
  return dense_layout_entry<dg::MODE_NN>(A, sfa, B, sfb, C, D, M, N, K, stream, "fp8_gemm_nn");
}

dg_status dg_fp8_gemm_tn(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream) {
  return dense_layout_entry<dg::MODE_TN>(A, sfa, B, sfb, C, D, M, N, K, stream, "fp8_gemm_tn");
}

dg_status dg_fp8_gemm_tt(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream) {
  return dense_layout_entry<dg::MODE_TT>(A, sfa, B, sfb, C, D, M, N, K, stream, "fp8_gemm_tt");
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* A, const float* sfa, const void* B,
                                              const float* sfb, const int32_t* m_indices,
                                              const void* C, void* D, int Mt, int N, int K, int G,
                                              void* stream) {
  if (Mt < 0 || N < 0 || K < 0 || G < 1) return DG_ERR_INVALID_ARG;
  if (Mt % 128 != 0 || K % 128 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (Mt == 0 || N == 0) return DG_OK;
  if (!D || !m_indices) return DG_ERR_INVALID_ARG;
  if (K == 0) return DG_ERR_UNSUPPORTED_SHAPE;
  if (!A || !B || !sfa || !sfb) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb) || !aligned16(D) ||
      !aligned16(m_indices) || (C && !aligned16(C)))
    return DG_ERR_MISALIGNED;
  if (static_cast<long long>(G) * N > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
  const long long mb = Mt / 128;
  return run_nt<dg::MODE_CONTIG>(A, sfa, Mt, B, sfb, m_indices, nullptr, C, D, Mt, Mt, N, K, G, mb,
                                 mb, static_cast<cudaStream_t>(stream),
                                 "m_grouped_fp8_gemm_nt_contiguous");
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* A, const float* sfa, const void* B,
                                          const float* sfb, const int32_t* masked_m, void* D,
                                          int G, int max_m, int expected_m, int N, int K,
                                          void* stream) {
  if (G < 1 || max_m < 0 || N < 0 || K < 0) return DG_ERR_INVALID_ARG;
  if (G > dg::kMaxMaskedGroups || K % 128 != 0 || N % 8 != 0 || K == 0)
    return DG_ERR_UNSUPPORTED_SHAPE;
  if (max_m == 0 || N == 0) return DG_OK;
  if (!A || !B || !sfa || !sfb || !masked_m || !D) return DG_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfa) || !aligned16(sfb) || !aligned16(D) ||
      !aligned16(masked_m))
    return DG_ERR_MISALIGNED;
  if (static_cast<long long>(G) * max_m > 0x7fffffffll ||
      static_cast<long long>(G) * N > 0x7fffffffll)
    return DG_ERR_UNSUPPORTED_SHAPE;
  const int ld = (max_m + 3) / 4 * 4;
  const long long mb_bound = static_cast<long long>(G) * ((max_m + 127) / 128);
  const int em = expected_m <= 0 ? max_m : std::min(expected_m, max_m);
  const long long mb_plan = static_cast<long long>(G) * ((em + 127) / 128);
  return run_nt<dg::MODE_MASKED>(A, sfa, ld, B, sfb, nullptr, masked_m, nullptr, D, G * max_m,
                                 max_m, N, K, G, mb_bound, -1, static_cast<cudaStream_t>(stream),
                                 "m_grouped_fp8_gemm_nt_masked", mb_plan);
}

dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* A, const float* sfa, const void* B,
                                              const float* sfb, const int* ks, const float* C,
                                              float* D, int G, int M, int N, void* stream) {
  if (G < 1 || M < 0 || N < 0 || !ks) return DG_ERR_INVALID_ARG;
  if (G > dg::kMaxKGroups || M % 16 != 0 || N % 16 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
  long long sumK = 0;
  for (int g = 0; g < G; ++g) {
    if (ks[g] < 0) return DG_ERR_INVALID_ARG;
    if (ks[g] % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    sumK += ks[g];
  }
  if (sumK > 0x7fffffffll) return DG_ERR_UNSUPPORTED_SHAPE;
  return run_k_grouped(A, sfa, B, sfb, ks, nullptr, sumK, C, D, G, M, N, stream);
}

dg_status dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(const void* A, const float* sfa,
                                                     const void* B, const float* sfb,
                                                     const int32_t* ks_dev, int k_capacity,
                                                     const float* C, float* D, int G, int M, int N,
                                                     void* stream) {
  if (G < 1 || M < 0 || N < 0 || k_capacity < 0) return DG_ERR_INVALID_ARG;
  if (G > dg::kMaxKGroups || M % 16 != 0 || N % 16 != 0 || k_capacity % 128 != 0)
    return DG_ERR_UNSUPPORTED_SHAPE;
  if (k_capacity > 0 && !ks_dev) return DG_ERR_INVALID_ARG;
  if (ks_dev && !aligned4(ks_dev)) return DG_ERR_MISALIGNED;
  return run_k_grouped(A, sfa, B, sfb, nullptr, ks_dev, k_capacity, C, D, G, M, N, stream);
}

}  // extern "C"
