// quant.cuh -- BF16/FP32 -> E4M3 quantisers with FP32 scales, sm_100a.
//
// scale = max(amax, 1e-4f) / 448 (IEEE division) and
// code = E4M3_RN_satfinite(x / scale) with the quotient rounded exactly as the
// IEEE division would round it (see quotient()); this file must not be built
// with --use_fast_math. Three scale granularities:
//   ROW   one scale per (row, 128-column strip), stored transposed [cols/128][ld]
//   BLOCK one scale per 128x128 block, [ceil(rows/128)][ceil(cols/128)]
//   COL   one scale per (128-row strip, column), [rows/128][cols]
// All three are single-pass, HBM-bound kernels: every input byte is read once,
// every code and scale written once.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace dg {

struct In4 {
  float v[4];
};

template <bool BF16>
__device__ __forceinline__ In4 load4(const void* x, int64_t i) {
  In4 r;
  if constexpr (BF16) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(x) + i));
    r.v[0] = __uint_as_float(u.x << 16);
    r.v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    r.v[2] = __uint_as_float(u.y << 16);
    r.v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  } else {
    const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + i));
    r.v[0] = f.x;
    r.v[1] = f.y;
    r.v[2] = f.z;
    r.v[3] = f.w;
  }
  return r;
}

// x / s rounded to nearest (the IEEE quotient), from r = 1/s correctly rounded
// and one FMA correction step (Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990: if r is
// 1/s within half an ulp and q0 is within one ulp of x/s, q0 + r*(x - s*q0)
// rounds to the correctly rounded quotient). The residual is exact unless
// |x| < 2^-103; with s >= 1e-4/448 such quotients are below 2^-81 and encode
// to a signed zero either way, so the E4M3 code always equals that of the
// IEEE division. The sign is taken from x so that -0 / s = -0.
__device__ __forceinline__ float quotient(float x, float s, float r) {
  const float ax = fabsf(x);
  const float q0 = __fmul_rn(ax, r);
  const float e = fmaf(-q0, s, ax);
  return copysignf(fmaf(e, r, q0), x);
}

// max(amax, 1e-4f) / 448 rounded exactly as the IEEE division (same method:
// the dividend is >= 1e-4, far from underflow).
__device__ __forceinline__ float scale_from_amax(float amax) {
  constexpr float kInv448 = 1.0f / 448.0f;  // correctly rounded at compile time
  return quotient(fmaxf(amax, 1e-4f), 448.0f, kInv448);
}

// Power-of-two scale for the UE8M0 variant: s = 2^e with e = ceil(log2 t),
// t = max(amax, 1e-4f) / 448 (the FP32 mode's quotient, rounded up to the
// next power of two so that no code saturates). t is normal (>= 2^-22), so e
// is its exponent, plus one unless its mantissa is zero. Returns e.
__device__ __forceinline__ int pow2_exponent(float amax) {
  const uint32_t b = __float_as_uint(scale_from_amax(amax));
  const int e = static_cast<int>((b >> 23) & 0xFFu) - 127;
  return (b & 0x7FFFFFu) ? e + 1 : e;
}

// 2^e as a float, for -126 <= e <= 127.
__device__ __forceinline__ float exp2_exact(int e) {
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// Byte offset of (row, K-block) in the packed UE8M0 layout
// [ceil(K/512)][ceil(R/128)][32][4] int32 (byte b of word [q][rb][i][j] is row
// 128 rb + 32 j + i, K-block 4 q + b).
__device__ __forceinline__ long long packed_offset(int row, int kb, int rblocks) {
  const long long word =
      ((static_cast<long long>(kb >> 2) * rblocks + (row >> 7)) * 32 + (row & 31)) * 4 +
      ((row >> 5) & 3);
  return word * 4 + (kb & 3);
}

// Four E4M3 codes packed little-endian (element 0 in the low byte).
__device__ __forceinline__ uint32_t encode4(const float (&v)[4], float s, float r) {
  const float y0 = quotient(v[0], s, r), y1 = quotient(v[1], s, r);
  const float y2 = quotient(v[2], s, r), y3 = quotient(v[3], s, r);
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(y2, y3), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 16 consecutive inputs starting at element i (i a multiple of 16).
template <bool BF16>
__device__ __forceinline__ void load16(const void* x, int64_t i, float (&v)[16]) {
  if constexpr (BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + i);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = __ldg(p + h);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[h * 8 + 2 * k] = __uint_as_float(w[k] << 16);
        v[h * 8 + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + i);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 f = __ldg(p + h);
      v[4 * h] = f.x;
      v[4 * h + 1] = f.y;
      v[4 * h + 2] = f.z;
      v[4 * h + 3] = f.w;
    }
  }
}

// ROW_1x128: strips enumerated (batch, row, strip) with the strip index
// fastest, so strip s covers elements [128 s, 128 s + 128) of x. Eight lanes
// share a strip, each holding 16 consecutive values (the strip's amax takes 3
// shuffles, its 128 codes go out as 8 x 16-byte stores); a warp covers 4
// strips per round and keeps 2 rounds (8 strips, 4 KB of FP32 input) in
// flight. Requires batch * rows * (cols/128) < 2^31.
// POW2: power-of-two scales (see pow2_exponent); the UE8M0 bytes also go to
// `packed` (batch 1) and `scales` may be null.
template <bool BF16, bool POW2 = false>
__global__ void __launch_bounds__(256) quant_row_kernel(const void* __restrict__ x, int batch,
                                                        int rows, int cols,
                                                        uint8_t* __restrict__ codes,
                                                        float* __restrict__ scales, int ld,
                                                        uint8_t* __restrict__ packed) {
  constexpr int U = 2;  // rounds of 4 strips in flight per warp
  pdl_trigger();  // the next launch's PDL wait still waits for this grid
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int g = lane >> 3;   // strip of this lane within a round
  const int li = lane & 7;   // 16-value slice of the strip
  const uint32_t kbs = static_cast<uint32_t>(cols) >> 7;
  const uint32_t nstrips = static_cast<uint32_t>(batch) * static_cast<uint32_t>(rows) * kbs;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  for (uint32_t s0 = warp0 * (4 * U); s0 < nstrips; s0 += nwarps * (4 * U)) {
    float v[U][16];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t st = s0 + 4 * u + g;
      if (st < nstrips) {
        load16<BF16>(x, static_cast<int64_t>(st) * 128 + li * 16, v[u]);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[u][k] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t st = s0 + 4 * u + g;
      float amax = 0.0f;
#pragma unroll
      for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[u][k]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      float sc, rc;
      int e = 0;
      if constexpr (POW2) {
        e = pow2_exponent(amax);
        sc = exp2_exact(e);
        rc = exp2_exact(-e);  // exact: the quotient below is then x * 2^-e
      } else {
        sc = scale_from_amax(amax);
        rc = __frcp_rn(sc);
      }
      if (st < nstrips) {
        uint4 o;
        o.x = encode4(*reinterpret_cast<const float(*)[4]>(&v[u][0]), sc, rc);
        o.y = encode4(*reinterpret_cast<const float(*)[4]>(&v[u][4]), sc, rc);
        o.z = encode4(*reinterpret_cast<const float(*)[4]>(&v[u][8]), sc, rc);
        o.w = encode4(*reinterpret_cast<const float(*)[4]>(&v[u][12]), sc, rc);
        *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(st) * 128 + li * 16) = o;
        if (li == 0) {
          const uint32_t br = st / kbs;  // batch * rows + row
          const uint32_t kb = st - br * kbs;
          const uint32_t b = br / static_cast<uint32_t>(rows);
          const uint32_t r = br - b * static_cast<uint32_t>(rows);
          if (!POW2 || scales) scales[(static_cast<int64_t>(b) * kbs + kb) * ld + r] = sc;
          if constexpr (POW2)
            packed[packed_offset(static_cast<int>(r), static_cast<int>(kb), (rows + 127) >> 7)] =
                static_cast<uint8_t>(e + 127);
        }
      }
    }
  }
}

// BLOCK_128x128: one 256-thread CTA per 128x128 block; warp w holds rows
// [16w, 16w+16) of the block, lane l columns [4l, 4l+4). Blocks at the
// bottom and right edges hold only the rows and columns that exist
// (cols % 4 == 0, so a lane's four columns are all in or all out).
// POW2: power-of-two scales; the block's UE8M0 byte is written for all 128
// rows of the block into `packed` (batch 1), and `scales` may be null.
template <bool BF16, bool POW2 = false>
__global__ void __launch_bounds__(256, 2) quant_block_kernel(const void* __restrict__ x, int batch,
                                                          int rows, int cols,
                                                          uint8_t* __restrict__ codes,
                                                          float* __restrict__ scales,
                                                          uint8_t* __restrict__ packed) {
  __shared__ float red[8];
  pdl_trigger();  // the next launch's PDL wait still waits for this grid
  pdl_wait();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int kbs = (cols + 127) >> 7, nbs = (rows + 127) >> 7;
  const int64_t blk = blockIdx.x;
  const int kb = static_cast<int>(blk % kbs);
  const int nb = static_cast<int>((blk / kbs) % nbs);
  const int64_t b = blk / (static_cast<int64_t>(kbs) * nbs);
  // rows this lane reads: none where its four columns lie past the right edge
  const int lane_rows = (kb << 7) + (lane << 2) < cols ? rows : 0;
  In4 v[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = (nb << 7) + (w << 4) + i;
    if (r < lane_rows) {
      v[i] = load4<BF16>(x, (b * rows + r) * cols + (kb << 7) + (lane << 2));
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].v[0]), fabsf(v[i].v[1])),
                               fmaxf(fabsf(v[i].v[2]), fabsf(v[i].v[3]))));
    }
  }
  amax = warp_max(amax);
  if (lane == 0) red[w] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
  float sc, rc;
  int e = 0;
  if constexpr (POW2) {
    e = pow2_exponent(a);
    sc = exp2_exact(e);
    rc = exp2_exact(-e);
  } else {
    sc = scale_from_amax(a);
    rc = __frcp_rn(sc);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = (nb << 7) + (w << 4) + i;
    if (r < lane_rows)
      *reinterpret_cast<uint32_t*>(codes + (b * rows + r) * cols + (kb << 7) + (lane << 2)) =
          encode4(v[i].v, sc, rc);
  }
  if (threadIdx.x == 0 && (!POW2 || scales)) scales[(b * nbs + nb) * kbs + kb] = sc;
  if constexpr (POW2) {
    if (threadIdx.x < 128)
      packed[packed_offset((nb << 7) + static_cast<int>(threadIdx.x), kb, nbs)] =
          static_cast<uint8_t>(e + 127);
  }
}

// COL_128x1: one 256-thread CTA per (batch, 128-row strip, 64-column slab);
// thread t holds columns [4(t%16), +4) of rows (t/16) + 16i, i < 8.
template <bool BF16>
__global__ void __launch_bounds__(256) quant_col_kernel(const void* __restrict__ x, int batch,
                                                        int rows, int cols,
                                                        uint8_t* __restrict__ codes,
                                                        float* __restrict__ scales) {
  __shared__ float red[16][64];
  __shared__ float sc_s[64];
  __shared__ float rc_s[64];
  pdl_trigger();  // the next launch's PDL wait still waits for this grid
  pdl_wait();
  const int cg = threadIdx.x & 15, rg = threadIdx.x >> 4;
  const int slabs = (cols + 63) >> 6, rbs = rows >> 7;
  const int64_t blk = blockIdx.x;
  const int slab = static_cast<int>(blk % slabs);
  const int rb = static_cast<int>((blk / slabs) % rbs);
  const int64_t b = blk / (static_cast<int64_t>(slabs) * rbs);
  const int c = (slab << 6) + (cg << 2);
  const bool col_ok = c < cols;
  In4 v[8];
  float m4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = (rb << 7) + rg + (i << 4);
    if (col_ok) {
      v[i] = load4<BF16>(x, (b * rows + r) * cols + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) m4[j] = fmaxf(m4[j], fabsf(v[i].v[j]));
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) red[rg][(cg << 2) + j] = m4[j];
  __syncthreads();
  if (threadIdx.x < 64) {
    float a = red[0][threadIdx.x];
#pragma unroll
    for (int i = 1; i < 16; ++i) a = fmaxf(a, red[i][threadIdx.x]);
    const float sc = scale_from_amax(a);
    sc_s[threadIdx.x] = sc;
    rc_s[threadIdx.x] = __frcp_rn(sc);
    const int cc = (slab << 6) + threadIdx.x;
    if (cc < cols) scales[(b * rbs + rb) * cols + cc] = sc;
  }
  __syncthreads();
  if (!col_ok) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = (rb << 7) + rg + (i << 4);
    const int c0 = cg << 2;
    const float y0 = quotient(v[i].v[0], sc_s[c0 + 0], rc_s[c0 + 0]);
    const float y1 = quotient(v[i].v[1], sc_s[c0 + 1], rc_s[c0 + 1]);
    const float y2 = quotient(v[i].v[2], sc_s[c0 + 2], rc_s[c0 + 2]);
    const float y3 = quotient(v[i].v[3], sc_s[c0 + 3], rc_s[c0 + 3]);
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(y2, y3), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(codes + (b * rows + r) * cols + c) = (lo & 0xFFFFu) | (hi << 16);
  }
}

// ---------------------------------------------------------------- FP4 (E2M1)
// E2M1 (OCP Microscaling Formats v1.0, section 5.3.3): 1 sign bit, 2 exponent
// bits (bias 1), 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. Round
// to nearest, ties to the even code: the thresholds are the midpoints of
// neighbouring magnitudes, strict where the lower neighbour has the even code
// and inclusive where the upper one has; |y| > 6 gives the largest code.
// Two values to E2M1 codes, round to nearest even with saturation to +-6
// (the hardware conversion; a negative value that rounds to zero keeps its
// sign bit): `lo` in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// Exponent e of the FP4 scale 2^e = 2^ceil(log2 t), t = max(amax, 1e-4f) / 6
// rounded exactly as the IEEE division (quotient(); t >= 1.6e-5 is normal).
__device__ __forceinline__ int fp4_exponent(float amax) {
  constexpr float kInv6 = 1.0f / 6.0f;  // correctly rounded at compile time
  const uint32_t b = __float_as_uint(quotient(fmaxf(amax, 1e-4f), 6.0f, kInv6));
  const int e = static_cast<int>((b >> 23) & 0xFFu) - 127;
  return (b & 0x7FFFFFu) ? e + 1 : e;
}

// FP4 quantiser: x [rows][cols] (cols % 128 == 0) -> codes [rows][cols/2]
// (element 2j in the low nibble of byte j), one power-of-two scale per
// (row, 32-column strip): FP32 copies in scales [rows][cols/32] (optional) and
// UE8M0 bytes in `packed` at packed_offset(row, strip), i.e. the block-scaled
// MMA's layout with 32-wide strips in place of K-blocks. Lanes as in
// quant_row_kernel: 8 lanes per 128-column strip, 16 values each, so a lane
// pair holds one 32-wide strip; U rounds of 4 strips in flight per warp.
template <bool BF16>
__global__ void __launch_bounds__(256) quant_fp4_kernel(const void* __restrict__ x, int rows,
                                                        int cols, uint8_t* __restrict__ codes,
                                                        float* __restrict__ scales,
                                                        uint8_t* __restrict__ packed) {
  constexpr int U = 2;
  pdl_trigger();  // the next launch's PDL wait still waits for this grid
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int g = lane >> 3;
  const int li = lane & 7;
  const uint32_t kbs = static_cast<uint32_t>(cols) >> 7;
  const uint32_t nstrips = static_cast<uint32_t>(rows) * kbs;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int rblocks = (rows + 127) >> 7;
  for (uint32_t s0 = warp0 * (4 * U); s0 < nstrips; s0 += nwarps * (4 * U)) {
    float v[U][16];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t st = s0 + 4 * u + g;
      if (st < nstrips) {
        load16<BF16>(x, static_cast<int64_t>(st) * 128 + li * 16, v[u]);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[u][k] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t st = s0 + 4 * u + g;
      float amax = 0.0f;
#pragma unroll
      for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[u][k]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      const int e = fp4_exponent(amax);
      const float rc = exp2_exact(-e);  // x * 2^-e is the exact quotient x / s
      if (st < nstrips) {
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t acc = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            acc |= e2m1x2(v[u][h * 8 + 2 * j] * rc, v[u][h * 8 + 2 * j + 1] * rc) << (8 * j);
          w[h] = acc;
        }
        *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(st) * 64 + li * 8) =
            make_uint2(w[0], w[1]);
        if ((li & 1) == 0) {
          const uint32_t r = st / kbs;
          const uint32_t kb = st - r * kbs;
          const int strip = static_cast<int>(kb) * 4 + (li >> 1);
          if (scales) scales[static_cast<int64_t>(st) * 4 + (li >> 1)] = exp2_exact(e);
          packed[packed_offset(static_cast<int>(r), strip, rblocks)] = static_cast<uint8_t>(e + 127);
        }
      }
    }
  }
}

}  // namespace dg
