// Per-row FP8 quantisation of the indexer inputs (page "DeepseekV3.2 拆解",
// section "核心组件 / 闪电索引器": the indexer runs in FP8; one scale per row
// of d^I values, scale = amax / 448, amax = 0 -> scale 1).
//
//   codes[r, d] = E4M3(clamp(x[r, d] / scale[r], -448, 448)),  round to
//   nearest even, saturating; scale and x / scale in fp32 (IEEE division).
//
// A warp converts four rows; a lane holds dim / 32 consecutive values of each,
// so a warp reads a row as one contiguous 2·dim-byte segment and writes dim
// bytes. All four rows are loaded before any is converted, to keep enough
// bytes in flight. The kernel is bound by HBM bandwidth: 3 bytes per element.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kQuantWarps = 8;          // warps per CTA
constexpr int kQuantRowsPerWarp = 4;    // rows a warp loads before it converts any
constexpr int kQuantRowsPerCta = kQuantWarps * kQuantRowsPerWarp;

template <int PER>   // values per lane: dim = 32 * PER
__global__ void __launch_bounds__(32 * kQuantWarps)
    quantize_e4m3_rows_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                              float* __restrict__ scales, long long rows) {
  constexpr int DIM = 32 * PER;
  constexpr int NB = PER / 2 > 0 ? PER / 2 : 1;   // 32-bit words of bf16 per lane
  const int lane = threadIdx.x & 31;
  const long long r0 = static_cast<long long>(blockIdx.x) * kQuantRowsPerCta +
                       (threadIdx.x >> 5) * kQuantRowsPerWarp;
  // All of the warp's row loads first (more bytes in flight per warp).
  uint32_t bits[kQuantRowsPerWarp][NB];
#pragma unroll
  for (int k = 0; k < kQuantRowsPerWarp; ++k) {
    const long long r = r0 + k;
    if (r >= rows) continue;
    const uint16_t* xr = x + r * DIM + lane * PER;
    if constexpr (PER == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(xr);
      bits[k][0] = u.x;
      bits[k][1] = u.y;
    } else if constexpr (PER == 2) {
      bits[k][0] = *reinterpret_cast<const uint32_t*>(xr);
    } else {
      bits[k][0] = *xr;
    }
  }
#pragma unroll
  for (int k = 0; k < kQuantRowsPerWarp; ++k) {
    const long long r = r0 + k;
    if (r >= rows) break;   // uniform across the warp
    float v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const uint32_t h = PER == 1 ? bits[k][0] : (bits[k][j / 2] >> (16 * (j & 1))) & 0xffffu;
      v[j] = __uint_as_float(h << 16);   // bf16 is the upper half of an fp32
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < PER; ++j) amax = fmaxf(amax, fabsf(v[j]));
    // non-negative floats order like their bit patterns
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const float y = fminf(448.f, fmaxf(-448.f, __fdiv_rn(v[j], scale)));
      const uint32_t c =
          static_cast<uint32_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
      packed |= c << (8 * j);
    }
    uint8_t* cr = codes + r * DIM + lane * PER;
    if constexpr (PER == 4) {
      *reinterpret_cast<uint32_t*>(cr) = packed;
    } else if constexpr (PER == 2) {
      *reinterpret_cast<uint16_t*>(cr) = static_cast<uint16_t>(packed);
    } else {
      *cr = static_cast<uint8_t>(packed);
    }
    if (lane == 0) scales[r] = scale;
  }
}

}  // namespace dsa
