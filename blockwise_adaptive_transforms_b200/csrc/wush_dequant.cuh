// Dequantisation of packed 4-bit codes back to fp32 values (the "fake quantisation"
// the layerwise-loss measurements use: paper-graph-ui analysis, section 5, "Metrics"
// and "Per-Layer Quantization Loss (Table 1)").
//
//   MXFP4:  e2m1(code) * 2^(scale - 127)               (exact in fp32)
//   NVFP4:  (e2m1(code) * e4m3(scale)) * s_t            (first product exact, one rounding)
//   INT4:   q * scale, q the two's-complement nibble    (one rounding)
//
// so every value equals the float64 product rounded once to fp32.  HBM-bound
// elementwise work: each thread turns one 32-bit word of codes (8 values) into two
// 16-byte stores; grid-stride loop over a grid sized in multiples of the SM count.
#pragma once
#include <cstdint>

namespace wush {

__device__ __forceinline__ float e2m1_value(uint32_t c) {
  // codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign
  const uint32_t m = c & 7u;
  const float mag = m < 4u ? 0.5f * static_cast<float>(m) : static_cast<float>(m == 4u ? 2 : (m == 5u ? 3 : (m == 6u ? 4 : 6)));
  return (c & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e4m3_decode_value(uint32_t b) {
  // E4M3 (bias 7, no infinities): subnormal for exponent field 0
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  const float mag = e == 0u ? ldexpf(static_cast<float>(m), -9) : ldexpf(static_cast<float>(8u + m), static_cast<int>(e) - 10);
  return (b & 0x80u) ? -mag : mag;
}

template <int FMT>
__global__ void __launch_bounds__(256) wush_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const void* __restrict__ scales,
                                                          const float* __restrict__ tensor_scale, long long rows,
                                                          int d_in, int G, float* __restrict__ out) {
  const int words_per_row = d_in / 8;
  const long long n_words = rows * words_per_row;
  const float s_t = FMT == kNVFP4 ? *tensor_scale : 0.0f;
  const int C = d_in / G;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_words;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / words_per_row;
    const int w = static_cast<int>(i - r * words_per_row);
    const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + r * (d_in / 2) + 4 * w);
    const int blk = (8 * w) / G;
    float s;
    if (FMT == kMXFP4) {
      const uint32_t e = static_cast<const uint8_t*>(scales)[r * C + blk];
      s = __uint_as_float(e == 0u ? 0x00400000u : e << 23);      // 2^(e - 127)
    } else if (FMT == kNVFP4) {
      s = e4m3_decode_value(static_cast<const uint8_t*>(scales)[r * C + blk]);
    } else {
      s = static_cast<const float*>(scales)[r * C + blk];
    }
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t c = (word >> (4 * k)) & 0xFu;
      if (FMT == kINT4) {
        const int q = c >= 8u ? static_cast<int>(c) - 16 : static_cast<int>(c);
        v[k] = __fmul_rn(static_cast<float>(q), s);
      } else if (FMT == kNVFP4) {
        v[k] = __fmul_rn(e2m1_value(c) * s, s_t);               // e2m1 * e4m3 is exact
      } else {
        v[k] = e2m1_value(c) * s;                               // power-of-two scale: exact
      }
    }
    float4* o = reinterpret_cast<float4*>(out + r * d_in + 8 * w);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

}  // namespace wush
