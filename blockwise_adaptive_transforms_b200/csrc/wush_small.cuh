// Decode-sized batches on CUDA cores: the same per-block transform and group
// quantisation as the fused tensor-core kernel (paper-graph-ui analysis, section 3.2
// "Online Activation Transform + Quantize Kernel": per token t and block i,
// y[t, iG + r] = sum_c T_i[r, c] x[t, iG + c], then RTN AbsMax quantisation of the
// group), for batches of a few to ~100 token rows.  There the fused kernel's fixed
// latency (TMA set-up, transform split into bf16 hi/lo panels, MMA pipeline fill) is most
// of the call; here one CTA takes one block i and up to 128 rows, stages T_i (fp32) in
// shared memory, and each thread forms its row's group with fp32 FMAs (sequential over c,
// so y is within a few fp32 ulps of the exact sum) and quantises it with the fused
// kernel's group quantisers.  Rows of the same CTA read T_i as shared-memory broadcasts.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "wush_fused.cuh"

namespace wush {

constexpr int kSmallRows = 128;   // rows (threads) per CTA

// Stages T_i in shared memory and forms this thread's row group y = T_i x (zeros for rows
// past the batch).  Every thread of the CTA must call it (it synchronises the CTA).
template <int G, bool SHARED_T>
__device__ __forceinline__ void small_transform(const __nv_bfloat16* __restrict__ x, const FusedParams& p,
                                                float* Ts, float (&y)[G], bool& valid, long long& row) {
  const int blk = static_cast<int>(blockIdx.x);
  row = static_cast<long long>(blockIdx.y) * kSmallRows + threadIdx.x;
  valid = row < p.n_rows;
  const float4* tg = reinterpret_cast<const float4*>(p.T + (SHARED_T ? 0ll : static_cast<long long>(blk) * G * G));
  for (int k = threadIdx.x; k < G * G / 4; k += kSmallRows) reinterpret_cast<float4*>(Ts)[k] = tg[k];
  __syncthreads();
  if (valid) {
    float xv[G];
    const uint4* xs = reinterpret_cast<const uint4*>(x + row * p.d_in + static_cast<long long>(blk) * G);
#pragma unroll
    for (int k = 0; k < G / 8; ++k) {   // 8 bf16 per 16-byte load; bf16 -> fp32 is exact
      const uint4 u = xs[k];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xv[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
        xv[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int r = 0; r < G; ++r) {
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < G; ++c) acc = __fmaf_rn(Ts[r * G + c], xv[c], acc);
      y[r] = acc;
    }
  } else {
#pragma unroll
    for (int r = 0; r < G; ++r) y[r] = 0.0f;
  }
}

template <int G, int FMT, bool AMAX_ONLY, bool EMIT_Y, bool SHARED_T>
__global__ void __launch_bounds__(kSmallRows)
    wush_small_kernel(const __nv_bfloat16* __restrict__ x, const FusedParams p) {
  __shared__ __align__(16) float Ts[G * G];
  // launched with programmatic stream serialisation: nothing is read before this wait
  grid_dependency_wait();
  grid_launch_dependents();
  const int blk = static_cast<int>(blockIdx.x);
  float y[G];
  bool valid;
  long long row;
  small_transform<G, SHARED_T>(x, p, Ts, y, valid, row);

  if constexpr (AMAX_ONLY) {
    float m = group_absmax<G>(y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(p.amax_word, __float_as_uint(m));
    return;
  }
  if (!valid) return;
  if (EMIT_Y) {
    float4* yd = reinterpret_cast<float4*>(p.y_out + row * p.d_in + static_cast<long long>(blk) * G);
#pragma unroll
    for (int k = 0; k < G / 4; ++k) yd[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
  }
  uint32_t words[G / 8];
  uint8_t* cdst = p.codes + row * (p.d_in / 2) + static_cast<long long>(blk) * (G / 2);
  // one-byte scales go row-major or, for the block-scaled GEMM, to the scale-atom layout:
  // row 128 r + i + 32 j, column 4 c + k at byte (r * atom_cols + c) * 512 + 16 i + 4 j + k
  uint8_t* sdst = static_cast<uint8_t*>(p.scales) + row * p.C + blk;
  if (FMT != kINT4 && p.scale_atoms) {
    const int rr = static_cast<int>(row & 127);
    sdst = static_cast<uint8_t*>(p.scales) + ((row >> 7) * p.atom_cols + (blk >> 2)) * 512 + (rr & 31) * 16 +
           (rr >> 5) * 4 + (blk & 3);
  }
  if constexpr (FMT == kMXFP4) {
    *sdst = static_cast<uint8_t>(quant_mx<G>(y, words));
  } else if constexpr (FMT == kNVFP4) {
    const float s_t = *p.tensor_scale;
    *sdst = static_cast<uint8_t>(quant_nv<G>(y, s_t, __fmul_rn(6.0f, s_t), words));
  } else {
    static_cast<float*>(p.scales)[row * p.C + blk] = quant_int4<G>(y, words);
  }
  if constexpr (G == 32) *reinterpret_cast<uint4*>(cdst) = make_uint4(words[0], words[1], words[2], words[3]);
  else *reinterpret_cast<uint2*>(cdst) = make_uint2(words[0], words[1]);
}

// NVFP4 in one launch for decode-sized batches.  The tensor scale s_t = amax / 2688 needs
// max |y| over the whole batch before any group can be quantised, so the CTAs meet once:
// each folds its maximum into ws[0] (float bits, atomicMax), counts itself into ws[1], and
// waits (bounded in time) until ws[1] reaches the grid size; then every CTA quantises
// with the same s_t, and the last CTA to leave (ws[2]) puts the three words back to zero.
// The CTAs wait on one another, so the host launches this only as a cooperative launch
// whose grid is resident at once.  ws: three words, zero before the launch, zero after a
// launch that completed without error.
template <bool EMIT_Y, bool SHARED_T>
__global__ void __launch_bounds__(kSmallRows)
    wush_small_nvfp4_onepass_kernel(const __nv_bfloat16* __restrict__ x, const FusedParams p, unsigned int* ws) {
  __shared__ __align__(16) float Ts[16 * 16];
  __shared__ float warp_max[kSmallRows / 32];
  __shared__ float s_amax;
  __shared__ int s_ok;
  const int blk = static_cast<int>(blockIdx.x);
  float y[16];
  bool valid;
  long long row;
  small_transform<16, SHARED_T>(x, p, Ts, y, valid, row);

  float m = group_absmax<16>(y);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float cm = warp_max[0];
#pragma unroll
    for (int w = 1; w < kSmallRows / 32; ++w) cm = fmaxf(cm, warp_max[w]);
    const unsigned int total = gridDim.x * gridDim.y;
    if (cm > 0.0f) atomicMax(&ws[0], __float_as_uint(cm));
    red_add_release_gpu(&ws[1]);                // the maximum above is ordered before the count
    const uint64_t t0 = global_timer_ns();
    int ok = 1;
    while (ld_acquire_gpu(&ws[1]) < total) {
      __nanosleep(64);
      if (global_timer_ns() - t0 > p.wait_limit_ns) {   // a CTA never arrived
        atomicOr(&g_wush_device_error, 128u);
        ok = 0;
        break;
      }
    }
    s_amax = __uint_as_float(ld_acquire_gpu(&ws[0]));   // ordered after the poll's acquire
    s_ok = ok;
    if (ok && atomicAdd(&ws[2], 1u) == total - 1) {     // every CTA has read the maximum
      ws[0] = 0u;
      ws[1] = 0u;
      ws[2] = 0u;
      __threadfence();
    }
  }
  __syncthreads();
  if (!s_ok) return;
  const float s_t = __fdiv_rn(s_amax, 2688.0f);
  if (blk == 0 && blockIdx.y == 0 && threadIdx.x == 0) *const_cast<float*>(p.tensor_scale) = s_t;
  if (!valid) return;
  if (EMIT_Y) {
    float4* yd = reinterpret_cast<float4*>(p.y_out + row * p.d_in + static_cast<long long>(blk) * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) yd[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
  }
  uint32_t words[2];
  static_cast<uint8_t*>(p.scales)[row * p.C + blk] =
      static_cast<uint8_t>(quant_nv<16>(y, s_t, __fmul_rn(6.0f, s_t), words));
  *reinterpret_cast<uint2*>(p.codes + row * (p.d_in / 2) + static_cast<long long>(blk) * 8) =
      make_uint2(words[0], words[1]);
}

}  // namespace wush
