// Fused per-block transform + AbsMax 4-bit quantisation for sm_100a.
//
// Operation (paper-graph-ui analysis of arXiv 2512.00956, §3.2 "Online Activation
// Transform + Quantize Kernel" and §3.4.7 "GPU Kernel Design"): the rows of a
// [n_rows][d_in] matrix are split along d_in into C = d_in / G blocks; block i of
// every row is multiplied by its own G x G matrix T_i (y = T_i x), then each group of
// G transformed values is AbsMax-quantised to MXFP4 / NVFP4 / INT4 and packed.
//
// B200 design (not the pages' CUTLASS kernel, which targeted RTX 5090):
//  * persistent CTAs, one per SM, each owning a contiguous run of 128-row x CH-channel
//    tiles, column-tile major so consecutive tiles share their transforms;
//  * warp 0 streams the input tiles with TMA (128-byte swizzle) through a STAGES-deep
//    mbarrier ring; warps 2-5 split each fp32 T_i into bf16 hi + lo panels in shared
//    memory (and, for fp32 weights, split the weight tile into bf16 hi + lo operands);
//  * warp 1 issues tcgen05.mma (M=128, N=G, K=16) with fp32 accumulators in TMEM:
//    X*T_hi^T + X*T_lo^T for bf16 activations, W_hi*T_hi^T + W_hi*T_lo^T + W_lo*T_hi^T
//    for fp32 weights, double-buffered in TMEM;
//  * warps 6-13 read the accumulators with tcgen05.ld (one token row per thread, a
//    whole group in registers), compute the AbsMax scale, round and pack, and store
//    16-byte vectors directly to global memory.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "wush_ptx.cuh"

namespace wush {

enum : int { kMXFP4 = 0, kNVFP4 = 1, kINT4 = 2 };

struct FusedParams {
  const float* T;           // [C][G][G] fp32 transforms, row-major per block
  uint8_t* codes;           // [n_rows][d_in/2]
  void* scales;             // [n_rows][C]  u8 (MXFP4 / NVFP4) or fp32 (INT4)
  float* y_out;             // optional [n_rows][d_in] fp32 transformed values (debug)
  unsigned int* amax_word;  // NVFP4 pass 1: running max of |y| as float bits
  const float* tensor_scale;  // NVFP4 pass 2: s_t (already final)
  long long n_rows;
  int d_in;
  int C;
  int n_row_tiles;
  int total_tiles;
  unsigned long long wait_limit_ns;
};

template <int G_, int FMT_, bool IN_F32_, bool AMAX_ONLY_, bool EMIT_Y_>
struct FusedCfg {
  static constexpr int G = G_;
  static constexpr int FMT = FMT_;
  static constexpr bool IN_F32 = IN_F32_;
  static constexpr bool AMAX_ONLY = AMAX_ONLY_;
  static constexpr bool EMIT_Y = EMIT_Y_;
  static constexpr int BM = 128;                       // rows per tile = UMMA M
  static constexpr int CH = IN_F32 ? 64 : 128;         // channels per tile
  static constexpr int BPT = CH / G;                   // blocks per tile
  static constexpr int SUB = CH / 64;                  // 128-byte-wide bf16 operand sub-tiles
  static constexpr int STAGES = IN_F32 ? 3 : 5;
  static constexpr int STAGE_BYTES = IN_F32 ? BM * CH * 4 : BM * CH * 2;  // 32 KiB
  static constexpr int OPER_BYTES = BM * CH * 2;       // one bf16 operand tile (hi or lo)
  static constexpr int BLK_PER_PANEL = 32 / G;         // blocks whose hi|lo rows share a 128 B row
  static constexpr int PANEL_BYTES = G * 128;
  static constexpr int N_PANELS = BPT / BLK_PER_PANEL;
  static constexpr int TSLOT_BYTES = N_PANELS * PANEL_BYTES;
  static constexpr int TMEM_COLS = 2 * CH;             // two accumulator buffers
  static constexpr int N_EPI_WARPS = 8;
  static constexpr int BPW = BPT / 2;                  // blocks per epilogue warp
  static constexpr int THREADS = 14 * 32;
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_OPER = OFF_STAGE + STAGES * STAGE_BYTES;
  static constexpr int OFF_T = OFF_OPER + (IN_F32 ? 2 * 2 * OPER_BYTES : 0);
  static constexpr int OFF_BAR = OFF_T + 2 * TSLOT_BYTES;
  // barriers: full[S], empty[S], ofull[2], oempty[2], tfull[2], tempty[2], afull[2], aempty[2], drain
  static constexpr int N_BARS = 2 * STAGES + 13;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;   // + alignment slack
  static_assert(G == 16 || G == 32, "G must be 16 or 32");
  static_assert(!(FMT == kMXFP4 && G != 32) && !(FMT == kNVFP4 && G != 16), "format/group mismatch");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// byte offset of logical 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// Split 8 fp32 values into bf16 hi = rn(v) and lo = rn(v - hi), packed 2 per word.
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat16 a = __float2bfloat16_rn(v[2 * k]), b = __float2bfloat16_rn(v[2 * k + 1]);
    __nv_bfloat16 ar = __float2bfloat16_rn(v[2 * k] - __bfloat162float(a));
    __nv_bfloat16 br = __float2bfloat16_rn(v[2 * k + 1] - __bfloat162float(b));
    h[k] = bf16x2_bits(a, b);
    l[k] = bf16x2_bits(ar, br);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ---------------------------------------------------------------- group quantisers
// Each consumes the G transformed values of one (row, block) group held in registers
// and produces G/8 packed code words plus the group's scale.

// MXFP4: scale 2^e with e the least integer such that amax <= 6 * 2^e (clamped to
// [-127, 127]); the E8M0 byte is e + 127.  With amax = m * 2^E (1 <= m < 2),
// e = E - 2 when m <= 1.5 and E - 1 otherwise, read off the float's bits.
template <int NV>
__device__ __forceinline__ uint32_t quant_mx(const float* v, uint32_t* words) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < NV; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const uint32_t ab = __float_as_uint(amax);
  int sb = static_cast<int>(ab >> 23) - 2 + ((ab & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  sb = max(sb, 0);
  // multiplier 2^-e = 2^(127 - sb): exponent field 254 - sb, or the subnormal 2^-127
  const float mul = __uint_as_float(sb < 254 ? static_cast<uint32_t>(254 - sb) << 23 : 0x00400000u);
  float w[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) w[j] = v[j] * mul;   // exact: multiplication by a power of two
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) words[k] = e2m1_pack8(w + 8 * k);
  return static_cast<uint32_t>(sb);
}

// NVFP4: r = amax / (6 s_t), block scale = E4M3(r), S = dec(sb) * s_t,
// codes = E2M1(y * (1/S)); every step rounded to fp32 (IEEE division / reciprocal).
template <int NV>
__device__ __forceinline__ uint32_t quant_nv(const float* v, float s_t, float d6, uint32_t* words) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < NV; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const float r = d6 > 0.0f ? __fdiv_rn(amax, d6) : 0.0f;
  const uint32_t sb = e4m3_byte(r);
  const float S = __fmul_rn(e4m3_value(sb), s_t);
  float inv = S > 0.0f ? __frcp_rn(S) : 0.0f;
  if (isinf(inv)) inv = 0.0f;       // scale below the fp32 reciprocal range: group encodes as zero
  float w[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) w[j] = __fmul_rn(v[j], inv);
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) words[k] = e2m1_pack8(w + 8 * k);
  return sb;
}

// INT4 symmetric: s = amax / 7, q = clamp(rne(y * (1/s)), -7, 7), two's-complement nibbles.
template <int NV>
__device__ __forceinline__ float quant_int4(const float* v, uint32_t* words) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < NV; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const float s = __fdiv_rn(amax, 7.0f);
  float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (isinf(inv)) inv = 0.0f;
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) {
    uint32_t wd = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int q = __float2int_rn(__fmul_rn(v[8 * k + e], inv));
      q = min(7, max(-7, q));
      wd |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
    }
    words[k] = wd;
  }
  return s;
}

template <typename T>
__device__ __forceinline__ T* offset_ptr(void* base, long long bytes) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(base) + bytes);
}

// ---------------------------------------------------------------- the kernel
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    wush_fused_kernel(const __grid_constant__ CUtensorMap tmap_in, const FusedParams p) {
  constexpr int G = Cfg::G, CH = Cfg::CH, BPT = Cfg::BPT, STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  const uint32_t bar0 = smem_addr(bars);
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int B_FULL = 0, B_EMPTY = STAGES, B_OFULL = 2 * STAGES, B_OEMPTY = 2 * STAGES + 2,
            B_TFULL = 2 * STAGES + 4, B_TEMPTY = 2 * STAGES + 6, B_AFULL = 2 * STAGES + 8,
            B_AEMPTY = 2 * STAGES + 10, B_DRAIN = 2 * STAGES + 12;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.total_tiles, nrt = p.n_row_tiles;
  const int t_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * total / gridDim.x);
  const int t_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * total / gridDim.x);
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(BAR(B_FULL + s), 1);
      mbar_init(BAR(B_EMPTY + s), Cfg::IN_F32 ? 128 : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(BAR(B_OFULL + k), 128);
      mbar_init(BAR(B_OEMPTY + k), 1);
      mbar_init(BAR(B_TFULL + k), 128);
      mbar_init(BAR(B_TEMPTY + k), 1);
      mbar_init(BAR(B_AFULL + k), 1);
      mbar_init(BAR(B_AEMPTY + k), Cfg::N_EPI_WARPS);
    }
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_in);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[STAGES];
      bool issued[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
      for (int t = t_begin; t < t_end; ++t) {
        if (!wait_bounded(BAR(B_EMPTY + stage), phase ^ 1u, abort_flag, 1u, lim)) break;
        const int ct = t / nrt, rt = t - ct * nrt;
        const uint32_t dst = sbase + Cfg::OFF_STAGE + stage * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(BAR(B_FULL + stage), Cfg::STAGE_BYTES);
        if (Cfg::IN_F32) {
          tma_load_2d(dst, &tmap_in, BAR(B_FULL + stage), ct * CH, rt * 128, pol);
        } else {
#pragma unroll
          for (int s = 0; s < Cfg::SUB; ++s)
            tma_load_2d(dst + s * 16384, &tmap_in, BAR(B_FULL + stage), ct * CH + 64 * s, rt * 128, pol);
        }
        issued[stage] = true;
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
      if (*abort_flag) {  // let every copy still in flight land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) {
            volatile int no_abort = 0;
            wait_bounded(BAR(B_FULL + s), static_cast<uint32_t>(issued_parity[s]), &no_abort, 16u, lim);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, G);
      int stage = 0, obuf = 0;
      uint32_t phase = 0, ophase = 0;
      int epoch = -1, prev_ct = -1;
      int it = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t, ++it) {
        const int ct = t / nrt;
        if (ct != prev_ct) {
          ++epoch;
          prev_ct = ct;
          if (!wait_bounded(BAR(B_TFULL + (epoch & 1)), static_cast<uint32_t>((epoch >> 1) & 1), abort_flag, 2u, lim)) { ok = false; break; }
        }
        const int tslot = epoch & 1;
        uint32_t a_hi, a_lo = 0;
        if (Cfg::IN_F32) {
          if (!wait_bounded(BAR(B_OFULL + obuf), ophase, abort_flag, 2u, lim)) { ok = false; break; }
          a_hi = sbase + Cfg::OFF_OPER + obuf * 2 * Cfg::OPER_BYTES;
          a_lo = a_hi + Cfg::OPER_BYTES;
        } else {
          if (!wait_bounded(BAR(B_FULL + stage), phase, abort_flag, 2u, lim)) { ok = false; break; }
          a_hi = sbase + Cfg::OFF_STAGE + stage * Cfg::STAGE_BYTES;
        }
        const int acc = it & 1;
        if (!wait_bounded(BAR(B_AEMPTY + acc), static_cast<uint32_t>(((it >> 1) & 1) ^ 1), abort_flag, 2u, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tbase = sbase + Cfg::OFF_T + tslot * Cfg::TSLOT_BYTES;
#pragma unroll
        for (int b = 0; b < BPT; ++b) {
          const uint32_t d = tmem_base + static_cast<uint32_t>(acc * CH + b * G);
          // A: block b occupies bytes [b*2G, b*2G + 2G) of the 128-byte rows of sub-tile (b*G)/64
          const uint32_t a_off = static_cast<uint32_t>(((b * G) / 64) * 16384 + ((b * G) % 64) * 2);
          // B: panel b / BLK_PER_PANEL; hi at byte (b % BLK_PER_PANEL) * 4G, lo 2G further
          const uint32_t p_off = static_cast<uint32_t>((b / Cfg::BLK_PER_PANEL) * Cfg::PANEL_BYTES +
                                                        (b % Cfg::BLK_PER_PANEL) * 4 * G);
#pragma unroll
          for (int kk = 0; kk < G / 16; ++kk) {
            const uint64_t ah = desc_k_sw128(a_hi + a_off + kk * 32);
            const uint64_t bh = desc_k_sw128(tbase + p_off + kk * 32);
            const uint64_t bl = desc_k_sw128(tbase + p_off + 2 * G + kk * 32);
            umma_bf16(d, ah, bh, idesc, kk > 0 ? 1u : 0u);
            umma_bf16(d, ah, bl, idesc, 1u);
            if (Cfg::IN_F32) {
              const uint64_t al = desc_k_sw128(a_lo + a_off + kk * 32);
              umma_bf16(d, al, bh, idesc, 1u);
            }
          }
        }
        if (Cfg::IN_F32) {
          umma_commit(BAR(B_OEMPTY + obuf));
          if (++obuf == 2) obuf = 0, ophase ^= 1u;
        } else {
          umma_commit(BAR(B_EMPTY + stage));
          if (++stage == STAGES) stage = 0, phase ^= 1u;
        }
        umma_commit(BAR(B_AFULL + acc));
        if (t + 1 == t_end || (t + 1) / nrt != ct) umma_commit(BAR(B_TEMPTY + tslot));
      }
      // every MMA issued above has finished before TMEM can be released
      umma_commit(BAR(B_DRAIN));
      volatile int no_abort = 0;
      wait_bounded(BAR(B_DRAIN), 0u, &no_abort, 16u, lim);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ converters (128 threads)
    const int ct_id = threadIdx.x - 64;
    int epoch = -1, prev_ct = -1;
    int stage = 0, obuf = 0;
    uint32_t phase = 0, ophase = 0;
    for (int t = t_begin; t < t_end; ++t) {
      const int ct = t / nrt;
      if (ct != prev_ct) {
        ++epoch;
        prev_ct = ct;
        const int slot = epoch & 1;
        if (!wait_bounded(BAR(B_TEMPTY + slot), static_cast<uint32_t>(((epoch >> 1) & 1) ^ 1), abort_flag, 4u, lim)) break;
        uint8_t* tdst = smem + Cfg::OFF_T + slot * Cfg::TSLOT_BYTES;
        // BPT blocks x G rows x (G/8) chunks of 8 values
        constexpr int CHUNKS = BPT * G * (G / 8);
        for (int q = ct_id; q < CHUNKS; q += 128) {
          const int b = q / (G * (G / 8));
          const int rem = q - b * (G * (G / 8));
          const int r = rem / (G / 8), j = rem - r * (G / 8);
          const int blk = ct * BPT + b;
          float v[8];
          if (blk < p.C) {
            const float4* src = reinterpret_cast<const float4*>(p.T + (static_cast<long long>(blk) * G + r) * G + 8 * j);
            const float4 u0 = __ldg(src), u1 = __ldg(src + 1);
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
            v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.0f;
          }
          uint4 hi, lo;
          split8(v, hi, lo);
          uint8_t* panel = tdst + (b / Cfg::BLK_PER_PANEL) * Cfg::PANEL_BYTES;
          // a block's hi|lo row span is 4G bytes = G/4 chunks; hi first, lo G/8 chunks later
          const int c0 = (b % Cfg::BLK_PER_PANEL) * (G / 4);
          *reinterpret_cast<uint4*>(panel + sw128_off(r, c0 + j)) = hi;
          *reinterpret_cast<uint4*>(panel + sw128_off(r, c0 + G / 8 + j)) = lo;
        }
        fence_proxy_async_smem();
        mbar_arrive(BAR(B_TFULL + slot));
      }
      if (Cfg::IN_F32) {
        if (!wait_bounded(BAR(B_FULL + stage), phase, abort_flag, 4u, lim)) break;
        if (!wait_bounded(BAR(B_OEMPTY + obuf), ophase ^ 1u, abort_flag, 4u, lim)) break;
        const uint8_t* src = smem + Cfg::OFF_STAGE + stage * Cfg::STAGE_BYTES;     // [128][CH] fp32, dense
        uint8_t* dhi = smem + Cfg::OFF_OPER + obuf * 2 * Cfg::OPER_BYTES;
        uint8_t* dlo = dhi + Cfg::OPER_BYTES;
        constexpr int CPR = CH / 8;    // 16-byte output chunks per row
        for (int q = ct_id; q < 128 * CPR; q += 128) {
          const int r = q / CPR, j = q - r * CPR;
          const float4* s4 = reinterpret_cast<const float4*>(src + r * CH * 4 + j * 32);
          const float4 u0 = s4[0], u1 = s4[1];
          const float v[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          uint4 hi, lo;
          split8(v, hi, lo);
          const int sub = j / 8, jc = j % 8;
          *reinterpret_cast<uint4*>(dhi + sub * 16384 + sw128_off(r, jc)) = hi;
          *reinterpret_cast<uint4*>(dlo + sub * 16384 + sw128_off(r, jc)) = lo;
        }
        fence_proxy_async_smem();
        mbar_arrive(BAR(B_EMPTY + stage));
        mbar_arrive(BAR(B_OFULL + obuf));
        if (++stage == STAGES) stage = 0, phase ^= 1u;
        if (++obuf == 2) obuf = 0, ophase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quad = warp & 3;                 // TMEM lanes this warp may read
    const int half = (warp - 6) >> 2;          // which half of the tile's blocks
    const int C = p.C;
    float s_t = 0.0f, d6 = 0.0f;
    if (Cfg::FMT == kNVFP4 && !Cfg::AMAX_ONLY) {
      s_t = *p.tensor_scale;
      d6 = __fmul_rn(6.0f, s_t);
    }
    float run_max = 0.0f;
    int it = 0;
    for (int t = t_begin; t < t_end; ++t, ++it) {
      const int acc = it & 1;
      if (!wait_bounded(BAR(B_AFULL + acc), static_cast<uint32_t>((it >> 1) & 1), abort_flag, 8u, lim)) break;
      tc_fence_after();
      const int ct = t / nrt, rt = t - ct * nrt;
      float v[Cfg::BPW][G];
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * CH);
#pragma unroll
      for (int bb = 0; bb < Cfg::BPW; ++bb) {
        const uint32_t ta = tq + static_cast<uint32_t>((half * Cfg::BPW + bb) * G);
        if (G == 32) tmem_ld_x32(ta, v[bb]); else tmem_ld_x16(ta, v[bb]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_AEMPTY + acc));

      const long long row = static_cast<long long>(rt) * 128 + quad * 32 + lane;
      const bool row_ok = row < p.n_rows;
      const int blk0 = ct * BPT + half * Cfg::BPW;
      if (Cfg::AMAX_ONLY) {
#pragma unroll
        for (int bb = 0; bb < Cfg::BPW; ++bb)
          if (row_ok && blk0 + bb < C)
#pragma unroll
            for (int j = 0; j < G; ++j) run_max = fmaxf(run_max, fabsf(v[bb][j]));
        continue;
      }
#pragma unroll
      for (int bb = 0; bb < Cfg::BPW; ++bb) {
        const int blk = blk0 + bb;
        if (!row_ok || blk >= C) continue;
        uint32_t words[G / 8];
        const long long cbyte = row * (p.d_in / 2) + static_cast<long long>(blk) * (G / 2);
        if (Cfg::FMT == kMXFP4) {
          const uint32_t sb = quant_mx<G>(v[bb], words);
          offset_ptr<uint8_t>(p.scales, row * C + blk)[0] = static_cast<uint8_t>(sb);
        } else if (Cfg::FMT == kNVFP4) {
          const uint32_t sb = quant_nv<G>(v[bb], s_t, d6, words);
          offset_ptr<uint8_t>(p.scales, row * C + blk)[0] = static_cast<uint8_t>(sb);
        } else {
          const float s = quant_int4<G>(v[bb], words);
          offset_ptr<float>(p.scales, (row * C + blk) * 4)[0] = s;
        }
        if (G == 32) {
          *offset_ptr<uint4>(p.codes, cbyte) = make_uint4(words[0], words[1], words[2], words[3]);
        } else {
          *offset_ptr<uint2>(p.codes, cbyte) = make_uint2(words[0], words[1]);
        }
        if (Cfg::EMIT_Y) {
          float4* yd = reinterpret_cast<float4*>(p.y_out + row * p.d_in + static_cast<long long>(blk) * G);
#pragma unroll
          for (int k = 0; k < G / 4; ++k)
            yd[k] = make_float4(v[bb][4 * k], v[bb][4 * k + 1], v[bb][4 * k + 2], v[bb][4 * k + 3]);
        }
      }
    }
    if (Cfg::AMAX_ONLY) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) run_max = fmaxf(run_max, __shfl_xor_sync(0xffffffffu, run_max, o));
      if (lane == 0 && run_max > 0.0f) atomicMax(p.amax_word, __float_as_uint(run_max));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// NVFP4: turn the running |y| maximum (float bits) into the fp32 tensor scale
// s_t = amax / (6 * 448), in place.
__global__ void wush_nvfp4_tensor_scale_kernel(float* tensor_scale) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(tensor_scale));
    *tensor_scale = __fdiv_rn(amax, 2688.0f);
  }
}

}  // namespace wush
