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
//    mbarrier ring and bulk-copies each column tile's fp32 matrices into a transform
//    slot; warps 2-3 split them in place into bf16 hi and lo, stacked along N (for fp32
//    weights warps 2-3 and 8-11 also split each staged weight tile into bf16 hi + lo
//    operands);
//  * warp 1 issues tcgen05.mma (M=128, N=2G, K=16) into fp32 TMEM accumulators,
//    double-buffered: one MMA per block and K-step yields X*T_hi^T and X*T_lo^T side
//    by side (fp32 weights add W_lo*T_hi^T into the first half; the dropped W_lo*T_lo
//    term is below 2^-16 relative).  Each tcgen05.mma costs the issuing thread ~50
//    cycles whatever N is, so stacking hi|lo halves the issue work of the tile;
//  * two epilogue groups (warps 4-7 and 8-11; one group, warps 4-7, for fp32 weights)
//    take alternate tiles: they read the accumulators with tcgen05.ld (one token row
//    per thread, 64 columns per load), add the hi and lo halves, compute the AbsMax
//    scale, round and pack, stage the tile's codes in shared memory for one TMA store and
//    write the row's scales (row-major, or in the block-scaled MMA's scale-atom layout).
//  * every wait is an mbarrier try_wait with a suspend-time hint, so waiting warps do
//    not take issue slots from the working ones.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <type_traits>
#include "wush_ptx.cuh"

// Tuning of the bf16 activation path (channels per tile, input stages in flight).
#ifndef WUSH_ACT_TILE_CH
#define WUSH_ACT_TILE_CH 128
#endif
#ifndef WUSH_ACT_STAGES
#define WUSH_ACT_STAGES 5
#endif

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
  int codes_via_tma;        // 1: codes leave through the TMA store map (needs d_in % 32 == 0)
  int scale_atoms;          // MXFP4 only: 1 = scales in the block-scaled MMA's scale-atom layout
  int atom_cols;            // scale atoms per 128-row block (C padded to 4, / 4)
  int prefetch_tiles;       // input tiles per CTA warmed in L2 before the dependency wait
  unsigned long long wait_limit_ns;
};

template <int G_, int FMT_, bool IN_F32_, bool AMAX_ONLY_, bool EMIT_Y_, bool SHARED_T_ = false>
struct FusedCfg {
  static constexpr int G = G_;
  static constexpr int FMT = FMT_;
  // SHARED_T: one G x G matrix for every block (the H+Quant comparator); it is converted
  // once per CTA and the transform slot is never refilled
  static constexpr bool SHARED_T = SHARED_T_;
  static constexpr bool IN_F32 = IN_F32_;
  static constexpr bool AMAX_ONLY = AMAX_ONLY_;
  static constexpr bool EMIT_Y = EMIT_Y_;
  static constexpr int BM = 128;                       // rows per tile = UMMA M
  static constexpr int CH = IN_F32 ? 64 : WUSH_ACT_TILE_CH;   // channels per tile
  static constexpr int BPT = CH / G;                   // blocks per tile
  static constexpr int SUB = CH / 64;                  // 128-byte-wide bf16 operand sub-tiles
  static constexpr int STAGES = IN_F32 ? 3 : WUSH_ACT_STAGES;
  static constexpr int STAGE_BYTES = IN_F32 ? BM * CH * 4 : BM * CH * 2;  // 32 KiB fp32, 16 KiB bf16
  static constexpr int OPER_BYTES = BM * CH * 2;       // one bf16 operand tile (hi or lo)
  // transform panels: 2G rows (hi rows then lo rows) x 128 bytes of K; a 128-byte row
  // holds the K = G values of BPP = 64/G blocks side by side
  static constexpr int BPP = 64 / G;
  static constexpr int PANEL_BYTES = 2 * G * 128;
  static constexpr int N_PANELS = BPT / BPP;
  static constexpr int TSLOT_BYTES = N_PANELS * PANEL_BYTES;
  static constexpr int ACC_COLS = 2 * CH;              // hi|lo of every block of a tile
  static constexpr int NACC = 512 / ACC_COLS;          // accumulator buffers in TMEM
  static constexpr int TMEM_COLS = NACC * ACC_COLS;
  // fp32 (weight) tiles need their hi/lo split, a job for more threads than the two
  // converter warps: there warps 8-11 convert too and one epilogue group remains
  static constexpr int N_GROUPS = IN_F32 ? 1 : 2;      // epilogue groups, alternate tiles
  static constexpr int CONV_THREADS = IN_F32 ? 192 : 64;
  static constexpr int GROUP_WARPS = 4;                // one warp per TMEM lane quadrant
  static constexpr int THREADS = 12 * 32;
  static constexpr int CODE_STAGE = 128 * CH / 2;      // one tile of packed codes
  static_assert(NACC % N_GROUPS == 0, "each group owns whole accumulator buffers");
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_OPER = OFF_STAGE + STAGES * STAGE_BYTES;
  static constexpr int OFF_T = OFF_OPER + (IN_F32 ? 2 * 2 * OPER_BYTES : 0);
  static constexpr int OFF_CODES = OFF_T + 2 * TSLOT_BYTES;   // [group][2] code staging buffers
  static constexpr int OFF_BAR = OFF_CODES + N_GROUPS * 2 * CODE_STAGE;
  // barriers: full[S], empty[S], ofull[2], oempty[2], tfull[2], tempty[2], afull[NACC], aempty[NACC], drain,
  // tload[2], tread[2]
  static constexpr int N_BARS = 2 * STAGES + 13 + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int OFF_NVTAB = OFF_MISC + 64;     // NVFP4: 128 fp32 scale reciprocals
  static constexpr int SMEM_BYTES = OFF_NVTAB + 512 + 1024;   // + alignment slack
  static_assert(G == 16 || G == 32, "G must be 16 or 32");
  static_assert(!(SHARED_T && IN_F32), "the shared-matrix variant is an activation path");
  static_assert(!(FMT == kMXFP4 && G != 32) && !(FMT == kNVFP4 && G != 16), "format/group mismatch");
  static_assert(TMEM_COLS <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_CODES % 1024 == 0 && CODE_STAGE % 1024 == 0, "swizzled staging alignment");
};

// byte offset of logical 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}


// Split 8 fp32 values into bf16 hi = rn(v) and lo = rn(v - hi), packed 2 per word (the
// first value in the low half).  v - hi is exact in fp32, so lo is the one rounding of
// the remainder; pairs go through cvt.rn.bf16x2.f32 and one packed fp32 subtraction.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo_half, float hi_half) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi_half), "f"(lo_half));
  return r;
}
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    h[k] = cvt_bf16x2(v[2 * k], v[2 * k + 1]);
    float r0 = v[2 * k], r1 = v[2 * k + 1];
    const float b0 = __uint_as_float(h[k] << 16), b1 = __uint_as_float(h[k] & 0xFFFF0000u);
    asm("{\n\t.reg .b64 ra, rb;\n\t"
        "mov.b64 ra, {%0, %1};\n\t"
        "mov.b64 rb, {%2, %3};\n\t"
        "sub.rn.f32x2 ra, ra, rb;\n\t"
        "mov.b64 {%0, %1}, ra;\n\t}"
        : "+f"(r0), "+f"(r1)
        : "f"(b0), "f"(b1));
    l[k] = cvt_bf16x2(r0, r1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Packed fp32 pair arithmetic (sm_100a add/mul .f32x2): each is the IEEE round-to-nearest
// result of the two scalar operations.
__device__ __forceinline__ void add2_rn(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2_rn(float& a0, float& a1, float m) {
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %2};\n\t"
      "mul.rn.f32x2 ra, ra, rb;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(m));
}

// Largest |v_j| of a group, as a balanced tree (max is exact, so the order is free).
template <int NV>
__device__ __forceinline__ float group_absmax(const float* v) {
  float m[NV / 2];
#pragma unroll
  for (int j = 0; j < NV / 2; ++j) m[j] = fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1]));
#pragma unroll
  for (int w = NV / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; ++j) m[j] = fmaxf(m[j], m[j + w]);
  return m[0];
}

// ---------------------------------------------------------------- group quantisers
// Each consumes the G transformed values of one (row, block) group held in registers
// and produces G/8 packed code words plus the group's scale.

// MXFP4: scale 2^e with e the least integer such that amax <= 6 * 2^e (clamped to
// [-127, 127]); the E8M0 byte is e + 127.  With amax = m * 2^E (1 <= m < 2),
// e = E - 2 when m <= 1.5 and E - 1 otherwise, read off the float's bits.
template <int NV>
__device__ __forceinline__ uint32_t quant_mx(const float* v, uint32_t* words) {
  const float amax = group_absmax<NV>(v);
  const uint32_t ab = __float_as_uint(amax);
  int sb = static_cast<int>(ab >> 23) - 2 + ((ab & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  sb = max(sb, 0);
  // multiplier 2^-e = 2^(127 - sb): exponent field 254 - sb, or the subnormal 2^-127
  const float mul = __uint_as_float(sb < 254 ? static_cast<uint32_t>(254 - sb) << 23 : 0x00400000u);
  float w[NV];
#pragma unroll
  for (int j = 0; j < NV; j += 2) {   // exact: multiplication by a power of two
    w[j] = v[j];
    w[j + 1] = v[j + 1];
    mul2_rn(w[j], w[j + 1], mul);
  }
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) words[k] = e2m1_pack8(w + 8 * k);
  return static_cast<uint32_t>(sb);
}

// NVFP4: r = amax / (6 s_t), block scale = E4M3(r), S = dec(sb) * s_t,
// codes = E2M1(y * (1/S)); every step rounded to fp32 (IEEE division / reciprocal).
template <int NV>
__device__ __forceinline__ uint32_t quant_nv(const float* v, float s_t, float d6, uint32_t* words) {
  const float amax = group_absmax<NV>(v);
  const float r = d6 > 0.0f ? __fdiv_rn(amax, d6) : 0.0f;
  const uint32_t sb = e4m3_byte(r);
  const float S = __fmul_rn(e4m3_value(sb), s_t);
  float inv = S > 0.0f ? __frcp_rn(S) : 0.0f;
  if (isinf(inv)) inv = 0.0f;       // scale below the fp32 reciprocal range: group encodes as zero
  float w[NV];
#pragma unroll
  for (int j = 0; j < NV; j += 2) {   // each product rounded to fp32
    w[j] = v[j];
    w[j + 1] = v[j + 1];
    mul2_rn(w[j], w[j + 1], inv);
  }
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) words[k] = e2m1_pack8(w + 8 * k);
  return sb;
}

// The same NVFP4 group quantiser with the per-call constants of its scale chain hoisted:
//  * r = fl32(amax / d6) by Markstein's correction of a reciprocal product (P. Markstein,
//    IBM J. Res. Dev. 34(1), 1990; see also Muller et al., Handbook of Floating-Point
//    Arithmetic, the theorem on division by fused multiply-add): with inv_d6 = RN(1/d6),
//    q = RN(amax * inv_d6) is within one ulp of the quotient, the residual amax - q * d6 is
//    exact in one FMA, and RN(q + residual * inv_d6) is the correctly rounded quotient,
//    for normal results.  A quotient below the fp32 normal range is far below E4M3's
//    smallest step (2^-9) and encodes as 0 either way; one far above 448 saturates either
//    way.  `exact_div` selects the division
//    itself when inv_d6 is not a normal number (d6 = 0 or extreme);
//  * inv = fl32(1 / fl32(dec(sb) * s_t)) is looked up in a table of the 128 possible block
//    scale bytes, filled once per CTA with those very operations.
// The results are bit-identical to quant_nv.
template <int NV>
__device__ __forceinline__ uint32_t quant_nv_tab(const float* v, float d6, float inv_d6, bool exact_div,
                                                 const float* inv_tab, uint32_t* words) {
  const float amax = group_absmax<NV>(v);
  float r;
  if (exact_div) {
    r = d6 > 0.0f ? __fdiv_rn(amax, d6) : 0.0f;
  } else {
    const float q = __fmul_rn(amax, inv_d6);
    const float res = __fmaf_rn(-q, d6, amax);
    // far above E4M3's largest value (a caller's tensor scale below amax / 2688) the
    // quotient only needs to saturate, and the correction could overflow
    r = q <= 1048576.0f ? __fmaf_rn(res, inv_d6, q) : q;
  }
  const uint32_t sb = e4m3_byte(r);
  const float inv = inv_tab[sb & 127u];
  float w[NV];
#pragma unroll
  for (int j = 0; j < NV; j += 2) {   // each product rounded to fp32
    w[j] = v[j];
    w[j + 1] = v[j + 1];
    mul2_rn(w[j], w[j + 1], inv);
  }
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) words[k] = e2m1_pack8(w + 8 * k);
  return sb;
}

// INT4 symmetric: s = amax / 7, q = clamp(rne(y * (1/s)), -7, 7), two's-complement nibbles.
template <int NV>
__device__ __forceinline__ float quant_int4(const float* v, uint32_t* words) {
  const float amax = group_absmax<NV>(v);
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

// The same INT4 quantiser, bit-identical, without a per-element float-to-integer
// conversion (a reduced-rate instruction):
//  * s = fl32(amax / 7) by the Markstein-corrected reciprocal product (see quant_nv_tab)
//    with inv7 = RN(1/7), for amax >= 2^-122 where the quotient is a normal fp32; the
//    division itself below that;
//  * each product y * inv is clamped to [-7, 7] (equivalent to clamping after rounding,
//    the range being symmetric and integer-bounded) and 1.5 * 2^23 is added: in
//    [2^23, 2^24) the fp32 spacing is 1, so the sum is RNE(v) + 1.5 * 2^23 (that constant
//    is even, so ties still go to the even integer), and the low 4 bits of the sum's
//    encoding are RNE(v) as a two's-complement nibble;
//  * each nibble enters its word by one bit-field insert.
__device__ __forceinline__ uint32_t bfi4(uint32_t word, uint32_t bits, int pos) {
  uint32_t out;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(out) : "r"(bits), "r"(word), "r"(pos));
  return out;
}
template <int NV>
__device__ __forceinline__ float quant_int4_fast(const float* v, float inv7, uint32_t* words) {
  const float amax = group_absmax<NV>(v);
  float s;
  if (amax >= 1.8807909613e-37f) {   // 2^-122
    const float q = __fmul_rn(amax, inv7);
    const float res = __fmaf_rn(-q, 7.0f, amax);
    s = __fmaf_rn(res, inv7, q);
  } else {
    s = __fdiv_rn(amax, 7.0f);
  }
  float inv = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (isinf(inv)) inv = 0.0f;
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
#pragma unroll
  for (int k = 0; k < NV / 8; ++k) {
    float w[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      w[e] = v[8 * k + e];
      w[e + 1] = v[8 * k + e + 1];
      mul2_rn(w[e], w[e + 1], inv);
      w[e] = fminf(fmaxf(w[e], -7.0f), 7.0f);
      w[e + 1] = fminf(fmaxf(w[e + 1], -7.0f), 7.0f);
      add2_rn(w[e], w[e + 1], kRound, kRound);
    }
    uint32_t wd = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) wd = bfi4(wd, __float_as_uint(w[e]), 4 * e);
    words[k] = wd;
  }
  return s;
}

template <typename T>
__device__ __forceinline__ T* offset_ptr(void* base, long long bytes) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(base) + bytes);
}

// ---------------------------------------------------------------- the kernel
// REV: walk the tiles from the last to the first (CTA b takes the run CTA grid-1-b would
// take, backwards).  The NVFP4 quantising pass does, so that it first reads the tiles the
// amax pass loaded last, while they are still in L2.
//
// ONEPASS (NVFP4 only): the whole NVFP4 call in one cooperative launch.  Each CTA walks its
// run twice, forwards for max |y| and then backwards to quantise (so that its first
// quantised tiles are the ones it loaded last, still in L2); in between, the CTAs fold
// their maxima into a three-word workspace (p.amax_word) and wait for one another
// (bounded in time, error bit 128), then quantise with the common tensor scale.
template <class Cfg, bool REV = false, bool ONEPASS = false>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    wush_fused_kernel(const __grid_constant__ CUtensorMap tmap_in, const __grid_constant__ CUtensorMap tmap_codes,
                      const FusedParams p) {
  constexpr int G = Cfg::G, CH = Cfg::CH, BPT = Cfg::BPT, STAGES = Cfg::STAGES;
  constexpr int NCH = CH / 32;                 // 16-byte code chunks per staged row
  constexpr int SW_SHIFT = NCH == 4 ? 1 : 2;   // staging swizzle = TMA 64B / 32B swizzle pattern
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Cfg::OFF_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int B_FULL = 0, B_EMPTY = STAGES, B_OFULL = 2 * STAGES, B_OEMPTY = 2 * STAGES + 2,
            B_TFULL = 2 * STAGES + 4, B_TEMPTY = 2 * STAGES + 6, B_AFULL = 2 * STAGES + 8,
            B_AEMPTY = 2 * STAGES + 8 + Cfg::NACC, B_DRAIN = 2 * STAGES + 8 + 2 * Cfg::NACC,
            B_TLOAD = B_DRAIN + 1, B_TREAD = B_DRAIN + 3;
  constexpr int NACC = Cfg::NACC;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.total_tiles, nrt = p.n_row_tiles;
  // Runs of total / grid tiles, one longer for the first total % grid CTAs.  The CTAs with
  // the highest indices are dispatched last, onto the SMs the previous kernel frees last,
  // and so start late: they take the short runs.
  const int run_s = total / static_cast<int>(gridDim.x), n_long = total - run_s * static_cast<int>(gridDim.x);
  const int bx = static_cast<int>(blockIdx.x);
  const int t_begin = bx < n_long ? bx * (run_s + 1) : n_long * (run_s + 1) + (bx - n_long) * run_s;
  const int t_end = t_begin + run_s + (bx < n_long ? 1 : 0);
  const uint64_t lim = p.wait_limit_ns;
  auto tile_at = [&](int t) { return REV ? total - 1 - t : t; };   // tile number -> tile
  static_assert(!ONEPASS || (Cfg::FMT == kNVFP4 && !Cfg::AMAX_ONLY && !Cfg::IN_F32 && !Cfg::SHARED_T && !REV),
                "the one-launch walk is an NVFP4 activation path");
  // the walk: the CTA's run, and for ONEPASS the same run backwards after it
  const int run_len = t_end - t_begin;
  const int walk_len = ONEPASS ? 2 * run_len : run_len;
  auto walk_tile = [&](int i) { return (!ONEPASS || i < run_len) ? t_begin + i : t_end - 1 - (i - run_len); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(BAR(B_FULL + s), 1);
      mbar_init(BAR(B_EMPTY + s), Cfg::IN_F32 ? Cfg::CONV_THREADS : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(BAR(B_OFULL + k), Cfg::CONV_THREADS);
      mbar_init(BAR(B_OEMPTY + k), 1);
      mbar_init(BAR(B_TFULL + k), 64);
      mbar_init(BAR(B_TEMPTY + k), 1);
    }
    for (int k = 0; k < NACC; ++k) {
      mbar_init(BAR(B_AFULL + k), 1);
      mbar_init(BAR(B_AEMPTY + k), Cfg::GROUP_WARPS);
    }
    mbar_init(BAR(B_DRAIN), 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(BAR(B_TLOAD + k), 1);
      mbar_init(BAR(B_TREAD + k), 64);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_in);
    if (p.codes_via_tma) tma_prefetch_desc(&tmap_codes);
    // Warm L2 with the CTA's first input tiles and its first column tile's matrices while
    // the previous kernel in the stream drains.  A prefetch hands no data to this CTA and
    // L2 is the point of coherence, so the loads issued after the dependency wait still
    // see everything the previous kernel wrote.
    for (int k = 0; k < p.prefetch_tiles && t_begin + k < t_end; ++k) {
      const int t = tile_at(t_begin + k);
      const int ct = t / nrt, rt = t - ct * nrt;
#pragma unroll
      for (int s = 0; s < Cfg::SUB; ++s) tma_prefetch_l2_2d(&tmap_in, ct * CH + 64 * s, rt * 128);
    }
    if (p.prefetch_tiles > 0 && t_begin < t_end) {
      const int ct = tile_at(t_begin) / nrt;
      const int nblk = Cfg::SHARED_T ? 1 : min(BPT, p.C - ct * BPT);
      bulk_prefetch_l2(p.T + (Cfg::SHARED_T ? 0ll : static_cast<long long>(ct) * BPT * G * G),
                       static_cast<uint32_t>(nblk * G * G * 4));
    }
  }
  // Launched with programmatic stream serialisation: everything above overlapped the end
  // of the previous kernel in the stream; its results are visible only after this wait.
  grid_dependency_wait();
  grid_launch_dependents();
  // A column tile's matrices (BPT blocks x G x G fp32, contiguous in global memory) reach
  // their transform slot by one bulk copy; the converter warps then split them in place
  // into the bf16 hi/lo panels.
  constexpr int T_CHUNKS = BPT * G * (G / 8);            // 8-value chunks of one column tile
  constexpr int T_PER_THREAD = (T_CHUNKS + 63) / 64;    // converter id v takes v, v + 64, ...
  auto t_copy = [&](int ct, int slot) {                  // one thread
    const int nblk = Cfg::SHARED_T ? 1 : min(BPT, p.C - ct * BPT);
    const uint32_t bytes = static_cast<uint32_t>(nblk * G * G * 4);
    const float* src = p.T + (Cfg::SHARED_T ? 0ll : static_cast<long long>(ct) * BPT * G * G);
    mbar_arrive_expect_tx(BAR(B_TLOAD + slot), bytes);
    bulk_load_1d(sbase + Cfg::OFF_T + slot * Cfg::TSLOT_BYTES, src, bytes, BAR(B_TLOAD + slot));
  };
  // one 8-value chunk q of a slot's raw fp32 matrices -> registers (the shared-matrix
  // variant reads the one matrix for every block)
  auto load_chunk = [&](int q, const uint8_t* slot_raw, float4& a, float4& b) {
    const int qs = Cfg::SHARED_T ? q % (G * (G / 8)) : q;
    const float4* src = reinterpret_cast<const float4*>(slot_raw + qs * 32);
    a = src[0];
    b = src[1];
  };
  // its hi/lo split into the K-major SW128 panels of the slot
  auto store_chunk = [&](int q, const float4& a, const float4& b4, uint8_t* tdst) {
    const int b = q / (G * (G / 8));
    const int rem = q - b * (G * (G / 8));
    const int r = rem / (G / 8), j = rem - r * (G / 8);
    const float vals[8] = {a.x, a.y, a.z, a.w, b4.x, b4.y, b4.z, b4.w};
    uint4 hi, lo;
    split8(vals, hi, lo);
    uint8_t* panel = tdst + (b / Cfg::BPP) * Cfg::PANEL_BYTES;
    const int c = (b % Cfg::BPP) * (G / 8) + j;     // 16-byte chunk along K
    *reinterpret_cast<uint4*>(panel + sw128_off(r, c)) = hi;
    *reinterpret_cast<uint4*>(panel + sw128_off(G + r, c)) = lo;
  };
  // raw fp32 chunks of a slot -> registers (converter id v takes v, v + 64, ...)
  auto read_T = [&](int v, const uint8_t* slot_raw, float4 (&u)[T_PER_THREAD][2]) {
#pragma unroll
    for (int k = 0; k < T_PER_THREAD; ++k)
      if (v + 64 * k < T_CHUNKS) load_chunk(v + 64 * k, slot_raw, u[k][0], u[k][1]);
  };
  auto store_T = [&](int v, const float4 (&u)[T_PER_THREAD][2], uint8_t* tdst) {
#pragma unroll
    for (int k = 0; k < T_PER_THREAD; ++k)
      if (v + 64 * k < T_CHUNKS) store_chunk(v + 64 * k, u[k][0], u[k][1], tdst);
  };
  // On the bf16 path the first column tile's matrices are split by the converter and the
  // epilogue warps together (warps 2-11, at most two chunks per thread): the first MMA
  // waits for this split, and the epilogue has nothing to do before the first
  // accumulator lands.  Both roles call it exactly once; the named barriers are reached
  // whether or not the copy arrived in time.
  constexpr int NC0 = 320;
  constexpr int PER0 = (T_CHUNKS + NC0 - 1) / NC0;
  auto first_split = [&]() -> bool {
    const int c0 = static_cast<int>(threadIdx.x) - 64;
    uint8_t* tdst = smem + Cfg::OFF_T;
    const bool ok = wait_bounded(BAR(B_TLOAD), 0u, abort_flag, 4u, lim);
    float4 u[PER0][2];
#pragma unroll
    for (int k = 0; k < PER0; ++k)
      if (ok && c0 + NC0 * k < T_CHUNKS) load_chunk(c0 + NC0 * k, tdst, u[k][0], u[k][1]);
    named_bar_sync(4, NC0);   // every raw chunk is in registers before any panel overwrites it
#pragma unroll
    for (int k = 0; k < PER0; ++k)
      if (ok && c0 + NC0 * k < T_CHUNKS) store_chunk(c0 + NC0 * k, u[k][0], u[k][1], tdst);
    fence_proxy_async_smem();
    named_bar_sync(4, NC0);   // the panels are complete
    return ok;
  };
  // Thread 0, which initialised the barriers, issues the first input tile, then the
  // transform copies of the CTA's first (and, if its tiles reach it, second) column tile,
  // then the second input tile; the producer loop issues the other stages after the
  // set-up (this order and depth measured fastest: the first tile and its matrices
  // arrive ahead of the rest of the burst).  Every converter thread knows which copies
  // exist.
  const int ct_first = tile_at(t_begin) / nrt;        // the run's first column tile
  const bool t_second = !Cfg::SHARED_T && t_begin < t_end && tile_at(t_end - 1) / nrt != ct_first;
  int t_issued[2] = {t_begin < t_end ? 1 : 0, t_second ? 1 : 0};
  const uint64_t l2_pol = l2_policy_evict_first();
  int n_preloaded = 0;
  if (threadIdx.x == 0) {
    auto issue_x = [&]() {
      if (n_preloaded < STAGES && t_begin + n_preloaded < t_end) {
        const int t = tile_at(t_begin + n_preloaded);
        const int ct = t / nrt, rt = t - ct * nrt;
        const uint32_t dst = sbase + Cfg::OFF_STAGE + n_preloaded * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(BAR(B_FULL + n_preloaded), Cfg::STAGE_BYTES);
#pragma unroll
        for (int s = 0; s < Cfg::SUB; ++s)
          tma_load_2d(dst + s * 16384, &tmap_in, BAR(B_FULL + n_preloaded), ct * CH + 64 * s, rt * 128, l2_pol);
        ++n_preloaded;
      }
    };
    issue_x();
    if (t_begin < t_end) t_copy(ct_first, 0);
    if (t_second) t_copy(REV ? ct_first - 1 : ct_first + 1, 1);
    while (n_preloaded < 2 && t_begin + n_preloaded < t_end) issue_x();   // the rest after the set-up
  }
  __syncwarp();
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
      const uint64_t pol = l2_pol;
      int n_loaded = n_preloaded;
      int stage = n_preloaded % STAGES;
      uint32_t phase = n_preloaded == STAGES ? 1u : 0u;
      for (int i = n_preloaded; i < walk_len; ++i) {
        if (!wait_bounded(BAR(B_EMPTY + stage), phase ^ 1u, abort_flag, 1u, lim)) break;
        const int tt = tile_at(walk_tile(i));
        const int ct = tt / nrt, rt = tt - ct * nrt;
        const uint32_t dst = sbase + Cfg::OFF_STAGE + stage * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(BAR(B_FULL + stage), Cfg::STAGE_BYTES);
        if (Cfg::IN_F32) {
          tma_load_2d(dst, &tmap_in, BAR(B_FULL + stage), ct * CH, rt * 128, pol);
        } else {
#pragma unroll
          for (int s = 0; s < Cfg::SUB; ++s)
            tma_load_2d(dst + s * 16384, &tmap_in, BAR(B_FULL + stage), ct * CH + 64 * s, rt * 128, pol);
        }
        ++n_loaded;
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
      if (*abort_flag) {  // let the copies still in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int k = (n_loaded > STAGES ? n_loaded - STAGES : 0); k < n_loaded; ++k)
          wait_bounded(BAR(B_FULL + k % STAGES), static_cast<uint32_t>((k / STAGES) & 1), &no_abort, 16u, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // This thread's wait -> issue -> commit chain bounds the tile rate, so it carries as
    // little arithmetic as possible: operand descriptors, barrier addresses and the
    // accumulator column advance incrementally, and on the bf16 path the epilogue (not
    // this thread) frees the input stage once it has seen the tile's accumulator land.
    if (lane == 0) {
      constexpr uint32_t idesc_hl = idesc_bf16_f32(128, 2 * G);   // hi|lo stacked along N
      constexpr uint32_t idesc_h = idesc_bf16_f32(128, G);        // hi only
      constexpr int NBUF = Cfg::IN_F32 ? 2 : STAGES;                // operand buffers cycled through
      constexpr uint32_t A_STEP = (Cfg::IN_F32 ? 2 * Cfg::OPER_BYTES : Cfg::STAGE_BYTES) >> 4;
      const uint64_t da_first = desc_k_sw128(sbase + (Cfg::IN_F32 ? Cfg::OFF_OPER : Cfg::OFF_STAGE));
      const uint64_t db_slot0 = desc_k_sw128(sbase + Cfg::OFF_T);
      const uint32_t full_first = BAR(Cfg::IN_F32 ? B_OFULL : B_FULL);
      int buf = 0;
      uint32_t phase = 0;
      uint64_t da_hi = da_first;
      uint32_t full_bar = full_first;
      int epoch = -1, prev_ct = -1;
      int it = 0;
      int ct = ct_first, rt = tile_at(t_begin) - ct_first * nrt;
      uint64_t db = db_slot0;
      for (int t = t_begin; t < (ONEPASS ? t_begin + walk_len : t_end); ++t, ++it) {
        if constexpr (ONEPASS) {   // coordinates from the walk (this mode is not the hot loop)
          const int tw = walk_tile(it);
          ct = tw / nrt;
          rt = tw - ct * nrt;
        }
        if (Cfg::SHARED_T ? it == 0 : ct != prev_ct) {
          ++epoch;
          prev_ct = ct;
          db = db_slot0 + ((epoch & 1) ? static_cast<uint64_t>(Cfg::TSLOT_BYTES >> 4) : 0ull);
          if (!wait_bounded(BAR(B_TFULL + (epoch & 1)), static_cast<uint32_t>((epoch >> 1) & 1), abort_flag, 2u, lim)) break;
        }
        const int acc = it & (NACC - 1);
        if (!wait_bounded(full_bar, phase, abort_flag, 2u, lim)) break;
        if (!wait_bounded(BAR(B_AEMPTY + acc), static_cast<uint32_t>(((it / NACC) & 1) ^ 1), abort_flag, 2u, lim)) break;
        tc_fence_after();
        const uint64_t da_lo = da_hi + (Cfg::OPER_BYTES >> 4);
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(acc * Cfg::ACC_COLS);
#pragma unroll
        for (int b = 0; b < BPT; ++b) {
          // A: block b occupies bytes [b*2G, b*2G + 2G) of the 128-byte rows of sub-tile (b*G)/64
          const uint32_t a_off = static_cast<uint32_t>(((b * G) / 64) * 16384 + ((b * G) % 64) * 2);
          // B: panel b / BPP, K bytes [(b % BPP) * 2G, +2G) of its 2G rows (hi rows, then lo rows)
          const uint32_t p_off = static_cast<uint32_t>((b / Cfg::BPP) * Cfg::PANEL_BYTES + (b % Cfg::BPP) * 2 * G);
#pragma unroll
          for (int kk = 0; kk < G / 16; ++kk) {
            const uint64_t bd = db + ((p_off + kk * 32) >> 4);
            umma_bf16(d0 + static_cast<uint32_t>(b * 2 * G), da_hi + ((a_off + kk * 32) >> 4), bd, idesc_hl,
                      kk > 0 ? 1u : 0u);
            if (Cfg::IN_F32)
              umma_bf16(d0 + static_cast<uint32_t>(b * 2 * G), da_lo + ((a_off + kk * 32) >> 4), bd, idesc_h, 1u);
          }
        }
        umma_commit(BAR(B_AFULL + acc));
        if (Cfg::IN_F32) umma_commit(BAR(B_OEMPTY + buf));
        if constexpr (ONEPASS) {   // the slot is free once the walk leaves its column tile
          if (it + 1 == walk_len || walk_tile(it + 1) / nrt != ct) umma_commit(BAR(B_TEMPTY + (epoch & 1)));
        } else if (!Cfg::SHARED_T && (t + 1 == t_end || (REV ? rt == 0 : rt + 1 == nrt))) {
          umma_commit(BAR(B_TEMPTY + (epoch & 1)));
        }
        if constexpr (REV) {
          if (rt-- == 0) rt = nrt - 1, --ct;
        } else {
          if (++rt == nrt) rt = 0, ++ct;
        }
        if (++buf == NBUF) {
          buf = 0, phase ^= 1u, da_hi = da_first, full_bar = full_first;
        } else {
          da_hi += A_STEP, full_bar += 8u;
        }
      }
      // every MMA issued above has finished before TMEM can be released
      umma_commit(BAR(B_DRAIN));
      volatile int no_abort = 0;
      wait_bounded(BAR(B_DRAIN), 0u, &no_abort, 16u, lim);
    }
  } else if (warp < 4 || (Cfg::IN_F32 && warp >= 8)) {
    // ------------------------------------------------------------ converters
    // warps 2-3 (ids 0..63) split the transforms; on the fp32 path warps 2-3 and 8-11
    // (ids 0..191) split the input tiles
    const int v0 = warp < 4 ? threadIdx.x - 64 : 64 + (threadIdx.x - 256);
    const bool t_conv = v0 < 64;
    int t_landed[2] = {0, 0};
    int epoch = -1, prev_ct = -1;
    int stage = 0, obuf = 0;
    uint32_t phase = 0, ophase = 0;
    bool conv_ok = true;
    if (!Cfg::IN_F32 && t_begin < t_end) {
      conv_ok = first_split();
      // the split kept the slot's read-done barrier out of it: arrive on it here so that
      // its phases stay in step with the slot's later refills (a third column tile of the
      // walk lands in slot 0 again and waits on that barrier's next phase)
      mbar_arrive(BAR(B_TREAD));
      if (conv_ok) {
        mbar_arrive(BAR(B_TFULL));   // slot 0 holds the first column tile's panels
        t_landed[0] = 1;
        epoch = 0;
        prev_ct = ct_first;
      }
    }
    for (int i = 0; conv_ok && i < walk_len; ++i) {
      const int ct = tile_at(walk_tile(i)) / nrt;
      if (t_conv && (Cfg::SHARED_T ? epoch < 0 : ct != prev_ct)) {
        ++epoch;
        prev_ct = ct;
        const int slot = epoch & 1;
        uint8_t* tdst = smem + Cfg::OFF_T + slot * Cfg::TSLOT_BYTES;
        const uint32_t par = static_cast<uint32_t>((epoch >> 1) & 1);
        if (epoch >= 2) {     // the first two copies were issued at the start
          if (!wait_bounded(BAR(B_TEMPTY + slot), par ^ 1u, abort_flag, 4u, lim)) break;
          if (v0 == 0) t_copy(ct, slot), ++t_issued[slot];
        }
        if (!wait_bounded(BAR(B_TLOAD + slot), par, abort_flag, 4u, lim)) break;
        ++t_landed[slot];
        float4 u[T_PER_THREAD][2];
        read_T(v0, tdst, u);
        // every raw chunk of the slot is in registers before any panel overwrites it
        mbar_arrive(BAR(B_TREAD + slot));
        if (!wait_bounded(BAR(B_TREAD + slot), par, abort_flag, 4u, lim)) break;
        store_T(v0, u, tdst);
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
        constexpr int PER = (128 * CPR + Cfg::CONV_THREADS - 1) / Cfg::CONV_THREADS;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int q = v0 + k * Cfg::CONV_THREADS;
          if (q >= 128 * CPR) break;
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
    if (v0 == 0) {   // an aborted run still lets its transform copies land before the CTA exits
      volatile int no_abort = 0;
      for (int sl = 0; sl < 2; ++sl)
        for (; t_landed[sl] < t_issued[sl]; ++t_landed[sl])
          wait_bounded(BAR(B_TLOAD + sl), static_cast<uint32_t>(t_landed[sl] & 1), &no_abort, 4u, lim);
    }
  } else {
    // ------------------------------------------------------------ epilogue: 2 groups x 4 warps
    // Group g takes the tiles with local index = g (mod 2) and the accumulator buffers of
    // those tiles; the groups run independently, so one group's TMEM loads, barrier and
    // store overlap the other group's arithmetic.  Thread = token row of the tile; it
    // handles the tile's blocks one after the other.
    const int grp = (warp - 4) >> 2;           // epilogue group (warps 4-7: 0, 8-11: 1)
    const int quad = warp & 3;                 // TMEM lanes this warp may read
    const int row = quad * 32 + lane;          // row within the tile
    const bool store_leader = (quad == 0) && lane == 0;
    const int C = p.C;
    const int code_row_bytes = p.d_in / 2;
    const bool vec16 = (code_row_bytes % 16) == 0;
    using ScaleT = typename std::conditional<Cfg::FMT == kINT4, float, uint8_t>::type;
    if (!Cfg::IN_F32 && t_begin < t_end) first_split();   // with the converter warps
    const float inv7 = __frcp_rn(7.0f);   // INT4: RN(1/7)
    float s_t = 0.0f, d6 = 0.0f, inv_d6 = 0.0f;
    bool exact_div = true;
    float* nv_tab = reinterpret_cast<float*>(smem + Cfg::OFF_NVTAB);
    if constexpr (Cfg::FMT == kNVFP4 && !Cfg::AMAX_ONLY && !ONEPASS) {
      s_t = *p.tensor_scale;
      d6 = __fmul_rn(6.0f, s_t);
      inv_d6 = d6 > 0.0f ? __frcp_rn(d6) : 0.0f;
      exact_div = !(inv_d6 >= 1.17549435e-38f && inv_d6 <= 3.40282347e+38f);   // not a normal fp32
      // the 128 block-scale reciprocals, one per thread of the first 128 epilogue threads
      const int e_tid = threadIdx.x - 128;
      if (e_tid < 128) {
        const float S = __fmul_rn(e4m3_value(static_cast<uint32_t>(e_tid)), s_t);
        float inv = S > 0.0f ? __frcp_rn(S) : 0.0f;
        if (isinf(inv)) inv = 0.0f;
        nv_tab[e_tid] = inv;
      }
      named_bar_sync(3, 128 * Cfg::N_GROUPS);   // the table is complete
    }
    bool live = true;
    float run_max = 0.0f;
    int m = 0;                                  // tiles handled by this group so far
    int it_first = grp;
    bool met = false;                           // ONEPASS, thread 128: the grid has met
    if constexpr (ONEPASS) {
      // ---- first half of the walk: max |y| over this CTA's run
      for (int it = grp; it < run_len; it += Cfg::N_GROUPS) {
        const int t = tile_at(walk_tile(it));
        const int ct = t / nrt, rt = t - ct * nrt;
        const int acc = it % NACC;
        if (live && !wait_bounded(BAR(B_AFULL + acc), static_cast<uint32_t>((it / NACC) & 1), abort_flag, 8u, lim))
          live = false;
        if (quad == 0 && lane == 0 && live) mbar_arrive(BAR(B_EMPTY + it % STAGES));
        const bool warp_live = __all_sync(0xffffffffu, live) && !*abort_flag;
        const bool row_ok = static_cast<long long>(rt) * 128 + row < p.n_rows;
        const uint32_t tq = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * Cfg::ACC_COLS);
        if (warp_live) tc_fence_after();
        constexpr int BPL = 32 / G;
#pragma unroll
        for (int bl = 0; bl < BPT / BPL; ++bl) {
          float hl[64];
          if (warp_live) tmem_ld64_sync(tq + static_cast<uint32_t>(bl * 64), hl);
          if (bl == BPT / BPL - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(B_AEMPTY + acc));
          }
          if (!warp_live) continue;
#pragma unroll
          for (int u = 0; u < BPL; ++u) {
            float* v = hl + u * 2 * G;
#pragma unroll
            for (int jj = 0; jj < G; jj += 2) add2_rn(v[jj], v[jj + 1], v[G + jj], v[G + jj + 1]);  // hi + lo
            if (row_ok && ct * BPT + bl * BPL + u < C) run_max = fmaxf(run_max, group_absmax<G>(v));
          }
        }
      }
      // ---- the grid's maximum: one value per CTA into the workspace, then wait for all
      // CTAs (they are resident together: cooperative launch), bounded in time
      float* scratch = nv_tab;                   // the table is filled only after this
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) run_max = fmaxf(run_max, __shfl_xor_sync(0xffffffffu, run_max, o));
      if (lane == 0) scratch[warp - 4] = run_max;
      named_bar_sync(5, 128 * Cfg::N_GROUPS);
      if (threadIdx.x == 128) {
        unsigned int* ws = p.amax_word;          // [0] max bits, [1] arrivals, [2] departures
        float cm = scratch[0];
        for (int w = 1; w < 4 * Cfg::N_GROUPS; ++w) cm = fmaxf(cm, scratch[w]);
        const unsigned int grid = gridDim.x;
        if (cm > 0.0f) atomicMax(&ws[0], __float_as_uint(cm));
        red_add_release_gpu(&ws[1]);             // the maximum above is ordered before the count
        const uint64_t t0 = global_timer_ns();
        int ok = 1;
        while (ld_acquire_gpu(&ws[1]) < grid) {
          __nanosleep(100);
          if (global_timer_ns() - t0 > lim) {     // a CTA never arrived
            atomicOr(&g_wush_device_error, 128u);
            ok = 0;
            break;
          }
        }
        // the acquire poll above ordered this read after every CTA's maximum; a load, not an
        // atomic: the whole grid reads the word at once here
        const float amax = __uint_as_float(ld_acquire_gpu(&ws[0]));
        met = ok != 0;
        const float st = __fdiv_rn(amax, 2688.0f);
        if (ok && blockIdx.x == 0) *const_cast<float*>(p.tensor_scale) = st;
        scratch[8] = st;
        scratch[9] = ok ? 1.0f : 0.0f;
      }
      named_bar_sync(5, 128 * Cfg::N_GROUPS);
      s_t = scratch[8];
      if (scratch[9] == 0.0f) live = false;
      named_bar_sync(5, 128 * Cfg::N_GROUPS);   // read before the table overwrites them
      d6 = __fmul_rn(6.0f, s_t);
      inv_d6 = d6 > 0.0f ? __frcp_rn(d6) : 0.0f;
      exact_div = !(inv_d6 >= 1.17549435e-38f && inv_d6 <= 3.40282347e+38f);
      const int e_tid = threadIdx.x - 128;
      if (e_tid < 128) {
        const float S = __fmul_rn(e4m3_value(static_cast<uint32_t>(e_tid)), s_t);
        float inv = S > 0.0f ? __frcp_rn(S) : 0.0f;
        if (isinf(inv)) inv = 0.0f;
        nv_tab[e_tid] = inv;
      }
      named_bar_sync(5, 128 * Cfg::N_GROUPS);   // the table is complete
      // ---- second half of the walk: quantise, backwards
      it_first = run_len + ((grp ^ run_len) & 1);
    }
    for (int it = it_first; it < walk_len; it += Cfg::N_GROUPS, ++m) {
      const int t = tile_at(walk_tile(it));
      const int ct = t / nrt, rt = t - ct * nrt;
      const int acc = it % NACC;
      if (live && !wait_bounded(BAR(B_AFULL + acc), static_cast<uint32_t>((it / NACC) & 1), abort_flag, 8u, lim))
        live = false;
      // bf16 path: the accumulator has landed, so the MMAs that read this tile's input
      // stage are done; hand the stage back to the producer
      if (!Cfg::IN_F32 && quad == 0 && lane == 0 && live) mbar_arrive(BAR(B_EMPTY + it % STAGES));
      const bool warp_live = __all_sync(0xffffffffu, live) && !*abort_flag;
      const long long grow = static_cast<long long>(rt) * 128 + row;
      const bool row_ok = grow < p.n_rows;
      uint8_t* cstage = smem + Cfg::OFF_CODES + (grp * 2 + (m & 1)) * Cfg::CODE_STAGE;
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * Cfg::ACC_COLS);
      ScaleT sc[BPT];
      if (warp_live) tc_fence_after();
      // one 64-column TMEM load per step: one G = 32 block, or two G = 16 blocks whose
      // quantisation chains are independent, so the scheduler can interleave them
      constexpr int BPL = 32 / G;                     // blocks per load
#pragma unroll
      for (int bl = 0; bl < BPT / BPL; ++bl) {
        float hl[64];
        if (warp_live) tmem_ld64_sync(tq + static_cast<uint32_t>(bl * 64), hl);
        if (bl == BPT / BPL - 1) {      // the whole accumulator buffer has been read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(B_AEMPTY + acc));
        }
        if (!warp_live) continue;
#pragma unroll
        for (int u = 0; u < BPL; ++u) {
          float* v = hl + u * 2 * G;
#pragma unroll
          for (int jj = 0; jj < G; jj += 2) add2_rn(v[jj], v[jj + 1], v[G + jj], v[G + jj + 1]);  // hi + lo
        }
        if constexpr (Cfg::AMAX_ONLY) {
#pragma unroll
          for (int u = 0; u < BPL; ++u)
            if (row_ok && ct * BPT + bl * BPL + u < C) run_max = fmaxf(run_max, group_absmax<G>(hl + u * 2 * G));
        } else {
          uint32_t words[BPL][G / 8];
#pragma unroll
          for (int u = 0; u < BPL; ++u) {
            const float* v = hl + u * 2 * G;
            const int b = bl * BPL + u;
            const int blk = ct * BPT + b;
            if (Cfg::EMIT_Y && row_ok && blk < C) {
              float4* yd = reinterpret_cast<float4*>(p.y_out + grow * p.d_in + static_cast<long long>(blk) * G);
#pragma unroll
              for (int k = 0; k < G / 4; ++k) yd[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
            if (Cfg::FMT == kMXFP4) sc[b] = static_cast<ScaleT>(quant_mx<G>(v, words[u]));
            else if (Cfg::FMT == kNVFP4) sc[b] = static_cast<ScaleT>(quant_nv_tab<G>(v, d6, inv_d6, exact_div, nv_tab, words[u]));
            else sc[b] = static_cast<ScaleT>(quant_int4_fast<G>(v, inv7, words[u]));
          }
          // the load's 32 elements are one 16-byte chunk of this row's codes
          const int pc = bl ^ ((row >> SW_SHIFT) & (NCH - 1));
          const uint32_t* w = &words[0][0];
          *reinterpret_cast<uint4*>(cstage + row * (CH / 2) + pc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (Cfg::AMAX_ONLY) continue;
      // scales: this thread's row of the tile, straight from registers
      if (Cfg::FMT != kINT4 && p.scale_atoms) {
        // scale-atom layout: row 128 r + i + 32 j, scale column 4 c + k at byte
        // (r * atom_cols + c) * 512 + 16 i + 4 j + k; each aligned group of four of this
        // tile's columns is one 32-bit word of an atom
        if (warp_live && row_ok) {
          const int col0 = ct * BPT;
          const int rr = static_cast<int>(grow & 127);
          uint8_t* row_base = static_cast<uint8_t*>(p.scales) + (grow >> 7) * p.atom_cols * 512 + (rr & 31) * 16 +
                              (rr >> 5) * 4;
          const int nb = min(BPT, C - col0);
          if constexpr (BPT % 4 == 0) {
#pragma unroll
            for (int w4 = 0; w4 < BPT / 4; ++w4) {
              uint8_t* word = row_base + ((col0 >> 2) + w4) * 512;
              if (4 * w4 + 4 <= nb) {
                *reinterpret_cast<uint32_t*>(word) =
                    static_cast<uint32_t>(sc[4 * w4]) | (static_cast<uint32_t>(sc[4 * w4 + 1]) << 8) |
                    (static_cast<uint32_t>(sc[4 * w4 + 2]) << 16) | (static_cast<uint32_t>(sc[4 * w4 + 3]) << 24);
              } else {
#pragma unroll
                for (int k = 4 * w4; k < 4 * w4 + 4; ++k)   // compile-time indices keep sc in registers
                  if (k < nb) word[k - 4 * w4] = static_cast<uint8_t>(sc[k]);
              }
            }
          } else {
#pragma unroll
            for (int k = 0; k < BPT; ++k)
              if (k < nb) row_base[((col0 + k) >> 2) * 512 + ((col0 + k) & 3)] = static_cast<uint8_t>(sc[k]);
          }
        }
      } else if (warp_live && row_ok) {
        const int nb = min(BPT, C - ct * BPT);
        ScaleT* dst = reinterpret_cast<ScaleT*>(p.scales) + grow * C + static_cast<long long>(ct) * BPT;
        constexpr int RB = BPT * static_cast<int>(sizeof(ScaleT));   // 2..32 bytes
        if (nb == BPT && (reinterpret_cast<uintptr_t>(dst) % (RB >= 16 ? 16 : RB)) == 0) {
          if constexpr (RB == 2) {
            *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(sc[0] | (sc[1] << 8));
          } else if constexpr (RB == 4 && sizeof(ScaleT) == 1) {
            *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(sc[0]) | (static_cast<uint32_t>(sc[1]) << 8) |
                                                (static_cast<uint32_t>(sc[2]) << 16) | (static_cast<uint32_t>(sc[3]) << 24);
          } else if constexpr (RB == 8 && sizeof(ScaleT) == 1) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) lo |= static_cast<uint32_t>(sc[k]) << (8 * k), hi |= static_cast<uint32_t>(sc[4 + k]) << (8 * k);
            *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
          } else if constexpr (sizeof(ScaleT) == 4 && RB % 16 == 0) {
#pragma unroll
            for (int k = 0; k < BPT / 4; ++k)
              reinterpret_cast<float4*>(dst)[k] = make_float4(sc[4 * k], sc[4 * k + 1], sc[4 * k + 2], sc[4 * k + 3]);
          } else {
#pragma unroll
            for (int k = 0; k < BPT; ++k) dst[k] = sc[k];
          }
        } else {
#pragma unroll
          for (int k = 0; k < BPT; ++k)
            if (k < nb) dst[k] = sc[k];
        }
      }
      if (warp_live && p.codes_via_tma) fence_proxy_async_smem();
      // the buffer this group writes next time was stored one group-tile ago: make sure
      // that store has read it before anyone of the group moves past this barrier
      if (store_leader && p.codes_via_tma) bulk_wait_read_all();
      named_bar_sync(1 + grp, 128);  // the tile's codes are staged
      if (!warp_live) continue;
      if (p.codes_via_tma) {
        if (store_leader) {
          tma_store_2d(&tmap_codes, smem_addr(cstage), ct * (CH / 2), rt * 128);
          bulk_commit_group();
        }
      } else {
        // consecutive threads of the group write consecutive 16-byte chunks of a row
        const int gtid = quad * 32 + lane;
        const long long col0 = static_cast<long long>(ct) * (CH / 2);
#pragma unroll
        for (int c = gtid; c < 128 * NCH; c += 128) {
          const int r = c / NCH, q = c - r * NCH;
          const long long gr = static_cast<long long>(rt) * 128 + r;
          const long long gc = col0 + q * 16;
          if (gr >= p.n_rows || gc >= code_row_bytes) continue;
          const uint4 val = *reinterpret_cast<const uint4*>(cstage + r * (CH / 2) + ((q ^ ((r >> SW_SHIFT) & (NCH - 1))) << 4));
          uint8_t* dst = p.codes + gr * code_row_bytes + gc;
          if (vec16 && gc + 16 <= code_row_bytes) {
            *reinterpret_cast<uint4*>(dst) = val;
          } else {
            *reinterpret_cast<uint2*>(dst) = make_uint2(val.x, val.y);
            if (gc + 8 < code_row_bytes) *reinterpret_cast<uint2*>(dst + 8) = make_uint2(val.z, val.w);
          }
        }
      }
    }
    if (Cfg::AMAX_ONLY) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) run_max = fmaxf(run_max, __shfl_xor_sync(0xffffffffu, run_max, o));
      if (lane == 0 && run_max > 0.0f) atomicMax(p.amax_word, __float_as_uint(run_max));
    }
    // the last stores must have read their staging buffers before the CTA's shared
    // memory goes away; their global writes complete with the grid
    if (store_leader && p.codes_via_tma) bulk_wait_read_all();
    if constexpr (ONEPASS) {
      // this CTA read the maximum long ago; the last one to leave puts the workspace back
      // to zero.  Counting departures here rather than right after the meeting spreads the
      // grid's atomics on ws[2] over the CTAs' different finishing times.
      if (threadIdx.x == 128 && met) {
        unsigned int* ws = p.amax_word;
        if (atomicAdd(&ws[2], 1u) == gridDim.x - 1) {
          ws[0] = 0u;
          ws[1] = 0u;
          ws[2] = 0u;
          __threadfence();
        }
      }
    }
  }

  // Every warp reconverges before the CTA-wide barrier: the producer and MMA roles ran on
  // one lane, and an aligned barrier reached by a diverged warp did not hold the late
  // lane's warp-mates back (observed on B200: the producer lane passed it while the
  // epilogue warps were still at work).  TMEM is released only after every warp, the
  // epilogue's last accumulator reads included, has passed it.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// NVFP4: turn the running |y| maximum (float bits) into the fp32 tensor scale
// s_t = amax / (6 * 448), in place.
// Both one-thread kernels below wait for the previous kernel in the stream before touching
// the word (a no-op unless launched with programmatic stream serialisation) and then let
// the next kernel start its set-up.
__global__ void wush_nvfp4_tensor_scale_kernel(float* tensor_scale) {
  grid_dependency_wait();
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(tensor_scale));
    *tensor_scale = __fdiv_rn(amax, 2688.0f);
  }
  grid_launch_dependents();
}

// Clears the running-max word of the NVFP4 amax pass.
__global__ void wush_nvfp4_amax_reset_kernel(float* word) {
  grid_dependency_wait();
  if (threadIdx.x == 0 && blockIdx.x == 0) *word = 0.0f;
  grid_launch_dependents();
}

}  // namespace wush
