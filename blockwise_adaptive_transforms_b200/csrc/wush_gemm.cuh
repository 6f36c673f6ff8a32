// Block-scaled FP4 x FP4 -> bf16 GEMM for sm_100a on tcgen05 MMAs: the consumer of the
// quantised operands (the pages' "WUSH + Quant + FP4 MatMul" layer: paper-graph-ui
// analysis, section 3.4.7 "GPU Kernel Design" and section 5 "GPU Kernel Benchmarks
// (Figure 2)").
//
//   D[m][n] = alpha * sum_k A[m][k] * B[n][k]
//
// A (activations, M rows) and B (weights, N rows = output channels) are E2M1 codes packed
// two per byte along K (low nibble = even k).  MXFP4: each 32-element group has an E8M0
// scale and alpha = 1.  NVFP4: each 16-element group has an E4M3 scale and alpha is the
// product of the two fp32 tensor scales.  The scales are read in the layout the
// block-scaled MMA consumes ("tcgen05 scale atoms"): for rows [128 r, 128 r + 128) and
// scale columns [4 c, 4 c + 4) one 512-byte atom at byte (r * (C / 4) + c) * 512, in which
// row 128 r + i + 32 j, scale 4 c + k sits at byte 16 i + 4 j + k (i < 32, j < 4, k < 4).
//
// Tiles of 128 x 256 outputs, 256 K-elements (128 bytes of codes per row) per pipeline
// stage; per stage the producer brings A (16 KB) and B (32 KB) by TMA with 128-byte
// swizzle and the stage's scale atoms (A: 2 (MX) or 4 (NV); B: twice that, for its two
// 128-row halves) by bulk copies; four scale warps, one per TMEM lane quadrant, write the
// atoms into the stage's TMEM scale slot with tcgen05.st (each quadrant receives the same
// 32 rows of 16 bytes, the layout a 32x128b.warpx4 copy would give), so that no copy sits
// in the MMA issue queue; the MMA thread waits for them and issues four M=128, N=256, K=64
// MMAs (kind::mxf4 block32, or kind::mxf4nvf4 block16); four epilogue warps read the fp32
// accumulator (tcgen05.ld), scale by alpha, round to bf16 and store through shared memory
// and TMA.  Persistent CTAs, one per SM.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "wush_ptx.cuh"

namespace wush {

struct GemmParams {
  const uint8_t* sfa;        // A scale atoms
  const uint8_t* sfb;        // B scale atoms
  const float* ts_a;         // NVFP4: A's fp32 tensor scale (device)
  const float* ts_b;         // NVFP4: B's fp32 tensor scale (device)
  __nv_bfloat16* d;          // [M][N]
  int M, N, K;
  int tiles_m, tiles_n;
  unsigned long long wait_limit_ns;
};

// NV = false: MXFP4 (E8M0 scales per 32 elements, kind::mxf4 block32);
// NV = true:  NVFP4 (E4M3 scales per 16 elements, kind::mxf4nvf4 block16, times the two
//             fp32 tensor scales in the epilogue).
template <bool NV_>
struct GemmCfg {
  static constexpr bool NV = NV_;
  static constexpr int VS = NV ? 16 : 32;              // elements per scale
  static constexpr int BM = 128, BN = 256, BK = 256;   // BK in elements (128 bytes of codes)
  static constexpr int STAGES = 4;
  static constexpr int ATOM_K = 4 * VS;                // K elements one scale atom covers
  static constexpr int ATOMS_PER_STAGE = BK / ATOM_K;  // MX 2, NV 4
  static constexpr int A_BYTES = BM * BK / 2;          // 16 KB
  static constexpr int B_BYTES = BN * BK / 2;          // 32 KB
  static constexpr int SFA_BYTES = ATOMS_PER_STAGE * 512;          // one atom per K chunk
  static constexpr int SFB_BYTES = 2 * ATOMS_PER_STAGE * 512;      // and per 128-row half
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int OFF_A = 0, OFF_B = A_BYTES, OFF_SFA = A_BYTES + B_BYTES, OFF_SFB = OFF_SFA + SFA_BYTES;
  // output staging: 128 rows x D_COLS bf16, 128-byte (MX) or 64-byte (NV: its larger scale
  // atoms leave room for half the width) swizzle
  static constexpr int D_COLS = NV ? 32 : 64;
  static constexpr int OFF_D = STAGES * STAGE_BYTES;
  static constexpr int D_BYTES = BM * D_COLS * 2;
  static constexpr int OFF_BAR = OFF_D + D_BYTES;
  static constexpr int N_BARS = 3 * STAGES + 3;        // full[S], empty[S], afull, aempty, drain, scales[S]
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static constexpr int THREADS = 12 * 32;  // producer, MMA, 2 idle, 4 epilogue, 4 scale warps
  // TMEM: accumulator columns [0, 256); per stage slot the scale columns from 256: A atom
  // a at +4a, B atom a of half h at +4 * ATOMS_PER_STAGE + 8a + 4h
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 256, SFB_COL = 4 * ATOMS_PER_STAGE, SF_SLOT_COLS = 12 * ATOMS_PER_STAGE;
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SF_COL0 + STAGES * SF_SLOT_COLS <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Instruction descriptor of the block-scaled FP4 MMAs (kind::mxf4 / kind::mxf4nvf4):
// E2M1 A and B (format 1), K-major, scale type in bit 23 (1 = E8M0, 0 = UE4M3),
// M = 128, N = 256, dense K = 64; the scale-factor ids (bits 29-30 for A, 4-5 for B)
// select the byte of the TMEM word the first scale sits in (always 0 for block16, whose
// four scales fill the word).
__device__ __forceinline__ uint32_t idesc_mxf4(int M, int N, uint32_t sf_id, bool e8m0) {
  return (sf_id << 4)                               // B scale-factor id
         | (1u << 7)                                // A format: E2M1
         | (1u << 10)                               // B format: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | ((e8m0 ? 1u : 0u) << 23)                 // scale format: E8M0 or UE4M3
         | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
         | (sf_id << 29);                           // A scale-factor id
}

__device__ __forceinline__ void umma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared-memory descriptor of one scale atom (32 rows x 16 bytes, rows contiguous, no
// swizzle): 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);   // start address
  d |= static_cast<uint64_t>(1) << 16;                     // leading byte offset (one core matrix wide)
  d |= static_cast<uint64_t>(128 >> 4) << 32;              // stride byte offset: 8 rows x 16 B
  d |= static_cast<uint64_t>(1) << 46;                     // descriptor version for sm_100
  return d;                                                // layout type 0: no swizzle
}

// Four consecutive 32-bit TMEM columns of this thread's lane (in its warp's lane
// quadrant) from registers; tmem_wait_st waits for the thread's stores to land.
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One stage's scale atoms from shared memory into this warp's lane quadrant of the
// stage's TMEM scale slot: A atom a at columns +4a, B atom a of half h at
// +SFB_COL + 8a + 4h, lane i of the quadrant taking row i (16 bytes) of each atom.
template <class Cfg>
__device__ __forceinline__ void write_scale_slot(uint32_t slot_taddr, const uint8_t* st, int lane) {
#pragma unroll
  for (int a = 0; a < Cfg::ATOMS_PER_STAGE; ++a) {
    tmem_st_x4(slot_taddr + 4 * a, *reinterpret_cast<const uint4*>(st + Cfg::OFF_SFA + a * 512 + 16 * lane));
#pragma unroll
    for (int h = 0; h < 2; ++h)
      tmem_st_x4(slot_taddr + Cfg::SFB_COL + 8 * a + 4 * h,
                 *reinterpret_cast<const uint4*>(st + Cfg::OFF_SFB + h * Cfg::ATOMS_PER_STAGE * 512 + a * 512 +
                                                 16 * lane));
  }
  tmem_wait_st();
}

// Epilogue of one 128 x BN accumulator by four warps (quad = warp & 3 = TMEM lane
// quadrant; thread = row 32 quad + lane).  Each D_COLS-column slice goes from TMEM to
// bf16 (times alpha), into the shared-memory staging buffer in the swizzle the store's
// tensor map names, and out by one TMA store to columns [x0 + D_COLS q, ...) of rows
// [y0, y0 + 128), issued by the first thread once all four warps have written; the
// buffer is rewritten only after the previous store has read it.  release() runs in
// every warp once its last slice is in registers (the accumulator may be overwritten).
// Every thread of the four warps reaches the same named barriers, live or not.
template <class Cfg, class Release>
__device__ __forceinline__ void epilogue_tile(uint32_t tmem_base, int quad, int lane, bool warp_live, float alpha,
                                              uint8_t* dstage, const CUtensorMap* tmap_d, int x0, int y0,
                                              volatile int* abort_flag, Release release) {
  constexpr int DC = Cfg::D_COLS;
  const int row_in_tile = quad * 32 + lane;
  const bool lead = quad == 0 && lane == 0;
#pragma unroll 1
  for (int q = 0; q < Cfg::BN / DC; ++q) {
    uint32_t packed[DC / 2];
    if (warp_live) {
#pragma unroll
      for (int h = 0; h < DC / 32; ++h) {
        float v[32];
        tmem_ld32_sync(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(DC * q + 32 * h), v);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const __nv_bfloat162 b2 = Cfg::NV ? __floats2bfloat162_rn(v[2 * k] * alpha, v[2 * k + 1] * alpha)
                                            : __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
          packed[16 * h + k] = *reinterpret_cast<const uint32_t*>(&b2);
        }
      }
    }
    if (q == Cfg::BN / DC - 1) {
      tc_fence_before();
      __syncwarp();
      release();
    }
    if (lead) bulk_wait_read_all();   // the previous store has read the staging buffer
    named_bar_sync(1, 128);
    if (warp_live) {
      constexpr int NCK = DC / 8;                       // 16-byte chunks per staged row
      const int sw = DC == 64 ? (row_in_tile & 7) : ((row_in_tile >> 1) & 3);
#pragma unroll
      for (int c = 0; c < NCK; ++c)
        *reinterpret_cast<uint4*>(dstage + row_in_tile * (DC * 2) + ((c ^ sw) << 4)) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (lead && warp_live && !*abort_flag) {
      tma_store_2d(tmap_d, smem_addr(dstage), x0 + DC * q, y0);
      bulk_commit_group();
    }
  }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    wush_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_d, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Cfg::OFF_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int STAGES = Cfg::STAGES;
  const int B_FULL = 0, B_EMPTY = STAGES, B_AFULL = 2 * STAGES, B_AEMPTY = 2 * STAGES + 1, B_DRAIN = 2 * STAGES + 2,
            B_SF = 2 * STAGES + 3;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;
  const int n_tiles = p.tiles_m * p.tiles_n;
  const int k_stages = p.K / Cfg::BK;
  const int k_chunks = p.K / Cfg::ATOM_K;               // scale atoms along K per 128-row block

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(BAR(B_FULL + s), 1);
      mbar_init(BAR(B_EMPTY + s), 1);
      mbar_init(BAR(B_SF + s), 4);
    }
    mbar_init(BAR(B_AFULL), 1);
    mbar_init(BAR(B_AEMPTY), 4);
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    tma_prefetch_desc(&tmap_d);
  }
  grid_dependency_wait();
  grid_launch_dependents();
  if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int stage = 0, n_issued = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!wait_bounded(BAR(B_EMPTY + stage), phase ^ 1u, abort_flag, 1u, lim)) break;
          const uint32_t dst = sbase + stage * Cfg::STAGE_BYTES;
          const uint32_t fb = BAR(B_FULL + stage);
          mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
          tma_load_2d(dst + Cfg::OFF_A, &tmap_a, fb, ks * 128, tm * Cfg::BM, 0ull);
          tma_load_2d(dst + Cfg::OFF_B, &tmap_b, fb, ks * 128, tn * Cfg::BN, pol);
          // scale atoms of this stage's K chunks, for the tile's A row block and B's two halves
          constexpr uint32_t APS = Cfg::ATOMS_PER_STAGE;
          bulk_load_1d(dst + Cfg::OFF_SFA, p.sfa + (static_cast<long long>(tm) * k_chunks + APS * ks) * 512,
                       APS * 512u, fb);
          for (int h = 0; h < 2; ++h)
            bulk_load_1d(dst + Cfg::OFF_SFB + h * APS * 512,
                         p.sfb + (static_cast<long long>(2 * tn + h) * k_chunks + APS * ks) * 512, APS * 512u, fb);
          ++n_issued;
          if (++stage == STAGES) stage = 0, phase ^= 1u;
        }
      }
      if (*abort_flag) {   // copies in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int k = (n_issued > STAGES ? n_issued - STAGES : 0); k < n_issued; ++k)
          wait_bounded(BAR(B_FULL + k % STAGES), static_cast<uint32_t>((k / STAGES) & 1), &no_abort, 16u, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        if (!wait_bounded(BAR(B_AEMPTY), static_cast<uint32_t>((it & 1) ^ 1), abort_flag, 2u, lim)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < k_stages; ++ks) {
          // the operands have landed and the scale warps have written the stage's scale slot
          if (!wait_bounded(BAR(B_FULL + stage), phase, abort_flag, 2u, lim) ||
              !wait_bounded(BAR(B_SF + stage), phase, abort_flag, 2u, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * Cfg::STAGE_BYTES;
          const uint32_t sf_cols = tmem_base + static_cast<uint32_t>(Cfg::SF_COL0 + stage * Cfg::SF_SLOT_COLS);
          const uint64_t da = desc_k_sw128(st + Cfg::OFF_A);
          const uint64_t db = desc_k_sw128(st + Cfg::OFF_B);
#pragma unroll
          for (int j = 0; j < 4; ++j) {        // K = 64 each: 32 bytes along the 128-byte rows
            // MXFP4: two MMAs per atom word, scales at byte 0 or 2; NVFP4: one word per MMA
            const int a = Cfg::NV ? j : (j >> 1);
            const uint32_t sub = Cfg::NV ? 0u : static_cast<uint32_t>(2 * (j & 1));
            const uint32_t sfa = (sf_cols + 4 * a) | (sub << 30);
            const uint32_t sfb = (sf_cols + Cfg::SFB_COL + 8 * a) | (sub << 30);
            const uint32_t idesc = idesc_mxf4(128, 256, sub, !Cfg::NV);
            if constexpr (Cfg::NV)
              umma_nvf4(tmem_base, da + ((j * 32) >> 4), db + ((j * 32) >> 4), idesc, sfa, sfb, (ks > 0 || j > 0) ? 1u : 0u);
            else
              umma_mxf4(tmem_base, da + ((j * 32) >> 4), db + ((j * 32) >> 4), idesc, sfa, sfb, (ks > 0 || j > 0) ? 1u : 0u);
          }
          umma_commit(BAR(B_EMPTY + stage));
          if (++stage == STAGES) stage = 0, phase ^= 1u;
        }
        if (!ok) break;
        umma_commit(BAR(B_AFULL));
      }
      umma_commit(BAR(B_DRAIN));
      volatile int no_abort = 0;
      wait_bounded(BAR(B_DRAIN), 0u, &no_abort, 16u, lim);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue (4 warps)
    const int quad = warp & 3;
    const float alpha = Cfg::NV ? __fmul_rn(*p.ts_a, *p.ts_b) : 1.0f;
    int it = 0;
    bool live = true;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      if (live && !wait_bounded(BAR(B_AFULL), static_cast<uint32_t>(it & 1), abort_flag, 8u, lim)) live = false;
      const bool warp_live = __all_sync(0xffffffffu, live) && !*abort_flag;
      if (warp_live) tc_fence_after();
      epilogue_tile<Cfg>(tmem_base, quad, lane, warp_live, alpha, smem + Cfg::OFF_D, &tmap_d, tn * Cfg::BN,
                         tm * Cfg::BM, abort_flag, [&] {   // the next tile's MMAs may go
                           if (lane == 0) mbar_arrive(BAR(B_AEMPTY));
                         });
    }
    if (quad == 0 && lane == 0) bulk_wait_read_all();   // the last store has read the buffer
  } else if (warp >= 8) {
    // ------------------------------------------------------------ scale warps (4)
    // Warp 8 + q writes lane quadrant q of each stage's TMEM scale slot.  The slot's
    // previous readers (the MMAs of the stage one ring round earlier) completed before
    // the producer refilled the stage, so the operands having landed frees the slot too.
    // A wait that expires reports as a converter wait (error bit 4).
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    int stage = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int tile = blockIdx.x; tile < n_tiles && live; tile += gridDim.x) {
      for (int ks = 0; ks < k_stages; ++ks) {
        const bool landed = wait_bounded(BAR(B_FULL + stage), phase, abort_flag, 4u, lim);
        if (!__all_sync(0xffffffffu, landed) || *abort_flag) {
          live = false;
          break;
        }
        tc_fence_after();
        write_scale_slot<Cfg>(lane_base + static_cast<uint32_t>(Cfg::SF_COL0 + stage * Cfg::SF_SLOT_COLS),
                              smem + stage * Cfg::STAGE_BYTES, lane);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_SF + stage));
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA-pair variant
// The same GEMM on pairs of CTAs (a cluster of two on two SMs) sharing one M = 256 MMA:
// CTA v of the pair holds rows [128 v, 128 v + 128) of the pair's A tile and rows
// [128 v, 128 v + 128) of its 256-row B tile (B split along N), plus its rows' A scale
// atoms and the whole B tile's scale atoms; its TMEM accumulator holds its 128 rows x all
// 256 columns.  Each SM thus streams 32 KB of operands per 256-K stage instead of 48 KB
// for the same multiply-adds, which is what bounds the one-CTA kernel (operand bytes in
// flight per SM against L2 latency).  Both CTAs' TMA loads complete on the even CTA's
// full barrier; only the even CTA waits on it, copies the scale atoms into both CTAs'
// TMEM (tcgen05.cp.cta_group::2: writing them with tcgen05.st from each CTA's own scale
// warps, as the single-CTA kernel does, measured 1.8x slower here) and issues the MMAs;
// its commits reach both CTAs' barriers; the odd CTA's epilogue warps arrive on the even
// CTA's accumulator-empty barrier.  No load is multicast.
template <bool NV_>
struct GemmPairCfg {
  static constexpr bool NV = NV_;
  static constexpr int VS = NV ? 16 : 32;
  static constexpr int BM = 128, BN = 256, BK = 256;   // per CTA: 128 rows, all 256 columns
  static constexpr int PAIR_M = 2 * BM;
  static constexpr int ATOM_K = 4 * VS;
  static constexpr int ATOMS_PER_STAGE = BK / ATOM_K;  // MX 2, NV 4
  static constexpr int STAGES = NV ? 5 : 6;
  static constexpr int A_BYTES = BM * BK / 2;          // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK / 2;    // 16 KB: this CTA's half of B
  static constexpr int SFA_BYTES = ATOMS_PER_STAGE * 512;
  static constexpr int SFB_BYTES = 2 * ATOMS_PER_STAGE * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int OFF_A = 0, OFF_B = A_BYTES, OFF_SFA = A_BYTES + B_BYTES, OFF_SFB = OFF_SFA + SFA_BYTES;
  static constexpr int D_COLS = NV ? 64 : 32;          // output staging width (MX: six stages leave 8 KB)
  static constexpr int OFF_D = STAGES * STAGE_BYTES;
  static constexpr int D_BYTES = BM * D_COLS * 2;
  static constexpr int OFF_BAR = OFF_D + D_BYTES;
  static constexpr int N_BARS = 2 * STAGES + 3;        // full[S], empty[S], afull, aempty, drain
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static constexpr int THREADS = 8 * 32;               // producer, MMA, 2 idle, 4 epilogue warps
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_COL0 = 256, SFB_COL = 4 * ATOMS_PER_STAGE, SF_SLOT_COLS = 12 * ATOMS_PER_STAGE;
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SF_COL0 + STAGES * SF_SLOT_COLS <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA 2-D load into this CTA's shared memory whose bytes complete on a barrier of either
// CTA of the pair (given as a shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// 32 lanes x 128 bits from each CTA's shared memory into the same TMEM address of each CTA
__device__ __forceinline__ void tmem_cp_pair_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void umma_pair_fp4(bool nv, uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  if (nv)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// completion of this thread's earlier tcgen05 operations arrives once on the barrier at
// the same shared-memory offset in both CTAs of the pair
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// wait_bounded for a barrier that threads of the other CTA of the pair arrive on: the
// wait acquires at cluster scope, so their writes before the arrive are visible.  No
// suspend-time hint: the waiting thread polls.
__device__ __forceinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity, volatile int* abort,
                                                     uint32_t code, uint64_t limit_ns) {
  auto try_wait = [&]() -> bool {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
  };
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (try_wait()) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      atomicOr(&g_wush_device_error, code);
      *abort = 1;
      return false;
    }
  }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    wush_gemm_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                              const __grid_constant__ CUtensorMap tmap_sfa,
                              const __grid_constant__ CUtensorMap tmap_sfb,
                              const __grid_constant__ CUtensorMap tmap_d, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Cfg::OFF_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int STAGES = Cfg::STAGES;
  constexpr uint32_t APS = Cfg::ATOMS_PER_STAGE;
  const int B_FULL = 0, B_EMPTY = STAGES, B_AFULL = 2 * STAGES, B_AEMPTY = 2 * STAGES + 1, B_DRAIN = 2 * STAGES + 2;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();           // 0: issues the MMAs, 1: its partner
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);
  const uint64_t lim = p.wait_limit_ns;
  const int n_tiles = p.tiles_m * p.tiles_n;         // pair tiles of 256 x 256
  const int k_stages = p.K / Cfg::BK;
  const int k_chunks = p.K / Cfg::ATOM_K;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(BAR(B_FULL + s), 1);
      mbar_init(BAR(B_EMPTY + s), 1);
    }
    mbar_init(BAR(B_AFULL), 1);
    mbar_init(BAR(B_AEMPTY), 2 * 4);                 // four epilogue warps in each CTA
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    tma_prefetch_desc(&tmap_sfa);
    tma_prefetch_desc(&tmap_sfb);
    tma_prefetch_desc(&tmap_d);
  }
  grid_dependency_wait();
  grid_launch_dependents();
  if (warp == 1) {                                    // the same warp of both CTAs
    tmem_alloc_pair(smem_addr(const_cast<uint32_t*>(tmem_slot)), Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();                                 // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < n_tiles && !*abort_flag; tile += n_pairs) {
        const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
        const int a_row = tm * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM;
        const int b_row = tn * Cfg::BN + static_cast<int>(rank) * (Cfg::BN / 2);
        const int a_blk = tm * 2 + static_cast<int>(rank);     // this CTA's 128-row scale block
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!wait_bounded(BAR(B_EMPTY + stage), phase ^ 1u, abort_flag, 1u, lim)) break;
          const uint32_t dst = sbase + stage * Cfg::STAGE_BYTES;
          const uint32_t fb = mapa_shared(BAR(B_FULL + stage), 0);   // the even CTA's full barrier
          if (rank == 0) mbar_arrive_expect_tx(BAR(B_FULL + stage), 2u * Cfg::STAGE_BYTES);
          tma_load_2d_pair(dst + Cfg::OFF_A, &tmap_a, fb, ks * 128, a_row, 0ull);
          tma_load_2d_pair(dst + Cfg::OFF_B, &tmap_b, fb, ks * 128, b_row, pol);
          // scale atoms as 128-byte rows: APS atoms of this CTA's A block, APS of each B half
          tma_load_2d_pair(dst + Cfg::OFF_SFA, &tmap_sfa, fb, 0,
                           static_cast<int>((a_blk * k_chunks + APS * ks) * 4), 0ull);
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(dst + Cfg::OFF_SFB + h * APS * 512, &tmap_sfb, fb, 0,
                             static_cast<int>(((2 * tn + h) * k_chunks + APS * ks) * 4), 0ull);
          if (++stage == STAGES) stage = 0, phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < n_tiles; tile += n_pairs, ++it) {
        if (!wait_bounded_cluster(BAR(B_AEMPTY), static_cast<uint32_t>((it & 1) ^ 1), abort_flag, 2u, lim)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!wait_bounded(BAR(B_FULL + stage), phase, abort_flag, 2u, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + stage * Cfg::STAGE_BYTES;
          const uint32_t sf_cols = tmem_base + static_cast<uint32_t>(Cfg::SF_COL0 + stage * Cfg::SF_SLOT_COLS);
#pragma unroll
          for (int a = 0; a < Cfg::ATOMS_PER_STAGE; ++a) {
            tmem_cp_pair_32x128b_x4(sf_cols + 4 * a, desc_sf_atom(st + Cfg::OFF_SFA + a * 512));
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tmem_cp_pair_32x128b_x4(sf_cols + Cfg::SFB_COL + 8 * a + 4 * h,
                                      desc_sf_atom(st + Cfg::OFF_SFB + h * Cfg::ATOMS_PER_STAGE * 512 + a * 512));
          }
          const uint64_t da = desc_k_sw128(st + Cfg::OFF_A);
          const uint64_t db = desc_k_sw128(st + Cfg::OFF_B);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int a = Cfg::NV ? j : (j >> 1);
            const uint32_t sub = Cfg::NV ? 0u : static_cast<uint32_t>(2 * (j & 1));
            const uint32_t sfa = (sf_cols + 4 * a) | (sub << 30);
            const uint32_t sfb = (sf_cols + Cfg::SFB_COL + 8 * a) | (sub << 30);
            umma_pair_fp4(Cfg::NV, tmem_base, da + ((j * 32) >> 4), db + ((j * 32) >> 4),
                          idesc_mxf4(Cfg::PAIR_M, Cfg::BN, sub, !Cfg::NV), sfa, sfb, (ks > 0 || j > 0) ? 1u : 0u);
          }
          umma_commit_pair(BAR(B_EMPTY + stage));
          if (++stage == STAGES) stage = 0, phase ^= 1u;
        }
        if (!ok) break;
        umma_commit_pair(BAR(B_AFULL));
      }
      umma_commit_pair(BAR(B_DRAIN));
    }
    if (lane == 0) {   // both CTAs: every MMA writing this CTA's TMEM has finished
      volatile int no_abort = 0;
      wait_bounded(BAR(B_DRAIN), 0u, &no_abort, 16u, lim);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue (4 warps, both CTAs)
    const int quad = warp & 3;
    const float alpha = Cfg::NV ? __fmul_rn(*p.ts_a, *p.ts_b) : 1.0f;
    const uint32_t aempty_leader = mapa_shared(BAR(B_AEMPTY), 0);
    int it = 0;
    bool live = true;
    for (int tile = pair; tile < n_tiles; tile += n_pairs, ++it) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      if (live && !wait_bounded(BAR(B_AFULL), static_cast<uint32_t>(it & 1), abort_flag, 8u, lim)) live = false;
      const bool warp_live = __all_sync(0xffffffffu, live) && !*abort_flag;
      if (warp_live) tc_fence_after();
      epilogue_tile<Cfg>(tmem_base, quad, lane, warp_live, alpha, smem + Cfg::OFF_D, &tmap_d, tn * Cfg::BN,
                         tm * Cfg::PAIR_M + static_cast<int>(rank) * Cfg::BM, abort_flag, [&] {
                           if (lane == 0) mbar_arrive_cluster(aempty_leader);
                         });
    }
    if (quad == 0 && lane == 0) bulk_wait_read_all();   // the last store has read the buffer
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                                 // no remote arrive or commit is still on its way
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

// Row-major one-byte scales [rows][C] -> tcgen05 scale atoms (rows padded to a multiple
// of 128 with zero bytes, C to a multiple of 4).
__global__ void wush_scales_to_atoms_kernel(const uint8_t* __restrict__ src, long long rows, int C,
                                            uint8_t* __restrict__ dst, long long rows_pad, int C_pad) {
  const long long n = rows_pad * C_pad;
  const int k_chunks = C_pad / 4;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / C_pad;
    const int c = static_cast<int>(i - r * C_pad);
    const uint8_t v = (r < rows && c < C) ? src[r * C + c] : static_cast<uint8_t>(0);
    const long long rb = r >> 7;
    const int rr = static_cast<int>(r & 127);
    dst[(rb * k_chunks + (c >> 2)) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3)] = v;
  }
}

}  // namespace wush
