// Host side of the C ABI declared in include/wush.h: argument validation, TMA
// descriptor encoding, kernel selection and launch.  No allocation, no host
// synchronisation on the quantisation calls.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "wush.h"
#include "wush_fused.cuh"
#include "wush_build.cuh"
#include "wush_dequant.cuh"
#include "wush_gemm.cuh"
#include "wush_small.cuh"

namespace wush {
// Waits on an mbarrier that no thread ever arrives on; the bounded wait must give up.
__global__ void wush_selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(smem_addr(&bar), 0u, &abort_word, 32u, limit_ns);
}
// Scratch of wush_quant_act_nvfp4_onepass_noalloc: 256 bytes, of which the one-launch
// NVFP4 kernel uses the first three words.  Zero at module load; every call that ends
// without a device error leaves it zero.
constexpr int kNoAllocScratchWords = 64;
constexpr int kOnepassWorkspaceWords = 3;
static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoAllocScratchWords];
static_assert(kOnepassWorkspaceWords <= kNoAllocScratchWords, "scratch too small for the one-launch workspace");

}  // namespace wush

#ifndef WUSH_USE_PDL
#define WUSH_USE_PDL 1
#endif
#ifndef WUSH_NV_REVERSE
#define WUSH_NV_REVERSE true
#endif

namespace {

constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

// The failing call behind the last WUSH_ERR_CUDA returned on this host thread: what was
// called, where, and the runtime's (or the driver's) error code.
struct CudaFailure {
  const char* what = nullptr;
  int line = 0;
  int code = 0;
  bool driver = false;
};
thread_local CudaFailure t_cuda_failure;

int cuda_fail(int code, const char* what, int line, bool driver = false) {
  t_cuda_failure.what = what;
  t_cuda_failure.line = line;
  t_cuda_failure.code = code;
  t_cuda_failure.driver = driver;
  return WUSH_ERR_CUDA;
}

// status of the kernel launch just issued on this thread
int launch_status(int line) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? WUSH_OK : cuda_fail(e, "kernel launch", line);
}

#define WUSH_CUDA_CHECK(call)                                                    \
  do {                                                                           \
    const cudaError_t wush_e_ = (call);                                          \
    if (wush_e_ != cudaSuccess) return cuda_fail(wush_e_, #call, __LINE__);     \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

PFN_cuCtxGetCurrent_v4000 context_getter() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuCtxGetCurrent_v4000>(nullptr);
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  }();
  return fn;
}

// Driver-API calls (the tensor-map encoder) act on the context current on the calling host
// thread.  The runtime binds the current device's primary context to a thread lazily, at
// its first call there that needs one, so a thread whose first CUDA work is a call into
// this library may have no context yet; bind it before the first driver call.
int ensure_context() {
  auto get = context_getter();
  if (!get) return cuda_fail(0, "cudaGetDriverEntryPoint(cuCtxGetCurrent)", __LINE__, true);
  CUcontext c = nullptr;
  const CUresult r = get(&c);
  if (r != CUDA_SUCCESS) return cuda_fail(r, "cuCtxGetCurrent", __LINE__, true);
  if (c) return WUSH_OK;
  int dev = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaSetDevice(dev));   // initialises the primary context and makes it current
  return WUSH_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// 2-D row-major [rows][cols] tensor, box {box_cols, 128 rows}.
int encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, int64_t rows,
              int64_t cols, int box_cols, CUtensorMapSwizzle swz) {
  const int ctx = ensure_context();
  if (ctx != WUSH_OK) return ctx;
  auto enc = tensor_map_encoder();
  if (!enc) return cuda_fail(0, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", __LINE__, true);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * static_cast<cuuint64_t>(elem_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), 128u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WUSH_OK : cuda_fail(r, "cuTensorMapEncodeTiled", __LINE__, true);
}

// 2-D row-major uint8 [rows][cols] tensor, box {box_cols, box_rows}, no swizzle.
int encode_u8_plain(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  const int ctx = ensure_context();
  if (ctx != WUSH_OK) return ctx;
  auto enc = tensor_map_encoder();
  if (!enc) return cuda_fail(0, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", __LINE__, true);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WUSH_OK : cuda_fail(r, "cuTensorMapEncodeTiled", __LINE__, true);
}

// 2-D row-major uint8 [rows][cols] tensor, box {box_cols, box_rows}, 128-byte swizzle.
int encode_u8_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  const int ctx = ensure_context();
  if (ctx != WUSH_OK) return ctx;
  auto enc = tensor_map_encoder();
  if (!enc) return cuda_fail(0, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", __LINE__, true);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WUSH_OK : cuda_fail(r, "cuTensorMapEncodeTiled", __LINE__, true);
}

template <class Cfg, bool REV = false, bool ONEPASS = false>
int launch_fused(const CUtensorMap& map, const CUtensorMap& cmap, wush::FusedParams p, cudaStream_t stream) {
  int dev = 0, sms = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  static std::atomic<unsigned long long> configured{0ull};   // one bit per device ordinal
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    WUSH_CUDA_CHECK(cudaFuncSetAttribute(wush::wush_fused_kernel<Cfg, REV, ONEPASS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  int grid = p.total_tiles < sms ? p.total_tiles : sms;
  // Long bf16 MXFP4 runs take the largest grid (down to 3/4 of the SMs) that gives every
  // CTA the same whole fraction, or whole multiple, of a column tile.  The CTAs then step
  // through the same row band together and read whole rows between them.  Measured on
  // B200: 16384 x 8192 takes 61.5 us on 128 CTAs against 72.7 us on 148.  The fp32 weight
  // path (60.3 -> 66.5 us), NVFP4 (59.0 -> 67.4 us on 112) and INT4 (21.2 -> 23.1 us at
  // 8192 x 4096) do more work per tile and lose more with the SMs than they gain.
  if (Cfg::FMT == wush::kMXFP4 && !Cfg::IN_F32 && p.total_tiles / grid >= 32) {
    for (int g = grid; g >= (3 * grid) / 4; --g) {
      if (p.total_tiles % g) continue;
      const int per = p.total_tiles / g;
      if (per % p.n_row_tiles == 0 || p.n_row_tiles % per == 0) {
        grid = g;
        break;
      }
    }
  }
  // Input tiles each CTA warms in L2 before its dependency wait.  Measured on B200: two for
  // runs of a few tiles per CTA (4096 x 4096 MXFP4 with the short runs on the last CTAs:
  // 9.81 us with one, 9.75 with two; deeper prefetches still in flight delay the first
  // loads), three for long runs, whose predecessor ends over a longer window (16384 x 8192:
  // 74.8 -> 73.0).
  p.prefetch_tiles = p.total_tiles / grid >= 32 ? 3 : 2;
  // programmatic stream serialisation: the CTAs may be scheduled while the previous kernel
  // in the stream drains; they do their set-up and then wait (griddepcontrol.wait) for it
  // to complete before reading any input
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(grid));
  lc.blockDim = dim3(Cfg::THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = stream;
  // ONEPASS: the CTAs wait on one another, so all of them must be resident at once
  // (cooperative launch); programmatic serialisation still lets them be scheduled while
  // the previous kernel drains (measured 0.5 us less per call than cooperative alone)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = ONEPASS ? (WUSH_USE_PDL ? 2 : 1) : (WUSH_USE_PDL ? 1 : 0);
  if (ONEPASS && !WUSH_USE_PDL) lc.attrs = attr + 1;
  WUSH_CUDA_CHECK(cudaLaunchKernelEx(&lc, wush::wush_fused_kernel<Cfg, REV, ONEPASS>, map, cmap, p));
  return launch_status(__LINE__);
}

// A launch with programmatic stream serialisation, for kernels that call
// griddepcontrol.wait before their first global read.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = WUSH_USE_PDL ? 1 : 0;
  WUSH_CUDA_CHECK(cudaLaunchKernelEx(&lc, kern, args...));
  return launch_status(__LINE__);
}

template <int G, int FMT, bool IN_F32, bool AMAX_ONLY, bool SHARED, bool REV = false>
int launch_pick_y(const CUtensorMap& map, const CUtensorMap& cmap, const wush::FusedParams& p, bool emit_y,
                  cudaStream_t s) {
  if (emit_y) return launch_fused<wush::FusedCfg<G, FMT, IN_F32, AMAX_ONLY, true, SHARED>, REV>(map, cmap, p, s);
  return launch_fused<wush::FusedCfg<G, FMT, IN_F32, AMAX_ONLY, false, SHARED>, REV>(map, cmap, p, s);
}

// NVFP4 stages: the whole call, the amax pass alone (for a max-reduction across ranks
// before the scale is fixed), or the quantising pass with a given tensor scale
enum NvMode { kNvAll = 0, kNvAmaxOnly = 1, kNvWithScale = 2 };

template <bool IN_F32, bool SHARED>
int dispatch(const CUtensorMap& map, const CUtensorMap& cmap, wush::FusedParams p, int G, int fmt, bool emit_y,
             float* tensor_scale, cudaStream_t s, int nv_mode = kNvAll) {
  if (fmt == WUSH_MXFP4) return launch_pick_y<32, wush::kMXFP4, IN_F32, false, SHARED>(map, cmap, p, emit_y, s);
  if (fmt == WUSH_INT4) {
    if (G == 32) return launch_pick_y<32, wush::kINT4, IN_F32, false, SHARED>(map, cmap, p, emit_y, s);
    return launch_pick_y<16, wush::kINT4, IN_F32, false, SHARED>(map, cmap, p, emit_y, s);
  }
  // NVFP4: pass 1 finds amax|y| (float bits, running max in *tensor_scale), a one-thread
  // kernel turns it into s_t in place, pass 2 quantises with s_t.
  if (nv_mode != kNvWithScale) {
    int st = launch_pdl(wush::wush_nvfp4_amax_reset_kernel, dim3(1), dim3(32), s, tensor_scale);
    if (st != WUSH_OK) return st;
    wush::FusedParams p1 = p;
    p1.amax_word = reinterpret_cast<unsigned int*>(tensor_scale);
    p1.codes_via_tma = 0;
    st = launch_fused<wush::FusedCfg<16, wush::kNVFP4, IN_F32, true, false, SHARED>>(map, cmap, p1, s);
    if (st != WUSH_OK) return st;
    if (nv_mode == kNvAmaxOnly) return WUSH_OK;
    st = launch_pdl(wush::wush_nvfp4_tensor_scale_kernel, dim3(1), dim3(32), s, tensor_scale);
    if (st != WUSH_OK) return st;
  }
  p.tensor_scale = tensor_scale;
  // walked backwards: the quantising pass first reads what the amax pass loaded last
  return launch_pick_y<16, wush::kNVFP4, IN_F32, false, SHARED, WUSH_NV_REVERSE>(map, cmap, p, emit_y, s);
}

// Activation batches of at most this many rows take the CUDA-core path (wush_small.cuh);
// 0 sends every batch to the fused tensor-core kernel, -1 selects the per-format default
// (measured crossovers at d_in = 4096: MXFP4 between 64 and 128 rows, INT4 and NVFP4
// between 256 and 512).
std::atomic<long long> g_small_rows{-1};
long long small_rows_limit(int fmt) {
  const long long v = g_small_rows.load(std::memory_order_relaxed);
  if (v >= 0) return v;
  return fmt == WUSH_MXFP4 ? 64 : 256;
}

template <int G, int FMT, bool AMAX_ONLY, bool SHARED>
int launch_small(const void* x, const wush::FusedParams& p, bool emit_y, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.C), static_cast<unsigned>((p.n_rows + wush::kSmallRows - 1) / wush::kSmallRows));
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (emit_y && !AMAX_ONLY)
    return launch_pdl(wush::wush_small_kernel<G, FMT, AMAX_ONLY, true, SHARED>, grid, dim3(wush::kSmallRows), s, xb, p);
  return launch_pdl(wush::wush_small_kernel<G, FMT, AMAX_ONLY, false, SHARED>, grid, dim3(wush::kSmallRows), s, xb, p);
}

template <bool SHARED>
int small_dispatch(const void* x, wush::FusedParams p, int G, int fmt, bool emit_y, float* tensor_scale,
                   cudaStream_t s, int nv_mode) {
  if (fmt == WUSH_MXFP4) return launch_small<32, wush::kMXFP4, false, SHARED>(x, p, emit_y, s);
  if (fmt == WUSH_INT4)
    return G == 32 ? launch_small<32, wush::kINT4, false, SHARED>(x, p, emit_y, s)
                   : launch_small<16, wush::kINT4, false, SHARED>(x, p, emit_y, s);
  if (nv_mode != kNvWithScale) {   // NVFP4: amax pass, tensor scale, quantising pass
    int st = launch_pdl(wush::wush_nvfp4_amax_reset_kernel, dim3(1), dim3(32), s, tensor_scale);
    if (st != WUSH_OK) return st;
    wush::FusedParams p1 = p;
    p1.amax_word = reinterpret_cast<unsigned int*>(tensor_scale);
    st = launch_small<16, wush::kNVFP4, true, SHARED>(x, p1, false, s);
    if (st != WUSH_OK || nv_mode == kNvAmaxOnly) return st;
    st = launch_pdl(wush::wush_nvfp4_tensor_scale_kernel, dim3(1), dim3(32), s, tensor_scale);
    if (st != WUSH_OK) return st;
  }
  p.tensor_scale = tensor_scale;
  return launch_small<16, wush::kNVFP4, false, SHARED>(x, p, emit_y, s);
}

int quant_common(const void* in, bool in_f32, const float* T, int64_t rows, int64_t d_in, int G, int fmt,
                 uint8_t* codes, void* scales, float* tensor_scale, float* y_out, bool debug,
                 wush_stream_t stream, bool shared_T = false, bool scale_atoms = false, int nv_mode = kNvAll) {
  if (fmt != WUSH_MXFP4 && fmt != WUSH_NVFP4 && fmt != WUSH_INT4) return WUSH_ERR_UNSUPPORTED;
  const bool amax_only = fmt == WUSH_NVFP4 && nv_mode == kNvAmaxOnly;   // no codes or scales written
  const bool g_ok = (fmt == WUSH_MXFP4 && G == 32) || (fmt == WUSH_NVFP4 && G == 16) ||
                    (fmt == WUSH_INT4 && (G == 16 || G == 32));
  if (!g_ok) return WUSH_ERR_UNSUPPORTED;
  if (rows < 0 || d_in <= 0 || d_in % G != 0) return WUSH_ERR_INVALID_ARG;
  if (rows > INT_MAX || d_in > INT_MAX) return WUSH_ERR_INVALID_ARG;
  if (rows == 0) {                 // empty batch: nothing to read or write
    if (!amax_only) return WUSH_OK;
    if (!tensor_scale || !aligned(tensor_scale, 4)) return tensor_scale ? WUSH_ERR_MISALIGNED : WUSH_ERR_INVALID_ARG;
    // an empty shard still contributes its amax (0) to a reduction across ranks
    WUSH_CUDA_CHECK(cudaMemsetAsync(tensor_scale, 0, sizeof(float), reinterpret_cast<cudaStream_t>(stream)));
    return WUSH_OK;
  }
  if (!in || !T || (!amax_only && (!codes || !scales))) return WUSH_ERR_INVALID_ARG;
  if (fmt == WUSH_NVFP4 && !tensor_scale) return WUSH_ERR_INVALID_ARG;
  if (debug && !y_out) return WUSH_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(T, 16) || (codes && !aligned(codes, 16))) return WUSH_ERR_MISALIGNED;
  if (fmt == WUSH_INT4 && !aligned(scales, 4)) return WUSH_ERR_MISALIGNED;
  if (scale_atoms && !aligned(scales, 16)) return WUSH_ERR_MISALIGNED;
  if (tensor_scale && !aligned(tensor_scale, 4)) return WUSH_ERR_MISALIGNED;
  if (debug && !aligned(y_out, 16)) return WUSH_ERR_MISALIGNED;

  if (!in_f32 && rows <= small_rows_limit(fmt)) {
    wush::FusedParams p{};
    p.scale_atoms = scale_atoms ? 1 : 0;
    p.atom_cols = static_cast<int>((d_in / G + 3) / 4);
    p.T = T;
    p.codes = codes;
    p.scales = scales;
    p.y_out = y_out;
    p.n_rows = rows;
    p.d_in = static_cast<int>(d_in);
    p.C = static_cast<int>(d_in / G);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return shared_T ? small_dispatch<true>(in, p, G, fmt, debug, tensor_scale, s, nv_mode)
                    : small_dispatch<false>(in, p, G, fmt, debug, tensor_scale, s, nv_mode);
  }

  const int ch = in_f32 ? 64 : WUSH_ACT_TILE_CH;   // channels per tile, as in FusedCfg
  const long long n_row_tiles = (rows + 127) / 128;
  const long long n_col_tiles = (d_in + ch - 1) / ch;
  if (n_row_tiles * n_col_tiles > INT_MAX) return WUSH_ERR_INVALID_ARG;

  CUtensorMap map;
  int st = in_f32 ? encode_2d(&map, in, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, d_in, 64,
                              CU_TENSOR_MAP_SWIZZLE_NONE)
                  : encode_2d(&map, in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, d_in, 64,
                              CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != WUSH_OK) return st;
  // codes leave through a TMA store when the row pitch allows it (a multiple of 16 bytes);
  // the store map's swizzle matches the kernel's staging layout (64-byte rows: 64B
  // swizzle, 32-byte rows: 32B swizzle)
  CUtensorMap cmap = map;
  const bool codes_tma = !amax_only && ((d_in / 2) % 16) == 0;
  if (codes_tma) {
    st = encode_2d(&cmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, d_in / 2, ch / 2,
                   ch == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != WUSH_OK) return st;
  }

  wush::FusedParams p{};
  p.codes_via_tma = codes_tma ? 1 : 0;
  p.scale_atoms = scale_atoms ? 1 : 0;
  p.atom_cols = static_cast<int>((d_in / G + 3) / 4);
  p.T = T;
  p.codes = codes;
  p.scales = scales;
  p.y_out = y_out;
  p.amax_word = nullptr;
  p.tensor_scale = nullptr;
  p.n_rows = rows;
  p.d_in = static_cast<int>(d_in);
  p.C = static_cast<int>(d_in / G);
  p.n_row_tiles = static_cast<int>(n_row_tiles);
  p.total_tiles = static_cast<int>(n_row_tiles * n_col_tiles);
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (shared_T) return dispatch<false, true>(map, cmap, p, G, fmt, debug, tensor_scale, s, nv_mode);
  return in_f32 ? dispatch<true, false>(map, cmap, p, G, fmt, debug, tensor_scale, s, nv_mode)
                : dispatch<false, false>(map, cmap, p, G, fmt, debug, tensor_scale, s, nv_mode);
}

}  // namespace

extern "C" {

int wush_quant_act(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, int G, int fmt,
                   uint8_t* codes, void* scales, float* tensor_scale, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, G, fmt, codes, scales, tensor_scale, nullptr, false,
                      stream);
}

int wush_quant_weight(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in, int G, int fmt,
                      uint8_t* codes, void* scales, float* tensor_scale, wush_stream_t stream) {
  return quant_common(w_f32, true, T_blocks, d_out, d_in, G, fmt, codes, scales, tensor_scale, nullptr, false,
                      stream);
}

int wush_quant_act_debug(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, int G, int fmt,
                         uint8_t* codes, void* scales, float* tensor_scale, float* y_out, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, G, fmt, codes, scales, tensor_scale, y_out, true,
                      stream);
}

int wush_quant_weight_debug(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in, int G,
                            int fmt, uint8_t* codes, void* scales, float* tensor_scale, float* y_out,
                            wush_stream_t stream) {
  return quant_common(w_f32, true, T_blocks, d_out, d_in, G, fmt, codes, scales, tensor_scale, y_out, true,
                      stream);
}

int wush_quant_act_shared(const void* x_bf16, const float* T_shared, int64_t n_tok, int64_t d_in, int G, int fmt,
                          uint8_t* codes, void* scales, float* tensor_scale, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_shared, n_tok, d_in, G, fmt, codes, scales, tensor_scale, nullptr, false,
                      stream, true);
}

int wush_quant_act_shared_debug(const void* x_bf16, const float* T_shared, int64_t n_tok, int64_t d_in, int G,
                                int fmt, uint8_t* codes, void* scales, float* tensor_scale, float* y_out,
                                wush_stream_t stream) {
  return quant_common(x_bf16, false, T_shared, n_tok, d_in, G, fmt, codes, scales, tensor_scale, y_out, true,
                      stream, true);
}

int wush_dequant(const uint8_t* codes, const void* scales, const float* tensor_scale, int64_t rows, int64_t d_in,
                 int G, int fmt, float* out, wush_stream_t stream) {
  if (fmt != WUSH_MXFP4 && fmt != WUSH_NVFP4 && fmt != WUSH_INT4) return WUSH_ERR_UNSUPPORTED;
  const bool g_ok = (fmt == WUSH_MXFP4 && G == 32) || (fmt == WUSH_NVFP4 && G == 16) ||
                    (fmt == WUSH_INT4 && (G == 16 || G == 32));
  if (!g_ok) return WUSH_ERR_UNSUPPORTED;
  if (rows < 0 || d_in <= 0 || d_in % G != 0 || d_in > INT_MAX) return WUSH_ERR_INVALID_ARG;
  if (rows == 0) return WUSH_OK;
  if (!codes || !scales || !out || (fmt == WUSH_NVFP4 && !tensor_scale)) return WUSH_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(out, 16) || (fmt == WUSH_INT4 && !aligned(scales, 4)) ||
      (tensor_scale && !aligned(tensor_scale, 4)))
    return WUSH_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const long long n_words = rows * (d_in / 8);
  const long long want = (n_words + 255) / 256;
  const int grid = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int di = static_cast<int>(d_in);
  if (fmt == WUSH_MXFP4)
    wush::wush_dequant_kernel<wush::kMXFP4><<<grid, 256, 0, s>>>(codes, scales, tensor_scale, rows, di, G, out);
  else if (fmt == WUSH_NVFP4)
    wush::wush_dequant_kernel<wush::kNVFP4><<<grid, 256, 0, s>>>(codes, scales, tensor_scale, rows, di, G, out);
  else
    wush::wush_dequant_kernel<wush::kINT4><<<grid, 256, 0, s>>>(codes, scales, tensor_scale, rows, di, G, out);
  return launch_status(__LINE__);
}

int wush_mx_scales_to_atoms(const uint8_t* scales, int64_t rows, int64_t C, uint8_t* atoms, wush_stream_t stream) {
  if (rows < 0 || C <= 0 || C > INT_MAX / 4) return WUSH_ERR_INVALID_ARG;
  if (rows == 0) return WUSH_OK;
  if (!scales || !atoms) return WUSH_ERR_INVALID_ARG;
  const long long rows_pad = (rows + 127) / 128 * 128;
  const int C_pad = static_cast<int>((C + 3) / 4 * 4);
  const long long n = rows_pad * C_pad;
  int dev = 0, sms = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const long long want = (n + 255) / 256;
  const int grid = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  wush::wush_scales_to_atoms_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      scales, rows, static_cast<int>(C), atoms, rows_pad, C_pad);
  return launch_status(__LINE__);
}

}  // extern "C"

namespace {

// Opt-in (wush_set_gemm_cta_pairs): for M a multiple of 256, pairs of CTAs share M = 256
// MMAs (wush_gemm_fp4_pair_kernel).  Off by default: on B200 it measured 4-11 % slower
// than single CTAs at the benchmarked shapes.
std::atomic<int> g_gemm_pairs{0};

template <bool NV>
int gemm_fp4_pair(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts, const uint8_t* b_codes,
                  const uint8_t* b_atoms, const float* b_ts, int64_t M, int64_t N, int64_t K, void* d_bf16,
                  wush_stream_t stream) {
  using Cfg = wush::GemmPairCfg<NV>;
  CUtensorMap ma, mb, msa, msb;
  int st = encode_u8_sw128(&ma, a_codes, M, K / 2, 128, Cfg::BM);
  if (st != WUSH_OK) return st;
  st = encode_u8_sw128(&mb, b_codes, N, K / 2, 128, Cfg::BN / 2);
  if (st != WUSH_OK) return st;
  // scale atoms as rows of 128 bytes: a stage's atoms of one 128-row block are 4 * APS rows
  const long long c_pad = (K / Cfg::VS + 3) / 4 * 4;
  st = encode_u8_plain(&msa, a_atoms, M * c_pad / 128, 128, 128, 4 * Cfg::ATOMS_PER_STAGE);
  if (st != WUSH_OK) return st;
  st = encode_u8_plain(&msb, b_atoms, N * c_pad / 128, 128, 128, 4 * Cfg::ATOMS_PER_STAGE);
  if (st != WUSH_OK) return st;
  CUtensorMap md;   // the bf16 result, stored D_COLS columns x 128 rows at a time
  st = encode_2d(&md, d_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, Cfg::D_COLS,
                 Cfg::D_COLS == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != WUSH_OK) return st;
  wush::GemmParams p{};
  p.sfa = a_atoms;
  p.sfb = b_atoms;
  p.ts_a = a_ts;
  p.ts_b = b_ts;
  p.d = static_cast<__nv_bfloat16*>(d_bf16);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.tiles_m = static_cast<int>(M / Cfg::PAIR_M);
  p.tiles_n = static_cast<int>(N / Cfg::BN);
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  int dev = 0, sms = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  static std::atomic<unsigned long long> configured{0ull};
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    WUSH_CUDA_CHECK(cudaFuncSetAttribute(wush::wush_gemm_fp4_pair_kernel<Cfg>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  const long long tiles = static_cast<long long>(p.tiles_m) * p.tiles_n;
  if (tiles > INT_MAX / 2) return WUSH_ERR_INVALID_ARG;
  const long long pairs = tiles < sms / 2 ? tiles : sms / 2;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  lc.blockDim = dim3(Cfg::THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = WUSH_USE_PDL ? 2 : 1;
  WUSH_CUDA_CHECK(cudaLaunchKernelEx(&lc, wush::wush_gemm_fp4_pair_kernel<Cfg>, ma, mb, msa, msb, md, p));
  return launch_status(__LINE__);
}

// One launch of the block-scaled FP4 GEMM (MXFP4 or NVFP4 operands).
template <bool NV>
int gemm_fp4(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts, const uint8_t* b_codes,
             const uint8_t* b_atoms, const float* b_ts, int64_t M, int64_t N, int64_t K, void* d_bf16,
             wush_stream_t stream) {
  using Cfg = wush::GemmCfg<NV>;
  if (M < 0 || N <= 0 || K <= 0) return WUSH_ERR_INVALID_ARG;
  if (M % Cfg::BM || N % Cfg::BN || K % Cfg::BK) return WUSH_ERR_UNSUPPORTED;
  if (M > INT_MAX || N > INT_MAX || K > INT_MAX) return WUSH_ERR_INVALID_ARG;
  if (M == 0) return WUSH_OK;
  if (!a_codes || !a_atoms || !b_codes || !b_atoms || !d_bf16) return WUSH_ERR_INVALID_ARG;
  if (NV && (!a_ts || !b_ts)) return WUSH_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_atoms, 16) || !aligned(b_atoms, 16) ||
      !aligned(d_bf16, 16))
    return WUSH_ERR_MISALIGNED;
  if (NV && (!aligned(a_ts, 4) || !aligned(b_ts, 4))) return WUSH_ERR_MISALIGNED;
  if (M % 256 == 0 && g_gemm_pairs.load(std::memory_order_relaxed))
    return gemm_fp4_pair<NV>(a_codes, a_atoms, a_ts, b_codes, b_atoms, b_ts, M, N, K, d_bf16, stream);
  CUtensorMap ma, mb;
  int st = encode_u8_sw128(&ma, a_codes, M, K / 2, 128, Cfg::BM);
  if (st != WUSH_OK) return st;
  st = encode_u8_sw128(&mb, b_codes, N, K / 2, 128, Cfg::BN);
  if (st != WUSH_OK) return st;
  CUtensorMap md;   // the bf16 result, stored D_COLS columns x 128 rows at a time
  st = encode_2d(&md, d_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, Cfg::D_COLS,
                 Cfg::D_COLS == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != WUSH_OK) return st;
  wush::GemmParams p{};
  p.sfa = a_atoms;
  p.sfb = b_atoms;
  p.ts_a = a_ts;
  p.ts_b = b_ts;
  p.d = static_cast<__nv_bfloat16*>(d_bf16);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.tiles_m = static_cast<int>(M / Cfg::BM);
  p.tiles_n = static_cast<int>(N / Cfg::BN);
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  int dev = 0, sms = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  static std::atomic<unsigned long long> configured{0ull};
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    WUSH_CUDA_CHECK(cudaFuncSetAttribute(wush::wush_gemm_fp4_kernel<Cfg>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  const long long tiles = static_cast<long long>(p.tiles_m) * p.tiles_n;
  if (tiles > INT_MAX) return WUSH_ERR_INVALID_ARG;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(grid));
  lc.blockDim = dim3(Cfg::THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = WUSH_USE_PDL ? 1 : 0;
  WUSH_CUDA_CHECK(cudaLaunchKernelEx(&lc, wush::wush_gemm_fp4_kernel<Cfg>, ma, mb, md, p));
  return launch_status(__LINE__);
}

}  // namespace

extern "C" {

int wush_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_atoms, const uint8_t* b_codes, const uint8_t* b_atoms,
                    int64_t M, int64_t N, int64_t K, void* d_bf16, wush_stream_t stream) {
  return gemm_fp4<false>(a_codes, a_atoms, nullptr, b_codes, b_atoms, nullptr, M, N, K, d_bf16, stream);
}

int wush_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_tensor_scale,
                    const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_tensor_scale, int64_t M, int64_t N,
                    int64_t K, void* d_bf16, wush_stream_t stream) {
  return gemm_fp4<true>(a_codes, a_atoms, a_tensor_scale, b_codes, b_atoms, b_tensor_scale, M, N, K, d_bf16, stream);
}

int wush_quant_act_mx_atoms(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, uint8_t* codes,
                            uint8_t* scale_atoms, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, 32, WUSH_MXFP4, codes, scale_atoms, nullptr, nullptr,
                      false, stream, false, true);
}

int wush_quant_weight_mx_atoms(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in, uint8_t* codes,
                               uint8_t* scale_atoms, wush_stream_t stream) {
  return quant_common(w_f32, true, T_blocks, d_out, d_in, 32, WUSH_MXFP4, codes, scale_atoms, nullptr, nullptr,
                      false, stream, false, true);
}

int wush_quant_act_shared_mx_atoms(const void* x_bf16, const float* T_shared, int64_t n_tok, int64_t d_in,
                                   uint8_t* codes, uint8_t* scale_atoms, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_shared, n_tok, d_in, 32, WUSH_MXFP4, codes, scale_atoms, nullptr, nullptr,
                      false, stream, true, true);
}

int wush_quant_act_nv_atoms(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, uint8_t* codes,
                            uint8_t* scale_atoms, float* tensor_scale, wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, 16, WUSH_NVFP4, codes, scale_atoms, tensor_scale, nullptr,
                      false, stream, false, true);
}

int wush_quant_weight_nv_atoms(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in, uint8_t* codes,
                               uint8_t* scale_atoms, float* tensor_scale, wush_stream_t stream) {
  return quant_common(w_f32, true, T_blocks, d_out, d_in, 16, WUSH_NVFP4, codes, scale_atoms, tensor_scale, nullptr,
                      false, stream, false, true);
}

int wush_quant_act_nvfp4_amax(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, float* amax,
                              wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, 16, WUSH_NVFP4, nullptr, nullptr, amax, nullptr, false,
                      stream, false, false, kNvAmaxOnly);
}

int wush_nvfp4_scale_from_amax(float* amax_to_scale, wush_stream_t stream) {
  if (!amax_to_scale) return WUSH_ERR_INVALID_ARG;
  if (!aligned(amax_to_scale, 4)) return WUSH_ERR_MISALIGNED;
  wush::wush_nvfp4_tensor_scale_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(amax_to_scale);
  return launch_status(__LINE__);
}

int wush_quant_act_nvfp4_with_scale(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                                    uint8_t* codes, uint8_t* scales, const float* tensor_scale,
                                    wush_stream_t stream) {
  return quant_common(x_bf16, false, T_blocks, n_tok, d_in, 16, WUSH_NVFP4, codes, scales,
                      const_cast<float*>(tensor_scale), nullptr, false, stream, false, false, kNvWithScale);
}

}  // extern "C"

namespace {

// Host-side checks shared by both one-launch NVFP4 entry points, made before any CUDA
// call.  Returns WUSH_OK when the call should go on to the launch, kSkipLaunch for an
// empty batch, or the error status.
constexpr int kSkipLaunch = -1;
int onepass_check(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, const uint8_t* codes,
                  const uint8_t* scales, const float* tensor_scale) {
  if (n_tok < 0 || d_in <= 0 || d_in % 16 != 0 || n_tok > INT_MAX || d_in > INT_MAX) return WUSH_ERR_INVALID_ARG;
  if (n_tok == 0) return kSkipLaunch;
  if (!x_bf16 || !T_blocks || !codes || !scales || !tensor_scale) return WUSH_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(T_blocks, 16) || !aligned(codes, 16) || !aligned(tensor_scale, 4))
    return WUSH_ERR_MISALIGNED;
  return WUSH_OK;
}

// NVFP4 in one launch of the tensor-core kernel (batches above the CUDA-core threshold):
// one CTA per SM at most, launched cooperatively, the workspace's three words shared by
// the CTAs (see the ONEPASS walk of wush_fused_kernel).  scale_atoms: the scales go to
// the block-scaled MMA's scale-atom layout instead of row-major [rows][C].
int onepass_fused(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, uint8_t* codes,
                  uint8_t* scales, float* tensor_scale, uint32_t* workspace, wush_stream_t stream,
                  bool scale_atoms = false) {
  const int ch = WUSH_ACT_TILE_CH;
  const long long n_row_tiles = (n_tok + 127) / 128;
  const long long n_col_tiles = (d_in + ch - 1) / ch;
  if (n_row_tiles * n_col_tiles > INT_MAX) return WUSH_ERR_INVALID_ARG;
  CUtensorMap map;
  int st = encode_2d(&map, x_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_tok, d_in, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != WUSH_OK) return st;
  CUtensorMap cmap = map;
  const bool codes_tma = ((d_in / 2) % 16) == 0;
  if (codes_tma) {
    st = encode_2d(&cmap, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, n_tok, d_in / 2, ch / 2,
                   ch == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != WUSH_OK) return st;
  }
  wush::FusedParams p{};
  p.codes_via_tma = codes_tma ? 1 : 0;
  p.scale_atoms = scale_atoms ? 1 : 0;
  p.atom_cols = static_cast<int>((d_in / 16 + 3) / 4);
  p.T = T_blocks;
  p.codes = codes;
  p.scales = scales;
  p.amax_word = reinterpret_cast<unsigned int*>(workspace);
  p.tensor_scale = tensor_scale;
  p.n_rows = n_tok;
  p.d_in = static_cast<int>(d_in);
  p.C = static_cast<int>(d_in / 16);
  p.n_row_tiles = static_cast<int>(n_row_tiles);
  p.total_tiles = static_cast<int>(n_row_tiles * n_col_tiles);
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  return launch_fused<wush::FusedCfg<16, wush::kNVFP4, false, false, false, false>, false, true>(
      map, cmap, p, reinterpret_cast<cudaStream_t>(stream));
}

// The one-launch NVFP4 kernel on a checked argument set and a 16-byte aligned workspace:
// batches above the CUDA-core threshold on the tensor-core kernel when `allow_fused`,
// the CUDA-core kernel otherwise.
int onepass_launch(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, uint8_t* codes,
                   uint8_t* scales, float* tensor_scale, uint32_t* workspace, wush_stream_t stream,
                   bool allow_fused) {
  if (allow_fused && n_tok > small_rows_limit(WUSH_NVFP4))
    return onepass_fused(x_bf16, T_blocks, n_tok, d_in, codes, scales, tensor_scale, workspace, stream);
  const long long C = d_in / 16;
  const long long gy = (n_tok + wush::kSmallRows - 1) / wush::kSmallRows;
  int dev = 0, sms = 0, per_sm = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  WUSH_CUDA_CHECK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  auto kern = wush::wush_small_nvfp4_onepass_kernel<false, false>;
  WUSH_CUDA_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, wush::kSmallRows, 0));
  // the CTAs wait on one another: the whole grid must be resident at once
  if (C * gy > static_cast<long long>(per_sm) * sms || gy > 65535) return WUSH_ERR_UNSUPPORTED;
  wush::FusedParams p{};
  p.T = T_blocks;
  p.codes = codes;
  p.scales = scales;
  p.tensor_scale = tensor_scale;
  p.n_rows = n_tok;
  p.d_in = static_cast<int>(d_in);
  p.C = static_cast<int>(C);
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(C), static_cast<unsigned>(gy));
  lc.blockDim = dim3(wush::kSmallRows);
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  WUSH_CUDA_CHECK(cudaLaunchKernelEx(&lc, kern, static_cast<const __nv_bfloat16*>(x_bf16), p,
                                     reinterpret_cast<unsigned int*>(workspace)));
  return launch_status(__LINE__);
}

PFN_cuCtxGetId_v12000 context_id_getter() {
  static PFN_cuCtxGetId_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuCtxGetId_v12000>(nullptr);
    return reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  }();
  return fn;
}

}  // namespace

extern "C" {

int wush_quant_act_nvfp4_onepass(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                                 uint8_t* codes, uint8_t* scales, float* tensor_scale, uint32_t* workspace,
                                 wush_stream_t stream) {
  const int st = onepass_check(x_bf16, T_blocks, n_tok, d_in, codes, scales, tensor_scale);
  if (st == kSkipLaunch) return WUSH_OK;
  if (st != WUSH_OK) return st;
  if (!workspace) return WUSH_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return WUSH_ERR_MISALIGNED;
  return onepass_launch(x_bf16, T_blocks, n_tok, d_in, codes, scales, tensor_scale, workspace, stream, true);
}

int wush_quant_act_nv_atoms_onepass(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                                    uint8_t* codes, uint8_t* scale_atoms, float* tensor_scale, uint32_t* workspace,
                                    wush_stream_t stream) {
  const int st = onepass_check(x_bf16, T_blocks, n_tok, d_in, codes, scale_atoms, tensor_scale);
  if (st == kSkipLaunch) return WUSH_OK;
  if (st != WUSH_OK) return st;
  if (!workspace) return WUSH_ERR_INVALID_ARG;
  if (!aligned(workspace, 16) || !aligned(scale_atoms, 16)) return WUSH_ERR_MISALIGNED;
  return onepass_fused(x_bf16, T_blocks, n_tok, d_in, codes, scale_atoms, tensor_scale, workspace, stream, true);
}

int wush_quant_act_nvfp4_onepass_noalloc(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                                         uint8_t* codes, uint8_t* scales, float* tensor_scale, wush_stream_t stream) {
  // the arguments first: a rejected call touches neither CUDA nor the scratch record
  const int st = onepass_check(x_bf16, T_blocks, n_tok, d_in, codes, scales, tensor_scale);
  if (st == kSkipLaunch) return WUSH_OK;
  if (st != WUSH_OK) return st;
  int dev = 0;
  WUSH_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return WUSH_ERR_UNSUPPORTED;
  // The scratch address belongs to the module as loaded into one context.  It is recorded
  // per device together with that context's id and taken again when the id changes (the
  // primary context was reset and the module reloaded).
  const int ctx_st = ensure_context();
  if (ctx_st != WUSH_OK) return ctx_st;
  auto get_ctx = context_getter();
  auto get_id = context_id_getter();
  if (!get_id) return cuda_fail(0, "cudaGetDriverEntryPoint(cuCtxGetId)", __LINE__, true);
  CUcontext ctx = nullptr;
  unsigned long long ctx_id = 0;
  CUresult r = get_ctx(&ctx);
  if (r != CUDA_SUCCESS) return cuda_fail(r, "cuCtxGetCurrent", __LINE__, true);
  r = get_id(ctx, &ctx_id);
  if (r != CUDA_SUCCESS) return cuda_fail(r, "cuCtxGetId", __LINE__, true);
  static std::mutex mu;
  static void* scratch[64] = {};
  static unsigned long long scratch_ctx[64] = {};
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!scratch[dev] || scratch_ctx[dev] != ctx_id) {   // with that device current
      void* a = nullptr;
      WUSH_CUDA_CHECK(cudaGetSymbolAddress(&a, wush::g_noalloc_scratch));
      if (!a) return cuda_fail(cudaErrorInvalidSymbol, "cudaGetSymbolAddress", __LINE__);
      scratch[dev] = a;
      scratch_ctx[dev] = ctx_id;
    }
    ws = scratch[dev];
  }
  return onepass_launch(x_bf16, T_blocks, n_tok, d_in, codes, scales, tensor_scale, static_cast<uint32_t*>(ws),
                        stream, false);
}

int wush_set_gemm_cta_pairs(int enable) {
  g_gemm_pairs.store(enable ? 1 : 0, std::memory_order_relaxed);
  return WUSH_OK;
}

int wush_set_small_batch_rows(int64_t rows) {
  if (rows < 0) rows = -1;
  if (rows > (1 << 20)) return WUSH_ERR_INVALID_ARG;
  g_small_rows.store(rows, std::memory_order_relaxed);
  return WUSH_OK;
}

int wush_build_transforms(const float* w_f32, const void* xcal_bf16, int64_t d_out, int64_t n_cal, int64_t d_in,
                          int G, double lambda, int use_hadamard, float* T_wush, float* T_xvsh, double* T_wush64,
                          double* T_xvsh64, double* s_out, wush_stream_t stream) {
  if (G != 16 && G != 32) return WUSH_ERR_UNSUPPORTED;
  if (d_out <= 0 || n_cal <= 0 || d_in <= 0 || d_in % G != 0 || d_in > INT_MAX) return WUSH_ERR_INVALID_ARG;
  if (!(lambda >= 0.0) || lambda > 1e30) return WUSH_ERR_INVALID_ARG;
  if (!w_f32 || !xcal_bf16 || !T_wush || !T_xvsh) return WUSH_ERR_INVALID_ARG;
  if (!aligned(w_f32, 4) || !aligned(xcal_bf16, 2) || !aligned(T_wush, 4) || !aligned(T_xvsh, 4) ||
      !aligned(T_wush64, 8) || !aligned(T_xvsh64, 8) || !aligned(s_out, 8))
    return WUSH_ERR_MISALIGNED;
  wush::BuildParams p{};
  p.w = w_f32;
  p.xcal = static_cast<const __nv_bfloat16*>(xcal_bf16);
  p.d_out = d_out;
  p.n_cal = n_cal;
  p.d_in = static_cast<int>(d_in);
  p.C = static_cast<int>(d_in / G);
  p.lambda = lambda;
  p.use_hadamard = use_hadamard ? 1 : 0;
  p.T_wush = T_wush;
  p.T_xvsh = T_xvsh;
  p.T_wush64 = T_wush64;
  p.T_xvsh64 = T_xvsh64;
  p.s_out = s_out;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (G == 32) {
    constexpr int bytes = wush::BuildSmem<32>::BYTES;
    WUSH_CUDA_CHECK(
        cudaFuncSetAttribute(wush::wush_build_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    wush::wush_build_kernel<32><<<p.C, wush::kBuildThreads, bytes, s>>>(p);
  } else {
    constexpr int bytes = wush::BuildSmem<16>::BYTES;
    WUSH_CUDA_CHECK(
        cudaFuncSetAttribute(wush::wush_build_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    wush::wush_build_kernel<16><<<p.C, wush::kBuildThreads, bytes, s>>>(p);
  }
  return launch_status(__LINE__);
}

int wush_hadamard(int G, int64_t copies, float* out, wush_stream_t stream) {
  if (G < 1 || G > 256 || (G & (G - 1)) != 0) return WUSH_ERR_UNSUPPORTED;
  if (copies < 0 || copies > (int64_t(1) << 40) / (int64_t(G) * G)) return WUSH_ERR_INVALID_ARG;
  if (copies == 0) return WUSH_OK;
  if (!out) return WUSH_ERR_INVALID_ARG;
  if (!aligned(out, 4)) return WUSH_ERR_MISALIGNED;
  const long long total = static_cast<long long>(copies) * G * G;
  const long long blocks = (total + 255) / 256;
  wush::wush_hadamard_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(G, total, out);
  return launch_status(__LINE__);
}

int wush_device_status(wush_stream_t stream, uint32_t* bits) {
  WUSH_CUDA_CHECK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned int word = 0u, zero = 0u;
  WUSH_CUDA_CHECK(cudaMemcpyFromSymbol(&word, wush::g_wush_device_error, sizeof(word)));
  if (word) WUSH_CUDA_CHECK(cudaMemcpyToSymbol(wush::g_wush_device_error, &zero, sizeof(zero)));
  if (bits) *bits = word;
  return word ? WUSH_ERR_DEVICE_TIMEOUT : WUSH_OK;
}

int wush_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns ? ns : kDefaultWaitLimitNs, std::memory_order_relaxed);
  return WUSH_OK;
}

int wush_selftest_wait_timeout(uint64_t limit_ns, wush_stream_t stream, uint32_t* bits) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wush::wush_selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns);
  WUSH_CUDA_CHECK(cudaGetLastError());
  uint32_t word = 0;
  const int st = wush_device_status(stream, &word);
  if (bits) *bits = word;
  return st;
}

const char* wush_status_string(int status) {
  switch (status) {
    case WUSH_OK: return "WUSH_OK";
    case WUSH_ERR_INVALID_ARG: return "WUSH_ERR_INVALID_ARG: null pointer or bad size";
    case WUSH_ERR_UNSUPPORTED: return "WUSH_ERR_UNSUPPORTED: format or group size not supported";
    case WUSH_ERR_MISALIGNED: return "WUSH_ERR_MISALIGNED: pointer alignment requirement not met";
    case WUSH_ERR_CUDA: return "WUSH_ERR_CUDA: CUDA runtime error";
    case WUSH_ERR_DEVICE_TIMEOUT: return "WUSH_ERR_DEVICE_TIMEOUT: an in-kernel wait expired";
    default: return "unknown wush status";
  }
}

int wush_last_error_detail(char* buf, size_t len) {
  const CudaFailure f = t_cuda_failure;
  char tmp[512];
  if (!f.what) {
    snprintf(tmp, sizeof(tmp), "no CUDA failure recorded on this thread");
  } else if (f.driver) {
    snprintf(tmp, sizeof(tmp), "%s (wush_api.cu:%d) failed: CUresult %d", f.what, f.line, f.code);
  } else {
    const cudaError_t e = static_cast<cudaError_t>(f.code);
    snprintf(tmp, sizeof(tmp), "%s (wush_api.cu:%d) failed: %s: %s", f.what, f.line, cudaGetErrorName(e),
             cudaGetErrorString(e));
  }
  const int n = static_cast<int>(strlen(tmp));
  if (buf && len) {
    const size_t k = static_cast<size_t>(n) < len - 1 ? static_cast<size_t>(n) : len - 1;
    memcpy(buf, tmp, k);
    buf[k] = '\0';
  }
  return n;
}

int wush_version(void) { return 100; }

}  // extern "C"
