/*
 * wush.h - C ABI of the B200 (sm_100a) fused WUSH transform + 4-bit quantisation library.
 *
 * What the library computes.  Sources are pages describing arXiv 2512.00956, "WUSH:
 * Near-Optimal Adaptive Transforms for LLM Quantization":
 *   - paper-graph-ui analysis, section 3.2 "Big-Picture Architecture": the "Online
 *     Activation Transform + Quantize Kernel" multiplies each incoming activation block
 *     by its own T_wush,i and quantises it on the fly; the "Weight Pre-Quantizer"
 *     applies the weight-side transform to the weight block and quantises it with RTN.
 *   - same page, section 3.4.7 "GPU Kernel Design": tokens x d_in activations; C = d_in/G
 *     independent (M x G) x (G x G) products, one G x G matrix per block.
 *   - same page, section 3.4.1: block size G = quantisation group size (32 for MXFP4,
 *     16 for NVFP4); G is a power of two dividing d_in.
 *   - ai.info summary, authors' abstract: "RTN AbsMax-scaled block quantizers".
 *   - papernotes.org summary, section "整体框架": activations use T_wush, weights use
 *     T_xvsh = T_wush^-T.
 *
 * Layouts (all row-major, no padding):
 *   x          bf16  [n_tok][d_in]            activations, one row per token
 *   w          fp32  [d_out][d_in]            weights, one row per output channel
 *   T_blocks   fp32  [C][G][G]                element (i, r, c) at (i*G + r)*G + c is
 *                                             (T_i)_{r,c}; y_r = sum_c (T_i)_{r,c} x_c
 *   codes      u8    [rows][d_in/2]           4-bit codes, byte j holds element 2j in the
 *                                             low nibble and element 2j+1 in the high one
 *   scales     MXFP4: u8 [rows][C]            E8M0 byte e + 127, group value = code * 2^e
 *              NVFP4: u8 [rows][C]            E4M3 block scale, value = code * dec * s_t
 *              INT4 : fp32 [rows][C]          value = signed nibble * scale
 *   tensor_scale fp32 [1]                     NVFP4 only: s_t = amax|y| / (6 * 448)
 * with rows = n_tok (activations) or d_out (weights).
 *
 * Codes.  E2M1 (MXFP4, NVFP4): bit 3 is the sign, bits 0-2 index the grid
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}; rounding is to nearest with ties to the even code and
 * saturation at 6; 0x0 and 0x8 both encode zero.  INT4: two's-complement nibble in
 * [-7, 7], round to nearest even.  Scale rules:
 *   MXFP4  e = least integer with amax <= 6 * 2^e, clamped to [-127, 127]
 *   NVFP4  sb = E4M3(amax / (6 s_t)); y is multiplied by the fp32 reciprocal of dec(sb)*s_t
 *   INT4   s = amax / 7; y is multiplied by the fp32 reciprocal of s
 * A group whose scale reciprocal is not a finite fp32 encodes as all zero.
 *
 * Supported (fmt, G): (MXFP4, 32), (NVFP4, 16), (INT4, 16), (INT4, 32).
 *
 * Ownership and execution.  Every pointer argument of the quantisation calls is
 * caller-owned DEVICE memory on the current CUDA device.  Calls are asynchronous on
 * `stream` (0 = legacy default stream), never synchronise the host, allocate nothing
 * and keep no state between calls except the device error word described at
 * wush_device_status().  Inputs must be finite; NaN or Inf gives unspecified codes.
 * Calls may be made from several host threads and on several streams at once.
 *
 * Launch order.  The quantisers, the NVFP4 steps and the FP4 GEMMs launch with
 * programmatic stream serialisation.  Each kernel lets the next kernel in the stream
 * begin early, but reads nothing before the previous kernel has completed
 * (griddepcontrol.wait).  A kernel of the caller's that follows one of these
 * launches in the same stream behaves normally.  If it is launched with the
 * programmatic-serialisation attribute itself, it must likewise wait
 * (griddepcontrol.wait, or cudaGridDependencySynchronize) before reading their outputs.
 *
 * Errors.  Arguments are checked on the host before any launch:
 *   WUSH_ERR_INVALID_ARG   NULL pointer, n_tok/d_out < 0, d_in <= 0, d_in % G != 0,
 *                          a size beyond 2^31 - 1 rows or 2^31 - 1 channels
 *   WUSH_ERR_UNSUPPORTED   unknown fmt or an unsupported (fmt, G) pair
 *   WUSH_ERR_MISALIGNED    x, w, T_blocks, codes, y_out not 16-byte aligned; INT4 scales
 *                          or tensor_scale not 4-byte aligned
 *   WUSH_ERR_CUDA          a CUDA runtime error while launching (including a missing or
 *                          non-sm_100 device); wush_last_error_detail() names the call
 * Bits of the device error word (wush_device_status): 1/2/4/8/16 a wait of the TMA
 * producer / MMA issuer / converter / epilogue / final drain expired, 32 the wait
 * self-test expired (expected), 64 a Cholesky pivot was not positive, 128 a CTA of the
 * one-launch NVFP4 path waited in vain for the rest of its grid.
 * rows == 0 (with a supported fmt/G and a valid d_in) returns WUSH_OK without launching
 * anything; its pointers are then not checked and may be NULL.
 */
#ifndef WUSH_H_
#define WUSH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* wush_stream_t;

typedef enum { WUSH_MXFP4 = 0, WUSH_NVFP4 = 1, WUSH_INT4 = 2 } wush_fmt;

typedef enum {
  WUSH_OK = 0,
  WUSH_ERR_INVALID_ARG = 1,
  WUSH_ERR_UNSUPPORTED = 2,
  WUSH_ERR_MISALIGNED = 3,
  WUSH_ERR_CUDA = 4,
  WUSH_ERR_DEVICE_TIMEOUT = 5
} wush_status;

/* Online activation path: y = T_wush,i x per token and block, then AbsMax quantise.
 * For NVFP4 the call makes two passes over x (the first finds amax|y| for s_t) and
 * writes s_t to *tensor_scale, which also serves as the running-max word of the first
 * pass; tensor_scale may be NULL for the other formats. */
int wush_quant_act(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in, int G,
                   int fmt, uint8_t* codes, void* scales, float* tensor_scale, wush_stream_t stream);

/* Weight pre-quantisation: W_bar = T_xvsh,i w per output channel and block, then AbsMax
 * quantise; w is fp32 [d_out][d_in].  Same outputs and rules as wush_quant_act. */
int wush_quant_weight(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in, int G,
                      int fmt, uint8_t* codes, void* scales, float* tensor_scale,
                      wush_stream_t stream);

/* Test variants: identical kernels that additionally write the fp32 transformed values
 * y [rows][d_in] they quantised (device memory, 16-byte aligned), so that the
 * quantiser can be checked bit for bit against an independent implementation fed the
 * same y. */
int wush_quant_act_debug(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                         int G, int fmt, uint8_t* codes, void* scales, float* tensor_scale,
                         float* y_out, wush_stream_t stream);
int wush_quant_weight_debug(const float* w_f32, const float* T_blocks, int64_t d_out, int64_t d_in,
                            int G, int fmt, uint8_t* codes, void* scales, float* tensor_scale,
                            float* y_out, wush_stream_t stream);

/* H+Quant comparator: the same fused kernel with ONE G x G matrix shared by every block
 * (the pages' uniform blockwise Hadamard baseline "H + Quant", against which the fused
 * per-block WUSH kernel is compared: paper-graph-ui analysis, section 3.4.7 "GPU Kernel
 * Design" and section 5 "GPU Kernel Benchmarks (Figure 2)").
 *   y[t, iG + r] = sum_c T_shared[r, c] x[t, iG + c]   for every block i,
 * then the same quantisers, layouts, tensor-scale handling and errors as wush_quant_act.
 * T_shared: fp32 [G][G] row-major (device memory, 16-byte aligned), e.g. the normalised
 * Sylvester Hadamard matrix rounded to fp32.  The matrix is converted once per CTA and
 * stays resident in shared memory.  The _debug form also writes the fp32 y it quantised. */
int wush_quant_act_shared(const void* x_bf16, const float* T_shared, int64_t n_tok, int64_t d_in,
                          int G, int fmt, uint8_t* codes, void* scales, float* tensor_scale,
                          wush_stream_t stream);
int wush_quant_act_shared_debug(const void* x_bf16, const float* T_shared, int64_t n_tok,
                                int64_t d_in, int G, int fmt, uint8_t* codes, void* scales,
                                float* tensor_scale, float* y_out, wush_stream_t stream);

/* Dequantisation: codes + scales (the layouts written by the calls above) -> fp32
 * values out [rows][d_in] (device memory, 16-byte aligned; codes 4-byte aligned).
 *   MXFP4: e2m1 * 2^(scale - 127);  NVFP4: e2m1 * e4m3(scale) * (*tensor_scale);
 *   INT4:  q * scale.
 * Each value is the exact product rounded once to fp32.  This is the "fake quantised"
 * operand of the layerwise-loss measurements (paper-graph-ui analysis, section 5,
 * "Metrics" and "Per-Layer Quantization Loss (Table 1)").  Same G / format rules and
 * errors as wush_quant_act; rows == 0 returns WUSH_OK without touching the pointers. */
int wush_dequant(const uint8_t* codes, const void* scales, const float* tensor_scale, int64_t rows,
                 int64_t d_in, int G, int fmt, float* out, wush_stream_t stream);

/* FP4 GEMM consumer: D = A * B^T in bf16 from MXFP4 operands, on block-scaled tcgen05
 * MMAs (the "FP4 MatMul" after WUSH + Quant: paper-graph-ui analysis, section 3.4.7
 * "GPU Kernel Design"; section 5 "GPU Kernel Benchmarks (Figure 2)").
 *   D[m][n] = sum_k A[m][k] B[n][k]      (fp32 accumulation, one bf16 rounding)
 * a_codes u8 [M][K/2] (e.g. wush_quant_act's MXFP4 codes), b_codes u8 [N][K/2] (e.g.
 * wush_quant_weight's, one row per output channel), both E2M1 pairs, low nibble = even k.
 * a_atoms / b_atoms: the E8M0 scales in the tcgen05 scale-atom layout (see
 * wush_mx_scales_to_atoms).  d_bf16: [M][N] row-major.  All device memory, 16-byte aligned.
 * Supported: M % 128 == 0, N % 256 == 0, K % 256 == 0 (else WUSH_ERR_UNSUPPORTED).
 * Asynchronous on `stream`; allocates nothing. */
int wush_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_atoms, const uint8_t* b_codes,
                    const uint8_t* b_atoms, int64_t M, int64_t N, int64_t K, void* d_bf16,
                    wush_stream_t stream);

/* The same GEMM for NVFP4 operands: E2M1 codes with one E4M3 scale per 16 elements
 * (kind::mxf4nvf4 block16 MMAs) and one fp32 tensor scale per operand:
 *   D[m][n] = s_A s_B sum_k (e2m1 e4m3)_A[m][k] (e2m1 e4m3)_B[n][k]
 * (fp32 accumulation, the sum times fl32(s_A s_B) in fp32, one bf16 rounding).
 * a_atoms / b_atoms: the E4M3 scale bytes [rows][K/16] in the scale-atom layout (see
 * wush_mx_scales_to_atoms, which relays out any one-byte scales, or the *_nv_atoms
 * quantisers); a_tensor_scale / b_tensor_scale: device fp32 (the quantisers' s_t).
 * Same shapes, alignment and errors as wush_gemm_mxfp4 (NULL tensor scales:
 * WUSH_ERR_INVALID_ARG; not 4-byte aligned: WUSH_ERR_MISALIGNED). */
int wush_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_tensor_scale,
                    const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_tensor_scale,
                    int64_t M, int64_t N, int64_t K, void* d_bf16, wush_stream_t stream);

/* MXFP4 (G = 32) quantisation that writes its E8M0 scales straight into the scale-atom
 * layout wush_gemm_mxfp4 reads (instead of row-major [rows][C]): the same kernels,
 * codes and errors as wush_quant_act / wush_quant_weight / wush_quant_act_shared with
 * fmt = MXFP4.  scale_atoms (device) must hold atom_bytes = rows_pad * C_pad bytes
 * (rows padded to 128, C = d_in / 32 padded to 4); bytes of padding rows and columns
 * are not written. */
int wush_quant_act_mx_atoms(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                            uint8_t* codes, uint8_t* scale_atoms, wush_stream_t stream);
int wush_quant_weight_mx_atoms(const float* w_f32, const float* T_blocks, int64_t d_out,
                               int64_t d_in, uint8_t* codes, uint8_t* scale_atoms,
                               wush_stream_t stream);
int wush_quant_act_shared_mx_atoms(const void* x_bf16, const float* T_shared, int64_t n_tok,
                                   int64_t d_in, uint8_t* codes, uint8_t* scale_atoms,
                                   wush_stream_t stream);

/* NVFP4 (G = 16) quantisation that writes its E4M3 scales in the scale-atom layout
 * wush_gemm_nvfp4 reads: the same kernels, codes, tensor scale and errors as
 * wush_quant_act / wush_quant_weight with fmt = NVFP4.  scale_atoms (device, 16-byte
 * aligned) must hold atom_bytes = rows_pad * C_pad bytes (C = d_in / 16); bytes of
 * padding rows and columns are not written.  tensor_scale: device fp32, written. */
int wush_quant_act_nv_atoms(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                            uint8_t* codes, uint8_t* scale_atoms, float* tensor_scale,
                            wush_stream_t stream);
int wush_quant_weight_nv_atoms(const float* w_f32, const float* T_blocks, int64_t d_out,
                               int64_t d_in, uint8_t* codes, uint8_t* scale_atoms,
                               float* tensor_scale, wush_stream_t stream);

/* NVFP4 activations in stages, for a batch whose rows are split across ranks: the
 * tensor scale s_t = amax / (6 * 448) must then come from the AbsMax over all ranks'
 * transformed values (a max-reduction between the stages; the single-call
 * wush_quant_act does all three steps on one device).
 *   wush_quant_act_nvfp4_amax: *amax (device fp32) = max |y| over this batch (0 for an
 *     empty batch), y = the G = 16 WUSH transform of x; writes no codes or scales.
 *   wush_nvfp4_scale_from_amax: in place, *p = fl32(*p / 2688) (one thread).
 *   wush_quant_act_nvfp4_with_scale: codes and E4M3 scales of x under the given device
 *     fp32 tensor scale (read only) — the quantising pass of wush_quant_act.
 * Same layouts, alignment and errors as wush_quant_act with fmt = NVFP4, G = 16; the
 * three calls together give wush_quant_act's result bit for bit.  Asynchronous on
 * `stream`, allocate nothing. */
int wush_quant_act_nvfp4_amax(const void* x_bf16, const float* T_blocks, int64_t n_tok, int64_t d_in,
                              float* amax, wush_stream_t stream);
int wush_nvfp4_scale_from_amax(float* amax_to_scale, wush_stream_t stream);
int wush_quant_act_nvfp4_with_scale(const void* x_bf16, const float* T_blocks, int64_t n_tok,
                                    int64_t d_in, uint8_t* codes, uint8_t* scales,
                                    const float* tensor_scale, wush_stream_t stream);

/* Row-major one-byte scales [rows][C] (E8M0 or E4M3) -> the scale-atom layout the
 * block-scaled MMA reads:
 * rows padded to a multiple of 128 and C to a multiple of 4 (zero bytes); the atom of
 * row block r and scale columns [4c, 4c + 4) is the 512 bytes at (r * (C_pad/4) + c) * 512,
 * holding row 128 r + i + 32 j, column 4 c + k at byte 16 i + 4 j + k (i < 32, j < 4,
 * k < 4).  `atoms` (device) must hold rows_pad * C_pad bytes.  This layout is NVIDIA's
 * tcgen05 block-scale format, not something the pages define. */
int wush_mx_scales_to_atoms(const uint8_t* scales, int64_t rows, int64_t C, uint8_t* atoms,
                            wush_stream_t stream);

/* Transform construction for one layer, on the device, in fp64 (one CTA per block).
 * Sources: paper-graph-ui analysis, section 3.2 "Second-Moment Computer" and "Transform
 * Constructor", sections 3.4.2 and 3.4.4 (Eq. 8); papernotes.org summary, "关键设计";
 * ai.info summary, "Methodology in Plain English" (damping of the diagonals).
 *   Sigma_w = d_out^-1 W_(i) W_(i)^T, Sigma_x = n_cal^-1 X_(i) X_(i)^T          per block i
 *   Sigma  += lambda * mean(diag Sigma) * I                                   (both sides)
 *   W' = chol(Sigma_w), X' = chol(Sigma_x)  (lower);  W'^T X' = U S V^T
 *   T_wush = H S^-1/2 U^T W'^T,  T_xvsh = H S^-1/2 V^T X'^T = T_wush^-T
 * H is the normalised Sylvester Hadamard matrix (use_hadamard = 0 replaces it by I).
 * Singular values are sorted descending; each pair (u_k, v_k) is flipped so that the
 * largest-magnitude entry of u_k is positive.
 * Inputs (device): w_f32 [d_out][d_in], xcal_bf16 [n_cal][d_in] calibration activations.
 * Outputs (device): T_wush, T_xvsh fp32 [C][G][G] (the fp64 results rounded once);
 * optional (may be NULL) T_wush64, T_xvsh64 fp64 [C][G][G] and s_out fp64 [C][G].
 * G in {16, 32}.  A Cholesky pivot at or below 1e-12 of the mean (damped) diagonal
 * (e.g. lambda = 0 on rank-deficient data) sets bit 64 of the device error word (see
 * wush_device_status) and yields unusable T.
 * Errors: WUSH_ERR_UNSUPPORTED (G), WUSH_ERR_INVALID_ARG (NULL input/output, sizes,
 * lambda < 0 or not finite), WUSH_ERR_MISALIGNED (fp32 pointers not 4-byte, bf16 not
 * 2-byte, fp64 not 8-byte aligned), WUSH_ERR_CUDA.  Asynchronous on `stream`, allocates
 * nothing. */
int wush_build_transforms(const float* w_f32, const void* xcal_bf16, int64_t d_out, int64_t n_cal,
                          int64_t d_in, int G, double lambda, int use_hadamard, float* T_wush,
                          float* T_xvsh, double* T_wush64, double* T_xvsh64, double* s_out,
                          wush_stream_t stream);

/* Writes `copies` consecutive copies of the normalised Sylvester Hadamard matrix H of
 * order G into out, fp32 [copies][G][G] row-major: entry (r, c) = (-1)^popcount(r & c) /
 * sqrt(G), i.e. H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]] scaled by G^-1/2, so that
 * H H^T = I.  This is the H of T = H S^-1/2 U^T W'^T (paper-graph-ui analysis, sections
 * 3.4.4 "Hadamard" and 3.2; papernotes.org "关键设计"); one copy is the shared matrix of
 * wush_quant_act_shared (the H+Quant comparator), `C` copies are the per-block matrices of
 * the Hadamard-only transform.  Entries are formed in fp64 and rounded once to fp32.
 * out: caller-owned device memory of copies * G * G floats, 4-byte aligned.
 * Errors: WUSH_ERR_UNSUPPORTED (G not a power of two in [1, 256]), WUSH_ERR_INVALID_ARG
 * (copies < 0 or more than 2^40 entries, out NULL with copies > 0), WUSH_ERR_MISALIGNED,
 * WUSH_ERR_CUDA.  copies = 0 returns WUSH_OK without a launch.  Asynchronous on `stream`. */
int wush_hadamard(int G, int64_t copies, float* out, wush_stream_t stream);

/* Every wait inside the kernels is bounded in time (default 2 s).  When one expires
 * the kernel records a bit in a per-device error word and returns early; outputs of
 * that call are then unspecified.  wush_device_status() synchronises `stream`, reads
 * and clears the word of the current device and returns WUSH_OK or
 * WUSH_ERR_DEVICE_TIMEOUT (WUSH_ERR_CUDA if the runtime reports an error).  If
 * `bits` is not NULL it receives the raw word. */
int wush_device_status(wush_stream_t stream, uint32_t* bits);

/* enable != 0: the FP4 GEMMs with M % 256 == 0 run on pairs of CTAs (clusters of two SMs
 * sharing M = 256 block-scaled MMAs, B split between them along N); enable = 0 (the
 * default) keeps every call on single CTAs, which measured faster on B200 at the
 * benchmarked shapes.  Same results either way up to the order of fp32 accumulation.
 * Applies to later calls; returns WUSH_OK. */
int wush_set_gemm_cta_pairs(int enable);

/* NVFP4 activations in ONE launch (wush_quant_act with fmt = NVFP4 takes four: a clear of
 * the tensor-scale word, the amax pass, the tensor-scale step and the quantising pass).
 * The tensor scale s_t = amax|y| / 2688 needs the whole batch's maximum before any group
 * can be quantised, so the CTAs meet once through the caller's workspace: each folds its
 * max |y| into workspace[0], counts itself into workspace[1] and waits — bounded by the
 * wait limit, error bit 128 on expiry — until the whole grid has arrived, then quantises
 * with s_t; the last CTA to leave returns the words to zero.  The grid is launched
 * cooperatively (all of it resident at once).
 *   - Batches of at most the CUDA-core threshold (wush_set_small_batch_rows; 256 rows by
 *     default) run on CUDA cores, one CTA per 16-channel block and 128 rows; such a grid
 *     that cannot be resident at once returns WUSH_ERR_UNSUPPORTED (use wush_quant_act).
 *   - Larger batches run on the tensor-core kernel, one CTA per SM: each CTA walks its
 *     tiles forwards for max |y| and, after the meeting, backwards to quantise, so that it
 *     first re-reads the tiles it loaded last while they are still in L2.
 * Outputs and layouts as wush_quant_act with fmt = NVFP4, G = 16; codes, scales and
 * tensor scale bit-identical to it whenever both take the same kind of kernel (both at
 * most the threshold, or both above it).
 * workspace: device memory of at least 16 bytes, 16-byte aligned, ZERO before the first
 * call; every call that completes without a device error leaves it zero again.  Calls
 * that may overlap (other streams) need workspaces of their own.
 * Other errors as wush_quant_act; the workspace must be 16-byte aligned.
 * The pages have no counterpart: it is a launch-count path (the tensor scale's two passes
 * in one launch). */
int wush_quant_act_nvfp4_onepass(const void* x_bf16, const float* T_blocks, int64_t n_tok,
                                 int64_t d_in, uint8_t* codes, uint8_t* scales,
                                 float* tensor_scale, uint32_t* workspace, wush_stream_t stream);

/* As wush_quant_act_nvfp4_onepass, with the E4M3 scales written in the scale-atom layout
 * wush_gemm_nvfp4 reads (as wush_quant_act_nv_atoms): the activation side of an NVFP4
 * layer in one launch.  Every batch, decode-sized ones included, runs on the tensor-core
 * kernel (one cooperative launch, one CTA per SM at most).  Codes, scale atoms and tensor
 * scale are bit-identical to wush_quant_act_nv_atoms whenever that call takes the
 * tensor-core kernel too (batches above the CUDA-core threshold).  scale_atoms (device,
 * 16-byte aligned) must hold atom_bytes = rows_pad * C_pad bytes (C = d_in / 16); bytes of
 * padding rows and columns are not written.  workspace: as wush_quant_act_nvfp4_onepass
 * (16 bytes, 16-byte aligned, zero before the first call and left zero by each; one per
 * stream whose calls may overlap).  Errors as wush_quant_act_nvfp4_onepass. */
int wush_quant_act_nv_atoms_onepass(const void* x_bf16, const float* T_blocks, int64_t n_tok,
                                    int64_t d_in, uint8_t* codes, uint8_t* scale_atoms,
                                    float* tensor_scale, uint32_t* workspace, wush_stream_t stream);

/* The one-launch NVFP4 path without a caller workspace: it uses a 256-byte file-scope
 * static device array of the library (3 words of it), whose address is taken once per
 * device with cudaGetSymbolAddress; nothing is allocated.  The scratch is zero when the
 * library is loaded and every call that completes without a device error leaves it zero;
 * after a call that records error bit 128 it is not zero any more and this entry point
 * must not be used again in the process (wush_quant_act_nvfp4_onepass with a fresh
 * workspace still works).  All calls share the one scratch per device: calls that may
 * overlap (several streams, several host threads) race and give wrong results — use
 * wush_quant_act_nvfp4_onepass with a workspace each there.  Arguments are checked
 * first; a rejected call makes no CUDA call.  The first accepted call on a device, and
 * the first after that device's context was reset (the library notices the new context
 * id and takes the address again), resolves the scratch address: make it before any
 * stream capture.  Requests the
 * one-launch path cannot take (a grid of d_in/16 x ceil(n_tok/128) CTAs that is not
 * resident at once) return WUSH_ERR_UNSUPPORTED; a current device ordinal above 63 also
 * returns WUSH_ERR_UNSUPPORTED; otherwise as wush_quant_act_nvfp4_onepass.
 * It always takes the CUDA-core kernel (batches above the CUDA-core threshold included);
 * wush_quant_act_nvfp4_onepass with a workspace also has the tensor-core one-launch path.
 * The pages have no counterpart: it only spares the caller a workspace allocation. */
int wush_quant_act_nvfp4_onepass_noalloc(const void* x_bf16, const float* T_blocks, int64_t n_tok,
                                         int64_t d_in, uint8_t* codes, uint8_t* scales,
                                         float* tensor_scale, wush_stream_t stream);

/* Activation batches (bf16 input; row-major scales or the scale-atom layout) of at most
 * `rows` rows take a
 * CUDA-core path instead of the fused tensor-core kernel: one CTA per block and 128 rows,
 * T_i staged in shared memory, y = T_i x in fp32 FMAs, then the same group quantisers
 * (codes, scales and NVFP4 tensor scale in the same layouts; y differs from the tensor-core
 * path's by fp32 rounding only).  At decode sizes the fused kernel's fixed start-up
 * latency dominates.  rows = 0 sends every batch to the fused kernel; rows < 0 restores
 * the default, which depends on the format (MXFP4 64 rows, INT4 and NVFP4 256: the
 * measured crossovers at d_in = 4096); rows > 0 applies to every format.  Applies to later
 * calls on every device; returns WUSH_OK, or WUSH_ERR_INVALID_ARG above 2^20 rows. */
int wush_set_small_batch_rows(int64_t rows);

/* Sets the bound of every in-kernel wait for later launches, in nanoseconds
 * (0 restores the default of 2 s).  Returns WUSH_OK. */
int wush_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded-wait path: launches one CTA that waits on an mbarrier no
 * thread ever arrives on, with a limit of `limit_ns`; the wait must give up, record
 * its bit and return.  Synchronises `stream` and returns the error word it produced
 * (expected: 32).  Does not fault or hang the device. */
int wush_selftest_wait_timeout(uint64_t limit_ns, wush_stream_t stream, uint32_t* bits);

/* Human-readable name of a wush_status value (static string, never NULL). */
const char* wush_status_string(int status);

/* The call behind the last WUSH_ERR_CUDA that a wush_* function returned on the calling
 * host thread: its name, the source line in the library, and the CUDA runtime's error
 * name and message (or the driver's CUresult for a tensor-map encoding).  The record is
 * per host thread and is overwritten by the next such failure on that thread; it is not
 * cleared by calls that succeed.  Writes at most len - 1 characters and a terminating NUL
 * into buf (nothing if buf is NULL or len is 0) and returns the full length of the
 * message.  Never fails. */
int wush_last_error_detail(char* buf, size_t len);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int wush_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WUSH_H_ */
