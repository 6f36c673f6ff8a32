// Per-block WUSH transform construction on the GPU, in fp64, one CTA per block.
//
// Steps (paper-graph-ui analysis of arXiv 2512.00956, §3.2 "Second-Moment Computer" and
// "Transform Constructor", §3.4.2 and §3.4.4 Eq. (8); papernotes.org summary, 关键设计):
//   Sigma_w = d_out^-1 W_(i) W_(i)^T,  Sigma_x = d_batch^-1 X_(i) X_(i)^T
//   Sigma  <- Sigma + lambda * mean(diag Sigma) * I             (damping; value not on the pages)
//   W' = chol(Sigma_w), X' = chol(Sigma_x)                        (lower triangular)
//   W'^T X' = U S V^T                                             (one-sided Jacobi SVD)
//   T_wush = H S^-1/2 U^T W'^T   (activations),  T_xvsh = H S^-1/2 V^T X'^T   (weights)
// with H the normalised Sylvester Hadamard matrix (entry (r, c) = (-1)^popcount(r & c) / sqrt(G)).
// Singular values are sorted descending; each pair (u_k, v_k) is flipped so that the
// largest-magnitude entry of u_k is positive (lowest index on ties).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "wush_ptx.cuh"

namespace wush {

struct BuildParams {
  const float* w;               // [d_out][d_in] fp32
  const __nv_bfloat16* xcal;    // [n_cal][d_in] bf16
  long long d_out, n_cal;
  int d_in, C;
  double lambda;
  int use_hadamard;
  float* T_wush;                // [C][G][G]
  float* T_xvsh;
  double* T_wush64;             // optional
  double* T_xvsh64;             // optional
  double* s_out;                // optional [C][G]
};

constexpr int kBuildThreads = 256;
constexpr int kBuildRows = 64;    // rows staged per pass of the second-moment loop

template <int G>
struct BuildSmem {
  static constexpr int GG = G * G;
  // doubles: Sw, Sx (become W', X'), A (col-major, becomes U*S), V (col-major), U2, V2, Bw, Bx,
  // staging [kBuildRows][G], sigma[G], misc
  static constexpr int OFF_SW = 0, OFF_SX = GG, OFF_A = 2 * GG, OFF_V = 3 * GG, OFF_U2 = 4 * GG,
                       OFF_V2 = 5 * GG, OFF_BW = 6 * GG, OFF_BX = 7 * GG, OFF_STAGE = 8 * GG,
                       OFF_SIG = OFF_STAGE + kBuildRows * G, OFF_SIG2 = OFF_SIG + G, N_DOUBLES = OFF_SIG2 + G;
  static constexpr int BYTES = N_DOUBLES * 8 + 16;
};

__device__ __forceinline__ double warp_sum_seg(double v, int seg) {
  for (int o = seg >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Accumulate the G x G second moment of `rows` rows of block `blk` into per-thread
// partial sums (entries t, t + 256, ...), reading fp32 or bf16 rows.
template <int G, typename SrcT>
__device__ void second_moment(const SrcT* src, long long rows, int d_in, int blk, double* stage,
                              double* out) {
  constexpr int GG = G * G;
  constexpr int PER = (GG + kBuildThreads - 1) / kBuildThreads;
  double acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.0;
  for (long long r0 = 0; r0 < rows; r0 += kBuildRows) {
    const int nr = static_cast<int>(rows - r0 < kBuildRows ? rows - r0 : kBuildRows);
    for (int idx = threadIdx.x; idx < kBuildRows * G; idx += kBuildThreads) {
      const int rr = idx / G, cc = idx - rr * G;
      double v = 0.0;
      if (rr < nr) {
        const SrcT e = src[(r0 + rr) * d_in + static_cast<long long>(blk) * G + cc];
        if constexpr (sizeof(SrcT) == 4) v = static_cast<double>(e);
        else v = static_cast<double>(__bfloat162float(e));
      }
      stage[idx] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + k * kBuildThreads;
      if (e < GG) {
        const int r = e / G, c = e - r * G;
        double a = acc[k];
        for (int rr = 0; rr < nr; ++rr) a = fma(stage[rr * G + r], stage[rr * G + c], a);
        acc[k] = a;
      }
    }
    __syncthreads();
  }
  const double inv_n = 1.0 / static_cast<double>(rows);
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + k * kBuildThreads;
    if (e < GG) out[e] = acc[k] * inv_n;
  }
}

template <int G>
__global__ void __launch_bounds__(kBuildThreads) wush_build_kernel(const BuildParams p) {
  using L = BuildSmem<G>;
  constexpr int GG = G * G;
  extern __shared__ double bsm[];
  double* Sw = bsm + L::OFF_SW;
  double* Sx = bsm + L::OFF_SX;
  double* A = bsm + L::OFF_A;    // column-major: A[c * G + r]
  double* V = bsm + L::OFF_V;    // column-major
  double* U2 = bsm + L::OFF_U2;
  double* V2 = bsm + L::OFF_V2;
  double* Bw = bsm + L::OFF_BW;
  double* Bx = bsm + L::OFF_BX;
  double* stage = bsm + L::OFF_STAGE;
  double* sig = bsm + L::OFF_SIG;
  double* sig2 = bsm + L::OFF_SIG2;
  int* flag = reinterpret_cast<int*>(bsm + L::N_DOUBLES);
  const int blk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- second moments
  second_moment<G, float>(p.w, p.d_out, p.d_in, blk, stage, Sw);
  second_moment<G, __nv_bfloat16>(p.xcal, p.n_cal, p.d_in, blk, stage, Sx);
  __syncthreads();

  // ---- damping: Sigma += lambda * tr(Sigma) / G * I
  // pivots at or below 1e-12 of the mean diagonal count as "not positive definite"
  double* piv_floor = sig2;   // two doubles of scratch until the SVD needs sig2
  if (tid < 2) {
    double* S = tid == 0 ? Sw : Sx;
    double tr = 0.0;
    for (int k = 0; k < G; ++k) tr += S[k * G + k];
    const double add = p.lambda * tr / G;
    for (int k = 0; k < G; ++k) S[k * G + k] += add;
    piv_floor[tid] = 1e-12 * (tr / G + add);
  }
  if (tid == 0) flag[0] = 0;
  __syncthreads();

  // ---- Cholesky, right-looking, in place (threads 0..127 on Sw, 128..255 on Sx)
  {
    double* S = tid < 128 ? Sw : Sx;
    const double floor_k = piv_floor[tid < 128 ? 0 : 1];
    const int lt = tid & 127;
    for (int k = 0; k < G; ++k) {
      if (lt == 0) {
        const double piv = S[k * G + k];
        if (!(piv > floor_k)) {
          atomicOr(&g_wush_device_error, 64u);
          S[k * G + k] = 1.0;
        } else {
          S[k * G + k] = sqrt(piv);
        }
      }
      __syncthreads();
      const double d = S[k * G + k];
      for (int i = k + 1 + lt; i < G; i += 128) S[i * G + k] /= d;
      __syncthreads();
      const int m = G - k - 1;
      for (int q = lt; q < m * m; q += 128) {
        const int i = k + 1 + q / m, j = k + 1 + q % m;
        if (j <= i) S[i * G + j] -= S[i * G + k] * S[j * G + k];
      }
      __syncthreads();
    }
    for (int q = lt; q < GG; q += 128) {
      const int i = q / G, j = q % G;
      if (j > i) S[i * G + j] = 0.0;
    }
  }
  __syncthreads();

  // ---- A = W'^T X' (stored column-major), V = I
  for (int e = tid; e < GG; e += kBuildThreads) {
    const int r = e % G, c = e / G;   // A[c*G + r] = (W'^T X')[r][c] = sum_k W'[k][r] X'[k][c]
    double a = 0.0;
    for (int k = 0; k < G; ++k) a = fma(Sw[k * G + r], Sx[k * G + c], a);
    A[c * G + r] = a;
    V[c * G + r] = (r == c) ? 1.0 : 0.0;
  }
  __syncthreads();

  // ---- one-sided Jacobi: rotate column pairs of A (and V) until mutually orthogonal.
  // Round-robin schedule: in round s, column G-1 meets column s, and (s+i) meets (s-i) mod (G-1).
  constexpr int SEG = G;                 // lanes per column pair (one lane per row)
  constexpr int PAIRS_PER_WARP = 32 / SEG;
  constexpr int NPAIRS = G / 2;
  const int seg = lane / SEG, row = lane % SEG;
  for (int sweep = 0; sweep < 40; ++sweep) {
    if (tid == 0) flag[1] = 0;
    __syncthreads();
    for (int s = 0; s < G - 1; ++s) {
      for (int pm = warp * PAIRS_PER_WARP + seg; pm < NPAIRS; pm += (kBuildThreads / 32) * PAIRS_PER_WARP) {
        int pc, qc;
        if (pm == 0) {
          pc = s;
          qc = G - 1;
        } else {
          pc = (s + pm) % (G - 1);
          qc = (s - pm + (G - 1)) % (G - 1);
        }
        const double ap = A[pc * G + row], aq = A[qc * G + row];
        const double alpha = warp_sum_seg(ap * ap, SEG);
        const double beta = warp_sum_seg(aq * aq, SEG);
        const double gamma = warp_sum_seg(ap * aq, SEG);
        if (fabs(gamma) > 1e-15 * sqrt(alpha * beta) && gamma != 0.0) {
          const double zeta = (beta - alpha) / (2.0 * gamma);
          const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          const double c = 1.0 / sqrt(1.0 + t * t), sn = c * t;
          A[pc * G + row] = c * ap - sn * aq;
          A[qc * G + row] = sn * ap + c * aq;
          const double vp = V[pc * G + row], vq = V[qc * G + row];
          V[pc * G + row] = c * vp - sn * vq;
          V[qc * G + row] = sn * vp + c * vq;
          if (row == 0) flag[1] = 1;
        }
      }
      __syncthreads();
    }
    if (flag[1] == 0) break;
    __syncthreads();
  }

  // ---- singular values, sorted descending (stable by index), U = A S^-1
  if (tid < G) {
    double n2 = 0.0;
    for (int r = 0; r < G; ++r) n2 = fma(A[tid * G + r], A[tid * G + r], n2);
    sig[tid] = sqrt(n2);
  }
  __syncthreads();
  if (tid < G) {
    const double me = sig[tid];
    int rank = 0;
    for (int j = 0; j < G; ++j) rank += (sig[j] > me) || (sig[j] == me && j < tid);
    sig2[rank] = me;
    const double inv = me > 0.0 ? 1.0 / me : 0.0;
    for (int r = 0; r < G; ++r) {
      U2[rank * G + r] = A[tid * G + r] * inv;
      V2[rank * G + r] = V[tid * G + r];
    }
  }
  __syncthreads();
  // sign convention
  if (tid < G) {
    int jm = 0;
    double best = -1.0;
    for (int r = 0; r < G; ++r) {
      const double a = fabs(U2[tid * G + r]);
      if (a > best) best = a, jm = r;
    }
    if (U2[tid * G + jm] < 0.0) {
      for (int r = 0; r < G; ++r) {
        U2[tid * G + r] = -U2[tid * G + r];
        V2[tid * G + r] = -V2[tid * G + r];
      }
    }
    if (p.s_out) p.s_out[static_cast<long long>(blk) * G + tid] = sig2[tid];
  }
  __syncthreads();

  // ---- B = S^-1/2 U^T W'^T and S^-1/2 V^T X'^T:  B[k][c] = sig_k^-1/2 sum_m U[m][k] W'[c][m]
  for (int e = tid; e < GG; e += kBuildThreads) {
    const int k = e / G, c = e % G;
    const double sc = 1.0 / sqrt(sig2[k]);
    double bw = 0.0, bx = 0.0;
    for (int m = 0; m <= c; ++m) {   // W', X' lower triangular: W'[c][m] = 0 for m > c
      bw = fma(U2[k * G + m], Sw[c * G + m], bw);
      bx = fma(V2[k * G + m], Sx[c * G + m], bx);
    }
    Bw[k * G + c] = bw * sc;
    Bx[k * G + c] = bx * sc;
  }
  __syncthreads();

  // ---- T = H B
  const double hs = 1.0 / sqrt(static_cast<double>(G));
  for (int e = tid; e < GG; e += kBuildThreads) {
    const int r = e / G, c = e % G;
    double tw, tx;
    if (p.use_hadamard) {
      tw = 0.0, tx = 0.0;
      for (int k = 0; k < G; ++k) {
        const double h = (__popc(r & k) & 1) ? -hs : hs;
        tw = fma(h, Bw[k * G + c], tw);
        tx = fma(h, Bx[k * G + c], tx);
      }
    } else {
      tw = Bw[r * G + c];
      tx = Bx[r * G + c];
    }
    const long long o = static_cast<long long>(blk) * GG + e;
    p.T_wush[o] = static_cast<float>(tw);
    p.T_xvsh[o] = static_cast<float>(tx);
    if (p.T_wush64) p.T_wush64[o] = tw;
    if (p.T_xvsh64) p.T_xvsh64[o] = tx;
  }
}


// `copies` back-to-back copies of the normalised Sylvester Hadamard matrix of order G
// (paper-graph-ui analysis, section 3.4.4: H is the orthonormal Hadamard that spreads
// S^-1/2 evenly over a block): entry (r, c) = (-1)^popcount(r & c) / sqrt(G), the
// recursion H_2n = [[H, H], [H, -H]] written out, formed in fp64 and rounded once to
// fp32.  Grid-stride over the copies * G * G outputs.
__global__ void wush_hadamard_kernel(int G, long long total, float* out) {
  const double hs = 1.0 / sqrt(static_cast<double>(G));
  const long long GG = static_cast<long long>(G) * G;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i % GG);
    const int r = e / G, c = e - (e / G) * G;
    out[i] = static_cast<float>((__popc(r & c) & 1) ? -hs : hs);
  }
}

}  // namespace wush
