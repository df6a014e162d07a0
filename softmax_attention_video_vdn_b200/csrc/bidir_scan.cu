// bidir_scan.cu - per-frame solve and bidirectional scan of the VDA states.
//
// besthub.dev, "Video Delta Attention (VDA)": all tokens of a frame jointly
// solve one state update, and the update is non-expansive. The closed form
// used here: M_f = (G_f + lambda I)^-1, S <- S A_f + B_f with
//   A_f = I - beta G_f M_f = (1 - beta) I + beta lambda M_f   (G M = I - lambda M)
//   B_f = beta C_f M_f.
// sd114.wiki, bidirectional linear branch: the forward state of a block
// summarises the frames before its window, the backward state the frames
// after it; anchor frames take no part.
//
// frame_solve_kernel: one CTA per frame, all in fp64 shared memory: Cholesky
//   factor L of G_f + lambda I (right-looking, one column per step), L^-1 in
//   place, M = L^-T L^-1 and B_f = beta C_f M by 8x8 register tiles. A
//   non-positive pivot writes VDN_ERR_NUMERIC. A_f and B_f are stored in fp32.
// bidir_scan_kernel: the state rows are independent (row r of S A + B uses
//   only row r of S), so one CTA runs the whole frame sequence for 16 rows of
//   one (b, h) and one direction, with the state in fp32 shared memory, and
//   stores S_fwd / S_bwd of every block when its window boundary is reached.
#include "kernels.h"

namespace vdn {

constexpr int kSolveThreads = 256;

__device__ __forceinline__ bool is_anchor(int f, int T, int anchors) {
  return anchors && (f == 0 || f == T - 1);
}

// Shared memory: R [d][d+1] fp64 (padded rows), CT [d][dv] fp32 (C^T),
// col [d] fp64, one flag.
size_t solve_smem_bytes(int d, int dv) {
  return (size_t)d * (d + 1) * 8 + (size_t)d * dv * 4 + (size_t)d * 8 + 16;
}

__global__ void __launch_bounds__(kSolveThreads)
    frame_solve_kernel(const float* __restrict__ G, const float* __restrict__ C,
                       float* __restrict__ Aout, float* __restrict__ Bout, int T, int d, int dv,
                       float lambda, float beta, int anchors, int32_t* dev_status) {
  extern __shared__ double shd[];
  const int ld = d + 1;
  double* R = shd;                                          // [d][ld]
  float* CT = reinterpret_cast<float*>(R + (size_t)d * ld);  // [d][dv]
  double* col = reinterpret_cast<double*>(CT + (size_t)d * dv);
  int* bad = reinterpret_cast<int*>(col + d);
  const int frame = blockIdx.x;
  const int f = frame % T;
  if (is_anchor(f, T, anchors)) return;  // identity map, never applied
  const int t = threadIdx.x;
  const float* Gf = G + (size_t)frame * d * d;
  const float* Cf = C + (size_t)frame * dv * d;

  for (int e = t; e < d * d; e += kSolveThreads) {
    const int i = e / d, j = e - i * d;
    R[i * ld + j] = (double)Gf[e] + (i == j ? (double)lambda : 0.0);
  }
  for (int e = t; e < dv * d; e += kSolveThreads) {
    const int r = e / d, i = e - r * d;
    CT[i * dv + r] = Cf[e];
  }
  if (t == 0) *bad = 0;
  __syncthreads();

  // ---- Cholesky R = L L^T (lower triangle of R becomes L)
  const int warp = t >> 5, lane = t & 31;
  for (int k = 0; k < d; ++k) {
    if (t == 0) {
      const double p = R[k * ld + k];
      if (!(p > 0.0)) {
        *bad = 1;
      } else {
        R[k * ld + k] = sqrt(p);
      }
    }
    __syncthreads();
    if (*bad) {
      if (t == 0) report_status(dev_status, VDN_ERR_NUMERIC);
      return;
    }
    const double lkk = R[k * ld + k];
    for (int i = k + 1 + t; i < d; i += kSolveThreads) {
      const double v = R[i * ld + k] / lkk;
      R[i * ld + k] = v;
      col[i] = v;
    }
    __syncthreads();
    for (int i = k + 1 + warp; i < d; i += kSolveThreads / 32) {
      const double li = col[i];
      for (int j = k + 1 + lane; j <= i; j += 32) R[i * ld + j] -= li * col[j];
    }
    __syncthreads();
  }

  // ---- L^-1 in place, columns right to left:
  // X[j][j] = 1/L[j][j]; X[i][j] = -(sum_{k=j+1..i} X[i][k] L[k][j]) / L[j][j]
  for (int j = d - 1; j >= 0; --j) {
    double v = 0.0;
    const int i = j + t;
    const double ljj = R[j * ld + j];
    if (i < d) {
      if (i == j) {
        v = 1.0 / ljj;
      } else {
        double s = 0.0;
        for (int k = j + 1; k <= i; ++k) s += R[i * ld + k] * R[k * ld + j];
        v = -s / ljj;
      }
    }
    __syncthreads();
    if (i < d) R[i * ld + j] = v;
    __syncthreads();
  }
  // clear the upper triangle so the products below may run over all k
  for (int e = t; e < d * d; e += kSolveThreads) {
    const int i = e / d, j = e - i * d;
    if (j > i) R[i * ld + j] = 0.0;
  }
  __syncthreads();

  // ---- M = X^T X by 8x8 tiles (X = L^-1, lower triangular)
  const int tiles = d / 8;
  const bool has_tile = t < tiles * tiles;
  const int ti = has_tile ? (t / tiles) * 8 : 0, tj = has_tile ? (t % tiles) * 8 : 0;
  double acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0;
  if (has_tile) {
    for (int k = 0; k < d; ++k) {
      double xa[8], xb[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        xa[a] = R[k * ld + ti + a];
        xb[a] = R[k * ld + tj + a];
      }
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fma(xa[a], xb[b], acc[a][b]);
    }
  }
  __syncthreads();
  if (has_tile) {
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) R[(ti + a) * ld + tj + b] = acc[a][b];
  }
  __syncthreads();

  // ---- A_f = (1 - beta) I + beta lambda M
  float* Af = Aout + (size_t)frame * d * d;
  const double bl = (double)beta * (double)lambda;
  for (int e = t; e < d * d; e += kSolveThreads) {
    const int i = e / d, j = e - i * d;
    Af[e] = (float)(bl * R[i * ld + j] + (i == j ? 1.0 - (double)beta : 0.0));
  }

  // ---- B_f = beta C M, rows of C against columns of M
  const int rt = dv / 8;
  float* Bf = Bout + (size_t)frame * dv * d;
  for (int tt = t; tt < rt * tiles; tt += kSolveThreads) {
    const int r0 = (tt / tiles) * 8, j0 = (tt % tiles) * 8;
    double bacc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) bacc[a][b] = 0.0;
    for (int i = 0; i < d; ++i) {
      double cv[8], mv[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        cv[a] = (double)CT[i * dv + r0 + a];
        mv[a] = R[i * ld + j0 + a];
      }
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) bacc[a][b] = fma(cv[a], mv[b], bacc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) Bf[(size_t)(r0 + a) * d + j0 + b] = (float)((double)beta * bacc[a][b]);
  }
}

// ---------------------------------------------------------------- the scan
constexpr int kScanRows = 16;
constexpr int kScanThreads = 256;

// Blocks whose forward state is the state before frame f (window start == f).
__device__ __forceinline__ void fwd_blocks(int f, int bf, int W, int nb, int* lo, int* hi) {
  if (f == 0) {
    *lo = 0;
    *hi = min(W, nb - 1);
  } else if (f % bf == 0 && f / bf + W < nb) {
    *lo = *hi = f / bf + W;
  } else {
    *lo = 1;
    *hi = 0;
  }
}
// Blocks whose backward state is the state before frame f in decreasing order
// (window end == f + 1).
__device__ __forceinline__ void bwd_blocks(int f, int T, int bf, int W, int nb, int* lo, int* hi) {
  const int e = f + 1;
  if (e == T) {
    // every block whose window reaches the end: (b + W + 1) * bf >= T
    int first = (T + bf - 1) / bf - W - 1;
    *lo = max(first, 0);
    *hi = nb - 1;
  } else if (e % bf == 0 && e / bf - W - 1 >= 0) {
    *lo = *hi = e / bf - W - 1;
  } else {
    *lo = 1;
    *hi = 0;
  }
}

__global__ void __launch_bounds__(kScanThreads)
    bidir_scan_kernel(const float* __restrict__ Aall, const float* __restrict__ Ball,
                      float* __restrict__ S_fwd, float* __restrict__ S_bwd, int T, int d, int dv,
                      int bf, int W, int anchors, int nb) {
  __shared__ float S[kScanRows * 128];  // rows of this slab, [r][k]
  const int bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int row0 = blockIdx.z * kScanRows;
  const int rows = min(kScanRows, dv - row0);
  const int t = threadIdx.x;
  const int groups = kScanThreads / d;      // thread groups over the columns
  const int j = t % d, g = t / d;
  const int rpt = (kScanRows + groups - 1) / groups;  // rows per thread (<= 8 for d = 128)
  float* Sout = dir == 0 ? S_fwd : S_bwd;
  for (int e = t; e < kScanRows * d; e += kScanThreads) S[e] = 0.f;
  __syncthreads();

  for (int step = 0; step < T; ++step) {
    const int f = dir == 0 ? step : T - 1 - step;
    int lo, hi;
    if (dir == 0)
      fwd_blocks(f, bf, W, nb, &lo, &hi);
    else
      bwd_blocks(f, T, bf, W, nb, &lo, &hi);
    for (int b = lo; b <= hi; ++b) {
      float* dst = Sout + (((size_t)bh * nb + b) * dv + row0) * d;
      for (int e = t; e < rows * d; e += kScanThreads) dst[e] = S[e];
    }
    if (is_anchor(f, T, anchors)) continue;
    const float* Af = Aall + ((size_t)bh * T + f) * d * d;
    const float* Bf = Ball + ((size_t)bh * T + f) * dv * d;
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = g * rpt + u;
      acc[u] = (u < rpt && r < rows) ? __ldg(Bf + (size_t)(row0 + r) * d + j) : 0.f;
    }
    if (g < groups) {
#pragma unroll 4
      for (int k = 0; k < d; ++k) {
        const float a = __ldg(Af + (size_t)k * d + j);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (u < rpt) acc[u] = fmaf(S[(g * rpt + u) * d + k], a, acc[u]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = g * rpt + u;
      if (g < groups && u < rpt && r < kScanRows) S[r * d + j] = acc[u];
    }
    __syncthreads();
  }
  // blocks whose range reaches past the last frame take the final state
  // (covered above: every block is written exactly once at its boundary)
}

}  // namespace vdn
