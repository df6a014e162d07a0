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
// frame_solve_mma_kernel (d = dv = 128) and frame_solve_kernel (other
//   sizes): one CTA per frame, fp64: (G_f + lambda I)^-1 by the symmetric
//   sweep (square-root-free Cholesky elimination carried to the inverse),
//   then B_f = beta C_f M; the first blocked eight pivots at a time, its
//   rank-8 updates and the product as fp64 tensor-path MMAs. A non-positive
//   pivot writes VDN_ERR_NUMERIC. A_f and B_f are stored in fp32.
// bidir_scan_kernel: the state rows are independent (row r of S A + B uses
//   only row r of S), so one CTA runs the whole frame sequence for 64 rows of
//   one (b, h) and one direction, with the state in fp32 shared memory, and
//   stores S_fwd / S_bwd of every block when its window boundary is reached.
//   A_f and B_f stream in by bulk copies, double-buffered.
#include "kernels.h"
#include "scan_blocks.cuh"

namespace vdn {

constexpr int kSolveThreads = 256;


// Shared vectors and matrix rows are padded by one element after every 8
// (index i -> i + i/8), so that threads reading 8 consecutive elements at
// 8-element offsets from each other hit different banks.
__device__ __forceinline__ int pad8(int i) { return i + (i >> 3); }

// Shared memory: M [d][pad8(d) + 8] fp64 (a row stride of 8 mod 16 doubles,
// so the four k rows of an MMA B fragment fall in two bank halves), CT
// [d][pad8(dv)] fp32 (C^T), two pivot-column buffers [2][pad8(d) + 1] fp64
// (the column, then 1 / pivot), one flag.
__host__ __device__ inline int solve_m_ld(int d) { return d + d / 8 + 8; }
size_t solve_smem_bytes(int d, int dv) {
  const size_t pd = d + d / 8, pv = dv + dv / 8;
  return (size_t)d * solve_m_ld(d) * 8 + (size_t)d * pv * 4 + 2 * (pd + 1) * 8 + 16;
}

// D += A B for one 8 x 8 fp64 tile on the tensor path (m8n8k4: A 8 x 4 row
// fragment, one element per thread at (lane / 4, lane % 4); B 4 x 8 column
// fragment at (lane % 4, lane / 4); D two elements at (lane / 4, 2 (lane % 4)
// + {0, 1})).
// (Not volatile: the compiler may interleave independent tiles' products.)
__device__ __forceinline__ void dmma_8x8x4(double (&dfr)[2], double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
      : "+d"(dfr[0]), "+d"(dfr[1])
      : "d"(a), "d"(b));
}

// 1 / p in fp64: the hardware's approximate reciprocal refined by two steps
// of Newton's method for f(x) = 1/x - p, x <- x (2 - p x); each step doubles
// the number of correct bits.
__device__ __forceinline__ double recip_newton(double p) {
  double x;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(x) : "d"(p));
  x = x * fma(-p, x, 2.0);
  x = x * fma(-p, x, 2.0);
  return x;
}

// M_f = (G_f + lambda I)^-1 by the symmetric sweep operator (Gauss-Jordan
// elimination in symmetric form, i.e. a square-root-free Cholesky / LDL^T
// elimination carried to the inverse): sweeping pivot k of a symmetric a
// with p = a_kk > 0 sets a_kk = -1/p, a_ik = a_ik/p, a_kj = a_kj/p and
// a_ij -= a_ik a_kj / p elsewhere; after sweeping every pivot in order a
// holds -(G_f + lambda I)^-1. The pivots are the squared diagonal entries of
// the Cholesky factor, so a pivot that is not > 0 means G_f + lambda I is not
// numerically SPD (VDN_ERR_NUMERIC). Each thread keeps an 8x8 tile of a in
// fp64 registers; pivot column k (= row k by symmetry) and 1 / pivot (computed
// once, by the thread that holds the pivot) are broadcast through a
// double-buffered shared vector, one barrier per pivot. Then
// A_f = (1 - beta) I + beta lambda M and B_f = beta C_f M (8x8 register tiles
// over M in shared memory), stored in fp32. This form serves the sizes other
// than d = dv = 128 (the fp32 path); frame_solve_mma_kernel below takes
// d = dv = 128.
__global__ void __launch_bounds__(kSolveThreads)
    frame_solve_kernel(const float* __restrict__ G, const float* __restrict__ C,
                       float* __restrict__ Aout, float* __restrict__ Bout,
                       float* __restrict__ Mout, int T, int d, int dv, float lambda, float beta,
                       int anchors, int32_t* dev_status) {
  extern __shared__ double shd[];
  const int ld = d + d / 8, ldc = dv + dv / 8, ldm = solve_m_ld(d);
  double* Msh = shd;                                            // [d][ldm]
  float* CT = reinterpret_cast<float*>(Msh + (size_t)d * ldm);  // [d][ldc]
  double* colbuf = reinterpret_cast<double*>(CT + (size_t)d * ldc);  // [2][ld + 1]
  int* bad = reinterpret_cast<int*>(colbuf + 2 * (ld + 1));
  const int frame = blockIdx.x;
  const int f = frame % T;
  if (is_anchor(f, T, anchors)) return;  // identity map, never applied
  const int t = threadIdx.x;
  const float* Gf = G + (size_t)frame * d * d;
  const float* Cf = C + (size_t)frame * dv * d;
  const int nt = d / 8;                  // tiles per dimension
  const bool has_tile = t < nt * nt;
  const int ti = has_tile ? t / nt : 0, tj = has_tile ? t % nt : 0;

  for (int e = t; e < dv * d; e += kSolveThreads) {
    const int i = e / dv, r = e - i * dv;   // consecutive threads: consecutive r
    CT[i * ldc + pad8(r)] = Cf[r * d + i];
  }
  if (t == 0) *bad = 0;
  double a[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = 8 * ti + r, j = 8 * tj + c;
      a[r][c] = has_tile ? (double)Gf[i * d + j] + (i == j ? (double)lambda : 0.0) : 0.0;
    }
  __syncthreads();

  // ---- symmetric sweep over every pivot
  bool pivot_bad = false;
#pragma unroll 1
  for (int kb = 0; kb < nt; ++kb) {
#pragma unroll
    for (int kr = 0; kr < 8; ++kr) {
      const int k = 8 * kb + kr;
      double* cb = colbuf + (k & 1) * (ld + 1);
      if (has_tile && tj == kb) {
#pragma unroll
        for (int r = 0; r < 8; ++r) cb[9 * ti + r] = a[r][kr];
        // the owner of the pivot publishes its reciprocal once for all
        if (ti == kb) cb[ld] = recip_newton(a[kr][kr]);
      }
      __syncthreads();
      const double p = cb[pad8(k)];
      if (!(p > 0.0)) pivot_bad = true;
      const double inv = cb[ld];
      if (has_tile) {
        double ci[8], cj[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          ci[u] = cb[9 * ti + u];
          cj[u] = cb[9 * tj + u];
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const double cs = -ci[r] * inv;
#pragma unroll
          for (int c = 0; c < 8; ++c) a[r][c] = fma(cs, cj[c], a[r][c]);
        }
        if (ti == kb) {
#pragma unroll
          for (int c = 0; c < 8; ++c) a[kr][c] = cj[c] * inv;
        }
        if (tj == kb) {
#pragma unroll
          for (int r = 0; r < 8; ++r) a[r][kr] = ci[r] * inv;
        }
        if (ti == kb && tj == kb) a[kr][kr] = -inv;
      }
    }
  }
  if (__syncthreads_or(pivot_bad)) {
    if (t == 0) report_status(dev_status, VDN_ERR_NUMERIC);
    return;
  }

  // ---- M = -a; A_f = (1 - beta) I + beta lambda M
  float* Af = Aout + (size_t)frame * d * d;
  const double bl = (double)beta * (double)lambda;
  if (has_tile) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = 8 * ti + r;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int j = 8 * tj + c;
        const double m = -a[r][c];
        Msh[i * ldm + pad8(j)] = m;
        Af[i * d + j] = (float)(bl * m + (i == j ? 1.0 - (double)beta : 0.0));
        if (Mout) Mout[(size_t)frame * d * d + i * d + j] = (float)m;
      }
    }
  }
  __syncthreads();

  // ---- B_f = beta C M, rows of C against columns of M
  const int rt = dv / 8;
  float* Bf = Bout + (size_t)frame * dv * d;
  for (int tt = t; tt < rt * nt; tt += kSolveThreads) {
    const int r0 = (tt / nt) * 8, j0 = (tt % nt) * 8;
    double bacc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) bacc[u][v] = 0.0;
    for (int i = 0; i < d; ++i) {
      double cv[8], mv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cv[u] = (double)CT[i * ldc + pad8(r0) + u];
        mv[u] = Msh[i * ldm + pad8(j0) + u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) bacc[u][v] = fma(cv[u], mv[v], bacc[u][v]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) Bf[(size_t)(r0 + u) * d + j0 + v] = (float)((double)beta * bacc[u][v]);
  }
}

// ------------------------------------------------- solve, d = dv = 128
// The same inverse by blocked sweeps with the matrix in FP64 tensor-path
// accumulator fragments. Warp w keeps rows 32 (w / 2) + [0, 32) and columns
// 64 (w % 2) + [0, 64) of the 128 x 128 matrix as 4 x 8 tiles of 8 x 8 (in
// the m8n8k4 D layout: lane l holds row l / 4, columns 2 (l % 4) + {0, 1} of
// each tile). The pivots are swept eight at a time, panel kb = pivots
// 8 kb + [0, 8) = the columns of tile column kb; sweeping a panel P in one
// step is the block form of its eight single sweeps: A_PP <- -A_PP^-1,
// A_iP <- A_iP A_PP^-1, A_Pj <- A_PP^-1 A_Pj, A_ij <- A_ij - A_iP A_PP^-1 A_Pj.
// Per panel: the four warps holding tile column kb store it (Y = A_.P) in
// shared memory; 128 threads, one panel row each, run the eight single
// sweeps on it (the pivot row and 1 / pivot through shared memory, a
// 128-thread barrier per pivot), which leaves X = [A_iP A_PP^-1; -A_PP^-1];
// then every tile outside the panel takes D <- D - X_i Y_j^T as two
// m8n8k4 MMAs (tiles of the pivot rows start from 0, since
// A_PP^-1 A_Pj = -X_PP Y_j^T) and the panel's tiles take X. Two CTA barriers
// per eight pivots. Afterwards M = -a goes to shared memory for A_f and
// B_f = beta C M, as in frame_solve_kernel.
constexpr int kPanelLd = 12;  // doubles per panel row: a fragment's 32 loads in two wavefronts

__global__ void __launch_bounds__(kSolveThreads)
    frame_solve_mma_kernel(const float* __restrict__ G, const float* __restrict__ C,
                           float* __restrict__ Aout, float* __restrict__ Bout,
                           float* __restrict__ Mout, int T, float lambda, float beta,
                           int anchors, int32_t* dev_status) {
  constexpr int d = 128, dv = 128;
  extern __shared__ double shd[];
  constexpr int ldcr = d + 4;  // C row stride: a fragment's 32 loads in 32 banks
  const int ldm = solve_m_ld(d);
  double* Msh = shd;                                              // [d][ldm]
  double* Xs = shd;                                               // [2][d][kPanelLd]
  double* Ys = shd + 2 * d * kPanelLd;                            // [2][d][kPanelLd]
  float* Cs = reinterpret_cast<float*>(Msh + (size_t)d * ldm);    // [dv][ldcr]
  double* prow = reinterpret_cast<double*>(Cs + (size_t)dv * ldcr);  // [8][9]
  // G_f staged past the panel buffers, in the M region (free until M is written)
  float* Gs = reinterpret_cast<float*>(shd + 4 * d * kPanelLd);    // [d][ldcr]
  __shared__ __align__(8) uint64_t bar_in;
  __shared__ int abort_sh;
  const int frame = blockIdx.x;
  const int f = frame % T;
  if (is_anchor(f, T, anchors)) return;  // identity map, never applied
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rb = (warp >> 1) * 32, cb = (warp & 1) * 64;  // this warp's block
  const float* Gf = G + (size_t)frame * d * d;
  const float* Cf = C + (size_t)frame * dv * d;

  // G_f and C_f row by row (512-byte bulk copies into rows padded to ldcr
  // floats), both on one barrier
  if (t == 0) {
    mbar_init(&bar_in, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const Abort ab{&abort_sh, dev_status};
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(&bar_in, 2u * d * d * 4);
    __syncwarp();
    for (int r = lane; r < d; r += 32) {
      bulk_load(Gs + r * ldcr, Gf + r * d, d * 4, &bar_in);
      bulk_load(Cs + r * ldcr, Cf + r * d, d * 4, &bar_in);
    }
  }
  if (!__syncthreads_and(mbar_wait(&bar_in, 0, ab))) {
    if (t == 0) mbar_wait_drain(&bar_in, 0);  // the copies land before the CTA exits
    __syncthreads();
    return;
  }
  double acc[4][8][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = rb + 8 * i + g, col = cb + 8 * j + 2 * q;
      const float2 gv = *reinterpret_cast<const float2*>(Gs + row * ldcr + col);
      acc[i][j][0] = (double)gv.x + (row == col ? (double)lambda : 0.0);
      acc[i][j][1] = (double)gv.y + (row == col + 1 ? (double)lambda : 0.0);
    }

  bool pivot_bad = false;
  // the eight single sweeps of panel kb on its stored column Yp into Xp, by
  // threads 0-127 (one panel row each; a 128-thread barrier per pivot)
  auto sweep_panel = [&](int kb, const double* Yp, double* Xp) {
    double pr[8];
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const double2 v = *reinterpret_cast<const double2*>(Yp + t * kPanelLd + c);
      pr[c] = v.x;
      pr[c + 1] = v.y;
    }
#pragma unroll
    for (int kr = 0; kr < 8; ++kr) {
      const int k = 8 * kb + kr;
      if (t == k) {  // the pivot row publishes itself and 1 / pivot
        const double p = pr[kr];
        if (!(p > 0.0)) pivot_bad = true;
#pragma unroll
        for (int c = 0; c < 8; ++c) prow[kr * 9 + c] = pr[c];
        prow[kr * 9 + 8] = recip_newton(p);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      double rowk[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) rowk[c] = prow[kr * 9 + c];
      const double inv = prow[kr * 9 + 8];
      if (t == k) {
#pragma unroll
        for (int c = 0; c < 8; ++c) pr[c] = c == kr ? -inv : rowk[c] * inv;
      } else {
        const double fr = pr[kr] * inv;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (c != kr) pr[c] = fma(-fr, rowk[c], pr[c]);
        pr[kr] = fr;
      }
    }
#pragma unroll
    for (int c = 0; c < 8; c += 2)
      *reinterpret_cast<double2*>(Xp + t * kPanelLd + c) = make_double2(pr[c], pr[c + 1]);
  };
  // panel 0: stored by the warps holding tile column 0, swept
  if ((warp & 1) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<double2*>(Ys + (rb + 8 * i + g) * kPanelLd + 2 * q) =
          make_double2(acc[i][0][0], acc[i][0][1]);
  }
  __syncthreads();
  if (t < 128) sweep_panel(0, Ys, Xs);
  __syncthreads();
  // panel kb = 8 hf + jj (its tile column is tile jj of the warps with
  // w % 2 = hf; jj and the next panel's tile jn are compile-time indices into
  // the fragments). With panel kb swept into X, Y: the warps holding the next
  // panel's tile column update it first and store it; threads 0-127 sweep the
  // next panel while every warp updates its other tiles with panel kb.
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const int kb = 8 * hf + jj;
    const int buf = jj & 1;
    const double* X = Xs + buf * d * kPanelLd;
    const double* Y = Ys + buf * d * kPanelLd;
    double* Xn = Xs + (buf ^ 1) * d * kPanelLd;
    double* Yn = Ys + (buf ^ 1) * d * kPanelLd;
    const int jn = (jj + 1) & 7;
    const bool owner = (warp & 1) == hf;
    const bool has_next = kb < 15;
    const bool owner_n = has_next && (warp & 1) == (jj == 7 ? hf + 1 : hf);
    double xa[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int s = 0; s < 2; ++s) xa[i][s] = -X[(rb + 8 * i + g) * kPanelLd + 4 * s + q];
    // k-step s of D - X_i Y_j^T for the four tiles of column j (pivot rows
    // from 0); both k-steps of a tile are dependent, so each pass covers
    // every tile before the next k-step
    auto update_step = [&](int j, int s) {
      const double yb = Y[(cb + 8 * j + g) * kPanelLd + 4 * s + q];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (s == 0 && (rb >> 3) + i == kb) acc[i][j][0] = acc[i][j][1] = 0.0;
        dmma_8x8x4(acc[i][j], xa[i][s], yb);
      }
    };
    // 1. the next panel's tile column: updated, then stored
    if (owner_n) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == jn) {
          update_step(j, 0);
          update_step(j, 1);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<double2*>(Yn + (rb + 8 * i + g) * kPanelLd + 2 * q) =
                make_double2(acc[i][j][0], acc[i][j][1]);
        }
    }
    __syncthreads();
    // 2. threads 0-127 sweep the next panel
    if (has_next && t < 128) sweep_panel(kb + 1, Yn, Xn);
    // 3. the other tiles: the panel's tiles take X, the rest D - X_i Y_j^T
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (!(owner && j == jj) && !(owner_n && j == jn)) update_step(j, s);
    if (owner) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double2 v = *reinterpret_cast<const double2*>(X + (rb + 8 * i + g) * kPanelLd + 2 * q);
        acc[i][jj][0] = v.x;
        acc[i][jj][1] = v.y;
      }
    }
    __syncthreads();
  }
  if (__syncthreads_or(pivot_bad)) {
    if (t == 0) report_status(dev_status, VDN_ERR_NUMERIC);
    return;
  }

  // ---- M = -a into shared memory, then A_f = (1 - beta) I + beta lambda M
  // (and M itself when asked) with coalesced stores
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = rb + 8 * i + g, col = cb + 8 * j + 2 * q;
      Msh[row * ldm + pad8(col)] = -acc[i][j][0];
      Msh[row * ldm + pad8(col + 1)] = -acc[i][j][1];
    }
  __syncthreads();
  float* Af = Aout + (size_t)frame * d * d;
  const double bl = (double)beta * (double)lambda;
  for (int e = t; e < d * d; e += kSolveThreads) {
    const int i = e >> 7, j = e & 127;
    const double m = Msh[i * ldm + pad8(j)];
    Af[e] = (float)(bl * m + (i == j ? 1.0 - (double)beta : 0.0));
    if (Mout) Mout[(size_t)frame * d * d + e] = (float)m;
  }

  // ---- B_f = beta C M on the FP64 tensor path (as in frame_solve_kernel)
  float* Bf = Bout + (size_t)frame * dv * d;
  double bacc[4][8][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) bacc[i][j][0] = bacc[i][j][1] = 0.0;
#pragma unroll 2
  for (int k0 = 0; k0 < 128; k0 += 4) {
    double af[4], bfr[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) af[i] = (double)Cs[(rb + 8 * i + g) * ldcr + k0 + q];
#pragma unroll
    for (int j = 0; j < 8; ++j) bfr[j] = Msh[(k0 + q) * ldm + pad8(cb + 8 * j + g)];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) dmma_8x8x4(bacc[i][j], af[i], bfr[j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float2*>(Bf + (size_t)(rb + 8 * i + g) * 128 + cb + 8 * j + 2 * q) =
          make_float2((float)((double)beta * bacc[i][j][0]), (float)((double)beta * bacc[i][j][1]));
}

size_t solve_mma_smem_bytes() {
  const size_t m = (size_t)128 * solve_m_ld(128) * 8, panels = (size_t)4 * 128 * kPanelLd * 8;
  return (m > panels ? m : panels) + (size_t)128 * 132 * 4 + 8 * 9 * 8;
}

cudaError_t launch_frame_solve(const float* G, const float* C, float* A, float* B, float* M,
                               unsigned frames, int T, int d, int dv, float lambda, float beta,
                               int anchors, int32_t* dev_status, cudaStream_t s) {
  cudaError_t e;
  if (d == 128 && dv == 128) {
    const size_t sm = solve_mma_smem_bytes();
    if ((e = cudaFuncSetAttribute(frame_solve_mma_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) !=
        cudaSuccess)
      return e;
    frame_solve_mma_kernel<<<frames, kSolveThreads, sm, s>>>(G, C, A, B, M, T, lambda, beta,
                                                             anchors, dev_status);
  } else {
    const size_t sm = solve_smem_bytes(d, dv);
    if ((e = cudaFuncSetAttribute(frame_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm)) != cudaSuccess)
      return e;
    frame_solve_kernel<<<frames, kSolveThreads, sm, s>>>(G, C, A, B, M, T, d, dv, lambda, beta,
                                                         anchors, dev_status);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- the scan
// Shared memory of the scan: A_f ring [2][d*d], B_f row slab ring
// [2][kStateScanRows*d], state [kStateScanRows][d].
size_t scan_smem_bytes(int d) {
  return (size_t)2 * d * d * 4 + (size_t)2 * kStateScanRows * d * 4 +
         (size_t)kStateScanRows * d * 4;
}

// One CTA runs all frames of one (b, h) and one direction for kStateScanRows
// rows of the state. Each step's A_f and the slab's rows of B_f arrive by 1-D
// bulk copies into a double-buffered ring; each thread owns 8 rows x 4
// columns of the new state: S_new[r][c] = B_f[r][c] + sum_k S[r][k] A_f[k][c],
// summed in increasing k. The step is bound by the number of shared-memory
// load instructions: per 4 k a thread loads 4 rows of A_f (16 bytes each)
// and 8 state rows (16-byte broadcasts) for 128 FMAs, four times the FMAs per
// load of 2 x 4 tiles.
__global__ void __launch_bounds__(kScanThreads)
    bidir_scan_kernel(const float* __restrict__ Aall, const float* __restrict__ Ball,
                      float* __restrict__ S_fwd, float* __restrict__ S_bwd,
                      float* __restrict__ S_all, int T, int d, int dv, int bf, int W, int anchors,
                      int nb, int32_t* dev_status) {
  extern __shared__ __align__(128) uint8_t scan_smem[];
  __shared__ __align__(8) uint64_t bar_full[2];
  __shared__ int abort_sh;
  float* As = reinterpret_cast<float*>(scan_smem);  // [2][d*d]
  float* Bs = As + 2 * d * d;                   // [2][kStateScanRows*d]
  float* S = Bs + 2 * kStateScanRows * d;       // [kStateScanRows][d]
  const int bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int row0 = blockIdx.z * kStateScanRows;
  const int rows = min(kStateScanRows, dv - row0);
  const int t = threadIdx.x;
  constexpr int kR = 8;                             // rows per thread
  const int col_threads = d / 4;                    // 4 columns per thread
  const int c0 = (t % col_threads) * 4;
  const int r0 = (t / col_threads) * kR;            // a warp shares its rows
  const bool active = r0 < kStateScanRows;
  float* Sout = dir == 0 ? S_fwd : S_bwd;
  // non-anchor frames in this direction's order
  const int first = anchors ? 1 : 0;
  const int n_lin = anchors ? (T >= 2 ? T - 2 : 0) : T;
  auto lin_frame = [&](int j) { return dir == 0 ? first + j : first + n_lin - 1 - j; };
  const uint32_t a_bytes = (uint32_t)d * d * 4, b_bytes = (uint32_t)rows * d * 4;

  if (t == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  for (int e = t; e < kStateScanRows * d; e += kScanThreads) S[e] = 0.f;
  __syncthreads();
  const Abort ab{&abort_sh, dev_status};
  auto issue = [&](int j) {  // load step j's maps into buffer j & 1
    const int f = lin_frame(j);
    const int buf = j & 1;
    mbar_arrive_expect_tx(&bar_full[buf], a_bytes + b_bytes);
    bulk_load(As + buf * d * d, Aall + ((size_t)bh * T + f) * d * d, a_bytes, &bar_full[buf]);
    bulk_load(Bs + buf * kStateScanRows * d, Ball + (((size_t)bh * T + f) * dv + row0) * d, b_bytes,
              &bar_full[buf]);
  };
  if (t == 0) {
    for (int j = 0; j < 2 && j < n_lin; ++j) issue(j);
  }

  int lin = 0;    // non-anchor frames consumed
  bool ok = true;
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
    if (S_all) {
      float* dst = S_all + ((((size_t)bh * 2 + dir) * T + f) * dv + row0) * d;
      for (int e = t; e < rows * d; e += kScanThreads) dst[e] = S[e];
    }
    if (is_anchor(f, T, anchors)) continue;
    const int buf = lin & 1;
    const bool got = mbar_wait(&bar_full[buf], (lin >> 1) & 1, ab);
    if (!__syncthreads_and(got)) { ok = false; break; }
    const float* A = As + buf * d * d;
    const float* Bv = Bs + buf * kStateScanRows * d;
    float acc[kR][4];
#pragma unroll
    for (int u = 0; u < kR; ++u) {
      const int r = r0 + u;
      const bool live = active && r < rows;
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = live ? Bv[r * d + c0 + v] : 0.f;
    }
    if (active) {
#pragma unroll 2
      for (int k = 0; k < d; k += 4) {
        float4 a[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) a[kk] = *reinterpret_cast<const float4*>(A + (k + kk) * d + c0);
#pragma unroll
        for (int u = 0; u < kR; ++u) {
          const float4 sv = *reinterpret_cast<const float4*>(S + (r0 + u) * d + k);
          const float s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            acc[u][0] = fmaf(s4[kk], a[kk].x, acc[u][0]);
            acc[u][1] = fmaf(s4[kk], a[kk].y, acc[u][1]);
            acc[u][2] = fmaf(s4[kk], a[kk].z, acc[u][2]);
            acc[u][3] = fmaf(s4[kk], a[kk].w, acc[u][3]);
          }
        }
      }
    }
    __syncthreads();  // every read of S and of this buffer is done
    if (active) {
#pragma unroll
      for (int u = 0; u < kR; ++u)
        *reinterpret_cast<float4*>(S + (r0 + u) * d + c0) =
            make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    if (t == 0 && lin + 2 < n_lin) {
      fence_proxy_async_smem();  // the buffer's generic reads precede the copy into it
      issue(lin + 2);
    }
    ++lin;
    __syncthreads();
  }
  if (!ok && t == 0) {
    // let issued copies land before shared memory is released
    for (int j = lin; j < lin + 2 && j < n_lin; ++j) mbar_wait_drain(&bar_full[j & 1], (j >> 1) & 1);
  }
}

}  // namespace vdn
