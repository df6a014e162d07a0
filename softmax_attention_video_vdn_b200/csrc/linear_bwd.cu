// linear_bwd.cu - backward of the VDA linear branch on sm_100a.
//
// Forward (besthub.dev, "Video Delta Attention (VDA)"; sd114.wiki,
// bidirectional linear branch), per (b, h):
//   G_f = K_f^T K_f, C_f = V_f^T K_f, M_f = (G_f + lambda I)^-1,
//   A_f = (1 - beta) I + beta lambda M_f, B_f = beta C_f M_f,
//   forward / backward scans X' = X A_f + B_f over the non-anchor frames,
//   o_t = (S_fwd(b) + S_bwd(b)) q_t for the non-anchor tokens of block b.
// Backward, given do (the cotangent of o):
//   dq_t = (S_fwd(b) + S_bwd(b))^T do_t                     readout kernel, transposed
//   dS(b) = sum_t do_t q_t^T = sum_f (do^T q)_f             frame stats on (q, do) +
//                                                            block_sum_kernel
//   adjoint scans: L' = L A_f (A_f symmetric, as M_f is), plus dS(b) where
//     the forward read block b's state; the cotangent after frame f is
//     recorded per frame and direction                    adjoint_scan_kernel
//   dA_f = sum_dir X_f^T L_f, dB_f = sum_dir L_f   (X_f: the state before f)
//   dM = beta lambda dA + beta C^T dB, dC = beta dB M, dG = -M dM M
//                                                          frame_grad_kernel
//   dK_f = K_f (dG + dG^T) + V_f dC, dV_f = K_f dC^T       stats_bwd_kernel
// Anchor frames and context tokens have no linear branch: their rows of dq,
// dk and dv are written as zeros.
#include "kernels.h"
#include "scan_blocks.cuh"

namespace vdn {

// --------------------------------------------------------------- block sums
// dS[bh][b] = sum of Cq[bh][f] over the non-anchor frames f of block b.
__global__ void block_sum_kernel(const float* __restrict__ Cq, float* __restrict__ dS, int T,
                                 int bf, int anchors, int nb, int mat) {
  const int bh = blockIdx.x / nb, b = blockIdx.x - (blockIdx.x / nb) * nb;
  const int f0 = b * bf, f1 = min(T, (b + 1) * bf);
  float* out = dS + (size_t)blockIdx.x * mat;
  for (int e = threadIdx.x; e < mat; e += blockDim.x) {
    float acc = 0.f;
    for (int f = f0; f < f1; ++f)
      if (!is_anchor(f, T, anchors)) acc += __ldg(Cq + ((size_t)bh * T + f) * mat + e);
    out[e] = acc;
  }
}

// ------------------------------------------------------------- adjoint scan
// One CTA per (b, h), direction and slab of kStateScanRows cotangent rows
// (the rows are independent, as in the forward scan). Visits the frames in
// the reverse of the direction's order with L = dL/d(state after the current
// frame): records L for the frame, applies L <- L A_f, then adds the
// cotangents of the block states that the forward scan read before the
// frame. A_f arrives by bulk copies, double-buffered. Each thread owns 8 rows
// x 4 columns of L A_f, summed in increasing k, as in the forward scan.
size_t adjoint_smem_bytes(int d) {
  return (size_t)2 * d * d * 4 + (size_t)kStateScanRows * d * 4;
}

__global__ void __launch_bounds__(kScanThreads)
    adjoint_scan_kernel(const float* __restrict__ Aall, const float* __restrict__ dS,
                        float* __restrict__ Lam_all, int T, int d, int dv, int bf, int W,
                        int anchors, int nb, int32_t* dev_status) {
  extern __shared__ __align__(128) uint8_t adj_smem[];
  __shared__ __align__(8) uint64_t bar_full[2];
  __shared__ int abort_sh;
  float* As = reinterpret_cast<float*>(adj_smem);  // [2][d*d]
  float* Lm = As + 2 * d * d;                        // [kStateScanRows][d]
  const int bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int row0 = blockIdx.z * kStateScanRows;
  const int rows = min(kStateScanRows, dv - row0);
  const int t = threadIdx.x;
  constexpr int kR = 8;                   // rows per thread
  const int col_threads = d / 4;
  const int c0 = (t % col_threads) * 4;
  const int r0 = (t / col_threads) * kR;
  const bool active = r0 < kStateScanRows;
  const int first = anchors ? 1 : 0;
  const int n_lin = anchors ? (T >= 2 ? T - 2 : 0) : T;
  // j-th non-anchor frame of the adjoint's visiting order (the reverse of
  // the direction's order)
  auto rev_frame = [&](int j) { return dir == 0 ? first + n_lin - 1 - j : first + j; };
  const uint32_t a_bytes = (uint32_t)d * d * 4;

  if (t == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  for (int e = t; e < kStateScanRows * d; e += kScanThreads) Lm[e] = 0.f;
  __syncthreads();
  const Abort ab{&abort_sh, dev_status};
  auto issue = [&](int j) {
    const int f = rev_frame(j);
    const int buf = j & 1;
    mbar_arrive_expect_tx(&bar_full[buf], a_bytes);
    bulk_load(As + buf * d * d, Aall + ((size_t)bh * T + f) * d * d, a_bytes, &bar_full[buf]);
  };
  if (t == 0) {
    for (int j = 0; j < 2 && j < n_lin; ++j) issue(j);
  }

  int lin = 0;
  bool ok = true;
  for (int step = T - 1; step >= 0; --step) {
    const int f = dir == 0 ? step : T - 1 - step;
    if (!is_anchor(f, T, anchors)) {
      float* dst = Lam_all + ((((size_t)bh * 2 + dir) * T + f) * dv + row0) * d;
      for (int e = t; e < rows * d; e += kScanThreads) dst[e] = Lm[e];
      const int buf = lin & 1;
      const bool got = mbar_wait(&bar_full[buf], (lin >> 1) & 1, ab);
      if (!__syncthreads_and(got)) { ok = false; break; }
      const float* A = As + buf * d * d;
      float acc[kR][4];
#pragma unroll
      for (int u = 0; u < kR; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      if (active) {
#pragma unroll 1
        for (int k = 0; k < d; k += 4) {
          float4 a[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            a[kk] = *reinterpret_cast<const float4*>(A + (k + kk) * d + c0);
#pragma unroll
          for (int u = 0; u < kR; ++u) {
            const float4 sv = *reinterpret_cast<const float4*>(Lm + (r0 + u) * d + k);
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
      __syncthreads();  // every read of Lm and of this buffer is done
      if (active) {
#pragma unroll
        for (int u = 0; u < kR; ++u)
          *reinterpret_cast<float4*>(Lm + (r0 + u) * d + c0) =
              make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
      }
      if (t == 0 && lin + 2 < n_lin) {
        fence_proxy_async_smem();
        issue(lin + 2);
      }
      ++lin;
      __syncthreads();
    }
    // cotangents of the block states stored before frame f
    int lo, hi;
    if (dir == 0)
      fwd_blocks(f, bf, W, nb, &lo, &hi);
    else
      bwd_blocks(f, T, bf, W, nb, &lo, &hi);
    if (lo <= hi) {
      for (int b = lo; b <= hi; ++b) {
        const float* src = dS + (((size_t)bh * nb + b) * dv + row0) * d;
        for (int e = t; e < rows * d; e += kScanThreads) Lm[e] += __ldg(src + e);
      }
      __syncthreads();
    }
  }
  if (!ok && t == 0) {
    for (int j = lin; j < lin + 2 && j < n_lin; ++j)
      mbar_wait_drain(&bar_full[j & 1], (j >> 1) & 1);
  }
}

// --------------------------------------------------------- per-frame grads
// One CTA of 256 threads per (b, h, f), d = dv = 128. Each thread owns an
// 8 x 8 tile (rows 8*(t/16), columns 8*(t%16)) of every 128 x 128 product,
// all of the form Z = X^T Y (both operands read by rows from shared memory,
// rows padded to kFgLd floats); a product's transpose is written by storing
// the register tile transposed.
constexpr int kFgThreads = 256;
constexpr int kFgLd = 132;
constexpr size_t kFgSmem = (size_t)3 * 128 * kFgLd * 4;

__device__ __forceinline__ void fg_load(float* dst, const float* __restrict__ src) {
  for (int e = threadIdx.x; e < 128 * 32; e += kFgThreads) {
    const int r = e >> 5, c = (e & 31) * 4;
    *reinterpret_cast<float4*>(dst + r * kFgLd + c) =
        __ldg(reinterpret_cast<const float4*>(src + r * 128 + c));
  }
}

// acc[u][v] += sum_r X[r][i0 + u] Y[r][j0 + v]
__device__ __forceinline__ void fg_tn(const float* X, const float* Y, int i0, int j0,
                                      float (&acc)[8][8]) {
#pragma unroll 2
  for (int r = 0; r < 128; ++r) {
    const float4 x0 = *reinterpret_cast<const float4*>(X + r * kFgLd + i0);
    const float4 x1 = *reinterpret_cast<const float4*>(X + r * kFgLd + i0 + 4);
    const float4 y0 = *reinterpret_cast<const float4*>(Y + r * kFgLd + j0);
    const float4 y1 = *reinterpret_cast<const float4*>(Y + r * kFgLd + j0 + 4);
    const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    const float ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(xs[u], ys[v], acc[u][v]);
  }
}

__device__ __forceinline__ void fg_zero(float (&a)[8][8]) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) a[u][v] = 0.f;
}

// tile -> dst rows i0.., columns j0.. (ld = row stride)
__device__ __forceinline__ void fg_store(float* dst, int ld, int i0, int j0,
                                         const float (&a)[8][8]) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    *reinterpret_cast<float4*>(dst + (size_t)(i0 + u) * ld + j0) =
        make_float4(a[u][0], a[u][1], a[u][2], a[u][3]);
    *reinterpret_cast<float4*>(dst + (size_t)(i0 + u) * ld + j0 + 4) =
        make_float4(a[u][4], a[u][5], a[u][6], a[u][7]);
  }
}
// transposed: dst[j0 + v][i0 + u] = a[u][v]
__device__ __forceinline__ void fg_store_t(float* dst, int ld, int i0, int j0,
                                           const float (&a)[8][8]) {
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    *reinterpret_cast<float4*>(dst + (size_t)(j0 + v) * ld + i0) =
        make_float4(a[0][v], a[1][v], a[2][v], a[3][v]);
    *reinterpret_cast<float4*>(dst + (size_t)(j0 + v) * ld + i0 + 4) =
        make_float4(a[4][v], a[5][v], a[6][v], a[7][v]);
  }
}

__global__ void __launch_bounds__(kFgThreads, 1)
    frame_grad_kernel(const float* __restrict__ S_all, const float* __restrict__ Lam_all,
                      const float* __restrict__ C, const float* __restrict__ M,
                      float* __restrict__ Gsym, float* __restrict__ dC, float* __restrict__ dCt,
                      int T, float lambda, float beta, int anchors) {
  extern __shared__ __align__(16) float fg_smem[];
  float* bA = fg_smem;
  float* bB = bA + 128 * kFgLd;
  float* bC = bB + 128 * kFgLd;
  const int frame = blockIdx.x;
  const int bh = frame / T, f = frame - (frame / T) * T;
  if (is_anchor(f, T, anchors)) return;  // zero rows are written by stats_bwd_kernel
  const int t = threadIdx.x;
  const int i0 = 8 * (t >> 4), j0 = 8 * (t & 15);
  const size_t mat = (size_t)128 * 128;
  const float* Xf = S_all + (((size_t)bh * 2 + 0) * T + f) * mat;
  const float* Xb = S_all + (((size_t)bh * 2 + 1) * T + f) * mat;
  const float* Lf = Lam_all + (((size_t)bh * 2 + 0) * T + f) * mat;
  const float* Lb = Lam_all + (((size_t)bh * 2 + 1) * T + f) * mat;

  // dA = X_fwd^T L_fwd + X_bwd^T L_bwd; dB = L_fwd + L_bwd (row-major in bB)
  float dA[8][8];
  fg_zero(dA);
  fg_load(bA, Xf);
  fg_load(bB, Lf);
  __syncthreads();
  fg_tn(bA, bB, i0, j0, dA);
  __syncthreads();
  fg_load(bA, Xb);
  fg_load(bC, Lb);
  __syncthreads();
  fg_tn(bA, bC, i0, j0, dA);
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) bB[(i0 + u) * kFgLd + j0 + v] += bC[(i0 + u) * kFgLd + j0 + v];
  __syncthreads();
  // dM = beta lambda dA + beta C^T dB
  fg_load(bA, C + (size_t)frame * mat);
  __syncthreads();
  {
    float dm[8][8];
    fg_zero(dm);
    fg_tn(bA, bB, i0, j0, dm);
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) dm[u][v] = beta * lambda * dA[u][v] + beta * dm[u][v];
    __syncthreads();           // reads of C (bA) and dB (bB) are done
    fg_store_t(bA, kFgLd, i0, j0, dm);   // bA = dM^T
  }
  {
    float db[8][8];            // this thread's tile of dB, stored transposed into bC
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) db[u][v] = bB[(i0 + u) * kFgLd + j0 + v];
    fg_store_t(bC, kFgLd, i0, j0, db);   // bC = dB^T
  }
  __syncthreads();
  fg_load(bB, M + (size_t)frame * mat);  // bB = M (symmetric)
  __syncthreads();
  {
    // dC = beta dB M = beta sum_k (dB^T)[k][r] M[k][j]
    float dc[8][8];
    fg_zero(dc);
    fg_tn(bC, bB, i0, j0, dc);
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) dc[u][v] *= beta;
    fg_store(dC + (size_t)frame * mat, 128, i0, j0, dc);
    fg_store_t(dCt + (size_t)frame * mat, 128, i0, j0, dc);
  }
  {
    // T1 = dM M = sum_k (dM^T)[k][i] M[k][j]
    float t1[8][8];
    fg_zero(t1);
    fg_tn(bA, bB, i0, j0, t1);
    __syncthreads();           // reads of dB^T (bC) and dM^T (bA) are done
    fg_store(bC, kFgLd, i0, j0, t1);
  }
  __syncthreads();
  {
    // dG = -M T1 = -sum_k M[k][i] T1[k][j]; G_sym = dG + dG^T
    float dg[8][8];
    fg_zero(dg);
    fg_tn(bB, bC, i0, j0, dg);
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) dg[u][v] = -dg[u][v];
    fg_store(bA, kFgLd, i0, j0, dg);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) dg[u][v] += bA[(j0 + v) * kFgLd + i0 + u];
    fg_store(Gsym + (size_t)frame * mat, 128, i0, j0, dg);
  }
}

// ------------------------------------------------------------ stats backward
// dK_f = K_f G_sym + V_f dC_f and dV_f = K_f dC_f^T, 128 tokens at a time.
// One CTA per (b, h, f) (plus one per (b, h) for the context rows).
// Accuracy: with fewer tokens than dimensions in a frame, G_f is singular and
// M_f reaches 1/lambda, so G_sym and dC carry large terms that cancel in dK;
// rounding them once to bf16 would cost several percent. Each fp32 operand X
// is therefore split into two bf16 matrices, hi = bf16(X) and
// lo = bf16(X - hi), and multiplied twice (K and V are bf16 already), which
// keeps about 16 bits of every product's operand.
// The epilogue warps first write the six 128 x 128 B operands (hi and lo of
// G_sym, dC^T and dC: [N][K] rows, K-major, 128-byte swizzle) into shared
// memory; the frame's K and V tiles then stream as 128-token x 64-dimension
// chunks (K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127) through a
// 2-slot TMA ring; one thread issues the products into a double-buffered
// TMEM accumulator (dK and dV, 256 columns per buffer). Warp roles (192
// threads): warp 0 TMA, warp 1 MMA, warps 2-5 operands and epilogue.
constexpr int kSbThreads = 192;
constexpr uint32_t kSbTile = 128 * 128 * 2;   // one 128 x 128 bf16 operand
constexpr uint32_t kSbChunk = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
static_assert(kStatsBwdSmem >= 1024 + 6 * kSbTile + 2 * kSbChunk, "stats backward smem");

__device__ __forceinline__ uint64_t sb_kdesc(const uint8_t* tile, int ks) {
  return sdesc_sw128(smem_u32(tile) + (ks >> 2) * kSbChunk + (ks & 3) * 32, 16, 1024);
}

// Row `row` of a fp32 128 x 128 matrix as the bf16 pair (hi, lo) into two
// K-major swizzled tiles.
__device__ __forceinline__ void sb_operand_row(uint8_t* hi, uint8_t* lo,
                                               const float* __restrict__ src, int row) {
  const float4* s4 = reinterpret_cast<const float4*>(src + (size_t)row * 128);
#pragma unroll 2
  for (int g = 0; g < 16; ++g) {
    const float4 a0 = __ldg(s4 + g * 2), a1 = __ldg(s4 + g * 2 + 1);
    const float x[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * u], x[2 * u + 1]);
      const float2 hf = __bfloat1622float2(hb);
      h[u] = *reinterpret_cast<const uint32_t*>(&hb);
      l[u] = pack_bf16(x[2 * u] - hf.x, x[2 * u + 1] - hf.y);
    }
    const int chunk = g >> 3, gg = g & 7;
    const uint32_t off = chunk * kSbChunk + row * 128 + ((gg ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

__device__ __forceinline__ void zero_rows(__nv_bfloat16* base, long t0, long t1, int tid,
                                          int nthreads) {
  for (long t = t0 + tid; t < t1; t += nthreads) {
    uint4* d4 = reinterpret_cast<uint4*>(base + (size_t)t * 128);
#pragma unroll
    for (int u = 0; u < 16; ++u) d4[u] = make_uint4(0, 0, 0, 0);
  }
}

// D (+)= A B over one 64-wide K chunk: A a 128 x 64 K-major chunk, B the
// K-range `kr` (0 or 1) of a 128 x 128 K-major operand. `first` clears D.
__device__ __forceinline__ void sb_mma_chunk(uint32_t d, const uint8_t* a, const uint8_t* b,
                                             int kr, uint32_t idesc, bool first) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    umma_ss(d, sdesc_sw128(smem_u32(a) + ks * 32, 16, 1024), sb_kdesc(b, 4 * kr + ks), idesc,
            (first && ks == 0) ? 0u : 1u);
}

__global__ void __launch_bounds__(kSbThreads, 1)
    stats_bwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ Gsym,
                     const float* __restrict__ dC, const float* __restrict__ dCt,
                     __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int BH,
                     int T, int N, int n_ctx, int anchors, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[2], bar_empty[2], bar_acc_full[2], bar_acc_empty[2],
      bar_ops, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const long TN = (long)T * N, L = TN + n_ctx;
  if ((int)blockIdx.x >= BH * T) {
    // context rows of one (b, h): no linear branch
    const int bh = blockIdx.x - BH * T;
    zero_rows(dk + (size_t)bh * L * 128, TN, L, threadIdx.x, kSbThreads);
    zero_rows(dv + (size_t)bh * L * 128, TN, L, threadIdx.x, kSbThreads);
    return;
  }
  const int frame = blockIdx.x;
  const int bh = frame / T, f = frame - (frame / T) * T;
  __nv_bfloat16* dk_bh = dk + (size_t)bh * L * 128;
  __nv_bfloat16* dv_bh = dv + (size_t)bh * L * 128;
  if (is_anchor(f, T, anchors)) {
    zero_rows(dk_bh, (long)f * N, (long)(f + 1) * N, threadIdx.x, kSbThreads);
    zero_rows(dv_bh, (long)f * N, (long)(f + 1) * N, threadIdx.x, kSbThreads);
    return;
  }
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // B operands: G_sym (B of K G_sym), dC^T (B of V dC), dC (B of K dC^T), each hi, lo
  uint8_t* sGh = base;
  uint8_t* sGl = base + kSbTile;
  uint8_t* sTh = base + 2 * kSbTile;
  uint8_t* sTl = base + 3 * kSbTile;
  uint8_t* sCh = base + 4 * kSbTile;
  uint8_t* sCl = base + 5 * kSbTile;
  uint8_t* sIn = base + 6 * kSbTile;   // ring slot s at sIn + s * kSbChunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long r0 = (long)f * N;
  const int ntiles = (N + 127) / 128;
  const int nchunks = 4 * ntiles;      // K 0-63, K 64-127, V 0-63, V 64-127 per tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], 4);
    }
    mbar_init(&bar_ops, 4);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, dev_status};

  if (warp == 0) {
    if (lane == 0) {
      int c = 0;
      for (; c < nchunks; ++c) {
        const int slot = c & 1, use = c >> 1, j = c & 3;
        if (use > 0 && !mbar_wait(&bar_empty[slot], (use - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&bar_full[slot], kSbChunk);
        const int row = (int)(r0 + (long)(c >> 2) * 128);
        tma_load_3d(sIn + slot * kSbChunk, j < 2 ? &tm_k : &tm_v, &bar_full[slot], (j & 1) * 64,
                    row, bh);
      }
      if (c < nchunks)
        for (int cc = (c > 2 ? c - 2 : 0); cc < c; ++cc)
          mbar_wait_drain(&bar_full[cc & 1], (cc >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      bool ok = mbar_wait(&bar_ops, 0, ab);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int a = i & 1;
        if (i >= 2 && !mbar_wait(&bar_acc_empty[a], ((i >> 1) - 1) & 1, ab)) break;
        const uint32_t d_k = tmem + a * 256, d_v = d_k + 128;
        for (int j = 0; j < 4; ++j) {
          const int c = 4 * i + j, slot = c & 1;
          if (!mbar_wait(&bar_full[slot], (c >> 1) & 1, ab)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* A = sIn + slot * kSbChunk;
          const int kr = j & 1;
          if (j < 2) {
            sb_mma_chunk(d_k, A, sGh, kr, idesc, j == 0);   // K G_sym
            sb_mma_chunk(d_k, A, sGl, kr, idesc, false);
            sb_mma_chunk(d_v, A, sCh, kr, idesc, j == 0);   // K dC^T
            sb_mma_chunk(d_v, A, sCl, kr, idesc, false);
          } else {
            sb_mma_chunk(d_k, A, sTh, kr, idesc, false);    // V dC
            sb_mma_chunk(d_k, A, sTl, kr, idesc, false);
          }
          umma_commit(&bar_empty[slot]);
        }
        if (!ok) break;
        umma_commit(&bar_acc_full[a]);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const size_t mo = (size_t)frame * 128 * 128;
    sb_operand_row(sGh, sGl, Gsym + mo, row);
    sb_operand_row(sTh, sTl, dCt + mo, row);
    sb_operand_row(sCh, sCl, dC + mo, row);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_ops);
    for (int i = 0; i < ntiles; ++i) {
      const int a = i & 1;
      if (!warp_wait(&bar_acc_full[a], (i >> 1) & 1, ab)) break;
      tc_fence_after();
      const long tr = (long)i * 128 + row;   // token within the frame
      const bool live = tr < N;
      const size_t o = (size_t)(r0 + tr) * 128;
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        __nv_bfloat16* dst = (m == 0 ? dk_bh : dv_bh) + o;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + a * 256 + m * 128 + c * 32, r);
          tmem_ld_wait();
          if (live) {
            uint4 pk[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
            for (int u = 0; u < 16; ++u)
              pw[u] = pack_bf16(__uint_as_float(r[2 * u]), __uint_as_float(r[2 * u + 1]));
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) d4[u] = pk[u];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ launch
cudaError_t launch_linear_bwd_kernels(const LinearBwdLaunch& p, cudaStream_t s) {
  const int BH = p.BH, T = p.T, d = 128, dv = 128, nb = p.nb;
  const int mat = d * dv;
  block_sum_kernel<<<BH * nb, 256, 0, s>>>(p.Cq, p.dS, T, p.bf, p.anchors, nb, mat);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t adj_sm = adjoint_smem_bytes(d);
  e = cudaFuncSetAttribute(adjoint_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)adj_sm);
  if (e != cudaSuccess) return e;
  adjoint_scan_kernel<<<dim3(BH, 2, (dv + kStateScanRows - 1) / kStateScanRows), kScanThreads,
                        adj_sm, s>>>(
      p.A, p.dS, p.Lam_all, T, d, dv, p.bf, p.W, p.anchors, nb, p.dev_status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(frame_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kFgSmem);
  if (e != cudaSuccess) return e;
  frame_grad_kernel<<<BH * T, kFgThreads, kFgSmem, s>>>(p.S_all, p.Lam_all, p.C, p.M, p.Gsym,
                                                        p.dC, p.dCt, T, p.lambda, p.beta,
                                                        p.anchors);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(stats_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kStatsBwdSmem);
  if (e != cudaSuccess) return e;
  stats_bwd_kernel<<<BH * T + (p.n_ctx > 0 ? BH : 0), kSbThreads, kStatsBwdSmem, s>>>(
      *p.tm_k, *p.tm_v, p.Gsym, p.dC, p.dCt, p.dk, p.dv, BH, T, p.N, p.n_ctx, p.anchors,
      p.dev_status);
  return cudaGetLastError();
}

}  // namespace vdn
