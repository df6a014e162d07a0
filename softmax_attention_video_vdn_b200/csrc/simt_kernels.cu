// simt_kernels.cu - CUDA-core kernels of the VDN layer for fp32 inputs:
//  * the readout: o_lin = (S_fwd(b) + S_bwd(b)) q for tokens of non-anchor
//    frames, 0 for anchor frames (sd114.wiki, bidirectional linear branch:
//    the query reads both states and the results are summed), optionally
//    scaled by 1 - g_h into the linear half of Z;
//  * the softmax branch (with the same optional gate and readout as the bf16
//    path): one warp per query row, online softmax in fp32 over the key
//    frames of the row's mask (sd114.wiki, bidirectional sliding-window
//    softmax branch).
#include "kernels.h"

namespace vdn {

constexpr int kReadoutTokens = 64;

// grid (ceil(N/64), T, B*H), 256 threads. Shared: Ssum [dv][d+1], q [64][d].
// Token t of (b, h) goes to o + (b*L + t) * o_tok_stride + o_head_off + h*dv.
__global__ void __launch_bounds__(256)
    readout_kernel(const float* __restrict__ q, const float* __restrict__ S_fwd,
                   const float* __restrict__ S_bwd, float* __restrict__ o, int H, int Tf, int N,
                   int d, int dv, int bf, int anchors, int nb, long o_tok_stride, long o_head_off,
                   const float* __restrict__ gate) {
  extern __shared__ float shr[];
  const int ld = d + 1;
  float* Ss = shr;                 // [dv][ld]
  float* qs = shr + (size_t)dv * ld;  // [64][d]
  const int f = blockIdx.y, bh = blockIdx.z;
  const int n0 = blockIdx.x * kReadoutTokens;
  const int cnt = min(kReadoutTokens, N - n0);
  const int b = bh / H, h = bh - b * H;
  const long L = (long)Tf * N;
  const bool anchor = anchors && (f == 0 || f == Tf - 1);
  const int t = threadIdx.x;
  float* ob = o + ((size_t)b * L + (long)f * N + n0) * o_tok_stride + o_head_off + (size_t)h * dv;
  if (anchor) {
    for (int e = t; e < cnt * dv; e += blockDim.x) {
      const int tt = e / dv, j = e - tt * dv;
      ob[tt * o_tok_stride + j] = 0.f;
    }
    return;
  }
  const float cg = gate ? 1.f - 1.f / (1.f + expf(-gate[h])) : 1.f;
  const int blk = f / bf;
  const float* sf = S_fwd + ((size_t)bh * nb + blk) * dv * d;
  const float* sb = S_bwd + ((size_t)bh * nb + blk) * dv * d;
  for (int e = t; e < dv * d; e += blockDim.x) {
    const int j = e / d, k = e - j * d;
    Ss[j * ld + k] = sf[e] + sb[e];
  }
  const float* qb = q + ((size_t)bh * L + (long)f * N + n0) * d;
  for (int e = t; e < kReadoutTokens * d; e += blockDim.x) {
    const int tt = e / d;
    qs[e] = tt < cnt ? qb[e] : 0.f;
  }
  __syncthreads();
  const int groups = blockDim.x / dv;      // dv divides 256
  const int j = t % dv, g = t / dv;
  const int per = kReadoutTokens / groups;  // tokens per thread
  for (int u0 = 0; u0 < per; u0 += 16) {
    float acc[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] = 0.f;
    for (int k = 0; k < d; ++k) {
      const float s = Ss[j * ld + k];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int tt = g * per + u0 + u;
        if (u0 + u < per) acc[u] = fmaf(s, qs[tt * d + k], acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int tt = g * per + u0 + u;
      if (u0 + u < per && tt < cnt) ob[tt * o_tok_stride + j] = cg * acc[u];
    }
  }
}

cudaError_t launch_readout_f32(const void* q, const float* S_fwd, const float* S_bwd, void* o,
                               int B, int H, int Tf, int N, int d, int dv, int bf, int anchors,
                               int nb, long o_tok_stride, long o_head_off, const float* gate,
                               cudaStream_t stream) {
  dim3 grid((N + kReadoutTokens - 1) / kReadoutTokens, Tf, B * H);
  const size_t sm = ((size_t)dv * (d + 1) + (size_t)kReadoutTokens * d) * 4;
  cudaError_t e =
      cudaFuncSetAttribute(readout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  readout_kernel<<<grid, 256, sm, stream>>>(static_cast<const float*>(q), S_fwd, S_bwd,
                                            static_cast<float*>(o), H, Tf, N, d, dv, bf, anchors,
                                            nb, o_tok_stride, o_head_off, gate);
  return cudaGetLastError();
}

// fp32 softmax branch. One warp per query token; lane c holds elements
// c, c+32, c+64, c+96 of q and of the output row (d, dv <= 128).
__global__ void __launch_bounds__(256)
    softmax_window_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                              const float* __restrict__ v, const float* __restrict__ S_fwd,
                              const float* __restrict__ S_bwd, const float* __restrict__ gate,
                              float* __restrict__ out, int B, int H, int Tf, int N, int d, int dv,
                              int bf, int W, int anchors, int nb, float scale) {
  const int lane = threadIdx.x & 31;
  const long gw = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long L = (long)Tf * N;
  if (gw >= (long)B * H * L) return;
  const int bh = (int)(gw / L);
  const long tok = gw - (long)bh * L;
  const int b = bh / H, h = bh - b * H;
  const int fq = (int)(tok / N);
  const float* qr = q + ((size_t)bh * L + tok) * d;
  float qv[4], acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    qv[u] = c < d ? qr[c] * scale : 0.f;
    acc[u] = 0.f;
  }
  int k0[3], k1[3];
  const int nr = frame_row_ranges(Tf, bf, W, anchors, fq, k0, k1);
  float m = -INFINITY, l = 0.f;
  const float* kb = k + (size_t)bh * L * d;
  const float* vb = v + (size_t)bh * L * dv;
  for (int r = 0; r < nr; ++r) {
    for (long kt = (long)k0[r] * N; kt < (long)k1[r] * N; ++kt) {
      float s = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        if (c < d) s = fmaf(qv[u], kb[kt * d + c], s);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float mn = fmaxf(m, s);
      const float corr = expf(m - mn);
      const float p = expf(s - mn);
      l = l * corr + p;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        acc[u] = acc[u] * corr + (c < dv ? p * vb[kt * dv + c] : 0.f);
      }
      m = mn;
    }
  }
  const float inv_l = 1.f / l;
  if (gate == nullptr) {
    float* o = out + (((size_t)b * L + tok) * H + h) * dv;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dv) o[c] = acc[u] * inv_l;
    }
    return;
  }
  const float g = 1.f / (1.f + expf(-gate[h]));
  float* zs = out + (((size_t)b * L + tok) * 2 * H + h) * dv;
  if (S_fwd == nullptr) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane + 32 * u;
      if (c < dv) zs[c] = g * acc[u] * inv_l;
    }
    return;
  }
  float* zl = zs + (size_t)H * dv;
  const bool anchor = anchors && (fq == 0 || fq == Tf - 1);
  const int blk = fq / bf;
  const float* sf = S_fwd + ((size_t)bh * nb + blk) * dv * d;
  const float* sb = S_bwd + ((size_t)bh * nb + blk) * dv * d;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    if (c < dv) {
      zs[c] = g * acc[u] * inv_l;
      float ol = 0.f;
      if (!anchor)
        for (int kk = 0; kk < d; ++kk) ol = fmaf(sf[(size_t)c * d + kk] + sb[(size_t)c * d + kk], qr[kk], ol);
      zl[c] = (1.f - g) * ol;
    }
  }
}

}  // namespace vdn
