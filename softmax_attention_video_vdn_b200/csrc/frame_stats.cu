// frame_stats.cu - per-frame sums of the VDA update on sm_100a:
//   G_f = K_f^T K_f (d x d) and C_f = V_f^T K_f (dv x d).
// besthub.dev, "Video Delta Attention (VDA)": all spatial tokens of a frame
// jointly solve one state update; these two sums are all of the frame that
// the closed-form update needs.
//
// bf16: one CTA per (b, h, f). TMA streams 64-token chunks of K_f and V_f
// (a 4-D tensor map whose token extent is N, so the tail of the last chunk is
// zero-filled and never reaches into the next frame) through a 3-stage ring;
// one thread issues two tcgen05 MMAs per 16-token step, both with the K chunk
// as the MN-major B operand: A = K^T gives G, A = V^T gives C. Accumulators
// live in TMEM (2 x 128 columns) and four warps drain them.
// f32: a SIMT kernel with fp64 accumulation (exact products of fp32 inputs).
#include "kernels.h"

namespace vdn {


__global__ void __launch_bounds__(128)
    frame_stats_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, float* __restrict__ G,
                            float* __restrict__ C, int T, int N, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStatsStages], bar_empty[kStatsStages], bar_done, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int frame = blockIdx.x;  // (b*H + h)*T + f
  const int bh = frame / T, f = frame - bh * T;
  const int nchunks = (N + 63) / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStatsStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_done, 1);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, dev_status};

  if (warp == 0) {
    if (lane == 0) {
      int c = 0;
      for (; c < nchunks; ++c) {
        const int st = c % kStatsStages;
        const int use = c / kStatsStages;
        if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, ab)) break;
        uint8_t* s = base + st * kStatsStageBytes;
        mbar_arrive_expect_tx(&bar_full[st], kStatsStageBytes);
        tma_load_4d(s, &tm_k, &bar_full[st], 0, c * 64, f, bh);
        tma_load_4d(s + kStatsChunk, &tm_k, &bar_full[st], 64, c * 64, f, bh);
        tma_load_4d(s + 2 * kStatsChunk, &tm_v, &bar_full[st], 0, c * 64, f, bh);
        tma_load_4d(s + 3 * kStatsChunk, &tm_v, &bar_full[st], 64, c * 64, f, bh);
      }
      if (c < nchunks)  // aborted: let the issued copies land before exit
        for (int cc = (c > kStatsStages ? c - kStatsStages : 0); cc < c; ++cc)
          mbar_wait_drain(&bar_full[cc % kStatsStages], (cc / kStatsStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 1, 1);
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % kStatsStages;
        if (!mbar_wait(&bar_full[st], (c / kStatsStages) & 1, ab)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(base + st * kStatsStageBytes);
        const uint32_t sv = sk + 2 * kStatsChunk;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          // MN-major, 128B swizzle: 64-element dim chunks kStatsChunk apart,
          // 8-token groups 1024 B apart; 16 tokens per step.
          const uint64_t dk = sdesc_sw128(sk + ks * 2048, kStatsChunk, 1024);
          const uint64_t dv = sdesc_sw128(sv + ks * 2048, kStatsChunk, 1024);
          const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
          umma_ss(tmem + 0, dk, dk, idesc, acc);    // G += K^T K
          umma_ss(tmem + 128, dv, dk, idesc, acc);  // C += V^T K
        }
        umma_commit(&bar_empty[st]);
      }
      if (ok) umma_commit(&bar_done);
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  }

  // all four warps: TMEM lanes 32w..32w+31 hold rows of G and C
  if (warp_wait(&bar_done, 0, ab)) {
    tc_fence_after();
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
    float* g_row = G + ((size_t)frame * 128 + row) * 128;
    float* c_row = C + ((size_t)frame * 128 + row) * 128;
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      float* dst = part ? c_row : g_row;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + part * 128 + c * 32, r);
        tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                              __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// fp32 inputs: G and C with fp64 accumulation. One CTA per frame; 32-token
// chunks of K_f and V_f staged in shared memory; each thread owns a set of
// (i, j) entries of G and C.
__global__ void __launch_bounds__(256)
    frame_stats_f32_kernel(const float* __restrict__ k, const float* __restrict__ v,
                           float* __restrict__ G, float* __restrict__ C, int T, int N, int d,
                           int dv) {
  extern __shared__ float sh[];
  float* sk = sh;            // [32][d]
  float* sv = sh + 32 * d;   // [32][dv]
  const int frame = blockIdx.x;
  const size_t tok0 = (size_t)frame * N;  // (b*H+h)*L + f*N
  const int nG = d * d, nC = dv * d;
  const int per = (nG + nC + blockDim.x - 1) / blockDim.x;  // <= 128 for d = dv = 128
  double acc[128];
#pragma unroll
  for (int e = 0; e < 128; ++e) acc[e] = 0.0;
  for (int n0 = 0; n0 < N; n0 += 32) {
    const int cnt = min(32, N - n0);
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * d; e += blockDim.x) {
      const int t = e / d, c = e - t * d;
      sk[e] = t < cnt ? k[(tok0 + n0 + t) * d + c] : 0.f;
    }
    for (int e = threadIdx.x; e < 32 * dv; e += blockDim.x) {
      const int t = e / dv, c = e - t * dv;
      sv[e] = t < cnt ? v[(tok0 + n0 + t) * dv + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int u = 0; u < per && u < 128; ++u) {
      const int e = threadIdx.x + u * blockDim.x;
      if (e >= nG + nC) break;
      double a = acc[u];
      if (e < nG) {
        const int i = e / d, j = e - i * d;
        for (int t = 0; t < cnt; ++t) a += (double)sk[t * d + i] * (double)sk[t * d + j];
      } else {
        const int e2 = e - nG;
        const int i = e2 / d, j = e2 - i * d;
        for (int t = 0; t < cnt; ++t) a += (double)sv[t * dv + i] * (double)sk[t * d + j];
      }
      acc[u] = a;
    }
  }
#pragma unroll 1
  for (int u = 0; u < per && u < 128; ++u) {
    const int e = threadIdx.x + u * blockDim.x;
    if (e >= nG + nC) break;
    if (e < nG)
      G[(size_t)frame * nG + e] = (float)acc[u];
    else
      C[(size_t)frame * nC + (e - nG)] = (float)acc[u];
  }
}

}  // namespace vdn
