// frame_stats.cu - per-frame sums of the VDA update on sm_100a:
//   G_f = K_f^T K_f (d x d) and C_f = V_f^T K_f (dv x d).
// besthub.dev, "Video Delta Attention (VDA)": all spatial tokens of a frame
// jointly solve one state update; these two sums are all of the frame that
// the closed-form update needs.
//
// bf16: persistent, one CTA per SM; CTA c takes frames c, c + grid, ... and
// streams them back to back. TMA brings 64-token chunks of K_f and V_f (a
// 4-D tensor map whose token extent is N, so the tail of a frame's last
// chunk is zero-filled and never reaches into the next frame) through a
// 6-stage ring; one thread issues two tcgen05 MMAs per 16-token step, both
// with the K chunk as the MN-major B operand: A = K^T gives G, A = V^T gives
// C. Partials of 128 tokens alternate between two TMEM buffers, and eight
// drain warps add each partial into running totals held in their registers
// (see kStatsGroupChunks), then store a frame's G and C while the next
// frame's partials accumulate.
// f32: a SIMT kernel with fp64 accumulation (exact products of fp32 inputs).
#include "kernels.h"

namespace vdn {

// Accuracy: the tensor core's accumulation error grows with the length of
// the sum it accumulates. Each group of kStatsGroupChunks 64-token chunks is
// therefore accumulated into a fresh TMEM partial (256 columns: G then C),
// and the drain warps add the partials of a frame in order into fp32 totals
// with IEEE round-to-nearest adds.
constexpr int kStatsGroupChunks = 2;

// 32 lanes x 8 columns of 32-bit values (thread i: lane quarter*32 + i).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
constexpr int kStatsDrainWarps = 8;   // 2 per TMEM lane quarter: G columns, C columns
constexpr int kStatsThreads = 64 + 32 * kStatsDrainWarps;  // warp 0 TMA, warp 1 MMA, drain

__global__ void __launch_bounds__(kStatsThreads, 1)
    frame_stats_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, float* __restrict__ G,
                            float* __restrict__ C, int frames, int T, int N,
                            int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStatsStages], bar_empty[kStatsStages];
  __shared__ __align__(8) uint64_t bar_part_full[2], bar_part_empty[2], bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = (N + 63) / 64;
  const int ngroups = (nchunks + kStatsGroupChunks - 1) / kStatsGroupChunks;
  // frames of this CTA: blockIdx.x + i * gridDim.x for i < my_frames
  const int my_frames =
      frames > (int)blockIdx.x ? (frames - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStatsStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_part_full[i], 1);
      mbar_init(&bar_part_empty[i], kStatsDrainWarps);
    }
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
      int q = 0;  // chunks issued
      bool ok = true;
      for (int fi = 0; fi < my_frames && ok; ++fi) {
        const int frame = (int)blockIdx.x + fi * (int)gridDim.x;  // (b*H + h)*T + f
        const int bh = frame / T, f = frame - bh * T;
        for (int c = 0; c < nchunks; ++c) {
          const int st = q % kStatsStages, use = q / kStatsStages;
          if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, ab)) { ok = false; break; }
          uint8_t* s = base + st * kStatsStageBytes;
          mbar_arrive_expect_tx(&bar_full[st], kStatsStageBytes);
          tma_load_4d(s, &tm_k, &bar_full[st], 0, c * 64, f, bh);
          tma_load_4d(s + kStatsChunk, &tm_k, &bar_full[st], 64, c * 64, f, bh);
          tma_load_4d(s + 2 * kStatsChunk, &tm_v, &bar_full[st], 0, c * 64, f, bh);
          tma_load_4d(s + 3 * kStatsChunk, &tm_v, &bar_full[st], 64, c * 64, f, bh);
          ++q;
        }
      }
      if (!ok)  // aborted: let the issued copies land before exit
        for (int j = (q > kStatsStages ? q - kStatsStages : 0); j < q; ++j)
          mbar_wait_drain(&bar_full[j % kStatsStages], (j / kStatsStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 1, 1);
      int q = 0, gg = 0;  // chunks consumed, groups issued
      bool ok = true;
      for (int fi = 0; fi < my_frames && ok; ++fi) {
        for (int g = 0; g < ngroups; ++g, ++gg) {
          const int p = gg & 1;
          // the drain warps must have read partial buffer p two groups ago
          if (gg >= 2 && !mbar_wait(&bar_part_empty[p], ((gg >> 1) - 1) & 1, ab)) {
            ok = false;
            break;
          }
          const int c_end = min(nchunks, (g + 1) * kStatsGroupChunks);
          for (int c = g * kStatsGroupChunks; c < c_end; ++c, ++q) {
            const int st = q % kStatsStages;
            if (!mbar_wait(&bar_full[st], (q / kStatsStages) & 1, ab)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sk = smem_u32(base + st * kStatsStageBytes);
            const uint32_t sv = sk + 2 * kStatsChunk;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              // MN-major, 128B swizzle: 64-element dim chunks kStatsChunk
              // apart, 8-token groups 1024 B apart; 16 tokens per step.
              const uint64_t dk = sdesc_sw128(sk + ks * 2048, kStatsChunk, 1024);
              const uint64_t dv = sdesc_sw128(sv + ks * 2048, kStatsChunk, 1024);
              const uint32_t acc = (c > g * kStatsGroupChunks || ks > 0) ? 1u : 0u;
              umma_ss(tmem + p * 256, dk, dk, idesc, acc);        // partial G += K^T K
              umma_ss(tmem + p * 256 + 128, dv, dk, idesc, acc);  // partial C += V^T K
            }
            umma_commit(&bar_empty[st]);
          }
          if (!ok) break;
          umma_commit(&bar_part_full[p]);
        }
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    // drain warps: TMEM lane quarter (warp % 4) holds rows of G and C; warps
    // 2-5 own the G columns of a partial, warps 6-9 the C columns
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int half = warp >= 2 + kStatsDrainWarps / 2 ? 1 : 0;
    const uint32_t src0 = tmem + (uint32_t(wq * 32) << 16) + half * 128;
    float* const out = half ? C : G;
    float tot[128];
    int gg = 0;
    bool ok = true;
    for (int fi = 0; fi < my_frames && ok; ++fi) {
#pragma unroll
      for (int i = 0; i < 128; ++i) tot[i] = 0.0f;
      for (int g = 0; g < ngroups; ++g, ++gg) {
        const int p = gg & 1;
        if (!warp_wait(&bar_part_full[p], (gg >> 1) & 1, ab)) { ok = false; break; }
        tc_fence_after();
        // 8 columns per load: the totals take 128 registers of the 168 a
        // thread has with ten warps per SM
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          uint32_t r[8];
          tmem_ld8(src0 + p * 256 + c * 8, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) tot[c * 8 + i] += __uint_as_float(r[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_part_empty[p]);
      }
      if (!ok) break;
      const int frame = (int)blockIdx.x + fi * (int)gridDim.x;
      float4* d4 = reinterpret_cast<float4*>(out + ((size_t)frame * 128 + row) * 128);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        d4[i] = make_float4(tot[4 * i], tot[4 * i + 1], tot[4 * i + 2], tot[4 * i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_frame_stats_bf16(const CUtensorMap& tm_k, const CUtensorMap& tm_v, float* G,
                                    float* C, int frames, int T, int N, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(frame_stats_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kStatsSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  frame_stats_bf16_kernel<<<min(frames, sms), kStatsThreads, kStatsSmem, stream>>>(
      tm_k, tm_v, G, C, frames, T, N, nullptr);
  return cudaGetLastError();
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
