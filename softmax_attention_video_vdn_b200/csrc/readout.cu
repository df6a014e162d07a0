// readout.cu - linear-branch readout on sm_100a (bf16 inputs):
//   o_lin[t] = c_h (S_fwd(b) + S_bwd(b)) q_t   for tokens t of non-anchor
//   frames of block b, and 0 for anchor frames; c_h = 1, or 1 - sigmoid(gate
//   logit of head h) when the result is the linear half of the gated Z.
//   With transpose_s the kernel multiplies by (S_fwd(b) + S_bwd(b))^T: the
//   backward's dq_t = S^T do_t, with do in place of q.
// sd114.wiki, bidirectional linear branch: the query reads both states and
// the results are summed.
//
// One CTA per (b, h, block). The epilogue warps first write S_fwd + S_bwd as
// bf16 into shared memory in the 128-byte-swizzled K-major layout (the B
// operand, N = dv rows, K = d), then the CTA streams the block's 128-row Q
// tiles through a 2-stage TMA ring; one thread issues M=128, N=128, K=16
// tcgen05 MMAs into a double-buffered TMEM accumulator (2 x 128 columns);
// four warps convert the rows to bf16 and store them. Warp roles (192
// threads): warp 0 TMA, warp 1 MMA, warps 2-5 operand + epilogue.
#include "kernels.h"

namespace vdn {

constexpr int kRoThreads = 192;
constexpr uint32_t kRoTile = 128 * 128 * 2;   // 128 x 128 bf16
constexpr uint32_t kRoChunk = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
constexpr size_t kRoSmem = 1024 + 3 * kRoTile;  // Ssum + 2 Q stages

__device__ __forceinline__ uint64_t ro_kdesc(const uint8_t* tile, int ks) {
  return sdesc_sw128(smem_u32(tile) + (ks >> 2) * kRoChunk + (ks & 3) * 32, 16, 1024);
}

__global__ void __launch_bounds__(kRoThreads, 1)
    readout_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const float* __restrict__ S_fwd,
                        const float* __restrict__ S_bwd, __nv_bfloat16* __restrict__ o, int H,
                        int T, int N, int bf, int anchors, int nb, int n_ctx,
                        const ReadoutOut out, int transpose_s,
                        const float* __restrict__ gate_logits, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q_full[2], bar_q_empty[2], bar_acc_full[2],
      bar_acc_empty[2], bar_sum_full, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sSum = base;
  uint8_t* sQ = base + kRoTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbx = nb + (n_ctx > 0 ? 1 : 0);   // blocks per (b, h), plus the context rows
  const int bh = blockIdx.x / nbx, blk = blockIdx.x - (blockIdx.x / nbx) * nbx;
  const int b = bh / H, h = bh - b * H;
  const long TN = (long)T * N;                 // video tokens of a head
  const long L = TN + n_ctx;                   // tokens of a head
  // row of token t of this (b, h) in the output
  __nv_bfloat16* const obh = o + (size_t)b * out.b_stride + (size_t)h * out.h_stride + out.off;
  if (blk == nb) {
    // context tokens have no linear branch: zero rows
    for (long t = TN + threadIdx.x; t < L; t += kRoThreads) {
      uint4* d4 = reinterpret_cast<uint4*>(obh + (size_t)t * out.tok_stride);
#pragma unroll
      for (int u = 0; u < 16; ++u) d4[u] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  // frames of the block; the anchor frames (0 and T-1) are at its ends
  int f0 = blk * bf, f1 = min(T, (blk + 1) * bf);
  const bool first_anchor = anchors && f0 == 0;
  const bool last_anchor = anchors && f1 == T;
  const int g0 = first_anchor ? 1 : f0;
  const int g1 = last_anchor ? max(g0, T - 1) : f1;
  const long r0 = (long)g0 * N, r1 = (long)g1 * N;   // tokens read by the MMA path
  const int ntiles = (int)((r1 - r0 + 127) / 128);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_q_full[i], 1);
      mbar_init(&bar_q_empty[i], 1);
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], 4);
    }
    mbar_init(&bar_sum_full, 4);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, dev_status};

  if (warp == 0) {
    if (lane == 0) {
      int i = 0;
      for (; i < ntiles; ++i) {
        const int st = i & 1;
        if (i >= 2 && !mbar_wait(&bar_q_empty[st], ((i >> 1) - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&bar_q_full[st], kRoTile);
        const int row = (int)(r0 + (long)i * 128);
        tma_load_3d(sQ + st * kRoTile, &tm_q, &bar_q_full[st], 0, row, bh);
        tma_load_3d(sQ + st * kRoTile + kRoChunk, &tm_q, &bar_q_full[st], 64, row, bh);
      }
      if (i < ntiles)  // aborted: let the issued copies land
        for (int j = (i > 2 ? i - 2 : 0); j < i; ++j)
          mbar_wait_drain(&bar_q_full[j & 1], (j >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      bool ok = ntiles == 0 || mbar_wait(&bar_sum_full, 0, ab);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i & 1, a = i & 1;
        if (!mbar_wait(&bar_q_full[st], (i >> 1) & 1, ab)) break;
        if (i >= 2 && !mbar_wait(&bar_acc_empty[a], ((i >> 1) - 1) & 1, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_ss(tmem + a * 128, ro_kdesc(sQ + st * kRoTile, ks), ro_kdesc(sSum, ks), idesc,
                  ks > 0);
        umma_commit(&bar_q_empty[st]);
        umma_commit(&bar_acc_full[a]);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;             // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;      // accumulator row = state row for the operand
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    // zero rows of the anchor frames in this block
    const long zrows[2][2] = {{first_anchor ? 0L : 0L, first_anchor ? (long)N : 0L},
                              {last_anchor ? (long)(T - 1) * N : 0L, last_anchor ? TN : 0L}};
    for (int z = 0; z < 2; ++z)
      for (long t = zrows[z][0] + (threadIdx.x - 64); t < zrows[z][1]; t += 128) {
        uint4* d4 = reinterpret_cast<uint4*>(obh + (size_t)t * out.tok_stride);
#pragma unroll
        for (int u = 0; u < 16; ++u) d4[u] = make_uint4(0, 0, 0, 0);
      }
    const float cg = gate_logits ? 1.0f - sigmoidf_dev(__ldg(gate_logits + h)) : 1.0f;
    if (ntiles > 0) {
      // operand: row `row` of (S_fwd + S_bwd) (or of its transpose) as bf16,
      // K-major, 128B swizzle
      const size_t sbase = ((size_t)bh * nb + blk) * 128 * 128;
      if (!transpose_s) {
        const float4* Sf = reinterpret_cast<const float4*>(S_fwd + sbase + (size_t)row * 128);
        const float4* Sb = reinterpret_cast<const float4*>(S_bwd + sbase + (size_t)row * 128);
#pragma unroll 4
        for (int g = 0; g < 16; ++g) {
          const float4 a0 = __ldg(Sf + g * 2), a1 = __ldg(Sf + g * 2 + 1);
          const float4 b0 = __ldg(Sb + g * 2), b1 = __ldg(Sb + g * 2 + 1);
          uint4 pk;
          pk.x = pack_bf16(a0.x + b0.x, a0.y + b0.y);
          pk.y = pack_bf16(a0.z + b0.z, a0.w + b0.w);
          pk.z = pack_bf16(a1.x + b1.x, a1.y + b1.y);
          pk.w = pack_bf16(a1.z + b1.z, a1.w + b1.w);
          const int chunk = g >> 3, gg = g & 7;
          *reinterpret_cast<uint4*>(sSum + chunk * kRoChunk + row * 128 + ((gg ^ (row & 7)) << 4)) = pk;
        }
      } else {
        // column `row` of S: at each k the 128 threads read one S row, coalesced
        const float* Sf = S_fwd + sbase + row;
        const float* Sb = S_bwd + sbase + row;
#pragma unroll 2
        for (int g = 0; g < 16; ++g) {
          float a[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            a[u] = __ldg(Sf + (size_t)(g * 8 + u) * 128) + __ldg(Sb + (size_t)(g * 8 + u) * 128);
          uint4 pk;
          pk.x = pack_bf16(a[0], a[1]);
          pk.y = pack_bf16(a[2], a[3]);
          pk.z = pack_bf16(a[4], a[5]);
          pk.w = pack_bf16(a[6], a[7]);
          const int chunk = g >> 3, gg = g & 7;
          *reinterpret_cast<uint4*>(sSum + chunk * kRoChunk + row * 128 + ((gg ^ (row & 7)) << 4)) = pk;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sum_full);
      for (int i = 0; i < ntiles; ++i) {
        const int a = i & 1;
        if (!warp_wait(&bar_acc_full[a], (i >> 1) & 1, ab)) break;
        tc_fence_after();
        const long t = r0 + (long)i * 128 + row;
        const bool live = t < r1;
        __nv_bfloat16* dst = obh + (size_t)t * out.tok_stride;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + a * 128 + c * 32, r);
          tmem_ld_wait();
          if (live) {
            uint4 pk[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
            for (int u = 0; u < 16; ++u)
              pw[u] = pack_bf16(__uint_as_float(r[2 * u]) * cg, __uint_as_float(r[2 * u + 1]) * cg);
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) d4[u] = pk[u];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_acc_empty[a]);
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

cudaError_t launch_readout_bf16(const CUtensorMap& tm_q, const float* S_fwd, const float* S_bwd,
                                void* o, int B, int H, int T, int N, int bf, int anchors, int nb,
                                int n_ctx, const ReadoutOut& out, bool transpose_s,
                                const float* gate_logits, int32_t* dev_status,
                                cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(readout_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRoSmem);
  if (e != cudaSuccess) return e;
  readout_bf16_kernel<<<B * H * (nb + (n_ctx > 0 ? 1 : 0)), kRoThreads, kRoSmem, stream>>>(
      tm_q, S_fwd, S_bwd, static_cast<__nv_bfloat16*>(o), H, T, N, bf, anchors, nb, n_ctx, out,
      transpose_s ? 1 : 0, gate_logits, dev_status);
  return cudaGetLastError();
}

}  // namespace vdn
