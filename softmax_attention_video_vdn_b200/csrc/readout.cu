// readout.cu - linear-branch readout on sm_100a (bf16 inputs):
//   o_lin[t] = c_h (S_fwd(b) + S_bwd(b)) q_t   for tokens t of non-anchor
//   frames of block b, and 0 for anchor frames; c_h = 1, or 1 - sigmoid(gate
//   logit of head h) when the result is the linear half of the gated Z.
//   With transpose_s the kernel multiplies by (S_fwd(b) + S_bwd(b))^T: the
//   backward's dq_t = S^T do_t, with do in place of q.
// sd114.wiki, bidirectional linear branch: the query reads both states and
// the results are summed.
//
// Persistent: one CTA per SM. The 128-row Q tiles of all (b, h, block) are
// numbered in order (b, h major, then block, then tile), and CTA c takes the
// contiguous range [c * total / grid, (c + 1) * total / grid), so every SM
// streams the same number of tiles whatever the block count. A range crosses
// a few (b, h, block) segments; the epilogue warps write S_fwd + S_bwd of a
// segment as bf16 into one of two shared-memory operand buffers (128-byte-
// swizzled K-major: the B operand, N = dv rows, K = d), the next segment's
// while the current one's tiles stream, so the tensor core never waits for
// an operand. Q tiles come through a 3-stage TMA ring; one thread issues
// M=128, N=128, K=16 tcgen05 MMAs into four TMEM accumulators (4 x 128
// columns); each of four warps converts its 32 rows to bf16 into a
// double-buffered, 128-byte-swizzled staging tile in shared memory and
// stores it with two TMA tensor stores (coalesced full rows instead of 32
// rows per store instruction). The last tile of a block, whose rows run into
// the next block, is stored row by row for its rows inside the block only.
// The rows that are zero (anchor frames, context tokens) are split evenly
// over the CTAs as well. Warp roles (192 threads): warp 0 TMA, warp 1 MMA,
// warps 2-5 operand + epilogue.
#include "kernels.h"

namespace vdn {

constexpr int kRoThreads = 192;
constexpr int kRoStages = 3;                  // Q ring depth
constexpr int kRoAcc = 4;                     // TMEM accumulators (128 columns each)
constexpr uint32_t kRoTile = 128 * 128 * 2;   // 128 x 128 bf16
constexpr uint32_t kRoChunk = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
constexpr uint32_t kRoStage = 32 * 128 * 2;   // staging: 32 rows x 128 bf16 (two TMA boxes)
// 2 operands + Q ring + 4 warps x 2 staging tiles
constexpr size_t kRoSmem = 1024 + (2 + kRoStages) * kRoTile + 8 * kRoStage;

// TMA tensor store of a 4-D box from shared memory (bulk async-group).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
      :
      : "l"(map), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most n bulk groups of this thread still reading shared memory
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}
template <int n>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(n) : "memory");
}

__device__ __forceinline__ uint64_t ro_kdesc(const uint8_t* tile, int ks) {
  return sdesc_sw128(smem_u32(tile) + (ks >> 2) * kRoChunk + (ks & 3) * 32, 16, 1024);
}

// Rows [r0, r1) of one (b, h) that block blk multiplies by its states: the
// block's frames without the anchor frames (0 and T-1) at its ends; nt
// 128-row tiles cover them (the last one ragged).
struct RoSpan {
  long r0, r1;
  int nt;
};
__device__ __forceinline__ RoSpan ro_span(int blk, int T, int N, int bf, int anchors) {
  const int f0 = blk * bf, f1 = min(T, f0 + bf);
  const int g0 = (anchors && f0 == 0) ? 1 : f0;
  const int g1 = (anchors && f1 == T) ? max(g0, T - 1) : f1;
  RoSpan sp;
  sp.r0 = (long)g0 * N;
  sp.r1 = (long)max(g0, g1) * N;
  sp.nt = (int)((sp.r1 - sp.r0 + 127) / 128);
  return sp;
}

struct RoShape {
  int T, N, bf, anchors, nb;
};

// A position in the tile order: tile i of block blk of (b, h) = bh.
struct RoCursor {
  int bh, blk, i;
  RoSpan sp;
};

// The cursor at tile g of the order (per_bh tiles per (b, h), g < B*H*per_bh).
__device__ __forceinline__ RoCursor ro_locate(long g, long per_bh, const RoShape& S) {
  RoCursor c;
  c.bh = (int)(g / per_bh);
  long rem = g - (long)c.bh * per_bh;
  c.blk = 0;
  c.sp = ro_span(0, S.T, S.N, S.bf, S.anchors);
  while (rem >= c.sp.nt) {  // ends inside this (b, h): rem < per_bh
    rem -= c.sp.nt;
    ++c.blk;
    c.sp = ro_span(c.blk, S.T, S.N, S.bf, S.anchors);
  }
  c.i = (int)rem;
  return c;
}

// The (b, h, block) segment after (bh, blk) that has tiles (per_bh > 0).
__device__ __forceinline__ void ro_next_segment(int& bh, int& blk, const RoShape& S) {
  do {
    if (++blk == S.nb) {
      blk = 0;
      ++bh;
    }
  } while (ro_span(blk, S.T, S.N, S.bf, S.anchors).nt == 0);
}

__device__ __forceinline__ void ro_advance(RoCursor& c, const RoShape& S) {
  if (++c.i < c.sp.nt) return;
  c.i = 0;
  ro_next_segment(c.bh, c.blk, S);
  c.sp = ro_span(c.blk, S.T, S.N, S.bf, S.anchors);
}

__global__ void __launch_bounds__(kRoThreads, 1)
    readout_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_o, int o_tok_dim,
                        const float* __restrict__ S_fwd,
                        const float* __restrict__ S_bwd, __nv_bfloat16* __restrict__ o, int BH,
                        int H, int T, int N, int bf, int anchors, int nb, int n_ctx,
                        const ReadoutOut out, int transpose_s,
                        const float* __restrict__ gate_logits, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q_full[kRoStages], bar_q_empty[kRoStages],
      bar_acc_full[kRoAcc], bar_acc_empty[kRoAcc], bar_sum_full[2], bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sSum = base;                // 2 operand buffers
  uint8_t* sQ = base + 2 * kRoTile;    // Q ring
  uint8_t* sStage = sQ + kRoStages * kRoTile;  // [4 warps][2][32 rows x 256 B]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RoShape shp{T, N, bf, anchors, nb};
  const long TN = (long)T * N;         // video tokens of a head
  // tiles per (b, h) and this CTA's range of the tile order
  long per_bh = 0;
  for (int blk = 0; blk < nb; ++blk) per_bh += ro_span(blk, T, N, bf, anchors).nt;
  const long total = (long)BH * per_bh;
  const long start = total * blockIdx.x / gridDim.x;
  const long end = total * (blockIdx.x + 1) / gridDim.x;
  const int ntiles = (int)(end - start);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRoStages; ++i) {
      mbar_init(&bar_q_full[i], 1);
      mbar_init(&bar_q_empty[i], 1);
    }
    for (int i = 0; i < kRoAcc; ++i) {
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], 4);
    }
    mbar_init(&bar_sum_full[0], 4);
    mbar_init(&bar_sum_full[1], 4);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 128 * kRoAcc);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, dev_status};

  if (warp == 0) {
    if (lane == 0 && ntiles > 0) {
      RoCursor cur = ro_locate(start, per_bh, shp);
      int n = 0;
      for (; n < ntiles; ++n) {
        const int st = n % kRoStages, use = n / kRoStages;
        if (use > 0 && !mbar_wait(&bar_q_empty[st], (use - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&bar_q_full[st], kRoTile);
        const int row = (int)(cur.sp.r0 + (long)cur.i * 128);
        tma_load_3d(sQ + st * kRoTile, &tm_q, &bar_q_full[st], 0, row, cur.bh);
        tma_load_3d(sQ + st * kRoTile + kRoChunk, &tm_q, &bar_q_full[st], 64, row, cur.bh);
        if (n + 1 < ntiles) ro_advance(cur, shp);
      }
      if (n < ntiles)  // aborted: let the issued copies land
        for (int j = (n > kRoStages ? n - kRoStages : 0); j < n; ++j)
          mbar_wait_drain(&bar_q_full[j % kRoStages], (j / kRoStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      if (ntiles > 0) {
        RoCursor cur = ro_locate(start, per_bh, shp);
        int seg = -1;
        for (int n = 0; n < ntiles; ++n) {
          if (n == 0 || cur.i == 0) {  // first tile of a segment: its operand
            ++seg;
            if (!mbar_wait(&bar_sum_full[seg & 1], (seg >> 1) & 1, ab)) break;
          }
          const int st = n % kRoStages, a = n % kRoAcc;
          if (!mbar_wait(&bar_q_full[st], (n / kRoStages) & 1, ab)) break;
          if (n >= kRoAcc && !mbar_wait(&bar_acc_empty[a], ((n / kRoAcc) - 1) & 1, ab)) break;
          tc_fence_after();
          const uint8_t* sB = sSum + (seg & 1) * kRoTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_ss(tmem + a * 128, ro_kdesc(sQ + st * kRoTile, ks), ro_kdesc(sB, ks), idesc,
                    ks > 0);
          umma_commit(&bar_q_empty[st]);
          umma_commit(&bar_acc_full[a]);
          if (n + 1 < ntiles) ro_advance(cur, shp);
        }
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    const int wq = warp & 3;             // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;      // accumulator row = state row for the operand
    const int et = threadIdx.x - 64;     // 0..127
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    auto head_out = [&](int bh) {
      const int b = bh / H, h = bh - b * H;
      return o + (size_t)b * out.b_stride + (size_t)h * out.h_stride + out.off;
    };
    // zero rows, this CTA's share: per (b, h) frame 0 and frame T-1 (with
    // anchors; the same rows when T = 1), then the context tokens
    {
      const long za = anchors ? (long)N : 0;
      const long zper = 2 * za + n_ctx;
      const long ztot = (long)BH * zper;
      const long zs = ztot * blockIdx.x / gridDim.x, ze = ztot * (blockIdx.x + 1) / gridDim.x;
      for (long zr = zs + (et >> 4); zr < ze; zr += 8) {
        const int bh = (int)(zr / zper);
        const long j = zr - (long)bh * zper;
        const long t = j < za ? j : (j < 2 * za ? (long)(T - 1) * N + (j - za) : TN + (j - 2 * za));
        reinterpret_cast<uint4*>(head_out(bh) + (size_t)t * out.tok_stride)[et & 15] =
            make_uint4(0, 0, 0, 0);
      }
    }
    // operand of segment (bh, blk) into buffer buf: row `row` of
    // S_fwd + S_bwd (or of its transpose) as bf16, K-major, 128B swizzle
    auto build = [&](int bh, int blk, int buf) {
      uint8_t* dstS = sSum + buf * kRoTile;
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
          *reinterpret_cast<uint4*>(dstS + chunk * kRoChunk + row * 128 + ((gg ^ (row & 7)) << 4)) = pk;
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
          *reinterpret_cast<uint4*>(dstS + chunk * kRoChunk + row * 128 + ((gg ^ (row & 7)) << 4)) = pk;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sum_full[buf]);
    };
    if (ntiles > 0) {
      RoCursor cur = ro_locate(start, per_bh, shp);
      // segments 0 and 1 of the range
      build(cur.bh, cur.blk, 0);
      if (start - cur.i + cur.sp.nt < end) {
        int bh1 = cur.bh, blk1 = cur.blk;
        ro_next_segment(bh1, blk1, shp);
        build(bh1, blk1, 1);
      }
      int seg = 0;
      bool prev_staged = false;
      for (int n = 0; n < ntiles; ++n) {
        if (n > 0 && cur.i == 0) {
          // first tile of segment seg + 1; every tile of segment seg - 1 has
          // been drained, so its MMAs are done and its buffer is free for
          // segment seg + 2
          ++seg;
          if (start + n + cur.sp.nt < end) {
            int bh2 = cur.bh, blk2 = cur.blk;
            ro_next_segment(bh2, blk2, shp);
            build(bh2, blk2, (seg + 1) & 1);
          }
        }
        const int a = n % kRoAcc;
        if (!warp_wait(&bar_acc_full[a], (n / kRoAcc) & 1, ab)) break;
        tc_fence_after();
        const int hh = cur.bh % H;
        const float cg = gate_logits ? 1.0f - sigmoidf_dev(__ldg(gate_logits + hh)) : 1.0f;
        const long tw = cur.sp.r0 + (long)cur.i * 128 + wq * 32;  // this warp's first row
        const long t = tw + lane;
        // a warp whose 32 rows all lie in the block stores through TMA
        const bool staged = tw + 32 <= cur.sp.r1;
        const bool live = t < cur.sp.r1;
        uint8_t* stg = sStage + ((wq * 2 + (n & 1)) * kRoStage);
        if (staged) {
          // the store issued from this staging tile two tiles ago has read
          // it (the last group may stay in flight if it is the previous
          // tile's, which used the other tile)
          if (lane == 0) {
            if (prev_staged)
              bulk_wait_read<1>();
            else
              bulk_wait_read<0>();
          }
          __syncwarp();
        }
        prev_staged = staged;
        __nv_bfloat16* dst = head_out(cur.bh) + (size_t)t * out.tok_stride;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + a * 128 + c * 32, r);
          tmem_ld_wait();
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pw[u] = pack_bf16(__uint_as_float(r[2 * u]) * cg, __uint_as_float(r[2 * u + 1]) * cg);
          if (staged) {
            // box c >> 1 (64 columns), row `lane` of 128 bytes, 16-byte
            // chunks (c & 1) * 4 + u, 128-byte swizzle
            uint8_t* rowp = stg + (c >> 1) * (kRoStage / 2) + lane * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              *reinterpret_cast<uint4*>(rowp + ((((c & 1) * 4 + u) ^ (lane & 7)) << 4)) = pk[u];
          } else if (live) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) d4[u] = pk[u];
          }
        }
        tc_fence_before();
        if (staged) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar_acc_empty[a]);
          if (staged) {
            const int b = cur.bh / H;
            const int y = (int)tw;
            if (o_tok_dim == 1) {  // dims (dv, L, H, B)
              tma_store_4d(&tm_o, stg, 0, y, hh, b);
              tma_store_4d(&tm_o, stg + kRoStage / 2, 64, y, hh, b);
            } else {               // dims (dv, H, L, B)
              tma_store_4d(&tm_o, stg, 0, hh, y, b);
              tma_store_4d(&tm_o, stg + kRoStage / 2, 64, hh, y, b);
            }
            bulk_commit_group();
          }
        }
        if (n + 1 < ntiles) ro_advance(cur, shp);
      }
      if (lane == 0) bulk_wait<0>();  // every tensor store complete
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128 * kRoAcc);
  }
}

cudaError_t launch_readout_bf16(const CUtensorMap& tm_q, const float* S_fwd, const float* S_bwd,
                                void* o, int B, int H, int T, int N, int bf, int anchors, int nb,
                                int n_ctx, const ReadoutOut& out, bool transpose_s,
                                const float* gate_logits, int32_t* dev_status,
                                cudaStream_t stream) {
  // output map over the same addressing as the row stores, dimensions in
  // increasing stride order: (dv, L, H, B) or (dv, H, L, B)
  const long L = (long)T * N + n_ctx;
  const bool tok_first = out.tok_stride < out.h_stride;  // equal only when H = 1
  CUtensorMap tm_o;
  const cuuint64_t dims[4] = {128, (cuuint64_t)(tok_first ? L : H), (cuuint64_t)(tok_first ? H : L),
                              (cuuint64_t)B};
  const cuuint64_t str[3] = {(cuuint64_t)(tok_first ? out.tok_stride : out.h_stride) * 2,
                             (cuuint64_t)(tok_first ? out.h_stride : out.tok_stride) * 2,
                             (cuuint64_t)out.b_stride * 2};
  const cuuint32_t box[4] = {64, tok_first ? 32u : 1u, tok_first ? 1u : 32u, 1};
  if (!make_map(&tm_o, static_cast<__nv_bfloat16*>(o) + out.off, 4, dims, str, box))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(readout_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRoSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  readout_bf16_kernel<<<sms, kRoThreads, kRoSmem, stream>>>(
      tm_q, tm_o, tok_first ? 1 : 2, S_fwd, S_bwd, static_cast<__nv_bfloat16*>(o), B * H, H, T,
      N, bf, anchors, nb, n_ctx, out, transpose_s ? 1 : 0, gate_logits, dev_status);
  return cudaGetLastError();
}

}  // namespace vdn
