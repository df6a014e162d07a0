// gated_merge.cu - the two branches' separate output projections on sm_100a.
// mlsanity abstract: separate output projections and learnable gates
// calibrate the two branches. The gate is already applied to Z (by the
// softmax epilogue), so the merge is one product with the stacked weights:
//   Y [M, d_out] = Z [M, 2*H*dv] x [W1; W2],  M = B*L tokens.
//
// bf16: a persistent kernel, one CTA per SM, looping over 128 x 256 output
// tiles. TMA brings 64-wide K chunks of Z (K-major) and of W1 or W2
// (row-major [K, d_out], i.e. MN-major for the tensor core) through a
// 4-stage ring that runs on across tiles; one thread issues M=128, N=256,
// K=16 tcgen05 MMAs into one of two 256-column TMEM accumulators (tiles
// alternate), and four epilogue warps convert the other one to bf16, so a
// tile's epilogue overlaps the next tile's main loop. Rows past M and
// columns past d_out are zero-filled on load and masked on store.
// The same kernel also reads Z in the layout a head-sharded layer receives it
// in after its all-to-all (MergeGroups): [B, G, Ls, 2, H/G, dv], the K row of
// token (b, l) split into G segments of 2*(H/G)*dv, one per head group. A
// 4-D tensor map walks it; the K chunks are taken in the same global order
// (branch, head, 64 columns) as for the plain [B*L, 2, H, dv] layout, so the
// two layouts give the same Y bit for bit.
// f32 (and the per-head shared-weight form): a SIMT kernel.
#include "kernels.h"

namespace vdn {


__global__ void __launch_bounds__(kMergeThreads, 1)
    gated_merge_bf16_kernel(const __grid_constant__ CUtensorMap tm_z,
                            const __grid_constant__ CUtensorMap tm_w1,
                            const __grid_constant__ CUtensorMap tm_w2,
                            __nv_bfloat16* __restrict__ Y, int M, int n_out, int K1,
                            MergeGroups grp, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kMergeStages], bar_empty[kMergeStages];
  __shared__ __align__(8) uint64_t bar_acc_full[2], bar_acc_empty[2], bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tiles in N-fastest raster: the CTAs working at the same time cover a few
  // 128-row blocks of Z with all their column tiles, so each block of Z is
  // read from DRAM about once. Rows: plain layout, one run of M rows;
  // grouped layout, M / Ls runs (batch items) of Ls rows each, tiled per run.
  const int n_tiles = (n_out + 255) / 256;
  const int rows = grp.groups ? grp.Ls : M;
  const int m_tiles = (rows + 127) / 128;
  const int runs = grp.groups ? M / grp.Ls : 1;
  const int total = runs * m_tiles * n_tiles;
  const int nchunks = (2 * K1) / 64;
  const int k1_chunks = K1 / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMergeStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], 4);   // the four epilogue warps
    }
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_z);
    tma_prefetch_desc(&tm_w1);
    tma_prefetch_desc(&tm_w2);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, dev_status};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t cg = 0;   // chunks issued so far (ring position, across tiles)
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int mt = tile / n_tiles, n0 = (tile - mt * n_tiles) * 256;
        const int b = mt / m_tiles, m0 = (mt - b * m_tiles) * 128;
        int half = 0, src = 0, hl = 0, cc = 0;  // grouped layout: chunk c's place
        for (int c = 0; c < nchunks; ++c, ++cg) {
          const int st = cg % kMergeStages;
          const uint32_t use = cg / kMergeStages;
          if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, ab)) { ok = false; break; }
          uint8_t* s = base + st * kMergeStageBytes;
          mbar_arrive_expect_tx(&bar_full[st], kMergeStageBytes);
          if (grp.groups == 0) {
            tma_load_2d(s, &tm_z, &bar_full[st], c * 64, m0);
          } else {
            // chunk c = (branch, head h, 64-column piece cc) of the plain K
            // order; head h lives in group h / Hs at local head h % Hs
            tma_load_3d(s, &tm_z, &bar_full[st], ((half * grp.Hs + hl) * grp.dv_chunks + cc) * 64,
                        m0, b * grp.groups + src);
            if (++cc == grp.dv_chunks) {
              cc = 0;
              if (++hl == grp.Hs) {
                hl = 0;
                if (++src == grp.groups) {
                  src = 0;
                  ++half;
                }
              }
            }
          }
          const CUtensorMap* wm = c < k1_chunks ? &tm_w1 : &tm_w2;
          const int wrow = (c < k1_chunks ? c : c - k1_chunks) * 64;
#pragma unroll
          for (int nb = 0; nb < 4; ++nb)
            tma_load_2d(s + kMergeABytes + nb * kMergeBBox, wm, &bar_full[st], n0 + nb * 64, wrow);
        }
      }
      if (!ok)  // aborted: let the issued copies land before exit
        for (uint32_t x = (cg > kMergeStages ? cg - kMergeStages : 0); x < cg; ++x)
          mbar_wait_drain(&bar_full[x % kMergeStages], (x / kMergeStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    // Tile i accumulates in TMEM columns 256 * (i % 2), so the epilogue of
    // one tile overlaps the main loop of the next.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 256, 0, 1);
      uint32_t cg = 0;
      int tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tcount) {
        const int buf = tcount & 1;
        const uint32_t use = tcount >> 1;
        if (use > 0 && !mbar_wait(&bar_acc_empty[buf], (use - 1) & 1, ab)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dtm = tmem + buf * 256;
        for (int c = 0; c < nchunks; ++c, ++cg) {
          const int st = cg % kMergeStages;
          if (!mbar_wait(&bar_full[st], (cg / kMergeStages) & 1, ab)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + st * kMergeStageBytes);
          const uint32_t sb = sa + kMergeABytes;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t da = sdesc_sw128(sa + ks * 32, 16, 1024);          // K-major
            const uint64_t db = sdesc_sw128(sb + ks * 2048, kMergeBBox, 1024);  // MN-major
            umma_ss(dtm, da, db, idesc, (c > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bar_empty[st]);
        }
        if (!ok) break;
        umma_commit(&bar_acc_full[buf]);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue
    // Warps 2-5: TMEM lane quarter warp % 4, one output row per thread.
    const int q = warp & 3;
    const uint32_t lane_addr = uint32_t(q * 32) << 16;
    int tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const int buf = tcount & 1;
      if (!warp_wait(&bar_acc_full[buf], (tcount >> 1) & 1, ab)) break;
      tc_fence_after();
      const int mt = tile / n_tiles, n0 = (tile - mt * n_tiles) * 256;
      const int b = mt / m_tiles, m0 = (mt - b * m_tiles) * 128;
      const int m = m0 + q * 32 + lane;  // row within this run
      __nv_bfloat16* yrow = Y + ((size_t)b * rows + m) * n_out;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + buf * 256 + c * 32, r);
        tmem_ld_wait();
        uint4 pk[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pw[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        if (m < rows) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = n0 + c * 32 + i * 8;
            if (col < n_out) *reinterpret_cast<uint4*>(yrow + col) = pk[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// fp32 merge. Z [B*L, 2, H, dv]. w_per_head = 0: Y[m, :] = sum over the 2*H*dv
// inputs of the row times [W1; W2]. w_per_head = 1: Y[m, h, :] =
// Z[m,0,h,:] W1 + Z[m,1,h,:] W2. One thread per output element, fp32 FMA.
__global__ void gated_merge_f32_kernel(const float* __restrict__ Z, const float* __restrict__ W1,
                                       const float* __restrict__ W2, float* __restrict__ Y,
                                       long M, int H, int dv, int n_out, int w_per_head) {
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (!w_per_head) {
    const long total = M * n_out;
    if (idx >= total) return;
    const long m = idx / n_out;
    const int o = (int)(idx - m * n_out);
    const int HD = H * dv;
    const float* z = Z + m * 2 * HD;
    float acc = 0.f;
    for (int kk = 0; kk < HD; ++kk) acc = fmaf(z[kk], W1[(size_t)kk * n_out + o], acc);
    for (int kk = 0; kk < HD; ++kk) acc = fmaf(z[HD + kk], W2[(size_t)kk * n_out + o], acc);
    Y[idx] = acc;
  } else {
    const long total = M * H * n_out;
    if (idx >= total) return;
    const long mh = idx / n_out;
    const int o = (int)(idx - mh * n_out);
    const long m = mh / H;
    const int h = (int)(mh - m * H);
    const float* zs = Z + (m * 2 * H + h) * dv;
    const float* zl = Z + ((m * 2 + 1) * H + h) * dv;
    float acc = 0.f;
    for (int kk = 0; kk < dv; ++kk) acc = fmaf(zs[kk], W1[(size_t)kk * n_out + o], acc);
    for (int kk = 0; kk < dv; ++kk) acc = fmaf(zl[kk], W2[(size_t)kk * n_out + o], acc);
    Y[idx] = acc;
  }
}

}  // namespace vdn
