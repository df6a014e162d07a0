// softmax_window.cu - block-sparse softmax branch of the VDN hybrid layer on
// sm_100a, with the linear-branch readout and the gate fused in the epilogue.
//
// sd114.wiki, bidirectional sliding-window softmax branch: each query attends
// the key frames of its 3-block window plus the first and last frames (which
// themselves attend every frame). Same article, bidirectional linear branch:
// the query also reads the forward and backward states and the results are
// summed. mlsanity abstract: the branches are calibrated by learnable gates.
//
// One CTA per SM runs a persistent loop over work items; an item is a pair of
// 128-row query tiles (tile 0, tile 1) of one segment and one (b, h), so each
// K/V tile fetched from L2 feeds 256 query rows. Items are taken from a global
// counter (the producer fetches, and hands the index to the other roles
// through a 4-slot ring in shared memory), so the items in flight are always
// consecutive and share their key windows in L2. Warp roles (384 threads):
//   warp 0      TMA producer: Q pair, then K and V tiles of every key range
//   warp 1      tcgen05 issuer
//   warps 2-3   readout operand (S_fwd + S_bwd) as bf16 in shared memory
//   warps 4-7   softmax + epilogue of tile 0     (setmaxnreg 208)
//   warps 8-11  softmax + epilogue of tile 1     (setmaxnreg 208)
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// P_t (bf16) overwrites the first 64 columns of S_t; after the last key tile
// the readout OL_t = Q_t (S_fwd + S_bwd)^T is computed into S_t.
// MMA issue order per key tile j: PV0(j-1), S0(j), PV1(j-1), S1(j). MMAs of
// one thread execute in issue order, so S_t(j) overwrites P_t(j-1) only after
// PV_t(j-1) has read it, and every commit of S_t(j) also covers PV_t(j-1):
// when a softmax warpgroup sees S_t(j), O_t is stable and may be rescaled.
// Each softmax warpgroup thus has two MMAs of the other tile to hide behind.
// The online softmax keeps a per-row reference maximum and rescales O only
// when a new row maximum exceeds it by more than 2^8; the final division by
// the row sum uses the same reference.
#include "kernels.h"

namespace vdn {

constexpr int kSmThreads = 384;
constexpr uint32_t kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one TMA box)
constexpr uint32_t kColS = 0, kColO = 256;    // S_t at t*128, O_t at 256 + t*128
constexpr int kRegsSoftmax = 208, kRegsOther = 88;  // 208*256 + 88*128 = 168*384
// Work-item ring: the producer publishes item indices, read by the MMA
// thread (1 arrival), the readout warps (2) and the softmax warps (8).
constexpr int kItemSlots = 4;
constexpr int kItemConsumers = 11;
static_assert(kRegsSoftmax * 256 + kRegsOther * 128 <= 168 * kSmThreads, "register split");

struct Item {
  int bh, seg, q_start, q_rows, nkv;
};

// Work items run segment by segment (heaviest segments first), then head by
// head, then pair by pair: the CTAs in flight at any time share one or two
// heads' key window, which therefore stays in L2.
__device__ __forceinline__ Item decode_item(const SoftmaxPlan& P, int BH, int w) {
  Item it;
  int s = 0;
  while (s + 1 < P.n_seg && P.tile_begin[s + 1] * BH <= w) ++s;
  const int np = (s + 1 < P.n_seg ? P.tile_begin[s + 1] : P.total_tiles) - P.tile_begin[s];
  const int e = w - P.tile_begin[s] * BH;
  it.bh = e / np;
  const int pair = e - it.bh * np;
  it.seg = s;
  it.q_start = P.q0[s] + pair * (2 * kQTile);
  const int rem = P.q1[s] - it.q_start;
  it.q_rows = rem < 2 * kQTile ? rem : 2 * kQTile;  // valid rows of the pair
  int n = 0;
  for (int r = 0; r < P.nr[s]; ++r) n += (P.k1[s][r] - P.k0[s][r] + kKvTile - 1) / kKvTile;
  it.nkv = n;
  return it;
}

// Walks the key tiles of an item: start token and number of valid rows.
struct KvWalk {
  int r, pos;
  __device__ __forceinline__ void init(const SoftmaxPlan& P, int s) {
    r = 0;
    pos = P.k0[s][0];
  }
  __device__ __forceinline__ int valid(const SoftmaxPlan& P, int s) const {
    const int rem = P.k1[s][r] - pos;
    return rem < kKvTile ? rem : kKvTile;
  }
  __device__ __forceinline__ void next(const SoftmaxPlan& P, int s) {
    pos += kKvTile;
    if (pos >= P.k1[s][r]) {
      ++r;
      if (r < P.nr[s]) pos = P.k0[s][r];
    }
  }
};

// K-major operand (rows x 128 bf16, two 64-wide TMA chunks), K step `ks`
// (16 elements) of 8.
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile, int ks) {
  return sdesc_sw128(smem_u32(tile) + (ks >> 2) * kChunkBytes + (ks & 3) * 32, 16, 1024);
}
// MN-major operand (128 k-rows x 128 n, two 64-wide n chunks), K step `ks`.
__device__ __forceinline__ uint64_t mnmajor_desc(const uint8_t* tile, int ks) {
  return sdesc_sw128(smem_u32(tile) + ks * 2048, kChunkBytes, 1024);
}

// Consumer side of the work-item ring: wait for slot it % kItemSlots, read
// the item index (-1 = no more work), release the slot. Returns false when
// the CTA is aborting. `arrive` is true for the one lane per warp that
// counts towards the slot's release.
__device__ __forceinline__ bool next_item(uint64_t* full, uint64_t* empty, const int* slot,
                                          int it, bool arrive, const Abort& ab, int* w) {
  const int sl = it % kItemSlots;
  if (!mbar_wait(&full[sl], (it / kItemSlots) & 1, ab)) return false;
  *w = *reinterpret_cast<const volatile int*>(&slot[sl]);
  if (arrive) mbar_arrive(&empty[sl]);
  return true;
}

// Warp-uniform form for the softmax warps (followed by tcgen05.ld).
__device__ __forceinline__ bool warp_next_item(uint64_t* full, uint64_t* empty, const int* slot,
                                               int it, bool arrive, const Abort& ab, int* w) {
  const bool ok = next_item(full, empty, slot, it, arrive, ab, w);
  *w = __shfl_sync(0xffffffffu, *w, 0);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
}
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
}

__global__ void __launch_bounds__(kSmThreads, 1)
    softmax_window_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ SoftmaxArgs A) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q_full, bar_q_empty;
  __shared__ __align__(8) uint64_t bar_k_full[kKvStages], bar_v_full[kKvStages],
      bar_k_empty[kKvStages], bar_v_empty[kKvStages];
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_p_full[2], bar_o_full[2], bar_o_empty[2];
  __shared__ __align__(8) uint64_t bar_sum_full, bar_sum_empty, bar_drain;
  __shared__ __align__(8) uint64_t bar_item_full[kItemSlots], bar_item_empty[kItemSlots];
  __shared__ int item_slot[kItemSlots];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = base;                       // tile 0, tile 1
  uint8_t* sSum = base + 2 * kTileBytes;
  uint8_t* sK = base + 3 * kTileBytes;
  uint8_t* sV = base + (3 + kKvStages) * kTileBytes;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const SoftmaxPlan& P = A.plan;
  const bool fused = A.S_fwd != nullptr;
  const int n_items = P.total_tiles * A.BH;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    for (int i = 0; i < kKvStages; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
      mbar_init(&bar_v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_p_full[t], 4);
      mbar_init(&bar_o_full[t], 1);
      mbar_init(&bar_o_empty[t], 4);
    }
    mbar_init(&bar_sum_full, 2);
    mbar_init(&bar_sum_empty, 1);
    mbar_init(&bar_drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&bar_item_full[i], 1);
      mbar_init(&bar_item_empty[i], kItemConsumers);
    }
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, A.dev_status};

  // Register budget per role is set as the first statement of each role's
  // branch so that the whole role body is compiled against it.
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec();
    if (lane == 0) {
      uint32_t kvc = 0, q_issued = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        // fetch the next item and publish it to the other roles
        const int sl = it % kItemSlots;
        if (it >= kItemSlots &&
            !mbar_wait(&bar_item_empty[sl], ((it / kItemSlots) - 1) & 1, ab)) {
          ok = false;
          break;
        }
        int w = atomicAdd(A.work_counter, 1);
        if (w >= n_items) w = -1;
        item_slot[sl] = w;
        mbar_arrive(&bar_item_full[sl]);
        if (w < 0) break;
        const Item I = decode_item(P, A.BH, w);
        if (it > 0 && !mbar_wait(&bar_q_empty, (it - 1) & 1, ab)) { ok = false; break; }
        ++q_issued;
        mbar_arrive_expect_tx(&bar_q_full, 2 * kTileBytes);
        for (int t = 0; t < 2; ++t) {
          tma_load_3d(sQ + t * kTileBytes, &tm_q, &bar_q_full, 0, I.q_start + t * kQTile, I.bh);
          tma_load_3d(sQ + t * kTileBytes + kChunkBytes, &tm_q, &bar_q_full, 64,
                      I.q_start + t * kQTile, I.bh);
        }
        KvWalk kw;
        kw.init(P, I.seg);
        for (int j = 0; j < I.nkv; ++j) {
          const int st = kvc % kKvStages;
          const uint32_t use = kvc / kKvStages;
          uint8_t* k_dst = sK + st * kTileBytes;
          uint8_t* v_dst = sV + st * kTileBytes;
          if (use > 0 && !mbar_wait(&bar_k_empty[st], (use - 1) & 1, ab)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar_k_full[st], kTileBytes);
          tma_load_3d(k_dst, &tm_k, &bar_k_full[st], 0, kw.pos, I.bh);
          tma_load_3d(k_dst + kChunkBytes, &tm_k, &bar_k_full[st], 64, kw.pos, I.bh);
          if (use > 0 && !mbar_wait(&bar_v_empty[st], (use - 1) & 1, ab)) {
            // the K copy of this tile is in flight: drain it below
            mbar_wait_drain(&bar_k_full[st], use & 1);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[st], kTileBytes);
          tma_load_3d(v_dst, &tm_v, &bar_v_full[st], 0, kw.pos, I.bh);
          tma_load_3d(v_dst + kChunkBytes, &tm_v, &bar_v_full[st], 64, kw.pos, I.bh);
          kw.next(P, I.seg);
          ++kvc;
        }
      }
      if (!ok) {
        // let every issued copy land before shared memory is released
        if (q_issued > 0) mbar_wait_drain(&bar_q_full, (q_issued - 1) & 1);
        for (uint32_t c = (kvc > kKvStages ? kvc - kKvStages : 0); c < kvc; ++c) {
          mbar_wait_drain(&bar_k_full[c % kKvStages], (c / kKvStages) & 1);
          mbar_wait_drain(&bar_v_full[c % kKvStages], (c / kKvStages) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    setmaxnreg_dec();
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
      uint32_t kvc = 0, sc = 0, fc = 0;  // key tiles, S MMAs per query tile, fused items
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int w;
        if (!next_item(bar_item_full, bar_item_empty, item_slot, it, true, ab, &w)) break;
        if (w < 0) break;
        const Item I = decode_item(P, A.BH, w);
        const bool lin = fused && P.blk[I.seg] >= 0;
        if (!mbar_wait(&bar_q_full, it & 1, ab)) break;
        // key tile j = 0: S_t(0). The epilogue of the previous item must have
        // read O_t and S_t (which held the readout) first.
        {
          const int st = kvc % kKvStages;
          if (!mbar_wait(&bar_k_full[st], (kvc / kKvStages) & 1, ab)) break;
          for (int t = 0; t < 2; ++t) {
            if (it > 0 && !mbar_wait(&bar_o_empty[t], (it - 1) & 1, ab)) { ok = false; break; }
            tc_fence_after();
            const uint8_t* kt = sK + st * kTileBytes;
            const uint8_t* qt = sQ + t * kTileBytes;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              umma_ss(tmem + kColS + t * 128, kmajor_desc(qt, ks), kmajor_desc(kt, ks), idesc_qk,
                      ks > 0);
            umma_commit(&bar_s_full[t]);
          }
          if (!ok) break;
          umma_commit(&bar_k_empty[st]);
        }
        // key tiles j = 1 .. nkv: PV_t(j-1) then S_t(j) (or the readout after the last)
        for (int j = 1; j <= I.nkv && ok; ++j) {
          const int pst = kvc % kKvStages;            // stage of key tile j-1
          const uint32_t puse = kvc / kKvStages;
          const int st = (kvc + 1) % kKvStages;       // stage of key tile j
          const uint32_t use = (kvc + 1) / kKvStages;
          const bool last = (j == I.nkv);
          if (!mbar_wait(&bar_v_full[pst], puse & 1, ab)) { ok = false; break; }
          if (!last && !mbar_wait(&bar_k_full[st], use & 1, ab)) { ok = false; break; }
          if (last && lin && !mbar_wait(&bar_sum_full, fc & 1, ab)) { ok = false; break; }
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait(&bar_p_full[t], sc & 1, ab)) { ok = false; break; }
            tc_fence_after();
            const uint8_t* vt = sV + pst * kTileBytes;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              umma_ts(tmem + kColO + t * 128, tmem + kColS + t * 128 + ks * 8,
                      mnmajor_desc(vt, ks), idesc_pv, (j > 1 || ks > 0) ? 1u : 0u);
            const uint8_t* qt = sQ + t * kTileBytes;
            if (!last) {
              const uint8_t* kt = sK + st * kTileBytes;
#pragma unroll
              for (int ks = 0; ks < 8; ++ks)
                umma_ss(tmem + kColS + t * 128, kmajor_desc(qt, ks), kmajor_desc(kt, ks),
                        idesc_qk, ks > 0);
              umma_commit(&bar_s_full[t]);
            } else {
              if (lin) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                  umma_ss(tmem + kColS + t * 128, kmajor_desc(qt, ks), kmajor_desc(sSum, ks),
                          idesc_qk, ks > 0);
              }
              umma_commit(&bar_o_full[t]);
            }
          }
          if (!ok) break;
          umma_commit(&bar_v_empty[pst]);
          if (!last) umma_commit(&bar_k_empty[st]);
          ++sc;
          ++kvc;
        }
        if (!ok) break;
        if (lin) {
          umma_commit(&bar_sum_empty);
          ++fc;
        }
        umma_commit(&bar_q_empty);
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // --------------------------------------- readout operand (S_fwd + S_bwd)
    setmaxnreg_dec();
    {
      const int rt = threadIdx.x - 64;  // 0..63, rows rt and rt + 64
      uint32_t fc = 0;
      for (int it = 0;; ++it) {
        int w;
        if (!warp_next_item(bar_item_full, bar_item_empty, item_slot, it, lane == 0, ab, &w)) break;
        if (w < 0) break;
        const Item I = decode_item(P, A.BH, w);
        const int blk = P.blk[I.seg];
        if (!fused || blk < 0) continue;
        if (fc > 0 && !warp_wait(&bar_sum_empty, (fc - 1) & 1, ab)) break;
        const size_t off = ((size_t)I.bh * A.nb + blk) * 128 * 128;
        const float4* Sf = reinterpret_cast<const float4*>(A.S_fwd + off);
        const float4* Sb = reinterpret_cast<const float4*>(A.S_bwd + off);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int n = rt + rr * 64;
#pragma unroll 4
          for (int g = 0; g < 16; ++g) {
            const float4 a0 = __ldg(Sf + n * 32 + g * 2), a1 = __ldg(Sf + n * 32 + g * 2 + 1);
            const float4 b0 = __ldg(Sb + n * 32 + g * 2), b1 = __ldg(Sb + n * 32 + g * 2 + 1);
            uint4 pk;
            pk.x = pack_bf16(a0.x + b0.x, a0.y + b0.y);
            pk.y = pack_bf16(a0.z + b0.z, a0.w + b0.w);
            pk.z = pack_bf16(a1.x + b1.x, a1.y + b1.y);
            pk.w = pack_bf16(a1.z + b1.z, a1.w + b1.w);
            const int chunk = g >> 3, gg = g & 7;
            *reinterpret_cast<uint4*>(sSum + chunk * kChunkBytes + n * 128 + ((gg ^ (n & 7)) << 4)) = pk;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_sum_full);
        ++fc;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax + epilogue
    setmaxnreg_inc();
    const int t = (warp - 4) >> 2;          // query tile of this warpgroup
    const int wq = warp & 3;                // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;         // query row within the tile
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr + kColS + t * 128;
    const uint32_t o_addr = tmem + lane_addr + kColO + t * 128;
    const float sl2 = A.scale_log2;
    uint32_t sc = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int w;
      if (!warp_next_item(bar_item_full, bar_item_empty, item_slot, it, lane == 0, ab, &w)) break;
      if (w < 0) break;
      const Item I = decode_item(P, A.BH, w);
      KvWalk kw;
      kw.init(P, I.seg);
      float m_ref = -INFINITY;   // reference maximum (log2 units) of the exponentials
      uint64_t l_acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};  // packed row sums
      for (int j = 0; j < I.nkv; ++j, ++sc) {
        const int valid = kw.valid(P, I.seg);
        kw.next(P, I.seg);
        if (!warp_wait(&bar_s_full[t], sc & 1, ab)) { ok = false; break; }
        tc_fence_after();
        uint32_t s[128];
        tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        tmem_ld_wait();
        if (valid < kKvTile) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) s[c] = __float_as_uint(-INFINITY);
        }
        // row maximum: 8 independent chains of three-input maxima
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(s[u]);
#pragma unroll
        for (int c = 8; c < 128; c += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmax3(mx8[u], __uint_as_float(s[c + u]), __uint_as_float(s[c + 8 + u]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7])) * sl2;
        const bool need = mx > m_ref + 8.0f;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O_t already holds every PV of this item issued before S_t(j)
          const float alpha = need ? ex2(m_ref - mx) : 1.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(o_addr + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(o_addr + c * 32, r);
          }
          if (need) {
            const uint64_t a2 = f2_pack(alpha, alpha);
            l_acc[0] = f2_fma(l_acc[0], a2, f2_pack(0.f, 0.f));
            l_acc[1] = f2_fma(l_acc[1], a2, f2_pack(0.f, 0.f));
          }
        }
        if (need) m_ref = mx;
        // p = 2^(s * scale * log2(e) - m_ref) in packed pairs; row sums in two
        // packed accumulators; P to TMEM as bf16 pairs
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint64_t negx2 = f2_pack(-m_ref, -m_ref);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[h * 64 + 2 * i]),
                                               __uint_as_float(s[h * 64 + 2 * i + 1])),
                                       sl2x2, negx2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint64_t p2 = f2_pack(ex2(x0), ex2(x1));
            l_acc[i & 1] = f2_add(l_acc[i & 1], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            pk[i] = pack_bf16(p0, p1);
          }
          tmem_st32(s_addr + h * 32, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_full[t]);
      }
      if (!ok) break;
      // epilogue: o_sm = O / l; gated Z or o_sm to global memory
      if (!warp_wait(&bar_o_full[t], it & 1, ab)) break;
      tc_fence_after();
      const bool lin = fused && P.blk[I.seg] >= 0;
      const int b = I.bh / A.H, h = I.bh - b * A.H;
      const int trow = t * kQTile + row;
      const int tok = I.q_start + trow;
      const bool live = trow < I.q_rows;
      float l0, l1, l2, l3;
      f2_unpack(l_acc[0], l0, l1);
      f2_unpack(l_acc[1], l2, l3);
      const float inv_l = 1.0f / ((l0 + l1) + (l2 + l3));
      const float g = fused ? sigmoidf_dev(__ldg(A.gate_logits + h)) : 1.0f;
      __nv_bfloat16* dst_sm;
      __nv_bfloat16* dst_lin = nullptr;
      if (fused) {
        dst_sm = A.out + (((size_t)b * A.L + tok) * 2 * A.H + h) * 128;
        dst_lin = dst_sm + (size_t)A.H * 128;
      } else {
        dst_sm = A.out + (((size_t)b * A.L + tok) * A.H + h) * 128;
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(o_addr + c * 32, r);
        tmem_ld_wait();
        uint4 pk[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
        const float so = inv_l * g;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pw[i] = pack_bf16(__uint_as_float(r[2 * i]) * so, __uint_as_float(r[2 * i + 1]) * so);
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(dst_sm + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = pk[i];
        }
        if (fused) {
          if (lin) {
            tmem_ld32(s_addr + c * 32, r);
            tmem_ld_wait();
            const float sl = 1.0f - g;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pw[i] = pack_bf16(__uint_as_float(r[2 * i]) * sl, __uint_as_float(r[2 * i + 1]) * sl);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pw[i] = 0u;
          }
          if (live) {
            uint4* d4 = reinterpret_cast<uint4*>(dst_lin + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = pk[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_o_empty[t]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vdn
