// softmax_window.cu - block-sparse softmax branch of the VDN hybrid layer on
// sm_100a, with the gate fused in the epilogue.
//
// sd114.wiki, bidirectional sliding-window softmax branch: each query attends
// the key frames of its 3-block window plus the first and last frames (which
// themselves attend every frame). mlsanity abstract: the branches are
// calibrated by learnable gates; this kernel writes g * o_sm, the softmax half
// of Z (the linear half comes from the readout kernel).
//
// One CTA per SM runs a persistent loop over work items; an item is a pair of
// 128-row query tiles (tile 0, tile 1) of one segment and one (b, h), so each
// K/V tile fetched from L2 feeds 256 query rows. Items are taken from a global
// counter (the producer fetches, and hands the index to the other roles
// through a 4-slot ring in shared memory), so the items in flight are always
// consecutive and share their key windows in L2. Warp roles (640 threads):
//   warp 0       TMA producer: Q pair, then K (3-stage ring) and V (2-stage
//                ring) tiles of every key range
//   warp 1       tcgen05 issuer
//   warps 2-3    idle (they complete the first warpgroup)
//   warps 4-11   softmax + epilogue of tile 0     (setmaxnreg 104)
//   warps 12-19  softmax + epilogue of tile 1     (setmaxnreg 104)
// Each 32-lane TMEM quarter of a tile is served by two warps of 16 rows, and
// each row by two threads (.16x32bx2 shape), so that four softmax warps share
// every scheduler and keep its exponential unit busy.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// P_t overwrites the first 64 (bf16: two per column) or 32 (e4m3: four per
// column) columns of S_t.
// MMA issue order per key tile j: PV0(j-1), S0(j), PV1(j-1), S1(j); each PV
// is issued in two halves of 64 keys as the softmax warps release them. MMAs of
// one thread execute in issue order, so S_t(j) overwrites P_t(j-1) only after
// PV_t(j-1) has read it, and every commit of S_t(j) also covers PV_t(j-1):
// when the softmax warps of tile t see S_t(j), O_t is stable and may be
// rescaled. Each tile's softmax thus has two MMAs of the other tile to hide
// behind.
// The online softmax keeps a per-row reference maximum and rescales O only
// when a new row maximum exceeds it by more than 2^8; the final division by
// the row sum uses the same reference.
#include "softmax_window.h"

namespace vdn {

constexpr int kSmThreads = 640;
constexpr uint32_t kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one TMA box)
constexpr uint32_t kColS = 0, kColO = 256;    // S_t at t*128, O_t at 256 + t*128
constexpr int kRegsSoftmax = 112, kRegsOther = 32;  // 112*512 + 32*128 <= 96*640
// Work-item ring: the producer publishes item indices, read by the MMA
// warp (1 arrival) and the softmax warps (16).
constexpr int kItemSlots = 4;
constexpr int kItemConsumers = 17;
// Registers per thread at launch: 65536 / 640 rounded down to a multiple of 8.
constexpr int kRegsLaunch = 96;
static_assert(kRegsSoftmax * 512 + kRegsOther * 128 <= kRegsLaunch * kSmThreads, "register split");

struct Item {
  int bh, seg, q_start, q_rows, nkv;
};

// Work items run head by head, then segment by segment (heaviest segments
// first; segments of equal weight in frame order), then pair by pair. The
// CTAs in flight at any time work on one or two heads and, within a head, on
// neighbouring segments, whose key windows overlap by all but one block: the
// head's keys and values are fetched from DRAM about once and then served
// from L2. (Segment-major order streamed every (segment, head) window from
// DRAM separately: 3.3x the algorithmic traffic at 768p.)
__device__ __forceinline__ Item decode_item(const SoftmaxPlan& P, int BH, int w) {
  Item it;
  it.bh = w / P.total_tiles;
  const int e = w - it.bh * P.total_tiles;
  int s = 0;
  while (s + 1 < P.n_seg && P.tile_begin[s + 1] <= e) ++s;
  const int pair = e - P.tile_begin[s];
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

// Per input type: bytes of one 128 x 128 tile, the TMA boxes per tile (64
// bf16 or 128 e4m3 columns each), the MMA k-steps per 128-wide product, the
// instruction kind and the shared-memory byte stride of one k-step of V.
template <bool F8>
struct Elem {
  static constexpr uint32_t kTile = F8 ? 128 * 128 : 128 * 128 * 2;
  static constexpr int kBoxes = F8 ? 1 : 2;
  static constexpr int kKSteps = F8 ? 4 : 8;      // 32 e4m3 or 16 bf16 per step
  static constexpr uint32_t kVStep = F8 ? 4096 : 2048;
  static constexpr uint32_t kPCols = F8 ? 32 : 64;  // TMEM columns of P (4 or 2 per column)
};

// S_t = Q_t K^T (8 bf16 k-steps in two 64-wide chunks, or 4 e4m3 k-steps).
template <bool F8>
__device__ __forceinline__ void mma_qk(uint32_t ld, uint32_t d, uint64_t qd, uint64_t kd,
                                       uint32_t idesc) {
  if constexpr (F8) {
    umma_ss4_f8_w<0, 2, 4, 6, 0, 2, 4, 6>(ld, d, qd, kd, idesc, 0);
  } else {
    constexpr int C = kChunkBytes >> 4;
    umma_ss4_w<0, 2, 4, 6, 0, 2, 4, 6>(ld, d, qd, kd, idesc, 0);
    umma_ss4_w<C, C + 2, C + 4, C + 6, C, C + 2, C + 4, C + 6>(ld, d, qd, kd, idesc, 1);
  }
}
// Half hf of O_t += P_t V: keys [64 hf, 64 hf + 64), P from TMEM.
template <bool F8>
__device__ __forceinline__ void mma_pv_half(uint32_t ld, uint32_t d_o, uint32_t p_tmem,
                                            uint64_t vd, int hf, uint32_t idesc,
                                            uint32_t accumulate) {
  constexpr uint32_t kStep = Elem<F8>::kVStep >> 4;
  constexpr int kHalfSteps = Elem<F8>::kKSteps / 2;
  if constexpr (F8)
    umma_ts2_f8_w<kStep>(ld, d_o, p_tmem + hf * kHalfSteps * 8, vd + hf * kHalfSteps * kStep, idesc,
                         accumulate);
  else
    umma_ts4_w<kStep>(ld, d_o, p_tmem + hf * kHalfSteps * 8, vd + hf * kHalfSteps * kStep, idesc,
                      accumulate);
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

template <bool F8>
__device__ __forceinline__ void softmax_window_body(const CUtensorMap& tm_q,
                                                    const CUtensorMap& tm_k,
                                                    const CUtensorMap& tm_v,
                                                    const SoftmaxArgs& A) {
  using E = Elem<F8>;
  constexpr uint32_t kTileBytes = E::kTile;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q_full, bar_q_empty;
  __shared__ __align__(8) uint64_t bar_k_full[kKStages], bar_k_empty[kKStages],
      bar_v_full[kVStages], bar_v_empty[kVStages];
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_p_full[2][2], bar_o_full[2], bar_o_empty[2];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ __align__(8) uint64_t bar_item_full[kItemSlots], bar_item_empty[kItemSlots];
  __shared__ int item_slot[kItemSlots];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = base;                       // tile 0, tile 1
  uint8_t* sK = base + 2 * kTileBytes;
  uint8_t* sV = base + (2 + kKStages) * kTileBytes;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const SoftmaxPlan& P = A.plan;
  const bool gated = A.gate_logits != nullptr;
  const int n_items = P.total_tiles * A.BH;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_p_full[t][0], 8);
      mbar_init(&bar_p_full[t][1], 8);
      mbar_init(&bar_o_full[t], 1);
      mbar_init(&bar_o_empty[t], 8);
    }
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
      const uint64_t q_policy = l2_policy_evict_first();
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
        // q is read once: evict it from L2 first, ahead of the shared keys
        for (int t = 0; t < 2; ++t)
          for (int x = 0; x < E::kBoxes; ++x)
            tma_load_3d_hint(sQ + t * kTileBytes + x * kChunkBytes, &tm_q, &bar_q_full, x * 64,
                             I.q_start + t * kQTile, I.bh, q_policy);
        KvWalk kw;
        kw.init(P, I.seg);
        for (int j = 0; j < I.nkv; ++j) {
          const int ks = kvc % kKStages, vs = kvc % kVStages;
          const uint32_t kuse = kvc / kKStages, vuse = kvc / kVStages;
          uint8_t* k_dst = sK + ks * kTileBytes;
          uint8_t* v_dst = sV + vs * kTileBytes;
          if (kuse > 0 && !mbar_wait(&bar_k_empty[ks], (kuse - 1) & 1, ab)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar_k_full[ks], kTileBytes);
          for (int x = 0; x < E::kBoxes; ++x)
            tma_load_3d(k_dst + x * kChunkBytes, &tm_k, &bar_k_full[ks], x * 64, kw.pos, I.bh);
          if (vuse > 0 && !mbar_wait(&bar_v_empty[vs], (vuse - 1) & 1, ab)) {
            // the K copy of this tile is in flight: drain it below
            mbar_wait_drain(&bar_k_full[ks], kuse & 1);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[vs], kTileBytes);
          for (int x = 0; x < E::kBoxes; ++x)
            tma_load_3d(v_dst + x * kChunkBytes, &tm_v, &bar_v_full[vs], x * 64, kw.pos, I.bh);
          kw.next(P, I.seg);
          ++kvc;
        }
      }
      if (!ok) {
        // let every issued copy land before shared memory is released
        if (q_issued > 0) mbar_wait_drain(&bar_q_full, (q_issued - 1) & 1);
        for (uint32_t c = (kvc > kKStages ? kvc - kKStages : 0); c < kvc; ++c)
          mbar_wait_drain(&bar_k_full[c % kKStages], (c / kKStages) & 1);
        for (uint32_t c = (kvc > kVStages ? kvc - kVStages : 0); c < kvc; ++c)
          mbar_wait_drain(&bar_v_full[c % kVStages], (c / kVStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    // The whole warp runs this role with warp-uniform values (descriptors,
    // counters, waits); lane 0 alone issues the MMAs and their commits.
    setmaxnreg_dec();
    const uint32_t ld = lane == 0 ? 1u : 0u;
    const uint32_t idesc_qk = F8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t idesc_pv = F8 ? idesc_e4m3_f32(128, 128, 0, 1) : idesc_bf16_f32(128, 128, 0, 1);
    // Shared-memory descriptors at k-step 0; a k step or a tile moves only the
    // start-address field (address >> 4, shared memory < 256 KB: no carry).
    const uint64_t dQ = kmajor_desc(sQ, 0), dK = kmajor_desc(sK, 0), dV = mnmajor_desc(sV, 0);
    constexpr uint32_t kTileStep = kTileBytes >> 4;
    uint32_t kvc = 0, sc = 0;  // key tiles, S MMAs per query tile
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int w;
      if (!warp_next_item(bar_item_full, bar_item_empty, item_slot, it, lane == 0, ab, &w)) break;
      if (w < 0) break;
      const Item I = decode_item(P, A.BH, w);
      if (!warp_wait(&bar_q_full, it & 1, ab)) break;
      // key tile j = 0: S_t(0). The epilogue of the previous item must have
      // read O_t first.
      {
        const int ks0 = kvc % kKStages;
        if (!warp_wait(&bar_k_full[ks0], (kvc / kKStages) & 1, ab)) break;
        for (int t = 0; t < 2; ++t) {
          if (it > 0 && !warp_wait(&bar_o_empty[t], (it - 1) & 1, ab)) { ok = false; break; }
          tc_fence_after();
          mma_qk<F8>(ld, tmem + kColS + t * 128, dQ + t * kTileStep, dK + ks0 * kTileStep,
                     idesc_qk);
          umma_commit_w(ld, &bar_s_full[t]);
        }
        if (!ok) break;
        umma_commit_w(ld, &bar_k_empty[ks0]);
      }
      // key tiles j = 1 .. nkv: PV_t(j-1) then S_t(j) (nothing after the last)
      for (int j = 1; j <= I.nkv && ok; ++j) {
        const int vs = kvc % kVStages;              // V stage of key tile j-1
        const uint32_t vuse = kvc / kVStages;
        const int kst = (kvc + 1) % kKStages;       // K stage of key tile j
        const uint32_t kuse = (kvc + 1) / kKStages;
        const bool last = (j == I.nkv);
        if (!warp_wait(&bar_v_full[vs], vuse & 1, ab)) { ok = false; break; }
        if (!last && !warp_wait(&bar_k_full[kst], kuse & 1, ab)) { ok = false; break; }
        const uint64_t vd = dV + vs * kTileStep, kd = dK + kst * kTileStep;
        for (int t = 0; t < 2; ++t) {
          // P_t arrives in two halves of 64 keys
          for (int hf = 0; hf < 2 && ok; ++hf) {
            if (!warp_wait(&bar_p_full[t][hf], sc & 1, ab)) { ok = false; break; }
            tc_fence_after();
            mma_pv_half<F8>(ld, tmem + kColO + t * 128, tmem + kColS + t * 128, vd, hf, idesc_pv,
                            (j > 1 || hf > 0) ? 1u : 0u);
          }
          if (!ok) break;
          if (!last) {
            mma_qk<F8>(ld, tmem + kColS + t * 128, dQ + t * kTileStep, kd, idesc_qk);
            umma_commit_w(ld, &bar_s_full[t]);
          } else {
            umma_commit_w(ld, &bar_o_full[t]);
          }
        }
        if (!ok) break;
        umma_commit_w(ld, &bar_v_empty[vs]);
        if (!last) umma_commit_w(ld, &bar_k_empty[kst]);
        ++sc;
        ++kvc;
      }
      if (!ok) break;
      umma_commit_w(ld, &bar_q_empty);
    }
    // every MMA issued by lane 0 completes before TMEM is released
    umma_commit_w(ld, &bar_drain);
    if (lane == 0) mbar_wait_drain(&bar_drain, 0);
    __syncwarp();
  } else if (warp < 4) {
    // warps 2-3 complete the first warpgroup (register reallocation is per
    // warpgroup) and have no work
    setmaxnreg_dec();
  } else {
    // ------------------------------------------------ softmax + epilogue
    // Two warps per TMEM lane quarter and tile: warp half hs takes the 16
    // rows 32*wq + 16*hs + [0, 16); within the warp, lanes l and l + 16 share
    // row l (.16x32bx2 shape), each taking half of every 64-key group of S
    // and half of the columns of O.
    setmaxnreg_inc();
    const int v = warp - 4;
    const int t = v >> 3;                   // query tile of this warp
    const int hs = (v >> 2) & 1;            // 16-row half of the lane quarter
    const int wq = warp & 3;                // TMEM lane quarter (warp % 4)
    const int ch = lane >> 4;               // key half of the row in this thread
    const int row = wq * 32 + hs * 16 + (lane & 15);  // query row within the tile
    const uint32_t lane_addr = uint32_t(wq * 32 + hs * 16) << 16;
    const uint32_t s_addr = tmem + lane_addr + kColS + t * 128;
    const uint32_t o_addr = tmem + lane_addr + kColO + t * 128;
    uint32_t sc = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int w;
      if (!warp_next_item(bar_item_full, bar_item_empty, item_slot, it, lane == 0, ab, &w)) break;
      if (w < 0) break;
      const Item I = decode_item(P, A.BH, w);
      KvWalk kw;
      kw.init(P, I.seg);
      // scores to log2 units; e4m3 inputs carry their (b, h) scales
      const float sl2 = F8 ? A.scale_log2 * __ldg(A.q_scale + I.bh) * __ldg(A.k_scale + I.bh)
                           : A.scale_log2;
      float m_ref = -INFINITY;   // reference maximum (log2 units) of the exponentials
      uint64_t l_acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};  // packed partial row sums
      for (int j = 0; j < I.nkv; ++j, ++sc) {
        const int valid = kw.valid(P, I.seg);
        kw.next(P, I.seg);
        if (!warp_wait(&bar_s_full[t], sc & 1, ab)) { ok = false; break; }
        tc_fence_after();
        // first pass: the row maximum over all 128 keys. This thread holds
        // keys ch*32 + [0, 32) and 64 + ch*32 + [0, 32).
        float mxh;
        uint32_t s[64];
        {
          tmem_ld16x2_32<32>(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
          tmem_ld16x2_32<32>(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
          tmem_ld_wait();
          if (valid < kKvTile) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if ((c >> 5) * 64 + ch * 32 + (c & 31) >= valid) s[c] = __float_as_uint(-INFINITY);
          }
          float mx8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(s[u]);
#pragma unroll
          for (int c = 8; c < 56; c += 16)
#pragma unroll
            for (int u = 0; u < 8; ++u)
              mx8[u] = fmax3(mx8[u], __uint_as_float(s[c + u]), __uint_as_float(s[c + 8 + u]));
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(mx8[u], __uint_as_float(s[56 + u]));
          mxh = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                      fmaxf(mx8[6], mx8[7]));
        }
        mxh = fmaxf(mxh, __shfl_xor_sync(0xffffffffu, mxh, 16));
        const float mx = mxh * sl2;
        const bool need = mx > m_ref + 8.0f;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O_t already holds every PV of this item issued before S_t(j);
          // this thread rescales its 64 columns of the row
          const float alpha = need ? ex2(m_ref - mx) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld16x2_32<64>(o_addr + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16x2_32<64>(o_addr + c * 32, r);
          }
          if (need) {
            const uint64_t a2 = f2_pack(alpha, alpha);
            l_acc[0] = f2_fma(l_acc[0], a2, f2_pack(0.f, 0.f));
            l_acc[1] = f2_fma(l_acc[1], a2, f2_pack(0.f, 0.f));
          }
        }
        if (need) m_ref = mx;
        // second pass, in two halves h of 64 keys, on the scores the first
        // pass left in registers: this thread takes keys h*64 + ch*32 +
        // [0, 32), p = 2^(s * scale * log2(e) - m_ref) in packed
        // pairs, row sums in two packed accumulators, and P as bf16 pairs into
        // TMEM columns h*32 + ch*16 + [0, 16) of S_t (key order; columns whose
        // scores were read in this or the previous half), handed to the MMA
        // warp as soon as the half is stored.
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint64_t negx2 = f2_pack(-m_ref, -m_ref);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // the scores of this half are still in registers from the first
          // pass (masked there)
          const uint32_t* q = &s[h * 32];
          // bf16: two P values per TMEM column; e4m3: four
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(q[2 * i]),
                                               __uint_as_float(q[2 * i + 1])),
                                       sl2x2, negx2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint64_t p2 = f2_pack(ex2(x0), ex2(x1));
            l_acc[i & 1] = f2_add(l_acc[i & 1], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            if constexpr (F8) {
              const uint32_t b2 = pack_e4m3x2(p0, p1);
              pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (b2 << 16)) : b2;
            } else {
              pk[i] = pack_bf16(p0, p1);
            }
          }
          if constexpr (F8)
            tmem_st16x2_8<8>(s_addr + h * 16, *reinterpret_cast<const uint32_t(*)[8]>(&pk[0]));
          else
            tmem_st16x2_16<16>(s_addr + h * 32, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_p_full[t][h]);
        }
      }
      if (!ok) break;
      // epilogue: o_sm = O / l; gated Z or o_sm to global memory
      if (!warp_wait(&bar_o_full[t], it & 1, ab)) break;
      tc_fence_after();
      const int b = I.bh / A.H, h = I.bh - b * A.H;
      const int trow = t * kQTile + row;
      const int tok = I.q_start + trow;
      const bool live = trow < I.q_rows;
      float l0, l1, l2, l3;
      f2_unpack(l_acc[0], l0, l1);
      f2_unpack(l_acc[1], l2, l3);
      float lh = (l0 + l1) + (l2 + l3);
      lh += __shfl_xor_sync(0xffffffffu, lh, 16);
      // log2-domain log-sum-exp of the row's scaled scores, for the backward:
      // p = 2^(s * sl2 - lse2) recovers the softmax weights exactly
      if (A.lse != nullptr && live && ch == 0)
        A.lse[(size_t)I.bh * A.L + tok] = m_ref + log2f(lh);
      const float g = gated ? sigmoidf_dev(__ldg(A.gate_logits + h)) : 1.0f;
      const float so = (F8 ? g * __ldg(A.v_scale + I.bh) : g) / lh;
      // o_sm [B, L, H, dv], or the softmax half of Z [B, L, 2, H, dv]
      __nv_bfloat16* dst = A.out + ((size_t)b * A.L + tok) * (gated ? 2 : 1) * A.H * 128 +
                           h * 128 + ch * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld16x2_32<64>(o_addr + c * 32, r);
        tmem_ld_wait();
        uint4 pk[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pw[i] = pack_bf16(__uint_as_float(r[2 * i]) * so, __uint_as_float(r[2 * i + 1]) * so);
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = pk[i];
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

__global__ void __launch_bounds__(kSmThreads, 1)
    softmax_window_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ SoftmaxArgs A) {
  softmax_window_body<false>(tm_q, tm_k, tm_v, A);
}

// e4m3 q, k, v with per-(b, h) scales: kind::f8f6f4 products, P stored to
// TMEM as e4m3 (four per column); the scales enter the exponent and the
// epilogue.
__global__ void __launch_bounds__(kSmThreads, 1)
    softmax_window_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ SoftmaxArgs A) {
  softmax_window_body<true>(tm_q, tm_k, tm_v, A);
}

}  // namespace vdn
