// softmax_bwd.cu - backward of the block-sparse softmax branch on sm_100a.
//
// With P = softmax(scale q k^T) over the allowed keys and o = P v, the
// cotangent do of o gives, tile by tile with the forward's row statistics:
//   P_ij  = 2^(s_ij * scale * log2(e) - lse2_i)   (lse2: the forward's log2-domain
//                                                   log-sum-exp of row i)
//   dP_ij = do_i . v_j,   D_i = sum_j P_ij dP_ij = do_i . o_i
//   dS_ij = P_ij (dP_ij - D_i)
//   dv_j = sum_i P_ij do_i,  dk_j = scale sum_i dS_ij q_i,  dq_i = scale sum_j dS_ij k_j.
// The window mask is symmetric (sd114.wiki, sliding-window softmax branch:
// frame i sees frame j exactly when j sees i, anchors included; context
// tokens see and are seen by every token), so the forward's segments serve
// both directions: the key ranges of a segment are also, for the key tiles of
// that segment, the ranges of the queries that see them.
//
// softmax_bwd_dkdv_kernel: one CTA per 128-key tile of a segment and (b, h).
//   K and V of the tile stay in shared memory; the query tiles of the ranges
//   stream in 128-row tiles (q and do) through a 2-stage TMA ring. Per tile:
//     S^T = K q^T, dP^T = V do^T      two SS MMAs, M = N = 128 (keys on TMEM lanes)
//     P^T, dS^T                       16 elementwise warps, bf16 into TMEM
//     dV += P^T do, dK += dS^T q      two TS MMAs (A from TMEM, K = 128)
// softmax_bwd_dq_kernel: one CTA per 128-query tile: q and do stay, the K and
//   V tiles of the ranges stream; S = q K^T, dP = do V^T, dS, dQ += dS K.
// TMEM (512 columns): the scores S (or S^T) in [0, 128), dP in [128, 256),
// the accumulators at 256 (dV or dQ) and 384 (dK; in dq a second dP buffer,
// used by odd tiles, so that both score products of the next tile follow as
// soon as the current one is loaded). Every product is 128 wide:
// the elementwise warps read S and dP of tile j into registers and signal it,
// the MMA thread then computes S of tile j + 1 into [0, 128) while they work;
// their bf16 P and dS (dq: dS only) go into [128, 256), which they fill
// exactly (64 columns each), the TS products of tile j read them from there,
// and dP of tile j + 1 follows those products into the same columns.
// Warp roles (640 threads): warp 0 TMA, warp 1 MMA issue (lane 0), warps 2-3
// (dkdv) stage each inner tile's 128 (lse, D) pairs in a shared-memory ring
// beside the TMA ring, warps 4-19 elementwise + epilogue: four warps per TMEM
// lane quarter, each thread taking 32 of a row's 128 columns.
#include "kernels.h"

namespace vdn {

constexpr uint32_t kBwdTile = 128 * 128 * 2;   // a 128 x 128 bf16 tile
constexpr uint32_t kBwdChunk = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
constexpr int kInRows = 128;                   // rows of an inner tile
constexpr uint32_t kColD = 128, kColAcc0 = 256, kColAcc1 = 384;
constexpr uint32_t kColD2 = 384;   // dq: the second dP buffer (dkdv keeps dK there)
constexpr int kRegsEw = 104, kRegsCtl = 56;    // 104*512 + 56*128 <= 96*640
static_assert(kSoftmaxBwdSmem >= 1024 + 2 * kBwdTile + kBwdStages * 2 * kBwdTile +
                                     kBwdStages * kInRows * sizeof(float2),
              "smem size");
static_assert(kRegsEw * 512 + kRegsCtl * 128 <= 96 * kSoftmaxBwdThreads, "register split");

struct BwdItem {
  int bh, seg, start, rows;
};

// Items run segment by segment, then head by head, then tile by tile, so the
// CTAs in flight share one head's ranges in L2.
__device__ __forceinline__ BwdItem decode_bwd_item(const SoftmaxPlan& P, int BH, int w) {
  BwdItem it;
  int s = 0;
  while (s + 1 < P.n_seg && P.tile_begin[s + 1] * BH <= w) ++s;
  const int nt = (s + 1 < P.n_seg ? P.tile_begin[s + 1] : P.total_tiles) - P.tile_begin[s];
  const int e = w - P.tile_begin[s] * BH;
  it.bh = e / nt;
  const int tile = e - it.bh * nt;
  it.seg = s;
  it.start = P.q0[s] + tile * kQTile;
  const int rem = P.q1[s] - it.start;
  it.rows = rem < kQTile ? rem : kQTile;
  return it;
}

__device__ __forceinline__ int range_tiles(const SoftmaxPlan& P, int s) {
  int n = 0;
  for (int r = 0; r < P.nr[s]; ++r) n += (P.k1[s][r] - P.k0[s][r] + kInRows - 1) / kInRows;
  return n;
}

// Walks the 128-token tiles of a segment's ranges: start token, valid rows.
struct RangeWalk {
  int r, pos;
  __device__ __forceinline__ void init(const SoftmaxPlan& P, int s) {
    r = 0;
    pos = P.k0[s][0];
  }
  __device__ __forceinline__ int valid(const SoftmaxPlan& P, int s) const {
    const int rem = P.k1[s][r] - pos;
    return rem < kInRows ? rem : kInRows;
  }
  __device__ __forceinline__ void next(const SoftmaxPlan& P, int s) {
    pos += kInRows;
    if (pos >= P.k1[s][r]) {
      ++r;
      if (r < P.nr[s]) pos = P.k0[s][r];
    }
  }
};

__device__ __forceinline__ uint64_t bwd_kdesc(const uint8_t* tile) {
  return sdesc_sw128(smem_u32(tile), 16, 1024);
}
// MN-major 128 x 128 tile: 128 k-rows, N = 128 in two 64-wide chunks
__device__ __forceinline__ uint64_t bwd_mndesc(const uint8_t* tile) {
  return sdesc_sw128(smem_u32(tile), kBwdChunk, 1024);
}

// D [128 x 128] = A B^T with K = 128 (8 k-steps in two 64-wide chunks), A and
// B K-major 128-row tiles.
__device__ __forceinline__ void mma_nt(uint32_t ld, uint32_t d, uint64_t ad, uint64_t bd,
                                       uint32_t idesc) {
  constexpr int C = kBwdChunk >> 4;
  umma_ss4_w<0, 2, 4, 6, 0, 2, 4, 6>(ld, d, ad, bd, idesc, 0);
  umma_ss4_w<C, C + 2, C + 4, C + 6, C, C + 2, C + 4, C + 6>(ld, d, ad, bd, idesc, 1);
}
// D [128 x 128] (+)= A B with A the bf16 pairs in TMEM columns [a, a + 64)
// (K = 128) and B an MN-major 128 x 128 tile.
__device__ __forceinline__ void mma_tn(uint32_t ld, uint32_t d, uint32_t a_tmem, uint64_t bd,
                                       uint32_t idesc, uint32_t accumulate) {
  constexpr uint32_t kStep = 2048 >> 4;  // one k-step: 16 rows of 128 bytes
  umma_ts4_w<kStep>(ld, d, a_tmem, bd, idesc, accumulate);
  umma_ts4_w<kStep>(ld, d, a_tmem + 32, bd + 4 * kStep, idesc, 1);
}

// Adds `sc` times 32 fp32 accumulator columns to 32 bf16 outputs at dst
// (optionally on top of the bf16 values already there).
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&r)[32], float sc,
                                            bool accumulate) {
  uint4 pk[4];
  uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
  if (accumulate) {
    const uint4* s4 = reinterpret_cast<const uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) pk[i] = s4[i];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[i]));
      pw[i] = pack_bf16(o.x + __uint_as_float(r[2 * i]) * sc,
                        o.y + __uint_as_float(r[2 * i + 1]) * sc);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pw[i] = pack_bf16(__uint_as_float(r[2 * i]) * sc, __uint_as_float(r[2 * i + 1]) * sc);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = pk[i];
}

// The two kernels share everything but the operand roles; DQ selects the
// query-outer form. Maps: the two outer and the two inner tensors, all with
// 128-row boxes.
template <bool DQ>
__device__ __forceinline__ void softmax_bwd_body(const CUtensorMap& tm_o0, const CUtensorMap& tm_o1,
                                                 const CUtensorMap& tm_i0, const CUtensorMap& tm_i1,
                                                 const SoftmaxBwdArgs& A) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_outer, bar_in_full[kBwdStages], bar_in_empty[kBwdStages];
  __shared__ __align__(8) uint64_t bar_s_full, bar_s_loaded, bar_p_full, bar_acc_full, bar_drain;
  __shared__ __align__(8) uint64_t bar_stat_full[kBwdStages], bar_stat_empty[kBwdStages];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // outer tiles: dkdv K and V, dq q and do; stage st holds the inner pair at
  // sX + st * 2 tiles: dkdv (q, do), dq (K, V)
  uint8_t* sA = base;
  uint8_t* sB = base + kBwdTile;
  uint8_t* sX = base + 2 * kBwdTile;
  // dkdv: (lse, D) of the 128 query rows of inner tile j at stage j % kBwdStages
  float2* sStat = reinterpret_cast<float2*>(sX + kBwdStages * 2 * kBwdTile);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SoftmaxPlan& P = A.plan;
  const BwdItem I = decode_bwd_item(P, A.BH, blockIdx.x);
  const int n_in = range_tiles(P, I.seg);

  if (threadIdx.x == 0) {
    mbar_init(&bar_outer, 1);
    for (int i = 0; i < kBwdStages; ++i) {
      mbar_init(&bar_in_full[i], 1);
      mbar_init(&bar_in_empty[i], 1);
      mbar_init(&bar_stat_full[i], 64);   // the 64 threads of warps 2-3
      mbar_init(&bar_stat_empty[i], 16);  // the 16 elementwise warps
    }
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_s_loaded, 16);
    mbar_init(&bar_p_full, 16);
    mbar_init(&bar_acc_full, 1);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_o0);
    tma_prefetch_desc(&tm_o1);
    tma_prefetch_desc(&tm_i0);
    tma_prefetch_desc(&tm_i1);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const Abort ab{&abort_sh, A.dev_status};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_outer, 2 * kBwdTile);
      for (int x = 0; x < 2; ++x) {
        tma_load_3d(sA + x * kBwdChunk, &tm_o0, &bar_outer, x * 64, I.start, I.bh);
        tma_load_3d(sB + x * kBwdChunk, &tm_o1, &bar_outer, x * 64, I.start, I.bh);
      }
      RangeWalk rw;
      rw.init(P, I.seg);
      int i = 0;
      for (; i < n_in; ++i) {
        const int st = i % kBwdStages;
        const int use = i / kBwdStages;
        if (use > 0 && !mbar_wait(&bar_in_empty[st], (use - 1) & 1, ab)) break;
        uint8_t* dst = sX + st * 2 * kBwdTile;
        mbar_arrive_expect_tx(&bar_in_full[st], 2 * kBwdTile);
        for (int x = 0; x < 2; ++x) {
          tma_load_3d(dst + x * kBwdChunk, &tm_i0, &bar_in_full[st], x * 64, rw.pos, I.bh);
          tma_load_3d(dst + kBwdTile + x * kBwdChunk, &tm_i1, &bar_in_full[st], x * 64, rw.pos,
                      I.bh);
        }
        rw.next(P, I.seg);
      }
      if (i < n_in) {
        // aborted: let every issued copy land before shared memory is released
        mbar_wait_drain(&bar_outer, 0);
        for (int c = (i > kBwdStages ? i - kBwdStages : 0); c < i; ++c)
          mbar_wait_drain(&bar_in_full[c % kBwdStages], (c / kBwdStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    const uint32_t ld = lane == 0 ? 1u : 0u;
    const uint32_t idesc_ss = idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t idesc_ts = idesc_bf16_f32(128, 128, 0, 1);
    const uint64_t dA = bwd_kdesc(sA), dB = bwd_kdesc(sB), dX = bwd_kdesc(sX);
    const uint64_t dXm = bwd_mndesc(sX);
    constexpr uint32_t kTile = kBwdTile >> 4;
    bool ok = warp_wait(&bar_outer, 0, ab);
    // tile 0: both score products
    if (ok && n_in > 0) {
      ok = warp_wait(&bar_in_full[0], 0, ab);
      if (ok) {
        tc_fence_after();
        mma_nt(ld, tmem, dA, dX, idesc_ss);
        mma_nt(ld, tmem + kColD, dB, dX + kTile, idesc_ss);
        umma_commit_w(ld, &bar_s_full);
      }
    }
    if constexpr (DQ) {
      // dq: dP alternates between [128, 256) and [384, 512), so both score
      // products of tile j + 1 follow as soon as the elementwise warps hold
      // tile j; only dQ += dS K waits for their dS
      for (int j = 0; j < n_in && ok; ++j) {
        const int st = j % kBwdStages, st1 = (j + 1) % kBwdStages;
        const uint32_t xo = st * 2 * kTile, xo1 = st1 * 2 * kTile;
        if (j + 1 < n_in) {
          if (!warp_wait(&bar_s_loaded, j & 1, ab)) { ok = false; break; }
          if (!warp_wait(&bar_in_full[st1], ((j + 1) / kBwdStages) & 1, ab)) { ok = false; break; }
          tc_fence_after();
          mma_nt(ld, tmem, dA, dX + xo1, idesc_ss);
          mma_nt(ld, tmem + ((j + 1) & 1 ? kColD2 : kColD), dB, dX + xo1 + kTile, idesc_ss);
          umma_commit_w(ld, &bar_s_full);
        }
        if (!warp_wait(&bar_p_full, j & 1, ab)) { ok = false; break; }
        tc_fence_after();
        mma_tn(ld, tmem + kColAcc0, tmem + (j & 1 ? kColD2 : kColD), dXm + xo, idesc_ts,
               j > 0 ? 1u : 0u);
        umma_commit_w(ld, &bar_in_empty[st]);
      }
    }
    for (int j = 0; j < n_in && ok && !DQ; ++j) {
      const int st = j % kBwdStages, st1 = (j + 1) % kBwdStages;
      const uint32_t xo = st * 2 * kTile, xo1 = st1 * 2 * kTile;
      const bool more = j + 1 < n_in;
      if (more) {
        // S of tile j + 1 into [0, 128) once the elementwise warps hold S(j)
        if (!warp_wait(&bar_s_loaded, j & 1, ab)) { ok = false; break; }
        if (!warp_wait(&bar_in_full[st1], ((j + 1) / kBwdStages) & 1, ab)) { ok = false; break; }
        tc_fence_after();
        mma_nt(ld, tmem, dA, dX + xo1, idesc_ss);
      }
      if (!warp_wait(&bar_p_full, j & 1, ab)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = j > 0 ? 1u : 0u;
      // dV += P^T do, dK += dS^T q
      mma_tn(ld, tmem + kColAcc0, tmem + kColD, dXm + xo + kTile, idesc_ts, acc);
      mma_tn(ld, tmem + kColAcc1, tmem + kColD + 64, dXm + xo, idesc_ts, acc);
      umma_commit_w(ld, &bar_in_empty[st]);
      if (more) {
        // dP of tile j + 1 into [128, 256), after the products that read P, dS
        mma_nt(ld, tmem + kColD, dB, dX + xo1 + kTile, idesc_ss);
        umma_commit_w(ld, &bar_s_full);
      }
    }
    if (ok) umma_commit_w(ld, &bar_acc_full);
    // every MMA issued by lane 0 completes before TMEM is released
    umma_commit_w(ld, &bar_drain);
    if (lane == 0) mbar_wait_drain(&bar_drain, 0);
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------- (lse, D) staging (dkdv)
    // Thread i of warps 2-3 copies the pairs of query rows pos + i and
    // pos + 64 + i of every inner tile into the tile's stage (rows past the
    // tile's end: zeros).
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
    if constexpr (!DQ) {
      const int i = threadIdx.x - 64;
      const float2* rs = A.rowstat + (size_t)I.bh * A.L;
      RangeWalk rw;
      rw.init(P, I.seg);
      for (int j = 0; j < n_in; ++j) {
        const int st = j % kBwdStages;
        const int use = j / kBwdStages;
        const int pos = rw.pos, valid = rw.valid(P, I.seg);
        rw.next(P, I.seg);
        const float2 v0 = i < valid ? __ldg(rs + pos + i) : make_float2(0.f, 0.f);
        const float2 v1 = i + 64 < valid ? __ldg(rs + pos + 64 + i) : make_float2(0.f, 0.f);
        if (use > 0 && !mbar_wait(&bar_stat_empty[st], (use - 1) & 1, ab)) break;
        sStat[st * kInRows + i] = v0;
        sStat[st * kInRows + 64 + i] = v1;
        mbar_arrive(&bar_stat_full[st]);
      }
    }
  } else {
    // ------------------------------------------- elementwise + epilogue
    // 16 warps: TMEM lane quarter wq = warp % 4 (one row per thread), column
    // quarter cq = (warp - 4) / 4 (32 of the tile's 128 columns).
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEw));
    const int wq = warp & 3;
    const int cq = (warp - 4) >> 2;
    const int row = wq * 32 + lane;      // row of the outer tile
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const float2* rs = A.rowstat + (size_t)I.bh * A.L;
    const bool live = row < I.rows;
    // dq: the row's own statistics (dead rows contribute nothing)
    float2 own = make_float2(0.f, 0.f);
    if (DQ && live) own = __ldg(rs + I.start + row);
    RangeWalk rw;
    rw.init(P, I.seg);
    bool ok = true;
    const uint32_t s_addr = tmem + lane_addr;
    for (int j = 0; j < n_in; ++j) {
      // dq: dP (and then dS) of tile j in [128, 256) or [384, 512)
      const uint32_t d_addr = tmem + lane_addr + (DQ && (j & 1) ? kColD2 : kColD);
      const int valid = rw.valid(P, I.seg);
      rw.next(P, I.seg);
      const int st = j % kBwdStages;
      if (!warp_wait(&bar_s_full, j & 1, ab)) { ok = false; break; }
      if (!DQ && !warp_wait(&bar_stat_full[st], (j / kBwdStages) & 1, ab)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[32], dp[32];
      tmem_ld32(s_addr + cq * 32, sv);
      tmem_ld32(d_addr + cq * 32, dp);
      tmem_ld_wait();
      // S(j) and dP(j) are in registers: the scores' columns may take S(j + 1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_s_loaded);
      const float4* stat4 = reinterpret_cast<const float4*>(sStat + st * kInRows + cq * 32);
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int u = 0; u < 32; u += 2) {
        float pv[2], dv[2];
        // dkdv: the (lse, D) pairs of columns u and u + 1, one 16-byte
        // shared-memory load read by every lane of the warp
        float4 st2 = make_float4(0.f, 0.f, 0.f, 0.f);
        if constexpr (!DQ) st2 = stat4[u >> 1];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = cq * 32 + u + e;   // column: inner token pos + c
          float p = 0.f, ds = 0.f;
          const bool on = DQ ? (live && c < valid) : (c < valid);
          if (on) {
            const float2 stat = DQ ? own : (e ? make_float2(st2.z, st2.w)
                                              : make_float2(st2.x, st2.y));
            p = ex2(fmaf(__uint_as_float(sv[u + e]), A.scale_log2, -stat.x));
            ds = p * (__uint_as_float(dp[u + e]) - stat.y);
          }
          pv[e] = p;
          dv[e] = ds;
        }
        pp[u / 2] = pack_bf16(pv[0], pv[1]);
        pd[u / 2] = pack_bf16(dv[0], dv[1]);
      }
      if (!DQ && lane == 0) mbar_arrive(&bar_stat_empty[st]);
      // P and dS overwrite dP's columns, which the other warps of this lane
      // quarter read: wait until every warp holds its dP(j)
      if (!warp_wait(&bar_s_loaded, j & 1, ab)) { ok = false; break; }
      tc_fence_after();
      if constexpr (DQ) {
        tmem_st16(d_addr + cq * 16, pd);                // dS
      } else {
        tmem_st16(d_addr + cq * 16, pp);                // P^T
        tmem_st16(d_addr + 64 + cq * 16, pd);           // dS^T
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p_full);
    }
    if (ok && warp_wait(&bar_acc_full, 0, ab)) {
      tc_fence_after();
      const size_t o = ((size_t)I.bh * A.L + I.start + row) * 128 + cq * 32;
      const bool acc = A.accumulate != 0;
      uint32_t r[32];
      tmem_ld32(tmem + lane_addr + kColAcc0 + cq * 32, r);
      tmem_ld_wait();
      // dq: out0 = scale dQ; dkdv: out1 = dV
      if (live) store_row32((DQ ? A.out0 : A.out1) + o, r, DQ ? A.scale : 1.0f, acc);
      if constexpr (!DQ) {
        tmem_ld32(tmem + lane_addr + kColAcc1 + cq * 32, r);
        tmem_ld_wait();
        if (live) store_row32(A.out0 + o, r, A.scale, acc);   // dK
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void __launch_bounds__(kSoftmaxBwdThreads, 1)
    softmax_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ SoftmaxBwdArgs A) {
  softmax_bwd_body<false>(tm_k, tm_v, tm_q, tm_do, A);
}

__global__ void __launch_bounds__(kSoftmaxBwdThreads, 1)
    softmax_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ SoftmaxBwdArgs A) {
  softmax_bwd_body<true>(tm_q, tm_do, tm_k, tm_v, A);
}

}  // namespace vdn
