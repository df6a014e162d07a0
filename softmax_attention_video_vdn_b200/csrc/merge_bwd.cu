// merge_bwd.cu - backward of the gated merge on sm_100a, and the
// elementwise preparation of the branch cotangents.
//
// Forward (mlsanity abstract: separate output projections, learnable gates):
//   Z = [g_h o_sm,h | (1 - g_h) o_lin,h],  Y = Z [W1; W2],  g_h = sigmoid(logit_h).
// Backward, for the output cotangent dY:
//   dZ = dY [W1; W2]^T                     merge_dgrad_kernel (tcgen05)
//   dW1, dW2 = Z_sm^T dY, Z_lin^T dY        merge_wgrad_kernel (tcgen05, split-K)
//   do_sm = g dZ_sm, do_lin = (1 - g) dZ_lin,
//   D = do_sm . o_sm = dZ_sm . Z_sm (the softmax backward's row term),
//   dlogit_h = sum_t (1 - g) dZ_sm . Z_sm - g dZ_lin . Z_lin
//                                           bwd_prep_kernel
// (the last line is g (1 - g) (dZ_sm . o_sm - dZ_lin . o_lin) with the
// gated values Z in place of o).
#include <algorithm>

#include "kernels.h"

namespace vdn {

constexpr int kMbStages = 4;
constexpr uint32_t kMbHalf = 128 * 64 * 2;          // 128 rows x 64 K (K-major box)
constexpr uint32_t kMbStage = 3 * kMbHalf;          // A (128 rows) + B (256 rows)
constexpr size_t kMbSmem = 1024 + kMbStages * kMbStage;
constexpr uint32_t kWgBox = 64 * 64 * 2;            // 64 x 64 (MN-major box)
constexpr uint32_t kWgStage = 2 * kWgBox + 4 * kWgBox;  // A (128 features) + B (256 columns)
constexpr size_t kWgSmem = 1024 + kMbStages * kWgStage;
constexpr int kWgTokens = 16384;                    // tokens per split of the K loop

// Shared structure of the two GEMMs: warp 0 TMA producer, warp 1 MMA issuer,
// all four warps drain the 128 x 256 fp32 accumulator.
template <bool WGRAD>
__device__ __forceinline__ void merge_bwd_body(const CUtensorMap& tm_a, const CUtensorMap& tm_b0,
                                               const CUtensorMap& tm_b1, void* out0, float* out1,
                                               int M, int n_out, int K1, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kMbStages], bar_empty[kMbStages], bar_done, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  constexpr uint32_t kStage = WGRAD ? kWgStage : kMbStage;
  constexpr uint32_t kABytes = WGRAD ? 2 * kWgBox : kMbHalf;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n2 = 2 * K1;
  const int n_tiles = (WGRAD ? (n_out + 255) / 256 : n2 / 256);
  // dgrad: 128 tokens x 256 features of dZ, K = n_out.
  // wgrad: 128 features x 256 output columns of dW, K = a split of the tokens.
  int m0, n0, c_begin, c_end;
  if constexpr (WGRAD) {
    const int m_tiles = n2 / 128;
    const int per_split = m_tiles * n_tiles;
    const int split = blockIdx.x / per_split;
    const int rem = blockIdx.x - split * per_split;
    m0 = (rem / n_tiles) * 128;
    n0 = (rem % n_tiles) * 256;
    c_begin = split * (kWgTokens / 64);
    c_end = min((M + 63) / 64, c_begin + kWgTokens / 64);
  } else {
    m0 = (blockIdx.x / n_tiles) * 128;
    n0 = (blockIdx.x % n_tiles) * 256;
    c_begin = 0;
    c_end = (n_out + 63) / 64;
  }
  const int nchunks = c_end - c_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMbStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_done, 1);
    mbar_init(&bar_drain, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b0);
    tma_prefetch_desc(&tm_b1);
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
        const int st = c % kMbStages;
        const int use = c / kMbStages;
        if (use > 0 && !mbar_wait(&bar_empty[st], (use - 1) & 1, ab)) break;
        uint8_t* s = base + st * kStage;
        mbar_arrive_expect_tx(&bar_full[st], kStage);
        const int k0 = (c_begin + c) * 64;
        if constexpr (WGRAD) {
          // A: Z [tokens k0.., features m0..m0+127] (two 64-feature boxes);
          // B: dY [tokens k0.., columns n0..n0+255] (four 64-column boxes)
          for (int x = 0; x < 2; ++x)
            tma_load_2d(s + x * kWgBox, &tm_a, &bar_full[st], m0 + x * 64, k0);
          for (int x = 0; x < 4; ++x)
            tma_load_2d(s + kABytes + x * kWgBox, &tm_b0, &bar_full[st], n0 + x * 64, k0);
        } else {
          // A: dY [tokens m0.., K k0..]; B: 256 rows of [W1; W2] in two halves
          tma_load_2d(s, &tm_a, &bar_full[st], k0, m0);
          for (int x = 0; x < 2; ++x) {
            const int n = n0 + x * 128;
            const CUtensorMap* wm = n < K1 ? &tm_b0 : &tm_b1;
            tma_load_2d(s + kABytes + x * kMbHalf, wm, &bar_full[st], k0, n < K1 ? n : n - K1);
          }
        }
      }
      if (c < nchunks)  // aborted: let the issued copies land before exit
        for (int cc = (c > kMbStages ? c - kMbStages : 0); cc < c; ++cc)
          mbar_wait_drain(&bar_full[cc % kMbStages], (cc / kMbStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = WGRAD ? idesc_bf16_f32(128, 256, 1, 1) : idesc_bf16_f32(128, 256, 0, 0);
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % kMbStages;
        if (!mbar_wait(&bar_full[st], (c / kMbStages) & 1, ab)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(base + st * kStage);
        const uint32_t sb = sa + kABytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint64_t da, db;
          if constexpr (WGRAD) {
            da = sdesc_sw128(sa + ks * 2048, kWgBox, 1024);   // MN-major, 64-feature chunks
            db = sdesc_sw128(sb + ks * 2048, kWgBox, 1024);   // MN-major, 64-column chunks
          } else {
            da = sdesc_sw128(sa + ks * 32, 16, 1024);         // K-major
            db = sdesc_sw128(sb + ks * 32, 16, 1024);         // K-major, 256 rows
          }
          umma_ss(tmem, da, db, idesc, (c > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bar_empty[st]);
      }
      if (ok) umma_commit(&bar_done);
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
    }
    __syncwarp();
  }

  if (nchunks > 0 && warp_wait(&bar_done, 0, ab)) {
    tc_fence_after();
    const int row = warp * 32 + lane;
    const int m = m0 + row;
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_addr + c * 32, r);
      tmem_ld_wait();
      if constexpr (WGRAD) {
        // feature row m of [dW1; dW2], columns n0 + c*32 ..
        float* wrow = m < K1 ? out1 + (size_t)m * n_out
                             : static_cast<float*>(out0) + (size_t)(m - K1) * n_out;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int col = n0 + c * 32 + i * 4;
          if (col < n_out)
            atomicAdd(reinterpret_cast<float4*>(wrow + col),
                      make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                  __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
        }
      } else {
        if (m < M) {
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pw[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          __nv_bfloat16* zrow = static_cast<__nv_bfloat16*>(out0) + (size_t)m * n2 + n0 + c * 32;
#pragma unroll
          for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(zrow)[i] = pk[i];
        }
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

__global__ void __launch_bounds__(128, 1)
    merge_dgrad_kernel(const __grid_constant__ CUtensorMap tm_dy,
                       const __grid_constant__ CUtensorMap tm_w1,
                       const __grid_constant__ CUtensorMap tm_w2, __nv_bfloat16* dZ, int M,
                       int n_out, int K1, int32_t* dev_status) {
  merge_bwd_body<false>(tm_dy, tm_w1, tm_w2, dZ, nullptr, M, n_out, K1, dev_status);
}

__global__ void __launch_bounds__(128, 1)
    merge_wgrad_kernel(const __grid_constant__ CUtensorMap tm_z,
                       const __grid_constant__ CUtensorMap tm_dy, float* dW1, float* dW2, int M,
                       int n_out, int K1, int32_t* dev_status) {
  // out1 receives the rows < K1 (dW1), out0 the rest (dW2)
  merge_bwd_body<true>(tm_z, tm_dy, tm_dy, dW2, dW1, M, n_out, K1, dev_status);
}

// ------------------------------------------------------------- preparation
// One half-warp (16 lanes x 8 values) per (token, head).
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const __nv_bfloat16* __restrict__ dZ, const __nv_bfloat16* __restrict__ Z,
                    const float* __restrict__ gate_logits, const float* __restrict__ lse,
                    __nv_bfloat16* __restrict__ do_sm, __nv_bfloat16* __restrict__ do_lin,
                    float2* __restrict__ rowstat, float* __restrict__ dgate, int B, int H,
                    long L) {
  extern __shared__ float gsum[];  // [H]
  for (int h = threadIdx.x; h < H; h += blockDim.x) gsum[h] = 0.f;
  __syncthreads();
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
  const unsigned hmask = 0xffffu << (16 * (hw & 1));
  const int hws = blockDim.x >> 4;
  const long pairs = (long)B * L * H;
  for (long p = (long)blockIdx.x * hws + hw; p < pairs; p += (long)gridDim.x * hws) {
    const long m = p / H;                 // token row b*L + t
    const int h = (int)(p - m * H);
    const int b = (int)(m / L);
    const long t = m - (long)b * L;
    const float g = sigmoidf_dev(__ldg(gate_logits + h));
    const size_t zo = (size_t)m * 2 * H * 128 + (size_t)h * 128 + hl * 8;
    const size_t lo = (size_t)H * 128;    // the linear half of a token row
    const uint4 a = *reinterpret_cast<const uint4*>(dZ + zo);
    const uint4 c = *reinterpret_cast<const uint4*>(dZ + zo + lo);
    const uint4 za = *reinterpret_cast<const uint4*>(Z + zo);
    const uint4 zc = *reinterpret_cast<const uint4*>(Z + zo + lo);
    const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(&c);
    const uint32_t* zaw = reinterpret_cast<const uint32_t*>(&za);
    const uint32_t* zcw = reinterpret_cast<const uint32_t*>(&zc);
    float D = 0.f, E = 0.f;
    uint4 os, ol;
    uint32_t* osw = reinterpret_cast<uint32_t*>(&os);
    uint32_t* olw = reinterpret_cast<uint32_t*>(&ol);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 dzs = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 dzl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cw[i]));
      const float2 zs = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zaw[i]));
      const float2 zl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zcw[i]));
      D = fmaf(dzs.x, zs.x, fmaf(dzs.y, zs.y, D));
      E = fmaf(dzl.x, zl.x, fmaf(dzl.y, zl.y, E));
      osw[i] = pack_bf16(g * dzs.x, g * dzs.y);
      olw[i] = pack_bf16((1.f - g) * dzl.x, (1.f - g) * dzl.y);
    }
    const size_t ro = ((size_t)b * H + h) * L + t;   // row of (b, h, t), head-major
    *reinterpret_cast<uint4*>(do_sm + ro * 128 + hl * 8) = os;
    *reinterpret_cast<uint4*>(do_lin + ro * 128 + hl * 8) = ol;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      D += __shfl_xor_sync(hmask, D, off);
      E += __shfl_xor_sync(hmask, E, off);
    }
    if (hl == 0) {
      rowstat[ro] = make_float2(__ldg(lse + ro), D);
      atomicAdd(&gsum[h], (1.f - g) * D - g * E);
    }
  }
  __syncthreads();
  for (int h = threadIdx.x; h < H; h += blockDim.x) atomicAdd(dgate + h, gsum[h]);
}

// For the standalone softmax backward: o and do token-major [B][L][H][128];
// rowstat[r] = (lse[r], o . do) and a head-major copy of do for row
// r = (b*H + h)*L + t. One half-warp per row.
__global__ void __launch_bounds__(256)
    rowstat_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                   const float* __restrict__ lse, float2* __restrict__ rowstat,
                   __nv_bfloat16* __restrict__ do_hm, int H, long L, long rows) {
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
  const unsigned hmask = 0xffffu << (16 * (hw & 1));
  const int hws = blockDim.x >> 4;
  for (long r = (long)blockIdx.x * hws + hw; r < rows; r += (long)gridDim.x * hws) {
    const long bh = r / L, t = r - bh * L;
    const long b = bh / H, h = bh - b * H;
    const size_t src = ((size_t)(b * L + t) * H + h) * 128 + hl * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + src);
    const uint4 c = *reinterpret_cast<const uint4*>(dout + src);
    *reinterpret_cast<uint4*>(do_hm + (size_t)r * 128 + hl * 8) = c;
    const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(&c);
    float D = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cw[i]));
      D = fmaf(x.x, y.x, fmaf(x.y, y.y, D));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) D += __shfl_xor_sync(hmask, D, off);
    if (hl == 0) rowstat[r] = make_float2(__ldg(lse + r), D);
  }
}

// ------------------------------------------------------------------ launch
namespace {
// 2-D bf16 map of a row-major [rows][cols] matrix, 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* p, long cols, long rows, int box_cols, int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t str[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  return make_map(m, p, 2, dims, str, box);
}
}  // namespace

cudaError_t launch_merge_dgrad(const void* dY, const void* W1, const void* W2, void* dZ, long M,
                               int n_out, int K1, int32_t* dev_status, cudaStream_t s) {
  CUtensorMap ta, t1, t2;
  if (!map2d(&ta, dY, n_out, M, 64, 128) || !map2d(&t1, W1, n_out, K1, 64, 128) ||
      !map2d(&t2, W2, n_out, K1, 64, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(merge_dgrad_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMbSmem);
  if (e != cudaSuccess) return e;
  const long tiles = ((M + 127) / 128) * ((2L * K1) / 256);
  merge_dgrad_kernel<<<(unsigned)tiles, 128, kMbSmem, s>>>(
      ta, t1, t2, static_cast<__nv_bfloat16*>(dZ), (int)M, n_out, K1, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_merge_wgrad(const void* Z, const void* dY, float* dW1, float* dW2, long M,
                               int n_out, int K1, int32_t* dev_status, cudaStream_t s) {
  CUtensorMap tz, ty;
  if (!map2d(&tz, Z, 2L * K1, M, 64, 64) || !map2d(&ty, dY, n_out, M, 64, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(merge_wgrad_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWgSmem);
  if (e != cudaSuccess) return e;
  const long splits = (M + kWgTokens - 1) / kWgTokens;
  const long tiles = (2L * K1 / 128) * ((n_out + 255) / 256) * splits;
  merge_wgrad_kernel<<<(unsigned)tiles, 128, kWgSmem, s>>>(tz, ty, dW1, dW2, (int)M, n_out, K1,
                                                            dev_status);
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(const void* dZ, const void* Z, const float* gate_logits,
                            const float* lse, void* do_sm, void* do_lin, float2* rowstat,
                            float* dgate_logits, int B, int H, long L, int sms, cudaStream_t s) {
  const long pairs = (long)B * L * H;
  const long want = (pairs + 15) / 16;
  const unsigned grid = (unsigned)std::min<long>(want, (long)sms * 8);
  bwd_prep_kernel<<<grid, 256, (size_t)H * 4, s>>>(
      static_cast<const __nv_bfloat16*>(dZ), static_cast<const __nv_bfloat16*>(Z), gate_logits,
      lse, static_cast<__nv_bfloat16*>(do_sm), static_cast<__nv_bfloat16*>(do_lin), rowstat,
      dgate_logits, B, H, L);
  return cudaGetLastError();
}

cudaError_t launch_rowstat(const void* o, const void* dout, const float* lse, float2* rowstat,
                           void* do_hm, int B, int H, long L, int sms, cudaStream_t s) {
  const long rows = (long)B * H * L;
  const long want = (rows + 15) / 16;
  const unsigned grid = (unsigned)std::min<long>(want, (long)sms * 8);
  rowstat_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(o),
                                      static_cast<const __nv_bfloat16*>(dout), lse, rowstat,
                                      static_cast<__nv_bfloat16*>(do_hm), H, L, rows);
  return cudaGetLastError();
}

}  // namespace vdn
