// quantize.cu - e4m3 quantisation of q, k, v for the FP8 softmax branch.
//
// The pages say only that the fastest configuration runs in FP8 (README,
// "Your first render"; "Performance Results": Ulysses parallelism and FP8).
// This library's reading: OCP e4m3 codes, one fp32 scale per (b, h) and
// tensor, scale = amax / 448 (1 when amax = 0), code = round-to-nearest-even
// of the fp32 quotient x / scale, saturating at +-448.
//
// Two launches per tensor: a max-abs reduction per (b, h) into a workspace
// word (atomicMax on the bit pattern, which orders non-negative floats), then
// the conversion, 16 elements per thread (two 16-byte loads, one 16-byte
// store). HBM-bound: 2 + 2 + 1 bytes per element.
#include "kernels.h"

namespace vdn {

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
    fp8_amax_kernel(const __nv_bfloat16* __restrict__ x, long per_head, uint32_t* amax_bits) {
  const int bh = blockIdx.y;
  const uint4* xv = reinterpret_cast<const uint4*>(x + (size_t)bh * per_head);
  const long n8 = per_head / 8;
  float m = 0.f;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long)gridDim.x * blockDim.x) {
    const uint4 u = __ldg(xv + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // |bf16| as fp32: clear the sign bit, move the 16 bits up
      m = fmaxf(m, __uint_as_float((w[k] & 0x7FFFu) << 16));
      m = fmaxf(m, __uint_as_float(w[k] & 0x7FFF0000u));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, red[i]);
    atomicMax(amax_bits + bh, __float_as_uint(m));
  }
}

// Two floats to two e4m3 codes (lo in the low byte), rounding to nearest
// even and saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kQuantThreads)
    fp8_quantize_kernel(const __nv_bfloat16* __restrict__ x, long per_head,
                        const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ x8,
                        float* __restrict__ scale) {
  const int bh = blockIdx.y;
  const float amax = __uint_as_float(amax_bits[bh]);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[bh] = s;
  const uint4* xv = reinterpret_cast<const uint4*>(x + (size_t)bh * per_head);
  uint4* ov = reinterpret_cast<uint4*>(x8 + (size_t)bh * per_head);
  const long n16 = per_head / 16;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
       i += (long)gridDim.x * blockDim.x) {
    const uint4 a = __ldg(xv + 2 * i), b = __ldg(xv + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w0 = w[2 * k], w1 = w[2 * k + 1];
      const float f0 = __fdiv_rn(__uint_as_float(w0 << 16), s);
      const float f1 = __fdiv_rn(__uint_as_float(w0 & 0xFFFF0000u), s);
      const float f2 = __fdiv_rn(__uint_as_float(w1 << 16), s);
      const float f3 = __fdiv_rn(__uint_as_float(w1 & 0xFFFF0000u), s);
      o[k] = e4m3x2(f0, f1) | (e4m3x2(f2, f3) << 16);
    }
    ov[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_quantize_fp8(const void* x, long per_head, int BH, void* x8, float* scale,
                                uint32_t* amax_ws, int sms, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax_ws, 0, sizeof(uint32_t) * BH, stream);
  if (e != cudaSuccess) return e;
  // about four waves of blocks over all heads
  long want = (4L * sms * 2048 / kQuantThreads + BH - 1) / BH;
  const long maxb = (per_head / 16 + kQuantThreads - 1) / kQuantThreads;
  const unsigned gx = (unsigned)std::max(1L, std::min(want, maxb));
  fp8_amax_kernel<<<dim3(gx, BH), kQuantThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), per_head, amax_ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fp8_quantize_kernel<<<dim3(gx, BH), kQuantThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), per_head, amax_ws, static_cast<uint8_t*>(x8), scale);
  return cudaGetLastError();
}

}  // namespace vdn
