// kernels.h - launch-side declarations of the VDN kernels and of the data
// they share with the host code in api.cu.
#pragma once

#include "common.cuh"
#include "plan.h"

namespace vdn {

// ---- block-sparse softmax (softmax_window.cu)
constexpr int kKStages = 3, kVStages = 2;  // softmax K and V rings
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128x128 bf16 tile
constexpr size_t kSoftmaxSmem = 1024 + kTileBytes * (2 + kKStages + kVStages);  // Q0, Q1, K, V
constexpr int kSoftmaxThreads = 640;

struct SoftmaxArgs {
  SoftmaxPlan plan;
  int BH, H, L, nb;
  float scale_log2;
  const float* gate_logits;  // NULL: write o_sm; else g * o_sm into the softmax half of Z
  const float* q_scale;      // e4m3 kernel: per-(b, h) scales of q, k, v
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* out;
  int32_t* dev_status;
  int* work_counter;   // zeroed before the launch; items are taken with atomicAdd
};

__global__ void softmax_window_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                           const __grid_constant__ CUtensorMap tm_k,
                                           const __grid_constant__ CUtensorMap tm_v,
                                           const __grid_constant__ SoftmaxArgs A);
__global__ void softmax_window_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                                          const __grid_constant__ CUtensorMap tm_k,
                                          const __grid_constant__ CUtensorMap tm_v,
                                          const __grid_constant__ SoftmaxArgs A);
constexpr size_t kSoftmaxSmemF8 = 1024 + (kTileBytes / 2) * (2 + kKStages + kVStages);

// ---- e4m3 quantisation (quantize.cu): per-(b, h) scale amax / 448 of x
// [BH][per_head] bf16 into x8 (bytes) and scale[BH]; amax_ws holds BH words.
cudaError_t launch_quantize_fp8(const void* x, long per_head, int BH, void* x8, float* scale,
                                uint32_t* amax_ws, int sms, cudaStream_t stream);

// ---- frame stats (frame_stats.cu)
constexpr int kStatsStages = 4;  // 129 KB of shared memory: one CTA (512 TMEM columns) per SM
constexpr uint32_t kStatsChunk = 64 * 64 * 2;          // 64 tokens x 64 dims bf16
constexpr uint32_t kStatsStageBytes = 4 * kStatsChunk;  // K (2 chunks) + V (2 chunks)
constexpr size_t kStatsSmem = 1024 + kStatsStages * kStatsStageBytes;

__global__ void frame_stats_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                                        const __grid_constant__ CUtensorMap tm_v, float* G,
                                        float* C, int T, int N, int32_t* dev_status);
__global__ void frame_stats_f32_kernel(const float* k, const float* v, float* G, float* C, int T,
                                       int N, int d, int dv);

// ---- merge (gated_merge.cu)
constexpr int kMergeStages = 4;
constexpr uint32_t kMergeABytes = 128 * 64 * 2;  // 128 rows x 64 K
constexpr uint32_t kMergeBBox = 64 * 64 * 2;     // 64 K rows x 64 N
constexpr uint32_t kMergeStageBytes = kMergeABytes + 4 * kMergeBBox;
constexpr size_t kMergeSmem = 1024 + kMergeStages * kMergeStageBytes;

__global__ void gated_merge_bf16_kernel(const __grid_constant__ CUtensorMap tm_z,
                                        const __grid_constant__ CUtensorMap tm_w1,
                                        const __grid_constant__ CUtensorMap tm_w2,
                                        __nv_bfloat16* Y, int M, int n_out, int K1,
                                        int32_t* dev_status);
__global__ void gated_merge_f32_kernel(const float* Z, const float* W1, const float* W2, float* Y,
                                       long M, int H, int dv, int n_out, int w_per_head);

// ---- linear branch (bidir_scan.cu)
size_t solve_smem_bytes(int d, int dv);
__global__ void frame_solve_kernel(const float* G, const float* C, float* Aout, float* Bout, int T,
                                   int d, int dv, float lambda, float beta, int anchors,
                                   int32_t* dev_status);
constexpr int kScanRows = 16;
constexpr int kScanThreads = 256;
size_t scan_smem_bytes(int d);
__global__ void bidir_scan_kernel(const float* Aall, const float* Ball, float* S_fwd, float* S_bwd,
                                  int T, int d, int dv, int bf, int W, int anchors, int nb,
                                  int32_t* dev_status);

// ---- scratch of the no-allocation scan (noalloc.cu)
cudaError_t noalloc_scratch(void** out);
size_t noalloc_scratch_bytes();

// ---- tensor-core readout (readout.cu)
// o + ((b*L + t) * o_tok_stride + o_head_off + h*128) receives token t of
// (b, h): o_tok_stride = H*128 (o_lin) or 2*H*128 with o_head_off = H*128
// (the linear half of Z); gate_logits non-NULL scales by 1 - sigmoid.
// n_ctx context tokens follow the T*N video tokens of each (b, h); their rows
// are written as zeros.
cudaError_t launch_readout_bf16(const CUtensorMap& tm_q, const float* S_fwd, const float* S_bwd,
                                void* o, int B, int H, int T, int N, int bf, int anchors, int nb,
                                int n_ctx, long o_tok_stride, long o_head_off,
                                const float* gate_logits, int32_t* dev_status,
                                cudaStream_t stream);

// ---- bounded-wait self-test (selftest.cu)
cudaError_t launch_wait_timeout(int32_t* dev_status, int limit_ms, cudaStream_t stream);

// ---- CUDA-core kernels (simt_kernels.cu)
// fp32 readout (CUDA cores); output addressing and gate as launch_readout_bf16.
cudaError_t launch_readout_f32(const void* q, const float* S_fwd, const float* S_bwd, void* o,
                               int B, int H, int Tf, int N, int d, int dv, int bf, int anchors,
                               int nb, long o_tok_stride, long o_head_off, const float* gate,
                               cudaStream_t stream);
__global__ void softmax_window_f32_kernel(const float* q, const float* k, const float* v,
                                          const float* S_fwd, const float* S_bwd,
                                          const float* gate, float* out, int B, int H, int Tf,
                                          int N, int d, int dv, int bf, int W, int anchors, int nb,
                                          float scale);

}  // namespace vdn
