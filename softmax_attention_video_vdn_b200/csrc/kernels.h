// kernels.h - launch-side declarations of the VDN kernels and of the data
// they share with the host code in api.cu.
#pragma once

#include "common.cuh"
#include "plan.h"
#include "softmax_window.h"

namespace vdn {

// ---- TMA tensor maps (tensor_map.cu)
// Tiled map with 128-byte swizzle over a `rank`-dimensional tensor; dims[0]
// is the contiguous dimension, strides_bytes[i] the stride of dims[i + 1].
// Returns false if the driver's encoder is unavailable or rejects the map.
bool make_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, const cuuint32_t* box,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

// ---- block-sparse softmax (softmax_window.cu): softmax_window.h

// ---- softmax backward (softmax_bwd.cu)
constexpr int kBwdStages = 2;              // inner (128-row) tile pairs in flight
constexpr int kSoftmaxBwdThreads = 640;
// outer pair + ring of inner tile pairs + ring of the inner tiles' (lse, D)
// pairs (128 float2 per stage)
constexpr size_t kSoftmaxBwdSmem =
    1024 + kTileBytes * (2 + 2 * kBwdStages) + kBwdStages * 128 * 8;

struct SoftmaxBwdArgs {
  SoftmaxPlan plan;          // the forward's segments; tile_begin / total_tiles count
                             // single 128-row tiles
  int BH, L;
  float scale_log2, scale;
  const float2* rowstat;     // [BH][L]: (lse2, D) of each query row
  __nv_bfloat16* out0;       // dkdv: dk, dq: dq   ([BH][L][128])
  __nv_bfloat16* out1;       // dkdv: dv
  int accumulate;            // 1: add to the bf16 values already in the outputs
  int32_t* dev_status;
};

// Outer and inner tensors with 128-row boxes.
__global__ void softmax_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k,
                                        const __grid_constant__ CUtensorMap tm_v,
                                        const __grid_constant__ CUtensorMap tm_q,
                                        const __grid_constant__ CUtensorMap tm_do,
                                        const __grid_constant__ SoftmaxBwdArgs A);
__global__ void softmax_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                                      const __grid_constant__ CUtensorMap tm_do,
                                      const __grid_constant__ CUtensorMap tm_k,
                                      const __grid_constant__ CUtensorMap tm_v,
                                      const __grid_constant__ SoftmaxBwdArgs A);

// ---- e4m3 quantisation (quantize.cu): per-(b, h) scale amax / 448 of x
// [BH][per_head] bf16 into x8 (bytes) and scale[BH]; amax_ws holds BH words.
cudaError_t launch_quantize_fp8(const void* x, long per_head, int BH, void* x8, float* scale,
                                uint32_t* amax_ws, int sms, cudaStream_t stream);

// ---- frame stats (frame_stats.cu)
constexpr int kStatsStages = 6;  // 193 KB of shared memory: one CTA (512 TMEM columns) per SM
constexpr uint32_t kStatsChunk = 64 * 64 * 2;          // 64 tokens x 64 dims bf16
constexpr uint32_t kStatsStageBytes = 4 * kStatsChunk;  // K (2 chunks) + V (2 chunks)
constexpr size_t kStatsSmem = 1024 + kStatsStages * kStatsStageBytes;

// G_f = K_f^T K_f and C_f = V_f^T K_f for frames = B*H*T frames of N tokens,
// read through 4-D maps (dims 128, N, T, B*H; box 64 x 64 x 1 x 1).
cudaError_t launch_frame_stats_bf16(const CUtensorMap& tm_k, const CUtensorMap& tm_v, float* G,
                                    float* C, int frames, int T, int N, cudaStream_t stream);
__global__ void frame_stats_f32_kernel(const float* k, const float* v, float* G, float* C, int T,
                                       int N, int d, int dv);

// ---- merge (gated_merge.cu)
constexpr int kMergeStages = 4;
constexpr uint32_t kMergeABytes = 128 * 64 * 2;  // 128 rows x 64 K
constexpr uint32_t kMergeBBox = 64 * 64 * 2;     // 64 K rows x 64 N
constexpr uint32_t kMergeStageBytes = kMergeABytes + 4 * kMergeBBox;
constexpr size_t kMergeSmem = 1024 + kMergeStages * kMergeStageBytes;
constexpr int kMergeThreads = 192;   // TMA, MMA, four epilogue warps

// Layout of Z for the merge: groups = 0, plain [M, 2, H, dv]; otherwise the
// head-sharded layer's received layout [B, groups, Ls, 2, Hs, dv] (Hs = H /
// groups heads per group, dv_chunks = dv / 64).
struct MergeGroups {
  int groups, Hs, dv_chunks, Ls;
};
__global__ void gated_merge_bf16_kernel(const __grid_constant__ CUtensorMap tm_z,
                                        const __grid_constant__ CUtensorMap tm_w1,
                                        const __grid_constant__ CUtensorMap tm_w2,
                                        __nv_bfloat16* Y, int M, int n_out, int K1,
                                        MergeGroups grp, int32_t* dev_status);
__global__ void gated_merge_f32_kernel(const float* Z, const float* W1, const float* W2, float* Y,
                                       long M, int H, int dv, int n_out, int w_per_head);

// ---- head-sharded layer's layout copy (reshard.cu): x [B, Ls, H, 128] bf16
// -> out [B, Hs, G, Ls, 128], H = G * Hs, rows = B * H * Ls
__global__ void pack_head_groups_kernel(const uint4* x, uint4* out, int rows, int Ls, int H,
                                        int Hs, int G);

// ---- linear branch (bidir_scan.cu)
// Per frame A_f = (1 - beta) I + beta lambda M_f and B_f = beta C_f M_f with
// M_f = (G_f + lambda I)^-1 (fp64; the FP64 tensor-path kernel for d = dv =
// 128). M: NULL, or [frames][d][d] receiving M_f in fp32.
cudaError_t launch_frame_solve(const float* G, const float* C, float* A, float* B, float* M,
                               unsigned frames, int T, int d, int dv, float lambda, float beta,
                               int anchors, int32_t* dev_status, cudaStream_t s);
constexpr int kScanThreads = 256;
constexpr int kStateScanRows = 64;   // state rows per CTA of the scan and of its adjoint
size_t scan_smem_bytes(int d);
// S_all: NULL, or [BH][2][T][dv][d] receiving, for each direction, the state
// before every frame in that direction's order (the backward's checkpoints).
__global__ void bidir_scan_kernel(const float* Aall, const float* Ball, float* S_fwd, float* S_bwd,
                                  float* S_all, int T, int d, int dv, int bf, int W, int anchors,
                                  int nb, int32_t* dev_status);

// ---- linear-branch backward (linear_bwd.cu), d = dv = 128
constexpr size_t kStatsBwdSmem = 1024 + (size_t)7 * 128 * 128 * 2;  // 3 operands + 2 K/V stages

struct LinearBwdLaunch {
  int BH, T, N, n_ctx, nb, bf, W, anchors;
  float lambda, beta;
  const float* Cq;        // [BH][T][dv][d]: per-frame do^T q
  float* dS;              // [BH][nb][dv][d]: block sums of Cq
  const float* A;         // [BH][T][d][d]: the forward's A_f
  float* Lam_all;         // [BH][2][T][dv][d]: cotangent after each frame, per direction
  const float* S_all;     // [BH][2][T][dv][d]: state before each frame, per direction
  const float* C;         // [BH][T][dv][d]: the forward's C_f
  const float* M;         // [BH][T][d][d]: M_f
  float *Gsym, *dC, *dCt; // [BH][T][d][d], [BH][T][dv][d], [BH][T][d][dv]
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
  __nv_bfloat16 *dk, *dv; // [BH][L][128], overwritten with the linear branch's part
  int32_t* dev_status;
};
// block sums, adjoint scan, per-frame grads and the stats backward, in order
cudaError_t launch_linear_bwd_kernels(const LinearBwdLaunch& p, cudaStream_t s);

// ---- merge backward and the backward's preparation (merge_bwd.cu)
// dZ [M][2K1] = dY [M][n_out] [W1; W2]^T (bf16 out); dW1, dW2 [K1][n_out]
// (fp32, accumulated with atomics: zero them first) += Z^T dY.
cudaError_t launch_merge_dgrad(const void* dY, const void* W1, const void* W2, void* dZ, long M,
                               int n_out, int K1, int32_t* dev_status, cudaStream_t s);
cudaError_t launch_merge_wgrad(const void* Z, const void* dY, float* dW1, float* dW2, long M,
                               int n_out, int K1, int32_t* dev_status, cudaStream_t s);
// From dZ and Z ([B*L][2][H][128] bf16), the gate logits and the forward's
// lse ([BH][L]): do_sm = g dZ_sm, do_lin = (1 - g) dZ_lin ([BH][L][128] bf16),
// rowstat = (lse, D = dZ_sm . Z_sm) and dgate_logits[h] += sum over tokens of
// (1 - g) D - g dZ_lin . Z_lin (zero it first).
cudaError_t launch_bwd_prep(const void* dZ, const void* Z, const float* gate_logits,
                            const float* lse, void* do_sm, void* do_lin, float2* rowstat,
                            float* dgate_logits, int B, int H, long L, int sms, cudaStream_t s);
// Standalone softmax backward: from o and do token-major [B][L][H][128],
// rowstat = (lse, o . do) per row and do_hm, a head-major copy of do.
cudaError_t launch_rowstat(const void* o, const void* dout, const float* lse, float2* rowstat,
                           void* do_hm, int B, int H, long L, int sms, cudaStream_t s);

// ---- scratch of the no-allocation scan (noalloc.cu)
cudaError_t noalloc_scratch(void** out);
size_t noalloc_scratch_bytes();

// ---- tensor-core readout (readout.cu)
// Output addressing, in elements: token t of (b, h) goes to
// o + b*b_stride + t*tok_stride + h*h_stride + off.
//   o_lin [B, L, H, dv]:      b_stride L*H*128,  tok_stride H*128,   h_stride 128, off 0
//   linear half of Z:         b_stride L*2H*128, tok_stride 2*H*128, h_stride 128, off H*128
//   head-major [B, H, L, d]:  b_stride H*L*128,  tok_stride 128,     h_stride L*128, off 0
struct ReadoutOut {
  long b_stride, tok_stride, h_stride, off;
};
// gate_logits non-NULL scales by 1 - sigmoid. transpose_s: multiply by
// (S_fwd + S_bwd)^T instead (the backward's dq = S^T do). n_ctx context tokens
// follow the T*N video tokens of each (b, h); their rows are written as zeros.
cudaError_t launch_readout_bf16(const CUtensorMap& tm_q, const float* S_fwd, const float* S_bwd,
                                void* o, int B, int H, int T, int N, int bf, int anchors, int nb,
                                int n_ctx, const ReadoutOut& out, bool transpose_s,
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
