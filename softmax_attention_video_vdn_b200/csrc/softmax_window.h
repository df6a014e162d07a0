// softmax_window.h - the forward softmax kernel's launch parameters and
// declarations (shared by softmax_window.cu and the host code).
#pragma once

#include "common.cuh"
#include "plan.h"

namespace vdn {

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
  float* lse;          // NULL, or [BH][L]: log2-domain log-sum-exp of each row's scaled scores
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

}  // namespace vdn
