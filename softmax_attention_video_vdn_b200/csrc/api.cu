// api.cu - the extern "C" entry points declared in include/vdn.h: argument
// validation, TMA tensor maps, the window plan and the kernel launches.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "kernels.h"


using namespace vdn;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

vdn_status check_cfg(const vdn_config* c) {
  if (!c) return VDN_ERR_INVALID_ARG;
  if (c->B < 1 || c->H < 1 || c->T < 1 || c->N < 1) return VDN_ERR_INVALID_ARG;
  if (c->d < 8 || c->dv < 8 || c->d > 128 || c->dv > 128 || (c->d % 8) || (c->dv % 8))
    return VDN_ERR_INVALID_ARG;
  if (c->block_frames < 1 || c->window_blocks < 0 || (c->anchors != 0 && c->anchors != 1))
    return VDN_ERR_INVALID_ARG;
  if (!(c->lambda > 0.f) || !isfinite(c->lambda)) return VDN_ERR_INVALID_ARG;
  if (!(c->beta > 0.f && c->beta <= 1.f)) return VDN_ERR_INVALID_ARG;
  if (!(c->softmax_scale >= 0.f) || !isfinite(c->softmax_scale)) return VDN_ERR_INVALID_ARG;
  if (c->dtype != VDN_F32 && c->dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (c->n_ctx < 0) return VDN_ERR_INVALID_ARG;
  if ((long long)c->T * c->N + c->n_ctx > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  if (c->n_ctx > 0 && c->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  if ((long long)c->B * c->H * c->T > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  if (c->dtype == VDN_BF16 && (c->d != 128 || c->dv != 128)) return VDN_ERR_UNSUPPORTED;
  if (c->dtype == VDN_F32 && (!is_pow2(c->d) || !is_pow2(c->dv))) return VDN_ERR_UNSUPPORTED;
  return VDN_OK;
}

inline size_t elem_bytes(const vdn_config* c) { return c->dtype == VDN_BF16 ? 2 : 4; }
inline int n_blocks(const vdn_config* c) { return (c->T + c->block_frames - 1) / c->block_frames; }
// Tokens per (b, h): T*N video tokens, then n_ctx context tokens.
inline long long tokens(const vdn_config* c) { return (long long)c->T * c->N + c->n_ctx; }

// Text of the last CUDA failure seen by this thread (vdn_last_error).
thread_local char g_last_error[256] = "";

vdn_status cuda_fail(const char* where, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return VDN_ERR_CUDA;
}
vdn_status check(const char* where, cudaError_t e) {
  return e == cudaSuccess ? VDN_OK : cuda_fail(where, e);
}
vdn_status launch_status(const char* where) { return check(where, cudaGetLastError()); }
vdn_status set_smem(const void* fn, size_t bytes, const char* where) {
  return check(where, cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)bytes));
}


// Readout addressing of a token-major output [B, L, halves, H, 128] at
// element offset `off` within a token row.
ReadoutOut token_major_out(const vdn_config* c, int halves, long off) {
  const long tok = (long)halves * c->H * 128;
  return ReadoutOut{(long)tokens(c) * tok, tok, 128, off};
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

struct LayerWs {
  float *G, *C, *S_fwd, *S_bwd;
  void* Z;
  void *q8, *k8, *v8;      // e4m3 copies (FP8 layer only)
  float* scales;           // q, k, v scales [3][B*H]
  uint32_t* amax;          // quantiser workspace [B*H]
  void* scan_ws;
  size_t scan_bytes;
  void* sm_ws;
  size_t sm_bytes;
  size_t total;
};

size_t scan_ws_bytes(const vdn_config* c) {
  const size_t frames = (size_t)c->B * c->H * c->T;
  return align256(frames * c->d * c->d * 4) + align256(frames * c->dv * c->d * 4);
}

LayerWs layer_ws(const vdn_config* c, void* base, bool fp8 = false) {
  LayerWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const size_t frames = (size_t)c->B * c->H * c->T;
  const size_t states = (size_t)c->B * c->H * n_blocks(c) * c->dv * c->d;
  w.G = reinterpret_cast<float*>(take(frames * c->d * c->d * 4));
  w.C = reinterpret_cast<float*>(take(frames * c->dv * c->d * 4));
  w.S_fwd = reinterpret_cast<float*>(take(states * 4));
  w.S_bwd = reinterpret_cast<float*>(take(states * 4));
  w.Z = take((size_t)c->B * tokens(c) * 2 * c->H * c->dv * elem_bytes(c));
  w.scan_bytes = scan_ws_bytes(c);
  w.scan_ws = take(w.scan_bytes);
  w.sm_bytes = 256;
  w.sm_ws = take(w.sm_bytes);
  if (fp8) {
    const size_t bhl = (size_t)c->B * c->H * tokens(c);
    w.q8 = take(bhl * c->d);
    w.k8 = take(bhl * c->d);
    w.v8 = take(bhl * c->dv);
    w.scales = reinterpret_cast<float*>(take((size_t)3 * c->B * c->H * 4));
    w.amax = reinterpret_cast<uint32_t*>(take((size_t)c->B * c->H * 4));
  }
  w.total = off;
  return w;
}

// Token-level segments of the window plan, heaviest first. Context tokens
// [TN, TN + n_ctx) are one more key range of every video segment (merged with
// a range that ends at TN) and their own query segment over every key.
struct TokSeg {
  int q0, q1, nr, k0[kMaxRanges], k1[kMaxRanges];
  long long cost;
};

std::vector<TokSeg> token_segments(const vdn_config* cfg) {
  const int T = cfg->T, N = cfg->N, bf = cfg->block_frames;
  std::vector<FrameSegment> segs = build_segments(T, bf, cfg->window_blocks, cfg->anchors);
  const int TN = T * N, L = (int)tokens(cfg), n_ctx = cfg->n_ctx;
  std::vector<TokSeg> ts;
  for (const auto& fs : segs) {
    TokSeg t{};
    t.q0 = fs.q0 * N;
    t.q1 = fs.q1 * N;
    for (int r = 0; r < fs.nr; ++r) {
      t.k0[r] = fs.k0[r] * N;
      t.k1[r] = fs.k1[r] * N;
    }
    t.nr = fs.nr;
    if (n_ctx > 0) {
      if (t.k1[t.nr - 1] == TN) {
        t.k1[t.nr - 1] = L;
      } else {
        t.k0[t.nr] = TN;
        t.k1[t.nr] = L;
        ++t.nr;
      }
    }
    for (int r = 0; r < t.nr; ++r) t.cost += t.k1[r] - t.k0[r];
    ts.push_back(t);
  }
  if (n_ctx > 0) {
    TokSeg t{};
    t.q0 = TN;
    t.q1 = L;
    t.nr = 1;
    t.k0[0] = 0;
    t.k1[0] = L;
    t.cost = L;
    ts.push_back(t);
  }
  std::stable_sort(ts.begin(), ts.end(),
                   [](const TokSeg& a, const TokSeg& b) { return a.cost > b.cost; });
  return ts;
}

// Segments [first, last) into a launch plan whose work items are groups of
// `tile_rows` query rows; returns the items per (b, h).
int fill_plan(SoftmaxPlan* plan, const std::vector<TokSeg>& ts, size_t first, size_t last,
              int tile_rows) {
  int tiles = 0;
  for (size_t i = first; i < last; ++i) {
    const TokSeg& t = ts[i];
    const int si = (int)(i - first);
    plan->q0[si] = t.q0;
    plan->q1[si] = t.q1;
    plan->tile_begin[si] = tiles;
    tiles += (t.q1 - t.q0 + tile_rows - 1) / tile_rows;
    plan->nr[si] = t.nr;
    for (int r = 0; r < t.nr; ++r) {
      plan->k0[si][r] = t.k0[r];
      plan->k1[si][r] = t.k1[r];
    }
  }
  plan->n_seg = (int)(last - first);
  plan->total_tiles = tiles;
  return tiles;
}

// Launches the tensor-core softmax kernel (bf16 or e4m3 inputs) over the
// token-level segments of the window plan, heaviest first, in chunks of at
// most kMaxLaunchSegments segments per launch. lse: NULL, or [BH][L] log2-domain
// row log-sum-exps for the backward.
vdn_status launch_softmax_tc(const vdn_config* cfg, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, bool fp8, float scale,
                             const float* gate_logits, const float* q_scale,
                             const float* k_scale, const float* v_scale, void* out, void* ws,
                             int32_t* dev_status, cudaStream_t s, float* lse = nullptr) {
  const int BH = cfg->B * cfg->H;
  const void* kern = fp8 ? (const void*)softmax_window_fp8_kernel
                         : (const void*)softmax_window_bf16_kernel;
  const size_t smem = fp8 ? kSoftmaxSmemF8 : kSoftmaxSmem;
  vdn_status st = set_smem(kern, smem, "softmax smem attribute");
  if (st != VDN_OK) return st;
  const std::vector<TokSeg> ts = token_segments(cfg);
  const int nsm = sm_count();
  for (size_t first = 0; first < ts.size(); first += kMaxLaunchSegments) {
    SoftmaxArgs A;
    memset(&A, 0, sizeof(A));
    const size_t last = std::min(ts.size(), first + (size_t)kMaxLaunchSegments);
    const int tiles = fill_plan(&A.plan, ts, first, last, 2 * kQTile);  // pairs of q tiles
    A.BH = BH;
    A.H = cfg->H;
    A.L = (int)tokens(cfg);
    A.nb = n_blocks(cfg);
    A.scale_log2 = scale * 1.4426950408889634f;
    A.gate_logits = gate_logits;
    A.q_scale = q_scale;
    A.k_scale = k_scale;
    A.v_scale = v_scale;
    A.out = static_cast<__nv_bfloat16*>(out);
    A.lse = lse;
    A.dev_status = dev_status;
    A.work_counter = static_cast<int*>(ws);
    st = check("softmax work counter reset", cudaMemsetAsync(ws, 0, sizeof(int), s));
    if (st != VDN_OK) return st;
    const long long items = (long long)tiles * BH;
    const unsigned grid = (unsigned)std::min<long long>(items, nsm);
    if (fp8)
      softmax_window_fp8_kernel<<<grid, kSoftmaxThreads, smem, s>>>(tq, tk, tv, A);
    else
      softmax_window_bf16_kernel<<<grid, kSoftmaxThreads, smem, s>>>(tq, tk, tv, A);
    st = launch_status("softmax launch");
    if (st != VDN_OK) return st;
  }
  return VDN_OK;
}

// [BH][L][128] bf16 tensor map of q, k, v or do (64-column boxes of
// box_rows rows).
bool head_major_map(CUtensorMap* m, const void* p, const vdn_config* cfg, int box_rows = 128) {
  const cuuint64_t dims[3] = {128, (cuuint64_t)tokens(cfg), (cuuint64_t)cfg->B * cfg->H};
  const cuuint64_t str[2] = {256, (cuuint64_t)tokens(cfg) * 256};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  return make_map(m, p, 3, dims, str, box);
}

// Both softmax backward kernels (dk, dv by key tiles; dq by query tiles) over
// the forward's segments.
vdn_status launch_softmax_bwd(const vdn_config* cfg, const void* q, const void* k, const void* v,
                              const void* dout, const float2* rowstat, void* dq, void* dk,
                              void* dv, bool accumulate, int32_t* dev_status, cudaStream_t s) {
  // outer tiles and streamed inner tiles: 128-row boxes
  CUtensorMap tq, tk, tv, tdo;
  if (!head_major_map(&tq, q, cfg) || !head_major_map(&tk, k, cfg) ||
      !head_major_map(&tv, v, cfg) || !head_major_map(&tdo, dout, cfg))
    return cuda_fail("softmax backward tensor map", cudaErrorInvalidValue);
  vdn_status st = set_smem((const void*)softmax_bwd_dkdv_kernel, kSoftmaxBwdSmem,
                           "softmax backward smem attribute");
  if (st != VDN_OK) return st;
  st = set_smem((const void*)softmax_bwd_dq_kernel, kSoftmaxBwdSmem,
                "softmax backward smem attribute");
  if (st != VDN_OK) return st;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)cfg->d);
  const int BH = cfg->B * cfg->H;
  const std::vector<TokSeg> ts = token_segments(cfg);
  for (size_t first = 0; first < ts.size(); first += kMaxLaunchSegments) {
    SoftmaxBwdArgs A;
    memset(&A, 0, sizeof(A));
    const size_t last = std::min(ts.size(), first + (size_t)kMaxLaunchSegments);
    const int tiles = fill_plan(&A.plan, ts, first, last, kQTile);
    A.BH = BH;
    A.L = (int)tokens(cfg);
    A.scale_log2 = scale * 1.4426950408889634f;
    A.scale = scale;
    A.rowstat = rowstat;
    A.accumulate = accumulate ? 1 : 0;
    A.dev_status = dev_status;
    const long long items = (long long)tiles * BH;
    if (items > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
    A.out0 = static_cast<__nv_bfloat16*>(dk);
    A.out1 = static_cast<__nv_bfloat16*>(dv);
    softmax_bwd_dkdv_kernel<<<(unsigned)items, kSoftmaxBwdThreads, kSoftmaxBwdSmem, s>>>(
        tk, tv, tq, tdo, A);
    st = launch_status("softmax backward (dk, dv) launch");
    if (st != VDN_OK) return st;
    A.out0 = static_cast<__nv_bfloat16*>(dq);
    A.out1 = nullptr;
    softmax_bwd_dq_kernel<<<(unsigned)items, kSoftmaxBwdThreads, kSoftmaxBwdSmem, s>>>(
        tq, tdo, tk, tv, A);
    st = launch_status("softmax backward (dq) launch");
    if (st != VDN_OK) return st;
  }
  return VDN_OK;
}

// Workspace of the linear-branch backward (d = dv = 128).
struct LinBwdWs {
  float *G, *C, *A, *Bm, *M, *Cq, *Gsym, *dC, *dCt, *S_fwd, *S_bwd, *dS, *S_all, *Lam;
  size_t total;
};

LinBwdWs lin_bwd_ws(const vdn_config* c, void* base) {
  LinBwdWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    float* r = p ? reinterpret_cast<float*>(p + off) : nullptr;
    off += align256(bytes);
    return r;
  };
  const size_t mat = (size_t)128 * 128 * 4;
  const size_t BH = (size_t)c->B * c->H;
  const size_t frames = BH * c->T, blocks = BH * n_blocks(c);
  w.G = take(frames * mat);
  w.C = take(frames * mat);
  w.A = take(frames * mat);
  w.Bm = take(frames * mat);
  w.M = take(frames * mat);
  w.Cq = take(frames * mat);
  w.Gsym = take(frames * mat);   // also receives the unused q^T q of the stats call
  w.dC = take(frames * mat);
  w.dCt = take(frames * mat);
  w.S_fwd = take(blocks * mat);
  w.S_bwd = take(blocks * mat);
  w.dS = take(blocks * mat);
  w.S_all = take(frames * 2 * mat);
  w.Lam = take(frames * 2 * mat);
  w.total = off;
  return w;
}

// Workspace of the layer backward: dZ, the branch cotangents, the row
// statistics, then the linear-branch workspace.
struct BwdWs {
  void *dZ, *do_sm, *do_lin;
  float2* rowstat;
  void* lin;
  size_t lin_bytes;
  size_t total;
};

BwdWs bwd_ws(const vdn_config* c, void* base) {
  BwdWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const size_t rows = (size_t)c->B * c->H * tokens(c);
  w.dZ = take(rows * 2 * 128 * 2);
  w.do_sm = take(rows * 128 * 2);
  w.do_lin = take(rows * 128 * 2);
  w.rowstat = reinterpret_cast<float2*>(take(rows * sizeof(float2)));
  w.lin_bytes = lin_bwd_ws(c, nullptr).total;
  w.lin = take(w.lin_bytes);
  w.total = off;
  return w;
}

// Standalone softmax backward: row statistics and a head-major copy of do.
size_t softmax_bwd_ws_bytes(const vdn_config* c) {
  const size_t rows = (size_t)c->B * c->H * tokens(c);
  return align256(rows * sizeof(float2)) + align256(rows * 128 * 2);
}

// The backward paths need the bf16 tensor-core configuration.
vdn_status check_bwd_cfg(const vdn_config* cfg) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (cfg->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  return VDN_OK;
}

}  // namespace

extern "C" {

const char* vdn_last_error(void) { return g_last_error; }

const char* vdn_status_string(vdn_status s) {
  switch (s) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument";
    case VDN_ERR_UNSUPPORTED: return "unsupported configuration";
    case VDN_ERR_CUDA: return "CUDA error";
    case VDN_ERR_WORKSPACE: return "workspace missing or too small";
    case VDN_ERR_TIMEOUT: return "device wait timed out";
    case VDN_ERR_NUMERIC: return "non-positive Cholesky pivot";
  }
  return "unknown status";
}

vdn_status vdn_window_plan(const vdn_config* cfg, uint8_t* mask, int32_t* plan, size_t* plan_len) {
  if (!cfg || !plan_len) return VDN_ERR_INVALID_ARG;
  if (cfg->T < 1 || cfg->block_frames < 1 || cfg->window_blocks < 0 ||
      (cfg->anchors != 0 && cfg->anchors != 1))
    return VDN_ERR_INVALID_ARG;
  const int T = cfg->T;
  const std::vector<FrameSegment> segs =
      build_segments(T, cfg->block_frames, cfg->window_blocks, cfg->anchors);
  size_t need = 0;
  for (const auto& s : segs) need += 3 + 2 * s.nr;
  if (mask) {
    memset(mask, 0, (size_t)T * T);
    for (const auto& s : segs)
      for (int i = s.q0; i < s.q1; ++i)
        for (int r = 0; r < s.nr; ++r)
          for (int j = s.k0[r]; j < s.k1[r]; ++j) mask[(size_t)i * T + j] = 1;
  }
  if (plan) {
    if (*plan_len < need) {
      *plan_len = need;
      return VDN_ERR_INVALID_ARG;
    }
    size_t o = 0;
    for (const auto& s : segs) {
      plan[o++] = s.q0;
      plan[o++] = s.q1;
      plan[o++] = s.nr;
      for (int r = 0; r < s.nr; ++r) {
        plan[o++] = s.k0[r];
        plan[o++] = s.k1[r];
      }
    }
  }
  *plan_len = need;
  return VDN_OK;
}

size_t vdn_workspace_size(const vdn_config* cfg, int kind) {
  if (check_cfg(cfg) != VDN_OK) return 0;
  switch (kind) {
    case VDN_WS_SCAN: return scan_ws_bytes(cfg);
    case VDN_WS_SOFTMAX: return 256;
    case VDN_WS_LAYER: return layer_ws(cfg, nullptr).total;
    case VDN_WS_QUANT: return align256((size_t)cfg->B * cfg->H * 4);
    case VDN_WS_LAYER_FP8:
      return cfg->dtype == VDN_BF16 ? layer_ws(cfg, nullptr, true).total : 0;
    case VDN_WS_SOFTMAX_BWD: return cfg->dtype == VDN_BF16 ? softmax_bwd_ws_bytes(cfg) : 0;
    case VDN_WS_LINEAR_BWD: return cfg->dtype == VDN_BF16 ? lin_bwd_ws(cfg, nullptr).total : 0;
    case VDN_WS_BACKWARD: return cfg->dtype == VDN_BF16 ? bwd_ws(cfg, nullptr).total : 0;
  }
  return 0;
}

vdn_status vda_frame_stats(const vdn_config* cfg, const void* k, const void* v, float* G, float* C,
                           void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!k || !v || !G || !C) return VDN_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(G) || !aligned16(C)) return VDN_ERR_INVALID_ARG;
  const int BH = cfg->B * cfg->H;
  const unsigned frames = (unsigned)BH * cfg->T;
  cudaStream_t s = as_stream(stream);
  if (cfg->dtype == VDN_BF16) {
    CUtensorMap tk, tv;
    const cuuint64_t dims[4] = {128, (cuuint64_t)cfg->N, (cuuint64_t)cfg->T, (cuuint64_t)BH};
    const cuuint64_t str[3] = {256, (cuuint64_t)cfg->N * 256, (cuuint64_t)tokens(cfg) * 256};
    const cuuint32_t box[4] = {64, 64, 1, 1};
    if (!make_map(&tk, k, 4, dims, str, box) || !make_map(&tv, v, 4, dims, str, box))
      return cuda_fail("frame_stats tensor map", cudaErrorInvalidValue);
    return check("frame_stats launch",
                 launch_frame_stats_bf16(tk, tv, G, C, (int)frames, cfg->T, cfg->N, s));
  } else {
    const size_t sm = (size_t)32 * (cfg->d + cfg->dv) * 4;
    frame_stats_f32_kernel<<<frames, 256, sm, s>>>(static_cast<const float*>(k),
                                                   static_cast<const float*>(v), G, C, cfg->T,
                                                   cfg->N, cfg->d, cfg->dv);
  }
  return launch_status("frame_stats launch");
}

vdn_status vda_bidir_scan(const vdn_config* cfg, const float* G, const float* C, float* S_fwd,
                          float* S_bwd, void* ws, size_t ws_bytes, int32_t* dev_status,
                          void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!G || !C || !S_fwd || !S_bwd) return VDN_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(C) || !aligned16(S_fwd) || !aligned16(S_bwd))
    return VDN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < scan_ws_bytes(cfg) || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const int BH = cfg->B * cfg->H;
  const size_t frames = (size_t)BH * cfg->T;
  float* Aall = static_cast<float*>(ws);
  float* Ball = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         align256(frames * cfg->d * cfg->d * 4));
  st = check("frame_solve launch",
             launch_frame_solve(G, C, Aall, Ball, nullptr, (unsigned)frames, cfg->T, cfg->d,
                                cfg->dv, cfg->lambda, cfg->beta, cfg->anchors, dev_status, s));
  if (st != VDN_OK) return st;
  dim3 grid(BH, 2, (cfg->dv + kStateScanRows - 1) / kStateScanRows);
  const size_t scan_sm = scan_smem_bytes(cfg->d);
  st = set_smem((const void*)bidir_scan_kernel, scan_sm, "bidir_scan smem attribute");
  if (st != VDN_OK) return st;
  bidir_scan_kernel<<<grid, kScanThreads, scan_sm, s>>>(Aall, Ball, S_fwd, S_bwd, nullptr, cfg->T,
                                                        cfg->d,
                                                        cfg->dv, cfg->block_frames,
                                                        cfg->window_blocks, cfg->anchors,
                                                        n_blocks(cfg), dev_status);
  return launch_status("bidir_scan launch");
}

vdn_status vda_bidir_scan_noalloc(const vdn_config* cfg, const float* G, const float* C,
                                  float* S_fwd, float* S_bwd, int32_t* dev_status,
                                  void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!G || !C || !S_fwd || !S_bwd) return VDN_ERR_INVALID_ARG;
  const size_t need = scan_ws_bytes(cfg);
  if (need > noalloc_scratch_bytes()) {
    snprintf(g_last_error, sizeof(g_last_error),
             "vda_bidir_scan_noalloc: needs %zu bytes of scratch, the library holds %zu", need,
             noalloc_scratch_bytes());
    return VDN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  st = check("no-allocation scratch address", noalloc_scratch(&scratch));
  if (st != VDN_OK) return st;
  return vda_bidir_scan(cfg, G, C, S_fwd, S_bwd, scratch, noalloc_scratch_bytes(), dev_status,
                        stream);
}

vdn_status vda_readout(const vdn_config* cfg, const void* q, const float* S_fwd,
                       const float* S_bwd, void* o_lin, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !S_fwd || !S_bwd || !o_lin) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(S_fwd) || !aligned16(S_bwd) || !aligned16(o_lin))
    return VDN_ERR_INVALID_ARG;
  if (cfg->dtype == VDN_BF16) {
    CUtensorMap tq;
    const cuuint64_t dims[3] = {128, (cuuint64_t)tokens(cfg), (cuuint64_t)cfg->B * cfg->H};
    const cuuint64_t str[2] = {256, (cuuint64_t)tokens(cfg) * 256};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!make_map(&tq, q, 3, dims, str, box))
      return cuda_fail("readout tensor map", cudaErrorInvalidValue);
    return check("readout launch",
                 launch_readout_bf16(tq, S_fwd, S_bwd, o_lin, cfg->B, cfg->H, cfg->T, cfg->N,
                                     cfg->block_frames, cfg->anchors, n_blocks(cfg), cfg->n_ctx,
                                     token_major_out(cfg, 1, 0), false, nullptr, nullptr,
                                     as_stream(stream)));
  }
  return check("readout launch",
               launch_readout_f32(q, S_fwd, S_bwd, o_lin, cfg->B, cfg->H, cfg->T, cfg->N,
                                  cfg->d, cfg->dv, cfg->block_frames, cfg->anchors, n_blocks(cfg),
                                  (long)cfg->H * cfg->dv, 0, nullptr, as_stream(stream)));
}

vdn_status vda_readout_gated(const vdn_config* cfg, const void* q, const float* S_fwd,
                             const float* S_bwd, const float* gate_logits, void* Z,
                             void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !S_fwd || !S_bwd || !gate_logits || !Z) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(S_fwd) || !aligned16(S_bwd) || !aligned16(Z))
    return VDN_ERR_INVALID_ARG;
  const long hs = (long)cfg->H * cfg->dv;
  if (cfg->dtype == VDN_BF16) {
    CUtensorMap tq;
    const cuuint64_t dims[3] = {128, (cuuint64_t)tokens(cfg), (cuuint64_t)cfg->B * cfg->H};
    const cuuint64_t str[2] = {256, (cuuint64_t)tokens(cfg) * 256};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!make_map(&tq, q, 3, dims, str, box))
      return cuda_fail("readout tensor map", cudaErrorInvalidValue);
    return check("readout launch",
                 launch_readout_bf16(tq, S_fwd, S_bwd, Z, cfg->B, cfg->H, cfg->T, cfg->N,
                                     cfg->block_frames, cfg->anchors, n_blocks(cfg), cfg->n_ctx,
                                     token_major_out(cfg, 2, hs), false,
                                     gate_logits, nullptr, as_stream(stream)));
  }
  return check("readout launch",
               launch_readout_f32(q, S_fwd, S_bwd, Z, cfg->B, cfg->H, cfg->T, cfg->N, cfg->d,
                                  cfg->dv, cfg->block_frames, cfg->anchors, n_blocks(cfg), 2 * hs,
                                  hs, gate_logits, as_stream(stream)));
}

vdn_status vdn_softmax_window(const vdn_config* cfg, const void* q, const void* k, const void* v,
                              const float* S_fwd, const float* S_bwd, const float* gate_logits,
                              void* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                              void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !out) return VDN_ERR_INVALID_ARG;
  const bool fused = S_fwd != nullptr;
  if (fused != (S_bwd != nullptr) || (fused && !gate_logits)) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return VDN_ERR_INVALID_ARG;
  if (fused && (!aligned16(S_fwd) || !aligned16(S_bwd))) return VDN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256) return VDN_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)cfg->d);
  const int BH = cfg->B * cfg->H;
  const int T = cfg->T, N = cfg->N, bf = cfg->block_frames;
  if (cfg->dtype == VDN_F32) {
    const long long rows = (long long)BH * tokens(cfg);
    const unsigned grid = (unsigned)((rows + 7) / 8);
    softmax_window_f32_kernel<<<grid, 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        S_fwd, S_bwd, gate_logits, static_cast<float*>(out), cfg->B, cfg->H, T, N, cfg->d, cfg->dv,
        bf, cfg->window_blocks, cfg->anchors, n_blocks(cfg), scale);
    return launch_status("softmax_f32 launch");
  }

  // bf16 tensor-core path
  CUtensorMap tq, tk, tv;
  const cuuint64_t dims[3] = {128, (cuuint64_t)tokens(cfg), (cuuint64_t)BH};
  const cuuint64_t str[2] = {256, (cuuint64_t)tokens(cfg) * 256};
  const cuuint32_t box[3] = {64, 128, 1};
  if (!make_map(&tq, q, 3, dims, str, box) || !make_map(&tk, k, 3, dims, str, box) ||
      !make_map(&tv, v, 3, dims, str, box))
    return cuda_fail("softmax tensor map", cudaErrorInvalidValue);
  st = launch_softmax_tc(cfg, tq, tk, tv, false, scale, gate_logits, nullptr, nullptr, nullptr,
                         out, ws, dev_status, s);
  if (st != VDN_OK) return st;
  if (fused) {
    // the linear half of Z: (1 - g) (S_fwd + S_bwd) q, read through the same
    // query tensor map
    const long hs = (long)cfg->H * 128;
    st = check("readout launch",
               launch_readout_bf16(tq, S_fwd, S_bwd, out, cfg->B, cfg->H, T, N, bf, cfg->anchors,
                                   n_blocks(cfg), cfg->n_ctx, token_major_out(cfg, 2, hs), false,
                                   gate_logits, dev_status, s));
    if (st != VDN_OK) return st;
  }
  return VDN_OK;
}

// The bf16 merge Y = Z [W1; W2] over M = B * (tokens per batch) rows; Z is
// plain [M, 2, H, dv] (groups = 0) or the head-sharded layer's received
// layout [B, groups, Ls, 2, H / groups, dv].
static vdn_status merge_bf16(const vdn_config* cfg, int groups, const void* Z, const void* W1,
                             const void* W2, void* Y, cudaStream_t s) {
  if (cfg->w_per_head) return VDN_ERR_UNSUPPORTED;
  if (cfg->d_out % 8) return VDN_ERR_UNSUPPORTED;
  const long long Ls = tokens(cfg);
  const long long M = (long long)cfg->B * Ls;
  if (M > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  const int K1 = cfg->H * cfg->dv;
  MergeGroups grp{0, 0, 0, 0};
  CUtensorMap tz, tw1, tw2;
  if (groups == 1) groups = 0;   // one group is the plain layout
  if (groups == 0) {
    const cuuint64_t dims[2] = {(cuuint64_t)2 * K1, (cuuint64_t)M};
    const cuuint64_t str[1] = {(cuuint64_t)2 * K1 * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!make_map(&tz, Z, 2, dims, str, box)) return cuda_fail("merge tensor map", cudaErrorInvalidValue);
  } else {
    grp = MergeGroups{groups, cfg->H / groups, cfg->dv / 64, (int)Ls};
    const cuuint64_t seg = (cuuint64_t)2 * grp.Hs * cfg->dv;   // K elements per group
    // (batch item, group) pairs are evenly spaced: one dimension b * G + g
    const cuuint64_t dims[3] = {seg, (cuuint64_t)Ls, (cuuint64_t)groups * cfg->B};
    const cuuint64_t str[2] = {seg * 2, seg * 2 * Ls};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!make_map(&tz, Z, 3, dims, str, box)) return cuda_fail("merge tensor map", cudaErrorInvalidValue);
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)cfg->d_out, (cuuint64_t)K1};
    const cuuint64_t str[1] = {(cuuint64_t)cfg->d_out * 2};
    const cuuint32_t box[2] = {64, 64};
    if (!make_map(&tw1, W1, 2, dims, str, box) || !make_map(&tw2, W2, 2, dims, str, box))
      return cuda_fail("merge tensor map", cudaErrorInvalidValue);
  }
  vdn_status st = set_smem((const void*)gated_merge_bf16_kernel, kMergeSmem, "merge smem attribute");
  if (st != VDN_OK) return st;
  const long long m_tiles = groups == 0 ? (M + 127) / 128 : (long long)cfg->B * ((Ls + 127) / 128);
  const long long tiles = m_tiles * (long long)((cfg->d_out + 255) / 256);
  if (tiles > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  if (tiles == 0) return VDN_OK;
  // persistent: one CTA per SM (or per tile, if fewer)
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  dim3 grid((unsigned)(tiles < sms ? tiles : sms));
  gated_merge_bf16_kernel<<<grid, kMergeThreads, kMergeSmem, s>>>(tz, tw1, tw2,
                                                             static_cast<__nv_bfloat16*>(Y), (int)M,
                                                             cfg->d_out, K1, grp, nullptr);
  return launch_status("merge launch");
}

vdn_status vdn_gated_merge(const vdn_config* cfg, const void* Z, const void* W1, const void* W2,
                           void* Y, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!Z || !W1 || !W2 || !Y || cfg->d_out < 1) return VDN_ERR_INVALID_ARG;
  if (cfg->w_per_head != 0 && cfg->w_per_head != 1) return VDN_ERR_INVALID_ARG;
  if (!aligned16(Z) || !aligned16(W1) || !aligned16(W2) || !aligned16(Y)) return VDN_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const long long M = (long long)cfg->B * tokens(cfg);
  if (cfg->dtype == VDN_F32) {
    const long long total = M * (cfg->w_per_head ? cfg->H : 1) * cfg->d_out;
    gated_merge_f32_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
        static_cast<const float*>(Z), static_cast<const float*>(W1), static_cast<const float*>(W2),
        static_cast<float*>(Y), (long)M, cfg->H, cfg->dv, cfg->d_out, cfg->w_per_head);
    return launch_status("merge_f32 launch");
  }
  return merge_bf16(cfg, 0, Z, W1, W2, Y, s);
}

vdn_status vdn_gated_merge_head_groups(const vdn_config* cfg, int n_groups, const void* Z,
                                       const void* W1, const void* W2, void* Y, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!Z || !W1 || !W2 || !Y || cfg->d_out < 1) return VDN_ERR_INVALID_ARG;
  if (n_groups < 1 || cfg->H % n_groups) return VDN_ERR_INVALID_ARG;
  if (!aligned16(Z) || !aligned16(W1) || !aligned16(W2) || !aligned16(Y)) return VDN_ERR_INVALID_ARG;
  if (cfg->dtype != VDN_BF16 || cfg->w_per_head || cfg->dv % 64) return VDN_ERR_UNSUPPORTED;
  return merge_bf16(cfg, n_groups, Z, W1, W2, Y, as_stream(stream));
}

vdn_status vdn_pack_head_groups(const vdn_config* cfg, int n_groups, const void* x, void* out,
                                void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!x || !out || n_groups < 1 || cfg->H % n_groups) return VDN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return VDN_ERR_INVALID_ARG;
  if (cfg->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  const long long rows = (long long)cfg->B * cfg->H * tokens(cfg);
  if (rows > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long need = (rows * 16 + 255) / 256;
  const int grid = (int)(need < 8LL * sms ? need : 8LL * sms);
  pack_head_groups_kernel<<<grid, 256, 0, as_stream(stream)>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(out), (int)rows, (int)tokens(cfg),
      cfg->H, cfg->H / n_groups, n_groups);
  return launch_status("pack_head_groups launch");
}

vdn_status vdn_hybrid_forward(const vdn_config* cfg, const void* q, const void* k, const void* v,
                              const float* gate_logits, const void* W1, const void* W2, void* Y,
                              void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !gate_logits || !W1 || !W2 || !Y) return VDN_ERR_INVALID_ARG;
  const LayerWs w0 = layer_ws(cfg, nullptr);
  if (!ws || ws_bytes < w0.total || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  const LayerWs w = layer_ws(cfg, ws);
  st = vda_frame_stats(cfg, k, v, w.G, w.C, stream);
  if (st != VDN_OK) return st;
  st = vda_bidir_scan(cfg, w.G, w.C, w.S_fwd, w.S_bwd, w.scan_ws, w.scan_bytes, dev_status, stream);
  if (st != VDN_OK) return st;
  st = vdn_softmax_window(cfg, q, k, v, w.S_fwd, w.S_bwd, gate_logits, w.Z, w.sm_ws, w.sm_bytes,
                          dev_status, stream);
  if (st != VDN_OK) return st;
  return vdn_gated_merge(cfg, w.Z, W1, W2, Y, stream);
}

vdn_status vdn_quantize_fp8(const vdn_config* cfg, const void* x, void* x8, float* scale,
                            void* ws, size_t ws_bytes, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (cfg->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  if (!x || !x8 || !scale) return VDN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || reinterpret_cast<uintptr_t>(scale) % 4 != 0)
    return VDN_ERR_INVALID_ARG;
  const int BH = cfg->B * cfg->H;
  if (!ws || ws_bytes < (size_t)BH * 4 || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  return check("quantize launch",
               launch_quantize_fp8(x, (long)tokens(cfg) * cfg->d, BH, x8, scale,
                                   static_cast<uint32_t*>(ws), sm_count(), as_stream(stream)));
}

vdn_status vdn_softmax_window_fp8(const vdn_config* cfg, const void* q8, const void* k8,
                                  const void* v8, const float* q_scale, const float* k_scale,
                                  const float* v_scale, const float* gate_logits, void* out,
                                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (cfg->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  if (!q8 || !k8 || !v8 || !q_scale || !k_scale || !v_scale || !out) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(out))
    return VDN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256) return VDN_ERR_WORKSPACE;
  const int BH = cfg->B * cfg->H;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)cfg->d);
  CUtensorMap tq, tk, tv;
  const cuuint64_t dims[3] = {128, (cuuint64_t)tokens(cfg), (cuuint64_t)BH};
  const cuuint64_t str[2] = {128, (cuuint64_t)tokens(cfg) * 128};
  const cuuint32_t box[3] = {128, 128, 1};
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (!make_map(&tq, q8, 3, dims, str, box, u8) || !make_map(&tk, k8, 3, dims, str, box, u8) ||
      !make_map(&tv, v8, 3, dims, str, box, u8))
    return cuda_fail("softmax fp8 tensor map", cudaErrorInvalidValue);
  return launch_softmax_tc(cfg, tq, tk, tv, true, scale, gate_logits, q_scale, k_scale, v_scale,
                           out, ws, dev_status, as_stream(stream));
}

vdn_status vdn_hybrid_forward_fp8(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, const float* gate_logits, const void* W1,
                                  const void* W2, void* Y, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, void* stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (cfg->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !gate_logits || !W1 || !W2 || !Y) return VDN_ERR_INVALID_ARG;
  const LayerWs w0 = layer_ws(cfg, nullptr, true);
  if (!ws || ws_bytes < w0.total || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  const LayerWs w = layer_ws(cfg, ws, true);
  const int BH = cfg->B * cfg->H;
  st = vda_frame_stats(cfg, k, v, w.G, w.C, stream);
  if (st != VDN_OK) return st;
  st = vda_bidir_scan(cfg, w.G, w.C, w.S_fwd, w.S_bwd, w.scan_ws, w.scan_bytes, dev_status, stream);
  if (st != VDN_OK) return st;
  const void* src[3] = {q, k, v};
  void* dst[3] = {w.q8, w.k8, w.v8};
  for (int i = 0; i < 3; ++i) {
    st = vdn_quantize_fp8(cfg, src[i], dst[i], w.scales + i * BH, w.amax, (size_t)BH * 4, stream);
    if (st != VDN_OK) return st;
  }
  st = vdn_softmax_window_fp8(cfg, w.q8, w.k8, w.v8, w.scales, w.scales + BH, w.scales + 2 * BH,
                              gate_logits, w.Z, w.sm_ws, w.sm_bytes, dev_status, stream);
  if (st != VDN_OK) return st;
  st = vda_readout_gated(cfg, q, w.S_fwd, w.S_bwd, gate_logits, w.Z, stream);
  if (st != VDN_OK) return st;
  return vdn_gated_merge(cfg, w.Z, W1, W2, Y, stream);
}

vdn_status vdn_softmax_window_lse(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, void* o_sm, float* lse, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !o_sm || !lse) return VDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_sm) || !aligned16(lse))
    return VDN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256) return VDN_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv;
  if (!head_major_map(&tq, q, cfg) || !head_major_map(&tk, k, cfg) || !head_major_map(&tv, v, cfg))
    return cuda_fail("softmax tensor map", cudaErrorInvalidValue);
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)cfg->d);
  return launch_softmax_tc(cfg, tq, tk, tv, false, scale, nullptr, nullptr, nullptr, nullptr, o_sm,
                           ws, dev_status, as_stream(stream), lse);
}

vdn_status vdn_softmax_window_bwd(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, const void* o_sm, const float* lse,
                                  const void* do_sm, void* dq, void* dk, void* dv, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !o_sm || !lse || !do_sm || !dq || !dk || !dv) return VDN_ERR_INVALID_ARG;
  const void* ptrs[9] = {q, k, v, o_sm, lse, do_sm, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return VDN_ERR_INVALID_ARG;
  const size_t rows = (size_t)cfg->B * cfg->H * tokens(cfg);
  if (!ws || ws_bytes < softmax_bwd_ws_bytes(cfg) || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  float2* rowstat = static_cast<float2*>(ws);
  void* do_hm = static_cast<uint8_t*>(ws) + align256(rows * sizeof(float2));
  st = check("rowstat launch", launch_rowstat(o_sm, do_sm, lse, rowstat, do_hm, cfg->B, cfg->H,
                                              (long)tokens(cfg), sm_count(), s));
  if (st != VDN_OK) return st;
  return launch_softmax_bwd(cfg, q, k, v, do_hm, rowstat, dq, dk, dv, false, dev_status, s);
}

vdn_status vda_linear_bwd(const vdn_config* cfg, const void* q, const void* k, const void* v,
                          const void* do_lin, void* dq, void* dk, void* dv, void* ws,
                          size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !do_lin || !dq || !dk || !dv) return VDN_ERR_INVALID_ARG;
  const void* ptrs[7] = {q, k, v, do_lin, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return VDN_ERR_INVALID_ARG;
  const LinBwdWs w0 = lin_bwd_ws(cfg, nullptr);
  if (!ws || ws_bytes < w0.total || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  const LinBwdWs w = lin_bwd_ws(cfg, ws);
  cudaStream_t s = as_stream(stream);
  const int BH = cfg->B * cfg->H, T = cfg->T, nb = n_blocks(cfg);
  const unsigned frames = (unsigned)BH * T;
  // forward quantities: G, C; A, B and M; the states before every frame
  st = vda_frame_stats(cfg, k, v, w.G, w.C, stream);
  if (st != VDN_OK) return st;
  st = check("frame_solve launch",
             launch_frame_solve(w.G, w.C, w.A, w.Bm, w.M, frames, T, 128, 128, cfg->lambda,
                                cfg->beta, cfg->anchors, dev_status, s));
  if (st != VDN_OK) return st;
  const size_t scan_sm = scan_smem_bytes(128);
  st = set_smem((const void*)bidir_scan_kernel, scan_sm, "bidir_scan smem attribute");
  if (st != VDN_OK) return st;
  bidir_scan_kernel<<<dim3(BH, 2, 128 / kStateScanRows), kScanThreads, scan_sm, s>>>(
      w.A, w.Bm, w.S_fwd, w.S_bwd, w.S_all, T, 128, 128, cfg->block_frames, cfg->window_blocks,
      cfg->anchors, nb, dev_status);
  st = launch_status("bidir_scan launch");
  if (st != VDN_OK) return st;
  // dq = (S_fwd + S_bwd)^T do, head-major; zero rows for anchors and context
  CUtensorMap tdo, tk, tv;
  if (!head_major_map(&tdo, do_lin, cfg) || !head_major_map(&tk, k, cfg) ||
      !head_major_map(&tv, v, cfg))
    return cuda_fail("linear backward tensor map", cudaErrorInvalidValue);
  const long L = (long)tokens(cfg);
  const ReadoutOut hm{(long)cfg->H * L * 128, 128, L * 128, 0};
  st = check("readout (dq) launch",
             launch_readout_bf16(tdo, w.S_fwd, w.S_bwd, dq, cfg->B, cfg->H, T, cfg->N,
                                 cfg->block_frames, cfg->anchors, nb, cfg->n_ctx, hm, true,
                                 nullptr, dev_status, s));
  if (st != VDN_OK) return st;
  // per-frame do^T q (the q^T q half of the call is not used)
  st = vda_frame_stats(cfg, q, do_lin, w.Gsym, w.Cq, stream);
  if (st != VDN_OK) return st;
  LinearBwdLaunch p{};
  p.BH = BH;
  p.T = T;
  p.N = cfg->N;
  p.n_ctx = cfg->n_ctx;
  p.nb = nb;
  p.bf = cfg->block_frames;
  p.W = cfg->window_blocks;
  p.anchors = cfg->anchors;
  p.lambda = cfg->lambda;
  p.beta = cfg->beta;
  p.Cq = w.Cq;
  p.dS = w.dS;
  p.A = w.A;
  p.Lam_all = w.Lam;
  p.S_all = w.S_all;
  p.C = w.C;
  p.M = w.M;
  p.Gsym = w.Gsym;
  p.dC = w.dC;
  p.dCt = w.dCt;
  p.tm_k = &tk;
  p.tm_v = &tv;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dev_status = dev_status;
  return check("linear backward launch", launch_linear_bwd_kernels(p, s));
}

vdn_status vdn_gated_merge_bwd(const vdn_config* cfg, const void* Z, const void* W1,
                               const void* W2, const void* dY, void* dZ, float* dW1, float* dW2,
                               int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!Z || !W1 || !W2 || !dY || !dZ || !dW1 || !dW2 || cfg->d_out < 1) return VDN_ERR_INVALID_ARG;
  if (cfg->w_per_head) return VDN_ERR_UNSUPPORTED;
  if (cfg->d_out % 8) return VDN_ERR_UNSUPPORTED;
  const void* ptrs[7] = {Z, W1, W2, dY, dZ, dW1, dW2};
  for (const void* p : ptrs)
    if (!aligned16(p)) return VDN_ERR_INVALID_ARG;
  const long long M = (long long)cfg->B * tokens(cfg);
  if (M > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  const int K1 = cfg->H * 128;
  cudaStream_t s = as_stream(stream);
  st = check("merge dgrad launch",
             launch_merge_dgrad(dY, W1, W2, dZ, (long)M, cfg->d_out, K1, dev_status, s));
  if (st != VDN_OK) return st;
  const size_t wbytes = (size_t)K1 * cfg->d_out * 4;
  st = check("dW reset", cudaMemsetAsync(dW1, 0, wbytes, s));
  if (st == VDN_OK) st = check("dW reset", cudaMemsetAsync(dW2, 0, wbytes, s));
  if (st != VDN_OK) return st;
  return check("merge wgrad launch",
               launch_merge_wgrad(Z, dY, dW1, dW2, (long)M, cfg->d_out, K1, dev_status, s));
}

vdn_status vdn_hybrid_forward_train(const vdn_config* cfg, const void* q, const void* k,
                                    const void* v, const float* gate_logits, const void* W1,
                                    const void* W2, void* Y, void* Z, float* lse, void* ws,
                                    size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !gate_logits || !W1 || !W2 || !Y || !Z || !lse) return VDN_ERR_INVALID_ARG;
  if (!aligned16(Z) || !aligned16(lse) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return VDN_ERR_INVALID_ARG;
  const LayerWs w0 = layer_ws(cfg, nullptr);
  if (!ws || ws_bytes < w0.total || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  const LayerWs w = layer_ws(cfg, ws);
  cudaStream_t s = as_stream(stream);
  st = vda_frame_stats(cfg, k, v, w.G, w.C, stream);
  if (st != VDN_OK) return st;
  st = vda_bidir_scan(cfg, w.G, w.C, w.S_fwd, w.S_bwd, w.scan_ws, w.scan_bytes, dev_status, stream);
  if (st != VDN_OK) return st;
  CUtensorMap tq, tk, tv;
  if (!head_major_map(&tq, q, cfg) || !head_major_map(&tk, k, cfg) || !head_major_map(&tv, v, cfg))
    return cuda_fail("softmax tensor map", cudaErrorInvalidValue);
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)cfg->d);
  st = launch_softmax_tc(cfg, tq, tk, tv, false, scale, gate_logits, nullptr, nullptr, nullptr, Z,
                         w.sm_ws, dev_status, s, lse);
  if (st != VDN_OK) return st;
  const long hs = (long)cfg->H * 128;
  st = check("readout launch",
             launch_readout_bf16(tq, w.S_fwd, w.S_bwd, Z, cfg->B, cfg->H, cfg->T, cfg->N,
                                 cfg->block_frames, cfg->anchors, n_blocks(cfg), cfg->n_ctx,
                                 token_major_out(cfg, 2, hs), false, gate_logits, dev_status, s));
  if (st != VDN_OK) return st;
  return vdn_gated_merge(cfg, Z, W1, W2, Y, stream);
}

vdn_status vdn_hybrid_backward(const vdn_config* cfg, const void* q, const void* k, const void* v,
                               const float* gate_logits, const void* W1, const void* W2,
                               const void* Z, const float* lse, const void* dY, void* dq,
                               void* dk, void* dv, float* dgate_logits, float* dW1, float* dW2,
                               void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!q || !k || !v || !gate_logits || !W1 || !W2 || !Z || !lse || !dY || !dq || !dk || !dv ||
      !dgate_logits || !dW1 || !dW2)
    return VDN_ERR_INVALID_ARG;
  if (!aligned16(lse)) return VDN_ERR_INVALID_ARG;
  const BwdWs w0 = bwd_ws(cfg, nullptr);
  if (!ws || ws_bytes < w0.total || !aligned16(ws)) return VDN_ERR_WORKSPACE;
  const BwdWs w = bwd_ws(cfg, ws);
  cudaStream_t s = as_stream(stream);
  // merge: dZ, dW1, dW2
  st = vdn_gated_merge_bwd(cfg, Z, W1, W2, dY, w.dZ, dW1, dW2, dev_status, stream);
  if (st != VDN_OK) return st;
  // branch cotangents, row statistics and the gate
  st = check("dgate reset", cudaMemsetAsync(dgate_logits, 0, (size_t)cfg->H * 4, s));
  if (st != VDN_OK) return st;
  st = check("backward prep launch",
             launch_bwd_prep(w.dZ, Z, gate_logits, lse, w.do_sm, w.do_lin, w.rowstat, dgate_logits,
                             cfg->B, cfg->H, (long)tokens(cfg), sm_count(), s));
  if (st != VDN_OK) return st;
  // linear branch (writes dq, dk, dv), then the softmax branch on top
  st = vda_linear_bwd(cfg, q, k, v, w.do_lin, dq, dk, dv, w.lin, w.lin_bytes, dev_status, stream);
  if (st != VDN_OK) return st;
  return launch_softmax_bwd(cfg, q, k, v, w.do_sm, w.rowstat, dq, dk, dv, true, dev_status, s);
}

vdn_status vdn_selftest_timeout(int32_t* dev_status, int limit_ms, void* stream) {
  if (!dev_status || limit_ms < 1 || limit_ms > 10000) return VDN_ERR_INVALID_ARG;
  return check("selftest launch", launch_wait_timeout(dev_status, limit_ms, as_stream(stream)));
}

vdn_status vdn_read_status(int32_t* dev_status, void* stream) {
  if (!dev_status) return VDN_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  int32_t h = 0;
  vdn_status st = check("status copy", cudaMemcpyAsync(&h, dev_status, sizeof(h),
                                                     cudaMemcpyDeviceToHost, s));
  if (st == VDN_OK) st = check("status reset", cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s));
  if (st == VDN_OK) st = check("status synchronize", cudaStreamSynchronize(s));
  if (st != VDN_OK) return st;
  if (h < 0 || h > VDN_ERR_NUMERIC) return VDN_ERR_CUDA;
  return static_cast<vdn_status>(h);
}

}  // extern "C"
