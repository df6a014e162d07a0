/*
 * vdn.h - C ABI of the Video DeltaNet (VDN) hybrid attention layer,
 * video-to-video forward pass, on NVIDIA B200 (sm_100a).
 *
 * Source pages: "Video DeltaNet: A Video-Native Hybrid Attention for
 * Livestream Video Generation" (mlsanity index page, abstract), the
 * besthub.dev article on VDN-H3 (sections "Hybrid Attention Architecture" and
 * "Video Delta Attention (VDA)"), the sd114.wiki article on VDN-Minimax-H3
 * (sections on the bidirectional sliding-window softmax branch and the
 * bidirectional linear branch) and the flyP critical read (method breakdown).
 *
 * Notation. Per batch item b and head h: K_f, Q_f are the N x d rows of
 * latent frame f, V_f the N x dv rows; token index t = f*N + n (n = row-major
 * position in the spatial grid); L = T*N + n_ctx tokens per (b, h), the
 * n_ctx context tokens (text / audio, see vdn_config) last. Frame f lies in block
 * f / block_frames; nb = ceil(T / block_frames). The VDA closed form used
 * throughout (the pages state only that the update is per frame, joint over
 * the frame's tokens and non-expansive):
 *     G_f = K_f^T K_f, C_f = V_f^T K_f, M_f = (G_f + lambda I)^-1,
 *     S <- S (I - beta G_f M_f) + beta C_f M_f,  output (S_fwd + S_bwd) q.
 *
 * Conventions for every entry point:
 *  - `cfg` is a host pointer. Every other tensor pointer is a DEVICE pointer
 *    (cudaMalloc / torch CUDA memory) with a 16-byte aligned base, dense
 *    row-major in the layout given. The caller owns all memory; the library
 *    allocates nothing and keeps no state between calls (the one exception,
 *    vda_bidir_scan_noalloc, says so), so calls are re-entrant and may be
 *    captured in a CUDA graph.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Work is enqueued asynchronously on it.
 *  - Validation is synchronous: a non-VDN_OK status is returned before
 *    anything is launched. A launch failure returns VDN_ERR_CUDA.
 *  - Conditions found on the device (a bounded wait that ran out, a
 *    non-positive Cholesky pivot) are written to `dev_status` (a device
 *    int32, zero on entry) and read back by vdn_read_status().
 *  - dtype VDN_BF16: q, k, v, W1, W2 and every non-fp32 output are bf16
 *    (round to nearest even), d = dv = 128. dtype VDN_F32: they are fp32,
 *    d and dv are powers of two from 8 to 128. G, C, S_fwd, S_bwd and the gate
 *    logits are fp32 in both cases.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, bad parameter */
  VDN_ERR_UNSUPPORTED = 2, /* valid but not built: e.g. bf16 with d != 128 */
  VDN_ERR_CUDA = 3,        /* a CUDA call or launch failed */
  VDN_ERR_WORKSPACE = 4,   /* ws is NULL or ws_bytes < vdn_workspace_size() */
  VDN_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out (pipeline stall) */
  VDN_ERR_NUMERIC = 6      /* device: a Cholesky pivot of G_f + lambda I was not > 0 */
} vdn_status;

typedef enum { VDN_F32 = 0, VDN_BF16 = 1 } vdn_dtype;

typedef struct vdn_config {
  int32_t B, H;           /* batch items, heads */
  int32_t T, N;           /* latent frames, spatial tokens per frame */
  int32_t d, dv;          /* query/key dim, value dim */
  int32_t block_frames;   /* frames per block (5 on the pages) */
  int32_t window_blocks;  /* a block attends blocks b-w .. b+w (1 on the pages) */
  int32_t anchors;        /* 1: first/last-frame anchors on (the pages), 0: off */
  int32_t dtype;          /* vdn_dtype */
  float lambda;           /* ridge term, > 0 */
  float beta;             /* step, 0 < beta <= 1 */
  float softmax_scale;    /* score scale; 0 means 1/sqrt(d) */
  int32_t d_out;          /* merge output width */
  int32_t w_per_head;     /* 1: W1, W2 are dv x d_out shared by all heads (fp32 only) */
  int32_t n_ctx;          /* context (text / audio) tokens after the video tokens; 0: none */
} vdn_config;

/*
 * Token layout. Each (b, h) holds L = T*N + n_ctx tokens: the T*N video
 * tokens (token f*N + n is spatial token n of frame f), then n_ctx context
 * tokens. Every [.., L, ..] dimension below has this length. mlsanity
 * abstract: the hybrid applies to video-to-video interactions only, and
 * interactions involving text or audio keep softmax; so a video query
 * attends its window and anchor frames plus every context token in one
 * softmax, a context query attends every token, the linear branch (frame
 * statistics, scan) uses the video tokens only, and o_lin = 0 on context
 * rows. n_ctx > 0 needs dtype bf16.
 */

/* Workspace kinds for vdn_workspace_size(). */
enum { VDN_WS_SCAN = 1, VDN_WS_SOFTMAX = 2, VDN_WS_LAYER = 3, VDN_WS_QUANT = 4,
       VDN_WS_LAYER_FP8 = 5, VDN_WS_SOFTMAX_BWD = 6, VDN_WS_LINEAR_BWD = 7,
       VDN_WS_BACKWARD = 8 };

/*
 * vdn_window_plan - the softmax branch's frame mask and query segments (host).
 * sd114.wiki, bidirectional sliding-window softmax branch: frames are packed
 * into blocks of block_frames; frame i attends frame j when
 * |i/bf - j/bf| <= window_blocks, or (anchors) when j or i is 0 or T-1.
 *   mask      host uint8 [T*T], mask[i*T + j]; may be NULL.
 *   plan      host int32 buffer; may be NULL to query the length. For each
 *             query segment (a maximal run of frames of one block with equal
 *             mask rows): q_f0, q_f1, n_ranges, then n_ranges pairs
 *             k_f0, k_f1 (maximal runs of ones of the row), frames [f0, f1).
 *   plan_len  in: capacity of plan in int32 elements; out: length used.
 * Returns VDN_ERR_INVALID_ARG if plan is too short (plan_len then holds the
 * needed length). Only T, block_frames, window_blocks, anchors are read.
 */
vdn_status vdn_window_plan(const vdn_config* cfg, uint8_t* mask, int32_t* plan,
                           size_t* plan_len);

/* Bytes of device workspace an operation needs (0 on an invalid cfg).
 * VDN_WS_SCAN: vda_bidir_scan; VDN_WS_SOFTMAX: vdn_softmax_window and
 * vdn_softmax_window_fp8; VDN_WS_LAYER: vdn_hybrid_forward (includes G, C,
 * S_fwd, S_bwd, Z); VDN_WS_QUANT: vdn_quantize_fp8; VDN_WS_LAYER_FP8:
 * vdn_hybrid_forward_fp8 (the layer's plus the e4m3 copies of q, k, v);
 * VDN_WS_SOFTMAX_BWD: vdn_softmax_window_bwd; VDN_WS_LINEAR_BWD:
 * vda_linear_bwd; VDN_WS_BACKWARD: vdn_hybrid_backward. The three backward
 * kinds return 0 unless dtype is bf16. */
size_t vdn_workspace_size(const vdn_config* cfg, int kind);

/*
 * vda_frame_stats - per-frame sums of the VDA update (besthub.dev, "Video
 * Delta Attention (VDA)": all spatial tokens of a frame jointly solve one
 * state update).
 *   k  [B,H,L,d], v [B,H,L,dv] (dtype)
 *   G  [B,H,T,d,d]  fp32 out, G_f = K_f^T K_f
 *   C  [B,H,T,dv,d] fp32 out, C_f = V_f^T K_f
 * bf16: tensor-core products with fp32 accumulation; f32: fp64 accumulation.
 */
vdn_status vda_frame_stats(const vdn_config* cfg, const void* k, const void* v, float* G,
                           float* C, void* stream);

/*
 * vda_bidir_scan - per-frame solve and bidirectional scan of the VDA states
 * (sd114.wiki, bidirectional linear branch: for frame i the forward state
 * summarises the frames before i's window, the backward state the frames
 * after it; the ranges exclude the window and the anchor frames).
 * Per frame f (anchor frames excluded): M_f = (G_f + lambda I)^-1 in fp64
 * by the symmetric sweep (Gauss-Jordan in symmetric form: a square-root-free
 * Cholesky, LDL^T, elimination carried to the inverse; its pivots are the
 * squared Cholesky diagonal), A_f = I - beta G_f M_f = (1-beta) I +
 * beta lambda M_f, B_f = beta C_f M_f. Then S <- S A_f + B_f applied from
 * S = 0 in increasing frame order (forward) and in decreasing order
 * (backward), the state held in fp32.
 *   G, C     as produced by vda_frame_stats
 *   S_fwd    [B,H,nb,dv,d] fp32 out: state after frames [0, ws(b)), where
 *            ws(b) = max(0, (b - window_blocks) * block_frames)
 *   S_bwd    [B,H,nb,dv,d] fp32 out: state after frames [we(b), T) taken in
 *            decreasing order, we(b) = min(T, (b + window_blocks + 1) * bf)
 *   ws       device workspace of at least vdn_workspace_size(cfg, VDN_WS_SCAN)
 *   dev_status  device int32; VDN_ERR_NUMERIC if a pivot was not positive
 */
vdn_status vda_bidir_scan(const vdn_config* cfg, const float* G, const float* C, float* S_fwd,
                          float* S_bwd, void* ws, size_t ws_bytes, int32_t* dev_status,
                          void* stream);

/*
 * vda_bidir_scan_noalloc - vda_bidir_scan without a caller workspace, for
 * callers that cannot allocate device memory when they call the layer (code
 * inside another framework's allocator or plugin hook, a real-time loop that
 * forbids allocation). The paper has no counterpart; it is a deployment aid.
 * Same arguments, outputs and numerics as vda_bidir_scan. The scratch is a
 * 16 MiB array inside the library. Under CUDA's default lazy module loading
 * a GPU holds it from this entry point's first call on that GPU (under
 * CUDA_MODULE_LOADING=EAGER, from the moment the library is loaded) until
 * the process exits; shapes needing more
 * (B*H*T*(d*d + dv*d)*4 bytes, i.e. B*H*T <= 128 at d = dv = 128) return
 * VDN_ERR_WORKSPACE with the sizes in vdn_last_error(). The call allocates
 * nothing. Its first call on a device looks up the scratch address on that
 * device (make that first call before any stream capture); the address is
 * cached per device together with the ID of the current context, so after a
 * device reset (cudaDeviceReset) or a recreated primary context the next call
 * looks it up again (that call, too, belongs before any capture). Every call shares
 * the one array and leaves its contents behind (each call overwrites what it
 * reads, nothing needs to start at zero), so calls that overlap on the GPU,
 * in different streams or threads, race on it: issue them in one stream.
 */
vdn_status vda_bidir_scan_noalloc(const vdn_config* cfg, const float* G, const float* C,
                                  float* S_fwd, float* S_bwd, int32_t* dev_status, void* stream);

/*
 * vda_readout - linear-branch output (sd114.wiki, bidirectional linear
 * branch: the query reads both states and the results are summed).
 *   q      [B,H,L,d] (dtype)
 *   o_lin  [B,L,H,dv] (dtype) out: (S_fwd(b) + S_bwd(b)) q_t for tokens of
 *          non-anchor frames of block b; 0 for anchor frames.
 * bf16: (S_fwd + S_bwd) rounded to bf16, tensor-core product with fp32
 * accumulation; f32: CUDA-core fp32.
 */
vdn_status vda_readout(const vdn_config* cfg, const void* q, const float* S_fwd,
                       const float* S_bwd, void* o_lin, void* stream);

/*
 * vda_readout_gated - the linear half of the gated Z (mlsanity abstract: the
 * branches are calibrated by learnable gates; sd114.wiki: the query reads
 * both states and the results are summed).
 *   q, S_fwd, S_bwd as in vda_readout; gate_logits [H] fp32
 *   Z      [B,L,2,H,dv] (dtype): only Z[.,.,1,h] = (1 - g_h) o_lin is written,
 *          g_h = sigmoid(gate_logits[h]); Z[.,.,0,.] is left unchanged
 */
vdn_status vda_readout_gated(const vdn_config* cfg, const void* q, const float* S_fwd,
                             const float* S_bwd, const float* gate_logits, void* Z,
                             void* stream);

/*
 * vdn_softmax_window - block-sparse softmax branch, optionally gated, and
 * optionally followed by the linear readout into the other half of Z.
 * Each query attends exactly the key frames of its mask row (vdn_window_plan;
 * union of window and anchors, each frame once), scores q.k * softmax_scale,
 * softmax accumulated online in fp32.
 *   q, k [B,H,L,d], v [B,H,L,dv] (dtype)
 *   gate_logits [H] fp32 or NULL; g_h = sigmoid(gate_logits[h])
 *   S_fwd, S_bwd both NULL, or both non-NULL (then gate_logits is required)
 *   out    gate_logits NULL: o_sm [B,L,H,dv]. Otherwise gated Z [B,L,2,H,dv]:
 *          Z[.,.,0,h] = g_h o_sm, and, when S_fwd is given, also
 *          Z[.,.,1,h] = (1 - g_h) o_lin as vda_readout_gated writes it (dtype)
 *   ws     device workspace of at least vdn_workspace_size(cfg, VDN_WS_SOFTMAX)
 *   dev_status  device int32; VDN_ERR_TIMEOUT if a pipeline wait ran out
 */
vdn_status vdn_softmax_window(const vdn_config* cfg, const void* q, const void* k,
                              const void* v, const float* S_fwd, const float* S_bwd,
                              const float* gate_logits, void* out, void* ws, size_t ws_bytes,
                              int32_t* dev_status, void* stream);

/*
 * FP8 softmax branch. The pages report the fastest configuration with FP8
 * (README "Your first render": the fp8 inference script; "Performance
 * Results": branch-specific Ulysses sequence parallelism and FP8 give 1.4 s
 * per step on 8 B200) without fixing a format. This library's reading: OCP
 * e4m3 codes for q, k and v with one fp32 scale per (b, h) and tensor.
 *
 * vdn_quantize_fp8 - e4m3 codes of x [B,H,L,w] (bf16, w = cfg->d):
 *   scale[b*H + h] = amax / 448 over that head's elements (1 if amax = 0),
 *   computed in fp32; x8 = round-to-nearest-even(x / scale) with the
 *   quotient in fp32, saturating to +-448. x8 [B,H,L,w] bytes, scale [B*H]
 *   fp32, both outputs; ws at least vdn_workspace_size(cfg, VDN_WS_QUANT).
 *   Requires dtype bf16 and d = dv = 128.
 */
vdn_status vdn_quantize_fp8(const vdn_config* cfg, const void* x, void* x8, float* scale,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * vdn_softmax_window_fp8 - vdn_softmax_window on e4m3 q, k, v (as written by
 * vdn_quantize_fp8): scores (q8 . k8) q_scale k_scale * softmax_scale with
 * fp32 accumulation of the e4m3 products, online softmax in fp32, P rounded
 * to e4m3 (round to nearest even) for the P V product, output times
 * v_scale. q_scale, k_scale, v_scale: [B*H] fp32 device arrays.
 *   gate_logits NULL: out = o_sm [B,L,H,dv] bf16; else out = the softmax
 *   half of the gated Z [B,L,2,H,dv] bf16 (vda_readout_gated writes the other
 *   half from the bf16 q).
 *   ws, dev_status as in vdn_softmax_window. cfg->dtype is the output type
 *   and must be bf16.
 */
vdn_status vdn_softmax_window_fp8(const vdn_config* cfg, const void* q8, const void* k8,
                                  const void* v8, const float* q_scale, const float* k_scale,
                                  const float* v_scale, const float* gate_logits, void* out,
                                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * vdn_hybrid_forward_fp8 - vdn_hybrid_forward with the softmax branch in
 * e4m3: frame statistics, scan and readout from the bf16 inputs; q, k, v
 * quantised per (b, h); vdn_softmax_window_fp8; vdn_gated_merge.
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_LAYER_FP8) bytes
 */
vdn_status vdn_hybrid_forward_fp8(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, const float* gate_logits, const void* W1,
                                  const void* W2, void* Y, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);

/*
 * vdn_gated_merge - separate output projections of the two branches
 * (mlsanity abstract: separate output projections and learnable gates).
 * Z is already gated (as written by vdn_softmax_window).
 *   Z   [B,L,2,H,dv] (dtype)
 *   w_per_head = 0: W1, W2 [H*dv, d_out]; Y [B,L,d_out] =
 *                   sum_h Z[.,.,0,h] W1[h*dv:(h+1)*dv] + Z[.,.,1,h] W2[h*dv:(h+1)*dv]
 *   w_per_head = 1: W1, W2 [dv, d_out]; Y [B,L,H,d_out] =
 *                   Z[.,.,0,h] W1 + Z[.,.,1,h] W2 (fp32 only)
 * bf16: tensor-core product with fp32 accumulation, d_out % 8 == 0.
 */
vdn_status vdn_gated_merge(const vdn_config* cfg, const void* Z, const void* W1, const void* W2,
                           void* Y, void* stream);

/*
 * vdn_gated_merge_head_groups - vdn_gated_merge for Z in the layout a
 * head-sharded layer receives after re-sharding by tokens ("Performance
 * Results": branch-specific Ulysses sequence parallelism on 8 B200). Each of
 * n_groups ranks computed the gated Z of H / n_groups heads for every token
 * and sent each rank its tokens, so this rank holds
 *   Z   [B, n_groups, Ls, 2, H/n_groups, dv] bf16 (group g = heads
 *       [g*H/n_groups, (g+1)*H/n_groups)), Ls = cfg->T * cfg->N + cfg->n_ctx
 *       tokens per batch item (this rank's share),
 *   W1, W2 [H*dv, d_out] bf16 (all heads), Y [B, Ls, d_out] bf16 out.
 * Y equals vdn_gated_merge on the same values in the plain layout bit for
 * bit (the K products are taken in the same order). n_groups = 1 is the plain
 * layout. Needs bf16, w_per_head = 0, H % n_groups == 0, d_out % 8 == 0;
 * otherwise VDN_ERR_INVALID_ARG or VDN_ERR_UNSUPPORTED before any launch.
 */
vdn_status vdn_gated_merge_head_groups(const vdn_config* cfg, int n_groups, const void* Z,
                                       const void* W1, const void* W2, void* Y, void* stream);

/*
 * vdn_pack_head_groups - the layout copy before a head-sharded layer's input
 * exchange ("Performance Results": branch-specific Ulysses sequence
 * parallelism). A rank holds its token shard of q, k or v and sends rank g
 * the heads of group g; this copy makes each (batch item, local head) one
 * contiguous run over the groups, so that one all-to-all per (b, local
 * head) sends and receives contiguous buffers:
 *   x    [B, Ls, H, 128] bf16 (token-major; Ls = cfg->T*cfg->N + cfg->n_ctx)
 *   out  [B, H/n_groups, n_groups, Ls, 128] bf16,
 *        out[b][h][g][l] = x[b][l][g*H/n_groups + h]
 * Needs bf16 (d = 128), H % n_groups == 0, 16-byte aligned buffers,
 * B*H*Ls < 2^31; otherwise VDN_ERR_INVALID_ARG or VDN_ERR_UNSUPPORTED.
 */
vdn_status vdn_pack_head_groups(const vdn_config* cfg, int n_groups, const void* x, void* out,
                                void* stream);

/*
 * vdn_hybrid_forward - the whole layer: vda_frame_stats, vda_bidir_scan,
 * vdn_softmax_window (gated, with the readout) and vdn_gated_merge in stream
 * order, the intermediates kept in ws.
 *   q, k, v, gate_logits, W1, W2 as above; Y out as in vdn_gated_merge
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_LAYER) bytes
 */
vdn_status vdn_hybrid_forward(const vdn_config* cfg, const void* q, const void* k, const void* v,
                              const float* gate_logits, const void* W1, const void* W2, void* Y,
                              void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * ---------------------------------------------------------------- backward
 * The layer is trained (mlsanity abstract and the flyP critical read: a
 * layer-wise alignment stage fits the hybrid layer to the softmax attention
 * it replaces), but the pages give no gradient formula: these entry points
 * compute the exact derivative of the forward closed form above, for a loss
 * L with output cotangent dY = dL/dY. All need dtype bf16 (d = dv = 128);
 * other dtypes return VDN_ERR_UNSUPPORTED. Cotangents of q, k, v are bf16
 * [B,H,L,128]; those of the gate logits and of W1, W2 are fp32.
 */

/*
 * vdn_softmax_window_lse - the softmax branch alone (ungated o_sm [B,L,H,128]
 * bf16, as vdn_softmax_window with S_fwd = NULL and no gate) plus lse
 * [B,H,L] fp32: the log2-domain log-sum-exp of each row's scaled scores, so
 * that a row's softmax weights are 2^(s * scale * log2(e) - lse).
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_SOFTMAX) bytes
 */
vdn_status vdn_softmax_window_lse(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, void* o_sm, float* lse, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * vdn_softmax_window_bwd - cotangents of q, k, v through the softmax branch
 * (sd114.wiki, sliding-window softmax branch, window and anchors; context
 * tokens as in the forward), given the forward's o_sm and lse
 * (vdn_softmax_window_lse) and the cotangent do_sm of o_sm.
 *   o_sm, do_sm  [B,L,H,128] bf16 (token-major, the layout of o_sm)
 *   dq, dk, dv   [B,H,L,128] bf16 out (overwritten)
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_SOFTMAX_BWD) bytes
 */
vdn_status vdn_softmax_window_bwd(const vdn_config* cfg, const void* q, const void* k,
                                  const void* v, const void* o_sm, const float* lse,
                                  const void* do_sm, void* dq, void* dk, void* dv, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * vda_linear_bwd - cotangents of q, k, v through the linear branch (frame
 * statistics, per-frame solve, both scans, readout), given the cotangent
 * do_lin [B,H,L,128] bf16 of o_lin (head-major). Recomputes the forward's
 * per-frame quantities. dq, dk, dv [B,H,L,128] bf16 out (overwritten; zero
 * on anchor frames and context tokens).
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_LINEAR_BWD) bytes
 * A non-positive pivot is reported through dev_status as in vda_bidir_scan.
 */
vdn_status vda_linear_bwd(const vdn_config* cfg, const void* q, const void* k, const void* v,
                          const void* do_lin, void* dq, void* dk, void* dv, void* ws,
                          size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * vdn_gated_merge_bwd - backward of the merge product Y = Z [W1; W2]:
 *   dZ        [B,L,2,H,128] bf16 out: dY [W1; W2]^T
 *   dW1, dW2  [H*128, d_out] fp32 out: Z_sm^T dY, Z_lin^T dY (overwritten)
 * Z is the forward's gated Z. Needs w_per_head = 0 and d_out % 8 == 0.
 */
vdn_status vdn_gated_merge_bwd(const vdn_config* cfg, const void* Z, const void* W1,
                               const void* W2, const void* dY, void* dZ, float* dW1, float* dW2,
                               int32_t* dev_status, void* stream);

/*
 * vdn_hybrid_forward_train - vdn_hybrid_forward that also returns what the
 * backward needs: the gated Z [B,L,2,H,128] bf16 and lse [B,H,L] fp32 (as in
 * vdn_softmax_window_lse). ws at least vdn_workspace_size(cfg, VDN_WS_LAYER).
 */
vdn_status vdn_hybrid_forward_train(const vdn_config* cfg, const void* q, const void* k,
                                    const void* v, const float* gate_logits, const void* W1,
                                    const void* W2, void* Y, void* Z, float* lse, void* ws,
                                    size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * vdn_hybrid_backward - the whole layer's backward for Y = merge(gate,
 * softmax branch, linear branch):
 *   Z, lse         from vdn_hybrid_forward_train on the same inputs
 *   dY             [B,L,d_out] bf16
 *   dq, dk, dv     [B,H,L,128] bf16 out
 *   dgate_logits   [H] fp32 out
 *   dW1, dW2       [H*128, d_out] fp32 out
 *   ws  at least vdn_workspace_size(cfg, VDN_WS_BACKWARD) bytes
 * Steps: merge backward (dZ, dW1, dW2); gate and branch cotangents
 * do_sm = g dZ_sm, do_lin = (1 - g) dZ_lin; linear-branch backward; softmax
 * backward added on top.
 */
vdn_status vdn_hybrid_backward(const vdn_config* cfg, const void* q, const void* k, const void* v,
                               const float* gate_logits, const void* W1, const void* W2,
                               const void* Z, const float* lse, const void* dY, void* dq,
                               void* dk, void* dv, float* dgate_logits, float* dW1, float* dW2,
                               void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* Diagnostic of the failure path: launches a one-warp kernel whose mbarrier
 * wait is never satisfied. The bounded wait gives up after limit_ms
 * milliseconds (1..10000), writes VDN_ERR_TIMEOUT to *dev_status (a device
 * int32) and the kernel exits normally, so the CUDA context stays usable.
 * Every pipeline wait of the library ends the same way, after 2 seconds. */
vdn_status vdn_selftest_timeout(int32_t* dev_status, int limit_ms, void* stream);

/* Synchronise `stream`, read *dev_status, reset it to 0 and return it as a
 * vdn_status (VDN_ERR_CUDA if the synchronisation or copy failed). */
vdn_status vdn_read_status(int32_t* dev_status, void* stream);

/* Static description of a status code. */
const char* vdn_status_string(vdn_status s);

/* Text of the last CUDA failure seen by the calling thread: the call site in
 * the library, the CUDA error name and message ("" if none yet). The pointer
 * stays valid until the thread's next failing call. */
const char* vdn_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VDN_H_ */
