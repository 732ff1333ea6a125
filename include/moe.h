/*
 * moe.h -- C ABI of the B200 (sm_100a) Stable LatentMoE layer forward pass.
 *
 * The layer (web page "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何が
 * ズレるか、ルーターは何を選んでいるのか", section "K3のエキスパートは896個の
 * 小型LLMではない", the three layer equations; section "ルーターは計算の割当器",
 * the router equation):
 *
 *   s   = Sigmoid(W_r x)                          router scores, one per routed expert
 *   S   = the k experts with the largest s + b    b: frozen per-expert balancing bias
 *   p_j = s_{S_j} / sum_{j'} s_{S_j'}             mixture weights from the UNBIASED scores
 *   z   = W_down x                                latent projection (H -> L)
 *   u   = sum_j p_j E_{S_j}(z)                    routed GLU experts on the latent
 *   y   = E1_shared(x) + ... + ES_shared(x) + W_up RMSNorm(u)
 *
 * with every expert E(a) = W_o SiTU-GLU(W_g a, W_v a) and
 *   SiTU-GLU(g, v) = sigmoid(g) * c*tanh(g/c) * c*tanh(v/c)        (c = situ_c)
 * (tech-report summary "幅のスケーリング：Stable LatentMoE" describes SiTU-GLU only
 * as SwiGLU with smooth caps on the linear and up branches; this closed form is
 * the library's reading), and RMSNorm(u) = gamma * u / sqrt(mean(u^2) + eps).
 * Inference uses the fixed bias with plain top-k selection (page "Kimi K3の
 * 二軸スケーリング戦略とは何か", section "Stable LatentMoE：条件付きの大容量を
 * 安定させる").  Routing is dropless: every token gets its k experts.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers (cudaMalloc / PyTorch CUDA memory)
 *    on the current device, row-major and contiguous in the stated shape,
 *    16-byte aligned.  The caller allocates and owns every buffer, including
 *    the workspace; the library never allocates, frees or synchronises (except
 *    moe_device_error, which says so).
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED for a
 *    combination this build does not implement) and launches nothing.
 *  - A failed launch returns MOE_ERR_CUDA.  No C++ exception crosses the ABI.
 *  - Work is enqueued on `stream` in order; results are ready when the stream
 *    reaches that point.  Identical inputs give bitwise-identical outputs.
 *  - Device-side faults the host cannot see beforehand (an expert index out of
 *    range in a caller-supplied topk_idx, a pipeline wait that ran out of time)
 *    are recorded in a device flag read by moe_device_error; kernels then skip
 *    the offending access, so memory stays in bounds.
 *
 * Supported type combinations (moe_dims.act / routed):
 *  - MOE_F32 / MOE_F32     fp32 everywhere (CUDA-core path, small layers);
 *  - MOE_BF16 / MOE_BF16   bf16 operands, fp32 accumulation (tcgen05 path);
 *    H, L, I and Is must be multiples of 64, S <= 3, E <= 1024, k <= 32;
 *  - MOE_BF16 / MOE_MXFP4  routed-expert weights in OCP MXFP4 (the serving
 *    format of page "ai-tech-express.jp" on K3, section "量子化を前提とした学習
 *    「MXFP4 Quantization-Aware Training」"), everything else bf16; the kernels
 *    decode each weight exactly to bf16 in shared memory and multiply in bf16
 *    with fp32 accumulation.  Additionally L and I must be multiples of 512.
 *  - MOE_BF16 / MOE_MXFP4_A8  the same MXFP4 routed weights, and the routed
 *    experts' input activations (the expert-major z rows and h) quantised to
 *    OCP MXFP8: per row, blocks of 32 consecutive elements along K, each with
 *    an E8M0 scale 2^s, s = floor(log2(max |v|)) - 8 clamped to [-127, 127]
 *    (-127 for an all-zero block), and E4M3 codes round-to-nearest-even(v / 2^s)
 *    saturated to +-448 (the pages name no activation format; this is the OCP
 *    MX v1.0 rule, the library's reading).  Both expert GEMMs then run on the
 *    block-scaled tensor-core MMA (tcgen05.mma kind::mxf8f6f4), which applies
 *    the scales of both operands; accumulation is fp32.  The weight scales are
 *    read in the tiled order of moe_mx_tile_scales (moe_weights.Sgv_tiled,
 *    So_tiled); Wg, Wv and Wo must be 32-byte aligned.  Same dims rules as
 *    MOE_MXFP4.
 *  - MOE_BF16 / MOE_MXFP4_A4  as MOE_MXFP4_A8 with the expert inputs quantised
 *    to OCP MXFP4 instead: per block of 32 the E8M0 scale 2^s,
 *    s = floor(log2(max |v|)) - 2 clamped to [-127, 127] (-127 for an all-zero
 *    block), and E2M1 codes round-to-nearest-even(v / 2^s) saturated to +-6,
 *    two per byte (the even element in the low nibble).  Both expert GEMMs run
 *    on tcgen05.mma kind::mxf4 (both operands 4-bit); same scale tiles,
 *    alignment and dims rules as MOE_MXFP4_A8.
 * Stored activations (z, expert h, shared h, n) are held in the activation type;
 * y_perm, u and the router scores are fp32.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream); NULL means the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null / misaligned pointer, inconsistent sizes, workspace too small */
  MOE_ERR_UNSUPPORTED = 2, /* valid but not implemented in this build (type combination, dims) */
  MOE_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  MOE_ERR_DEVICE = 4       /* moe_device_error only: a kernel recorded a device-side fault */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_MXFP4 = 2, MOE_MXFP4_A8 = 3, MOE_MXFP4_A4 = 4 } moe_dtype;

/* Layer shape and numerics.  K3 values: H=7168, L=3584, E=896, k=16, I=3072,
 * S=2, Is=3072 (dimension table of the page cited above). */
typedef struct {
  int64_t T;         /* tokens in this call (>= 0; 0 is a no-op) */
  int32_t H;         /* hidden size */
  int32_t L;         /* latent size */
  int32_t E;         /* routed experts */
  int32_t k;         /* experts per token, 1 <= k <= min(E, 32) */
  int32_t I;         /* routed-expert intermediate size */
  int32_t S;         /* shared experts (>= 0) */
  int32_t Is;        /* shared-expert intermediate size */
  float situ_c;      /* SiTU-GLU cap c (> 0); 10 in the measured configurations */
  float rms_eps;     /* RMSNorm epsilon (>= 0); 1e-6 */
  moe_dtype act;     /* x, dense weights and stored activations: MOE_F32 or MOE_BF16 */
  moe_dtype routed;  /* routed-expert weights: equal to act, or MOE_MXFP4 with act = MOE_BF16 */
  moe_dtype y_out;   /* y: MOE_F32, or equal to act */
} moe_dims;

/* Layer weights (device pointers, type `act` unless stated). */
typedef struct {
  const void* Wr;      /* [E, H]    router projection */
  const float* bias;   /* [E]       fp32 selection bias (frozen) */
  const void* Wdown;   /* [L, H]    latent down-projection */
  const void* Wup;     /* [H, L]    latent up-projection */
  const float* gamma;  /* [L]       fp32 RMSNorm gain */
  const void* Wg;      /* [E, I, L] routed gate projections (type `routed`); MXFP4: [E, I, L/2] bytes */
  const void* Wv;      /* [E, I, L] routed up projections;                   MXFP4: [E, I, L/2] bytes */
  const void* Wo;      /* [E, L, I] routed down projections;                 MXFP4: [E, L, I/2] bytes */
  /* MXFP4 only (NULL otherwise): E8M0 scale bytes, one per 32 consecutive
   * elements along K (value 2^(s-127); 255 = NaN).  Codes are E2M1, two per
   * byte, the even-K element in the low nibble, bit 3 of a code the sign. */
  const uint8_t* Sg;   /* [E, I, L/32] */
  const uint8_t* Sv;   /* [E, I, L/32] */
  const uint8_t* So;   /* [E, L, I/32] */
  const void* Wsg;     /* [S, Is, H] shared gate projections */
  const void* Wsv;     /* [S, Is, H] shared up projections */
  const void* Wso;     /* [S, H, Is] shared down projections */
  /* MOE_MXFP4_A8 / MOE_MXFP4_A4 only (NULL otherwise): the E8M0 scales of W_g / W_v and of
   * W_o in the tiled order written by moe_mx_tile_scales (Sg, Sv, So are not
   * read on that path and may be NULL). */
  const uint8_t* Sgv_tiled;
  const uint8_t* So_tiled;
} moe_weights;

/* Stages of moe_layer_forward, in launch order (for moe_aux.stage_events). */
#define MOE_STAGE_ROUTER 0         /* router GEMM + sigmoid -> scores */
#define MOE_STAGE_TOPK 1           /* bias + top-k + renormalisation */
#define MOE_STAGE_LATENT_DOWN 2    /* z = W_down x */
#define MOE_STAGE_SHARED_GATE_UP 3 /* shared experts' SiTU-GLU(W_sg x, W_sv x) */
#define MOE_STAGE_PERMUTE 4        /* expert-major order of the (token, slot) pairs */
#define MOE_STAGE_GATHER 5         /* z rows into expert-major order */
#define MOE_STAGE_EXPERT_GATE_UP 6 /* routed experts' SiTU-GLU(W_g z, W_v z) */
#define MOE_STAGE_EXPERT_DOWN 7    /* routed experts' W_o h */
#define MOE_STAGE_COMBINE 8        /* weighted combine + RMSNorm */
#define MOE_STAGE_OUTPUT 9         /* y = [h_shared | n] . [W_so | W_up]^T */
#define MOE_NUM_STAGES 10

/* Optional extra outputs of moe_layer_forward; every field may be NULL.
 * Given buffers receive the intermediate directly (no extra pass). */
typedef struct {
  float* scores;            /* [T, E]  fp32 router scores s = sigmoid(W_r x) */
  int32_t* topk_idx;        /* [T, k]  selected experts, descending key, ties to lower index */
  float* topk_w;            /* [T, k]  mixture weights p (fp32, sum to 1 per token) */
  int32_t* expert_offsets;  /* [E+1]   CSR offsets of the expert-contiguous pair order */
  float* u;                 /* [T, L]  fp32 mixture before RMSNorm */
  void* n;                  /* [T, L]  RMSNorm(u) in the activation type */
  void* z;                  /* [T, L]  W_down x in the activation type */
  /* Host array of 2 * MOE_NUM_STAGES caller-created CUDA events (cudaEvent_t),
   * or NULL.  Event 2i is recorded on `stream` before stage i and event 2i+1
   * after it, so cudaEventElapsedTime gives each stage's device time. */
  void* const* stage_events;
} moe_aux;

/* Bytes of workspace moe_layer_forward needs for these dims (also enough for
 * moe_permute and moe_expert_ffn).  0 for invalid dims.  The workspace must be
 * 256-byte aligned; its contents need not be initialised and are clobbered. */
MOE_API size_t moe_workspace_size(const moe_dims* d);

/* Router and selection ("ルーターは計算の割当器": s = Sigmoid(W_r x); bias added
 * for the choice only; mixture weights = original scores normalised over the
 * chosen experts).
 *   from_scores == 0: scores[T,E] (fp32, written) = sigmoid(x[T,H] . Wr[E,H]^T),
 *                     accumulated in fp32; then selection from those scores.
 *   from_scores != 0: scores[T,E] is INPUT; x and Wr are not read (may be NULL).
 * Selection: key_e = fl32(scores[t,e] + bias[e]); the k largest keys, listed
 * in descending key order, equal keys to the lower expert index;
 * topk_w[t,j] = scores[t,idx_j] / sum_j' scores[t,idx_j'] (fp32, summed in slot
 * order).  Outputs topk_idx[T,k] int32, topk_w[T,k] fp32. */
MOE_API moe_status moe_router_topk(const moe_dims* d, const void* x, const void* Wr, const float* bias, float* scores,
                           int from_scores, int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Dispatch: stable counting sort of the T*k (token, slot) pairs by expert.
 * Pairs of expert e occupy positions expert_offsets[e] .. expert_offsets[e+1]-1
 * in ascending token order; perm_token[pos] = token of the pair at pos;
 * inv_perm[t*k + j] = position of pair (t, j).  If z ([T,L], act) and z_perm
 * ([T*k, L], act) are both non-NULL, z_perm[pos] = z[perm_token[pos]].
 * topk_idx rows must hold k distinct experts in [0, E).
 * Workspace: at least moe_workspace_size(d) bytes. */
MOE_API moe_status moe_permute(const moe_dims* d, const int32_t* topk_idx, const void* z, int32_t* expert_offsets,
                       int32_t* perm_token, int32_t* inv_perm, void* z_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* Routed experts on expert-contiguous latent rows ("K3のエキスパートは896個の小型
 * LLMではない": the selected experts run on z).  For every expert e and every row
 * r in expert_offsets[e] .. expert_offsets[e+1]-1:
 *   h = SiTU-GLU(z_perm[r] . Wg[e]^T, z_perm[r] . Wv[e]^T)   (stored in act type)
 *   y_perm[r] = h . Wo[e]^T                                    (fp32 [T*k, L])
 * Only w->Wg, w->Wv, w->Wo (and for MXFP4 w->Sg, w->Sv, w->So; for
 * MOE_MXFP4_A8 / MOE_MXFP4_A4 w->Sgv_tiled, w->So_tiled, with z_perm and h
 * quantised to MXFP8 / MXFP4 first) are read.
 * Workspace: moe_workspace_size(d) bytes. */
MOE_API moe_status moe_expert_ffn(const moe_dims* d, const moe_weights* w, const void* z_perm,
                          const int32_t* expert_offsets, float* y_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Weighted combine and RMSNorm ("K3のエキスパートは896個の小型LLMではない":
 * u = sum p_i E_i(z); y = ... + W_up RMSNorm(u)).
 *   u[t]   = sum_{j=0}^{k-1} topk_w[t,j] * y_perm[inv_perm[t*k+j]]   (fp32, j ascending)
 *   n_out[t] = gamma * u[t] / sqrt(mean(u[t]^2) + rms_eps)           (act type [T, L])
 * u_out ([T, L] fp32) may be NULL. */
MOE_API moe_status moe_combine(const moe_dims* d, const float* y_perm, const int32_t* inv_perm, const float* topk_w,
                       const float* gamma, float* u_out, void* n_out, moe_stream_t stream);

/* The whole layer: y[T, H] (type y_out) for x[T, H] (type act).  aux may be
 * NULL.  Workspace: at least moe_workspace_size(d) bytes. */
MOE_API moe_status moe_layer_forward(const moe_dims* d, const moe_weights* w, const void* x, void* y, const moe_aux* aux,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* The x-side dense steps of the layer ("K3のエキスパートは896個の小型LLMではない":
 * z = W_down x; the shared experts' E_shared,i(x) up to their down projection):
 *   z[T, L]        = x[T, H] . Wdown[L, H]^T, stored in the activation type;
 *   h_s[T, S*Is]   = SiTU-GLU(x . Wsg[i]^T, x . Wsv[i]^T) for i < S, expert i in
 *                    columns [i*Is, (i+1)*Is), stored in the activation type.
 * Reads w->Wdown, w->Wsg, w->Wsv only.  h_s may be NULL when S = 0.  For
 * callers that run the layer stage by stage (e.g. with the routed experts on
 * other GPUs); moe_layer_forward does the same work internally. */
MOE_API moe_status moe_latent_shared(const moe_dims* d, const moe_weights* w, const void* x, void* z, void* h_s,
                                     moe_stream_t stream);

/* The output projection (same section: y = E1_shared(x) + E2_shared(x) +
 * W_up RMSNorm(u)), as one GEMM over the concatenation [h_s | n]:
 *   y[T, H] = sum_i h_s[:, i*Is:(i+1)*Is] . Wso[i]^T + n[T, L] . Wup[H, L]^T
 * in type y_out, accumulated in fp32.  Reads w->Wso, w->Wup only. */
MOE_API moe_status moe_output(const moe_dims* d, const moe_weights* w, const void* h_s, const void* n, void* y,
                              moe_stream_t stream);

/* Routed experts over rows that arrive as n_blocks expert-major blocks of the
 * same E experts -- the rows an expert-parallel rank receives from each
 * sending rank (the pages' MoonEP, "Kimi K3の二軸スケーリング戦略とは何か",
 * section "MoonEP：疎なMoEを実際に動かす通信層"; the expert computation is that
 * of moe_expert_ffn).
 *  - x_rows [n_rows, L] (act type); block b's rows of expert e are
 *    block_offsets[b*(E+1) + e] .. block_offsets[b*(E+1) + e + 1] - 1 (int32,
 *    absolute row numbers in x_rows, non-decreasing within a block); rows no
 *    block names are not computed.
 *  - y_rows [n_rows, L] fp32: y_rows[r] = W_o[e] SiTU-GLU(W_g[e] x_r, W_v[e] x_r)
 *    for the expert e of row r (same positions as x_rows).
 *  - w->Wg / Wv / Wo (and Sg / Sv / So for MXFP4) hold the E experts of this
 *    call (e.g. one rank's partition); other weight fields are not read.
 *  - Workspace: moe_expert_ffn_blocks_workspace_size(d, n_rows, n_blocks)
 *    bytes, 256-byte aligned.  Offsets outside [0, n_rows] are recorded as a
 *    device fault (moe_device_error) and their segment is skipped.  After the
 *    call the workspace begins with h [n_rows, I] in the activation type (the
 *    stored SiTU-GLU rows, before any quantisation), for inspection.
 * d->T and d->k are not used. */
MOE_API size_t moe_expert_ffn_blocks_workspace_size(const moe_dims* d, int64_t n_rows, int32_t n_blocks);
MOE_API moe_status moe_expert_ffn_blocks(const moe_dims* d, const moe_weights* w, const void* x_rows, int64_t n_rows,
                                         const int32_t* block_offsets, int32_t n_blocks, float* y_rows, void* ws,
                                         size_t ws_bytes, moe_stream_t stream);

/* Allocation-free variant of moe_permute (the pages have no counterpart; this
 * is a library facility).  For callers that cannot allocate device memory when
 * they route tokens -- code running inside an allocator or memory-pool
 * callback, runtimes that forbid cudaMalloc after start-up to keep a fixed
 * footprint, hosts that own no allocator -- it takes no workspace: its scratch
 * (per-tile expert counts and in-tile ranks) lives in a fixed device array of
 * MOE_PERMUTE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library keeps until the process exits.  The call itself allocates
 * nothing.  Arguments and outputs are those of moe_permute.
 *  - Scratch needed: 4*ceil(T/128)*E and 4*T*k bytes, each rounded up to 256;
 *    larger dims return MOE_ERR_INVALID_ARG (K3 shape: up to about 45k tokens).
 *  - The first call on a device looks up the array's device address (once per
 *    device and context, with that device current); make that first call
 *    before any stream capture.  After cudaDeviceReset (or with another
 *    context current) the next call looks it up again, so that call too must
 *    come before any capture.
 *  - All calls share the one array: calls whose work overlaps on the GPU
 *    (different streams, or different host threads without ordering) race and
 *    give wrong results.  Successive calls on one stream are safe; nothing in
 *    the array needs clearing between them. */
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (4u << 20)
MOE_API moe_status moe_permute_noalloc(const moe_dims* d, const int32_t* topk_idx, const void* z,
                                       int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                                       void* z_perm, moe_stream_t stream);

/* Quantile Balancing bias update: the training-time step beside the router
 * ("Kimi K3の896エキスパート…", section 「ルーター専用の独立訓練はない」: each
 * expert's selection bias is updated from the boundary, read off quantiles of
 * the router scores, at which it receives its target number of tokens; Kimi
 * K3 tech-report summary, section 「幅のスケーリング：Stable LatentMoE」: the
 * quantiles come from a histogram of the router's score margins).
 *  - scores [T, E] fp32 (the router's sigmoid scores, e.g. moe_router_topk's
 *    scores_out), bias_in [E] fp32: the current bias.  Uses d->T, d->E, d->k
 *    only (2 <= E <= 1024, 0 < k < E, 1 <= floor(T*k/E) < T).
 *  - Margin of expert e for token t: fl32(s + b_e) minus the k-th largest key
 *    fl32(s + b) among the token's OTHER experts (ties rank the lower index
 *    first); e is selected exactly when its margin is positive.
 *  - hist [E, nbins] uint32: caller-owned workspace, overwritten with the
 *    per-expert margin histogram on [lo, hi) (nbins equal bins, a multiple of
 *    32 in [32, 65536]; margins outside go to the end bins; the bin index is
 *    floor(fl32(fl32(m - lo) * fl32(nbins / (hi - lo))))).
 *  - bias_out[e] = bias_in[e] - q[e], with q[e] the rank-c boundary of e's
 *    margins, c = floor(T*k/E), read from the histogram with the margins
 *    spread evenly within a bin; quantile_out [E] (may be NULL) receives q.
 *    bias_out may alias bias_in.
 *  - Errors: MOE_ERR_INVALID_ARG for bad dims, bins or range, NULL or
 *    misaligned (4-byte) pointers; MOE_ERR_CUDA for a failed launch. */
MOE_API moe_status moe_qb_bias_update(const moe_dims* d, const float* scores, const float* bias_in, float* bias_out,
                                      float* quantile_out, uint32_t* hist, int32_t nbins, float lo, float hi,
                                      moe_stream_t stream);

/* Gradients of moe_layer_backward, fp32, in the shapes of the weights
 * (moe_weights) and of x.  Every pointer must be non-NULL (dWsg / dWsv / dWso
 * may be NULL when S = 0); all are overwritten. */
typedef struct {
  float* dx;      /* [T, H] */
  float* dWr;     /* [E, H] */
  float* dWdown;  /* [L, H] */
  float* dWup;    /* [H, L] */
  float* dgamma;  /* [L] */
  float* dWg;     /* [E, I, L] */
  float* dWv;     /* [E, I, L] */
  float* dWo;     /* [E, L, I] */
  float* dWsg;    /* [S, Is, H] */
  float* dWsv;    /* [S, Is, H] */
  float* dWso;    /* [S, H, Is] */
} moe_grads;

/* Backward pass of the layer with the expert selection held fixed: the
 * vector-Jacobian product of y(x, weights) with dy = dLoss/dy.  The top-k
 * choice is discrete and has no gradient; the mixture weights
 * p_j = s_{e_j} / sum_j' s_{e_j'} are differentiable in the router scores
 * s = Sigmoid(W_r x), so gradients reach the router through p only and the
 * selection bias gets none (page "Kimi K3の896エキスパートを「896人の専門家」と
 * 呼ぶと何がズレるか", sections "ルーターは計算の割当器" and "ルーター専用の
 * 独立訓練はない": the router trains with the model, the bias is set by
 * Quantile Balancing).  Experts no token selected get zero gradients.
 *  - x [T, H] (act), dy [T, H] fp32, topk_idx [T, k] int32: the selection the
 *    forward pass made (moe_aux.topk_idx of moe_layer_forward); rows must hold
 *    k distinct experts in [0, E).
 *  - The forward quantities are recomputed in fp32 from x and the weights,
 *    without the forward pass's bf16 storage rounding, so the result is the
 *    gradient of the layer function itself; accumulation is fp32 and the
 *    order of every sum is fixed (deterministic).
 *  - Supported: act = routed = MOE_F32 or MOE_BF16 (no MXFP4).
 *  - Workspace: moe_backward_workspace_size(d) bytes, 256-byte aligned. */
MOE_API size_t moe_backward_workspace_size(const moe_dims* d);
MOE_API moe_status moe_layer_backward(const moe_dims* d, const moe_weights* w, const void* x, const float* dy,
                                      const int32_t* topk_idx, const moe_grads* g, void* ws, size_t ws_bytes,
                                      moe_stream_t stream);

/* The activation quantiser of the block-scaled path (routed = MOE_MXFP4_A8),
 * on its own: rows of x [rows, K] bf16 -> OCP MXFP8 codes [rows, K] (E4M3,
 * uint8) and E8M0 scale bytes [rows, K/32] (row-major), by the rule stated at
 * MOE_MXFP4_A8 above.  K a multiple of 32; x and codes 16-byte aligned;
 * device pointers owned by the caller.  rows = 0 is a no-op. */
MOE_API moe_status moe_mx8_quantize(const void* x, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales,
                                    moe_stream_t stream);

/* The activation quantiser of the MXFP4-input path (routed = MOE_MXFP4_A4),
 * on its own: rows of x [rows, K] bf16 -> OCP MXFP4 codes [rows, K/2] (E2M1,
 * two per byte, the even element in the low nibble) and E8M0 scale bytes
 * [rows, K/32] (row-major), by the rule stated at MOE_MXFP4_A4 above.  Same
 * argument rules as moe_mx8_quantize. */
MOE_API moe_status moe_mx4_quantize(const void* x, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales,
                                    moe_stream_t stream);

/* Row gather for the expert-parallel exchange (the pages have no counterpart;
 * a library facility): dst[r] = src[idx[r]] for r in [0, n), rows of
 * row_bytes bytes.  The balanced expert-parallel step reorders its
 * expert-major token rows by destination rank with it before the dispatch
 * all-to-all, and puts the returned expert outputs back in expert-major
 * order after the combine all-to-all.
 *  - src [src_rows, row_bytes] and dst [n, row_bytes]: device, 16-byte
 *    aligned, row_bytes a multiple of 16; idx [n] int32 device; all owned by
 *    the caller; src and dst must not overlap.
 *  - n = 0 is a no-op.  An index outside [0, src_rows) is recorded as a device
 *    fault (moe_device_error, site code 15) and its row of dst is zero-filled.
 *  - Enqueued on `stream`; no allocation. */
MOE_API moe_status moe_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx,
                                   int64_t n, void* dst, moe_stream_t stream);

/* Weight scales for the block-scaled routed experts (routed = MOE_MXFP4_A8 or
 * MOE_MXFP4_A4).
 * The block-scaled MMA takes its scales from tensor memory, loaded from
 * shared memory in 512-byte atoms of 128 rows x 4 blocks of 32 along K (byte
 * 16*(m%32) + 4*(m/32) + j = row m, block j); moe_mx_tile_scales re-orders the
 * row-major E8M0 scales once, at load time, into the atoms each 2-CTA weight
 * tile reads:
 *   Sgv_tiled [E][I/128][2][L/128][512]: CTA c of weight tile t holds rows
 *             t*128 + c*64 .. +63 of Sg (atom rows 0-63) and of Sv (64-127);
 *   So_tiled  [E][L/256][2][I/128][512]: CTA c of tile t holds rows
 *             t*256 + c*128 .. +127 of So.
 * moe_mx_tiled_scales_size gives both sizes (each equals the row-major
 * scales' size: E*I*L/16 and E*L*I/32 bytes).  Requires L and I multiples of
 * 512 (MOE_ERR_UNSUPPORTED otherwise); Sg, Sv, So [E, I, L/32], [E, I, L/32],
 * [E, L, I/32] as in moe_weights; all pointers device, 16-byte aligned, owned
 * by the caller.  Enqueued on `stream`; no allocation. */
MOE_API moe_status moe_mx_tiled_scales_size(const moe_dims* d, size_t* gate_up_bytes, size_t* down_bytes);
MOE_API moe_status moe_mx_tile_scales(const moe_dims* d, const uint8_t* Sg, const uint8_t* Sv, const uint8_t* So,
                                      uint8_t* Sgv_tiled, uint8_t* So_tiled, moe_stream_t stream);

/* Human-readable name of a status. */
MOE_API const char* moe_status_str(moe_status s);

/* SYNCHRONISING diagnostic: waits for `stream`, then reports and clears the
 * device-side fault flag of the current device.  *code = 0 when no kernel
 * recorded a fault; otherwise a nonzero site code, and MOE_ERR_DEVICE is
 * returned. */
MOE_API moe_status moe_device_error(int* code, moe_stream_t stream);

/* Number of kernels the last successful moe_layer_forward call on this thread
 * enqueued (for launch accounting). */
MOE_API int moe_last_launch_count(void);

/* Diagnostics, no counterpart in the pages: checks that the kernels' bounded
 * pipeline waits end.  Launches one thread that waits on an mbarrier nothing
 * completes (no copy or MMA in flight); after limit_ms (1..2000) it gives up,
 * records MOE_FAULT_SELFTEST_WAIT in the device fault flag (read and cleared
 * by moe_device_error) and writes the time it waited, in ns, to *waited_ns
 * (a device pointer).  The context stays usable. */
#define MOE_FAULT_SELFTEST_WAIT 9
MOE_API moe_status moe_selftest_wait_timeout(int32_t limit_ms, unsigned long long* waited_ns, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
