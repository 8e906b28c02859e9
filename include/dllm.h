/*
 * dllm.h — C ABI of the B200 (sm_100a) library for one block-diffusion denoising step of the LLaDA2.0-Uni MoE
 * dLLM backbone.
 *
 * Sources of the operations (page title, section):
 *   [R] "[논문 리뷰] LLaDA2.0-Uni: Unifying Multimodal Understanding and Generation with Diffusion Large Language
 *       Model" (paper review, baba9811.github.io): "Block Diffusion Language Model (BDLM)", "MoE 백본과 Block-wise
 *       Attention", "Positional Embedding & 임의 해상도", "SPRINT — 학습 없는 추론 가속", "Load Balancing".
 *   [M] "LLaDA2.0-Uni：基于扩散大型语言模型的多模态理解与生成统一框架" (HF-mirror README, ai.gitcode.com):
 *       "SPRINT 加速技术" and the usage examples.
 *
 * Conventions shared by every call:
 *   - Every pointer argument is DEVICE memory owned by the caller, unless a comment says "host". The library
 *     never allocates, frees or synchronises; every call is asynchronous on the caller's stream.
 *   - Tensors are dense row-major with the listed shapes; the last dimension is contiguous.
 *   - Storage type: DLLM_BF16 (bf16 weights and activations, tcgen05 tensor-core path) or DLLM_F32 (fp32
 *     storage, SIMT path). Accumulation is fp32 in both; router scores, softmax and confidences are fp32 or
 *     wider. Logits are stored in the storage type.
 *   - Every call validates its arguments before launching anything and returns a status code; on error
 *     nothing is launched and dllm_last_error() (thread-local) describes the problem.
 *   - Bf16 tensors read by TMA need 16-byte aligned bases and row strides (DLLM_ERR_ALIGN otherwise).
 *   - A workspace is caller-provided device scratch of at least the size the matching *_workspace_size query
 *     returns, 256-byte aligned. Its first 256 bytes hold a status word that kernels set when a bounded wait
 *     gives up (DLLM_ERR_TIMEOUT through dllm_status_check) and the expert GEMMs' work counters (reset by the
 *     kernels themselves; the caller never initialises them). Calls that share a workspace must be ordered
 *     (same stream); calls on different workspaces are independent and re-entrant.
 */
#ifndef DLLM_H_
#define DLLM_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define DLLM_API __attribute__((visibility("default")))
#else
#define DLLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------------------------------------- status codes */
#define DLLM_OK 0
#define DLLM_ERR_INVALID_ARG 1 /* null pointer, negative size, out-of-range parameter */
#define DLLM_ERR_SHAPE 2       /* inconsistent dimensions */
#define DLLM_ERR_ALIGN 3       /* pointer or stride not 16-byte aligned where TMA reads it */
#define DLLM_ERR_UNSUPPORTED 4 /* valid but not implemented dtype/shape combination */
#define DLLM_ERR_WORKSPACE 5   /* workspace missing, misaligned or too small */
#define DLLM_ERR_CUDA 6        /* a CUDA runtime/driver call failed (message in dllm_last_error) */
#define DLLM_ERR_TIMEOUT 7     /* a kernel gave up on a bounded wait (see dllm_status_check) */

#define DLLM_BF16 0
#define DLLM_F32 1

#define DLLM_UNMASK_FIXED 0     /* k_t = ceil(m / (T_s - t)) */
#define DLLM_UNMASK_THRESHOLD 1 /* k_t = min(m, max(ceil(m / (T_s - t)), min(k_max, #{c > tau}))) */

/* How the still-masked positions are ranked ([M] "SPRINT 加速技术" names the strategies low_confidence, top_k_margin
 * and neg_entropy; their formulas are not on the pages, these are the plain readings), from p = softmax(z). The
 * threshold acceptance counts the positions whose largest probability exceeds tau whatever the ranking. */
#define DLLM_SCORE_LOW_CONFIDENCE 0 /* p_(1), the largest probability */
#define DLLM_SCORE_TOP_K_MARGIN 1   /* p_(1) - p_(2), the two largest probabilities over vocabulary entries */
#define DLLM_SCORE_NEG_ENTROPY 2    /* sum_v p_v log p_v */

/* ---------------------------------------------------------------------------------------------- B7 helpers */
/* Library version string (host, static storage). */
DLLM_API const char* dllm_version(void);
/* Description of the last error on the calling host thread (host, valid until the next call on the thread). */
DLLM_API const char* dllm_last_error(void);
/* Number of kernels this library has launched in the process so far (all threads). */
DLLM_API unsigned long long dllm_launch_count(void);
/* Reads and clears the status word at the head of a workspace. Synchronises the stream (the one call that
 * does). Returns DLLM_OK, DLLM_ERR_TIMEOUT (a kernel stopped after a bounded wait), or DLLM_ERR_CUDA. */
DLLM_API int dllm_status_check(void* ws, cudaStream_t stream);

/* Failure-path self-test: launches one kernel that waits on an mbarrier nothing arrives at, through the same
 * bounded wait the tensor-core kernels use (with a short bound), so that it gives up, records DLLM_ERR_TIMEOUT's
 * cause in the workspace status word and returns. dllm_status_check(ws) then reports DLLM_ERR_TIMEOUT (and clears
 * the word). No GPU state is left behind. */
DLLM_API int dllm_selftest_bounded_wait(void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------------------------- weights */
/*
 * FP8 weights (the FP8 checkpoint of the card news "FP8 추론" and the HF-mirror README's FP8 version; the pages give
 * no format): a matrix W [M, K] is stored as M x K E4M3 codes (OCP 8-bit float without infinities, one byte each,
 * row-major) plus one fp32 scale per row, W[m, k] = value(code[m, k]) * scale[m]. Products with FP8 weights are
 * scale[m] * sum_k x[k] value(code[m, k]) accumulated in fp32 (the codes' values are exact in bf16). Only the large
 * matrices take this form: the routed and shared experts and the LM head. Their K (H, and I for the down
 * projection) must be a multiple of 128 (one 128-byte row of codes per pipeline stage).
 */
#define DLLM_WEIGHTS_BF16 0 /* weights in the storage type */
#define DLLM_WEIGHTS_FP8 1  /* experts and LM head as E4M3 codes with per-row fp32 scales */

/* ---------------------------------------------------------------------------------------------- dense GEMM */
/*
 * Y[n, m] = sum_k X[n, k] * W[m, k] for n < N, m < M: the projection primitive of the backbone (QKV, output
 * projection, LM head). X [N, K], W [M, K], Y [N, M] with row stride ldy elements; Y has the storage type
 * (or fp32 when y_f32 != 0). bf16 path: K % 64 == 0, M % 128 == 0. If residual != 0, Y = Y_in + X W^T
 * (in place, rounded once). n_rows_dev (nullable) overrides N with a device-resident count <= N.
 * w_fp8 != 0: W holds E4M3 codes and w_scale [M] their row scales (bf16 storage only, no residual); otherwise
 * w_scale is ignored (may be NULL).
 */
typedef struct {
  int32_t N, M, K;
  int32_t ldy;
  int32_t dtype;
  int32_t y_f32;
  int32_t residual;
  int32_t w_fp8;
} dllm_gemm_desc;
DLLM_API int dllm_gemm(const dllm_gemm_desc* desc, const void* x, const void* w, const float* w_scale, void* y,
                       const int32_t* n_rows_dev, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_gemm_workspace_size(const dllm_gemm_desc* desc);

/*
 * Grouped projection, the primitive of the routed experts (B4: [R] "MoE 백본과 Block-wise Attention", each token's
 * chosen experts applied to it): rows [offsets[g], offsets[g] + counts[g]) of X form group g < G and are multiplied
 * by the group's weight W[g] ([M', K], M' = 2M with swiglu: rows [0, M) gate, [M, 2M) up, else M' = M); with
 * w_extra != NULL the last extra_rows rows of X form one more group with weight w_extra [M', K] (the shared
 * expert). Y[r, :] = X[r] W_g^T, or with swiglu silu(X[r] W_gate^T) * (X[r] W_up^T) in fp32 rounded once to the
 * storage type. X [rows, K]; Y [rows, M] in the storage type (fp32 when y_f32 != 0, not with swiglu); rows of X in
 * no group are not written. counts, offsets: [G] int32 device arrays (groups may not overlap). max_rows_hint: the
 * typical group size (chooses the tile width). bf16 only: K % 64 == 0, M % 128 == 0 (swiglu: M % 64 == 0).
 * w_fp8 != 0: W and w_extra hold E4M3 codes, w_scale [G, M'] and w_extra_scale [M'] their row scales.
 */
typedef struct {
  int32_t G, rows, K, M;
  int32_t swiglu;
  int32_t extra_rows;
  int32_t max_rows_hint;
  int32_t dtype;
  int32_t y_f32;
  int32_t w_fp8;
} dllm_grouped_gemm_desc;
DLLM_API int dllm_grouped_gemm(const dllm_grouped_gemm_desc* desc, const void* x, const void* w, const void* w_extra,
                               const float* w_scale, const float* w_extra_scale, const int32_t* counts,
                               const int32_t* offsets, void* y, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_grouped_gemm_workspace_size(const dllm_grouped_gemm_desc* desc);

/* ---------------------------------------------------------------------------------------------- B1 attention */
/*
 * Block-causal attention ([R] "Block Diffusion Language Model (BDLM)", "MoE 백본과 Block-wise Attention"):
 * for query i of row b at absolute position q_pos0 + i and head h, o = softmax(q k^T * scale + M) v over the
 * row's keys, where the kv head is floor(h * Hkv / Hq) and M[i, j] = 0 iff floor(pos_j / blk_len) <=
 * floor(pos_i / blk_len), else -inf (bidirectional inside a block, causal across blocks). A denoising pass is
 * the special case where the queries are the last block and every key is visible.
 *   q        [B, Lq, Hq, d]
 *   k_cache  [B, Hkv, cap, d]  keys in rows [0, n_keys) (already rotated by RoPE)
 *   v_cache  [B, Hkv, cap, d]
 *   key_pos  [B, n_keys] int32 absolute position of each key row, or NULL for positions 0..n_keys-1
 *            (a SPRINT-thinned cache lists the kept prefix positions followed by the block's positions)
 *   out      [B, Lq, Hq * d]
 * scale <= 0 selects 1/sqrt(d). bf16: d == 128. f32: d <= 128, d % 4 == 0.
 */
typedef struct {
  int32_t B, Lq, Hq, Hkv, d;
  int32_t blk_len;
  int32_t q_pos0;
  int32_t n_keys;
  int32_t cap;
  int32_t dtype;
  float scale;
} dllm_attn_desc;
DLLM_API int dllm_block_attn(const dllm_attn_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* key_pos, void* out, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_block_attn_workspace_size(const dllm_attn_desc* desc);

/* ---------------------------------------------------------------------------------------------- B2 SPRINT */
/*
 * SPRINT sparse prefix retention ([R] "SPRINT — 학습 없는 추론 가속"; [M] "SPRINT 加速技术", keep_ratio and the
 * modality keep ratios): per row b, the key norm l_i = mean over kv heads of ||K[b, h, i, :]||_2, normalised by its
 * mean over i < P (l~_i); the importance s_i = alpha l~_i + (1 - alpha) conf[b, i] (alpha = 1 or conf == NULL: the
 * key-norm term alone; the page's alpha is 0.5, conf the position's top-1 confidence). The n_keep highest-importance
 * positions are kept (ties -> lower position), listed in increasing position in keep_pos[b, 0:n_keep], and their K/V
 * rows are copied, in that order, to rows [0, n_keep) of k_thin / v_thin. With modality != NULL ([P] uint8, 1 =
 * image position) n_keep_img of them are image positions and the rest text positions, each the best of its
 * modality (a modality with fewer positions than its count keeps all of them and the other keeps the rest).
 *   k_cache, v_cache [B, Hkv, cap, d];  k_thin, v_thin [B, Hkv, cap_thin, d];  keep_pos [B, cap_thin] int32
 *   conf [B, P] fp32 (nullable); modality [P] uint8 (nullable);
 *   scores [B, P] fp32 (nullable): the importance (the mean-normalised key norm without confidences).
 * Requires n_keep <= P <= 8192, n_keep <= cap_thin, 0 <= alpha <= 1, 0 <= n_keep_img <= n_keep.
 */
typedef struct {
  int32_t B, Hkv, d, P, cap;
  int32_t n_keep, cap_thin;
  int32_t dtype;
  float alpha;
  int32_t n_keep_img;
} dllm_retain_desc;
DLLM_API int dllm_prefix_retain(const dllm_retain_desc* desc, const void* k_cache, const void* v_cache,
                       const float* conf, const uint8_t* modality, int32_t* keep_pos, void* k_thin, void* v_thin,
                       float* scores, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_prefix_retain_workspace_size(const dllm_retain_desc* desc);

/* ---------------------------------------------------------------------------------------------- B3 router */
/*
 * MoE router ([R] "MoE 백본과 Block-wise Attention": top-k experts per token; [R] "Load Balancing": per-expert
 * bias used for selection only): s = sigmoid(h W_r^T) in fp32; ids = the k experts with the largest s + bias
 * (ties -> lower id), slots ordered by biased score; gates = s[ids] / sum(s[ids]). s is accumulated in fp32 (on the
 * tensor cores for bf16 with E % 128 == 0), so experts whose exact scores differ by less than its error (a few
 * 1e-6 at H = 2048) can be chosen or ordered either way.
 * Then the token permutation used by the grouped expert GEMMs: counts[e] = #assignments to e; offsets =
 * exclusive prefix sum (offsets[E] = Tk * k); perm[r] = t * k + j of the assignment stored at sorted row r
 * (rows of one expert in increasing t); inv[t * k + j] = r.
 *   h [Tk, H]; w_router [E, H]; bias [E] fp32; ids [Tk, k] int32; gates [Tk, k] fp32; counts [E]; offsets [E+1];
 *   perm, inv [Tk * k] int32; scores [Tk, E] fp32 (nullable): the sigmoid scores.
 * Requires E <= 1024, k <= 32, k <= E.
 */
typedef struct {
  int32_t Tk, H, E, k;
  int32_t dtype;
} dllm_route_desc;
DLLM_API int dllm_moe_route(const dllm_route_desc* desc, const void* h, const void* w_router, const float* bias,
                   int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                   float* scores, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_moe_route_workspace_size(const dllm_route_desc* desc);

/* ---------------------------------------------------------------------------------------------- B4 experts */
/*
 * MoE FFN of the backbone ([R] "MoE 백본과 Block-wise Attention": each token's FFN is the mixture of the top-k
 * experts the router picked, weighted by its gates; the shared expert, applied to every token, and the SwiGLU form
 * of each expert are the stated layer configuration of this library's workloads). Routed experts plus shared
 * expert, added to the residual:
 *   x[t] <- x[t] + shared(h[t]) + sum_j gates[t, j] * expert_{ids[t, j]}(h[t]),
 * expert_e(v) = W_down[e] (silu(W_gate[e] v) * (W_up[e] v)) (SwiGLU; the SwiGLU activation and each expert's
 * output row, accumulated in fp32, are stored in the storage type), the shared row then the gate-weighted rows
 * summed onto the residual in slot order j = 0..k-1 in fp32 and rounded once.
 *   h [Tk, H]; w_gu [E, 2I, H] (rows [0, I) gate, [I, 2I) up); w_down [E, H, I]; w_gu_shared [2I, H] and
 *   w_down_shared [H, I] (both NULL: no shared expert); counts/offsets/perm/inv/gates as produced by
 *   dllm_moe_route; x_inout [Tk, H].
 * bf16: H % 128 == 0, I % 64 == 0.
 * w_fp8 != 0: the four weights hold E4M3 codes with row scales w_gu_scale [E, 2I], w_down_scale [E, H],
 * w_gu_shared_scale [2I], w_down_shared_scale [H] (NULL without a shared expert).
 */
typedef struct {
  int32_t Tk, H, E, k, I;
  int32_t dtype;
  int32_t w_fp8;
} dllm_expert_desc;
DLLM_API int dllm_moe_experts(const dllm_expert_desc* desc, const void* h, const void* w_gu, const void* w_down,
                     const void* w_gu_shared, const void* w_down_shared, const float* w_gu_scale,
                     const float* w_down_scale, const float* w_gu_shared_scale, const float* w_down_shared_scale,
                     const int32_t* counts, const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                     const float* gates, void* x_inout, void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_moe_experts_workspace_size(const dllm_expert_desc* desc);

/* ---------------------------------------------------------------------------------------------- B5 unmask */
/*
 * Confidence and unmasking ([R] "SPRINT — 학습 없는 추론 가속": c = max_v p(v | x_t), accept every c > tau, at
 * least ceil(m / (T - t)) per step; [M] "SPRINT 加速技术": k = ceil(remaining / steps_left), batch acceptance).
 * For each still-masked position r (n_rows of them; row r is flat position row_pos[r] = b * L + i of the
 * logical rows): z = logits[r]; with cfg 1 z = zu + cfg_scale * (zc - zu) in fp32, zc = logits[r],
 * zu = logits[n_rows + r] ([M] text-to-image usage, cfg_scale); with cfg 2, editing guidance ([M] note under
 * "SPRINT 加速技术": three-way guidance through cfg_text_scale and cfg_image_scale; formula not printed, plain
 * reading) z = a + cfg_scale * (zc - zi), a = zu + cfg_image_scale * (zi - zu), each operation rounded to fp32 in
 * that order, zi = logits[n_rows + r] (image only), zu = logits[2 n_rows + r]; candidate = vocab_offset + lowest
 * argmax of z; c = 1 / sum_v exp(z_v - max z).
 * Per logical row b with m masked positions: k_t positions by the ranking score descending (c itself by default;
 * rounded to fp32; equal values -> lower position) get their
 * candidate written to tokens and their mask cleared; with cfg the guidance rows b + g * B (g = 1 .. cfg) get the
 * same update.
 *   logits [n_rows * (1 + cfg), V] in the storage type; row_pos [>= n_rows] int32: the still-masked flat
 *   positions of the logical rows in increasing order (row r of the logits belongs to the r-th masked position;
 *   every masked position must be listed, otherwise the results for the logical row are undefined);
 *   n_rows_dev [1] int32 (device count of masked positions; a count above max_rows is read as max_rows); tokens [B * (1 + cfg), L] int32; mask [B * (1 + cfg), L] uint8;
 *   sel [B, L] int32 (chosen positions in rank order, -1 after nsel[b]); nsel [B]; conf [B, L] fp32 (the largest
 *   probability; 0 at unmasked positions); remaining [1] int32: masked positions left over all logical rows.
 * Requires L <= 32 (one warp per block row for the selection) and B <= 1024.
 */
typedef struct {
  int32_t B, L, V;
  int32_t max_rows;
  int32_t t, T_s;
  int32_t mode;
  float tau;
  int32_t k_max;
  int32_t cfg;
  float cfg_scale;
  int32_t vocab_offset;
  int32_t dtype;
  int32_t score;     /* DLLM_SCORE_*: the ranking of the positions */
  float cfg_image_scale;   /* cfg 2: the image scale of the editing guidance (cfg_scale is the text scale) */
} dllm_unmask_desc;
DLLM_API int dllm_unmask(const dllm_unmask_desc* desc, const void* logits, const int32_t* row_pos, const int32_t* n_rows_dev,
                int32_t* tokens, uint8_t* mask, int32_t* sel, int32_t* nsel, float* conf, int32_t* remaining,
                void* ws, size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_unmask_workspace_size(const dllm_unmask_desc* desc);

/*
 * dllm_unmask without a workspace, for callers that cannot allocate device memory (a plug-in inside a host
 * application that owns the device's memory pool and exposes no allocator; a serving loop that forbids cudaMalloc
 * after start-up because it can synchronise the device). The paper has no counterpart: this is a deployment
 * variant of the same computation. Same arguments and results as dllm_unmask minus ws / ws_bytes; the caller
 * still owns every input and output. The per-chunk scratch lives in a fixed 256 KiB array inside the library,
 * held on every GPU that loads it until the process exits; calls with max_rows x vocabulary chunks needing more
 * (more than 16384 partial entries of 16 bytes) return DLLM_ERR_UNSUPPORTED. The first call on each device looks up the
 * array's device address (make it before any stream capture). All calls share the array: calls that overlap on
 * the GPU race and must be ordered by the caller (one stream, or events).
 */
DLLM_API int dllm_unmask_noalloc(const dllm_unmask_desc* desc, const void* logits, const int32_t* row_pos,
                                 const int32_t* n_rows_dev, int32_t* tokens, uint8_t* mask, int32_t* sel, int32_t* nsel,
                                 float* conf, int32_t* remaining, cudaStream_t stream);

/* ---------------------------------------------------------------------------------------------- B6 step */
/* Weights of one layer (device pointers, storage type unless stated). */
typedef struct {
  const void* attn_norm;     /* [H] */
  const void* w_qkv;         /* [(Hq + 2 Hkv) d, H]: q rows, then k rows, then v rows */
  const void* w_o;           /* [H, Hq d] */
  const void* ffn_norm;      /* [H] */
  const void* w_router;      /* [E, H] */
  const float* router_bias;  /* [E] fp32 */
  const void* w_gu;          /* [E, 2I, H] */
  const void* w_down;        /* [E, H, I] */
  const void* w_gu_shared;   /* [2I, H] */
  const void* w_down_shared; /* [H, I] */
  void* k_cache;             /* [B, Hkv, cap, d] full cache: prefix rows [0, P) */
  void* v_cache;
  void* k_thin;              /* [B, Hkv, cap_thin, d] SPRINT-thinned cache (NULL without SPRINT) */
  void* v_thin;
  int32_t* keep_pos;         /* [B, cap_thin] positions of the thinned rows (NULL without SPRINT) */
  /* row scales of the expert weights when the model's weight_format is DLLM_WEIGHTS_FP8 (the weights above then
     hold E4M3 codes), else NULL */
  const float* w_gu_scale;          /* [E, 2I] */
  const float* w_down_scale;        /* [E, H] */
  const float* w_gu_shared_scale;   /* [2I] */
  const float* w_down_shared_scale; /* [H] */
} dllm_layer;

typedef struct {
  int32_t n_layers, H, Hq, Hkv, d, E, k, I, V;
  int32_t dtype;
  float eps;       /* RMSNorm epsilon */
  float rope_base; /* RoPE base; rotate-half pairing over the full head dim */
  int32_t mask_id; /* embedding row used at masked positions */
  const void* embed;      /* [V, H] */
  const void* final_norm; /* [H] */
  const void* w_lm;       /* [V, H] */
  const dllm_layer* layers; /* host array of n_layers */
  int32_t weight_format;    /* DLLM_WEIGHTS_BF16, or DLLM_WEIGHTS_FP8 (bf16 storage only): experts and w_lm as E4M3 codes */
  const float* w_lm_scale;  /* [V] row scales of w_lm with DLLM_WEIGHTS_FP8, else NULL */
} dllm_model;

/* Decoding state of one block (device pointers except the sizes). */
typedef struct {
  int32_t B;         /* batch rows (cfg 1: B/2 conditional rows then B/2 unconditional rows; cfg 2: B/3 rows
                        conditioned on instruction and image, B/3 on the image only, B/3 unconditional) */
  int32_t L;         /* block length (<= 32) */
  int32_t P;         /* clean positions in the cache before this block (the block sits at [P, P + L)) */
  int32_t cap;       /* rows per (row, kv head) of the full caches, >= P + L */
  int32_t cap_thin;  /* rows of the thinned caches, >= n_keep + L */
  int32_t* tokens;   /* [B, L] */
  uint8_t* mask;     /* [B, L] 1 = still masked */
  float* prefix_conf;              /* [B, cap] (nullable): top-1 confidence of every cache position; each denoising
                                      pass writes the confidences of the positions it accepts at P + i, SPRINT
                                      selection reads [0, P) when sprint_alpha < 1 (prompt positions: the caller's) */
  const uint8_t* prefix_modality;  /* [cap] (nullable): 1 = image position, for the modality keep counts */
} dllm_state;

typedef struct {
  int32_t t, T_s;       /* step index (0-based) and steps per block */
  int32_t mode;         /* DLLM_UNMASK_FIXED or DLLM_UNMASK_THRESHOLD */
  float tau;
  int32_t k_max;
  int32_t cfg;          /* 1: rows pair as (b, b + B/2) = (cond, uncond); 2 (editing guidance, no SPRINT): rows
                           (b, b + B/3, b + 2B/3) = (instruction and image, image only, uncond) */
  float cfg_scale;
  int32_t vocab_offset; /* LM-head rows [vocab_offset, vocab_offset + vocab_len) are scored */
  int32_t vocab_len;    /* 0 = V */
  int32_t sprint;       /* 1: attention reads the thinned caches */
  int32_t n_keep;       /* kept prefix rows (sprint) */
  int32_t retain;       /* 1 (with sprint, normally at t == 0): run SPRINT selection first */
  int32_t commit;       /* 1: commit pass over the finished block (no LM head / unmask); writes the block's
                           clean K/V into rows [P, P + L) of the full caches */
  /* outputs of the unmasking (device, ignored by a commit pass) */
  int32_t* sel;       /* [B', L] */
  int32_t* nsel;      /* [B'] */
  float* conf;        /* [B', L] */
  int32_t* remaining; /* [1] */
  int32_t score;      /* DLLM_SCORE_*: the ranking of the still-masked positions */
  float sprint_alpha;   /* SPRINT importance mix (1: key norm alone; needs state->prefix_conf otherwise) */
  int32_t n_keep_img;   /* with state->prefix_modality: image positions among the n_keep kept */
  float cfg_image_scale; /* cfg 2: the image scale of the editing guidance (cfg_scale is the text scale) */
} dllm_step_params;

/*
 * One denoising pass of the backbone over the current block ([R] BDLM: blocks decoded left to right, the block
 * itself under bidirectional attention over the clean cached prefix; [M] SPRINT: prefix KV computed once and
 * reused, pruned at the first step of a block; confidence-based unmasking), on one stream with no host sync:
 *   embed -> per layer [RMSNorm, QKV + RoPE (block K/V into the cache), (SPRINT selection), block attention,
 *   output projection + residual, RMSNorm, router, routed + shared experts + residual] -> final RMSNorm ->
 *   LM head on the still-masked rows -> (CFG) -> confidence + unmasking.
 * B' = B / (1 + cfg) logical rows. Workspace from dllm_denoise_step_workspace_size with the same arguments.
 * Early finish: a denoising pass over a block with no masked position left (threshold acceptance can finish a
 * block before its last step) changes nothing: its first kernel finds no masked position, and every later kernel of
 * the pass returns at entry (no weight or cache is read, no cache row written; sel is all -1, nsel 0, remaining 0),
 * so the remaining passes of a finished block cost only their launches and need no host synchronisation. A commit
 * pass always runs.
 */
DLLM_API int dllm_denoise_step(const dllm_model* model, const dllm_state* state, const dllm_step_params* params, void* ws,
                      size_t ws_bytes, cudaStream_t stream);
DLLM_API size_t dllm_denoise_step_workspace_size(const dllm_model* model, const dllm_state* state,
                                        const dllm_step_params* params);

/*
 * A whole block as one CUDA graph: the T_s denoising passes (t = 0 .. T_s - 1, SPRINT selection at t = 0 when
 * params->sprint) and the commit pass, every pass inside a conditional node that runs it only while the block still
 * has masked positions (the unmasking of each pass sets the condition on the device), so the passes after a
 * threshold-mode block finished are not launched at all. The passes are those dllm_denoise_step would run with the
 * same arguments (params is the template: t, retain and commit are set per pass; it must describe a denoising
 * pass). The graph is captured on capture_stream (a created stream, not capturing, not the legacy default stream),
 * once; its kernels read the state, caches and outputs at the addresses given here on every launch, so the caller
 * refills tokens / mask and launches it again for the next block of the same shapes. Host memory only: the library
 * allocates no device memory (instantiating the graph may reserve driver resources). Destroy with
 * dllm_block_graph_destroy. Where the driver refuses conditional nodes the passes follow one another unconditionally
 * (those after an early finish then return at entry, see dllm_denoise_step); dllm_block_graph_skips_finished_passes
 * tells which (1: conditional).
 */
typedef struct dllm_block_graph dllm_block_graph;
DLLM_API int dllm_block_graph_create(const dllm_model* model, const dllm_state* state, const dllm_step_params* params,
                                     void* ws, size_t ws_bytes, cudaStream_t capture_stream,
                                     dllm_block_graph** out /* host */);
DLLM_API int dllm_block_graph_launch(const dllm_block_graph* graph, cudaStream_t stream);
DLLM_API void dllm_block_graph_destroy(dllm_block_graph* graph);
DLLM_API int dllm_block_graph_skips_finished_passes(const dllm_block_graph* graph);

/* Device addresses, inside a step workspace, of intermediate results of the last dllm_denoise_step that used it
 * (read-only views for inspection; valid until the workspace is reused). */
typedef struct {
  const void* logits;      /* [rows, vocab_len] storage type: the masked rows' logits (cond rows, then uncond) */
  const int32_t* row_pos;  /* [B' L] flat positions of the masked logical rows, ascending */
  const int32_t* n_rows;   /* [1] number of masked logical rows at the start of the pass */
  const void* x_final;     /* [B L, H] storage type: hidden state after the last layer (before the final norm) */
  const int32_t* expert_counts; /* [n_layers, E + 1]: per layer, the assignments routed to each expert by the last
                                   pass that ran that layer (entry E unused) */
  const int32_t* live;     /* [1]: 1 if the last denoising pass found a masked position (and ran), else 0 */
} dllm_step_views;
DLLM_API int dllm_denoise_step_views(const dllm_model* model, const dllm_state* state, const dllm_step_params* params,
                            void* ws, size_t ws_bytes, dllm_step_views* views /* host */);

#ifdef __cplusplus
}
#endif
#endif /* DLLM_H_ */
