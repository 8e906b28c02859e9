// Internal launchers of the helper kernels (not part of the public ABI).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace dllm {

int launch_embed(int dtype, const int32_t* tokens, const uint8_t* mask, int mask_id, const void* table, void* x,
                 int rows, int H, cudaStream_t s);
int launch_rmsnorm(int dtype, const void* x, const void* g, void* out, int rows, int H, float eps,
                   const int32_t* row_pos, const int32_t* n_dev, int groups, int group_off, cudaStream_t s);
int launch_masked_rows(const uint8_t* mask, int n_pos, int halves, int32_t* row_pos, int32_t* n_out,
                       cudaStream_t s);
// live (nullable, every launcher below that takes it): device word; 0 = the denoising pass has no masked position
// left, and the kernel returns at once
// ctr_a, ctr_b (nullable): device words set to 0 once the kernels before the gather are done (the work counters
// of the expert GEMMs after it)
int launch_gather_rows(int dtype, const void* h, const int32_t* perm, int k, int Tk, int shared, void* xp, int H,
                       cudaStream_t s, const int32_t* live = nullptr, unsigned* ctr_a = nullptr,
                       unsigned* ctr_b = nullptr);
int launch_combine(int dtype, void* x, const void* y, const float* gates, const int32_t* inv, int k, int Tk,
                   int shared, int H, cudaStream_t s, const int32_t* live = nullptr);
// Fused row stages (bf16 rows of up to 8192 elements, fp32 up to 4096: kRowVecs 16-byte vectors per thread).
constexpr int kRowVecs = 4;
enum NormMode { NORM_NEXT = 0, NORM_FINAL = 1 };
// RoPE table of a block (head dim 128): tab[i * 64 + m] = (cos, sin) of (pos0 + i) * base^(-2 m / 128) for i < L,
// m < 64, evaluated in fp64 and rounded once to fp32 (tab == nullptr: no table).
struct RopeTable {
  float2* tab = nullptr;
  int pos0 = 0, L = 0;
  float base = 10000.f;
};
int launch_rope_table(const RopeTable& r, cudaStream_t s);
// the embedding kernel also fills the RoPE table (extra CTAs) when rope.tab is set
int launch_embed_norm(int dtype, const int32_t* tokens, const uint8_t* mask, int mask_id, const void* table, void* x,
                      void* h, const void* g, int rows, int H, float eps, const uint8_t* list_mask, int n_pos,
                      int halves, int32_t* row_pos, int32_t* n_out, cudaStream_t s,
                      const RopeTable& rope = RopeTable());
int launch_combine_norm(int dtype, void* x, const void* y, const float* gates, const int32_t* inv, int k, int Tk,
                        int shared, int H, const void* g, float eps, void* out, int mode, const uint8_t* mask,
                        int n_half_pos, const int32_t* n_dev, cudaStream_t s, const int32_t* live = nullptr);

// router
int num_sms();

// seg_scratch: route_scratch_bytes(Tk, E, k) bytes, 256-byte aligned (per-segment histograms of the permutation and
// the near-tie thresholds of the selection)
int launch_route(int dtype, const void* h, const void* w_router, const float* bias, int Tk, int H, int E, int k,
                 int32_t* ids, float* gates, float* scores, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* inv, void* seg_scratch, cudaStream_t s, const int32_t* live = nullptr);
int route_segment_tokens(int Tk, int k);
size_t route_scratch_bytes(int Tk, int E, int k);

// unmask
struct UnmaskArgs {
  int B, L, V, max_rows, t, T_s, mode, k_max, cfg, vocab_offset, dtype;
  float tau, cfg_scale;
  const void* logits;
  const int32_t* row_pos;
  const int32_t* n_rows;
  int32_t* tokens;
  uint8_t* mask;
  int32_t* sel;
  int32_t* nsel;
  float* conf;
  int32_t* remaining;
  void* partials;  // workspace: max_rows * n_chunks entries
  int n_chunks;
  int partials_ready = 0;  // 1: the partials were written by the LM head's fused epilogue (no reduction launch)
  cudaGraphConditionalHandle cond = 0;  // with set_cond: the selection sets this graph condition to (remaining > 0)
  int set_cond = 0;
  int score = 0;                 // DLLM_SCORE_*: how positions are ranked (the threshold counts largest probabilities)
  void* extras = nullptr;        // score != 0: max_rows * n_chunks ConfExtra, then B * L floats of ranking scores
  float* conf_hist = nullptr;    // nullable: accepted positions' confidences at conf_hist[row * stride + off + i]
  int conf_hist_stride = 0, conf_hist_off = 0;
  float cfg_image_scale = 1.f;   // cfg 2: the image scale s_i of the editing guidance (cfg_scale is s_t)
};
int unmask_chunks(int max_rows, int V);
size_t unmask_partials_bytes(int max_rows, int n_chunks);
// scratch beside the partials for the scores other than the largest probability (0 for that one)
size_t unmask_extras_bytes(int score, int max_rows, int n_chunks, int B, int L);
int launch_unmask(const UnmaskArgs& a, cudaStream_t s);

// attention
struct AttnArgs {
  int B, Lq, Hq, Hkv, d, blk_len, q_pos0, n_keys, cap, dtype;
  float scale;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* key_pos;
  void* out;
  void* ws;
  size_t ws_bytes;
  const int32_t* live = nullptr;   // nullable: *live == 0 = nothing to do (see launch_gather_rows)
};
size_t attn_workspace_bytes(int B, int Lq, int Hq, int Hkv, int d, int n_keys, int dtype);
int launch_attn(const AttnArgs& a, int32_t* status, cudaStream_t s);
// SIMT (any storage type) and tensor-core (bf16, d = 128) variants
size_t attn_simt_workspace_bytes(int B, int Lq, int Hq, int Hkv, int d, int n_keys);
int launch_attn_simt(const AttnArgs& a, cudaStream_t s);
bool attn_tc_supported(int dtype, int Hq, int Hkv, int d);
size_t attn_tc_workspace_bytes(int B, int Lq, int Hq, int Hkv, int n_keys);
int launch_attn_tc(const AttnArgs& a, int32_t* status, cudaStream_t s);
int launch_attn_merge(const AttnArgs& a, int n_splits, float* po, float* pm, float* pl, cudaStream_t s);

// SPRINT retention
struct RetainArgs {
  int B, Hkv, d, P, cap, n_keep, cap_thin, dtype;
  const void* k;
  const void* v;
  int32_t* keep_pos;
  void* k_thin;
  void* v_thin;
  float* scores;
  float* raw;  // workspace [B, P]
  int block_len;  // > 0: also write keep_pos[n_keep + i] = P + i for i < block_len
  const float* conf = nullptr;        // [B, conf_stride] top-1 confidences of the prefix positions (nullable)
  int conf_stride = 0;
  float alpha = 1.0f;                 // importance = alpha * normalised key norm + (1 - alpha) * conf
  const uint8_t* modality = nullptr;  // [P] 1 = image position (nullable: one selection over the prefix)
  int n_keep_img = 0;                 // image positions kept (with a modality mask); the rest of n_keep are text
};
size_t retain_workspace_bytes(int B, int P);
int launch_retain(const RetainArgs& a, cudaStream_t s);

}  // namespace dllm
