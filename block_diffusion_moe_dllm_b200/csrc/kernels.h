// Internal host interface between the C-ABI entry points and the kernels (not part of the public ABI).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace dllm {

enum EpiKind : int {
  EPI_STORE = 0,   // out[row, m] = acc                 (storage type, or fp32 if out_f32)
  EPI_RESID = 1,   // out[row, m] = out[row, m] + acc   (rounded once)
  EPI_SWIGLU = 2,  // out[row, i] = silu(acc_gate) * acc_up
  EPI_QKV = 3,     // RoPE on q/k heads; q -> q_out, k/v -> cache rows
};

// Confidence partial of one (token row, vocabulary slice): the slice's largest logit, the lowest vocabulary index
// attaining it, and the sum over the slice of exp(z - m). Written by the confidence reduction and by the LM head's
// fused epilogue, merged by the unmask selection.
struct ConfPartial {
  float m;
  int idx;
  double s;
};

// The statistics the other position scores need, beside a ConfPartial of the same slice: the second largest
// logit m2 (over distinct vocabulary entries, so equal to m when the largest value occurs twice; -inf for one entry)
// and t = sum over the slice of exp(z - m) (z - m), from which the entropy follows.
struct ConfExtra {
  float m2;
  float pad;
  double t;
};

struct EpiParams {
  int kind = EPI_STORE;
  void* out = nullptr;
  int64_t ldo = 0;
  int out_f32 = 0;
  // EPI_QKV
  void* q_out = nullptr;            // [rows, Hq, d]
  void* k_dst = nullptr;            // [B, Hkv, cap, d]
  void* v_dst = nullptr;
  void* k_dst2 = nullptr;           // optional second destination (nullable)
  void* v_dst2 = nullptr;
  int cap = 0, slot0 = 0, cap2 = 0, slot2 = 0;
  int Hq = 0, Hkv = 0, d = 0, L = 1, pos0 = 0;
  float rope_base = 10000.f;         // fp32 path (the SIMT epilogue evaluates the angles itself)
  const float2* rope_tab = nullptr;  // [L][64] (cos, sin) of the block's positions (RopeTable), tensor-core path
  // EPI_STORE of bf16 logits: also the confidence partial of every token row over the vocabulary rows this CTA
  // produced, at conf_part[row * conf_nparts + CTA index] (only with gemm_conf_parts(...) == conf_nparts)
  ConfPartial* conf_part = nullptr;
  int conf_nparts = 0;
};

// Y = X W^T over groups of X rows. Group g < n_dev reads rows [grp_off[g], grp_off[g] + grp_cnt[g]) of X and
// weight rows [g * w_group_stride, ...) of W; the optional extra group reads rows [extra_off, extra_off +
// extra_cnt) of X with weights W2. With no device groups and no extra group there is one group of X rows
// [0, cnt) with cnt = *cnt_dev if cnt_dev else host_cnt.
struct GemmArgs {
  const void* x = nullptr;
  int64_t x_rows = 0;
  const void* w = nullptr;
  int64_t w_rows = 0;
  const void* w2 = nullptr;
  int64_t w2_rows = 0;
  int K = 0;
  int M = 0;               // outputs per group (swiglu: I)
  int swiglu = 0;          // weight tile = rows [m, m+64) and [I + m, I + m + 64)
  int64_t w_group_stride = 0;
  int n_dev = 0;
  const int32_t* grp_off = nullptr;
  const int32_t* grp_cnt = nullptr;
  int has_extra = 0;
  int extra_off = 0, extra_cnt = 0;
  const int32_t* cnt_dev = nullptr;
  int host_cnt = 0;
  int max_cnt = 0;         // typical largest group (chooses the tensor-core N tile; larger groups take more tiles)
  int cnt_bound = 0;       // true upper bound of rows in any group (sizes the SIMT grid)
  int dtype = 0;           // DLLM_BF16 / DLLM_F32
  const int32_t* live = nullptr;  // nullable device word: 0 = the pass has nothing left to do (every group empty)
  unsigned* zero_word = nullptr;   // nullable device word the kernel sets to 0 once the kernels before it are done
  unsigned* work_ctr = nullptr;    // grouped launches: nullable work counter, zero at launch (dynamic tile schedule)
  // FP8 weights: W and W2 hold E4M3 codes (one byte each, same row layout) and w_scale / w2_scale one fp32 scale per
  // weight row (w_scale indexed like the rows of W, w2_scale like those of W2); the output is scale[row] * (X q^T)
  int w_fp8 = 0;
  const float* w_scale = nullptr;
  const float* w2_scale = nullptr;
  EpiParams epi;
  int32_t* status = nullptr;
  float* f32_scratch = nullptr;  // f32 path: [x_rows, M (x2 for swiglu)] raw products
};

int gemm_bf16_tc(const GemmArgs& a, cudaStream_t s);
int bn_for(int max_cnt);
int gemm_bn(const GemmArgs& a);
int gemm_splitk_factor(const GemmArgs& a, int bn);
// N tile and K slices of a dense projection run as wide split-K clusters (ks > 1), or ks = 1 when the plain or the
// 32-row split-K kernel serves it better.
struct WideSplit {
  int bn = 0, ks = 1;
};
WideSplit wide_splitk_plan(const GemmArgs& a);

int gemm_f32_simt(const GemmArgs& a, cudaStream_t s);
size_t gemm_f32_scratch_bytes(int64_t x_rows, int M, int swiglu);

// Partial slots per token row when the LM-head GEMM described by a (dense, bf16, rows from a device count) can
// fuse the confidence reduction into its epilogue: one per persistent CTA. 0 when it cannot (more rows than one
// 32-row N tile, or split-K).
int gemm_conf_parts(const GemmArgs& a);
// True when the GEMM runs as CTA pairs sharing each MMA (N tile 256, an even number of 128-row weight tiles).
bool gemm_uses_pairs(const GemmArgs& a);

int num_sms();

}  // namespace dllm
