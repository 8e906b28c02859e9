// SPRINT sparse prefix retention: per batch row, score every cached prefix position by the mean over kv heads of
// the L2 norm of its key (optionally mixed with the position's top-1 confidence, and per modality), keep the n_keep
// best (ties -> lower position) and compact their K/V rows, in position order, into the thinned cache that the
// attention of the following steps reads.
// Source: LLaDA2.0-Uni paper review, section "SPRINT — 학습 없는 추론 가속" (importance from the mean-normalised
// key norm; pruning at the first step of each block), HF-mirror README, section "SPRINT 加速技术" (keep_ratio;
// the prefix KV is computed once and reused).
//
// Selection without sorting: the n_keep-th largest score is found by a most-significant-bit-first search over
// the fp32 bit patterns (scores are non-negative, so bit order is value order), counting with block
// reductions; equal scores at the threshold are taken in position order.
#include "common.cuh"
#include "misc.h"

namespace dllm {
namespace {

// raw[b, i] = mean_h ||K[b, h, i, :]||_2 (fp32), one warp per position
template <typename T>
__global__ void retain_scores_kernel(const T* __restrict__ k, int B, int Hkv, int d, int P, int cap,
                                     float* __restrict__ raw) {
  pdl_enter();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= B * P) return;
  const int b = warp / P, i = warp - b * P;
  float tot = 0.f;
  for (int h = 0; h < Hkv; ++h) {
    const T* row = k + (((int64_t)b * Hkv + h) * cap + i) * d;
    float ss = 0.f;
    for (int c = lane; c < d; c += 32) {
      float v = to_f32(row[c]);
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    tot += sqrtf(ss);
  }
  if (lane == 0) raw[warp] = tot / (float)Hkv;
}

// One CTA (1024 threads) per batch row: importance, threshold search, stable selection, keep_pos and scores.
// Importance: the key norm, or with confidences alpha * (key norm / its mean over the prefix) + (1 - alpha) * conf
// (fp32, non-negative). With a modality mask the image positions (mask 1) keep n_keep_img and the text positions the
// rest, each its best ones (a modality with fewer positions than its count keeps them all and the other modality
// keeps the rest, so exactly n_keep positions are kept).
__global__ void retain_select_kernel(const float* __restrict__ raw, int P, int n_keep, int cap_thin,
                                     int32_t* __restrict__ keep_pos, float* __restrict__ scores, int block_len,
                                     const float* __restrict__ conf, int conf_stride, float alpha,
                                     const uint8_t* __restrict__ modality, int n_keep_img) {
  pdl_enter();
  __shared__ int red[32];
  __shared__ double dred[32];
  __shared__ int base;
  __shared__ float rs[8192];     // this row's importance (P <= 8192): the counting passes read shared memory
  __shared__ uint8_t grp[8192];  // modality of each position (0 without a mask)
  __shared__ uint32_t thr_s[2];
  __shared__ int need_s[2];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  for (int i = tid; i < P; i += blockDim.x) {
    rs[i] = raw[(int64_t)b * P + i];
    grp[i] = modality ? (modality[i] ? 1 : 0) : 0;
  }
  __syncthreads();

  auto block_sum_i = [&](int c) -> int {
    c = warp_sum_i(c);
    __syncthreads();
    if (lane == 0) red[w] = c;
    __syncthreads();
    int t = 0;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
  };
  // positions of group g (g < 0: every position) whose bit pattern is >= thr (> thr when strictly)
  auto block_count = [&](int g, uint32_t thr, bool strictly) -> int {
    int c = 0;
    for (int i = tid; i < P; i += blockDim.x) {
      const uint32_t u = __float_as_uint(rs[i]);
      c += (g < 0 || grp[i] == g) && (strictly ? (u > thr) : (u >= thr));
    }
    return block_sum_i(c);
  };

  // mean of the key norms (for the normalised scores and the mixed importance)
  const bool mix = conf != nullptr && alpha != 1.0f;
  if (scores || mix) {
    double s = 0.0;
    for (int i = tid; i < P; i += blockDim.x) s += (double)rs[i];
    s = warp_sum(s);
    if (lane == 0) dred[w] = s;
    __syncthreads();
    double tot = 0.0;
    for (int i = 0; i < nw; ++i) tot += dred[i];
    const float mean = (float)(tot / (double)P);
    __syncthreads();
    for (int i = tid; i < P; i += blockDim.x) {
      float v = rs[i] / mean;
      if (mix) v = alpha * v + (1.0f - alpha) * conf[(int64_t)b * conf_stride + i];
      if (mix) rs[i] = fmaxf(v, 0.0f);
      if (scores) scores[(int64_t)b * P + i] = mix ? rs[i] : v;
    }
    __syncthreads();
  }

  // per selection group: the count it keeps, the largest bit pattern T with #{u >= T} >= count, and how many
  // positions equal to T it takes
  const int ng = modality ? 2 : 1;
  int nk[2] = {n_keep, 0};
  if (modality) {
    const int n_img = block_count(1, 0u, false);
    const int n_txt = P - n_img;
    int ki = min(n_keep_img, n_img);
    int kt = n_keep - ki;
    if (kt > n_txt) { kt = n_txt; ki = n_keep - n_txt; }
    nk[0] = ki;
    nk[1] = kt;
  }
  for (int gi = 0; gi < ng; ++gi) {
    const int g = modality ? (gi == 0 ? 1 : 0) : -1;
    uint32_t prefix = 0;
    int need_eq = 0;
    if (nk[gi] > 0) {
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = prefix | (1u << bit);
        if (block_count(g, cand, false) >= nk[gi]) prefix = cand;
      }
      need_eq = nk[gi] - block_count(g, prefix, true);
    } else {
      prefix = 0xffffffffu;   // no position has a larger pattern (importance is finite): nothing kept
      need_eq = 0;
    }
    if (tid == 0) { thr_s[gi] = prefix; need_s[gi] = need_eq; }
  }
  __syncthreads();

  // stable compaction: kept = (u > T_g) or (u == T_g and among the first need_g equal positions of group g)
  __shared__ int eq_base[2];
  if (tid == 0) { base = 0; eq_base[0] = 0; eq_base[1] = 0; }
  __syncthreads();
  for (int c0 = 0; c0 < P; c0 += blockDim.x) {
    const int i = c0 + tid;
    const int gi = (i < P && modality) ? (grp[i] ? 0 : 1) : 0;
    const uint32_t u = i < P ? __float_as_uint(rs[i]) : 0u;
    const uint32_t T = thr_s[gi];
    int keep = 0;
    int tot_eq[2] = {0, 0};
    for (int q = 0; q < ng; ++q) {
      // rank of this position among the equal positions of selection group q
      const int is_eq = (i < P && gi == q && u == thr_s[q] && thr_s[q] != 0xffffffffu) ? 1 : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, is_eq);
      if (lane == 0) red[w] = __popc(bal);
      __syncthreads();
      int before = 0, tot = 0;
      for (int k2 = 0; k2 < nw; ++k2) {
        if (k2 < w) before += red[k2];
        tot += red[k2];
      }
      const int eq_rank = eq_base[q] + before + __popc(bal & ((1u << lane) - 1u));
      __syncthreads();
      if (is_eq && eq_rank < need_s[q]) keep = 1;
      tot_eq[q] = tot;
    }
    if (i < P && T != 0xffffffffu && u > T) keep = 1;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) red[w] = __popc(bal);
    __syncthreads();
    int kb = 0, ktot = 0;
    for (int k2 = 0; k2 < nw; ++k2) {
      if (k2 < w) kb += red[k2];
      ktot += red[k2];
    }
    if (keep) keep_pos[(int64_t)b * cap_thin + base + kb + __popc(bal & ((1u << lane) - 1u))] = i;
    __syncthreads();
    if (tid == 0) {
      base += ktot;
      eq_base[0] += tot_eq[0];
      eq_base[1] += tot_eq[1];
    }
    __syncthreads();
  }
  // positions of the block rows appended after the kept prefix
  for (int i = tid; i < block_len; i += blockDim.x) keep_pos[(int64_t)b * cap_thin + n_keep + i] = P + i;
}

// k_thin[b, h, j] = k[b, h, keep_pos[b, j]] (and v), 16-byte vectors, one warp per (b, h, j)
template <typename T>
__global__ void retain_copy_kernel(const T* __restrict__ k, const T* __restrict__ v, const int32_t* __restrict__ keep_pos,
                                   int B, int Hkv, int d, int cap, int n_keep, int cap_thin, T* __restrict__ kt,
                                   T* __restrict__ vt) {
  pdl_enter();
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)B * Hkv * n_keep) return;
  const int j = warp % n_keep;
  const int bh = warp / n_keep;
  const int b = bh / Hkv;
  const int src = keep_pos[(int64_t)b * cap_thin + j];
  const int nvec = d * (int)sizeof(T) / 16;
  const uint4* ks = reinterpret_cast<const uint4*>(k + ((int64_t)bh * cap + src) * d);
  const uint4* vs = reinterpret_cast<const uint4*>(v + ((int64_t)bh * cap + src) * d);
  uint4* kd = reinterpret_cast<uint4*>(kt + ((int64_t)bh * cap_thin + j) * d);
  uint4* vd = reinterpret_cast<uint4*>(vt + ((int64_t)bh * cap_thin + j) * d);
  for (int i = lane; i < nvec; i += 32) {
    kd[i] = ks[i];
    vd[i] = vs[i];
  }
}

}  // namespace

size_t retain_workspace_bytes(int B, int P) { return (size_t)B * P * sizeof(float) + 256; }

int launch_retain(const RetainArgs& a, cudaStream_t s) {
  const int64_t rows = (int64_t)a.B * a.P;
  const int blocks = (int)((rows * 32 + 255) / 256);
  if (a.dtype == DLLM_BF16)
    launch_pdl(retain_scores_kernel<__nv_bfloat16>, blocks, 256, 0, s, (const __nv_bfloat16*)a.k, a.B, a.Hkv, a.d, a.P, a.cap, a.raw);
  else
    launch_pdl(retain_scores_kernel<float>, blocks, 256, 0, s, (const float*)a.k, a.B, a.Hkv, a.d, a.P, a.cap, a.raw);
  DLLM_CHECK_LAUNCH("retain_scores_kernel");
  launch_pdl(retain_select_kernel, a.B, 1024, 0, s, a.raw, a.P, a.n_keep, a.cap_thin, a.keep_pos, a.scores, a.block_len,
             a.conf, a.conf_stride, a.alpha, a.modality, a.n_keep_img);
  DLLM_CHECK_LAUNCH("retain_select_kernel");
  const int64_t copies = (int64_t)a.B * a.Hkv * a.n_keep;
  if (copies > 0) {
    const int cb = (int)((copies * 32 + 255) / 256);
    if (a.dtype == DLLM_BF16)
      launch_pdl(retain_copy_kernel<__nv_bfloat16>, cb, 256, 0, s, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v, a.keep_pos,
                                                          a.B, a.Hkv, a.d, a.cap, a.n_keep, a.cap_thin,
                                                          (__nv_bfloat16*)a.k_thin, (__nv_bfloat16*)a.v_thin);
    else
      launch_pdl(retain_copy_kernel<float>, cb, 256, 0, s, (const float*)a.k, (const float*)a.v, a.keep_pos, a.B, a.Hkv, a.d,
                                                   a.cap, a.n_keep, a.cap_thin, (float*)a.k_thin, (float*)a.v_thin);
    DLLM_CHECK_LAUNCH("retain_copy_kernel");
  }
  return DLLM_OK;
}

}  // namespace dllm
