// Block-causal attention of the block's queries over the cached (optionally SPRINT-thinned) prefix and the
// block itself: o = softmax(q k^T / sqrt(d) + M) v with M[i, j] = 0 iff floor(pos_j / L) <= floor(pos_i / L).
// Source: LLaDA2.0-Uni paper review, sections "Block Diffusion Language Model (BDLM)" (bidirectional inside a
// block, left-to-right across blocks, earlier blocks clean) and "MoE 백본과 Block-wise Attention".
//
// SIMT flash-decoding kernel: one CTA per (row b, kv head, tile of queries, key split). The CTA's 64 query
// rows are the Hq/Hkv query heads sharing the kv head times 64/(Hq/Hkv) queries, so every K/V row staged in
// shared memory serves all heads of the group (GQA packing). Four threads own one query row: each scores 8 of
// the 32 keys of a staged block, the row's online-softmax state is kept in sync by shuffles, and each thread
// accumulates a quarter of the head dim of the output. Key splits are merged by log-sum-exp.
#include "common.cuh"
#include "misc.h"

namespace dllm {
namespace {

constexpr int ROWS = 64;
constexpr int KB = 32;
constexpr int DP = 129;  // padded row length in shared memory (floats)

struct AttnK {
  int B, Lq, Hq, Hkv, d, blk_len, q_pos0, n_keys, cap;
  int qt_rows;     // queries per CTA
  int n_qtiles;
  int n_splits;
  int keys_per_split;
  float scale_log2;  // scale * log2(e)
  const void* q;
  const void* k;
  const void* v;
  const int32_t* key_pos;
  void* out;
  float* po;  // [splits, B, Lq, Hq, d] partial outputs (unnormalised) when n_splits > 1
  float* pm;  // [splits, B, Lq, Hq] running max (log2 domain)
  float* pl;  // [splits, B, Lq, Hq] running sum
  const int32_t* live;  // nullable: *live == 0 = nothing to do
};

template <typename T>
__global__ void __launch_bounds__(256) attn_simt_kernel(const AttnK p) {
  pdl_enter();
  if (p.live && *p.live == 0) return;   // a pass with no masked position left does nothing
  extern __shared__ float sm[];
  float* qs = sm;                  // [ROWS][DP]
  float* ks = qs + ROWS * DP;      // [KB][DP]
  float* vs = ks + KB * DP;        // [KB][DP]
  int* kp = reinterpret_cast<int*>(vs + KB * DP);  // [KB]

  const int G = p.Hq / p.Hkv;
  int bx = blockIdx.x;
  const int qt = bx % p.n_qtiles;
  bx /= p.n_qtiles;
  const int g = bx % p.Hkv;
  const int b = bx / p.Hkv;
  const int split = blockIdx.y;
  const int tid = threadIdx.x, row = tid >> 2, sub = tid & 3;
  const int d = p.d;

  // query rows: row r -> head g*G + r / qt_rows, query qt*qt_rows + r % qt_rows
  const T* Q = static_cast<const T*>(p.q);
  for (int i = tid; i < ROWS * d; i += 256) {
    int r = i / d, c = i - r * d;
    int hh = r / p.qt_rows, qi = qt * p.qt_rows + r % p.qt_rows;
    float v = 0.f;
    if (hh < G && qi < p.Lq) v = to_f32(Q[(((int64_t)b * p.Lq + qi) * p.Hq + g * G + hh) * d + c]);
    qs[r * DP + c] = v * p.scale_log2;
  }
  const int my_h = row / p.qt_rows, my_q = qt * p.qt_rows + row % p.qt_rows;
  const bool row_ok = my_h < G && my_q < p.Lq;
  const int qblk = (p.q_pos0 + my_q) / p.blk_len;

  float m = -INFINITY, l = 0.f;
  float o[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) o[c] = 0.f;

  const T* K = static_cast<const T*>(p.k) + ((int64_t)b * p.Hkv + g) * p.cap * d;
  const T* V = static_cast<const T*>(p.v) + ((int64_t)b * p.Hkv + g) * p.cap * d;
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.n_keys, k_begin + p.keys_per_split);
  const int cw = d / 4;  // output columns per thread

  for (int j0 = k_begin; j0 < k_end; j0 += KB) {
    __syncthreads();
    const int nk = min(KB, k_end - j0);
    for (int i = tid; i < KB * d; i += 256) {
      int r = i / d, c = i - r * d;
      float kv = 0.f, vv = 0.f;
      if (r < nk) {
        kv = to_f32(K[(int64_t)(j0 + r) * d + c]);
        vv = to_f32(V[(int64_t)(j0 + r) * d + c]);
      }
      ks[r * DP + c] = kv;
      vs[r * DP + c] = vv;
    }
    if (tid < KB) {
      int j = j0 + tid;
      kp[tid] = tid < nk ? (p.key_pos ? p.key_pos[(int64_t)b * p.n_keys + j] : j) : 0x7fffffff;
    }
    __syncthreads();
    // scores of keys sub, sub + 4, ..., sub + 28
    float s[8];
    float bmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = sub + 4 * jj;
      float acc = 0.f;
      const float* qr = qs + row * DP;
      const float* kr = ks + j * DP;
      for (int c = 0; c < d; ++c) acc = fmaf(qr[c], kr[c], acc);
      const bool vis = j < nk && (kp[j] / p.blk_len) <= qblk;
      s[jj] = vis ? acc : -INFINITY;
      bmax = fmaxf(bmax, s[jj]);
    }
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
    const float m_new = fmaxf(m, bmax);
    float pr[8];
    float psum = 0.f;
    if (m_new == -INFINITY) {
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) pr[jj] = 0.f;
    } else {
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        pr[jj] = exp2f(s[jj] - m_new);
        psum += pr[jj];
      }
      const float alpha = exp2f(m - m_new);
      l *= alpha;
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] *= alpha;
      m = m_new;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l += psum;
    // o[c] += sum_j p_j v[j][sub * cw + c]
    const int lane_base = (threadIdx.x & 31) & ~3;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
#pragma unroll
      for (int ss = 0; ss < 4; ++ss) {
        const float pj = __shfl_sync(0xffffffffu, pr[jj], lane_base + ss);
        const float* vr = vs + (ss + 4 * jj) * DP + sub * cw;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < cw) o[c] = fmaf(pj, vr[c], o[c]);
      }
    }
  }
  if (!row_ok) return;
  const int64_t qh = ((int64_t)b * p.Lq + my_q) * p.Hq + g * G + my_h;
  if (p.n_splits == 1) {
    T* out = static_cast<T*>(p.out) + qh * d + sub * cw;
    const float inv = 1.0f / l;
    for (int c = 0; c < cw; ++c) out[c] = from_f32<T>(o[c] * inv);
  } else {
    const int64_t nq = (int64_t)p.B * p.Lq * p.Hq;
    float* po = p.po + ((int64_t)split * nq + qh) * d + sub * cw;
    for (int c = 0; c < cw; ++c) po[c] = o[c];
    if (sub == 0) {
      p.pm[split * nq + qh] = m;
      p.pl[split * nq + qh] = l;
    }
  }
}

// out[q, h, :] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
template <typename T>
__global__ void attn_merge_kernel(const AttnK p) {
  pdl_enter();
  if (p.live && *p.live == 0) return;
  const int64_t nq = (int64_t)p.B * p.Lq * p.Hq;
  const int64_t qh = blockIdx.x;
  if (qh >= nq) return;
  float M = -INFINITY;
  for (int s = 0; s < p.n_splits; ++s) M = fmaxf(M, p.pm[s * nq + qh]);
  float L = 0.f;
  for (int s = 0; s < p.n_splits; ++s) {
    float ms = p.pm[s * nq + qh];
    if (ms != -INFINITY) L += exp2f(ms - M) * p.pl[s * nq + qh];
  }
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
      float ms = p.pm[s * nq + qh];
      if (ms != -INFINITY) acc += exp2f(ms - M) * p.po[((int64_t)s * nq + qh) * p.d + c];
    }
    static_cast<T*>(p.out)[qh * p.d + c] = from_f32<T>(acc / L);
  }
}

void plan(int B, int Lq, int Hq, int Hkv, int n_keys, int& qt_rows, int& n_qtiles, int& n_splits, int& kps) {
  const int G = Hq / Hkv;
  qt_rows = ROWS / G;
  n_qtiles = (Lq + qt_rows - 1) / qt_rows;
  const int base = B * Hkv * n_qtiles;
  int want = (2 * num_sms() + base - 1) / base;
  int most = max(1, (n_keys + 127) / 128);
  n_splits = max(1, min(want, most));
  kps = ((n_keys + n_splits - 1) / n_splits + KB - 1) / KB * KB;
  n_splits = (n_keys + kps - 1) / kps;
  if (n_splits < 1) n_splits = 1;
}

}  // namespace

size_t attn_simt_workspace_bytes(int B, int Lq, int Hq, int Hkv, int d, int n_keys) {
  int qt, nqt, ns, kps;
  plan(B, Lq, Hq, Hkv, n_keys, qt, nqt, ns, kps);
  if (ns <= 1) return 0;
  const size_t nq = (size_t)B * Lq * Hq;
  return ns * nq * (size_t)d * 4 + 2 * ns * nq * 4 + 512;
}

int launch_attn_simt(const AttnArgs& a, cudaStream_t s) {
  AttnK p;
  p.B = a.B; p.Lq = a.Lq; p.Hq = a.Hq; p.Hkv = a.Hkv; p.d = a.d; p.blk_len = a.blk_len; p.q_pos0 = a.q_pos0;
  p.n_keys = a.n_keys; p.cap = a.cap;
  plan(a.B, a.Lq, a.Hq, a.Hkv, a.n_keys, p.qt_rows, p.n_qtiles, p.n_splits, p.keys_per_split);
  const float scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)a.d);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.q = a.q; p.k = a.k; p.v = a.v; p.key_pos = a.key_pos; p.out = a.out; p.live = a.live;
  p.po = p.pm = p.pl = nullptr;
  if (p.n_splits > 1) {
    const size_t nq = (size_t)a.B * a.Lq * a.Hq;
    const size_t need = p.n_splits * nq * (size_t)a.d * 4 + 2 * p.n_splits * nq * 4;
    DLLM_REQUIRE(a.ws && a.ws_bytes >= need, DLLM_ERR_WORKSPACE, "attention workspace too small (%zu < %zu)",
                 a.ws_bytes, need);
    p.po = static_cast<float*>(a.ws);
    p.pm = p.po + p.n_splits * nq * a.d;
    p.pl = p.pm + p.n_splits * nq;
  }
  const size_t smem = (size_t)(ROWS * DP + 2 * KB * DP) * 4 + KB * 4;
  dim3 grid(a.B * a.Hkv * p.n_qtiles, p.n_splits);
  if (a.dtype == DLLM_BF16) {
    static bool cfg = false;
    if (!cfg) { cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); cfg = true; }
    launch_pdl(attn_simt_kernel<__nv_bfloat16>, grid, 256, smem, s, p);
  } else {
    static bool cfg = false;
    if (!cfg) { cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); cfg = true; }
    launch_pdl(attn_simt_kernel<float>, grid, 256, smem, s, p);
  }
  DLLM_CHECK_LAUNCH("attn_simt_kernel");
  if (p.n_splits > 1) {
    const int nq = a.B * a.Lq * a.Hq;
    if (a.dtype == DLLM_BF16) launch_pdl(attn_merge_kernel<__nv_bfloat16>, nq, 128, 0, s, p);
    else launch_pdl(attn_merge_kernel<float>, nq, 128, 0, s, p);
    DLLM_CHECK_LAUNCH("attn_merge_kernel");
  }
  return DLLM_OK;
}

size_t attn_workspace_bytes(int B, int Lq, int Hq, int Hkv, int d, int n_keys, int dtype) {
  if (attn_tc_supported(dtype, Hq, Hkv, d)) return attn_tc_workspace_bytes(B, Lq, Hq, Hkv, n_keys);
  return attn_simt_workspace_bytes(B, Lq, Hq, Hkv, d, n_keys);
}

int launch_attn(const AttnArgs& a, int32_t* status, cudaStream_t s) {
  if (attn_tc_supported(a.dtype, a.Hq, a.Hkv, a.d)) return launch_attn_tc(a, status, s);
  return launch_attn_simt(a, s);
}

int launch_attn_merge(const AttnArgs& a, int n_splits, float* po, float* pm, float* pl, cudaStream_t s) {
  AttnK p{};
  p.B = a.B; p.Lq = a.Lq; p.Hq = a.Hq; p.d = a.d; p.n_splits = n_splits;
  p.po = po; p.pm = pm; p.pl = pl; p.out = a.out;
  const int nq = a.B * a.Lq * a.Hq;
  if (a.dtype == DLLM_BF16) launch_pdl(attn_merge_kernel<__nv_bfloat16>, nq, 128, 0, s, p);
  else launch_pdl(attn_merge_kernel<float>, nq, 128, 0, s, p);
  DLLM_CHECK_LAUNCH("attn_merge_kernel");
  return DLLM_OK;
}

}  // namespace dllm
