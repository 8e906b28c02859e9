// MoE router: sigmoid expert scores, bias-steered top-k selection with renormalised unbiased gates, and the
// stable per-expert permutation of the (token, slot) assignments consumed by the grouped expert GEMMs.
// Source: LLaDA2.0-Uni paper review, sections "MoE 백본과 Block-wise Attention" (top-k experts per token) and
// "Load Balancing — Auxiliary-loss-free MoE Bias" (a per-expert bias that steers which experts are picked).
#include "common.cuh"
#include "misc.h"

namespace dllm {
namespace {

constexpr int TT = 16;   // tokens per CTA of the score kernel
constexpr int EW = 8;    // experts per CTA (one per warp)

DLLM_DEV void load8(const __nv_bfloat16* p, float* f) { bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f); }
DLLM_DEV void load8(const float* p, float* f) {
  float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// scores[t, e] = sigmoid(sum_i h[t, i] w[e, i]) in fp32. One warp per expert streams its router row in 8-element
// vectors (lane l owns elements l*8 + 256 j + u) and applies each vector to the CTA's TT token rows held in shared
// memory; each lane sums its elements in increasing j, u, then a fixed butterfly adds the lanes, so the order of
// the fp32 sum is the same on every run.
template <typename T>
__global__ void __launch_bounds__(256) route_scores_kernel(const T* __restrict__ h, const T* __restrict__ w, int Tk,
                                                           int H, int E, float* __restrict__ scores) {
  extern __shared__ __align__(16) unsigned char hs_raw[];
  T* hs = reinterpret_cast<T*>(hs_raw);  // [TT][H]
  const int e0 = blockIdx.x * EW, t0 = blockIdx.y * TT;
  const int nt = min(TT, Tk - t0);
  const int vec = 16 / (int)sizeof(T);
  const int nvec = TT * H / vec;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const int tt = (i * vec) / H;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tt < nt) v = reinterpret_cast<const uint4*>(h + (int64_t)t0 * H)[i];
    reinterpret_cast<uint4*>(hs)[i] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = e0 + warp;
  if (e >= E) return;
  const T* wr = w + (int64_t)e * H;
  float acc[TT];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) acc[tt] = 0.f;
#pragma unroll 4
  for (int c = lane * 8; c < H; c += 256) {
    float wf[8];
    load8(wr + c, wf);
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      float hf[8];
      load8(hs + tt * H + c, hf);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[tt] = fmaf(wf[u], hf[u], acc[tt]);
    }
  }
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    const float v = warp_sum(acc[tt]);
    if (lane == 0 && tt < nt) scores[(int64_t)(t0 + tt) * E + e] = 1.0f / (1.0f + expf(-v));
  }
}

// One warp per token: k rounds of warp arg-max over s + bias (ties -> lower expert id); gates = s / sum(s).
__global__ void route_topk_kernel(const float* __restrict__ scores, const float* __restrict__ bias, int Tk, int E,
                                  int k, int32_t* __restrict__ ids, float* __restrict__ gates) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= Tk) return;
  const float* s = scores + (int64_t)warp * E;
  float val[32];
  const int per = (E + 31) / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    int e = i * 32 + lane;
    val[i] = (i < per && e < E) ? s[e] + bias[e] : -INFINITY;
  }
  float gsum = 0.f;
  float sel_s[32];
  int sel_e[32];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      int e = i * 32 + lane;
      if (val[i] > bv || (val[i] == bv && e < be)) { bv = val[i]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i * 32 + lane == be) val[i] = -INFINITY;
    sel_e[j] = be;
    sel_s[j] = s[be];
    gsum += sel_s[j];
  }
  if (lane == 0) {
    for (int j = 0; j < k; ++j) {
      ids[(int64_t)warp * k + j] = sel_e[j];
      gates[(int64_t)warp * k + j] = sel_s[j] / gsum;
    }
  }
}

// Exclusive scan of n <= 1024 ints in shared memory by 256 threads (4 consecutive items per thread).
__device__ void block_exclusive_scan(int* a, int n, int* total) {
  __shared__ int wsum[8];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int v[4], s = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    int i = tid * 4 + u;
    v[u] = i < n ? a[i] : 0;
    s += v[u];
  }
  int inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[w] = inc;
  __syncthreads();
  int before = 0, tot = 0;
  for (int i = 0; i < 8; ++i) {
    if (i < w) before += wsum[i];
    tot += wsum[i];
  }
  int run = before + inc - s;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    int i = tid * 4 + u;
    if (i < n) a[i] = run;
    run += v[u];
  }
  if (total) *total = tot;
  __syncthreads();
}

// One CTA per expert: histogram of all assignments, offsets by exclusive scan, then this expert's rows in
// increasing assignment order (t * k + j), which keeps the rows of an expert sorted by token.
__global__ void route_permute_kernel(const int32_t* __restrict__ ids, int n_assign, int E, int32_t* counts,
                                     int32_t* offsets, int32_t* perm, int32_t* inv) {
  __shared__ int hist[1024];
  __shared__ int cnt_e;
  __shared__ int wtot[8];
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int a = tid; a < n_assign; a += blockDim.x) atomicAdd(&hist[ids[a]], 1);
  __syncthreads();
  if (tid == 0) cnt_e = hist[e];
  __syncthreads();
  int total = 0;
  if (blockIdx.x == 0)
    for (int i = tid; i < E; i += blockDim.x) counts[i] = hist[i];
  __syncthreads();
  block_exclusive_scan(hist, E, &total);
  const int off = hist[e];
  if (blockIdx.x == 0) {
    for (int i = tid; i < E; i += blockDim.x) offsets[i] = hist[i];
    if (tid == 0) offsets[E] = total;
  }
  if (cnt_e == 0) return;
  int base = 0;
  for (int a0 = 0; a0 < n_assign; a0 += blockDim.x) {
    const int a = a0 + tid;
    const int f = (a < n_assign && ids[a] == e) ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wtot[w] = __popc(bal);
    __syncthreads();
    int before = 0, tot = 0;
    for (int i = 0; i < 8; ++i) {
      if (i < w) before += wtot[i];
      tot += wtot[i];
    }
    if (f) {
      const int r = off + base + before + __popc(bal & ((1u << lane) - 1u));
      perm[r] = a;
      inv[a] = r;
    }
    base += tot;
    __syncthreads();
  }
}

}  // namespace

int launch_route(int dtype, const void* h, const void* w_router, const float* bias, int Tk, int H, int E, int k,
                 int32_t* ids, float* gates, float* scores, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* inv, cudaStream_t s) {
  if (Tk <= 0) return DLLM_OK;
  dim3 g1((E + EW - 1) / EW, (Tk + TT - 1) / TT);
  const size_t smem = (size_t)TT * H * (dtype == DLLM_BF16 ? 2 : 4);
  if (dtype == DLLM_BF16) {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_scores_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           200 * 1024);
      cfg = true;
    }
    route_scores_kernel<__nv_bfloat16><<<g1, 256, smem, s>>>((const __nv_bfloat16*)h,
                                                             (const __nv_bfloat16*)w_router, Tk, H, E, scores);
  } else {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_scores_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cfg = true;
    }
    route_scores_kernel<float><<<g1, 256, smem, s>>>((const float*)h, (const float*)w_router, Tk, H, E, scores);
  }
  DLLM_CHECK_LAUNCH("route_scores_kernel");
  route_topk_kernel<<<(Tk + 7) / 8, 256, 0, s>>>(scores, bias, Tk, E, k, ids, gates);
  DLLM_CHECK_LAUNCH("route_topk_kernel");
  route_permute_kernel<<<E, 256, 0, s>>>(ids, Tk * k, E, counts, offsets, perm, inv);
  DLLM_CHECK_LAUNCH("route_permute_kernel");
  return DLLM_OK;
}

}  // namespace dllm
