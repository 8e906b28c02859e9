// MoE router: sigmoid expert scores, bias-steered top-k selection with renormalised unbiased gates, and the
// stable per-expert permutation of the (token, slot) assignments consumed by the grouped expert GEMMs.
// Source: LLaDA2.0-Uni paper review, sections "MoE 백본과 Block-wise Attention" (top-k experts per token) and
// "Load Balancing — Auxiliary-loss-free MoE Bias" (a per-expert bias that steers which experts are picked).
#include "common.cuh"
#include "misc.h"
#include "kernels.h"

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
  pdl_enter();
  extern __shared__ __align__(16) unsigned char hs_raw[];
  T* hs = reinterpret_cast<T*>(hs_raw);  // [TT][H]
  const int e0 = blockIdx.x * EW, t0 = blockIdx.y * TT;
  const int nt = min(TT, Tk - t0);
  const int vec = 16 / (int)sizeof(T);
  const int nvec = TT * H / vec;
  const int valid_vec = nt * H / vec;            // vectors of the valid token rows (rows are contiguous)
  const uint4* src = reinterpret_cast<const uint4*>(h + (int64_t)t0 * H);
  // 8 independent loads in flight per thread
  for (int i0 = threadIdx.x; i0 < nvec; i0 += 8 * blockDim.x) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      v[u] = (i < valid_vec) ? src[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < nvec) reinterpret_cast<uint4*>(hs)[i] = v[u];
    }
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
// Lane l holds experts l, l + 32, ... in registers (biased and unbiased); the winner's unbiased score comes from the
// owning lane by a shuffle, so the rounds touch no memory.
// With from_logits the row holds router logits: the sigmoid scores replace them in place.
__global__ void route_topk_kernel(float* __restrict__ scores, const float* __restrict__ bias, int Tk, int E, int k,
                                  int from_logits, int32_t* __restrict__ ids, float* __restrict__ gates) {
  pdl_enter();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= Tk) return;
  float* s = scores + (int64_t)warp * E;
  float val[32], raw[32];
  const int per = (E + 31) / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = i * 32 + lane;
    const bool in = i < per && e < E;
    float v = in ? s[e] : 0.f;
    if (from_logits && in) {
      v = 1.0f / (1.0f + expf(-v));
      s[e] = v;
    }
    raw[i] = v;
    val[i] = in ? v + bias[e] : -INFINITY;
  }
  float gsum = 0.f, my_gate = 0.f;
  int my_id = 0;
  // each lane's best (value, expert); only the winning lane rescans its own values after a round
  auto lane_best = [&](float& bv, int& be) {
    bv = -INFINITY;
    be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = i * 32 + lane;
      if (i < per && (val[i] > bv || (val[i] == bv && e < be))) { bv = val[i]; be = e; }
    }
  };
  float lbv;
  int lbe;
  lane_best(lbv, lbe);
  for (int j = 0; j < k; ++j) {
    float bv = lbv;
    int be = lbe;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    float mine = 0.f;
    if ((be & 31) == lane) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i * 32 + lane == be) { mine = raw[i]; val[i] = -INFINITY; }
      lane_best(lbv, lbe);
    }
    const float sc = __shfl_sync(0xffffffffu, mine, be & 31);
    gsum += sc;
    if (lane == j) { my_id = be; my_gate = sc; }
  }
  if (lane < k) {
    ids[(int64_t)warp * k + lane] = my_id;
    gates[(int64_t)warp * k + lane] = my_gate / gsum;
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
  pdl_enter();
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
  // bf16 with a tensor-core friendly shape: router logits through the tcgen05 projection (fp32 out, accumulated
  // in fp32 in the MMA's fixed order); otherwise the SIMT score kernel
  const bool tc_logits = dtype == DLLM_BF16 && E % 128 == 0 && H % 64 == 0;
  if (tc_logits) {
    GemmArgs g;
    g.x = h; g.x_rows = Tk; g.w = w_router; g.w_rows = E; g.K = H; g.M = E; g.host_cnt = Tk; g.max_cnt = Tk;
    g.cnt_bound = Tk; g.dtype = DLLM_BF16;
    g.epi.kind = EPI_STORE; g.epi.out = scores; g.epi.ldo = E; g.epi.out_f32 = 1;
    int st = gemm_bf16_tc(g, s);
    if (st) return st;
    launch_pdl(route_topk_kernel, (Tk + 7) / 8, 256, 0, s, scores, bias, Tk, E, k, 1, ids, gates);
    DLLM_CHECK_LAUNCH("route_topk_kernel");
    launch_pdl(route_permute_kernel, E, 256, 0, s, ids, Tk * k, E, counts, offsets, perm, inv);
    DLLM_CHECK_LAUNCH("route_permute_kernel");
    return DLLM_OK;
  }
  dim3 g1((E + EW - 1) / EW, (Tk + TT - 1) / TT);
  const size_t smem = (size_t)TT * H * (dtype == DLLM_BF16 ? 2 : 4);
  if (dtype == DLLM_BF16) {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_scores_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           200 * 1024);
      cfg = true;
    }
    launch_pdl(route_scores_kernel<__nv_bfloat16>, g1, 256, smem, s, (const __nv_bfloat16*)h,
                                                             (const __nv_bfloat16*)w_router, Tk, H, E, scores);
  } else {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_scores_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cfg = true;
    }
    launch_pdl(route_scores_kernel<float>, g1, 256, smem, s, (const float*)h, (const float*)w_router, Tk, H, E, scores);
  }
  DLLM_CHECK_LAUNCH("route_scores_kernel");
  launch_pdl(route_topk_kernel, (Tk + 7) / 8, 256, 0, s, scores, bias, Tk, E, k, 0, ids, gates);
  DLLM_CHECK_LAUNCH("route_topk_kernel");
  launch_pdl(route_permute_kernel, E, 256, 0, s, ids, Tk * k, E, counts, offsets, perm, inv);
  DLLM_CHECK_LAUNCH("route_permute_kernel");
  return DLLM_OK;
}

}  // namespace dllm
