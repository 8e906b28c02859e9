// MoE router: sigmoid expert scores, bias-steered top-k selection with renormalised unbiased gates, and the
// stable per-expert permutation of the (token, slot) assignments consumed by the grouped expert GEMMs.
// Source: LLaDA2.0-Uni paper review, sections "MoE 백본과 Block-wise Attention" (top-k experts per token) and
// "Load Balancing — Auxiliary-loss-free MoE Bias" (a per-expert bias that steers which experts are picked).
#include "common.cuh"
#include "misc.h"
#include "kernels.h"
#include <algorithm>

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
// Top-k of one token's expert scores, one warp. Lane l owns experts e = i * 32 + l (i < PER); the selection key is
// the biased score val = raw + bias (ties to the lower expert), the gate the unbiased raw score, renormalised over
// the chosen k. Each lane sorts its PER candidates with an insertion network (descending val, ascending e); then
// k rounds take the warp-wide best head (a 5-step butterfly on (val, e)) and the winning lane pops its head.
// With from_logits the raw scores are sigmoid(logit) and are written back over the logits.
template <int PER>
DLLM_DEV void warp_topk(float* __restrict__ srow, const float* __restrict__ bias, int E, int k, int from_logits,
                        int lane, int& my_id, float& my_gate) {
  float v[PER], r[PER];
  int e[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int ex = i * 32 + lane;
    const bool in = ex < E;
    float x = in ? srow[ex] : 0.f;
    if (from_logits && in) {
      x = 1.0f / (1.0f + expf(-x));
      srow[ex] = x;
    }
    r[i] = x;
    v[i] = in ? x + bias[ex] : -INFINITY;
    e[i] = in ? ex : 0x7fffffff;
  }
  // insertion network: after step i, entries [0, i] are sorted (PER <= 8; wider rows keep the unsorted
  // candidates and the winning lane rescans them, below)
#pragma unroll
  for (int i = 1; i < (PER <= 8 ? PER : 1); ++i) {
#pragma unroll
    for (int j = i; j > 0; --j) {
      const bool sw = v[j] > v[j - 1] || (v[j] == v[j - 1] && e[j] < e[j - 1]);
      const float tv = v[j], tr = r[j];
      const int te = e[j];
      v[j] = sw ? v[j - 1] : tv; r[j] = sw ? r[j - 1] : tr; e[j] = sw ? e[j - 1] : te;
      v[j - 1] = sw ? tv : v[j - 1]; r[j - 1] = sw ? tr : r[j - 1]; e[j - 1] = sw ? te : e[j - 1];
    }
  }
  if (PER > 8) {
#pragma unroll
    for (int i = 1; i < PER; ++i) {
      const bool sw = v[i] > v[0] || (v[i] == v[0] && e[i] < e[0]);
      const float tv = v[i], tr = r[i];
      const int te = e[i];
      v[i] = sw ? v[0] : tv; r[i] = sw ? r[0] : tr; e[i] = sw ? e[0] : te;
      v[0] = sw ? tv : v[0]; r[0] = sw ? tr : r[0]; e[0] = sw ? te : e[0];
    }
  }
  float gsum = 0.f;
  my_id = 0;
  my_gate = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = v[0];
    int be = e[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    const int win = be & 31;
    const float sc = __shfl_sync(0xffffffffu, r[0], win);
    if (lane == win) {
      if (PER <= 8) {   // pop the sorted head
#pragma unroll
        for (int i = 0; i + 1 < PER; ++i) { v[i] = v[i + 1]; r[i] = r[i + 1]; e[i] = e[i + 1]; }
        v[PER - 1] = -INFINITY;
        e[PER - 1] = 0x7fffffff;
      } else {          // drop the winner and move this lane's next best to slot 0
        v[0] = -INFINITY;
        e[0] = 0x7fffffff;
#pragma unroll
        for (int i = 1; i < PER; ++i) {
          const bool sw = v[i] > v[0] || (v[i] == v[0] && e[i] < e[0]);
          const float tv = v[i], tr = r[i];
          const int te = e[i];
          v[i] = sw ? v[0] : tv; r[i] = sw ? r[0] : tr; e[i] = sw ? e[0] : te;
          v[0] = sw ? tv : v[0]; r[0] = sw ? tr : r[0]; e[0] = sw ? te : e[0];
        }
      }
    }
    gsum += sc;
    if (lane == j) { my_id = be; my_gate = sc; }
  }
  my_gate = my_gate / gsum;
}

// One warp per token.
template <int PER>
__global__ void route_topk_kernel(float* __restrict__ scores, const float* __restrict__ bias, int Tk, int E, int k,
                                  int from_logits, int32_t* __restrict__ ids, float* __restrict__ gates) {
  pdl_enter();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= Tk) return;
  int my_id;
  float my_gate;
  warp_topk<PER>(scores + (int64_t)warp * E, bias, E, k, from_logits, lane, my_id, my_gate);
  if (lane < k) {
    ids[(int64_t)warp * k + lane] = my_id;
    gates[(int64_t)warp * k + lane] = my_gate;
  }
}

// Few tokens (Tk <= 32, Tk * k <= 1024, E <= 256): top-k and the stable per-expert permutation in one CTA of
// 1024 threads. Assignment a = t * k + j; chunk c = a / 32 is handled by one warp, whose lanes with the same expert
// find each other with __match_any_sync: an assignment's position is offsets[e] + (assignments of e in earlier
// chunks) + (lanes of e before it in its chunk), which is the order of a, as in the general permutation kernel.
template <int PER>
__global__ void __launch_bounds__(1024) route_small_kernel(float* __restrict__ scores, const float* __restrict__ bias,
                                                           int Tk, int E, int k, int from_logits,
                                                           int32_t* __restrict__ ids, float* __restrict__ gates,
                                                           int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  pdl_enter();
  extern __shared__ int rs_sm[];
  const int n = Tk * k, W = (n + 31) / 32;
  int* hist = rs_sm;                 // [W][E]: counts per chunk, then their exclusive prefix over chunks
  int* ids_s = hist + W * E;         // [n]
  int* rk_s = ids_s + n;             // [n]: rank among the chunk's lanes with the same expert
  int* off_s = rk_s + n;             // [E]
  __shared__ int wtot[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  for (int i = tid; i < W * E; i += blockDim.x) hist[i] = 0;
  for (int t = warp; t < Tk; t += nw) {
    int my_id;
    float my_gate;
    warp_topk<PER>(scores + (int64_t)t * E, bias, E, k, from_logits, lane, my_id, my_gate);
    if (lane < k) {
      ids[(int64_t)t * k + lane] = my_id;
      gates[(int64_t)t * k + lane] = my_gate;
      ids_s[t * k + lane] = my_id;
    }
  }
  __syncthreads();
  for (int c = warp; c < W; c += nw) {
    const int a = c * 32 + lane;
    const int ex = a < n ? ids_s[a] : -1;
    const unsigned grp = __match_any_sync(0xffffffffu, ex);
    if (a < n) {
      rk_s[a] = __popc(grp & ((1u << lane) - 1u));
      if (lane == __ffs(grp) - 1) hist[c * E + ex] = __popc(grp);
    }
  }
  __syncthreads();
  // per expert: prefix over chunks, total count
  for (int ex = tid; ex < E; ex += blockDim.x) {
    int run = 0;
    for (int c = 0; c < W; ++c) {
      const int h = hist[c * E + ex];
      hist[c * E + ex] = run;
      run += h;
    }
    off_s[ex] = run;
  }
  __syncthreads();
  // exclusive scan of the counts over experts (E <= 1024 = one entry per thread)
  const int cnt = tid < E ? off_s[tid] : 0;
  int inc = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wtot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int x = lane < nw ? wtot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    wtot[lane] = x;   // inclusive over warps
  }
  __syncthreads();
  const int excl = inc - cnt + (warp > 0 ? wtot[warp - 1] : 0);
  __syncthreads();
  if (tid < E) {
    off_s[tid] = excl;
    counts[tid] = cnt;
    offsets[tid] = excl;
  }
  if (tid == 0) offsets[E] = n;
  __syncthreads();
  for (int a = tid; a < n; a += blockDim.x) {
    const int ex = ids_s[a];
    const int pos = off_s[ex] + hist[(a >> 5) * E + ex] + rk_s[a];
    perm[pos] = a;
    inv[a] = pos;
  }
}

// Stable permutation for many assignments, in three launches over segments of `seg` consecutive assignments
// (seg a multiple of 256): per-segment expert histograms; one CTA turns them into counts, offsets and every segment's
// first output position per expert; then each segment writes its assignments' positions in order. Positions within
// an expert follow the assignment index a = t * k + j, so an expert's rows stay sorted by token.

// seg_hist[s][e] = assignments of expert e in segment s.
__global__ void __launch_bounds__(256) route_seg_hist_kernel(const int32_t* __restrict__ ids, int n, int E, int seg,
                                                             int32_t* __restrict__ seg_hist) {
  pdl_enter();
  extern __shared__ int sh_hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sh_hist[i] = 0;
  __syncthreads();
  const int a0 = blockIdx.x * seg, a1 = min(n, a0 + seg);
  for (int a = a0 + threadIdx.x; a < a1; a += blockDim.x) atomicAdd(&sh_hist[ids[a]], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) seg_hist[(int64_t)blockIdx.x * E + i] = sh_hist[i];
}

// counts = column sums of the segment histograms, offsets = their exclusive scan over experts (offsets[E] = n), and
// seg_hist[s][e] replaced by offsets[e] + (assignments of e in segments before s). 1024 threads: G = 1024 / E32
// groups of segments per expert column (E32 = E rounded up to 32), each summing its contiguous share of the
// segments; the groups' sums are prefixed per expert in shared memory.
__global__ void __launch_bounds__(1024) route_seg_scan_kernel(int32_t* __restrict__ seg_hist, int S, int E, int n,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets) {
  pdl_enter();
  __shared__ int part[1024];   // [group][expert]
  __shared__ int wtot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E32 = (E + 31) & ~31, G = 1024 / E32;
  const int g = tid / E32, e = tid - g * E32;
  const int per = (S + G - 1) / G, s0 = min(S, g * per), s1 = min(S, s0 + per);
  int sum = 0;
  if (g < G && e < E) {
#pragma unroll 8
    for (int sg = s0; sg < s1; ++sg) sum += seg_hist[(int64_t)sg * E + e];
  }
  part[tid] = sum;
  __syncthreads();
  // expert totals and their exclusive scan: threads of group 0 (one per expert column)
  int cnt = 0;
  if (tid < E32)
    for (int q = 0; q < G; ++q) cnt += part[q * E32 + tid];
  int inc = cnt;
  if (warp < E32 / 32) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wtot[warp] = inc;
  }
  __syncthreads();
  if (warp == 0) {
    int x = lane < E32 / 32 ? wtot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    wtot[lane] = x;   // inclusive over warps
  }
  __syncthreads();
  if (tid < E32) {
    const int excl = inc - cnt + (warp > 0 ? wtot[warp - 1] : 0);
    if (tid < E) { counts[tid] = cnt; offsets[tid] = excl; }
    // the groups' starting positions per expert
    int run = excl;
    for (int q = 0; q < G; ++q) {
      const int v = part[q * E32 + tid];
      part[q * E32 + tid] = run;
      run += v;
    }
  }
  if (tid == 0) offsets[E] = n;
  __syncthreads();
  if (g < G && e < E) {
    int run = part[tid];
    for (int sg = s0; sg < s1; ++sg) {
      const int v = seg_hist[(int64_t)sg * E + e];
      seg_hist[(int64_t)sg * E + e] = run;
      run += v;
    }
  }
}

// Segment s: its 8 warps take seg / 8 consecutive assignments each (whole 32-assignment chunks). Pass 1 counts
// each warp's assignments per expert (lanes with the same expert find each other with __match_any_sync and the
// group's first lane adds the group size); the warps' counts are prefixed per expert on top of the segment's first
// positions; pass 2 walks the chunks again and writes position = warp's running base + rank among the chunk's
// lanes with the same expert.
__global__ void __launch_bounds__(256) route_seg_scatter_kernel(const int32_t* __restrict__ ids, int n, int E, int seg,
                                                                const int32_t* __restrict__ seg_base,
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  pdl_enter();
  extern __shared__ int wh[];   // [8][E]
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < 8 * E; i += blockDim.x) wh[i] = 0;
  __syncthreads();
  const int per = seg / 8;
  const int w0 = blockIdx.x * seg + w * per, w1 = min(n, w0 + per);
  for (int c = w0; c < w1; c += 32) {
    const int a = c + lane;
    const int ex = a < w1 ? ids[a] : -1;
    const unsigned grp = __match_any_sync(0xffffffffu, ex);
    if (a < w1 && lane == __ffs(grp) - 1) wh[w * E + ex] += __popc(grp);
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = seg_base[(int64_t)blockIdx.x * E + e];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int v = wh[q * E + e];
      wh[q * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  for (int c = w0; c < w1; c += 32) {
    const int a = c + lane;
    const int ex = a < w1 ? ids[a] : -1;
    const unsigned grp = __match_any_sync(0xffffffffu, ex);
    if (a < w1) {
      const int pos = wh[w * E + ex] + __popc(grp & ((1u << lane) - 1u));
      perm[pos] = a;
      inv[a] = pos;
    }
    __syncwarp();
    if (a < w1 && lane == __ffs(grp) - 1) wh[w * E + ex] += __popc(grp);
    __syncwarp();
  }
}

}  // namespace

template <int PER>
int launch_select_per(float* scores, const float* bias, int Tk, int E, int k, int from_logits, int32_t* ids,
                      float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                      int32_t* seg_scratch, cudaStream_t s) {
  if constexpr (PER <= 8) {   // E <= 256: the single-CTA kernel fits its 64 registers per thread
    const int n = Tk * k, W = (n + 31) / 32;
    const size_t smem = ((size_t)W * E + 2 * (size_t)n + E) * sizeof(int);
    if (Tk <= 32 && n <= 1024 && smem <= 96 * 1024) {
      static bool cfg = false;
      if (!cfg) {
        cudaFuncSetAttribute(route_small_kernel<PER>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        cfg = true;
      }
      launch_pdl(route_small_kernel<PER>, 1, 1024, smem, s, scores, bias, Tk, E, k, from_logits, ids, gates, counts,
                 offsets, perm, inv);
      DLLM_CHECK_LAUNCH("route_small_kernel");
      return DLLM_OK;
    }
  }
  // one warp per token, 4 per CTA: many tokens spread over all the SMs (one thread per token, tried for thousands
  // of tokens, reads each 1 KB score row with 32 lines in flight per warp instruction and was 2x slower)
  launch_pdl(route_topk_kernel<PER>, (Tk + 3) / 4, 128, 0, s, scores, bias, Tk, E, k, from_logits, ids, gates);
  DLLM_CHECK_LAUNCH("route_topk_kernel");
  const int n = Tk * k, seg = route_segment(n), S = (n + seg - 1) / seg;
  launch_pdl(route_seg_hist_kernel, S, 256, (size_t)E * sizeof(int), s, (const int32_t*)ids, n, E, seg, seg_scratch);
  DLLM_CHECK_LAUNCH("route_seg_hist_kernel");
  launch_pdl(route_seg_scan_kernel, 1, 1024, 0, s, seg_scratch, S, E, n, counts, offsets);
  DLLM_CHECK_LAUNCH("route_seg_scan_kernel");
  launch_pdl(route_seg_scatter_kernel, S, 256, (size_t)8 * E * sizeof(int), s, (const int32_t*)ids, n, E, seg,
             (const int32_t*)seg_scratch, perm, inv);
  DLLM_CHECK_LAUNCH("route_seg_scatter_kernel");
  return DLLM_OK;
}

// Selection and permutation from fp32 scores (sigmoid applied here when from_logits), E <= 1024.
int launch_select(float* scores, const float* bias, int Tk, int E, int k, int from_logits, int32_t* ids,
                  float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* seg,
                  cudaStream_t s) {
  if (E <= 32) return launch_select_per<1>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
  if (E <= 64) return launch_select_per<2>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
  if (E <= 128) return launch_select_per<4>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
  if (E <= 256) return launch_select_per<8>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
  if (E <= 512) return launch_select_per<16>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
  return launch_select_per<32>(scores, bias, Tk, E, k, from_logits, ids, gates, counts, offsets, perm, inv, seg, s);
}

int route_segment(int n_assign) {
  // a multiple of 256 assignments (8 warps x 32), at most about 128 segments
  return std::max(256, ((n_assign + 127) / 128 + 255) / 256 * 256);
}

size_t route_scratch_bytes(int Tk, int E, int k) {
  const int n = std::max(Tk, 0) * k, seg = route_segment(n);
  return (size_t)std::max(1, (n + seg - 1) / seg) * (size_t)E * sizeof(int32_t);
}

int launch_route(int dtype, const void* h, const void* w_router, const float* bias, int Tk, int H, int E, int k,
                 int32_t* ids, float* gates, float* scores, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* inv, int32_t* seg_scratch, cudaStream_t s) {
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
    return launch_select(scores, bias, Tk, E, k, 1, ids, gates, counts, offsets, perm, inv, seg_scratch, s);
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
  return launch_select(scores, bias, Tk, E, k, 0, ids, gates, counts, offsets, perm, inv, seg_scratch, s);
}

}  // namespace dllm
