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
                                                           int H, int E, float* __restrict__ scores,
                                                           const int32_t* __restrict__ live,
                                                           unsigned* __restrict__ zero_word) {
  pdl_enter();
  if (zero_word && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *zero_word = 0u;   // the next kernel's ticket
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
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

// Guard band of the fp32 selection. The fp32 scores (tensor-core or SIMT accumulation over H, then an fp32
// sigmoid) are within a few 1e-6 of the exact scores of the same inputs; a token whose fp32 biased scores have two
// neighbours among its top k + 1 closer than kRouteGuard (so that rounding could change the chosen set or the slot
// order) is decided again from exact scores (exact_redecide). Any expert whose fp32 biased score is below the
// (k+1)-th by more than the guard cannot reach the top k, so only the experts within the guard of the (k+1)-th
// score or above it are re-scored.
constexpr float kRouteGuard = 1e-5f;

// Order-preserving map of a float to an unsigned key (and back): larger floats get larger keys, -inf the smallest.
DLLM_DEV uint32_t ord_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
DLLM_DEV float ord_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k of one token's expert scores, one warp. Lane l owns experts e = i * 32 + l (i < PER); the selection key is
// the biased score val = raw + bias (ties to the lower expert), the gate the unbiased raw score, renormalised over
// the chosen k. Each lane sorts its PER candidates with an insertion network (descending val, ascending e); then
// k rounds take the warp-wide best head (two warp reductions: the largest val, then the lowest e holding it) and
// the winning lane pops its head; one
// more round reads the (k+1)-th value without popping it. With from_logits the raw scores are sigmoid(logit) and
// are written back over the logits. Returns (warp-uniform) whether two consecutive values among the top k + 1
// are closer than kRouteGuard; thr is then the (k+1)-th value minus the guard (-inf when k == E).
template <int PER>
DLLM_DEV bool warp_topk(float* __restrict__ srow, const float* __restrict__ bias, int E, int k, int from_logits,
                        int lane, int& my_id, float& my_gate, float& thr) {
  float v[PER], r[PER];
  int e[PER];
  // every load of the row (and of the bias) in flight before the first use: the row was just written by another
  // kernel, and loads issued one after another behind the write-back of each sigmoid would pay the L2 round trip
  // PER times
  float xs[PER], bs[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int ex = i * 32 + lane;
    xs[i] = ex < E ? __ldcg(srow + ex) : 0.f;
    bs[i] = ex < E ? __ldg(bias + ex) : 0.f;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int ex = i * 32 + lane;
    const bool in = ex < E;
    float x = xs[i];
    if (from_logits && in) {
      // intrinsic exponential and approximate divide: within about 1e-6 relative of the rounded sigmoid, an order
      // below the guard band
      x = __fdividef(1.0f, 1.0f + __expf(-x));
      srow[ex] = x;
    }
    r[i] = x;
    v[i] = in ? x + bs[i] : -INFINITY;
    e[i] = in ? ex : 0x7fffffff;
  }
  // each lane's candidates in order, largest first (ties: lower expert first). Eight: Batcher's odd-even merge
  // network (19 comparators in 6 layers, so the chain of dependent compares is 6 long); fewer: an insertion
  // network; more than eight: the lane keeps them unsorted and the winning lane rescans them (below)
  auto cas = [&](int i, int j) {   // entry i gets the better of entries i and j
    const bool sw = v[j] > v[i] || (v[j] == v[i] && e[j] < e[i]);
    const float tv = v[i], tr = r[i];
    const int te = e[i];
    v[i] = sw ? v[j] : tv; r[i] = sw ? r[j] : tr; e[i] = sw ? e[j] : te;
    v[j] = sw ? tv : v[j]; r[j] = sw ? tr : r[j]; e[j] = sw ? te : e[j];
  };
  if constexpr (PER == 8) {
    cas(0, 1); cas(2, 3); cas(4, 5); cas(6, 7);
    cas(0, 2); cas(1, 3); cas(4, 6); cas(5, 7);
    cas(1, 2); cas(5, 6);
    cas(0, 4); cas(1, 5); cas(2, 6); cas(3, 7);
    cas(2, 4); cas(3, 5);
    cas(1, 2); cas(3, 4); cas(5, 6);
  }
#pragma unroll
  for (int i = 1; i < (PER < 8 ? PER : 1); ++i) {
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
  float gsum = 0.f, prev = 0.f;
  bool near = false;
  thr = -INFINITY;
  my_id = 0;
  my_gate = 0.f;
  const int rounds = k < E ? k + 1 : k;
  for (int j = 0; j < rounds; ++j) {
    // the warp's best head: the largest value (an order-preserving unsigned image of the float, one warp
    // reduction), then the lowest expert among the heads that hold it (a second one)
    const uint32_t key = ord_key(v[0]);
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
    const int be = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)e[0] : 0xffffffffu);
    const float bv = ord_value(kmax);
    if (j > 0 && prev - bv < kRouteGuard) near = true;
    prev = bv;
    if (j == k) {   // the (k+1)-th value: read, not taken
      thr = bv - kRouteGuard;
      break;
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
  return near;
}

// Exact dot product of two rows of H elements (H % 8 == 0), one warp; every lane returns the sum. A product of two
// bf16 values is exact in fp32 (8 + 8 significant bits), so bf16 rows add fp32 products in fp64; fp32 rows use
// fp64 fused multiply-adds. Either way the sum of H = 2048 terms is within about 1e-13 of the exact value. Each
// lane has UNR 8-element chunks of both rows in flight at a time (the rows come from L2).
DLLM_DEV void dot_chunk(const uint4& ua, const uint4& ub, double& s0, double& s1, const __nv_bfloat16*) {
  float fa[8], fb[8];
  bf16x8_to_f32(ua, fa);
  bf16x8_to_f32(ub, fb);
#pragma unroll
  for (int u = 0; u < 8; u += 2) {
    s0 += (double)(fa[u] * fb[u]);
    s1 += (double)(fa[u + 1] * fb[u + 1]);
  }
}
template <int UNR = 4, typename T>
DLLM_DEV double warp_dot64(const T* __restrict__ a, const T* __restrict__ b, int H, int lane) {
  constexpr int VE = 16 / sizeof(T);          // elements per 16-byte load
  constexpr int CH = 8;                        // elements per lane per chunk
  double s0 = 0.0, s1 = 0.0;
  for (int c0 = lane * CH; c0 < H; c0 += UNR * 32 * CH) {
    uint4 ua[UNR][CH / VE], ub[UNR][CH / VE];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int c = c0 + u * 32 * CH;
#pragma unroll
      for (int v = 0; v < CH / VE; ++v) {
        ua[u][v] = c < H ? *reinterpret_cast<const uint4*>(a + c + v * VE) : make_uint4(0, 0, 0, 0);
        ub[u][v] = c < H ? *reinterpret_cast<const uint4*>(b + c + v * VE) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      if constexpr (sizeof(T) == 2) {
        dot_chunk(ua[u][0], ub[u][0], s0, s1, a);
      } else {
#pragma unroll
        for (int v = 0; v < CH / VE; ++v) {
          const float fa[4] = {__uint_as_float(ua[u][v].x), __uint_as_float(ua[u][v].y), __uint_as_float(ua[u][v].z),
                               __uint_as_float(ua[u][v].w)};
          const float fb[4] = {__uint_as_float(ub[u][v].x), __uint_as_float(ub[u][v].y), __uint_as_float(ub[u][v].z),
                               __uint_as_float(ub[u][v].w)};
          s0 = fma((double)fa[0], (double)fb[0], s0);
          s1 = fma((double)fa[1], (double)fb[1], s1);
          s0 = fma((double)fa[2], (double)fb[2], s0);
          s1 = fma((double)fa[3], (double)fb[3], s1);
        }
      }
    }
  }
  return warp_sum(s0 + s1);
}

// The selection of one token decided from exact scores, one warp: every expert whose fp32 biased score is at
// least thr (the (k+1)-th fp32 value minus the guard; -inf when k == E) is re-scored as sigmoid(h . w_e) + bias_e
// in fp64 from the router's own inputs, then k rounds of warp arg-max over those (ties -> lower expert) give the
// slots in order and the gates (unbiased fp64 scores renormalised, rounded once to fp32). Lane j < k returns slot j.
template <int PER, typename T>
DLLM_DEV void exact_redecide(const float* __restrict__ srow, const float* __restrict__ bias, int E, int k,
                             const T* __restrict__ hrow, const T* __restrict__ w, int H, float thr, int lane,
                             int& my_id, float& my_gate) {
  __syncwarp();   // the warp's own write-back of the sigmoid scores is visible to every lane
  double d[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int ex = i * 32 + lane;
    d[i] = -INFINITY;
    const bool cand = ex < E && srow[ex] + bias[ex] >= thr;
    unsigned bal = __ballot_sync(0xffffffffu, cand);
    while (bal) {
      const int b = __ffs(bal) - 1;
      bal &= bal - 1;
      const int eb = i * 32 + b;
      const double dot = warp_dot64<2>(hrow, w + (int64_t)eb * H, H, lane);
      if (lane == b) d[i] = 1.0 / (1.0 + exp(-dot)) + (double)bias[eb];
    }
  }
  double gsum = 0.0, mine = 0.0;
  my_id = 0;
  for (int j = 0; j < k; ++j) {
    double bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int ex = i * 32 + lane;
      if (ex < E && (d[i] > bv || (d[i] == bv && ex < be))) { bv = d[i]; be = ex; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (i * 32 + lane == be) d[i] = -INFINITY;
    const double sc = bv - (double)bias[be];
    gsum += sc;
    if (lane == j) { my_id = be; mine = sc; }
  }
  my_gate = (float)(mine / gsum);
}

// Exact dot-product terms of one 16-byte chunk of a row pair, added in fp64: bf16 products are exact in fp32, fp32
// products are formed in fp64.
DLLM_DEV void acc16(const uint4& hv, const uint4& wv, double& s, const __nv_bfloat16*) {
  float fh[8], fw[8];
  bf16x8_to_f32(hv, fh);
  bf16x8_to_f32(wv, fw);
  double a = 0.0, b = 0.0;
#pragma unroll
  for (int u = 0; u < 8; u += 2) {
    a += (double)(fh[u] * fw[u]);
    b += (double)(fh[u + 1] * fw[u + 1]);
  }
  s += a + b;
}
DLLM_DEV void acc16(const uint4& hv, const uint4& wv, double& s, const float*) {
  s = fma((double)__uint_as_float(hv.x), (double)__uint_as_float(wv.x), s);
  s = fma((double)__uint_as_float(hv.y), (double)__uint_as_float(wv.y), s);
  s = fma((double)__uint_as_float(hv.z), (double)__uint_as_float(wv.z), s);
  s = fma((double)__uint_as_float(hv.w), (double)__uint_as_float(wv.w), s);
}

// One lane-strided pass of a weight row against the token row chunks hv (CH 16-byte chunks per lane, block b0):
// loads of the row's chunks into wv.
template <int CH, typename T>
DLLM_DEV void load_row_chunks(const T* __restrict__ row, int H, int b0, int lane, uint4 (&wv)[CH]) {
  constexpr int VE = 16 / sizeof(T);
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    const int c = b0 + (j * 32 + lane) * VE;
    wv[j] = c < H ? *reinterpret_cast<const uint4*>(row + c) : make_uint4(0, 0, 0, 0);
  }
}

// A token's selection decided exactly when there are more than 32 candidates (only with many equal scores):
// kept out of line, it is never on a hot path.
template <typename T>
__device__ __noinline__ void exact_select_many(const float* __restrict__ srow, const float* __restrict__ bias, int E,
                                               int k, const T* __restrict__ hrow, const T* __restrict__ w, int H,
                                               float thr, int lane, int* my_id, float* my_gate) {
  double gsum = 0.0, mine = 0.0;
  double last = INFINITY;
  int last_e = -1;
  *my_id = 0;
  for (int j = 0; j < k; ++j) {
    // the best candidate below (last, last_e) in (score desc, expert asc) order, rescoring every candidate
    double bv = -INFINITY;
    int be = 0x7fffffff;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int ex = e0 + lane;
      unsigned bal = __ballot_sync(0xffffffffu, ex < E && srow[ex] + bias[ex] >= thr);
      while (bal) {
        const int src = __ffs(bal) - 1;
        bal &= bal - 1;
        const int eb = e0 + src;
        const double v = 1.0 / (1.0 + exp(-warp_dot64<2>(hrow, w + (int64_t)eb * H, H, lane))) + (double)bias[eb];
        const bool below = v < last || (v == last && eb > last_e);
        if (below && (v > bv || (v == bv && eb < be))) { bv = v; be = eb; }
      }
    }
    last = bv;
    last_e = be;
    const double sc = bv - (double)bias[be];
    gsum += sc;
    if (lane == j) { *my_id = be; mine = sc; }
  }
  *my_gate = (float)(mine / gsum);
}

// Exact selection of one near-tie token by its own warp. The candidate experts (fp32 biased score at least thr,
// the (k+1)-th value minus the guard) are compacted into lanes and sorted by their fp32 biased score (ties -> lower
// expert). A candidate whose fp32 value is within kRouteGuard of a neighbour in that order is uncertain; only the
// uncertain ones are scored exactly (a warp-wide dot product of the token row, held in registers, with the
// expert's row, the next uncertain expert's row loading while the current one is summed: bf16 products are exact
// in fp32 and are added in fp64). Every fp32 score is within half the guard of its exact value, so a certain
// candidate's fp32 value orders it against every other candidate exactly as the exact values would; the selection
// (k rounds of a warp arg-max on exact values where computed, fp32 values elsewhere) therefore equals the exact
// one, with the gates from the same scores. Returns false (the fp32 decision stands) only when fewer than k
// experts pass the threshold, which takes non-finite scores.
template <typename T>
DLLM_DEV bool warp_exact_select(const float* __restrict__ srow, const float* __restrict__ bias, int E, int k,
                                const T* __restrict__ hrow, const T* __restrict__ w, int H, float thr, int lane,
                                int& my_id, float& my_gate) {
  constexpr int VE = 16 / sizeof(T);   // elements per 16-byte chunk
  constexpr int CH = 8;                // chunks per lane per block of the row
  constexpr int BLK = 32 * VE * CH;    // row elements per block
  int n = 0, ce = 0x7fffffff;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int ex = e0 + lane;
    unsigned bal = __ballot_sync(0xffffffffu, ex < E && srow[ex] + bias[ex] >= thr);
    while (bal) {
      const int src = __ffs(bal) - 1;
      bal &= bal - 1;
      if (lane == n) ce = e0 + src;
      ++n;
    }
  }
  if (n < k) return false;
  if (n > 32) {
    exact_select_many<T>(srow, bias, E, k, hrow, w, H, thr, lane, &my_id, &my_gate);
    return true;
  }
  // sort the candidates by (fp32 biased value desc, expert asc): bitonic network over the warp
  float fv = lane < n ? srow[ce] + bias[ce] : -INFINITY;
  int fe = lane < n ? ce : 0x7fffffff;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, fv, stride);
      const int oe = __shfl_xor_sync(0xffffffffu, fe, stride);
      const bool other_first = ov > fv || (ov == fv && oe < fe);   // the partner precedes this lane's entry
      const bool lower = (lane & stride) == 0;                     // this lane takes the earlier position
      const bool desc = (lane & size) == 0 || size == 32;          // the final merge runs one way
      if ((lower == desc) == other_first) { fv = ov; fe = oe; }
    }
  }
  const float prv = __shfl_up_sync(0xffffffffu, fv, 1), nxt = __shfl_down_sync(0xffffffffu, fv, 1);
  const bool unc = lane < n && ((lane > 0 && prv - fv < kRouteGuard) || (lane + 1 < n && fv - nxt < kRouteGuard));
  const unsigned ubal = __ballot_sync(0xffffffffu, unc);
  double dot = 0.0;   // uncertain lanes: the candidate's exact dot product
  const int nu = __popc(ubal);
  for (int b0 = 0; b0 < H && nu > 0; b0 += BLK) {
    uint4 hv[CH], wa[CH], wb[CH];
    unsigned rest = ubal;
    int cur = __ffs(rest) - 1;
    rest &= rest - 1;
    load_row_chunks<CH>(hrow, H, b0, lane, hv);
    load_row_chunks<CH>(w + (int64_t)__shfl_sync(0xffffffffu, fe, cur) * H, H, b0, lane, wa);
#pragma unroll 1
    while (cur >= 0) {
      const int nx = rest ? __ffs(rest) - 1 : -1;
      if (rest) rest &= rest - 1;
      if (nx >= 0) load_row_chunks<CH>(w + (int64_t)__shfl_sync(0xffffffffu, fe, nx) * H, H, b0, lane, wb);
      double acc = 0.0;
#pragma unroll
      for (int j = 0; j < CH; ++j) acc16(hv[j], wa[j], acc, hrow);
      acc = warp_sum(acc);
      if (lane == cur) dot += acc;
      cur = nx;
      if (cur < 0) break;
      const int nx2 = rest ? __ffs(rest) - 1 : -1;
      if (rest) rest &= rest - 1;
      if (nx2 >= 0) load_row_chunks<CH>(w + (int64_t)__shfl_sync(0xffffffffu, fe, nx2) * H, H, b0, lane, wa);
      double acc1 = 0.0;
#pragma unroll
      for (int j = 0; j < CH; ++j) acc16(hv[j], wb[j], acc1, hrow);
      acc1 = warp_sum(acc1);
      if (lane == cur) dot += acc1;
      cur = nx2;
    }
  }
  // selection keys: exact biased and unbiased scores where computed, fp32 elsewhere
  const int eb = lane < n ? fe : 0;
  const double raw = unc ? 1.0 / (1.0 + exp(-dot)) : (double)srow[eb];
  double v = lane < n ? (unc ? raw + (double)bias[eb] : (double)fv) : -INFINITY;
  const int e = lane < n ? fe : 0x7fffffff;
  double gsum = 0.0, mine = 0.0;
  my_id = 0;
  for (int j = 0; j < k; ++j) {
    double bv = v;
    int be = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    const double sc = __shfl_sync(0xffffffffu, raw, __ffs(__ballot_sync(0xffffffffu, e == be)) - 1);
    if (e == be) v = -INFINITY;
    gsum += sc;
    if (lane == j) { my_id = be; mine = sc; }
  }
  my_gate = (float)(mine / gsum);
  return true;
}

// Cooperative exact re-decision of a CTA's near-tie tokens. The warps first list their flagged tokens; then, in
// rounds of one flagged token per warp, (a) each warp lists its token's candidate experts (those whose fp32 biased
// score is at least the token's threshold, at most 32 of them), (b) all warps of the CTA compute the candidates'
// exact scores together (one warp per (token, expert) pair, so that a round costs about one dot product's latency),
// (c) each warp ranks its token's candidates (lane j holds candidate j) into slots and gates. A token with more than
// 32 candidates (only with many exactly tied scores) is decided by its warp alone (exact_redecide).
constexpr int kMaxFlagged = 256;

template <int NW>
struct RedecideSmem {
  int n_flag;
  int ftok[kMaxFlagged];
  float fthr[kMaxFlagged];
  int cand_n[NW];
  int cand_e[NW][32];
  double cand_v[NW][32];
};

// Called by every thread of the CTA after each warp has appended its flagged tokens to rs (n_flag counted with
// shared-memory atomics, then a barrier). out(t, lane, id, gate) writes lane's slot of token t.
template <int PER, int NW, typename T, typename Out>
DLLM_DEV void cta_redecide(RedecideSmem<NW>& rs, const float* __restrict__ scores, const float* __restrict__ bias,
                           int E, int k, const T* __restrict__ h, const T* __restrict__ w, int H, Out out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nf = min(rs.n_flag, kMaxFlagged);
  for (int r0 = 0; r0 < nf; r0 += NW) {
    const int f = r0 + warp;
    if (f < nf) {   // (a) candidates of this warp's token
      const int t = rs.ftok[f];
      const float thr = rs.fthr[f];
      const float* srow = scores + (int64_t)t * E;
      int n = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int ex = i * 32 + lane;
        const bool cand = ex < E && srow[ex] + bias[ex] >= thr;
        const unsigned bal = __ballot_sync(0xffffffffu, cand);
        const int slot = n + __popc(bal & ((1u << lane) - 1u));
        if (cand && slot < 32) rs.cand_e[warp][slot] = ex;
        n += __popc(bal);
      }
      if (lane == 0) rs.cand_n[warp] = n <= 32 ? n : -1;
    } else if (lane == 0) {
      rs.cand_n[warp] = 0;
    }
    __syncthreads();
    // (b) every (token, candidate) pair of the round, one warp each
    for (int p = warp; p < NW * 32; p += NW) {
      const int ow = p >> 5, j = p & 31;
      if (j >= rs.cand_n[ow]) continue;
      const int t = rs.ftok[r0 + ow], e = rs.cand_e[ow][j];
      const double dot = warp_dot64<NW >= 32 ? 2 : 4>(h + (int64_t)t * H, w + (int64_t)e * H, H, lane);
      if (lane == 0) rs.cand_v[ow][j] = 1.0 / (1.0 + exp(-dot)) + (double)bias[e];
    }
    __syncthreads();
    // (c) slots and gates of this warp's token
    if (f < nf) {
      const int t = rs.ftok[f], n = rs.cand_n[warp];
      int my_id = 0;
      float my_gate = 0.f;
      if (n < 0) {
        exact_redecide<PER>(scores + (int64_t)t * E, bias, E, k, h + (int64_t)t * H, w, H, rs.fthr[f], lane, my_id,
                            my_gate);
      } else {
        double v = lane < n ? rs.cand_v[warp][lane] : -INFINITY;
        const int e = lane < n ? rs.cand_e[warp][lane] : 0x7fffffff;
        double gsum = 0.0, mine = 0.0;
        for (int j = 0; j < k; ++j) {
          double bv = v;
          int be = e;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
          }
          if (e == be) v = -INFINITY;
          const double sc = bv - (double)bias[be];
          gsum += sc;
          if (lane == j) { my_id = be; mine = sc; }
        }
        my_gate = (float)(mine / gsum);
      }
      out(t, lane, my_id, my_gate);
    }
    __syncthreads();
  }
}

// Many tokens: one warp per token, the fp32 selection. A token whose selection is a near-tie (see kRouteGuard) gets
// fix_thr[t] = its candidate threshold, every other token NaN; route_exact_kernel decides those tokens again.
template <int PER>
__global__ void route_topk_kernel(float* __restrict__ scores, const float* __restrict__ bias, int Tk, int E, int k,
                                  int from_logits, int32_t* __restrict__ ids, float* __restrict__ gates,
                                  float* __restrict__ fix_thr, const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= Tk) return;
  int my_id;
  float my_gate, thr;
  const bool near = warp_topk<PER>(scores + (int64_t)warp * E, bias, E, k, from_logits, lane, my_id, my_gate, thr);
  if (lane < k) {
    ids[(int64_t)warp * k + lane] = my_id;
    gates[(int64_t)warp * k + lane] = my_gate;
  }
  if (lane == 0) fix_thr[warp] = near ? thr : __int_as_float(0x7fc00000);
}

// The near-tie tokens flagged by route_topk_kernel, decided again exactly, one warp per token (warp_exact_select):
// a persistent grid whose warp w takes the tokens w, w + W, w + 2W, ... (W warps in all), reading 32 of their flags
// at once, so near-ties that cluster in neighbouring tokens still spread over every warp. Kept apart from the top-k
// kernel, whose register budget it would otherwise set.
template <typename T>
__global__ void __launch_bounds__(256) route_exact_kernel(const float* __restrict__ scores,
                                                         const float* __restrict__ bias, int Tk, int E, int k,
                                                         const T* __restrict__ h, const T* __restrict__ w, int H,
                                                         const float* __restrict__ fix_thr,
                                                         int32_t* __restrict__ ids, float* __restrict__ gates,
                                                         const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int W = gridDim.x * (blockDim.x >> 5);
  for (int base = gw; base < Tk; base += 32 * W) {
    const int t = base + lane * W;
    const float th = t < Tk ? fix_thr[t] : __int_as_float(0x7fc00000);
    unsigned bal = __ballot_sync(0xffffffffu, !isnan(th));
    while (bal) {
      const int j = __ffs(bal) - 1;
      bal &= bal - 1;
      const int tt = base + j * W;
      int my_id = 0;
      float my_gate = 0.f;
      if (warp_exact_select<T>(scores + (int64_t)tt * E, bias, E, k, h + (int64_t)tt * H, w, H,
                               __shfl_sync(0xffffffffu, th, j), lane, my_id, my_gate) && lane < k) {
        ids[(int64_t)tt * k + lane] = my_id;
        gates[(int64_t)tt * k + lane] = my_gate;
      }
    }
  }
}

// Few tokens (Tk <= 32, Tk * k <= 1024, E <= 256): top-k (with the exact re-decision of near-ties) and the stable
// per-expert permutation in one CTA of 1024 threads. Assignment a = t * k + j; chunk c = a / 32 is handled by one
// warp, whose lanes with the same expert find each other with __match_any_sync: an assignment's position is
// offsets[e] + (assignments of e in earlier chunks) + (lanes of e before it in its chunk), which is the order of a,
// as in the general permutation kernel.
template <int PER, typename T>
__global__ void __launch_bounds__(1024) route_small_kernel(float* __restrict__ scores, const float* __restrict__ bias,
                                                           int Tk, int E, int k, int from_logits,
                                                           const T* __restrict__ h, const T* __restrict__ w, int H,
                                                           int32_t* __restrict__ ids, float* __restrict__ gates,
                                                           int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                           const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  extern __shared__ int rs_sm[];
  const int n = Tk * k, W = (n + 31) / 32;
  int* hist = rs_sm;                 // [W][E]: counts per chunk, then their exclusive prefix over chunks
  int* ids_s = hist + W * E;         // [n]
  int* rk_s = ids_s + n;             // [n]: rank among the chunk's lanes with the same expert
  int* off_s = rk_s + n;             // [E]
  __shared__ int wtot[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  __shared__ RedecideSmem<32> rd;
  for (int i = tid; i < W * E; i += blockDim.x) hist[i] = 0;
  if (tid == 0) rd.n_flag = 0;
  __syncthreads();
  for (int t = warp; t < Tk; t += nw) {
    int my_id;
    float my_gate, thr;
    if (warp_topk<PER>(scores + (int64_t)t * E, bias, E, k, from_logits, lane, my_id, my_gate, thr) && lane == 0) {
      const int f = atomicAdd(&rd.n_flag, 1);   // Tk <= 32 <= kMaxFlagged
      rd.ftok[f] = t;
      rd.fthr[f] = thr;
    }
    if (lane < k) {
      ids[(int64_t)t * k + lane] = my_id;
      gates[(int64_t)t * k + lane] = my_gate;
      ids_s[t * k + lane] = my_id;
    }
  }
  __syncthreads();
  cta_redecide<PER, 32>(rd, scores, bias, E, k, h, w, H, [&](int t, int ln, int id, float g) {
    if (ln < k) {
      ids[(int64_t)t * k + ln] = id;
      gates[(int64_t)t * k + ln] = g;
      ids_s[t * k + ln] = id;
    }
  });
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
      const int hh = hist[c * E + ex];
      hist[c * E + ex] = run;
      run += hh;
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

// Stable permutation for many assignments, in three launches over segments of seg_tok consecutive tokens (seg_tok
// * k assignments, a multiple of 256): per-segment expert histograms; one CTA turns them into counts, offsets and every segment's first output position per expert;
// then each segment writes its assignments' positions in order. Positions within an expert follow the assignment
// index a = t * k + j, so an expert's rows stay sorted by token.

// seg_hist[s][e] = assignments of expert e in segment s.
__global__ void __launch_bounds__(256) route_seg_hist_kernel(const int32_t* __restrict__ ids, int Tk, int k,
                                                             int E, int seg_tok, int32_t* __restrict__ seg_hist,
                                                             const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  extern __shared__ int sh_hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sh_hist[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * seg_tok, t1 = min(Tk, t0 + seg_tok);
  const int a0 = t0 * k, a1 = t1 * k;
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
                                                              int32_t* __restrict__ offsets,
                                                              const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
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
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
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

// Mid-size routing (Tk * k <= kPermCtaMax): after route_topk_kernel, one CTA of 1024 threads builds counts, offsets
// and the stable permutation, in place of the segmented three launches. Warp w takes the assignments
// [w per, (w + 1) per) (per a multiple of 32); pass 1 counts them per expert (__match_any_sync groups), the 32
// warps' counts are prefixed per expert on top of the expert's offset, and pass 2 writes position = warp's running
// base + rank among the chunk's lanes with the same expert, so positions within an expert follow the assignment
// index a = t k + j, as in the other permutation kernels.
constexpr int kPermCtaMax = 8192;

// The stable permutation of n assignments by one CTA of NW warps (E <= 32 NW): counts, offsets and each
// assignment's position. Warp w takes the assignments [w per, (w + 1) per) (per a multiple of 32); pass 1 counts
// them per expert (__match_any_sync groups), the warps' counts are prefixed per expert on top of the expert's
// offset, and pass 2 writes position = warp's running base + rank among the chunk's lanes with the same expert.
// wh: NW x E ints of shared memory, wtot: 32 ints.
template <int NW>
DLLM_DEV void cta_permutation(const int32_t* __restrict__ ids, int n, int E, int32_t* __restrict__ counts,
                              int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                              int* wh, int* wtot) {
  // every chunk of this warp's assignments is loaded once, up front (n <= kPermCtaMax): the two passes below then
  // run on registers instead of one dependent trip to L2 per chunk
  constexpr int MAXC = (kPermCtaMax + NW * 32 - 1) / (NW * 32);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < NW * E; i += NW * 32) wh[i] = 0;
  const int per = ((n + NW - 1) / NW + 31) & ~31;
  const int a0 = min(n, warp * per), a1 = min(n, a0 + per);
  int ex[MAXC];
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int a = a0 + c * 32 + lane;
    ex[c] = a < a1 ? __ldcg(ids + a) : -1;   // from L2: other CTAs of the launch may have written them
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    if (a0 + c * 32 >= a1) break;
    const int a = a0 + c * 32 + lane;
    const unsigned grp = __match_any_sync(0xffffffffu, ex[c]);
    if (a < a1 && lane == __ffs(grp) - 1) wh[warp * E + ex[c]] += __popc(grp);
  }
  __syncthreads();
  // per expert (one thread each): prefix over the warps, total count, then the exclusive scan of the totals
  int cnt = 0;
  if (tid < E) {
#pragma unroll 8
    for (int q = 0; q < NW; ++q) {
      const int v = wh[q * E + tid];
      wh[q * E + tid] = cnt;
      cnt += v;
    }
  }
  int inc = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wtot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int x = lane < NW ? wtot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    wtot[lane] = x;   // inclusive over warps
  }
  __syncthreads();
  if (tid < E) {
    const int excl = inc - cnt + (warp > 0 ? wtot[warp - 1] : 0);
    counts[tid] = cnt;
    offsets[tid] = excl;
#pragma unroll 8
    for (int q = 0; q < NW; ++q) wh[q * E + tid] += excl;
  }
  if (tid == 0) offsets[E] = n;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    if (a0 + c * 32 >= a1) break;
    const int a = a0 + c * 32 + lane;
    const unsigned grp = __match_any_sync(0xffffffffu, ex[c]);
    if (a < a1) {
      const int pos = wh[warp * E + ex[c]] + __popc(grp & ((1u << lane) - 1u));
      perm[pos] = a;
      inv[a] = pos;
    }
    __syncwarp();
    if (a < a1 && lane == __ffs(grp) - 1) wh[warp * E + ex[c]] += __popc(grp);
    __syncwarp();
  }
}

// Mid-size routing (Tk * k <= kPermCtaMax) when the fused decode kernel does not apply: after route_topk_kernel
// (and the exact re-decisions), one CTA of 1024 threads builds counts, offsets and the stable permutation, in place
// of the segmented three launches.
__global__ void __launch_bounds__(1024) route_perm_cta_kernel(const int32_t* __restrict__ ids, int Tk, int E, int k,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                              const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  extern __shared__ int wh[];        // [32][E]
  __shared__ int wtot[32];
  cta_permutation<32>(ids, Tk * k, E, counts, offsets, perm, inv, wh, wtot);
}

// Decode-sized routing (E <= 256, Tk * k <= kPermCtaMax) in one launch after the logits: a warp per token takes the
// fp32 top-k (warp_topk) and, for a near-tie, decides it again exactly in place (warp_exact_select); the last CTA to
// finish (a ticket counter, zeroed before the first launch and by that CTA after use) builds the permutation from
// every CTA's ids (the threadfence / ticket pattern makes them visible to it).
template <int PER, typename T>
__global__ void __launch_bounds__(256, 1) route_decode_kernel(float* __restrict__ scores,
                                                              const float* __restrict__ bias, int Tk, int E, int k,
                                                              int from_logits, const T* __restrict__ h,
                                                              const T* __restrict__ w, int H,
                                                              int32_t* __restrict__ ids, float* __restrict__ gates,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                              unsigned* __restrict__ ticket,
                                                              const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  __shared__ int wh[8 * 256];
  __shared__ int wtot[32];
  __shared__ bool last;
  const int lane = threadIdx.x & 31;
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < Tk; t += gridDim.x * 8) {
    int my_id;
    float my_gate, thr;
    float* srow = scores + (int64_t)t * E;
    if (warp_topk<PER>(srow, bias, E, k, from_logits, lane, my_id, my_gate, thr)) {
      __syncwarp();   // this warp's write-back of the sigmoid scores is visible to all its lanes
      int eid = my_id;
      float egate = my_gate;
      if (warp_exact_select<T>(srow, bias, E, k, h + (int64_t)t * H, w, H, thr, lane, eid, egate)) {
        my_id = eid;
        my_gate = egate;
      }
    }
    if (lane < k) {
      ids[(int64_t)t * k + lane] = my_id;
      gates[(int64_t)t * k + lane] = my_gate;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  cta_permutation<8>(ids, Tk * k, E, counts, offsets, perm, inv, wh, wtot);
  if (threadIdx.x == 0) *ticket = 0u;   // ready for the next launch
}

}  // namespace

// Layout of the router scratch: per-segment expert histograms, one fp32 near-tie threshold per token, and the
// ticket counter of route_decode_kernel.
struct RouteScratch {
  int seg_tok, S;
  int32_t* seg_hist;
  float* fix_thr;
  unsigned* ticket;
};

RouteScratch route_scratch(int Tk, int E, int k, void* base) {
  RouteScratch r;
  r.seg_tok = route_segment_tokens(Tk, k);
  r.S = std::max(1, (Tk + r.seg_tok - 1) / r.seg_tok);
  const size_t hist = ((size_t)r.S * E * sizeof(int32_t) + 255) & ~size_t(255);
  const size_t thr = ((size_t)std::max(Tk, 1) * sizeof(float) + 255) & ~size_t(255);
  r.seg_hist = static_cast<int32_t*>(base);
  r.fix_thr = base ? reinterpret_cast<float*>(static_cast<char*>(base) + hist) : nullptr;
  r.ticket = base ? reinterpret_cast<unsigned*>(static_cast<char*>(base) + hist + thr) : nullptr;
  return r;
}

template <int PER, typename T>
int launch_select_per(float* scores, const float* bias, int Tk, int E, int k, int from_logits, const T* h,
                      const T* w, int H, int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                      int32_t* inv, void* scratch, cudaStream_t s, const int32_t* live) {
  if constexpr (PER <= 8) {   // E <= 256: the single-CTA kernel fits its 64 registers per thread
    const int n = Tk * k, W = (n + 31) / 32;
    const size_t smem = ((size_t)W * E + 2 * (size_t)n + E) * sizeof(int);
    if (Tk <= 32 && n <= 1024 && smem <= 96 * 1024) {
      static bool cfg = false;
      if (!cfg) {
        cudaFuncSetAttribute(route_small_kernel<PER, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        cfg = true;
      }
      launch_pdl(route_small_kernel<PER, T>, 1, 1024, smem, s, scores, bias, Tk, E, k, from_logits, h, w, H, ids,
                 gates, counts, offsets, perm, inv, live);
      DLLM_CHECK_LAUNCH("route_small_kernel");
      return DLLM_OK;
    }
  }
  const RouteScratch rs = route_scratch(Tk, E, k, scratch);
  if constexpr (PER <= 8) {
    if (Tk * k <= kPermCtaMax) {   // one launch: top-k, exact re-decisions and (last CTA) the permutation
      launch_pdl(route_decode_kernel<PER, T>, std::min(num_sms(), (Tk + 7) / 8), 256, 0, s, scores, bias, Tk, E, k,
                 from_logits, h, w, H, ids, gates, counts, offsets, perm, inv, rs.ticket, live);
      DLLM_CHECK_LAUNCH("route_decode_kernel");
      return DLLM_OK;
    }
  }
  // one warp per token, 4 per CTA: many tokens spread over all the SMs (one thread per token, tried for thousands
  // of tokens, reads each 1 KB score row with 32 lines in flight per warp instruction and was 2x slower)
  launch_pdl(route_topk_kernel<PER>, (Tk + 3) / 4, 128, 0, s, scores, bias, Tk, E, k, from_logits, ids, gates,
             rs.fix_thr, live);
  DLLM_CHECK_LAUNCH("route_topk_kernel");
  launch_pdl(route_exact_kernel<T>, std::min(num_sms(), (Tk + 7) / 8), 256, 0, s, (const float*)scores, bias, Tk, E,
             k, h, w, H, (const float*)rs.fix_thr, ids, gates, live);
  DLLM_CHECK_LAUNCH("route_exact_kernel");
  const int n = Tk * k, seg = rs.seg_tok * k;
  if (n <= kPermCtaMax) {   // one CTA builds the permutation
    const size_t smem = (size_t)32 * E * sizeof(int);
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_perm_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
      cfg = true;
    }
    launch_pdl(route_perm_cta_kernel, 1, 1024, smem, s, (const int32_t*)ids, Tk, E, k, counts, offsets, perm, inv,
               live);
    DLLM_CHECK_LAUNCH("route_perm_cta_kernel");
    return DLLM_OK;
  }
  launch_pdl(route_seg_hist_kernel, rs.S, 256, (size_t)E * sizeof(int), s, (const int32_t*)ids, Tk, k, E,
             rs.seg_tok, rs.seg_hist, live);
  DLLM_CHECK_LAUNCH("route_seg_hist_kernel");
  launch_pdl(route_seg_scan_kernel, 1, 1024, 0, s, rs.seg_hist, rs.S, E, n, counts, offsets, live);
  DLLM_CHECK_LAUNCH("route_seg_scan_kernel");
  launch_pdl(route_seg_scatter_kernel, rs.S, 256, (size_t)8 * E * sizeof(int), s, (const int32_t*)ids, n, E, seg,
             (const int32_t*)rs.seg_hist, perm, inv, live);
  DLLM_CHECK_LAUNCH("route_seg_scatter_kernel");
  return DLLM_OK;
}

// Selection and permutation from fp32 scores (sigmoid applied here when from_logits), E <= 1024; h and w are the
// router's inputs, read again only for near-tie tokens.
template <typename T>
int launch_select(float* scores, const float* bias, int Tk, int E, int k, int from_logits, const T* h, const T* w,
                  int H, int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                  void* scratch, cudaStream_t s, const int32_t* live) {
#define DLLM_SELECT(P) \
  launch_select_per<P, T>(scores, bias, Tk, E, k, from_logits, h, w, H, ids, gates, counts, offsets, perm, inv, scratch, \
                          s, live)
  if (E <= 32) return DLLM_SELECT(1);
  if (E <= 64) return DLLM_SELECT(2);
  if (E <= 128) return DLLM_SELECT(4);
  if (E <= 256) return DLLM_SELECT(8);
  if (E <= 512) return DLLM_SELECT(16);
  return DLLM_SELECT(32);
#undef DLLM_SELECT
}

int route_segment_tokens(int Tk, int k) {
  // whole tokens per segment, seg_tok * k a multiple of 256 assignments (8 warps x 32), at most 128 segments
  int g = 256, kk = std::max(k, 1);
  while (kk) { const int t = g % kk; g = kk; kk = t; }   // gcd(256, k)
  const int unit = 256 / g;
  const int want = (std::max(Tk, 0) + 127) / 128;
  return std::max(unit, (want + unit - 1) / unit * unit);
}

size_t route_scratch_bytes(int Tk, int E, int k) {
  const RouteScratch r = route_scratch(Tk, E, k, nullptr);
  const size_t hist = ((size_t)r.S * E * sizeof(int32_t) + 255) & ~size_t(255);
  const size_t thr = ((size_t)std::max(Tk, 1) * sizeof(float) + 255) & ~size_t(255);
  return hist + thr + 256;
}

int launch_route(int dtype, const void* h, const void* w_router, const float* bias, int Tk, int H, int E, int k,
                 int32_t* ids, float* gates, float* scores, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* inv, void* seg_scratch, cudaStream_t s, const int32_t* live) {
  if (Tk <= 0) return DLLM_OK;
  // bf16 with a tensor-core friendly shape: router logits through the tcgen05 projection (fp32 out, accumulated
  // in fp32 in the MMA's fixed order); otherwise the SIMT score kernel
  const bool tc_logits = dtype == DLLM_BF16 && E % 128 == 0 && H % 64 == 0;
  if (tc_logits) {
    GemmArgs g;
    g.x = h; g.x_rows = Tk; g.w = w_router; g.w_rows = E; g.K = H; g.M = E; g.host_cnt = Tk; g.max_cnt = Tk;
    g.cnt_bound = Tk; g.dtype = DLLM_BF16; g.live = live;
    g.epi.kind = EPI_STORE; g.epi.out = scores; g.epi.ldo = E; g.epi.out_f32 = 1;
    g.zero_word = route_scratch(Tk, E, k, seg_scratch).ticket;   // route_decode_kernel's ticket
    int st = gemm_bf16_tc(g, s);
    if (st) return st;
    return launch_select(scores, bias, Tk, E, k, 1, (const __nv_bfloat16*)h, (const __nv_bfloat16*)w_router, H, ids,
                         gates, counts, offsets, perm, inv, seg_scratch, s, live);
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
               (const __nv_bfloat16*)w_router, Tk, H, E, scores, live, route_scratch(Tk, E, k, seg_scratch).ticket);
  } else {
    static bool cfg = false;
    if (!cfg) {
      cudaFuncSetAttribute(route_scores_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cfg = true;
    }
    launch_pdl(route_scores_kernel<float>, g1, 256, smem, s, (const float*)h, (const float*)w_router, Tk, H, E, scores,
               live, route_scratch(Tk, E, k, seg_scratch).ticket);
  }
  DLLM_CHECK_LAUNCH("route_scores_kernel");
  if (dtype == DLLM_BF16)
    return launch_select(scores, bias, Tk, E, k, 0, (const __nv_bfloat16*)h, (const __nv_bfloat16*)w_router, H, ids,
                         gates, counts, offsets, perm, inv, seg_scratch, s, live);
  return launch_select(scores, bias, Tk, E, k, 0, (const float*)h, (const float*)w_router, H, ids, gates, counts,
                       offsets, perm, inv, seg_scratch, s, live);
}

}  // namespace dllm
