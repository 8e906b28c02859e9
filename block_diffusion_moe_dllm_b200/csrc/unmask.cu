// Confidence and unmasking: vocabulary-wide max / arg-max / sum-of-exponentials per still-masked position
// (optionally on classifier-free-guided logits), then per block row the choice of the positions to unmask.
// Source: LLaDA2.0-Uni paper review, section "SPRINT — 학습 없는 추론 가속" (c_i = max_v p(v | x_t); accept every
// position with c above tau, at least ceil(m / (T - t)) per step; the standard schedule ceil(m / T)), and the
// HF-mirror README, section "SPRINT 加速技术" (k = ceil(remaining / steps_left); batch acceptance above the
// threshold).
//
// Reduction: one CTA per (row, vocabulary chunk); 256 threads stream the chunk with 16-byte non-allocating
// loads, keep a running (max, lowest arg-max, sum of exp(z - max)) per thread (sum in fp64, exponentials in
// fp32), merge in registers and shared memory and write one partial per CTA. Selection: one warp per block row
// merges its rows' partials, computes c = 1 / sum, counts, ranks and writes tokens, mask and the step outputs.
#include "common.cuh"
#include "kernels.h"
#include "misc.h"

namespace dllm {
namespace {

constexpr int kRegVpt = 16;                      // most 16-byte vectors a thread keeps in registers
constexpr int kRegChunk = kRegVpt * 256 * 8;     // vocabulary entries per CTA of the register path (32768)

// CTAs of the register path resident per SM for a given register depth (launch bound: registers per thread)
constexpr int kPrefVpt = 16;                     // register depth the chunking aims for when rows are many
template <int VPT> constexpr int reg_min_blocks() { return VPT >= 16 ? 3 : VPT >= 12 ? 4 : VPT >= 8 ? 5 : 6; }
constexpr int kMergeSerial = 8;                  // partials per row merged by one lane; more: a warp per row

// (max logit, lowest index attaining it within the scored slice, sum over the chunk of exp(z - max))
using Partial = ConfPartial;

DLLM_DEV void merge(Partial& a, const Partial& b) {
  if (b.s == 0.0) return;
  if (a.s == 0.0) { a = b; return; }
  if (b.m > a.m || (b.m == a.m && b.idx < a.idx)) {
    const double f = (b.m == a.m) ? 1.0 : (double)expf(a.m - b.m);
    a.s = a.s * f + b.s;
    a.m = b.m;
    a.idx = b.idx;
  } else {
    const double f = (b.m == a.m) ? 1.0 : (double)expf(b.m - a.m);
    a.s = a.s + b.s * f;
  }
}

DLLM_DEV float guided(float zc, float zu, float s) {
  // z = zu + s * (zc - zu), each operation rounded to fp32 in this order (no contraction)
  return __fadd_rn(zu, __fmul_rn(s, __fsub_rn(zc, zu)));
}

DLLM_DEV float guided3(float zc, float zi, float zu, float st, float si) {
  // editing guidance: a = zu + si * (zi - zu), z = a + st * (zc - zi), each operation rounded to fp32 in this order
  const float a = __fadd_rn(zu, __fmul_rn(si, __fsub_rn(zi, zu)));
  return __fadd_rn(a, __fmul_rn(st, __fsub_rn(zc, zi)));
}

// The guided value of one vocabulary entry from the rows of its position: CFG 0 the row itself; CFG 1 the pair
// (z1 = unconditional) with scale st; CFG 2 the triple (z1 = image only, z2 = unconditional) with scales st, si.
template <int CFG>
DLLM_DEV float guide(float zc, float z1, float z2, float st, float si) {
  if constexpr (CFG == 1) return guided(zc, z1, st);
  else if constexpr (CFG == 2) return guided3(zc, z1, z2, st, si);
  else return zc;
}

// The hardware base-2 exponential (ex2.approx.ftz: relative error about 2^-22, results below 2^-126 flushed to 0,
// which against a maximum term of 1 is far below fp32 resolution). Sums and scalings of fp32 pairs use the sm_100
// packed instructions (__fadd2_rn / __fmul2_rn: one issue for two lanes' worth).
DLLM_DEV float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Merge of the 32 lanes' partials (empty ones have s == 0): the lanes' maximum M, each sum rescaled by
// 2^((m - M) log2 e), the fp64 sum of those, and the lowest index among the lanes with m == M. Every lane returns
// the result.
DLLM_DEV Partial warp_merge(Partial p) {
  const bool has = p.s != 0.0;
  const float M = warp_max(has ? p.m : -INFINITY);
  double s = !has ? 0.0 : p.m == M ? p.s : p.s * (double)ex2((p.m - M) * 1.4426950408889634f);
  s = warp_sum(s);
  const int idx = __reduce_min_sync(0xffffffffu, (has && p.m == M) ? p.idx : 0x7fffffff);
  return Partial{M, idx, s};
}

// Running update of one thread's partial with 8 consecutive values starting at vocabulary index v.
DLLM_DEV void update8(Partial& p, const float* z, int v) {
  float vm = z[0];
  int vi = 0;
#pragma unroll
  for (int u = 1; u < 8; ++u)
    if (z[u] > vm) { vm = z[u]; vi = u; }
  if (p.s == 0.0 || vm > p.m) {
    p.s = (p.s == 0.0) ? 0.0 : p.s * exp((double)p.m - (double)vm);
    p.m = vm;
    p.idx = v + vi;
  }
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) acc += expf(z[u] - p.m);
  p.s += (double)acc;
}

DLLM_DEV void load8f(const __nv_bfloat16* p, float* f) { bf16x8_to_f32(ld_nc_v4(p), f); }
DLLM_DEV void load8f(const float* p, float* f) {
  uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + 4);
  f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}

// Rows of the guidance: the position's row r among the n_rows of each group, group g at rows [g * n, (g + 1) * n).
template <typename T, int CFG>
__global__ void __launch_bounds__(256) unmask_reduce_kernel(const T* __restrict__ logits,
                                                            const int32_t* __restrict__ n_rows, int max_rows, int V,
                                                            int chunk, float st, float si, Partial* __restrict__ part,
                                                            int n_chunks) {
  pdl_enter();
  const int r = blockIdx.x, c = blockIdx.y;
  const int n = min(*n_rows, max_rows);   // the device count never exceeds the rows the buffers hold
  if (r >= n) return;
  const T* zc = logits + (int64_t)r * V;
  const T* z1 = logits + (int64_t)(r + n) * V;
  const T* z2 = logits + (int64_t)(r + 2 * n) * V;   // read only with CFG 2
  const int v0 = c * chunk, v1 = min(V, v0 + chunk);
  Partial p{-INFINITY, 0x7fffffff, 0.0};
  const int nvec = (v1 - v0) >> 3;
  const bool vec_ok = ((V * (int)sizeof(T)) % 16 == 0) && (v0 % 8 == 0);
  if (vec_ok) {
    int i = threadIdx.x;
    // two vectors in flight per thread per iteration
    for (; i + 256 < nvec; i += 512) {
      float a[8], b[8];
      load8f(zc + v0 + i * 8, a);
      load8f(zc + v0 + (i + 256) * 8, b);
      if constexpr (CFG == 1) {
        float ua[8], ub[8];
        load8f(z1 + v0 + i * 8, ua);
        load8f(z1 + v0 + (i + 256) * 8, ub);
#pragma unroll
        for (int u = 0; u < 8; ++u) { a[u] = guided(a[u], ua[u], st); b[u] = guided(b[u], ub[u], st); }
      } else if constexpr (CFG == 2) {
        float ia[8], ib[8], ua[8], ub[8];
        load8f(z1 + v0 + i * 8, ia);
        load8f(z1 + v0 + (i + 256) * 8, ib);
        load8f(z2 + v0 + i * 8, ua);
        load8f(z2 + v0 + (i + 256) * 8, ub);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          a[u] = guided3(a[u], ia[u], ua[u], st, si);
          b[u] = guided3(b[u], ib[u], ub[u], st, si);
        }
      }
      update8(p, a, v0 + i * 8);
      update8(p, b, v0 + (i + 256) * 8);
    }
    for (; i < nvec; i += 256) {
      float a[8];
      load8f(zc + v0 + i * 8, a);
      if constexpr (CFG == 1) {
        float ua[8];
        load8f(z1 + v0 + i * 8, ua);
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = guided(a[u], ua[u], st);
      } else if constexpr (CFG == 2) {
        float ia[8], ua[8];
        load8f(z1 + v0 + i * 8, ia);
        load8f(z2 + v0 + i * 8, ua);
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = guided3(a[u], ia[u], ua[u], st, si);
      }
      update8(p, a, v0 + i * 8);
    }
  }
  // scalar part: the whole chunk when vector loads are not possible, else the tail
  for (int v = v0 + (vec_ok ? nvec * 8 : 0) + threadIdx.x; v < v1; v += 256) {
    const float z = guide<CFG>(to_f32(zc[v]), CFG ? to_f32(z1[v]) : 0.f, CFG == 2 ? to_f32(z2[v]) : 0.f, st, si);
    Partial q{z, v, 1.0};
    merge(p, q);
  }
  // warp merge then block merge
  p = warp_merge(p);
  __shared__ Partial wp[8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) wp[w] = p;
  __syncthreads();
  if (w == 0) {
    Partial a = lane < 8 ? wp[lane] : Partial{-INFINITY, 0x7fffffff, 0.0};
    a = warp_merge(a);
    if (lane == 0) part[(int64_t)r * n_chunks + c] = a;
  }
}

// ---- the statistics of the other position scores (top-2 margin, entropy)
// A running (m, idx, s) with (m2, t): m2 the second largest value seen (over entries), t = sum exp(z - m) (z - m).
struct ExtPartial {
  float m;
  int idx;
  double s;
  float m2;
  double t;
};

DLLM_DEV ExtPartial ext_empty() { return ExtPartial{-INFINITY, 0x7fffffff, 0.0, -INFINITY, 0.0}; }

// Union of two partials. The maximum M, each side's sums moved to it (t by t' = e^(m - M) (t + (m - M) s)), the
// lowest index at M, and the second largest value of the union.
DLLM_DEV void ext_merge(ExtPartial& a, const ExtPartial& b) {
  if (b.s == 0.0) return;
  if (a.s == 0.0) { a = b; return; }
  const float M = fmaxf(a.m, b.m);
  const double fa = a.m == M ? 1.0 : exp((double)a.m - (double)M);
  const double fb = b.m == M ? 1.0 : exp((double)b.m - (double)M);
  const double ta = fa * (a.t + ((double)a.m - (double)M) * a.s);
  const double tb = fb * (b.t + ((double)b.m - (double)M) * b.s);
  float m2;
  int idx;
  if (a.m > b.m) { m2 = fmaxf(a.m2, b.m); idx = a.idx; }
  else if (b.m > a.m) { m2 = fmaxf(b.m2, a.m); idx = b.idx; }
  else { m2 = a.m; idx = min(a.idx, b.idx); }   // the maximum occurs on both sides
  a = ExtPartial{M, idx, a.s * fa + b.s * fb, m2, ta + tb};
}

DLLM_DEV ExtPartial ext_one(float z, int v) { return ExtPartial{z, v, 1.0, -INFINITY, 0.0}; }

// One more value z (vocabulary index v, visited in increasing v by this thread) into a running partial; the
// per-value exponential in fp32, the sums in fp64.
DLLM_DEV void ext_add(ExtPartial& p, float z, int v) {
  if (p.s == 0.0) { p = ext_one(z, v); return; }
  if (z > p.m) {
    const float d = p.m - z;                      // < 0: the old terms scale by e^d
    const double f = (double)expf(d);
    p.t = f * (p.t + (double)d * p.s);
    p.s = p.s * f + 1.0;
    p.m2 = p.m;
    p.m = z;
    p.idx = v;
  } else {
    const float d = z - p.m;
    const double e = (double)expf(d);
    p.s += e;
    p.t += e * (double)d;
    p.m2 = fmaxf(p.m2, z);
  }
}

DLLM_DEV ExtPartial ext_warp_merge(ExtPartial p) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ExtPartial q;
    q.m = __shfl_xor_sync(0xffffffffu, p.m, o);
    q.idx = __shfl_xor_sync(0xffffffffu, p.idx, o);
    q.s = __shfl_xor_sync(0xffffffffu, p.s, o);
    q.m2 = __shfl_xor_sync(0xffffffffu, p.m2, o);
    q.t = __shfl_xor_sync(0xffffffffu, p.t, o);
    // merge in a fixed order (lower lane first) so that every lane computes the same result
    if ((threadIdx.x & o) == 0) ext_merge(p, q);
    else { ext_merge(q, p); p = q; }
  }
  return p;
}

// CTA per (row, chunk), any storage type, optional guidance: the extended partial of the chunk, stored as the
// ConfPartial (m, idx, s) and its ConfExtra (m2, t).
template <typename T, int CFG>
__global__ void __launch_bounds__(256) unmask_reduce_ext_kernel(const T* __restrict__ logits,
                                                                const int32_t* __restrict__ n_rows, int max_rows,
                                                                int V, int chunk, float st, float si,
                                                                Partial* __restrict__ part,
                                                                ConfExtra* __restrict__ extra, int n_chunks) {
  pdl_enter();
  const int r = blockIdx.x, c = blockIdx.y;
  const int n = min(*n_rows, max_rows);
  if (r >= n) return;
  const T* zc = logits + (int64_t)r * V;
  const T* z1 = logits + (int64_t)(r + n) * V;
  const T* z2 = logits + (int64_t)(r + 2 * n) * V;   // read only with CFG 2
  const int v0 = c * chunk, v1 = min(V, v0 + chunk);
  ExtPartial p = ext_empty();
  for (int v = v0 + threadIdx.x; v < v1; v += 256) {
    const float z = guide<CFG>(to_f32(zc[v]), CFG ? to_f32(z1[v]) : 0.f, CFG == 2 ? to_f32(z2[v]) : 0.f, st, si);
    ext_add(p, z, v);
  }
  p = ext_warp_merge(p);
  __shared__ ExtPartial wp[8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) wp[w] = p;
  __syncthreads();
  if (w == 0) {
    ExtPartial a = lane < 8 ? wp[lane] : ext_empty();
    a = ext_warp_merge(a);
    if (lane == 0) {
      part[(int64_t)r * n_chunks + c] = Partial{a.m, a.idx, a.s};
      extra[(int64_t)r * n_chunks + c] = ConfExtra{a.m2, 0.f, a.t};
    }
  }
}

// bf16 logits without guidance: each thread keeps its VPT 16-byte vectors of a chunk in registers. Pass 1 finds
// the maximum with packed bf16x2 max (and the first vector holding it); pass 2 sums exp(z - max) as
// 2^((z - max) * log2(e)) with the subtraction and the scaling done on fp32 pairs (z - max is exact near the
// maximum), accumulated per thread in fp32 over at most VPT * 8 terms and then in fp64; the lowest arg-max comes
// from the first vector that holds the maximum, fetched again (reload(k)) before pass 2 so that its latency hides
// behind it. Missing vectors hold bf16 -inf.
template <int VPT, typename Reload>
DLLM_DEV Partial chunk_partial(const uint4 (&u)[VPT], int vbase, Reload reload) {
  float m = -INFINITY;
  int best = -1;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[k]);
    const __nv_bfloat162 a = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
    const float vm = fmaxf(__low2float(a), __high2float(a));
    if (vm > m) { m = vm; best = k; }
  }
  Partial p{-INFINITY, 0x7fffffff, 0.0};
  if (best >= 0) {
    const uint4 bv = reload(best);
    const float log2e = 1.4426950408889634f;
    const float2 negm2 = make_float2(-m, -m), l2 = make_float2(log2e, log2e);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 zz = make_float2(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xffff0000u));
        const float2 x = __fmul2_rn(__fadd2_rn(zz, negm2), l2);
        acc = __fadd2_rn(acc, make_float2(ex2(x.x), ex2(x.y)));
      }
    }
    // lowest index attaining m inside the first vector that holds it
    float f[8];
    bf16x8_to_f32(bv, f);
    int e = 7;
#pragma unroll
    for (int q = 7; q >= 0; --q)
      if (f[q] == m) e = q;
    p.m = m;
    p.idx = vbase + (threadIdx.x + best * 256) * 8 + e;
    p.s = (double)acc.x + (double)acc.y;
  }
  return p;
}

// Block merge of the 256 threads' partials (warp, then block: the maximum, every sum rescaled to it, the sum, and
// the lowest index among the partials that attain it); thread 0 stores the result. Reuses wp: the caller orders a
// second use after the first with a barrier.
DLLM_DEV void block_store(Partial p, Partial* wp, Partial* dst) {
  p = warp_merge(p);
  const int lane = threadIdx.x & 31, wv = threadIdx.x >> 5;
  if (lane == 0) wp[wv] = p;
  __syncthreads();
  if (wv == 0) {
    Partial a = lane < 8 ? wp[lane] : Partial{-INFINITY, 0x7fffffff, 0.0};
    a = warp_merge(a);
    if (lane == 0) *dst = a;
  }
}

template <int VPT>
DLLM_DEV void load_chunk_regs(uint4 (&u)[VPT], const __nv_bfloat16* src, int nvec) {
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * 256;
    u[k] = i < nvec ? ld_nc_v4(src + i * 8) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
  }
}

// One CTA per (row, chunk); a row's chunks are adjacent CTAs (contiguous memory). V % 8 == 0.
template <int VPT>
__global__ void __launch_bounds__(256, reg_min_blocks<VPT>()) unmask_reduce_bf16_kernel(const __nv_bfloat16* __restrict__ logits,
                                                                 const int32_t* __restrict__ n_rows, int max_rows, int V,
                                                                 int chunk, Partial* __restrict__ part, int n_chunks) {
  pdl_enter();
  const int r = blockIdx.y, c = blockIdx.x;
  if (r >= min(*n_rows, max_rows)) return;
  const __nv_bfloat16* z = logits + (int64_t)r * V;
  const int v0 = c * chunk, v1 = min(V, v0 + chunk);
  const int nvec = (v1 - v0) >> 3;
  uint4 u[VPT];
  load_chunk_regs<VPT>(u, z + v0, nvec);
  const Partial p = chunk_partial<VPT>(u, v0, [&](int k) { return ld_nc_v4(z + v0 + (threadIdx.x + k * 256) * 8); });
  __shared__ Partial wp[8];
  block_store(p, wp, part + (int64_t)r * n_chunks + c);
}

// Selection, in two phases of one CTA. Phase A, per masked row r (the r-th still-masked position row_pos[r], cond
// half): merge its partials (one thread per row, or a warp per row when there are many partials, as the LM head's
// fused epilogue writes one per CTA), and park c = 1 / sum (fp32) and the candidate at the row's position in the
// conf and sel outputs. Phase B, one warp per logical block row b (lane i = position i): the schedule, the rank of
// each masked position (higher c first, lower position on equal c) and the writes. Positions whose confidences
// are equal in fp32 rank by position.
__global__ void __launch_bounds__(1024) unmask_select_kernel(Partial* part, int n_chunks, const int32_t* __restrict__ row_pos,
                                     const int32_t* __restrict__ n_rows, int max_rows, int B, int L, int t, int T_s, int mode,
                                     float tau, int k_max, int cfg, int vocab_offset, int32_t* tokens, uint8_t* mask,
                                     int32_t* sel, int32_t* nsel, float* conf, int32_t* remaining,
                                     cudaGraphConditionalHandle cond, int set_cond, int score,
                                     const ConfExtra* __restrict__ extra, float* __restrict__ rank,
                                     float* __restrict__ conf_hist, int hist_stride, int hist_off) {
  pdl_enter();
  __shared__ int rem_w[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // this warp's first block row's mask, loaded ahead of phase A
  const bool mk0 = w < B && lane < L && mask[w * L + lane] != 0;
  const int nr = min(*n_rows, max_rows);   // partials exist for at most max_rows rows
  if (extra) {
    // other position scores: a thread per row merges its partials with their extras in chunk order, parks the
    // largest probability (threshold) in conf and the ranking score in rank
    for (int r = threadIdx.x; r < nr; r += blockDim.x) {
      const int pos = row_pos[r];
      ExtPartial a = ext_empty();
      for (int c = 0; c < n_chunks; ++c) {
        const Partial q = part[(int64_t)r * n_chunks + c];
        const ConfExtra x = extra[(int64_t)r * n_chunks + c];
        ext_merge(a, ExtPartial{q.m, q.idx, q.s, x.m2, x.t});
      }
      if (pos >= 0 && pos < B * L) {
        const double p1 = 1.0 / a.s;
        double sc;
        if (score == DLLM_SCORE_TOP_K_MARGIN) sc = (1.0 - exp((double)a.m2 - (double)a.m)) * p1;
        else sc = a.t * p1 - log(a.s);   // neg_entropy: sum p log p = t / s - log s
        conf[pos] = (float)p1;
        rank[pos] = (float)sc;
        sel[pos] = a.idx + vocab_offset;
      }
    }
  } else if (n_chunks > kMergeSerial) {
    for (int r = w; r < nr; r += nw) {
      const Partial* pr = part + (int64_t)r * n_chunks;
      const int pos = row_pos[r];
      Partial a{-INFINITY, 0x7fffffff, 0.0};
      for (int c0 = 0; c0 < n_chunks; c0 += 128) {
        Partial b4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u * 32 + lane;
          b4[u] = c < n_chunks ? pr[c] : Partial{-INFINITY, 0x7fffffff, 0.0};
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) merge(a, b4[u]);
      }
      a = warp_merge(a);
      if (lane == 0 && pos >= 0 && pos < B * L) {
        conf[pos] = (float)(1.0 / a.s);
        sel[pos] = a.idx + vocab_offset;
      }
    }
  } else {
    for (int r = threadIdx.x; r < nr; r += blockDim.x) {
      const Partial* pr = part + (int64_t)r * n_chunks;
      const int pos = row_pos[r];
      Partial a = pr[0];
      // batches of 8 independent loads, merged in chunk order
      for (int q0 = 1; q0 < n_chunks; q0 += 8) {
        Partial b8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (q0 + u < n_chunks) b8[u] = pr[q0 + u];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (q0 + u < n_chunks) merge(a, b8[u]);
      }
      if (pos >= 0 && pos < B * L) {
        conf[pos] = (float)(1.0 / a.s);
        sel[pos] = a.idx + vocab_offset;
      }
    }
  }
  __syncthreads();
  int rem_acc = 0;
  for (int b = w; b < B; b += nw) {
    const int p = b * L + lane;
    const bool valid = lane < L;
    const bool masked = b == w ? mk0 : (valid && mask[p] != 0);
    const unsigned mball = __ballot_sync(0xffffffffu, masked);
    const float c = masked ? conf[p] : 0.f;
    const float rk = masked ? (extra ? rank[p] : c) : 0.f;   // the ranking score (the threshold counts c)
    const int cand = masked ? sel[p] : -1;
    __syncwarp();
    const int m = __popc(mball);
    int kt = 0;
    if (m > 0) {
      const int floor_k = (m + (T_s - t) - 1) / (T_s - t);
      if (mode == DLLM_UNMASK_FIXED) {
        kt = min(m, floor_k);
      } else {
        const int above = __popc(__ballot_sync(0xffffffffu, masked && c > tau));
        kt = min(m, max(floor_k, min(k_max, above)));
      }
    }
    int rnk = 0;
    for (int j = 0; j < 32; ++j) {
      const float rj = __shfl_sync(0xffffffffu, rk, j);
      if (((mball >> j) & 1u) && (rj > rk || (rj == rk && j < lane))) ++rnk;
    }
    const bool chosen = masked && rnk < kt;
    if (valid) {
      sel[b * L + lane] = -1;
      conf[b * L + lane] = c;
    }
    __syncwarp();
    if (chosen) {
      sel[b * L + rnk] = lane;
      tokens[p] = cand;
      mask[p] = 0;
      for (int g = 1; g <= cfg; ++g) {   // the guidance rows of the position take the same token
        tokens[p + g * B * L] = cand;
        mask[p + g * B * L] = 0;
      }
      if (conf_hist) {   // the accepted position's confidence, for the importance of later SPRINT selections
        for (int g = 0; g <= cfg; ++g) conf_hist[(int64_t)(b + g * B) * hist_stride + hist_off + lane] = c;
      }
    }
    if (lane == 0) {
      nsel[b] = kt;
      rem_acc += m - kt;
    }
  }
  if (lane == 0) rem_w[w] = rem_acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s2 = 0;
    for (int i = 0; i < nw; ++i) s2 += rem_w[i];
    *remaining = s2;
    // inside a block graph: the next pass runs only while masked positions are left
    if (set_cond) cudaGraphSetConditional(cond, s2 > 0 ? 1u : 0u);
  }
}

}  // namespace

int unmask_chunks(int max_rows, int V) {
  // enough CTAs to cover the SMs a few times when every row is masked, chunks of at least 2048 entries, and at most
  // kPrefVpt * 2048 entries so that a thread's share of a chunk fits in registers
  int want = (4 * num_sms() + max(max_rows, 1) - 1) / max(max_rows, 1);
  int most = max(1, V / 2048);
  int least = (V + kPrefVpt * 2048 - 1) / (kPrefVpt * 2048);
  return max(1, max(least, min(want, min(most, 64))));
}

size_t unmask_partials_bytes(int max_rows, int n_chunks) {
  return (size_t)max(max_rows, 1) * (size_t)n_chunks * sizeof(Partial);
}

size_t unmask_extras_bytes(int score, int max_rows, int n_chunks, int B, int L) {
  if (score == DLLM_SCORE_LOW_CONFIDENCE) return 0;
  const size_t ex = ((size_t)max(max_rows, 1) * (size_t)n_chunks * sizeof(ConfExtra) + 255) & ~size_t(255);
  return ex + (size_t)B * L * sizeof(float);
}

// The reduction kernels for the guidance mode a.cfg (0 none, 1 two-way, 2 editing).
template <typename T>
void launch_reduce(const T* z, const UnmaskArgs& a, dim3 grid, int chunk, Partial* part, cudaStream_t s) {
  const float st = a.cfg_scale, si = a.cfg_image_scale;
  if (a.cfg == 2) launch_pdl((unmask_reduce_kernel<T, 2>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, a.n_chunks);
  else if (a.cfg == 1) launch_pdl((unmask_reduce_kernel<T, 1>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, a.n_chunks);
  else launch_pdl((unmask_reduce_kernel<T, 0>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, a.n_chunks);
}

template <typename T>
void launch_reduce_ext(const T* z, const UnmaskArgs& a, dim3 grid, int chunk, Partial* part, ConfExtra* extra,
                       cudaStream_t s) {
  const float st = a.cfg_scale, si = a.cfg_image_scale;
  if (a.cfg == 2) launch_pdl((unmask_reduce_ext_kernel<T, 2>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, extra, a.n_chunks);
  else if (a.cfg == 1) launch_pdl((unmask_reduce_ext_kernel<T, 1>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, extra, a.n_chunks);
  else launch_pdl((unmask_reduce_ext_kernel<T, 0>), grid, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, st, si, part, extra, a.n_chunks);
}

int launch_unmask(const UnmaskArgs& a, cudaStream_t s) {
  const int chunk = ((a.V + a.n_chunks - 1) / a.n_chunks + 7) & ~7;
  const bool ext = a.score != DLLM_SCORE_LOW_CONFIDENCE;
  ConfExtra* extra = nullptr;
  float* rank = nullptr;
  if (ext) {
    DLLM_REQUIRE(a.extras != nullptr && !a.partials_ready, DLLM_ERR_INVALID_ARG,
                 "unmask: the position scores need their scratch and the separate reduction");
    extra = static_cast<ConfExtra*>(a.extras);
    const size_t ex = ((size_t)max(a.max_rows, 1) * (size_t)a.n_chunks * sizeof(ConfExtra) + 255) & ~size_t(255);
    rank = reinterpret_cast<float*>(static_cast<char*>(a.extras) + ex);
  }
  if (a.max_rows > 0 && ext) {
    dim3 grid(a.max_rows, a.n_chunks);
    Partial* part = static_cast<Partial*>(a.partials);
    if (a.dtype == DLLM_BF16) launch_reduce_ext(static_cast<const __nv_bfloat16*>(a.logits), a, grid, chunk, part, extra, s);
    else launch_reduce_ext(static_cast<const float*>(a.logits), a, grid, chunk, part, extra, s);
    DLLM_CHECK_LAUNCH("unmask_reduce_ext_kernel");
  } else if (a.max_rows > 0 && !a.partials_ready) {
    dim3 grid(a.max_rows, a.n_chunks);
    Partial* part = static_cast<Partial*>(a.partials);
    if (a.dtype == DLLM_BF16) {
      const __nv_bfloat16* z = static_cast<const __nv_bfloat16*>(a.logits);
      if (a.cfg) launch_reduce(z, a, grid, chunk, part, s);
      else if (a.V % 8 == 0 && chunk <= kRegChunk) {
        // the shallowest register depth that holds a thread's share of the chunk
        const int vpt = (chunk / 8 + 255) / 256;
        const dim3 g2(a.n_chunks, a.max_rows);
        if (vpt <= 4) launch_pdl(unmask_reduce_bf16_kernel<4>, g2, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, part, a.n_chunks);
        else if (vpt <= 8) launch_pdl(unmask_reduce_bf16_kernel<8>, g2, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, part, a.n_chunks);
        else if (vpt <= 12) launch_pdl(unmask_reduce_bf16_kernel<12>, g2, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, part, a.n_chunks);
        else launch_pdl(unmask_reduce_bf16_kernel<16>, g2, 256, 0, s, z, a.n_rows, a.max_rows, a.V, chunk, part, a.n_chunks);
      }
      else launch_reduce(z, a, grid, chunk, part, s);
    } else {
      launch_reduce(static_cast<const float*>(a.logits), a, grid, chunk, part, s);
    }
    DLLM_CHECK_LAUNCH("unmask_reduce_kernel");
  }
  const int threads = (a.n_chunks > kMergeSerial || ext) ? 1024 : 32 * min(32, max(1, a.B));
  launch_pdl(unmask_select_kernel, 1, threads, 0, s, static_cast<Partial*>(a.partials), a.n_chunks, a.row_pos, a.n_rows,
                                             a.max_rows, a.B, a.L, a.t, a.T_s, a.mode, a.tau, a.k_max, a.cfg, a.vocab_offset,
                                             a.tokens, a.mask, a.sel, a.nsel, a.conf, a.remaining, a.cond,
                                             a.set_cond, a.score, (const ConfExtra*)extra, rank, a.conf_hist,
                                             a.conf_hist_stride, a.conf_hist_off);
  DLLM_CHECK_LAUNCH("unmask_select_kernel");
  return DLLM_OK;
}

}  // namespace dllm
