// Memory-bound helper kernels of the denoising step: embedding gather, RMSNorm, masked-row compaction,
// expert-row gather, gate-weighted combine, and the fp32 SIMT projection path (storage type fp32).
#include "common.cuh"
#include "kernels.h"
#include "misc.h"

namespace dllm {

// ------------------------------------------------------------------------------------------------ embedding
// x[t] = embed[mask[t] ? mask_id : tokens[t]]  (block tokens, masked positions read the mask embedding row)
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const uint8_t* __restrict__ mask, int mask_id,
                             const T* __restrict__ table, T* __restrict__ x, int H) {
  pdl_enter();
  const int t = blockIdx.x;
  const int id = (mask && mask[t]) ? mask_id : tokens[t];
  const uint4* src = reinterpret_cast<const uint4*>(table + (int64_t)id * H);
  uint4* dst = reinterpret_cast<uint4*>(x + (int64_t)t * H);
  const int nvec = H * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) dst[i] = src[i];
}

int launch_embed(int dtype, const int32_t* tokens, const uint8_t* mask, int mask_id, const void* table, void* x,
                 int rows, int H, cudaStream_t s) {
  if (rows <= 0) return DLLM_OK;
  if (dtype == DLLM_BF16)
    launch_pdl(embed_kernel<__nv_bfloat16>, rows, 128, 0, s, tokens, mask, mask_id, (const __nv_bfloat16*)table,
                                                     (__nv_bfloat16*)x, H);
  else
    launch_pdl(embed_kernel<float>, rows, 128, 0, s, tokens, mask, mask_id, (const float*)table, (float*)x, H);
  DLLM_CHECK_LAUNCH("embed_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ RMSNorm
// out[r] = x[src(r)] / sqrt(mean(x^2) + eps) * g, fp32 math. src(r) = r, or through a compacted row list:
// row r = g * n + j (n = *n_dev, group g < groups) comes from row_pos[j] + g * group_off.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ x, const T* __restrict__ g,
                                                      T* __restrict__ out, int H, float eps,
                                                      const int32_t* __restrict__ row_pos,
                                                      const int32_t* __restrict__ n_dev, int groups,
                                                      int group_off) {
  pdl_enter();
  int r = blockIdx.x;
  int src = r;
  if (row_pos) {
    const int n = *n_dev;
    if (r >= n * groups) return;
    const int g = r / n;
    src = row_pos[r - g * n] + g * group_off;
  }
  const T* xr = x + (int64_t)src * H;
  T* o = out + (int64_t)r * H;
  constexpr int VE = 16 / sizeof(T);      // elements per 16-byte vector
  constexpr int MAXV = 4;                 // vectors kept in registers per thread
  const int nvec = H / VE;
  __shared__ float red[32];
  float ss = 0.f;
  const bool vec = (H % VE == 0) && nvec <= MAXV * (int)blockDim.x && ((reinterpret_cast<uintptr_t>(xr) |
                   reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(g)) & 15) == 0;
  uint4 keep[MAXV];
  if (vec) {
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
      const int i = threadIdx.x + k * blockDim.x;
      if (i < nvec) {
        keep[k] = reinterpret_cast<const uint4*>(xr)[i];
        const T* e = reinterpret_cast<const T*>(&keep[k]);
#pragma unroll
        for (int u = 0; u < VE; ++u) {
          const float v = to_f32(e[u]);
          ss += v * v;
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
      float v = to_f32(xr[i]);
      ss += v * v;
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv = 1.0f / sqrtf(red[0] / (float)H + eps);
  if (vec) {
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
      const int i = threadIdx.x + k * blockDim.x;
      if (i < nvec) {
        const uint4 gv = reinterpret_cast<const uint4*>(g)[i];
        const T* e = reinterpret_cast<const T*>(&keep[k]);
        const T* ge = reinterpret_cast<const T*>(&gv);
        uint4 res;
        T* re = reinterpret_cast<T*>(&res);
#pragma unroll
        for (int u = 0; u < VE; ++u) re[u] = from_f32<T>(to_f32(e[u]) * inv * to_f32(ge[u]));
        reinterpret_cast<uint4*>(o)[i] = res;
      }
    }
  } else {
    for (int i = threadIdx.x; i < H; i += blockDim.x) o[i] = from_f32<T>(to_f32(xr[i]) * inv * to_f32(g[i]));
  }
}

int launch_rmsnorm(int dtype, const void* x, const void* g, void* out, int rows, int H, float eps,
                   const int32_t* row_pos, const int32_t* n_dev, int groups, int group_off, cudaStream_t s) {
  if (rows <= 0) return DLLM_OK;
  if (dtype == DLLM_BF16)
    launch_pdl(rmsnorm_kernel<__nv_bfloat16>, rows, 256, 0, s, (const __nv_bfloat16*)x, (const __nv_bfloat16*)g,
                                                       (__nv_bfloat16*)out, H, eps, row_pos, n_dev, groups,
                                                       group_off);
  else
    launch_pdl(rmsnorm_kernel<float>, rows, 256, 0, s, (const float*)x, (const float*)g, (float*)out, H, eps, row_pos,
                                               n_dev, groups, group_off);
  DLLM_CHECK_LAUNCH("rmsnorm_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ masked rows
// Ascending list of the still-masked flat positions of the first n_pos positions (the logical rows), their
// count n_out[0] and n_out[1] = n_out[0] * halves (rows the LM head scores).
__global__ void masked_rows_kernel(const uint8_t* __restrict__ mask, int n_pos, int halves, int32_t* row_pos,
                                   int32_t* n_out) {
  pdl_enter();
  __shared__ int warp_tot[32];
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c0 = 0; c0 < n_pos; c0 += blockDim.x) {
    const int p = c0 + threadIdx.x;
    const int f = (p < n_pos && mask[p]) ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[w] = __popc(bal);
    __syncthreads();
    int before = 0, tot = 0;
    for (int i = 0; i < nw; ++i) {
      if (i < w) before += warp_tot[i];
      tot += warp_tot[i];
    }
    if (f) row_pos[base + before + in_warp] = p;
    __syncthreads();
    if (threadIdx.x == 0) base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    n_out[0] = base;
    n_out[1] = base * halves;
    n_out[2] = base > 0;   // live word of the pass: 0 once the block has no masked position left
  }
}

int launch_masked_rows(const uint8_t* mask, int n_pos, int halves, int32_t* row_pos, int32_t* n_out,
                       cudaStream_t s) {
  launch_pdl(masked_rows_kernel, 1, 1024, 0, s, mask, n_pos, halves, row_pos, n_out);
  DLLM_CHECK_LAUNCH("masked_rows_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ expert rows
// Xp[r] = h[perm[r] / k] for r < Tk * k (assignments grouped by expert), Xp[Tk * k + t] = h[t] (shared expert).
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ h, const int32_t* __restrict__ perm, int k, int n_assign,
                                   int shared, T* __restrict__ xp, int H, const int32_t* __restrict__ live,
                                   unsigned* __restrict__ ctr_a, unsigned* __restrict__ ctr_b) {
  pdl_enter();
  // the work counters of the two expert GEMMs that follow (every kernel before this one is done with them)
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (ctr_a) *ctr_a = 0u;
    if (ctr_b) *ctr_b = 0u;
  }
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  const int r = blockIdx.x;
  int src;
  if (r < n_assign) src = perm[r] / k;
  else if (shared) src = r - n_assign;
  else return;
  const uint4* a = reinterpret_cast<const uint4*>(h + (int64_t)src * H);
  uint4* b = reinterpret_cast<uint4*>(xp + (int64_t)r * H);
  const int nvec = H * (int)sizeof(T) / 16;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) b[i] = a[i];
}

int launch_gather_rows(int dtype, const void* h, const int32_t* perm, int k, int Tk, int shared, void* xp, int H,
                       cudaStream_t s, const int32_t* live, unsigned* ctr_a, unsigned* ctr_b) {
  const int rows = Tk * k + (shared ? Tk : 0);
  if (rows <= 0) return DLLM_OK;
  if (dtype == DLLM_BF16)
    launch_pdl(gather_rows_kernel<__nv_bfloat16>, rows, 128, 0, s, (const __nv_bfloat16*)h, perm, k, Tk * k, shared,
               (__nv_bfloat16*)xp, H, live, ctr_a, ctr_b);
  else
    launch_pdl(gather_rows_kernel<float>, rows, 128, 0, s, (const float*)h, perm, k, Tk * k, shared, (float*)xp, H,
               live, ctr_a, ctr_b);
  DLLM_CHECK_LAUNCH("gather_rows_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ combine
// Four consecutive expert-output values as fp32 (rows in the storage type: bf16 rows are 8-byte loads).
__device__ __forceinline__ float4 load_y4(const float* y) { return *reinterpret_cast<const float4*>(y); }
__device__ __forceinline__ float4 load_y4(const __nv_bfloat16* y) {
  const uint2 u = *reinterpret_cast<const uint2*>(y);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// x[t] = x[t] + (y[Tk*k + t] + sum_j gates[t, j] * y[inv[t*k + j]]), summed in fp32 in slot order, rounded once.
template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(T* __restrict__ x, const T* __restrict__ y,
                                                      const float* __restrict__ gates, const int32_t* __restrict__ inv,
                                                      int k, int n_assign, int shared, int H,
                                                      const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing
  // grid (tokens, H / 512): each thread owns 4 consecutive hidden elements
  const int t = blockIdx.x;
  const int h0 = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (h0 >= H) return;
  float4 acc = shared ? load_y4(y + (int64_t)(n_assign + t) * H + h0) : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float gj = gates[t * k + j];
    const float4 v = load_y4(y + (int64_t)inv[t * k + j] * H + h0);
    acc.x += gj * v.x;
    acc.y += gj * v.y;
    acc.z += gj * v.z;
    acc.w += gj * v.w;
  }
  T* xr = x + (int64_t)t * H + h0;
  xr[0] = from_f32<T>(to_f32(xr[0]) + acc.x);
  xr[1] = from_f32<T>(to_f32(xr[1]) + acc.y);
  xr[2] = from_f32<T>(to_f32(xr[2]) + acc.z);
  xr[3] = from_f32<T>(to_f32(xr[3]) + acc.w);
}

int launch_combine(int dtype, void* x, const void* y, const float* gates, const int32_t* inv, int k, int Tk,
                   int shared, int H, cudaStream_t s, const int32_t* live) {
  if (Tk <= 0) return DLLM_OK;
  dim3 grid(Tk, (H / 4 + 127) / 128);
  if (dtype == DLLM_BF16)
    launch_pdl(combine_kernel<__nv_bfloat16>, grid, 128, 0, s, (__nv_bfloat16*)x, (const __nv_bfloat16*)y, gates, inv,
               k, Tk * k, shared, H, live);
  else
    launch_pdl(combine_kernel<float>, grid, 128, 0, s, (float*)x, (const float*)y, gates, inv, k, Tk * k, shared, H,
               live);
  DLLM_CHECK_LAUNCH("combine_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ fused rows
// The step's row-wise stages that end in an RMSNorm are fused with the norm: the kernel that produces a residual
// row keeps it in registers and writes both the row and its normalised copy, saving a launch and a re-read.
// norm: out = v / sqrt(mean(v^2) + eps) * g in fp32 over the row as stored (rounded to T).

// Sum over the CTA (256 threads) of one float per thread; every thread gets the total.
DLLM_DEV float block_sum256(float v, float* red) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += red[i];
  return t;
}

template <typename T>
DLLM_DEV void store_norm_row(const uint4* keep, int nvec, float inv, const T* __restrict__ g, T* __restrict__ o) {
  constexpr int VE = 16 / sizeof(T);
#pragma unroll
  for (int k = 0; k < kRowVecs; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < nvec) {
      const uint4 gv = reinterpret_cast<const uint4*>(g)[i];
      const T* e = reinterpret_cast<const T*>(&keep[k]);
      const T* ge = reinterpret_cast<const T*>(&gv);
      uint4 res;
      T* re = reinterpret_cast<T*>(&res);
#pragma unroll
      for (int u = 0; u < VE; ++u) re[u] = from_f32<T>(to_f32(e[u]) * inv * to_f32(ge[u]));
      reinterpret_cast<uint4*>(o)[i] = res;
    }
  }
}

// CTA t < rows: x[t] = embed[mask[t] ? mask_id : tokens[t]] and h[t] = norm(x[t]) * g. With the masked-row list
// requested, one extra CTA writes it (the ascending still-masked positions of the first n_pos, their count and
// count * halves), as masked_rows_kernel does.
// Entry idx of a block's RoPE table (see RopeTable): the angle and its cosine and sine in fp64, rounded once.
DLLM_DEV void rope_entry(const RopeTable& r, int idx) {
  if (!r.tab || idx >= r.L * 64) return;
  const int i = idx >> 6, m = idx & 63;
  const double a = (double)(r.pos0 + i) * pow((double)r.base, -2.0 * (double)m / 128.0);
  double sn, cs;
  sincos(a, &sn, &cs);
  r.tab[idx] = make_float2((float)cs, (float)sn);
}

__global__ void __launch_bounds__(256) rope_table_kernel(RopeTable r) {
  pdl_enter();
  rope_entry(r, (int)blockIdx.x * 256 + (int)threadIdx.x);
}

template <typename T>
__global__ void __launch_bounds__(256) embed_norm_kernel(const int32_t* __restrict__ tokens,
                                                         const uint8_t* __restrict__ mask, int mask_id,
                                                         const T* __restrict__ table, T* __restrict__ x,
                                                         T* __restrict__ h, const T* __restrict__ g, int rows, int H,
                                                         float eps, const uint8_t* __restrict__ list_mask, int n_pos,
                                                         int halves, int32_t* row_pos, int32_t* n_out,
                                                         RopeTable rope) {
  pdl_enter();
  const int first_rope = rows + (row_pos ? 1 : 0);
  if ((int)blockIdx.x >= first_rope) {   // the block's RoPE table
    rope_entry(rope, ((int)blockIdx.x - first_rope) * 256 + (int)threadIdx.x);
    return;
  }
  __shared__ float red[8];
  if ((int)blockIdx.x == rows) {
    __shared__ int warp_tot[8];
    __shared__ int base;
    if (threadIdx.x == 0) base = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int c0 = 0; c0 < n_pos; c0 += 256) {
      const int p = c0 + threadIdx.x;
      const int f = (p < n_pos && list_mask[p]) ? 1 : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) warp_tot[w] = __popc(bal);
      __syncthreads();
      int before = 0, tot = 0;
      for (int i = 0; i < 8; ++i) {
        if (i < w) before += warp_tot[i];
        tot += warp_tot[i];
      }
      if (f) row_pos[base + before + __popc(bal & ((1u << lane) - 1u))] = p;
      __syncthreads();
      if (threadIdx.x == 0) base += tot;
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      n_out[0] = base;
      n_out[1] = base * halves;
      n_out[2] = base > 0;   // live word of the pass: 0 once the block has no masked position left
    }
    return;
  }
  constexpr int VE = 16 / sizeof(T);
  const int t = blockIdx.x;
  const int id = (mask && mask[t]) ? mask_id : tokens[t];
  const uint4* src = reinterpret_cast<const uint4*>(table + (int64_t)id * H);
  uint4* dst = reinterpret_cast<uint4*>(x + (int64_t)t * H);
  const int nvec = H / VE;
  uint4 keep[kRowVecs];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kRowVecs; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < nvec) {
      keep[k] = src[i];
      dst[i] = keep[k];
      const T* e = reinterpret_cast<const T*>(&keep[k]);
#pragma unroll
      for (int u = 0; u < VE; ++u) {
        const float v = to_f32(e[u]);
        ss += v * v;
      }
    }
  }
  ss = block_sum256(ss, red);
  store_norm_row<T>(keep, nvec, 1.0f / sqrtf(ss / (float)H + eps), g, h + (int64_t)t * H);
}

int launch_rope_table(const RopeTable& r, cudaStream_t s) {
  if (!r.tab || r.L <= 0) return DLLM_OK;
  launch_pdl(rope_table_kernel, (r.L * 64 + 255) / 256, 256, 0, s, r);
  DLLM_CHECK_LAUNCH("rope_table_kernel");
  return DLLM_OK;
}

int launch_embed_norm(int dtype, const int32_t* tokens, const uint8_t* mask, int mask_id, const void* table, void* x,
                      void* h, const void* g, int rows, int H, float eps, const uint8_t* list_mask, int n_pos,
                      int halves, int32_t* row_pos, int32_t* n_out, cudaStream_t s, const RopeTable& rope) {
  if (rows <= 0) return launch_rope_table(rope, s);
  const int ctas = rows + (row_pos ? 1 : 0) + (rope.tab ? (rope.L * 64 + 255) / 256 : 0);
  if (dtype == DLLM_BF16)
    launch_pdl(embed_norm_kernel<__nv_bfloat16>, ctas, 256, 0, s, tokens, mask, mask_id,
               (const __nv_bfloat16*)table, (__nv_bfloat16*)x, (__nv_bfloat16*)h, (const __nv_bfloat16*)g, rows, H,
               eps, list_mask, n_pos, halves, row_pos, n_out, rope);
  else
    launch_pdl(embed_norm_kernel<float>, ctas, 256, 0, s, tokens, mask, mask_id, (const float*)table, (float*)x,
               (float*)h, (const float*)g, rows, H, eps, list_mask, n_pos, halves, row_pos, n_out, rope);
  DLLM_CHECK_LAUNCH("embed_norm_kernel");
  return DLLM_OK;
}

// CTA t: x[t] += y[Tk*k + t] + sum_j gates[t, j] * y[inv[t*k + j]] (fp32, slot order, rounded once), then the
// norm of the new row: mode NORM_NEXT writes out[t] (the next layer's attention input); mode NORM_FINAL writes the
// final-norm row of a still-masked position only, at its place in the LM head's row list (rank among the masked
// positions of its half, plus n for the unconditional half), which is the order masked_rows_kernel produces.
template <typename T>
__global__ void __launch_bounds__(256) combine_norm_kernel(T* __restrict__ x, const T* __restrict__ y,
                                                           const float* __restrict__ gates,
                                                           const int32_t* __restrict__ inv, int k, int n_assign,
                                                           int shared, int H, const T* __restrict__ g, float eps,
                                                           T* __restrict__ out, int mode,
                                                           const uint8_t* __restrict__ mask, int n_half_pos,
                                                           const int32_t* __restrict__ n_dev,
                                                           const int32_t* __restrict__ live) {
  pdl_enter();
  if (live && *live == 0) return;   // a pass with no masked position left does nothing (the whole CTA leaves)
  __shared__ float red[8];
  constexpr int VE = 16 / sizeof(T);
  const int t = blockIdx.x;
  const int nvec = H / VE;
  T* xr = x + (int64_t)t * H;
  uint4 keep[kRowVecs];
  float ss = 0.f;
#pragma unroll
  for (int kk = 0; kk < kRowVecs; ++kk) {
    const int i = threadIdx.x + kk * 256;
    if (i < nvec) {
      const int h0 = i * VE;
      float acc[VE];
#pragma unroll
      for (int u = 0; u < VE; u += 4) {
        const float4 v = shared ? load_y4(y + (int64_t)(n_assign + t) * H + h0 + u) : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[u] = v.x; acc[u + 1] = v.y; acc[u + 2] = v.z; acc[u + 3] = v.w;
      }
      for (int j = 0; j < k; ++j) {
        const float gj = gates[t * k + j];
        const T* yr = y + (int64_t)inv[t * k + j] * H + h0;
#pragma unroll
        for (int u = 0; u < VE; u += 4) {
          const float4 v = load_y4(yr + u);
          acc[u] += gj * v.x; acc[u + 1] += gj * v.y; acc[u + 2] += gj * v.z; acc[u + 3] += gj * v.w;
        }
      }
      uint4 xv = reinterpret_cast<const uint4*>(xr)[i];
      T* e = reinterpret_cast<T*>(&xv);
#pragma unroll
      for (int u = 0; u < VE; ++u) {
        e[u] = from_f32<T>(to_f32(e[u]) + acc[u]);
        const float v = to_f32(e[u]);
        ss += v * v;
      }
      reinterpret_cast<uint4*>(xr)[i] = xv;
      keep[kk] = xv;
    }
  }
  int row = t;
  if (mode == NORM_FINAL) {
    // rank of this position among the masked positions of its half (counted by the whole CTA)
    const int half = t / n_half_pos, tp = t - half * n_half_pos;
    int c = 0;
    for (int p = threadIdx.x; p < tp; p += 256) c += mask[p] ? 1 : 0;
    const float tot = block_sum256((float)c, red);
    if (!mask[tp]) {
      ss = block_sum256(ss, red);   // every thread takes part in the reductions, then none of them writes
      return;
    }
    row = (int)tot + half * n_dev[0];
  }
  ss = block_sum256(ss, red);
  store_norm_row<T>(keep, nvec, 1.0f / sqrtf(ss / (float)H + eps), g, out + (int64_t)row * H);
}

int launch_combine_norm(int dtype, void* x, const void* y, const float* gates, const int32_t* inv, int k, int Tk,
                        int shared, int H, const void* g, float eps, void* out, int mode, const uint8_t* mask,
                        int n_half_pos, const int32_t* n_dev, cudaStream_t s, const int32_t* live) {
  if (Tk <= 0) return DLLM_OK;
  if (dtype == DLLM_BF16)
    launch_pdl(combine_norm_kernel<__nv_bfloat16>, Tk, 256, 0, s, (__nv_bfloat16*)x, (const __nv_bfloat16*)y, gates,
               inv, k, Tk * k, shared,
               H, (const __nv_bfloat16*)g, eps, (__nv_bfloat16*)out, mode, mask, n_half_pos, n_dev, live);
  else
    launch_pdl(combine_norm_kernel<float>, Tk, 256, 0, s, (float*)x, (const float*)y, gates, inv, k, Tk * k, shared, H,
               (const float*)g, eps, (float*)out, mode, mask, n_half_pos, n_dev, live);
  DLLM_CHECK_LAUNCH("combine_norm_kernel");
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ fp32 path
// SIMT GEMM over groups: raw[row, f] = sum_k X[row, k] W[g * wstride + f, k], f < Mw, fp32 throughout.
// Tiles of 32 rows x 64 features, 256 threads, 2 x 4 outputs per thread.
struct SimtGroups {
  int n_dev, has_extra, extra_off, extra_cnt, host_cnt;
  const int32_t* grp_off;
  const int32_t* grp_cnt;
  const int32_t* cnt_dev;
  const int32_t* live;   // nullable: *live == 0 empties every group
};

__device__ __forceinline__ void group_of(const SimtGroups& G, int g, int& off, int& cnt) {
  if (G.live && *G.live == 0) {
    off = 0;
    cnt = 0;
  } else if (g < G.n_dev) {
    off = G.grp_off[g];
    cnt = G.grp_cnt[g];
  } else if (G.has_extra) {
    off = G.extra_off;
    cnt = G.extra_cnt;
  } else {
    off = 0;
    cnt = G.cnt_dev ? min(*G.cnt_dev, G.host_cnt) : G.host_cnt;
  }
}

__global__ void simt_gemm_f32_kernel(const float* __restrict__ X, const float* __restrict__ W,
                                     const float* __restrict__ W2, int K, int Mw, int64_t wstride, SimtGroups G,
                                     float* __restrict__ raw) {
  pdl_enter();
  const int g = blockIdx.z;
  int off, cnt;
  group_of(G, g, off, cnt);
  const int n0 = blockIdx.x * 32, f0 = blockIdx.y * 64;
  if (n0 >= cnt) return;
  const bool extra = G.has_extra && g == G.n_dev;
  const float* Wg = extra ? W2 : W + (int64_t)g * wstride * K;
  __shared__ float xs[32][33];
  __shared__ float ws[64][33];
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[2][4] = {};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = threadIdx.x; i < 32 * 32; i += 256) {
      int r = i >> 5, c = i & 31;
      xs[r][c] = (n0 + r < cnt && k0 + c < K) ? X[(int64_t)(off + n0 + r) * K + k0 + c] : 0.f;
    }
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      int r = i >> 5, c = i & 31;
      ws[r][c] = (f0 + r < Mw && k0 + c < K) ? Wg[(int64_t)(f0 + r) * K + k0 + c] : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < 32; ++c) {
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] += xs[ty * 2 + a][c] * ws[tx * 4 + b][c];
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int r = n0 + ty * 2 + a, f = f0 + tx * 4 + b;
      if (r < cnt && f < Mw) raw[(int64_t)(off + r) * Mw + f] = acc[a][b];
    }
}

// Epilogue of the fp32 SIMT path from raw fp32 products, over every valid row of every group (nsplit partials
// split_stride elements apart are summed first). T is the storage type.
template <typename T>
__global__ void raw_epilogue_kernel(const float* __restrict__ raw, int nsplit, int64_t split_stride, int Mw, int M,
                                    SimtGroups G, EpiParams e) {
  pdl_enter();
  const int g = blockIdx.y;
  int off, cnt;
  group_of(G, g, off, cnt);
  const int n = blockIdx.x;
  if (n >= cnt) return;
  const int row = off + n;
  const float* rr = raw + (int64_t)row * Mw;
  auto val = [&](int f) {
    float v = rr[f];
    for (int s = 1; s < nsplit; ++s) v += rr[s * split_stride + f];
    return v;
  };
  if (e.kind == EPI_SWIGLU) {
    T* out = static_cast<T*>(e.out);
    for (int i = threadIdx.x; i < M; i += blockDim.x) {
      float gt = val(i), up = val(M + i);
      out[(int64_t)row * e.ldo + i] = from_f32<T>(gt / (1.0f + expf(-gt)) * up);
    }
  } else if (e.kind == EPI_QKV) {
    const int d = e.d, half = d / 2, nh = e.Hq + 2 * e.Hkv;
    const int b = row / e.L, i = row % e.L, pos = e.pos0 + i;
    for (int idx = threadIdx.x; idx < nh * half; idx += blockDim.x) {
      const int hh = idx / half, m = idx % half;
      float x1 = val(hh * d + m), x2 = val(hh * d + m + half);
      float y1 = x1, y2 = x2;
      if (hh < e.Hq + e.Hkv) {
        double sn, cs;
        sincos((double)pos * pow((double)e.rope_base, -2.0 * (double)m / (double)d), &sn, &cs);
        float c = (float)cs, s = (float)sn;
        y1 = x1 * c - x2 * s;
        y2 = x2 * c + x1 * s;
      }
      const T t1 = from_f32<T>(y1), t2 = from_f32<T>(y2);
      T* dst;
      if (hh < e.Hq) {
        dst = static_cast<T*>(e.q_out) + ((int64_t)row * e.Hq + hh) * d;
      } else {
        const bool is_k = hh < e.Hq + e.Hkv;
        const int gk = is_k ? hh - e.Hq : hh - e.Hq - e.Hkv;
        dst = static_cast<T*>(is_k ? e.k_dst : e.v_dst) + (((int64_t)b * e.Hkv + gk) * e.cap + e.slot0 + i) * d;
        void* d2v = is_k ? e.k_dst2 : e.v_dst2;
        if (d2v) {
          T* d2 = static_cast<T*>(d2v) + (((int64_t)b * e.Hkv + gk) * e.cap2 + e.slot2 + i) * d;
          d2[m] = t1;
          d2[m + half] = t2;
        }
      }
      dst[m] = t1;
      dst[m + half] = t2;
    }
  } else if (e.out_f32) {
    float* out = static_cast<float*>(e.out);
    for (int f = threadIdx.x; f < M; f += blockDim.x) {
      int64_t o = (int64_t)row * e.ldo + f;
      out[o] = (e.kind == EPI_RESID) ? out[o] + val(f) : val(f);
    }
  } else {
    T* out = static_cast<T*>(e.out);
    for (int f = threadIdx.x; f < M; f += blockDim.x) {
      int64_t o = (int64_t)row * e.ldo + f;
      out[o] = from_f32<T>((e.kind == EPI_RESID) ? to_f32(out[o]) + val(f) : val(f));
    }
  }
}

size_t gemm_f32_scratch_bytes(int64_t x_rows, int M, int swiglu) {
  return (size_t)x_rows * (size_t)(swiglu ? 2 * M : M) * sizeof(float);
}

int gemm_f32_simt(const GemmArgs& a, cudaStream_t s) {
  DLLM_REQUIRE(a.f32_scratch != nullptr, DLLM_ERR_WORKSPACE, "fp32 projection needs scratch");
  SimtGroups G{a.n_dev, a.has_extra, a.extra_off, a.extra_cnt, a.host_cnt, a.grp_off, a.grp_cnt, a.cnt_dev, a.live};
  const int n_groups = a.n_dev + a.has_extra + ((a.n_dev + a.has_extra) == 0 ? 1 : 0);
  const int Mw = a.swiglu ? 2 * a.M : a.M;
  const int max_cnt = a.cnt_bound > 0 ? a.cnt_bound : 1;
  dim3 grid((max_cnt + 31) / 32, (Mw + 63) / 64, n_groups);
  launch_pdl(simt_gemm_f32_kernel, grid, 256, 0, s, (const float*)a.x, (const float*)a.w, (const float*)a.w2, a.K, Mw,
                                            a.w_group_stride, G, a.f32_scratch);
  DLLM_CHECK_LAUNCH("simt_gemm_f32_kernel");
  dim3 g2(max_cnt, n_groups);
  launch_pdl(raw_epilogue_kernel<float>, g2, 128, 0, s, a.f32_scratch, 1, 0, Mw, a.M, G, a.epi);
  DLLM_CHECK_LAUNCH("raw_epilogue_kernel");
  return DLLM_OK;
}

}  // namespace dllm
