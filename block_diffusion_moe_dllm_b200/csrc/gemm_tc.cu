// Weight-streaming grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
// Y[row, m] = sum_k X[row, k] W[m, k] over groups of X rows (one group per expert, or a single group for the
// dense projections and the LM head). At the decode shapes of the denoising step every weight tile is read
// exactly once and the token count per group is small (1..64), so the kernel is built around streaming W:
//   * swap-AB: the weight tile is the M = 128 operand (A), the group's tokens the N operand (B); the MMA's N
//     is chosen per tile at run time (tokens rounded up to 16), so a group of 3 tokens issues N = 16 MMAs;
//   * persistent CTAs (one per SM) walk a flat tile list (group, m-tile, n-tile) built on the device from the
//     router's counts, so no host synchronisation is needed;
//   * warp specialisation: warp 0 issues TMA loads into a STAGES-deep shared-memory ring, warp 1 issues
//     tcgen05.mma from one thread into a double-buffered TMEM accumulator, warps 2..5 drain TMEM
//     (tcgen05.ld), stage through shared memory and run the fused epilogue (store, residual add, SwiGLU, or
//     RoPE + KV-cache write) with coalesced global stores;
//   * weights are loaded with an L2 evict-first hint (read once), activations with evict-last.
// Every mbarrier wait is bounded; on expiry the kernel records a status word and drains its own copies.
#include "common.cuh"
#include "tc.cuh"
#include "kernels.h"
#include <cuda.h>
#include <cmath>
#include <mutex>
#include <algorithm>

namespace dllm {

namespace {

constexpr int BK = 64;                 // K elements per stage (one 128-byte swizzled row)
constexpr int A_BYTES = 128 * BK * 2;  // 16 KB weight tile per stage
constexpr int XBOX_ROWS = 32;          // X rows per TMA box
constexpr int XBOX_BYTES = XBOX_ROWS * BK * 2;
constexpr int STAGE_COLS = 32;         // epilogue column chunk
constexpr int STAGING_BYTES = 128 * STAGE_COLS * 4;
constexpr int MAX_GROUPS = 1040;
constexpr int NUM_THREADS = 192;
constexpr int NUM_THREADS_SPLIT = 224;   // bf16 weights in a ring of their own: warp 6 loads the activations
constexpr int NUM_THREADS_F8 = 480;    // FP8 weights: two groups of four warps convert alternate E4M3 tiles, one
                                       // more warp loads the activation tiles
constexpr int F8_KS = 2;               // FP8 weights: 64-wide K blocks per stage (one 128-byte row of codes)
constexpr int RAW_BYTES = 128 * BK * F8_KS;   // 16 KB E4M3 weight tile per stage
constexpr int SMEM_LIMIT = 232448;

struct Smem {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t conv[16];                // FP8: A slot's 128 TMEM rows written (128 converter arrivals)
  uint64_t mempty[16];              // FP8: A slot free again (MMA commit)
  uint64_t bfull[8];                // FP8: activation stage landed (TMA)
  uint64_t bempty[8];               // FP8: activation stage read by the MMAs (MMA commit)
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t wq_full[4];              // dynamic schedule: work item published by the producer thread
  uint64_t wq_empty[4];             // dynamic schedule: work item read by every other role
  uint64_t done;
  int wq_item[4];
  uint32_t tmem_base;
  int abort_flag;
  int drained;                      // CTA pairs: the leader saw every issued stage of both CTAs land
  int n_groups;
  int total_tiles;
  int tile_prefix[MAX_GROUPS + 1];  // exclusive prefix of tiles per group
  int grp_off[MAX_GROUPS];
  int grp_cnt[MAX_GROUPS];
  int chunk_sum[NUM_THREADS_F8];
};

struct KParams {
  int K, M, swiglu, m_tiles;
  int ksplit;              // > 1: the K slices of one tile run as one thread-block cluster (rank = slice); the
                           // slices' accumulators are summed through distributed shared memory in rank order
  int64_t w_group_stride;
  int n_dev, has_extra, extra_off, extra_cnt, host_cnt;
  const int32_t* grp_off;
  const int32_t* grp_cnt;
  const int32_t* cnt_dev;
  const int32_t* live;     // nullable: *live == 0 empties every group (a denoising pass with no masked position)
  unsigned* zero_word;     // nullable: set to 0 by CTA 0 after the dependency wait (the next kernel's ticket)
  unsigned* work_ctr;      // nullable: dynamic schedule (see work_produce); zero when the kernel starts
  const float* w_scale;    // FP8 weights: per weight row of W / W2 (null otherwise)
  const float* w2_scale;
  EpiParams epi;
  int32_t* status;
  int prefetch_w;          // 1: dense with at most BN rows, so a CTA's first tile is m-tile = its first tile index and
                           // its weight stages may be loaded before the kernels ahead of it finish
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status, int code) {
  uint32_t n = 0;
  while (!tc::mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (++n > (1u << 22)) {
      *abort_flag = 1;
      if (status) atomicExch(status, code);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool wait_bar_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                 int32_t* status, int code) {
  uint32_t n = 0;
  while (!tc::mbar_try_wait_cluster(bar, parity)) {
    if (*abort_flag) return false;
    if (++n > (1u << 22)) {
      *abort_flag = 1;
      if (status) atomicExch(status, code);
      return false;
    }
  }
  return true;
}

// Tile t -> (group, m-tile, first row of the n-tile, rows in the n-tile). n-tiles of one weight tile are adjacent.
template <int BN>
__device__ __forceinline__ void decode_tile(const Smem& sm, int m_tiles, int t, int& g, int& mt, int& n0,
                                            int& nval) {
  // t is a tile index (work index / ksplit)
  int lo = 0, hi = sm.n_groups - 1;
  while (lo < hi) {  // last g with tile_prefix[g] <= t
    int mid = (lo + hi + 1) >> 1;
    if (sm.tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  int local = t - sm.tile_prefix[g];
  int ntl = (sm.grp_cnt[g] + BN - 1) / BN;
  mt = local / ntl;
  int nt = local - mt * ntl;
  n0 = nt * BN;
  nval = min(BN, sm.grp_cnt[g] - n0);
}

// Work items. Static schedule: CTA c takes items c, c + step, ... Dynamic schedule (grouped launches given a work
// counter, zeroed by the kernel that gathers their rows): warp 0's producer thread takes the next item from the
// counter when its operand ring has room for it, so a CTA that finished its tiles early takes more, and hands it to
// the other roles through a ring of WQ entries in shared memory (full: published; empty: read by the MMA thread and
// one lane of every other consuming warp). The tiles of one expert launch differ widely in cost: an expert with a
// few rows streams its weight tile from HBM for them, a crowded one re-reads its weight tiles from L2 once per N
// tile. Item -1 ends the loop; -2 means a wait gave up (the abort flag is set).
constexpr int WQ = 4;

__device__ __forceinline__ int work_produce(Smem& sm, const KParams& p, uint32_t q, int begin, int step, int total,
                                            volatile int* abort_flag) {
  if (!p.work_ctr) {
    const int w = begin + (int)q * step;
    return w < total ? w : -1;
  }
  const uint32_t s = q % WQ;
  if (!wait_bar(&sm.wq_empty[s], ((q / WQ) & 1) ^ 1, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) return -2;
  const unsigned u = atomicAdd(p.work_ctr, 1u);
  const int w = u < (unsigned)total ? (int)u : -1;
  sm.wq_item[s] = w;
  tc::mbar_arrive(&sm.wq_full[s]);   // release: the item is visible to the roles that wait on the barrier
  return w;
}

// Consumer side: by one thread (warp_wide false) or by all lanes of a warp together (lane 0 waits, reads, arrives
// for the warp and broadcasts the item).
__device__ __forceinline__ int work_consume(Smem& sm, const KParams& p, uint32_t q, int begin, int step, int total,
                                            volatile int* abort_flag, int code, bool warp_wide) {
  if (!p.work_ctr) {
    const int w = begin + (int)q * step;
    return w < total ? w : -1;
  }
  const uint32_t s = q % WQ;
  int w = -2;
  if (!warp_wide || (threadIdx.x & 31) == 0) {
    if (wait_bar(&sm.wq_full[s], (q / WQ) & 1, abort_flag, p.status, code)) {
      w = *reinterpret_cast<volatile int*>(&sm.wq_item[s]);
      tc::mbar_arrive(&sm.wq_empty[s]);
    }
  }
  if (warp_wide) w = __shfl_sync(0xffffffffu, w, 0);
  return w;
}

// Tile of work item wk (K slice ks of it in cluster split-K mode). The dynamic schedule starts with the extra
// group (the shared expert: every token's row, the longest run of full tiles) so that it does not form the tail.
__device__ __forceinline__ int work_tile(const Smem& sm, const KParams& p, int wk, int& ks) {
  const int t = wk / p.ksplit;
  ks = wk - t * p.ksplit;
  if (p.work_ctr && p.has_extra) {
    const int r = t + sm.tile_prefix[p.n_dev];
    return r >= sm.total_tiles ? r - sm.total_tiles : r;
  }
  return t;
}

// Wait for this thread's outstanding tcgen05.ld; the 32 registers are in-out operands, so no use of them can be
// scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld32(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
// 32 columns of this lane without the wait (valid after tmem_wait_ld32 on the same registers).
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// Barrier over every thread of every CTA of the cluster (release / acquire on shared memory).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Split cluster barrier, usable from divergent code (no .aligned).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// 16-byte load from the same shared-memory offset in the CTA of the cluster with the given rank. Not volatile and
// without a memory clobber, so that a thread's loads from every rank are issued back to back and their round
// trips overlap; the cluster barriers (volatile, memory clobber) keep them inside the window where the data is
// valid.
__device__ __forceinline__ float4 ld_dsmem4(const float* local, uint32_t rank) {
  uint32_t remote;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(tc::smem_u32(local)), "r"(rank));
  float4 v;
  asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(remote));
  return v;
}

// Eight consecutive staging values of token column j from feature m0 (two 16-byte shared-memory loads).
__device__ __forceinline__ void stage8(const float* stage, int j, int m0, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(stage + j * 128 + m0);
  const float4 b = *reinterpret_cast<const float4*>(stage + j * 128 + m0 + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  uint4 r;
  __nv_bfloat162 t;
  t = __floats2bfloat162_rn(v[0], v[1]); r.x = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[2], v[3]); r.y = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[4], v[5]); r.z = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[6], v[7]); r.w = *reinterpret_cast<uint32_t*>(&t);
  return r;
}

// Epilogue of up to STAGE_COLS token columns held in shared memory as stage[j * 128 + m] (m = tile row = output
// feature). Every thread handles 4 or 8 consecutive features of one token, so each output write is one 8- or
// 16-byte store; QKV rows keep their RoPE pair (m, m + 64) in the same thread.
template <int BN>
__device__ void epilogue_chunk(const KParams& p, const float* stage, int g, int mt, int n0, int nval, int c0,
                               int row0, int tid) {
  const EpiParams& e = p.epi;
  const int ncols = min(STAGE_COLS, nval - c0);
  if (e.kind == EPI_SWIGLU) {
    // 64 gate rows then 64 up rows: 16 threads per token (4 features each), 8 tokens per round
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(e.out);
    const int m0 = (tid & 15) * 4;
    for (int j = tid >> 4; j < ncols; j += 8) {
      const float4 gt = *reinterpret_cast<const float4*>(stage + j * 128 + m0);
      const float4 up = *reinterpret_cast<const float4*>(stage + j * 128 + 64 + m0);
      __nv_bfloat162 t0 = __floats2bfloat162_rn(silu_f(gt.x) * up.x, silu_f(gt.y) * up.y);
      __nv_bfloat162 t1 = __floats2bfloat162_rn(silu_f(gt.z) * up.z, silu_f(gt.w) * up.w);
      const int64_t row = row0 + n0 + c0 + j;
      *reinterpret_cast<uint2*>(out + row * e.ldo + mt * 64 + m0) =
          make_uint2(*reinterpret_cast<uint32_t*>(&t0), *reinterpret_cast<uint32_t*>(&t1));
    }
  } else if (e.kind == EPI_QKV) {
    // m-tile = one head of d = 128 rows: q heads, then k heads, then v heads. RoPE pairs (i, i + 64); 16 threads
    // per token (4 pairs each), 8 tokens per round
    const int hh = mt;
    const bool rot = hh < e.Hq + e.Hkv;
    const int m0 = (tid & 15) * 4;
    for (int j = tid >> 4; j < ncols; j += 8) {
      const int tr = row0 + n0 + c0 + j;  // token row = b * L + i
      const float4 a1 = *reinterpret_cast<const float4*>(stage + j * 128 + m0);
      const float4 a2 = *reinterpret_cast<const float4*>(stage + j * 128 + 64 + m0);
      const float x1[4] = {a1.x, a1.y, a1.z, a1.w}, x2[4] = {a2.x, a2.y, a2.z, a2.w};
      float y1[4], y2[4];
      if (rot) {
        // (cos, sin) of pairs m0 .. m0 + 3 at the token's position: two 16-byte loads of the block's table
        const float4* cs = reinterpret_cast<const float4*>(e.rope_tab + (tr % e.L) * 64 + m0);
        const float4 c01 = cs[0], c23 = cs[1];
        const float c[4] = {c01.x, c01.z, c23.x, c23.z}, sn[4] = {c01.y, c01.w, c23.y, c23.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          y1[u] = x1[u] * c[u] - x2[u] * sn[u];
          y2[u] = x2[u] * c[u] + x1[u] * sn[u];
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) { y1[u] = x1[u]; y2[u] = x2[u]; }
      }
      __nv_bfloat162 t0 = __floats2bfloat162_rn(y1[0], y1[1]), t1 = __floats2bfloat162_rn(y1[2], y1[3]);
      __nv_bfloat162 t2 = __floats2bfloat162_rn(y2[0], y2[1]), t3 = __floats2bfloat162_rn(y2[2], y2[3]);
      const uint2 b1 = make_uint2(*reinterpret_cast<uint32_t*>(&t0), *reinterpret_cast<uint32_t*>(&t1));
      const uint2 b2 = make_uint2(*reinterpret_cast<uint32_t*>(&t2), *reinterpret_cast<uint32_t*>(&t3));
      if (hh < e.Hq) {
        __nv_bfloat16* q = static_cast<__nv_bfloat16*>(e.q_out) + ((int64_t)tr * e.Hq + hh) * 128;
        *reinterpret_cast<uint2*>(q + m0) = b1;
        *reinterpret_cast<uint2*>(q + 64 + m0) = b2;
      } else {
        const int b = tr / e.L, i = tr % e.L;
        const bool is_k = hh < e.Hq + e.Hkv;
        const int gk = is_k ? hh - e.Hq : hh - e.Hq - e.Hkv;
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(is_k ? e.k_dst : e.v_dst) +
                             (((int64_t)b * e.Hkv + gk) * e.cap + e.slot0 + i) * 128;
        *reinterpret_cast<uint2*>(dst + m0) = b1;
        *reinterpret_cast<uint2*>(dst + 64 + m0) = b2;
        void* d2v = is_k ? e.k_dst2 : e.v_dst2;
        if (d2v) {
          __nv_bfloat16* d2 = static_cast<__nv_bfloat16*>(d2v) + (((int64_t)b * e.Hkv + gk) * e.cap2 + e.slot2 + i) * 128;
          *reinterpret_cast<uint2*>(d2 + m0) = b1;
          *reinterpret_cast<uint2*>(d2 + 64 + m0) = b2;
        }
      }
    }
  } else {
    // plain store or residual add: 16 threads per token, 8 tokens per round
    const int m0 = (tid & 15) * 8;
    const int64_t col = (int64_t)mt * 128 + m0;
    for (int j = tid >> 4; j < ncols; j += 8) {
      float v[8];
      stage8(stage, j, m0, v);
      const int64_t off = (int64_t)(row0 + n0 + c0 + j) * e.ldo + col;
      if (e.out_f32) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(e.out) + off);
        if (e.kind == EPI_RESID) {
          const float4 r0 = o[0], r1 = o[1];
          v[0] += r0.x; v[1] += r0.y; v[2] += r0.z; v[3] += r0.w;
          v[4] += r1.x; v[5] += r1.y; v[6] += r1.z; v[7] += r1.w;
        }
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
      } else {
        uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(e.out) + off);
        if (e.kind == EPI_RESID) {
          float r[8];
          bf16x8_to_f32(*o, r);
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] += r[u];
        }
        *o = pack_bf16x8(v);
      }
    }
  }
}

// Running confidence partials of the four token rows whose 16-lane group this thread leads (rows (tid >> 4) + 8 i
// of the single 32-row N tile).
struct ConfRun {
  float m[4];
  int idx[4];
  double s[4];
};

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// LM-head epilogue with the confidence reduction fused (single 32-row N tile). Token row j of the tile is handled
// by the 16 threads with tid >> 4 == j % 8 in round j / 8, each owning 8 consecutive vocabulary rows. The logits are
// rounded to bf16 and stored, and the partial is taken over the rounded values, as a reduction reading them back
// would see them: the 8-value maximum with its lowest index and the sum of 2^((z - max) log2 e) in fp32; then the
// 16 lanes combine by the maximum M, each lane's sum rescaled to M and summed, and the lowest index among the lanes
// at M. The group's first lane folds that into its running partial (fp64 sum; on equal maxima the lower index,
// which comes first).
__device__ __forceinline__ void epilogue_logits_conf(const KParams& p, const float* stage, int mt, int nval,
                                                     int row0, int tid, ConfRun& run) {
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.epi.out);
  const int m0 = (tid & 15) * 8;
  const int col = mt * 128 + m0;
  const float log2e = 1.4426950408889634f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = (tid >> 4) + 8 * i;
    const bool act = j < nval;   // uniform over the 16 lanes of the row
    float lm = -INFINITY, ls = 0.f;
    int li = 0x7fffffff;
    if (act) {
      float v[8];
      stage8(stage, j, m0, v);
      const uint4 pk = pack_bf16x8(v);
      *reinterpret_cast<uint4*>(out + (int64_t)(row0 + j) * p.epi.ldo + col) = pk;
      float f[8];
      bf16x8_to_f32(pk, f);
      lm = f[0];
      li = 0;
#pragma unroll
      for (int q = 1; q < 8; ++q)
        if (f[q] > lm) { lm = f[q]; li = q; }
      li += col;
#pragma unroll
      for (int q = 0; q < 8; ++q) ls += ex2_approx((f[q] - lm) * log2e);
    }
    float hm = lm;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
    float sc = act ? ls * ex2_approx((lm - hm) * log2e) : 0.f;
    int ci = (act && lm == hm) ? li : 0x7fffffff;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      sc += __shfl_xor_sync(0xffffffffu, sc, o);
      ci = min(ci, __shfl_xor_sync(0xffffffffu, ci, o));
    }
    if ((tid & 15) == 0 && act) {
      if (run.s[i] == 0.0) {
        run.m[i] = hm; run.idx[i] = ci; run.s[i] = sc;
      } else if (hm > run.m[i]) {
        run.s[i] = run.s[i] * (double)expf(run.m[i] - hm) + (double)sc;
        run.m[i] = hm; run.idx[i] = ci;
      } else if (hm == run.m[i]) {
        run.s[i] += (double)sc;
        run.idx[i] = min(run.idx[i], ci);
      } else {
        run.s[i] += (double)sc * (double)expf(hm - run.m[i]);
      }
    }
  }
}

// Two E4M3 codes (bytes 0 and 1, or 2 and 3, of w, as selected by prmt_sel) as a bf16 pair, exactly. The code
// s.eeee.mmm placed as the bf16 bit pattern s.0000eeee.mmm0000 is value(code) * 2^-120 for every code, the
// subnormal ones included (both formats scale their subnormals by their fixed minimum exponent), so the pair is
// formed with integer operations (a byte permute that also replicates each code's sign bit, a shift and a mask)
// and multiplied by 2^120, exact in bf16 arithmetic (which keeps subnormal inputs). No conversion instruction is
// needed, so the pairs come from the integer and fused multiply-add pipes. NaN codes are not expected in weights.
template <uint32_t PRMT_SEL>
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w) {
  uint32_t q;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(q) : "r"(w), "n"(PRMT_SEL));
  const uint32_t bits = (q << 4) & 0x87f087f0u;
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(bits), "r"(0x7b807b80u));   // x 2^120
  return r;
}

// FP8 weights: row r of one stage's E4M3 tile (128 codes) as 64 columns of bf16 pairs in TMEM lane r, the A
// operand the MMA reads from tensor memory. The TMA box lands row r at byte r * 128 of the stage with 128-byte
// swizzling (its eight 16-byte pieces XOR-permuted by r & 7), so the eight rows a quarter-warp reads hit eight
// different bank groups. The tile holds the codes' values unscaled; the per-row scale is applied to the
// accumulator.
__device__ __forceinline__ void convert_e4m3_row_to_tmem(const uint8_t* raw, int row, uint32_t taddr) {
  const int sw = row & 7;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t o[32];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
      const int piece = half * 4 + pp;
      const uint4 q = *reinterpret_cast<const uint4*>(raw + row * 128 + ((piece ^ sw) << 4));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // selectors: bytes (c0, sign(c0), c1, sign(c1)) and (c2, sign(c2), c3, sign(c3))
        o[pp * 8 + 2 * i] = e4m3x2_to_bf16x2<0x9180u>(w[i]);
        o[pp * 8 + 2 * i + 1] = e4m3x2_to_bf16x2<0xB3A2u>(w[i]);
      }
    }
    tc::tmem_st32(taddr + half * 32, o);
  }
}

// Scale of tile row r of tile (g, mt) for FP8 weights: the row of W (or W2 for the extra group) it came from.
__device__ __forceinline__ float f8_row_scale(const KParams& p, int g, int mt, int r) {
  const bool extra = p.has_extra && g == p.n_dev;
  const float* sc = extra ? p.w2_scale : p.w_scale + (extra ? 0 : (int64_t)g * p.w_group_stride);
  const int wr = p.swiglu ? (r < 64 ? mt * 64 + r : p.M + mt * 64 + r - 64) : mt * 128 + r;
  return sc[wr];
}

template <int BN, int STAGES, bool F8 = false, int BST = 1>
__global__ void __launch_bounds__(F8 ? NUM_THREADS_F8 : (BST > 1 ? NUM_THREADS_SPLIT : NUM_THREADS), 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_w2,
               const __grid_constant__ CUtensorMap tmap_x, const KParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int NT = F8 ? NUM_THREADS_F8 : (BST > 1 ? NUM_THREADS_SPLIT : NUM_THREADS);
  // separate rings of weight tiles and of activation tiles (always for FP8; for bf16 when BST > 1): the weight ring's
  // depth alone then sets the weight bytes in flight, which bounds a CTA's share of HBM bandwidth when its tiles
  // stream weights for a few rows each
  constexpr bool SPLIT = F8 || BST > 1;
  constexpr int XWARP = F8 ? 14 : 6;          // the activation producer's warp in split mode
  // a stage covers KS 64-wide K blocks: one for bf16 weights (a 128-byte row of 64 elements), two for FP8 (a
  // 128-byte row of 128 codes, so that each weight row read from HBM per stage is as long as in bf16)
  constexpr int KS = F8 ? F8_KS : 1;
  constexpr int SBK = BK * KS;                // K elements per stage
  constexpr int B_HALF = BN * BK * 2;         // the activation tile of one 64-wide K block
  constexpr int B_BYTES = B_HALF * KS;
  // bf16 weights: STAGES stages of [A weight tile][B activation tile]. FP8 weights: a ring of STAGES E4M3 weight
  // tiles (the HBM stream, released by the converter warps as soon as they have read a tile, so that its depth alone
  // sets the weight bytes in flight), a ring of BST activation tiles (from L2, released by the MMAs), and MS A
  // operand slots in tensor memory that the converter warps fill from the codes. The slots fill the tensor memory
  // the two accumulators leave free: a slot is busy from its conversion through the MMA's completion.
  constexpr int SLOT_COLS = 32 * KS;           // TMEM columns of one A slot (bf16 pairs of a stage's K)
  constexpr int MS = F8 ? ((512 - 2 * BN) / SLOT_COLS < 16 ? (512 - 2 * BN) / SLOT_COLS : 16) : 0;
  constexpr int MSD = MS > 0 ? MS : 1;        // slot count as a divisor (the bf16 instantiations use no slots)
  constexpr int W_BYTES = F8 ? RAW_BYTES : A_BYTES;
  constexpr int STAGE_BYTES = SPLIT ? W_BYTES : W_BYTES + B_BYTES;
  constexpr uint32_t W_TX = W_BYTES;                                      // weight bytes a stage's TMA brings
  // two accumulators of BN columns; the allocation is a power of two (N tile 96: 256 columns)
  constexpr uint32_t TMEM_COLS = F8 ? 512 : (2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512);
  static_assert(!F8 || 2 * BN + MS * SLOT_COLS <= 512, "FP8 A slots exceed the tensor memory");
  static_assert(BST <= 8, "activation ring");
  uint8_t* stages = base;
  uint8_t* bring = base + STAGES * STAGE_BYTES;                           // split mode: activation ring
  float* staging = reinterpret_cast<float*>(bring + (SPLIT ? BST * B_BYTES : 0));
  Smem& sm = *reinterpret_cast<Smem*>(reinterpret_cast<uint8_t*>(staging) + STAGING_BYTES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  const int n_groups = p.n_dev + p.has_extra + ((p.n_dev + p.has_extra) == 0 ? 1 : 0);
  if (tid == 0) {
    sm.n_groups = n_groups;
    sm.abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1);
      tc::mbar_init(&sm.empty[s], F8 ? 128 : 1);   // FP8: released by the 128 converter threads that read it
    }
    for (int s = 0; s < MS; ++s) {
      tc::mbar_init(&sm.conv[s], 128);   // the slot's 128 TMEM rows written
      tc::mbar_init(&sm.mempty[s], 1);   // the slot read by the MMAs
    }
    if (SPLIT)
      for (int b = 0; b < BST; ++b) {
        tc::mbar_init(&sm.bfull[b], 1);
        tc::mbar_init(&sm.bempty[b], 1);
      }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&sm.tfull[b], 1);
      tc::mbar_init(&sm.tempty[b], 128);
    }
    for (int q = 0; q < WQ; ++q) {
      tc::mbar_init(&sm.wq_full[q], 1);
      // readers of an item: the MMA thread, the four epilogue warps, in split mode the activation producer thread
      // and for FP8 the eight converter warps
      tc::mbar_init(&sm.wq_empty[q], F8 ? 14 : (SPLIT ? 6 : 5));
    }
    tc::mbar_init(&sm.done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&sm.tmem_base, TMEM_COLS);
  __syncthreads();
  // Weights are never written by the kernels ahead of this one: the first tile's first weight stages can stream
  // in before the dependency wait (their transaction bytes are expected now; the arrival, with the activation
  // bytes, comes in the producer loop). Every lane of warp 0 derives the same count. Dense launches whose row count
  // is fixed on the host know their first tile's weight tile here (tile t0 -> m-tile t0 / N tiles per weight tile);
  // measured on a 20-layer understanding block (the 512-row QKV, output and router-logit projections): 141.2 ->
  // 140.4 ms.
  const int kblocks = p.K / SBK;
  int npf = 0;
  if (p.prefetch_w) {
    const int t0 = p.ksplit > 1 ? (int)blockIdx.y : (int)blockIdx.x;
    const int ks0 = p.ksplit > 1 ? (int)blockIdx.x : 0;
    const int kb0 = ks0 * kblocks / p.ksplit, kb1 = (ks0 + 1) * kblocks / p.ksplit;
    const int ntl = max(1, (p.host_cnt + BN - 1) / BN);   // N tiles per weight tile (row count fixed on the host)
    if (t0 < p.m_tiles * ntl) npf = min(STAGES, kb1 - kb0);
    if (warp == 0 && npf > 0 && tc::elect_one()) {
      tc::prefetch_tmap(&tmap_w);
      const uint64_t pol_w = tc::policy_evict_first();
      for (int i = 0; i < npf; ++i) {
        tc::mbar_expect_tx(&sm.full[i], W_TX);
        tc::tma_load_2d(stages + i * STAGE_BYTES, &tmap_w, (kb0 + i) * SBK, (t0 / ntl) * 128, &sm.full[i], pol_w);
      }
    }
  }
  // everything above reads only the weights and on-chip state; the group counts below come from the kernels
  // before this one
  pdl_enter();
  if (p.zero_word && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.zero_word = 0u;
  // ---- group table: counts, offsets and the exclusive prefix of tiles per group
  const bool dead = p.live && *p.live == 0;
  for (int g = tid; g < n_groups; g += NT) {
    int off, cnt;
    if (g < p.n_dev) {
      off = p.grp_off[g];
      cnt = p.grp_cnt[g];
    } else if (p.has_extra) {
      off = p.extra_off;
      cnt = p.extra_cnt;
    } else {
      off = 0;
      cnt = p.cnt_dev ? min(*p.cnt_dev, p.host_cnt) : p.host_cnt;
    }
    sm.grp_off[g] = off;
    sm.grp_cnt[g] = dead ? 0 : max(cnt, 0);
  }
  __syncthreads();
  // prefix of tiles per group: contiguous chunks per thread, a shuffle scan of the thread sums inside each warp,
  // then the warp totals
  {
    int* warp_tot = sm.chunk_sum;
    const int per = (n_groups + NT - 1) / NT;
    const int g0 = tid * per, g1 = min(n_groups, g0 + per);
    int s = 0;
    for (int g = g0; g < g1; ++g) s += ((sm.grp_cnt[g] + BN - 1) / BN) * p.m_tiles;
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w2 = 0; w2 < NT / 32; ++w2) {
      const int v = warp_tot[w2];
      if (w2 < warp) before += v;
      all += v;
    }
    int run = before + inc - s;
    for (int g = g0; g < g1; ++g) {
      sm.tile_prefix[g] = run;
      run += ((sm.grp_cnt[g] + BN - 1) / BN) * p.m_tiles;
    }
    if (tid == 0) sm.total_tiles = all;
    __syncthreads();
  }
  const int total = sm.total_tiles * p.ksplit;
  // persistent CTAs stride over the work list; in cluster split-K mode CTA (rank, tile) owns exactly one item
  const int wk_begin = p.ksplit > 1 ? (int)(blockIdx.y * p.ksplit + blockIdx.x) : (int)blockIdx.x;
  const int wk_step = p.ksplit > 1 ? total : (int)gridDim.x;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tmap_w);
      tc::prefetch_tmap(&tmap_x);
      if (p.has_extra) tc::prefetch_tmap(&tmap_w2);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_x = tc::policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t q = 0; ok; ++q) {
        const int wk = work_produce(sm, p, q, wk_begin, wk_step, total, abort_flag);
        if (wk < 0) {
          ok = wk == -1;
          break;
        }
        int ks;
        const int t = work_tile(sm, p, wk, ks);
        const int kb0 = ks * kblocks / p.ksplit, kb1 = (ks + 1) * kblocks / p.ksplit;
        int g, mt, n0, nval;
        decode_tile<BN>(sm, p.m_tiles, t, g, mt, n0, nval);
        const bool extra = p.has_extra && g == p.n_dev;
        const CUtensorMap* wm = extra ? &tmap_w2 : &tmap_w;
        const int64_t wrow = extra ? 0 : (int64_t)g * p.w_group_stride;
        const int nb = (nval + XBOX_ROWS - 1) / XBOX_ROWS;
        const uint32_t bytes = W_TX + KS * nb * XBOX_BYTES;
        const int xrow = sm.grp_off[g] + n0;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait_bar(&sm.empty[s], ph ^ 1, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) { ok = false; break; }
          uint8_t* a = stages + s * STAGE_BYTES;
          uint8_t* b = a + W_BYTES;
          if (it < (uint32_t)npf) {   // weight stage already in flight: arrive with the activation bytes
            if (SPLIT) tc::mbar_arrive(&sm.full[s]);
            else tc::mbar_arrive_expect_tx(&sm.full[s], bytes - W_TX);
          } else {
            tc::mbar_arrive_expect_tx(&sm.full[s], SPLIT ? W_TX : bytes);
            if (p.swiglu) {
              tc::tma_load_2d(a, wm, kb * SBK, (int)(wrow + mt * 64), &sm.full[s], pol_w);
              tc::tma_load_2d(a + W_TX / 2, wm, kb * SBK, (int)(wrow + p.M + mt * 64), &sm.full[s], pol_w);
            } else {
              tc::tma_load_2d(a, wm, kb * SBK, (int)(wrow + mt * 128), &sm.full[s], pol_w);
            }
          }
          if constexpr (!SPLIT)
            for (int j = 0; j < nb; ++j)
              tc::tma_load_2d(b + j * XBOX_BYTES, &tmap_x, kb * SBK, xrow + j * XBOX_ROWS, &sm.full[s], pol_x);
        }
      }
      if (!ok) {
        // drain: wait (bounded) for the copies of the last issued stages to land before leaving
        uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t i = first; i < it; ++i) tc::mbar_wait(&sm.full[i % STAGES], (i / STAGES) & 1, 1u << 16);
      }
      // prefetched weight stages no work item consumed (no rows after all): complete their phase and let the
      // copies land before the CTA leaves
      for (uint32_t i = it; i < (uint32_t)npf; ++i) {
        tc::mbar_arrive(&sm.full[i]);
        tc::mbar_wait(&sm.full[i], 0, 1u << 16);
      }
    }
  } else if (SPLIT && warp == XWARP) {
    // ------------------------------------------------------------------ split mode: activation producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tmap_x);
      const uint64_t pol_x = tc::policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t q = 0; ok; ++q) {
        const int wk = work_consume(sm, p, q, wk_begin, wk_step, total, abort_flag, ST_TIMEOUT_PRODUCER, false);
        if (wk < 0) {
          ok = wk == -1;
          break;
        }
        int ks;
        const int t = work_tile(sm, p, wk, ks);
        const int kb0 = ks * kblocks / p.ksplit, kb1 = (ks + 1) * kblocks / p.ksplit;
        int g, mt, n0, nval;
        decode_tile<BN>(sm, p.m_tiles, t, g, mt, n0, nval);
        const int nb = (nval + XBOX_ROWS - 1) / XBOX_ROWS;
        const int xrow = sm.grp_off[g] + n0;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int bb = it % BST;
          if (!wait_bar(&sm.bempty[bb], ((it / BST) & 1) ^ 1, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* b = bring + bb * B_BYTES;
          tc::mbar_arrive_expect_tx(&sm.bfull[bb], (uint32_t)(KS * nb * XBOX_BYTES));
#pragma unroll
          for (int hk = 0; hk < KS; ++hk)
            for (int j = 0; j < nb; ++j)
              tc::tma_load_2d(b + hk * B_HALF + j * XBOX_BYTES, &tmap_x, kb * SBK + hk * BK, xrow + j * XBOX_ROWS,
                              &sm.bfull[bb], pol_x);
        }
      }
      if (!ok) {
        // drain: wait (bounded) for the copies of the last issued stages to land before leaving
        const uint32_t first = it > (uint32_t)BST ? it - BST : 0;
        for (uint32_t i = first; i < it; ++i) tc::mbar_wait(&sm.bfull[i % BST], (i / BST) & 1, 1u << 16);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (uint32_t q = 0; ok; ++q, ++tcount) {
        const int wk = work_consume(sm, p, q, wk_begin, wk_step, total, abort_flag, ST_TIMEOUT_MMA, false);
        if (wk < 0) {
          ok = wk == -1;
          break;
        }
        int ks;
        const int t = work_tile(sm, p, wk, ks);
        const int kb0 = ks * kblocks / p.ksplit, kb1 = (ks + 1) * kblocks / p.ksplit;
        int g, mt, n0, nval;
        decode_tile<BN>(sm, p.m_tiles, t, g, mt, n0, nval);
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!wait_bar(&sm.tempty[buf], tph ^ 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t N = max(16, (nval + 15) & ~15);
        const uint32_t idesc = tc::idesc_bf16_f32(128, N);
        const uint32_t d = sm.tmem_base + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          if constexpr (F8) {
            // A from tensor memory (the converted slot of this stage), B from the activation ring
            const int ms = it % MSD, bb = it % BST;
            if (!wait_bar(&sm.bfull[bb], (it / BST) & 1, abort_flag, p.status, ST_TIMEOUT_MMA) ||
                !wait_bar(&sm.conv[ms], (it / MSD) & 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t b = tc::smem_u32(bring + bb * B_BYTES);
            const uint32_t ta = sm.tmem_base + 2 * BN + ms * SLOT_COLS;
#pragma unroll
            for (int kk = 0; kk < SBK / 16; ++kk)
              tc::mma_bf16_tmem_a(d, ta + kk * 8, tc::sdesc_k128(b + (kk >> 2) * B_HALF + (kk & 3) * 32), idesc,
                                  (kb != kb0) || kk != 0);
            tc::mma_commit(&sm.mempty[ms]);
            tc::mma_commit(&sm.bempty[bb]);
          } else {
            const int s = it % STAGES, bb = it % BST;
            const uint32_t ph = (it / STAGES) & 1;
            if (!wait_bar(&sm.full[s], ph, abort_flag, p.status, ST_TIMEOUT_MMA) ||
                (SPLIT && !wait_bar(&sm.bfull[bb], (it / BST) & 1, abort_flag, p.status, ST_TIMEOUT_MMA))) {
              ok = false;
              break;
            }
            const uint32_t a = tc::smem_u32(stages + s * STAGE_BYTES);
            const uint32_t b = SPLIT ? tc::smem_u32(bring + bb * B_BYTES) : a + W_BYTES;
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc::mma_bf16(d, tc::sdesc_k128(a + kk * 32), tc::sdesc_k128(b + kk * 32), idesc, (kb != kb0) || kk != 0);
            tc::mma_commit(&sm.empty[s]);
            if (SPLIT) tc::mma_commit(&sm.bempty[bb]);
          }
        }
        if (!ok) break;
        tc::mma_commit(&sm.tfull[buf]);
      }
      // all issued MMAs complete before TMEM is released
      tc::mma_commit(&sm.done);
      tc::mbar_wait(&sm.done, 0, 1u << 20);
    }
  } else if (F8 && warp >= 6) {
    // ------------------------------------------------------------------ FP8: converter warps 6..13 (warp 14 took
    // the branch above)
    // two groups of four warps (one per TMEM lane quadrant) take alternate k-blocks, so that one group's loads,
    // conversions and store waits overlap the other's. Per k-block, in the MMA's order: once the A slot is free and
    // the stage's codes have landed, each thread writes its TMEM lane of the slot from its row of codes, waits for
    // its stores, and arrives on the slot's conv barrier
    const int row = (warp & 3) * 32 + lane;   // the TMEM lane this warp may access
    const uint32_t cg = (uint32_t)(warp - 6) >> 2;
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t qi = 0; ok; ++qi) {
      const int wk = work_consume(sm, p, qi, wk_begin, wk_step, total, abort_flag, ST_TIMEOUT_MMA, true);
      if (wk < 0) break;
      int ks;
      (void)work_tile(sm, p, wk, ks);
      const int kb0 = ks * kblocks / p.ksplit, kb1 = (ks + 1) * kblocks / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if ((it & 1u) != cg) continue;   // the other group's k-block
        const int s = it % STAGES, ms = it % MSD;
        if (!wait_bar(&sm.mempty[ms], ((it / MSD) & 1) ^ 1, abort_flag, p.status, ST_TIMEOUT_MMA) ||
            !wait_bar(&sm.full[s], (it / STAGES) & 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
        tc::fence_after_sync();
        convert_e4m3_row_to_tmem(stages + s * STAGE_BYTES, row,
                                 sm.tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + 2 * BN + ms * SLOT_COLS);
        tc::mbar_arrive(&sm.empty[s]);   // this thread's codes are read (release orders the loads before it)
        tc::tmem_st_wait();
        tc::fence_before_sync();
        tc::mbar_arrive(&sm.conv[ms]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;   // tile row m (TMEM lane)
    const int etid = tid - 64;       // 0..127
    ConfRun run;
#pragma unroll
    for (int i = 0; i < 4; ++i) { run.m[i] = -INFINITY; run.idx[i] = 0x7fffffff; run.s[i] = 0.0; }
    uint32_t tcount = 0;
    for (uint32_t qi = 0;; ++qi, ++tcount) {
      const int wk = work_consume(sm, p, qi, wk_begin, wk_step, total, abort_flag, ST_TIMEOUT_EPILOGUE, true);
      if (wk < 0) break;
      int ks;
      const int t = work_tile(sm, p, wk, ks);
      int g, mt, n0, nval;
      decode_tile<BN>(sm, p.m_tiles, t, g, mt, n0, nval);
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      if (!wait_bar(&sm.tfull[buf], tph, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) break;
      tc::fence_after_sync();
      if (p.ksplit == 1) {
        const float rs = F8 ? f8_row_scale(p, g, mt, row) : 1.f;
        for (int c0 = 0; c0 < nval; c0 += STAGE_COLS) {
          float v[STAGE_COLS];
          const uint32_t taddr = sm.tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + c0;
          tc::tmem_ld16(taddr, v);
          tc::tmem_ld16(taddr + 16, v + 16);
          tc::named_bar_sync(1, 128);  // staging free (previous chunk consumed)
#pragma unroll
          for (int j = 0; j < STAGE_COLS; ++j) staging[j * 128 + row] = F8 ? v[j] * rs : v[j];
          tc::named_bar_sync(1, 128);
          if constexpr (BN == 32) {
            if (p.epi.conf_part) {
              epilogue_logits_conf(p, staging, mt, nval, sm.grp_off[g] + n0, etid, run);
              continue;
            }
          }
          epilogue_chunk<BN>(p, staging, g, mt, n0, nval, c0, sm.grp_off[g], etid);
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&sm.tempty[buf]);
      } else {
        // cluster split-K: this slice's accumulator as [column][128 rows] fp32, in the staging tile (N tile 32) or
        // in the operand ring, idle now (wider N tiles; this CTA's one work item has been consumed)
        float* accs = BN == 32 ? staging : reinterpret_cast<float*>(stages);
        for (int c0 = 0; c0 < nval; c0 += STAGE_COLS) {
          float v[STAGE_COLS];
          const uint32_t taddr = sm.tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + c0;
          tc::tmem_ld16(taddr, v);
          tc::tmem_ld16(taddr + 16, v + 16);
#pragma unroll
          for (int j = 0; j < STAGE_COLS; ++j) accs[(c0 + j) * 128 + row] = v[j];
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&sm.tempty[buf]);
      }
    }
    if constexpr (BN == 32) {
      // one confidence partial per token row and CTA (empty when this CTA produced no tile of the row)
      if (p.epi.conf_part && (etid & 15) == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = (etid >> 4) + 8 * i;
          if (j < sm.grp_cnt[0])
            p.epi.conf_part[(int64_t)(sm.grp_off[0] + j) * p.epi.conf_nparts + blockIdx.x] =
                ConfPartial{run.m[i], run.idx[i], run.s[i]};
        }
      }
    }
  }
  if (p.ksplit > 1) {
    // every slice's staging tile is complete; rank r sums columns [r*nval/ks, (r+1)*nval/ks) over the slices in
    // rank order (distributed shared memory: each thread takes 8 rows of one column and has its loads from every
    // rank in flight together) and runs the epilogue on them. The second cluster barrier keeps each CTA's shared
    // memory alive until its peers have read it: arrive once the reads are done, wait at exit.
    __syncthreads();
    cluster_sync();
    bool arrived = false;
    // a cluster past the device count's tiles (or of an emptied pass) owns no tile: nothing to reduce
    if (warp >= 2 && !*abort_flag && (int)blockIdx.y < sm.total_tiles) {
      const int t = (int)blockIdx.y;
      const int rank = (int)blockIdx.x;
      int g, mt, n0, nval;
      decode_tile<BN>(sm, p.m_tiles, t, g, mt, n0, nval);
      const int etid = tid - 64;
      const int cb = rank * nval / p.ksplit, ce = (rank + 1) * nval / p.ksplit;
      // every slice's accumulator (see above) and, after it, this rank's sums (the operand ring is idle now)
      const float* accs = BN == 32 ? staging : reinterpret_cast<const float*>(stages);
      float* red = reinterpret_cast<float*>(stages) + (BN == 32 ? 0 : 128 * BN);
      // the share is columns [cb, ce) of every slice, one contiguous run of 128-row columns: each thread sums
      // 16-byte vectors of it over the slices in rank order, two vectors at a time with the loads from every
      // slice issued before the first add (2 x ksplit loads from distributed shared memory in flight per thread)
      const int n4 = (ce - cb) * 32;   // float4 vectors in the share
      const float4* src = reinterpret_cast<const float4*>(accs + cb * 128);
      float4* dst = reinterpret_cast<float4*>(red);
      for (int i0 = etid; i0 < n4; i0 += 2 * 128) {
        float4 v[8][2];
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
#pragma unroll
          for (int u = 0; u < 2; ++u)
            v[sp][u] = (sp < p.ksplit && i0 + u * 128 < n4)
                           ? ld_dsmem4(reinterpret_cast<const float*>(src + i0 + u * 128), (uint32_t)sp)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float4 a = v[0][u];
#pragma unroll
          for (int sp = 1; sp < 8; ++sp)
            if (sp < p.ksplit) { a.x += v[sp][u].x; a.y += v[sp][u].y; a.z += v[sp][u].z; a.w += v[sp][u].w; }
          if (i0 + u * 128 < n4) dst[i0 + u * 128] = a;
        }
      }
      cluster_arrive();
      arrived = true;
      tc::named_bar_sync(1, 128);
      for (int c = 0; c < ce - cb; c += STAGE_COLS)
        epilogue_chunk<BN>(p, red + c * 128, g, mt, n0 + cb + c, ce - cb - c, 0, sm.grp_off[g], etid);
    }
    if (!arrived) cluster_arrive();
    cluster_wait();
  }
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(sm.tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------------- CTA pairs
// Compute-bound shapes (N tile 256): a (2, 1, 1) cluster shares every MMA (tcgen05.mma.cta_group::2, M = 256). Rank r
// of the pair owns m-tile 2 mp + r of tile pair mp: it loads that m-tile's 128 weight rows and its half of the N
// tile's token rows (the MMA takes N / 2 rows of B from each CTA, N rounded up to 32) and receives its m-tile's
// accumulator in its own TMEM. Per CTA a stage moves 16 KB of weights and 16 KB of tokens for 128 x 256 x 64 MACs,
// two thirds of a single-CTA 128 x 256 tile's 48 KB, which is what bounds the single-CTA mainloop (operand traffic
// into shared memory per SM).
// Roles: warp 0 of each CTA loads its own operands, both CTAs' copies completing on the leader's full barrier (the
// leader arms it for both); warp 1 of the leader waits for it and issues the MMAs, committing stage release (empty)
// and accumulator ready (tfull) to the barriers of both CTAs; warps 2-5 of each CTA drain their TMEM half and arrive on the
// leader's tempty (128 + 128 arrivals). Measured with the peer instead forwarding each landed stage to the leader
// (a remote arrive after waiting on its own barrier): 2.5x slower, the extra hop stalling every stage.
// The epilogue bounds this kernel at the prefill shape: with its stores left out (a timing build) the down expert
// GEMM at 32768 tokens (K = 512, eight k-steps per tile) took 475 us instead of 937. Its chunks therefore run as a
// pipeline: the next chunk's columns are loaded from TMEM while this one is staged and stored, and the staging
// area is double-buffered, so a chunk needs one barrier instead of two (5 operand stages make room for it):
// 937-955 -> 828-830 us for that GEMM, 1221 -> 1195 us for the SwiGLU GEMM, the 512-row LM head unchanged.
constexpr int PAIR_BN = 256;
constexpr int PAIR_STAGES = 5;
constexpr int PAIR_B_BYTES = (PAIR_BN / 2) * BK * 2;
constexpr int PAIR_STAGE_BYTES = A_BYTES + PAIR_B_BYTES;
constexpr int PAIR_SMEM = 1024 + PAIR_STAGES * PAIR_STAGE_BYTES + 2 * STAGING_BYTES + (int)sizeof(Smem);

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_w2,
                    const __grid_constant__ CUtensorMap tmap_x, const KParams p) {
  constexpr int STAGES = PAIR_STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  float* staging = reinterpret_cast<float*>(base + STAGES * PAIR_STAGE_BYTES);
  Smem& sm = *reinterpret_cast<Smem*>(base + STAGES * PAIR_STAGE_BYTES + 2 * STAGING_BYTES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = tc::cluster_ctarank();
  const bool leader = rank == 0;
  const int m_pairs = p.m_tiles / 2;

  const int n_groups = p.n_dev + p.has_extra + ((p.n_dev + p.has_extra) == 0 ? 1 : 0);
  if (tid == 0) {
    sm.n_groups = n_groups;
    sm.abort_flag = 0;
    sm.drained = 1;   // the leader overwrites the peer's copy at its end (before the final cluster barrier)
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1);
      tc::mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&sm.tfull[b], 1);
      tc::mbar_init(&sm.tempty[b], 256);
    }
    tc::mbar_init(&sm.done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc_pair(&sm.tmem_base, 2 * PAIR_BN);
  __syncthreads();
  cluster_sync();   // both CTAs' barriers exist before any cross-CTA arrive
  pdl_enter();
  if (p.zero_word && blockIdx.x == 0 && threadIdx.x == 0) *p.zero_word = 0u;
  // ---- group table (tiles counted in m-tile pairs)
  const bool dead = p.live && *p.live == 0;
  for (int g = tid; g < n_groups; g += NUM_THREADS) {
    int off, cnt;
    if (g < p.n_dev) {
      off = p.grp_off[g];
      cnt = p.grp_cnt[g];
    } else if (p.has_extra) {
      off = p.extra_off;
      cnt = p.extra_cnt;
    } else {
      off = 0;
      cnt = p.cnt_dev ? min(*p.cnt_dev, p.host_cnt) : p.host_cnt;
    }
    sm.grp_off[g] = off;
    sm.grp_cnt[g] = dead ? 0 : max(cnt, 0);
  }
  __syncthreads();
  {
    int* warp_tot = sm.chunk_sum;
    const int per = (n_groups + NUM_THREADS - 1) / NUM_THREADS;
    const int g0 = tid * per, g1 = min(n_groups, g0 + per);
    int s = 0;
    for (int g = g0; g < g1; ++g) s += ((sm.grp_cnt[g] + PAIR_BN - 1) / PAIR_BN) * m_pairs;
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w2 = 0; w2 < NUM_THREADS / 32; ++w2) {
      const int v = warp_tot[w2];
      if (w2 < warp) before += v;
      all += v;
    }
    int run = before + inc - s;
    for (int g = g0; g < g1; ++g) {
      sm.tile_prefix[g] = run;
      run += ((sm.grp_cnt[g] + PAIR_BN - 1) / PAIR_BN) * m_pairs;
    }
    if (tid == 0) sm.total_tiles = all;
    __syncthreads();
  }
  const int total = sm.total_tiles;
  const int pair = (int)blockIdx.x >> 1, n_pairs = (int)gridDim.x >> 1;
  const int kblocks = p.K / BK;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (each CTA, its own halves)
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tmap_w);
      tc::prefetch_tmap(&tmap_x);
      if (p.has_extra) tc::prefetch_tmap(&tmap_w2);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_x = tc::policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      const uint32_t full0 = tc::mapa_u32(tc::smem_u32(&sm.full[0]), 0);   // the leader's full barriers
      for (int t = pair; t < total && ok; t += n_pairs) {
        int g, mp, n0, nval;
        decode_tile<PAIR_BN>(sm, m_pairs, t, g, mp, n0, nval);
        const bool extra = p.has_extra && g == p.n_dev;
        const CUtensorMap* wm = extra ? &tmap_w2 : &tmap_w;
        const int64_t wrow = extra ? 0 : (int64_t)g * p.w_group_stride;
        const int mt = 2 * mp + (int)rank;
        const int half = min(PAIR_BN, (nval + 31) & ~31) / 2;
        const int nb = (half + XBOX_ROWS - 1) / XBOX_ROWS;
        const uint32_t bytes = A_BYTES + nb * XBOX_BYTES;
        const int xrow = sm.grp_off[g] + n0 + (int)rank * half;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait_bar(&sm.empty[s], ph ^ 1, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) { ok = false; break; }
          uint8_t* a = stages + s * PAIR_STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          // both halves complete on the leader's full barrier, armed by the leader for both CTAs' bytes
          if (leader) tc::mbar_arrive_expect_tx(&sm.full[s], 2 * bytes);
          const uint32_t fb = full0 + 8u * s;
          if (p.swiglu) {
            tc::tma_load_2d_pair(a, wm, kb * BK, (int)(wrow + mt * 64), fb, pol_w);
            tc::tma_load_2d_pair(a + A_BYTES / 2, wm, kb * BK, (int)(wrow + p.M + mt * 64), fb, pol_w);
          } else {
            tc::tma_load_2d_pair(a, wm, kb * BK, (int)(wrow + mt * 128), fb, pol_w);
          }
          for (int j = 0; j < nb; ++j)
            tc::tma_load_2d_pair(b + j * XBOX_BYTES, &tmap_x, kb * BK, xrow + j * XBOX_ROWS, fb, pol_x);
        }
      }
      if (leader) {
        // every issued stage of both CTAs lands before the pair can leave (bounded); the peer passes the final
        // cluster barrier only after this and then reads whether it succeeded
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        bool landed = true;
        for (uint32_t i = first; i < it; ++i)
          landed = tc::mbar_wait(&sm.full[i % STAGES], (i / STAGES) & 1, 1u << 20) && landed;
        // tell the peer (its own shared memory; visible to it after the final cluster barrier)
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(tc::mapa_u32(tc::smem_u32(&sm.drained), 1)),
                     "r"(landed ? 1 : 0) : "memory");
      }
    }
  } else if (warp == 1) {
    if (leader && tc::elect_one()) {
      // ---------------------------------------------------------------- leader: MMA issuer for the pair
      // stage release and accumulator-ready go to the barriers at the same offsets in both CTAs
      const uint32_t own_cl = tc::mapa_u32(tc::smem_u32(&sm), 0), peer_cl = tc::mapa_u32(tc::smem_u32(&sm), 1);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += n_pairs, ++tcount) {
        int g, mp, n0, nval;
        decode_tile<PAIR_BN>(sm, m_pairs, t, g, mp, n0, nval);
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!wait_bar_cluster(&sm.tempty[buf], tph ^ 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t N = (uint32_t)min(PAIR_BN, (nval + 31) & ~31);
        const uint32_t idesc = tc::idesc_bf16_f32(256, N);
        const uint32_t d = sm.tmem_base + buf * PAIR_BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait_bar(&sm.full[s], ph, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t a = tc::smem_u32(stages + s * PAIR_STAGE_BYTES);
          const uint32_t b = a + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc::mma_bf16_pair(d, tc::sdesc_k128(a + kk * 32), tc::sdesc_k128(b + kk * 32), idesc, kb != 0 || kk != 0);
          tc::mma_commit_pair(own_cl + (uint32_t)((uint8_t*)&sm.empty[s] - (uint8_t*)&sm));
          tc::mma_commit_pair(peer_cl + (uint32_t)((uint8_t*)&sm.empty[s] - (uint8_t*)&sm));
        }
        if (!ok) break;
        tc::mma_commit_pair(own_cl + (uint32_t)((uint8_t*)&sm.tfull[buf] - (uint8_t*)&sm));
        tc::mma_commit_pair(peer_cl + (uint32_t)((uint8_t*)&sm.tfull[buf] - (uint8_t*)&sm));
      }
      tc::mma_commit_pair(own_cl + (uint32_t)((uint8_t*)&sm.done - (uint8_t*)&sm));   // all pair MMAs done
      tc::mbar_wait(&sm.done, 0, 1u << 20);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps 2..5 (each CTA, its half)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int etid = tid - 64;
    const uint32_t tempty0 = tc::mapa_u32(tc::smem_u32(&sm.tempty[0]), 0);
    uint32_t tcount = 0, chunk = 0;
    for (int t = pair; t < total; t += n_pairs, ++tcount) {
      int g, mp, n0, nval;
      decode_tile<PAIR_BN>(sm, m_pairs, t, g, mp, n0, nval);
      const int mt = 2 * mp + (int)rank;
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      if (!wait_bar(&sm.tfull[buf], tph, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) break;
      tc::fence_after_sync();
      // the next chunk's columns are in flight while this one is staged and stored
      const uint32_t tb = sm.tmem_base + ((uint32_t)(q * 32) << 16) + buf * PAIR_BN;
      const int nch = (nval + STAGE_COLS - 1) / STAGE_COLS;
      uint32_t ra[STAGE_COLS], rb[STAGE_COLS];
      auto stage_store = [&](const uint32_t* r, int ci) {
        float* st = staging + (chunk & 1) * (STAGING_BYTES / 4);
#pragma unroll
        for (int j = 0; j < STAGE_COLS; ++j) st[j * 128 + row] = __uint_as_float(r[j]);
        tc::named_bar_sync(1, 128);
        epilogue_chunk<PAIR_BN>(p, st, g, mt, n0, nval, ci * STAGE_COLS, sm.grp_off[g], etid);
        ++chunk;
      };
      tmem_ld32_issue(tb, ra);
      for (int ci = 0; ci < nch; ci += 2) {
        tmem_wait_ld32(ra);
        if (ci + 1 < nch) tmem_ld32_issue(tb + (ci + 1) * STAGE_COLS, rb);
        stage_store(ra, ci);
        if (ci + 1 >= nch) break;
        tmem_wait_ld32(rb);
        if (ci + 2 < nch) tmem_ld32_issue(tb + (ci + 2) * STAGE_COLS, ra);
        stage_store(rb, ci + 1);
      }
      tc::fence_before_sync();
      tc::mbar_arrive_cluster(tempty0 + 8u * buf);
    }
  }
  // neither CTA leaves (nor frees TMEM) while its peer may still signal its barriers or read its shared memory
  __syncthreads();
  cluster_sync();
  if (!leader && tid == 0) {
    // the peer's copies complete on the leader's barriers, which the leader drained and reported here: if that
    // drain gave up, copies into this CTA's shared memory may still be in flight. Report it and give them a
    // bounded time to land.
    const int drained = *reinterpret_cast<volatile int*>(&sm.drained);
    if (!drained) {
      if (p.status) atomicExch(p.status, ST_TIMEOUT_PRODUCER);
      for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(sm.tmem_base, 2 * PAIR_BN);
  }
}

// ---------------------------------------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 [rows, K] with 128-byte swizzled boxes of 64 x box_rows, or (u8) E4M3 codes [rows, K] with 128-byte swizzled
// boxes of 128 codes x box_rows (the converter warps read them row by row)
int make_map(CUtensorMap* m, const void* ptr, int64_t rows, int K, int box_rows, bool u8 = false) {
  EncodeTiledFn enc = get_encode();
  if (!enc) {
    dllm_host::set_error("cuTensorMapEncodeTiled unavailable");
    return DLLM_ERR_CUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * (u8 ? 1 : 2)};
  cuuint32_t box[2] = {(cuuint32_t)(u8 ? BK * F8_KS : BK), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    dllm_host::set_error("cuTensorMapEncodeTiled failed (%d) rows=%lld K=%d box_rows=%d", (int)r, (long long)rows,
                         K, box_rows);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

// Cluster split-K launch: grid (ksplit, tiles), cluster (ksplit, 1, 1), one work item per CTA.
int launch_cluster_splitk(const GemmArgs& a, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                          const KParams& kp, cudaStream_t s);

template <int BN, int STAGES, bool F8 = false, int BST = 1>
int launch(const GemmArgs& a, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
           const KParams& kp, cudaStream_t s) {
  // (matches the kernel's layout: bf16 stages of [weights][activations], or with BST > 1 a ring of weight tiles and
  // one of activation tiles; FP8 rings of codes and of activations)
  constexpr int SMEM = F8 ? 1024 + STAGES * RAW_BYTES + BST * BN * BK * 2 * F8_KS + STAGING_BYTES + (int)sizeof(Smem)
                     : BST > 1 ? 1024 + STAGES * A_BYTES + BST * BN * BK * 2 + STAGING_BYTES + (int)sizeof(Smem)
                               : 1024 + STAGES * (A_BYTES + BN * BK * 2) + STAGING_BYTES + (int)sizeof(Smem);
  static_assert(SMEM <= SMEM_LIMIT, "shared memory budget");
  // With programmatic dependent launch a CTA allocates tensor memory before it waits for the kernels ahead of it.
  // More than half an SM's shared memory per CTA keeps two tensor-memory kernels from sharing an SM, so a later
  // kernel can never hold the columns an earlier one is still waiting to allocate.
  static_assert(SMEM > 233472 / 2, "tensor-memory kernels must not share an SM");
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES, F8, BST>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaFuncSetAttribute(gemm_tc)");
    configured = true;
  }
  launch_pdl((gemm_tc_kernel<BN, STAGES, F8, BST>), num_sms(),
             F8 ? NUM_THREADS_F8 : (BST > 1 ? NUM_THREADS_SPLIT : NUM_THREADS), SMEM, s, mw, mw2, mx, kp);
  DLLM_CHECK_LAUNCH("gemm_tc_kernel");
  return DLLM_OK;
}

constexpr int SPLITK_BN = 32, SPLITK_STAGES = 9;

// Output tiles of a dense split-K GEMM: 128-row weight tiles x 32-row N tiles.
static int splitk_tiles(const GemmArgs& a) { return (a.M / 128) * ((a.host_cnt + SPLITK_BN - 1) / SPLITK_BN); }
constexpr int SPLITK_SMEM = 1024 + SPLITK_STAGES * (A_BYTES + SPLITK_BN * BK * 2) + STAGING_BYTES + (int)sizeof(Smem);

static cudaError_t configure_splitk() {
  static cudaError_t st = cudaFuncSetAttribute(gemm_tc_kernel<SPLITK_BN, SPLITK_STAGES>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, SPLITK_SMEM);
  return st;
}

// How many clusters of ks split-K CTAs can be resident at once (each cluster must sit inside one GPC, so sizes that
// do not divide the GPCs' SM counts leave SMs unused); cached per size.
static int max_active_clusters(int ks) {
  static int cache[9] = {0};
  if (ks < 1 || ks > 8) return 0;
  if (cache[ks] > 0) return cache[ks];
  int n = 0;
  if (configure_splitk() == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ks, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SPLITK_SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<SPLITK_BN, SPLITK_STAGES>, &cfg) != cudaSuccess) n = 0;
  }
  if (n <= 0) {
    cudaGetLastError();
    n = num_sms() / (2 * ks);   // conservative when the query is unavailable
  }
  cache[ks] = std::max(n, 1);
  return cache[ks];
}

int launch_cluster_splitk(const GemmArgs& a, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                          const KParams& kp, cudaStream_t s) {
  constexpr int SMEM = SPLITK_SMEM;
  {
    cudaError_t e = configure_splitk();
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaFuncSetAttribute(gemm_tc cluster)");
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kp.ksplit, splitk_tiles(a), 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kp.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<SPLITK_BN, SPLITK_STAGES>, mw, mw2, mx, kp);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaLaunchKernelEx(gemm_tc cluster split-K)");
  DLLM_CHECK_LAUNCH("gemm_tc_kernel (cluster split-K)");
  return DLLM_OK;
}

// ---- wide split-K: dense projections over several N tiles of rows (the 512 rows of a denoising block) whose
// 128-row tiles would each stream a whole K of weights and tokens on fewer SMs than the GPU has. N tiles of 64, 128
// or 256 rows split along K over a thread-block cluster put every SM to work on a slice with less operand traffic per
// SM; each slice's accumulator goes through the idle operand ring to the cluster's reduction.
template <int BN, int STAGES>
constexpr int splitk_smem() {
  return 1024 + STAGES * (A_BYTES + BN * BK * 2) + STAGING_BYTES + (int)sizeof(Smem);
}

template <int BN, int STAGES>
static cudaError_t configure_splitk_t() {
  static cudaError_t st = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               splitk_smem<BN, STAGES>());
  return st;
}

template <int BN, int STAGES>
static int max_active_clusters_t(int ks) {
  static int cache[9] = {0};
  if (ks < 1 || ks > 8) return 0;
  if (cache[ks] > 0) return cache[ks];
  int n = 0;
  if (configure_splitk_t<BN, STAGES>() == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ks, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = splitk_smem<BN, STAGES>();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<BN, STAGES>, &cfg) != cudaSuccess) n = 0;
  }
  if (n <= 0) {
    cudaGetLastError();
    n = num_sms() / (2 * ks);
  }
  cache[ks] = std::max(n, 1);
  return cache[ks];
}

template <int BN, int STAGES>
static int launch_wide_splitk(const GemmArgs& a, const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx,
                              const KParams& kp, cudaStream_t s) {
  static_assert(splitk_smem<BN, STAGES>() <= SMEM_LIMIT, "shared memory budget");
  static_assert(STAGES * (A_BYTES + BN * BK * 2) >= 128 * BN * 4 + 128 * (BN / 2) * 4,
                "the operand ring holds a slice's accumulator and a rank's sums");
  cudaError_t e = configure_splitk_t<BN, STAGES>();
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaFuncSetAttribute(gemm_tc wide split-K)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kp.ksplit, (a.M / 128) * ((a.host_cnt + BN - 1) / BN), 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = splitk_smem<BN, STAGES>();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kp.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, STAGES>, mw, mw2, mx, kp);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaLaunchKernelEx(gemm_tc wide split-K)");
  DLLM_CHECK_LAUNCH("gemm_tc_kernel (wide split-K)");
  return DLLM_OK;
}

static_assert(PAIR_SMEM <= SMEM_LIMIT, "shared memory budget (CTA pairs)");
static_assert(PAIR_SMEM > 233472 / 2, "tensor-memory kernels must not share an SM");

// Clusters of two resident at once for the CTA-pair kernel (cached).
static int pair_clusters() {
  static int n = 0;
  if (n > 0) return n;
  int m = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&m, gemm_tc_pair_kernel, &cfg) != cudaSuccess || m <= 0) {
    cudaGetLastError();
    m = num_sms() / 2;
  }
  n = std::max(1, m);
  return n;
}

int launch_pair(const CUtensorMap& mw, const CUtensorMap& mw2, const CUtensorMap& mx, const KParams& kp,
                cudaStream_t s) {
  static cudaError_t st = cudaFuncSetAttribute(gemm_tc_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               PAIR_SMEM);
  if (st != cudaSuccess) return dllm_host::cuda_status(st, "cudaFuncSetAttribute(gemm_tc pair)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pair_clusters(), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tc_pair_kernel, mw, mw2, mx, kp);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaLaunchKernelEx(gemm_tc pair)");
  DLLM_CHECK_LAUNCH("gemm_tc_pair_kernel");
  return DLLM_OK;
}

}  // namespace

int gemm_bf16_tc(const GemmArgs& a, cudaStream_t s) {
  DLLM_REQUIRE(a.K % BK == 0 && a.K > 0, DLLM_ERR_UNSUPPORTED, "gemm: K=%d must be a positive multiple of 64", a.K);
  DLLM_REQUIRE(a.swiglu ? (a.M % 64 == 0) : (a.M % 128 == 0), DLLM_ERR_UNSUPPORTED,
               "gemm: M=%d must be a multiple of %d", a.M, a.swiglu ? 64 : 128);
  DLLM_REQUIRE(a.n_dev + a.has_extra <= MAX_GROUPS, DLLM_ERR_UNSUPPORTED, "gemm: too many groups");
  DLLM_REQUIRE(((uintptr_t)a.x % 16 == 0) && ((uintptr_t)a.w % 16 == 0) && (!a.w2 || (uintptr_t)a.w2 % 16 == 0),
               DLLM_ERR_ALIGN, "gemm: operands must be 16-byte aligned");
  if (a.epi.kind == EPI_QKV)
    DLLM_REQUIRE(a.epi.d == 128 && a.epi.rope_tab != nullptr && ((uintptr_t)a.epi.rope_tab % 16) == 0,
                 DLLM_ERR_UNSUPPORTED, "gemm: QKV epilogue needs head dim 128 and the block's RoPE table");
  const int box_rows = a.swiglu ? 64 : 128;
  const bool f8 = a.w_fp8 != 0;
  if (f8) {
    DLLM_REQUIRE(a.w_scale && (!a.w2 || a.w2_scale), DLLM_ERR_INVALID_ARG, "gemm: FP8 weights need their row scales");
    DLLM_REQUIRE(a.epi.kind == EPI_STORE || a.epi.kind == EPI_SWIGLU, DLLM_ERR_UNSUPPORTED,
                 "gemm: FP8 weights take the store or SwiGLU epilogue");
    DLLM_REQUIRE(a.K % (BK * F8_KS) == 0, DLLM_ERR_UNSUPPORTED, "gemm: FP8 weights need K=%d a multiple of %d",
                 a.K, BK * F8_KS);
  }
  CUtensorMap mw, mw2, mx;
  int st = make_map(&mw, a.w, a.w_rows, a.K, box_rows, f8);
  if (st) return st;
  st = make_map(&mw2, a.w2 ? a.w2 : a.w, a.w2 ? a.w2_rows : a.w_rows, a.K, box_rows, f8);
  if (st) return st;
  st = make_map(&mx, a.x, a.x_rows, a.K, XBOX_ROWS);
  if (st) return st;
  KParams kp;
  kp.K = a.K;
  kp.M = a.M;
  kp.swiglu = a.swiglu;
  kp.m_tiles = a.swiglu ? a.M / 64 : a.M / 128;
  kp.w_group_stride = a.w_group_stride;
  kp.n_dev = a.n_dev;
  kp.has_extra = a.has_extra;
  kp.extra_off = a.extra_off;
  kp.extra_cnt = a.extra_cnt;
  kp.host_cnt = a.host_cnt;
  kp.grp_off = a.grp_off;
  kp.grp_cnt = a.grp_cnt;
  kp.cnt_dev = a.cnt_dev;
  kp.live = a.live;
  kp.zero_word = a.zero_word;
  kp.w_scale = a.w_scale;
  kp.w2_scale = a.w2_scale;
  kp.epi = a.epi;
  kp.status = a.status;
  const WideSplit wide = wide_splitk_plan(a);
  const int bn = wide.ks > 1 ? wide.bn : gemm_bn(a);
  const int ks = wide.ks > 1 ? wide.ks : gemm_splitk_factor(a, bn);
  if (a.epi.conf_part)
    DLLM_REQUIRE(a.epi.conf_nparts > 0 && gemm_conf_parts(a) == a.epi.conf_nparts, DLLM_ERR_UNSUPPORTED,
                 "gemm: fused confidence epilogue unsupported for this shape");
  kp.ksplit = ks;
  // grouped launches of single-CTA tiles take their tiles from the work counter (the CTA pair kernel keeps its
  // static schedule)
  kp.work_ctr = ((a.swiglu || a.n_dev || a.has_extra) && ks == 1) ? a.work_ctr : nullptr;
  kp.prefetch_w = (!a.swiglu && !a.n_dev && !a.has_extra && (a.host_cnt <= (ks > 1 ? 32 : bn) || !a.cnt_dev)) ? 1 : 0;
  int st2;
  if (f8) {   // single-CTA tiles, no split-K (the weight-streaming shapes FP8 weights serve)
    // (weight-code ring, activation ring): the activation ring also has to cover a load from L2 plus the wait for
    // the stage's conversion and MMA, so it is not kept minimal
    if (bn == 32) st2 = launch<32, 9, true, 6>(a, mw, mw2, mx, kp, s);
    else if (bn == 64) st2 = launch<64, 8, true, 4>(a, mw, mw2, mx, kp, s);
    else st2 = launch<128, 6, true, 3>(a, mw, mw2, mx, kp, s);
  } else if (gemm_uses_pairs(a)) {
    kp.prefetch_w = 0;
    st2 = launch_pair(mw, mw2, mx, kp, s);
  } else if (wide.ks > 1) {
    st2 = wide.bn == 64 ? launch_wide_splitk<64, 8>(a, mw, mw2, mx, kp, s)
          : wide.bn == 128 ? launch_wide_splitk<128, 6>(a, mw, mw2, mx, kp, s)
                           : launch_wide_splitk<256, 4>(a, mw, mw2, mx, kp, s);
  } else if (ks > 1) st2 = launch_cluster_splitk(a, mw, mw2, mx, kp, s);
  else {
    // single-CTA tiles: a weight ring and an activation ring. Measured on a 20-layer block at N tile 128 (same
    // GPU, weight + activation stages of the expert GEMMs): 8 + 4 took 150.7 ms, 7 + 5 151.3, 6 + 6 151.9, 9 + 3
    // 153.1, a shared ring of 6 stages 153.9; the same split for the dense projections (QKV, output) 150.5 -> 150.1
    if (bn == 32) st2 = launch<32, 11, false, 4>(a, mw, mw2, mx, kp, s);
    else if (bn == 64) st2 = launch<64, 10, false, 4>(a, mw, mw2, mx, kp, s);
    else if (bn == 96) st2 = launch<96, 8, false, 5>(a, mw, mw2, mx, kp, s);
    else if (bn == 128) st2 = launch<128, 8, false, 4>(a, mw, mw2, mx, kp, s);
    else st2 = launch<256, 6, false, 2>(a, mw, mw2, mx, kp, s);
  }
  return st2;
}

int bn_for(int max_cnt) {
  if (max_cnt <= 32) return 32;
  if (max_cnt <= 64) return 64;
  if (max_cnt <= 128) return 128;
  return 256;
}

static bool dense(const GemmArgs& a) { return !a.swiglu && !a.n_dev && !a.has_extra; }

// N tile: the smallest that covers the largest group, except that a dense projection with too few output tiles to
// occupy half the SMs takes narrower N tiles first (the extra re-reads of its weight tiles hit L2). Narrower still
// loses: measured at 512 rows, N tile 128 (96 QKV tiles) beats 64 (192) and 32 (384), whose small MMAs and extra
// operand traffic cost more than the idle SMs.
int gemm_bn(const GemmArgs& a) {
  int bn = bn_for(a.max_cnt);
  if (a.w_fp8) return std::min(bn, 128);   // FP8 weights: single-CTA tiles of at most 128 rows
  if (dense(a)) {
    const int mt = a.M / 128;
    while (bn > 32 && mt * ((a.max_cnt + bn - 1) / bn) < num_sms() / 2) bn /= 2;
    // N tile 96 where 128 leaves more than a quarter of the SMs without a tile and 96 still fits one wave (the QKV
    // projection of 512 rows: 96 -> 144 tiles, each CTA moving 7/8 of the operand bytes)
    if (bn == 128 && mt * ((a.max_cnt + 127) / 128) < num_sms() * 3 / 4 && mt * ((a.max_cnt + 95) / 96) <= num_sms())
      bn = 96;
  }
  return bn;
}

// Split-K for dense projections that still leave most SMs idle at N tile 32 (all rows in one tile): K slices of
// at least two 64-wide blocks, at most 8 (the portable cluster size), and only as many as let every tile's cluster
// be resident at once (a second wave would double the kernel's time).
int gemm_splitk_factor(const GemmArgs& a, int bn) {
  // the grid is (slices, tiles) with the tile count fixed on the host: rows from a device count are excluded,
  // except that a single N tile stays a single N tile for any count
  if (a.dtype != DLLM_BF16 || !dense(a) || bn != 32 || a.w_fp8) return 1;
  if (a.cnt_dev && a.host_cnt > 32) return 1;
  const int tiles = splitk_tiles(a);
  const int kblocks = a.K / BK;
  if (tiles <= 0 || tiles * 2 > num_sms() || kblocks < 4) return 1;
  int ks = std::max(1, std::min(std::min(kblocks / 2, 8), num_sms() / tiles));
  while (ks > 1 && tiles > max_active_clusters(ks)) --ks;
  return ks;
}

// Wide split-K plan (see launch_wide_splitk) for a dense bf16 projection over more than one 32-row tile with a
// row count fixed on the host and at most four 128-row weight tiles (the router's logits): among N tiles of 64,
// 128 and 256 rows and 2..8 K slices whose clusters all fit in one wave, the one with the least operand traffic per
// CTA ((128 + N tile) x K / slices), taken when it is at most three quarters of the plain kernel's. Measured at 512
// rows: the router (256 experts x 2048) 32.1 -> 29.4 us for logits, top-k and permutation with N tile 128 (64 CTAs),
// and N tile 64 (128 CTAs) took a 20-layer block from 149.6 to 147.6 ms; the wider QKV and output projections
// gained nothing (15.9 us both ways) or lost (12.5 -> 15.0 us): their slices' 64-128 KB accumulators cost as much
// to stage and reduce as the operand traffic saved.
WideSplit wide_splitk_plan(const GemmArgs& a) {
  WideSplit best;
  if (a.dtype != DLLM_BF16 || !dense(a) || a.w_fp8 || a.epi.conf_part || a.cnt_dev || a.host_cnt <= 32) return best;
  if (a.M > 512) return best;
  const int kblocks = a.K / BK, mt = a.M / 128, rows = a.host_cnt, sms = num_sms();
  const int bn0 = gemm_bn(a);
  const int tiles0 = mt * ((rows + bn0 - 1) / bn0);
  const double base = (double)(128 + std::min(bn0, rows)) * a.K * ((tiles0 + sms - 1) / sms);
  double cost = 0.75 * base;
  for (int bn : {64, 128, 256}) {
    const int tiles = mt * ((rows + bn - 1) / bn);
    for (int ks = 2; ks <= 8 && 2 * ks <= kblocks; ++ks) {
      if (tiles * ks > sms) break;
      const int act = bn == 64 ? max_active_clusters_t<64, 8>(ks)
                      : bn == 128 ? max_active_clusters_t<128, 6>(ks) : max_active_clusters_t<256, 4>(ks);
      if (tiles > act) continue;
      const double c = (double)(128 + std::min(bn, rows)) * a.K / ks;
      if (c < cost) { cost = c; best.bn = bn; best.ks = ks; }
    }
  }
  return best;
}

bool gemm_uses_pairs(const GemmArgs& a) {
  if (a.dtype != DLLM_BF16 || a.w_fp8 || a.epi.conf_part || gemm_bn(a) != 256 || gemm_splitk_factor(a, 256) != 1)
    return false;
  return a.swiglu ? (a.M / 64) % 2 == 0 : (a.M / 128) % 2 == 0;
}

int gemm_conf_parts(const GemmArgs& a) {
  if (a.dtype != DLLM_BF16 || !dense(a) || a.epi.kind != EPI_STORE || a.epi.out_f32) return 0;
  if (a.host_cnt > 32 || a.max_cnt > 32) return 0;
  const int bn = gemm_bn(a);
  if (bn != 32 || gemm_splitk_factor(a, bn) != 1) return 0;
  return num_sms();   // the persistent grid: every CTA writes its slot of every row
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace dllm
