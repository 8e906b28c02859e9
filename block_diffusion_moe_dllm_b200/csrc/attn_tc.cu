// Block-causal attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16, head dim 128.
// Source: LLaDA2.0-Uni paper review, sections "Block Diffusion Language Model (BDLM)" (bidirectional inside a
// block, left-to-right across blocks) and "MoE 백본과 Block-wise Attention".
//
// One CTA per (batch row, kv head, tile of queries, key split). The 128-row M tile packs the G = Hq / Hkv query
// heads that share the kv head with 128 / G queries (row r = query r / G, head r % G), so every K/V tile staged in
// shared memory serves the whole group. Per 128-key tile j:
//   S_j = Q K_j^T   tcgen05.mma M=128 N=128 K=128 (Q, K K-major, TMA 128-byte swizzled) -> TMEM (two buffers)
//   softmax         two groups of 4 warps take alternate tiles (group j mod 2), one thread per query row: mask,
//                   scale, maximum; P_j = 2^(s - m_ref) as bf16, written back into the first 64 columns of S_j's
//                   TMEM buffer (one buffer per group)
//   O_g += P_j V_j  tcgen05.mma with A = P_j from TMEM and B = V_j (MN-major, straight from the [key][d] cache);
//                   each group accumulates its own O_g in TMEM across its tiles, and the two are combined by
//                   log-sum-exp at the end. While one group waits on loads, barriers and TMEM, the other's
//                   exponentials keep the special-function unit busy.
// m_ref is a per-row reference maximum that only moves when a tile's maximum exceeds it by more than 2^8 (then
// O in TMEM and the row sum are rescaled once); in between, P values up to 2^8 are exact in bf16's range and the
// result is the same softmax. Warp 0 issues TMA (Q once; K and V through a 3-stage ring), warp 1 issues the MMAs
// from one thread, warps 2..9 run the softmax, combine O_0 and O_1 and write the output; with several key splits
// (a thread-block cluster) every split pushes its unnormalised rows into the owning CTA's shared memory and the
// owners merge them by log-sum-exp. Every mbarrier wait is bounded; on expiry the kernel records a status word
// and leaves.
#include "common.cuh"
#include "tc.cuh"
#include "misc.h"
#include <cuda.h>
#include <algorithm>
#include <mutex>

namespace dllm {
namespace {

constexpr int NT = 320;                     // warp 0 TMA, warp 1 MMA, warps 2..9 softmax (two per query row)
constexpr int KT = 128;                     // keys per tile
constexpr int CHUNK = 128 * 64 * 2;         // one 64-wide K-major chunk of a 128-row tile: 16 KB
constexpr int TILE = 2 * CHUNK;             // 128 rows x 128 elements: 32 KB
constexpr int STAGES = 3;
constexpr int BARS_BYTES = 2048;
constexpr short kNoKey = 0x7fff;            // relative block of a key past n_keys (never visible)
constexpr float kRescaleLog2 = 8.f;
// named barriers: 1 + g = softmax group g's 128 threads inside its loop; kBarAll = all 256 softmax threads after
// the loops (distinct ids, since one group can leave its loop while the other still synchronises inside its own)
constexpr int kBarAll = 3;         // O and the row sum are rescaled when the maximum grows by > 2^8
constexpr int kRecvStride = 132;            // floats per exchanged row: o[128], m, l, 2 pad (16-byte multiple)
constexpr int SMEM = 1024 + TILE /*Q*/ + STAGES * 2 * TILE /*K,V*/ + BARS_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
// with programmatic dependent launch, tensor memory is allocated before the wait for earlier kernels: one such
// CTA per SM (more than half the SM's shared memory) keeps a later kernel from holding columns an earlier needs
static_assert(SMEM > 233472 / 2, "tensor-memory kernels must not share an SM");
static_assert(135 * kRecvStride * 4 <= STAGES * 2 * TILE,
              "split exchange (n_splits * ceil(128 / n_splits) rows, at most 8 splits) exceeds the K/V ring");

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[STAGES];
  uint64_t kv_empty[STAGES];
  uint64_t s_full[2];   // per softmax group: S of the group's next tile is in the group's TMEM buffer
  uint64_t p_ready[2];  // per group: P of its tile written over S (and the group's O rescaled if needed)
  uint64_t o_full[2];   // per group: phase i completes when the group's i-th P V is accumulated into its O
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  short kblk[2][2][KT];     // [group][tile parity within the group][key]: block of the key relative to the CTA's
                            // first query block, clamped to [-32768, 32766] (kNoKey past n_keys)
  unsigned vis_w[2][2][4];  // [group][parity][warp]: ballots of "key visible to every query of the CTA"
};
static_assert(sizeof(Bars) <= BARS_BYTES, "barrier block exceeds its shared-memory reservation");

struct AttnTcParams {
  int B, Lq, Hq, Hkv, G, QT, n_qtiles, n_keys, cap, blk_len, q_pos0;
  int n_splits, tiles_per_split;
  uint32_t blk_magic, blk_shift;   // key position / blk_len = (pos * blk_magic) >> blk_shift for 0 <= pos < 2^31
  float scale_log2;
  const int32_t* key_pos;
  __nv_bfloat16* out;   // [B, Lq, Hq, 128]
  int32_t* status;
  const int32_t* live;  // nullable: *live == 0 = a denoising pass with no masked position left (nothing to do)
};

// Shared-memory descriptor of an MN-major operand with 128-byte swizzling: rows of 128 bytes along K (one key per
// row), 8-row atoms 1024 bytes apart (stride byte offset), and 64-element N groups lbo bytes apart (leading byte
// offset). Version 1, layout type 2.
__device__ __forceinline__ uint64_t sdesc_mn128(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Integer division by the block length without the divide sequence (which would queue on the special-function unit
// behind the softmax's exponentials): multiply by m = ceil(2^(31+s) / d), 2^(s-1) < d <= 2^s, and keep the bits
// above 31 + s; exact for 0 <= n < 2^31 since n (m d - 2^(31+s)) < 2^(31+s) (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994).
__device__ __forceinline__ int div_blk(int n, uint32_t m, uint32_t shift) {
  return (int)(((uint64_t)(uint32_t)n * m) >> shift);
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                         int code) {
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

// Named barrier over n threads that also ORs a predicate across them: every participant gets the same answer.
__device__ __forceinline__ bool bar_sync_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 32 columns without the wait: the registers are valid after tcgen05.wait::ld.
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

// Each lane reads 64 consecutive 32-bit columns of its own TMEM lane (two loads in flight, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  tmem_ld32_issue(taddr, r);
  tmem_ld32_issue(taddr + 32, r + 32);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// A whole 128-column row of S: four loads in flight, one wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t r[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32_issue(taddr + 32 * c, r + 32 * c);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// Packed fp32 pairs (sm_100 f32x2 instructions) and the hardware base-2 exponential (ex2.approx.ftz: relative
// error about 2^-22; results below 2^-126 flush to 0, negligible next to the row's reference term 1).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__global__ void __launch_bounds__(NT, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const AttnTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + TILE;                    // [STAGES][TILE]
  uint8_t* sV = sK + STAGES * TILE;           // [STAGES][TILE]
  Bars& bar = *reinterpret_cast<Bars*>(sV + STAGES * TILE);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int bx = blockIdx.y;
  const int qt = bx % p.n_qtiles;
  bx /= p.n_qtiles;
  const int g = bx % p.Hkv;
  const int b = bx / p.Hkv;
  const int split = blockIdx.x;      // = rank in the cluster of this tile's key splits
  const int q0 = qt * p.QT;

  // key tiles of this split; causal bound: a query tile never sees keys of blocks after its last query's block
  int n_keys_eff = p.n_keys;
  if (!p.key_pos) {
    const int last_q = min(p.Lq, q0 + p.QT) - 1;
    const int lim = ((p.q_pos0 + last_q) / p.blk_len + 1) * p.blk_len;
    n_keys_eff = min(n_keys_eff, lim);
  }
  const int n_tiles_all = (n_keys_eff + KT - 1) / KT;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(n_tiles_all, t_begin + p.tiles_per_split);
  const int ntile = max(0, t_end - t_begin);

  if (tid == 0) {
    bar.abort_flag = 0;
    tc::mbar_init(&bar.q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&bar.kv_full[s], 1);
      tc::mbar_init(&bar.kv_empty[s], 1);
    }
    for (int g2 = 0; g2 < 2; ++g2) {
      tc::mbar_init(&bar.s_full[g2], 1);
      tc::mbar_init(&bar.p_ready[g2], 128);
      tc::mbar_init(&bar.o_full[g2], 1);
    }
    tc::mbar_init(&bar.done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&bar.tmem_base, 512);
  __syncthreads();
  pdl_enter();         // everything above is on-chip set-up
  if (p.live && *p.live == 0) {
    // nothing to do: no copy or MMA was issued, so free the tensor memory and leave (every CTA of every cluster
    // reads the same word and leaves here, before any cluster barrier or distributed shared memory access)
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(bar.tmem_base, 512);
    return;
  }
  volatile int* abort_flag = &bar.abort_flag;
  const uint32_t tS = bar.tmem_base;          // S buffers (group 0, group 1) at columns [0,128) and [128,256)
  const uint32_t tO = bar.tmem_base + 256;    // O_0, O_1 at columns [256,384) and [384,512)

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      const uint64_t pol_kv = tc::policy_evict_first();
      const uint64_t pol_q = tc::policy_evict_last();
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      if (ntile > 0) {
        tc::mbar_arrive_expect_tx(&bar.q_full, TILE);
        for (int c = 0; c < 2; ++c) {
          // box (64 d, G heads, QT queries, 1 row) at (64c, g*G, q0, b)
          asm volatile(
              "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
              " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(tc::smem_u32(sQ + c * CHUNK)),
              "l"(reinterpret_cast<uint64_t>(&tm_q)), "r"(64 * c), "r"(g * p.G), "r"(q0), "r"(b),
              "r"(tc::smem_u32(&bar.q_full)), "l"(pol_q)
              : "memory");
        }
      }
      bool ok = true;
      int it = 0;
      for (int j = 0; j < ntile && ok; ++j, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!wait_bar(&bar.kv_empty[s], ph ^ 1, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) { ok = false; break; }
        // the rest of the ring only once the first tile has landed: every CTA of the launch requests its first
        // tile alone, so those arrive first (with the whole ring requested at once by every CTA, the first tiles
        // came in late, behind the others' later stages)
        if (it == 1 && !wait_bar(&bar.kv_full[0], 0, abort_flag, p.status, ST_TIMEOUT_PRODUCER)) { ok = false; break; }
        const int key0 = (t_begin + j) * KT;
        const int bg = b * p.Hkv + g;
        tc::mbar_arrive_expect_tx(&bar.kv_full[s], 2 * TILE);
        for (int c = 0; c < 2; ++c) {
          // box (64 d, 128 keys, 1) at (64c, key0, b*Hkv + g); keys >= n_keys are out of the map: zero-filled
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
              " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(tc::smem_u32(sK + s * TILE + c * CHUNK)),
              "l"(reinterpret_cast<uint64_t>(&tm_k)), "r"(64 * c), "r"(key0), "r"(bg),
              "r"(tc::smem_u32(&bar.kv_full[s])), "l"(pol_kv)
              : "memory");
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
              " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(tc::smem_u32(sV + s * TILE + c * CHUNK)),
              "l"(reinterpret_cast<uint64_t>(&tm_v)), "r"(64 * c), "r"(key0), "r"(bg),
              "r"(tc::smem_u32(&bar.kv_full[s])), "l"(pol_kv)
              : "memory");
        }
      }
      if (!ok) {
        uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t i = first; i < (uint32_t)it; ++i) tc::mbar_wait(&bar.kv_full[i % STAGES], (i / STAGES) & 1, 1u << 16);
        if (ntile > 0) tc::mbar_wait(&bar.q_full, 0, 1u << 16);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idesc_s = tc::idesc_bf16_f32(128, 128);                  // A, B K-major
      const uint32_t idesc_o = tc::idesc_bf16_f32(128, 128) | (1u << 16);     // B MN-major
      const uint32_t aQ = tc::smem_u32(sQ);
      bool ok = ntile > 0 && wait_bar(&bar.q_full, 0, abort_flag, p.status, ST_TIMEOUT_MMA);
      auto issue_s = [&](int j) -> bool {
        const int s = j % STAGES;
        if (!wait_bar(&bar.kv_full[s], (j / STAGES) & 1, abort_flag, p.status, ST_TIMEOUT_MMA)) return false;
        tc::fence_after_sync();
        const uint32_t aK = tc::smem_u32(sK + s * TILE);
        const uint32_t d = tS + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
          tc::mma_bf16(d, tc::sdesc_k128(aQ + off), tc::sdesc_k128(aK + off), idesc_s, kk != 0);
        }
        tc::mma_commit(&bar.s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && ntile > 1) ok = issue_s(1);
      for (int j = 0; j < ntile && ok; ++j) {
        const int g = j & 1;
        // P_j written over S_j in group g's buffer (and O_g rescaled if needed)
        if (!wait_bar(&bar.p_ready[g], (j >> 1) & 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
        tc::fence_after_sync();
        const int s = j % STAGES;
        const uint32_t aV = tc::smem_u32(sV + s * TILE);
        const uint32_t tP = tS + g * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_tmem_a(tO + g * 128, tP + kk * 8, sdesc_mn128(aV + kk * 2048, CHUNK), idesc_o,
                          (j >= 2 || kk != 0) ? 1u : 0u);
        tc::mma_commit(&bar.o_full[g]);
        tc::mma_commit(&bar.kv_empty[s]);
        // S_{j+2} reuses group g's buffer: the tcgen05 MMAs of this thread execute in issue order, so it cannot
        // overwrite P_j before P_j V_j has read it
        if (j + 2 < ntile && !issue_s(j + 2)) { ok = false; break; }
      }
      tc::mma_commit(&bar.done);
      tc::mbar_wait(&bar.done, 0, 1u << 20);
    }
  }

  // ------------------------------------------------------------------ softmax / output warps 2..9
  // Group grp = 0 (warps 2..5) takes the split's tiles 0, 2, 4, ..., group 1 (warps 6..9) tiles 1, 3, 5, ...; in a
  // group, one thread per query row (TMEM lane). At the end every thread of either group combines O_0 and O_1 for
  // its row over output columns [64 grp, 64 grp + 64).
  const int q4 = warp & 3;
  const int row = q4 * 32 + lane;      // TMEM lane = tile row
  const int grp = (warp - 2) >> 2;
  const int gtid = ((warp - 2) & 3) * 32 + lane;   // 0..127 within the group
  const int col0 = 64 * grp;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  float o[64];
  float m_ref = -INFINITY, l_row = 0.f;
  if (warp >= 2) {
    const int qi = row / p.G;
    const int qg = q0 + qi;              // query index in the row
    const int qblk_min = (p.q_pos0 + q0) / p.blk_len;  // rows of the tile past Lq never write output
    const int qrel = (p.q_pos0 + qg) / p.blk_len - qblk_min;
    const uint64_t scale2 = pk2(p.scale_log2, p.scale_log2);
    const uint32_t tSg = tS + grp * 128 + lane_off;
    const uint32_t tOg = tO + grp * 128 + lane_off;
    const int n_my = ntile > grp ? (ntile - grp + 1) / 2 : 0;
    float mg = -INFINITY, l = 0.f;
    bool ok = true;
    // A failed wait marks this thread (and the shared abort flag); the group's 128 threads leave the loop
    // together at the next tile-start barrier, so no named barrier is left waiting for threads that have gone.
    for (int i = 0; i < n_my; ++i) {
      const int jt = t_begin + grp + 2 * i;
      // block index of every key of this tile, and whether the whole tile is visible to the whole query tile
      {
        const int key = jt * KT + gtid;
        int rel = kNoKey;
        if (key < n_keys_eff) {
          const int kb = div_blk(p.key_pos ? p.key_pos[(int64_t)b * p.n_keys + key] : key, p.blk_magic, p.blk_shift);
          rel = max(-32768, min(32766, kb - qblk_min));   // the queries' relative blocks lie in [0, 128]
        }
        bar.kblk[grp][i & 1][gtid] = (short)rel;
        const unsigned bal = __ballot_sync(0xffffffffu, rel <= 0);
        if (lane == 0) bar.vis_w[grp][i & 1][gtid >> 5] = bal;
      }
      if (bar_sync_or(1 + grp, 128, !ok || *abort_flag)) { ok = false; break; }
      const unsigned* vw = bar.vis_w[grp][i & 1];
      const bool fast = (vw[0] & vw[1] & vw[2] & vw[3]) == 0xffffffffu;
      const short* kbt = bar.kblk[grp][i & 1];
      if (!wait_bar(&bar.s_full[grp], i & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) ok = false;
      tc::fence_after_sync();
      // the row of S (one TMEM round trip), then the maximum of its visible scores
      float sv[128];
      tmem_ld128(tSg, sv);
      float mt = -INFINITY;
      if (fast) {
#pragma unroll
        for (int u = 0; u < 128; ++u) mt = fmaxf(mt, sv[u]);
      } else {
#pragma unroll
        for (int u = 0; u < 128; ++u)
          if (kbt[u] <= qrel) mt = fmaxf(mt, sv[u]);
      }
      mt *= p.scale_log2;
      // the reference maximum moves only when this tile's maximum exceeds it by more than 2^8
      float alpha = 1.f;
      if (mt > mg + kRescaleLog2) {
        alpha = (mg == -INFINITY) ? 1.f : ex2(mg - mt);
        mg = mt;
      }
      // P = 2^(s * scale - mg) as bf16 pairs, 64 keys at a time, written over the S columns already read; the
      // row sum adds the fp32 values (the bf16 rounding of P is unbiased and below 2^-9 per term)
      uint64_t rs2 = pk2(0.f, 0.f);
      const uint64_t negm2 = pk2(-mg, -mg);
      const bool any = mg != -INFINITY;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float* v = sv + 64 * c;
        uint32_t pk[32];
        if (fast) {     // every key visible: the tile maximum is finite, so mg is too
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            float x0, x1;
            upk2(fma2(pk2(v[2 * c2], v[2 * c2 + 1]), scale2, negm2), x0, x1);
            const float e0 = ex2(x0), e1 = ex2(x1);
            __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
            pk[c2] = *reinterpret_cast<uint32_t*>(&pr);
            rs2 = add2(rs2, pk2(e0, e1));
          }
        } else {
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            float x0, x1;
            upk2(fma2(pk2(v[2 * c2], v[2 * c2 + 1]), scale2, negm2), x0, x1);
            float e0 = ex2(x0), e1 = ex2(x1);
            if (!any || !(kbt[64 * c + 2 * c2] <= qrel)) e0 = 0.f;
            if (!any || !(kbt[64 * c + 2 * c2 + 1] <= qrel)) e1 = 0.f;
            __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
            pk[c2] = *reinterpret_cast<uint32_t*>(&pr);
            rs2 = add2(rs2, pk2(e0, e1));
          }
        }
        // keys [64c, 64c + 64) -> columns [32c, 32c + 32) (S has been read into registers)
        tc::tmem_st32(tSg + 32 * c, pk);
      }
      // O_g holds the group's previous P V once that phase completes (every phase is waited in order, so the
      // parity is unambiguous: the next phase needs this group's P)
      if (i > 0 && !wait_bar(&bar.o_full[grp], (i - 1) & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) ok = false;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float w[32];
          tmem_ld32(tOg + 32 * c, w);
          uint32_t r32[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) r32[u] = __float_as_uint(w[u] * alpha);
          tc::tmem_st32(tOg + 32 * c, r32);
        }
      }
      float rs0, rs1;
      upk2(rs2, rs0, rs1);
      l = l * alpha + (rs0 + rs1);
      tc::tmem_st_wait();
      tc::fence_before_sync();
      tc::mbar_arrive(&bar.p_ready[grp]);
    }
    bool fin = ok && n_my > 0;
    if (fin) fin = wait_bar(&bar.o_full[grp], (n_my - 1) & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE);
    // combine the groups: (m, l) through the K ring, idle once both groups' last P V have completed (every S
    // product was issued before one of them), O_0 and O_1 straight from TMEM
    tc::named_bar_sync(kBarAll, 256);
    float2* xch = reinterpret_cast<float2*>(sK);      // [group][row]
    xch[grp * 128 + row] = make_float2(fin ? mg : -INFINITY, fin ? l : 0.f);
    tc::named_bar_sync(kBarAll, 256);
    const float2 ma = xch[row], mb = xch[128 + row];
    const float M = fmaxf(ma.x, mb.x);
    const float wa = ma.x == -INFINITY ? 0.f : ex2(ma.x - M), wb = mb.x == -INFINITY ? 0.f : ex2(mb.x - M);
    l_row = wa * ma.y + wb * mb.y;
    m_ref = M;
#pragma unroll
    for (int u = 0; u < 64; ++u) o[u] = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < 2; ++g2) {
      const float w = g2 == 0 ? wa : wb;
      if (__any_sync(0xffffffffu, w != 0.f)) {       // tcgen05.ld is warp-wide
        tc::fence_after_sync();
        float x[64];
        tmem_ld64(tO + g2 * 128 + col0 + lane_off, x);
        if (w != 0.f) {
#pragma unroll
          for (int u = 0; u < 64; ++u) o[u] = fmaf(w, x[u], o[u]);
        }
      }
    }
    tc::fence_before_sync();
    if (p.n_splits == 1 && qg < p.Lq && !*abort_flag) {
      const int64_t qh = ((int64_t)b * p.Lq + qg) * p.Hq + g * p.G + row % p.G;
      const float inv = l_row > 0.f ? 1.0f / l_row : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.out + qh * 128 + col0);
#pragma unroll
      for (int c = 0; c < 64; c += 8) {
        __nv_bfloat162 a0 = __floats2bfloat162_rn(o[c] * inv, o[c + 1] * inv);
        __nv_bfloat162 a1 = __floats2bfloat162_rn(o[c + 2] * inv, o[c + 3] * inv);
        __nv_bfloat162 a2 = __floats2bfloat162_rn(o[c + 4] * inv, o[c + 5] * inv);
        __nv_bfloat162 a3 = __floats2bfloat162_rn(o[c + 6] * inv, o[c + 7] * inv);
        dst[c >> 3] = make_uint4(*reinterpret_cast<uint32_t*>(&a0), *reinterpret_cast<uint32_t*>(&a1),
                                 *reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&a3));
      }
    }
  }
  if (p.n_splits > 1) {
    // merge the splits of this query tile inside the cluster. Rank r owns rows [r*LR, (r+1)*LR). Once every CTA
    // of the cluster is done with its K/V ring (first cluster barrier), the threads of each row another rank owns
    // store their unnormalised row (o relative to their maximum, m, l) straight into the owner's ring through
    // distributed shared memory; after the second cluster barrier (release / acquire: the stores are visible) the
    // two threads of every owned row fold the other splits' copies into the row they hold in registers (splits in
    // order) and write the output.
    const int ns = p.n_splits;
    const int LR = (128 + ns - 1) / ns;
    const int r0 = split * LR, n_loc = max(0, min(128, r0 + LR) - r0);
    float* pbuf = reinterpret_cast<float*>(sK);                   // [ns][LR][kRecvStride]: the others' copies
    const bool mine = row >= r0 && row < r0 + n_loc;
    cluster_arrive();
    cluster_wait();
    if (warp >= 2 && !mine && !*abort_flag) {
      const int owner = row / LR, lr = row - owner * LR;
      const uint32_t dst =
          tc::mapa_u32(tc::smem_u32(pbuf + ((size_t)split * LR + lr) * kRecvStride + col0), (uint32_t)owner);
#pragma unroll
      for (int c = 0; c < 64; c += 4)
        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + c * 4), "f"(o[c]),
                     "f"(o[c + 1]), "f"(o[c + 2]), "f"(o[c + 3])
                     : "memory");
      if (grp == 0)
        asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(dst + (128 - col0) * 4), "f"(m_ref),
                     "f"(l_row)
                     : "memory");
    }
    cluster_arrive();
    cluster_wait();
    if (warp >= 2) {
      const int qg = q0 + row / p.G;
      if (mine && qg < p.Lq && !*abort_flag) {
        const int lr = row - r0;
        float M = m_ref;
        for (int sp = 0; sp < ns; ++sp)
          if (sp != split) M = fmaxf(M, pbuf[((size_t)sp * LR + lr) * kRecvStride + 128]);
        const float ws0 = m_ref == -INFINITY ? 0.f : ex2(m_ref - M);
        float L = ws0 * l_row;
#pragma unroll
        for (int u = 0; u < 64; ++u) o[u] *= ws0;
        for (int sp = 0; sp < ns; ++sp) {
          if (sp == split) continue;
          const float* rp = pbuf + ((size_t)sp * LR + lr) * kRecvStride;
          const float ms = rp[128];
          if (ms == -INFINITY) continue;
          const float w = ex2(ms - M);
          L += w * rp[129];
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(rp + col0 + c);
            o[c] = fmaf(w, v4.x, o[c]);
            o[c + 1] = fmaf(w, v4.y, o[c + 1]);
            o[c + 2] = fmaf(w, v4.z, o[c + 2]);
            o[c + 3] = fmaf(w, v4.w, o[c + 3]);
          }
        }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        const int64_t qh = ((int64_t)b * p.Lq + qg) * p.Hq + g * p.G + row % p.G;
        uint4* dst = reinterpret_cast<uint4*>(p.out + qh * 128 + col0);
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          __nv_bfloat162 a0 = __floats2bfloat162_rn(o[c] * inv, o[c + 1] * inv);
          __nv_bfloat162 a1 = __floats2bfloat162_rn(o[c + 2] * inv, o[c + 3] * inv);
          __nv_bfloat162 a2 = __floats2bfloat162_rn(o[c + 4] * inv, o[c + 5] * inv);
          __nv_bfloat162 a3 = __floats2bfloat162_rn(o[c + 6] * inv, o[c + 7] * inv);
          dst[c >> 3] = make_uint4(*reinterpret_cast<uint32_t*>(&a0), *reinterpret_cast<uint32_t*>(&a1),
                                   *reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&a3));
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(bar.tmem_base, 512);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
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

int encode(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
           const cuuint32_t* box) {
  EncodeTiledFn enc = encoder();
  if (!enc) {
    dllm_host::set_error("cuTensorMapEncodeTiled unavailable");
    return DLLM_ERR_CUDA;
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    dllm_host::set_error("attention: cuTensorMapEncodeTiled failed (%d)", (int)r);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

cudaError_t configure_attn() {
  static cudaError_t st = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  return st;
}

// How many clusters of ns CTAs can be resident at once (a cluster must fit inside one GPC); cached per size.
int max_active_clusters(int ns) {
  static int cache[9] = {0};
  if (ns < 1 || ns > 8) return 0;
  if (cache[ns] > 0) return cache[ns];
  int n = 0;
  if (configure_attn() == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ns, 1, 1);
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ns;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) != cudaSuccess) n = 0;
  }
  if (n <= 0) {
    cudaGetLastError();
    n = num_sms() / (2 * ns);
  }
  cache[ns] = std::max(n, 1);
  return cache[ns];
}

void plan_tc(int B, int Lq, int Hq, int Hkv, int n_keys, int& QT, int& n_qtiles, int& n_splits, int& tps) {
  const int G = Hq / Hkv;
  QT = 128 / G;
  n_qtiles = (Lq + QT - 1) / QT;
  const int tiles = (n_keys + KT - 1) / KT;
  const int base = B * Hkv * n_qtiles;
  // key splits fill at most one wave of the GPU (one CTA per SM): a second wave would repeat every split's
  // fixed cost (setup, first loads, merge) for a sliver of the keys
  const int want = num_sms() / base;
  n_splits = max(1, min(min(want, tiles), 8));
  while (n_splits > 1 && base > max_active_clusters(n_splits)) --n_splits;
  tps = (tiles + n_splits - 1) / n_splits;
  n_splits = max(1, (tiles + tps - 1) / tps);
}

}  // namespace

bool attn_tc_supported(int dtype, int Hq, int Hkv, int d) {
  if (dtype != DLLM_BF16 || d != 128 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G >= 1 && G <= 128 && (128 % G) == 0;
}

size_t attn_tc_workspace_bytes(int, int, int, int, int) {
  return 0;   // the key splits merge through distributed shared memory
}

int launch_attn_tc(const AttnArgs& a, int32_t* status, cudaStream_t s) {
  DLLM_REQUIRE(((uintptr_t)a.q % 16 == 0) && ((uintptr_t)a.k % 16 == 0) && ((uintptr_t)a.v % 16 == 0),
               DLLM_ERR_ALIGN, "attention: q, k, v must be 16-byte aligned");
  AttnTcParams p;
  p.B = a.B; p.Lq = a.Lq; p.Hq = a.Hq; p.Hkv = a.Hkv; p.G = a.Hq / a.Hkv; p.n_keys = a.n_keys; p.cap = a.cap;
  p.blk_len = a.blk_len; p.q_pos0 = a.q_pos0;
  {
    uint32_t sh = 0;
    while ((1u << sh) < (uint32_t)a.blk_len) ++sh;                     // 2^(sh-1) < blk_len <= 2^sh
    p.blk_magic = (uint32_t)((((uint64_t)1 << (31 + sh)) + (uint64_t)a.blk_len - 1) / (uint64_t)a.blk_len);
    p.blk_shift = 31 + sh;
  }
  plan_tc(a.B, a.Lq, a.Hq, a.Hkv, a.n_keys, p.QT, p.n_qtiles, p.n_splits, p.tiles_per_split);
  const float scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)a.d);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.key_pos = a.key_pos;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.status = status;
  p.live = a.live;
  CUtensorMap mq, mk, mv;
  {
    cuuint64_t dims[4] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.Lq, (cuuint64_t)a.B};
    cuuint64_t str[3] = {128 * 2, (cuuint64_t)a.Hq * 128 * 2, (cuuint64_t)a.Lq * a.Hq * 128 * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)p.G, (cuuint32_t)p.QT, 1};
    int st = encode(&mq, a.q, 4, dims, str, box);
    if (st) return st;
  }
  {
    // [B*Hkv][n_keys][128]: rows past n_keys of a (row, kv head) read as zeros, never as another row's keys
    cuuint64_t dims[3] = {128, (cuuint64_t)a.n_keys, (cuuint64_t)a.B * a.Hkv};
    cuuint64_t str[2] = {128 * 2, (cuuint64_t)a.cap * 128 * 2};
    cuuint32_t box[3] = {64, KT, 1};
    int st = encode(&mk, a.k, 3, dims, str, box);
    if (st) return st;
    st = encode(&mv, a.v, 3, dims, str, box);
    if (st) return st;
  }
  {
    cudaError_t e = configure_attn();
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaFuncSetAttribute(attn_tc)");
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, a.B * a.Hkv * p.n_qtiles, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.n_splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel, mq, mk, mv, p);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaLaunchKernelEx(attn_tc_kernel)");
  DLLM_CHECK_LAUNCH("attn_tc_kernel");
  return DLLM_OK;
}

}  // namespace dllm
