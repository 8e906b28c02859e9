// Block-causal attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16, head dim 128.
// Source: LLaDA2.0-Uni paper review, sections "Block Diffusion Language Model (BDLM)" (bidirectional inside a
// block, left-to-right across blocks) and "MoE 백본과 Block-wise Attention".
//
// One CTA per (batch row, kv head, tile of queries, key split). The 128-row M tile packs the G = Hq / Hkv query
// heads that share the kv head with 128 / G queries (row r = query r / G, head r % G), so every K/V tile staged in
// shared memory serves the whole group. Per 128-key tile:
//   S = Q K^T      tcgen05.mma M=128 N=128 K=128 (Q, K K-major, TMA 128-byte swizzled) -> TMEM (double buffered)
//   softmax        4 warps, one TMEM lane (query row) per thread: mask, scale, online max/sum, P = exp2(...) as
//                  bf16 written to shared memory in the swizzled K-major layout
//   O_t = P V      tcgen05.mma M=128 N=128 K=128 (P K-major, V MN-major straight from the [key][d] cache) -> TMEM
//   o += O_t       accumulated in fp32 registers with the online-softmax rescale.
// Warp 0 issues TMA (Q once; K and V tiles through a 2-stage ring), warp 1 issues the MMAs from one thread,
// warps 2..5 run the softmax and write the output (or per-split partials merged by log-sum-exp).
// Every mbarrier wait is bounded; on expiry the kernel records a status word and leaves.
#include "common.cuh"
#include "tc.cuh"
#include "misc.h"
#include <cuda.h>
#include <mutex>

namespace dllm {
namespace {

constexpr int NT = 320;                     // warp 0 TMA, warp 1 MMA, warps 2..9 softmax (two per query row)
constexpr int KT = 128;                     // keys per tile
constexpr int CHUNK = 128 * 64 * 2;         // one 64-wide K-major chunk of a 128-row tile: 16 KB
constexpr int TILE = 2 * CHUNK;             // 128 rows x 128 elements: 32 KB
constexpr int STAGES = 2;
constexpr int BARS_BYTES = 2048;
constexpr short kNoKey = 0x7fff;   // relative block of a key past n_keys (never visible)
constexpr int SMEM = 1024 + TILE /*Q*/ + STAGES * 2 * TILE /*K,V*/ + 2 * TILE /*P, double buffered*/ + BARS_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[STAGES];
  uint64_t kv_empty[STAGES];
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t o_full[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  short kblk[2][KT];    // block of each key of the tile relative to the CTA's first query block, clamped to
                        // [-32768, 32766] (kNoKey past n_keys), per tile parity
  unsigned vis_w[2][4]; // per tile, ballots of "key visible to every query of the CTA" (4 warps x 32 keys)
  float rowmax[2][128]; // per column half, per row: the half-row maximum (the tile-start barrier separates uses)
};
static_assert(sizeof(Bars) <= BARS_BYTES, "barrier block exceeds its shared-memory reservation");

struct AttnTcParams {
  int B, Lq, Hq, Hkv, G, QT, n_qtiles, n_keys, cap, blk_len, q_pos0;
  int n_splits, tiles_per_split;
  float scale_log2;
  const int32_t* key_pos;
  __nv_bfloat16* out;   // [B, Lq, Hq, 128]
  int32_t* status;
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

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(tc::smem_u32(local)), "r"(rank));
  return remote;
}
__device__ __forceinline__ float ld_dsmem(const float* local, uint32_t rank) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(dsmem_addr(local, rank)) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_dsmem4(const float* local, uint32_t rank) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(dsmem_addr(local, rank))
               : "memory");
  return v;
}

// Each lane reads 64 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  tmem_ld32(taddr, v);
  tmem_ld32(taddr + 32, v + 32);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(NT, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const AttnTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + TILE;                    // [STAGES][TILE]
  uint8_t* sV = sK + STAGES * TILE;           // [STAGES][TILE]
  uint8_t* sP = sV + STAGES * TILE;            // [2][TILE]
  Bars& bar = *reinterpret_cast<Bars*>(sP + 2 * TILE);

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
    tc::mbar_init(&bar.s_full[0], 1);
    tc::mbar_init(&bar.s_full[1], 1);
    tc::mbar_init(&bar.p_ready, 256);
    tc::mbar_init(&bar.o_full[0], 1);
    tc::mbar_init(&bar.o_full[1], 1);
    tc::mbar_init(&bar.done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&bar.tmem_base, 512);
  __syncthreads();
  volatile int* abort_flag = &bar.abort_flag;
  const uint32_t tS = bar.tmem_base;          // S buffers at columns [0,128) and [128,256)
  const uint32_t tO = bar.tmem_base + 256;    // O tiles at columns [256,384) and [384,512)

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
      const uint32_t aQ = tc::smem_u32(sQ), aP = tc::smem_u32(sP);
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
      for (int j = 0; j < ntile && ok; ++j) {
        if (j + 1 < ntile && !issue_s(j + 1)) { ok = false; break; }
        // P_j written (and O tile of j-1 read) by the softmax warps
        if (!wait_bar(&bar.p_ready, j & 1, abort_flag, p.status, ST_TIMEOUT_MMA)) { ok = false; break; }
        tc::fence_after_sync();
        const int s = j % STAGES;
        const uint32_t aV = tc::smem_u32(sV + s * TILE);
        const uint32_t aPj = aP + (j & 1) * TILE;
        const uint32_t tOj = tO + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offp = (kk >> 2) * CHUNK + (kk & 3) * 32;
          tc::mma_bf16(tOj, tc::sdesc_k128(aPj + offp), sdesc_mn128(aV + kk * 2048, CHUNK), idesc_o, kk != 0);
        }
        tc::mma_commit(&bar.o_full[j & 1]);
        tc::mma_commit(&bar.kv_empty[s]);
      }
      tc::mma_commit(&bar.done);
      tc::mbar_wait(&bar.done, 0, 1u << 20);
    }
  } else {
    // ------------------------------------------------------------------ softmax / output warps 2..9
    // Two threads per query row (TMEM lane): warp w in 2..5 takes keys / output columns [0, 64), warp w + 4 takes
    // [64, 128). The half-row maxima are exchanged through shared memory once per tile.
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;      // TMEM lane = tile row
    const int half = (warp - 2) >> 2;    // 0: columns [0, 64), 1: [64, 128)
    const int etid = tid - 64;           // 0..255
    const int qi = row / p.G, hh = row % p.G;
    const int qg = q0 + qi;              // query index in the row
    const bool row_ok = qg < p.Lq;
    const int qblk_min = (p.q_pos0 + q0) / p.blk_len;  // rows of the tile past Lq never write output
    const int qrel = (p.q_pos0 + qg) / p.blk_len - qblk_min;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int col0 = 64 * half;
    float o[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) o[c] = 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntile && ok; ++j) {
      const int jt = t_begin + j;
      // block index of every key of this tile, and whether the whole tile is visible to the whole query tile
      if (etid < 128) {
        const int key = jt * KT + etid;
        int rel = kNoKey;
        if (key < n_keys_eff) {
          const int kb = (p.key_pos ? p.key_pos[(int64_t)b * p.n_keys + key] : key) / p.blk_len;
          rel = max(-32768, min(32766, kb - qblk_min));   // the queries' relative blocks lie in [0, 128]
        }
        bar.kblk[j & 1][etid] = (short)rel;
        const unsigned bal = __ballot_sync(0xffffffffu, rel <= 0);
        if (lane == 0) bar.vis_w[j & 1][etid >> 5] = bal;
      }
      tc::named_bar_sync(1, 256);
      const bool fast = (bar.vis_w[j & 1][0] & bar.vis_w[j & 1][1] & bar.vis_w[j & 1][2] & bar.vis_w[j & 1][3]) ==
                        0xffffffffu;
      if (!wait_bar(&bar.s_full[j & 1], (j >> 1) & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t sbase = tS + (j & 1) * 128 + col0 + lane_off;
      const short* kbt = bar.kblk[j & 1] + col0;
      float v[64];
      tmem_ld64(sbase, v);
      // pass 1: half-row maximum of the visible scores, exchanged with the partner thread
      float mt = -INFINITY;
      if (fast) {
#pragma unroll
        for (int u = 0; u < 64; ++u) mt = fmaxf(mt, v[u]);
      } else {
#pragma unroll
        for (int u = 0; u < 64; ++u)
          if (kbt[u] <= qrel) mt = fmaxf(mt, v[u]);
      }
      bar.rowmax[half][row] = mt;
      tc::named_bar_sync(2, 256);
      mt = fmaxf(bar.rowmax[0][row], bar.rowmax[1][row]) * p.scale_log2;
      const float m_new = fmaxf(m, mt);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
      // pass 2: P = exp2(s - m_new) as bf16 into this half's chunk of the tile's swizzled K-major P buffer
      uint8_t* sPj = sP + (j & 1) * TILE + half * CHUNK;
      float rs = 0.f;
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        uint32_t packed[4];
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {
          float pv[2];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int c = u8 * 8 + h2 * 2 + e2;
            const bool vis = (fast || kbt[c] <= qrel) && m_new != -INFINITY;
            pv[e2] = vis ? exp2f(v[c] * p.scale_log2 - m_new) : 0.f;
          }
          __nv_bfloat162 pr = __floats2bfloat162_rn(pv[0], pv[1]);
          rs += __bfloat162float(pr.x) + __bfloat162float(pr.y);
          packed[h2] = *reinterpret_cast<uint32_t*>(&pr);
        }
        uint8_t* dst = sPj + row * 128 + ((u8 ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&bar.p_ready);
      // fold in the previous tile's P V (previous max's scale), then move to this tile's scale
      if (j > 0) {
        if (!wait_bar(&bar.o_full[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        float w[64];
        tmem_ld64(tO + ((j - 1) & 1) * 128 + col0 + lane_off, w);
#pragma unroll
        for (int u = 0; u < 64; ++u) o[u] += w[u];
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] *= alpha;
      l = l * alpha + rs;          // this half's share of the row sum
      m = m_new;
    }
    if (ok && ntile > 0) {
      const int jl = ntile - 1;
      if (wait_bar(&bar.o_full[jl & 1], (jl >> 1) & 1, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) {
        tc::fence_after_sync();
        float w[64];
        tmem_ld64(tO + (jl & 1) * 128 + col0 + lane_off, w);
#pragma unroll
        for (int u = 0; u < 64; ++u) o[u] += w[u];
      }
    }
    // row sums: the two halves' shares
    float* lsum = &bar.rowmax[0][0];             // reused: [2][128]
    tc::named_bar_sync(1, 256);
    lsum[half * 128 + row] = l;
    tc::named_bar_sync(1, 256);
    const float l_row = lsum[row] + lsum[128 + row];
    if (p.n_splits == 1) {
      if (row_ok && !*abort_flag) {
        const int64_t qh = ((int64_t)b * p.Lq + qg) * p.Hq + g * p.G + hh;
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
    } else {
      // this split's unnormalised row (log2-domain max; an empty split leaves (-inf, 0)) into the idle K/V ring:
      // o at [row][128] with the 16-byte units rotated by the row to spread banks, then m and l
      float* so = reinterpret_cast<float*>(sK);
      float4* orow = reinterpret_cast<float4*>(so + row * 128);
#pragma unroll
      for (int c = 0; c < 64; c += 4)
        orow[(((col0 + c) >> 2) + row) & 31] = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      if (half == 0) {
        so[128 * 128 + row] = m;
        so[128 * 128 + 128 + row] = l_row;
      }
    }
  }
  if (p.n_splits > 1) {
    // merge the splits of this tile: rank r owns rows [r*128/ns, (r+1)*128/ns); it reads every split's (o, m, l)
    // of its rows through distributed shared memory, in rank order
    __syncthreads();
    cluster_sync();
    if (warp >= 2 && !*abort_flag) {
      const int ns = p.n_splits;
      const int r0 = split * 128 / ns, r1 = (split + 1) * 128 / ns;
      const float* so = reinterpret_cast<const float*>(sK);
      const int etid = tid - 64;
      const int d4 = etid & 31;               // this thread's 4 output columns
      for (int rr = r0 + (etid >> 5); rr < r1; rr += 8) {
        const int qi = rr / p.G, hh2 = rr % p.G, qg = q0 + qi;
        float ms[8];
        float M = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < 8; ++sp) {
          ms[sp] = sp < ns ? ld_dsmem(so + 128 * 128 + rr, (uint32_t)sp) : -INFINITY;
          M = fmaxf(M, ms[sp]);
        }
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int sp = 0; sp < 8; ++sp) {
          const float w = (sp < ns && ms[sp] != -INFINITY) ? exp2f(ms[sp] - M) : 0.f;
          if (w != 0.f) {
            L += w * ld_dsmem(so + 128 * 128 + 128 + rr, (uint32_t)sp);
            const float4 v4 = ld_dsmem4(so + rr * 128 + (((d4 + rr) & 31) << 2), (uint32_t)sp);
            acc.x += w * v4.x;
            acc.y += w * v4.y;
            acc.z += w * v4.z;
            acc.w += w * v4.w;
          }
        }
        if (qg < p.Lq) {
          const float inv = L > 0.f ? 1.0f / L : 0.f;
          const int64_t qh = ((int64_t)b * p.Lq + qg) * p.Hq + g * p.G + hh2;
          __nv_bfloat162 a0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
          __nv_bfloat162 a1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
          uint2* dst = reinterpret_cast<uint2*>(p.out + qh * 128 + d4 * 4);
          *dst = make_uint2(*reinterpret_cast<uint32_t*>(&a0), *reinterpret_cast<uint32_t*>(&a1));
        }
      }
    }
    cluster_sync();
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

void plan_tc(int B, int Lq, int Hq, int Hkv, int n_keys, int& QT, int& n_qtiles, int& n_splits, int& tps) {
  const int G = Hq / Hkv;
  QT = 128 / G;
  n_qtiles = (Lq + QT - 1) / QT;
  const int tiles = (n_keys + KT - 1) / KT;
  const int base = B * Hkv * n_qtiles;
  int want = (3 * num_sms() / 2 + base - 1) / base;
  n_splits = max(1, min(min(want, tiles), 8));
  tps = (tiles + n_splits - 1) / n_splits;
  n_splits = max(1, (tiles + tps - 1) / tps);
}

}  // namespace

bool attn_tc_supported(int dtype, int Hq, int Hkv, int d) {
  if (dtype != DLLM_BF16 || d != 128 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G >= 1 && G <= 128 && (128 % G) == 0;
}

size_t attn_tc_workspace_bytes(int, int, int, int, int) { return 0; }  // splits merge on chip

int launch_attn_tc(const AttnArgs& a, int32_t* status, cudaStream_t s) {
  DLLM_REQUIRE(((uintptr_t)a.q % 16 == 0) && ((uintptr_t)a.k % 16 == 0) && ((uintptr_t)a.v % 16 == 0),
               DLLM_ERR_ALIGN, "attention: q, k, v must be 16-byte aligned");
  AttnTcParams p;
  p.B = a.B; p.Lq = a.Lq; p.Hq = a.Hq; p.Hkv = a.Hkv; p.G = a.Hq / a.Hkv; p.n_keys = a.n_keys; p.cap = a.cap;
  p.blk_len = a.blk_len; p.q_pos0 = a.q_pos0;
  plan_tc(a.B, a.Lq, a.Hq, a.Hkv, a.n_keys, p.QT, p.n_qtiles, p.n_splits, p.tiles_per_split);
  const float scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)a.d);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.key_pos = a.key_pos;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.status = status;
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
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaFuncSetAttribute(attn_tc)");
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, a.B * a.Hkv * p.n_qtiles, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.n_splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel, mq, mk, mv, p);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "cudaLaunchKernelEx(attn_tc_kernel)");
  DLLM_CHECK_LAUNCH("attn_tc_kernel");
  return DLLM_OK;
}

}  // namespace dllm
