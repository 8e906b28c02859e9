// C-ABI entry points: argument validation, workspace carving and the composition of one denoising pass.
// Every entry point validates before launching; nothing is launched on error. No entry point allocates device
// memory or synchronises, except dllm_status_check, which reads the workspace status word.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cmath>
#include "common.cuh"
#include "kernels.h"
#include "misc.h"
#include "tc.cuh"

#include <atomic>
#include <algorithm>
#include <cuda.h>
#include <mutex>
#include <vector>

namespace dllm_host {
static thread_local char g_err[512] = "";
static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}
int cuda_status(cudaError_t e, const char* what) {
  set_error("%s: %s", what, cudaGetErrorString(e));
  return DLLM_ERR_CUDA;
}
}  // namespace dllm_host

using namespace dllm;

namespace {

constexpr size_t kStatusBytes = 256;
// words of the status block past the status word: the expert GEMMs' work counters (own 64-byte lines)
constexpr int kWorkCtr1 = 16, kWorkCtr2 = 32;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int esize(int dtype) { return dtype == DLLM_BF16 ? 2 : 4; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Bump carver over a caller workspace (base == nullptr only measures).
struct Carver {
  char* base;
  size_t off = kStatusBytes;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T = void>
  T* take(size_t bytes) {
    off = align256(off);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += bytes;
    return p;
  }
};

#define REQ(cond, code, ...) DLLM_REQUIRE(cond, code, __VA_ARGS__)

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  REQ(ws != nullptr, DLLM_ERR_WORKSPACE, "workspace is NULL");
  REQ(((uintptr_t)ws & 255u) == 0, DLLM_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  REQ(ws_bytes >= need, DLLM_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return DLLM_OK;
}

int32_t* status_word(void* ws) { return static_cast<int32_t*>(ws); }

// ------------------------------------------------------------------------------------------------ GEMM dispatch
int run_gemm(GemmArgs& a, cudaStream_t s) {
  return a.dtype == DLLM_BF16 ? gemm_bf16_tc(a, s) : gemm_f32_simt(a, s);
}

// ------------------------------------------------------------------------------------------------ experts
struct ExpertBufs {
  void* xp;
  void* act;
  void* y;        // expert output rows in the storage type
  float* scratch;
};

void carve_experts(Carver& c, int dtype, int Tk, int H, int k, int I, int shared, ExpertBufs& b) {
  const int64_t rows = (int64_t)Tk * k + (shared ? Tk : 0);
  b.xp = c.take(rows * H * esize(dtype));
  b.act = c.take(rows * I * esize(dtype));
  b.y = c.take(rows * H * esize(dtype));
  b.scratch = dtype == DLLM_F32 ? c.take<float>(gemm_f32_scratch_bytes(rows, std::max(2 * I, H), 0)) : nullptr;
}

// N tile of the expert GEMMs (the host cannot see the routed counts): wide enough for four times the average rows
// per expert and at least 128, since a denoising block's masked positions share most of their routing (the block
// starts from one mask token), which piles many rows on a few experts; an expert with more rows than the N tile
// streams its weight tiles once per extra tile (measured: 128 instead of 64 took one understanding layer from 463
// to 449 us; random routing is unaffected).
int expert_bn_hint(int Tk, int k, int E) {
  const int avg = (Tk * k + E - 1) / E;
  return std::min(Tk, std::max(128, 4 * avg));
}

// The combine's follow-up RMSNorm, fused into it (PostNorm::g == nullptr: plain combine).
struct PostNorm {
  const void* g = nullptr;
  float eps = 0.f;
  void* out = nullptr;
  int mode = NORM_NEXT;
  const uint8_t* mask = nullptr;   // NORM_FINAL: block mask, positions per half, masked count
  int n_half_pos = 0;
  const int32_t* n_dev = nullptr;
};

// Row scales of FP8 expert weights (all NULL for weights in the storage type).
struct ExpertScales {
  const float* gu = nullptr;
  const float* down = nullptr;
  const float* gu_shared = nullptr;
  const float* down_shared = nullptr;
};

int run_experts(int dtype, int Tk, int H, int E, int k, int I, const void* h, const void* w_gu, const void* w_down,
                const void* w_gu_s, const void* w_down_s, const int32_t* counts, const int32_t* offsets,
                const int32_t* perm, const int32_t* inv, const float* gates, void* x, const ExpertBufs& b,
                int32_t* status, cudaStream_t s, const PostNorm& pn = PostNorm(), const int32_t* live = nullptr,
                const ExpertScales& sc = ExpertScales()) {
  const int fp8 = sc.gu != nullptr;
  const int shared = w_gu_s != nullptr;
  const int n_assign = Tk * k;
  const int64_t rows = (int64_t)n_assign + (shared ? Tk : 0);
  // the two GEMMs' work counters sit in the workspace's status block (the status word is its first word)
  unsigned* ctr1 = reinterpret_cast<unsigned*>(status) + kWorkCtr1;
  unsigned* ctr2 = reinterpret_cast<unsigned*>(status) + kWorkCtr2;
  int st = launch_gather_rows(dtype, h, perm, k, Tk, shared, b.xp, H, s, live, ctr1, ctr2);
  if (st) return st;
  GemmArgs g1;
  g1.x = b.xp; g1.x_rows = rows;
  g1.w = w_gu; g1.w_rows = (int64_t)E * 2 * I;
  g1.w2 = w_gu_s; g1.w2_rows = 2 * I;
  g1.K = H; g1.M = I; g1.swiglu = 1; g1.w_group_stride = 2 * I;
  g1.n_dev = E; g1.grp_off = offsets; g1.grp_cnt = counts;
  g1.has_extra = shared; g1.extra_off = n_assign; g1.extra_cnt = Tk;
  g1.max_cnt = expert_bn_hint(Tk, k, E); g1.cnt_bound = Tk;
  g1.dtype = dtype; g1.status = status; g1.f32_scratch = b.scratch; g1.live = live; g1.work_ctr = ctr1;
  g1.w_fp8 = fp8; g1.w_scale = sc.gu; g1.w2_scale = sc.gu_shared;
  g1.epi.kind = EPI_SWIGLU; g1.epi.out = b.act; g1.epi.ldo = I;
  st = run_gemm(g1, s);
  if (st) return st;
  GemmArgs g2 = g1;
  g2.x = b.act; g2.K = I; g2.M = H; g2.swiglu = 0;
  g2.w = w_down; g2.w_rows = (int64_t)E * H; g2.w2 = w_down_s; g2.w2_rows = H; g2.w_group_stride = H;
  g2.w_scale = sc.down; g2.w2_scale = sc.down_shared; g2.work_ctr = ctr2;
  g2.epi = EpiParams();
  g2.epi.kind = EPI_STORE; g2.epi.out = b.y; g2.epi.ldo = H; g2.epi.out_f32 = dtype == DLLM_F32;
  st = run_gemm(g2, s);
  if (st) return st;
  if (pn.g)
    return launch_combine_norm(dtype, x, b.y, gates, inv, k, Tk, shared, H, pn.g, pn.eps, pn.out, pn.mode, pn.mask,
                               pn.n_half_pos, pn.n_dev, s, live);
  return launch_combine(dtype, x, b.y, gates, inv, k, Tk, shared, H, s, live);
}

// Rows the fused row kernels handle: 16-byte vectors, at most kRowVecs of them per thread of a 256-thread CTA.
static bool fused_rows_ok(int dtype, int H) {
  const int ve = dtype == DLLM_BF16 ? 8 : 4;
  return H % ve == 0 && H / ve <= kRowVecs * 256;
}

// ------------------------------------------------------------------------------------------------ step plan
struct StepPlan {
  int B, L, Bl, halves, Tk, vlen, n_keys, max_rows, n_chunks;
  void* x;
  void* h;
  void* q;
  void* ao;
  void* attn_ws;
  size_t attn_ws_bytes;
  float* scores;
  int32_t* ids;
  float* gates;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  int32_t* route_seg;
  ExpertBufs eb;
  float* proj_scratch;
  int32_t* row_pos;
  int32_t* n_rows;
  void* xf;
  void* logits;
  void* partials;
  int conf_parts;   // > 0: the LM head writes this many confidence partials per row (fused epilogue)
  float2* rope_tab;  // [L][64] RoPE (cos, sin) of the block's positions (tensor-core QKV epilogue)
  void* unmask_extras;   // the other position scores' statistics (null for the largest probability)
  float* retain_raw;
  size_t total;
};

int validate_step(const dllm_model* m, const dllm_state* st, const dllm_step_params* p) {
  REQ(m && st && p, DLLM_ERR_INVALID_ARG, "denoise_step: NULL descriptor");
  REQ(m->dtype == DLLM_BF16 || m->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "denoise_step: bad dtype %d", m->dtype);
  REQ(m->n_layers >= 1 && m->layers, DLLM_ERR_INVALID_ARG, "denoise_step: no layers");
  REQ(m->H > 0 && m->Hq > 0 && m->Hkv > 0 && m->d > 0 && m->E > 0 && m->k > 0 && m->I > 0 && m->V > 0,
      DLLM_ERR_SHAPE, "denoise_step: non-positive model dimension");
  REQ(m->Hq % m->Hkv == 0, DLLM_ERR_SHAPE, "denoise_step: Hq %% Hkv != 0");
  REQ(m->k <= m->E && m->k <= 32 && m->E <= 1024, DLLM_ERR_UNSUPPORTED, "denoise_step: k/E out of range");
  REQ(m->H % 8 == 0, DLLM_ERR_SHAPE, "denoise_step: H must be a multiple of 8");
  REQ((size_t)16 * m->H * (m->dtype == DLLM_BF16 ? 2 : 4) <= 200 * 1024, DLLM_ERR_UNSUPPORTED,
      "denoise_step: H too large for the router");
  REQ(st->B >= 1 && st->B <= 1024 && st->L >= 1 && st->L <= 32 && st->P >= 0, DLLM_ERR_SHAPE,
      "denoise_step: bad B/L/P (B <= 1024, L <= 32)");
  REQ(st->cap >= st->P + st->L, DLLM_ERR_SHAPE, "denoise_step: cap %d < P + L", st->cap);
  REQ(st->tokens && st->mask, DLLM_ERR_INVALID_ARG, "denoise_step: NULL tokens/mask");
  REQ(m->embed && m->final_norm && m->w_lm, DLLM_ERR_INVALID_ARG, "denoise_step: NULL embed/final_norm/w_lm");
  REQ(p->T_s >= 1 && p->t >= 0 && p->t < p->T_s, DLLM_ERR_INVALID_ARG, "denoise_step: step %d of %d", p->t, p->T_s);
  REQ(p->mode == DLLM_UNMASK_FIXED || p->mode == DLLM_UNMASK_THRESHOLD, DLLM_ERR_INVALID_ARG, "bad unmask mode");
  REQ(p->score >= DLLM_SCORE_LOW_CONFIDENCE && p->score <= DLLM_SCORE_NEG_ENTROPY, DLLM_ERR_INVALID_ARG,
      "denoise_step: bad score %d", p->score);
  REQ(p->cfg >= 0 && p->cfg <= 2, DLLM_ERR_INVALID_ARG, "denoise_step: cfg %d (0, 1 or 2)", p->cfg);
  REQ(st->B % (1 + p->cfg) == 0, DLLM_ERR_SHAPE, "denoise_step: cfg %d needs B a multiple of %d", p->cfg, 1 + p->cfg);
  REQ(p->cfg != 2 || !p->sprint, DLLM_ERR_UNSUPPORTED,
      "denoise_step: SPRINT with editing guidance (cfg 2) is not supported; run those blocks on the full caches");
  const int vlen = p->vocab_len ? p->vocab_len : m->V;
  REQ(p->vocab_offset >= 0 && p->vocab_offset + vlen <= m->V, DLLM_ERR_SHAPE, "denoise_step: vocab slice out of range");
  if (p->sprint) {
    REQ(p->n_keep >= 1 && p->n_keep <= st->P && p->n_keep <= 8192, DLLM_ERR_SHAPE, "denoise_step: bad n_keep");
    REQ(p->sprint_alpha >= 0.f && p->sprint_alpha <= 1.f, DLLM_ERR_INVALID_ARG, "denoise_step: sprint_alpha in [0, 1]");
    REQ(p->sprint_alpha == 1.f || st->prefix_conf, DLLM_ERR_INVALID_ARG,
        "denoise_step: sprint_alpha < 1 needs state->prefix_conf");
    REQ(!st->prefix_modality || (p->n_keep_img >= 0 && p->n_keep_img <= p->n_keep), DLLM_ERR_INVALID_ARG,
        "denoise_step: n_keep_img must be in [0, n_keep]");
    REQ(st->cap_thin >= p->n_keep + st->L, DLLM_ERR_SHAPE, "denoise_step: cap_thin too small");
    REQ(st->P <= 8192, DLLM_ERR_UNSUPPORTED, "denoise_step: SPRINT needs P <= 8192");
  }
  if (!p->commit) REQ(p->sel && p->nsel && p->conf && p->remaining, DLLM_ERR_INVALID_ARG, "denoise_step: NULL outputs");
  for (int l = 0; l < m->n_layers; ++l) {
    const dllm_layer& L = m->layers[l];
    REQ(L.attn_norm && L.w_qkv && L.w_o && L.ffn_norm && L.w_router && L.router_bias && L.w_gu && L.w_down &&
            L.k_cache && L.v_cache,
        DLLM_ERR_INVALID_ARG, "denoise_step: layer %d has a NULL weight or cache", l);
    REQ((L.w_gu_shared == nullptr) == (L.w_down_shared == nullptr), DLLM_ERR_INVALID_ARG,
        "denoise_step: layer %d: shared expert weights must both be set or both NULL", l);
    if (p->sprint) REQ(L.k_thin && L.v_thin && L.keep_pos, DLLM_ERR_INVALID_ARG, "layer %d: NULL thinned cache", l);
    if (m->dtype == DLLM_BF16)
      REQ(aligned16(L.w_qkv) && aligned16(L.w_o) && aligned16(L.w_gu) && aligned16(L.w_down), DLLM_ERR_ALIGN,
          "layer %d: weights must be 16-byte aligned", l);
  }
  REQ(m->weight_format == DLLM_WEIGHTS_BF16 || m->weight_format == DLLM_WEIGHTS_FP8, DLLM_ERR_INVALID_ARG,
      "denoise_step: bad weight_format %d", m->weight_format);
  if (m->weight_format == DLLM_WEIGHTS_FP8) {
    REQ(m->dtype == DLLM_BF16, DLLM_ERR_UNSUPPORTED, "denoise_step: FP8 weights need bf16 storage");
    REQ(m->w_lm_scale, DLLM_ERR_INVALID_ARG, "denoise_step: FP8 weights need w_lm_scale");
    REQ(m->H % 128 == 0 && m->I % 128 == 0, DLLM_ERR_UNSUPPORTED,
        "denoise_step: FP8 weights need H and I multiples of 128");
    for (int l = 0; l < m->n_layers; ++l) {
      const dllm_layer& L = m->layers[l];
      REQ(L.w_gu_scale && L.w_down_scale && (!L.w_gu_shared || (L.w_gu_shared_scale && L.w_down_shared_scale)),
          DLLM_ERR_INVALID_ARG, "denoise_step: layer %d: FP8 expert weights need their row scales", l);
    }
  }
  if (m->dtype == DLLM_BF16) {
    REQ(m->d == 128, DLLM_ERR_UNSUPPORTED, "denoise_step: bf16 path needs head dim 128");
    REQ(m->H % 128 == 0 && m->I % 64 == 0, DLLM_ERR_UNSUPPORTED, "denoise_step: bf16 path needs H %% 128 == 0, I %% 64 == 0");
    REQ(vlen % 128 == 0, DLLM_ERR_UNSUPPORTED, "denoise_step: scored vocabulary must be a multiple of 128");
    REQ(aligned16(m->w_lm) && aligned16(m->embed), DLLM_ERR_ALIGN, "denoise_step: LM head / embedding alignment");
    for (int l = 0; l < m->n_layers; ++l) {   // the QKV epilogue writes 16-byte vectors into the caches
      const dllm_layer& L = m->layers[l];
      REQ(aligned16(L.k_cache) && aligned16(L.v_cache) && (!p->sprint || (aligned16(L.k_thin) && aligned16(L.v_thin))),
          DLLM_ERR_ALIGN, "layer %d: KV caches must be 16-byte aligned", l);
    }
  } else {
    REQ(m->d <= 128 && m->d % 4 == 0, DLLM_ERR_UNSUPPORTED, "denoise_step: fp32 path needs d <= 128, d %% 4 == 0");
  }
  return DLLM_OK;
}

void plan_step(const dllm_model* m, const dllm_state* st, const dllm_step_params* p, void* ws, StepPlan& s) {
  Carver c(ws);
  const int es = esize(m->dtype);
  s.B = st->B;
  s.L = st->L;
  s.halves = 1 + p->cfg;   // row groups: (cond), (cond, uncond) or (cond, image only, uncond)
  s.Bl = st->B / s.halves;
  s.Tk = st->B * st->L;
  s.vlen = p->vocab_len ? p->vocab_len : m->V;
  s.n_keys = p->sprint ? p->n_keep + st->L : st->P + st->L;
  s.max_rows = s.Bl * st->L;
  s.n_chunks = unmask_chunks(s.max_rows, s.vlen);
  s.conf_parts = 0;
  if (m->dtype == DLLM_BF16 && !p->cfg && p->score == DLLM_SCORE_LOW_CONFIDENCE) {
    GemmArgs g;   // the LM head's shape (see the step below)
    g.dtype = DLLM_BF16; g.K = m->H; g.M = s.vlen; g.host_cnt = s.max_rows; g.max_cnt = s.max_rows;
    g.cnt_bound = s.max_rows; g.epi.kind = EPI_STORE; g.w_fp8 = m->weight_format == DLLM_WEIGHTS_FP8;
    s.conf_parts = gemm_conf_parts(g);
  }
  const int H = m->H, QD = m->Hq * m->d;
  s.x = c.take((size_t)s.Tk * H * es);
  s.h = c.take((size_t)s.Tk * H * es);
  s.q = c.take((size_t)s.Tk * QD * es);
  s.ao = c.take((size_t)s.Tk * QD * es);
  s.attn_ws_bytes = attn_workspace_bytes(st->B, st->L, m->Hq, m->Hkv, m->d, s.n_keys, m->dtype);
  s.attn_ws = c.take(s.attn_ws_bytes);
  s.scores = c.take<float>((size_t)s.Tk * m->E * 4);
  s.ids = c.take<int32_t>((size_t)s.Tk * m->k * 4);
  s.gates = c.take<float>((size_t)s.Tk * m->k * 4);
  s.counts = c.take<int32_t>((size_t)m->n_layers * (m->E + 1) * 4);   // one histogram per layer (kept for views)
  s.offsets = c.take<int32_t>((size_t)(m->E + 1) * 4);
  s.perm = c.take<int32_t>((size_t)s.Tk * m->k * 4);
  s.inv = c.take<int32_t>((size_t)s.Tk * m->k * 4);
  s.route_seg = c.take<int32_t>(route_scratch_bytes(s.Tk, m->E, m->k));
  carve_experts(c, m->dtype, s.Tk, H, m->k, m->I, 1, s.eb);
  const int proj_n = (m->Hq + 2 * m->Hkv) * m->d;
  s.proj_scratch = m->dtype == DLLM_F32
                       ? c.take<float>((size_t)std::max(s.Tk, s.halves * s.max_rows) *
                                       std::max(std::max(proj_n, H), s.vlen) * 4)
                       : nullptr;
  s.rope_tab = m->dtype == DLLM_BF16 ? c.take<float2>((size_t)st->L * 64 * sizeof(float2)) : nullptr;
  s.row_pos = c.take<int32_t>((size_t)s.max_rows * 4);
  s.n_rows = c.take<int32_t>(16);
  s.xf = c.take((size_t)s.halves * s.max_rows * H * es);
  s.logits = c.take((size_t)s.halves * s.max_rows * s.vlen * es);
  s.partials = c.take(unmask_partials_bytes(s.max_rows, std::max(s.n_chunks, s.conf_parts)));
  {
    const size_t exb = unmask_extras_bytes(p->score, s.max_rows, s.n_chunks, s.Bl, st->L);
    s.unmask_extras = exb ? c.take(exb) : nullptr;
  }
  s.retain_raw = p->sprint ? c.take<float>(retain_workspace_bytes(st->B, st->P)) : nullptr;
  s.total = align256(c.off);
}

}  // namespace

// A kernel that waits on an mbarrier nothing ever arrives at, with the same bounded poll loop as the tensor-core
// kernels (a short bound here), then records the timeout in the status word and returns.
__global__ void selftest_wait_kernel(int32_t* status, uint32_t max_polls) {
  dllm::pdl_enter();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    dllm::tc::mbar_init(&bar, 1);
    dllm::tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !dllm::tc::mbar_wait(&bar, 0, max_polls)) atomicExch(status, dllm::ST_TIMEOUT_MMA);
}

// ================================================================================================== ABI
extern "C" {

int dllm_selftest_bounded_wait(void* ws, size_t ws_bytes, cudaStream_t stream) {
  int st = check_ws(ws, ws_bytes, kStatusBytes);
  if (st) return st;
  dllm::launch_pdl(selftest_wait_kernel, 1, 32, 0, stream, status_word(ws), 1u << 12);
  DLLM_CHECK_LAUNCH("selftest_wait_kernel");
  return DLLM_OK;
}

const char* dllm_version(void) { return "dllm-b200 0.1 (sm_100a)"; }
const char* dllm_last_error(void) { return dllm_host::g_err; }
unsigned long long dllm_launch_count(void) { return dllm_host::g_launches.load(std::memory_order_relaxed); }

int dllm_status_check(void* ws, cudaStream_t stream) {
  REQ(ws != nullptr, DLLM_ERR_WORKSPACE, "status_check: NULL workspace");
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "status_check");
  if (h != 0) {
    int32_t zero = 0;
    cudaMemcpyAsync(ws, &zero, sizeof(int32_t), cudaMemcpyHostToDevice, stream);
    cudaStreamSynchronize(stream);
    dllm_host::set_error("a kernel gave up on a bounded wait (code %d)", h);
    return DLLM_ERR_TIMEOUT;
  }
  return DLLM_OK;
}

// ------------------------------------------------------------------------------------------------ dense GEMM
size_t dllm_gemm_workspace_size(const dllm_gemm_desc* d) {
  if (!d) return 0;
  size_t n = kStatusBytes;
  if (d->dtype == DLLM_F32) n = align256(n) + gemm_f32_scratch_bytes(d->N, d->M, 0);
  return align256(n);
}

int dllm_gemm(const dllm_gemm_desc* d, const void* x, const void* w, const float* w_scale, void* y,
              const int32_t* n_rows_dev, void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && x && w && y, DLLM_ERR_INVALID_ARG, "gemm: NULL argument");
  REQ(d->N >= 0 && d->M > 0 && d->K > 0 && d->ldy >= d->M, DLLM_ERR_SHAPE, "gemm: bad N/M/K/ldy");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "gemm: bad dtype");
  if (d->w_fp8) {
    REQ(d->dtype == DLLM_BF16 && !d->residual, DLLM_ERR_UNSUPPORTED, "gemm: FP8 weights need bf16 storage, no residual");
    REQ(w_scale != nullptr, DLLM_ERR_INVALID_ARG, "gemm: FP8 weights need w_scale");
  }
  int st = check_ws(ws, ws_bytes, dllm_gemm_workspace_size(d));
  if (st) return st;
  if (d->N == 0) return DLLM_OK;
  if (d->dtype == DLLM_BF16) {
    REQ(d->K % 64 == 0 && d->M % 128 == 0, DLLM_ERR_UNSUPPORTED, "gemm: bf16 needs K %% 64 == 0 and M %% 128 == 0");
    REQ(aligned16(x) && aligned16(w), DLLM_ERR_ALIGN, "gemm: X and W must be 16-byte aligned");
    // the epilogue writes 16-byte vectors of 8 (bf16) or 4 (fp32) outputs
    REQ(aligned16(y) && d->ldy % (d->y_f32 ? 4 : 8) == 0, DLLM_ERR_ALIGN,
        "gemm: Y must be 16-byte aligned with ldy a multiple of %d", d->y_f32 ? 4 : 8);
  }
  Carver c(ws);
  GemmArgs a;
  a.x = x; a.x_rows = d->N; a.w = w; a.w_rows = d->M; a.K = d->K; a.M = d->M;
  a.cnt_dev = n_rows_dev; a.host_cnt = d->N; a.max_cnt = d->N; a.cnt_bound = d->N;
  a.dtype = d->dtype; a.status = status_word(ws);
  a.w_fp8 = d->w_fp8; a.w_scale = d->w_fp8 ? w_scale : nullptr;
  a.f32_scratch = d->dtype == DLLM_F32 ? c.take<float>(gemm_f32_scratch_bytes(d->N, d->M, 0)) : nullptr;
  a.epi.kind = d->residual ? EPI_RESID : EPI_STORE;
  a.epi.out = y; a.epi.ldo = d->ldy; a.epi.out_f32 = d->y_f32 || d->dtype == DLLM_F32;
  return run_gemm(a, stream);
}

// ------------------------------------------------------------------------------------------------ grouped GEMM
size_t dllm_grouped_gemm_workspace_size(const dllm_grouped_gemm_desc* d) {
  if (!d) return 0;
  return align256(kStatusBytes);
}

int dllm_grouped_gemm(const dllm_grouped_gemm_desc* d, const void* x, const void* w, const void* w_extra,
                      const float* w_scale, const float* w_extra_scale, const int32_t* counts,
                      const int32_t* offsets, void* y, void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && x && w && counts && offsets && y, DLLM_ERR_INVALID_ARG, "grouped_gemm: NULL argument");
  REQ(d->G >= 1 && d->G <= 4096 && d->rows >= 0 && d->K > 0 && d->M > 0 && d->extra_rows >= 0 &&
          d->extra_rows <= d->rows,
      DLLM_ERR_SHAPE, "grouped_gemm: bad G/rows/K/M/extra_rows");
  REQ((w_extra != nullptr) == (d->extra_rows > 0), DLLM_ERR_INVALID_ARG,
      "grouped_gemm: w_extra must be given exactly when extra_rows > 0");
  REQ(d->dtype == DLLM_BF16, DLLM_ERR_UNSUPPORTED, "grouped_gemm: bf16 only");
  REQ(d->K % 64 == 0 && (d->swiglu ? d->M % 64 == 0 : d->M % 128 == 0), DLLM_ERR_UNSUPPORTED,
      "grouped_gemm: needs K %% 64 == 0 and M %% 128 == 0 (swiglu: M %% 64 == 0)");
  REQ(!(d->swiglu && d->y_f32), DLLM_ERR_UNSUPPORTED, "grouped_gemm: swiglu output is in the storage type");
  REQ(!d->w_fp8 || (w_scale && (!w_extra || w_extra_scale)), DLLM_ERR_INVALID_ARG,
      "grouped_gemm: FP8 weights need their row scales");
  REQ(aligned16(x) && aligned16(w) && (!w_extra || aligned16(w_extra)) && aligned16(y), DLLM_ERR_ALIGN,
      "grouped_gemm: X, W, W_extra and Y must be 16-byte aligned");
  int st = check_ws(ws, ws_bytes, dllm_grouped_gemm_workspace_size(d));
  if (st) return st;
  if (d->rows == 0) return DLLM_OK;
  const int Mw = d->swiglu ? 2 * d->M : d->M;
  GemmArgs a;
  a.x = x; a.x_rows = d->rows;
  a.w = w; a.w_rows = (int64_t)d->G * Mw; a.w2 = w_extra; a.w2_rows = w_extra ? Mw : 0;
  a.K = d->K; a.M = d->M; a.swiglu = d->swiglu; a.w_group_stride = Mw;
  a.n_dev = d->G; a.grp_off = offsets; a.grp_cnt = counts;
  a.has_extra = w_extra != nullptr; a.extra_off = d->rows - d->extra_rows; a.extra_cnt = d->extra_rows;
  a.max_cnt = std::max(1, std::min(d->max_rows_hint > 0 ? d->max_rows_hint : d->rows, d->rows));
  a.cnt_bound = d->rows; a.dtype = DLLM_BF16; a.status = status_word(ws);
  a.w_fp8 = d->w_fp8; a.w_scale = d->w_fp8 ? w_scale : nullptr; a.w2_scale = d->w_fp8 ? w_extra_scale : nullptr;
  a.epi.kind = d->swiglu ? EPI_SWIGLU : EPI_STORE; a.epi.out = y; a.epi.ldo = d->M; a.epi.out_f32 = d->y_f32;
  return run_gemm(a, stream);
}

// ------------------------------------------------------------------------------------------------ attention
size_t dllm_block_attn_workspace_size(const dllm_attn_desc* d) {
  if (!d) return 0;
  return align256(align256(kStatusBytes) + attn_workspace_bytes(d->B, d->Lq, d->Hq, d->Hkv, d->d, d->n_keys, d->dtype));
}

int dllm_block_attn(const dllm_attn_desc* d, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* key_pos, void* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && q && k_cache && v_cache && out, DLLM_ERR_INVALID_ARG, "block_attn: NULL argument");
  REQ(d->B >= 1 && d->Lq >= 1 && d->Hq >= 1 && d->Hkv >= 1 && d->d >= 1 && d->blk_len >= 1 && d->n_keys >= 1 &&
          d->q_pos0 >= 0,
      DLLM_ERR_SHAPE, "block_attn: non-positive dimension");
  REQ(d->Hq % d->Hkv == 0 && d->Hq / d->Hkv <= 64, DLLM_ERR_SHAPE, "block_attn: Hq must be a multiple of Hkv (group <= 64)");
  REQ(d->cap >= d->n_keys, DLLM_ERR_SHAPE, "block_attn: cap < n_keys");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "block_attn: bad dtype");
  REQ(d->dtype == DLLM_BF16 ? d->d == 128 : (d->d <= 128 && d->d % 4 == 0), DLLM_ERR_UNSUPPORTED,
      "block_attn: unsupported head dim %d", d->d);
  int st = check_ws(ws, ws_bytes, dllm_block_attn_workspace_size(d));
  if (st) return st;
  Carver c(ws);
  AttnArgs a;
  a.B = d->B; a.Lq = d->Lq; a.Hq = d->Hq; a.Hkv = d->Hkv; a.d = d->d; a.blk_len = d->blk_len; a.q_pos0 = d->q_pos0;
  a.n_keys = d->n_keys; a.cap = d->cap; a.dtype = d->dtype; a.scale = d->scale;
  a.q = q; a.k = k_cache; a.v = v_cache; a.key_pos = key_pos; a.out = out;
  a.ws_bytes = attn_workspace_bytes(d->B, d->Lq, d->Hq, d->Hkv, d->d, d->n_keys, d->dtype);
  a.ws = c.take(a.ws_bytes);
  return launch_attn(a, status_word(ws), stream);
}

// ------------------------------------------------------------------------------------------------ SPRINT
size_t dllm_prefix_retain_workspace_size(const dllm_retain_desc* d) {
  if (!d) return 0;
  return align256(align256(kStatusBytes) + retain_workspace_bytes(d->B, d->P));
}

int dllm_prefix_retain(const dllm_retain_desc* d, const void* k_cache, const void* v_cache, const float* conf,
                       const uint8_t* modality, int32_t* keep_pos, void* k_thin, void* v_thin, float* scores,
                       void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && k_cache && v_cache && keep_pos && k_thin && v_thin, DLLM_ERR_INVALID_ARG, "prefix_retain: NULL argument");
  REQ(d->B >= 1 && d->Hkv >= 1 && d->d >= 1 && d->P >= 1 && d->cap >= d->P, DLLM_ERR_SHAPE, "prefix_retain: bad shape");
  REQ(d->n_keep >= 1 && d->n_keep <= d->P && d->n_keep <= d->cap_thin, DLLM_ERR_SHAPE, "prefix_retain: bad n_keep");
  REQ(d->P <= 8192, DLLM_ERR_UNSUPPORTED, "prefix_retain: P > 8192");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "prefix_retain: bad dtype");
  REQ((d->d * esize(d->dtype)) % 16 == 0, DLLM_ERR_UNSUPPORTED, "prefix_retain: row bytes must be a multiple of 16");
  REQ(d->alpha >= 0.f && d->alpha <= 1.f, DLLM_ERR_INVALID_ARG, "prefix_retain: alpha must be in [0, 1]");
  REQ(!modality || (d->n_keep_img >= 0 && d->n_keep_img <= d->n_keep), DLLM_ERR_INVALID_ARG,
      "prefix_retain: n_keep_img must be in [0, n_keep]");
  int st = check_ws(ws, ws_bytes, dllm_prefix_retain_workspace_size(d));
  if (st) return st;
  Carver c(ws);
  RetainArgs a;
  a.B = d->B; a.Hkv = d->Hkv; a.d = d->d; a.P = d->P; a.cap = d->cap; a.n_keep = d->n_keep; a.cap_thin = d->cap_thin;
  a.dtype = d->dtype; a.k = k_cache; a.v = v_cache; a.keep_pos = keep_pos; a.k_thin = k_thin; a.v_thin = v_thin;
  a.scores = scores; a.raw = c.take<float>(retain_workspace_bytes(d->B, d->P)); a.block_len = 0;
  a.conf = conf; a.conf_stride = d->P; a.alpha = conf ? d->alpha : 1.f; a.modality = modality;
  a.n_keep_img = d->n_keep_img;
  return launch_retain(a, stream);
}

// ------------------------------------------------------------------------------------------------ router
size_t dllm_moe_route_workspace_size(const dllm_route_desc* d) {
  if (!d) return 0;
  return align256(align256(align256(kStatusBytes) + (size_t)d->Tk * d->E * 4) + route_scratch_bytes(d->Tk, d->E, d->k));
}

int dllm_moe_route(const dllm_route_desc* d, const void* h, const void* w_router, const float* bias, int32_t* ids,
                   float* gates, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, float* scores,
                   void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && h && w_router && bias && ids && gates && counts && offsets && perm && inv, DLLM_ERR_INVALID_ARG,
      "moe_route: NULL argument");
  REQ(d->Tk >= 0 && d->H > 0 && d->E >= 1 && d->k >= 1, DLLM_ERR_SHAPE, "moe_route: bad shape");
  REQ(d->E <= 1024 && d->k <= 32 && d->k <= d->E, DLLM_ERR_UNSUPPORTED, "moe_route: needs E <= 1024, k <= min(32, E)");
  REQ(d->H % 8 == 0, DLLM_ERR_SHAPE, "moe_route: H must be a multiple of 8");
  REQ((size_t)16 * d->H * (d->dtype == DLLM_BF16 ? 2 : 4) <= 200 * 1024, DLLM_ERR_UNSUPPORTED, "moe_route: H too large");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "moe_route: bad dtype");
  REQ(aligned16(h) && aligned16(w_router), DLLM_ERR_ALIGN, "moe_route: h and w_router must be 16-byte aligned");
  REQ(scores == nullptr || aligned16(scores), DLLM_ERR_ALIGN, "moe_route: scores must be 16-byte aligned");
  int st = check_ws(ws, ws_bytes, dllm_moe_route_workspace_size(d));
  if (st) return st;
  Carver c(ws);
  float* sc = c.take<float>((size_t)d->Tk * d->E * 4);
  if (scores) sc = scores;
  int32_t* seg = c.take<int32_t>(route_scratch_bytes(d->Tk, d->E, d->k));
  return launch_route(d->dtype, h, w_router, bias, d->Tk, d->H, d->E, d->k, ids, gates, sc, counts, offsets, perm,
                      inv, seg, stream);
}

// ------------------------------------------------------------------------------------------------ experts
size_t dllm_moe_experts_workspace_size(const dllm_expert_desc* d) {
  if (!d) return 0;
  Carver c(nullptr);
  ExpertBufs b;
  carve_experts(c, d->dtype, d->Tk, d->H, d->k, d->I, 1, b);
  return align256(c.off);
}

int dllm_moe_experts(const dllm_expert_desc* d, const void* h, const void* w_gu, const void* w_down,
                     const void* w_gu_shared, const void* w_down_shared, const float* w_gu_scale,
                     const float* w_down_scale, const float* w_gu_shared_scale, const float* w_down_shared_scale,
                     const int32_t* counts, const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                     const float* gates, void* x_inout, void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && h && w_gu && w_down && counts && offsets && perm && inv && gates && x_inout, DLLM_ERR_INVALID_ARG,
      "moe_experts: NULL argument");
  REQ((w_gu_shared == nullptr) == (w_down_shared == nullptr), DLLM_ERR_INVALID_ARG,
      "moe_experts: shared expert weights must both be set or both NULL");
  REQ(d->Tk >= 0 && d->H > 0 && d->E >= 1 && d->k >= 1 && d->k <= d->E && d->I > 0, DLLM_ERR_SHAPE,
      "moe_experts: bad shape");
  REQ(d->E <= 1024 && d->k <= 32, DLLM_ERR_UNSUPPORTED, "moe_experts: needs E <= 1024, k <= 32");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "moe_experts: bad dtype");
  REQ((d->H * esize(d->dtype)) % 16 == 0, DLLM_ERR_SHAPE, "moe_experts: H row bytes must be a multiple of 16");
  if (d->w_fp8) {
    REQ(d->dtype == DLLM_BF16, DLLM_ERR_UNSUPPORTED, "moe_experts: FP8 weights need bf16 storage");
    REQ(d->H % 128 == 0 && d->I % 128 == 0, DLLM_ERR_UNSUPPORTED, "moe_experts: FP8 weights need H, I multiples of 128");
    REQ(w_gu_scale && w_down_scale && (!w_gu_shared || (w_gu_shared_scale && w_down_shared_scale)),
        DLLM_ERR_INVALID_ARG, "moe_experts: FP8 weights need their row scales");
  }
  if (d->dtype == DLLM_BF16) {
    REQ(d->H % 128 == 0 && d->I % 64 == 0, DLLM_ERR_UNSUPPORTED, "moe_experts: bf16 needs H %% 128 == 0, I %% 64 == 0");
    REQ(aligned16(h) && aligned16(w_gu) && aligned16(w_down) && (!w_gu_shared || (aligned16(w_gu_shared) && aligned16(w_down_shared))),
        DLLM_ERR_ALIGN, "moe_experts: operands must be 16-byte aligned");
  }
  int st = check_ws(ws, ws_bytes, dllm_moe_experts_workspace_size(d));
  if (st) return st;
  if (d->Tk == 0) return DLLM_OK;
  Carver c(ws);
  ExpertBufs b;
  carve_experts(c, d->dtype, d->Tk, d->H, d->k, d->I, 1, b);
  ExpertScales esc;
  if (d->w_fp8) {
    esc.gu = w_gu_scale; esc.down = w_down_scale; esc.gu_shared = w_gu_shared_scale; esc.down_shared = w_down_shared_scale;
  }
  return run_experts(d->dtype, d->Tk, d->H, d->E, d->k, d->I, h, w_gu, w_down, w_gu_shared, w_down_shared, counts,
                     offsets, perm, inv, gates, x_inout, b, status_word(ws), stream, PostNorm(), nullptr, esc);
}

// ------------------------------------------------------------------------------------------------ unmask
size_t dllm_unmask_workspace_size(const dllm_unmask_desc* d) {
  if (!d) return 0;
  const int nc = unmask_chunks(d->max_rows, d->V);
  return align256(align256(align256(kStatusBytes) + unmask_partials_bytes(d->max_rows, nc)) +
                  unmask_extras_bytes(d->score, d->max_rows, nc, d->B, d->L));
}

int dllm_unmask(const dllm_unmask_desc* d, const void* logits, const int32_t* row_pos, const int32_t* n_rows_dev,
                int32_t* tokens, uint8_t* mask, int32_t* sel, int32_t* nsel, float* conf, int32_t* remaining,
                void* ws, size_t ws_bytes, cudaStream_t stream) {
  REQ(d && logits && row_pos && n_rows_dev && tokens && mask && sel && nsel && conf && remaining,
      DLLM_ERR_INVALID_ARG, "unmask: NULL argument");
  REQ(d->B >= 1 && d->B <= 1024 && d->L >= 1 && d->L <= 32 && d->V >= 1 && d->max_rows >= 0 &&
          d->max_rows <= d->B * d->L,
      DLLM_ERR_SHAPE, "unmask: bad shape (B <= 1024, L <= 32, max_rows <= B*L)");
  REQ(d->T_s >= 1 && d->t >= 0 && d->t < d->T_s, DLLM_ERR_INVALID_ARG, "unmask: step %d of %d", d->t, d->T_s);
  REQ(d->mode == DLLM_UNMASK_FIXED || d->mode == DLLM_UNMASK_THRESHOLD, DLLM_ERR_INVALID_ARG, "unmask: bad mode");
  REQ(d->mode == DLLM_UNMASK_FIXED || d->k_max >= 1, DLLM_ERR_INVALID_ARG, "unmask: k_max must be >= 1");
  REQ(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "unmask: bad dtype");
  REQ(d->vocab_offset >= 0, DLLM_ERR_INVALID_ARG, "unmask: negative vocab_offset");
  REQ(d->cfg >= 0 && d->cfg <= 2, DLLM_ERR_INVALID_ARG, "unmask: cfg %d (0, 1 or 2)", d->cfg);
  REQ(d->score >= DLLM_SCORE_LOW_CONFIDENCE && d->score <= DLLM_SCORE_NEG_ENTROPY, DLLM_ERR_INVALID_ARG,
      "unmask: bad score %d", d->score);
  int st = check_ws(ws, ws_bytes, dllm_unmask_workspace_size(d));
  if (st) return st;
  Carver c(ws);
  UnmaskArgs a;
  a.B = d->B; a.L = d->L; a.V = d->V; a.max_rows = d->max_rows; a.t = d->t; a.T_s = d->T_s; a.mode = d->mode;
  a.k_max = d->k_max; a.cfg = d->cfg; a.vocab_offset = d->vocab_offset; a.dtype = d->dtype; a.tau = d->tau;
  a.cfg_scale = d->cfg_scale; a.cfg_image_scale = d->cfg_image_scale; a.logits = logits; a.row_pos = row_pos; a.n_rows = n_rows_dev; a.tokens = tokens;
  a.mask = mask; a.sel = sel; a.nsel = nsel; a.conf = conf; a.remaining = remaining;
  a.n_chunks = unmask_chunks(d->max_rows, d->V);
  a.partials = c.take(unmask_partials_bytes(d->max_rows, a.n_chunks));
  a.score = d->score;
  const size_t exb = unmask_extras_bytes(d->score, d->max_rows, a.n_chunks, d->B, d->L);
  a.extras = exb ? c.take(exb) : nullptr;
  return launch_unmask(a, stream);
}

// ------------------------------------------------------------------------------------------------ step
size_t dllm_denoise_step_workspace_size(const dllm_model* m, const dllm_state* st, const dllm_step_params* p) {
  if (validate_step(m, st, p) != DLLM_OK) return 0;
  StepPlan s;
  plan_step(m, st, p, nullptr, s);
  return s.total;
}

int dllm_denoise_step_views(const dllm_model* m, const dllm_state* st, const dllm_step_params* p, void* ws,
                            size_t ws_bytes, dllm_step_views* v) {
  int r = validate_step(m, st, p);
  if (r) return r;
  REQ(v != nullptr, DLLM_ERR_INVALID_ARG, "denoise_step_views: NULL views");
  StepPlan s;
  plan_step(m, st, p, nullptr, s);
  r = check_ws(ws, ws_bytes, s.total);
  if (r) return r;
  plan_step(m, st, p, ws, s);
  v->logits = s.logits;
  v->row_pos = s.row_pos;
  v->n_rows = s.n_rows;
  v->x_final = s.x;
  v->expert_counts = s.counts;
  v->live = s.n_rows + 2;
  return DLLM_OK;
}

}  // extern "C"

namespace {
// One pass; with set_cond the unmask selection also sets the graph condition `cond` to (masked positions left > 0).
int denoise_step_impl(const dllm_model* m, const dllm_state* st, const dllm_step_params* p, void* ws,
                      size_t ws_bytes, cudaStream_t stream, cudaGraphConditionalHandle cond, int set_cond) {
  int r = validate_step(m, st, p);
  if (r) return r;
  StepPlan s;
  plan_step(m, st, p, nullptr, s);
  r = check_ws(ws, ws_bytes, s.total);
  if (r) return r;
  plan_step(m, st, p, ws, s);
  const int dt = m->dtype, H = m->H, QD = m->Hq * m->d, es = esize(dt);
  const int P = st->P, L = st->L;
  int32_t* status = status_word(ws);
#define TRY(x)            \
  do {                    \
    int _r = (x);         \
    if (_r) return _r;    \
  } while (0)

  // live word of a denoising pass (written by the masked-row list below): once the block has no masked position
  // left, every later kernel of the pass returns at once, so extra passes of a finished block cost only their
  // launches. A commit pass always runs.
  const int32_t* live = p->commit ? nullptr : s.n_rows + 2;
  const bool fuse = fused_rows_ok(dt, H);
  RopeTable rope;   // the block's RoPE angles, for the tensor-core QKV epilogue
  rope.tab = s.rope_tab; rope.pos0 = P; rope.L = L; rope.base = m->rope_base;
  if (fuse) {
    // embedding, layer 0's attention-input norm, (denoising passes) the masked-row list and the RoPE table in one
    // launch
    TRY(launch_embed_norm(dt, st->tokens, p->commit ? nullptr : st->mask, m->mask_id, m->embed, s.x, s.h,
                          m->layers[0].attn_norm, s.Tk, H, m->eps, st->mask, s.Bl * L, s.halves,
                          p->commit ? nullptr : s.row_pos, s.n_rows, stream, rope));
  } else {
    if (!p->commit) TRY(launch_masked_rows(st->mask, s.Bl * L, s.halves, s.row_pos, s.n_rows, stream));
    TRY(launch_embed(dt, st->tokens, p->commit ? nullptr : st->mask, m->mask_id, m->embed, s.x, s.Tk, H, stream));
    TRY(launch_rope_table(rope, stream));
  }
  for (int l = 0; l < m->n_layers; ++l) {
    const dllm_layer& Ly = m->layers[l];
    const bool last = l == m->n_layers - 1;
    // the attention-input norm comes fused with the embedding (layer 0) or the previous layer's combine
    if (!fuse) TRY(launch_rmsnorm(dt, s.x, Ly.attn_norm, s.h, s.Tk, H, m->eps, nullptr, nullptr, 0, 0, stream));
    if (p->sprint && p->retain) {
      RetainArgs ra;
      ra.B = st->B; ra.Hkv = m->Hkv; ra.d = m->d; ra.P = P; ra.cap = st->cap; ra.n_keep = p->n_keep;
      ra.cap_thin = st->cap_thin; ra.dtype = dt; ra.k = Ly.k_cache; ra.v = Ly.v_cache; ra.keep_pos = Ly.keep_pos;
      ra.k_thin = Ly.k_thin; ra.v_thin = Ly.v_thin; ra.scores = nullptr; ra.raw = s.retain_raw; ra.block_len = L;
      ra.conf = p->sprint_alpha < 1.f ? st->prefix_conf : nullptr; ra.conf_stride = st->cap;
      ra.alpha = p->sprint_alpha; ra.modality = st->prefix_modality; ra.n_keep_img = p->n_keep_img;
      TRY(launch_retain(ra, stream));
    }
    // QKV projection + RoPE; block K/V into the cache the attention reads (and the full cache on commit)
    GemmArgs g;
    g.x = s.h; g.x_rows = s.Tk; g.w = Ly.w_qkv; g.w_rows = (int64_t)(m->Hq + 2 * m->Hkv) * m->d; g.K = H;
    g.M = (m->Hq + 2 * m->Hkv) * m->d; g.host_cnt = s.Tk; g.max_cnt = s.Tk; g.cnt_bound = s.Tk; g.dtype = dt;
    g.status = status; g.f32_scratch = s.proj_scratch; g.live = live;
    g.epi.kind = EPI_QKV; g.epi.q_out = s.q; g.epi.Hq = m->Hq; g.epi.Hkv = m->Hkv; g.epi.d = m->d; g.epi.L = L;
    g.epi.pos0 = P; g.epi.rope_base = m->rope_base; g.epi.rope_tab = s.rope_tab;
    if (p->sprint) {
      g.epi.k_dst = Ly.k_thin; g.epi.v_dst = Ly.v_thin; g.epi.cap = st->cap_thin; g.epi.slot0 = p->n_keep;
      if (p->commit) { g.epi.k_dst2 = Ly.k_cache; g.epi.v_dst2 = Ly.v_cache; g.epi.cap2 = st->cap; g.epi.slot2 = P; }
    } else {
      g.epi.k_dst = Ly.k_cache; g.epi.v_dst = Ly.v_cache; g.epi.cap = st->cap; g.epi.slot0 = P;
    }
    TRY(run_gemm(g, stream));
    // block attention
    AttnArgs aa;
    aa.B = st->B; aa.Lq = L; aa.Hq = m->Hq; aa.Hkv = m->Hkv; aa.d = m->d; aa.blk_len = L; aa.q_pos0 = P;
    aa.n_keys = s.n_keys; aa.cap = p->sprint ? st->cap_thin : st->cap; aa.dtype = dt; aa.scale = 0.f;
    aa.q = s.q; aa.k = p->sprint ? Ly.k_thin : Ly.k_cache; aa.v = p->sprint ? Ly.v_thin : Ly.v_cache;
    aa.key_pos = p->sprint ? Ly.keep_pos : nullptr; aa.out = s.ao; aa.ws = s.attn_ws; aa.ws_bytes = s.attn_ws_bytes;
    aa.live = live;
    TRY(launch_attn(aa, status, stream));
    // output projection + residual
    GemmArgs go;
    go.x = s.ao; go.x_rows = s.Tk; go.w = Ly.w_o; go.w_rows = H; go.K = QD; go.M = H; go.host_cnt = s.Tk;
    go.max_cnt = s.Tk; go.cnt_bound = s.Tk; go.dtype = dt; go.status = status; go.f32_scratch = s.proj_scratch;
    go.live = live;
    go.epi.kind = EPI_RESID; go.epi.out = s.x; go.epi.ldo = H; go.epi.out_f32 = dt == DLLM_F32;
    TRY(run_gemm(go, stream));
    if (p->commit && last) break;  // the last layer's FFN output has no consumer in a commit pass
    // MoE FFN
    TRY(launch_rmsnorm(dt, s.x, Ly.ffn_norm, s.h, s.Tk, H, m->eps, nullptr, nullptr, 0, 0, stream));
    int32_t* counts = s.counts + (size_t)l * (m->E + 1);
    TRY(launch_route(dt, s.h, Ly.w_router, Ly.router_bias, s.Tk, H, m->E, m->k, s.ids, s.gates, s.scores, counts,
                     s.offsets, s.perm, s.inv, s.route_seg, stream, live));
    PostNorm pn;
    if (fuse && !last) {           // next layer's attention-input norm
      pn.g = m->layers[l + 1].attn_norm; pn.eps = m->eps; pn.out = s.h; pn.mode = NORM_NEXT;
    } else if (fuse && !p->commit) {   // final norm of the still-masked rows, in the LM head's row order
      pn.g = m->final_norm; pn.eps = m->eps; pn.out = s.xf; pn.mode = NORM_FINAL; pn.mask = st->mask;
      pn.n_half_pos = s.Bl * L; pn.n_dev = s.n_rows;
    }
    ExpertScales esc;
    if (m->weight_format == DLLM_WEIGHTS_FP8) {
      esc.gu = Ly.w_gu_scale; esc.down = Ly.w_down_scale;
      esc.gu_shared = Ly.w_gu_shared_scale; esc.down_shared = Ly.w_down_shared_scale;
    }
    TRY(run_experts(dt, s.Tk, H, m->E, m->k, m->I, s.h, Ly.w_gu, Ly.w_down, Ly.w_gu_shared, Ly.w_down_shared,
                    counts, s.offsets, s.perm, s.inv, s.gates, s.x, s.eb, status, stream, pn, live, esc));
  }
  if (p->commit) return DLLM_OK;
  // final norm on the masked rows (one group after the other) unless fused above, LM head, confidence + unmasking
  if (!fuse)
    TRY(launch_rmsnorm(dt, s.x, m->final_norm, s.xf, s.halves * s.max_rows, H, m->eps, s.row_pos, s.n_rows,
                       s.halves, s.Bl * L, stream));
  GemmArgs gl;
  gl.x = s.xf; gl.x_rows = (int64_t)s.halves * s.max_rows;
  const bool lm_fp8 = m->weight_format == DLLM_WEIGHTS_FP8;
  gl.w = static_cast<const char*>(m->w_lm) + (size_t)p->vocab_offset * H * (lm_fp8 ? 1 : es); gl.w_rows = s.vlen;
  gl.w_fp8 = lm_fp8;
  gl.w_scale = lm_fp8 ? m->w_lm_scale + p->vocab_offset : nullptr;
  gl.K = H; gl.M = s.vlen; gl.cnt_dev = s.n_rows + 1; gl.host_cnt = s.halves * s.max_rows;
  gl.max_cnt = s.halves * s.max_rows; gl.cnt_bound = s.halves * s.max_rows; gl.dtype = dt; gl.status = status;
  gl.f32_scratch = s.proj_scratch;
  gl.epi.kind = EPI_STORE; gl.epi.out = s.logits; gl.epi.ldo = s.vlen; gl.epi.out_f32 = dt == DLLM_F32;
  if (s.conf_parts) {   // confidence partials from the LM head's epilogue: no separate reduction pass
    gl.epi.conf_part = static_cast<ConfPartial*>(s.partials);
    gl.epi.conf_nparts = s.conf_parts;
  }
  TRY(run_gemm(gl, stream));
  UnmaskArgs ua;
  ua.B = s.Bl; ua.L = L; ua.V = s.vlen; ua.max_rows = s.max_rows; ua.t = p->t; ua.T_s = p->T_s; ua.mode = p->mode;
  ua.k_max = p->k_max; ua.cfg = p->cfg; ua.vocab_offset = p->vocab_offset; ua.dtype = dt; ua.tau = p->tau;
  ua.cfg_scale = p->cfg_scale; ua.cfg_image_scale = p->cfg_image_scale; ua.logits = s.logits; ua.row_pos = s.row_pos;
  ua.n_rows = s.n_rows;
  ua.tokens = st->tokens; ua.mask = st->mask; ua.sel = p->sel; ua.nsel = p->nsel; ua.conf = p->conf;
  ua.remaining = p->remaining; ua.partials = s.partials;
  ua.n_chunks = s.conf_parts ? s.conf_parts : s.n_chunks;
  ua.partials_ready = s.conf_parts ? 1 : 0;
  ua.cond = cond;
  ua.set_cond = set_cond;
  ua.score = p->score;
  ua.extras = s.unmask_extras;
  ua.conf_hist = st->prefix_conf;
  ua.conf_hist_stride = st->cap;
  ua.conf_hist_off = P;
  TRY(launch_unmask(ua, stream));
#undef TRY
  return DLLM_OK;
}
}  // namespace

extern "C" {

int dllm_denoise_step(const dllm_model* m, const dllm_state* st, const dllm_step_params* p, void* ws,
                      size_t ws_bytes, cudaStream_t stream) {
  return denoise_step_impl(m, st, p, ws, ws_bytes, stream, cudaGraphConditionalHandle(), 0);
}

// ------------------------------------------------------------------------------------------------ block graph
struct dllm_block_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int passes = 0;
  int conditional = 0;   // 1: the passes sit in conditional nodes (passes after an early finish are skipped)
};

void dllm_block_graph_destroy(dllm_block_graph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

int dllm_block_graph_skips_finished_passes(const dllm_block_graph* g) { return g ? g->conditional : 0; }

}  // extern "C"

namespace {
// Conditional (IF) nodes through the driver API, with the context given explicitly (the node, its handle and the
// kernels of its body must share one context: the current one). cuGraphAddNode is requested at the ABI of CUDA 12.2
// (no per-edge data): measured on driver 13.0, that entry point adds the IF node, while the 12.3 one with per-edge
// data (null here) refuses it with CUDA_ERROR_INVALID_VALUE, and so did the default query, which returns the 12.3
// one under a 12.x runtime.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CondHandleCreateFn)(CUgraphConditionalHandle*, CUgraph, CUcontext, unsigned int, unsigned int);
typedef CUresult (*GraphAddNodeFn)(CUgraphNode*, CUgraph, const CUgraphNode*, size_t, CUgraphNodeParams*);

struct CondApi {
  CtxGetCurrentFn ctx_get = nullptr;
  CondHandleCreateFn handle_create = nullptr;
  GraphAddNodeFn add_node = nullptr;
};

const CondApi& cond_api() {
  static CondApi api;
  static std::once_flag once;
  std::call_once(once, [] {
    auto get = [](const char* name, unsigned version) -> void* {
      void* p = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion(name, &p, version, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess)
        return nullptr;
      return p;
    };
    api.ctx_get = reinterpret_cast<CtxGetCurrentFn>(get("cuCtxGetCurrent", 12030));
    api.handle_create = reinterpret_cast<CondHandleCreateFn>(get("cuGraphConditionalHandleCreate", 12030));
    api.add_node = reinterpret_cast<GraphAddNodeFn>(get("cuGraphAddNode", 12020));
  });
  return api;
}

// Why the last block graph was built without conditional nodes (CUresult codes), for dllm_last_error.
static thread_local char g_cond_note[160] = "";

// One IF node after `prev` (nullable) in `graph`; its body graph is returned in *body.
bool add_if_node(cudaGraph_t graph, cudaGraphConditionalHandle cond, CUcontext ctx, cudaGraphNode_t prev,
                 cudaGraphNode_t* node, cudaGraph_t* body) {
  const CondApi& api = cond_api();
  if (!api.add_node) return false;
  CUgraphNodeParams np;
  memset(&np, 0, sizeof(np));
  np.type = CU_GRAPH_NODE_TYPE_CONDITIONAL;
  np.conditional.handle = cond;
  np.conditional.type = CU_GRAPH_COND_TYPE_IF;
  np.conditional.size = 1;
  np.conditional.ctx = ctx;
  CUgraphNode n = nullptr;
  CUgraphNode dep = reinterpret_cast<CUgraphNode>(prev);
  const CUresult rc = api.add_node(&n, reinterpret_cast<CUgraph>(graph), prev ? &dep : nullptr, prev ? 1 : 0, &np);
  if (rc != CUDA_SUCCESS) {
    snprintf(g_cond_note, sizeof(g_cond_note), "conditional node refused: cuGraphAddNode returned %d", (int)rc);
    return false;
  }
  *node = reinterpret_cast<cudaGraphNode_t>(n);
  *body = reinterpret_cast<cudaGraph_t>(np.conditional.phGraph_out[0]);
  return true;
}
}  // namespace

extern "C" {

int dllm_block_graph_create(const dllm_model* m, const dllm_state* st, const dllm_step_params* p, void* ws,
                            size_t ws_bytes, cudaStream_t capture_stream, dllm_block_graph** out) {
  REQ(out != nullptr, DLLM_ERR_INVALID_ARG, "block_graph_create: NULL output");
  *out = nullptr;
  REQ(capture_stream != nullptr, DLLM_ERR_INVALID_ARG,
      "block_graph_create: capture needs a created stream (not the legacy default stream)");
  int r = validate_step(m, st, p);
  if (r) return r;
  REQ(!p->commit, DLLM_ERR_INVALID_ARG, "block_graph_create: the template must describe a denoising pass");
  {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(capture_stream, &cs);
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "block_graph_create: cudaStreamIsCapturing");
    REQ(cs == cudaStreamCaptureStatusNone, DLLM_ERR_INVALID_ARG, "block_graph_create: the stream is capturing");
  }
  // every pass (with and without SPRINT selection) and the commit pass fit the workspace
  dllm_step_params pp = *p;
  for (int variant = 0; variant < 3; ++variant) {
    pp.retain = variant == 1 ? (p->sprint ? 1 : 0) : 0;
    pp.commit = variant == 2;
    StepPlan s;
    plan_step(m, st, &pp, nullptr, s);
    r = check_ws(ws, ws_bytes, s.total);
    if (r) return r;
  }
  dllm_block_graph* g = new dllm_block_graph();
  auto fail = [&](cudaError_t e, const char* what) {
    dllm_block_graph_destroy(g);
    return dllm_host::cuda_status(e, what);
  };
  cudaError_t e = cudaGraphCreate(&g->graph, 0);
  if (e != cudaSuccess) return fail(e, "block_graph_create: cudaGraphCreate");
  // conditional passes when the driver offers them (the handle and the nodes on the current context); otherwise
  // the passes follow one another unconditionally and those after an early finish return at entry
  // A conditional handle serves one node (measured on driver 13.0: a second IF node on the handle of the first is
  // refused with CUDA_ERROR_INVALID_VALUE, one on a handle of its own is added), so pass t has handle t. Every
  // handle is reset at each launch of the graph: handle 0 to 1 (the first pass always runs), the others to 0; the
  // unmask selection of pass t sets handle t + 1 to (masked positions left > 0), so a pass that is skipped leaves
  // every later one skipped too.
  const CondApi& api = cond_api();
  CUcontext ctx = nullptr;
  std::vector<cudaGraphConditionalHandle> conds(p->T_s, cudaGraphConditionalHandle());
  bool use_cond = false;
  g_cond_note[0] = 0;
  if (!(api.ctx_get && api.handle_create && api.add_node)) {
    snprintf(g_cond_note, sizeof(g_cond_note), "conditional nodes: driver entry points unavailable");
  } else {
    const CUresult rc0 = api.ctx_get(&ctx);
    CUresult rc1 = (rc0 == CUDA_SUCCESS && ctx) ? CUDA_SUCCESS : CUDA_ERROR_INVALID_CONTEXT;
    for (int t = 0; t < p->T_s && rc1 == CUDA_SUCCESS; ++t)
      rc1 = api.handle_create(reinterpret_cast<CUgraphConditionalHandle*>(&conds[t]),
                              reinterpret_cast<CUgraph>(g->graph), ctx, t == 0 ? 1u : 0u,
                              CU_GRAPH_COND_ASSIGN_DEFAULT);
    use_cond = rc1 == CUDA_SUCCESS;
    if (!use_cond)
      snprintf(g_cond_note, sizeof(g_cond_note), "conditional handle refused: cuCtxGetCurrent %d, handle %d",
               (int)rc0, (int)rc1);
  }
  auto capture_pass = [&](cudaGraph_t target, const cudaGraphNode_t* deps, size_t n_deps, int t, int commit,
                          cudaGraphConditionalHandle next, bool set_next) -> int {
    cudaError_t ce = cudaStreamBeginCaptureToGraph(capture_stream, target, deps, nullptr, n_deps,
                                                   cudaStreamCaptureModeThreadLocal);
    if (ce != cudaSuccess) return dllm_host::cuda_status(ce, "block_graph_create: cudaStreamBeginCaptureToGraph");
    dllm_step_params q = *p;
    q.t = commit ? 0 : t;
    q.commit = commit;
    q.retain = !commit && p->sprint && t == 0 ? 1 : 0;
    int rr = denoise_step_impl(m, st, &q, ws, ws_bytes, capture_stream, next, set_next ? 1 : 0);
    cudaGraph_t captured = nullptr;
    ce = cudaStreamEndCapture(capture_stream, &captured);
    if (rr) return rr;
    if (ce != cudaSuccess) return dllm_host::cuda_status(ce, "block_graph_create: cudaStreamEndCapture");
    return DLLM_OK;
  };
  if (use_cond) {
    cudaGraphNode_t prev = nullptr;
    for (int t = 0; t < p->T_s && !r; ++t) {
      cudaGraphNode_t node = nullptr;
      cudaGraph_t body = nullptr;
      if (!add_if_node(g->graph, conds[t], ctx, prev, &node, &body)) {
        r = DLLM_ERR_CUDA;
        break;
      }
      const bool last = t + 1 == p->T_s;
      r = capture_pass(body, nullptr, 0, t, 0, last ? cudaGraphConditionalHandle() : conds[t + 1], !last);
      prev = node;
    }
    if (!r) r = capture_pass(g->graph, &prev, 1, 0, 1, cudaGraphConditionalHandle(), false);
    if (!r) {
      e = cudaGraphInstantiate(&g->exec, g->graph, 0);
      if (e != cudaSuccess) {
        snprintf(g_cond_note, sizeof(g_cond_note), "conditional graph not instantiated: %s", cudaGetErrorString(e));
        r = DLLM_ERR_CUDA;
      }
    } else if (!g_cond_note[0]) {
      snprintf(g_cond_note, sizeof(g_cond_note), "conditional body not captured: %s", dllm_last_error());
    }
    if (r) {
      // the conditional build failed part way: start again with one unconditional capture
      (void)cudaGetLastError();
      use_cond = false;
      r = DLLM_OK;
      if (g->exec) cudaGraphExecDestroy(g->exec);
      g->exec = nullptr;
      cudaGraphDestroy(g->graph);
      g->graph = nullptr;
      e = cudaGraphCreate(&g->graph, 0);
      if (e != cudaSuccess) return fail(e, "block_graph_create: cudaGraphCreate");
    }
  }
  if (!use_cond) {
    // one capture of the whole block: the passes and the commit pass in stream order
    e = cudaStreamBeginCaptureToGraph(capture_stream, g->graph, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return fail(e, "block_graph_create: cudaStreamBeginCaptureToGraph");
    for (int t = 0; t <= p->T_s && !r; ++t) {
      dllm_step_params q = *p;
      q.t = t < p->T_s ? t : 0;
      q.commit = t == p->T_s;
      q.retain = !q.commit && p->sprint && t == 0 ? 1 : 0;
      r = denoise_step_impl(m, st, &q, ws, ws_bytes, capture_stream, cudaGraphConditionalHandle(), 0);
    }
    cudaGraph_t captured = nullptr;
    e = cudaStreamEndCapture(capture_stream, &captured);
    if (!r && e != cudaSuccess) r = dllm_host::cuda_status(e, "block_graph_create: cudaStreamEndCapture");
  }
  if (r) {
    dllm_block_graph_destroy(g);
    return r;
  }
  if (!g->exec) {
    e = cudaGraphInstantiate(&g->exec, g->graph, 0);
    if (e != cudaSuccess) return fail(e, "block_graph_create: cudaGraphInstantiate");
  }
  g->passes = p->T_s;
  g->conditional = use_cond ? 1 : 0;
  // leave the reason for a graph without conditions in the thread's last-error text (the call still succeeds)
  if (!use_cond) dllm_host::set_error("block_graph_create: passes unconditional (%s)", g_cond_note);
  *out = g;
  return DLLM_OK;
}

int dllm_block_graph_launch(const dllm_block_graph* g, cudaStream_t stream) {
  REQ(g != nullptr && g->exec != nullptr, DLLM_ERR_INVALID_ARG, "block_graph_launch: NULL graph");
  cudaError_t e = cudaGraphLaunch(g->exec, stream);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "block_graph_launch: cudaGraphLaunch");
  return DLLM_OK;
}

}  // extern "C"
