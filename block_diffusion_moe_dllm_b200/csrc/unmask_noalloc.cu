// dllm_unmask_noalloc: the confidence + unmasking call for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch: a plug-in running inside a host application that owns the
// device's memory pool and hands out no allocator, or a serving loop that forbids cudaMalloc once it has started
// because cudaMalloc can synchronise the device and stall every stream. They still own their inputs and outputs,
// but cannot provide the workspace dllm_unmask needs for its per-chunk partial results. This entry point keeps
// that scratch in a fixed array inside the library instead.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes (256 KiB: 16384 partial entries). Every GPU that loads the library
// holds it until the process exits. Host code must never pass the array's name to a kernel: on the host that
// name is a stand-in, not a device address. Its device address is taken once per device, with that device
// current, through cudaGetSymbolAddress (the first call on each device does this set-up; make that first call
// before any stream capture). Every call shares the one array and it keeps the last call's contents; nothing in it
// has to start at zero, since every partial the selection reads is written earlier in the same call. Calls whose
// kernels overlap on the GPU (different streams, or no ordering between them) race on the array.
#include <mutex>
#include "common.cuh"
#include "misc.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(256) << 10;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_unmask_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use, then cached).
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dllm_host::cuda_status(e, "unmask_noalloc: cudaGetDevice");
  DLLM_REQUIRE(dev >= 0 && dev < kMaxDevices, DLLM_ERR_UNSUPPORTED, "unmask_noalloc: device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_unmask_scratch);
    if (e != cudaSuccess) return dllm_host::cuda_status(e, "unmask_noalloc: cudaGetSymbolAddress");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DLLM_OK;
}

}  // namespace

extern "C" int dllm_unmask_noalloc(const dllm_unmask_desc* d, const void* logits, const int32_t* row_pos,
                                   const int32_t* n_rows_dev, int32_t* tokens, uint8_t* mask, int32_t* sel,
                                   int32_t* nsel, float* conf, int32_t* remaining, cudaStream_t stream) {
  using namespace dllm;
  DLLM_REQUIRE(d && logits && row_pos && n_rows_dev && tokens && mask && sel && nsel && conf && remaining,
               DLLM_ERR_INVALID_ARG, "unmask_noalloc: NULL argument");
  DLLM_REQUIRE(d->B >= 1 && d->B <= 1024 && d->L >= 1 && d->L <= 32 && d->V >= 1 && d->max_rows >= 0 &&
                   d->max_rows <= d->B * d->L,
               DLLM_ERR_SHAPE, "unmask_noalloc: bad shape (B <= 1024, L <= 32, max_rows <= B*L)");
  DLLM_REQUIRE(d->T_s >= 1 && d->t >= 0 && d->t < d->T_s, DLLM_ERR_INVALID_ARG, "unmask_noalloc: step %d of %d", d->t,
               d->T_s);
  DLLM_REQUIRE(d->mode == DLLM_UNMASK_FIXED || d->mode == DLLM_UNMASK_THRESHOLD, DLLM_ERR_INVALID_ARG,
               "unmask_noalloc: bad mode");
  DLLM_REQUIRE(d->mode == DLLM_UNMASK_FIXED || d->k_max >= 1, DLLM_ERR_INVALID_ARG, "unmask_noalloc: k_max must be >= 1");
  DLLM_REQUIRE(d->dtype == DLLM_BF16 || d->dtype == DLLM_F32, DLLM_ERR_INVALID_ARG, "unmask_noalloc: bad dtype");
  DLLM_REQUIRE(d->vocab_offset >= 0, DLLM_ERR_INVALID_ARG, "unmask_noalloc: negative vocab_offset");
  DLLM_REQUIRE(d->cfg >= 0 && d->cfg <= 2, DLLM_ERR_INVALID_ARG, "unmask_noalloc: cfg %d (0, 1 or 2)", d->cfg);
  DLLM_REQUIRE(d->score >= DLLM_SCORE_LOW_CONFIDENCE && d->score <= DLLM_SCORE_NEG_ENTROPY, DLLM_ERR_INVALID_ARG,
               "unmask_noalloc: bad score %d", d->score);
  const int n_chunks = unmask_chunks(d->max_rows, d->V);
  const size_t part_bytes = (unmask_partials_bytes(d->max_rows, n_chunks) + 255) & ~size_t(255);
  const size_t need = part_bytes + unmask_extras_bytes(d->score, d->max_rows, n_chunks, d->B, d->L);
  DLLM_REQUIRE(need <= kNoAllocScratchBytes, DLLM_ERR_UNSUPPORTED,
               "unmask_noalloc: %d rows x %d vocabulary chunks need %zu bytes of scratch, above the fixed %zu",
               d->max_rows, n_chunks, need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st) return st;
  UnmaskArgs a;
  a.B = d->B; a.L = d->L; a.V = d->V; a.max_rows = d->max_rows; a.t = d->t; a.T_s = d->T_s; a.mode = d->mode;
  a.k_max = d->k_max; a.cfg = d->cfg; a.vocab_offset = d->vocab_offset; a.dtype = d->dtype; a.tau = d->tau;
  a.cfg_scale = d->cfg_scale; a.cfg_image_scale = d->cfg_image_scale; a.logits = logits; a.row_pos = row_pos; a.n_rows = n_rows_dev; a.tokens = tokens;
  a.mask = mask; a.sel = sel; a.nsel = nsel; a.conf = conf; a.remaining = remaining;
  a.partials = scratch;
  a.n_chunks = n_chunks;
  a.score = d->score;
  a.extras = d->score != DLLM_SCORE_LOW_CONFIDENCE ? static_cast<char*>(scratch) + part_bytes : nullptr;
  return launch_unmask(a, stream);
}
