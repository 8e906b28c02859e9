// Shared device helpers of the denoising-step library (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "../../include/dllm.h"

#define DLLM_DEV __device__ __forceinline__

namespace dllm {

// Status word written by kernels that give up on a bounded wait (lives at the head of the workspace).
enum : int32_t { ST_OK = 0, ST_TIMEOUT_PRODUCER = 1, ST_TIMEOUT_MMA = 2, ST_TIMEOUT_EPILOGUE = 3 };

DLLM_DEV float to_f32(float x) { return x; }
DLLM_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> DLLM_DEV T from_f32(float x);
template <> DLLM_DEV float from_f32<float>(float x) { return x; }
template <> DLLM_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

DLLM_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
DLLM_DEV double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
DLLM_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
DLLM_DEV int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16-byte vector of 8 bf16 values unpacked to fp32.
DLLM_DEV void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Programmatic dependent launch. Every kernel of the library is launched so that the next kernel in the stream
// may be scheduled before it finishes (pdl_trigger lets that happen as soon as every CTA has started), and every
// kernel waits for the kernels before it to complete and their writes to be visible (pdl_wait) before it reads or
// writes any global memory; only on-chip set-up (barriers, tensor memory, descriptor prefetch) may precede it.
// Both are no-ops for a launch without the attribute.
DLLM_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
DLLM_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
DLLM_DEV void pdl_enter() {
  pdl_trigger();
  pdl_wait();
}

DLLM_DEV uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Launch with programmatic stream serialization (see pdl_wait); errors surface through cudaGetLastError.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace dllm

// Host-side error plumbing shared by the entry points.
namespace dllm_host {
void set_error(const char* fmt, ...);
int cuda_status(cudaError_t e, const char* what);
void count_launch();
}  // namespace dllm_host

// Every kernel launch is followed by this check, which also counts the launch (dllm_launch_count).
#define DLLM_CHECK_LAUNCH(what)                                                   \
  do {                                                                            \
    dllm_host::count_launch();                                                    \
    cudaError_t _e = cudaGetLastError();                                          \
    if (_e != cudaSuccess) return dllm_host::cuda_status(_e, what);               \
  } while (0)

#define DLLM_REQUIRE(cond, code, ...)                                             \
  do {                                                                            \
    if (!(cond)) {                                                                \
      dllm_host::set_error(__VA_ARGS__);                                          \
      return code;                                                                \
    }                                                                             \
  } while (0)
