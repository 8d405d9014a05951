// Shared helpers of the CUDA library: status plumbing, BF16 bit helpers,
// device error word. Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "../../include/exactmoe.h"

namespace moe {

// ---------------------------------------------------------------- host side
int set_error(int status, const char *fmt, ...);
// Checks the launch status and adds n to the process-wide count of kernels
// this library has enqueued.
int check_launch(const char *what, int n = 1);
void count_launches(int n);
// Raises a kernel's dynamic shared-memory limit on the current device (once
// per device and kernel; later calls are a lookup).
int allow_dynamic_smem(const void *kernel, size_t bytes, const char *what);
// Enqueues x [n8 * 8] BF16 -> x16 FP16 (programmatic dependent launch);
// MOE_DEVERR_RANGE goes to *err (if not NULL) for a value beyond FP16's range.
int launch_bf16_to_f16(const uint16_t *x, uint16_t *x16, int64_t n8, int32_t *err, cudaStream_t s, const char *what);

static inline cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// A named NVTX range over an entry point's host work (argument checks and
// launches), so a timeline profiler shows each call of the layer step; a
// no-op unless a profiler is attached.
struct NvtxScope {
  explicit NvtxScope(const char *name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
  NvtxScope(const NvtxScope &) = delete;
  NvtxScope &operator=(const NvtxScope &) = delete;
};

static inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int GROUP = 128;
constexpr int MAX_E = 256;
constexpr int MAX_K = 32;
constexpr size_t WS_HEADER = 256;  // error word + scheduler counters

// ---------------------------------------------------------------- device side
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&b);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Eight BF16 values -> eight FP16 values (round to nearest even); `bad` is
// set if any lies outside FP16's finite range. Exact for 2^-17 <= |v| <=
// 65504 and for zero; smaller magnitudes round to a multiple of 2^-24.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 v, bool &bad) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float lo = bf16_lo(in[c]), hi = bf16_hi(in[c]);
    bad |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
    const __half2 hv = __floats2half2_rn(lo, hi);
    out[c] = *reinterpret_cast<const uint32_t *>(&hv);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// First writer wins; later codes are dropped.
__device__ __forceinline__ void flag_error(int32_t *err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

// SiLU with CUDA's fast exponential and fast divide (a few ulp in fp32, far
// below the BF16 rounding of h that follows; for g < -88 the denominator is
// +inf and the result 0).
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Programmatic dependent launch: every hot-path kernel lets the next kernel of
// the stream be scheduled as soon as all of its own CTAs are running
// (pdl_trigger), and waits for the previous kernel's results before reading
// anything (pdl_wait). Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kernel` with the programmatic-stream-serialization attribute, so
// its launch overlaps the tail of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
