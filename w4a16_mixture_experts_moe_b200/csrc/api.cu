// Status plumbing and small host-side entry points of the C ABI.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace moe {

static thread_local char g_last_error[512] = "";

int set_error(int status, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }

int check_launch(const char *what, int n) {
  count_launches(n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MOE_OK;
}

int allow_dynamic_smem(const void *kernel, size_t bytes, const char *what) {
  struct Entry { const void *kernel; int device; size_t bytes; };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s: cudaGetDevice failed", what);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (table[i].kernel == kernel && table[i].device == dev && table[i].bytes >= bytes) return MOE_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s: cannot allow %zu B of shared memory: %s", what, bytes, cudaGetErrorString(e));
  for (int i = 0; i < used; ++i)
    if (table[i].kernel == kernel && table[i].device == dev) { table[i].bytes = bytes; return MOE_OK; }
  if (used < 256) table[used++] = Entry{kernel, dev, bytes};
  return MOE_OK;
}

}  // namespace moe

extern "C" {

const char *moe_last_error(void) { return moe::g_last_error; }

int moe_abi_version(void) { return 1; }

uint64_t moe_launch_counter(void) { return moe::g_launches.load(std::memory_order_relaxed); }

int moe_expert_record_layout(int H, int I, moe_record_layout *out) {
  if (!out) return moe::set_error(MOE_ERR_INVALID_ARG, "moe_expert_record_layout: out is NULL");
  if (H <= 0 || I <= 0 || H % moe::GROUP || I % moe::GROUP)
    return moe::set_error(MOE_ERR_SHAPE, "moe_expert_record_layout: H=%d I=%d must be positive multiples of 128", H, I);
  const int64_t q = int64_t(I) * H / 2;        // packed bytes of one matrix
  const int64_t s = int64_t(I) * H / 128 * 2;  // scale bytes of one matrix
  auto up256 = [](int64_t v) { return (v + 255) / 256 * 256; };
  out->gate_q = 0;
  out->up_q = up256(q);
  out->down_q = out->up_q + up256(q);
  out->gate_s = out->down_q + up256(q);
  out->up_s = out->gate_s + up256(s);
  out->down_s = out->up_s + up256(s);
  out->bytes = out->down_s + up256(s);
  return MOE_OK;
}

int moe_read_device_error(void *ws, moe_stream_t stream, int32_t *code) {
  if (!ws) return moe::set_error(MOE_ERR_INVALID_ARG, "moe_read_device_error: ws is NULL");
  int32_t v = 0;
  cudaStream_t s = moe::as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(v), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return moe::set_error(MOE_ERR_CUDA, "moe_read_device_error: %s", cudaGetErrorString(e));
  if (code) *code = v;
  if (v != MOE_DEVERR_NONE) {
    const char *what = v == MOE_DEVERR_EXPERT_ID     ? "expert id out of range"
                       : v == MOE_DEVERR_NOT_RESIDENT ? "active expert not resident in any slot"
                       : v == MOE_DEVERR_TIMEOUT      ? "bounded pipeline wait timed out"
                       : v == MOE_DEVERR_RANGE        ? "activation outside FP16 range on the tensor-core path"
                                                      : "unknown device error";
    return moe::set_error(MOE_ERR_DEVICE, "device error %d: %s", v, what);
  }
  return MOE_OK;
}

}  // extern "C"
