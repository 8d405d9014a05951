// A4 — deterministic grouping of (token, slot) pairs by chosen expert
// (ExactMoE paper, Figure 1 caption: the tokens are gathered per chosen expert).
//
// A stable counting sort over the P = T*k flat pair indices, in chunks of
// 1024 pairs (one pair per thread):
//   hist    — per-chunk expert histogram (shared-memory atomics; counts only,
//             so their order does not matter) into the workspace table;
//   scan    — one CTA turns the [chunks][E] table into per-chunk bases and
//             writes counts and offsets;
//   scatter — each chunk ranks its pairs stably (warp match + per-warp
//             counts scanned across warps) and writes sorted_pair/pair_pos.
// With a single chunk (P <= 1024, every decode size) the three phases run in
// one kernel launch.
#include <mutex>

#include "common.cuh"

namespace moe {

constexpr int GT_CHUNK = 1024;  // pairs per CTA, one per thread

struct GroupWs {
  int32_t *err;
  int32_t *table;  // [chunks][E]
};

static GroupWs group_ws(void *ws) {
  GroupWs g;
  g.err = reinterpret_cast<int32_t *>(ws);
  g.table = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(ws) + WS_HEADER);
  return g;
}

__device__ __forceinline__ int read_id(const int32_t *ids, int p, int P, int E, int32_t *err) {
  if (p >= P) return -1;
  const int e = ids[p];
  if (e < 0 || e >= E) {
    if (err) flag_error(err, MOE_DEVERR_EXPERT_ID);
    return -1;
  }
  return e;
}

// Warp-cooperative exclusive scan of in[0..E) (E <= 256) into out[0..E);
// returns the total on every lane. Lane l owns entries 8l .. 8l+7.
__device__ int warp_exclusive_scan(const int32_t *in, int32_t *out, int E) {
  const int lane = threadIdx.x & 31;
  int v[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int x = lane * 8 + i;
    v[i] = x < E ? in[x] : 0;
    local += v[i];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  int run = incl - local;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int x = lane * 8 + i;
    if (x < E) out[x] = run;
    run += v[i];
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// Stable rank of this thread's pair among the chunk's pairs of the same
// expert; `wcnt` is [warps][E] shared scratch, `base` [E] the chunk's first
// position per expert. Writes the outputs for valid pairs.
__device__ void chunk_scatter(int e, int p, int E, int32_t *wcnt, const int32_t *base, int32_t *sorted_pair,
                              int32_t *pair_pos, bool in_range) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int i = threadIdx.x; i < nwarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int lane_rank = __popc(same & ((1u << lane) - 1u));
  if (e >= 0 && lane_rank == 0) wcnt[warp * E + e] = __popc(same);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {  // exclusive scan down each expert column
    int run = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int c = wcnt[w * E + x];
      wcnt[w * E + x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (e >= 0) {
    const int pos = base[e] + wcnt[warp * E + e] + lane_rank;
    sorted_pair[pos] = p;
    pair_pos[p] = pos;
  } else if (in_range) {
    pair_pos[p] = -1;
  }
}

// One-launch path: P <= GT_CHUNK, one thread per pair (a single warp at T=1..4).
__global__ void __launch_bounds__(GT_CHUNK) group_small_kernel(const int32_t *__restrict__ ids, int P, int E,
                                                               int32_t *counts, int32_t *offsets,
                                                               int32_t *sorted_pair, int32_t *pair_pos,
                                                               int32_t *err) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t hist[MAX_E + 1];
  __shared__ int32_t base[MAX_E];
  __shared__ int32_t wcnt[32 * MAX_E];
  const int p = threadIdx.x;
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int e = read_id(ids, p, P, E, err);
  if (e >= 0) atomicAdd(&hist[e], 1);
  __syncthreads();
  if (threadIdx.x < 32) {
    const int total = warp_exclusive_scan(hist, base, E);
    __syncwarp();
    for (int x = threadIdx.x; x < E; x += 32) {
      offsets[x] = base[x];
      counts[x] = hist[x];
    }
    if (threadIdx.x == 0) offsets[E] = total;
  }
  __syncthreads();
  chunk_scatter(e, p, E, wcnt, base, sorted_pair, pair_pos, p < P);
}

__global__ void __launch_bounds__(GT_CHUNK) group_hist_kernel(const int32_t *__restrict__ ids, int P, int E,
                                                              int32_t *table, int32_t *err) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t hist[MAX_E];
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int p = blockIdx.x * GT_CHUNK + threadIdx.x;
  const int e = read_id(ids, p, P, E, err);
  if (e >= 0) atomicAdd(&hist[e], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) table[blockIdx.x * E + i] = hist[i];
}

__global__ void __launch_bounds__(MAX_E) group_scan_kernel(int chunks, int E, int32_t *table, int32_t *counts,
                                                          int32_t *offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t tot[MAX_E];
  __shared__ int32_t off[MAX_E];
  const int x = threadIdx.x;
  int run = 0;
  if (x < E) {
    for (int c = 0; c < chunks; ++c) {
      const int v = table[c * E + x];
      table[c * E + x] = run;
      run += v;
    }
    tot[x] = run;
    counts[x] = run;
  }
  __syncthreads();
  if (x < 32) {
    const int total = warp_exclusive_scan(tot, off, E);
    if (x == 0) offsets[E] = total;
  }
  __syncthreads();
  if (x < E) {
    offsets[x] = off[x];
    for (int c = 0; c < chunks; ++c) table[c * E + x] += off[x];
  }
}

__global__ void __launch_bounds__(GT_CHUNK) group_scatter_kernel(const int32_t *__restrict__ ids, int P, int E,
                                                                 const int32_t *table, int32_t *sorted_pair,
                                                                 int32_t *pair_pos) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t base[MAX_E];
  __shared__ int32_t wcnt[32 * MAX_E];
  for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = table[blockIdx.x * E + i];
  const int p = blockIdx.x * GT_CHUNK + threadIdx.x;
  const int e = read_id(ids, p, P, E, nullptr);
  __syncthreads();
  chunk_scatter(e, p, E, wcnt, base, sorted_pair, pair_pos, p < P);
}

}  // namespace moe

extern "C" size_t moe_group_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return moe::WS_HEADER;
  const int64_t P = int64_t(T) * k;
  const int64_t chunks = (P + moe::GT_CHUNK - 1) / moe::GT_CHUNK;
  return size_t(moe::WS_HEADER + ((chunks * E * 4 + 255) / 256) * 256);
}

extern "C" int moe_group_tokens(const int32_t *topk_ids, int T, int k, int E, int32_t *counts, int32_t *offsets,
                                int32_t *sorted_pair, int32_t *pair_pos, void *ws, size_t ws_bytes,
                                moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_group_tokens");
  using namespace moe;
  if (T < 0 || E < 1 || E > MAX_E || k < 1 || k > E || k > MAX_K)
    return set_error(MOE_ERR_SHAPE, "moe_group_tokens: T=%d E=%d k=%d (need T>=0, 1<=E<=256, 1<=k<=min(E,32))", T, E, k);
  const int64_t P64 = int64_t(T) * k;
  if (P64 > (int64_t(1) << 30)) return set_error(MOE_ERR_SHAPE, "moe_group_tokens: T*k=%lld too large", (long long)P64);
  if (!counts || !offsets || !ws || (P64 > 0 && (!topk_ids || !sorted_pair || !pair_pos)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_group_tokens: NULL pointer");
  if (!aligned(ws, 256)) return set_error(MOE_ERR_INVALID_ARG, "moe_group_tokens: ws must be 256-byte aligned");
  if (ws_bytes < moe_group_workspace_size(T, k, E))
    return set_error(MOE_ERR_INVALID_ARG, "moe_group_tokens: workspace %zu B < %zu B", ws_bytes,
                     moe_group_workspace_size(T, k, E));
  cudaStream_t s = as_stream(stream);
  const int P = int(P64);
  GroupWs g = group_ws(ws);
  cudaError_t e;
  if (P <= GT_CHUNK) {
    const int threads = P <= 32 ? 32 : (P + 31) / 32 * 32;
    e = launch_pdl(group_small_kernel, dim3(1), dim3(threads), 0, s, topk_ids, P, E, counts, offsets, sorted_pair,
                   pair_pos, g.err);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_group_tokens: %s", cudaGetErrorString(e));
    return check_launch("moe_group_tokens");
  }
  const int chunks = (P + GT_CHUNK - 1) / GT_CHUNK;
  e = launch_pdl(group_hist_kernel, dim3(chunks), dim3(GT_CHUNK), 0, s, topk_ids, P, E, g.table, g.err);
  if (e == cudaSuccess) e = launch_pdl(group_scan_kernel, dim3(1), dim3(MAX_E), 0, s, chunks, E, g.table, counts, offsets);
  if (e == cudaSuccess)
    e = launch_pdl(group_scatter_kernel, dim3(chunks), dim3(GT_CHUNK), 0, s, topk_ids, P, E,
                   static_cast<const int32_t *>(g.table), sorted_pair, pair_pos);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_group_tokens: %s", cudaGetErrorString(e));
  return check_launch("moe_group_tokens", 3);
}

// ---------------------------------------------------------------------------
// Grouping for callers that cannot allocate device memory.
//
// Same computation and kernels as moe_group_tokens; the only difference is
// where the scratch lives: a file-scope device array sized for at most
// MOE_NOALLOC_MAX_PAIRS pairs and 256 experts, which every GPU that loads
// this library keeps until the process exits. Host code must not use the
// array's name as a device address (on the host it is only a stand-in), so
// the address is looked up with cudaGetSymbolAddress with the device current.
// A call made outside stream capture looks it up every time (a device reset
// or a new primary context moves the array); a call made under capture
// reuses the address of the last call on that device, so the first call on a
// device belongs before any capture.
namespace moe {

constexpr size_t NOALLOC_SCRATCH_BYTES =
    WS_HEADER + size_t((MOE_NOALLOC_MAX_PAIRS + GT_CHUNK - 1) / GT_CHUNK) * MAX_E * sizeof(int32_t);

static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

static int noalloc_scratch(cudaStream_t stream, void **out) {
  static std::mutex mu;
  static void *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_group_tokens_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return set_error(MOE_ERR_UNSUPPORTED, "moe_group_tokens_noalloc: device %d", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) cap = cudaStreamCaptureStatusActive;  // e.g. the legacy
  std::lock_guard<std::mutex> lock(mu);                                                         // stream during a capture
  if (!addr[dev] || cap == cudaStreamCaptureStatusNone) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(MOE_ERR_CUDA, "moe_group_tokens_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_group_tokens_noalloc(const int32_t *topk_ids, int T, int k, int E, int32_t *counts,
                                        int32_t *offsets, int32_t *sorted_pair, int32_t *pair_pos,
                                        moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_group_tokens_noalloc");
  using namespace moe;
  if (T < 0 || k < 1 || int64_t(T) * k > MOE_NOALLOC_MAX_PAIRS)
    return set_error(MOE_ERR_SHAPE, "moe_group_tokens_noalloc: T*k = %lld pairs exceeds the fixed scratch limit of %d",
                     (long long)(int64_t(T) * (k < 1 ? 1 : k)), MOE_NOALLOC_MAX_PAIRS);
  void *ws = nullptr;
  const int st = noalloc_scratch(as_stream(stream), &ws);
  if (st != MOE_OK) return st;
  return moe_group_tokens(topk_ids, T, k, E, counts, offsets, sorted_pair, pair_pos, ws, NOALLOC_SCRATCH_BYTES,
                          stream);
}
