// A7 — router-weighted combine of the k expert outputs of each token, with
// an optional residual: out[t] = bf16_rn(res[t] + sum_j w[t][j] * y[pos(t,j)]),
// fp32 expert outputs, fp32 accumulation in increasing j (deterministic). A
// CTA covers CB_THREADS * 4 hidden elements of one token (grid: tokens x hidden
// slices, so a small decode batch still spreads over many SMs); each thread
// owns 4 consecutive elements and issues the loads of up to CB_J expert rows
// before the first multiply-add, so a token costs one round trip to L2 per
// CB_J rows instead of one per row.
#include "common.cuh"

namespace moe {

constexpr int CB_THREADS = 128;
constexpr int CB_J = 8;

__global__ void __launch_bounds__(CB_THREADS) combine_kernel(const float *__restrict__ y,
                                                              const float *__restrict__ topk_w,
                                                              const int32_t *__restrict__ pair_pos,
                                                              const uint16_t *residual, int k, int H,
                                                              uint16_t *out) {
  __shared__ float ws[MAX_K];
  __shared__ int32_t ps[MAX_K];
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    ws[threadIdx.x] = topk_w[int64_t(t) * k + threadIdx.x];
    ps[threadIdx.x] = pair_pos[int64_t(t) * k + threadIdx.x];
  }
  __syncthreads();
  const int c = blockIdx.y * CB_THREADS + threadIdx.x;  // 4-element piece of the row
  if (c >= H / 4) return;
  float acc[4];
  if (residual) {
    const uint2 r = reinterpret_cast<const uint2 *>(residual + int64_t(t) * H)[c];
    acc[0] = bf16_lo(r.x); acc[1] = bf16_hi(r.x); acc[2] = bf16_lo(r.y); acc[3] = bf16_hi(r.y);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0.f;
  }
  for (int j0 = 0; j0 < k; j0 += CB_J) {
    float4 v[CB_J];
#pragma unroll
    for (int u = 0; u < CB_J; ++u) {
      const int j = j0 + u;
      const int pos = j < k ? ps[j] : -1;
      v[u] = pos >= 0 ? __ldg(reinterpret_cast<const float4 *>(y + int64_t(pos) * H) + c)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < CB_J; ++u) {
      const int j = j0 + u;
      if (j < k && ps[j] >= 0) {  // dropped pairs contribute nothing, not even a zero
        const float w = ws[j];
        acc[0] = fmaf(w, v[u].x, acc[0]); acc[1] = fmaf(w, v[u].y, acc[1]);
        acc[2] = fmaf(w, v[u].z, acc[2]); acc[3] = fmaf(w, v[u].w, acc[3]);
      }
    }
  }
  uint2 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  reinterpret_cast<uint2 *>(out + int64_t(t) * H)[c] = o;
}

}  // namespace moe

extern "C" int moe_combine(const float *y, const float *topk_w, const int32_t *pair_pos,
                           const moe_bf16 *residual, int T, int k, int H, moe_bf16 *out, moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_combine");
  using namespace moe;
  if (T < 0 || k < 1 || k > MAX_K || H < 8 || H % 8)
    return set_error(MOE_ERR_SHAPE, "moe_combine: T=%d k=%d H=%d (need T>=0, 1<=k<=32, H a multiple of 8)", T, k, H);
  if (T == 0) return MOE_OK;
  if (!y || !topk_w || !pair_pos || !out) return set_error(MOE_ERR_INVALID_ARG, "moe_combine: NULL pointer");
  if (!aligned(y, 16) || !aligned(out, 16) || (residual && !aligned(residual, 16)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_combine: y, residual and out must be 16-byte aligned");
  const dim3 grid(unsigned(T), unsigned((H / 4 + CB_THREADS - 1) / CB_THREADS));
  cudaError_t e = launch_pdl(combine_kernel, grid, dim3(CB_THREADS), 0, as_stream(stream), y, topk_w, pair_pos,
                             residual, k, H, out);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_combine: %s", cudaGetErrorString(e));
  return check_launch("moe_combine");
}
