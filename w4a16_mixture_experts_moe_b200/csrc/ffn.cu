// Entry point of the grouped W4A16 SwiGLU expert FFN (A5 + A6): argument
// checks, workspace layout and the choice between the decode-sized GEMV path
// and the prefill-sized tensor-core path.
#include <atomic>

#include "ffn.cuh"

namespace moe {

static size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// Average rows per expert at which the tensor-core path takes over.
constexpr int TC_MIN_ROWS_PER_EXPERT = 32;

// x [T][H] BF16 -> FP16 copy, the decode path's gate/up input: exact for
// BF16 values v with 2^-17 <= |v| <= 65504 and for zero; smaller magnitudes
// round to a multiple of 2^-24 (absolute error at most 2^-25); values above
// FP16's finite range are flagged.
__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t *__restrict__ x, uint16_t *__restrict__ x16,
                                                       int64_t n8, int32_t *err) {
  pdl_trigger();
  pdl_wait();
  bool bad = false;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x)
    reinterpret_cast<uint4 *>(x16)[i] = bf16x8_to_f16x8(__ldg(reinterpret_cast<const uint4 *>(x) + i), bad);
  if (bad) flag_error(err, MOE_DEVERR_RANGE);
}

// xs[r] = FP16(x[sorted_pair[r] / k]) for the P rows in group order: the
// tensor-core gate/up pass then loads each token tile of an expert as one
// contiguous block of rows. One warp per row (grid-stride over rows); each
// lane issues all its loads of a pass before converting and storing, so a
// row costs one round trip rather than one per 16-byte piece. F16IN: x
// already holds FP16 values, which are copied as they are.
template <bool F16IN>
__global__ void __launch_bounds__(256) gather_x_f16_kernel(const uint16_t *__restrict__ x,
                                                           const int32_t *__restrict__ sorted_pair, int k, int T,
                                                           int H8, int64_t P, uint16_t *__restrict__ xs,
                                                           int32_t *err) {
  pdl_trigger();
  pdl_wait();
  constexpr int U = 8;
  bool bad = false;
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5; r < P; r += nw) {
    const int t = sorted_pair[r] / k;
    const bool ok = t >= 0 && t < T;
    if (!ok && lane == 0) flag_error(err, MOE_DEVERR_EXPERT_ID);
    const uint4 *src = reinterpret_cast<const uint4 *>(x + int64_t(ok ? t : 0) * H8 * 8);
    uint4 *dst = reinterpret_cast<uint4 *>(xs) + r * H8;
    for (int c0 = lane; c0 < H8; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = c0 + 32 * u < H8 ? __ldg(src + c0 + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < H8)
          dst[c0 + 32 * u] = !ok ? make_uint4(0, 0, 0, 0) : F16IN ? v[u] : bf16x8_to_f16x8(v[u], bad);
    }
  }
  if (bad) flag_error(err, MOE_DEVERR_RANGE);
}

static std::atomic<int> g_tc_stall{0};

int take_tc_stall() {
  int v = g_tc_stall.load();
  while (v > 0 && !g_tc_stall.compare_exchange_weak(v, v - 1)) {
  }
  return v > 0 ? 1 : 0;
}

int launch_bf16_to_f16(const uint16_t *x, uint16_t *x16, int64_t n8, int32_t *err, cudaStream_t s, const char *what) {
  const int64_t want = (n8 + 255) / 256, cap = 148 * 8;
  const int blocks = int(want < cap ? (want > 0 ? want : 1) : cap);
  const cudaError_t e = launch_pdl(x_to_f16_kernel, dim3(blocks), dim3(256), 0, s, x, x16, n8, err);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s (x to fp16): %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

int launch_x_to_f16(const FfnArgs &a, cudaStream_t s) {
  if (a.x_f16) return MOE_OK;  // the caller's x is the FP16 copy already
  return launch_bf16_to_f16(a.x, a.x16, int64_t(a.T) * a.H / 8, a.err, s, "moe_grouped_w4a16_ffn (x to fp16)");
}

int launch_gather_x_f16(const FfnArgs &a, cudaStream_t s) {
  const int64_t P = int64_t(a.T) * a.k;
  const int64_t want = (P + 7) / 8, cap = 148 * 16;  // 8 rows (warps) per block
  const int blocks = int(want < cap ? (want > 0 ? want : 1) : cap);
  const cudaError_t e =
      a.x_f16 ? launch_pdl(gather_x_f16_kernel<true>, dim3(blocks), dim3(256), 0, s, a.x, a.sorted_pair, a.k, a.T,
                           a.H / 8, P, a.xs, a.err)
              : launch_pdl(gather_x_f16_kernel<false>, dim3(blocks), dim3(256), 0, s, a.x, a.sorted_pair, a.k, a.T,
                           a.H / 8, P, a.xs, a.err);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (gather x): %s", cudaGetErrorString(e));
  return check_launch("moe_grouped_w4a16_ffn (gather x)");
}

}  // namespace moe

extern "C" int moe_debug_stall_next_tc_ffn(int calls) {
  if (calls < 0) return moe::set_error(MOE_ERR_INVALID_ARG, "moe_debug_stall_next_tc_ffn: calls < 0");
  moe::g_tc_stall.store(calls);
  return MOE_OK;
}

namespace moe {
// The tensor-core path may run for this call (AUTO's choice, before any
// fallback to the GEMV path on other hardware).
static bool may_use_tc(int T, int k, int E, int path) {
  if (path == MOE_PATH_TC) return true;
  if (path == MOE_PATH_GEMV || path == MOE_PATH_SEQUENTIAL) return false;
  return int64_t(T) * k >= int64_t(TC_MIN_ROWS_PER_EXPERT) * E;
}
}  // namespace moe

extern "C" size_t moe_ffn_workspace_size(int T, int k, int E, int H, int I, int path) {
  path &= ~MOE_FFN_X_F16;
  if (T < 0 || k < 1 || I < 0 || H < 0) return moe::WS_HEADER;
  // header | h [T*k][I] 16-bit | x as FP16: [T][H] (GEMV) or [T*k][H] in group order (tensor cores)
  const size_t xrows = moe::may_use_tc(T, k, E, path) ? size_t(T) * size_t(k) : size_t(T);
  return moe::WS_HEADER + moe::round256(size_t(T) * size_t(k) * size_t(I) * 2) + moe::round256(xrows * size_t(H) * 2);
}

extern "C" int moe_grouped_w4a16_ffn(const moe_bf16 *x, const int32_t *sorted_pair, const int32_t *offsets,
                                     const void *bank, int64_t record_bytes, const int32_t *expert_slot,
                                     int n_slots, int T, int k, int E, int H, int I, int path, float *y,
                                     void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_grouped_w4a16_ffn");
  using namespace moe;
  if (T < 0 || E < 1 || E > MAX_E || k < 1 || k > E || k > MAX_K)
    return set_error(MOE_ERR_SHAPE, "moe_grouped_w4a16_ffn: T=%d E=%d k=%d (need T>=0, 1<=E<=256, 1<=k<=min(E,32))",
                     T, E, k);
  if (H < GROUP || I < GROUP || H % GROUP || I % GROUP)
    return set_error(MOE_ERR_SHAPE, "moe_grouped_w4a16_ffn: H=%d I=%d must be positive multiples of 128", H, I);
  if (int64_t(T) * k > (int64_t(1) << 30))
    return set_error(MOE_ERR_SHAPE, "moe_grouped_w4a16_ffn: T*k too large");
  const bool x_f16 = (path & MOE_FFN_X_F16) != 0;
  path &= ~MOE_FFN_X_F16;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_GEMV && path != MOE_PATH_TC && path != MOE_PATH_SEQUENTIAL)
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: unknown path %d", path);
  moe_record_layout L;
  int st = moe_expert_record_layout(H, I, &L);
  if (st != MOE_OK) return st;
  if (!offsets || !bank || !ws || (T > 0 && (!x || !sorted_pair || !y)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: NULL pointer");
  if (record_bytes < L.bytes || record_bytes % 256)
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: record_bytes=%lld (need >= %lld, multiple of 256)",
                     (long long)record_bytes, (long long)L.bytes);
  if (n_slots < 1 || (!expert_slot && n_slots < E))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: n_slots=%d (identity mapping needs >= E)", n_slots);
  if (!aligned(bank, 256) || !aligned(ws, 256) || (T > 0 && (!aligned(x, 16) || !aligned(y, 16))))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: bank/ws need 256-byte, x/y 16-byte alignment");
  if (ws_bytes < moe_ffn_workspace_size(T, k, E, H, I, path))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: workspace %zu B < %zu B", ws_bytes,
                     moe_ffn_workspace_size(T, k, E, H, I, path));

  cudaStream_t s = as_stream(stream);
  FfnArgs a;
  a.x = x; a.sorted_pair = sorted_pair; a.offsets = offsets;
  a.bank = static_cast<const uint8_t *>(bank); a.expert_slot = expert_slot;
  a.rec = record_bytes; a.n_slots = n_slots;
  a.T = T; a.k = k; a.E = E; a.H = H; a.I = I;
  a.off_gq = L.gate_q; a.off_uq = L.up_q; a.off_dq = L.down_q;
  a.off_gs = L.gate_s; a.off_us = L.up_s; a.off_ds = L.down_s;
  a.err = static_cast<int32_t *>(ws);
  a.h = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + WS_HEADER);
  a.xs = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + WS_HEADER +
                                      round256(size_t(T) * size_t(k) * size_t(I) * 2));
  a.x_f16 = x_f16;
  a.x16 = x_f16 ? const_cast<uint16_t *>(x) : a.xs;
  a.y = y;
  a.stall = 0;
  a.e0 = 0;
  a.compact = 0;
  if (T == 0) return MOE_OK;
  if (path == MOE_PATH_SEQUENTIAL) return launch_ffn_sequential(a, s);

  if (may_use_tc(T, k, E, path)) {
    a.stall = take_tc_stall();
    st = launch_ffn_tc(a, s);
    if (st != MOE_ERR_UNSUPPORTED || path == MOE_PATH_TC) return st;
  }
  return launch_ffn_gemv(a, s);
}
