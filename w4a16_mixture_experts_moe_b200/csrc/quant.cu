// A1 — symmetric group-128 int4 quantisation and packing, run once offline
// (ExactMoE paper, Abstract: group-128 four-bit weights for the routed
// experts; Figure 1 caption: packing happens a single time, into the form
// the kernels read).
//
// One warp per (expert, row, 128-group). Lane l holds k = 4l .. 4l+3 of the
// group; lanes 2m and 2m+1 together form packed word m of the group.
#include "common.cuh"

namespace moe {

__device__ __forceinline__ uint32_t quant_code(float v, float s) {
  if (s == 0.0f) return 8u;                      // all-zero group: q = 0
  float r = rintf(__fdiv_rn(v, s));              // IEEE fp32 divide, ties to even
  r = fminf(fmaxf(r, -8.0f), 7.0f);
  return uint32_t(int(r) + 8);                   // offset-binary nibble
}

__global__ void __launch_bounds__(256) quantize_pack_kernel(
    const uint16_t *__restrict__ w, int E, int N, int K, uint8_t *__restrict__ packed,
    int64_t packed_stride, uint8_t *__restrict__ scales, int64_t scales_stride) {
  const int G = K / GROUP;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = int64_t(E) * N * G;
  if (warp >= total) return;
  const int g = int(warp % G);
  const int64_t en = warp / G;
  const int n = int(en % N);
  const int e = int(en / N);

  const uint2 raw = *reinterpret_cast<const uint2 *>(w + (int64_t(e) * N + n) * K + g * GROUP + lane * 4);
  const float v0 = bf16_lo(raw.x), v1 = bf16_hi(raw.x), v2 = bf16_lo(raw.y), v3 = bf16_hi(raw.y);
  float am = fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3)));
#pragma unroll
  for (int o = 16; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const uint16_t sbits = f_to_bf16(__fdiv_rn(am, 7.0f));
  const float s = bf16_to_f(sbits);

  const uint32_t u0 = quant_code(v0, s), u1 = quant_code(v1, s);
  const uint32_t u2 = quant_code(v2, s), u3 = quant_code(v3, s);
  // k = 2i + h of the word sits at bits 4(i + 4h). The even lane holds word
  // k 0..3 (slots 0, 4, 1, 5), the odd lane k 4..7 (slots 2, 6, 3, 7).
  const uint32_t part = (lane & 1) ? ((u0 << 8) | (u1 << 24) | (u2 << 12) | (u3 << 28))
                                   : (u0 | (u1 << 16) | (u2 << 4) | (u3 << 20));
  const uint32_t word = part | __shfl_xor_sync(0xffffffffu, part, 1);
  if (!(lane & 1)) {
    uint8_t *dst = packed + int64_t(e) * packed_stride + int64_t(n) * (K / 2) + g * (GROUP / 2) + (lane >> 1) * 4;
    *reinterpret_cast<uint32_t *>(dst) = word;
  }
  if (lane == 0) {
    uint16_t *sd = reinterpret_cast<uint16_t *>(scales + int64_t(e) * scales_stride) + int64_t(n) * G + g;
    *sd = sbits;
  }
}

}  // namespace moe

extern "C" int moe_quantize_pack(const moe_bf16 *w, int E, int N, int K, uint8_t *packed,
                                 int64_t packed_stride, moe_bf16 *scales, int64_t scales_stride,
                                 moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_quantize_pack");
  using namespace moe;
  if (!w || !packed || !scales) return set_error(MOE_ERR_INVALID_ARG, "moe_quantize_pack: NULL pointer");
  if (E < 1 || N < 1 || K < GROUP || K % GROUP)
    return set_error(MOE_ERR_SHAPE, "moe_quantize_pack: E=%d N=%d K=%d (need E,N >= 1, K a positive multiple of 128)", E, N, K);
  const int64_t need_p = int64_t(N) * K / 2, need_s = int64_t(N) * (K / GROUP) * 2;
  if (E > 1 && (packed_stride < need_p || scales_stride < need_s))
    return set_error(MOE_ERR_INVALID_ARG, "moe_quantize_pack: expert strides smaller than one expert");
  if ((E > 1 && (packed_stride % 4 || scales_stride % 2)) || !aligned(w, 8) || !aligned(packed, 4) ||
      !aligned(scales, 2))
    return set_error(MOE_ERR_INVALID_ARG,
                     "moe_quantize_pack: need w 8-byte, packed 4-byte, scales 2-byte aligned (strides likewise)");
  const int64_t warps = int64_t(E) * N * (K / GROUP);
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return set_error(MOE_ERR_SHAPE, "moe_quantize_pack: too many groups");
  quantize_pack_kernel<<<unsigned(blocks), 256, 0, as_stream(stream)>>>(
      w, E, N, K, packed, packed_stride, reinterpret_cast<uint8_t *>(scales), scales_stride);
  return check_launch("moe_quantize_pack");
}
