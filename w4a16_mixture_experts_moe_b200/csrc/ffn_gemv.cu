// A5 + A6, decode-sized groups: a weight-streaming grouped GEMV on the
// warp-level tensor-core MMA (mma.sync m16n8k16, BF16 in, fp32 out).
//
// A warp owns 16 output rows of one expert and walks K one 128-wide
// quantisation group at a time. Lane (g, t) = (lane/4, lane%4) loads 16 bytes
// (32 codes) of rows g and g+8 per matrix: the group's four lanes read 64
// contiguous bytes of each row. The codes never leave registers: each packed
// word turns into four BF16x2 code pairs (exact integers) that are used
// directly as A fragments. Because a dot product does not depend on the order
// of its K terms, lane t's fragment slots are bound to ITS OWN 32 consecutive
// k of the group (not the PTX fragment's k order); the B fragment (the
// token's activations) is loaded with the same binding, so lane t reads 64
// contiguous bytes of each token row. The fp32 sum of q*x over one group is
// then multiplied by that row's group scale, so the dequantised weight q*s is
// never rounded.
#include "ffn.cuh"

namespace moe {

constexpr int GV_WARPS = 4;  // 64 rows per CTA

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One packed word of rows g (w0) and g+8 (w1) against the lane's 8 activations
// (xb: BF16 pairs k 0-1, 2-3, 4-5, 6-7 of the word): two MMA k-steps.
__device__ __forceinline__ void mma_word(float (&acc)[4], uint32_t w0, uint32_t w1, const uint4 &xb) {
  uint32_t q0[4], q1[4];
  dequant_codes(w0, q0);
  dequant_codes(w1, q1);
  mma_16816(acc, q0[0], q1[0], q0[1], q1[1], xb.x, xb.y);
  mma_16816(acc, q0[2], q1[2], q0[3], q1[3], xb.z, xb.w);
}

__device__ __forceinline__ void mma_group(float (&acc)[4], const uint4 &w0, const uint4 &w1, const uint4 (&xb)[4]) {
  mma_word(acc, w0.x, w1.x, xb[0]);
  mma_word(acc, w0.y, w1.y, xb[1]);
  mma_word(acc, w0.z, w1.z, xb[2]);
  mma_word(acc, w0.w, w1.w, xb[3]);
}

// gate/up + SwiGLU: h[r][row] for the expert's rows r, 16 features per warp.
__global__ void __launch_bounds__(GV_WARPS * 32) gemv_gateup_kernel(const FfnArgs a) {
  const int e = blockIdx.y;
  const int lo = a.offsets[e], cnt = a.offsets[e + 1] - lo;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row0 = (blockIdx.x * GV_WARPS + warp) * 16;
  if (row0 >= a.I) return;
  const uint8_t *rec = expert_record(a, e);
  if (!rec) return;
  const int H = a.H, KB = H / 2, G = H / GROUP;
  const uint8_t *gq0 = rec + a.off_gq + int64_t(row0 + g) * KB + t * 16;
  const uint8_t *uq0 = rec + a.off_uq + int64_t(row0 + g) * KB + t * 16;
  const uint16_t *gs = reinterpret_cast<const uint16_t *>(rec + a.off_gs) + int64_t(row0 + g) * G;
  const uint16_t *us = reinterpret_cast<const uint16_t *>(rec + a.off_us) + int64_t(row0 + g) * G;

  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool ok = n0 + g < cnt;
    const int token = ok ? a.sorted_pair[lo + n0 + g] / a.k : 0;
    const uint16_t *xr = a.x + int64_t(token) * H + t * 32;
    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
    for (int grp = 0; grp < G; ++grp) {
      const uint4 g0 = ld_stream(gq0 + grp * 64), g1 = ld_stream(gq0 + 8 * KB + grp * 64);
      const uint4 u0 = ld_stream(uq0 + grp * 64), u1 = ld_stream(uq0 + 8 * KB + grp * 64);
      uint4 xb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        xb[q] = ok ? __ldg(reinterpret_cast<const uint4 *>(xr + grp * GROUP) + q) : make_uint4(0, 0, 0, 0);
      float pg[4] = {0.f, 0.f, 0.f, 0.f}, pu[4] = {0.f, 0.f, 0.f, 0.f};
      mma_group(pg, g0, g1, xb);
      mma_group(pu, u0, u1, xb);
      const float sg0 = bf16_to_f(gs[grp]), sg1 = bf16_to_f(gs[8 * G + grp]);
      const float su0 = bf16_to_f(us[grp]), su1 = bf16_to_f(us[8 * G + grp]);
      ag[0] = fmaf(sg0, pg[0], ag[0]); ag[1] = fmaf(sg0, pg[1], ag[1]);
      ag[2] = fmaf(sg1, pg[2], ag[2]); ag[3] = fmaf(sg1, pg[3], ag[3]);
      au[0] = fmaf(su0, pu[0], au[0]); au[1] = fmaf(su0, pu[1], au[1]);
      au[2] = fmaf(su1, pu[2], au[2]); au[3] = fmaf(su1, pu[3], au[3]);
    }
    // accumulator (c0, c1) = row g, tokens 2t, 2t+1; (c2, c3) = row g+8
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int r = n0 + 2 * t + c;
      if (r < cnt) {
        uint16_t *hr = a.h + int64_t(lo + r) * a.I + row0 + g;
        hr[0] = f_to_bf16(silu_f(ag[c]) * au[c]);
        hr[8] = f_to_bf16(silu_f(ag[2 + c]) * au[2 + c]);
      }
    }
  }
}

// down: y[r][row] = h[r] . Wd[row], 16 output features per warp.
__global__ void __launch_bounds__(GV_WARPS * 32) gemv_down_kernel(const FfnArgs a) {
  const int e = blockIdx.y;
  const int lo = a.offsets[e], cnt = a.offsets[e + 1] - lo;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int row0 = (blockIdx.x * GV_WARPS + warp) * 16;
  if (row0 >= a.H) return;
  const uint8_t *rec = expert_record(a, e);
  if (!rec) return;
  const int I = a.I, KB = I / 2, G = I / GROUP;
  const uint8_t *dq0 = rec + a.off_dq + int64_t(row0 + g) * KB + t * 16;
  const uint16_t *ds = reinterpret_cast<const uint16_t *>(rec + a.off_ds) + int64_t(row0 + g) * G;

  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool ok = n0 + g < cnt;
    const uint16_t *hr = a.h + int64_t(lo + (ok ? n0 + g : 0)) * I + t * 32;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int grp = 0; grp < G; ++grp) {
      const uint4 w0 = ld_stream(dq0 + grp * 64), w1 = ld_stream(dq0 + 8 * KB + grp * 64);
      uint4 xb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        xb[q] = ok ? *(reinterpret_cast<const uint4 *>(hr + grp * GROUP) + q) : make_uint4(0, 0, 0, 0);
      float p[4] = {0.f, 0.f, 0.f, 0.f};
      mma_group(p, w0, w1, xb);
      const float s0 = bf16_to_f(ds[grp]), s1 = bf16_to_f(ds[8 * G + grp]);
      acc[0] = fmaf(s0, p[0], acc[0]); acc[1] = fmaf(s0, p[1], acc[1]);
      acc[2] = fmaf(s1, p[2], acc[2]); acc[3] = fmaf(s1, p[3], acc[3]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int r = n0 + 2 * t + c;
      if (r < cnt) {
        float *yr = a.y + int64_t(lo + r) * a.H + row0 + g;
        yr[0] = acc[c];
        yr[8] = acc[2 + c];
      }
    }
  }
}

int launch_ffn_gemv(const FfnArgs &a, cudaStream_t s) {
  const int rows_per_cta = GV_WARPS * 16;
  dim3 g1((a.I + rows_per_cta - 1) / rows_per_cta, a.E);
  gemv_gateup_kernel<<<g1, GV_WARPS * 32, 0, s>>>(a);
  int st = check_launch("moe_grouped_w4a16_ffn (gemv gate/up)");
  if (st != MOE_OK) return st;
  dim3 g2((a.H + rows_per_cta - 1) / rows_per_cta, a.E);
  gemv_down_kernel<<<g2, GV_WARPS * 32, 0, s>>>(a);
  return check_launch("moe_grouped_w4a16_ffn (gemv down)");
}

}  // namespace moe
