// A5 + A6, decode-sized groups: a weight-streaming grouped GEMV on the
// warp-level tensor-core MMA (mma.sync m16n8k16, FP16 in, fp32 out).
//
// A warp owns 32 (gate/up: two 16-row slices of both matrices) or 64 (down:
// four slices) output rows of one expert and walks K one 128-wide
// quantisation group at a time. Lane (g, t) =
// (lane/4, lane%4) copies 16 bytes (32 codes) of rows g, g+8, g+16 and g+24
// per matrix: the group's four lanes read 64 contiguous bytes of each row.
// The codes never leave registers once read: each packed word turns into four
// FP16x2 code pairs (exact integers) used directly as A fragments. Because a
// dot product does not depend on the order of its K terms, lane t's fragment
// slots are bound to ITS OWN 32 consecutive k of the group (not the PTX
// fragment's k order); the B fragment (the tokens' activations, FP16 copies,
// or h in the down pass) is loaded with the same binding, so lane t reads 64
// contiguous bytes of each token row, and one B fragment feeds every MMA tile
// of the warp (four in gate/up and in down). The fp32 sum of q*x over one
// group is then multiplied by that row's group scale, so the dequantised
// weight q*s is never rounded.
//
// The codes stream through a per-warp shared-memory ring filled by cp.async,
// DEPTH - 1 groups ahead of the math (4 KB slots, 2 deep), while each group's
// B fragment and scales are loaded one group ahead into registers. Each lane copies, and later reads back, only its
// own 16-byte pieces, so its own cp.async waits suffice.
//
// Why FP16 operands: unpacking codes costs integer instructions, and FP16's
// 10-bit mantissa lets a nibble sit at bits 4-7 of a half: one LOP3 yields
// (1024 + u) and another (1024 + 16u) for the next code, with no shift. Codes
// are exact in FP16. A BF16 value v is exact in FP16 when 2^-17 <= |v| <=
// 65504 (or v = 0); a smaller one rounds to a multiple of 2^-24 (an absolute
// error of at most 2^-25), and a larger one does not fit: the FP16 copy of x
// and the h store flag MOE_DEVERR_RANGE for it.
#include <cmath>

#include "ffn.cuh"

namespace moe {

constexpr int GV_WARPS = 4;  // per CTA: 128 rows, or 128 / KS with a K split
constexpr int GV_DEPTH_DOWN = 2;    // down: ring slots (groups of codes) per warp, 4 KB each
constexpr int GV_DEPTH_GATEUP = 2;  // gate/up: ring slots per warp, 4 KB each

// 16-byte asynchronous copy global -> shared, cached in L2 only.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
// The same copy with an L2 eviction-priority policy from createpolicy.
__device__ __forceinline__ void cp_async16_hint(void *dst, const void *src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "l"(policy)
               : "memory");
}
// Codes are read exactly once per call: marking them evict-first keeps the
// small, reused data (activations, h, scales) resident in L2 instead.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t x, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(magic));  // (x & mask) | magic
  return r;
}

// One packed word -> FP16x2 code pairs (q_{2i}, q_{2i+1}), i = 0..3. The word
// holds k = 2i + h at bits 4(i + 4h): nibbles at bits 0-3/16-19 are pair 0,
// 4-7/20-23 pair 1; after one right shift by 8, pairs 2 and 3 sit at the same
// places. Low nibbles: (1024 + u) - 1032 = u - 8. High nibbles: (1024 + 16u)
// / 16 - 72 = u - 8. Every step is exact in FP16. This is the published
// fast int4 -> FP16 conversion by exponent-field insertion (Kim et al., 2022,
// "Who Says Elephants Can't Run: Bringing Large Scale MoE Models into Cloud
// Scale Production", the method FasterTransformer's int4 kernels use), here
// applied to this library's own interleaved word layout.
__device__ __forceinline__ void dequant_codes_f16(uint32_t w, uint32_t (&q)[4]) {
  const __half2 lo_bias = __floats2half2_rn(1032.0f, 1032.0f);
  const __half2 hi_scale = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 hi_bias = __floats2half2_rn(-72.0f, -72.0f);
  const uint32_t w8 = w >> 8;
  uint32_t t0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  uint32_t t1 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  uint32_t t2 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
  uint32_t t3 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
  __half2 v0 = __hsub2(*reinterpret_cast<__half2 *>(&t0), lo_bias);
  __half2 v1 = __hfma2(*reinterpret_cast<__half2 *>(&t1), hi_scale, hi_bias);
  __half2 v2 = __hsub2(*reinterpret_cast<__half2 *>(&t2), lo_bias);
  __half2 v3 = __hfma2(*reinterpret_cast<__half2 *>(&t3), hi_scale, hi_bias);
  q[0] = *reinterpret_cast<uint32_t *>(&v0);
  q[1] = *reinterpret_cast<uint32_t *>(&v1);
  q[2] = *reinterpret_cast<uint32_t *>(&v2);
  q[3] = *reinterpret_cast<uint32_t *>(&v3);
}

// One packed word of rows g (w0) and g+8 (w1) against the lane's 8 activations
// (xb: FP16 pairs k 0-1, 2-3, 4-5, 6-7 of the word): two MMA k-steps.
__device__ __forceinline__ void mma_word(float (&acc)[4], uint32_t w0, uint32_t w1, const uint4 &xb) {
  uint32_t q0[4], q1[4];
  dequant_codes_f16(w0, q0);
  dequant_codes_f16(w1, q1);
  mma_16816(acc, q0[0], q1[0], q0[1], q1[1], xb.x, xb.y);
  mma_16816(acc, q0[2], q1[2], q0[3], q1[3], xb.z, xb.w);
}

__device__ __forceinline__ void mma_group(float (&acc)[4], const uint4 &w0, const uint4 &w1, const uint4 (&xb)[4]) {
  mma_word(acc, w0.x, w1.x, xb[0]);
  mma_word(acc, w0.y, w1.y, xb[1]);
  mma_word(acc, w0.z, w1.z, xb[2]);
  mma_word(acc, w0.w, w1.w, xb[3]);
}

// gate/up + SwiGLU: h[r][row] for the expert's rows r. A warp owns 32 rows
// (two 16-row slices side by side) of both matrices: per 128-wide group it
// copies 4 KB of codes (rows g, g+8, g+16, g+24 of gate and of up) and runs
// four MMA tiles on one x fragment, which it loads one group ahead with the
// group's eight scales. KS warps share a slice pair and split its groups
// (group % KS == the warp's index) when there are few active experts; their
// partial sums meet in shared memory. h is the BF16-rounded value stored as
// FP16 (exact), the down pass's B. (One slice per warp with a 4-deep ring,
// and two slices with a 3-deep ring, measured 2-8 % slower.)
// The expert of this CTA: grid row blockIdx.y (+ e0), or, on a compact grid
// (few (token, expert) pairs against many experts, most of them without rows),
// the blockIdx.y-th expert that has rows, found by warp 0 from the group
// offsets; -1 past the last one. Every thread of the CTA calls it.
__device__ __forceinline__ int cta_expert(const FfnArgs &a) {
  if (!a.compact) return int(blockIdx.y) + a.e0;
  __shared__ int s_expert;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int seen = 0, found = -1;
    for (int e0 = 0; e0 < a.E && found < 0; e0 += 32) {  // warp-uniform loop
      const int e = e0 + lane;
      const unsigned m = __ballot_sync(0xffffffffu, e < a.E && a.offsets[e + 1] > a.offsets[e]);
      const int want = int(blockIdx.y) - seen;
      if (want < __popc(m)) {
        unsigned mm = m;
        for (int i = 0; i < want; ++i) mm &= mm - 1;  // drop the lowest `want` set bits
        found = e0 + __ffs(int(mm)) - 1;
      }
      seen += __popc(m);
    }
    if (lane == 0) s_expert = found;
  }
  __syncthreads();
  return s_expert;
}

template <int KS>
__global__ void __launch_bounds__(GV_WARPS * 32) gemv_gateup_kernel(const FfnArgs a) {
  __shared__ float red[KS > 1 ? KS - 1 : 1][GV_WARPS / KS][KS > 1 ? 16 : 1][32];
  __shared__ uint4 rings[GV_WARPS][GV_DEPTH_GATEUP * 8 * 32];  // [slot][gate g, g+8, g+16, g+24, up ...][lane]
  pdl_trigger();
  pdl_wait();
  const int e = cta_expert(a);
  if (e < 0) return;
  const int lo = a.offsets[e], cnt = a.offsets[e + 1] - lo;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int sl = warp / KS, kq = warp % KS;
  const int row0 = (blockIdx.x * (GV_WARPS / KS) + sl) * 32;
  if (blockIdx.x * (GV_WARPS / KS) * 32 >= a.I) return;
  const bool rows_ok = row0 < a.I;  // I is a multiple of 128, so then all 32 rows are
  const uint8_t *rec = expert_record(a, e);
  if (!rec) return;
  const uint64_t stream_policy = l2_evict_first_policy();
  const int H = a.H, KB = H / 2, G = H / GROUP;
  const int rr = rows_ok ? row0 + g : 0;
  const uint8_t *gq0 = rec + a.off_gq + int64_t(rr) * KB + t * 16;
  const uint8_t *uq0 = rec + a.off_uq + int64_t(rr) * KB + t * 16;
  const uint16_t *gs = reinterpret_cast<const uint16_t *>(rec + a.off_gs) + int64_t(rr) * G;
  const uint16_t *us = reinterpret_cast<const uint16_t *>(rec + a.off_us) + int64_t(rr) * G;

  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool ok = n0 + g < cnt;
    const int token = ok ? a.sorted_pair[lo + n0 + g] / a.k : 0;
    const uint16_t *xr = a.x16 + int64_t(token) * H + t * 32;
    float ag[2][4] = {}, au[2][4] = {};
    const int ngrp = rows_ok && kq < G ? (G - 1 - kq) / KS + 1 : 0;
    uint4 *ring = rings[warp];
    auto issue = [&](int i) {
      const int grp = kq + i * KS;
      uint4 *d = ring + (i % GV_DEPTH_GATEUP) * (8 * 32) + lane;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        cp_async16_hint(d + 32 * r, gq0 + r * 8 * KB + grp * 64, stream_policy);
        cp_async16_hint(d + 128 + 32 * r, uq0 + r * 8 * KB + grp * 64, stream_policy);
      }
    };
#pragma unroll
    for (int i = 0; i < GV_DEPTH_GATEUP - 1; ++i) {
      if (i < ngrp) issue(i);
      cp_async_commit();
    }
    uint4 xn[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      xn[q] = ok && ngrp > 0 ? __ldg(reinterpret_cast<const uint4 *>(xr + kq * GROUP) + q) : make_uint4(0, 0, 0, 0);
    uint32_t sgn[2] = {0, 0}, sun[2] = {0, 0};  // BF16 scale pairs: rows (g, g+8), (g+16, g+24)
    auto load_s = [&](int grp) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        sgn[h] = uint32_t(gs[16 * h * G + grp]) | (uint32_t(gs[(16 * h + 8) * G + grp]) << 16);
        sun[h] = uint32_t(us[16 * h * G + grp]) | (uint32_t(us[(16 * h + 8) * G + grp]) << 16);
      }
    };
    if (ngrp > 0) load_s(kq);
    for (int i = 0; i < ngrp; ++i) {
      const int grp = kq + i * KS;
      if (i + GV_DEPTH_GATEUP - 1 < ngrp) issue(i + GV_DEPTH_GATEUP - 1);
      cp_async_commit();
      uint4 xb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) xb[q] = xn[q];
      const uint32_t sg[2] = {sgn[0], sgn[1]}, su[2] = {sun[0], sun[1]};
      if (i + 1 < ngrp) {
        load_s(grp + KS);
        if (ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) xn[q] = __ldg(reinterpret_cast<const uint4 *>(xr + (grp + KS) * GROUP) + q);
        }
      }
      cp_async_wait<GV_DEPTH_GATEUP - 1>();  // group i's copies (this lane's) have landed
      const uint4 *sr = ring + (i % GV_DEPTH_GATEUP) * (8 * 32) + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float pg[4] = {0.f, 0.f, 0.f, 0.f}, pu[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group(pg, sr[64 * h], sr[64 * h + 32], xb);
        mma_group(pu, sr[128 + 64 * h], sr[128 + 64 * h + 32], xb);
        const float g0 = bf16_lo(sg[h]), g1 = bf16_hi(sg[h]), u0 = bf16_lo(su[h]), u1 = bf16_hi(su[h]);
        ag[h][0] = fmaf(g0, pg[0], ag[h][0]); ag[h][1] = fmaf(g0, pg[1], ag[h][1]);
        ag[h][2] = fmaf(g1, pg[2], ag[h][2]); ag[h][3] = fmaf(g1, pg[3], ag[h][3]);
        au[h][0] = fmaf(u0, pu[0], au[h][0]); au[h][1] = fmaf(u0, pu[1], au[h][1]);
        au[h][2] = fmaf(u1, pu[2], au[h][2]); au[h][3] = fmaf(u1, pu[3], au[h][3]);
      }
    }
    if (KS > 1) {
      __syncthreads();
      if (kq > 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 4; ++c) { red[kq - 1][sl][8 * h + c][lane] = ag[h][c]; red[kq - 1][sl][8 * h + 4 + c][lane] = au[h][c]; }
      }
      __syncthreads();
      if (kq == 0) {
#pragma unroll
        for (int q = 0; q < KS - 1; ++q)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 4; ++c) { ag[h][c] += red[q][sl][8 * h + c][lane]; au[h][c] += red[q][sl][8 * h + 4 + c][lane]; }
      }
    }
    bool bad = false;  // an h outside FP16's finite range cannot be the down pass's operand
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int r = n0 + 2 * t + c;
      if (kq == 0 && rows_ok && r < cnt) {
        uint16_t *hr = a.h + int64_t(lo + r) * a.I + row0 + g;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float v0 = bf16_to_f(f_to_bf16(silu_f(ag[h][c]) * au[h][c]));
          const float v1 = bf16_to_f(f_to_bf16(silu_f(ag[h][2 + c]) * au[h][2 + c]));
          bad |= fabsf(v0) > 65504.f || fabsf(v1) > 65504.f;
          hr[16 * h] = __half_as_ushort(__float2half_rn(v0));
          hr[16 * h + 8] = __half_as_ushort(__float2half_rn(v1));
        }
      }
    }
    if (bad) flag_error(a.err, MOE_DEVERR_RANGE);
  }
}

// down: y[r][row] = h[r] . Wd[row] (fp32). A warp owns DOWN_RS = 4 16-row
// slices side by side (64 output rows): per 128-wide group it copies 16 bytes
// of each of its rows g + 8j (4 KB per warp) and runs all four slices' MMAs
// on the same h fragment, which it loads one group ahead with the group's
// scales. KS warps split the groups of a slice set as in the gate/up pass.
// (Two slices per warp with a 4-deep ring measured 5 % slower at T = 16, one
// slice per warp 3-10 % slower still.)
constexpr int DOWN_RS = 4;
template <int KS>
__global__ void __launch_bounds__(GV_WARPS * 32) gemv_down_kernel(const FfnArgs a) {
  constexpr int RS = DOWN_RS, NP = 2 * RS, DEPTH = GV_DEPTH_DOWN;  // NP: 16-byte pieces per lane per group
  __shared__ float red[KS > 1 ? KS - 1 : 1][GV_WARPS / KS][KS > 1 ? 4 * RS : 1][32];
  __shared__ uint4 rings[GV_WARPS][DEPTH * NP * 32];  // [slot][piece: rows g, g+8, g+16, ...][lane]
  pdl_trigger();
  pdl_wait();
  const int e = cta_expert(a);
  if (e < 0) return;
  const int lo = a.offsets[e], cnt = a.offsets[e + 1] - lo;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int sl = warp / KS, kq = warp % KS;  // slice set within the CTA, K part
  const int row0 = (blockIdx.x * (GV_WARPS / KS) + sl) * 16 * RS;
  if (blockIdx.x * (GV_WARPS / KS) * 16 * RS >= a.H) return;  // whole CTA out of range (uniform)
  const bool rows_ok = row0 < a.H;  // H is a multiple of 128, a multiple of 16 * RS: then all 64 rows are
  const uint8_t *rec = expert_record(a, e);
  if (!rec) return;
  const int I = a.I, KB = I / 2, G = I / GROUP;
  const int rr = rows_ok ? row0 + g : 0;
  const uint8_t *dq0 = rec + a.off_dq + int64_t(rr) * KB + t * 16;
  const uint16_t *ds = reinterpret_cast<const uint16_t *>(rec + a.off_ds) + int64_t(rr) * G;

  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool ok = n0 + g < cnt;
    const uint16_t *hr = a.h + int64_t(lo + (ok ? n0 + g : 0)) * I + t * 32;
    float acc[RS][4] = {};
    const int ngrp = rows_ok && kq < G ? (G - 1 - kq) / KS + 1 : 0;
    uint4 *ring = rings[warp];
    auto issue = [&](int i) {
      const int grp = kq + i * KS;
      uint4 *d = ring + (i % DEPTH) * (NP * 32) + lane;
#pragma unroll
      for (int j = 0; j < NP; ++j) cp_async16(d + 32 * j, dq0 + j * 8 * KB + grp * 64);
    };
#pragma unroll
    for (int i = 0; i < DEPTH - 1; ++i) {
      if (i < ngrp) issue(i);
      cp_async_commit();
    }
    uint4 xn[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      xn[q] = ok && ngrp > 0 ? *(reinterpret_cast<const uint4 *>(hr + kq * GROUP) + q) : make_uint4(0, 0, 0, 0);
    uint32_t sn[RS];  // BF16 scale pairs of rows (g + 16 s, g + 16 s + 8)
    auto load_s = [&](int grp) {
#pragma unroll
      for (int r = 0; r < RS; ++r)
        sn[r] = uint32_t(ds[16 * r * G + grp]) | (uint32_t(ds[(16 * r + 8) * G + grp]) << 16);
    };
    if (ngrp > 0) load_s(kq);
    for (int i = 0; i < ngrp; ++i) {
      const int grp = kq + i * KS;
      if (i + DEPTH - 1 < ngrp) issue(i + DEPTH - 1);
      cp_async_commit();
      uint4 xb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) xb[q] = xn[q];
      uint32_t sc[RS];
#pragma unroll
      for (int r = 0; r < RS; ++r) sc[r] = sn[r];
      if (i + 1 < ngrp) {
        load_s(grp + KS);
        if (ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) xn[q] = *(reinterpret_cast<const uint4 *>(hr + (grp + KS) * GROUP) + q);
        }
      }
      cp_async_wait<DEPTH - 1>();  // group i's copies (this lane's) have landed
      const uint4 *sr = ring + (i % DEPTH) * (NP * 32) + lane;
#pragma unroll
      for (int r = 0; r < RS; ++r) {
        float p[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group(p, sr[64 * r], sr[64 * r + 32], xb);
        const float c0 = bf16_lo(sc[r]), c1 = bf16_hi(sc[r]);
        acc[r][0] = fmaf(c0, p[0], acc[r][0]); acc[r][1] = fmaf(c0, p[1], acc[r][1]);
        acc[r][2] = fmaf(c1, p[2], acc[r][2]); acc[r][3] = fmaf(c1, p[3], acc[r][3]);
      }
    }
    if (KS > 1) {  // K parts 1.. hand their sums to part 0 of the slice set
      __syncthreads();
      if (kq > 0) {
#pragma unroll
        for (int r = 0; r < RS; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) red[kq - 1][sl][4 * r + c][lane] = acc[r][c];
      }
      __syncthreads();
      if (kq == 0) {
#pragma unroll
        for (int q = 0; q < KS - 1; ++q)
#pragma unroll
          for (int r = 0; r < RS; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] += red[q][sl][4 * r + c][lane];
      }
    }
    // accumulator (c0, c1) = row g, tokens 2t, 2t+1; (c2, c3) = row g+8
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int r = n0 + 2 * t + c;
      if (kq == 0 && rows_ok && r < cnt) {
        float *yr = a.y + int64_t(lo + r) * a.H + row0 + g;
#pragma unroll
        for (int s = 0; s < RS; ++s) {
          yr[16 * s] = acc[s][c];
          yr[16 * s + 8] = acc[s][2 + c];
        }
      }
    }
  }
}

template <int KS>
static cudaError_t launch_gemv_pair(const FfnArgs &a0, cudaStream_t s) {
  // with at most E/4 (token, expert) pairs, most experts have no rows: the
  // grid then has one row per possible active expert instead of one per
  // expert, so no wave of empty CTAs stands between the others and the SMs
  // (one-token decode step 0.453 -> 0.404 ms; at E/2 pairs the experts' scan
  // in every CTA cost more than it saved, 0.654 -> 0.661 ms)
  FfnArgs a = a0;
  const int64_t pairs = int64_t(a.T) * a.k;
  a.compact = pairs * 4 <= a.E;
  const unsigned ny = unsigned(a.compact ? pairs : a.E);
  const int rows_per_cta = (GV_WARPS / KS) * 16;
  dim3 g1((a.I + rows_per_cta * 2 - 1) / (rows_per_cta * 2), ny);  // two slices per warp
  cudaError_t e = launch_pdl(gemv_gateup_kernel<KS>, g1, dim3(GV_WARPS * 32), 0, s, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  // the down pass splits K half as far as gate/up when KS = 4 on a full grid
  // (a four-token step: 0.655 -> 0.636 ms); at one token, and at KS = 2, the
  // same split as gate/up measured best (halving it: 0.403 -> 0.429 ms at
  // T = 1, and 1.388 -> 1.434 ms at T = 64)
  if (KS == 4 && !a.compact) {
    const int rpd = (GV_WARPS / 2) * 16;
    dim3 g2((a.H + rpd * DOWN_RS - 1) / (rpd * DOWN_RS), ny);  // DOWN_RS slices per warp
    e = launch_pdl(gemv_down_kernel<2>, g2, dim3(GV_WARPS * 32), 0, s, a);
  } else {
    dim3 g2((a.H + rows_per_cta * DOWN_RS - 1) / (rows_per_cta * DOWN_RS), ny);  // DOWN_RS slices per warp
    e = launch_pdl(gemv_down_kernel<KS>, g2, dim3(GV_WARPS * 32), 0, s, a);
  }
  if (e == cudaSuccess) count_launches(1);
  return e;
}

// Warps that share a 32-row slice pair, from the expected number of active
// experts E (1 - (1 - k/E)^T): enough warps to keep every SM streaming when a
// decode step touches few experts (same-box measurements on the OLMoE decode
// stack chose the thresholds; at T = 16 two warps per pair gave the same FFN
// time as one but a 2 us shorter layer step, the FFN overlapping its
// neighbours better).
static int pick_ksplit(const FfnArgs &a) {
  const double miss = 1.0 - double(a.k) / double(a.E);
  double n_act = double(a.E) * (1.0 - std::pow(miss, double(a.T)));
  if (n_act < 1.0) n_act = 1.0;
  const double warps = n_act * (a.I / 32);  // one warp per slice pair of every active expert
  const double want = 148.0 * 24.0;
  // with 4+ rows per expert on average (several token chunks per CTA) two
  // warps per slice shorten each CTA's life enough to pay for the reduction
  const bool many_rows = int64_t(a.T) * a.k >= 4 * int64_t(a.E);
  return warps * 2 <= want ? 4 : (warps * 1.25 <= want || many_rows ? 2 : 1);
}

// The sequential reference (the per-expert W4 baseline of the pages, Abstract):
// the same kernels launched once per expert, gate/up then down, expert after
// expert, each launch covering one expert's rows with the widest K split.
// Experts without rows still get their (empty) launches: the host does not
// know the group sizes without a synchronisation.
int launch_ffn_sequential(const FfnArgs &a, cudaStream_t s) {
  int st = launch_x_to_f16(a, s);
  if (st != MOE_OK) return st;
  constexpr int KS = 4;
  const int rows_per_cta = (GV_WARPS / KS) * 16;
  for (int e = 0; e < a.E; ++e) {
    FfnArgs b = a;
    b.e0 = e;
    cudaError_t err =
        launch_pdl(gemv_gateup_kernel<KS>, dim3((a.I + rows_per_cta * 2 - 1) / (rows_per_cta * 2), 1),
                   dim3(GV_WARPS * 32), 0, s, b);
    if (err == cudaSuccess) {
      count_launches(1);
      err = launch_pdl(gemv_down_kernel<KS>, dim3((a.H + rows_per_cta * DOWN_RS - 1) / (rows_per_cta * DOWN_RS), 1),
                       dim3(GV_WARPS * 32), 0, s, b);
    }
    if (err != cudaSuccess)
      return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (sequential): %s", cudaGetErrorString(err));
    count_launches(1);
  }
  return check_launch("moe_grouped_w4a16_ffn (sequential)", 0);
}

int launch_ffn_gemv(const FfnArgs &a, cudaStream_t s) {
  int st = launch_x_to_f16(a, s);
  if (st != MOE_OK) return st;
  const int ks = pick_ksplit(a);
  const cudaError_t e = ks == 4 ? launch_gemv_pair<4>(a, s) : ks == 2 ? launch_gemv_pair<2>(a, s) : launch_gemv_pair<1>(a, s);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (gemv): %s", cudaGetErrorString(e));
  return check_launch("moe_grouped_w4a16_ffn (gemv)", 0);
}

}  // namespace moe
