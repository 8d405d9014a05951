// The BF16 grouped expert FFN: the same grouped SwiGLU as A5 + A6 with the
// experts kept in BF16 instead of int4 (the pages' BF16 baseline: Abstract and
// Table 1 compare W4A16 decode with the BF16 model). It exists to measure what
// the int4 packing buys on this GPU; it is not on the W4A16 hot path.
//
// Weight-streaming GEMV on the warp-level MMA (mma.sync m16n8k16, BF16 in,
// fp32 out). A CTA of four warps owns 16 output rows of one expert (both gate
// and up rows in the gate/up pass) and splits K four ways: warp w takes the
// 32-wide k-chunks c = w, w+4, ...; the four partial sums meet in shared
// memory. Lane (g, t) = (lane/4, lane%4) loads 16 bytes (8 weights) of rows g
// and g+8 at k = 32c + 8t: a dot product does not depend on the order of its
// terms, so the lane's fragment slots of the two MMAs of a chunk are bound to
// ITS OWN eight consecutive k, and the activations are loaded with the same
// binding (16 bytes of token g's row). Each chunk's loads are issued one
// chunk ahead of its MMAs. h is rounded to BF16 (the A16 intermediate) and
// kept in BF16, the down pass's operand, so no FP16 range applies.
#include "common.cuh"

namespace moe {

constexpr int BF_WARPS = 4;
constexpr int BF_ROWS = 16;  // output rows per CTA

struct Bf16Args {
  const uint16_t *x;           // [T][H]
  const int32_t *sorted_pair;  // [P]
  const int32_t *offsets;      // [E+1]
  const uint8_t *bank;         // records of `rec` bytes
  int64_t rec, off_g, off_u, off_d;
  int T, k, E, H, I;
  uint16_t *h;  // [P][I] BF16, sorted order
  float *y;     // [P][H] fp32, sorted order
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 32-wide k-chunk: rows g (w0) and g+8 (w1) against the lane's 8 k of x.
__device__ __forceinline__ void mma_chunk(float (&acc)[4], const uint4 &w0, const uint4 &w1, const uint4 &xv) {
  mma_bf16_16816(acc, w0.x, w1.x, w0.y, w1.y, xv.x, xv.y);
  mma_bf16_16816(acc, w0.z, w1.z, w0.w, w1.w, xv.z, xv.w);
}

template <bool GATEUP>
__global__ void __launch_bounds__(BF_WARPS * 32) gemv_bf16_kernel(const Bf16Args a) {
  __shared__ float red[BF_WARPS - 1][8][32];
  pdl_trigger();
  pdl_wait();
  const int e = blockIdx.y;
  const int lo = a.offsets[e], cnt = a.offsets[e + 1] - lo;
  if (cnt <= 0) return;
  const int NOUT = GATEUP ? a.I : a.H, KD = GATEUP ? a.H : a.I;
  const int row0 = blockIdx.x * BF_ROWS;
  if (row0 >= NOUT) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint8_t *rec = a.bank + int64_t(e) * a.rec;
  const uint16_t *w0 = reinterpret_cast<const uint16_t *>(rec + (GATEUP ? a.off_g : a.off_d)) +
                       int64_t(row0 + g) * KD + 8 * t;
  const uint16_t *w1 = reinterpret_cast<const uint16_t *>(rec + a.off_u) + int64_t(row0 + g) * KD + 8 * t;
  const int64_t r8 = int64_t(8) * KD;  // row g+8
  const int NC = KD / 32;

  for (int n0 = 0; n0 < cnt; n0 += 8) {
    const bool ok = n0 + g < cnt;
    const uint16_t *xr;
    if (GATEUP) {
      const int token = ok ? a.sorted_pair[lo + n0 + g] / a.k : 0;
      xr = a.x + int64_t(token) * a.H + 8 * t;
    } else {
      xr = a.h + int64_t(lo + (ok ? n0 + g : 0)) * a.I + 8 * t;
    }
    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
    const uint4 zero = make_uint4(0, 0, 0, 0);
    auto ld = [](const uint16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); };
    int c = warp;
    uint4 g0, g1, u0, u1, xv;
    if (c < NC) {
      g0 = ld(w0 + c * 32); g1 = ld(w0 + r8 + c * 32);
      if (GATEUP) { u0 = ld(w1 + c * 32); u1 = ld(w1 + r8 + c * 32); }
      xv = ok ? ld(xr + c * 32) : zero;
    }
    for (; c < NC; c += BF_WARPS) {
      const uint4 cg0 = g0, cg1 = g1, cx = xv;
      uint4 cu0, cu1;
      if (GATEUP) { cu0 = u0; cu1 = u1; }
      const int cn = c + BF_WARPS;
      if (cn < NC) {  // the next chunk's loads go out before this chunk's MMAs
        g0 = ld(w0 + cn * 32); g1 = ld(w0 + r8 + cn * 32);
        if (GATEUP) { u0 = ld(w1 + cn * 32); u1 = ld(w1 + r8 + cn * 32); }
        xv = ok ? ld(xr + cn * 32) : zero;
      }
      mma_chunk(ag, cg0, cg1, cx);
      if (GATEUP) mma_chunk(au, cu0, cu1, cx);
    }
    // the four K parts meet in warp 0
    __syncthreads();
    if (warp > 0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) { red[warp - 1][q][lane] = ag[q]; red[warp - 1][4 + q][lane] = au[q]; }
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int wq = 0; wq < BF_WARPS - 1; ++wq)
#pragma unroll
        for (int q = 0; q < 4; ++q) { ag[q] += red[wq][q][lane]; au[q] += red[wq][4 + q][lane]; }
      // accumulator (c0, c1) = row g, tokens 2t, 2t+1; (c2, c3) = row g+8
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int r = n0 + 2 * t + cc;
        if (r < cnt) {
          if (GATEUP) {
            uint16_t *hr = a.h + int64_t(lo + r) * a.I + row0 + g;
            hr[0] = f_to_bf16(silu_f(ag[cc]) * au[cc]);
            hr[8] = f_to_bf16(silu_f(ag[2 + cc]) * au[2 + cc]);
          } else {
            float *yr = a.y + int64_t(lo + r) * a.H + row0 + g;
            yr[0] = ag[cc];
            yr[8] = ag[2 + cc];
          }
        }
      }
    }
  }
}

}  // namespace moe

extern "C" int moe_bf16_record_layout(int H, int I, moe_bf16_layout *out) {
  using namespace moe;
  if (!out) return set_error(MOE_ERR_INVALID_ARG, "moe_bf16_record_layout: out is NULL");
  if (H < GROUP || I < GROUP || H % GROUP || I % GROUP)
    return set_error(MOE_ERR_SHAPE, "moe_bf16_record_layout: H=%d I=%d must be positive multiples of 128", H, I);
  const int64_t m = (int64_t(H) * I * 2 + 255) / 256 * 256;
  out->gate = 0;
  out->up = m;
  out->down = 2 * m;
  out->bytes = 3 * m;
  return MOE_OK;
}

extern "C" size_t moe_bf16_ffn_workspace_size(int T, int k, int E, int H, int I) {
  (void)E; (void)H;
  if (T < 0 || k < 1 || I < 0) return moe::WS_HEADER;
  return moe::WS_HEADER + (size_t(T) * size_t(k) * size_t(I) * 2 + 255) / 256 * 256;
}

extern "C" int moe_grouped_bf16_ffn(const moe_bf16 *x, const int32_t *sorted_pair, const int32_t *offsets,
                                    const void *bank, int64_t record_bytes, int T, int k, int E, int H, int I,
                                    float *y, void *ws, size_t ws_bytes, moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_grouped_bf16_ffn");
  using namespace moe;
  if (T < 0 || E < 1 || E > MAX_E || k < 1 || k > E || k > MAX_K)
    return set_error(MOE_ERR_SHAPE, "moe_grouped_bf16_ffn: T=%d E=%d k=%d (need T>=0, 1<=E<=256, 1<=k<=min(E,32))",
                     T, E, k);
  moe_bf16_layout L;
  int st = moe_bf16_record_layout(H, I, &L);
  if (st != MOE_OK) return st;
  if (int64_t(T) * k > (int64_t(1) << 30)) return set_error(MOE_ERR_SHAPE, "moe_grouped_bf16_ffn: T*k too large");
  if (!offsets || !bank || !ws || (T > 0 && (!x || !sorted_pair || !y)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_bf16_ffn: NULL pointer");
  if (record_bytes < L.bytes || record_bytes % 256)
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_bf16_ffn: record_bytes=%lld (need >= %lld, multiple of 256)",
                     (long long)record_bytes, (long long)L.bytes);
  if (!aligned(bank, 256) || !aligned(ws, 256) || (T > 0 && (!aligned(x, 16) || !aligned(y, 16))))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_bf16_ffn: bank/ws need 256-byte, x/y 16-byte alignment");
  if (ws_bytes < moe_bf16_ffn_workspace_size(T, k, E, H, I))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_bf16_ffn: workspace %zu B < %zu B", ws_bytes,
                     moe_bf16_ffn_workspace_size(T, k, E, H, I));
  if (T == 0) return MOE_OK;
  Bf16Args a;
  a.x = x; a.sorted_pair = sorted_pair; a.offsets = offsets;
  a.bank = static_cast<const uint8_t *>(bank);
  a.rec = record_bytes; a.off_g = L.gate; a.off_u = L.up; a.off_d = L.down;
  a.T = T; a.k = k; a.E = E; a.H = H; a.I = I;
  a.h = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + WS_HEADER);
  a.y = y;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_pdl(gemv_bf16_kernel<true>, dim3(I / BF_ROWS, E), dim3(BF_WARPS * 32), 0, s, a);
  if (e == cudaSuccess) {
    count_launches(1);
    e = launch_pdl(gemv_bf16_kernel<false>, dim3(H / BF_ROWS, E), dim3(BF_WARPS * 32), 0, s, a);
  }
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_bf16_ffn: %s", cudaGetErrorString(e));
  return check_launch("moe_grouped_bf16_ffn");
}
