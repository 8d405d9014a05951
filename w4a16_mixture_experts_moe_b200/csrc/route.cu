// A2 + A3 — BF16 router logits, full softmax, unchanged top-k
// (ExactMoE paper, Abstract: the router stays BF16 and top-k routing is
// left as it was; Figure 1 caption: the model's own BF16 router picks the
// experts).
//
// One thread-block cluster of 8 CTAs serves TOK tokens (8 for large batches;
// 2 for decode-sized ones, so their few tokens still spread over many SMs).
// CTA rank r computes the logits of experts [r*EPC, (r+1)*EPC)
// (EPC = ceil(E/8)) for all TOK tokens:
// the tokens' activations are staged in shared memory, each warp takes one
// expert at a time with every lane's slice of the router row loaded at once
// (fp32 sums, one BF16 rounding per logit). After a cluster barrier, CTA r
// runs softmax and top-k for token r, reading the other CTAs' logits through
// distributed shared memory; lane l holds experts l, l+32, ... and k rounds of
// a shuffle argmax pick the experts. Splitting the router rows over 8 SMs
// keeps a decode step (T of 1-64) from waiting on one SM's load latency.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

constexpr int RT_CLUSTER = 8;  // CTAs per cluster (at most one token per CTA for top-k)
constexpr int RT_THREADS = 256;
constexpr int RT_MAX_EPC = MAX_E / RT_CLUSTER;

__device__ __forceinline__ bool key_better(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

__device__ __forceinline__ float dot8(const uint4 &w, const uint4 &x, float a) {
  a = fmaf(bf16_lo(w.x), bf16_lo(x.x), a); a = fmaf(bf16_hi(w.x), bf16_hi(x.x), a);
  a = fmaf(bf16_lo(w.y), bf16_lo(x.y), a); a = fmaf(bf16_hi(w.y), bf16_hi(x.y), a);
  a = fmaf(bf16_lo(w.z), bf16_lo(x.z), a); a = fmaf(bf16_hi(w.z), bf16_hi(x.z), a);
  a = fmaf(bf16_lo(w.w), bf16_lo(x.w), a); a = fmaf(bf16_hi(w.w), bf16_hi(x.w), a);
  return a;
}

// Softmax over all E keys and the top-k of one token, by one warp. keys: the
// token's fp32 logits (+ bias, NaN turned into -inf) in shared memory. The
// rank of each key in the order (key descending, expert ascending) is its
// place among the top-k: each lane counts the keys that beat each of its own.
// With MOE_IDS_GIVEN the ids are read and only their weights are written.
__device__ void topk_warp(const float *keys, int E, int k, int flags, int32_t *ids, float *wout, int lane) {
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) mx = fmaxf(mx, keys[e]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int e = lane; e < E; e += 32) sum += expf(keys[e] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  float wsum = 0.f;
  if (flags & MOE_IDS_GIVEN) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[j];
      const float p = (e >= 0 && e < E) ? expf(keys[e] - mx) / sum : 0.f;
      wsum += p;
      if (lane == 0) wout[j] = p;
    }
  } else {
    for (int e = lane; e < E; e += 32) {
      const float ke = keys[e];
      int rank = 0;
      for (int j = 0; j < E; ++j) rank += key_better(keys[j], j, ke, e) ? 1 : 0;
      if (rank < k) {
        const float p = expf(ke - mx) / sum;
        ids[rank] = e;
        wout[rank] = p;
        wsum += p;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  }
  if (flags & MOE_RENORM) {
    __syncwarp();
    for (int j = lane; j < k; j += 32) wout[j] = wout[j] / wsum;
  }
}

template <int TOK>
__global__ void __cluster_dims__(RT_CLUSTER, 1, 1) __launch_bounds__(RT_THREADS)
    route_topk_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, int T, int H, int E, int k,
                      const float *__restrict__ bias, int flags, uint16_t *__restrict__ logits,
                      int32_t *__restrict__ topk_ids, float *__restrict__ topk_w, uint16_t *__restrict__ x16,
                      int32_t *err) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float part[TOK][RT_MAX_EPC];  // this CTA's logits (as fp32 of the BF16 value)
  __shared__ float keys[MAX_E];                   // the token this CTA ranks
  cg::cluster_group cluster = cg::this_cluster();
  pdl_trigger();
  const int rank = int(cluster.block_rank());
  const int t0 = (blockIdx.x / RT_CLUSTER) * TOK;
  const int nt = min(TOK, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int EPC = (E + RT_CLUSTER - 1) / RT_CLUSTER;
  const int e_lo = rank * EPC, e_hi = min(E, e_lo + EPC);
  const bool given = flags & MOE_LOGITS_GIVEN;
  // this warp's first router row: the router weights are not written by the
  // preceding kernel, so these loads go out before waiting for it
  constexpr int PRE = 8;
  uint4 wpre[PRE];
  const int e_first = e_lo + warp;
  if (!given) {
#pragma unroll
    for (int u = 0; u < PRE; ++u) {
      const int hc = lane + 32 * u;
      wpre[u] = (e_first < e_hi && hc < H / 8) ? __ldg(reinterpret_cast<const uint4 *>(wr + int64_t(e_first) * H) + hc)
                                              : make_uint4(0, 0, 0, 0);
    }
  }
  pdl_wait();

  if (!given) {
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);  // [TOK][H]
    const int chunks = H / 8;
    // the 8 tokens' rows, RT_THREADS 16-byte pieces per pass with all of a
    // batch's loads issued before any store (one round trip, not one per piece)
    constexpr int XB = 8;
    for (int c0 = threadIdx.x; c0 < TOK * chunks; c0 += RT_THREADS * XB) {
      uint4 v[XB];
#pragma unroll
      for (int u = 0; u < XB; ++u) {
        const int c = c0 + u * RT_THREADS;
        const int tt = c / chunks, hc = c % chunks;
        v[u] = (c < TOK * chunks && tt < nt) ? __ldg(reinterpret_cast<const uint4 *>(x + int64_t(t0 + tt) * H) + hc)
                                                  : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < XB; ++u) {
        const int c = c0 + u * RT_THREADS;
        if (c < TOK * chunks) reinterpret_cast<uint4 *>(xs + (c / chunks) * H)[c % chunks] = v[u];
      }
    }
    __syncthreads();
    if (x16) {
      // the FP16 copy of the staged rows for the grouped FFN: the cluster's
      // CTAs hold the same rows, so each writes its share of the 16-byte pieces
      const int per = (chunks + RT_CLUSTER - 1) / RT_CLUSTER;
      const int c_lo = rank * per, n_c = max(0, min(chunks, c_lo + per) - c_lo);
      bool bad = false;
      for (int q = threadIdx.x; q < nt * n_c; q += RT_THREADS) {
        const int tt = q / n_c, c = c_lo + q % n_c;
        reinterpret_cast<uint4 *>(x16 + int64_t(t0 + tt) * H)[c] =
            bf16x8_to_f16x8(reinterpret_cast<const uint4 *>(xs + tt * H)[c], bad);
      }
      if (bad) flag_error(err, MOE_DEVERR_RANGE);
    }
    for (int e = e_lo + warp; e < e_hi; e += RT_THREADS / 32) {
      float acc[TOK];
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) acc[tt] = 0.f;
      const uint4 *wrow = reinterpret_cast<const uint4 *>(wr + int64_t(e) * H);
      int hc = lane;
      for (; hc + 32 * 7 < chunks; hc += 32 * 8) {  // eight 16-byte loads in flight per lane
        uint4 wv[8];
        const bool prefetched = (e == e_first && hc == lane);
#pragma unroll
        for (int u = 0; u < 8; ++u) wv[u] = prefetched ? wpre[u] : __ldg(wrow + hc + 32 * u);
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int tt = 0; tt < TOK; ++tt)
            acc[tt] = dot8(wv[u], reinterpret_cast<const uint4 *>(xs + tt * H)[hc + 32 * u], acc[tt]);
      }
      for (; hc < chunks; hc += 32) {
        const uint4 wv = __ldg(wrow + hc);
#pragma unroll
        for (int tt = 0; tt < TOK; ++tt)
          acc[tt] = dot8(wv, reinterpret_cast<const uint4 *>(xs + tt * H)[hc], acc[tt]);
      }
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) {
        float a = acc[tt];
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == tt) {
          const uint16_t lb = f_to_bf16(a);
          part[tt][e - e_lo] = bf16_to_f(lb);
          if (tt < nt) logits[int64_t(t0 + tt) * E + e] = lb;
        }
      }
    }
  }
  cluster.sync();  // every CTA's logits are in its shared memory

  // ---- softmax + top-k for token t0 + rank (warp 0 of each CTA)
  const int t = t0 + rank;
  if (warp == 0 && rank < nt) {
    for (int e = lane; e < E; e += 32) {
      float v;
      if (given) {
        v = bf16_to_f(logits[int64_t(t) * E + e]);
      } else {
        const float *remote = cluster.map_shared_rank(&part[0][0], e / EPC);
        v = remote[rank * RT_MAX_EPC + (e % EPC)];
      }
      if (bias) v = v + bias[e];
      if (v != v) v = -INFINITY;  // NaN never wins
      keys[e] = v;
    }
    __syncwarp();
    topk_warp(keys, E, k, flags, topk_ids + int64_t(t) * k, topk_w + int64_t(t) * k, lane);
  }
  cluster.sync();  // keep this CTA's shared memory alive until every reader is done
}

// ---------------------------------------------------------------- large batches
// For T > 64 the logits are a real GEMM (T x H by H x E): warp-level tensor-core
// MMAs (mma.sync m16n8k16, BF16 in, fp32 accumulate, one BF16 rounding per
// logit, the same arithmetic reading as the cluster kernel), then one warp
// per token for softmax + top-k.
constexpr int LG_TM = 64;   // tokens per CTA
constexpr int LG_TE = 64;   // experts per CTA
constexpr int LG_KC = 64;   // K per shared-memory chunk
constexpr int LG_LD = 72;   // padded row (bf16): 144-byte rows, ldmatrix without bank conflicts

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// logits[t][e] = bf16_rn(sum_h x[t][h] Wr[e][h]) for a 64 x 64 (token x expert)
// tile; warp w owns tokens 16w..16w+15 and all 64 experts (8 n-tiles). The K
// chunks are double-buffered with cp.async; rows past T / E and columns past H
// read as zero.
__global__ void __launch_bounds__(128) logits_mma_kernel(const uint16_t *__restrict__ x,
                                                         const uint16_t *__restrict__ wr, int T, int H, int E,
                                                         uint16_t *__restrict__ logits) {
  __shared__ __align__(16) uint16_t xs[2][LG_TM][LG_LD];
  __shared__ __align__(16) uint16_t ws[2][LG_TE][LG_LD];
  pdl_trigger();
  pdl_wait();
  const int t0 = blockIdx.x * LG_TM, e0 = blockIdx.y * LG_TE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int nchunk = (H + LG_KC - 1) / LG_KC;
  auto load = [&](int c, int buf) {  // 64 rows x 64 k of x and of Wr, 16 bytes per copy
    const int k0 = c * LG_KC;
    for (int i = threadIdx.x; i < LG_TM * (LG_KC / 8); i += 128) {
      const int r = i >> 3, cc = i & 7, kk = k0 + cc * 8;
      const bool vx = t0 + r < T && kk < H, vw = e0 + r < E && kk < H;
      cp_async16_zfill(&xs[buf][r][cc * 8], x + (vx ? int64_t(t0 + r) * H + kk : 0), vx);
      cp_async16_zfill(&ws[buf][r][cc * 8], wr + (vw ? int64_t(e0 + r) * H + kk : 0), vw);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
  load(0, 0);
  for (int c = 0; c < nchunk; ++c) {
    const int buf = c & 1;
    if (c + 1 < nchunk) {
      load(c + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < LG_KC / 16; ++kk) {
      uint32_t af[4];
      ldmatrix_x4(af, &xs[buf][warp * 16 + (lane & 15)][kk * 16 + (lane >> 4) * 8]);
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {  // two n-tiles of experts per ldmatrix
        uint32_t bf[4];
        ldmatrix_x4(bf, &ws[buf][jp * 16 + (lane & 7) + ((lane >> 4) << 3)][kk * 16 + ((lane >> 3) & 1) * 8]);
        mma_bf16_16816(acc[2 * jp], af, bf[0], bf[1]);
        mma_bf16_16816(acc[2 * jp + 1], af, bf[2], bf[3]);
      }
    }
    __syncthreads();  // the buffer is refilled next iteration
  }
  // accumulator (c0, c1) = token g, experts 2t, 2t+1 of the n-tile; (c2, c3) = token g+8
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = t0 + warp * 16 + g + (c >> 1) * 8;
      const int e = e0 + j * 8 + 2 * t + (c & 1);
      if (tok < T && e < E) logits[int64_t(tok) * E + e] = f_to_bf16(acc[j][c]);
    }
}

// Softmax + top-k from given logits, one warp per token.
__global__ void __launch_bounds__(256) topk_kernel(const uint16_t *__restrict__ logits, int T, int E, int k,
                                                   const float *__restrict__ bias, int flags, int32_t *topk_ids,
                                                   float *topk_w) {
  __shared__ float keys[8][MAX_E];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  for (int e = lane; e < E; e += 32) {
    float v = bf16_to_f(logits[int64_t(t) * E + e]);
    if (bias) v = v + bias[e];
    if (v != v) v = -INFINITY;  // NaN never wins
    keys[warp][e] = v;
  }
  __syncwarp();
  topk_warp(keys[warp], E, k, flags, topk_ids + int64_t(t) * k, topk_w + int64_t(t) * k, lane);
}

}  // namespace moe

namespace moe {
// Both entry points: x16 (nullable) receives the FP16 copy of x, fused into
// the decode-sized router kernel or as a conversion pass after the routing.
static int route_impl(const moe_bf16 *x, const moe_bf16 *w_router, int T, int H, int E, int k, const float *bias,
                      int flags, moe_bf16 *logits, int32_t *topk_ids, float *topk_w, uint16_t *x16, int32_t *err,
                      moe_stream_t stream) {
  if (flags & ~(MOE_RENORM | MOE_LOGITS_GIVEN | MOE_IDS_GIVEN))
    return set_error(MOE_ERR_INVALID_ARG, "moe_route_topk: unknown flag bits 0x%x", flags);
  if (T < 0 || E < 1 || E > MAX_E || k < 1 || k > E || k > MAX_K)
    return set_error(MOE_ERR_SHAPE, "moe_route_topk: T=%d E=%d k=%d (need T>=0, 1<=E<=256, 1<=k<=min(E,32))", T, E, k);
  const bool need_x = !(flags & MOE_LOGITS_GIVEN);
  if (need_x && (H < 8 || H % 8))
    return set_error(MOE_ERR_SHAPE, "moe_route_topk: H=%d must be a positive multiple of 8", H);
  if (T == 0) return MOE_OK;
  if (!logits || !topk_ids || !topk_w || (need_x && (!x || !w_router)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_route_topk: NULL pointer");
  if (need_x && (!aligned(x, 16) || !aligned(w_router, 16)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_route_topk: x and w_router must be 16-byte aligned");
  cudaError_t e;
  if (T > 64 && (!need_x || H % 16 == 0)) {
    // large batch: tensor-core logits GEMM (unless given), then top-k per token
    if (need_x) {
      e = launch_pdl(logits_mma_kernel, dim3(unsigned((T + LG_TM - 1) / LG_TM), unsigned((E + LG_TE - 1) / LG_TE)),
                     dim3(128), 0, as_stream(stream), x, w_router, T, H, E, logits);
      if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_route_topk (logits): %s", cudaGetErrorString(e));
      const int st = check_launch("moe_route_topk (logits)");
      if (st != MOE_OK) return st;
    }
    e = launch_pdl(topk_kernel, dim3(unsigned((T + 7) / 8)), dim3(256), 0, as_stream(stream), logits, T, E, k, bias,
                   flags, topk_ids, topk_w);
    if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_route_topk: %s", cudaGetErrorString(e));
    const int st = check_launch("moe_route_topk");
    if (st != MOE_OK || !x16) return st;
    return launch_bf16_to_f16(x, x16, int64_t(T) * H / 8, err, as_stream(stream), "moe_route_topk_x16");
  }
  const bool small = T <= 64;  // decode-sized: 2 tokens per cluster
  const int tok = small ? 2 : 8;
  const size_t smem = need_x ? size_t(tok) * H * 2 : 0;
  if (smem > 200 * 1024) return set_error(MOE_ERR_SHAPE, "moe_route_topk: H=%d too large", H);
  if (smem > 48 * 1024) {
    int st = allow_dynamic_smem(small ? reinterpret_cast<const void *>(route_topk_kernel<2>)
                                      : reinterpret_cast<const void *>(route_topk_kernel<8>),
                                smem, "moe_route_topk");
    if (st != MOE_OK) return st;
  }
  const int64_t blocks = int64_t((T + tok - 1) / tok) * RT_CLUSTER;
  if (blocks > 0x7fffffffLL) return set_error(MOE_ERR_SHAPE, "moe_route_topk: T too large");
  // the router kernel writes x16 only from rows it stages (not with given logits)
  uint16_t *x16_fused = need_x ? x16 : nullptr;
  e = small ? launch_pdl(route_topk_kernel<2>, dim3(unsigned(blocks)), dim3(RT_THREADS), smem, as_stream(stream), x,
                         w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, x16_fused, err)
            : launch_pdl(route_topk_kernel<8>, dim3(unsigned(blocks)), dim3(RT_THREADS), smem, as_stream(stream), x,
                         w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, x16_fused, err);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_route_topk: %s", cudaGetErrorString(e));
  const int st = check_launch("moe_route_topk");
  if (st != MOE_OK || !x16 || x16_fused) return st;
  return launch_bf16_to_f16(x, x16, int64_t(T) * H / 8, err, as_stream(stream), "moe_route_topk_x16");
}
}  // namespace moe

extern "C" int moe_route_topk(const moe_bf16 *x, const moe_bf16 *w_router, int T, int H, int E, int k,
                              const float *bias, int flags, moe_bf16 *logits, int32_t *topk_ids,
                              float *topk_w, moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_route_topk");
  return moe::route_impl(x, w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, nullptr, nullptr, stream);
}

extern "C" int moe_route_topk_x16(const moe_bf16 *x, const moe_bf16 *w_router, int T, int H, int E, int k,
                                  const float *bias, int flags, moe_bf16 *logits, int32_t *topk_ids,
                                  float *topk_w, uint16_t *x16, int32_t *err, moe_stream_t stream) {
  moe::NvtxScope nvtx_scope("moe_route_topk_x16");
  using namespace moe;
  if (H < 8 || H % 8)
    return set_error(MOE_ERR_SHAPE, "moe_route_topk_x16: H=%d must be a positive multiple of 8", H);
  if (T > 0 && (!x || !x16))
    return set_error(MOE_ERR_INVALID_ARG, "moe_route_topk_x16: x and x16 are required");
  if (T > 0 && (!aligned(x, 16) || !aligned(x16, 16)))
    return set_error(MOE_ERR_INVALID_ARG, "moe_route_topk_x16: x and x16 must be 16-byte aligned");
  return route_impl(x, w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, T > 0 ? x16 : nullptr, err,
                    stream);
}
