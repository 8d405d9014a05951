// A5 + A6, prefill-sized groups: grouped W4A16 GEMM on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// "Swap AB": the MMA's M dimension is 128 output features of one expert, its
// N dimension is up to 256 of that expert's tokens (rows of the group, so a
// small group runs a narrow MMA instead of a padded one), and K walks the
// input features 64 at a time. N = 256 halves the shared-memory traffic per
// FLOP of the dequantised A tile, which bounds this kernel. Per CTA (one per SM, persistent over a tile
// list built on the device from the group offsets):
//   warps 0-3  producers: gather the tile's token rows (cp.async, written in
//              the 128-byte-swizzled K-major layout the MMA reads), copy the
//              packed codes of their weight row, and dequantise them in
//              registers to FP16 q*s straight into the swizzled A tile;
//              fence.proxy.async, then arrive on `full`.
//   warp 4     allocates tensor memory; one thread issues the MMAs
//              (kind::f16 with FP16 A and B, fp32 accumulate) and commits each
//              stage back to its `empty` barrier and each finished tile to
//              `tmem_full`.
//   warps 5-8  epilogue: tcgen05.ld of the accumulator (lane = feature,
//              column = token), SwiGLU (gate/up pass) or the plain output
//              (down pass), BF16 stores to h / y in group-sorted row order.
// Why FP16 operands: q*s has at most 3 + 8 significant bits (|q| <= 8 and an
// 8-bit BF16 scale significand) and FP16 holds 11, so the dequantised weight
// is exact; a BF16 activation (8 significant bits) converts to FP16 exactly
// too. The MMA then sums exact products in fp32, the same arithmetic as the
// GEMV path (scale applied to fp32 group sums). This holds while activations
// stay within FP16's range (|v| <= 65504; values below 2^-17 round by at most
// 2^-25) and scales are >= 2^-14; a pre-pass converts x to FP16 and flags
// MOE_DEVERR_RANGE for an activation out of range. The gate/up epilogue
// rounds h to BF16 (the method's A16 intermediate) and stores that value in
// FP16, which again is exact.
// The down pass keeps two accumulator buffers so the epilogue of tile i
// overlaps the mainloop of tile i+1; gate + up at N = 256 fill all 512
// tensor-memory columns with one buffer. Every wait is bounded (about two seconds of %globaltimer); a wait
// that runs out flags MOE_DEVERR_TIMEOUT and all roles drain and exit.
#include "ffn.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;         // features per tile (MMA M)
constexpr int BN = 256;         // max tokens per tile (MMA N)
constexpr int BK = 64;          // K per stage (128 bytes of BF16 = one swizzle row)
constexpr int MAX_STAGES = 5;
constexpr int PRODUCERS = 256;  // warps 0-7: two threads per weight / token row of the tile
constexpr int MMA_WARP = 8;
constexpr int THREADS = 416;    // + warp 8 (MMA) + warps 9-12 (epilogue)
constexpr uint64_t WAIT_NS = 2000000000ull;

template <bool GATEUP>
struct Cfg {
  static constexpr int NMAT = GATEUP ? 2 : 1;
  static constexpr int A_BYTES = BM * BK * 2;         // 16 KB per matrix
  static constexpr int B_BYTES = BN * BK * 2;         // 32 KB
  static constexpr int NIB_BYTES = BM * 32 * NMAT;    // 32 bytes of codes per row and matrix
  static constexpr int STAGE_BYTES = NMAT * A_BYTES + B_BYTES + NIB_BYTES;
  static constexpr int STAGES = GATEUP ? 3 : 4;       // as many as fit in 227 KB
  static constexpr int ACC_COLS = NMAT * BN;          // columns per accumulator buffer
  static constexpr int TMEM_COLS = 512;
  static constexpr int NBUF = TMEM_COLS / ACC_COLS;   // 1 (gate/up) or 2 (down) accumulator buffers
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 4096 /*tables, barriers*/;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 128 bytes stacked 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);        // start address
  d |= uint64_t(1) << 16;                      // leading byte offset (unused for swizzled K-major)
  d |= uint64_t(1024 >> 4) << 32;              // stride byte offset
  d |= uint64_t(1) << 46;                      // version
  d |= uint64_t(2) << 61;                      // SWIZZLE_128B
  return d;
}

// Instruction descriptor: fp32 accumulate (bits 4-5 = 1), FP16 A and B
// (format fields 0), both K-major, N>>3 at bit 17, M>>4 at bit 24.
__device__ __forceinline__ uint32_t idesc_f16(int n) {
  return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ shared state
struct Shared {
  uint64_t full[MAX_STAGES], empty[MAX_STAGES], tmem_full[2], tmem_empty[2], drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles;
  int32_t off[MAX_E + 1];    // group offsets
  int32_t tstart[MAX_E + 1]; // first tile of each expert
};

// Bounded wait: false (and the CTA-wide abort flag set) after WAIT_NS, or
// as soon as another role aborted unless `drain` is set (a drain wait only
// gives up on its own time limit, so tensor memory is never released under
// MMAs still in flight).
__device__ __noinline__ bool wait_bounded(Shared &sh, uint64_t *bar, uint32_t parity, int32_t *err,
                                          bool drain = false) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try(bar, parity)) return true;
    if ((spin & 255) == 0) {
      if (!drain && *(volatile int32_t *)&sh.abort) return false;
      if (globaltimer() - t0 > WAIT_NS) {
        atomicExch(&sh.abort, 1);
        flag_error(err, MOE_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

struct Tile {
  int e, lo, n0, nvalid, f0;
};

__device__ __forceinline__ Tile decode_tile(const Shared &sh, int E, int FT, int t) {
  int lo_e = 0, hi_e = E;  // largest e with tstart[e] <= t
  while (hi_e - lo_e > 1) {
    const int mid = (lo_e + hi_e) >> 1;
    if (sh.tstart[mid] <= t) lo_e = mid; else hi_e = mid;
  }
  Tile x;
  x.e = lo_e;
  const int r = t - sh.tstart[lo_e];
  x.lo = sh.off[lo_e];
  x.n0 = (r / FT) * BN;
  x.f0 = (r % FT) * BM;
  x.nvalid = min(BN, sh.off[lo_e + 1] - x.lo - x.n0);
  return x;
}

template <bool GATEUP>
__global__ void __launch_bounds__(THREADS, 1) tc_ffn_kernel(const FfnArgs a) {
  using C = Cfg<GATEUP>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + STAGES * C::STAGE_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const int NOUT = GATEUP ? a.I : a.H;   // output features
  const int KD = GATEUP ? a.H : a.I;     // reduction length
  const int FT = NOUT / BM;              // feature tiles per token tile
  const int KS = KD / BK;                // k-stages per tile
  const int G = KD / GROUP;
  pdl_trigger();
  pdl_wait();

  // ---- prologue: barriers, tensor memory, tile table
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&sh.full[s], PRODUCERS); mbar_init(&sh.empty[s], 1); }
    for (int b = 0; b < C::NBUF; ++b) { mbar_init(&sh.tmem_full[b], 1); mbar_init(&sh.tmem_empty[b], 128); }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 0) {  // per-expert tile counts -> prefix (experts without a slot get none)
    int v[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      v[i] = 0;
      if (e <= E) sh.off[e] = a.offsets[e];
      if (e < E) {
        const int cnt = a.offsets[e + 1] - a.offsets[e];
        if (cnt > 0) {
          const int slot = a.expert_slot ? a.expert_slot[e] : e;
          if (slot >= 0 && slot < a.n_slots) v[i] = ((cnt + BN - 1) / BN) * FT;
          else flag_error(a.err, MOE_DEVERR_NOT_RESIDENT);
        }
      }
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
      const int e = lane * 8 + i;
      if (e < E) sh.tstart[e] = run;
      run += v[i];
    }
    if (lane == 31) { sh.tstart[E] = incl; sh.total_tiles = incl; sh.off[E] = a.offsets[E]; }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int total = sh.total_tiles;
  const int my_tiles = total > int(blockIdx.x) ? (total - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int iters = my_tiles * KS;
  auto stage_ptr = [&](int s) { return smem + s * C::STAGE_BYTES; };

  if (warp < PRODUCERS / 32) {
    // ================================================================ producers
    // Thread (p, i): i = row of the tile (weight row f0+i and token row i),
    // p = which half of the row's work: the matrix (gate/up pass) or the K
    // half of the stage (down pass), and half of the token row's 8 chunks.
    const int p = tid >> 7, i = tid & 127;
    // per-tile state of the copy stream, refreshed when the stream enters a tile
    int cur_tile = -1;
    const uint8_t *qrow = nullptr;    // this thread's packed-code row
    const uint16_t *srow = nullptr;   // its scale row
    const uint16_t *brow_src[BN / BM] = {};
    bool bvalid[BN / BM] = {};
    auto enter_tile = [&](int tl_i) {
      const int t = int(blockIdx.x) + tl_i * int(gridDim.x);
      const Tile tl = decode_tile(sh, E, FT, t);
      const int slot = a.expert_slot ? a.expert_slot[tl.e] : tl.e;
      const uint8_t *rec = a.bank + int64_t(slot) * a.rec;
      const int m = GATEUP ? p : 0;
      qrow = rec + (GATEUP ? (m ? a.off_uq : a.off_gq) : a.off_dq) + int64_t(tl.f0 + i) * (KD / 2);
      srow = reinterpret_cast<const uint16_t *>(rec + (GATEUP ? (m ? a.off_us : a.off_gs) : a.off_ds)) +
             int64_t(tl.f0 + i) * G;
#pragma unroll
      for (int h = 0; h < BN / BM; ++h) {
        const int r = i + h * BM;
        bvalid[h] = r < tl.nvalid;
        if (GATEUP) {
          const int tok = bvalid[h] ? a.sorted_pair[tl.lo + tl.n0 + r] / a.k : 0;
          brow_src[h] = a.x16 + int64_t(tok) * KD;
        } else {
          brow_src[h] = a.h + int64_t(bvalid[h] ? tl.lo + tl.n0 + r : 0) * KD;
        }
      }
      cur_tile = tl_i;
    };
    // per-tile state of the dequant stream (lags the copies by D stages)
    int deq_tile = -1;
    const uint16_t *deq_srow = nullptr;
    auto scale_row = [&](int tl_i) {
      const Tile tl = decode_tile(sh, E, FT, int(blockIdx.x) + tl_i * int(gridDim.x));
      const int slot = a.expert_slot ? a.expert_slot[tl.e] : tl.e;
      const uint8_t *rec = a.bank + int64_t(slot) * a.rec;
      const int m = GATEUP ? p : 0;
      return reinterpret_cast<const uint16_t *>(rec + (GATEUP ? (m ? a.off_us : a.off_gs) : a.off_ds)) +
             int64_t(tl.f0 + i) * G;
    };
    // Copies of stage `it` (cp.async); its group scale is prefetched into L1
    // so the dequant D stages later reads it without a long stall.
    auto issue = [&](int it) {
      if (it / KS != cur_tile) enter_tile(it / KS);
      const int ks = it % KS;
      uint8_t *st = stage_ptr(it % STAGES);
      const uint32_t nib = smem_u32(st + C::NMAT * C::A_BYTES + C::B_BYTES);
      if (GATEUP) {  // matrix p: 32 bytes (64 codes) of row i; chunk c at slot c ^ ((i >> 2) & 1)
        const uint32_t d = nib + (p * BM + i) * 32;
        const int r = (i >> 2) & 1;
        cp_async16(d + ((0 ^ r) << 4), qrow + ks * (BK / 2), 16);
        cp_async16(d + ((1 ^ r) << 4), qrow + ks * (BK / 2) + 16, 16);
      } else {       // K half p: 16 bytes (32 codes) of row i
        cp_async16(nib + (i * 2 + p) * 16, qrow + ks * (BK / 2) + p * 16, 16);
      }
#pragma unroll
      for (int h = 0; h < BN / BM; ++h) {  // token rows i and i + 128
        const uint32_t brow = smem_u32(st + C::NMAT * C::A_BYTES) + (i + h * BM) * 128;
#pragma unroll
        for (int c = 4 * p; c < 4 * p + 4; ++c)
          cp_async16(brow + ((c ^ (i & 7)) << 4), brow_src[h] + ks * BK + c * 8, bvalid[h] ? 16 : 0);
      }
      asm volatile("prefetch.global.L1 [%0];" ::"l"(srow + (ks * BK) / GROUP));
    };
    constexpr int D = C::STAGES - 1;  // copy-ahead distance in stages
    bool ok = true;
#pragma unroll
    for (int j = 0; j < D; ++j) {
      if (j < iters && ok) {
        ok = wait_bounded(sh, &sh.empty[j % STAGES], ((j / STAGES) & 1) ^ 1, a.err);
        if (ok) issue(j);
      }
      cp_async_commit();
    }
    const __half2 h1032 = __floats2half2_rn(1032.0f, 1032.0f);
    const __half2 h16th = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 hm72 = __floats2half2_rn(-72.0f, -72.0f);
    // Per iteration: dequantise stage `it` and hand it to the MMA first, then
    // refill the buffer the MMA has just finished with (stage it + D), so the
    // dequant never waits for an MMA and the MMA finds each stage ready.
    for (int it = 0; it < iters && ok; ++it) {
      if (it / KS != deq_tile) { deq_tile = it / KS; deq_srow = scale_row(deq_tile); }
      const uint16_t sbits = deq_srow[((it % KS) * BK) / GROUP];  // L1 hit (prefetched)
      cp_async_wait<D - 1>();  // the copies of stage `it` have landed
      // dequantise this thread's codes of stage `it` into the swizzled A tile
      uint8_t *st = stage_ptr(it % STAGES);
      const uint8_t *nib = st + C::NMAT * C::A_BYTES + C::B_BYTES;
      const __half2 sc = __half2half2(__float2half_rn(bf16_to_f(sbits)));
      uint32_t words[8];
      int nw, c0;
      uint8_t *arow;
      if (GATEUP) {
        const uint8_t *src = nib + (p * BM + i) * 32;
        const int r = (i >> 2) & 1;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(src + ((0 ^ r) << 4));
        const uint4 w1 = *reinterpret_cast<const uint4 *>(src + ((1 ^ r) << 4));
        words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
        words[4] = w1.x; words[5] = w1.y; words[6] = w1.z; words[7] = w1.w;
        nw = 8; c0 = 0;
        arow = st + p * C::A_BYTES + i * 128;
      } else {
        const uint4 w0 = *reinterpret_cast<const uint4 *>(nib + (i * 2 + p) * 16);
        words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
        words[4] = words[5] = words[6] = words[7] = 0;
        nw = 4; c0 = 4 * p;
        arow = st + i * 128;
      }
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {
        if (wd >= nw) break;
        // k = 2i + h sits at bits 4(i + 4h): OR-ing the nibbles at bits 0-3 /
        // 16-19 into FP16 1024.0 gives (1024 + u), those at bits 4-7 / 20-23
        // give (1024 + 16u); one shift by 8 brings pairs 2 and 3 to the same
        // places. (1024 + u) - 1032 = q and (1024 + 16u) / 16 - 72 = q, exact.
        const uint32_t w0 = words[wd], w8 = words[wd] >> 8;
        const uint32_t tq[4] = {(w0 & 0x000F000Fu) | 0x64006400u, (w0 & 0x00F000F0u) | 0x64006400u,
                                (w8 & 0x000F000Fu) | 0x64006400u, (w8 & 0x00F000F0u) | 0x64006400u};
        uint32_t outp[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const __half2 t2 = *reinterpret_cast<const __half2 *>(&tq[pp]);
          const __half2 q = (pp & 1) ? __hfma2(t2, h16th, hm72) : __hsub2(t2, h1032);
          __half2 v = __hmul2(q, sc);
          outp[pp] = *reinterpret_cast<uint32_t *>(&v);
        }
        const int c = c0 + wd;
        *reinterpret_cast<uint4 *>(arow + ((c ^ (i & 7)) << 4)) = make_uint4(outp[0], outp[1], outp[2], outp[3]);
      }
      fence_proxy_async();
      if (!a.stall) mbar_arrive(&sh.full[it % STAGES]);
      const int nx = it + D;
      if (nx < iters) {
        ok = wait_bounded(sh, &sh.empty[nx % STAGES], ((nx / STAGES) & 1) ^ 1, a.err);
        if (ok) issue(nx);
      }
      cp_async_commit();
    }
    cp_async_wait<0>();
  } else if (warp == MMA_WARP) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tl_i = 0; tl_i < my_tiles && ok; ++tl_i) {
        const int t = int(blockIdx.x) + tl_i * int(gridDim.x);
        const Tile tl = decode_tile(sh, E, FT, t);
        const int n_mma = max(16, (tl.nvalid + 15) & ~15);
        const uint32_t idesc = idesc_f16(n_mma);
        const int b = tl_i % C::NBUF;
        ok = wait_bounded(sh, &sh.tmem_empty[b], ((tl_i / C::NBUF) & 1) ^ 1, a.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d0 = tmem + b * C::ACC_COLS;
        for (int ks = 0; ks < KS; ++ks, ++it) {
          const int s = it % STAGES;
          ok = wait_bounded(sh, &sh.full[s], (it / STAGES) & 1, a.err);
          if (!ok) break;
          tc_fence_after();
          uint8_t *st = stage_ptr(s);
          const uint64_t bdesc = sw128_desc(smem_u32(st + C::NMAT * C::A_BYTES));
#pragma unroll
          for (int m = 0; m < C::NMAT; ++m) {
            const uint64_t adesc = sw128_desc(smem_u32(st + m * C::A_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_f16(d0 + m * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) != 0);
          }
          mma_commit(&sh.empty[s]);
        }
        if (ok) mma_commit(&sh.tmem_full[b]);
      }
      // all issued MMAs have completed before tensor memory is released
      mma_commit(&sh.drain);
      wait_bounded(sh, &sh.drain, 0, a.err, true);
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue
    const int q = warp & 3;            // tensor-memory lane quadrant of this warp
    const int frow = q * 32 + lane;    // feature within the tile
    for (int tl_i = 0; tl_i < my_tiles; ++tl_i) {
      const int t = int(blockIdx.x) + tl_i * int(gridDim.x);
      const Tile tl = decode_tile(sh, E, FT, t);
      const int b = tl_i % C::NBUF;
      if (!wait_bounded(sh, &sh.tmem_full[b], (tl_i / C::NBUF) & 1, a.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + b * C::ACC_COLS;
      const int f = tl.f0 + frow;
      for (int j0 = 0; j0 < tl.nvalid; j0 += 16) {
        uint32_t g[16];
        tmem_ld16(tbase + j0, g);
        if (GATEUP) {
          uint32_t u[16];
          tmem_ld16(tbase + BN + j0, u);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = j0 + jj;
            if (j < tl.nvalid) {
              const float gv = __uint_as_float(g[jj]), uv = __uint_as_float(u[jj]);
              const float hv = bf16_to_f(f_to_bf16(silu_f(gv) * uv));  // A16: h is BF16
              a.h[int64_t(tl.lo + tl.n0 + j) * NOUT + f] = __half_as_ushort(__float2half_rn(hv));
            }
          }
        } else {
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = j0 + jj;
            if (j < tl.nvalid) a.y[int64_t(tl.lo + tl.n0 + j) * NOUT + f] = __uint_as_float(g[jj]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.tmem_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

}  // namespace tc

static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

int launch_ffn_tc(const FfnArgs &a, cudaStream_t s) {
  int dev = 0, major = 0, minor = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return set_error(MOE_ERR_UNSUPPORTED, "moe_grouped_w4a16_ffn: tensor-core path needs sm_100 (found sm_%d%d)", major,
                     minor);
  if (a.H % tc::BM || a.I % tc::BM)
    return set_error(MOE_ERR_UNSUPPORTED, "moe_grouped_w4a16_ffn: tensor-core path needs H, I multiples of 128");
  const int grid = sm_count();
  int st0 = launch_x_to_f16(a, s);
  if (st0 != MOE_OK) return st0;
  const size_t smem_gu = tc::Cfg<true>::SMEM, smem_dn = tc::Cfg<false>::SMEM;
  int st = allow_dynamic_smem(reinterpret_cast<const void *>(tc::tc_ffn_kernel<true>), smem_gu, "ffn tc gate/up");
  if (st != MOE_OK) return st;
  st = allow_dynamic_smem(reinterpret_cast<const void *>(tc::tc_ffn_kernel<false>), smem_dn, "ffn tc down");
  if (st != MOE_OK) return st;
  cudaError_t e = launch_pdl(tc::tc_ffn_kernel<true>, dim3(grid), dim3(tc::THREADS), smem_gu, s, a);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (tc gate/up): %s", cudaGetErrorString(e));
  st = check_launch("moe_grouped_w4a16_ffn (tc gate/up)");
  if (st != MOE_OK) return st;
  e = launch_pdl(tc::tc_ffn_kernel<false>, dim3(grid), dim3(tc::THREADS), smem_dn, s, a);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (tc down): %s", cudaGetErrorString(e));
  return check_launch("moe_grouped_w4a16_ffn (tc down)");
}

}  // namespace moe
