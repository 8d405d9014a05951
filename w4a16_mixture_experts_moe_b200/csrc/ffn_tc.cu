// A5 + A6, prefill-sized groups: grouped W4A16 GEMM on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// "Swap AB": the MMA's M dimension is 128 output features of one expert, its
// N dimension is up to 256 of that expert's tokens (rows of the group, so a
// small group runs a narrow MMA instead of a padded one), and K walks the
// input features 64 at a time. Per CTA (one per SM, persistent over a tile
// list built on the device from the group offsets), three rings of
// shared-memory buffers, each k-step taking one slot of each:
//   codes  the packed int4 codes of the tile's 128 weight rows (per matrix),
//          3 slots of 8 KB, refilled as soon as the dequant warps hold a
//          slot's codes in registers;
//   B      256 FP16 activation rows (gate/up: x gathered into group order by
//          a pre-pass; down: h), 128-byte-swizzled K-major as the MMA reads;
//   A      the dequantised FP16 weights q*s, same swizzled layout.
// Roles:
//   warps 0-7   dequant: two threads per weight row read the codes from the
//               codes ring (releasing the slot at once), wait for a free A
//               slot, write FP16 q*s into it, fence.proxy.async, arrive.
//   warps 8-23  epilogue: four warps per tensor-memory lane quadrant, each a
//               quarter of the token columns: tcgen05.ld of the accumulator
//               (lane = feature, column = token), SwiGLU (gate/up pass) or the
//               plain fp32 output (down pass), stores to h / y in group order.
//               The epilogue cannot overlap the next tile's MMAs (the two N =
//               256 accumulators fill tensor memory), and it is latency-bound
//               on its SwiGLU arithmetic: four warps per quadrant instead of
//               two shortened it enough to lift OLMoE prefill from 39.7 to
//               41.8 % of peak at T = 2048 (the kernel fits in 72 registers).
//   warp 24     allocates tensor memory; one elected lane issues the MMAs
//               (kind::f16 with FP16 A and B, fp32 accumulate) and commits
//               each k-step back to its A and B slots and each finished tile
//               to `tmem_full`. It touches no memory inside the loop: a
//               warp's loads, stores and mbarrier waits issued behind
//               tcgen05.mma are held until those MMAs finish, which would
//               drain the tensor core's short queue at every k-step.
//   warp 27     waiter: performs the bounded mbarrier waits for the MMA warp
//               (stage landed and dequantised, accumulator buffer free) and
//               hands each k-step over with a named-barrier reduction
//               (bar.red.popc) carrying the tile's MMA width and an abort bit.
//   warp 25     one thread issues the TMA loads of the codes ring (a 3-D box
//               over the record bank: 32 bytes x 128 rows x 1 record).
//   warp 26     one thread issues the TMA loads of the B ring (a 64 x 256
//               FP16 box).
// Why FP16 operands: q*s has at most 3 + 8 significant bits (|q| <= 8 and an
// 8-bit BF16 scale significand) and is a multiple of the scale's last bit.
// Each weight row is moved by a power of two 2^a (a per row, from its largest
// scale: that scale times 2^a lies in [2^-4, 2^-3)), so the dequantised value
// q*s*2^a has magnitude <= 1 and is exact in FP16 for every scale of the row
// down to 2^-13 of the largest (a normal FP16 holds 11 significant bits; FP16
// subnormals are multiples of 2^-24). The epilogue multiplies the row's fp32
// sum by 2^-a, which is exact, so the tile computes x.(q*s) with exact
// products summed in fp32, like the GEMV path (which applies each group scale
// to an fp32 partial sum), whatever the weights' magnitude: without it a scale
// below 2^-17 would be rounded and one above 8188 would overflow FP16. (The
// target is deliberately small: rows moved up to |q*s*2^a| ~ 2^15 measured
// far less accurate sums on the tensor cores, errors of up to 30 % at K =
// 4096, while operands of magnitude <= 1 match the oracle.) A BF16 activation converts to FP16 exactly
// when 2^-17 <= |v| <= 65504 (or v = 0); smaller ones round to a multiple of
// 2^-24 (absolute error at most 2^-25). A pre-pass converts x to FP16 and
// flags MOE_DEVERR_RANGE for an activation above 65504 in magnitude. The
// gate/up epilogue rounds h to BF16 (the method's A16 intermediate), stores
// that value in FP16 and flags the same error for an h that does not fit.
// Both passes run two 128-row blocks of A against each activation box (gate
// and up of the same features; or 256 consecutive down-output features), so
// the two N = 256 accumulators fill all 512 tensor-memory columns with one
// buffer: the epilogue is kept short (sixteen warps, fast-divide SiLU)
// instead of overlapped. Every wait is bounded (about two
// seconds of %globaltimer); a wait that runs out flags MOE_DEVERR_TIMEOUT and
// all roles drain and exit.
#include <mutex>

#include "ffn.cuh"
#include "tma.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;         // features per tile (MMA M)
constexpr int BN = 256;         // max tokens per tile (MMA N)
constexpr int BK = 64;          // K per k-step (128 bytes of FP16 = one swizzle row)
constexpr int MAX_RING = 8;
constexpr int DEQUANT = 256;    // warps 0-7
constexpr int EPI_WARP0 = 8;    // warps 8-23
constexpr int EPILOGUE = 512;
constexpr int MMA_WARP = 24;
constexpr int TMA_CODES_WARP = 25;
constexpr int TMA_B_WARP = 26;
constexpr int WAITER_WARP = 27;
constexpr int THREADS = 896;
constexpr int HANDOFF_BAR = 1;  // named barrier: waiter warp + MMA warp

template <bool GATEUP>
struct Cfg {
  // A holds two 128-row blocks: gate and up rows of the same 128 features
  // (gate/up pass), or two consecutive 128-row blocks of the down matrix (down
  // pass: 256 output features per tile, so each activation box feeds twice
  // the MMA work)
  static constexpr int NMAT = 2;
  static constexpr int A_BYTES = NMAT * BM * BK * 2;  // 16 KB per matrix
  static constexpr int B_BYTES = BN * BK * 2;         // 32 KB
  static constexpr int C_BYTES = NMAT * BM * BK / 2;  // 4 KB of codes per matrix
  static constexpr int S = 3;                         // A and B ring depth (one commit frees both)
  static constexpr int CS = 3;                        // codes ring depth
  static constexpr int FW = GATEUP ? BM : 2 * BM;     // output features per tile
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + S * A_BYTES;
  static constexpr int C_OFF = B_OFF + S * B_BYTES;
  static constexpr int RING_BYTES = C_OFF + CS * C_BYTES;
  static constexpr int ACC_COLS = NMAT * BN;          // columns per accumulator buffer
  static constexpr int TMEM_COLS = 512;
  static constexpr int NBUF = TMEM_COLS / ACC_COLS;   // accumulator buffers (1: two N = 256 blocks fill TMEM)
  static constexpr int SMEM = RING_BYTES + 1024 /*align*/ + 6144 /*tables, barriers*/;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(S <= MAX_RING && CS <= MAX_RING, "ring depth");
  static_assert(B_OFF % 1024 == 0 && C_OFF % 1024 == 0, "swizzled buffers need 1024-byte alignment");
};

// ------------------------------------------------------------------ PTX wrappers
using namespace tma;

// Named-barrier handoff between the waiter and the MMA warp (64 threads):
// returns the number of participating threads whose predicate is true.
__device__ __forceinline__ uint32_t handoff(uint32_t pred) {
  uint32_t cnt;
  asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n bar.red.popc.u32 %0, %2, 64, p;\n}\n"
               : "=r"(cnt)
               : "r"(pred), "n"(HANDOFF_BAR)
               : "memory");
  return cnt;
}
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
// Two 32-lane x 16-column accumulator loads and the wait for them, in ONE asm
// statement: the destination registers of tcgen05.ld hold their values only
// after tcgen05.wait::ld, and a separate wait statement (tied to the loads
// by nothing but a memory clobber) lets the compiler schedule arithmetic on
// those registers ahead of it, reading whatever they held before.
__device__ __forceinline__ void tmem_ld16(uint32_t ta, uint32_t (&a)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15])
      : "r"(ta)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15])
      : "r"(ta), "r"(tb)
      : "memory");
}

// ------------------------------------------------------------------ shared state
struct Shared {
  uint64_t c_loaded[MAX_RING], c_free[MAX_RING];  // codes ring: TMA bytes / dequant threads
  uint64_t b_loaded[MAX_RING], a_full[MAX_RING];  // stage s: B rows landed (TMA bytes) / A written (dequant warps)
  uint64_t s_free[MAX_RING];                      // stage s: its MMAs completed (commit)
  uint64_t tmem_full[2], tmem_empty[2], drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_tiles, full_tiles;
  int32_t off[MAX_E + 1];    // group offsets
  int32_t tstart[MAX_E + 1]; // first full-width tile of each expert (full tiles come first)
  int16_t prow[MAX_E];       // rows of the expert's last, narrower token tile (0: none)
  int16_t porder[MAX_E];     // experts with a narrower tile, widest first (ties: lower index)
  // power-of-two exponent of each weight row of a tile, written by the
  // dequant warps at the tile's start, read by the epilogue after the tile's
  // accumulator is complete; indexed by tile % ROWEXP_SLOTS ([block][row])
  int16_t row_exp[4][2][128];
};
constexpr int ROWEXP_SLOTS = 4;  // tiles in flight between the two: at most three
static_assert(sizeof(Shared) <= 6144, "shared tables budget");

// Bounded wait on the CTA's abort flag (see tma::wait_bounded).
__device__ __forceinline__ bool wait_bounded(Shared &sh, uint64_t *bar, uint32_t parity, int32_t *err,
                                             bool drain = false) {
  return tma::wait_bounded(&sh.abort, bar, parity, err, drain);
}

struct Tile {
  int e, lo, n0, nvalid, f0;
};

// v * 2^n for |n| <= 252, as two multiplications by exact powers of two
// (each factor a normal fp32), so the result is exact unless it is subnormal.
__device__ __forceinline__ float mul_pow2(float v, int n) {
  const int n1 = n / 2, n2 = n - n1;
  return v * __uint_as_float(uint32_t(127 + n1) << 23) * __uint_as_float(uint32_t(127 + n2) << 23);
}

// Exponent a of a weight row's power-of-two normalisation: the row's largest
// BF16 scale times 2^a lies in [2^-4, 2^-3), so every dequantised weight
// q*s*2^a has magnitude <= 1 (a = 0 for an all-zero row). Scales are never
// negative, so their bit patterns order like their values.
__device__ __forceinline__ int row_exponent(const uint16_t *srow, int G) {
  uint32_t mx = 0;
  if ((G & 7) == 0) {  // rows of whole 16-byte pieces: eight scales per load, the loads issued together
#pragma unroll 4
    for (int g = 0; g < G; g += 8) {
      const uint4 v = *reinterpret_cast<const uint4 *>(srow + g);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) mx = max(mx, max(w[j] & 0xFFFFu, w[j] >> 16));
    }
  } else {
#pragma unroll 4
    for (int g = 0; g < G; ++g) mx = max(mx, uint32_t(srow[g]));
  }
  if (mx == 0) return 0;
  const int e = min(127, max(-133, ilogbf(bf16_to_f(uint16_t(mx)))));  // floor(log2(largest scale))
  return -4 - e;
}

// The tile list, in the order it is handed out: every full-width (BN-token)
// tile first, expert by expert, then each expert's narrower last token tile,
// widest first. A narrow tile costs nearly the dequantisation and k-step
// chain of a full one for a fraction of its MMAs, so handing the tiles out
// from the longest down evens out the CTAs' finishing times (the
// longest-processing-time-first rule).
template <int FW>
__device__ __forceinline__ Tile decode_tile(const Shared &sh, int E, int FT, int t) {
  Tile x;
  if (t < sh.full_tiles) {
    int lo_e = 0, hi_e = E;  // largest e with tstart[e] <= t
    while (hi_e - lo_e > 1) {
      const int mid = (lo_e + hi_e) >> 1;
      if (sh.tstart[mid] <= t) lo_e = mid; else hi_e = mid;
    }
    const int r = t - sh.tstart[lo_e];
    x.e = lo_e;
    x.n0 = (r / FT) * BN;
    x.f0 = (r % FT) * FW;
    x.nvalid = BN;
  } else {
    const int q = t - sh.full_tiles;
    x.e = sh.porder[q / FT];
    x.f0 = (q % FT) * FW;
    x.nvalid = sh.prow[x.e];
    x.n0 = sh.off[x.e + 1] - sh.off[x.e] - x.nvalid;
  }
  x.lo = sh.off[x.e];
  return x;
}

// The CTA's i-th tile: position i*G + b of the list on even rounds and
// i*G + (G - 1 - b) on odd ones (a snake over the CTAs), so that the CTAs
// which took the longest tiles of one round take the shortest of the next.
__device__ __forceinline__ int sched_pos(int i) {
  const int G = int(gridDim.x), b = int(blockIdx.x);
  return i * G + ((i & 1) ? G - 1 - b : b);
}

// tm_b: activation rows in group order (gate/up: FP16 x gathered by the
// pre-pass; down: h), box 64 x 256, 128-byte swizzle. tm_q0 / tm_q1: packed
// codes of A's first / second 128-row block over the record bank (gate and up;
// or the down matrix twice, at rows f0 and f0 + 128), box 32 B x 128 rows x 1
// record.
template <bool GATEUP>
__global__ void __launch_bounds__(THREADS, 1)
    tc_ffn_kernel(const FfnArgs a, const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_q0,
                  const __grid_constant__ CUtensorMap tm_q1) {
  using C = Cfg<GATEUP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + C::RING_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const int NOUT = GATEUP ? a.I : a.H;   // output features
  const int KD = GATEUP ? a.H : a.I;     // reduction length
  const int FT = (NOUT + C::FW - 1) / C::FW;  // feature tiles per token tile
  const int KS = KD / BK;                // k-steps per tile
  const int G = KD / GROUP;
  pdl_trigger();
  pdl_wait();

  // ---- prologue: barriers, tensor memory, tile table
  if (tid == 0) {
    // consumer-side barriers count one elected arrival per warp
    for (int s = 0; s < C::CS; ++s) { mbar_init(&sh.c_loaded[s], 1); mbar_init(&sh.c_free[s], DEQUANT / 32); }
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&sh.b_loaded[s], 1);
      mbar_init(&sh.a_full[s], DEQUANT / 32);
      mbar_init(&sh.s_free[s], 1);
    }
    for (int b = 0; b < C::NBUF; ++b) { mbar_init(&sh.tmem_full[b], 1); mbar_init(&sh.tmem_empty[b], EPILOGUE / 32); }
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
    int v[8], local = 0, nparts = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      v[i] = 0;
      if (e <= E) sh.off[e] = a.offsets[e];
      if (e < E) {
        const int cnt = a.offsets[e + 1] - a.offsets[e];
        int rows = 0;
        if (cnt > 0) {
          const int slot = a.expert_slot ? a.expert_slot[e] : e;
          if (slot >= 0 && slot < a.n_slots) rows = cnt;
          else if (slot != MOE_SLOT_SKIP) flag_error(a.err, MOE_DEVERR_NOT_RESIDENT);
        }
        v[i] = (rows / BN) * FT;
        sh.prow[e] = int16_t(rows % BN);
        nparts += (rows % BN) != 0;
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
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nparts += __shfl_xor_sync(0xffffffffu, nparts, o);
    if (lane == 31) {
      sh.tstart[E] = incl;
      sh.full_tiles = incl;
      sh.total_tiles = incl + nparts * FT;
      sh.off[E] = a.offsets[E];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid < E && sh.prow[tid] > 0) {  // rank of this expert's narrow tile: widest first, ties by index
    const int mine = sh.prow[tid];
    int rank = 0;
    for (int e = 0; e < E; ++e) {
      const int r = sh.prow[e];
      rank += r > mine || (r == mine && e < tid);
    }
    sh.porder[rank] = int16_t(tid);
  }
  __syncthreads();
  const uint32_t tmem = sh.tmem_base;
  const int total = sh.total_tiles;
  const int rounds = total / int(gridDim.x), rem = total % int(gridDim.x);
  const int my_tiles = rounds + (rem > 0 && ((rounds & 1) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x)) < rem);
  const int iters = my_tiles * KS;
  uint8_t *const ringA = smem + C::A_OFF, *const ringB = smem + C::B_OFF, *const ringC = smem + C::C_OFF;

  if (warp < DEQUANT / 32) {
    // ================================================================ dequant
    // Thread (p, i): weight row f0+i of the tile; p = the matrix (gate/up
    // pass) or the K half of the k-step (down pass).
    const int p = tid >> 7, i = tid & 127;
    int deq_tile = -1, ks = 0, deq_a = 0;
    const uint16_t *deq_srow = nullptr;
    // the row's scale of the current group, and the next group's, loaded a
    // whole group (two k-steps) ahead so its latency is never exposed
    int cur_grp = -1;
    uint16_t sbits = 0, next_bits = 0;
    const __half2 h1032 = __floats2half2_rn(1032.0f, 1032.0f);
    const __half2 h16th = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 hm72 = __floats2half2_rn(-72.0f, -72.0f);
    bool ok = true;
    for (int it = 0; it < iters && ok; ++it, ++ks) {
      if (ks == KS || deq_tile < 0) {
        ks = 0;
        ++deq_tile;
        const Tile tl = decode_tile<C::FW>(sh, E, FT, sched_pos(deq_tile));
        const int slot = a.expert_slot ? a.expert_slot[tl.e] : tl.e;
        const uint8_t *rec = a.bank + int64_t(slot) * a.rec;
        // row of this thread's weights; down rows past H (a ragged last
        // tile) get a zero scale, their codes arrive as zeros
        const int row = tl.f0 + (GATEUP ? 0 : p * BM) + i;
        deq_srow = row < NOUT ? reinterpret_cast<const uint16_t *>(rec + (GATEUP ? (p ? a.off_us : a.off_gs) : a.off_ds)) +
                                    int64_t(row) * G
                              : nullptr;
        deq_a = deq_srow ? row_exponent(deq_srow, G) : 0;
        // the epilogue of this tile undoes the same power of two; the write is
        // ordered before it by this tile's first a_full arrival, the MMAs and
        // the tile's accumulator commit
        sh.row_exp[deq_tile % ROWEXP_SLOTS][p][i] = int16_t(deq_a);
        cur_grp = -1;
        next_bits = deq_srow ? deq_srow[0] : uint16_t(0);  // in L1: row_exponent just read the row
      }
      if ((ks * BK) / GROUP != cur_grp) {
        cur_grp = (ks * BK) / GROUP;
        sbits = next_bits;
        next_bits = deq_srow && cur_grp + 1 < G ? deq_srow[cur_grp + 1] : uint16_t(0);
      }
      const int cs = it % C::CS, as = it % C::S;
      // wait results are made warp-uniform: a lane never leaves the loop
      // while the rest of its warp goes on to a __syncwarp
      ok = __all_sync(0xffffffffu, wait_bounded(sh, &sh.c_loaded[cs], (it / C::CS) & 1, a.err));
      if (!ok) break;
      const uint8_t *nib = ringC + cs * C::C_BYTES;  // [matrix][128 rows][32 B]
      uint32_t words[8];
      {
        const uint8_t *src = nib + (p * BM + i) * 32;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(src);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(src + 16);
        words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
        words[4] = w1.x; words[5] = w1.y; words[6] = w1.z; words[7] = w1.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.c_free[cs]);  // the warp's codes are in registers: the slot may be refilled
      ok = __all_sync(0xffffffffu, wait_bounded(sh, &sh.s_free[as], ((it / C::S) & 1) ^ 1, a.err));
      if (!ok) break;
      const __half2 sc = __half2half2(__float2half_rn(mul_pow2(bf16_to_f(sbits), deq_a)));  // s * 2^a, exact
      constexpr int NW = 8;
      const int c0 = 0;
      uint8_t *arow = ringA + as * C::A_BYTES + p * (BM * BK * 2) + i * 128;
#pragma unroll
      for (int wd = 0; wd < NW; ++wd) {
        // k = 2i + h sits at bits 4(i + 4h): OR-ing the nibbles at bits 0-3 /
        // 16-19 into FP16 1024.0 gives (1024 + u), those at bits 4-7 / 20-23
        // give (1024 + 16u); one shift by 8 brings pairs 2 and 3 to the same
        // places. (1024 + u) - 1032 = q and (1024 + 16u) / 16 - 72 = q, exact.
        // (The published int4 -> FP16 conversion by exponent-field insertion:
        // Kim et al., 2022, "Who Says Elephants Can't Run".)
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
      fence_proxy_async();  // this thread's A writes -> visible to the tensor core
      __syncwarp();
      if (lane == 0 && !a.stall) mbar_arrive(&sh.a_full[as]);
    }
  } else if (warp < EPI_WARP0 + EPILOGUE / 32) {
    // ================================================================ epilogue
    const int q = warp & 3;                          // tensor-memory lane quadrant of this warp
    const int quarter = (warp - EPI_WARP0) >> 2;     // which quarter of the token columns
    const int frow = q * 32 + lane;                  // feature within the tile
    for (int tl_i = 0; tl_i < my_tiles; ++tl_i) {
      const Tile tl = decode_tile<C::FW>(sh, E, FT, sched_pos(tl_i));
      const int b = tl_i % C::NBUF;
      const int f = tl.f0 + frow;
      if (!__all_sync(0xffffffffu, wait_bounded(sh, &sh.tmem_full[b], (tl_i / C::NBUF) & 1, a.err))) break;
      tc_fence_after();
      // undo the dequant warps' power-of-two row normalisation: block 0 =
      // gate row f (gate/up pass) or down row f; block 1 = up row f or down
      // row f + 128. (The epilogue issues no global loads of its own ahead of
      // the accumulator wait: a version that read the row scales there, as
      // the dequant warps do, measured corrupted tiles that no barrier
      // analysis explained, while the same loads in the dequant warps and
      // plain delays in the epilogue did not.)
      const float unscale0 = mul_pow2(1.0f, -int(sh.row_exp[tl_i % ROWEXP_SLOTS][0][frow]));
      const float unscale1 = mul_pow2(1.0f, -int(sh.row_exp[tl_i % ROWEXP_SLOTS][1][frow]));
      const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + b * C::ACC_COLS;
      const int j_lo = quarter * (BN / 4), j_hi = min(tl.nvalid, j_lo + BN / 4);
      const int64_t row0 = int64_t(tl.lo + tl.n0);
      for (int j0 = j_lo; j0 < j_hi; j0 += 16) {
        if constexpr (GATEUP) {
          uint32_t g[16], u[16];  // gate and up sums of 16 tokens
          tmem_ld16x2(tbase + j0, tbase + BN + j0, g, u);
          uint16_t *hp = a.h + (row0 + j0) * NOUT + f;
          bool bad = false;  // an h outside FP16's finite range cannot be the down pass's operand
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            if (j0 + jj < j_hi) {
              const float gv = __uint_as_float(g[jj]) * unscale0, uv = __uint_as_float(u[jj]) * unscale1;
              const float hv = bf16_to_f(f_to_bf16(silu_f(gv) * uv));  // A16: h is BF16
              bad |= fabsf(hv) > 65504.f;
              hp[jj * NOUT] = __half_as_ushort(__float2half_rn(hv));
            }
          }
          if (bad) flag_error(a.err, MOE_DEVERR_RANGE);
        } else {
          // the two 128-row output blocks one after the other (16 accumulator
          // registers live instead of 32); the second block exists for the
          // whole warp or for none of it: f0 is a multiple of 256 and H of 128
          float *yp = a.y + (row0 + j0) * NOUT + f;
          uint32_t v[16];
          tmem_ld16(tbase + j0, v);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (j0 + jj < j_hi) yp[jj * NOUT] = __uint_as_float(v[jj]) * unscale0;
          if (tl.f0 + 2 * BM <= NOUT) {
            tmem_ld16(tbase + BN + j0, v);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (j0 + jj < j_hi) yp[jj * NOUT + BM] = __uint_as_float(v[jj]) * unscale1;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tmem_empty[b]);
    }
  } else if (warp == MMA_WARP) {
    // ================================================================ MMA issuer
    // Per k-step: one handoff from the waiter (count = n16 = MMA width / 16,
    // 1..16, or > 16 to stop), then the MMAs and commits from one elected
    // lane. Tile boundaries are found by counting k-steps.
    int ks = 0, tl_i = 0;
    for (int it = 0; it < iters; ++it) {
      const uint32_t v = handoff(0);
      if (v > 16) break;
      tc_fence_after();
      const int s = it % C::S, b = tl_i % C::NBUF;
      const uint32_t idesc = idesc_f16(int(v) * 16);
      const uint32_t d0 = tmem + b * C::ACC_COLS;
      const uint64_t bdesc = sw128_desc(smem_u32(ringB + s * C::B_BYTES));
      const uint64_t adesc0 = sw128_desc(smem_u32(ringA + s * C::A_BYTES));
      if (elect_one()) {
#pragma unroll
        for (int m = 0; m < C::NMAT; ++m) {
          const uint64_t adesc = adesc0 + uint64_t((m * (BM * BK * 2)) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_f16(d0 + m * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) != 0);
        }
        mma_commit(&sh.s_free[s]);
        if (ks + 1 == KS) mma_commit(&sh.tmem_full[b]);
      }
      __syncwarp();
      if (++ks == KS) { ks = 0; ++tl_i; }
    }
    // all issued MMAs have completed before tensor memory is released
    if (elect_one()) mma_commit(&sh.drain);
    __syncwarp();
    wait_bounded(sh, &sh.drain, 0, a.err, true);
    __syncwarp();
  } else if (warp == WAITER_WARP) {
    // ================================================================ waiter
    // For each k-step of the MMA warp: (at a tile's first k-step) its
    // accumulator buffer has been drained by the epilogue, then the stage's
    // B rows have landed and its A tile is written; every wait bounded. The
    // handoff carries n16 = MMA width / 16 (lanes below n16 vote), plus 16
    // votes (lanes 16-31) when a wait failed, after which both warps stop.
    int ks = 0, tl_i = 0, n16 = 1;
    for (int it = 0; it < iters; ++it) {
      bool ok = true;
      if (ks == 0) {
        const Tile tl = decode_tile<C::FW>(sh, E, FT, sched_pos(tl_i));
        n16 = max(1, (tl.nvalid + 15) >> 4);
        ok = wait_bounded(sh, &sh.tmem_empty[tl_i % C::NBUF], ((tl_i / C::NBUF) & 1) ^ 1, a.err);
      }
      const int s = it % C::S;
      ok = ok && wait_bounded(sh, &sh.b_loaded[s], (it / C::S) & 1, a.err) &&
           wait_bounded(sh, &sh.a_full[s], (it / C::S) & 1, a.err);
      ok = __all_sync(0xffffffffu, ok);
      handoff(lane < n16 || (!ok && lane >= 16));
      if (!ok) break;
      if (++ks == KS) { ks = 0; ++tl_i; }
    }
  } else if (warp == TMA_CODES_WARP || warp == TMA_B_WARP) {
    // ================================================================ TMA
    // converged warp; every lane waits, one elected lane issues
    const bool codes = warp == TMA_CODES_WARP;
    const int RING = codes ? C::CS : C::S;
    uint64_t *loaded = codes ? sh.c_loaded : sh.b_loaded;
    uint64_t *freed = codes ? sh.c_free : sh.s_free;
    int cur = -1, ks = 0, row_b = 0, f0 = 0, slot = 0, issued = 0;
    bool ok = true;
    for (int it = 0; it < iters && ok; ++it, ++ks) {
      const int s = it % RING;
      ok = __all_sync(0xffffffffu, wait_bounded(sh, &freed[s], ((it / RING) & 1) ^ 1, a.err));
      if (!ok) break;
      if (cur < 0 || ks == KS) {
        ks = 0;
        ++cur;
        const Tile tl = decode_tile<C::FW>(sh, E, FT, sched_pos(cur));
        slot = a.expert_slot ? a.expert_slot[tl.e] : tl.e;
        row_b = tl.lo + tl.n0;  // first activation row of the tile, in group order
        f0 = tl.f0;
      }
      if (elect_one()) {
        if (codes) {
          uint8_t *dst = ringC + s * C::C_BYTES;
          mbar_arrive_expect_tx(&loaded[s], C::C_BYTES);
          tma_load_3d(dst, &tm_q0, ks * (BK / 2), f0, slot, &loaded[s]);
          tma_load_3d(dst + BM * (BK / 2), &tm_q1, ks * (BK / 2), f0 + (GATEUP ? 0 : BM), slot, &loaded[s]);
        } else {
          mbar_arrive_expect_tx(&loaded[s], C::B_BYTES);
          tma_load_2d(ringB + s * C::B_BYTES, &tm_b, ks * BK, row_b, &loaded[s]);
        }
      }
      __syncwarp();
      issued = it + 1;
    }
    // every issued copy has landed before shared memory is released
    for (int j = (issued > RING ? issued - RING : 0); j < issued; ++j)
      wait_bounded(sh, &loaded[j % RING], (j / RING) & 1, a.err, true);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

}  // namespace tc

int sm_count() {
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

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// FP16 rows [rows][cols] (cols contiguous), box 64 x 256 with the 128-byte
// swizzle the MMA descriptors expect; rows past the end read as zero.
static bool map_rows_f16(CUtensorMap *m, const void *base, int rows, int cols) {
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  const cuuint32_t box[2] = {tc::BK, tc::BN};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed codes of one matrix in every record of the bank: bytes
// [n_slots][nout][kd/2], box 32 bytes x 128 rows x 1 record, no swizzle.
static bool map_codes(CUtensorMap *m, const uint8_t *bank, int64_t off, int64_t rec, int n_slots, int nout, int kd) {
  const cuuint64_t dims[3] = {cuuint64_t(kd / 2), cuuint64_t(nout), cuuint64_t(n_slots)};
  const cuuint64_t strides[2] = {cuuint64_t(kd / 2), cuuint64_t(rec)};
  const cuuint32_t box[3] = {tc::BK / 2, tc::BM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(bank + off), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  if (!tensor_map_encoder())
    return set_error(MOE_ERR_UNSUPPORTED, "moe_grouped_w4a16_ffn: cuTensorMapEncodeTiled is not available");
  const int P = a.T * a.k;
  CUtensorMap tm_xs, tm_h, tm_gq, tm_uq, tm_dq;
  if (!map_rows_f16(&tm_xs, a.xs, P, a.H) || !map_rows_f16(&tm_h, a.h, P, a.I) ||
      !map_codes(&tm_gq, a.bank, a.off_gq, a.rec, a.n_slots, a.I, a.H) ||
      !map_codes(&tm_uq, a.bank, a.off_uq, a.rec, a.n_slots, a.I, a.H) ||
      !map_codes(&tm_dq, a.bank, a.off_dq, a.rec, a.n_slots, a.H, a.I))
    return set_error(MOE_ERR_INVALID_ARG, "moe_grouped_w4a16_ffn: tensor map encoding failed (pointers or strides)");
  const int grid = sm_count();
  int st0 = launch_gather_x_f16(a, s);
  if (st0 != MOE_OK) return st0;
  const size_t smem_gu = tc::Cfg<true>::SMEM, smem_dn = tc::Cfg<false>::SMEM;
  int st = allow_dynamic_smem(reinterpret_cast<const void *>(tc::tc_ffn_kernel<true>), smem_gu, "ffn tc gate/up");
  if (st != MOE_OK) return st;
  st = allow_dynamic_smem(reinterpret_cast<const void *>(tc::tc_ffn_kernel<false>), smem_dn, "ffn tc down");
  if (st != MOE_OK) return st;
  cudaError_t e = launch_pdl(tc::tc_ffn_kernel<true>, dim3(grid), dim3(tc::THREADS), smem_gu, s, a, tm_xs, tm_gq, tm_uq);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (tc gate/up): %s", cudaGetErrorString(e));
  st = check_launch("moe_grouped_w4a16_ffn (tc gate/up)");
  if (st != MOE_OK) return st;
  e = launch_pdl(tc::tc_ffn_kernel<false>, dim3(grid), dim3(tc::THREADS), smem_dn, s, a, tm_h, tm_dq, tm_dq);
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "moe_grouped_w4a16_ffn (tc down): %s", cudaGetErrorString(e));
  return check_launch("moe_grouped_w4a16_ffn (tc down)");
}

}  // namespace moe
