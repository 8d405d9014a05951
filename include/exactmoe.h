/*
 * exactmoe.h — C ABI of the fused grouped W4A16 routed-expert MoE layer.
 *
 * Method: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference"
 * (A. Saab, arXiv 2608.15383). The Abstract fixes four-bit symmetric
 * quantisation in groups of 128 for the routed experts only, a BF16 router
 * whose top-k is left as it was, and fused grouped expert kernels fed by a
 * slot cache on the GPU over experts kept in pinned host memory. The Figure 1
 * caption fixes the order of the steps: the experts are packed ahead of time;
 * the BF16 router picks experts; the tokens are gathered per chosen expert;
 * fused grouped kernels run the active experts; a cache miss copies packed
 * codes and scales, and no FP16 copy of an expert is ever made.
 *
 * Conventions for every entry point below:
 *  - Pointers are DEVICE pointers unless a parameter says "host". The caller
 *    owns every buffer; no hot-path call allocates device memory. Scratch
 *    space is passed in as a workspace whose size the *_workspace_size
 *    functions return.
 *  - BF16 values travel as raw 16-bit patterns (moe_bf16).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and never synchronise, except moe_read_device_error.
 *  - Every call returns MOE_OK or an error status; moe_last_error() gives a
 *    message for the calling host thread. A failed argument check launches
 *    nothing. Errors found on the device (an expert id out of range, an expert
 *    that is not resident) are written to the first word of the workspace,
 *    where the first one stays until moe_read_device_error reads and clears
 *    it; zero a workspace once before its first use.
 *  - Kernels are launched with programmatic dependent launch, so each one's
 *    launch overlaps the tail of the previous kernel on the stream; each
 *    waits for its predecessor's results before reading them.
 *  - Shapes: hidden H and expert intermediate I are multiples of 128 (the
 *    quantisation group); 1 <= E <= 256 experts; 1 <= k <= min(E, 32).
 *
 * Packed weight format (defined by this library; the pages' MARLIN format is
 * prior art for a different GPU): for an nn.Linear weight W[N][K] (out x in),
 *  - scale s[n][g] = bf16_rn(absmax(W[n][128g .. 128g+127]) / 7), fp32 divide;
 *  - code q[n][k] = clamp(rint(W[n][k] / s[n][k/128]), -8, 7), fp32 divide,
 *    ties to even, q = 0 where s = 0; stored offset-binary u = q + 8;
 *  - row n of the packed matrix is K/2 bytes = K/8 little-endian 32-bit words;
 *    word j holds k in [8j, 8j+8), with k = 8j + 2i + h (i = 0..3, h = 0..1)
 *    at bits [4(i + 4h), 4(i + 4h) + 4). Shifting a word right by 4i and
 *    masking 0x000F000F yields the codes of k = 8j+2i and 8j+2i+1 in the two
 *    16-bit halves, which is what the kernels' in-register dequant consumes;
 *  - scales are row-major [N][K/128] BF16.
 * One expert is one record: gate [I][H/2], up [I][H/2], down [H][I/2] packed
 * bytes, then the gate, up and down scales (moe_expert_record_layout gives
 * the offsets). A bank is an array of records with a fixed stride; a slot is
 * one record of a bank.
 */
#ifndef EXACTMOE_H
#define EXACTMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;   /* raw BF16 bit pattern */
typedef void *moe_stream_t;  /* a cudaStream_t */

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad flag, buffer too small */
  MOE_ERR_SHAPE = 2,       /* shape outside the supported range */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  MOE_ERR_CAPACITY = 4,    /* more distinct experts than cache slots */
  MOE_ERR_DEVICE = 5,      /* a kernel flagged bad data (see device codes) */
  MOE_ERR_UNSUPPORTED = 6  /* no path for this request on this device */
};

/* Device error codes written to workspace word 0 (first writer wins). */
enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_EXPERT_ID = 1,   /* a top-k id outside [0, E) */
  MOE_DEVERR_NOT_RESIDENT = 2,/* an active expert has no valid slot */
  MOE_DEVERR_TIMEOUT = 3,     /* a bounded pipeline wait ran out */
  MOE_DEVERR_RANGE = 4        /* an activation x or an expert intermediate h
                                 outside FP16's finite range (|v| > 65504):
                                 the FFN's FP16 operand copies cannot hold it */
};

/* Message for the last failed call on this host thread ("" if none). */
const char *moe_last_error(void);

/* ABI version, bumped on any incompatible change. */
int moe_abi_version(void);

/* Number of kernels this library has enqueued in this process (a host-side
 * count taken at each launch site; a CUDA graph captured from these calls
 * replays its kernels without counting again). */
uint64_t moe_launch_counter(void);

/* Byte offsets of the six parts of one expert record, and its size.
 * All offsets are multiples of 256 bytes. */
typedef struct {
  int64_t gate_q, up_q, down_q; /* packed codes */
  int64_t gate_s, up_s, down_s; /* BF16 scales */
  int64_t bytes;                /* record size */
} moe_record_layout;

int moe_expert_record_layout(int H, int I, moe_record_layout *out);

/*
 * A1 — quantise and pack (Abstract: symmetric group-128 int4 weights for the
 * routed experts; Figure 1 caption: packing happens a single time, offline).
 *   w       [E][N][K] BF16, one nn.Linear weight per expert (K = in).
 *   packed  expert e's codes at packed + e*packed_stride, [N][K/2] bytes.
 *   scales  expert e's scales at (char*)scales + e*scales_stride, [N][K/128].
 * Strides are in bytes (packed a multiple of 4, scales of 2; ignored when
 * E == 1), so the output can land directly in the records of a bank.
 * w must be 8-byte, packed 4-byte and scales 2-byte aligned. K % 128 == 0,
 * N >= 1. Bit-exact with the format defined above.
 */
int moe_quantize_pack(const moe_bf16 *w, int E, int N, int K,
                      uint8_t *packed, int64_t packed_stride,
                      moe_bf16 *scales, int64_t scales_stride,
                      moe_stream_t stream);

/* Flags of moe_route_topk. */
#define MOE_RENORM 1       /* divide the k weights by their sum */
#define MOE_LOGITS_GIVEN 2 /* read `logits` instead of computing them */
#define MOE_IDS_GIVEN 4    /* read `topk_ids`, only produce their weights */

/*
 * A2 + A3 — BF16 router logits, full softmax and unchanged top-k
 * (Abstract: the router stays BF16 and top-k routing is left as it was;
 * Figure 1 caption: the model's own BF16 router picks the experts).
 *   x         [T][H] BF16 activations.
 *   w_router  [E][H] BF16 (nn.Linear convention).
 *   bias      [E] fp32 added to the logits before softmax/top-k, or NULL.
 *   logits    [T][E] BF16: written (fp32 sum rounded to BF16), or read when
 *             MOE_LOGITS_GIVEN is set.
 *   topk_ids  [T][k] int32: the k largest keys fp32(logit)+bias (NaN counts
 *             as -inf), ties to the lower index, ordered by descending key
 *             then ascending index. Read instead when MOE_IDS_GIVEN is set
 *             (ids outside [0, E) get weight 0; moe_group_tokens flags them).
 *   topk_w    [T][k] fp32: softmax probabilities (over all E) of the ids,
 *             renormalised over the k when MOE_RENORM is set.
 * T may be 0 (no launch).
 */
int moe_route_topk(const moe_bf16 *x, const moe_bf16 *w_router,
                   int T, int H, int E, int k,
                   const float *bias, int flags,
                   moe_bf16 *logits, int32_t *topk_ids, float *topk_w,
                   moe_stream_t stream);

/*
 * moe_route_topk that also writes x16 [T][H], the FP16 copy of x that the
 * grouped FFN multiplies (pass it to moe_grouped_w4a16_ffn with
 * MOE_FFN_X_F16): for decode-sized T (<= 64) the router kernel converts the
 * rows it has already staged, so the FFN needs no conversion pass of its own;
 * otherwise a separate conversion kernel runs after the routing. x is
 * required (also with MOE_LOGITS_GIVEN), x16 must be 16-byte aligned. A value
 * v converts exactly when 2^-17 <= |v| <= 65504 or v = 0; smaller magnitudes
 * round to a multiple of 2^-24; a larger one sets MOE_DEVERR_RANGE in *err
 * (a device int32 error word, e.g. word 0 of the FFN workspace, which
 * moe_read_device_error reads; NULL: not reported).
 */
int moe_route_topk_x16(const moe_bf16 *x, const moe_bf16 *w_router,
                       int T, int H, int E, int k,
                       const float *bias, int flags,
                       moe_bf16 *logits, int32_t *topk_ids, float *topk_w,
                       uint16_t *x16, int32_t *err, moe_stream_t stream);

/*
 * A4 — group the T*k (token, slot) pairs by expert (Figure 1 caption: the
 * tokens are gathered per chosen expert).
 *   topk_ids    [T][k] int32.
 *   counts      [E] int32 pairs per expert.
 *   offsets     [E+1] int32 exclusive prefix sum of counts.
 *   sorted_pair [T*k] int32 flat pair indices p = t*k + j, ordered by expert
 *               and, within an expert, by p (a stable counting sort; the
 *               result is unique and deterministic).
 *   pair_pos    [T*k] int32 inverse: sorted_pair[pair_pos[p]] == p; -1 for a
 *               pair whose id is out of range (also flagged on the device).
 *   ws          workspace of at least moe_group_workspace_size(T, k, E) bytes,
 *               256-byte aligned, zeroed once before first use. Word 0 is the
 *               device error word.
 */
size_t moe_group_workspace_size(int T, int k, int E);
int moe_group_tokens(const int32_t *topk_ids, int T, int k, int E,
                     int32_t *counts, int32_t *offsets,
                     int32_t *sorted_pair, int32_t *pair_pos,
                     void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_group_tokens without a workspace, for callers that cannot allocate
 * device memory: code that runs under CUDA stream capture (where cudaMalloc
 * is not allowed), or inside a host framework that owns every device
 * allocation and offers no scratch space. (The paper has no counterpart;
 * this exists only for such callers.)
 *
 * Same arguments, outputs and results as moe_group_tokens minus ws/ws_bytes.
 * The scratch is a fixed array inside this library (about 64 KiB), which
 * every GPU that loads the library holds until the process exits; it allows
 * at most MOE_NOALLOC_MAX_PAIRS = T*k pairs (larger calls return
 * MOE_ERR_SHAPE and launch nothing). This call allocates nothing and calls no
 * cudaMalloc/cudaFree. It looks up the array's device address
 * (cudaGetSymbolAddress) with the current device on every call made outside
 * stream capture, so a device reset does not leave it stale; a call under
 * capture reuses the address found by the last call on that device, so make
 * the first call on a device before any stream capture. All calls share the
 * one array: calls whose kernels overlap on the GPU (other streams, other
 * host threads) race and corrupt each other's results, so serialise them.
 * Device-side errors are not reported through a workspace word here (the
 * array's error word is written but never read): a pair with an out-of-range
 * id gets pair_pos = -1, which the caller can check.
 */
#define MOE_NOALLOC_MAX_PAIRS 65536
int moe_group_tokens_noalloc(const int32_t *topk_ids, int T, int k, int E,
                             int32_t *counts, int32_t *offsets,
                             int32_t *sorted_pair, int32_t *pair_pos,
                             moe_stream_t stream);

/* expert_slot value of an expert that a grouped FFN call leaves to another
 * call (another wave of the same step). */
#define MOE_SLOT_SKIP (-2)

/* FFN execution paths. */
#define MOE_PATH_AUTO 0 /* chosen from the average rows per expert, T*k/E */
#define MOE_PATH_GEMV 1 /* decode-sized groups: weight-streaming, HBM-bound */
#define MOE_PATH_TC 2   /* prefill-sized groups: tcgen05 tensor cores */
#define MOE_PATH_SEQUENTIAL 3 /* reference only: the GEMV kernels launched
                                 once per expert, expert after expert (the
                                 pages' sequential W4 baseline, Abstract) */
#define MOE_FFN_X_F16 0x100   /* flag OR-ed into the path: x holds the FP16
                                 copy of the activations (moe_route_topk_x16)
                                 instead of BF16, so no conversion pass runs */

/*
 * A5 + A6 — the grouped SwiGLU expert FFN with in-kernel int4 dequantisation
 * (Abstract: fused grouped kernels over W4A16 experts; Figure 1 caption:
 * the kernels read packed codes and scales, with no FP16 copy of an expert).
 * For sorted row r of expert e (offsets[e] <= r < offsets[e+1]) and token
 * t = sorted_pair[r] / k:
 *   h[r] = bf16_rn(silu(x[t] Wg_e^T) * (x[t] Wu_e^T))      (fp32 sums)
 *   y[r] = h[r] Wd_e^T                                      (fp32 sums, fp32)
 *   x            [T][H] BF16, or FP16 when the path carries MOE_FFN_X_F16.
 *   bank         device array of expert records with stride record_bytes
 *                (moe_expert_record_layout(H, I).bytes or larger, multiple
 *                of 256).
 *   expert_slot  [E] int32 record index of each expert in the bank, or NULL
 *                for the identity (record e holds expert e). An expert marked
 *                MOE_SLOT_SKIP is not computed by this call (its rows of y
 *                are left as they are: another call of the same step, one
 *                wave of a slot cache, computes them). An active expert with
 *                any other slot outside [0, n_slots) is skipped and flagged
 *                (MOE_DEVERR_NOT_RESIDENT).
 *   y            [T*k][H] fp32, rows in sorted order (the expert outputs
 *                are kept unrounded until the combine).
 *   ws           at least moe_ffn_workspace_size(T, k, E, H, I, path) bytes,
 *                256-byte aligned, zeroed once before first use; holds the
 *                error word, h and (tensor-core path) an FP16 copy of x.
 * Both paths sum products of the weights q*s and FP16 copies of the
 * activations (x, and h for the down pass) in fp32. A BF16 value v copies to
 * FP16 exactly when 2^-17 <= |v| <= 65504 or v = 0; a smaller magnitude
 * rounds to a multiple of 2^-24 (absolute error <= 2^-25), and a larger one
 * is flagged MOE_DEVERR_RANGE (for h as well as x; the affected rows are then
 * not meaningful). The GEMV path multiplies FP16 codes q and applies each
 * group's scale to the fp32 partial sum over that group, exact for every
 * scale. The tensor-core path dequantises q*s*2^a to FP16, with a per-row
 * power of two 2^a that brings the row's largest scale to [2^-4, 2^-3) and is
 * undone exactly on the fp32 sum: exact for every group whose scale is at
 * least 2^-13 of its row's largest (smaller ones are rounded to a multiple of
 * 2^-24 relative to that normalisation).
 */
size_t moe_ffn_workspace_size(int T, int k, int E, int H, int I, int path);
int moe_grouped_w4a16_ffn(const moe_bf16 *x, const int32_t *sorted_pair,
                          const int32_t *offsets, const void *bank,
                          int64_t record_bytes, const int32_t *expert_slot,
                          int n_slots, int T, int k, int E, int H, int I,
                          int path, float *y, void *ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * The BF16 grouped expert FFN (the pages' BF16 baseline, Abstract and
 * Table 1): the same grouped SwiGLU with unquantised BF16 experts, for
 * measuring what the int4 packing buys. Not part of the W4A16 path.
 * A BF16 record holds gate [I][H], up [I][H] and down [H][I] BF16 weights
 * (nn.Linear layout) at the offsets moe_bf16_record_layout gives (multiples
 * of 256). For sorted row r of expert e and token t = sorted_pair[r] / k:
 *   h[r] = bf16_rn(silu(x[t] Wg_e^T) * (x[t] Wu_e^T))  (fp32 sums, h in BF16)
 *   y[r] = h[r] Wd_e^T                                  (fp32 sums, fp32)
 * Arguments as moe_grouped_w4a16_ffn (identity expert -> record mapping);
 * ws holds the error word and h.
 */
typedef struct {
  int64_t gate, up, down; /* byte offsets of the three matrices */
  int64_t bytes;          /* record size */
} moe_bf16_layout;

int moe_bf16_record_layout(int H, int I, moe_bf16_layout *out);
size_t moe_bf16_ffn_workspace_size(int T, int k, int E, int H, int I);
int moe_grouped_bf16_ffn(const moe_bf16 *x, const int32_t *sorted_pair,
                         const int32_t *offsets, const void *bank,
                         int64_t record_bytes, int T, int k, int E, int H,
                         int I, float *y, void *ws, size_t ws_bytes,
                         moe_stream_t stream);

/*
 * Test hook for the failure path of the tensor-core FFN: the next `calls`
 * tensor-core launches run with producers that never publish a stage, so the
 * kernels' bounded waits (about two seconds each) run out, the kernels drain
 * and return, and MOE_DEVERR_TIMEOUT is left in the workspace error word. The
 * GPU context stays usable. Not for production use.
 */
int moe_debug_stall_next_tc_ffn(int calls);

/*
 * A7 — router-weighted combine (implied by the MoE layer; the pages do not
 * spell it out):
 *   out[t] = bf16_rn(residual[t] + sum_{j=0..k-1} topk_w[t][j] * y[pair_pos[t*k+j]])
 * with y the fp32 expert outputs [T*k][H], summed in fp32 in increasing j.
 * residual may be NULL (zero); pairs with pair_pos < 0 contribute nothing.
 * out may alias residual.
 */
int moe_combine(const float *y, const float *topk_w,
                const int32_t *pair_pos, const moe_bf16 *residual,
                int T, int k, int H, moe_bf16 *out, moe_stream_t stream);

/*
 * Synchronises `stream`, reads the device error word of a workspace written
 * by moe_group_tokens or moe_grouped_w4a16_ffn, clears it, and returns
 * MOE_OK or MOE_ERR_DEVICE (the code is stored in *code if code != NULL).
 */
int moe_read_device_error(void *ws, moe_stream_t stream, int32_t *code);

/*
 * A8 — expert slot cache on the GPU over a pinned host pool (Abstract: the
 * experts live in pinned host memory and a slot cache of configurable size
 * holds some of them on the GPU; Figure 1 caption: the host pool holds every
 * packed expert and a miss copies its packed codes and scales; Figure 2
 * caption: once the cache holds all E experts no hit rate is counted).
 *
 * The cache owns only host bookkeeping (an LRU per layer) and two CUDA
 * events per layer; all memory is the caller's:
 *   pinned_pool   host, page-locked, [layers][E] records of record_bytes.
 *   device_slots  device, [layers][slots] records of record_bytes.
 *   expert_slot   device, [layers][E] int32, the table the FFN reads.
 *                 slot_cache_fill writes it for the layer's last lookup: the
 *                 looked-up experts' slots; MOE_SLOT_SKIP for the other
 *                 experts of a step planned by slot_cache_plan_waves; -1 for
 *                 every other expert (flagged by the FFN if a token selects
 *                 it). Initialise it to -1.
 * With all three NULL the cache only simulates the policy (no CUDA call is
 * made): slot_cache_fill counts the misses' bytes as copied and copies
 * nothing, slot_cache_release does nothing. Hit rates and traffic of a
 * routing trace can be measured that way without a GPU.
 *
 * Replacement policy (the pages name none; this is the library's reading):
 * a step's distinct ids are taken in first-occurrence order; ids already held
 * are hits and their slots are protected for the step; each miss takes the
 * lowest empty slot, else the least recently used unprotected slot, the lower
 * slot index on ties.
 */
typedef struct moe_slot_cache moe_slot_cache;

int slot_cache_create(moe_slot_cache **out, int layers, int E, int slots,
                      int64_t record_bytes, const void *pinned_pool,
                      void *device_slots, int32_t *expert_slot);

/* Looks up the n expert ids (host) one step needs in `layer`. For each id
 * writes its slot (host slot_of_id[n]); misses are assigned a victim slot,
 * the least recently used slot that this step does not need, and listed in
 * miss_ids (host, capacity n). Duplicate ids count once. More distinct ids
 * than slots -> MOE_ERR_CAPACITY. Resident caches (slots >= E) never miss
 * and count nothing. If the layer's previous lookup assigned slots that no
 * successful slot_cache_fill copied, those assignments are undone first
 * (the experts count as absent again). */
int slot_cache_lookup(moe_slot_cache *c, int layer, const int32_t *ids_host,
                      int n, int32_t *slot_of_id_host,
                      int32_t *miss_ids_host, int *n_miss);

/* Copies the records of the missed experts from the pinned pool into their
 * slots on `side` (one cudaMemcpyAsync each, after the layer's previous
 * readers released it), makes `compute` wait for the copies, and rewrites the
 * layer's device expert_slot table on `compute` when it changes (a one-block
 * kernel). Call it after every lookup, also with n_miss = 0. */
int slot_cache_fill(moe_slot_cache *c, int layer, const int32_t *miss_ids_host,
                    int n_miss, moe_stream_t side, moe_stream_t compute);

/* Marks the end of this step's reads of `layer`'s slots on `compute`; the
 * next fill of the layer waits for this point before overwriting a slot. */
int slot_cache_release(moe_slot_cache *c, int layer, moe_stream_t compute);

/*
 * Cache-sized waves (Figure 1 caption: the active experts run in waves sized
 * to the cache). Splits the n expert ids (host) one step of
 * `layer` needs into waves of at most `slots` distinct experts: the
 * distinct ids in first-occurrence order, those already held in a slot
 * first (so they run before anything can evict them), cut into consecutive
 * waves. Writes the ordered ids to wave_ids (host, capacity n), the start of
 * wave w to wave_start[w] (host, capacity n + 1; wave_start[n_waves] is the
 * total) and the count to *n_waves (0 when n == 0). Per wave: lookup of its
 * ids, fill, one grouped FFN call with the same grouping of the whole step
 * (it computes only that wave's experts), release; the combine follows the
 * last wave. Planning marks the step's experts so that each wave's table
 * skips the others; call it at the start of every step run in waves.
 */
int slot_cache_plan_waves(moe_slot_cache *c, int layer, const int32_t *ids_host, int n,
                          int32_t *wave_ids_host, int32_t *wave_start_host, int *n_waves);

int slot_cache_stats(const moe_slot_cache *c, uint64_t *hits,
                     uint64_t *misses, uint64_t *h2d_bytes);

/* Test hook: the next `count` fills fail with MOE_ERR_CUDA before copying
 * (host-side fault injection; no device is touched). */
int slot_cache_inject_fill_failure(moe_slot_cache *c, int count);

void slot_cache_destroy(moe_slot_cache *c);

/*
 * The packed pool as a file, so the packing is done a single time (Figure 1
 * caption: the experts are quantised and packed ahead of time, and the pinned
 * host pool holds every packed expert). Host-only calls (no CUDA),
 * so a pool can be written once and reloaded into pinned memory, a bank or
 * a slot cache's pool without re-quantising.
 *   pool    host, [layers][E] records of record_bytes, the layout of a bank
 *           (records as moe_quantize_pack writes them).
 * File: a 64-byte little-endian header (magic "EXMOEPK1", format version 1,
 * header size, layers, E, H, I, record_bytes, payload bytes, and a 64-bit
 * FNV-1a checksum of the payload taken as little-endian 64-bit words), then
 * the records. moe_pool_save writes path.tmp and renames it over path.
 * moe_pool_load checks the header, the shape, the buffer's capacity (bytes),
 * the file's length and the checksum, and returns MOE_ERR_INVALID_ARG with a
 * message on any mismatch (MOE_ERR_UNSUPPORTED for another format version).
 */
typedef struct {
  int32_t layers, E, H, I;
  int64_t record_bytes; /* >= moe_expert_record_layout(H, I).bytes, multiple of 256 */
} moe_pool_info;

int moe_pool_save(const char *path, const moe_pool_info *info, const void *pool_host);
int moe_pool_file_info(const char *path, moe_pool_info *info);
int moe_pool_load(const char *path, void *pool_host, size_t capacity_bytes, moe_pool_info *info);

#ifdef __cplusplus
}
#endif

#endif /* EXACTMOE_H */
