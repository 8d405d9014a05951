// Shared declarations of the grouped W4A16 expert FFN paths.
#pragma once

#include "common.cuh"

namespace moe {

// Everything a grouped-FFN kernel needs, passed by value.
struct FfnArgs {
  const uint16_t *x;           // [T][H]
  const int32_t *sorted_pair;  // [P]
  const int32_t *offsets;      // [E+1]
  const uint8_t *bank;         // records of `rec` bytes
  const int32_t *expert_slot;  // [E] or nullptr (identity)
  int64_t rec;
  int n_slots;
  int T, k, E, H, I;
  int64_t off_gq, off_uq, off_dq, off_gs, off_us, off_ds;  // record layout
  uint16_t *h;    // [P][I] workspace, sorted order: the BF16-rounded value
                  // stored as FP16 (exact), the down pass's B operand
  uint16_t *x16;  // [T][H] FP16 copy of x, the decode path's gate/up input
  uint16_t *xs;   // [P][H] FP16 rows of x in group order (row r = token
                  // sorted_pair[r] / k), the tensor-core gate/up B operand;
                  // shares x16's workspace region
  float *y;       // [P][H] fp32 expert outputs, sorted order
  int32_t *err;   // device error word
  int stall;      // test hook: producers never publish a stage (bounded waits run out)
  int e0;         // first expert of the launch (blockIdx.y + e0; the sequential path launches one expert)
  int x_f16;      // x already holds FP16 values (MOE_FFN_X_F16): x16 = x and no conversion pass
  int compact;    // GEMV grid row y = the y-th expert with rows (few pairs, many experts), not expert y
};

// Test hook state (moe_debug_stall_next_tc_ffn): number of tensor-core FFN
// calls still to be launched with their producers stalled.
int take_tc_stall();

// Record of expert e, or nullptr if this call does not compute it: an expert
// marked MOE_SLOT_SKIP (another wave's) silently, any other slot outside
// [0, n_slots) with the error flagged.
__device__ __forceinline__ const uint8_t *expert_record(const FfnArgs &a, int e) {
  const int slot = a.expert_slot ? a.expert_slot[e] : e;
  if (slot < 0 || slot >= a.n_slots) {
    if (slot != MOE_SLOT_SKIP) flag_error(a.err, MOE_DEVERR_NOT_RESIDENT);
    return nullptr;
  }
  return a.bank + int64_t(slot) * a.rec;
}

int launch_x_to_f16(const FfnArgs &a, cudaStream_t s);
int launch_gather_x_f16(const FfnArgs &a, cudaStream_t s);
int launch_ffn_gemv(const FfnArgs &a, cudaStream_t s);
int launch_ffn_sequential(const FfnArgs &a, cudaStream_t s);
int launch_ffn_tc(const FfnArgs &a, cudaStream_t s);

}  // namespace moe
