// prefill.h -- host-side interface of the batched prefill kernels (prefill.cu) for the
// runtime (moe_api.cu).  Plain structs of device pointers and sizes.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {

// Model and weights (all resident): what the runtime owns.
struct PrefillArgs {
  int L, H, E, K, I, Is, use_norm, T;
  int n_sm;  // the device's SM count: persistent GEMM grids
  float eps;
  const uint8_t* pool;
  int64_t pool_slots;  // slots in the pool (the weight tensor maps' extent)
  uint64_t slot_bytes;
  SlotLayout lay, slay;
  const uint8_t* shared_pool;
  uint64_t shared_slot_bytes;
  const float* bias;       // [L][E] or null
  const float* gain;       // [L][H]
  const int32_t* pin_slot;    // [L][E], every entry valid
  const int32_t* layer_base;  // [L]
  uint32_t* hist;             // [L][E] routing histogram, accumulated
  const uint16_t* router_rows;  // [L][E][H] bf16, the router in plain row order
  const float* wnorm;           // [L] max_e ||w_e||_2, rounded up
};

// Per-call device buffers for T tokens (R = T * K + T rows when there is a shared
// expert, else T * K).
struct PrefillScratch {
  float* h;          // [T][H] residual stream; holds x on entry
  float* y;          // [T][H] output (caller's)
  float* h_trace;    // [(L+1)][T][H] or null
  int32_t* sel_trace;  // [L][T][K] or null
  int32_t* sel;      // [T][K]
  float* u;          // [T][H] router input u = g * h (or h)
  __nv_bfloat16* ua; // [T][3H] u split into three bf16 parts
  float* inv;        // [T] RMSNorm scale
  float* unorm;      // [T] ||u||_2, rounded up
  float* part;       // [8][T][E] router partial sums per K split
  float* w;          // [T][K]
  __half *x_hi, *x_lo;    // [T][H]
  __half *xg_hi, *xg_lo;  // [R][H]
  __half *a_hi, *a_lo;    // [R][max(I, Is)]
  float* obuf;       // [H / 16][R][16] expert outputs over grouped rows
  int32_t* gpos;     // [T][K + 1] grouped row of each (token, rank)
  int32_t* counts;   // [E]
  int32_t* cursor;   // [E + 1]
  int32_t* offsets;  // [E + 2]
  int32_t* jobs;     // [R / 128 + E + 1]
  int32_t* n_jobs;   // [1]
  int32_t* error;    // device error word (MOE_DEVERR_*)
};

// 1 when the shape fits the prefill kernels (H % 128 == 0, I and Is % 64 == 0, ...).
int prefill_supported(int H, int E, int K, int I, int Is);
// Opt the kernels in to their shared-memory sizes (once per device).
cudaError_t prefill_configure(int H, int E);
// Enqueue the whole prefill on st (x already in s.h).  encode_fn: the driver's
// cuTensorMapEncodeTiled.  0, -1 when a tensor map could not be encoded, else a
// cudaError_t of a launch.
int prefill_run(const PrefillArgs& a, const PrefillScratch& s, void* encode_fn, cudaStream_t st);

}  // namespace moe
