// moe_internal.h -- layouts shared by the host runtime and the kernels of libmoe.
//
// Expert slot layout (device slot pool and pinned host tier alike).  An expert of
// SwiGLU width W is W/32 "units"; unit rb holds everything the decode kernel needs to
// turn rows 32rb..32rb+31 of the SwiGLU activation into that block's share of the
// expert's output, as one contiguous run of 54H bytes:
//
//   [0, 36H)    gate/up: four tiles of 9H bytes, gate rows 32rb..+15, gate rows
//               32rb+16..+31, up rows 32rb..+15, up rows 32rb+16..+31; a tile is
//               [16 rows x H/32 blocks x 16 nibble bytes][16 rows x H/32 fp16 scales]
//   [36H, 52H)  down nibbles: for every output row j of H, the 16 bytes of Q4_0 block
//               rb of down row j (columns 32rb..32rb+31 of the width)
//   [52H, 54H)  down scales: the fp16 scale of the same block of every row j
//
// The canonical Q4_0 block (GGUF convention: fp16 scale d + 16 bytes, byte j = weight j
// in the low nibble and weight j+16 in the high nibble; weight = (q - 8) d) is moved
// byte for byte, never changed, so a slot is the same expert wherever it lives and full
// residency stays bit-identical to partial residency.
#pragma once
#include <stdint.h>

namespace moe {

constexpr int kThreads = 256;  // threads per CTA of the decode kernel
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 16;     // columns per canonical router / norm chunk
constexpr int kUnitRows = 32;  // SwiGLU rows per work unit (one Q4_0 block of the activation)
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxR = 32;
constexpr int kMaxH = 4096;
constexpr int kMboxCap = 256;  // miss-request mailbox entries
constexpr int kAccBufs = 3;    // rotating per-layer output accumulators
constexpr int kMaxLikely = 32; // likely experts per layer the kernel may load ahead of routing
constexpr int kMaxPreload = 16;  // of which preloaded into shared memory
// Fixed-point scale of the per-layer output accumulator: every unit adds its share of
// y as round(v * 2^28) into 64-bit integers, so the sum does not depend on the order in
// which units finish.  A share must satisfy |v| < 2^26 (else MOE_DEVERR_RANGE).
constexpr float kAccScale = 268435456.0f;        // 2^28
constexpr float kAccInvScale = 1.0f / 268435456.0f;
constexpr float kAccLimit = 67108864.0f;         // 2^26

// Bytes of one Q4_0 matrix [rows x cols] in the slot layout (== canonical size).
inline constexpr uint64_t q4_bytes(uint64_t rows, uint64_t cols) {
  return rows * cols / 32 * 18;
}

struct SlotLayout {
  uint64_t unit;   // bytes of one unit: 54H
  uint64_t bytes;  // slot bytes: (W/32) units, rounded up to 256
};

inline SlotLayout slot_layout(int H, int W) {
  SlotLayout s;
  s.unit = 54ull * H;
  s.bytes = ((uint64_t)(W / 32) * s.unit + 255) / 256 * 256;
  return s;
}

// Offsets inside a unit.
inline constexpr uint64_t unit_gu_tile(int H, int st) { return (uint64_t)st * 9 * H; }
inline constexpr uint64_t unit_down_nib(int H) { return 36ull * H; }
inline constexpr uint64_t unit_down_scl(int H) { return 52ull * H; }

// One miss request in the host-mapped mailbox.  The kernel fills the fields, then
// publishes seq last; the proxy thread copies expert (layer, expert) of the pinned host
// tier into pool slot dst_slot and then writes seq to the device word done_seq.
struct MissReq {
  uint32_t seq;
  uint32_t layer;
  uint32_t expert;
  uint32_t dst_slot;
};

// Device control block (one per context).  The words every CTA polls live on cache
// lines of their own so that polling one does not slow the atomics on another.
struct alignas(128) Ctrl {
  uint32_t step;     // decode steps completed
  uint32_t req_seq;  // miss requests issued so far
  uint32_t pad0[30];
  int32_t error;  // MOE_DEVERR_* or 0
  uint32_t pad1[31];
  uint32_t bar_count;  // arrivals: one per CTA after the prologue and after each layer; zeroed before every launch
  uint32_t pad2[31];
  unsigned long long pin_hits, ring_hits, misses, evictions, staged, pulled;
};

// Miss-path variants.
constexpr int kMissProxy = 0;  // host proxy thread + copy engine (cudaMemcpyAsync on a side stream)
constexpr int kMissPull = 1;   // the unit CTAs read the expert from mapped pinned host memory

struct DecodeParams {
  // shape
  int L, H, E, K, I, Is, R, use_norm;
  float eps;
  int n_units;     // K * I / 32 + Is / 32
  int rx_per_cta;  // router experts per CTA: ceil(E / grid)
  int down_late;   // 1: a unit's down part is loaded after its gate/up part (large H)
  int miss_mode;   // kMissProxy or kMissPull
  int nan_on_error;  // 1: a launch that fails writes NaN to y (callers without moe_sync)
  // weights
  const uint8_t* pool;  // slot pool
  uint64_t slot_bytes;
  uint64_t unit_bytes;  // 54H
  const uint8_t* shared_pool;  // [L] shared slots
  uint64_t shared_slot_bytes;
  const uint16_t* router;  // [L][E][H] bf16 rows
  const float* bias;       // [L][E] or null
  const float* gain;       // [L][H] or null
  // cache tables
  const int32_t* pin_slot;    // [L][E] (logical slot << 16) | physical pinned slot, or -1
  const int32_t* layer_base;  // [L] pool index of the layer's pinned slot 0
  const int32_t* n_pinned;    // [L]
  int32_t* ring_owner;        // [2][L][R]
  uint32_t* ring_stamp;       // [2][L][R]
  uint32_t* ring_clock;       // [2][L]
  int32_t staging_base;       // pool index of staging slot 0 (k of them)
  // io
  const float* x;
  float* y;
  float* h_trace;  // [(L+1)][H] or null
  float* w_trace;  // [L][K] or null
  // exchange scratch
  unsigned long long* acc;  // [kAccBufs][H] fixed-point layer outputs
  unsigned long long* zll;  // [E] published logits: (epoch << 32) | float bits
  // stats
  uint32_t* hist;  // [L][E]
  int32_t* log;    // [log_steps][L][K][7]
  int log_steps;
  Ctrl* ctrl;
  // miss path
  MissReq* mbox;                 // host-mapped, kMboxCap entries (proxy mode)
  const uint32_t* done_seq;      // device word, written by the proxy's stream
  const uint8_t* host_tier;      // device view of the mapped pinned host tier (pull mode)
  unsigned long long timeout_ns;
  unsigned long long* phase_trace;  // see moe_set_phase_trace, or null
  // speculative loads while a layer's routing runs, from its most frequently routed
  // pinned experts in order ([L][kMaxLikely] pool slots and expert ids, -1 = none): the
  // first n_pre are preloaded unit by unit into the shared memory of CTAs 0..n_pre*I/32-1,
  // the next n_l2 are prefetched into L2
  const int32_t* likely_slot;
  const int32_t* likely_e;
  int n_pre, n_l2;
};

// Words of the phase trace for L layers on a grid of n CTAs.
inline uint64_t phase_trace_words(int L, int n) { return (uint64_t)(L + 1) * 32 + (uint64_t)L * n * 4; }

}  // namespace moe
