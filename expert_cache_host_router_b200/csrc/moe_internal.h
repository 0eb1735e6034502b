// moe_internal.h -- layouts shared by the host runtime and the decode kernel of libmoe.
//
// Expert slot layout (device slot pool and pinned host tier alike).  The canonical
// Q4_0 blocks (GGUF convention: fp16 scale d + 16 bytes, byte j = weight j low nibble,
// weight j+16 high nibble) are regrouped into tiles of 16 matrix rows, each tile one
// contiguous run that a single bulk (TMA) copy brings into shared memory:
//
//   tile = [ qs: 16 rows x (K/32 blocks) x 16 bytes ][ d: 16 rows x (K/32) fp16 ]
//
//   gate/up part: for every 32-row block rb of the expert's width I, four tiles:
//     gate rows 32rb..+15, gate rows 32rb+16..+31, up rows 32rb..+15, up rows 32rb+16..+31
//     (K = H, 9H bytes each)
//   down part: for every 16-row chunk c of H, one tile of down rows 16c..16c+15
//     (K = I, 9I bytes each)
//
// Values are the canonical blocks' bytes moved, never changed, so a slot is the same
// expert wherever it lives and full residency stays bit-identical to partial residency.
#pragma once
#include <stdint.h>

namespace moe {

constexpr int kThreads = 256;  // threads per CTA of the decode kernel
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 16;     // rows of h per router / down-projection chunk
constexpr int kUnitRows = 32;  // gate/up rows per work unit (one Q4_0 block of a)
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxR = 32;
constexpr int kMaxH = 4096;
constexpr int kMboxCap = 256;  // miss-request mailbox entries
constexpr int kMaxOwn = 4;     // chunks of h one CTA may own
constexpr int kACodeBytes = 80;  // one quantised block of a: 32 int16, scale, sum, pad

// Bytes of one Q4_0 matrix [rows x cols] in the slot layout (== canonical size).
inline constexpr uint64_t q4_bytes(uint64_t rows, uint64_t cols) {
  return rows * cols / 32 * 18;
}

struct SlotLayout {
  uint64_t gu;     // offset of gate/up tile (rb, st): gu + (4 rb + st) * 9H
  uint64_t down;   // offset of down tile c: down + c * 9I
  uint64_t bytes;  // rounded up to 256
};

inline SlotLayout slot_layout(int H, int I) {
  SlotLayout s;
  s.gu = 0;
  s.down = (uint64_t)(I / 32) * 4 * 9 * H;
  s.bytes = (s.down + (uint64_t)(H / 16) * 9 * I + 255) / 256 * 256;
  return s;
}

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
  uint32_t bar_count;  // grid barrier arrivals, zeroed before every launch
  uint32_t pad2[31];
  uint32_t z_count;  // CTAs that have published this launch's logits, per layer (zeroed per launch)
  uint32_t pad3[31];
  uint32_t a_count;  // CTAs that have published this launch's activation codes (zeroed per launch)
  uint32_t pad4[31];
  unsigned long long pin_hits, ring_hits, misses, evictions, staged;
};

struct DecodeParams {
  // shape
  int L, H, E, K, I, Is, R, use_norm;
  float eps;
  int nch;      // H / kChunk
  int n_units;  // K * I / 32 + Is / 32
  int n_exp;    // K + (Is > 0)
  int nown;     // max chunks of h per CTA: ceil(nch / grid)
  // weights
  const uint8_t* pool;  // slot pool
  uint64_t slot_bytes;
  SlotLayout lay;       // routed-expert slot layout
  const uint8_t* shared_pool;  // [L] shared slots
  uint64_t shared_slot_bytes;
  SlotLayout slay;
  const uint16_t* router;  // [L][nch][E][16] bf16
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
  float* h;        // [H]
  float* part;     // [E][nch]
  float* sq;       // [nch]
  float* z;        // [E]
  uint8_t* acodes;  // [n_exp][Imax/32][kACodeBytes]
  // stats
  uint32_t* hist;  // [L][E]
  int32_t* log;    // [log_steps][L][K][7]
  int log_steps;
  Ctrl* ctrl;
  // miss path
  MissReq* mbox;                 // host-mapped, kMboxCap entries
  const uint32_t* done_seq;      // device word, written by the proxy's stream
  unsigned long long timeout_ns;
  unsigned long long* phase_trace;  // [L+1][8] globaltimer stamps of CTA 0, or null
};

}  // namespace moe
