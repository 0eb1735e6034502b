// moe_internal.h -- layouts shared by the host runtime and the decode kernel of libmoe.
//
// Expert slot layout (device slot pool and pinned host tier alike).  Q4_0 blocks
// (GGUF convention: fp16 scale d + 16 bytes, byte j = weight j low nibble, weight j+16
// high nibble) are split structure-of-arrays so that every 16-byte nibble group is
// 16-byte aligned for vector and bulk (TMA) loads:
//
//   gate:  qs [I][H/32][16]  then  d [I][H/32] fp16
//   up:    qs [I][H/32][16]  then  d [I][H/32] fp16
//   down:  qs [H][I/32][16]  then  d [H][I/32] fp16
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
constexpr int kACodeBytes = 80;  // one quantised block of a: 32 int16, scale, sum, pad

// Bytes of one Q4_0 matrix [rows x cols] in the slot layout (== canonical size).
inline constexpr uint64_t q4_bytes(uint64_t rows, uint64_t cols) {
  return rows * cols / 32 * 18;
}

struct MatView {  // offsets of one matrix inside a slot
  uint64_t qs, d;
};

struct SlotLayout {
  MatView gate, up, down;
  uint64_t bytes;  // rounded up to 256
};

inline SlotLayout slot_layout(int H, int I) {
  SlotLayout s;
  uint64_t off = 0;
  auto mat = [&](uint64_t rows, uint64_t cols) {
    MatView m;
    m.qs = off;
    off += rows * cols / 2;
    m.d = off;
    off += rows * cols / 16;
    return m;
  };
  s.gate = mat(I, H);
  s.up = mat(I, H);
  s.down = mat(H, I);
  s.bytes = (off + 255) / 256 * 256;
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

// Device control block (one per context).
struct Ctrl {
  uint32_t step;        // decode steps completed
  uint32_t req_seq;     // miss requests issued so far
  int32_t error;        // MOE_DEVERR_* or 0
  uint32_t bar_count;   // grid barrier arrivals
  uint32_t bar_gen;     // grid barrier generation
  uint32_t pad[3];
  unsigned long long pin_hits, ring_hits, misses, evictions, staged;
};

struct DecodeParams {
  // shape
  int L, H, E, K, I, Is, R, use_norm;
  float eps;
  int nch;      // H / kChunk
  int n_units;  // K * I / 32 + Is / 32
  int n_exp;    // K + (Is > 0)
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
  const int32_t* pin_slot;    // [L][E] pinned index or -1
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
  uint8_t* acodes; // [n_exp][Imax/32][kACodeBytes]
  // stats
  uint32_t* hist;  // [L][E]
  int32_t* log;    // [log_steps][L][K][7]
  int log_steps;
  Ctrl* ctrl;
  // miss path
  MissReq* mbox;                 // host-mapped, kMboxCap entries
  const uint32_t* done_seq;      // device word, written by the proxy's stream
  unsigned long long timeout_ns;
};

}  // namespace moe
