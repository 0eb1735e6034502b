// decode_kernel.cu -- one persistent sm_100a kernel that runs a whole decode token
// (all L MoE layers) for libmoe.
//
// Luce Spark (theneuralfeed.com write-up, key-components paragraph) runs the whole
// token as one graph instead of one per layer; here the token is one cooperative
// kernel launch, captured in a CUDA graph by the runtime.  Every CTA keeps the whole
// residual stream h in shared memory.  Per layer:
//
//   1. h += y of the previous layer, read from a 64-bit fixed-point accumulator that
//      the previous layer's units added into (the layer's one grid-wide exchange)
//   2. RMSNorm scale and the canonical-order router logits of this CTA's experts
//      (router rows staged in shared memory one layer ahead), published as 8-byte
//      words that carry the layer as an epoch, so readers need no separate flag
//   3. every CTA reads all logits: warp-shuffle top-k (value desc, index asc), routing
//      weights (softmax over the kept logits), the cache decision (pinned / ring hit /
//      miss into the LRU ring slot, key-components item 2); CTA 0 commits the ring
//      state, the event log, the atomic routing histogram and the miss requests
//   4. units: unit (expert, rb) = gate/up rows 32rb..32rb+31 and down column block rb
//      of one expert, one contiguous run of the slot streamed into shared memory by
//      bulk (TMA) copies; Q4_0 x int16 dot products (dp2a) give g and u,
//      a = silu(g) * u is quantised per block, and the unit's share of the layer output
//      w_i * D_i[:, rb] a_rb is added into the accumulator (fixed point: the sum does
//      not depend on the order in which units finish, so outputs are bit-identical
//      across residency levels and runs)
//   5. one release add per CTA on the arrival counter
//
// Shared-expert units do not depend on routing: a CTA whose first unit is a shared one
// loads the next layer's unit as soon as its buffer is free.  Every wait is bounded by a
// globaltimer deadline; a wait that runs out sets the error word and the CTA returns, so
// a lost miss signal ends the launch instead of hanging.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_cache.h"
#include "moe_internal.h"

namespace moe {

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* ptr) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* ptr) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ptr) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* ptr, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(ptr), "l"(v) : "memory");
}

__device__ __forceinline__ void red_add_u64(unsigned long long* ptr, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(ptr), "l"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_volatile(const int32_t* ptr) {
  return *reinterpret_cast<const volatile int32_t*>(ptr);
}

__device__ __forceinline__ void set_error(Ctrl* c, int code) { atomicCAS(&c->error, 0, code); }
__device__ __forceinline__ bool has_error(const Ctrl* c) { return ld_volatile(&c->error) != 0; }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bulk (non-tensor TMA) copy global -> shared with an L2 evict-first policy: streamed
// expert and router weights are read once per token, so they do not push the kernel's
// code and the small exchange buffers out of L2.  dst, src 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (bytes a multiple of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Two-way dot products: a holds two int16 (signed), b four uint8; .lo uses bytes 0-1,
// .hi bytes 2-3.
__device__ __forceinline__ int dp2a_lo(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 16 * sum_e q_e * c_e over one Q4_0 block: q from the 16 nibble bytes, c the block's 32
// int16 codes packed in pairs (x0..x3 = codes 0-7, 8-15, 16-23, 24-31).  Low nibbles
// are weights 0-15, high nibbles (kept in place, i.e. times 16) weights 16-31.
__device__ __forceinline__ int q4_block_dot16(const uint4 q, const int4 x0, const int4 x1,
                                              const int4 x2, const int4 x3) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  const int xw[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                      x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
  int lo = 0, hi = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t l4 = w[k] & 0x0F0F0F0Fu, h4 = w[k] & 0xF0F0F0F0u;
    lo = dp2a_lo(xw[2 * k], l4, lo);
    lo = dp2a_hi(xw[2 * k + 1], l4, lo);
    hi = dp2a_lo(xw[8 + 2 * k], h4, hi);
    hi = dp2a_hi(xw[9 + 2 * k], h4, hi);
  }
  return 16 * lo + hi;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// The canonical fold's last step: xor-butterfly offsets 16, 8, 4, 2, 1; every lane ends
// with the total.
__device__ __forceinline__ float butterfly_sum(float acc) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
  return acc;
}

// Quantise one 32-value block held one value per lane to int16 codes:
// code = rint(v * 32767 / amax); scale16 = amax / (32767 * 16) reconstructs 16 * v / code;
// csum = sum of the block's codes.  Same arithmetic in every CTA: deterministic.
__device__ __forceinline__ int quant_block(float v, float& scale16, int& csum) {
  const float amax = warp_max(fabsf(v));
  int code = 0;
  if (amax > 0.0f) {
    code = __float2int_rn(v * __fdividef(32767.0f, amax));
    code = max(-32767, min(32767, code));
  }
  scale16 = amax * (1.0f / (32767.0f * 16.0f));
  csum = warp_sum_int(code);
  return code;
}

// Orderable 64-bit routing key: larger logit first, then lower expert index; -0 == +0;
// a NaN logit gets key 0 and is never preferred.
__device__ __forceinline__ uint64_t route_key(float v, int e) {
  if (v == 0.0f) v = 0.0f;
  const uint32_t u = __float_as_uint(v);
  uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  if (v != v) o = 0;
  return ((uint64_t)o << 32) | (uint32_t)(~(uint32_t)e);
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int off) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, off);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), off);
  return ((uint64_t)hi << 32) | lo;
}

__host__ __device__ inline int pow2_ceil_le32(int n) {
  int g = 1;
  while (g < n && g < 32) g <<= 1;
  return g;
}

// ------------------------------------------------------------------ shared memory plan

struct Misc {
  uint64_t bar_u[4];  // the four gate/up tiles of the unit in flight
  uint64_t bar_d;     // its down part
  uint64_t bar_r;     // this CTA's router rows of the current layer
  const uint8_t* src[kMaxK + 1];  // slot base of each active expert (rank order, then shared)
  uint32_t miss_seq[kMaxK + 1];   // proxy copy to wait for (0: none)
  long long pull[kMaxK + 1];      // pull mode: the expert's byte offset in the host tier, or -1
  int32_t sel[kMaxK];
  float w[kMaxK];
  int32_t fix_dst[kMaxR], fix_src[kMaxR];  // deferred ring fills (pool indices)
  int32_t n_fix;
  int32_t ring_owner[kMaxR];
  uint32_t ring_stamp[kMaxR];
  uint32_t ring_clock;
  float gu[2 * kUnitRows];
  float inv;
  float bias[kWarps];  // router bias of this CTA's experts, current layer
  uint32_t step, seq_base, n_miss;
  int32_t flag;
  int32_t P_l, base_l;
  // preload matching of the current layer
  int32_t lk_e[kMaxPreload];  // expert of each preloaded group (-1: none)
  int32_t hit[kMaxPreload];   // its rank in the layer's top-k, or -1
  int32_t unc[kMaxK];         // ranks whose expert no group preloaded, in rank order
  int32_t n_unc, n_avail;
  int32_t early;  // 1: this layer's first unit was issued as soon as routing was known
};

struct SmemPlan {
  uint32_t unit, rrows, h, g, pc, xcodes, xs, xc, z, pinrow, cand, misc, params, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemPlan smem_plan(int H, int E, int rx, int down_late) {
  SmemPlan s;
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) {
    off = align_up(off, 128);
    const uint32_t r = off;
    off += bytes;
    return r;
  };
  const uint32_t nch = (uint32_t)H / kChunk;
  s.unit = take((down_late ? 36u : 54u) * H);
  s.rrows = take(2u * H * (uint32_t)rx);
  s.h = take(4u * H);
  s.g = take(4u * H);
  s.pc = take(4u * nch * (1u + (uint32_t)rx));  // chunk partials: the norm's, then one row per router expert
  s.xcodes = take(2u * H);
  s.xs = take(4u * (H / 32));
  s.xc = take(4u * (H / 32));
  s.z = take(4u * E);
  s.pinrow = take(4u * E);
  s.cand = take(8u * kWarps * kMaxK + 8u * kThreads);
  s.misc = take(sizeof(Misc));
  s.params = take(sizeof(DecodeParams));
  s.total = align_up(off, 128);
  return s;
}

// ------------------------------------------------------------------ waits

// Out-of-line slow paths of the bounded waits: the common case (already there) stays
// inline; the spin loops live in separate functions so the per-layer code stays small
// enough for the SM instruction cache.

// Spin until *count >= target (acquire), with back-off; false on timeout / error.
__device__ __noinline__ bool spin_count(const uint32_t* count, uint32_t target, uint64_t timeout_ns, Ctrl* ctrl) {
  const uint64_t t0 = gtimer();
  for (uint32_t polls = 1; ld_acquire(count) < target; ++polls) {
    __nanosleep(32);
    if ((polls & 15u) == 0) {
      if (has_error(ctrl)) return false;
      if (gtimer() - t0 > timeout_ns) {
        set_error(ctrl, MOE_DEVERR_BARRIER);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ bool wait_count(const DecodeParams& p, const uint32_t* count, uint32_t target) {
  return ld_acquire(count) >= target || spin_count(count, target, p.timeout_ns, p.ctrl);
}

// Thread 0: wait until the proxy has signalled miss copy seq (0: nothing to wait for).
__device__ __noinline__ bool spin_miss(const uint32_t* done_seq, uint32_t seq, uint64_t timeout_ns, Ctrl* ctrl) {
  const uint64_t t0 = gtimer();
  while ((int32_t)(ld_acquire(done_seq) - seq) < 0) {
    if (has_error(ctrl)) return false;
    if (gtimer() - t0 > timeout_ns) {
      set_error(ctrl, MOE_DEVERR_MISS);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool wait_miss(const DecodeParams& p, uint32_t seq) {
  if (seq == 0) return true;
  if ((int32_t)(ld_acquire(p.done_seq) - seq) < 0 && !spin_miss(p.done_seq, seq, p.timeout_ns, p.ctrl)) return false;
  fence_proxy_async();  // the copy engine's writes, then bulk-copy reads of the same slot
  return true;
}

// Wait for the bulk copies counted on bar to land (bounded).
__device__ __noinline__ bool spin_mbar(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, Ctrl* ctrl) {
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(bar, parity)) {
    if (gtimer() - t0 > timeout_ns) {
      set_error(ctrl, MOE_DEVERR_TMA);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool mbar_wait(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  return mbar_try_wait(bar, parity) || spin_mbar(bar, parity, p.timeout_ns, p.ctrl);
}

// Barrier + agreement: true when every thread of the CTA passed ok, so that the CTA
// leaves as a whole.  A failure elsewhere in the grid reaches this CTA through its own
// bounded waits (every spin loop also watches the error word), so the common path reads
// no global memory here.
__device__ __forceinline__ bool cta_ok(const DecodeParams&, bool ok) { return __syncthreads_and(ok) != 0; }

// CTA 0's marks are SM clock cycles (clock64: fine-grained, one SM); the kernel's start
// and end are also taken on the global timer so that cycles convert to ns.
template <bool ON>
__device__ __forceinline__ void stamp(const DecodeParams& p, int l, int k) {
  if (ON && p.phase_trace && blockIdx.x == 0 && threadIdx.x == 0) p.phase_trace[l * 32 + k] = clock64();
}

template <bool ON>
__device__ __forceinline__ void stamp_both(const DecodeParams& p, int k_clock, int k_timer) {
  if (ON && p.phase_trace && blockIdx.x == 0 && threadIdx.x == 0) {
    p.phase_trace[p.L * 32 + k_clock] = clock64();
    p.phase_trace[p.L * 32 + k_timer] = gtimer();
  }
}

// Per-CTA marks (every CTA, thread 0): after [(L+1)][32] come [L][gridDim][4] stamps.
template <bool ON>
__device__ __forceinline__ void cta_stamp(const DecodeParams& p, int l, int k) {
  if (ON && p.phase_trace && threadIdx.x == 0)
    p.phase_trace[(size_t)(p.L + 1) * 32 + ((size_t)l * gridDim.x + blockIdx.x) * 4 + k] = gtimer();
}

// ------------------------------------------------------------------ routing

__device__ __forceinline__ void issue_unit(const DecodeParams& p, Misc& m, uint8_t* ubuf, const uint8_t* src);

// Top-k for more than 256 experts: keys re-read from shared memory every round.
__device__ __noinline__ int topk_large(const DecodeParams& p, const float* zs) {
  const int lane = threadIdx.x & 31;
  int my_e = -1;
  uint32_t taken = 0;
  for (int i = 0; i < p.K; ++i) {
    uint64_t best = 0;
    for (int k = 0; lane + 32 * k < p.E; ++k)
      if (!((taken >> k) & 1u)) {
        const uint64_t kk = route_key(zs[lane + 32 * k], lane + 32 * k);
        best = kk > best ? kk : best;
      }
    for (int off = 16; off >= 1; off >>= 1) {
      const uint64_t o = shfl_xor_u64(best, off);
      best = o > best ? o : best;
    }
    const int e = (int)(~(uint32_t)best);
    if ((best >> 32) == 0ull && lane == 0) set_error(p.ctrl, MOE_DEVERR_ROUTE);
    if ((e & 31) == lane) taken |= 1u << (e >> 5);
    if (lane == i) my_e = e;
  }
  return my_e;
}

// Warp 0: top-k of z (value desc, index asc) and the renormalised softmax weights.
// Keys live in registers (E <= 256: 8 per lane); each round is a lane-local max and a
// redux max / min.  Lane i returns the expert of rank i (and m.sel / m.w are set).
__device__ __noinline__ int topk_weights(const DecodeParams& p, Misc& m, const float* zs) {
  const int lane = threadIdx.x & 31;
  const int E = p.E;
  int my_e = -1;
  if (E <= 256) {
    uint32_t ord[8];  // orderable logit bits; 0 marks a taken (or NaN) entry
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = lane + 32 * k;
      ord[k] = e < E ? (uint32_t)(route_key(zs[e], e) >> 32) : 0u;
    }
    for (int i = 0; i < p.K; ++i) {
      uint32_t lv = ord[0];
#pragma unroll
      for (int k = 1; k < 8; ++k) lv = max(lv, ord[k]);
      const uint32_t gv = __reduce_max_sync(0xffffffffu, lv);
      uint32_t li = 0xffffffffu;
#pragma unroll
      for (int k = 7; k >= 0; --k)
        if (ord[k] == gv) li = (uint32_t)(lane + 32 * k);
      const int e = (int)__reduce_min_sync(0xffffffffu, li);
      if (gv == 0u && lane == 0) set_error(p.ctrl, MOE_DEVERR_ROUTE);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (lane + 32 * k == e) ord[k] = 0u;
      if (lane == i) my_e = e;
    }
  } else {
    my_e = topk_large(p, zs);
  }
  if (my_e < 0 || my_e >= E) my_e = 0;  // lanes >= k (and a failed route)
  const float zmax = __shfl_sync(0xffffffffu, zs[my_e], 0);
  const float ex = lane < p.K ? expf(zs[my_e] - zmax) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < p.K) {
    m.sel[lane] = my_e;
    m.w[lane] = __fdividef(ex, sum);
  }
  __syncwarp();
  return my_e;
}

// The top-k of topk_weights (m.sel only) for E <= 256 and k = K (compile time), in two
// parallel steps.  (1) topk_rank_warp: warp w ranks its 32 experts 32w + lane by 64-bit
// key (logit desc, index asc), reading the warp's keys as shared-memory broadcasts; a
// rank below K makes a candidate, stored at w K + rank.  A warp needs only its own 32
// logits, so it runs as soon as they are there.  (2) topk_rank_candidates, after a CTA
// barrier: a candidate's global rank is the number of larger candidates over the 8
// warps' lists (a list with K larger keys puts it out of the top K, as its count shows):
// 256 / (8 K) threads per candidate, at most 8, each count some of the lists and add up
// with shuffles.
template <int K>
__device__ __forceinline__ void topk_rank_warp(const DecodeParams& p, unsigned long long key,
                                               unsigned long long* cand) {
  static_assert(K >= 1 && K <= 32, "k");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned long long* keys = cand + kWarps * kMaxK;  // [256] after the candidate slots
  keys[tid] = key;
  if (lane < K) cand[warp * K + lane] = 0ull;
  __syncwarp();
  int rank = 0;  // among this warp's 32 keys
  {
    const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys + warp * 32);
    ulonglong2 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = k2[u];
#pragma unroll
    for (int u = 0; u < 16; ++u) rank += (v[u].x > key) + (v[u].y > key);
  }
  if (key != 0ull && rank < K) cand[warp * K + rank] = key;
}

//
// The thread that places the candidate of rank early_rank (>= 0: the rank whose unit this
// CTA computes first, known before routing) issues that unit's loads at once when the
// expert is pinned (unit block early_rb), and sets m.early.
template <int K>
__device__ __forceinline__ void topk_rank_candidates(const DecodeParams& p, Misc& m, const unsigned long long* cand,
                                                     const int32_t* pinrow, uint8_t* ubuf, int early_rank,
                                                     int early_rb) {
  const int tid = threadIdx.x;
  constexpr int nc = kWarps * K;  // candidate slots
  constexpr int tpc = kThreads / nc >= 8 ? 8 : kThreads / nc >= 4 ? 4 : kThreads / nc >= 2 ? 2 : 1;
  constexpr int lpt = kWarps / tpc;  // lists per thread
  const int ci = tid / tpc, sub = tid % tpc;
#pragma unroll
  for (int c0 = 0; c0 < nc; c0 += kThreads / tpc) {  // one pass unless K > 16
    const int cc = c0 + ci;
    const unsigned long long c = cc < nc ? cand[cc] : 0ull;
    int r = 0;
#pragma unroll
    for (int w = 0; w < lpt; ++w) {
      const unsigned long long* lw = cand + (sub * lpt + w) * K;
#pragma unroll
      for (int q = 0; q < K; ++q) r += lw[q] > c;
    }
#pragma unroll
    for (int off = 1; off < tpc; off <<= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    if (sub == 0 && c != 0ull && r < K) {
      const int e = (int)(~(uint32_t)c);
      m.sel[r] = e;
      if ((c >> 32) == 0ull) set_error(p.ctrl, MOE_DEVERR_ROUTE);  // a NaN logit was needed
      if (r == early_rank) {
        const int ps = pinrow[e];
        if (ps >= 0) {
          issue_unit(p, m, ubuf,
                     p.pool + (size_t)(m.base_l + (ps & 0xffff)) * p.slot_bytes + (size_t)early_rb * p.unit_bytes);
          m.early = 1;
        }
      }
    }
  }
  __syncthreads();
}

// Warp 0, after the top-k: the renormalised softmax weights of the selected experts
// (lane i: rank i), exactly as topk_weights forms them.
__device__ __forceinline__ void route_weights(const DecodeParams& p, Misc& m, const float* zs, int my_e) {
  const int lane = threadIdx.x & 31;
  const float zmax = __shfl_sync(0xffffffffu, zs[my_e], 0);
  const float ex = lane < p.K ? expf(zs[my_e] - zmax) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < p.K) m.w[lane] = __fdividef(ex, sum);
}

// Thread 0 of every CTA: the cache decision for layer l (identical in all CTAs), from
// the layer's pinned-slot row and ring state staged in shared memory.  CTA 0 also
// commits the next ring state, the event log, histogram, counters and (proxy mode) the
// miss requests.
__device__ __noinline__ void cache_decide(const DecodeParams& p, Misc& m, int l, const int32_t* pinrow) {
  const int R = p.R, K = p.K;
  const int par = m.step & 1;
  const bool commit = blockIdx.x == 0;
  const int P = m.P_l;
  const int base = m.base_l;
  bool busy[kMaxR];
  int32_t fix[kMaxR];
  uint32_t clock = m.ring_clock;
  for (int r = 0; r < R; ++r) {
    busy[r] = false;
    fix[r] = -1;
  }
  unsigned long long n_pin = 0, n_ring = 0, n_miss = 0, n_evict = 0, n_staged = 0;
  for (int i = 0; i < K; ++i) {
    const int e = m.sel[i];
    const int ps = pinrow[e];
    int kind, slot_log, evicted = -1, pool_idx;
    uint32_t seq = 0;
    long long pull = -1;
    if (ps >= 0) {  // (logical slot << 16) | physical slot within the layer's pinned region
      kind = MOE_PIN_HIT;
      slot_log = ps >> 16;
      pool_idx = base + (ps & 0xffff);
      ++n_pin;
    } else {
      int r = -1;
      for (int rr = 0; rr < R; ++rr)
        if (m.ring_owner[rr] == e) r = rr;
      if (r >= 0) {
        kind = MOE_RING_HIT;
        m.ring_stamp[r] = ++clock;
        busy[r] = true;
        slot_log = P + r;
        pool_idx = base + P + r;
        ++n_ring;
      } else if (R == 0) {
        set_error(p.ctrl, MOE_DEVERR_SLOT);
        kind = MOE_MISS;
        slot_log = -1;
        pool_idx = base;  // any valid slot; the launch is already failed
      } else {
        int v = -1;
        for (int rr = 0; rr < R && v < 0; ++rr)
          if (m.ring_owner[rr] < 0) v = rr;
        if (v < 0) {
          v = 0;
          for (int rr = 1; rr < R; ++rr)
            if (m.ring_stamp[rr] < m.ring_stamp[v]) v = rr;
        }
        evicted = m.ring_owner[v];
        m.ring_owner[v] = e;
        m.ring_stamp[v] = ++clock;
        kind = MOE_MISS;
        slot_log = P + v;
        if (busy[v]) {  // slot still read by an earlier rank of this layer: stage
          pool_idx = p.staging_base + i;
          fix[v] = pool_idx;
          ++n_staged;
        } else {
          pool_idx = base + P + v;
          busy[v] = true;
          fix[v] = -1;
        }
        ++n_miss;
        if (evicted >= 0) ++n_evict;
        if (p.miss_mode == kMissPull) {
          pull = (long long)(((size_t)l * p.E + e) * p.slot_bytes);
        } else {
          seq = m.seq_base + 1 + m.n_miss++;
          if (commit) {
            MissReq* q = p.mbox + (seq % kMboxCap);
            volatile uint32_t* qv = reinterpret_cast<volatile uint32_t*>(q);
            qv[1] = (uint32_t)l;
            qv[2] = (uint32_t)e;
            qv[3] = (uint32_t)pool_idx;
            __threadfence_system();
            qv[0] = seq;
            __threadfence_system();
          }
        }
      }
    }
    m.src[i] = p.pool + (size_t)pool_idx * p.slot_bytes;
    m.miss_seq[i] = seq;
    m.pull[i] = pull;
    if (commit) {
      int32_t* ev = p.log + (((size_t)(m.step % (uint32_t)p.log_steps) * p.L + l) * K + i) * 7;
      ev[0] = (int32_t)m.step;
      ev[1] = l;
      ev[2] = i;
      ev[3] = e;
      ev[4] = kind;
      ev[5] = slot_log;
      ev[6] = evicted;
      atomicAdd(p.hist + (size_t)l * p.E + e, 1u);
    }
  }
  m.n_fix = 0;
  for (int r = 0; r < R; ++r)
    if (fix[r] >= 0) {
      m.fix_dst[m.n_fix] = base + P + r;
      m.fix_src[m.n_fix] = fix[r];
      ++m.n_fix;
    }
  if (commit) {
    const size_t ws = ((size_t)(par ^ 1) * p.L + l) * R;
    for (int r = 0; r < R; ++r) {
      p.ring_owner[ws + r] = m.ring_owner[r];
      p.ring_stamp[ws + r] = m.ring_stamp[r];
    }
    p.ring_clock[(size_t)(par ^ 1) * p.L + l] = clock;
    atomicAdd(&p.ctrl->pin_hits, n_pin);
    atomicAdd(&p.ctrl->ring_hits, n_ring);
    atomicAdd(&p.ctrl->misses, n_miss);
    atomicAdd(&p.ctrl->evictions, n_evict);
    atomicAdd(&p.ctrl->staged, n_staged);
    if (p.miss_mode == kMissPull) atomicAdd(&p.ctrl->pulled, n_miss);
  }
}

// Warp 0: the common case where every selected expert is pinned; lane i handles rank
// i.  Returns false (nothing written) when some expert is not pinned; else the slots are
// set and cache_pinned_commit records the layer.
__device__ __forceinline__ bool cache_pinned_lookup(const DecodeParams& p, Misc& m, const int32_t* pinrow, int my_e) {
  const int lane = threadIdx.x & 31;
  const int ps = lane < p.K ? pinrow[my_e] : 0;
  if (!__all_sync(0xffffffffu, ps >= 0)) return false;
  if (lane < p.K) {
    m.src[lane] = p.pool + (size_t)(m.base_l + (ps & 0xffff)) * p.slot_bytes;
    m.miss_seq[lane] = 0;
    m.pull[lane] = -1;
  }
  __syncwarp();
  return true;
}

// Warp 0, after cache_pinned_lookup: CTA 0 writes the event log, histogram and counters
// and carries the untouched ring to the next token's copy; every CTA has no ring fill.
__device__ __noinline__ void cache_pinned_commit(const DecodeParams& p, Misc& m, int l, const int32_t* pinrow,
                                                 int my_e) {
  const int lane = threadIdx.x & 31;
  const bool commit = blockIdx.x == 0;
  if (commit && lane < p.K) {
    const int ps = pinrow[my_e];
    int32_t* ev = p.log + (((size_t)(m.step % (uint32_t)p.log_steps) * p.L + l) * p.K + lane) * 7;
    ev[0] = (int32_t)m.step;
    ev[1] = l;
    ev[2] = lane;
    ev[3] = my_e;
    ev[4] = MOE_PIN_HIT;
    ev[5] = ps >> 16;
    ev[6] = -1;
    atomicAdd(p.hist + (size_t)l * p.E + my_e, 1u);
  }
  if (commit && lane < p.R) {
    const int par = m.step & 1;
    const size_t ws = ((size_t)(par ^ 1) * p.L + l) * p.R;
    p.ring_owner[ws + lane] = m.ring_owner[lane];
    p.ring_stamp[ws + lane] = m.ring_stamp[lane];
  }
  if (lane == 0) {
    m.n_fix = 0;
    if (commit) {
      p.ring_clock[(size_t)((m.step & 1) ^ 1) * p.L + l] = m.ring_clock;
      atomicAdd(&p.ctrl->pin_hits, (unsigned long long)p.K);
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ units

// Thread 0: bulk-load a unit (src = its first byte in a slot) into the unit buffer:
// four gate/up tiles on bar_u[0..3] and, unless the down part comes later, the down
// nibbles and scales (one run of 18H bytes) on bar_d.
__device__ __forceinline__ void issue_unit(const DecodeParams& p, Misc& m, uint8_t* ubuf, const uint8_t* src) {
  const uint32_t tb = 9u * p.H;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    mbar_expect_tx(&m.bar_u[st], tb);
    bulk_g2s_stream(ubuf + st * tb, src + st * tb, tb, &m.bar_u[st]);
  }
  if (!p.down_late) {
    mbar_expect_tx(&m.bar_d, 18u * p.H);
    bulk_g2s_stream(ubuf + 36u * p.H, src + 36u * p.H, 18u * p.H, &m.bar_d);
  }
}

// All threads: wait until a unit issued ahead has landed (its copies complete the
// current phase of the unit barriers), then advance the parities past it.
__device__ __forceinline__ bool drain_unit(const DecodeParams& p, Misc& m, uint32_t (&par_u)[4], uint32_t& par_d) {
  bool ok = true;
#pragma unroll
  for (int st = 0; st < 4; ++st) ok = ok && mbar_wait(p, &m.bar_u[st], par_u[st]);
  if (!p.down_late) ok = ok && mbar_wait(p, &m.bar_d, par_d);
#pragma unroll
  for (int st = 0; st < 4; ++st) par_u[st] ^= 1u;
  if (!p.down_late) par_d ^= 1u;
  return ok;
}

// All threads: copy a unit from the mapped pinned host tier into its slot (pull mode),
// then order those writes before the bulk copies that read the slot back.
__device__ __noinline__ void pull_unit(const DecodeParams& p, const uint8_t* host, uint8_t* dst) {
  const uint4* s = reinterpret_cast<const uint4*>(host);
  uint4* d = reinterpret_cast<uint4*>(dst);
  const uint32_t n16 = (uint32_t)(p.unit_bytes / 16);
  constexpr int kBatch = 8;
  for (uint32_t base = threadIdx.x; base < n16; base += kThreads * kBatch) {
    uint4 v[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const uint32_t t = base + k * kThreads;
      if (t < n16) v[k] = __ldcv(s + t);
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const uint32_t t = base + k * kThreads;
      if (t < n16) __stcg(d + t, v[k]);
    }
  }
  fence_proxy_async();
}

// One thread: this CTA's share of a layer's speculative prefetch: the slots of the
// layer's most frequently routed pinned experts (slots, loaded beforehand), as one byte
// range split evenly over the grid.
__device__ __noinline__ void prefetch_likely(const DecodeParams& p, const int32_t (&slots)[kMaxLikely]) {
  const uint64_t sb = p.slot_bytes, total = (uint64_t)p.n_l2 * sb;
  const uint64_t per = ((total + gridDim.x - 1) / gridDim.x + 255) / 256 * 256;
  uint64_t lo = (uint64_t)blockIdx.x * per;
  const uint64_t hi = lo + per < total ? lo + per : total;
  while (lo < hi) {
    const int m = (int)(lo / sb);
    const uint64_t in = lo - (uint64_t)m * sb, end = (uint64_t)(m + 1) * sb < hi ? (uint64_t)(m + 1) * sb : hi;
    int32_t slot = -1;
#pragma unroll
    for (int q = 0; q < kMaxLikely; ++q)
      if (q == m + p.n_pre) slot = slots[q];
    if (slot >= 0) bulk_prefetch_l2(p.pool + (size_t)slot * sb + in, (uint32_t)(end - lo));
    lo = end;
  }
}

// The k-th unit of CTA b in this layer: rank i (K = the shared expert), block rb, and
// whether its bytes are already in flight (issued ahead).  With at least one CTA per
// unit: CTAs [0, n_pre Ur) hold a preload of unit b mod Ur of likely expert b / Ur and
// compute it if that expert was routed (any rank); CTAs [routed, n_units) own the
// shared expert's units; every other CTA (a wrong preload, no preload, no unit) is
// "available" and the j-th of them takes the j-th unit of the ranks no preload covered,
// in rank order.  Every CTA derives the same assignment from the same routing.
struct UnitRef {
  int i, rb;
  bool shared, issued;
};

__device__ __forceinline__ bool unit_of(const DecodeParams& p, int n_pre, const Misc& m, bool pre, int b, int G, int k,
                                        UnitRef& u) {
  const int Ur = p.I / 32, routed = p.K * Ur;
  if (G < p.n_units) {  // fewer CTAs than units: round robin, no preload
    const int uu = b + k * G;
    if (uu >= p.n_units) return false;
    u.shared = uu >= routed;
    u.i = u.shared ? p.K : uu / Ur;
    u.rb = u.shared ? uu - routed : uu % Ur;
    u.issued = k == 0 && pre && u.shared;
    return true;
  }
  const int npc = n_pre * Ur;
  if (b >= routed && b < p.n_units) {
    if (k > 0) return false;
    u.shared = true;
    u.i = p.K;
    u.rb = b - routed;
    u.issued = pre;
    return true;
  }
  if (b < npc && m.hit[b / Ur] >= 0) {
    if (k > 0) return false;
    u.shared = false;
    u.i = m.hit[b / Ur];
    u.rb = b % Ur;
    u.issued = true;
    return true;
  }
  // available CTAs in order: those without a unit (no preload to wait for), those that
  // preloaded nothing, then those whose preload was not routed
  int a;
  const int idle = max(G - p.n_units, 0);
  if (b >= p.n_units) {
    a = b - p.n_units;
  } else if (b >= npc) {
    a = idle + (b - npc);
  } else {
    a = idle + (routed - npc) + b % Ur;
    for (int q = 0; q < b / Ur; ++q)
      if (m.hit[q] < 0) a += Ur;
  }
  const int j = a + k * m.n_avail;
  if (j >= m.n_unc * Ur) return false;
  u.shared = false;
  u.i = m.unc[j / Ur];
  u.rb = j % Ur;
  u.issued = false;
  return true;
}

// All threads of every CTA: the deferred ring fills (staging slot -> ring slot), split
// over the grid.
__device__ __noinline__ void ring_fills(const DecodeParams& p, const Misc& m) {
  const size_t n16 = p.slot_bytes / 16;
  for (int f = 0; f < m.n_fix; ++f) {
    const uint4* s = reinterpret_cast<const uint4*>(p.pool + (size_t)m.fix_src[f] * p.slot_bytes);
    uint4* d = reinterpret_cast<uint4*>(const_cast<uint8_t*>(p.pool) + (size_t)m.fix_dst[f] * p.slot_bytes);
    for (size_t t = (size_t)blockIdx.x * kThreads + threadIdx.x; t < n16; t += (size_t)gridDim.x * kThreads)
      d[t] = __ldcg(s + t);
  }
}

// One thread: the pool slots of layer l's likely experts.
__device__ __noinline__ void load_likely(const DecodeParams& p, int l, int32_t (&lk)[kMaxLikely]) {
#pragma unroll
  for (int q = 0; q < kMaxLikely; ++q) lk[q] = __ldg(p.likely_slot + (size_t)l * kMaxLikely + q);
}

// All threads: the layer's input h (h += y of the previous layer from its accumulator,
// or h = y without the residual; acc null: h as it is) and, per 16-column chunk c, the
// canonical partials of the norm and of my router rows: plain fmaf chains over the
// chunk's columns in order from +0, of h^2 into pc[c] and of w_k * u (u = g * h, or h
// without the norm) into pc[(1 + k) nch + c].  A chunk is two lanes of 8 columns; the
// even lane's chain carries on in the odd lane, which makes it the one sequential chain
// over the 16 columns.
__device__ __forceinline__ void head_pass(const DecodeParams& p, int H, const unsigned long long* acc, float* hs,
                                          const float* gs, const uint16_t* rrows, int nrx, float* pc, float* trace) {
  const int nch = H / kChunk, n8 = H / 8;
  const int lane = threadIdx.x & 31;
  const bool odd = lane & 1;
  for (int q0 = threadIdx.x & ~31; q0 < n8; q0 += kThreads) {  // warp-uniform: the shuffles need every lane
    const int q = q0 + lane;
    const bool live = q < n8;  // n8 is even: both lanes of a chunk are live or neither
    const int qq = live ? q : n8 - 1;
    float h[8];
    {
      const float4* h4 = reinterpret_cast<const float4*>(hs + 8 * qq);
      const float4 a = h4[0], c = h4[1];
      h[0] = a.x; h[1] = a.y; h[2] = a.z; h[3] = a.w;
      h[4] = c.x; h[5] = c.y; h[6] = c.z; h[7] = c.w;
    }
    if (acc) {
      const ulonglong2* a2 = reinterpret_cast<const ulonglong2*>(acc + 8 * qq);
      ulonglong2 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = __ldcg(a2 + k);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float y0 = __ll2float_rn((long long)v[k].x) * kAccInvScale;
        const float y1 = __ll2float_rn((long long)v[k].y) * kAccInvScale;
        h[2 * k] = p.use_norm ? __fadd_rn(h[2 * k], y0) : y0;
        h[2 * k + 1] = p.use_norm ? __fadd_rn(h[2 * k + 1], y1) : y1;
      }
      if (live) {
        float4* h4 = reinterpret_cast<float4*>(hs + 8 * q);
        h4[0] = make_float4(h[0], h[1], h[2], h[3]);
        h4[1] = make_float4(h[4], h[5], h[6], h[7]);
        if (trace) {
          float4* t4 = reinterpret_cast<float4*>(trace + 8 * q);
          t4[0] = make_float4(h[0], h[1], h[2], h[3]);
          t4[1] = make_float4(h[4], h[5], h[6], h[7]);
        }
      }
    }
    if (p.use_norm) {
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) s = fmaf(h[i], h[i], s);
      float t = __shfl_up_sync(0xffffffffu, s, 1);
#pragma unroll
      for (int i = 0; i < 8; ++i) t = fmaf(h[i], h[i], t);
      if (live && odd) pc[q >> 1] = t;
    }
    if (nrx > 0) {
      float u[8];
      if (p.use_norm) {
        const float4* g4 = reinterpret_cast<const float4*>(gs + 8 * qq);
        const float4 a = g4[0], c = g4[1];
        u[0] = __fmul_rn(a.x, h[0]); u[1] = __fmul_rn(a.y, h[1]);
        u[2] = __fmul_rn(a.z, h[2]); u[3] = __fmul_rn(a.w, h[3]);
        u[4] = __fmul_rn(c.x, h[4]); u[5] = __fmul_rn(c.y, h[5]);
        u[6] = __fmul_rn(c.z, h[6]); u[7] = __fmul_rn(c.w, h[7]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = h[i];
      }
      // rows two at a time (their chains are independent and interleave), then a last one
      int k = 0;
      for (; k + 1 < nrx; k += 2) {
        const uint4 w0 = *reinterpret_cast<const uint4*>(rrows + (size_t)k * H + 8 * qq);
        const uint4 w1 = *reinterpret_cast<const uint4*>(rrows + (size_t)(k + 1) * H + 8 * qq);
        const float f0[8] = {bf16_lo(w0.x), bf16_hi(w0.x), bf16_lo(w0.y), bf16_hi(w0.y),
                             bf16_lo(w0.z), bf16_hi(w0.z), bf16_lo(w0.w), bf16_hi(w0.w)};
        const float f1[8] = {bf16_lo(w1.x), bf16_hi(w1.x), bf16_lo(w1.y), bf16_hi(w1.y),
                             bf16_lo(w1.z), bf16_hi(w1.z), bf16_lo(w1.w), bf16_hi(w1.w)};
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s0 = fmaf(f0[i], u[i], s0);
          s1 = fmaf(f1[i], u[i], s1);
        }
        float t0 = __shfl_up_sync(0xffffffffu, s0, 1);
        float t1 = __shfl_up_sync(0xffffffffu, s1, 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          t0 = fmaf(f0[i], u[i], t0);
          t1 = fmaf(f1[i], u[i], t1);
        }
        if (live && odd) {
          pc[(1 + k) * nch + (q >> 1)] = t0;
          pc[(2 + k) * nch + (q >> 1)] = t1;
        }
      }
      if (k < nrx) {
        const uint4 w = *reinterpret_cast<const uint4*>(rrows + (size_t)k * H + 8 * qq);
        const float wf[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                             bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(wf[i], u[i], s);
        float t = __shfl_up_sync(0xffffffffu, s, 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) t = fmaf(wf[i], u[i], t);
        if (live && odd) pc[(1 + k) * nch + (q >> 1)] = t;
      }
    }
  }
}

// One warp: the canonical fold of a row of chunk partials: lane l adds chunks l, l + 32,
// ... in order from +0, then the xor butterfly (16, 8, 4, 2, 1); every lane gets the sum.
__device__ __forceinline__ float fold_chunks(const float* pc, int nch) {
  float acc = 0.0f;
  for (int c = threadIdx.x & 31; c < nch; c += 32) acc = __fadd_rn(acc, pc[c]);
  return butterfly_sum(acc);
}

// All threads: h += y (or h = y without the residual) from a layer's accumulator; all of
// a thread's loads are issued before any of them is used (one L2 round trip, not one
// per element).  trace: where to write the new h, or null.
__device__ __forceinline__ void add_layer_output(const DecodeParams& p, int H, const unsigned long long* acc, float* hs,
                                                 float* trace) {
  constexpr int kPer = 8;
  for (int j0 = 0; j0 < H; j0 += kPer * kThreads) {
    long long v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int j = j0 + threadIdx.x + k * kThreads;
      v[k] = j < H ? (long long)__ldcg(acc + j) : 0;
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int j = j0 + threadIdx.x + k * kThreads;
      if (j < H) {
        const float y = __ll2float_rn(v[k]) * kAccInvScale;
        const float hn = p.use_norm ? __fadd_rn(hs[j], y) : y;
        hs[j] = hn;
        if (trace) trace[j] = hn;
      }
    }
  }
}

// a[i] of a 4-element register array for a run-time i (selects, no local memory)
__device__ __forceinline__ uint32_t pick4(const uint32_t (&a)[4], int i) {
  return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

// ------------------------------------------------------------------ the kernel

// BPL: Q4_0 blocks of a gate/up row per lane (ceil(H / 1024), at least 1).  HC: the
// hidden size when it is 1024 BPL (a lane holds blocks lane + 32 mb exactly; every size
// and offset below is then a compile-time constant), else 0 (sizes read at run time).
template <int BPL, int HC, bool FULL>
__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ DecodeParams p) {
  static_assert(HC == 0 || HC == 1024 * BPL, "HC is 0 or 1024 BPL");
  // the speculative loads and the phase marks exist only in the FULL instances: the lean
  // ones leave their code out of the per-layer instruction stream
  const int n_pre = FULL ? p.n_pre : 0, n_l2 = FULL ? p.n_l2 : 0;
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = HC ? HC : p.H;
  const SmemPlan S = smem_plan(H, p.E, p.rx_per_cta, p.down_late);
  Misc& m = *reinterpret_cast<Misc*>(smem + S.misc);
  // a shared-memory copy of the parameters for the out-of-line helpers (a reference to
  // it is a plain shared address; the kernel body reads the parameters directly)
  DecodeParams& sp = *reinterpret_cast<DecodeParams*>(smem + S.params);
  for (int i = threadIdx.x; i < (int)(sizeof(DecodeParams) / 4); i += kThreads)
    reinterpret_cast<uint32_t*>(&sp)[i] = reinterpret_cast<const uint32_t*>(&p)[i];
  uint8_t* ubuf = smem + S.unit;
  const uint16_t* rrows = reinterpret_cast<const uint16_t*>(smem + S.rrows);
  float* hs = reinterpret_cast<float*>(smem + S.h);
  float* gs = reinterpret_cast<float*>(smem + S.g);
  float* pcs = reinterpret_cast<float*>(smem + S.pc);
  int16_t* xcodes = reinterpret_cast<int16_t*>(smem + S.xcodes);
  float* xs = reinterpret_cast<float*>(smem + S.xs);
  int32_t* xc = reinterpret_cast<int32_t*>(smem + S.xc);
  float* zs = reinterpret_cast<float*>(smem + S.z);
  int32_t* pinrow = reinterpret_cast<int32_t*>(smem + S.pinrow);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + S.cand);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, b = blockIdx.x;
  const int nb = H / 32, nch = H / kChunk;
  const int routed = p.K * (p.I / 32);
  const bool has_gain = p.use_norm && p.gain;
  const int nrx = b < p.E ? min(p.rx_per_cta, (p.E - b + G - 1) / G) : 0;  // my router experts b, b+G, ...
  const bool first_shared = b < p.n_units && b >= routed;  // my first unit does not depend on routing
  const int Ur = p.I / 32;
  const int npc = n_pre * Ur;  // CTAs that preload a likely expert's unit
  // with no preloads and a CTA per unit, the routed unit j this CTA computes is fixed
  // before routing (the idle CTAs take units 0.., then CTA b < routed unit idle + b):
  // rank j / Ur, block j % Ur; its loads go out as soon as that rank's expert is known
  int early_rank = -1, early_rb = 0;
  if (n_pre == 0 && G >= p.n_units) {
    const int j = b >= p.n_units ? b - p.n_units : b < routed ? (G - p.n_units) + b : -1;
    if (j >= 0 && j < routed) {
      early_rank = j / Ur;
      early_rb = j % Ur;
    }
  }
  // a unit was issued ahead for the current layer (the shared expert's, or a preload);
  // every thread keeps the same value
  bool pre = first_shared;
  int32_t pre_slot = -1;  // the slot this layer's preload reads (issued at the counter), or -1
  const uint32_t gbase = 0;  // arrival counter starts at 0 every launch
  uint32_t par_u[4] = {0, 0, 0, 0}, par_d = 0, par_r = 0;  // mbarrier parities (uniform)
  bool ok = true;

  if (tid == 0) {
    for (int k = 0; k < 4; ++k) mbar_init(&m.bar_u[k], 1);
    mbar_init(&m.bar_d, 1);
    mbar_init(&m.bar_r, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    m.step = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->step);
    m.seq_base = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->req_seq);
    m.n_miss = 0;
    m.n_fix = 0;
  }
  stamp_both<FULL>(p, 0, 4);
  if (!cta_ok(p, true)) goto fail;

  // ---- prologue: accumulators 0 and 1 and the logit words zeroed, h = x, first loads
  for (int j = b * kThreads + tid; j < 2 * H; j += G * kThreads) p.acc[j] = 0ull;
  for (int e = b * kThreads + tid; e < p.E; e += G * kThreads) p.zll[e] = 0ull;
  for (int j = tid; j < H; j += kThreads) hs[j] = __ldg(p.x + j);
  if (tid == 0) {
    if (nrx > 0) {
      mbar_expect_tx(&m.bar_r, 2u * H * nrx);
      for (int k = 0; k < nrx; ++k)
        bulk_g2s_stream(const_cast<uint16_t*>(rrows) + (size_t)k * H, p.router + (size_t)(b + k * G) * H, 2u * H,
                        &m.bar_r);
    }
    if (first_shared) issue_unit(sp, m, ubuf, p.shared_pool + (size_t)(b - routed) * p.unit_bytes);
  }
  if (b < npc) {  // preload: unit b mod Ur of layer 0's likely expert b / Ur
    const int32_t slot = __ldg(p.likely_slot + b / Ur);
    if (slot >= 0) {
      if (tid == 0) issue_unit(sp, m, ubuf, p.pool + (size_t)slot * p.slot_bytes + (size_t)(b % Ur) * p.unit_bytes);
      pre = true;
    }
  }
  int32_t lk[kMaxLikely];  // thread 32: the likely experts' slots of the current layer
  if (tid == 32 && n_l2 > 0) {
    load_likely(sp, 0, lk);
    prefetch_likely(sp, lk);
  }
  if (b == 0 && p.h_trace)
    for (int j = tid; j < H; j += kThreads) p.h_trace[j] = hs[j];
  __syncthreads();
  if (tid == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&p.ctrl->bar_count) : "memory");
    ok = wait_count(p, &p.ctrl->bar_count, gbase + G);
  }
  if (!cta_ok(p, ok)) goto fail;
  stamp<FULL>(p, p.L, 1);

  for (int l = 0; l < p.L; ++l) {
    stamp<FULL>(p, l, 0);
    const bool next = l + 1 < p.L;
    // ---------------------------------------------------------------- layer inputs
    // loads that do not depend on the previous layer go out first
    {
      const float4* g4 = has_gain ? reinterpret_cast<const float4*>(p.gain + (size_t)l * H) : nullptr;
      for (int t = tid; t < H / 4; t += kThreads)
        reinterpret_cast<float4*>(gs)[t] = has_gain ? __ldg(g4 + t) : make_float4(1.f, 1.f, 1.f, 1.f);
      for (int e = tid; e < p.E; e += kThreads) pinrow[e] = __ldg(p.pin_slot + (size_t)l * p.E + e);
      const int par = m.step & 1;
      const size_t rs = ((size_t)par * p.L + l) * p.R;
      if (tid < p.R) {
        m.ring_owner[tid] = __ldcg(p.ring_owner + rs + tid);
        m.ring_stamp[tid] = __ldcg(p.ring_stamp + rs + tid);
      }
      if (tid == kThreads - 1) m.ring_clock = __ldcg(p.ring_clock + (size_t)par * p.L + l);
      if (tid == kThreads - 2) m.P_l = __ldg(p.n_pinned + l);
      if (tid == kThreads - 3) m.base_l = __ldg(p.layer_base + l);
      if (tid == kThreads - 4) m.early = 0;
      if (tid < nrx) m.bias[tid] = p.bias ? __ldg(p.bias + (size_t)l * p.E + b + tid * G) : 0.0f;
      if (tid == 32 && n_l2 > 0 && l > 0) load_likely(sp, l, lk);
      if (tid < n_pre) m.lk_e[tid] = __ldg(p.likely_e + (size_t)l * kMaxLikely + tid);
      pre_slot = (l > 0 && b < npc) ? __ldg(p.likely_slot + (size_t)l * kMaxLikely + b / Ur) : -1;
    }
    if (l > 0) {
      // ---------------------------------------------------------------- h += y(l - 1)
      if (tid == 0) {
        ok = wait_count(p, &p.ctrl->bar_count, gbase + (uint32_t)(l + 1) * G);
        // every unit of layer l - 1 is done: the HBM is free for this layer's guess
        if (ok && pre_slot >= 0)
          issue_unit(sp, m, ubuf, p.pool + (size_t)pre_slot * p.slot_bytes + (size_t)(b % Ur) * p.unit_bytes);
      }
      if (pre_slot >= 0) pre = true;
      // the HBM is idle until this layer's routing is known: fetch its likely experts
      // (a thread off the critical path, after the wait)
      if (tid == 32 && n_l2 > 0) {
        if (wait_count(p, &p.ctrl->bar_count, gbase + (uint32_t)(l + 1) * G)) prefetch_likely(sp, lk);
      }
      if (!cta_ok(p, ok)) goto fail;
      stamp<FULL>(p, l, 1);
      add_layer_output(p, H, p.acc + (size_t)((l - 1) % kAccBufs) * H, hs,
                       (b == 0 && p.h_trace) ? p.h_trace + (size_t)l * H : nullptr);
      // deferred ring fills of layer l - 1 (a layer that missed more often than it has
      // ring slots): its readers are done
      if (m.n_fix > 0) ring_fills(sp, m);
      // the accumulator of layer l + 1 was last read at the start of layer l - 1, by CTAs
      // that have all published layer l - 1's logits since
      if (next) {
        unsigned long long* z = p.acc + (size_t)((l + 1) % kAccBufs) * H;
        for (int j = b * kThreads + tid; j < H; j += G * kThreads) z[j] = 0ull;
      }
    }
    __syncthreads();
    stamp<FULL>(p, l, 2);

    // ---------------------------------------------------------------- norm and router
    // chunk partials of the norm and of my router rows (this layer's rows landed during
    // the previous layer), then the canonical folds
    if (nrx > 0 && !__all_sync(0xffffffffu, ok && mbar_wait(p, &m.bar_r, par_r))) ok = false;
    head_pass(p, H, nullptr, hs, gs, rrows, nrx, pcs, nullptr);
    __syncthreads();
    // inv = 1 / sqrt(ss / H + eps), folded by every warp (the same bits everywhere)
    const float inv =
        p.use_norm ? __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(fold_chunks(pcs, nch), (float)H), p.eps))) : 1.0f;
    stamp<FULL>(p, l, 10);
    // logits of my experts: warp k folds expert b + k G
    if (warp < nrx) {
      const float S_e = fold_chunks(pcs + (size_t)(1 + warp) * nch, nch);
      if (lane == 0 && ok) {
        const int e = b + warp * G;
        const float z = fmaf(S_e, inv, m.bias[warp]);
        st_relaxed_u64(p.zll + e, ((unsigned long long)(uint32_t)(l + 1) << 32) | __float_as_uint(z));
        if (warp == 0) stamp<FULL>(p, l, 11);
      }
    }
    // quantised expert input x = RMSNorm(h) (or h): four lanes per 32-block, each lane 8
    // values; the block's largest |x| and code sum combine over the four lanes
    {
      const int j4 = tid & 3;
      for (int b0 = tid >> 2; b0 < ((nb + 63) / 64) * 64; b0 += kThreads / 4) {
        const int bb = b0 < nb ? b0 : nb - 1;  // lanes past the end repeat a block, write nothing
        float v[8];
        const float4* h4 = reinterpret_cast<const float4*>(hs + bb * 32 + 8 * j4);
        const float4* g4 = reinterpret_cast<const float4*>(gs + bb * 32 + 8 * j4);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float4 hv = h4[q];
          if (p.use_norm) {
            const float4 gv = g4[q];
            hv.x = __fmul_rn(__fmul_rn(hv.x, inv), gv.x);
            hv.y = __fmul_rn(__fmul_rn(hv.y, inv), gv.y);
            hv.z = __fmul_rn(__fmul_rn(hv.z, inv), gv.z);
            hv.w = __fmul_rn(__fmul_rn(hv.w, inv), gv.w);
          }
          v[4 * q] = hv.x;
          v[4 * q + 1] = hv.y;
          v[4 * q + 2] = hv.z;
          v[4 * q + 3] = hv.w;
        }
        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(v[q]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const float mult = amax > 0.0f ? __fdividef(32767.0f, amax) : 0.0f;
        int c[8];
        int csum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          c[q] = max(-32767, min(32767, __float2int_rn(v[q] * mult)));
          csum += c[q];
        }
        csum += __shfl_xor_sync(0xffffffffu, csum, 1);
        csum += __shfl_xor_sync(0xffffffffu, csum, 2);
        if (b0 < nb) {  // quarter-major ([4][nb] x 16 B): a warp's reads of one quarter are contiguous
          reinterpret_cast<uint4*>(xcodes)[j4 * nb + bb] =
              make_uint4(((uint32_t)c[0] & 0xffffu) | ((uint32_t)c[1] << 16),
                         ((uint32_t)c[2] & 0xffffu) | ((uint32_t)c[3] << 16),
                         ((uint32_t)c[4] & 0xffffu) | ((uint32_t)c[5] << 16),
                         ((uint32_t)c[6] & 0xffffu) | ((uint32_t)c[7] << 16));
          if (j4 == 0) {
            xs[bb] = amax * (1.0f / (32767.0f * 16.0f));
            xc[bb] = csum;
          }
        }
      }
    }
    stamp<FULL>(p, l, 12);
    if (!cta_ok(p, ok)) goto fail;
    stamp<FULL>(p, l, 3);
    cta_stamp<FULL>(p, l, 3);
    // this layer's router rows are read: the buffer takes the next layer's
    if (nrx > 0) {
      if (tid == 0 && next) {
        mbar_expect_tx(&m.bar_r, 2u * H * nrx);
        for (int k = 0; k < nrx; ++k)
          bulk_g2s_stream(const_cast<uint16_t*>(rrows) + (size_t)k * H,
                          p.router + ((size_t)(l + 1) * p.E + b + k * G) * H, 2u * H, &m.bar_r);
      }
      par_r ^= 1u;
    }

    // ---------------------------------------------------------------- routing
    // top-k: all threads for the common k = 8 over at most 256 experts (each warp ranks
    // its 32 experts as soon as their logits are in), else warp 0 after all are read
    const bool topk8 = p.E <= kThreads && p.K == 8;
    {
      // a warp polls its 32 words together: one coalesced load per round for the lanes
      // still missing (per-lane spins would send one request per lane to the few L2
      // lines that every CTA polls)
      const uint32_t epoch = (uint32_t)(l + 1);
      for (int e0 = tid & ~31; e0 < p.E; e0 += kThreads) {  // warp-uniform
        const int e = e0 + lane;
        const bool mine = e < p.E;
        unsigned long long v = mine ? ld_relaxed_u64(p.zll + e) : 0ull;
        bool have = !mine || (uint32_t)(v >> 32) == epoch;
        if (!__all_sync(0xffffffffu, have)) {
          const uint64_t t0 = gtimer();
          for (uint32_t polls = 1;; ++polls) {
            __nanosleep(32);
            if (!have) {
              v = ld_relaxed_u64(p.zll + e);
              have = (uint32_t)(v >> 32) == epoch;
            }
            if (__all_sync(0xffffffffu, have)) break;
            if ((polls & 15u) == 0) {  // lane 0 decides for the warp
              int stop = 0;
              if (lane == 0) {
                if (has_error(p.ctrl)) {
                  stop = 1;
                } else if (gtimer() - t0 > p.timeout_ns) {
                  set_error(p.ctrl, MOE_DEVERR_BARRIER);
                  stop = 1;
                }
              }
              if (__shfl_sync(0xffffffffu, stop, 0)) break;
            }
          }
        }
        if (!__all_sync(0xffffffffu, have)) {
          ok = false;
          break;
        }
        if (mine) zs[e] = __uint_as_float((uint32_t)v);
      }
      if (topk8) topk_rank_warp<8>(p, tid < p.E && ok ? route_key(zs[tid], tid) : 0ull, cand);
    }
    if (!cta_ok(p, ok)) goto fail;
    stamp<FULL>(p, l, 4);
    if (topk8) topk_rank_candidates<8>(p, m, cand, pinrow, ubuf, early_rank, early_rb);
    if (warp == 0) {
      int my_e;
      if (topk8) {
        my_e = lane < p.K ? m.sel[lane] : 0;
        if (my_e < 0 || my_e >= p.E) my_e = 0;
      } else {
        my_e = topk_weights(sp, m, zs);
      }
      stamp<FULL>(p, l, 13);
      const bool fast = cache_pinned_lookup(p, m, pinrow, my_e);
      if (fast && n_pre == 0) {
        // no preloads: every rank is uncovered, and one unit per CTA is known now; its
        // loads go out before the rest of the bookkeeping
        if (lane < p.K) m.unc[lane] = lane;
        if (lane == 0) {
          m.n_unc = p.K;
          m.n_avail = routed + max(G - p.n_units, 0);
        }
        __syncwarp();
        if (lane == 0 && G >= p.n_units && !m.early) {
          UnitRef ur;
          if (unit_of(p, n_pre, m, pre, b, G, 0, ur) && !ur.issued && !ur.shared) {
            issue_unit(sp, m, ubuf, m.src[ur.i] + (size_t)ur.rb * p.unit_bytes);
            m.early = 1;
          }
        }
      }
      stamp<FULL>(p, l, 15);
      if (topk8) route_weights(p, m, zs, my_e);
      if (fast) cache_pinned_commit(sp, m, l, pinrow, my_e);
      else if (lane == 0) cache_decide(sp, m, l, pinrow);
      if (!(fast && n_pre == 0)) {
        if (lane == 0) {  // preload matching: which group holds which rank, which ranks are left
          uint32_t covered = 0;
          int wrong = 0;
          for (int q = 0; q < n_pre; ++q) {
            int r = -1;
            for (int i = 0; i < p.K; ++i)
              if (m.sel[i] == m.lk_e[q]) r = i;
            m.hit[q] = r;
            if (r >= 0) covered |= 1u << r;
            else ++wrong;
          }
          int nu = 0;
          for (int i = 0; i < p.K; ++i)
            if (!((covered >> i) & 1u)) m.unc[nu++] = i;
          m.n_unc = nu;
          m.n_avail = wrong * Ur + (routed - npc) + max(G - p.n_units, 0);
        }
      }
      __syncwarp();
      stamp<FULL>(p, l, 14);
    }
    __syncthreads();
    if (b == 0 && p.w_trace && tid < p.K) p.w_trace[(size_t)l * p.K + tid] = m.w[tid];
    stamp<FULL>(p, l, 5);
    cta_stamp<FULL>(p, l, 0);

    // ---------------------------------------------------------------- units
    {
      // this lane's blocks of the quantised input: lane groups of GS lanes per row,
      // each lane BPL blocks of the row
      const int GS = pow2_ceil_le32(nb), RPW = 32 / GS, g = lane % GS, sub = lane / GS;
      const int rstep = kWarps * RPW;
      int4 xq[BPL][4];
      float xsc[BPL];
      int xsum[BPL];
#pragma unroll
      for (int mb = 0; mb < BPL; ++mb) {
        const int bb = g + GS * mb;
        if (bb < nb) {
          const int4* src = reinterpret_cast<const int4*>(xcodes);
          xq[mb][0] = src[bb];
          xq[mb][1] = src[nb + bb];
          xq[mb][2] = src[2 * nb + bb];
          xq[mb][3] = src[3 * nb + bb];
          xsc[mb] = xs[bb];
          xsum[mb] = xc[bb];
        } else {
          xq[mb][0] = xq[mb][1] = xq[mb][2] = xq[mb][3] = make_int4(0, 0, 0, 0);
          xsc[mb] = 0.0f;
          xsum[mb] = 0;
        }
      }
      unsigned long long* acc_l = p.acc + (size_t)(l % kAccBufs) * H;
      const bool early = m.early != 0;
      UnitRef ur;
      for (int k = 0; unit_of(p, n_pre, m, pre, b, G, k, ur); ++k) {
        const bool shared = ur.shared;
        const int i = ur.i, rb = ur.rb;
        const float wi = shared ? 1.0f : m.w[i];
        const uint8_t* usrc = (shared ? p.shared_pool + (size_t)l * p.shared_slot_bytes : m.src[i]) +
                              (size_t)rb * p.unit_bytes;
        if (!ur.issued && !(k == 0 && early)) {
          if (pre) {  // a preload that routing did not use: let it land before the buffer is reused
            ok = drain_unit(sp, m, par_u, par_d);
            if (!cta_ok(p, ok)) goto fail;
            pre = false;
          }
          if (!shared && m.pull[i] >= 0) {  // pull mode miss: this CTA fills its unit of the slot
            pull_unit(sp, p.host_tier + m.pull[i] + (size_t)rb * p.unit_bytes, const_cast<uint8_t*>(usrc));
            __syncthreads();
          }
          if (tid == 0) {
            ok = shared || wait_miss(p, m.miss_seq[i]);
            if (ok) issue_unit(sp, m, ubuf, usrc);
          }
          if (!cta_ok(p, ok)) goto fail;
        }
        stamp<FULL>(p, l, 6);
        // gate/up: rows r = gate 0..31, up 0..31 of the unit, tile r / 16; warp w takes rows
        // w + 8 j (j = 0..7: tile j / 2, row w + 8 (j % 2) of it)
        if constexpr (HC != 0) {
          // lane l holds blocks l + 32 mb; four rows (two tiles) per pass, one butterfly
          // for all eight rows at the end
          constexpr int NB = HC / 32;
          float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int j0 = 0; j0 < 8; j0 += 4) {
            bool w_ok = ok;
            w_ok = w_ok && mbar_wait(p, &m.bar_u[j0 / 2], pick4(par_u, j0 / 2));
            w_ok = w_ok && mbar_wait(p, &m.bar_u[j0 / 2 + 1], pick4(par_u, j0 / 2 + 1));
            if (!__all_sync(0xffffffffu, w_ok)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int j = j0 + q;
              const uint8_t* tile = ubuf + (j / 2) * 9u * HC;
              const int rt = warp + 8 * (j % 2);  // row in the tile
              const uint8_t* nib = tile + (size_t)rt * NB * 16;
              const __half* dsc = reinterpret_cast<const __half*>(tile + 8u * HC) + rt * NB;
#pragma unroll
              for (int mb = 0; mb < BPL; ++mb) {
                const int bb = lane + 32 * mb;
                const uint4 qv = *reinterpret_cast<const uint4*>(nib + bb * 16);
                const float d = __half2float(dsc[bb]);
                const int v = q4_block_dot16(qv, xq[mb][0], xq[mb][1], xq[mb][2], xq[mb][3]) - 128 * xsum[mb];
                acc[j] = fmaf(d * xsc[mb], (float)v, acc[j]);
              }
            }
          }
          if (ok) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
              for (int q = 0; q < 8; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], off);
            if (lane == 0)
#pragma unroll
              for (int q = 0; q < 8; ++q) m.gu[warp + 8 * q] = acc[q];
          }
        } else {
          for (int rw = warp * RPW; rw < 2 * kUnitRows; rw += 2 * rstep) {  // warp-uniform
            const int rows[2] = {rw + sub, rw + sub + rstep};
            const bool live0 = rows[0] < 2 * kUnitRows, live1 = rows[1] < 2 * kUnitRows;
            bool w_ok = ok;
            if (w_ok && live0) w_ok = mbar_wait(p, &m.bar_u[rows[0] / 16], pick4(par_u, rows[0] / 16));
            if (w_ok && live1) w_ok = mbar_wait(p, &m.bar_u[rows[1] / 16], pick4(par_u, rows[1] / 16));
            if (!__all_sync(0xffffffffu, w_ok)) {
              ok = false;
              break;
            }
            float acc[2] = {0.0f, 0.0f};
#pragma unroll
            for (int mb = 0; mb < BPL; ++mb) {
              const int bb = g + GS * mb;
              if (bb >= nb) continue;
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                if ((q == 0 && !live0) || (q == 1 && !live1)) continue;
                const int r = rows[q];
                const uint8_t* tile = ubuf + (r / 16) * 9u * H;
                const uint4 qv = *reinterpret_cast<const uint4*>(tile + ((size_t)(r % 16) * nb + bb) * 16);
                const float d = __half2float(reinterpret_cast<const __half*>(tile + 8u * H)[(r % 16) * nb + bb]);
                const int v = q4_block_dot16(qv, xq[mb][0], xq[mb][1], xq[mb][2], xq[mb][3]) - 128 * xsum[mb];
                acc[q] = fmaf(d * xsc[mb], (float)v, acc[q]);
              }
            }
            for (int off = GS / 2; off >= 1; off >>= 1) {
              acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
              acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], off);
            }
            if (g == 0) {
              if (live0) m.gu[rows[0]] = acc[0];
              if (live1) m.gu[rows[1]] = acc[1];
            }
          }
        }
        if (!cta_ok(p, ok)) goto fail;
        stamp<FULL>(p, l, 7);
        // a = silu(g) * u, quantised as one int16 block: every warp forms it (the same
        // bits in each) and holds the 32 codes in pairs in registers, so the down rows
        // start without another CTA barrier
        int4 a0, a1, a2, a3;
        float asc;
        int cs128;
        {
          const float gv = m.gu[lane], uv = m.gu[kUnitRows + lane];
          const float a = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
          int csum;
          const int code = quant_block(a, asc, csum);
          cs128 = 128 * csum;
          // pair q = codes 2q (low half) and 2q + 1 (high half)
          const int nxt = __shfl_down_sync(0xffffffffu, code, 1);
          const int pk = (int)(((uint32_t)code & 0xffffu) | ((uint32_t)nxt << 16));
          int pr[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) pr[q] = __shfl_sync(0xffffffffu, pk, 2 * q);
          a0 = make_int4(pr[0], pr[1], pr[2], pr[3]);
          a1 = make_int4(pr[4], pr[5], pr[6], pr[7]);
          a2 = make_int4(pr[8], pr[9], pr[10], pr[11]);
          a3 = make_int4(pr[12], pr[13], pr[14], pr[15]);
          if (warp == 0 && lane == 0) stamp<FULL>(p, l, 16);
        }
        const uint8_t* dn = ubuf + (p.down_late ? 0u : 36u * H);
        if (p.down_late && tid == 0) {
          mbar_expect_tx(&m.bar_d, 18u * H);
          bulk_g2s_stream(ubuf, usrc + 36u * H, 18u * H, &m.bar_d);
        }
        if (!mbar_wait(p, &m.bar_d, par_d)) ok = false;
        stamp<FULL>(p, l, 17);
        if (ok) {
          // down: output row j against the unit's activation block; the weighted share
          // w_i * d_j * scale * dot goes into the accumulator as round(v * 2^28)
          const __half* dsc = reinterpret_cast<const __half*>(dn + 16u * H);
          bool range_ok = true;
#pragma unroll 4
          for (int j = tid; j < H; j += kThreads) {
            const uint4 qv = *reinterpret_cast<const uint4*>(dn + 16 * j);
            const int v = q4_block_dot16(qv, a0, a1, a2, a3) - cs128;
            float c = (__half2float(dsc[j]) * asc) * (float)v;
            if (!shared) c *= wi;
            long long qf = 0;
            if (fabsf(c) < kAccLimit) {
              qf = __float2ll_rn(c * kAccScale);
            } else {
              range_ok = false;
            }
            red_add_u64(acc_l + j, (unsigned long long)qf);
          }
          if (!range_ok) set_error(p.ctrl, MOE_DEVERR_RANGE);
          stamp<FULL>(p, l, 18);
          stamp<FULL>(p, l, 19);
        }
        if (!cta_ok(p, ok)) goto fail;
#pragma unroll
        for (int st = 0; st < 4; ++st) par_u[st] ^= 1u;
        par_d ^= 1u;
        pre = false;
      }
    }
    if (pre) {  // a preload left unused (no unit for this CTA): let it land
      ok = drain_unit(sp, m, par_u, par_d);
      if (!cta_ok(p, ok)) goto fail;
      pre = false;
    }
    stamp<FULL>(p, l, 8);
    cta_stamp<FULL>(p, l, 1);
    // the next layer's shared-expert unit does not depend on routing, and a likely
    // expert's unit is worth guessing: load them now
    if (next && first_shared) {
      if (tid == 0)
        issue_unit(sp, m, ubuf,
                   p.shared_pool + (size_t)(l + 1) * p.shared_slot_bytes + (size_t)(b - routed) * p.unit_bytes);
      pre = true;
    }
    // arrival: the CTA barrier that ended the unit ordered every thread's adds before
    // this release (a CTA without a unit added nothing)
    if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&p.ctrl->bar_count) : "memory");
    stamp<FULL>(p, l, 9);
    cta_stamp<FULL>(p, l, 2);
  }

  // ---- the last layer's output
  if (tid == 0) ok = wait_count(p, &p.ctrl->bar_count, gbase + (uint32_t)(p.L + 1) * G);
  if (!cta_ok(p, ok)) goto fail;
  {
    add_layer_output(p, H, p.acc + (size_t)((p.L - 1) % kAccBufs) * H, hs, nullptr);
    for (int j0 = b * kThreads; j0 < H; j0 += G * kThreads)
      if (j0 + tid < H) p.y[j0 + tid] = hs[j0 + tid];
    if (b == 0 && p.h_trace)
      for (int j = tid; j < H; j += kThreads) p.h_trace[(size_t)p.L * H + j] = hs[j];
    if (m.n_fix > 0) ring_fills(sp, m);
  }
  stamp_both<FULL>(p, 2, 5);
  if (b == 0 && tid == 0) {
    p.ctrl->step = m.step + 1;
    p.ctrl->req_seq = m.seq_base + m.n_miss;
  }
  return;

fail:
  // a failed launch: the error word says why (moe_sync); callers that cannot read it
  // see NaN outputs
  if (p.nan_on_error)
    for (int j0 = b * kThreads; j0 < H; j0 += G * kThreads)
      if (j0 + tid < H) p.y[j0 + tid] = __int_as_float(0x7fc00000);
}

// ------------------------------------------------------------------ host-side launch

// Blocks of one gate/up row each lane covers: 1 below 1024 columns, else H / 1024.
static int bpl_of(int H) {
  const int nb = H / 32;
  return nb <= 32 ? 1 : (nb + 31) / 32;
}

// The instance for hidden size H: compile-time sizes where there is one; the lean
// instance (no phase marks, no speculative loads) unless full is asked for.
template <typename F>
static cudaError_t with_kernel(int H, bool full, F f) {
  if (!full) switch (H) {
      case 1024: return f(moe_decode_kernel<1, 1024, false>);
      case 2048: return f(moe_decode_kernel<2, 2048, false>);
      case 3072: return f(moe_decode_kernel<3, 3072, false>);
      case 4096: return f(moe_decode_kernel<4, 4096, false>);
      default: break;
    }
  switch (H) {
    case 1024: return f(moe_decode_kernel<1, 1024, true>);
    case 2048: return f(moe_decode_kernel<2, 2048, true>);
    case 3072: return f(moe_decode_kernel<3, 3072, true>);
    case 4096: return f(moe_decode_kernel<4, 4096, true>);
    default: break;
  }
  switch (bpl_of(H)) {
    case 1: return f(moe_decode_kernel<1, 0, true>);
    case 2: return f(moe_decode_kernel<2, 0, true>);
    case 3: return f(moe_decode_kernel<3, 0, true>);
    default: return f(moe_decode_kernel<4, 0, true>);
  }
}

uint32_t decode_smem_bytes(int H, int E, int rx, int down_late) { return smem_plan(H, E, rx, down_late).total; }

// Shape-dependent launch settings: router experts per CTA and whether a unit's down part
// must reuse its gate/up buffer; false when no setting fits in smem_optin.
bool decode_plan(int H, int E, int grid, int smem_optin, int* rx, int* down_late, uint32_t* smem) {
  *rx = (E + grid - 1) / grid;
  if (*rx > kWarps) return false;
  for (int late = 0; late < 2; ++late) {
    const uint32_t bytes = decode_smem_bytes(H, E, *rx, late);
    if (bytes <= (uint32_t)smem_optin) {
      *down_late = late;
      *smem = bytes;
      return true;
    }
  }
  return false;
}

// Every instance of the kernel may use up to limit bytes of dynamic shared memory; set
// for all of them at once, so that contexts or calls of different shapes never leave
// one instance below what another call needs.
cudaError_t decode_configure(int limit) {
  cudaError_t e = cudaSuccess;
  auto set = [&](auto kern) { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, limit); };
  for (int H : {1024, 2048, 3072, 4096, 32, 1056, 2080, 3104})  // every instance
    for (int full = 0; full < 2 && e == cudaSuccess; ++full) e = with_kernel(H, full != 0, set);
  return e;
}

cudaError_t decode_max_blocks_per_sm(int H, uint32_t smem, int* out) {
  return with_kernel(H, true, [&](auto kern) { return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kern, kThreads, smem); });
}

cudaError_t decode_launch(const DecodeParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(p.H, p.E, p.rx_per_cta, p.down_late);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const bool full = p.phase_trace != nullptr || p.n_pre > 0 || p.n_l2 > 0;
  return with_kernel(p.H, full, [&](auto kern) { return cudaLaunchKernelEx(&cfg, kern, p); });
}

}  // namespace moe
