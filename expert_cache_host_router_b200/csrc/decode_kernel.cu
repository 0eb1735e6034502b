// decode_kernel.cu -- one persistent sm_100a kernel that runs a whole decode token
// (all L MoE layers) for libmoe.
//
// Luce Spark (theneuralfeed.com write-up, key-components paragraph) runs the whole
// token as one graph instead of one per layer; here the token is one cooperative
// kernel launch, captured in a CUDA graph by the runtime.  Per layer:
//
//   R  router logits z_e = fmaf(S_e, inv, b_e) for this CTA's experts, where S_e folds
//      the per-chunk partials that the previous layer's D phase produced (canonical
//      order: lane l adds chunks l, l+32, ... from +0, then xor-butterfly 16..1)
//   -- grid barrier --
//      every CTA: warp-shuffle top-k (value desc, index asc), routing weights (softmax
//      over the kept logits), the cache decision (pinned / ring hit / miss into the LRU
//      ring slot, key-components item 2), and the quantised activations x
//      (int16 per 32-block) for the integer expert GEMVs; CTA 0 alone commits the ring
//      state, the event log, the atomic routing histogram and the miss requests that
//      the host proxy turns into copy-engine copies from pinned host memory
//   G  gate/up GEMV + SwiGLU: work unit = 32 rows of gate and up of one expert,
//      streamed into shared memory by bulk (TMA) copies; a = silu(g) * u is quantised
//      per 32-block and published
//   -- grid barrier --
//   D  down GEMV + weighted combine + shared expert + residual for 16 rows of h per
//      chunk, then the next layer's router partials and RMSNorm partial sums over the
//      same 16 columns
//   -- grid barrier --
//
// Every wait is bounded by a globaltimer deadline; a wait that runs out sets the error
// word and the CTA returns, so a lost miss signal ends the launch instead of hanging.
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

// Bulk (non-tensor TMA) copy global -> shared; completion counted on bar in bytes.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same copy with an L2 cache policy: streamed expert and router weights are read once
// per token, so they are marked evict-first and do not push the kernel's code and the
// small exchange buffers out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  const uint64_t pol = l2_evict_first_policy();
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* ptr) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* ptr, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
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
// int16 codes packed in pairs (xw[m] = {c[2m], c[2m+1]}).  Low nibbles are weights 0-15,
// high nibbles (kept in place, i.e. times 16) weights 16-31.
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

// Canonical fold of n partials (n <= 256, stride 1) by one warp; every lane returns
// the total.  Lane l adds parts l, l+32, ... from +0 in that order, then the lanes
// combine by xor-butterfly offsets 16, 8, 4, 2, 1.
__device__ __forceinline__ float canonical_fold(const float* parts, int n, int lane) {
  float v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = lane + 32 * k < n ? __ldcg(parts + lane + 32 * k) : 0.0f;
  float acc = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (lane + 32 * k < n) acc = __fadd_rn(acc, v[k]);
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
  uint64_t bar_u[4];  // gate/up unit, four 16-row stages
  uint64_t bar_r;     // next layer's router columns of the owned chunks
  const uint8_t* src[kMaxK + 1];  // slot base of each active expert (rank order, then shared)
  uint32_t miss_seq[kMaxK + 1];   // copy to wait for (0: resident)
  int32_t sel[kMaxK];
  float w[kMaxK];
  int32_t fix_dst[kMaxR], fix_src[kMaxR];  // deferred ring fills (pool indices)
  int32_t n_fix;
  int32_t ring_owner[kMaxR];
  uint32_t ring_stamp[kMaxR];
  uint32_t ring_clock;
  float hown[kMaxOwn][kChunk];   // this CTA's rows of the residual stream
  float gnext[kMaxOwn][kChunk];  // next layer's RMSNorm gain on those rows
  float u[kChunk];
  float gu[2 * kUnitRows];
  float inv;
  uint32_t step, seq_base, n_miss, gen;
  int32_t flag;
  int32_t P_l, base_l;  // pinned count and pool base of the current layer
  int32_t unit_ok;   // first gate/up unit issued
  int32_t d_issued;  // down rows of the first owned chunk issued during routing
};

struct SmemPlan {
  uint32_t unit, rchunk, hbuf, gbuf, pinrow, z, xcodes, xs, xc, o, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemPlan smem_plan(int H, int E, int K, int I, int Is, int nown) {
  SmemPlan s;
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) {
    off = align_up(off, 128);
    const uint32_t r = off;
    off += bytes;
    return r;
  };
  const int n_exp = K + (Is > 0);
  const int imax = I > Is ? I : Is;
  s.unit = take(36u * H);                        // gate qs|d, up qs|d for 32 rows
  s.rchunk = take(32u * E * nown);               // router columns of the owned chunks
  s.hbuf = take(4u * H);
  s.gbuf = take(4u * H);
  s.pinrow = take(4u * E);
  s.z = take(4u * E);
  s.xcodes = take(2u * H);
  s.xs = take(4u * (H / 32));
  s.xc = take(4u * (H / 32));
  s.o = take(4u * n_exp * kChunk);
  s.misc = take(sizeof(Misc));
  s.total = align_up(off, 128);
  return s;
}

// ------------------------------------------------------------------ barriers and waits

// Out-of-line slow paths of the bounded waits: the common case (already there) stays
// inline and short; the spin loops live in separate functions so that the code each
// layer runs through stays small enough for the SM instruction cache.

// Spin until *count >= target (acquire), with back-off; false on timeout / error.
__device__ __noinline__ bool spin_count(const DecodeParams& p, const uint32_t* count, uint32_t target) {
  const uint64_t t0 = gtimer();
  for (uint32_t polls = 1; ld_acquire(count) < target; ++polls) {
    __nanosleep(32);
    if ((polls & 31u) == 0) {
      if (has_error(p.ctrl)) return false;
      if (gtimer() - t0 > p.timeout_ns) {
        set_error(p.ctrl, MOE_DEVERR_BARRIER);
        return false;
      }
    }
  }
  return true;
}

// Grid barrier over all CTAs (co-resident by cooperative launch).  The arrival counter
// only grows during a launch (the graph zeroes it before the kernel), so barrier b of
// the launch completes when it reaches (b + 1) * gridDim.x.  Returns false when the
// wait ran out or another CTA flagged an error.
__device__ bool grid_sync(const DecodeParams& p, Misc& m) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t target = (m.gen + 1) * gridDim.x;
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&p.ctrl->bar_count) : "memory");
    int ok = ld_acquire(&p.ctrl->bar_count) >= target || spin_count(p, &p.ctrl->bar_count, target);
    m.gen += 1;
    m.flag = ok;
  }
  __syncthreads();
  return m.flag != 0;
}

__device__ __forceinline__ void stamp(const DecodeParams& p, int l, int k) {
  if (p.phase_trace && blockIdx.x == 0 && threadIdx.x == 0) p.phase_trace[l * 32 + k] = gtimer();
}

// Per-CTA marks (every CTA, thread 0): after [(L+1)][32] come [L][gridDim][4] stamps.
__device__ __forceinline__ void cta_stamp(const DecodeParams& p, int l, int k) {
  if (p.phase_trace && threadIdx.x == 0)
    p.phase_trace[(size_t)(p.L + 1) * 32 + ((size_t)l * gridDim.x + blockIdx.x) * 4 + k] = gtimer();
}

// Counted exchange: a producer CTA publishes with one release add after its stores;
// a consumer CTA's thread 0 waits (with back-off) until the count reaches target, then
// the CTA reads the data.  Only producers arrive and only consumers wait.
__device__ __forceinline__ void publish(const DecodeParams& p, uint32_t* count) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
}

__device__ bool await_count(const DecodeParams& p, Misc& m, const uint32_t* count, uint32_t target) {
  if (threadIdx.x == 0) {
    const int ok = ld_acquire(count) >= target || spin_count(p, count, target);
    m.flag = ok && !has_error(p.ctrl);
  }
  __syncthreads();
  return m.flag != 0;
}

// Thread 0: wait until the proxy has signalled miss copy seq (0: nothing to wait for).
__device__ __noinline__ bool spin_miss(const DecodeParams& p, uint32_t seq) {
  const uint64_t t0 = gtimer();
  while ((int32_t)(ld_acquire(p.done_seq) - seq) < 0) {
    if (has_error(p.ctrl)) return false;
    if (gtimer() - t0 > p.timeout_ns) {
      set_error(p.ctrl, MOE_DEVERR_MISS);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool wait_miss(const DecodeParams& p, uint32_t seq) {
  if (seq == 0) return true;
  if ((int32_t)(ld_acquire(p.done_seq) - seq) < 0 && !spin_miss(p, seq)) return false;
  fence_proxy_async();
  return true;
}

// Wait for the bulk copies counted on bar to land (bounded).
__device__ __noinline__ bool spin_mbar(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(bar, parity)) {
    if (gtimer() - t0 > p.timeout_ns) {
      set_error(p.ctrl, MOE_DEVERR_TMA);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool mbar_wait(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  return mbar_try_wait(bar, parity) || spin_mbar(p, bar, parity);
}

// CTA-uniform check of the error word: one thread reads it, everyone acts on that read
// (threads reading it themselves could disagree and split at the next barrier).
__device__ __forceinline__ bool cta_ok(const DecodeParams& p, int32_t& flag) {
  __syncthreads();
  if (threadIdx.x == 0) flag = !has_error(p.ctrl);
  __syncthreads();
  return flag != 0;
}

// ------------------------------------------------------------------ phases

// Router partials of layer l over chunk c (16 columns): every thread e folds
// w[e][t] * u_t, u_t = g_t * h_t (g = 1 without a gain; u = h without the norm), from
// +0 in ascending column order; plus the chunk's sum of squares of h.  wrow(e) points
// at the 16 bf16 weights of expert e for this chunk (global or shared memory).
template <typename WRow>
__device__ void router_partials(const DecodeParams& p, Misc& m, int c, const float* hv, const float* gv,
                                WRow wrow) {
  const int tid = threadIdx.x;
  if (tid < kChunk) m.u[tid] = (p.use_norm && gv) ? __fmul_rn(gv[tid], hv[tid]) : hv[tid];
  __syncthreads();
  for (int e = tid; e < p.E; e += kThreads) {
    const uint4* wp = wrow(e);
    const uint4 w0 = wp[0], w1 = wp[1];
    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float acc = 0.0f;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      acc = fmaf(bf16_lo(ws[t]), m.u[2 * t], acc);
      acc = fmaf(bf16_hi(ws[t]), m.u[2 * t + 1], acc);
    }
    __stcg(p.part + (size_t)e * p.nch + c, acc);
  }
  if (tid == 0 && p.use_norm) {
    float s = 0.0f;
#pragma unroll
    for (int t = 0; t < kChunk; ++t) s = fmaf(hv[t], hv[t], s);
    __stcg(p.sq + c, s);
  }
}

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
// 64-bit butterfly max.  Lane i returns the expert of rank i (and m.sel / m.w are set).
__device__ int topk_weights(const DecodeParams& p, Misc& m, const float* zs) {
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

// Thread 0 of every CTA: the cache decision for layer l (identical in all CTAs), from
// the layer's pinned-slot row and ring state staged in shared memory.  CTA 0 also
// commits the next ring state, the event log, histogram, counters and miss requests.
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
        seq = m.seq_base + 1 + m.n_miss++;
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
    m.src[i] = p.pool + (size_t)pool_idx * p.slot_bytes;
    m.miss_seq[i] = seq;
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
  if (p.Is > 0) {
    m.src[K] = p.shared_pool + (size_t)l * p.shared_slot_bytes;
    m.miss_seq[K] = 0;
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
  }
}

// Layer 0's router partials over chunk c from global router weights (once per launch).
__device__ __noinline__ void prologue_partials(const DecodeParams& p, Misc& m, int c, int k, bool has_gain) {
  router_partials(p, m, c, m.hown[k], has_gain ? m.gnext[k] : nullptr, [&](int e) {
    return reinterpret_cast<const uint4*>(p.router + ((size_t)c * p.E + e) * kChunk);
  });
}

// Warp 0: the common case where every selected expert is pinned; lane i handles rank
// i.  Returns false (nothing written) when some expert is not pinned.
__device__ bool cache_all_pinned(const DecodeParams& p, Misc& m, int l, const int32_t* pinrow, int my_e) {
  const int lane = threadIdx.x & 31;
  const int ps = lane < p.K ? pinrow[my_e] : 0;
  if (!__all_sync(0xffffffffu, ps >= 0)) return false;
  const bool commit = blockIdx.x == 0;
  if (lane < p.K) {
    m.src[lane] = p.pool + (size_t)(m.base_l + (ps & 0xffff)) * p.slot_bytes;
    m.miss_seq[lane] = 0;
    if (commit) {
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
  }
  if (commit && lane < p.R) {  // the ring is untouched: carry it to the next token's copy
    const int par = m.step & 1;
    const size_t ws = ((size_t)(par ^ 1) * p.L + l) * p.R;
    p.ring_owner[ws + lane] = m.ring_owner[lane];
    p.ring_stamp[ws + lane] = m.ring_stamp[lane];
  }
  if (lane == 0) {
    if (p.Is > 0) {
      m.src[p.K] = p.shared_pool + (size_t)l * p.shared_slot_bytes;
      m.miss_seq[p.K] = 0;
    }
    m.n_fix = 0;
    if (commit) {
      p.ring_clock[(size_t)((m.step & 1) ^ 1) * p.L + l] = m.ring_clock;
      atomicAdd(&p.ctrl->pin_hits, (unsigned long long)p.K);
    }
  }
  __syncwarp();
  return true;
}

// Thread 0: bulk-load gate/up unit u (32 rows of gate and of up of one expert) into
// shared memory as four 16-row tiles, one bulk copy each, after its miss copy (if any)
// has landed.
__device__ bool issue_unit(const DecodeParams& p, Misc& m, uint8_t* unit, int u) {
  const int per = p.I / 32, routed = p.K * per;
  const int i = u < routed ? u / per : p.K;
  const int rb = u < routed ? u % per : u - routed;
  const SlotLayout& L = i < p.K ? p.lay : p.slay;
  if (!wait_miss(p, m.miss_seq[i])) return false;
  const uint32_t tb = 9u * p.H;
  const uint8_t* src = m.src[i] + L.gu + (size_t)rb * 4 * tb;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    mbar_expect_tx(&m.bar_u[st], tb);
    bulk_g2s_stream(unit + st * tb, src + st * tb, tb, &m.bar_u[st]);
  }
  return true;
}

// All threads: pull the down tiles of chunk c of every resident active expert into L2
// (one prefetch per 128-byte line), so that the down phase reads them from L2.
__device__ void prefetch_dchunk_l2(const DecodeParams& p, const Misc& m, int c) {
  const uint32_t t_r = 9u * p.I, t_s = 9u * p.Is;
  const uint32_t routed_bytes = (uint32_t)p.K * t_r, total = routed_bytes + (p.Is > 0 ? t_s : 0);
  for (uint32_t off = 128u * threadIdx.x; off < total; off += 128u * kThreads) {
    const int i = off < routed_bytes ? (int)(off / t_r) : p.K;
    if (m.miss_seq[i] != 0) continue;  // its slot is still being filled
    const uint32_t in_tile = off < routed_bytes ? off - (uint32_t)i * t_r : off - routed_bytes;
    const SlotLayout& L = i < p.K ? p.lay : p.slay;
    const uint8_t* src = m.src[i] + L.down + (size_t)c * (i < p.K ? t_r : t_s) + in_tile;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(src));
  }
}

// Thread 0: bulk-load layer lr's router columns of the owned chunks into rch.
__device__ void prefetch_router(const DecodeParams& p, Misc& m, uint8_t* rch, int lr, int n_own) {
  mbar_expect_tx(&m.bar_r, 32u * p.E * n_own);
  for (int k = 0; k < n_own; ++k) {
    const int c = blockIdx.x + k * gridDim.x;
    bulk_g2s_stream(rch + (size_t)k * 32u * p.E, p.router + (((size_t)lr * p.nch + c) * p.E) * kChunk, 32u * p.E,
                    &m.bar_r);
  }
}

// ------------------------------------------------------------------ the kernel

template <int BPL>
__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemPlan S = smem_plan(p.H, p.E, p.K, p.I, p.Is, p.nown);
  Misc& m = *reinterpret_cast<Misc*>(smem + S.misc);
  float* zs = reinterpret_cast<float*>(smem + S.z);
  float* hbuf = reinterpret_cast<float*>(smem + S.hbuf);
  float* gbuf = reinterpret_cast<float*>(smem + S.gbuf);
  int32_t* pinrow = reinterpret_cast<int32_t*>(smem + S.pinrow);
  int16_t* xcodes = reinterpret_cast<int16_t*>(smem + S.xcodes);
  float* xs = reinterpret_cast<float*>(smem + S.xs);
  int32_t* xc = reinterpret_cast<int32_t*>(smem + S.xc);
  float* os = reinterpret_cast<float*>(smem + S.o);
  uint8_t* unit = smem + S.unit;
  uint8_t* rch = smem + S.rchunk;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, nb = H / 32;
  const int imax = p.I > p.Is ? p.I : p.Is;
  const int rec_per_exp = imax / 32;
  const bool has_gain = p.use_norm && p.gain;
  int n_own = 0;  // chunks of h owned by this CTA
  while (n_own < p.nown && (int)blockIdx.x + n_own * (int)gridDim.x < p.nch) ++n_own;

  if (tid == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(&m.bar_u[b], 1);
    mbar_init(&m.bar_r, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    m.step = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->step);
    m.seq_base = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->req_seq);
    m.gen = 0;
    m.n_miss = 0;
    m.flag = !has_error(p.ctrl);
  }
  __syncthreads();
  if (!m.flag) return;
  uint32_t par_u[4] = {0, 0, 0, 0}, par_r = 0;  // mbarrier parities (uniform)
  stamp(p, p.L, 0);

  // ---- prologue: h = x on the owned rows, and layer 0's router partials
  for (int k = 0; k < n_own; ++k) {
    const int c = blockIdx.x + k * gridDim.x;
    if (tid < kChunk) {
      const float v = p.x[c * kChunk + tid];
      m.hown[k][tid] = v;
      m.gnext[k][tid] = has_gain ? p.gain[c * kChunk + tid] : 1.0f;
      __stcg(p.h + c * kChunk + tid, v);
      if (p.h_trace) p.h_trace[c * kChunk + tid] = v;
    }
    __syncthreads();
    prologue_partials(p, m, c, k, has_gain);
    __syncthreads();
  }
  if (tid == 0 && p.L > 1 && n_own > 0) prefetch_router(p, m, rch, 1, n_own);
  if (!grid_sync(p, m)) return;
  stamp(p, p.L, 1);

  for (int l = 0; l < p.L; ++l) {
    stamp(p, l, 0);
    const bool next = l + 1 < p.L;
    // ---------------------------------------------------------------- R phase
    // stage this layer's inputs: every load of the phase is issued before any is used
    float4 hreg[4], greg[4];
    int32_t preg[4];
    {
      const float4* h4 = reinterpret_cast<const float4*>(p.h);
      const float4* g4 = has_gain ? reinterpret_cast<const float4*>(p.gain + (size_t)l * H) : nullptr;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = tid + q * kThreads;
        if (t < H / 4) {
          hreg[q] = __ldcg(h4 + t);
          if (has_gain) greg[q] = __ldg(g4 + t);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = tid + q * kThreads;
        if (e < p.E) preg[q] = __ldg(p.pin_slot + (size_t)l * p.E + e);
      }
      const int par = m.step & 1;
      const size_t rs = ((size_t)par * p.L + l) * p.R;
      if (tid < p.R) {
        m.ring_owner[tid] = __ldcg(p.ring_owner + rs + tid);
        m.ring_stamp[tid] = __ldcg(p.ring_stamp + rs + tid);
      }
      if (tid == kThreads - 1) m.ring_clock = __ldcg(p.ring_clock + (size_t)par * p.L + l);
      if (tid == kThreads - 2) m.P_l = __ldg(p.n_pinned + l);
      if (tid == kThreads - 3) m.base_l = __ldg(p.layer_base + l);
      if (next && tid < n_own * kChunk) {
        const int k = tid / kChunk, t = tid % kChunk;
        const int c = blockIdx.x + k * gridDim.x;
        m.gnext[k][t] = has_gain ? __ldg(p.gain + (size_t)(l + 1) * H + c * kChunk + t) : 1.0f;
      }
    }
    // logits of this CTA's experts (and the norm scale, in every CTA)
    {
      float inv = 1.0f;
      if (p.use_norm) {
        const float ss = canonical_fold(p.sq, p.nch, lane);
        inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)H), p.eps)));
      }
      if (warp == 0 && lane == 0) m.inv = inv;
      for (int e = blockIdx.x * kWarps + warp; e < p.E; e += gridDim.x * kWarps) {
        const float sum = canonical_fold(p.part + (size_t)e * p.nch, p.nch, lane);
        if (lane == 0) __stcg(p.z + e, fmaf(sum, inv, p.bias ? __ldg(p.bias + (size_t)l * p.E + e) : 0.0f));
      }
    }
    const int n_folders = min((int)gridDim.x, (p.E + kWarps - 1) / kWarps);  // CTAs holding logits
    if ((int)blockIdx.x < n_folders) publish(p, &p.ctrl->z_count);
    {
      float4* hb4 = reinterpret_cast<float4*>(hbuf);
      float4* gb4 = reinterpret_cast<float4*>(gbuf);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = tid + q * kThreads;
        if (t < H / 4) {
          hb4[t] = hreg[q];
          if (has_gain) gb4[t] = greg[q];
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = tid + q * kThreads;
        if (e < p.E) pinrow[e] = preg[q];
      }
    }
    __syncthreads();
    // quantised activations x = RMSNorm(h) (or h): four lanes per 32-block, each lane 8
    // values; the block's largest |x| and code sum combine over the four lanes
    {
      const float inv = m.inv;
      const int j4 = tid & 3;
      for (int b0 = tid >> 2; b0 < ((nb + 63) / 64) * 64; b0 += kThreads / 4) {
        const int b = b0 < nb ? b0 : nb - 1;  // lanes past the end repeat a block, write nothing
        float v[8];
        const float4* h4 = reinterpret_cast<const float4*>(hbuf + b * 32 + 8 * j4);
        const float4* g4 = reinterpret_cast<const float4*>(gbuf + b * 32 + 8 * j4);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float4 hv = h4[q];
          if (p.use_norm) {
            hv.x = __fmul_rn(hv.x, inv);
            hv.y = __fmul_rn(hv.y, inv);
            hv.z = __fmul_rn(hv.z, inv);
            hv.w = __fmul_rn(hv.w, inv);
            if (has_gain) {
              const float4 gv = g4[q];
              hv.x = __fmul_rn(hv.x, gv.x);
              hv.y = __fmul_rn(hv.y, gv.y);
              hv.z = __fmul_rn(hv.z, gv.z);
              hv.w = __fmul_rn(hv.w, gv.w);
            }
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
        if (b0 < nb) {
          reinterpret_cast<uint4*>(xcodes + b * 32)[j4] =
              make_uint4(((uint32_t)c[0] & 0xffffu) | ((uint32_t)c[1] << 16),
                         ((uint32_t)c[2] & 0xffffu) | ((uint32_t)c[3] << 16),
                         ((uint32_t)c[4] & 0xffffu) | ((uint32_t)c[5] << 16),
                         ((uint32_t)c[6] & 0xffffu) | ((uint32_t)c[7] << 16));
          if (j4 == 0) {
            xs[b] = amax * (1.0f / (32767.0f * 16.0f));
            xc[b] = csum;
          }
        }
      }
    }
    __syncthreads();
    stamp(p, l, 1);

    // ---------------------------------------------------------------- routing
    if (!await_count(p, m, &p.ctrl->z_count, (uint32_t)(l + 1) * n_folders)) return;
    for (int e = tid; e < p.E; e += kThreads) zs[e] = __ldcg(p.z + e);
    if (!cta_ok(p, m.flag)) return;
    stamp(p, l, 8);
    if (warp == 0) {
      const int my_e = topk_weights(p, m, zs);
      stamp(p, l, 9);
      const bool fast = cache_all_pinned(p, m, l, pinrow, my_e);
      if (lane == 0) {
        if (!fast) cache_decide(p, m, l, pinrow);
        stamp(p, l, 10);
        m.unit_ok = (int)blockIdx.x < p.n_units ? issue_unit(p, m, unit, blockIdx.x) : 1;
        stamp(p, l, 11);
        m.d_issued = 0;
        stamp(p, l, 12);
      }
    }
    __syncthreads();
    if (!m.unit_ok) return;
    if (blockIdx.x == 0 && p.w_trace && tid < p.K) p.w_trace[(size_t)l * p.K + tid] = m.w[tid];
    for (int k = 0; k < n_own; ++k) prefetch_dchunk_l2(p, m, blockIdx.x + k * gridDim.x);
    stamp(p, l, 2);
    cta_stamp(p, l, 0);

    // ---------------------------------------------------------------- G phase
    {
      // lane groups of GS lanes per row; each lane covers BPL blocks of the row
      const int GS = pow2_ceil_le32(nb), RPW = 32 / GS, g = lane % GS, sub = lane / GS;
      const int rows_per_lane = (2 * kUnitRows + kWarps * RPW - 1) / (kWarps * RPW);
      int4 xq[BPL][4];
      float xsc[BPL];
      int xsum[BPL];
#pragma unroll
      for (int mb = 0; mb < BPL; ++mb) {
        const int b = g + GS * mb;
        if (b < nb) {
          const int4* src = reinterpret_cast<const int4*>(xcodes + b * 32);
          xq[mb][0] = src[0];
          xq[mb][1] = src[1];
          xq[mb][2] = src[2];
          xq[mb][3] = src[3];
          xsc[mb] = xs[b];
          xsum[mb] = xc[b];
        } else {
          xq[mb][0] = xq[mb][1] = xq[mb][2] = xq[mb][3] = make_int4(0, 0, 0, 0);
          xsc[mb] = 0.0f;
          xsum[mb] = 0;
        }
      }
      const int routed = p.K * (p.I / 32);
      for (int u = blockIdx.x, k = 0; u < p.n_units; u += gridDim.x, ++k) {
        const int i = u < routed ? u / (p.I / 32) : p.K;
        const int rb = u < routed ? u % (p.I / 32) : u - routed;
        if (k > 0) {
          __syncthreads();  // the previous unit's buffer is free
          if (tid == 0) m.flag = issue_unit(p, m, unit, u);
          __syncthreads();
          if (!m.flag) return;
        }
        uint32_t done = 0;
        // four rows at a time per lane group, their dot products and reductions
        // interleaved; row r of the unit: gate rows 0-31, then up rows 0-31
        for (int k0 = 0; k0 < rows_per_lane; k0 += 4) {
          int rows[4];
          float acc[4];
          bool live[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            rows[q] = warp * RPW + sub + (k0 + q) * kWarps * RPW;
            live[q] = k0 + q < rows_per_lane && rows[q] < 2 * kUnitRows;
            acc[q] = 0.0f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (!live[q]) continue;
            const int st = rows[q] / 16;
            if (!((done >> st) & 1u)) {
              if (!mbar_wait(p, &m.bar_u[st], par_u[st])) return;
              done |= 1u << st;
            }
          }
          stamp(p, l, 7);
#pragma unroll
          for (int mb = 0; mb < BPL; ++mb) {
            const int b = g + GS * mb;
            if (b >= nb) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (!live[q]) continue;
              const int r = rows[q];
              const uint8_t* tile = unit + (r / 16) * 9u * H;
              const uint4 qv = *reinterpret_cast<const uint4*>(tile + ((size_t)(r % 16) * nb + b) * 16);
              const float d = __half2float(reinterpret_cast<const __half*>(tile + 8u * H)[(r % 16) * nb + b]);
              const int v = q4_block_dot16(qv, xq[mb][0], xq[mb][1], xq[mb][2], xq[mb][3]) - 128 * xsum[mb];
              acc[q] = fmaf(d * xsc[mb], (float)v, acc[q]);
            }
          }
          for (int off = GS / 2; off >= 1; off >>= 1) {
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], off);
          }
          if (g == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (live[q]) m.gu[rows[q]] = acc[q];
          }
        }
#pragma unroll
        for (int st = 0; st < 4; ++st) par_u[st] ^= 1u;
        stamp(p, l, 16);
        __syncthreads();
        stamp(p, l, 17);
        if (warp == 0) {
          const float gv = m.gu[lane], uv = m.gu[kUnitRows + lane];
          const float a = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
          stamp(p, l, 18);
          float sc;
          int csum;
          const int code = quant_block(a, sc, csum);
          stamp(p, l, 19);
          uint8_t* rec = p.acodes + ((size_t)i * rec_per_exp + rb) * kACodeBytes;
          __stcg(reinterpret_cast<int16_t*>(rec) + lane, (int16_t)code);
          if (lane == 0) {
            __stcg(reinterpret_cast<float*>(rec + 64), sc);
            __stcg(reinterpret_cast<int32_t*>(rec + 68), csum);
          }
          stamp(p, l, 20);
        }
      }
    }
    const int n_producers = min((int)gridDim.x, p.n_units);  // CTAs holding gate/up units
    stamp(p, l, 21);
    if ((int)blockIdx.x < n_producers) publish(p, &p.ctrl->a_count);
    stamp(p, l, 3);
    cta_stamp(p, l, 1);
    stamp(p, l, 4);

    // ---------------------------------------------------------------- D phase
    // (CTAs that own rows) wait for every activation record of the layer and for the miss
    // copies the down tiles depend on; tiles and records are then read from L2
    if (n_own > 0) {
      if (tid == 0) {
        m.flag = 1;
        for (int i = 0; i < p.n_exp; ++i)
          if (!wait_miss(p, m.miss_seq[i])) m.flag = 0;
      }
      if (!await_count(p, m, &p.ctrl->a_count, (uint32_t)(l + 1) * n_producers)) return;
    }
    if (!cta_ok(p, m.flag)) return;
    stamp(p, l, 13);
    for (int k = 0; k < n_own; ++k) {
      const int c = blockIdx.x + k * gridDim.x;
      stamp(p, l, 14);
      // thread (expert i, block column b0): all 16 rows of chunk c against block b0 (then
      // b0+16, ...) of a_i, every load of a block issued before any is used; then a
      // 15-shuffle transpose reduction over the expert's 16 lanes leaves row b0 in lane b0
      {
        const int b0 = tid & 15;
        // warp-uniform loop: lanes 0-15 take expert base, lanes 16-31 expert base + 1
        for (int base = 2 * warp; base < p.n_exp; base += 2 * kWarps) {
          const int i = base + (lane >> 4);
          const bool act = i < p.n_exp;
          const int Ii = !act ? 0 : (i < p.K ? p.I : p.Is);
          const int nbd = Ii / 32;
          const uint8_t* tile =
              act ? m.src[i] + (i < p.K ? p.lay.down : p.slay.down) + (size_t)c * 9u * Ii : nullptr;
          float acc[kChunk];
#pragma unroll
          for (int r = 0; r < kChunk; ++r) acc[r] = 0.0f;
          for (int b = b0; b < nbd; b += 16) {
            const uint4* rec = reinterpret_cast<const uint4*>(p.acodes + ((size_t)i * rec_per_exp + b) * kACodeBytes);
            const uint4 r0 = __ldcg(rec), r1 = __ldcg(rec + 1), r2 = __ldcg(rec + 2), r3 = __ldcg(rec + 3),
                        r4 = __ldcg(rec + 4);
            uint4 qv[kChunk];
            unsigned short dv[kChunk];
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
              qv[r] = __ldcg(reinterpret_cast<const uint4*>(tile + ((size_t)r * nbd + b) * 16));
              dv[r] = __ldcg(reinterpret_cast<const unsigned short*>(tile + 8u * Ii) + (size_t)r * nbd + b);
            }
            const int4 a0 = make_int4(r0.x, r0.y, r0.z, r0.w), a1 = make_int4(r1.x, r1.y, r1.z, r1.w),
                       a2 = make_int4(r2.x, r2.y, r2.z, r2.w), a3 = make_int4(r3.x, r3.y, r3.z, r3.w);
            const float sc = __uint_as_float(r4.x);
            const int cs128 = 128 * (int)r4.y;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
              const int v = q4_block_dot16(qv[r], a0, a1, a2, a3) - cs128;
              acc[r] = fmaf(__half2float(__ushort_as_half(dv[r])) * sc, (float)v, acc[r]);
            }
          }
#pragma unroll
          for (int h = 8; h >= 1; h >>= 1) {
            const bool up = (b0 & h) != 0;
#pragma unroll
            for (int r = 0; r < h; ++r) {
              const float send = up ? acc[r] : acc[r + h];
              const float keep = up ? acc[r + h] : acc[r];
              acc[r] = keep + __shfl_xor_sync(0xffffffffu, send, h);
            }
          }
          if (act) os[i * kChunk + b0] = acc[0];
        }
      }
      __syncthreads();
      stamp(p, l, 15);
      if (tid < kChunk) {
        const int j = c * kChunk + tid;
        float y = 0.0f;
        for (int i = 0; i < p.K; ++i) y = fmaf(m.w[i], os[i * kChunk + tid], y);
        if (p.Is > 0) y = __fadd_rn(y, os[p.K * kChunk + tid]);
        const float hn = p.use_norm ? __fadd_rn(m.hown[k][tid], y) : y;
        m.hown[k][tid] = hn;
        __stcg(p.h + j, hn);
        if (p.h_trace) p.h_trace[(size_t)(l + 1) * H + j] = hn;
        if (l == p.L - 1) p.y[j] = hn;
      }
      if (next) {
        if (k == 0 && !mbar_wait(p, &m.bar_r, par_r)) return;
        router_partials(p, m, c, m.hown[k], has_gain ? m.gnext[k] : nullptr, [&](int e) {
          return reinterpret_cast<const uint4*>(rch + (size_t)k * 32u * p.E + (size_t)e * 32u);
        });
      }
      __syncthreads();
    }
    if (next && n_own > 0) par_r ^= 1u;
    // the router columns for layer l + 2 load during the barrier (rch is free again)
    if (tid == 0 && l + 2 < p.L && n_own > 0) prefetch_router(p, m, rch, l + 2, n_own);
    stamp(p, l, 5);
    cta_stamp(p, l, 2);
    if (!grid_sync(p, m)) return;
    stamp(p, l, 6);
    cta_stamp(p, l, 3);

    // deferred ring fills (only when a layer misses more often than it has ring slots)
    for (int f = 0; f < m.n_fix; ++f) {
      const uint4* s = reinterpret_cast<const uint4*>(p.pool + (size_t)m.fix_src[f] * p.slot_bytes);
      uint4* d = reinterpret_cast<uint4*>(const_cast<uint8_t*>(p.pool) + (size_t)m.fix_dst[f] * p.slot_bytes);
      const size_t n16 = p.slot_bytes / 16;
      for (size_t t = (size_t)blockIdx.x * kThreads + tid; t < n16; t += (size_t)gridDim.x * kThreads)
        d[t] = __ldcg(s + t);
    }
  }
  stamp(p, p.L, 2);
  if (blockIdx.x == 0 && tid == 0) {
    p.ctrl->step = m.step + 1;
    p.ctrl->req_seq = m.seq_base + m.n_miss;
  }
}

// ------------------------------------------------------------------ host-side launch

uint32_t decode_smem_bytes(int H, int E, int K, int I, int Is, int nown) {
  return smem_plan(H, E, K, I, Is, nown).total;
}

// Blocks of one gate/up row each lane covers: 1 below 1024 columns, else H / 1024.
static int bpl_of(int H) {
  const int nb = H / 32;
  return nb <= 32 ? 1 : (nb + 31) / 32;
}

template <typename F>
static cudaError_t with_kernel(int H, F f) {
  switch (bpl_of(H)) {
    case 1: return f(moe_decode_kernel<1>);
    case 2: return f(moe_decode_kernel<2>);
    case 3: return f(moe_decode_kernel<3>);
    default: return f(moe_decode_kernel<4>);
  }
}

cudaError_t decode_configure(int H, int E, int K, int I, int Is, int nown) {
  const uint32_t bytes = decode_smem_bytes(H, E, K, I, Is, nown);
  return with_kernel(H, [&](auto kern) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  });
}

cudaError_t decode_max_blocks_per_sm(int H, int E, int K, int I, int Is, int nown, int* out) {
  return with_kernel(H, [&](auto kern) {
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kern, kThreads, decode_smem_bytes(H, E, K, I, Is, nown));
  });
}

cudaError_t decode_launch(const DecodeParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(p.H, p.E, p.K, p.I, p.Is, p.nown);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return with_kernel(p.H, [&](auto kern) { return cudaLaunchKernelEx(&cfg, kern, p); });
}

}  // namespace moe
