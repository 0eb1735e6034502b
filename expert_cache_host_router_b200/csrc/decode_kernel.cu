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

// Canonical fold of n partials (stride 1) by one warp; every lane returns the total.
__device__ __forceinline__ float canonical_fold(const float* parts, int n, int lane) {
  float acc = 0.0f;
  for (int m = lane; m < n; m += 32) acc = __fadd_rn(acc, __ldcg(parts + m));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
  return acc;
}

__host__ __device__ inline int pow2_ceil_le32(int n) {
  int g = 1;
  while (g < n && g < 32) g <<= 1;
  return g;
}

// ------------------------------------------------------------------ shared memory plan

struct Misc {
  uint64_t bar[2];
  const uint8_t* src[kMaxK + 1];  // slot base of each active expert (rank order, then shared)
  uint32_t miss_seq[kMaxK + 1];   // copy to wait for (0: resident)
  int32_t sel[kMaxK];
  float w[kMaxK];
  int32_t fix_dst[kMaxR], fix_src[kMaxR];  // deferred ring fills (pool indices)
  int32_t n_fix;
  float hchunk[kChunk];
  float u[kChunk];
  float gu[2 * kUnitRows];
  float inv;
  uint32_t step, seq_base, n_miss, gen;
  int32_t flag;
};

struct SmemPlan {
  uint32_t unit, dchunk, z, xcodes, xs, xc, acodes, o, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemPlan smem_plan(int H, int E, int K, int I, int Is) {
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
  s.unit = take(36u * H);                       // gate qs|d, up qs|d for 32 rows
  s.dchunk = take(9u * (uint32_t)(K * I + Is)); // down rows of one chunk, all experts
  s.z = take(4u * E);
  s.xcodes = take(2u * H);
  s.xs = take(4u * (H / 32));
  s.xc = take(4u * (H / 32));
  s.acodes = take((uint32_t)kACodeBytes * n_exp * (imax / 32));
  s.o = take(4u * n_exp * kChunk);
  s.misc = take(sizeof(Misc));
  s.total = align_up(off, 128);
  return s;
}

// ------------------------------------------------------------------ barriers and waits

// Grid barrier over all CTAs (co-resident by cooperative launch).  Returns false when
// the wait ran out or another CTA flagged an error.
__device__ bool grid_sync(const DecodeParams& p, Misc& m) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint32_t gen = m.gen;
    __threadfence();
    const uint32_t arrived = atomicAdd(&p.ctrl->bar_count, 1u);
    if (arrived == gridDim.x - 1) {
      atomicExch(&p.ctrl->bar_count, 0u);
      __threadfence();
      atomicExch(&p.ctrl->bar_gen, gen + 1);
    } else {
      const uint64_t t0 = gtimer();
      while (ld_acquire(&p.ctrl->bar_gen) == gen) {
        if (has_error(p.ctrl)) {
          ok = 0;
          break;
        }
        if (gtimer() - t0 > p.timeout_ns) {
          set_error(p.ctrl, MOE_DEVERR_BARRIER);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    m.gen = gen + 1;
    m.flag = ok && !has_error(p.ctrl);
  }
  __syncthreads();
  return m.flag != 0;
}

// Thread 0: wait until the proxy has signalled miss copy seq (0: nothing to wait for).
__device__ bool wait_miss(const DecodeParams& p, uint32_t seq) {
  if (seq == 0) return true;
  if ((int32_t)(ld_acquire(p.done_seq) - seq) >= 0) {
    fence_proxy_async();
    return true;
  }
  const uint64_t t0 = gtimer();
  while ((int32_t)(ld_acquire(p.done_seq) - seq) < 0) {
    if (has_error(p.ctrl)) return false;
    if (gtimer() - t0 > p.timeout_ns) {
      set_error(p.ctrl, MOE_DEVERR_MISS);
      return false;
    }
  }
  fence_proxy_async();
  return true;
}

// All threads: wait for the bulk copies counted on bar to land (bounded).
__device__ bool mbar_wait(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(bar, parity)) {
    if (gtimer() - t0 > p.timeout_ns) {
      set_error(p.ctrl, MOE_DEVERR_TMA);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ phases

// Router partials of layer l over chunk c (16 columns of h held in m.hchunk), and the
// chunk's sum of squares for the RMSNorm of layer l.
__device__ void router_partials(const DecodeParams& p, Misc& m, int l, int c) {
  const int tid = threadIdx.x;
  if (tid < kChunk) {
    const float hv = m.hchunk[tid];
    float u = hv;
    if (p.use_norm && p.gain) u = __fmul_rn(p.gain[(size_t)l * p.H + c * kChunk + tid], hv);
    m.u[tid] = u;
  }
  __syncthreads();
  for (int e = tid; e < p.E; e += kThreads) {
    const uint4* wp = reinterpret_cast<const uint4*>(p.router + (((size_t)l * p.nch + c) * p.E + e) * kChunk);
    const uint4 w0 = __ldg(wp), w1 = __ldg(wp + 1);
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
    for (int t = 0; t < kChunk; ++t) s = fmaf(m.hchunk[t], m.hchunk[t], s);
    __stcg(p.sq + c, s);
  }
}

// Warp 0: top-k of z (value desc, index asc) and the renormalised softmax weights.
__device__ void topk_weights(const DecodeParams& p, Misc& m, const float* zs) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;
  for (int i = 0; i < p.K; ++i) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    for (int mb = 0; lane + 32 * mb < p.E; ++mb) {
      const int e = lane + 32 * mb;
      if ((taken >> mb) & 1u) continue;
      const float v = zs[e];
      if (v > bv || (v == bv && e < be)) {
        bv = v;
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be == 0x7fffffff) {
      if (lane == 0) set_error(p.ctrl, MOE_DEVERR_ROUTE);
      be = 0;
    }
    if (lane == (be & 31)) taken |= 1u << (be >> 5);
    if (lane == 0) m.sel[i] = be;
  }
  __syncwarp();
  if (lane == 0) {
    const float zmax = zs[m.sel[0]];
    float ex[kMaxK];
    float s = 0.0f;
    for (int i = 0; i < p.K; ++i) {
      ex[i] = expf(zs[m.sel[i]] - zmax);
      s += ex[i];
    }
    for (int i = 0; i < p.K; ++i) m.w[i] = ex[i] / s;
  }
}

// Thread 0 of every CTA: the cache decision for layer l (identical in all CTAs).  CTA 0
// also commits the next ring state, the event log, histogram, counters and requests.
__device__ void cache_decide(const DecodeParams& p, Misc& m, int l) {
  const int R = p.R, E = p.E, K = p.K;
  const int par = m.step & 1;
  const bool commit = blockIdx.x == 0;
  const int P = p.n_pinned[l];
  const int base = p.layer_base[l];
  int32_t owner[kMaxR];
  uint32_t stamp[kMaxR];
  bool busy[kMaxR];
  int32_t fix[kMaxR];
  const size_t rs = ((size_t)par * p.L + l) * R;
  uint32_t clock = __ldcg(p.ring_clock + (size_t)par * p.L + l);
  for (int r = 0; r < R; ++r) {
    owner[r] = __ldcg(p.ring_owner + rs + r);
    stamp[r] = __ldcg(p.ring_stamp + rs + r);
    busy[r] = false;
    fix[r] = -1;
  }
  unsigned long long n_pin = 0, n_ring = 0, n_miss = 0, n_evict = 0, n_staged = 0;
  for (int i = 0; i < K; ++i) {
    const int e = m.sel[i];
    const int ps = p.pin_slot[(size_t)l * E + e];
    int kind, slot_log, evicted = -1, pool_idx;
    uint32_t seq = 0;
    if (ps >= 0) {
      kind = MOE_PIN_HIT;
      slot_log = ps;
      pool_idx = base + ps;
      ++n_pin;
    } else {
      int r = -1;
      for (int rr = 0; rr < R; ++rr)
        if (owner[rr] == e) r = rr;
      if (r >= 0) {
        kind = MOE_RING_HIT;
        stamp[r] = ++clock;
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
          if (owner[rr] < 0) v = rr;
        if (v < 0) {
          v = 0;
          for (int rr = 1; rr < R; ++rr)
            if (stamp[rr] < stamp[v]) v = rr;
        }
        evicted = owner[v];
        owner[v] = e;
        stamp[v] = ++clock;
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
      atomicAdd(p.hist + (size_t)l * E + e, 1u);
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
      p.ring_owner[ws + r] = owner[r];
      p.ring_stamp[ws + r] = stamp[r];
    }
    p.ring_clock[(size_t)(par ^ 1) * p.L + l] = clock;
    p.ctrl->pin_hits += n_pin;
    p.ctrl->ring_hits += n_ring;
    p.ctrl->misses += n_miss;
    p.ctrl->evictions += n_evict;
    p.ctrl->staged += n_staged;
  }
}

// ------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemPlan S = smem_plan(p.H, p.E, p.K, p.I, p.Is);
  Misc& m = *reinterpret_cast<Misc*>(smem + S.misc);
  float* zs = reinterpret_cast<float*>(smem + S.z);
  int16_t* xcodes = reinterpret_cast<int16_t*>(smem + S.xcodes);
  float* xs = reinterpret_cast<float*>(smem + S.xs);
  int32_t* xc = reinterpret_cast<int32_t*>(smem + S.xc);
  uint8_t* acs = smem + S.acodes;
  float* os = reinterpret_cast<float*>(smem + S.o);
  uint8_t* unit = smem + S.unit;
  uint8_t* dch = smem + S.dchunk;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, nb = H / 32;
  const int imax = p.I > p.Is ? p.I : p.Is;
  const int rec_per_exp = imax / 32;

  if (tid == 0) {
    mbar_init(&m.bar[0], 1);
    mbar_init(&m.bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    m.step = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->step);
    m.seq_base = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->req_seq);
    m.gen = *reinterpret_cast<volatile uint32_t*>(&p.ctrl->bar_gen);
    m.n_miss = 0;
    m.flag = !has_error(p.ctrl);
  }
  __syncthreads();
  if (!m.flag) return;
  uint32_t par0 = 0, par1 = 0;  // mbarrier phase parities (uniform across threads)

  // ---- prologue: h = x, and layer 0's router partials
  for (int c = blockIdx.x; c < p.nch; c += gridDim.x) {
    if (tid < kChunk) {
      const float v = p.x[c * kChunk + tid];
      m.hchunk[tid] = v;
      __stcg(p.h + c * kChunk + tid, v);
      if (p.h_trace) p.h_trace[c * kChunk + tid] = v;
    }
    __syncthreads();
    router_partials(p, m, 0, c);
    __syncthreads();
  }
  if (!grid_sync(p, m)) return;

  for (int l = 0; l < p.L; ++l) {
    // ---------------------------------------------------------------- R phase
    if (warp == 0) {
      float inv = 1.0f;
      if (p.use_norm) {
        const float ss = canonical_fold(p.sq, p.nch, lane);
        inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)H), p.eps)));
      }
      if (lane == 0) m.inv = inv;
    }
    __syncthreads();
    {
      const float inv = m.inv;
      for (int e = blockIdx.x * kWarps + warp; e < p.E; e += gridDim.x * kWarps) {
        const float s = canonical_fold(p.part + (size_t)e * p.nch, p.nch, lane);
        if (lane == 0) __stcg(p.z + e, fmaf(s, inv, p.bias ? p.bias[(size_t)l * p.E + e] : 0.0f));
      }
    }
    if (!grid_sync(p, m)) return;

    // ---------------------------------------------------------------- routing
    for (int e = tid; e < p.E; e += kThreads) zs[e] = __ldcg(p.z + e);
    __syncthreads();
    if (warp == 0) topk_weights(p, m, zs);
    __syncthreads();
    if (tid == 0) cache_decide(p, m, l);
    if (blockIdx.x == 0 && p.w_trace && tid < p.K) p.w_trace[(size_t)l * p.K + tid] = m.w[tid];
    // quantised activations: x = RMSNorm(h) (or h), int16 codes per 32-block
    {
      const float inv = m.inv;
      for (int b = warp; b < nb; b += kWarps) {
        const int j = b * 32 + lane;
        const float hv = __ldcg(p.h + j);
        float xv = hv;
        if (p.use_norm) {
          xv = __fmul_rn(hv, inv);
          if (p.gain) xv = __fmul_rn(xv, p.gain[(size_t)l * H + j]);
        }
        const float amax = warp_max(fabsf(xv));
        int code = 0;
        if (amax > 0.0f) {
          code = __float2int_rn(xv * (32767.0f / amax));
          code = max(-32767, min(32767, code));
        }
        const int csum = warp_sum_int(code);
        xcodes[j] = (int16_t)code;
        if (lane == 0) {
          xs[b] = amax > 0.0f ? (amax / 32767.0f) * 0.0625f : 0.0f;
          xc[b] = csum;
        }
      }
    }
    __syncthreads();

    // ---------------------------------------------------------------- G phase
    {
      const int GS = pow2_ceil_le32(nb), RPW = 32 / GS, g = lane % GS, sub = lane / GS;
      const int bpl = (nb + GS - 1) / GS;
      int4 xq[4][4];
      float xsc[4];
      int xsum[4];
#pragma unroll
      for (int mb = 0; mb < 4; ++mb) {
        const int b = g + GS * mb;
        if (mb < bpl && b < nb) {
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
      const int units_routed = p.K * (p.I / 32);
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int i = u < units_routed ? u / (p.I / 32) : p.K;
        const int rb = u < units_routed ? u % (p.I / 32) : u - units_routed;
        const SlotLayout& L = i < p.K ? p.lay : p.slay;
        if (tid == 0) {
          int ok = wait_miss(p, m.miss_seq[i]);
          if (ok) {
            const uint8_t* s = m.src[i];
            const uint32_t qb = 16u * H, db = 2u * H;  // 32 rows
            mbar_expect_tx(&m.bar[0], 2 * (qb + db));
            bulk_g2s(unit, s + L.gate.qs + (size_t)rb * qb, qb, &m.bar[0]);
            bulk_g2s(unit + qb, s + L.gate.d + (size_t)rb * db, db, &m.bar[0]);
            bulk_g2s(unit + qb + db, s + L.up.qs + (size_t)rb * qb, qb, &m.bar[0]);
            bulk_g2s(unit + 2 * qb + db, s + L.up.d + (size_t)rb * db, db, &m.bar[0]);
          }
          m.flag = ok;
        }
        __syncthreads();
        if (!m.flag) return;
        if (!mbar_wait(p, &m.bar[0], par0)) return;
        par0 ^= 1u;
        for (int r = warp * RPW + sub; r < 2 * kUnitRows; r += kWarps * RPW) {
          const uint8_t* qbase = unit + (r < kUnitRows ? 0 : 18u * H) + (size_t)(r % kUnitRows) * nb * 16;
          const __half* dbase = reinterpret_cast<const __half*>(unit + (r < kUnitRows ? 0 : 18u * H) + 16u * H) +
                                (size_t)(r % kUnitRows) * nb;
          float acc = 0.0f;
#pragma unroll
          for (int mb = 0; mb < 4; ++mb) {
            const int b = g + GS * mb;
            if (mb < bpl && b < nb) {
              const uint4 q = *reinterpret_cast<const uint4*>(qbase + b * 16);
              const float d = __half2float(dbase[b]);
              const int v = q4_block_dot16(q, xq[mb][0], xq[mb][1], xq[mb][2], xq[mb][3]) - 128 * xsum[mb];
              acc = fmaf(d * xsc[mb], (float)v, acc);
            }
          }
          for (int off = GS / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (g == 0) m.gu[r] = acc;
        }
        __syncthreads();
        if (warp == 0) {
          const float gv = m.gu[lane], uv = m.gu[kUnitRows + lane];
          const float a = __fdiv_rn(gv, 1.0f + expf(-gv)) * uv;
          const float amax = warp_max(fabsf(a));
          int code = 0;
          if (amax > 0.0f) {
            code = __float2int_rn(a * (32767.0f / amax));
            code = max(-32767, min(32767, code));
          }
          const int csum = warp_sum_int(code);
          uint8_t* rec = p.acodes + ((size_t)i * rec_per_exp + rb) * kACodeBytes;
          reinterpret_cast<int16_t*>(rec)[lane] = (int16_t)code;
          if (lane == 0) {
            reinterpret_cast<float*>(rec + 64)[0] = amax > 0.0f ? (amax / 32767.0f) * 0.0625f : 0.0f;
            reinterpret_cast<int32_t*>(rec + 68)[0] = csum;
          }
        }
        __syncthreads();
      }
    }
    if (!grid_sync(p, m)) return;

    // ---------------------------------------------------------------- D phase
    {
      const int n_rec = p.n_exp * rec_per_exp * (kACodeBytes / 8);
      const uint2* srcr = reinterpret_cast<const uint2*>(p.acodes);
      uint2* dstr = reinterpret_cast<uint2*>(acs);
      for (int t = tid; t < n_rec; t += kThreads) dstr[t] = __ldcg(srcr + t);
    }
    __syncthreads();
    for (int c = blockIdx.x; c < p.nch; c += gridDim.x) {
      if (tid == 0) {
        int ok = 1;
        uint32_t total = 0;
        for (int i = 0; i < p.n_exp; ++i) total += 9u * (i < p.K ? p.I : p.Is);
        for (int i = 0; i < p.n_exp && ok; ++i) ok = wait_miss(p, m.miss_seq[i]);
        if (ok) {
          mbar_expect_tx(&m.bar[1], total);
          uint32_t off = 0;
          for (int i = 0; i < p.n_exp; ++i) {
            const int Ii = i < p.K ? p.I : p.Is;
            const SlotLayout& L = i < p.K ? p.lay : p.slay;
            const uint32_t qb = 8u * Ii, db = (uint32_t)Ii;  // 16 rows
            bulk_g2s(dch + off, m.src[i] + L.down.qs + (size_t)c * qb, qb, &m.bar[1]);
            bulk_g2s(dch + off + qb, m.src[i] + L.down.d + (size_t)c * db, db, &m.bar[1]);
            off += qb + db;
          }
        }
        m.flag = ok;
      }
      __syncthreads();
      if (!m.flag) return;
      if (!mbar_wait(p, &m.bar[1], par1)) return;
      par1 ^= 1u;
      // tasks: (expert i, row group); each warp handles whole row groups
      {
        int task = 0;
        uint32_t off = 0;
        for (int i = 0; i < p.n_exp; ++i) {
          const int Ii = i < p.K ? p.I : p.Is;
          const int nbd = Ii / 32, GS = pow2_ceil_le32(nbd), RPW = 32 / GS, g = lane % GS, sub = lane / GS;
          const int passes = (kChunk + RPW - 1) / RPW;
          const uint8_t* qbase0 = dch + off;
          const __half* dbase0 = reinterpret_cast<const __half*>(dch + off + 8u * Ii);
          for (int ps = 0; ps < passes; ++ps, ++task) {
            if (task % kWarps != warp) continue;
            const int r = ps * RPW + sub;
            float acc = 0.0f;
            if (r < kChunk) {
              for (int b = g; b < nbd; b += GS) {
                const uint8_t* rec = acs + ((size_t)i * rec_per_exp + b) * kACodeBytes;
                const int4* ap = reinterpret_cast<const int4*>(rec);
                const uint4 q = *reinterpret_cast<const uint4*>(qbase0 + ((size_t)r * nbd + b) * 16);
                const float d = __half2float(dbase0[(size_t)r * nbd + b]);
                const float sc = reinterpret_cast<const float*>(rec + 64)[0];
                const int cs = reinterpret_cast<const int32_t*>(rec + 68)[0];
                const int v = q4_block_dot16(q, ap[0], ap[1], ap[2], ap[3]) - 128 * cs;
                acc = fmaf(d * sc, (float)v, acc);
              }
            }
            for (int o2 = GS / 2; o2 >= 1; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
            if (g == 0 && r < kChunk) os[i * kChunk + r] = acc;
          }
          off += 9u * Ii;
        }
      }
      __syncthreads();
      if (tid < kChunk) {
        const int j = c * kChunk + tid;
        float y = 0.0f;
        for (int i = 0; i < p.K; ++i) y = fmaf(m.w[i], os[i * kChunk + tid], y);
        if (p.Is > 0) y = __fadd_rn(y, os[p.K * kChunk + tid]);
        const float hn = p.use_norm ? __fadd_rn(__ldcg(p.h + j), y) : y;
        m.hchunk[tid] = hn;
        __stcg(p.h + j, hn);
        if (p.h_trace) p.h_trace[(size_t)(l + 1) * H + j] = hn;
        if (l == p.L - 1) p.y[j] = hn;
      }
      __syncthreads();
      if (l + 1 < p.L) router_partials(p, m, l + 1, c);
      __syncthreads();
    }
    if (!grid_sync(p, m)) return;

    // deferred ring fills (only when a layer misses more often than it has ring slots)
    for (int f = 0; f < m.n_fix; ++f) {
      const uint4* s = reinterpret_cast<const uint4*>(p.pool + (size_t)m.fix_src[f] * p.slot_bytes);
      uint4* d = reinterpret_cast<uint4*>(const_cast<uint8_t*>(p.pool) + (size_t)m.fix_dst[f] * p.slot_bytes);
      const size_t n16 = p.slot_bytes / 16;
      for (size_t t = (size_t)blockIdx.x * kThreads + tid; t < n16; t += (size_t)gridDim.x * kThreads)
        d[t] = __ldcg(s + t);
    }
  }
  if (!grid_sync(p, m)) return;
  if (blockIdx.x == 0 && tid == 0) {
    p.ctrl->step = m.step + 1;
    p.ctrl->req_seq = m.seq_base + m.n_miss;
  }
}

// ------------------------------------------------------------------ host-side launch

uint32_t decode_smem_bytes(int H, int E, int K, int I, int Is) { return smem_plan(H, E, K, I, Is).total; }

cudaError_t decode_configure(int H, int E, int K, int I, int Is) {
  const uint32_t bytes = decode_smem_bytes(H, E, K, I, Is);
  return cudaFuncSetAttribute(moe_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t decode_max_blocks_per_sm(int H, int E, int K, int I, int Is, int* out) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, moe_decode_kernel, kThreads,
                                                       decode_smem_bytes(H, E, K, I, Is));
}

cudaError_t decode_launch(const DecodeParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(p.H, p.E, p.K, p.I, p.Is);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel, p);
}

}  // namespace moe
