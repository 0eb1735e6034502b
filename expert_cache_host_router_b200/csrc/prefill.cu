// prefill.cu -- batched prefill of T tokens through the MoE stack (every expert resident)
// for libmoe: routing for every token in the same canonical fp32 order as decode, tokens
// grouped by expert, and the expert FFNs as a grouped GEMM on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, activation tiles brought in by TMA).
//
// The write-up serves decode; a prompt's tokens all pass the same layers at once, which
// turns each expert's GEMVs into GEMMs [n_e x H] x [H x 2I] and [n_e x I] x [I x H]
// (n_e = tokens routed to expert e): a dense contraction, so it runs on the tensor
// cores.  Per layer, in stream order:
//   route    8 tokens per CTA: RMSNorm scale, router logits in the canonical
//            order, top-k, weights, histogram, per-expert counts; x = RMSNorm(h) split
//            into fp16 hi + lo (x = hi + lo to about 2^-22 relative)
//   scan     expert offsets and the list of 128-row m-tiles
//   scatter  one warp per token: its rows of x copied to their place in expert order
//            (within an expert the order is whatever the atomics give: a GEMM row does
//            not depend on the other rows of its tile, so results are deterministic)
//   gemm     one CTA per 128 x 128 output tile: A (activation rows, fp16 hi and lo) by
//            TMA, B (Q4_0 weights) dequantised to fp16 into 128B-swizzled shared memory,
//            two tcgen05.mma per 16-wide K step (A_hi B and A_lo B) into one fp32
//            accumulator in tensor memory; gate/up tiles hold 64 gate and the matching
//            64 up columns so the epilogue forms a = silu(g) * u (stored as fp16 hi + lo);
//            down tiles write each row's expert output to its (token, rank) slot
//   combine  h += sum_rank w * o_rank + o_shared in rank order
// The activations are split because fp16 operands alone put the element-wise error at
// the tolerance; the weights are fp16((q - 8) * d), a relative error of at most 2^-12.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_cache.h"
#include "moe_internal.h"
#include "prefill.h"

namespace moe {

constexpr int kPT = 256;  // threads per prefill CTA
constexpr int kTM = 128;  // GEMM tile rows (tokens)
constexpr int kTN = 256;  // GEMM tile columns (weight rows of the B operand)
constexpr int kTK = 64;   // K per pipeline stage: one 128-byte swizzle row of fp16
constexpr int kStages = 3;
constexpr uint32_t kTileBytes = kTM * kTK * 2;   // 16 KB: one activation tile (hi or lo)
constexpr uint32_t kBTileBytes = kTN * kTK * 2;  // 32 KB: the weight tile
constexpr uint32_t kStageBytes = 2 * kTileBytes + kBTileBytes;
// Swizzled operand tiles first, each at a multiple of 1024 bytes (the 128-byte swizzle's
// period: TMA and the MMA take its phase from the address), then the raw weight bytes.
constexpr uint32_t kTilesBytes = kStageBytes * kStages;
static_assert(kTileBytes % 1024 == 0 && kBTileBytes % 1024 == 0, "operand tiles must keep the swizzle phase");

struct PrefillParams {
  int L, H, E, K, I, Is, use_norm, T, nch, tpc;
  int t_base, T_total;  // this chunk's first token and the call's token count (trace rows)
  int R;                // grouped rows of this chunk: T * k (+ T with a shared expert)
  float eps;
  const uint8_t* pool;  // layer l expert e at pool + (base[l] + (pin[l][e] & 0xffff)) * slot_bytes
  uint64_t slot_bytes;
  SlotLayout lay, slay;
  const uint8_t* shared_pool;
  uint64_t shared_slot_bytes;
  const uint16_t* router;  // [L][nch][E][16] bf16
  const float* bias;       // [L][E] or null
  const float* gain;       // [L][H]
  const int32_t* pin_slot;
  const int32_t* layer_base;
  uint32_t* hist;
  PrefillScratch s;
};

__device__ __forceinline__ uint32_t smem_u32p(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ float bf16_lo_p(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_p(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ const uint8_t* expert_slot(const PrefillParams& p, int l, int e) {
  if (e >= p.E) return p.shared_pool + (size_t)l * p.shared_slot_bytes;
  return p.pool + (size_t)(p.layer_base[l] + (p.pin_slot[(size_t)l * p.E + e] & 0xffff)) * p.slot_bytes;
}

// ------------------------------------------------------------------ route

constexpr int kRTok = 4;  // tokens per warp in the router

// Row stride of u in shared memory: 16-column chunks padded to 20 floats, so the four
// chunks that a warp's lanes read at once (one per residue, r chunks apart) fall in four
// different bank groups.
constexpr int kUChunk = 20;

// CTA of 8 warps, p.tpc (8) tokens.  Logit z_e of a token is the canonical fold of
// its 16-column chunk partials (each an fmaf chain from +0): fold lane q adds chunks
// q, q + 32, ... from +0, then the 32 lane sums combine as the xor butterfly 16, 8, 4, 2,
// 1 does.  In that butterfly's tree the sums of lanes q = r (mod 4) meet first (levels
// 16, 8, 4) and the four results meet last (levels 2, 1).  So here warp lane
// 4 * slot + r evaluates residue r's 8-leaf subtree (leaves in bit-reversed order, a
// 3-deep stack) for 4 tokens x 2 experts, and the last two levels are shuffles.  Lanes of
// one residue read the same u (one shared-memory wavefront for 8 lanes) and each weight
// a lane loads serves 4 tokens.
__global__ void __launch_bounds__(kPT, 2) prefill_route(const PrefillParams p, int l) {
  extern __shared__ __align__(16) float rsm[];
  const int H = p.H, E = p.E, nch = p.nch, TPC = p.tpc;
  const int ustride = nch * kUChunk;
  float* us = rsm;                        // [TPC][nch][20]  u = g * h (or h), padded chunks
  float* zs = us + (size_t)TPC * ustride;  // [TPC][E]
  float* invs = zs + (size_t)TPC * E;     // [TPC]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * TPC;
  const float* g = p.gain + (size_t)l * H;

  // 1. per token: inv (canonical fold of the squares), u into shared memory, x hi/lo out
  for (int tl = warp; tl < TPC; tl += kPT / 32) {
    const int t = t0 + tl;
    float* u = us + (size_t)tl * ustride;
    if (t >= p.T) {
      for (int j = lane; j < H; j += 32) u[(j >> 4) * kUChunk + (j & 15)] = 0.0f;
      if (lane == 0) invs[tl] = 1.0f;
      continue;
    }
    const float* hrow = p.s.h + (size_t)t * H;
    float inv = 1.0f;
    if (p.use_norm) {
      float acc = 0.0f;
      for (int c = lane; c < nch; c += 32) {
        const float4* hp = reinterpret_cast<const float4*>(hrow + c * 16);
        float pc = 0.0f;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float4 q = hp[v];
          pc = fmaf(q.x, q.x, pc);
          pc = fmaf(q.y, q.y, pc);
          pc = fmaf(q.z, q.z, pc);
          pc = fmaf(q.w, q.w, pc);
        }
        acc = __fadd_rn(acc, pc);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
      inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(acc, (float)H), p.eps)));
    }
    if (lane == 0) invs[tl] = inv;
    for (int j = lane; j < H; j += 32) {
      const float hv = hrow[j];
      float xv = hv;
      float* uj = u + (j >> 4) * kUChunk + (j & 15);
      if (p.use_norm) {
        *uj = __fmul_rn(g[j], hv);
        xv = __fmul_rn(__fmul_rn(hv, inv), g[j]);
      } else {
        *uj = hv;
      }
      const __half hi = __float2half_rn(xv);
      p.s.x_hi[(size_t)t * H + j] = hi;
      p.s.x_lo[(size_t)t * H + j] = __float2half_rn(xv - __half2float(hi));
    }
  }
  __syncthreads();

  // 2. logits: warp job = (token group of 4, block of 16 experts); lane = 4 * slot + r
  const int ntg = TPC / kRTok, nblk = (E + 15) / 16;
  const int r4 = lane & 3, slot = lane >> 2;
  for (int job = warp; job < ntg * nblk; job += kPT / 32) {
    const int tg = job % ntg, e0 = (job / ntg) * 16 + 2 * slot, e1 = e0 + 1;
    const bool v0 = e0 < E, v1 = e1 < E;
    const float* ub = us + (size_t)tg * kRTok * ustride;
    auto wload = [&](int c, uint4 (&w)[4]) {
      const uint4* w0p = reinterpret_cast<const uint4*>(p.router + (((size_t)l * nch + c) * E + e0) * kChunk);
      w[0] = w[1] = w[2] = w[3] = make_uint4(0, 0, 0, 0);
      if (v0) {
        w[0] = __ldg(w0p);
        w[1] = __ldg(w0p + 1);
      }
      if (v1) {
        w[2] = __ldg(w0p + 2);  // expert e0 + 1 follows e0 in the same chunk row
        w[3] = __ldg(w0p + 3);
      }
    };
    // leaf i' of this residue: fold lane r + 4 * brev3(i')
    auto leaf_q = [&](int i) { return r4 + 4 * (int)(__brev((unsigned)i) >> 29); };
    float stk[3][kRTok][2];
    float cr[kRTok][2];
    uint4 cw[4];
    if (leaf_q(0) < nch) wload(leaf_q(0), cw);
    for (int i = 0; i < 8; ++i) {
      const int q = leaf_q(i);
      float ls[kRTok][2];
#pragma unroll
      for (int t = 0; t < kRTok; ++t) ls[t][0] = ls[t][1] = 0.0f;
      for (int c = q; c < nch; c += 32) {
        // the next chunk this lane visits, loaded while this one is summed
        int cn = c + 32;
        if (cn >= nch) {
          cn = -1;
          for (int i2 = i + 1; i2 < 8; ++i2)
            if (leaf_q(i2) < nch) {
              cn = leaf_q(i2);
              break;
            }
        }
        uint4 nw[4];
        if (cn >= 0) wload(cn, nw);
        const uint32_t wa[8] = {cw[0].x, cw[0].y, cw[0].z, cw[0].w, cw[1].x, cw[1].y, cw[1].z, cw[1].w};
        const uint32_t wb[8] = {cw[2].x, cw[2].y, cw[2].z, cw[2].w, cw[3].x, cw[3].y, cw[3].z, cw[3].w};
        float pc[kRTok][2];
#pragma unroll
        for (int t = 0; t < kRTok; ++t) pc[t][0] = pc[t][1] = 0.0f;
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
#pragma unroll
          for (int t = 0; t < kRTok; ++t) {
            const float4 uv = *reinterpret_cast<const float4*>(ub + (size_t)t * ustride + c * kUChunk + 4 * j4);
            pc[t][0] = fmaf(bf16_lo_p(wa[2 * j4]), uv.x, pc[t][0]);
            pc[t][1] = fmaf(bf16_lo_p(wb[2 * j4]), uv.x, pc[t][1]);
            pc[t][0] = fmaf(bf16_hi_p(wa[2 * j4]), uv.y, pc[t][0]);
            pc[t][1] = fmaf(bf16_hi_p(wb[2 * j4]), uv.y, pc[t][1]);
            pc[t][0] = fmaf(bf16_lo_p(wa[2 * j4 + 1]), uv.z, pc[t][0]);
            pc[t][1] = fmaf(bf16_lo_p(wb[2 * j4 + 1]), uv.z, pc[t][1]);
            pc[t][0] = fmaf(bf16_hi_p(wa[2 * j4 + 1]), uv.w, pc[t][0]);
            pc[t][1] = fmaf(bf16_hi_p(wb[2 * j4 + 1]), uv.w, pc[t][1]);
          }
        }
#pragma unroll
        for (int t = 0; t < kRTok; ++t) {
          ls[t][0] = __fadd_rn(ls[t][0], pc[t][0]);
          ls[t][1] = __fadd_rn(ls[t][1], pc[t][1]);
        }
        if (cn >= 0) {
          cw[0] = nw[0];
          cw[1] = nw[1];
          cw[2] = nw[2];
          cw[3] = nw[3];
        }
      }
      // binary counter over the 8 leaves: level b combines while bit b of i is set
      bool carry = true;
#pragma unroll
      for (int b = 0; b < 3; ++b) {
        if (carry) {
          if ((i >> b) & 1) {
#pragma unroll
            for (int t = 0; t < kRTok; ++t) {
              ls[t][0] = __fadd_rn(stk[b][t][0], ls[t][0]);
              ls[t][1] = __fadd_rn(stk[b][t][1], ls[t][1]);
            }
          } else {
#pragma unroll
            for (int t = 0; t < kRTok; ++t) {
              stk[b][t][0] = ls[t][0];
              stk[b][t][1] = ls[t][1];
            }
            carry = false;
          }
        }
      }
      if (carry) {
#pragma unroll
        for (int t = 0; t < kRTok; ++t) {
          cr[t][0] = ls[t][0];
          cr[t][1] = ls[t][1];
        }
      }
    }
    // butterfly levels 2 and 1 across the four residues
#pragma unroll
    for (int off = 2; off >= 1; off >>= 1) {
#pragma unroll
      for (int t = 0; t < kRTok; ++t) {
        cr[t][0] = __fadd_rn(cr[t][0], __shfl_xor_sync(0xffffffffu, cr[t][0], off));
        cr[t][1] = __fadd_rn(cr[t][1], __shfl_xor_sync(0xffffffffu, cr[t][1], off));
      }
    }
    const float b0 = (p.bias && v0) ? __ldg(p.bias + (size_t)l * E + e0) : 0.0f;
    const float b1 = (p.bias && v1) ? __ldg(p.bias + (size_t)l * E + e1) : 0.0f;
#pragma unroll
    for (int t = 0; t < kRTok; ++t) {
      if ((t & 3) != r4) continue;  // the four residue lanes hold the same sums: share the stores
      const float inv = invs[tg * kRTok + t];
      if (v0) zs[(size_t)(tg * kRTok + t) * E + e0] = fmaf(cr[t][0], inv, b0);
      if (v1) zs[(size_t)(tg * kRTok + t) * E + e1] = fmaf(cr[t][1], inv, b1);
    }
  }
  __syncthreads();

  // 3. top-k by (logit desc, index asc; -0 == +0; NaN never preferred), weights, counts
  for (int tl = warp; tl < TPC; tl += kPT / 32) {
    const int t = t0 + tl;
    if (t >= p.T) continue;
    const float* z = zs + (size_t)tl * E;
    int my_e = -1;
    uint32_t taken = 0;
    for (int i = 0; i < p.K; ++i) {
      uint64_t best = 0;
      for (int k = 0; lane + 32 * k < E; ++k) {
        if ((taken >> k) & 1u) continue;
        const int e = lane + 32 * k;
        float v = z[e];
        if (v == 0.0f) v = 0.0f;
        const uint32_t uu = __float_as_uint(v);
        uint32_t o = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
        if (v != v) o = 0;
        const uint64_t key = ((uint64_t)o << 32) | (uint32_t)(~(uint32_t)e);
        best = key > best ? key : best;
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)best, off);
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(best >> 32), off);
        const uint64_t o = ((uint64_t)hi << 32) | lo;
        best = o > best ? o : best;
      }
      int e = (int)(~(uint32_t)best);
      if ((best >> 32) == 0ull) {  // only NaN logits left
        if (lane == 0) atomicCAS(p.s.error, 0, MOE_DEVERR_ROUTE);
        e = 0;
      }
      if ((e & 31) == lane) taken |= 1u << (e >> 5);
      if (lane == i) my_e = e;
    }
    const float zmax = __shfl_sync(0xffffffffu, lane < p.K ? z[my_e] : 0.0f, 0);
    const float ex = lane < p.K ? expf(z[my_e] - zmax) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < p.K) {
      p.s.sel[(size_t)t * p.K + lane] = my_e;
      p.s.w[(size_t)t * p.K + lane] = __fdividef(ex, sum);
      atomicAdd(p.hist + (size_t)l * E + my_e, 1u);
      atomicAdd(p.s.counts + my_e, 1);
      if (p.s.sel_trace) p.s.sel_trace[((size_t)l * p.T_total + p.t_base + t) * p.K + lane] = my_e;
    }
  }
}

// ------------------------------------------------------------------ grouping

// One CTA of 1024 threads: exclusive offsets over experts 0..E (E = the shared expert,
// which takes every token), the list of 128-row m-tiles, and the counters zeroed for the
// next layer.
__global__ void __launch_bounds__(1024) prefill_scan(const PrefillParams p) {
  __shared__ int wsum[32], wtil[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_ent = p.E + 1;
  int n[2] = {0, 0}, m[2] = {0, 0};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = 2 * tid + k;
    if (e < p.E) n[k] = p.s.counts[e];
    if (e == p.E) n[k] = p.Is > 0 ? p.T : 0;
    m[k] = (n[k] + kTM - 1) / kTM;
  }
  int a = n[0] + n[1], b = m[0] + m[1];
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {  // inclusive warp scans
    const int ya = __shfl_up_sync(0xffffffffu, a, off), yb = __shfl_up_sync(0xffffffffu, b, off);
    if (lane >= off) {
      a += ya;
      b += yb;
    }
  }
  if (lane == 31) {
    wsum[warp] = a;
    wtil[warp] = b;
  }
  __syncthreads();
  if (warp == 0) {
    int x = wsum[lane], y = wtil[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int xa = __shfl_up_sync(0xffffffffu, x, off), yb = __shfl_up_sync(0xffffffffu, y, off);
      if (lane >= off) {
        x += xa;
        y += yb;
      }
    }
    wsum[lane] = x;
    wtil[lane] = y;
  }
  __syncthreads();
  int off_n = a - n[0] - n[1] + (warp ? wsum[warp - 1] : 0);
  int off_m = b - m[0] - m[1] + (warp ? wtil[warp - 1] : 0);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = 2 * tid + k;
    if (e < n_ent) {
      p.s.offsets[e] = off_n;
      for (int mt = 0; mt < m[k]; ++mt) p.s.jobs[off_m + mt] = (e << 20) | mt;
      p.s.cursor[e] = 0;
      if (e < p.E) p.s.counts[e] = 0;
    }
    if (e == n_ent - 1) {
      p.s.offsets[n_ent] = off_n + n[k];
      *p.s.n_jobs = off_m + m[k];
    }
    off_n += n[k];
    off_m += m[k];
  }
}

// One warp per token: each of its k routed rows (and its shared-expert row) takes a
// place in its expert's group, and the token's x row (hi and lo) is copied there.
__global__ void __launch_bounds__(kPT) prefill_scatter(const PrefillParams p) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kPT / 32) + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int nr = p.K + (p.Is > 0 ? 1 : 0);
  const int vec = p.H / 8;
  const uint4* src_hi = reinterpret_cast<const uint4*>(p.s.x_hi + (size_t)t * p.H);
  const uint4* src_lo = reinterpret_cast<const uint4*>(p.s.x_lo + (size_t)t * p.H);
  for (int r = 0; r < nr; ++r) {
    int pos = 0;
    if (lane == 0) {
      if (r < p.K) {
        const int e = p.s.sel[(size_t)t * p.K + r];
        pos = p.s.offsets[e] + atomicAdd(p.s.cursor + e, 1);
      } else {
        pos = p.s.offsets[p.E] + t;
      }
      p.s.gpos[(size_t)t * (p.K + 1) + r] = pos;
    }
    pos = __shfl_sync(0xffffffffu, pos, 0);
    uint4* dh = reinterpret_cast<uint4*>(p.s.xg_hi + (size_t)pos * p.H);
    uint4* dl = reinterpret_cast<uint4*>(p.s.xg_lo + (size_t)pos * p.H);
    for (int c = lane; c < vec; c += 32) {
      dh[c] = src_hi[c];
      dl[c] = src_lo[c];
    }
  }
}

// ------------------------------------------------------------------ tcgen05 grouped GEMM

__device__ __forceinline__ void pmbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32p(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool pmbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32p(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the layout a 64-column fp16 TMA box with 128-byte swizzle writes).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);  // start address / 16
  d |= (uint64_t)1 << 16;                  // leading byte offset (unused when swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset / 16
  d |= (uint64_t)1 << 46;                  // descriptor version of sm_100
  d |= (uint64_t)2 << 61;                  // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: f16 x f16 -> f32, A and B K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kTN >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}" ::"r"(tmem),
      "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Wait for this thread's tensor-memory loads.  The registers they fill pass through the
// wait as operands, so no copy of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// Bounded wait shared by the CTA's roles: false after about 2 s, or at once when another
// role already gave up (then the tile's result is garbage, the error word says so, and
// every role still runs to its end).
__device__ __forceinline__ bool pmbar_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (pmbar_try(bar, parity)) return true;
  uint64_t t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (!pmbar_try(bar, parity)) {
    if (*abort) return false;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > 2000000000ull) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void pmbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32p(bar)) : "memory");
}

// fp16 pair of Q4_0 weights (q - 8) * d from two nibbles at bits 0..3 and 16..19 of v:
// 0x6400 | q is the fp16 1024 + q, so subtracting 1032 leaves q - 8 exactly and the
// product with d is the correctly rounded fp16((q - 8) * d).
__device__ __forceinline__ uint32_t q4_pair(uint32_t v, __half2 d2) {
  const uint32_t m = (v & 0x000F000Fu) | 0x64006400u;
  const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&m), __half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408)));
  const __half2 w = __hmul2(q, d2);
  return *reinterpret_cast<const uint32_t*>(&w);
}

constexpr int kRawStages = 2;  // raw weight-byte ring depth (TMA, shared by the dequant warps)
// raw stage: [256 rows x 32 bytes of nibbles: two Q4_0 blocks of each row]
//            [256 rows x 16 bytes of scales: eight blocks of each row, i.e. four K stages]
constexpr uint32_t kRawNib = kTN * 32;
constexpr uint32_t kRawStage = kRawNib + kTN * 16;
constexpr uint32_t kRawRing = kRawStages * kRawStage;
constexpr int kGT = 512;           // threads of a GEMM CTA: 16 warps
constexpr int kAccCols = 2 * kTN;  // two accumulator buffers in tensor memory (all 512 columns)
constexpr int kTileCap = 64;       // tiles one GEMM CTA may take (its tile table's size)

// One output tile: 128 grouped rows of expert e (m-tile) x 256 columns (n-tile nt); nK == 0
// marks a tile with no work (past the width of a narrower shared expert).
struct GemmTile {
  int row0, nvalid, nK, nt, e, Ie;
  int slot;  // pool slot of a routed expert, layer of the shared one
  int pad;
};
static_assert(sizeof(GemmTile) == 32, "tile table entry");

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(m), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* m, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
      "%6}], [%7];" ::"r"(dst),
      "l"(m), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

// Tensor maps of one GEMM launch: the activation tiles and, for routed and shared
// experts, the weight tile's nibble and scale bytes read straight out of the slot layout.
struct GemmMaps {
  CUtensorMap a_hi, a_lo;
  CUtensorMap nib[2], scl[2];  // [0] routed experts (pool), [1] the shared expert
};

// Persistent grouped GEMM.  CTA b takes tiles b, b + grid, ... of the list (m-tile job,
// n-tile); two otherwise idle warps first resolve them into a table in shared memory so
// that no role waits on global loads at a tile boundary.  Warp roles, joined by mbarriers:
//   warps 0..3     epilogue: warp w owns tile rows 32 w .. 32 w + 31 (its tensor-memory
//                  lane quarter); it drains one accumulator buffer while the MMAs fill
//                  the other
//   warp 4 lane 0  A producer: TMA of the activation tiles (hi, lo) of each K stage
//   warp 5 lane 0  MMA issuer: 2 x 4 tcgen05.mma (128 x 256 x 16) per stage into the
//                  tile's buffer; commits free the stage and, after the last stage, hand
//                  the buffer over
//   warps 6, 7     the tile table; then warp 6 lane 0 is the raw producer: TMA of the
//                  weight tile's Q4_0 nibbles (two blocks of 256 rows) and scales per stage
//   warps 8..15    B producers: thread r owns row r of the weight tile; it dequantises its
//                  two blocks of each stage into the 128B-swizzled K-major fp16 tile
// A 256-wide weight tile halves the activation bytes the MMAs read from shared memory per
// FLOP against a 128-wide one: with both operands in shared memory, an M = 128, N = 128
// MMA alone asks for about the whole shared-memory bandwidth.  The raw bytes come by TMA
// because each row's 32 bytes of a stage lie in a different 1 KB-strided row of the slot:
// per-thread copies cost one cache line per thread.
template <int MODE>  // 0: gate/up + SwiGLU, 1: down
__global__ void __launch_bounds__(kGT, 1)
    prefill_gemm(const PrefillParams p, int l, const __grid_constant__ GemmMaps maps) {
  extern __shared__ __align__(1024) uint8_t psm_raw[];
  const int imax = p.I > p.Is ? p.I : p.Is;
  const int ntn = MODE == 0 ? (2 * imax) / kTN : p.H / kTN;
  const int total = *p.s.n_jobs * ntn;
  const int grid = gridDim.x;
  if ((int)blockIdx.x >= total) return;
  const int n_my = (total - (int)blockIdx.x + grid - 1) / grid;
  if (n_my > kTileCap) {  // the host sizes the token chunks so that this cannot happen
    if (threadIdx.x == 0) atomicCAS(p.s.error, 0, MOE_DEVERR_SLOT);
    return;
  }

  // [A_hi 16K | A_lo 16K | B 32K] x S from a 1024-byte boundary, raw ring, tile table, barriers
  uint8_t* psm = psm_raw + ((1024u - (smem_u32p(psm_raw) & 1023u)) & 1023u);
  uint8_t* raw = psm + kTilesBytes;
  GemmTile* tiles = reinterpret_cast<GemmTile*>(raw + kRawRing);
  uint64_t* full_a = reinterpret_cast<uint64_t*>(tiles + kTileCap);
  uint64_t* full_b = full_a + kStages;
  uint64_t* empty = full_b + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* raw_full = acc_empty + 2;
  uint64_t* raw_empty = raw_full + kRawStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(raw_empty + kRawStages);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto a_hi = [&](int s) { return psm + s * kStageBytes; };
  auto a_lo = [&](int s) { return psm + s * kStageBytes + kTileBytes; };
  auto b_t = [&](int s) { return psm + s * kStageBytes + 2 * kTileBytes; };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      pmbar_init(&full_a[s], 1);
      pmbar_init(&full_b[s], 8);
      pmbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      pmbar_init(&acc_full[b], 1);
      pmbar_init(&acc_empty[b], 4);
    }
    for (int s = 0; s < kRawStages; ++s) {
      pmbar_init(&raw_full[s], 1);
      pmbar_init(&raw_empty[s], 8);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32p(tmem_slot)),
                 "r"(kAccCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 6 || warp == 7) {
    for (int i = tid - 192; i < n_my; i += 64) {
      const int tile = (int)blockIdx.x + i * grid;
      const int je = p.s.jobs[tile / ntn];
      GemmTile t;
      t.nt = tile % ntn;
      t.e = je >> 20;
      const int mt = je & 0xFFFFF;
      t.Ie = t.e < p.E ? p.I : p.Is;
      const int g0 = p.s.offsets[t.e];
      const int n_e = p.s.offsets[t.e + 1] - g0;
      t.row0 = g0 + mt * kTM;
      t.nvalid = n_e - mt * kTM;
      t.nK = (MODE == 0 && t.nt * (kTN / 2) >= t.Ie) ? 0 : (MODE == 0 ? p.H : t.Ie) / kTK;
      t.slot = t.e < p.E ? p.layer_base[l] + (p.pin_slot[(size_t)l * p.E + t.e] & 0xffff) : l;
      t.pad = 0;
      tiles[i] = t;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ---------------------------------------------------------------- epilogue
    const int row = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int tc = 0;
    for (int i = 0; i < n_my; ++i) {
      const GemmTile t = tiles[i];
      if (t.nK == 0) continue;
      const int b = tc & 1;
      // the tensor-memory loads below are warp-collective: the whole warp goes on or stops
      const bool ok = __all_sync(0xffffffffu, pmbar_wait_ab(&acc_full[b], (uint32_t)(tc >> 1) & 1u, abort));
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t taddr = tmem + lane_base + (uint32_t)(b * kTN);
      const bool valid = row < t.nvalid;
      const int grow = t.row0 + row;
      if (MODE == 0) {  // gate columns 0..127, up columns 128..255
#pragma unroll 1
        for (int c0 = 0; c0 < kTN / 2; c0 += 16) {
          uint32_t gr[16], ur[16];
          tmem_ld16(taddr + c0, gr);
          tmem_ld16(taddr + kTN / 2 + c0, ur);
          tmem_wait16(gr);
          tmem_wait16(ur);
          if (valid) {
            __align__(16) __half hi[16];
            __align__(16) __half lo[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float gv = __uint_as_float(gr[j]), uv = __uint_as_float(ur[j]);
              const float a = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
              hi[j] = __float2half_rn(a);
              lo[j] = __float2half_rn(a - __half2float(hi[j]));
            }
            const size_t off = (size_t)grow * imax + t.nt * (kTN / 2) + c0;
            uint4* dh = reinterpret_cast<uint4*>(p.s.a_hi + off);
            uint4* dl = reinterpret_cast<uint4*>(p.s.a_lo + off);
            dh[0] = reinterpret_cast<const uint4*>(hi)[0];
            dh[1] = reinterpret_cast<const uint4*>(hi)[1];
            dl[0] = reinterpret_cast<const uint4*>(lo)[0];
            dl[1] = reinterpret_cast<const uint4*>(lo)[1];
          }
        }
      } else {  // expert outputs as [H / 16][R][16]: a warp's 32 rows x 16 columns are 2 KB in a row
#pragma unroll 1
        for (int c0 = 0; c0 < kTN; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(taddr + c0, o);
          tmem_wait16(o);
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(p.s.obuf + (((size_t)(t.nt * kTN + c0) / 16) * p.R + grow) * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_float4(__uint_as_float(o[4 * j]), __uint_as_float(o[4 * j + 1]),
                                  __uint_as_float(o[4 * j + 2]), __uint_as_float(o[4 * j + 3]));
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) pmbar_arrive(&acc_empty[b]);
      ++tc;
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------------- A producer
    if (lane == 0) {
      int it = 0;
      bool stop = false;
      for (int i = 0; i < n_my && !stop; ++i) {
        const GemmTile t = tiles[i];
        for (int ks = 0; ks < t.nK; ++ks, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !pmbar_wait_ab(&empty[s], (uint32_t)(it / kStages - 1) & 1u, abort)) {
            stop = true;
            break;
          }
          const uint32_t bar = smem_u32p(&full_a[s]);
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2 * kTileBytes)
                       : "memory");
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
              "[%4];" ::"r"(smem_u32p(a_hi(s))),
              "l"(&maps.a_hi), "r"(ks * kTK), "r"(t.row0), "r"(bar)
              : "memory");
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
              "[%4];" ::"r"(smem_u32p(a_lo(s))),
              "l"(&maps.a_lo), "r"(ks * kTK), "r"(t.row0), "r"(bar)
              : "memory");
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, tc = 0;
      bool stop = false;
      for (int i = 0; i < n_my && !stop; ++i) {
        const GemmTile t = tiles[i];
        if (t.nK == 0) continue;
        const int b = tc & 1;
        if (tc >= 2 && !pmbar_wait_ab(&acc_empty[b], (uint32_t)((tc >> 1) - 1) & 1u, abort)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t acc = tmem + (uint32_t)(b * kTN);
        for (int ks = 0; ks < t.nK; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!pmbar_wait_ab(&full_a[s], ph, abort) || !pmbar_wait_ab(&full_b[s], ph, abort)) {
            stop = true;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t sh = smem_u32p(a_hi(s)), sl = smem_u32p(a_lo(s)), sb = smem_u32p(b_t(s));
#pragma unroll
          for (int kk = 0; kk < kTK / 16; ++kk) {
            const uint64_t db = umma_desc(sb + kk * 32);
            umma_f16(acc, umma_desc(sh + kk * 32), db, (ks > 0 || kk > 0) ? 1u : 0u);
            umma_f16(acc, umma_desc(sl + kk * 32), db, 1u);
          }
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32p(&empty[s]))
                       : "memory");
        }
        if (stop) break;
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32p(&acc_full[b]))
                     : "memory");
        ++tc;
      }
    }
  } else if (warp == 6) {
    // ---------------------------------------------------------------- raw producer
    if (lane == 0) {
      int it = 0;
      bool stop = false;
      for (int i = 0; i < n_my && !stop; ++i) {
        const GemmTile t = tiles[i];
        const int sh = t.e < p.E ? 0 : 1;
        for (int ks = 0; ks < t.nK; ++ks, ++it) {
          const int rs = it % kRawStages;
          if (it >= kRawStages && !pmbar_wait_ab(&raw_empty[rs], (uint32_t)(it / kRawStages - 1) & 1u, abort)) {
            stop = true;
            break;
          }
          const uint32_t bar = smem_u32p(&raw_full[rs]);
          const uint32_t dq = smem_u32p(raw + rs * kRawStage), dd = dq + kRawNib;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kRawStage)
                       : "memory");
          if (MODE == 0) {  // 128 gate rows then the same 128 up rows: row blocks 4 nt .. 4 nt + 3
            for (int half = 0; half < 2; ++half) {
              tma_load_5d(dq + half * (kRawNib / 2), &maps.nib[sh], ks * 32, 0, 2 * half, 4 * t.nt, t.slot, bar);
              tma_load_5d(dd + half * (kTN / 2) * 16, &maps.scl[sh], (ks >> 2) * 16, 0, 2 * half, 4 * t.nt, t.slot,
                          bar);
            }
          } else {  // 256 down rows: 16-row tiles 16 nt .. 16 nt + 15
            tma_load_4d(dq, &maps.nib[sh], ks * 32, 0, 16 * t.nt, t.slot, bar);
            tma_load_4d(dd, &maps.scl[sh], (ks >> 2) * 16, 0, 16 * t.nt, t.slot, bar);
          }
        }
      }
    }
  } else if (warp >= 8) {
    // ---------------------------------------------------------------- B producers
    const int r = tid - 256;
    int it = 0;
    bool stop = false;
    for (int i = 0; i < n_my && !stop; ++i) {
      const int nK = tiles[i].nK;
      for (int ks = 0; ks < nK; ++ks, ++it) {
        const int rs = it % kRawStages;
        if (!pmbar_wait_ab(&raw_full[rs], (uint32_t)(it / kRawStages) & 1u, abort)) {
          stop = true;
          break;
        }
        const uint8_t* rq = raw + rs * kRawStage + r * 32;
        const uint4 q0 = *reinterpret_cast<const uint4*>(rq);
        const uint4 q1 = *reinterpret_cast<const uint4*>(rq + 16);
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(raw + rs * kRawStage + kRawNib + r * 16 + (ks & 3) * 4);
        const int s = it % kStages;
        if (it >= kStages && !pmbar_wait_ab(&empty[s], (uint32_t)(it / kStages - 1) & 1u, abort)) {
          stop = true;
          break;
        }
        uint8_t* brow = b_t(s) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const uint4 q = blk ? q1 : q0;
          const __half dh = __ushort_as_half((unsigned short)(blk ? (sc >> 16) : (sc & 0xFFFF)));
          const __half2 d2 = __half2(dh, dh);
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
          uint32_t lo[8], hi[8];  // half2 pairs of weights (2j, 2j + 1) and (16 + 2j, 17 + 2j)
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t r01 = __byte_perm(qw[w], 0, 0x4140), r23 = __byte_perm(qw[w], 0, 0x4342);
            lo[2 * w] = q4_pair(r01, d2);
            lo[2 * w + 1] = q4_pair(r23, d2);
            hi[2 * w] = q4_pair(r01 >> 4, d2);
            hi[2 * w + 1] = q4_pair(r23 >> 4, d2);
          }
          // 16-byte chunks of the block: weights 0-7, 8-15 (low nibbles), 16-23, 24-31 (high)
          const int c0 = blk * 4;
          *reinterpret_cast<uint4*>(brow + (((c0 + 0) ^ (r & 7)) * 16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint4*>(brow + (((c0 + 1) ^ (r & 7)) * 16)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
          *reinterpret_cast<uint4*>(brow + (((c0 + 2) ^ (r & 7)) * 16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(brow + (((c0 + 3) ^ (r & 7)) * 16)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        }
        // the fence also orders this warp's reads of the raw slot before the TMA that refills it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          pmbar_arrive(&full_b[s]);
          pmbar_arrive(&raw_empty[rs]);
        }
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *abort) atomicCAS(p.s.error, 0, MOE_DEVERR_TMA);
  if (warp == 5) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kAccCols));
  }
}

// ------------------------------------------------------------------ combine

// h[t] += sum_rank w * o_rank + o_shared in rank order (without the norm: h = that sum).
// Expert outputs are column-block-major over grouped rows ([H / 16][R][16]); the token's
// grouped positions come from the scatter.  Thread: 4 columns; the outputs of those
// columns are loaded 10 ranks at a time (streaming, read once) before they are summed.
constexpr int kCombineGroup = 10;
__global__ void __launch_bounds__(kPT) prefill_combine(const PrefillParams p, int l) {
  const int t = blockIdx.x;
  const float* w = p.s.w + (size_t)t * p.K;
  const int* gp = p.s.gpos + (size_t)t * (p.K + 1);
  const int nr = p.K + (p.Is > 0 ? 1 : 0);
  for (int j = threadIdx.x * 4; j < p.H; j += kPT * 4) {
    const float* col = p.s.obuf + (size_t)(j / 16) * p.R * 16 + (j & 15);
    float4 y = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int r0 = 0; r0 < nr; r0 += kCombineGroup) {
      float4 o[kCombineGroup];
#pragma unroll
      for (int i = 0; i < kCombineGroup; ++i)
        if (r0 + i < nr) o[i] = __ldcs(reinterpret_cast<const float4*>(col + (size_t)gp[r0 + i] * 16));
#pragma unroll
      for (int i = 0; i < kCombineGroup; ++i) {
        const int r = r0 + i;
        if (r < p.K) {
          const float wr = w[r];
          y.x = fmaf(wr, o[i].x, y.x);
          y.y = fmaf(wr, o[i].y, y.y);
          y.z = fmaf(wr, o[i].z, y.z);
          y.w = fmaf(wr, o[i].w, y.w);
        } else if (r == p.K && p.Is > 0) {  // the shared expert, unweighted, last
          y.x = __fadd_rn(y.x, o[i].x);
          y.y = __fadd_rn(y.y, o[i].y);
          y.z = __fadd_rn(y.z, o[i].z);
          y.w = __fadd_rn(y.w, o[i].w);
        }
      }
    }
    const size_t at = (size_t)t * p.H + j;
    float4 hn = y;
    if (p.use_norm) {
      const float4 h = *reinterpret_cast<const float4*>(p.s.h + at);
      hn = make_float4(__fadd_rn(h.x, y.x), __fadd_rn(h.y, y.y), __fadd_rn(h.z, y.z), __fadd_rn(h.w, y.w));
    }
    *reinterpret_cast<float4*>(p.s.h + at) = hn;
    if (p.s.h_trace)
      *reinterpret_cast<float4*>(p.s.h_trace + ((size_t)(l + 1) * p.T_total + p.t_base + t) * p.H + j) = hn;
    if (l == p.L - 1) *reinterpret_cast<float4*>(p.s.y + at) = hn;
  }
}

// ------------------------------------------------------------------ host side

static uint32_t gemm_smem() {
  return kTilesBytes + kRawRing + kTileCap * sizeof(GemmTile) + (3 * kStages + 4 + 2 * kRawStages) * 8 + 16 + 1024;
}
static int gemm_grid(int max_tiles, int n_sm) { return max_tiles < n_sm ? max_tiles : n_sm; }
static size_t route_floats(int tpc, int H, int E) { return (size_t)tpc * ((size_t)H / kChunk * kUChunk + E) + 16; }
static int route_tpc(int, int) { return 2 * kRTok; }  // small enough for two CTAs per SM at hidden 2048
static uint32_t route_smem(int H, int E) { return (uint32_t)(route_floats(route_tpc(H, E), H, E) * 4); }

int prefill_supported(int H, int E, int K, int I, int Is) {
  // 256-wide tiles; scale rows (K / 16 bytes) must be TMA strides, multiples of 16 bytes
  if (H % kTN || H > kMaxH || I % 256 || Is % 256 || E > kMaxE || K > 32) return 0;
  return route_smem(H, E) <= 227 * 1024;
}

cudaError_t prefill_configure(int H, int E) {
  cudaError_t e = cudaFuncSetAttribute(prefill_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_route, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)route_smem(H, E));
  return e;
}

typedef CUresult (*PfnEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Row-major fp16 [rows x cols] -> tensor map of 64-column x 128-row boxes, 128-byte swizzle.
static int make_map(PfnEncodeTiled enc, CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTK, (cuuint32_t)kTM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

// Byte tensor map over the slot layout (no swizzle): dims[0] is one row's bytes.
static int make_byte_map(PfnEncodeTiled enc, CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                         const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

// Nibble and scale maps of one weight kind.  Gate/up (MODE 0): a slot's tiles are
// (row block rb of I/32, subtile st of 4) at (4 rb + st) * 9H, each [16 rows x H/32 x 16 B]
// then [16 rows x H/32 x 2 B]; a box is 16 rows x 2 subtiles x 4 row blocks = 128 rows.
// Down (MODE 1): 16-row tiles c of H at down + c * 9I; a box is 16 rows x 16 tiles = 256 rows.
static int make_weight_maps(PfnEncodeTiled enc, int mode, const uint8_t* pool, uint64_t n_slots, uint64_t slot_bytes,
                            const SlotLayout& lay, int H, int I, CUtensorMap* nib, CUtensorMap* scl) {
  if (mode == 0) {
    const uint64_t nbk = H / 32, tile = 9ull * H;
    const cuuint64_t dq[5] = {nbk * 16, 16, 4, (cuuint64_t)I / 32, n_slots};
    const cuuint64_t sq[4] = {nbk * 16, tile, 4 * tile, slot_bytes};
    const cuuint32_t bq[5] = {32, 16, 2, 4, 1};
    const cuuint64_t dd[5] = {nbk * 2, 16, 4, (cuuint64_t)I / 32, n_slots};
    const cuuint64_t sd[4] = {nbk * 2, tile, 4 * tile, slot_bytes};
    const cuuint32_t bd[5] = {16, 16, 2, 4, 1};
    return make_byte_map(enc, nib, pool + lay.gu, 5, dq, sq, bq) ||
           make_byte_map(enc, scl, pool + lay.gu + 16 * nbk * 16, 5, dd, sd, bd);
  }
  const uint64_t nbk = I / 32, tile = 9ull * I;
  const cuuint64_t dq[4] = {nbk * 16, 16, (cuuint64_t)H / 16, n_slots};
  const cuuint64_t sq[3] = {nbk * 16, tile, slot_bytes};
  const cuuint32_t bq[4] = {32, 16, 16, 1};
  const cuuint64_t dd[4] = {nbk * 2, 16, (cuuint64_t)H / 16, n_slots};
  const cuuint64_t sd[3] = {nbk * 2, tile, slot_bytes};
  const cuuint32_t bd[4] = {16, 16, 16, 1};
  return make_byte_map(enc, nib, pool + lay.down, 4, dq, sq, bq) ||
         make_byte_map(enc, scl, pool + lay.down + 16 * nbk * 16, 4, dd, sd, bd);
}

// Tokens per pass: every GEMM CTA's tiles must fit its tile table.
static int prefill_chunk(int T, int H, int E, int K, int I, int Is, int grid) {
  const int imax = I > Is ? I : Is;
  const int64_t ntn = (2 * imax) / kTN > H / kTN ? (2 * imax) / kTN : H / kTN;
  int tc = T;
  while (tc > 1) {
    const int64_t R = (int64_t)tc * K + (Is > 0 ? tc : 0);
    const int64_t max_tiles = ((R + kTM - 1) / kTM + E + 1) * ntn;
    if ((max_tiles + grid - 1) / grid <= kTileCap) break;
    tc = (tc + 1) / 2;
  }
  return tc;
}

int prefill_run(const PrefillArgs& a, const PrefillScratch& s, void* encode_fn, cudaStream_t st) {
  const int T = a.T, H = a.H, E = a.E;
  const int imax = a.I > a.Is ? a.I : a.Is;
  const int grid0 = gemm_grid(1 << 30, a.n_sm);
  const int tcmax = prefill_chunk(T, H, E, a.K, a.I, a.Is, grid0);
  if ((((int64_t)E + 2) * ((2 * imax) / kTN > H / kTN ? (2 * imax) / kTN : H / kTN) + grid0 - 1) / grid0 > kTileCap)
    return -1;  // even one token per pass would overflow a tile table
  PfnEncodeTiled enc = reinterpret_cast<PfnEncodeTiled>(encode_fn);
  if (s.h_trace) {
    cudaError_t e = cudaMemcpyAsync(s.h_trace, s.h, sizeof(float) * T * H, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return (int)e;
  }
  for (int t0 = 0; t0 < T; t0 += tcmax) {
    const int Tc = T - t0 < tcmax ? T - t0 : tcmax;
    PrefillParams p{};
    p.L = a.L;
    p.H = H;
    p.E = E;
    p.K = a.K;
    p.I = a.I;
    p.Is = a.Is;
    p.use_norm = a.use_norm;
    p.T = Tc;
    p.t_base = t0;
    p.T_total = T;
    p.eps = a.eps;
    p.nch = H / kChunk;
    p.tpc = route_tpc(H, E);
    p.pool = a.pool;
    p.slot_bytes = a.slot_bytes;
    p.lay = a.lay;
    p.slay = a.slay;
    p.shared_pool = a.shared_pool;
    p.shared_slot_bytes = a.shared_slot_bytes;
    p.router = a.router;
    p.bias = a.bias;
    p.gain = a.gain;
    p.pin_slot = a.pin_slot;
    p.layer_base = a.layer_base;
    p.hist = a.hist;
    p.s = s;
    p.s.h = s.h + (size_t)t0 * H;
    p.s.y = s.y + (size_t)t0 * H;
    const int R = Tc * a.K + (a.Is > 0 ? Tc : 0);
    p.R = R;
    GemmMaps m0, m1;  // gate/up, down
    if (make_map(enc, &m0.a_hi, s.xg_hi, R, H) || make_map(enc, &m0.a_lo, s.xg_lo, R, H) ||
        make_map(enc, &m1.a_hi, s.a_hi, R, imax) || make_map(enc, &m1.a_lo, s.a_lo, R, imax))
      return -1;
    for (int mode = 0; mode < 2; ++mode) {
      GemmMaps& g = mode == 0 ? m0 : m1;
      if (make_weight_maps(enc, mode, a.pool, (uint64_t)a.pool_slots, a.slot_bytes, a.lay, H, a.I, &g.nib[0],
                           &g.scl[0]))
        return -1;
      if (a.Is > 0) {
        if (make_weight_maps(enc, mode, a.shared_pool, (uint64_t)a.L, a.shared_slot_bytes, a.slay, H, a.Is, &g.nib[1],
                             &g.scl[1]))
          return -1;
      } else {
        g.nib[1] = g.nib[0];
        g.scl[1] = g.scl[0];
      }
    }
    const int max_jobs = (R + kTM - 1) / kTM + E + 1;
    cudaError_t e = cudaMemsetAsync(s.counts, 0, sizeof(int32_t) * E, st);
    if (e != cudaSuccess) return (int)e;
    for (int l = 0; l < a.L; ++l) {
      prefill_route<<<(Tc + p.tpc - 1) / p.tpc, kPT, route_smem(H, E), st>>>(p, l);
      prefill_scan<<<1, 1024, 0, st>>>(p);
      prefill_scatter<<<(Tc + kPT / 32 - 1) / (kPT / 32), kPT, 0, st>>>(p);
      prefill_gemm<0><<<gemm_grid(max_jobs * ((2 * imax) / kTN), a.n_sm), kGT, gemm_smem(), st>>>(p, l, m0);
      prefill_gemm<1><<<gemm_grid(max_jobs * (H / kTN), a.n_sm), kGT, gemm_smem(), st>>>(p, l, m1);
      prefill_combine<<<Tc, kPT, 0, st>>>(p, l);
      e = cudaGetLastError();
      if (e != cudaSuccess) return (int)e;
    }
  }
  return 0;
}

}  // namespace moe
