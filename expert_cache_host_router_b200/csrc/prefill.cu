// prefill.cu -- batched prefill of T tokens through the MoE stack (every expert resident)
// for libmoe: each token's top-k in the same canonical fp32 order as decode, tokens
// grouped by expert, and the expert FFNs as a grouped GEMM on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, operands brought in by TMA).
//
// The write-up serves decode; a prompt's tokens all pass the same layers at once, which
// turns each expert's GEMVs into GEMMs [n_e x H] x [H x 2I] and [n_e x I] x [I x H]
// (n_e = tokens routed to expert e): a dense contraction, so it runs on the tensor
// cores.  Per layer, in stream order:
//   route    RMSNorm scale and x = RMSNorm(h) split into fp16 hi + lo (x = hi + lo to
//            about 2^-22 relative); router logits approximated on the tensor cores, the
//            top-k certified with exact canonical-order logits of the candidates (see the
//            certified-router section); weights, histogram, per-expert counts
//   scan     expert offsets and the list of 128-row m-tiles
//   scatter  one warp per token: its rows of x copied to their place in expert order
//            (within an expert the order is whatever the atomics give: a GEMM row does
//            not depend on the other rows of its tile, so results are deterministic)
//   gemm     persistent, one CTA per SM, 128 x 256 output tiles: A (activation rows, fp16
//            hi and lo) and the raw Q4_0 weight bytes by TMA, the weights dequantised to
//            fp16 into 128B-swizzled shared memory, two tcgen05.mma per 16-wide K step
//            (A_hi B and A_lo B) into one fp32 accumulator in tensor memory; gate/up tiles
//            hold 128 gate and the matching 128 up columns so the epilogue forms
//            a = silu(g) * u (stored as fp16 hi + lo); down tiles write fp32 outputs
//            column-block-major over grouped rows
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
  int L, H, E, K, I, Is, use_norm, T, nch;
  int t_base, T_total;  // this chunk's first token and the call's token count (trace rows)
  int R;                // grouped rows of this chunk: T * k (+ T with a shared expert)
  float eps;
  const float* bias;          // [L][E] or null
  const float* gain;          // [L][H]
  const int32_t* pin_slot;    // [L][E]: pool slot of expert e at layer l is base[l] + (entry & 0xffff)
  const int32_t* layer_base;  // [L]
  uint32_t* hist;
  const float* wnorm;  // [L] max_e ||w_e||_2 of the router rows, rounded up
  const uint16_t* router_rows;  // [L][E][H] bf16
  PrefillScratch s;
};

__device__ __forceinline__ uint32_t smem_u32p(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ float bf16_lo_p(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_p(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }


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
// place in its expert's group, and the token's x row (hi and lo) is copied there; each
// 2048-column piece of the row is read once and stored k + 1 times.
constexpr int kScatterRegs = 8;  // 16-byte pieces per lane and array: 2048 columns per pass
__global__ void __launch_bounds__(kPT) prefill_scatter(const PrefillParams p) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kPT / 32) + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int nr = p.K + (p.Is > 0 ? 1 : 0);
  int32_t* gp = p.s.gpos + (size_t)t * (p.K + 1);
  if (lane == 0)
    for (int r = 0; r < nr; ++r) {
      if (r < p.K) {
        const int e = p.s.sel[(size_t)t * p.K + r];
        gp[r] = p.s.offsets[e] + atomicAdd(p.s.cursor + e, 1);
      } else {
        gp[r] = p.s.offsets[p.E] + t;
      }
    }
  __syncwarp();
  const int vec = p.H / 8;  // 16-byte pieces per row
  const uint4* src_hi = reinterpret_cast<const uint4*>(p.s.x_hi + (size_t)t * p.H);
  const uint4* src_lo = reinterpret_cast<const uint4*>(p.s.x_lo + (size_t)t * p.H);
  for (int base = 0; base < vec; base += 32 * kScatterRegs) {
    uint4 rh[kScatterRegs], rl[kScatterRegs];
#pragma unroll
    for (int i = 0; i < kScatterRegs; ++i) {
      const int c = base + lane + 32 * i;
      if (c < vec) {
        rh[i] = src_hi[c];
        rl[i] = src_lo[c];
      }
    }
    for (int r = 0; r < nr; ++r) {
      const size_t pos = (size_t)gp[r];
      uint4* dh = reinterpret_cast<uint4*>(p.s.xg_hi + pos * p.H);
      uint4* dl = reinterpret_cast<uint4*>(p.s.xg_lo + pos * p.H);
#pragma unroll
      for (int i = 0; i < kScatterRegs; ++i) {
        const int c = base + lane + 32 * i;
        if (c < vec) {
          dh[c] = rh[i];
          dl[c] = rl[i];
        }
      }
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
          } else {  // 256 down rows 256 nt..: blocks 2 ks, 2 ks + 1 (units), scales of 8 units
            tma_load_4d(dq, &maps.nib[sh], 0, 16 * t.nt, 2 * ks, t.slot, bar);
            tma_load_4d(dd, &maps.scl[sh], 0, 2 * t.nt, 8 * (ks >> 2), t.slot, bar);
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
        // row r's two Q4_0 blocks of this K stage and their fp16 scales (low, high half)
        uint4 q0, q1;
        uint32_t sc;
        if (MODE == 0) {  // [row][2 blocks x 16 B]; scales [row][8 blocks x 2 B]
          const uint8_t* rq = raw + rs * kRawStage + r * 32;
          q0 = *reinterpret_cast<const uint4*>(rq);
          q1 = *reinterpret_cast<const uint4*>(rq + 16);
          sc = *reinterpret_cast<const uint32_t*>(raw + rs * kRawStage + kRawNib + r * 16 + (ks & 3) * 4);
        } else {  // [2 blocks][row][16 B]; scales [8 blocks][row][2 B]
          const uint8_t* rq = raw + rs * kRawStage + r * 16;
          q0 = *reinterpret_cast<const uint4*>(rq);
          q1 = *reinterpret_cast<const uint4*>(rq + kTN * 16);
          const uint8_t* rd = raw + rs * kRawStage + kRawNib + (ks & 3) * 2 * (kTN * 2) + r * 2;
          sc = (uint32_t)*reinterpret_cast<const uint16_t*>(rd) |
               ((uint32_t)*reinterpret_cast<const uint16_t*>(rd + kTN * 2) << 16);
        }
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

// ------------------------------------------------------------------ certified router
//
// The canonical-order logits above cost H x E fp32 FMAs per token on CUDA cores.  The
// routing decision only needs them for the experts that can make the top-k, so:
//   prep    u = g * h (fp32) split exactly into three bf16 parts (u = u0 + u1 + u2), plus
//           inv, ||u||_2 and x hi/lo
//   gemm    approximate S~ = sum_p u_p . w_e on the tensor cores (bf16 x bf16, products exact
//           in fp32, fp32 accumulation), split over K, partials summed in a fixed order
//   select  per token: with delta = 2^-9 * ||u|| * max_e ||w_e|| * inv, twice a bound on
//           |z~ - z| (the accumulation error of S~ is at most 2^-10 * sum_j |w_j u_j| <=
//           2^-10 ||u|| ||w_e||, Cauchy-Schwarz), every expert whose approximate logit is
//           within 2 delta of the k-th largest (or above it) is a candidate; the rest have
//           exact logits strictly below the k-th exact one.  The candidates are evaluated
//           exactly in the canonical order and the top-k among them is the answer.
// Every selection is therefore the canonical one, bit for bit.
constexpr int kRParts = 3;   // bf16 parts of u
constexpr int kRSplit = 8;   // K splits of the router GEMM
constexpr int kRGT = 192;    // router GEMM threads: 6 warps
constexpr int kRStages = 4;

// Warp per token: inv (canonical fold of the squares), u and its three bf16 parts, ||u||,
// and x = RMSNorm(h) as fp16 hi + lo; four consecutive columns per lane.
__global__ void __launch_bounds__(kPT) prefill_route_prep(const PrefillParams p, int l) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kPT / 32) + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int H = p.H, nch = p.nch;
  const float* hrow = p.s.h + (size_t)t * H;
  const float* g = p.gain + (size_t)l * H;
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
  float uu = 0.0f;
  float* urow = p.s.u + (size_t)t * H;
  __nv_bfloat16* ua = p.s.ua + (size_t)t * kRParts * H;
  for (int j = lane * 4; j < H; j += 128) {
    const float4 h4 = *reinterpret_cast<const float4*>(hrow + j);
    const float hv[4] = {h4.x, h4.y, h4.z, h4.w};
    float4 g4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
    if (p.use_norm) g4 = *reinterpret_cast<const float4*>(g + j);
    const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
    float u[4];
    __nv_bfloat16 b0[4], b1[4], b2[4];
    __half xh[4], xl[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[i] = p.use_norm ? __fmul_rn(gv[i], hv[i]) : hv[i];
      const float xv = p.use_norm ? __fmul_rn(__fmul_rn(hv[i], inv), gv[i]) : hv[i];
      b0[i] = __float2bfloat16_rn(u[i]);
      const float r1 = u[i] - __bfloat162float(b0[i]);
      b1[i] = __float2bfloat16_rn(r1);
      b2[i] = __float2bfloat16_rn(r1 - __bfloat162float(b1[i]));
      uu = fmaf(u[i], u[i], uu);
      xh[i] = __float2half_rn(xv);
      xl[i] = __float2half_rn(xv - __half2float(xh[i]));
    }
    *reinterpret_cast<float4*>(urow + j) = make_float4(u[0], u[1], u[2], u[3]);
    *reinterpret_cast<uint2*>(ua + j) = *reinterpret_cast<const uint2*>(b0);
    *reinterpret_cast<uint2*>(ua + H + j) = *reinterpret_cast<const uint2*>(b1);
    *reinterpret_cast<uint2*>(ua + 2 * H + j) = *reinterpret_cast<const uint2*>(b2);
    *reinterpret_cast<uint2*>(p.s.x_hi + (size_t)t * H + j) = *reinterpret_cast<const uint2*>(xh);
    *reinterpret_cast<uint2*>(p.s.x_lo + (size_t)t * H + j) = *reinterpret_cast<const uint2*>(xl);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) uu += __shfl_xor_sync(0xffffffffu, uu, off);
  if (lane == 0) {
    p.s.inv[t] = inv;
    // fp32 sum of H squares: relative error below H * 2^-23; 1e-3 covers it for H <= 4096
    p.s.unorm[t] = __fsqrt_ru(uu * 1.001f);
  }
}

// Approximate router logits before the norm scale: part[split][t][e] = sum over the
// split's K range of [u0|u1|u2] . [w|w|w].  CTA = 128 tokens x N experts x one K split;
// warp 0 lane 0 TMA, warp 1 lane 0 MMA (tensor memory allocated by warp 1), warps 2..5
// the epilogue (one tensor-memory lane quarter each).
__global__ void __launch_bounds__(kRGT, 1)
    prefill_router_gemm(const PrefillParams p, const __grid_constant__ CUtensorMap ma,
                        const __grid_constant__ CUtensorMap mb, int N, int kst_per_split) {
  extern __shared__ __align__(1024) uint8_t rsm_raw[];
  const int m0 = blockIdx.x * kTM, n0 = blockIdx.y * N, split = blockIdx.z;
  const int total_k = kRParts * p.H / kTK;
  const int k0 = split * kst_per_split;
  const int nK = (k0 + kst_per_split < total_k ? k0 + kst_per_split : total_k) - k0;
  if (nK <= 0) return;
  const uint32_t a_bytes = kTM * kTK * 2, b_bytes = (uint32_t)N * kTK * 2;
  const uint32_t stage = a_bytes + ((b_bytes + 1023) & ~1023u);
  uint8_t* sm = rsm_raw + ((1024u - (smem_u32p(rsm_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kRStages * stage);
  uint64_t* empty = full + kRStages;
  uint64_t* done = empty + kRStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ncols = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  if (tid == 0) {
    for (int s = 0; s < kRStages; ++s) {
      pmbar_init(&full[s], 1);
      pmbar_init(&empty[s], 1);
    }
    pmbar_init(done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32p(tmem_slot)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  // bf16 x bf16 -> f32, K-major A and B, M = 128, N
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < nK; ++i) {
      const int s = i % kRStages, ks = k0 + i;
      if (i >= kRStages && !pmbar_wait_ab(&empty[s], (uint32_t)(i / kRStages - 1) & 1u, abort)) break;
      const uint32_t bar = smem_u32p(&full[s]);
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(a_bytes + b_bytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
          "[%4];" ::"r"(smem_u32p(sm + s * stage)),
          "l"(&ma), "r"(ks * kTK), "r"(m0), "r"(bar)
          : "memory");
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
          "[%4];" ::"r"(smem_u32p(sm + s * stage + a_bytes)),
          "l"(&mb), "r"((ks * kTK) % p.H), "r"(n0), "r"(bar)
          : "memory");
    }
  } else if (warp == 1 && lane == 0) {
    for (int i = 0; i < nK; ++i) {
      const int s = i % kRStages;
      if (!pmbar_wait_ab(&full[s], (uint32_t)(i / kRStages) & 1u, abort)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = smem_u32p(sm + s * stage), sb = sa + a_bytes;
#pragma unroll
      for (int kk = 0; kk < kTK / 16; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q;\n\t}" ::"r"(tmem),
            "l"(umma_desc(sa + kk * 32)), "l"(umma_desc(sb + kk * 32)), "r"(idesc), "r"(acc)
            : "memory");
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32p(&empty[s]))
                   : "memory");
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32p(done))
                 : "memory");
  } else if (warp >= 2) {
    const int q = warp & 3;  // tensor-memory lane quarter of this warp
    const bool ok = __all_sync(0xffffffffu, pmbar_wait_ab(done, 0, abort));
    if (ok) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int t = m0 + q * 32 + lane;
      float* dst = p.s.part + ((size_t)split * p.T + t) * p.E + n0;
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t o[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + c0, o);
        tmem_wait16(o);
        if (t < p.T) {
          if (n0 + c0 + 16 <= p.E) {
            float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_float4(__uint_as_float(o[4 * j]), __uint_as_float(o[4 * j + 1]),
                                  __uint_as_float(o[4 * j + 2]), __uint_as_float(o[4 * j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n0 + c0 + j < p.E) dst[c0 + j] = __uint_as_float(o[j]);
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *abort) atomicCAS(p.s.error, 0, MOE_DEVERR_TMA);
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
  }
}

// Canonical logits of nc experts (cand[0..nc)) for the token whose u the lanes read; lane
// = fold lane: each lane sums its chunks of every candidate (all loads in flight at once),
// then one butterfly per candidate.  zx[cand[i]] receives the logit.
constexpr int kCandBatch = 16;
__device__ __forceinline__ void canonical_logits(const PrefillParams& p, int l, const float* urow,
                                                 const uint32_t* cand, int nc, float inv, float* zx, int lane) {
  for (int i0 = 0; i0 < nc; i0 += kCandBatch) {
    float acc[kCandBatch];
#pragma unroll
    for (int i = 0; i < kCandBatch; ++i) acc[i] = 0.0f;
    for (int c = lane; c < p.nch; c += 32) {
      const float4* up = reinterpret_cast<const float4*>(urow + c * kChunk);
      const float4 ua = up[0], ub = up[1], uc = up[2], ud = up[3];
#pragma unroll
      for (int i = 0; i < kCandBatch; ++i) {
        if (i0 + i < nc) {
          const int e = (int)cand[i0 + i];
          // plain-row copy: a warp's 32 chunks of one expert are 1 KB in a row
          const uint4* wp = reinterpret_cast<const uint4*>(p.router_rows + ((size_t)l * p.E + e) * p.H + c * kChunk);
          const uint4 w0 = __ldg(wp), w1 = __ldg(wp + 1);
          float pc = 0.0f;
          pc = fmaf(bf16_lo_p(w0.x), ua.x, pc);
          pc = fmaf(bf16_hi_p(w0.x), ua.y, pc);
          pc = fmaf(bf16_lo_p(w0.y), ua.z, pc);
          pc = fmaf(bf16_hi_p(w0.y), ua.w, pc);
          pc = fmaf(bf16_lo_p(w0.z), ub.x, pc);
          pc = fmaf(bf16_hi_p(w0.z), ub.y, pc);
          pc = fmaf(bf16_lo_p(w0.w), ub.z, pc);
          pc = fmaf(bf16_hi_p(w0.w), ub.w, pc);
          pc = fmaf(bf16_lo_p(w1.x), uc.x, pc);
          pc = fmaf(bf16_hi_p(w1.x), uc.y, pc);
          pc = fmaf(bf16_lo_p(w1.y), uc.z, pc);
          pc = fmaf(bf16_hi_p(w1.y), uc.w, pc);
          pc = fmaf(bf16_lo_p(w1.z), ud.x, pc);
          pc = fmaf(bf16_hi_p(w1.z), ud.y, pc);
          pc = fmaf(bf16_lo_p(w1.w), ud.z, pc);
          pc = fmaf(bf16_hi_p(w1.w), ud.w, pc);
          acc[i] = __fadd_rn(acc[i], pc);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kCandBatch; ++i) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc[i] = __fadd_rn(acc[i], __shfl_xor_sync(0xffffffffu, acc[i], off));
    }
#pragma unroll
    for (int i = 0; i < kCandBatch; ++i)
      if (lane == i && i0 + i < nc) {
        const int e = (int)cand[i0 + i];
        zx[e] = fmaf(acc[i], inv, p.bias ? __ldg(p.bias + (size_t)l * p.E + e) : 0.0f);
      }
  }
}

// Order key of a logit: larger first, equal -> lower expert index, -0 == +0, NaN last.
__device__ __forceinline__ uint64_t logit_key(float v, int e) {
  if (v == 0.0f) v = 0.0f;
  const uint32_t uu = __float_as_uint(v);
  uint32_t o = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
  if (v != v) o = 0;
  return ((uint64_t)o << 32) | (uint32_t)(~(uint32_t)e);
}
__device__ __forceinline__ uint64_t warp_max_key(uint64_t k) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)k, off);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(k >> 32), off);
    const uint64_t o = ((uint64_t)hi << 32) | lo;
    k = o > k ? o : k;
  }
  return k;
}

// Warp per token: approximate logits, exact candidates, certified top-k, weights, counts.
// Shared memory per warp: approximate logits [E], exact logits [E], candidate list [E],
// flags [E] (1 = candidate, 2 = selected).
__global__ void __launch_bounds__(kPT) prefill_route_select(const PrefillParams p, int l, int nsplit) {
  extern __shared__ __align__(16) float ssm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (kPT / 32) + warp;
  if (t >= p.T) return;
  const int E = p.E, K = p.K;
  float* za = ssm + (size_t)warp * 3 * E;
  float* zx = za + E;
  uint32_t* cand = reinterpret_cast<uint32_t*>(zx + E);
  uint8_t* flag = reinterpret_cast<uint8_t*>(ssm + (size_t)(kPT / 32) * 3 * E) + (size_t)warp * E;
  const float inv = p.s.inv[t];
  const float* urow = p.s.u + (size_t)t * p.H;
  for (int e = lane; e < E; e += 32) {
    float v[kRSplit];  // the split partials are independent loads, summed in split order
#pragma unroll
    for (int sp = 0; sp < kRSplit; ++sp) v[sp] = sp < nsplit ? p.s.part[((size_t)sp * p.T + t) * E + e] : 0.0f;
    float S = 0.0f;
#pragma unroll
    for (int sp = 0; sp < kRSplit; ++sp) S += v[sp];
    za[e] = fmaf(S, inv, p.bias ? __ldg(p.bias + (size_t)l * E + e) : 0.0f);
    flag[e] = 0;
  }
  __syncwarp();
  const float delta = 0x1p-9f * p.s.unorm[t] * p.wnorm[l] * inv * 1.001f + 1e-30f;
  // best approximate logit among experts that are not candidates yet
  auto best_left = [&]() {
    uint64_t best = 0;
    for (int e = lane; e < E; e += 32)
      if (flag[e] == 0) {
        const uint64_t k = logit_key(za[e], e);
        best = k > best ? k : best;
      }
    return warp_max_key(best);
  };
  // 1. the k-th largest approximate logit.  Fast path (at most 256 experts, no NaN): its
  //    value by k rounds of warp max over orderable 32-bit keys, each round taking out
  //    one instance of the maximum, so equal logits count once each; every expert at or
  //    above it is a candidate below anyway.  Otherwise k rounds over (logit, index) keys.
  float zk_approx = 0.0f;
  bool nan = false;
  for (int e = lane; e < E; e += 32) nan |= za[e] != za[e];
  const bool fast = E <= 256 && !__any_sync(0xffffffffu, nan);
  if (fast) {
    uint32_t ord[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = lane + 32 * k;
      ord[k] = e < E ? (uint32_t)(logit_key(za[e], e) >> 32) : 0u;
    }
    uint32_t gv = 0;
    for (int r = 0; r < K; ++r) {
      uint32_t lv = ord[0];
#pragma unroll
      for (int k = 1; k < 8; ++k) lv = max(lv, ord[k]);
      gv = __reduce_max_sync(0xffffffffu, lv);
      const unsigned holders = __ballot_sync(0xffffffffu, lv == gv);
      if (lane == __ffs(holders) - 1) {
        bool done = false;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (!done && ord[k] == gv) {
            ord[k] = 0u;
            done = true;
          }
      }
    }
    zk_approx = __uint_as_float((gv & 0x80000000u) ? (gv & 0x7FFFFFFFu) : ~gv);
  } else {
    for (int r = 0; r < K; ++r) {
      const int e = (int)(~(uint32_t)best_left());
      zk_approx = za[e];
      if (lane == 0) flag[e] = 1;
      __syncwarp();
    }
  }
  // 2. candidates: the k best approximate logits and every expert within 2 delta below
  //    the k-th.  An expert outside has z~ < z~(k) - 2 delta, so its exact logit is below
  //    z~(k) - delta, which the k-th exact logit is not: the exact top-k is inside.
  const float thr = zk_approx - 2.0f * delta;
  int nc = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const bool in = e < E && (flag[e] == 1 || za[e] >= thr);
    const unsigned b = __ballot_sync(0xffffffffu, in);
    if (in) {
      cand[nc + __popc(b & ((1u << lane) - 1u))] = (uint32_t)e;
      flag[e] = 1;
    }
    nc += __popc(b);
  }
  __syncwarp();
  canonical_logits(p, l, urow, cand, nc, inv, zx, lane);
  __syncwarp();
  // 3. top-k of the candidates by exact logit; lane r keeps rank r.  Up to 32 candidates:
  //    each lane ranks its own against all of them (shuffles); else k rounds of warp max.
  int sel_e = -1;
  float sel_z = 0.0f;
  if (nc <= 32) {
    const int ce = lane < nc ? (int)cand[lane] : 0;
    const uint64_t mk = lane < nc ? logit_key(zx[ce], ce) : 0ull;
    int rank = 0;
    for (int i = 0; i < nc; ++i) {
      const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)mk, i);
      const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(mk >> 32), i);
      rank += (((uint64_t)hi << 32) | lo) > mk;
    }
    int* rsel = reinterpret_cast<int*>(za);  // the approximate logits are no longer read
    __syncwarp();
    if (lane < nc && rank < K) rsel[rank] = ce;
    __syncwarp();
    if (lane < K) {
      sel_e = rsel[lane];
      sel_z = zx[sel_e];
    }
    __syncwarp();
  } else {
  for (int r = 0; r < K; ++r) {
    uint64_t best = 0;
    for (int i = lane; i < nc; i += 32) {
      const int e = (int)cand[i];
      if (flag[e] == 1) {
        const uint64_t k = logit_key(zx[e], e);
        best = k > best ? k : best;
      }
    }
    best = warp_max_key(best);
    const int e = (int)(~(uint32_t)best);
    if (lane == r) {
      sel_e = e;
      sel_z = zx[e];
    }
    __syncwarp();
    if (lane == 0) flag[e] = 2;
    __syncwarp();
  }
  }
  if ((logit_key(__shfl_sync(0xffffffffu, sel_z, 0), 0) >> 32) == 0 && lane == 0)
    atomicCAS(p.s.error, 0, MOE_DEVERR_ROUTE);  // a NaN logit won
  const float zmax = __shfl_sync(0xffffffffu, sel_z, 0);
  const float ex = lane < K ? expf(sel_z - zmax) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < K) {
    p.s.sel[(size_t)t * K + lane] = sel_e;
    p.s.w[(size_t)t * K + lane] = __fdividef(ex, sum);
    atomicAdd(p.hist + (size_t)l * E + sel_e, 1u);
    atomicAdd(p.s.counts + sel_e, 1);
    if (p.s.sel_trace) p.s.sel_trace[((size_t)l * p.T_total + p.t_base + t) * K + lane] = sel_e;
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

static int router_n(int E) { return E <= 256 ? E : 256; }
static uint32_t router_gemm_smem(int E) {
  const uint32_t b = ((uint32_t)router_n(E) * kTK * 2 + 1023) & ~1023u;
  return kRStages * (kTM * kTK * 2 + b) + (2 * kRStages + 1) * 8 + 16 + 1024;
}
static uint32_t route_select_smem(int E) { return (uint32_t)(kPT / 32) * 13u * E; }

int prefill_supported(int H, int E, int K, int I, int Is) {
  if (E % 16) return 0;  // router GEMM: N = E (or 256) is a multiple of 16
  // 256-wide tiles; scale rows (K / 16 bytes) must be TMA strides, multiples of 16 bytes
  if (H % kTN || H > kMaxH || I % 256 || Is % 256 || E > kMaxE || K > 32) return 0;
  return route_select_smem(E) <= 227 * 1024 && router_gemm_smem(E) <= 227 * 1024;
}

cudaError_t prefill_configure(int, int E) {
  cudaError_t e = cudaFuncSetAttribute(prefill_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_router_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)router_gemm_smem(E));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_route_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)route_select_smem(E));
  return e;
}

typedef CUresult (*PfnEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Row-major 16-bit [rows x cols] -> tensor map of 64-column x box_rows boxes, 128-byte swizzle.
static int make_map(PfnEncodeTiled enc, CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_FLOAT16, uint32_t box_rows = kTM) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

// Nibble and scale maps of one weight kind over the unit layout of moe_internal.h (unit
// rb of a slot at rb * unit).  Gate/up (MODE 0): tiles (rb, subtile st of 4) at
// rb * unit + st * 9H, each [16 rows x H/32 x 16 B] then [16 rows x H/32 x 2 B]; a box
// is 16 rows x 2 subtiles x 4 units = 128 rows, 2 blocks (nibbles) or 8 blocks (scales)
// wide.  Down (MODE 1): unit rb holds block rb of every row j, nibbles at 36H + 16 j and
// scales at 52H + 2 j; a nibble box is 256 rows x 2 units, a scale box 256 rows x 8 units.
static int make_weight_maps(PfnEncodeTiled enc, int mode, const uint8_t* pool, uint64_t n_slots, uint64_t slot_bytes,
                            const SlotLayout& lay, int H, int I, CUtensorMap* nib, CUtensorMap* scl) {
  if (mode == 0) {
    const uint64_t nbk = H / 32, tile = 9ull * H;
    const cuuint64_t dq[5] = {nbk * 16, 16, 4, (cuuint64_t)I / 32, n_slots};
    const cuuint64_t sq[4] = {nbk * 16, tile, lay.unit, slot_bytes};
    const cuuint32_t bq[5] = {32, 16, 2, 4, 1};
    const cuuint64_t dd[5] = {nbk * 2, 16, 4, (cuuint64_t)I / 32, n_slots};
    const cuuint64_t sd[4] = {nbk * 2, tile, lay.unit, slot_bytes};
    const cuuint32_t bd[5] = {16, 16, 2, 4, 1};
    return make_byte_map(enc, nib, pool, 5, dq, sq, bq) || make_byte_map(enc, scl, pool + 16 * nbk * 16, 5, dd, sd, bd);
  }
  const cuuint64_t dq[4] = {256, (cuuint64_t)H / 16, (cuuint64_t)I / 32, n_slots};
  const cuuint64_t sq[3] = {256, lay.unit, slot_bytes};
  const cuuint32_t bq[4] = {256, 16, 2, 1};
  const cuuint64_t dd[4] = {256, (cuuint64_t)H / 128, (cuuint64_t)I / 32, n_slots};
  const cuuint64_t sd[3] = {256, lay.unit, slot_bytes};
  const cuuint32_t bd[4] = {256, 2, 8, 1};
  return make_byte_map(enc, nib, pool + unit_down_nib(H), 4, dq, sq, bq) ||
         make_byte_map(enc, scl, pool + unit_down_scl(H), 4, dd, sd, bd);
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
    p.bias = a.bias;
    p.gain = a.gain;
    p.pin_slot = a.pin_slot;
    p.layer_base = a.layer_base;
    p.hist = a.hist;
    p.wnorm = a.wnorm;
    p.router_rows = a.router_rows;
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
    CUtensorMap mua;
    if (make_map(enc, &mua, s.ua, Tc, (uint64_t)kRParts * H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) return -1;
    const int rn = router_n(E), total_k = kRParts * H / kTK;
    const int nsplit = kRSplit < total_k ? kRSplit : total_k;
    const int kps = (total_k + nsplit - 1) / nsplit;
    const dim3 rgrid((Tc + kTM - 1) / kTM, (E + rn - 1) / rn, nsplit);
    for (int l = 0; l < a.L; ++l) {
      CUtensorMap mw;
      if (make_map(enc, &mw, a.router_rows + (size_t)l * E * H, E, H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rn)) return -1;
      prefill_route_prep<<<(Tc + kPT / 32 - 1) / (kPT / 32), kPT, 0, st>>>(p, l);
      prefill_router_gemm<<<rgrid, kRGT, router_gemm_smem(E), st>>>(p, mua, mw, rn, kps);
      prefill_route_select<<<(Tc + kPT / 32 - 1) / (kPT / 32), kPT, route_select_smem(E), st>>>(p, l, nsplit);
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
