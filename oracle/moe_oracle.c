/*
 * moe_oracle.c -- CPU oracle of the sparse MoE decode step with a bounded expert cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Plain, slow, single-threaded C (built with -O2
 * -ffp-contract=off, no SIMD intrinsics).  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg load it; the CUDA library never does, and the two share no
 * code, header, table or constant.
 *
 * What it computes.  The method (Luce Spark; theneuralfeed.com, "Luce Spark runs 35B
 * MoE models on 16GB GPU without speed loss", key-components paragraph) routes every
 * token of an A3B MoE to about 8 of 256 experts, keeps the experts that calibration
 * found hot pinned in GPU memory, copies a cold expert into a bounded ring of spare
 * slots on demand while evicting the least recently used entry, and runs the token as
 * one graph.  Caching changes where a weight lives, never its value, so the write-up's
 * claim that full residency is bit-identical to all-GPU makes the exact MoE layer the
 * oracle's definition.  The MoE layer itself (router, top-k, SwiGLU experts, shared
 * expert, RMSNorm, Q4_0) is not spelled out on the pages; the readings used here are:
 *
 *   Q4_0 (named, not defined, in the Baidu "Mixture-of-Experts: The Key to Breaking
 *   VRAM Limitations" page, quantisation section; public GGUF convention): 32 weights
 *   per 18-byte block, fp16 scale d then 16 bytes; byte j holds weight j (low nibble)
 *   and weight j+16 (high nibble); weight = (q - 8) * d.
 *
 *   Router: z_e = sum_j W_r[e,j] * x_j + b_e, W_r in bf16; softmax over all experts,
 *   keep the top-k, renormalise (equal to a softmax over the kept logits).  Top-k
 *   order: larger logit first, equal logits -> lower expert index.
 *
 *   Routing decides integers, so the logits are formed in fp32 in one canonical order
 *   that the GPU kernel follows too: column chunks of 16, each an fmaf chain from +0;
 *   chunk partials folded by orc_canonical_sum (lane l of 32 adds chunks l, l+32, ...
 *   from +0, then xor-butterfly offsets 16, 8, 4, 2, 1).  With the pre-norm stack the
 *   norm's scale is applied after the fold: z_e = fmaf(S_e, inv, b_e), S_e over
 *   u_j = g_j * h_j and inv = 1 / sqrt(ss / H + eps), ss folded the same way.  This is
 *   the definition up to fp32 rounding order; the tests pin it to the fp64 dot within
 *   the standard error bound.
 *
 *   Experts: a = silu(G x) (.) (U x), silu(t) = t / (1 + e^-t); o = D a.  Combine:
 *   y = sum_i w_i o_i + o_shared (shared expert ungated).  Stack: h <- h + y on
 *   RMSNorm(h) input; single layer without norm: y = MoE(x).  All in fp64.
 *
 *   Recalibration: score <- floor(score / 2) + window count, re-pin top-P by score,
 *   the ring emptied at every re-pin (orc_cache_set_pinned).
 *
 *   Cache (key-components item 2): per layer, accesses in the token's rank order;
 *   pinned -> PIN_HIT; resident in the ring -> RING_HIT and refresh recency; else MISS
 *   into the lowest-index empty ring slot, else into the least recently used one.
 *   Pinned set (item 1): the top-P experts by accumulated routing count, ties -> lower
 *   index.  Slots are numbered: pinned experts 0..P-1 in ascending expert order, ring
 *   slot r -> P + r.
 *
 * Every function here is pinned by a -m "not gpu" test (hand-built blocks, brute force,
 * closed forms, library routines); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_CHUNK 16
#define ORC_LANES 32

/* ---------------------------------------------------------------- conversions */

/* IEEE half -> float, from the binary16 definition (exact). */
float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1, exp = (h >> 10) & 0x1f, man = h & 0x3ff;
  float v;
  if (exp == 0)
    v = ldexpf((float)man, -24); /* subnormal: man * 2^-24 */
  else if (exp == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexpf((float)(man | 0x400), exp - 25);
  return sign ? -v : v;
}

/* bf16 -> float: the bf16 bits are the high half of the float. */
float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---------------------------------------------------------------- Q4_0 */

/* Dequantise n_blocks canonical Q4_0 blocks into out[32 * n_blocks]. */
void orc_dequant_q4_0(const uint8_t *blocks, int64_t n_blocks, double *out) {
  for (int64_t b = 0; b < n_blocks; ++b) {
    const uint8_t *blk = blocks + 18 * b;
    double d = (double)orc_f16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
    const uint8_t *qs = blk + 2;
    for (int j = 0; j < 16; ++j) {
      out[32 * b + j] = (double)((qs[j] & 15) - 8) * d;
      out[32 * b + 16 + j] = (double)((qs[j] >> 4) - 8) * d;
    }
  }
}

/* ---------------------------------------------------------------- canonical fp32 */

/* Fold n partial sums in the canonical order (see header). */
float orc_canonical_sum(const float *parts, int n) {
  float lane[ORC_LANES], next[ORC_LANES];
  for (int l = 0; l < ORC_LANES; ++l) {
    float acc = 0.0f;
    for (int m = l; m < n; m += ORC_LANES) acc = acc + parts[m];
    lane[l] = acc;
  }
  for (int off = ORC_LANES / 2; off >= 1; off /= 2) {
    for (int l = 0; l < ORC_LANES; ++l) next[l] = lane[l] + lane[l ^ off];
    memcpy(lane, next, sizeof lane);
  }
  return lane[0];
}

/* 1 / sqrt(mean(h^2) + eps) in fp32, canonical order.  H % 16 == 0. */
float orc_rms_inv(const float *h, int H, float eps) {
  int nch = H / ORC_CHUNK;
  float *parts = (float *)malloc(sizeof(float) * (size_t)nch);
  for (int c = 0; c < nch; ++c) {
    float p = 0.0f;
    for (int t = 0; t < ORC_CHUNK; ++t) p = fmaf(h[c * ORC_CHUNK + t], h[c * ORC_CHUNK + t], p);
    parts[c] = p;
  }
  float ss = orc_canonical_sum(parts, nch);
  free(parts);
  float mean = ss / (float)H;
  float r = sqrtf(mean + eps);
  return 1.0f / r;
}

/* Router logits z[E] in fp32, canonical order.  w: [E][H] bf16; gain may be NULL (no
 * norm: u = h, and the caller passes inv = 1); bias may be NULL (zero). */
void orc_router_logits(const uint16_t *w, const float *h, const float *gain, float inv,
                       const float *bias, int E, int H, float *z) {
  int nch = H / ORC_CHUNK;
  float *u = (float *)malloc(sizeof(float) * (size_t)H);
  float *parts = (float *)malloc(sizeof(float) * (size_t)nch);
  for (int j = 0; j < H; ++j) u[j] = gain ? gain[j] * h[j] : h[j];
  for (int e = 0; e < E; ++e) {
    const uint16_t *row = w + (size_t)e * H;
    for (int c = 0; c < nch; ++c) {
      float p = 0.0f;
      for (int t = 0; t < ORC_CHUNK; ++t) {
        int j = c * ORC_CHUNK + t;
        p = fmaf(orc_bf16_to_f32(row[j]), u[j], p);
      }
      parts[c] = p;
    }
    float s = orc_canonical_sum(parts, nch);
    z[e] = fmaf(s, inv, bias ? bias[e] : 0.0f);
  }
  free(parts);
  free(u);
}

/* ---------------------------------------------------------------- routing */

/* Top-k by (logit desc, index asc). */
void orc_topk(const float *z, int E, int k, int32_t *sel) {
  uint8_t *taken = (uint8_t *)calloc((size_t)E, 1);
  for (int i = 0; i < k; ++i) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || z[e] > z[best]) best = e;
    }
    taken[best] = 1;
    sel[i] = best;
  }
  free(taken);
}

/* Softmax over all E, keep sel, renormalise == softmax over the kept logits. */
void orc_route_weights(const float *z, const int32_t *sel, int k, double *w) {
  double zmax = (double)z[sel[0]];
  for (int i = 1; i < k; ++i)
    if ((double)z[sel[i]] > zmax) zmax = (double)z[sel[i]];
  double s = 0.0;
  for (int i = 0; i < k; ++i) s += exp((double)z[sel[i]] - zmax);
  for (int i = 0; i < k; ++i) w[i] = exp((double)z[sel[i]] - zmax) / s;
}

/* ---------------------------------------------------------------- experts */

double orc_silu(double t) { return t / (1.0 + exp(-t)); }

/* One SwiGLU expert over canonical Q4_0 gate|up|down: out[H] = D (silu(G x) * (U x)). */
void orc_expert_ffn(const uint8_t *q4, int H, int I, const double *x, double *out) {
  const int64_t rowblk_gu = H / 32, rowblk_d = I / 32;
  const uint8_t *G = q4, *U = q4 + (size_t)I * rowblk_gu * 18,
                *D = q4 + (size_t)2 * I * rowblk_gu * 18;
  double *row = (double *)malloc(sizeof(double) * (size_t)(H > I ? H : I));
  double *a = (double *)malloc(sizeof(double) * (size_t)I);
  for (int r = 0; r < I; ++r) {
    double g = 0.0, u = 0.0;
    orc_dequant_q4_0(G + (size_t)r * rowblk_gu * 18, rowblk_gu, row);
    for (int j = 0; j < H; ++j) g += row[j] * x[j];
    orc_dequant_q4_0(U + (size_t)r * rowblk_gu * 18, rowblk_gu, row);
    for (int j = 0; j < H; ++j) u += row[j] * x[j];
    a[r] = orc_silu(g) * u;
  }
  for (int j = 0; j < H; ++j) {
    double o = 0.0;
    orc_dequant_q4_0(D + (size_t)j * rowblk_d * 18, rowblk_d, row);
    for (int r = 0; r < I; ++r) o += row[r] * a[r];
    out[j] = o;
  }
  free(a);
  free(row);
}

typedef struct {
  int32_t hidden, n_experts, top_k, inter, shared_inter, use_rmsnorm;
  float rms_eps;
} orc_dims;

typedef struct {
  const uint8_t *const *experts; /* [E] canonical Q4_0 gate|up|down */
  const uint8_t *shared;         /* shared expert or NULL */
  const uint16_t *router;        /* [E][H] bf16 */
  const float *bias;             /* [E] or NULL */
  const float *gain;             /* [H] or NULL (ones) */
} orc_layer_w;

/* One MoE layer.  h32 is the fp32 input used for the routing decision, h64 the same
 * input carried in fp64 for everything else (teacher forcing passes h64 = h32).
 * Outputs: z[E], sel[k], w[k], y[H] = MoE output, h_out[H] = h + y (stack) or y. */
void orc_moe_layer(const orc_dims *d, const orc_layer_w *lw, const float *h32,
                   const double *h64, float *z, int32_t *sel, double *w, double *y,
                   double *h_out) {
  const int H = d->hidden, E = d->n_experts, k = d->top_k;
  double *x = (double *)malloc(sizeof(double) * (size_t)H);
  double *o = (double *)malloc(sizeof(double) * (size_t)H);
  float inv = 1.0f;
  const float *gain = NULL;
  float *ones = NULL;
  if (d->use_rmsnorm) {
    inv = orc_rms_inv(h32, H, d->rms_eps);
    if (lw->gain) {
      gain = lw->gain;
    } else {
      ones = (float *)malloc(sizeof(float) * (size_t)H);
      for (int j = 0; j < H; ++j) ones[j] = 1.0f;
      gain = ones;
    }
    double ss = 0.0;
    for (int j = 0; j < H; ++j) ss += h64[j] * h64[j];
    double inv64 = 1.0 / sqrt(ss / H + (double)d->rms_eps);
    for (int j = 0; j < H; ++j) x[j] = h64[j] * inv64 * (double)gain[j];
  } else {
    for (int j = 0; j < H; ++j) x[j] = h64[j];
  }
  orc_router_logits(lw->router, h32, gain, inv, lw->bias, E, H, z);
  orc_topk(z, E, k, sel);
  orc_route_weights(z, sel, k, w);
  for (int j = 0; j < H; ++j) y[j] = 0.0;
  for (int i = 0; i < k; ++i) {
    orc_expert_ffn(lw->experts[sel[i]], H, d->inter, x, o);
    for (int j = 0; j < H; ++j) y[j] += w[i] * o[j];
  }
  if (d->shared_inter > 0 && lw->shared) {
    orc_expert_ffn(lw->shared, H, d->shared_inter, x, o);
    for (int j = 0; j < H; ++j) y[j] += o[j];
  }
  for (int j = 0; j < H; ++j) h_out[j] = d->use_rmsnorm ? h64[j] + y[j] : y[j];
  free(ones);
  free(o);
  free(x);
}

/* A free-running decode of one token through n_layers layers (fp64 carried between
 * layers; each layer's routing sees the fp32 rounding of its input).  sel_out [L][k]
 * and trace [(L+1)][H] (input, then each layer's output) may be NULL. */
void orc_decode_token(const orc_dims *d, int n_layers, const orc_layer_w *layers,
                      const float *x, double *h_out, int32_t *sel_out, double *trace) {
  const int H = d->hidden, E = d->n_experts, k = d->top_k;
  double *h = (double *)malloc(sizeof(double) * (size_t)H);
  double *hn = (double *)malloc(sizeof(double) * (size_t)H);
  double *y = (double *)malloc(sizeof(double) * (size_t)H);
  float *h32 = (float *)malloc(sizeof(float) * (size_t)H);
  float *z = (float *)malloc(sizeof(float) * (size_t)E);
  int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
  double *w = (double *)malloc(sizeof(double) * (size_t)k);
  for (int j = 0; j < H; ++j) h[j] = (double)x[j];
  if (trace) memcpy(trace, h, sizeof(double) * (size_t)H);
  for (int l = 0; l < n_layers; ++l) {
    for (int j = 0; j < H; ++j) h32[j] = (float)h[j];
    orc_moe_layer(d, &layers[l], h32, h, z, sel, w, y, hn);
    memcpy(h, hn, sizeof(double) * (size_t)H);
    if (sel_out) memcpy(sel_out + (size_t)l * k, sel, sizeof(int32_t) * (size_t)k);
    if (trace) memcpy(trace + (size_t)(l + 1) * H, h, sizeof(double) * (size_t)H);
  }
  memcpy(h_out, h, sizeof(double) * (size_t)H);
  free(w);
  free(sel);
  free(z);
  free(h32);
  free(y);
  free(hn);
  free(h);
}

/* ---------------------------------------------------------------- placement */

/* Pinned set: the top-P experts by count, ties -> lower index.  mask[E] out. */
void orc_select_pinned(const uint32_t *hist, int E, int P, uint8_t *mask) {
  memset(mask, 0, (size_t)E);
  for (int p = 0; p < P; ++p) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (mask[e]) continue;
      if (best < 0 || hist[e] > hist[best]) best = e;
    }
    mask[best] = 1;
  }
}

/* Online recalibration (reading of the write-up's "self-tunes over time" with routing
 * frequencies accumulated from real requests): per expert, score <- floor(score / 2) +
 * the routing count of the window since the previous recalibration; the pinned set is
 * then orc_select_pinned over the scores. */
void orc_recal_score(uint32_t *score, const uint32_t *window, int n) {
  for (int i = 0; i < n; ++i) score[i] = (score[i] >> 1) + window[i];
}

/* ---------------------------------------------------------------- cache simulator */

enum { ORC_PIN_HIT = 0, ORC_RING_HIT = 1, ORC_MISS = 2 };

typedef struct {
  int32_t step, layer, rank, expert, kind, slot, evicted;
} orc_event;

typedef struct {
  int n_layers, n_experts, ring_slots;
  int32_t *pin_slot;   /* [L][E] pinned slot or -1 */
  int32_t *n_pinned;   /* [L] */
  int32_t *ring_owner; /* [L][R], -1 empty */
  uint64_t *ring_used; /* [L][R] recency stamp */
  uint64_t *clock;     /* [L] */
} orc_cache;

orc_cache *orc_cache_create(int n_layers, int n_experts, int ring_slots) {
  orc_cache *c = (orc_cache *)calloc(1, sizeof(orc_cache));
  c->n_layers = n_layers;
  c->n_experts = n_experts;
  c->ring_slots = ring_slots;
  c->pin_slot = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_layers * n_experts);
  c->n_pinned = (int32_t *)calloc((size_t)n_layers, sizeof(int32_t));
  c->ring_owner = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_layers * (ring_slots ? ring_slots : 1));
  c->ring_used = (uint64_t *)calloc((size_t)n_layers * (ring_slots ? ring_slots : 1), sizeof(uint64_t));
  c->clock = (uint64_t *)calloc((size_t)n_layers, sizeof(uint64_t));
  for (int64_t i = 0; i < (int64_t)n_layers * n_experts; ++i) c->pin_slot[i] = -1;
  for (int64_t i = 0; i < (int64_t)n_layers * ring_slots; ++i) c->ring_owner[i] = -1;
  return c;
}

void orc_cache_destroy(orc_cache *c) {
  if (!c) return;
  free(c->pin_slot);
  free(c->n_pinned);
  free(c->ring_owner);
  free(c->ring_used);
  free(c->clock);
  free(c);
}

/* Set a layer's pinned set from mask[E] and empty its ring. */
void orc_cache_set_pinned(orc_cache *c, int layer, const uint8_t *mask) {
  int p = 0;
  for (int e = 0; e < c->n_experts; ++e)
    c->pin_slot[(size_t)layer * c->n_experts + e] = mask[e] ? p++ : -1;
  c->n_pinned[layer] = p;
  for (int r = 0; r < c->ring_slots; ++r) {
    c->ring_owner[(size_t)layer * c->ring_slots + r] = -1;
    c->ring_used[(size_t)layer * c->ring_slots + r] = 0;
  }
  c->clock[layer] = 0;
}

/* One token's accesses to one layer, in rank order.  Writes k events. */
void orc_cache_access(orc_cache *c, int step, int layer, const int32_t *sel, int k,
                      orc_event *ev) {
  const int R = c->ring_slots, P = c->n_pinned[layer];
  int32_t *owner = c->ring_owner + (size_t)layer * R;
  uint64_t *used = c->ring_used + (size_t)layer * R;
  for (int i = 0; i < k; ++i) {
    int e = sel[i];
    orc_event *v = &ev[i];
    v->step = step;
    v->layer = layer;
    v->rank = i;
    v->expert = e;
    v->evicted = -1;
    int ps = c->pin_slot[(size_t)layer * c->n_experts + e];
    if (ps >= 0) {
      v->kind = ORC_PIN_HIT;
      v->slot = ps;
      continue;
    }
    int hit = -1;
    for (int r = 0; r < R; ++r)
      if (owner[r] == e) hit = r;
    if (hit >= 0) {
      v->kind = ORC_RING_HIT;
      v->slot = P + hit;
      used[hit] = ++c->clock[layer];
      continue;
    }
    if (R == 0) { /* no ring: a cold access has nowhere to go */
      v->kind = ORC_MISS;
      v->slot = -1;
      continue;
    }
    int victim = -1;
    for (int r = 0; r < R && victim < 0; ++r)
      if (owner[r] < 0) victim = r;
    if (victim < 0) {
      victim = 0;
      for (int r = 1; r < R; ++r)
        if (used[r] < used[victim]) victim = r;
    }
    v->kind = ORC_MISS;
    v->slot = P + victim;
    v->evicted = owner[victim];
    owner[victim] = e;
    used[victim] = ++c->clock[layer];
  }
}

/* Read back a layer's ring (owner[R]) for checks. */
void orc_cache_ring(const orc_cache *c, int layer, int32_t *owner_out) {
  memcpy(owner_out, c->ring_owner + (size_t)layer * c->ring_slots,
         sizeof(int32_t) * (size_t)c->ring_slots);
}
