// moe_api.cu -- host runtime and C ABI of libmoe (see include/moe_cache.h).
//
// Owns: the pinned host tier holding every routed expert in the slot layout (the
// write-up's "long tail lives in system RAM", baguaai.com event core; "copied
// asynchronously from pinned host memory", theneuralfeed.com key components item 2),
// the device slot pool (pinned experts, ring slots, staging slots), the cache tables,
// the exchange scratch of the decode kernel, the event log and histogram, the
// per-token CUDA graphs (key components item 3), and the miss proxy: a host thread
// that watches the host-mapped mailbox the kernel writes on a miss, issues the
// copy-engine transfer pinned host -> ring slot on a non-blocking side stream, and then
// signals the kernel with a stream memory write, so the slot is refilled by the copy
// engine in stream order after its last reader (the kernel issues the request only
// after the layer's routing, when no reader of the victim slot is left).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "../../include/moe_cache.h"
#include "moe_internal.h"
#include "prefill.h"

namespace moe {
bool decode_plan(int H, int E, int grid, int smem_optin, int* rx, int* down_late, uint32_t* smem);
cudaError_t decode_configure(int limit);
cudaError_t decode_max_blocks_per_sm(int H, uint32_t smem, int* out);
cudaError_t decode_launch(const DecodeParams& p, int grid, cudaStream_t stream);
}  // namespace moe

using namespace moe;

typedef CUresult (*PfnWriteValue32)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);

struct moe_ctx {
  moe_config cfg{};
  int L = 0, H = 0, E = 0, K = 0, I = 0, Is = 0, R = 0;
  int nsm = 0, grid = 0, rx = 1, down_late = 0;
  uint32_t smem = 0;
  int miss_mode = kMissProxy;
  SlotLayout lay{}, slay{};
  uint64_t slot_bytes = 0, shared_slot_bytes = 0;
  // host tier (mapped: the kernel reads it directly in the SM-pull miss path)
  uint8_t* host_tier = nullptr;
  const uint8_t* host_tier_dev = nullptr;
  std::vector<uint8_t> loaded;
  // device
  uint8_t* shared_pool = nullptr;
  std::atomic<uint8_t*> pool{nullptr};
  int64_t pool_slots = 0;
  uint16_t* router_rows = nullptr;  // [L][E][H] bf16 (decode router rows; prefill's router GEMM)
  float* wnorm = nullptr;           // [L] max_e ||w_e||_2 rounded up (prefill's routing bound)
  float* bias = nullptr;
  float* gain = nullptr;
  bool has_bias = false, has_gain = false;
  int32_t *pin_slot = nullptr, *layer_base = nullptr, *n_pinned = nullptr, *ring_owner = nullptr;
  uint32_t *ring_stamp = nullptr, *ring_clock = nullptr;
  unsigned long long* acc = nullptr;  // [kAccBufs][H] fixed-point layer outputs
  unsigned long long* zll = nullptr;  // [E] published logits
  int32_t* likely = nullptr;  // [2][L][kMaxLikely]: pool slots, then expert ids, of the likeliest pinned experts
  int n_pre = 0, n_l2 = 0;
  uint32_t* hist = nullptr;
  int32_t* log = nullptr;
  int log_steps = 0;
  Ctrl* ctrl = nullptr;
  uint32_t* done_seq = nullptr;
  float *x_buf = nullptr, *y_buf = nullptr;
  float *x_pin = nullptr, *y_pin = nullptr;
  int32_t* err_pin = nullptr;
  MissReq *mbox_host = nullptr, *mbox_dev = nullptr;
  // residency and online recalibration
  std::vector<int32_t> pin_host;   // [L][E] the device table's entries
  std::vector<int32_t> phys_owner; // [L][P] expert in each physical pinned slot
  std::vector<uint32_t> score;     // [L][E] decayed routing counts
  std::vector<uint32_t> hist_snap; // [L][E] device histogram at the last (re)calibration
  uint64_t repins = 0, repin_copies = 0;
  bool resident = false;
  float residency = 0.0f;
  int placement = 0, P = 0, staging_base = 0;
  // streams and graphs
  cudaStream_t side = nullptr, own = nullptr;
  cudaGraphExec_t g_dev = nullptr, g_host = nullptr;
  cudaGraph_t gr_dev = nullptr;       // the graph g_dev was instantiated from (kept for its node)
  cudaGraphNode_t kn_dev = nullptr;   // its kernel node: new x / y pointers update it in place
  const float* g_x = nullptr;
  float* g_y = nullptr;
  // proxy
  std::thread proxy;
  std::atomic<bool> stop{false};
  std::atomic<uint32_t> proxy_next{1};
  std::atomic<int> drop{0};
  std::atomic<int> proxy_err{0};
  // timing of the proxy's copies: event pairs recorded around each cudaMemcpyAsync on
  // the side stream, harvested by moe_stats (a copy finds no free pair: untimed)
  static constexpr int kCopyTimers = 64;
  cudaEvent_t ev_start[kCopyTimers] = {}, ev_end[kCopyTimers] = {};
  std::mutex timer_mu;
  std::vector<int> timer_free, timer_pending;
  uint64_t copy_ns = 0, copies_timed = 0;
  PfnWriteValue32 write_value32 = nullptr;
  // tracing and log reading
  float *h_trace = nullptr, *w_trace = nullptr;
  unsigned long long* phase_trace = nullptr;
  size_t phase_trace_words = 0;
  uint64_t log_read_step = 0, log_dropped = 0;
  // batched prefill: scratch for up to prefill_cap tokens (one allocation), tracing
  uint8_t* prefill_mem = nullptr;
  int prefill_cap = 0;
  PrefillScratch pf{};
  bool prefill_configured = false;
  void* encode_tiled = nullptr;
  float* pf_h_trace = nullptr;
  int32_t* pf_sel_trace = nullptr;
  // the captured prefill pass and what it was captured for
  cudaGraphExec_t g_pf = nullptr;
  const float* gpf_x = nullptr;
  float* gpf_y = nullptr;
  int gpf_T = 0;
  float* gpf_ht = nullptr;
  int32_t* gpf_st = nullptr;
  const uint8_t* gpf_pool = nullptr;
  const uint8_t* gpf_mem = nullptr;
};

#define CK(call)                                  \
  do {                                            \
    cudaError_t e_ = (call);                      \
    if (e_ != cudaSuccess) return cuda_fail(e_);  \
  } while (0)

static int cuda_fail(cudaError_t e) {
  if (e == cudaErrorMemoryAllocation) return MOE_ERR_NOMEM;
  return MOE_ERR_CUDA;
}

static int deverr_status(int32_t e) {
  if (e == 0) return MOE_OK;
  if (e == MOE_DEVERR_BARRIER || e == MOE_DEVERR_MISS || e == MOE_DEVERR_TMA) return MOE_ERR_TIMEOUT;
  return MOE_ERR_DEVICE;
}

// ------------------------------------------------------------------ proxy

static void cpu_relax() {
#if defined(__x86_64__)
  __builtin_ia32_pause();
#endif
}

static void proxy_main(moe_ctx* c) {
  cudaSetDevice(c->cfg.device);
  auto last_work = std::chrono::steady_clock::now();
  while (!c->stop.load(std::memory_order_relaxed)) {
    const uint32_t next = c->proxy_next.load(std::memory_order_relaxed);
    volatile MissReq* q = &c->mbox_host[next % kMboxCap];
    if (q->seq != next) {
      cpu_relax();
      if (std::chrono::steady_clock::now() - last_work > std::chrono::milliseconds(20))
        std::this_thread::sleep_for(std::chrono::microseconds(50));
      continue;
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    const uint32_t layer = q->layer, expert = q->expert, dst = q->dst_slot;
    uint8_t* pool = c->pool.load(std::memory_order_acquire);
    if (layer >= (uint32_t)c->L || expert >= (uint32_t)c->E || (int64_t)dst >= c->pool_slots || !pool) {
      c->proxy_err.store(1);  // leave it unsignalled: the kernel's bounded wait reports it
    } else {
      int timer = -1;
      {
        std::lock_guard<std::mutex> lk(c->timer_mu);
        if (!c->timer_free.empty()) {
          timer = c->timer_free.back();
          c->timer_free.pop_back();
        }
      }
      if (timer >= 0) cudaEventRecord(c->ev_start[timer], c->side);
      const cudaError_t ce = cudaMemcpyAsync(pool + (size_t)dst * c->slot_bytes,
                                             c->host_tier + ((size_t)layer * c->E + expert) * c->slot_bytes,
                                             c->slot_bytes, cudaMemcpyHostToDevice, c->side);
      if (timer >= 0) {
        cudaEventRecord(c->ev_end[timer], c->side);
        std::lock_guard<std::mutex> lk(c->timer_mu);
        c->timer_pending.push_back(timer);
      }
      if (ce != cudaSuccess) {
        // a copy that was not enqueued must not be signalled: the slot would be read
        // stale; the kernel's bounded wait turns the missing signal into MOE_ERR_TIMEOUT
        c->proxy_err.store(2);
      } else if (c->drop.load() > 0) {
        c->drop.fetch_sub(1);
      } else if (c->write_value32((CUstream)c->side, (CUdeviceptr)c->done_seq, next, 0) != CUDA_SUCCESS) {
        c->proxy_err.store(3);
      }
    }
    c->proxy_next.store(next + 1, std::memory_order_release);
    last_work = std::chrono::steady_clock::now();
  }
}

// ------------------------------------------------------------------ helpers

static DecodeParams make_params(const moe_ctx* c, const float* x, float* y) {
  DecodeParams p{};
  p.L = c->L;
  p.H = c->H;
  p.E = c->E;
  p.K = c->K;
  p.I = c->I;
  p.Is = c->Is;
  p.R = c->R;
  p.use_norm = c->cfg.use_rmsnorm;
  p.eps = c->cfg.rms_eps;
  p.n_units = c->K * (c->I / 32) + c->Is / 32;
  p.rx_per_cta = c->rx;
  p.down_late = c->down_late;
  p.miss_mode = c->miss_mode;
  p.nan_on_error = 0;
  p.pool = c->pool.load();
  p.slot_bytes = c->slot_bytes;
  p.unit_bytes = c->lay.unit;
  p.shared_pool = c->shared_pool;
  p.shared_slot_bytes = c->shared_slot_bytes;
  p.router = c->router_rows;
  p.bias = c->has_bias ? c->bias : nullptr;
  p.gain = c->has_gain ? c->gain : nullptr;
  p.pin_slot = c->pin_slot;
  p.layer_base = c->layer_base;
  p.n_pinned = c->n_pinned;
  p.ring_owner = c->ring_owner;
  p.ring_stamp = c->ring_stamp;
  p.ring_clock = c->ring_clock;
  p.staging_base = c->staging_base;
  p.x = x;
  p.y = y;
  p.h_trace = c->h_trace;
  p.w_trace = c->w_trace;
  p.acc = c->acc;
  p.zll = c->zll;
  p.hist = c->hist;
  p.log = c->log;
  p.log_steps = c->log_steps;
  p.ctrl = c->ctrl;
  p.mbox = c->mbox_dev;
  p.done_seq = c->done_seq;
  p.host_tier = c->host_tier_dev;
  p.timeout_ns = (unsigned long long)c->cfg.wait_timeout_ms * 1000000ull;
  p.phase_trace = c->phase_trace;
  p.likely_slot = c->likely;
  p.likely_e = c->likely + (size_t)c->L * kMaxLikely;
  p.n_pre = c->n_pre;
  p.n_l2 = c->n_l2;
  return p;
}

static void drop_graphs(moe_ctx* c) {
  if (c->g_dev) cudaGraphExecDestroy(c->g_dev);
  if (c->gr_dev) cudaGraphDestroy(c->gr_dev);
  c->gr_dev = nullptr;
  c->kn_dev = nullptr;
  if (c->g_host) cudaGraphExecDestroy(c->g_host);
  if (c->g_pf) cudaGraphExecDestroy(c->g_pf);
  c->g_dev = c->g_host = c->g_pf = nullptr;
  c->g_x = nullptr;
  c->g_y = nullptr;
}

// Capture one token: [optional H2D of x] -> decode kernel -> [optional D2H of y, error].
// keep, when non-null, receives the captured graph (not destroyed) and knode its kernel node.
static int capture_token(moe_ctx* c, const float* x, float* y, bool host_io, cudaGraphExec_t* out,
                         cudaGraph_t* keep = nullptr, cudaGraphNode_t* knode = nullptr) {
  cudaGraph_t graph = nullptr;
  CK(cudaStreamBeginCapture(c->own, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = cudaSuccess;
  if (host_io) e = cudaMemcpyAsync(c->x_buf, c->x_pin, sizeof(float) * c->H, cudaMemcpyHostToDevice, c->own);
  // the launch's arrival counter starts at 0
  if (e == cudaSuccess) e = cudaMemsetAsync(&c->ctrl->bar_count, 0, sizeof(uint32_t), c->own);
  if (e == cudaSuccess) e = decode_launch(make_params(c, x, y), c->grid, c->own);
  if (e == cudaSuccess && host_io)
    e = cudaMemcpyAsync(c->y_pin, c->y_buf, sizeof(float) * c->H, cudaMemcpyDeviceToHost, c->own);
  if (e == cudaSuccess && host_io)
    e = cudaMemcpyAsync(c->err_pin, &c->ctrl->error, sizeof(int32_t), cudaMemcpyDeviceToHost, c->own);
  cudaError_t e2 = cudaStreamEndCapture(c->own, &graph);
  if (e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return cuda_fail(e);
  }
  if (e2 != cudaSuccess) return cuda_fail(e2);
  e = cudaGraphInstantiate(out, graph, 0);
  if (e == cudaSuccess && keep) {
    size_t n = 0;
    e = cudaGraphGetNodes(graph, nullptr, &n);
    std::vector<cudaGraphNode_t> nodes(n);
    if (e == cudaSuccess && n) e = cudaGraphGetNodes(graph, nodes.data(), &n);
    *knode = nullptr;
    for (size_t i = 0; i < n && e == cudaSuccess; ++i) {
      cudaGraphNodeType t;
      e = cudaGraphNodeGetType(nodes[i], &t);
      if (e == cudaSuccess && t == cudaGraphNodeTypeKernel) *knode = nodes[i];
    }
    if (e == cudaSuccess && !*knode) e = cudaErrorInvalidValue;
    if (e == cudaSuccess) {
      *keep = graph;
      return MOE_OK;
    }
    cudaGraphExecDestroy(*out);
    *out = nullptr;
  }
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return cuda_fail(e);
  return MOE_OK;
}

template <typename T>
static cudaError_t dalloc(T** p, size_t count) {
  return cudaMalloc((void**)p, sizeof(T) * (count ? count : 1));
}

// Canonical Q4_0 rows [rows x cols] -> 16-row tiles; tile_of(row) gives the tile's offset.
template <typename TileOf>
static void repack_rows(const uint8_t* src, uint8_t* dst, int64_t rows, int64_t cols, TileOf tile_of) {
  const int64_t nb = cols / 32;
  for (int64_t r = 0; r < rows; ++r) {
    uint8_t* tile = dst + tile_of(r);
    const int64_t rr = r % 16;
    uint8_t* qs = tile + rr * nb * 16;
    uint8_t* d = tile + 16 * nb * 16 + rr * nb * 2;
    for (int64_t b = 0; b < nb; ++b) {
      const uint8_t* blk = src + (r * nb + b) * 18;
      memcpy(d + 2 * b, blk, 2);
      memcpy(qs + 16 * b, blk + 2, 16);
    }
  }
}

// Canonical gate | up | down of one expert (width I) -> the unit layout of moe_internal.h.
static void repack_expert(const uint8_t* src, uint8_t* dst, const SlotLayout& s, int H, int I) {
  const uint64_t gu = q4_bytes(I, H);
  const uint64_t t_gu = 9ull * H;
  repack_rows(src, dst, I, H,
              [&](int64_t r) { return (r / 32) * s.unit + unit_gu_tile(H, (int)((r % 32) / 16)); });
  repack_rows(src + gu, dst, I, H,
              [&](int64_t r) { return (r / 32) * s.unit + unit_gu_tile(H, 2 + (int)((r % 32) / 16)); });
  (void)t_gu;
  // down [H x I]: block rb of row j -> unit rb, nibbles at j * 16, scale at j * 2
  const uint8_t* D = src + 2 * gu;
  const int nbd = I / 32;
  for (int64_t j = 0; j < H; ++j)
    for (int rb = 0; rb < nbd; ++rb) {
      const uint8_t* blk = D + (j * nbd + rb) * 18;
      uint8_t* u = dst + rb * s.unit;
      memcpy(u + unit_down_nib(H) + j * 16, blk + 2, 16);
      memcpy(u + unit_down_scl(H) + j * 2, blk, 2);
    }
}

// Placement: top-P experts by count (ties -> lower index), or experts 0..P-1.
static void top_p_mask(const uint32_t* count, int E, int P, int placement, uint8_t* mask) {
  std::vector<int> order(E);
  for (int e = 0; e < E; ++e) {
    order[e] = e;
    mask[e] = 0;
  }
  if (placement == MOE_PLACE_UNIFORM) {
    for (int e = 0; e < P; ++e) mask[e] = 1;
    return;
  }
  std::stable_sort(order.begin(), order.end(), [count](int a, int b) { return count[a] > count[b]; });
  for (int p = 0; p < P; ++p) mask[order[p]] = 1;
}

static int empty_rings(moe_ctx* c, cudaStream_t s) {
  const size_t nr = (size_t)2 * c->L * std::max(c->R, 1);
  CK(cudaMemsetAsync(c->ring_owner, 0xff, nr * 4, s));
  CK(cudaMemsetAsync(c->ring_stamp, 0, nr * 4, s));
  CK(cudaMemsetAsync(c->ring_clock, 0, (size_t)2 * c->L * 4, s));
  return MOE_OK;
}

// Speculative-load table from the recalibration score (the placement histogram,
// decayed): per layer, the pool slots and ids of the n_pre + n_l2 pinned experts with the
// highest counts (ties -> lower index); unused entries -1.
static int upload_likely(moe_ctx* c, cudaStream_t s) {
  const size_t n = (size_t)c->L * kMaxLikely;
  std::vector<int32_t> t(2 * n, -1);
  std::vector<int> order(c->E);
  const int want = c->n_pre + c->n_l2;
  for (int l = 0; l < c->L && want > 0; ++l) {
    const uint32_t* cnt = c->score.data() + (size_t)l * c->E;
    const int32_t* row = c->pin_host.data() + (size_t)l * c->E;
    for (int e = 0; e < c->E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(), [cnt](int a, int b) { return cnt[a] > cnt[b]; });
    int k = 0;
    for (int q = 0; q < c->E && k < want; ++q) {
      const int e = order[q];
      if (row[e] < 0) continue;
      t[(size_t)l * kMaxLikely + k] = l * (c->P + c->R) + (row[e] & 0xffff);
      t[n + (size_t)l * kMaxLikely + k] = e;
      ++k;
    }
  }
  CK(cudaMemcpyAsync(c->likely, t.data(), t.size() * 4, cudaMemcpyHostToDevice, s));
  return cudaStreamSynchronize(s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Add the durations of the proxy's timed copies that have completed (device idle).
static void harvest_copy_timers(moe_ctx* c) {
  std::lock_guard<std::mutex> lk(c->timer_mu);
  for (int t : c->timer_pending) {
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, c->ev_start[t], c->ev_end[t]) == cudaSuccess) {
      c->copy_ns += (uint64_t)((double)ms * 1e6);
      ++c->copies_timed;
    }
    c->timer_free.push_back(t);
  }
  c->timer_pending.clear();
}

// ------------------------------------------------------------------ C ABI

extern "C" {

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument or configuration";
    case MOE_ERR_NOMEM: return "out of memory";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case MOE_ERR_STATE: return "call out of order";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or feature";
    case MOE_ERR_DEVICE: return "the kernel flagged a bad route or slot";
    default: return "unknown status";
  }
}

void moe_destroy(moe_ctx* c) {
  if (!c) return;
  if (c->proxy.joinable()) {
    c->stop.store(true);
    c->proxy.join();
  }
  cudaSetDevice(c->cfg.device);
  cudaDeviceSynchronize();
  drop_graphs(c);
  for (int t = 0; t < moe_ctx::kCopyTimers; ++t) {
    if (c->ev_start[t]) cudaEventDestroy(c->ev_start[t]);
    if (c->ev_end[t]) cudaEventDestroy(c->ev_end[t]);
  }
  if (c->side) cudaStreamDestroy(c->side);
  if (c->own) cudaStreamDestroy(c->own);
  void* dev[] = {c->shared_pool, c->pool.load(), c->bias, c->gain, c->pin_slot,
                 c->layer_base, c->n_pinned, c->ring_owner, c->ring_stamp, c->ring_clock,
                 c->acc, c->zll, c->likely, c->hist, c->log, c->ctrl, c->done_seq,
                 c->x_buf, c->y_buf, c->prefill_mem, c->router_rows, c->wnorm};
  for (void* p : dev)
    if (p) cudaFree(p);
  void* hst[] = {c->host_tier, c->x_pin, c->y_pin, c->err_pin, c->mbox_host};
  for (void* p : hst)
    if (p) cudaFreeHost(p);
  delete c;
}

int moe_load_layer(moe_ctx* c, int32_t l, const uint8_t* const* experts, const uint8_t* shared,
                   const uint16_t* router_bf16, const float* bias, const float* gain) {
  if (!c || l < 0 || l >= c->L || !experts || !router_bf16) return MOE_ERR_INVALID;
  if (c->Is > 0 && !shared) return MOE_ERR_INVALID;
  for (int e = 0; e < c->E; ++e)
    if (!experts[e]) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  // routed experts -> pinned host tier (slot layout), in parallel over experts
  {
    const int nthr = std::max(1, std::min(16, (int)std::thread::hardware_concurrency()));
    std::vector<std::thread> th;
    for (int t = 0; t < nthr; ++t)
      th.emplace_back([=]() {
        for (int e = t; e < c->E; e += nthr)
          repack_expert(experts[e], c->host_tier + ((size_t)l * c->E + e) * c->slot_bytes, c->lay, c->H, c->I);
      });
    for (auto& t : th) t.join();
  }
  if (c->Is > 0) {
    std::vector<uint8_t> tmp(c->shared_slot_bytes, 0);
    repack_expert(shared, tmp.data(), c->slay, c->H, c->Is);
    CK(cudaMemcpy(c->shared_pool + (size_t)l * c->shared_slot_bytes, tmp.data(), c->shared_slot_bytes,
                  cudaMemcpyHostToDevice));
  }
  {  // router rows [E][H] as given
    CK(cudaMemcpy(c->router_rows + (size_t)l * c->E * c->H, router_bf16, (size_t)c->E * c->H * 2,
                  cudaMemcpyHostToDevice));
    double wmax = 0.0;  // the largest router row norm, for the prefill routing error bound
    for (int e = 0; e < c->E; ++e) {
      double ss = 0.0;
      for (int j = 0; j < c->H; ++j) {
        uint32_t bits = (uint32_t)router_bf16[(size_t)e * c->H + j] << 16;
        float w;
        memcpy(&w, &bits, 4);
        ss += (double)w * w;
      }
      wmax = std::max(wmax, std::sqrt(ss));
    }
    const float wn = std::nextafter((float)(wmax * (1.0 + 1e-9)), INFINITY);
    CK(cudaMemcpy(c->wnorm + l, &wn, sizeof(float), cudaMemcpyHostToDevice));
  }
  if (bias) {
    CK(cudaMemcpy(c->bias + (size_t)l * c->E, bias, sizeof(float) * c->E, cudaMemcpyHostToDevice));
    c->has_bias = true;
  } else {
    CK(cudaMemset(c->bias + (size_t)l * c->E, 0, sizeof(float) * c->E));
  }
  if (gain) {
    CK(cudaMemcpy(c->gain + (size_t)l * c->H, gain, sizeof(float) * c->H, cudaMemcpyHostToDevice));
    c->has_gain = true;
  } else {
    std::vector<float> ones(c->H, 1.0f);
    CK(cudaMemcpy(c->gain + (size_t)l * c->H, ones.data(), sizeof(float) * c->H, cudaMemcpyHostToDevice));
  }
  c->loaded[l] = 1;
  c->resident = false;
  drop_graphs(c);
  return MOE_OK;
}

int moe_create(const moe_config* cfg_in, const moe_weights* w, moe_ctx** out) {
  if (!cfg_in || !out) return MOE_ERR_INVALID;
  moe_config cfg = *cfg_in;
  if (cfg.n_layers < 1 || cfg.hidden < 32 || cfg.hidden % 32 || cfg.hidden > kMaxH) return MOE_ERR_INVALID;
  if (cfg.top_k < 1 || cfg.top_k > kMaxK || cfg.n_experts < cfg.top_k || cfg.n_experts > kMaxE)
    return MOE_ERR_INVALID;
  if (cfg.inter < 32 || cfg.inter % 32 || cfg.shared_inter < 0 || cfg.shared_inter % 32) return MOE_ERR_INVALID;
  if (cfg.ring_slots < 0 || cfg.ring_slots > kMaxR) return MOE_ERR_INVALID;
  if (cfg.use_rmsnorm != 0 && cfg.use_rmsnorm != 1) return MOE_ERR_INVALID;
  if (!(cfg.rms_eps >= 0.0f)) return MOE_ERR_INVALID;
  if (cfg.log_steps < 0) return MOE_ERR_INVALID;
  if (cfg.log_steps == 0) cfg.log_steps = 4096;
  if (cfg.wait_timeout_ms == 0) cfg.wait_timeout_ms = 2000;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || cfg.device < 0 || cfg.device >= ndev) return MOE_ERR_INVALID;

  moe_ctx* c = new (std::nothrow) moe_ctx();
  if (!c) return MOE_ERR_NOMEM;
  c->cfg = cfg;
  c->L = cfg.n_layers;
  c->H = cfg.hidden;
  c->E = cfg.n_experts;
  c->K = cfg.top_k;
  c->I = cfg.inter;
  c->Is = cfg.shared_inter;
  c->R = cfg.ring_slots;
  c->lay = slot_layout(c->H, c->I);
  c->slay = slot_layout(c->H, c->Is > 0 ? c->Is : 32);
  c->slot_bytes = c->lay.bytes;
  c->shared_slot_bytes = c->Is > 0 ? c->slay.bytes : 0;
  c->log_steps = cfg.log_steps;
  c->loaded.assign(c->L, 0);
  int st = MOE_OK;
  auto fail = [&](int s) {
    moe_destroy(c);
    return s;
  };
#define CKC(call)                                       \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return fail(cuda_fail(e_));  \
  } while (0)
  CKC(cudaSetDevice(cfg.device));
  CKC(cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, cfg.device));
  int smem_optin = 0, coop = 0;
  CKC(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, cfg.device));
  CKC(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, cfg.device));
  c->grid = c->nsm;  // one persistent CTA per SM
  if (!coop || !decode_plan(c->H, c->E, c->grid, smem_optin, &c->rx, &c->down_late, &c->smem))
    return fail(MOE_ERR_UNSUPPORTED);
  CKC(decode_configure(smem_optin));
  int per_sm = 0;
  CKC(decode_max_blocks_per_sm(c->H, c->smem, &per_sm));
  if (per_sm < 1) return fail(MOE_ERR_UNSUPPORTED);

  CKC(dalloc(&c->router_rows, (size_t)c->L * c->E * c->H));
  CKC(dalloc(&c->wnorm, c->L));
  CKC(dalloc(&c->bias, (size_t)c->L * c->E));
  CKC(dalloc(&c->gain, (size_t)c->L * c->H));
  if (c->Is > 0) CKC(dalloc(&c->shared_pool, (size_t)c->L * c->shared_slot_bytes));
  CKC(dalloc(&c->pin_slot, (size_t)c->L * c->E));
  CKC(dalloc(&c->layer_base, c->L));
  CKC(dalloc(&c->n_pinned, c->L));
  CKC(dalloc(&c->ring_owner, (size_t)2 * c->L * std::max(c->R, 1)));
  CKC(dalloc(&c->ring_stamp, (size_t)2 * c->L * std::max(c->R, 1)));
  CKC(dalloc(&c->ring_clock, (size_t)2 * c->L));
  CKC(dalloc(&c->acc, (size_t)kAccBufs * c->H));
  CKC(dalloc(&c->zll, c->E));
  CKC(dalloc(&c->likely, (size_t)2 * c->L * kMaxLikely));
  CKC(dalloc(&c->hist, (size_t)c->L * c->E));
  CKC(dalloc(&c->log, (size_t)c->log_steps * c->L * c->K * 7));
  CKC(dalloc(&c->ctrl, 1));
  CKC(dalloc(&c->done_seq, 1));
  CKC(dalloc(&c->x_buf, c->H));
  CKC(dalloc(&c->y_buf, c->H));
  CKC(cudaMemset(c->hist, 0, sizeof(uint32_t) * c->L * c->E));
  CKC(cudaMemset(c->ctrl, 0, sizeof(Ctrl)));
  CKC(cudaMemset(c->done_seq, 0, sizeof(uint32_t)));
  CKC(cudaMemset(c->acc, 0, sizeof(unsigned long long) * kAccBufs * c->H));
  CKC(cudaMemset(c->zll, 0, sizeof(unsigned long long) * c->E));
  CKC(cudaHostAlloc((void**)&c->host_tier, (size_t)c->L * c->E * c->slot_bytes,
                    cudaHostAllocPortable | cudaHostAllocMapped));
  {
    void* dp = nullptr;
    CKC(cudaHostGetDevicePointer(&dp, c->host_tier, 0));
    c->host_tier_dev = static_cast<const uint8_t*>(dp);
  }
  CKC(cudaHostAlloc((void**)&c->x_pin, sizeof(float) * c->H, cudaHostAllocPortable));
  CKC(cudaHostAlloc((void**)&c->y_pin, sizeof(float) * c->H, cudaHostAllocPortable));
  CKC(cudaHostAlloc((void**)&c->err_pin, sizeof(int32_t), cudaHostAllocPortable));
  CKC(cudaHostAlloc((void**)&c->mbox_host, sizeof(MissReq) * kMboxCap, cudaHostAllocMapped | cudaHostAllocPortable));
  memset(c->mbox_host, 0, sizeof(MissReq) * kMboxCap);
  CKC(cudaHostGetDevicePointer((void**)&c->mbox_dev, c->mbox_host, 0));
  CKC(cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking));
  CKC(cudaStreamCreateWithFlags(&c->own, cudaStreamNonBlocking));
  {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    CKC(cudaGetDriverEntryPointByVersion("cuStreamWriteValue32", &fn, 12000, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return fail(MOE_ERR_UNSUPPORTED);
    c->write_value32 = (PfnWriteValue32)fn;
  }
  for (int t = 0; t < moe_ctx::kCopyTimers; ++t) {
    CKC(cudaEventCreate(&c->ev_start[t]));
    CKC(cudaEventCreate(&c->ev_end[t]));
    c->timer_free.push_back(t);
  }
  c->proxy = std::thread(proxy_main, c);
  if (w) {
    if (!w->expert_q4_0 || !w->router_bf16 || (c->Is > 0 && !w->shared_q4_0)) return fail(MOE_ERR_INVALID);
    for (int l = 0; l < c->L; ++l) {
      st = moe_load_layer(c, l, w->expert_q4_0 + (size_t)l * c->E, c->Is > 0 ? w->shared_q4_0[l] : nullptr,
                          w->router_bf16 + (size_t)l * c->E * c->H,
                          w->router_bias ? w->router_bias + (size_t)l * c->E : nullptr,
                          w->rms_gain ? w->rms_gain + (size_t)l * c->H : nullptr);
      if (st != MOE_OK) return fail(st);
    }
  }
#undef CKC
  *out = c;
  return MOE_OK;
}

int moe_set_residency(moe_ctx* c, float fraction, const uint32_t* hist, int32_t placement) {
  if (!c || !(fraction >= 0.0f && fraction <= 1.0f)) return MOE_ERR_INVALID;
  if (placement != MOE_PLACE_CALIBRATED && placement != MOE_PLACE_UNIFORM) return MOE_ERR_INVALID;
  for (int l = 0; l < c->L; ++l)
    if (!c->loaded[l]) return MOE_ERR_STATE;
  const int P = (int)std::lround((double)fraction * c->E);
  if (P < c->E && c->R == 0) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  std::vector<uint32_t> h((size_t)c->L * c->E, 0);
  if (hist) {
    memcpy(h.data(), hist, h.size() * sizeof(uint32_t));
  } else {
    CK(cudaMemcpy(h.data(), c->hist, h.size() * sizeof(uint32_t), cudaMemcpyDeviceToHost));
  }
  // slot pool: per layer P pinned + R ring slots, then k staging slots
  const int64_t need = (int64_t)c->L * (P + c->R) + c->K;
  if (need > c->pool_slots) {
    drop_graphs(c);
    uint8_t* old = c->pool.exchange(nullptr);
    if (old) cudaFree(old);
    c->pool_slots = 0;
    uint8_t* np = nullptr;
    CK(cudaMalloc((void**)&np, (size_t)need * c->slot_bytes));
    c->pool.store(np);
    c->pool_slots = need;
  }
  uint8_t* pool = c->pool.load();
  std::vector<int32_t> pin((size_t)c->L * c->E, -1), base(c->L), npin(c->L, P);
  c->phys_owner.assign((size_t)c->L * std::max(P, 1), -1);
  std::vector<uint8_t> mask(c->E);
  for (int l = 0; l < c->L; ++l) {
    base[l] = l * (P + c->R);
    top_p_mask(h.data() + (size_t)l * c->E, c->E, P, placement, mask.data());
    int p = 0;
    for (int e = 0; e < c->E; ++e)
      if (mask[e]) {  // logical slot == physical slot == rank in ascending expert order
        pin[(size_t)l * c->E + e] = (p << 16) | p;
        c->phys_owner[(size_t)l * std::max(P, 1) + p] = e;
        CK(cudaMemcpyAsync(pool + (size_t)(base[l] + p) * c->slot_bytes,
                           c->host_tier + ((size_t)l * c->E + e) * c->slot_bytes, c->slot_bytes,
                           cudaMemcpyHostToDevice, c->own));
        ++p;
      }
  }
  c->pin_host = pin;
  c->repins = c->repin_copies = 0;
  c->score = h;  // the histogram this placement came from seeds the recalibration score
  c->hist_snap.assign((size_t)c->L * c->E, 0);
  CK(cudaMemcpyAsync(c->hist_snap.data(), c->hist, c->hist_snap.size() * 4, cudaMemcpyDeviceToHost, c->own));
  c->staging_base = c->L * (P + c->R);
  CK(cudaMemcpyAsync(c->pin_slot, pin.data(), pin.size() * 4, cudaMemcpyHostToDevice, c->own));
  CK(cudaMemcpyAsync(c->layer_base, base.data(), base.size() * 4, cudaMemcpyHostToDevice, c->own));
  CK(cudaMemcpyAsync(c->n_pinned, npin.data(), npin.size() * 4, cudaMemcpyHostToDevice, c->own));
  const size_t nr = (size_t)2 * c->L * std::max(c->R, 1);
  CK(cudaMemsetAsync(c->ring_owner, 0xff, nr * 4, c->own));
  CK(cudaMemsetAsync(c->ring_stamp, 0, nr * 4, c->own));
  CK(cudaMemsetAsync(c->ring_clock, 0, (size_t)2 * c->L * 4, c->own));
  CK(cudaStreamSynchronize(c->own));
  c->P = P;
  c->residency = fraction;
  c->placement = placement;
  c->resident = true;
  drop_graphs(c);
  return upload_likely(c, c->own);
}

int moe_decode_step(moe_ctx* c, const float* x_dev, float* y_dev, void* stream) {
  if (!c || !x_dev || !y_dev) return MOE_ERR_INVALID;
  if (!c->resident) return MOE_ERR_STATE;
  if (!c->g_dev) {
    const int st = capture_token(c, x_dev, y_dev, false, &c->g_dev, &c->gr_dev, &c->kn_dev);
    if (st != MOE_OK) return st;
    c->g_x = x_dev;
    c->g_y = y_dev;
  } else if (c->g_x != x_dev || c->g_y != y_dev) {
    // other buffers: the same graph with the kernel node's x / y updated in place
    DecodeParams p = make_params(c, x_dev, y_dev);
    cudaKernelNodeParams kp;
    CK(cudaGraphKernelNodeGetParams(c->kn_dev, &kp));
    void* args[1] = {&p};
    kp.kernelParams = args;
    kp.extra = nullptr;
    CK(cudaGraphExecKernelNodeSetParams(c->g_dev, c->kn_dev, &kp));
    c->g_x = x_dev;
    c->g_y = y_dev;
  }
  CK(cudaGraphLaunch(c->g_dev, (cudaStream_t)stream));
  return MOE_OK;
}

int moe_decode_step_host(moe_ctx* c, const float* x_host, float* y_host) {
  if (!c || !x_host || !y_host) return MOE_ERR_INVALID;
  if (!c->resident) return MOE_ERR_STATE;
  if (!c->g_host) {
    const int st = capture_token(c, c->x_buf, c->y_buf, true, &c->g_host);
    if (st != MOE_OK) return st;
  }
  memcpy(c->x_pin, x_host, sizeof(float) * c->H);
  CK(cudaGraphLaunch(c->g_host, c->own));
  CK(cudaStreamSynchronize(c->own));
  memcpy(y_host, c->y_pin, sizeof(float) * c->H);
  return deverr_status(*c->err_pin);
}

// Carve the prefill scratch for T tokens out of one allocation (256-byte aligned parts).
static int prefill_reserve(moe_ctx* c, int T) {
  if (T <= c->prefill_cap) return MOE_OK;
  CK(cudaDeviceSynchronize());
  if (c->prefill_mem) cudaFree(c->prefill_mem);
  c->prefill_mem = nullptr;
  c->prefill_cap = 0;
  const size_t H = c->H, K = c->K, E = c->E, imax = std::max(c->I, c->Is);
  const size_t R = (size_t)T * K + (c->Is > 0 ? (size_t)T : 0);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += (bytes + 255) / 256 * 256;
    return at;
  };
  const size_t o_h = take((size_t)T * H * 4), o_sel = take((size_t)T * K * 4), o_w = take((size_t)T * K * 4),
               o_xh = take((size_t)T * H * 2), o_xl = take((size_t)T * H * 2), o_gh = take(R * H * 2),
               o_u = take((size_t)T * H * 4), o_ua = take((size_t)T * 3 * H * 2), o_inv = take((size_t)T * 4),
               o_un = take((size_t)T * 4), o_part = take((size_t)8 * T * E * 4),
               o_gl = take(R * H * 2), o_ah = take(R * imax * 2), o_al = take(R * imax * 2),
               o_ob = take(R * H * 4), o_gp = take((size_t)T * (K + 1) * 4), o_cnt = take(E * 4),
               o_cur = take((E + 1) * 4),
               o_off = take((E + 2) * 4), o_jobs = take((R / 128 + E + 2) * 4),
               o_nj = take(4);
  uint8_t* m = nullptr;
  CK(cudaMalloc((void**)&m, off));
  c->prefill_mem = m;
  c->prefill_cap = T;
  PrefillScratch& s = c->pf;
  s.h = reinterpret_cast<float*>(m + o_h);
  s.sel = reinterpret_cast<int32_t*>(m + o_sel);
  s.w = reinterpret_cast<float*>(m + o_w);
  s.u = reinterpret_cast<float*>(m + o_u);
  s.ua = reinterpret_cast<__nv_bfloat16*>(m + o_ua);
  s.inv = reinterpret_cast<float*>(m + o_inv);
  s.unorm = reinterpret_cast<float*>(m + o_un);
  s.part = reinterpret_cast<float*>(m + o_part);
  s.x_hi = reinterpret_cast<__half*>(m + o_xh);
  s.x_lo = reinterpret_cast<__half*>(m + o_xl);
  s.xg_hi = reinterpret_cast<__half*>(m + o_gh);
  s.xg_lo = reinterpret_cast<__half*>(m + o_gl);
  s.a_hi = reinterpret_cast<__half*>(m + o_ah);
  s.a_lo = reinterpret_cast<__half*>(m + o_al);
  s.obuf = reinterpret_cast<float*>(m + o_ob);
  s.gpos = reinterpret_cast<int32_t*>(m + o_gp);
  s.counts = reinterpret_cast<int32_t*>(m + o_cnt);
  s.cursor = reinterpret_cast<int32_t*>(m + o_cur);
  s.offsets = reinterpret_cast<int32_t*>(m + o_off);
  s.jobs = reinterpret_cast<int32_t*>(m + o_jobs);
  s.n_jobs = reinterpret_cast<int32_t*>(m + o_nj);
  return MOE_OK;
}

int moe_prefill(moe_ctx* c, const float* x_dev, int32_t n_tokens, float* y_dev, void* stream) {
  if (!c || !x_dev || !y_dev || n_tokens < 1 || n_tokens > (1 << 20)) return MOE_ERR_INVALID;
  if (!c->resident || c->P != c->E) return MOE_ERR_STATE;
  if (!prefill_supported(c->H, c->E, c->K, c->I, c->Is)) return MOE_ERR_UNSUPPORTED;
  CK(cudaSetDevice(c->cfg.device));
  if (!c->prefill_configured) {
    CK(prefill_configure(c->H, c->E));
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    CK(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return MOE_ERR_UNSUPPORTED;
    c->encode_tiled = fn;
    c->prefill_configured = true;
  }
  const int st = prefill_reserve(c, n_tokens);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // one captured graph per pass (x copy-in, then every layer's launches), replayed while
  // the tokens, buffers, trace and slot pool stay the same
  if (c->g_pf && c->gpf_x == x_dev && c->gpf_y == y_dev && c->gpf_T == n_tokens && c->gpf_ht == c->pf_h_trace &&
      c->gpf_st == c->pf_sel_trace && c->gpf_pool == c->pool.load() && c->gpf_mem == c->prefill_mem) {
    CK(cudaGraphLaunch(c->g_pf, s));
    return MOE_OK;
  }
  if (c->g_pf) cudaGraphExecDestroy(c->g_pf);
  c->g_pf = nullptr;
  PrefillScratch sc = c->pf;
  sc.y = y_dev;
  sc.h_trace = c->pf_h_trace;
  sc.sel_trace = c->pf_sel_trace;
  sc.error = &c->ctrl->error;
  PrefillArgs a{};
  a.L = c->L;
  a.H = c->H;
  a.E = c->E;
  a.K = c->K;
  a.I = c->I;
  a.Is = c->Is;
  a.use_norm = c->cfg.use_rmsnorm;
  a.T = n_tokens;
  a.n_sm = c->nsm;
  a.eps = c->cfg.rms_eps;
  a.pool = c->pool.load();
  a.pool_slots = c->pool_slots;
  a.slot_bytes = c->slot_bytes;
  a.lay = c->lay;
  a.slay = c->slay;
  a.shared_pool = c->shared_pool;
  a.shared_slot_bytes = c->shared_slot_bytes;
  a.bias = c->has_bias ? c->bias : nullptr;
  a.gain = c->gain;
  a.pin_slot = c->pin_slot;
  a.layer_base = c->layer_base;
  a.hist = c->hist;
  a.router_rows = c->router_rows;
  a.wnorm = c->wnorm;
  cudaGraph_t graph = nullptr;
  CK(cudaStreamBeginCapture(c->own, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = cudaMemcpyAsync(sc.h, x_dev, sizeof(float) * n_tokens * c->H, cudaMemcpyDeviceToDevice, c->own);
  const int r = e == cudaSuccess ? prefill_run(a, sc, c->encode_tiled, c->own) : (int)e;
  const cudaError_t e2 = cudaStreamEndCapture(c->own, &graph);
  if (r != 0 || e2 != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    if (r == -1) return MOE_ERR_UNSUPPORTED;
    return cuda_fail(r != 0 ? (cudaError_t)r : e2);
  }
  e = cudaGraphInstantiate(&c->g_pf, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) {
    c->g_pf = nullptr;
    return cuda_fail(e);
  }
  c->gpf_x = x_dev;
  c->gpf_y = y_dev;
  c->gpf_T = n_tokens;
  c->gpf_ht = c->pf_h_trace;
  c->gpf_st = c->pf_sel_trace;
  c->gpf_pool = c->pool.load();
  c->gpf_mem = c->prefill_mem;
  CK(cudaGraphLaunch(c->g_pf, s));
  return MOE_OK;
}

int moe_set_prefill_trace(moe_ctx* c, float* h_trace_dev, int32_t* sel_trace_dev) {
  if (!c) return MOE_ERR_INVALID;
  c->pf_h_trace = h_trace_dev;
  c->pf_sel_trace = sel_trace_dev;
  return MOE_OK;
}

int moe_sync(moe_ctx* c) {
  if (!c) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  int32_t err = 0;
  CK(cudaMemcpy(&err, &c->ctrl->error, sizeof(err), cudaMemcpyDeviceToHost));
  return deverr_status(err);
}

int moe_clear_error(moe_ctx* c) {
  if (!c) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  // let the proxy drain every request the failed launch published
  for (int spin = 0; spin < 2000; ++spin) {
    const uint32_t next = c->proxy_next.load();
    if (c->mbox_host[next % kMboxCap].seq != next) break;
    std::this_thread::sleep_for(std::chrono::microseconds(500));
  }
  CK(cudaStreamSynchronize(c->side));
  Ctrl ctl;
  CK(cudaMemcpy(&ctl, c->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
  const uint32_t last = c->proxy_next.load() - 1;
  ctl.req_seq = last;
  ctl.error = 0;
  ctl.bar_count = 0;  // (the graphs zero it before every launch too)
  CK(cudaMemcpy(c->ctrl, &ctl, sizeof(Ctrl), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(c->done_seq, &last, sizeof(uint32_t), cudaMemcpyHostToDevice));
  // published logits carry a per-launch epoch: a failed launch may leave some behind
  CK(cudaMemset(c->zll, 0, sizeof(unsigned long long) * c->E));
  const size_t nr = (size_t)2 * c->L * std::max(c->R, 1);
  CK(cudaMemset(c->ring_owner, 0xff, nr * 4));
  CK(cudaMemset(c->ring_stamp, 0, nr * 4));
  CK(cudaMemset(c->ring_clock, 0, (size_t)2 * c->L * 4));
  c->proxy_err.store(0);
  c->drop.store(0);
  return MOE_OK;
}

int moe_stats(moe_ctx* c, moe_stats_t* out, uint32_t* hist_out, moe_event* log_out, size_t log_cap,
              size_t* log_n, int32_t reset) {
  if (!c) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  Ctrl ctl;
  CK(cudaMemcpy(&ctl, c->ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost));
  if (out) {
    memset(out, 0, sizeof(*out));
    out->steps = ctl.step;
    out->pin_hits = ctl.pin_hits;
    out->ring_hits = ctl.ring_hits;
    out->misses = ctl.misses;
    out->evictions = ctl.evictions;
    out->accesses = ctl.pin_hits + ctl.ring_hits + ctl.misses;
    out->bytes_copied = ctl.misses * c->slot_bytes;
    out->staged_misses = ctl.staged;
    out->device_error = ctl.error;
    out->n_pinned = c->P;
    out->residency = c->residency;
    out->placement = c->placement;
    out->repins = c->repins;
    out->repin_copies = c->repin_copies;
    out->miss_requests = ctl.req_seq;
    out->miss_served = c->proxy_next.load() - 1;
    out->proxy_error = c->proxy_err.load();
    out->miss_path = c->miss_mode == kMissPull ? MOE_MISS_SM_PULL : MOE_MISS_COPY_ENGINE;
    out->pulled_misses = ctl.pulled;
  }
  harvest_copy_timers(c);
  if (out) {
    out->copies_timed = c->copies_timed;
    out->copy_ns_timed = c->copy_ns;
  }
  if (hist_out)
    CK(cudaMemcpy(hist_out, c->hist, sizeof(uint32_t) * c->L * c->E, cudaMemcpyDeviceToHost));
  const uint64_t step = ctl.step;
  if (step > c->log_read_step + (uint64_t)c->log_steps) {
    c->log_dropped += (step - c->log_read_step - c->log_steps) * (uint64_t)c->L * c->K;
    c->log_read_step = step - c->log_steps;
  }
  size_t n = 0;
  if (log_out) {
    const size_t per_step = (size_t)c->L * c->K;
    while (c->log_read_step < step && n + per_step <= log_cap) {
      const size_t slot = (size_t)(c->log_read_step % (uint64_t)c->log_steps);
      CK(cudaMemcpy(log_out + n, c->log + slot * per_step * 7, per_step * sizeof(moe_event),
                    cudaMemcpyDeviceToHost));
      n += per_step;
      ++c->log_read_step;
    }
  }
  if (log_n) *log_n = n;
  if (out) out->log_dropped = c->log_dropped;
  if (reset) {
    ctl.pin_hits = ctl.ring_hits = ctl.misses = ctl.evictions = ctl.staged = ctl.pulled = 0;
    CK(cudaMemcpy(&c->ctrl->pin_hits, &ctl.pin_hits, 6 * sizeof(unsigned long long), cudaMemcpyHostToDevice));
    CK(cudaMemset(c->hist, 0, sizeof(uint32_t) * c->L * c->E));
    std::fill(c->hist_snap.begin(), c->hist_snap.end(), 0u);  // recalibration windows restart at 0
    c->copy_ns = c->copies_timed = 0;
  }
  return MOE_OK;
}

int moe_recalibrate(moe_ctx* c) {
  if (!c) return MOE_ERR_INVALID;
  if (!c->resident) return MOE_ERR_STATE;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  const size_t n = (size_t)c->L * c->E;
  std::vector<uint32_t> h(n);
  CK(cudaMemcpy(h.data(), c->hist, n * 4, cudaMemcpyDeviceToHost));
  for (size_t i = 0; i < n; ++i) {
    const uint32_t window = h[i] >= c->hist_snap[i] ? h[i] - c->hist_snap[i] : h[i];  // a reset restarts it
    c->score[i] = (c->score[i] >> 1) + window;
  }
  c->hist_snap = h;
  const int P = c->P, Pw = std::max(P, 1);
  uint8_t* pool = c->pool.load();
  std::vector<uint8_t> mask(c->E);
  std::vector<int> freed, entering;
  for (int l = 0; l < c->L; ++l) {
    top_p_mask(c->score.data() + (size_t)l * c->E, c->E, P, MOE_PLACE_CALIBRATED, mask.data());
    int32_t* row = c->pin_host.data() + (size_t)l * c->E;
    freed.clear();
    entering.clear();
    for (int e = 0; e < c->E; ++e) {
      if (row[e] >= 0 && !mask[e]) {
        freed.push_back(row[e] & 0xffff);
        row[e] = -1;
      } else if (row[e] < 0 && mask[e]) {
        entering.push_back(e);
      }
    }
    std::sort(freed.begin(), freed.end());
    for (size_t k = 0; k < entering.size(); ++k) {  // an entering expert takes a freed slot
      const int e = entering[k], ph = freed[k];
      row[e] = ph;
      c->phys_owner[(size_t)l * Pw + ph] = e;
      CK(cudaMemcpyAsync(pool + (size_t)(l * (P + c->R) + ph) * c->slot_bytes,
                         c->host_tier + ((size_t)l * c->E + e) * c->slot_bytes, c->slot_bytes,
                         cudaMemcpyHostToDevice, c->own));
      ++c->repin_copies;
    }
    int rank = 0;  // logical slots: ranks in ascending expert order
    for (int e = 0; e < c->E; ++e)
      if (row[e] >= 0) row[e] = (rank++ << 16) | (row[e] & 0xffff);
  }
  CK(cudaMemcpyAsync(c->pin_slot, c->pin_host.data(), n * 4, cudaMemcpyHostToDevice, c->own));
  const int st = empty_rings(c, c->own);
  if (st != MOE_OK) return st;
  CK(cudaStreamSynchronize(c->own));
  ++c->repins;
  return upload_likely(c, c->own);
}

int moe_set_prefetch(moe_ctx* c, int32_t n_preload, int32_t n_l2) {
  if (!c || n_preload < 0 || n_l2 < 0 || n_preload > std::min(c->K, kMaxPreload) || n_preload + n_l2 > kMaxLikely)
    return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  // the preload needs one CTA per unit (a CTA guessing wrong takes another unit)
  const int n_units = c->K * (c->I / 32) + c->Is / 32;
  c->n_pre = c->grid >= n_units ? n_preload : 0;
  c->n_l2 = n_l2;
  drop_graphs(c);
  return c->resident ? upload_likely(c, c->own) : MOE_OK;
}

int moe_set_router_bias(moe_ctx* c, int32_t layer, const float* bias) {
  if (!c || layer < 0 || layer >= c->L) return MOE_ERR_INVALID;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  if (bias) {
    CK(cudaMemcpy(c->bias + (size_t)layer * c->E, bias, sizeof(float) * c->E, cudaMemcpyHostToDevice));
  } else {
    CK(cudaMemset(c->bias + (size_t)layer * c->E, 0, sizeof(float) * c->E));
  }
  if (bias && !c->has_bias) {
    c->has_bias = true;  // the kernel now reads the bias table: recapture
    drop_graphs(c);
  }
  return MOE_OK;
}

int moe_set_trace(moe_ctx* c, float* h_trace_dev, float* w_trace_dev) {
  if (!c) return MOE_ERR_INVALID;
  c->h_trace = h_trace_dev;
  c->w_trace = w_trace_dev;
  drop_graphs(c);
  return MOE_OK;
}

int moe_set_phase_trace(moe_ctx* c, uint64_t* stamps_dev, size_t n_words) {
  if (!c) return MOE_ERR_INVALID;
  if (stamps_dev && n_words < phase_trace_words(c->L, c->grid)) return MOE_ERR_INVALID;
  c->phase_trace = reinterpret_cast<unsigned long long*>(stamps_dev);
  c->phase_trace_words = stamps_dev ? n_words : 0;
  drop_graphs(c);
  return MOE_OK;
}

int moe_set_miss_path(moe_ctx* c, int32_t mode) {
  if (!c || (mode != MOE_MISS_COPY_ENGINE && mode != MOE_MISS_SM_PULL)) return MOE_ERR_INVALID;
  const int m = mode == MOE_MISS_SM_PULL ? kMissPull : kMissProxy;
  if (m != c->miss_mode) {
    CK(cudaSetDevice(c->cfg.device));
    CK(cudaDeviceSynchronize());
    c->miss_mode = m;
    drop_graphs(c);
  }
  return MOE_OK;
}

int moe_measure_h2d(moe_ctx* c, int32_t n_copies, double* gbs) {
  if (!c || n_copies < 1 || !gbs) return MOE_ERR_INVALID;
  if (!c->resident) return MOE_ERR_STATE;
  CK(cudaSetDevice(c->cfg.device));
  CK(cudaDeviceSynchronize());
  uint8_t* pool = c->pool.load();
  cudaEvent_t a = nullptr, b = nullptr;
  CK(cudaEventCreate(&a));
  cudaError_t e = cudaEventCreate(&b);
  const size_t n_src = (size_t)c->L * c->E;
  for (int pass = 0; pass < 2 && e == cudaSuccess; ++pass) {  // pass 0 warms the path up
    if (pass == 1) e = cudaEventRecord(a, c->side);
    for (int i = 0; i < n_copies && e == cudaSuccess; ++i) {
      const size_t src = ((size_t)i * 7919) % n_src;  // spread over the tier
      e = cudaMemcpyAsync(pool + (size_t)(c->staging_base + i % c->K) * c->slot_bytes,
                          c->host_tier + src * c->slot_bytes, c->slot_bytes, cudaMemcpyHostToDevice, c->side);
    }
    if (pass == 1 && e == cudaSuccess) e = cudaEventRecord(b, c->side);
  }
  float ms = 0.0f;
  if (e == cudaSuccess) e = cudaEventSynchronize(b);
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e != cudaSuccess) return cuda_fail(e);
  *gbs = (double)n_copies * (double)c->slot_bytes / ((double)ms * 1e-3) / 1e9;
  return MOE_OK;
}

int moe_debug_drop_signals(moe_ctx* c, int32_t n) {
  if (!c || n < 0) return MOE_ERR_INVALID;
  c->drop.store(n);
  return MOE_OK;
}

}  // extern "C"
