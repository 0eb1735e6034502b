// moe_noalloc.cu -- moe_decode_step_noalloc: the decode kernel with its scratch in a
// static device array, for callers that cannot allocate device memory.
//
// Everything the kernel writes besides y lives in g_scratch: the control block (arrival
// counter, error word, counters), the output accumulators, the published logit words,
// the slot tables of a fully resident model, the routing histogram and one step of event
// log.  The array is carved per call from the shape; nothing is allocated.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe_cache.h"
#include "moe_internal.h"

namespace moe {
bool decode_plan(int H, int E, int grid, int smem_optin, int* rx, int* down_late, uint32_t* smem);
cudaError_t decode_configure(int limit);
cudaError_t decode_launch(const DecodeParams& p, int grid, cudaStream_t stream);
}  // namespace moe

using namespace moe;

constexpr size_t kScratchBytes = 2u << 20;  // 2 MiB per device

// The scratch array.  In host code this name is only a stand-in for the symbol, not a
// device address: the address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_mu;
uint8_t* g_addr[kMaxDevices];  // device address of g_scratch, per device
bool g_configured[kMaxDevices];  // kernel shared-memory limit raised to the device maximum

struct Carve {
  size_t ctrl, acc, zll, pin, base, npin, rown, rstamp, rclock, done, reset_end, hist, log, total;
};

// Everything a step depends on comes first and is reset by every call (one memset);
// the histogram and log after it are only written by the kernel.
Carve carve(int L, int H, int E, int K) {
  Carve c{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = (off + 255) / 256 * 256;
    const size_t r = off;
    off += bytes;
    return r;
  };
  c.ctrl = take(sizeof(Ctrl));
  c.acc = take(8u * kAccBufs * (size_t)H);
  c.zll = take(8u * (size_t)E);
  c.pin = take(4u * (size_t)L * E);
  c.base = take(4u * L);
  c.npin = take(4u * L);
  c.rown = take(4u * 2 * L);
  c.rstamp = take(4u * 2 * L);
  c.rclock = take(4u * 2 * L);
  c.done = take(4u);
  c.reset_end = off;
  c.hist = take(4u * (size_t)L * E);
  c.log = take(4u * 7 * (size_t)L * K);
  c.total = off;
  return c;
}

// Slot tables of a fully resident model: expert e of layer l is slot l * E + e.
__global__ void resident_tables(int32_t* pin, int32_t* base, int32_t* npin, int L, int E) {
  const int n = L * E;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
    pin[t] = ((t % E) << 16) | (t % E);  // logical slot == physical slot == expert
    if (t % E == 0) {
      base[t / E] = t;
      npin[t / E] = E;
    }
  }
}

}  // namespace

extern "C" int moe_decode_step_noalloc(const moe_config* cfg, const moe_noalloc_weights* w,
                                       const float* x_dev, float* y_dev, void* stream) {
  if (!cfg || !w || !x_dev || !y_dev || !w->experts_dev || !w->router_dev) return MOE_ERR_INVALID;
  const int L = cfg->n_layers, H = cfg->hidden, E = cfg->n_experts, K = cfg->top_k, I = cfg->inter,
            Is = cfg->shared_inter;
  if (L < 1 || H < 32 || H % 32 || H > kMaxH || K < 1 || K > kMaxK || E < K || E > kMaxE) return MOE_ERR_INVALID;
  if (I < 32 || I % 32 || Is < 0 || Is % 32 || (Is > 0 && !w->shared_dev)) return MOE_ERR_INVALID;
  if ((cfg->use_rmsnorm != 0 && cfg->use_rmsnorm != 1) || !(cfg->rms_eps >= 0.0f)) return MOE_ERR_INVALID;
  const Carve cv = carve(L, H, E, K);
  if (cv.total > kScratchBytes) return MOE_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != cfg->device || dev < 0 || dev >= kMaxDevices)
    return MOE_ERR_INVALID;
  int nsm = 0, optin = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  int rx = 0, down_late = 0;
  uint32_t smem = 0;
  if (!decode_plan(H, E, nsm, optin, &rx, &down_late, &smem)) return MOE_ERR_UNSUPPORTED;
  uint8_t* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {  // first call on this device: where the array lives there
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
      g_addr[dev] = static_cast<uint8_t*>(ptr);
    }
    if (!g_configured[dev]) {  // every kernel instance, up to the device's limit
      if (decode_configure(optin) != cudaSuccess) return MOE_ERR_CUDA;
      g_configured[dev] = true;
    }
    base = g_addr[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  DecodeParams p{};
  p.L = L;
  p.H = H;
  p.E = E;
  p.K = K;
  p.I = I;
  p.Is = Is;
  p.R = 0;
  p.use_norm = cfg->use_rmsnorm;
  p.eps = cfg->rms_eps;
  p.n_units = K * (I / 32) + Is / 32;
  p.rx_per_cta = rx;
  p.down_late = down_late;
  p.miss_mode = kMissProxy;  // never used: every expert is resident
  p.nan_on_error = 1;        // no moe_sync here: a failed step shows as NaN outputs
  p.pool = w->experts_dev;
  p.slot_bytes = slot_layout(H, I).bytes;
  p.unit_bytes = slot_layout(H, I).unit;
  p.shared_pool = w->shared_dev;
  p.shared_slot_bytes = Is > 0 ? slot_layout(H, Is).bytes : 0;
  p.router = w->router_dev;
  p.bias = w->bias_dev;
  p.gain = w->gain_dev;
  p.pin_slot = reinterpret_cast<const int32_t*>(base + cv.pin);
  p.layer_base = reinterpret_cast<const int32_t*>(base + cv.base);
  p.n_pinned = reinterpret_cast<const int32_t*>(base + cv.npin);
  p.ring_owner = reinterpret_cast<int32_t*>(base + cv.rown);
  p.ring_stamp = reinterpret_cast<uint32_t*>(base + cv.rstamp);
  p.ring_clock = reinterpret_cast<uint32_t*>(base + cv.rclock);
  p.staging_base = 0;
  p.x = x_dev;
  p.y = y_dev;
  p.h_trace = nullptr;
  p.w_trace = nullptr;
  p.acc = reinterpret_cast<unsigned long long*>(base + cv.acc);
  p.zll = reinterpret_cast<unsigned long long*>(base + cv.zll);
  p.hist = reinterpret_cast<uint32_t*>(base + cv.hist);
  p.log = reinterpret_cast<int32_t*>(base + cv.log);
  p.log_steps = 1;
  p.ctrl = reinterpret_cast<Ctrl*>(base + cv.ctrl);
  p.mbox = nullptr;
  p.done_seq = reinterpret_cast<const uint32_t*>(base + cv.done);
  p.host_tier = nullptr;
  p.timeout_ns = (unsigned long long)(cfg->wait_timeout_ms ? cfg->wait_timeout_ms : 2000) * 1000000ull;
  p.phase_trace = nullptr;
  p.likely_slot = nullptr;
  p.likely_e = nullptr;
  p.n_pre = 0;
  p.n_l2 = 0;

  // a clean start every call: control block (step 0, no error, counter 0), accumulators,
  // logit words and tables
  if (cudaMemsetAsync(base, 0, cv.reset_end, st) != cudaSuccess) return MOE_ERR_CUDA;
  resident_tables<<<(L * E + 255) / 256, 256, 0, st>>>(reinterpret_cast<int32_t*>(base + cv.pin),
                                                       reinterpret_cast<int32_t*>(base + cv.base),
                                                       reinterpret_cast<int32_t*>(base + cv.npin), L, E);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (decode_launch(p, nsm, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
