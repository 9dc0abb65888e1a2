// Per-device runtime state of the library (host code): SM count and a private
// stream-ordered memory pool for the prefill's scratch.  The pool keeps its
// memory between calls (release threshold = everything), so a steady stream of
// calls does not go back to the driver.
#include <mutex>
#include <vector>

#include "kda_common.cuh"
#include "segments.cuh"

namespace kda {
namespace {

struct DeviceCtx {
  bool init = false, pool_init = false;
  int sms = 148;
  cudaMemPool_t pool = nullptr;
};
std::mutex g_mu;
DeviceCtx g_ctx[64];

}  // namespace

bool device_ctx(int* sms, cudaMemPool_t* pool) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceCtx& d = g_ctx[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    d.init = true;
  }
  if (pool && !d.pool_init) {     // the pool is created on first use
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&d.pool, &props) == cudaSuccess) {
      uint64_t keep = UINT64_MAX;
      cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
    } else {
      d.pool = nullptr;
      (void)cudaGetLastError();
    }
    d.pool_init = true;
  }
  if (sms) *sms = d.sms;
  if (pool) *pool = d.pool;
  return true;
}

int pool_used_high(bool reset, unsigned long long* used_high) {
  int sms = 0;
  cudaMemPool_t pool = nullptr;
  if (!device_ctx(&sms, &pool) || !pool) return KDA_ERR_CUDA;
  uint64_t v = 0;
  if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &v) != cudaSuccess) {
    (void)cudaGetLastError();
    return KDA_ERR_CUDA;
  }
  *used_high = (unsigned long long)v;
  if (reset) {
    uint64_t zero = 0;
    if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero) != cudaSuccess) {
      (void)cudaGetLastError();
      return KDA_ERR_CUDA;
    }
  }
  return KDA_OK;
}

bool once_per_device(int site, bool (*setup)()) {
  static std::mutex mu;
  static bool done[kOnceSites][64] = {};
  int dev = 0;
  if (site < 0 || site >= kOnceSites || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return false;
  std::lock_guard<std::mutex> lk(mu);
  if (!done[site][dev]) {
    if (!setup()) {
      (void)cudaGetLastError();
      return false;
    }
    done[site][dev] = true;
  }
  return true;
}

}  // namespace kda

// ---------------------------------------------------------------------------
// Per-kernel timing (kda_timing_*): events around each launch while enabled.
namespace kda {
namespace {

constexpr size_t kMaxTimed = 65536;
struct TimedLaunch {
  int kind;
  cudaEvent_t a, b;
};
struct Timing {
  std::mutex mu;
  bool on = false;
  std::vector<TimedLaunch> recs;
  std::vector<cudaEvent_t> pool;      // events released by kda_timing_start / stop
};
Timing g_timing;

cudaEvent_t take_event() {
  cudaEvent_t e = nullptr;
  if (!g_timing.pool.empty()) {
    e = g_timing.pool.back();
    g_timing.pool.pop_back();
    return e;
  }
  if (cudaEventCreate(&e) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return e;
}
void release_all() {
  for (auto& r : g_timing.recs) {
    g_timing.pool.push_back(r.a);
    g_timing.pool.push_back(r.b);
  }
  g_timing.recs.clear();
}

}  // namespace

int timing_begin(int kind, cudaStream_t stream) {
  if (!g_timing.on) return -1;
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (!g_timing.on || g_timing.recs.size() >= kMaxTimed) return -1;
  TimedLaunch t{kind, take_event(), take_event()};
  if (!t.a || !t.b || cudaEventRecord(t.a, stream) != cudaSuccess) {
    (void)cudaGetLastError();
    if (t.a) g_timing.pool.push_back(t.a);
    if (t.b) g_timing.pool.push_back(t.b);
    return -1;
  }
  g_timing.recs.push_back(t);
  return (int)g_timing.recs.size() - 1;
}

void timing_end(int handle, cudaStream_t stream) {
  if (handle < 0) return;
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if ((size_t)handle < g_timing.recs.size())
    if (cudaEventRecord(g_timing.recs[handle].b, stream) != cudaSuccess) (void)cudaGetLastError();
}

}  // namespace kda

extern "C" {

int kda_timing_start(void) {
  std::lock_guard<std::mutex> lk(kda::g_timing.mu);
  kda::release_all();
  kda::g_timing.on = true;
  return KDA_OK;
}

int kda_timing_stop(void) {
  std::lock_guard<std::mutex> lk(kda::g_timing.mu);
  kda::g_timing.on = false;
  return KDA_OK;
}

int kda_timing_read(int kind, unsigned long long* launches, double* total_ms) {
  if (kind < 0 || kind >= KDA_KERNEL_KINDS || !launches || !total_ms) return KDA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(kda::g_timing.mu);
  unsigned long long n = 0;
  double ms = 0.0;
  for (auto& r : kda::g_timing.recs) {
    if (r.kind != kind) continue;
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      (void)cudaGetLastError();
      return KDA_ERR_CUDA;
    }
    ++n;
    ms += t;
  }
  *launches = n;
  *total_ms = ms;
  return KDA_OK;
}

}  // extern "C"
