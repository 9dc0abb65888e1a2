// Per-device runtime state of the library (host code): SM count and a private
// stream-ordered memory pool for the prefill's scratch.  The pool keeps its
// memory between calls (release threshold = everything), so a steady stream of
// calls does not go back to the driver.
#include <mutex>

#include "kda_common.cuh"
#include "segments.cuh"

namespace kda {
namespace {

struct DeviceCtx {
  bool init = false;
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
    d.init = true;
  }
  if (sms) *sms = d.sms;
  if (pool) *pool = d.pool;
  return true;
}

}  // namespace kda
