// Host-side caches that keep per-call launch overhead low: the SM count of
// each device and the dynamic shared-memory limit already granted to each
// kernel on each device (cudaFuncSetAttribute is called only when a launch
// needs more than was granted before).
#include <cuda_runtime.h>

#include <map>
#include <tuple>
#include <mutex>
#include <utility>

#include "launch.h"

namespace misa {

namespace {
std::mutex g_mu;
std::map<int, int> g_sms;
std::map<std::pair<int, const void*>, int> g_smem;
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_sms.find(dev);
  if (it != g_sms.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  g_sms[dev] = n;
  return n;
}

cudaError_t ensure_dynamic_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(dev, func);
  auto it = g_smem.find(key);
  if (it != g_smem.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem[key] = bytes;
  return e;
}

int occupancy_blocks(const void* func, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  static std::map<std::tuple<int, const void*, int, size_t>, int> cache;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_tuple(dev, func, threads, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess || n < 1) n = 1;
  cache[key] = n;
  return n;
}

}  // namespace misa
