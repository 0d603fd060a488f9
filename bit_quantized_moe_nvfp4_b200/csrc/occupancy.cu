// occupancy.cu -- per-device launch facts shared by the kernel launchers: the SM count and
// how many blocks of a kernel fit on one SM, each looked up once and cached.
#include <atomic>
#include <mutex>
#include <vector>

#include "moe.cuh"

namespace nvfp4 {

// SM count of the current device, looked up once per device (devices may differ).
int num_sms() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cached[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = kNumSMs;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Blocks of kernel k that fit on one SM at once with this block size and shared memory,
// after raising the kernel's dynamic shared-memory limit to at least `smem`.  The limit is a
// per-kernel, per-device attribute that only ever grows here (a call with less memory must
// not lower it under a size another call still launches with), and the occupancy answer is
// cached per kernel, device, block size and memory, so a steady stream of calls pays for
// neither query again.
int resident_blocks_fn(const void *fn, int threads, size_t smem) {
  struct Limit {
    const void *fn;
    int dev;
    size_t smem;
  };
  struct Entry {
    const void *fn;
    int dev, threads;
    size_t smem;
    int nb;
  };
  static std::mutex mu;
  static std::vector<Limit> limits;
  static std::vector<Entry> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  Limit *lim = nullptr;
  for (Limit &l : limits)
    if (l.fn == fn && l.dev == dev) lim = &l;
  if (!lim || lim->smem < smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return -1;
    }
    if (lim)
      lim->smem = smem;
    else
      limits.push_back({fn, dev, smem});
  }
  for (const Entry &c : cache)
    if (c.fn == fn && c.dev == dev && c.threads == threads && c.smem == smem) return c.nb;
  int nb = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return -1;
  }
  if (cache.size() < 256) cache.push_back({fn, dev, threads, smem, nb});
  return nb;
}

}  // namespace nvfp4
