// status.cu -- the per-device status word, device queries, and the bounded
// wait self-test kernel.
#include <cuda_runtime.h>

#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// One status word per device: 0 = OK, else the first sq_status a kernel
// recorded (atomicCAS from 0).  Read and cleared by sq_sync_status().
__device__ unsigned int g_sq_status = 0u;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
}  // namespace

unsigned int* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sq_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = (unsigned int*)p;
  }
  return g_status_ptr[dev];
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

// One thread initialises an mbarrier that expects one arrival which never
// comes, then waits on it with a limit: the wait runs out, the kernel records
// SQ_ERR_TIMEOUT and returns.  Nothing faults and nothing hangs.
__global__ void wait_selftest_kernel(int64_t limit_ns, unsigned int* status) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x != 0) return;
  const uint32_t addr = (uint32_t)__cvta_generic_to_shared(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(addr) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const uint64_t t0 = global_ns();
  bool done = false;
  while (!done) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(0u)
        : "memory");
    if (ok) break;
    if (global_ns() - t0 > (uint64_t)limit_ns) {
      set_status(status, kStatusTimeout);
      done = true;
    }
  }
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(addr) : "memory");
}

// One thread checks an offset equal to its (4-element) tensor's extent and
// touches no memory: a bounds-checked build records SQ_ERR_BOUNDS.
__global__ void bounds_selftest_kernel(unsigned int* status) {
  if (threadIdx.x == 0) (void)in_bounds(4, 1, 4, status);
}

cudaError_t launch_bounds_selftest(cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return cudaErrorInvalidDevice;
  bounds_selftest_kernel<<<1, 32, 0, st>>>(sw);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int64_t limit_ns, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return cudaErrorInvalidDevice;
  wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, sw);
  return cudaGetLastError();
}

}  // namespace sq
