// Device twin of kv_cache_serving_ws_b200/synth.py: fills a bf16 tensor with
// the seeded synthetic N(0,1) values that the numpy generator gives for the
// same (key, flat index).  Input generation for the tests and the benchmark
// only (large caches are filled on the device); no attention, cache or Euler
// arithmetic.  Built into its own library, libws_synth.so.
//
// value(key, i) = vals[#{k : thr[k] <= r}],  r = top 32 bits of
// SplitMix64(key + (i + 1) * 0x9E3779B97F4A7C15)   (Steele, Lea, Flood 2014).
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/ws_synth.h"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxTable = 8192;
constexpr int kMaxDevices = 64;   // per-device kernel attribute flags

__device__ __forceinline__ uint32_t mix_top32(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z = z ^ (z >> 31);
  return static_cast<uint32_t>(z >> 32);
}

__global__ void __launch_bounds__(kThreads) fill_kernel(uint16_t* dst, int64_t n, uint64_t key, int64_t index0,
                                                        const uint64_t* thr, const uint16_t* vals, int len) {
  extern __shared__ uint8_t sm[];
  uint64_t* s_thr = reinterpret_cast<uint64_t*>(sm);
  uint16_t* s_val = reinterpret_cast<uint16_t*>(sm + sizeof(uint64_t) * len);
  for (int k = threadIdx.x; k < len; k += blockDim.x) {
    s_thr[k] = thr[k];
    s_val[k] = vals[k];
  }
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t idx = static_cast<uint64_t>(index0 + i);
    const uint64_t r = mix_top32(key + (idx + 1ull) * 0x9E3779B97F4A7C15ull);
    int lo = 0, hi = len;   // first k with thr[k] > r
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s_thr[mid] <= r) lo = mid + 1; else hi = mid;
    }
    dst[i] = s_val[lo < len ? lo : len - 1];
  }
}

}  // namespace

extern "C" int ws_synth_fill_normal_bf16(uint16_t* dst, int64_t n, uint64_t key, int64_t index0,
                                         const uint64_t* table_thr, const uint16_t* table_vals, int32_t table_len,
                                         cudaStream_t stream) {
  if (n < 0 || table_len < 1 || table_len > kMaxTable || index0 < 0) return -1;
  if (n == 0) return 0;
  if (!dst || !table_thr || !table_vals) return -1;
  const size_t smem = (sizeof(uint64_t) + sizeof(uint16_t)) * (size_t)table_len;
  // the shared-memory opt-in is a per-device attribute of the kernel
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -7;
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)((sizeof(uint64_t) + sizeof(uint16_t)) * kMaxTable)) != cudaSuccess)
      return -7;
    configured[dev].store(true, std::memory_order_release);
  }
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  int64_t blocks = (n + kThreads - 1) / kThreads;
  if (blocks > (int64_t)sms * 4) blocks = (int64_t)sms * 4;
  fill_kernel<<<(unsigned)blocks, kThreads, smem, stream>>>(dst, n, key, index0, table_thr, table_vals,
                                                           table_len);
  return cudaGetLastError() == cudaSuccess ? 0 : -7;
}
