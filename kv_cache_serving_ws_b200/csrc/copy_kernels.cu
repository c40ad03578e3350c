// In-place K/V cache writes and readback (HBM-bound, 16-byte vectors).
//
// Each incoming K/V slice is written straight into its slot of the
// preallocated cache ("Wan-Streamer v0.2：更高分辨率，相同延迟",
// paper.rainbus.top, section 前置知识, entry K/V缓存预分片; "Technical Summary:
// Wan-Streamer v0.2", gist.science, section Methodology, item 2).  The slice is
// token-major [L][n][H][D]; the cache is head-major, plane (l*2 + kv)*H + h
// holding rows [C*T][D], so that a head's keys are contiguous for the
// attention kernel's TMA tiles.  A thread owns one 16-byte vector position
// (head, column block) of a token row and walks the tokens; a warp reads 512
// contiguous source bytes per token and writes runs of D*2 contiguous bytes.
#include <cuda_runtime.h>

#include <atomic>

#include "kernels.cuh"

namespace ws {

namespace {

constexpr int kCopyThreads = 256;
constexpr int kTokUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// blockIdx.y = l*2 + kv (layer of the slice, K or V); blockIdx.x strides over tokens.
__global__ void __launch_bounds__(kCopyThreads) append_kernel(const __grid_constant__ AppendParams p) {
  griddep_wait();                 // the slice may come from the previous kernel of the stream
  griddep_launch_dependents();
  const int l = blockIdx.y >> 1;
  const int kv = blockIdx.y & 1;
  if (!index_ok(((int64_t)(p.layer0 + l) * 2 + kv + 1) * p.n_heads <= p.planes && p.row0 >= 0 &&
                    p.row0 + p.n_tokens <= p.plane_rows,
                p.status))
    return;
  const int vpr = p.head_dim >> 3;          // 16-byte vectors per head row
  const int row_vecs = p.n_heads * vpr;     // vectors per token
  const uint4* src = reinterpret_cast<const uint4*>(kv ? p.src_v : p.src_k) + (size_t)l * p.n_tokens * row_vecs;
  const int64_t plane0 = ((int64_t)(p.layer0 + l) * 2 + kv) * p.n_heads;
  for (int e = threadIdx.x; e < row_vecs; e += blockDim.x) {
    const int hh = e / vpr;
    const int vv = e - hh * vpr;
    const uint4* s = src + e;
    uint4* d = reinterpret_cast<uint4*>(p.cache + ((plane0 + hh) * p.plane_rows + p.row0) * p.head_dim) + vv;
    int t = blockIdx.x * kTokUnroll;
    const int step = gridDim.x * kTokUnroll;
    for (; t + kTokUnroll <= p.n_tokens; t += step) {
      uint4 v[kTokUnroll];
#pragma unroll
      for (int u = 0; u < kTokUnroll; ++u) v[u] = ld_stream(s + (size_t)(t + u) * row_vecs);
#pragma unroll
      for (int u = 0; u < kTokUnroll; ++u) d[(size_t)(t + u) * vpr] = v[u];
    }
  }
  // ragged tail: the last n_tokens % kTokUnroll tokens, handled by block 0
  const int tail0 = (p.n_tokens / kTokUnroll) * kTokUnroll;
  if (blockIdx.x == 0 && tail0 < p.n_tokens) {
    for (int e = threadIdx.x; e < row_vecs; e += blockDim.x) {
      const int hh = e / vpr;
      const int vv = e - hh * vpr;
      uint4* d = reinterpret_cast<uint4*>(p.cache + ((plane0 + hh) * p.plane_rows + p.row0) * p.head_dim) + vv;
      for (int t = tail0; t < p.n_tokens; ++t) d[(size_t)t * vpr] = ld_stream(src + e + (size_t)t * row_vecs);
    }
  }
}

// blockIdx.y = kv; copies rows row0 .. row0+n-1 of one layer back to [n][H][D].
__global__ void __launch_bounds__(kCopyThreads) read_kernel(const __grid_constant__ ReadParams p) {
  const int kv = blockIdx.y;
  if (!index_ok(((int64_t)p.layer * 2 + kv + 1) * p.n_heads <= p.planes && p.row0 >= 0 &&
                    p.row0 + p.n_tokens <= p.plane_rows,
                p.status))
    return;
  const int vpr = p.head_dim >> 3;
  const int row_vecs = p.n_heads * vpr;
  uint4* dst = reinterpret_cast<uint4*>(kv ? p.dst_v : p.dst_k);
  const int64_t plane0 = ((int64_t)p.layer * 2 + kv) * p.n_heads;
  for (int e = threadIdx.x; e < row_vecs; e += blockDim.x) {
    const int hh = e / vpr;
    const int vv = e - hh * vpr;
    const uint4* s =
        reinterpret_cast<const uint4*>(p.cache + ((plane0 + hh) * p.plane_rows + p.row0) * p.head_dim) + vv;
    for (int t = blockIdx.x; t < p.n_tokens; t += gridDim.x) dst[(size_t)t * row_vecs + e] = s[(size_t)t * vpr];
  }
}

}  // namespace

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int sm_count() {
  // one entry per device: a process may drive GPUs of different sizes
  static std::atomic<int> count[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return 148;
  int n = count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  if (p.n_tokens <= 0 || p.n_layers <= 0) return cudaSuccess;
  const int pairs = p.n_layers * 2;
  // enough blocks to fill the SMs several times over; each block walks tokens
  int gx = (p.n_tokens + kTokUnroll - 1) / kTokUnroll;
  const int want = sm_count() * 8;
  if (gx * pairs > want) gx = (want + pairs - 1) / pairs;
  if (gx < 1) gx = 1;
  dim3 grid(gx, pairs);
  PdlLaunch l(grid, dim3(kCopyThreads), 0, stream);
  return cudaLaunchKernelEx(&l.cfg, append_kernel, p);
}

cudaError_t launch_read(const ReadParams& p, cudaStream_t stream) {
  if (p.n_tokens <= 0) return cudaSuccess;
  int gx = p.n_tokens < 1024 ? p.n_tokens : 1024;
  dim3 grid(gx, 2);
  read_kernel<<<grid, kCopyThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ws
