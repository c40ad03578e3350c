// ws_attention_noalloc: the block-causal attention kernel for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is unavailable or forbidden --
// under a host framework that owns every device allocation through its own pool
// and hands out only fixed buffers, or in a real-time loop that may not take the
// allocator's locks or risk an out-of-memory failure halfway through a 160 ms
// unit.  Such a caller cannot create a ws_cache (which allocates the cache and
// its workspace), so this entry point works on K/V planes the caller already
// owns and keeps its own scratch -- the fp32 partials of query tiles whose key
// range is cut between two CTAs, the in-kernel merge counters and the kernel's
// status word -- in one file-scope device array instead of allocated memory.
//
// Limits and sharing: the array holds kScratchBytes (48 MiB) on every device
// that loads this part of the library, until the process exits.  The partials
// take two slots per CTA (at most one CTA per SM unless the query blocks
// outnumber the SMs): 39 MB at head_dim 128 on 148 SMs; the merge counters
// (one int per item, Q tile and warp) a few KB more.  Requests whose
// partials would not fit are rejected with WS_ERR_UNSUPPORTED.  All
// calls share the array, and it keeps the last call's contents: calls that
// overlap on the GPU (different streams, or different host threads without
// ordering) race on it and must be serialised by the caller.  The status word
// and the merge counters are cleared at the start of every call; the partials
// need no clearing, because every slot a merge reads is written first by the
// same call.
//
// Set-up: in host code the array's name stands for a host-side shadow, not for
// device memory, so its device address is looked up with cudaGetSymbolAddress
// with the device current, once per device and CUDA context (a device reset
// creates a new context, in which the module and the array may sit elsewhere);
// the context's unique ID tells a stale address apart.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ws.h"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(48) << 20;
constexpr size_t kStatusBytes = 256;            // the status word, padded to keep the partials aligned
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_setup_mutex;
struct ScratchSlot {
  unsigned long long ctx_id;   // CUDA context the address belongs to (0 = none yet)
  void* ptr;
};
ScratchSlot g_slot[ws::kMaxDevices] = {};
int g_stall_tile = -1;          // test hook (ws_debug_inject_stall with a NULL cache)

// ID of the calling thread's current context, 0 if none is bound yet.
int current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return WS_ERR_CUDA;
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return WS_ERR_CUDA;
  *id = 0;
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return WS_ERR_CUDA;
  return WS_OK;
}

// Device address of g_scratch on the current device (set up on first use there).
int scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long id = 0;
  if (current_context_id(&id) != WS_OK) return WS_ERR_CUDA;
  ScratchSlot& slot = g_slot[dev];
  if (id == 0 || id != slot.ctx_id || !slot.ptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return WS_ERR_CUDA;
    }
    if (current_context_id(&id) != WS_OK || id == 0) return WS_ERR_CUDA;
    slot.ctx_id = id;
    slot.ptr = ptr;
  }
  *out = slot.ptr;
  return WS_OK;
}

uint64_t wait_bound_ns() {
  if (const char* t = std::getenv("WS_WAIT_TIMEOUT_MS")) {
    const long long ms = std::atoll(t);
    if (ms > 0) return (uint64_t)ms * 1000000ull;
  }
  return kDefaultWaitNs;
}

int noalloc_impl(const uint16_t* q, const uint16_t* kv, uint16_t* out, int32_t n_query, int32_t n_keys,
                 int32_t n_heads, int32_t head_dim, cudaStream_t stream) {
  using namespace ws;
  if (!q || !kv || !out || n_query < 1 || n_keys < 1 || n_heads < 1) return WS_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return WS_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kv) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return WS_ERR_ALIGN;
  if ((int64_t)n_heads * 2 >= ((int64_t)1 << 31)) return WS_ERR_ARG;
  const int dev = current_device();
  if (dev < 0) return WS_ERR_CUDA;
  // the scratch used is the current device's: the stream must belong to it
  int stream_dev = -1;
  if (cudaStreamGetDevice(stream, &stream_dev) != cudaSuccess) {
    cudaGetLastError();
    return WS_ERR_ARG;
  }
  if (stream_dev != dev) return WS_ERR_ARG;

  // one query unit, one run of visible keys: rows [0, n_keys) of every plane
  AttnParams p{};
  p.qu.n_units = 1;
  p.qu.rows = n_query;
  p.qu.run_first[0] = 0;
  p.qu.run_first[1] = 1;
  p.qu.tile_start[0] = 0;
  p.qu.tile_start[1] = (n_keys + kBlockN - 1) / kBlockN;
  p.runs.n_runs = 1;
  p.runs.row_begin[0] = 0;
  p.runs.rows[0] = n_keys;
  p.runs.tile_begin[0] = 0;

  // scratch layout: [status | merge counters | part_ml | part_o], two partial slots per CTA
  const int n_qtiles = (n_query + kItemRows - 1) / kItemRows;
  decompose(p.dec, n_qtiles, n_heads, p.qu.tile_start[1], 0, attention_workers(head_dim));
  const size_t slots = (size_t)partial_slots(p.dec);
  const size_t slot_bytes = (size_t)kItemRows * (head_dim + 2) * sizeof(float);
  const size_t fix_bytes = ((size_t)fix_counters(1, n_qtiles, n_heads) * sizeof(int) + 255) & ~(size_t)255;
  if (kStatusBytes + fix_bytes + slots * slot_bytes > kScratchBytes) return WS_ERR_UNSUPPORTED;

  void* base = nullptr;
  const int st = scratch_address(dev, &base);
  if (st != WS_OK) return st;
  unsigned char* b = static_cast<unsigned char*>(base);
  p.status = reinterpret_cast<int*>(b);
  p.fix_count = reinterpret_cast<int*>(b + kStatusBytes);
  p.part_ml = reinterpret_cast<float*>(b + kStatusBytes + fix_bytes);
  p.part_o = reinterpret_cast<float*>(b + kStatusBytes + fix_bytes + slots * kItemRows * 2 * sizeof(float));

  p.n_heads = n_heads;
  p.plane_k = 0;
  p.plane_v = n_heads;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
  p.out = out;
  p.timeout_ns = wait_bound_ns();
  p.out_rows = n_query;
  p.part_slots = (int64_t)slots;
  p.fix_slots = (int64_t)(fix_bytes / sizeof(int));
  p.plane_rows = n_keys;
  p.planes = (int64_t)2 * n_heads;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p.debug_skip_v_tile = g_stall_tile;
  }

  CUtensorMap q_map, kv_map, k_half_map;
  if (encode_q_map(&q_map, q, head_dim, n_heads, n_query) != 0) return WS_ERR_CUDA;
  if (encode_kv_map(&kv_map, kv, head_dim, n_keys, (int64_t)2 * n_heads) != 0) return WS_ERR_CUDA;
  if (encode_kv_map_box(&k_half_map, kv, head_dim, n_keys, (int64_t)2 * n_heads, 64) != 0) return WS_ERR_CUDA;

  // the status word and the merge counters start at zero (a call that gave up may have left them set)
  if (cudaMemsetAsync(p.status, 0, kStatusBytes + fix_bytes, stream) != cudaSuccess) return WS_ERR_CUDA;
  p.fixup = use_fixup(p.dec) ? 1 : 0;
  if (launch_attention(q_map, kv_map, k_half_map, nullptr, p, head_dim, nullptr, stream) != cudaSuccess)
    return WS_ERR_CUDA;
  bool any_split = false;
  for (int qt = 0; qt < n_qtiles && !any_split && !p.fixup; ++qt)
    for (int h = 0; h < n_heads && !any_split; ++h) {
      int lane, c_first, pieces, end0;
      item_span(p.dec, p.qu, 0, qt, h, lane, c_first, pieces, end0);
      any_split = pieces > 1;
    }
  if (any_split && launch_merge(p, head_dim, stream) != cudaSuccess) return WS_ERR_CUDA;
  return WS_OK;
}

}  // namespace

namespace ws {
void set_noalloc_stall(int tile) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  g_stall_tile = tile;
}
}  // namespace ws

extern "C" int ws_attention_noalloc(const uint16_t* q, const uint16_t* kv, uint16_t* out, int32_t n_query,
                                    int32_t n_keys, int32_t n_heads, int32_t head_dim, cudaStream_t stream) {
  nvtxRangePushA("ws_attention_noalloc");   // a range for profilers (no cost without one)
  const int st = noalloc_impl(q, kv, out, n_query, n_keys, n_heads, head_dim, stream);
  nvtxRangePop();
  return st;
}

extern "C" int ws_attention_noalloc_sync(cudaStream_t stream) {
  nvtxRangePushA("ws_attention_noalloc_sync");
  int st = WS_OK;
  int s = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess ||
      cudaMemcpyFromSymbol(&s, g_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    st = WS_ERR_CUDA;
  } else if (s != 0) {
    const int zero = 0;
    st = cudaMemcpyToSymbol(g_scratch, &zero, sizeof(int), 0, cudaMemcpyHostToDevice) != cudaSuccess
             ? WS_ERR_CUDA
             : (s == ws::kStatusIndex ? WS_ERR_DEVICE_CHECK : WS_ERR_DEVICE_TIMEOUT);
  }
  nvtxRangePop();
  return st;
}
