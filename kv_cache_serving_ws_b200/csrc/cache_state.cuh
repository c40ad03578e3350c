// Host-side state of a cache handle, shared by the C-ABI translation units
// (ws_api.cu: cache, attention and Euler entry points; unit_graph.cu: the
// captured unit program).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ws.h"
#include "kernels.cuh"

// An NVTX range around an entry point, for profilers (no cost without one).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

struct EventPool {
  std::vector<cudaEvent_t> ev;   // pairs: 2*i start, 2*i+1 end
  int used = 0;
  int64_t launches = 0;
  double ms = 0.0;
  void create(int pairs) {
    ev.resize(2 * pairs);
    for (auto& e : ev) cudaEventCreate(&e);
    used = 0;
  }
  void destroy() {
    for (auto& e : ev) cudaEventDestroy(e);
    ev.clear();
  }
  void flush() {
    for (int i = 0; i < used; ++i) {
      cudaEventSynchronize(ev[2 * i + 1]);
      float t = 0.f;
      if (cudaEventElapsedTime(&t, ev[2 * i], ev[2 * i + 1]) == cudaSuccess) ms += t;
    }
    launches += used;
    used = 0;
  }
  cudaEvent_t* next() {
    if (ev.empty()) return nullptr;
    if (2 * used >= (int)ev.size()) flush();
    return &ev[2 * (used++)];
  }
};

// Ring bookkeeping of one session (one conversation's stream of units).
struct Ring {
  int64_t newest = -1;
  std::vector<int64_t> slot_unit;     // C entries, -1 = empty
  std::vector<uint8_t> latent_ready;  // C * L: slot s holds latent rows of layer l
};

// A cache holds n_sessions independent rings in one allocation: session s owns
// rows [s*C*T, (s+1)*C*T) of every (layer, K|V, head) plane, so one tensor map
// covers every session and one attention launch can serve several of them.
struct ws_cache {
  ws_cache_config cfg{};
  int device = 0;
  int C = 0, T = 0, Nq = 0;
  int n_sessions = 1;
  int64_t session_rows = 0;           // C * T
  std::vector<Ring> rings;            // one per session
  uint16_t* kv = nullptr;
  size_t kv_bytes = 0;
  float* part_o = nullptr;
  float* part_ml = nullptr;
  size_t ws_bytes = 0;
  int* d_status = nullptr;
  int* d_fix = nullptr;               // arrival counters of the in-kernel merge of cut items
  size_t fix_bytes = 0;
  CUtensorMap kv_map;           // boxes of a whole key tile (128 rows)
  CUtensorMap k_half_map;       // boxes of half a K tile (64 rows), for the paired kernel
  int force_lane_ctas = 0;
  int64_t slot_cap = 0;
  uint64_t timeout_ns = 2000000000ull;
  int debug_skip_v_tile = -1;
  bool profiling = false;
  bool capturing = false;   // launches are being recorded into a unit program: no profiling events
  EventPool ev_attn, ev_comb, ev_lat;
  int last_split = 0, last_ctas = 0;
  int64_t last_keys = 0;
  int last_kernel = 0;
};

namespace ws {

// Entry-point bodies shared with the unit program (ws_api.cu).  Each validates
// its arguments, updates the host bookkeeping and enqueues its launches on
// `stream`; none synchronises.
int append_impl(ws_cache* h, int session, int64_t unit, int seg, const uint16_t* k_slice, const uint16_t* v_slice,
                cudaStream_t stream);
// Query unit j is (sessions[j], units[j]); its queries are rows [j*Nq, (j+1)*Nq)
// of q, k_new, v_new and out.
int attention_impl(ws_cache* h, int layer, const int32_t* sessions, const int64_t* units, int n, const uint16_t* q,
                   const uint16_t* k_new, const uint16_t* v_new, uint16_t* out, cudaStream_t stream);
int flow_step_impl(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream);

}  // namespace ws
