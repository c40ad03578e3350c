// Unit program: the device work of one streaming unit (conditioning append,
// S x L attention calls with their latent writes (and merge launches when a call
// is too short to merge its cut items in-kernel), S Euler updates,
// latent commit) recorded as a CUDA graph and replayed once per unit.
//
// Each launch records the unit's calls on a private capture stream through the
// same entry-point bodies as the direct calls, so validation, the ring
// bookkeeping and every kernel parameter are those of the direct path.  The
// recorded graph then refreshes the executable graph in place: in steady state
// only the unit's slot rows change between units, which cudaGraphExecUpdate
// applies without a new instantiation.  Recording costs host time (a few
// microseconds per launch) but runs ahead of the GPU, which spends ~200 ms on a
// unit of the 640x368 stream; what the graph removes is the per-launch work on
// the GPU's side between consecutive kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <chrono>
#include <cstdint>
#include <new>
#include <vector>

#include "../../include/ws.h"
#include "cache_state.cuh"
#include "kernels.cuh"

struct ws_unit_graph {
  ws_cache* h = nullptr;
  ws_unit_io io{};
  cudaStream_t cap = nullptr;
  cudaGraphExec_t exec = nullptr;
  ws_unit_graph_stats stats{};
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host bookkeeping of the program's session, restored when recording a unit fails halfway.
struct Snapshot {
  int session;
  Ring ring;
  int last_split, last_ctas;
  int64_t last_keys;
  Snapshot(const ws_cache* h, int s)
      : session(s), ring(h->rings[(size_t)s]), last_split(h->last_split), last_ctas(h->last_ctas),
        last_keys(h->last_keys) {}
  void restore(ws_cache* h) const {
    h->rings[(size_t)session] = ring;
    h->last_split = last_split;
    h->last_ctas = last_ctas;
    h->last_keys = last_keys;
  }
};

// The unit's calls, in order, on `s`.
int record_unit(ws_unit_graph* g, int64_t unit, cudaStream_t s) {
  ws_cache* h = g->h;
  const ws_unit_io& io = g->io;
  const int L = h->cfg.n_layers;
  const size_t call_elems = (size_t)h->Nq * h->cfg.n_heads * h->cfg.head_dim;
  const int32_t sess = io.session;
  int st = ws::append_impl(h, sess, unit, WS_SEG_COND, io.cond_k, io.cond_v, s);
  for (int step = 0; step < io.n_steps && st == WS_OK; ++step) {
    for (int l = 0; l < L && st == WS_OK; ++l) {
      const size_t off = ((size_t)step * L + l) * call_elems;
      st = ws::attention_impl(h, l, &sess, &unit, 1, io.q + off, io.k_new + off, io.v_new + off,
                              io.out + (io.out_per_call ? off : 0), s);
    }
    if (st == WS_OK) st = ws::flow_step_impl(io.x, io.vel + (size_t)step * io.n_latent, io.dt, io.n_latent, s);
  }
  if (st == WS_OK) st = ws::append_impl(h, sess, unit, WS_SEG_LATENT, io.commit_k, io.commit_v, s);
  return st;
}

}  // namespace

extern "C" {

int ws_unit_graph_create(ws_unit_graph_t** out, ws_cache_t* h, const ws_unit_io* io) {
  if (!out || !h || !io || io->n_steps < 1 || io->n_latent < 0) return WS_ERR_ARG;
  if (io->session < 0 || io->session >= h->n_sessions) return WS_ERR_ARG;
  const void* ptrs[] = {io->cond_k, io->cond_v, io->q, io->k_new, io->v_new, io->out,
                        io->x, io->vel, io->commit_k, io->commit_v};
  for (const void* p : ptrs) {
    if (!p) return WS_ERR_ARG;
    if (!aligned16(p)) return WS_ERR_ALIGN;
  }
  ws_unit_graph* g = new (std::nothrow) ws_unit_graph();
  if (!g) return WS_ERR_OOM;
  g->h = h;
  g->io = *io;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaSetDevice(h->device);
  const cudaError_t e = cudaStreamCreateWithFlags(&g->cap, cudaStreamNonBlocking);
  cudaSetDevice(dev);
  if (e != cudaSuccess) {
    delete g;
    return WS_ERR_CUDA;
  }
  *out = g;
  return WS_OK;
}

int ws_unit_graph_launch(ws_unit_graph_t* g, int64_t unit, cudaStream_t stream) {
  const NvtxRange range("ws_unit_graph_launch");
  if (!g || unit < 0) return WS_ERR_ARG;
  ws_cache* h = g->h;
  const auto t0 = std::chrono::steady_clock::now();
  const Snapshot before(h, g->io.session);

  if (cudaStreamBeginCapture(g->cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return WS_ERR_CUDA;
  }
  h->capturing = true;
  int st = record_unit(g, unit, g->cap);
  h->capturing = false;
  cudaGraph_t graph = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(g->cap, &graph);
  if (st == WS_OK && (ec != cudaSuccess || !graph)) st = WS_ERR_CUDA;
  if (st != WS_OK) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    before.restore(h);
    return st;
  }

  size_t nodes = 0;
  cudaGraphGetNodes(graph, nullptr, &nodes);
  bool updated = false;
  if (g->exec) {
    cudaGraphExecUpdateResultInfo info{};
    if (cudaGraphExecUpdate(g->exec, graph, &info) == cudaSuccess) {
      updated = true;
    } else {
      cudaGetLastError();
      cudaGraphExecDestroy(g->exec);
      g->exec = nullptr;
    }
  }
  if (!g->exec && cudaGraphInstantiate(&g->exec, graph, 0) != cudaSuccess) {
    cudaGetLastError();
    g->exec = nullptr;
    cudaGraphDestroy(graph);
    before.restore(h);
    return WS_ERR_CUDA;
  }
  cudaGraphDestroy(graph);
  if (cudaGraphLaunch(g->exec, stream) != cudaSuccess) {
    cudaGetLastError();
    before.restore(h);
    return WS_ERR_CUDA;
  }
  const auto t1 = std::chrono::steady_clock::now();
  g->stats.launches += 1;
  g->stats.updates += updated ? 1 : 0;
  g->stats.instantiations += updated ? 0 : 1;
  g->stats.nodes = (int64_t)nodes;
  g->stats.record_ms += std::chrono::duration<double, std::milli>(t1 - t0).count();
  return WS_OK;
}

int ws_unit_graph_get_stats(const ws_unit_graph_t* g, ws_unit_graph_stats* out) {
  if (!g || !out) return WS_ERR_ARG;
  *out = g->stats;
  return WS_OK;
}

int ws_unit_graph_destroy(ws_unit_graph_t* g) {
  if (!g) return WS_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaSetDevice(g->h->device);
  const cudaError_t e = cudaDeviceSynchronize();
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->cap) cudaStreamDestroy(g->cap);
  cudaSetDevice(dev);
  delete g;
  return e == cudaSuccess ? WS_OK : WS_ERR_CUDA;
}

}  // extern "C"
