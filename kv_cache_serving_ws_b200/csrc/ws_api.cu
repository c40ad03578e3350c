// C ABI of libws: handle, argument validation, the unit-slot ring bookkeeping,
// the visible-row planner and the launches.  Declarations and the contract of
// every entry point are in include/ws.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <new>
#include <vector>

#include "../../include/ws.h"
#include "cache_state.cuh"
#include "kernels.cuh"

using namespace ws;

// Work decomposition of one attention call (see Decomp in kernels.cuh).  The
// query blocks are grouped into lanes so that the lanes together hold one CTA
// per SM; the group size minimises the iterations of the busiest CTA (ties:
// the smaller group, which re-reads K/V fewer times).  A CTA gets at least 2
// iterations.  `forced` > 0 fixes the CTAs per lane.
void ws::decompose(Decomp& d, int n_qtiles, int heads, int tiles, int forced, int workers) {
  const int sms = workers > 0 ? workers : 1;
  d.n_qtiles = n_qtiles;
  d.heads = heads;
  d.tiles = tiles;
  int best_g = 1, best_cpl = 1;
  long long best_cost = -1;
  int prev_lanes = -1;
  for (int g = 1; g <= n_qtiles; ++g) {
    const int lanes = (n_qtiles + g - 1) / g;
    if (lanes == prev_lanes) continue;
    prev_lanes = lanes;
    const long long work = (long long)g * heads * tiles;
    long long cpl = forced > 0 ? forced : std::max(1, sms / lanes);
    cpl = std::min<long long>(cpl, std::max<long long>(1, forced > 0 ? work : work / 2));
    cpl = std::min<long long>(cpl, kMaxLaneCtas);
    const long long cost = (work + cpl - 1) / cpl;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_g = g;
      best_cpl = (int)cpl;
    }
  }
  d.group = best_g;
  d.lanes = (n_qtiles + best_g - 1) / best_g;
  d.lane_ctas = best_cpl;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool config_ok(const ws_cache_config* c) {
  if (!c) return false;
  if (c->n_layers < 1 || c->n_heads < 1 || c->head_dim < 1) return false;
  if (c->n_video < 0 || c->n_audio < 0 || c->n_cond < 0 || c->history_units < 0) return false;
  const int64_t nq = (int64_t)c->n_video + c->n_audio;
  if (nq < 1) return false;
  const int64_t T = nq + c->n_cond;
  const int64_t C = (int64_t)c->history_units + 1;
  if (T * C >= (int64_t)1 << 31) return false;
  if ((int64_t)c->n_layers * 2 * c->n_heads >= (int64_t)1 << 31) return false;
  if (nq * c->n_heads * (int64_t)c->head_dim >= (int64_t)1 << 40) return false;
  return true;
}

// status of `unit` in a session's ring: resident, evicted (its slot holds a newer unit) or never appended
int resident(const ws_cache* h, int session, int64_t unit) {
  if (unit < 0) return WS_ERR_ARG;
  const int64_t holder = h->rings[(size_t)session].slot_unit[(size_t)(unit % h->C)];
  if (holder == unit) return WS_OK;
  return holder > unit ? WS_ERR_EVICTED : WS_ERR_NOT_READY;
}

int plan_runs(const ws_cache_config& cfg, const int64_t* slot_unit, const uint8_t* latent_ready, int layer,
              int64_t unit, int64_t new_from, int32_t* row_begin, int32_t* rows, int32_t max_runs, int32_t* n_runs) {
  const int C = cfg.history_units + 1;
  const int Nq = cfg.n_video + cfg.n_audio;
  const int T = cfg.n_cond + Nq;
  const int64_t lo = unit - cfg.history_units;
  int n = 0;
  int64_t run_end = -1;
  for (int s = 0; s < C; ++s) {
    const int64_t u = slot_unit[s];
    if (u < 0 || u < lo || u > unit) continue;
    // units from new_from on are the call's own: their latent rows come from k_new / v_new
    const bool lat = (new_from < 0 || u < new_from) && ((u == unit) || latent_ready[(size_t)s * cfg.n_layers + layer]);
    const int64_t b = (int64_t)s * T;
    const int64_t e = b + cfg.n_cond + (lat ? Nq : 0);
    if (e == b) continue;
    if (n > 0 && b == run_end) {
      rows[n - 1] += (int32_t)(e - b);
    } else {
      if (n == max_runs) return WS_ERR_UNSUPPORTED;
      row_begin[n] = (int32_t)b;
      rows[n] = (int32_t)(e - b);
      ++n;
    }
    run_end = e;
  }
  *n_runs = n;
  return WS_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? WS_OK : WS_ERR_CUDA; }

void free_all(ws_cache* h) {
  if (h->kv) cudaFree(h->kv);
  if (h->part_o) cudaFree(h->part_o);
  if (h->part_ml) cudaFree(h->part_ml);
  if (h->d_status) cudaFree(h->d_status);
  if (h->d_fix) cudaFree(h->d_fix);
  h->ev_attn.destroy();
  h->ev_comb.destroy();
  h->ev_lat.destroy();
}

}  // namespace

namespace ws {

// Attention of n query units at `layer`: the current unit of several sessions,
// and/or consecutive units of one session (a prefill).  Writes each unit's
// k_new/v_new into its latent rows, plans each unit's visible runs in its
// session's rows, and launches the kernel.  Items whose key range is cut
// between CTAs are merged inside the kernel when every CTA runs a long range,
// else by a merge launch after it.
int attention_impl(ws_cache* h, int layer, const int32_t* sessions, const int64_t* units, int n, const uint16_t* q,
                   const uint16_t* k_new, const uint16_t* v_new, uint16_t* out, cudaStream_t stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers || !sessions || !units || n < 1) return WS_ERR_ARG;
  if (n > kMaxQUnits) return WS_ERR_UNSUPPORTED;
  if (!q || !k_new || !v_new || !out) return WS_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return WS_ERR_ALIGN;
  const int H = h->cfg.n_heads, D = h->cfg.head_dim, L = h->cfg.n_layers, U = h->cfg.history_units;
  const int S = h->n_sessions;
  for (int j = 0; j < n; ++j)
    if (sessions[j] < 0 || sessions[j] >= S || units[j] < 0) return WS_ERR_ARG;
  // The query units of one session form one stretch of consecutive units in the
  // list, ending at the session's newest unit.  Every query unit must be
  // resident, and no unit of any query window evicted.
  std::vector<uint8_t> seen((size_t)S, 0);
  for (int j = 0; j < n;) {
    const int sess = sessions[j];
    if (seen[(size_t)sess]) return WS_ERR_ARG;
    seen[(size_t)sess] = 1;
    int k = j;
    while (k + 1 < n && sessions[k + 1] == sess) {
      if (units[k + 1] != units[k] + 1) return WS_ERR_ARG;
      ++k;
    }
    const Ring& r = h->rings[(size_t)sess];
    const int64_t u_first = units[j], u_last = units[k];
    if (r.newest < 0 || u_last > r.newest) return WS_ERR_NOT_READY;
    if (u_last < r.newest) return WS_ERR_UNIT_ORDER;
    for (int64_t u = u_first; u <= u_last; ++u) {
      const int st = resident(h, sess, u);
      if (st != WS_OK) return st;
    }
    // units before the first query unit lie in some query window; one whose slot
    // now holds a newer unit (a later query unit of a long prefill) is gone
    for (int64_t u = std::max<int64_t>(0, u_first - U); u < u_first; ++u)
      if (r.slot_unit[(size_t)(u % h->C)] > u) return WS_ERR_EVICTED;
    j = k + 1;
  }

  // plan first (pure host work), so that an unsupported layout changes nothing
  std::vector<std::vector<uint8_t>> ready((size_t)S);
  for (int j = 0; j < n; ++j) {
    auto& rd = ready[(size_t)sessions[j]];
    if (rd.empty()) rd = h->rings[(size_t)sessions[j]].latent_ready;
    rd[(size_t)(units[j] % h->C) * L + layer] = 1;
  }
  // The single-SM kernel writes the call's latent K/V itself and reads those key rows
  // from k_new / v_new (no separate write launch) when every session has one query
  // unit in the call.  In a prefill stretch the cache interleaves each unit's
  // conditioning rows with its latent rows, so reading the latents elsewhere would cut
  // the key runs into short tiles: those calls, and the paired kernel, write first and
  // read the cache.
  bool fold = !attention_uses_pairs(D);
  for (int j = 1; j < n; ++j)
    if (sessions[j] == sessions[j - 1]) fold = false;
  AttnParams p{};
  p.qu.n_units = n;
  p.qu.rows = h->Nq;
  int runs = 0, tiles = 0;
  int64_t keys = 0;
  int j_first = 0;   // first query unit of the current session's stretch
  for (int j = 0; j < n; ++j) {
    if (j > 0 && sessions[j] != sessions[j - 1]) j_first = j;
    p.qu.run_first[j] = runs;
    p.qu.tile_start[j] = tiles;
    int32_t nr = 0;
    const int sess = sessions[j];
    const int64_t u_first = units[j_first];
    const int st = plan_runs(h->cfg, h->rings[(size_t)sess].slot_unit.data(), ready[(size_t)sess].data(), layer,
                             units[j], fold ? u_first : -1, p.runs.row_begin + runs, p.runs.rows + runs,
                             kMaxRuns - runs, &nr);
    if (st != WS_OK) return st;
    for (int r = runs; r < runs + nr; ++r) {
      p.runs.row_begin[r] += (int32_t)(sess * h->session_rows);
      p.runs.from_new[r] = 0;
    }
    if (fold) {
      // the visible units of the stretch, u_lo .. units[j]: consecutive token rows of k_new
      const int64_t u_lo = std::max<int64_t>(u_first, units[j] - U);
      if (runs + nr == kMaxRuns) return WS_ERR_UNSUPPORTED;
      p.runs.row_begin[runs + nr] = (int32_t)((j_first + (u_lo - u_first)) * h->Nq);
      p.runs.rows[runs + nr] = (int32_t)((units[j] - u_lo + 1) * h->Nq);
      p.runs.from_new[runs + nr] = 1;
      ++nr;
    }
    int t = 0;
    for (int r = runs; r < runs + nr; ++r) {
      p.runs.tile_begin[r] = t;
      t += (p.runs.rows[r] + kBlockN - 1) / kBlockN;
      keys += p.runs.rows[r];
    }
    runs += nr;
    tiles += t;
  }
  p.qu.run_first[n] = runs;
  p.qu.tile_start[n] = tiles;
  p.runs.n_runs = runs;

  const int n_qtiles = (h->Nq + kItemRows - 1) / kItemRows;
  const int workers = attention_workers(D);
  decompose(p.dec, n_qtiles, H, tiles, h->force_lane_ctas, workers);
  while (partial_slots(p.dec) > h->slot_cap && p.dec.lane_ctas > 1)
    decompose(p.dec, n_qtiles, H, tiles, std::max(1, p.dec.lane_ctas / 2), workers);
  if (partial_slots(p.dec) > h->slot_cap) return WS_ERR_UNSUPPORTED;
  p.fixup = use_fixup(p.dec) ? 1 : 0;
  bool any_split = false;
  for (int j = 0; j < n && !any_split && !p.fixup; ++j)
    for (int qt = 0; qt < n_qtiles && !any_split; ++qt)
      for (int hh = 0; hh < H && !any_split; ++hh) {
        int lane, c_first, pieces, end0;
        item_span(p.dec, p.qu, j, qt, hh, lane, c_first, pieces, end0);
        any_split = pieces > 1;
      }

  CUtensorMap q_map;
  if (encode_q_map(&q_map, q, D, H, n * h->Nq) != 0) return WS_ERR_CUDA;

  // 1. the query units' latent K/V of this layer into their slots: inside the
  //    attention launch (fold), else by one write launch per unit
  const size_t unit_elems = (size_t)h->Nq * H * D;
  CUtensorMap new_maps[2];
  if (fold) {
    if (encode_q_map(&new_maps[0], k_new, D, H, n * h->Nq) != 0) return WS_ERR_CUDA;
    if (encode_q_map(&new_maps[1], v_new, D, H, n * h->Nq) != 0) return WS_ERR_CUDA;
    p.fold = 1;
    p.k_new = k_new;
    p.v_new = v_new;
    p.cache = h->kv;
  }
  for (int j = 0; j < n; ++j) {
    const size_t slot = (size_t)(units[j] % h->C);
    p.latent_row0[j] = sessions[j] * h->session_rows + (int64_t)slot * h->T + h->cfg.n_cond;
    if (fold) {
      h->rings[(size_t)sessions[j]].latent_ready[slot * L + layer] = 1;
      continue;
    }
    AppendParams a{};
    a.src_k = k_new + j * unit_elems;
    a.src_v = v_new + j * unit_elems;
    a.cache = h->kv;
    a.n_layers = 1;
    a.layer0 = layer;
    a.n_tokens = h->Nq;
    a.n_heads = H;
    a.head_dim = D;
    a.plane_rows = h->session_rows * h->n_sessions;
    a.row0 = sessions[j] * h->session_rows + (int64_t)slot * h->T + h->cfg.n_cond;
    a.planes = (int64_t)L * 2 * H;
    a.status = h->d_status;
    cudaEvent_t* ev = h->profiling && !h->capturing ? h->ev_lat.next() : nullptr;
    if (ev) cudaEventRecord(ev[0], stream);
    if (launch_append(a, stream) != cudaSuccess) return WS_ERR_CUDA;
    if (ev) cudaEventRecord(ev[1], stream);
    h->rings[(size_t)sessions[j]].latent_ready[slot * L + layer] = 1;
  }

  // 2. attention (+ merge of the partials of cut items)
  p.n_heads = H;
  p.plane_k = (layer * 2 + 0) * H;
  p.plane_v = (layer * 2 + 1) * H;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.out = out;
  p.part_o = h->part_o;
  p.part_ml = h->part_ml;
  p.status = h->d_status;
  p.fix_count = h->d_fix;
  p.timeout_ns = h->timeout_ns;
  p.debug_skip_v_tile = h->debug_skip_v_tile;
  p.out_rows = (int64_t)n * h->Nq;
  p.part_slots = h->slot_cap;
  p.fix_slots = (int64_t)(h->fix_bytes / sizeof(int));
  p.plane_rows = h->session_rows * h->n_sessions;
  p.planes = (int64_t)L * 2 * H;
  cudaEvent_t* ev = h->profiling && !h->capturing ? h->ev_attn.next() : nullptr;
  if (ev) cudaEventRecord(ev[0], stream);
  int ctas = 0;
  if (launch_attention(q_map, h->kv_map, h->k_half_map, fold ? new_maps : nullptr, p, D, &ctas, stream) !=
      cudaSuccess)
    return WS_ERR_CUDA;
  if (ev) cudaEventRecord(ev[1], stream);
  if (any_split) {
    ev = h->profiling && !h->capturing ? h->ev_comb.next() : nullptr;
    if (ev) cudaEventRecord(ev[0], stream);
    if (launch_merge(p, D, stream) != cudaSuccess) return WS_ERR_CUDA;
    if (ev) cudaEventRecord(ev[1], stream);
  }
  h->last_split = p.dec.lane_ctas;
  h->last_ctas = ctas;
  h->last_keys = keys;
  h->last_kernel = attention_uses_pairs(D) ? 2 : 1;
  return WS_OK;
}

int append_impl(ws_cache* h, int session, int64_t unit, int seg, const uint16_t* k_slice, const uint16_t* v_slice,
                cudaStream_t stream) {
  if (!h || unit < 0 || (seg != WS_SEG_COND && seg != WS_SEG_LATENT)) return WS_ERR_ARG;
  if (session < 0 || session >= h->n_sessions) return WS_ERR_ARG;
  Ring& r = h->rings[(size_t)session];
  const int n = seg == WS_SEG_COND ? h->cfg.n_cond : h->Nq;
  if (n > 0) {
    if (!k_slice || !v_slice) return WS_ERR_ARG;
    if (!aligned16(k_slice) || !aligned16(v_slice)) return WS_ERR_ALIGN;
  }
  const size_t slot = (size_t)(unit % h->C);
  if (seg == WS_SEG_COND) {
    if (unit < r.newest) return WS_ERR_UNIT_ORDER;
  } else {
    const int st = resident(h, session, unit);
    if (st != WS_OK) return st;
  }
  AppendParams p{};
  p.src_k = k_slice;
  p.src_v = v_slice;
  p.cache = h->kv;
  p.n_layers = h->cfg.n_layers;
  p.layer0 = 0;
  p.n_tokens = n;
  p.n_heads = h->cfg.n_heads;
  p.head_dim = h->cfg.head_dim;
  p.plane_rows = h->session_rows * h->n_sessions;
  p.row0 = session * h->session_rows + (int64_t)slot * h->T + (seg == WS_SEG_COND ? 0 : h->cfg.n_cond);
  p.planes = (int64_t)h->cfg.n_layers * 2 * h->cfg.n_heads;
  p.status = h->d_status;
  const cudaError_t e = launch_append(p, stream);
  if (e != cudaSuccess) return WS_ERR_CUDA;
  if (seg == WS_SEG_COND) {
    if (unit > r.newest) {
      r.slot_unit[slot] = unit;
      std::fill(r.latent_ready.begin() + slot * h->cfg.n_layers, r.latent_ready.begin() + (slot + 1) * h->cfg.n_layers,
                0);
      r.newest = unit;
    }
  } else {
    std::fill(r.latent_ready.begin() + slot * h->cfg.n_layers, r.latent_ready.begin() + (slot + 1) * h->cfg.n_layers,
              1);
  }
  return WS_OK;
}

int flow_step_impl(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream) {
  if (n < 0) return WS_ERR_ARG;
  if (n == 0) return WS_OK;
  if (!x || !v) return WS_ERR_ARG;
  if (!aligned16(x) || !aligned16(v)) return WS_ERR_ALIGN;
  return cuda_status(launch_euler(x, v, dt, n, stream));
}

}  // namespace ws

extern "C" {

const char* ws_status_string(int status) {
  switch (status) {
    case WS_OK: return "ok";
    case WS_ERR_ARG: return "invalid argument";
    case WS_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case WS_ERR_OOM: return "device allocation failed";
    case WS_ERR_UNIT_ORDER: return "unit older than the newest conditioned unit";
    case WS_ERR_EVICTED: return "unit evicted from the ring (its slot holds a newer unit)";
    case WS_ERR_NOT_READY: return "unit or segment not written yet";
    case WS_ERR_CUDA: return "CUDA error";
    case WS_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
    case WS_ERR_UNSUPPORTED: return "request outside what this build supports";
    case WS_ERR_DEVICE_CHECK: return "a device-side index check failed (debug build)";
    default: return "unknown status";
  }
}

int ws_plan_visible(const ws_cache_config* cfg, const int64_t* slot_unit, const uint8_t* latent_ready, int layer,
                    int64_t unit, int32_t* row_begin, int32_t* rows, int32_t max_runs, int32_t* n_runs) {
  if (!config_ok(cfg) || !slot_unit || !latent_ready || !row_begin || !rows || !n_runs || max_runs < 0)
    return WS_ERR_ARG;
  if (layer < 0 || layer >= cfg->n_layers || unit < 0) return WS_ERR_ARG;
  return plan_runs(*cfg, slot_unit, latent_ready, layer, unit, -1, row_begin, rows, max_runs, n_runs);
}

int ws_pool_create(ws_cache_t** out, const ws_cache_config* cfg, int32_t n_sessions, cudaStream_t stream) {
  if (!out || !config_ok(cfg) || n_sessions < 1) return WS_ERR_ARG;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return WS_ERR_UNSUPPORTED;
  const int64_t T64 = (int64_t)cfg->n_cond + cfg->n_video + cfg->n_audio;
  if (T64 * (cfg->history_units + 1) * n_sessions >= (int64_t)1 << 31) return WS_ERR_UNSUPPORTED;
  ws_cache* h = new (std::nothrow) ws_cache();
  if (!h) return WS_ERR_OOM;
  h->cfg = *cfg;
  cudaGetDevice(&h->device);
  h->Nq = cfg->n_video + cfg->n_audio;
  h->T = cfg->n_cond + h->Nq;
  h->C = cfg->history_units + 1;
  h->n_sessions = n_sessions;
  h->session_rows = (int64_t)h->C * h->T;
  h->rings.resize((size_t)n_sessions);
  for (Ring& r : h->rings) {
    r.slot_unit.assign(h->C, -1);
    r.latent_ready.assign((size_t)h->C * cfg->n_layers, 0);
  }
  if (const char* t = std::getenv("WS_WAIT_TIMEOUT_MS")) {
    const long long ms = std::atoll(t);
    if (ms > 0) h->timeout_ns = (uint64_t)ms * 1000000ull;
  }
  const int L = cfg->n_layers, H = cfg->n_heads, D = cfg->head_dim;
  const int64_t rows = h->session_rows * n_sessions;
  h->kv_bytes = (size_t)L * 2 * H * rows * D * 2;
  // partial slots: two per CTA; an automatic decomposition has at most one CTA
  // per SM (more only when the query blocks outnumber the SMs)
  const int64_t n_qtiles = (h->Nq + kItemRows - 1) / kItemRows;
  h->slot_cap = 2 * std::max<int64_t>(sm_count(), n_qtiles);
  const size_t part_o_bytes = (size_t)h->slot_cap * kItemRows * D * 4;
  const size_t part_ml_bytes = (size_t)h->slot_cap * kItemRows * 2 * 4;
  h->fix_bytes = (size_t)fix_counters(kMaxQUnits, (int)n_qtiles, H) * sizeof(int);
  h->ws_bytes = part_o_bytes + part_ml_bytes + h->fix_bytes;
  int st = WS_OK;
  if (cudaMalloc(&h->kv, h->kv_bytes) != cudaSuccess || cudaMalloc(&h->part_o, part_o_bytes) != cudaSuccess ||
      cudaMalloc(&h->part_ml, part_ml_bytes) != cudaSuccess || cudaMalloc(&h->d_status, sizeof(int)) != cudaSuccess ||
      cudaMalloc(&h->d_fix, h->fix_bytes) != cudaSuccess)
    st = WS_ERR_OOM;
  if (st == WS_OK && (cudaMemsetAsync(h->kv, 0, h->kv_bytes, stream) != cudaSuccess ||
                      cudaMemsetAsync(h->d_status, 0, sizeof(int), stream) != cudaSuccess ||
                      cudaMemsetAsync(h->d_fix, 0, h->fix_bytes, stream) != cudaSuccess))
    st = WS_ERR_CUDA;
  if (st == WS_OK && (encode_kv_map(&h->kv_map, h->kv, D, rows, (int64_t)L * 2 * H) != 0 ||
                      encode_kv_map_box(&h->k_half_map, h->kv, D, rows, (int64_t)L * 2 * H, 64) != 0))
    st = WS_ERR_CUDA;
  if (st != WS_OK) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return st;
  }
  *out = h;
  return WS_OK;
}

int ws_cache_create(ws_cache_t** out, const ws_cache_config* cfg, cudaStream_t stream) {
  return ws_pool_create(out, cfg, 1, stream);
}

int ws_cache_destroy(ws_cache_t* h) {
  if (!h) return WS_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaSetDevice(h->device);
  const cudaError_t e = cudaDeviceSynchronize();
  free_all(h);
  delete h;
  cudaSetDevice(dev);
  return cuda_status(e);
}

int ws_cache_append(ws_cache_t* h, int64_t unit, int seg, const uint16_t* k_slice, const uint16_t* v_slice,
                    cudaStream_t stream) {
  const NvtxRange range("ws_cache_append");
  return append_impl(h, 0, unit, seg, k_slice, v_slice, stream);
}

int ws_session_append(ws_cache_t* h, int32_t session, int64_t unit, int seg, const uint16_t* k_slice,
                      const uint16_t* v_slice, cudaStream_t stream) {
  const NvtxRange range("ws_session_append");
  return append_impl(h, session, unit, seg, k_slice, v_slice, stream);
}

int ws_unit_attention(ws_cache_t* h, int layer, int64_t unit, const uint16_t* q, const uint16_t* k_new,
                      const uint16_t* v_new, uint16_t* out, cudaStream_t stream) {
  const NvtxRange range("ws_unit_attention");
  const int32_t s0 = 0;
  return attention_impl(h, layer, &s0, &unit, 1, q, k_new, v_new, out, stream);
}

int ws_prefill_attention(ws_cache_t* h, int layer, int64_t unit_first, int32_t n_units, const uint16_t* q,
                         const uint16_t* k_new, const uint16_t* v_new, uint16_t* out, cudaStream_t stream) {
  const NvtxRange range("ws_prefill_attention");
  if (!h || unit_first < 0 || n_units < 1) return WS_ERR_ARG;
  if (n_units > kMaxQUnits) return WS_ERR_UNSUPPORTED;
  int32_t sess[kMaxQUnits];
  int64_t units[kMaxQUnits];
  for (int j = 0; j < n_units; ++j) {
    sess[j] = 0;
    units[j] = unit_first + j;
  }
  return attention_impl(h, layer, sess, units, n_units, q, k_new, v_new, out, stream);
}

int ws_session_attention(ws_cache_t* h, int layer, int32_t n, const int32_t* sessions, const int64_t* units,
                         const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, uint16_t* out,
                         cudaStream_t stream) {
  const NvtxRange range("ws_session_attention");
  return attention_impl(h, layer, sessions, units, n, q, k_new, v_new, out, stream);
}

int ws_flow_step(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream) {
  const NvtxRange range("ws_flow_step");
  return flow_step_impl(x, v, dt, n, stream);
}

int ws_session_read(ws_cache_t* h, int32_t session, int layer, int64_t unit, int seg, uint16_t* k_out,
                    uint16_t* v_out, cudaStream_t stream) {
  const NvtxRange range("ws_session_read");
  if (!h || layer < 0 || layer >= h->cfg.n_layers || unit < 0) return WS_ERR_ARG;
  if (session < 0 || session >= h->n_sessions) return WS_ERR_ARG;
  if (seg != WS_SEG_COND && seg != WS_SEG_LATENT) return WS_ERR_ARG;
  const int n = seg == WS_SEG_COND ? h->cfg.n_cond : h->Nq;
  if (n > 0) {
    if (!k_out || !v_out) return WS_ERR_ARG;
    if (!aligned16(k_out) || !aligned16(v_out)) return WS_ERR_ALIGN;
  }
  const int st = resident(h, session, unit);
  if (st != WS_OK) return st;
  const size_t slot = (size_t)(unit % h->C);
  if (seg == WS_SEG_LATENT && !h->rings[(size_t)session].latent_ready[slot * h->cfg.n_layers + layer])
    return WS_ERR_NOT_READY;
  ReadParams p{};
  p.cache = h->kv;
  p.dst_k = k_out;
  p.dst_v = v_out;
  p.layer = layer;
  p.n_tokens = n;
  p.n_heads = h->cfg.n_heads;
  p.head_dim = h->cfg.head_dim;
  p.plane_rows = h->session_rows * h->n_sessions;
  p.row0 = session * h->session_rows + (int64_t)slot * h->T + (seg == WS_SEG_COND ? 0 : h->cfg.n_cond);
  p.planes = (int64_t)h->cfg.n_layers * 2 * h->cfg.n_heads;
  p.status = h->d_status;
  return cuda_status(launch_read(p, stream));
}

int ws_cache_read(ws_cache_t* h, int layer, int64_t unit, int seg, uint16_t* k_out, uint16_t* v_out,
                  cudaStream_t stream) {
  return ws_session_read(h, 0, layer, unit, seg, k_out, v_out, stream);
}

int ws_session_slot_table(const ws_cache_t* h, int32_t session, int64_t* slot_unit_host) {
  if (!h || !slot_unit_host || session < 0 || session >= h->n_sessions) return WS_ERR_ARG;
  const Ring& r = h->rings[(size_t)session];
  std::copy(r.slot_unit.begin(), r.slot_unit.end(), slot_unit_host);
  return WS_OK;
}

int ws_cache_slot_table(const ws_cache_t* h, int64_t* slot_unit_host) {
  return ws_session_slot_table(h, 0, slot_unit_host);
}

int ws_session_reset(ws_cache_t* h, int32_t session) {
  if (!h || session < 0 || session >= h->n_sessions) return WS_ERR_ARG;
  Ring& r = h->rings[(size_t)session];
  r.newest = -1;
  std::fill(r.slot_unit.begin(), r.slot_unit.end(), -1);
  std::fill(r.latent_ready.begin(), r.latent_ready.end(), 0);
  return WS_OK;
}

int ws_cache_get_info(const ws_cache_t* h, ws_cache_info* info) {
  if (!h || !info) return WS_ERR_ARG;
  info->slots = h->C;
  info->tokens_per_unit = h->T;
  info->n_query = h->Nq;
  info->newest_unit = h->rings[0].newest;
  info->n_sessions = h->n_sessions;
  info->cache_bytes = h->kv_bytes;
  info->workspace_bytes = h->ws_bytes;
  return WS_OK;
}

int ws_cache_set_splits(ws_cache_t* h, int n_split) {
  if (!h || n_split < 0 || n_split > kMaxLaneCtas) return WS_ERR_ARG;
  h->force_lane_ctas = n_split;
  return WS_OK;
}

int ws_debug_inject_stall(ws_cache_t* h, int tile) {
  if (tile < -1) return WS_ERR_ARG;
  if (!h) {
    set_noalloc_stall(tile);
    return WS_OK;
  }
  h->debug_skip_v_tile = tile;
  return WS_OK;
}

int ws_sync(ws_cache_t* h, cudaStream_t stream) {
  const NvtxRange range("ws_sync");
  if (!h) return WS_ERR_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return WS_ERR_CUDA;
  int s = 0;
  if (cudaMemcpy(&s, h->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WS_ERR_CUDA;
  if (s != 0) {
    // a kernel that gave up may have left merge counters mid-count
    if (cudaMemset(h->d_status, 0, sizeof(int)) != cudaSuccess) return WS_ERR_CUDA;
    if (cudaMemset(h->d_fix, 0, h->fix_bytes) != cudaSuccess) return WS_ERR_CUDA;
    return s == kStatusIndex ? WS_ERR_DEVICE_CHECK : WS_ERR_DEVICE_TIMEOUT;
  }
  return WS_OK;
}

int ws_profile_enable(ws_cache_t* h, int enable) {
  if (!h) return WS_ERR_ARG;
  if (enable && !h->profiling) {
    // enough pairs for ~100 unit steps of 160 calls before a mid-run flush
    h->ev_attn.create(16384);
    h->ev_comb.create(16384);
    h->ev_lat.create(16384);
  } else if (!enable && h->profiling) {
    cudaDeviceSynchronize();
    h->ev_attn.destroy();
    h->ev_comb.destroy();
    h->ev_lat.destroy();
  }
  h->profiling = enable != 0;
  for (EventPool* e : {&h->ev_attn, &h->ev_comb, &h->ev_lat}) {
    e->used = 0;
    e->launches = 0;
    e->ms = 0.0;
  }
  return WS_OK;
}

int ws_profile_read(ws_cache_t* h, ws_profile* out) {
  if (!h || !out) return WS_ERR_ARG;
  h->ev_attn.flush();
  h->ev_comb.flush();
  h->ev_lat.flush();
  out->attention_launches = h->ev_attn.launches;
  out->attention_ms = h->ev_attn.ms;
  out->combine_launches = h->ev_comb.launches;
  out->combine_ms = h->ev_comb.ms;
  out->latent_write_launches = h->ev_lat.launches;
  out->latent_write_ms = h->ev_lat.ms;
  out->last_n_split = h->last_split;
  out->last_ctas = h->last_ctas;
  out->last_keys = h->last_keys;
  out->last_kernel = h->last_kernel;
  return WS_OK;
}

}  // extern "C"
