// Internal launch interface between the C ABI (ws_api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ws {

constexpr int kBlockM = 128;   // query rows per Q tile (one TMEM lane each)
constexpr int kQTiles = 2;     // Q tiles per item (ping-pong softmax warpgroups)
constexpr int kItemRows = kBlockM * kQTiles;
constexpr int kBlockN = 128;   // keys per tile
constexpr int kMaxRuns = 192;  // visible row runs per attention call, over all its query units
constexpr int kMaxQUnits = 64; // query units per attention call
constexpr int kMaxLaneCtas = 1024;

// Visible key rows of one (layer, head) plane as runs of consecutive rows.
// Query unit j of a call owns runs [QueryUnits::run_first[j], run_first[j+1]);
// each run is cut into kBlockN-row tiles, and tile_begin[r] is the first tile
// of run r among its unit's tiles.
// A run flagged from_new holds rows of the call's own k_new/v_new ([n_units*Nq][H][D],
// row_begin counting their token rows) instead of cache rows.
struct KeyRuns {
  int32_t n_runs;
  int32_t row_begin[kMaxRuns];
  int32_t rows[kMaxRuns];
  int32_t tile_begin[kMaxRuns];
  int8_t from_new[kMaxRuns];
};

// The query units of one call (one for the per-unit step, several for a
// prefill): unit j's queries are rows [j*rows, (j+1)*rows) of q and out, and
// see tile_start[j+1] - tile_start[j] key tiles.
struct QueryUnits {
  int32_t n_units;
  int32_t rows;                        // query rows per unit (Nq)
  int32_t tile_start[kMaxQUnits + 1];  // prefix sums of the units' key tiles
  int32_t run_first[kMaxQUnits + 1];
};

// Work decomposition.  An item is (query unit j, block qt of kItemRows query
// rows, head h) over that unit's key tiles.  The blocks are cut into lanes of
// `group` consecutive blocks; every lane has `lane_ctas` CTAs, and CTA idx of a
// lane processes the iterations [idx*per, (idx+1)*per) of its lane's sequence
// (head, block of the lane, query unit, key tile), head major.  CTAs with the
// same idx in different lanes then read the same K/V tiles at about the same
// time (L2 reuse).  An item covered by one CTA is written as bf16 directly; an
// item cut by a CTA boundary is written as fp32 partials and merged.  Only the
// first and the last item of a CTA's range can be cut, so the partials need two
// slots per CTA: slot (cta, 0) for its first item, (cta, 1) for its last.
struct Decomp {
  int32_t n_qtiles;         // query blocks per unit
  int32_t group;            // query blocks per lane
  int32_t lanes;
  int32_t lane_ctas;
  int32_t tiles;            // key tiles of one (head, block) over all query units (sum over units)
  int32_t heads;
};

__host__ __device__ inline int lane_qtiles(const Decomp& d, int lane) {
  const int left = d.n_qtiles - lane * d.group;
  return left < d.group ? left : d.group;
}
__host__ __device__ inline long long lane_work(const Decomp& d, int lane) {
  return (long long)lane_qtiles(d, lane) * d.heads * d.tiles;
}
// Quotient of non-negative a by positive b; 32-bit division when both fit (the
// common case: a 64-bit division is a long instruction sequence on the GPU).
__host__ __device__ inline long long div_nonneg(long long a, long long b) {
  if (a >= 0 && a <= 0x7fffffffLL && b <= 0x7fffffffLL) return (long long)((unsigned)a / (unsigned)b);
  return a / b;
}
__host__ __device__ inline long long lane_per(const Decomp& d, int lane) {
  return div_nonneg(lane_work(d, lane) + d.lane_ctas - 1, d.lane_ctas);
}
// The CTAs (lane-local) that cover item (j, qt, h), and the partial slot index
// of its first piece (0 when the item starts exactly at that CTA's range).
__host__ __device__ inline void item_span(const Decomp& d, const QueryUnits& u, int j, int qt, int h,
                                          int& lane, int& first_cta, int& pieces, int& first_slot_end) {
  lane = qt / d.group;
  const int a = qt - lane * d.group;
  const long long start = ((long long)h * lane_qtiles(d, lane) + a) * d.tiles + u.tile_start[j];
  const int len = u.tile_start[j + 1] - u.tile_start[j];
  const long long per = lane_per(d, lane);
  first_cta = (int)div_nonneg(start, per);
  pieces = (int)(len > 0 ? div_nonneg(start + len - 1, per) : (start + len - 1) / per) - first_cta + 1;
  first_slot_end = start == (long long)first_cta * per ? 0 : 1;
}
__host__ __device__ inline size_t partial_slot(const Decomp& d, int lane, int cta, int end) {
  return ((size_t)lane * d.lane_ctas + cta) * 2 + end;
}

// Device status values written by kernels into a status word (read by ws_sync).
constexpr int kStatusTimeout = 1;   // a bounded wait ran out
constexpr int kStatusIndex = 2;     // a device index check failed (WS_DEBUG_CHECKS builds)

// Device index checks.  A build with -DWS_DEBUG_CHECKS (libws_debug.so) tests every
// computed cache row, output row, partial slot and merge counter against the bounds
// the host passes; a failed check records kStatusIndex in the status word and the
// access is skipped (no trap, no fault).  In the normal build the checks compile away.
#ifdef WS_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool index_ok(bool ok, int* status) {
  if (kDebugChecks && !ok) {
    if (status) atomicCAS(status, 0, kStatusIndex);
    return false;
  }
  return true;
}

struct AttnParams {
  int32_t n_heads;          // H
  int32_t plane_k;          // KV-map plane index of head 0's K of this layer
  int32_t plane_v;          // same for V
  float scale_log2;         // log2(e) / sqrt(D)
  uint16_t* out;            // [n_units * Nq][H][D] bf16
  float* part_o;            // [2 * CTAs][kItemRows][D] fp32
  float* part_ml;           // [2 * CTAs][kItemRows][2] (reference max in log2 units, sum)
  int* fix_count;           // [fix_counters()] arrivals per (cut item, Q tile, warp); zero between launches
  int32_t fixup;            // 1: cut items merged inside the kernel; 0: by launch_merge afterwards
  int* status;              // device status word
  uint64_t timeout_ns;      // bound of every wait
  int32_t debug_skip_v_tile;  // test hook: never load V of this CTA-local tile (-1 = off)
  // bounds for the index checks of debug builds
  int64_t out_rows;         // rows of out (n_units * Nq)
  int64_t part_slots;       // partial slots behind part_o / part_ml
  int64_t fix_slots;        // merge counters behind fix_count
  int64_t plane_rows;       // rows of each K/V plane
  int64_t planes;           // planes of the K/V maps
  // The call's own latent K/V.  fold = 1: the kernel reads those key rows from k_new /
  // v_new (runs flagged from_new) and writes them into their cache rows itself; fold =
  // 0: they were written into the cache before the launch.
  int32_t fold;
  const uint16_t* k_new;    // [n_units * Nq][H][D] bf16
  const uint16_t* v_new;
  uint16_t* cache;          // the K/V planes [planes][plane_rows][D]
  int64_t latent_row0[kMaxQUnits];  // plane row of query unit j's first latent row
  Decomp dec;
  QueryUnits qu;
  KeyRuns runs;
};

// Encodes the tensor maps used by the attention kernels.  `kv` points at the
// cache planes [planes][rows][D], read in boxes of 64 columns x `box_rows` rows
// (128 rows: a whole key tile; 64 rows: half a K tile, for the paired kernel);
// `q` at [Nq][H][D].
int encode_kv_map_box(CUtensorMap* map, const void* kv, int head_dim, int64_t rows, int64_t planes, int box_rows);
inline int encode_kv_map(CUtensorMap* map, const void* kv, int head_dim, int64_t rows, int64_t planes) {
  return encode_kv_map_box(map, kv, head_dim, rows, planes, kBlockN);
}
int encode_q_map(CUtensorMap* map, const void* q, int head_dim, int n_heads, int n_query);

// The attention launch: the single-SM kernel (attention.cu) for both head sizes,
// or, with WS_ATTENTION_KERNEL=pair and head_dim 128, the kernel on pairs of SMs
// (attention_pair.cu) where the device can hold its clusters.  `kv_map` has
// whole-tile boxes, `k_half_map` boxes of 64 rows.  `p.dec` must come from
// decompose() with attention_workers(head_dim) workers.
// With p.fold = 1, new_maps[0] and new_maps[1] map k_new and v_new like q_map (the
// single-SM kernel only; the paired kernel takes p.fold = 0).
cudaError_t launch_attention(const CUtensorMap& q_map, const CUtensorMap& kv_map, const CUtensorMap& k_half_map,
                             const CUtensorMap* new_maps, const AttnParams& p, int head_dim, int* ctas,
                             cudaStream_t stream);
// Workers (CTAs, or CTA pairs) of the kernel launch_attention uses for head_dim.
int attention_workers(int head_dim);
bool attention_uses_pairs(int head_dim);
// CTA pairs that can be resident at once for the paired kernel (0: none).
int pair_workers();
cudaError_t launch_attention_pair(const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                                  const AttnParams& p, int* ctas, cudaStream_t stream);
// Chooses the work decomposition of one attention call (defined in ws_api.cu):
// the Q-block lanes together hold one worker per resident slot (`workers`), or
// `forced` workers per lane.
void decompose(Decomp& d, int n_qtiles, int heads, int tiles, int forced, int workers);
// Partial slots a decomposition needs (two per worker).
inline int64_t partial_slots(const Decomp& d) { return (int64_t)d.lanes * d.lane_ctas * 2; }

// Merge of cut items as its own launch (when p.fixup == 0).
cudaError_t launch_merge(const AttnParams& p, int head_dim, cudaStream_t stream);
// In-kernel merging pays a fence and an atomic per cut item on the CTA's path and
// puts the last merge on the kernel's tail: worth it once a CTA runs this many
// iterations (the separate merge launch then costs more).
constexpr long long kFixupMinIterations = 64;
inline bool use_fixup(const Decomp& d) { return lane_per(d, 0) >= kFixupMinIterations; }
// Arrival counters of a call: kFixPerTile per (item, Q tile), one per softmax warp
// that owns rows of the tile.
constexpr int kFixPerTile = 4;
inline int64_t fix_counters(int n_units, int n_qtiles, int heads) {
  return (int64_t)n_units * n_qtiles * heads * kQTiles * kFixPerTile;
}

// Copy a [L][n][H][D] token-major slice into the head-major cache planes:
// plane (l*2 + kv)*H + h, rows row0 .. row0+n-1 of each plane.
struct AppendParams {
  const uint16_t* src_k;
  const uint16_t* src_v;
  uint16_t* cache;
  int32_t n_layers;      // layers in the slice
  int32_t layer0;        // first cache layer written
  int32_t n_tokens;      // n
  int32_t n_heads;
  int32_t head_dim;
  int64_t plane_rows;    // C*T
  int64_t row0;          // slot*T + segment offset
  int64_t planes;        // planes of the cache (bound for debug builds)
  int* status;           // device status word (debug builds' index checks)
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

// The reverse copy of one layer's segment (readback).
struct ReadParams {
  const uint16_t* cache;
  uint16_t* dst_k;
  uint16_t* dst_v;
  int32_t layer;
  int32_t n_tokens;
  int32_t n_heads;
  int32_t head_dim;
  int64_t plane_rows;
  int64_t row0;
  int64_t planes;        // planes of the cache (bound for debug builds)
  int* status;           // device status word (debug builds' index checks)
};
cudaError_t launch_read(const ReadParams& p, cudaStream_t stream);

cudaError_t launch_euler(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream);

// Programmatic dependent launch.  The append, attention and merge kernels of a call
// are launched with programmatic stream serialization: a kernel may start while the
// previous kernel of the stream is finishing, runs its prologue (barrier setup,
// tensor-memory allocation, index arithmetic on its parameters: no global memory),
// then waits in griddep_wait() until the previous grid has completed and its writes
// are visible.  Every thread that touches global memory passes that wait.  A kernel
// calls griddep_launch_dependents() once its own prologue or main loop is done, so
// the next kernel's launch overlaps its tail; the next kernel can only start once
// every CTA of this one has been scheduled (so it cannot take an SM that one of them
// still needs).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// A launch recorded into a CUDA graph (stream capture) goes without the attribute:
// with programmatic edges in it, updating the unit program's executable graph in
// place made the host wait for the previous unit's execution.
struct PdlLaunch {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t stream) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
      cudaGetLastError();
      cs = cudaStreamCaptureStatusActive;
    }
    cfg.numAttrs = cs == cudaStreamCaptureStatusNone ? 1 : 0;
  }
};

// Host helpers.  Kernel attributes and SM counts are per device: a process may
// drive several GPUs, so every cached value is kept per device ordinal.
constexpr int kMaxDevices = 64;
int current_device();   // the current device's ordinal, or -1 (error or >= kMaxDevices)
int sm_count();         // SMs of the current device
// Test hook of ws_attention_noalloc (noalloc.cu): the V tile its CTAs leave out, -1 = none.
void set_noalloc_stall(int tile);

}  // namespace ws
