// Internal launch interface between the C ABI (ws_api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ws {

constexpr int kBlockM = 128;   // query rows per CTA (one TMEM lane each)
constexpr int kBlockN = 128;   // keys per tile
constexpr int kMaxRuns = 192;  // visible row runs per attention call (>= slots of any ring with gaps)
constexpr int kMaxSplits = 16;

// Visible key rows of one (layer, head) plane: runs of consecutive rows, cut
// into kBlockN-row tiles; tile_begin[r] is the first global tile of run r.
struct KeyRuns {
  int32_t n_runs;
  int32_t total_tiles;
  int32_t row_begin[kMaxRuns];
  int32_t rows[kMaxRuns];
  int32_t tile_begin[kMaxRuns + 1];
};

struct AttnParams {
  int32_t n_query;          // Nq
  int32_t n_heads;          // H
  int32_t n_qtiles;         // ceil(Nq / kBlockM)
  int32_t n_split;          // key-range splits (1 = write bf16 output directly)
  int32_t tiles_per_split;
  int32_t plane_k;          // KV-map plane index of head 0's K of this layer
  int32_t plane_v;          // same for V
  float scale_log2;         // log2(e) / sqrt(D)
  uint16_t* out;            // [Nq][H][D] bf16, when n_split == 1
  float* part_o;            // [n_split][H][n_qtiles*kBlockM][D] fp32, when n_split > 1
  float* part_ml;           // [n_split][H][n_qtiles*kBlockM][2]  (running max in log2 units, sum)
  int* status;              // device status word
  uint64_t timeout_ns;      // bound of every wait
  int32_t debug_skip_v_tile;  // test hook: never load V of this local tile (-1 = off)
  KeyRuns runs;
};

// Encodes the tensor maps used by the attention kernel.  `kv` points at the
// cache planes [planes][rows][D]; `q` at [Nq][H][D].
int encode_kv_map(CUtensorMap* map, const void* kv, int head_dim, int64_t rows, int64_t planes);
int encode_q_map(CUtensorMap* map, const void* q, int head_dim, int n_heads, int n_query);

cudaError_t launch_attention(const CUtensorMap& q_map, const CUtensorMap& kv_map, const AttnParams& p,
                             int head_dim, int* ctas, cudaStream_t stream);
cudaError_t launch_combine(const AttnParams& p, int head_dim, cudaStream_t stream);

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
};
cudaError_t launch_read(const ReadParams& p, cudaStream_t stream);

cudaError_t launch_euler(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream);

int sm_count();

}  // namespace ws
