// Block-causal unit attention over the K/V history cache (sm_100a).
//
// Operation: for each head h and query row i of the current unit,
//   out[i][h] = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j
// over the key rows the query unit may see: every token of its own unit and of
// the U earlier units held in the cache (block-causal attention with one block
// per 160 ms unit, "通义实验室发布 Wan-Streamer v0.2…", remio.ai, section
// 为什么端到端模型对级联式 AI 智能体构成挑战; the cached K/V are reused, not
// recomputed, section 思考者与执行者的分工掩盖了更高分辨率的成本).  The host
// turns the visible units into runs of consecutive cache rows; rows of units
// that are not visible are never loaded (whole-unit skipping), and the last
// tile of each run masks the rows past its end.
//
// One CTA computes a 128-row query tile of one head over one range of key tiles:
//   warps 0-3  softmax: one query row per thread (= one TMEM lane), fp32 online
//              softmax in base 2, P rounded to bf16 into swizzled shared memory,
//              rescale of the O accumulator in TMEM when the running max moves
//              by more than 2^8, epilogue;
//   warp 4     TMA producer: Q once, then K and V tiles (2 stages each);
//   warp 5     MMA issuer: S = Q K^T into one of two TMEM buffers, O += P V.
// With several key ranges per (tile, head) the CTAs write fp32 partials (O, max,
// sum) and a second kernel merges them by their log-sum-exp weights.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

#include "kernels.cuh"
#include "sm100.cuh"

namespace ws {

namespace {

enum Bar : int {
  kQFull = 0,
  kKFull = 1,   // +stage
  kKEmpty = 3,  // +stage
  kVFull = 5,   // +stage
  kVEmpty = 7,  // +stage
  kSFull = 9,   // +buffer
  kSEmpty = 11, // +buffer
  kPFull = 13,
  kPVDone = 14,
  kMmaDone = 15,
  kNumBars = 16
};

constexpr int kThreads = 192;
constexpr int kTmemCols = 512;   // S buffers at columns [0,128) and [128,256), O at [256, 256+D)
constexpr int kRowBytes = 128;   // one 128-byte swizzle row = 64 bf16

template <int D>
struct Smem {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = kBlockM * D * 2;
  static constexpr int kTileBytes = kBlockN * D * 2;
  static constexpr int kPBytes = kBlockM * kBlockN * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + 2 * kTileBytes;
  static constexpr int kOffP = kOffV + 2 * kTileBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  // One CTA per SM: its 512 TMEM columns are the whole TMEM of the SM.
  static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
};

__device__ __forceinline__ void tile_info(const KeyRuns& r, int t, int& row0, int& valid) {
  int k = 0, hi = r.n_runs - 1;          // last run with tile_begin <= t
  while (k < hi) {
    const int mid = (k + hi + 1) >> 1;
    if (r.tile_begin[mid] <= t) k = mid; else hi = mid - 1;
  }
  const int local = t - r.tile_begin[k];
  row0 = r.row_begin[k] + local * kBlockN;
  valid = min(kBlockN, r.rows[k] - local * kBlockN);
}

// Bounded wait used only to drain in-flight copies and MMAs on the way out.
__device__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < (1u << 28); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 31u && global_timer_ns() - t0 > timeout_ns) return false;
  }
  return false;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    unit_attention_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap kv_map,
                          const __grid_constant__ AttnParams p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sQ = smem + S::kOffQ;
  uint8_t* sK = smem + S::kOffK;
  uint8_t* sV = smem + S::kOffV;
  uint8_t* sP = smem + S::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x % p.n_qtiles;
  const int rest = blockIdx.x / p.n_qtiles;
  const int split = rest % p.n_split;
  const int h = rest / p.n_split;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(p.runs.total_tiles, t_begin + p.tiles_per_split);
  const int n_tiles = t_end - t_begin;
  const int q0 = qt * kBlockM;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kKEmpty + s], 1);
      mbar_init(&bars[kVFull + s], 1);
      mbar_init(&bars[kVEmpty + s], 1);
      mbar_init(&bars[kSFull + s], 1);
      mbar_init(&bars[kSEmpty + s], 4);
    }
    mbar_init(&bars[kPFull], 4);
    mbar_init(&bars[kPVDone], 1);
    mbar_init(&bars[kMmaDone], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&q_map);
    prefetch_tensormap(&kv_map);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard guard{abort_flag, p.status, p.timeout_ns};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[kQFull], S::kQBytes);
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d(sQ + c * kBlockM * kRowBytes, &q_map, &bars[kQFull], c * 64, h, q0);
      int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
      bool ok = true;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i & 1;
        const uint32_t use = (uint32_t)i >> 1;
        int row0, valid;
        tile_info(p.runs, t_begin + i, row0, valid);
        if (use > 0 && !wait_phase(&bars[kKEmpty + s], (use - 1) & 1, guard)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars[kKFull + s], S::kTileBytes);
        for (int c = 0; c < S::kChunks; ++c)
          tma_load_3d(sK + s * S::kTileBytes + c * kBlockN * kRowBytes, &kv_map, &bars[kKFull + s], c * 64, row0,
                      p.plane_k + h);
        last_k[s] = i;
        if (use > 0 && !wait_phase(&bars[kVEmpty + s], (use - 1) & 1, guard)) { ok = false; break; }
        if (i != p.debug_skip_v_tile) {
          mbar_arrive_expect_tx(&bars[kVFull + s], S::kTileBytes);
          for (int c = 0; c < S::kChunks; ++c)
            tma_load_3d(sV + s * S::kTileBytes + c * kBlockN * kRowBytes, &kv_map, &bars[kVFull + s], c * 64,
                        row0, p.plane_v + h);
          last_v[s] = i;
        }
      }
      if (!ok || *abort_flag) {
        // leaving early: let every copy already issued land before the CTA exits
        drain_wait(&bars[kQFull], 0, p.timeout_ns);
        for (int s = 0; s < 2; ++s) {
          if (last_k[s] >= 0) drain_wait(&bars[kKFull + s], ((uint32_t)last_k[s] >> 1) & 1, p.timeout_ns);
          if (last_v[s] >= 0) drain_wait(&bars[kVFull + s], ((uint32_t)last_v[s] >> 1) & 1, p.timeout_ns);
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32(kBlockM, D, false, true);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV), p_base = smem_u32(sP);
      bool ok = wait_phase(&bars[kQFull], 0, guard);
      for (int i = 0; ok && i <= n_tiles; ++i) {
        if (i < n_tiles) {
          const int s = i & 1;
          if (!wait_phase(&bars[kKFull + s], ((uint32_t)i >> 1) & 1, guard)) break;
          if (i >= 2 && !wait_phase(&bars[kSEmpty + s], ((uint32_t)(i - 2) >> 1) & 1, guard)) break;
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem + (uint32_t)(s * kBlockN);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * kBlockM * kRowBytes + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * kBlockN * kRowBytes + (kk & 3) * 32);
            const uint64_t a = umma_smem_desc_sw128(q_base + off, 16, 1024);
            const uint64_t b = umma_smem_desc_sw128(k_base + s * S::kTileBytes + koff, 16, 1024);
            umma_bf16_ss(d_tmem, a, b, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[kKEmpty + s]);
          umma_commit(&bars[kSFull + s]);
        }
        if (i >= 1) {
          const int j = i - 1;
          const int s = j & 1;
          if (!wait_phase(&bars[kPFull], (uint32_t)j & 1, guard)) break;
          if (!wait_phase(&bars[kVFull + s], ((uint32_t)j >> 1) & 1, guard)) break;
          tc_fence_after_sync();
          const uint32_t o_tmem = tmem + 2 * kBlockN;
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk) {
            const uint32_t poff = (uint32_t)((kk >> 2) * kBlockM * kRowBytes + (kk & 3) * 32);
            const uint64_t a = umma_smem_desc_sw128(p_base + poff, 16, 1024);
            // V tile: MN-major B operand; 16 keys = 16 rows of 128 bytes; the next
            // 64 head-dim columns sit one chunk (kBlockN rows) further.
            const uint64_t b = umma_smem_desc_sw128(v_base + s * S::kTileBytes + kk * 16 * kRowBytes,
                                                    kBlockN * kRowBytes, 1024);
            umma_bf16_ss(o_tmem, a, b, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars[kVEmpty + s]);
          umma_commit(&bars[kPVDone]);
        }
      }
      umma_commit(&bars[kMmaDone]);
      drain_wait(&bars[kMmaDone], 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int row = threadIdx.x;  // TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t t_s = tmem + lane_base;
    const uint32_t t_o = tmem + lane_base + 2 * kBlockN;
    float m_ref = -INFINITY;  // reference max of this row, log2 units
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      ok = wait_phase(&bars[kSFull + s], ((uint32_t)j >> 1) & 1, guard);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after_sync();
      uint32_t sr[kBlockN];
      tmem_load_128(t_s + (uint32_t)(s * kBlockN), sr);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kSEmpty + s]);

      int row0, valid;
      tile_info(p.runs, t_begin + j, row0, valid);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBlockN; ++c) {
        float v = __uint_as_float(sr[c]);
        if (c >= valid) v = -INFINITY;
        sr[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      const float m_cand = mx * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (m_cand > m_ref + 8.f) {
        alpha = ex2_approx(m_ref - m_cand);
        l_sum *= alpha;
        m_ref = m_cand;
        rescale = true;
      }
      const float neg_m = -m_ref;
      float rs = 0.f;
      uint32_t packed[kBlockN / 2];
#pragma unroll
      for (int c = 0; c < kBlockN / 2; ++c) {
        const float a = ex2_approx(fmaf(__uint_as_float(sr[2 * c]), p.scale_log2, neg_m));
        const float b = ex2_approx(fmaf(__uint_as_float(sr[2 * c + 1]), p.scale_log2, neg_m));
        rs += a + b;
        packed[c] = pack_bf16x2(a, b);
      }
      l_sum += rs;

      if (j > 0) {
        // the previous P.V has finished: the P buffer is free and O is stable
        ok = wait_phase(&bars[kPVDone], (uint32_t)(j - 1) & 1, guard);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_load_32(t_o + (uint32_t)c, o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_store_32(t_o + (uint32_t)c, o);
          }
        }
      }
      // P row -> shared memory, K-major with the 128-byte swizzle: 16-byte piece
      // `pc` of a 128-byte row lands at position pc ^ (row & 7).
#pragma unroll
      for (int c16 = 0; c16 < kBlockN / 8; ++c16) {
        const int chunk = c16 >> 3, piece = c16 & 7;
        uint8_t* dst = sP + chunk * kBlockM * kRowBytes + row * kRowBytes + ((piece ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(packed[4 * c16], packed[4 * c16 + 1], packed[4 * c16 + 2], packed[4 * c16 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kPFull]);
    }

    if (ok) {
      ok = wait_phase(&bars[kPVDone], (uint32_t)(n_tiles - 1) & 1, guard);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after_sync();
      const int q_row = q0 + row;
      if (p.n_split == 1) {
        const float inv = 1.f / l_sum;
        uint16_t* dst = p.out + ((size_t)q_row * p.n_heads + h) * D;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_load_32(t_o + (uint32_t)c, o);
          if (q_row < p.n_query) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + c + 8 * k) = w;
            }
          }
        }
      } else {
        const size_t rows_pad = (size_t)p.n_qtiles * kBlockM;
        const size_t base = ((size_t)split * p.n_heads + h) * rows_pad + (size_t)q_row;
        float* po = p.part_o + base * D;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_load_32(t_o + (uint32_t)c, o);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(po + c + 4 * k) = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
        }
        *reinterpret_cast<float2*>(p.part_ml + base * 2) = make_float2(m_ref, l_sum);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge of the split-K partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One warp per (row, head); each lane owns D/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ AttnParams p) {
  constexpr int kPer = D / 32;
  const int gw = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.n_query * p.n_heads) return;
  const int row = gw / p.n_heads;
  const int h = gw - row * p.n_heads;
  const size_t rows_pad = (size_t)p.n_qtiles * kBlockM;
  float m_all = -INFINITY;
  for (int s = 0; s < p.n_split; ++s)
    m_all = fmaxf(m_all, p.part_ml[(((size_t)s * p.n_heads + h) * rows_pad + row) * 2]);
  float l_all = 0.f;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  for (int s = 0; s < p.n_split; ++s) {
    const size_t base = ((size_t)s * p.n_heads + h) * rows_pad + row;
    const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + base * 2);
    const float w = ex2_approx(ml.x - m_all);
    l_all += w * ml.y;
    const float* po = p.part_o + base * D + lane * kPer;
    if constexpr (kPer == 4) {
      const float4 o = *reinterpret_cast<const float4*>(po);
      acc[0] += w * o.x; acc[1] += w * o.y; acc[2] += w * o.z; acc[3] += w * o.w;
    } else {
      const float2 o = *reinterpret_cast<const float2*>(po);
      acc[0] += w * o.x; acc[1] += w * o.y;
    }
  }
  const float inv = 1.f / l_all;
  uint16_t* dst = p.out + ((size_t)row * p.n_heads + h) * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* sym = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &sym, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(sym);
  }
  return fn;
}

}  // namespace

int encode_kv_map(CUtensorMap* map, const void* kv, int head_dim, int64_t rows, int64_t planes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)rows * head_dim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kBlockN, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int encode_q_map(CUtensorMap* map, const void* q, int head_dim, int n_heads, int n_query) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)n_heads, (cuuint64_t)n_query};
  const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)n_heads * head_dim * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlockM};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

template <int D>
static cudaError_t launch_attention_d(const CUtensorMap& q_map, const CUtensorMap& kv_map, const AttnParams& p,
                                      int* ctas, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(unit_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<D>::kAlloc);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = p.n_qtiles * p.n_heads * p.n_split;
  if (ctas) *ctas = grid;
  unit_attention_kernel<D><<<grid, kThreads, Smem<D>::kAlloc, stream>>>(q_map, kv_map, p);
  return cudaGetLastError();
}

cudaError_t launch_attention(const CUtensorMap& q_map, const CUtensorMap& kv_map, const AttnParams& p, int head_dim,
                             int* ctas, cudaStream_t stream) {
  if (head_dim == 128) return launch_attention_d<128>(q_map, kv_map, p, ctas, stream);
  if (head_dim == 64) return launch_attention_d<64>(q_map, kv_map, p, ctas, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const AttnParams& p, int head_dim, cudaStream_t stream) {
  const long long warps = (long long)p.n_query * p.n_heads;
  const int grid = (int)((warps * 32 + 255) / 256);
  if (head_dim == 128)
    combine_kernel<128><<<grid, 256, 0, stream>>>(p);
  else if (head_dim == 64)
    combine_kernel<64><<<grid, 256, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace ws
