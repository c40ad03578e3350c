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
// Persistent kernel, one CTA per SM, stream-K style: every CTA gets the same
// number of (Q block, head, key tile) iterations (see Decomp); an item cut
// between CTAs is merged by whichever of them finishes its share last.  A CTA works on a
// block of two 128-row query tiles of one head at a time:
//   warpgroup 0, 1  softmax of query tile 0 and 1: one query row per thread (=
//              one TMEM lane); fp32 online softmax in base 2 with a lazily moved
//              reference max, taken only when a row's P sum shows it may have to
//              move; P is rounded to bf16 and written back into the TMEM
//              columns of its own S (A operand of the P.V product); epilogue of
//              each item;
//   warp 8     TMA producer: the two Q tiles of each item, K and V tiles (2 stages);
//   warp 9     MMA issuer: S_a = Q_a K^T (A and B from shared memory) and
//              O_a += P_a V (A from TMEM, V as an MN-major B operand), ordered
//              PV0(j), S0(j+1), PV1(j), S1(j+1): while one warpgroup runs its
//              softmax the tensor core works on the other tile's products.  The
//              whole warp runs the issue loop, so descriptors stay warp-uniform,
//              and one elected lane executes each tcgen05 instruction: issued from
//              a lone thread, a 128x128x16 MMA took about 85 cycles instead of 64.
// TMEM: S0 [0,128), O0 [128,128+D), S1 [256,384), O1 [384,384+D).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <string>
#include <type_traits>

#include "attn_common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace ws {

namespace {

enum Bar : int {
  kQFull = 0,
  kQEmpty = 1,
  kKFull = 2,    // +stage
  kKEmpty = 4,   // +stage
  kVFull = 6,    // +stage
  kVEmpty = 8,   // +stage
  kSFull = 10,   // +Q tile
  kPFull = 12,   // +Q tile
  kOFull = 14,   // +Q tile
  kOFree = 16,   // +Q tile
  kMmaDone = 18,
  kNumBars = 19
};

constexpr int kSoftmaxWarps = 4 * kQTiles;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kCopyWarp = kSoftmaxWarps + 2;   // writes the call's latent K/V into the cache
// 352 threads, one CTA per SM: three warps share some SM sub-partitions, which
// caps a thread at 168 registers; the softmax fits without spills.
constexpr int kThreads = 32 * (kSoftmaxWarps + 3);
constexpr int kTmemCols = 512;
constexpr int kRowBytes = 128;   // one 128-byte swizzle row = 64 bf16

template <int D>
struct Smem {
  static constexpr int kChunks = D / 64;
  static constexpr int kQTileBytes = kBlockM * D * 2;
  static constexpr int kTileBytes = kBlockN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQTiles * kQTileBytes;
  static constexpr int kOffV = kOffK + 2 * kTileBytes;
  static constexpr int kOffBar = kOffV + 2 * kTileBytes;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  // one CTA per SM: its 512 TMEM columns are all of the SM's TMEM
  static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
};

__device__ __forceinline__ uint32_t tmem_s(uint32_t base, int a) { return base + (uint32_t)(a * 256); }
__device__ __forceinline__ uint32_t tmem_o(uint32_t base, int a) { return base + (uint32_t)(a * 256 + 128); }

// The latent write folded into the attention launch: the call's k_new / v_new token
// rows [n_units*Nq][H][D] go to plane rows latent_row0[j] + t of planes plane_k + h
// (K) and plane_v + h (V) -- the in-place cache write of the unit's K/V slice
// ("Wan-Streamer v0.2：更高分辨率，相同延迟", paper.rainbus.top, section 前置知识, entry
// K/V缓存预分片).  The key tiles of those rows are loaded from k_new / v_new anyway;
// every whole tile is stored from shared memory by TMA (store_latent_tiles below), once
// per (head, tile).  This function copies the rest: each unit's last Nq % 128 rows,
// which no whole tile covers.  CTA b of the grid takes an equal share of those rows
// (K rows, then V rows); `nthr` threads of it walk the share's 16-byte vectors, four
// loads in flight per thread.  Nothing in the launch reads these cache rows.
template <int D>
__device__ void copy_latent_tail(const AttnParams& p, int tid, int nthr) {
  constexpr int kVd = D / 8;                  // 16-byte vectors per head row
  constexpr int kDepth = 4;
  const int nq = p.qu.rows;
  const int t0 = (nq / kBlockN) * kBlockN;    // first row not covered by a whole tile
  const int tail = nq - t0;
  const int rows_all = p.qu.n_units * tail;
  const int row_vecs = p.n_heads * kVd;
  const int total = 2 * rows_all;
  if (total == 0) return;
  const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
  const int r0 = (int)blockIdx.x * per;
  const int r1 = min(total, r0 + per);
  if (r0 >= r1) return;
  const int nv = (r1 - r0) * row_vecs;
  for (int f0 = tid; f0 < nv; f0 += kDepth * nthr) {
    uint4 v[kDepth];
    uint4* dst[kDepth];
#pragma unroll
    for (int u = 0; u < kDepth; ++u) {
      const int f = f0 + u * nthr;
      dst[u] = nullptr;
      if (f < nv) {
        const int r = r0 + f / row_vecs;
        const int e = f - (r - r0) * row_vecs;
        const int kv = r >= rows_all ? 1 : 0;
        const int rr = r - kv * rows_all;
        const int j = rr / tail;
        const int t = t0 + (rr - j * tail);   // row within unit j
        const int64_t row = p.latent_row0[j] + t;
        const int h = e / kVd;
        const int64_t plane = (int64_t)(kv ? p.plane_v : p.plane_k) + h;
        if (index_ok(row >= 0 && row < p.plane_rows && plane < p.planes, p.status)) {
          const size_t tok = (size_t)j * nq + t;
          v[u] = ld_global_nc_v4(reinterpret_cast<const uint4*>(kv ? p.v_new : p.k_new) + tok * row_vecs + e);
          dst[u] = reinterpret_cast<uint4*>(p.cache + ((size_t)plane * p.plane_rows + row) * D) + (e - h * kVd);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kDepth; ++u)
      if (dst[u]) *dst[u] = v[u];
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    unit_attention_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap kv_map,
                          const __grid_constant__ CUtensorMap knew_map, const __grid_constant__ CUtensorMap vnew_map,
                          const __grid_constant__ AttnParams p) {
  using S = Smem<D>;
  const Decomp& d = p.dec;
  Range rg;
  rg.lane = blockIdx.x / d.lane_ctas;
  rg.idx = blockIdx.x - rg.lane * d.lane_ctas;
  rg.gq = lane_qtiles(d, rg.lane);
  {
    const long long per = lane_per(d, rg.lane);
    const long long work = lane_work(d, rg.lane);
    rg.start = (long long)rg.idx * per;
    const long long end = rg.start + per < work ? rg.start + per : work;
    rg.len = end > rg.start ? (int)(end - rg.start) : 0;
  }
  if (rg.len == 0) {                       // whole CTA: nothing allocated yet
    griddep_wait();                        // (every CTA completes after the previous grid)
    if (p.fold) copy_latent_tail<D>(p, threadIdx.x, kThreads);
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sQ = smem + S::kOffQ;
  uint8_t* sK = smem + S::kOffK;
  uint8_t* sV = smem + S::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int len = rg.len;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kQEmpty], 1);
    // with the fold, a stage is free once the MMAs and the latent store are done with it
    const uint32_t empty_count = p.fold ? 2 : 1;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kKEmpty + s], empty_count);
      mbar_init(&bars[kVFull + s], 1);
      mbar_init(&bars[kVEmpty + s], empty_count);
    }
    for (int a = 0; a < kQTiles; ++a) {
      mbar_init(&bars[kSFull + a], 1);
      mbar_init(&bars[kPFull + a], 4);
      mbar_init(&bars[kOFull + a], 1);
      mbar_init(&bars[kOFree + a], 4);
    }
    mbar_init(&bars[kMmaDone], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&q_map);
    prefetch_tensormap(&kv_map);
    if (p.fold) {
      prefetch_tensormap(&knew_map);
      prefetch_tensormap(&vnew_map);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard guard{abort_flag, p.status, p.timeout_ns};
  griddep_wait();   // Q, the cache and the partials may be in use by the previous kernel

  if (warp >= kSoftmaxWarps) {
    if (warp == kProducerWarp && lane == 0) {
      // ---------------------------------------------------------- producer
      int last_k[2] = {-1, -1}, last_v[2] = {-1, -1}, last_q = -1;
      bool ok = true;
      TileIter it;
      it.init(d, p.qu, p.runs, rg);
      for (int g = 0; g < len && ok; ++g, it.next(p.qu, p.runs)) {
        if (it.first) {
          if (it.n > 0 && !wait_phase(&bars[kQEmpty], (uint32_t)(it.n - 1) & 1, guard)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars[kQFull], kQTiles * S::kQTileBytes);
          for (int a = 0; a < kQTiles; ++a)
            for (int c = 0; c < S::kChunks; ++c)
              tma_load_3d(sQ + a * S::kQTileBytes + c * kBlockM * kRowBytes, &q_map, &bars[kQFull], c * 64, it.h,
                          it.j * p.qu.rows + it.qt() * kItemRows + a * kBlockM);
          last_q = it.n;
        }
        const int s = g & 1;
        const uint32_t use = (uint32_t)g >> 1;
        const int row0 = it.row0();
        it.check_run(p);
        if (use > 0 && !wait_phase(&bars[kKEmpty + s], (use - 1) & 1, guard)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars[kKFull + s], S::kTileBytes);
        for (int c = 0; c < S::kChunks; ++c) {
          uint8_t* dst = sK + s * S::kTileBytes + c * kBlockN * kRowBytes;
          if (it.run_new)   // the call's own latent rows: k_new [rows][H][D]
            tma_load_3d(dst, &knew_map, &bars[kKFull + s], c * 64, it.h, row0);
          else
            tma_load_3d(dst, &kv_map, &bars[kKFull + s], c * 64, row0, p.plane_k + it.h);
        }
        last_k[s] = g;
        if (use > 0 && !wait_phase(&bars[kVEmpty + s], (use - 1) & 1, guard)) { ok = false; break; }
        if (g != p.debug_skip_v_tile) {
          mbar_arrive_expect_tx(&bars[kVFull + s], S::kTileBytes);
          for (int c = 0; c < S::kChunks; ++c) {
            uint8_t* dst = sV + s * S::kTileBytes + c * kBlockN * kRowBytes;
            if (it.run_new)
              tma_load_3d(dst, &vnew_map, &bars[kVFull + s], c * 64, it.h, row0);
            else
              tma_load_3d(dst, &kv_map, &bars[kVFull + s], c * 64, row0, p.plane_v + it.h);
          }
          last_v[s] = g;
        }
      }
      if (!ok || *abort_flag) {
        // leaving early: let every copy already issued land before the CTA exits
        if (last_q >= 0) drain_wait(&bars[kQFull], (uint32_t)last_q & 1, p.timeout_ns);
        for (int s = 0; s < 2; ++s) {
          if (last_k[s] >= 0) drain_wait(&bars[kKFull + s], ((uint32_t)last_k[s] >> 1) & 1, p.timeout_ns);
          if (last_v[s] >= 0) drain_wait(&bars[kVFull + s], ((uint32_t)last_v[s] >> 1) & 1, p.timeout_ns);
        }
      }
    } else if (warp == kCopyWarp && p.fold) {
      // ------------------------------------------------- latent write (fold)
      copy_latent_tail<D>(p, lane, 32);
      __syncwarp();
      if (lane == 0) {
        // Follows the producer's stages: once a stage's K and V have landed, a whole
        // tile of the call's own latent rows, seen by query block 0, is stored to its
        // cache rows (each (head, tile) once); then the stage is released.
        bool ok = true;
        TileIter it;
        it.init(d, p.qu, p.runs, rg);
        for (int g = 0; g < len && ok; ++g, it.next(p.qu, p.runs)) {
          const int s = g & 1;
          const uint32_t ph = ((uint32_t)g >> 1) & 1;
          const bool store = it.run_new && it.qt() == 0 && it.valid() == kBlockN;
          const int64_t row = p.latent_row0[it.j] + (it.row0() - it.j * p.qu.rows);
          const bool row_ok = !store || index_ok(row >= 0 && row + kBlockN <= p.plane_rows, p.status);
          if (!wait_phase(&bars[kKFull + s], ph, guard)) { ok = false; break; }
          if (store && row_ok) {
            fence_proxy_async_smem();
            for (int c = 0; c < S::kChunks; ++c)
              tma_store_3d(&kv_map, sK + s * S::kTileBytes + c * kBlockN * kRowBytes, c * 64, (int32_t)row,
                           p.plane_k + it.h);
          }
          if (!wait_phase(&bars[kVFull + s], ph, guard)) { ok = false; break; }
          if (store && row_ok) {
            for (int c = 0; c < S::kChunks; ++c)
              tma_store_3d(&kv_map, sV + s * S::kTileBytes + c * kBlockN * kRowBytes, c * 64, (int32_t)row,
                           p.plane_v + it.h);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
          mbar_arrive(&bars[kKEmpty + s]);
          mbar_arrive(&bars[kVEmpty + s]);
        }
        bulk_wait_group0();
      }
    } else if (warp == kMmaWarp) {
      // -------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32(kBlockM, D, false, true);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      // S_a(g) = Q_a K(g)^T
      auto issue_s = [&](const TileIter& it, int a) -> bool {
        const int s = it.g & 1;
        if (a == 0) {
          if (it.first && !warp_wait(&bars[kQFull], (uint32_t)it.n & 1, guard)) return false;
          if (!warp_wait(&bars[kKFull + s], ((uint32_t)it.g >> 1) & 1, guard)) return false;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_s(tmem, a);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kBlockM * kRowBytes + (kk & 3) * 32);
          const uint32_t koff = (uint32_t)((kk >> 2) * kBlockN * kRowBytes + (kk & 3) * 32);
          const uint64_t da = umma_smem_desc_sw128(q_base + a * S::kQTileBytes + off, 16, 1024);
          const uint64_t db = umma_smem_desc_sw128(k_base + s * S::kTileBytes + koff, 16, 1024);
          if (elect_one()) umma_bf16_ss(d_tmem, da, db, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (elect_one()) umma_commit(&bars[kSFull + a]);
        if (a == kQTiles - 1) {
          if (elect_one()) umma_commit(&bars[kKEmpty + s]);
          if (it.last && elect_one()) umma_commit(&bars[kQEmpty]);
        }
        return true;
      };
      // O_a += P_a(g) V(g), P_a in the TMEM columns of S_a, two bf16 per column.
      // Rows of a partial tile past the end of its run belong to keys the query
      // must not see (another unit's slot, stale latent rows, another session):
      // their P is 0, but 0 * inf or 0 * NaN is NaN in the product.  The K loop
      // stops at the 16-key step that holds the last visible key, and the rows of
      // that step past the run's end are zeroed in shared memory first.
      auto issue_pv = [&](const TileIter& it, int a) -> bool {
        const int s = it.g & 1;
        const int valid = it.valid();
        if (a == 0) {
          if (!warp_wait(&bars[kVFull + s], ((uint32_t)it.g >> 1) & 1, guard)) return false;
          if (valid & 15) {
            const int r0 = valid, nz = 16 - (valid & 15);          // rows [r0, r0 + nz)
            for (int i = lane; i < nz * S::kChunks * 8; i += 32) {
              const int c = i / (nz * 8), rem = i - c * nz * 8;
              uint8_t* dst = sV + s * S::kTileBytes + c * kBlockN * kRowBytes + (r0 + rem / 8) * kRowBytes +
                             (rem & 7) * 16;
              *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
        }
        if (!warp_wait(&bars[kPFull + a], (uint32_t)it.g & 1, guard)) return false;
        if (it.first && it.n > 0 && !warp_wait(&bars[kOFree + a], (uint32_t)(it.n - 1) & 1, guard)) return false;
        tc_fence_after_sync();
        const uint32_t o_tmem = tmem_o(tmem, a);
        const uint32_t p_tmem = tmem_s(tmem, a);
        // 16 keys = 8 TMEM columns; V: 16 rows of 128 bytes, the next 64 head-dim
        // columns one chunk (kBlockN rows) further
        auto pv_step = [&](int kk) {
          const uint64_t db = umma_smem_desc_sw128(v_base + s * S::kTileBytes + kk * 16 * kRowBytes,
                                                   kBlockN * kRowBytes, 1024);
          if (elect_one()) umma_bf16_ts(o_tmem, p_tmem + (uint32_t)(kk * 8), db, idesc_o, (!it.first || kk > 0) ? 1u : 0u);
        };
        if (valid == kBlockN) {
          // whole tile (all but a run's last): the 8 steps with no per-step test
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk) pv_step(kk);
        } else {
          // a run's last tile: stop after the 16-key step holding its last valid row
          const int steps = (valid + 15) >> 4;
#pragma unroll 1
          for (int kk = 0; kk < steps; ++kk) pv_step(kk);
        }
        if (it.last && elect_one()) umma_commit(&bars[kOFull + a]);
        if (a == kQTiles - 1 && elect_one()) umma_commit(&bars[kVEmpty + s]);
        return true;
      };
      TileIter it_s, it_pv;                  // it_s runs one iteration ahead of it_pv
      it_s.init(d, p.qu, p.runs, rg);
      it_pv = it_s;
      bool ok = issue_s(it_s, 0) && issue_s(it_s, 1);
      for (int g = 0; ok && g < len; ++g) {
        const bool more = g + 1 < len;
        if (more) it_s.next(p.qu, p.runs);
        ok = issue_pv(it_pv, 0);
        if (ok && more) ok = issue_s(it_s, 0);
        if (ok) ok = issue_pv(it_pv, 1);
        if (ok && more) ok = issue_s(it_s, 1);
        it_pv.next(p.qu, p.runs);
      }
      if (elect_one()) umma_commit(&bars[kMmaDone]);
      drain_wait(&bars[kMmaDone], 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int a = warp >> 2;                 // query tile of this warpgroup
    const int row = threadIdx.x & 127;       // TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem_s(tmem, a) + lane_base;
    const uint32_t t_o = tmem_o(tmem, a) + lane_base;
    float m_ref = -INFINITY;  // reference max of this row, log2 units
    float l_sum = 0.f;
    bool ok = true;
    TileIter it;
    it.init(d, p.qu, p.runs, rg);
    for (int g = 0; g < len; ++g, it.next(p.qu, p.runs)) {
      if (it.first) {
        m_ref = -INFINITY;
        l_sum = 0.f;
      }
      // S_a(g) complete; it was issued after P_a(g-1) V, which is complete too
      ok = wait_phase(&bars[kSFull + a], (uint32_t)g & 1, guard);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after_sync();
      const int valid = it.valid();
      const uint64_t scale2 = f32x2(p.scale_log2, p.scale_log2);
      uint64_t rs2[4];
      uint32_t pk[kBlockN / 2];
      float alpha = 1.f;
      bool move = false;
      // Past an item's first tile the reference max rarely moves, so P is first
      // computed against the current reference without taking the row max.  The
      // reference must move only if some P exceeds 2^8, and then the fp32 sum of
      // the row's P reaches 2^8 too (a rounded sum of positive terms is never
      // below its largest term; the threshold 255 leaves room for the error of
      // ex2.approx).  Only a warp with such a row takes the max and recomputes
      // the tile from S, still intact in TMEM (P is written back after the
      // check); a row whose own sum triggered it moves its reference to the row
      // max, so that a slowly rising max cannot trigger a recomputation on every
      // tile.  Whenever no row sum reaches 255, P, the sums and the reference are
      // exactly those of taking the max first.
      bool redo = it.first;
      bool hot = false;
      if (!it.first) {
        uint32_t sr[kBlockN];
        tmem_load_128(t_s, sr);
        if (valid < kBlockN) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
        }
        const uint64_t negm2 = f32x2(-m_ref, -m_ref);
#pragma unroll
        for (int k = 0; k < 4; ++k) rs2[k] = f32x2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kBlockN / 2; ++c) {
          const float s0 = __uint_as_float(sr[2 * c]), s1 = __uint_as_float(sr[2 * c + 1]);
          const uint64_t x = fma_f32x2(f32x2(s0, s1), scale2, negm2);
          float x0, x1;
          f32x2_split(x, x0, x1);
          const float e0 = ex2_approx(x0);
          const float e1 = ex2_approx(x1);
          rs2[c & 3] = add_f32x2(rs2[c & 3], f32x2(e0, e1));
          pk[c] = pack_bf16x2(e0, e1);
        }
        float rs[8];
        f32x2_split(rs2[0], rs[0], rs[1]);
        f32x2_split(rs2[1], rs[2], rs[3]);
        f32x2_split(rs2[2], rs[4], rs[5]);
        f32x2_split(rs2[3], rs[6], rs[7]);
        const float tile_sum = ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        hot = !(tile_sum < 255.f);
        redo = __any_sync(0xffffffffu, hot);
      }
      if (redo) {
        uint32_t sr[kBlockN];
        tmem_load_128(t_s, sr);
        if (valid < kBlockN) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
        }
        // row max: 4 independent chains of three-input max (8 chains need more
        // registers than the 168 a thread has here)
        float mx[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) mx[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[4 + k]));
#pragma unroll
        for (int c = 8; c < kBlockN; c += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mx[k] = max3_f32(mx[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 4 + k]));
        static_assert(kBlockN % 8 == 0, "the row max takes the columns in groups of 8");
        const float m_cand = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
        // Move the reference max when P would exceed 2^8, for a new item, or to
        // the row max when this row's sum triggered the recomputation.
        move = it.first || m_cand > m_ref + 8.f || (hot && m_cand > m_ref);
        if (move) {
          alpha = ex2_approx(m_ref - m_cand);
          l_sum *= alpha;
          m_ref = m_cand;
        }
        // P = 2^(s * log2(e)/sqrt(D) - m): scale and shift on fp32 pairs, one ex2
        // per element, sums on fp32 pairs (4 independent chains)
        const uint64_t negm2 = f32x2(-m_ref, -m_ref);
#pragma unroll
        for (int k = 0; k < 4; ++k) rs2[k] = f32x2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kBlockN / 2; ++c) {
          const uint64_t x =
              fma_f32x2(f32x2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale2, negm2);
          float x0, x1;
          f32x2_split(x, x0, x1);
          const float e0 = ex2_approx(x0);
          const float e1 = ex2_approx(x1);
          rs2[c & 3] = add_f32x2(rs2[c & 3], f32x2(e0, e1));
          pk[c] = pack_bf16x2(e0, e1);
        }
      }
      float rs[8];
      f32x2_split(rs2[0], rs[0], rs[1]);
      f32x2_split(rs2[1], rs[2], rs[3]);
      f32x2_split(rs2[2], rs[4], rs[5]);
      f32x2_split(rs2[3], rs[6], rs[7]);
      l_sum += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      tmem_store_64(t_s, pk);                // keys 2c, 2c+1 -> column c of S_a
      if (__any_sync(0xffffffffu, move && !it.first)) {
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_load_32(t_o + (uint32_t)c, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_store_32(t_o + (uint32_t)c, o);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kPFull + a]);

      if (it.last) {
        // ---- epilogue of the item (qt, h), rows of query tile a
        ok = wait_phase(&bars[kOFull + a], (uint32_t)it.n & 1, guard);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after_sync();
        const int r_unit = it.qt() * kItemRows + a * kBlockM + row;   // row within the query unit
        int lane_i, c_first, pieces, end0;
        item_span(d, p.qu, it.j, it.qt(), it.h, lane_i, c_first, pieces, end0);
        const float inv = 1.f / l_sum;
        const bool in_unit =
            r_unit < p.qu.rows && index_ok((int64_t)it.j * p.qu.rows + r_unit < p.out_rows, p.status);
        uint16_t* dst = p.out + ((size_t)(it.j * p.qu.rows + r_unit) * p.n_heads + it.h) * D;
        size_t prow = 0;
        bool part_ok = true;
        if (pieces > 1) {
          // this CTA's first item takes slot (cta, 0), any later one slot (cta, 1)
          const size_t slot = partial_slot(d, rg.lane, rg.idx, it.n == 0 ? 0 : 1);
          prow = slot * kItemRows + (size_t)(a * kBlockM + row);
          part_ok = index_ok(slot < (size_t)p.part_slots, p.status);
          if (part_ok) *reinterpret_cast<float2*>(p.part_ml + prow * 2) = make_float2(m_ref, l_sum);
        }
        // O in 32-column chunks: bf16 output of a whole item, fp32 partial otherwise
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_load_32(t_o + (uint32_t)c, o);
          if (pieces == 1) {
            if (in_unit) {
#pragma unroll
              for (int k = 0; k < 32; k += 8) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[k + 0]) * inv, __uint_as_float(o[k + 1]) * inv);
                v.y = pack_bf16x2(__uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
                v.z = pack_bf16x2(__uint_as_float(o[k + 4]) * inv, __uint_as_float(o[k + 5]) * inv);
                v.w = pack_bf16x2(__uint_as_float(o[k + 6]) * inv, __uint_as_float(o[k + 7]) * inv);
                *reinterpret_cast<uint4*>(dst + c + k) = v;
              }
            }
          } else if (part_ok) {
            float* po = p.part_o + prow * D + c;
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<uint4*>(po + k) = make_uint4(o[k], o[k + 1], o[k + 2], o[k + 3]);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kOFree + a]);
        if (pieces > 1 && p.fixup) {
          // Stream-K fix-up: the last piece of the item to arrive merges these 32
          // rows from the pieces' partials (counted per warp: no block barrier).
          __threadfence();
          __syncwarp();
          const size_t ci =
              ((((size_t)it.j * d.n_qtiles + it.qt()) * p.n_heads + it.h) * kQTiles + a) * kFixPerTile + (warp & 3);
          int last = 0;
          if (lane == 0 && index_ok(ci < (size_t)p.fix_slots && part_ok, p.status))
            last = atomicAdd(p.fix_count + ci, 1) == pieces - 1;
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            if (lane == 0) p.fix_count[ci] = 0;
            __threadfence();
            if (in_unit) merge_row<D>(p, lane_i, c_first, pieces, end0, a * kBlockM + row, dst);
          }
        }
      }
    }
  }

  griddep_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge of the partials of items cut between CTAs as a separate launch (calls
// whose CTAs run few iterations, see AttnParams::fixup):
//   out = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k,   M = max_k m_k.
// One warp per output row, each lane D/32 consecutive columns; a block takes 8 rows
// of one item (query unit j, query block qt, head h).  The kernel is latency-bound
// (one or two waves of short warps), so a warp issues its loads in one round trip:
// lane k loads piece k's (max, sum) pair while every lane loads its columns of the
// first kPre pieces' partial rows; the weights then come from warp shuffles.
constexpr int kMergeRowsPerBlock = 8;
template <int D>
__global__ void __launch_bounds__(32 * kMergeRowsPerBlock) merge_kernel(const __grid_constant__ AttnParams p) {
  constexpr int kPer = D / 32;
  constexpr int kPre = 4;
  constexpr int kChunks = kItemRows / kMergeRowsPerBlock;
  using Vec = typename std::conditional<kPer == 4, float4, float2>::type;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x / kChunks;                   // (j * n_qtiles + qt) * H + h
  const int chunk = blockIdx.x - item * kChunks;
  griddep_launch_dependents();
  const int h = item % p.n_heads;
  const int jq = item / p.n_heads;
  const int qt = jq % p.dec.n_qtiles;
  const int j = jq / p.dec.n_qtiles;
  int lane_i, c_first, pieces, end0;
  item_span(p.dec, p.qu, j, qt, h, lane_i, c_first, pieces, end0);
  const int r = chunk * kMergeRowsPerBlock + warp;         // row within the item's block
  const int r_unit = qt * kItemRows + r;
  griddep_wait();                                          // the partials of the attention kernel
  if (pieces == 1 || r_unit >= p.qu.rows) return;          // pieces == 1: written directly by its CTA
  const int64_t row = (int64_t)j * p.qu.rows + r_unit;
  if (!index_ok(partial_slot(p.dec, lane_i, c_first + pieces - 1, 0) < (size_t)p.part_slots && row < p.out_rows,
                p.status))
    return;
  // piece k was written by CTA c_first + k: its last item for k = 0 (unless the
  // item starts exactly at that CTA's range), its first item otherwise
  auto prow_of = [&](int k) -> size_t {
    return partial_slot(p.dec, lane_i, c_first + k, k == 0 ? end0 : 0) * kItemRows + r;
  };
  auto load_cols = [&](int k) -> Vec {
    return __ldcg(reinterpret_cast<const Vec*>(p.part_o + prow_of(k) * D) + lane);
  };
  auto fma_cols = [](float* acc, float w, const Vec& v) {
    if constexpr (kPer == 4) {
      acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
    } else {
      acc[0] += w * v.x; acc[1] += w * v.y;
    }
  };
  // 1. one round trip: (m, l) of pieces 0..31 and the first kPre partial rows
  const float2 ml0 = lane < pieces ? __ldcg(reinterpret_cast<const float2*>(p.part_ml + prow_of(lane) * 2))
                                   : make_float2(-INFINITY, 0.f);
  Vec pre[kPre];
#pragma unroll
  for (int k = 0; k < kPre; ++k) pre[k] = k < pieces ? load_cols(k) : Vec{};
  // 2. M over all pieces (more than 32 only for very small per-CTA ranges)
  float m_all = ml0.x;
  for (int k0 = 32; k0 < pieces; k0 += 32)
    if (k0 + lane < pieces) m_all = fmaxf(m_all, __ldcg(p.part_ml + prow_of(k0 + lane) * 2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m_all = fmaxf(m_all, __shfl_xor_sync(0xffffffffu, m_all, o));
  // 3. weights 2^(m_k - M), the weighted rows and the weighted sums
  float w = lane < pieces ? ex2_approx(ml0.x - m_all) : 0.f;
  float l_all = w * ml0.y;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
#pragma unroll
  for (int k = 0; k < kPre; ++k) fma_cols(acc, __shfl_sync(0xffffffffu, w, k), pre[k]);
  const int n0 = pieces < 32 ? pieces : 32;
#pragma unroll 4
  for (int k = kPre; k < n0; ++k) fma_cols(acc, __shfl_sync(0xffffffffu, w, k), load_cols(k));
  for (int k0 = 32; k0 < pieces; k0 += 32) {
    const int n = pieces - k0 < 32 ? pieces - k0 : 32;
    const float2 ml = lane < n ? __ldcg(reinterpret_cast<const float2*>(p.part_ml + prow_of(k0 + lane) * 2))
                               : make_float2(-INFINITY, 0.f);
    w = lane < n ? ex2_approx(ml.x - m_all) : 0.f;
    l_all += w * ml.y;
#pragma unroll 4
    for (int k = 0; k < n; ++k) fma_cols(acc, __shfl_sync(0xffffffffu, w, k), load_cols(k0 + k));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l_all += __shfl_xor_sync(0xffffffffu, l_all, o);
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

int encode_kv_map_box(CUtensorMap* map, const void* kv, int head_dim, int64_t rows, int64_t planes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)rows * head_dim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
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
static cudaError_t launch_attention_d(const CUtensorMap& q_map, const CUtensorMap& kv_map,
                                      const CUtensorMap* new_maps, const AttnParams& p, int* ctas,
                                      cudaStream_t stream) {
  // the shared-memory opt-in is a per-device attribute of the kernel
  static std::atomic<bool> configured[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(unit_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<D>::kAlloc);
    if (e != cudaSuccess) return e;
    configured[dev].store(true, std::memory_order_release);
  }
  const int grid = p.dec.lanes * p.dec.lane_ctas;
  if (ctas) *ctas = grid;
  PdlLaunch l(dim3(grid), dim3(kThreads), Smem<D>::kAlloc, stream);
  // without the fold the k_new / v_new maps are never read: q_map stands in for them
  const CUtensorMap& km = p.fold ? new_maps[0] : q_map;
  const CUtensorMap& vm = p.fold ? new_maps[1] : q_map;
  const cudaError_t e = cudaLaunchKernelEx(&l.cfg, unit_attention_kernel<D>, q_map, kv_map, km, vm, p);
  if (e != cudaSuccess && std::getenv("WS_DEBUG")) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, unit_attention_kernel<D>);
    std::fprintf(stderr, "ws: attention launch failed: %s (grid %d, block %d, smem %d; kernel regs %d, max threads %d)\n",
                 cudaGetErrorString(e), grid, kThreads, Smem<D>::kAlloc, fa.numRegs, fa.maxThreadsPerBlock);
  }
  return e;
}

namespace {
// head_dim 128 runs on the single-SM kernel, which is the faster of the two on
// every measured shape; WS_ATTENTION_KERNEL=pair (read once per process) selects
// the kernel on pairs of SMs (attention_pair.cu) instead, where the device can
// hold its clusters.
bool use_pair_kernel(int head_dim) {
  static const bool pair = [] {
    const char* e = std::getenv("WS_ATTENTION_KERNEL");
    return e && std::string(e) == "pair";
  }();
  return head_dim == 128 && pair && pair_workers() > 0;
}
}  // namespace

int attention_workers(int head_dim) { return use_pair_kernel(head_dim) ? pair_workers() : sm_count(); }
bool attention_uses_pairs(int head_dim) { return use_pair_kernel(head_dim); }

cudaError_t launch_attention(const CUtensorMap& q_map, const CUtensorMap& kv_map, const CUtensorMap& k_half_map,
                             const CUtensorMap* new_maps, const AttnParams& p, int head_dim, int* ctas,
                             cudaStream_t stream) {
  if (p.fold && !new_maps) return cudaErrorInvalidValue;
  if (use_pair_kernel(head_dim)) {
    if (p.fold) return cudaErrorInvalidValue;   // the paired kernel reads the cache only
    return launch_attention_pair(q_map, k_half_map, kv_map, p, ctas, stream);
  }
  if (head_dim == 128) return launch_attention_d<128>(q_map, kv_map, new_maps, p, ctas, stream);
  if (head_dim == 64) return launch_attention_d<64>(q_map, kv_map, new_maps, p, ctas, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge(const AttnParams& p, int head_dim, cudaStream_t stream) {
  const long long items = (long long)p.qu.n_units * p.dec.n_qtiles * p.n_heads;
  const int grid = (int)(items * (kItemRows / kMergeRowsPerBlock));
  PdlLaunch l(dim3(grid), dim3(32 * kMergeRowsPerBlock), 0, stream);
  if (head_dim == 128) return cudaLaunchKernelEx(&l.cfg, merge_kernel<128>, p);
  if (head_dim == 64) return cudaLaunchKernelEx(&l.cfg, merge_kernel<64>, p);
  return cudaErrorInvalidValue;
}

}  // namespace ws
