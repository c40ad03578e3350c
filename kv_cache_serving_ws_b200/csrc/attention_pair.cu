// Block-causal unit attention, head_dim 128, on pairs of SMs (sm_100a).
//
// Same operation, visibility rule and work decomposition as attention.cu:
//   out[i][h] = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j
// over the key rows the query unit may see -- every token of its own unit and of
// the U earlier units held in the cache (block-causal attention with one block
// per 160 ms unit, "通义实验室发布 Wan-Streamer v0.2…", remio.ai, section
// 为什么端到端模型对级联式 AI 智能体构成挑战).  The host turns the visible units
// into runs of consecutive cache rows; rows of units that are not visible are
// never loaded, and the last tile of each run masks the rows past its end.
//
// A worker of the stream-K decomposition is a cluster of two CTAs on two SMs.
// Item = (query unit, block of 256 query rows, head); CTA rank r of the pair owns
// query rows [128 r, 128 r + 128) of the block.  The leader (rank 0) issues every
// tensor-core product as one M = 256 tcgen05.mma.cta_group::2:
//   S = Q K^T      A = Q (each CTA its 128 rows), B = K tile: the leader holds
//                  keys 0-63 of the 128-key tile, the peer keys 64-127;
//   O += P V       A = P from each SM's TMEM, B = V tile: the leader holds head
//                  columns 0-63 of all 128 keys, the peer columns 64-127.
// So one K/V tile serves 256 query rows while each SM stores only half of it,
// and each SM's 512 TMEM columns hold O (128) plus three S buffers: the tensor
// core computes S(g+1) and S(g+2) while the softmax works on S(g), so the
// softmax is no longer waiting on the products of its own previous tile.
//
// Roles in each CTA (256 threads):
//   warps 0-3  softmax of this CTA's 128 rows (one row per thread = TMEM lane):
//              fp32 online softmax in base 2 with a lazily moved reference max,
//              P rounded to bf16 into the TMEM columns of its own S; the
//              rescale of O when the reference moves; each item's epilogue;
//   warp 4     TMA producer of Q (two buffers) and of this CTA's half of every
//              K tile (four stages);
//   warp 5     TMA producer of this CTA's half of every V tile (three stages);
//              in a partial tile it zeroes the value rows past the run's end;
//   warp 6     leader: issues every P.V product; both CTAs: TMEM allocation;
//   warp 7     leader: issues every S product.
// Issuing one M = 256 product takes the issuing warp longer than the tensor core
// takes to run it, so the two kinds of product come from two warps.  S(g+3)
// overwrites the S buffer whose P the product P.V(g) reads: the S warp waits for
// that product's completion (a commit) before it issues S(g+3).
// TMEM (each SM): O [0,128), S buffer b at [128 + 128 b, 256 + 128 b).
//
// Cross-CTA signalling: copies of both CTAs complete on the leader's "full"
// barriers (cta_group::2 TMA with the leader's barrier), the leader's commits
// arrive on both CTAs' barriers (one commit per barrier, the peer's addressed
// through the shared::cluster window), and the peer's softmax and V producer
// arrive remotely on the leader's barriers.  Those remote arrivals are plain
// counts: P and O live in TMEM, ordered by tcgen05.wait and the tcgen05
// thread-sync fences, and V halves by their transaction bytes -- except a
// partial V tile whose rows the peer zeroed with ordinary stores, which it
// reports with a release at cluster scope that the leader acquires.  Every wait
// is bounded; a wait that runs out raises the abort flag of both CTAs and
// stores a status for ws_sync.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>

#include "attn_common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace ws {

namespace {

constexpr int kPD = 128;            // head_dim of this kernel
constexpr int kSBufs = 3;           // S buffers in TMEM
constexpr int kKStages = 4;
constexpr int kVStages = 3;
constexpr int kSoftWarps = 4;
constexpr int kKWarp = 4;
constexpr int kVWarp = 5;
constexpr int kPvWarp = 6;
constexpr int kSWarp = 7;
constexpr int kPairThreads = 32 * 8;
constexpr int kRowB = 128;          // one 128-byte swizzle row = 64 bf16

enum PBar : int {
  pQFull = 0,       // +2  leader: Q of both CTAs (tx)
  pQEmpty = 2,      // +2  both: Q buffer free (leader's commit)
  pKFull = 4,       // +4  leader: K halves of both CTAs (tx)
  pKEmpty = 8,      // +4  both
  pVFull = 12,      // +3  leader: two arrivals (one per CTA) + tx of both halves
  pVEmpty = 15,     // +3  both
  pVLocal = 18,     // +3  both: a partial tile's V half, loaded to be zeroed
  pSFull = 21,      // +3  both
  pPFull = 24,      // +3  leader: 8 warps (4 per CTA)
  pPVDone = 27,     // +2  both: P.V of tiles with this parity
  pOFull = 29,      //     both: O of an item complete
  pOFree = 30,      //     leader: 8 warps have read O
  pPvDone = 31,     //     leader: every P.V product complete (leaving)
  pSBufFree = 32,   // +3  leader: P.V of the buffer's tile complete
  pSDone = 35,      //     leader: every S product complete (leaving)
  pNumBars = 36
};

struct PSmem {
  static constexpr int kQBytes = 128 * kPD * 2;       // this CTA's 128 query rows
  static constexpr int kKBytes = 64 * kPD * 2;        // 64 keys x 128 columns
  static constexpr int kVBytes = 128 * 64 * 2;        // 128 keys x 64 columns
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKBytes;
  static constexpr int kOffBar = kOffV + kVStages * kVBytes;
  static constexpr int kOffMisc = kOffBar + pNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int N>
struct RingPos {
  int idx = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next() {
    if (++idx == N) {
      idx = 0;
      ph ^= 1u;
    }
  }
};

// Abort state of a pair: the local flag, the peer's flag (cluster address), the status word.
struct PairGuard {
  volatile int* abort_flag;
  uint32_t peer_abort;
  int* status;
  uint64_t timeout_ns;
};

// Waits acquire at CTA scope, except pair_wait_cluster (see the signalling notes).
__device__ __noinline__ bool pair_wait_slow(uint64_t* bar, uint32_t parity, const PairGuard& g, bool cluster) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < (1u << 28); ++it) {
    if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 31u) {
      if (*g.abort_flag) return false;
      if (global_timer_ns() - t0 > g.timeout_ns) break;
    }
  }
  *g.abort_flag = 1;
  st_cluster_u32(g.peer_abort, 1u);
  atomicCAS(g.status, 0, kStatusTimeout);
  return false;
}
__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, const PairGuard& g) {
  if (mbar_try_wait(bar, parity)) return true;
  return pair_wait_slow(bar, parity, g, false);
}
__device__ __forceinline__ bool pair_wait_cluster(uint64_t* bar, uint32_t parity, const PairGuard& g) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  return pair_wait_slow(bar, parity, g, true);
}
__device__ __forceinline__ bool pair_warp_wait(uint64_t* bar, uint32_t parity, const PairGuard& g) {
  return __all_sync(0xffffffffu, pair_wait(bar, parity, g));
}
__device__ __forceinline__ bool pair_warp_wait_cluster(uint64_t* bar, uint32_t parity, const PairGuard& g) {
  return __all_sync(0xffffffffu, pair_wait_cluster(bar, parity, g));
}

// P = 2^(s * log2(e)/sqrt(D) - m) of one row's 128 S values, packed to bf16 pairs in pk,
// the fp32 sums in four chains of pairs.
__device__ __forceinline__ void softmax_pairs(const uint32_t (&sr)[kBlockN], uint64_t scale2, uint64_t negm2,
                                              uint64_t (&rs2)[4], uint32_t (&pk)[kBlockN / 2]) {
#pragma unroll
  for (int c = 0; c < kBlockN / 2; ++c) {
    const uint64_t x = fma_f32x2(f32x2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale2, negm2);
    float x0, x1;
    f32x2_split(x, x0, x1);
    const float e0 = ex2_approx(x0);
    const float e1 = ex2_approx(x1);
    rs2[c & 3] = add_f32x2(rs2[c & 3], f32x2(e0, e1));
    pk[c] = pack_bf16x2(e0, e1);
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    pair_attention_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                          const __grid_constant__ CUtensorMap v_map, const __grid_constant__ AttnParams p) {
  using S = PSmem;
  const Decomp& d = p.dec;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1);
  Range rg;
  rg.lane = pair / d.lane_ctas;
  rg.idx = pair - rg.lane * d.lane_ctas;
  rg.gq = lane_qtiles(d, rg.lane);
  {
    const long long per = lane_per(d, rg.lane);
    const long long work = lane_work(d, rg.lane);
    rg.start = (long long)rg.idx * per;
    const long long end = rg.start + per < work ? rg.start + per : work;
    rg.len = end > rg.start ? (int)(end - rg.start) : 0;
  }
  if (rg.len == 0) return;                 // both CTAs of the pair: nothing allocated yet

  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;          // the same offset in both CTAs (same kernel, same layout)
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
    for (int i = 0; i < pNumBars; ++i) {
      uint32_t count = 1;
      if (i >= pVFull && i < pVFull + kVStages) count = 2;
      if ((i >= pPFull && i < pPFull + kSBufs) || i == pOFree) count = 2 * kSoftWarps;
      mbar_init(&bars[i], count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kPvWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (warp == kKWarp && lane == 0) {
    prefetch_tensormap(&q_map);
    prefetch_tensormap(&k_map);
    prefetch_tensormap(&v_map);
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();                      // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t lead_bar0 = mapa_shared(bar0, 0);     // the leader's barriers, cluster addresses
  const uint32_t peer_bar0 = mapa_shared(bar0, 1);     // the peer's barriers
  auto lead_bar = [&](int i) { return lead_bar0 + (uint32_t)(i * 8); };
  auto peer_bar = [&](int i) { return peer_bar0 + (uint32_t)(i * 8); };
  const PairGuard guard{abort_flag, mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u), p.status,
                        p.timeout_ns};

  if (warp == kKWarp) {
    if (lane == 0) {
      // ------------------------------------------------ Q and K producer
      int issued_q[2] = {-1, -1}, issued_k[kKStages];
      for (int i = 0; i < kKStages; ++i) issued_k[i] = -1;
      RingPos<kKStages> kr;
      TileIter it;
      it.init(d, p.qu, p.runs, rg);
      bool ok = true;
      for (int g = 0; g < len && ok; ++g, it.next(p.qu, p.runs)) {
        if (it.first) {
          const int qb = it.n & 1;
          if (it.n >= 2 && !pair_wait(&bars[pQEmpty + qb], (uint32_t)((it.n >> 1) - 1) & 1, guard)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&bars[pQFull + qb], 2 * S::kQBytes);
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(sQ + qb * S::kQBytes + c * 128 * kRowB, &q_map, lead_bar(pQFull + qb), c * 64, it.h,
                             it.j * p.qu.rows + it.qt() * kItemRows + (int)rank * kBlockM);
          issued_q[qb] = it.n;
        }
        it.check_run(p);
        if (g >= kKStages && !pair_wait(&bars[pKEmpty + kr.idx], kr.ph ^ 1u, guard)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(&bars[pKFull + kr.idx], 2 * S::kKBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_3d_pair(sK + kr.idx * S::kKBytes + c * 64 * kRowB, &k_map, lead_bar(pKFull + kr.idx), c * 64,
                           it.row0() + (int)rank * 64, p.plane_k + it.h);
        issued_k[kr.idx] = g;
        kr.next();
      }
      if (!ok || *abort_flag) {
        // leaving early: the leader waits (bounded) for the copies it expected,
        // which count both CTAs' bytes; the peer gives its own copies time to land
        if (leader) {
          for (int qb = 0; qb < 2; ++qb)
            if (issued_q[qb] >= 0) drain_wait(&bars[pQFull + qb], (uint32_t)(issued_q[qb] >> 1) & 1, p.timeout_ns);
          for (int i = 0; i < kKStages; ++i)
            if (issued_k[i] >= 0) drain_wait(&bars[pKFull + i], (uint32_t)(issued_k[i] / kKStages) & 1, p.timeout_ns);
        } else {
          __nanosleep(100000);
        }
      }
    }
  } else if (warp == kVWarp) {
    // ------------------------------------------------------ V producer
    RingPos<kVStages> vr;
    uint32_t local_ph = 0;                 // phase bits of the pVLocal barriers, one per stage
    int issued_local[kVStages];
    for (int i = 0; i < kVStages; ++i) issued_local[i] = 0;
    TileIter it;
    it.init(d, p.qu, p.runs, rg);
    bool ok = true;
    for (int g = 0; g < len && ok; ++g, it.next(p.qu, p.runs)) {
      if (g >= kVStages && !pair_warp_wait(&bars[pVEmpty + vr.idx], vr.ph ^ 1u, guard)) {
        ok = false;
        break;
      }
      const int valid = it.valid();
      uint8_t* dst = sV + vr.idx * S::kVBytes;
      if (g == p.debug_skip_v_tile) {
        // test hook: this tile's V never arrives, so the MMA warp's wait runs out
      } else if ((valid & 15) == 0) {
        // two arrivals: the leader's (with the bytes of both halves), the peer's
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&bars[pVFull + vr.idx], 2 * S::kVBytes);
          tma_load_3d_pair(dst, &v_map, lead_bar(pVFull + vr.idx), (int)rank * 64, it.row0(), p.plane_v + it.h);
          if (!leader) mbar_arrive_cluster_relaxed(lead_bar(pVFull + vr.idx));
        }
      } else {
        // Rows of this tile past the end of the run belong to keys the query must
        // not see; their P is 0, but 0 * inf or 0 * NaN is NaN in the product.  The
        // P.V loop stops at the 16-key step holding the run's last key, and the
        // rows of that step past the run's end are zeroed here, before the leader
        // is told that this half of the tile is ready.
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[pVLocal + vr.idx], S::kVBytes);
          tma_load_3d(dst, &v_map, &bars[pVLocal + vr.idx], (int)rank * 64, it.row0(), p.plane_v + it.h);
        }
        issued_local[vr.idx] = 1;
        const uint32_t par = (local_ph >> vr.idx) & 1u;
        local_ph ^= 1u << vr.idx;
        if (!pair_warp_wait(&bars[pVLocal + vr.idx], par, guard)) {
          ok = false;
          break;
        }
        issued_local[vr.idx] = 0;
        const int nz = 16 - (valid & 15);                 // rows [valid, valid + nz)
        for (int i = lane; i < nz * 8; i += 32)
          *reinterpret_cast<uint4*>(dst + (valid + (i >> 3)) * kRowB + (i & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(&bars[pVFull + vr.idx]);
          else
            mbar_arrive_cluster(lead_bar(pVFull + vr.idx));
        }
      }
      vr.next();
    }
    // one decision for the whole warp (lanes may read the abort flag at different times)
    if (__any_sync(0xffffffffu, !ok || *abort_flag)) {
      if (lane == 0) {
        for (int i = 0; i < kVStages; ++i)
          if (issued_local[i]) drain_wait(&bars[pVLocal + i], ((local_ph >> i) & 1u) ^ 1u, p.timeout_ns);
        __nanosleep(100000);               // copies counted on the leader's barriers
      }
      __syncwarp();
    }
  } else if (warp == kPvWarp || warp == kSWarp) {
    if (leader) {
      // ---------------------------------------------------- MMA issuers
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto commit_both = [&](int i) {
        if (elect_one()) {
          umma_commit_pair(lead_bar(i));
          umma_commit_pair(peer_bar(i));
        }
      };
      TileIter it;
      it.init(d, p.qu, p.runs, rg);
      RingPos<kSBufs> sb;
      bool ok = true;
      if (warp == kSWarp) {
        // S(g) = Q K(g)^T into S buffer g mod 3, once P.V(g-3) has read that buffer's P
        constexpr uint32_t idesc_s = umma_idesc_bf16_f32(256, kBlockN, false, false);
        RingPos<kKStages> kr;
        for (int g = 0; ok && g < len; ++g, it.next(p.qu, p.runs)) {
          const int qb = it.n & 1;
          if (g >= kSBufs && !pair_warp_wait(&bars[pSBufFree + sb.idx], sb.ph ^ 1u, guard)) ok = false;
          if (ok && it.first && !pair_warp_wait(&bars[pQFull + qb], (uint32_t)(it.n >> 1) & 1, guard)) ok = false;
          if (ok && !pair_warp_wait(&bars[pKFull + kr.idx], kr.ph, guard)) ok = false;
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem + 128u + 128u * (uint32_t)sb.idx;
          // descriptors of the chunk starts; a K step adds its byte offset / 16 to the address field
          const uint64_t da0 = umma_smem_desc_sw128(q_base + qb * S::kQBytes, 16, 1024);
          const uint64_t db0 = umma_smem_desc_sw128(k_base + kr.idx * S::kKBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kPD / 16; ++kk) {
            const uint32_t qoff = (uint32_t)((kk >> 2) * 128 * kRowB + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * 64 * kRowB + (kk & 3) * 32);
            const uint64_t da = da0 + (uint64_t)(qoff >> 4);
            const uint64_t db = db0 + (uint64_t)(koff >> 4);
            if (elect_one()) umma_bf16_ss_pair(d_tmem, da, db, idesc_s, kk > 0 ? 1u : 0u);
          }
          commit_both(pSFull + sb.idx);
          commit_both(pKEmpty + kr.idx);
          if (it.last) commit_both(pQEmpty + qb);
          sb.next();
          kr.next();
        }
        if (elect_one()) umma_commit_pair(lead_bar(pSDone));
        drain_wait(&bars[pSDone], 0, p.timeout_ns);
      } else {
        // O += P(g) V(g), P in the TMEM columns of its S buffer, two bf16 per column
        constexpr uint32_t idesc_o = umma_idesc_bf16_f32(256, kPD, false, true);
        RingPos<kVStages> vr;
        for (int g = 0; ok && g < len; ++g, it.next(p.qu, p.runs)) {
          const int valid = it.valid();
          // a partial tile's V rows were zeroed by ordinary stores, in the peer too
          if ((valid & 15) != 0) ok = pair_warp_wait_cluster(&bars[pVFull + vr.idx], vr.ph, guard);
          else ok = pair_warp_wait(&bars[pVFull + vr.idx], vr.ph, guard);
          if (ok && !pair_warp_wait(&bars[pPFull + sb.idx], sb.ph, guard)) ok = false;
          if (ok && it.first && it.n > 0 && !pair_warp_wait(&bars[pOFree], (uint32_t)(it.n - 1) & 1, guard)) ok = false;
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t p_tmem = tmem + 128u + 128u * (uint32_t)sb.idx;
          const int steps = (valid + 15) >> 4;
          const uint64_t dv0 = umma_smem_desc_sw128(v_base + vr.idx * S::kVBytes, 128 * kRowB, 1024);
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk) {
            if (kk >= steps) break;
            // 16 keys = 8 TMEM columns of P; V: 16 rows of 128 bytes
            const uint64_t db = dv0 + (uint64_t)((kk * 16 * kRowB) >> 4);
            if (elect_one()) umma_bf16_ts_pair(tmem, p_tmem + (uint32_t)(kk * 8), db, idesc_o, (!it.first || kk > 0) ? 1u : 0u);
          }
          if (elect_one()) umma_commit_pair(lead_bar(pSBufFree + sb.idx));
          commit_both(pVEmpty + vr.idx);
          commit_both(pPVDone + (g & 1));
          if (it.last) commit_both(pOFull);
          sb.next();
          vr.next();
        }
        if (elect_one()) umma_commit_pair(lead_bar(pPvDone));
        drain_wait(&bars[pPvDone], 0, p.timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x & 127;       // TMEM lane = query row of this CTA
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base;
    float m_ref = -INFINITY;                 // reference max of this row, log2 units
    float l_sum = 0.f;
    RingPos<kSBufs> sb;
    TileIter it;
    it.init(d, p.qu, p.runs, rg);
    const uint64_t scale2 = f32x2(p.scale_log2, p.scale_log2);
    for (int g = 0; g < len; ++g, it.next(p.qu, p.runs)) {
      if (it.first) {
        m_ref = -INFINITY;
        l_sum = 0.f;
      }
      if (!__all_sync(0xffffffffu, pair_wait(&bars[pSFull + sb.idx], sb.ph, guard))) break;
      tc_fence_after_sync();
      const uint32_t t_s = tmem + 128u + 128u * (uint32_t)sb.idx + lane_base;
      const int valid = it.valid();
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
      // the tile from S, still intact in TMEM; a row whose own sum triggered it
      // moves its reference to the row max.
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
        softmax_pairs(sr, scale2, negm2, rs2, pk);
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
        // row max: 8 independent chains, two-input max over columns 0..15, then
        // three-input max over each further group of 16 columns
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[8 + k]));
#pragma unroll
        for (int c = 16; c < kBlockN; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx[k] = max3_f32(mx[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
        const float m_cand =
            max3_f32(max3_f32(mx[0], mx[1], mx[2]), max3_f32(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
            p.scale_log2;
        move = it.first || m_cand > m_ref + 8.f || (hot && m_cand > m_ref);
        if (move) {
          alpha = ex2_approx(m_ref - m_cand);
          l_sum *= alpha;
          m_ref = m_cand;
        }
        const uint64_t negm2 = f32x2(-m_ref, -m_ref);
#pragma unroll
        for (int k = 0; k < 4; ++k) rs2[k] = f32x2(0.f, 0.f);
        softmax_pairs(sr, scale2, negm2, rs2, pk);
      }
      {
        float rs[8];
        f32x2_split(rs2[0], rs[0], rs[1]);
        f32x2_split(rs2[1], rs[2], rs[3]);
        f32x2_split(rs2[2], rs[4], rs[5]);
        f32x2_split(rs2[3], rs[6], rs[7]);
        l_sum += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      }
      tmem_store_64(t_s, pk);                // keys 2c, 2c+1 -> column c of the S buffer
      if (__any_sync(0xffffffffu, move && !it.first)) {
        // O holds the products up to tile g-1; P.V(g-1) may still be running
        if (!__all_sync(0xffffffffu, pair_wait(&bars[pPVDone + ((g - 1) & 1)], (uint32_t)((g - 1) >> 1) & 1, guard)))
          break;
        tc_fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < kPD; c += 32) {
          uint32_t o[32];
          tmem_load_32(t_o + (uint32_t)c, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_store_32(t_o + (uint32_t)c, o);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&bars[pPFull + sb.idx]);
        else
          mbar_arrive_cluster_relaxed(lead_bar(pPFull + sb.idx));
      }
      sb.next();

      if (it.last) {
        // ---- epilogue of the item: this CTA's 128 rows of the 256-row block
        if (!__all_sync(0xffffffffu, pair_wait(&bars[pOFull], (uint32_t)it.n & 1, guard))) break;
        tc_fence_after_sync();
        const int a = (int)rank;
        const int r_unit = it.qt() * kItemRows + a * kBlockM + row;   // row within the query unit
        int lane_i, c_first, pieces, end0;
        item_span(d, p.qu, it.j, it.qt(), it.h, lane_i, c_first, pieces, end0);
        const float inv = 1.f / l_sum;
        const bool in_unit =
            r_unit < p.qu.rows && index_ok((int64_t)it.j * p.qu.rows + r_unit < p.out_rows, p.status);
        uint16_t* dst = p.out + ((size_t)(it.j * p.qu.rows + r_unit) * p.n_heads + it.h) * kPD;
        size_t prow = 0;
        bool part_ok = true;
        if (pieces > 1) {
          // this worker's first item takes slot (worker, 0), any later one slot (worker, 1)
          const size_t slot = partial_slot(d, rg.lane, rg.idx, it.n == 0 ? 0 : 1);
          prow = slot * kItemRows + (size_t)(a * kBlockM + row);
          part_ok = index_ok(slot < (size_t)p.part_slots, p.status);
          if (part_ok) *reinterpret_cast<float2*>(p.part_ml + prow * 2) = make_float2(m_ref, l_sum);
        }
#pragma unroll 1
        for (int c = 0; c < kPD; c += 32) {
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
            float* po = p.part_o + prow * kPD + c;
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<uint4*>(po + k) = make_uint4(o[k], o[k + 1], o[k + 2], o[k + 3]);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(&bars[pOFree]);
          else
            mbar_arrive_cluster_relaxed(lead_bar(pOFree));
        }
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
            if (in_unit) merge_row<kPD>(p, lane_i, c_first, pieces, end0, a * kBlockM + row, dst);
          }
        }
      }
    }
  }

  // Neither CTA leaves (or frees TMEM) while the other may still signal its barriers
  // or, for the leader's products, write its TMEM.
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  if (warp == kPvWarp) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Pairs that can be resident at once on this device with the kernel's shared
// memory (one CTA per SM): the number of workers of a decomposition.
std::atomic<int> g_pair_workers[kMaxDevices];

}  // namespace

int pair_workers() {
  const int dev = current_device();
  if (dev < 0) return 0;
  int n = g_pair_workers[dev].load(std::memory_order_acquire);
  if (n != 0) return n > 0 ? n : 0;
  n = -1;
  if (cudaFuncSetAttribute(pair_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PSmem::kAlloc) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (unsigned)sm_count(), 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = PSmem::kAlloc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, pair_attention_kernel, &cfg) == cudaSuccess && clusters > 0)
      n = clusters;
  }
  cudaGetLastError();
  g_pair_workers[dev].store(n, std::memory_order_release);
  return n > 0 ? n : 0;
}

cudaError_t launch_attention_pair(const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                                  const AttnParams& p, int* ctas, cudaStream_t stream) {
  if (pair_workers() <= 0) return cudaErrorInvalidConfiguration;
  const int grid = 2 * p.dec.lanes * p.dec.lane_ctas;
  if (ctas) *ctas = grid;
  pair_attention_kernel<<<grid, kPairThreads, PSmem::kAlloc, stream>>>(q_map, k_map, v_map, p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess && std::getenv("WS_DEBUG")) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, pair_attention_kernel);
    std::fprintf(stderr, "ws: pair attention launch failed: %s (grid %d, block %d, smem %d; kernel regs %d)\n",
                 cudaGetErrorString(e), grid, kPairThreads, PSmem::kAlloc, fa.numRegs);
  }
  return e;
}

}  // namespace ws
