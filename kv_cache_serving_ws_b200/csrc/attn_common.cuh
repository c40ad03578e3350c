// Device-side pieces shared by the attention kernels (attention.cu, attention_pair.cu):
// the per-worker tile iterator of the stream-K decomposition, the bounded drain wait
// and the merge of one row of an item cut between workers.  A "worker" is a CTA of
// the single-SM kernel or a CTA pair of the paired kernel; Decomp counts workers.
#pragma once
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.cuh"
#include "sm100.cuh"

namespace ws {

// Walks a worker's iterations in order: head h, query block of the lane a, query
// unit j, key tile t, item ordinal n, and the key tile's run (first row, valid
// rows) -- all kept in registers and advanced incrementally, so the hot loops do
// no divisions and no indexed parameter loads except when a run or an item ends.
struct Range {
  int lane, idx, gq;        // lane, worker index in the lane, query blocks of the lane
  long long start;          // first lane iteration
  int len;                  // iterations of this worker
};
struct TileIter {
  int g, len, tiles, gq, qt0, n_units;
  int a, h, j, t, tiles_j, n;
  int run, run_off, run_row0, run_rows, run_new;
  bool first, last;
  __device__ __forceinline__ int qt() const { return qt0 + a; }
  __device__ __forceinline__ int row0() const { return run_row0 + run_off; }
  __device__ __forceinline__ int valid() const { return min(kBlockN, run_rows - run_off); }
  __device__ __forceinline__ void flags() {
    first = (g == 0) || (t == 0);
    last = (g == len - 1) || (t == tiles_j - 1);
  }
  __device__ __forceinline__ void load_run(const KeyRuns& r) {
    run_row0 = r.row_begin[run];
    run_rows = r.rows[run];
    run_new = r.from_new[run];
  }
  // debug builds: the current run lies inside the K/V planes (or inside k_new / v_new,
  // whose rows are those of out), and so does head h's plane
  __device__ __forceinline__ void check_run(const AttnParams& p) const {
    const int64_t lim = run_new ? p.out_rows : p.plane_rows;
    index_ok(run_row0 >= 0 && run_rows > 0 && (int64_t)run_row0 + run_rows <= lim && (!run_new || p.fold) &&
                 h >= 0 && h < p.n_heads && p.plane_k + h < p.planes && p.plane_v + h < p.planes,
             p.status);
  }
  __device__ void init(const Decomp& d, const QueryUnits& u, const KeyRuns& r, const Range& rg) {
    g = 0;
    len = rg.len;
    tiles = d.tiles;
    gq = rg.gq;
    qt0 = rg.lane * d.group;
    n_units = u.n_units;
    const long long grp = rg.start / tiles;
    const int rem = (int)(rg.start - grp * tiles);
    h = (int)(grp / gq);
    a = (int)(grp - (long long)h * gq);
    j = 0;
    while (j + 1 < n_units && u.tile_start[j + 1] <= rem) ++j;
    t = rem - u.tile_start[j];
    tiles_j = u.tile_start[j + 1] - u.tile_start[j];
    n = 0;
    run = u.run_first[j];
    while (run + 1 < u.run_first[j + 1] && r.tile_begin[run + 1] <= t) ++run;
    run_off = (t - r.tile_begin[run]) * kBlockN;
    load_run(r);
    flags();
  }
  __device__ __forceinline__ void next(const QueryUnits& u, const KeyRuns& r) {
    ++g;
    ++t;
    run_off += kBlockN;
    if (t == tiles_j) {
      t = 0;
      ++n;
      if (++j == n_units) {
        j = 0;
        if (++a == gq) {
          a = 0;
          ++h;
        }
      }
      tiles_j = u.tile_start[j + 1] - u.tile_start[j];
      run = u.run_first[j];
      run_off = 0;
      load_run(r);
    } else if (run_off >= run_rows) {
      ++run;
      run_off = 0;
      load_run(r);
    }
    flags();
  }
};


// Bounded wait used only to drain in-flight copies and MMAs on the way out.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < (1u << 28); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 31u && global_timer_ns() - t0 > timeout_ns) return false;
  }
  return false;
}

// Merge of the partials of one row of an item cut between workers:
//   out = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k,   M = max_k m_k.
// Piece k was written by CTA c_first + k of the lane: its last item for k = 0
// (unless the item starts exactly at that CTA's range), its first item
// otherwise.  The partials were written by other SMs in this launch: read them
// through L2 only.
template <int D>
static __device__ __noinline__ void merge_row(const AttnParams& p, int lane_i, int c_first, int pieces, int end0, int r,
                                              uint16_t* dst) {
  constexpr int kCached = 8;                 // pieces whose (m, l) stay in registers
  auto row_of = [&](int k) -> size_t {
    return partial_slot(p.dec, lane_i, c_first + k, k == 0 ? end0 : 0) * kItemRows + r;
  };
  if (!index_ok(partial_slot(p.dec, lane_i, c_first + pieces - 1, 0) < (size_t)p.part_slots && r < kItemRows,
                p.status))
    return;
  // every piece's (reference max, sum): independent loads, one round trip
  float2 ml[kCached];
  float m_all = -INFINITY;
#pragma unroll
  for (int k = 0; k < kCached; ++k) {
    ml[k] = k < pieces ? __ldcg(reinterpret_cast<const float2*>(p.part_ml + row_of(k) * 2)) : make_float2(-INFINITY, 0.f);
    m_all = fmaxf(m_all, ml[k].x);
  }
  for (int k = kCached; k < pieces; ++k) m_all = fmaxf(m_all, __ldcg(p.part_ml + row_of(k) * 2));
  float w[kCached];
  float l_all = 0.f;
#pragma unroll
  for (int k = 0; k < kCached; ++k) {
    w[k] = k < pieces ? ex2_approx(ml[k].x - m_all) : 0.f;
    l_all += w[k] * ml[k].y;
  }
  for (int k = kCached; k < pieces; ++k) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(p.part_ml + row_of(k) * 2));
    l_all += ex2_approx(v.x - m_all) * v.y;
  }
  const float inv = 1.f / l_all;
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    float acc[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) acc[k] = 0.f;
    // two pieces' 32 columns in flight per round trip
#pragma unroll 1
    for (int k = 0; k < pieces; k += 2) {
      const bool two = k + 1 < pieces;
      const float4* p0 = reinterpret_cast<const float4*>(p.part_o + row_of(k) * D + c);
      const float4* p1 = reinterpret_cast<const float4*>(p.part_o + row_of(two ? k + 1 : k) * D + c);
      float4 o0[8], o1[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        o0[q] = __ldcg(p0 + q);
        o1[q] = two ? __ldcg(p1 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const float w0 = k < kCached ? w[k] : ex2_approx(__ldcg(p.part_ml + row_of(k) * 2) - m_all);
      const float w1 = !two ? 0.f : (k + 1 < kCached ? w[k + 1] : ex2_approx(__ldcg(p.part_ml + row_of(k + 1) * 2) - m_all));
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        acc[4 * q + 0] += w0 * o0[q].x + w1 * o1[q].x;
        acc[4 * q + 1] += w0 * o0[q].y + w1 * o1[q].y;
        acc[4 * q + 2] += w0 * o0[q].z + w1 * o1[q].z;
        acc[4 * q + 3] += w0 * o0[q].w + w1 * o1[q].w;
      }
    }
#pragma unroll
    for (int k = 0; k < 32; k += 8) {
      uint4 v;
      v.x = pack_bf16x2(acc[k + 0] * inv, acc[k + 1] * inv);
      v.y = pack_bf16x2(acc[k + 2] * inv, acc[k + 3] * inv);
      v.z = pack_bf16x2(acc[k + 4] * inv, acc[k + 5] * inv);
      v.w = pack_bf16x2(acc[k + 6] * inv, acc[k + 7] * inv);
      *reinterpret_cast<uint4*>(dst + c + k) = v;
    }
  }
}

}  // namespace ws
