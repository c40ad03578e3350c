// Fused flow-matching Euler update of a bf16 latent, in place:
//   x <- RN_bf16( fl64( x + fl64(dt * v) ) )
// ("Wan-Streamer v0.2：更高分辨率，相同延迟", paper.rainbus.top, section 核心方法:
// the performer generates the next unit's latents by flow matching; the update
// x += dt*v and its rounding are this library's reading).
//
// dt (an fp32) times a bf16 has at most 32 significant bits, so the fp64
// product is exact; the sum is rounded once to fp64 and once to bf16 with
// round-to-nearest-even.  The kernel moves 6 bytes per element and has ample
// fp64 throughput for two fp64 operations per element at HBM speed.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace ws {

namespace {

// Round a double to the nearest bf16 (ties to even), from the IEEE 754 encoding:
// keep the top 8 significant bits of the 53-bit significand (fewer below the
// bf16 normal range, where the step is 2^-133), round the dropped bits half to
// even, let a carry ripple into the exponent, saturate to infinity past the
// largest finite value.  Every NaN becomes 0x7FC0.
__device__ __forceinline__ uint32_t bf16_rne_from_f64(double d) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(d));
  const uint32_t sign = static_cast<uint32_t>(b >> 48) & 0x8000u;
  const uint32_t bexp = static_cast<uint32_t>(b >> 52) & 0x7FFu;
  const uint64_t frac = b & 0x000FFFFFFFFFFFFFull;
  if (bexp == 0x7FFu) return frac ? 0x7FC0u : (sign | 0x7F80u);
  if (bexp == 0u) return sign;                      // |d| < 2^-1022: far below half the smallest bf16 step
  const int e = static_cast<int>(bexp) - 1023;      // |d| = 1.frac * 2^e
  const uint64_t sig = frac | (1ull << 52);
  int shift;
  uint32_t bias;
  if (e >= -126) {
    shift = 45;                                     // 53 - 8 significant bits
    bias = (static_cast<uint32_t>(e + 127) << 7) - 128u;
  } else {
    shift = -81 - e;                                // sig * 2^(e-52) / 2^-133
    if (shift > 53) return sign;                    // below half the smallest subnormal step
    bias = 0u;
  }
  uint64_t q = sig >> shift;
  const uint64_t rem = sig & ((1ull << shift) - 1ull);
  const uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1ull))) ++q;
  uint32_t mag = bias + static_cast<uint32_t>(q);
  if (mag >= 0x7F80u) mag = 0x7F80u;
  return sign | mag;
}

__device__ __forceinline__ uint32_t euler2(uint32_t x2, uint32_t v2, double dt) {
  const double x_lo = static_cast<double>(__uint_as_float(x2 << 16));
  const double x_hi = static_cast<double>(__uint_as_float(x2 & 0xFFFF0000u));
  const double v_lo = static_cast<double>(__uint_as_float(v2 << 16));
  const double v_hi = static_cast<double>(__uint_as_float(v2 & 0xFFFF0000u));
  const uint32_t lo = bf16_rne_from_f64(__dadd_rn(x_lo, __dmul_rn(dt, v_lo)));
  const uint32_t hi = bf16_rne_from_f64(__dadd_rn(x_hi, __dmul_rn(dt, v_hi)));
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(256) euler_kernel(uint16_t* x, const uint16_t* v, float dt,
                                                    int64_t n) {
  const double dtd = static_cast<double>(dt);
  const int64_t nvec = n >> 3;
  uint4* xv = reinterpret_cast<uint4*>(x);
  const uint4* vv = reinterpret_cast<const uint4*>(v);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    uint4 a = xv[i];
    const uint4 b = vv[i];
    a.x = euler2(a.x, b.x, dtd);
    a.y = euler2(a.y, b.y, dtd);
    a.z = euler2(a.z, b.z, dtd);
    a.w = euler2(a.w, b.w, dtd);
    xv[i] = a;
  }
  // ragged tail (n % 8 elements)
  if (blockIdx.x == 0) {
    const int64_t i = (nvec << 3) + threadIdx.x;
    if (threadIdx.x < 8 && i < n) {
      const double xd = static_cast<double>(__uint_as_float(static_cast<uint32_t>(x[i]) << 16));
      const double vd = static_cast<double>(__uint_as_float(static_cast<uint32_t>(v[i]) << 16));
      x[i] = static_cast<uint16_t>(bf16_rne_from_f64(__dadd_rn(xd, __dmul_rn(dtd, vd))));
    }
  }
}

}  // namespace

cudaError_t launch_euler(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t nvec = n >> 3;
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;   // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  euler_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, v, dt, n);
  return cudaGetLastError();
}

}  // namespace ws
