// Fused flow-matching Euler update of a bf16 latent, in place:
//   x <- RN_bf16( fl64( x + fl64(dt * v) ) )
// ("Wan-Streamer v0.2：更高分辨率，相同延迟", paper.rainbus.top, section 核心方法:
// the performer generates the next unit's latents by flow matching; the update
// x += dt*v and its rounding are this library's reading).
//
// dt (an fp32) times a bf16 has at most 32 significant bits, so the fp64
// product is exact; the sum is rounded once to fp64 and once to bf16 with
// round-to-nearest-even.  The kernel moves 6 bytes per element; per element it
// spends one fp64 FMA and a few conversions, well within the fp64 rate at HBM
// speed.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace ws {

namespace {

// Round a double to the nearest bf16, ties to even, in two steps: to fp32 with
// round-to-odd (truncate, then set the last bit when the truncation was
// inexact), then fp32 -> bf16 with the hardware's round-to-nearest-even.
// Rounding to odd at a precision with at least two more bits than the target
// and then to nearest gives the correctly rounded result (Boldo and Melquiond,
// "When double rounding is odd", 2005); fp32 keeps 16 more significant bits than
// bf16 at every exponent, subnormals included.  Every NaN becomes 0x7FC0.
__device__ __forceinline__ float f64_to_f32_odd(double d) {
  const float t = __double2float_rz(d);
  uint32_t u = __float_as_uint(t);
  if (static_cast<double>(t) != d) u |= 1u;   // inexact (or NaN): sticky bit
  return __uint_as_float(u);
}

__device__ __forceinline__ uint32_t bf16x2_rne_from_f64(double lo, double hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(f64_to_f32_odd(lo)), "f"(f64_to_f32_odd(hi)));
  if (lo != lo) r = (r & 0xFFFF0000u) | 0x7FC0u;
  if (hi != hi) r = (r & 0x0000FFFFu) | 0x7FC00000u;
  return r;
}

// x + dt*v for two packed bf16 pairs: dt*v is exact in fp64, so one fused
// multiply-add rounds the sum once, exactly as the separate product and sum do.
__device__ __forceinline__ uint32_t euler2(uint32_t x2, uint32_t v2, double dt) {
  const double x_lo = static_cast<double>(__uint_as_float(x2 << 16));
  const double x_hi = static_cast<double>(__uint_as_float(x2 & 0xFFFF0000u));
  const double v_lo = static_cast<double>(__uint_as_float(v2 << 16));
  const double v_hi = static_cast<double>(__uint_as_float(v2 & 0xFFFF0000u));
  return bf16x2_rne_from_f64(__fma_rn(dt, v_lo, x_lo), __fma_rn(dt, v_hi, x_hi));
}

__device__ __forceinline__ uint4 euler8(uint4 a, const uint4 b, double dt) {
  a.x = euler2(a.x, b.x, dt);
  a.y = euler2(a.y, b.y, dt);
  a.z = euler2(a.z, b.z, dt);
  a.w = euler2(a.w, b.w, dt);
  return a;
}

__global__ void __launch_bounds__(256) euler_kernel(uint16_t* x, const uint16_t* v, float dt, int64_t n) {
  const double dtd = static_cast<double>(dt);
  const int64_t nvec = n >> 3;
  uint4* xv = reinterpret_cast<uint4*>(x);
  const uint4* vv = reinterpret_cast<const uint4*>(v);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // four vectors per thread and iteration: eight 16-byte loads in flight
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 a[4], b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = xv[i + k * stride];
#pragma unroll
    for (int k = 0; k < 4; ++k) b[k] = vv[i + k * stride];
#pragma unroll
    for (int k = 0; k < 4; ++k) xv[i + k * stride] = euler8(a[k], b[k], dtd);
  }
  for (; i < nvec; i += stride) xv[i] = euler8(xv[i], vv[i], dtd);
  // ragged tail (n % 8 elements)
  if (blockIdx.x == 0) {
    const int64_t j = (nvec << 3) + threadIdx.x;
    if (threadIdx.x < 8 && j < n) {
      const double xd = static_cast<double>(__uint_as_float(static_cast<uint32_t>(x[j]) << 16));
      const double vd = static_cast<double>(__uint_as_float(static_cast<uint32_t>(v[j]) << 16));
      x[j] = static_cast<uint16_t>(bf16x2_rne_from_f64(__fma_rn(dtd, vd, xd), 0.0) & 0xFFFFu);
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
