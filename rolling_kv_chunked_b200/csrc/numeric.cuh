// bf16 <-> fp32/fp64 helpers shared by the kernels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace rkv {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// fp64 -> bf16, round to nearest even, without double rounding: first round
// toward zero to fp32 and set the last fp32 bit when anything was dropped
// ("round to odd"), then round that fp32 to bf16 to nearest even. Rounding to
// odd in a format with at least two more bits than the target, followed by
// round-to-nearest, gives the correctly rounded result (Boldo & Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using
// rounding to odd", IEEE Trans. Computers 57(4), 2008). fp32 keeps 16 more
// significand bits than bf16, in the normal and the subnormal range alike.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const float f = __double2float_rz(x);
  uint32_t u = __float_as_uint(f);
  if (static_cast<double>(f) != x) u |= 1u;
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return static_cast<uint16_t>(u);
}

// bf16 -> fp64, exact.
__device__ __forceinline__ double bf16_to_f64(uint32_t b) {
  return static_cast<double>(bf16_to_f32(static_cast<uint16_t>(b)));
}

// x0 = xt - sigma * v; xt' = (1 - sigma') * x0 + sigma' * eps, in fp64 with every
// operation rounded on its own (no fused multiply-add).
struct FlowStep {
  double sigma, one_minus_next, sigma_next;
  bool renoise;
  __device__ __forceinline__ void apply(double xt, double v, double eps, uint16_t& x0_out,
                                        uint16_t& xn_out) const {
    const double x0 = __dsub_rn(xt, __dmul_rn(sigma, v));
    x0_out = f64_to_bf16_rne(x0);
    if (renoise) xn_out = f64_to_bf16_rne(__dadd_rn(__dmul_rn(one_minus_next, x0), __dmul_rn(sigma_next, eps)));
  }
  // the same on bf16 bit patterns (low 16 bits of each argument)
  __device__ __forceinline__ void apply_bits(uint32_t xt, uint32_t v, uint32_t eps, uint16_t& x0_out,
                                             uint16_t& xn_out) const {
    apply(bf16_to_f64(xt & 0xFFFFu), bf16_to_f64(v & 0xFFFFu), renoise ? bf16_to_f64(eps & 0xFFFFu) : 0.0, x0_out,
          xn_out);
  }
  // classifier-free guidance first: v = u + scale * (c - u), each operation rounded on its own,
  // v kept in fp64 for the step
  __device__ __forceinline__ void apply_cfg_bits(uint32_t xt, uint32_t c, uint32_t u, uint32_t eps, double scale,
                                                 uint16_t& x0_out, uint16_t& xn_out) const {
    const double ud = bf16_to_f64(u & 0xFFFFu);
    const double v = __dadd_rn(ud, __dmul_rn(scale, __dsub_rn(bf16_to_f64(c & 0xFFFFu), ud)));
    apply(bf16_to_f64(xt & 0xFFFFu), v, renoise ? bf16_to_f64(eps & 0xFFFFu) : 0.0, x0_out, xn_out);
  }
};

}  // namespace rkv
