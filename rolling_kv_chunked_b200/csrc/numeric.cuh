// bf16 <-> fp32/fp64 helpers shared by the kernels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace rkv {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// fp64 -> bf16, round to nearest even in one conversion (cvt.rn.bf16.f64 through the
// __double2bfloat16 intrinsic): correctly rounded, ties to even, subnormal results kept,
// overflow to infinity. One special-function-unit instruction per value; the GPU tests
// check it bit for bit against the oracle's rounding over every finite bf16 input pattern.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) { return __bfloat16_as_ushort(__double2bfloat16(x)); }

// bf16 -> fp64, exact.
__device__ __forceinline__ double bf16_to_f64(uint32_t b) {
  return static_cast<double>(bf16_to_f32(static_cast<uint16_t>(b)));
}

// x0 = xt - sigma * v; xt' = (1 - sigma') * x0 + sigma' * eps, in fp64 with every
// operation rounded on its own (no fused multiply-add).
struct FlowStep {
  double sigma, one_minus_next, sigma_next;
  bool renoise;
  __device__ __forceinline__ void apply(double xt, double v, double eps, uint16_t& x0_out, uint16_t& xn_out) const {
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

// One 16-byte vector (8 elements) of the step: x0 and (with renoise) xt' packed as bf16x2
// words. kCfg: v is the conditional prediction and u the unconditional one.
template <bool kCfg>
__device__ __forceinline__ void flow_vec8(const FlowStep& step, double scale, const uint32_t (&xw)[4],
                                          const uint32_t (&vw)[4], const uint32_t (&uw)[4], const uint32_t (&ew)[4],
                                          uint32_t (&ow)[4], uint32_t (&nw)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint16_t o0, o1, n0 = 0, n1 = 0;
    if (kCfg) {
      step.apply_cfg_bits(xw[q], vw[q], uw[q], ew[q], scale, o0, n0);
      step.apply_cfg_bits(xw[q] >> 16, vw[q] >> 16, uw[q] >> 16, ew[q] >> 16, scale, o1, n1);
    } else {
      step.apply_bits(xw[q], vw[q], ew[q], o0, n0);
      step.apply_bits(xw[q] >> 16, vw[q] >> 16, ew[q] >> 16, o1, n1);
    }
    ow[q] = static_cast<uint32_t>(o0) | (static_cast<uint32_t>(o1) << 16);
    nw[q] = static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n1) << 16);
  }
}

}  // namespace rkv
