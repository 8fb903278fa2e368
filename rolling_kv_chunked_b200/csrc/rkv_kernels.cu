// Memory-bound kernels of the rolling-cache path:
//  * frame runs: the commit / write-back copy into the ring (K1) and the 3D RoPE
//    rotation of queries, chunk keys and (relative mode) the visible window (K3);
//  * the fp64 flow-matching x0 / renoise epilogue (K4), optionally preceded by the
//    classifier-free guidance combine of a conditional and an unconditional prediction.
// All move 16-byte vectors (8 bf16) per thread with grid-stride loops sized to the SM count.
#include <algorithm>

#include "numeric.cuh"
#include "rkv_internal.h"

namespace rkv {
namespace {

int sm_count() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

// (cos, sin) of the four adjacent pairs 4*vec .. 4*vec+3 at a token's position. Pair p
// belongs to the time axis if p < pairs_t, to the row axis if p < pairs_t + pairs_h, else to
// the column axis; each axis has its own table indexed by the token's position on that axis.
__device__ __forceinline__ void pair_cos_sin(int vec, int t_id, int hh, int ww, const FrameRunParams& p,
                                             float2 (&cs)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int pair = vec * 4 + q;
    if (pair < p.pairs_t) {
      cs[q] = __ldg(&p.tab_t[t_id * p.pairs_t + pair]);
    } else if (pair < p.pairs_t + p.pairs_h) {
      cs[q] = __ldg(&p.tab_h[hh * p.pairs_h + (pair - p.pairs_t)]);
    } else {
      cs[q] = __ldg(&p.tab_w[ww * p.pairs_w + (pair - p.pairs_t - p.pairs_h)]);
    }
  }
}

// Rotate the four pairs of one 16-byte vector: (a, b) -> (a c - b s, a s + b c) in fp32,
// rounded to bf16 to nearest even.
__device__ __forceinline__ uint4 rotate_vec(uint4 val, const float2 (&cs)[4]) {
  uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float a = bf16_to_f32(static_cast<uint16_t>(w[q] & 0xFFFFu));
    const float b = bf16_to_f32(static_cast<uint16_t>(w[q] >> 16));
    const __nv_bfloat162 r = __floats2bfloat162_rn(a * cs[q].x - b * cs[q].y, a * cs[q].y + b * cs[q].x);
    w[q] = *reinterpret_cast<const uint32_t*>(&r);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// One warp per token. Lane l always handles the 16-byte vector l % 16 of heads
// l / 16, l / 16 + 2, ... (kPer heads in flight, their loads issued before the (cos, sin)
// lookups), so a half-warp moves one head's 256 contiguous bytes per instruction and each
// lane fetches its four (cos, sin) pairs once per kPer heads. blockIdx.y selects the run.
// kPer = 8 (blocks of 256 threads) in general; kPer = 12 (blocks of 128) when a token has
// 17-24 heads, so that all of a token's heads are in flight at once and a launch of one
// chunk (a few thousand tokens, every warp resident) waits on one DRAM round trip, not two.
template <int kPer>
__global__ void __launch_bounds__(kPer == 8 ? 256 : 128) frame_runs_kernel(const __grid_constant__ FrameRunParams p) {
  const int r = blockIdx.y;
  if (r >= p.n_runs) return;
  const FrameRun& run = p.run[r];
  const int lane = threadIdx.x & 31;
  const int vec = lane & 15;
  const int h0 = lane >> 4;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < run.n_tok; t += warps) {
    const uint16_t* src = run.src + static_cast<long long>(run.src_tok0 + t) * run.src_tok_stride + vec * 8;
    uint16_t* dst = run.dst + static_cast<long long>(run.dst_tok0 + t) * run.dst_tok_stride + vec * 8;
    for (int hb = h0; hb < p.H; hb += 2 * kPer) {
      uint4 val[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int h = hb + 2 * u;
        if (h < p.H) val[u] = __ldg(reinterpret_cast<const uint4*>(src + h * run.src_head_stride));
      }
      float2 cs[4];
      if (run.rotate) {
        const int frame = t / p.T;
        const int tok = t - frame * p.T;
        const int hh = tok / p.grid_w;
        pair_cos_sin(vec, min(max(run.t0 + frame, p.t_lo), p.t_hi), hh, tok - hh * p.grid_w, p, cs);
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int h = hb + 2 * u;
        if (h < p.H) {
          uint4 v = val[u];
          if (run.rotate) v = rotate_vec(v, cs);
          *reinterpret_cast<uint4*>(dst + h * run.dst_head_stride) = v;
        }
      }
    }
  }
}

template <bool kCfg>
__device__ __forceinline__ uint4 flow_x0(const FlowStep& step, double scale, uint4 xt, uint4 v, uint4 u, uint4 e,
                                         uint4& xn) {
  const uint32_t xw[4] = {xt.x, xt.y, xt.z, xt.w};
  const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
  const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
  const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
  uint32_t ow[4], nw[4];
  flow_vec8<kCfg>(step, scale, xw, vw, uw, ew, ow, nw);
  xn = make_uint4(nw[0], nw[1], nw[2], nw[3]);
  return make_uint4(ow[0], ow[1], ow[2], ow[3]);
}

// One 16-byte vector of each operand per thread per iteration. The bf16 <-> fp64
// conversions run on the special-function unit (five per element: three in, one per
// output, the output ones as one fp64 -> bf16 rounding each) and keep it busy, so HBM stays
// busy only with many resident warps: 40 registers per thread (six blocks of 256 threads per
// SM) and a grid of 16 blocks per SM.
template <bool kCfg>
__global__ void __launch_bounds__(256, 6) flow_kernel(const FlowParams p) {
  FlowStep step;
  step.sigma = p.sigma;
  step.renoise = p.sigma_next >= 0.0;
  step.sigma_next = step.renoise ? p.sigma_next : 0.0;
  step.one_minus_next = __dsub_rn(1.0, step.sigma_next);
  const long long n_vec = p.n >> 3;
  const long long threads = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint4* xtp = reinterpret_cast<const uint4*>(p.xt);
  const uint4* vp = reinterpret_cast<const uint4*>(p.v);
  const uint4* up = reinterpret_cast<const uint4*>(p.v_uncond);
  const uint4* ep = reinterpret_cast<const uint4*>(p.eps);
  uint4* x0p = reinterpret_cast<uint4*>(p.x0);
  uint4* xnp = reinterpret_cast<uint4*>(p.xt_next);
  for (long long i = gid; i < n_vec; i += threads) {
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4 xa = __ldg(xtp + i), va = __ldg(vp + i);
    const uint4 ua = kCfg ? __ldg(up + i) : zero;
    const uint4 ea = step.renoise ? __ldg(ep + i) : zero;
    uint4 na;
    x0p[i] = flow_x0<kCfg>(step, p.cfg_scale, xa, va, ua, ea, na);
    if (step.renoise) xnp[i] = na;
  }
  // ragged tail (n not a multiple of 8): one element per thread of the first block
  const long long tail0 = n_vec << 3;
  if (gid < p.n - tail0) {
    const long long j = tail0 + gid;
    uint16_t o, nx = 0;
    const uint32_t e = step.renoise ? p.eps[j] : 0u;
    if (kCfg) {
      step.apply_cfg_bits(p.xt[j], p.v[j], p.v_uncond[j], e, p.cfg_scale, o, nx);
    } else {
      step.apply_bits(p.xt[j], p.v[j], e, o, nx);
    }
    p.x0[j] = o;
    if (step.renoise) p.xt_next[j] = nx;
  }
}

}  // namespace

cudaError_t launch_frame_runs(const FrameRunParams& p, int max_tok, cudaStream_t stream) {
  if (p.n_runs <= 0) return cudaSuccess;
  const long long per_run = p.n_runs > 1 ? p.n_runs : 1;
  if (p.H > 16 && p.H <= 24) {
    long long blocks = (static_cast<long long>(max_tok) + 3) / 4;  // 4 warps (tokens) per block
    const long long cap = static_cast<long long>(sm_count()) * 16 / per_run + 1;
    blocks = std::max(1LL, std::min(blocks, cap));
    dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(p.n_runs));
    frame_runs_kernel<12><<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
  }
  long long blocks = (static_cast<long long>(max_tok) + 7) / 8;  // 8 warps (tokens) per block
  const long long cap = static_cast<long long>(sm_count()) * 8 / per_run + 1;
  blocks = std::max(1LL, std::min(blocks, cap));
  dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(p.n_runs));
  frame_runs_kernel<8><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_flow(const FlowParams& p, cudaStream_t stream) {
  if (p.n <= 0) return cudaSuccess;
  const long long vecs = std::max(1LL, p.n >> 3);
  long long blocks = (vecs + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 16;
  blocks = std::max(1LL, std::min(blocks, cap));
  if (p.v_uncond != nullptr) {
    flow_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  } else {
    flow_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace rkv
