// Memory-bound kernels of the rolling-cache path:
//  * frame runs: the commit / write-back copy into the ring (K1) and the 3D RoPE
//    rotation of queries, chunk keys and (relative mode) the visible window (K3);
//  * the fp64 flow-matching x0 / renoise epilogue (K4).
// All move 16-byte vectors (8 bf16) per thread with grid-stride loops sized to
// the SM count.
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

// Rotation of one 16-byte vector: elements 8*vec .. 8*vec+7 of a (token, head)
// row are the four adjacent pairs 4*vec .. 4*vec+3. Pair p belongs to the time
// axis if p < pairs_t, to the row axis if p < pairs_t + pairs_h, else to the
// column axis; its (cos, sin) comes from that axis' table at the token's position.
__device__ __forceinline__ uint4 rotate_vec(uint4 val, int vec, int t_id, int hh, int ww,
                                            const FrameRunParams& p) {
  uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int pair = vec * 4 + q;
    float2 cs;
    if (pair < p.pairs_t) {
      cs = __ldg(&p.tab_t[t_id * p.pairs_t + pair]);
    } else if (pair < p.pairs_t + p.pairs_h) {
      cs = __ldg(&p.tab_h[hh * p.pairs_h + (pair - p.pairs_t)]);
    } else {
      cs = __ldg(&p.tab_w[ww * p.pairs_w + (pair - p.pairs_t - p.pairs_h)]);
    }
    const float a = bf16_to_f32(static_cast<uint16_t>(w[q] & 0xFFFFu));
    const float b = bf16_to_f32(static_cast<uint16_t>(w[q] >> 16));
    const float ra = a * cs.x - b * cs.y;
    const float rb = a * cs.y + b * cs.x;
    w[q] = static_cast<uint32_t>(f32_to_bf16_rne(ra)) | (static_cast<uint32_t>(f32_to_bf16_rne(rb)) << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(256) frame_runs_kernel(const __grid_constant__ FrameRunParams p) {
  const int r = blockIdx.y;
  if (r >= p.n_runs) return;
  const FrameRun& run = p.run[r];
  const long long n_vec = static_cast<long long>(run.n_tok) * p.H * (kHeadDim / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
    const int vec = static_cast<int>(i & 15);
    const long long th = i >> 4;
    const int h = static_cast<int>(th % p.H);
    const int t = static_cast<int>(th / p.H);
    const uint16_t* s = run.src + static_cast<long long>(run.src_tok0 + t) * run.src_tok_stride +
                        static_cast<long long>(h) * run.src_head_stride + vec * 8;
    uint16_t* d = run.dst + static_cast<long long>(run.dst_tok0 + t) * run.dst_tok_stride +
                  static_cast<long long>(h) * run.dst_head_stride + vec * 8;
    uint4 val = __ldg(reinterpret_cast<const uint4*>(s));
    if (run.rotate) {
      const int frame = t / p.T;
      const int tok = t - frame * p.T;
      const int t_id = min(max(run.t0 + frame, p.t_lo), p.t_hi);
      val = rotate_vec(val, vec, t_id, tok / p.grid_w, tok % p.grid_w, p);
    }
    *reinterpret_cast<uint4*>(d) = val;
  }
}

__global__ void __launch_bounds__(256) flow_kernel(const FlowParams p) {
  FlowStep step;
  step.sigma = p.sigma;
  step.renoise = p.sigma_next >= 0.0;
  step.sigma_next = step.renoise ? p.sigma_next : 0.0;
  step.one_minus_next = __dsub_rn(1.0, step.sigma_next);
  const long long n_vec = p.n >> 3;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long long i = gid; i < n_vec; i += stride) {
    const uint4 xt = __ldg(reinterpret_cast<const uint4*>(p.xt) + i);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.v) + i);
    uint4 e = make_uint4(0, 0, 0, 0);
    if (step.renoise) e = __ldg(reinterpret_cast<const uint4*>(p.eps) + i);
    const uint32_t xw[4] = {xt.x, xt.y, xt.z, xt.w};
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
    const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
    uint32_t ow[4], nw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint16_t o0, o1, n0 = 0, n1 = 0;
      step.apply(bf16_to_f32(xw[q] & 0xFFFFu), bf16_to_f32(vw[q] & 0xFFFFu), bf16_to_f32(ew[q] & 0xFFFFu), o0,
                 n0);
      step.apply(bf16_to_f32(xw[q] >> 16), bf16_to_f32(vw[q] >> 16), bf16_to_f32(ew[q] >> 16), o1, n1);
      ow[q] = static_cast<uint32_t>(o0) | (static_cast<uint32_t>(o1) << 16);
      nw[q] = static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n1) << 16);
    }
    reinterpret_cast<uint4*>(p.x0)[i] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    if (step.renoise) reinterpret_cast<uint4*>(p.xt_next)[i] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
  }
  // ragged tail (n not a multiple of 8): one element per thread of the first block
  const long long tail0 = n_vec << 3;
  if (gid < p.n - tail0) {
    const long long j = tail0 + gid;
    uint16_t o, nx = 0;
    step.apply(bf16_to_f32(p.xt[j]), bf16_to_f32(p.v[j]), step.renoise ? bf16_to_f32(p.eps[j]) : 0.0, o, nx);
    p.x0[j] = o;
    if (step.renoise) p.xt_next[j] = nx;
  }
}

}  // namespace

cudaError_t launch_frame_runs(const FrameRunParams& p, int max_tok, cudaStream_t stream) {
  if (p.n_runs <= 0) return cudaSuccess;
  const long long vecs = static_cast<long long>(max_tok) * p.H * (kHeadDim / 8);
  long long blocks = (vecs + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  blocks = std::max(1LL, std::min(blocks, cap));
  dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(p.n_runs));
  frame_runs_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_flow(const FlowParams& p, cudaStream_t stream) {
  if (p.n <= 0) return cudaSuccess;
  const long long vecs = std::max(1LL, p.n >> 3);
  long long blocks = (vecs + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  blocks = std::max(1LL, std::min(blocks, cap));
  flow_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rkv
