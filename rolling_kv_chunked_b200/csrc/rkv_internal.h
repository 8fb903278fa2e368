// Internal interface between the host state machine (rkv_host.cpp) and the
// kernel translation units (rkv_kernels.cu, rkv_attention.cu). Not installed.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace rkv {

constexpr int kHeadDim = 128;
// TMA box heights of the attention kernel's tensor maps: queries are loaded in
// 128-row tiles, keys and values in 128-row tiles.
constexpr int kQueryBox = 128;
constexpr int kKeyBox = 128;
constexpr int kMaxRuns = 8;
constexpr int kMaxTextTokens = 1 << 16;  // cross-attention context length limit
constexpr int kMaxSegs = 4;
constexpr int kTimeTable = 65536;  // time ids in [0, kTimeTable) have cos/sin rows

// Device status word bits.
constexpr unsigned kStatusTimeout = 1u;

// ---------------------------------------------------------------- frame runs
// A run is a contiguous block of n_tok tokens copied (and optionally rotated)
// from src to dst. Element (token t, head h, dim c) lives at
//   base + (tok0 + t) * tok_stride + h * head_stride + c   (strides in elements),
// which covers both the caller's token-major [tokens, H, d] layout and the
// library's head-major [H][rows][d] rings.
struct FrameRun {
  const uint16_t* src;
  uint16_t* dst;
  long long src_tok_stride, src_head_stride;
  long long dst_tok_stride, dst_head_stride;
  int src_tok0, dst_tok0, n_tok;
  int t0;      // time id of the run's first frame (before clamping)
  int rotate;  // 0 = plain copy, 1 = 3D RoPE rotation
};

struct FrameRunParams {
  FrameRun run[kMaxRuns];
  int n_runs;
  int H, T, grid_w;
  int pairs_t, pairs_h, pairs_w;
  int t_lo, t_hi;  // time ids are clamped to [t_lo, t_hi]
  const float2* tab_t;  // [kTimeTable][pairs_t] (cos, sin)
  const float2* tab_h;  // [grid_h][pairs_h]
  const float2* tab_w;  // [grid_w][pairs_w]
};

cudaError_t launch_frame_runs(const FrameRunParams& p, int max_tok, cudaStream_t stream);

// ---------------------------------------------------------------- flow epilogue
struct FlowParams {
  const uint16_t* xt;
  const uint16_t* v;         // the flow prediction; with guidance the conditional one
  const uint16_t* v_uncond;  // non-null: v = v_uncond + cfg_scale * (v - v_uncond)
  double cfg_scale;
  const uint16_t* eps;
  uint16_t* x0;
  uint16_t* xt_next;
  double sigma, sigma_next;  // sigma_next < 0: last step
  long long n;
};

cudaError_t launch_flow(const FlowParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- attention
// One key segment: K rows [k_row0, k_row0 + n_rows) of the rotated-K buffer and
// V rows [v_row0, ...) of either the cache V ring (src 0) or the caller's v (src 1).
// tm_q and tm_o must use boxes of kQueryBox rows; tm_k, tm_vc and tm_vn boxes of kKeyBox rows.
// tm_o maps the output [Lq][H][d] token-major (coordinates x, head, row).
struct AttnSeg {
  int src;
  int k_row0;
  int v_row0;
  int n_rows;
};

struct AttnParams {
  int q_token_major;  // tm_q maps [Lq][H][d] (coordinates x, head, row) instead of [H][rows][d]
  AttnSeg seg[kMaxSegs];
  int n_segs;
  int n_tiles;  // sum over segments of ceil(n_rows / kKeyBox)
  int H, Lq;
  float scale_log2;  // log2(e) / sqrt(d)
  uint16_t* out;     // [Lq, H, d]
  // fused flow epilogue on the latent [Lq, H*d] (flow != 0)
  int flow;
  const uint16_t* xt;
  const uint16_t* eps;
  uint16_t* x0;
  uint16_t* xt_next;
  double sigma, sigma_next;
  // classifier-free guidance in the epilogue (v_cond non-null): this launch is the
  // unconditional branch u, v = u + cfg_scale * (v_cond - u)
  const uint16_t* v_cond;
  double cfg_scale;
  unsigned* status;
  unsigned long long wait_limit_ns;
  // Scratch for splitting the last, partial wave of a long key stream into two key halves
  // (launch_attention decides; null: never split): fp32 partial rows of kPartRow floats
  // (O unnormalised, then the reference and the sum), room for part_ctas CTAs of 256 rows.
  float* part;
  int part_ctas;
  // set by launch_attention: units u >= split_first (u = head * query blocks + block) run as
  // two CTAs over key tiles [0, split_tiles) and [split_tiles, n_tiles)
  int split_first;
  int split_tiles;
};

constexpr int kPartRow = 132;  // floats per partial row: 128 of O, the reference, the sum, 2 unused

cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_vc,
                             const CUtensorMap& tm_vn, const CUtensorMap& tm_o, const AttnParams& p,
                             cudaStream_t stream);

}  // namespace rkv
