// Host side of librkv.so: argument checks, the per-layer ring state machine,
// RoPE tables, TMA tensor maps and kernel launches. Every exported function is
// declared and documented in include/rkv.h.
//
// Ring placement (one layer, W frames of T tokens, S sinks, R = W - S): frame f
// lives in slot f if f < S, else in slot S + (f - S) mod R. That keeps the
// logical order of the pages' shift-left-after-sink cache ("从40步到4步：
// LingBot-World 2.0实时推理蒸馏（causal_fast）原理与关键代码解读", §3: the KV after the
// sink shifts left as a whole, overwriting the oldest part, and the new KV is
// appended) without moving memory: the visible window of chunk
// [f0, f0 + C) is the sinks min(S, f0), then the latest min(R - C, f0 - S)
// committed non-sink frames (at most two contiguous slot runs because of the
// wrap), then the chunk itself.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/rkv.h"
#include "rkv_internal.h"

#define RKV_API extern "C" __attribute__((visibility("default")))

using rkv::AttnParams;
using rkv::AttnSeg;
using rkv::FrameRun;
using rkv::FrameRunParams;
using rkv::kHeadDim;
using rkv::kTimeTable;

namespace {

struct Seg {
  int src;     // 0 = ring slots, 1 = the call's chunk
  int first;   // first slot (src 0) or first chunk frame (src 1)
  int n;       // frames
  int frame0;  // absolute id of the first frame
};

struct Layer {
  int committed = 0;
  std::vector<int> slot_frame;
  uint16_t* k = nullptr;       // [H][W*T][d] raw K ring
  uint16_t* v = nullptr;       // [H][W*T][d] V ring
  uint16_t* rotk = nullptr;    // [H][(2W-S)*T][d]: rotated K ring, then the chunk area
  uint16_t* qstage = nullptr;  // [H][R*T][d]: rotated queries of the current call
  long long rot_f0 = -1;       // relative mode: rotated ring valid for this (f0, C)
  int rot_c = -1;
  CUtensorMap tm_q, tm_k, tm_vc;
  // cross-attention cache of the text context: K and V, [H][n_text][d] each
  uint16_t* text_k = nullptr;
  uint16_t* text_v = nullptr;
  int n_text = 0;    // 0 = not set
  int text_cap = 0;  // tokens the buffers can hold
  CUtensorMap tm_tk, tm_tv;
};

}  // namespace

struct rkv_ctx {
  int layers = 0, H = 0, d = 0, T = 0, W = 0, S = 0, R = 0, mode = 0;
  bool grid_set = false;
  int gh = 0, gw = 0, pt = 0, ph = 0, pw = 0;
  double theta = 0;
  float2* tab_t = nullptr;
  float2* tab_h = nullptr;
  float2* tab_w = nullptr;
  unsigned* status = nullptr;
  // fp32 partial rows of the key-split last wave of long-stream attention launches
  // (one CTA per SM, 256 rows each; shared by the handle's layers, whose calls run in order)
  float* part = nullptr;
  int part_ctas = 0;
  unsigned long long wait_ns = 2000000000ull;
  std::vector<Layer> L;
  // optional per-launch timing of the attention kernel
  bool timing = false;
  int timing_max = 0, timing_n = 0;
  std::vector<cudaEvent_t> ev_start, ev_stop;
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3D bf16 map, innermost dimension d = 128 elements, box {64, box1, box2}, 128-byte swizzle.
bool encode_map(CUtensorMap* m, const void* base, uint64_t dim1, uint64_t dim2, uint64_t stride1_bytes,
                uint64_t stride2_bytes, uint32_t box1, uint32_t box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), dim1, dim2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {64, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// head-major [H][rows][d], boxes of box_rows rows of one head
bool encode_head_major(CUtensorMap* m, const void* base, int rows, int H, int box_rows) {
  return encode_map(m, base, rows, H, kHeadDim * 2, static_cast<uint64_t>(rows) * kHeadDim * 2, box_rows, 1);
}

// token-major [rows][H][d], boxes of box_rows tokens of one head
bool encode_token_major(CUtensorMap* m, const void* base, int rows, int H, int box_rows) {
  return encode_map(m, base, H, rows, kHeadDim * 2, static_cast<uint64_t>(H) * kHeadDim * 2, 1, box_rows);
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int plan(int W, int S, int committed, int C, int f0, Seg* out, int* n) {
  if (W <= 0 || S < 0 || S >= W || C <= 0 || f0 < 0 || committed < 0) return RKV_ERR_ARG;
  if (f0 != committed) return RKV_ERR_ORDER;
  if (C > W - S) return RKV_ERR_CAPACITY;
  const int R = W - S;
  int k = 0;
  const int s_vis = std::min(S, f0);
  if (s_vis > 0) out[k++] = {0, 0, s_vis, 0};
  if (f0 > S) {
    const int a = std::max(S, f0 + C - R);
    const int cnt = f0 - a;
    if (cnt > 0) {
      const int slot = S + (a - S) % R;
      const int first = std::min(cnt, W - slot);
      out[k++] = {0, slot, first, a};
      if (cnt > first) out[k++] = {0, S, cnt - first, a + first};
    }
  }
  out[k++] = {1, 0, C, f0};
  *n = k;
  return RKV_OK;
}

int slot_of(int f, int S, int R) { return f < S ? f : S + (f - S) % R; }

FrameRunParams base_runs(const rkv_ctx* h) {
  FrameRunParams p;
  std::memset(&p, 0, sizeof(p));
  p.H = h->H;
  p.T = h->T;
  p.grid_w = h->gw;
  p.pairs_t = h->pt;
  p.pairs_h = h->ph;
  p.pairs_w = h->pw;
  p.t_lo = 0;
  p.t_hi = h->mode == RKV_ROPE_ABSOLUTE ? kTimeTable - 1 : h->W - 1;
  p.tab_t = h->tab_t;
  p.tab_h = h->tab_h;
  p.tab_w = h->tab_w;
  return p;
}

// Strides (elements) of the caller's token-major [tokens, H, d] layout and of a
// head-major ring with `rows` rows per head.
void token_major(FrameRun& r, bool is_src, int H) {
  if (is_src) {
    r.src_tok_stride = static_cast<long long>(H) * kHeadDim;
    r.src_head_stride = kHeadDim;
  } else {
    r.dst_tok_stride = static_cast<long long>(H) * kHeadDim;
    r.dst_head_stride = kHeadDim;
  }
}
void head_major(FrameRun& r, bool is_src, long long rows) {
  if (is_src) {
    r.src_tok_stride = kHeadDim;
    r.src_head_stride = rows * kHeadDim;
  } else {
    r.dst_tok_stride = kHeadDim;
    r.dst_head_stride = rows * kHeadDim;
  }
}

void add_run(FrameRunParams& p, const FrameRun& r) { p.run[p.n_runs++] = r; }

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? RKV_OK : RKV_ERR_CUDA; }

// Runs that copy frames [f0, f0+n) of the caller's k / v into their ring slots
// (and, in absolute mode, the chunk's rotated keys from `rot_src_row0` of the
// rotated-K buffer, or the caller's k rotated on the way, into the rotated ring).
void commit_runs(const rkv_ctx* h, const Layer& L, FrameRunParams& p, const void* k, const void* v, int f0,
                 int n, int& max_tok, bool abs_rot_from_chunk_area, bool abs_rot_from_caller) {
  const long long ring_rows = static_cast<long long>(h->W) * h->T;
  const long long rot_rows = static_cast<long long>(2 * h->W - h->S) * h->T;
  int i = 0;
  while (i < n) {
    const int s0 = slot_of(f0 + i, h->S, h->R);
    int len = 1;
    while (i + len < n && slot_of(f0 + i + len, h->S, h->R) == s0 + len) ++len;
    FrameRun r;
    std::memset(&r, 0, sizeof(r));
    r.src_tok0 = i * h->T;
    r.dst_tok0 = s0 * h->T;
    r.n_tok = len * h->T;
    token_major(r, true, h->H);
    head_major(r, false, ring_rows);
    r.src = static_cast<const uint16_t*>(k);
    r.dst = L.k;
    add_run(p, r);
    r.src = static_cast<const uint16_t*>(v);
    r.dst = L.v;
    add_run(p, r);
    if (abs_rot_from_chunk_area) {
      FrameRun q;
      std::memset(&q, 0, sizeof(q));
      q.src = L.rotk;
      q.dst = L.rotk;
      head_major(q, true, rot_rows);
      head_major(q, false, rot_rows);
      q.src_tok0 = static_cast<int>(ring_rows) + i * h->T;
      q.dst_tok0 = s0 * h->T;
      q.n_tok = len * h->T;
      add_run(p, q);
    } else if (abs_rot_from_caller) {
      FrameRun q = r;
      q.src = static_cast<const uint16_t*>(k);
      q.dst = L.rotk;
      head_major(q, false, rot_rows);
      q.t0 = f0 + i;
      q.rotate = 1;
      add_run(p, q);
    }
    max_tok = std::max(max_tok, len * h->T);
    i += len;
  }
}

void advance(rkv_ctx* h, Layer& L, int f0, int n) {
  for (int i = 0; i < n; ++i) L.slot_frame[slot_of(f0 + i, h->S, h->R)] = f0 + i;
  L.committed = f0 + n;
  L.rot_f0 = -1;
  L.rot_c = -1;
}

void free_layer(Layer& L) {
  cudaFree(L.k);
  cudaFree(L.v);
  cudaFree(L.rotk);
  cudaFree(L.qstage);
  cudaFree(L.text_k);
  cudaFree(L.text_v);
  L.k = L.v = L.rotk = L.qstage = L.text_k = L.text_v = nullptr;
  L.n_text = L.text_cap = 0;
}

int check_layer(const rkv_ctx* h, int layer) {
  if (h == nullptr || layer < 0 || layer >= h->layers) return RKV_ERR_ARG;
  return RKV_OK;
}

}  // namespace

// ======================================================================= API

RKV_API int rkv_create(int layers, int H, int d, int tokens_per_frame, int window_frames, int sink_frames,
                       int rope_mode, rkv_handle* out) {
  if (out == nullptr) return RKV_ERR_ARG;
  *out = nullptr;
  if (layers <= 0 || H <= 0 || d <= 0 || tokens_per_frame <= 0 || window_frames <= 0 || sink_frames < 0 ||
      sink_frames >= window_frames)
    return RKV_ERR_ARG;
  if (rope_mode != RKV_ROPE_ABSOLUTE && rope_mode != RKV_ROPE_RELATIVE && rope_mode != RKV_ROPE_RELATIVE_SLOTS)
    return RKV_ERR_ARG;
  if (d != kHeadDim || window_frames > 256) return RKV_ERR_UNSUPPORTED;
  const long long ring_rows = static_cast<long long>(window_frames) * tokens_per_frame;
  const long long rot_rows = static_cast<long long>(2 * window_frames - sink_frames) * tokens_per_frame;
  if (rot_rows * H * kHeadDim >= (1LL << 40) || rot_rows >= (1LL << 31)) return RKV_ERR_UNSUPPORTED;

  rkv_ctx* h = new (std::nothrow) rkv_ctx();
  if (h == nullptr) return RKV_ERR_CUDA;
  h->layers = layers;
  h->H = H;
  h->d = d;
  h->T = tokens_per_frame;
  h->W = window_frames;
  h->S = sink_frames;
  h->R = window_frames - sink_frames;
  h->mode = rope_mode;
  h->L.resize(layers);
  const long long q_rows = static_cast<long long>(h->R) * tokens_per_frame;
  int rc = RKV_OK;
  if (cudaMalloc(&h->status, sizeof(unsigned)) != cudaSuccess || cudaMemset(h->status, 0, sizeof(unsigned)) != cudaSuccess)
    rc = RKV_ERR_CUDA;
  if (rc == RKV_OK) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0 ||
        cudaMalloc(&h->part, static_cast<size_t>(sms) * 2 * rkv::kQueryBox * rkv::kPartRow * sizeof(float)) !=
            cudaSuccess)
      rc = RKV_ERR_CUDA;
    else
      h->part_ctas = sms;
  }
  for (int l = 0; l < layers && rc == RKV_OK; ++l) {
    Layer& L = h->L[l];
    L.slot_frame.assign(window_frames, -1);
    const size_t ring_b = static_cast<size_t>(ring_rows) * H * kHeadDim * 2;
    const size_t rot_b = static_cast<size_t>(rot_rows) * H * kHeadDim * 2;
    const size_t q_b = static_cast<size_t>(q_rows) * H * kHeadDim * 2;
    if (cudaMalloc(&L.k, ring_b) != cudaSuccess || cudaMalloc(&L.v, ring_b) != cudaSuccess ||
        cudaMalloc(&L.rotk, rot_b) != cudaSuccess || cudaMalloc(&L.qstage, q_b) != cudaSuccess) {
      rc = RKV_ERR_CUDA;
      break;
    }
    // zero-filled so that keys beyond a segment (masked, weight exactly 0) are finite
    if (cudaMemset(L.k, 0, ring_b) != cudaSuccess || cudaMemset(L.v, 0, ring_b) != cudaSuccess ||
        cudaMemset(L.rotk, 0, rot_b) != cudaSuccess || cudaMemset(L.qstage, 0, q_b) != cudaSuccess) {
      rc = RKV_ERR_CUDA;
      break;
    }
    if (!encode_head_major(&L.tm_q, L.qstage, static_cast<int>(q_rows), H, rkv::kQueryBox) ||
        !encode_head_major(&L.tm_k, L.rotk, static_cast<int>(rot_rows), H, rkv::kKeyBox) ||
        !encode_head_major(&L.tm_vc, L.v, static_cast<int>(ring_rows), H, rkv::kKeyBox)) {
      rc = RKV_ERR_CUDA;
      break;
    }
  }
  if (rc == RKV_OK && cudaDeviceSynchronize() != cudaSuccess) rc = RKV_ERR_CUDA;
  if (rc != RKV_OK) {
    rkv_destroy(h);
    return rc;
  }
  *out = h;
  return RKV_OK;
}

RKV_API int rkv_set_rope_grid(rkv_handle h, int grid_h, int grid_w, double theta, int pairs_t, int pairs_h,
                              int pairs_w) {
  if (h == nullptr || grid_h <= 0 || grid_w <= 0 || grid_h * grid_w != h->T || !(theta > 0.0) || pairs_t < 0 ||
      pairs_h < 0 || pairs_w < 0 || 2 * (pairs_t + pairs_h + pairs_w) != h->d)
    return RKV_ERR_ARG;
  std::vector<float2> tt(static_cast<size_t>(kTimeTable) * std::max(pairs_t, 1));
  std::vector<float2> th(static_cast<size_t>(grid_h) * std::max(pairs_h, 1));
  std::vector<float2> tw(static_cast<size_t>(grid_w) * std::max(pairs_w, 1));
  auto fill = [theta](std::vector<float2>& tab, int npos, int npairs) {
    for (int j = 0; j < npairs; ++j) {
      const double omega = std::pow(theta, -static_cast<double>(j) / npairs);
      for (int pos = 0; pos < npos; ++pos) {
        const double a = pos * omega;
        tab[static_cast<size_t>(pos) * npairs + j] = make_float2(static_cast<float>(std::cos(a)),
                                                                 static_cast<float>(std::sin(a)));
      }
    }
  };
  fill(tt, kTimeTable, pairs_t);
  fill(th, grid_h, pairs_h);
  fill(tw, grid_w, pairs_w);
  cudaFree(h->tab_t);
  cudaFree(h->tab_h);
  cudaFree(h->tab_w);
  h->tab_t = h->tab_h = h->tab_w = nullptr;
  h->grid_set = false;
  if (cudaMalloc(&h->tab_t, tt.size() * sizeof(float2)) != cudaSuccess ||
      cudaMalloc(&h->tab_h, th.size() * sizeof(float2)) != cudaSuccess ||
      cudaMalloc(&h->tab_w, tw.size() * sizeof(float2)) != cudaSuccess)
    return RKV_ERR_CUDA;
  if (cudaMemcpy(h->tab_t, tt.data(), tt.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->tab_h, th.data(), th.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->tab_w, tw.data(), tw.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess)
    return RKV_ERR_CUDA;
  h->gh = grid_h;
  h->gw = grid_w;
  h->theta = theta;
  h->pt = pairs_t;
  h->ph = pairs_h;
  h->pw = pairs_w;
  h->grid_set = true;
  for (Layer& L : h->L) {
    L.rot_f0 = -1;
    L.rot_c = -1;
  }
  return RKV_OK;
}

RKV_API int rkv_plan_window(int window_frames, int sink_frames, int frames_committed, int n_frames,
                            int start_frame, int* seg_out, int max_segs, int* n_segs) {
  if (seg_out == nullptr || n_segs == nullptr || max_segs < 1) return RKV_ERR_ARG;
  Seg segs[rkv::kMaxSegs];
  int n = 0;
  const int rc = plan(window_frames, sink_frames, frames_committed, n_frames, start_frame, segs, &n);
  if (rc != RKV_OK) return rc;
  if (n > max_segs) return RKV_ERR_ARG;
  for (int i = 0; i < n; ++i) {
    seg_out[4 * i + 0] = segs[i].src;
    seg_out[4 * i + 1] = segs[i].first;
    seg_out[4 * i + 2] = segs[i].n;
    seg_out[4 * i + 3] = segs[i].frame0;
  }
  *n_segs = n;
  return RKV_OK;
}

RKV_API int rkv_write_chunk(rkv_handle h, int layer, const void* k, const void* v, int n_frames, int start_frame,
                            void* stream) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (!aligned16(k) || !aligned16(v) || n_frames <= 0) return RKV_ERR_ARG;
  Layer& L = h->L[layer];
  if (start_frame != L.committed) return RKV_ERR_ORDER;
  if (n_frames > h->R) return RKV_ERR_CAPACITY;
  const bool abs_mode = h->mode == RKV_ROPE_ABSOLUTE;
  if (abs_mode && !h->grid_set) return RKV_ERR_STATE;
  if (abs_mode && start_frame + n_frames > kTimeTable) return RKV_ERR_UNSUPPORTED;
  FrameRunParams p = base_runs(h);
  int max_tok = 0;
  commit_runs(h, L, p, k, v, start_frame, n_frames, max_tok, false, abs_mode);
  rc = cuda_rc(rkv::launch_frame_runs(p, max_tok, static_cast<cudaStream_t>(stream)));
  if (rc) return rc;
  advance(h, L, start_frame, n_frames);
  return RKV_OK;
}

namespace {

int chunk_attention_impl(rkv_handle h, int layer, const void* q, const void* k, const void* v, void* out,
                         int n_frames, int start_frame, int commit, const rkv_flow_epilogue* epi,
                         const void* v_cond, double cfg_scale, void* stream) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || n_frames <= 0) return RKV_ERR_ARG;
  if (epi != nullptr) {
    if (!aligned16(epi->xt) || !aligned16(epi->x0_out)) return RKV_ERR_ARG;
    if (epi->sigma_next >= 0.0 && (!aligned16(epi->eps) || !aligned16(epi->xt_next_out))) return RKV_ERR_ARG;
  }
  if (v_cond != nullptr) {
    if (epi == nullptr || !aligned16(v_cond) || !std::isfinite(cfg_scale)) return RKV_ERR_ARG;
    const long long bytes = static_cast<long long>(n_frames) * h->T * h->H * kHeadDim * 2;
    const char* c0 = static_cast<const char*>(v_cond);
    const char* o0 = static_cast<const char*>(out);
    if (c0 < o0 + bytes && o0 < c0 + bytes) return RKV_ERR_ARG;  // v_cond must not overlap out
  }
  Layer& L = h->L[layer];
  Seg segs[rkv::kMaxSegs];
  int ns = 0;
  rc = plan(h->W, h->S, L.committed, n_frames, start_frame, segs, &ns);
  if (rc) return rc;
  if (!h->grid_set) return RKV_ERR_STATE;
  const bool abs_mode = h->mode == RKV_ROPE_ABSOLUTE;
  const int C = n_frames, T = h->T, W = h->W;
  if (abs_mode && start_frame + C > kTimeTable) return RKV_ERR_UNSUPPORTED;
  // relative re-basing origin: the chunk's last frame gets id W-1 (clamped mode), or
  // the number of non-sink frames evicted so far (slot-order mode, where ids are
  // positions in the visible window and sinks keep their own frame index)
  const bool slot_mode = h->mode == RKV_ROPE_RELATIVE_SLOTS;
  const long long end = static_cast<long long>(start_frame) + C;
  const long long base = slot_mode ? std::max<long long>(0, end - W) : end - W;
  const int t_chunk0 = abs_mode ? start_frame : static_cast<int>(start_frame - base);
  const long long ring_rows = static_cast<long long>(W) * T;
  const long long rot_rows = static_cast<long long>(2 * W - h->S) * T;
  const long long q_rows = static_cast<long long>(h->R) * T;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // 1) RoPE on the way in: queries -> staging, chunk keys -> chunk area, and in
  //    relative mode the visible ring once per (start_frame, n_frames).
  FrameRunParams p = base_runs(h);
  int max_tok = C * T;
  {
    FrameRun r;
    std::memset(&r, 0, sizeof(r));
    token_major(r, true, h->H);
    head_major(r, false, q_rows);
    r.src = static_cast<const uint16_t*>(q);
    r.dst = L.qstage;
    r.n_tok = C * T;
    r.t0 = t_chunk0;
    r.rotate = 1;
    add_run(p, r);
    head_major(r, false, rot_rows);
    r.src = static_cast<const uint16_t*>(k);
    r.dst = L.rotk;
    r.dst_tok0 = static_cast<int>(ring_rows);
    add_run(p, r);
  }
  const bool rerotate = !abs_mode && (L.rot_f0 != start_frame || L.rot_c != C);
  if (rerotate) {
    for (int i = 0; i < ns; ++i) {
      if (segs[i].src != 0) continue;
      FrameRun r;
      std::memset(&r, 0, sizeof(r));
      head_major(r, true, ring_rows);
      head_major(r, false, rot_rows);
      r.src = L.k;
      r.dst = L.rotk;
      r.src_tok0 = r.dst_tok0 = segs[i].first * T;
      r.n_tok = segs[i].n * T;
      const bool sinks = segs[i].frame0 < h->S;  // the sink segment starts at frame 0
      r.t0 = static_cast<int>(slot_mode && sinks ? segs[i].frame0 : segs[i].frame0 - base);  // clamped in the kernel
      r.rotate = 1;
      add_run(p, r);
      max_tok = std::max(max_tok, r.n_tok);
    }
  }
  rc = cuda_rc(rkv::launch_frame_runs(p, max_tok, st));
  if (rc) return rc;
  if (!abs_mode) {
    L.rot_f0 = start_frame;
    L.rot_c = C;
  }

  // 2) attention over the segmented key stream
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.n_segs = ns;
  for (int i = 0; i < ns; ++i) {
    AttnSeg& s = ap.seg[i];
    s.src = segs[i].src;
    s.n_rows = segs[i].n * T;
    if (segs[i].src == 0) {
      s.k_row0 = s.v_row0 = segs[i].first * T;
    } else {
      s.k_row0 = static_cast<int>(ring_rows);
      s.v_row0 = 0;
    }
    ap.n_tiles += (s.n_rows + rkv::kKeyBox - 1) / rkv::kKeyBox;
  }
  ap.H = h->H;
  ap.Lq = C * T;
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim)));
  ap.out = static_cast<uint16_t*>(out);
  if (epi != nullptr) {
    ap.flow = 1;
    ap.xt = static_cast<const uint16_t*>(epi->xt);
    ap.eps = static_cast<const uint16_t*>(epi->eps);
    ap.x0 = static_cast<uint16_t*>(epi->x0_out);
    ap.xt_next = static_cast<uint16_t*>(epi->xt_next_out);
    ap.sigma = epi->sigma;
    ap.sigma_next = epi->sigma_next;
    ap.v_cond = static_cast<const uint16_t*>(v_cond);
    ap.cfg_scale = cfg_scale;
  } else {
    ap.sigma_next = -1.0;
  }
  ap.status = h->status;
  ap.wait_limit_ns = h->wait_ns;
  ap.part = h->part;
  ap.part_ctas = h->part_ctas;
  CUtensorMap tm_vn, tm_o;
  if (!encode_token_major(&tm_vn, v, C * T, h->H, rkv::kKeyBox) ||
      !encode_token_major(&tm_o, out, C * T, h->H, rkv::kQueryBox))
    return RKV_ERR_CUDA;
  const bool timed = h->timing && h->timing_n < h->timing_max;
  if (timed && cudaEventRecord(h->ev_start[h->timing_n], st) != cudaSuccess) return RKV_ERR_CUDA;
  rc = cuda_rc(rkv::launch_attention(L.tm_q, L.tm_k, L.tm_vc, tm_vn, tm_o, ap, st));
  if (rc) return rc;
  if (timed) {
    if (cudaEventRecord(h->ev_stop[h->timing_n], st) != cudaSuccess) return RKV_ERR_CUDA;
    ++h->timing_n;
  }

  // 3) the clean write-back
  if (commit) {
    FrameRunParams c = base_runs(h);
    int mt = 0;
    commit_runs(h, L, c, k, v, start_frame, C, mt, abs_mode, false);
    rc = cuda_rc(rkv::launch_frame_runs(c, mt, st));
    if (rc) return rc;
    advance(h, L, start_frame, C);
  }
  return RKV_OK;
}

}  // namespace

RKV_API int rkv_chunk_attention_flow(rkv_handle h, int layer, const void* q, const void* k, const void* v, void* out,
                                     int n_frames, int start_frame, int commit, const rkv_flow_epilogue* epi,
                                     void* stream) {
  return chunk_attention_impl(h, layer, q, k, v, out, n_frames, start_frame, commit, epi, nullptr, 0.0, stream);
}

RKV_API int rkv_chunk_attention_cfg_flow(rkv_handle h, int layer, const void* q, const void* k, const void* v,
                                         void* out, int n_frames, int start_frame, int commit,
                                         const rkv_flow_epilogue* epi, const void* v_cond, double cfg_scale,
                                         void* stream) {
  if (epi == nullptr || v_cond == nullptr) return RKV_ERR_ARG;
  return chunk_attention_impl(h, layer, q, k, v, out, n_frames, start_frame, commit, epi, v_cond, cfg_scale, stream);
}

RKV_API int rkv_chunk_attention(rkv_handle h, int layer, const void* q, const void* k, const void* v, void* out,
                                int n_frames, int start_frame, int commit, void* stream) {
  return chunk_attention_impl(h, layer, q, k, v, out, n_frames, start_frame, commit, nullptr, nullptr, 0.0, stream);
}

RKV_API int rkv_set_text_kv(rkv_handle h, int layer, const void* k_text, const void* v_text, int n_text,
                            void* stream) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (!aligned16(k_text) || !aligned16(v_text) || n_text <= 0) return RKV_ERR_ARG;
  if (n_text > rkv::kMaxTextTokens) return RKV_ERR_UNSUPPORTED;
  Layer& L = h->L[layer];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_text > L.text_cap) {
    // earlier launches may still read the old buffers
    if (cudaDeviceSynchronize() != cudaSuccess) return RKV_ERR_CUDA;
    cudaFree(L.text_k);
    cudaFree(L.text_v);
    L.text_k = L.text_v = nullptr;
    L.n_text = L.text_cap = 0;
    const size_t b = static_cast<size_t>(n_text) * h->H * kHeadDim * 2;
    if (cudaMalloc(&L.text_k, b) != cudaSuccess || cudaMalloc(&L.text_v, b) != cudaSuccess) {
      cudaFree(L.text_k);
      cudaFree(L.text_v);
      L.text_k = L.text_v = nullptr;
      return RKV_ERR_CUDA;
    }
    L.text_cap = n_text;
  }
  if (!encode_head_major(&L.tm_tk, L.text_k, n_text, h->H, rkv::kKeyBox) ||
      !encode_head_major(&L.tm_tv, L.text_v, n_text, h->H, rkv::kKeyBox)) {
    L.n_text = 0;
    return RKV_ERR_CUDA;
  }
  // token-major [n_text, H, d] -> head-major [H][n_text][d], K and V (a bit copy)
  FrameRunParams p = base_runs(h);
  FrameRun r;
  std::memset(&r, 0, sizeof(r));
  token_major(r, true, h->H);
  head_major(r, false, n_text);
  r.n_tok = n_text;
  r.src = static_cast<const uint16_t*>(k_text);
  r.dst = L.text_k;
  add_run(p, r);
  r.src = static_cast<const uint16_t*>(v_text);
  r.dst = L.text_v;
  add_run(p, r);
  rc = cuda_rc(rkv::launch_frame_runs(p, n_text, st));
  if (rc) {
    L.n_text = 0;
    return rc;
  }
  L.n_text = n_text;
  return RKV_OK;
}

RKV_API int rkv_cross_attention(rkv_handle h, int layer, const void* q, void* out, int n_tokens, void* stream) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(out) || n_tokens <= 0) return RKV_ERR_ARG;
  if (static_cast<long long>(n_tokens) * h->H * kHeadDim >= (1LL << 40)) return RKV_ERR_UNSUPPORTED;
  Layer& L = h->L[layer];
  if (L.n_text <= 0) return RKV_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.q_token_major = 1;
  ap.n_segs = 1;
  ap.seg[0].src = 0;
  ap.seg[0].k_row0 = 0;
  ap.seg[0].v_row0 = 0;
  ap.seg[0].n_rows = L.n_text;
  ap.n_tiles = (L.n_text + rkv::kKeyBox - 1) / rkv::kKeyBox;
  ap.H = h->H;
  ap.Lq = n_tokens;
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim)));
  ap.out = static_cast<uint16_t*>(out);
  ap.sigma_next = -1.0;
  ap.status = h->status;
  ap.wait_limit_ns = h->wait_ns;
  ap.part = h->part;
  ap.part_ctas = h->part_ctas;
  CUtensorMap tm_q, tm_o;
  if (!encode_token_major(&tm_q, q, n_tokens, h->H, rkv::kQueryBox) ||
      !encode_token_major(&tm_o, out, n_tokens, h->H, rkv::kQueryBox))
    return RKV_ERR_CUDA;
  const bool timed = h->timing && h->timing_n < h->timing_max;
  if (timed && cudaEventRecord(h->ev_start[h->timing_n], st) != cudaSuccess) return RKV_ERR_CUDA;
  rc = cuda_rc(rkv::launch_attention(tm_q, L.tm_tk, L.tm_tv, L.tm_tv, tm_o, ap, st));
  if (rc) return rc;
  if (timed) {
    if (cudaEventRecord(h->ev_stop[h->timing_n], st) != cudaSuccess) return RKV_ERR_CUDA;
    ++h->timing_n;
  }
  return RKV_OK;
}

RKV_API int rkv_rope_apply(rkv_handle h, void* x, int n_frames, int start_frame, int window_end_frame,
                           void* stream) {
  if (h == nullptr || !aligned16(x) || n_frames <= 0 || start_frame < 0) return RKV_ERR_ARG;
  if (!h->grid_set) return RKV_ERR_STATE;
  const bool abs_mode = h->mode == RKV_ROPE_ABSOLUTE;
  if (abs_mode && static_cast<long long>(start_frame) + n_frames > kTimeTable) return RKV_ERR_UNSUPPORTED;
  FrameRunParams p = base_runs(h);
  FrameRun r;
  std::memset(&r, 0, sizeof(r));
  token_major(r, true, h->H);
  token_major(r, false, h->H);
  r.src = static_cast<const uint16_t*>(x);
  r.dst = static_cast<uint16_t*>(x);
  r.n_tok = n_frames * h->T;
  r.rotate = 1;
  auto clamp30 = [](long long t) { return static_cast<int>(std::max<long long>(std::min<long long>(t, 1 << 30), -(1 << 30))); };
  if (abs_mode) {
    r.t0 = start_frame;
  } else if (h->mode == RKV_ROPE_RELATIVE) {
    r.t0 = clamp30(static_cast<long long>(start_frame) - (static_cast<long long>(window_end_frame) - h->W));
  } else {
    // slot order: sink frames keep their index, later frames lose the evicted count
    const long long evicted = std::max<long long>(0, static_cast<long long>(window_end_frame) - h->W);
    const int n_sink = std::max(0, std::min(n_frames, h->S - start_frame));
    if (n_sink > 0) {
      FrameRun rs = r;
      rs.n_tok = n_sink * h->T;
      rs.t0 = start_frame;
      add_run(p, rs);
      r.src_tok0 = r.dst_tok0 = rs.n_tok;
      r.n_tok -= rs.n_tok;
    }
    r.t0 = clamp30(static_cast<long long>(start_frame) + n_sink - evicted);
    if (r.n_tok == 0) return cuda_rc(rkv::launch_frame_runs(p, n_sink * h->T, static_cast<cudaStream_t>(stream)));
  }
  const int max_tok = std::max(r.n_tok, p.n_runs ? p.run[0].n_tok : 0);
  add_run(p, r);
  return cuda_rc(rkv::launch_frame_runs(p, max_tok, static_cast<cudaStream_t>(stream)));
}

RKV_API int rkv_copy_heads(const rkv_head_copy* runs, int n_runs, int n_heads, void* stream) {
  if (n_runs < 0 || (n_runs > 0 && runs == nullptr) || n_heads < 1) return RKV_ERR_ARG;
  for (int i = 0; i < n_runs; ++i) {
    const rkv_head_copy& c = runs[i];
    if (c.n_tok < 0 || !aligned16(c.src) || !aligned16(c.dst)) return RKV_ERR_ARG;
    if (c.n_tok > 0 && (c.src == nullptr || c.dst == nullptr)) return RKV_ERR_ARG;
    for (long long st : {c.src_tok_stride, c.src_head_stride, c.dst_tok_stride, c.dst_head_stride})
      if (st < 0 || st % 8 != 0) return RKV_ERR_ARG;
  }
  for (int i0 = 0; i0 < n_runs; i0 += rkv::kMaxRuns) {
    FrameRunParams p;
    std::memset(&p, 0, sizeof(p));
    p.H = n_heads;
    p.T = 1;
    p.grid_w = 1;
    int max_tok = 0;
    for (int i = i0; i < n_runs && i < i0 + rkv::kMaxRuns; ++i) {
      const rkv_head_copy& c = runs[i];
      if (c.n_tok == 0) continue;
      FrameRun r;
      std::memset(&r, 0, sizeof(r));
      r.src = static_cast<const uint16_t*>(c.src);
      r.dst = static_cast<uint16_t*>(c.dst);
      r.src_tok_stride = c.src_tok_stride;
      r.src_head_stride = c.src_head_stride;
      r.dst_tok_stride = c.dst_tok_stride;
      r.dst_head_stride = c.dst_head_stride;
      r.n_tok = c.n_tok;
      r.rotate = 0;
      add_run(p, r);
      max_tok = std::max(max_tok, c.n_tok);
    }
    const int rc = cuda_rc(rkv::launch_frame_runs(p, max_tok, static_cast<cudaStream_t>(stream)));
    if (rc) return rc;
  }
  return RKV_OK;
}

RKV_API int rkv_flow_x0_renoise(const void* xt, const void* v, const void* eps, double sigma, double sigma_next,
                                void* x0_out, void* xt_next_out, long long n, void* stream) {
  if (n < 0) return RKV_ERR_ARG;
  if (n == 0) return RKV_OK;
  if (!aligned16(xt) || !aligned16(v) || !aligned16(x0_out)) return RKV_ERR_ARG;
  if (sigma_next >= 0.0 && (!aligned16(eps) || !aligned16(xt_next_out))) return RKV_ERR_ARG;
  rkv::FlowParams p;
  std::memset(&p, 0, sizeof(p));
  p.xt = static_cast<const uint16_t*>(xt);
  p.v = static_cast<const uint16_t*>(v);
  p.eps = static_cast<const uint16_t*>(eps);
  p.x0 = static_cast<uint16_t*>(x0_out);
  p.xt_next = static_cast<uint16_t*>(xt_next_out);
  p.sigma = sigma;
  p.sigma_next = sigma_next;
  p.n = n;
  return cuda_rc(rkv::launch_flow(p, static_cast<cudaStream_t>(stream)));
}

RKV_API int rkv_flow_cfg_x0_renoise(const void* xt, const void* v_cond, const void* v_uncond, const void* eps,
                                    double cfg_scale, double sigma, double sigma_next, void* x0_out,
                                    void* xt_next_out, long long n, void* stream) {
  if (n < 0) return RKV_ERR_ARG;
  if (n == 0) return RKV_OK;
  if (!aligned16(xt) || !aligned16(v_cond) || !aligned16(v_uncond) || !aligned16(x0_out)) return RKV_ERR_ARG;
  if (!std::isfinite(cfg_scale)) return RKV_ERR_ARG;
  if (sigma_next >= 0.0 && (!aligned16(eps) || !aligned16(xt_next_out))) return RKV_ERR_ARG;
  rkv::FlowParams p;
  std::memset(&p, 0, sizeof(p));
  p.xt = static_cast<const uint16_t*>(xt);
  p.v = static_cast<const uint16_t*>(v_cond);
  p.v_uncond = static_cast<const uint16_t*>(v_uncond);
  p.cfg_scale = cfg_scale;
  p.eps = static_cast<const uint16_t*>(eps);
  p.x0 = static_cast<uint16_t*>(x0_out);
  p.xt_next = static_cast<uint16_t*>(xt_next_out);
  p.sigma = sigma;
  p.sigma_next = sigma_next;
  p.n = n;
  return cuda_rc(rkv::launch_flow(p, static_cast<cudaStream_t>(stream)));
}

RKV_API int rkv_slot_frames(rkv_handle h, int layer, int* frames_out) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (frames_out == nullptr) return RKV_ERR_ARG;
  std::copy(h->L[layer].slot_frame.begin(), h->L[layer].slot_frame.end(), frames_out);
  return RKV_OK;
}

RKV_API int rkv_frames_committed(rkv_handle h, int layer, int* out) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (out == nullptr) return RKV_ERR_ARG;
  *out = h->L[layer].committed;
  return RKV_OK;
}

RKV_API int rkv_cache_ptrs(rkv_handle h, int layer, void** k, void** v) {
  int rc = check_layer(h, layer);
  if (rc) return rc;
  if (k == nullptr || v == nullptr) return RKV_ERR_ARG;
  *k = h->L[layer].k;
  *v = h->L[layer].v;
  return RKV_OK;
}

RKV_API int rkv_reset(rkv_handle h) {
  if (h == nullptr) return RKV_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return RKV_ERR_CUDA;
  const size_t ring_b = static_cast<size_t>(h->W) * h->T * h->H * kHeadDim * 2;
  const size_t rot_b = static_cast<size_t>(2 * h->W - h->S) * h->T * h->H * kHeadDim * 2;
  for (Layer& L : h->L) {
    if (cudaMemset(L.k, 0, ring_b) != cudaSuccess || cudaMemset(L.v, 0, ring_b) != cudaSuccess ||
        cudaMemset(L.rotk, 0, rot_b) != cudaSuccess)
      return RKV_ERR_CUDA;
    L.committed = 0;
    std::fill(L.slot_frame.begin(), L.slot_frame.end(), -1);
    L.rot_f0 = -1;
    L.rot_c = -1;
    L.n_text = 0;  // the text context must be set again
  }
  return cudaDeviceSynchronize() == cudaSuccess ? RKV_OK : RKV_ERR_CUDA;
}

RKV_API int rkv_timing_begin(rkv_handle h, int max_launches) {
  if (h == nullptr || max_launches <= 0) return RKV_ERR_ARG;
  while (static_cast<int>(h->ev_start.size()) < max_launches) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return RKV_ERR_CUDA;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return RKV_ERR_CUDA;
    }
    h->ev_start.push_back(a);
    h->ev_stop.push_back(b);
  }
  h->timing = true;
  h->timing_max = max_launches;
  h->timing_n = 0;
  return RKV_OK;
}

RKV_API int rkv_timing_end(rkv_handle h, float* ms_out, int max, int* n_out) {
  if (h == nullptr || n_out == nullptr || (max > 0 && ms_out == nullptr)) return RKV_ERR_ARG;
  h->timing = false;
  int n = std::min(h->timing_n, std::max(max, 0));
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(h->ev_stop[i]) != cudaSuccess) return RKV_ERR_CUDA;
    if (cudaEventElapsedTime(&ms_out[i], h->ev_start[i], h->ev_stop[i]) != cudaSuccess) return RKV_ERR_CUDA;
  }
  *n_out = n;
  h->timing_n = 0;
  return RKV_OK;
}

RKV_API int rkv_destroy(rkv_handle h) {
  if (h == nullptr) return RKV_ERR_ARG;
  cudaDeviceSynchronize();
  for (size_t i = 0; i < h->ev_start.size(); ++i) {
    cudaEventDestroy(h->ev_start[i]);
    cudaEventDestroy(h->ev_stop[i]);
  }
  for (Layer& L : h->L) free_layer(L);
  cudaFree(h->tab_t);
  cudaFree(h->tab_h);
  cudaFree(h->tab_w);
  cudaFree(h->status);
  cudaFree(h->part);
  delete h;
  return RKV_OK;
}

RKV_API const char* rkv_status_string(int status) {
  switch (status) {
    case RKV_OK: return "ok";
    case RKV_ERR_ARG: return "invalid argument";
    case RKV_ERR_ORDER: return "start_frame does not follow the frames committed so far";
    case RKV_ERR_CAPACITY: return "chunk larger than window_frames - sink_frames";
    case RKV_ERR_UNSUPPORTED: return "unsupported size (d != 128, window > 256 frames or time id beyond table)";
    case RKV_ERR_CUDA: return "CUDA runtime or driver error";
    case RKV_ERR_TIMEOUT: return "a bounded device wait expired";
    case RKV_ERR_STATE: return "required state not set (rkv_set_rope_grid, or rkv_set_text_kv for cross-attention)";
    default: return "unknown status";
  }
}

RKV_API int rkv_poll_device_status(rkv_handle h, void* stream) {
  if (h == nullptr) return RKV_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RKV_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, h->status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return RKV_ERR_CUDA;
  if (word != 0 && cudaMemset(h->status, 0, sizeof(unsigned)) != cudaSuccess) return RKV_ERR_CUDA;
  return (word & rkv::kStatusTimeout) ? RKV_ERR_TIMEOUT : RKV_OK;
}

RKV_API int rkv_set_wait_limit(rkv_handle h, long long nanoseconds) {
  if (h == nullptr || nanoseconds <= 0) return RKV_ERR_ARG;
  h->wait_ns = static_cast<unsigned long long>(nanoseconds);
  return RKV_OK;
}
