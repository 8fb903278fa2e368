// Chunk attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs under an allocator
// they do not own (a host framework's caching pool that must see every byte), in
// a process whose allocation calls are forbidden after start-up (real-time
// loops, certified or sandboxed runtimes), or inside a library that may only use
// the buffers its own caller hands in. They cannot create an rkv handle (the
// handle allocates its rings and staging). This entry point serves them: the
// caller keeps the window itself, in logical order, and passes it in; the
// rotated queries and keys, the RoPE tables and a status word go to one
// file-scope static device array of fixed size instead of to allocated scratch.
//
// The array is kStaticScratchBytes (32 MiB) per device, created when the module
// is loaded on that device and held until the process exits. Every call shares
// it and it keeps the last call's contents: two calls that overlap on the GPU
// (different streams, no ordering between them) race on it.
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/rkv.h"
#include "rkv_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kNoAllocMaxTime = 4096;   // absolute time ids must stay below this
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mu;
unsigned char* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device. In host code the symbol
// name is only a host-side stand-in, so the address is asked for once per device,
// with that device current, and cached.
int scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return RKV_ERR_CUDA;
    g_addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_addr[dev];
  return RKV_OK;
}

// (cos, sin) of pos * theta^(-j/n) for the three axis tables laid out back to back:
// time [n_t][pt], row [gh][ph], column [gw][pw]; double precision, stored as fp32.
__global__ void rope_tables_kernel(float2* tab, int n_t, int pt, int gh, int ph, int gw, int pw, double theta) {
  const int nt = n_t * pt, nh = gh * ph, nw = gw * pw;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt + nh + nw; i += gridDim.x * blockDim.x) {
    int pos, j, n;
    if (i < nt) {
      pos = i / pt; j = i % pt; n = pt;
    } else if (i < nt + nh) {
      pos = (i - nt) / ph; j = (i - nt) % ph; n = ph;
    } else {
      pos = (i - nt - nh) / pw; j = (i - nt - nh) % pw; n = pw;
    }
    const double a = pos * pow(theta, -static_cast<double>(j) / n);
    double s, c;
    sincos(a, &s, &c);
    tab[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

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

bool encode(CUtensorMap* m, const void* base, uint64_t dim1, uint64_t dim2, uint64_t s1, uint64_t s2, uint32_t b1,
            uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(rkv::kHeadDim), dim1, dim2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {64, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" __attribute__((visibility("default"))) int rkv_chunk_attention_noalloc(
    const void* q, const void* k_window, const void* v_window, void* out, int H, int tokens_per_frame, int grid_h,
    int grid_w, int window_frames, int rope_mode, int n_frames, int start_frame, const int* frame_ids,
    int n_window_frames, void* stream) {
  using namespace rkv;
  if (!aligned16(q) || !aligned16(k_window) || !aligned16(v_window) || !aligned16(out) || frame_ids == nullptr)
    return RKV_ERR_ARG;
  if (H <= 0 || tokens_per_frame <= 0 || grid_h <= 0 || grid_w <= 0 ||
      static_cast<long long>(grid_h) * grid_w != tokens_per_frame || n_frames <= 0 || n_window_frames < n_frames ||
      window_frames <= 0 || start_frame < 0)
    return RKV_ERR_ARG;
  if (rope_mode != RKV_ROPE_ABSOLUTE && rope_mode != RKV_ROPE_RELATIVE) return RKV_ERR_ARG;
  const bool abs_mode = rope_mode == RKV_ROPE_ABSOLUTE;
  // the window is held in logical order: ids strictly increasing, the chunk's n_frames last
  for (int i = 0; i < n_window_frames; ++i) {
    if (frame_ids[i] < 0) return RKV_ERR_ARG;
    if (i > 0 && frame_ids[i] <= frame_ids[i - 1]) return RKV_ERR_ARG;
  }
  for (int i = 0; i < n_frames; ++i)
    if (frame_ids[n_window_frames - n_frames + i] != start_frame + i) return RKV_ERR_ARG;
  // relative mode: the caller's window cannot hold more frames than the window size
  if (!abs_mode && n_window_frames > window_frames) return RKV_ERR_ARG;
  const int max_id = frame_ids[n_window_frames - 1];
  if (abs_mode && max_id >= kNoAllocMaxTime) return RKV_ERR_UNSUPPORTED;
  if (!abs_mode && window_frames > kNoAllocMaxTime) return RKV_ERR_UNSUPPORTED;  // time-table rows
  // one rotation launch: the query run plus one run per block of consecutive frames
  int key_runs = 1;
  for (int i = 1; i < n_window_frames; ++i) key_runs += frame_ids[i] != frame_ids[i - 1] + 1;
  if (1 + key_runs > kMaxRuns) return RKV_ERR_UNSUPPORTED;
  const long long base = static_cast<long long>(start_frame) + n_frames - window_frames;

  const int T = tokens_per_frame, pt = 22, ph = 21, pw = 21;
  const int n_t = abs_mode ? max_id + 1 : window_frames;
  const long long Lq = static_cast<long long>(n_frames) * T;
  const long long Lk = static_cast<long long>(n_window_frames) * T;
  // every row of every head takes 256 bytes of the array: bound the counts before the sizes
  const long long max_rows = static_cast<long long>(kStaticScratchBytes / (kHeadDim * 2));
  if (Lk > max_rows || static_cast<long long>(H) > max_rows || Lk * H > max_rows || grid_h > max_rows ||
      grid_w > max_rows)
    return RKV_ERR_CAPACITY;
  const size_t off_tab = 256;
  const size_t tab_b = (static_cast<size_t>(n_t) * pt + static_cast<size_t>(grid_h) * ph +
                        static_cast<size_t>(grid_w) * pw) * sizeof(float2);
  const size_t off_q = align256(off_tab + tab_b);
  const size_t off_k = align256(off_q + static_cast<size_t>(H) * Lq * kHeadDim * 2);
  const size_t end = align256(off_k + static_cast<size_t>(H) * Lk * kHeadDim * 2);
  if (end > kStaticScratchBytes) return RKV_ERR_CAPACITY;  // window does not fit the fixed scratch

  unsigned char* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != RKV_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = reinterpret_cast<unsigned*>(scratch);
  float2* tab = reinterpret_cast<float2*>(scratch + off_tab);
  uint16_t* qs = reinterpret_cast<uint16_t*>(scratch + off_q);
  uint16_t* ks = reinterpret_cast<uint16_t*>(scratch + off_k);

  // the status word must start at zero; rows are fully rewritten below
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return RKV_ERR_CUDA;
  rope_tables_kernel<<<64, 256, 0, st>>>(tab, n_t, pt, grid_h, ph, grid_w, pw, 1.0e4);
  if (cudaGetLastError() != cudaSuccess) return RKV_ERR_CUDA;

  FrameRunParams p;
  std::memset(&p, 0, sizeof(p));
  p.H = H;
  p.T = T;
  p.grid_w = grid_w;
  p.pairs_t = pt;
  p.pairs_h = ph;
  p.pairs_w = pw;
  p.t_lo = 0;
  p.t_hi = n_t - 1;
  p.tab_t = tab;
  p.tab_h = tab + n_t * pt;
  p.tab_w = tab + n_t * pt + grid_h * ph;
  auto tid = [&](int f) { return abs_mode ? f : static_cast<int>(f - base); };  // clamped in the kernel
  {
    FrameRun r;
    std::memset(&r, 0, sizeof(r));
    r.src = static_cast<const uint16_t*>(q);
    r.dst = qs;
    r.src_tok_stride = static_cast<long long>(H) * kHeadDim;
    r.src_head_stride = kHeadDim;
    r.dst_tok_stride = kHeadDim;
    r.dst_head_stride = Lq * kHeadDim;
    r.n_tok = static_cast<int>(Lq);
    r.t0 = tid(start_frame);
    r.rotate = 1;
    p.run[p.n_runs++] = r;
  }
  for (int a = 0; a < n_window_frames;) {
    int b = a + 1;
    while (b < n_window_frames && frame_ids[b] == frame_ids[b - 1] + 1) ++b;
    FrameRun r;
    std::memset(&r, 0, sizeof(r));
    r.src = static_cast<const uint16_t*>(k_window);
    r.dst = ks;
    r.src_tok_stride = static_cast<long long>(H) * kHeadDim;
    r.src_head_stride = kHeadDim;
    r.dst_tok_stride = kHeadDim;
    r.dst_head_stride = Lk * kHeadDim;
    r.src_tok0 = r.dst_tok0 = a * T;
    r.n_tok = (b - a) * T;
    r.t0 = tid(frame_ids[a]);
    r.rotate = 1;
    p.run[p.n_runs++] = r;
    a = b;
  }
  rc = launch_frame_runs(p, static_cast<int>(Lk > Lq ? Lk : Lq), st) == cudaSuccess ? RKV_OK : RKV_ERR_CUDA;
  if (rc != RKV_OK) return rc;

  CUtensorMap tm_q, tm_k, tm_v, tm_o;
  if (!encode(&tm_q, qs, Lq, H, kHeadDim * 2, Lq * kHeadDim * 2, kQueryBox, 1) ||
      !encode(&tm_o, out, H, Lq, kHeadDim * 2, static_cast<uint64_t>(H) * kHeadDim * 2, 1, kQueryBox) ||
      !encode(&tm_k, ks, Lk, H, kHeadDim * 2, Lk * kHeadDim * 2, kKeyBox, 1) ||
      !encode(&tm_v, v_window, H, Lk, kHeadDim * 2, static_cast<uint64_t>(H) * kHeadDim * 2, 1, kKeyBox))
    return RKV_ERR_CUDA;
  AttnParams ap;
  std::memset(&ap, 0, sizeof(ap));
  ap.n_segs = 1;
  ap.seg[0].src = 1;  // values come token-major from the caller's window
  ap.seg[0].k_row0 = 0;
  ap.seg[0].v_row0 = 0;
  ap.seg[0].n_rows = static_cast<int>(Lk);
  ap.n_tiles = static_cast<int>((Lk + kKeyBox - 1) / kKeyBox);
  ap.H = H;
  ap.Lq = static_cast<int>(Lq);
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim)));
  ap.out = static_cast<uint16_t*>(out);
  ap.sigma_next = -1.0;
  ap.status = status;
  ap.wait_limit_ns = 2000000000ull;
  return launch_attention(tm_q, tm_k, tm_v, tm_v, tm_o, ap, st) == cudaSuccess ? RKV_OK : RKV_ERR_CUDA;
}
