// Chunk attention over the rolling window on sm_100a (K2).
//
// O = softmax(Q K^T / sqrt(d)) V for one chunk's queries against the logical key
// stream "sinks, ring run 1, ring run 2 (wrap), current chunk" (up to four
// segments). Block-causal at chunk granularity means there is no mask inside
// that stream ("ABot-World流式因果推理深度解析", §机制二: a new block's queries see
// their own block plus the history blocks of the window, frames inside a block see
// each other; "从40步到4步：LingBot-World 2.0实时推理蒸馏（causal_fast）原理与关键代码
// 解读", §3: window slice then attention(roped_query, k_cache, v_cache)). Keys
// outside the window are never loaded, so masked tiles are never issued; the
// only masking is of the ragged last tile of each segment.
//
// Queries and keys arrive already rotated (RoPE applied by the frame-run kernel on
// their way into the head-major staging / rotated-K ring), V raw. The same kernels serve
// the cross-attention over the cached text K/V: one key segment, queries read token-major
// straight from the caller's buffer, no rotation.
//
// Two kernels: chunk_attention_kernel (one CTA per unit of one head x 256 query rows) for
// long key streams, and chunk_attention_short_kernel, a persistent form for key streams of
// at most kShortStreamTiles tiles (described at its definition). Both share the structure
// and the softmax below.
//
// Structure of one CTA (one head, 256 query rows = two 128-row tiles Q0, Q1):
//   warps 0-3  softmax for Q0 (one thread per query row = TMEM lane)
//   warps 4-7  softmax for Q1
//   warp 8     TMA producer: Q0/Q1 once, then K and V tiles (128 keys) into a
//              2-stage ring each
//   warp 9     TMEM allocator and tcgen05.mma issuer (one thread)
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; the bf16
// probabilities P overwrite the first 64 columns of their S tile and feed the PV
// product straight from TMEM. MMA issue order per key tile j:
//   S0(j) = Q0 K_j^T, PV1(j-1), S1(j) = Q1 K_j^T, PV0(j)
// so that while one softmax warpgroup works on its tile the tensor core runs the
// other tile's products. PV0(j) -> S0(j+1) is query tile 0's critical chain, so the
// issuer observes V(j) and probes K(j+1) before it waits for P0(j) (where it is idle):
// nothing but that wait stands between P0(j) and the 16 products PV0(j), S0(j+1).
// Online softmax in the log2 domain against a running reference: each thread reads its
// S row once (64 columns at a time) and forms the numerators
// 2^(s/sqrt(d) log2 e - reference) directly; the tile's numerator sum both feeds the row
// sum and bounds the tile's largest numerator, so the reference moves (and O is rescaled,
// at the start of the next tile) only when that sum exceeds 2^8, and a sum above 2^64
// sends the warp to an exact path that takes the row maximum first (always used for the
// first tile). Exponentials run on the special-function unit, two pairs in eight on the
// FMA pipe as a polynomial; P is rounded to bf16 (nearest even) in pairs.
//
// Every mbarrier wait is bounded in wall time; on expiry the kernel records
// kStatusTimeout in the status word, stops issuing work, waits (bounded) for the
// copies and MMAs it already issued, frees TMEM and returns.
#include <algorithm>
#include <cfloat>
#include <mutex>

#include "numeric.cuh"
#include "ptx_sm100.cuh"
#include "rkv_internal.h"

namespace rkv {
namespace {

constexpr int kBM = 128;                  // query rows per tile (TMEM lanes)
constexpr int kBN = 128;                  // keys per tile
constexpr int kSlab = 128 * 64 * 2;       // 128 rows x 64 bf16, one 128-byte swizzle span per row
constexpr int kTile = 2 * kSlab;          // 128 rows x 128 bf16
constexpr int kThreads = 320;
constexpr int kSmemQ = 0;                 // Q0, Q1
constexpr int kSmemK = 2 * kTile;         // K stage 0, 1
constexpr int kSmemV = 4 * kTile;         // V stage 0, 1
constexpr int kSmemBar = 6 * kTile;
constexpr int kSmemBytes = 6 * kTile + 256 + 1024;  // tiles + barriers + alignment slack
constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr float kLazyRescale = 8.0f;    // exact path: move the reference when a maximum grows by > 2^8
constexpr float kLazySum = 256.0f;      // one-pass path: move the reference when a tile sum exceeds 2^8
constexpr float kSumSlack = 18446744073709551616.0f;  // 2^64: largest accepted one-pass tile sum

enum : int {
  kBarQ = 0,
  kBarKFull = 1,   // +stage
  kBarKEmpty = 3,  // +stage
  kBarVFull = 5,   // +stage
  kBarVEmpty = 7,  // +stage
  kBarSFull = 9,   // +tile (0, 1)
  kBarPFull = 11,  // +tile
  kBarODone = 13,
  kBarDrain = 14,
  kNumBars = 15
};

// TMEM column of the S / P tile and of the O accumulator of query tile t (0 or 1).
__device__ __forceinline__ constexpr uint32_t col_s(int t) { return static_cast<uint32_t>(t) * 128u; }
__device__ __forceinline__ constexpr uint32_t col_o(int t) { return 256u + static_cast<uint32_t>(t) * 128u; }
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kBM, kBN, false);        // K-major A and B
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBM, kHeadDim, true);   // B (V) MN-major

__device__ __forceinline__ void tile_of(const AttnParams& p, int j, int& src, int& krow, int& vrow,
                                        int& valid) {
  int t = j;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s < p.n_segs) {
      const int nt = (p.seg[s].n_rows + kBN - 1) / kBN;
      if (t < nt) {
        src = p.seg[s].src;
        krow = p.seg[s].k_row0 + t * kBN;
        vrow = p.seg[s].v_row0 + t * kBN;
        valid = min(kBN, p.seg[s].n_rows - t * kBN);
        return;
      }
      t -= nt;
    }
  }
  src = 0;
  krow = vrow = 0;
  valid = 0;
}

// K-major operand (Q or K tile): k-step kk covers elements [16kk, 16kk+16) of every row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_addr, int kk) {
  return ptx::smem_desc_sw128(tile_addr + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
}

// MN-major operand (V tile as B of O += P V): k-step kk covers keys [16kk, 16kk+16);
// the two 64-column halves of d are kSlab apart.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile_addr, int kk) {
  return ptx::smem_desc_sw128(tile_addr + kk * 2048, kSlab, 1024);
}

// two fp32 -> packed bf16x2 (lo in the low half), round to nearest even, one conversion
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 2^x for two lanes on the FMA / integer pipes instead of the special-function unit:
// t = x + 1.5*2^23 rounds x to the nearest integer r (kept in t's low mantissa bits),
// f = x - r in [-1/2, 1/2], 2^f by a degree-3 polynomial (max relative error 7.5e-5,
// coefficients fitted for minimal relative error by tests/exp2_poly.py),
// then r is added to the exponent field (the bits of 1.5*2^23 vanish under << 23).
// x is clamped to [-125, 126] so the result stays a positive normal number (a score far
// above the reference then shows up as a huge tile sum, as it does on the other path).
__device__ __forceinline__ void exp2_poly_x2(uint64_t x2, float& y0, float& y1) {
  float x0, x1;
  ptx::f2_unpack(x2, x0, x1);
  const uint64_t x = ptx::f2_pack(fminf(fmaxf(x0, -125.0f), 126.0f), fminf(fmaxf(x1, -125.0f), 126.0f));
  const uint64_t magic = ptx::f2_pack(12582912.0f, 12582912.0f);
  const uint64_t neg_magic = ptx::f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t neg_one = ptx::f2_pack(-1.0f, -1.0f);
  const uint64_t t = ptx::f2_add(x, magic);
  const uint64_t r = ptx::f2_add(t, neg_magic);
  const uint64_t f = ptx::f2_fma(r, neg_one, x);
  uint64_t q = ptx::f2_fma(ptx::f2_pack(0.05517166493030145f, 0.05517166493030145f), f,
                           ptx::f2_pack(0.24261112187715117f, 0.24261112187715117f));
  q = ptx::f2_fma(q, f, ptx::f2_pack(0.6932609862225388f, 0.6932609862225388f));
  q = ptx::f2_fma(q, f, ptx::f2_pack(0.9999280735783096f, 0.9999280735783096f));
  float t0, t1, q0, q1;
  ptx::f2_unpack(t, t0, t1);
  ptx::f2_unpack(q, q0, q1);
  y0 = __uint_as_float((__float_as_uint(t0) << 23) + __float_as_uint(q0));
  y1 = __uint_as_float((__float_as_uint(t1) << 23) + __float_as_uint(q1));
}

// Softmax numerators of 64 keys (one half of a 128-key row): p = 2^(s * sl2 - m), rounded to
// bf16 (nearest even, one paired conversion) and packed in pairs into 32 TMEM columns at tP;
// row sums (of the unrounded values) accumulate in acc.
// kPoly: kPolyPairs of every 8 pairs take the polynomial path (full tiles only).
#ifndef RKV_POLY_PAIRS
#define RKV_POLY_PAIRS 2
#endif
constexpr int kPolyPairs = RKV_POLY_PAIRS;
template <bool kPoly>
__device__ __forceinline__ void softmax_half(const uint32_t* sh, uint64_t c2, uint64_t nm2, uint32_t tP,
                                             uint64_t (&acc)[4]) {
  uint32_t pk[kBN / 4];
#pragma unroll
  for (int k = 0; k < kBN / 4; ++k) {
    const uint64_t x = ptx::f2_fma(ptx::f2_pack(__uint_as_float(sh[2 * k]), __uint_as_float(sh[2 * k + 1])), c2, nm2);
    float a, b;
    if (kPoly && (k & 7) < kPolyPairs) {
      exp2_poly_x2(x, a, b);
    } else {
      float x0, x1;
      ptx::f2_unpack(x, x0, x1);
      a = ptx::ex2(x0);
      b = ptx::ex2(x1);
    }
    acc[k & 3] = ptx::f2_add(acc[k & 3], ptx::f2_pack(a, b));
    pk[k] = pack_bf16x2(a, b);
  }
  ptx::tmem_st32(tP, pk);
}

// The same numerators for a whole 64-key half computed against the running reference
// (nm2 = -m) without storing them: packed pairs go to pk[0..31], so that the caller can
// check the tile sum before S is overwritten.
template <bool kPoly>
__device__ __forceinline__ void numerators_half(const uint32_t* sh, uint64_t c2, uint64_t nm2, uint32_t* pk,
                                                uint64_t (&acc)[4]) {
#pragma unroll
  for (int k = 0; k < kBN / 4; ++k) {
    const uint64_t x = ptx::f2_fma(ptx::f2_pack(__uint_as_float(sh[2 * k]), __uint_as_float(sh[2 * k + 1])), c2, nm2);
    float a, b;
    if (kPoly && (k & 7) < kPolyPairs) {
      exp2_poly_x2(x, a, b);
    } else {
      float x0, x1;
      ptx::f2_unpack(x, x0, x1);
      a = ptx::ex2(x0);
      b = ptx::ex2(x1);
    }
    acc[k & 3] = ptx::f2_add(acc[k & 3], ptx::f2_pack(a, b));
    pk[k] = pack_bf16x2(a, b);
  }
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// O (this thread's row, 128 fp32 TMEM columns at tO) *= f
__device__ __forceinline__ void scale_o(uint32_t tO, float f) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t rr[32];
    ptx::tmem_ld32(tO + 32 * c, rr);
#pragma unroll
    for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
    ptx::tmem_st32(tO + 32 * c, rr);
  }
}

// The x0 / renoise step (and the guidance combine when v_cond is set; this launch is then the
// unconditional branch, its output u) on 32 consecutive elements of this thread's row:
// ob holds the attention output of those elements as stored (bf16 pairs), off their index
// in the latent [Lq, H * d].
__device__ __forceinline__ void flow_epilogue32(const AttnParams& p, const FlowStep& step, long long off,
                                                const uint32_t (&ob)[16]) {
  const uint4* xtp = reinterpret_cast<const uint4*>(p.xt + off);
  const uint4* ep = reinterpret_cast<const uint4*>(p.eps + off);
  uint4* x0p = reinterpret_cast<uint4*>(p.x0 + off);
  uint4* xnp = reinterpret_cast<uint4*>(p.xt_next + off);
  const uint4* cp = reinterpret_cast<const uint4*>(p.v_cond + off);
  const bool cfg = p.v_cond != nullptr;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 xv = __ldg(xtp + v);
    uint4 ev = make_uint4(0, 0, 0, 0), cv = make_uint4(0, 0, 0, 0);
    if (step.renoise) ev = __ldg(ep + v);
    if (cfg) cv = __ldg(cp + v);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
    uint32_t o0[4], o1[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t vw = ob[4 * v + q];
      uint16_t a0, a1, b0 = 0, b1 = 0;
      if (cfg) {
        step.apply_cfg_bits(xw[q], cw[q], vw, ew[q], p.cfg_scale, a0, b0);
        step.apply_cfg_bits(xw[q] >> 16, cw[q] >> 16, vw >> 16, ew[q] >> 16, p.cfg_scale, a1, b1);
      } else {
        step.apply_bits(xw[q], vw, ew[q], a0, b0);
        step.apply_bits(xw[q] >> 16, vw >> 16, ew[q] >> 16, a1, b1);
      }
      o0[q] = static_cast<uint32_t>(a0) | (static_cast<uint32_t>(a1) << 16);
      o1[q] = static_cast<uint32_t>(b0) | (static_cast<uint32_t>(b1) << 16);
    }
    x0p[v] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
    if (step.renoise) xnp[v] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
  }
}

// The ragged last tile of each key segment: its index in the key stream and its number of
// valid keys (-1 and kBN for absent segments).
__device__ __forceinline__ void ragged_tiles(const AttnParams& p, int (&rag_j)[kMaxSegs], int (&rag_v)[kMaxSegs]) {
  int first = 0;
#pragma unroll
  for (int sg = 0; sg < kMaxSegs; ++sg) {
    rag_j[sg] = -1;
    rag_v[sg] = kBN;
    if (sg < p.n_segs) {
      const int nt = (p.seg[sg].n_rows + kBN - 1) / kBN;
      rag_j[sg] = first + nt - 1;
      rag_v[sg] = p.seg[sg].n_rows - (nt - 1) * kBN;
      first += nt;
    }
  }
}

// valid keys of key tile j (kBN unless it is a segment's ragged last tile)
__device__ __forceinline__ int tile_valid(int j, const int (&rag_j)[kMaxSegs], const int (&rag_v)[kMaxSegs]) {
  int valid = kBN;
#pragma unroll
  for (int sg = 0; sg < kMaxSegs; ++sg)
    if (j == rag_j[sg]) valid = rag_v[sg];
  return valid;
}

// One key tile of this thread's query row: apply a pending change of reference to O and l,
// form the numerators of S(j) (one pass against the running reference, or the exact path
// on the first tile and after a score far above the reference) and leave P over S in TMEM.
// m_used: reference of the numerators in log2 units (p = 2^(s * sl2 - m_used)); l: row sum
// of the numerators in that reference's scale; pend: change of reference decided on this
// tile, applied at the next (when PV(j) has completed). The caller waits for the TMEM
// stores and signals P.
__device__ __forceinline__ void softmax_tile(int j, int valid, uint32_t tS, uint32_t tO, float sl2, uint64_t c2,
                                             float& m_used, float& l, float& pend) {
  // S(j) complete implies PV(j-1) complete: O now holds every product in the previous
  // reference's scale, so a pending change applies to O and l together
  if (__any_sync(0xffffffffu, pend != 1.0f)) scale_o(tO, pend);
  l *= pend;
  pend = 1.0f;
  bool stored = false;
  if (j > 0) {
    // one pass against the running reference
    const uint64_t nm2 = ptx::f2_pack(-m_used, -m_used);
    uint64_t acc[4] = {0, 0, 0, 0};
    uint32_t pk[kBN / 2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t sh[kBN / 2];
      ptx::tmem_ld64(tS + 64 * hh, sh);
      if (valid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i)
          if (64 * hh + i >= valid) sh[i] = 0xff800000u;
        numerators_half<false>(sh, c2, nm2, pk + 32 * hh, acc);
      } else {
        numerators_half<true>(sh, c2, nm2, pk + 32 * hh, acc);
      }
    }
    float rs[4];
    ptx::f2_unpack(ptx::f2_add(acc[0], acc[1]), rs[0], rs[1]);
    ptx::f2_unpack(ptx::f2_add(acc[2], acc[3]), rs[2], rs[3]);
    const float lt = (rs[0] + rs[1]) + (rs[2] + rs[3]);
    // the tile's numerator sum bounds its largest numerator: 2^max <= lt <= 128 * 2^max.
    // A sum above 2^64 (or not a number) sends the warp to the exact path below.
    if (!__any_sync(0xffffffffu, !(lt <= kSumSlack))) {
      l += lt;
      if (lt > kLazySum) {  // move the reference up by log2(lt) from the next tile on
        const float sh = lg2_approx(lt);
        pend = ptx::ex2(-sh);
        m_used += sh;
      }
      ptx::tmem_st64(tS, pk);
      stored = true;
    }
  }
  if (!stored) {
    // exact path (the first tile, or a score far above the reference): the row maximum
    // first, then the numerators
    float m_tile;
    {
      uint32_t sr[kBN];
      ptx::tmem_ld128(tS, sr);
      if (valid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i >= valid) sr[i] = 0xff800000u;
      }
      float mq[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t* t = sr + 32 * c;
        float m = ptx::fmax3(__uint_as_float(t[0]), __uint_as_float(t[1]), __uint_as_float(t[2]));
#pragma unroll
        for (int i = 3; i < 31; i += 2) m = ptx::fmax3(m, __uint_as_float(t[i]), __uint_as_float(t[i + 1]));
        mq[c] = fmaxf(m, __uint_as_float(t[31]));
      }
      m_tile = ptx::fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * sl2;
    }
    const bool need = m_tile > m_used + kLazyRescale;
    float alpha = 1.0f;
    if (need) {
      alpha = ptx::ex2(m_used - m_tile);
      m_used = m_tile;
    }
    l *= alpha;
    if (j > 0 && __any_sync(0xffffffffu, need)) scale_o(tO, alpha);
    const uint64_t nm2 = ptx::f2_pack(-m_used, -m_used);
    uint64_t acc[4] = {0, 0, 0, 0};
    // reload 64 columns at a time; P of the first half overwrites S columns 0..31,
    // already read, the second half's loads touch columns 64..127 only
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t sh[kBN / 2];
      ptx::tmem_ld64(tS + 64 * hh, sh);
      if (valid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i)
          if (64 * hh + i >= valid) sh[i] = 0xff800000u;
        softmax_half<false>(sh, c2, nm2, tS + 32 * hh, acc);
      } else {
        softmax_half<true>(sh, c2, nm2, tS + 32 * hh, acc);
      }
    }
    float rs[4];
    ptx::f2_unpack(ptx::f2_add(acc[0], acc[1]), rs[0], rs[1]);
    ptx::f2_unpack(ptx::f2_add(acc[2], acc[3]), rs[2], rs[3]);
    l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    chunk_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_vn,
                           const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // unit u = head * query blocks + block; CTAs from split_first on take half a unit's keys
  const int n_qb = (p.Lq + 2 * kBM - 1) / (2 * kBM);
  const int b = static_cast<int>(blockIdx.x);
  const int half = b >= p.split_first ? (b - p.split_first) & 1 : -1;
  const int u = half < 0 ? b : p.split_first + ((b - p.split_first) >> 1);
  const int head = u / n_qb;
  const int m0 = (u - head * n_qb) * (2 * kBM);
  const int j0 = half == 1 ? p.split_tiles : 0;  // first key tile of this CTA in the stream
  const int n_tiles = half < 0 ? p.n_tiles : (half == 0 ? p.split_tiles : p.n_tiles - p.split_tiles);
  const unsigned long long limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars[kBarQ], 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars[kBarKFull + s], 1);
      ptx::mbar_init(&bars[kBarKEmpty + s], 1);
      ptx::mbar_init(&bars[kBarVFull + s], 1);
      ptx::mbar_init(&bars[kBarVEmpty + s], 1);
      ptx::mbar_init(&bars[kBarSFull + s], 1);
      ptx::mbar_init(&bars[kBarPFull + s], kBM);
    }
    ptx::mbar_init(&bars[kBarODone], 1);
    ptx::mbar_init(&bars[kBarDrain], 1);
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_vc);
      ptx::prefetch_tmap(&tm_vn);
      ptx::mbar_arrive_expect_tx(&bars[kBarQ], 2 * kTile);
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < 2; ++c)
          if (p.q_token_major)
            ptx::tma_load_3d(smem + kSmemQ + t * kTile + c * kSlab, &tm_q, &bars[kBarQ], c * 64, head, m0 + t * kBM);
          else
            ptx::tma_load_3d(smem + kSmemQ + t * kTile + c * kSlab, &tm_q, &bars[kBarQ], c * 64, m0 + t * kBM, head);
      bool ok = true;
      int nk = 0, nv = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        int src, krow, vrow, valid;
        tile_of(p, j0 + j, src, krow, vrow, valid);
        if (j >= 2 && !ptx::mbar_wait(&bars[kBarKEmpty + s], ((j - 2) >> 1) & 1, limit)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bars[kBarKFull + s], kTile);
        for (int c = 0; c < 2; ++c)
          ptx::tma_load_3d(smem + kSmemK + s * kTile + c * kSlab, &tm_k, &bars[kBarKFull + s], c * 64, krow, head);
        nk = j + 1;
        if (j >= 2 && !ptx::mbar_wait(&bars[kBarVEmpty + s], ((j - 2) >> 1) & 1, limit)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bars[kBarVFull + s], kTile);
        for (int c = 0; c < 2; ++c) {
          if (src == 0)
            ptx::tma_load_3d(smem + kSmemV + s * kTile + c * kSlab, &tm_vc, &bars[kBarVFull + s], c * 64, vrow, head);
          else
            ptx::tma_load_3d(smem + kSmemV + s * kTile + c * kSlab, &tm_vn, &bars[kBarVFull + s], c * 64, head, vrow);
        }
        nv = j + 1;
      }
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // every copy issued must land before the CTA may exit
      ptx::mbar_wait(&bars[kBarQ], 0, kDrainNs);
      for (int j = (nk > 2 ? nk - 2 : 0); j < nk; ++j) ptx::mbar_wait(&bars[kBarKFull + (j & 1)], (j >> 1) & 1, kDrainNs);
      for (int j = (nv > 2 ? nv - 2 : 0); j < nv; ++j) ptx::mbar_wait(&bars[kBarVFull + (j & 1)], (j >> 1) & 1, kDrainNs);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr[2] = {ptx::smem_u32(smem + kSmemQ), ptx::smem_u32(smem + kSmemQ + kTile)};
      const uint32_t k_addr = ptx::smem_u32(smem + kSmemK);
      const uint32_t v_addr = ptx::smem_u32(smem + kSmemV);
      bool ok = ptx::mbar_wait(&bars[kBarQ], 0, limit);

      auto issue_s = [&](int t, uint32_t kt) {
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          ptx::mma_ss(tmem + col_s(t), desc_kmajor(q_addr[t], kk), desc_kmajor(kt, kk), kIdescS, kk > 0 ? 1u : 0u);
      };
      // O_t += P_t(jj) V(jj) with V(jj) already observed; returns false if a wait expired
      auto issue_pv = [&](int t, int jj) -> bool {
        if (!ptx::mbar_wait(&bars[kBarPFull + t], jj & 1, limit)) return false;
        ptx::tc_fence_after();
        const uint32_t vt = v_addr + (jj & 1) * kTile;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          ptx::mma_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, desc_v(vt, kk), kIdescPV,
                      (jj > 0 || kk > 0) ? 1u : 0u);
        if (t == 1) ptx::mma_commit(&bars[kBarVEmpty + (jj & 1)]);
        return true;
      };

      // The waits on K(j+1) and V(j) are taken before the wait for P0(j), where this thread is
      // idle anyway, so that PV0(j) and S0(j+1) follow P0(j) with no other wait between them.
      bool k_ready = ok && ptx::mbar_wait(&bars[kBarKFull + 0], 0, limit);
      if (!k_ready) ok = false;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1;
        if (!k_ready && !ptx::mbar_wait(&bars[kBarKFull + s], (j >> 1) & 1, limit)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t kt = k_addr + s * kTile;
        issue_s(0, kt);
        ptx::mma_commit(&bars[kBarSFull + 0]);
        if (j > 0 && !issue_pv(1, j - 1)) { ok = false; break; }
        issue_s(1, kt);
        ptx::mma_commit(&bars[kBarSFull + 1]);
        ptx::mma_commit(&bars[kBarKEmpty + s]);
        if (!ptx::mbar_wait(&bars[kBarVFull + s], (j >> 1) & 1, limit)) { ok = false; break; }
        k_ready = j + 1 < n_tiles && ptx::mbar_try_wait(&bars[kBarKFull + (s ^ 1)], ((j + 1) >> 1) & 1);
        if (!issue_pv(0, j)) { ok = false; break; }
      }
      if (ok && !issue_pv(1, n_tiles - 1)) ok = false;
      if (ok) ptx::mma_commit(&bars[kBarODone]);
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // everything issued must complete before TMEM is released
      ptx::mma_commit(&bars[kBarDrain]);
      ptx::mbar_wait(&bars[kBarDrain], 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;         // 0 or 1
    const int wq = warp & 3;          // warp within the warpgroup -> TMEM lanes 32*wq..
    const int r = threadIdx.x & 127;  // query row within the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t tS = lane_base + col_s(wg);
    const uint32_t tO = lane_base + col_o(wg);
    const float sl2 = p.scale_log2;
    const uint64_t c2 = ptx::f2_pack(sl2, sl2);
    float m_used = -INFINITY;  // reference of the numerators, log2 units: p = 2^(s * sl2 - m_used)
    float l = 0.f;             // row sum of the numerators, in the scale of the reference
    float pend = 1.0f;         // change of reference decided on the previous tile, not yet applied
    // the ragged last tile of each key segment: its index in the stream and its valid keys
    int rag_j[kMaxSegs], rag_v[kMaxSegs];
    ragged_tiles(p, rag_j, rag_v);
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = ptx::mbar_wait(&bars[kBarSFull + wg], j & 1, limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const int valid = tile_valid(j0 + j, rag_j, rag_v);
      softmax_tile(j, valid, tS, tO, sl2, c2, m_used, l, pend);
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars[kBarPFull + wg]);
    }
    if (ok) {
      ok = ptx::mbar_wait(&bars[kBarODone], 0, limit);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kStatusTimeout);
    } else if (half >= 0) {
      // half of a split unit: the unnormalised O row and its sum in the scale of the current
      // reference (a change decided on the last tile applied here), and the reference, for
      // the combine launch that follows
      ptx::tc_fence_after();
      float* po = p.part + (static_cast<long long>(b - p.split_first) * (2 * kBM) + wg * kBM + r) * kPartRow;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        ptx::tmem_ld32(tO + 32 * c, rr);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          reinterpret_cast<float4*>(po + 32 * c)[v] =
              make_float4(__uint_as_float(rr[4 * v]) * pend, __uint_as_float(rr[4 * v + 1]) * pend,
                          __uint_as_float(rr[4 * v + 2]) * pend, __uint_as_float(rr[4 * v + 3]) * pend);
      }
      reinterpret_cast<float4*>(po + 128)[0] = make_float4(m_used, l * pend, 0.f, 0.f);
    } else {
      ptx::tc_fence_after();
      const int row = m0 + wg * kBM + r;
      const bool live = row < p.Lq;
      const float inv_l = 1.0f / l;
      const long long base = (static_cast<long long>(row) * p.H + head) * kHeadDim;
      FlowStep step;
      step.sigma = p.sigma;
      step.renoise = p.sigma_next >= 0.0;
      step.sigma_next = step.renoise ? p.sigma_next : 0.0;
      step.one_minus_next = __dsub_rn(1.0, step.sigma_next);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        ptx::tmem_ld32(tO + 32 * c, rr);
        if (live) {
          uint32_t ob[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            ob[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv_l, __uint_as_float(rr[2 * i + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(p.out + base + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(ob[4 * v], ob[4 * v + 1], ob[4 * v + 2], ob[4 * v + 3]);
          if (p.flow) flow_epilogue32(p, step, base + 32 * c, ob);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------------------------
// Short key streams (at most kShortStreamTiles tiles: the cross-attention over a prompt's text
// tokens, the first chunks of a rollout). Each CTA stays resident and walks the units (head,
// 256-row query block) b, b + G, b + 2G, ... (G = gridDim.x <= SM count) with one running
// count of key tiles across units, so the stage and phase bookkeeping continues from one unit
// to the next. What this form adds over the long-stream kernel:
//   * the next unit's queries are loaded as soon as the current unit's last score products
//     have completed (a Q-empty barrier committed after them), and its first score product
//     S0 is issued before the current unit's last value product PV1, so the tensor core and
//     the softmax pipeline run across unit boundaries instead of draining per CTA;
//   * each query tile's epilogue starts when its own last value products complete (one
//     output barrier per tile) and overlaps the other tile's last softmax;
//   * the bf16 output leaves by TMA stores from a 16 KB staging buffer per query tile (one
//     64-column half at a time, the second half's TMEM reads overlapping the first half's
//     store), instead of one row per thread (each warp store instruction would touch 32
//     token rows H * 256 bytes apart).
// Warp roles, TMEM layout, the softmax and the bounded waits are those of the long-stream
// kernel above.
constexpr int kSmemStage = 6 * kTile;               // two 16 KB output halves, one per query tile
constexpr int kSmemBarShort = 6 * kTile + 2 * kSlab;
constexpr int kSmemBytesShort = kSmemBarShort + 256 + 1024;
static_assert(kSmemBytesShort <= 232448, "short-stream form exceeds the shared-memory limit");

enum : int {
  kSbQ = 0,        // queries of the current unit landed
  kSbQEmpty = 1,   // every score product of a unit completed: its query buffer is free
  kSbKFull = 2,    // +stage
  kSbKEmpty = 4,   // +stage
  kSbVFull = 6,    // +stage
  kSbVEmpty = 8,   // +stage
  kSbSFull = 10,   // +tile
  kSbPFull = 12,   // +tile
  kSbODone = 14,   // +tile: that tile's output of the unit is final
  kSbDrain = 16,
  kSbCount = 17
};

__global__ void __launch_bounds__(kThreads, 1)
    chunk_attention_short_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                 const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_vn,
                                 const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBarShort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kSbCount + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned long long limit = p.wait_limit_ns;
  const int n_qb = (p.Lq + 2 * kBM - 1) / (2 * kBM);
  const int n_units = n_qb * p.H;
  const int G = gridDim.x;
  const int n_my = (n_units - static_cast<int>(blockIdx.x) + G - 1) / G;  // units of this CTA (>= 1)

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars[kSbQ], 1);
    ptx::mbar_init(&bars[kSbQEmpty], 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars[kSbKFull + s], 1);
      ptx::mbar_init(&bars[kSbKEmpty + s], 1);
      ptx::mbar_init(&bars[kSbVFull + s], 1);
      ptx::mbar_init(&bars[kSbVEmpty + s], 1);
      ptx::mbar_init(&bars[kSbSFull + s], 1);
      ptx::mbar_init(&bars[kSbPFull + s], kBM);
      ptx::mbar_init(&bars[kSbODone + s], 1);
    }
    ptx::mbar_init(&bars[kSbDrain], 1);
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = p.n_tiles;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_vc);
      ptx::prefetch_tmap(&tm_vn);
      ptx::prefetch_tmap(&tm_o);
      bool ok = true;
      int nq = 0, nk = 0, nv = 0;  // loads issued (units for Q, global tiles for K and V)
      for (int i = 0; ok && i < n_my; ++i) {
        const int u = static_cast<int>(blockIdx.x) + i * G;
        const int head = u / n_qb;
        const int m0 = (u - head * n_qb) * (2 * kBM);
        if (i > 0 && !ptx::mbar_wait(&bars[kSbQEmpty], (i - 1) & 1, limit)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bars[kSbQ], 2 * kTile);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < 2; ++c)
            if (p.q_token_major)
              ptx::tma_load_3d(smem + kSmemQ + t * kTile + c * kSlab, &tm_q, &bars[kSbQ], c * 64, head, m0 + t * kBM);
            else
              ptx::tma_load_3d(smem + kSmemQ + t * kTile + c * kSlab, &tm_q, &bars[kSbQ], c * 64, m0 + t * kBM, head);
        nq = i + 1;
        for (int j = 0; j < n_tiles; ++j) {
          const int g = i * n_tiles + j;
          const int s = g & 1;
          int src, krow, vrow, valid;
          tile_of(p, j, src, krow, vrow, valid);
          if (g >= 2 && !ptx::mbar_wait(&bars[kSbKEmpty + s], ((g - 2) >> 1) & 1, limit)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&bars[kSbKFull + s], kTile);
          for (int c = 0; c < 2; ++c)
            ptx::tma_load_3d(smem + kSmemK + s * kTile + c * kSlab, &tm_k, &bars[kSbKFull + s], c * 64, krow, head);
          nk = g + 1;
          if (g >= 2 && !ptx::mbar_wait(&bars[kSbVEmpty + s], ((g - 2) >> 1) & 1, limit)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&bars[kSbVFull + s], kTile);
          for (int c = 0; c < 2; ++c) {
            if (src == 0)
              ptx::tma_load_3d(smem + kSmemV + s * kTile + c * kSlab, &tm_vc, &bars[kSbVFull + s], c * 64, vrow, head);
            else
              ptx::tma_load_3d(smem + kSmemV + s * kTile + c * kSlab, &tm_vn, &bars[kSbVFull + s], c * 64, head, vrow);
          }
          nv = g + 1;
        }
      }
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // every copy issued must land before the CTA may exit
      if (nq > 0) ptx::mbar_wait(&bars[kSbQ], (nq - 1) & 1, kDrainNs);
      for (int g = (nk > 2 ? nk - 2 : 0); g < nk; ++g) ptx::mbar_wait(&bars[kSbKFull + (g & 1)], (g >> 1) & 1, kDrainNs);
      for (int g = (nv > 2 ? nv - 2 : 0); g < nv; ++g) ptx::mbar_wait(&bars[kSbVFull + (g & 1)], (g >> 1) & 1, kDrainNs);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr[2] = {ptx::smem_u32(smem + kSmemQ), ptx::smem_u32(smem + kSmemQ + kTile)};
      const uint32_t k_addr = ptx::smem_u32(smem + kSmemK);
      const uint32_t v_addr = ptx::smem_u32(smem + kSmemV);
      auto issue_s = [&](int t, uint32_t kt) {
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          ptx::mma_ss(tmem + col_s(t), desc_kmajor(q_addr[t], kk), desc_kmajor(kt, kk), kIdescS, kk > 0 ? 1u : 0u);
      };
      // O_t += P_t(g) V(g) for global tile g, the unit's local tile index jl (0: overwrite O);
      // V(g) already observed. Returns false if a wait expired.
      auto issue_pv = [&](int t, int g, int jl) -> bool {
        if (!ptx::mbar_wait(&bars[kSbPFull + t], g & 1, limit)) return false;
        ptx::tc_fence_after();
        const uint32_t vt = v_addr + (g & 1) * kTile;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          ptx::mma_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, desc_v(vt, kk), kIdescPV,
                      (jl > 0 || kk > 0) ? 1u : 0u);
        if (t == 1) ptx::mma_commit(&bars[kSbVEmpty + (g & 1)]);
        return true;
      };
      bool ok = true;
      int g = 0;
      bool k_ready = false;
      for (int i = 0; ok && i < n_my; ++i) {
        if (!ptx::mbar_wait(&bars[kSbQ], i & 1, limit)) { ok = false; break; }
        for (int j = 0; j < n_tiles; ++j, ++g) {
          const int s = g & 1;
          if (!k_ready && !ptx::mbar_wait(&bars[kSbKFull + s], (g >> 1) & 1, limit)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t kt = k_addr + s * kTile;
          issue_s(0, kt);
          ptx::mma_commit(&bars[kSbSFull + 0]);
          if (g > 0) {
            // the previous tile's PV1; at j == 0 it is the previous unit's last
            if (!issue_pv(1, g - 1, j > 0 ? j - 1 : n_tiles - 1)) { ok = false; break; }
            if (j == 0) ptx::mma_commit(&bars[kSbODone + 1]);
          }
          issue_s(1, kt);
          ptx::mma_commit(&bars[kSbSFull + 1]);
          ptx::mma_commit(&bars[kSbKEmpty + s]);
          if (j == n_tiles - 1) ptx::mma_commit(&bars[kSbQEmpty]);
          if (!ptx::mbar_wait(&bars[kSbVFull + s], (g >> 1) & 1, limit)) { ok = false; break; }
          // the next tile's K, probed where this thread would otherwise wait for P0
          const bool more = j + 1 < n_tiles || i + 1 < n_my;
          k_ready = more && ptx::mbar_try_wait(&bars[kSbKFull + (s ^ 1)], ((g + 1) >> 1) & 1);
          if (!issue_pv(0, g, j)) { ok = false; break; }
          if (j == n_tiles - 1) ptx::mma_commit(&bars[kSbODone + 0]);
        }
      }
      if (ok && g > 0) {
        if (issue_pv(1, g - 1, n_tiles - 1))
          ptx::mma_commit(&bars[kSbODone + 1]);
        else
          ok = false;
      }
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // everything issued must complete before TMEM is released
      ptx::mma_commit(&bars[kSbDrain]);
      ptx::mbar_wait(&bars[kSbDrain], 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;         // 0 or 1
    const int wq = warp & 3;          // warp within the warpgroup -> TMEM lanes 32*wq..
    const int r = threadIdx.x & 127;  // query row within the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t tS = lane_base + col_s(wg);
    const uint32_t tO = lane_base + col_o(wg);
    const float sl2 = p.scale_log2;
    const uint64_t c2 = ptx::f2_pack(sl2, sl2);
    uint8_t* ostage = smem + kSmemStage + wg * kSlab;
    int rag_j[kMaxSegs], rag_v[kMaxSegs];
    ragged_tiles(p, rag_j, rag_v);
    FlowStep step;
    step.sigma = p.sigma;
    step.renoise = p.sigma_next >= 0.0;
    step.sigma_next = step.renoise ? p.sigma_next : 0.0;
    step.one_minus_next = __dsub_rn(1.0, step.sigma_next);
    // After an expired wait a warp skips all further waits and work but still runs every
    // named barrier of its warpgroup, so the warpgroup's four warps never part ways there.
    bool ok = true;
    int g = 0;
    for (int i = 0; i < n_my; ++i) {
      const int u = static_cast<int>(blockIdx.x) + i * G;
      const int head = u / n_qb;
      const int row0 = (u - head * n_qb) * (2 * kBM) + wg * kBM;
      float m_used = -INFINITY;
      float l = 0.f;
      float pend = 1.0f;
      for (int j = 0; j < n_tiles; ++j, ++g) {
        if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&bars[kSbSFull + wg], g & 1, limit));
        if (!ok) continue;
        ptx::tc_fence_after();
        const int valid = tile_valid(j, rag_j, rag_v);
        softmax_tile(j, valid, tS, tO, sl2, c2, m_used, l, pend);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars[kSbPFull + wg]);
      }
      if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&bars[kSbODone + wg], i & 1, limit));
      if (ok) ptx::tc_fence_after();
      // -------------------------------------------------------- epilogue of this unit's tile
      const int row = row0 + r;
      const bool live = row < p.Lq;
      const float inv_l = 1.0f / l;
      const long long base = (static_cast<long long>(row) * p.H + head) * kHeadDim;
      const bool store = ok && row0 < p.Lq;  // a tile wholly past Lq writes nothing
      // the previous unit's second-half store must have read the staging buffer
      if (r == 0) ptx::bulk_wait_read_all();
      ptx::named_bar_sync(1 + wg, kBM);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        if (c == 2) {
          // first half staged: store it, and wait for its read before the second half
          ptx::fence_proxy_async_smem();
          ptx::named_bar_sync(1 + wg, kBM);
          if (r == 0 && store) {
            ptx::tma_store_3d(&tm_o, ostage, 0, head, row0);
            ptx::bulk_commit_group();
            ptx::bulk_wait_read_all();
          }
          ptx::named_bar_sync(1 + wg, kBM);
        }
        if (!ok) continue;
        uint32_t rr[32];
        ptx::tmem_ld32(tO + 32 * c, rr);
        uint32_t ob[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          ob[q] = pack_bf16x2(__uint_as_float(rr[2 * q]) * inv_l, __uint_as_float(rr[2 * q + 1]) * inv_l);
        uint8_t* orow = ostage + r * 128;
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(orow + (((((c & 1) << 2) + v) ^ (r & 7)) << 4)) =
              make_uint4(ob[4 * v], ob[4 * v + 1], ob[4 * v + 2], ob[4 * v + 3]);
        if (live && p.flow) flow_epilogue32(p, step, base + 32 * c, ob);
      }
      ptx::fence_proxy_async_smem();
      ptx::named_bar_sync(1 + wg, kBM);
      if (r == 0 && store) {
        ptx::tma_store_3d(&tm_o, ostage, 64, head, row0);
        ptx::bulk_commit_group();  // read completion is awaited before the buffer is reused
      }
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeout);
    if (r == 0) ptx::bulk_wait_read_all();  // the buffer must stay until the last copy has read it
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, 512);
}


// The combine of a key-split unit (the last, partial wave of a long stream run as twice as
// many CTAs over half the keys each): one warp per query row, lane l owning columns
// 4l .. 4l+3. With the halves' references m_a, m_b and sums l_a, l_b (each half's O and sum
// in the scale of its own reference), m = max(m_a, m_b) and
//   O = (O_a 2^(m_a - m) + O_b 2^(m_b - m)) / (l_a 2^(m_a - m) + l_b 2^(m_b - m)),
// rounded to bf16 (nearest even) and stored token-major; the fused x0 / renoise step (and the
// guidance combine) then runs on the stored values, as in the attention kernels' epilogue.
__global__ void __launch_bounds__(256) attention_combine_kernel(const __grid_constant__ AttnParams p) {
  const int n_qb = (p.Lq + 2 * kBM - 1) / (2 * kBM);
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long n_split = static_cast<long long>(n_qb) * p.H - p.split_first;
  if (gw >= n_split * (2 * kBM)) return;
  const int t = static_cast<int>(gw / (2 * kBM));
  const int rr = static_cast<int>(gw - static_cast<long long>(t) * (2 * kBM));
  const int u = p.split_first + t;
  const int head = u / n_qb;
  const int row = (u - head * n_qb) * (2 * kBM) + rr;
  if (row >= p.Lq) return;
  const float* pa = p.part + (static_cast<long long>(2 * t) * (2 * kBM) + rr) * kPartRow;
  const float* pb = pa + static_cast<long long>(2 * kBM) * kPartRow;
  const float ma = pa[128], la = pa[129], mb = pb[128], lb = pb[129];
  const float m = fmaxf(ma, mb);
  const float fa = exp2f(ma - m), fb = exp2f(mb - m);
  const float inv = 1.0f / (la * fa + lb * fb);
  const float4 oa = reinterpret_cast<const float4*>(pa)[lane];
  const float4 ob = reinterpret_cast<const float4*>(pb)[lane];
  const uint32_t w0 = pack_bf16x2((oa.x * fa + ob.x * fb) * inv, (oa.y * fa + ob.y * fb) * inv);
  const uint32_t w1 = pack_bf16x2((oa.z * fa + ob.z * fb) * inv, (oa.w * fa + ob.w * fb) * inv);
  const long long off = (static_cast<long long>(row) * p.H + head) * kHeadDim + 4 * lane;
  *reinterpret_cast<uint2*>(p.out + off) = make_uint2(w0, w1);
  if (!p.flow) return;
  FlowStep step;
  step.sigma = p.sigma;
  step.renoise = p.sigma_next >= 0.0;
  step.sigma_next = step.renoise ? p.sigma_next : 0.0;
  step.one_minus_next = __dsub_rn(1.0, step.sigma_next);
  const bool cfg = p.v_cond != nullptr;
  const uint2 xv = __ldg(reinterpret_cast<const uint2*>(p.xt + off));
  const uint2 ev = step.renoise ? __ldg(reinterpret_cast<const uint2*>(p.eps + off)) : make_uint2(0, 0);
  const uint2 cv = cfg ? __ldg(reinterpret_cast<const uint2*>(p.v_cond + off)) : make_uint2(0, 0);
  const uint32_t xw[2] = {xv.x, xv.y}, ew[2] = {ev.x, ev.y}, cw[2] = {cv.x, cv.y}, vw[2] = {w0, w1};
  uint32_t o0[2], o1[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint16_t a0, a1, b0 = 0, b1 = 0;
    if (cfg) {
      step.apply_cfg_bits(xw[q], cw[q], vw[q], ew[q], p.cfg_scale, a0, b0);
      step.apply_cfg_bits(xw[q] >> 16, cw[q] >> 16, vw[q] >> 16, ew[q] >> 16, p.cfg_scale, a1, b1);
    } else {
      step.apply_bits(xw[q], vw[q], ew[q], a0, b0);
      step.apply_bits(xw[q] >> 16, vw[q] >> 16, ew[q] >> 16, a1, b1);
    }
    o0[q] = static_cast<uint32_t>(a0) | (static_cast<uint32_t>(a1) << 16);
    o1[q] = static_cast<uint32_t>(b0) | (static_cast<uint32_t>(b1) << 16);
  }
  *reinterpret_cast<uint2*>(p.x0 + off) = make_uint2(o0[0], o0[1]);
  if (step.renoise) *reinterpret_cast<uint2*>(p.xt_next + off) = make_uint2(o1[0], o1[1]);
}

}  // namespace

// Key streams of at most this many 128-key tiles take the short-stream form.
constexpr int kShortStreamTiles = 16;
// A unit is split in two only if each half keeps at least this many key tiles.
constexpr int kSplitMinTiles = 16;

cudaError_t launch_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_vc,
                             const CUtensorMap& tm_vn, const CUtensorMap& tm_o, const AttnParams& p,
                             cudaStream_t stream) {
  // the dynamic shared-memory limit is a per-device setting: raised once on every device
  // this process launches on, whichever host thread gets there first
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static bool configured[kMaxDevices] = {};
  static int sms[kMaxDevices] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      err = cudaFuncSetAttribute(chunk_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (err == cudaSuccess)
        err = cudaFuncSetAttribute(chunk_attention_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kSmemBytesShort);
      if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (err != cudaSuccess) return err;
      configured[dev] = true;
    }
  }
  const int n_qb = (p.Lq + 2 * kBM - 1) / (2 * kBM);
  const long long units = static_cast<long long>(n_qb) * p.H;
  const int sm = sms[dev] > 0 ? sms[dev] : 1;
  if (p.n_tiles <= kShortStreamTiles) {
    const unsigned grid = static_cast<unsigned>(std::min<long long>(units, sm));
    chunk_attention_short_kernel<<<grid, kThreads, kSmemBytesShort, stream>>>(tm_q, tm_k, tm_vc, tm_vn, tm_o, p);
    return cudaGetLastError();
  }
  // One CTA per unit, all of equal length: with U units on the SMs the last wave runs
  // U mod SMs of them while the other SMs idle. When that tail is at most half a wave (and
  // the stream long enough), its units run as two CTAs over half the keys each, so the tail
  // takes half as long; a combine launch then merges the halves.
  AttnParams q = p;
  q.split_first = static_cast<int>(units);
  q.split_tiles = 0;
  const long long tail = units % sm;
  if (p.part != nullptr && units > sm && tail > 0 && 2 * tail <= sm && 2 * tail <= p.part_ctas &&
      p.n_tiles >= 2 * kSplitMinTiles) {
    q.split_first = static_cast<int>(units - tail);
    q.split_tiles = p.n_tiles / 2;
  }
  const unsigned grid = static_cast<unsigned>(q.split_first + 2 * (units - q.split_first));
  chunk_attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_k, tm_vc, tm_vn, q);
  err = cudaGetLastError();
  if (err != cudaSuccess || q.split_first == units) return err;
  const long long warps = (units - q.split_first) * (2 * kBM);
  attention_combine_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(q);
  return cudaGetLastError();
}

}  // namespace rkv
