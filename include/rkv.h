/*
 * rkv.h - C ABI of librkv.so: block-causal chunk attention over a fixed-size
 * rolling KV cache with never-evicted sink frames, 3D RoPE (absolute or
 * relative), the clean t=0 K/V write-back, and the flow-matching x0/renoise
 * epilogue, as hand-written sm_100a (B200) CUDA kernels.
 *
 * Pages cited by title and section:
 *  [P1] "LingBot-World 2.0因果预训练范式深度剖析：为什么它能持续生成视频而不“掉画质”"
 *       (sheratonhq.com/news/156439)
 *  [P2] "从40步到4步：LingBot-World 2.0实时推理蒸馏（causal_fast）原理与关键代码解读"
 *       (hmyw.cn/news/135683)
 *  [P3] LingBot-World 2.0 wan/ source-map article (kwkr.cn/news/564388)
 *  [P4] "ABot-World流式因果推理深度解析：KV缓存与块级注意力如何让24小时连续生成不漂移"
 *       (lpnh.cn/news/2488095)
 *
 * Conventions for every call:
 *  - Tensors are bf16, contiguous, token-major: [tokens, H, d] with tokens
 *    ordered frame, then latent grid row, then grid column. d must be 128.
 *  - Pointers named q/k/v/out/x/xt/eps/x0_out/xt_next_out are DEVICE
 *    pointers owned by the caller; they must be 16-byte aligned. The library
 *    never frees them and keeps no reference after the call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every device launch is asynchronous on that stream; host state
 *    (frames committed, slot map) advances when the call is enqueued.
 *  - Calls on one handle must be issued from one host thread and be ordered on
 *    one stream (the per-layer scratch and the handle's scratch for the split
 *    last wave of long attention launches are reused); separate handles may run
 *    on separate streams concurrently.
 *  - Return value: RKV_OK or one of the RKV_ERR_* codes below. Argument,
 *    order and capacity errors are detected on the host before anything is
 *    launched; then no state changes.
 */
#ifndef RKV_H_
#define RKV_H_

#ifdef __cplusplus
extern "C" {
#endif

#define RKV_OK 0
#define RKV_ERR_ARG 1         /* bad pointer, size, layer index or alignment            */
#define RKV_ERR_ORDER 2       /* start_frame != frames committed so far for that layer  */
#define RKV_ERR_CAPACITY 3    /* n_frames > window_frames - sink_frames                 */
#define RKV_ERR_UNSUPPORTED 4 /* d != 128, window > 256 frames, time id beyond table    */
#define RKV_ERR_CUDA 5        /* a CUDA runtime / driver call failed                    */
#define RKV_ERR_TIMEOUT 6     /* a bounded device wait expired (read via poll)          */
#define RKV_ERR_STATE 7       /* call needs rkv_set_rope_grid (or rkv_set_text_kv) first */

#define RKV_ROPE_ABSOLUTE 0   /* time id = absolute frame index                         */
#define RKV_ROPE_RELATIVE 1   /* time id re-based to the window and clamped to [0, W-1] */
#define RKV_ROPE_RELATIVE_SLOTS 2 /* time id = the frame's position in the visible window:
                                     sinks 0..S-1, then the kept history and the chunk up to
                                     W-1 (the slot-order reading of [P4] §机制三)        */

typedef struct rkv_ctx* rkv_handle;

/*
 * rkv_create - allocate the per-layer rolling caches.
 *  Window of `window_frames` frames ([P1] §滑动窗口 KV 缓存 local_attn_size; [P4] §机制一
 *  cache size local_attn_size x tokens per frame), of which the first
 *  `sink_frames` frames ever written are never evicted ([P1] §Attention Sink sink_size;
 *  [P4] §机制一 reference-view sinks). `tokens_per_frame` = T; `rope_mode` is
 *  RKV_ROPE_ABSOLUTE, RKV_ROPE_RELATIVE or RKV_ROPE_RELATIVE_SLOTS ([P3] §改造③
 *  start_frame; [P4] §机制三). The two relative modes agree except on the sink frames
 *  once older non-sink frames have been evicted: clamped re-basing gives such sinks id 0,
 *  slot order gives sink f id f.
 *  Device memory per layer (library-owned, freed by rkv_destroy, zero-filled):
 *  raw K and V rings [H][window*T][d], a rotated-K ring plus chunk area
 *  [H][(2*window - sink)*T][d] and a rotated-Q staging area [H][(window-sink)*T][d].
 *  Errors: RKV_ERR_ARG (non-positive sizes, sink >= window, null out),
 *  RKV_ERR_UNSUPPORTED (d != 128, window_frames > 256), RKV_ERR_CUDA (allocation).
 */
int rkv_create(int layers, int H, int d, int tokens_per_frame, int window_frames,
               int sink_frames, int rope_mode, rkv_handle* out);

/*
 * rkv_set_rope_grid - the latent grid and rotary layout (required before any
 *  call that rotates). grid_h * grid_w must equal tokens_per_frame; token i of
 *  a frame sits at row i / grid_w, column i % grid_w. The d/2 adjacent pairs
 *  (x[2p], x[2p+1]) are split pairs_t (time), pairs_h (row), pairs_w (column),
 *  in that order; pair j of an axis with n pairs turns by pos * theta^(-j/n).
 *  cos/sin tables are built on the host in double and stored as fp32.
 *  Errors: RKV_ERR_ARG (grid mismatch, pairs_t+pairs_h+pairs_w != d/2, theta <= 0).
 */
int rkv_set_rope_grid(rkv_handle h, int grid_h, int grid_w, double theta,
                      int pairs_t, int pairs_h, int pairs_w);

/*
 * rkv_write_chunk - commit `n_frames` frames of raw K/V ([n_frames*T, H, d]) to
 *  `layer` without attending (e.g. the five reference views that become the
 *  sinks, [P4] §一次流式生成 / §机制一). start_frame must equal the frames
 *  committed so far. Eviction follows [P2] §3: frames after the sinks are
 *  dropped oldest first. Errors: RKV_ERR_ARG, RKV_ERR_ORDER, RKV_ERR_CAPACITY,
 *  RKV_ERR_STATE (absolute mode needs the grid), RKV_ERR_CUDA.
 */
int rkv_write_chunk(rkv_handle h, int layer, const void* k, const void* v,
                    int n_frames, int start_frame, void* stream);

/*
 * rkv_chunk_attention - O = softmax(RoPE(Q) RoPE(K)^T / sqrt(d)) V for the
 *  chunk [start_frame, start_frame + n_frames) of `layer`: the chunk's queries
 *  see the sinks, the latest committed history that still fits the window, and
 *  the chunk itself, with no mask inside that set ([P2] §3 window slice then
 *  attention(roped_query, k_cache, v_cache); [P4] §机制二 block-causal mask).
 *  q, k, v, out: [n_frames*T, H, d]. commit = 0: a denoise read, the cache is
 *  unchanged. commit = 1: the clean t=0 pass ([P2] §3; [P4] §机制二 干净上下文回写):
 *  same attention, then k/v are written into the ring (raw K in both modes).
 *  Errors: RKV_ERR_ARG, RKV_ERR_ORDER, RKV_ERR_CAPACITY, RKV_ERR_STATE,
 *  RKV_ERR_UNSUPPORTED (absolute time id >= 65536), RKV_ERR_CUDA.
 */
int rkv_chunk_attention(rkv_handle h, int layer, const void* q, const void* k, const void* v,
                        void* out, int n_frames, int start_frame, int commit, void* stream);

/*
 * Flow-matching epilogue fused into the attention output store: the attention
 *  output (rounded to bf16, exactly the value written to `out`) is taken as the
 *  flow prediction v of the latent [n_frames*T, H*d] and the epilogue of
 *  rkv_flow_x0_renoise is applied to it in the same kernel. Fields as there.
 */
typedef struct {
  const void* xt;        /* [n_frames*T, H*d] bf16, current noisy latent        */
  const void* eps;       /* [n_frames*T, H*d] bf16, noise for the renoise step  */
  double sigma;          /* sigma of this step                                  */
  double sigma_next;     /* next sigma; < 0 marks the last step (no renoise)    */
  void* x0_out;          /* [n_frames*T, H*d] bf16 out                          */
  void* xt_next_out;     /* [n_frames*T, H*d] bf16 out; may be NULL on last step */
} rkv_flow_epilogue;

/* rkv_chunk_attention_flow - rkv_chunk_attention plus the fused epilogue
 *  (`epi` NULL = no epilogue). Errors as rkv_chunk_attention. */
int rkv_chunk_attention_flow(rkv_handle h, int layer, const void* q, const void* k,
                             const void* v, void* out, int n_frames, int start_frame,
                             int commit, const rkv_flow_epilogue* epi, void* stream);

/*
 * rkv_chunk_attention_cfg_flow - the unconditional branch of a classifier-free
 *  guidance step with the guided epilogue fused into its output store. The
 *  causal pre-training mode samples every chunk in 40 steps with guidance
 *  scale 5.0, two forwards per step ([P2] §为什么需要, mode table), and keeps
 *  one KV cache per branch ([P3] §两种推理模式): create one handle per branch,
 *  run the conditional branch with rkv_chunk_attention on its handle first,
 *  then this call on the unconditional handle `h` with v_cond = that output.
 *  The epilogue takes u = this call's bf16 output (the value written to
 *  `out`), v = u + cfg_scale * (c - u) in fp64 with c = v_cond, and then
 *  applies the step of rkv_flow_x0_renoise to v.
 *  v_cond: [n_frames*T, H*d] bf16, device, 16-byte aligned, caller-owned, read
 *  only; it must not overlap out. epi must be non-NULL. Other arguments and
 *  errors as rkv_chunk_attention_flow.
 */
int rkv_chunk_attention_cfg_flow(rkv_handle h, int layer, const void* q, const void* k,
                                 const void* v, void* out, int n_frames, int start_frame,
                                 int commit, const rkv_flow_epilogue* epi, const void* v_cond,
                                 double cfg_scale, void* stream);

/*
 * rkv_set_text_kv - fill the cross-attention cache of `layer` with the text
 *  context's K and V. The text K/V are computed once per prompt and reused by
 *  every later chunk ([P1] §核心答案 CrossAttention_KVCache; [P2] §3 cross-attn
 *  cache; [P4] §一次流式生成的完整链路 step 1: the 512-token text embedding is
 *  computed once, and a prompt change rebuilds only this cache while the
 *  self-attention history stays). k_text, v_text: [n_text, H, d] bf16 device
 *  pointers, token-major, 16-byte aligned, caller-owned, copied (bit copy) on
 *  `stream` into library-owned [H][n_text][d] buffers, so the caller may reuse
 *  its buffers once the copy has run on that stream. 1 <= n_text <= 65536. No
 *  RoPE is applied (cross-attention has no positions). Growing n_text beyond
 *  the largest value set so far on this layer reallocates and synchronises the
 *  device. rkv_reset clears the cache. Errors: RKV_ERR_ARG, RKV_ERR_UNSUPPORTED
 *  (n_text > 65536), RKV_ERR_CUDA.
 */
int rkv_set_text_kv(rkv_handle h, int layer, const void* k_text, const void* v_text, int n_text,
                    void* stream);

/*
 * rkv_cross_attention - out = softmax(q K_text^T / sqrt(d)) V_text per head over
 *  all n_text cached text tokens, no mask and no RoPE. q, out: [n_tokens, H, d]
 *  bf16 device pointers, token-major, 16-byte aligned, caller-owned; any
 *  n_tokens >= 1 (a chunk's video tokens: n_frames * T). Runs the tcgen05
 *  attention kernel with one key segment. Needs no rope grid and no frame
 *  order; the self-attention cache is neither read nor changed. Errors:
 *  RKV_ERR_ARG, RKV_ERR_STATE (no text K/V set on this layer), RKV_ERR_CUDA.
 */
int rkv_cross_attention(rkv_handle h, int layer, const void* q, void* out, int n_tokens,
                        void* stream);

/*
 * rkv_rope_apply - rotate x [n_frames*T, H, d] in place with the handle's 3D
 *  RoPE. Absolute mode: t = frame index ([P3] §改造③ rope_apply(..., start_frame)).
 *  Relative mode: t = clamp(f - (window_end_frame - window_frames), 0, W-1),
 *  window_end_frame = one past the last frame of the window ([P4] §机制三).
 *  Slot-order mode: t = f for a sink frame (f < sink_frames), otherwise
 *  f - max(0, window_end_frame - window_frames), then clamped to [0, W-1] (the
 *  frame's position in that window). window_end_frame is ignored in absolute mode. fp32 arithmetic, bf16 round-to-nearest-even out.
 *  Errors: RKV_ERR_ARG, RKV_ERR_STATE, RKV_ERR_UNSUPPORTED, RKV_ERR_CUDA.
 */
int rkv_rope_apply(rkv_handle h, void* x, int n_frames, int start_frame,
                   int window_end_frame, void* stream);

/*
 * rkv_flow_x0_renoise - x0 = xt - sigma * v; if sigma_next >= 0 also
 *  xt_next = (1 - sigma_next) * x0 + sigma_next * eps ([P2] §2 _convert_flow_pred_to_x0
 *  and re-noise to the next timestep; §精度 flow->x0 in double). n elements,
 *  bf16 in/out, fp64 arithmetic without fused multiply-add, round-to-nearest-even
 *  on output; renoise uses the unrounded fp64 x0. eps / xt_next_out may be NULL
 *  when sigma_next < 0. Errors: RKV_ERR_ARG, RKV_ERR_CUDA.
 */
int rkv_flow_x0_renoise(const void* xt, const void* v, const void* eps, double sigma,
                        double sigma_next, void* x0_out, void* xt_next_out, long long n,
                        void* stream);

/*
 * rkv_flow_cfg_x0_renoise - classifier-free guidance combine, then the step of
 *  rkv_flow_x0_renoise: v = v_uncond + cfg_scale * (v_cond - v_uncond) in fp64
 *  (each operation rounded on its own), x0 = xt - sigma * v, and if
 *  sigma_next >= 0 xt_next = (1 - sigma_next) * x0 + sigma_next * eps
 *  ([P2] §为什么需要: causal pre-training samples with guidance scale 5.0;
 *  [P3] §两种推理模式: a conditional and an unconditional branch). n elements,
 *  bf16 in/out, all device pointers 16-byte aligned; eps / xt_next_out may be
 *  NULL when sigma_next < 0. Errors: RKV_ERR_ARG, RKV_ERR_CUDA.
 */
int rkv_flow_cfg_x0_renoise(const void* xt, const void* v_cond, const void* v_uncond,
                            const void* eps, double cfg_scale, double sigma, double sigma_next,
                            void* x0_out, void* xt_next_out, long long n, void* stream);

/* rkv_slot_frames - host copy of the slot -> frame map of `layer`: frames_out[W],
 *  -1 = empty. Slots [0, S) hold the sinks; frame f >= S lives in slot
 *  S + (f - S) mod (W - S). Errors: RKV_ERR_ARG. */
int rkv_slot_frames(rkv_handle h, int layer, int* frames_out);

/* rkv_frames_committed - frames committed so far to `layer`. Errors: RKV_ERR_ARG. */
int rkv_frames_committed(rkv_handle h, int layer, int* out);

/* rkv_cache_ptrs - device pointers of the raw K and V rings of `layer`, each
 *  [H][W*T][d] bf16 with slot s at rows [s*T, (s+1)*T). Library-owned, valid
 *  until rkv_destroy; for read-back only. Errors: RKV_ERR_ARG. */
int rkv_cache_ptrs(rkv_handle h, int layer, void** k, void** v);

/* rkv_reset - forget all frames of every layer and zero the caches (synchronous).
 *  Errors: RKV_ERR_ARG, RKV_ERR_CUDA. */
int rkv_reset(rkv_handle h);

/* rkv_destroy - free everything the handle owns (synchronises the device). */
int rkv_destroy(rkv_handle h);

/* rkv_status_string - static text for a status code. */
const char* rkv_status_string(int status);

/* rkv_poll_device_status - synchronise `stream`, read and clear the handle's
 *  device status word. RKV_ERR_TIMEOUT if a kernel's bounded wait expired since
 *  the last poll (that kernel stopped early and its output is invalid). */
int rkv_poll_device_status(rkv_handle h, void* stream);

/* rkv_set_wait_limit - cap, in nanoseconds, on each bounded device wait of the
 *  attention kernel's main loop (default 2e9). Diagnostic: a tiny cap makes the
 *  wait expire so the timeout path can be tested. Errors: RKV_ERR_ARG. */
int rkv_set_wait_limit(rkv_handle h, long long nanoseconds);

/*
 * rkv_chunk_attention_noalloc - chunk attention without a handle and without
 *  allocating device memory, for callers that may not call cudaMalloc (a host
 *  framework whose allocator must own every byte, a real-time or sandboxed
 *  process that forbids allocation after start-up, a library limited to the
 *  buffers its caller passes in). The pages have no counterpart: this is an
 *  interface for such callers, not a step of the method.
 *  The caller holds the window itself: k_window / v_window are the
 *  n_window_frames frames the chunk attends to, in logical order (sinks,
 *  history, then the chunk's own n_frames frames last), token-major
 *  [n_window_frames*T, H, 128] bf16; frame_ids (host, n_window_frames ints) are
 *  their absolute frame indices, non-negative and strictly increasing, the last
 *  n_frames being start_frame.. . q and out are [n_frames*T, H, 128]. RoPE: theta
 *  1e4, pairs 22/21/21, time id the frame index (RKV_ROPE_ABSOLUTE, ids < 4096) or
 *  re-based and clamped to [0, window_frames-1] (RKV_ROPE_RELATIVE; then
 *  n_window_frames <= window_frames <= 4096). Output as rkv_chunk_attention.
 *  Scratch: one static device array of 32 MiB per device (RoPE tables, rotated
 *  Q and K, a status word), held from the library's first use on that device
 *  until exit. The first call on a device looks up the array's device address;
 *  make that first call before any stream capture. Calls share the array: calls
 *  that overlap on the GPU race. An expired device wait is not reported here.
 *  Errors: RKV_ERR_ARG, RKV_ERR_UNSUPPORTED (absolute id >= 4096, relative
 *  window_frames > 4096, window in more than 7 runs of consecutive frames),
 *  RKV_ERR_CAPACITY (the window, queries and
 *  tables need more than the 32 MiB array), RKV_ERR_CUDA. Argument and size
 *  errors launch nothing.
 */
int rkv_chunk_attention_noalloc(const void* q, const void* k_window, const void* v_window, void* out,
                                int H, int tokens_per_frame, int grid_h, int grid_w, int window_frames,
                                int rope_mode, int n_frames, int start_frame, const int* frame_ids,
                                int n_window_frames, void* stream);

/* rkv_timing_begin - start recording a CUDA event pair around each attention
 *  kernel launch (on the caller's stream), for at most max_launches launches.
 *  Instrumentation only: nothing is skipped. Errors: RKV_ERR_ARG, RKV_ERR_CUDA. */
int rkv_timing_begin(rkv_handle h, int max_launches);

/* rkv_timing_end - synchronise the recorded events, write the duration (ms) of
 *  each recorded attention launch to ms_out[0 .. *n_out) (at most max) and stop
 *  recording. Errors: RKV_ERR_ARG, RKV_ERR_CUDA. */
int rkv_timing_end(rkv_handle h, float* ms_out, int max, int* n_out);

/*
 * rkv_plan_window - host-only planner (no GPU needed): the key segments that
 *  chunk [start_frame, start_frame + n_frames) attends to, in logical order,
 *  given `frames_committed` frames already in a window of W frames with S sinks.
 *  Writes up to max_segs records of 4 ints to seg_out:
 *    {source (0 = ring slots, 1 = the call's own chunk), first slot (source 0) or
 *     first chunk frame (source 1), number of frames, absolute id of the first frame}
 *  and their count to *n_segs. Errors: RKV_ERR_ARG, RKV_ERR_ORDER, RKV_ERR_CAPACITY.
 */
int rkv_plan_window(int window_frames, int sink_frames, int frames_committed, int n_frames,
                    int start_frame, int* seg_out, int max_segs, int* n_segs);

/*
 * rkv_copy_heads - strided copies of per-head vectors (d = 128 bf16 each), the data
 *  movement around the sequence <-> head exchange of head-sharded attention
 *  ("从40步到4步..." / LingBot-World `wan/` source map, §多卡加速: Ulysses sequence
 *  parallelism, an all-to-all before and after attention with ulysses_size | num_heads).
 *  Each of the n_runs records copies n_tok tokens x n_heads heads: head vector (t, h)
 *  moves from src + t * src_tok_stride + h * src_head_stride to the same offsets in dst
 *  (strides in bf16 elements, multiples of 8; src and dst 16-byte aligned, not
 *  overlapping). Device pointers; asynchronous on `stream`; runs are issued up to eight
 *  per kernel launch. A bit copy: no arithmetic. Errors: RKV_ERR_ARG (null or misaligned
 *  pointer, negative count or stride not a multiple of 8, n_heads < 1), RKV_ERR_CUDA.
 */
typedef struct rkv_head_copy {
  const void* src;
  void* dst;
  long long src_tok_stride, src_head_stride;
  long long dst_tok_stride, dst_head_stride;
  int n_tok;
} rkv_head_copy;
int rkv_copy_heads(const rkv_head_copy* runs, int n_runs, int n_heads, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H_ */
