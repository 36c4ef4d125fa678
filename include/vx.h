/*
 * vx.h -- C ABI of libvx, B200 (sm_100a) kernels for the Voxtral Realtime
 * causal sliding-window audio encoder.
 *
 * Source of the operations: transcribe.cpp porting notes "Voxtral", section
 * "Architecture -> Voxtral Realtime 2602 (voxtral_realtime)" (causal conv stem,
 * 32 causal sliding-window (750) layers, RoPE theta 1e6 / head_dim 64, RMSNorm
 * pre-norm, SwiGLU MLP, 32-head MHA, no k_proj bias, FFN bias only on down) and
 * its "Streaming schedule" paragraph (4 encoder frames per 80 ms step); the
 * Core AI model card "Voxtral Mini 4B Realtime -- Core AI", section "Usage /
 * Known limitations" (the pages' streaming encoder keeps an append-only frame
 * buffer; this library replaces it with a W-slot ring).
 *
 * Conventions (all entry points):
 *  - Every pointer argument is a DEVICE pointer owned by the caller unless the
 *    comment says "host".  The library never allocates or frees device memory;
 *    scratch space is the caller's workspace `ws` of `ws_bytes` bytes, sized by
 *    the matching vx_*_workspace() query.  ws must be 256-byte aligned.
 *  - Work is enqueued on `stream` and is asynchronous; nothing synchronises the
 *    host except vx_status_check().
 *  - Activations are row-major and frame-major: [B, T, C] with C contiguous.
 *    Attention tensors are [B, T, H, D] with D contiguous.
 *  - bf16 tensors are passed as `const void*` holding IEEE bfloat16 bit patterns.
 *  - Return value: VX_OK, or an error code with a message in vx_last_error()
 *    (thread-local).  Argument errors are detected on the host before any work
 *    is enqueued.  A kernel whose bounded wait ran out records
 *    VX_ERR_DEVICE_TIMEOUT in the workspace status word (first 256 bytes of
 *    ws); read it with vx_status_check() and clear it with vx_status_reset().
 *  - Calls on distinct streams with distinct workspaces are thread-safe.
 *    Unsupported shapes return VX_ERR_UNSUPPORTED; there is no fallback path.
 */
#ifndef VX_H_
#define VX_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define VX_API __attribute__((visibility("default")))
#else
#define VX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vx_status {
  VX_OK = 0,
  VX_ERR_INVALID_ARG = 1,     /* null pointer, bad shape, misalignment, small ws */
  VX_ERR_UNSUPPORTED = 2,     /* valid but not built (e.g. head_dim != 64)       */
  VX_ERR_CUDA = 3,            /* a CUDA runtime/driver call or launch failed     */
  VX_ERR_DEVICE_TIMEOUT = 4   /* a bounded in-kernel wait expired                */
} vx_status;

typedef enum vx_dtype { VX_F32 = 0, VX_BF16 = 1 } vx_dtype;

/* Shape of one encoder layer.  Supported: head_dim 64, d_model a multiple of
 * 128 and <= 2048, n_heads*head_dim a multiple of 128, ffn_hidden a multiple
 * of 64, window >= 1.  Voxtral Realtime 2602: {1280, 32, 64, 5120, 750, 1e6, 1e-5}. */
typedef struct vx_layer_cfg {
  int d_model;
  int n_heads;
  int head_dim;
  int ffn_hidden;
  int window;        /* W: query i sees keys j with i - W < j <= i */
  float rope_theta;  /* inv_freq_m = theta^(-2m/head_dim), split-halves pairing */
  float eps;         /* RMSNorm epsilon */
} vx_layer_cfg;

/* One layer's parameters as the checkpoint holds them (PyTorch [out, in]
 * order, all bf16).  bg/bu may be NULL (the 2602 encoder has no gate/up bias).
 * Input of vx_pack_layer only. */
typedef struct vx_layer_params {
  const void *attn_norm_g;          /* [d]            */
  const void *wq, *wk, *wv;         /* [HD, d] each   */
  const void *bq, *bv;              /* [HD] each (k has no bias) */
  const void *wo;                   /* [d, HD]        */
  const void *bo;                   /* [d]            */
  const void *ffn_norm_g;           /* [d]            */
  const void *wg, *wu;              /* [F, d] each    */
  const void *bg, *bu;              /* [F] or NULL    */
  const void *wd;                   /* [d, F]         */
  const void *bd;                   /* [d]            */
} vx_layer_params;

/* A layer in the layout the kernels read (built by vx_pack_layer). */
typedef struct vx_layer_weights {
  const void *attn_norm_g;  /* [d] bf16                                        */
  const void *wqkv;         /* [3*HD, d] bf16: rows q | k | v                   */
  const void *bqkv;         /* [3*HD] bf16: bq | 0 | bv                         */
  const void *wo;           /* [d, HD] bf16                                     */
  const void *bo;           /* [d] bf16                                         */
  const void *ffn_norm_g;   /* [d] bf16                                         */
  const void *wgu;          /* [2F, d] bf16: gate/up rows interleaved in blocks
                               of 64 (gate f0..f0+63, up f0..f0+63, gate ...)   */
  const void *bgu;          /* [2F] bf16, same interleave (zeros if no bias)    */
  const void *wd;           /* [d, F] bf16                                      */
  const void *bd;           /* [d] bf16                                         */
} vx_layer_weights;

/* Per-layer ring-buffer K/V cache of `window` slots for n_streams streams.
 * k and v are [n_layers][n_streams][n_heads][window][head_dim] bf16; frame f of
 * stream s sits in slot f mod window.  pos[s] (device int64) counts the frames
 * already appended to stream s; the ring holds frames max(0,pos-W) .. pos-1. */
typedef struct vx_kv_ring {
  void *k;
  void *v;
  int64_t *pos;
  int n_layers;
  int n_streams;
  int window;
} vx_kv_ring;

/* ---------------------------------------------------------------- utilities */

VX_API const char *vx_last_error(void);       /* thread-local message of the last error */
VX_API const char *vx_version(void);
/* Bounded-wait limit for every in-kernel wait (default 1e9 ns).  Host setting,
 * read at launch time; affects launches enqueued afterwards (all threads). */
VX_API void vx_set_wait_timeout_ns(uint64_t ns);
/* Per-launch timing: while enabled (per calling thread), every kernel this
 * library enqueues is bracketed by CUDA events recorded on its launch stream.
 * vx_trace_read() synchronises those events, writes one "name milliseconds"
 * line per launch (in launch order) into buf (host, NUL-terminated, truncated
 * to cap), forgets them and returns how many there were.  Do not enable it
 * while capturing a CUDA graph. */
VX_API void vx_trace_enable(int on);
VX_API int vx_trace_read(char *buf, size_t cap);
/* Number of kernels this library has enqueued since it was loaded (all threads). */
VX_API uint64_t vx_launch_count(void);
/* Clears the status word at the start of ws (async on stream). */
VX_API vx_status vx_status_reset(void *ws, cudaStream_t stream);
/* Synchronises `stream`, then returns VX_ERR_DEVICE_TIMEOUT if a kernel
 * recorded an expired wait in ws, else VX_OK (or VX_ERR_CUDA). */
VX_API vx_status vx_status_check(const void *ws, cudaStream_t stream);

/* Fills the packed layout of one layer.  packed_wqkv: [3*HD, d] bf16,
 * packed_bqkv: [3*HD] bf16, packed_wgu: [2F, d] bf16, packed_bgu: [2F] bf16.
 * The caller then points vx_layer_weights at these buffers and at the
 * unchanged norm gains, wo, bo, wd, bd. */
VX_API vx_status vx_pack_layer(const vx_layer_cfg *cfg, const vx_layer_params *in,
                        void *packed_wqkv, void *packed_bqkv,
                        void *packed_wgu, void *packed_bgu, cudaStream_t stream);

/* Reorders a Conv1d weight [out, in, 3] (PyTorch) to [out, 3, in], the
 * layout vx_conv_stem_fwd reads (bf16 both). */
VX_API vx_status vx_pack_conv_weight(const void *w, void *w_packed, int out_ch, int in_ch,
                              cudaStream_t stream);

/* ------------------------------------------------------------- operations */

/* Causal sliding-window multi-head attention with RoPE: the attention of
 * the encoder layer in the transcribe.cpp notes "Voxtral", section
 * "Architecture -> Voxtral Realtime 2602" (causal attention over a sliding
 * window of 750 frames, RoPE theta 1e6, head_dim 64, 32 heads): each frame
 * attends to itself and the W-1 frames before it.
 *   o_i = sum_{j: i-W < j <= i} softmax_j(<q'_i, k'_j> * scale) v_j per head,
 * with q', k' = RoPE(q, k) at positions pos0 + t when apply_rope != 0
 * (split-halves pairing, inv_freq_m = rope_theta^(-2m/D)).
 * q, k, v, o: [B, T, H, D] of dtype dt (VX_F32: fp32 CUDA-core path;
 * VX_BF16: tcgen05 tensor-core path, fp32 softmax).  D must be 64.
 * scale <= 0 selects 1/sqrt(D).  Workspace: vx_swa_attn_workspace(). */
VX_API vx_status vx_swa_attn_fwd(const void *q, const void *k, const void *v, void *o,
                          vx_dtype dt, int B, int T, int H, int D, int window,
                          int apply_rope, float rope_theta, int64_t pos0, float scale,
                          void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_swa_attn_workspace(vx_dtype dt, int B, int T, int H, int D, int apply_rope);

/* vx_swa_attn_fwd_noalloc: the same operation, arguments and results as
 * vx_swa_attn_fwd, for callers that cannot allocate device memory when they
 * run attention (real-time audio callbacks that must not wait on the
 * driver's allocator, plug-in hosts that own every device allocation, code
 * under a fixed memory budget).  It takes no workspace and allocates nothing:
 * its scratch (the RoPE-rotated q and k, and the status word of the bounded
 * waits) is one static device array of 32 MiB + 256 bytes inside this
 * library, held by every GPU that loads the library until the process exits.
 * Inputs and outputs are still the caller's.
 * Limit: with apply_rope, each rotated tensor takes B*T*H*64*es bytes
 * (es = 2 for bf16, 4 for fp32) rounded up to a multiple of 256; 2 * that
 * rounded size must be at most 32 MiB (33554432 bytes).  For bf16 that is
 * B*T*H <= 131072 (e.g. B=1, H=32: T <= 4096); for fp32, B*T*H <= 65536.
 * Without RoPE no scratch beyond the status word is used and any size runs.
 * Larger calls return VX_ERR_INVALID_ARG with a message and enqueue nothing.
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it together with the current context; it
 * is looked up again when the context changes (e.g. after cudaDeviceReset).
 * Make that first call before any stream capture.  Its kernels are counted by
 * vx_launch_count and timed by vx_trace_enable / vx_trace_read like those of
 * vx_swa_attn_fwd.  Every call clears the status word and overwrites the
 * rotated q/k,
 * and all calls share the one array: calls whose work overlaps on the GPU
 * (other streams, other threads) race on it.  A bounded wait that expires is
 * recorded only in that private status word; use vx_swa_attn_fwd with a
 * workspace to read it through vx_status_check.  (The pages describe no
 * counterpart: this entry point exists for those callers only.) */
VX_API vx_status vx_swa_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *o,
                                         vx_dtype dt, int B, int T, int H, int D, int window,
                                         int apply_rope, float rope_theta, int64_t pos0, float scale,
                                         cudaStream_t stream);

/* RMSNorm with optional residual add:
 *   h = x + r (r may be NULL), y = h / sqrt(mean(h^2) + eps) * g.
 * x, r, h_out: [M, d] fp32 (h_out may be NULL); g: [d] bf16;
 * y: [M, d] of dtype y_dt (bf16 for GEMM operands, fp32 for the final norm). */
VX_API vx_status vx_rms_norm_fwd(const float *x, const float *r, const void *g, float *h_out,
                          void *y, vx_dtype y_dt, int M, int d, float eps,
                          void *ws, size_t ws_bytes, cudaStream_t stream);

/* One encoder layer over B clips of T frames (whole-sequence, causal), as the
 * transcribe.cpp notes "Voxtral", section "Architecture -> Voxtral Realtime
 * 2602", state it: RMSNorm pre-norm, q/v/o projections with bias and k
 * without, RoPE (theta 1e6, head_dim 64), causal sliding-window attention
 * (750), and a SwiGLU MLP with bias on the down projection only:
 *   y0 = RMSNorm(x); q,k,v = y0 W^T + b; RoPE(q,k) at pos0 + t;
 *   h = x + SWA(q,k,v) Wo^T + bo; out = h + (silu(y1 Wg^T + bg) * (y1 Wu^T + bu)) Wd^T + bd,
 *   y1 = RMSNorm(h).
 * x, y: [B, T, d] fp32 (y may alias nothing in ws; x == y is allowed).
 * Workspace: vx_encoder_layer_workspace(). */
VX_API vx_status vx_encoder_layer_fwd(const vx_layer_cfg *cfg, const vx_layer_weights *w,
                               const float *x, float *y, int B, int T, int64_t pos0,
                               void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_encoder_layer_workspace(const vx_layer_cfg *cfg, int B, int T);

/* Causal conv stem (transcribe.cpp notes "Voxtral", section "Architecture ->
 * Voxtral Realtime 2602": causal convolutions with left padding only; shapes
 * of the stem as in the 2507 section): left-pad-only
 * Conv1d(n_mels -> d, k3, s1) + GELU, then
 * Conv1d(d -> d, k3, s2) + GELU (exact erf GELU, left zero padding of 2 frames
 * before each conv).  mel: [B, n_mels, Tm] fp32; w1p: [d, 3, n_mels] and
 * w2p: [d, 3, d] bf16 (vx_pack_conv_weight); b1, b2: [d] bf16;
 * out: [B, T_out, d] fp32 with T_out = (Tm - 1) / 2 + 1.
 * n_mels must be a multiple of 64.  Workspace: vx_conv_stem_workspace(). */
VX_API vx_status vx_conv_stem_fwd(const float *mel, const void *w1p, const void *b1,
                           const void *w2p, const void *b2, float *out,
                           int B, int n_mels, int Tm, int d,
                           void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_conv_stem_workspace(int B, int n_mels, int Tm, int d);

/* Streaming conv stem step with a conv padding cache (transcribe.cpp notes
 * "Voxtral", section "Frontend": the Realtime model's conv padding cache
 * carries continuity across streaming chunks; section "Architecture ->
 * Voxtral Realtime 2602": 8 mel frames = 4 encoder frames per step).
 * One chunk of n_new mel frames per stream continues the causal conv stem of
 * everything the stream has seen: conv1 reads mel frames t-2 .. t, conv2
 * output u reads conv1 outputs 2u-2 .. 2u, and the two frames before the
 * chunk come from the cache instead of the zero padding of vx_conv_stem_fwd.
 *   mel_new:  [S, n_mels, n_new] fp32, n_new even (8 for the 80 ms schedule)
 *   cache_x:  [S, 2, n_mels] bf16, the last two mel frames seen (rounded to bf16)
 *   cache_h1: [S, 2, d] bf16, the last two conv1 outputs (after GELU)
 *   out:      [S, n_new / 2, d] fp32
 * Both caches are read, then overwritten with this chunk's last two rows;
 * zero them before a stream's first chunk.  Weights as vx_conv_stem_fwd.
 * Returns VX_ERR_UNSUPPORTED for odd n_new.  Workspace:
 * vx_conv_stem_step_workspace().  The caches are owned by the caller and must
 * not be shared by concurrent calls. */
VX_API vx_status vx_conv_stem_step(const float *mel_new, const void *w1p, const void *b1,
                            const void *w2p, const void *b2, void *cache_x, void *cache_h1,
                            float *out, int S, int n_mels, int n_new, int d,
                            void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_conv_stem_step_workspace(int S, int n_mels, int n_new, int d);

/* Streaming log-mel frontend of the Realtime model (transcribe.cpp notes
 * "Voxtral", section "Frontend"): 16 kHz audio, 400-sample frames with a
 * periodic Hann window at hop 160 (n_fft 400), power spectrum, slaney mel
 * filterbank of 128 bands over 0-8000 Hz (area normalised), log10 of
 * max(mel, 1e-10), the fixed global maximum of the Realtime model
 * (max(log, 1.5 - 8)), then (x + 4) / 4.  Every frame depends on its own 400
 * samples only, so a stream is processed chunk by chunk.
 *   audio: [B, N] fp32;  mel: [B, 128, F] fp32 (the layout vx_conv_stem_fwd reads)
 *   center = 1 (a whole clip, or a stream's first chunk): reflect-padded by 200
 *     samples on both sides, the last frame dropped: F = N / 160 (N > 200, else
 *     VX_ERR_UNSUPPORTED);
 *   center = 0 (later chunks): the frames lying wholly inside the samples,
 *     F = 1 + (N - 400) / 160 (0 when N < 400); pass the samples from
 *     160 t0 - 200 on to continue the centred frame grid at frame t0.
 * With F = 0 nothing is read or written.  Arithmetic in fp32.  Workspace:
 * vx_log_mel_workspace(). */
VX_API vx_status vx_log_mel_fwd(const float *audio, float *mel, int B, int N, int center,
                         void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_log_mel_workspace(int B, int N);

/* Audio projector (transcribe.cpp notes "Voxtral", section "Architecture ->
 * Voxtral Realtime 2602", Projector): the encoder output x [B, T, d] fp32 is
 * reshaped to [B, T/4, 4d] (frames 4j .. 4j+3 concatenated in time order, the
 * last T % 4 frames dropped), then out = GELU(tok w1^T) w2^T without biases.
 *   w1: [hidden, 4d] bf16;  w2: [hidden, hidden] bf16;  out: [B, T/4, hidden] fp32
 * Tokens and the hidden activation are bf16 tensor-core operands (fp32
 * accumulate); GELU is the exact erf form.  d % 16 == 0, hidden % 128 == 0
 * (else VX_ERR_UNSUPPORTED).  With T < 4 there is no token: the call returns
 * VX_OK without reading or writing anything (the pointers may then be null).
 * Workspace: vx_projector_workspace(). */
VX_API vx_status vx_projector_fwd(const float *x, const void *w1, const void *w2, float *out,
                           int B, int T, int d, int hidden,
                           void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_projector_workspace(int B, int T, int d, int hidden);

/* Whole-clip encoder: conv stem -> n_layers encoder layers (positions from 0)
 * -> final RMSNorm with gain final_g ([d] bf16).  layers: HOST array of
 * n_layers weight structs (device pointers inside).  out: [B, T_out, d] fp32.
 * Workspace: vx_encoder_workspace(). */
VX_API vx_status vx_encoder_fwd(const vx_layer_cfg *cfg, const float *mel, int B, int n_mels, int Tm,
                         const void *w1p, const void *b1, const void *w2p, const void *b2,
                         const vx_layer_weights *layers, int n_layers, const void *final_g,
                         float *out, void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_encoder_workspace(const vx_layer_cfg *cfg, int B, int n_mels, int Tm);

/* Streaming prefill: runs the whole-sequence forward over the first T frames
 * of each of the ring's streams through the ring's n_layers layers, writes
 * each layer's K/V of frames max(0,T-W) .. T-1 into the ring (slot f mod W)
 * and sets pos[s] = T.  x: [S, T, d] fp32 layer-0 input, y: [S, T, d] fp32
 * output of the last layer (final RMSNorm applied when final_g != NULL).
 * Workspace: vx_encoder_layer_workspace(cfg, S, T). */
VX_API vx_status vx_stream_prefill(const vx_layer_cfg *cfg, const vx_layer_weights *layers,
                            const vx_kv_ring *ring, const float *x, float *y, int T,
                            const void *final_g, void *ws, size_t ws_bytes,
                            cudaStream_t stream);

/* Streaming step (transcribe.cpp notes "Voxtral", section "Architecture ->
 * Voxtral Realtime 2602": 8 mel frames = 4 encoder frames per 80 ms step; the
 * W-slot ring replaces the append-only frame buffer of the Core AI card's
 * streaming encoder, section "Usage / Known limitations"): n_new (1..8) new
 * frames per stream, for every stream of the ring, through the ring's
 * n_layers layers.  Per layer, new frame f = pos[s]+t
 * attends frames f' with f - W < f' <= f: older frames from the ring, the rest
 * from this step; every in-window ring slot is read before the new K/V are
 * written to slots (pos[s] + t) mod W.  Advances pos[s] += n_new at the end.
 * x_new, y: [S, n_new, d] fp32 (final RMSNorm applied when final_g != NULL).
 * The call enqueues only kernels (no host sync), so it can be captured in a
 * CUDA graph and replayed.  Workspace: vx_stream_step_workspace(). */
VX_API vx_status vx_stream_step(const vx_layer_cfg *cfg, const vx_layer_weights *layers,
                         const vx_kv_ring *ring, const float *x_new, float *y, int n_new,
                         const void *final_g, void *ws, size_t ws_bytes, cudaStream_t stream);
VX_API size_t vx_stream_step_workspace(const vx_layer_cfg *cfg, int S, int n_new);

/* Test hook for the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing arrives on, with a limit of timeout_ns, then records
 * VX_ERR_DEVICE_TIMEOUT in ws and returns.  Nothing faults or hangs. */
VX_API vx_status vx_selftest_wait_timeout(void *ws, size_t ws_bytes, uint64_t timeout_ns,
                                   cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VX_H_ */
