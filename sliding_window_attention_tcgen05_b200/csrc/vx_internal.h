// vx_internal.h -- host-side launchers shared between the libvx translation
// units.  Not part of the public ABI (include/vx.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string>
#include <utility>

#include "vx_common.cuh"

namespace vx {

// Error reporting (thread-local message, see vx_last_error()).
void set_error(const char* fmt, ...);
const char* last_error();

// Launch context of one public call.
struct Launch {
  cudaStream_t stream;
  DevStatus* status;   // status word inside the caller's workspace
  uint64_t limit_ns;   // bounded-wait limit
  int sm_count;        // SMs of the current device
};

int current_sm_count();
uint64_t wait_limit_ns();

// A kernel launched with more than 48 KB of dynamic shared memory needs
// cudaFuncAttributeMaxDynamicSharedMemorySize on every device that runs it:
// sets it once per (kernel, current device).  Thread-safe.
cudaError_t ensure_dynamic_smem(const void* kernel, size_t smem);

// Launches `k` on `stream` with programmatic dependent launch (the kernel may
// start while the previous kernel of the stream runs; see pdl_wait()).
template <class... KArgs, class... Args>
cudaError_t launch_kernel(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args&&... args) {
  if (smem > 48 * 1024) {
    if (cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(k), smem)) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// ------------------------------------------------------------- tracing --
// Every kernel launch goes through traced(): it counts the launches and,
// while tracing is enabled for the calling thread (vx_trace_enable), brackets
// them with CUDA events recorded on the launch stream (read by vx_trace_read).
void count_launches(int n);
bool trace_enabled();
cudaEvent_t trace_event();   // from a per-thread pool; null if none could be made
void trace_record(const char* name, cudaEvent_t a, cudaEvent_t b);

template <class F>
cudaError_t traced(const Launch& L, const char* name, int kernels, F&& f) {
  count_launches(kernels);
  if (!trace_enabled()) return f();
  cudaEvent_t a = trace_event(), b = trace_event();
  if (a) cudaEventRecord(a, L.stream);
  const cudaError_t e = f();
  if (b) cudaEventRecord(b, L.stream);
  if (a && b) trace_record(name, a, b);
  return e;
}

// Trace name of an RMSNorm / partial-sum reduction launch (static string).
constexpr int kMaxSplitsTraced = 8;
const char* rms_trace_name(int nparts, bool h_out, int y_kind /* 0 none, 1 bf16, 2 fp32 */);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);

// 2-D bf16 K-major operand view with a 64-element (128-byte) inner box and a
// 128-byte swizzle: `rows` rows of `cols` elements, `row_stride` elements apart.
bool tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                  uint64_t row_stride, uint32_t box_rows);

// ------------------------------------------------------------------ GEMM --
enum EpiKind : int {
  EPI_F32 = 0,        // out fp32 = acc + bias + residual
  EPI_QKV_ROPE = 1,   // out bf16 = RoPE(acc + bias) on the first rope_cols columns
  EPI_SWIGLU = 2,     // out bf16 [.., N/2] = silu(gate + bg) * (up + bu), 64-blocks interleaved
  EPI_GELU_BF16 = 3,  // out bf16 = GELU(acc + bias)
  EPI_GELU_F32 = 4,   // out fp32 = GELU(acc + bias)
};

constexpr int kOrderMFastest = 0, kOrderNFastest = 1, kOrderGrouped = 2;
constexpr int kOrderGroupRows = 4;

struct GemmArgs {
  int M, N, K;
  // Split-K: the K loop is cut into k_splits equal parts; part ks writes its
  // fp32 partial sums (EPI_F32, no bias / residual) at out + ks * split_stride.
  int k_splits;
  int64_t split_stride;
  // A addressing of K-block kb (64 wide): tap = kb / kb_per_tap,
  // c = (kb % kb_per_tap) * 64, x = (tap % a_stride) * a_tap_ch + c, y = m0 + tap / a_stride.
  int kb_per_tap, a_stride, a_tap_ch;
  void* out;
  int64_t ld_out;          // elements
  const uint16_t* bias;    // [N] bf16 or null
  const float* res;        // [.., ld_res] fp32 or null (EPI_F32 only)
  int64_t ld_res;
  // Row mapping: source row m -> (b, t) = (m / in_rows, m % in_rows); rows with
  // t >= t_valid (or m >= M) are not stored; destination row b * out_rows + out_off + t.
  int in_rows, t_valid, out_rows, out_off;
  // RoPE (EPI_QKV_ROPE): position of (b, t) = (pos_arr ? pos_arr[b] : pos0) + t.
  const int64_t* pos_arr;
  int64_t pos0;
  int rope_cols;           // columns [0, rope_cols) are rotated in 64-wide heads
  float inv_freq_hi[32];   // inv_freq_m as float, and its residual to the exact value
  float inv_freq_lo[32];
  // Output through TMA tile stores (identity row mapping, EPI_F32 / QKV / SwiGLU):
  // tmD is then a 3-D map {columns, M, splits} with a 64-byte swizzled box of
  // 64 bytes x 32 rows.
  int tma_store;
  // Work-unit order (kOrder*), set by launch_gemm: M-fastest (consecutive
  // units share a weight panel of B through L2), N-fastest (the units of one
  // row panel of A run together, so A crosses DRAM once) or groups of
  // kOrderGroupRows row panels, M-fastest inside a group.
  int order;
  // Pair kernel, EPI_F32 without K splits, N == 1280: when norm_g is set, the
  // epilogue warps also normalise the output once it is stored: out row r ->
  // norm_y row r = out_r / rms(out_r) * norm_g (RMSNorm, eps norm_eps; bf16
  // when norm_y_bf16, else fp32; norm_y may be out itself).  norm_ctr: one int
  // per 32 rows (stores of that row group done: 2 per column tile), a work
  // counter and a finished-CTA counter, all zero at launch; the kernel's last
  // CTA sets them back to zero.
  const uint16_t* norm_g;
  void* norm_y;
  int norm_y_bf16;
  float norm_eps;
  int* norm_ctr;
  DevStatus* status;
  uint64_t limit_ns;
};

// Tile shape of one GEMM launch: one CTA per 128 x bn tile, or a cluster of
// two CTAs per 256 x bn tile (pair); `splits` K-splits writing fp32 partials.
struct GemmPlan {
  bool pair;
  int bn;       // 64, 128 or 256 (pair: 128 or 256); 0 = no shape fits
  int splits;
};

// The fastest shape for an M x N x K GEMM with epilogue `epi` on `sm` SMs by
// the launch-time model in gemm.cu (split-K only for EPI_F32, up to max_splits).
GemmPlan plan_gemm(int M, int N, int K, int epi, int max_splits, int sm);

// D[M, N] = A[M, K] * B[N, K]^T with the given epilogue, in the shape `plan`.
// tmA: 2-D bf16 map with 128-byte swizzle and box {64, 128}; tmB: the same
// with box {64, plan.pair ? plan.bn / 2 : plan.bn}.  args.k_splits must equal
// plan.splits; N % bn == 0; K % 64 == 0; (K / 64) % splits == 0.  tmD: the
// output map when args.tma_store (see GemmArgs), else unused.
cudaError_t launch_gemm(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                        const GemmArgs& args, int epi, const GemmPlan& plan);

void fill_rope_freqs(GemmArgs* a, float theta, int head_dim);

// ------------------------------------------------------------- attention --
struct AttnArgs {
  void* out;                   // bf16 [B, T, H, 64] with the strides below
  int64_t o_row, o_head, o_batch;  // element strides of t, h, b in out
  int B, T, H, window;
  float scale_log2;            // softmax scale * log2(e)
  DevStatus* status;
  uint64_t limit_ns;
};
// Keys per tile of the bf16 attention kernel.
constexpr int kAttnKeyTile = 64;
// q, k, v: bf16 [B, T, H, 64] with element strides row_stride (t) and
// batch_stride (b) (heads contiguous in 64s); read through 4-D TMA maps.
struct AttnOperands {
  const void* q;
  const void* k;
  const void* v;
  int64_t row_stride, batch_stride;
};
cudaError_t launch_attn_bf16(const Launch& L, const AttnOperands& op, const AttnArgs& a);

// fp32 CUDA-core sliding-window attention on pre-rotated q, k: [B, T, H, 64].
cudaError_t launch_attn_f32(const Launch& L, const float* q, const float* k, const float* v,
                            float* o, int B, int T, int H, int window, float scale);

// RoPE of q and k ([B, T, H, 64], fp32 or bf16) into qr and kr (same layout
// and dtype), one kernel.
cudaError_t launch_rope(const Launch& L, const void* q, const void* k, void* qr, void* kr, bool bf16, int B, int T,
                        int H, int64_t pos0, float theta);

// ---------------------------------------------------------------- others --
// h = x + bias + sum_{k < nparts} parts[k * part_stride + .]  (parts/bias optional);
// h_out (optional) = h; y (optional, with g) = h * rsqrt(mean(h^2) + eps) * g.
cudaError_t launch_rmsnorm(const Launch& L, const float* x, const float* parts, int nparts, int64_t part_stride,
                           const uint16_t* bias, const uint16_t* g, float* h_out, void* y, bool y_bf16, int M,
                           int d, float eps);

// Ring attention of one layer of a streaming step (see vx_stream_step).
cudaError_t launch_ring_attn(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD,
                             uint16_t* ring_k, uint16_t* ring_v, const int64_t* pos, int S,
                             int H, int W, int n_new, uint16_t* out, float scale_log2);
// Writes the K/V of frames max(0,T-W)..T-1 of qkv ([S*T, ld]) into one layer's ring.
cudaError_t launch_ring_fill(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD,
                             uint16_t* ring_k, uint16_t* ring_v, int S, int T, int H, int W);
cudaError_t launch_pos_add(const Launch& L, int64_t* pos, int S, int64_t n, bool set);
// p[0 .. n) = 0.
cudaError_t launch_zero_ints(const Launch& L, int* p, int n);

cudaError_t launch_pack_layer(const Launch& L, int d, int HD, int F, const uint16_t* wq,
                              const uint16_t* wk, const uint16_t* wv, const uint16_t* bq,
                              const uint16_t* bv, const uint16_t* wg, const uint16_t* wu,
                              const uint16_t* bg, const uint16_t* bu, uint16_t* wqkv,
                              uint16_t* bqkv, uint16_t* wgu, uint16_t* bgu);
cudaError_t launch_pack_conv(const Launch& L, const uint16_t* w, uint16_t* wp, int O, int C);
// mel [B, C, Tm] fp32 -> xpad [B, P, C] bf16 (rows 0,1 and >= Tm+2 zero); also
// zeroes rows 0, 1 and Tm+2 .. P-1 of h1pad [B, P, d].
cudaError_t launch_conv_prep(const Launch& L, const float* mel, uint16_t* xpad, uint16_t* h1pad,
                             int B, int C, int Tm, int P, int d, const uint16_t* cache_x = nullptr,
                             const uint16_t* cache_h1 = nullptr);
// (with cache_x [B, 2, C] / cache_h1 [B, 2, d]: rows 0, 1 come from the caches instead of zeros)
// Saves the last two rows of each clip of xpad / h1pad into the caches.
cudaError_t launch_conv_cache_save(const Launch& L, const uint16_t* xpad, const uint16_t* h1pad, uint16_t* cache_x,
                                   uint16_t* cache_h1, int B, int P, int C, int d);
// x [B, T, d] fp32 -> tok [B * (T/4), 4 d] bf16 (frames 4j..4j+3 of a clip form token j).
cudaError_t launch_frames_to_tokens(const Launch& L, const float* x, uint16_t* tok, int B, int T, int d);

// Log-mel frontend (16 kHz, n_fft 400, hop 160, 128 slaney bands, fixed max 1.5):
// audio [B, N] fp32 -> mel [B, 128, log_mel_frames(N, center)] fp32; tables:
// log_mel_table_bytes() of scratch (filterbank, window, twiddles).
int log_mel_frames(int N, int center);
size_t log_mel_table_bytes();
cudaError_t launch_log_mel(const Launch& L, const float* audio, float* mel, int B, int N, int center, void* tables);

cudaError_t launch_selftest_wait(const Launch& L);

}  // namespace vx
