// api.cu -- the C ABI of libvx (include/vx.h): argument validation, workspace
// carving, tensor-map encoding and the kernel sequences of each operation.
//
// Encoder layer (transcribe.cpp notes "Voxtral", Voxtral Realtime 2602
// architecture), as enqueued by run_layer():
//   1. RMSNorm(x)                 -> y0   (bf16)
//   2. y0 Wqkv^T + bqkv, RoPE     -> qkv  (bf16, [M, 3*HD], tcgen05 GEMM)
//   3. sliding-window attention   -> att  (bf16, tcgen05 flash kernel, or the
//                                          ring kernel in a streaming step)
//   4. att Wo^T + bo + x          -> h    (fp32, residual fused in the epilogue,
//                                          or split-K partials reduced in 5.)
//   5. RMSNorm(h)                 -> y1   (bf16)
//   6. silu(y1 Wg^T) * (y1 Wu^T)  -> act  (bf16, gate/up packed, SwiGLU epilogue)
//   7. act Wd^T + bd + h          -> y    (fp32; fused, or partials reduced by
//                                          the next layer's RMSNorm 1.)
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <cmath>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include <cudaTypedefs.h>

#include "vx.h"
#include "vx_internal.h"

namespace vx {

// ------------------------------------------------------------ utilities --
static thread_local char g_err[1024] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}
const char* last_error() { return g_err; }

static std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

cudaError_t ensure_dynamic_smem(const void* kernel, size_t smem) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;   // (kernel, device) -> bytes set
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({kernel, dev});
  if (it != done.end() && it->second >= smem) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) done[{kernel, dev}] = smem;
  return e;
}

// ------------------------------------------------------------- tracing --
static std::atomic<uint64_t> g_launches{0};
struct TraceRec {
  const char* name;
  cudaEvent_t a, b;
};
static thread_local bool t_trace = false;
static thread_local std::vector<TraceRec> t_recs;
static thread_local std::vector<cudaEvent_t> t_pool;
static thread_local size_t t_pool_used = 0;

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }
bool trace_enabled() { return t_trace; }

cudaEvent_t trace_event() {
  if (t_pool_used == t_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    t_pool.push_back(e);
  }
  return t_pool[t_pool_used++];
}

void trace_record(const char* name, cudaEvent_t a, cudaEvent_t b) { t_recs.push_back({name, a, b}); }

const char* rms_trace_name(int nparts, bool h_out, int y_kind) {
  // "rmsnorm_p<n>[_h][_y16|_y32]": the partial sums it reduces, whether it
  // writes h, and the normalised output's type (none when it only reduces).
  static const std::vector<std::string> names = [] {
    std::vector<std::string> v;
    for (int n = 0; n <= kMaxSplitsTraced; ++n)
      for (int h = 0; h < 2; ++h)
        for (int y = 0; y < 3; ++y)
          v.push_back("rmsnorm_p" + std::to_string(n) + (h ? "_h" : "") + (y == 1 ? "_y16" : y == 2 ? "_y32" : ""));
    return v;
  }();
  if (nparts < 0 || nparts > kMaxSplitsTraced || y_kind < 0 || y_kind > 2) return "rmsnorm";
  return names[(nparts * 2 + (h_out ? 1 : 0)) * 3 + y_kind].c_str();
}

int current_sm_count() {
  static std::atomic<int> cache[64];   // per device; 0 = not looked up yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled is not available from the CUDA driver");
    return false;
  }
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; bx[i] = box[i]; es[i] = 1; }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  const CUresult r = fn(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (CUresult %d, rank %d)", static_cast<int>(r), rank);
    return false;
  }
  return true;
}

bool tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride,
                  uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {row_stride * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace vx

using namespace vx;

namespace {

constexpr size_t kStatusBytes = 256;
constexpr size_t kAlign = 1024;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Bump allocator over the caller's workspace (or a size counter when base is null).
struct Carve {
  uint8_t* base;
  size_t off;
  void* take(size_t bytes) {
    off = align_up(off, kAlign);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

#define VX_CHECK_ARG(cond, ...)   \
  do {                            \
    if (!(cond)) {                \
      set_error(__VA_ARGS__);     \
      return VX_ERR_INVALID_ARG;  \
    }                             \
  } while (0)

#define VX_CUDA(call)                                                          \
  do {                                                                         \
    cudaError_t e_ = (call);                                                   \
    if (e_ != cudaSuccess) {                                                   \
      set_error("%s failed: %s", #call, cudaGetErrorString(e_));               \
      return VX_ERR_CUDA;                                                      \
    }                                                                          \
  } while (0)

vx_status make_launch(Launch* L, void* ws, size_t ws_bytes, size_t need, cudaStream_t stream) {
  VX_CHECK_ARG(ws != nullptr, "workspace is null");
  VX_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255) == 0, "workspace must be 256-byte aligned");
  VX_CHECK_ARG(ws_bytes >= need, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  L->stream = stream;
  L->status = static_cast<DevStatus*>(ws);
  L->limit_ns = wait_limit_ns();
  L->sm_count = current_sm_count();
  if (L->sm_count <= 0) {
    set_error("no CUDA device is current");
    return VX_ERR_CUDA;
  }
  return VX_OK;
}

// A traced RMSNorm / partial-sum reduction launch (see launch_rmsnorm).
cudaError_t rmsnorm(const Launch& L, const float* x, const float* parts, int nparts, int64_t part_stride,
                    const uint16_t* bias, const uint16_t* g, float* h_out, void* y, bool y_bf16, int M, int d,
                    float eps) {
  const int yk = (g && y) ? (y_bf16 ? 1 : 2) : 0;
  return traced(L, rms_trace_name(nparts, h_out != nullptr, yk), 1, [&] {
    return launch_rmsnorm(L, x, parts, nparts, part_stride, bias, g, h_out, y, y_bf16, M, d, eps);
  });
}

vx_status check_cfg(const vx_layer_cfg* c) {
  VX_CHECK_ARG(c != nullptr, "cfg is null");
  if (c->head_dim != 64) {
    set_error("head_dim %d unsupported (64 only)", c->head_dim);
    return VX_ERR_UNSUPPORTED;
  }
  const int HD = c->n_heads * c->head_dim;
  VX_CHECK_ARG(c->n_heads > 0 && c->d_model > 0 && c->ffn_hidden > 0 && c->window >= 1, "bad layer cfg");
  if (c->d_model % 128 != 0 || c->d_model > 2048 || HD % 128 != 0 || c->ffn_hidden % 64 != 0) {
    set_error("unsupported layer shape d=%d HD=%d F=%d (need d%%128==0, d<=2048, HD%%128==0, F%%64==0)",
              c->d_model, HD, c->ffn_hidden);
    return VX_ERR_UNSUPPORTED;
  }
  VX_CHECK_ARG(c->eps > 0.f && c->rope_theta > 0.f, "eps and rope_theta must be positive");
  return VX_OK;
}

vx_status check_weights(const vx_layer_cfg& c, const vx_layer_weights* w) {
  VX_CHECK_ARG(w != nullptr, "layer weights are null");
  const void* ptrs[] = {w->attn_norm_g, w->wqkv, w->bqkv, w->wo, w->bo, w->ffn_norm_g, w->wgu, w->bgu, w->wd, w->bd};
  for (const void* p : ptrs) {
    VX_CHECK_ARG(p != nullptr, "a layer weight pointer is null");
    VX_CHECK_ARG(aligned16(p), "layer weight pointers must be 16-byte aligned");
  }
  (void)c;
  return VX_OK;
}

struct LayerBufs {
  uint16_t* y0;    // [M, d]     bf16 normed input (reused for the second norm)
  uint16_t* qkv;   // [M, 3*HD]  bf16
  uint16_t* att;   // [M, HD]    bf16
  float* h;        // [M, d]     fp32 post-attention residual stream
  uint16_t* act;   // [M, F]     bf16 SwiGLU output
  float* xmat;     // [M, d]     fp32 materialised layer input (when it arrives as partial sums)
  float* parts;    // [split_cap(M), M, d] fp32 split-K partial sums (null when split_cap(M) == 1)
  int* norm_ctr;   // [M/32 + 2] counters of an RMSNorm run in a residual GEMM's tail (or null)
};

// Most K-splits a GEMM with M rows may use: few-row GEMMs have too few output
// tiles to fill the GPU; from a few thousand rows on they never need one.
constexpr int kMaxSplits = 8;
int split_cap(int64_t M) { return M <= 512 ? kMaxSplits : (M <= 4096 ? 2 : 1); }

LayerBufs carve_layer(Carve& cv, const vx_layer_cfg& c, int64_t M) {
  const int64_t d = c.d_model, HD = int64_t(c.n_heads) * c.head_dim, F = c.ffn_hidden;
  LayerBufs b;
  b.y0 = static_cast<uint16_t*>(cv.take(M * d * 2));
  b.qkv = static_cast<uint16_t*>(cv.take(M * 3 * HD * 2));
  b.att = static_cast<uint16_t*>(cv.take(M * HD * 2));
  b.h = static_cast<float*>(cv.take(M * d * 4));
  b.act = static_cast<uint16_t*>(cv.take(M * F * 2));
  const int cap = split_cap(M);
  b.xmat = cap > 1 ? static_cast<float*>(cv.take(M * d * 4)) : nullptr;
  b.parts = cap > 1 ? static_cast<float*>(cv.take(cap * M * d * 4)) : nullptr;
  b.norm_ctr = (cap == 1 && d == 1280) ? static_cast<int*>(cv.take(((M + 31) / 32 + 2) * 4)) : nullptr;
  return b;
}

// The tail-norm counters start at zero (each kernel that uses them leaves them
// at zero again).
vx_status init_norm_ctr(const Launch& L, const LayerBufs& b, int64_t M) {
  if (b.norm_ctr) VX_CUDA(traced(L, "zero_ctr", 1, [&] {
    return launch_zero_ints(L, b.norm_ctr, static_cast<int>((M + 31) / 32 + 2));
  }));
  return VX_OK;
}

size_t layer_ws_bytes(const vx_layer_cfg& c, int64_t M) {
  Carve cv{nullptr, kStatusBytes};
  carve_layer(cv, c, M);
  return align_up(cv.off, kAlign);
}

GemmArgs base_args(const Launch& L, int M, int N, int K) {
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = M; a.N = N; a.K = K;
  a.k_splits = 1;
  a.kb_per_tap = K / 64; a.a_stride = 1; a.a_tap_ch = K;
  a.in_rows = M; a.t_valid = M; a.out_rows = M; a.out_off = 0;
  a.status = L.status;
  a.limit_ns = L.limit_ns;
  return a;
}

// Encodes B's tensor map for and launches one GEMM in the shape `p`
// (a.k_splits must already equal p.splits).
// Tensor map for TMA stores of a GEMM's output ({columns, M, splits}, a
// 64-byte x 32-row box with the 64-byte swizzle of the epilogue's staging
// buffer), or false when the output does not map rows 1:1 or is misaligned.
bool tmap_gemm_out(CUtensorMap* m, const GemmArgs& a, int epi) {
  const bool identity = a.out_rows == a.in_rows && a.out_off == 0 && a.t_valid == a.in_rows;
  if (!identity || !aligned16(a.out)) return false;
  if (epi == EPI_F32) {
    const int64_t zs = a.k_splits > 1 ? a.split_stride : a.ld_out * a.M;
    if ((a.ld_out * 4) % 16 != 0 || (zs * 4) % 16 != 0) return false;
    const uint64_t dims[3] = {static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M),
                              static_cast<uint64_t>(a.k_splits)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.ld_out) * 4, static_cast<uint64_t>(zs) * 4};
    const uint32_t box[3] = {16, 32, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (epi == EPI_QKV_ROPE || epi == EPI_SWIGLU) {
    if ((a.ld_out * 2) % 16 != 0) return false;
    const uint64_t cols = epi == EPI_SWIGLU ? a.N / 2 : a.N;
    const uint64_t dims[3] = {cols, static_cast<uint64_t>(a.M), 1};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.ld_out) * 2, static_cast<uint64_t>(a.ld_out) * 2 * a.M};
    const uint32_t box[3] = {32, 32, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  return false;
}

vx_status launch_planned(const Launch& L, const char* name, const CUtensorMap* tmA, const void* Bw, int64_t ldb,
                         const GemmArgs& a_in, int epi, const GemmPlan& p) {
  if (p.bn == 0) {
    set_error("%s: no GEMM tile shape fits N=%d K=%d", name, a_in.N, a_in.K);
    return VX_ERR_UNSUPPORTED;
  }
  CUtensorMap tmB, tmD;
  if (!tmap_bf16_2d(&tmB, Bw, a_in.K, a_in.N, ldb, p.pair ? p.bn / 2 : p.bn)) return VX_ERR_CUDA;
  GemmArgs a = a_in;
  std::memset(&tmD, 0, sizeof(tmD));
  a.tma_store = tmap_gemm_out(&tmD, a, epi) ? 1 : 0;
  VX_CUDA(traced(L, name, 1, [&] { return launch_gemm(L, *tmA, tmB, tmD, a, epi, p); }));
  return VX_OK;
}

// One GEMM without K-splits: plan, then launch.
vx_status launch_any_gemm(const Launch& L, const char* name, const CUtensorMap* tmA, const void* Bw, int64_t ldb,
                          const GemmArgs& a, int epi) {
  return launch_planned(L, name, tmA, Bw, ldb, a, epi, plan_gemm(a.M, a.N, a.K, epi, 1, L.sm_count));
}

vx_status gemm(const Launch& L, const char* name, const void* A, int64_t lda, const void* Bw, const GemmArgs& a,
               int epi, const GemmPlan* p = nullptr) {
  CUtensorMap tmA;
  if (!tmap_bf16_2d(&tmA, A, a.K, a.M, lda, 128)) return VX_ERR_CUDA;
  if (p) return launch_planned(L, name, &tmA, Bw, a.K, a, epi, *p);
  return launch_any_gemm(L, name, &tmA, Bw, a.K, a, epi);
}

// The pending (unreduced) value of an fp32 [M, d] activation:
// base + bias + sum_{k < nparts} parts[k].
struct Pending {
  const float* base;
  const float* parts;
  int nparts;
  const uint16_t* bias;
  bool normed;   // its consumer's RMSNorm has been written already (by the producing GEMM)
};

// An RMSNorm of a residual GEMM's output, run in that GEMM's tail: gain g,
// output y (bf16 or fp32; may be the GEMM's own output).
struct NormFuse {
  const uint16_t* g;
  void* y;
  bool y_bf16;
};

// A residual GEMM  out = A W^T + bias + res  in the planned shape: fused into
// the epilogue when the plan has one K-split, else as fp32 partial sums whose
// reduction (with bias and residual) is left pending for the next RMSNorm.
// With one K-split, a CTA-pair plan, d = 1280 and tail counters, the RMSNorm
// nf of the output runs in the GEMM's tail (result->normed).
vx_status residual_gemm(const Launch& L, const char* name, const void* A, int64_t lda, const void* W, int M, int N,
                        int K, const uint16_t* bias, const float* res, float* out, float* parts, int max_splits,
                        Pending* result, const NormFuse* nf = nullptr, int* norm_ctr = nullptr, float eps = 0.f) {
  GemmArgs a = base_args(L, M, N, K);
  const GemmPlan p = plan_gemm(M, N, K, EPI_F32, parts ? max_splits : 1, L.sm_count);
  a.ld_out = N;
  if (p.splits > 1) {
    a.out = parts;
    a.k_splits = p.splits;
    a.split_stride = static_cast<int64_t>(M) * N;
    *result = Pending{res, parts, p.splits, bias};
  } else {
    a.out = out;
    a.bias = bias;
    a.res = res; a.ld_res = N;
    *result = Pending{out, nullptr, 0, nullptr};
    if (nf && norm_ctr && p.pair && N == 1280) {
      a.norm_g = nf->g;
      a.norm_y = nf->y;
      a.norm_y_bf16 = nf->y_bf16 ? 1 : 0;
      a.norm_eps = eps;
      a.norm_ctr = norm_ctr;
      result->normed = true;
    }
  }
  return gemm(L, name, A, lda, W, a, EPI_F32, &p);
}


struct RingLayer {
  uint16_t* k;
  uint16_t* v;
  const int64_t* pos;
  int W;
  bool fill;   // whole-sequence prefill: write the last W frames' K/V
  bool step;   // streaming step: attend through the ring
};

// One layer over nseq sequences of `rows` frames.  The input arrives pending
// (the previous layer's output may still be split-K partial sums); so may the
// output: `out` is either y itself or the pending sum that the next RMSNorm
// (the next layer's, the final norm, or a plain reduction) completes.  With
// split-K the layer still runs seven kernels: each RMSNorm also reduces.
//   x_l = reduce(in);  y0 = RMSNorm(x_l)
//   qkv = RoPE(y0 Wqkv^T + bqkv);  att = attention(qkv)
//   h   = x_l + bo + att Wo^T         (fused, or pending into RMSNorm 2)
//   y1  = RMSNorm(h);  act = SwiGLU(y1 Wgu^T + bgu)
//   out = h + bd + act Wd^T           (fused into y, or pending)
vx_status run_layer(const Launch& L, const vx_layer_cfg& c, const vx_layer_weights& w, const Pending& in,
                    Pending* out, float* y, int nseq, int rows, int64_t pos0, const LayerBufs& bf,
                    const RingLayer* ring, const NormFuse* next_norm = nullptr) {
  const int d = c.d_model, H = c.n_heads, HD = H * c.head_dim, F = c.ffn_hidden;
  const int M = nseq * rows;
  const int64_t pstride = static_cast<int64_t>(M) * d;
  const int cap = bf.parts ? split_cap(M) : 1;
  const float sl2 = (1.0f / std::sqrt(static_cast<float>(c.head_dim))) * 1.4426950408889634f;
  const bool step = ring && ring->step;
  vx_status st;
  // 1. x_l = reduce(in); y0 = RMSNorm(x_l) (unless the previous GEMM wrote it)
  const bool pending_in = in.parts != nullptr || in.bias != nullptr;
  const float* xl = pending_in ? bf.xmat : in.base;
  if (!in.normed)
    VX_CUDA(rmsnorm(L, in.base, in.parts, in.nparts, pstride, in.bias, static_cast<const uint16_t*>(w.attn_norm_g),
                    pending_in ? bf.xmat : nullptr, bf.y0, true, M, d, c.eps));
  // 2. QKV + bias + RoPE at (pos[s] or pos0) + t
  {
    GemmArgs a = base_args(L, M, 3 * HD, d);
    a.out = bf.qkv; a.ld_out = 3 * HD;
    a.bias = static_cast<const uint16_t*>(w.bqkv);
    a.in_rows = rows; a.t_valid = rows; a.out_rows = rows;
    a.pos_arr = step ? ring->pos : nullptr;
    a.pos0 = pos0;
    a.rope_cols = 2 * HD;
    fill_rope_freqs(&a, c.rope_theta, c.head_dim);
    if ((st = gemm(L, "gemm_qkv_rope", bf.y0, d, w.wqkv, a, EPI_QKV_ROPE)) != VX_OK) return st;
  }
  // 3. attention: through the ring (streaming step), or windowed over the sequence
  if (step) {
    VX_CUDA(traced(L, "ring_attn", 1, [&] {
      return launch_ring_attn(L, bf.qkv, 3LL * HD, HD, ring->k, ring->v, ring->pos, nseq, H, ring->W, rows, bf.att,
                              sl2);
    }));
  } else {
    const AttnOperands op{bf.qkv, bf.qkv + HD, bf.qkv + 2 * HD, 3LL * HD, static_cast<int64_t>(rows) * 3 * HD};
    AttnArgs aa;
    aa.out = bf.att; aa.o_row = HD; aa.o_head = 64; aa.o_batch = static_cast<int64_t>(rows) * HD;
    aa.B = nseq; aa.T = rows; aa.H = H; aa.window = c.window; aa.scale_log2 = sl2;
    aa.status = L.status; aa.limit_ns = L.limit_ns;
    VX_CUDA(traced(L, "swa_attn_tc", 1, [&] { return launch_attn_bf16(L, op, aa); }));
    if (ring && ring->fill)
      VX_CUDA(traced(L, "ring_fill", 1, [&] {
        return launch_ring_fill(L, bf.qkv, 3LL * HD, HD, ring->k, ring->v, nseq, rows, H, ring->W);
      }));
  }
  // 4. h = x_l + bo + att Wo^T (with 5. in its tail when it can)
  Pending hp;
  const NormFuse norm2{static_cast<const uint16_t*>(w.ffn_norm_g), bf.y0, true};
  if ((st = residual_gemm(L, "gemm_o_residual", bf.att, HD, w.wo, M, d, HD, static_cast<const uint16_t*>(w.bo), xl,
                          bf.h, bf.parts, cap, &hp, &norm2, bf.norm_ctr, c.eps)) != VX_OK)
    return st;
  // 5. y1 = RMSNorm(h), materialising h when it is pending
  const bool pending_h = hp.parts != nullptr;
  if (!hp.normed)
    VX_CUDA(rmsnorm(L, hp.base, hp.parts, hp.nparts, pstride, hp.bias, static_cast<const uint16_t*>(w.ffn_norm_g),
                    pending_h ? bf.h : nullptr, bf.y0, true, M, d, c.eps));
  // 6. gate/up + SwiGLU
  {
    GemmArgs a = base_args(L, M, 2 * F, d);
    a.out = bf.act; a.ld_out = F;
    a.bias = static_cast<const uint16_t*>(w.bgu);
    if ((st = gemm(L, "gemm_gate_up_swiglu", bf.y0, d, w.wgu, a, EPI_SWIGLU)) != VX_OK) return st;
  }
  // 7. out = h + bd + act Wd^T (with the next RMSNorm in its tail when the caller names one and it can)
  return residual_gemm(L, "gemm_down_residual", bf.act, F, w.wd, M, d, F, static_cast<const uint16_t*>(w.bd), bf.h, y,
                       bf.parts, cap, out, next_norm, bf.norm_ctr, c.eps);
}

// y = reduce(p) unless p already is y.
cudaError_t reduce_into(const Launch& L, const Pending& p, float* y, int M, int d) {
  if (p.base == y && p.parts == nullptr && p.bias == nullptr) return cudaSuccess;
  return rmsnorm(L, p.base, p.parts, p.nparts, static_cast<int64_t>(M) * d, p.bias, nullptr, y, nullptr, false,
                        M, d, 1.0f);
}

// ------------------------------------------------------------- conv stem --
int conv_rows_per_clip(int Tm) { return ((Tm + 2) + 1) / 2 * 2; }   // Tm + 2 rounded up to even

struct ConvBufs {
  uint16_t* xpad;    // [B, P, C]
  uint16_t* h1pad;   // [B, P, d]
};

ConvBufs carve_conv(Carve& cv, int B, int C, int Tm, int d) {
  const int64_t P = conv_rows_per_clip(Tm);
  ConvBufs b;
  b.xpad = static_cast<uint16_t*>(cv.take(int64_t(B) * P * C * 2));
  b.h1pad = static_cast<uint16_t*>(cv.take(int64_t(B) * P * d * 2));
  return b;
}

// cache_x / cache_h1 (both or neither): the conv padding cache of a streaming
// chunk (see vx_conv_stem_step); rows 0, 1 of xpad / h1pad come from it and
// are replaced by the chunk's last two rows afterwards.
vx_status run_conv_stem(const Launch& L, const float* mel, const void* w1p, const void* b1, const void* w2p,
                        const void* b2, float* out, int B, int C, int Tm, int d, const ConvBufs& cb,
                        uint16_t* cache_x = nullptr, uint16_t* cache_h1 = nullptr) {
  const int P = conv_rows_per_clip(Tm);
  const int To = (Tm - 1) / 2 + 1;
  VX_CUDA(traced(L, "conv_prep", 2, [&] {
    return launch_conv_prep(L, mel, cb.xpad, cb.h1pad, B, C, Tm, P, d, cache_x, cache_h1);
  }));
  vx_status st;
  // conv1: rows r = b*P + t of xpad; taps read rows r, r+1, r+2 -> h1pad row b*P + 2 + t.
  {
    GemmArgs a = base_args(L, B * P, d, 3 * C);
    a.kb_per_tap = C / 64; a.a_stride = 1; a.a_tap_ch = C;
    a.out = cb.h1pad; a.ld_out = d;
    a.bias = static_cast<const uint16_t*>(b1);
    a.in_rows = P; a.t_valid = Tm; a.out_rows = P; a.out_off = 2;
    CUtensorMap tmA;
    if (!tmap_bf16_2d(&tmA, cb.xpad, C, int64_t(B) * P, C, 128)) return VX_ERR_CUDA;
    if ((st = launch_any_gemm(L, "gemm_conv1_gelu", &tmA, w1p, 3 * C, a, EPI_GELU_BF16)) != VX_OK) return st;
  }
  // conv2 (stride 2): h1pad viewed as [B*P/2, 2d]; output t of clip b reads
  // padded rows 2t, 2t+1, 2t+2 = (pair t, half 0), (pair t, half 1), (pair t+1, half 0).
  {
    const int pairs = P / 2;
    GemmArgs a = base_args(L, B * pairs, d, 3 * d);
    a.kb_per_tap = d / 64; a.a_stride = 2; a.a_tap_ch = d;
    a.out = out; a.ld_out = d;
    a.bias = static_cast<const uint16_t*>(b2);
    a.in_rows = pairs; a.t_valid = To; a.out_rows = To; a.out_off = 0;
    CUtensorMap tmA;
    if (!tmap_bf16_2d(&tmA, cb.h1pad, 2LL * d, int64_t(B) * pairs, 2LL * d, 128)) return VX_ERR_CUDA;
    if ((st = launch_any_gemm(L, "gemm_conv2_gelu", &tmA, w2p, 3 * d, a, EPI_GELU_F32)) != VX_OK) return st;
  }
  if (cache_x)
    VX_CUDA(traced(L, "conv_cache_save", 1, [&] {
      return launch_conv_cache_save(L, cb.xpad, cb.h1pad, cache_x, cache_h1, B, P, C, d);
    }));
  return VX_OK;
}

vx_status check_ring(const vx_layer_cfg& c, const vx_kv_ring* r, int n_layers_needed) {
  VX_CHECK_ARG(r != nullptr && r->k && r->v && r->pos, "ring or its k/v/pos pointers are null");
  VX_CHECK_ARG(aligned16(r->k) && aligned16(r->v) && (reinterpret_cast<uintptr_t>(r->pos) & 7) == 0,
               "ring k/v must be 16-byte aligned and pos 8-byte aligned");
  VX_CHECK_ARG(r->n_layers >= n_layers_needed && r->n_layers >= 1 && r->n_streams >= 1, "bad ring shape");
  VX_CHECK_ARG(r->window == c.window, "ring window (%d) must equal the layer window (%d)", r->window, c.window);
  return VX_OK;
}

}  // namespace

// ====================================================================== ABI

extern "C" {

const char* vx_last_error(void) { return vx::last_error(); }
const char* vx_version(void) { return "vx 0.1 (sm_100a)"; }
void vx_set_wait_timeout_ns(uint64_t ns) { g_wait_limit_ns.store(ns > 0 ? ns : 1); }

void vx_trace_enable(int on) { t_trace = on != 0; }

int vx_trace_read(char* buf, size_t cap) {
  std::string out;
  int n = 0;
  for (const TraceRec& r : t_recs) {
    float ms = -1.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess) cudaEventElapsedTime(&ms, r.a, r.b);
    char line[160];
    snprintf(line, sizeof(line), "%s %.6f\n", r.name, ms);
    out += line;
    ++n;
  }
  t_recs.clear();
  t_pool_used = 0;
  if (buf && cap > 0) {
    const size_t m = out.size() < cap - 1 ? out.size() : cap - 1;
    std::memcpy(buf, out.data(), m);
    buf[m] = '\0';
  }
  return n;
}

uint64_t vx_launch_count(void) { return g_launches.load(); }

vx_status vx_status_reset(void* ws, cudaStream_t stream) {
  VX_CHECK_ARG(ws != nullptr, "workspace is null");
  VX_CUDA(cudaMemsetAsync(ws, 0, kStatusBytes, stream));
  return VX_OK;
}

vx_status vx_status_check(const void* ws, cudaStream_t stream) {
  VX_CHECK_ARG(ws != nullptr, "workspace is null");
  DevStatus h;
  VX_CUDA(cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, stream));
  VX_CUDA(cudaStreamSynchronize(stream));
  if (h.code == kStatusTimeout) {
    set_error("a device-side wait expired (wait tag %d, block %u)", h.where, h.block);
    return VX_ERR_DEVICE_TIMEOUT;
  }
  return VX_OK;
}

vx_status vx_pack_layer(const vx_layer_cfg* cfg, const vx_layer_params* in, void* packed_wqkv, void* packed_bqkv,
                        void* packed_wgu, void* packed_bgu, cudaStream_t stream) {
  vx_status st = check_cfg(cfg);
  if (st != VX_OK) return st;
  VX_CHECK_ARG(in && in->wq && in->wk && in->wv && in->bq && in->bv && in->wg && in->wu, "null layer parameter");
  VX_CHECK_ARG(packed_wqkv && packed_bqkv && packed_wgu && packed_bgu, "null packed buffer");
  const void* al[] = {in->wq, in->wk, in->wv, in->wg, in->wu, packed_wqkv, packed_wgu};
  for (const void* p : al) VX_CHECK_ARG(aligned16(p), "weight buffers must be 16-byte aligned");
  Launch L{stream, nullptr, wait_limit_ns(), 1};
  const int HD = cfg->n_heads * cfg->head_dim;
  g_launches.fetch_add(4);
  VX_CUDA(launch_pack_layer(L, cfg->d_model, HD, cfg->ffn_hidden, static_cast<const uint16_t*>(in->wq),
                            static_cast<const uint16_t*>(in->wk), static_cast<const uint16_t*>(in->wv),
                            static_cast<const uint16_t*>(in->bq), static_cast<const uint16_t*>(in->bv),
                            static_cast<const uint16_t*>(in->wg), static_cast<const uint16_t*>(in->wu),
                            static_cast<const uint16_t*>(in->bg), static_cast<const uint16_t*>(in->bu),
                            static_cast<uint16_t*>(packed_wqkv), static_cast<uint16_t*>(packed_bqkv),
                            static_cast<uint16_t*>(packed_wgu), static_cast<uint16_t*>(packed_bgu)));
  return VX_OK;
}

vx_status vx_pack_conv_weight(const void* w, void* w_packed, int out_ch, int in_ch, cudaStream_t stream) {
  VX_CHECK_ARG(w && w_packed && out_ch > 0 && in_ch > 0, "bad conv weight arguments");
  Launch L{stream, nullptr, wait_limit_ns(), 1};
  g_launches.fetch_add(1);
  VX_CUDA(launch_pack_conv(L, static_cast<const uint16_t*>(w), static_cast<uint16_t*>(w_packed), out_ch, in_ch));
  return VX_OK;
}

size_t vx_swa_attn_workspace(vx_dtype dt, int B, int T, int H, int D, int apply_rope) {
  if (B <= 0 || T <= 0 || H <= 0 || D <= 0) return kStatusBytes;
  Carve cv{nullptr, kStatusBytes};
  if (apply_rope) {
    const size_t es = dt == VX_F32 ? 4 : 2;
    cv.take(size_t(B) * T * H * D * es);
    cv.take(size_t(B) * T * H * D * es);
  }
  return align_up(cv.off, kAlign);
}

vx_status vx_swa_attn_fwd(const void* q, const void* k, const void* v, void* o, vx_dtype dt, int B, int T, int H,
                          int D, int window, int apply_rope, float rope_theta, int64_t pos0, float scale, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  VX_CHECK_ARG(q && k && v && o, "q/k/v/o must not be null");
  VX_CHECK_ARG(B > 0 && T > 0 && H > 0 && window >= 1, "bad shape B=%d T=%d H=%d window=%d", B, T, H, window);
  VX_CHECK_ARG(dt == VX_F32 || dt == VX_BF16, "bad dtype");
  if (D != 64) {
    set_error("head_dim %d unsupported (64 only)", D);
    return VX_ERR_UNSUPPORTED;
  }
  VX_CHECK_ARG(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(o), "q/k/v/o must be 16-byte aligned");
  VX_CHECK_ARG(!apply_rope || rope_theta > 0.f, "rope_theta must be positive");
  VX_CHECK_ARG(pos0 >= 0, "pos0 must be >= 0");
  Launch L;
  vx_status st = make_launch(&L, ws, ws_bytes, vx_swa_attn_workspace(dt, B, T, H, D, apply_rope), stream);
  if (st != VX_OK) return st;
  if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const void* qq = q;
  const void* kk = k;
  if (apply_rope) {
    const size_t es = dt == VX_F32 ? 4 : 2;
    void* qr = cv.take(size_t(B) * T * H * D * es);
    void* kr = cv.take(size_t(B) * T * H * D * es);
    VX_CUDA(traced(L, "rope", 1, [&] { return launch_rope(L, q, k, qr, kr, dt == VX_BF16, B, T, H, pos0, rope_theta); }));
    qq = qr;
    kk = kr;
  }
  if (dt == VX_F32) {
    VX_CUDA(traced(L, "swa_attn_f32", 1, [&] {
      return launch_attn_f32(L, static_cast<const float*>(qq), static_cast<const float*>(kk),
                             static_cast<const float*>(v), static_cast<float*>(o), B, T, H, window, scale);
    }));
    return VX_OK;
  }
  const int64_t rs = int64_t(H) * 64, bs = int64_t(T) * H * 64;
  const AttnOperands op{qq, kk, v, rs, bs};
  AttnArgs aa;
  aa.out = o; aa.o_row = rs; aa.o_head = 64; aa.o_batch = bs;
  aa.B = B; aa.T = T; aa.H = H; aa.window = window;
  aa.scale_log2 = scale * 1.4426950408889634f;
  aa.status = L.status; aa.limit_ns = L.limit_ns;
  VX_CUDA(traced(L, "swa_attn_tc", 1, [&] { return launch_attn_bf16(L, op, aa); }));
  return VX_OK;
}

vx_status vx_rms_norm_fwd(const float* x, const float* r, const void* g, float* h_out, void* y, vx_dtype y_dt, int M,
                          int d, float eps, void* ws, size_t ws_bytes, cudaStream_t stream) {
  VX_CHECK_ARG(x && g && y, "x/g/y must not be null");
  VX_CHECK_ARG(M >= 0 && d > 0 && eps > 0.f, "bad shape or eps");
  if (d % 128 != 0 || d > 2048) {
    set_error("d=%d unsupported (multiple of 128, <= 2048)", d);
    return VX_ERR_UNSUPPORTED;
  }
  VX_CHECK_ARG(aligned16(x) && aligned16(y) && (!r || aligned16(r)) && (!h_out || aligned16(h_out)) &&
                   (reinterpret_cast<uintptr_t>(g) & 7) == 0,
               "x/r/h/y must be 16-byte aligned, g 8-byte aligned");
  Launch L;
  vx_status st = make_launch(&L, ws, ws_bytes, kStatusBytes, stream);
  if (st != VX_OK) return st;
  VX_CUDA(rmsnorm(L, x, r, r ? 1 : 0, 0, nullptr, static_cast<const uint16_t*>(g), h_out, y, y_dt == VX_BF16,
                          M, d, eps));
  return VX_OK;
}

size_t vx_encoder_layer_workspace(const vx_layer_cfg* cfg, int B, int T) {
  if (!cfg || B <= 0 || T <= 0) return kStatusBytes;
  return layer_ws_bytes(*cfg, int64_t(B) * T);
}

vx_status vx_encoder_layer_fwd(const vx_layer_cfg* cfg, const vx_layer_weights* w, const float* x, float* y, int B,
                               int T, int64_t pos0, void* ws, size_t ws_bytes, cudaStream_t stream) {
  vx_status st = check_cfg(cfg);
  if (st != VX_OK) return st;
  if ((st = check_weights(*cfg, w)) != VX_OK) return st;
  VX_CHECK_ARG(x && y && aligned16(x) && aligned16(y), "x/y must be non-null and 16-byte aligned");
  VX_CHECK_ARG(B > 0 && T > 0 && pos0 >= 0, "bad B=%d T=%d pos0=%lld", B, T, static_cast<long long>(pos0));
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_encoder_layer_workspace(cfg, B, T), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const LayerBufs bf = carve_layer(cv, *cfg, int64_t(B) * T);
  if ((st = init_norm_ctr(L, bf, int64_t(B) * T)) != VX_OK) return st;
  Pending out;
  if ((st = run_layer(L, *cfg, *w, Pending{x, nullptr, 0, nullptr}, &out, y, B, T, pos0, bf, nullptr)) != VX_OK)
    return st;
  if (out.base != y || out.parts || out.bias)
    VX_CUDA(reduce_into(L, out, y, B * T, cfg->d_model));
  return VX_OK;
}

size_t vx_conv_stem_workspace(int B, int n_mels, int Tm, int d) {
  if (B <= 0 || n_mels <= 0 || Tm <= 0 || d <= 0) return kStatusBytes;
  Carve cv{nullptr, kStatusBytes};
  carve_conv(cv, B, n_mels, Tm, d);
  return align_up(cv.off, kAlign);
}

static vx_status check_conv_args(const float* mel, const void* w1p, const void* b1, const void* w2p, const void* b2,
                                 const float* out, int B, int n_mels, int Tm, int d) {
  VX_CHECK_ARG(mel && w1p && b1 && w2p && b2 && out, "conv stem pointers must not be null");
  VX_CHECK_ARG(aligned16(w1p) && aligned16(w2p) && aligned16(b1) && aligned16(b2) && aligned16(out),
               "conv weights/bias/out must be 16-byte aligned");
  VX_CHECK_ARG(B > 0 && Tm > 0 && n_mels > 0 && d > 0, "bad conv shape");
  if (n_mels % 64 != 0 || d % 128 != 0) {
    set_error("conv stem needs n_mels %% 64 == 0 and d %% 128 == 0 (got %d, %d)", n_mels, d);
    return VX_ERR_UNSUPPORTED;
  }
  return VX_OK;
}

vx_status vx_conv_stem_fwd(const float* mel, const void* w1p, const void* b1, const void* w2p, const void* b2,
                           float* out, int B, int n_mels, int Tm, int d, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
  vx_status st = check_conv_args(mel, w1p, b1, w2p, b2, out, B, n_mels, Tm, d);
  if (st != VX_OK) return st;
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_conv_stem_workspace(B, n_mels, Tm, d), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const ConvBufs cb = carve_conv(cv, B, n_mels, Tm, d);
  return run_conv_stem(L, mel, w1p, b1, w2p, b2, out, B, n_mels, Tm, d, cb);
}

size_t vx_conv_stem_step_workspace(int S, int n_mels, int n_new, int d) {
  return vx_conv_stem_workspace(S, n_mels, n_new, d);
}

vx_status vx_conv_stem_step(const float* mel_new, const void* w1p, const void* b1, const void* w2p, const void* b2,
                            void* cache_x, void* cache_h1, float* out, int S, int n_mels, int n_new, int d, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
  vx_status st = check_conv_args(mel_new, w1p, b1, w2p, b2, out, S, n_mels, n_new, d);
  if (st != VX_OK) return st;
  VX_CHECK_ARG(cache_x && cache_h1 && aligned16(cache_x) && aligned16(cache_h1),
               "cache_x / cache_h1 must be non-null and 16-byte aligned");
  if (n_new % 2 != 0) {
    set_error("vx_conv_stem_step: n_new=%d must be even (the stride-2 conv keeps its phase across chunks)", n_new);
    return VX_ERR_UNSUPPORTED;
  }
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_conv_stem_step_workspace(S, n_mels, n_new, d), stream)) != VX_OK)
    return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const ConvBufs cb = carve_conv(cv, S, n_mels, n_new, d);
  return run_conv_stem(L, mel_new, w1p, b1, w2p, b2, out, S, n_mels, n_new, d, cb, static_cast<uint16_t*>(cache_x),
                       static_cast<uint16_t*>(cache_h1));
}

size_t vx_projector_workspace(int B, int T, int d, int hidden) {
  if (B <= 0 || T < 4 || d <= 0 || hidden <= 0) return kStatusBytes;
  const int64_t rows = static_cast<int64_t>(B) * (T / 4);
  Carve cv{nullptr, kStatusBytes};
  cv.take(rows * 4 * d * 2);
  cv.take(rows * hidden * 2);
  return align_up(cv.off, kAlign);
}

vx_status vx_projector_fwd(const float* x, const void* w1, const void* w2, float* out, int B, int T, int d, int hidden,
                           void* ws, size_t ws_bytes, cudaStream_t stream) {
  VX_CHECK_ARG(B > 0 && T > 0 && d > 0 && hidden > 0, "bad projector shape B=%d T=%d d=%d hidden=%d", B, T, d, hidden);
  if (d % 16 != 0 || hidden % 128 != 0) {
    set_error("projector needs d %% 16 == 0 and hidden %% 128 == 0 (got %d, %d)", d, hidden);
    return VX_ERR_UNSUPPORTED;
  }
  const int T4 = T / 4;
  if (T4 == 0) return VX_OK;   // fewer than 4 frames: no token, nothing is read or written
  VX_CHECK_ARG(x && w1 && w2 && out, "x / w1 / w2 / out must not be null");
  VX_CHECK_ARG(aligned16(x) && aligned16(w1) && aligned16(w2) && aligned16(out), "pointers must be 16-byte aligned");
  Launch L;
  vx_status st;
  if ((st = make_launch(&L, ws, ws_bytes, vx_projector_workspace(B, T, d, hidden), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const int M = B * T4;
  uint16_t* tok = static_cast<uint16_t*>(cv.take(static_cast<int64_t>(M) * 4 * d * 2));
  uint16_t* hid = static_cast<uint16_t*>(cv.take(static_cast<int64_t>(M) * hidden * 2));
  VX_CUDA(traced(L, "frames_to_tokens", 1, [&] { return launch_frames_to_tokens(L, x, tok, B, T, d); }));
  {
    GemmArgs a = base_args(L, M, hidden, 4 * d);
    a.out = hid; a.ld_out = hidden;
    if ((st = gemm(L, "gemm_proj1_gelu", tok, 4 * d, w1, a, EPI_GELU_BF16)) != VX_OK) return st;
  }
  {
    GemmArgs a = base_args(L, M, hidden, hidden);
    a.out = out; a.ld_out = hidden;
    if ((st = gemm(L, "gemm_proj2", hid, hidden, w2, a, EPI_F32)) != VX_OK) return st;
  }
  return VX_OK;
}

size_t vx_log_mel_workspace(int B, int N) {
  (void)B;
  (void)N;
  return align_up(kStatusBytes + align_up(log_mel_table_bytes(), kAlign), kAlign);
}

vx_status vx_log_mel_fwd(const float* audio, float* mel, int B, int N, int center, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  VX_CHECK_ARG(B > 0 && N > 0, "bad log-mel shape B=%d N=%d", B, N);
  if (center && N <= 200) {
    set_error("vx_log_mel_fwd: centred frames need more than 200 samples (got %d) for the reflect padding", N);
    return VX_ERR_UNSUPPORTED;
  }
  if (log_mel_frames(N, center) == 0) return VX_OK;   // no whole frame: nothing is read or written
  VX_CHECK_ARG(audio && mel, "audio / mel must not be null");
  Launch L;
  vx_status st;
  if ((st = make_launch(&L, ws, ws_bytes, vx_log_mel_workspace(B, N), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  void* tables = cv.take(log_mel_table_bytes());
  VX_CUDA(traced(L, "log_mel", 2, [&] { return launch_log_mel(L, audio, mel, B, N, center, tables); }));
  return VX_OK;
}

size_t vx_encoder_workspace(const vx_layer_cfg* cfg, int B, int n_mels, int Tm) {
  if (!cfg || B <= 0 || Tm <= 0) return kStatusBytes;
  const int To = (Tm - 1) / 2 + 1;
  const size_t a = vx_conv_stem_workspace(B, n_mels, Tm, cfg->d_model);
  const size_t b = layer_ws_bytes(*cfg, int64_t(B) * To);
  return a > b ? a : b;
}

vx_status vx_encoder_fwd(const vx_layer_cfg* cfg, const float* mel, int B, int n_mels, int Tm, const void* w1p,
                         const void* b1, const void* w2p, const void* b2, const vx_layer_weights* layers,
                         int n_layers, const void* final_g, float* out, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  vx_status st = check_cfg(cfg);
  if (st != VX_OK) return st;
  if ((st = check_conv_args(mel, w1p, b1, w2p, b2, out, B, n_mels, Tm, cfg->d_model)) != VX_OK) return st;
  VX_CHECK_ARG(layers != nullptr && n_layers >= 0, "layers must not be null");
  VX_CHECK_ARG(final_g && (reinterpret_cast<uintptr_t>(final_g) & 7) == 0, "final_g must be 8-byte aligned");
  for (int l = 0; l < n_layers; ++l)
    if ((st = check_weights(*cfg, &layers[l])) != VX_OK) return st;
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_encoder_workspace(cfg, B, n_mels, Tm), stream)) != VX_OK) return st;
  const int To = (Tm - 1) / 2 + 1;
  {
    Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
    const ConvBufs cb = carve_conv(cv, B, n_mels, Tm, cfg->d_model);
    if ((st = run_conv_stem(L, mel, w1p, b1, w2p, b2, out, B, n_mels, Tm, cfg->d_model, cb)) != VX_OK) return st;
  }
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const LayerBufs bf = carve_layer(cv, *cfg, int64_t(B) * To);
  if ((st = init_norm_ctr(L, bf, int64_t(B) * To)) != VX_OK) return st;
  Pending cur{out, nullptr, 0, nullptr};
  for (int l = 0; l < n_layers; ++l) {
    Pending next;
    // The layer's last GEMM may run the next RMSNorm: the next layer's (into
    // its normalised input) or the final one (in place, fp32).
    const NormFuse nn = l + 1 < n_layers ? NormFuse{static_cast<const uint16_t*>(layers[l + 1].attn_norm_g), bf.y0, true}
                                         : NormFuse{static_cast<const uint16_t*>(final_g), out, false};
    if ((st = run_layer(L, *cfg, layers[l], cur, &next, out, B, To, 0, bf, nullptr, &nn)) != VX_OK) return st;
    cur = next;
  }
  if (!cur.normed) {
    const int64_t pstride = static_cast<int64_t>(B) * To * cfg->d_model;
    VX_CUDA(rmsnorm(L, cur.base, cur.parts, cur.nparts, pstride, cur.bias, static_cast<const uint16_t*>(final_g),
                    nullptr, out, false, B * To, cfg->d_model, cfg->eps));
  }
  return VX_OK;
}

vx_status vx_stream_prefill(const vx_layer_cfg* cfg, const vx_layer_weights* layers, const vx_kv_ring* ring,
                            const float* x, float* y, int T, const void* final_g, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
  vx_status st = check_cfg(cfg);
  if (st != VX_OK) return st;
  if ((st = check_ring(*cfg, ring, 1)) != VX_OK) return st;
  VX_CHECK_ARG(layers != nullptr, "layers must not be null");
  for (int l = 0; l < ring->n_layers; ++l)
    if ((st = check_weights(*cfg, &layers[l])) != VX_OK) return st;
  VX_CHECK_ARG(x && y && aligned16(x) && aligned16(y) && T > 0, "bad x/y/T");
  const int S = ring->n_streams;
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_encoder_layer_workspace(cfg, S, T), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const LayerBufs bf = carve_layer(cv, *cfg, int64_t(S) * T);
  if ((st = init_norm_ctr(L, bf, int64_t(S) * T)) != VX_OK) return st;
  const int64_t layer_elems = int64_t(S) * cfg->n_heads * ring->window * cfg->head_dim;
  Pending cur{x, nullptr, 0, nullptr};
  for (int l = 0; l < ring->n_layers; ++l) {
    RingLayer rl{static_cast<uint16_t*>(ring->k) + l * layer_elems, static_cast<uint16_t*>(ring->v) + l * layer_elems,
                 ring->pos, ring->window, true, false};
    Pending next;
    if ((st = run_layer(L, *cfg, layers[l], cur, &next, y, S, T, 0, bf, &rl)) != VX_OK) return st;
    cur = next;
  }
  const int64_t pstride = static_cast<int64_t>(S) * T * cfg->d_model;
  if (final_g) {
    VX_CUDA(rmsnorm(L, cur.base, cur.parts, cur.nparts, pstride, cur.bias,
                            static_cast<const uint16_t*>(final_g), nullptr, y, false, S * T, cfg->d_model, cfg->eps));
  } else if (cur.base != y || cur.parts || cur.bias) {
    VX_CUDA(reduce_into(L, cur, y, S * T, cfg->d_model));
  }
  VX_CUDA(traced(L, "pos_add", 1, [&] { return launch_pos_add(L, ring->pos, S, T, true); }));
  return VX_OK;
}

size_t vx_stream_step_workspace(const vx_layer_cfg* cfg, int S, int n_new) {
  if (!cfg || S <= 0 || n_new <= 0) return kStatusBytes;
  return layer_ws_bytes(*cfg, int64_t(S) * n_new);
}

vx_status vx_stream_step(const vx_layer_cfg* cfg, const vx_layer_weights* layers, const vx_kv_ring* ring,
                         const float* x_new, float* y, int n_new, const void* final_g, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  vx_status st = check_cfg(cfg);
  if (st != VX_OK) return st;
  if ((st = check_ring(*cfg, ring, 1)) != VX_OK) return st;
  VX_CHECK_ARG(layers != nullptr, "layers must not be null");
  for (int l = 0; l < ring->n_layers; ++l)
    if ((st = check_weights(*cfg, &layers[l])) != VX_OK) return st;
  VX_CHECK_ARG(x_new && y && aligned16(x_new) && aligned16(y), "bad x_new/y");
  VX_CHECK_ARG(!final_g || (reinterpret_cast<uintptr_t>(final_g) & 7) == 0, "final_g must be 8-byte aligned");
  if (n_new < 1 || n_new > 8 || n_new > cfg->window) {
    set_error("n_new=%d unsupported (1..8 and <= window)", n_new);
    return VX_ERR_UNSUPPORTED;
  }
  const int S = ring->n_streams;
  const int M = S * n_new;
  Launch L;
  if ((st = make_launch(&L, ws, ws_bytes, vx_stream_step_workspace(cfg, S, n_new), stream)) != VX_OK) return st;
  Carve cv{static_cast<uint8_t*>(ws), kStatusBytes};
  const LayerBufs bf = carve_layer(cv, *cfg, M);
  if ((st = init_norm_ctr(L, bf, M)) != VX_OK) return st;
  const int64_t layer_elems = int64_t(S) * cfg->n_heads * ring->window * cfg->head_dim;
  Pending cur{x_new, nullptr, 0, nullptr};
  for (int l = 0; l < ring->n_layers; ++l) {
    RingLayer rl{static_cast<uint16_t*>(ring->k) + l * layer_elems, static_cast<uint16_t*>(ring->v) + l * layer_elems,
                 ring->pos, ring->window, false, true};
    Pending next;
    if ((st = run_layer(L, *cfg, layers[l], cur, &next, y, S, n_new, 0, bf, &rl)) != VX_OK) return st;
    cur = next;
  }
  // y = reduce(last layer output), then the optional final RMSNorm.
  const int64_t pstride = static_cast<int64_t>(M) * cfg->d_model;
  VX_CUDA(rmsnorm(L, cur.base, cur.parts, cur.nparts, pstride, cur.bias,
                          static_cast<const uint16_t*>(final_g), final_g ? nullptr : y, final_g ? y : nullptr, false,
                          M, cfg->d_model, cfg->eps));
  VX_CUDA(traced(L, "pos_add", 1, [&] { return launch_pos_add(L, ring->pos, S, n_new, false); }));
  return VX_OK;
}

vx_status vx_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns, cudaStream_t stream) {
  Launch L;
  vx_status st = make_launch(&L, ws, ws_bytes, kStatusBytes, stream);
  if (st != VX_OK) return st;
  L.limit_ns = timeout_ns > 0 ? timeout_ns : 1;
  VX_CUDA(traced(L, "selftest_wait", 1, [&] { return launch_selftest_wait(L); }));
  return VX_OK;
}

}  // extern "C"
