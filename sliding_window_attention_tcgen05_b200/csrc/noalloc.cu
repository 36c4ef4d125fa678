// noalloc.cu -- vx_swa_attn_fwd_noalloc: the sliding-window attention call
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run attention: real-time audio callbacks that must not block on the
// driver's allocator, plug-in hosts that own every device allocation, and
// code running under a fixed memory budget that may not grow.  This entry
// point takes no workspace.  Its scratch -- the RoPE-rotated q and k and the
// status word of the bounded waits -- lives in one file-scope device array of
// kNoAllocScratchBytes that every GPU loading this library holds until the
// process exits.  Inputs and outputs are still the caller's.
#include <cstring>
#include <mutex>

#include "vx.h"
#include "vx_internal.h"

namespace {

// 256 bytes of status word, then room for the rotated q and k.
constexpr size_t kNoAllocStatusBytes = 256;
constexpr size_t kNoAllocScratchBytes = (32u << 20) + kNoAllocStatusBytes;   // 32 MiB + status

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct ScratchAddr {
  CUcontext ctx;   // the context the address was looked up in
  void* ptr;
};
ScratchAddr g_noalloc_addr[kMaxDevices] = {};

// The current context, through the runtime's driver entry point (no -lcuda).
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<Fn>(nullptr);
    return reinterpret_cast<Fn>(p);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a stand-in, so the address is looked up (with the
// device current) on the first call on each device and cached.  The cache
// also remembers the context it came from and looks the address up again
// when that context has changed (after cudaDeviceReset, say).
vx_status noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    vx::set_error("vx_swa_attn_fwd_noalloc: no usable current CUDA device (%s)", cudaGetErrorString(e));
    return VX_ERR_CUDA;
  }
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  ScratchAddr& c = g_noalloc_addr[dev];
  if (c.ptr == nullptr || ctx == nullptr || c.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      vx::set_error("vx_swa_attn_fwd_noalloc: cudaGetSymbolAddress of the static scratch failed: %s",
                    cudaGetErrorString(e));
      return VX_ERR_CUDA;
    }
    c.ctx = current_context();   // the lookup made the runtime's context current
    c.ptr = p;
  }
  *out = c.ptr;
  return VX_OK;
}

}  // namespace

extern "C" {

vx_status vx_swa_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, vx_dtype dt, int B, int T,
                                  int H, int D, int window, int apply_rope, float rope_theta, int64_t pos0,
                                  float scale, cudaStream_t stream) {
  using namespace vx;
  if (!(q && k && v && o)) {
    set_error("vx_swa_attn_fwd_noalloc: q/k/v/o must not be null");
    return VX_ERR_INVALID_ARG;
  }
  if (B <= 0 || T <= 0 || H <= 0 || window < 1 || (dt != VX_F32 && dt != VX_BF16) || pos0 < 0 ||
      (apply_rope && !(rope_theta > 0.f))) {
    set_error("vx_swa_attn_fwd_noalloc: bad arguments B=%d T=%d H=%d window=%d", B, T, H, window);
    return VX_ERR_INVALID_ARG;
  }
  if (D != 64) {
    set_error("vx_swa_attn_fwd_noalloc: head_dim %d unsupported (64 only)", D);
    return VX_ERR_UNSUPPORTED;
  }
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o);
  if (al & 15) {
    set_error("vx_swa_attn_fwd_noalloc: q/k/v/o must be 16-byte aligned");
    return VX_ERR_INVALID_ARG;
  }
  const size_t es = dt == VX_F32 ? 4 : 2;
  const size_t one = static_cast<size_t>(B) * T * H * D * es;   // one rotated tensor
  const size_t need = apply_rope ? 2 * ((one + 255) / 256 * 256) : 0;
  if (need > kNoAllocScratchBytes - kNoAllocStatusBytes) {
    set_error("vx_swa_attn_fwd_noalloc: B*T*H = %lld needs %zu bytes of scratch for the rotated q/k, more than "
              "the %zu-byte static limit (use vx_swa_attn_fwd with a workspace)",
              static_cast<long long>(B) * T * H, need, kNoAllocScratchBytes - kNoAllocStatusBytes);
    return VX_ERR_INVALID_ARG;
  }
  void* base = nullptr;
  vx_status st = noalloc_scratch(&base);
  if (st != VX_OK) return st;
  int sms = current_sm_count();
  if (sms <= 0) {
    set_error("vx_swa_attn_fwd_noalloc: no CUDA device is current");
    return VX_ERR_CUDA;
  }
  Launch L{stream, static_cast<DevStatus*>(base), wait_limit_ns(), sms};
  // The status word must start at zero; the rotated q/k are fully overwritten.
  cudaError_t e = cudaMemsetAsync(base, 0, kNoAllocStatusBytes, stream);
  if (e != cudaSuccess) {
    set_error("vx_swa_attn_fwd_noalloc: clearing the status word failed: %s", cudaGetErrorString(e));
    return VX_ERR_CUDA;
  }
  if (scale <= 0.f) scale = 0.125f;   // 1/sqrt(64)
  const void* qq = q;
  const void* kk = k;
  if (apply_rope) {
    unsigned char* sc = static_cast<unsigned char*>(base) + kNoAllocStatusBytes;
    void* qr = sc;
    void* kr = sc + (one + 255) / 256 * 256;
    if ((e = traced(L, "rope", 1, [&] {
           return launch_rope(L, q, k, qr, kr, dt == VX_BF16, B, T, H, pos0, rope_theta);
         })) != cudaSuccess) {
      set_error("vx_swa_attn_fwd_noalloc: RoPE launch failed: %s", cudaGetErrorString(e));
      return VX_ERR_CUDA;
    }
    qq = qr;
    kk = kr;
  }
  if (dt == VX_F32) {
    e = traced(L, "swa_attn_f32", 1, [&] {
      return launch_attn_f32(L, static_cast<const float*>(qq), static_cast<const float*>(kk),
                             static_cast<const float*>(v), static_cast<float*>(o), B, T, H, window, scale);
    });
  } else {
    const int64_t rs = int64_t(H) * 64, bs = int64_t(T) * H * 64;
    const AttnOperands op{qq, kk, v, rs, bs};
    AttnArgs aa;
    aa.out = o; aa.o_row = rs; aa.o_head = 64; aa.o_batch = bs;
    aa.B = B; aa.T = T; aa.H = H; aa.window = window;
    aa.scale_log2 = scale * 1.4426950408889634f;
    aa.status = L.status; aa.limit_ns = L.limit_ns;
    e = traced(L, "swa_attn_tc", 1, [&] { return launch_attn_bf16(L, op, aa); });
  }
  if (e != cudaSuccess) {
    set_error("vx_swa_attn_fwd_noalloc: attention launch failed: %s", cudaGetErrorString(e));
    return VX_ERR_CUDA;
  }
  return VX_OK;
}

}  // extern "C"
