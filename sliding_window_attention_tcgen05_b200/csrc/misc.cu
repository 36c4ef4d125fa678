// misc.cu -- bandwidth-bound helpers: RMSNorm (+ residual), weight packing,
// conv-stem input staging, and the bounded-wait self test.
#include "vx_internal.h"

namespace vx {

namespace {

// ---------------------------------------------------------------- RMSNorm --
// RMSNorm with the pending residual sum folded in:
//   h = x + bias + sum_{k < nparts} parts[k]   (split-K partial sums of the GEMM before)
//   y = h * rsqrt(mean(h^2) + eps) * g          (skipped when y is null)
// Every load of a row (x, each partial sum, bias, gain) is issued before any
// arithmetic, so a row costs one memory round trip whatever nparts is.

__device__ __forceinline__ float4 add4f(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 add_bf16x4(float4 a, uint2 w) {
  return make_float4(a.x + bf16lo(w.x), a.y + bf16hi(w.x), a.z + bf16lo(w.y), a.w + bf16hi(w.y));
}
__device__ __forceinline__ float sumsq4(float4 a, float s) {
  return fmaf(a.x, a.x, fmaf(a.y, a.y, fmaf(a.z, a.z, fmaf(a.w, a.w, s))));
}
template <bool BF16_OUT>
__device__ __forceinline__ void store_norm4(void* y, int64_t idx4, float4 a, float inv, uint2 gw) {
  const float o0 = a.x * inv * bf16lo(gw.x), o1 = a.y * inv * bf16hi(gw.x);
  const float o2 = a.z * inv * bf16lo(gw.y), o3 = a.w * inv * bf16hi(gw.y);
  if constexpr (BF16_OUT) {
    uint2 w;
    w.x = pack_bf16x2(o0, o1);
    w.y = pack_bf16x2(o2, o3);
    reinterpret_cast<uint2*>(y)[idx4] = w;
  } else {
    reinterpret_cast<float4*>(y)[idx4] = make_float4(o0, o1, o2, o3);
  }
}

// One warp per row of d = 128 NV fp32 values (lane i holds float4 columns
// i, i + 32, ...), at most MAXP partial sums; four rows per CTA (a row holds
// up to 3 NV float4 in flight per lane, so CTAs stay small enough for every
// row of a one-layer batch to be resident at once).
template <bool BF16_OUT, int NV, int MAXP>
__global__ void __launch_bounds__(128)
rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ parts, int nparts, int64_t part_stride,
               const uint16_t* __restrict__ bias, const uint16_t* __restrict__ g, float* __restrict__ h_out,
               void* __restrict__ y, int M, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= M) return;
  const int64_t roff = static_cast<int64_t>(row) * d;
  float4 v[NV];
  float4 pp[MAXP > 0 ? MAXP : 1][NV];
  uint2 bw[NV], gw[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = reinterpret_cast<const float4*>(x + roff)[lane + 32 * i];
#pragma unroll
  for (int k = 0; k < MAXP; ++k)
    if (k < nparts) {
#pragma unroll
      for (int i = 0; i < NV; ++i) pp[k][i] = reinterpret_cast<const float4*>(parts + k * part_stride + roff)[lane + 32 * i];
    }
  if (bias) {
#pragma unroll
    for (int i = 0; i < NV; ++i) bw[i] = __ldg(reinterpret_cast<const uint2*>(bias) + lane + 32 * i);
  }
  if (y) {
#pragma unroll
    for (int i = 0; i < NV; ++i) gw[i] = __ldg(reinterpret_cast<const uint2*>(g) + lane + 32 * i);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
#pragma unroll
    for (int k = 0; k < MAXP; ++k)
      if (k < nparts) v[i] = add4f(v[i], pp[k][i]);
    if (bias) v[i] = add_bf16x4(v[i], bw[i]);
    ss = sumsq4(v[i], ss);
  }
  if (h_out) {
#pragma unroll
    for (int i = 0; i < NV; ++i) reinterpret_cast<float4*>(h_out + roff)[lane + 32 * i] = v[i];
  }
  if (y == nullptr) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / static_cast<float>(d) + eps);
#pragma unroll
  for (int i = 0; i < NV; ++i) store_norm4<BF16_OUT>(y, roff / 4 + lane + 32 * i, v[i], inv, gw[i]);
}

// Few-row variant: one CTA of d/4 threads per row (one float4 each), so that a
// handful of rows still spreads over the SMs; up to MAXP partial sums.
template <bool BF16_OUT, int MAXP>
__global__ void __launch_bounds__(512)
rmsnorm_row_kernel(const float* __restrict__ x, const float* __restrict__ parts, int nparts, int64_t part_stride,
                   const uint16_t* __restrict__ bias, const uint16_t* __restrict__ g, float* __restrict__ h_out,
                   void* __restrict__ y, int M, int d, float eps) {
  __shared__ float red[16];
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  const int c4 = threadIdx.x;
  const int64_t roff = static_cast<int64_t>(row) * d;
  float4 a = reinterpret_cast<const float4*>(x + roff)[c4];
  float4 pp[MAXP];
#pragma unroll
  for (int k = 0; k < MAXP; ++k)
    if (k < nparts) pp[k] = reinterpret_cast<const float4*>(parts + k * part_stride + roff)[c4];
  uint2 bw = make_uint2(0u, 0u), gw = make_uint2(0u, 0u);
  if (bias) bw = __ldg(reinterpret_cast<const uint2*>(bias) + c4);
  if (y) gw = __ldg(reinterpret_cast<const uint2*>(g) + c4);
#pragma unroll
  for (int k = 0; k < MAXP; ++k)
    if (k < nparts) a = add4f(a, pp[k]);
  if (bias) a = add_bf16x4(a, bw);
  if (h_out) reinterpret_cast<float4*>(h_out + roff)[c4] = a;
  if (y == nullptr) return;   // uniform over the CTA
  float ss = sumsq4(a, 0.f);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
  const float inv = rsqrtf(tot / static_cast<float>(d) + eps);
  store_norm4<BF16_OUT>(y, roff / 4 + c4, a, inv, gw);
}

// ---------------------------------------------------------------- packing --
// Row gather: output row rr (of `cols` bf16) comes from src_of(rr) or is zero.
struct PackSrc {
  const uint16_t* a;   // first source (q rows / gate rows)
  const uint16_t* b;   // second source (k rows / up rows)
  const uint16_t* c;   // third source (v rows)
  int mode;            // 0: concat a|b|c in blocks of `blk` rows; 1: interleave a,b in blocks of `blk`
  int blk;
};

__device__ __forceinline__ const uint16_t* pack_src_row(const PackSrc& p, int64_t rr, int64_t cols) {
  if (p.mode == 0) {
    const int64_t part = rr / p.blk, r = rr % p.blk;
    const uint16_t* s = part == 0 ? p.a : (part == 1 ? p.b : p.c);
    return s ? s + r * cols : nullptr;
  }
  const int64_t blk2 = 2 * p.blk;
  const int64_t g = rr / blk2, w = rr % blk2;
  const uint16_t* s = w < p.blk ? p.a : p.b;
  return s ? s + (g * p.blk + (w % p.blk)) * cols : nullptr;
}

// cols must be a multiple of 8 when > 1 (vector path) ; cols == 1 packs vectors.
__global__ void pack_rows_kernel(PackSrc p, uint16_t* __restrict__ out, int64_t rows, int64_t cols) {
  const int64_t chunks = cols >= 8 ? cols / 8 : 1;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (cols >= 8) {
    if (idx >= rows * chunks) return;
    const int64_t rr = idx / chunks, ch = idx % chunks;
    const uint16_t* s = pack_src_row(p, rr, cols);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (s) v = *reinterpret_cast<const uint4*>(s + ch * 8);
    *reinterpret_cast<uint4*>(out + rr * cols + ch * 8) = v;
  } else {
    if (idx >= rows) return;
    const uint16_t* s = pack_src_row(p, idx, 1);
    out[idx] = s ? *s : static_cast<uint16_t>(0);
  }
}

// Conv1d weight [O, C, 3] -> [O, 3, C].
__global__ void pack_conv_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ wp, int O, int C) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(O) * C * 3;
  if (idx >= total) return;
  const int64_t c = idx % C;
  const int64_t k = (idx / C) % 3;
  const int64_t o = idx / (3 * static_cast<int64_t>(C));
  wp[idx] = w[(o * C + c) * 3 + k];
}

// --------------------------------------------------------------- conv prep --
// mel [B, C, Tm] fp32 -> xpad [B, P, C] bf16, xpad[b, tp, c] = mel[b, c, tp - 2]
// for 2 <= tp < Tm + 2, else 0.  32 x 32 tiles through shared memory.
__global__ void conv_prep_kernel(const float* __restrict__ mel, uint16_t* __restrict__ xpad,
                                 int C, int Tm, int P, const uint16_t* __restrict__ cache_x) {
  pdl_wait();
  pdl_trigger();
  __shared__ float tile[32][33];
  const int tp0 = blockIdx.x * 32, c0 = blockIdx.y * 32, b = blockIdx.z;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int k = ty; k < 32; k += 8) {
    const int c = c0 + k, tp = tp0 + tx;
    float v = 0.f;
    if (c < C && tp >= 2 && tp < Tm + 2) v = mel[(static_cast<int64_t>(b) * C + c) * Tm + (tp - 2)];
    if (c < C && tp < 2 && cache_x) v = bf16_to_f(cache_x[(static_cast<int64_t>(b) * 2 + tp) * C + c]);
    tile[k][tx] = v;
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int tp = tp0 + k, c = c0 + tx;
    if (tp < P && c < C) {
      const __nv_bfloat16 h = __float2bfloat16_rn(tile[tx][k]);
      xpad[(static_cast<int64_t>(b) * P + tp) * C + c] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

// Rows {0, 1} of every clip of h1pad [B, P, d]: the two cached conv1 outputs
// (cache_h1 [B, 2, d]) or zeros; rows [Tm + 2, P): zeros.
__global__ void conv_pad_zero_kernel(uint16_t* __restrict__ h1pad, int Tm, int P, int d,
                                     const uint16_t* __restrict__ cache_h1) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int which = blockIdx.x;     // 0, 1, or 2 + (row - Tm - 2)
  const int row = which < 2 ? which : Tm + which;
  if (row >= P) return;
  uint16_t* r = h1pad + (static_cast<int64_t>(b) * P + row) * d;
  const uint16_t* src = (which < 2 && cache_h1) ? cache_h1 + (static_cast<int64_t>(b) * 2 + which) * d : nullptr;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8)
    *reinterpret_cast<uint4*>(r + c) = src ? *reinterpret_cast<const uint4*>(src + c) : make_uint4(0, 0, 0, 0);
}

// Conv padding cache after a chunk: the last two rows of each clip's xpad
// [B, P, C] and h1pad [B, P, d] (the chunk's last two mel frames and conv1
// outputs) into cache_x [B, 2, C] and cache_h1 [B, 2, d].
__global__ void conv_cache_save_kernel(const uint16_t* __restrict__ xpad, const uint16_t* __restrict__ h1pad,
                                       uint16_t* __restrict__ cache_x, uint16_t* __restrict__ cache_h1, int P, int C,
                                       int d) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y, j = blockIdx.x;   // j: 0, 1 -> xpad rows; 2, 3 -> h1pad rows
  const bool is_x = j < 2;
  const int width = is_x ? C : d;
  const int row = P - 2 + (j & 1);
  const uint16_t* src = (is_x ? xpad : h1pad) + (static_cast<int64_t>(b) * P + row) * width;
  uint16_t* dst = (is_x ? cache_x : cache_h1) + (static_cast<int64_t>(b) * 2 + (j & 1)) * width;
  for (int c = threadIdx.x * 8; c < width; c += blockDim.x * 8)
    *reinterpret_cast<uint4*>(dst + c) = *reinterpret_cast<const uint4*>(src + c);
}

// Projector tokens: frames 4j .. 4j+3 of clip b ([B, T, d] fp32) as the bf16
// row b * T4 + j of tok [B * T4, 4 d]; the last T % 4 frames are not read.
__global__ void frames_to_tokens_kernel(const float* __restrict__ x, uint16_t* __restrict__ tok, int T, int T4,
                                        int d, int64_t n8) {
  pdl_wait();
  pdl_trigger();
  const int64_t row_len8 = static_cast<int64_t>(d) / 2;   // 8-element groups per token row (4 d / 8)
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / row_len8, e = (i - row * row_len8) * 8;   // element of the token row
    const int64_t b = row / T4, j = row - b * T4;
    const float* src = x + (b * T + 4 * j) * d + e;   // 4 consecutive frames are contiguous
    const float4 lo = *reinterpret_cast<const float4*>(src);
    const float4 hi = *reinterpret_cast<const float4*>(src + 4);
    *reinterpret_cast<uint4*>(tok + row * 4 * d + e) =
        make_uint4(pack_bf16x2(lo.x, lo.y), pack_bf16x2(lo.z, lo.w), pack_bf16x2(hi.x, hi.y), pack_bf16x2(hi.z, hi.w));
  }
}

// --------------------------------------------------------------- selftest --
__global__ void selftest_wait_kernel(DevStatus* st, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{st, &abort_flag, limit_ns};
    mbar_wait(smem_addr(&bar), 0, wc, 99);   // nothing ever arrives
  }
}

// Sets n ints to zero (counters in a caller's workspace), as a kernel of the
// stream rather than a copy-engine memset, which could queue behind the
// caller's copies.
__global__ void zero_ints_kernel(int* __restrict__ p, int n) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

}  // namespace

// Without partial sums the row needs no registers for them: a separate
// instantiation keeps the register count (and so the rows in flight per SM)
// of the common case at its lowest.
template <bool BF16, int NV>
static cudaError_t launch_rms_warp(const Launch& L, const float* x, const float* parts, int nparts, int64_t ps,
                                   const uint16_t* bias, const uint16_t* g, float* h_out, void* y, int M, int d,
                                   float eps) {
  if (nparts == 0)
    return launch_kernel(rmsnorm_kernel<BF16, NV, 0>, dim3((M + 3) / 4), dim3(128), 0, L.stream, x, parts, nparts,
                         ps, bias, g, h_out, y, M, d, eps);
  return launch_kernel(rmsnorm_kernel<BF16, NV, 2>, dim3((M + 3) / 4), dim3(128), 0, L.stream, x, parts, nparts, ps,
                       bias, g, h_out, y, M, d, eps);
}

template <bool BF16>
static cudaError_t launch_rms(const Launch& L, const float* x, const float* parts, int nparts, int64_t ps,
                              const uint16_t* bias, const uint16_t* g, float* h_out, void* y, int M, int d, float eps) {
  if (M <= 512 || nparts > 2)   // few rows, or many partial sums: a CTA per row
    return launch_kernel(rmsnorm_row_kernel<BF16, 8>, dim3(M), dim3(d / 4), 0, L.stream, x, parts, nparts, ps, bias,
                         g, h_out, y, M, d, eps);
  switch (d / 128) {
#define VX_RMS_NV(n) \
  case n: return launch_rms_warp<BF16, n>(L, x, parts, nparts, ps, bias, g, h_out, y, M, d, eps);
    VX_RMS_NV(1) VX_RMS_NV(2) VX_RMS_NV(3) VX_RMS_NV(4) VX_RMS_NV(5) VX_RMS_NV(6) VX_RMS_NV(7) VX_RMS_NV(8)
    VX_RMS_NV(9) VX_RMS_NV(10) VX_RMS_NV(11) VX_RMS_NV(12) VX_RMS_NV(13) VX_RMS_NV(14) VX_RMS_NV(15) VX_RMS_NV(16)
#undef VX_RMS_NV
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rmsnorm(const Launch& L, const float* x, const float* parts, int nparts, int64_t part_stride,
                           const uint16_t* bias, const uint16_t* g, float* h_out, void* y, bool y_bf16, int M,
                           int d, float eps) {
  if (M <= 0) return cudaSuccess;
  if (nparts < 0 || nparts > 8 || d % 128 != 0 || d > 2048) return cudaErrorInvalidValue;
  if (y_bf16) return launch_rms<true>(L, x, parts, nparts, part_stride, bias, g, h_out, y, M, d, eps);
  return launch_rms<false>(L, x, parts, nparts, part_stride, bias, g, h_out, y, M, d, eps);
}

static cudaError_t pack_rows(const Launch& L, PackSrc p, uint16_t* out, int64_t rows, int64_t cols) {
  const int64_t work = cols >= 8 ? rows * (cols / 8) : rows;
  const int threads = 256;
  pack_rows_kernel<<<static_cast<unsigned>((work + threads - 1) / threads), threads, 0, L.stream>>>(p, out, rows, cols);
  return cudaGetLastError();
}

cudaError_t launch_pack_layer(const Launch& L, int d, int HD, int F, const uint16_t* wq, const uint16_t* wk,
                              const uint16_t* wv, const uint16_t* bq, const uint16_t* bv, const uint16_t* wg,
                              const uint16_t* wu, const uint16_t* bg, const uint16_t* bu, uint16_t* wqkv,
                              uint16_t* bqkv, uint16_t* wgu, uint16_t* bgu) {
  cudaError_t e;
  if ((e = pack_rows(L, PackSrc{wq, wk, wv, 0, HD}, wqkv, 3LL * HD, d)) != cudaSuccess) return e;
  if ((e = pack_rows(L, PackSrc{bq, nullptr, bv, 0, HD}, bqkv, 3LL * HD, 1)) != cudaSuccess) return e;
  if ((e = pack_rows(L, PackSrc{wg, wu, nullptr, 1, 64}, wgu, 2LL * F, d)) != cudaSuccess) return e;
  return pack_rows(L, PackSrc{bg, bu, nullptr, 1, 64}, bgu, 2LL * F, 1);
}

cudaError_t launch_pack_conv(const Launch& L, const uint16_t* w, uint16_t* wp, int O, int C) {
  const int64_t total = static_cast<int64_t>(O) * C * 3;
  pack_conv_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, L.stream>>>(w, wp, O, C);
  return cudaGetLastError();
}

cudaError_t launch_conv_prep(const Launch& L, const float* mel, uint16_t* xpad, uint16_t* h1pad, int B, int C,
                             int Tm, int P, int d, const uint16_t* cache_x, const uint16_t* cache_h1) {
  cudaError_t e = launch_kernel(conv_prep_kernel, dim3((P + 31) / 32, (C + 31) / 32, B), dim3(32, 8), 0, L.stream,
                                mel, xpad, C, Tm, P, cache_x);
  if (e != cudaSuccess) return e;
  return launch_kernel(conv_pad_zero_kernel, dim3(2 + (P - Tm - 2), B), dim3(128), 0, L.stream, h1pad, Tm, P, d,
                       cache_h1);
}

cudaError_t launch_conv_cache_save(const Launch& L, const uint16_t* xpad, const uint16_t* h1pad, uint16_t* cache_x,
                                   uint16_t* cache_h1, int B, int P, int C, int d) {
  return launch_kernel(conv_cache_save_kernel, dim3(4, B), dim3(128), 0, L.stream, xpad, h1pad, cache_x, cache_h1, P,
                       C, d);
}

cudaError_t launch_frames_to_tokens(const Launch& L, const float* x, uint16_t* tok, int B, int T, int d) {
  const int T4 = T / 4;
  const int64_t n8 = static_cast<int64_t>(B) * T4 * d / 2;
  if (n8 == 0) return cudaSuccess;
  const int64_t blocks = (n8 + 255) / 256;
  return launch_kernel(frames_to_tokens_kernel, dim3(static_cast<unsigned>(blocks < 4096 ? blocks : 4096)), dim3(256),
                       0, L.stream, x, tok, T, T4, d, n8);
}

cudaError_t launch_zero_ints(const Launch& L, int* p, int n) {
  return launch_kernel(zero_ints_kernel, dim3((n + 255) / 256), dim3(256), 0, L.stream, p, n);
}

cudaError_t launch_selftest_wait(const Launch& L) {
  selftest_wait_kernel<<<1, 32, 0, L.stream>>>(L.status, L.limit_ns);
  return cudaGetLastError();
}

}  // namespace vx
