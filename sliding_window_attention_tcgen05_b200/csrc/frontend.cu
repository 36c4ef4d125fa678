// frontend.cu -- streaming log-mel frontend of the Realtime model
// (transcribe.cpp notes "Voxtral", section "Frontend"): 16 kHz audio, 400-
// sample frames (periodic Hann, n_fft 400, hop 160), power spectrum, slaney
// mel filterbank (128 bands, 0-8000 Hz, area normalised), log10 of
// max(mel, 1e-10), the fixed global maximum 1.5 (max(log, 1.5 - 8)) and
// (x + 4) / 4.  With centring (a clip, or a stream's first chunk) the audio is
// reflect-padded by 200 samples on both sides and the last frame is dropped.
//
// mel_tables_kernel: filterbank (transposed, [201 bins][128 bands]), window
//   [400] and the twiddle table cos / sin(2 pi m / 400) into the workspace
//   (double-precision arithmetic).
// log_mel_kernel: one CTA per 32 consecutive frames of a clip.  The 400-point
//   DFT runs on CUDA cores in fp32 with the twiddle index (k n) mod 400 kept
//   exact, as a register-tiled product: each thread owns 4 frames x 7 bins,
//   so one 16-byte load of 4 frames' samples and one twiddle load per bin
//   feed 8 FMAs per bin (the twiddle address is shared by the 8 lanes of a
//   bin group, the samples by the 4 bin groups of a frame group).  The mel
//   product then runs with lanes over frames and 16 bands per warp, so the
//   filterbank reads are warp-uniform and the output rows are written 32
//   frames at a time.  Each output is the same sequence of fp32 operations
//   as a frame-at-a-time evaluation: sum over n in order, then over bins in
//   order.  The step is small (0.3 MFLOP per 10 ms frame) and
//   precision-sensitive, so it stays off the tensor cores.
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kNfft = 400, kHop = 160, kBins = kNfft / 2 + 1, kMels = 128;
constexpr int kFpc = 32;                       // frames per CTA
constexpr int kXsStride = kFpc + 4;            // samples [n][frame], row padded (16-byte aligned)
constexpr int kBinSlots = 224;                 // 7 bins per thread x 32 bin groups (201 used)
constexpr int kMelThreads = 256;
constexpr int kMelSmem = (kNfft * kXsStride + 2 * kNfft) * 4;   // samples | twiddles

__device__ double hz_to_mel_slaney(double f) {
  return f >= 1000.0 ? 15.0 + log(f / 1000.0) / (log(6.4) / 27.0) : f / (200.0 / 3.0);
}
__device__ double mel_to_hz_slaney(double m) {
  return m >= 15.0 ? 1000.0 * exp((m - 15.0) * (log(6.4) / 27.0)) : m * (200.0 / 3.0);
}

// Blocks 0 .. 127: filterbank band m (column m of the [bin][band] table);
// block 128: window and twiddles.
__global__ void mel_tables_kernel(float* __restrict__ fb, float* __restrict__ win, float2* __restrict__ tw) {
  pdl_wait();
  pdl_trigger();
  const int m = blockIdx.x;
  if (m < kMels) {
    const double mel_hi = hz_to_mel_slaney(8000.0);
    const double lo = mel_to_hz_slaney(mel_hi * m / (kMels + 1));
    const double mid = mel_to_hz_slaney(mel_hi * (m + 1) / (kMels + 1));
    const double hi = mel_to_hz_slaney(mel_hi * (m + 2) / (kMels + 1));
    for (int k = threadIdx.x; k < kBins; k += blockDim.x) {
      const double f = k * (16000.0 / kNfft);
      const double w = fmax(0.0, fmin((f - lo) / (mid - lo), (hi - f) / (hi - mid))) * (2.0 / (hi - lo));
      fb[k * kMels + m] = static_cast<float>(w);
    }
  } else {
    for (int n = threadIdx.x; n < kNfft; n += blockDim.x) {
      double s, c;
      sincospi(2.0 * n / kNfft, &s, &c);
      win[n] = static_cast<float>(0.5 - 0.5 * c);
      tw[n] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
  }
}

__global__ void __launch_bounds__(kMelThreads, 3)   // 3 CTAs (24 warps) per SM
log_mel_kernel(const float* __restrict__ audio, float* __restrict__ mel, const float* __restrict__ fbt,
               const float* __restrict__ win, const float2* __restrict__ tw, int N, int F, int center) {
  extern __shared__ __align__(16) float smem_f[];
  float* xs = smem_f;                                             // [400][kXsStride] windowed samples
  float2* stw = reinterpret_cast<float2*>(smem_f + kNfft * kXsStride);
  float* pw = smem_f;                                             // [kBinSlots][32] power, after the DFT
  pdl_wait();
  pdl_trigger();
  const int t0 = blockIdx.x * kFpc, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* x = audio + static_cast<int64_t>(b) * N;
  for (int i = tid; i < kFpc * kNfft; i += kMelThreads) {
    const int f = i / kNfft, n = i - f * kNfft;
    const int t = t0 + f;
    float v = 0.f;
    if (t < F) {
      int j = t * kHop + n - (center ? kNfft / 2 : 0);
      if (j < 0) j = -j;                      // reflect padding (edge sample not repeated)
      if (j >= N) j = 2 * (N - 1) - j;
      v = x[j] * win[n];
    }
    xs[n * kXsStride + f] = v;
  }
  for (int i = tid; i < kNfft; i += kMelThreads) stw[i] = tw[i];
  __syncthreads();

  // DFT: frames 4 fg .. 4 fg + 3, bins kb + 32 j (j < 7), kb = 4 warp + bg.
  const int fg = lane & 7, kb = 4 * warp + (lane >> 3);
  float re[7][4], im[7][4];
  int idx[7];
#pragma unroll
  for (int j = 0; j < 7; ++j) {
    idx[j] = 0;                               // (k n) mod 400 at n = 0
#pragma unroll
    for (int e = 0; e < 4; ++e) re[j][e] = im[j][e] = 0.f;
  }
#pragma unroll 2
  for (int n = 0; n < kNfft; ++n) {
    const float4 xv = *reinterpret_cast<const float4*>(xs + n * kXsStride + 4 * fg);
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      const float2 c = stw[idx[j]];
      re[j][0] = fmaf(xv.x, c.x, re[j][0]); im[j][0] = fmaf(xv.x, c.y, im[j][0]);
      re[j][1] = fmaf(xv.y, c.x, re[j][1]); im[j][1] = fmaf(xv.y, c.y, im[j][1]);
      re[j][2] = fmaf(xv.z, c.x, re[j][2]); im[j][2] = fmaf(xv.z, c.y, im[j][2]);
      re[j][3] = fmaf(xv.w, c.x, re[j][3]); im[j][3] = fmaf(xv.w, c.y, im[j][3]);
      idx[j] += kb + 32 * j;
      if (idx[j] >= kNfft) idx[j] -= kNfft;
    }
  }
  __syncthreads();   // every thread is done with the samples: pw reuses them
#pragma unroll
  for (int j = 0; j < 7; ++j) {
    float4 pv;
    pv.x = re[j][0] * re[j][0] + im[j][0] * im[j][0];
    pv.y = re[j][1] * re[j][1] + im[j][1] * im[j][1];
    pv.z = re[j][2] * re[j][2] + im[j][2] * im[j][2];
    pv.w = re[j][3] * re[j][3] + im[j][3] * im[j][3];
    *reinterpret_cast<float4*>(pw + (kb + 32 * j) * kFpc + 4 * fg) = pv;
  }
  __syncthreads();

  // Mel bands 16 warp .. 16 warp + 15 of frame t0 + lane.
  float acc[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) acc[q] = 0.f;
  const float4* wrow = reinterpret_cast<const float4*>(fbt + 16 * warp);
#pragma unroll 2
  for (int k = 0; k < kBins; ++k) {
    const float p = pw[k * kFpc + lane];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const float4 w = __ldg(wrow + k * (kMels / 4) + q4);
      acc[4 * q4 + 0] = fmaf(w.x, p, acc[4 * q4 + 0]);
      acc[4 * q4 + 1] = fmaf(w.y, p, acc[4 * q4 + 1]);
      acc[4 * q4 + 2] = fmaf(w.z, p, acc[4 * q4 + 2]);
      acc[4 * q4 + 3] = fmaf(w.w, p, acc[4 * q4 + 3]);
    }
  }
  const int t = t0 + lane;
  if (t < F) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      float v = log10f(fmaxf(acc[q], 1e-10f));
      v = fmaxf(v, 1.5f - 8.0f);
      mel[(static_cast<int64_t>(b) * kMels + 16 * warp + q) * F + t] = (v + 4.0f) * 0.25f;
    }
  }
}

}  // namespace

int log_mel_frames(int N, int center) {
  if (center) return N / kHop;
  return N >= kNfft ? 1 + (N - kNfft) / kHop : 0;
}

size_t log_mel_table_bytes() { return (kMels * kBins + kNfft) * sizeof(float) + kNfft * sizeof(float2); }

cudaError_t launch_log_mel(const Launch& L, const float* audio, float* mel, int B, int N, int center, void* tables) {
  const int F = log_mel_frames(N, center);
  if (F <= 0 || B <= 0) return cudaSuccess;
  float* fb = static_cast<float*>(tables);   // [201][128]
  float* win = fb + kMels * kBins;
  float2* tw = reinterpret_cast<float2*>(win + kNfft);
  cudaError_t e = launch_kernel(mel_tables_kernel, dim3(kMels + 1), dim3(256), 0, L.stream, fb, win, tw);
  if (e != cudaSuccess) return e;
  return launch_kernel(log_mel_kernel, dim3((F + kFpc - 1) / kFpc, B), dim3(kMelThreads), kMelSmem, L.stream, audio,
                       mel, static_cast<const float*>(fb), static_cast<const float*>(win),
                       static_cast<const float2*>(tw), N, F, center);
}

}  // namespace vx
