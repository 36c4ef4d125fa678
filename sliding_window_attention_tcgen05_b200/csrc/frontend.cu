// frontend.cu -- streaming log-mel frontend of the Realtime model
// (transcribe.cpp notes "Voxtral", section "Frontend"): 16 kHz audio, 400-
// sample frames (periodic Hann, n_fft 400, hop 160), power spectrum, slaney
// mel filterbank (128 bands, 0-8000 Hz, area normalised), log10 of
// max(mel, 1e-10), the fixed global maximum 1.5 (max(log, 1.5 - 8)) and
// (x + 4) / 4.  With centring (a clip, or a stream's first chunk) the audio is
// reflect-padded by 200 samples on both sides and the last frame is dropped.
//
// mel_tables_kernel: filterbank [128][201], window [400] and the twiddle table
//   cos / sin(2 pi m / 400) into the workspace (double-precision arithmetic).
// log_mel_kernel: one CTA per frame; the 400-point DFT runs on CUDA cores in
//   fp32 with the twiddle index (k n) mod 400 kept exact; thread k < 201 owns
//   frequency bin k, thread m < 128 then owns mel band m.  The step is small
//   (0.3 MFLOP per 10 ms frame) and precision-sensitive, so it stays off the
//   tensor cores.
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kNfft = 400, kHop = 160, kBins = kNfft / 2 + 1, kMels = 128;

__device__ double hz_to_mel_slaney(double f) {
  return f >= 1000.0 ? 15.0 + log(f / 1000.0) / (log(6.4) / 27.0) : f / (200.0 / 3.0);
}
__device__ double mel_to_hz_slaney(double m) {
  return m >= 15.0 ? 1000.0 * exp((m - 15.0) * (log(6.4) / 27.0)) : m * (200.0 / 3.0);
}

// Blocks 0 .. 127: filterbank row m; block 128: window and twiddles.
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
      fb[m * kBins + k] = static_cast<float>(w);
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

__global__ void __launch_bounds__(256)
log_mel_kernel(const float* __restrict__ audio, float* __restrict__ mel, const float* __restrict__ fb,
               const float* __restrict__ win, const float2* __restrict__ tw, int N, int F, int center) {
  __shared__ float xw[kNfft];
  __shared__ float2 stw[kNfft];
  __shared__ float pw[kBins];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x, b = blockIdx.y;
  const float* x = audio + static_cast<int64_t>(b) * N;
  for (int n = threadIdx.x; n < kNfft; n += blockDim.x) {
    int j = t * kHop + n - (center ? kNfft / 2 : 0);
    if (j < 0) j = -j;                        // reflect padding (edge sample not repeated)
    if (j >= N) j = 2 * (N - 1) - j;
    xw[n] = x[j] * win[n];
    stw[n] = tw[n];
  }
  __syncthreads();
  const int k = threadIdx.x;
  if (k < kBins) {
    float re = 0.f, im = 0.f;
    int idx = 0;                              // (k n) mod 400
    for (int n = 0; n < kNfft; ++n) {
      const float2 c = stw[idx];
      re = fmaf(xw[n], c.x, re);
      im = fmaf(xw[n], c.y, im);
      idx += k;
      if (idx >= kNfft) idx -= kNfft;
    }
    pw[k] = re * re + im * im;
  }
  __syncthreads();
  const int m = threadIdx.x;
  if (m < kMels) {
    const float* row = fb + m * kBins;
    float acc = 0.f;
    for (int kk = 0; kk < kBins; ++kk) acc = fmaf(__ldg(row + kk), pw[kk], acc);
    float v = log10f(fmaxf(acc, 1e-10f));
    v = fmaxf(v, 1.5f - 8.0f);
    mel[(static_cast<int64_t>(b) * kMels + m) * F + t] = (v + 4.0f) * 0.25f;
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
  float* fb = static_cast<float*>(tables);
  float* win = fb + kMels * kBins;
  float2* tw = reinterpret_cast<float2*>(win + kNfft);
  cudaError_t e = launch_kernel(mel_tables_kernel, dim3(kMels + 1), dim3(256), 0, L.stream, fb, win, tw);
  if (e != cudaSuccess) return e;
  return launch_kernel(log_mel_kernel, dim3(F, B), dim3(256), 0, L.stream, audio, mel, fb, win,
                       static_cast<const float2*>(tw), N, F, center);
}

}  // namespace vx
