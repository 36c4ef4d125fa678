// gemm.cu -- persistent, warp-specialised tcgen05 GEMM for sm_100a with the
// fused epilogues of the encoder layer (bias, RoPE, SwiGLU, GELU, residual).
//
//   D[M, N] = A[M, K] * B[N, K]^T,  A and B bf16 K-major, fp32 accumulate in TMEM.
//
// CTA = 6 warps: warps 0-3 epilogue (TMEM lanes 0-127 = tile rows), warp 4 TMA
// producer, warp 5 MMA issuer (owns the TMEM allocation).  128 x BN x 64 tiles,
// a STAGES-deep TMA -> shared memory ring guarded by mbarriers, and two TMEM
// accumulators so the epilogue of tile i overlaps the main loop of tile i+1.
// Tiles are visited M-fastest so the CTAs resident at one time share the same
// weight (B) panel through L2.
#include <cmath>
#include <cstdio>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;

// LEAN: about 96 KB of pipeline so that two CTAs share an SM (few-row GEMMs,
// whose work units must all be resident in one round).
template <int BN, bool LEAN>
struct GemmCfg {
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = LEAN ? (96 * 1024) / kStageBytes : ((BN == 256) ? 4 : (BN == 128 ? 6 : 8));
  static constexpr int kTmemCols = 2 * BN;  // two accumulators
  static constexpr int kSmem = kStages * kStageBytes + 1024 + 256;
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ void add_bias32(float (&v)[32], const uint16_t* bias) {
  const uint4* bp = reinterpret_cast<const uint4*>(bias);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 w = __ldg(bp + j);
    v[8 * j + 0] += bf16lo(w.x); v[8 * j + 1] += bf16hi(w.x);
    v[8 * j + 2] += bf16lo(w.y); v[8 * j + 3] += bf16hi(w.y);
    v[8 * j + 4] += bf16lo(w.z); v[8 * j + 5] += bf16hi(w.z);
    v[8 * j + 6] += bf16lo(w.w); v[8 * j + 7] += bf16hi(w.w);
  }
}

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    st_global_v4(dst + 8 * j, pack_bf16x2(v[8 * j + 0], v[8 * j + 1]),
                 pack_bf16x2(v[8 * j + 2], v[8 * j + 3]), pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                 pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
  }
}

__device__ __forceinline__ void store_f32x32(float* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    st_global_v4(dst + 4 * j, __float_as_uint(v[4 * j + 0]), __float_as_uint(v[4 * j + 1]),
                 __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
  }
}

template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tacc, int m, int n0, int ks) {
  const bool in_range = m < a.M;
  const int b = m / a.in_rows;
  const int t = m - b * a.in_rows;
  const bool valid = in_range && t < a.t_valid;
  const int64_t drow = static_cast<int64_t>(b) * a.out_rows + a.out_off + t;

  if constexpr (EPI == EPI_QKV_ROPE && BN == 64) {
    // one head per tile: rotate while reading (no sin/cos table kept)
    uint32_t r0[32], r1[32];
    tmem_ld32(tacc, r0);
    tmem_ld32(tacc + 32, r1);
    tmem_ld_wait();
    if (valid) {
      float x0[32], x1[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) { x0[i] = __uint_as_float(r0[i]); x1[i] = __uint_as_float(r1[i]); }
      if (a.bias) { add_bias32(x0, a.bias + n0); add_bias32(x1, a.bias + n0 + 32); }
      if (n0 < a.rope_cols) {
        const float posf = static_cast<float>((a.pos_arr ? a.pos_arr[b] : a.pos0) + t);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float sn, cs;
          rope_sincos(posf, a.inv_freq_hi[j], a.inv_freq_lo[j], &sn, &cs);
          const float u = x0[j], w = x1[j];
          x0[j] = u * cs - w * sn;
          x1[j] = w * cs + u * sn;
        }
      }
      uint16_t* dst = static_cast<uint16_t*>(a.out) + drow * a.ld_out + n0;
      store_bf16x32(dst, x0);
      store_bf16x32(dst + 32, x1);
    }
  } else if constexpr (EPI == EPI_QKV_ROPE) {
    float cs[32], sn[32];
    const bool rope_tile = n0 < a.rope_cols;
    if (rope_tile && valid) {
      const int64_t pos = (a.pos_arr ? a.pos_arr[b] : a.pos0) + t;
      const float posf = static_cast<float>(pos);
#pragma unroll
      for (int j = 0; j < 32; ++j) rope_sincos(posf, a.inv_freq_hi[j], a.inv_freq_lo[j], &sn[j], &cs[j]);
    }
#pragma unroll 1
    for (int c = 0; c < BN; c += 64) {
      uint32_t r0[32], r1[32];
      tmem_ld32(tacc + c, r0);
      tmem_ld32(tacc + c + 32, r1);
      tmem_ld_wait();
      if (valid) {
        const int n = n0 + c;
        float x0[32], x1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) { x0[i] = __uint_as_float(r0[i]); x1[i] = __uint_as_float(r1[i]); }
        if (a.bias) { add_bias32(x0, a.bias + n); add_bias32(x1, a.bias + n + 32); }
        if (n < a.rope_cols) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float u = x0[j], w = x1[j];
            x0[j] = u * cs[j] - w * sn[j];
            x1[j] = w * cs[j] + u * sn[j];
          }
        }
        uint16_t* dst = static_cast<uint16_t*>(a.out) + drow * a.ld_out + n;
        store_bf16x32(dst, x0);
        store_bf16x32(dst + 32, x1);
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll 1
    for (int g = 0; g < BN; g += 128) {
#pragma unroll 1
      for (int hh = 0; hh < 64; hh += 32) {
        uint32_t rg[32], ru[32];
        tmem_ld32(tacc + g + hh, rg);
        tmem_ld32(tacc + g + 64 + hh, ru);
        tmem_ld_wait();
        if (valid) {
          float gv[32], uv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) { gv[i] = __uint_as_float(rg[i]); uv[i] = __uint_as_float(ru[i]); }
          if (a.bias) { add_bias32(gv, a.bias + n0 + g + hh); add_bias32(uv, a.bias + n0 + g + 64 + hh); }
#pragma unroll
          for (int i = 0; i < 32; ++i) gv[i] = silu_f(gv[i]) * uv[i];
          const int f = (n0 + g) / 2 + hh;
          store_bf16x32(static_cast<uint16_t*>(a.out) + drow * a.ld_out + f, gv);
        }
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tacc + c, r);
      tmem_ld_wait();
      if (valid) {
        const int n = n0 + c;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if (a.bias) add_bias32(v, a.bias + n);
        if constexpr (EPI == EPI_F32) {
          if (a.res) {
            const float4* rp = reinterpret_cast<const float4*>(a.res + drow * a.ld_res + n);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 q = rp[j];
              v[4 * j] += q.x; v[4 * j + 1] += q.y; v[4 * j + 2] += q.z; v[4 * j + 3] += q.w;
            }
          }
          store_f32x32(static_cast<float*>(a.out) + ks * a.split_stride + drow * a.ld_out + n, v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
          if constexpr (EPI == EPI_GELU_BF16) {
            store_bf16x32(static_cast<uint16_t*>(a.out) + drow * a.ld_out + n, v);
          } else {
            store_f32x32(static_cast<float*>(a.out) + drow * a.ld_out + n, v);
          }
        }
      }
    }
  }
}

template <int BN, int EPI, bool LEAN>
__global__ void __launch_bounds__(kThreads, LEAN ? 2 : 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ GemmArgs a) {
  using C = GemmCfg<BN, LEAN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  // bars: full[S], empty[S], acc_full[2], acc_empty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto full = [&](int s) { return smem_addr(bars + s); };
  auto empty = [&](int s) { return smem_addr(bars + S + s); };
  auto acc_full = [&](int i) { return smem_addr(bars + 2 * S + i); };
  auto acc_empty = [&](int i) { return smem_addr(bars + 2 * S + 2 + i); };
  const uint32_t drain = smem_addr(bars + 2 * S + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  // Work unit u -> (m tile, K split, n tile), M fastest so that the units
  // resident at one time share a weight panel through L2.
  const int m_tiles = (a.M + kBM - 1) / kBM;
  const int splits = a.k_splits;
  const int num_tiles = m_tiles * (a.N / BN) * splits;
  const int nkb = a.K / kBK / splits;
  auto decode = [&](int u, int& m0, int& n0, int& ks) {
    const int mt = u % m_tiles;
    const int r = u / m_tiles;
    ks = r % splits;
    m0 = mt * kBM;
    n0 = (r / splits) * BN;
  };

  // The weights (B) do not depend on the previous kernel of the stream: the
  // producer starts streaming the first stages' B tiles before waiting for it.
  int npre = 0;
  if (warp == 4 && lane == 0 && blockIdx.x < num_tiles) {
    int m0, n0, ks;
    decode(blockIdx.x, m0, n0, ks);
    npre = nkb < S ? nkb : S;
    for (int i = 0; i < npre; ++i) {
      mbar_arrive_expect_tx(full(i), C::kStageBytes);
      tma_load_2d(smem_addr(sB + i * C::kBBytes), &tmB, full(i), (ks * nkb + i) * kBK, n0);
    }
  }
  // Inputs written by the previous kernel of the stream are read below.
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;  // bit s: stage s was filled at least once
      uint32_t last_par = 0;  // bit s: parity of the last fill of stage s
      int it = 0;           // k-block iterations issued so far
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int m0, n0, ks;
        decode(tile, m0, n0, ks);
        bool ok = true;
        for (int kb = ks * nkb; kb < (ks + 1) * nkb; ++kb, ++it) {
          const bool pre = it < npre;   // B already in flight, barrier already armed
          if (!pre) {
            if (!mbar_wait(empty(stage), phase ^ 1, wc, 1)) { ok = false; break; }
            mbar_arrive_expect_tx(full(stage), C::kStageBytes);
          }
          const int tap = kb / a.kb_per_tap;
          const int c = (kb - tap * a.kb_per_tap) * kBK;
          const int ax = (tap % a.a_stride) * a.a_tap_ch + c;
          const int ay = m0 + tap / a.a_stride;
          tma_load_2d(smem_addr(sA + stage * kABytes), &tmA, full(stage), ax, ay);
          if (!pre) tma_load_2d(smem_addr(sB + stage * C::kBBytes), &tmB, full(stage), kb * kBK, n0);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      // Wait (bounded, even after an abort) for the copies this thread issued.
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) mbar_wait(full(s), (last_par >> s) & 1u, dw, 5);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, BN, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
        const int ab = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(acc_empty(ab), acc_par ^ 1, wc, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full(stage), phase, wc, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(sA + stage * kABytes);
          const uint32_t b0 = smem_addr(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            umma_bf16(d_tmem, smem_desc_sw128(a0 + 32 * k, 16, 1024),
                      smem_desc_sw128(b0 + 32 * k, 16, 1024), idesc, (kb | k) != 0);
          }
          umma_commit(empty(stage));
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(acc_full(ab));
      }
      // Make sure no MMA of this CTA is still running before TMEM is released.
      umma_commit(drain);
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(drain, 0, dw, 6);
    }
  } else {
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      int m0, n0, ks;
      decode(tile, m0, n0, ks);
      const int ab = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      bool ok = mbar_wait(acc_full(ab), acc_par, wc, 4);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + ab * BN + (static_cast<uint32_t>(warp * 32) << 16);
      epilogue_tile<BN, EPI>(a, tacc, m0 + warp * 32 + lane, n0, ks);
      tc_fence_before();
      mbar_arrive(acc_empty(ab));
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------ CTA pairs --
// Two-CTA variant for many-row GEMMs: a cluster of two CTAs computes a
// 256 x 256 tile with tcgen05.mma.cta_group::2 (M = 256).  CTA r loads its own
// 128 rows of A and rows [128 r, 128 r + 128) of the tile's 256 B rows, so each
// SM stages 32 KB per 64-wide K block for 128 x 256 x 64 of MMA work (the
// one-CTA 128 x 256 tile stages 48 KB); the leader (CTA 0) issues the MMAs.
// TMA completions of both CTAs land on the leader's full barriers; MMA
// completions are multicast to the empty / accumulator barriers of both CTAs;
// both CTAs' epilogue warps release an accumulator on the leader's barrier.
// Each CTA's epilogue handles its 128 rows x 256 columns from its own TMEM.
constexpr int kPairBN = 256;
constexpr int kPairStages = 6;
constexpr int kPairStageBytes = kABytes + 128 * kBK * 2;   // A (128 rows) + half of B (128 rows)
constexpr int kPairSmem = kPairStages * kPairStageBytes + 1024 + 256;

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs a) {
  constexpr int S = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * kPairStageBytes);
  // bars: full[S] (used in CTA 0), empty[S], acc_full[2], acc_empty[2] (CTA 0), drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  auto full = [&](int s) { return smem_addr(bars + s); };
  auto empty = [&](int s) { return smem_addr(bars + S + s); };
  auto acc_full = [&](int i) { return smem_addr(bars + 2 * S + i); };
  auto acc_empty = [&](int i) { return smem_addr(bars + 2 * S + 2 + i); };
  const uint32_t drain = smem_addr(bars + 2 * S + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), 8); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc_pair(smem_addr(tmem_slot), 2 * kPairBN);
    tmem_relinquish_pair();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  const int m_tiles = (a.M + 255) / 256;
  const int num_tiles = m_tiles * (a.N / kPairBN);
  const int nkb = a.K / kBK;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  if (warp == 4) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      for (int tile = cluster; tile < num_tiles; tile += nclusters) {
        const int m0 = (tile % m_tiles) * 256 + 128 * rank;
        const int n0 = (tile / m_tiles) * kPairBN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1, wc, 31)) { ok = false; break; }
          const uint32_t fb = map_to_cta(full(stage), 0);   // the leader's full barrier
          if (rank == 0) mbar_arrive_expect_tx(full(stage), 2 * kPairStageBytes);
          const int tap = kb / a.kb_per_tap;
          const int c = (kb - tap * a.kb_per_tap) * kBK;
          const int ax = (tap % a.a_stride) * a.a_tap_ch + c;
          const int ay = m0 + tap / a.a_stride;
          tma_load_2d_pair(smem_addr(sA + stage * kABytes), &tmA, fb, ax, ay);
          tma_load_2d_pair(smem_addr(sB + stage * 128 * kBK * 2), &tmB, fb, kb * kBK, n0 + 128 * rank);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      if (rank == 0) {   // bounded wait for the pair's copies still in flight
        int zero = 0;
        WaitCtx dw = wc;
        dw.abort_flag = &zero;
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) mbar_wait(full(s), (last_par >> s) & 1u, dw, 35);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, kPairBN, 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
        const int ab = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(acc_empty(ab), acc_par ^ 1, wc, 32)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kPairBN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full(stage), phase, wc, 33)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(sA + stage * kABytes);
          const uint32_t b0 = smem_addr(sB + stage * 128 * kBK * 2);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, smem_desc_sw128(a0 + 32 * k, 16, 1024), smem_desc_sw128(b0 + 32 * k, 16, 1024),
                           idesc, (kb | k) != 0);
          umma_commit_pair(empty(stage), 0x3);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(acc_full(ab), 0x3);
      }
      umma_commit_pair(drain, 0x1);
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(drain, 0, dw, 36);
    }
  } else {
    int local = 0;
    const uint32_t acc_empty_leader0 = map_to_cta(acc_empty(0), 0);
    const uint32_t acc_empty_leader1 = map_to_cta(acc_empty(1), 0);
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
      const int m0 = (tile % m_tiles) * 256 + 128 * rank;
      const int n0 = (tile / m_tiles) * kPairBN;
      const int ab = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      bool ok = mbar_wait(acc_full(ab), acc_par, wc, 34);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + ab * kPairBN + (static_cast<uint32_t>(warp * 32) << 16);
      epilogue_tile<kPairBN, EPI>(a, tacc, m0 + warp * 32 + lane, n0, 0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ab ? acc_empty_leader1 : acc_empty_leader0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA of the pair still uses TMEM or the peer's barriers
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kPairBN);
  }
}

template <int EPI>
cudaError_t launch_pair(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tiles = ((a.M + 255) / 256) * (a.N / kPairBN);
  const int pairs = L.sm_count / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  return launch_kernel(gemm_tc2_kernel<EPI>, dim3(grid), dim3(kThreads), kPairSmem, L.stream, tmA, tmB, a);
}

template <int BN, int EPI, bool LEAN>
cudaError_t launch_one(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a) {
  using C = GemmCfg<BN, LEAN>;
  static bool attr_set = false;  // per instantiation; benign race (idempotent call)
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, LEAN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int m_tiles = (a.M + kBM - 1) / kBM;
  const int tiles = m_tiles * (a.N / BN) * a.k_splits;
  const int slots = (LEAN ? 2 : 1) * L.sm_count;
  const int grid = tiles < slots ? tiles : slots;
  return launch_kernel(gemm_tc_kernel<BN, EPI, LEAN>, dim3(grid), dim3(kThreads), C::kSmem, L.stream, tmA, tmB, a);
}

template <int BN, bool LEAN>
cudaError_t launch_bn(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB,
                      const GemmArgs& a, int epi) {
  switch (epi) {
    case EPI_F32: return launch_one<BN, EPI_F32, LEAN>(L, tmA, tmB, a);
    case EPI_QKV_ROPE: return launch_one<BN, EPI_QKV_ROPE, LEAN>(L, tmA, tmB, a);
    case EPI_SWIGLU:
      if constexpr (BN >= 128) return launch_one<BN, EPI_SWIGLU, LEAN>(L, tmA, tmB, a);
      else return cudaErrorInvalidValue;
    case EPI_GELU_BF16:
      if constexpr (!LEAN) return launch_one<BN, EPI_GELU_BF16, LEAN>(L, tmA, tmB, a);
      else return cudaErrorInvalidValue;
    case EPI_GELU_F32:
      if constexpr (!LEAN) return launch_one<BN, EPI_GELU_F32, LEAN>(L, tmA, tmB, a);
      else return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_gemm_pair(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const GemmArgs& args, int epi) {
  if (args.M <= 0) return cudaSuccess;
  if (args.k_splits != 1 || args.N % kPairBN != 0 || args.K % kBK != 0) return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_F32: return launch_pair<EPI_F32>(L, tmA, tmB, args);
    case EPI_QKV_ROPE: return launch_pair<EPI_QKV_ROPE>(L, tmA, tmB, args);
    case EPI_SWIGLU: return launch_pair<EPI_SWIGLU>(L, tmA, tmB, args);
    case EPI_GELU_BF16: return launch_pair<EPI_GELU_BF16>(L, tmA, tmB, args);
    case EPI_GELU_F32: return launch_pair<EPI_GELU_F32>(L, tmA, tmB, args);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const GemmArgs& args, int epi, int bn, bool lean) {
  if (args.M <= 0) return cudaSuccess;
  if (args.k_splits < 1 || (args.K / kBK) % args.k_splits != 0) return cudaErrorInvalidValue;
  if (lean) {
    if (bn == 128) return launch_bn<128, true>(L, tmA, tmB, args, epi);
    if (bn == 64) return launch_bn<64, true>(L, tmA, tmB, args, epi);
    return cudaErrorInvalidValue;
  }
  if (bn == 256) return launch_bn<256, false>(L, tmA, tmB, args, epi);
  if (bn == 128) return launch_bn<128, false>(L, tmA, tmB, args, epi);
  if (bn == 64) return launch_bn<64, false>(L, tmA, tmB, args, epi);
  return cudaErrorInvalidValue;
}

void fill_rope_freqs(GemmArgs* a, float theta, int head_dim) {
  for (int m = 0; m < 32; ++m) {
    const double inv = std::pow(static_cast<double>(theta), -2.0 * m / head_dim);
    const float hi = static_cast<float>(inv);
    a->inv_freq_hi[m] = hi;
    a->inv_freq_lo[m] = static_cast<float>(inv - static_cast<double>(hi));
  }
}

}  // namespace vx
