// attn.cu -- causal sliding-window attention kernels.
//
// swa_attn_tc_kernel: flash-style bf16 attention on tcgen05 tensor cores.
//   One CTA per (128-query tile, head, clip).  Only the key tiles that meet
//   the causal window (i - W, i] of some query of the tile are visited; the
//   masks are evaluated only on the edge tiles.  K/V tiles arrive by TMA into
//   a 3-stage ring; S = Q K^T and O_j = P_j V_j accumulate in TMEM
//   (S double-buffered in columns 0..255, O_j in 256..383); the softmax warps
//   read S from TMEM, keep the running max / sum in registers, write P (bf16)
//   to shared memory as the A operand of the P V product, and fold each O_j
//   into a register accumulator with the online-softmax rescale.
//   Warps 0-3: softmax (TMEM lane = query row), warp 4: TMA, warp 5: MMA.
// swa_attn_f32_kernel: fp32 CUDA-core reference-precision path (one warp per
//   query row), used for fp32 inputs.
// rope_kernel: RoPE pre-pass for vx_swa_attn_fwd on raw q, k.
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kAttnThreads = 192;
constexpr int kNS = 3;                      // K/V pipeline stages
constexpr int kTile = 128 * 64 * 2;         // one 128 x 64 bf16 tile
constexpr int kPBytes = 128 * 128 * 2;      // one P tile (128 queries x 128 keys)
constexpr int kAttnSmem = kTile * (1 + 2 * kNS) + 2 * kPBytes + 1024 + 512;
constexpr uint32_t kTmemCols = 512;

__global__ void __launch_bounds__(kAttnThreads, 1)
swa_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTile;
  uint8_t* sV = sK + kNS * kTile;
  uint8_t* sP = sV + kNS * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kPBytes);
  // barrier indices
  constexpr int QF = 0, KF = 1, VF = KF + kNS, KVE = VF + kNS, SF = KVE + kNS, SE = SF + 2,
                PF = SE + 2, PE = PF + 2, OF = PE + 2, OE = OF + 2, DR = OE + 2, NBAR = DR + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int W = a.window;
  const int lo_key = max(0, q0 - W + 1);
  const int hi_key = min(a.T - 1, q0 + 127);
  const int kt0 = lo_key / 128;
  const int n = hi_key / 128 - kt0 + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(QF), 1);
    for (int s = 0; s < kNS; ++s) { mbar_init(bar(KF + s), 1); mbar_init(bar(VF + s), 1); mbar_init(bar(KVE + s), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(SF + i), 1); mbar_init(bar(SE + i), 128);
      mbar_init(bar(PF + i), 128); mbar_init(bar(PE + i), 1);
      mbar_init(bar(OF + i), 1); mbar_init(bar(OE + i), 128);
    }
    mbar_init(bar(DR), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(QF), kTile);
      tma_load_4d(smem_addr(sQ), &tmQ, bar(QF), 0, h, q0, b);
      uint32_t last_par = 0;
      int filled = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kNS;
        const uint32_t ph = (j / kNS) & 1;
        if (!mbar_wait(bar(KVE + st), ph ^ 1, wc, 11)) break;
        const int key0 = (kt0 + j) * 128;
        mbar_arrive_expect_tx(bar(KF + st), kTile);
        tma_load_4d(smem_addr(sK + st * kTile), &tmK, bar(KF + st), 0, h, key0, b);
        mbar_arrive_expect_tx(bar(VF + st), kTile);
        tma_load_4d(smem_addr(sV + st * kTile), &tmV, bar(VF + st), 0, h, key0, b);
        last_par = (last_par & ~(1u << st)) | (ph << st);
        filled = j + 1;
      }
      // Bounded wait for every copy still in flight (also after an abort).
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(QF), 0, dw, 12);
      for (int s = 0; s < kNS && s < filled; ++s) {
        mbar_wait(bar(KF + s), (last_par >> s) & 1u, dw, 12);
        mbar_wait(bar(VF + s), (last_par >> s) & 1u, dw, 12);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, 1);
      bool ok = mbar_wait(bar(QF), 0, wc, 13);
      const uint32_t qa = smem_addr(sQ);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % kNS;
        const int pb = jj & 1;
        const uint32_t pph = (jj >> 1) & 1;
        if (!mbar_wait(bar(PF + pb), pph, wc, 14)) return false;
        if (!mbar_wait(bar(VF + st), (jj / kNS) & 1, wc, 15)) return false;
        if (!mbar_wait(bar(OE + pb), pph ^ 1, wc, 16)) return false;
        tc_fence_after();
        const uint32_t pa = smem_addr(sP + pb * kPBytes);
        const uint32_t va = smem_addr(sV + st * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(pa + (k >> 2) * (kPBytes / 2) + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(va + k * 2048, kTile, 1024);
          umma_bf16(tmem + 256 + pb * 64, ad, bd, idesc_o, k > 0);
        }
        umma_commit(bar(OF + pb));
        umma_commit(bar(PE + pb));
        umma_commit(bar(KVE + st));
        return true;
      };
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % kNS;
        const int sb = j & 1;
        if (!(ok = mbar_wait(bar(SE + sb), ((j >> 1) & 1) ^ 1, wc, 17))) break;
        if (!(ok = mbar_wait(bar(KF + st), (j / kNS) & 1, wc, 18))) break;
        tc_fence_after();
        const uint32_t ka = smem_addr(sK + st * kTile);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + sb * 128, smem_desc_sw128(qa + 32 * k, 16, 1024),
                    smem_desc_sw128(ka + 32 * k, 16, 1024), idesc_s, k > 0);
        umma_commit(bar(SF + sb));
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(n - 1);
      umma_commit(bar(DR));
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(DR), 0, dw, 19);
    }
  } else {
    // ---------------- softmax / output warps: thread r owns query row q0 + r
    const int r = threadIdx.x;
    const int i = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float o[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) o[d] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, mu_o = -INFINITY, mu0 = 0.f, mu1 = 0.f;
    bool ok = true;

    auto consume_o = [&](int jj) -> bool {
      const int ob = jj & 1;
      bool w = mbar_wait(bar(OF + ob), (jj >> 1) & 1, wc, 20);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + 256 + ob * 64 + lane_off, r0);
      tmem_ld32(tmem + 256 + ob * 64 + 32 + lane_off, r1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(OE + ob));
      const float mu_j = ob ? mu1 : mu0;
      const float f = (mu_o == -INFINITY) ? 0.f : ex2_approx(mu_o - mu_j);
#pragma unroll
      for (int d = 0; d < 32; ++d) {
        o[d] = fmaf(o[d], f, __uint_as_float(r0[d]));
        o[d + 32] = fmaf(o[d + 32], f, __uint_as_float(r1[d]));
      }
      mu_o = mu_j;
      return true;
    };

    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t sph = (j >> 1) & 1;
      bool w = mbar_wait(bar(SF + sb), sph, wc, 21);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      {
        uint32_t s0[32], s1[32], s2[32], s3[32];
        const uint32_t ta = tmem + sb * 128 + lane_off;
        tmem_ld32(ta, s0);
        tmem_ld32(ta + 32, s1);
        tmem_ld32(ta + 64, s2);
        tmem_ld32(ta + 96, s3);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(s0[c]) * sl2;
          x[c + 32] = __uint_as_float(s1[c]) * sl2;
          x[c + 64] = __uint_as_float(s2[c]) * sl2;
          x[c + 96] = __uint_as_float(s3[c]) * sl2;
        }
      }
      tc_fence_before();
      mbar_arrive(bar(SE + sb));
      const int key0 = (kt0 + j) * 128;
      // Edge tile: some (row, key) pair of the tile is outside (i - W, i].
      if (key0 + 127 > q0 || key0 <= q0 + 127 - W) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int key = key0 + c;
          if (key > i || key <= i - W) x[c] = -INFINITY;
        }
      }
      float tmax = x[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) tmax = fmaxf(tmax, x[c]);
      const float m_new = fmaxf(m_run, tmax);
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2_approx(m_run - mu);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        x[c] = ex2_approx(x[c] - mu);
        rs += x[c];
      }
      l_run = fmaf(l_run, alpha, rs);
      m_run = m_new;
      if (sb) mu1 = mu; else mu0 = mu;

      w = mbar_wait(bar(PE + sb), sph ^ 1, wc, 22);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      // P row r: keys 0..63 in the first 16 KB half, 64..127 in the second,
      // 128-byte rows with the 16-byte chunk index XOR-ed by (r & 7).
      uint8_t* prow = sP + sb * kPBytes + r * 128;
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const uint32_t off = (cc >> 3) * (kPBytes / 2) + ((((cc & 7) ^ (r & 7))) << 4);
        const uint32_t addr = smem_addr(prow + off);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                     "r"(pack_bf16x2(x[cc * 8 + 0], x[cc * 8 + 1])), "r"(pack_bf16x2(x[cc * 8 + 2], x[cc * 8 + 3])),
                     "r"(pack_bf16x2(x[cc * 8 + 4], x[cc * 8 + 5])), "r"(pack_bf16x2(x[cc * 8 + 6], x[cc * 8 + 7]))
                     : "memory");
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(PF + sb));
      if (j > 0 && !(ok = consume_o(j - 1))) break;
    }
    if (ok) ok = consume_o(n - 1);
    if (ok && i < a.T) {
      const float inv_l = 1.0f / l_run;
      uint16_t* dst = static_cast<uint16_t*>(a.out) + static_cast<int64_t>(b) * a.o_batch +
                      static_cast<int64_t>(i) * a.o_row + static_cast<int64_t>(h) * a.o_head;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        st_global_v4(dst + 8 * c, pack_bf16x2(o[8 * c] * inv_l, o[8 * c + 1] * inv_l),
                     pack_bf16x2(o[8 * c + 2] * inv_l, o[8 * c + 3] * inv_l),
                     pack_bf16x2(o[8 * c + 4] * inv_l, o[8 * c + 5] * inv_l),
                     pack_bf16x2(o[8 * c + 6] * inv_l, o[8 * c + 7] * inv_l));
      }
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------- fp32 path --
__global__ void __launch_bounds__(128)
swa_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                    float* __restrict__ o, int T, int H, int W, float scale) {
  pdl_wait();
  pdl_trigger();
  __shared__ float qs[4][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  if (i >= T) return;
  const int64_t rs = static_cast<int64_t>(H) * 64;
  const int64_t base = static_cast<int64_t>(b) * T * rs + static_cast<int64_t>(h) * 64;
  qs[warp][lane] = q[base + i * rs + lane];
  qs[warp][lane + 32] = q[base + i * rs + lane + 32];
  __syncwarp();
  const int lo = max(0, i - W + 1);
  float m = -INFINITY, l = 0.f, acc0 = 0.f, acc1 = 0.f;
  for (int j0 = lo; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j <= i) {
      const float4* kr = reinterpret_cast<const float4*>(k + base + j * rs);
      float dot = 0.f;
#pragma unroll
      for (int d4 = 0; d4 < 16; ++d4) {
        const float4 kv = kr[d4];
        dot = fmaf(qs[warp][4 * d4], kv.x, dot);
        dot = fmaf(qs[warp][4 * d4 + 1], kv.y, dot);
        dot = fmaf(qs[warp][4 * d4 + 2], kv.z, dot);
        dot = fmaf(qs[warp][4 * d4 + 3], kv.w, dot);
      }
      s = dot * scale;
    }
    float cmax = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
    const float m_new = fmaxf(m, cmax);
    const float p = (j <= i) ? expf(s - m_new) : 0.f;
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    float psum = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * alpha + psum;
    acc0 *= alpha;
    acc1 *= alpha;
    const int nj = min(32, i - j0 + 1);
    for (int jj = 0; jj < nj; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const float2 vv = reinterpret_cast<const float2*>(v + base + (j0 + jj) * rs)[lane];
      acc0 = fmaf(pj, vv.x, acc0);
      acc1 = fmaf(pj, vv.y, acc1);
    }
    m = m_new;
  }
  reinterpret_cast<float2*>(o + base + i * rs)[lane] = make_float2(acc0 / l, acc1 / l);
}

// ------------------------------------------------------------------ RoPE --
struct RopeArgs {
  float hi[32];
  float lo[32];
};

template <bool BF16>
__global__ void rope_kernel(const void* __restrict__ x, void* __restrict__ y, int64_t rows, int T, int H,
                            int64_t pos0, const __grid_constant__ RopeArgs f) {
  pdl_wait();
  pdl_trigger();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = rows * H * 32;
  if (idx >= total) return;
  const int m = static_cast<int>(idx & 31);
  const int64_t rh = idx >> 5;          // (row, head)
  const int64_t row = rh / H;
  const int t = static_cast<int>(row % T);
  float s, c;
  rope_sincos(static_cast<float>(pos0 + t), f.hi[m], f.lo[m], &s, &c);
  const int64_t e = rh * 64 + m;
  if constexpr (BF16) {
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    uint16_t* ys = static_cast<uint16_t*>(y);
    const float u = bf16_to_f(xs[e]), w = bf16_to_f(xs[e + 32]);
    const __nv_bfloat16 r1 = __float2bfloat16_rn(u * c - w * s);
    const __nv_bfloat16 r2 = __float2bfloat16_rn(w * c + u * s);
    ys[e] = *reinterpret_cast<const uint16_t*>(&r1);
    ys[e + 32] = *reinterpret_cast<const uint16_t*>(&r2);
  } else {
    const float* xs = static_cast<const float*>(x);
    float* ys = static_cast<float*>(y);
    const float u = xs[e], w = xs[e + 32];
    ys[e] = u * c - w * s;
    ys[e + 32] = w * c + u * s;
  }
}

}  // namespace

bool tmap_attn_operand(CUtensorMap* map, const void* base, int B, int T, int H, int64_t row_stride,
                       int64_t batch_stride) {
  const uint64_t dims[4] = {64, static_cast<uint64_t>(H), static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
  const uint64_t strides[3] = {128, static_cast<uint64_t>(row_stride) * 2, static_cast<uint64_t>(batch_stride) * 2};
  const uint32_t box[4] = {64, 1, 128, 1};
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_attn_bf16(const Launch& L, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const AttnArgs& a) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(swa_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const dim3 grid((a.T + 127) / 128, a.H, a.B);
  return launch_kernel(swa_attn_tc_kernel, grid, dim3(kAttnThreads), kAttnSmem, L.stream, tmQ, tmK, tmV, a);
}

cudaError_t launch_attn_f32(const Launch& L, const float* q, const float* k, const float* v, float* o,
                            int B, int T, int H, int window, float scale) {
  const dim3 grid((T + 3) / 4, H, B);
  return launch_kernel(swa_attn_f32_kernel, grid, dim3(128), 0, L.stream, q, k, v, o, T, H, window, scale);
}

cudaError_t launch_rope(const Launch& L, const void* x, void* y, bool bf16, int B, int T, int H,
                        int64_t pos0, float theta) {
  RopeArgs f;
  for (int m = 0; m < 32; ++m) {
    const double inv = std::pow(static_cast<double>(theta), -2.0 * m / 64.0);
    f.hi[m] = static_cast<float>(inv);
    f.lo[m] = static_cast<float>(inv - static_cast<double>(f.hi[m]));
  }
  const int64_t rows = static_cast<int64_t>(B) * T;
  const int64_t total = rows * H * 32;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (bf16)
    return launch_kernel(rope_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, L.stream, x, y,
                         rows, T, H, pos0, f);
  return launch_kernel(rope_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, L.stream, x, y,
                       rows, T, H, pos0, f);
}

}  // namespace vx
