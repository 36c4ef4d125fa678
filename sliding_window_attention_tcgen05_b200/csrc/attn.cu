// attn.cu -- causal sliding-window attention kernels.
//
// swa_attn_tc_kernel: flash-style bf16 attention on tcgen05 tensor cores.
//   One CTA per (128-query tile, head, clip); its key tiles alternate between
//   two softmax warpgroups (each with its own running max / sum / output,
//   merged at the end) so that one warpgroup's exponentials overlap the other
//   warpgroup's tensor-core products.  Only the key tiles that meet the causal
//   window (i - W, i] of some query are visited; the masks are evaluated only
//   on the edge tiles.  K/V tiles arrive
//   by TMA into a 3-stage ring; S = Q K^T and O_j = P_j V_j accumulate in
//   TMEM; the softmax warps read S from TMEM (two passes: max, then
//   exponentials), keep the running max / sum in registers, write P (bf16) to
//   shared memory as the A operand of the P V product, and fold each O_j into
//   a register accumulator with the online-softmax rescale.
// swa_attn_f32_kernel: fp32 CUDA-core reference-precision path (one warp per
//   query row), used for fp32 inputs.
// rope_kernel: RoPE pre-pass for vx_swa_attn_fwd on raw q, k.
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kAttnThreads = 320;           // 2 softmax warpgroups, TMA warp, MMA warp
constexpr int kNS = 3;                      // K/V pipeline stages
constexpr int kTile = 128 * 64 * 2;         // one 128 x 64 bf16 tile
constexpr int kPBytes = 128 * 128 * 2;      // one P tile (128 queries x 128 keys)
constexpr int kAttnSmem = kTile * (2 + 2 * kNS) + 2 * kPBytes + 1024 + 512;   // Q slot 2 spare
constexpr uint32_t kTmemCols = 512;

// Max / sum of 32 values as a balanced tree (short dependency chains).
__device__ __forceinline__ float tree_max32(const float (&v)[32]) {
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i] = fmaxf(v[i], v[i + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
  return t[0];
}

// One CTA per (128-query tile, head, clip).  The key tiles of 128 that meet
// the tile's causal window are split between two softmax warpgroups: tile u
// goes to warpgroup X = u % 2, which keeps its own online-softmax state for
// the same 128 rows; the two states are merged at the end.  The MMA warp
// issues in key-tile order -- S(0), S(1), PV(0), S(2), PV(1), ... -- so one
// warpgroup's exponentials overlap the other's products.
// TMEM columns: S_X at 128 X, O_X double buffer at 256 + 128 X + 64 j.
// Warps 0-3 / 4-7: warpgroups X = 0 / 1 (TMEM lane = query row), warp 8: TMA,
// warp 9: MMA.  K/V tiles arrive by TMA into a 3-stage ring.
__global__ void __launch_bounds__(kAttnThreads, 1)
swa_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 2 * kTile;             // (second Q slot unused)
  uint8_t* sV = sK + kNS * kTile;
  uint8_t* sP = sV + kNS * kTile;           // P_0 | P_1
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kPBytes);
  constexpr int QF = 0, KF = 1, VF = KF + kNS, KVE = VF + kNS, SF = KVE + kNS, SE = SF + 2, PF = SE + 2,
                PE = PF + 2, OF = PE + 2, OE = OF + 4, DR = OE + 4, NBAR = DR + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int W = a.window;
  const int T = a.T;
  const int kt0 = max(0, q0 - W + 1) / 128;
  const int n = min(T - 1, q0 + 127) / 128 - kt0 + 1;   // key tiles of this query tile

  if (threadIdx.x == 0) {
    mbar_init(bar(QF), 1);
    for (int s = 0; s < kNS; ++s) { mbar_init(bar(KF + s), 1); mbar_init(bar(VF + s), 1); mbar_init(bar(KVE + s), 1); }
    for (int X = 0; X < 2; ++X) {
      mbar_init(bar(SF + X), 1); mbar_init(bar(SE + X), 128);
      mbar_init(bar(PF + X), 128); mbar_init(bar(PE + X), 1);
      for (int j = 0; j < 2; ++j) { mbar_init(bar(OF + 2 * X + j), 1); mbar_init(bar(OE + 2 * X + j), 128); }
    }
    mbar_init(bar(DR), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  pdl_wait();
  pdl_trigger();

  if (warp == 8) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(QF), kTile);
      tma_load_4d(smem_addr(sQ), &tmQ, bar(QF), 0, h, q0, b);
      uint32_t last_par = 0;
      int filled = 0;
      for (int u = 0; u < n; ++u) {
        const int st = u % kNS;
        const uint32_t ph = (u / kNS) & 1;
        if (!mbar_wait(bar(KVE + st), ph ^ 1, wc, 11)) break;
        const int key0 = (kt0 + u) * 128;
        mbar_arrive_expect_tx(bar(KF + st), kTile);
        tma_load_4d(smem_addr(sK + st * kTile), &tmK, bar(KF + st), 0, h, key0, b);
        mbar_arrive_expect_tx(bar(VF + st), kTile);
        tma_load_4d(smem_addr(sV + st * kTile), &tmV, bar(VF + st), 0, h, key0, b);
        last_par = (last_par & ~(1u << st)) | (ph << st);
        filled = u + 1;
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
  } else if (warp == 9) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, 1);
      bool ok = mbar_wait(bar(QF), 0, wc, 13);
      const uint32_t qa = smem_addr(sQ);
      // S(u) -> S_{u%2}: tile u is the (u/2)-th of its warpgroup.
      auto issue_s = [&](int u) -> bool {
        const int X = u & 1, j = u >> 1, st = u % kNS;
        if (!mbar_wait(bar(SE + X), (j & 1) ^ 1, wc, 17)) return false;
        if (!mbar_wait(bar(KF + st), (u / kNS) & 1, wc, 18)) return false;
        tc_fence_after();
        const uint32_t ka = smem_addr(sK + st * kTile);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem + X * 128, smem_desc_sw128(qa + 32 * k, 16, 1024), smem_desc_sw128(ka + 32 * k, 16, 1024),
                    idesc_s, k > 0);
        umma_commit(bar(SF + X));
        return true;
      };
      auto issue_pv = [&](int u) -> bool {
        const int X = u & 1, j = u >> 1, st = u % kNS, ob = j & 1;
        if (!mbar_wait(bar(PF + X), j & 1, wc, 14)) return false;
        if (!mbar_wait(bar(VF + st), (u / kNS) & 1, wc, 15)) return false;
        if (!mbar_wait(bar(OE + 2 * X + ob), ((j >> 1) & 1) ^ 1, wc, 16)) return false;
        tc_fence_after();
        const uint32_t pa = smem_addr(sP + X * kPBytes);
        const uint32_t va = smem_addr(sV + st * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(pa + (k >> 2) * (kPBytes / 2) + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(va + k * 2048, kTile, 1024);
          umma_bf16(tmem + 256 + X * 128 + ob * 64, ad, bd, idesc_o, k > 0);
        }
        umma_commit(bar(OF + 2 * X + ob));
        umma_commit(bar(PE + X));
        umma_commit(bar(KVE + st));   // K/V tile u: its S and PV products are the last users
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int u = 0; ok && u < n; ++u) {
        ok = issue_pv(u);
        if (ok && u + 2 < n) ok = issue_s(u + 2);
      }
      umma_commit(bar(DR));
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(DR), 0, dw, 19);
    }
  } else {
    // ------------- softmax: warpgroup X takes key tiles X, X + 2, ...; thread r owns row q0 + r
    const int X = warp >> 2;
    const int r = threadIdx.x & 127;
    const int i = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + X * 128 + lane_off;
    const uint32_t tO = tmem + 256 + X * 128 + lane_off;
    const float sl2 = a.scale_log2;
    float o[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) o[d] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, mu_o = -INFINITY, mu0 = 0.f, mu1 = 0.f;
    bool ok = true;
    const int nX = (n + 1 - X) / 2;   // tiles u = X, X + 2, ... < n

    auto consume_o = [&](int jj) -> bool {
      const int ob = jj & 1;
      bool w = mbar_wait(bar(OF + 2 * X + ob), (jj >> 1) & 1, wc, 20);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tO + ob * 64, r0);
      tmem_ld32(tO + ob * 64 + 32, r1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(OE + 2 * X + ob));
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

    for (int j = 0; j < nX; ++j) {
      const int key0 = (kt0 + X + 2 * j) * 128;
      bool w = mbar_wait(bar(SF + X), j & 1, wc, 21);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      // Edge tile: some (row, key) pair of the tile is outside (i - W, i].
      const bool edge = key0 + 127 > q0 || key0 <= q0 + 127 - W;
      // pass 1: row max of the raw scores (masked)
      float smax = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(tS + c * 32, rr);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = __uint_as_float(rr[e]);
          if (edge) {
            const int key = key0 + c * 32 + e;
            if (key > i || key <= i - W) v[e] = -INFINITY;
          }
        }
        smax = fmaxf(smax, tree_max32(v));
      }
      const float m_new = fmaxf(m_run, smax * sl2);
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2_approx(m_run - mu);
      m_run = m_new;
      if (j & 1) mu1 = mu; else mu0 = mu;

      w = mbar_wait(bar(PE + X), (j & 1) ^ 1, wc, 22);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      // pass 2: p = 2^(s * scale_log2 - mu), row sum, P (bf16) into shared memory:
      // row r, 128-byte rows, 16-byte chunk index XOR (r & 7), keys 64.. in the second half.
      float rs = 0.f;
      uint8_t* prow = sP + X * kPBytes + r * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(tS + c * 32, rr);
        tmem_ld_wait();
        if (c == 3) {   // S_X fully read: the next S of this warpgroup may overwrite it
          tc_fence_before();
          mbar_arrive(bar(SE + X));
        }
        float pv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float x = fmaf(__uint_as_float(rr[e]), sl2, -mu);
          if (edge) {
            const int key = key0 + c * 32 + e;
            if (key > i || key <= i - W) x = -INFINITY;
          }
          pv[e] = ex2_approx(x);
        }
        float t[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) t[e] = pv[e] + pv[e + 16];
#pragma unroll
        for (int wdt = 8; wdt >= 1; wdt >>= 1)
#pragma unroll
          for (int e = 0; e < wdt; ++e) t[e] += t[e + wdt];
        rs += t[0];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cc = c * 4 + q;     // 16-byte chunk 0..15 of the row
          const uint32_t off = (cc >> 3) * (kPBytes / 2) + ((((cc & 7) ^ (r & 7))) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(prow + off)),
                       "r"(pack_bf16x2(pv[q * 8 + 0], pv[q * 8 + 1])), "r"(pack_bf16x2(pv[q * 8 + 2], pv[q * 8 + 3])),
                       "r"(pack_bf16x2(pv[q * 8 + 4], pv[q * 8 + 5])), "r"(pack_bf16x2(pv[q * 8 + 6], pv[q * 8 + 7]))
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(PF + X));
      l_run = fmaf(l_run, alpha, rs);
      if (j > 0 && !(ok = consume_o(j - 1))) break;
    }
    if (ok && nX > 0) ok = consume_o(nX - 1);

    // Merge: warpgroup 1 hands (m, l, o) to warpgroup 0 through shared memory
    // (the P buffers are idle now); warpgroup 0 writes the output.
    float* xo = reinterpret_cast<float*>(sP + kPBytes);          // [128][64]
    float* xm = reinterpret_cast<float*>(sP);                    // [128] m, [128] l
    const bool okall = ok;
    if (X == 1) {
      asm volatile("bar.sync 1, 256;" ::: "memory");   // P_1 no longer read by the tensor cores
#pragma unroll
      for (int d = 0; d < 64; ++d) xo[r * 64 + ((d + r) & 63)] = o[d];
      xm[r] = m_run;
      xm[128 + r] = okall ? l_run : 0.f;
      asm volatile("bar.sync 2, 256;" ::: "memory");
    } else {
      asm volatile("bar.sync 1, 256;" ::: "memory");
      asm volatile("bar.sync 2, 256;" ::: "memory");
      const float m1 = xm[r], l1 = xm[128 + r];
      const float M = fmaxf(m_run, m1);
      const float f0 = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - M);
      const float f1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
      const float inv_l = 1.0f / (l_run * f0 + l1 * f1);
      if (ok && i < T) {
        uint16_t* dst = static_cast<uint16_t*>(a.out) + static_cast<int64_t>(b) * a.o_batch +
                        static_cast<int64_t>(i) * a.o_row + static_cast<int64_t>(h) * a.o_head;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = 8 * c + e;
            v[e] = (o[d] * f0 + xo[r * 64 + ((d + r) & 63)] * f1) * inv_l;
          }
          st_global_v4(dst + 8 * c, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
        }
      }
    }
  }

  __syncthreads();
  if (warp == 9) {
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

// table[t][m] = (cos, sin) of (pos0 + t) * inv_freq_m, t < T, m < 32.
__global__ void rope_table_kernel(float2* __restrict__ table, int T, int64_t pos0, const __grid_constant__ RopeArgs f) {
  pdl_wait();
  pdl_trigger();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * 32) return;
  const int t = idx >> 5, m = idx & 31;
  float sn, cs;
  rope_sincos(static_cast<float>(pos0 + t), f.hi[m], f.lo[m], &sn, &cs);
  table[idx] = make_float2(cs, sn);
}

// Rotates q and k ([B, T, H, 64]) into qr and kr with the table: thread
// handles pairs (m, m + 32) for 8 consecutive m of one (tensor, row, head).
template <bool BF16>
__global__ void rope_apply_kernel(const void* __restrict__ q, const void* __restrict__ k, void* __restrict__ qr,
                                  void* __restrict__ kr, const float2* __restrict__ table, int64_t rows, int T, int H) {
  pdl_wait();
  pdl_trigger();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per = rows * H * 4;          // per tensor: (row, head, 8-pair group)
  if (idx >= 2 * per) return;
  const int which = idx >= per;
  const int64_t j = which ? idx - per : idx;
  const int g = static_cast<int>(j & 3);      // m = 8 g .. 8 g + 7
  const int64_t rh = j >> 2;
  const int t = static_cast<int>((rh / H) % T);
  const int64_t e = rh * 64 + g * 8;
  const float2* tb = table + t * 32 + g * 8;
  float u[8], w[8];
  if constexpr (BF16) {
    const uint16_t* src = static_cast<const uint16_t*>(which ? k : q);
    const uint4 a = *reinterpret_cast<const uint4*>(src + e);
    const uint4 c = *reinterpret_cast<const uint4*>(src + e + 32);
    u[0] = bf16lo(a.x); u[1] = bf16hi(a.x); u[2] = bf16lo(a.y); u[3] = bf16hi(a.y);
    u[4] = bf16lo(a.z); u[5] = bf16hi(a.z); u[6] = bf16lo(a.w); u[7] = bf16hi(a.w);
    w[0] = bf16lo(c.x); w[1] = bf16hi(c.x); w[2] = bf16lo(c.y); w[3] = bf16hi(c.y);
    w[4] = bf16lo(c.z); w[5] = bf16hi(c.z); w[6] = bf16lo(c.w); w[7] = bf16hi(c.w);
  } else {
    const float* src = static_cast<const float*>(which ? k : q);
#pragma unroll
    for (int i = 0; i < 8; ++i) { u[i] = src[e + i]; w[i] = src[e + 32 + i]; }
  }
  float y1[8], y2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 cs = tb[i];
    y1[i] = u[i] * cs.x - w[i] * cs.y;
    y2[i] = w[i] * cs.x + u[i] * cs.y;
  }
  if constexpr (BF16) {
    uint16_t* dst = static_cast<uint16_t*>(which ? kr : qr);
    *reinterpret_cast<uint4*>(dst + e) = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]),
                                                    pack_bf16x2(y1[4], y1[5]), pack_bf16x2(y1[6], y1[7]));
    *reinterpret_cast<uint4*>(dst + e + 32) = make_uint4(pack_bf16x2(y2[0], y2[1]), pack_bf16x2(y2[2], y2[3]),
                                                         pack_bf16x2(y2[4], y2[5]), pack_bf16x2(y2[6], y2[7]));
  } else {
    float* dst = static_cast<float*>(which ? kr : qr);
#pragma unroll
    for (int i = 0; i < 8; ++i) { dst[e + i] = y1[i]; dst[e + 32 + i] = y2[i]; }
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

cudaError_t launch_rope(const Launch& L, const void* q, const void* k, void* qr, void* kr, void* table, bool bf16,
                        int B, int T, int H, int64_t pos0, float theta) {
  RopeArgs f;
  for (int m = 0; m < 32; ++m) {
    const double inv = std::pow(static_cast<double>(theta), -2.0 * m / 64.0);
    f.hi[m] = static_cast<float>(inv);
    f.lo[m] = static_cast<float>(inv - static_cast<double>(f.hi[m]));
  }
  float2* tb = static_cast<float2*>(table);
  cudaError_t e = launch_kernel(rope_table_kernel, dim3((T * 32 + 255) / 256), dim3(256), 0, L.stream, tb, T, pos0, f);
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(B) * T;
  const int64_t total = 2 * rows * H * 4;
  const dim3 grid(static_cast<unsigned>((total + 255) / 256));
  if (bf16)
    return launch_kernel(rope_apply_kernel<true>, grid, dim3(256), 0, L.stream, q, k, qr, kr,
                         static_cast<const float2*>(tb), rows, T, H);
  return launch_kernel(rope_apply_kernel<false>, grid, dim3(256), 0, L.stream, q, k, qr, kr,
                       static_cast<const float2*>(tb), rows, T, H);
}

}  // namespace vx
