// stream.cu -- the streaming-step kernels over the per-layer ring KV cache.
//
// ring_attn_kernel: one CTA per (head, stream).  The NQ new frames of the
//   stream (positions p .. p+NQ-1, p = pos[s]) attend their causal window:
//   the n_old = min(p, W-1) newest cached frames (ring slots f mod W) plus the
//   new frames themselves.  K/V rows are streamed from HBM with 16-byte
//   loads, 8 lanes per 128-byte row; each 8-lane group keeps an online
//   softmax per query; the groups are merged by warp shuffles, then the
//   eight warps through shared memory.
//   Only after every ring read of the CTA has completed are the NQ new K/V
//   rows written to slots (p + t) mod W (a slot about to be overwritten may
//   still be inside an earlier query's window).  The (stream, head) ring
//   segment is touched by this CTA only, so no other ordering is needed.
// ring_fill_kernel: writes the K/V of the last W frames of a whole-sequence
//   forward into the ring (streaming prefill).
// pos_add_kernel: pos[s] += n (or = n).
#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kRingThreads = 256;
constexpr int kGroups = kRingThreads / 8;   // 8-lane groups per CTA

template <int NQ>
__global__ void __launch_bounds__(kRingThreads, 2)
ring_attn_kernel(const uint16_t* __restrict__ qkv, int64_t ld_qkv, int HD,
                 uint16_t* __restrict__ ring_k, uint16_t* __restrict__ ring_v,
                 const int64_t* __restrict__ pos, int H, int W, uint16_t* __restrict__ out,
                 float scale_log2) {
  constexpr int kWarps = kRingThreads / 32;
  __shared__ float sm_m[kWarps][NQ];
  __shared__ float sm_l[kWarps][NQ];
  __shared__ float sm_o[kWarps][NQ][64];

  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x;
  const int sub = tid & 7;         // dims sub*8 .. sub*8+7
  const int64_t p = pos[s];
  const int n_old = static_cast<int>(p < W - 1 ? p : W - 1);
  const int total = n_old + NQ;
  const int64_t seg = (static_cast<int64_t>(s) * H + h) * W * 64;   // ring segment of (s, h)
  const uint16_t* rk = ring_k + seg;
  const uint16_t* rv = ring_v + seg;
  const uint16_t* qbase = qkv + static_cast<int64_t>(s) * NQ * ld_qkv + h * 64 + sub * 8;

  float q[NQ][8];
#pragma unroll
  for (int qi = 0; qi < NQ; ++qi) {
    const uint4 w = *reinterpret_cast<const uint4*>(qbase + qi * ld_qkv);
    q[qi][0] = bf16lo(w.x) * scale_log2; q[qi][1] = bf16hi(w.x) * scale_log2;
    q[qi][2] = bf16lo(w.y) * scale_log2; q[qi][3] = bf16hi(w.y) * scale_log2;
    q[qi][4] = bf16lo(w.z) * scale_log2; q[qi][5] = bf16hi(w.z) * scale_log2;
    q[qi][6] = bf16lo(w.w) * scale_log2; q[qi][7] = bf16hi(w.w) * scale_log2;
  }
  float m[NQ], l[NQ], o[NQ][8];
#pragma unroll
  for (int qi = 0; qi < NQ; ++qi) {
    m[qi] = -INFINITY; l[qi] = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) o[qi][d] = 0.f;
  }

  // The first old frame is p - n_old; key index kk is frame f0 + kk.  Each
  // 8-lane group takes kU keys per iteration (kk = kb + gw + 32u), issuing all
  // their K/V loads before any math so that 2 * kU 16-byte loads per lane are
  // in flight.  Every lane of a warp runs the same number of iterations (the
  // shuffles are warp-collective); keys past the end are masked.
  constexpr int kU = 4;
  const int64_t f0 = p - n_old;
  const int f0_slot = static_cast<int>(f0 % W);
  const int warp_id = tid >> 5;
  const int gw = (tid >> 3) & 3;           // group within the warp
  for (int kb = warp_id * 4; kb < total; kb += kGroups * kU) {
    uint4 kw[kU], vw[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int kk = kb + gw + kGroups * u;
      kw[u] = make_uint4(0, 0, 0, 0);
      vw[u] = make_uint4(0, 0, 0, 0);
      if (kk < total) {
        const uint16_t* krow;
        const uint16_t* vrow;
        if (kk < n_old) {
          const int slot = (f0_slot + kk) % W;
          krow = rk + static_cast<int64_t>(slot) * 64;
          vrow = rv + static_cast<int64_t>(slot) * 64;
        } else {
          const int t = kk - n_old;
          krow = qkv + (static_cast<int64_t>(s) * NQ + t) * ld_qkv + HD + h * 64;
          vrow = krow + HD;
        }
        kw[u] = ld_global_cs_v4(krow + sub * 8);
        vw[u] = ld_global_cs_v4(vrow + sub * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int kk = kb + gw + kGroups * u;
      const float kf[8] = {bf16lo(kw[u].x), bf16hi(kw[u].x), bf16lo(kw[u].y), bf16hi(kw[u].y),
                           bf16lo(kw[u].z), bf16hi(kw[u].z), bf16lo(kw[u].w), bf16hi(kw[u].w)};
      float sc[NQ];
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = fmaf(q[qi][e], kf[e], d);
        sc[qi] = d;
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) sc[qi] += __shfl_xor_sync(0xffffffffu, sc[qi], off);
      }
      if (kk >= total) continue;
      const float vf[8] = {bf16lo(vw[u].x), bf16hi(vw[u].x), bf16lo(vw[u].y), bf16hi(vw[u].y),
                           bf16lo(vw[u].z), bf16hi(vw[u].z), bf16lo(vw[u].w), bf16hi(vw[u].w)};
      const int64_t f = f0 + kk;   // absolute frame of this key
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        const int64_t fq = p + qi;
        if (f > fq || f <= fq - W) continue;   // outside the causal window of query qi
        const float m_new = fmaxf(m[qi], sc[qi]);
        const float alpha = ex2_approx(m[qi] - m_new);
        const float pr = ex2_approx(sc[qi] - m_new);
        l[qi] = fmaf(l[qi], alpha, pr);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[qi][e] = fmaf(o[qi][e], alpha, pr * vf[e]);
        m[qi] = m_new;
      }
    }
  }

  // Merge the four 8-lane groups of each warp (lanes differing in bits 3, 4) ...
#pragma unroll
  for (int off = 8; off < 32; off <<= 1) {
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[qi], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[qi], off);
      const float M = fmaxf(m[qi], mo);
      const float as = (m[qi] == -INFINITY) ? 0.f : ex2_approx(m[qi] - M);
      const float ao = (mo == -INFINITY) ? 0.f : ex2_approx(mo - M);
      l[qi] = l[qi] * as + lo * ao;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[qi][e], off);
        o[qi][e] = o[qi][e] * as + oo * ao;
      }
      m[qi] = M;
    }
  }
  // ... then the eight warps through shared memory.
  const int warp = tid >> 5;
  if ((tid & 31) < 8) {
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      if (sub == 0) { sm_m[warp][qi] = m[qi]; sm_l[warp][qi] = l[qi]; }
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_o[warp][qi][sub * 8 + e] = o[qi][e];
    }
  }
  __syncthreads();   // also orders every ring read of this CTA before the writes below
  for (int idx = tid; idx < NQ * 64; idx += kRingThreads) {
    const int qi = idx >> 6, d = idx & 63;
    float M = -INFINITY;
    for (int g = 0; g < kWarps; ++g) M = fmaxf(M, sm_m[g][qi]);
    float Lsum = 0.f, acc = 0.f;
    for (int g = 0; g < kWarps; ++g) {
      const float mg = sm_m[g][qi];
      if (mg == -INFINITY) continue;
      const float w = ex2_approx(mg - M);
      Lsum = fmaf(sm_l[g][qi], w, Lsum);
      acc = fmaf(sm_o[g][qi][d], w, acc);
    }
    const __nv_bfloat16 r = __float2bfloat16_rn(acc / Lsum);
    out[(static_cast<int64_t>(s) * NQ + qi) * HD + h * 64 + d] = *reinterpret_cast<const uint16_t*>(&r);
  }
  // Append the new frames: slot (p + t) mod W.
  if (tid < NQ * 16) {
    const int t = tid >> 4;
    const int part = (tid >> 3) & 1;   // 0: K, 1: V
    const int c = tid & 7;
    const uint16_t* src = qkv + (static_cast<int64_t>(s) * NQ + t) * ld_qkv + (1 + part) * HD + h * 64 + c * 8;
    const int dslot = static_cast<int>((p + t) % W);
    uint16_t* dst = (part ? ring_v : ring_k) + seg + static_cast<int64_t>(dslot) * 64 + c * 8;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

// Grid (frames, S); 256 threads cover H heads x 8 chunks of 16 bytes x {K, V}.
__global__ void ring_fill_kernel(const uint16_t* __restrict__ qkv, int64_t ld_qkv, int HD,
                                 uint16_t* __restrict__ ring_k, uint16_t* __restrict__ ring_v,
                                 int T, int H, int W, int first) {
  pdl_wait();
  pdl_trigger();
  const int f = first + blockIdx.x;
  const int s = blockIdx.y;
  const int slot = f % W;
  const uint16_t* row = qkv + (static_cast<int64_t>(s) * T + f) * ld_qkv;
  for (int idx = threadIdx.x; idx < H * 16; idx += blockDim.x) {
    const int h = idx >> 4;
    const int part = (idx >> 3) & 1;
    const int c = idx & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(row + (1 + part) * HD + h * 64 + c * 8);
    uint16_t* dst = (part ? ring_v : ring_k) + ((static_cast<int64_t>(s) * H + h) * W + slot) * 64 + c * 8;
    *reinterpret_cast<uint4*>(dst) = v;
  }
}

__global__ void pos_add_kernel(int64_t* pos, int S, int64_t n, int set) {
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s < S) pos[s] = set ? n : pos[s] + n;
}

template <int NQ>
cudaError_t launch_ring_nq(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD, uint16_t* rk,
                           uint16_t* rv, const int64_t* pos, int S, int H, int W, uint16_t* out, float sl2) {
  return launch_kernel(ring_attn_kernel<NQ>, dim3(H, S), dim3(kRingThreads), 0, L.stream, qkv, ld_qkv, HD, rk, rv,
                       pos, H, W, out, sl2);
}

}  // namespace

cudaError_t launch_ring_attn(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD,
                             uint16_t* ring_k, uint16_t* ring_v, const int64_t* pos, int S, int H,
                             int W, int n_new, uint16_t* out, float scale_log2) {
  switch (n_new) {
    case 1: return launch_ring_nq<1>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 2: return launch_ring_nq<2>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 3: return launch_ring_nq<3>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 4: return launch_ring_nq<4>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 5: return launch_ring_nq<5>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 6: return launch_ring_nq<6>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 7: return launch_ring_nq<7>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    case 8: return launch_ring_nq<8>(L, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_ring_fill(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD, uint16_t* ring_k,
                             uint16_t* ring_v, int S, int T, int H, int W) {
  const int first = T > W ? T - W : 0;
  const int nf = T - first;
  if (nf <= 0 || S <= 0) return cudaSuccess;
  return launch_kernel(ring_fill_kernel, dim3(nf, S), dim3(256), 0, L.stream, qkv, ld_qkv, HD, ring_k, ring_v, T, H,
                       W, first);
}

cudaError_t launch_pos_add(const Launch& L, int64_t* pos, int S, int64_t n, bool set) {
  return launch_kernel(pos_add_kernel, dim3((S + 127) / 128), dim3(128), 0, L.stream, pos, S, n, set ? 1 : 0);
}

}  // namespace vx
