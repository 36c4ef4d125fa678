// stream.cu -- the streaming-step kernels over the per-layer ring KV cache.
//
// ring_attn_tma_kernel: one CTA per (head, stream).  The NQ new frames of the
//   stream (positions p .. p+NQ-1, p = pos[s]) attend their causal window:
//   the cached frames still inside it (ring slot f mod W) plus the new frames
//   themselves.  The kernel is bound by HBM (each (stream, head) reads 192 KB
//   of K/V for 4 query rows); K/V chunks arrive by TMA and the dot products
//   run on mma.sync fragments, which keeps the instruction count per key far
//   below the load time (tcgen05's M >= 64 tiles would be almost all padding
//   for 4 rows).  Only after every ring read of the CTA has completed are the
//   NQ new K/V rows written to slots (p + t) mod W (a slot about to be
//   overwritten may still be inside an earlier query's window).  The
//   (stream, head) ring segment is touched by this CTA only, so no other
//   ordering is needed.
// ring_fill_kernel: writes the K/V of the last W frames of a whole-sequence
//   forward into the ring (streaming prefill).
// pos_add_kernel: pos[s] += n (or = n).
#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kChunk = 64;                 // keys per pipeline stage
constexpr int kStageBytes = 2 * kChunk * 128;   // K and V rows of one chunk (8 KB each)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte column c of row r in a 128-byte-row tile, XOR-swizzled
// so that eight rows at the same column hit eight different bank groups.
__device__ __forceinline__ uint32_t swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

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

// ---------------------------------------------------------------------------
// ring_attn_tma_kernel: the same step with the ring read by TMA.  Softmax is a
// set operation, so the ring is walked in slot order instead of time order:
// every chunk of 64 slots is then one contiguous, 8-row-aligned block of the
// (stream, head) segment, fetched by a single TMA tile load (128-byte swizzle,
// the layout the ldmatrix addressing below expects) issued by a producer warp;
// the four consumer warps wait on mbarriers instead of a CTA barrier per chunk.
// Slot j holds frame f = p - W + d, d = (j - p) mod W, when f >= 0; it is a key
// of new frame p + r iff d >= r + 1 (i.e. f > p + r - W).  The NQ new frames
// are attended by warp 0 in one extra 16-key block read from the qkv rows.
constexpr int kRingTmaThreads = 160;   // 4 consumer warps + 1 TMA producer warp
// Three 16 KB stages (54.5 KB of shared memory) let four CTAs share an SM
// (86 registers also allow four).  Measured on the 64-stream, 32-layer step:
// the kernel is bound by how many CTAs run at once more than by the stages in
// flight per CTA (3 / 4 / 6 / 8 stages = 4 / 3 / 2 / 1 CTAs per SM: 75.5 /
// 76.2 / 92.4 / 154 us; 2 stages, still 4 CTAs per SM: 78.2 us).
constexpr int kRingTmaStages = 3;
constexpr int kRingTmaSmem = 1024 + kRingTmaStages * kStageBytes + 2 * 16 * 128 + 256;

template <int NQ>
__global__ void __launch_bounds__(kRingTmaThreads)
ring_attn_tma_kernel(const __grid_constant__ CUtensorMap tmRK, const __grid_constant__ CUtensorMap tmRV,
                     const uint16_t* __restrict__ qkv, int64_t ld_qkv, int HD, uint16_t* __restrict__ ring_k,
                     uint16_t* __restrict__ ring_v, const int64_t* __restrict__ pos, int H, int W,
                     uint16_t* __restrict__ out, float scale_log2, DevStatus* status, uint64_t limit_ns) {
  static_assert(NQ >= 1 && NQ <= 8, "1..8 new frames");
  constexpr int S = kRingTmaStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage_base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* newb = stage_base + S * kStageBytes;                 // new K rows [16][128 B] | new V rows [16][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(newb + 2 * 16 * 128);   // full[S], empty[S]
  int* abort_flag = reinterpret_cast<int*>(bars + 2 * S);
  // merge buffers reuse the stage memory once every chunk has been consumed
  float* sm_m = reinterpret_cast<float*>(stage_base);          // [4 warps][8]
  float* sm_l = sm_m + 4 * 8;                                   // [4][8]
  float* sm_o = sm_l + 4 * 8;                                   // [4][8][64]

  const int h = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  auto full = [&](int i) { return smem_addr(bars + i); };
  auto empty = [&](int i) { return smem_addr(bars + S + i); };
  if (tid == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(full(i), 1); mbar_init(empty(i), 4); }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) { tma_prefetch_desc(&tmRK); tma_prefetch_desc(&tmRV); }
  __syncthreads();
  const WaitCtx wc{status, abort_flag, limit_ns};
  pdl_wait();
  pdl_trigger();

  const int64_t p = pos[s];
  const int nslots = static_cast<int>(p < W ? p : W);          // slots that can hold a cached frame
  const int nchunks = (nslots + kChunk - 1) / kChunk;
  const int64_t seg_row = (static_cast<int64_t>(s) * H + h) * W;
  const int pmod = static_cast<int>(p % W);
  const uint16_t* newk = qkv + static_cast<int64_t>(s) * NQ * ld_qkv + HD + h * 64;

  if (warp == 4) {
    if (lane == 0) {
      uint32_t last_par = 0;
      int filled = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % S;
        const uint32_t ph = (c / S) & 1;
        if (!mbar_wait(empty(st), ph ^ 1, wc, 41)) break;
        mbar_arrive_expect_tx(full(st), kStageBytes);
        const uint32_t kb = smem_addr(stage_base + st * kStageBytes);
        const int row = static_cast<int>(seg_row + static_cast<int64_t>(c) * kChunk);
        tma_load_2d(kb, &tmRK, full(st), 0, row);
        tma_load_2d(kb + kChunk * 128, &tmRV, full(st), 0, row);
        last_par = (last_par & ~(1u << st)) | (ph << st);
        filled = c + 1;
      }
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int st = 0; st < S && st < filled; ++st) mbar_wait(full(st), (last_par >> st) & 1u, dw, 42);
    }
    __syncthreads();   // the merge barrier below
    return;
  }

  // Q as the A operand (rows = queries, zero beyond NQ), 4 k-steps of 16 dims.
  const int qrow = lane >> 2;             // this lane's query row (c0/c1); c2/c3 are rows + 8 (padding)
  const int qcol = (lane & 3) * 2;
  uint32_t qa[4][2];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    qa[ks][0] = 0; qa[ks][1] = 0;
    if (qrow < NQ) {
      const uint16_t* qr = qkv + (static_cast<int64_t>(s) * NQ + qrow) * ld_qkv + h * 64 + ks * 16 + qcol;
      qa[ks][0] = *reinterpret_cast<const uint32_t*>(qr);
      qa[ks][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
    }
  }
  // Warp 0 stages the NQ new K/V rows (zeros beyond) for the extra block.
  if (warp == 0) {
    for (int idx = lane; idx < 2 * 16 * 8; idx += 32) {
      const int part = idx >> 7, r = (idx >> 3) & 15, col = idx & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < NQ) v = *reinterpret_cast<const uint4*>(newk + static_cast<int64_t>(r) * ld_qkv + part * HD + col * 8);
      *reinterpret_cast<uint4*>(newb + part * 16 * 128 + swz(r, col)) = v;
    }
    __syncwarp();
  }

  float o[8][4];
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;   // row qrow: running max; this lane's share of the row sum

  // One 16-key block: S = Q K^T (keys at kb rows r0 ..), mask via valid(key e),
  // online softmax, O += P V (V rows at vb rows r0 ..).
  auto block = [&](uint32_t kb, uint32_t vb, int r0, auto&& valid) {
    float sacc[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      sacc[nb][0] = sacc[nb][1] = sacc[nb][2] = sacc[nb][3] = 0.f;
      const int krow = r0 + nb * 8 + (lane & 7);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz(krow, half * 4 + (lane >> 3)), b0, b1, b2, b3);
        mma_bf16_16816(sacc[nb], qa[2 * half][0], 0u, qa[2 * half][1], 0u, b0, b1);
        mma_bf16_16816(sacc[nb], qa[2 * half + 1][0], 0u, qa[2 * half + 1][1], 0u, b2, b3);
      }
    }
    float x[2][2];
    float cmax = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = qrow < NQ && valid(nb * 8 + qcol + e);
        x[nb][e] = ok ? sacc[nb][e] * scale_log2 : -INFINITY;
        cmax = fmaxf(cmax, x[nb][e]);
      }
    }
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
    const float m_new = fmaxf(m_run, cmax);
    const float mu = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = ex2_approx(m_run - mu);
    float pr[2][2];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) pr[nb][e] = ex2_approx(x[nb][e] - mu);
    l_part = l_part * alpha + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
    m_run = m_new;
    const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
    const uint32_t pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) { o[nb][0] *= alpha; o[nb][1] *= alpha; }
#pragma unroll
    for (int dc = 0; dc < 8; dc += 2) {
      uint32_t b0, b1, b2, b3;
      const int vrow = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int vcol = dc + (lane >> 4);
      ldsm_x4_t(vb + swz(vrow, vcol), b0, b1, b2, b3);
      mma_bf16_16816(o[dc], pa0, 0u, pa2, 0u, b0, b1);
      mma_bf16_16816(o[dc + 1], pa0, 0u, pa2, 0u, b2, b3);
    }
  };

  const int r0 = warp * 16;               // this warp's 16 slots within each chunk
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % S;
    bool okw = mbar_wait(full(st), (c / S) & 1, wc, 43);
    if (!__all_sync(0xffffffffu, okw)) break;
    const uint32_t kb = smem_addr(stage_base + st * kStageBytes);
    const int slot0 = c * kChunk + r0;
    if (slot0 + 16 > nslots) {
      // Rows past the cached frames (never-written slots, or the next
      // segment's rows) may hold anything: their P is 0, but 0 * NaN is not,
      // so this warp zeroes its V rows there before the product.
      uint8_t* vrows = stage_base + st * kStageBytes + kChunk * 128;
      for (int idx = lane; idx < 16 * 8; idx += 32) {
        const int rr = idx >> 3, col = idx & 7;
        if (slot0 + rr >= nslots) *reinterpret_cast<uint4*>(vrows + swz(r0 + rr, col)) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();   // ordered before the stage's next TMA fill
      __syncwarp();
    }
    block(kb, kb + kChunk * 128, r0, [&](int e) {
      const int slot = slot0 + e;
      int d = slot - pmod;
      if (d < 0) d += W;
      return slot < nslots && d >= qrow + 1 && p - W + d >= 0;
    });
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }
  if (warp == 0) {   // the NQ new frames: key t is seen by query r iff t <= r
    const uint32_t nk = smem_addr(newb);
    block(nk, nk + 16 * 128, 0, [&](int e) { return e < NQ && e <= qrow; });
  }

  // Per warp: full row sums, then merge the four warps through shared memory
  // (the stage memory, free once every consumer warp is past its last chunk).
  float l_row = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_row += __shfl_xor_sync(0xffffffffu, l_row, 2);
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (qrow < NQ) {
    if ((lane & 3) == 0) {
      sm_m[warp * 8 + qrow] = m_run;
      sm_l[warp * 8 + qrow] = l_row;
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      sm_o[(warp * 8 + qrow) * 64 + nb * 8 + qcol] = o[nb][0];
      sm_o[(warp * 8 + qrow) * 64 + nb * 8 + qcol + 1] = o[nb][1];
    }
  }
  __syncthreads();   // also orders every ring read of this CTA (TMA included) before the writes below
  for (int idx = tid; idx < NQ * 64; idx += 128) {
    const int qi = idx >> 6, d = idx & 63;
    float M = -INFINITY;
#pragma unroll
    for (int g = 0; g < 4; ++g) M = fmaxf(M, sm_m[g * 8 + qi]);
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float mg = sm_m[g * 8 + qi];
      if (mg == -INFINITY) continue;
      const float w = ex2_approx(mg - M);
      Lsum = fmaf(sm_l[g * 8 + qi], w, Lsum);
      acc = fmaf(sm_o[(g * 8 + qi) * 64 + d], w, acc);
    }
    const __nv_bfloat16 r = __float2bfloat16_rn(acc / Lsum);
    out[(static_cast<int64_t>(s) * NQ + qi) * HD + h * 64 + d] = *reinterpret_cast<const uint16_t*>(&r);
  }
  // Append the new frames: slot (p + t) mod W.
  const int64_t seg = seg_row * 64;
  for (int idx = tid; idx < NQ * 16; idx += 128) {
    const int t = idx >> 4;
    const int part = (idx >> 3) & 1;   // 0: K, 1: V
    const int c = idx & 7;
    const uint16_t* src = newk + static_cast<int64_t>(t) * ld_qkv + part * HD + c * 8;
    const int dslot = static_cast<int>((p + t) % W);
    uint16_t* dst = (part ? ring_v : ring_k) + seg + static_cast<int64_t>(dslot) * 64 + c * 8;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

template <int NQ>
cudaError_t launch_ring_tma_nq(const Launch& L, const CUtensorMap& tk, const CUtensorMap& tv, const uint16_t* qkv,
                               int64_t ld_qkv, int HD, uint16_t* rk, uint16_t* rv, const int64_t* pos, int S, int H,
                               int W, uint16_t* out, float sl2) {
  return launch_kernel(ring_attn_tma_kernel<NQ>, dim3(H, S), dim3(kRingTmaThreads), kRingTmaSmem, L.stream, tk, tv,
                       qkv, ld_qkv, HD, rk, rv, pos, H, W, out, sl2, L.status, L.limit_ns);
}

}  // namespace

cudaError_t launch_ring_attn(const Launch& L, const uint16_t* qkv, int64_t ld_qkv, int HD,
                             uint16_t* ring_k, uint16_t* ring_v, const int64_t* pos, int S, int H,
                             int W, int n_new, uint16_t* out, float scale_log2) {
  // One layer's ring as [S * H * W rows, 64] bf16 tiles of 64 rows.
  CUtensorMap tk, tv;
  const uint64_t rows = static_cast<uint64_t>(S) * H * W;
  if (!tmap_bf16_2d(&tk, ring_k, 64, rows, 64, kChunk) || !tmap_bf16_2d(&tv, ring_v, 64, rows, 64, kChunk))
    return cudaErrorInvalidValue;
  switch (n_new) {
#define VX_RING_TMA(n) \
  case n: return launch_ring_tma_nq<n>(L, tk, tv, qkv, ld_qkv, HD, ring_k, ring_v, pos, S, H, W, out, scale_log2);
    VX_RING_TMA(1) VX_RING_TMA(2) VX_RING_TMA(3) VX_RING_TMA(4)
    VX_RING_TMA(5) VX_RING_TMA(6) VX_RING_TMA(7) VX_RING_TMA(8)
#undef VX_RING_TMA
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
