// attn.cu -- causal sliding-window attention kernels.
//
// swa_attn_tc_kernel: flash-style bf16 attention on tcgen05 tensor cores.
//   One CTA per (128-query tile, head, clip); its key tiles alternate between
//   two softmax warpgroups (each with its own running max / sum / output,
//   merged at the end) so that one warpgroup's exponentials overlap the other
//   warpgroup's tensor-core products.  Only the key tiles that meet the causal
//   window (i - W, i] of some query are visited; the masks are evaluated only
//   on the edge tiles.  K/V tiles arrive by TMA into a 4-stage ring; S, P and
//   O all live in TMEM (P is the TMEM A operand of the P V product, O is
//   accumulated in place and rescaled lazily).
// swa_attn_f32_kernel: fp32 CUDA-core reference-precision path (one warp per
//   query row), used for fp32 inputs.
// rope_table_kernel / rope_apply_kernel: RoPE pre-pass of vx_swa_attn_fwd on raw
//   q, k (a per-position cos/sin table, then one vectorised rotation pass).
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kAttnThreads = 384;           // 2 softmax warpgroups; TMA, 2 MMA and 1 idle warp
constexpr int kNS = 4;                      // K/V pipeline stages
constexpr int kTile = 128 * 64 * 2;         // one 128 x 64 bf16 tile
constexpr int kAttnSmemPair = kTile * (4 + 2 * kNS) + 1024 + 512;    // + barriers, TMEM slot
constexpr int kAttnSmemSplit = kTile * (2 + 2 * kNS) + 1024 + 4608;  // + barriers, TMEM slot, merge (m, l) x 2
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleSlack = 8.0f;       // O is rescaled only when a row max grows by more than 2^8

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_global_v4(dst + 8 * j, pack_bf16x2(v[8 * j + 0], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                 pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}

// The softmax of a 128-key tile is bound by the softmax warps' instruction
// issue, so the exponent arguments and the row sums use sm_100's packed
// fp32x2 FMA / add (each lane of a packed op rounds like the scalar op, so
// the results are those of the scalar code).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Max of 32 values as a balanced tree (short dependency chains).
__device__ __forceinline__ float tree_max32(const float* v) {
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i] = fmaxf(v[i], v[i + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
  return t[0];
}

// pv[e] = 2^(s[e] * sl2 - mu) for 32 scores, the argument two at a time.
__device__ __forceinline__ void exp2_scaled32(const float* s, float sl2, float mu, float (&pv)[32]) {
  const uint64_t sc = f2_pack(sl2, sl2), nm = f2_pack(-mu, -mu);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float x0, x1;
    f2_unpack(ffma2(f2_pack(s[e], s[e + 1]), sc, nm), x0, x1);
    pv[e] = ex2_approx(x0);
    pv[e + 1] = ex2_approx(x1);
  }
}

// Sum of 32 values as the tree t[e] = v[e] + v[e + 16], then halving; two
// neighbouring nodes of a level per packed add.
__device__ __forceinline__ float sum32_tree(const float (&v)[32]) {
  uint64_t t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = fadd2(f2_pack(v[2 * i], v[2 * i + 1]), f2_pack(v[2 * i + 16], v[2 * i + 17]));
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] = fadd2(t[i], t[i + w]);
  float a, b;
  f2_unpack(t[0], a, b);
  return a + b;
}

// swa_attn_pair_kernel (many work items): one CTA per SM walks pairs of work
// items (128-query tile, head,
// clip); pair p = blockIdx.x + k * gridDim.x holds items 2p and 2p + 1 (query
// tiles fastest: usually two neighbouring query tiles of one head, which share
// most of their key tiles through L2).  Softmax warpgroup X owns item 2p + X
// entirely: it runs the online softmax over all the key tiles of 128 that meet
// its tile's causal window and normalises its own output, so there is no
// merge and the two warpgroups never wait for each other.  Per warpgroup X,
// TMEM holds S_X (128 columns fp32), P_X (64 columns, bf16 pairs) and O_X (64
// columns): the softmax threads copy S_X to registers and release it at once,
// so the next S of the warpgroup (possibly of its next item) is computed while
// they exponentiate; P goes back to TMEM and is the A operand of
// O_X += P_X V; O_X is rescaled in place only when a row's max grows by more
// than kRescaleSlack (the exponents are taken against a stale max otherwise,
// which cancels in O / l).  Each warpgroup has a double-buffered Q; the K/V
// ring carries both items' tiles interleaved (A0, B0, A1, B1, ...) and runs on
// across pairs.
// Warps 0-3 / 4-7: softmax warpgroups 0 / 1 (TMEM lane = query row); warp 8:
// TMA; warps 9 / 10: the tensor-core products of warpgroup 0 / 1; warp 11
// idles.  The softmax warpgroups take most of the register file (setmaxnreg).
constexpr int kSoftmaxRegs = 224;   // 8 softmax warps x 224 + 4 other warps x 56 = 384 x 168 launched
constexpr int kOtherRegs = 56;

struct AttnItem {
  int q0, h, b, kt0, n;   // first query, head, clip, first key tile, key tiles
};
__device__ __forceinline__ AttnItem item_at(const AttnArgs& a, int qt, int h, int b) {
  AttnItem it;
  it.h = h;
  it.b = b;
  it.q0 = qt * 128;
  it.kt0 = max(0, it.q0 - a.window + 1) / 128;
  it.n = min(a.T - 1, it.q0 + 127) / 128 - it.kt0 + 1;
  return it;
}
// Item `item` in query-tile-fastest order.
__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, int item) {
  const int nqt = (a.T + 127) / 128;
  const int r = item / nqt;
  return item_at(a, item % nqt, r % a.H, r / a.H);
}
// Round r of this CTA in the split kernel's order: items sorted heaviest first
// (query tiles in descending order; a tile's key-tile count never decreases
// with its index), dealt to the CTAs round by round in alternating
// directions, which evens out the CTAs' total key tiles.  False past this
// CTA's last item (only the last round can be partial).
__device__ __forceinline__ bool split_item(const AttnArgs& a, int n_items, int r, AttnItem& it) {
  const int G = gridDim.x, x = blockIdx.x;
  const int pos = r * G + ((r & 1) ? G - 1 - x : x);
  if (pos >= n_items) return false;
  const int hb = a.H * a.B;
  const int rest = pos % hb;
  it = item_at(a, (a.T + 127) / 128 - 1 - pos / hb, rest % a.H, rest / a.H);
  return true;
}
// Ring position of tile t of item X in a pair whose items have nA, nB tiles,
// loaded interleaved (A0, B0, A1, B1, ...), then the longer item's rest.
__device__ __forceinline__ int pair_pos(int X, int t, int nA, int nB) {
  const int m = nA < nB ? nA : nB;
  return t < m ? 2 * t + X : m + t;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
swa_attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // Q[X][buffer]: 4 tiles
  uint8_t* sK = sQ + 4 * kTile;
  uint8_t* sV = sK + kNS * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kNS * kTile);
  // QF/QE: [X * 2 + buffer]
  constexpr int QF = 0, QE = 4, KF = 8, VF = KF + kNS, KVE = VF + kNS, SF = KVE + kNS, SE = SF + 2, PF = SE + 2,
                PE = PF + 2, OD = PE + 2, OFREE = OD + 2, DR = OFREE + 2, NBAR = DR + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = ((a.T + 127) / 128) * a.H * a.B;
  const int n_pairs = (n_items + 1) / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) { mbar_init(bar(QF + i), 1); mbar_init(bar(QE + i), 1); }
    for (int s = 0; s < kNS; ++s) { mbar_init(bar(KF + s), 1); mbar_init(bar(VF + s), 1); mbar_init(bar(KVE + s), 1); }
    for (int X = 0; X < 2; ++X) {
      mbar_init(bar(SF + X), 1); mbar_init(bar(SE + X), 128);
      mbar_init(bar(PF + X), 128); mbar_init(bar(PE + X), 1);
      mbar_init(bar(OD + X), 1);
      mbar_init(bar(OFREE + X), 4);
      mbar_init(bar(DR + X), 1);
    }
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

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == 8 && lane == 0) {
      uint32_t last_par = 0, q_issued = 0, q_par = 0;
      int filled = 0;
      int U = 0;   // K/V tiles loaded so far (ring position)
      bool ok = true;
      for (int p = blockIdx.x, k = 0; ok && p < n_pairs; p += gridDim.x, ++k) {
        const int iA = 2 * p;
        const bool hasB = iA + 1 < n_items;
        const AttnItem A = attn_item(a, iA);
        const AttnItem Bi = hasB ? attn_item(a, iA + 1) : A;
        const int nA = A.n, nB = hasB ? Bi.n : 0;
        const int qb = k & 1;
        for (int X = 0; X < (hasB ? 2 : 1); ++X) {
          const AttnItem& it = X ? Bi : A;
          const int qi = X * 2 + qb;
          if (!mbar_wait(bar(QE + qi), ((k >> 1) & 1) ^ 1, wc, 10)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(QF + qi), kTile);
          tma_load_4d(smem_addr(sQ + qi * kTile), &tmQ, bar(QF + qi), 0, it.h, it.q0, it.b);
          q_issued |= 1u << qi;
          q_par = (q_par & ~(1u << qi)) | (((k >> 1) & 1u) << qi);
        }
        const int m = nA < nB ? nA : nB;
        const int total = nA + nB;
        for (int pos = 0; ok && pos < total; ++pos, ++U) {
          // pos -> (item, tile): interleaved while both have tiles, then the longer one
          int X, t;
          if (pos < 2 * m) { X = pos & 1; t = pos >> 1; } else { X = nA > nB ? 0 : 1; t = pos - m; }
          const AttnItem& it = X ? Bi : A;
          const int st = U % kNS;
          const uint32_t ph = (U / kNS) & 1;
          if (!mbar_wait(bar(KVE + st), ph ^ 1, wc, 11)) { ok = false; break; }
          const int key0 = (it.kt0 + t) * 128;
          mbar_arrive_expect_tx(bar(KF + st), kTile);
          tma_load_4d(smem_addr(sK + st * kTile), &tmK, bar(KF + st), 0, it.h, key0, it.b);
          mbar_arrive_expect_tx(bar(VF + st), kTile);
          tma_load_4d(smem_addr(sV + st * kTile), &tmV, bar(VF + st), 0, it.h, key0, it.b);
          last_par = (last_par & ~(1u << st)) | (ph << st);
          filled = U + 1;
        }
      }
      // Bounded wait for every copy still in flight (also after an abort).
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int qi = 0; qi < 4; ++qi)
        if (q_issued & (1u << qi)) mbar_wait(bar(QF + qi), (q_par >> qi) & 1u, dw, 12);
      for (int s = 0; s < kNS && s < filled; ++s) {
        mbar_wait(bar(KF + s), (last_par >> s) & 1u, dw, 12);
        mbar_wait(bar(VF + s), (last_par >> s) & 1u, dw, 12);
      }
    } else if ((warp == 9 || warp == 10) && lane == 0) {
      // Products of warpgroup X = warp - 9: every key tile of its item of each pair.
      const int X = warp - 9;
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, 1);
      int jg = 0;      // this warpgroup's tiles so far (all items)
      int ubase = 0;   // ring position of the current pair's first tile
      int kc = 0;      // this warpgroup's items so far
      bool ok = true;
      for (int p = blockIdx.x, k = 0; ok && p < n_pairs; p += gridDim.x, ++k) {
        const int iA = 2 * p;
        const bool hasB = iA + 1 < n_items;
        const int nA = attn_item(a, iA).n, nB = hasB ? attn_item(a, iA + 1).n : 0;
        const int nX = X ? nB : nA;
        if (nX > 0) {
          const int qi = X * 2 + (k & 1);
          ok = mbar_wait(bar(QF + qi), (k >> 1) & 1, wc, 13);
          const uint32_t qa = smem_addr(sQ + qi * kTile);
          auto issue_s = [&](int j) -> bool {   // S(j) into S_X
            const int U = ubase + pair_pos(X, j, nA, nB), st = U % kNS, g = jg + j;
            if (!mbar_wait(bar(SE + X), (g & 1) ^ 1, wc, 17)) return false;
            if (!mbar_wait(bar(KF + st), (U / kNS) & 1, wc, 18)) return false;
            tc_fence_after();
            const uint32_t ka = smem_addr(sK + st * kTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tmem + X * 256, smem_desc_sw128(qa + 32 * kk, 16, 1024),
                        smem_desc_sw128(ka + 32 * kk, 16, 1024), idesc_s, kk > 0);
            umma_commit(bar(SF + X));
            return true;
          };
          auto issue_pv = [&](int j) -> bool {
            const int U = ubase + pair_pos(X, j, nA, nB), st = U % kNS, g = jg + j;
            if (!mbar_wait(bar(PF + X), g & 1, wc, 14)) return false;
            if (!mbar_wait(bar(VF + st), (U / kNS) & 1, wc, 15)) return false;
            // O_X is overwritten by the item's first product: the warpgroup's
            // previous item must have been read out.
            if (j == 0 && !mbar_wait(bar(OFREE + X), (kc & 1) ^ 1, wc, 16)) return false;
            tc_fence_after();
            const uint32_t va = smem_addr(sV + st * kTile);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 8 TMEM columns of P, 2 K-rows groups of V
              umma_bf16_ts(tmem + X * 256 + 192, tmem + X * 256 + 128 + 8 * kk,
                           smem_desc_sw128(va + kk * 2048, kTile, 1024), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar(PE + X));
            umma_commit(bar(KVE + st));   // K/V tile U: S(U) and PV(U) were its last users
            return true;
          };
          if (ok) ok = issue_s(0);
          for (int j = 0; ok && j < nX; ++j) {
            if (j + 1 < nX) ok = issue_s(j + 1);
            if (ok) ok = issue_pv(j);
          }
          umma_commit(bar(OD + X));    // O_X of this item is final once its products are done
          umma_commit(bar(QE + qi));   // and so is the use of its Q buffer
          jg += nX;
          ++kc;
        }
        ubase += nA + nB;
      }
      umma_commit(bar(DR + X));
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(DR + X), 0, dw, 19);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------- softmax: warpgroup X owns item 2p + X; thread r owns row q0 + r
    const int X = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + X * 256 + lane_off;
    const uint32_t tP = tS + 128;
    const uint32_t tO = tS + 192;
    const float sl2 = a.scale_log2;
    const int W = a.window;
    int jg = 0;   // this warpgroup's tiles so far (all items)
    int kc = 0;   // this warpgroup's items so far
    bool ok = true;

    for (int p = blockIdx.x; ok && p < n_pairs; p += gridDim.x) {
      const int item = 2 * p + X;
      if (item >= n_items) continue;
      const AttnItem it = attn_item(a, item);
      const int q0 = it.q0;
      const int i = q0 + r;
      float m_used = -INFINITY, l_run = 0.f;

      for (int j = 0; j < it.n; ++j, ++jg) {
        const int key0 = (it.kt0 + j) * 128;
        bool w = mbar_wait(bar(SF + X), jg & 1, wc, 21);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        float sv[128];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(r0[e]);
            sv[e + 32] = __uint_as_float(r1[e]);
            sv[e + 64] = __uint_as_float(r2[e]);
            sv[e + 96] = __uint_as_float(r3[e]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(SE + X));      // S_X may be overwritten by the next product
        // Edge tile: keys outside (i - W, i] of this row, i.e. outside columns
        // [lo, hi] of the tile, are masked.
        if (key0 + 127 > q0 || key0 <= q0 + 127 - W) {
          const int lo = i - W + 1 - key0, hi = i - key0;
#pragma unroll
          for (int e = 0; e < 128; ++e) sv[e] = (e >= lo && e <= hi) ? sv[e] : -INFINITY;
        }
        const float m_tile = fmaxf(fmaxf(tree_max32(sv), tree_max32(sv + 32)),
                                   fmaxf(tree_max32(sv + 64), tree_max32(sv + 96))) * sl2;
        // Rescale decision (per row): a first finite max just sets m_used (l and O
        // are still zero); a max more than the slack above m_used rescales.
        float corr = 1.f;
        if (m_tile > m_used + kRescaleSlack) {
          if (m_used != -INFINITY) corr = ex2_approx(m_used - m_tile);
          m_used = m_tile;
        }
        l_run *= corr;
        const float mu = (m_used == -INFINITY) ? 0.f : m_used;

        // P_X and O_X are free once the previous P V product of this warpgroup is done.
        w = mbar_wait(bar(PE + X), (jg & 1) ^ 1, wc, 22);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
          uint32_t o0[32], o1[32];
          tmem_ld32(tO, o0);
          tmem_ld32(tO + 32, o1);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o0[e] = __float_as_uint(__uint_as_float(o0[e]) * corr);
            o1[e] = __float_as_uint(__uint_as_float(o1[e]) * corr);
          }
          tmem_st32(tO, o0);
          tmem_st32(tO + 32, o1);
        }
        // p = 2^(s * scale_log2 - mu), row sum, P (bf16 pairs) into TMEM
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float pv[32];
          exp2_scaled32(sv + c * 32, sl2, mu, pv);
          rs += sum32_tree(pv);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
          tmem_st16(tP + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(PF + X));
        l_run += rs;
      }
      if (!ok) break;

      // Output: O_X / l once the item's last product is done; O_X is then
      // released for the warpgroup's next item.
      bool w = mbar_wait(bar(OD + X), kc & 1, wc, 23);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      uint32_t x0[32], x1[32];
      tmem_ld32(tO, x0);
      tmem_ld32(tO + 32, x1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(OFREE + X));
      ++kc;
      if (i < a.T) {
        const float inv_l = 1.0f / l_run;
        uint16_t* dst = static_cast<uint16_t*>(a.out) + static_cast<int64_t>(it.b) * a.o_batch +
                        static_cast<int64_t>(i) * a.o_row + static_cast<int64_t>(it.h) * a.o_head;
        float v0[32], v1[32];
#pragma unroll
        for (int d = 0; d < 32; ++d) {
          v0[d] = __uint_as_float(x0[d]) * inv_l;
          v1[d] = __uint_as_float(x1[d]) * inv_l;
        }
        store_bf16x32(dst, v0);
        store_bf16x32(dst + 32, v1);
      }
    }
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// swa_attn_split_kernel (few work items): one CTA per SM walks work items
// (128-query tile, head, clip) in the order of split_item (heaviest first,
// alternating directions; with few items, all K/V tiles stay in L2).  Within an item the key tiles
// of 128 that meet the tile's causal window alternate between two softmax
// warpgroups (tile u -> warpgroup u % 2), each keeping its own running max /
// sum / output for the same 128 rows; the two are merged at the end of the
// item.  Per warpgroup X, TMEM holds S_X (128 columns fp32), P_X (64 columns,
// bf16 pairs) and O_X (64 columns): the softmax threads copy S_X to registers
// and release it at once, so the next S of the warpgroup (possibly of the
// next item) is computed while they exponentiate or merge; P goes back to TMEM
// and is the A operand of O_X += P_X V; O_X is rescaled in place only when a
// row's max grows by more than kRescaleSlack (the exponents are taken against
// a stale max otherwise, which cancels in O / l).  Q is double-buffered and
// the K/V ring runs on across items, so the next item's loads and first
// product overlap the current item's merge.
// Warps 0-3 / 4-7: softmax warpgroups 0 / 1 (TMEM lane = query row); warp 8:
// TMA; warps 9 / 10: the tensor-core products of warpgroup 0 / 1; warp 11
// idles.  The softmax warpgroups take most of the register file (setmaxnreg).
__global__ void __launch_bounds__(kAttnThreads, 1)
swa_attn_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // two Q buffers
  uint8_t* sK = sQ + 2 * kTile;
  uint8_t* sV = sK + kNS * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kNS * kTile);
  constexpr int QF = 0, QE = 2, KF = 4, VF = KF + kNS, KVE = VF + kNS, SF = KVE + kNS, SE = SF + 2, PF = SE + 2,
                PE = PF + 2, OD = PE + 2, OFREE = OD + 2, DR = OFREE + 2, NBAR = DR + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* xml = reinterpret_cast<float*>(abort_flag + 3);   // [2 items][2 WG][m 128, l 128]
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = ((a.T + 127) / 128) * a.H * a.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(bar(QF + i), 1); mbar_init(bar(QE + i), 2); }
    for (int s = 0; s < kNS; ++s) { mbar_init(bar(KF + s), 1); mbar_init(bar(VF + s), 1); mbar_init(bar(KVE + s), 1); }
    for (int X = 0; X < 2; ++X) {
      mbar_init(bar(SF + X), 1); mbar_init(bar(SE + X), 128);
      mbar_init(bar(PF + X), 128); mbar_init(bar(PE + X), 1);
      mbar_init(bar(OD + X), 1);
      mbar_init(bar(OFREE + X), 8);
      mbar_init(bar(DR + X), 1);
    }
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

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == 8 && lane == 0) {
      uint32_t last_par = 0, q_issued = 0, q_par = 0;
      int filled = 0;
      int U = 0;   // K/V tiles loaded so far (ring position)
      bool ok = true;
      AttnItem it;
      for (int k = 0; ok && split_item(a, n_items, k, it); ++k) {
        const int qb = k & 1;
        if (!mbar_wait(bar(QE + qb), ((k >> 1) & 1) ^ 1, wc, 10)) break;   // both issuers are done with it
        mbar_arrive_expect_tx(bar(QF + qb), kTile);
        tma_load_4d(smem_addr(sQ + qb * kTile), &tmQ, bar(QF + qb), 0, it.h, it.q0, it.b);
        q_issued |= 1u << qb;
        q_par = (q_par & ~(1u << qb)) | (((k >> 1) & 1u) << qb);
        for (int u = 0; u < it.n; ++u, ++U) {
          const int st = U % kNS;
          const uint32_t ph = (U / kNS) & 1;
          if (!mbar_wait(bar(KVE + st), ph ^ 1, wc, 11)) { ok = false; break; }
          const int key0 = (it.kt0 + u) * 128;
          mbar_arrive_expect_tx(bar(KF + st), kTile);
          tma_load_4d(smem_addr(sK + st * kTile), &tmK, bar(KF + st), 0, it.h, key0, it.b);
          mbar_arrive_expect_tx(bar(VF + st), kTile);
          tma_load_4d(smem_addr(sV + st * kTile), &tmV, bar(VF + st), 0, it.h, key0, it.b);
          last_par = (last_par & ~(1u << st)) | (ph << st);
          filled = U + 1;
        }
      }
      // Bounded wait for every copy still in flight (also after an abort).
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int qb = 0; qb < 2; ++qb)
        if (q_issued & (1u << qb)) mbar_wait(bar(QF + qb), (q_par >> qb) & 1u, dw, 12);
      for (int s = 0; s < kNS && s < filled; ++s) {
        mbar_wait(bar(KF + s), (last_par >> s) & 1u, dw, 12);
        mbar_wait(bar(VF + s), (last_par >> s) & 1u, dw, 12);
      }
    } else if ((warp == 9 || warp == 10) && lane == 0) {
      // Products of warpgroup X = warp - 9: its tiles u = X, X + 2, ... of every item.
      const int X = warp - 9;
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, 1);
      int jg = 0;      // this warpgroup's tiles so far (all items)
      int ubase = 0;   // ring position of the current item's tile 0
      bool ok = true;
      AttnItem it;
      for (int k = 0; ok && split_item(a, n_items, k, it); ++k) {
        const int nX = (it.n + 1 - X) / 2;
        const int qb = k & 1;
        ok = mbar_wait(bar(QF + qb), (k >> 1) & 1, wc, 13);
        const uint32_t qa = smem_addr(sQ + qb * kTile);
        auto issue_s = [&](int j) -> bool {   // S(u) into S_X, u = X + 2 j of this item
          const int U = ubase + X + 2 * j, st = U % kNS, g = jg + j;
          if (!mbar_wait(bar(SE + X), (g & 1) ^ 1, wc, 17)) return false;
          if (!mbar_wait(bar(KF + st), (U / kNS) & 1, wc, 18)) return false;
          tc_fence_after();
          const uint32_t ka = smem_addr(sK + st * kTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + X * 256, smem_desc_sw128(qa + 32 * kk, 16, 1024), smem_desc_sw128(ka + 32 * kk, 16, 1024),
                      idesc_s, kk > 0);
          umma_commit(bar(SF + X));
          return true;
        };
        auto issue_pv = [&](int j) -> bool {
          const int U = ubase + X + 2 * j, st = U % kNS, g = jg + j;
          if (!mbar_wait(bar(PF + X), g & 1, wc, 14)) return false;
          if (!mbar_wait(bar(VF + st), (U / kNS) & 1, wc, 15)) return false;
          if (j == 0 && !mbar_wait(bar(OFREE + X), (k & 1) ^ 1, wc, 16)) return false;   // previous item merged
          tc_fence_after();
          const uint32_t va = smem_addr(sV + st * kTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 8 TMEM columns of P, 2 K-rows groups of V
            umma_bf16_ts(tmem + X * 256 + 192, tmem + X * 256 + 128 + 8 * kk,
                         smem_desc_sw128(va + kk * 2048, kTile, 1024), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(PE + X));
          umma_commit(bar(KVE + st));   // K/V tile U: S(U) and PV(U) were its last users
          return true;
        };
        if (ok && nX > 0) ok = issue_s(0);
        for (int j = 0; ok && j < nX; ++j) {
          if (j + 1 < nX) ok = issue_s(j + 1);
          if (ok) ok = issue_pv(j);
        }
        // Without a tile in this item, still wait for the previous item's merge
        // before signalling this one: no per-item barrier may complete twice
        // before its waiters have seen the first completion (parity waits).
        if (ok && nX == 0) ok = mbar_wait(bar(OFREE + X), (k & 1) ^ 1, wc, 16);
        umma_commit(bar(OD + X));   // O_X of this item is final once its products are done
        umma_commit(bar(QE + qb));  // and so is this issuer's use of the Q buffer
        jg += nX;
        ubase += it.n;
      }
      umma_commit(bar(DR + X));
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(DR + X), 0, dw, 19);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------- softmax: warpgroup X takes key tiles X, X + 2, ...; thread r owns row q0 + r
    const int X = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + X * 256 + lane_off;
    const uint32_t tP = tS + 128;
    const uint32_t tO = tS + 192;
    const float sl2 = a.scale_log2;
    const int W = a.window;
    int jg = 0;   // this warpgroup's tiles so far (all items)

    AttnItem it;
    for (int k = 0; split_item(a, n_items, k, it); ++k) {
      const int q0 = it.q0;
      const int i = q0 + r;
      const int nX = (it.n + 1 - X) / 2;   // tiles u = X, X + 2, ... < n
      float m_used = -INFINITY, l_run = 0.f;
      bool ok = true;

      for (int j = 0; j < nX; ++j, ++jg) {
        const int key0 = (it.kt0 + X + 2 * j) * 128;
        bool w = mbar_wait(bar(SF + X), jg & 1, wc, 21);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        float sv[128];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(r0[e]);
            sv[e + 32] = __uint_as_float(r1[e]);
            sv[e + 64] = __uint_as_float(r2[e]);
            sv[e + 96] = __uint_as_float(r3[e]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(SE + X));      // S_X may be overwritten by the next product
        // Edge tile: keys outside (i - W, i] of this row, i.e. outside columns
        // [lo, hi] of the tile, are masked.
        if (key0 + 127 > q0 || key0 <= q0 + 127 - W) {
          const int lo = i - W + 1 - key0, hi = i - key0;
#pragma unroll
          for (int e = 0; e < 128; ++e) sv[e] = (e >= lo && e <= hi) ? sv[e] : -INFINITY;
        }
        const float m_tile = fmaxf(fmaxf(tree_max32(sv), tree_max32(sv + 32)),
                                   fmaxf(tree_max32(sv + 64), tree_max32(sv + 96))) * sl2;
        // Rescale decision (per row): a first finite max just sets m_used (l and O
        // are still zero); a max more than the slack above m_used rescales.
        float corr = 1.f;
        if (m_tile > m_used + kRescaleSlack) {
          if (m_used != -INFINITY) corr = ex2_approx(m_used - m_tile);
          m_used = m_tile;
        }
        l_run *= corr;
        const float mu = (m_used == -INFINITY) ? 0.f : m_used;

        // P_X and O_X are free once the previous P V product of this warpgroup is done.
        w = mbar_wait(bar(PE + X), (jg & 1) ^ 1, wc, 22);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
          uint32_t o0[32], o1[32];
          tmem_ld32(tO, o0);
          tmem_ld32(tO + 32, o1);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o0[e] = __float_as_uint(__uint_as_float(o0[e]) * corr);
            o1[e] = __float_as_uint(__uint_as_float(o1[e]) * corr);
          }
          tmem_st32(tO, o0);
          tmem_st32(tO + 32, o1);
        }
        // p = 2^(s * scale_log2 - mu), row sum, P (bf16 pairs) into TMEM
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float pv[32];
          exp2_scaled32(sv + c * 32, sl2, mu, pv);
          rs += sum32_tree(pv);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
          tmem_st16(tP + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(PF + X));
        l_run += rs;
      }

      // Merge: the warpgroups swap (m, l) through shared memory (one buffer per
      // item parity); then each reads both O_0 and O_1 from TMEM for its half
      // of the 64 output columns and releases them for the next item.
      float* xk = xml + (k & 1) * 512;
      xk[X * 128 + r] = m_used;
      xk[256 + X * 128 + r] = ok ? l_run : 0.f;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      bool w = mbar_wait(bar(OD + 0), k & 1, wc, 23) && mbar_wait(bar(OD + 1), k & 1, wc, 24);
      if (!__all_sync(0xffffffffu, w)) ok = false;
      tc_fence_after();
      const float m0v = xk[r], l0v = xk[256 + r], m1v = xk[128 + r], l1v = xk[384 + r];
      const float M = fmaxf(m0v, m1v);
      const float f0 = (m0v == -INFINITY) ? 0.f : ex2_approx(m0v - M);
      const float f1 = (m1v == -INFINITY) ? 0.f : ex2_approx(m1v - M);
      const float inv_l = 1.0f / (l0v * f0 + l1v * f1);
      uint32_t x0[32], x1[32];
      tmem_ld32(tmem + 192 + 32 * X + lane_off, x0);
      tmem_ld32(tmem + 256 + 192 + 32 * X + lane_off, x1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) { mbar_arrive(bar(OFREE + 0)); mbar_arrive(bar(OFREE + 1)); }
      if (ok && i < a.T) {
        uint16_t* dst = static_cast<uint16_t*>(a.out) + static_cast<int64_t>(it.b) * a.o_batch +
                        static_cast<int64_t>(i) * a.o_row + static_cast<int64_t>(it.h) * a.o_head + 32 * X;
        float v[32];
#pragma unroll
        for (int d = 0; d < 32; ++d) {
          // a warpgroup without keys for this row contributes nothing (its O may be stale)
          const float y0 = f0 != 0.f ? __uint_as_float(x0[d]) * f0 : 0.f;
          const float y1 = f1 != 0.f ? __uint_as_float(x1[d]) * f1 : 0.f;
          v[d] = (y0 + y1) * inv_l;
        }
        store_bf16x32(dst, v);
      }
      // Both warpgroups take the same decision on the CTA's abort flag (an OR
      // over all 256 threads at this barrier), so a timeout ends the item loop
      // of both and no one is left waiting at the barrier.
      uint32_t stop;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\t"
          "setp.ne.s32 p, %1, 0;\n\t"
          "bar.red.or.pred q, 1, 256, p;\n\t"
          "selp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(stop)
          : "r"(*reinterpret_cast<volatile int*>(abort_flag))
          : "memory");
      if (stop) break;
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
    cudaError_t e = cudaFuncSetAttribute(swa_attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kAttnSmemPair);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(swa_attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmemSplit);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // Persistent grids of one CTA per SM.  Measured per key tile of an item:
  // ~1.6 us per round of items when the two warpgroups split an item's tiles
  // (a merge per item), ~2.6 us per round of item pairs when each warpgroup
  // owns an item; the rounds count decides which is shorter.
  const int64_t items = static_cast<int64_t>((a.T + 127) / 128) * a.H * a.B;
  const int64_t pairs = (items + 1) / 2;
  const int64_t sm = L.sm_count > 0 ? L.sm_count : 1;
  const double t_split = 1.6 * static_cast<double>((items + sm - 1) / sm);
  const double t_pair = 2.6 * static_cast<double>((pairs + sm - 1) / sm);
  if (t_pair < t_split) {
    const int grid = static_cast<int>(pairs < sm ? pairs : sm);
    return launch_kernel(swa_attn_pair_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmemPair, L.stream, tmQ, tmK,
                         tmV, a);
  }
  const int grid = static_cast<int>(items < sm ? items : sm);
  return launch_kernel(swa_attn_split_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmemSplit, L.stream, tmQ, tmK,
                       tmV, a);
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
