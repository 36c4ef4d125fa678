// attn.cu -- causal sliding-window attention kernels.
//
// swa_attn_ws_kernel: flash-style bf16 attention on tcgen05 tensor cores
//   (see its comment below): persistent CTAs over pairs of neighbouring
//   128-query tiles, 64-key tiles by TMA, S / P / O / row sums in TMEM, only
//   the key tiles that meet the causal window visited.
// swa_attn_f32_kernel: fp32 CUDA-core reference-precision path (one warp per
//   query row), used for fp32 inputs.
// rope_rows_kernel: RoPE pre-pass of vx_swa_attn_fwd on raw q, k (one pass,
//   each angle computed once per row).
#include <cmath>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kAttnThreads = 384;           // 2 softmax warpgroups; TMA, 2 MMA and 1 idle warp
constexpr int kTile = 128 * 64 * 2;         // one 128 x 64 bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleSlack = 8.0f;       // O is rescaled only when a row max grows by more than 2^8

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_global_v4(dst + 8 * j, pack_bf16x2(v[8 * j + 0], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                 pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}

// The exponent arguments use sm_100's packed fp32x2 FMA (each lane of a
// packed op rounds like the scalar op, so the results are those of the
// scalar code), halving their instruction count in the softmax.
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

// Three-input maximum (sm_100's max.f32 with three sources).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max of 64 values: a three-input tree (64 -> 22 -> 8 -> 3 -> 1), short
// dependency chains, 32 instructions.
__device__ __forceinline__ float tree_max64(const float* v) {
  float t[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) t[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  t[21] = v[63];
  float u[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) u[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  u[7] = t[21];
  return fmax3(fmax3(u[0], u[1], u[2]), fmax3(u[3], u[4], u[5]), fmaxf(u[6], u[7]));
}

// v[e] = v[e] * sl2 - mu for 64 scores, two at a time.
__device__ __forceinline__ void exp2_args64(float (&v)[64], float sl2, float mu) {
  const uint64_t sc = f2_pack(sl2, sl2), nm = f2_pack(-mu, -mu);
#pragma unroll
  for (int e = 0; e < 64; e += 2) f2_unpack(ffma2(f2_pack(v[e], v[e + 1]), sc, nm), v[e], v[e + 1]);
}

// 2^x on the MUFU unit as a volatile asm: the compiler keeps these in
// program order with the token hand-off around them.
__device__ __forceinline__ float ex2_ordered(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// The softmax warpgroups take most of the register file (setmaxnreg): 8
// softmax warps x 224 + 4 other warps x 56 = 384 threads x 168 at launch.
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;

// swa_attn_ws_kernel: one CTA per SM walks "pair items": two neighbouring
// 128-query tiles (2p, 2p+1) of one (clip, head).  Softmax warpgroup X owns
// query tile 2p+X entirely (online softmax over its key tiles, its own output)
// and has its own tensor-core issuer thread; the two share one TMA producer
// and one K/V ring that carries the union of their key ranges once (the two
// windows overlap in all but two 64-key tiles, so each K/V tile crosses L2
// once for both).  Key tiles are 64 keys wide so that each warpgroup's TMEM
// holds three S buffers (64 columns each) and its output O (64 columns): S of
// the next two tiles is computed while the softmax of a tile runs, and P(j)
// is written back (bf16 pairs) into S(j)'s own columns, whose next use is
// tile j+3.  O is rescaled in place only when a row's running maximum grows by
// more than kRescaleSlack.  Only the key tiles that meet the causal window are
// visited, and masks are applied only on edge tiles, per warp.
// Measured on B200 (per-phase clock stamps of one CTA): a 64-key tile costs a
// softmax warp ~470 cycles outside its exponentials and ~550 cycles of MUFU
// issue (64 warp-wide ex2 at 8 cycles each); the tensor core is ~20% busy and
// the MMA issue rate (~50 cycles per instruction per issuing thread) is not
// the limit.  Warp q of each warpgroup shares a scheduler's MUFU with warp q
// of the other, so the two take turns at their exponentials (a token passed
// through an mbarrier, see the softmax loop); computing part of the
// exponentials on the FMA pipe instead measured slower.
// Warps 0-3 / 4-7: softmax warpgroups 0 / 1 (TMEM lane = query row); warp 8:
// TMA producer; warps 9 / 10: the tensor-core products of warpgroup 0 / 1.
constexpr int kWsStages = 6;                     // K/V ring stages (64-key tiles)
constexpr int kKvTile = kAttnKeyTile * 64 * 2;   // 8 KB: 64 keys x 64 dims bf16
constexpr int kSBuf = 3;                         // S buffers per warpgroup
constexpr int kAttnSmemWs = 4 * kTile + 2 * kWsStages * kKvTile + 1024 + 512;

struct PairItem {
  int b, h, p;        // clip, head, pair index (query tiles 2p, 2p+1)
  int q0[2];          // first query of each tile (q0[1] < 0: no second tile)
  int kt0[2], n[2];   // first 64-key tile and tile count of each query tile
  int u0, nu;         // union: first key tile (= kt0[0]) and tile count
};

__device__ __forceinline__ void pair_item_at(const AttnArgs& a, int b, int h, int p, PairItem& it) {
  it.b = b;
  it.h = h;
  it.p = p;
  for (int X = 0; X < 2; ++X) {
    const int q0 = (2 * p + X) * 128;
    if (q0 >= a.T) {
      it.q0[X] = -1;
      it.kt0[X] = 0;
      it.n[X] = 0;
      continue;
    }
    it.q0[X] = q0;
    it.kt0[X] = max(0, q0 - a.window + 1) / kAttnKeyTile;
    it.n[X] = min(a.T - 1, q0 + 127) / kAttnKeyTile - it.kt0[X] + 1;
  }
  it.u0 = it.kt0[0];
  it.nu = (it.n[1] > 0 ? it.kt0[1] + it.n[1] : it.kt0[0] + it.n[0]) - it.u0;
}

// Round r of this CTA: pair items sorted heaviest first (higher pair index
// first; a tile's key count never decreases with its index), dealt to the
// CTAs round by round in alternating directions.  False past the CTA's last item.
__device__ __forceinline__ bool ws_item(const AttnArgs& a, int n_items, int r, PairItem& it) {
  const int G = gridDim.x, x = blockIdx.x;
  const int pos = r * G + ((r & 1) ? G - 1 - x : x);
  if (pos >= n_items) return false;
  const int hb = a.H * a.B;
  const int np = ((a.T + 127) / 128 + 1) / 2;
  const int rest = pos % hb;
  pair_item_at(a, rest / a.H, rest % a.H, np - 1 - pos / hb, it);
  return true;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
swa_attn_ws_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // Q[X][buffer]: 4 tiles of 16 KB
  uint8_t* sK = sQ + 4 * kTile;                        // K ring: kWsStages x 8 KB
  uint8_t* sV = sK + kWsStages * kKvTile;              // V ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kWsStages * kKvTile);
  // per warpgroup X: QF/QE [X*2 + buf], SF/PF/BF [X*3 + b], OD/OFREE/DR [X]
  // KF[stage]: the stage's K and V tiles have landed (one barrier, both copies' bytes)
  constexpr int QF = 0, QE = 4, KF = 8, KVE = KF + kWsStages, SF = KVE + kWsStages,
                PF = SF + 2 * kSBuf, BF = PF + 2 * kSBuf, OD = BF + 2 * kSBuf, OFREE = OD + 2, DR = OFREE + 2,
                TOK = DR + 2, NBAR = TOK + 8;   // TOK[X * 4 + q]: warp q of warpgroup X may exponentiate
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = (((a.T + 127) / 128 + 1) / 2) * a.H * a.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) { mbar_init(bar(QF + i), 1); mbar_init(bar(QE + i), 1); }
    for (int s = 0; s < kWsStages; ++s) { mbar_init(bar(KF + s), 1); mbar_init(bar(KVE + s), 2); }
    for (int i = 0; i < 2 * kSBuf; ++i) { mbar_init(bar(SF + i), 1); mbar_init(bar(PF + i), 128); mbar_init(bar(BF + i), 1); }
    for (int X = 0; X < 2; ++X) { mbar_init(bar(OD + X), 1); mbar_init(bar(OFREE + X), 4); mbar_init(bar(DR + X), 1); }
    for (int i = 0; i < 8; ++i) mbar_init(bar(TOK + i), 1);
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
      // ------------- TMA producer: both Q tiles of a pair item, then the union of their key tiles
      uint32_t last_par = 0, q_issued = 0, q_par = 0;
      int filled = 0;
      int U = 0;              // K/V tiles loaded so far (ring position)
      int qc[2] = {0, 0};     // Q tiles loaded per warpgroup
      bool ok = true;
      PairItem it;
      for (int r = 0; ok && ws_item(a, n_items, r, it); ++r) {
        for (int X = 0; X < 2 && ok; ++X) {
          if (it.n[X] == 0) continue;
          const int qi = X * 2 + (qc[X] & 1);
          if (!mbar_wait(bar(QE + qi), ((qc[X] >> 1) & 1) ^ 1, wc, 50)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(QF + qi), kTile);
          tma_load_4d(smem_addr(sQ + qi * kTile), &tmQ, bar(QF + qi), 0, it.h, it.q0[X], it.b);
          q_issued |= 1u << qi;
          q_par = (q_par & ~(1u << qi)) | ((static_cast<uint32_t>(qc[X] >> 1) & 1u) << qi);
          ++qc[X];
        }
        for (int u = 0; ok && u < it.nu; ++u, ++U) {
          const int st = U % kWsStages;
          const uint32_t ph = (U / kWsStages) & 1;
          if (!mbar_wait(bar(KVE + st), ph ^ 1, wc, 51)) { ok = false; break; }
          const int kt = it.u0 + u;
          mbar_arrive_expect_tx(bar(KF + st), 2 * kKvTile);
          tma_load_4d(smem_addr(sK + st * kKvTile), &tmK, bar(KF + st), 0, it.h, kt * kAttnKeyTile, it.b);
          tma_load_4d(smem_addr(sV + st * kKvTile), &tmV, bar(KF + st), 0, it.h, kt * kAttnKeyTile, it.b);
          // The stage is released by each warpgroup that uses the tile (its
          // last product's commit); for a tile only one uses, the producer
          // arrives in the other's place (after the previous phase completed).
          int users = 0;
          for (int X = 0; X < 2; ++X) users += (kt >= it.kt0[X] && kt < it.kt0[X] + it.n[X]) ? 1 : 0;
          if (users < 2) mbar_arrive(bar(KVE + st));
          last_par = (last_par & ~(1u << st)) | (ph << st);
          filled = U + 1;
        }
      }
      // Bounded wait for every copy still in flight (also after an abort).
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int qi = 0; qi < 4; ++qi)
        if (q_issued & (1u << qi)) mbar_wait(bar(QF + qi), (q_par >> qi) & 1u, dw, 52);
      for (int s = 0; s < kWsStages && s < filled; ++s) {
        mbar_wait(bar(KF + s), (last_par >> s) & 1u, dw, 52);
      }
    } else if ((warp == 9 || warp == 10) && lane == 0) {
      // ------------- tensor-core products of warpgroup X
      const int X = warp - 9;
      const uint32_t tX = tmem + X * 256;
      const uint32_t idesc_s = idesc_bf16_f32(128, kAttnKeyTile, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64, 1);
      int jg = 0;      // this warpgroup's key tiles so far (all items)
      int kc = 0;      // this warpgroup's items so far
      int ubase = 0;   // ring position of the current pair item's first union tile
      bool ok = true;
      PairItem it;
      for (int r = 0; ok && ws_item(a, n_items, r, it); ++r) {
        const int n = it.n[X];
        if (n > 0) {
          const int qi = X * 2 + (kc & 1);
          ok = mbar_wait(bar(QF + qi), (kc >> 1) & 1, wc, 53);
          const uint32_t qa = smem_addr(sQ + qi * kTile);
          const int uoff = it.kt0[X] - it.u0;
          auto issue_s = [&](int t) -> bool {   // S(t) into buffer (jg + t) % 3
            const int g = jg + t, bsel = g % kSBuf, U = ubase + uoff + t, st = U % kWsStages;
            if (!mbar_wait(bar(BF + X * kSBuf + bsel), ((g / kSBuf) & 1) ^ 1, wc, 54)) return false;   // P(t-3) consumed
            if (!mbar_wait(bar(KF + st), (U / kWsStages) & 1, wc, 55)) return false;
            tc_fence_after();
            const uint32_t ka = smem_addr(sK + st * kKvTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tX + 64 * bsel, smem_desc_sw128(qa + 32 * kk, 16, 1024),
                        smem_desc_sw128(ka + 32 * kk, 16, 1024), idesc_s, kk > 0);
            umma_commit(bar(SF + X * kSBuf + bsel));
            return true;
          };
          auto issue_pv = [&](int t) -> bool {   // O += P V (P in S(t)'s columns)
            const int g = jg + t, bsel = g % kSBuf, U = ubase + uoff + t, st = U % kWsStages;
            if (!mbar_wait(bar(PF + X * kSBuf + bsel), (g / kSBuf) & 1, wc, 56)) return false;
            // O is overwritten by the item's first product: the warpgroup's
            // previous item must have been read out.
            if (t == 0 && !mbar_wait(bar(OFREE + X), (kc & 1) ^ 1, wc, 58)) return false;
            tc_fence_after();
            const uint32_t va = smem_addr(sV + st * kKvTile);
            const uint32_t pa = tX + 64 * bsel;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: 8 TMEM columns of P, 16 rows of V
              umma_bf16_ts(tX + 192, pa + 8 * kk, smem_desc_sw128(va + kk * 2048, kKvTile, 1024), idesc_o,
                           (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar(BF + X * kSBuf + bsel));   // S buffer free; O holds tile t
            umma_commit(bar(KVE + st));            // K/V tile: S(t) and P V (t) were this group's uses
            return true;
          };
          if (ok) ok = issue_s(0);
          if (ok && n > 1) ok = issue_s(1);
          for (int t = 0; ok && t < n; ++t) {
            if (t + 2 < n) ok = issue_s(t + 2);
            if (ok) ok = issue_pv(t);
          }
          umma_commit(bar(OD + X));   // O of this item is final once its products are done
          umma_commit(bar(QE + qi));  // and so is the use of its Q buffer
          jg += n;
          ++kc;
        }
        ubase += it.nu;
      }
      umma_commit(bar(DR + X));
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      mbar_wait(bar(DR + X), 0, dw, 59);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------- softmax: warpgroup X owns query tile 2p + X; thread r owns row q0 + r
    const int X = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tX = tmem + X * 256 + lane_off;
    const uint32_t tO = tX + 192;
    const float sl2 = a.scale_log2;
    const int W = a.window;
    int jg = 0;   // this warpgroup's key tiles so far (all items)
    int kc = 0;   // this warpgroup's items so far
    // Warp q of each warpgroup shares a scheduler (and its MUFU) with warp q
    // of the other.  Their exponentials would otherwise run at the same time
    // and their other phases too, leaving the MUFU idle in between; so over
    // the first min(nA, nB) tiles of each pair item the two take turns,
    // passing a token (an mbarrier, waited with the bounded wait) after each
    // tile's exponentials.  Warpgroup 0 holds the token first.  Both count
    // the same turns per item, so the phases always match.
    const int q = warp & 3;
    const uint32_t tok_mine = bar(TOK + X * 4 + q), tok_other = bar(TOK + (X ^ 1) * 4 + q);
    int turns = 0;   // token-protected tiles so far
    if (X == 1 && lane == 0) mbar_arrive(tok_other);
    bool ok = true;
    PairItem it;
    for (int rr = 0; ok && ws_item(a, n_items, rr, it); ++rr) {
      const int n = it.n[X];
      if (n == 0) continue;
      const int m_turns = min(it.n[0], it.n[1]);
      const int q0 = it.q0[X];
      const int i = q0 + r;
      float m_used = -INFINITY, l_run = 0.f;
      for (int t = 0; t < n; ++t) {
        const int g = jg + t, bsel = g % kSBuf;
        const int key0 = (it.kt0[X] + t) * kAttnKeyTile;
        bool w = mbar_wait(bar(SF + X * kSBuf + bsel), (g / kSBuf) & 1, wc, 60);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tX + 64 * bsel;
        float sv[64];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(r0[e]);
            sv[e + 32] = __uint_as_float(r1[e]);
          }
        }
        // Edge tile: keys outside (i - W, i] of this row, i.e. outside
        // columns [lo, hi] of the tile, are masked.  A tile meets the causal
        // edge (keys after some row: e > hi) or the window's start (keys too
        // old for some row: e < lo), both only when W < 192; each test is
        // skipped when no row of this warp (rows wq0 .. wq0 + 31) needs it.
        {
          const int wq0 = q0 + (warp & 3) * 32;
          const int lo = i - W + 1 - key0, hi = i - key0;
          const bool causal = key0 + kAttnKeyTile - 1 > wq0;        // some row of the warp has hi < 63
          const bool window = key0 < wq0 + 31 - W + 1;              // some row of the warp has lo > 0
          if (causal && window) {
#pragma unroll
            for (int e = 0; e < 64; ++e) sv[e] = (e >= lo && e <= hi) ? sv[e] : -INFINITY;
          } else if (causal) {
#pragma unroll
            for (int e = 0; e < 64; ++e) sv[e] = e <= hi ? sv[e] : -INFINITY;
          } else if (window) {
#pragma unroll
            for (int e = 0; e < 64; ++e) sv[e] = e >= lo ? sv[e] : -INFINITY;
          }
        }
        const float m_tile = tree_max64(sv) * sl2;
        // Rescale decision (per row): a first finite max just sets m_used (O
        // and l are still zero); a max more than the slack above m_used
        // rescales O and l (all of this warpgroup's earlier products must be
        // done: the one of tile t-1 completes BF of its buffer).
        float corr = 1.f;
        if (m_tile > m_used + kRescaleSlack) {
          if (m_used != -INFINITY) corr = ex2_approx(m_used - m_tile);
          m_used = m_tile;
        }
        l_run *= corr;
        if (t > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
          const int gp = g - 1;
          w = mbar_wait(bar(BF + X * kSBuf + gp % kSBuf), (gp / kSBuf) & 1, wc, 61);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          tc_fence_after();
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
        const float mu = (m_used == -INFINITY) ? 0.f : m_used;
        // p = 2^(s * scale_log2 - mu): the arguments first, then (holding the
        // token) only the 64 exponentials back to back, then the row sum and
        // P as bf16 pairs over S's first 32 columns while the partner warp
        // exponentiates.
        exp2_args64(sv, sl2, mu);
        const bool turn = t < m_turns;
        if (turn) {
          w = mbar_wait(tok_mine, turns & 1, wc, 63);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        }
#pragma unroll
        for (int e = 0; e < 64; ++e) sv[e] = ex2_ordered(sv[e]);
        if (turn) {   // every exponential above is issued before this point (ordered asm): pass the token
          __syncwarp();
          if (lane == 0) mbar_arrive(tok_other);
          ++turns;
        }
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          rs += sum32_tree(*reinterpret_cast<const float(*)[32]>(sv + c * 32));
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]);
          tmem_st16(tS + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(PF + X * kSBuf + bsel));
        l_run += rs;
      }
      if (!ok) break;
      jg += n;

      // Output: O / l once the item's last product is done; O is then
      // released for the warpgroup's next item.
      bool w = mbar_wait(bar(OD + X), kc & 1, wc, 62);
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

// Rotates q and k ([B, T, H, 64]) into qr and kr in one pass: warp per
// (row, tensor).  Lane m computes the angle (pos0 + t) * inv_freq_m once;
// each lane then takes the 8-pair groups g = lane % 4 (pairs m = 8g .. 8g+7
// with m + 32) of heads lane / 4, lane / 4 + 8, ..., with its group's eight
// cos / sin from the other lanes by shuffles, so every access is 16 bytes
// and each angle is computed once per row and tensor.
template <bool BF16>
__global__ void __launch_bounds__(256) rope_rows_kernel(const void* __restrict__ q, const void* __restrict__ k,
                                                        void* __restrict__ qr, void* __restrict__ kr, int64_t rows,
                                                        int T, int H, int64_t pos0, const __grid_constant__ RopeArgs f) {
  pdl_wait();
  pdl_trigger();
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= 2 * rows) return;   // whole warps leave together
  const int64_t row = wid >> 1;
  const int which = static_cast<int>(wid & 1);
  const int t = static_cast<int>(row % T);
  float sn_m, cs_m;
  rope_sincos(static_cast<float>(pos0 + t), f.hi[lane], f.lo[lane], &sn_m, &cs_m);
  const int g = lane & 3;
  float cs[8], sn[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    cs[i] = __shfl_sync(0xffffffffu, cs_m, 8 * g + i);
    sn[i] = __shfl_sync(0xffffffffu, sn_m, 8 * g + i);
  }
  for (int h = lane >> 2; h < H; h += 8) {
    const int64_t e = (row * H + h) * 64 + 8 * g;
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
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(which ? k : q) + e);
      const float4 a0 = src[0], a1 = src[1], c0 = src[8], c1 = src[9];
      u[0] = a0.x; u[1] = a0.y; u[2] = a0.z; u[3] = a0.w; u[4] = a1.x; u[5] = a1.y; u[6] = a1.z; u[7] = a1.w;
      w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w; w[4] = c1.x; w[5] = c1.y; w[6] = c1.z; w[7] = c1.w;
    }
    float y1[8], y2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      y1[i] = u[i] * cs[i] - w[i] * sn[i];
      y2[i] = w[i] * cs[i] + u[i] * sn[i];
    }
    if constexpr (BF16) {
      uint16_t* dst = static_cast<uint16_t*>(which ? kr : qr);
      *reinterpret_cast<uint4*>(dst + e) = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]),
                                                      pack_bf16x2(y1[4], y1[5]), pack_bf16x2(y1[6], y1[7]));
      *reinterpret_cast<uint4*>(dst + e + 32) = make_uint4(pack_bf16x2(y2[0], y2[1]), pack_bf16x2(y2[2], y2[3]),
                                                           pack_bf16x2(y2[4], y2[5]), pack_bf16x2(y2[6], y2[7]));
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(which ? kr : qr) + e);
      dst[0] = make_float4(y1[0], y1[1], y1[2], y1[3]);
      dst[1] = make_float4(y1[4], y1[5], y1[6], y1[7]);
      dst[8] = make_float4(y2[0], y2[1], y2[2], y2[3]);
      dst[9] = make_float4(y2[4], y2[5], y2[6], y2[7]);
    }
  }
}

}  // namespace

// 4-D bf16 map {64 (d), H, T, B} with a box of `rows` frames of one head.
static bool tmap_attn_operand(CUtensorMap* map, const void* base, int B, int T, int H, int64_t row_stride,
                       int64_t batch_stride, int rows) {
  const uint64_t dims[4] = {64, static_cast<uint64_t>(H), static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
  const uint64_t strides[3] = {128, static_cast<uint64_t>(row_stride) * 2, static_cast<uint64_t>(batch_stride) * 2};
  const uint32_t box[4] = {64, 1, static_cast<uint32_t>(rows), 1};
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_attn_bf16(const Launch& L, const AttnOperands& op, const AttnArgs& a) {
  CUtensorMap tq, tk, tv;
  if (!tmap_attn_operand(&tq, op.q, a.B, a.T, a.H, op.row_stride, op.batch_stride, 128) ||
      !tmap_attn_operand(&tk, op.k, a.B, a.T, a.H, op.row_stride, op.batch_stride, kAttnKeyTile) ||
      !tmap_attn_operand(&tv, op.v, a.B, a.T, a.H, op.row_stride, op.batch_stride, kAttnKeyTile))
    return cudaErrorInvalidValue;
  // Persistent grid of one CTA per SM over the pair items.
  const int64_t items = static_cast<int64_t>(((a.T + 127) / 128 + 1) / 2) * a.H * a.B;
  const int64_t sm = L.sm_count > 0 ? L.sm_count : 1;
  const int grid = static_cast<int>(items < sm ? items : sm);
  return launch_kernel(swa_attn_ws_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmemWs, L.stream, tq, tk, tv, a);
}

cudaError_t launch_attn_f32(const Launch& L, const float* q, const float* k, const float* v, float* o,
                            int B, int T, int H, int window, float scale) {
  const dim3 grid((T + 3) / 4, H, B);
  return launch_kernel(swa_attn_f32_kernel, grid, dim3(128), 0, L.stream, q, k, v, o, T, H, window, scale);
}

cudaError_t launch_rope(const Launch& L, const void* q, const void* k, void* qr, void* kr, bool bf16, int B, int T,
                        int H, int64_t pos0, float theta) {
  RopeArgs f;
  for (int m = 0; m < 32; ++m) {
    const double inv = std::pow(static_cast<double>(theta), -2.0 * m / 64.0);
    f.hi[m] = static_cast<float>(inv);
    f.lo[m] = static_cast<float>(inv - static_cast<double>(f.hi[m]));
  }
  const int64_t rows = static_cast<int64_t>(B) * T;
  const dim3 grid(static_cast<unsigned>((2 * rows + 7) / 8));   // 8 warps per block
  if (bf16)
    return launch_kernel(rope_rows_kernel<true>, grid, dim3(256), 0, L.stream, q, k, qr, kr, rows, T, H, pos0, f);
  return launch_kernel(rope_rows_kernel<false>, grid, dim3(256), 0, L.stream, q, k, qr, kr, rows, T, H, pos0, f);
}

}  // namespace vx
