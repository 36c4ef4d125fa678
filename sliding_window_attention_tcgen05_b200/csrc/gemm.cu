// gemm.cu -- persistent, warp-specialised tcgen05 GEMMs for sm_100a with the
// fused epilogues of the encoder layer (bias, RoPE, SwiGLU, GELU, residual).
//
//   D[M, N] = A[M, K] * B[N, K]^T,  A and B bf16 K-major, fp32 accumulate in TMEM.
//
// Two kernels share one structure and one epilogue:
//   gemm_tc_kernel<BN>   one CTA per 128 x BN tile (BN 128 / 256);
//   gemm_tc2_kernel<BN>  a cluster of two CTAs per 256 x BN tile, issued as
//                        tcgen05.mma.cta_group::2 (M = 256) by the leader CTA.
// CTA = 11 warps: warps 0-7 epilogue (warp w reads TMEM lanes 32 (w % 4) ..,
// i.e. 32 tile rows, and half of the tile's columns), warps 8 and 10 TMA
// producers (even / odd ring stages), warp 9 MMA issuer (owns the TMEM
// allocation).  A 192 KB TMA ->
// shared memory ring guarded by mbarriers feeds the MMAs; two TMEM
// accumulators let the epilogue of one tile overlap the main loop of the next.
// Work units (m tile, K split, n tile) are visited M-fastest, so the CTAs
// resident at one time share a weight (B) panel through L2, N-fastest when A
// is the larger operand and too large for L2 (it then crosses DRAM once), or
// in groups of four row panels (launch_gemm chooses).
//
// The main loop is bound by how fast TMA can fill one SM's shared memory, so
// the tile shape is chosen to move the fewest bytes per MMA: a CTA pair
// stages 16 KB of A and BN/2 rows of B per 64-wide K block for 128 x BN of
// MMA work (plan_gemm picks the shape, see below).  Issuing a 16 KB tile load
// keeps the issuing thread ~160-250 cycles (measured), and with its barrier
// wait and bookkeeping one thread needs about as long per K block as the
// MMAs of a 256-wide block take, so it could never run ahead of them; two
// producer threads in separate warps split the ring's stages (even / odd).
//
// Epilogue: each warp reads 32 rows x 32 columns at a time from TMEM (one row
// per lane), applies the row-wise part of the epilogue (bias, RoPE pairs,
// SwiGLU gate x up, GELU), transposes the chunk through a swizzled 2 KB
// shared-memory buffer and stores it with four lanes per row, so every store
// writes whole 32-byte sectors.  The tile's bias is staged in shared memory,
// and the rows' positions and the residual of the first chunk are prepared
// before the accumulator is ready.
#include <cmath>
#include <cstdio>

#include "vx_internal.h"

namespace vx {

namespace {

constexpr int kThreads = 352;   // warps 0-7 epilogue, 8 and 10 TMA producers, 9 MMA issuer
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kProducer2Warp = 10;

// Producer index of a warp (0, 1), or -1.
__device__ __forceinline__ int producer_of(int warp) {
  return warp == kProducerWarp ? 0 : (warp == kProducer2Warp ? 1 : -1);
}
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kSmemBytes = 227 * 1024;        // per CTA
constexpr int kStgBufBytes = 2048;            // 32 rows x 64 bytes
constexpr int kBiasBytes = 8 * 256 * 2;       // per epilogue warp: the tile's bias, BN <= 256
constexpr int kBarBytes = 256;

// Staging buffers per epilogue warp: two for the QKV epilogue, whose stores
// would otherwise wait for one another (measured: 4 x 3000 frame encoder, QKV
// 144 -> 138 us), one elsewhere (a second one would cost a ring stage).
constexpr int stg_bufs(int epi) { return epi == EPI_QKV_ROPE ? 2 : 1; }

// Shared memory: [ring][staging][bias][barriers], 1024-aligned base; the TMA
// ring takes as many stages as fit.
template <int STAGE_BYTES, int NBUF>
struct SmemCfg {
  static constexpr int kStgBytes = 8 * NBUF * kStgBufBytes;
  static constexpr int kStages = (kSmemBytes - kStgBytes - kBiasBytes - kBarBytes - 1024) / STAGE_BYTES;
  static constexpr int kStg = kStages * STAGE_BYTES;
  static constexpr int kBias = kStg + kStgBytes;
  static constexpr int kBars = kBias + kBiasBytes;
  static constexpr int kTotal = kBars + kBarBytes + 1024;
  static_assert(kStages >= 3 && kStages <= 12, "ring depth");
  static_assert(kTotal <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// silu(x) = x * sigmoid(x) = x / (1 + 2^(-x log2 e)); the hardware 2^x and
// reciprocal are accurate to ~2^-22 relative, far below the bf16 rounding of
// the result.  Saturates correctly: x -> -inf gives -0, x -> +inf gives x.
__device__ __forceinline__ float silu_f(float x) {
  return x * rcp_approx(1.0f + ex2_approx(-1.4426950408889634f * x));
}

// Waits for this thread's outstanding tcgen05.ld; the registers are passed
// through so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld2_wait(uint32_t (&r0)[32], uint32_t (&r1)[32]) {
  tmem_ld_wait_regs(r0);
  asm volatile("" : "+r"(r1[0]), "+r"(r1[1]), "+r"(r1[2]), "+r"(r1[3]), "+r"(r1[4]), "+r"(r1[5]), "+r"(r1[6]),
               "+r"(r1[7]), "+r"(r1[8]), "+r"(r1[9]), "+r"(r1[10]), "+r"(r1[11]), "+r"(r1[12]), "+r"(r1[13]),
               "+r"(r1[14]), "+r"(r1[15]), "+r"(r1[16]), "+r"(r1[17]), "+r"(r1[18]), "+r"(r1[19]), "+r"(r1[20]),
               "+r"(r1[21]), "+r"(r1[22]), "+r"(r1[23]), "+r"(r1[24]), "+r"(r1[25]), "+r"(r1[26]), "+r"(r1[27]),
               "+r"(r1[28]), "+r"(r1[29]), "+r"(r1[30]), "+r"(r1[31]));
}

// v[i] += bias[i], i < 32, bias in shared memory (every lane reads the same words).
__device__ __forceinline__ void add_bias32_smem(float (&v)[32], const uint16_t* sb) {
  const uint4* bp = reinterpret_cast<const uint4*>(sb);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 w = bp[j];
    v[8 * j + 0] += bf16lo(w.x); v[8 * j + 1] += bf16hi(w.x);
    v[8 * j + 2] += bf16lo(w.y); v[8 * j + 3] += bf16hi(w.y);
    v[8 * j + 4] += bf16lo(w.z); v[8 * j + 5] += bf16hi(w.z);
    v[8 * j + 6] += bf16lo(w.w); v[8 * j + 7] += bf16hi(w.w);
  }
}

// Staging buffer of one warp: 32 rows x four 16-byte slots (32 bf16 or 16
// fp32 per row).  Slot j of row r sits at j ^ ((r >> 1) & 3), so that the
// row-wise writes (one row per lane) and the column-wise reads (four lanes per
// row) both touch eight distinct 16-byte bank groups per quarter warp.
__device__ __forceinline__ int stg_slot(int r, int j) { return r * 4 + (j ^ ((r >> 1) & 3)); }

__device__ __forceinline__ void stage_bf16x32(uint4* stg, int lane, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    stg[stg_slot(lane, j)] = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                        pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}
__device__ __forceinline__ void stage_f32x16(uint4* stg, int lane, const float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    stg[stg_slot(lane, j)] = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                                        __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
}

__device__ __forceinline__ void st_global_u4(void* p, uint4 v) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Output row of source row m (see GemmArgs); ok = the row is stored.
__device__ __forceinline__ int64_t out_row(const GemmArgs& a, int m, bool& ok, int& b, int& t) {
  b = m / a.in_rows;
  t = m - b * a.in_rows;
  ok = m < a.M && t < a.t_valid;
  return static_cast<int64_t>(b) * a.out_rows + a.out_off + t;
}

// Rows this lane stores in the column-wise phase: mw + (lane >> 2) + 8 i.
struct StoreRows {
  int64_t drow[4];
  uint32_t ok;
};
__device__ __forceinline__ StoreRows store_rows(const GemmArgs& a, int mw, int lane) {
  StoreRows s;
  s.ok = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bool ok;
    int b, t;
    s.drow[i] = out_row(a, mw + (lane >> 2) + 8 * i, ok, b, t);
    s.ok |= static_cast<uint32_t>(ok) << i;
  }
  return s;
}

// Stores the warp's staged bf16 chunk: 8 columns col0 + 8 (lane & 3) .. +7 of
// rows (lane >> 2) + 8 i.
__device__ __forceinline__ void store_bf16_chunk(uint16_t* out, int64_t ld_out, const StoreRows& sr, const uint4* stg,
                                                 int lane, int col0) {
  const int jj = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = (lane >> 2) + 8 * i;
    const uint4 v = stg[stg_slot(rr, jj)];
    if (sr.ok & (1u << i)) st_global_u4(out + sr.drow[i] * ld_out + col0 + 8 * jj, v);
  }
}

// Output path of one staged chunk.  With TMA stores the chunk leaves shared
// memory as one 64-byte x 32-row box (the staging swizzle is the tensor map's
// 64-byte swizzle), written by lane 0.  With two staging buffers they take
// turns, so a chunk is staged while the copy engine still reads the previous
// one: before a buffer is refilled, lane 0 waits until at most one store (the
// other buffer's) is still reading; with one, until none is.  Without TMA
// stores one buffer serves.
struct ChunkOut {
  const CUtensorMap* tmD;   // null: stores from registers
  int row0;                 // first tile row of this warp
  int z;                    // K-split index (third map coordinate)
  uint4* stg;               // the warp's staging buffers (128 x 16 bytes each)
  int nbuf;                 // 1 or 2
  int n;                    // chunks stored by this warp so far (across tiles)
};
__device__ __forceinline__ void bulk_wait_read_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// The buffer for the next chunk, free to be written.
__device__ __forceinline__ uint4* stage_buf(const ChunkOut& co, int lane) {
  if (!co.tmD) return co.stg;
  if (lane == 0) {
    if (co.nbuf == 2)
      bulk_wait_read_but_one();
    else
      bulk_wait_read_all();
  }
  __syncwarp();
  return co.nbuf == 2 ? co.stg + 128 * (co.n & 1) : co.stg;
}
__device__ __forceinline__ void tma_flush(ChunkOut& co, const uint4* buf, int lane, int col0) {
  fence_proxy_async_smem();   // this lane's staging writes, visible to the copy engine
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(co.tmD, smem_addr(buf), col0, co.row0, co.z);
    bulk_commit_group();
  }
  ++co.n;
}

// Per warp: TMEM lane quarter q = warp & 3 (tile rows 32 q ..), and one half
// of the tile's column work (warp >> 2).  Everything of a tile's epilogue
// that does not need the accumulator is done before waiting for it: the bias
// into this warp's shared-memory copy, the position of this lane's row, the
// residual of the first chunk.  The RoPE angles are computed per head where
// they are used (hardware sine / cosine): holding all 32 would spill.  Warps never wait for one another, so a warp
// that leaves the tile loop on a timeout cannot stall the others.
template <int BN, int EPI>
struct EpiPre {
  StoreRows sr;
  float posf;
  float4 res[EPI == EPI_F32 ? 4 : 1];
};

// First column of this warp's half of an EPI_F32 / GELU tile.
template <int BN>
__device__ __forceinline__ int half_col0(int warp) { return (warp >> 2) * (BN / 2); }

__device__ __forceinline__ float4 ld_res4(const GemmArgs& a, const StoreRows& sr, int i, int col) {
  return __ldg(reinterpret_cast<const float4*>(a.res + sr.drow[i] * a.ld_res + col));
}

template <int BN, int EPI>
__device__ __forceinline__ void epilogue_prepare(const GemmArgs& a, EpiPre<BN, EPI>& p, uint16_t* sbias, int m0,
                                                 int n0, int ks, int warp, int lane) {
  const bool first_part = ks == 0;
  if (a.bias && first_part) {   // the previous tile's reads of sbias ended at a __syncwarp
    const uint4* src = reinterpret_cast<const uint4*>(a.bias + n0);
    for (int i = lane; i < BN / 8; i += 32) reinterpret_cast<uint4*>(sbias)[i] = __ldg(src + i);
  }
  const int mw = m0 + (warp & 3) * 32;
  p.sr = store_rows(a, mw, lane);
  if constexpr (EPI == EPI_QKV_ROPE) {
    if (n0 < a.rope_cols) {
      bool ok;
      int b, t;
      out_row(a, mw + lane, ok, b, t);
      const int64_t pos = (a.pos_arr ? (ok ? a.pos_arr[b] : 0) : a.pos0) + t;
      p.posf = static_cast<float>(pos);
    }
  }
  if constexpr (EPI == EPI_F32) {
    const int col = n0 + half_col0<BN>(warp) + 4 * (lane & 3);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p.res[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.res && first_part && (p.sr.ok & (1u << i))) p.res[i] = ld_res4(a, p.sr, i, col);
    }
  }
  __syncwarp();   // the bias is visible to the whole warp
}

// The accumulator part: tacc = this warp's TMEM lanes at the tile's column 0.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, EpiPre<BN, EPI>& p, const uint16_t* sbias,
                                              uint32_t tacc, int n0, int ks, int warp, int lane, ChunkOut& co) {
  const bool use_bias = a.bias != nullptr && ks == 0;
  const int hf = warp >> 2;
  if constexpr (EPI == EPI_QKV_ROPE) {
    // heads of 64 columns; this warp takes half of them
    const bool rope = n0 < a.rope_cols;
    uint16_t* out = static_cast<uint16_t*>(a.out);
#pragma unroll 1
    for (int c = hf * (BN / 2); c < (hf + 1) * (BN / 2); c += 64) {
      uint32_t r0[32], r1[32];
      tmem_ld32(tacc + c, r0);
      tmem_ld32(tacc + c + 32, r1);
      tmem_ld2_wait(r0, r1);
      float x0[32], x1[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) { x0[i] = __uint_as_float(r0[i]); x1[i] = __uint_as_float(r1[i]); }
      if (use_bias) { add_bias32_smem(x0, sbias + c); add_bias32_smem(x1, sbias + c + 32); }
      if (rope) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float sn, cs;
          rope_sincos_fast(p.posf, a.inv_freq_hi[j], a.inv_freq_lo[j], &sn, &cs);
          const float u = x0[j], w = x1[j];
          x0[j] = u * cs - w * sn;
          x1[j] = w * cs + u * sn;
        }
      }
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint4* stg = stage_buf(co, lane);
        stage_bf16x32(stg, lane, part ? x1 : x0);
        if (co.tmD) {
          tma_flush(co, stg, lane, n0 + c + 32 * part);
        } else {
          __syncwarp();
          store_bf16_chunk(out, a.ld_out, p.sr, stg, lane, n0 + c + 32 * part);
          __syncwarp();
        }
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // units of 32 outputs: gate columns g + hh .., up columns g + 64 + hh ..
    constexpr int kUnits = BN / 64;
    uint16_t* out = static_cast<uint16_t*>(a.out);
#pragma unroll 1
    for (int u = hf * (kUnits / 2); u < (hf + 1) * (kUnits / 2); ++u) {
      const int g = (u >> 1) * 128, hh = (u & 1) * 32;
      uint32_t rg[32], ru[32];
      tmem_ld32(tacc + g + hh, rg);
      tmem_ld32(tacc + g + 64 + hh, ru);
      tmem_ld2_wait(rg, ru);
      float gv[32], uv[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) { gv[i] = __uint_as_float(rg[i]); uv[i] = __uint_as_float(ru[i]); }
      if (use_bias) { add_bias32_smem(gv, sbias + g + hh); add_bias32_smem(uv, sbias + g + 64 + hh); }
#pragma unroll
      for (int i = 0; i < 32; ++i) gv[i] = silu_f(gv[i]) * uv[i];
      uint4* stg = stage_buf(co, lane);
      stage_bf16x32(stg, lane, gv);
      if (co.tmD) {
        tma_flush(co, stg, lane, (n0 + g) / 2 + hh);
      } else {
        __syncwarp();
        store_bf16_chunk(out, a.ld_out, p.sr, stg, lane, (n0 + g) / 2 + hh);
        __syncwarp();
      }
    }
  } else {
    const bool use_res = EPI == EPI_F32 && a.res != nullptr && ks == 0;
    const int jj = lane & 3;
    const int c0 = half_col0<BN>(warp);
#pragma unroll 1
    for (int c = c0; c < c0 + BN / 2; c += 32) {
      uint32_t r[32];
      tmem_ld32(tacc + c, r);
      tmem_ld_wait_regs(r);
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      if (use_bias) add_bias32_smem(v, sbias + c);
      if constexpr (EPI == EPI_GELU_BF16) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
        uint4* stg = co.stg;   // no TMA stores for GELU outputs
        stage_bf16x32(stg, lane, v);
        __syncwarp();
        store_bf16_chunk(static_cast<uint16_t*>(a.out), a.ld_out, p.sr, stg, lane, n0 + c);
        __syncwarp();
      } else {
        float* out = static_cast<float*>(a.out);
        if constexpr (EPI == EPI_F32) out += ks * a.split_stride;
        if constexpr (EPI == EPI_GELU_F32) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
        }
#pragma unroll
        for (int h16 = 0; h16 < 32; h16 += 16) {
          uint4* stg = stage_buf(co, lane);
          stage_f32x16(stg, lane, v + h16);
          __syncwarp();
          float4 o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = stg[stg_slot((lane >> 2) + 8 * i, jj)];
            o[i] = make_float4(__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z), __uint_as_float(w.w));
            if constexpr (EPI == EPI_F32) {
              o[i].x += p.res[i].x; o[i].y += p.res[i].y; o[i].z += p.res[i].z; o[i].w += p.res[i].w;
            }
          }
          if (co.tmD) {
            if (use_res) {   // the residual went in column-wise: back into the same slots
#pragma unroll
              for (int i = 0; i < 4; ++i)
                stg[stg_slot((lane >> 2) + 8 * i, jj)] =
                    make_uint4(__float_as_uint(o[i].x), __float_as_uint(o[i].y), __float_as_uint(o[i].z),
                               __float_as_uint(o[i].w));
            }
            if constexpr (EPI == EPI_F32) {
              const int nxt = c + h16 + 16;
              if (use_res && nxt < c0 + BN / 2) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (p.sr.ok & (1u << i)) p.res[i] = ld_res4(a, p.sr, i, n0 + nxt + 4 * jj);
              }
            }
            tma_flush(co, stg, lane, n0 + c + h16);
            continue;
          }
          __syncwarp();
          const int col = n0 + c + h16 + 4 * jj;
          if constexpr (EPI == EPI_F32) {
            const int nxt = c + h16 + 16;   // the next 16 columns' residual, in flight during the stores
            if (use_res && nxt < c0 + BN / 2) {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (p.sr.ok & (1u << i)) p.res[i] = ld_res4(a, p.sr, i, n0 + nxt + 4 * jj);
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (p.sr.ok & (1u << i)) st_global_u4(out + p.sr.drow[i] * a.ld_out + col,
                                                  make_uint4(__float_as_uint(o[i].x), __float_as_uint(o[i].y),
                                                             __float_as_uint(o[i].z), __float_as_uint(o[i].w)));
        }
      }
    }
  }
}

// Work unit u -> (m tile, n tile, K split) in the launch's order (GemmArgs::order;
// the grouped order is only set without K splits).
__device__ __forceinline__ void unit_coords(const GemmArgs& a, int u, int m_tiles, int n_tiles, int& mt, int& nt,
                                            int& ks) {
  const int splits = a.k_splits;
  if (a.order == kOrderGrouped) {
    const int per = kOrderGroupRows * n_tiles;   // units of one group of row panels
    const int g = u / per, r = u - g * per;
    const int rem = m_tiles - g * kOrderGroupRows;
    const int gm = rem < kOrderGroupRows ? rem : kOrderGroupRows;
    mt = g * kOrderGroupRows + r % gm;
    nt = r / gm;
    ks = 0;
  } else if (a.order == kOrderNFastest) {
    nt = u % n_tiles;
    const int r = u / n_tiles;
    ks = r % splits;
    mt = r / splits;
  } else {
    mt = u % m_tiles;
    const int r = u / m_tiles;
    ks = r % splits;
    nt = r / splits;
  }
}

// A-operand coordinates of consecutive K blocks (GemmArgs: tap = kb /
// kb_per_tap, c = kb % kb_per_tap, x = (tap % a_stride) a_tap_ch + 64 c,
// y = m0 + tap / a_stride), advanced one block at a time.
struct ACoord {
  int tap, c, x0, y;
  __device__ __forceinline__ void set(const GemmArgs& a, int m0) {
    x0 = (tap % a.a_stride) * a.a_tap_ch;
    y = m0 + tap / a.a_stride;
  }
  __device__ __forceinline__ void start(const GemmArgs& a, int kb, int m0) {
    tap = kb / a.kb_per_tap;
    c = kb - tap * a.kb_per_tap;
    set(a, m0);
  }
  __device__ __forceinline__ int x() const { return x0 + c * kBK; }
  __device__ __forceinline__ void next(const GemmArgs& a, int m0) {
    if (++c == a.kb_per_tap) {
      c = 0;
      ++tap;
      set(a, m0);
    }
  }
};

// ---------------------------------------------------------------- 1 CTA --
template <int BN, int EPI>
struct OneCfg {
  static constexpr int kBBytes = BN * kBK * 2;
  using S = SmemCfg<kABytes + kBBytes, stg_bufs(EPI)>;
  static constexpr int kTmemCols = 2 * BN;   // two accumulators
};

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const __grid_constant__ GemmArgs a) {
  using C = OneCfg<BN, EPI>;
  constexpr int S = C::S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kABytes;
  uint8_t* stg_all = smem + C::S::kStg;
  uint16_t* sbias_all = reinterpret_cast<uint16_t*>(smem + C::S::kBias);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::S::kBars);
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
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), 8); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (a.tma_store) tma_prefetch_desc(&tmD);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  const int m_tiles = (a.M + kBM - 1) / kBM;
  const int splits = a.k_splits;
  const int num_tiles = m_tiles * (a.N / BN) * splits;
  const int nkb = a.K / kBK / splits;
  const int n_tiles = a.N / BN;
  auto decode = [&](int u, int& m0, int& n0, int& ks) {
    int mt, nt;
    unit_coords(a, u, m_tiles, n_tiles, mt, nt, ks);
    m0 = mt * kBM;
    n0 = nt * BN;
  };

  // The weights (B) do not depend on the previous kernel of the stream: the
  // producers start streaming the first stages' B tiles before waiting for
  // it.  Their completions may reach a full barrier before it is armed (a
  // barrier's transaction count may run negative within a phase).
  const int prod = producer_of(warp);
  int npre = 0;
  if (prod >= 0 && lane == 0 && blockIdx.x < num_tiles) {
    int m0, n0, ks;
    decode(blockIdx.x, m0, n0, ks);
    npre = nkb < S ? nkb : S;
    for (int i = prod; i < npre; i += 2)
      tma_load_2d(smem_addr(sB + i * C::kBBytes), &tmB, full(i), (ks * nkb + i) * kBK, n0);
  }
  // Inputs written by the previous kernel of the stream are read below.
  pdl_wait();
  pdl_trigger();

  if (prod >= 0) {
    // Producer `prod` fills the ring stages s with s % 2 == prod (so every
    // fill of a stage, and its drain below, belongs to one thread).
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;    // bit s: this thread filled stage s at least once
      uint32_t last_par = 0;  // bit s: parity of its last fill of stage s
      int it = 0;             // k-block iterations so far
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int m0, n0, ks;
        decode(tile, m0, n0, ks);
        ACoord ac;
        ac.start(a, ks * nkb, m0);
        bool ok = true;
        for (int i = 0; i < nkb; ++i, ++it) {
          if ((stage & 1) == prod) {
            if (!mbar_wait(empty(stage), phase ^ 1, wc, 1)) { ok = false; break; }
            mbar_arrive_expect_tx(full(stage), kABytes + C::kBBytes);
            tma_load_2d(smem_addr(sA + stage * kABytes), &tmA, full(stage), ac.x(), ac.y);
            if (it >= npre)   // the first npre B tiles are in flight already
              tma_load_2d(smem_addr(sB + stage * C::kBBytes), &tmB, full(stage), (ks * nkb + i) * kBK, n0);
            issued |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
          }
          ac.next(a, m0);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      // Wait (bounded, even after an abort) for the stages this thread armed.
      int zero = 0;
      WaitCtx dw = wc;
      dw.abort_flag = &zero;
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) mbar_wait(full(s), (last_par >> s) & 1u, dw, 5);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, BN, 0);
      // Descriptors of stage 0's A and B; a stage, and a 16-deep K step (32
      // bytes) inside the 128-byte swizzled rows, add to the address field
      // (address / 16, 14 bits: shared memory stays below 256 KB).
      const uint64_t desc_a0 = smem_desc_sw128(smem_addr(sA), 16, 1024);
      const uint64_t desc_b0 = smem_desc_sw128(smem_addr(sB), 16, 1024);
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
          const uint64_t da = desc_a0 + static_cast<uint32_t>(stage * (kABytes >> 4));
          const uint64_t db = desc_b0 + static_cast<uint32_t>(stage * (C::kBBytes >> 4));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) umma_bf16(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
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
    uint4* stg = reinterpret_cast<uint4*>(stg_all) + warp * (stg_bufs(EPI) * 128);
    int stg_n = 0;   // chunks this warp has stored (the staging buffers alternate across tiles)
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      int m0, n0, ks;
      decode(tile, m0, n0, ks);
      const int ab = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      uint16_t* sbias = sbias_all + warp * 256;
      EpiPre<BN, EPI> pre;
      epilogue_prepare<BN, EPI>(a, pre, sbias, m0, n0, ks, warp, lane);
      bool ok = mbar_wait(acc_full(ab), acc_par, wc, 4);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + ab * BN + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      ChunkOut co{a.tma_store ? &tmD : nullptr, m0 + (warp & 3) * 32, ks, stg, stg_bufs(EPI), stg_n};
      epilogue_tile<BN, EPI>(a, pre, sbias, tacc, n0, ks, warp, lane, co);
      stg_n = co.n;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(ab));
    }
    if (a.tma_store && lane == 0) bulk_wait_all();   // this warp's output stores are complete
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------- RMSNorm in the tail --
// A residual GEMM whose output feeds an RMSNorm normalises it in the same
// kernel: the O and down projections of the 4 x 3000 frame encoder have 235
// tiles for 74 CTA pairs, so most pairs sit idle through the last round, and
// their epilogue warps normalise the rows that are already complete instead.
// Each epilogue warp publishes its 32 rows of a tile (release add on the row
// group's counter once its stores are complete); a warp normalising two rows
// first waits (bounded) for their group's count to reach 2 per column tile.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// The group counter *c reaches target (bounded: false after the wait limit or
// once another wait of the CTA gave up).  Lane 0 polls.
__device__ __forceinline__ bool norm_wait_group(const int* c, int target, const WaitCtx& w, int lane) {
  int ok = 1;
  if (lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(c) < target) {
      if (*w.abort_flag) { ok = 0; break; }
      if (globaltimer_ns() - t0 > w.limit_ns) {
        *w.abort_flag = 1;
        report_timeout(w.status, 39);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) (void)ld_acquire(c);   // every lane acquires the stores it is about to read
  return ok != 0;
}

// Normalises rows two at a time (taken from the work counter) once their row
// group is complete: d = 1280 = 10 float4 per lane.
__device__ __forceinline__ void norm_tail_rows(const GemmArgs& a, int n_tiles, int lane, const WaitCtx& w) {
  constexpr int NV = 10;
  const int ngroups = (a.M + 31) >> 5;
  int* work = a.norm_ctr + ngroups;
  const int target = 2 * n_tiles;
  uint2 gw[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) gw[i] = __ldg(reinterpret_cast<const uint2*>(a.norm_g) + lane + 32 * i);
  const float* out = static_cast<const float*>(a.out);
  while (true) {
    int r0 = 0;
    if (lane == 0) r0 = atomicAdd(work, 2);
    r0 = __shfl_sync(0xffffffffu, r0, 0);
    if (r0 >= a.M) break;
    if (!norm_wait_group(a.norm_ctr + (r0 >> 5), target, w, lane)) break;
    const int nr = a.M - r0 < 2 ? a.M - r0 : 2;
    float4 v[2][NV];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      if (rr < nr) {
#pragma unroll
        for (int i = 0; i < NV; ++i)
          v[rr][i] = __ldcg(reinterpret_cast<const float4*>(out + static_cast<int64_t>(r0 + rr) * a.ld_out) + lane + 32 * i);
      }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      if (rr >= nr) break;
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i)
        ss = fmaf(v[rr][i].x, v[rr][i].x, fmaf(v[rr][i].y, v[rr][i].y, fmaf(v[rr][i].z, v[rr][i].z, fmaf(v[rr][i].w, v[rr][i].w, ss))));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = rsqrtf(ss / static_cast<float>(a.N) + a.norm_eps);
      const int64_t row = static_cast<int64_t>(r0 + rr) * a.N;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const float4 x = v[rr][i];
        const uint2 g = gw[i];
        const float o0 = x.x * inv * bf16lo(g.x), o1 = x.y * inv * bf16hi(g.x);
        const float o2 = x.z * inv * bf16lo(g.y), o3 = x.w * inv * bf16hi(g.y);
        if (a.norm_y_bf16) {
          reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.norm_y) + row)[lane + 32 * i] =
              make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
        } else {
          reinterpret_cast<float4*>(static_cast<float*>(a.norm_y) + row)[lane + 32 * i] = make_float4(o0, o1, o2, o3);
        }
      }
    }
  }
}

// ------------------------------------------------------------ CTA pairs --
// A cluster of two CTAs computes a 256 x BN tile with tcgen05.mma.cta_group::2
// (M = 256).  CTA r loads its own 128 rows of A and rows [r BN/2, (r+1) BN/2)
// of the tile's B rows; the leader (CTA 0) issues the MMAs.  TMA completions of
// both CTAs land on the leader's full barriers; MMA completions are multicast
// to the empty / accumulator barriers of both CTAs; both CTAs' epilogue warps
// release an accumulator on the leader's barrier.  Each CTA's epilogue handles
// its 128 rows x BN columns from its own TMEM.
template <int BN, int EPI>
struct PairCfg {
  static constexpr int kBHalfBytes = (BN / 2) * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBHalfBytes;
  using S = SmemCfg<kStageBytes, stg_bufs(EPI)>;
  static constexpr int kTmemCols = 2 * BN;
};

template <int BN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmD, const __grid_constant__ GemmArgs a) {
  using C = PairCfg<BN, EPI>;
  constexpr int S = C::S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kABytes;
  uint8_t* stg_all = smem + C::S::kStg;
  uint16_t* sbias_all = reinterpret_cast<uint16_t*>(smem + C::S::kBias);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::S::kBars);
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
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), 16); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (a.tma_store) tma_prefetch_desc(&tmD);
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtx wc{a.status, abort_flag, a.limit_ns};
  const int m_tiles = (a.M + 255) / 256;
  const int splits = a.k_splits;
  const int num_tiles = m_tiles * (a.N / BN) * splits;
  const int nkb = a.K / kBK / splits;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int n_tiles = a.N / BN;
  auto decode = [&](int u, int& m0, int& n0, int& ks) {
    int mt, nt;
    unit_coords(a, u, m_tiles, n_tiles, mt, nt, ks);
    m0 = mt * 256 + 128 * rank;
    n0 = nt * BN;
  };

  // The weights (B) do not depend on the previous kernel of the stream: the
  // producers of each CTA start streaming their halves of the first stages'
  // B tiles before waiting for it.  Their completions may reach the leader's
  // full barriers before they are armed (a barrier's transaction count may
  // run negative within a phase).
  const int prod = producer_of(warp);
  int npre = 0;
  if (prod >= 0 && lane == 0 && cluster < num_tiles) {
    int m0, n0, ks;
    decode(cluster, m0, n0, ks);
    npre = nkb < S ? nkb : S;
    for (int i = prod; i < npre; i += 2)
      tma_load_2d_pair(smem_addr(sB + i * C::kBHalfBytes), &tmB, map_to_cta(full(i), 0), (ks * nkb + i) * kBK,
                       n0 + (BN / 2) * rank);
  }
  // Inputs written by the previous kernel of the stream are read below.
  pdl_wait();
  pdl_trigger();

  if (prod >= 0) {
    // Producer `prod` fills the ring stages s with s % 2 == prod (so every
    // fill of a stage, and its drain below, belongs to one thread); the
    // leader's arms their full barriers for the pair's four copies.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      int it = 0;   // k-block iterations so far
      for (int tile = cluster; tile < num_tiles; tile += nclusters) {
        int m0, n0, ks;
        decode(tile, m0, n0, ks);
        ACoord ac;
        ac.start(a, ks * nkb, m0);
        bool ok = true;
        for (int i = 0; i < nkb; ++i, ++it) {
          if ((stage & 1) == prod) {
            if (!mbar_wait(empty(stage), phase ^ 1, wc, 31)) { ok = false; break; }
            const uint32_t fb = map_to_cta(full(stage), 0);   // the leader's full barrier
            if (rank == 0) mbar_arrive_expect_tx(full(stage), 2 * C::kStageBytes);
            tma_load_2d_pair(smem_addr(sA + stage * kABytes), &tmA, fb, ac.x(), ac.y);
            if (it >= npre)   // the first npre B tiles are in flight already
              tma_load_2d_pair(smem_addr(sB + stage * C::kBHalfBytes), &tmB, fb, (ks * nkb + i) * kBK,
                               n0 + (BN / 2) * rank);
            issued |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
          }
          ac.next(a, m0);
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
  } else if (warp == kMmaWarp) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, BN, 0);
      // Descriptors of stage 0's A and B; a stage, and a 16-deep K step (32
      // bytes) inside the 128-byte swizzled rows, add to the address field
      // (address / 16, 14 bits: shared memory stays below 256 KB).
      const uint64_t desc_a0 = smem_desc_sw128(smem_addr(sA), 16, 1024);
      const uint64_t desc_b0 = smem_desc_sw128(smem_addr(sB), 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
        const int ab = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(acc_empty(ab), acc_par ^ 1, wc, 32)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full(stage), phase, wc, 33)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = desc_a0 + static_cast<uint32_t>(stage * (kABytes >> 4));
          const uint64_t db = desc_b0 + static_cast<uint32_t>(stage * (C::kBHalfBytes >> 4));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) umma_bf16_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
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
    uint4* stg = reinterpret_cast<uint4*>(stg_all) + warp * (stg_bufs(EPI) * 128);
    int stg_n = 0;   // chunks this warp has stored (the staging buffers alternate across tiles)
    int local = 0;
    const uint32_t acc_empty_leader0 = map_to_cta(acc_empty(0), 0);
    const uint32_t acc_empty_leader1 = map_to_cta(acc_empty(1), 0);
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
      int m0, n0, ks;
      decode(tile, m0, n0, ks);
      const int ab = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      uint16_t* sbias = sbias_all + warp * 256;
      EpiPre<BN, EPI> pre;
      epilogue_prepare<BN, EPI>(a, pre, sbias, m0, n0, ks, warp, lane);
      bool ok = mbar_wait(acc_full(ab), acc_par, wc, 34);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + ab * BN + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      ChunkOut co{a.tma_store ? &tmD : nullptr, m0 + (warp & 3) * 32, ks, stg, stg_bufs(EPI), stg_n};
      epilogue_tile<BN, EPI>(a, pre, sbias, tacc, n0, ks, warp, lane, co);
      stg_n = co.n;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ab ? acc_empty_leader1 : acc_empty_leader0);
      if (EPI == EPI_F32 && a.norm_g) {   // publish this warp's 32 rows of the tile once stored
        if (!a.tma_store) __threadfence();
        __syncwarp();
        const int grp = (m0 + (warp & 3) * 32) >> 5;
        if (lane == 0) {
          if (a.tma_store) {
            bulk_wait_all();             // its TMA stores are complete ...
            fence_proxy_async_global();  // ... and ordered before the generic release below
          }
          __threadfence();
          if (grp < ((a.M + 31) >> 5)) red_release_add(a.norm_ctr + grp, 1);
        }
      }
    }
    if (a.tma_store && lane == 0) bulk_wait_all();   // this warp's output stores are complete
    if (EPI == EPI_F32 && a.norm_g && !*abort_flag) norm_tail_rows(a, n_tiles, lane, wc);
  }

  tc_fence_before();
  __syncthreads();
  if (EPI == EPI_F32 && a.norm_g && threadIdx.x == 0) {
    // The last CTA to finish sets the counters back to zero for the next launch.
    const int ngroups = (a.M + 31) >> 5;
    __threadfence();
    if (atomicAdd(a.norm_ctr + ngroups + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      for (int i = 0; i < ngroups + 2; ++i) a.norm_ctr[i] = 0;
      __threadfence();
    }
  }
  cluster_sync_all();   // no CTA of the pair still uses TMEM or the peer's barriers
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------- launchers --
template <int BN, int EPI>
cudaError_t launch_one(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                       const GemmArgs& a) {
  using C = OneCfg<BN, EPI>;
  const int tiles = ((a.M + kBM - 1) / kBM) * (a.N / BN) * a.k_splits;
  const int grid = tiles < L.sm_count ? tiles : L.sm_count;
  return launch_kernel(gemm_tc_kernel<BN, EPI>, dim3(grid), dim3(kThreads), C::S::kTotal, L.stream, tmA, tmB, tmD,
                       a);
}

template <int BN, int EPI>
cudaError_t launch_pair(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                        const GemmArgs& a) {
  using C = PairCfg<BN, EPI>;
  const int tiles = ((a.M + 255) / 256) * (a.N / BN) * a.k_splits;
  const int pairs = L.sm_count / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  return launch_kernel(gemm_tc2_kernel<BN, EPI>, dim3(grid), dim3(kThreads), C::S::kTotal, L.stream, tmA, tmB, tmD,
                       a);
}

template <int EPI>
cudaError_t launch_epi(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                       const GemmArgs& a, const GemmPlan& p) {
  if (p.pair) {
    if (p.bn == 256) return launch_pair<256, EPI>(L, tmA, tmB, tmD, a);
    if (p.bn == 128) return launch_pair<128, EPI>(L, tmA, tmB, tmD, a);
    return cudaErrorInvalidValue;
  }
  if (p.bn == 256) return launch_one<256, EPI>(L, tmA, tmB, tmD, a);
  if (p.bn == 128) return launch_one<128, EPI>(L, tmA, tmB, tmD, a);
  return cudaErrorInvalidValue;
}

}  // namespace

// Time model of one GEMM launch, used to choose among the shapes below.
// Measured on B200 (one CTA per SM, 64-wide K blocks):
//  * a tcgen05.mma with M = 128 rows per CTA and K = 16 takes ~73 ns for any
//    N <= 256, so a K block costs ~0.29 us whatever the tile width: only
//    N = 256 runs the tensor core at its peak;
//  * a TMA tile load costs ~0.13 us of the SM's copy engine (L2 source) to
//    ~0.17 us (HBM source), nearly independent of its size up to 48 KB, so a
//    K block (two loads) costs 0.27 - 0.34 us of copy time;
//  * HBM bounds the weight streaming of few-row GEMMs.
// A K-split adds the fp32 round trip of its partial sums through L2 and the
// last tile's epilogue is exposed.
static double plan_time_us(const GemmPlan& p, int M, int N, int K, int sm) {
  const int nkb = K / kBK / p.splits;
  const int rows = p.pair ? 256 : 128;
  const long units = static_cast<long>((M + rows - 1) / rows) * (N / p.bn) * p.splits;
  const long slots = p.pair ? sm / 2 : sm;
  const long waves = (units + slots - 1) / slots;
  const double kb_us = 0.30;
  const double hbm_us = (static_cast<double>(N) * K * 2 + static_cast<double>(M) * K * 2) / 6.5e6;
  const double split_us = p.splits > 1 ? static_cast<double>(p.splits) * M * N * 4 * 2 / 20e6 : 0.0;
  const double epi_us = 0.5 + 0.004 * p.bn;
  const double body = waves * nkb * kb_us;
  return (body > hbm_us ? body : hbm_us) + split_us + epi_us;
}

GemmPlan plan_gemm(int M, int N, int K, int epi, int max_splits, int sm) {
  GemmPlan best{false, 0, 1};
  double best_t = 1e30;
  const int nkb = K / kBK;
  const bool can_split = epi == EPI_F32;
  for (int pair = 1; pair >= 0; --pair) {
    for (int bn = 256; bn >= 128; bn /= 2) {
      if (N % bn != 0) continue;
      for (int s = 1; s <= (can_split ? max_splits : 1); s *= 2) {
        if (nkb % s != 0 || nkb / s < 2) break;
        const GemmPlan p{pair != 0, bn, s};
        const double t = plan_time_us(p, M, N, K, sm);
        if (t < best_t * 0.98) { best_t = t; best = p; }
      }
    }
  }
  return best;
}

cudaError_t launch_gemm(const Launch& L, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                        const GemmArgs& args, int epi, const GemmPlan& p) {
  if (args.M <= 0) return cudaSuccess;
  if (args.out == nullptr || args.k_splits != p.splits || p.splits < 1 || (args.K / kBK) % p.splits != 0 || args.K % kBK != 0 ||
      p.bn <= 0 || args.N % p.bn != 0 || (p.splits > 1 && epi != EPI_F32) ||
      (args.tma_store && epi != EPI_F32 && epi != EPI_QKV_ROPE && epi != EPI_SWIGLU) ||
      (args.norm_g && (epi != EPI_F32 || !p.pair || p.splits != 1 || args.N != 1280 || args.ld_out != args.N ||
                       !args.norm_y || !args.norm_ctr)))
    return cudaErrorInvalidValue;
  // Walk the work units so that the larger operand crosses DRAM once: A
  // goes first when it is the larger one and too large to stay in L2 while
  // it is walked once per column tile (the encoder's 123 MB down-projection
  // input read it ~2.5 times over in M-fastest order).  Activations of
  // 16-64 MB (the encoder's QKV, gate/up and O inputs) are walked in groups
  // of four row panels: measured on the 4 x 3000 frame encoder, the QKV
  // projection 148 -> 142 us against either plain order, the others
  // unchanged; a one-layer batch's 6-15 MB inputs keep the M-fastest order.
  GemmArgs a2 = args;
  const int64_t a_bytes = static_cast<int64_t>(args.M) * args.K * 2, b_bytes = static_cast<int64_t>(args.N) * args.K * 2;
  if (a_bytes > b_bytes && a_bytes >= (int64_t(64) << 20))
    a2.order = kOrderNFastest;
  else if (a_bytes >= (int64_t(16) << 20) && args.k_splits == 1)
    a2.order = kOrderGrouped;
  else
    a2.order = kOrderMFastest;
  const GemmArgs& a = a2;
  switch (epi) {
    case EPI_F32: return launch_epi<EPI_F32>(L, tmA, tmB, tmD, a, p);
    case EPI_QKV_ROPE: return launch_epi<EPI_QKV_ROPE>(L, tmA, tmB, tmD, a, p);
    case EPI_SWIGLU: return launch_epi<EPI_SWIGLU>(L, tmA, tmB, tmD, a, p);
    case EPI_GELU_BF16: return launch_epi<EPI_GELU_BF16>(L, tmA, tmB, tmD, a, p);
    case EPI_GELU_F32: return launch_epi<EPI_GELU_F32>(L, tmA, tmB, tmD, a, p);
    default: return cudaErrorInvalidValue;
  }
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
