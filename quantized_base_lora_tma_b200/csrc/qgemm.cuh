// Dequant-in-shared-memory tcgen05 GEMM: D[M, Nd] = A[M, Kd] * deq(W)^T-or-deq(W) (+ LoRA k-blocks).
//
// This is the base matmul of the layer (the recipe's llama.cpp-style quantized and grouped matmuls, Show HN: LoRA over
// GGUF, "Things involved in the training"; the fused dequant-matmul that expands packed weights on
// chip without an fp16 intermediate in memory, ai-manual.ru, "Fused dequant-matmul и MoE kernels").
// It is designed for sm_100a rather than after those kernels:
//
//   * TMA copies packed GGUF groups (256 weights of a row, 272 or 144 bytes) of W into a shared
//     memory ring; dequant warps expand them to bf16 directly in the 128-byte-swizzled canonical
//     UMMA layout of the B operand; the full-precision weight never exists in HBM.
//   * Forward (TRANS = false): B[n, k] = deq(W)[n, k], K-major. Input-gradient (TRANS = true):
//     B[k, n] = deq(W)[n, k] with the reduction over W's rows; the same decode writes an MN-major
//     tile. Tiles are BM x 128 with BM = 128 * MS: with MS = 2 every dequantized B tile feeds two
//     M = 128 MMAs (two TMEM accumulators), halving the dequant work per FLOP.
//   * The A operand (X or dY rows) arrives by TMA with the 128-byte swizzle.
//   * One elected thread issues tcgen05.mma (bf16 x bf16 -> fp32) into a double-buffered TMEM
//     accumulator; four epilogue warps drain it with tcgen05.ld while the next tile accumulates.
//   * The rank-r adapter product is folded in as extra 64-wide k-blocks: A-side [hi(v) | lo(v)]
//     (a bf16 pair whose sum carries v = s*H or G to ~2^-16 relative), B-side [Bop | Bop]; so the
//     LoRA term is accumulated by the tensor core into the same TMEM tile, in fp32.
//   * Grouped mode walks a device-side list of (expert, 128-row block) segments of a routed batch.
//   * Persistent: one CTA per SM loops over tiles. Every wait is bounded (ptx.cuh).
#pragma once
#include <cuda_bf16.h>

#include "decode.cuh"
#include "ptx.cuh"

namespace qlora {

enum EpiKind { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_PAIR_OUT = 2, EPI_SWIGLU_BWD = 3 };

constexpr int kBK = 64;
constexpr int kNumEpiWarps = 4;   // warps 0..3 (TMEM lane quadrants 0..3)
constexpr int kWarpTmaA = 4;
constexpr int kWarpMma = 5;
constexpr int kWarpTmaW = 6;
constexpr int kWarpDq0 = 7;
constexpr int kNumDqWarps = 16;  // two groups of eight, taking alternate stages
constexpr int kGemmThreads = (kWarpDq0 + kNumDqWarps) * 32;  // 736

// Adapter row products computed inside a dense pair-GEMM launch, by the clusters the tiles leave
// idle (see gemm2_rows_role): out = oscale Y Z^T and la = split(lscale Y Z^T) for the GEMM's A
// operand Y, plus LB and hs, with counters the LoRA k-blocks (and a later column reduction) wait on.
struct RowsFuse {
  int r, RP, nt;               // rank, padded rank (LA / LB are 2RP wide), 8-column tiles of Z^T
  int ztr;                     // the adapter box is [k][j] (j contiguous) rather than [j][k]
  int kc;                      // 64-wide k chunks per ring stage
  int stages;                  // TMA ring depth
  float oscale, lscale;
  float* out;                  // fp32 [M x r] (nullable)
  __nv_bfloat16* la;           // [M x 2RP] = [hi | lo]
  const __nv_bfloat16* lbz;    // LB[n] = [Z(n, :) | Z(n, :)], Z(n, j) = lbz[n lbzn + j lbzj] (nullable)
  long lbzn, lbzj;
  int lb_rows;
  __nv_bfloat16* lb;
  const float* hin;            // hs = split(hscale hin), [M x 2RP] (nullable)
  float hscale;
  __nv_bfloat16* hs;
  unsigned long long* ctr;  // tagged counters (seq): [0] CTAs whose LB / hs share is written,
                            // [1] CTAs done, [2 + mb] 128-row blocks of M block mb written
  unsigned seq;             // this launch's tag
  int* zc;                  // counters of a later launch, zeroed here (nullable)
  int zn;
};

struct GemmParams {
  int M;           // rows of the A operand (tokens; routed pairs in grouped mode)
  int Nd;          // output columns
  int Kd;          // quantized reduction length
  int n_lora_kb;   // extra 64-wide LoRA k-blocks
  int num_n_tiles;
  int num_m_blocks;  // dense mode: ceil(M / BM)
  int ksplit;        // dense mode: the K range of every output tile is split into ksplit parts
  int kb_per_split;  // k-blocks per part (a multiple of 4 in forward mode: whole raw groups)
  long split_stride; // ksplit > 1: part ks of the fp32 output starts at out + ks * split_stride
  // weight rows
  int w_rows_per_expert;  // rows of W per expert (grouped); 0 in dense mode
  int lb_rows_per_expert; // rows of the LoRA B operand per expert (grouped)
  int I;                  // SwiGLU: width of the gate (and up) half
  // grouped
  int E;                  // 0 = dense
  const int* seg_off;     // [E+1] first pair row of each expert
  const int* mblk_off;    // [E+1] prefix sum of ceil(count_e / BM)
  // epilogue
  void* out;
  int out_dtype;
  long ldo;
  float* out_gf;               // SWIGLU: g, u [M x I] in fp32 (the SwiGLU derivative takes them unrounded)
  float* out_uf;
  __nv_bfloat16* out_h;        // SWIGLU: bf16 h [M x I]
  __nv_bfloat16* out_g;        // SWIGLU_BWD: bf16 d[g|u] [M x 2I]
  __nv_bfloat16* out_lo;       // SWIGLU: h - bf16(h); SWIGLU_BWD: d[g|u] - bf16(d[g|u]) (nullable)
  const float* in_gf;          // SWIGLU_BWD: saved fp32 g, u [M x I]
  const float* in_uf;
  const float* row_w;          // PAIR_OUT, SWIGLU_BWD: routing weight per row
  float* dw_part;              // SWIGLU_BWD: [M x num_n_tiles] partial <dh_u, h>
  float2* row_stats;           // pair GEMM, fp32 output without K split (nullable): per row and
                               // column tile, (max, sum of exp(x - max)) of the tile's outputs
  // dense pair GEMM: clusters [0, rx) compute the adapter row products (0 = none: the LoRA
  // operands are the previous launch's output)
  int rx;
  RowsFuse rf;
};

// BN = 128 or 256 output columns per tile. With BN = 256 every A tile feeds twice the columns and
// each M = 128 MMA is N = 256, which needs a quarter less shared-memory operand bandwidth per FLOP:
// the single-CTA tile is bound by shared-memory bandwidth (the MMAs' operand reads plus the TMA and
// dequant traffic), not by the tensor pipe.
template <int QT, bool TRANS, int MS, int BN_ = 128>
struct GemmCfg {
  static constexpr int BM = 128 * MS;
  static constexpr int BN = BN_;
  static constexpr int GB = QTraits<QT>::kGroupBytes;
  static constexpr int A_BYTES = BM * kBK * 2;               // 16 / 32 KB
  static constexpr int B_BYTES = BN * kBK * 2;               // 16 / 32 KB
  static constexpr int RAW_ROWS = TRANS ? 64 : BN;           // W rows per raw chunk (one group each)
  static constexpr int RAW_BYTES = RAW_ROWS * GB;
  static constexpr int STAGES = (MS == 2 || BN == 256) ? 3 : 4;
  static constexpr int RAW_SLOTS = TRANS ? (GB > 200 ? 4 : 6) : (GB > 200 ? 2 : (BN == 256 ? 2 : 3));
  static constexpr int UNITS = BN / 128;                     // 32-weight units per dequant thread and stage
  static constexpr int MN_SBO = BN / 64 * 1024;              // MN-major B: bytes per 8 k-rows
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_RAW = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_RAW + RAW_SLOTS * RAW_BYTES;
  // barriers: full[S], empty[S], raw_full[R], raw_empty[R], tfull[2], tempty[2], drain, tmem ptr
  static constexpr int NUM_BARS = 2 * STAGES + 2 * RAW_SLOTS + 5;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;  // + alignment slack
  static constexpr int ACC_COLS = MS * BN;   // TMEM columns of one tile's accumulators
  static constexpr int TMEM_COLS = 512;      // two tiles in flight
  static_assert(2 * ACC_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(RAW_BYTES % 128 == 0, "raw slot alignment");
};

struct TileInfo {
  int row0;     // first A row
  int row_end;  // one past the last valid row
  int nb;       // output column block
  int e;        // expert (0 in dense mode)
  int ks;       // K part (0 without split)
  int kb_lo;    // first quantized k-block of this tile's part
  int kb_hi;    // one past the last
  int lora;     // this part also accumulates the LoRA k-blocks
};

template <int BM>
__device__ __forceinline__ bool gemm_tile(const GemmParams& p, int t, TileInfo& ti) {
  const int kb_main = p.Kd / kBK;
  if (p.E == 0) {
    if (t >= p.num_m_blocks * p.num_n_tiles * p.ksplit) return false;
    ti.ks = t % p.ksplit;
    const int rest = t / p.ksplit;
    const int mb = rest % p.num_m_blocks;
    ti.nb = rest / p.num_m_blocks;
    ti.row0 = mb * BM;
    ti.row_end = p.M;
    ti.e = 0;
    ti.kb_lo = ti.ks * p.kb_per_split;
    ti.kb_hi = min(kb_main, ti.kb_lo + p.kb_per_split);
    ti.lora = ti.ks == p.ksplit - 1;
    return true;
  }
  ti.ks = 0;
  ti.kb_lo = 0;
  ti.kb_hi = kb_main;
  ti.lora = 1;
  const int total_mb = __ldg(p.mblk_off + p.E);
  if (t >= total_mb * p.num_n_tiles) return false;
  // the output-column tiles of one 128-row block are consecutive: their A rows are read from L2
  const int gm = t / p.num_n_tiles;
  ti.nb = t - gm * p.num_n_tiles;
  // last expert e with mblk_off[e] <= gm
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.mblk_off + mid) <= gm) lo = mid; else hi = mid - 1;
  }
  ti.e = lo;
  ti.row0 = __ldg(p.seg_off + lo) + (gm - __ldg(p.mblk_off + lo)) * BM;
  ti.row_end = min(__ldg(p.seg_off + lo + 1), p.M);  // rows past M are never written
  if (ti.row0 < 0) ti.row0 = 0;
  return true;
}

// All 32 lanes wait; the outcome is made warp-uniform.
template <bool CLUSTER = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int site) {
  const bool r = mbar_wait<CLUSTER>(bar, parity, site);
  return __all_sync(0xffffffffu, r);
}

// 8 fp32 values as a bf16 pair per value: hi = RNE_bf16(f), lo = RNE_bf16(f - hi).
__device__ __forceinline__ void split_bf16x8(const float (&f)[8], uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    h[j] = __bfloat162float(__float2bfloat16_rn(f[j]));
    l[j] = f[j] - h[j];
  }
  hi = pack_bf16x8(h);
  lo = pack_bf16x8(l);
}

// sigma(g) = 1 / (1 + e^-g) from the fast exponential and a fast reciprocal: relative error of order
// 1e-6 for the gate values that occur, far below the bf16 resolution of what the epilogues store;
// e^-g = inf (g < -88) gives 0 and e^-g = 0 gives 1.
__device__ __forceinline__ float sigmoid_fast(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_fast(g); }

// Store epilogue of the pair GEMM: this thread owns output row `row` (valid or not: the TMEM loads
// are warp-collective) and reads BN fp32 columns starting at TMEM address tbase; 64 bytes of bf16
// (or 128 of fp32) of its row per 32 columns.
template <int BN>
__device__ __forceinline__ void epilogue_rows_store(const GemmParams& p, const TileInfo& ti, int row, bool valid,
                                                  uint32_t tbase) {
  const bool split = p.ksplit > 1;  // fp32 partial of K part ti.ks
  const bool stats = p.row_stats != nullptr;
  float sm = -INFINITY, ss = 0.0f;  // the row's running max and sum of exp(x - max) over the tile
#pragma unroll 1
  for (int jc = 0; jc < BN / 32; ++jc) {
    uint32_t v[32];
    tmem_ld32(tbase + 32 * jc, v);
    tmem_ld_wait();
    const int col0 = ti.nb * BN + 32 * jc;
    if (stats && valid && col0 < p.Nd) {
      float bm = __uint_as_float(v[0]);
#pragma unroll
      for (int i = 1; i < 32; ++i) bm = fmaxf(bm, __uint_as_float(v[i]));
      const float nm = fmaxf(sm, bm);
      float acc = sm == -INFINITY ? 0.0f : ss * expf(sm - nm);
#pragma unroll
      for (int i = 0; i < 32; ++i) acc += expf(__uint_as_float(v[i]) - nm);
      sm = nm;
      ss = acc;
    }
    if (valid && col0 < p.Nd) {
      if (p.out_dtype == QL_F32 || split) {
        float* base = reinterpret_cast<float*>(p.out) + (split ? ti.ks * p.split_stride : 0);
        float4* o = reinterpret_cast<float4*>(base + (long)row * p.ldo + col0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                             __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
      } else {
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + (long)row * p.ldo + col0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = __uint_as_float(v[8 * i + j]);
          o[i] = pack_bf16x8(f);
        }
      }
    }
  }
  if (stats && valid) p.row_stats[(long)row * p.num_n_tiles + ti.nb] = make_float2(sm, ss);
}

// SwiGLU-backward epilogue, one accumulator row per thread (32x32b TMEM loads, 16 columns per
// batch): its outputs are bf16, for which the 16x256b shape gains nothing per byte stored and
// needs twice the store instructions.
template <int BN>
__device__ __forceinline__ void epilogue_rows_swiglu_bwd(const GemmParams& p, const TileInfo& ti, int row, bool valid,
                                                         uint32_t tbase) {
  // dh_u = accumulator; dh = w dh_u; the SwiGLU derivative from the saved fp32 g, u; <dh_u, h>
  // with h = silu(g) u recomputed at fp32 accuracy. The saved g, u are read-only here: 16 columns
  // of both are loaded together ahead of the arithmetic and stores, one memory latency per batch.
  const float* __restrict__ gin = p.in_gf;
  const float* __restrict__ uin = p.in_uf;
  __nv_bfloat16* __restrict__ go = p.out_g;
  __nv_bfloat16* __restrict__ gl = p.out_lo;
  float wr = 0.0f, dwp = 0.0f;
  if (valid) wr = __ldg(p.row_w + row);
  // the g and u of a batch are asked of L2 kPf batches ahead, so each batch's loads find them
  // there instead of waiting a full memory latency (64 bytes of each per batch and row)
  constexpr int kPf = 3;
  auto prefetch_batch = [&](int jc) {
    const int j0 = ti.nb * BN + 16 * jc;
    if (valid && jc < BN / 16 && j0 < p.I) {
      prefetch_l2(gin + (long)row * p.I + j0);
      prefetch_l2(uin + (long)row * p.I + j0);
    }
  };
#pragma unroll
  for (int jc = 0; jc < kPf; ++jc) prefetch_batch(jc);
#pragma unroll 1
  for (int jc = 0; jc < BN / 16; ++jc) {
    prefetch_batch(jc + kPf);
    uint32_t v[16];
    tmem_ld16(tbase + 16 * jc, v);
    const int j0 = ti.nb * BN + 16 * jc;
    const bool act = valid && j0 < p.I;
    float4 gq[4], uq[4];
    if (act) {
      const float4* g4 = reinterpret_cast<const float4*>(gin + (long)row * p.I + j0);
      const float4* u4 = reinterpret_cast<const float4*>(uin + (long)row * p.I + j0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gq[q] = __ldg(g4 + q);
        uq[q] = __ldg(u4 + q);
      }
    }
    tmem_ld_wait();
    if (act) {
      const float* gf = reinterpret_cast<const float*>(gq);
      const float* uf = reinterpret_cast<const float*>(uq);
      const long od = (long)row * 2 * p.I + j0;
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        float dg[8], du[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float a = __uint_as_float(v[8 * hlf + j]);
          const float g = gf[8 * hlf + j], u = uf[8 * hlf + j];
          const float sg = sigmoid_fast(g);
          const float dh = wr * a;
          const float sl = g * sg;  // silu(g)
          dg[j] = dh * u * sg * (1.0f + g * (1.0f - sg));
          du[j] = dh * sl;
          // <dh_u, h> with h at fp32 accuracy: a flip of a bf16 h would move a heavy-tailed term
          dwp = fmaf(a, sl * u, dwp);
        }
        uint4 gh, glo, uh, ulo;
        split_bf16x8(dg, gh, glo);
        split_bf16x8(du, uh, ulo);
        *reinterpret_cast<uint4*>(go + od + 8 * hlf) = gh;
        *reinterpret_cast<uint4*>(go + od + p.I + 8 * hlf) = uh;
        if (gl != nullptr) {
          *reinterpret_cast<uint4*>(gl + od + 8 * hlf) = glo;
          *reinterpret_cast<uint4*>(gl + od + p.I + 8 * hlf) = ulo;
        }
      }
    }
  }
  if (valid) p.dw_part[(long)row * p.num_n_tiles + ti.nb] = dwp;
}

__device__ __forceinline__ uint32_t bf16x2_of(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Epilogue of one warp's 32 accumulator rows (rows rbase .. rbase + 31 of the tile, TMEM address tw
// at the first of them and the tile's first column). The rows are read as two halves of 16 lanes
// with the 16x256b shape: a thread holds rows a = rbase + 16 half + lane/4 and b = a + 8, two
// adjacent columns 2(lane%4), +1 of every group of 8. Four consecutive lanes thus cover 8
// consecutive columns of a row, so every global access of a warp moves whole 32-byte sectors of
// 8 rows rather than half sectors of 32 rows.
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_warp(const GemmParams& p, const TileInfo& ti, int rbase, uint32_t tw) {
  const int lane = threadIdx.x & 31;
  const int cc = 2 * (lane & 3);
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    const int ra = rbase + 16 * half + (lane >> 2), rb = ra + 8;
    const bool va = ra < ti.row_end, vb = rb < ti.row_end;
    const uint32_t th = tw + ((uint32_t)(16 * half) << 16);
    if (EPI == EPI_STORE || EPI == EPI_PAIR_OUT) {
      float wa = 1.0f, wb = 1.0f;
      if (EPI == EPI_PAIR_OUT) {
        if (va) wa = __ldg(p.row_w + ra);
        if (vb) wb = __ldg(p.row_w + rb);
      }
      const bool split = p.ksplit > 1;  // fp32 partial of K part ti.ks
      const bool f32 = p.out_dtype == QL_F32 || split;
#pragma unroll 1
      for (int jc = 0; jc < BN / 32; ++jc) {
        uint32_t v[16];
        tmem_ld_16x256_x4(th + 32 * jc, v);
        tmem_ld_wait();
        const int col0 = ti.nb * BN + 32 * jc;
        if (col0 >= p.Nd) continue;
        if (f32) {
          float* base = reinterpret_cast<float*>(p.out) + (split ? ti.ks * p.split_stride : 0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = col0 + 8 * q + cc;
            if (va)
              *reinterpret_cast<float2*>(base + (long)ra * p.ldo + col) =
                  make_float2(wa * __uint_as_float(v[4 * q]), wa * __uint_as_float(v[4 * q + 1]));
            if (vb)
              *reinterpret_cast<float2*>(base + (long)rb * p.ldo + col) =
                  make_float2(wb * __uint_as_float(v[4 * q + 2]), wb * __uint_as_float(v[4 * q + 3]));
          }
        } else {
          __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = col0 + 8 * q + cc;
            if (va)
              *reinterpret_cast<uint32_t*>(base + (long)ra * p.ldo + col) =
                  bf16x2_of(wa * __uint_as_float(v[4 * q]), wa * __uint_as_float(v[4 * q + 1]));
            if (vb)
              *reinterpret_cast<uint32_t*>(base + (long)rb * p.ldo + col) =
                  bf16x2_of(wb * __uint_as_float(v[4 * q + 2]), wb * __uint_as_float(v[4 * q + 3]));
          }
        }
      }
    } else if (EPI == EPI_SWIGLU) {
      // tile columns [0, BN/2) are gate j = nb*BN/2 + c, [BN/2, BN) are up for the same j; 32 j at a time
#pragma unroll 1
      for (int jp = 0; jp < BN / 64; ++jp) {
        uint32_t vg[16], vu[16];
        tmem_ld_16x256_x4(th + 32 * jp, vg);
        tmem_ld_16x256_x4(th + BN / 2 + 32 * jp, vu);
        tmem_ld_wait();
        const int j0 = ti.nb * (BN / 2) + 32 * jp;
        if (j0 >= p.I) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int row = rr ? rb : ra;
            if (!(rr ? vb : va)) continue;
            const float g0 = __uint_as_float(vg[4 * q + 2 * rr]), g1 = __uint_as_float(vg[4 * q + 2 * rr + 1]);
            const float u0 = __uint_as_float(vu[4 * q + 2 * rr]), u1 = __uint_as_float(vu[4 * q + 2 * rr + 1]);
            const float h0 = silu_f(g0) * u0, h1 = silu_f(g1) * u1;
            const long o = (long)row * p.I + j0 + 8 * q + cc;
            *reinterpret_cast<float2*>(p.out_gf + o) = make_float2(g0, g1);
            *reinterpret_cast<float2*>(p.out_uf + o) = make_float2(u0, u1);
            const __nv_bfloat162 hh = __floats2bfloat162_rn(h0, h1);
            *reinterpret_cast<__nv_bfloat162*>(p.out_h + o) = hh;
            if (p.out_lo != nullptr)
              *reinterpret_cast<uint32_t*>(p.out_lo + o) =
                  bf16x2_of(h0 - __low2float(hh), h1 - __high2float(hh));
          }
        }
      }

    }
  }
}

template <int QT, bool TRANS, int EPI, int MS, int BN_ = 128>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmLB,
                 const GemmParams p) {
  using C = GemmCfg<QT, TRANS, MS, BN_>;
  constexpr int BN = C::BN;
  constexpr int BM = C::BM;
  extern __shared__ uint8_t smem_raw_[];
  const uint32_t base_u32 = (smem_u32(smem_raw_) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw_ + (base_u32 - smem_u32(smem_raw_));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t sA = base_u32 + C::OFF_A;
  const uint32_t sB = base_u32 + C::OFF_B;
  const uint32_t sRaw = base_u32 + C::OFF_RAW;
  const uint32_t bar0 = base_u32 + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto rfull_bar = [&](int s) { return bar0 + 8u * (2 * C::STAGES + s); };
  auto rempty_bar = [&](int s) { return bar0 + 8u * (2 * C::STAGES + C::RAW_SLOTS + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 * C::RAW_SLOTS + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 * C::RAW_SLOTS + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 2 * C::RAW_SLOTS + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NUM_BARS * 8);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1 + kNumDqWarps / 2);  // TMA + the warps of one group
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < C::RAW_SLOTS; ++s) {
      mbar_init(rfull_bar(s), 1);
      mbar_init(rempty_bar(s), TRANS ? kNumDqWarps / 2 : kNumDqWarps);  // every reader of the chunk
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kNumEpiWarps);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kWarpTmaA && lane == 0) {
    prefetch_tmap(&tmA);
    if (p.n_lora_kb) { prefetch_tmap(&tmLA); prefetch_tmap(&tmLB); }
  }
  if (warp == kWarpTmaW && lane == 0) prefetch_tmap(&tmW);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  pdl_launch_dependents();  // after the wait: a dependent may rely on what this launch waited for

  const int kb_main = p.Kd / kBK;
  // k-block of step i of a tile: its quantized part first, then (if it carries them) the LoRA blocks
  auto tile_steps = [&](const TileInfo& ti) { return (ti.kb_hi - ti.kb_lo) + (ti.lora ? p.n_lora_kb : 0); };
  auto step_kb = [&](const TileInfo& ti, int i) {
    const int nq = ti.kb_hi - ti.kb_lo;
    return i < nq ? ti.kb_lo + i : kb_main + (i - nq);
  };

  if (warp == kWarpTmaA) {
    // ---------------- A operand (and LoRA operands) producer ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      int last_phase[8];
      for (int s = 0; s < C::STAGES; ++s) last_phase[s] = -1;
      TileInfo ti;
      for (int t = blockIdx.x; ok && gemm_tile<BM>(p, t, ti); t += gridDim.x) {
        const int nsteps = tile_steps(ti);
        for (int i = 0; i < nsteps; ++i, ++it) {
          const int kb = step_kb(ti, i);
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, 1)) { ok = false; break; }
          if (kb < kb_main) {
            mbar_arrive_expect_tx(full_bar(s), C::A_BYTES);
            tma_load_2d(sA + s * C::A_BYTES, &tmA, full_bar(s), kb * kBK, ti.row0);
          } else {
            const int x = (kb - kb_main) * kBK;
            mbar_arrive_expect_tx(full_bar(s), C::A_BYTES + C::B_BYTES);
            tma_load_2d(sA + s * C::A_BYTES, &tmLA, full_bar(s), x, ti.row0);
            const int lb0 = ti.e * p.lb_rows_per_expert;
#pragma unroll
            for (int i = 0; i < BN / 64; ++i) {
              int y;
              // SWIGLU tiles: columns [0, BN/2) are gate rows, [BN/2, BN) the up rows of the same j
              if (EPI == EPI_SWIGLU)
                y = lb0 + (i < BN / 128 ? ti.nb * (BN / 2) + 64 * i : p.I + ti.nb * (BN / 2) + 64 * (i - BN / 128));
              else y = lb0 + ti.nb * BN + 64 * i;
              tma_load_2d(sB + s * C::B_BYTES + i * 64 * 128, &tmLB, full_bar(s), x, y);
            }
          }
          last_phase[s] = (int)ph;
        }
      }
      if (!ok) {  // let copies already issued land before the CTA can exit
        for (int s = 0; s < C::STAGES; ++s)
          if (last_phase[s] >= 0) mbar_wait(full_bar(s), (uint32_t)last_phase[s], 0, false, 2000000ull);
      }
    }
  } else if (warp == kWarpTmaW) {
    // ---------------- packed weight producer ----------------
    if (lane == 0) {
      int rc = 0;
      bool ok = true;
      int last_phase[8];
      for (int s = 0; s < C::RAW_SLOTS; ++s) last_phase[s] = -1;
      constexpr int GW = C::GB / 4;  // group width in 32-bit words
      TileInfo ti;
      for (int t = blockIdx.x; ok && gemm_tile<BM>(p, t, ti); t += gridDim.x) {
        const int wbase = ti.e * p.w_rows_per_expert;
        const int c_lo = TRANS ? ti.kb_lo : ti.kb_lo / 4;
        const int c_hi = TRANS ? ti.kb_hi : ti.kb_hi / 4;
        for (int c = c_lo; c < c_hi; ++c, ++rc) {
          const int s = rc % C::RAW_SLOTS;
          const uint32_t ph = (rc / C::RAW_SLOTS) & 1;
          if (!mbar_wait(rempty_bar(s), ph ^ 1, 2)) { ok = false; break; }
          mbar_arrive_expect_tx(rfull_bar(s), C::RAW_BYTES);
          const uint32_t dst = sRaw + s * C::RAW_BYTES;
          if (TRANS) {
            // the 256-column group holding the tile's columns
            tma_load_2d(dst, &tmW, rfull_bar(s), (ti.nb * BN / 256) * GW, wbase + c * 64);
          } else {
            // BN rows of W in 64-row boxes (SWIGLU: BN/2 gate rows, then the BN/2 up rows)
#pragma unroll
            for (int b = 0; b < BN / 64; ++b) {
              int y;
              if (EPI == EPI_SWIGLU)
                y = wbase + (b < BN / 128 ? ti.nb * (BN / 2) + 64 * b : p.I + ti.nb * (BN / 2) + 64 * (b - BN / 128));
              else y = wbase + ti.nb * BN + 64 * b;
              tma_load_2d(dst + b * 64 * C::GB, &tmW, rfull_bar(s), c * GW, y);
            }
          }
          last_phase[s] = (int)ph;
        }
      }
      if (!ok) {
        for (int s = 0; s < C::RAW_SLOTS; ++s)
          if (last_phase[s] >= 0) mbar_wait(rfull_bar(s), (uint32_t)last_phase[s], 0, false, 2000000ull);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------- tensor-core issuer ----------------
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      bool issued = false;
      TileInfo ti;
      constexpr uint32_t idesc_main = idesc_bf16(128, BN, TRANS);
      constexpr uint32_t idesc_kmaj = idesc_bf16(128, BN, false);
      for (int t = blockIdx.x; ok && gemm_tile<BM>(p, t, ti); t += gridDim.x, ++tc) {
        const int buf = tc & 1;
        if (!mbar_wait(tempty_bar(buf), ((tc >> 1) & 1) ^ 1, 3)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * C::ACC_COLS;
        const int nsteps = tile_steps(ti);
        for (int i = 0; i < nsteps; ++i, ++it) {
          const int kb = step_kb(ti, i);
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(full_bar(s), ph, 4)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = sA + s * C::A_BYTES;
          const uint32_t b0 = sB + s * C::B_BYTES;
          const bool kmaj = !TRANS || kb >= kb_main;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            uint64_t bd;
            if (kmaj) bd = smem_desc_sw128(b0 + 32 * k, 16, 1024);
            else bd = smem_desc_sw128(b0 + 2 * C::MN_SBO * k, 1024, C::MN_SBO);
#pragma unroll
            for (int h = 0; h < MS; ++h) {
              const uint64_t ad = smem_desc_sw128(a0 + h * 16384 + 32 * k, 16, 1024);
              umma_bf16(d_tmem + h * BN, ad, bd, kmaj ? idesc_kmaj : idesc_main, (i | k) != 0);
            }
          }
          umma_commit(empty_bar(s));
          issued = true;
        }
        if (!ok) break;
        umma_commit(tfull_bar(buf));
      }
      if (issued) {  // every MMA issued has completed before TMEM can be released
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, 0, false, 2000000ull);
      }
    }
  } else if (warp >= kWarpDq0) {
    // ---------------- dequant workers ----------------
    // Two groups of eight warps take alternate stages, so one group's fence and barrier round
    // trip overlaps the other group's decoding, and eight warps per group hide the latency of
    // the decode's dependent chains. Each thread decodes one 32-weight unit per stage.
    const int dq = threadIdx.x - kWarpDq0 * 32;  // 0..511
    const int grp = dq >> 8;                     // stage parity this group handles
    const int gt = dq & 255;                     // thread within the group
    int it = 0, rc = 0;
    bool ok = true;
    TileInfo ti;
    for (int t = blockIdx.x; ok && gemm_tile<BM>(p, t, ti); t += gridDim.x) {
      if (!TRANS) {
        for (int g = ti.kb_lo / 4; ok && g < ti.kb_hi / 4; ++g, ++rc) {
          const int rs = rc % C::RAW_SLOTS;
          if (!warp_wait(rfull_bar(rs), (rc / C::RAW_SLOTS) & 1, 5)) { ok = false; break; }
          const uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_BYTES;
          for (int sub = 0; sub < 4; ++sub, ++it) {
            if ((it & 1) != grp) continue;
            const int s = it % C::STAGES;
            if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 6)) { ok = false; break; }
            uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
#pragma unroll
            for (int u = 0; u < C::UNITS; ++u) {
              // row gt/2 (+ 128 u) of the tile, 32-weight unit 2*sub + gt%2 of the group
              const int row = (gt >> 1) + 128 * u, uh = gt & 1;
              uint4 v[4];
              decode_unit_bf16<QT>(raw + row * C::GB, 2 * sub + uh, v);
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                const int c8 = 4 * uh + cc;
                *reinterpret_cast<uint4*>(sb + row * 128 + ((c8 ^ (row & 7)) << 4)) = v[cc];
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(full_bar(s));
          }
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(rempty_bar(rs));
        }
      } else {
        for (int kb = ti.kb_lo; ok && kb < ti.kb_hi; ++kb, ++rc, ++it) {
          if ((it & 1) != grp) continue;
          const int rs = rc % C::RAW_SLOTS;
          if (!warp_wait(rfull_bar(rs), (rc / C::RAW_SLOTS) & 1, 5)) { ok = false; break; }
          const int s = it % C::STAGES;
          if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 6)) { ok = false; break; }
          const uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_BYTES;
          uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
#pragma unroll
          for (int u = 0; u < C::UNITS; ++u) {
            // 32-column unit: row kk = gt/4 of the chunk, unit 4u + gt%4 of the tile's columns; the
            // tile's BN columns are (part of) the 256-column group: unit 4 (nb & 1) + ... for BN = 128
            const int kk = gt >> 2, ul = 4 * u + (gt & 3);
            const int gunit = BN == 256 ? ul : 4 * (ti.nb & 1) + ul;
            uint4 v[4];
            decode_unit_bf16<QT>(raw + kk * C::GB, gunit, v);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int gc = 4 * ul + cc;  // 16-byte chunk within the tile's BN columns
              const int off = (kk >> 3) * C::MN_SBO + (gc >> 3) * 1024 + (kk & 7) * 128 + (((gc & 7) ^ (kk & 7)) << 4);
              *reinterpret_cast<uint4*>(sb + off) = v[cc];
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(full_bar(s));
            mbar_arrive(rempty_bar(rs));
          }
        }
      }
      // LoRA k-blocks: operands come by TMA; the group whose turn it is accounts for the stage.
      for (int i = 0; ok && ti.lora && i < p.n_lora_kb; ++i, ++it) {
        if ((it & 1) != grp) continue;
        const int s = it % C::STAGES;
        if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 7)) { ok = false; break; }
        __syncwarp();
        if (lane == 0) mbar_arrive(full_bar(s));
      }
    }
  } else if (warp < kNumEpiWarps) {
    // ---------------- epilogue ----------------
    int tc = 0;
    TileInfo ti;
    for (int t = blockIdx.x; gemm_tile<BM>(p, t, ti); t += gridDim.x, ++tc) {
      const int buf = tc & 1;
      if (!warp_wait(tfull_bar(buf), (tc >> 1) & 1, 8)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < MS; ++h) {
        const uint32_t tw = tmem_base + ((uint32_t)(warp * 32) << 16) + buf * C::ACC_COLS + h * BN;
        if (EPI == EPI_SWIGLU_BWD) {
          const int row = ti.row0 + h * 128 + warp * 32 + lane;
          epilogue_rows_swiglu_bwd<BN>(p, ti, row, row < ti.row_end, tw);
        } else {
          epilogue_warp<EPI, BN>(p, ti, ti.row0 + h * 128 + warp * 32, tw);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
