// Pair (two-CTA) dequant-in-shared-memory GEMM for the dense layer: D = A deq(W)^T (forward) or
// A deq(W) (input gradient), plus the LoRA k-blocks, on 256 x 256 output tiles computed by a CTA pair
// with tcgen05.mma.cta_group::2.
//
// Why pairs: with 128-wide N tiles every CTA streams its A rows once per 128 output columns and the
// A ring cannot cover the TMA latency within shared memory. A pair tile holds A split by M (each CTA
// its own 128 rows) and B split by N (each CTA dequantizes its own 128 W rows, or its own 128 of
// the output columns in the input-gradient direction), so per SM the bytes moved per FLOP halve and
// the freed shared memory deepens the ring. Each CTA keeps its own producers (TMA for its A rows and
// its packed groups, sixteen dequant warps); the leader CTA (rank 0) issues the pair MMAs, which
// read both CTAs' shared memory and write both CTAs' TMEM (each its own 128 rows x 256 columns).
//
// Barrier protocol (full barriers live in the leader):
//   full[s]   leader: 1 arrive.expect_tx (both CTAs' TMA bytes, plus 16 signal bytes per peer
//             dequant warp on quantized steps) + the leader's dequant group. The peer's TMA copies
//             complete_tx on the leader's barrier; each peer dequant warp, once its part of the B half
//             is written and fenced for the async proxy, signals by a 16-byte bulk copy into the
//             leader that also completes tx there. Counting the peer through the copy engine keeps a
//             cluster-scope release fence (which costs about a thousand cycles) off the per-stage path.
//   empty[s]  each CTA: one pair commit arriving on both CTAs
//   tfull[b]  each CTA: one pair commit arriving on both; tempty[b] leader: 4 + 4 epilogue warps
// Every wait is bounded (ptx.cuh); both CTAs always reach the final cluster barrier.
#pragma once
#include "lora.cuh"
#include "qgemm.cuh"

namespace qlora {

// Warp roles. The MMA issuer (warp 5) runs on scheduler 1 (warp % 4 == 1); no dequant warp is
// placed there, so the issuer's short dependent chain between stages is not starved of issue slots
// by decode arithmetic. Dequant warps are the warps 7..27 with warp % 4 != 1 (sixteen of them);
// warps 9, 13, 17, 21, 25 have no role and wait at the final barrier.
constexpr int kGemm2Warps = 28;
constexpr int kGemm2Threads = kGemm2Warps * 32;  // 896
__device__ __forceinline__ int gemm2_dq_warp(int warp) {  // ordinal of a dequant warp, or -1
  if (warp < kWarpDq0 || (warp & 3) == 1) return -1;
  const int q = warp - kWarpDq0;
  return q - (q + 1) / 4;
}

// MS = 1: 256 x 256 pair tiles (each CTA 128 A rows), double-buffered accumulators.
// MS = 2: 512 x 256 pair tiles: each CTA holds two 128-row A blocks per stage and every dequantized
// B half feeds two pair MMAs (half the dequant work per FLOP); the two accumulators fill TMEM, so
// the epilogue of a tile is not overlapped with the next tile's main loop.
template <int QT, bool TRANS, int MS>
struct Gemm2Cfg {
  static constexpr int BN = 256;                 // pair tile N (output columns)
  static constexpr int HN = 128;                 // this CTA's half of N
  static constexpr int BM = 256 * MS;            // pair tile M
  static constexpr int GB = QTraits<QT>::kGroupBytes;
  static constexpr int A_BYTES = MS * 128 * kBK * 2;  // 16 / 32 KB
  static constexpr int B_BYTES = HN * kBK * 2;   // 16 KB
  static constexpr int RAW_ROWS = TRANS ? 64 : 128;
  static constexpr int RAW_BYTES = RAW_ROWS * GB;
  static constexpr int STAGES = MS == 2 ? 3 : (GB > 150 ? 4 : 5);
  static constexpr int RAW_SLOTS = TRANS ? (GB > 200 ? (MS == 2 ? 4 : 5) : 6) : (GB > 200 ? 2 : 3);
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_RAW = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_RAW + RAW_SLOTS * RAW_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * RAW_SLOTS + 5;
  static constexpr int SIG_BYTES = 16 * (kNumDqWarps / 2);  // peer dequant signals per quantized step
  static constexpr int OFF_SIG = (OFF_BAR + NUM_BARS * 8 + 16 + 127) / 128 * 128;  // signal landing area
  static constexpr int SMEM_BYTES = OFF_SIG + 16 * kNumDqWarps + 1024;
  static constexpr int ACC_COLS = MS * BN;       // TMEM columns of one tile's accumulators
  static constexpr int NBUF = MS == 1 ? 2 : 1;   // accumulator buffers
  static constexpr int TMEM_COLS = 512;
  static_assert(NBUF * ACC_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(RAW_BYTES % 128 == 0, "raw slot alignment");
};

// Dense pair tiles: t -> (BM-row block, 256-column block, K part).
template <int BM>
__device__ __forceinline__ bool gemm2_tile(const GemmParams& p, int t, TileInfo& ti) {
  const int kb_main = p.Kd / kBK;
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

// ---------------- adapter row products inside the GEMM's launch ----------------
// The pair tiles of a dense GEMM often leave SM pairs idle (64 tiles of 512 x 256 on 74 pairs).
// In a fused launch the first rx clusters take those SMs and compute, for the GEMM's own A operand
// Y (X in the forward, dY in the input gradient), out = oscale Y Z^T and la = split(lscale Y Z^T)
// by 128-row blocks, plus LB and hs, while the tiles' main loops run; the tiles' LoRA k-blocks
// come last and wait for the counters. Every CTA first writes its share of LB and hs, then streams
// its blocks through a TMA ring, kc 64-wide k chunks per stage in one copy of each operand.
// tmY views Y as [rows][k chunk][64] with a 128 x kc x 64 box, 128-byte swizzled, so a stage holds
// 128-byte lines (row y, chunk z) at line y kc + z; tmZ views the adapter Z stored [j][k] the same
// way (RN x kc x 64), or, stored [k][j], as 64 kc k-rows of RN unswizzled. Warps 0..7 own 16 rows
// each (ldmatrix, mma.sync, fp32 accumulation over the whole k range in order), warp 8 lane 0
// produces.
template <int NT, int MS>
__device__ __noinline__ void gemm2_rows_role(const CUtensorMap* tmY, const CUtensorMap* tmZ, const GemmParams& p, uint32_t base) {
  const RowsFuse& f = p.rf;
  constexpr int RN = 8 * NT;
  constexpr int XB = 128 * 128;  // one chunk of Y: 128 rows x 64 k
  constexpr int ZB = RN * 128;   // one chunk of Z: RN x 64
  const int S = f.stages, KC = f.kc;
  const int SB = KC * (XB + ZB);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, ncta = 2 * p.rx;
  pdl_wait();  // Y and the adapters may be the previous launch's output
  pdl_launch_dependents();
  if (cta == 0 && f.zc != nullptr)
    for (int i = tid; i < f.zn; i += blockDim.x) f.zc[i] = 0;
  lora_bop_share(BopArgs{f.lbz, f.lbzn, f.lbzj, f.lb_rows}, f.r, f.RP, f.lb, cta, ncta);
  if (f.hs != nullptr)
    for (long i = (long)cta * blockDim.x + tid; i < (long)p.M * f.RP; i += (long)ncta * blockDim.x) {
      const long m = i / f.RP;
      const int j = (int)(i % f.RP);
      const float x = j < f.r ? f.hscale * f.hin[m * f.r + j] : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      f.hs[m * 2 * f.RP + j] = hi;
      f.hs[m * 2 * f.RP + f.RP + j] = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
  fence_proxy_async_global();
  const uint32_t bar0 = base + (uint32_t)(S * SB);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 8);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) tagged_add(f.ctr, f.seq);  // this CTA's LB and hs share is out

  const int nblk = (p.M + 127) / 128;
  const int ksteps = (p.Kd / kBK + KC - 1) / KC;  // stages per block (chunks past the end read as zero)
  if (warp == 8) {
    if (lane == 0) {
      prefetch_tmap(tmY);
      prefetch_tmap(tmZ);
      int it = 0;
      bool ok = true;
      for (int b = cta; ok && b < nblk; b += ncta)
        for (int kt = 0; kt < ksteps; ++kt, ++it) {
          const int s = it % S;
          if (!mbar_wait(empty_bar(s), ((it / S) & 1) ^ 1, 61)) {
            ok = false;
            break;
          }
          const uint32_t st = base + (uint32_t)(s * SB);
          mbar_arrive_expect_tx(full_bar(s), (uint32_t)SB);
          tma_load_3d(st, tmY, full_bar(s), 0, kt * KC, b * 128);
          if (f.ztr) tma_load_2d(st + KC * XB, tmZ, full_bar(s), 0, kt * KC * kBK);
          else tma_load_3d(st + KC * XB, tmZ, full_bar(s), 0, kt * KC, 0);
        }
      if (!ok && it > 0) spin_ns(2000000ull);  // copies in flight land before the CTA exits
    }
  } else if (warp < 8) {
    const int a_row = 16 * warp + (lane & 15), a_col = 8 * (lane >> 4);
    const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
    const int t_k = (lane & 7) + 8 * ((lane >> 3) & 1), t_j = 8 * (lane >> 4);
    const int g = lane >> 2, c = lane & 3;
    // after a failed wait a warp skips the work but keeps taking the same named-barrier steps
    int it = 0;
    bool ok = true;
    for (int b = cta; b < nblk; b += ncta) {
      float acc[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
      for (int kt = 0; ok && kt < ksteps; ++kt, ++it) {
        const int s = it % S;
        if (!warp_wait(full_bar(s), (it / S) & 1, 62)) {
          ok = false;
          break;
        }
        const uint32_t xs = base + (uint32_t)(s * SB), zs = xs + (uint32_t)(KC * XB);
        for (int z = 0; z < KC; ++z) {
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(sw128_addr(xs, a_row * KC + z, 16 * k16 + a_col), a0, a1, a2, a3);
#pragma unroll
            for (int tp = 0; tp < NT / 2; ++tp) {
              uint32_t b0, b1, b2, b3;
              if (f.ztr)
                ldsm_x4_t(zs + (uint32_t)(((z * kBK + 16 * k16 + t_k) * RN + 16 * tp + t_j) * 2), b0, b1, b2, b3);
              else
                ldsm_x4(sw128_addr(zs, (16 * tp + b_row) * KC + z, 16 * k16 + b_col), b0, b1, b2, b3);
              mma_16816(acc[2 * tp], a0, a1, a2, a3, b0, b1);
              mma_16816(acc[2 * tp + 1], a0, a1, a2, a3, b2, b3);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
      }
      // rows 16 warp + g and + 8 of the block: out, and la = [hi | lo] zero past r
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = b * 128 + 16 * warp + g + 8 * h;
        if (!ok || m >= p.M) continue;
        __nv_bfloat16* lam = f.la + (long)m * 2 * f.RP;
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 8 * t + 2 * c + e;
            if (j >= f.RP) continue;
            const float v = acc[t][2 * h + e];
            if (f.out != nullptr && j < f.r) f.out[(long)m * f.r + j] = f.oscale * v;
            const float x = j < f.r ? f.lscale * v : 0.f;
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            lam[j] = hi;
            lam[f.RP + j] = __float2bfloat16_rn(x - __bfloat162float(hi));
          }
        for (int j = RN + c; j < f.RP; j += 4) {
          lam[j] = __float2bfloat16(0.f);
          lam[f.RP + j] = __float2bfloat16(0.f);
        }
      }
      fence_proxy_async_global();
      asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight row warps
      if (tid == 0 && !dev_aborted()) tagged_add(f.ctr + 2 + b / (2 * MS), f.seq);
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (tid == 0 && !dev_aborted()) tagged_add(f.ctr + 1, f.seq);
  }
}

template <int QT, bool TRANS, int MS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemm2Threads, 1)
    qgemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                  const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmLB,
                  const __grid_constant__ CUtensorMap tmRY, const __grid_constant__ CUtensorMap tmZ,
                  const __grid_constant__ GemmParams p) {
  using C = Gemm2Cfg<QT, TRANS, MS>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw_[];
  const uint32_t base_u32 = (smem_u32(smem_raw_) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw_ + (base_u32 - smem_u32(smem_raw_));

  if ((int)(blockIdx.x >> 1) < p.rx) {  // a cluster of the fused adapter row products
    if (p.rf.nt == 2) gemm2_rows_role<2, MS>(&tmRY, &tmZ, p, base_u32);
    else if (p.rf.nt == 4) gemm2_rows_role<4, MS>(&tmRY, &tmZ, p, base_u32);
    else gemm2_rows_role<8, MS>(&tmRY, &tmZ, p, base_u32);
    return;
  }
  if (p.rx > 0) {
    // fused: A and W may be the previous launch's output too
    pdl_wait();
    pdl_launch_dependents();
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank_in_cluster();  // 0 = leader
  const bool leader = rank == 0;
  const int cid = (int)(blockIdx.x >> 1) - p.rx;  // tile clusters follow the row clusters
  const int ncl = (int)(gridDim.x >> 1) - p.rx;

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
      mbar_init(full_bar(s), 1 + kNumDqWarps / 2);  // leader TMA (+ peer signal bytes) + leader dequant group
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < C::RAW_SLOTS; ++s) {
      mbar_init(rfull_bar(s), 1);
      mbar_init(rempty_bar(s), TRANS ? kNumDqWarps / 2 : kNumDqWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kNumEpiWarps);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == kWarpTmaA && lane == 0) {
    prefetch_tmap(&tmA);
    if (p.n_lora_kb) { prefetch_tmap(&tmLA); prefetch_tmap(&tmLB); }
  }
  if (warp == kWarpTmaW && lane == 0) prefetch_tmap(&tmW);
  tc_fence_before();
  __syncthreads();
  cluster_arrive_wait();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  // Unfused, A and W come from before the previous kernel in the stream (the row kernel, which
  // waited for its own predecessor before it let this launch start), so the main loop streams them
  // at once; only the LoRA operands are that kernel's output: the A producer waits for it before
  // their first copy, and epilogue warp 0 waits for it before it lets the next launch start (which
  // may rely on what this launch waited for) and so that this launch completes only after it.
  // Fused, everything waited above, and the A producer waits for the row clusters' counters
  // (LB and hs shares, then the 128-row blocks of the tile's M block) before the LoRA copies.

  const int kb_main = p.Kd / kBK;
  auto tile_steps = [&](const TileInfo& ti) { return (ti.kb_hi - ti.kb_lo) + (ti.lora ? p.n_lora_kb : 0); };
  auto step_kb = [&](const TileInfo& ti, int i) {
    const int nq = ti.kb_hi - ti.kb_lo;
    return i < nq ? ti.kb_lo + i : kb_main + (i - nq);
  };
  // the leader's copies of the full / tempty barriers, as cluster addresses
  auto full_leader = [&](int s) { return map_to_rank(full_bar(s), 0); };
  auto tempty_leader = [&](int b) { return map_to_rank(tempty_bar(b), 0); };

  if (warp == kWarpTmaA) {
    // ---------------- A rows (and LoRA operands) of this CTA ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      bool issued = false;
      bool waited = false;
      int mb_ready = -1;
      TileInfo ti;
      for (int t = cid; ok && gemm2_tile<C::BM>(p, t, ti); t += ncl) {
        const int nsteps = tile_steps(ti);
        const int arow = ti.row0 + 128 * (int)rank;
        const int mb = ti.row0 / C::BM;
        for (int i = 0; i < nsteps; ++i, ++it) {
          const int kb = step_kb(ti, i);
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, 11)) { ok = false; break; }
          const uint32_t fb = full_leader(s);
          if (kb < kb_main) {
            if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * C::A_BYTES + C::SIG_BYTES);
#pragma unroll
            for (int h = 0; h < MS; ++h)
              tma_load_2d_pair(sA + s * C::A_BYTES + h * 16384, &tmA, fb, kb * kBK, arow + 256 * h);
          } else {
            if (!waited) {
              if (p.rx == 0) pdl_wait();  // the LoRA operands are the previous kernel's output
              else if (!wait_tagged(p.rf.ctr, p.rf.seq, 2 * p.rx, 63)) { ok = false; break; }
              waited = true;
            }
            if (p.rx > 0 && mb != mb_ready) {
              const int blocks = min(2 * MS, (p.M + 127) / 128 - 2 * MS * mb);
              if (!wait_tagged(p.rf.ctr + 2 + mb, p.rf.seq, blocks, 64)) { ok = false; break; }
              fence_proxy_async_global();
              mb_ready = mb;
            }
            const int x = (kb - kb_main) * kBK;
            if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * (C::A_BYTES + C::B_BYTES));
#pragma unroll
            for (int h = 0; h < MS; ++h)
              tma_load_2d_pair(sA + s * C::A_BYTES + h * 16384, &tmLA, fb, x, arow + 256 * h);
            const int lb = ti.nb * BN + C::HN * (int)rank;
            tma_load_2d_pair(sB + s * C::B_BYTES, &tmLB, fb, x, lb);
            tma_load_2d_pair(sB + s * C::B_BYTES + 64 * 128, &tmLB, fb, x, lb + 64);
          }
          issued = true;
        }
      }
      // copies still in flight complete on the leader's barrier, which this CTA cannot wait on
      // once the pipeline has given up: give them time to land before the CTA may exit
      if (!ok && issued) spin_ns(2000000ull);
    }
  } else if (warp == kWarpTmaW) {
    // ---------------- packed groups of this CTA's half ----------------
    if (lane == 0) {
      int rc = 0;
      bool ok = true;
      int last_phase[8];
      for (int s = 0; s < C::RAW_SLOTS; ++s) last_phase[s] = -1;
      constexpr int GW = C::GB / 4;
      TileInfo ti;
      for (int t = cid; ok && gemm2_tile<C::BM>(p, t, ti); t += ncl) {
        const int c_lo = TRANS ? ti.kb_lo : ti.kb_lo / 4;
        const int c_hi = TRANS ? ti.kb_hi : ti.kb_hi / 4;
        for (int c = c_lo; c < c_hi; ++c, ++rc) {
          const int s = rc % C::RAW_SLOTS;
          const uint32_t ph = (rc / C::RAW_SLOTS) & 1;
          if (!mbar_wait(rempty_bar(s), ph ^ 1, 12)) { ok = false; break; }
          mbar_arrive_expect_tx(rfull_bar(s), C::RAW_BYTES);
          const uint32_t dst = sRaw + s * C::RAW_BYTES;
          if (TRANS) {
            tma_load_2d(dst, &tmW, rfull_bar(s), ti.nb * GW, c * 64);
          } else {
            const int y0 = ti.nb * BN + C::HN * (int)rank;
            tma_load_2d(dst, &tmW, rfull_bar(s), c * GW, y0);
            tma_load_2d(dst + 64 * C::GB, &tmW, rfull_bar(s), c * GW, y0 + 64);
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
    // ---------------- pair MMA issuer (leader) ----------------
    if (lane == 0 && leader) {
      int s = 0, tc = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool issued = false;
      TileInfo ti;
      constexpr uint32_t idesc_main = idesc_bf16(256, BN, TRANS);
      constexpr uint32_t idesc_kmaj = idesc_bf16(256, BN, false);
      // descriptors of stage 0; stage s adds s * bytes / 16 to the start-address field
      const uint64_t adesc0 = smem_desc_sw128(sA, 16, 1024);
      const uint64_t bdesc0_k = smem_desc_sw128(sB, 16, 1024);
      const uint64_t bdesc0_mn = smem_desc_sw128(sB, 1024, 2048);
      for (int t = cid; ok && gemm2_tile<C::BM>(p, t, ti); t += ncl, ++tc) {
        const int buf = tc % C::NBUF;
        if (!mbar_wait<true>(tempty_bar(buf), ((tc / C::NBUF) & 1) ^ 1, 13)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * C::ACC_COLS;
        const int nq = ti.kb_hi - ti.kb_lo;
        const int nsteps = tile_steps(ti);
        for (int i = 0; i < nsteps; ++i) {
          if (!mbar_wait(full_bar(s), ph, 14)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)(s * (C::A_BYTES >> 4));
          const bool kmaj = !TRANS || i >= nq;
          // the MS A blocks of a stage are 16 KB (1024 descriptor units) apart and share the B half
          if (kmaj) {
            const uint64_t bd = bdesc0_k + (uint64_t)(s * (C::B_BYTES >> 4));
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
#pragma unroll
              for (int h = 0; h < MS; ++h)
                umma_bf16_pair(d_tmem + h * BN, ad + 1024 * h + 2 * k, bd + 2 * k, idesc_kmaj, (i | k) != 0);
          } else {
            const uint64_t bd = bdesc0_mn + (uint64_t)(s * (C::B_BYTES >> 4));
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
#pragma unroll
              for (int h = 0; h < MS; ++h)
                umma_bf16_pair(d_tmem + h * BN, ad + 1024 * h + 2 * k, bd + 256 * k, idesc_main, (i | k) != 0);
          }
          umma_commit_pair_both(empty_bar(s));
          issued = true;
          if (++s == C::STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair_both(tfull_bar(buf));
      }
      if (issued) {
        umma_commit_pair(map_to_rank(drain_bar, 0));
        mbar_wait(drain_bar, 0, 0, false, 2000000ull);
      }
    }
  } else if (gemm2_dq_warp(warp) >= 0) {
    // ---------------- dequant workers: this CTA's half of B ----------------
    const int dq = gemm2_dq_warp(warp) * 32 + lane;
    const int grp = dq >> 8;
    const int gt = dq & 255;
    // this warp's 16-byte slot of the signal area (the same offset in both CTAs)
    const uint32_t sig = base_u32 + C::OFF_SIG + 16u * (uint32_t)(dq >> 5);
    auto signal_full = [&](int s) {
      if (leader) mbar_arrive(full_bar(s));
      else bulk_signal_peer(map_to_rank(sig, 0), sig, 16, full_leader(s));
    };
    int it = 0, rc = 0;
    bool ok = true;
    TileInfo ti;
    for (int t = cid; ok && gemm2_tile<C::BM>(p, t, ti); t += ncl) {
      if (!TRANS) {
        for (int g = ti.kb_lo / 4; ok && g < ti.kb_hi / 4; ++g, ++rc) {
          const int rs = rc % C::RAW_SLOTS;
          if (!warp_wait(rfull_bar(rs), (rc / C::RAW_SLOTS) & 1, 15)) { ok = false; break; }
          const uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_BYTES;
          for (int sub = 0; sub < 4; ++sub, ++it) {
            if ((it & 1) != grp) continue;
            const int s = it % C::STAGES;
            if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 16)) { ok = false; break; }
            uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
            {
              const int row = gt >> 1, uh = gt & 1;
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
            if (lane == 0) signal_full(s);
          }
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(rempty_bar(rs));
        }
      } else {
        for (int kb = ti.kb_lo; ok && kb < ti.kb_hi; ++kb, ++rc, ++it) {
          if ((it & 1) != grp) continue;
          const int rs = rc % C::RAW_SLOTS;
          if (!warp_wait(rfull_bar(rs), (rc / C::RAW_SLOTS) & 1, 15)) { ok = false; break; }
          const int s = it % C::STAGES;
          if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 16)) { ok = false; break; }
          const uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_BYTES;
          uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
          {
            // this CTA's 128 output columns are half `rank` of the 256-column group
            const int kk = gt >> 2, ul = gt & 3;
            uint4 v[4];
            decode_unit_bf16<QT>(raw + kk * C::GB, 4 * (int)rank + ul, v);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int gc = 4 * ul + cc;
              const int off = (kk >> 3) * 2048 + (gc >> 3) * 1024 + (kk & 7) * 128 + (((gc & 7) ^ (kk & 7)) << 4);
              *reinterpret_cast<uint4*>(sb + off) = v[cc];
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            signal_full(s);
            mbar_arrive(rempty_bar(rs));
          }
        }
      }
      for (int i = 0; ok && ti.lora && i < p.n_lora_kb; ++i, ++it) {
        if ((it & 1) != grp) continue;
        const int s = it % C::STAGES;
        if (!warp_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 17)) { ok = false; break; }
        __syncwarp();
        if (lane == 0 && leader) mbar_arrive(full_bar(s));  // the peer has nothing to signal here
      }
    }
  } else if (warp < kNumEpiWarps) {
    // ---------------- epilogue: this CTA's MS x 128 rows x 256 columns ----------------
    if (warp == 0) {
      pdl_wait();
      pdl_launch_dependents();
    }
    int tc = 0;
    TileInfo ti;
    for (int t = cid; gemm2_tile<C::BM>(p, t, ti); t += ncl, ++tc) {
      const int buf = tc % C::NBUF;
      if (!warp_wait(tfull_bar(buf), (tc / C::NBUF) & 1, 18)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < MS; ++h) {
        const int row = ti.row0 + 256 * h + 128 * (int)rank + warp * 32 + lane;
        const bool valid = row < ti.row_end;
        const uint32_t tbase = tmem_base + ((uint32_t)(warp * 32) << 16) + buf * C::ACC_COLS + h * BN;
        epilogue_rows_store<BN>(p, ti, row, valid, tbase);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader(buf));
    }
  }

  tc_fence_before();
  // after a wait gave up, copies issued before it (TMA loads, peer signals) may still be in flight
  // towards either CTA's shared memory: let them land before the pair can exit
  if (threadIdx.x == 0 && dev_aborted()) spin_ns(2000000ull);
  __syncthreads();
  cluster_arrive_wait();  // no CTA leaves while the pair MMAs or the peer may still touch it
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
