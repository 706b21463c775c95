// Adapter-side kernels of the layer (bandwidth-bound; warp-level bf16 MMA, fp32 accumulation):
//
//   rows     out[m, j] = oscale * sum_k Y[m, k] Z(j, k)        H = X A^T,  G = s dY B
//            and the tensor-core operand LA[m] = [hi(v) | lo(v)], v = lscale * sum
//   bop      LB[n] = [Z(n, :) | Z(n, :)]                        B (forward) or A^T (dX)
//   colred   out[c, j] = sum_m Y[m, c] Z[m, j] over row slices, then an ordered sum over the
//            slices: dB = dY^T split(s H), dA = split(G)^T X (deterministic: no float atomics)
//
// Dense layer: lora_rows_cluster_kernel streams its bf16 operand through a TMA ring and sums its k
// slices in-cluster; colred_flow_kernel streams through a TMA ring, takes units of work from
// a counter and sums a block's row slices in slice order. Routed (grouped) layer:
// lora_rows_seg_kernel, colred_mma_kernel + colred_reduce_kernel, lora_bop_vec_kernel.
//
// The fast LoRA backward these implement is the plain chain rule of the layer (Show HN: LoRA over
// GGUF, "Things involved in the training", which names an Unsloth-style fast LoRA backward for the
// linear and the MoE layer). Adapter gradients stay in fp32 end to end.
#pragma once
#include <cuda_bf16.h>

#include "decode.cuh"
#include "ptx.cuh"

namespace qlora {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 q, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// ------------------------------------------------------------------------------------------------
// Tensor-core (mma.sync m16n8k16, bf16 in, fp32 accumulate) versions of the two adapter reductions.
// These are small, bandwidth-bound contractions with r <= 64 output columns; the warp-level MMA
// keeps them at memory speed without a CUDA-core FMA bottleneck.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }

__device__ __forceinline__ uint32_t pack2_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// ---- streamed tiles: 16-byte cp.async copies into a shared-memory ring ----------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  // src-size 0 fills the 16 bytes with zeros and reads nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Column reductions on tensor cores: part[slice][c][j] = sum_{m in slice} Y[m][c] * Zs[m][j], where
// Zs = Z * zw (optional per-row weight) is fed as a bf16 hi + lo pair (fp32-accurate).
// A operand: Zs^T (rows j, k = m); B operand: Y (k = m, n = c) through ldmatrix.trans.
// Grid (ceil(C/128), slices), 128 threads: warp w owns columns 128*bx + 32w .. +31. A slice is one
// 128-row block of an expert segment (E > 0) or of the rows (E == 0). Its whole 128 x 128 tile of Y
// (and of Ylo) goes to shared memory in one round of 16-byte asynchronous copies (rows past the
// segment zero-filled), while the threads stage Zs^T, so a CTA waits for memory once.
// JT = ceil(r/16) tiles of 16 rows of j.
constexpr int kCrYS = 128 + 8;  // padded row (bf16): 272 bytes, ldmatrix rows hit distinct banks
__host__ __device__ constexpr int colred_mma_smem(int JT, bool two) {
  return (two ? 2 : 1) * 128 * kCrYS * 2 + 2 * JT * 16 * kCrYS * 2;
}
template <int JT>
__global__ void __launch_bounds__(128) colred_mma_kernel(const __nv_bfloat16* __restrict__ Y, long ldy, int Ccols,
                                                         const float* __restrict__ Z, int r, int M,
                                                         const float* __restrict__ zw, const int* __restrict__ seg_off,
                                                         const int* __restrict__ mblk_off, int E,
                                                         float* __restrict__ part,
                                                         const __nv_bfloat16* __restrict__ Ylo,
                                                         const int32_t* __restrict__ rowmap, int rk) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  // Ylo (nullable): a second bf16 term of Y (Y = Y + Ylo to ~2^-16), same layout.
  // rowmap (nullable): row m of the slice is row rowmap[m] / rk of Y (a pair's token row read in
  // place, instead of from a gathered copy).
  constexpr int YS = kCrYS;
  extern __shared__ __align__(16) uint8_t crm_smem[];
  __nv_bfloat16* zh = reinterpret_cast<__nv_bfloat16*>(crm_smem);  // [JT*16][YS]: Zs^T hi
  __nv_bfloat16* zl = zh + JT * 16 * YS;                           // lo
  __nv_bfloat16* ys = zl + JT * 16 * YS;                           // [128][YS]
  __nv_bfloat16* ysl = ys + 128 * YS;                              // [128][YS] (two terms only)
  const int slice = blockIdx.y;
  int lo, hi;
  if (E == 0) {
    lo = slice * 128;
    hi = min(M, lo + 128);
  } else {
    const int total = __ldg(mblk_off + E);
    if (slice >= total) return;
    int a = 0, b = E - 1;
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (__ldg(mblk_off + mid) <= slice) a = mid; else b = mid - 1;
    }
    lo = __ldg(seg_off + a) + (slice - __ldg(mblk_off + a)) * 128;
    hi = min(__ldg(seg_off + a + 1), lo + 128);
  }
  const int n = max(0, hi - lo);
  const int c0 = blockIdx.x * 128;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const bool two = Ylo != nullptr;
  const int kmax = (n + 15) & ~15;  // rows past n are zero in both operands
  for (int i = tid; i < (kmax << 4); i += 128) {
    const int m = i >> 4, q = i & 15;
    const bool in = m < n && c0 + 8 * q < Ccols;
    const long yrow = rowmap != nullptr ? (long)(in ? __ldg(rowmap + lo + m) / rk : 0) : (long)(lo + m);
    const long o = in ? yrow * ldy + c0 + 8 * q : 0;
    cp_async16(smem_u32(ys + m * YS + 8 * q), Y + o, in);
    if (two) cp_async16(smem_u32(ysl + m * YS + 8 * q), Ylo + o, in);
  }
  cp_async_commit();
  // stage Zs^T as hi / lo bf16 while the copies are in flight
  for (int i = tid; i < JT * 16 * kmax; i += 128) {
    const int j = i / kmax, m = i - j * kmax;
    float z = 0.f;
    if (m < n && j < r) {
      z = __ldg(Z + (long)(lo + m) * r + j);
      if (zw != nullptr) z *= __ldg(zw + lo + m);
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(z);
    zh[j * YS + m] = h;
    zl[j * YS + m] = __float2bfloat16_rn(z - __bfloat162float(h));
  }
  cp_async_wait<0>();
  __syncthreads();
  float acc[JT][4][4];
#pragma unroll
  for (int jt = 0; jt < JT; ++jt)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[jt][t][0] = acc[jt][t][1] = acc[jt][t][2] = acc[jt][t][3] = 0.f;
  const int wc = warp * 32;  // warp's first column within the CTA tile
  for (int k = 0; k < kmax; k += 16) {
#pragma unroll
    for (int term = 0; term < 2; ++term) {
      if (term == 1 && !two) break;
      const __nv_bfloat16* src = term ? ysl : ys;
      // B fragments for 4 n8 tiles: two ldmatrix.x4.trans, each covering 2 tiles x k16
      uint32_t b[4][2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int mat = lane >> 3, rr = lane & 7;
        const int krow = k + ((mat & 1) ? 8 : 0) + rr;
        const int ncol = wc + 16 * h2 + ((mat & 2) ? 8 : 0);
        ldsm_x4_t(smem_u32(src + krow * YS + ncol), b[2 * h2][0], b[2 * h2][1], b[2 * h2 + 1][0], b[2 * h2 + 1][1]);
      }
#pragma unroll
      for (int jt = 0; jt < JT; ++jt) {
        const int j0 = 16 * jt;
        const uint32_t ah0 = *reinterpret_cast<const uint32_t*>(zh + (j0 + g) * YS + k + 2 * c);
        const uint32_t ah1 = *reinterpret_cast<const uint32_t*>(zh + (j0 + g + 8) * YS + k + 2 * c);
        const uint32_t ah2 = *reinterpret_cast<const uint32_t*>(zh + (j0 + g) * YS + k + 2 * c + 8);
        const uint32_t ah3 = *reinterpret_cast<const uint32_t*>(zh + (j0 + g + 8) * YS + k + 2 * c + 8);
#pragma unroll
        for (int t = 0; t < 4; ++t) mma_16816(acc[jt][t], ah0, ah1, ah2, ah3, b[t][0], b[t][1]);
        if (term == 0) {  // Z_lo * Y (Z_lo * Y_lo is below fp32 resolution)
          const uint32_t al0 = *reinterpret_cast<const uint32_t*>(zl + (j0 + g) * YS + k + 2 * c);
          const uint32_t al1 = *reinterpret_cast<const uint32_t*>(zl + (j0 + g + 8) * YS + k + 2 * c);
          const uint32_t al2 = *reinterpret_cast<const uint32_t*>(zl + (j0 + g) * YS + k + 2 * c + 8);
          const uint32_t al3 = *reinterpret_cast<const uint32_t*>(zl + (j0 + g + 8) * YS + k + 2 * c + 8);
#pragma unroll
          for (int t = 0; t < 4; ++t) mma_16816(acc[jt][t], al0, al1, al2, al3, b[t][0], b[t][1]);
        }
      }
    }
  }
  // acc[jt][t]: rows j = 16jt + g (+8), columns c0 + wc + 8t + 2c (+1)
#pragma unroll
  for (int jt = 0; jt < JT; ++jt)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int col = c0 + wc + 8 * t + 2 * c;
      const int j0 = 16 * jt + g, j1 = j0 + 8;
      float* o = part + (long)slice * Ccols * r;
      if (col < Ccols) {
        if (j0 < r) { o[(long)col * r + j0] = acc[jt][t][0]; o[(long)(col + 1) * r + j0] = acc[jt][t][1]; }
        if (j1 < r) { o[(long)col * r + j1] = acc[jt][t][2]; o[(long)(col + 1) * r + j1] = acc[jt][t][3]; }
      }
    }
}

// ------------------------------------------------------------------------------------------------
// Cluster versions (dense layer): the split-K / split-M partials are summed through distributed
// shared memory inside one kernel, in a fixed rank order (deterministic), so no reduction launch
// and no partial buffer in HBM are needed.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t a = smem_u32(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

// sum over cluster ranks 0 .. n-1 (n <= 8) of the value at this shared address, added in rank
// order; the remote loads are all issued before the first add
__device__ __forceinline__ float cluster_sum_ordered(const float* local, int n) {
  float x[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) x[q] = q < n ? ld_dsmem_f32(local, (uint32_t)q) : 0.f;
  float v = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (q < n) v += x[q];
  return v;
}

struct BopArgs {            // LB[n] = [Z(n, :) | Z(n, :)], zero padded (nullptr Z = none)
  const __nv_bfloat16* Z;
  long zn, zjs;
  int rows;
};

// Share cta of ncta CTAs of LB, 8 columns per item.
__device__ __forceinline__ void lora_bop_share(const BopArgs& bop, int r, int RP, __nv_bfloat16* __restrict__ LB,
                                               long cta, long ncta) {
  if (bop.Z == nullptr) return;
  const long items = (long)bop.rows * (2 * RP / 8);
  for (long i = cta * blockDim.x + threadIdx.x; i < items; i += ncta * blockDim.x) {
    const int n = (int)(i / (2 * RP / 8));
    const int j0 = (int)(i % (2 * RP / 8)) * 8;
    __nv_bfloat16 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = (j0 + e) % RP;
      v[e] = j < r ? bop.Z[(long)n * bop.zn + (long)j * bop.zjs] : __float2bfloat16(0.f);
    }
    *reinterpret_cast<uint4*>(LB + (long)n * 2 * RP + j0) = *reinterpret_cast<const uint4*>(v);
  }
}


// Element (row, col) of a 128-byte-swizzled box of 64 bf16 columns: 16-byte chunk col/8 of row
// `row` sits at chunk position (col/8) ^ (row % 8).
__device__ __forceinline__ uint32_t sw128_addr(uint32_t box, int row, int col) {
  return box + (uint32_t)(row * 128) + ((uint32_t)(((col >> 3) ^ (row & 7))) << 4) + (uint32_t)((col & 7) * 2);
}

constexpr int kRowsStages = 4;    // TMA ring depth of the dense row products
constexpr int kRowsTileK = 128;   // k per streamed tile: 64 rows x 128 bf16, two 128-byte-swizzled boxes
constexpr int kRowsStageBytes = 64 * kRowsTileK * 2;

// Dynamic shared memory of lora_rows_cluster_kernel<NT> for a k range of kchunk: the ring, the Z
// slice ([RN][kchunk + 8], k contiguous, or ztr: [kchunk][RN + 8], j contiguous), the partials, the
// ring's barriers and the alignment slack.
__host__ __device__ constexpr size_t rows_zs_halves(int NT, int kchunk, bool ztr) {
  return ztr ? (size_t)kchunk * (8 * NT + 8) : (size_t)8 * NT * (kchunk + 8);
}
__host__ __device__ constexpr size_t rows_smem_bytes(int NT, int kchunk, bool ztr) {
  return (size_t)kRowsStages * kRowsStageBytes + rows_zs_halves(NT, kchunk, ztr) * 2 + (size_t)64 * 8 * NT * 4 +
         2 * kRowsStages * 8 + 1024;
}

// Rows of out = Y Z^T for 64 rows per cluster column (warp w owns rows 16w .. 16w+15); cluster rank
// q sums k in [q * kchunk, (q + 1) * kchunk). Z(j, k) = Z[j*zj + k*zk] is staged once per CTA as
// it lies in memory: [j][k] when k is contiguous (read by ldmatrix), [k][j] when j is (read by
// ldmatrix.trans, no transpose on the way in). The rows of Y (tensor map tmY, 64 x 64 boxes,
// 128-byte swizzle) stream by TMA through a ring of 64 x 128 tiles (kRowsStages deep, mbarrier
// guarded; thread 0 refills a slot once the four warps have released it) into mma.sync. The ranks' partials are summed through
// distributed shared memory in rank order. Writes out = oscale * sum (fp32 [M x r]) and
// la = split(lscale * sum) ([M x 2RP] bf16). The aux CTAs (blockIdx.x >= row_blocks, whole
// clusters, when the launch has room for them in its one wave) write the LB operand (bop) and,
// when hin is given, hs = split(hscale * hin), beside the row CTAs; without them every CTA takes a
// share of that while its first copies are in flight.
template <int NT>
__global__ void __launch_bounds__(128) lora_rows_cluster_kernel(
    const __grid_constant__ CUtensorMap tmY, int M, int Kin, int kchunk, const __nv_bfloat16* __restrict__ Z,
    long zj, long zk, int r, float oscale, float lscale, float* __restrict__ out, __nv_bfloat16* __restrict__ la,
    int RP, BopArgs bop, __nv_bfloat16* __restrict__ LB, int row_blocks, const float* __restrict__ hin, float hscale,
    __nv_bfloat16* __restrict__ hs, int* __restrict__ zc, int zn) {
  constexpr int RN = 8 * NT;
  constexpr int S = kRowsStages, TK = kRowsTileK, SB = kRowsStageBytes;
  extern __shared__ uint8_t rows_smem_raw[];
  const uint32_t base = (smem_u32(rows_smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = rows_smem_raw + (base - smem_u32(rows_smem_raw));
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < zn; i += blockDim.x) zc[i] = 0;  // counters of a later kernel
  // LB and hs: by the aux CTAs when the launch has them, else by every CTA before its cluster sync
  auto aux_share = [&](long cta, long ncta) {
    lora_bop_share(bop, r, RP, LB, cta, ncta);
    if (hs != nullptr)
      for (long i = cta * blockDim.x + threadIdx.x; i < (long)M * RP; i += ncta * blockDim.x) {
        const long m = i / RP;
        const int j = (int)(i % RP);
        const float x = j < r ? hscale * hin[m * r + j] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        hs[m * 2 * RP + j] = hi;
        hs[m * 2 * RP + RP + j] = __float2bfloat16_rn(x - __bfloat162float(hi));
      }
  };
  const bool aux_ctas = (int)gridDim.x > row_blocks;
  if ((int)blockIdx.x >= row_blocks) {
    aux_share((long)(blockIdx.x - row_blocks) * gridDim.y + blockIdx.y, (long)(gridDim.x - row_blocks) * gridDim.y);
    return;
  }
  const bool ztr = zk != 1;  // Z staged [k][j]
  const int ZS = kchunk + 8, ZT = RN + 8;
  __nv_bfloat16* zs = reinterpret_cast<__nv_bfloat16*>(smem + S * SB);
  float* part = reinterpret_cast<float*>(zs + rows_zs_halves(NT, kchunk, ztr));
  const uint32_t bar0 = smem_u32(part + 64 * RN);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KS = gridDim.y;
  const uint32_t rank = cluster_ctarank();
  const int m0 = blockIdx.x * 64;
  const int kb = (int)rank * kchunk;
  const int ke = min(Kin, kb + kchunk);
  const int nk = max(0, ke - kb);
  const int ntiles = (nk + TK - 1) / TK;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 4);
    }
    fence_mbar_init();
    prefetch_tmap(&tmY);
  }
  __syncthreads();
  auto issue = [&](int t) {  // tile t into slot t % S: k [kb + 128 t, + 128) of rows [m0, m0 + 64)
    const int s = t % S;
    const uint32_t st = base + (uint32_t)(s * SB);
    mbar_arrive_expect_tx(full_bar(s), (uint32_t)SB);
    tma_load_2d(st, &tmY, full_bar(s), kb + t * TK, m0);
    tma_load_2d(st + SB / 2, &tmY, full_bar(s), kb + t * TK + 64, m0);
  };
  // the Z slice by cp.async where rows are whole 16-byte chunks, otherwise element by element; its
  // requests go out ahead of the ring's first tiles, which would otherwise queue them behind the
  // whole grid's tile traffic
  const uint32_t zdst = smem_u32(zs);
  if (!ztr) {
    for (int i = tid; i < RN * (kchunk / 8); i += 128) {
      const int j = i / (kchunk / 8), q = i % (kchunk / 8);
      const bool v = j < r && 8 * q < nk;
      cp_async16(zdst + (uint32_t)(j * ZS + 8 * q) * 2, v ? (const void*)(Z + (long)j * zj + kb + 8 * q) : (const void*)Z,
                 v);
    }
  } else if (zj == 1 && (r & 7) == 0 && (zk & 7) == 0) {
    for (int i = tid; i < kchunk * (RN / 8); i += 128) {
      const int kk = i / (RN / 8), q = i % (RN / 8);
      const bool v = 8 * q < r && kk < nk;
      cp_async16(zdst + (uint32_t)(kk * ZT + 8 * q) * 2, v ? (const void*)(Z + (long)(kb + kk) * zk + 8 * q) : (const void*)Z,
                 v);
    }
  } else {
    for (int i = tid; i < kchunk * RN; i += 128) {
      const int kk = i / RN, j = i % RN;
      zs[kk * ZT + j] = (j < r && kk < nk) ? Z[(long)j * zj + (long)(kb + kk) * zk] : __float2bfloat16(0.f);
    }
  }
  cp_async_commit();
  if (tid == 0)
    for (int t = 0; t < min(ntiles, S); ++t) issue(t);
  // without aux CTAs, this CTA's share of LB and hs while the first copies are in flight
  if (!aux_ctas) aux_share((long)blockIdx.y * gridDim.x + blockIdx.x, (long)gridDim.x * gridDim.y);
  cp_async_wait<0>();
  __syncthreads();  // the Z slice is visible to every warp

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  // ldmatrix lane addresses: A = rows 16w + lane%16, k offset 8*(lane/16) (in the swizzled boxes).
  // B, [j][k]: Z rows (n) lane%8 + 8*(lane/16) of an n-tile pair, k offset 8*((lane/8)%2); B, [k][j]
  // (.trans): k rows lane%8 + 8*((lane/8)%2), j offset 8*(lane/16). Both give (tile 0: k 0-7,
  // k 8-15; tile 1: ..).
  const int a_row = 16 * warp + (lane & 15), a_col = 8 * (lane >> 4);
  const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
  const int t_k = (lane & 7) + 8 * ((lane >> 3) & 1), t_j = 8 * (lane >> 4);
  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % S;
    if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), (uint32_t)((t / S) & 1), 51))) {
      ok = false;
      break;
    }
    const uint32_t st = base + (uint32_t)(s * SB);
    const uint32_t bbase = ztr ? smem_u32(zs + (t * TK + t_k) * ZT + t_j) : smem_u32(zs + b_row * ZS + t * TK + b_col);
#pragma unroll
    for (int k16 = 0; k16 < TK / 16; ++k16) {
      const int kk = 16 * k16 + a_col;  // k within the tile
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sw128_addr(st + (uint32_t)((kk >> 6) * (SB / 2)), a_row, kk & 63), a0, a1, a2, a3);
#pragma unroll
      for (int tp = 0; tp < NT / 2; ++tp) {
        uint32_t b0, b1, b2, b3;
        if (ztr) ldsm_x4_t(bbase + (uint32_t)(16 * k16 * ZT) * 2 + 32 * tp, b0, b1, b2, b3);
        else ldsm_x4(bbase + (uint32_t)(16 * tp * ZS) * 2 + 32 * k16, b0, b1, b2, b3);
        mma_16816(acc[2 * tp], a0, a1, a2, a3, b0, b1);
        mma_16816(acc[2 * tp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
    if (warp == 0 && t + S < ntiles) {
      // thread 0 refills this slot once all four warps have released it
      bool w = true;
      if (lane == 0) {
        w = mbar_wait(empty_bar(s), (uint32_t)((t / S) & 1), 52);
        if (w) issue(t + S);
      }
      if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) { ok = false; break; }
    }
  }
  if (!ok || dev_aborted()) spin_ns(2000000ull);  // copies issued before a wait gave up land first
  {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = 8 * t + 2 * c;
      const int lr = warp * 16 + g;
      part[lr * RN + j] = acc[t][0];
      part[lr * RN + j + 1] = acc[t][1];
      part[(lr + 8) * RN + j] = acc[t][2];
      part[(lr + 8) * RN + j + 1] = acc[t][3];
    }
  }
  cluster_sync_all();
  // rank q reduces rows [q*64/KS, (q+1)*64/KS) of the cluster's 64 rows, over ranks in order
  const int rows_per = (64 + KS - 1) / KS;
  const int lr0 = (int)rank * rows_per;
  for (int i = tid; i < rows_per * RP; i += 128) {
    const int lr = lr0 + i / RP, j = i % RP;
    const int m = m0 + lr;
    if (lr >= 64 || m >= M) continue;
    float v = 0.f;
    if (j < r) v = cluster_sum_ordered(&part[lr * RN + j], KS);
    if (out != nullptr && j < r) out[(long)m * r + j] = oscale * v;
    if (la != nullptr) {
      const float x = lscale * v;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      la[(long)m * 2 * RP + j] = j < r ? hi : __float2bfloat16(0.f);
      la[(long)m * 2 * RP + RP + j] = j < r ? lo : __float2bfloat16(0.f);
    }
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its partials
}

// Dense column reductions (dB and dA of the backward) in one launch, as units of work claimed
// from a counter: out_p = scale_p * sum_m Y_p[m][c] Z_p[m][j] for Y_p [M x C_p] and the split
// operand Z_p [M x 2RP] = [hi | lo] bf16 of an fp32 tensor (the two together carry it to about
// 2^-16 relative), both read through tensor maps (128-byte swizzled 64 x 64 boxes).
struct ColredOut {
  int C;
  float scale;
  int transpose;  // 0: out[c][j]; 1: out[j][c]
  float* out;
};
// The columns of both problems form nblk blocks of 128 (the first nb0 of problem 0); the rows form
// csu chunks of mchunk (a multiple of the tile height tr, every chunk non-empty). A unit is one
// (block, chunk),
// u = block * csu + chunk. With csu > 1 each unit leaves its fp32 partial [16 JT][128] in part, and
// whichever CTA finishes the last chunk of a block sums that block's partials in chunk order, so
// the result does not depend on which CTA took which unit.
struct ColredFlow {
  ColredOut o0, o1;
  int nb0, nblk, M, r, RP, mchunk, csu;
  int tr;          // rows per streamed tile (64, 128 or 256): the height of every TMA box
  int defer_wait;  // 1: the previous kernel in the stream already waited for this launch's inputs
  float* part;     // [nblk * csu][16 JT][128]
  int* ctr;        // [0]: next unit to claim, [1 + b]: chunks of block b finished; zero at launch
  const unsigned long long* gate;  // with defer_wait: a tagged count (gate_seq) of the previous
  unsigned gate_seq;               // launch that reaches gate_target once the split operands and
  int gate_target;                 // the zeroed counters are written (nullable)
};

constexpr int kColTmaStagesMax = 6;
constexpr int kColWarps = 9;  // eight consumer warps and one producer warp
constexpr int kColCombStride = 136;
// Bytes of one ring stage: two tr x 64 Y boxes and 2RP/64 boxes of the split operand, 128-byte rows.
__host__ __device__ constexpr int colred_stage_bytes(int RP, int tr) { return (2 + 2 * RP / 64) * tr * 128; }
__host__ __device__ constexpr int colred_comb_bytes(int JT) { return 16 * JT * kColCombStride * 4; }
// Ring stages: as many as fit beside the combine tile, the tags and barriers (256 bytes) and the
// alignment slack, up to six.
__host__ __device__ constexpr int colred_stages(int RP, int JT, int tr) {
  return (232448 - 1024 - 256 - colred_comb_bytes(JT)) / colred_stage_bytes(RP, tr) < kColTmaStagesMax
             ? (232448 - 1024 - 256 - colred_comb_bytes(JT)) / colred_stage_bytes(RP, tr)
             : kColTmaStagesMax;
}
__host__ __device__ constexpr size_t colred_smem_bytes(int RP, int JT, int tr) {
  return (size_t)colred_stages(RP, JT, tr) * colred_stage_bytes(RP, tr) + colred_comb_bytes(JT) + 256 + 1024;
}


__device__ __forceinline__ void colred_store(const ColredOut& O, int r, int j, int col, float v) {
  if (j < r && col < O.C) O.out[O.transpose ? (long)j * O.C + col : (long)col * r + j] = O.scale * v;
}

// Sum of block d's partials in chunk order (the 256 consumer threads).
template <int JT>
__device__ void colred_reduce_block(const ColredFlow& P, int d, int tid) {
  const bool second = d >= P.nb0;
  const ColredOut& O = second ? P.o1 : P.o0;
  const int c0 = (second ? d - P.nb0 : d) * 128;
  const float* src = P.part + (size_t)d * P.csu * (16 * JT * 128);
  for (int i = tid; i < 16 * JT * 32; i += 256) {
    const int j = i >> 5, c4 = (i & 31) * 4;
    if (j >= P.r) continue;
    float4 a = __ldcg(reinterpret_cast<const float4*>(src + j * 128 + c4));
    for (int q = 1; q < P.csu; ++q) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)q * (16 * JT * 128) + j * 128 + c4));
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    colred_store(O, P.r, j, c0 + c4, a.x);
    colred_store(O, P.r, j, c0 + c4 + 1, a.y);
    colred_store(O, P.r, j, c0 + c4 + 2, a.z);
    colred_store(O, P.r, j, c0 + c4 + 3, a.w);
  }
}

// Persistent column reduction. Warp 8 (one lane) claims units from ctr[0], one ahead, and streams
// their 64-row tiles of Y and Z by TMA into a ring of mbarrier-guarded stages, each stage tagged
// with its unit and whether it opens or closes it. Consumer warp w takes columns 32 (w % 4) ..
// +31 of the block and rows 32 (w / 4) .. +31 of each tile, through ldmatrix.trans and mma.sync
// (A = Z^T, B = Y); at a unit's end the two row halves are added through shared memory and the
// result goes out (csu = 1) or to the unit's partial. With defer_wait the wait for the previous
// kernel moves to the end, so that the launch can run beside it on SMs it leaves idle.
template <int JT>
__global__ void __launch_bounds__(32 * kColWarps) colred_flow_kernel(const __grid_constant__ CUtensorMap tmY0,
                                                                     const __grid_constant__ CUtensorMap tmY1,
                                                                     const __grid_constant__ CUtensorMap tmZ0,
                                                                     const __grid_constant__ CUtensorMap tmZ1,
                                                                     const ColredFlow P) {
  extern __shared__ uint8_t col_smem_raw[];
  const uint32_t base = (smem_u32(col_smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = col_smem_raw + (base - smem_u32(col_smem_raw));
  pdl_launch_dependents();
  const int S = colred_stages(P.RP, JT, P.tr);
  const int SB = colred_stage_bytes(P.RP, P.tr);
  const int YB = P.tr * 128;  // bytes of one box
  const int zboxes = 2 * P.RP / 64;
  float* comb = reinterpret_cast<float*>(smem + (size_t)S * SB);
  volatile int* meta = reinterpret_cast<volatile int*>(smem + (size_t)S * SB + colred_comb_bytes(JT));
  volatile int* pend_smem = meta + 2 * kColTmaStagesMax;
  const uint32_t bar0 = base + (uint32_t)(S * SB + colred_comb_bytes(JT) + 64);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kColTmaStagesMax + s); };
  const uint32_t sync_bar = bar0 + 8u * (2 * kColTmaStagesMax);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = P.nblk * P.csu;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 8);
    }
    mbar_init(sync_bar, 8);
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmY0);
    prefetch_tmap(&tmY1);
    prefetch_tmap(&tmZ0);
    prefetch_tmap(&tmZ1);
  }
  __syncthreads();
  if (!P.defer_wait) pdl_wait();

  bool ok = true;
  if (warp == 8) {
    if (lane == 0 && P.gate != nullptr) {
      ok = wait_tagged(P.gate, P.gate_seq, P.gate_target, 65);
      fence_proxy_async_global();
    }
    if (lane == 0 && ok) {
      int it = 0;
      int u = atomicAdd(P.ctr, 1);
      while (true) {
        const int nxt = u < U ? atomicAdd(P.ctr, 1) : U;  // the next claim travels while this unit streams
        if (u >= U) {
          // no work left: a tile-less stage tagged -1 tells the consumers
          const int s = it % S;
          if (it >= S && !mbar_wait(empty_bar(s), (uint32_t)((it / S - 1) & 1), 33)) {
            ok = false;
            break;
          }
          meta[2 * s] = -1;
          mbar_arrive(full_bar(s));
          break;
        }
        const int b = u / P.csu, q = u - b * P.csu;
        const bool second = b >= P.nb0;
        const CUtensorMap* tmY = second ? &tmY1 : &tmY0;
        const CUtensorMap* tmZ = second ? &tmZ1 : &tmZ0;
        const int c0 = (second ? b - P.nb0 : b) * 128;
        const int lo = q * P.mchunk, hi = min(P.M, lo + P.mchunk);
        const int nt = (hi - lo + P.tr - 1) / P.tr;
        for (int t = 0; t < nt && ok; ++t, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(empty_bar(s), (uint32_t)((it / S - 1) & 1), 33)) {
            ok = false;
            break;
          }
          meta[2 * s] = u;
          meta[2 * s + 1] = (t == 0 ? 1 : 0) | (t == nt - 1 ? 2 : 0);
          const uint32_t st = base + (uint32_t)(s * SB);
          const int mb = lo + P.tr * t;
          mbar_arrive_expect_tx(full_bar(s), (uint32_t)SB);
          tma_load_2d(st, tmY, full_bar(s), c0, mb);
          tma_load_2d(st + YB, tmY, full_bar(s), c0 + 64, mb);
          for (int zb = 0; zb < zboxes; ++zb) tma_load_2d(st + (2 + zb) * YB, tmZ, full_bar(s), 64 * zb, mb);
        }
        if (!ok) break;
        u = nxt;
      }
    }
    // the idle lanes must not run ahead to the final wait: griddepcontrol.wait would hold the
    // whole warp, lane 0 included, until the previous kernel completes
    __syncwarp();
  } else {
    const int cg = warp & 3, kh = warp >> 2;
    float acc[JT][4][4];
    // ldmatrix.trans lane addresses. B (Y, k = m, n = c): matrices (m 0-7 | 8-15) x (c 0-7 | 8-15).
    // A (Z^T, rows j, k = m): matrices (j 0-7, m 0-7), (j 8-15, m 0-7), (j 0-7, m 8-15), (j 8-15, m 8-15).
    const int mat = lane >> 3, rr = lane & 7;
    const int yb_row = ((mat & 1) ? 8 : 0) + rr, yb_col = 32 * (cg & 1) + ((mat & 2) ? 8 : 0);
    const int za_row = rr + ((mat & 2) ? 8 : 0), za_col = (mat & 1) ? 8 : 0;
    const int g = lane >> 2, c = lane & 3;
    uint32_t sync_par = 0;
    auto consumer_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(sync_bar);
      const bool w = __all_sync(0xffffffffu, mbar_wait(sync_bar, sync_par, 34));
      sync_par ^= 1u;
      return w;
    };
    int pend_b = -1, pend_tok = 0;  // thread 0: the last unit's block and its count before this CTA's add
    int it = 0;
    while (true) {
      const int s = it % S;
      if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), (uint32_t)((it / S) & 1), 31))) {
        ok = false;
        break;
      }
      const int u = meta[2 * s], fl = meta[2 * s + 1];
      if (u < 0) break;
      if (fl & 1) {
#pragma unroll
        for (int jt = 0; jt < JT; ++jt)
#pragma unroll
          for (int n = 0; n < 4; ++n) acc[jt][n][0] = acc[jt][n][1] = acc[jt][n][2] = acc[jt][n][3] = 0.f;
      }
      const uint32_t st = base + (uint32_t)(s * SB);
      const uint32_t ybox = st + (uint32_t)YB * (uint32_t)(cg >> 1);
      const uint32_t zbox = st + 2u * (uint32_t)YB;
      const int half = P.tr >> 1;
#pragma unroll 2
      for (int kk = 0; kk < half; kk += 16) {
        const int k = half * kh + kk;
        uint32_t bf[4][2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t x0, x1, x2, x3;
          ldsm_x4_t(sw128_addr(ybox, k + yb_row, yb_col + 16 * h2), x0, x1, x2, x3);
          bf[2 * h2][0] = x0;
          bf[2 * h2][1] = x1;
          bf[2 * h2 + 1][0] = x2;
          bf[2 * h2 + 1][1] = x3;
        }
#pragma unroll
        for (int jt = 0; jt < JT; ++jt) {
          const int ch = za_col + 16 * jt, cl = ch + P.RP;  // hi and lo columns of the split operand
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          ldsm_x4_t(sw128_addr(zbox + (uint32_t)YB * (uint32_t)(ch >> 6), k + za_row, ch & 63), h0, h1, h2, h3);
          ldsm_x4_t(sw128_addr(zbox + (uint32_t)YB * (uint32_t)(cl >> 6), k + za_row, cl & 63), l0, l1, l2, l3);
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            mma_16816(acc[jt][n], h0, h1, h2, h3, bf[n][0], bf[n][1]);
            mma_16816(acc[jt][n], l0, l1, l2, l3, bf[n][0], bf[n][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
      ++it;
      if (!(fl & 2)) continue;

      // end of unit u: add the row halves, then the output or the partial
      const int b = u / P.csu;
      if (kh == 1) {
#pragma unroll
        for (int jt = 0; jt < JT; ++jt)
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            const int col = 32 * cg + 8 * n + 2 * c, j0 = 16 * jt + g;
            *reinterpret_cast<float2*>(comb + j0 * kColCombStride + col) = make_float2(acc[jt][n][0], acc[jt][n][1]);
            *reinterpret_cast<float2*>(comb + (j0 + 8) * kColCombStride + col) =
                make_float2(acc[jt][n][2], acc[jt][n][3]);
          }
      }
      if (!consumer_sync()) {
        ok = false;
        break;
      }
      if (kh == 0) {
        const bool second = b >= P.nb0;
        const ColredOut& O = second ? P.o1 : P.o0;
        const int c0 = (second ? b - P.nb0 : b) * 128;
        float* dst = P.part + (size_t)u * (16 * JT * 128);
#pragma unroll
        for (int jt = 0; jt < JT; ++jt)
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            const int col = 32 * cg + 8 * n + 2 * c, j0 = 16 * jt + g;
            const float2 lo2 = *reinterpret_cast<const float2*>(comb + j0 * kColCombStride + col);
            const float2 hi2 = *reinterpret_cast<const float2*>(comb + (j0 + 8) * kColCombStride + col);
            const float v0 = acc[jt][n][0] + lo2.x, v1 = acc[jt][n][1] + lo2.y;
            const float v2 = acc[jt][n][2] + hi2.x, v3 = acc[jt][n][3] + hi2.y;
            if (P.csu == 1) {
              colred_store(O, P.r, j0, c0 + col, v0);
              colred_store(O, P.r, j0, c0 + col + 1, v1);
              colred_store(O, P.r, j0 + 8, c0 + col, v2);
              colred_store(O, P.r, j0 + 8, c0 + col + 1, v3);
            } else {
              *reinterpret_cast<float2*>(dst + j0 * 128 + col) = make_float2(v0, v1);
              *reinterpret_cast<float2*>(dst + (j0 + 8) * 128 + col) = make_float2(v2, v3);
            }
          }
        if (P.csu > 1) __threadfence();
      }
      if (P.csu > 1 && tid == 0) {
        // the count taken at the previous unit's end has long arrived: was that the block's last chunk?
        const int d = (pend_b >= 0 && pend_tok == P.csu - 1) ? pend_b : -1;
        if (d >= 0) __threadfence();
        *pend_smem = d;
      }
      if (!consumer_sync()) {
        ok = false;
        break;
      }
      if (P.csu > 1) {
        const int d = *pend_smem;
        if (tid == 0) {
          __threadfence();
          pend_b = b;
          pend_tok = atomicAdd(P.ctr + 1 + b, 1);
        }
        if (d >= 0) colred_reduce_block<JT>(P, d, tid);
      }
    }
    if (ok && P.csu > 1) {
      if (tid == 0) {
        const int d = (pend_b >= 0 && pend_tok == P.csu - 1) ? pend_b : -1;
        if (d >= 0) __threadfence();
        *pend_smem = d;
      }
      if (consumer_sync()) {
        const int d = *pend_smem;
        if (d >= 0) colred_reduce_block<JT>(P, d, tid);
      }
    }
  }
  if (!ok || dev_aborted()) spin_ns(2000000ull);  // copies issued before a wait gave up land first
  if (P.defer_wait) pdl_wait();
}

// Grouped (routed) row products: one CTA per 128-row block of an expert segment (the grouped
// GEMM's block list), rows sharing one expert e: out[p] = oscale * Y[p] Z_e^T and
// la[p] = split(lscale * Y[p] Z_e^T), Z_e(j, k) = Z[e*zes + j*zj + k*zk]. CTAs past the block
// count exit. 256 threads: warp w owns rows 16w .. 16w + 15 of the block.
template <int NT>
__global__ void __launch_bounds__(256) lora_rows_seg_kernel(const __nv_bfloat16* __restrict__ Y, long ldy, int Kin,
                                                            const __nv_bfloat16* __restrict__ Z, long zj, long zk,
                                                            long zes, const int* __restrict__ seg_off,
                                                            const int* __restrict__ mblk_off, int E, int r, float oscale,
                                                            float lscale, float* __restrict__ out,
                                                            __nv_bfloat16* __restrict__ la, int RP) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  constexpr int RN = 8 * NT;
  constexpr int SK = 128;
  constexpr int ZS = SK + 8;
  __shared__ __align__(16) __nv_bfloat16 zs[RN * ZS];
  const int total = __ldg(mblk_off + E);
  const int blk = blockIdx.x;
  if (blk >= total) return;
  int a = 0, b = E - 1;
  while (a < b) {
    const int mid = (a + b + 1) >> 1;
    if (__ldg(mblk_off + mid) <= blk) a = mid; else b = mid - 1;
  }
  const int e = a;
  const int row_lo = __ldg(seg_off + e) + (blk - __ldg(mblk_off + e)) * 128;
  const int row_hi = min(__ldg(seg_off + e + 1), row_lo + 128);
  const __nv_bfloat16* Ze = Z + (long)e * zes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r0 = row_lo + warp * 16 + g, r1 = r0 + 8;
  const bool v0 = r0 < row_hi, v1 = r1 < row_hi;
  const __nv_bfloat16* y0 = Y + (long)(v0 ? r0 : row_lo) * ldy;
  const __nv_bfloat16* y1 = Y + (long)(v1 ? r1 : row_lo) * ldy;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  for (int k0 = 0; k0 < Kin; k0 += SK) {
    const int nk = min(SK, Kin - k0);
    uint4 xa[SK / 32], xb[SK / 32];
#pragma unroll
    for (int q = 0; q < SK / 32; ++q) {
      const int k = k0 + 32 * q + 8 * c;
      const bool in = 32 * q < nk;
      xa[q] = (v0 && in) ? __ldg(reinterpret_cast<const uint4*>(y0 + k)) : make_uint4(0, 0, 0, 0);
      xb[q] = (v1 && in) ? __ldg(reinterpret_cast<const uint4*>(y1 + k)) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    if (zk == 1) {
      for (int i = threadIdx.x; i < RN * (SK / 8); i += 256) {
        const int j = i / (SK / 8), q = i % (SK / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < r && 8 * q < nk) v = __ldg(reinterpret_cast<const uint4*>(Ze + (long)j * zj + k0 + 8 * q));
        *reinterpret_cast<uint4*>(zs + j * ZS + 8 * q) = v;
      }
    } else {
      for (int i = threadIdx.x; i < RN * SK; i += 256) {
        const int kk = i / RN, j = i % RN;
        __nv_bfloat16 v = __float2bfloat16(0.f);
        if (j < r && kk < nk) v = Ze[(long)j * zj + (long)(k0 + kk) * zk];
        zs[j * ZS + kk] = v;
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < SK / 32; ++q) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint4 zq = *reinterpret_cast<const uint4*>(zs + (8 * t + g) * ZS + 32 * q + 8 * c);
        mma_16816(acc[t], xa[q].x, xb[q].x, xa[q].y, xb[q].y, zq.x, zq.y);
        mma_16816(acc[t], xa[q].z, xb[q].z, xa[q].w, xb[q].w, zq.z, zq.w);
      }
    }
  }
  // C fragment: rows r0 / r1, columns 8t + 2c (+1)
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int row = hh ? r1 : r0;
      if (!(hh ? v1 : v0)) continue;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int j = 8 * t + 2 * c + q;
        const float v = acc[t][2 * hh + q];
        if (out != nullptr && j < r) out[(long)row * r + j] = oscale * v;
        if (la != nullptr && j < RP) {
          const float x = lscale * v;
          const __nv_bfloat16 hi = __float2bfloat16_rn(x);
          const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
          la[(long)row * 2 * RP + j] = j < r ? hi : __float2bfloat16(0.f);
          la[(long)row * 2 * RP + RP + j] = j < r ? lo : __float2bfloat16(0.f);
        }
      }
    }
  }
  // padding columns of la beyond RN (RP > RN happens for r <= 16: RN = 16, RP = 32)
  if (la != nullptr && RP > RN) {
    for (int i = threadIdx.x; i < 128 * (RP - RN); i += 256) {
      const int lr = i / (RP - RN), j = RN + i % (RP - RN);
      const int row = row_lo + lr;
      if (row < row_hi) {
        la[(long)row * 2 * RP + j] = __float2bfloat16(0.f);
        la[(long)row * 2 * RP + RP + j] = __float2bfloat16(0.f);
      }
    }
  }
}

// Bytes of shared memory of lora_rows_seg_z_kernel: the whole adapter slice [RN][Kin + 8].
__host__ __device__ constexpr size_t rows_seg_z_smem(int NT, int Kin) { return (size_t)8 * NT * (Kin + 8) * 2; }

// The grouped row products of lora_rows_seg_kernel with the expert's whole adapter slice resident
// in shared memory ([RN][Kin + 8], k contiguous; staged once, transposed on the way in when j is the
// contiguous index), so the stream of Y needs no barrier: each thread keeps the next 128-wide
// chunk of its two rows in flight while it multiplies the current one. Kin % 256 == 0.
//
// The block's rows make nrt = ceil(rows / 16) row tiles; the 8 warps split into 8 / nrt groups
// that take interleaved 128-wide k chunks of every tile, so a short segment (a tiny expert) keeps
// all warps streaming instead of one. The groups' partials are summed in group order through
// shared memory (the adapter slice is no longer needed by then), so the result does not depend on
// timing.
template <int NT>
__global__ void __launch_bounds__(256, 2) lora_rows_seg_z_kernel(
    const __nv_bfloat16* __restrict__ Y, long ldy, int Kin, const __nv_bfloat16* __restrict__ Z, long zj, long zk,
    long zes, const int* __restrict__ seg_off, const int* __restrict__ mblk_off, int E, int r, float oscale,
    float lscale, float* __restrict__ out, __nv_bfloat16* __restrict__ la, int RP) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  constexpr int RN = 8 * NT;
  constexpr int SK = 128;
  extern __shared__ __align__(16) __nv_bfloat16 zsd[];
  const int ZS = Kin + 8;
  const int total = __ldg(mblk_off + E);
  const int blk = blockIdx.x;
  if (blk >= total) return;
  int a = 0, b = E - 1;
  while (a < b) {
    const int mid = (a + b + 1) >> 1;
    if (__ldg(mblk_off + mid) <= blk) a = mid; else b = mid - 1;
  }
  const int e = a;
  const int row_lo = __ldg(seg_off + e) + (blk - __ldg(mblk_off + e)) * 128;
  const int row_hi = min(__ldg(seg_off + e + 1), row_lo + 128);
  const int nrt = (row_hi - row_lo + 15) >> 4;  // 1..8
  const int ngrp = 8 / nrt;
  const __nv_bfloat16* Ze = Z + (long)e * zes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = warp % nrt, grp = warp / nrt;
  const bool active = grp < ngrp;
  const int g = lane >> 2, c = lane & 3;
  const int r0 = row_lo + rt * 16 + g, r1 = r0 + 8;
  const bool v0 = active && r0 < row_hi, v1 = active && r1 < row_hi;
  const __nv_bfloat16* y0 = Y + (long)(v0 ? r0 : row_lo) * ldy;
  const __nv_bfloat16* y1 = Y + (long)(v1 ? r1 : row_lo) * ldy;
  auto load = [&](uint4 (&xa)[SK / 32], uint4 (&xb)[SK / 32], int k0) {
#pragma unroll
    for (int q = 0; q < SK / 32; ++q) {
      const int k = k0 + 32 * q + 8 * c;
      const bool in = k < Kin;
      xa[q] = (v0 && in) ? __ldg(reinterpret_cast<const uint4*>(y0 + k)) : make_uint4(0, 0, 0, 0);
      xb[q] = (v1 && in) ? __ldg(reinterpret_cast<const uint4*>(y1 + k)) : make_uint4(0, 0, 0, 0);
    }
  };
  const int kstep = ngrp * SK;
  // the first chunk is on its way while the adapter slice is staged
  uint4 xa0[SK / 32], xb0[SK / 32], xa1[SK / 32], xb1[SK / 32];
  load(xa0, xb0, grp * SK);
  // Only rows j < r of the slice are staged: a row j >= r of the shared tile only feeds accumulator
  // column j, which is never written out, so its contents do not matter.
  if (zk == 1) {
    const int n8 = r * (Kin / 8);
#pragma unroll 4
    for (int i = tid; i < n8; i += 256) {
      const int j = i / (Kin / 8), q = i - j * (Kin / 8);
      *reinterpret_cast<uint4*>(zsd + j * ZS + 8 * q) = __ldg(reinterpret_cast<const uint4*>(Ze + (long)j * zj + 8 * q));
    }
  } else if (zj == 1 && zk == r && (reinterpret_cast<uintptr_t>(Ze) & 15) == 0) {
    // [Kin][r] contiguous: 16-byte loads, scattered to [j][k]
#pragma unroll 4
    for (int i = tid; i < Kin * r / 8; i += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(Ze) + i);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int f = 8 * i + q, kk = f / r, j = f - kk * r;
        zsd[j * ZS + kk] = h[q];
      }
    }
  } else {
    for (int i = tid; i < Kin * r; i += 256) {
      const int kk = i / r, j = i - kk * r;
      zsd[j * ZS + kk] = Ze[(long)j * zj + (long)kk * zk];
    }
  }
  __syncthreads();
  const int nt_used = (r + 7) >> 3;  // tiles of 8 adapter columns holding a column j < r
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  auto compute = [&](const uint4 (&xa)[SK / 32], const uint4 (&xb)[SK / 32], int k0) {
#pragma unroll
    for (int q = 0; q < SK / 32; ++q) {
      const int k = k0 + 32 * q + 8 * c;
      const bool in = k < Kin;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t >= nt_used) break;
        const uint4 zq = in ? *reinterpret_cast<const uint4*>(zsd + (8 * t + g) * ZS + k) : make_uint4(0, 0, 0, 0);
        mma_16816(acc[t], xa[q].x, xb[q].x, xa[q].y, xb[q].y, zq.x, zq.y);
        mma_16816(acc[t], xa[q].z, xb[q].z, xa[q].w, xb[q].w, zq.z, zq.w);
      }
    }
  };
  if (active) {
    for (int k0 = grp * SK; k0 < Kin; k0 += 2 * kstep) {
      if (k0 + kstep < Kin) load(xa1, xb1, k0 + kstep);
      compute(xa0, xb0, k0);
      if (k0 + kstep < Kin) {
        if (k0 + 2 * kstep < Kin) load(xa0, xb0, k0 + 2 * kstep);
        compute(xa1, xb1, k0 + kstep);
      }
    }
  }
  if (ngrp > 1) {
    // partials of groups 1.. through shared memory: red[grp - 1][rt][lane][NT * 4]
    float* red = reinterpret_cast<float*>(zsd);
    __syncthreads();
    if (active && grp > 0) {
      float* dst = red + ((long)((grp - 1) * nrt + rt) * 32 + lane) * (NT * 4);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        *reinterpret_cast<float4*>(dst + 4 * t) = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
    }
    __syncthreads();
    if (grp == 0) {
      for (int o = 1; o < ngrp; ++o) {
        const float* src = red + ((long)((o - 1) * nrt + rt) * 32 + lane) * (NT * 4);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 v = *reinterpret_cast<const float4*>(src + 4 * t);
          acc[t][0] += v.x;
          acc[t][1] += v.y;
          acc[t][2] += v.z;
          acc[t][3] += v.w;
        }
      }
    }
  }
  // C fragment: rows r0 / r1, columns 8t + 2c (+1); written by the first group
  if (grp == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = hh ? r1 : r0;
        if (!(hh ? v1 : v0)) continue;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = 8 * t + 2 * c + q;
          const float v = acc[t][2 * hh + q];
          if (out != nullptr && j < r) out[(long)row * r + j] = oscale * v;
          if (la != nullptr && j < RP) {
            const float x = lscale * v;
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
            la[(long)row * 2 * RP + j] = j < r ? hi : __float2bfloat16(0.f);
            la[(long)row * 2 * RP + RP + j] = j < r ? lo : __float2bfloat16(0.f);
          }
        }
      }
    }
  }
  // padding columns of la beyond RN (RP > RN happens for r <= 16: RN = 16, RP = 32)
  if (la != nullptr && RP > RN) {
    for (int i = tid; i < 128 * (RP - RN); i += 256) {
      const int lr = i / (RP - RN), j = RN + i % (RP - RN);
      const int row = row_lo + lr;
      if (row < row_hi) {
        la[(long)row * 2 * RP + j] = __float2bfloat16(0.f);
        la[(long)row * 2 * RP + RP + j] = __float2bfloat16(0.f);
      }
    }
  }
}

// LB[e][n] = [Z_e(n, :) | Z_e(n, :)] zero padded to 2*RP columns; Z_e(n, j) = Z[e*zes + n*zn + j*zjs].
// blockIdx.y is the expert; an expert whose segment is empty (seg_off given) is skipped, since no
// GEMM tile reads its rows. One thread per row n: its r values are loaded together, then the
// 2*RP-wide row goes out as 16-byte stores.
__global__ void lora_bop_vec_kernel(const __nv_bfloat16* __restrict__ Z, long zn, long zjs, long zes, int rows,
                                    const int* __restrict__ seg_off, int r, int RP, __nv_bfloat16* __restrict__ LB) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  const int e = blockIdx.y;
  if (seg_off != nullptr && __ldg(seg_off + e) == __ldg(seg_off + e + 1)) return;
  const __nv_bfloat16* Ze = Z + (long)e * zes;
  __nv_bfloat16* LBe = LB + (long)e * rows * 2 * RP;
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < rows; n += gridDim.x * blockDim.x) {
    const __nv_bfloat16* zp = Ze + (long)n * zn;
    uint4* out = reinterpret_cast<uint4*>(LBe + (long)n * 2 * RP);
    for (int j0 = 0; j0 < RP; j0 += 8) {  // 8 rank columns at a time, written to both halves
      __nv_bfloat16 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = j0 + q < r ? zp[(long)(j0 + q) * zjs] : __float2bfloat16(0.f);
      const uint4 w = *reinterpret_cast<const uint4*>(v);
      out[j0 / 8] = w;
      out[(RP + j0) / 8] = w;
    }
  }
}

// out = scale * ordered sum over the slices of each expert (dense: all slices, E = 0, one output).
// transpose = 0: out[e][c][j]; transpose = 1: out[e][j][c]. blockIdx.y is the expert; an expert
// without slices (no tokens) gets exact zeros, 16 bytes per store (Ccols * r % 4 == 0).
__global__ void colred_reduce_kernel(const float* __restrict__ part, int Ccols, int r, int nslices_dense,
                                     const int* __restrict__ mblk_off, int E, float scale, int transpose,
                                     float* __restrict__ out) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  const int e = blockIdx.y;
  const int per_e = Ccols * r;
  int s0, s1;
  if (E == 0) { s0 = 0; s1 = nslices_dense; }
  else { s0 = __ldg(mblk_off + e); s1 = __ldg(mblk_off + e + 1); }
  float* oe = out + (long)e * per_e;
  if (s0 == s1) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < per_e / 4; i += gridDim.x * blockDim.x)
      reinterpret_cast<float4*>(oe)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  // i runs over the expert's output in its own order (consecutive threads write consecutive floats)
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < per_e; i += gridDim.x * blockDim.x) {
    int c, j;
    if (transpose) {
      j = i / Ccols;
      c = i - j * Ccols;
    } else {
      c = i / r;
      j = i - c * r;
    }
    float acc = 0.f;
    for (int s = s0; s < s1; ++s) acc += part[(long)s * per_e + c * r + j];
    oe[i] = scale * acc;
  }
}

// Ordered sum of the split-K partials of a dense GEMM: out[m][n] = sum_ks part[ks][m][n].
__global__ void split_reduce_kernel(const float* __restrict__ part, int ksplit, long stride, long count,
                                    void* __restrict__ out, int out_dtype) {
  pdl_wait();
  pdl_launch_dependents();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; 4 * i < count; i += (long)gridDim.x * blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int ks = 0; ks < ksplit; ++ks) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(part + ks * stride) + i);
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    if (out_dtype == QL_F32) {
      reinterpret_cast<float4*>(out)[i] = a;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      uint2 r;
      r.x = *reinterpret_cast<const uint32_t*>(&lo);
      r.y = *reinterpret_cast<const uint32_t*>(&hi);
      reinterpret_cast<uint2*>(out)[i] = r;
    }
  }
}

// Standalone dequant. fp32 output: one thread per 8 consecutive weights (decode8); bf16 output:
// one thread per 32-weight unit through the same decoder the tensor-core producers use.
template <int QT>
__global__ void gguf_dequant_kernel(const uint8_t* __restrict__ wq, long rows, long cols, void* __restrict__ out,
                                    int out_dtype) {
  const long groups_per_row = cols / 256;
  const long row_bytes = groups_per_row * QTraits<QT>::kGroupBytes;
  if (out_dtype == QL_F32) {
    const long total = rows * (cols / 8);
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
      const long row = i / (cols / 8);
      const long c8 = i % (cols / 8);  // chunk of 8 within the row
      const uint8_t* g = wq + row * row_bytes + (c8 / 32) * QTraits<QT>::kGroupBytes;
      float w[8];
      decode8<QT>(g, (int)(c8 % 32), w);
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + row * cols + c8 * 8);
      o[0] = make_float4(w[0], w[1], w[2], w[3]);
      o[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
  } else {
    const long total = rows * (cols / 32);
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
      const long row = i / (cols / 32);
      const long u = i % (cols / 32);  // unit of 32 within the row
      const uint8_t* g = wq + row * row_bytes + (u / 8) * QTraits<QT>::kGroupBytes;
      uint4 v[4];
      decode_unit_bf16<QT>(g, (int)(u % 8), v);
      uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + row * cols + u * 32);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) o[cc] = v[cc];
    }
  }
}

// A block that waits on a barrier no one arrives at (bounded-wait self-check).
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(smem_u32(&bar), 0, 99, true, limit_ns)) {
      // the wait recorded QL_ERR_TIMEOUT; nothing else to undo
    }
  }
  __syncthreads();
}

}  // namespace qlora
