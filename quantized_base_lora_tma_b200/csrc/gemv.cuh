// Small-M forward of the layer (M <= 16 tokens, decode-shaped): Y = X deq(W)^T + s (X A^T) B^T and
// H = X A^T. This is the weight-streaming regime of the layer (the quantized matmul at a few tokens, Show HN:
// LoRA over GGUF, "Things involved in the training"): every packed weight byte is read once and
// each weight is used M times, so the kernels are built to keep HBM busy with as few instructions
// per weight as the decode allows. Three launches:
//
//   * gemv_h_kernel: H in one CTA. The weight stream does not need it and runs beside it.
//   * qgemv_fwd_kernel: persistent, two CTAs per SM, each a balanced range of steps (ROWS rows of W
//     x 256 k) that may span the end of one row block and the start of the next (stream-K). One
//     producer thread streams the packed groups and the X tile (tokens padded to 8 or 16 rows by
//     the copy's zero fill) into a shared-memory ring by TMA (no multicast), each stage tagged with
//     its row block. Warp w takes the block pair w % 4 of every step (two 32-weight blocks, 4-byte
//     aligned) for half of the rows; it builds the X fragments of its two blocks once per step and
//     reuses them for all its row tiles, and decodes its rows' bytes straight into the A
//     fragments of mma.sync (bf16 in, fp32 accumulate). The k order inside a block is free (X
//     follows it), so a bf16 pair costs one shift and one LOP3:
//       Q4_0: a 32-bit word of qs holds bytes 4c .. 4c + 3; (w >> 8s) & 0x000F000F | 0x43004300
//       puts two nibbles n into two bf16 lanes reading 128 + n, exactly. The offset (136 per
//       weight, i.e. 128 + 8) is removed through the accumulator input of the block's first MMA:
//       -136 times the block's sum of X, itself an MMA of the X fragments with a constant -136.
//       Q8_0: q via the 2^23 magic float, exact, then to bf16.
//     Each 32-weight block's exact integer-by-X sum is scaled by its fp16 scale d in fp32. At the
//     end of a row block's piece the four block pairs' partials are summed in order into the
//     piece's slot in global memory.
//   * gemv_finish_kernel: per 32 rows, the row block's slots in order plus s H B^T (fp32).
//
// Numerics: sum over blocks of d * (sum_k (q - 8) x) (Q4_0) or d * (sum_k q x) (Q8_0), fp32
// accumulation in a fixed order; the decoded weight is never rounded.
#pragma once
#include <cuda_bf16.h>

#include "decode.cuh"
#include "lora.cuh"
#include "ptx.cuh"

namespace qlora {

constexpr int kGvCompute = 8;     // compute warps
constexpr int kGvWarpP = 8;       // the producer warp
constexpr int kGvWarpL = 9;       // the warp that releases the next launch
constexpr int kGvWarps = 10;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvMaxRank = 16;    // adapter ranks this path takes

template <int QT, int MT>
struct GvCfg {
  static constexpr int ROWS = QT == QL_Q4_0 ? 128 : 64;  // W rows per K step
  static constexpr int RT = ROWS / 32;                    // row tiles (16 rows) per warp
  static constexpr int GB = QTraits<QT>::kGroupBytes;     // bytes per 256 weights of a row
  static constexpr int PB = GB / 4;                       // bytes per block pair
  static constexpr int W_BYTES = ROWS * GB;
  static constexpr int XR = 8 * MT;                       // token rows of the X tile
  static constexpr int X_BOX = XR * 128;                  // one 64-wide k box
  static constexpr int X_BYTES = 4 * X_BOX;
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = MT == 2 ? 3 : 4;
  static constexpr int OFF_PART = STAGES * STAGE;         // [4 pairs][XR tokens][ROWS] fp32
  static constexpr int OFF_META = OFF_PART + 4 * XR * ROWS * 4;  // per stage: row block, piece flags
  static constexpr int OFF_BAR = OFF_META + 2 * 4 * STAGES + 16;
  static constexpr int SMEM_BYTES = OFF_BAR + (2 * STAGES + 1) * 8 + 1024;  // + alignment slack
  static_assert(W_BYTES % 1024 == 0 && X_BOX % 1024 == 0, "128-byte-swizzled boxes need 1 KB alignment");
  static_assert(SMEM_BYTES <= 116 * 1024, "two CTAs per SM");
};

// Work of the weight-streaming kernel: T = NRB * KSTEPS steps (ROWS rows x 256 k each), step
// t = row block * KSTEPS + K step; CTA i of G takes steps [i T / G, (i + 1) T / G). The part of a
// row block inside one CTA's range is a piece; its fp32 partial goes to slot (CTA - first CTA of
// the row block), and gemv_finish_kernel sums a row block's slots in order.
struct GvParams {
  int N, K, M, r;
  uint32_t nib_mask, bf16_magic;  // 0x000F000F, 0x43004300 (registers for the Q4_0 decode)
  int ksteps, T, maxslots;
  float* gpart;            // [NRB][maxslots][XR][ROWS] piece partials
};

// First step of CTA i's range, and the CTA whose range holds step s.
__host__ __device__ __forceinline__ long gv_start(int i, int T, int G) { return (long)i * T / G; }
__host__ __device__ __forceinline__ int gv_cta_of(long s, int T, int G) {
  int i = (int)(s * G / T);
  while (i + 1 < G && gv_start(i + 1, T, G) <= s) ++i;
  while (i > 0 && gv_start(i, T, G) > s) --i;
  return i;
}

// mma.sync m16n8k16 with a zero accumulator input.
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// mma.sync m16n8k16 with a separate accumulator input.
__device__ __forceinline__ void mma_16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1, const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// Element k of token row `row` of a 128-byte-swizzled box of 64 k (row pitch 128 bytes).
__device__ __forceinline__ const uint8_t* gv_x_at(const uint8_t* box, int row, int k) {
  return box + row * 128 + ((((k >> 3) ^ (row & 7))) << 4) + (k & 7) * 2;
}

// (a & b) | c in one LOP3. The masks come in as registers (kernel parameters): with both as
// immediates the compiler would split the operation in two.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Q4_0: w holds qs bytes 4c .. 4c + 3 of a block (low nibbles: weights 4c .. 4c + 3, high nibbles:
// 16 + 4c ..). p[0] = (4c, 4c + 2), p[1] = (4c + 1, 4c + 3), p[2] = (16 + 4c, 16 + 4c + 2),
// p[3] = (16 + 4c + 1, 16 + 4c + 3), each lane the bf16 128 + n (nm = 0x000F000F,
// mg = 0x43004300).
__device__ __forceinline__ void gv_q4_pairs(uint32_t w, uint32_t nm, uint32_t mg, uint32_t (&p)[4]) {
  p[0] = and_or(w, nm, mg);
  p[1] = and_or(w >> 8, nm, mg);
  p[2] = and_or(w >> 4, nm, mg);
  p[3] = and_or(w >> 12, nm, mg);
}

// Q8_0: w holds 4 int8 weights (k, k + 1, k + 2, k + 3) -> bf16 pairs (k, k + 1), (k + 2, k + 3).
__device__ __forceinline__ void gv_q8_pairs(uint32_t w, uint32_t& p01, uint32_t& p23) {
  float f[4];
  magic4(w ^ 0x80808080u, f);
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  const float2 a = __fadd2_rn(make_float2(f[0], f[1]), bias);
  const float2 b = __fadd2_rn(make_float2(f[2], f[3]), bias);
  p01 = bf16x2_bits(a.x, a.y);
  p23 = bf16x2_bits(b.x, b.y);
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __low2float(*reinterpret_cast<const __half2*>(&w)); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __high2float(*reinterpret_cast<const __half2*>(&w)); }

// One row's registers for the block pair at rb (4-byte aligned; rbc = rb + 4c): fr[blk] = the
// A-fragment words of the block's two MMAs in order (MMA0 k slots 2c.., 2c+8..; MMA1 the same), and
// the blocks' scales.
template <int QT>
__device__ __forceinline__ void gv_row_pair(const uint8_t* rb, const uint8_t* rbc, uint32_t nm, uint32_t mg,
                                            uint32_t (&fr)[2][4], float (&d)[2]) {
  const uint32_t* W = reinterpret_cast<const uint32_t*>(rb);
  const uint32_t* Wc = reinterpret_cast<const uint32_t*>(rbc);
  if (QT == QL_Q4_0) {
    // block A: fp16 d at 0, qs at 2 .. 17; block B: d at 18, qs at 20 .. 35
    d[0] = half_lo(W[0]);
    d[1] = half_hi(W[4]);
    gv_q4_pairs(__funnelshift_r(Wc[0], Wc[1], 16), nm, mg, fr[0]);
    gv_q4_pairs(Wc[5], nm, mg, fr[1]);
  } else {
    // block A: d at 0, qs at 2 .. 33; block B: d at 34, qs at 36 .. 67
    d[0] = half_lo(W[0]);
    d[1] = half_hi(W[8]);
    gv_q8_pairs(__funnelshift_r(Wc[0], Wc[1], 16), fr[0][0], fr[0][1]);  // weights 4c .. 4c + 3
    gv_q8_pairs(__funnelshift_r(Wc[4], Wc[5], 16), fr[0][2], fr[0][3]);  // 16 + 4c ..
    gv_q8_pairs(Wc[9], fr[1][0], fr[1][1]);
    gv_q8_pairs(Wc[13], fr[1][2], fr[1][3]);
  }
}

// H = X A^T for m < M <= 16, j < r <= 16, in one CTA: warp w takes the k16 steps w, w + 32, .. (mma.sync,
// A = X rows, B = adapter rows; four steps' loads in flight at a time) and the 32 warps' sums are
// added in order. Writes hf [16][16] (zero past M and r) for the finish kernel and H [M x r].
// It runs beside the weight stream.
constexpr int kGvHWarps = 32;
__global__ void __launch_bounds__(kGvHWarps * 32) gemv_h_kernel(const __nv_bfloat16* __restrict__ X,
                                                                const __nv_bfloat16* __restrict__ A, int M, int K,
                                                                int r, float* __restrict__ hf, float* __restrict__ H) {
  __shared__ float red[kGvHWarps][256];
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  float acc[2][4];
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) acc[jt][0] = acc[jt][1] = acc[jt][2] = acc[jt][3] = 0.f;
  auto ld = [&](const __nv_bfloat16* p, int row, int rows, int k) -> uint32_t {
    return row < rows ? __ldg(reinterpret_cast<const unsigned int*>(p + (long)row * K + k)) : 0u;
  };
  constexpr int U = 4;
  for (int k0 = 16 * warp; k0 < K; k0 += 16 * kGvHWarps * U) {
    uint32_t a[U][4], b[U][2][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + 16 * kGvHWarps * u;
      const bool in = k < K;
      a[u][0] = in ? ld(X, g, M, k + 2 * c) : 0u;
      a[u][1] = in ? ld(X, g + 8, M, k + 2 * c) : 0u;
      a[u][2] = in ? ld(X, g, M, k + 2 * c + 8) : 0u;
      a[u][3] = in ? ld(X, g + 8, M, k + 2 * c + 8) : 0u;
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) {
        b[u][jt][0] = in ? ld(A, 8 * jt + g, r, k + 2 * c) : 0u;
        b[u][jt][1] = in ? ld(A, 8 * jt + g, r, k + 2 * c + 8) : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) mma_16816(acc[jt], a[u][0], a[u][1], a[u][2], a[u][3], b[u][jt][0], b[u][jt][1]);
  }
  // acc[jt]: (m = g, j = 8 jt + 2c, + 1) and (m = g + 8, same j)
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    const int j = 8 * jt + 2 * c;
    red[warp][g * 16 + j] = acc[jt][0];
    red[warp][g * 16 + j + 1] = acc[jt][1];
    red[warp][(g + 8) * 16 + j] = acc[jt][2];
    red[warp][(g + 8) * 16 + j + 1] = acc[jt][3];
  }
  __syncthreads();
  if (threadIdx.x < 256) {
    float v = 0.f;
    for (int w = 0; w < kGvHWarps; ++w) v += red[w][threadIdx.x];
    hf[threadIdx.x] = v;
    const int m = threadIdx.x >> 4, j = threadIdx.x & 15;
    if (H != nullptr && m < M && j < r) H[m * r + j] = v;
  }
}

// The backward's row products for m < M <= 16, j < r <= 16, in one CTA like gemv_h_kernel:
// G = s dY B with B [N x r] (j contiguous: each B fragment pairs two rows of B), written as
// la = split(G) [M x 2RP] (zero past r); hs = split(s H) [M x 2RP] for the column reductions,
// whose counters (zc, zn) it zeroes.
__global__ void __launch_bounds__(kGvHWarps * 32) gemv_g_kernel(const __nv_bfloat16* __restrict__ dY,
                                                                const __nv_bfloat16* __restrict__ B,
                                                                const float* __restrict__ H, int M, int N, int r,
                                                                float scale, int RP, __nv_bfloat16* __restrict__ la,
                                                                __nv_bfloat16* __restrict__ hs, int* __restrict__ zc,
                                                                int zn) {
  __shared__ float red[kGvHWarps][256];
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < zn; i += blockDim.x) zc[i] = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  float acc[2][4];
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) acc[jt][0] = acc[jt][1] = acc[jt][2] = acc[jt][3] = 0.f;
  auto ldy = [&](int row, int k) -> uint32_t {
    return row < M ? __ldg(reinterpret_cast<const unsigned int*>(dY + (long)row * N + k)) : 0u;
  };
  auto ldb = [&](int j, int k) -> uint32_t {  // (B[k][j], B[k + 1][j])
    if (j >= r) return 0u;
    const unsigned short lo = __ldg(reinterpret_cast<const unsigned short*>(B + (long)k * r + j));
    const unsigned short hi = __ldg(reinterpret_cast<const unsigned short*>(B + (long)(k + 1) * r + j));
    return (uint32_t)lo | ((uint32_t)hi << 16);
  };
  constexpr int U = 4;
  for (int k0 = 16 * warp; k0 < N; k0 += 16 * kGvHWarps * U) {
    uint32_t a[U][4], b[U][2][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + 16 * kGvHWarps * u;
      const bool in = k < N;
      a[u][0] = in ? ldy(g, k + 2 * c) : 0u;
      a[u][1] = in ? ldy(g + 8, k + 2 * c) : 0u;
      a[u][2] = in ? ldy(g, k + 2 * c + 8) : 0u;
      a[u][3] = in ? ldy(g + 8, k + 2 * c + 8) : 0u;
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) {
        b[u][jt][0] = in ? ldb(8 * jt + g, k + 2 * c) : 0u;
        b[u][jt][1] = in ? ldb(8 * jt + g, k + 2 * c + 8) : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) mma_16816(acc[jt], a[u][0], a[u][1], a[u][2], a[u][3], b[u][jt][0], b[u][jt][1]);
  }
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    const int j = 8 * jt + 2 * c;
    red[warp][g * 16 + j] = acc[jt][0];
    red[warp][g * 16 + j + 1] = acc[jt][1];
    red[warp][(g + 8) * 16 + j] = acc[jt][2];
    red[warp][(g + 8) * 16 + j + 1] = acc[jt][3];
  }
  __syncthreads();
  if (threadIdx.x < 256) {
    float v = 0.f;
    for (int w = 0; w < kGvHWarps; ++w) v += red[w][threadIdx.x];
    const int m = threadIdx.x >> 4, j = threadIdx.x & 15;
    if (m < M) {
      const float x = j < r ? scale * v : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      la[(long)m * 2 * RP + j] = hi;
      la[(long)m * 2 * RP + RP + j] = __float2bfloat16_rn(x - __bfloat162float(hi));
      for (int jj = 16 + j; jj < RP; jj += 16) {
        la[(long)m * 2 * RP + jj] = __float2bfloat16(0.f);
        la[(long)m * 2 * RP + RP + jj] = __float2bfloat16(0.f);
      }
    }
  }
  for (int i = threadIdx.x; i < M * RP; i += blockDim.x) {
    const int m = i / RP, j = i % RP;
    const float x = j < r ? scale * H[m * r + j] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    hs[(long)m * 2 * RP + j] = hi;
    hs[(long)m * 2 * RP + RP + j] = __float2bfloat16_rn(x - __bfloat162float(hi));
  }
}

// The weight-streaming kernel (stream-K over row blocks x K steps; see GvParams).
template <int QT, int MT>
__global__ void __launch_bounds__(kGvThreads, 2) qgemv_fwd_kernel(const __grid_constant__ CUtensorMap tmW,
                                                               const __grid_constant__ CUtensorMap tmX,
                                                               const GvParams p) {
  using C = GvCfg<QT, MT>;
  extern __shared__ uint8_t gv_smem_raw[];
  const uint32_t base_u32 = (smem_u32(gv_smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = gv_smem_raw + (base_u32 - smem_u32(gv_smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int G = gridDim.x;
  const long s0 = gv_start(blockIdx.x, p.T, G), s1 = gv_start(blockIdx.x + 1, p.T, G);
  const int nsteps = (int)(s1 - s0);
  const uint32_t bar0 = base_u32 + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  const uint32_t sync_bar = bar0 + 8u * (2 * C::STAGES);
  float* part = reinterpret_cast<float*>(smem + C::OFF_PART);
  volatile int* meta = reinterpret_cast<volatile int*>(smem + C::OFF_META);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kGvCompute);
    }
    mbar_init(sync_bar, kGvCompute);
    fence_mbar_init();
  }
  if (warp == kGvWarpP && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  // W and X come from before the H kernel that precedes this launch (it waited for its predecessor
  // before it let this launch start), so the stream needs no wait.

  bool ok = true;
  if (warp == kGvWarpP) {
    // ---- producer: lane 0 streams the range's steps, tagging each stage with its row block and
    // whether it opens or closes a piece ----
    if (lane == 0) {
      for (int it = 0; it < nsteps; ++it) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES && !mbar_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 41)) {
          ok = false;
          break;
        }
        // ramp: stages 2 and 3 only once stages 0 and 1 have landed, so that the first data of
        // every CTA is not queued behind the whole ring's worth of every other CTA
        if (it >= 2 && it < C::STAGES && !mbar_wait(full_bar(it - 2), 0u, 42)) {
          ok = false;
          break;
        }
        const long t = s0 + it;
        const int rb = (int)(t / p.ksteps), ks = (int)(t - (long)rb * p.ksteps);
        meta[2 * s] = rb;
        meta[2 * s + 1] = (it == 0 || ks == 0 ? 1 : 0) | (it == nsteps - 1 || ks == p.ksteps - 1 ? 2 : 0);
        const uint32_t st = base_u32 + s * C::STAGE;
        mbar_arrive_expect_tx(full_bar(s), C::STAGE);
        tma_load_2d(st, &tmW, full_bar(s), ks * (C::GB / 4), rb * C::ROWS);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tma_load_2d(st + C::W_BYTES + q * C::X_BOX, &tmX, full_bar(s), ks * 256 + 64 * q, 0);
      }
    }
    __syncwarp();  // the idle lanes wait here, not at the final wait (which would hold lane 0)
  } else if (warp < kGvCompute) {
    const int tid = threadIdx.x;                   // 0 .. 255
    const int bp = warp & 3;                       // block pair of every K step
    const int rbase = (warp >> 2) * (C::ROWS / 2);  // first row of this warp's half
    const int thr_off = (rbase + g) * C::GB + bp * C::PB;
    const uint32_t nm = p.nib_mask, mg = p.bf16_magic;
    uint32_t sync_par = 0;
    auto consumer_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(sync_bar);
      const bool w = __all_sync(0xffffffffu, mbar_wait(sync_bar, sync_par, 44));
      sync_par ^= 1u;
      return w;
    };
    float acc[C::RT][MT][4];
    for (int it = 0; it < nsteps; ++it) {
      const int s = it % C::STAGES;
      if (!warp_wait(full_bar(s), (it / C::STAGES) & 1, 43)) { ok = false; break; }
      const int rb = meta[2 * s], fl = meta[2 * s + 1];
      if (fl & 1) {
#pragma unroll
        for (int t = 0; t < C::RT; ++t)
#pragma unroll
          for (int tt = 0; tt < MT; ++tt) acc[t][tt][0] = acc[t][tt][1] = acc[t][tt][2] = acc[t][tt][3] = 0.f;
      }
      const uint8_t* ws = smem + s * C::STAGE;
      const uint8_t* xbox = ws + C::W_BYTES + bp * C::X_BOX;  // blocks 2bp, 2bp + 1: k 64 bp .. + 63
      // X fragments of the two blocks (per token tile) in the k order of the A fragments, and for
      // Q4_0 the offset term -136 * (block sum of X) in accumulator layout
      uint32_t xf[2][MT][4];
      float cz[2][MT][4];
#pragma unroll
      for (int blk = 0; blk < 2; ++blk)
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
          const int row = 8 * tt + g;
          const uint2 u0 = *reinterpret_cast<const uint2*>(gv_x_at(xbox, row, 32 * blk + 4 * c));
          const uint2 u1 = *reinterpret_cast<const uint2*>(gv_x_at(xbox, row, 32 * blk + 16 + 4 * c));
          if (QT == QL_Q4_0) {
            xf[blk][tt][0] = __byte_perm(u0.x, u0.y, 0x5410);  // x(4c), x(4c + 2)
            xf[blk][tt][1] = __byte_perm(u0.x, u0.y, 0x7632);  // x(4c + 1), x(4c + 3)
            xf[blk][tt][2] = __byte_perm(u1.x, u1.y, 0x5410);
            xf[blk][tt][3] = __byte_perm(u1.x, u1.y, 0x7632);
            const uint32_t m136 = 0xC308C308u;  // bf16 (-136, -136)
            mma_16816_z(cz[blk][tt], m136, m136, m136, m136, xf[blk][tt][0], xf[blk][tt][1]);
            mma_16816(cz[blk][tt], m136, m136, m136, m136, xf[blk][tt][2], xf[blk][tt][3]);
          } else {
            xf[blk][tt][0] = u0.x;
            xf[blk][tt][1] = u0.y;
            xf[blk][tt][2] = u1.x;
            xf[blk][tt][3] = u1.y;
          }
        }
      const uint8_t* rbp = ws + thr_off;  // the thread's first row, its block pair
#pragma unroll
      for (int t = 0; t < C::RT; ++t) {
        uint32_t f0[2][4], f1[2][4];
        float d0[2], d1[2];
        gv_row_pair<QT>(rbp + 16 * t * C::GB, rbp + 16 * t * C::GB + 4 * c, nm, mg, f0, d0);
        gv_row_pair<QT>(rbp + (16 * t + 8) * C::GB, rbp + (16 * t + 8) * C::GB + 4 * c, nm, mg, f1, d1);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk)
#pragma unroll
          for (int tt = 0; tt < MT; ++tt) {
            float dblk[4];
            if (QT == QL_Q4_0)
              mma_16816_c(dblk, f0[blk][0], f1[blk][0], f0[blk][1], f1[blk][1], xf[blk][tt][0], xf[blk][tt][1],
                          cz[blk][tt]);
            else
              mma_16816_z(dblk, f0[blk][0], f1[blk][0], f0[blk][1], f1[blk][1], xf[blk][tt][0], xf[blk][tt][1]);
            mma_16816(dblk, f0[blk][2], f1[blk][2], f0[blk][3], f1[blk][3], xf[blk][tt][2], xf[blk][tt][3]);
            acc[t][tt][0] = fmaf(d0[blk], dblk[0], acc[t][tt][0]);
            acc[t][tt][1] = fmaf(d0[blk], dblk[1], acc[t][tt][1]);
            acc[t][tt][2] = fmaf(d1[blk], dblk[2], acc[t][tt][2]);
            acc[t][tt][3] = fmaf(d1[blk], dblk[3], acc[t][tt][3]);
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
      if (!(fl & 2)) continue;

      // ---- end of a piece of row block rb: the four pairs' partials, summed in order, go to the
      // piece's slot ----
      {
        float* pw = part + bp * (C::XR * C::ROWS);
#pragma unroll
        for (int t = 0; t < C::RT; ++t)
#pragma unroll
          for (int tt = 0; tt < MT; ++tt) {
            const int R0 = rbase + 16 * t + g, m = 8 * tt + 2 * c;
            pw[m * C::ROWS + R0] = acc[t][tt][0];
            pw[(m + 1) * C::ROWS + R0] = acc[t][tt][1];
            pw[m * C::ROWS + R0 + 8] = acc[t][tt][2];
            pw[(m + 1) * C::ROWS + R0 + 8] = acc[t][tt][3];
          }
      }
      if (!consumer_sync()) { ok = false; break; }
      constexpr int SZ = C::XR * C::ROWS;
      const int cfirst = gv_cta_of((long)rb * p.ksteps, p.T, G);
      float* gp = p.gpart + ((long)rb * p.maxslots + (blockIdx.x - cfirst)) * SZ;
      for (int i = tid; i < p.M * C::ROWS; i += kGvCompute * 32)  // i = m ROWS + R
        gp[i] = ((part[i] + part[SZ + i]) + part[2 * SZ + i]) + part[3 * SZ + i];
      if (!consumer_sync()) { ok = false; break; }  // part is free for the next piece
    }
  }
  if (!ok || dev_aborted()) spin_ns(2000000ull);  // copies issued before a wait gave up land first
  if (warp == kGvWarpL && lane == 0) {
    // the next launch may start once every CTA has seen the H kernel complete
    pdl_wait();
    pdl_launch_dependents();
  }
  pdl_wait();  // this launch completes only after the H kernel has
}

// Y[m][n] = sum over the row block's slots in order + s sum_j H[m][j] B[n][j], for the 32 rows
// [32 blockIdx.x, + 32) of the block's row block (of `rows` rows).
__global__ void __launch_bounds__(128) gemv_finish_kernel(const float* __restrict__ gpart, int maxslots, int xr,
                                                          int rows, int ksteps, int T, int G,
                                                          const float* __restrict__ hf,
                                                          const __nv_bfloat16* __restrict__ B, int N, int M, int r,
                                                          float scale, void* __restrict__ Y, int y_dtype) {
  pdl_wait();
  pdl_launch_dependents();
  const int n0 = 32 * blockIdx.x;
  const int rb = n0 / rows, R0 = n0 - rb * rows;
  const long t0 = (long)rb * ksteps;
  const int cfirst = gv_cta_of(t0, T, G);
  const int np = gv_cta_of(t0 + ksteps - 1, T, G) - cfirst + 1;
  const long sz = (long)xr * rows;
  const float* gb = gpart + (long)rb * maxslots * sz;
  for (int i = threadIdx.x; i < M * 32; i += blockDim.x) {
    const int m = i >> 5, R = R0 + (i & 31), n = rb * rows + R;
    if (n >= N) continue;  // rows past N (zero filled by the copy) of the last row block
    float y = 0.f;
    for (int q = 0; q < np; ++q) y += gb[q * sz + m * rows + R];
    float l = 0.f;
    for (int j = 0; j < r; ++j) l = fmaf(hf[m * 16 + j], __bfloat162float(B[(long)n * r + j]), l);
    y = fmaf(scale, l, y);
    if (y_dtype == QL_F32) reinterpret_cast<float*>(Y)[(long)m * N + n] = y;
    else reinterpret_cast<__nv_bfloat16*>(Y)[(long)m * N + n] = __float2bfloat16_rn(y);
  }
}

}  // namespace qlora

namespace qlora {

// ------------------------------------------------------------------------------------------------
// Small-M input gradient (M <= 16, Q4_0): dX = dY deq(W) + G A with G = s dY B (from the row kernel,
// as its split operand LA = [hi | lo]). Two launches:
//   * qgemv_dx_kernel: persistent, stream-K over steps (k group of 256 columns of W, 128 rows of W),
//     t = k group * NB + row block, so that a CTA's range walks down the rows of one k group (a
//     piece) into the next. Warp w owns block w of the k group (32 columns of W = 32 outputs) and
//     all 128 rows of a step; the reduction runs over the rows of W, so the MMA is
//     D[k][token] += sum_n W[n][k] dY[token][n] with A = W^T (16 k x 16 rows) and B = dY^T.
//     The k order inside an MMA tile is free: tile row g is byte 2g of the block's qs and tile row
//     g + 8 byte 2g + 1 (low nibbles in the first k tile, high nibbles in the second), so one byte
//     permute of two rows' byte pairs gives a word that decodes like a forward word (one shift and
//     one LOP3 per bf16 pair, 128 + q). The row scale d[n] cannot come out of a sum over rows: it
//     multiplies the B operand in fp32 (dY[token][n] d[n], fed as a bf16 hi + lo pair, so the
//     whole product is fp32-accurate), and the offset (136 per weight) enters as MMAs of a
//     constant -136 with that B. Each warp writes its 32
//     columns of the piece's partial straight from its accumulators.
//   * qgemv_dx_finish_kernel: per 256 columns, the k group's slots in CTA order plus G A (fp32).
// ------------------------------------------------------------------------------------------------
template <int MT>
struct GvdCfg {
  static constexpr int ROWS = 128;                        // rows of W per step
  static constexpr int GB = QTraits<QL_Q4_0>::kGroupBytes;  // 144
  static constexpr int W_BYTES = ROWS * GB;
  static constexpr int XR = 8 * MT;                       // token rows of the dY tile
  static constexpr int Y_BOX = XR * 128;                  // 64 rows of W (n) x XR tokens
  static constexpr int Y_BYTES = 2 * Y_BOX;
  static constexpr int STAGE = W_BYTES + Y_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int OFF_META = STAGES * STAGE;
  static constexpr int OFF_BAR = OFF_META + 2 * 4 * STAGES + 16;
  static constexpr int SMEM_BYTES = OFF_BAR + 2 * STAGES * 8 + 1024;
  static_assert(W_BYTES % 1024 == 0 && Y_BOX % 1024 == 0, "128-byte-swizzled boxes need 1 KB alignment");
  static_assert(SMEM_BYTES <= 116 * 1024, "two CTAs per SM");
};

struct GvdParams {
  int N, K, M;
  uint32_t nib_mask, bf16_magic;  // 0x000F000F, 0x43004300
  int nb, T, maxslots;            // row blocks of 128, steps, slots per k group
  float* gpart;                   // [K/256][maxslots][XR][256] piece partials
};

template <int MT>
__global__ void __launch_bounds__(kGvThreads, 2) qgemv_dx_kernel(const __grid_constant__ CUtensorMap tmW,
                                                                 const __grid_constant__ CUtensorMap tmY,
                                                                 const GvdParams p) {
  using C = GvdCfg<MT>;
  extern __shared__ uint8_t gvd_smem_raw[];
  const uint32_t base_u32 = (smem_u32(gvd_smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = gvd_smem_raw + (base_u32 - smem_u32(gvd_smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int G = gridDim.x;
  const long s0 = gv_start(blockIdx.x, p.T, G), s1 = gv_start(blockIdx.x + 1, p.T, G);
  const int nsteps = (int)(s1 - s0);
  const uint32_t bar0 = base_u32 + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  volatile int* meta = reinterpret_cast<volatile int*>(smem + C::OFF_META);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kGvCompute);
    }
    fence_mbar_init();
  }
  if (warp == kGvWarpP && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmY);
  }
  __syncthreads();
  // W and dY come from before the row kernel that precedes this launch (it waited for its
  // predecessor before it let this launch start): the stream needs no wait.

  bool ok = true;
  if (warp == kGvWarpP) {
    if (lane == 0) {
      for (int it = 0; it < nsteps; ++it) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES && !mbar_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, 45)) {
          ok = false;
          break;
        }
        if (it >= 2 && it < C::STAGES && !mbar_wait(full_bar(it - 2), 0u, 46)) {
          ok = false;
          break;
        }
        const long t = s0 + it;
        const int kg = (int)(t / p.nb), nbk = (int)(t - (long)kg * p.nb);
        meta[2 * s] = kg;
        meta[2 * s + 1] = (it == 0 || nbk == 0 ? 1 : 0) | (it == nsteps - 1 || nbk == p.nb - 1 ? 2 : 0);
        const uint32_t st = base_u32 + s * C::STAGE;
        mbar_arrive_expect_tx(full_bar(s), C::STAGE);
        tma_load_2d(st, &tmW, full_bar(s), kg * (C::GB / 4), nbk * C::ROWS);
        tma_load_2d(st + C::W_BYTES, &tmY, full_bar(s), nbk * C::ROWS, 0);
        tma_load_2d(st + C::W_BYTES + C::Y_BOX, &tmY, full_bar(s), nbk * C::ROWS + 64, 0);
      }
    }
    __syncwarp();  // the idle lanes wait here, not at the final wait (which would hold lane 0)
  } else if (warp < kGvCompute) {
    const uint32_t nm = p.nib_mask, mg = p.bf16_magic;
    const int b = warp;                        // block of the k group
    const uint32_t m136 = 0xC308C308u;         // bf16 (-136, -136)
    float acc[2][MT][4];                       // k tiles (low / high nibbles) x token tiles
    for (int it = 0; it < nsteps; ++it) {
      const int s = it % C::STAGES;
      if (!warp_wait(full_bar(s), (it / C::STAGES) & 1, 47)) { ok = false; break; }
      const int kg = meta[2 * s], fl = meta[2 * s + 1];
      if (fl & 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int tt = 0; tt < MT; ++tt) acc[h][tt][0] = acc[h][tt][1] = acc[h][tt][2] = acc[h][tt][3] = 0.f;
      }
      const uint8_t* ws = smem + s * C::STAGE;
      const uint8_t* ys = ws + C::W_BYTES;
#pragma unroll 2
      for (int nt = 0; nt < C::ROWS / 16; ++nt) {
        // this thread's rows of W: n0 = 16 nt + 2c, n0 + 1, n0 + 8, n0 + 9 (the MMA's k columns)
        const int n0 = 16 * nt + 2 * c;
        const uint8_t* r0 = ws + n0 * C::GB + 18 * b;
        const uint32_t q0 = *reinterpret_cast<const uint16_t*>(r0 + 2 + 2 * g);
        const uint32_t q1 = *reinterpret_cast<const uint16_t*>(r0 + C::GB + 2 + 2 * g);
        const uint32_t q2 = *reinterpret_cast<const uint16_t*>(r0 + 8 * C::GB + 2 + 2 * g);
        const uint32_t q3 = *reinterpret_cast<const uint16_t*>(r0 + 9 * C::GB + 2 + 2 * g);
        const float d0 = __half2float(*reinterpret_cast<const __half*>(r0));
        const float d1 = __half2float(*reinterpret_cast<const __half*>(r0 + C::GB));
        const float d2 = __half2float(*reinterpret_cast<const __half*>(r0 + 8 * C::GB));
        const float d3 = __half2float(*reinterpret_cast<const __half*>(r0 + 9 * C::GB));
        // bytes (2g, 2g + 1) of rows n0, n0 + 1 -> tile rows g, g + 8 of columns 2c, 2c + 1
        uint32_t pa[4], pb[4];
        gv_q4_pairs(__byte_perm(q0, q1, 0x5410), nm, mg, pa);  // pa: a0 t0, a1 t0, a0 t1, a1 t1
        gv_q4_pairs(__byte_perm(q2, q3, 0x5410), nm, mg, pb);  // pb: a2 t0, a3 t0, a2 t1, a3 t1
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
          const int row = 8 * tt + g;  // token
          const uint8_t* yb = ys + (n0 >> 6) * C::Y_BOX;
          const uint32_t y01 = *reinterpret_cast<const uint32_t*>(gv_x_at(yb, row, n0 & 63));
          const uint32_t y23 = *reinterpret_cast<const uint32_t*>(gv_x_at(yb, row, (n0 + 8) & 63));
          const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&y01));
          const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&y23));
          // B = dY d as a bf16 hi + lo pair (fp32-accurate): the weight integers are exact, so the
          // sum over rows carries no rounding of its own beyond fp32
          const float e0 = f01.x * d0, e1 = f01.y * d1, e2 = f23.x * d2, e3 = f23.y * d3;
          const uint32_t h0 = bf16x2_bits(e0, e1), h1 = bf16x2_bits(e2, e3);
          const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h0));
          const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h1));
          const uint32_t l0 = bf16x2_bits(e0 - g01.x, e1 - g01.y), l1 = bf16x2_bits(e2 - g23.x, e3 - g23.y);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            mma_16816(acc[h][tt], m136, m136, m136, m136, h0, h1);
            mma_16816(acc[h][tt], m136, m136, m136, m136, l0, l1);
            mma_16816(acc[h][tt], pa[2 * h], pa[2 * h + 1], pb[2 * h], pb[2 * h + 1], h0, h1);
            mma_16816(acc[h][tt], pa[2 * h], pa[2 * h + 1], pb[2 * h], pb[2 * h + 1], l0, l1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
      if (!(fl & 2)) continue;
      // end of a piece of k group kg: this warp's 32 columns x tokens straight to the slot.
      // acc[h][tt]: rows (k) g, g + 8 of tile h -> columns 32b + 16h + 2g, + 1; tokens 8tt + 2c, + 1
      const int cfirst = gv_cta_of((long)kg * p.nb, p.T, G);
      float* gp = p.gpart + ((long)kg * p.maxslots + (blockIdx.x - cfirst)) * (C::XR * 256);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
          const int col = 32 * b + 16 * h + 2 * g, m = 8 * tt + 2 * c;
          *reinterpret_cast<float2*>(gp + m * 256 + col) = make_float2(acc[h][tt][0], acc[h][tt][2]);
          *reinterpret_cast<float2*>(gp + (m + 1) * 256 + col) = make_float2(acc[h][tt][1], acc[h][tt][3]);
        }
    }
  }
  if (!ok || dev_aborted()) spin_ns(2000000ull);  // copies issued before a wait gave up land first
  if (warp == kGvWarpL && lane == 0) {
    pdl_wait();
    pdl_launch_dependents();
  }
  pdl_wait();
}

// dX[m][k] = the k group's slots in CTA order + sum_j G[m][j] A[j][k], G = hi + lo of LA [M x 2RP];
// one CTA per k group (256 columns).
__global__ void __launch_bounds__(256) qgemv_dx_finish_kernel(const float* __restrict__ gpart, int maxslots, int xr,
                                                              int nb, int T, int G, const __nv_bfloat16* __restrict__ LA,
                                                              int RP, const __nv_bfloat16* __restrict__ A, int r, int M,
                                                              int K, void* __restrict__ dX, int dx_dtype) {
  __shared__ float gs[8][64];
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < 8 * 64; i += blockDim.x) {
    const int m = i >> 6, j = i & 63;
    gs[m][j] = (m < M && j < r)
                   ? __bfloat162float(LA[(long)m * 2 * RP + j]) + __bfloat162float(LA[(long)m * 2 * RP + RP + j])
                   : 0.f;
  }
  const int kg = blockIdx.x;
  const long t0 = (long)kg * nb;
  const int cfirst = gv_cta_of(t0, T, G);
  const int np = gv_cta_of(t0 + nb - 1, T, G) - cfirst + 1;
  const long sz = (long)xr * 256;
  const float* gb = gpart + (long)kg * maxslots * sz + threadIdx.x;
  const int k = kg * 256 + threadIdx.x;
  // thread = output column k for every token (M <= 8): the slot loads of all tokens, then the
  // adapter column, go out together
  float y[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) y[m] = 0.f;
  for (int q = 0; q < np; ++q)
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (m < M) y[m] += gb[q * sz + m * 256];
  float l[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) l[m] = 0.f;
  __syncthreads();  // gs
#pragma unroll 8
  for (int j = 0; j < r; ++j) {
    const float av = __bfloat162float(A[(long)j * K + k]);
#pragma unroll
    for (int m = 0; m < 8; ++m) l[m] = fmaf(gs[m][j], av, l[m]);
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    if (m >= M) break;
    const float v = y[m] + l[m];
    if (dx_dtype == QL_F32) reinterpret_cast<float*>(dX)[(long)m * K + k] = v;
    else reinterpret_cast<__nv_bfloat16*>(dX)[(long)m * K + k] = __float2bfloat16_rn(v);
  }
}

}  // namespace qlora
