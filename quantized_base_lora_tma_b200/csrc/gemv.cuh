// Small-M forward of the layer (M <= 16 tokens, decode-shaped): Y = X deq(W)^T + s (X A^T) B^T and
// H = X A^T, in one launch. This is the weight-streaming regime of the layer ("MMQ" for a few
// tokens, Show HN: LoRA over GGUF, "Things involved in the training"): every packed weight byte is
// read once and each weight is used M times, so the kernel is built to keep HBM busy rather than
// the tensor cores:
//
//   * A CTA owns 64 rows of W and a K slice; the KS CTAs of a cluster share the row block and split
//     K. One producer thread streams, per 256-wide K step, the 64 packed groups of the rows and the
//     X tile (tokens padded to 8 or 16 rows by the copy's zero fill) into a shared-memory ring by
//     TMA (no multicast).
//   * Eight warps share the 64 rows: two per 16-row set, each taking half of the eight 32-weight
//     blocks of a K step. A thread decodes its two rows' 8-weight runs straight into the A
//     fragments of mma.sync (bf16 in, fp32 accumulate; B = the X tile): the Q4_0 / Q8_0 block's
//     integers q - 8 / q are exact in bf16, so each 32-weight block is one exact integer-by-X
//     product pair of MMAs, scaled by the block's fp16 scale d in fp32 afterwards. The dequantized
//     weight never exists in any memory.
//   * The same warps accumulate H = X A^T over the slice on the tensor cores (two of the sixteen
//     k16 steps of a K step each); a ninth warp only issues the copies.
//   * Partials of the K slices (and of H) are summed through distributed shared memory in rank
//     order (deterministic); the adapter term s H B^T is added in fp32 in the same epilogue.
//
// Numerics: sum over blocks of d * (sum_k (q - 8) x) with fp32 accumulation, i.e. the exact decode
// d (q - 8) is applied without an intermediate bf16 rounding of the weight.
#pragma once
#include <cuda_bf16.h>

#include "decode.cuh"
#include "lora.cuh"
#include "ptx.cuh"

namespace qlora {

constexpr int kGvRows = 64;                    // W rows per CTA
constexpr int kGvWarps = 9;                    // 8 compute warps + producer / adapter warp
constexpr int kGvWarpA = 8;                    // the producer / adapter warp
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvMaxRank = 16;                 // adapter ranks this path takes (RN = 8 or 16)

template <int QT, int MT>
struct GvCfg {
  static constexpr int GB = QTraits<QT>::kGroupBytes;
  static constexpr int W_BYTES = kGvRows * GB;        // 64 packed groups
  static constexpr int XR = 8 * MT;                   // token rows of the X tile
  static constexpr int X_BOX = XR * 128;              // one 64-wide k box
  static constexpr int X_BYTES = 4 * X_BOX;
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int STAGES = 3;
  static constexpr int OFF_PART = STAGES * STAGE;                 // [2][64][16] fp32 partial outputs
  static constexpr int OFF_HP = OFF_PART + 2 * kGvRows * 16 * 4;  // [9][16][16] fp32: 8 warps' H, their sum
  static constexpr int OFF_HF = OFF_HP + 9 * 16 * 16 * 4;         // [16][16] fp32 summed H
  static constexpr int OFF_BAR = OFF_HF + 16 * 16 * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 2 * STAGES * 8 + 1024;  // + alignment slack
  static_assert(W_BYTES % 1024 == 0 && X_BOX % 1024 == 0, "128-byte-swizzled boxes need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct GvParams {
  int N, K, M, r;
  int kgroups;     // 256-wide K steps per cluster rank
  float scale;
  const __nv_bfloat16* A;  // [r x K]
  const __nv_bfloat16* B;  // [N x r]
  void* Y;                 // [M x N]
  int y_dtype;
  float* H;                // [M x r]
};

// mma.sync m16n8k16 with a zero accumulator input.
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// 8 bytes at p (2-byte aligned; MIS = p % 4 known at compile time) as two words.
template <int MIS>
__device__ __forceinline__ void lds8(const uint8_t* p, uint32_t& x0, uint32_t& x1) {
  if (MIS == 0) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);  // 8-byte aligned here (see callers)
    x0 = v.x;
    x1 = v.y;
  } else {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(p - 2);
    const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
    x0 = __funnelshift_r(w0, w1, 16);
    x1 = __funnelshift_r(w1, w2, 16);
  }
}

// Low-nibble pair -> exact bf16 pair: the bytes picked by sel land in the low and high halves;
// with the bf16 exponent of 128 OR-ed in, a nibble n reads 128 + n (bf16 has 7 mantissa bits, so
// only a low nibble can be placed this way), and one subtraction of 136 gives n - 8 exactly.
__device__ __forceinline__ uint32_t nib2_bf16(uint32_t x, uint32_t sel) {
  const uint32_t t = __byte_perm(x, 0u, sel);
  return bf16x2_sub((t & 0x000F000Fu) | 0x43004300u, 0x43084308u /* bf16 (136, 136) */);
}

// Integers of weights [8c, 8c + 8) of block `blk` of a packed 256-weight group at g, as four bf16
// pairs (consecutive k), and the block's scale. Q4_0: q - 8; Q8_0: q.
template <int QT, int BLK>
__device__ __forceinline__ void gv_decode(const uint8_t* g, int c, uint32_t (&a)[4], float& d);

template <int QT, int BLK>
__device__ __forceinline__ void gv_decode(const uint8_t* g, int c, uint32_t (&a)[4], float& d) {
  if (QT == QL_Q4_0) {
    // block: fp16 d, 16 bytes; byte j = weight j (low nibble) and j + 16 (high nibble).
    // weights [8c, 8c + 8): bytes 8 (c & 1) .. + 8, nibble c >> 1. Block start 18 BLK: the bytes
    // start at 18 BLK + 2 + 8 (c & 1), which is 4-aligned for odd BLK (the group is 16-aligned).
    const uint8_t* b = g + 18 * BLK;
    d = __half2float(*reinterpret_cast<const __half*>(b));
    uint32_t x0, x1;
    const uint8_t* p = b + 2 + 8 * (c & 1);
    if (BLK & 1) {
      x0 = *reinterpret_cast<const uint32_t*>(p);
      x1 = *reinterpret_cast<const uint32_t*>(p + 4);
    } else {
      lds8<2>(p, x0, x1);
    }
    // lanes taking high nibbles shift them down first (a per-lane amount: no divergence)
    const uint32_t sh = (uint32_t)(c >> 1) * 4u;
    x0 >>= sh;
    x1 >>= sh;
    a[0] = nib2_bf16(x0, 0x4140u);
    a[1] = nib2_bf16(x0, 0x4342u);
    a[2] = nib2_bf16(x1, 0x4140u);
    a[3] = nib2_bf16(x1, 0x4342u);
  } else {
    // Q8_0 block: fp16 d, 32 int8; weights [8c, 8c + 8) are bytes 2 + 8c .. + 8 (4-aligned for
    // odd BLK). int8 -> exact fp32 by the 2^23 magic (q + 128 biased byte), then to bf16.
    const uint8_t* b = g + 34 * BLK;
    d = __half2float(*reinterpret_cast<const __half*>(b));
    uint32_t x0, x1;
    const uint8_t* p = b + 2 + 8 * c;
    if (BLK & 1) {
      x0 = *reinterpret_cast<const uint32_t*>(p);
      x1 = *reinterpret_cast<const uint32_t*>(p + 4);
    } else {
      lds8<2>(p, x0, x1);
    }
    const float2 bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t x = (h ? x1 : x0) ^ 0x80808080u;
      float f[4];
      magic4(x, f);
      const float2 p0 = __fadd2_rn(make_float2(f[0], f[1]), bias);
      const float2 p1 = __fadd2_rn(make_float2(f[2], f[3]), bias);
      a[2 * h] = bf16x2_bits(p0.x, p0.y);
      a[2 * h + 1] = bf16x2_bits(p1.x, p1.y);
    }
  }
}

// X or adapter-A element pair (row, k, k + 1) of a 128-byte-swizzled box of 64 k (row pitch 128 B).
__device__ __forceinline__ uint32_t sw128_pair(const uint8_t* box, int row, int kk) {
  return *reinterpret_cast<const uint32_t*>(box + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4) + (kk & 7) * 2);
}
__device__ __forceinline__ uint4 sw128_chunk(const uint8_t* box, int row, int chunk) {
  return *reinterpret_cast<const uint4*>(box + row * 128 + ((chunk ^ (row & 7)) << 4));
}

// One 256-wide K step of rows g0 and g1 (= g0 + 8 rows): eight 32-weight blocks, each two exact
// integer MMAs per token tile and one fp32 scale-accumulate per output.
template <int QT, int MT, int BLK>
__device__ __forceinline__ void gv_block(const uint8_t* g0, const uint8_t* g1, const uint8_t* xs, int c, int g,
                                         float (&acc)[MT][4]) {
  uint32_t a[4], b[4];
  float d0, d1;
  gv_decode<QT, BLK>(g0, c, a, d0);
  gv_decode<QT, BLK>(g1, c, b, d1);
  const uint8_t* xb = xs + (BLK >> 1) * GvCfg<QT, MT>::X_BOX;
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const uint4 xv = sw128_chunk(xb, 8 * t + g, 4 * (BLK & 1) + c);
    float dblk[4];
    mma_16816_z(dblk, a[0], b[0], a[1], b[1], xv.x, xv.y);
    mma_16816(dblk, a[2], b[2], a[3], b[3], xv.z, xv.w);
    acc[t][0] = fmaf(d0, dblk[0], acc[t][0]);
    acc[t][1] = fmaf(d0, dblk[1], acc[t][1]);
    acc[t][2] = fmaf(d1, dblk[2], acc[t][2]);
    acc[t][3] = fmaf(d1, dblk[3], acc[t][3]);
  }
}
// Blocks [4 HALF, 4 HALF + 4) of a K step (two warps share a row set, one half each).
template <int QT, int MT, int HALF>
__device__ __forceinline__ void gv_block_half(const uint8_t* g0, const uint8_t* g1, const uint8_t* xs, int c, int g,
                                              float (&acc)[MT][4]) {
  gv_block<QT, MT, 4 * HALF + 0>(g0, g1, xs, c, g, acc);
  gv_block<QT, MT, 4 * HALF + 1>(g0, g1, xs, c, g, acc);
  gv_block<QT, MT, 4 * HALF + 2>(g0, g1, xs, c, g, acc);
  gv_block<QT, MT, 4 * HALF + 3>(g0, g1, xs, c, g, acc);
}

template <int QT, int MT>
__global__ void __launch_bounds__(kGvThreads) qgemv_fwd_kernel(const __grid_constant__ CUtensorMap tmW,
                                                               const __grid_constant__ CUtensorMap tmX,
                                                               const GvParams p) {
  using C = GvCfg<QT, MT>;
  extern __shared__ uint8_t gv_smem_raw[];
  const uint32_t base_u32 = (smem_u32(gv_smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = gv_smem_raw + (base_u32 - smem_u32(gv_smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int KS = gridDim.y;
  const int n0 = blockIdx.x * kGvRows;
  const int kg0 = (int)rank * p.kgroups;                        // first 256-wide K step of the slice
  const int nst = max(0, min(p.kgroups, p.K / 256 - kg0));      // steps of this slice
  const uint32_t bar0 = base_u32 + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  float* part = reinterpret_cast<float*>(smem + C::OFF_PART);
  float* hp = reinterpret_cast<float*>(smem + C::OFF_HP);
  float* hf = reinterpret_cast<float*>(smem + C::OFF_HF);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kGvWarps - 1);  // the compute warps
    }
    fence_mbar_init();
  }
  if (warp == kGvWarpA && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  __syncthreads();
  pdl_wait();  // inputs of the previous kernel in the stream are complete from here on
  pdl_launch_dependents();  // after the wait: a dependent may rely on what this launch waited for

  auto issue = [&](int i) {  // stage i of this slice into slot i % STAGES
    const int s = i % C::STAGES;
    const uint32_t st = base_u32 + s * C::STAGE;
    const int kg = kg0 + i;
    mbar_arrive_expect_tx(full_bar(s), C::STAGE);
    tma_load_2d(st, &tmW, full_bar(s), kg * (C::GB / 4), n0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      tma_load_2d(st + C::W_BYTES + q * C::X_BOX, &tmX, full_bar(s), kg * 256 + 64 * q, 0);
    }
  };

  bool ok = true;
  float acc[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  float hacc[2][4];
#pragma unroll
  for (int t = 0; t < 2; ++t) hacc[t][0] = hacc[t][1] = hacc[t][2] = hacc[t][3] = 0.f;

  if (warp == kGvWarpA) {
    // ---- producer: lane 0 refills each slot as soon as the compute warps release it ----
    if (lane == 0) {
      for (int i = 0; i < nst; ++i) {
        if (i >= C::STAGES && !mbar_wait(empty_bar(i % C::STAGES), ((i / C::STAGES) & 1) ^ 1, 41)) {
          ok = false;
          break;
        }
        issue(i);
      }
    }
  } else {
    // ---- weight rows 16 (warp % 4) + g and + 8; blocks of half warp / 4 of each K step; and
    // H = X A^T over k16 steps warp and warp + 8 of each K step ----
    const int R0 = 16 * (warp & 3) + g;
    const int half = warp >> 2;
    for (int i = 0; i < nst; ++i) {
      const int s = i % C::STAGES;
      if (!warp_wait(full_bar(s), (i / C::STAGES) & 1, 43)) { ok = false; break; }
      const uint8_t* ws = smem + s * C::STAGE;
      const uint8_t* xs = ws + C::W_BYTES;
      const uint8_t* g0 = ws + R0 * C::GB;
      const uint8_t* g1 = g0 + 8 * C::GB;
      if (half == 0) gv_block_half<QT, MT, 0>(g0, g1, xs, c, g, acc);
      else gv_block_half<QT, MT, 1>(g0, g1, xs, c, g, acc);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int k16 = warp + 8 * h2;
        const int q = k16 >> 2, kk = (k16 & 3) * 16;
        const uint8_t* xb = xs + q * C::X_BOX;
        const long kglob = (long)(kg0 + i) * 256 + 64 * q + kk;  // this k16 step of the adapter A
        const uint32_t a0 = sw128_pair(xb, g, kk + 2 * c);
        const uint32_t a2 = sw128_pair(xb, g, kk + 2 * c + 8);
        const uint32_t a1 = MT == 2 ? sw128_pair(xb, g + 8, kk + 2 * c) : 0u;
        const uint32_t a3 = MT == 2 ? sw128_pair(xb, g + 8, kk + 2 * c + 8) : 0u;
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
          if (jt == 1 && p.r <= 8) break;
          const int j = 8 * jt + g;
          uint32_t b0 = 0u, b1 = 0u;
          if (j < p.r) {
            const __nv_bfloat16* ar = p.A + (long)j * p.K + kglob + 2 * c;
            b0 = __ldg(reinterpret_cast<const unsigned int*>(ar));
            b1 = __ldg(reinterpret_cast<const unsigned int*>(ar + 8));
          }
          mma_16816(hacc[jt], a0, a1, a2, a3, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
    // this warp's H partial: rows m = g, g + 8; cols j = 8 jt + 2c, + 1
    float* hw = hp + warp * 256;
#pragma unroll
    for (int jt = 0; jt < 2; ++jt) {
      const int j = 8 * jt + 2 * c;
      hw[g * 16 + j] = hacc[jt][0];
      hw[g * 16 + j + 1] = hacc[jt][1];
      hw[(g + 8) * 16 + j] = hacc[jt][2];
      hw[(g + 8) * 16 + j + 1] = hacc[jt][3];
    }
    // partial outputs of this half: rows R0, R0 + 8; tokens 8t + 2c, + 1
    float* ph = part + half * kGvRows * 16;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int m = 8 * t + 2 * c;
      ph[R0 * 16 + m] = acc[t][0];
      ph[R0 * 16 + m + 1] = acc[t][1];
      ph[(R0 + 8) * 16 + m] = acc[t][2];
      ph[(R0 + 8) * 16 + m + 1] = acc[t][3];
    }
  }
  if (!ok || dev_aborted()) spin_ns(2000000ull);  // copies issued before a wait gave up land first
  __syncthreads();
  // the two halves of every K step, and the eight warps' H partials, in a fixed order
  for (int i = threadIdx.x; i < kGvRows * 16; i += kGvThreads) part[i] += part[kGvRows * 16 + i];
  for (int i = threadIdx.x; i < 256; i += kGvThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += hp[w * 256 + i];
    hp[8 * 256 + i] = v;
  }
  cluster_sync_all();
  // H = sum over the cluster's slices, in rank order
  for (int i = threadIdx.x; i < 16 * 16; i += kGvThreads) hf[i] = cluster_sum_ordered(&hp[8 * 256 + i], KS);
  __syncthreads();
  if (blockIdx.x == 0 && rank == 0 && p.H != nullptr)
    for (int i = threadIdx.x; i < p.M * p.r; i += kGvThreads) p.H[i] = hf[(i / p.r) * 16 + i % p.r];
  // rank q finishes rows [q * rows_per, (q + 1) * rows_per) of the block
  const int rows_per = (kGvRows + KS - 1) / KS;
  const int rlo = (int)rank * rows_per;
  const int rhi = min(kGvRows, rlo + rows_per);
  for (int i = threadIdx.x; i < (rhi - rlo) * p.M; i += kGvThreads) {
    const int m = i / (rhi - rlo), R = rlo + i % (rhi - rlo);
    const int n = n0 + R;
    float y = cluster_sum_ordered(&part[R * 16 + m], KS);
    float l = 0.f;
    for (int j = 0; j < p.r; ++j) l = fmaf(hf[m * 16 + j], __bfloat162float(p.B[(long)n * p.r + j]), l);
    y = fmaf(p.scale, l, y);
    if (p.y_dtype == QL_F32) reinterpret_cast<float*>(p.Y)[(long)m * p.N + n] = y;
    else reinterpret_cast<__nv_bfloat16*>(p.Y)[(long)m * p.N + n] = __float2bfloat16_rn(y);
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its partials
}

}  // namespace qlora
