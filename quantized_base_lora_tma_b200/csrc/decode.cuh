// GGUF block decode on the device: 8 consecutive weights of one 256-weight group of a packed row.
//
// A "group" is the packed bytes of 256 consecutive weights of one row: 8 Q8_0 blocks (272 B),
// 8 Q4_0 blocks (144 B), or one Q4_K (144 B), Q5_K (176 B) or Q6_K (210 B) superblock. Groups are the
// unit every kernel here moves: except Q6_K's, their byte size is a multiple of 16, so they can be
// copied by TMA and rows of K % 256 == 0 weights start 16-byte aligned.
//
// Values are the exact decode rounded once to fp32 (each product below is exact in fp32; the Q4_K /
// Q5_K difference is formed by one fused multiply-add, i.e. one rounding), which a caller then rounds
// to bf16 (nearest even) for the tensor cores.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "qlora.h"

namespace qlora {

template <int QT>
struct QTraits;
template <>
struct QTraits<QL_Q8_0> {
  static constexpr int kGroupBytes = 272;
};
template <>
struct QTraits<QL_Q4_0> {
  static constexpr int kGroupBytes = 144;
};
template <>
struct QTraits<QL_Q4_K> {
  static constexpr int kGroupBytes = 144;
};
template <>
struct QTraits<QL_Q5_K> {
  static constexpr int kGroupBytes = 176;
};
// 84 bytes is not a multiple of 16 either: like Q6_K, Q2_K is read by the standalone dequant only.
template <>
struct QTraits<QL_Q2_K> {
  static constexpr int kGroupBytes = 84;
};
// 210 bytes is not a multiple of 16: Q6_K groups cannot be TMA-copied one by one, so only the
// standalone dequant (byte and half-word loads) reads them.
template <>
struct QTraits<QL_Q6_K> {
  static constexpr int kGroupBytes = 210;
};

__device__ __forceinline__ uint32_t pack2_same(__nv_bfloat16 h) {
  const uint32_t u = __bfloat16_as_ushort(h);
  return u | (u << 16);
}

__device__ __forceinline__ float half_at(const uint8_t* p) {
  return __half2float(*reinterpret_cast<const __half*>(p));
}

// 8 bytes starting at a 2-byte aligned address.
__device__ __forceinline__ uint2 load8_a2(const uint8_t* p) {
  const uint16_t* h = reinterpret_cast<const uint16_t*>(p);
  uint16_t a = h[0], b = h[1], c = h[2], d = h[3];
  return make_uint2((uint32_t)a | ((uint32_t)b << 16), (uint32_t)c | ((uint32_t)d << 16));
}

// Decode weights [8c, 8c+8) of the group starting at g (c in [0, 32)).
template <int QT>
__device__ __forceinline__ void decode8(const uint8_t* g, int c, float (&w)[8]);

// Q8_0: block b = c/4 (34 B: fp16 d, 32 int8 q); w = d * q.
template <>
__device__ __forceinline__ void decode8<QL_Q8_0>(const uint8_t* g, int c, float (&w)[8]) {
  const uint8_t* b = g + 34 * (c >> 2);
  const float d = half_at(b);
  const uint2 q = load8_a2(b + 2 + 8 * (c & 3));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = d * (float)(int8_t)(q.x >> (8 * i));
    w[4 + i] = d * (float)(int8_t)(q.y >> (8 * i));
  }
}

// Q4_0: block b = c/4 (18 B: fp16 d, 16 bytes); byte j holds element j (low nibble) and j+16
// (high nibble); w = d * (q - 8). Chunk c&3 = 0,1 -> low nibbles of bytes 0..7 / 8..15;
// 2,3 -> high nibbles of bytes 0..7 / 8..15.
template <>
__device__ __forceinline__ void decode8<QL_Q4_0>(const uint8_t* g, int c, float (&w)[8]) {
  const uint8_t* b = g + 18 * (c >> 2);
  const float d = half_at(b);
  const int sub = c & 3;
  const uint2 q = load8_a2(b + 2 + 8 * (sub & 1));
  const int sh = (sub >> 1) * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = d * (float)((int)((q.x >> (8 * i + sh)) & 15u) - 8);
    w[4 + i] = d * (float)((int)((q.y >> (8 * i + sh)) & 15u) - 8);
  }
}

// Q4_K superblock (144 B): fp16 d, fp16 dmin, 12 bytes S of 6-bit (sc, m) for 8 sub-blocks of 32,
// 128 bytes of nibbles (32-byte group i: sub-block 2i low nibbles, 2i+1 high nibbles);
// w = d*sc*q - dmin*m.
template <>
__device__ __forceinline__ void decode8<QL_Q4_K>(const uint8_t* g, int c, float (&w)[8]) {
  const float d = half_at(g);
  const float dmin = half_at(g + 2);
  const uint8_t* S = g + 4;
  const int j = c >> 2;
  int sc, m;
  if (j < 4) {
    sc = S[j] & 63;
    m = S[j + 4] & 63;
  } else {
    sc = (S[j + 4] & 15) | ((S[j - 4] >> 6) << 4);
    m = (S[j + 4] >> 4) | ((S[j] >> 6) << 4);
  }
  const float ds = d * (float)sc;      // exact (11 + 6 bits)
  const float dm = -(dmin * (float)m);  // exact
  const uint2 q = *reinterpret_cast<const uint2*>(g + 16 + 32 * (j >> 1) + 8 * (c & 3));
  const int sh = (j & 1) * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = fmaf(ds, (float)((q.x >> (8 * i + sh)) & 15u), dm);
    w[4 + i] = fmaf(ds, (float)((q.y >> (8 * i + sh)) & 15u), dm);
  }
}

// The 6-bit (sc, m) pair of sub-block j from the 12 scale bytes S shared by Q4_K and Q5_K.
__device__ __forceinline__ void k_scale_min(const uint8_t* S, int j, int& sc, int& m) {
  if (j < 4) {
    sc = S[j] & 63;
    m = S[j + 4] & 63;
  } else {
    sc = (S[j + 4] & 15) | ((S[j - 4] >> 6) << 4);
    m = (S[j + 4] >> 4) | ((S[j] >> 6) << 4);
  }
}

// Q5_K superblock (176 B): fp16 d, fp16 dmin, the 12 scale bytes, 32 bytes qh, 128 bytes of nibbles
// (as Q4_K); weight l of sub-block j: q = nibble + 16 * bit j of qh[l]; w = d*sc*q - dmin*m.
template <>
__device__ __forceinline__ void decode8<QL_Q5_K>(const uint8_t* g, int c, float (&w)[8]) {
  const float d = half_at(g);
  const float dmin = half_at(g + 2);
  const int j = c >> 2, l0 = 8 * (c & 3);
  int sc, m;
  k_scale_min(g + 4, j, sc, m);
  const float ds = d * (float)sc;       // exact (11 + 6 bits)
  const float dm = -(dmin * (float)m);  // exact
  const uint2 q = *reinterpret_cast<const uint2*>(g + 48 + 32 * (j >> 1) + l0);
  const uint2 h = *reinterpret_cast<const uint2*>(g + 16 + l0);
  const int sh = (j & 1) * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q0 = (int)((q.x >> (8 * i + sh)) & 15u) | (int)(((h.x >> (8 * i + j)) & 1u) << 4);
    const int q1 = (int)((q.y >> (8 * i + sh)) & 15u) | (int)(((h.y >> (8 * i + j)) & 1u) << 4);
    w[i] = fmaf(ds, (float)q0, dm);
    w[4 + i] = fmaf(ds, (float)q1, dm);
  }
}

// Q6_K superblock (210 B): 128 bytes ql, 64 bytes qh, 16 int8 scales, fp16 d. Weight 32a + l of half
// h: q = (nibble (a >> 1) of ql[64h + 32(a & 1) + l]) | ((qh[32h + l] >> 2a) & 3) << 4, scale
// scales[8h + 2a + l / 16]; w = d * scale * (q - 32), exact in fp32 (at most 11 + 7 + 6 bits). The
// superblocks are only 2-byte aligned.
template <>
__device__ __forceinline__ void decode8<QL_Q6_K>(const uint8_t* g, int c, float (&w)[8]) {
  const int h = c >> 4, p0 = 8 * (c & 15);
  const int a = p0 >> 5, l0 = p0 & 31;
  const float ds = half_at(g + 208) * (float)(int8_t)g[192 + 8 * h + 2 * a + (l0 >> 4)];
  const uint2 lo = load8_a2(g + 64 * h + 32 * (a & 1) + l0);
  const uint2 hi = load8_a2(g + 128 + 32 * h + l0);
  const int sl = 4 * (a >> 1), shh = 2 * a;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q0 = (int)((lo.x >> (8 * i + sl)) & 15u) | (int)(((hi.x >> (8 * i + shh)) & 3u) << 4);
    const int q1 = (int)((lo.y >> (8 * i + sl)) & 15u) | (int)(((hi.y >> (8 * i + shh)) & 3u) << 4);
    w[i] = ds * (float)(q0 - 32);
    w[4 + i] = ds * (float)(q1 - 32);
  }
}

// Q2_K superblock (84 B): 16 scale bytes (low nibble scale, high nibble min, one per 16 weights),
// 64 bytes of 2-bit codes, fp16 d at 80, fp16 dmin at 82. Weight 32a + l of half h: code
// (qs[32h + l] >> 2a) & 3, scale byte S = scales[8h + 2a + l / 16]; w = d*(S & 15)*q - dmin*(S >> 4).
// Both products are exact in fp32 (at most 11 + 4 + 2 bits); one fp32 FMA rounds the difference
// once. The superblocks are 4-byte aligned; the 8 codes of a chunk are two aligned words.
template <>
__device__ __forceinline__ void decode8<QL_Q2_K>(const uint8_t* g, int c, float (&w)[8]) {
  const int h = c >> 4, p0 = 8 * (c & 15);
  const int a = p0 >> 5, l0 = p0 & 31;
  const int S = g[8 * h + 2 * a + (l0 >> 4)];
  const float ds = half_at(g + 80) * (float)(S & 15);
  const float dm = -(half_at(g + 82) * (float)(S >> 4));
  const uint32_t* qw = reinterpret_cast<const uint32_t*>(g + 16 + 32 * h + l0);
  const uint32_t q0 = qw[0] >> (2 * a), q1 = qw[1] >> (2 * a);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = __fmaf_rn(ds, (float)((q0 >> (8 * i)) & 3u), dm);
    w[4 + i] = __fmaf_rn(ds, (float)((q1 >> (8 * i)) & 3u), dm);
  }
}

// ------------------------------------------------------------------------------------------------
// Whole-unit decode to bf16 for the tensor-core producers: weights [32u, 32u + 32) of a group
// (one Q8_0 / Q4_0 block, or 32 weights of a K-quant superblock) as four 16-byte chunks
// of 8 bf16. Every result equals RNE_bf16 of the exact decoded value (which is exact in fp32).
// Integer-to-float conversion uses the 2^23 magic: the float with bit pattern 0x4B000000 | b is
// 2^23 + b for a byte b, so one byte permute plus one subtraction yields an exact small integer.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 32 bytes starting at a 2-byte aligned address p, as 8 words (the read stays inside [p, p+32)
// rounded out to whole words).
// The aligned base is formed by pointer arithmetic on p (not through an integer), so the compiler
// keeps p's address space (shared-memory loads stay LDS).
__device__ __forceinline__ void load32_a2(const uint8_t* p, uint32_t (&x)[8]) {
  const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(p) & 3u);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(p - mis);
  const uint32_t sh = mis * 8u;
  uint32_t v[9];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = w[i];
  v[8] = sh ? w[8] : 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __funnelshift_r(v[i], v[i + 1], sh);
}

// 16 bytes starting at a 2-byte aligned address p, as 4 words.
__device__ __forceinline__ void load16_a2(const uint8_t* p, uint32_t (&x)[4]) {
  const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(p) & 3u);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(p - mis);
  const uint32_t sh = mis * 8u;
  uint32_t v[5];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = w[i];
  v[4] = sh ? w[4] : 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = __funnelshift_r(v[i], v[i + 1], sh);
}

// Four bytes of a word (each the low 8 bits of 2^23 + b) -> four exact floats 2^23 + b.
__device__ __forceinline__ void magic4(uint32_t x, float (&f)[4]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) f[e] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440u + e));
}

template <int QT>
__device__ __forceinline__ void decode_unit_bf16(const uint8_t* g, int u, uint4 (&out)[4]);

// Q8_0: w = d * q, q int8. Bytes are biased to q + 128 so that 2^23 + (q + 128) is the magic float.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q8_0>(const uint8_t* g, int u, uint4 (&out)[4]) {
  const uint8_t* b = g + 34 * u;
  const float d = half_at(b);
  uint32_t x[8];
  load32_a2(b + 2, x);
  const float2 dd = make_float2(d, d);
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[4];
    magic4(x[i] ^ 0x80808080u, f);
    const float2 a = __fmul2_rn(__fadd2_rn(make_float2(f[0], f[1]), bias), dd);
    const float2 c = __fmul2_rn(__fadd2_rn(make_float2(f[2], f[3]), bias), dd);
    o[2 * i] = bf16x2_bits(a.x, a.y);
    o[2 * i + 1] = bf16x2_bits(c.x, c.y);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) out[cc] = make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Q4_0: w = d * (q - 8). d (fp16, 11 significant bits) = d1 + d2 with d1 = bf16(d) and d2 = d - d1
// (at most 3 significant bits, so exact in bf16). v = q - 8 is exact in bf16 and d2 * v has at most
// 7 significant bits, so c = d2 * v is exact and one fused bf16 FMA d1 * v + c rounds d * v once:
// the result is RNE_bf16 of the exact value. The bf16 magic 0x4300 | n is 128 + n for a nibble n.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q4_0>(const uint8_t* g, int u, uint4 (&out)[4]) {
  const uint8_t* b = g + 18 * u;
  const float d = half_at(b);
  const __nv_bfloat16 d1 = __float2bfloat16_rn(d);
  const __nv_bfloat16 d2 = __float2bfloat16_rn(d - __bfloat162float(d1));
  const uint32_t D1 = pack2_same(d1), D2 = pack2_same(d2);
  const uint32_t B136 = 0x43084308u;  // bf16 pair (136, 136)
  uint32_t x[4];
  load16_a2(b + 2, x);
  uint32_t o[16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // h = 0: low nibbles (weights 0..15), 1: high nibbles (16..31)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w = h ? (x[i] >> 4) : x[i];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const uint32_t t = __byte_perm(w, 0u, (uint32_t)(2 * pr) | 0x4000u | ((uint32_t)(2 * pr + 1) << 8) | 0x40u);
        const uint32_t m = (t & 0x000F000Fu) | 0x43004300u;
        const uint32_t v = bf16x2_sub(m, B136);
        o[8 * h + 2 * i + pr] = bf16x2_fma(v, D1, bf16x2_mul(v, D2));
      }
    }
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) out[cc] = make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
}

// Q4_K sub-block u: w = (d*sc) * q - dmin*m with both products exact in fp32; one fp32 FMA rounds
// the difference once, then one bf16 rounding.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q4_K>(const uint8_t* g, int u, uint4 (&out)[4]) {
  const float d = half_at(g);
  const float dmin = half_at(g + 2);
  const uint8_t* S = g + 4;
  const int j = u;
  int sc, m;
  if (j < 4) {
    sc = S[j] & 63;
    m = S[j + 4] & 63;
  } else {
    sc = (S[j + 4] & 15) | ((S[j - 4] >> 6) << 4);
    m = (S[j + 4] >> 4) | ((S[j] >> 6) << 4);
  }
  const float ds = d * (float)sc;
  const float dm = -(dmin * (float)m);
  const uint4* qp = reinterpret_cast<const uint4*>(g + 16 + 32 * (j >> 1));
  const uint4 q0 = qp[0], q1 = qp[1];
  const uint32_t xs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  const uint32_t sh = (uint32_t)(j & 1) * 4u;
  const float2 dsv = make_float2(ds, ds), dmv = make_float2(dm, dm);
  const float2 bias = make_float2(-8388608.0f, -8388608.0f);  // -2^23
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[4];
    magic4((xs[i] >> sh) & 0x0F0F0F0Fu, f);
    const float2 a = __ffma2_rn(__fadd2_rn(make_float2(f[0], f[1]), bias), dsv, dmv);
    const float2 c = __ffma2_rn(__fadd2_rn(make_float2(f[2], f[3]), bias), dsv, dmv);
    o[2 * i] = bf16x2_bits(a.x, a.y);
    o[2 * i + 1] = bf16x2_bits(c.x, c.y);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) out[cc] = make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
}

// Q5_K sub-block u: as Q4_K with the fifth bit of each code from bit u of the 32 qh bytes; one fp32
// FMA rounds d*sc*q - dmin*m once, then one bf16 rounding.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q5_K>(const uint8_t* g, int u, uint4 (&out)[4]) {
  const float d = half_at(g);
  const float dmin = half_at(g + 2);
  int sc, m;
  k_scale_min(g + 4, u, sc, m);
  const float ds = d * (float)sc;
  const float dm = -(dmin * (float)m);
  const uint4* qp = reinterpret_cast<const uint4*>(g + 48 + 32 * (u >> 1));
  const uint4* hp = reinterpret_cast<const uint4*>(g + 16);
  const uint4 q0 = qp[0], q1 = qp[1], h0 = hp[0], h1 = hp[1];
  const uint32_t xs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  const uint32_t hs[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const uint32_t sh = (uint32_t)(u & 1) * 4u;
  const float2 dsv = make_float2(ds, ds), dmv = make_float2(dm, dm);
  const float2 bias = make_float2(-8388608.0f, -8388608.0f);  // -2^23
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[4];
    magic4(((xs[i] >> sh) & 0x0F0F0F0Fu) | (((hs[i] >> u) & 0x01010101u) << 4), f);
    const float2 a = __ffma2_rn(__fadd2_rn(make_float2(f[0], f[1]), bias), dsv, dmv);
    const float2 c = __ffma2_rn(__fadd2_rn(make_float2(f[2], f[3]), bias), dsv, dmv);
    o[2 * i] = bf16x2_bits(a.x, a.y);
    o[2 * i + 1] = bf16x2_bits(c.x, c.y);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) out[cc] = make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
}

// Q6_K unit u (32 weights 32a + l of half h = u / 4, a = u % 4): two scales (l < 16, l >= 16);
// d * scale * (q - 32) is exact in fp32, then one bf16 rounding. 2-byte aligned loads.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q6_K>(const uint8_t* g, int u, uint4 (&out)[4]) {
  const int h = u >> 2, a = u & 3;
  const float d = half_at(g + 208);
  const float ds0 = d * (float)(int8_t)g[192 + 8 * h + 2 * a];
  const float ds1 = d * (float)(int8_t)g[192 + 8 * h + 2 * a + 1];
  uint32_t lo[8], hi[8];
  load32_a2(g + 64 * h + 32 * (a & 1), lo);
  load32_a2(g + 128 + 32 * h, hi);
  const uint32_t sl = 4u * (uint32_t)(a >> 1), shh = 2u * (uint32_t)a;
  const float2 bias = make_float2(-8388640.0f, -8388640.0f);  // -(2^23 + 32)
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 dsv = i < 4 ? make_float2(ds0, ds0) : make_float2(ds1, ds1);
    float f[4];
    magic4(((lo[i] >> sl) & 0x0F0F0F0Fu) | (((hi[i] >> shh) & 0x03030303u) << 4), f);
    const float2 x = __fmul2_rn(__fadd2_rn(make_float2(f[0], f[1]), bias), dsv);
    const float2 y = __fmul2_rn(__fadd2_rn(make_float2(f[2], f[3]), bias), dsv);
    o[2 * i] = bf16x2_bits(x.x, x.y);
    o[2 * i + 1] = bf16x2_bits(y.x, y.y);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) out[cc] = make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
}

// 8 fp32 values -> 8 bf16 (round to nearest even) packed in 16 bytes.
__device__ __forceinline__ uint4 pack_bf16x8(const float (&w)[8]) {
  uint4 o;
  __nv_bfloat162 t;
  t = __floats2bfloat162_rn(w[0], w[1]);
  o.x = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(w[2], w[3]);
  o.y = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(w[4], w[5]);
  o.z = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(w[6], w[7]);
  o.w = *reinterpret_cast<uint32_t*>(&t);
  return o;
}

template <int QT>
__device__ __forceinline__ uint4 decode8_bf16(const uint8_t* g, int c) {
  float w[8];
  decode8<QT>(g, c, w);
  return pack_bf16x8(w);
}

// Q2_K unit u (weights 32u .. 32u + 31): the four 8-weight chunks of decode8, each rounded to bf16.
template <>
__device__ __forceinline__ void decode_unit_bf16<QL_Q2_K>(const uint8_t* g, int u, uint4 (&out)[4]) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    float w[8];
    decode8<QL_Q2_K>(g, 4 * u + cc, w);
    out[cc] = pack_bf16x8(w);
  }
}

}  // namespace qlora
