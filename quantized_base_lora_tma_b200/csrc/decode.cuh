// GGUF block decode on the device: 8 consecutive weights of one 256-weight group of a packed row.
//
// A "group" is the packed bytes of 256 consecutive weights of one row: 8 Q8_0 blocks (272 B),
// 8 Q4_0 blocks (144 B) or one Q4_K superblock (144 B). Groups are the unit every kernel here
// moves: their byte size is a multiple of 16, so they can be copied by TMA and rows of K % 256 == 0
// weights start 16-byte aligned.
//
// Values are the exact decode rounded once to fp32 (each product below is exact in fp32; the Q4_K
// difference is formed by one fused multiply-add, i.e. one rounding), which a caller then rounds
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

}  // namespace qlora
