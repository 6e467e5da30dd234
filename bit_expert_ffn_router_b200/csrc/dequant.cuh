// Dot products of packed 2/3-bit rows with an activation vector on the CUDA
// cores, using 2-way integer dot products (dp2a: two signed 16-bit values
// times two unsigned bytes, accumulated in int32).
//
// Activations (x for gate/up, h for down) are cut into blocks of 32 values,
// the blocks the weight scales use, and each block is requantised once per
// CTA to int16 against its own largest magnitude m:
//   xq_i = rint(x_i * 32767 / m),   x_i ~= sx * xq_i,   sx = m / 32767,
// an error of at most m / 65534 per value. A weight block then contributes
//   s_w * sx * (sum_i q_i * xq_i - 2^(b-1) * sum_i xq_i)
// where the integer sums are exact (|sum| < 2^23), so the block term is the
// only rounding; blocks are added in ascending order in fp32.
//
// Codes reach dp2a without per-code unpacking: (w >> 2s) & 0x03030303 puts
// codes s, s+4, s+8, s+12 of a 16-code word into the four bytes of a word,
// and the activations are stored as the matching int16 pairs. The high bits
// of 3-bit codes (one 32-bit word per block, bit c = code c) go the same way
// with (h >> t) & 0x01010101 (codes t, t+8, t+16, t+24).
//
// Every sum is exact or runs in a fixed order, so a token's result does not
// depend on the other tokens in the batch or on how rows are split.
#pragma once

#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ int dp2a_lo(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int dp2a_hi(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ------------------------------------------------------------------ quantised vectors in shared memory
// A vector of nb blocks is stored for a row-dot geometry of `lpr` lanes per
// row and `bpl` blocks per lane: block b = gl*bpl + bb sits in column
// col = bb*lpr + gl, so the lanes of a warp read consecutive words.
//   word (k*nb + col),      k = 0..15 : 2-bit-plane pairs
//   word ((16+k)*nb + col), k = 0..15 : high-plane pairs (3-bit only)
//   word (kSX*nb + col)               : sx (float bits)
//   word ((kSX+1)*nb + col)           : sum of xq
template <int BITS>
struct QV {
  static constexpr int kSX = BITS == 3 ? 32 : 16;
  static constexpr int kWords = kSX + 2;  // words per block
};

// Requantises 32 fp32 values into block column `col` of a QV vector.
// rint(v * inv) comes from one FMA with 1.5 * 2^23: the integer then sits in
// the low 22 bits of the float's bit pattern, whose low 16 bits are exactly
// the int16 two's-complement value dp2a wants.
template <int BITS>
__device__ __forceinline__ void quant_block(const float* v, int* vec, int nb, int col) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  const float inv = m > 0.f ? 32767.f / m : 0.f;
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  int r[32];
  unsigned usum = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    r[i] = __float_as_int(fmaf(v[i], inv, kMagic));
    usum += static_cast<unsigned>(r[i]);
  }
  // modulo 2^32 this is the true sum of the integers, |sum| < 2^21
  const int sum = static_cast<int>(usum - 32u * 0x4B400000u);
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      vec[(8 * j + s) * nb + col] = static_cast<int>(__byte_perm(r[16 * j + s], r[16 * j + s + 4], 0x5410));
      vec[(8 * j + 4 + s) * nb + col] = static_cast<int>(__byte_perm(r[16 * j + s + 8], r[16 * j + s + 12], 0x5410));
    }
  if (BITS == 3) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      vec[(16 + t) * nb + col] = static_cast<int>(__byte_perm(r[t], r[t + 8], 0x5410));
      vec[(24 + t) * nb + col] = static_cast<int>(__byte_perm(r[t + 16], r[t + 24], 0x5410));
    }
  }
  vec[QV<BITS>::kSX * nb + col] = __float_as_int(m * (1.f / 32767.f));
  vec[(QV<BITS>::kSX + 1) * nb + col] = sum;
}

// The same, spread over an aligned group of 4 lanes: lane q of the group
// holds v[k] = block value q + 4k (k = 0..7). Every int16 pair a lane stores
// is made of its own values; the block max and sum come from 2 shuffles.
// All 32 lanes of the warp must call it (dummy groups pass zeros).
template <int BITS>
__device__ __forceinline__ void quant_quad(const float* v, int* vec, int nb, int col, int q, bool store) {
  float m = fmaxf(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))),
                  fmaxf(fmaxf(fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7]))));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const float inv = m > 0.f ? 32767.f / m : 0.f;
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  int r[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) r[k] = __float_as_int(fmaf(v[k], inv, kMagic));
  unsigned us = (static_cast<unsigned>(r[0]) + static_cast<unsigned>(r[1])) +
                (static_cast<unsigned>(r[2]) + static_cast<unsigned>(r[3])) +
                ((static_cast<unsigned>(r[4]) + static_cast<unsigned>(r[5])) +
                 (static_cast<unsigned>(r[6]) + static_cast<unsigned>(r[7])));
  us += __shfl_xor_sync(0xffffffffu, us, 1);
  us += __shfl_xor_sync(0xffffffffu, us, 2);
  if (!store) return;
  // words j = 0, 1: values (16j+q, 16j+q+4) and (16j+q+8, 16j+q+12)
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    vec[(8 * j + q) * nb + col] = static_cast<int>(__byte_perm(r[4 * j], r[4 * j + 1], 0x5410));
    vec[(8 * j + 4 + q) * nb + col] = static_cast<int>(__byte_perm(r[4 * j + 2], r[4 * j + 3], 0x5410));
  }
  if (BITS == 3) {  // high-plane pairs (t, t+8), (t+16, t+24) for t = q, q+4
    vec[(16 + q) * nb + col] = static_cast<int>(__byte_perm(r[0], r[2], 0x5410));
    vec[(16 + q + 4) * nb + col] = static_cast<int>(__byte_perm(r[1], r[3], 0x5410));
    vec[(24 + q) * nb + col] = static_cast<int>(__byte_perm(r[4], r[6], 0x5410));
    vec[(24 + q + 4) * nb + col] = static_cast<int>(__byte_perm(r[5], r[7], 0x5410));
  }
  if (q == 0) {
    vec[QV<BITS>::kSX * nb + col] = __float_as_int(m * (1.f / 32767.f));
    vec[(QV<BITS>::kSX + 1) * nb + col] = static_cast<int>(us - 32u * 0x4B400000u);
  }
}

// 2-bit layout only: the same block quantisation as quant_quad, for a thread
// q of the block's four that holds the eight consecutive values 8q .. 8q+7
// (two 16-byte loads instead of eight strided ones). Word 8(q/2) + 4(q%2) + i
// of the block is the pair (8q + i, 8q + i + 4), exactly the words
// quant_quad writes for those values.
__device__ __forceinline__ void quant_quad_c2(const float* v, int* vec, int nb, int col, int q, bool store) {
  float m = fmaxf(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))),
                  fmaxf(fmaxf(fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7]))));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const float inv = m > 0.f ? 32767.f / m : 0.f;
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  int r[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) r[k] = __float_as_int(fmaf(v[k], inv, kMagic));
  unsigned us = (static_cast<unsigned>(r[0]) + static_cast<unsigned>(r[1])) +
                (static_cast<unsigned>(r[2]) + static_cast<unsigned>(r[3])) +
                ((static_cast<unsigned>(r[4]) + static_cast<unsigned>(r[5])) +
                 (static_cast<unsigned>(r[6]) + static_cast<unsigned>(r[7])));
  us += __shfl_xor_sync(0xffffffffu, us, 1);
  us += __shfl_xor_sync(0xffffffffu, us, 2);
  if (!store) return;
  const int w0 = 8 * (q >> 1) + 4 * (q & 1);
#pragma unroll
  for (int i = 0; i < 4; ++i) vec[(w0 + i) * nb + col] = static_cast<int>(__byte_perm(r[i], r[i + 4], 0x5410));
  if (q == 0) {
    vec[QV<2>::kSX * nb + col] = __float_as_int(m * (1.f / 32767.f));
    vec[(QV<2>::kSX + 1) * nb + col] = static_cast<int>(us - 32u * 0x4B400000u);
  }
}

// One block of a quantised vector, in registers.
template <int BITS>
struct XR {
  int p[16];
  int ph[BITS == 3 ? 16 : 1];
  float sx;
  int sum;
};

template <int BITS, int BPL>
__device__ __forceinline__ void load_xr(const int* __restrict__ vec, int nb, int lpr, int gl, XR<BITS>* xr) {
#pragma unroll
  for (int bb = 0; bb < BPL; ++bb) {
    const int col = bb * lpr + gl;
#pragma unroll
    for (int k = 0; k < 16; ++k) xr[bb].p[k] = vec[k * nb + col];
    if (BITS == 3) {
#pragma unroll
      for (int k = 0; k < 16; ++k) xr[bb].ph[k] = vec[(16 + k) * nb + col];
    }
    xr[bb].sx = __int_as_float(vec[QV<BITS>::kSX * nb + col]);
    xr[bb].sum = vec[(QV<BITS>::kSX + 1) * nb + col];
  }
}

// sum_i (q_i - 2^(bits-1)) * xq_i over one block: w0, w1 are the block's two
// 2-bit-plane words, h its high-plane word (3-bit only).
// Four independent partial sums keep the dependent dp2a chains short.
template <int BITS>
__device__ __forceinline__ int block_dot(uint32_t w0, uint32_t w1, uint32_t h, const XR<BITS>& q) {
  int a[4] = {0, 0, 0, 0};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint32_t b0 = (w0 >> (2 * s)) & 0x03030303u;
    const uint32_t b1 = (w1 >> (2 * s)) & 0x03030303u;
    a[s] = dp2a_lo(q.p[s], b0, a[s]);
    a[s] = dp2a_hi(q.p[4 + s], b0, a[s]);
    a[s] = dp2a_lo(q.p[8 + s], b1, a[s]);
    a[s] = dp2a_hi(q.p[12 + s], b1, a[s]);
  }
  int acc = (a[0] + a[1]) + (a[2] + a[3]);
  if (BITS == 3) {
    int hi[2] = {0, 0};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t bh = (h >> t) & 0x01010101u;
      hi[t & 1] = dp2a_lo(q.ph[t], bh, hi[t & 1]);
      hi[t & 1] = dp2a_hi(q.ph[8 + t], bh, hi[t & 1]);
    }
    acc += 4 * (hi[0] + hi[1]);
  }
  return acc - (1 << (BITS - 1)) * q.sum;
}

template <int BPL>
__device__ __forceinline__ void load_words(const uint8_t* __restrict__ codes, int gl, uint32_t* w) {
  if (BPL % 2 == 0) {
    const uint4* q = reinterpret_cast<const uint4*>(codes) + gl * (BPL / 2);
#pragma unroll
    for (int i = 0; i < BPL / 2; ++i) {
      const uint4 t = q[i];
      w[4 * i] = t.x;
      w[4 * i + 1] = t.y;
      w[4 * i + 2] = t.z;
      w[4 * i + 3] = t.w;
    }
  } else {
    const uint2* q = reinterpret_cast<const uint2*>(codes) + gl * BPL;
#pragma unroll
    for (int i = 0; i < BPL; ++i) {
      const uint2 t = q[i];
      w[2 * i] = t.x;
      w[2 * i + 1] = t.y;
    }
  }
}

// Dot product of the lane's BPL blocks of one packed row (codes and fp16
// scales in shared memory) with the lane's quantised activation blocks.
template <int BITS, int BPL>
__device__ __forceinline__ float row_dot(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                                         int K, int gl, const XR<BITS>* xr) {
  uint32_t w[2 * BPL];
  load_words<BPL>(codes, gl, w);
  float total = 0.f;
#pragma unroll
  for (int b = 0; b < BPL; ++b) {
    const uint32_t h = BITS == 3 ? reinterpret_cast<const uint32_t*>(codes + K / 4)[gl * BPL + b] : 0u;
    const int d = block_dot<BITS>(w[2 * b], w[2 * b + 1], h, xr[b]);
    const float s = __half2float(__ushort_as_half(scales[gl * BPL + b]));
    total = fmaf(static_cast<float>(d), s * xr[b].sx, total);
  }
  return total;
}

// Two rows (gate and up of one channel) against the same activation blocks.
template <int BITS, int BPL>
__device__ __forceinline__ float2 row_dot2(const uint8_t* __restrict__ c0, const uint16_t* __restrict__ s0,
                                           const uint8_t* __restrict__ c1, const uint16_t* __restrict__ s1,
                                           int K, int gl, const XR<BITS>* xr) {
  uint32_t w0[2 * BPL], w1[2 * BPL];
  load_words<BPL>(c0, gl, w0);
  load_words<BPL>(c1, gl, w1);
  float g = 0.f, u = 0.f;
#pragma unroll
  for (int b = 0; b < BPL; ++b) {
    const uint32_t h0 = BITS == 3 ? reinterpret_cast<const uint32_t*>(c0 + K / 4)[gl * BPL + b] : 0u;
    const uint32_t h1 = BITS == 3 ? reinterpret_cast<const uint32_t*>(c1 + K / 4)[gl * BPL + b] : 0u;
    const int dg = block_dot<BITS>(w0[2 * b], w0[2 * b + 1], h0, xr[b]);
    const int du = block_dot<BITS>(w1[2 * b], w1[2 * b + 1], h1, xr[b]);
    g = fmaf(static_cast<float>(dg), __half2float(__ushort_as_half(s0[gl * BPL + b])) * xr[b].sx, g);
    u = fmaf(static_cast<float>(du), __half2float(__ushort_as_half(s1[gl * BPL + b])) * xr[b].sx, u);
  }
  return make_float2(g, u);
}

}  // namespace moe
