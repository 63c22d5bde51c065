// NVFP4 x NVFP4 warp dot products for the decode (GEMV) path.
//
// A warp computes dot products of 8*RP weight rows with NT activation rows.  Lanes split
// K into 16-byte chunks (32 codes, two 16-element blocks): L lanes per row, RP = 32/L rows
// per pass, lane (s, cl) = (lane / L, lane % L) takes chunks cl, cl+L, ... of row
// row0 + q*RP + s for q = 0..7.  Every weight load is a 128-bit load and a warp's loads
// of one row are contiguous.  Block sums are exact: codes are widened to f16 with the
// hardware cvt, eight products of two E2M1 values (each a multiple of 1/4 with magnitude
// <= 36) are accumulated per f16 half, which stays exact below 2048/4, and the two halves
// are added in fp32.  Each exact block sum is multiplied by the product of the two block
// scales and accumulated in fp32; the partial sums of the L lanes of a row are then
// combined with a shuffle butterfly.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace nvfp4moe {

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_u16(const uint8_t* p) {
  return static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p)));
}

// 16 bytes of codes -> 16 f16x2 (elements 2i, 2i+1 in f[i]).
__device__ __forceinline__ void decode_chunk(const uint4& v, uint32_t f[16]) {
  f16x2x4_from_e2m1x8(v.x, f + 0);
  f16x2x4_from_e2m1x8(v.y, f + 4);
  f16x2x4_from_e2m1x8(v.z, f + 8);
  f16x2x4_from_e2m1x8(v.w, f + 12);
}

// Two E4M3 scales (low 16 bits) -> two fp32.
__device__ __forceinline__ float2 decode_sf2(uint32_t s) {
  const uint32_t h2 = f16x2_from_e4m3x2(s);
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Exact sums of the two blocks of a chunk, scaled by the block scale products.
__device__ __forceinline__ float chunk_dot(const uint32_t w[16], const uint32_t x[16], float s0,
                                           float s1) {
  __half2 a0 = __float2half2_rn(0.0f), a1 = __float2half2_rn(0.0f);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    a0 = __hfma2(*reinterpret_cast<const __half2*>(&w[i]), *reinterpret_cast<const __half2*>(&x[i]), a0);
#pragma unroll
  for (int i = 8; i < 16; ++i)
    a1 = __hfma2(*reinterpret_cast<const __half2*>(&w[i]), *reinterpret_cast<const __half2*>(&x[i]), a1);
  const float2 f0 = __half22float2(a0), f1 = __half22float2(a1);
  return __fmaf_rn(f1.x + f1.y, s1, (f0.x + f0.y) * s0);
}

// tot[q][t] = sum over K of W[row(q)] . A[arow[t]] (block scales applied, tensor scales
// not), for row(q) = row0 + q*RP + lane/L.  The result is valid on every lane of the
// row's lane group.  Rows >= nrows contribute zero and are never read.
// Only chunks in [c_begin, c_end) are summed (split-K); pass 0, K/32 for the whole row.
template <int L, int NT>
__device__ __forceinline__ void warp_dot8(const uint8_t* __restrict__ wc, const uint8_t* __restrict__ wsf,
                                          int64_t row0, int64_t nrows, const uint8_t* __restrict__ ac,
                                          const uint8_t* __restrict__ asf, const int64_t arow[NT],
                                          int64_t K, int64_t c_begin, int64_t c_end, float tot[8][NT]) {
  constexpr int RP = 32 / L;
  const int lane = threadIdx.x & 31;
  const int s = lane / L, cl = lane % L;
  const int64_t rb = K / 2;
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int t = 0; t < NT; ++t) tot[q][t] = 0.0f;
  for (int64_t c = c_begin + cl; c < c_end; c += L) {
    uint4 wv[8];
    uint32_t ws[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int64_t r = row0 + q * RP + s;
      if (r < nrows) {
        wv[q] = ldg_stream16(wc + r * rb + c * 16);
        ws[q] = ldg_u16(wsf + sf_mma_offset(r, 2 * c, K));
      } else {
        wv[q] = make_uint4(0, 0, 0, 0);
        ws[q] = 0;
      }
    }
    uint32_t xf[NT][16];
    float2 xs[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(ac + arow[t] * rb + c * 16));
      decode_chunk(xv, xf[t]);
      xs[t] = decode_sf2(ldg_u16(asf + sf_mma_offset(arow[t], 2 * c, K)));
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t wf[16];
      decode_chunk(wv[q], wf);
      const float2 wsc = decode_sf2(ws[q]);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        tot[q][t] += chunk_dot(wf, xf[t], wsc.x * xs[t].x, wsc.y * xs[t].y);
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) tot[q][t] += __shfl_xor_sync(0xffffffffu, tot[q][t], o);
}

// bf16 halves of a 32-bit word (element 2i in the low half) as fp32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// c + w.lo * x.lo, then + w.hi * x.hi: two fused multiply-adds whose f16 (or bf16) operands are
// multiplied exactly and added in fp32 with one rounding each (the mixed-precision fma of sm_100)
__device__ __forceinline__ float fma2_f16_f32(uint32_t w, uint32_t x, float c) {
  asm("{\n .reg .f16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %0, wh, xh, %0;\n}"
      : "+f"(c)
      : "r"(w), "r"(x));
  return c;
}
__device__ __forceinline__ float fma2_bf16_f32(uint32_t w, uint32_t x, float c) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.bf16 %0, wl, xl, %0;\n fma.rn.f32.bf16 %0, wh, xh, %0;\n}"
      : "+f"(c)
      : "r"(w), "r"(x));
  return c;
}

}  // namespace nvfp4moe
