// mxfp8 weight rows to bf16 [mlx-lm PR #1192 "Add DeepSeek-v4 (Flash/Pro)",
// the FP8 re-quantisation thread: fp8 e4m3 weight bytes with e8m0 scales
// per 32 consecutive elements of a row, w = e4m3(byte) * 2^(e - 127)].
//
// Every such value is exact in bf16 (3 mantissa bits times a power of two),
// so the conversion is exact: e4m3 pairs widen to f16 pairs
// (cvt.rn.f16x2.e4m3x2, exact), then to fp32, are multiplied by the power
// of two (exact) and packed to bf16 (exact).  The kernel is a memory stream
// (1 + 1/32 bytes read and 2 written per element): each thread takes 8
// consecutive code bytes (one 64-bit load and their scale byte) and writes
// 16 bytes of bf16.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

constexpr int kFp8Threads = 256;

// 2^(e - 127) as fp32 (e = 0: the subnormal 2^-127; e = 255: +inf, outside
// the finite range the format stores)
MOE_DEV float e8m0_to_float(uint32_t e) { return __uint_as_float(e ? (e << 23) : 0x00400000u); }

// two e4m3 bytes (low byte first) -> two fp32 values
MOE_DEV float2 e4m3x2_to_float2(uint32_t two_bytes) {
  uint32_t h2;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n" : "=r"(h2) : "r"(two_bytes));
  const __half2 h = *reinterpret_cast<const __half2*>(&h2);
  return __half22float2(h);
}

MOE_DEV uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// 8 bytes of codes with their scale -> 16 bytes of bf16
MOE_DEV uint4 dequant8(const uint2 v, float s) {
  const float2 a = e4m3x2_to_float2(v.x & 0xFFFFu), b = e4m3x2_to_float2(v.x >> 16);
  const float2 c = e4m3x2_to_float2(v.y & 0xFFFFu), d = e4m3x2_to_float2(v.y >> 16);
  return make_uint4(pack_bf16x2(a.x * s, a.y * s), pack_bf16x2(b.x * s, b.y * s), pack_bf16x2(c.x * s, c.y * s),
                    pack_bf16x2(d.x * s, d.y * s));
}

constexpr int kFp8Unroll = 4;  // pieces a thread keeps in flight

// codes: [rows][n_in] bytes (16-byte aligned rows); scales: [rows][n_in/32];
// out: bf16 [rows][n_in].  The rows are one stream of 8-byte pieces (n_in is
// a multiple of 32, so a piece never straddles rows or groups): a warp
// instruction reads 256 contiguous code bytes and writes 512 contiguous
// output bytes, and a thread loads kFp8Unroll pieces a grid-width apart
// before converting any.
__global__ void __launch_bounds__(kFp8Threads) dequant_mxfp8_kernel(const uint8_t* __restrict__ codes,
                                                                  const uint8_t* __restrict__ scales,
                                                                  __nv_bfloat16* __restrict__ out, long long rows,
                                                                  int n_in) {
  const long long total = rows * (n_in / 8);  // pieces
  const long long stride = (long long)gridDim.x * blockDim.x;
  uint4* dst = reinterpret_cast<uint4*>(out);
  for (long long base = (long long)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * kFp8Unroll) {
    uint2 v[kFp8Unroll];
    float sc[kFp8Unroll];
#pragma unroll
    for (int u = 0; u < kFp8Unroll; ++u) {
      const long long i = base + u * stride;
      if (i < total) {
        v[u] = ldg_stream2(codes + i * 8);
        sc[u] = e8m0_to_float(__ldg(scales + i / 4));  // piece i: elements 8i..8i+7 of the stream
      }
    }
#pragma unroll
    for (int u = 0; u < kFp8Unroll; ++u) {
      const long long i = base + u * stride;
      if (i < total) __stcs(dst + i, dequant8(v[u], sc[u]));
    }
  }
}

}  // namespace moe
