// Preparation kernels of the tensor-core expert FFN: the fp16 copy of the
// token activations and the token-tile plan (one entry per <=128-token
// slice of each expert's sorted positions).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "ffn_tc.cuh"

namespace moe {

// x (bf16) -> x16 (fp16), 8 elements per thread per step; |x| > 65504 is
// flagged (fp16 overflow) and stored as inf.
__global__ void tc_x_to_f16_kernel(const __nv_bfloat16* __restrict__ x, __half* __restrict__ x16, size_t n8,
                                   int* __restrict__ err) {
  bool bad = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = bf16lo(in[j]), b = bf16hi(in[j]);
      bad |= !(fabsf(a) <= kF16Max) || !(fabsf(b) <= kF16Max);
      __half2 h = __floats2half2_rn(a, b);
      out[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(x16)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) set_error(err, kErrDeviceInput);
}

// Token tiles from the per-expert position ranges: expert e with n_e sorted
// positions gets ceil(n_e / 128) tiles {e, first position, tokens, 0}, in
// expert order.  One block of 1024 threads; E <= 1024.
__global__ void tc_plan_kernel(const int* __restrict__ offsets, int E, int4* __restrict__ tiles,
                               int* __restrict__ n_tiles) {
  __shared__ int warp_tot[32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int beg = e < E ? offsets[e] : 0;
  const int n = e < E ? offsets[e + 1] - beg : 0;
  const int c = (n + kTcN - 1) / kTcN;
  int incl = c;  // inclusive scan of tile counts across the block
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += v;
    }
    warp_tot[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  const int first = incl - c + (warp ? warp_tot[warp - 1] : 0);
  for (int i = 0; i < c; ++i) tiles[first + i] = make_int4(e, beg + i * kTcN, min(kTcN, n - i * kTcN), 0);
  if (e == blockDim.x - 1) *n_tiles = first + c;
}

}  // namespace moe
