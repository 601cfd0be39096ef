// Preparation kernels of the tensor-core expert FFN: the fp16 token rows in
// position order and the token-tile plans (one entry per slice of at most
// `tile` positions of each expert's sorted range).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "ffn_tc.cuh"

namespace moe {

// xs[p] = fp16(x[token of position p]) for the Tk routed positions (token =
// sorted_rows[p] / k), then xs[Tk + t] = fp16(x[t]) for the shared expert
// when `shared` is set.  8 elements per thread per step; |x| > 65504 is
// flagged (fp16 overflow) and stored as inf.
__global__ void tc_gather_f16_kernel(const __nv_bfloat16* __restrict__ x, const int* __restrict__ sorted_rows,
                                     int k, int Tk, int T, int d, int shared, __half* __restrict__ xs,
                                     int* __restrict__ err, const int* __restrict__ valid) {
  if (valid && !*valid) return;  // a caller permutation that failed its check: no expert runs
  const int c8 = d / 8;
  const size_t rows = (size_t)Tk + (shared ? T : 0);
  const size_t n8 = rows * c8;
  bool bad = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const size_t p = i / c8;
    const int c = (int)(i - p * c8);
    const int tok = p < (size_t)Tk ? __ldg(sorted_rows + p) / k : (int)(p - Tk);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)tok * d) + c);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = bf16lo(in[j]), b = bf16hi(in[j]);
      bad |= !(fabsf(a) <= kF16Max) || !(fabsf(b) <= kF16Max);
      __half2 h = __floats2half2_rn(a, b);
      out[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(xs)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) set_error(err, kErrDeviceInput);
}

// Token tiles from the per-expert position ranges, for two tile sizes at
// once: expert e with n_e sorted positions gets ceil(n_e / size) tiles
// {e, first position, tokens, 0}, in expert order.  One block of 1024
// threads; E <= 1024.  With `valid` given and zero (a caller permutation
// that failed its check) the plans are empty.
__global__ void tc_plan_kernel(const int* __restrict__ offsets, int E, int size_a, int4* __restrict__ tiles_a,
                               int* __restrict__ n_a, int size_b, int4* __restrict__ tiles_b,
                               int* __restrict__ n_b, const int* __restrict__ valid) {
  __shared__ int warp_tot[2][32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const bool ok = !valid || *valid;
  const int beg = e < E && ok ? offsets[e] : 0;
  const int n = e < E && ok ? offsets[e + 1] - beg : 0;
  const int c[2] = {(n + size_a - 1) / size_a, (n + size_b - 1) / size_b};
  int incl[2] = {c[0], c[1]};  // inclusive scans of the tile counts across the block
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int v = __shfl_up_sync(0xffffffffu, incl[t], o);
      if (lane >= o) incl[t] += v;
    }
  }
  if (lane == 31) {
    warp_tot[0][warp] = incl[0];
    warp_tot[1][warp] = incl[1];
  }
  __syncthreads();
  if (warp < 2) {
    int t = warp_tot[warp][lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += v;
    }
    warp_tot[warp][lane] = t;  // inclusive over warps
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int size = t ? size_b : size_a;
    int4* tiles = t ? tiles_b : tiles_a;
    const int first = incl[t] - c[t] + (warp ? warp_tot[t][warp - 1] : 0);
    for (int i = 0; i < c[t]; ++i) tiles[first + i] = make_int4(e, beg + i * size, min(size, n - i * size), 0);
    if (e == blockDim.x - 1) *(t ? n_b : n_a) = first + c[t];
  }
}

}  // namespace moe
