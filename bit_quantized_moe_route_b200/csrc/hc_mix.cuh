// mHC residual mixing (manifold-constrained hyper-connections): the residual
// stream carries n = hc_mult parallel copies h[t, 0..n-1, :] of the hidden
// state, recombined by a per-token doubly-stochastic matrix P obtained by
// Sinkhorn normalisation of mixing logits.
//
// [model card "mlx-community / DeepSeek-V4-Flash-4bit", Architecture, mHC:
//  hc_mult = 4 copies mixed through a Sinkhorn-normalised, doubly-stochastic
//  matrix; mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)", review note "Sinkhorn
//  normalization": a softmax then sum-and-divide iterations, which the fused
//  kernel does in one register-resident pass.]
//
//   P  = softmax of each row of the logits L[t] (n x n)
//   repeat iters times:  divide every column of P by its sum (+ eps),
//                        then every row by its sum (+ eps)
//   out[t, i, :] = sum_j P[i, j] * h[t, j, :]      (fp32, one bf16 rounding)
//
// One launch: per token, one warp normalises the n x n matrix in shared
// memory (n <= 8: two entries per lane) while the block's other threads
// already hold their slices of the n copies in registers; then every thread
// mixes its 8-element slices (16-byte loads and stores).  Bound: HBM, 2*n*d*2
// bytes per token.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kHcMaxN = 8;
constexpr int kHcThreads = 256;
constexpr int kHcSlices = 2;  // 8-element slices per thread held in registers (d <= 256*8*2 in one pass)

MOE_DEV void hc_normalise_warp(float* Ps, const float* __restrict__ logits, float* __restrict__ P_out, int n,
                               int iters, float eps) {
  const int lane = threadIdx.x & 31;
  const int nn = n * n;
  float v[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    v[r] = e < nn ? __ldg(logits + e) : 0.f;
    if (e < nn) Ps[e] = v[r];
  }
  __syncwarp();
  // row-wise softmax
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    if (e < nn) {
      const int i = e / n;
      float m = -INFINITY;
      for (int j = 0; j < n; ++j) m = fmaxf(m, Ps[i * n + j]);
      v[r] = expf(v[r] - m);
    }
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 2; ++r)
    if (lane + 32 * r < nn) Ps[lane + 32 * r] = v[r];
  __syncwarp();
  auto row_norm = [&](float add_eps) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = lane + 32 * r;
      if (e < nn) {
        const int i = e / n;
        float s = 0.f;
        for (int j = 0; j < n; ++j) s += Ps[i * n + j];
        v[r] = v[r] / (s + add_eps);
      }
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 2; ++r)
      if (lane + 32 * r < nn) Ps[lane + 32 * r] = v[r];
    __syncwarp();
  };
  row_norm(0.f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = lane + 32 * r;
      if (e < nn) {
        const int j = e % n;
        float s = 0.f;
        for (int i = 0; i < n; ++i) s += Ps[i * n + j];
        v[r] = v[r] / (s + eps);
      }
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 2; ++r)
      if (lane + 32 * r < nn) Ps[lane + 32 * r] = v[r];
    __syncwarp();
    row_norm(eps);
  }
  if (P_out) {
#pragma unroll
    for (int r = 0; r < 2; ++r)
      if (lane + 32 * r < nn) P_out[lane + 32 * r] = v[r];
  }
}

// grid: tokens (grid-stride); block: kHcThreads.  d % 8 == 0,
// d <= kHcThreads * 8 * kHcSlices per pass (larger d loops over passes).
template <int N>
__global__ void __launch_bounds__(kHcThreads)
hc_sinkhorn_mix_kernel(const float* __restrict__ logits, const __nv_bfloat16* __restrict__ h,
                       float* __restrict__ P_out, __nv_bfloat16* __restrict__ out, int T, int n, int d, int iters,
                       float eps) {
  __shared__ float Ps[kHcMaxN * kHcMaxN];
  const int warp = threadIdx.x >> 5;
  const int c8 = d / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const size_t tok_base = (size_t)t * N * d;
    for (int c0 = 0; c0 < c8; c0 += kHcThreads * kHcSlices) {
      // this thread's slices of the N copies, loaded before P is known
      uint4 hv[kHcSlices][N];
#pragma unroll
      for (int sl = 0; sl < kHcSlices; ++sl) {
        const int c = c0 + sl * kHcThreads + threadIdx.x;
#pragma unroll
        for (int j = 0; j < N; ++j)
          hv[sl][j] = c < c8 ? __ldcs(reinterpret_cast<const uint4*>(h + tok_base + (size_t)j * d) + c)
                             : make_uint4(0, 0, 0, 0);
      }
      if (c0 == 0 && warp == 0)
        hc_normalise_warp(Ps, logits + (size_t)t * N * N, P_out ? P_out + (size_t)t * N * N : nullptr, N, iters,
                          eps);
      __syncthreads();
      float P[N][N];
#pragma unroll
      for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) P[i][j] = Ps[i * N + j];
#pragma unroll
      for (int sl = 0; sl < kHcSlices; ++sl) {
        const int c = c0 + sl * kHcThreads + threadIdx.x;
        if (c >= c8) continue;
        float x[N][8];
#pragma unroll
        for (int j = 0; j < N; ++j) {
          const uint32_t w[4] = {hv[sl][j].x, hv[sl][j].y, hv[sl][j].z, hv[sl][j].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            x[j][2 * q] = bf16lo(w[q]);
            x[j][2 * q + 1] = bf16hi(w[q]);
          }
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int j = 0; j < N; ++j) {
              a = fmaf(P[i][j], x[j][2 * q], a);
              b = fmaf(P[i][j], x[j][2 * q + 1], b);
            }
            const __nv_bfloat162 r = __floats2bfloat162_rn(a, b);
            o[q] = *reinterpret_cast<const uint32_t*>(&r);
          }
          __stcs(reinterpret_cast<uint4*>(out + tok_base + (size_t)i * d) + c, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      if (c0 + kHcThreads * kHcSlices >= c8) __syncthreads();  // Ps is rewritten by the next token
    }
  }
}

}  // namespace moe
