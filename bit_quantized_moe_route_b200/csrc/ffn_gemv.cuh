// Step 3 of the layer for small token counts: the grouped SwiGLU expert FFN
// as a weight-streaming GEMV over packed experts.
//
//   stage 1:  h[p] = silu(W1[e] . x[t]) * (W3[e] . x[t])     (rows of d_ff)
//   stage 2:  y[p] = W2[e] . h[p]                            (rows of d_model)
//
// for every sorted position p of every active expert e (token t =
// sorted_rows[p] / k), plus the always-on shared expert at positions
// T*k + t [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": w1/w2/w3 are the
// gate/down/up projections of the switch MLP; model card
// "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit", precision table].
//
// Work decomposition: a persistent grid walks items (expert, block of rows).
// Each thread owns one 32-input chunk of a row (its x values live in
// registers for the whole item) and walks rows; partial dot products are
// reduced over the chunk owners of a row with warp shuffles and a small
// shared-memory pass.  Weights are dequantised in registers from the packed
// words: affine as s * sum(q*x) + b * sum(x) per group, mxfp4 as
// 2^(e-127) * sum(e2m1(c) * x) per 32-group [model card
// "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit", conversion notes; mlx-lm
// PR "Add DeepSeek-V4 model and safetensors/tokenizer fallback handling":
// E8M0 = 2^(b-127)].
#pragma once

#include "common.cuh"

namespace moe {



struct FfnParams {
  const __nv_bfloat16* x;  // stage 1 input [T, d]
  const float* hin;        // stage 2 input rows [P, ld_in]
  float* out;              // stage 1: h [P, ld_out]; stage 2: y [P, ld_out]
  int ld_in, ld_out;
  int T, k;
  QMatDev ra, rb;          // routed: stage 1 w1, w3; stage 2 w2
  const int* offsets;      // [E+1]
  const int* sorted_rows;  // [T*k]
  const int* active;       // [0] = n, [1..] expert ids
  int routed_items_per_expert;
  int has_shared;
  QMatDev sa, sb;
  int shared_items;
  int shared_pos0;         // = T*k
  int* err;
};

constexpr int kFfnThreads = 256;
constexpr int kFfnNT = 2;        // tokens per pass (x chunk held in registers)
constexpr int kRed = 4096;       // floats of reduction scratch


// e2m1 code -> value (sign | exponent(2) | mantissa(1), exponent bias 1).
MOE_DEV float e2m1_to_f(uint32_t c) {
  const uint32_t mag = c & 7u;
  uint32_t bits = (mag & 6u) ? ((mag + 0xFCu) << 22) : ((mag & 1u) ? 0x3F000000u : 0u);
  bits |= (c & 8u) << 28;
  return __uint_as_float(bits);
}

MOE_DEV float e8m0_to_f(uint32_t e) { return __uint_as_float(e ? (e << 23) : 0x00400000u); }

// Load the packed words of one 32-input chunk.
template <int FMT>
struct Chunk;

template <>
struct Chunk<F_A4> {
  static constexpr int kWords = 4;
  uint32_t w[4];
  MOE_DEV void load(const uint32_t* p) {
    const uint4 v = ldg_stream(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
  MOE_DEV uint32_t code(int i) const { return (w[i >> 3] >> (4 * (i & 7))) & 15u; }
};
template <>
struct Chunk<F_MX4> : Chunk<F_A4> {};
template <>
struct Chunk<F_A2> {
  static constexpr int kWords = 2;
  uint32_t w[2];
  MOE_DEV void load(const uint32_t* p) {
    const uint2 v = ldg_stream2(p);
    w[0] = v.x; w[1] = v.y;
  }
  MOE_DEV uint32_t code(int i) const { return (w[i >> 4] >> (2 * (i & 15))) & 3u; }
};
template <>
struct Chunk<F_A8> {
  static constexpr int kWords = 8;
  uint32_t w[8];
  MOE_DEV void load(const uint32_t* p) {
    const uint4 a = ldg_stream(p), b = ldg_stream(p + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
  MOE_DEV uint32_t code(int i) const { return (w[i >> 2] >> (8 * (i & 3))) & 255u; }
};
template <>
struct Chunk<F_A3> {
  static constexpr int kWords = 3;
  uint32_t w[3];
  MOE_DEV void load(const uint32_t* p) {
    w[0] = ldg_stream1(p); w[1] = ldg_stream1(p + 1); w[2] = ldg_stream1(p + 2);
  }
  MOE_DEV uint32_t code(int i) const {
    const int pos = 3 * i, wi = pos >> 5, sh = pos & 31;
    uint32_t v = w[wi] >> sh;
    if (sh > 29) v |= w[wi + 1] << (32 - sh);
    return v & 7u;
  }
};

template <int FMT>
constexpr int fmt_bits() {
  return FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
}

// acc[t] += dot(row chunk, x chunk of token t)
template <int FMT, int NT>
MOE_DEV void chunk_dot(const QMatDev& m, size_t row_abs, int c, const float (&xr)[NT][32],
                       const float (&xsum)[NT], int nt, float (&acc)[NT]) {
  Chunk<FMT> ch;
  ch.load(m.q + row_abs * (size_t)m.wpr + (size_t)c * Chunk<FMT>::kWords);
  if constexpr (FMT == F_MX4) {
    const size_t gi = row_abs * (size_t)m.gpr + c;
    const float sc = e8m0_to_f(reinterpret_cast<const uint8_t*>(m.scales)[gi]);
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = e2m1_to_f(ch.code(i));
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (t < nt) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) s = fmaf(v[i], xr[t][i], s);
        acc[t] = fmaf(sc, s, acc[t]);
      }
    }
  } else {
    const size_t gi = row_abs * (size_t)m.gpr + (size_t)(c * 32) / m.group;
    const float sc = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(m.scales)[gi]);
    const float bi = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(m.biases)[gi]);
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = magic_u2f(ch.code(i));
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (t < nt) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) s = fmaf(v[i], xr[t][i], s);
        acc[t] = fmaf(sc, s, fmaf(bi, xsum[t], acc[t]));
      }
    }
  }
}

template <int STAGE, int RPT, int FMT>
MOE_DEV void ffn_item(const FfnParams& p, float* red, const QMatDev& A, const QMatDev& B, int e,
                      int pos0, int npos, int rb, bool shared) {
  constexpr int NT = kFfnNT;
  constexpr int M = STAGE == 1 ? 2 : 1;
  constexpr int V = RPT * M * NT;
  const int tid = threadIdx.x;
  const int C = A.n_in >> 5;                 // chunks per row (<= 256)
  const int rows_par = kFfnThreads / C;
  const int c = tid % C, slot = tid / C;
  const bool act = slot < rows_par;
  const int RB = rows_par * RPT;
  const int r0 = rb * RB;
  const bool fast = C <= 32 ? ((C & (C - 1)) == 0) : (C % 32 == 0);
  const int nseg = C > 32 ? C / 32 : 1;
  const int seg = C > 32 ? (c >> 5) : 0;
  const int L = C < 32 ? C : 32;

  for (int tb = 0; tb < npos; tb += NT) {
    const int nt = min(NT, npos - tb);
    float xr[NT][32];
    float xsum[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      xsum[t] = 0.f;
      const bool live = act && t < nt;
      if constexpr (STAGE == 1) {
        int tok = 0;
        if (live) tok = shared ? (tb + t) : (p.sorted_rows[pos0 + tb + t] / p.k);
        const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)tok * A.n_in + c * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint4 u = live ? src[v4] : make_uint4(0, 0, 0, 0);
          xr[t][8 * v4 + 0] = bf16lo(u.x); xr[t][8 * v4 + 1] = bf16hi(u.x);
          xr[t][8 * v4 + 2] = bf16lo(u.y); xr[t][8 * v4 + 3] = bf16hi(u.y);
          xr[t][8 * v4 + 4] = bf16lo(u.z); xr[t][8 * v4 + 5] = bf16hi(u.z);
          xr[t][8 * v4 + 6] = bf16lo(u.w); xr[t][8 * v4 + 7] = bf16hi(u.w);
        }
      } else {
        const float4* src = reinterpret_cast<const float4*>(p.hin + (size_t)(pos0 + tb + t) * p.ld_in + c * 32);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
          const float4 u = live ? src[v4] : make_float4(0.f, 0.f, 0.f, 0.f);
          xr[t][4 * v4 + 0] = u.x; xr[t][4 * v4 + 1] = u.y;
          xr[t][4 * v4 + 2] = u.z; xr[t][4 * v4 + 3] = u.w;
        }
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) xsum[t] += xr[t][i];
    }

    float acc[RPT][M][NT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[i][m][t] = 0.f;

    if (act) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = r0 + slot + i * rows_par;
        if (r < A.n_out) {
          const size_t row_abs = (size_t)e * A.n_out + r;
          chunk_dot<FMT, NT>(A, row_abs, c, xr, xsum, nt, acc[i][0]);
          if constexpr (M == 2) chunk_dot<FMT, NT>(B, row_abs, c, xr, xsum, nt, acc[i][1]);
        }
      }
    }
    // Reduce the partial sums of the C chunk owners of each row slot.  Fast
    // path (C a power of two <= 32, or a multiple of 32): warp shuffles over
    // the lanes of a slot, then one partial per warp segment in shared memory.
    // Otherwise every thread parks its partials in shared memory.
    if (fast) {
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            float v = acc[i][m][t];
            for (int o = L >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[i][m][t] = v;
          }
    }
    if (act && (!fast || (c & 31) == 0)) {
      float* dst = red + (fast ? ((size_t)slot * nseg + seg) : (size_t)tid) * V;
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
          for (int t = 0; t < NT; ++t) dst[(i * M + m) * NT + t] = acc[i][m][t];
    }
    __syncthreads();
    // finalise: the threads of a slot stride over the (row i, token t) pairs
    for (int v = c; act && v < RPT * NT; v += C) {
      const int i = v / NT, t = v % NT;
      const int r = r0 + slot + i * rows_par;
      if (r < A.n_out && t < nt) {
        float g = 0.f, u = 0.f;
        const int nsum = fast ? nseg : C;
        for (int s = 0; s < nsum; ++s) {
          const float* src = red + (fast ? ((size_t)slot * nseg + s) : ((size_t)slot * C + s)) * V;
          g += src[(i * M + 0) * NT + t];
          if constexpr (M == 2) u += src[(i * M + 1) * NT + t];
        }
        const int prow = pos0 + tb + t;
        if constexpr (STAGE == 1) {
          p.out[(size_t)prow * p.ld_out + r] = silu(g) * u;
        } else {
          p.out[(size_t)prow * p.ld_out + r] = g;
        }
      }
    }
    __syncthreads();
  }
}

template <int STAGE, int RPT>
__global__ void __launch_bounds__(kFfnThreads)
ffn_gemv_kernel(const FfnParams p) {
  __shared__ float red[kRed];
  const int n_active = p.active[0];
  const int n_routed = n_active * p.routed_items_per_expert;
  const int total = n_routed + (p.has_shared ? p.shared_items : 0);
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    const bool shared = item >= n_routed;
    int e, pos0, npos, rb;
    const QMatDev* A;
    const QMatDev* B;
    if (!shared) {
      const int a = item / p.routed_items_per_expert;
      rb = item - a * p.routed_items_per_expert;
      e = p.active[1 + a];
      pos0 = p.offsets[e];
      npos = p.offsets[e + 1] - pos0;
      A = &p.ra;
      B = &p.rb;
    } else {
      rb = item - n_routed;
      e = 0;
      pos0 = p.shared_pos0;
      npos = p.T;
      A = &p.sa;
      B = &p.sb;
    }
    switch (A->fmt) {
      case F_A2: ffn_item<STAGE, RPT, F_A2>(p, red, *A, *B, e, pos0, npos, rb, shared); break;
      case F_A3: ffn_item<STAGE, RPT, F_A3>(p, red, *A, *B, e, pos0, npos, rb, shared); break;
      case F_A4: ffn_item<STAGE, RPT, F_A4>(p, red, *A, *B, e, pos0, npos, rb, shared); break;
      case F_A8: ffn_item<STAGE, RPT, F_A8>(p, red, *A, *B, e, pos0, npos, rb, shared); break;
      default:   ffn_item<STAGE, RPT, F_MX4>(p, red, *A, *B, e, pos0, npos, rb, shared); break;
    }
  }
}

// ---------------------------------------------------------------------------
// Step 4: out[t] = bf16( sum_j w[t,j] * y[inv[t*k+j]] + y_shared[t] )
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ y, const int* __restrict__ inv, const float* __restrict__ w,
               const float* __restrict__ y_shared, __nv_bfloat16* __restrict__ out, int T, int k, int d) {
  pdl_wait();  // y comes from the kernel before (possibly launched programmatically)
  const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
  if (c4 * 4 >= d) return;
  // tokens stride over gridDim.y (at most 65535 rows of blocks per launch)
  for (int t = blockIdx.y; t < T; t += gridDim.y) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int pidx = inv[(size_t)t * k + j];
      const float wt = w[(size_t)t * k + j];
      const float4 v = reinterpret_cast<const float4*>(y + (size_t)pidx * d)[c4];
      acc.x = fmaf(wt, v.x, acc.x);
      acc.y = fmaf(wt, v.y, acc.y);
      acc.z = fmaf(wt, v.z, acc.z);
      acc.w = fmaf(wt, v.w, acc.w);
    }
    if (y_shared) {
      const float4 v = reinterpret_cast<const float4*>(y_shared + (size_t)t * d)[c4];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(out + (size_t)t * d)[c4] = pk;
  }
}

}  // namespace moe
