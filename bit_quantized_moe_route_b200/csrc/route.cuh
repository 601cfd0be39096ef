// Step 1 of the layer: routing.
//
// learned: fp32 logits L = x . Wr^T, s = sqrt(logaddexp(L, 0)), top-k of the
//   keys s + bias (ties to the lower expert id), w = s[ids] / sum(s[ids])
//   [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": gate dtype row of the
//   cross-reference table, sqrtsoftplus stability note; model card
//   "mlx-community / DeepSeek-V4-Flash-4bit", Architecture; model card
//   "DeepSeek-V4-Flash-MLX-4bit", REAP-pruned builds: renormalise over the
//   kept experts].
// hash: ids = tid2eid[token_id] in table order; weights = renormalised
//   sqrtsoftplus of the fp32 logits of those experts, or 1/k without a
//   router [model card "mlx-community / DeepSeek-V4-Flash-4bit",
//   Architecture: "Hash-routed MoE"; model card "DeepSeek-V4-Flash-MLX-4bit",
//   "What this port implements": tid2eid keyed on token id].
#pragma once

#include "common.cuh"
#include "permute.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits for small T: one warp per (expert, token batch).  The batch of x
// rows sits in shared memory as bf16; each warp streams one router row with
// 128-bit loads.
// ---------------------------------------------------------------------------
constexpr int kLogitWarps = 4;

// Router weight rows are fp32 or bf16 (the checkpoints store the gate in
// bf16 [model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit",
// precision table]); either way the logits are fp32 dot products [mlx-lm PR
// "Add DeepSeek-v4 (Flash/Pro)", table row "MoE gate dtype"].  ldw4 returns
// elements 4*i4 .. 4*i4+3 of a row as floats (bf16 widens exactly).
MOE_DEV float4 ldw4(const float* __restrict__ W, size_t i4) { return __ldg(reinterpret_cast<const float4*>(W) + i4); }
MOE_DEV float4 ldw4(const __nv_bfloat16* __restrict__ W, size_t i4) {
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(W) + i4);
  return make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
}

template <int NTB, typename WT>
__global__ void __launch_bounds__(kLogitWarps * 32)
router_logits_small_kernel(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                           float* __restrict__ L, int T, int d, int E) {
  extern __shared__ __align__(16) uint32_t xs_raw[];
  const int t0 = blockIdx.y * NTB;
  const int nt = min(NTB, T - t0);
  const int tid = threadIdx.x;
  {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t0 * d);
    uint4* dst = reinterpret_cast<uint4*>(xs_raw);
    const int n16 = nt * d / 8;
    for (int i = tid; i < n16; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x * kLogitWarps + warp;
  if (e >= E) return;
  float acc[NTB];
#pragma unroll
  for (int t = 0; t < NTB; ++t) acc[t] = 0.f;
  const WT* wr = W + (size_t)e * d;
  const int n4 = d >> 2;
#pragma unroll 4
  for (int i = lane; i < n4; i += 32) {
    const float4 w = ldw4(wr, i);
#pragma unroll
    for (int t = 0; t < NTB; ++t) {
      if (t < nt) {
        const uint2 xv = reinterpret_cast<const uint2*>(xs_raw + (size_t)t * (d >> 1))[i];
        acc[t] = fmaf(w.x, bf16lo(xv.x), acc[t]);
        acc[t] = fmaf(w.y, bf16hi(xv.x), acc[t]);
        acc[t] = fmaf(w.z, bf16lo(xv.y), acc[t]);
        acc[t] = fmaf(w.w, bf16hi(xv.y), acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NTB; ++t) {
    const float v = warp_sum(acc[t]);
    if (lane == 0 && t < nt) L[(size_t)(t0 + t) * E + e] = v;
  }
}

// ---------------------------------------------------------------------------
// Logits for large T: tiled fp32 SIMT GEMM, 128 tokens x 64 experts per CTA,
// 8x4 outputs per thread, K in steps of 16 with register prefetch.  With
// gridDim.z = 2 each CTA sums one half of K into its own partial array
// (L + z*T*E); the top-k adds the two partials in a fixed order.
// ---------------------------------------------------------------------------
constexpr int kLBM = 128, kLBN = 64, kLBK = 16;

template <typename WT>
__global__ void __launch_bounds__(256)
router_logits_tiled_kernel(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                           float* __restrict__ L, int T, int d, int E) {
  __shared__ __align__(16) float xs[kLBK][kLBM + 4];
  __shared__ __align__(16) float wsm[kLBK][kLBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kLBM, n0 = blockIdx.x * kLBN;
  const int kspan = d / gridDim.z, kbeg = blockIdx.z * kspan, kend = kbeg + kspan;
  L += (size_t)blockIdx.z * T * E;
  // loaders: x tile 128 x 16 bf16 -> each thread 8 elements (one 16-byte load)
  const int xr = tid >> 1, xc = (tid & 1) * 8;
  // W tile 64 x 16 fp32 -> each thread 4 elements (one float4)
  const int wr = tid >> 2, wc = (tid & 3) * 4;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  uint4 xreg = make_uint4(0, 0, 0, 0);
  float4 wreg = make_float4(0.f, 0.f, 0.f, 0.f);
  auto load = [&](int k0) {
    const int gm = m0 + xr;
    xreg = (gm < T) ? *reinterpret_cast<const uint4*>(x + (size_t)gm * d + k0 + xc) : make_uint4(0, 0, 0, 0);
    const int gn = n0 + wr;
    wreg = (gn < E) ? ldw4(W + (size_t)gn * d + k0 + wc, 0) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  load(kbeg);
  for (int k0 = kbeg; k0 < kend; k0 += kLBK) {
    __syncthreads();
    xs[xc + 0][xr] = bf16lo(xreg.x);
    xs[xc + 1][xr] = bf16hi(xreg.x);
    xs[xc + 2][xr] = bf16lo(xreg.y);
    xs[xc + 3][xr] = bf16hi(xreg.y);
    xs[xc + 4][xr] = bf16lo(xreg.z);
    xs[xc + 5][xr] = bf16hi(xreg.z);
    xs[xc + 6][xr] = bf16lo(xreg.w);
    xs[xc + 7][xr] = bf16hi(xreg.w);
    wsm[wc + 0][wr] = wreg.x;
    wsm[wc + 1][wr] = wreg.y;
    wsm[wc + 2][wr] = wreg.z;
    wsm[wc + 3][wr] = wreg.w;
    __syncthreads();
    if (k0 + kLBK < kend) load(k0 + kLBK);
#pragma unroll
    for (int kk = 0; kk < kLBK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[kk][ty * 8 + 4]);
      const float4 b = *reinterpret_cast<const float4*>(&wsm[kk][tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + ty * 8 + i;
    if (gm >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < E) L[(size_t)gm * E + gn] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// sqrtsoftplus + biased top-k + renormalisation: one warp per token.
// Expert e lives in lane e % 32, slot e / 32.
// ---------------------------------------------------------------------------
template <int MAXPER>
MOE_DEV void topk_token(const float* __restrict__ Lrow, const float* __restrict__ bias, int E, int k,
                        int* __restrict__ ids_row, float* __restrict__ w_row,
                        const float* __restrict__ Lrow2 = nullptr) {
  const int lane = threadIdx.x & 31;
  float key[MAXPER], sc[MAXPER];
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    const int e = i * 32 + lane;
    if (e < E) {
      const float s = sqrt_softplus(Lrow2 ? __ldcg(Lrow + e) + __ldcg(Lrow2 + e) : __ldcg(Lrow + e));
      sc[i] = s;
      float kv = bias ? s + bias[e] : s;
      key[i] = (kv != kv) ? -INFINITY : kv;
    } else {
      sc[i] = 0.f;
      key[i] = -INFINITY;
    }
  }
  uint32_t taken = 0;  // bit i: slot i of this lane already selected
  float my_s = 0.f;
  int my_id = 0;
  float ssum = 0.f;
  for (int j = 0; j < k; ++j) {
    float best = -INFINITY;
    int bidx = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
      const int e = i * 32 + lane;
      const bool ok = (e < E) && !((taken >> i) & 1u);
      if (ok && (key[i] > best || (key[i] == best && e < bidx))) {
        best = key[i];
        bidx = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
      if (ob > best || (ob == best && oi < bidx)) {
        best = ob;
        bidx = oi;
      }
    }
    // owner lane publishes the unbiased score and marks the slot taken
    float s_sel = 0.f;
    const int owner = bidx & 31, slot = bidx >> 5;
    if (lane == owner) {
#pragma unroll
      for (int i = 0; i < MAXPER; ++i)
        if (i == slot) {
          s_sel = sc[i];
          taken |= 1u << i;
        }
    }
    s_sel = __shfl_sync(0xffffffffu, s_sel, owner);
    ssum += s_sel;
    if (lane == j) {
      my_s = s_sel;
      my_id = bidx;
    }
  }
  if (lane < k) {
    ids_row[lane] = my_id;
    w_row[lane] = ssum > 0.f ? my_s / ssum : 1.f / (float)k;
  }
}

template <int MAXPER>
__global__ void __launch_bounds__(256)
topk_kernel(const float* __restrict__ L, const float* __restrict__ bias, int T, int E, int k,
            int* __restrict__ ids, float* __restrict__ wts, const float* __restrict__ L2) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= T) return;
  topk_token<MAXPER>(L + (size_t)warp * E, bias, E, k, ids + (size_t)warp * k, wts + (size_t)warp * k,
                     L2 ? L2 + (size_t)warp * E : nullptr);
}

// ---------------------------------------------------------------------------
// Hash routing: one warp per token.  Out-of-range ids are reported through
// the error word and routed to expert 0 with weight 0.
// ---------------------------------------------------------------------------
template <int KMAX, typename WT>
MOE_DEV void route_hash_warp(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                             const int* __restrict__ token_ids, const int* __restrict__ table, int T, int d, int E,
                             int k, int vocab, int* __restrict__ ids, float* __restrict__ wts, int* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const int t = warp;
  const int tok = token_ids[t];
  const bool tok_ok = tok >= 0 && tok < vocab;
  int eid[KMAX];
  bool good[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    eid[j] = 0;
    good[j] = false;
    if (j < k && tok_ok) {
      const int e = table[(size_t)tok * k + j];
      good[j] = e >= 0 && e < E;
      eid[j] = good[j] ? e : 0;
    }
  }
  bool any_bad = !tok_ok;
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < k && !good[j]) any_bad = true;
  if (any_bad && lane == 0) set_error(err, kErrDeviceInput);
  float s[KMAX];
  if (W != nullptr) {
    float acc[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) acc[j] = 0.f;
    const uint2* xr = reinterpret_cast<const uint2*>(x + (size_t)t * d);
    for (int i = lane; i < (d >> 2); i += 32) {
      const uint2 xv = xr[i];
      const float x0 = bf16lo(xv.x), x1 = bf16hi(xv.x), x2 = bf16lo(xv.y), x3 = bf16hi(xv.y);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
          const float4 w = ldw4(W + (size_t)eid[j] * d, i);
          acc[j] = fmaf(w.x, x0, fmaf(w.y, x1, fmaf(w.z, x2, fmaf(w.w, x3, acc[j]))));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const float v = warp_sum(acc[j]);
      s[j] = (j < k && good[j]) ? sqrt_softplus(v) : 0.f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) s[j] = (j < k && good[j]) ? 1.f : 0.f;
  }
  float ssum = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) ssum += s[j];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k && lane == j) {
      ids[(size_t)t * k + j] = eid[j];
      float w = 0.f;
      if (good[j]) w = ssum > 0.f ? s[j] / ssum : 0.f;
      wts[(size_t)t * k + j] = w;
    }
  }
}

template <int KMAX, typename WT>
__global__ void __launch_bounds__(256)
route_hash_kernel(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                  const int* __restrict__ token_ids, const int* __restrict__ table, int T, int d, int E,
                  int k, int vocab, int* __restrict__ ids, float* __restrict__ wts, int* err) {
  route_hash_warp<KMAX, WT>(x, W, token_ids, table, T, d, E, k, vocab, ids, wts, err);
}

// ---------------------------------------------------------------------------
// Block-parallel tails for the fused routing kernels (one block, <= 1024
// threads, shared memory `sm` of at least 2*E + 2*N ints).
// ---------------------------------------------------------------------------
// Top-k of one token by ranks: expert e is selected at position rank(e) =
// #{j : key_j > key_e or (key_j == key_e and j < e)} when rank(e) < k.
__device__ void topk_token_block(const float* __restrict__ Lrow, const float* __restrict__ bias, int E, int k,
                                 int* __restrict__ ids_row, float* __restrict__ w_row, float* keys, float* scs,
                                 float* sel) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float s = sqrt_softplus(__ldcg(Lrow + e));
    const float kv = bias ? s + bias[e] : s;
    keys[e] = (kv != kv) ? -INFINITY : kv;
    scs[e] = s;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float ke = keys[e];
    int rank = 0;
    for (int j = 0; j < E; ++j) {
      const float kj = keys[j];
      rank += (kj > ke || (kj == ke && j < e)) ? 1 : 0;
    }
    if (rank < k) {
      ids_row[rank] = e;
      sel[rank] = scs[e];
    }
  }
  __syncthreads();
  if (threadIdx.x < k) {
    float ssum = 0.f;
    for (int j = 0; j < k; ++j) ssum += sel[j];  // same order in every thread
    w_row[threadIdx.x] = ssum > 0.f ? sel[threadIdx.x] / ssum : 1.f / (float)k;
  }
  __syncthreads();
}

// Stable grouping of N pairs by expert, by ranks: pair i goes to position
// #{j : (e_j, j) < (e_i, i)}; offsets[x] = #{j : e_j < x}; the active list
// holds each expert once, ascending.  Out-of-range ids are reported and
// treated as expert 0.
__device__ void permute_ranks_block(const int* __restrict__ ids, int N, int E, int* __restrict__ offsets,
                                    int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active,
                                    int* err, int* ev, int* first) {
  bool bad = false;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    int e = ids[i];
    if (e < 0 || e >= E) {
      bad = true;
      e = 0;
    }
    ev[i] = e;
  }
  if (bad) set_error(err, kErrDeviceInput);
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int e = ev[i];
    int rank = 0, f = 1;
    for (int j = 0; j < N; ++j) {
      const int ej = ev[j];
      rank += (ej < e || (ej == e && j < i)) ? 1 : 0;
      if (ej == e && j < i) f = 0;
    }
    sorted_rows[rank] = i;
    inv[i] = rank;
    first[i] = f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    if (first[i]) {
      const int e = ev[i];
      int dr = 0;
      for (int j = 0; j < N; ++j) dr += (first[j] && ev[j] < e) ? 1 : 0;
      active[1 + dr] = e;
    }
  }
  for (int x = threadIdx.x; x <= E; x += blockDim.x) {
    int c = 0;
    for (int j = 0; j < N; ++j) c += ev[j] < x ? 1 : 0;
    offsets[x] = c;
  }
  if (threadIdx.x == 0) {
    int nf = 0;
    for (int j = 0; j < N; ++j) nf += first[j];
    active[0] = nf;
  }
}

// ---------------------------------------------------------------------------
// Small-T fused routing: logits, top-k, renormalisation and the stable
// permutation in one launch.  Every block computes the logits of two experts
// (four warps per expert, each over a quarter of d_model) for all tokens; the
// last block to finish (arrival counter in the workspace, reset afterwards)
// selects the experts of every token and groups the pairs by expert.
// ---------------------------------------------------------------------------
constexpr int kFusedTB = 8;            // tokens per pass over the staged x rows
constexpr int kFusedMaxT = 32;

template <int MAXPER, typename WT>
__global__ void __launch_bounds__(256)
route_small_fused_kernel(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                         const float* __restrict__ bias, int T, int d, int E, int k, float* __restrict__ L,
                         int* __restrict__ ids, float* __restrict__ wts, int* __restrict__ offsets,
                         int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active,
                         int* counter, int* err) {
  extern __shared__ __align__(16) uint32_t sm_raw[];
  __shared__ float part[8][kFusedTB];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int is_last;
  pdl_trigger();  // the expert FFN may start its launch (it waits for this grid before reading)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x * 2 + (warp >> 2);
  const int quarter = warp & 3;
  const int q4 = d >> 4;  // float4 per quarter row
  // this warp's quarter row of the router weight, kept in registers
  float4 wv[8];
  const bool live = e < E;
  {
    const WT* wr = W + (size_t)min(e, E - 1) * d + (size_t)quarter * q4 * 4;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = lane + 32 * u;
      wv[u] = (live && i < q4) ? ldw4(wr, i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int t0 = 0; t0 < T; t0 += kFusedTB) {
    const int nt = min(kFusedTB, T - t0);
    __syncthreads();
    {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t0 * d);
      uint4* dst = reinterpret_cast<uint4*>(sm_raw);
      for (int i = tid; i < nt * d / 8; i += blockDim.x) dst[i] = src[i];
    }
    __syncthreads();
    float acc[kFusedTB];
#pragma unroll
    for (int t = 0; t < kFusedTB; ++t) acc[t] = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = lane + 32 * u;
      if (i < q4) {
#pragma unroll
        for (int t = 0; t < kFusedTB; ++t) {
          if (t < nt) {
            const uint2 xv = reinterpret_cast<const uint2*>(sm_raw + (size_t)t * (d >> 1))[quarter * q4 + i];
            acc[t] = fmaf(wv[u].x, bf16lo(xv.x), acc[t]);
            acc[t] = fmaf(wv[u].y, bf16hi(xv.x), acc[t]);
            acc[t] = fmaf(wv[u].z, bf16lo(xv.y), acc[t]);
            acc[t] = fmaf(wv[u].w, bf16hi(xv.y), acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kFusedTB; ++t) {
      const float v = warp_sum(acc[t]);
      if (lane == 0) part[warp][t] = v;
    }
    __syncthreads();
    if (tid < 2 * kFusedTB) {
      const int h = tid / kFusedTB, t = tid % kFusedTB;
      const int ee = blockIdx.x * 2 + h;
      if (ee < E && t < nt) {
        L[(size_t)(t0 + t) * E + ee] = part[4 * h][t] + part[4 * h + 1][t] + part[4 * h + 2][t] + part[4 * h + 3][t];
        __threadfence();  // publish before the arrival below
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    is_last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
    if (is_last) __threadfence();
  }
  __syncthreads();
  if (!is_last) return;
  // last block: every token's top-k, then the grouping of the T*k pairs
  float* fsm = reinterpret_cast<float*>(sm_raw);
  if (T <= 2) {
    for (int t = 0; t < T; ++t)
      topk_token_block(L + (size_t)t * E, bias, E, k, ids + (size_t)t * k, wts + (size_t)t * k, fsm, fsm + E,
                       fsm + 2 * E);
  } else {
    for (int t = warp; t < T; t += 8)
      topk_token<MAXPER>(L + (size_t)t * E, bias, E, k, ids + (size_t)t * k, wts + (size_t)t * k);
  }
  __threadfence_block();
  __syncthreads();
  int* ism = reinterpret_cast<int*>(sm_raw);
  permute_ranks_block(ids, T * k, E, offsets, sorted_rows, inv, active, err, ism, ism + T * k);
  if (tid == 0) *counter = 0;
  (void)warp_tot;
  (void)total;
}

// Hash routing of token t = blockIdx.x by the whole block: warp 0 gathers
// the token's table row, every warp dots x[t] with the k router rows over its
// slice of d (partials in `part`), warp 0 finishes the weights.  Same rules as
// route_hash_warp (bad ids: expert 0, weight 0, error word).
template <int KMAX, typename WT>
MOE_DEV void route_hash_block(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                              const int* __restrict__ token_ids, const int* __restrict__ table, int d, int E, int k,
                              int vocab, int* __restrict__ ids, float* __restrict__ wts, int* err,
                              float (*part)[KMAX], int* s_eid, int* s_good) {
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (warp == 0) {
    const int tok = token_ids[t];
    const bool tok_ok = tok >= 0 && tok < vocab;
    int e = 0;
    bool good = false;
    if (lane < k && tok_ok) {
      e = table[(size_t)tok * k + lane];
      good = e >= 0 && e < E;
      if (!good) e = 0;
    }
    const bool bad = !tok_ok || (lane < k && !good);
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, kErrDeviceInput);
    if (lane < KMAX) {
      s_eid[lane] = e;
      s_good[lane] = good ? 1 : 0;
    }
  }
  __syncthreads();
  if (W != nullptr) {
    float acc[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) acc[j] = 0.f;
    const int n4 = d >> 2;
    const int lo = n4 * warp / nw, hi = n4 * (warp + 1) / nw;
    const uint2* xr = reinterpret_cast<const uint2*>(x + (size_t)t * d);
    const WT* wr[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) wr[j] = W + (size_t)(j < k ? s_eid[j] : 0) * d;
    for (int i = lo + lane; i < hi; i += 32) {
      const uint2 xv = xr[i];
      const float x0 = bf16lo(xv.x), x1 = bf16hi(xv.x), x2 = bf16lo(xv.y), x3 = bf16hi(xv.y);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
          const float4 w = ldw4(wr[j], i);
          acc[j] = fmaf(w.x, x0, fmaf(w.y, x1, fmaf(w.z, x2, fmaf(w.w, x3, acc[j]))));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const float v = warp_sum(acc[j]);
      if (lane == 0 && j < k) part[warp][j] = v;
    }
  }
  __syncthreads();
  if (warp == 0) {
    float sj = 0.f;
    const bool gj = lane < k && s_good[lane] != 0;
    if (gj) {
      if (W != nullptr) {
        float l = 0.f;
        for (int w = 0; w < nw; ++w) l += part[w][lane];
        sj = sqrt_softplus(l);
      } else {
        sj = 1.f;
      }
    }
    const float ssum = warp_sum(sj);
    if (lane < k) {
      ids[(size_t)t * k + lane] = s_eid[lane];
      wts[(size_t)t * k + lane] = gj && ssum > 0.f ? sj / ssum : 0.f;
    }
  }
}

// Hash routing plus permutation, one launch: one block per token, the last
// block groups the pairs by expert.
template <int KMAX, typename WT>
__global__ void __launch_bounds__(256)
route_hash_fused_kernel(const __nv_bfloat16* __restrict__ x, const WT* __restrict__ W,
                        const int* __restrict__ token_ids, const int* __restrict__ table, int T, int d, int E,
                        int k, int vocab, int* __restrict__ ids, float* __restrict__ wts, int* __restrict__ offsets,
                        int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active,
                        int* counter, int* err) {
  extern __shared__ __align__(16) uint32_t sm_raw[];
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int is_last;
  __shared__ float part[8][KMAX];
  __shared__ int s_eid[KMAX], s_good[KMAX];
  pdl_trigger();  // the expert FFN may start its launch (it waits for this grid before reading)
  route_hash_block<KMAX, WT>(x, W, token_ids, table, d, E, k, vocab, ids, wts, err, part, s_eid, s_good);
  __threadfence();  // publish this token's ids/weights before the arrival below
  __syncthreads();
  if (threadIdx.x == 0) {
    is_last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
    if (is_last) __threadfence();
  }
  __syncthreads();
  if (!is_last) return;
  int* ism = reinterpret_cast<int*>(sm_raw);
  permute_ranks_block(ids, T * k, E, offsets, sorted_rows, inv, active, err, ism, ism + T * k);
  if (threadIdx.x == 0) *counter = 0;
  (void)warp_tot;
  (void)total;
}

}  // namespace moe
