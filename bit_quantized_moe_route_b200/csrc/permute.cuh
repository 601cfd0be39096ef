// Step 2 of the layer: group the T*k (token, slot) pairs by expert.
//
// A stable counting sort by expert id over the flat indices i = t*k + j:
// per-expert histogram, exclusive scan -> expert_offsets, then a stable
// scatter (ranks from warp match masks plus per-warp counts, tile by tile, so
// no unordered atomics decide an order).  Also emits the ascending list of
// experts that received at least one pair, used to size the FFN work lists.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kPermThreads = 1024;

// Block-wide exclusive scan of one int per thread (any multiple of 32
// threads up to 1024).  *total receives the block sum.
__device__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < nwarps ? warp_tot[lane] : 0;
    int winc = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += n;
    }
    if (lane < nwarps) warp_tot[lane] = winc - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = winc;
  }
  __syncthreads();
  const int r = warp_tot[warp] + inc - v;
  __syncthreads();
  return r;
}

// Stable counting sort of the N expert ids by expert, by one thread block of
// any size (multiple of 32).  sm: (2 + nwarps) * E ints of shared memory.
__device__ void permute_block(const int* __restrict__ ids, int N, int E, int* __restrict__ offsets,
                              int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active,
                              int* err, int* sm, int* warp_tot, int* total) {
  const int nthr = blockDim.x, nwarps = nthr >> 5;
  int* cnt = sm;            // [E] pairs per expert, later the running base
  int* off = sm + E;        // [E] exclusive offsets
  int* wc = sm + 2 * E;     // [nwarps][E] per-warp counts of the current tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < E; e += nthr) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int i = tid; i < N; i += nthr) {
    int e = ids[i];
    if (e < 0 || e >= E) {
      bad = true;
      e = 0;
    }
    atomicAdd(&cnt[e], 1);
  }
  if (bad) set_error(err, kErrDeviceInput);
  __syncthreads();
  int carry = 0, acarry = 0;
  for (int e0 = 0; e0 < E; e0 += nthr) {
    const int e = e0 + tid;
    const int c = e < E ? cnt[e] : 0;
    const int ex = block_exclusive_scan(c, warp_tot, total);
    const int chunk_total = *total;
    const int flag = c > 0 ? 1 : 0;
    const int aex = block_exclusive_scan(flag, warp_tot, total);
    const int achunk = *total;
    if (e < E) {
      off[e] = carry + ex;
      offsets[e] = carry + ex;
      if (flag) active[1 + acarry + aex] = e;
    }
    carry += chunk_total;
    acarry += achunk;
    __syncthreads();
  }
  if (tid == 0) {
    offsets[E] = carry;
    active[0] = acarry;
  }
  for (int e = tid; e < E; e += nthr) cnt[e] = 0;
  __syncthreads();

  const unsigned lt_mask = (1u << lane) - 1u;
  for (int t0 = 0; t0 < N; t0 += nthr) {
    for (int q = tid; q < nwarps * E; q += nthr) wc[q] = 0;
    __syncthreads();
    const int i = t0 + tid;
    int e = -1;
    if (i < N) {
      e = ids[i];
      if (e < 0 || e >= E) e = 0;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & lt_mask);
    if (e >= 0 && rank_w == 0) wc[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int pre = 0;
      for (int w = 0; w < warp; ++w) pre += wc[w * E + e];
      const int p = off[e] + cnt[e] + pre + rank_w;
      sorted_rows[p] = i;
      inv[i] = p;
    }
    __syncthreads();
    for (int x = tid; x < E; x += nthr) {
      int s = 0;
      for (int w = 0; w < nwarps; ++w) s += wc[w * E + x];
      cnt[x] += s;
    }
    __syncthreads();
  }
}

// The same stable grouping for N <= 32 pairs by a single warp: the sorted
// position of pair i is the number of pairs (e_j, j) ordered before (e_i, i).
__device__ void permute_warp(const int* __restrict__ ids, int N, int E, int* __restrict__ offsets,
                             int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active, int* err) {
  const int lane = threadIdx.x & 31;
  int e = 0x7fffffff;
  bool bad = false;
  if (lane < N) {
    e = ids[lane];
    if (e < 0 || e >= E) {
      bad = true;
      e = 0;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, kErrDeviceInput);
  // first occurrence of each expert among the pairs (lowest lane of its peers)
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int first = (lane < N && (__ffs(peers) - 1) == lane) ? 1 : 0;
  int rank = 0, drank = 0;
  for (int j = 0; j < N; ++j) {
    const int ej = __shfl_sync(0xffffffffu, e, j);
    const int fj = __shfl_sync(0xffffffffu, first, j);
    rank += (ej < e || (ej == e && j < lane)) ? 1 : 0;
    drank += (fj && ej < e) ? 1 : 0;
  }
  if (lane < N) {
    sorted_rows[rank] = lane;
    inv[lane] = rank;
    if (first) active[1 + drank] = e;
  }
  const int n_first = __popc(__ballot_sync(0xffffffffu, lane < N && first));
  if (lane == 0) active[0] = n_first;
  // offsets[x] = pairs with an expert id below x
  for (int x0 = 0; x0 <= E; x0 += 32) {
    const int x = x0 + lane;
    int c = 0;
    for (int j = 0; j < N; ++j) c += (__shfl_sync(0xffffffffu, e, j) < x) ? 1 : 0;
    if (x <= E) offsets[x] = c;
  }
}

// One CTA of 1024 threads.  Dynamic shared memory: (2 + 32) * E ints.
// active[0] = number of experts with pairs, active[1..] their ids ascending.
__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const int* __restrict__ ids, int N, int E, int* __restrict__ offsets,
               int* __restrict__ sorted_rows, int* __restrict__ inv, int* __restrict__ active,
               int* err) {
  extern __shared__ int sm[];
  __shared__ int warp_tot[32];
  __shared__ int total;
  permute_block(ids, N, E, offsets, sorted_rows, inv, active, err, sm, warp_tot, &total);
}

// ---------------------------------------------------------------------------
// The same stable grouping for large N in three launches: CTA b owns pairs
// [b*1024, (b+1)*1024).  The sorted position of pair i (expert e) is
// offsets[e] + #{pairs before i's chunk with expert e} + #{pairs of i's chunk
// before i with expert e}; the middle term comes from per-chunk counts.
// ---------------------------------------------------------------------------
// 1: per-chunk expert counts -> cnt[b * E + e]
__global__ void __launch_bounds__(kPermThreads)
permute_count_kernel(const int* __restrict__ ids, int N, int E, int* __restrict__ cnt, int* err) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += kPermThreads) hist[e] = 0;
  __syncthreads();
  const int i = blockIdx.x * kPermThreads + threadIdx.x;
  bool bad = false;
  if (i < N) {
    int e = ids[i];
    if (e < 0 || e >= E) {
      bad = true;
      e = 0;
    }
    atomicAdd(&hist[e], 1);
  }
  if (bad) set_error(err, kErrDeviceInput);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kPermThreads) cnt[(size_t)blockIdx.x * E + e] = hist[e];
}

// 2: one CTA: offsets[e], the active list, and cnt[b * E + e] turned into the
// first sorted position of expert e's pairs in chunk b
__global__ void __launch_bounds__(kPermThreads)
permute_scan_kernel(int* __restrict__ cnt, int n_chunks, int E, int* __restrict__ offsets,
                    int* __restrict__ active) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  int carry = 0, acarry = 0;
  for (int e0 = 0; e0 < E; e0 += kPermThreads) {
    const int e = e0 + threadIdx.x;
    int c = 0;
    if (e < E)
      for (int b = 0; b < n_chunks; ++b) c += cnt[(size_t)b * E + e];
    const int ex = block_exclusive_scan(c, warp_tot, &total);
    const int chunk_total = total;
    const int flag = c > 0 ? 1 : 0;
    const int aex = block_exclusive_scan(flag, warp_tot, &total);
    const int achunk = total;
    if (e < E) {
      offsets[e] = carry + ex;
      if (flag) active[1 + acarry + aex] = e;
      int run = carry + ex;
      for (int b = 0; b < n_chunks; ++b) {
        const int v = cnt[(size_t)b * E + e];
        cnt[(size_t)b * E + e] = run;
        run += v;
      }
    }
    carry += chunk_total;
    acarry += achunk;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    offsets[E] = carry;
    active[0] = acarry;
  }
}

// 3: each CTA places its chunk: warp-level ranks (match_any) plus the counts
// of the warps before it.  Dynamic shared memory: 32 * E ints.
__global__ void __launch_bounds__(kPermThreads)
permute_scatter_kernel(const int* __restrict__ ids, int N, int E, const int* __restrict__ base,
                       int* __restrict__ sorted_rows, int* __restrict__ inv) {
  extern __shared__ int wc[];  // [32 warps][E] counts of this chunk
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int q = tid; q < 32 * E; q += kPermThreads) wc[q] = 0;
  __syncthreads();
  const int i = blockIdx.x * kPermThreads + tid;
  int e = -1;
  if (i < N) {
    e = ids[i];
    if (e < 0 || e >= E) e = 0;
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank_w == 0) wc[warp * E + e] = __popc(peers);
  __syncthreads();
  if (e >= 0) {
    int pre = 0;
    for (int w = 0; w < warp; ++w) pre += wc[w * E + e];
    const int p = base[(size_t)blockIdx.x * E + e] + pre + rank_w;
    sorted_rows[p] = i;
    inv[i] = p;
  }
}

// Active-expert list from caller-provided offsets (single CTA).
__global__ void __launch_bounds__(kPermThreads)
active_from_offsets_kernel(const int* __restrict__ offsets, int E, int Tk, const int* __restrict__ sorted_rows,
                           int* __restrict__ active, int* __restrict__ err, int* __restrict__ valid) {
  // A caller-supplied permutation is checked before any expert FFN kernel
  // reads through it: offsets[0] = 0, offsets[E] = Tk, non-decreasing, and
  // every sorted row a flat pair index in [0, Tk).  A violation records
  // MOE_ERR_DEVICE_INPUT and leaves no active expert (and *valid = 0), so
  // nothing downstream touches memory through the bad lists.
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ int bad;
  if (threadIdx.x == 0) bad = (offsets[0] != 0 || offsets[E] != Tk) ? 1 : 0;
  __syncthreads();
  int mine = 0;
  for (int e = threadIdx.x; e < E; e += kPermThreads) {
    const int o0 = offsets[e], o1 = offsets[e + 1];
    mine |= (o0 < 0 || o1 < o0 || o1 > Tk) ? 1 : 0;
  }
  for (int p = threadIdx.x; p < Tk; p += kPermThreads) mine |= ((unsigned)sorted_rows[p] >= (unsigned)Tk) ? 1 : 0;
  if (mine) bad = 1;
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      active[0] = 0;
      if (valid) *valid = 0;
      set_error(err, kErrDeviceInput);
    }
    return;
  }
  int acarry = 0;
  for (int e0 = 0; e0 < E; e0 += kPermThreads) {
    const int e = e0 + threadIdx.x;
    const int flag = (e < E && offsets[e + 1] > offsets[e]) ? 1 : 0;
    const int ex = block_exclusive_scan(flag, warp_tot, &total);
    if (flag) active[1 + acarry + ex] = e;
    acarry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    active[0] = acarry;
    if (valid) *valid = 1;
  }
}

}  // namespace moe
