// Host side of the C ABI declared in include/moe_lowbit.h: argument
// validation, workspace carving and kernel launches.  Nothing here computes
// any part of the layer; every step runs in the kernels included below.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/moe_lowbit.h"
#include "common.cuh"
#include "ffn_gemv.cuh"
#include "stream_types.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "tc_prep.cuh"
#include "ffn_umma.cuh"
#include "dequant_fp8.cuh"
#include "hc_mix.cuh"
#include "ffn_decode.cuh"

#include <cudaTypedefs.h>

using namespace moe;

namespace {

thread_local char g_detail[512] = "";

// Benchmark timing hooks (see moe_set_timing_events).
struct TimingHook {
  void* const* events = nullptr;
  int n = 0;
  int used = 0;
  const char* labels[32] = {};
};
thread_local TimingHook g_hook;
thread_local int g_hook_count = 0;
thread_local const char* g_hook_labels[32] = {};

// A failed record disarms the hook and clears the CUDA error so that it
// cannot be mistaken for a kernel launch failure.
void hook_record(int i, cudaStream_t s) {
  if (!g_hook.events[i] || cudaEventRecord(reinterpret_cast<cudaEvent_t>(g_hook.events[i]), s) != cudaSuccess) {
    cudaGetLastError();
    g_hook.events = nullptr;
    g_hook.used = 0;
  }
}
void hook_begin(cudaStream_t s) {
  if (g_hook.events && g_hook.n > 0) {
    g_hook.used = 1;
    hook_record(0, s);
  }
}
void hook_mark(cudaStream_t s, const char* label) {
  if (g_hook.events && g_hook.used > 0 && g_hook.used < g_hook.n && g_hook.used <= 32) {
    g_hook.labels[g_hook.used - 1] = label;
    ++g_hook.used;
    hook_record(g_hook.used - 1, s);
  }
}
void hook_end() {
  if (g_hook.events) {
    g_hook_count = g_hook.used;
    for (int i = 0; i < 32; ++i) g_hook_labels[i] = g_hook.labels[i];
    g_hook = TimingHook{};
  }
}

moe_status_t fail(moe_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return st;
}

moe_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MOE_CHECK_LAUNCH(what)                        \
  do {                                                \
    cudaError_t _e = cudaGetLastError();              \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
  size_t hdr, logits, ids, wts, offsets, sorted, inv, active, h, y, xstage, tokstage, outstage;
  size_t x16, tiles, tiles2, ntiles;  // tensor-core FFN: fp16 token rows by position, token-tile plans
  size_t pchunks;                     // multi-CTA permutation: per-chunk expert counts / bases
  size_t dxp, dxsx, dhp, dhsx, dcnth, dsync;  // fused decode: planes, block steps, counters
  bool tc = false;            // the regions above exist
  size_t total;
};

int f_max_of(const moe_dims_t& d) { return std::max(d.d_ff, d.d_ff_shared); }
int shared_rows(const moe_dims_t& d) { return d.d_ff_shared > 0 ? d.T : 0; }

WsLayout layout_of(const moe_dims_t& d) {
  WsLayout L{};
  size_t o = 0;
  const size_t T = d.T, k = d.top_k, E = d.n_experts, D = d.d_model;
  const size_t P = T * k + shared_rows(d);
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.hdr = take(sizeof(WsHeader));
  L.logits = take(d.hash_mode ? 0 : 2 * T * E * sizeof(float));  // two K-half partials at large T
  L.ids = take(T * k * sizeof(int));
  L.wts = take(T * k * sizeof(float));
  L.offsets = take((E + 1) * sizeof(int));
  L.sorted = take(T * k * sizeof(int));
  L.inv = take(T * k * sizeof(int));
  L.active = take((E + 1) * sizeof(int));
  L.h = take(P * (size_t)f_max_of(d) * sizeof(float));
  L.y = take(P * D * sizeof(float));
  L.xstage = take(T * D * 2);
  L.tokstage = take(T * sizeof(int));
  L.outstage = take(T * D * 2);
  L.x16 = take(P * D * 2);
  L.tiles = take(((T * k + kTcN - 1) / kTcN + E) * sizeof(int4));
  L.tiles2 = take(((T * k + kUmN - 1) / kUmN + E) * sizeof(int4));
  L.ntiles = take(2 * sizeof(int));
  L.pchunks = take(((T * k + kPermThreads - 1) / kPermThreads) * E * sizeof(int));
  {
    // fused small-batch layer (T <= 32): activation planes of x (two layouts)
    // and of h, their per-64-input steps and sums, dependency counters
    const bool dec = T <= (size_t)kDecMaxT;
    const size_t fm = (size_t)f_max_of(d);
    L.dxp = take(dec ? 2 * T * D * 4 : 0);
    L.dxsx = take(dec ? T * (D / 64 + 1) * 16 : 0);
    L.dhp = take(dec ? P * fm * 4 : 0);
    L.dhsx = take(dec ? P * (fm / 64 + 1) * 16 : 0);
    L.dcnth = take(dec ? (kDecMaxPairs + 8) * sizeof(int) : 0);
    L.dsync = take(dec ? 4 * sizeof(int) : 0);
  }
  L.tc = true;
  L.total = o;
  return L;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

// The GEMV path gives each thread one 32-input chunk of a row: widths are
// multiples of 32 up to 8192 (at most 256 chunks per row).
bool width_ok(int n) { return n >= 32 && n <= 8192 && n % 32 == 0; }

moe_status_t check_dims(const moe_dims_t* d) {
  if (!d) return fail(MOE_ERR_INVALID_ARG, "dims is NULL");
  if (d->T < 1) return fail(MOE_ERR_INVALID_ARG, "T=%d must be >= 1", d->T);
  if (d->n_experts < 1 || d->n_experts > 1024)
    return fail(d->n_experts < 1 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED, "n_experts=%d outside [1,1024]",
                d->n_experts);
  if (d->top_k < 1 || d->top_k > d->n_experts || d->top_k > 32)
    return fail(MOE_ERR_INVALID_ARG, "top_k=%d must be in [1, min(n_experts, 32)]", d->top_k);
  if (!width_ok(d->d_model)) return fail(MOE_ERR_UNSUPPORTED, "d_model=%d not supported", d->d_model);
  if (!width_ok(d->d_ff)) return fail(MOE_ERR_UNSUPPORTED, "d_ff=%d not supported", d->d_ff);
  if (d->d_ff_shared < 0 || (d->d_ff_shared > 0 && !width_ok(d->d_ff_shared)))
    return fail(MOE_ERR_UNSUPPORTED, "d_ff_shared=%d not supported", d->d_ff_shared);
  if (d->hash_mode && d->vocab < 1) return fail(MOE_ERR_INVALID_ARG, "hash mode needs vocab >= 1");
  if (d->router_dtype != 0 && d->router_dtype != 1)
    return fail(MOE_ERR_UNSUPPORTED, "router_dtype=%d not in {0 (fp32), 1 (bf16)}", d->router_dtype);
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_dev_ptr(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_INVALID_ARG, "%s: cannot query pointer (%s)", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(MOE_ERR_INVALID_ARG, "%s is not device memory", name);
  return MOE_OK;
}

moe_status_t check_qmat(const moe_qmat_t* m, int n_in, const char* name, QMatDev* out, int n_out) {
  if (!m) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  int code;
  if (m->fmt == MOE_FMT_AFFINE) {
    switch (m->bits) {
      case 2: code = F_A2; break;
      case 3: code = F_A3; break;
      case 4: code = F_A4; break;
      case 8: code = F_A8; break;
      default: return fail(MOE_ERR_UNSUPPORTED, "%s: affine bits=%d not in {2,3,4,8}", name, m->bits);
    }
    if (m->group != 32 && m->group != 64 && m->group != 128)
      return fail(MOE_ERR_UNSUPPORTED, "%s: group=%d not in {32,64,128}", name, m->group);
    if (!m->biases) return fail(MOE_ERR_INVALID_ARG, "%s: affine biases is NULL", name);
  } else if (m->fmt == MOE_FMT_MXFP4) {
    if (m->bits != 4 || m->group != 32)
      return fail(MOE_ERR_UNSUPPORTED, "%s: mxfp4 needs bits=4 group=32", name);
    code = F_MX4;
  } else {
    return fail(MOE_ERR_UNSUPPORTED, "%s: unknown format %d", name, m->fmt);
  }
  if (n_in % m->group) return fail(MOE_ERR_INVALID_ARG, "%s: in=%d not a multiple of group", name, n_in);
  if (!m->q || !m->scales) return fail(MOE_ERR_INVALID_ARG, "%s: q/scales NULL", name);
  if (!aligned16(m->q) || !aligned16(m->scales) || (m->biases && !aligned16(m->biases)))
    return fail(MOE_ERR_INVALID_ARG, "%s: q/scales/biases must be 16-byte aligned", name);
  moe_status_t st = check_dev_ptr(m->q, name);
  if (st != MOE_OK) return st;
  out->q = m->q;
  out->scales = m->scales;
  out->biases = m->biases;
  out->fmt = code;
  out->group = m->group;
  out->n_in = n_in;
  out->n_out = n_out;
  out->wpr = n_in * m->bits / 32;
  out->gpr = n_in / m->group;
  return MOE_OK;
}

extern const StreamAttrFn kStreamAttrs[10];
extern const TcAttrFn kTcAttrs[10];
extern const UmAttrFn kUmAttrs[10];

template <typename WT>
void route_attrs() {
  cudaFuncSetAttribute(router_logits_small_kernel<8, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 8192 * 2);
  cudaFuncSetAttribute(route_small_fused_kernel<1, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(route_small_fused_kernel<8, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(route_small_fused_kernel<32, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(route_hash_fused_kernel<8, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  cudaFuncSetAttribute(route_hash_fused_kernel<32, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
}

struct DevInfo {
  int sms = 0;
  int ffn1_blocks = 0, ffn2_blocks = 0;
  int dec_blocks = 0;  // fused decode: co-resident CTAs (one per SM)
  int um_pairs[10] = {};  // TMA/TMEM FFN: resident CTA pairs per (stage, format) kernel
};
DevInfo g_dev[64];
std::atomic<int> g_dev_ready[64];

moe_status_t dev_info(DevInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  DevInfo& di = g_dev[dev];
  if (g_dev_ready[dev].load(std::memory_order_acquire) != 2) {
    int expect = 0;
    if (g_dev_ready[dev].compare_exchange_strong(expect, 1)) {
      cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
      cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 34 * 1024 * 4);
      cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 32 * 1024 * 4);
      route_attrs<float>();
      route_attrs<__nv_bfloat16>();
      for (StreamAttrFn f : kStreamAttrs) f();
      for (TcAttrFn f : kTcAttrs) f();
      for (int i = 0; i < 10; ++i) di.um_pairs[i] = kUmAttrs[i]();
      int b1 = 0, b2 = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b1, ffn_gemv_kernel<1, 4>, kFfnThreads, 0);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b2, ffn_gemv_kernel<2, 8>, kFfnThreads, 0);
      di.ffn1_blocks = std::max(1, b1);
      di.ffn2_blocks = std::max(1, b2);
      cudaFuncSetAttribute(ffn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemMax);
      int bd = 0;
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bd, ffn_decode_kernel, kDecThreads, kDecSmemMax);
      di.dec_blocks = std::min(bd, 1) * di.sms;
      cudaError_t le = cudaGetLastError();
      if (le != cudaSuccess) {
        g_dev_ready[dev].store(0);
        return cuda_fail(le, "device setup");
      }
      g_dev_ready[dev].store(2, std::memory_order_release);
    } else {
      while (g_dev_ready[dev].load(std::memory_order_acquire) == 1) {
      }
      if (g_dev_ready[dev].load(std::memory_order_acquire) != 2)
        return fail(MOE_ERR_CUDA, "device setup failed in another thread");
    }
  }
  *out = &di;
  return MOE_OK;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- launches
template <typename WT>
moe_status_t launch_route_t(const moe_dims_t& d, const void* x, const WT* rw, const float* rb,
                          const int* tok, const int* table, int* ids, float* wts, void* ws,
                          const WsLayout& L, cudaStream_t s) {
  int* err = &ws_at<WsHeader>(ws, L.hdr)->err;
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (d.hash_mode) {
    const int blocks = ceil_div(d.T * 32, 256);
    if (d.top_k <= 8)
      route_hash_kernel<8, WT><<<blocks, 256, 0, s>>>(xb, rw, tok, table, d.T, d.d_model, d.n_experts, d.top_k,
                                                  d.vocab, ids, wts, err);
    else
      route_hash_kernel<32, WT><<<blocks, 256, 0, s>>>(xb, rw, tok, table, d.T, d.d_model, d.n_experts, d.top_k,
                                                   d.vocab, ids, wts, err);
    MOE_CHECK_LAUNCH("route_hash_kernel");
    hook_mark(s, "route_hash");
    return MOE_OK;
  }
  float* logits = ws_at<float>(ws, L.logits);
  int split = 1;  // K halves of the logits GEMM (partials summed by the top-k)
  if (d.T <= 64) {
    dim3 grid(ceil_div(d.n_experts, kLogitWarps), ceil_div(d.T, 8));
    router_logits_small_kernel<8, WT><<<grid, kLogitWarps * 32, 8 * d.d_model * 2, s>>>(xb, rw, logits, d.T,
                                                                                      d.d_model, d.n_experts);
    MOE_CHECK_LAUNCH("router_logits_small_kernel");
    hook_mark(s, "router_logits");
  } else {
    // two K halves (more CTAs than SMs) when there is enough work
    split = d.T >= 256 && d.d_model % (2 * kLBK) == 0 ? 2 : 1;
    dim3 grid(ceil_div(d.n_experts, kLBN), ceil_div(d.T, kLBM), split);
    router_logits_tiled_kernel<WT><<<grid, 256, 0, s>>>(xb, rw, logits, d.T, d.d_model, d.n_experts);
    MOE_CHECK_LAUNCH("router_logits_tiled_kernel");
    hook_mark(s, "router_logits");
  }
  const int blocks = ceil_div(d.T * 32, 256);
  const float* L2 = split == 2 ? logits + (size_t)d.T * d.n_experts : nullptr;
  if (d.n_experts <= 32)
    topk_kernel<1><<<blocks, 256, 0, s>>>(logits, rb, d.T, d.n_experts, d.top_k, ids, wts, L2);
  else if (d.n_experts <= 256)
    topk_kernel<8><<<blocks, 256, 0, s>>>(logits, rb, d.T, d.n_experts, d.top_k, ids, wts, L2);
  else
    topk_kernel<32><<<blocks, 256, 0, s>>>(logits, rb, d.T, d.n_experts, d.top_k, ids, wts, L2);
  MOE_CHECK_LAUNCH("topk_kernel");
  hook_mark(s, "topk");
  return MOE_OK;
}

moe_status_t launch_route(const moe_dims_t& d, const void* x, const void* rw, const float* rb, const int* tok,
                          const int* table, int* ids, float* wts, void* ws, const WsLayout& L, cudaStream_t s) {
  if (d.router_dtype == 1)
    return launch_route_t(d, x, static_cast<const __nv_bfloat16*>(rw), rb, tok, table, ids, wts, ws, L, s);
  return launch_route_t(d, x, static_cast<const float*>(rw), rb, tok, table, ids, wts, ws, L, s);
}

// Routing and permutation in one launch for small batches.
bool fused_route_ok(const moe_dims_t& d) {
  return d.T <= kFusedMaxT && d.d_model <= 4096 && d.d_model % 64 == 0 && d.top_k <= 32;
}

template <typename WT>
moe_status_t launch_route_fused_t(const moe_dims_t& d, const void* x, const WT* rw, const float* rb, const int* tok,
                                const int* table, int* ids, float* wts, int* offsets, int* sorted, int* inv, void* ws,
                                const WsLayout& L, cudaStream_t s) {
  WsHeader* hdr = ws_at<WsHeader>(ws, L.hdr);
  int* active = ws_at<int>(ws, L.active);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  // tail scratch: top-k keys/scores/selected (2E + k floats), pair ids and flags (2 T*k ints)
  const size_t perm_smem = (size_t)(2 * d.n_experts + 32 + 2 * d.T * d.top_k) * sizeof(int);
  if (d.hash_mode) {
    const int blocks = d.T;  // one block (8 warps) per token
    if (d.top_k <= 8)
      route_hash_fused_kernel<8, WT><<<blocks, 256, perm_smem, s>>>(xb, rw, tok, table, d.T, d.d_model, d.n_experts,
                                                               d.top_k, d.vocab, ids, wts, offsets, sorted, inv,
                                                               active, &hdr->counters[1], &hdr->err);
    else
      route_hash_fused_kernel<32, WT><<<blocks, 256, perm_smem, s>>>(xb, rw, tok, table, d.T, d.d_model, d.n_experts,
                                                                d.top_k, d.vocab, ids, wts, offsets, sorted, inv,
                                                                active, &hdr->counters[1], &hdr->err);
    MOE_CHECK_LAUNCH("route_hash_fused_kernel");
    hook_mark(s, "route_hash_permute");
    return MOE_OK;
  }
  float* logits = ws_at<float>(ws, L.logits);
  const size_t smem = std::max((size_t)kFusedTB * d.d_model * 2, perm_smem);
  const int blocks = ceil_div(d.n_experts, 2);
  if (d.n_experts <= 32)
    route_small_fused_kernel<1, WT><<<blocks, 256, smem, s>>>(xb, rw, rb, d.T, d.d_model, d.n_experts, d.top_k, logits,
                                                          ids, wts, offsets, sorted, inv, active, &hdr->counters[0],
                                                          &hdr->err);
  else if (d.n_experts <= 256)
    route_small_fused_kernel<8, WT><<<blocks, 256, smem, s>>>(xb, rw, rb, d.T, d.d_model, d.n_experts, d.top_k, logits,
                                                          ids, wts, offsets, sorted, inv, active, &hdr->counters[0],
                                                          &hdr->err);
  else
    route_small_fused_kernel<32, WT><<<blocks, 256, smem, s>>>(xb, rw, rb, d.T, d.d_model, d.n_experts, d.top_k, logits,
                                                           ids, wts, offsets, sorted, inv, active, &hdr->counters[0],
                                                           &hdr->err);
  MOE_CHECK_LAUNCH("route_small_fused_kernel");
  hook_mark(s, "route_topk_permute");
  return MOE_OK;
}

moe_status_t launch_route_fused(const moe_dims_t& d, const void* x, const void* rw, const float* rb, const int* tok,
                                const int* table, int* ids, float* wts, int* offsets, int* sorted, int* inv, void* ws,
                                const WsLayout& L, cudaStream_t s) {
  if (d.router_dtype == 1)
    return launch_route_fused_t(d, x, static_cast<const __nv_bfloat16*>(rw), rb, tok, table, ids, wts, offsets,
                                sorted, inv, ws, L, s);
  return launch_route_fused_t(d, x, static_cast<const float*>(rw), rb, tok, table, ids, wts, offsets, sorted, inv,
                              ws, L, s);
}

moe_status_t launch_permute(const moe_dims_t& d, const int* ids, int* offsets, int* sorted, int* inv,
                            void* ws, const WsLayout& L, cudaStream_t s) {
  int* err = &ws_at<WsHeader>(ws, L.hdr)->err;
  int* active = ws_at<int>(ws, L.active);
  const int N = d.T * d.top_k;
  if (N > 4 * kPermThreads && L.pchunks) {
    // chunks of 1024 pairs on separate CTAs: counts, one scan, placement
    const int nb = ceil_div(N, kPermThreads);
    int* cnt = ws_at<int>(ws, L.pchunks);
    permute_count_kernel<<<nb, kPermThreads, d.n_experts * sizeof(int), s>>>(ids, N, d.n_experts, cnt, err);
    MOE_CHECK_LAUNCH("permute_count_kernel");
    hook_mark(s, "permute_count");
    permute_scan_kernel<<<1, kPermThreads, 0, s>>>(cnt, nb, d.n_experts, offsets, active);
    MOE_CHECK_LAUNCH("permute_scan_kernel");
    hook_mark(s, "permute_scan");
    permute_scatter_kernel<<<nb, kPermThreads, (size_t)32 * d.n_experts * sizeof(int), s>>>(
        ids, N, d.n_experts, cnt, sorted, inv);
    MOE_CHECK_LAUNCH("permute_scatter_kernel");
    hook_mark(s, "permute");
    return MOE_OK;
  }
  const size_t smem = (size_t)(2 + 32) * d.n_experts * sizeof(int);
  permute_kernel<<<1, kPermThreads, smem, s>>>(ids, N, d.n_experts, offsets, sorted, inv, active, err);
  MOE_CHECK_LAUNCH("permute_kernel");
  hook_mark(s, "permute");
  return MOE_OK;
}

// Streaming-kernel plan for one matrix: warps per row group and rows per
// tile, or ok = false when the matrix does not fit the kernel's constraints
// (n_in a multiple of 32*32*cpl with at most 8 warps per row, 16-byte row
// segments, a tile of at most one stage buffer).
struct StreamPlan {
  bool ok = false;
  int wpr = 1, rows = 0;
};

StreamPlan stream_plan(const QMatDev& A, int stage, int cpl, int max_units, int sms) {
  StreamPlan pl;
  const int C = A.n_in / 32;
  if (C % (32 * cpl)) return pl;
  const int wpr = C / (32 * cpl);
  if (wpr > kConsumerWarps || kConsumerWarps % wpr) return pl;
  const int M = stage == 1 ? 2 : 1;
  const bool mx = A.fmt == F_MX4;
  const int row_bytes = A.wpr * 4;
  const int sb_row = A.gpr * (mx ? 1 : 2);
  if (row_bytes % 16 || sb_row % 16) return pl;
  const int per_row = M * (row_bytes + sb_row * (mx ? 1 : 2));
  const int G = kConsumerWarps / wpr;
  int rpg = std::min(16, kStageBytes / (G * per_row));
  if (rpg < 1) return pl;
  // keep at least ~4 tiles per block so the contiguous ranges balance
  while (rpg > 1 && (long long)max_units * ((A.n_out + G * rpg - 1) / (G * rpg)) < 4LL * sms) rpg >>= 1;
  pl.ok = true;
  pl.wpr = wpr;
  pl.rows = G * rpg;
  return pl;
}

// Streaming launchers indexed by routed format code (F_A2..F_MX4).
const StreamLaunchFn kStreamLaunch[2][5] = {
    {launch_stream_s1_A2, launch_stream_s1_A3, launch_stream_s1_A4, launch_stream_s1_A8, launch_stream_s1_MX4},
    {launch_stream_s2_A2, launch_stream_s2_A3, launch_stream_s2_A4, launch_stream_s2_A8, launch_stream_s2_MX4}};
const StreamAttrFn kStreamAttrs[10] = {attrs_stream_s1_A2, attrs_stream_s1_A3, attrs_stream_s1_A4, attrs_stream_s1_A8,
                                       attrs_stream_s1_MX4, attrs_stream_s2_A2, attrs_stream_s2_A3, attrs_stream_s2_A4,
                                       attrs_stream_s2_A8, attrs_stream_s2_MX4};

// chunks per lane for a stage: as many as the activation registers allow
// (tokens per pass x chunks <= 4) and every matrix's width divides
int stream_cpl(int ntmax, int n_in_a, int n_in_b) {
  for (int cpl = 4 / ntmax; cpl >= 1; cpl >>= 1) {
    if ((n_in_a / 32) % (32 * cpl) == 0 && (n_in_b / 32) % (32 * cpl) == 0) return cpl;
  }
  return 0;
}

// Tensor-core launchers indexed by format code (F_A2..F_MX4).
const TcLaunchFn kTcLaunch[2][5] = {
    {launch_tc_s1_A2, launch_tc_s1_A3, launch_tc_s1_A4, launch_tc_s1_A8, launch_tc_s1_MX4},
    {launch_tc_s2_A2, launch_tc_s2_A3, launch_tc_s2_A4, launch_tc_s2_A8, launch_tc_s2_MX4}};
const TcAttrFn kTcAttrs[10] = {attrs_tc_s1_A2, attrs_tc_s1_A3, attrs_tc_s1_A4, attrs_tc_s1_A8, attrs_tc_s1_MX4,
                               attrs_tc_s2_A2, attrs_tc_s2_A3, attrs_tc_s2_A4, attrs_tc_s2_A8, attrs_tc_s2_MX4};

// Test hook of the calling thread (moe_test_stall_fused_wait): the next fused
// launches wait on a dependency count that nothing completes.
thread_local int g_stall_test = 0;

// Expert-FFN implementation choice of the calling thread (moe_set_ffn_path):
// one thread's setting never changes another thread's calls.
thread_local int g_ffn_path = MOE_FFN_AUTO;

// The tensor-core kernel tiles 128 output rows x 64 inputs.
bool tc_shape_ok(const QMatDev& A) { return A.n_out % kTcM == 0 && A.n_in % kTcK == 0; }

// Tensor-core path for the expert FFN: chosen from 4 tokens up (measured on
// B200: the weight-streaming GEMV wins at T = 1, the tensor-core kernels at
// T = 8 and 32 even with ~1-2 tokens per expert, since their dequantisation
// keeps pace with HBM) or when forced, if the workspace has its regions and
// every matrix has a supported shape.
bool use_tc(const moe_dims_t& d, const QMatDev& w1, const QMatDev& w2, const QMatDev* sh, const WsLayout& L) {
  const int mode = g_ffn_path;
  if (mode == MOE_FFN_GEMV || !L.tc) return false;
  if (!tc_shape_ok(w1) || !tc_shape_ok(w2) || (sh && (!tc_shape_ok(sh[0]) || !tc_shape_ok(sh[2])))) return false;
  if (mode == MOE_FFN_TENSOR_CORE) return true;
  return d.T >= 4;
}

// TMA/TMEM kernels indexed by format code (no 3-bit instance).
const UmLaunchFn kUmLaunch[2][5] = {
    {launch_um_s1_A2, launch_um_s1_A3, launch_um_s1_A4, launch_um_s1_A8, launch_um_s1_MX4},
    {launch_um_s2_A2, launch_um_s2_A3, launch_um_s2_A4, launch_um_s2_A8, launch_um_s2_MX4}};
const UmAttrFn kUmAttrs[10] = {attrs_um_s1_A2, attrs_um_s1_A3, attrs_um_s1_A4, attrs_um_s1_A8, attrs_um_s1_MX4,
                               attrs_um_s2_A2, attrs_um_s2_A3, attrs_um_s2_A4, attrs_um_s2_A8, attrs_um_s2_MX4};

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaGetLastError();
  });
  return g_encode;
}

// 2D tensor map: dim0 (contiguous) x dim1 rows, row stride in bytes, box b0 x b1.
moe_status_t tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t dim0, uint64_t dim1,
                     uint64_t stride, uint32_t b0, uint32_t b1, bool swizzle128) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {dim0, dim1};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOE_OK;
}

// Shapes the TMA/TMEM kernel takes: any packed format, rows of a multiple of
// 16 bytes, scale rows of a multiple of 16 bytes (the TMA stride rule), 128
// features (stage 1) or 256 output rows (stage 2) per pair item, an even number of
// 128-input stages.
bool um_ok(const QMatDev& Q, int stage) {
  if (Q.n_in % (2 * kUmK) || Q.n_out % (stage == 1 ? kUmRowsS1 : kUmRowsS2)) return false;
  // more dequant groups than two: every raw slot of a row must be whole
  // (2-bit slots hold 512 inputs), so that the groups reading it are fixed
  if (kUmGroups > 2 && Q.n_in % (Q.fmt == F_A2 ? 512 : 256)) return false;
  if ((Q.wpr * 4) % 16) return false;
  if (Q.group != 32 && Q.group != 64 && Q.group != 128) return false;
  return Q.fmt == F_MX4 ? Q.gpr % 16 == 0 : (Q.gpr * 2) % 16 == 0;
}

// Packed-code, scale and bias maps of matrix Q (E experts) for slot m.
moe_status_t um_weight_maps(UmParams& p, int m, const QMatDev& Q, int E, int rows_per_box) {
  const uint64_t rows = (uint64_t)E * Q.n_out;
  // 3-bit codes: 96-byte boxes (256 inputs) without swizzle; else 128-byte swizzled boxes
  const bool b3 = Q.fmt == F_A3;
  moe_status_t st = tmap_2d(&p.q_map[m], CU_TENSOR_MAP_DATA_TYPE_UINT8, Q.q, (uint64_t)Q.wpr * 4, rows,
                            (uint64_t)Q.wpr * 4, b3 ? 96 : 128, rows_per_box, !b3);
  if (st != MOE_OK) return st;
  if (Q.fmt == F_MX4)
    return tmap_2d(&p.s_map[m], CU_TENSOR_MAP_DATA_TYPE_UINT8, Q.scales, Q.gpr, rows, Q.gpr, 16, rows_per_box, false);
  st = tmap_2d(&p.s_map[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q.scales, Q.gpr, rows, (uint64_t)Q.gpr * 2, 8,
               rows_per_box, false);
  if (st != MOE_OK) return st;
  return tmap_2d(&p.z_map[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q.biases, Q.gpr, rows, (uint64_t)Q.gpr * 2, 8,
                 rows_per_box, false);
}

moe_status_t launch_ffn_tc(const moe_dims_t& d, const void* x, const int* offsets, const int* sorted,
                           const QMatDev& w1, const QMatDev& w3, const QMatDev& w2, const QMatDev* sh,
                           float* y, int ld_y, void* ws, const WsLayout& L, cudaStream_t s, const DevInfo& di,
                           const int* valid) {
  const int Tk = d.T * d.top_k;
  const int P = Tk + (sh ? d.T : 0);
  int* err = &ws_at<WsHeader>(ws, L.hdr)->err;
  __half* xs = ws_at<__half>(ws, L.x16);
  __half* h16 = ws_at<__half>(ws, L.h);
  const int ld_h = f_max_of(d);
  int* n_tiles = ws_at<int>(ws, L.ntiles);
  {
    const size_t n8 = (size_t)P * d.d_model / 8;
    const int grid = (int)std::min<size_t>((n8 + 255) / 256, (size_t)di.sms * 8);
    tc_gather_f16_kernel<<<std::max(grid, 1), 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(x), sorted,
                                                           d.top_k, Tk, d.T, d.d_model, sh ? 1 : 0, xs, err, valid);
    MOE_CHECK_LAUNCH("tc_gather_f16_kernel");
    hook_mark(s, "gather_f16");
    tc_plan_kernel<<<1, 1024, 0, s>>>(offsets, d.n_experts, kTcN, ws_at<int4>(ws, L.tiles), n_tiles, kUmN,
                                      ws_at<int4>(ws, L.tiles2), n_tiles + 1, valid);
    MOE_CHECK_LAUNCH("tc_plan_kernel");
    hook_mark(s, "tile_plan");
  }
  // One launch of stage `stage` for the routed experts (shared = nullptr) or
  // the shared expert: the TMA/TMEM kernel when the shapes allow, else the
  // per-thread-copy kernel.
  auto run = [&](int stage, const QMatDev& a0, const QMatDev& a1, bool shared, const char* label) -> moe_status_t {
    const int pos_base = shared ? Tk : 0;
    const int E = shared ? 1 : d.n_experts;
    const int um_pairs = di.um_pairs[(stage - 1) * 5 + a0.fmt];
    if (um_pairs > 0 && um_ok(a0, stage) && um_ok(a1, stage)) {
      UmParams q{};
      moe_status_t st = MOE_OK;
      for (int h = 0; h < 4 && st == MOE_OK; ++h) {  // half-tile token boxes of 16, 32, 64, 96 rows
        const uint32_t box_rows = h == 0 ? 16u : h == 1 ? 32u : h == 2 ? 64u : 96u;
        if (stage == 1)
          st = tmap_2d(&q.b_map[h], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xs, d.d_model, (uint64_t)P,
                       (uint64_t)d.d_model * 2, kUmKB, box_rows, true);
        else
          st = tmap_2d(&q.b_map[h], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, h16, a0.n_in, (uint64_t)P, (uint64_t)ld_h * 2,
                       kUmKB, box_rows, true);
      }
      if (st != MOE_OK) return st;
      if ((st = um_weight_maps(q, 0, a0, E, stage == 1 ? 64 : 128)) != MOE_OK) return st;
      if (stage == 1 && (st = um_weight_maps(q, 1, a1, E, 64)) != MOE_OK) return st;
      q.hout = h16;
      q.yout = y;
      q.ld_h = ld_h;
      q.ld_y = ld_y;
      q.n_in = a0.n_in;
      q.n_out = a0.n_out;
      q.group = a0.group;
      q.row_bytes = a0.wpr * 4;
      q.gpr = a0.gpr;
      q.lg_group = a0.group == 32 ? 5 : a0.group == 64 ? 6 : 7;
      q.T = d.T;
      q.shared = shared ? 1 : 0;
      q.tiles = ws_at<int4>(ws, L.tiles2);
      q.n_tiles = n_tiles + 1;
      q.pos_base = pos_base;
      q.err = err;
      const int rows_per_item = stage == 1 ? kUmRowsS1 : kUmRowsS2;
      const int pairs = shared ? std::min(um_pairs, (d.T + kUmN - 1) / kUmN * (a0.n_out / rows_per_item)) : um_pairs;
      if (!kUmLaunch[stage - 1][a0.fmt](q, pairs, s)) return fail(MOE_ERR_UNSUPPORTED, "no TMA/TMEM kernel");
    } else {
      TcParams q{};
      q.x16 = xs;
      q.hin = h16;
      q.ld_in = ld_h;
      q.hout = h16;
      q.ld_h = ld_h;
      q.yout = y;
      q.ld_y = ld_y;
      q.T = d.T;
      q.k = d.top_k;
      q.a0 = a0;
      q.a1 = a1;
      q.sorted_rows = shared ? nullptr : sorted;
      q.tiles = ws_at<int4>(ws, L.tiles);
      q.n_tiles = n_tiles;
      q.pos_base = pos_base;
      q.err = err;
      const int grid = shared ? std::min(di.sms, (d.T + kTcN - 1) / kTcN * (a0.n_out / kTcM)) : di.sms;
      if (!kTcLaunch[stage - 1][a0.fmt](q, grid, s)) return fail(MOE_ERR_UNSUPPORTED, "no tensor-core kernel");
    }
    MOE_CHECK_LAUNCH(label);
    hook_mark(s, label);
    return MOE_OK;
  };
  moe_status_t st;
  if ((st = run(1, w1, w3, false, "ffn_w13_swiglu")) != MOE_OK) return st;
  if (sh && (st = run(1, sh[0], sh[1], true, "ffn_w13_swiglu_shared")) != MOE_OK) return st;
  if ((st = run(2, w2, w2, false, "ffn_w2")) != MOE_OK) return st;
  if (sh && (st = run(2, sh[2], sh[2], true, "ffn_w2_shared")) != MOE_OK) return st;
  return MOE_OK;
}

// Stage 1 + stage 2 of the expert FFN (routed pairs, optional shared expert).
// `valid`: the flag the permutation check wrote for a caller-supplied
// permutation (NULL for the library's own).
moe_status_t launch_ffn(const moe_dims_t& d, const void* x, const int* offsets, const int* sorted,
                        const QMatDev& w1, const QMatDev& w3, const QMatDev& w2, const QMatDev* sh,
                        float* y, int ld_y, void* ws, const WsLayout& L, cudaStream_t s,
                        const int* valid = nullptr) {
  DevInfo* di = nullptr;
  moe_status_t st = dev_info(&di);
  if (st != MOE_OK) return st;
  if (use_tc(d, w1, w2, sh, L))
    return launch_ffn_tc(d, x, offsets, sorted, w1, w3, w2, sh, y, ld_y, ws, L, s, *di, valid);
  const int Tk = d.T * d.top_k;
  const int max_active = std::min(d.n_experts, Tk);
  float* h = ws_at<float>(ws, L.h);
  const int ld_h = f_max_of(d);
  FfnParams p{};
  p.x = reinterpret_cast<const __nv_bfloat16*>(x);
  p.T = d.T;
  p.k = d.top_k;
  p.offsets = offsets;
  p.sorted_rows = sorted;
  p.active = ws_at<int>(ws, L.active);
  p.err = &ws_at<WsHeader>(ws, L.hdr)->err;
  p.shared_pos0 = Tk;
  p.has_shared = sh != nullptr;
  // tokens per pass: experts rarely see more than two tokens at decode sizes
  const int ntmax = d.T >= 2 ? 2 : 1;
  const int fs = sh ? d.d_ff_shared : d.d_ff;
  const int cpl1 = stream_cpl(ntmax, d.d_model, d.d_model);
  const int cpl2 = stream_cpl(ntmax, d.d_ff, fs);
  StreamPlan r1, r2, s1, s2;
  if (cpl1 && cpl2) {
    r1 = stream_plan(w1, 1, cpl1, max_active, di->sms);
    r2 = stream_plan(w2, 2, cpl2, max_active, di->sms);
    s1 = sh ? stream_plan(sh[0], 1, cpl1, 1, di->sms) : r1;
    s2 = sh ? stream_plan(sh[2], 2, cpl2, 1, di->sms) : r2;
  }
  // the streaming kernels compile the routed format plus the 8-bit shared path
  const bool fmt_ok = !sh || ((sh[0].fmt == w1.fmt || sh[0].fmt == F_A8) && (sh[2].fmt == w2.fmt || sh[2].fmt == F_A8));
  if (fmt_ok && cpl1 && cpl2 && r1.ok && r2.ok && s1.ok && s2.ok) {
    StreamParams q{};
    q.x = p.x;
    q.T = d.T;
    q.k = d.top_k;
    q.offsets = offsets;
    q.sorted_rows = sorted;
    q.active = p.active;
    q.err = p.err;
    q.shared_pos0 = Tk;
    q.has_shared = sh != nullptr;
    q.out = h;
    q.ld_out = ld_h;
    q.ra = w1;
    q.rb = w3;
    q.r_rows = r1.rows;
    q.r_wpr = r1.wpr;
    q.sa = sh ? sh[0] : w1;
    q.sb = sh ? sh[1] : w3;
    q.s_rows = s1.rows;
    q.s_wpr = s1.wpr;
    if (!kStreamLaunch[0][w1.fmt](ntmax, cpl1, di->sms, s, q)) return fail(MOE_ERR_UNSUPPORTED, "no streaming kernel");
    MOE_CHECK_LAUNCH("ffn_stream_kernel<1>");
    hook_mark(s, "ffn_w13_swiglu");
    q.hin = h;
    q.ld_in = ld_h;
    q.out = y;
    q.ld_out = ld_y;
    q.ra = w2;
    q.rb = w2;
    q.r_rows = r2.rows;
    q.r_wpr = r2.wpr;
    q.sa = sh ? sh[2] : w2;
    q.sb = q.sa;
    q.s_rows = s2.rows;
    q.s_wpr = s2.wpr;
    if (!kStreamLaunch[1][w2.fmt](ntmax, cpl2, di->sms, s, q)) return fail(MOE_ERR_UNSUPPORTED, "no streaming kernel");
    MOE_CHECK_LAUNCH("ffn_stream_kernel<2>");
    hook_mark(s, "ffn_w2");
    return MOE_OK;
  }
  // stage 1: h = silu(W1 x) * (W3 x)
  {
    FfnParams q = p;
    q.out = h;
    q.ld_out = ld_h;
    q.ra = w1;
    q.rb = w3;
    const int rb_r = (kFfnThreads / (d.d_model / 32)) * 4;
    q.routed_items_per_expert = ceil_div(d.d_ff, rb_r);
    if (sh) {
      q.sa = sh[0];
      q.sb = sh[1];
      q.shared_items = ceil_div(d.d_ff_shared, rb_r);
    }
    const int items = max_active * q.routed_items_per_expert + (sh ? q.shared_items : 0);
    const int grid = std::max(1, std::min(items, di->sms * di->ffn1_blocks));
    ffn_gemv_kernel<1, 4><<<grid, kFfnThreads, 0, s>>>(q);
    MOE_CHECK_LAUNCH("ffn_gemv_kernel<1>");
    hook_mark(s, "ffn_w13_swiglu");
  }
  // stage 2: y = W2 h
  {
    FfnParams q = p;
    q.hin = h;
    q.ld_in = ld_h;
    q.out = y;
    q.ld_out = ld_y;
    q.ra = w2;
    q.routed_items_per_expert = ceil_div(d.d_model, (kFfnThreads / (d.d_ff / 32)) * 8);
    if (sh) {
      q.sa = sh[2];
      q.shared_items = ceil_div(d.d_model, (kFfnThreads / (d.d_ff_shared / 32)) * 8);
    }
    const int items = max_active * q.routed_items_per_expert + (sh ? q.shared_items : 0);
    const int grid = std::max(1, std::min(items, di->sms * di->ffn2_blocks));
    ffn_gemv_kernel<2, 8><<<grid, kFfnThreads, 0, s>>>(q);
    MOE_CHECK_LAUNCH("ffn_gemv_kernel<2>");
    hook_mark(s, "ffn_w2");
  }
  return MOE_OK;
}

// ---------------------------------------------------------------- fused small-batch layer
// Stage geometry of a packed matrix in the fused kernel: up to 1024 code
// bytes of every row per stage (3-bit: 768), as one chunk-major 3-D TMA box
// of 16 (W1, W3) or 32 (W2) rows; 8 consumer slices of whole 64-input blocks.
bool dec_mat(const QMatDev& Q, bool w2, DecMat* m) {
  m->fmt = Q.fmt;
  m->group = Q.group;
  m->n_out = Q.n_out;
  m->n_in = Q.n_in;
  const int bits = Q.fmt == F_A2 ? 2 : Q.fmt == F_A3 ? 3 : Q.fmt == F_A8 ? 8 : 4;
  const int row_bytes = Q.wpr * 4;
  m->R = w2 ? kDecR2 : kDecR1;
  m->lb = Q.fmt == F_A3 ? 96 : 128;
  m->seg = std::min(row_bytes, Q.fmt == F_A3 ? 768 : kDecMaxSeg);
  if (row_bytes <= 0 || m->seg % m->lb || row_bytes % m->seg) return false;
  if (row_bytes * 8 != Q.n_in * bits) return false;  // rows packed without padding
  m->nch = row_bytes / m->seg;
  m->K = m->seg * 8 / bits;
  if (m->K % (64 * kDecNkq)) return false;  // input slices of whole 64-input blocks
  m->nbw = m->K / (64 * kDecNkq);
  if (!dec_supported(Q.fmt, Q.group, m->nbw)) return false;  // the instantiated (format, group, slice) shapes
  if (m->K % Q.group) return false;
  m->sK = m->K / Q.group;
  const int esz = Q.fmt == F_MX4 ? 1 : 2;
  const int sbytes = m->sK * esz;
  if (sbytes % 16) return false;          // TMA box of scales
  if ((Q.gpr * esz) % 16) return false;   // TMA row stride of scales
  // scale rows land at an odd multiple of 16 bytes apart: the 8 rows a fold reads hit distinct banks
  m->spitch = (sbytes / 16) % 2 ? sbytes : sbytes + 16;
  if (m->spitch / esz > 256) return false;
  if (Q.n_out % kDecRows) return false;
  m->ptok = Q.n_in * 2 + 64;        // = 64 mod 128: token j and j+1 of a B load use different banks
  m->sxtok = Q.n_in / 64 * 16 + 16;  // = 16 mod 128: the four tokens of a record load use different banks
  return true;
}

// Shared-memory plan of one launch: ring slots, plane buffers.  False when
// the shapes do not fit the fused kernel.
bool dec_plan(const moe_dims_t& d, const QMatDev& w1, const QMatDev& w3, const QMatDev& w2, const QMatDev* sh,
              DecParams* p, size_t* smem) {
  if (d.T < 1 || d.T > kDecMaxT || d.T * d.top_k > kDecMaxPairs || d.n_experts > kDecMaxE) return false;
  // d_model a multiple of 256: the routing passes take 256-input chunks (8 inputs per lane)
  if (d.d_model % 256 || d.d_ff % kDecRows || (sh && d.d_ff_shared % kDecRows)) return false;
  const QMatDev* mats[6] = {&w1, &w3, &w2, sh ? &sh[0] : &w1, sh ? &sh[1] : &w3, sh ? &sh[2] : &w2};
  DecMat m[6];
  for (int i = 0; i < 6; ++i)
    if (!dec_mat(*mats[i], i % 3 == 2, &m[i])) return false;
  for (int b = 0; b < 6; b += 3)  // W1 and W3 of an expert stream side by side
    if (m[b].fmt != m[b + 1].fmt || m[b].group != m[b + 1].group || m[b].seg != m[b + 1].seg ||
        m[b].n_in != m[b + 1].n_in || m[b].n_out != m[b + 1].n_out)
      return false;
  const int ntmax = std::min(kDecMaxTok, d.hash_mode ? d.T * d.top_k : d.T);
  int pst = 0, sxs = 0, sc = 0;
  for (int i = 0; i < 6; ++i) {
    pst = std::max(pst, m[i].ptok);
    sxs = std::max(sxs, m[i].sxtok);
    const int nsb = m[i].fmt == F_MX4 ? 1 : 2;
    sc = std::max(sc, (i % 3 == 2 ? 1 : 2) * nsb * m[i].R * m[i].spitch);
  }
  const int sx_off = ntmax * pst;
  const int pbuf = (sx_off + ntmax * sxs + 127) / 128 * 128;
  const int slot_bytes = kDecCodeBytes + (sc + 1023) / 1024 * 1024;
  const long avail = (long)kDecSmemMax - 1024 - kDecFixedBytes - 2L * pbuf;
  const int nslot = (int)std::min<long>(kDecSlotCap, avail / slot_bytes);
  if (nslot < 2) return false;
  if (p) {
    for (int i = 0; i < 6; ++i) p->m[i] = m[i];
    p->nslot = nslot;
    p->slot_bytes = slot_bytes;
    p->pbuf = pbuf;
    p->sx_off = sx_off;
    p->ntmax = ntmax;
  }
  if (smem) *smem = 1024 + (size_t)nslot * slot_bytes + 2 * (size_t)pbuf + kDecFixedBytes;
  return true;
}

bool dec_eligible(const moe_dims_t& d, const QMatDev& w1, const QMatDev& w3, const QMatDev& w2, const QMatDev* sh) {
  return dec_plan(d, w1, w3, w2, sh, nullptr, nullptr);
}

bool use_dec(const moe_dims_t& d, const QMatDev& w1, const QMatDev& w3, const QMatDev& w2, const QMatDev* sh) {
  const int mode = g_ffn_path;
  if (mode == MOE_FFN_GEMV || mode == MOE_FFN_TENSOR_CORE) return false;
  return dec_eligible(d, w1, w3, w2, sh);
}

// Codes as a chunk-major 3-D view: (line of lb bytes, row, line index within
// the row), so a box of R rows x C lines lands as [line][row][lb].
moe_status_t tmap_rows_3d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t row_bytes, uint32_t lb,
                          uint32_t R, uint32_t C) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {lb, rows, row_bytes / lb};
  const cuuint64_t strides[2] = {row_bytes, lb};
  const cuuint32_t box[3] = {lb, R, C};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, lb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (3-D rows) failed (%d)", (int)r);
  return MOE_OK;
}

moe_status_t dec_maps(DecParams& p, int i, const QMatDev& Q, int E) {
  const DecMat& m = p.m[i];
  const uint64_t rows = (uint64_t)E * Q.n_out;
  moe_status_t st = tmap_rows_3d(&p.map[i], Q.q, rows, (uint64_t)Q.wpr * 4, m.lb, m.R, m.seg / m.lb);
  if (st != MOE_OK) return st;
  // scale boxes are spitch bytes wide: the stage's scales plus padding (the
  // next stage's scales, or zero fill past the row end)
  if (Q.fmt == F_MX4)
    return tmap_2d(&p.smap[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, Q.scales, Q.gpr, rows, Q.gpr, m.spitch, m.R, false);
  st = tmap_2d(&p.smap[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q.scales, Q.gpr, rows, (uint64_t)Q.gpr * 2,
               m.spitch / 2, m.R, false);
  if (st != MOE_OK) return st;
  return tmap_2d(&p.bmap[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q.biases, Q.gpr, rows, (uint64_t)Q.gpr * 2,
                 m.spitch / 2, m.R, false);
}

// An expert slice of the layer (expert parallelism): experts [e_begin,
// e_end), the shared expert when with_shared, fp32 partial to out_f32.
struct DecPart {
  int e_begin, e_end, with_shared;
  float* out_f32;
};

moe_status_t launch_decode_fused(const moe_dims_t& d, const void* x, const int32_t* token_ids, const void* router_w,
                                 const float* router_b, const int32_t* tid2eid, const QMatDev& q1, const QMatDev& q3,
                                 const QMatDev& q2, const QMatDev* qs, void* out, int32_t* ids_out, float* w_out,
                                 void* ws, const WsLayout& L, cudaStream_t s, const DevInfo& di, const DecPart& part) {
  DecParams p{};
  size_t smem = 0;
  if (!dec_plan(d, q1, q3, q2, qs, &p, &smem)) return fail(MOE_ERR_UNSUPPORTED, "shapes outside the fused kernel");
  const QMatDev* mats[6] = {&q1, &q3, &q2, qs ? &qs[0] : &q1, qs ? &qs[1] : &q3, qs ? &qs[2] : &q2};
  for (int i = 0; i < 6; ++i) {
    moe_status_t st = dec_maps(p, i, *mats[i], (i < 3 || !qs) ? d.n_experts : 1);
    if (st != MOE_OK) return st;
  }
  p.x = reinterpret_cast<const __nv_bfloat16*>(x);
  p.router_w = router_w;
  p.router_b = router_b;
  p.token_ids = token_ids;
  p.tid2eid = tid2eid;
  p.router_bf16 = d.router_dtype == 1;
  p.T = d.T;
  p.d = d.d_model;
  p.f = d.d_ff;
  p.fs = qs ? d.d_ff_shared : 0;
  p.E = d.n_experts;
  p.k = d.top_k;
  p.hash = d.hash_mode;
  p.vocab = d.vocab;
  p.has_shared = qs != nullptr;
  p.logits = ws_at<float>(ws, L.logits);
  p.hids = ws_at<int>(ws, L.ids);
  p.hw = ws_at<float>(ws, L.wts);
  p.xplanes = ws_at<uint8_t>(ws, L.dxp);
  p.xsx = ws_at<float4>(ws, L.dxsx);
  p.hplanes = ws_at<uint8_t>(ws, L.dhp);
  p.hsx = ws_at<float4>(ws, L.dhsx);
  p.y = ws_at<float>(ws, L.y);
  p.cnt_h = ws_at<int>(ws, L.dcnth);
  p.sync = ws_at<int>(ws, L.dsync);
  p.err = &ws_at<WsHeader>(ws, L.hdr)->err;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.ids_out = ids_out;
  p.w_out = w_out;
  p.stall_test = g_stall_test;
  p.e_begin = part.e_begin;
  p.e_end = part.e_end;
  p.with_shared = part.with_shared;
  p.out_f32 = part.out_f32;
  p.G = di.dec_blocks;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the kernel's CTAs wait on one another
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.G);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaLaunchKernelEx(&cfg, ffn_decode_kernel, p);
  if (le != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(le, "ffn_decode_kernel");
  }
  MOE_CHECK_LAUNCH("ffn_decode_kernel");
  hook_mark(s, "decode_fused");
  return MOE_OK;
}

moe_status_t launch_combine(const moe_dims_t& d, const float* y, const int* inv, const float* w,
                            const float* y_shared, void* out, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // combine_kernel waits for y itself
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ceil_div(d.d_model / 4, 256), std::min(d.T, 65535));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaLaunchKernelEx(&cfg, combine_kernel, y, inv, w, y_shared,
                                      reinterpret_cast<__nv_bfloat16*>(out), d.T, d.top_k, d.d_model);
  if (le != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(le, "combine_kernel");
  }
  MOE_CHECK_LAUNCH("combine_kernel");
  hook_mark(s, "combine");
  return MOE_OK;
}

moe_status_t check_ws(const moe_dims_t& d, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = layout_of(d);
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (ws_bytes < L->total)
    return fail(MOE_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, L->total);
  return check_dev_ptr(ws, "workspace");
}

moe_status_t check_route_args(const moe_dims_t& d, const void* x, const void* rw, const int* tok,
                              const int* table) {
  moe_status_t st = check_dev_ptr(x, "x");
  if (st != MOE_OK) return st;
  if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (d.hash_mode) {
    if ((st = check_dev_ptr(tok, "token_ids")) != MOE_OK) return st;
    if ((st = check_dev_ptr(table, "tid2eid")) != MOE_OK) return st;
    if (rw && !aligned16(rw)) return fail(MOE_ERR_INVALID_ARG, "router_w must be 16-byte aligned");
  } else {
    if ((st = check_dev_ptr(rw, "router_w")) != MOE_OK) return st;
    if (!aligned16(rw)) return fail(MOE_ERR_INVALID_ARG, "router_w must be 16-byte aligned");
  }
  return MOE_OK;
}

moe_status_t forward_launches(const moe_dims_t& d, const void* x, const int32_t* token_ids, const void* router_w,
                              const float* router_b, const int32_t* tid2eid, const QMatDev& q1, const QMatDev& q3,
                              const QMatDev& q2, const QMatDev* qs, void* out, int32_t* topk_ids_out,
                              float* topk_w_out, void* ws, const WsLayout& L, cudaStream_t s);

}  // namespace

// ======================================================================= ABI
extern "C" {

size_t moe_workspace_size(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  return layout_of(*dims).total;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_INPUT: return "out-of-range routing input on device";
  }
  return "unknown status";
}

const char* moe_last_error_detail(void) { return g_detail; }

int32_t moe_set_ffn_path(int32_t path) {
  if (path != MOE_FFN_AUTO && path != MOE_FFN_GEMV && path != MOE_FFN_TENSOR_CORE && path != MOE_FFN_DECODE_FUSED)
    return -1;
  const int prev = g_ffn_path;
  g_ffn_path = path;
  return prev;
}

moe_status_t moe_set_timing_events(void* const* events, int32_t n_events) {
  g_hook = TimingHook{};
  if (events && n_events > 0) {
    g_hook.events = events;
    g_hook.n = std::min<int32_t>(n_events, 33);
  }
  return MOE_OK;
}

int32_t moe_timing_count(void) { return g_hook_count; }

const char* moe_timing_label(int32_t i) {
  if (i < 0 || i >= 32 || i + 1 >= g_hook_count || !g_hook_labels[i]) return "";
  return g_hook_labels[i];
}

moe_status_t moe_route(const moe_dims_t* dims, const void* x, const void* router_w, const float* router_b,
                       const int32_t* token_ids, const int32_t* tid2eid, int32_t* topk_ids, float* topk_w,
                       void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  WsLayout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = check_route_args(d, x, router_w, token_ids, tid2eid)) != MOE_OK) return st;
  if ((st = check_dev_ptr(topk_ids, "topk_ids")) != MOE_OK) return st;
  if ((st = check_dev_ptr(topk_w, "topk_w")) != MOE_OK) return st;
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  return launch_route(d, x, router_w, router_b, token_ids, tid2eid, topk_ids, topk_w, ws, L,
                      reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(const moe_dims_t* dims, const int32_t* topk_ids, int32_t* expert_offsets,
                         int32_t* sorted_rows, int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  WsLayout L;
  if ((st = check_ws(*dims, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = check_dev_ptr(topk_ids, "topk_ids")) != MOE_OK) return st;
  if ((st = check_dev_ptr(expert_offsets, "expert_offsets")) != MOE_OK) return st;
  if ((st = check_dev_ptr(sorted_rows, "sorted_rows")) != MOE_OK) return st;
  if ((st = check_dev_ptr(inv, "inv")) != MOE_OK) return st;
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  return launch_permute(*dims, topk_ids, expert_offsets, sorted_rows, inv, ws, L,
                        reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn(const moe_dims_t* dims, const void* x, const int32_t* expert_offsets,
                            const int32_t* sorted_rows, const moe_qmat_t* w1, const moe_qmat_t* w3,
                            const moe_qmat_t* w2, float* y, void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  WsLayout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = check_dev_ptr(x, "x")) != MOE_OK) return st;
  if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if ((st = check_dev_ptr(expert_offsets, "expert_offsets")) != MOE_OK) return st;
  if ((st = check_dev_ptr(sorted_rows, "sorted_rows")) != MOE_OK) return st;
  if ((st = check_dev_ptr(y, "y")) != MOE_OK) return st;
  if (!aligned16(y)) return fail(MOE_ERR_INVALID_ARG, "y must be 16-byte aligned");
  QMatDev q1, q3, q2;
  if ((st = check_qmat(w1, d.d_model, "w1", &q1, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w3, d.d_model, "w3", &q3, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w2, d.d_ff, "w2", &q2, d.d_model)) != MOE_OK) return st;
  if (q1.fmt != q3.fmt || q1.group != q3.group)
    return fail(MOE_ERR_UNSUPPORTED, "w1 and w3 must share one format");
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = ws_at<WsHeader>(ws, L.hdr);
  active_from_offsets_kernel<<<1, kPermThreads, 0, s>>>(expert_offsets, d.n_experts, d.T * d.top_k, sorted_rows,
                                                        ws_at<int>(ws, L.active), &hdr->err, &hdr->counters[2]);
  MOE_CHECK_LAUNCH("active_from_offsets_kernel");
  moe_dims_t dn = d;
  dn.d_ff_shared = 0;
  return launch_ffn(dn, x, expert_offsets, sorted_rows, q1, q3, q2, nullptr, y, d.d_model, ws, L, s,
                    &hdr->counters[2]);
}

moe_status_t moe_combine(const moe_dims_t* dims, const float* y, const int32_t* inv, const float* topk_w,
                         const float* y_shared, void* out, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  if ((st = check_dev_ptr(y, "y")) != MOE_OK) return st;
  if ((st = check_dev_ptr(inv, "inv")) != MOE_OK) return st;
  if ((st = check_dev_ptr(topk_w, "topk_w")) != MOE_OK) return st;
  if ((st = check_dev_ptr(out, "out")) != MOE_OK) return st;
  if (y_shared && (st = check_dev_ptr(y_shared, "y_shared")) != MOE_OK) return st;
  if (!aligned16(y) || !aligned16(out) || (y_shared && !aligned16(y_shared)))
    return fail(MOE_ERR_INVALID_ARG, "y, y_shared and out must be 16-byte aligned");
  return launch_combine(*dims, y, inv, topk_w, y_shared, out, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
// The whole layer; `out_mapped`: `out` is the device address of page-locked
// host memory (moe_forward_host's direct output), not device memory.
moe_status_t forward_impl(const moe_dims_t* dims, const void* x, const int32_t* token_ids, const void* router_w,
                          const float* router_b, const int32_t* tid2eid, const moe_qmat_t* w1,
                          const moe_qmat_t* w3, const moe_qmat_t* w2, const moe_qmat_t* shared, void* out,
                          bool out_mapped, int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                          void* stream) {
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  WsLayout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = check_route_args(d, x, router_w, token_ids, tid2eid)) != MOE_OK) return st;
  if (!out_mapped && (st = check_dev_ptr(out, "out")) != MOE_OK) return st;
  if (!aligned16(out)) return fail(MOE_ERR_INVALID_ARG, "out must be 16-byte aligned");
  QMatDev q1, q3, q2, qs[3];
  if ((st = check_qmat(w1, d.d_model, "w1", &q1, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w3, d.d_model, "w3", &q3, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w2, d.d_ff, "w2", &q2, d.d_model)) != MOE_OK) return st;
  if (q1.fmt != q3.fmt || q1.group != q3.group)
    return fail(MOE_ERR_UNSUPPORTED, "w1 and w3 must share one format");
  if (d.d_ff_shared > 0) {
    if (!shared) return fail(MOE_ERR_INVALID_ARG, "d_ff_shared > 0 but shared is NULL");
    if ((st = check_qmat(&shared[0], d.d_model, "shared w1", &qs[0], d.d_ff_shared)) != MOE_OK) return st;
    if ((st = check_qmat(&shared[1], d.d_model, "shared w3", &qs[1], d.d_ff_shared)) != MOE_OK) return st;
    if ((st = check_qmat(&shared[2], d.d_ff_shared, "shared w2", &qs[2], d.d_model)) != MOE_OK) return st;
    if (qs[0].fmt != qs[1].fmt || qs[0].group != qs[1].group)
      return fail(MOE_ERR_UNSUPPORTED, "shared w1 and w3 must share one format");
  }
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = forward_launches(d, x, token_ids, router_w, router_b, tid2eid, q1, q3, q2, qs, out, topk_ids_out, topk_w_out,
                        ws, L, s);
  hook_end();
  return st;
}
}  // namespace

moe_status_t moe_forward(const moe_dims_t* dims, const void* x, const int32_t* token_ids, const void* router_w,
                         const float* router_b, const int32_t* tid2eid, const moe_qmat_t* w1,
                         const moe_qmat_t* w3, const moe_qmat_t* w2, const moe_qmat_t* shared, void* out,
                         int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  return forward_impl(dims, x, token_ids, router_w, router_b, tid2eid, w1, w3, w2, shared, out, false, topk_ids_out,
                      topk_w_out, ws, ws_bytes, stream);
}

moe_status_t moe_forward_partial(const moe_dims_t* dims, int32_t expert_begin, int32_t expert_end,
                                 int32_t include_shared, const void* x, const int32_t* token_ids,
                                 const void* router_w, const float* router_b, const int32_t* tid2eid,
                                 const moe_qmat_t* w1, const moe_qmat_t* w3, const moe_qmat_t* w2,
                                 const moe_qmat_t* shared, float* out_partial, int32_t* topk_ids_out,
                                 float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  if (expert_begin < 0 || expert_begin > expert_end || expert_end > d.n_experts)
    return fail(MOE_ERR_INVALID_ARG, "expert range [%d, %d) outside [0, %d]", expert_begin, expert_end, d.n_experts);
  if (include_shared != 0 && include_shared != 1) return fail(MOE_ERR_INVALID_ARG, "include_shared must be 0 or 1");
  WsLayout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = check_route_args(d, x, router_w, token_ids, tid2eid)) != MOE_OK) return st;
  if ((st = check_dev_ptr(out_partial, "out_partial")) != MOE_OK) return st;
  if (!aligned16(out_partial)) return fail(MOE_ERR_INVALID_ARG, "out_partial must be 16-byte aligned");
  QMatDev q1, q3, q2, qs[3];
  if ((st = check_qmat(w1, d.d_model, "w1", &q1, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w3, d.d_model, "w3", &q3, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w2, d.d_ff, "w2", &q2, d.d_model)) != MOE_OK) return st;
  if (d.d_ff_shared > 0) {
    if (!shared) return fail(MOE_ERR_INVALID_ARG, "d_ff_shared > 0 but shared is NULL");
    if ((st = check_qmat(&shared[0], d.d_model, "shared w1", &qs[0], d.d_ff_shared)) != MOE_OK) return st;
    if ((st = check_qmat(&shared[1], d.d_model, "shared w3", &qs[1], d.d_ff_shared)) != MOE_OK) return st;
    if ((st = check_qmat(&shared[2], d.d_ff_shared, "shared w2", &qs[2], d.d_model)) != MOE_OK) return st;
  }
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  const QMatDev* sh = d.d_ff_shared > 0 ? qs : nullptr;
  if (di->dec_blocks <= 0 || !dec_eligible(d, q1, q3, q2, sh))
    return fail(MOE_ERR_UNSUPPORTED, "expert slices run on the fused single-launch path only (T <= %d)", kDecMaxT);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  hook_begin(s);
  st = launch_decode_fused(d, x, token_ids, router_w, router_b, tid2eid, q1, q3, q2, sh, nullptr, topk_ids_out,
                           topk_w_out, ws, L, s, *di, DecPart{expert_begin, expert_end, include_shared, out_partial});
  hook_end();
  return st;
}

}  // extern "C"

namespace {
moe_status_t forward_launches(const moe_dims_t& d, const void* x, const int32_t* token_ids, const void* router_w,
                              const float* router_b, const int32_t* tid2eid, const QMatDev& q1, const QMatDev& q3,
                              const QMatDev& q2, const QMatDev* qs, void* out, int32_t* topk_ids_out,
                              float* topk_w_out, void* ws, const WsLayout& L, cudaStream_t s) {
  moe_status_t st;
  hook_begin(s);
  {
    DevInfo* di = nullptr;
    if ((st = dev_info(&di)) != MOE_OK) return st;
    const QMatDev* sh = d.d_ff_shared > 0 ? qs : nullptr;
    if (di->dec_blocks > 0 && use_dec(d, q1, q3, q2, sh))
      return launch_decode_fused(d, x, token_ids, router_w, router_b, tid2eid, q1, q3, q2, sh, out, topk_ids_out,
                                 topk_w_out, ws, L, s, *di, DecPart{0, (int)d.n_experts, 1, nullptr});
    if (g_ffn_path == MOE_FFN_DECODE_FUSED)
      return fail(MOE_ERR_UNSUPPORTED, "the fused decode path does not take these shapes or formats");
  }
  int* ids = topk_ids_out ? topk_ids_out : ws_at<int>(ws, L.ids);
  float* wts = topk_w_out ? topk_w_out : ws_at<float>(ws, L.wts);
  int* offsets = ws_at<int>(ws, L.offsets);
  int* sorted = ws_at<int>(ws, L.sorted);
  int* inv = ws_at<int>(ws, L.inv);
  if (fused_route_ok(d)) {
    if ((st = launch_route_fused(d, x, router_w, router_b, token_ids, tid2eid, ids, wts, offsets, sorted, inv, ws,
                                 L, s)) != MOE_OK)
      return st;
  } else {
    if ((st = launch_route(d, x, router_w, router_b, token_ids, tid2eid, ids, wts, ws, L, s)) != MOE_OK) return st;
    if ((st = launch_permute(d, ids, offsets, sorted, inv, ws, L, s)) != MOE_OK) return st;
  }
  float* y = ws_at<float>(ws, L.y);
  if ((st = launch_ffn(d, x, offsets, sorted, q1, q3, q2, d.d_ff_shared > 0 ? qs : nullptr, y, d.d_model, ws, L,
                       s)) != MOE_OK)
    return st;
  const float* y_sh = d.d_ff_shared > 0 ? y + (size_t)d.T * d.top_k * d.d_model : nullptr;
  return launch_combine(d, y, inv, wts, y_sh, out, s);
}
}  // namespace

extern "C" {

// Outputs up to this size go straight into mapped host memory (moe_forward_host).
constexpr size_t kHostDirectOutMax = 1u << 20;

moe_status_t moe_forward_host(const moe_dims_t* dims, const void* x_host, const int32_t* token_ids_host,
                              const void* router_w, const float* router_b, const int32_t* tid2eid,
                              const moe_qmat_t* w1, const moe_qmat_t* w3, const moe_qmat_t* w2,
                              const moe_qmat_t* shared, void* out_host, void* ws, size_t ws_bytes, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  if (!x_host || !out_host) return fail(MOE_ERR_INVALID_ARG, "x_host/out_host is NULL");
  if (d.hash_mode && !token_ids_host) return fail(MOE_ERR_INVALID_ARG, "token_ids_host is NULL");
  WsLayout L;
  if ((st = check_ws(d, ws, ws_bytes, &L)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* xd = ws_at<void>(ws, L.xstage);
  int* td = ws_at<int>(ws, L.tokstage);
  void* od = ws_at<void>(ws, L.outstage);
  const size_t xbytes = (size_t)d.T * d.d_model * 2;
  cudaError_t e = cudaMemcpyAsync(xd, x_host, xbytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy x to device");
  if (d.hash_mode) {
    e = cudaMemcpyAsync(td, token_ids_host, (size_t)d.T * sizeof(int), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy token ids to device");
  }
  // A small output into page-locked, device-mapped host memory is written
  // there by the layer's last kernel (no separate device-to-host copy);
  // otherwise it goes through the workspace and one copy.
  bool direct = false;
  if (xbytes <= kHostDirectOutMax) {
    cudaPointerAttributes pa{};
    if (cudaPointerGetAttributes(&pa, out_host) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
        pa.devicePointer != nullptr && aligned16(pa.devicePointer)) {
      od = pa.devicePointer;
      direct = true;
    } else {
      cudaGetLastError();  // pageable memory: not an error
    }
  }
  st = forward_impl(dims, xd, d.hash_mode ? td : nullptr, router_w, router_b, tid2eid, w1, w3, w2, shared, od, direct,
                    nullptr, nullptr, ws, ws_bytes, stream);
  if (st != MOE_OK) return st;
  if (!direct) {
    e = cudaMemcpyAsync(out_host, od, xbytes, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy out to host");
  }
  return MOE_OK;
}

moe_status_t moe_read_device_error(void* ws, int32_t* code_out, void* stream) {
  g_detail[0] = 0;
  if (!ws || !code_out) return fail(MOE_ERR_INVALID_ARG, "ws/code_out is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  e = cudaMemset(ws, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  *code_out = v;
  return MOE_OK;
}

}  // extern "C"

// ============================================================================
// Allocation-free variant of moe_expert_ffn.
//
// Some callers cannot hand the library a workspace: a host framework that owns
// the whole device memory pool and forbids foreign allocations, a plug-in
// that is only ever given its input and output buffers, or code that must not
// call cudaMalloc/cudaFree because those calls can synchronise the device.
// For them the expert FFN's scratch (the active-expert list and the SwiGLU
// hidden rows h) lives in one file-scope device array of fixed size instead.
// ============================================================================
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB on every device that loads the library
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_addr[64] = {};

// Device address of g_static_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
moe_status_t static_scratch_addr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    }
    // the error word starts at zero once; afterwards only the reader clears it
    e = cudaMemset(p, 0, sizeof(WsHeader));
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "clear static scratch header");
    }
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_expert_ffn_noalloc(const moe_dims_t* dims, const void* x, const int32_t* expert_offsets,
                                               const int32_t* sorted_rows, const moe_qmat_t* w1, const moe_qmat_t* w3,
                                               const moe_qmat_t* w2, float* y, void* stream) {
  g_detail[0] = 0;
  moe_status_t st = check_dims(dims);
  if (st != MOE_OK) return st;
  const moe_dims_t& d = *dims;
  // scratch layout inside the static array: [error word | active list | h]
  WsLayout Ls{};
  Ls.hdr = 0;
  Ls.active = align_up(sizeof(WsHeader));
  Ls.h = align_up(Ls.active + (size_t)(d.n_experts + 1) * sizeof(int));
  const size_t need = Ls.h + (size_t)d.T * d.top_k * d.d_ff * sizeof(float);
  if (need > kStaticScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED,
                "T*top_k*d_ff = %lld hidden values need %zu bytes of scratch; the allocation-free entry point "
                "has %zu (use moe_expert_ffn with a workspace)",
                (long long)d.T * d.top_k * d.d_ff, need, kStaticScratchBytes);
  if ((st = check_dev_ptr(x, "x")) != MOE_OK) return st;
  if (!aligned16(x)) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if ((st = check_dev_ptr(expert_offsets, "expert_offsets")) != MOE_OK) return st;
  if ((st = check_dev_ptr(sorted_rows, "sorted_rows")) != MOE_OK) return st;
  if ((st = check_dev_ptr(y, "y")) != MOE_OK) return st;
  if (!aligned16(y)) return fail(MOE_ERR_INVALID_ARG, "y must be 16-byte aligned");
  QMatDev q1, q3, q2;
  if ((st = check_qmat(w1, d.d_model, "w1", &q1, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w3, d.d_model, "w3", &q3, d.d_ff)) != MOE_OK) return st;
  if ((st = check_qmat(w2, d.d_ff, "w2", &q2, d.d_model)) != MOE_OK) return st;
  if (q1.fmt != q3.fmt || q1.group != q3.group)
    return fail(MOE_ERR_UNSUPPORTED, "w1 and w3 must share one format");
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  void* scratch = nullptr;
  if ((st = static_scratch_addr(&scratch)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the active list and h are fully rewritten before they are read; the
  // error word keeps the first device error since the last
  // moe_read_noalloc_error on this device
  WsHeader* hdr = ws_at<WsHeader>(scratch, Ls.hdr);
  active_from_offsets_kernel<<<1, kPermThreads, 0, s>>>(expert_offsets, d.n_experts, d.T * d.top_k, sorted_rows,
                                                        ws_at<int>(scratch, Ls.active), &hdr->err, nullptr);
  MOE_CHECK_LAUNCH("active_from_offsets_kernel");
  moe_dims_t dn = d;
  dn.d_ff_shared = 0;
  return launch_ffn(dn, x, expert_offsets, sorted_rows, q1, q3, q2, nullptr, y, d.d_model, scratch, Ls, s);
}

extern "C" moe_status_t moe_read_noalloc_error(int32_t* code_out, void* stream) {
  g_detail[0] = 0;
  if (!code_out) return fail(MOE_ERR_INVALID_ARG, "code_out is NULL");
  void* scratch = nullptr;
  moe_status_t st = static_scratch_addr(&scratch);
  if (st != MOE_OK) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpy(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  e = cudaMemset(scratch, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  *code_out = v;
  return MOE_OK;
}

extern "C" moe_status_t moe_hc_sinkhorn_mix(int32_t T, int32_t n, int32_t d, int32_t iters, float eps,
                                            const float* logits, const void* h, float* P_out, void* out,
                                            void* stream) {
  g_detail[0] = 0;
  if (T < 1) return fail(MOE_ERR_INVALID_ARG, "T=%d must be >= 1", T);
  if (n < 1 || n > kHcMaxN) return fail(MOE_ERR_UNSUPPORTED, "n=%d outside [1, %d]", n, kHcMaxN);
  if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
  if (iters < 0 || iters > 10000) return fail(MOE_ERR_INVALID_ARG, "iters=%d outside [0, 10000]", iters);
  if (!(eps >= 0.f) || eps > 1.f) return fail(MOE_ERR_INVALID_ARG, "eps must be in [0, 1]");
  moe_status_t st;
  if ((st = check_dev_ptr(logits, "logits")) != MOE_OK) return st;
  if ((st = check_dev_ptr(h, "h")) != MOE_OK) return st;
  if ((st = check_dev_ptr(out, "out")) != MOE_OK) return st;
  if (P_out && (st = check_dev_ptr(P_out, "P_out")) != MOE_OK) return st;
  if (!aligned16(h) || !aligned16(out)) return fail(MOE_ERR_INVALID_ARG, "h and out must be 16-byte aligned");
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int grid = std::min(T, di->sms * 8);
  const __nv_bfloat16* hb = reinterpret_cast<const __nv_bfloat16*>(h);
  __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(out);
  switch (n) {
#define MOE_HC_CASE(N)                                                                                  \
  case N:                                                                                               \
    hc_sinkhorn_mix_kernel<N><<<grid, kHcThreads, 0, s>>>(logits, hb, P_out, ob, T, n, d, iters, eps); \
    break;
    MOE_HC_CASE(1) MOE_HC_CASE(2) MOE_HC_CASE(3) MOE_HC_CASE(4)
    MOE_HC_CASE(5) MOE_HC_CASE(6) MOE_HC_CASE(7) MOE_HC_CASE(8)
#undef MOE_HC_CASE
  }
  MOE_CHECK_LAUNCH("hc_sinkhorn_mix_kernel");
  return MOE_OK;
}

extern "C" int32_t moe_test_stall_fused_wait(int32_t enable) {
  const int prev = g_stall_test;
  g_stall_test = enable ? 1 : 0;
  return prev;
}

extern "C" moe_status_t moe_dequant_mxfp8(const void* codes, const uint8_t* scales, int64_t rows, int32_t n_in,
                                          void* out, void* stream) {
  g_detail[0] = 0;
  if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "rows=%lld must be >= 0", (long long)rows);
  if (n_in < 32 || n_in % 32) return fail(MOE_ERR_INVALID_ARG, "n_in=%d must be a positive multiple of 32", n_in);
  if (rows == 0) return MOE_OK;
  moe_status_t st;
  if ((st = check_dev_ptr(codes, "codes")) != MOE_OK) return st;
  if ((st = check_dev_ptr(scales, "scales")) != MOE_OK) return st;
  if ((st = check_dev_ptr(out, "out")) != MOE_OK) return st;
  if (!aligned16(codes) || !aligned16(out)) return fail(MOE_ERR_INVALID_ARG, "codes and out must be 16-byte aligned");
  DevInfo* di;
  if ((st = dev_info(&di)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long work = rows * (long long)(n_in / 8);
  const int grid = (int)std::max<long long>(
      1, std::min<long long>((work + (long long)kFp8Threads * kFp8Unroll - 1) / ((long long)kFp8Threads * kFp8Unroll),
                             (long long)di->sms * 8));
  dequant_mxfp8_kernel<<<grid, kFp8Threads, 0, s>>>(reinterpret_cast<const uint8_t*>(codes), scales,
                                                    reinterpret_cast<__nv_bfloat16*>(out), (long long)rows, n_in);
  MOE_CHECK_LAUNCH("dequant_mxfp8_kernel");
  return MOE_OK;
}
