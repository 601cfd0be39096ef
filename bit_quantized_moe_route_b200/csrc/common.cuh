// Device-side helpers shared by the layer's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

constexpr int kErrDeviceInput = 6;  // MOE_ERR_DEVICE_INPUT
constexpr int kErrTimeout = 5;      // MOE_ERR_TIMEOUT

// Format codes used inside the kernels (one per packed layout).
enum FmtCode : int { F_A2 = 0, F_A3 = 1, F_A4 = 2, F_A8 = 3, F_MX4 = 4 };

// Workspace header: error word and small counters (256 bytes).
struct WsHeader {
  int err;
  int pad0[3];
  int counters[60];
};

// One stacked packed matrix as the kernels see it.
struct QMatDev {
  const uint32_t* q;
  const void* scales;
  const void* biases;
  int fmt;    // FmtCode
  int group;  // elements per scale group
  int n_out, n_in;
  int wpr;    // uint32 words per row
  int gpr;    // scale groups per row
};

MOE_DEV void set_error(int* err, int code) { atomicCAS(err, 0, code); }

// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may start before its predecessor in the
// stream has finished; pdl_wait() blocks until that predecessor has completed
// and its memory is visible (a no-op without the attribute), pdl_trigger()
// lets this kernel's own dependent start launching.
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

MOE_DEV float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

MOE_DEV float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
MOE_DEV float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Streaming 128-bit load that bypasses L1 allocation (weights are read once).
MOE_DEV uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
MOE_DEV uint2 ldg_stream2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
MOE_DEV uint32_t ldg_stream1(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Numerically stable sqrt(softplus(x)) = sqrt(max(x,0) + log1p(exp(-|x|))).
MOE_DEV float sqrt_softplus(float x) {
  return sqrtf(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
}

MOE_DEV float silu(float a) { return a / (1.f + expf(-a)); }

MOE_DEV float magic_u2f(uint32_t q) {  // exact for q < 2^23
  return __uint_as_float(0x4B000000u | q) - 8388608.f;
}

}  // namespace moe
