// Host/device definitions shared by the streaming expert-FFN kernels and
// the library's launch planner.
#pragma once

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------ configuration
constexpr int kStages = 3;
constexpr int kStageBytes = 72 * 1024;  // packed words + scales (+ biases) of one tile
constexpr int kConsumerWarps = 8;
constexpr int kStreamThreads = (kConsumerWarps + 1) * 32;  // + one copy-issuing warp
constexpr int kRedHalf = 1024;          // group partials: 8 warps x 16 rows x 2 values x NT<=4
constexpr int kRedFloats = 2 * kRedHalf;  // double buffered
constexpr size_t kStreamSmem = (size_t)kStages * kStageBytes + kRedFloats * 4 + 2 * kStages * 8 + 16;
static_assert(kStreamSmem <= 227 * 1024, "streaming kernel exceeds the per-block shared memory limit");

struct StreamParams {
  const __nv_bfloat16* x;  // stage 1 input [T, d]
  const float* hin;        // stage 2 input rows [P, ld_in]
  float* out;              // stage 1: h; stage 2: y
  int ld_in, ld_out;
  int T, k;
  QMatDev ra, rb;          // routed (stage 1: w1, w3; stage 2: w2)
  const int* offsets;
  const int* sorted_rows;
  const int* active;       // [0] = n, [1..] expert ids
  int has_shared;
  QMatDev sa, sb;
  int shared_pos0;         // = T*k
  int r_rows, s_rows;      // rows per tile: routed, shared (multiples of the group count)
  int r_wpr, s_wpr;        // warps per row group: routed, shared
  int* err;
};

// Launchers of the streaming kernels, one translation unit per (stage,
// routed format); the shared expert may use the routed format or 8-bit.
using StreamLaunchFn = bool (*)(int ntmax, int cpl, int grid, cudaStream_t s, const StreamParams& q);
using StreamAttrFn = void (*)();
#define MOE_STREAM_DECL(ST, F)                                                                   \
  bool launch_stream_s##ST##_##F(int ntmax, int cpl, int grid, cudaStream_t s, const StreamParams& q); \
  void attrs_stream_s##ST##_##F();
MOE_STREAM_DECL(1, A2)
MOE_STREAM_DECL(1, A3)
MOE_STREAM_DECL(1, A4)
MOE_STREAM_DECL(1, A8)
MOE_STREAM_DECL(1, MX4)
MOE_STREAM_DECL(2, A2)
MOE_STREAM_DECL(2, A3)
MOE_STREAM_DECL(2, A4)
MOE_STREAM_DECL(2, A8)
MOE_STREAM_DECL(2, MX4)
#undef MOE_STREAM_DECL

}  // namespace moe
