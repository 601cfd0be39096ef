// The whole routed-MoE layer for small batches (T <= 32 tokens) in ONE
// persistent launch: routing, both expert-FFN stages and the weighted
// combine.  [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": fp32 router logits,
// logaddexp-stable sqrtsoftplus, pre-stacked w1/w2/w3 = gate/down/up; model
// card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit": affine packs
// w = scale*q + bias, mxfp4 = e2m1 codes with e8m0 group scales; model card
// "DeepSeek-V4-Flash-MLX-4bit", "Why mixed-4_8bit": routed experts are ~98% of
// the weight bytes, so this path is a weight stream.]
//
// Phases (one CTA per SM, co-resident by a cooperative launch):
//   P0  every CTA: router logits of a slice of experts (learned) or the
//       table row and weights of one token (hash), and the fixed-point planes
//       of a slice of the activation blocks (dec_common.cuh);
//       grid barrier (bounded);
//   P1  every CTA, redundantly: top-k of every token (one warp per token),
//       per-expert counts, offsets and "groups" of <= ntmax (<= 4) tokens of one expert
//       (warp scans over 32-expert chunks, one chunk per warp; the shared
//       expert's tokens form their own groups),
//       the stable (token, slot) order within each expert (warp match);
//       for one token (learned routing) the top-k warp orders its k experts
//       itself, with no counting pass;
//   S1  units (group, 64 rows of d_ff): h = silu(W1 x) * (W3 x) for the
//       group's tokens, written as the planes W2 reads; a per-group counter
//       counts finished units;
//   S2  units (group, 128 rows of d_model): y = W2 h, whose weight stages
//       are issued at once and whose h planes follow once the group's S1
//       units are all counted;
//   C   grid barrier, then every CTA sums the k slots of a slice of the
//       output in ascending j, adds the shared expert and writes bf16 (one
//       rounding).
// Units are claimed dynamically in the order [S1 shared, S1 routed, S2 by
// group]: a CTA's first unit is its index, the next comes from a launch-wide
// counter, claimed once the current unit's weight stages are all issued.
//
// Weight stream.  One producer warp fills a ring of 32 KB stages; a stage is
// a set of WHOLE row segments: 16 rows of W1 and the same 16 rows of W3 (S1)
// or 32 rows of W2 (S2), each row contributing up to 1024 contiguous code
// bytes (768 for 3-bit).  Each matrix's segment arrives as ONE 3-D TMA box
// over a chunk-major view of the packed rows (dims: 128-byte line, row,
// line index within the row), so the box lands as [line][row][128 B] with the
// 128-byte swizzle keyed on the row: the 8 rows an ldmatrix phase reads sit in
// distinct banks, and DRAM sees 16 or 32 runs of 1 KB per box.  The scales
// and biases of those rows come as 2-D boxes.  The activation planes of the
// unit's tokens for the stage's inputs go to one of two plane buffers (bulk
// copies), loaded once per input chunk and shared by the chunk's 4 (S1) or 2
// (S2) row sets.  Eight consumer warps = 2 row tiles x 4 input slices: a S1
// tile is 8 rows of W1 stacked on the same 8 rows of W3 (so one thread holds
// both halves of its SwiGLU pair), a S2 tile 16 rows of W2.  They unpack
// codes to bytes, run m16n8k32 integer MMAs against the planes (exact int32
// sums per 64-input block) and fold each block into fp32 with the weight
// scale and bias; the slices are summed in a fixed order at the unit's end.
// Every wait is bounded: on timeout the kernel records MOE_ERR_TIMEOUT, keeps
// every warp's barrier sequence, lets in-flight copies land and returns.
#pragma once

#include "dec_common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kDecConsumerWarps = 8;
constexpr int kDecNkq = kDecConsumerWarps;          // input slices: one per consumer warp (both row tiles)
constexpr int kDecProducerWarp = kDecConsumerWarps;
constexpr int kDecServiceWarp = kDecConsumerWarps + 1;
constexpr int kDecWarps = kDecConsumerWarps + 2;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecConsumerThreads = kDecConsumerWarps * 32;
constexpr int kDecMaxSlots = 6;
constexpr int kDecSlotCap = 4;     // ring slots used (more 32 KB stages in flight lower the copy rate)
constexpr int kDecRows = 64;       // hidden rows per S1 unit (one 64-input block of W2's planes)
constexpr int kDecRows2 = 128;     // output rows per S2 unit
constexpr int kDecR1 = 16;         // rows of W1 (and of W3) per stage
constexpr int kDecR2 = 32;         // rows of W2 per stage
constexpr int kDecMaxTok = 4;      // tokens per group (B columns 0..7 of the MMA: hi and lo plane of each)
constexpr int kDecMaxT = 32;
constexpr int kDecMaxPairs = 256;  // T * top_k
static_assert(kDecMaxPairs <= kDecThreads, "hash weights take one (token, slot) pair per thread");
constexpr int kDecMaxE = 1024;
constexpr int kDecCodeBytes = 32768;  // code bytes of a stage, at most
constexpr int kDecMaxSeg = 1024;      // code bytes per row and stage, at most
constexpr int kDecRedFloats = kDecNkq * 4 * 16 * 8;
constexpr int kDecOffLen = kDecMaxE + 4;
constexpr int kDecMaxGroups = kDecMaxPairs + 8;
// fixed shared region (after the ring and the two plane buffers), byte offsets
constexpr int kDecFxRed = 0;
constexpr int kDecFxH = kDecFxRed + kDecRedFloats * 4;           // 2 buffers x 4 tokens x 64 h values
constexpr int kDecFxScr = kDecFxH + 2 * kDecMaxTok * kDecRows * 4;  // the service warp's scratch (64 ints)
constexpr int kDecFxIds = kDecFxScr + 256;
constexpr int kDecFxW = kDecFxIds + kDecMaxPairs * 4;
constexpr int kDecFxSorted = kDecFxW + kDecMaxPairs * 4;
constexpr int kDecFxInv = kDecFxSorted + kDecMaxPairs * 4;
constexpr int kDecFxOff = kDecFxInv + kDecMaxPairs * 4;
constexpr int kDecFxCur = kDecFxOff + kDecOffLen * 4;
constexpr int kDecFxGroups = kDecFxCur + kDecOffLen * 4;
constexpr int kDecFxBars = kDecFxGroups + kDecMaxGroups * 16;
constexpr int kDecFxMisc = kDecFxBars + (2 * kDecMaxSlots + 8) * 8;
constexpr int kDecFixedBytes = kDecFxMisc + 64;
constexpr int kDecSmemMax = 227 * 1024;
static_assert(kDecFxGroups % 16 == 0 && kDecFxBars % 8 == 0, "group records and barriers must stay aligned");

// One packed matrix as the fused kernel streams it.
struct DecMat {
  int fmt, group, n_out, n_in;
  int R;       // rows per stage and box: 16 (W1, W3) or 32 (W2)
  int lb;      // bytes per line of the box: 128 (swizzled) or 96 (3-bit, unswizzled)
  int seg;     // code bytes per row and stage (a multiple of lb)
  int nch;     // stages along a row (row bytes / seg)
  int K;       // inputs per stage
  int nbw;     // 64-input blocks per consumer warp and stage (K / 512)
  int sK;      // scale entries per row and stage
  int spitch;  // bytes per row of a scale box: the stage's scales padded to an odd multiple of 16
  int ptok;    // plane bytes per token in a plane buffer (n_in * 2, bank-padded)
  int sxtok;   // block-record bytes per token in a plane buffer (n_in / 64 * 16, bank-padded)
};

enum DecMatIdx { DM_W1 = 0, DM_W3 = 1, DM_W2 = 2, DM_S1 = 3, DM_S3 = 4, DM_S2 = 5 };

struct DecParams {
  CUtensorMap map[6];   // codes of w1, w3, w2, shared w1, w3, w2 (3-D, chunk-major)
  CUtensorMap smap[6];  // their scales
  CUtensorMap bmap[6];  // their biases (affine)
  DecMat m[6];
  const __nv_bfloat16* x;
  const void* router_w;
  const float* router_b;
  const int* token_ids;
  const int* tid2eid;
  int router_bf16;
  int T, d, f, fs, E, k, hash, vocab, has_shared;
  int G;           // grid size
  int nslot;       // ring slots
  int slot_bytes;  // 32 KB of codes + scales and biases (multiple of 1024)
  int pbuf;        // bytes per plane buffer (multiple of 128): one unit's activation rows
  int sx_off;      // offset of the per-block records within a plane buffer
  int ntmax;       // tokens per group (<= 4): the plane buffers hold this many rows
  // workspace
  float* logits;       // [T][E]
  int* hids;           // [T][k] (hash)
  float* hw;           // [T][k] (hash)
  uint8_t* xplanes;    // [2][T][d*4]: planes (d*2 bytes used) for the routed (0) and shared (1) W1/W3 formats
  float4* xsx;         // [T][d/64]: (step, sum of inputs 0..31, sum of 32..63, sum)
  uint8_t* hplanes;    // [P][fmax*4]
  float4* hsx;         // [P][fmax/64]
  float* y;            // [P][d]
  int* cnt_h;          // [kDecMaxGroups]
  int* sync;           // [0] barrier count, [1] barrier generation, [2] units claimed past the first G
  int* err;
  __nv_bfloat16* out;  // [T][d]
  int* ids_out;        // [T][k] or NULL
  float* w_out;        // [T][k] or NULL
  int stall_test;      // testing the timeout path: the first W2 dependency waits on a count nothing reaches
  // expert parallelism: only experts e_begin <= e < e_end run and enter the
  // combine, the shared expert only when with_shared; out_f32 (when not
  // NULL) receives the fp32 partial instead of the bf16 output
  int e_begin, e_end, with_shared;
  float* out_f32;
};

// ------------------------------------------------------------ grid barrier
// Generation barrier over the whole (co-resident) grid; bounded wait.  The
// arrive is one acquire-release atomic (its release covers the CTA's writes,
// ordered before it by bar.sync); the last arriver resets the count and
// publishes the next generation with a release, which the others acquire.
MOE_DEV void dec_grid_barrier(int* sync, int nblocks, int* err, volatile int* abort_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int* gen = sync + 1;
    int my_gen;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(my_gen) : "l"(gen) : "memory");
    int t;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(t) : "l"(sync) : "memory");
    if (t == nblocks - 1) {
      asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(sync), "r"(0) : "memory");
      red_release_add(gen, 1);
    } else {
      const long long t0 = clock64();
      while (ld_acquire(gen) == my_gen) {
        if (clock64() - t0 > kDecWaitCycles) {
          set_error(err, kErrTimeout);
          *abort_flag = 1;
          break;
        }
      }
    }
  }
  __syncthreads();
}

// 8 router weights of expert e at inputs i..i+7 as floats (fp32 or bf16 rows)
MOE_DEV void dec_router8(const DecParams& p, int e, int i, float (&w)[8]) {
  if (p.router_bf16) {
    const uint4 r =
        __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.router_w) + (size_t)e * p.d + i));
    w[0] = bf16lo(r.x); w[1] = bf16hi(r.x); w[2] = bf16lo(r.y); w[3] = bf16hi(r.y);
    w[4] = bf16lo(r.z); w[5] = bf16hi(r.z); w[6] = bf16lo(r.w); w[7] = bf16hi(r.w);
  } else {
    const float4* rr = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.router_w) + (size_t)e * p.d + i);
    const float4 a = __ldg(rr), b = __ldg(rr + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
}

// Sums each of 16 per-lane values over the warp with 16 shuffles: halves of
// the values are exchanged with lane ^ 16, ^ 8, ^ 4, ^ 2, then ^ 1.  Value
// 8*b4 + 4*b3 + 2*b2 + b1 (b: bits of the lane id) ends in the lane pair
// (2m, 2m+1) holding those bits; the order of additions is fixed.
MOE_DEV float dec_transpose_sum16(const float (&a)[16]) {
  const int lane = threadIdx.x & 31;
  float b[8], c[4], d2[2];
  const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4, h1 = lane & 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float send = h4 ? a[j] : a[8 + j], keep = h4 ? a[8 + j] : a[j];
    b[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float send = h3 ? b[j] : b[4 + j], keep = h3 ? b[4 + j] : b[j];
    c[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = h2 ? c[j] : c[2 + j], keep = h2 ? c[2 + j] : c[j];
    d2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float send = h1 ? d2[0] : d2[1], keep = h1 ? d2[1] : d2[0];
  const float e = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  return e + __shfl_xor_sync(0xffffffffu, e, 1);
}

// ------------------------------------------------------------ P0: planes
// The planes of one 64-input block of one activation row (64 values, two
// per lane, already in registers; lane l holds inputs 2l, 2l+1): warp-wide.
// `q_scratch`: 64 ints of this warp's shared scratch.  Writes the records of
// `perm` at `dst` (2 k-blocks x 4 threads x 16 bytes) and returns (step,
// dequantised sum of inputs 0..31, of 32..63, of all 64) to every lane.
MOE_DEV float4 dec_make_block(float v0, float v1, int perm, uint8_t* dst, int* q_scratch, int* err) {
  const int lane = threadIdx.x & 31;
  uint32_t e = max((__float_as_uint(v0) >> 23) & 0xFFu, (__float_as_uint(v1) >> 23) & 0xFFu);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
  if (e == 255u && lane == 0) set_error(err, kErrDeviceInput);  // inf / nan activation
  const float2 sc = fix_scales(e);
  const int q0 = __float2int_rn(v0 * sc.x), q1 = __float2int_rn(v1 * sc.x);
  int s = q0 + q1;  // lanes 0..15: inputs 0..31; lanes 16..31: inputs 32..63
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const int s_lo = __shfl_sync(0xffffffffu, s, 0), s_hi = __shfl_sync(0xffffffffu, s, 16);
  q_scratch[2 * lane] = q0;
  q_scratch[2 * lane + 1] = q1;
  __syncwarp();
  if (lane < 8) {
    const int kb2 = lane >> 2, t = lane & 3;
    uint32_t hw[2], lw[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t hp = 0, lp = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = q_scratch[plane_input(perm, kb2, t, h, j)];
        const int lo = (int)(signed char)(q & 0xFF);  // q = 256 * hi + lo, lo in [-128, 127]
        hp |= (uint32_t)(((q - lo) >> 8) & 0xFF) << (8 * j);
        lp |= (uint32_t)(lo & 0xFF) << (8 * j);
      }
      hw[h] = hp;
      lw[h] = lp;
    }
    *reinterpret_cast<uint4*>(dst + kb2 * 64 + t * 16) = make_uint4(hw[0], hw[1], lw[0], lw[1]);
  }
  __syncwarp();
  return make_float4(sc.y, sc.y * (float)s_lo, sc.y * (float)s_hi, sc.y * (float)(s_lo + s_hi));
}

// ------------------------------------------------------------ A operands
template <int FMT>
struct DecA {
  static constexpr int bits = FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
};

MOE_DEV void unpack_a4(uint32_t wg, uint32_t wg8, uint32_t (&a)[4]) {
  a[0] = wg & 0x0F0F0F0Fu;
  a[1] = wg8 & 0x0F0F0F0Fu;
  a[2] = (wg >> 4) & 0x0F0F0F0Fu;
  a[3] = (wg8 >> 4) & 0x0F0F0F0Fu;
}
// 2 * |e2m1| of codes 0..7 (sign bit clear): 0, 1, 2, 3, 4, 6, 8, 12; a
// selector nibble with its top bit set (a negative code) yields 0
MOE_DEV uint32_t mag4(uint32_t sel) {
  uint32_t r;  // prmt default mode: a selector nibble's top bit replicates the chosen byte's sign bit
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(0x03020100u), "r"(0x0C080604u), "r"(sel));
  return r;
}
MOE_DEV void unpack_mx4(uint32_t wg, uint32_t wg8, uint32_t (&a)[4], uint32_t (&an)[4]) {
  const uint32_t fg = wg ^ 0x88888888u, fg8 = wg8 ^ 0x88888888u;
  a[0] = mag4(wg);
  a[2] = mag4(wg >> 16);
  a[1] = mag4(wg8);
  a[3] = mag4(wg8 >> 16);
  an[0] = mag4(fg);
  an[2] = mag4(fg >> 16);
  an[1] = mag4(fg8);
  an[3] = mag4(fg8 >> 16);
}
template <int KB2>
MOE_DEV void unpack_a2(uint32_t wg, uint32_t wg8, uint32_t (&a)[4]) {
  a[0] = (wg >> (4 * KB2)) & 0x03030303u;
  a[1] = (wg8 >> (4 * KB2)) & 0x03030303u;
  a[2] = (wg >> (4 * KB2 + 2)) & 0x03030303u;
  a[3] = (wg8 >> (4 * KB2 + 2)) & 0x03030303u;
}
// four 3-bit codes (12 bits) -> bytes 0..3
MOE_DEV uint32_t spread3x4(uint32_t t) {
  const uint32_t ev = ((t & 0x1C7u) * 0x401u) & 0x00070007u;
  const uint32_t od = ((t & 0xE38u) * 0x8020u) & 0x07000700u;
  return ev | od;
}
// codes 8t..8t+7 of the 12-byte k-block at byte `off` of the 96-byte line
// starting at `line` (unswizzled)
MOE_DEV uint32_t codes3x8(uint32_t line, int off, int t) {
  const uint32_t base = line + off;
  const int bt = 3 * t;
  const uint32_t w0 = lds32u(base + (bt & ~3)), w1 = lds32u(base + (bt & ~3) + 4);
  return __funnelshift_r(w0, w1, 8 * (bt & 3)) & 0xFFFFFFu;
}

// ------------------------------------------------------------ one stage
// What a consumer warp needs to address its tile in any stage of a unit
// (shared addresses relative to the stage slot).  A rows 0..7 of the tile
// live in code box `a0` at box rows r0..r0+7, A rows 8..15 in box `a8` at
// rows r8..r8+7; their scales in scale boxes `s0` / `s8` (biases R * spitch
// bytes further).
struct DecWarp {
  uint32_t a0, a8, s0, s8;
  int r0, r8;    // tile 0; tile 1 is `tstep` rows further in every box
  int tstep;
  int R;   // rows per box
  int kq;  // input slice
  int spitch;
  int ptok, sxtok;
};

// Per-lane constants of a consumer warp for every stage of one unit.  All
// per-block offsets inside a stage are then compile-time immediates.
struct DecLane {
  uint32_t la;    // slot-relative ldmatrix row address of this lane (its A row, the slice's 128-byte line)
  uint32_t ly;    // XOR applied to the 16-byte chunk offset (the 128-byte swizzle and the chunk pair)
  uint32_t l3a, l3b;  // 3-bit: slot-relative address of this thread's codes of A rows g and g+8
  uint32_t sh3;   // 3-bit: bit offset of those codes in the loaded pair of words
  uint32_t b;     // plane-buffer-relative B address (token row, quad thread, plane)
  uint32_t sx;    // record-relative address (token, the slice's first block)
  uint32_t s0, s8, brow;  // slot-relative scale addresses of A rows g / g+8 (the slice's first group), bias offset
  uint32_t ta, ts;        // tile 1: code byte offset (tstep rows), scale byte offset
};


// Lanes whose B column or C column pair belongs to a token past the group
// read another token's data: those columns are never read back.
template <int FMT, int G, int NBW>
MOE_DEV DecLane dec_lane(const DecWarp& q, int ntok) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int mtx = lane >> 3, lr = lane & 7, csel = mtx >> 1;
  const uint32_t box = (mtx & 1) ? q.a8 : q.a0;
  const int row = ((mtx & 1) ? q.r8 : q.r0) + lr;
  const int bs0 = q.kq * NBW;  // the slice's first block in the stage
  DecLane L;
  int line = 0, mk = 0;
  if constexpr (FMT == F_A4 || FMT == F_MX4) {  // 32 bytes per block: 4 blocks per line, 2 chunks each
    line = bs0 >> 2;
    mk = bs0 & 3;
    L.ly = (uint32_t)(((2 * mk) ^ csel ^ lr) << 4);
  } else if constexpr (FMT == F_A8) {  // 64 bytes per block: 2 blocks (4 k-blocks of 2 chunks) per line
    line = (2 * bs0) >> 2;
    mk = (2 * bs0) & 3;
    L.ly = (uint32_t)(((2 * mk) ^ csel ^ lr) << 4);
  } else if constexpr (FMT == F_A2) {  // 16 bytes per block: 8 blocks per line
    line = bs0 >> 3;
    mk = bs0 & 7;
    L.ly = (uint32_t)((mk ^ lr) << 4);
  } else {
    L.ly = 0;
  }
  L.la = box + (uint32_t)((line * q.R + row) * 128);
  if constexpr (FMT == F_A3) {  // 24 bytes per block in 96-byte lines
    const int by = bs0 * 24, ln = by / 96, off = by - ln * 96 + ((3 * t) & ~3);
    L.l3a = q.a0 + (uint32_t)((ln * q.R + q.r0 + g) * 96 + off);
    L.l3b = q.a8 + (uint32_t)((ln * q.R + q.r8 + g) * 96 + off);
    L.sh3 = 8 * ((3 * t) & 3);
  } else {
    L.l3a = L.l3b = L.sh3 = 0;
  }
  const int jb = min(g >> 1, ntok - 1), jc = min(t, ntok - 1);
  L.b = (uint32_t)(jb * q.ptok + bs0 * 128 + t * 16 + (g & 1) * 8);
  L.sx = (uint32_t)(jc * q.sxtok + bs0 * 16);
  const int esz = FMT == F_MX4 ? 1 : 2;
  const int gbase = G == 32 ? 2 * bs0 : (bs0 * 64) / G;
  L.s0 = q.s0 + (uint32_t)((q.r0 + g) * q.spitch + esz * gbase);
  L.s8 = q.s8 + (uint32_t)((q.r8 + g) * q.spitch + esz * gbase);
  L.brow = (uint32_t)(q.R * q.spitch);
  L.ta = (uint32_t)(q.tstep * (FMT == F_A3 ? 96 : 128));
  L.ts = (uint32_t)(q.tstep * q.spitch);
  return L;
}

// acc[0] (A row g) and acc[1] (A row g+8) of token t += s_r * st * P + b_r * sm
// over one scale group: P = 256 * C[., 2t] + C[., 2t+1] is the exact
// integer sum of codes x fixed-point inputs, st the inputs' step, sm their
// dequantised sum; GI: the group's scale entry relative to the slice.
template <int FMT, int GI>
MOE_DEV void dec_fold(uint32_t s0, uint32_t s8, uint32_t brow, float st, float sm, const int (&c)[4],
                      float (&acc)[2]) {
  float sc0, b0, sc8, b8;
  if constexpr (FMT == F_MX4) {
    // 2^(e-127) / 2 (the A operand holds 2*e2m1)
    const uint32_t e0 = lds8u(s0 + GI), e8 = lds8u(s8 + GI);
    sc0 = __uint_as_float(e0 > 1 ? ((e0 - 1) << 23) : (e0 ? 0x00400000u : 0x00200000u));
    sc8 = __uint_as_float(e8 > 1 ? ((e8 - 1) << 23) : (e8 ? 0x00400000u : 0x00200000u));
    b0 = b8 = 0.f;
  } else {
    sc0 = bf16_bits_to_float(lds16u(s0 + 2 * GI));
    b0 = bf16_bits_to_float(lds16u(s0 + brow + 2 * GI));
    sc8 = bf16_bits_to_float(lds16u(s8 + 2 * GI));
    b8 = bf16_bits_to_float(lds16u(s8 + brow + 2 * GI));
  }
  if constexpr (FMT == F_MX4) {  // no bias term
    (void)b0;
    (void)b8;
    (void)sm;
    acc[0] = fmaf(sc0 * st, (float)(c[0] * 256 + c[1]), acc[0]);
    acc[1] = fmaf(sc8 * st, (float)(c[2] * 256 + c[3]), acc[1]);
  } else {
    acc[0] = fmaf(sc0 * st, (float)(c[0] * 256 + c[1]), fmaf(b0, sm, acc[0]));
    acc[1] = fmaf(sc8 * st, (float)(c[2] * 256 + c[3]), fmaf(b8, sm, acc[1]));
  }
}

// k-block H of block B of the warp's slice for one tile: A fragment, one MMA
// (two for mxfp4: positive and negative magnitudes) with the shared B.
template <int FMT, int B, int H>
MOE_DEV void dec_kblock(const DecLane& L, uint32_t la, uint32_t sl, uint32_t t3, const uint2 bv,
                        const uint32_t (&w)[4], int (&c)[4], int (&cn)[4]) {
  uint32_t a[4];
  if constexpr (FMT == F_A4) {
    unpack_a4(w[2 * H], w[2 * H + 1], a);
  } else if constexpr (FMT == F_MX4) {
    uint32_t an[4];
    unpack_mx4(w[2 * H], w[2 * H + 1], a, an);
    mma_u8s8(cn, an, bv.x, bv.y);
  } else if constexpr (FMT == F_A8) {  // a k-block is two chunks of the line
    ldsm_x4(la + ((uint32_t)((4 * B + 2 * H) << 4) ^ L.ly), a[0], a[1], a[2], a[3]);
  } else if constexpr (FMT == F_A2) {
    unpack_a2<H>(w[0], w[1], a);
  } else {  // 3-bit: 12-byte k-blocks, this thread's 8 codes of rows g and g+8
    const uint32_t pa = sl + L.l3a + t3 + (2 * B + H) * 12, pb = sl + L.l3b + t3 + (2 * B + H) * 12;
    const uint32_t v0 = __funnelshift_r(lds32u(pa), lds32u(pa + 4), L.sh3) & 0xFFFFFFu;
    const uint32_t v8 = __funnelshift_r(lds32u(pb), lds32u(pb + 4), L.sh3) & 0xFFFFFFu;
    a[0] = spread3x4(v0 & 0xFFFu);
    a[2] = spread3x4(v0 >> 12);
    a[1] = spread3x4(v8 & 0xFFFu);
    a[3] = spread3x4(v8 >> 12);
  }
  mma_u8s8(c, a, bv.x, bv.y);
}

// A fragments of block B (both k-blocks) for the tile whose ldmatrix row is `la`
template <int FMT, int B>
MOE_DEV void dec_loadA(const DecLane& L, uint32_t la, uint32_t (&w)[4]) {
  if constexpr (FMT == F_A4 || FMT == F_MX4)  // both k-blocks: two 16-byte chunks of the line
    ldsm_x4(la + ((uint32_t)(B << 5) ^ L.ly), w[0], w[1], w[2], w[3]);
  if constexpr (FMT == F_A2) {  // the block is one chunk; lanes 0..15 address rows 0..15
    const uint32_t ad = la + ((uint32_t)(B << 4) ^ L.ly);
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(ad));
  }
}

// One 64-input block B of the warp's slice for both row tiles (acc[0..1]:
// tile 0, acc[2..3]: tile 1), folded per scale group (G = 32: per k-block).
template <int FMT, int G, int B>
MOE_DEV void dec_block(const DecLane& L, uint32_t la, uint32_t sl, uint32_t bp, uint32_t xp, uint32_t s0,
                       uint32_t s8, float (&acc)[4]) {
  const float4 rec = lds_f4(xp + B * 16);
  uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u};
  dec_loadA<FMT, B>(L, la, w0);
  dec_loadA<FMT, B>(L, la + L.ta, w1);
  int c0[4] = {0, 0, 0, 0}, cn0[4] = {0, 0, 0, 0}, c1[4] = {0, 0, 0, 0}, cn1[4] = {0, 0, 0, 0};
  float a0[2] = {acc[0], acc[1]}, a1[2] = {acc[2], acc[3]};
  {
    const uint2 bv = lds64u(bp + B * 128);
    dec_kblock<FMT, B, 0>(L, la, sl, 0u, bv, w0, c0, cn0);
    dec_kblock<FMT, B, 0>(L, la + L.ta, sl, L.ta, bv, w1, c1, cn1);
  }
  if constexpr (G == 32) {
    int d0[4], d1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      d0[i] = c0[i] - cn0[i];
      d1[i] = c1[i] - cn1[i];
      c0[i] = cn0[i] = c1[i] = cn1[i] = 0;
    }
    dec_fold<FMT, 2 * B>(s0, s8, L.brow, rec.x, rec.y, d0, a0);
    dec_fold<FMT, 2 * B>(s0 + L.ts, s8 + L.ts, L.brow, rec.x, rec.y, d1, a1);
  }
  {
    const uint2 bv = lds64u(bp + B * 128 + 64);
    dec_kblock<FMT, B, 1>(L, la, sl, 0u, bv, w0, c0, cn0);
    dec_kblock<FMT, B, 1>(L, la + L.ta, sl, L.ta, bv, w1, c1, cn1);
  }
  int d0[4], d1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    d0[i] = c0[i] - cn0[i];
    d1[i] = c1[i] - cn1[i];
  }
  if constexpr (G == 32) {
    dec_fold<FMT, 2 * B + 1>(s0, s8, L.brow, rec.x, rec.z, d0, a0);
    dec_fold<FMT, 2 * B + 1>(s0 + L.ts, s8 + L.ts, L.brow, rec.x, rec.z, d1, a1);
  } else {
    dec_fold<FMT, (B * 64) / G>(s0, s8, L.brow, rec.x, rec.w, d0, a0);
    dec_fold<FMT, (B * 64) / G>(s0 + L.ts, s8 + L.ts, L.brow, rec.x, rec.w, d1, a1);
  }
  acc[0] = a0[0];
  acc[1] = a0[1];
  acc[2] = a1[0];
  acc[3] = a1[1];
}

template <int FMT, int G, int NBW, int B = 0>
MOE_DEV void dec_blocks(const DecLane& L, uint32_t la, uint32_t sl, uint32_t bp, uint32_t xp, uint32_t s0,
                        uint32_t s8, float (&acc)[4]) {
  if constexpr (B < NBW) {
    dec_block<FMT, G, B>(L, la, sl, bp, xp, s0, s8, acc);
    dec_blocks<FMT, G, NBW, B + 1>(L, la, sl, bp, xp, s0, s8, acc);
  }
}

// The warp's input slice of one stage for both row tiles (slot `sl`; `pl`:
// the stage's inputs in the plane buffer, `sxb`: their block records).
template <int FMT, int G, int NBW>
MOE_DEV void dec_stage(const DecLane& L, uint32_t sl, uint32_t pl, uint32_t sxb, float (&acc)[4]) {
  dec_blocks<FMT, G, NBW>(L, sl + L.la, sl, pl + L.b, sxb + L.sx, sl + L.s0, sl + L.s8, acc);
}

// Routing results and work groups, shared by every CTA (built in P1).
struct DecUnit {
  int stage;  // 1 or 2
  int grp;
  int u;      // 64-row block of the unit's output rows
  int mi;     // first matrix index (DecMatIdx)
  int row0;   // first weight row in the stacked matrix
};

MOE_DEV DecUnit dec_unit(const DecParams& p, const int4* groups, int nsg, int nrg, int i) {
  DecUnit U;
  const int ufs = p.fs / kDecRows, uf = p.f / kDecRows, ud = p.d / kDecRows2;
  const int U1s = nsg * ufs, U1 = U1s + nrg * uf;
  if (i < U1) {
    U.stage = 1;
    if (i < U1s) {
      U.grp = i / ufs;
      U.u = i % ufs;
      U.mi = DM_S1;
      U.row0 = kDecRows * U.u;
    } else {
      const int j = i - U1s;
      U.grp = nsg + j / uf;
      U.u = j % uf;
      U.mi = DM_W1;
      U.row0 = groups[U.grp].x * p.f + kDecRows * U.u;
    }
  } else {
    const int j = i - U1;
    U.stage = 2;
    U.grp = j / ud;
    U.u = j % ud;
    const bool sh = groups[U.grp].x < 0;
    U.mi = sh ? DM_S2 : DM_W2;
    U.row0 = (sh ? 0 : groups[U.grp].x * p.d) + kDecRows2 * U.u;
  }
  return U;
}

// Slot (flat index into the P = T*k + T activation rows) of token i of a group.
MOE_DEV int dec_slot(const DecParams& p, const int* sorted, int4 g, int i) {
  return g.x < 0 ? p.T * p.k + g.y + i : sorted[g.y + i];
}
MOE_DEV int dec_token(const DecParams& p, const int* sorted, int4 g, int i) {
  return g.x < 0 ? g.y + i : sorted[g.y + i] / p.k;
}

// Position in the stage ring: stage count, slot, and the parity of the
// slot's current use (advanced without division).
struct DecRing {
  int n, s, ph;
  MOE_DEV void next(int nslot) {
    ++n;
    if (++s == nslot) {
      s = 0;
      ph ^= 1;
    }
  }
};

// Bounded mbarrier wait of a consumer warp; false once the kernel aborts.
MOE_DEV bool dec_consumer_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err) {
  bool have = !*abort_flag;
  if (have && !dec_wait_bar(bar, parity, abort_flag, true)) {
    set_error(err, kErrTimeout);
    *abort_flag = 1;
    have = false;
  }
  return __all_sync(0xffffffffu, have);  // the MMAs need every lane
}

// Consumer side of one unit's stages, row set by row set (S1: W1/W3 in 4
// row sets of 16, else W2 in 4 row sets of 32, each over nch stages along
// the inputs).  Each row set's slice partials go to `red`: S1 [(kq*4 + rs)*16
// + row][token][W1 | W3], S2 [(kq*4 + rs)*32 + row][token].
template <int FMT, int G, int NBW>
MOE_DEV void dec_consume(const DecWarp& q, bool s1, int nch, int K, int ntok, uint32_t ring, int slot_bytes,
                         int nslot, uint32_t pl, uint32_t sx0, uint32_t full0, uint32_t empty0, DecRing& rg,
                         bool have_pl, volatile int* abort_flag, int* err, float* red) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const DecLane L = dec_lane<FMT, G, NBW>(q, ntok);
  const int nrs = s1 ? kDecRows / kDecR1 : kDecRows2 / kDecR2;  // 4 row sets either way
  for (int rs = 0; rs < nrs; ++rs) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int chn = 0; chn < nch; ++chn, rg.next(nslot)) {
      const int s = rg.s;
      const bool have = dec_consumer_wait(full0 + 8 * s, rg.ph, abort_flag, err) && have_pl;
      if (have) dec_stage<FMT, G, NBW>(L, ring + s * slot_bytes, pl + chn * K * 2, sx0 + chn * (K / 64) * 16, acc);
      __syncwarp();
      if (lane == 0 && have) dec_arrive(empty0 + 8 * s);
    }
    if (s1) {  // tile tt: W1 rows tt*8 + g (acc[2tt]) and the same W3 rows (acc[2tt+1])
      *reinterpret_cast<float2*>(red + ((q.kq * 4 + rs) * 16 + g) * 8 + 2 * t) = make_float2(acc[0], acc[1]);
      *reinterpret_cast<float2*>(red + ((q.kq * 4 + rs) * 16 + 8 + g) * 8 + 2 * t) = make_float2(acc[2], acc[3]);
    } else {  // tile tt: rows tt*16 + g and + 8
      float* rr = red + ((q.kq * 4 + rs) * 32 + g) * 4 + t;
      rr[0] = acc[0];
      rr[8 * 4] = acc[1];
      rr[16 * 4] = acc[2];
      rr[24 * 4] = acc[3];
    }
  }
}

// (format, scale group, blocks per slice) combinations the fused kernel
// instantiates; the host admits only these (dec_supported).
__host__ __device__ inline bool dec_supported(int fmt, int group, int nbw) {
  switch (fmt) {
    case F_A4:
    case F_A3: return (group == 32 || group == 64 || group == 128) && (nbw == 2 || nbw == 4);
    case F_A8: return (group == 32 || group == 64 || (group == 128 && nbw == 2)) && (nbw == 1 || nbw == 2);
    case F_A2: return (group == 64 || group == 128) && (nbw == 4 || nbw == 8);
    default: return group == 32 && (nbw == 2 || nbw == 4);
  }
}

MOE_DEV void dec_consume_any(int fmt, int group, int nbw, const DecWarp& q, bool s1, int nch, int K, int ntok,
                             uint32_t ring, int slot_bytes, int nslot, uint32_t pl, uint32_t sx0, uint32_t full0,
                             uint32_t empty0, DecRing& rg, bool have_pl, volatile int* abort_flag, int* err,
                             float* red) {
#define MOE_DC(F, GG, NB)                                                                                        \
  dec_consume<F, GG, NB>(q, s1, nch, K, ntok, ring, slot_bytes, nslot, pl, sx0, full0, empty0, rg, have_pl, abort_flag, \
                         err, red)
#define MOE_DC_G(F, NB)                  \
  do {                                   \
    if (group == 32) MOE_DC(F, 32, NB);  \
    else if (group == 64) MOE_DC(F, 64, NB); \
    else MOE_DC(F, 128, NB);             \
  } while (0)
  switch (fmt) {
    case F_A4:
      if (nbw == 4) MOE_DC_G(F_A4, 4); else MOE_DC_G(F_A4, 2);
      break;
    case F_A3:
      if (nbw == 4) MOE_DC_G(F_A3, 4); else MOE_DC_G(F_A3, 2);
      break;
    case F_A8:
      if (nbw == 2) MOE_DC_G(F_A8, 2);
      else if (group == 32) MOE_DC(F_A8, 32, 1);
      else MOE_DC(F_A8, 64, 1);
      break;
    case F_A2:
      if (nbw == 8) {
        if (group == 64) MOE_DC(F_A2, 64, 8); else MOE_DC(F_A2, 128, 8);
      } else {
        if (group == 64) MOE_DC(F_A2, 64, 4); else MOE_DC(F_A2, 128, 4);
      }
      break;
    default:
      if (nbw == 4) MOE_DC(F_MX4, 32, 4); else MOE_DC(F_MX4, 32, 2);
      break;
  }
#undef MOE_DC_G
#undef MOE_DC
}

// fp32 order as an unsigned order (larger float -> larger key); NaN is
// mapped to -inf's key, like the router kernels' NaN handling
MOE_DEV uint32_t dec_key(float v) {
  if (v != v) v = -INFINITY;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one token's router logits (one warp): scores sqrtsoftplus(L),
// keys score + bias, the k largest keys (ties: the smaller expert), weights
// the selected scores renormalised to sum 1 (same rule as topk_token in
// route.cuh).  Every load is issued before the first use; each round is a
// warp max of the lanes' best keys (redux.sync) and a min of the expert
// index among the lanes holding it.
template <int MAXPER>
MOE_DEV void dec_topk(const float* __restrict__ L, const float* __restrict__ bias, int E, int k, int* ids, float* w) {
  const int lane = threadIdx.x & 31;
  float lv[MAXPER], bv[MAXPER];
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    const int e = i * 32 + lane;
    lv[i] = e < E ? __ldcg(L + e) : 0.f;
    bv[i] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.f;
  }
  uint32_t key[MAXPER];  // 0: no expert (past E) or already taken; any real key is larger
  float sc[MAXPER];
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    sc[i] = sqrt_softplus(lv[i]);
    key[i] = i * 32 + lane < E ? dec_key(sc[i] + bv[i]) : 0u;
  }
  float ssum = 0.f, my_s = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bslot = 0;
#pragma unroll
    for (int i = 0; i < MAXPER; ++i)
      if (key[i] > bk) {  // strict: the lowest slot among equal keys
        bk = key[i];
        bslot = i;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const int e = bslot * 32 + lane;
    const int emin = __reduce_min_sync(0xffffffffu, bk == m ? e : 0x7fffffff);
    const int owner = emin & 31, oslot = emin >> 5;
    float s_sel = 0.f;
    if (lane == owner) {
#pragma unroll
      for (int i = 0; i < MAXPER; ++i)
        if (i == oslot) {
          s_sel = sc[i];
          key[i] = 0u;
        }
    }
    s_sel = __shfl_sync(0xffffffffu, s_sel, owner);
    ssum += s_sel;
    if (lane == j) {
      my_s = s_sel;
      my_id = emin;
    }
  }
  if (lane < k) {
    ids[lane] = my_id;
    w[lane] = ssum > 0.f ? my_s / ssum : 1.f / (float)k;
  }
}

__global__ void __launch_bounds__(kDecThreads, 1) ffn_decode_kernel(const __grid_constant__ DecParams p) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = su32(base);
  const uint32_t planes0 = ring + (uint32_t)(p.nslot * p.slot_bytes);
  uint8_t* fx = base + (size_t)p.nslot * p.slot_bytes + 2 * (size_t)p.pbuf;
  float* red = reinterpret_cast<float*>(fx + kDecFxRed);
  float* hbuf = reinterpret_cast<float*>(fx + kDecFxH);  // [2][4][64]
  int* r_ids = reinterpret_cast<int*>(fx + kDecFxIds);
  float* r_w = reinterpret_cast<float*>(fx + kDecFxW);
  int* r_sorted = reinterpret_cast<int*>(fx + kDecFxSorted);
  int* r_inv = reinterpret_cast<int*>(fx + kDecFxInv);
  int* r_off = reinterpret_cast<int*>(fx + kDecFxOff);
  int* r_cur = reinterpret_cast<int*>(fx + kDecFxCur);
  int4* r_groups = reinterpret_cast<int4*>(fx + kDecFxGroups);
  const uint32_t full0 = su32(fx + kDecFxBars), empty0 = full0 + 8 * kDecMaxSlots;
  const uint32_t pfull0 = empty0 + 8 * kDecMaxSlots, pempty0 = pfull0 + 16;
  const uint32_t efull0 = pempty0 + 16, eempty0 = efull0 + 16;  // unit epilogues: consumers -> service warp
  volatile int* misc = reinterpret_cast<volatile int*>(fx + kDecFxMisc);
  // misc: [0] abort, [1] groups shared, [2] groups routed, [4] the consumers' unit,
  // [8..11] unit of each plane-buffer use (producer -> consumers, -1: no more),
  // [12..13] unit of each epilogue buffer (consumers -> service warp, -1: no more)
  volatile int* abort_flag = misc;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, k = p.k, E = p.E, d = p.d;
  const int Tk = T * k;

  if (tid == 0) {
    for (int s = 0; s < p.nslot; ++s) {
      dec_bar_init(full0 + 8 * s, 1);  // the producer's expect_tx arrive; the copies complete the transactions
      dec_bar_init(empty0 + 8 * s, kDecConsumerWarps);
    }
    for (int b = 0; b < 2; ++b) {
      dec_bar_init(pfull0 + 8 * b, 1);
      dec_bar_init(pempty0 + 8 * b, kDecConsumerWarps);
      dec_bar_init(efull0 + 8 * b, kDecConsumerWarps);
      dec_bar_init(eempty0 + 8 * b, 1);
    }
    misc[0] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kDecProducerWarp && lane < 18) {
    const CUtensorMap* mp = lane < 6 ? &p.map[lane] : lane < 12 ? &p.smap[lane - 6] : &p.bmap[lane - 12];
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(mp)) : "memory");
  }
  if (warp == kDecServiceWarp && !p.hash && p.router_b != nullptr && lane * 32 < E) {
    // every CTA's top-k reads the selection bias right after the grid
    // barrier: bring its lines into L2 now, off that path
    asm volatile("prefetch.global.L2 [%0];" ::"l"((uint64_t)__cvta_generic_to_global(p.router_b + lane * 32)) : "memory");
  }
  for (int e = tid; e < E; e += kDecThreads) r_off[e] = 0;  // per-expert counts (P1)
  __syncthreads();

  // ------------------------------------------------------------ P0
  {
    // activation planes: (token, 64-input block) tasks over every warp of the
    // grid, from the last CTA down: the first CTAs take the most router rows
    const int nb = d / 64;
    const int gw = (p.G - 1 - (int)blockIdx.x) * kDecWarps + warp, W = p.G * kDecWarps;
    int* scratch = reinterpret_cast<int*>(red) + warp * 64;
    const int f0 = p.m[DM_W1].fmt, f1 = p.m[DM_S1].fmt;
    for (int it = gw; it < T * nb; it += W) {
      const int t = it / nb, b = it % nb;
      const uint32_t xv = __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)t * d + 64 * b) + lane);
      const float v0 = bf16lo(xv), v1 = bf16hi(xv);
      uint8_t* d0 = p.xplanes + (size_t)t * d * 4 + (size_t)b * 64 * plane_bytes_per_input(f0);
      const float4 sx = dec_make_block(v0, v1, perm_of(f0), d0, scratch, p.err);
      if (p.has_shared) {
        uint8_t* d1 = p.xplanes + ((size_t)T + t) * d * 4 + (size_t)b * 64 * plane_bytes_per_input(f1);
        dec_make_block(v0, v1, perm_of(f1), d1, scratch, p.err);
      }
      if (lane == 0) p.xsx[(size_t)t * nb + b] = sx;
    }
    __syncthreads();
    if (!p.hash) {
      // router logits of experts blockIdx.x, +G, ... for every token: passes
      // of (2 experts, 8 tokens); every warp takes 256-input chunks, loads the
      // chunk's x once for both experts, and reduces its 16 (expert, token)
      // partials with one transposed butterfly; the chunks' partials are then
      // summed in a fixed order (d is a multiple of 256 here)
      const int ne = (int)blockIdx.x < E ? (E - 1 - (int)blockIdx.x) / p.G + 1 : 0;
      const int nch = d / 256;
      float* part = red;  // [chunk][2 experts][8 tokens]
      for (int eb = 0; eb < ne; eb += 2) {
        const int ea = blockIdx.x + eb * p.G, ebx = ea + p.G;
        const bool two = eb + 1 < ne;
        for (int t0 = 0; t0 < T; t0 += 8) {
          // the router weights of the warp's next chunk are requested before
          // this chunk's sums, so a warp's chunks wait on DRAM together
          auto load = [&](int c, float(&a)[8], float(&b)[8]) {
            const int i = c * 256 + lane * 8;
            dec_router8(p, ea, i, a);
            if (two) dec_router8(p, ebx, i, b);
            else
#pragma unroll
              for (int q = 0; q < 8; ++q) b[q] = 0.f;
          };
          float wa[8], wb[8];
          if (warp < nch) load(warp, wa, wb);
          for (int c = warp; c < nch; c += kDecWarps) {
            const int i = c * 256 + lane * 8;
            const bool more = c + kDecWarps < nch;
            float na[8], nb[8];
            if (more) load(c + kDecWarps, na, nb);
            float acc[16];  // [expert][token]
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              float a0 = 0.f, a1 = 0.f;
              if (t0 + t < T) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + t) * d + i));
                const float xf[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                                     bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  a0 = fmaf(wa[q], xf[q], a0);
                  a1 = fmaf(wb[q], xf[q], a1);
                }
              }
              acc[t] = a0;
              acc[8 + t] = a1;
            }
            // value v = 8 * expert + token ends in lanes 2v' and 2v'+1, where
            // v' = 8*bit4 + 4*bit3 + 2*bit2 + bit1 of the lane
            const float tot = dec_transpose_sum16(acc);
            if ((lane & 1) == 0) {
              const int v = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
              part[c * 16 + v] = tot;
            }
            if (more)
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                wa[q] = na[q];
                wb[q] = nb[q];
              }
          }
          __syncthreads();
          if (tid < 16) {
            const int x = tid >> 3, t = tid & 7;
            if (t0 + t < T && (x == 0 || two)) {
              float sum = 0.f;
              for (int c = 0; c < nch; ++c) sum += part[c * 16 + tid];  // fixed order
              p.logits[(size_t)(t0 + t) * E + (x ? ebx : ea)] = sum;
            }
          }
          __syncthreads();
        }
      }
    } else {
      // hash routing: the (token, slot) pairs blockIdx.x, +G, ...: the table
      // entry and the fp32 logit of that expert (every warp takes 256-input
      // chunks, summed in a fixed order); P1 turns logits into weights.  An
      // out-of-range token id or table entry stores expert 0 with logit -inf
      // (weight 0) and is reported.
      int* s_e = reinterpret_cast<int*>(hbuf);
      const int nch = d / 256;
      for (int q = blockIdx.x; q < Tk; q += p.G) {
        const int t = q / k, j = q - t * k;
        if (tid == 0) {
          const int tok = p.token_ids[t];
          int e = 0, good = 0;
          if (tok >= 0 && tok < p.vocab) {
            e = p.tid2eid[(size_t)tok * k + j];
            good = e >= 0 && e < E;
            if (!good) e = 0;
          }
          if (!good) set_error(p.err, kErrDeviceInput);
          s_e[0] = e;
          s_e[1] = good;
        }
        __syncthreads();
        const int e = s_e[0], good = s_e[1];
        if (good && p.router_w != nullptr) {
          for (int c = warp; c < nch; c += kDecWarps) {
            const int i = c * 256 + lane * 8;
            float w[8];
            dec_router8(p, e, i, w);
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * d + i));
            const float xf[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                                 bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
            float a = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) a = fmaf(w[u], xf[u], a);
            a = warp_sum(a);
            if (lane == 0) red[c] = a;
          }
        }
        __syncthreads();
        if (tid == 0) {
          float l = -INFINITY;
          if (good) {
            l = 0.f;
            if (p.router_w != nullptr)
              for (int c = 0; c < nch; ++c) l += red[c];  // fixed order
          }
          p.hids[q] = e;
          p.hw[q] = l;
        }
        __syncthreads();
      }
    }
  }
  dec_grid_barrier(p.sync, p.G, p.err, abort_flag);

  // ------------------------------------------------------------ P1
  if (!p.hash) {
    for (int t = warp; t < T; t += kDecWarps) {
      if (E <= 32)
        dec_topk<1>(p.logits + (size_t)t * E, p.router_b, E, k, r_ids + t * k, r_w + t * k);
      else if (E <= 256)
        dec_topk<8>(p.logits + (size_t)t * E, p.router_b, E, k, r_ids + t * k, r_w + t * k);
      else
        dec_topk<32>(p.logits + (size_t)t * E, p.router_b, E, k, r_ids + t * k, r_w + t * k);
    }
  } else {
    // weights from the P0 logits: renormalised sqrtsoftplus over the token's
    // slots (uniform over its valid slots without a router; -inf marks an
    // invalid entry, weight 0); Tk <= 256 < threads: one pair per thread
    float sj = 0.f;
    if (tid < Tk) {
      r_ids[tid] = __ldcg(p.hids + tid);
      const float l = __ldcg(p.hw + tid);
      sj = l == -INFINITY ? 0.f : (p.router_w != nullptr ? sqrt_softplus(l) : 1.f);
      r_w[tid] = sj;
    }
    __syncthreads();
    if (tid < Tk) {
      const int t0 = tid - tid % k;
      float ssum = 0.f;
      for (int jj = 0; jj < k; ++jj) ssum += r_w[t0 + jj];  // ascending slot
      sj = ssum > 0.f ? sj / ssum : 0.f;
    }
    __syncthreads();
    if (tid < Tk) r_w[tid] = sj;
  }
  if (!p.hash && T == 1) {
    // one token: its k experts (distinct, in range: the top-k chose them)
    // are one pair and one group each, so warp 0, which chose them, orders
    // them itself: pair j's position is the number of its experts with a
    // smaller id, and its group follows the shared group and the owned
    // experts with smaller ids (what the counting path below yields)
    if (warp == 0) {
      __syncwarp();
      const int e = lane < k ? r_ids[lane] : 0x7fffffff;
      const bool own = lane < k && e >= p.e_begin && e < p.e_end;
      int pos = 0, gpre = 0;
      for (int i = 0; i < k; ++i) {
        const int ei = __shfl_sync(0xffffffffu, e, i);
        if (ei < e) {
          ++pos;
          gpre += ei >= p.e_begin && ei < p.e_end;
        }
      }
      const int nsg = p.has_shared && p.with_shared ? 1 : 0;
      if (lane < k) {
        r_sorted[pos] = lane;
        r_inv[lane] = pos;
      }
      if (own) r_groups[nsg + gpre] = make_int4(e, pos, 1, 0);
      const int nown = __popc(__ballot_sync(0xffffffffu, own));
      if (lane == 0) {
        misc[1] = nsg;
        misc[2] = nown;
        if (nsg) r_groups[0] = make_int4(-1, 0, 1, 0);
      }
    }
  } else {
    __syncthreads();
    // per-expert counts (out-of-range ids are reported and counted as expert 0)
    {
      bool bad = false;
      for (int i = tid; i < Tk; i += kDecThreads) {
        int e = r_ids[i];
        if (e < 0 || e >= E) {
          bad = true;
          e = 0;
        }
        atomicAdd(r_off + e, 1);
      }
      if (bad) set_error(p.err, kErrDeviceInput);
    }
    __syncthreads();
    {
      // offsets (exclusive scan of the counts), cursors and groups, one chunk of
      // 32 experts per warp at a time (lane l takes expert 32c + l:
      // conflict-free shared accesses): the first pass scans within each chunk
      // and records the chunk's totals, the second adds the totals of the
      // chunks before it.  Groups in ascending expert order after the shared
      // ones.
      const int gsz = p.ntmax;
      const int nsg = p.has_shared && p.with_shared ? (T + gsz - 1) / gsz : 0;
      const int nchk = (E + 31) >> 5;  // <= 32
      int* tot = reinterpret_cast<int*>(red);  // [chunk]: pairs, groups (red is free until the units)
      // groups of expert e's n pairs: ceil(n / gsz) for gsz in 1..4 without a
      // runtime division; none for an expert outside [e_begin, e_end)
      auto ngroups = [&](int e, int n) {
        if (e >= E || e < p.e_begin || e >= p.e_end) return 0;
        return gsz == 1 ? n : gsz == 2 ? (n + 1) >> 1 : gsz == 3 ? (n + 2) / 3 : (n + 3) >> 2;
      };
      for (int c = warp; c < nchk; c += kDecWarps) {
        const int e = 32 * c + lane;
        const int n = e < E ? r_off[e] : 0, ng = ngroups(e, n);
        int sc = n, sg = ng;  // inclusive warp scans
  #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int a = __shfl_up_sync(0xffffffffu, sc, o), b = __shfl_up_sync(0xffffffffu, sg, o);
          if (lane >= o) {
            sc += a;
            sg += b;
          }
        }
        if (e < E) r_cur[e] = (sc - n) | ((sg - ng) << 16);  // exclusive within the chunk (each < 2^16)
        if (lane == 31) {
          tot[2 * c] = sc;
          tot[2 * c + 1] = sg;
        }
      }
      __syncthreads();
      for (int c = warp; c < nchk; c += kDecWarps) {
        const int pc = __reduce_add_sync(0xffffffffu, lane < c ? tot[2 * lane] : 0);
        const int pg = __reduce_add_sync(0xffffffffu, lane < c ? tot[2 * lane + 1] : 0);
        const int e = 32 * c + lane;
        if (e < E) {
          const int n = r_off[e], w = r_cur[e];
          const int off = pc + (w & 0xffff);
          r_off[e] = off;
          r_cur[e] = off;
          if (ngroups(e, n) > 0)
            for (int q0 = 0, gi = nsg + pg + (w >> 16); q0 < n; q0 += gsz) r_groups[gi++] = make_int4(e, off + q0, min(gsz, n - q0), 0);
        }
      }
      if (warp == 0) {
        const int run = __reduce_add_sync(0xffffffffu, lane < nchk ? tot[2 * lane] : 0);
        const int ngr = __reduce_add_sync(0xffffffffu, lane < nchk ? tot[2 * lane + 1] : 0);
        if (lane == 0) {
          r_off[E] = run;
          misc[1] = nsg;
          misc[2] = ngr;
        }
        if (lane < nsg) r_groups[lane] = make_int4(-1, lane * gsz, min(gsz, T - lane * gsz), 0);
      }
      __syncthreads();
    }
    if (warp == 0) {
      // stable order within each expert: pairs in ascending flat index
      const unsigned lt = (1u << lane) - 1u;
      for (int c0 = 0; c0 < Tk; c0 += 32) {
        const int i = c0 + lane;
        int e = -1;
        if (i < Tk) {
          e = r_ids[i];
          if (e < 0 || e >= E) e = 0;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int base = 0;
        if (i < Tk) {
          base = r_cur[e];
          const int pos = base + __popc(peers & lt);
          r_sorted[pos] = i;
          r_inv[i] = pos;
        }
        __syncwarp();
        if (i < Tk && (peers >> lane) == 1u) r_cur[e] = base + __popc(peers);  // highest lane of its expert
        __syncwarp();
      }
    }
  }
  if (blockIdx.x == 0) {
    for (int i = tid; i < Tk; i += kDecThreads) {
      if (p.ids_out) p.ids_out[i] = r_ids[i];
      if (p.w_out) p.w_out[i] = r_w[i];
    }
  }
  __syncthreads();
  const int nsg = misc[1], nrg = misc[2];
  const int n_units = nsg * (p.fs / kDecRows) + nrg * (p.f / kDecRows) + (nsg + nrg) * (d / kDecRows2);
  const int fmax = max(p.f, p.fs);

  if (warp == kDecProducerWarp) {
    // ============================================================ producer
    DecRing rg{0, 0, 0};  // stages issued
    int np = 0;           // plane buffers issued
    if (lane == 0) {
      // units are claimed dynamically: the CTA's first is blockIdx.x, every
      // later one comes from the launch-wide counter
      int ui = blockIdx.x;
      while (!*abort_flag) {
        if (ui >= n_units) {
          // no more units: hand the consumers a -1 through the next plane buffer
          const int pb = np & 1;
          if (np >= 2 && !dec_wait_bar(pempty0 + 8 * pb, ((np >> 1) - 1) & 1, abort_flag, true)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          misc[8 + (np & 3)] = -1;
          dec_arrive(pfull0 + 8 * pb);
          ++np;
          break;
        }
        const DecUnit U = dec_unit(p, r_groups, nsg, nrg, ui);
        const int4 grp = r_groups[U.grp];
        const DecMat& m0 = p.m[U.mi];
        const bool s1 = U.stage == 1;
        const bool mx = m0.fmt == F_MX4;
        const int nsb = mx ? 1 : 2;
        const uint32_t box_bytes = (uint32_t)(m0.R * m0.seg);
        const uint32_t sc_bytes = (uint32_t)(m0.R * m0.spitch);
        const uint32_t tx = (s1 ? 2u : 1u) * (box_bytes + sc_bytes * nsb);
        const int nrs = s1 ? kDecRows / kDecR1 : kDecRows2 / kDecR2;
        const int nst = nrs * m0.nch;  // stages of the unit, row set by row set
        // one stage: codes of the row set's rows (and their W3 twins) and scales
        auto issue_stage = [&](int st) -> bool {
          const int rs = st / m0.nch, chn = st - rs * m0.nch;
          const int s = rg.s;
          if (rg.n >= p.nslot && !dec_wait_bar(empty0 + 8 * s, rg.ph ^ 1, abort_flag, true)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
            return false;
          }
          const uint32_t slot = ring + s * p.slot_bytes, full = full0 + 8 * s;
          const int row = U.row0 + rs * m0.R;
          const int cx = chn * (m0.seg / m0.lb);
          const int sxe = chn * m0.sK;
          dec_expect_tx(full, tx);
          for (int mm = 0; mm < (s1 ? 2 : 1); ++mm) {
            const int mi = U.mi + mm;
            dec_tma_3d(slot + mm * box_bytes, &p.map[mi], 0, row, cx, full);
            const uint32_t sb = slot + kDecCodeBytes + mm * nsb * sc_bytes;
            dec_tma_2d(sb, &p.smap[mi], sxe, row, full);
            if (!mx) dec_tma_2d(sb + sc_bytes, &p.bmap[mi], sxe, row, full);
          }
          rg.next(p.nslot);
          return true;
        };
        int st = 0;
        if (!s1) {
          // W2 weights do not depend on h: fill the ring with the unit's first
          // stages, then wait until the group's S1 units are all counted
          for (; st < nst && st < p.nslot; ++st)
            if (!issue_stage(st)) break;
          if (*abort_flag) break;
          const int target = p.stall_test ? 0x3fffffff : (grp.x < 0 ? p.fs / kDecRows : p.f / kDecRows);
          if (!dec_wait_count(p.cnt_h + U.grp, target, abort_flag, p.stall_test ? 2000000LL : kDecWaitCycles)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          fence_proxy_async_global();
        }
        {
          // the unit's activation rows (planes and block records) for every token of the group
          const int pb = np & 1;
          if (np >= 2 && !dec_wait_bar(pempty0 + 8 * pb, ((np >> 1) - 1) & 1, abort_flag, true)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          const uint32_t pl = planes0 + pb * p.pbuf;
          const int nin = m0.n_in;
          misc[8 + (np & 3)] = ui;
          dec_expect_tx(pfull0 + 8 * pb, (uint32_t)grp.z * (uint32_t)(nin * 2 + (nin / 64) * 16));
          for (int i = 0; i < grp.z; ++i) {
            const uint8_t* src;
            const float4* ssrc;
            if (s1) {
              const int tok = dec_token(p, r_sorted, grp, i);
              src = p.xplanes + ((size_t)(grp.x < 0 ? 1 : 0) * T + tok) * d * 4;
              ssrc = p.xsx + (size_t)tok * (d / 64);
            } else {
              const int sl = dec_slot(p, r_sorted, grp, i);
              src = p.hplanes + (size_t)sl * fmax * 4;
              ssrc = p.hsx + (size_t)sl * (fmax / 64);
            }
            dec_bulk(pl + i * m0.ptok, src, nin * 2, pfull0 + 8 * pb);
            dec_bulk(pl + p.sx_off + i * m0.sxtok, ssrc, (nin / 64) * 16, pfull0 + 8 * pb);
          }
          ++np;
        }
        for (; st < nst; ++st)
          if (!issue_stage(st)) break;
        // the next unit is claimed only now: a unit claimed while this one
        // still streams could wait behind it while another CTA idles
        ui = p.G + atomicAdd(p.sync + 2, 1);
      }
      // drain: every issued copy must land before the block exits
      for (int q = max(0, rg.n - p.nslot); q < rg.n; ++q) {
        const long long t0 = clock64();
        while (!dec_try_wait(full0 + 8 * (q % p.nslot), (q / p.nslot) & 1) && clock64() - t0 < kDecWaitCycles) {
        }
      }
      for (int q = max(0, np - 2); q < np; ++q) {
        const long long t0 = clock64();
        while (!dec_try_wait(pfull0 + 8 * (q & 1), (q >> 1) & 1) && clock64() - t0 < kDecWaitCycles) {
        }
      }
    }
    __syncwarp();
  } else if (warp == kDecServiceWarp) {
    // ============================================================ service
    // Unit epilogues that wait on global memory, off the consumers' path:
    // S1: the h block of every token -> W2's planes, then the group's count.
    int* scr = reinterpret_cast<int*>(fx + kDecFxScr);
    for (int ne = 0;; ++ne) {
      const int eb = ne & 1;
      bool ok = !*abort_flag;
      if (ok && !dec_wait_bar(efull0 + 8 * eb, (ne >> 1) & 1, abort_flag, true)) {
        if (lane == 0) set_error(p.err, kErrTimeout);
        *abort_flag = 1;
        ok = false;
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      const int ui = misc[12 + eb];
      if (ui < 0) break;
      const DecUnit U = dec_unit(p, r_groups, nsg, nrg, ui);
      const int4 grp = r_groups[U.grp];
      if (U.stage == 1) {
        const float* hb = hbuf + eb * kDecMaxTok * kDecRows;
        const int f2 = grp.x < 0 ? p.m[DM_S2].fmt : p.m[DM_W2].fmt;
        for (int i = 0; i < grp.z; ++i) {
          const int sl = dec_slot(p, r_sorted, grp, i);
          uint8_t* dst = p.hplanes + (size_t)sl * fmax * 4 + (size_t)U.u * 64 * plane_bytes_per_input(f2);
          const float4 sx = dec_make_block(hb[i * kDecRows + 2 * lane], hb[i * kDecRows + 2 * lane + 1], perm_of(f2),
                                           dst, scr, p.err);
          if (lane == 0) p.hsx[(size_t)sl * (fmax / 64) + U.u] = sx;
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          red_release_add(p.cnt_h + U.grp, 1);
        }
      }
      __syncwarp();
      if (lane == 0) dec_arrive(eempty0 + 8 * eb);
    }
  } else {
    // ============================================================ consumers
    const int kq = warp;  // input slice (both row tiles)
    DecRing rg{0, 0, 0};
    int np = 0;
    for (int ne = 0;; ++ne) {
      // the unit comes with its plane buffer; warp 0's view decides for every warp
      const int pb = np & 1;
      const bool have_pl = dec_consumer_wait(pfull0 + 8 * pb, (np >> 1) & 1, abort_flag, p.err);
      if (tid == 0) misc[4] = have_pl ? misc[8 + (np & 3)] : -1;
      asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerThreads) : "memory");
      const int ui = misc[4];
      const int eb = ne & 1;
      bool have_e = true;
      if (ne >= 2) have_e = dec_consumer_wait(eempty0 + 8 * eb, ((ne >> 1) - 1) & 1, abort_flag, p.err);
      if (ui < 0) {  // no more units: tell the service warp
        if (tid == 0) misc[12 + eb] = -1;
        __syncwarp();
        if (lane == 0) dec_arrive(efull0 + 8 * eb);
        break;
      }
      const DecUnit U = dec_unit(p, r_groups, nsg, nrg, ui);
      const int4 grp = r_groups[U.grp];
      const DecMat& m0 = p.m[U.mi];
      const bool s1 = U.stage == 1;
      DecWarp q;
      const int nsb = m0.fmt == F_MX4 ? 1 : 2;
      q.R = m0.R;
      q.kq = kq;
      q.spitch = m0.spitch;
      q.ptok = m0.ptok;
      q.sxtok = m0.sxtok;
      if (s1) {  // tile t: A rows 0..7 = W1 rows t*8.., rows 8..15 = the same rows of W3
        q.a0 = 0;
        q.a8 = m0.R * m0.seg;
        q.r0 = q.r8 = 0;
        q.tstep = 8;
        q.s0 = kDecCodeBytes;
        q.s8 = kDecCodeBytes + nsb * m0.R * m0.spitch;
      } else {  // tile t: A rows 0..15 = W2 rows t*16..
        q.a0 = q.a8 = 0;
        q.r0 = 0;
        q.r8 = 8;
        q.tstep = 16;
        q.s0 = q.s8 = kDecCodeBytes;
      }
      const uint32_t pl = planes0 + pb * p.pbuf;
      dec_consume_any(m0.fmt, m0.group, m0.nbw, q, s1, m0.nch, m0.K, grp.z, ring, p.slot_bytes, p.nslot, pl,
                      pl + p.sx_off, full0, empty0, rg, have_pl, abort_flag, p.err, red);
      __syncwarp();
      if (lane == 0 && have_pl) dec_arrive(pempty0 + 8 * pb);
      ++np;
      asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerThreads) : "memory");  // every slice partial is in red
      for (int i = tid; i < kDecMaxTok * (s1 ? kDecRows : kDecRows2); i += kDecConsumerThreads) {
        const int r = i >> 2, tok = i & 3;  // the unit's output row, token
        if (tok < grp.z) {
          if (s1) {
            const int rs = r >> 4, row = r & 15;
            float v1 = 0.f, v3 = 0.f;
#pragma unroll
            for (int sl = 0; sl < kDecNkq; ++sl) {  // input slices in a fixed order
              const float2 pr = *reinterpret_cast<const float2*>(red + ((sl * 4 + rs) * 16 + row) * 8 + tok * 2);
              v1 += pr.x;
              v3 += pr.y;
            }
            if (have_e) hbuf[(eb * kDecMaxTok + tok) * kDecRows + r] = v1 / (1.f + expf(-v1)) * v3;  // silu(g) * u
          } else {
            const int rs = r >> 5, row = r & 31;
            float v = 0.f;
#pragma unroll
            for (int sl = 0; sl < kDecNkq; ++sl) v += red[((sl * 4 + rs) * 32 + row) * 4 + tok];  // fixed order
            p.y[(size_t)dec_slot(p, r_sorted, grp, tok) * d + kDecRows2 * U.u + r] = v;
          }
        }
      }
      if (tid == 0) misc[12 + eb] = ui;
      asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerThreads) : "memory");  // red is free, the h block complete
      if (lane == 0) dec_arrive(efull0 + 8 * eb);
    }
  }
  // ------------------------------------------------------------ combine
  // Every y slot is final once the whole grid is here: out = sum_j w y (+ the
  // shared expert), ascending j, one rounding; a thread per 4 columns of a
  // token, its k slot loads issued together.
  __syncthreads();
  dec_grid_barrier(p.sync, p.G, p.err, abort_flag);
  {
    const int nc4 = d / 4;
    for (int i = blockIdx.x * kDecThreads + tid; i < T * nc4; i += p.G * kDecThreads) {
      const int t = i / nc4, c4 = (i - t * nc4) * 4;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < k; j0 += 4) {
        float4 v[4];
        bool own[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          own[jj] = false;
          if (j0 + jj < k) {
            int e = r_ids[t * k + j0 + jj];
            if (e < 0 || e >= E) e = 0;  // as counted in P1
            own[jj] = e >= p.e_begin && e < p.e_end;
            if (own[jj]) v[jj] = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)(t * k + j0 + jj) * d + c4));
          }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          if (own[jj]) {
            const float wj = r_w[t * k + j0 + jj];
            a.x = fmaf(wj, v[jj].x, a.x);
            a.y = fmaf(wj, v[jj].y, a.y);
            a.z = fmaf(wj, v[jj].z, a.z);
            a.w = fmaf(wj, v[jj].w, a.w);
          }
        }
      }
      if (p.has_shared && p.with_shared) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)(Tk + t) * d + c4));
        a.x += v.x;
        a.y += v.y;
        a.z += v.z;
        a.w += v.w;
      }
      if (p.out_f32 != nullptr) {
        *reinterpret_cast<float4*>(p.out_f32 + (size_t)t * d + c4) = a;
        continue;
      }
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      uint2 o;
      o.x = *reinterpret_cast<const uint32_t*>(&lo);
      o.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p.out + (size_t)t * d + c4) = o;
    }
  }
  // every unit is done: the dependency counters start the next launch at zero
  if (blockIdx.x == 0) {
    for (int i = tid; i < nsg + nrg; i += kDecThreads) p.cnt_h[i] = 0;
    if (tid == 0) p.sync[2] = 0;  // the unit counter
  }
}

}  // namespace moe
