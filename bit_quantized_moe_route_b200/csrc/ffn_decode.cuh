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
//   P1  every CTA, redundantly: top-k of every token, the stable grouping of
//       the (token, slot) pairs by expert, and "groups" of <= 8 tokens of one
//       expert (the shared expert's tokens form their own groups);
//   S1  units (group, 64 rows of d_ff): h = silu(W1 x) * (W3 x) for the
//       group's tokens, written as the planes W2 reads; a per-group counter
//       counts finished units;
//   S2  units (group, 64 rows of d_model): y = W2 h, started once the
//       group's S1 units are all counted; the CTA that finishes the last unit
//       of an output row block sums the k slots of every token in ascending
//       j, adds the shared expert and writes bf16 (one rounding).
// Units are dealt round-robin over the CTAs in the order [S1 shared, S1
// routed, S2 by group], so every CTA does the same amount of streaming.
//
// Inside a CTA one producer warp streams each unit's weights into a 3-slot
// ring, one stage = 512 code bytes of each of 32 rows of W1 and of W3 (S1;
// a unit's 64 rows are two halves) or of 64 rows of W2 (S2), as 128-byte
// wide TMA boxes with the 128-byte swizzle (3-bit: 96-byte unswizzled
// boxes), plus the rows' scales and biases (TMA) and the activation planes
// of the group's tokens (bulk copies).  Per-row runs of 512 bytes keep the
// weight stream near the copy rate (narrower runs cost DRAM and TMA
// efficiency).  16 consumer warps, one per (16-row tile, slice of the
// stage's inputs), unpack codes to bytes, run m16n8k32 integer MMAs against
// the planes (exact int32 sums per 64-input block) and fold each block into
// fp32 with the weight scale and bias.
// Every wait is bounded: on timeout the kernel records MOE_ERR_TIMEOUT, keeps
// every warp's barrier sequence, lets in-flight copies land and returns.
#pragma once

#include "dec_common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kDecConsumerWarps = 16;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecStages = 3;
constexpr int kDecRows = 64;        // weight rows per unit (S1: two halves of 32)
constexpr int kDecMaxTok = 4;       // tokens per group (B columns 0..3 of the MMA)
constexpr int kDecMaxT = 32;
constexpr int kDecMaxPairs = 256;   // T * top_k
constexpr int kDecStageRow = 512;   // code bytes per row and stage (3-bit: 384)
constexpr int kDecScaleRow = 64;    // scale (or bias) bytes per row and stage, at most
constexpr int kDecPlaneStride = 4160;  // per token and stage: <= 4096 plane bytes + bank padding
constexpr int kDecSxStride = 512;      // per token and stage: <= 32 blocks x (step, sum lo, sum hi, sum)
constexpr int kDecSlotCodes = 0;       // 32 KB: S1 32 rows x 512 B x 2 matrices, S2 64 rows x 512 B
constexpr int kDecSlotScales = 32768;  // 8 KB: scales and biases
constexpr int kDecSlotPlanes = kDecSlotScales + 8192;
constexpr int kDecSlotSx = kDecSlotPlanes + kDecMaxTok * kDecPlaneStride;
constexpr int kDecSlotBytes = ((kDecSlotSx + kDecMaxTok * kDecSxStride) + 1023) / 1024 * 1024;
constexpr int kDecRedBytes = 16 * 2 * 16 * 8 * 4;  // 16 warps x 2 matrices x 16 rows x 8 columns
constexpr int kDecHBytes = kDecMaxTok * kDecRows * 4;
constexpr int kDecOffLen = 1028;   // offsets / active list entries (E + 1 <= 1025, padded to 16 bytes)
constexpr int kDecRouteBytes = 6 * kDecMaxPairs * 4 + 2 * kDecOffLen * 4 + (kDecMaxPairs + 8) * 16;
constexpr int kDecMiscBytes = 256;
constexpr size_t kDecSmem = 1024 + (size_t)kDecStages * kDecSlotBytes + kDecRedBytes + kDecHBytes + kDecRouteBytes +
                            kDecMiscBytes;
static_assert(kDecSmem <= 227 * 1024, "fused decode kernel exceeds the per-block shared memory limit");
static_assert((kDecRedBytes + kDecHBytes) % 16 == 0 && (6 * kDecMaxPairs * 4 + 2 * kDecOffLen * 4) % 16 == 0,
              "the group records (int4) must stay 16-byte aligned");

// One packed matrix as the fused kernel reads it.
struct DecMat {
  int fmt, group, n_out, n_in;
  int rows;       // rows per stage: 32 (W1, W3) or 64 (W2)
  int box;        // TMA box width in bytes (128 swizzled, or 96 unswizzled for 3-bit); 4 boxes per stage
  int ks;         // inputs per stage
  int sbytes;     // scale (and bias) bytes per row and stage
};

enum DecMatIdx { DM_W1 = 0, DM_W3 = 1, DM_W2 = 2, DM_S1 = 3, DM_S3 = 4, DM_S2 = 5 };

struct DecParams {
  CUtensorMap map[6];   // codes of w1, w3, w2, shared w1, w3, w2
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
  int G;               // grid size
  // workspace
  float* logits;       // [T][E]
  int* hids;           // [T][k] (hash)
  float* hw;           // [T][k] (hash)
  uint8_t* xplanes;    // [2][T][d*4]: planes for the routed (0) and shared (1) W1/W3 formats
  float4* xsx;         // [T][d/64]: (step, sum of inputs 0..31, sum of 32..63, sum)
  uint8_t* hplanes;    // [P][fmax*4]
  float4* hsx;         // [P][fmax/64]
  float* y;            // [P][d]
  int* cnt_h;          // [kDecMaxPairs + 8]
  int* cnt_y;          // [d/64]
  int* sync;           // [0] barrier count, [1] barrier generation, [2] exit count
  int* err;
  __nv_bfloat16* out;  // [T][d]
  int* ids_out;        // [T][k] or NULL
  float* w_out;        // [T][k] or NULL
  int stall_test;      // testing the timeout path: the first W2 dependency waits on a count nothing reaches
};

// ------------------------------------------------------------ grid barrier
// Generation barrier over the whole (co-resident) grid; bounded wait.
MOE_DEV void dec_grid_barrier(int* sync, int nblocks, int* err, volatile int* abort_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* gen = sync + 1;
    const int my_gen = *gen;
    __threadfence();
    if (atomicAdd(sync, 1) == nblocks - 1) {
      sync[0] = 0;
      __threadfence();
      atomicAdd(sync + 1, 1);
    } else {
      const long long t0 = clock64();
      while (*gen == my_gen) {
        if (clock64() - t0 > kDecWaitCycles) {
          set_error(err, kErrTimeout);
          *abort_flag = 1;
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence();
  }
  __syncthreads();
}

// ------------------------------------------------------------ P0: planes
// The planes of one 64-input block of one activation row (64 values, two
// per lane, already in registers; lane l holds inputs 2l, 2l+1): warp-wide.
// `q_scratch`: 64 ints of this warp's shared scratch.  Writes the records of
// `perm` (and the negated records for mxfp4) at `dst` (2 k-blocks x 4
// threads) and returns (step, dequantised sum of inputs 0..31, of 32..63, of
// all 64) to every lane.
MOE_DEV float4 dec_make_block(float v0, float v1, int perm, bool with_neg, uint8_t* dst, int* q_scratch,
                              int* err) {
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
    uint32_t rec[2][4];  // [sign][hi b0, hi b1, lo b0, lo b1]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t hp = 0, lp = 0, hn = 0, ln = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = q_scratch[plane_input(perm, kb2, t, h, j)];
        hp |= (uint32_t)((q >> 8) & 0xFF) << (8 * j);
        lp |= (uint32_t)(q & 0xFF) << (8 * j);
        hn |= (uint32_t)(((-q) >> 8) & 0xFF) << (8 * j);
        ln |= (uint32_t)((-q) & 0xFF) << (8 * j);
      }
      rec[0][h] = hp;
      rec[0][2 + h] = lp;
      rec[1][h] = hn;
      rec[1][2 + h] = ln;
    }
    const int rb = with_neg ? 32 : 16;
    uint4* d0 = reinterpret_cast<uint4*>(dst + kb2 * 4 * rb + t * rb);
    d0[0] = make_uint4(rec[0][0], rec[0][1], rec[0][2], rec[0][3]);
    if (with_neg) d0[1] = make_uint4(rec[1][0], rec[1][1], rec[1][2], rec[1][3]);
  }
  __syncwarp();
  return make_float4(sc.y, sc.y * (float)s_lo, sc.y * (float)s_hi, sc.y * (float)(s_lo + s_hi));
}

// ------------------------------------------------------------ A operands
// Stage layout of one matrix's codes: 4 TMA boxes side by side along the row
// (box b = bytes [b*box, (b+1)*box) of each of `rows` rows), each box `rows`
// lines of `box` bytes; 128-byte boxes are swizzled (16-byte chunk c of line
// r sits at chunk c ^ (r & 7)), so the 8 rows an ldmatrix phase reads hit
// distinct banks.
struct DecTile {
  uint32_t codes;  // shared address of the matrix's first box
  int rows;        // lines per box
  int rt;          // 16-row tile
  int byte0;       // first code byte (in the stage row) of this warp's slice
};

MOE_DEV uint32_t swz(uint32_t box, int row, int chunk) {
  return box + (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
// ldmatrix x4 of two 16-byte chunks (bytes `byte`, `byte`+16 of the stage row)
// of the tile's rows: d[0] = (row g, chunk 0), d[1] = (g+8, chunk 0),
// d[2] = (g, chunk 1), d[3] = (g+8, chunk 1)
MOE_DEV void dec_ldsm2(const DecTile& tl, int byte, uint32_t (&d)[4]) {
  const int lane = threadIdx.x & 31, mtx = lane >> 3;
  const int row = tl.rt * 16 + (mtx & 1) * 8 + (lane & 7);
  const int b = byte + (mtx >> 1) * 16;
  ldsm_x4(swz(tl.codes + (b >> 7) * tl.rows * 128, row, (b & 127) >> 4), d[0], d[1], d[2], d[3]);
}

// ldmatrix x2 of one 16-byte chunk of the tile's rows: d[0] = row g, d[1] = row g+8
MOE_DEV void dec_ldsm1(const DecTile& tl, int byte, uint32_t (&d)[4]) {
  const int lane = threadIdx.x & 31;
  const int row = tl.rt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(d[0]), "=r"(d[1])
               : "r"(swz(tl.codes + (byte >> 7) * tl.rows * 128, row, (byte & 127) >> 4)));
}

// per format: bits per code, and how a k-block's codes become A registers
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
MOE_DEV void unpack_a2(uint32_t wg, uint32_t wg8, int kb2, uint32_t (&a)[4]) {
  const int s0 = 4 * kb2, s1 = 4 * kb2 + 2;
  a[0] = (wg >> s0) & 0x03030303u;
  a[1] = (wg8 >> s0) & 0x03030303u;
  a[2] = (wg >> s1) & 0x03030303u;
  a[3] = (wg8 >> s1) & 0x03030303u;
}
// four 3-bit codes (12 bits) -> bytes 0..3
MOE_DEV uint32_t spread3x4(uint32_t t) {
  const uint32_t ev = ((t & 0x1C7u) * 0x401u) & 0x00070007u;
  const uint32_t od = ((t & 0xE38u) * 0x8020u) & 0x07000700u;
  return ev | od;
}
// codes 8t..8t+7 of k-block (12 bytes) starting at stage byte `byte` of `row`
// (unswizzled 96-byte boxes)
MOE_DEV uint32_t codes3x8(const DecTile& tl, int row, int byte, int t) {
  const int box = byte / 96, off = byte - box * 96;
  const uint32_t base = tl.codes + box * tl.rows * 96 + row * 96 + off;
  const int bt = 3 * t;
  const uint32_t w0 = lds32u(base + (bt & ~3)), w1 = lds32u(base + (bt & ~3) + 4);
  return __funnelshift_r(w0, w1, 8 * (bt & 3)) & 0xFFFFFFu;
}
MOE_DEV void load_a3(const DecTile& tl, int byte, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint32_t vg = codes3x8(tl, tl.rt * 16 + g, byte, t), vg8 = codes3x8(tl, tl.rt * 16 + 8 + g, byte, t);
  a[0] = spread3x4(vg & 0xFFFu);
  a[2] = spread3x4(vg >> 12);
  a[1] = spread3x4(vg8 & 0xFFFu);
  a[3] = spread3x4(vg8 >> 12);
}

// ------------------------------------------------------------ one stage
// Consumer warp (rt, kq) over its slice of one stage: integer MMAs per
// k-block, folded into acc[m][4] once per 64-input block (or per 32-input
// group).  ntok tokens occupy B columns 0..ntok-1.
struct DecStageCtx {
  uint32_t slot;        // shared address of the stage slot
  int rt, kq, ntok;
  int group, ks, rows;  // of the unit's matrices
};

template <int FMT>
MOE_DEV void dec_scale_bias(const DecStageCtx& c, int m, int grp, int row, int sbytes, float& s, float& b) {
  const uint32_t sc = c.slot + kDecSlotScales + m * 4096 + row * sbytes;
  if constexpr (FMT == F_MX4) {
    const uint32_t e = lds8u(sc + grp);
    // 2^(e-127) / 2 (the A operand holds 2*e2m1)
    s = __uint_as_float(e > 1 ? ((e - 1) << 23) : (e ? 0x00400000u : 0x00200000u));
    b = 0.f;
  } else {
    s = bf16_bits_to_float(lds16u(sc + 2 * grp));
    b = bf16_bits_to_float(lds16u(sc + c.rows * kDecScaleRow + 2 * grp));
  }
}

// acc[0..3] += s_r * step_c * P_rc + b_r * sum_c for the C-fragment layout
// (rows g, g+8; columns 2t, 2t+1) of one group; `si` selects the sum over
// the group's inputs in the (step, sum lo, sum hi, sum) record of the block
template <int FMT>
MOE_DEV void dec_fold(const DecStageCtx& c, int m, int grp, int sbytes, int bs, int si, const int (&ch)[4],
                      const int (&cl)[4], float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int r0 = c.rt * 16 + g, r1 = r0 + 8;
  const int c0 = 2 * t, c1 = c0 + 1;
  const uint32_t sx = c.slot + kDecSlotSx + bs * 16;
  const float st0 = c0 < c.ntok ? lds_f32(sx + c0 * kDecSxStride) : 0.f;
  const float st1 = c1 < c.ntok ? lds_f32(sx + c1 * kDecSxStride) : 0.f;
  const float sm0 = c0 < c.ntok ? lds_f32(sx + c0 * kDecSxStride + 4 * si) : 0.f;
  const float sm1 = c1 < c.ntok ? lds_f32(sx + c1 * kDecSxStride + 4 * si) : 0.f;
  float s0, b0, s1, b1;
  dec_scale_bias<FMT>(c, m, grp, r0, sbytes, s0, b0);
  dec_scale_bias<FMT>(c, m, grp, r1, sbytes, s1, b1);
  acc[0] = fmaf(s0 * st0, (float)(ch[0] * 256 + cl[0]), fmaf(b0, sm0, acc[0]));
  acc[1] = fmaf(s0 * st1, (float)(ch[1] * 256 + cl[1]), fmaf(b0, sm1, acc[1]));
  acc[2] = fmaf(s1 * st0, (float)(ch[2] * 256 + cl[2]), fmaf(b1, sm0, acc[2]));
  acc[3] = fmaf(s1 * st1, (float)(ch[3] * 256 + cl[3]), fmaf(b1, sm1, acc[3]));
}

// M = 2: S1 (W1, W3; 2 tiles x 8 slices of 64 code bytes); M = 1: S2 (W2; 4
// tiles x 4 slices of 128 code bytes).  3-bit: slices of 48 / 96 bytes.
template <int FMT, int M>
MOE_DEV void dec_stage(const DecStageCtx& c, float (&acc)[2][4]) {
  constexpr int BITS = DecA<FMT>::bits;
  constexpr int WB = (FMT == F_A3 ? 48 : 64) * (M == 2 ? 1 : 2);  // code bytes of this warp per row
  constexpr int KBW = WB * 8 / BITS / 32;                         // k-blocks of this warp
  constexpr int KBB = 32 * BITS / 8;                              // code bytes per k-block and row
  constexpr bool MX = FMT == F_MX4;
  constexpr int REC = MX ? 32 : 16;  // plane record bytes per (k-block, thread)
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const bool live = g < c.ntok;
  const int pstride = c.ks * plane_bytes_per_input(FMT) + (MX ? 16 : 64);
  const uint32_t planes = c.slot + kDecSlotPlanes + (uint32_t)(live ? g : 0) * pstride + t * REC;
  const int group = c.group;
  const bool g32 = group == 32;  // 32-input groups: each k-block has its own scale
  const int sbytes = c.ks / group * (MX ? 1 : 2);
  const int kb0 = c.kq * KBW;    // first k-block (within the stage) of this warp
  const int byte0 = c.kq * WB;   // first code byte (within the stage row) of this warp
#pragma unroll
  for (int blk = 0; blk < KBW / 2; ++blk) {  // 64-input blocks
    const int kbs = kb0 + 2 * blk;           // stage k-block of the block's first half
    const int bs = kbs >> 1;                 // stage block index
    const int byte = byte0 + 2 * blk * KBB;  // the block's first code byte
#pragma unroll
    for (int m = 0; m < M; ++m) {
      DecTile tl;
      tl.codes = c.slot + kDecSlotCodes + m * 16384;
      tl.rows = c.rows;
      tl.rt = c.rt;
      int ch[4] = {0, 0, 0, 0}, cl[4] = {0, 0, 0, 0};
      uint32_t w[4];
      if constexpr (FMT == F_A4 || FMT == F_MX4) dec_ldsm2(tl, byte, w);  // both k-blocks
      if constexpr (FMT == F_A2) dec_ldsm1(tl, byte, w);                  // the block is one chunk
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 B = live ? lds128u(planes + (kbs + h) * 4 * REC) : make_uint4(0, 0, 0, 0);
        uint32_t a[4];
        if constexpr (FMT == F_A4) {
          unpack_a4(w[2 * h], w[2 * h + 1], a);
        } else if constexpr (FMT == F_MX4) {
          uint32_t an[4];
          unpack_mx4(w[2 * h], w[2 * h + 1], a, an);
          const uint4 Bn = live ? lds128u(planes + (kbs + h) * 4 * REC + 16) : make_uint4(0, 0, 0, 0);
          mma_u8s8(ch, an, Bn.x, Bn.y);
          mma_u8u8(cl, an, Bn.z, Bn.w);
        } else if constexpr (FMT == F_A8) {
          dec_ldsm2(tl, byte + h * 32, a);  // one k-block = two chunks
        } else if constexpr (FMT == F_A2) {
          unpack_a2(w[0], w[1], h, a);
        } else {
          load_a3(tl, byte + h * KBB, a);
        }
        mma_u8s8(ch, a, B.x, B.y);
        mma_u8u8(cl, a, B.z, B.w);
        if (g32) {  // fold each 32-input group on its own
          dec_fold<FMT>(c, m, kbs + h, sbytes, bs, 1 + h, ch, cl, acc[m]);
#pragma unroll
          for (int q = 0; q < 4; ++q) ch[q] = cl[q] = 0;
        }
      }
      if (!g32) dec_fold<FMT>(c, m, (bs * 64) / group, sbytes, bs, 3, ch, cl, acc[m]);
    }
  }
}

}  // namespace moe

namespace moe {

MOE_DEV void dec_stage_any(int fmt, int M, const DecStageCtx& c, float (&acc)[2][4]) {
  if (M == 2) {
    switch (fmt) {
      case F_A2: dec_stage<F_A2, 2>(c, acc); break;
      case F_A3: dec_stage<F_A3, 2>(c, acc); break;
      case F_A4: dec_stage<F_A4, 2>(c, acc); break;
      case F_A8: dec_stage<F_A8, 2>(c, acc); break;
      default: dec_stage<F_MX4, 2>(c, acc); break;
    }
  } else {
    switch (fmt) {
      case F_A2: dec_stage<F_A2, 1>(c, acc); break;
      case F_A3: dec_stage<F_A3, 1>(c, acc); break;
      case F_A4: dec_stage<F_A4, 1>(c, acc); break;
      case F_A8: dec_stage<F_A8, 1>(c, acc); break;
      default: dec_stage<F_MX4, 1>(c, acc); break;
    }
  }
}

// Routing results and work groups, shared by every CTA (built in P1).
struct DecRoute {
  int* ids;     // [T*k]
  float* w;     // [T*k]
  int* sorted;  // [T*k] flat pair indices grouped by expert
  int* inv;
  int* ev;
  int* first;
  int* off;     // [E+1]
  int* active;  // [1 + E]
  int4* groups; // {expert or -1 (shared), start (sorted position / first token), tokens, 0}
};

struct DecUnit {
  int stage;  // 1 or 2
  int grp;
  int u;      // 64-row block of the unit's output rows
  int mi;     // first matrix index (DecMatIdx)
  int M;      // matrices (2: W1 and W3; 1: W2)
  int row0;   // first weight row in the stacked matrix
  int nchunks;  // stages along the inputs
  int nhalf;    // S1: the 64 rows come as two stages of 32 rows (per input chunk); S2: 1
};

MOE_DEV DecUnit dec_unit(const DecParams& p, const int4* groups, int nsg, int nrg, int i) {
  DecUnit U;
  const int ufs = p.fs / kDecRows, uf = p.f / kDecRows, ud = p.d / kDecRows;
  const int U1s = nsg * ufs, U1 = U1s + nrg * uf;
  if (i < U1) {
    U.stage = 1;
    U.M = 2;
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
    U.M = 1;
    U.grp = j / ud;
    U.u = j % ud;
    const bool sh = groups[U.grp].x < 0;
    U.mi = sh ? DM_S2 : DM_W2;
    U.row0 = (sh ? 0 : groups[U.grp].x * p.d) + kDecRows * U.u;
  }
  U.nchunks = p.m[U.mi].n_in / p.m[U.mi].ks;
  U.nhalf = U.stage == 1 ? 2 : 1;
  return U;
}

// Slot (flat index into the P = T*k + T activation rows) of token i of a group.
MOE_DEV int dec_slot(const DecParams& p, const DecRoute& R, int4 g, int i) {
  return g.x < 0 ? p.T * p.k + g.y + i : R.sorted[g.y + i];
}
MOE_DEV int dec_token(const DecParams& p, const DecRoute& R, int4 g, int i) {
  return g.x < 0 ? g.y + i : R.sorted[g.y + i] / p.k;
}

__global__ void __launch_bounds__(kDecThreads, 1) ffn_decode_kernel(const __grid_constant__ DecParams p) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  float* red = reinterpret_cast<float*>(ring + (size_t)kDecStages * kDecSlotBytes);
  float* hbuf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + kDecRedBytes);
  int* rbase = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(hbuf) + kDecHBytes);
  DecRoute R;
  R.ids = rbase;
  R.w = reinterpret_cast<float*>(rbase + kDecMaxPairs);
  R.sorted = rbase + 2 * kDecMaxPairs;
  R.inv = rbase + 3 * kDecMaxPairs;
  R.ev = rbase + 4 * kDecMaxPairs;
  R.first = rbase + 5 * kDecMaxPairs;
  R.off = rbase + 6 * kDecMaxPairs;
  R.active = R.off + kDecOffLen;
  R.groups = reinterpret_cast<int4*>(R.active + kDecOffLen);  // 16-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(R.groups) + (kDecMaxPairs + 8) * 16);
  volatile int* misc = reinterpret_cast<volatile int*>(bars + 2 * kDecStages);
  volatile int* abort_flag = misc;  // [0] abort, [1] groups shared, [2] groups routed, [3] last flag
  const uint32_t full0 = su32(bars), empty0 = su32(bars + kDecStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, k = p.k, E = p.E, d = p.d;
  const int Tk = T * k;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      dec_bar_init(full0 + 8 * s, 1);  // the producer's expect_tx arrive; the copies complete the transactions
      dec_bar_init(empty0 + 8 * s, kDecConsumerWarps);
    }
    misc[0] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // ------------------------------------------------------------ P0
  {
    // activation planes: (token, 64-input block) tasks over every warp of the grid
    const int nb = d / 64;
    const int gw = blockIdx.x * (kDecConsumerWarps + 1) + warp, W = p.G * (kDecConsumerWarps + 1);
    int* scratch = reinterpret_cast<int*>(red) + warp * 64;
    const int f0 = p.m[DM_W1].fmt, f1 = p.m[DM_S1].fmt;
    for (int it = gw; it < T * nb; it += W) {
      const int t = it / nb, b = it % nb;
      const uint32_t xv = __ldg(reinterpret_cast<const uint32_t*>(p.x + (size_t)t * d + 64 * b) + lane);
      const float v0 = bf16lo(xv), v1 = bf16hi(xv);
      uint8_t* d0 = p.xplanes + (size_t)t * d * 4 + (size_t)b * 64 * plane_bytes_per_input(f0);
      const float4 sx = dec_make_block(v0, v1, perm_of(f0), f0 == F_MX4, d0, scratch, p.err);
      if (p.has_shared) {
        uint8_t* d1 = p.xplanes + ((size_t)T + t) * d * 4 + (size_t)b * 64 * plane_bytes_per_input(f1);
        dec_make_block(v0, v1, perm_of(f1), f1 == F_MX4, d1, scratch, p.err);
      }
      if (lane == 0) p.xsx[(size_t)t * nb + b] = sx;
    }
    __syncthreads();
    if (!p.hash) {
      // router logits of experts blockIdx.x, +G, ... for every token (warps 0..15 split d)
      for (int e = blockIdx.x; e < E; e += p.G) {
        if (warp < kDecConsumerWarps) {
          const int span = d / kDecConsumerWarps;
          for (int t0 = 0; t0 < T; t0 += 8) {  // tokens in groups of 8 (registers)
            float acc[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] = 0.f;
            for (int i = warp * span + lane * 8; i < (warp + 1) * span; i += 256) {
              float wv[8];
              if (p.router_bf16) {
                const uint4 r = __ldg(reinterpret_cast<const uint4*>(
                    reinterpret_cast<const __nv_bfloat16*>(p.router_w) + (size_t)e * d + i));
                wv[0] = bf16lo(r.x); wv[1] = bf16hi(r.x); wv[2] = bf16lo(r.y); wv[3] = bf16hi(r.y);
                wv[4] = bf16lo(r.z); wv[5] = bf16hi(r.z); wv[6] = bf16lo(r.w); wv[7] = bf16hi(r.w);
              } else {
                const float4* rr = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.router_w) +
                                                                   (size_t)e * d + i);
                const float4 a = __ldg(rr), bq = __ldg(rr + 1);
                wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w;
                wv[4] = bq.x; wv[5] = bq.y; wv[6] = bq.z; wv[7] = bq.w;
              }
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                if (t0 + t < T) {
                  const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + t) * d + i));
                  float a = acc[t];
                  a = fmaf(wv[0], bf16lo(xv.x), a); a = fmaf(wv[1], bf16hi(xv.x), a);
                  a = fmaf(wv[2], bf16lo(xv.y), a); a = fmaf(wv[3], bf16hi(xv.y), a);
                  a = fmaf(wv[4], bf16lo(xv.z), a); a = fmaf(wv[5], bf16hi(xv.z), a);
                  a = fmaf(wv[6], bf16lo(xv.w), a); a = fmaf(wv[7], bf16hi(xv.w), a);
                  acc[t] = a;
                }
              }
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              if (t0 + t < T) {
                const float v = warp_sum(acc[t]);
                if (lane == 0) red[warp * kDecMaxT + t0 + t] = v;
              }
            }
          }
        }
        __syncthreads();
        if (tid < T) {
          float s = 0.f;
          for (int w = 0; w < kDecConsumerWarps; ++w) s += red[w * kDecMaxT + tid];  // fixed order
          p.logits[(size_t)tid * E + e] = s;
        }
        __syncthreads();
      }
    } else if ((int)blockIdx.x < T) {
      // hash routing of token blockIdx.x: table row, logits of its experts, weights
      const int t = blockIdx.x;
      int* s_e = reinterpret_cast<int*>(hbuf);
      int* s_ok = s_e + 32;
      if (warp == 0) {
        const int tok = p.token_ids[t];
        const bool tok_ok = tok >= 0 && tok < p.vocab;
        int e = 0;
        bool good = false;
        if (lane < k && tok_ok) {
          e = p.tid2eid[(size_t)tok * k + lane];
          good = e >= 0 && e < E;
          if (!good) e = 0;
        }
        if (__any_sync(0xffffffffu, !tok_ok || (lane < k && !good)) && lane == 0) set_error(p.err, kErrDeviceInput);
        s_e[lane] = e;
        s_ok[lane] = good ? 1 : 0;
      }
      __syncthreads();
      if (p.router_w != nullptr && warp < kDecConsumerWarps) {
        const int span = d / kDecConsumerWarps;
        for (int j0 = 0; j0 < k; j0 += 8) {  // the table's experts in groups of 8 (registers)
          float acc[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = 0.f;
          for (int i = warp * span + lane * 8; i < (warp + 1) * span; i += 256) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * d + i));
            const float xf[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                                 bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j0 + j < k) {
                const size_t off = (size_t)s_e[j0 + j] * d + i;
                float wv[8];
                if (p.router_bf16) {
                  const uint4 r = __ldg(reinterpret_cast<const uint4*>(
                      reinterpret_cast<const __nv_bfloat16*>(p.router_w) + off));
                  wv[0] = bf16lo(r.x); wv[1] = bf16hi(r.x); wv[2] = bf16lo(r.y); wv[3] = bf16hi(r.y);
                  wv[4] = bf16lo(r.z); wv[5] = bf16hi(r.z); wv[6] = bf16lo(r.w); wv[7] = bf16hi(r.w);
                } else {
                  const float4* rr = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.router_w) + off);
                  const float4 a = __ldg(rr), bq = __ldg(rr + 1);
                  wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w;
                  wv[4] = bq.x; wv[5] = bq.y; wv[6] = bq.z; wv[7] = bq.w;
                }
                float a = acc[j];
#pragma unroll
                for (int q = 0; q < 8; ++q) a = fmaf(wv[q], xf[q], a);
                acc[j] = a;
              }
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j0 + j < k) {
              const float v = warp_sum(acc[j]);
              if (lane == 0) red[warp * 32 + j0 + j] = v;
            }
          }
        }
      }
      __syncthreads();
      if (warp == 0) {
        float sj = 0.f;
        const bool gj = lane < k && s_ok[lane];
        if (gj) {
          if (p.router_w != nullptr) {
            float l = 0.f;
            for (int w = 0; w < kDecConsumerWarps; ++w) l += red[w * 32 + lane];
            sj = sqrt_softplus(l);
          } else {
            sj = 1.f;
          }
        }
        const float ssum = warp_sum(sj);
        if (lane < k) {
          p.hids[t * k + lane] = s_e[lane];
          p.hw[t * k + lane] = gj && ssum > 0.f ? sj / ssum : 0.f;
        }
      }
    }
  }
  dec_grid_barrier(p.sync, p.G, p.err, abort_flag);

  // ------------------------------------------------------------ P1
  if (!p.hash) {
    for (int t = warp; t < T; t += kDecConsumerWarps + 1) {
      if (E <= 32)
        topk_token<1>(p.logits + (size_t)t * E, p.router_b, E, k, R.ids + t * k, R.w + t * k);
      else if (E <= 256)
        topk_token<8>(p.logits + (size_t)t * E, p.router_b, E, k, R.ids + t * k, R.w + t * k);
      else
        topk_token<32>(p.logits + (size_t)t * E, p.router_b, E, k, R.ids + t * k, R.w + t * k);
    }
  } else {
    for (int i = tid; i < Tk; i += kDecThreads) {
      R.ids[i] = __ldcg(p.hids + i);
      R.w[i] = __ldcg(p.hw + i);
    }
  }
  __syncthreads();
  permute_ranks_block(R.ids, Tk, E, R.off, R.sorted, R.inv, R.active, p.err, R.ev, R.first);
  __syncthreads();
  if (tid == 0) {
    int ng = 0;
    if (p.has_shared)
      for (int t0 = 0; t0 < T; t0 += kDecMaxTok) R.groups[ng++] = make_int4(-1, t0, min(kDecMaxTok, T - t0), 0);
    const int nsg = ng;
    for (int a = 0; a < R.active[0]; ++a) {
      const int e = R.active[1 + a];
      const int cnt = R.off[e + 1] - R.off[e];
      for (int s0 = 0; s0 < cnt; s0 += kDecMaxTok) R.groups[ng++] = make_int4(e, R.off[e] + s0, min(kDecMaxTok, cnt - s0), 0);
    }
    misc[1] = nsg;
    misc[2] = ng - nsg;
  }
  if (blockIdx.x == 0) {
    for (int i = tid; i < Tk; i += kDecThreads) {
      if (p.ids_out) p.ids_out[i] = R.ids[i];
      if (p.w_out) p.w_out[i] = R.w[i];
    }
  }
  __syncthreads();
  const int nsg = misc[1], nrg = misc[2];
  const int n_units = nsg * (p.fs / kDecRows) + nrg * (p.f / kDecRows) + (nsg + nrg) * (d / kDecRows);
  const int fmax = max(p.f, p.fs);

  if (warp == kDecConsumerWarps) {
    // ============================================================ producer
    int n = 0;  // stages issued
    bool ok = true;
    for (int ui = blockIdx.x; ui < n_units && ok; ui += p.G) {
      const DecUnit U = dec_unit(p, R.groups, nsg, nrg, ui);
      const int4 grp = R.groups[U.grp];
      const DecMat& m0 = p.m[U.mi];
      const bool mx = m0.fmt == F_MX4;
      const int pb = plane_bytes_per_input(m0.fmt);
      const int pstride = m0.ks * pb + (mx ? 16 : 64);
      const uint32_t box_bytes = (uint32_t)(m0.rows * m0.box);
      const uint32_t sc_bytes = (uint32_t)(m0.rows * m0.sbytes);
      const uint32_t tx = (uint32_t)U.M * (4 * box_bytes + sc_bytes * (mx ? 1 : 2)) +
                          (uint32_t)grp.z * (m0.ks * pb + (m0.ks / 64) * 16);
      bool dep_ok = U.stage == 1;
      for (int st = 0; st < U.nhalf * U.nchunks; ++st, ++n) {
        const int half = st / U.nchunks, kc = st % U.nchunks;
        const int row0 = U.row0 + half * m0.rows;
        const int s = n % kDecStages;
        const uint32_t slot = su32(ring + (size_t)s * kDecSlotBytes);
        const uint32_t full = full0 + 8 * s, empty = empty0 + 8 * s;
        if (lane == 0) {
          if (n >= kDecStages && !dec_wait_bar(empty, ((n / kDecStages) - 1) & 1, abort_flag)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
          }
          if (!*abort_flag) {
            dec_expect_tx(full, tx);
            for (int mm = 0; mm < U.M; ++mm) {
              const int mi = U.mi + mm;
              const uint32_t cbase = slot + kDecSlotCodes + mm * 16384;
              for (int b = 0; b < 4; ++b)
                dec_tma_2d(cbase + b * box_bytes, &p.map[mi], kc * 4 * m0.box + b * m0.box, row0, full);
              const uint32_t sbase = slot + kDecSlotScales + mm * 4096;
              const int sx = kc * (m0.ks / m0.group);  // first scale entry of the stage
              dec_tma_2d(sbase, &p.smap[mi], sx, row0, full);
              if (!mx) dec_tma_2d(sbase + m0.rows * kDecScaleRow, &p.bmap[mi], sx, row0, full);
            }
            if (!dep_ok) {
              // W2 stages read the group's h planes: wait for all its S1 units.
              // (On a timeout the plane copies below are still issued -- they
              // stay in bounds -- so the stage's transaction count completes.)
              const int target = p.stall_test ? 0x3fffffff : (grp.x < 0 ? p.fs / kDecRows : p.f / kDecRows);
              if (!dec_wait_count(p.cnt_h + U.grp, target, abort_flag, p.stall_test ? 2000000LL : kDecWaitCycles)) {
                set_error(p.err, kErrTimeout);
                *abort_flag = 1;
              }
              fence_proxy_async_global();
              dep_ok = true;
            }
            for (int i = 0; i < grp.z; ++i) {
              const uint8_t* src;
              const float4* ssrc;
              if (U.stage == 1) {
                const int tok = dec_token(p, R, grp, i);
                const int layout = grp.x < 0 ? 1 : 0;
                src = p.xplanes + ((size_t)layout * T + tok) * d * 4;
                ssrc = p.xsx + (size_t)tok * (d / 64);
              } else {
                const int sl = dec_slot(p, R, grp, i);
                src = p.hplanes + (size_t)sl * fmax * 4;
                ssrc = p.hsx + (size_t)sl * (fmax / 64);
              }
              dec_bulk(slot + kDecSlotPlanes + i * pstride, src + (size_t)kc * m0.ks * pb, m0.ks * pb, full);
              dec_bulk(slot + kDecSlotSx + i * kDecSxStride, ssrc + (size_t)kc * (m0.ks / 64), (m0.ks / 64) * 16,
                       full);
            }
          }
        }
        __syncwarp();
        if (*abort_flag) {
          ok = false;
          break;
        }
      }
    }
    // drain: every issued copy must land before the block exits
    if (lane == 0) {
      for (int q = max(0, n - kDecStages); q < n; ++q) {
        const uint32_t full = full0 + 8 * (q % kDecStages);
        const long long t0 = clock64();
        while (!dec_try_wait(full, (q / kDecStages) & 1) && clock64() - t0 < kDecWaitCycles) {
        }
      }
    }
  } else {
    // ============================================================ consumers
    const int g = lane >> 2, t4 = lane & 3;
    int n = 0;
    for (int ui = blockIdx.x; ui < n_units; ui += p.G) {
      const DecUnit U = dec_unit(p, R.groups, nsg, nrg, ui);
      const int4 grp = R.groups[U.grp];
      const DecMat& m0 = p.m[U.mi];
      DecStageCtx c;
      // S1: 2 row tiles x 8 input slices; S2: 4 row tiles x 4 input slices
      c.rt = U.M == 2 ? (warp & 1) : (warp & 3);
      c.kq = U.M == 2 ? (warp >> 1) : (warp >> 2);
      c.ntok = grp.z;
      c.group = m0.group;
      c.ks = m0.ks;
      c.rows = m0.rows;
      const int fmt = m0.fmt;
      for (int half = 0; half < U.nhalf; ++half) {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        for (int kc = 0; kc < U.nchunks; ++kc, ++n) {
          const int s = n % kDecStages;
          const uint32_t full = full0 + 8 * s;
          bool have = !*abort_flag;
          if (have && !dec_wait_bar(full, (n / kDecStages) & 1, abort_flag)) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
            have = false;
          }
          have = __all_sync(0xffffffffu, have);  // the MMAs below need every lane
          if (have) {
            c.slot = su32(ring + (size_t)s * kDecSlotBytes);
            dec_stage_any(fmt, U.M, c, acc);
          }
          __syncwarp();
          if (lane == 0 && have) dec_arrive(empty0 + 8 * s);
        }
        // ---- sum the input slices of every (row, token) of this half
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          if (m < U.M) {
            float* dst = red + ((warp * 2 + m) * 16) * 8;
            dst[g * 8 + 2 * t4] = acc[m][0];
            dst[g * 8 + 2 * t4 + 1] = acc[m][1];
            dst[(g + 8) * 8 + 2 * t4] = acc[m][2];
            dst[(g + 8) * 8 + 2 * t4 + 1] = acc[m][3];
          }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerWarps * 32) : "memory");
        {
          const int nrt = U.M == 2 ? 2 : 4, nkq = kDecConsumerWarps / nrt;
          const int row = tid >> 3, tok = tid & 7;  // S1: rows 0..31 (tid < 256); S2: rows 0..63
          if (row < nrt * 16 && tok < grp.z) {
            const int rtt = row >> 4, rl = row & 15;
            float v[2] = {0.f, 0.f};
            for (int q = 0; q < nkq; ++q)
              for (int m = 0; m < U.M; ++m) v[m] += red[(((q * nrt + rtt) * 2 + m) * 16 + rl) * 8 + tok];
            if (U.stage == 1) {
              hbuf[tok * kDecRows + half * 32 + row] = v[0] / (1.f + expf(-v[0])) * v[1];  // silu(g) * u
            } else {
              const int sl = dec_slot(p, R, grp, tok);
              p.y[(size_t)sl * d + kDecRows * U.u + row] = v[0];
            }
          }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerWarps * 32) : "memory");
      }
      if (U.stage == 1) {
        // h of each token over these 64 rows -> one 64-input block of W2's planes
        if (warp < grp.z) {
          const int sl = dec_slot(p, R, grp, warp);
          const int f2 = grp.x < 0 ? p.m[DM_S2].fmt : p.m[DM_W2].fmt;
          const int pb = plane_bytes_per_input(f2);
          uint8_t* dst = p.hplanes + (size_t)sl * fmax * 4 + (size_t)U.u * 64 * pb;
          const float4 sx = dec_make_block(hbuf[warp * kDecRows + 2 * lane], hbuf[warp * kDecRows + 2 * lane + 1],
                                           perm_of(f2), f2 == F_MX4, dst, reinterpret_cast<int*>(red) + warp * 64,
                                           p.err);
          if (lane == 0) p.hsx[(size_t)sl * (fmax / 64) + U.u] = sx;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerWarps * 32) : "memory");
        if (tid == 0) {
          __threadfence();
          red_release_add(p.cnt_h + U.grp, 1);
        }
      } else {
        if (tid == 0) {
          __threadfence();
          const int done = atomicAdd(p.cnt_y + U.u, 1) + 1;
          const int last = done == nsg + nrg;
          if (last) __threadfence();
          misc[3] = last;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerWarps * 32) : "memory");
        if (misc[3]) {
          // every slot of this 64-column block is final: out = sum_j w y (+ shared), one rounding
          for (int i = tid; i < T * kDecRows; i += kDecConsumerWarps * 32) {
            const int t = i / kDecRows, col = kDecRows * U.u + (i % kDecRows);
            float sacc = 0.f;
            for (int j = 0; j < k; ++j) sacc = fmaf(R.w[t * k + j], __ldcg(p.y + (size_t)(t * k + j) * d + col), sacc);
            if (p.has_shared) sacc += __ldcg(p.y + (size_t)(Tk + t) * d + col);
            p.out[(size_t)t * d + col] = __float2bfloat16_rn(sacc);
          }
          asm volatile("bar.sync 1, %0;" ::"r"(kDecConsumerWarps * 32) : "memory");
          if (tid == 0) p.cnt_y[U.u] = 0;
        }
      }
    }
  }
  // ------------------------------------------------------------ exit
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(p.sync + 2, 1) == p.G - 1) {
      for (int i = 0; i < nsg + nrg; ++i) p.cnt_h[i] = 0;
      for (int i = 0; i < d / kDecRows; ++i) p.cnt_y[i] = 0;
      p.sync[2] = 0;
      __threadfence();
    }
  }
}

}  // namespace moe
