// Step 3 for large token counts (prefill): the grouped SwiGLU expert FFN as
// a grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM).
//
//   stage 1 (per expert e):  H[p, :] = silu(X[p] . W1[e]^T) * (X[p] . W3[e]^T)
//   stage 2 (per expert e):  Y[p, :] = H[p] . W2[e]^T
//
// for the sorted positions p of expert e [mlx-lm PR "Add DeepSeek-v4
// (Flash/Pro)": w1/w2/w3 = gate/down/up of the switch MLP; model card
// "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit": affine w = scale*q + bias;
// mxfp4 = e2m1 * 2^(e-127)].
//
// Operand precision: weights, activations and H enter the tensor cores as
// fp16 (11-bit significand) with fp32 accumulation.  bf16 operands (8-bit
// significand) would round every dequantised weight s*q+b by up to 2^-9
// relative, which alone uses most of the layer's output tolerance; fp16
// rounds by 2^-12 at the same tensor-core rate.  Values beyond the fp16 range
// (|v| > 65504) are reported through the device error word.
//
// Shape: weights are the MMA's A operand (M = 128 weight rows per tile,
// K-major), tokens are B (N <= 128 tokens per tile, K-major), so ragged
// per-expert token counts cost at most a multiple-of-16 N padding.  One
// persistent block per SM walks work items (token tile, weight-row tile);
// consecutive items share a token tile.  Warp roles (512 threads):
//   warps 0-7   A producers: thread (row r, half hh) prefetches its row's
//               packed codes and group scale/bias for 32 inputs a few stages
//               ahead (cp.async into a private ring), then dequantises them to
//               fp16 straight into the 128B-swizzled K-major tile;
//   warps 8-9   B producers: gather the stage's token rows (cp.async with
//               zero fill past the tile's last token), two stages in flight;
//   warp 10     allocates TMEM; one thread issues tcgen05.mma + commits;
//   warps 12-15 epilogue: tcgen05.ld the fp32 accumulators (TMEM lane =
//               weight row), SwiGLU -> H (stage 1) or y (stage 2).
// Accumulators are double-buffered in TMEM so the epilogue of one item
// overlaps the MMAs of the next.  Every wait is bounded: a timeout records
// MOE_ERR_TIMEOUT, the block drains its copies and MMAs and frees TMEM.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {

constexpr int kTcM = 128;   // weight rows per tile (MMA M)
constexpr int kTcN = 128;   // tokens per tile (MMA N <= 128, multiple of 16)
constexpr int kTcK = 64;    // inputs per stage: one 128-byte swizzle row of fp16
constexpr int kTcThreads = 16 * 32;
constexpr int kTcAThreads = 256;  // warps 0-7
constexpr int kTcBThreads = 64;   // warps 8-9
constexpr int kTcMmaWarp = 10;
constexpr int kTcEpiWarp0 = 12;   // warps 12-15: warp % 4 = TMEM lane quarter
constexpr int kTcATile = kTcM * kTcK * 2;  // 16 KB
constexpr int kTcBTile = kTcN * kTcK * 2;  // 16 KB
constexpr int kTcBLook = 2;                // B copy groups in flight
constexpr float kF16Max = 65504.f;

struct TcParams {
  const __half* x16;     // stage 1 input: token rows in position order [P, n_in] fp16
  const __half* hin;     // stage 2 input: H rows [P, ld_in] fp16
  __half* hout;          // stage 1 output: H [P, ld_h]
  float* yout;           // stage 2 output: y [P, ld_y]
  int ld_in, ld_h, ld_y;
  int T, k;
  QMatDev a0, a1;        // stage 1: w1, w3; stage 2: w2 (a1 = a0)
  const int* sorted_rows;  // routed launch: non-NULL (tiles from the plan); NULL: shared expert over T rows
  const int4* tiles;     // token tiles {expert, first position, tokens, 0} (routed)
  const int* n_tiles;    // number of routed token tiles (device)
  int pos_base;          // row offset of this launch's positions in H / y
  int* err;
};

// Compile-time shape of one kernel instance.
template <int STAGE, int FMT>
struct TcCfg {
  static constexpr int bits = FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
  static constexpr int M = STAGE == 1 ? 2 : 1;                 // weight matrices per stage
  static constexpr int S = STAGE == 1 ? 3 : 5;                 // tile stages
  static constexpr int HB = 32 * bits / 8;                     // packed bytes per thread per matrix
  static constexpr int PB = (HB + 7) / 8 * 8;                  // ... padded in the ring
  static constexpr int SCO = (M * PB + 15) / 16 * 16;          // offset of the scale/bias words
  static constexpr int SB = SCO + 16;                          // ring bytes per thread per slot
  static constexpr int R = (STAGE == 1 && SB >= 64) ? 3 : 4;   // ring slots
  static constexpr int L = R - 1;                              // prefetch distance (stages)
  static constexpr int stage_bytes = M * kTcATile + kTcBTile;
  static constexpr int ring_bytes = R * kTcAThreads * SB;
  static constexpr int bar_bytes = 256;
  static constexpr size_t smem = 1024 + (size_t)S * stage_bytes + ring_bytes + bar_bytes;
  static constexpr uint32_t tmem_cols = STAGE == 1 ? 512u : 256u;  // 2 buffers x M x 128 columns
  static_assert(smem <= 227 * 1024, "tensor-core FFN exceeds the per-block shared memory limit");
  static_assert(kTcBLook <= S - 1, "B prefetch distance must leave a free stage");
};

// ------------------------------------------------------------ PTX wrappers
MOE_DEV uint32_t tc_smem(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MOE_DEV void tc_bar_init(uint32_t b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(n) : "memory");
}
MOE_DEV void tc_bar_arrive(uint32_t b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
}
MOE_DEV bool tc_bar_try(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(b), "r"(parity), "r"(20000)
      : "memory");
  return ok != 0;
}
constexpr long long kTcWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz: every wait gives up after this
// Wait for the phase with this parity; false once the block has aborted or
// this wait timed out (which aborts the block).
MOE_DEV bool tc_bar_wait(uint32_t b, uint32_t parity, volatile int* abort_flag) {
  if (tc_bar_try(b, parity)) return true;
  const long long t0 = clock64();
  while (!tc_bar_try(b, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kTcWaitCycles) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}
// generic-proxy shared-memory writes of this thread -> visible to the tensor core
MOE_DEV void tc_fence_proxy() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

MOE_DEV void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// 16-byte copy that reads src_bytes (0 or 16) and zero-fills the rest
MOE_DEV void cp16z(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
MOE_DEV void cp8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
MOE_DEV void cp4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
MOE_DEV void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEV void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

MOE_DEV uint4 tc_lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
MOE_DEV uint2 tc_lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
MOE_DEV uint32_t tc_lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV void tc_sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// K-major, 128-byte swizzle: 16-byte chunk c (inputs 8c..8c+7) of tile row r
// lives at r*128 + ((c ^ (r % 8)) * 16) inside a 1024-byte aligned tile.
MOE_DEV uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// UMMA shared-memory descriptor for such a tile: start address >> 4, 8-row
// groups 1024 B apart (stride byte offset), descriptor version 1,
// SWIZZLE_128B; the leading byte offset is unused for swizzled K-major.
MOE_DEV uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor, kind::f16: fp16 A and B (format 0), fp32 D,
// both K-major, M = 128, N = n.
MOE_DEV uint32_t umma_idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}
MOE_DEV void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier once every MMA this thread issued so far has completed
MOE_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// 32 TMEM lanes x 16 consecutive 32-bit columns -> 16 registers per thread
MOE_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------ work items
// Item i covers token tile i / n_mt and weight-row tile i % n_mt.
MOE_DEV int4 tc_tile(const TcParams& p, int j) {
  if (!p.sorted_rows) {
    const int pos0 = j * kTcN;
    return make_int4(0, pos0, min(kTcN, p.T - pos0), 0);
  }
  return __ldcg(p.tiles + j);
}

// Walks this block's stages (items blockIdx.x, +gridDim.x, ...; k-tiles
// 0..n_kt-1 within each) and keeps the next item's tile loaded ahead.
struct TcCursor {
  int item, kt, mt;
  int4 tile, nxt;
  MOE_DEV void init(const TcParams& p, int n_items, int n_mt) {
    item = blockIdx.x;
    kt = 0;
    mt = item % n_mt;
    tile = item < n_items ? tc_tile(p, item / n_mt) : make_int4(0, 0, 0, 0);
    const int n2 = item + gridDim.x;
    nxt = n2 < n_items ? tc_tile(p, n2 / n_mt) : make_int4(0, 0, 0, 0);
  }
  // returns true when the step moved to a new item
  MOE_DEV bool advance(const TcParams& p, int n_items, int n_mt, int n_kt) {
    if (++kt < n_kt) return false;
    kt = 0;
    item += gridDim.x;
    mt = item % n_mt;
    tile = nxt;
    const int n2 = item + gridDim.x;
    if (n2 < n_items) nxt = tc_tile(p, n2 / n_mt);
    return true;
  }
};

// ------------------------------------------------------------ dequantisation
MOE_DEV uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
MOE_DEV __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
MOE_DEV uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c) { return h2u(__hfma2(u2h(a), u2h(b), u2h(c))); }
MOE_DEV uint32_t hmul2u(uint32_t a, uint32_t b) { return h2u(__hmul2(u2h(a), u2h(b))); }
MOE_DEV uint32_t lop_or_and(uint32_t x, uint32_t mask, uint32_t orv) { return (x & mask) | orv; }

// fp16 pairs: 0x6400 | v is 1024 + v exactly for v < 1024.
constexpr uint32_t kMagic = 0x64006400u;
constexpr uint32_t kOne = 0x3C003C00u;        // (1, 1)
constexpr uint32_t kNeg1024 = 0xE400E400u;    // (-1024, -1024)

// Affine: the 32 codes of one thread -> 16 fp16 pairs (inputs 2i, 2i+1 in
// out[i]) of s*q + b, each rounded once (fma).  s2/b2 = (s, s) / (b, b).
// The codes are first recovered exactly as fp16 integers: a code sitting at
// bit offset j of a half is 1024*2^-j... scaled back by an exact fma.
template <int FMT>
MOE_DEV void tc_dequant32(const uint32_t* w, uint32_t s2, uint32_t b2, uint32_t (&out)[16]) {
  if constexpr (FMT == F_A4) {
    // byte j of word i holds codes 8i+2j (low nibble) and 8i+2j+1 (high)
    const uint32_t sc = 0x2C003C00u;   // (1, 1/16)
    const uint32_t off = 0xD400E400u;  // (-1024, -64)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t x = __byte_perm(w[i], 0u, 0x4040u | (j << 8) | j);  // byte j in both halves
        const uint32_t t = lop_or_and(x, 0x00F0000Fu, kMagic);   // (1024 + q0, 1024 + 16 q1)
        out[4 * i + j] = hfma2u(hfma2u(t, sc, off), s2, b2);
      }
    }
  } else if constexpr (FMT == F_A8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t x0 = __byte_perm(w[i], 0x64u, 0x4140u);  // (1024 + q0, 1024 + q1)
      const uint32_t x1 = __byte_perm(w[i], 0x64u, 0x4342u);  // (1024 + q2, 1024 + q3)
      out[2 * i] = hfma2u(hfma2u(x0, kOne, kNeg1024), s2, b2);
      out[2 * i + 1] = hfma2u(hfma2u(x1, kOne, kNeg1024), s2, b2);
    }
  } else if constexpr (FMT == F_A2) {
    // byte j of word i holds codes 16i+4j .. 16i+4j+3 (2 bits each)
    const uint32_t sc01 = 0x34003C00u, off01 = 0xDC00E400u;  // (1, 1/4), (-1024, -256)
    const uint32_t sc23 = 0x24002C00u, off23 = 0xCC00D400u;  // (1/16, 1/64), (-64, -16)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t x = __byte_perm(w[i], 0u, 0x4040u | (j << 8) | j);
        const uint32_t t0 = lop_or_and(x, 0x000C0003u, kMagic);  // (1024 + q0, 1024 + 4 q1)
        const uint32_t t1 = lop_or_and(x, 0x00C00030u, kMagic);  // (1024 + 16 q2, 1024 + 64 q3)
        out[8 * i + 2 * j] = hfma2u(hfma2u(t0, sc01, off01), s2, b2);
        out[8 * i + 2 * j + 1] = hfma2u(hfma2u(t1, sc23, off23), s2, b2);
      }
    }
  } else if constexpr (FMT == F_A3) {
    // 96 bits: window m (codes 8m..8m+7) = bits 24m..24m+23
    uint32_t u[4];
    u[0] = w[0];
    u[1] = __funnelshift_r(w[0], w[1], 24);
    u[2] = __funnelshift_r(w[1], w[2], 16);
    u[3] = w[2] >> 8;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t v = u[m] >> (6 * i);
        const uint32_t t = ((v << 13) & 0x00070000u) | lop_or_and(v, 7u, kMagic);  // (1024 + q0, 1024 + q1)
        out[4 * m + i] = hfma2u(hfma2u(t, kOne, kNeg1024), s2, b2);
      }
    }
  }
}

// mxfp4: e2m1 code n -> fp16 bits (n&8)<<12 | (n&7)<<9 is 2^-14 * e2m1(n)
// (exponent field = the code's 2-bit exponent, including its subnormal 0.5);
// f2 = (2^(e-113), 2^(e-113)) restores the block scale 2^(e-127).
MOE_DEV void tc_dequant32_mx(const uint32_t* w, uint32_t f2, uint32_t (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t y = __byte_perm(w[i], 0u, 0x4440u | j);  // byte j alone
      const uint32_t mag = (y * 0x00200200u) & 0x0E000E00u;    // low code -> bits 9-11, high -> 25-27
      const uint32_t sgn = (y * 0x01001000u) & 0x80008000u;    // signs -> bits 15, 31
      out[4 * i + j] = hmul2u(mag | sgn, f2);
    }
  }
}

// ------------------------------------------------------------ the kernel
template <int STAGE, int FMT>
__global__ void __launch_bounds__(kTcThreads, 1) ffn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = TcCfg<STAGE, FMT>;
  constexpr int M = C::M, S = C::S, R = C::R, L = C::L;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw32 = tc_smem(smem_raw);
  const uint32_t tiles32 = (raw32 + 1023u) & ~1023u;        // swizzled tiles need 1024-byte alignment
  const uint32_t ring32 = tiles32 + (uint32_t)(S * C::stage_bytes);
  const uint32_t bar32 = ring32 + (uint32_t)C::ring_bytes;
  uint8_t* bar_gen = smem_raw + (bar32 - raw32);
  // barriers: full_a[S] (256 arrivals), full_b[S] (64), empty[S] (1 commit),
  // acc_full[2] (1 commit), acc_empty[2] (128), drain (1 commit)
  auto full_a = [&](int s) { return bar32 + 8u * s; };
  auto full_b = [&](int s) { return bar32 + 8u * (S + s); };
  auto empty = [&](int s) { return bar32 + 8u * (2 * S + s); };
  auto acc_full = [&](int b) { return bar32 + 8u * (3 * S + b); };
  auto acc_empty = [&](int b) { return bar32 + 8u * (3 * S + 2 + b); };
  const uint32_t drain = bar32 + 8u * (3 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_gen + 8 * (3 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_out = p.a0.n_out, n_in = p.a0.n_in;
  const int n_mt = n_out / kTcM;
  const int n_kt = n_in / kTcK;
  const int n_tiles = p.sorted_rows ? __ldcg(p.n_tiles) : (p.T + kTcN - 1) / kTcN;
  const int n_items = n_tiles * n_mt;
  const int my_items = (int)blockIdx.x < n_items ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = my_items * n_kt;  // stages this block runs

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      tc_bar_init(full_a(s), kTcAThreads);
      tc_bar_init(full_b(s), kTcBThreads);
      tc_bar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc_bar_init(acc_full(b), 1);
      tc_bar_init(acc_empty(b), 128);
    }
    tc_bar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTcMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(tmem_slot)),
                 "r"(C::tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 8) {
    // ================= A producers: thread (row r, half hh)
    const int r = tid >> 1, hh = tid & 1;
    const uint32_t my_ring = ring32 + (uint32_t)(tid * C::SB);
    TcCursor pf, cs;
    pf.init(p, n_items, n_mt);
    cs = pf;
    // issue the copies of one stage (packed codes + scale/bias words) into ring slot `slot`
    auto issue = [&](const TcCursor& c, int slot) {
      const uint32_t dst = my_ring + (uint32_t)(slot * kTcAThreads * C::SB);
      const size_t row = (size_t)c.tile.x * n_out + (size_t)c.mt * kTcM + r;
      const int k0 = c.kt * kTcK + 32 * hh;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const QMatDev& Q = m ? p.a1 : p.a0;
        const uint8_t* src =
            reinterpret_cast<const uint8_t*>(Q.q) + row * (size_t)Q.wpr * 4 + (size_t)k0 * C::bits / 8;
        const uint32_t d = dst + (uint32_t)(m * C::PB);
        if constexpr (C::bits == 8) {
          cp16(d, src);
          cp16(d + 16, src + 16);
        } else if constexpr (C::bits == 4) {
          cp16(d, src);
        } else if constexpr (C::bits == 2) {
          cp8(d, src);
        } else {
          cp4(d, src);
          cp4(d + 4, src + 4);
          cp4(d + 8, src + 8);
        }
        // the aligned word holding this thread's group scale (and bias)
        const size_t gi = row * (size_t)Q.gpr + (size_t)(k0 / Q.group);
        if constexpr (FMT == F_MX4) {
          cp4(dst + C::SCO + 8 * m, reinterpret_cast<const uint8_t*>(Q.scales) + (gi & ~(size_t)3));
        } else {
          cp4(dst + C::SCO + 8 * m, reinterpret_cast<const uint8_t*>(Q.scales) + (gi & ~(size_t)1) * 2);
          cp4(dst + C::SCO + 8 * m + 4, reinterpret_cast<const uint8_t*>(Q.biases) + (gi & ~(size_t)1) * 2);
        }
      }
    };
    for (int g = 0; g < L; ++g) {
      if (g < total) {
        issue(pf, g % R);
        pf.advance(p, n_items, n_mt, n_kt);
      }
      cp_commit();
    }
    bool bad = false;
    for (int g = 0; g < total; ++g) {
      if (g + L < total) {
        issue(pf, (g + L) % R);
        pf.advance(p, n_items, n_mt, n_kt);
      }
      cp_commit();
      cp_wait<L>();  // this thread's copies of stage g have landed
      const int s = g % S;
      const int round = g / S;
      if (round > 0 && !tc_bar_wait(empty(s), (uint32_t)(round - 1) & 1u, abort_flag)) break;
      const uint32_t src = my_ring + (uint32_t)((g % R) * kTcAThreads * C::SB);
      const uint32_t tile = tiles32 + (uint32_t)(s * C::stage_bytes);
      const size_t row = (size_t)cs.tile.x * n_out + (size_t)cs.mt * kTcM + r;
      const int k0 = cs.kt * kTcK + 32 * hh;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const QMatDev& Q = m ? p.a1 : p.a0;
        const size_t gi = row * (size_t)Q.gpr + (size_t)(k0 / Q.group);
        uint32_t w[8];
        const uint32_t a = src + (uint32_t)(m * C::PB);
        if constexpr (C::bits == 8) {
          const uint4 v0 = tc_lds128(a), v1 = tc_lds128(a + 16);
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
          w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
        } else if constexpr (C::bits == 4) {
          const uint4 v0 = tc_lds128(a);
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        } else if constexpr (C::bits == 2) {
          const uint2 v0 = tc_lds64(a);
          w[0] = v0.x; w[1] = v0.y;
        } else {
          const uint2 v0 = tc_lds64(a);
          w[0] = v0.x; w[1] = v0.y; w[2] = tc_lds32(a + 8);
        }
        uint32_t out[16];
        if constexpr (FMT == F_MX4) {
          const uint32_t e = (tc_lds32(src + C::SCO + 8 * m) >> (8 * (gi & 3))) & 0xFFu;
          // 2^(e-113) as fp16: normal for e in [99, 128]; e > 128 overflows fp16
          // (flagged); e < 99 puts every weight of the block below 2^-25 (flushed)
          uint32_t f = 0;
          if (e > 128) bad = true;
          else if (e >= 99) f = (e - 98u) << 10;
          tc_dequant32_mx(w, f | (f << 16), out);
        } else {
          const uint32_t sw = tc_lds32(src + C::SCO + 8 * m), bw = tc_lds32(src + C::SCO + 8 * m + 4);
          const int sh = 16 * (int)(gi & 1);
          const float sf = __uint_as_float(((sw >> sh) & 0xFFFFu) << 16);
          const float bf = __uint_as_float(((bw >> sh) & 0xFFFFu) << 16);
          if (!(fabsf(sf) * (float)((1 << C::bits) - 1) + fabsf(bf) <= kF16Max)) bad = true;
          const __half hs = __float2half_rn(sf), hb = __float2half_rn(bf);
          tc_dequant32<FMT>(w, h2u(__halves2half2(hs, hs)), h2u(__halves2half2(hb, hb)), out);
        }
        const uint32_t t = tile + (uint32_t)(m * kTcATile);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc_sts128(t + sw128(r, 4 * hh + cc), out[4 * cc], out[4 * cc + 1], out[4 * cc + 2], out[4 * cc + 3]);
      }
      tc_fence_proxy();
      tc_bar_arrive(full_a(s));
      cs.advance(p, n_items, n_mt, n_kt);
    }
    cp_wait<0>();
    if (bad) set_error(p.err, kErrDeviceInput);
  } else if (warp < 10) {
    // ================= B producers: 64 threads, chunk c of rows q/8 + 8i
    const int q = tid - kTcAThreads;
    const int c = q & 7, n0 = q >> 3;
    TcCursor cur;
    cur.init(p, n_items, n_mt);
    const __half* rows = STAGE == 1 ? p.x16 : p.hin;
    const int ld = STAGE == 1 ? n_in : p.ld_in;
    for (int g = 0; g < total; ++g) {
      const int s = g % S;
      const int round = g / S;
      if (round > 0 && !tc_bar_wait(empty(s), (uint32_t)(round - 1) & 1u, abort_flag)) break;
      const uint32_t bt = tiles32 + (uint32_t)(s * C::stage_bytes + M * kTcATile);
      const int kofs = cur.kt * kTcK + 8 * c;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int n = n0 + 8 * i;
        const bool live = n < cur.tile.z;
        const __half* src = rows + (size_t)(p.pos_base + cur.tile.y + (live ? n : 0)) * ld + kofs;
        cp16z(bt + sw128(n, c), src, live ? 16u : 0u);
      }
      cp_commit();
      if (g >= kTcBLook) {
        cp_wait<kTcBLook>();
        tc_fence_proxy();
        tc_bar_arrive(full_b((g - kTcBLook) % S));
      }
      cur.advance(p, n_items, n_mt, n_kt);
    }
    cp_wait<0>();
    tc_fence_proxy();
    if (!*abort_flag)
      for (int g = max(0, total - kTcBLook); g < total; ++g) tc_bar_arrive(full_b(g % S));
  } else if (warp == kTcMmaWarp) {
    // ================= MMA issuer
    if (lane == 0) {
      TcCursor cur;
      cur.init(p, n_items, n_mt);
      int g = 0;
      for (int it = 0; it < my_items && !*abort_flag; ++it) {
        const int nt = (cur.tile.z + 15) & ~15;
        const uint32_t idesc = umma_idesc_f16(nt);
        const int ab = it & 1;
        if (it >= 2 && !tc_bar_wait(acc_empty(ab), (uint32_t)((it >> 1) - 1) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(ab * M * kTcN);
        bool ok = true;
        for (int kt = 0; kt < n_kt; ++kt, ++g) {
          const int s = g % S;
          const uint32_t par = (uint32_t)(g / S) & 1u;
          if (!tc_bar_wait(full_a(s), par, abort_flag) || !tc_bar_wait(full_b(s), par, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t at = tiles32 + (uint32_t)(s * C::stage_bytes);
          const uint32_t bt = at + (uint32_t)(M * kTcATile);
#pragma unroll
          for (int kk = 0; kk < kTcK / 16; ++kk) {  // K = 16 per MMA = 32 bytes along the swizzled row
            const uint64_t db = umma_desc(bt + 32u * kk);
#pragma unroll
            for (int m = 0; m < M; ++m)
              umma_f16(d0 + (uint32_t)(m * kTcN), umma_desc(at + (uint32_t)(m * kTcATile) + 32u * kk), db, idesc,
                       (kt | kk) ? 1u : 0u);
          }
          umma_commit(empty(s));  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(acc_full(ab));
        for (int kt = 0; kt < n_kt; ++kt) cur.advance(p, n_items, n_mt, n_kt);
      }
      // every MMA issued above has completed once the drain barrier flips
      umma_commit(drain);
      const long long t0 = clock64();
      while (!tc_bar_try(drain, 0) && clock64() - t0 < kTcWaitCycles) {
      }
    }
    __syncwarp();
  } else if (warp >= kTcEpiWarp0) {
    // ================= epilogue: TMEM lanes 32*(warp%4) .. +31 = weight rows
    const int qtr = warp & 3;
    const int r = qtr * 32 + lane;
    TcCursor cur;
    cur.init(p, n_items, n_mt);
    bool bad = false;
    for (int it = 0; it < my_items; ++it) {
      const int ab = it & 1;
      bool ok = tc_bar_wait(acc_full(ab), (uint32_t)(it >> 1) & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(qtr * 32) << 16) + (uint32_t)(ab * M * kTcN);
      const int wrow = cur.mt * kTcM + r;
      const int prow0 = p.pos_base + cur.tile.y;
      const int ntok = cur.tile.z;
      for (int nb = 0; nb < ntok; nb += 16) {
        float g16[16];
        tmem_ld16(tbase + (uint32_t)nb, g16);
        if constexpr (STAGE == 1) {
          float u16[16];
          tmem_ld16(tbase + (uint32_t)(kTcN + nb), u16);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (nb + j < ntok) {
              const float gv = g16[j];
              const float hv = __fdividef(gv * u16[j], 1.f + __expf(-gv));  // silu(g) * u
              bad |= !(fabsf(hv) <= kF16Max);
              p.hout[(size_t)(prow0 + nb + j) * p.ld_h + wrow] = __float2half_rn(hv);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (nb + j < ntok) p.yout[(size_t)(prow0 + nb + j) * p.ld_y + wrow] = g16[j];
        }
      }
      tc_fence_before();
      tc_bar_arrive(acc_empty(ab));
      for (int kt = 0; kt < n_kt; ++kt) cur.advance(p, n_items, n_mt, n_kt);
    }
    if (bad) set_error(p.err, kErrDeviceInput);
  }
  __syncthreads();
  if (tid == 0 && *abort_flag) set_error(p.err, kErrTimeout);
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::tmem_cols)
                 : "memory");
  }
}

// Launch helpers, one translation unit per (stage, format).
using TcLaunchFn = bool (*)(const TcParams& p, int grid, cudaStream_t s);
using TcAttrFn = void (*)();
#define MOE_TC_DECL(ST, F)                                                    \
  bool launch_tc_s##ST##_##F(const TcParams& p, int grid, cudaStream_t s); \
  void attrs_tc_s##ST##_##F();
MOE_TC_DECL(1, A2)
MOE_TC_DECL(1, A3)
MOE_TC_DECL(1, A4)
MOE_TC_DECL(1, A8)
MOE_TC_DECL(1, MX4)
MOE_TC_DECL(2, A2)
MOE_TC_DECL(2, A3)
MOE_TC_DECL(2, A4)
MOE_TC_DECL(2, A8)
MOE_TC_DECL(2, MX4)
#undef MOE_TC_DECL

}  // namespace moe
