// Building blocks of the fused decode kernel (ffn_decode.cuh): legacy
// tensor-core integer MMA and ldmatrix wrappers, the fixed-point activation
// planes, TMA / bulk-copy issue helpers and bounded waits.
//
// Activation planes.  The expert contraction runs on the int8 tensor-core
// path (mma.sync m16n8k32, unsigned A x signed B): weights are the A operand
// as unsigned code bytes (or e2m1 magnitudes), activations the B operand.
// An activation row (x for W1/W3, the SwiGLU hidden row h for W2) is cut
// into blocks of 64 inputs; each block is held as a fixed-point vector
// xq = rint(v * 2^(140-E)) (E: largest fp32 exponent field in the block, so
// |xq| <= 2^14) split as xq = 256 * hi + lo with lo the sign-extended low
// byte (both planes signed bytes, |hi| <= 64), together with the block's
// step xs = 2^(E-140) and its dequantised sums xs * sum(xq).  For every
// 32-input k-block and quad thread t the planes are stored as the 16 bytes
// {hi b0, hi b1, lo b0, lo b1}, b0 holding k-slots 4t..4t+3 and b1 k-slots
// 16+4t..16+4t+3; which inputs sit in those k-slots depends on how the
// weight format's codes reach the A fragment (the "permutation" of the
// consuming format, see plane_input).  The MMA takes token j's hi plane as
// B column 2j and its lo plane as column 2j+1, so one MMA gives a thread
// both halves of its (row, token) sum: 256 * C[., 2j] + C[., 2j+1].
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------ permutations
// How the 32 inputs of a k-block map to (quad thread t, half h, byte j) of
// the B fragment, per consuming weight format.
enum PlanePerm : int {
  PERM_NATURAL = 0,  // 8-bit codes: h=0 -> 4t+j, h=1 -> 16+4t+j
  PERM_EVENODD = 1,  // 4-bit codes: word t holds codes 8t..8t+7; even codes -> h=0, odd -> h=1
  PERM_HALVES = 2,   // mxfp4 / 3-bit: h=0 -> 8t+j, h=1 -> 8t+4+j
  PERM_2BIT = 3      // 2-bit: a 64-input segment holds two k-blocks, see plane_input
};

MOE_DEV int perm_of(int fmt) {
  return fmt == F_A8 ? PERM_NATURAL : fmt == F_A4 ? PERM_EVENODD : fmt == F_A2 ? PERM_2BIT : PERM_HALVES;
}
__host__ __device__ inline int plane_bytes_per_input(int) { return 2; }

// Input index (within a 64-input block) of byte j of half h of quad thread
// t's B fragment, for k-block kb2 (0 or 1) of the block.
MOE_DEV int plane_input(int perm, int kb2, int t, int h, int j) {
  switch (perm) {
    case PERM_NATURAL: return 32 * kb2 + (h ? 16 : 0) + 4 * t + j;
    case PERM_EVENODD: return 32 * kb2 + 8 * t + 2 * j + h;
    case PERM_HALVES: return 32 * kb2 + 8 * t + 4 * h + j;
    default: return 16 * t + 4 * j + 2 * kb2 + h;  // PERM_2BIT: word t = inputs 16t..16t+15, shift 2*(2*kb2+h)
  }
}

// ------------------------------------------------------------ MMA / ldmatrix
// D += A(16x32, unsigned bytes) * B(32x8, signed / unsigned bytes), s32
MOE_DEV void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// four 8x(16 bytes) matrices; lane i gives the row address of matrix i/8,
// row i%8; lane (g, t) receives bytes 4t..4t+3 of row g of each matrix
MOE_DEV void ldsm_x4(uint32_t addr, uint32_t& d0, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
               : "r"(addr));
}
MOE_DEV uint4 lds128u(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
MOE_DEV uint2 lds64u(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds32u(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds16u(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds8u(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
MOE_DEV float2 lds_f2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
MOE_DEV float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
MOE_DEV uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// ------------------------------------------------------------ copies
MOE_DEV void dec_tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
MOE_DEV void dec_tma_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
MOE_DEV void dec_bulk(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
MOE_DEV void dec_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
MOE_DEV void dec_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
MOE_DEV void dec_bar_init(uint32_t bar, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}
MOE_DEV bool dec_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
MOE_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

MOE_DEV int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

constexpr long long kDecWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz

// Spin (bounded by `limit` cycles) until *p >= target; false on timeout or abort.
MOE_DEV bool dec_wait_count(const int* p, int target, const volatile int* abort_flag,
                            long long limit = kDecWaitCycles) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire(p) < target) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) return false;
    __nanosleep(64);
  }
  return true;
}

// try_wait that may suspend the thread until the phase completes (for warps
// with nothing else to do: a spinning warp takes issue slots from the math)
MOE_DEV bool dec_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000)
      : "memory");
  return ok != 0;
}

// Mbarrier phase wait (bounded); false on timeout or abort.  A waiting warp
// backs off with nanosleep between polls (a spinning warp takes issue slots
// from the warps still computing) and checks the abort flag and the clock
// every 8 polls.
MOE_DEV bool dec_wait_bar(uint32_t bar, uint32_t parity, const volatile int* abort_flag, bool sleep = false) {
  if (dec_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (sleep ? dec_try_wait_sleep(bar, parity) : dec_try_wait(bar, parity)) return true;
    __nanosleep(32);
    if ((it & 7) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kDecWaitCycles) return false;
    }
  }
}

// ------------------------------------------------------------ fixed point
// Step of a block whose largest magnitude has fp32 exponent field emax:
// values map to |xq| <= 2^14.  Returns (scale_up, step); zero for tiny blocks.
MOE_DEV float2 fix_scales(uint32_t emax) {
  if (emax >= 14 && emax < 255)
    return make_float2(__uint_as_float((267u - emax) << 23), __uint_as_float((emax - 13u) << 23));
  return make_float2(0.f, 0.f);
}

}  // namespace moe
