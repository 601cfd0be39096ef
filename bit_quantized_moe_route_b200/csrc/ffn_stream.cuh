// Step 3 for small token counts, streaming version: the grouped SwiGLU expert
// FFN as a weight-streaming GEMV whose packed rows flow HBM -> shared memory
// through a ring of bulk asynchronous copies (cp.async.bulk + mbarrier
// transaction counts) issued by one producer warp, while eight consumer warps
// dequantise in registers.
//
//   stage 1:  h[p] = silu(W1[e] . x[t]) * (W3[e] . x[t])
//   stage 2:  y[p] = W2[e] . h[p]
//
// [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": w1/w2/w3 are the switch MLP's
// gate/down/up; model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit":
// affine packs w = scale*q + bias, mxfp4 = e2m1 codes with e8m0 group scales.]
//
// Work split.  A persistent block per SM walks a contiguous range of tiles
// (expert, block of R rows).  The eight consumer warps form groups of WPR
// warps; a group owns R/G whole rows of each tile (G = 8/WPR groups) and
// each of its lanes owns CPL 32-input chunks of every such row, so a row's
// dot product is finished by one warp reduction (plus a small shared-memory
// sum when WPR > 1) -- no block-wide barrier per tile.
//
// Arithmetic.  Per chunk and token the activations are held as a 16-bit
// fixed-point vector xq = rint(x * 2^(141-Emax)) (Emax: largest fp32 exponent
// field in the chunk; |xq| < 2^15), split into a signed high byte and an
// unsigned low byte so that sum(q_i * xq_i) = 256*dp4a(q, hi) + dp4a(q, lo)
// is an exact int32.  A bf16 x within 2^6 of the chunk's largest magnitude
// converts exactly; the error of smaller ones is below 2^-16 of the chunk
// maximum.  Per chunk:
//   affine: s * 2^(Emax-141) * sum(q*xq) + b * 2^(Emax-141) * sum(xq)
//   mxfp4 : 2^(e-128) * 2^(Emax-141) * sum(2*e2m1(c) * xq)
// accumulated in fp32.  3-bit codes reach byte lanes through two
// multiply-and-mask spreads per four codes.
#pragma once

#include "stream_types.cuh"

namespace moe {

// ------------------------------------------------------------ async proxy
MOE_DEV uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MOE_DEV uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
MOE_DEV uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds16(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
MOE_DEV uint32_t lds8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
MOE_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
MOE_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
MOE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
MOE_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// As above, but the thread may sleep up to ~0.1 ms inside the instruction
// until the phase completes (fewer polling iterations while waiting).
MOE_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(100000)
      : "memory");
  return ok != 0;
}
// Bulk copy global -> shared; completion is counted on `bar` in bytes.
// Both addresses 16-byte aligned, size a multiple of 16.
MOE_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz: every wait gives up after this

// Wait for the phase of parity `parity` of `bar`; false on timeout/abort.
MOE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

MOE_DEV void group_bar(int id, int nthreads) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory"); }

// ------------------------------------------------------------ integer dot
MOE_DEV int dp4a_us(uint32_t a_u8, uint32_t b_s8, int c) {  // unsigned a bytes x signed b bytes
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8), "r"(b_s8), "r"(c));
  return d;
}
MOE_DEV int dp4a_uu(uint32_t a_u8, uint32_t b_u8, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8), "r"(b_u8), "r"(c));
  return d;
}
MOE_DEV int dp4a_ss(uint32_t a_s8, uint32_t b_s8, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_s8), "r"(b_s8), "r"(c));
  return d;
}
MOE_DEV int dp4a_su(uint32_t a_s8, uint32_t b_u8, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_s8), "r"(b_u8), "r"(c));
  return d;
}

// Per format: how a chunk's 32 inputs meet the dp4a byte lanes (plane word
// w, byte lane l -> input index), and how many tokens one pass carries.
template <int FMT, int NTMAX>
struct SF {
  static constexpr int bits = FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
  static constexpr int NT = NTMAX;
  static constexpr int kChunkBytes = bits * 4;
  static MOE_DEV constexpr int order(int w, int l) {
    if constexpr (FMT == F_A4) return 8 * (w >> 1) + 2 * l + (w & 1);  // even/odd nibbles of each word
    if constexpr (FMT == F_A2) return 16 * (w >> 2) + 4 * l + (w & 3);  // 2-bit fields by shift
    return 4 * w + l;                                                   // natural order (A8, A3, MX4)
  }
};



// Incremental walk over the block's tile range: shared-expert tiles first,
// then the tiles of each active routed expert.  The routed expert's id and
// position range are read from global memory once per expert, not per tile.
struct Walker {
  long long g, g1;
  int n_sh, tpe, a, rb;
  int e, pos0, npos;
  MOE_DEV void load_seg(const StreamParams& p) {
    if (a >= 0) {
      e = __ldcg(p.active + 1 + a);
      pos0 = __ldcg(p.offsets + e);
      npos = __ldcg(p.offsets + e + 1) - pos0;
    } else {
      e = 0;
      pos0 = p.shared_pos0;
      npos = p.T;
    }
  }
  MOE_DEV void start(const StreamParams& p, long long g0, long long g_end, int n_sh_, int tpe_) {
    g = g0;
    g1 = g_end;
    n_sh = n_sh_;
    tpe = tpe_;
    if (g0 < n_sh) {
      a = -1;
      rb = (int)g0;
    } else {
      const long long h = g0 - n_sh;
      a = (int)(h / tpe);
      rb = (int)(h - (long long)a * tpe);
    }
    load_seg(p);
  }
  MOE_DEV void next(const StreamParams& p) {
    ++g;
    ++rb;
    if (a < 0) {
      if (rb >= n_sh) {
        a = 0;
        rb = 0;
        if (g < g1) load_seg(p);
      }
    } else if (rb >= tpe) {
      ++a;
      rb = 0;
      if (g < g1) load_seg(p);
    }
  }
};

struct Tile {
  const QMatDev* A;
  const QMatDev* B;
  int e, r0, rows, R, wpr, pos0, npos, seg;  // seg: -1 shared, else active index
};

MOE_DEV Tile tile_of(const StreamParams& p, const Walker& w) {
  Tile t;
  const bool sh = w.a < 0;
  t.A = sh ? &p.sa : &p.ra;
  t.B = sh ? &p.sb : &p.rb;
  t.R = sh ? p.s_rows : p.r_rows;
  t.wpr = sh ? p.s_wpr : p.r_wpr;
  t.e = w.e;
  t.pos0 = w.pos0;
  t.npos = w.npos;
  t.seg = w.a;
  t.r0 = w.rb * t.R;
  t.rows = min(t.R, t.A->n_out - t.r0);
  return t;
}

// Byte offsets of a tile's regions inside a stage buffer: packed rows of
// each matrix, then scales (and biases) of each matrix.
struct StageLayout {
  int q[2], s[2], b[2], total;
};
MOE_DEV StageLayout stage_layout(const QMatDev& A, int R, int M, int rows) {
  StageLayout L;
  const int row_bytes = A.wpr * 4;
  const bool mx = A.fmt == F_MX4;
  const int sb_row = A.gpr * (mx ? 1 : 2);
  const int per_m = R * sb_row * (mx ? 1 : 2);
  for (int m = 0; m < 2; ++m) {
    L.q[m] = m * R * row_bytes;
    L.s[m] = M * R * row_bytes + m * per_m;
    L.b[m] = L.s[m] + R * sb_row;
  }
  L.total = M * rows * (row_bytes + sb_row * (mx ? 1 : 2));
  return L;
}

// ------------------------------------------------------------ activations
// Activations of one pass for this lane's CPL chunks: 8 high-byte and 8
// low-byte plane words per (chunk, token), plus the fixed-point scale and
// the scaled chunk sum.
template <int NTMAX, int CPL>
struct XRegs {
  static constexpr int kWords = 16 * NTMAX * CPL;
  uint32_t w[kWords];
  float xs[CPL][NTMAX];
  float xsum[CPL][NTMAX];
};

template <int FMT, int STAGE, int NTMAX, int CPL>
MOE_DEV void load_x(const StreamParams& p, const Tile& t, int tb, int nt, int cbase, XRegs<NTMAX, CPL>& X) {
  using F = SF<FMT, NTMAX>;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < F::NT; ++j) {
    int tok = 0;
    if (STAGE == 1 && j < nt) tok = t.seg < 0 ? (tb + j) : (__ldcg(p.sorted_rows + t.pos0 + tb + j) / p.k);
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) {
      const int c = cbase + 32 * cc + lane;
      float v[32];
      if (j < nt) {
        if constexpr (STAGE == 1) {
          const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)tok * t.A->n_in + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u = __ldcg(src + q);
            v[8 * q + 0] = bf16lo(u.x); v[8 * q + 1] = bf16hi(u.x);
            v[8 * q + 2] = bf16lo(u.y); v[8 * q + 3] = bf16hi(u.y);
            v[8 * q + 4] = bf16lo(u.z); v[8 * q + 5] = bf16hi(u.z);
            v[8 * q + 6] = bf16lo(u.w); v[8 * q + 7] = bf16hi(u.w);
          }
        } else {
          const float4* src =
              reinterpret_cast<const float4*>(p.hin + (size_t)(t.pos0 + tb + j) * p.ld_in + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 u = __ldcg(src + q);
            v[4 * q + 0] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      uint32_t emax = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) emax = max(emax, (__float_as_uint(v[i]) >> 23) & 0xFFu);
      float scale = 0.f, inv = 0.f;
      if (emax >= 14 && emax < 255) {
        scale = __uint_as_float((268u - emax) << 23);  // 2^(141 - emax)
        inv = __uint_as_float((emax - 14u) << 23);     // 2^(emax - 141)
      }
      int q[32];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        q[i] = __float2int_rn(v[i] * scale);
        sum += q[i];
      }
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t hi = 0, lo = 0;
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int qi = q[F::order(w, l)];
          hi |= (uint32_t)((qi >> 8) & 0xFF) << (8 * l);
          lo |= (uint32_t)(qi & 0xFF) << (8 * l);
        }
        X.w[(j * CPL + cc) * 16 + w] = hi;
        X.w[(j * CPL + cc) * 16 + 8 + w] = lo;
      }
      X.xs[cc][j] = inv;
      X.xsum[cc][j] = inv * (float)sum;
      // keep one chunk's raw activations live at a time (register pressure)
      asm volatile("" ::: "memory");
    }
  }
}

// ------------------------------------------------------------ chunk dots
// Packed words of one 32-input chunk (as many as the format needs).
struct ChunkWords {
  uint32_t w[8];
};

template <int FMT>
MOE_DEV ChunkWords load_chunk(uint32_t a) {
  ChunkWords c;
  if constexpr (FMT == F_A8) {
    const uint4 x = lds128(a), y = lds128(a + 16);
    c.w[0] = x.x; c.w[1] = x.y; c.w[2] = x.z; c.w[3] = x.w;
    c.w[4] = y.x; c.w[5] = y.y; c.w[6] = y.z; c.w[7] = y.w;
  } else if constexpr (FMT == F_A2) {
    const uint2 x = lds64(a);
    c.w[0] = x.x; c.w[1] = x.y;
  } else if constexpr (FMT == F_A3) {
    c.w[0] = lds32(a); c.w[1] = lds32(a + 4); c.w[2] = lds32(a + 8);
  } else {
    const uint4 x = lds128(a);
    c.w[0] = x.x; c.w[1] = x.y; c.w[2] = x.z; c.w[3] = x.w;
  }
  return c;
}

// acc[j] += one chunk's contribution for tokens j < nt (all NT when FULL);
// chunk slot cc selects this lane's activation words.
template <int FMT, int NTMAX, int CPL, bool FULL>
MOE_DEV void chunk_dot_s(const ChunkWords& cw, float sc, float bi, const XRegs<NTMAX, CPL>& X, int cc, int nt,
                         float (&acc)[NTMAX]) {
  using F = SF<FMT, NTMAX>;
  uint32_t b8[8];
  if constexpr (FMT == F_A4) {
    // even nibbles masked into bytes; odd nibbles masked in place (16 * q)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      b8[2 * k] = cw.w[k] & 0x0F0F0F0Fu;
      b8[2 * k + 1] = cw.w[k] & 0xF0F0F0F0u;
    }
  } else if constexpr (FMT == F_A8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) b8[k] = cw.w[k];
  } else if constexpr (FMT == F_A2) {
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int s = 0; s < 4; ++s) b8[4 * k + s] = (cw.w[k] >> (2 * s)) & 0x03030303u;
  } else if constexpr (FMT == F_A3) {
    // 32 codes in 96 bits; plane word w holds codes 4w..4w+3 = stream bits
    // [12w, 12w+12).  Two multiply-and-mask spreads move the four 3-bit
    // fields to byte lanes (the shifted copies never overlap, so no carries).
    const uint32_t w0 = cw.w[0], w1 = cw.w[1], w2 = cw.w[2];
    const uint32_t tw[8] = {w0, w0 >> 12, __funnelshift_r(w0, w1, 24), w1 >> 4,
                            w1 >> 16, __funnelshift_r(w1, w2, 28), w2 >> 8, w2 >> 20};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const uint32_t t = tw[w];
      const uint32_t ev = ((t & 0x1C7u) * 0x401u) & 0x00070007u;   // codes 0,2 -> bytes 0,2
      const uint32_t od = ((t & 0xE38u) * 0x8020u) & 0x07000700u;  // codes 1,3 -> bytes 1,3
      b8[w] = ev | od;
    }
  } else {  // F_MX4: codes -> signed bytes 2*e2m1(c) by byte-permute lookups
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t mag = cw.w[k] & 0x77777777u;
      const uint32_t sgn = (cw.w[k] >> 1) & 0x44444444u;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? (mag >> 16) : mag;
        const uint32_t ssel = h ? (sgn >> 16) : sgn;
        const uint32_t pos = __byte_perm(0x03020100u, 0x0C080604u, sel);  // 0,1,2,3,4,6,8,12
        const uint32_t neg = __byte_perm(0xFDFEFF00u, 0xF4F8FAFCu, sel);  // their negatives
        const uint32_t msk = __byte_perm(0x00000000u, 0xFFFFFFFFu, ssel);
        b8[2 * k + h] = (pos & ~msk) | (neg & msk);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < F::NT; ++j) {
    if (FULL || j < nt) {
      const uint32_t* xw = &X.w[(j * CPL + cc) * 16];
      int P;
      if constexpr (FMT == F_MX4) {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_ss(b8[w], xw[w], ph);
          pl = dp4a_su(b8[w], xw[8 + w], pl);
        }
        P = ph * 256 + pl;
      } else if constexpr (FMT == F_A4) {
        int phe = 0, ple = 0, pho = 0, plo = 0;
#pragma unroll
        for (int w = 0; w < 8; w += 2) {
          phe = dp4a_us(b8[w], xw[w], phe);
          ple = dp4a_uu(b8[w], xw[8 + w], ple);
          pho = dp4a_us(b8[w + 1], xw[w + 1], pho);
          plo = dp4a_uu(b8[w + 1], xw[9 + w], plo);
        }
        P = (phe * 256 + ple) + ((pho * 256 + plo) >> 4);  // exact: the odd sum is a multiple of 16
      } else {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_us(b8[w], xw[w], ph);
          pl = dp4a_uu(b8[w], xw[8 + w], pl);
        }
        P = ph * 256 + pl;
      }
      acc[j] = fmaf(sc, (float)P * X.xs[cc][j], fmaf(bi, X.xsum[cc][j], acc[j]));
    }
  }
}

// Transposed warp reduction: V values per lane -> lane l ends up holding the
// warp-wide sum of value index (l >> (5 - log2 V)).
template <int V>
MOE_DEV float warp_transpose_reduce(float (&v)[V]) {
  const int lane = threadIdx.x & 31;
  int n = V;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool up = (lane & o) != 0;
      const int h = n >> 1;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < h) {
          const float send = up ? v[i] : v[i + h];
          const float keep = up ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

// Write one finished (row, token) result.
template <int STAGE>
MOE_DEV void emit(const StreamParams& p, const Tile& t, int rl, int tok_slot, float g, float u) {
  const int prow = t.pos0 + tok_slot;
  const int r = t.r0 + rl;
  if constexpr (STAGE == 1)
    p.out[(size_t)prow * p.ld_out + r] = __fdividef(g * u, 1.f + __expf(-g));  // silu(g) * u
  else
    p.out[(size_t)prow * p.ld_out + r] = g;
}

// Rows reduced together: one transposed warp reduction per block of RB rows.
template <int STAGE, int NT>
struct RowBlock {
  static constexpr int M = STAGE == 1 ? 2 : 1;
  static constexpr int RB = (STAGE == 1 ? 2 : 8) / NT > 0 ? (STAGE == 1 ? 2 : 8) / NT : 1;
  static constexpr int V = RB * M * NT;  // <= 8 values per lane
};

// The rows of one pass: a warp computes its lanes' partial sums for a block
// of RB rows, reduces them in one transposed warp reduction, and either
// writes the results (one warp per row) or parks them for the group's first
// warp.
template <int FMT, int STAGE, int NTMAX, int CPL, bool FULL>
MOE_DEV void tile_rows(const StreamParams& p, const Tile& t, const uint32_t (&qa)[2][CPL],
                       const uint32_t (&sa)[2][CPL], uint32_t boff, int row_bytes, int sb_row, int rpg, int grp,
                       int wig, int tb, int nt, float* red, int buf, const XRegs<NTMAX, CPL>& X) {
  using F = SF<FMT, NTMAX>;
  using RBk = RowBlock<STAGE, F::NT>;
  constexpr int M = RBk::M, NT = F::NT, RB = RBk::RB, V = RBk::V;
  const int lane = threadIdx.x & 31;
  const int rows_here = min(rpg, t.rows - grp * rpg);  // group-uniform
  for (int r0 = 0; r0 < rows_here; r0 += RB) {
    // values ordered (row b, token j, matrix m): g and u of a (row, token) sit side by side
    float vals[V];
#pragma unroll
    for (int v = 0; v < V; ++v) vals[v] = 0.f;
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      if (r0 + b < rows_here) {
        const int rl = grp * rpg + r0 + b;
        const uint32_t dq = (uint32_t)(rl * row_bytes), ds = (uint32_t)(rl * sb_row);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          float acc[NTMAX];
#pragma unroll
          for (int j = 0; j < NTMAX; ++j) acc[j] = 0.f;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) {
            const ChunkWords cw = load_chunk<FMT>(qa[m][cc] + dq);
            float sc, bi = 0.f;
            if constexpr (FMT == F_MX4) {
              const uint32_t e8 = lds8(sa[m][cc] + ds);
              sc = __uint_as_float(e8 > 1 ? ((e8 - 1) << 23) : (e8 ? 0x00400000u : 0x00200000u));  // 2^(e-128)
            } else {
              sc = bf16_bits_to_float(lds16(sa[m][cc] + ds));
              bi = bf16_bits_to_float(lds16(sa[m][cc] + ds + boff));
            }
            chunk_dot_s<FMT, NTMAX, CPL, FULL>(cw, sc, bi, X, cc, nt, acc);
          }
#pragma unroll
          for (int j = 0; j < NT; ++j) vals[(b * NT + j) * M + m] = acc[j];
        }
      }
    }
    const float red_v = warp_transpose_reduce<V>(vals);
    constexpr int rep = 32 / V;
    const float other = (M == 2) ? __shfl_down_sync(0xffffffffu, red_v, rep) : 0.f;
    const int vi = lane / rep;
    if ((lane & (rep - 1)) == 0 && (vi % M) == 0) {
      const int bj = vi / M;
      const int b = bj / NT, j = bj % NT;
      const int r = r0 + b;
      if (r < rows_here && (FULL || j < nt)) {
        if (t.wpr == 1) {
          emit<STAGE>(p, t, grp * rpg + r, tb + j, red_v, other);
        } else {
          float* dst = red + (size_t)buf * kRedHalf + ((grp * t.wpr + wig) * 16 + r) * 2 * NTMAX;
          dst[2 * j] = red_v;
          dst[2 * j + 1] = other;
        }
      }
    }
  }
}

// Issue the bulk copies of the tile at walker position w into stage s.
template <int STAGE>
MOE_DEV void issue_tile(const StreamParams& p, const Walker& w, uint8_t* smem, uint64_t* full, int s) {
  constexpr int M = STAGE == 1 ? 2 : 1;
  const Tile t = tile_of(p, w);
  const StageLayout Lay = stage_layout(*t.A, t.R, M, t.rows);
  uint8_t* sb = smem + (size_t)s * kStageBytes;
  mbar_expect_tx(&full[s], (uint32_t)Lay.total);
  const QMatDev* mats[2] = {t.A, t.B};
  const size_t row0 = (size_t)t.e * t.A->n_out + t.r0;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const QMatDev& Q = *mats[m];
    const uint32_t rbytes = Q.wpr * 4;
    bulk_g2s(sb + Lay.q[m], reinterpret_cast<const uint8_t*>(Q.q) + row0 * rbytes, t.rows * rbytes, &full[s]);
    const uint32_t sr = Q.gpr * (Q.fmt == F_MX4 ? 1 : 2);
    bulk_g2s(sb + Lay.s[m], reinterpret_cast<const uint8_t*>(Q.scales) + row0 * sr, t.rows * sr, &full[s]);
    if (Q.fmt != F_MX4)
      bulk_g2s(sb + Lay.b[m], reinterpret_cast<const uint8_t*>(Q.biases) + row0 * sr, t.rows * sr, &full[s]);
  }
}

// Consume a run of consecutive tiles of one segment (one expert), starting
// at the block's tile ordinal i0: per-expert addressing is set up once, then
// each tile is waited for, computed and released.
template <int FMT, int STAGE, int NTMAX, int CPL>
MOE_DEV bool consume_run(const StreamParams& p, const Walker& w0, int n_run, int i0, uint8_t* smem, uint64_t* full,
                         uint64_t* empty, volatile int* abort_flag, float* red, int& buf, XRegs<NTMAX, CPL>& X) {
  using F = SF<FMT, NTMAX>;
  constexpr int M = STAGE == 1 ? 2 : 1;
  constexpr int NT = F::NT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Tile t = tile_of(p, w0);
  const QMatDev A = *t.A;  // fields in registers for the whole run
  const int wpr = t.wpr;
  const int G = kConsumerWarps / wpr;
  const int grp = warp / wpr, wig = warp % wpr;
  const int rpg = t.R / G;
  const int cbase = wig * 32 * CPL;
  const StageLayout Lay = stage_layout(A, t.R, M, t.R);
  const int row_bytes = A.wpr * 4;
  constexpr bool mx = FMT == F_MX4;
  const int sb_row = A.gpr * (mx ? 1 : 2);
  const int gshift = A.group == 32 ? 0 : (A.group == 64 ? 1 : 2);  // chunk -> scale group
  uint32_t qrel[2][CPL], srel[2][CPL];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) {
      const int c = cbase + 32 * cc + lane;
      qrel[m][cc] = Lay.q[m] + c * F::kChunkBytes;
      srel[m][cc] = Lay.s[m] + (c >> gshift) * (mx ? 1 : 2);
    }
  const uint32_t boff = (uint32_t)(t.R * sb_row);  // biases follow the scales of each matrix
  const int ntb = (t.npos + NT - 1) / NT;
  const uint32_t smem32 = smem_u32(smem);

  for (int k = 0; k < n_run; ++k) {
    const int i = i0 + k;
    const int s = i % kStages;
    if (!mbar_wait(&full[s], (uint32_t)(i / kStages) & 1u, abort_flag)) {
      set_error(p.err, kErrTimeout);
      *abort_flag = 1;
      return false;
    }
    t.r0 = (w0.rb + k) * t.R;
    t.rows = min(t.R, A.n_out - t.r0);
    const uint32_t sb32 = smem32 + (uint32_t)s * kStageBytes;
    uint32_t qa[2][CPL], sa[2][CPL];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) {
        qa[m][cc] = sb32 + qrel[m][cc];
        sa[m][cc] = sb32 + srel[m][cc];
      }
    for (int b = 0; b < ntb; ++b) {
      const int tb = b * NT;
      const int nt = min(NT, t.npos - tb);
      if (k == 0 || ntb > 1) load_x<FMT, STAGE, NTMAX, CPL>(p, t, tb, nt, cbase, X);
      if constexpr (NT == 1) {
        tile_rows<FMT, STAGE, NTMAX, CPL, true>(p, t, qa, sa, boff, row_bytes, sb_row, rpg, grp, wig, tb, nt, red,
                                                buf, X);
      } else {
        if (nt == NT)
          tile_rows<FMT, STAGE, NTMAX, CPL, true>(p, t, qa, sa, boff, row_bytes, sb_row, rpg, grp, wig, tb, nt, red,
                                                  buf, X);
        else
          tile_rows<FMT, STAGE, NTMAX, CPL, false>(p, t, qa, sa, boff, row_bytes, sb_row, rpg, grp, wig, tb, nt,
                                                   red, buf, X);
      }
      if (b == ntb - 1) {  // every read of this stage by this warp is done
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (wpr > 1) {
        group_bar(1 + grp, wpr * 32);
        // lanes of the group's first warp sum the WPR partials of each (row, token)
        if (wig == 0) {
          const int nval = rpg * nt;
          for (int v = lane; v < nval; v += 32) {
            const int r = v / nt, j = v % nt;
            const int rl = grp * rpg + r;
            if (rl < t.rows) {
              float g = 0.f, u = 0.f;
              for (int ww = 0; ww < wpr; ++ww) {
                const float* src = red + (size_t)buf * kRedHalf + ((grp * wpr + ww) * 16 + r) * 2 * NTMAX;
                g += src[2 * j];
                u += src[2 * j + 1];
              }
              emit<STAGE>(p, t, rl, tb + j, g, u);
            }
          }
        }
        buf ^= 1;
      }
    }
  }
  return true;
}

template <int STAGE, int NTMAX, int CPL, int RFMT>
__global__ void __launch_bounds__(kStreamThreads, 1)
ffn_stream_kernel(const __grid_constant__ StreamParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem + (size_t)kStages * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kRedFloats);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Programmatic launch: stage 1 waits for the routing (it reads the active
  // list right away) and then releases stage 2; stage 2 releases the combine
  // at once and its copy warp starts streaming weights before stage 1 has
  // finished -- weights and routing were complete when stage 1 released it
  // -- while its consumers wait for stage 1 before reading h.
  if constexpr (STAGE == 1) pdl_wait();
  pdl_trigger();
  const int n_active = __ldcg(p.active);
  const int n_sh = p.has_shared ? (p.sa.n_out + p.s_rows - 1) / p.s_rows : 0;
  const int tpe = (p.ra.n_out + p.r_rows - 1) / p.r_rows;
  const long long total = (long long)n_sh + (long long)n_active * tpe;
  const long long g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  if (g0 >= g1) return;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one lane issues every copy
    if (lane != 0) return;
    Walker w;
    w.start(p, g0, g1, n_sh, tpe);
    int i = 0;
    for (; w.g < g1; w.next(p), ++i) {
      const int s = i % kStages;
      const uint32_t round = (uint32_t)(i / kStages);
      if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1u, abort_flag)) {
        set_error(p.err, kErrTimeout);
        *abort_flag = 1;
        break;
      }
      issue_tile<STAGE>(p, w, smem, full, s);
    }
    // drain: no copy may still be landing in shared memory when the block exits
    for (int q = max(0, i - kStages); q < i; ++q) {
      const int s = q % kStages;
      const long long t0 = clock64();
      while (!mbar_try_wait(&full[s], (uint32_t)(q / kStages) & 1u) && clock64() - t0 < kWaitCycles) {
      }
    }
    return;
  }

  // ---------------- consumers: runs of tiles of one expert at a time
  if constexpr (STAGE == 2) pdl_wait();  // h is written by stage 1
  XRegs<NTMAX, CPL> X;
  int buf = 0;
  int prev_wpr = 1;
  Walker w;
  w.start(p, g0, g1, n_sh, tpe);
  int i = 0;
  while (w.g < g1) {
    const int seg_tiles = w.a < 0 ? n_sh : tpe;
    const int n_run = (int)min((long long)(seg_tiles - w.rb), g1 - w.g);
    const Tile t = tile_of(p, w);
    // when the row-group shape changes, let every old finaliser finish with
    // the partial sums before another group may overwrite them
    if (t.wpr != prev_wpr && prev_wpr > 1) group_bar(9, kConsumerWarps * 32);
    prev_wpr = t.wpr;
    bool ok;
    // the routed format, or the 8-bit shared expert
    if (RFMT == F_A8 || t.A->fmt == RFMT)
      ok = consume_run<RFMT, STAGE, NTMAX, CPL>(p, w, n_run, i, smem, full, empty, abort_flag, red, buf, X);
    else
      ok = consume_run<F_A8, STAGE, NTMAX, CPL>(p, w, n_run, i, smem, full, empty, abort_flag, red, buf, X);
    if (!ok) break;
    for (int k = 0; k < n_run; ++k) w.next(p);
    i += n_run;
  }
}

}  // namespace moe
