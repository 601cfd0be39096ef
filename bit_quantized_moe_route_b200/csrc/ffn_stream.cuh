// Step 3 for small token counts, streaming version: the grouped SwiGLU expert
// FFN as a weight-streaming GEMV whose packed rows flow HBM -> shared memory
// through a ring of bulk asynchronous copies (cp.async.bulk + mbarrier
// transaction counts), fed by one producer warp, while eight consumer warps
// dequantise in registers and reduce.
//
//   stage 1:  h[p] = silu(W1[e] . x[t]) * (W3[e] . x[t])
//   stage 2:  y[p] = W2[e] . h[p]
//
// [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": w1/w2/w3 are the switch MLP's
// gate/down/up; model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit":
// affine packs w = scale*q + bias, mxfp4 = e2m1 codes with e8m0 group scales.]
//
// Arithmetic.  A thread owns one 32-input chunk of every row it touches.  Per
// chunk and token the activations are held as a 16-bit fixed-point vector
// xq = rint(x * 2^(141-Emax)) (Emax: largest fp32 exponent field in the
// chunk; |xq| < 2^15), split into a signed high byte and an unsigned low byte
// so that sum(q_i * xq_i) = 256*dp4a(q, hi) + dp4a(q, lo) is an exact int32.
// A bf16 x within 2^6 of the chunk's largest magnitude converts exactly; the
// error of smaller ones is below 2^-16 of the chunk maximum.  Per chunk:
//   affine: s * 2^(Emax-141) * sum(q*xq) + b * 2^(Emax-141) * sum(xq)
//   mxfp4 : 2^(e-128) * 2^(Emax-141) * sum(2*e2m1(c) * xq)
// accumulated in fp32.  3-bit codes (which do not split into bytes cheaply)
// keep fp32 activations and exact float codes instead.
#pragma once

#include "common.cuh"
#include "ffn_gemv.cuh"

namespace moe {

// ------------------------------------------------------------ async proxy
MOE_DEV uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

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
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

MOE_DEV void consumer_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

// ------------------------------------------------------------ formats
// Per format: rows per thread per tile (keeps a tile's packed words at
// <= 32 KiB), tokens per pass, and the order in which a chunk's inputs meet
// the dp4a byte lanes (plane word w, byte lane l -> input index).
template <int FMT, int STAGE, int NTMAX>
struct SF {
  static constexpr int M = STAGE == 1 ? 2 : 1;
  static constexpr int bits = FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
  static constexpr int RPT = (FMT == F_A3 ? 4 : 16 / bits) * (STAGE == 1 ? 1 : 2);
  static constexpr bool kInt = FMT != F_A3;
  static constexpr int NTc = 32 / (RPT * M);
  static constexpr int NTi = NTc > 4 ? 4 : NTc;
  static constexpr int NTf = kInt ? NTi : 2;
  static constexpr int NT = NTf < NTMAX ? NTf : NTMAX;  // tokens per pass
  static constexpr int V = RPT * M * NT;
  // input index fed to plane word w (0..7), byte lane l (0..3)
  static MOE_DEV constexpr int order(int w, int l) {
    if constexpr (FMT == F_A4) return 8 * (w >> 1) + 2 * l + (w & 1);  // even/odd nibbles of each word
    if constexpr (FMT == F_A2) return 16 * (w >> 2) + 4 * l + (w & 3);  // 2-bit fields by shift
    return 4 * w + l;                                                   // bytes in natural order (A8, MX4)
  }
};

constexpr int kStages = 4;
constexpr int kStageQBytes = 32 * 1024;
constexpr int kStageSBBytes = 8 * 1024;
constexpr int kStageBytes = kStageQBytes + kStageSBBytes;
constexpr int kConsumerWarps = 8;
constexpr int kStreamThreads = kConsumerWarps * 32;
constexpr int kRedFloats = 2 * kConsumerWarps * 32;
constexpr size_t kStreamSmem = (size_t)kStages * kStageBytes + kRedFloats * 4 + kStages * 8 + 16;

// register words holding one pass's activations
template <int NTMAX>
struct XWords {
  static constexpr int n = (16 * NTMAX > 32 * (NTMAX < 2 ? NTMAX : 2)) ? 16 * NTMAX : 32 * (NTMAX < 2 ? NTMAX : 2);
};

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
  int r_rows, s_rows;      // rows per tile: routed, shared
  int* err;
};

struct Tile {
  const QMatDev* A;
  const QMatDev* B;
  int e, r0, rows, R, pos0, npos, seg;  // seg: -1 shared, else active index
};

MOE_DEV Tile tile_at(const StreamParams& p, long long g, int n_sh, int tpe) {
  Tile t;
  if (g < n_sh) {
    t.A = &p.sa;
    t.B = &p.sb;
    t.e = 0;
    t.R = p.s_rows;
    t.r0 = (int)g * t.R;
    t.pos0 = p.shared_pos0;
    t.npos = p.T;
    t.seg = -1;
  } else {
    const long long h = g - n_sh;
    const int a = (int)(h / tpe);
    t.A = &p.ra;
    t.B = &p.rb;
    t.e = __ldcg(p.active + 1 + a);
    t.R = p.r_rows;
    t.r0 = (int)(h - (long long)a * tpe) * t.R;
    t.pos0 = __ldcg(p.offsets + t.e);
    t.npos = __ldcg(p.offsets + t.e + 1) - t.pos0;
    t.seg = a;
  }
  t.rows = min(t.R, t.A->n_out - t.r0);
  return t;
}

// Byte offsets of a tile's regions inside a stage buffer.
struct StageLayout {
  int q[2], s[2], b[2], total;
};
MOE_DEV StageLayout stage_layout(const QMatDev& A, int R, int M, int rows) {
  StageLayout L;
  const int row_bytes = A.wpr * 4;
  const int ssz = A.fmt == F_MX4 ? 1 : 2;
  const int sb_row = A.gpr * ssz;
  for (int m = 0; m < 2; ++m) {
    L.q[m] = m * R * row_bytes;
    L.s[m] = kStageQBytes + m * R * sb_row * (A.fmt == F_MX4 ? 1 : 2);
    L.b[m] = L.s[m] + R * sb_row;
  }
  L.total = M * rows * (row_bytes + sb_row * (A.fmt == F_MX4 ? 1 : 2));
  return L;
}

// ------------------------------------------------------------ activations
// Per-token chunk state: 8 high-byte and 8 low-byte plane words (integer
// formats) or 32 fp32 values (3-bit), plus the fixed-point scale and sum.
template <int FMT, int STAGE, int NTMAX>
MOE_DEV void load_x(const StreamParams& p, const Tile& t, int tb, int nt, int c, uint32_t (&xw)[XWords<NTMAX>::n],
                    float (&xs)[NTMAX], float (&xsum)[NTMAX]) {
  using F = SF<FMT, STAGE, NTMAX>;
#pragma unroll
  for (int j = 0; j < F::NT; ++j) {
    float v[32];
    if (j < nt) {
      if constexpr (STAGE == 1) {
        const int tok = t.seg < 0 ? (tb + j) : (__ldcg(p.sorted_rows + t.pos0 + tb + j) / p.k);
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
        const float4* src = reinterpret_cast<const float4*>(p.hin + (size_t)(t.pos0 + tb + j) * p.ld_in + c * 32);
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
    if constexpr (F::kInt) {
      uint32_t emax = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) emax = max(emax, (__float_as_uint(v[i]) >> 23) & 0xFFu);
      float scale = 0.f, inv = 0.f;
      if (emax >= 14 && emax < 255) {
        scale = __uint_as_float((268u - emax) << 23);   // 2^(141 - emax)
        inv = __uint_as_float((emax - 14u) << 23);      // 2^(emax - 141)
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
        xw[16 * j + w] = hi;
        xw[16 * j + 8 + w] = lo;
      }
      xs[j] = inv;
      xsum[j] = inv * (float)sum;
    } else {
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        xw[32 * j + i] = __float_as_uint(v[i]);
        sum += v[i];
      }
      xs[j] = 1.f;
      xsum[j] = sum;
    }
  }
}

// ------------------------------------------------------------ chunk dots
// acc[j] += contribution of one chunk (row of a matrix) for tokens j < nt.
template <int FMT, int STAGE, int NTMAX>
MOE_DEV void chunk_dot_s(const uint8_t* qs, float sc, float bi, const uint32_t (&xw)[XWords<NTMAX>::n],
                         const float (&xs)[NTMAX], const float (&xsum)[NTMAX], int nt, float* acc) {
  using F = SF<FMT, STAGE, NTMAX>;
  if constexpr (FMT == F_A4) {
    const uint4 w4 = *reinterpret_cast<const uint4*>(qs);
    const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
    uint32_t b8[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      b8[2 * k] = wd[k] & 0x0F0F0F0Fu;
      b8[2 * k + 1] = (wd[k] >> 4) & 0x0F0F0F0Fu;
    }
#pragma unroll
    for (int j = 0; j < F::NT; ++j) {
      if (j < nt) {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_us(b8[w], xw[16 * j + w], ph);
          pl = dp4a_uu(b8[w], xw[16 * j + 8 + w], pl);
        }
        const float P = (float)(ph * 256 + pl);
        acc[j] = fmaf(sc, P * xs[j], fmaf(bi, xsum[j], acc[j]));
      }
    }
  } else if constexpr (FMT == F_A8) {
    const uint4 a4 = *reinterpret_cast<const uint4*>(qs);
    const uint4 c4 = *reinterpret_cast<const uint4*>(qs + 16);
    const uint32_t b8[8] = {a4.x, a4.y, a4.z, a4.w, c4.x, c4.y, c4.z, c4.w};
#pragma unroll
    for (int j = 0; j < F::NT; ++j) {
      if (j < nt) {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_us(b8[w], xw[16 * j + w], ph);
          pl = dp4a_uu(b8[w], xw[16 * j + 8 + w], pl);
        }
        const float P = (float)(ph * 256 + pl);
        acc[j] = fmaf(sc, P * xs[j], fmaf(bi, xsum[j], acc[j]));
      }
    }
  } else if constexpr (FMT == F_A2) {
    const uint2 w2 = *reinterpret_cast<const uint2*>(qs);
    const uint32_t wd[2] = {w2.x, w2.y};
    uint32_t b8[8];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int s = 0; s < 4; ++s) b8[4 * k + s] = (wd[k] >> (2 * s)) & 0x03030303u;
#pragma unroll
    for (int j = 0; j < F::NT; ++j) {
      if (j < nt) {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_us(b8[w], xw[16 * j + w], ph);
          pl = dp4a_uu(b8[w], xw[16 * j + 8 + w], pl);
        }
        const float P = (float)(ph * 256 + pl);
        acc[j] = fmaf(sc, P * xs[j], fmaf(bi, xsum[j], acc[j]));
      }
    }
  } else if constexpr (FMT == F_MX4) {
    // codes -> signed bytes 2*e2m1(c) via byte-permute lookups:
    // magnitudes {0,1,2,3,4,6,8,12}, negatives as two's complement
    const uint4 w4 = *reinterpret_cast<const uint4*>(qs);
    const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
    uint32_t b8[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t mag = wd[k] & 0x77777777u;
      const uint32_t sgn = (wd[k] >> 1) & 0x44444444u;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? (mag >> 16) : mag;
        const uint32_t ssel = h ? (sgn >> 16) : sgn;
        const uint32_t pos = __byte_perm(0x03020100u, 0x0C080604u, sel);
        const uint32_t neg = __byte_perm(0xFDFEFF00u, 0xF4F8FAFCu, sel);
        const uint32_t msk = __byte_perm(0x00000000u, 0xFFFFFFFFu, ssel);
        b8[2 * k + h] = (pos & ~msk) | (neg & msk);
      }
    }
#pragma unroll
    for (int j = 0; j < F::NT; ++j) {
      if (j < nt) {
        int ph = 0, pl = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ph = dp4a_ss(b8[w], xw[16 * j + w], ph);
          pl = dp4a_su(b8[w], xw[16 * j + 8 + w], pl);
        }
        const float P = (float)(ph * 256 + pl);
        acc[j] = fmaf(sc, P * xs[j], acc[j]);
      }
    }
  } else {  // F_A3: exact float codes, fp32 activations
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(qs);
    const uint32_t wd[3] = {wp[0], wp[1], wp[2]};
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int pos = 3 * i, wi = pos >> 5, sh = pos & 31;
      uint32_t c = wd[wi] >> sh;
      if (sh > 29) c |= wd[wi + 1] << (32 - sh);
      v[i] = magic_u2f(c & 7u);
    }
#pragma unroll
    for (int j = 0; j < F::NT; ++j) {
      if (j < nt) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) s = fmaf(v[i], __uint_as_float(xw[32 * j + i]), s);
        acc[j] = fmaf(sc, s, fmaf(bi, xsum[j], acc[j]));
      }
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

template <int V>
struct Log2 {
  static constexpr int value = V <= 1 ? 0 : 1 + Log2<V / 2>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

struct Ring {
  uint8_t* base;
  uint64_t* full;
  volatile int* abort_flag;
};

// Issue the bulk copies of tile g into stage s (one thread).
template <int STAGE>
MOE_DEV void issue_tile(const StreamParams& p, const Ring& ring, long long g, int s, int n_sh, int tpe) {
  const Tile t = tile_at(p, g, n_sh, tpe);
  constexpr int M = STAGE == 1 ? 2 : 1;
  const StageLayout Lay = stage_layout(*t.A, t.R, M, t.rows);
  uint8_t* sb = ring.base + (size_t)s * kStageBytes;
  mbar_expect_tx(&ring.full[s], (uint32_t)Lay.total);
  const QMatDev* mats[2] = {t.A, t.B};
  const size_t row0 = (size_t)t.e * t.A->n_out + t.r0;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const QMatDev& Q = *mats[m];
    const uint32_t rb = Q.wpr * 4;
    bulk_g2s(sb + Lay.q[m], reinterpret_cast<const uint8_t*>(Q.q) + row0 * rb, t.rows * rb, &ring.full[s]);
    const uint32_t sr = Q.gpr * (Q.fmt == F_MX4 ? 1 : 2);
    bulk_g2s(sb + Lay.s[m], reinterpret_cast<const uint8_t*>(Q.scales) + row0 * sr, t.rows * sr, &ring.full[s]);
    if (Q.fmt != F_MX4)
      bulk_g2s(sb + Lay.b[m], reinterpret_cast<const uint8_t*>(Q.biases) + row0 * sr, t.rows * sr, &ring.full[s]);
  }
}

// Process one tile of format FMT held in stage `s`; after the last pass's
// barrier (every warp is done reading the stage) thread 0 refills the stage
// with tile `g_next` when there is one.
template <int FMT, int STAGE, int NTMAX>
MOE_DEV void consume_tile(const StreamParams& p, const Tile& t, const Ring& ring, int s, long long g_next,
                          long long g1, int n_sh, int tpe, float* red, int& buf,
                          uint32_t (&xw)[XWords<NTMAX>::n], float (&xs)[NTMAX], float (&xsum)[NTMAX],
                          int& cached_seg, int& cached_tb) {
  using F = SF<FMT, STAGE, NTMAX>;
  constexpr int M = F::M, RPT = F::RPT, NT = F::NT, V = F::V;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const QMatDev& A = *t.A;
  const int C = A.n_in >> 5;
  const int rows_par = kFfnThreads / C;
  const int c = tid % C, slot = tid / C;
  const int wps = C >> 5;  // warps per slot
  const StageLayout Lay = stage_layout(A, t.R, M, t.rows);
  const uint8_t* sb = ring.base + (size_t)s * kStageBytes;
  const int row_bytes = A.wpr * 4;
  const int ssz = FMT == F_MX4 ? 1 : 2;
  const int sb_row = A.gpr * ssz;
  const int gidx = (c * 32) / A.group;
  constexpr int kChunkBytes = F::bits * 4;

  const int ntb = (t.npos + NT - 1) / NT;
  for (int b = 0; b < ntb; ++b) {
    const int tb = b * NT;
    const int nt = min(NT, t.npos - tb);
    if (cached_seg != t.seg || cached_tb != tb) {
      load_x<FMT, STAGE, NTMAX>(p, t, tb, nt, c, xw, xs, xsum);
      cached_seg = t.seg;
      cached_tb = tb;
    }
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const int rl = slot + i * rows_par;
      if (rl < t.rows) {
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const uint8_t* qp = sb + Lay.q[m] + rl * row_bytes + c * kChunkBytes;
          float sc, bi = 0.f;
          if constexpr (FMT == F_MX4) {
            const uint32_t e8 = sb[Lay.s[m] + rl * sb_row + gidx];
            sc = __uint_as_float(e8 > 1 ? ((e8 - 1) << 23) : (e8 ? 0x00400000u : 0x00200000u));  // 2^(e-128)
          } else {
            sc = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(sb + Lay.s[m] + rl * sb_row + gidx * 2));
            bi = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(sb + Lay.b[m] + rl * sb_row + gidx * 2));
          }
          chunk_dot_s<FMT, STAGE, NTMAX>(qp, sc, bi, xw, xs, xsum, nt, &acc[(i * M + m) * NT]);
        }
      }
    }
    const float r = warp_transpose_reduce<V>(acc);
    constexpr int rep = 32 / V;
    if ((lane & (rep - 1)) == 0) red[(buf * kConsumerWarps + warp) * 32 + (lane / rep)] = r;
    consumer_bar();
    if (b == ntb - 1 && tid == 0 && g_next < g1) issue_tile<STAGE>(p, ring, g_next, s, n_sh, tpe);
    // finalise: one thread per (slot, row i, token j)
    const int nfin = rows_par * RPT * NT;
    if (tid < nfin) {
      const int fs = tid / (RPT * NT), rem = tid % (RPT * NT);
      const int i = rem / NT, j = rem % NT;
      const int rl = fs + i * rows_par;
      if (j < nt && rl < t.rows) {
        float g = 0.f, u = 0.f;
        for (int w = 0; w < wps; ++w) {
          const float* src = red + (buf * kConsumerWarps + fs * wps + w) * 32;
          g += src[(i * M + 0) * NT + j];
          if constexpr (M == 2) u += src[(i * M + 1) * NT + j];
        }
        const int prow = t.pos0 + tb + j;
        const int r = t.r0 + rl;
        if constexpr (STAGE == 1)
          p.out[(size_t)prow * p.ld_out + r] = silu(g) * u;
        else
          p.out[(size_t)prow * p.ld_out + r] = g;
      }
    }
    buf ^= 1;
  }
}

template <int STAGE, int NTMAX>
__global__ void __launch_bounds__(kStreamThreads, 1) ffn_stream_kernel(const __grid_constant__ StreamParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem + (size_t)kStages * kStageBytes);
  Ring ring;
  ring.base = smem;
  ring.full = reinterpret_cast<uint64_t*>(red + kRedFloats);
  ring.abort_flag = reinterpret_cast<volatile int*>(ring.full + kStages);
  const int tid = threadIdx.x;

  const int n_active = __ldcg(p.active);
  const int n_sh = p.has_shared ? (p.sa.n_out + p.s_rows - 1) / p.s_rows : 0;
  const int tpe = (p.ra.n_out + p.r_rows - 1) / p.r_rows;
  const long long total = (long long)n_sh + (long long)n_active * tpe;
  const long long g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  if (g0 >= g1) return;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&ring.full[s], 1);
    *ring.abort_flag = 0;
    fence_mbar_init();
    for (int s = 0; s < kStages && g0 + s < g1; ++s) issue_tile<STAGE>(p, ring, g0 + s, s, n_sh, tpe);
  }
  __syncthreads();

  uint32_t xw[XWords<NTMAX>::n];
  float xs[NTMAX], xsum[NTMAX];
  int cached_seg = -2, cached_tb = -1;
  int buf = 0;
  int i = 0;
  long long g = g0;
  for (; g < g1; ++g, ++i) {
    const int s = i % kStages;
    const uint32_t round = (uint32_t)(i / kStages);
    if (!mbar_wait(&ring.full[s], round & 1u, ring.abort_flag)) {
      set_error(p.err, kErrTimeout);
      *ring.abort_flag = 1;
      break;
    }
    const Tile t = tile_at(p, g, n_sh, tpe);
    const long long gn = g + kStages;
    switch (t.A->fmt) {
      case F_A2: consume_tile<F_A2, STAGE, NTMAX>(p, t, ring, s, gn, g1, n_sh, tpe, red, buf, xw, xs, xsum, cached_seg, cached_tb); break;
      case F_A3: consume_tile<F_A3, STAGE, NTMAX>(p, t, ring, s, gn, g1, n_sh, tpe, red, buf, xw, xs, xsum, cached_seg, cached_tb); break;
      case F_A4: consume_tile<F_A4, STAGE, NTMAX>(p, t, ring, s, gn, g1, n_sh, tpe, red, buf, xw, xs, xsum, cached_seg, cached_tb); break;
      case F_A8: consume_tile<F_A8, STAGE, NTMAX>(p, t, ring, s, gn, g1, n_sh, tpe, red, buf, xw, xs, xsum, cached_seg, cached_tb); break;
      default:   consume_tile<F_MX4, STAGE, NTMAX>(p, t, ring, s, gn, g1, n_sh, tpe, red, buf, xw, xs, xsum, cached_seg, cached_tb); break;
    }
  }
  // After an abort, wait (bounded) for copies still in flight before the
  // block's shared memory goes away.
  if (g < g1 && tid == 0) {
    const long long issued = min(g1, g0 + (long long)i + kStages);
    for (long long q = g0 + i; q < issued; ++q) {
      const int s = (int)((q - g0) % kStages);
      const long long t0 = clock64();
      while (!mbar_try_wait(&ring.full[s], (uint32_t)((q - g0) / kStages) & 1u) && clock64() - t0 < kWaitCycles) {
      }
    }
  }
}

}  // namespace moe
