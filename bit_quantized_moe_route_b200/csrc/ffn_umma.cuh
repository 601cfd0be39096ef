// Step 3 for large token counts (prefill), TMA + TMEM variant of the
// tensor-core grouped SwiGLU expert FFN:
//
//   stage 1 (per expert e):  H[p, :] = silu(X[p] . W1[e]^T) * (X[p] . W3[e]^T)
//   stage 2 (per expert e):  Y[p, :] = H[p] . W2[e]^T
//
// [mlx-lm PR "Add DeepSeek-v4 (Flash/Pro)": w1/w2/w3 = gate/down/up of the
// switch MLP; model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit":
// affine w = scale*q + bias; mxfp4 = e2m1 * 2^(e-127)].
//
// Data path of one CTA pair (a cluster of two CTAs on two SMs, persistent):
//   * an item is (token tile, 256 weight rows); each CTA of the pair owns
//     128 of the rows: stage 1 stacks 64 gate rows and the 64 up rows of the
//     same features (CTA r takes features 64r..64r+63 of the item's 128),
//     stage 2 takes output rows 128r..128r+127 of the item's 256;
//   * each CTA's packed codes and group scales/biases arrive by TMA (2D boxes
//     of 128 bytes x rows, 128-byte swizzle; 16-byte scale boxes) into its
//     own 3-slot ring, one slot = one 128-byte box of codes per row (256
//     inputs of 4-bit codes, 128 of 8-bit, 512 of 2-bit);
//   * the token rows (B operand, fp16, gathered into expert order
//     beforehand) arrive by TMA as two 64-input K-major column blocks per
//     128-input stage with the 128-byte swizzle the tensor core reads; the
//     tile's N tokens (rounded up to 32) are split between the two CTAs, N/2
//     rows each, and both CTAs' loads complete on the leader CTA's barrier;
//   * kUmGroups groups of 4 dequant warps per CTA (stage g goes to group
//     g mod kUmGroups) turn each 128-input stage of codes into fp16 weights
//     and write them straight into the CTA's tensor memory (tcgen05.st): the
//     weights are the MMA's A operand in TMEM, in a ring of kUmNA stage slots
//     of 64 columns, so the shared memory only carries the token tiles and
//     the packed codes;
//   * one thread of the leader CTA issues 8 tcgen05.mma.cta_group::2 per
//     stage (M = 256 over the pair: A from both CTAs' TMEM, B from both CTAs'
//     shared memory, fp32 accumulators in each CTA's TMEM: kUmNAcc buffers of
//     192 columns); its commits arrive on the barriers of both CTAs.  One
//     instruction covers both SMs' rows, and each SM reads only its half of
//     the token tile, which halves the MMA issue work and the shared-memory
//     operand traffic per flop against one-SM MMAs;
//   * the peer CTA's dequant and epilogue warps arrive on the leader's
//     barriers through shared::cluster addresses;
//   * 4 epilogue warps per CTA read that CTA's accumulators (tcgen05.ld) and
//     write H (SwiGLU, fp16) or y (fp32).
// In stage 1 every 32-lane TMEM quarter holds 16 W1 rows in lanes 0-15 and
// the W3 rows of the same 16 features in lanes 16-31, so the epilogue pairs
// them with one warp shuffle.
// Operands are fp16 (see ffn_tc.cuh for why); every wait is bounded, and
// both CTAs pass a cluster barrier before either frees its tensor memory.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ffn_tc.cuh"

namespace moe {

constexpr int kUmN = 192;        // tokens per tile (MMA N <= 192, a multiple of 32 for the pair MMA)
constexpr int kUmK = 128;        // inputs per MMA stage (8 MMAs of K = 16)
constexpr int kUmKB = 64;        // inputs per 128-byte swizzle atom of a token row
constexpr int kUmGroups = 2;     // dequant groups of 4 warps
constexpr int kUmNA = 2;         // A stage slots in TMEM
constexpr int kUmNAcc = 2;       // accumulator buffers in TMEM
constexpr int kUmDqWarps = 4 * kUmGroups;
constexpr int kUmMmaWarp = kUmDqWarps;
constexpr int kUmRawWarp = kUmDqWarps + 1;      // TMA issuer of packed codes / scales / biases
constexpr int kUmBWarp = kUmDqWarps + 2;        // TMA issuer of token tiles
constexpr int kUmEpiWarp0 = kUmDqWarps + 4;     // 4 epilogue warps: warp % 4 = TMEM lane quarter
constexpr int kUmThreads = (kUmEpiWarp0 + 4) * 32;
constexpr int kUmBStages = 4;
constexpr int kUmBHalf = kUmN / 2;              // token rows per CTA of the pair
constexpr int kUmBBlock = kUmBHalf * 128;       // one 64-input column block of this CTA's rows
constexpr int kUmBTile = 2 * kUmBBlock;         // 96 rows x 128 inputs fp16 = 24 KB
constexpr uint32_t kUmASlotCols = kUmK / 2;     // 64 TMEM columns per A stage slot
constexpr uint32_t kUmAccCol0 = kUmNA * kUmASlotCols;  // A slots first, then the accumulators
constexpr uint32_t kUmAccCols = kUmN;
constexpr uint32_t kUmTmemCols = 512;
constexpr int kUmRowsS1 = 128;   // stage-1 features per pair item (64 per CTA, W1 and W3 each)
constexpr int kUmRowsS2 = 256;   // stage-2 output rows per pair item (128 per CTA)
static_assert(kUmEpiWarp0 % 4 == 0, "epilogue warps must cover the four TMEM lane quarters in order");
static_assert(kUmAccCol0 + kUmNAcc * kUmAccCols <= kUmTmemCols, "TMEM columns");
static_assert(kUmNA >= kUmGroups, "every dequant group needs a stage slot");
static_assert(kUmN % 32 == 0 && kUmBBlock % 1024 == 0, "pair MMA N and swizzle atoms");

struct alignas(64) UmParams {
  CUtensorMap b_map[4];  // B rows: fp16 [rows, n_in], boxes {64, 16 / 64 / 128 / 192 rows}, 128B swizzle
  CUtensorMap q_map[2];  // packed codes: uint8 [E*n_out, row bytes], box {128, R}, 128B swizzle
  CUtensorMap s_map[2];  // scales: bf16 or e8m0 [E*n_out, groups], box {16 bytes, R}
  CUtensorMap z_map[2];  // biases: bf16 (affine)
  __half* hout;          // stage 1 output H [P, ld_h]
  float* yout;           // stage 2 output y [P, ld_y]
  int ld_h, ld_y;
  int n_in, n_out;       // per-expert shape of each A matrix
  int group;
  int row_bytes, gpr;    // packed bytes and scale groups per weight row
  int lg_group;          // log2(group)
  int T;                 // shared expert: tokens
  int shared;            // 1: one expert over positions 0..T-1 (no tile table)
  const int4* tiles;     // routed token tiles {expert, first position, tokens, 0}
  const int* n_tiles;
  int pos_base;          // row of position 0 in the B tensor and in H / y
  int* err;
};

template <int STAGE, int FMT>
struct UmCfg {
  static constexpr int bits = FMT == F_A2 ? 2 : FMT == F_A3 ? 3 : FMT == F_A8 ? 8 : 4;
  static constexpr bool mx = FMT == F_MX4;
  static constexpr int M = STAGE == 1 ? 2 : 1;          // matrices stacked in one tile
  static constexpr int R = 128 / M;                     // rows per matrix per tile
  // inputs per raw slot: one 128-byte box of codes per row (128B-swizzled),
  // for 3-bit codes a 96-byte box (256 inputs, no swizzle)
  static constexpr int KS = bits == 3 ? 256 : 128 * 8 / bits;
  static constexpr int BOXB = KS * bits / 8;            // packed bytes per row per slot
  static constexpr int QS = KS / kUmK;                  // MMA stages per raw slot (1, 2 or 4)
  static constexpr int PBOX = R * BOXB;
  static constexpr int SBOX = R * 16;
  static constexpr int NSB = bits == 2 ? 2 : 1;         // scale boxes reserved per matrix per slot
  static constexpr int packed_bytes = M * PBOX;
  static constexpr int scale_bytes = NSB * M * SBOX;
  static constexpr int slot_bytes = packed_bytes + 2 * scale_bytes;  // codes, scales, biases
  static constexpr int GBOX = mx ? 16 : 8;              // groups per 16-byte scale box
  static constexpr int ESZ = mx ? 1 : 2;                // scale element bytes
  static constexpr int NRS = 3;                         // raw slots
  // dequant warps reading one raw slot: its QS consecutive stages belong to
  // min(QS, groups) groups (the host admits only whole raw slots per row
  // when the groups do not all read every slot)
  static constexpr int RAW_USERS = 4 * (QS < kUmGroups ? QS : kUmGroups);
  static constexpr size_t smem = 1024 + NRS * (size_t)slot_bytes + (size_t)kUmBStages * kUmBTile + 256;
  static_assert(slot_bytes % 1024 == 0, "raw slots keep the 1024-byte alignment of the swizzled boxes");
  static_assert(smem <= 227 * 1024, "TMA/TMEM FFN exceeds the per-block shared memory limit");
};

// ------------------------------------------------------------ PTX wrappers
MOE_DEV void um_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// 2D tiled TMA load (no multicast) completing on `bar`
MOE_DEV void um_tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
MOE_DEV void um_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// this thread's 16 consecutive 32-bit TMEM columns of its lane (complete
// after tmem_st_wait)
MOE_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
MOE_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// D[tmem] (+)= A[tmem] . B[smem]^T, fp16 inputs, fp32 accumulation
MOE_DEV void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}
// the pair MMA: D[tmem] (+)= A[tmem, both CTAs] . B[smem, both CTAs]^T, M = 256
MOE_DEV void umma2_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive, once the pair MMAs issued so far have completed, on the barrier at
// this shared-memory offset in both CTAs of the pair
MOE_DEV void umma2_commit_both(uint32_t bar) {
  asm volatile(
      "{\n .reg .b16 m;\n mov.b16 m, 3;\n"
      " tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n}\n" ::"r"(
          bar)
      : "memory");
}
// kind::f16, fp16 A and B, fp32 D, both K-major, M = 256 (the pair), N = n
MOE_DEV uint32_t umma2_idesc_f16(int n) { return (1u << 4) | ((uint32_t)(n >> 3) << 17) | (16u << 24); }
// the same shared-memory offset in CTA `rank` of the cluster
MOE_DEV uint32_t cl_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// arrive on a barrier of either CTA of the pair (default release semantics;
// a cluster-scope release here costs about 1.5k cycles per arrive)
MOE_DEV void cl_arrive(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
MOE_DEV bool cl_bar_try(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(b), "r"(parity), "r"(20000)
      : "memory");
  return ok != 0;
}
// bounded wait on a barrier that the peer CTA or the pair MMA arrives on;
// false once this CTA has aborted or the wait gave up
MOE_DEV bool cl_bar_wait(uint32_t b, uint32_t parity, volatile int* abort_flag) {
  if (cl_bar_try(b, parity)) return true;
  const long long t0 = clock64();
  while (!cl_bar_try(b, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kTcWaitCycles) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}
// 2D tiled TMA load of this CTA's half of a pair operand, completing on the
// leader CTA's barrier (a shared::cluster address)
MOE_DEV void um_tma_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}
MOE_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
MOE_DEV uint32_t um_lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
MOE_DEV uint32_t um_lds8(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// ------------------------------------------------------------ work items
MOE_DEV int4 um_tile(const UmParams& p, int j) {
  if (p.shared) {
    const int pos0 = j * kUmN;
    return make_int4(0, pos0, min(kUmN, p.T - pos0), 0);
  }
  return __ldcg(p.tiles + j);
}

// Walks this pair's items (pair, +npairs, ...), each in n_sub sub-steps
// (MMA stages or raw slots), with the next item's tile loaded ahead; k counts
// the pair's items.
struct UmCursor {
  int item, sub, mt, k, step;
  int4 tile, nxt;
  MOE_DEV void init(const UmParams& p, int n_items, int n_mt, int pair, int npairs) {
    item = pair;
    step = npairs;
    sub = 0;
    k = 0;
    mt = item % n_mt;
    tile = item < n_items ? um_tile(p, item / n_mt) : make_int4(0, 0, 0, 0);
    const int n2 = item + step;
    nxt = n2 < n_items ? um_tile(p, n2 / n_mt) : make_int4(0, 0, 0, 0);
  }
  MOE_DEV void next_item(const UmParams& p, int n_items, int n_mt) {
    sub = 0;
    ++k;
    item += step;
    mt = item % n_mt;
    tile = nxt;
    const int n2 = item + step;
    if (n2 < n_items) nxt = um_tile(p, n2 / n_mt);
  }
  MOE_DEV void advance(const UmParams& p, int n_items, int n_mt, int n_sub) {
    if (++sub == n_sub) next_item(p, n_items, n_mt);
  }
};

// MMA width of a tile (tokens rounded up to 32: N/2 rows per CTA, 16-row multiples)
MOE_DEV int um_np(int tokens) { return tokens <= 32 ? 32 : (tokens + 31) & ~31; }
// token box of a CTA's half: 0..3 = 16, 32, 64, 96 rows
MOE_DEV int um_box(int half) { return half <= 16 ? 0 : half <= 32 ? 1 : half <= 64 ? 2 : 3; }
MOE_DEV int um_box_rows(int h) { return h == 0 ? 16 : h == 1 ? 32 : h == 2 ? 64 : 96; }

// ------------------------------------------------------------ the kernel
// Launched in clusters of two CTAs (gridDim.x even).
template <int STAGE, int FMT>
__global__ void __launch_bounds__(kUmThreads, 1) ffn_umma_kernel(const __grid_constant__ UmParams p) {
  using C = UmCfg<STAGE, FMT>;
  constexpr int M = C::M, QS = C::QS, NRS = C::NRS, NB = kUmBStages;
  constexpr int NA = kUmNA, NAC = kUmNAcc, NG = kUmGroups;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw32 = tc_smem(smem_raw);
  const uint32_t base = (raw32 + 1023u) & ~1023u;  // swizzled boxes need 1024-byte alignment
  const uint32_t slot0 = base;                      // raw slots: [codes | scales | biases] x NRS
  const uint32_t bt0 = base + (uint32_t)(NRS * C::slot_bytes);  // B stages
  const uint32_t bar = bt0 + (uint32_t)(NB * kUmBTile);
  uint8_t* bar_gen = smem_raw + (bar - raw32);
  // barriers marked (L) are used in the leader CTA only: the peer arrives on
  // the leader's copy; the others are per CTA
  constexpr int BA = 2 * NRS + 2 * NB;
  auto raw_full = [&](int s) { return bar + 8u * s; };                         // [NRS] TMA bytes
  auto raw_empty = [&](int s) { return bar + 8u * (NRS + s); };                // [NRS] dequant warps
  auto b_full = [&](int s) { return bar + 8u * (2 * NRS + s); };               // [NB] (L) TMA bytes of both CTAs
  auto b_empty = [&](int s) { return bar + 8u * (2 * NRS + NB + s); };         // [NB] pair MMA commit
  auto a_full = [&](int s) { return bar + 8u * (BA + s); };                    // [NA] (L) 4 + 4 dequant warps
  auto a_empty = [&](int s) { return bar + 8u * (BA + NA + s); };              // [NA] pair MMA commit
  auto acc_full = [&](int s) { return bar + 8u * (BA + 2 * NA + s); };         // [NAC] pair MMA commit
  auto acc_empty = [&](int s) { return bar + 8u * (BA + 2 * NA + NAC + s); };  // [NAC] (L) 4 + 4 epilogue warps
  const uint32_t drain = bar + 8u * (BA + 2 * NA + 2 * NAC);                   // (L)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_gen + 8 * (BA + 2 * NA + 2 * NAC + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert(8 * (BA + 2 * NA + 2 * NAC + 1) + 8 <= 256, "barrier block");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t rank, pair, npairs;
  asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  asm("mov.u32 %0, %%clusterid.x;" : "=r"(pair));
  asm("mov.u32 %0, %%nclusterid.x;" : "=r"(npairs));
  const bool leader = rank == 0;
  const int n_mt = p.n_out / (STAGE == 1 ? kUmRowsS1 : kUmRowsS2);
  const int n_kt = p.n_in / kUmK;
  const int n_rng = (n_kt + QS - 1) / QS;
  const int n_tiles = p.shared ? (p.T + kUmN - 1) / kUmN : __ldcg(p.n_tiles);
  const int n_items = n_tiles * n_mt;
  const int my_items = (int)pair < n_items ? (n_items - 1 - (int)pair) / (int)npairs + 1 : 0;
  const int total = my_items * n_kt;
  const int nsb = C::mx ? 1 : max(1, C::KS / p.group / 8);  // scale boxes per matrix per slot
  const int m_rows = STAGE == 1 ? 64 : 128;                  // rows per matrix of this CTA's A tile

  if (tid == 0) {
    for (int s = 0; s < NRS; ++s) {
      tc_bar_init(raw_full(s), 1);
      tc_bar_init(raw_empty(s), C::RAW_USERS);
    }
    for (int s = 0; s < NB; ++s) {
      tc_bar_init(b_full(s), 1);
      tc_bar_init(b_empty(s), 1);
    }
    for (int s = 0; s < NA; ++s) {
      tc_bar_init(a_full(s), 8);
      tc_bar_init(a_empty(s), 1);
    }
    for (int s = 0; s < NAC; ++s) {
      tc_bar_init(acc_full(s), 1);
      tc_bar_init(acc_empty(s), 8);
    }
    tc_bar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kUmMmaWarp) {  // the same warp in both CTAs allocates the pair's columns
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(tmem_slot)),
                 "r"(kUmTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kUmDqWarps) {
    // ================= dequant warps: group G takes the stages g = G mod NG
    // into A slot g mod NA; warp quarter q owns TMEM lanes 32q..32q+31 (= A rows)
    const int G = warp >> 2, q = warp & 3;
    const int m = STAGE == 1 ? (lane >> 4) : 0;                        // matrix of this lane's row
    const int rr = STAGE == 1 ? 16 * q + (lane & 15) : 32 * q + lane;  // row within that matrix's box
    UmCursor cur;
    cur.init(p, n_items, n_mt, pair, npairs);
    for (int i = 0; i < G && i < total; ++i) cur.advance(p, n_items, n_mt, n_kt);
    int held = -1;  // raw slot sequence number whose data this group is reading
    bool bad = false;
    for (int g = G; g < total; g += NG) {
      const int as = g % NA;
      const uint32_t tcol = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)as * kUmASlotCols;
      const int kt = cur.sub, qs = kt % QS, ri = kt / QS;
      const int seq = cur.k * n_rng + ri;
      const int rs = seq % NRS;
      bool ok = true;
      if (seq != held) {
        ok = tc_bar_wait(raw_full(rs), (uint32_t)(seq / NRS) & 1u, abort_flag);
        held = seq;
      }
      if (ok && g >= NA) ok = cl_bar_wait(a_empty(as), (uint32_t)(g / NA - 1) & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.st below is warp-collective
      const uint32_t slot = slot0 + (uint32_t)(rs * C::slot_bytes);
      const uint32_t prow = slot + (uint32_t)(m * C::PBOX + rr * C::BOXB);
      const int x0 = ((ri * C::KS) >> p.lg_group) & ~(C::GBOX - 1);
      uint32_t w3[12];  // 3-bit codes: the stage's 48 bytes of this row (unswizzled box)
      if constexpr (C::bits == 3) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const uint4 v = tc_lds128(prow + (uint32_t)(qs * 48 + 16 * c));
          w3[4 * c] = v.x; w3[4 * c + 1] = v.y; w3[4 * c + 2] = v.z; w3[4 * c + 3] = v.w;
        }
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {  // 32 inputs per block
        const int ko = qs * kUmK + 32 * b;        // input offset inside the slot
        const int bo = ko * C::bits / 8;          // byte offset inside the 128-byte row
        uint32_t w[8];
        if constexpr (C::bits == 8) {
          const uint4 v0 = tc_lds128(prow + (uint32_t)((((bo >> 4)) ^ (rr & 7)) << 4));
          const uint4 v1 = tc_lds128(prow + (uint32_t)((((bo >> 4) + 1) ^ (rr & 7)) << 4));
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
          w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
        } else if constexpr (C::bits == 4) {
          const uint4 v0 = tc_lds128(prow + (uint32_t)(((bo >> 4) ^ (rr & 7)) << 4));
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        } else if constexpr (C::bits == 3) {
          w[0] = w3[3 * b]; w[1] = w3[3 * b + 1]; w[2] = w3[3 * b + 2];
        } else {
          const uint2 v0 = tc_lds64(prow + (uint32_t)(((bo >> 4) ^ (rr & 7)) << 4) + (uint32_t)(bo & 15));
          w[0] = v0.x; w[1] = v0.y;
        }
        const int gi = ((ri * C::KS + ko) >> p.lg_group) - x0;
        const uint32_t saddr = slot + (uint32_t)(C::packed_bytes + ((gi / C::GBOX) * M + m) * C::SBOX + rr * 16 +
                                                 (gi % C::GBOX) * C::ESZ);
        uint32_t out[16];
        if constexpr (C::mx) {
          const uint32_t e = um_lds8(saddr);
          uint32_t f = 0;  // 2^(e-113) in fp16 (see tc_dequant32_mx)
          if (e > 128) bad = true;
          else if (e >= 99) f = (e - 98u) << 10;
          tc_dequant32_mx(w, f | (f << 16), out);
        } else {
          const float sf = __uint_as_float(um_lds16(saddr) << 16);
          const float bf = __uint_as_float(um_lds16(saddr + C::scale_bytes) << 16);
          if (!(fabsf(sf) * (float)((1 << C::bits) - 1) + fabsf(bf) <= kF16Max)) bad = true;
          const __half hs = __float2half_rn(sf), hb = __float2half_rn(bf);
          tc_dequant32<FMT>(w, h2u(__halves2half2(hs, hs)), h2u(__halves2half2(hb, hb)), out);
        }
        tmem_st16(tcol + 16u * b, out);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) cl_arrive(cl_addr(a_full(as), 0));
      for (int i = 0; i < NG && g + i < total; ++i) cur.advance(p, n_items, n_mt, n_kt);
      const int next_seq = g + NG < total ? cur.k * n_rng + cur.sub / QS : -1;
      if (next_seq != seq && lane == 0) tc_bar_arrive(raw_empty(rs));  // this group's last use of the slot
    }
    if (bad) set_error(p.err, kErrDeviceInput);
  } else if (warp == kUmRawWarp) {
    // ================= TMA issuer: this CTA's packed codes, scales, biases (up to NRS slots ahead)
    if (lane == 0) {
      for (int mm = 0; mm < M; ++mm) {
        um_prefetch_map(&p.q_map[mm]);
        um_prefetch_map(&p.s_map[mm]);
        if constexpr (!C::mx) um_prefetch_map(&p.z_map[mm]);
      }
      UmCursor rcur;
      rcur.init(p, n_items, n_mt, pair, npairs);
      const int raw_total = my_items * n_rng;
      for (int seq = 0; seq < raw_total; ++seq) {
        const int rs = seq % NRS;
        if (seq >= NRS && !tc_bar_wait(raw_empty(rs), (uint32_t)(seq / NRS - 1) & 1u, abort_flag)) break;
        const uint32_t slot = slot0 + (uint32_t)(rs * C::slot_bytes);
        const int ri = rcur.sub;
        const int row = rcur.tile.x * p.n_out + rcur.mt * 2 * m_rows + (int)rank * m_rows;
        const int xp = ri * C::BOXB;
        const int x0 = ((ri * C::KS) >> p.lg_group) & ~(C::GBOX - 1);
        const int ns = min(nsb, (p.gpr - x0 + C::GBOX - 1) / C::GBOX);  // boxes past the row end are skipped
        um_expect_tx(raw_full(rs), (uint32_t)(M * (C::PBOX + ns * C::SBOX * (C::mx ? 1 : 2))));
#pragma unroll
        for (int mm = 0; mm < M; ++mm) {
          um_tma_2d(slot + (uint32_t)(mm * C::PBOX), &p.q_map[mm], xp, row, raw_full(rs));
          for (int sb = 0; sb < ns; ++sb) {
            const uint32_t so = slot + (uint32_t)(C::packed_bytes + (sb * M + mm) * C::SBOX);
            um_tma_2d(so, &p.s_map[mm], x0 + sb * C::GBOX, row, raw_full(rs));
            if constexpr (!C::mx) um_tma_2d(so + C::scale_bytes, &p.z_map[mm], x0 + sb * C::GBOX, row, raw_full(rs));
          }
        }
        rcur.advance(p, n_items, n_mt, n_rng);
      }
    }
    __syncwarp();
  } else if (warp == kUmBWarp) {
    // ================= TMA issuer: this CTA's half of the token tile, two
    // 64-input column blocks per stage; both halves complete on the leader's
    // barrier, whose expected bytes the leader posts
    if (lane == 0) {
      for (int h = 0; h < 4; ++h) um_prefetch_map(&p.b_map[h]);
      UmCursor cur;
      cur.init(p, n_items, n_mt, pair, npairs);
      for (int g = 0; g < total; ++g) {
        const int bs = g % NB;
        if (g >= NB && !cl_bar_wait(b_empty(bs), (uint32_t)(g / NB - 1) & 1u, abort_flag)) break;
        const int half = um_np(cur.tile.z) >> 1;
        const int h = um_box(half);
        const int box_rows = um_box_rows(h);
        if (leader) um_expect_tx(b_full(bs), (uint32_t)(2 * 2 * box_rows * 128));
        const uint32_t dst = bt0 + (uint32_t)(bs * kUmBTile);
        const int y = p.pos_base + cur.tile.y + (int)rank * half;
        const uint32_t fb = cl_addr(b_full(bs), 0);
        um_tma_2d_pair(dst, &p.b_map[h], cur.sub * kUmK, y, fb);
        um_tma_2d_pair(dst + kUmBBlock, &p.b_map[h], cur.sub * kUmK + kUmKB, y, fb);
        cur.advance(p, n_items, n_mt, n_kt);
      }
    }
    __syncwarp();
  } else if (warp == kUmMmaWarp) {
    // ================= MMA issuer (leader CTA): 8 pair MMAs (K = 16 each) per stage
    if (leader && lane == 0) {
      UmCursor cur;
      cur.init(p, n_items, n_mt, pair, npairs);
      const uint64_t db_base = umma_desc(bt0);
      int g = 0;
      for (int it = 0; it < my_items && !*abort_flag; ++it) {
        const uint32_t idesc = umma2_idesc_f16(um_np(cur.tile.z));
        const int ab = it % NAC;
        if (it >= NAC && !cl_bar_wait(acc_empty(ab), (uint32_t)(it / NAC - 1) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + kUmAccCol0 + (uint32_t)ab * kUmAccCols;
        bool ok = true;
        for (int kt = 0; kt < n_kt; ++kt, ++g) {
          const int as = g % NA, bs = g % NB;
          if (!cl_bar_wait(a_full(as), (uint32_t)(g / NA) & 1u, abort_flag) ||
              !cl_bar_wait(b_full(bs), (uint32_t)(g / NB) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = tmem_base + (uint32_t)as * kUmASlotCols;
          // B descriptor start advances 32 bytes per K = 16 inside a column
          // block, and one column block after four MMAs
          const uint64_t db0 = db_base + (uint64_t)((bs * kUmBTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma2_f16_ts(d, a0 + 8u * kk, db0 + (uint64_t)(((kk >> 2) * kUmBBlock + (kk & 3) * 32) >> 4), idesc,
                         (kt | kk) ? 1u : 0u);
          umma2_commit_both(a_empty(as));
          umma2_commit_both(b_empty(bs));
        }
        if (!ok) break;
        umma2_commit_both(acc_full(ab));
        cur.next_item(p, n_items, n_mt);
      }
      umma2_commit_both(drain);
      const long long t0 = clock64();
      while (!cl_bar_try(drain, 0) && clock64() - t0 < kTcWaitCycles) {
      }
    }
    __syncwarp();
  } else if (warp >= kUmEpiWarp0) {
    // ================= epilogue: this CTA's 128 accumulator rows
    const int q = warp & 3;
    UmCursor cur;
    cur.init(p, n_items, n_mt, pair, npairs);
    bool bad = false;
    for (int it = 0; it < my_items; ++it) {
      const int ab = it % NAC;
      const bool ok = cl_bar_wait(acc_full(ab), (uint32_t)(it / NAC) & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld is warp-collective
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + kUmAccCol0 + (uint32_t)ab * kUmAccCols;
      const int ntok = cur.tile.z;
      const int prow0 = p.pos_base + cur.tile.y;
      for (int nb = 0; nb < ntok; nb += 16) {
        float v[16];
        tmem_ld16(taddr + (uint32_t)nb, v);
        if constexpr (STAGE == 1) {
          // lanes 0-15: gate of features f, lanes 16-31: up of the same f;
          // the low half finishes token columns 0-7, the high half 8-15
          const bool lo = lane < 16;
          const int f = cur.mt * kUmRowsS1 + (int)rank * 64 + 16 * q + (lane & 15);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float send = lo ? v[8 + jj] : v[jj];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const float gv = lo ? v[jj] : recv;
            const float uv = lo ? recv : v[8 + jj];
            const int n = nb + (lo ? jj : 8 + jj);
            if (n < ntok) {
              const float hv = __fdividef(gv * uv, 1.f + __expf(-gv));  // silu(g) * u
              bad |= !(fabsf(hv) <= kF16Max);
              p.hout[(size_t)(prow0 + n) * p.ld_h + f] = __float2half_rn(hv);
            }
          }
        } else {
          const int row = cur.mt * kUmRowsS2 + (int)rank * 128 + 32 * q + lane;
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            if (nb + jj < ntok) p.yout[(size_t)(prow0 + nb + jj) * p.ld_y + row] = v[jj];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) cl_arrive(cl_addr(acc_empty(ab), 0));
      cur.next_item(p, n_items, n_mt);
    }
    if (bad) set_error(p.err, kErrDeviceInput);
  }
  __syncthreads();
  tc_fence_before();
  cluster_sync_all();  // the pair's MMAs have drained; neither CTA's memory is read from now on
  tc_fence_after();
  if (tid == 0 && *abort_flag) set_error(p.err, kErrTimeout);
  if (warp == kUmMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kUmTmemCols)
                 : "memory");
}

// Launch helpers, one translation unit per (stage, format).
// launch_*: `pairs` clusters of two CTAs; attrs_*: sets the kernel's
// attributes and returns how many pairs can be resident at once (0: none).
using UmLaunchFn = bool (*)(const UmParams& p, int pairs, cudaStream_t s);
using UmAttrFn = int (*)();
#define MOE_UM_DECL(ST, F)                                                  \
  bool launch_um_s##ST##_##F(const UmParams& p, int pairs, cudaStream_t s); \
  int attrs_um_s##ST##_##F();
MOE_UM_DECL(1, A2)
MOE_UM_DECL(1, A3)
MOE_UM_DECL(1, A4)
MOE_UM_DECL(1, A8)
MOE_UM_DECL(1, MX4)
MOE_UM_DECL(2, A2)
MOE_UM_DECL(2, A3)
MOE_UM_DECL(2, A4)
MOE_UM_DECL(2, A8)
MOE_UM_DECL(2, MX4)
#undef MOE_UM_DECL

}  // namespace moe
