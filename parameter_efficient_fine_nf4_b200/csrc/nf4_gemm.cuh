// Tensor-core GEMMs whose weight operand is dequantised from NF4 inside the
// kernel ([P1] "What QLoRA freezes, and in how many bits": W is stored as NF4
// with double-quantised block constants and is dequantised to BF16 for the
// multiply, in the forward pass and again for the activation gradient).
//
//   forward  Y  = [X | sU] [W' | B]^T      (M = T, N = d, K = k (+ r))
//   backward dX = [dY | sG] [W' ; A]       (M = T, N = k, K = d (+ r))
//
// W' never exists in global memory.  Dequantising warps read the packed codes
// of one K-step (staged in shared memory by TMA and read back with 128-bit
// loads) and the fp32 block scales a' of its blocks.  Above 64 tokens the
// scales are formed once per call by nf4_block_scales in a TMA-friendly layout
// and staged with the codes; the few-token kernels form them in the
// dequantising threads from the stored constants.  Per 64-weight block the
// 16 products bf16(level[i] * a') are formed once, each weight's value is
// selected from them with byte permutes on registers, and the bf16 tile is
// written in exactly the 128B-swizzled layout a TMA load of W' would have
// produced (K-major rows for the forward, MN-major for dX).  So the MMA sees
// the same operand bytes as on a dequantised weight and the result is
// bit-identical to the plain-LoRA GEMM on W'.
//
// Above 64 tokens (gemm_nf4_kernel), by default a cluster of two CTAs per SM
// pair runs 256-row tcgen05 MMAs over both SMs (cta_group::2) on units of 512
// tokens by 256 columns; each CTA decodes 128 of the 256 weight rows of a
// K-step, so per SM the decode halves at the same MMA work.  A one-CTA build
// (units of 256 tokens, the whole weight tile decoded per CTA) gives the same
// bits.  Warps: 0 activation and rank-r tile loads, 1 TMEM + MMA issue (rank
// 0 of a pair), 2-5 epilogue, 6 code and block-scale loads, 7.. dequantisation.
//
// At most 64 tokens (gemm_nf4_small_kernel) the products are computed with
// the operands swapped and the depth split over CTAs; see its section below.
#pragma once
#include "gemm_tc.cuh"
#include "nf4_kernels.cuh"
#include "ptx.cuh"

namespace qlora {

// ------------------------------------------------------------------ decode
// Per-block tables: entry i = bf16(level[i] * a') split into its low bytes
// (lo[j] holds entries 4j..4j+3) and high bytes (hi[j]).
struct Nf4Lut {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ Nf4Lut nf4_block_lut(float a, const float (&lv)[16]) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // one fp32 product per level, one round-to-nearest-even to bf16
    const float e0 = __fmul_rn(lv[2 * j], a);
    const float e1 = __fmul_rn(lv[2 * j + 1], a);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(P[j]) : "f"(e1), "f"(e0));
  }
  Nf4Lut t;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    t.lo[j] = prmt(P[2 * j], P[2 * j + 1], 0x6420u);
    t.hi[j] = prmt(P[2 * j], P[2 * j + 1], 0x7531u);
  }
  return t;
}

// Eight codes (nibble e of w = element e) -> eight bf16 values, packed in
// pairs (element 2i in the low half of word i).  The low three bits of each
// code pick a byte from entries 0-7 and from entries 8-15 (one permute each
// for the low and the high bytes); the code's top bit then selects between
// the two; a last permute interleaves low and high bytes.
__device__ __forceinline__ uint4 nf4_decode8(uint32_t w, const Nf4Lut& t) {
  uint4 o;
  asm("{\n\t"
      ".reg .b32 m, mh, x, s, sh, a0, a1, b0, b1, la, ha, lb, hb;\n\t"
      "and.b32 m, %4, 0x77777777;\n\t"
      "shr.u32 mh, m, 16;\n\t"
      "shr.u32 x, %4, 1;\n\t"
      "lop3.b32 s, x, 0x44444444, 0x32103210, 0xEA;\n\t"   // (x & 0x4..) | 0x3210..
      "shr.u32 sh, s, 16;\n\t"
      "prmt.b32 a0, %5, %6, m;\n\t"
      "prmt.b32 a1, %7, %8, m;\n\t"
      "prmt.b32 la, a0, a1, s;\n\t"
      "prmt.b32 b0, %9, %10, m;\n\t"
      "prmt.b32 b1, %11, %12, m;\n\t"
      "prmt.b32 ha, b0, b1, s;\n\t"
      "prmt.b32 %0, la, ha, 0x5140;\n\t"
      "prmt.b32 %1, la, ha, 0x7362;\n\t"
      "prmt.b32 a0, %5, %6, mh;\n\t"
      "prmt.b32 a1, %7, %8, mh;\n\t"
      "prmt.b32 lb, a0, a1, sh;\n\t"
      "prmt.b32 b0, %9, %10, mh;\n\t"
      "prmt.b32 b1, %11, %12, mh;\n\t"
      "prmt.b32 hb, b0, b1, sh;\n\t"
      "prmt.b32 %2, lb, hb, 0x5140;\n\t"
      "prmt.b32 %3, lb, hb, 0x7362;\n\t"
      "}"
      : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
      : "r"(w), "r"(t.lo[0]), "r"(t.lo[1]), "r"(t.lo[2]), "r"(t.lo[3]), "r"(t.hi[0]), "r"(t.hi[1]),
        "r"(t.hi[2]), "r"(t.hi[3]));
  return o;
}

// A whole 64-weight block: 32 code bytes as two 16-byte words -> eight
// 16-byte chunks of bf16 (chunk j = elements 8j .. 8j+7).
__device__ __forceinline__ void nf4_decode_block(uint4 c0, uint4 c1, float a, const float (&lv)[16],
                                                 uint4 (&o)[8]) {
  const Nf4Lut t = nf4_block_lut(a, lv);
  o[0] = nf4_decode8(c0.x, t);
  o[1] = nf4_decode8(c0.y, t);
  o[2] = nf4_decode8(c0.z, t);
  o[3] = nf4_decode8(c0.w, t);
  o[4] = nf4_decode8(c1.x, t);
  o[5] = nf4_decode8(c1.y, t);
  o[6] = nf4_decode8(c1.z, t);
  o[7] = nf4_decode8(c1.w, t);
}

// Half a block: the 32 codes of one uint4, with the block's table.
__device__ __forceinline__ void nf4_decode_half(uint4 c, float a, const float (&lv)[16], uint4 (&o)[4]) {
  const Nf4Lut t = nf4_block_lut(a, lv);
  o[0] = nf4_decode8(c.x, t);
  o[1] = nf4_decode8(c.y, t);
  o[2] = nf4_decode8(c.z, t);
  o[3] = nf4_decode8(c.w, t);
}

// ------------------------------------------------------------------ kernel
struct Nf4GemmArgs {
  int M, N, K0, K1;           // M tokens, N output columns, K0 main depth, K1 = r
  int tiles_m, tiles_n;       // tiles_m counts 256-row units
  int group_m;                // raster: units walk group_m tile rows per column
  int tma_store;              // bf16 output through shared staging + TMA stores
  uint16_t* out;              // direct-store fallback (rows not 16-byte aligned)
  int64_t ldo;
  float levels[16];
};

// Two builds of the kernel:
//   kPair = false: one CTA per unit of 256 rows x 256 columns; it decodes the
//                  whole 256-wide weight tile of each K-step (8 dequantising
//                  warps) and runs two 128-row MMAs on it.
//   kPair = true:  a cluster of two CTAs per unit of 512 rows x 256 columns,
//                  running pair MMAs (tcgen05 cta_group::2, M = 256): each
//                  CTA holds 128 rows of each of the unit's two 256-row A
//                  tiles and decodes 128 of the weight tile's 256 rows into
//                  its own shared memory, which the pair MMA reads from both
//                  SMs.  Per SM the MMA work per K-step is the same as one
//                  CTA's, the decode half of it.  Rank 0 issues the MMAs;
//                  the operand-ready barriers live in rank 0, the stage-free
//                  and accumulator-ready barriers in both CTAs (the MMA
//                  completions are multicast to both).
template <bool kPair>
struct Nf4Cfg {
  static constexpr int kDqWarps = kPair ? 4 : 8;
  // warps: 0 activation / rank-r loads, 1 MMA, 2-5 epilogue, 6 code loads,
  // 7.. dequantisation
  static constexpr int kDqWarp0 = 7;
  static constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
  static constexpr int SA = kPair ? 4 : 3;        // activation stages: two 128 x 64 bf16 tiles (32 KB)
  static constexpr int SB = kPair ? 3 : 2;        // weight stages: this CTA's rows of the 256 x 64 tile
  static constexpr int SC = 3;                    // code stages: codes + block scales
  static constexpr int kABytes = 32768;
  static constexpr int kBBytes = kPair ? 16384 : 32768;
  static constexpr int kCodeBytes = kPair ? 4096 : 8192;   // this CTA's rows of codes
  static constexpr int kCBytes = kCodeBytes + 1024;
  static constexpr int kStgBoxes = 2;             // epilogue staging: 4 KB boxes per warp
  static constexpr int kStage = 4 * kStgBoxes * 4096;
  // mbarriers of the rings, accumulator full / empty and drain, and three words
  static constexpr int kBarBytes = (2 * (SA + SB + SC) + 3) * 8 + 16;
  static constexpr int kSmemBytes = SA * kABytes + SB * kBBytes + SC * kCBytes + kStage + 1024 + 512;
  static_assert(kBarBytes <= 512, "barrier region");
  // arrivals that complete a weight stage: every dequantising warp of the
  // unit (a rank-r stage: the TMA thread's expect_tx plus the rest)
  static constexpr int kBFull = kPair ? 2 * kDqWarps : kDqWarps;
  // arrivals that free the accumulators: the epilogue warps of the unit
  static constexpr int kAccEmpty = kPair ? 8 : 4;
  static constexpr int kRowsPerUnit = kPair ? 512 : 256;
};
constexpr int kNf4Threads = Nf4Cfg<false>::kThreads;         // 480
constexpr int kNf4PairThreads = Nf4Cfg<true>::kThreads;      // 352

struct Nf4Unit {
  int m0, n0;
};
// Unit u of the raster: tiles_m counts units of `rows` rows of M.
__device__ __forceinline__ Nf4Unit nf4_unit(const Nf4GemmArgs& p, int u, int rows) {
  const int per_group = p.group_m * p.tiles_n;
  const int gidx = u / per_group;
  const int first_m = gidx * p.group_m;
  const int gsize = min(p.group_m, p.tiles_m - first_m);
  const int in_group = u - gidx * per_group;
  Nf4Unit r;
  r.m0 = (first_m + in_group % gsize) * rows;
  r.n0 = (in_group / gsize) * 256;
  return r;
}

// Waits for a phase with a short limit, used only to let copies already in
// flight land before an aborting CTA exits.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t start = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - start > 10000000ull) return;
  }
}

// Waits (bounded, no abort flag) for the last `n` ring uses before `g` of a
// stage ring of S barriers to complete: used before exit so that no MMA
// completion is still on its way to this CTA's barriers.
template <int S>
__device__ __forceinline__ void wait_ring_tail(const uint64_t* bars, int g, int n) {
  for (int q = 0; q < n && g - 1 - q >= 0; ++q) {
    const int last = g - 1 - q;
    mbar_wait_bounded<true>(smem_u32(&bars[last % S]), (uint32_t)((last / S) & 1), nullptr);
  }
}

// Loads one activation (or rank-r operand) tile: into this CTA, completing on
// `bar` (a local barrier for one CTA; rank 0's, as a cluster address, in a pair).
template <bool kPair>
__device__ __forceinline__ void nf4_tile_load(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  if constexpr (kPair)
    tma_load_2d_pair(dst, map, bar, x, y);
  else
    tma_load_2d(dst, map, bar, x, y);
}

// kDx = false: forward (W' rows are N, K-major tiles); true: dX (W' rows are
// K, MN-major tiles).
template <bool kDx, bool kPair>
__global__ void __launch_bounds__(Nf4Cfg<kPair>::kThreads, 1)
    gemm_nf4_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmOut,
                    const __grid_constant__ Nf4GemmArgs p) {
  using Cfg = Nf4Cfg<kPair>;
  constexpr int SA = Cfg::SA, SB = Cfg::SB, SC = Cfg::SC;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  const uint32_t sA = sbase;
  const uint32_t sB = sA + SA * Cfg::kABytes;
  const uint32_t sC = sB + SB * Cfg::kBBytes;
  const uint32_t sStg = sC + SC * Cfg::kCBytes;
  uint8_t* stg_ptr = smem + (sStg - sbase);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (sStg - sbase) + Cfg::kStage);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + SA;
  uint64_t* b_full = a_empty + SA;
  uint64_t* b_empty = b_full + SB;
  uint64_t* c_full = b_empty + SB;
  uint64_t* c_empty = c_full + SC;
  uint64_t* acc_full = c_empty + SC;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain_bar = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  // a barrier that completes the unit's operands: this CTA's, or rank 0's in a pair
  auto lead_bar = [&](const uint64_t* b) -> uint32_t {
    return kPair ? mapa_shared(smem_u32(b), 0) : smem_u32(b);
  };
  const int unit0 = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ustride = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int units = p.tiles_m * p.tiles_n;
  const int steps0 = (p.K0 + 63) / 64;
  const int steps1 = (p.K1 + 63) / 64;
  const int steps = steps0 + steps1;
  // Rows of a unit held by this CTA: A tile t (t = 0, 1) starts at row
  // m0 + t * tile_step + row_off of the unit starting at m0.
  const int tile_step = kPair ? 256 : 128;
  const int row_off = kPair ? 128 * (int)rank : 0;
  // The unit's second tile (second 256 rows of a pair unit) is used only if
  // it holds rows below M; both CTAs of a pair decide alike.
  auto has_second = [&](int m0) -> bool { return m0 + tile_step < p.M; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < SA; ++i) {
      mbar_init(smem_u32(&a_full[i]), 1);
      mbar_init(smem_u32(&a_empty[i]), 1);
    }
    for (int i = 0; i < SB; ++i) {
      mbar_init(smem_u32(&b_full[i]), Cfg::kBFull);
      mbar_init(smem_u32(&b_empty[i]), 1);
    }
    for (int i = 0; i < SC; ++i) {
      mbar_init(smem_u32(&c_full[i]), 1);
      mbar_init(smem_u32(&c_empty[i]), Cfg::kDqWarps);
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_empty), Cfg::kAccEmpty);
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmS);
    if (steps1 > 0) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
    if (p.tma_store) tma_prefetch_desc(&tmOut);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the peer's barriers are initialised before anyone signals them
  if (kPair) cluster_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // (activation tiles, and the rank-r weight tiles of the extension steps)
    if (lane == 0) {
      int a_iss[SA];
      int b_last[SB];                  // ring use index of this warp's last weight-tile load per stage
      for (int i = 0; i < SA; ++i) a_iss[i] = 0;
      for (int i = 0; i < SB; ++i) b_last[i] = -1;
      int g = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += ustride) {
        const Nf4Unit c = nf4_unit(p, u, Cfg::kRowsPerUnit);
        const bool has2 = has_second(c.m0);
        const int mA = c.m0 + row_off;
        for (int step = 0; step < steps; ++step, ++g) {
          const int sa = g % SA;
          if (!mbar_wait_bounded<kPair>(smem_u32(&a_empty[sa]), (uint32_t)(((g / SA) & 1) ^ 1), abort_flag)) {
            ok = false;
            break;
          }
          const bool ext = step >= steps0;
          const int e = step - steps0;
          const uint32_t fa = lead_bar(&a_full[sa]);
          // rank 0 expects the tiles of both CTAs of a pair
          if (leader)
            mbar_arrive_expect_tx(smem_u32(&a_full[sa]), (uint32_t)((has2 ? 2 : 1) * 16384 * (kPair ? 2 : 1)));
          const CUtensorMap* ma = ext ? &tmA1 : &tmA0;
          const int x = ext ? e * 64 : step * 64;
          nf4_tile_load<kPair>(sA + sa * Cfg::kABytes, ma, fa, x, mA);
          if (has2) nf4_tile_load<kPair>(sA + sa * Cfg::kABytes + 16384, ma, fa, x, mA + tile_step);
          a_iss[sa] += 1;
          if (ext) {
            // rank-r weight operand: B rows (forward) or A columns (dX) by
            // TMA, this CTA's half of the tile in a pair
            const int sb = g % SB;
            if (!mbar_wait_bounded<kPair>(smem_u32(&b_empty[sb]), (uint32_t)(((g / SB) & 1) ^ 1), abort_flag)) {
              ok = false;
              break;
            }
            const uint32_t fb = lead_bar(&b_full[sb]);
            if (leader) {
              mbar_arrive_expect_tx(smem_u32(&b_full[sb]), (uint32_t)(kPair ? 2 * Cfg::kBBytes : Cfg::kBBytes));
              mbar_arrive_count(smem_u32(&b_full[sb]), Cfg::kBFull - 1);
            }
            const int nb = kPair ? 128 : 256;              // rows (forward) or MN columns (dX) loaded here
            const int n1 = c.n0 + (kPair ? 128 * (int)rank : 0);
            if (kDx) {
              for (int i = 0; i < nb / 64; ++i)
                nf4_tile_load<kPair>(sB + sb * Cfg::kBBytes + i * 8192, &tmB1, fb, n1 + 64 * i, e * 64);
            } else {
              nf4_tile_load<kPair>(sB + sb * Cfg::kBBytes, &tmB1, fb, e * 64, n1);
            }
            b_last[sb] = g / SB;
          }
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits (a pair's
        // operand loads complete on rank 0's barriers: rank 0 drains them)
        if (leader) {
          for (int i = 0; i < SA; ++i)
            if (a_iss[i] > 0) mbar_wait_drain(smem_u32(&a_full[i]), (uint32_t)((a_iss[i] - 1) & 1));
          for (int i = 0; i < SB; ++i)
            if (b_last[i] >= 0) mbar_wait_drain(smem_u32(&b_full[i]), (uint32_t)(b_last[i] & 1));
        }
      } else if (kPair) {
        // the last stage releases (rank 0's MMA completions) have reached this CTA
        wait_ring_tail<SA>(a_empty, g, SA);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ code loads
    // Codes and block scales of this CTA's rows of each main K-step's weight
    // tile; they run ahead of the MMA by as many stages as the decode allows.
    if (lane == 0) {
      int c_iss[SC];
      for (int i = 0; i < SC; ++i) c_iss[i] = 0;
      int gc = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += ustride) {
        const Nf4Unit c = nf4_unit(p, u, Cfg::kRowsPerUnit);
        for (int step = 0; step < steps0; ++step, ++gc) {
          const int sc = gc % SC;
          if (!mbar_wait_bounded(smem_u32(&c_empty[sc]), (uint32_t)(((gc / SC) & 1) ^ 1), abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fc = smem_u32(&c_full[sc]);
          const uint32_t cdst = sC + sc * Cfg::kCBytes;
          if (kDx) {
            mbar_arrive_expect_tx(fc, (uint32_t)(Cfg::kCodeBytes + 1024));
            // codes of 64 K-rows x this CTA's MN columns; scales of the
            // tile's 4 block columns
            tma_load_2d(cdst, &tmC, fc, c.n0 / 2 + (kPair ? 64 * (int)rank : 0), step * 64);
            tma_load_2d(cdst + Cfg::kCodeBytes, &tmS, fc, c.n0 / 64, step * 64);
          } else {
            const int rows = kPair ? 128 : 256;
            mbar_arrive_expect_tx(fc, (uint32_t)(Cfg::kCodeBytes + rows * 4));
            // codes and scales of this CTA's rows at block column `step`
            tma_load_2d(cdst, &tmC, fc, step * 32, c.n0 + (kPair ? 128 * (int)rank : 0));
            tma_load_2d(cdst + Cfg::kCodeBytes, &tmS, fc, c.n0 + (kPair ? 128 * (int)rank : 0), step);
          }
          c_iss[sc] += 1;
        }
      }
      if (*abort_flag) {
        for (int i = 0; i < SC; ++i)
          if (c_iss[i] > 0) mbar_wait_drain(smem_u32(&c_full[i]), (uint32_t)((c_iss[i] - 1) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      const uint64_t adesc = smem_desc_sw128(sA, 16, 1024);
      const uint64_t bdesc = kDx ? smem_desc_sw128(sB, 8192, 1024) : smem_desc_sw128(sB, 16, 1024);
      const uint32_t bstep = kDx ? 128u : 2u;
      const uint32_t idesc = idesc_bf16_f32(kPair ? 256 : 128, 256, 0, kDx ? 1 : 0);
      bool ok = true;
      int issued_any = 0;
      int g = 0, it = 0;
      for (int u = unit0; u < units && ok; u += ustride, ++it) {
        const Nf4Unit c = nf4_unit(p, u, Cfg::kRowsPerUnit);
        const bool has2 = has_second(c.m0);
        if (!mbar_wait_bounded<kPair>(smem_u32(acc_empty), (uint32_t)((it & 1) ^ 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int step = 0; step < steps; ++step, ++g) {
          const int sa = g % SA;
          const int sb = g % SB;
          if (!mbar_wait_bounded<kPair>(smem_u32(&a_full[sa]), (uint32_t)((g / SA) & 1), abort_flag) ||
              !mbar_wait_bounded<kPair>(smem_u32(&b_full[sb]), (uint32_t)((g / SB) & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool ext = step >= steps0;
          const int nsub = ext ? min(4, (p.K1 - (step - steps0) * 64 + 15) / 16) : 4;
          const uint64_t a0 = adesc + (uint64_t)((sa * Cfg::kABytes) >> 4);
          const uint64_t b0 = bdesc + (uint64_t)((sb * Cfg::kBBytes) >> 4);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nsub) {
              const uint32_t acc = (step == 0 && j == 0) ? 0u : 1u;
              const uint64_t aj = a0 + (uint64_t)(2 * j), bj = b0 + (uint64_t)(j * bstep);
              if constexpr (kPair) {
                umma_bf16_pair(tmem_base, aj, bj, idesc, acc);
                if (has2) umma_bf16_pair(tmem_base + 256u, aj + 1024u, bj, idesc, acc);
              } else {
                umma_bf16(tmem_base, aj, bj, idesc, acc);
                if (has2) umma_bf16(tmem_base + 256u, aj + 1024u, bj, idesc, acc);
              }
            }
          }
          issued_any = 1;
          if constexpr (kPair) {
            // both CTAs' stages are free once the pair MMA has read them
            umma_commit_pair(smem_u32(&a_empty[sa]), (uint16_t)0x3);
            umma_commit_pair(smem_u32(&b_empty[sb]), (uint16_t)0x3);
          } else {
            umma_commit(smem_u32(&a_empty[sa]));
            umma_commit(smem_u32(&b_empty[sb]));
          }
        }
        if (ok) {
          if constexpr (kPair)
            umma_commit_pair(smem_u32(acc_full), (uint16_t)0x3);
          else
            umma_commit(smem_u32(acc_full));
        }
      }
      if (!ok && issued_any) {
        if constexpr (kPair)
          umma_commit_pair(smem_u32(drain_bar), (uint16_t)0x1);
        else
          umma_commit(smem_u32(drain_bar));
        mbar_wait_bounded(smem_u32(drain_bar), 0, nullptr);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    uint8_t* stg = stg_ptr + (warp - 2) * (Cfg::kStgBoxes * 4096);
    const uint32_t stg_s = sStg + (uint32_t)((warp - 2) * (Cfg::kStgBoxes * 4096));
    int it = 0, nbox = 0;
    for (int u = unit0; u < units; u += ustride, ++it) {
      const Nf4Unit c = nf4_unit(p, u, Cfg::kRowsPerUnit);
      const bool has2 = has_second(c.m0);
      const bool ok = mbar_wait_bounded<kPair>(smem_u32(acc_full), (uint32_t)(it & 1), abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      for (int t = 0; t < (has2 ? 2 : 1); ++t) {
        const int mrow0 = c.m0 + t * tile_step + row_off + quarter * 32;
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(t * 256);
        if (p.tma_store) {
#pragma unroll 1
          for (int b = 0; b < 4; ++b) {
            uint32_t v0[32], v1[32];
            tmem_ld_32x32b_x32(taddr + (uint32_t)(b * 64), v0);
            tmem_ld_32x32b_x32(taddr + (uint32_t)(b * 64 + 32), v1);
            tmem_ld_wait();
            if (mrow0 >= p.M) continue;          // rows of this warp lie beyond M
            if (nbox >= Cfg::kStgBoxes) {
              // the store that used this buffer has read it
              if (lane == 0) {
                if (Cfg::kStgBoxes == 2)
                  bulk_wait_group_read1();
                else
                  bulk_wait_group_read0();
              }
              __syncwarp();
            }
            const int slot = nbox % Cfg::kStgBoxes;
            uint8_t* box = stg + slot * 4096;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint32_t(&v)[32] = q < 4 ? v0 : v1;
              const int o = (q & 3) * 8;
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[o + 0]), __uint_as_float(v[o + 1]));
              w.y = pack_bf16x2(__uint_as_float(v[o + 2]), __uint_as_float(v[o + 3]));
              w.z = pack_bf16x2(__uint_as_float(v[o + 4]), __uint_as_float(v[o + 5]));
              w.w = pack_bf16x2(__uint_as_float(v[o + 6]), __uint_as_float(v[o + 7]));
              *reinterpret_cast<uint4*>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmOut, stg_s + (uint32_t)(slot * 4096), c.n0 + 64 * b, mrow0);
              bulk_commit_group();
            }
            ++nbox;
          }
        } else {
          const int m = mrow0 + lane;
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32), v);
            tmem_ld_wait();
            const int n = c.n0 + ch * 32;
            if (m < p.M) {
              uint16_t* o = p.out + (int64_t)m * p.ldo + n;
              for (int i = 0; i < 32 && n + i < p.N; ++i) {
                const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
                o[i] = *reinterpret_cast<const uint16_t*>(&h);
              }
            }
          }
        }
      }
      // the accumulators may be overwritten once all epilogue warps of the
      // unit (both CTAs of a pair) are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair && rank != 0)
          mbar_arrive_remote(lead_bar(acc_empty));
        else
          mbar_arrive(smem_u32(acc_empty));
      }
    }
    if (p.tma_store && lane == 0) bulk_wait_group0();
  } else {
    // ------------------------------------------------------------ dequantisation
    // Thread i of these warps owns one 64-weight block of each K-step's
    // weight tile.  Forward: local tile row i (W' row n0 + i; in a pair, rank
    // 1 holds rows n0 + 128 + i), block column = the K-step.  dX: K-row
    // kk = i % 64 (W' row 64 * step + kk) and local chunk cl = i / 64 (W'
    // block column n0 / 64 + cc, cc = cl, or 2 rank + cl in a pair).
    const int i = threadIdx.x - Cfg::kDqWarp0 * 32;
    const int kk = i & 63;
    const int cl = i >> 6;
    const int cc = kPair ? 2 * (int)rank + cl : cl;
    int g = 0, gc = 0;
    bool live = true;
    for (int u = unit0; u < units && live; u += ustride) {
      for (int step = 0; step < steps0; ++step, ++g, ++gc) {
        const int sc = gc % SC;
        bool ok = mbar_wait_bounded(smem_u32(&c_full[sc]), (uint32_t)((gc / SC) & 1), abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          live = false;
          break;
        }
        uint4 c0, c1;
        const uint32_t cs = sC + sc * Cfg::kCBytes;
        const float* scl = reinterpret_cast<const float*>(smem + (cs - sbase) + Cfg::kCodeBytes);
        float a;
        if (kDx) {
          if (kPair) {
            // 64-byte rows (this CTA's 128 MN columns), 64B swizzle: chunk j at (j ^ ((row >> 1) & 3))
            const uint32_t row = cs + kk * 64;
            const int sw = (kk >> 1) & 3;
            c0 = ld_shared_v4(row + (((2 * cl) ^ sw) << 4));
            c1 = ld_shared_v4(row + (((2 * cl + 1) ^ sw) << 4));
          } else {
            // 128-byte rows (K-rows), 128B swizzle: 16-byte chunk j at (j ^ (row & 7))
            const uint32_t row = cs + kk * 128;
            const int sw = kk & 7;
            c0 = ld_shared_v4(row + (((2 * cc) ^ sw) << 4));
            c1 = ld_shared_v4(row + (((2 * cc + 1) ^ sw) << 4));
          }
          a = scl[kk * 4 + cc];
        } else {
          // 32-byte rows, 32B swizzle: chunk j at (j ^ ((row >> 2) & 1))
          const uint32_t row = cs + i * 32;
          const int sw = (i >> 2) & 1;
          c0 = ld_shared_v4(row + ((0 ^ sw) << 4));
          c1 = ld_shared_v4(row + ((1 ^ sw) << 4));
          a = scl[i];
        }
        uint4 o[8];
        nf4_decode_block(c0, c1, a, p.levels, o);
        // the codes and scales are consumed (the decode read them): release the stage
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&c_empty[sc]));
        const int sb = g % SB;
        ok = mbar_wait_bounded<kPair>(smem_u32(&b_empty[sb]), (uint32_t)(((g / SB) & 1) ^ 1), abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          live = false;
          break;
        }
        uint32_t dst;
        int sw;
        if (kDx) {
          dst = sB + sb * Cfg::kBBytes + cl * 8192 + kk * 128;
          sw = kk & 7;
        } else {
          dst = sB + sb * Cfg::kBBytes + i * 128;
          sw = i & 7;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) st_shared_v4(dst + ((j ^ sw) << 4), o[j]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (kPair && rank != 0)
            mbar_arrive_remote(lead_bar(&b_full[sb]));
          else
            mbar_arrive(smem_u32(&b_full[sb]));
        }
      }
      if (!live) break;
      g += steps1;     // the rank-r weight tiles arrive by TMA
    }
    // the last stage releases (rank 0's MMA completions) have reached this CTA
    if (kPair && live) wait_ring_tail<SB>(b_empty, g, SB);
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();
  if (warp == 1) {
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, 512);
    else
      tmem_dealloc(tmem_base, 512);
  }
}

// ===========================================================================
// Few tokens (T <= 64): the products with the operands swapped, so that the
// weight side is the 128-row MMA operand and the tokens are the (16, 32 or
// 64 wide) N side:
//   forward   Y^T  = [W' | B ] [X | sU]^T      (M = d,  K = k (+ r))
//   dX        dX^T = [W'^T | A^T] [dY | sG]^T  (M = k,  K = d (+ r))
//   U         U^T  = A X^T                     (M = r,  K = k)
//   G         G^T  = B^T dY^T                  (M = r,  K = d)
// With few tokens the layer is bound by the weight stream (0.52 bytes per NF4
// weight), so the depth is split across CTAs to put every SM to work.  The
// splits of a row tile are one thread-block cluster: each CTA keeps its fp32
// partial in its own shared memory and, after a cluster barrier, every CTA
// sums a share of the tile over the ranks' shared memory in split order, so
// results are deterministic and nothing round-trips through global memory.
// Warps: 0 TMA, 1 TMEM + MMA, 2-9 dequantisation (NF4 sources: two threads
// per 64-weight block, half a block each, which halves the latency of a
// K-step's decode); warps 2-5 then read the accumulator, and all eight sum
// the depth splits.
// ===========================================================================
enum SmallSrc : int {
  SRC_NF4_ROWS = 0,   // W' rows (forward), K-major tiles dequantised in the kernel
  SRC_NF4_COLS = 1,   // W' columns (dX), MN-major tiles dequantised in the kernel
  SRC_TMA_K = 2,      // a bf16 matrix whose rows are M (A for U), K-major tiles by TMA
  SRC_TMA_MN = 3      // a bf16 matrix whose rows are K (B for G), MN-major tiles by TMA
};
enum SmallOut : int {
  OUT_BF16 = 0,       // b16[t][m] = bf16(v)                         (Y, dX)
  OUT_U = 1,          // f32[t][m] = v, b16[t][m] = bf16(scale v)    (U and s U)
  OUT_HILO = 2        // b16[t][m] = hi, b16[t][lo_off + m] = lo of scale v   (s G)
};

struct Nf4SmallArgs {
  int T;                      // tokens (MMA N side, at most TN)
  int Mw;                     // output features (rows of the accumulator)
  int K0, K1;                 // main depth and r (rank-r extension of the NF4 products)
  int tiles_m, splits;        // depth splits per row tile: K-steps split as evenly as possible
  float* f32_out;             // OUT_U
  int ldf, nf;
  uint16_t* b16_out;
  int ldb, nb;                // row stride and columns written
  int lo_off;                 // OUT_HILO
  float scale;                // OUT_U / OUT_HILO: bf16 output = bf16(scale v)
  float f32_scale;            // OUT_U: fp32 output = f32_scale v
  // NF4 sources: the double-quantised block constants, read by the
  // dequantising threads themselves (kb = 64-blocks per W' row)
  const uint8_t* absmax_q;
  const float* scale2;
  const float* mean;
  int kb;
  float levels[16];
};

constexpr int kSmDqWarps = 8;
constexpr int kSmThreads = (2 + kSmDqWarps) * 32;       // 320
// depth splits per row tile (one cluster): 8 is the portable cluster size;
// 16 where the device schedules non-portable clusters of that size
constexpr int kSmMaxSplits = 16;
constexpr int kSmSumBatch = 8;                           // partials in flight per step of the split sum

template <int TN>
struct SmallCfg {
  // The codes ring holds a whole split's codes (the tiny per-step MMA cannot
  // hide a load latency per step) while two CTAs still fit on an SM.
  static constexpr int SA = 3;                 // weight tiles, 128 x 64 bf16
  static constexpr int SC = TN >= 64 ? 6 : 8;  // codes, 4 KB per K-step
  static constexpr int SB = 4;                 // activation tiles, TN x 64 bf16
  static constexpr int kABytes = 16384;
  static constexpr int kCodeBytes = 4096;
  static constexpr int kCBytes = kCodeBytes;
  static constexpr int kBBytes = TN * 128;
  // mbarriers (full and empty of each ring, accumulator, drain) and three words
  static constexpr int kBarBytes = (2 * (SA + SB + SC) + 2) * 8 + 16;
  // 1024 of slack for aligning the rings to the 128-byte swizzle atom's 1 KB
  static constexpr int kSmem = SA * kABytes + SC * kCBytes + SB * kBBytes + 1024 + kBarBytes;
  static constexpr int kTmemCols = TN < 32 ? 32 : TN;
};

template <int kOut>
__device__ __forceinline__ void small_emit(const Nf4SmallArgs& p, int m, int t, float v) {
  if (kOut == OUT_BF16) {
    if (m < p.nb) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      p.b16_out[(int64_t)t * p.ldb + m] = *reinterpret_cast<const uint16_t*>(&h);
    }
  } else {
    if (kOut == OUT_U && m < p.nf) p.f32_out[(int64_t)t * p.ldf + m] = __fmul_rn(p.f32_scale, v);
    if (m < p.nb) {
      const float x = __fmul_rn(p.scale, v);
      const __nv_bfloat16 h = __float2bfloat16_rn(x);
      p.b16_out[(int64_t)t * p.ldb + m] = *reinterpret_cast<const uint16_t*>(&h);
      if (kOut == OUT_HILO) {
        const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
        p.b16_out[(int64_t)t * p.ldb + p.lo_off + m] = *reinterpret_cast<const uint16_t*>(&l);
      }
    }
  }
}

template <int kSrc, int kOut, int TN>
__global__ void __launch_bounds__(kSmThreads, 2)
    gemm_nf4_small_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmAct1,
                          const __grid_constant__ Nf4SmallArgs p) {
  using Cfg = SmallCfg<TN>;
  static_assert(Cfg::kSmem <= 232448, "shared memory per CTA");
  constexpr bool kNf4 = kSrc == SRC_NF4_ROWS || kSrc == SRC_NF4_COLS;
  constexpr bool kMnA = kSrc == SRC_NF4_COLS || kSrc == SRC_TMA_MN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sA = raw_addr + pad;                       // weight tiles
  const uint32_t sB = sA + Cfg::SA * Cfg::kABytes;          // activation tiles
  const uint32_t sC = sB + Cfg::SB * Cfg::kBBytes;          // codes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::SA * Cfg::kABytes + Cfg::SB * Cfg::kBBytes +
                                               Cfg::SC * Cfg::kCBytes);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + Cfg::SA;
  uint64_t* b_full = a_empty + Cfg::SA;
  uint64_t* b_empty = b_full + Cfg::SB;
  uint64_t* c_full = b_empty + Cfg::SB;
  uint64_t* c_empty = c_full + Cfg::SC;
  uint64_t* acc_full = c_empty + Cfg::SC;
  uint64_t* drain_bar = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits;
  const int split = blockIdx.x - tile * p.splits;
  const int m0 = tile * 128;
  const int steps0 = (p.K0 + 63) / 64;
  // split z takes steps0 / splits K-steps, the first steps0 % splits one more
  const int s_base = steps0 / p.splits, s_rem = steps0 - s_base * p.splits;
  const int s_begin = split * s_base + min(split, s_rem);
  const int nmain = s_base + (split < s_rem ? 1 : 0);
  const int steps1 = (kNf4 && split == 0) ? (p.K1 + 63) / 64 : 0;
  const int steps = nmain + steps1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cfg::SA; ++i) {
      mbar_init(smem_u32(&a_full[i]), kSmDqWarps);
      mbar_init(smem_u32(&a_empty[i]), 1);
    }
    for (int i = 0; i < Cfg::SB; ++i) {
      mbar_init(smem_u32(&b_full[i]), 1);
      mbar_init(smem_u32(&b_empty[i]), 1);
    }
    for (int i = 0; i < Cfg::SC; ++i) {
      mbar_init(smem_u32(&c_full[i]), 1);
      mbar_init(smem_u32(&c_empty[i]), kSmDqWarps);
    }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmW);
    if (steps1 > 0) {
      tma_prefetch_desc(&tmW1);
      tma_prefetch_desc(&tmAct1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The prologue above overlaps the previous kernel of the stream.
  griddep_launch_dependents();
  // codes run ahead of the activations by up to SC K-steps (issued by warp 0
  // in step order, each when the decode of the step SC before it is done)
  int c_iss[Cfg::SC];
  for (int i = 0; i < Cfg::SC; ++i) c_iss[i] = 0;
  int cnext = 0;
  auto issue_codes = [&](int upto) -> bool {
    for (; cnext < nmain && cnext < upto; ++cnext) {
      const int sc = cnext % Cfg::SC;
      if (!mbar_wait_bounded(smem_u32(&c_empty[sc]), (uint32_t)(((cnext / Cfg::SC) & 1) ^ 1), abort_flag))
        return false;
      const uint32_t fc = smem_u32(&c_full[sc]);
      const int ks = s_begin + cnext;
      mbar_arrive_expect_tx(fc, (uint32_t)Cfg::kCodeBytes);
      if (kSrc == SRC_NF4_COLS)
        tma_load_2d(sC + sc * Cfg::kCBytes, &tmW, fc, m0 / 2, ks * 64);
      else
        tma_load_2d(sC + sc * Cfg::kCBytes, &tmW, fc, ks * 32, m0);
      c_iss[sc] += 1;
    }
    return true;
  };
  // The first SC code stages, and the dequantising threads' first block
  // constants, load before waiting for that kernel: the NF4 codes and
  // constants are written only by the quantiser, whose kernels let no
  // dependent kernel start before they complete.  All other global memory
  // (activations, the rank-r operands, the outputs) is touched only after
  // the wait, which every thread executes.
  const bool pre_ok = !(kNf4 && warp == 0 && lane == 0) || issue_codes(Cfg::SC);
  if (!(kNf4 && warp >= 2)) griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int b_iss[Cfg::SB];
      int a_last[Cfg::SA];
      for (int i = 0; i < Cfg::SB; ++i) b_iss[i] = 0;
      for (int i = 0; i < Cfg::SA; ++i) a_last[i] = -1;
      bool ok = pre_ok;
      for (int step = 0; step < steps && ok; ++step) {
        const bool main = step < nmain;
        const int ks = s_begin + step;
        const int e = step - nmain;
        if (kNf4 && !issue_codes(step + Cfg::SC)) break;
        const int sb = step % Cfg::SB;
        if (!mbar_wait_bounded(smem_u32(&b_empty[sb]), (uint32_t)(((step / Cfg::SB) & 1) ^ 1), abort_flag)) break;
        const uint32_t fb = smem_u32(&b_full[sb]);
        mbar_arrive_expect_tx(fb, (uint32_t)Cfg::kBBytes);
        if (main)
          tma_load_2d(sB + sb * Cfg::kBBytes, &tmAct, fb, ks * 64, 0);
        else
          tma_load_2d(sB + sb * Cfg::kBBytes, &tmAct1, fb, e * 64, 0);
        b_iss[sb] += 1;
        if (!(main && kNf4)) {
          // a bf16 weight-side tile by TMA: the main operand of U / G, or the
          // rank-r operand (B rows / A columns) of the NF4 products
          const int sa = step % Cfg::SA;
          if (!mbar_wait_bounded(smem_u32(&a_empty[sa]), (uint32_t)(((step / Cfg::SA) & 1) ^ 1), abort_flag))
            break;
          const uint32_t fa = smem_u32(&a_full[sa]);
          mbar_arrive_expect_tx(fa, (uint32_t)Cfg::kABytes);
          mbar_arrive_count(fa, kSmDqWarps - 1);
          const CUtensorMap* mw = main ? &tmW : &tmW1;
          const int kx = main ? ks * 64 : e * 64;
          if (kMnA) {
            tma_load_2d(sA + sa * Cfg::kABytes, mw, fa, m0, kx);
            tma_load_2d(sA + sa * Cfg::kABytes + 8192, mw, fa, m0 + 64, kx);
          } else {
            tma_load_2d(sA + sa * Cfg::kABytes, mw, fa, kx, m0);
          }
          a_last[sa] = step / Cfg::SA;
        }
      }
      if (*abort_flag) {
        for (int i = 0; i < Cfg::SB; ++i)
          if (b_iss[i] > 0) mbar_wait_drain(smem_u32(&b_full[i]), (uint32_t)((b_iss[i] - 1) & 1));
        for (int i = 0; i < Cfg::SC; ++i)
          if (c_iss[i] > 0) mbar_wait_drain(smem_u32(&c_full[i]), (uint32_t)((c_iss[i] - 1) & 1));
        for (int i = 0; i < Cfg::SA; ++i)
          if (a_last[i] >= 0) mbar_wait_drain(smem_u32(&a_full[i]), (uint32_t)(a_last[i] & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t adesc = kMnA ? smem_desc_sw128(sA, 8192, 1024) : smem_desc_sw128(sA, 16, 1024);
      const uint32_t astep = kMnA ? 128u : 2u;
      const uint64_t bdesc = smem_desc_sw128(sB, 16, 1024);
      const uint32_t idesc = idesc_bf16_f32(128, TN, kMnA ? 1 : 0, 0);
      bool ok = true;
      int issued_any = 0;
      for (int step = 0; step < steps; ++step) {
        const int sa = step % Cfg::SA;
        const int sb = step % Cfg::SB;
        if (!mbar_wait_bounded(smem_u32(&a_full[sa]), (uint32_t)((step / Cfg::SA) & 1), abort_flag) ||
            !mbar_wait_bounded(smem_u32(&b_full[sb]), (uint32_t)((step / Cfg::SB) & 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool ext = step >= nmain;
        const int nsub = ext ? min(4, (p.K1 - (step - nmain) * 64 + 15) / 16) : 4;
        const uint64_t a0 = adesc + (uint64_t)((sa * Cfg::kABytes) >> 4);
        const uint64_t b0 = bdesc + (uint64_t)((sb * Cfg::kBBytes) >> 4);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nsub)
            umma_bf16(tmem_base, a0 + (uint64_t)(j * astep), b0 + (uint64_t)(2 * j), idesc,
                      (step == 0 && j == 0) ? 0u : 1u);
        issued_any = 1;
        umma_commit(smem_u32(&a_empty[sa]));
        umma_commit(smem_u32(&b_empty[sb]));
      }
      if (ok) {
        umma_commit(smem_u32(acc_full));
      } else if (issued_any) {
        umma_commit(smem_u32(drain_bar));
        mbar_wait_bounded(smem_u32(drain_bar), 0, nullptr);
      }
    }
  } else {
    bool live = true;
    if (kNf4) {
      // -------------------------------------------------------- dequantisation
      // Thread i owns one block per K-step.  Rows: tile row i (W' row m0 + i,
      // block column = the K-step).  Columns: K-row kk = i % 64 (W' row
      // 64 * ks + kk) and MN chunk cc = i / 64 (W' block column m0 / 64 + cc).
      // The thread reads its blocks' constants itself, kAhead K-steps ahead
      // (a register ring), and forms each block scale
      // a' = fl(fl(absmax * scale2) + mean) exactly as the dequantiser does;
      // blocks past the weight's edge get a' = 0.
      const int h = (threadIdx.x - 64) >> 7;           // which half of the block
      const int i = (threadIdx.x - 64) & 127;
      const int kk = i & 63, cc = i >> 6;
      const int Mrows = kSrc == SRC_NF4_COLS ? p.kb : p.Mw;   // forward: W' rows; dX: block columns
      const float mu = *p.mean;
      auto block_of = [&](int step, int64_t& b) -> bool {
        const int ks = s_begin + step;
        if (kSrc == SRC_NF4_COLS) {
          const int bc = (m0 >> 6) + cc;                 // block column
          const int wr = ks * 64 + kk;                   // W' row
          b = (int64_t)wr * p.kb + bc;
          return bc < Mrows && wr < p.K0;
        }
        b = (int64_t)(m0 + i) * p.kb + ks;
        return m0 + i < Mrows;
      };
      constexpr int kAhead = 4;
      constexpr uint32_t kOutside = 0x100u;          // not a code byte: the block lies outside W'
      uint32_t q_r[kAhead];
      float s2_r[kAhead];
      auto load_step = [&](int step, uint32_t& q, float& s2) {
        int64_t b = 0;
        const bool in = step < nmain && block_of(step, b);
        q = in ? (uint32_t)__ldg(p.absmax_q + b) : kOutside;
        s2 = in ? __ldg(p.scale2 + b / kBlock2) : 0.f;
      };
#pragma unroll
      for (int j = 0; j < kAhead; ++j) load_step(j, q_r[j], s2_r[j]);
      griddep_wait();
      for (int s0 = 0; s0 < nmain && live; s0 += kAhead) {
#pragma unroll
        for (int jw = 0; jw < kAhead; ++jw) {
          const int step = s0 + jw;
          if (step >= nmain) break;
          const int sc = step % Cfg::SC;
          bool ok = mbar_wait_bounded(smem_u32(&c_full[sc]), (uint32_t)((step / Cfg::SC) & 1), abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            live = false;
            break;
          }
          uint4 c;
          const uint32_t cs = sC + sc * Cfg::kCBytes;
          const float a =
              q_r[jw] != kOutside ? __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)q_r[jw]), s2_r[jw]), mu) : 0.f;
          load_step(step + kAhead, q_r[jw], s2_r[jw]);
          if (kSrc == SRC_NF4_COLS) {
            // 64-byte rows, 64B swizzle: chunk j at (j ^ ((row >> 1) & 3))
            const uint32_t row = cs + kk * 64;
            const int sw = (kk >> 1) & 3;
            c = ld_shared_v4(row + (((2 * cc + h) ^ sw) << 4));
          } else {
            const uint32_t row = cs + i * 32;
            const int sw = (i >> 2) & 1;
            c = ld_shared_v4(row + ((h ^ sw) << 4));
          }
          uint4 o[4];
          nf4_decode_half(c, a, p.levels, o);
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&c_empty[sc]));
          const int sa = step % Cfg::SA;
          ok = mbar_wait_bounded(smem_u32(&a_empty[sa]), (uint32_t)(((step / Cfg::SA) & 1) ^ 1), abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            live = false;
            break;
          }
          uint32_t dst;
          int sw;
          if (kSrc == SRC_NF4_COLS) {
            dst = sA + sa * Cfg::kABytes + cc * 8192 + kk * 128;
            sw = kk & 7;
          } else {
            dst = sA + sa * Cfg::kABytes + i * 128;
            sw = i & 7;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) st_shared_v4(dst + (((4 * h + j) ^ sw) << 4), o[j]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&a_full[sa]));
        }
      }
    }
    // ---------------------------------------------------------- epilogue
    // warps 2-5 read the accumulator: lane quarter q = warp & 3 holds rows
    // m0 + 32 q .. + 31.  One split: emit.  Several: the partial goes to
    // P[t][row] at the start of this CTA's shared memory (the weight ring,
    // whose readers, the MMAs, are done).
    const bool acc_warp = warp < 6;
    const int quarter = warp & 3;
    const int mloc = quarter * 32 + lane;
    const int m = m0 + mloc;
    bool ok = live && mbar_wait_bounded(smem_u32(acc_full), 0u, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && acc_warp) {
      tc_fence_after();
      fence_proxy_async_smem();
      float* P = reinterpret_cast<float*>(smem);
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int t0 = 0; t0 < TN; t0 += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)t0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = t0 + j;
          if (t < p.T) {
            if (p.splits == 1) {
              if (m < p.Mw) small_emit<kOut>(p, m, t, __uint_as_float(v[j]));
            } else {
              P[t * 128 + mloc] = __uint_as_float(v[j]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (p.splits > 1) {
    // The depth splits of a row tile form one cluster (rank = split): once
    // every partial is in its CTA's shared memory, the eight dequantising /
    // epilogue warps of every CTA sum a share of the tile's outputs over the
    // ranks' shared memory, in rank (= split) order, so the result does not
    // depend on timing.
    cluster_sync();
    if (warp >= 2) {
      const int z0 = (int)cluster_ctarank();
      const int tid = threadIdx.x - 64;
      const int nthr = kSmDqWarps * 32;
      if ((p.Mw & 3) == 0) {
        for (int it = z0 * nthr + tid; it < p.T * 32; it += p.splits * nthr) {
          const int t = it >> 5;
          const int q4 = (it & 31) * 4;
          const int mq = m0 + q4;
          if (mq >= p.Mw) continue;
          const uint32_t a = sA + (uint32_t)((t * 128 + q4) * 4);
          float4 acc = ld_shared_cluster_f4(mapa_shared(a, 0u));
          for (int z0 = 1; z0 < p.splits; z0 += kSmSumBatch) {
            float4 v[kSmSumBatch];
#pragma unroll
            for (int z = 0; z < kSmSumBatch; ++z)
              if (z0 + z < p.splits) v[z] = ld_shared_cluster_f4(mapa_shared(a, (uint32_t)(z0 + z)));
#pragma unroll
            for (int z = 0; z < kSmSumBatch; ++z) {
              if (z0 + z < p.splits) {
                acc.x = __fadd_rn(acc.x, v[z].x);
                acc.y = __fadd_rn(acc.y, v[z].y);
                acc.z = __fadd_rn(acc.z, v[z].z);
                acc.w = __fadd_rn(acc.w, v[z].w);
              }
            }
          }
          small_emit<kOut>(p, mq, t, acc.x);
          small_emit<kOut>(p, mq + 1, t, acc.y);
          small_emit<kOut>(p, mq + 2, t, acc.z);
          small_emit<kOut>(p, mq + 3, t, acc.w);
        }
      } else {
        for (int it = z0 * nthr + tid; it < p.T * 128; it += p.splits * nthr) {
          const int t = it >> 7;
          const int r0 = it & 127;
          const int mm = m0 + r0;
          if (mm >= p.Mw) continue;
          const uint32_t a = sA + (uint32_t)((t * 128 + r0) * 4);
          float acc = ld_shared_cluster_f32(mapa_shared(a, 0u));
          for (int z0 = 1; z0 < p.splits; z0 += kSmSumBatch) {
            float v[kSmSumBatch];
#pragma unroll
            for (int z = 0; z < kSmSumBatch; ++z)
              if (z0 + z < p.splits) v[z] = ld_shared_cluster_f32(mapa_shared(a, (uint32_t)(z0 + z)));
#pragma unroll
            for (int z = 0; z < kSmSumBatch; ++z)
              if (z0 + z < p.splits) acc = __fadd_rn(acc, v[z]);
          }
          small_emit<kOut>(p, mm, t, acc);
        }
      }
    }
    // no CTA leaves while a peer may still read its shared memory
    cluster_sync();
  }
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

}  // namespace qlora
