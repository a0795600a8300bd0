// Deploy-time merge and unmerge ([P1] deploy paragraph; [P2] "The LoRA
// hypothesis": W = W0 + (alpha/r) B A; a task is removed by subtracting its
// scaled product again):
//   merge   W    = bf16(fp32(w' + s (B A)_fp32)),  w' = doubleDequant(codes)
//   unmerge W0'' = bf16(fp32(W  - s (B A)_fp32))
//
// Both are HBM-bound (2.5 and 4 bytes per weight) with a small rank-r
// product per tile, so the kernel is built around moving bytes in bulk:
//   * a persistent CTA walks 128 x 256 tiles of W;
//   * warp 0 brings, by TMA, the tile's rank-r operands (B rows, A columns)
//     and the tile's input (the 16 KB of NF4 codes, or the 64 KB of W) in
//     128-byte-swizzled form, double-buffered;
//   * warp 1 computes (B A) for the tile with tcgen05 into one of two TMEM
//     accumulators;
//   * sixteen epilogue warps (2-17, four per TMEM lane quarter) each combine
//     accumulator and input for one 32-row x 64-column box of the tile (one
//     quantisation block wide), write the bf16 result into a swizzled 4 KB
//     shared box of their own (in place over W for unmerge) and store it with
//     TMA themselves (lines marked evict-first in L2), so the warps never
//     wait for one another.
// Rows or columns beyond d or k are zero-filled by the loads and clipped by
// the stores, so no element masks are needed.
#pragma once
#include "gemm_tc.cuh"
#include "nf4_kernels.cuh"
#include "ptx.cuh"

namespace qlora {

struct DeployArgs {
  int d, k, r;
  int tiles_m, tiles_n;
  float alpha;                 // +s for merge, -s for unmerge
  const uint8_t* absmax_q;
  const float* scale2;
  const float* mean;
  float levels[16];
};

template <bool kMerge, int KS>
struct DeployCfg {
  static constexpr int kOpA = KS * 16384;               // B rows: 128 x 64 bf16 per K-step
  static constexpr int kOpB = KS * 32768;               // A columns: 4 atoms of 64 x 64 bf16 per K-step
  static constexpr int kOpBytes = kOpA + kOpB;
  // the operands of the next tile load while this tile's MMA runs (two
  // buffers); with two K-steps only one fits beside the input tiles
  static constexpr int kOpBufs = KS == 1 ? 2 : 1;
  static constexpr int kIo = kMerge ? 16384 : 65536;    // codes tile (128 x 128 B) or W tile
  // merge: one 32 x 64 bf16 staging box per epilogue warp (unmerge: in
  // place), and per warp a 16 x 32 table of the block's dequantised levels
  // (the per-warp level tables of merge are a static shared array)
  static constexpr int kOut = kMerge ? 16 * 4096 : 0;
  static constexpr int kBytes = kOpBufs * kOpBytes + 2 * kIo + kOut;
  static constexpr int kSmemBytes = kBytes + 1024 + 512;
};

// Warps: 0 producer, 1 MMA, 2-17 epilogue (four per TMEM lane quarter, each
// taking one 64-column box of the tile's 256 columns).
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kDeployThreads = 64 + kEpiThreads;

// L2 policy marking lines for early eviction: the output is written once and
// not read again here, so it should not displace other lines.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 2-D tiled TMA store from this CTA's shared memory with an L2 cache policy.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y,
                                                  uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "l"(pol)
      : "memory");
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-row,
// 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Eight merged weights from one 32-bit word of codes (element 2j in the low
// nibble of byte j) and their eight accumulator values, as one block of PTX:
//   code -> this lane's level table column (lut + code * 128) -> w',
//   W = bf16(fp32(w' + alpha * acc)), packed in pairs.
__device__ __forceinline__ uint4 merge8(uint32_t codes, const uint32_t* acc, float alpha, uint32_t lut) {
  uint4 o;
  asm("{\n\t"
      ".reg .b32 lo, hi, c<8>, a<8>;\n\t"
      ".reg .f32 w<8>, v<8>;\n\t"
      "and.b32 lo, %4, 0x0F0F0F0F;\n\t"
      "shr.b32 hi, %4, 4;\n\t"
      "and.b32 hi, hi, 0x0F0F0F0F;\n\t"
      "prmt.b32 c0, lo, 0, 17472;\n\t"
      "prmt.b32 c1, hi, 0, 17472;\n\t"
      "prmt.b32 c2, lo, 0, 17473;\n\t"
      "prmt.b32 c3, hi, 0, 17473;\n\t"
      "prmt.b32 c4, lo, 0, 17474;\n\t"
      "prmt.b32 c5, hi, 0, 17474;\n\t"
      "prmt.b32 c6, lo, 0, 17475;\n\t"
      "prmt.b32 c7, hi, 0, 17475;\n\t"
      "mad.lo.u32 a0, c0, 128, %14;\n\t"
      "mad.lo.u32 a1, c1, 128, %14;\n\t"
      "mad.lo.u32 a2, c2, 128, %14;\n\t"
      "mad.lo.u32 a3, c3, 128, %14;\n\t"
      "mad.lo.u32 a4, c4, 128, %14;\n\t"
      "mad.lo.u32 a5, c5, 128, %14;\n\t"
      "mad.lo.u32 a6, c6, 128, %14;\n\t"
      "mad.lo.u32 a7, c7, 128, %14;\n\t"
      "ld.shared.f32 w0, [a0];\n\t"
      "ld.shared.f32 w1, [a1];\n\t"
      "ld.shared.f32 w2, [a2];\n\t"
      "ld.shared.f32 w3, [a3];\n\t"
      "ld.shared.f32 w4, [a4];\n\t"
      "ld.shared.f32 w5, [a5];\n\t"
      "ld.shared.f32 w6, [a6];\n\t"
      "ld.shared.f32 w7, [a7];\n\t"
      "fma.rn.f32 v0, %13, %5, w0;\n\t"
      "fma.rn.f32 v1, %13, %6, w1;\n\t"
      "fma.rn.f32 v2, %13, %7, w2;\n\t"
      "fma.rn.f32 v3, %13, %8, w3;\n\t"
      "fma.rn.f32 v4, %13, %9, w4;\n\t"
      "fma.rn.f32 v5, %13, %10, w5;\n\t"
      "fma.rn.f32 v6, %13, %11, w6;\n\t"
      "fma.rn.f32 v7, %13, %12, w7;\n\t"
      "cvt.rn.bf16x2.f32 %0, v1, v0;\n\t"
      "cvt.rn.bf16x2.f32 %1, v3, v2;\n\t"
      "cvt.rn.bf16x2.f32 %2, v5, v4;\n\t"
      "cvt.rn.bf16x2.f32 %3, v7, v6;\n\t"
      "}"
      : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
      : "r"(codes), "f"(__uint_as_float(acc[0])), "f"(__uint_as_float(acc[1])), "f"(__uint_as_float(acc[2])),
        "f"(__uint_as_float(acc[3])), "f"(__uint_as_float(acc[4])), "f"(__uint_as_float(acc[5])),
        "f"(__uint_as_float(acc[6])), "f"(__uint_as_float(acc[7])), "f"(alpha), "r"(lut));
  return o;
}

template <bool kMerge, int KS>
__global__ void __launch_bounds__(kDeployThreads, 1)
    lora_deploy_kernel(const __grid_constant__ CUtensorMap tmOpA, const __grid_constant__ CUtensorMap tmOpB,
                       const __grid_constant__ CUtensorMap tmIo, const __grid_constant__ CUtensorMap tmOut,
                       const __grid_constant__ DeployArgs p) {
  using Cfg = DeployCfg<kMerge, KS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  const uint32_t sOp = sbase;                           // kOpBufs x {A part, B part}
  const uint32_t sIo = sOp + Cfg::kOpBufs * Cfg::kOpBytes;
  const uint32_t sOut = sIo + 2 * Cfg::kIo;
  uint8_t* gIo = smem + Cfg::kOpBufs * Cfg::kOpBytes;
  uint8_t* gOut = gIo + 2 * Cfg::kIo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBytes);
  uint64_t* op_full = bars + 0;      // [2]
  uint64_t* op_empty = bars + 2;     // [2]
  uint64_t* io_full = bars + 4;      // [2]
  uint64_t* io_empty = bars + 6;     // [2]
  uint64_t* acc_full = bars + 8;     // [2]
  uint64_t* acc_empty = bars + 10;   // [2]
  uint64_t* drain_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // static, so that table reads are a register plus a constant offset
  __shared__ float s_lut[16];
  // merge: s_wlut[warp][c][lane] = float(bf16(level[c] * a')) for the block of
  // that lane's row, so a code costs one conflict-free shared load
  __shared__ float s_wlut[kMerge ? kEpiWarps : 1][16][32];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&op_full[i]), 1);
      mbar_init(smem_u32(&op_empty[i]), 1);
      mbar_init(smem_u32(&io_full[i]), 1);
      mbar_init(smem_u32(&io_empty[i]), kEpiWarps);
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), kEpiWarps);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) s_lut[threadIdx.x] = p.levels[threadIdx.x];
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmOpA);
    tma_prefetch_desc(&tmOpB);
    tma_prefetch_desc(&tmIo);
    tma_prefetch_desc(&tmOut);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      int io_issued[2] = {0, 0};
      int op_issued[2] = {0, 0};
      for (int u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        const int m0 = (u / p.tiles_n) * 128;
        const int n0 = (u % p.tiles_n) * 256;
        const int s = it & 1;
        // rank-r operands, freed by the MMA commit of the tile that used them
        const int ob = it % Cfg::kOpBufs;
        const int oq = it / Cfg::kOpBufs;
        if (!mbar_wait_bounded(smem_u32(&op_empty[ob]), (uint32_t)((oq & 1) ^ 1), abort_flag)) break;
        const uint32_t fo = smem_u32(&op_full[ob]);
        const uint32_t sA = sOp + ob * Cfg::kOpBytes;
        const uint32_t sB = sA + Cfg::kOpA;
        mbar_arrive_expect_tx(fo, (uint32_t)Cfg::kOpBytes);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          tma_load_2d(sA + ks * 16384, &tmOpA, fo, ks * 64, m0);
#pragma unroll
          for (int i = 0; i < 4; ++i) tma_load_2d(sB + ks * 32768 + i * 8192, &tmOpB, fo, n0 + 64 * i, ks * 64);
        }
        op_issued[ob] = oq + 1;
        // input tile (double buffer, freed by the epilogue)
        if (!mbar_wait_bounded(smem_u32(&io_empty[s]), (uint32_t)(((it >> 1) & 1) ^ 1), abort_flag)) break;
        const uint32_t fi = smem_u32(&io_full[s]);
        mbar_arrive_expect_tx(fi, (uint32_t)Cfg::kIo);
        if (kMerge) {
          tma_load_2d(sIo + s * Cfg::kIo, &tmIo, fi, n0 / 2, m0);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) tma_load_2d(sIo + s * Cfg::kIo + i * 16384, &tmIo, fi, n0 + 64 * i, m0);
        }
        io_issued[s] = it + 1;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        for (int b = 0; b < 2; ++b) {
          if (op_issued[b] > 0)
            mbar_wait_bounded(smem_u32(&op_full[b]), (uint32_t)((op_issued[b] - 1) & 1), nullptr);
          if (io_issued[b] > 0)
            mbar_wait_bounded(smem_u32(&io_full[b]), (uint32_t)(((io_issued[b] - 1) >> 1) & 1), nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 256, 0, 1);
      bool ok = true;
      int issued_any = 0;
      int it = 0;
      for (int u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        const int s = it & 1;
        const int ob = it % Cfg::kOpBufs;
        const int oq = it / Cfg::kOpBufs;
        if (!mbar_wait_bounded(smem_u32(&acc_empty[s]), (uint32_t)(((it >> 1) & 1) ^ 1), abort_flag)) { ok = false; break; }
        if (!mbar_wait_bounded(smem_u32(&op_full[ob]), (uint32_t)(oq & 1), abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sA = sOp + ob * Cfg::kOpBytes;
        const uint64_t da = smem_desc_sw128(sA, 16, 1024);
        const uint64_t db = smem_desc_sw128(sA + Cfg::kOpA, 8192, 1024);
        const uint32_t d_tmem = tmem_base + (uint32_t)(s * 256);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int nsub = min(4, (p.r - ks * 64 + 15) / 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nsub) {
              umma_bf16(d_tmem, da + (uint64_t)((ks * 16384 + j * 32) >> 4), db + (uint64_t)((ks * 32768 + j * 2048) >> 4),
                        idesc, (ks > 0 || j > 0) ? 1u : 0u);
              issued_any = 1;
            }
          }
        }
        umma_commit(smem_u32(&op_empty[ob]));
        umma_commit(smem_u32(&acc_full[s]));
      }
      if (!ok && issued_any) {
        umma_commit(smem_u32(drain_bar));
        mbar_wait_bounded(smem_u32(drain_bar), 0, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Every warp works alone on one 32-row x 64-column box of the tile (the
    // box is one quantisation block wide) and stores it with TMA from its
    // lane 0, so no barrier spans the epilogue warps.  Merge stages the box
    // in a 4 KB buffer of the warp's own; unmerge writes in place over its
    // part of the W tile.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int bxi = ew >> 2;                      // box 0..3: columns 64 bxi .. 64 bxi + 63
    const int cA = 2 * bxi;                       // its two 32-column chunks: cA, cA + 1
    const int row = quarter * 32 + lane;
    const int kb = p.k / kBlock;                  // blocks per row of W
    const float mu = kMerge ? p.mean[0] : 0.f;
    const uint32_t lut_lane = smem_u32(&s_wlut[kMerge ? ew : 0][0][lane]);
    uint8_t* stg = gOut + ew * 4096;
    const uint64_t out_policy = l2_policy_evict_first();
    const uint32_t stg_s = sOut + (uint32_t)ew * 4096u;
    // raw scale inputs of this thread's block, loaded one tile ahead so their
    // latency hides behind a whole tile of work
    uint32_t nq = 0u;
    float ns2 = 0.f;
    auto fetch_scale = [&](int uu) {
      if (!kMerge || uu >= units) return;
      const int m = (uu / p.tiles_n) * 128 + row;
      const int n = (uu % p.tiles_n) * 256 + 64 * bxi;
      if (m < p.d && n < p.k) {
        const int64_t b = (int64_t)m * kb + n / 64;
        nq = p.absmax_q[b];
        ns2 = p.scale2[b / kBlock2];
      }
    };
    fetch_scale(blockIdx.x);
    int it = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++it) {
      const int m0 = (u / p.tiles_n) * 128;
      const int n0 = (u % p.tiles_n) * 256;
      const int s = it & 1;
      if (kMerge) {
        // this lane's column of the table (only this lane reads it)
        const float a = __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)nq), ns2), mu);
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const uint32_t pr = pack_bf16x2(__fmul_rn(s_lut[c], a), __fmul_rn(s_lut[c + 1], a));
          s_wlut[kMerge ? ew : 0][c][lane] = bf16_bits_to_f32(pr & 0xFFFFu);
          s_wlut[kMerge ? ew : 0][c + 1][lane] = bf16_bits_to_f32(pr >> 16);
        }
      }
      fetch_scale(u + gridDim.x);
      bool ok = mbar_wait_bounded(smem_u32(&io_full[s]), (uint32_t)((it >> 1) & 1), abort_flag);
      ok = ok && mbar_wait_bounded(smem_u32(&acc_full[s]), (uint32_t)((it >> 1) & 1), abort_flag);
      // the lanes leave together (the TMEM loads below are warp-collective)
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(s * 256);
      // merge: the store that last read this warp's staging box is done
      if (kMerge && it > 0 && lane == 0) bulk_wait_group_read0();
      __syncwarp();
      uint8_t* io = gIo + s * Cfg::kIo;
      // output rows of the box: merge -> staging (32 rows of 128 B); unmerge
      // -> in place, rows quarter*32.. of the W box bxi
      uint8_t* obox = kMerge ? stg : io + bxi * 16384 + quarter * 4096;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // one 32-column chunk per TMEM round trip keeps the register count low
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + (uint32_t)((cA + h) * 32), v);
        tmem_ld_wait();
        if (h == 1) {
          // accumulator drained
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&acc_empty[s]));
        }
        float wf[32];                         // the 32 inputs w' (merge) or W (unmerge) as fp32
        if (kMerge) {
          const uint4 cw = *reinterpret_cast<const uint4*>(io + sw128(row, cA + h));
          const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(obox + sw128(lane, h * 4 + q)) = merge8(words[q], v + 8 * q, p.alpha, lut_lane);
          continue;
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 x = *reinterpret_cast<const uint4*>(obox + sw128(lane, h * 4 + q));
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              wf[8 * q + 2 * j] = bf16_bits_to_f32(xs[j] & 0xFFFFu);
              wf[8 * q + 2 * j + 1] = bf16_bits_to_f32(xs[j] >> 16);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t r4[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float lo = __fmaf_rn(p.alpha, __uint_as_float(v[8 * q + 2 * j]), wf[8 * q + 2 * j]);
            const float hi = __fmaf_rn(p.alpha, __uint_as_float(v[8 * q + 2 * j + 1]), wf[8 * q + 2 * j + 1]);
            r4[j] = pack_bf16x2(lo, hi);
          }
          *reinterpret_cast<uint4*>(obox + sw128(lane, h * 4 + q)) = make_uint4(r4[0], r4[1], r4[2], r4[3]);
        }
      }
      // the box is written: lane 0 stores it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t src = kMerge ? stg_s : sIo + (uint32_t)(s * Cfg::kIo + bxi * 16384 + quarter * 4096);
        tma_store_2d_hint(&tmOut, src, n0 + 64 * bxi, m0 + quarter * 32, out_policy);
        bulk_commit_group();
        // input tile released: merge once the codes are read (they were, by
        // the __syncwarp above); unmerge once the store has read it
        if (!kMerge) bulk_wait_group_read0();
        mbar_arrive(smem_u32(&io_empty[s]));
      }
    }
    if (lane == 0) bulk_wait_group0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

}  // namespace qlora
