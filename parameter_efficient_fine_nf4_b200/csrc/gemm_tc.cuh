// Tensor-core GEMM engine for sm_100a (tcgen05 + TMEM + TMA).
//
//   C[M x N] (fp32, TMEM) = sum over K-steps of  A_tile * B_tile^T
//
// over two K segments: the main product (K0) followed by an optional
// extension (K1 = r) whose operands are the rank-r factors.  This is how the
// LoRA term joins the base product in one accumulator:
//   Y  = [X | sU] [W' | B]^T      (forward, [P1] forward equation)
//   dX = [dY | sG] [W' ; A]       (backward)
// Each operand of each segment is K-major or MN-major in global memory; TMA
// moves 64-wide (128-byte, 128B-swizzled) boxes into shared memory, so the
// same tile serves as a K-major or MN-major UMMA operand by descriptor alone.
//
// Roles (192 threads): warp 0 issues TMA, warp 1 owns TMEM and issues UMMA
// (one thread), warps 2-5 drain TMEM in the epilogue.  A STAGES-deep ring of
// full/empty mbarriers couples producer and MMA; tcgen05.commit frees a stage
// when the MMAs reading it finish.  All waits are bounded (see ptx.cuh).
#pragma once
#include "ptx.cuh"
#include "nf4_kernels.cuh"

namespace qlora {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 192;

enum EpiKind : int {
  EPI_BF16 = 0,      // out bf16 [M][ldo] = acc
  EPI_F32 = 1,       // out fp32 [M][ldo] = alpha*acc ; out2 bf16 = alpha2*acc
  EPI_F32_T = 2,     // out fp32 [N][ldo] = alpha*acc (transposed store)
  EPI_MERGE = 3,     // out bf16 = bf16(alpha*acc + dequant(codes))
  EPI_UNMERGE = 4,   // out bf16 = bf16(alpha*acc + w_in)
  EPI_DROPOUT = 5    // out bf16 = bf16(out + keep * alpha*acc), in place (the masked rank-r term of dX)
};

struct GemmArgs {
  int M, N;
  int K0, K1;
  int a0_mn, b0_mn, a1_mn, b1_mn;
  int k_per_split;            // K0 columns per blockIdx.y (multiple of 64)
  int tiles_m, tiles_n, group_m;
  int epi;
  void* out;
  int64_t ldo;
  int64_t split_stride;       // elements between split-K partial outputs
  float alpha;
  int n_store;
  uint16_t* out2;
  int64_t ldo2;
  float alpha2;
  int n_store2;
  int lo_offset;              // > 0: out2 also gets lo = bf16(v - bf16(v)) at this column offset
  int pair_offset;            // > 0: the result is acc[j] + acc[j + pair_offset] (hi/lo operand pair)
  int tma_store;              // EPI_BF16 through shared staging and TMA stores (tmOut)
  const uint8_t* codes;
  const uint8_t* absmax_q;
  const float* scale2;
  const float* mean;
  const uint16_t* w_in;
  int64_t ldw;
  const uint8_t* keep;        // EPI_DROPOUT: bit (m * ldk + n) of this array keeps element (m, n)
  int64_t ldk;
  float levels[16];
};

// One stage holds KSUB sub-blocks of 64 K-columns of each operand, laid out
// [A sub 0 | A sub 1 | ... | B sub 0 | B sub 1 | ...], each sub-block the same
// 128B-swizzled tile a one-sub-block stage would hold.  A wider stage requests
// several consecutive K-blocks of the same rows at once (512 contiguous bytes
// of each activation row with 4 sub-blocks), which streams the HBM-bound
// adapter products 13-15 % faster than one K-block per stage.
template <int BN, int KSUB = 1>
struct GemmCfg {
  static constexpr int kSubA = kBM * kBK * 2;                    // 16 KB
  static constexpr int kSubB = BN * kBK * 2;
  static constexpr int kABytes = KSUB * kSubA;
  static constexpr int kBBytes = KSUB * kSubB;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages =
      KSUB == 1 ? ((BN >= 256) ? 4 : (BN >= 128 ? 5 : 6)) : (200 * 1024) / kStageBytes;
  static constexpr int kTmemCols = 2 * BN;                       // two accumulators
  // bf16 output staging for TMA stores: 2 boxes of 32 x 64 per epilogue warp
  static constexpr int kStoreStage = (BN == 256) ? 4 * 2 * 4096 : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kStoreStage + 1024 /*align*/ + 512 /*bars*/;
  static_assert(kStages >= 2, "a stage ring needs two stages");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Work unit u -> (tile row, tile column, K split), tiles rasterised in groups
// of `group_m` tile rows so that concurrently running CTAs share A and B tiles
// in L2.
struct Unit {
  int m0, n0, split;
};
__device__ __forceinline__ Unit unit_coords(const GemmArgs& p, int u, int bn) {
  const int tiles = p.tiles_m * p.tiles_n;
  Unit r;
  r.split = u / tiles;
  const int t = u - r.split * tiles;
  const int per_group = p.group_m * p.tiles_n;
  const int gidx = t / per_group;
  const int first_m = gidx * p.group_m;
  const int gsize = min(p.group_m, p.tiles_m - first_m);
  const int in_group = t - gidx * per_group;
  r.m0 = (first_m + in_group % gsize) * kBM;
  r.n0 = (in_group / gsize) * bn;
  return r;
}

// Store one 32-column chunk of one accumulator row (row m, columns n..n+31).
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& p, uint32_t (&v)[32], int m, int n,
                                               int split, const float* s_lut) {
  if (p.epi == EPI_BF16) {
    uint16_t* out = reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n;
    if (n + 32 <= p.n_store && (p.ldo & 7) == 0) {
      uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
        w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
        w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
        w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
        o4[i] = w;
      }
    } else {
      for (int i = 0; i < 32 && n + i < p.n_store; ++i) {
        __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
        out[i] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  } else if (p.epi == EPI_F32) {
    if (p.out != nullptr) {
      float* out = reinterpret_cast<float*>(p.out) + (int64_t)split * p.split_stride + (int64_t)m * p.ldo + n;
      if (n + 32 <= p.n_store && (p.ldo & 3) == 0) {
        float4* o4 = reinterpret_cast<float4*>(out);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o4[i] = make_float4(p.alpha * __uint_as_float(v[4 * i]), p.alpha * __uint_as_float(v[4 * i + 1]),
                              p.alpha * __uint_as_float(v[4 * i + 2]), p.alpha * __uint_as_float(v[4 * i + 3]));
      } else {
        for (int i = 0; i < 32 && n + i < p.n_store; ++i) out[i] = p.alpha * __uint_as_float(v[i]);
      }
    }
    if (p.out2 != nullptr) {
      uint16_t* o2 = p.out2 + (int64_t)m * p.ldo2 + n;
      for (int i = 0; i < 32 && n + i < p.n_store2; ++i) {
        const float x = __fmul_rn(p.alpha2, __uint_as_float(v[i]));
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        o2[i] = *reinterpret_cast<const uint16_t*>(&h);
        if (p.lo_offset > 0) {
          const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
          o2[i + p.lo_offset] = *reinterpret_cast<const uint16_t*>(&l);
        }
      }
    }
  } else if (p.epi == EPI_F32_T) {
    float* out = reinterpret_cast<float*>(p.out) + (int64_t)split * p.split_stride + m;
    for (int i = 0; i < 32 && n + i < p.n_store; ++i) out[(int64_t)(n + i) * p.ldo] = p.alpha * __uint_as_float(v[i]);
  } else if (p.epi == EPI_MERGE) {
    // w' for row m, columns n..n+31: one 16-byte word of codes, one block
    const int64_t e0 = (int64_t)m * p.N + n;
    const uint4 cw = *reinterpret_cast<const uint4*>(p.codes + e0 / 2);
    const float a_scale = block_scale(p.absmax_q, p.scale2, p.mean[0], e0 / kBlock);
    uint32_t wq[16];
    dequant32(cw, a_scale, s_lut, wq);
    uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t r4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t wp = wq[4 * i + j];
        const float lo = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j]), bf16_bits_to_f32(wp & 0xFFFFu));
        const float hi = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j + 1]), bf16_bits_to_f32(wp >> 16));
        r4[j] = pack_bf16x2(lo, hi);
      }
      o4[i] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
    }
  } else if (p.epi == EPI_DROPOUT) {
    // 32 keep bits of row m, columns n..n+31 (n is a multiple of 32 and ldk of
    // 32, so the word is aligned); bit i keeps column n + i
    uint16_t* out = reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n;
    const uint32_t bits = *reinterpret_cast<const uint32_t*>(p.keep + ((int64_t)m * p.ldk + n) / 8);
    for (int i = 0; i < 32 && n + i < p.n_store; ++i) {
      const float base = bf16_bits_to_f32(out[i]);
      const float add = ((bits >> i) & 1u) ? __fmul_rn(p.alpha, __uint_as_float(v[i])) : 0.f;
      const __nv_bfloat16 h = __float2bfloat16_rn(__fadd_rn(base, add));
      out[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
  } else if (p.epi == EPI_UNMERGE) {
    const uint4* w4 = reinterpret_cast<const uint4*>(p.w_in + (int64_t)m * p.ldw + n);
    uint4 wv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) wv[i] = w4[i];
    uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t wr[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
      uint32_t r4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j]), bf16_bits_to_f32(wr[j] & 0xFFFFu));
        const float hi = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j + 1]), bf16_bits_to_f32(wr[j] >> 16));
        r4[j] = pack_bf16x2(lo, hi);
      }
      o4[i] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
    }
  }
}

// Merge / unmerge epilogue of one accumulator row: these kernels are bound by
// the epilogue's global traffic (one K-step of MMA per tile), so the loads of
// the codes (merge) or of W (unmerge) are issued ahead of the TMEM reads that
// consume them: all of a row's code words at once, W one chunk ahead.
template <int BN>
__device__ __forceinline__ void epilogue_merge_row(const GemmArgs& p, uint32_t taddr, int m, bool row_ok,
                                                   int n0, const float* s_lut) {
  constexpr int NC = BN / 32;
  if (p.epi == EPI_MERGE) {
    uint4 cw[NC];
    float asc[NC];
    const float mu = p.mean[0];
#pragma unroll
    for (int ch = 0; ch < NC; ++ch) {
      const int n = n0 + ch * 32;
      cw[ch] = make_uint4(0u, 0u, 0u, 0u);
      asc[ch] = 0.f;
      if (row_ok && n < p.N) {
        const int64_t e0 = (int64_t)m * p.N + n;
        cw[ch] = __ldg(reinterpret_cast<const uint4*>(p.codes + e0 / 2));
        asc[ch] = block_scale(p.absmax_q, p.scale2, mu, e0 / kBlock);
      }
    }
#pragma unroll
    for (int ch = 0; ch < NC; ++ch) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32), v);
      tmem_ld_wait();
      const int n = n0 + ch * 32;
      if (!row_ok || n >= p.N) continue;
      uint32_t wq[16];
      dequant32(cw[ch], asc[ch], s_lut, wq);
      uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t r4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t wp = wq[4 * i + j];
          const float lo = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j]), bf16_bits_to_f32(wp & 0xFFFFu));
          const float hi = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j + 1]), bf16_bits_to_f32(wp >> 16));
          r4[j] = pack_bf16x2(lo, hi);
        }
        o4[i] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
      }
    }
  } else {
    uint4 wv[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) wv[0][i] = make_uint4(0u, 0u, 0u, 0u);
    if (row_ok && n0 < p.N) {
      const uint4* w4 = reinterpret_cast<const uint4*>(p.w_in + (int64_t)m * p.ldw + n0);
#pragma unroll
      for (int i = 0; i < 4; ++i) wv[0][i] = __ldg(w4 + i);
    }
#pragma unroll
    for (int ch = 0; ch < NC; ++ch) {
      const int n = n0 + ch * 32;
      if (ch + 1 < NC) {
        const int nn = n + 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) wv[(ch + 1) & 1][i] = make_uint4(0u, 0u, 0u, 0u);
        if (row_ok && nn < p.N) {
          const uint4* w4 = reinterpret_cast<const uint4*>(p.w_in + (int64_t)m * p.ldw + nn);
#pragma unroll
          for (int i = 0; i < 4; ++i) wv[(ch + 1) & 1][i] = __ldg(w4 + i);
        }
      }
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32), v);
      tmem_ld_wait();
      if (!row_ok || n >= p.N) continue;
      uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + (int64_t)m * p.ldo + n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = wv[ch & 1][i];
        const uint32_t wr[4] = {w.x, w.y, w.z, w.w};
        uint32_t r4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j]), bf16_bits_to_f32(wr[j] & 0xFFFFu));
          const float hi = __fmaf_rn(p.alpha, __uint_as_float(v[8 * i + 2 * j + 1]), bf16_bits_to_f32(wr[j] >> 16));
          r4[j] = pack_bf16x2(lo, hi);
        }
        o4[i] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
      }
    }
  }
}

// Shared-memory descriptors of stage 0 for both segments; a stage or a K
// sub-step only adds a byte offset / 16 to the start-address field (the
// field never carries: shared addresses stay below 2^18).  K-major: 16
// elements = 32 bytes along the swizzled row; MN-major: 16 K-rows of 128 B.
struct StageDescs {
  uint64_t a[2], b[2];
  uint32_t astep[2], bstep[2];
  uint32_t idesc[2];
};
__device__ __forceinline__ StageDescs make_stage_descs(const GemmArgs& p, uint32_t sa0, uint32_t sb0, int M, int N) {
  StageDescs d;
  const int amn[2] = {p.a0_mn, p.a1_mn};
  const int bmn[2] = {p.b0_mn, p.b1_mn};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    d.a[s] = amn[s] ? smem_desc_sw128(sa0, 8192, 1024) : smem_desc_sw128(sa0, 16, 1024);
    d.b[s] = bmn[s] ? smem_desc_sw128(sb0, 8192, 1024) : smem_desc_sw128(sb0, 16, 1024);
    d.astep[s] = amn[s] ? 128u : 2u;
    d.bstep[s] = bmn[s] ? 128u : 2u;
    d.idesc[s] = idesc_bf16_f32(M, N, amn[s], bmn[s]);
  }
  return d;
}

__device__ __forceinline__ void issue_kstep(uint32_t d_tmem, const StageDescs& d, int seg, uint32_t a_off16,
                                            uint32_t b_off16, int nsub, bool first) {
  const uint64_t a = d.a[seg] + a_off16;
  const uint64_t b = d.b[seg] + b_off16;
  const uint32_t as = d.astep[seg], bs = d.bstep[seg], id = d.idesc[seg];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (j < nsub) {
      const uint32_t acc = (first && j == 0) ? 0u : 1u;
      umma_bf16(d_tmem, a + (uint64_t)(j * as), b + (uint64_t)(j * bs), id, acc);
    }
  }
}

// Persistent kernel: CTA b processes work units b, b + gridDim.x, ...  The
// shared-memory ring runs continuously across units; two TMEM accumulators
// (columns [0, BN) and [BN, 2 BN)) let the epilogue of one unit overlap the
// mainloop of the next (acc_full / acc_empty barriers per accumulator).
template <int BN, int KSUB>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ GemmArgs p) {
  using Cfg = GemmCfg<BN, KSUB>;
  constexpr int S = Cfg::kStages;
  constexpr int kStepK = kBK * KSUB;      // K columns per stage
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzle atoms
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  uint8_t* ctrl = smem + S * Cfg::kStageBytes + Cfg::kStoreStage;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* acc_full = empty_bar + S;       // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_lut = reinterpret_cast<float*>(tmem_slot + 4);        // 16 floats

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n * (int)((p.K0 + p.k_per_split - 1) / p.k_per_split);
  const int steps1 = (p.K1 + kStepK - 1) / kStepK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), 4);    // one arrive per epilogue warp
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) s_lut[threadIdx.x] = p.levels[threadIdx.x];
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (steps1 > 0) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[S];
#pragma unroll
      for (int i = 0; i < S; ++i) issued[i] = 0;
      int g = 0;                                     // global step counter (ring position)
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const Unit c = unit_coords(p, u, BN);
        const int k_begin = c.split * p.k_per_split;
        const int k_end0 = min(p.K0, k_begin + p.k_per_split);
        const int steps0 = (k_end0 - k_begin + kStepK - 1) / kStepK;
        const int steps = steps0 + (c.split == 0 ? steps1 : 0);
        bool ok = true;
        for (int step = 0; step < steps; ++step, ++g) {
          const int st = g % S;
          const uint32_t ph = (uint32_t)((g / S) & 1);
          if (!mbar_wait_bounded(smem_u32(&empty_bar[st]), ph ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full_bar[st]);
          const bool ext = step >= steps0;
          const int kk = ext ? (step - steps0) * kStepK : k_begin + step * kStepK;
          const int nk = min(KSUB, ((ext ? p.K1 : k_end0) - kk + kBK - 1) / kBK);   // sub-blocks in range
          mbar_arrive_expect_tx(fb, (uint32_t)(nk * (Cfg::kSubA + Cfg::kSubB)));
          const uint32_t sa0 = sbase + st * Cfg::kStageBytes;
          const CUtensorMap* ma = ext ? &tmA1 : &tmA0;
          const CUtensorMap* mb = ext ? &tmB1 : &tmB0;
          const int a_mn = ext ? p.a1_mn : p.a0_mn;
          const int b_mn = ext ? p.b1_mn : p.b0_mn;
          for (int j = 0; j < nk; ++j) {
            const uint32_t sa = sa0 + j * Cfg::kSubA;
            const uint32_t sb = sa0 + Cfg::kABytes + j * Cfg::kSubB;
            const int kj = kk + j * kBK;
            if (a_mn) {
              tma_load_2d(sa, ma, fb, c.m0, kj);
              tma_load_2d(sa + 8192, ma, fb, c.m0 + 64, kj);
            } else {
              tma_load_2d(sa, ma, fb, kj, c.m0);
            }
            if (b_mn) {
#pragma unroll
              for (int i = 0; i < BN / 64; ++i) tma_load_2d(sb + i * 8192, mb, fb, c.n0 + 64 * i, kj);
            } else {
              tma_load_2d(sb, mb, fb, kj, c.n0);
            }
          }
          issued[st] += 1;
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        for (int i = 0; i < S; ++i)
          if (issued[i] > 0) mbar_wait_bounded(smem_u32(&full_bar[i]), (uint32_t)((issued[i] - 1) & 1), nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const StageDescs dsc = make_stage_descs(p, sbase, sbase + Cfg::kABytes, kBM, BN);
      bool ok = true;
      int issued_any = 0;
      int g = 0, it = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++it) {
        const Unit c = unit_coords(p, u, BN);
        const int k_begin = c.split * p.k_per_split;
        const int k_end0 = min(p.K0, k_begin + p.k_per_split);
        const int steps0 = (k_end0 - k_begin + kStepK - 1) / kStepK;
        const int steps = steps0 + (c.split == 0 ? steps1 : 0);
        const int buf = it & 1;
        // the epilogue must have drained this accumulator (two units ago)
        if (!mbar_wait_bounded(smem_u32(&acc_empty[buf]), (uint32_t)(((it >> 1) & 1) ^ 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int step = 0; step < steps; ++step, ++g) {
          const int st = g % S;
          const uint32_t ph = (uint32_t)((g / S) & 1);
          if (!mbar_wait_bounded(smem_u32(&full_bar[st]), ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const bool ext = step >= steps0;
          const int kk = ext ? (step - steps0) * kStepK : k_begin + step * kStepK;
          const int nk = min(KSUB, ((ext ? p.K1 : k_end0) - kk + kBK - 1) / kBK);
          for (int j = 0; j < nk; ++j) {
            int nsub = 4;
            if (ext) nsub = min(4, (p.K1 - (kk + j * kBK) + 15) / 16);
            issue_kstep(d_tmem, dsc, ext ? 1 : 0, (uint32_t)(st * Cfg::kStageBytes + j * Cfg::kSubA) >> 4,
                        (uint32_t)(st * Cfg::kStageBytes + j * Cfg::kSubB) >> 4, nsub, step == 0 && j == 0);
          }
          issued_any = 1;
          umma_commit(smem_u32(&empty_bar[st]));
        }
        if (ok) umma_commit(smem_u32(&acc_full[buf]));
      }
      if (!ok && issued_any) {
        // wait for MMAs already issued before TMEM is released
        umma_commit(smem_u32(drain_bar));
        mbar_wait_bounded(smem_u32(drain_bar), 0, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;             // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;
    int it = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++it) {
      const Unit c = unit_coords(p, u, BN);
      const int buf = it & 1;
      if (!mbar_wait_bounded(smem_u32(&acc_full[buf]), (uint32_t)((it >> 1) & 1), abort_flag)) break;
      tc_fence_after();
      const int m = c.m0 + row;
      const bool row_ok = m < p.M;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if (Cfg::kStoreStage > 0 && p.tma_store) {
        // bf16 output through shared memory: this warp's 32 rows x 64 columns
        // per box, 128B-swizzled (conflict-free 16-byte writes), stored by TMA
        // (coalesced, clipped at the matrix edge); two boxes in flight per warp
        uint8_t* stg = smem + S * Cfg::kStageBytes + (warp - 2) * 8192;
        const uint32_t stg_s = sbase + S * Cfg::kStageBytes + (uint32_t)((warp - 2) * 8192);
#pragma unroll 1
        for (int b = 0; b < BN / 64; ++b) {
          uint32_t v0[32], v1[32];
          tmem_ld_32x32b_x32(taddr + (uint32_t)(b * 64), v0);
          tmem_ld_32x32b_x32(taddr + (uint32_t)(b * 64 + 32), v1);
          tmem_ld_wait();
          if (b >= 2) {
            if (lane == 0) bulk_wait_group_read1();       // the store that used this buffer
            __syncwarp();
          }
          uint8_t* box = stg + (b & 1) * 4096;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t (&v)[32] = q < 4 ? v0 : v1;
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
            tma_store_2d(&tmOut, stg_s + (uint32_t)((b & 1) * 4096), c.n0 + 64 * b, c.m0 + quarter * 32);
            bulk_commit_group();
          }
        }
        if (lane == 0) bulk_wait_group_read0();            // staging reusable by the next unit
        __syncwarp();
      } else if (p.epi == EPI_MERGE || p.epi == EPI_UNMERGE) {
        epilogue_merge_row<BN>(p, taddr, m, row_ok, c.n0, s_lut);
      } else
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        if (p.pair_offset > 0 && ch * 32 >= p.pair_offset) break;   // lo columns: consumed below
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32), v);
        tmem_ld_wait();
        if (p.pair_offset > 0) {
          uint32_t lo[32];
          tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32 + p.pair_offset), lo);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[i] = __float_as_uint(__fadd_rn(__uint_as_float(v[i]), __uint_as_float(lo[i])));
        }
        const int n = c.n0 + ch * 32;
        if (row_ok && n < p.N) epilogue_chunk(p, v, m, n, c.split, s_lut);
      }
      // this accumulator may be overwritten once all four warps are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
    }
    if (Cfg::kStoreStage > 0 && p.tma_store && lane == 0) bulk_wait_group0();   // stores complete
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

}  // namespace qlora
