// NF4 + double-quant storage kernels (HBM-streaming, CUDA cores).
//
// [P1] "LoRA and QLoRA fine-tuning: mechanics, and when not to fine-tune",
// section "What QLoRA freezes, and in how many bits": blockwise 4-bit
// NormalFloat with block 64; block constants quantised again to FP8 in
// blocks of 256 after subtracting their mean; doubleDequant in the forward
// equation.
//
// Arithmetic is pinned to fp32/fp64 round-to-nearest operations written out
// explicitly (__fmul_rn, __fadd_rn, ...) so that no contraction changes a
// rounding; the CPU oracle states the same steps.
#pragma once
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace qlora {

constexpr int kBlock = 64;
constexpr int kBlock2 = 256;
constexpr int kEncBins = 129;     // rint(64 x) + 64, x in [-1, 1]
constexpr int kFastBins = 33;     // rint(16 x) + 16, x in [-1, 1]

// Encoder tables.  Bin j holds every x with rint(64 x) = j - 64, i.e. the
// closed interval [(j - 64.5)/64, (j - 63.5)/64] (closed because a tie may
// round either way).  base[j] = the number of thresholds at or below the
// bin's lower edge; the only threshold that can lie inside the bin is then
// thr[base[j]] (the first one above the edge; thr[15] = +inf), because the
// smallest gap between thresholds (~0.08) exceeds the bin width 1/64 (the
// host builder checks it).  So code(x) = base[j] + (x >= thr[base[j]]): a
// threshold above the bin never satisfies the comparison.  Both tables are
// read with 1- and 4-byte shared loads that do not conflict across banks.
struct EncTable {
  uint8_t base[kEncBins + 3];
  float thr[16];
  // The same construction on bins of width 1/16 (j = rint(16 x) + 16), which
  // the gap between thresholds (> 1/16) still allows: 33 entries, so each
  // table fits one word per shared-memory bank.
  float fthr[kFastBins];
  uint32_t fbase[kFastBins];
};
struct NF4Levels {
  float q[16];
};

// Correctly rounded fp32 quotient w / a given y = RN(1/a) (Markstein 1990,
// "Computation of elementary functions on the IBM RISC System/6000 processor":
// if q0 is within one ulp of w/a and y = RN(1/a), then RN(q0 + r*y) with the
// exact remainder r = w - a*q0 is the correctly rounded quotient).  Valid for
// the ranges used here (|w| <= a, normal a); checked against IEEE division on
// the device by the test suite.
__device__ __forceinline__ float div_markstein(float w, float a, float y) {
  const float q0 = __fmul_rn(w, y);
  const float r = __fmaf_rn(-a, q0, w);
  return __fmaf_rn(r, y, q0);
}

// rint(64 x) for |x| <= 1 without a float-to-int conversion: adding 1.5 * 2^23
// leaves the rounded integer in the low mantissa bits (round to nearest even).
// (x * 64 is exact, so one fused multiply-add rounds exactly like the add.)
// The unsigned clamp keeps non-finite inputs inside the table.
__device__ __forceinline__ uint32_t enc_code(float x, const uint8_t* s_base, const float* s_thr) {
  const float t = __fmaf_rn(x, 64.0f, 12582912.0f);
  const uint32_t j = min((uint32_t)__float_as_int(t) - (uint32_t)(0x4B400000 - 64), (uint32_t)(kEncBins - 1));
  const uint32_t b = s_base[j];
  return b + (x >= s_thr[b] ? 1u : 0u);
}

// The fast encoder reads {fthr[j], fbase[j]} of the coarse bins from two
// 33-word shared arrays laid out back to back (fbase 33 words after fthr):
// no two bins but the outermost pair share a bank, and both loads use one
// address, bits(t) * 4 + K with t = x * 16 + 1.5 * 2^23 and
// K = table - (0x4B400000 - 16) * 4 (mod 2^32).  It is used only where
// |x| <= 1 is guaranteed, so the address needs no clamp.
// Eight codes of one thread's weights, packed (element i in nibble i), as
// one block of PTX so that nothing but the arithmetic below is emitted:
//   x_i  = RN(w_i / m)   Markstein: q = w y, r = w - m q (exact), x = q + r y
//   t_i  = x_i * 16 + 1.5 * 2^23        (rint(16 x_i) in the low bits)
//   a_i  = bits(t_i) * 4 + K            (address of bin rint(16 x_i) + 16)
//   code = fbase[a_i] + (x_i >= fthr[a_i]),  summed into nibble i (no carries)
__device__ __forceinline__ uint32_t encode8_fast(const float* w, float m, float y, uint32_t K) {
  uint32_t packed;
  asm("{\n\t"
      ".reg .f32 nm, q<8>, r<8>, x<8>, t<8>, th<8>;\n\t"
      ".reg .b32 a<8>, b<8>;\n\t"
      ".reg .pred p<8>;\n\t"
      "neg.f32 nm, %9;\n\t"
      "mul.rn.f32 q0, %1, %10;\n\t"
      "fma.rn.f32 r0, nm, q0, %1;\n\t"
      "fma.rn.f32 x0, r0, %10, q0;\n\t"
      "fma.rn.f32 t0, x0, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a0, t0;\n\t"
      "mad.lo.u32 a0, a0, 4, %11;\n\t"
      "mul.rn.f32 q1, %2, %10;\n\t"
      "fma.rn.f32 r1, nm, q1, %2;\n\t"
      "fma.rn.f32 x1, r1, %10, q1;\n\t"
      "fma.rn.f32 t1, x1, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a1, t1;\n\t"
      "mad.lo.u32 a1, a1, 4, %11;\n\t"
      "mul.rn.f32 q2, %3, %10;\n\t"
      "fma.rn.f32 r2, nm, q2, %3;\n\t"
      "fma.rn.f32 x2, r2, %10, q2;\n\t"
      "fma.rn.f32 t2, x2, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a2, t2;\n\t"
      "mad.lo.u32 a2, a2, 4, %11;\n\t"
      "mul.rn.f32 q3, %4, %10;\n\t"
      "fma.rn.f32 r3, nm, q3, %4;\n\t"
      "fma.rn.f32 x3, r3, %10, q3;\n\t"
      "fma.rn.f32 t3, x3, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a3, t3;\n\t"
      "mad.lo.u32 a3, a3, 4, %11;\n\t"
      "mul.rn.f32 q4, %5, %10;\n\t"
      "fma.rn.f32 r4, nm, q4, %5;\n\t"
      "fma.rn.f32 x4, r4, %10, q4;\n\t"
      "fma.rn.f32 t4, x4, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a4, t4;\n\t"
      "mad.lo.u32 a4, a4, 4, %11;\n\t"
      "mul.rn.f32 q5, %6, %10;\n\t"
      "fma.rn.f32 r5, nm, q5, %6;\n\t"
      "fma.rn.f32 x5, r5, %10, q5;\n\t"
      "fma.rn.f32 t5, x5, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a5, t5;\n\t"
      "mad.lo.u32 a5, a5, 4, %11;\n\t"
      "mul.rn.f32 q6, %7, %10;\n\t"
      "fma.rn.f32 r6, nm, q6, %7;\n\t"
      "fma.rn.f32 x6, r6, %10, q6;\n\t"
      "fma.rn.f32 t6, x6, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a6, t6;\n\t"
      "mad.lo.u32 a6, a6, 4, %11;\n\t"
      "mul.rn.f32 q7, %8, %10;\n\t"
      "fma.rn.f32 r7, nm, q7, %8;\n\t"
      "fma.rn.f32 x7, r7, %10, q7;\n\t"
      "fma.rn.f32 t7, x7, 0f41800000, 0f4B400000;\n\t"
      "mov.b32 a7, t7;\n\t"
      "mad.lo.u32 a7, a7, 4, %11;\n\t"
      "ld.shared.f32 th0, [a0];\n\t"
      "ld.shared.u32 b0, [a0+132];\n\t"
      "ld.shared.f32 th1, [a1];\n\t"
      "ld.shared.u32 b1, [a1+132];\n\t"
      "ld.shared.f32 th2, [a2];\n\t"
      "ld.shared.u32 b2, [a2+132];\n\t"
      "ld.shared.f32 th3, [a3];\n\t"
      "ld.shared.u32 b3, [a3+132];\n\t"
      "ld.shared.f32 th4, [a4];\n\t"
      "ld.shared.u32 b4, [a4+132];\n\t"
      "ld.shared.f32 th5, [a5];\n\t"
      "ld.shared.u32 b5, [a5+132];\n\t"
      "ld.shared.f32 th6, [a6];\n\t"
      "ld.shared.u32 b6, [a6+132];\n\t"
      "ld.shared.f32 th7, [a7];\n\t"
      "ld.shared.u32 b7, [a7+132];\n\t"
      "setp.ge.f32 p0, x0, th0;\n\t"
      "setp.ge.f32 p1, x1, th1;\n\t"
      "setp.ge.f32 p2, x2, th2;\n\t"
      "setp.ge.f32 p3, x3, th3;\n\t"
      "setp.ge.f32 p4, x4, th4;\n\t"
      "setp.ge.f32 p5, x5, th5;\n\t"
      "setp.ge.f32 p6, x6, th6;\n\t"
      "setp.ge.f32 p7, x7, th7;\n\t"
      "mov.u32 %0, b0;\n\t"
      "shl.b32 b1, b1, 4;\n\t"
      "add.u32 %0, %0, b1;\n\t"
      "shl.b32 b2, b2, 8;\n\t"
      "add.u32 %0, %0, b2;\n\t"
      "shl.b32 b3, b3, 12;\n\t"
      "add.u32 %0, %0, b3;\n\t"
      "shl.b32 b4, b4, 16;\n\t"
      "add.u32 %0, %0, b4;\n\t"
      "shl.b32 b5, b5, 20;\n\t"
      "add.u32 %0, %0, b5;\n\t"
      "shl.b32 b6, b6, 24;\n\t"
      "add.u32 %0, %0, b6;\n\t"
      "shl.b32 b7, b7, 28;\n\t"
      "add.u32 %0, %0, b7;\n\t"
      "@p0 add.u32 %0, %0, 1;\n\t"
      "@p1 add.u32 %0, %0, 16;\n\t"
      "@p2 add.u32 %0, %0, 256;\n\t"
      "@p3 add.u32 %0, %0, 4096;\n\t"
      "@p4 add.u32 %0, %0, 65536;\n\t"
      "@p5 add.u32 %0, %0, 1048576;\n\t"
      "@p6 add.u32 %0, %0, 16777216;\n\t"
      "@p7 add.u32 %0, %0, 268435456;\n\t"
      "}"
      : "=r"(packed)
      : "f"(w[0]), "f"(w[1]), "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7]),
        "f"(m), "f"(y), "r"(K));
  return packed;
}

// Eight codes by the general route (any block absmax): IEEE division and the
// clamped encoder; an all-zero (or NaN) block gives the zero level.
__device__ __forceinline__ uint32_t encode8_general(const float* w, float m, const uint8_t* s_base,
                                                    const float* s_thr) {
  if (!(m > 0.f)) return 0x77777777u;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= enc_code(__fdiv_rn(w[i], m), s_base, s_thr) << (4 * i);
  return packed;
}

// max(a, |b|) that returns NaN if either operand is NaN.
__device__ __forceinline__ float max_abs_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(fabsf(b)));
  return r;
}

// ---------------------------------------------------------------------------
// The mean of the block constants, formed by the last CTA of phase 1 (the one
// that takes the final ticket, so every group sum is in memory): S is the
// float64 pairwise tree over the n_g group sums padded with zeros to
// P = max(2^ceil(log2 n_g), 1024) leaves (zero leaves and zero subtrees add
// exactly nothing, so the padding does not change S).  mean = fp32(S / n_b).
// ---------------------------------------------------------------------------
constexpr int kMeanChunks = 1024;      // P / 1024 <= 1024 for n_g <= 2^20

// Lane l of a warp: the pairwise tree over the 8 consecutive leaves
// first + 8 l .. first + 8 l + 7 (zero beyond n), then the shuffle tree over
// the lanes: lane 0 returns the tree over the 256 leaves from `first`.
__device__ __forceinline__ double warp_tree256(const double* v, int64_t first, int64_t n, int lane) {
  const int64_t i0 = first + 8 * lane;
  double a[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    const int64_t i = i0 + j;
    if (i + 1 < n) {
      const double2 t = __ldcg(reinterpret_cast<const double2*>(v + i));
      a[j] = t.x;
      a[j + 1] = t.y;
    } else {
      a[j] = (i < n) ? __ldcg(v + i) : 0.0;
      a[j + 1] = 0.0;
    }
  }
  double s = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) s = s + __shfl_down_sync(0xffffffffu, s, off);
  return s;
}

// Run by one whole CTA.  Each warp takes aligned chunks of 1024 leaves as
// the tree of four 256-leaf subtrees; a shared-memory tree joins the P/1024
// chunk sums in s_v.
__device__ __forceinline__ void pairwise_mean(const double* group_sum, int64_t n_g, int64_t n_b,
                                              float* mean_out, double* s_v) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  int64_t P = 1024;
  while (P < n_g) P <<= 1;
  const int nch = (int)(P / 1024);
  for (int c = warp; c < nch; c += (int)(blockDim.x >> 5)) {
    const int64_t first = (int64_t)c * 1024;
    const double s0 = warp_tree256(group_sum, first, n_g, lane);
    const double s1 = warp_tree256(group_sum, first + 256, n_g, lane);
    const double s2 = warp_tree256(group_sum, first + 512, n_g, lane);
    const double s3 = warp_tree256(group_sum, first + 768, n_g, lane);
    if (lane == 0) s_v[c] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
  for (int st = 1; st < nch; st <<= 1) {
    for (int j = 2 * st * tid; j < nch; j += 2 * st * (int)blockDim.x) s_v[j] = s_v[j] + s_v[j + st];
    __syncthreads();
  }
  if (tid == 0) mean_out[0] = __double2float_rn(__ddiv_rn(s_v[0], (double)n_b));
}

// ---------------------------------------------------------------------------
// Phase 1: persistent CTAs, each taking groups of 256 blocks (16384 weights)
// in turn.  8 threads per block, 8 consecutive weights per thread.  Writes
// packed codes, the fp32 block absmax (scratch) and the fp64 pairwise sum of
// each group's absmax.
//
// Fast path (every block of the warp has its absmax a in [2^-125, 2^125]):
// x = w / a by Markstein's correction from y = RN(1/a) (all intermediates
// normal in that range, and |x| <= 1 because |w| <= a), then encode8_fast.
// Otherwise the warp takes the general route (needed for an all-zero,
// subnormal or huge absmax, or a NaN, which the NaN-propagating maximum
// exposes).  Both give RN(w / a) and the same code.  Only the last group
// checks bounds.  The CTA that finishes last also forms the mean.
// ---------------------------------------------------------------------------
template <bool kTail>
__device__ __forceinline__ void quantize_group(const float* __restrict__ W0, int64_t n_b, int64_t g,
                                               uint32_t* __restrict__ codes_u32, float* __restrict__ absmax,
                                               float* s_abs, uint32_t K, const uint8_t* s_base,
                                               const float* s_thr) {
  const int tid = threadIdx.x;
  const int sub = tid & 7;          // 8 threads per block
  const int lb0 = tid >> 3;         // 32 blocks per pass
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float4 v[4][2];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int64_t b = g * kBlock2 + (half * 4 + p) * 32 + lb0;
      if (!kTail || b < n_b) {
        const float4* src = reinterpret_cast<const float4*>(W0 + b * kBlock + sub * 8);
        v[p][0] = __ldcs(src);
        v[p][1] = __ldcs(src + 1);
      } else {
        v[p][0] = make_float4(0.f, 0.f, 0.f, 0.f);
        v[p][1] = v[p][0];
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int lb = (half * 4 + p) * 32 + lb0;
      const int64_t b = g * kBlock2 + lb;
      const float* w = reinterpret_cast<const float*>(&v[p][0]);
      float m = fabsf(w[0]);
#pragma unroll
      for (int i = 1; i < 8; ++i) m = max_abs_nan(m, w[i]);
      m = max_abs_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = max_abs_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = max_abs_nan(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const bool fast = m >= 0x1p-125f && m <= 0x1p125f;
      // (the general route gives the same codes for blocks the fast one takes)
      const uint32_t packed = __all_sync(0xffffffffu, fast) ? encode8_fast(w, m, __frcp_rn(m), K)
                                                            : encode8_general(w, m, s_base, s_thr);
      if (!kTail || b < n_b) {
        codes_u32[b * 8 + sub] = packed;
        if (sub == 0) absmax[b] = m;
      }
      if (sub == 0) s_abs[lb] = (!kTail || b < n_b) ? m : 0.f;
    }
  }
}

__global__ void __launch_bounds__(256) nf4_quantize_phase1(
    const float* __restrict__ W0, int64_t n_b, int64_t n_g, uint32_t* __restrict__ codes_u32,
    float* __restrict__ absmax, double* __restrict__ group_sum, unsigned int* __restrict__ ticket,
    float* __restrict__ mean_out, const __grid_constant__ EncTable tab) {
  __shared__ double s_v[kMeanChunks];
  __shared__ bool s_last;
  __shared__ uint32_t s_fast[2 * kFastBins];      // fthr (as bits), then fbase
  __shared__ uint8_t s_base[kEncBins + 3];
  __shared__ float s_thr[16];
  __shared__ float s_abs[2][kBlock2];             // block constants of two groups in turn
  const int tid = threadIdx.x;
  if (tid < kFastBins) {
    s_fast[tid] = __float_as_uint(tab.fthr[tid]);
    s_fast[kFastBins + tid] = tab.fbase[tid];
  }
  if (tid < kEncBins + 3) s_base[tid] = tab.base[tid];
  if (tid < 16) s_thr[tid] = tab.thr[tid];
  __syncthreads();
  const uint32_t K = smem_u32(s_fast) - (uint32_t)(0x4B400000 - 16) * 4u;
  // persistent: this CTA takes groups blockIdx.x, blockIdx.x + gridDim.x, ...
  int it = 0;
  for (int64_t g = blockIdx.x; g < n_g; g += gridDim.x, ++it) {
    float* sa = s_abs[it & 1];
    if ((g + 1) * kBlock2 <= n_b)
      quantize_group<false>(W0, n_b, g, codes_u32, absmax, sa, K, s_base, s_thr);
    else
      quantize_group<true>(W0, n_b, g, codes_u32, absmax, sa, K, s_base, s_thr);
    // one barrier per group: warp 0 reads this group's constants while the
    // other warps already fill the other half of s_abs with the next group
    __syncthreads();
    if (tid < 32) {
      // pairwise tree over the 256 constants: lane l sums leaves 8l..8l+7,
      // then the lanes are combined in halves (shfl_down by 1, 2, 4, 8, 16)
      double a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = (double)sa[tid * 8 + i];
      double s = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) s = s + __shfl_down_sync(0xffffffffu, s, off);
      if (tid == 0) group_sum[g] = s;
    }
  }
  // publish this CTA's sums, then take a ticket: the CTA with the last ticket
  // sees every group sum and forms the mean
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    pairwise_mean(group_sum, n_g, n_b, mean_out, s_v);
  }
}

// ---------------------------------------------------------------------------
// Phase 2: double quantisation, eight groups per CTA (thread t = block t of
// each group):
//   scale2_j   = fp32(max_b |fp32(a_b - mean)| / 448),
//   absmax_q_b = E4M3_RN_satfinite(fp32(fp32(a_b - mean) / scale2_j)).
// ---------------------------------------------------------------------------
constexpr int kDqGroups = 8;

__global__ void __launch_bounds__(256) nf4_quantize_dq(const float* __restrict__ absmax, int64_t n_g,
                                                       int64_t n_b, const float* __restrict__ mean,
                                                       uint8_t* __restrict__ absmax_q,
                                                       float* __restrict__ scale2) {
  __shared__ float s_max[kDqGroups][8];
  __shared__ float s_s1[kDqGroups], s_y1[kDqGroups];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const float mu = mean[0];
  const int64_t g0 = (int64_t)blockIdx.x * kDqGroups;
  float cen[kDqGroups];
#pragma unroll
  for (int i = 0; i < kDqGroups; ++i) {
    const int64_t b = (g0 + i) * kBlock2 + tid;
    cen[i] = (b < n_b) ? __fsub_rn(absmax[b], mu) : 0.f;
  }
#pragma unroll
  for (int i = 0; i < kDqGroups; ++i) {
    float m = fabsf(cen[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) s_max[i][warp] = m;
  }
  __syncthreads();
  if (tid < kDqGroups) {
    // one thread per group: scale2 and, where it is a comfortably normal
    // number, y = RN(1/scale2) for the quotients below
    float c1 = s_max[tid][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) c1 = fmaxf(c1, s_max[tid][w]);
    const float s1 = (c1 > 0.f) ? __fdiv_rn(c1, 448.0f) : 0.f;
    s_s1[tid] = s1;
    s_y1[tid] = (s1 >= 0x1p-100f && s1 <= 0x1p100f) ? __frcp_rn(s1) : 0.f;
    if (g0 + tid < n_g) scale2[g0 + tid] = s1;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kDqGroups; ++i) {
    const int64_t b = (g0 + i) * kBlock2 + tid;
    if (g0 + i < n_g && b < n_b) {
      // x = RN(cen / scale2): Markstein's correction from y (|x| <= 448, and
      // a quotient too small for the correction is below E4M3's smallest
      // step, where both round to a zero of the same sign), else IEEE
      // division
      const float s1 = s_s1[i], y1 = s_y1[i];
      uint8_t code = 0;
      if (s1 > 0.f) {
        const float x = (y1 != 0.f) ? div_markstein(cen[i], s1, y1) : __fdiv_rn(cen[i], s1);
        code = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
      }
      absmax_q[b] = code;
    }
  }
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}

// a'_b = fp32(fp32(E4M3(c2_b) * s1_j) + mean)
__device__ __forceinline__ float block_scale(const uint8_t* absmax_q, const float* scale2,
                                             float mu, int64_t b) {
  return __fadd_rn(__fmul_rn(e4m3_to_f32(absmax_q[b]), scale2[b / kBlock2]), mu);
}

// 32 codes (one 16-byte word) -> 32 bf16 values of level[code] * a'.
// 8 codes (one 32-bit word, element 2j in the low nibble of byte j) -> 8 bf16
// values of level[code] * a, packed in pairs.  Both nibbles of every byte are
// turned into byte offsets into the 16-entry level table with two logic ops,
// then each offset is taken out with one byte permute; `s_q` must be a
// shared-memory table so the load is a register-plus-offset address.
__device__ __forceinline__ void dequant8(uint32_t w, float a, const float* s_q, uint32_t* o) {
  const uint32_t lo = (w & 0x0F0F0F0Fu) << 2;      // byte j = 4 * code(2j)
  const uint32_t hi = (w >> 2) & 0x3C3C3C3Cu;      // byte j = 4 * code(2j + 1)
  const char* base = reinterpret_cast<const char*>(s_q);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t ol = __byte_perm(lo, 0u, 0x4440u + j);
    const uint32_t oh = __byte_perm(hi, 0u, 0x4440u + j);
    const float ql = *reinterpret_cast<const float*>(base + ol);
    const float qh = *reinterpret_cast<const float*>(base + oh);
    const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(ql, a), __fmul_rn(qh, a));
    o[j] = *reinterpret_cast<const uint32_t*>(&p);
  }
}

// 32 codes (one 16-byte word) -> 32 bf16 values of level[code] * a.
__device__ __forceinline__ void dequant32(const uint4 c, float a, const float* s_q, uint32_t (&o)[16]) {
  dequant8(c.x, a, s_q, o + 0);
  dequant8(c.y, a, s_q, o + 4);
  dequant8(c.z, a, s_q, o + 8);
  dequant8(c.w, a, s_q, o + 12);
}

// ---------------------------------------------------------------------------
// Dequantise to a bf16 d x k matrix.  Unit = 8 consecutive weights: a 4-byte
// code load and a 16-byte store, consecutive threads on consecutive units so
// both streams are fully coalesced; 4 independent units per thread in flight.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(
    const uint32_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
    const float* __restrict__ scale2, const float* __restrict__ mean, int64_t n_units,
    uint4* __restrict__ W_out, const __grid_constant__ NF4Levels lv) {
  __shared__ float s_q[16];
  if (threadIdx.x < 16) s_q[threadIdx.x] = lv.q[threadIdx.x];
  __syncthreads();
  const float mu = mean[0];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n_units; base += 4 * stride) {
    uint32_t c[4];
    float a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t u = base + j * stride;
      c[j] = 0u;
      a[j] = 0.f;
      if (u < n_units) {
        c[j] = __ldcs(codes + u);
        a[j] = block_scale(absmax_q, scale2, mu, u >> 3);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t u = base + j * stride;
      if (u < n_units) {
        uint32_t o[4];
        dequant8(c[j], a[j], s_q, o);
        __stcs(W_out + u, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Block scales a'_b = fp32(fp32(E4M3(absmax_q_b) * scale2_j) + mean) of every
// block, written once per GEMM call in the layout the dequantising GEMMs load
// by TMA next to the codes (one tile of scales per K-step):
//   transposed = 1: out[s * ld + n]  (block column s, row n: one K-step of the
//                   forward reads consecutive rows)
//   transposed = 0: out[n * ld + s]  (row n, block column s: one K-step of dX
//                   reads consecutive block columns of 64 rows)
// Threads of a 32 x 32 tile read the constants row by row and write through
// shared memory, so both the loads and the stores are coalesced.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nf4_block_scales(const uint8_t* __restrict__ absmax_q,
                                                        const float* __restrict__ scale2,
                                                        const float* __restrict__ mean, int64_t d, int64_t kb,
                                                        int transposed, int64_t ld, float* __restrict__ out) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;       // 32 x 8 threads
  const int64_t n0 = (int64_t)blockIdx.y * 32, s0 = (int64_t)blockIdx.x * 32;
  const float mu = mean[0];
  for (int j = ty; j < 32; j += 8) {
    const int64_t n = n0 + j, sc = s0 + tx;
    float a = 0.f;
    if (n < d && sc < kb) {
      const int64_t b = n * kb + sc;
      a = __fadd_rn(__fmul_rn(e4m3_to_f32(absmax_q[b]), scale2[b / kBlock2]), mu);
    }
    tile[j][tx] = a;
  }
  __syncthreads();
  if (transposed) {
    for (int j = ty; j < 32; j += 8) {
      const int64_t sc = s0 + j, n = n0 + tx;
      if (sc < kb && n < d) out[sc * ld + n] = tile[tx][j];
    }
  } else {
    for (int j = ty; j < 32; j += 8) {
      const int64_t n = n0 + j, sc = s0 + tx;
      if (n < d && sc < kb) out[n * ld + sc] = tile[j][tx];
    }
  }
}

// ---------------------------------------------------------------------------
// Small helpers for the rank-r operands.
// ---------------------------------------------------------------------------
// Adapter gradients for a few tokens (T <= 64), in fp32 on CUDA cores: with
// so few terms the T-reductions are a handful of FMAs per output, and the
// outputs (r x k and d x r fp32) are what costs.  Each output is summed over
// the tokens in order, so results are deterministic:
//   dA[i][j] = sum_t sG[t][i] X[t][j]          (r x k; sG = s G, fp32)
//   dB[i][j] = sum_t dY[t][i] fl(s U[t][j])    (d x r)
// A thread forms four outputs from 8-byte loads: blocks [0, nb_a) take dA,
// row i = block / kblk and four consecutive columns j per thread; the rest
// take dB, four consecutive rows i (d % 8 == 0) for one column j, 256 / r
// row quads of r columns per block (r <= 256).  Needs k % 4 == 0, d % 4 == 0
// and 8-byte aligned X and dY rows.
constexpr int kGradThreads = 256;
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__global__ void __launch_bounds__(kGradThreads) adapter_grads_small(const uint16_t* __restrict__ X,
                                                                    const uint16_t* __restrict__ dY,
                                                                    const float* __restrict__ U,
                                                                    const float* __restrict__ sG, float s, int T,
                                                                    int d, int k, int r, int kblk, int nb_a,
                                                                    float* __restrict__ dA, float* __restrict__ dB) {
  griddep_launch_dependents();
  griddep_wait();
  const int b = (int)blockIdx.x;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  if (b < nb_a) {
    const int i = b / kblk;
    const int j = 4 * ((b - i * kblk) * kGradThreads + (int)threadIdx.x);
    if (j >= k) return;
    // the loads of 16 tokens are all issued before their FMAs
    for (int t0 = 0; t0 < T; t0 += 16) {
      float g[16];
      uint2 x[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int t = min(t0 + q, T - 1);
        g[q] = __ldg(sG + t * r + i);
        x[q] = __ldg(reinterpret_cast<const uint2*>(X + (int64_t)t * k + j));
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (t0 + q < T) {
          a0 = __fmaf_rn(g[q], bf16_lo(x[q].x), a0);
          a1 = __fmaf_rn(g[q], bf16_hi(x[q].x), a1);
          a2 = __fmaf_rn(g[q], bf16_lo(x[q].y), a2);
          a3 = __fmaf_rn(g[q], bf16_hi(x[q].y), a3);
        }
      }
    }
    float* o = dA + (int64_t)i * k + j;
    o[0] = a0;
    o[1] = a1;
    o[2] = a2;
    o[3] = a3;
    return;
  }
  const int qpb = kGradThreads / r;                 // row quads of dB per block
  const int tq = (int)threadIdx.x / r;
  const int j = (int)threadIdx.x - tq * r;
  const int i = 4 * ((b - nb_a) * qpb + tq);
  if (tq >= qpb || i >= d) return;
  for (int t0 = 0; t0 < T; t0 += 16) {
    float u[16];
    uint2 y[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int t = min(t0 + q, T - 1);
      u[q] = __ldg(U + t * r + j);
      y[q] = __ldg(reinterpret_cast<const uint2*>(dY + (int64_t)t * d + i));
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if (t0 + q < T) {
        const float su = __fmul_rn(s, u[q]);
        a0 = __fmaf_rn(bf16_lo(y[q].x), su, a0);
        a1 = __fmaf_rn(bf16_hi(y[q].x), su, a1);
        a2 = __fmaf_rn(bf16_lo(y[q].y), su, a2);
        a3 = __fmaf_rn(bf16_hi(y[q].y), su, a3);
      }
    }
  }
  float* o = dB + (int64_t)i * r + j;
  o[0] = a0;
  o[r] = a1;
  o[2 * r] = a2;
  o[3 * r] = a3;
}

// dst (rows x ld_dst, bf16) = src (rows x cols, bf16) with zero columns
// [cols, ld_dst).
__global__ void pad_cols_bf16(const uint16_t* __restrict__ src, int64_t rows, int cols,
                              uint16_t* __restrict__ dst, int ld_dst) {
  const int64_t n = rows * ld_dst;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t rrow = i / ld_dst;
    const int c = (int)(i - rrow * ld_dst);
    dst[i] = (c < cols) ? src[rrow * cols + c] : (uint16_t)0;
  }
}

// Two-term bf16 split of v = fp32(scale * src): hi = bf16(v), lo = bf16(v - hi)
// (v - hi is exact in fp32), so hi + lo carries about 16 significant bits.
// dst row t: columns [0, half) hold hi, [half, 2*half) hold lo; columns at or
// beyond `cols` within each half are zero.
__global__ void scale_f32_to_bf16_hilo(const float* __restrict__ src, int64_t rows, int cols,
                                       float scale, uint16_t* __restrict__ dst, int half) {
  const int ld = 2 * half;
  const int64_t n = rows * half;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t rrow = i / half;
    const int c = (int)(i - rrow * half);
    const float v = (c < cols) ? __fmul_rn(scale, src[rrow * cols + c]) : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(h)));
    dst[rrow * ld + c] = *reinterpret_cast<const uint16_t*>(&h);
    dst[rrow * ld + half + c] = *reinterpret_cast<const uint16_t*>(&l);
  }
}

// out[i] = sum_z part[z * stride + i], z = 0, 1, ... in order (deterministic).
__global__ void splitk_reduce_f32(const float* __restrict__ part, int splits, int64_t n,
                                  float* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    float s = part[i];
    for (int z = 1; z < splits; ++z) s = __fadd_rn(s, part[(int64_t)z * n + i]);
    out[i] = s;
  }
}

// LoRA dropout on the adapter input: Xm = X with every element whose keep bit
// is 0 set to +0 (bf16 bit patterns; the kept elements are copied exactly).
// Unit = 8 consecutive elements: one 16-byte load of X, one byte of the
// bit-packed mask (bit i keeps element 8u + i), one 16-byte store.
__global__ void apply_keep_bf16(const uint4* __restrict__ X, const uint8_t* __restrict__ keep, int64_t n_units,
                                uint4* __restrict__ Xm) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n_units; u += stride) {
    const uint4 x = __ldcs(X + u);
    const uint32_t b = keep[u];
    const uint32_t m0 = ((b & 1u) ? 0x0000FFFFu : 0u) | ((b & 2u) ? 0xFFFF0000u : 0u);
    const uint32_t m1 = ((b & 4u) ? 0x0000FFFFu : 0u) | ((b & 8u) ? 0xFFFF0000u : 0u);
    const uint32_t m2 = ((b & 16u) ? 0x0000FFFFu : 0u) | ((b & 32u) ? 0xFFFF0000u : 0u);
    const uint32_t m3 = ((b & 64u) ? 0x0000FFFFu : 0u) | ((b & 128u) ? 0xFFFF0000u : 0u);
    Xm[u] = make_uint4(x.x & m0, x.y & m1, x.z & m2, x.w & m3);
  }
}

// ---------------------------------------------------------------------------
// Several unmerged adapters in one batch: token t uses adapter idx[t] of a
// stack (A_i r x k, B_i d x r, scale s_i).  Their rank-r operands are laid out
// side by side, R = n r columns, each token's values in its adapter's block of
// r columns and zeros elsewhere, so one GEMM with depth R computes every
// token's own adapter term.
// ---------------------------------------------------------------------------
constexpr int kMaxAdapters = 64;
struct AdapterScales {
  float s[kMaxAdapters];
};

// Bcat[row][i r + j] = Bs[i][row][j]  (d x R, bf16)
__global__ void cat_adapters_b(const uint16_t* __restrict__ Bs, int64_t d, int r, int n,
                               uint16_t* __restrict__ Bcat) {
  const int R = n * r;
  const int64_t total = d * R;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t row = e / R;
    const int c = (int)(e - row * R);
    const int i = c / r, j = c - i * r;
    Bcat[e] = Bs[((int64_t)i * d + row) * r + j];
  }
}

// From U_all = X [A_0; ...; A_{n-1}]^T (T x R fp32): the token's own
// U_save[t][j] = U_all[t][idx r + j], and sU[t][c] (T x ldo bf16) =
// bf16(s_idx U_all[t][c]) inside the token's block, 0 elsewhere.  A token
// whose index lies outside [0, n) has no block: its U_save row is 0.
__global__ void scatter_adapter_u(const float* __restrict__ U_all, const int32_t* __restrict__ idx, int64_t T,
                                  int r, int n, int ldo, const __grid_constant__ AdapterScales sc,
                                  float* __restrict__ U_save, uint16_t* __restrict__ sU) {
  const int R = n * r;
  const int64_t total = T * ldo;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t t = e / ldo;
    const int c = (int)(e - t * ldo);
    const int a = idx[t];
    const bool mine = c < R && c / r == a;
    const float u = mine ? U_all[t * R + c] : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(mine ? __fmul_rn(sc.s[a], u) : 0.f);
    sU[e] = *reinterpret_cast<const uint16_t*>(&h);
    if (mine) U_save[t * r + (c - a * r)] = u;
    else if ((a < 0 || a >= n) && c < r) U_save[t * r + c] = 0.f;
  }
}

// hi/lo pair of v = s_idx V (hi = bf16(v), lo = bf16(v - hi)) into the token's
// block: out row t has hi in columns [0, half) and lo in [half, 2 half), zero
// outside the block.  V is per token (T x r: the value of block column j is
// V[t][j]) or over all blocks (T x R: V[t][c]).
__global__ void scatter_adapter_hilo(const float* __restrict__ V, int per_token, const int32_t* __restrict__ idx,
                                     int64_t T, int r, int n, int half, const __grid_constant__ AdapterScales sc,
                                     uint16_t* __restrict__ out) {
  const int R = n * r;
  const int64_t total = T * half;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t t = e / half;
    const int c = (int)(e - t * half);
    const int a = idx[t];
    const bool mine = c < R && c / r == a;
    float v = 0.f;
    if (mine) v = __fmul_rn(sc.s[a], per_token ? V[t * r + (c - a * r)] : V[t * R + c]);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(h)));
    out[t * 2 * half + c] = *reinterpret_cast<const uint16_t*>(&h);
    out[t * 2 * half + half + c] = *reinterpret_cast<const uint16_t*>(&l);
  }
}

// fp32 v = s_idx V into the token's block of out (T x R), zero outside it
// (the operands of the few-token CUDA-core adapter gradients).  V is per token
// (T x r) or over all blocks (T x R), as for scatter_adapter_hilo.
__global__ void scatter_adapter_f32(const float* __restrict__ V, int per_token, const int32_t* __restrict__ idx,
                                    int64_t T, int r, int n, const __grid_constant__ AdapterScales sc,
                                    float* __restrict__ out) {
  const int R = n * r;
  const int64_t total = T * R;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t t = e / R;
    const int c = (int)(e - t * R);
    const int a = idx[t];
    const bool mine = c / r == a;
    out[e] = mine ? __fmul_rn(sc.s[a], per_token ? V[t * r + (c - a * r)] : V[t * R + c]) : 0.f;
  }
}

// dBs[i][row][j] = dBcat[row][i r + j]
__global__ void uncat_adapters_db(const float* __restrict__ dBcat, int64_t d, int r, int n, float* __restrict__ dBs) {
  const int R = n * r;
  const int64_t total = d * R;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t row = e / R;
    const int c = (int)(e - row * R);
    const int i = c / r, j = c - i * r;
    dBs[((int64_t)i * d + row) * r + j] = dBcat[e];
  }
}

// Bounded-wait self test: waits on a barrier that nothing completes.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait_suspend(smem_u32(&bar), 0, 100000u)) {
      if (globaltimer_ns() - start > limit_ns) {
        record_status(QLORA_ERR_TIMEOUT);
        break;
      }
    }
  }
}

}  // namespace qlora
