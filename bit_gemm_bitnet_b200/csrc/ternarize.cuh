// Absmean ternarisation of float32 weights (the load-time step before
// packing): BitLinear.from_dense on the bitnet-cpu page (one gamma per output
// row, clamped at 1e-8) and BitLinearKernel (one gamma for the tensor,
// clamped at 1e-5):
//   gamma = max(mean |w|, eps), code = clamp(round-half-even(w / gamma), -1, 1),
//   scale = bf16(gamma).
// The mean's sum is exact: |w| * 2^64 truncated toward zero is an integer
// (exact for |w| >= 2^-40; |w| < 2^47 is required), summed in 128 bits, so
// the result does not depend on the order of the additions. Then
// mean = float(double(sum) / count * 2^-64), each operation rounded to
// nearest even.
#pragma once
#include "common.cuh"

namespace bitnet {

typedef unsigned __int128 u128;

__device__ unsigned g_ternarize_bad;  // set when a weight is non-finite or >= 2^47

// |w| * 2^64, truncated toward zero; false for non-finite or |w| >= 2^47.
__device__ __forceinline__ bool abs_fixed(float w, u128* out) {
  const uint32_t bits = __float_as_uint(w) & 0x7FFFFFFFu;
  *out = 0;
  if (bits >= 0x57000000u) return false;  // 2^47 and above, Inf, NaN
  const int e = static_cast<int>(bits >> 23);
  if (e == 0) {  // zero and subnormals: below 2^-126, nothing above 2^-64
    *out = 0;
    return true;
  }
  const uint64_t m = (bits & 0x7FFFFFu) | 0x800000u;  // |w| = m * 2^(e - 150)
  const int sh = e - 86;                                // |w| * 2^64 = m * 2^sh
  if (sh >= 0) *out = static_cast<u128>(m) << sh;
  else if (sh > -64) *out = static_cast<u128>(m >> (-sh));
  else *out = 0;
  return true;
}

// The 128-bit integer rounded to the nearest double, halves to even.
__device__ __forceinline__ double u128_to_double_rn(u128 v) {
  const uint64_t hi = static_cast<uint64_t>(v >> 64), lo = static_cast<uint64_t>(v);
  if (hi == 0) return __ull2double_rn(lo);
  const int top = 127 - __clzll(static_cast<long long>(hi));  // highest set bit
  const int drop = top - 52;                                   // bits below the 53 kept
  const u128 kept = v >> drop;
  const u128 rest = v - (kept << drop);
  const u128 half = static_cast<u128>(1) << (drop - 1);
  uint64_t mant = static_cast<uint64_t>(kept);
  if (rest > half || (rest == half && (mant & 1u))) ++mant;  // may carry to 2^53: still exact
  return ldexp(static_cast<double>(mant), drop);
}

__device__ __forceinline__ float mean_of(u128 sum, double count) {
  return static_cast<float>(ldexp(__ddiv_rn(u128_to_double_rn(sum), count), -64));
}

// Sum of the |w| of the CTA's items, exact (integer additions in any order):
// a butterfly over each warp's 128-bit partial sums (two 64-bit halves with
// the carry), then thread 0 adds the warps' sums. `part` holds 2 words per
// warp.
__device__ __forceinline__ u128 cta_sum(u128 mine, uint64_t* part) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t lo = static_cast<uint64_t>(mine), hi = static_cast<uint64_t>(mine >> 64);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
    const uint64_t ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    const uint64_t nlo = lo + olo;
    hi = hi + ohi + (nlo < lo ? 1u : 0u);
    lo = nlo;
  }
  if (lane == 0) {
    part[2 * warp] = lo;
    part[2 * warp + 1] = hi;
  }
  __syncthreads();
  u128 total = 0;
  if (tid == 0)
    for (int w = 0; w < static_cast<int>(blockDim.x) / 32; ++w)
      total += (static_cast<u128>(part[2 * w + 1]) << 64) | part[2 * w];
  return total;  // valid in thread 0
}

constexpr int kTernThreads = 256;

// The code of one weight: clamp(round-half-even(fl(w / gamma)), -1, 1), which
// only depends on whether |fl(w / gamma)| is below, at or above 1/2. The
// product w * fl(1 / gamma) is within 2^-22 |w / gamma| of the quotient, so it
// decides alone unless it lies within 1e-6 of 1/2; there the exact quotient
// decides.
__device__ __forceinline__ uint32_t ternary1(float x, float gamma, float rgamma) {
  float y = __fmul_rn(x, rgamma);
  if (fabsf(fabsf(y) - 0.5f) < 1e-6f) y = __fdiv_rn(x, gamma);
  const float a = fabsf(y);
  const int r = a > 0.5f ? (y > 0.0f ? 1 : -1) : 0;  // a == 0.5 rounds to 0 (even)
  return static_cast<uint32_t>(r) & 0xFFu;
}

// Four codes of w[0..3] / gamma, packed little-endian.
__device__ __forceinline__ uint32_t ternary4(const float4& v, float gamma, float rgamma) {
  return ternary1(v.x, gamma, rgamma) | (ternary1(v.y, gamma, rgamma) << 8) |
         (ternary1(v.z, gamma, rgamma) << 16) | (ternary1(v.w, gamma, rgamma) << 24);
}

// Sum of trunc(|w| * 2^64) over four values (abs_fixed's terms), exact. With
// e the exponent field of |w| = m * 2^(e - 150) (m < 2^24), a term is the
// integer m * 2^(e - 86) when e >= 86 and 0 when e < 63. When every value is
// in one of those two classes and the first spans at most 38 binades below
// the largest exponent emax, each term is an integer below 2^62 in units of
// 2^(emax - 124): |w| * 2^(188 - emax), exact in fp32. The terms are
// converted exactly, summed in 64 bits and shifted into place once.
// Otherwise each goes through abs_fixed.
__device__ __forceinline__ u128 abs_sum4(const float4& v, bool* ok) {
  const uint32_t a[4] = {__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu,
                         __float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu};
  const uint32_t amax = max(max(a[0], a[1]), max(a[2], a[3]));
  const uint32_t emax = amax >> 23;
  if (amax < 0x57000000u) {  // below 2^47 and finite
    const uint32_t lo = emax > 124u ? emax - 38u : 86u;
    bool good = true;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t e = a[k] >> 23;
      good &= e < 63u || e >= lo;
    }
    if (good) {
      if (emax < 86u) return 0;  // every value below 2^-64
      const float sc = __int_as_float(static_cast<int>(315u - emax) << 23);  // 2^(188 - emax)
      uint64_t acc = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if ((a[k] >> 23) >= 63u) acc += __float2ull_rz(__fmul_rn(__uint_as_float(a[k]), sc));
      const int e2 = static_cast<int>(emax) - 124;
      return e2 >= 0 ? static_cast<u128>(acc) << e2 : static_cast<u128>(acc >> -e2);
    }
  }
  u128 s = 0, t = 0;
  *ok &= abs_fixed(v.x, &t);
  s += t;
  *ok &= abs_fixed(v.y, &t);
  s += t;
  *ok &= abs_fixed(v.z, &t);
  s += t;
  *ok &= abs_fixed(v.w, &t);
  s += t;
  return s;
}

__device__ __forceinline__ u128 row_abs_sum(const float4* row, int nvec, bool* ok) {
  u128 s = 0;
  for (int i = threadIdx.x; i < nvec; i += kTernThreads) s += abs_sum4(__ldg(row + i), ok);
  return s;
}

// One gamma per output row: one CTA per row (K % 4 == 0).
__global__ void __launch_bounds__(kTernThreads)
    ternarize_rows_kernel(int8_t* __restrict__ wt, float* __restrict__ scale,
                          const float* __restrict__ w, int K) {
  __shared__ uint64_t part[2 * (kTernThreads / 32)];
  __shared__ float gamma_s;
  const int64_t n = blockIdx.x;
  const float4* row = reinterpret_cast<const float4*>(w + n * K);
  const int nvec = K / 4;
  bool ok = true;
  const u128 total = cta_sum(row_abs_sum(row, nvec, &ok), part);
  if (!ok) atomicOr(&g_ternarize_bad, 1u);
  if (threadIdx.x == 0) {
    float g = mean_of(total, static_cast<double>(K));
    gamma_s = g < 1e-8f ? 1e-8f : g;
  }
  __syncthreads();
  const float gamma = gamma_s;
  const float rgamma = __fdiv_rn(1.0f, gamma);
  uint32_t* out = reinterpret_cast<uint32_t*>(wt + n * K);
  for (int i = threadIdx.x; i < nvec; i += kTernThreads)
    out[i] = ternary4(__ldg(row + i), gamma, rgamma);
  if (threadIdx.x == 0) scale[n] = bf16_bits_to_f32(f32_to_bf16_bits(gamma));
}

// One gamma for the tensor, step 1: each row's exact sum, kept in the first
// 16 bytes of the row's output (K % 16 == 0).
__global__ void __launch_bounds__(kTernThreads)
    ternarize_rowsum_kernel(int8_t* __restrict__ wt, const float* __restrict__ w, int K) {
  __shared__ uint64_t part[2 * (kTernThreads / 32)];
  const int64_t n = blockIdx.x;
  bool ok = true;
  const u128 total = cta_sum(row_abs_sum(reinterpret_cast<const float4*>(w + n * K), K / 4, &ok),
                             part);
  if (!ok) atomicOr(&g_ternarize_bad, 1u);
  if (threadIdx.x == 0) {
    uint64_t* dst = reinterpret_cast<uint64_t*>(wt + n * K);
    dst[0] = static_cast<uint64_t>(total);
    dst[1] = static_cast<uint64_t>(total >> 64);
  }
}

// Step 2 (one CTA): the tensor's sum, gamma (fp32) into scale[0].
__global__ void __launch_bounds__(kTernThreads)
    ternarize_total_kernel(float* __restrict__ scale, const int8_t* __restrict__ wt, int64_t N,
                           int K) {
  __shared__ uint64_t part[2 * (kTernThreads / 32)];
  u128 s = 0;
  for (int64_t n = threadIdx.x; n < N; n += kTernThreads) {
    const uint64_t* src = reinterpret_cast<const uint64_t*>(wt + n * K);
    s += (static_cast<u128>(src[1]) << 64) | src[0];
  }
  const u128 total = cta_sum(s, part);
  if (threadIdx.x == 0) {
    const float g = mean_of(total, static_cast<double>(N) * static_cast<double>(K));
    scale[0] = g < 1e-5f ? 1e-5f : g;
  }
}

// Step 3: the codes, with gamma from scale[0]; one CTA per row.
__global__ void __launch_bounds__(kTernThreads)
    ternarize_apply_kernel(int8_t* __restrict__ wt, const float* __restrict__ scale,
                           const float* __restrict__ w, int K) {
  const int64_t n = blockIdx.x;
  const float gamma = scale[0];
  const float rgamma = __fdiv_rn(1.0f, gamma);
  const float4* row = reinterpret_cast<const float4*>(w + n * K);
  uint32_t* out = reinterpret_cast<uint32_t*>(wt + n * K);
  for (int i = threadIdx.x; i < K / 4; i += kTernThreads)
    out[i] = ternary4(__ldg(row + i), gamma, rgamma);
}

// Step 4: scale[0] = bf16(gamma), once every row has its codes.
__global__ void ternarize_round_scale_kernel(float* scale) {
  if (threadIdx.x == 0) scale[0] = bf16_bits_to_f32(f32_to_bf16_bits(scale[0]));
}

}  // namespace bitnet
