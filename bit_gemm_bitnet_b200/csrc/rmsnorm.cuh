// RMSNorm fused with the per-token quantiser (BitLinearKernel on the
// bitnet-cpu page runs the module's rms_norm on its input before quantising).
// Per row: var = mean(x^2) with the sum of squares exact (each x^2 of a bf16
// x is exact in fp32, summed as a 128-bit integer in units of 2^-64),
// r = 1 / sqrt(var + eps) (IEEE sqrt and division), y = bf16(x * r),
// z = bf16(g * y); then the quantiser on z. One CTA per row, three passes over
// the row (L2-resident after the first): the sum of squares, the absmax of z,
// the codes (z recomputed).
#pragma once
#include "common.cuh"
#include "pack_quant.cuh"
#include "ternarize.cuh"

namespace bitnet {

__device__ __forceinline__ float rms_z(uint32_t xbits16, uint32_t gbits16, float r) {
  const float y = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(bf16_bits_to_f32(xbits16), r)));
  return bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(bf16_bits_to_f32(gbits16), y)));
}

// Sum over the 2*NW bf16 values packed in `w` of trunc(x^2 * 2^64), exact
// (the definition the slow path below spells out). A bf16 x with exponent
// field b >= 1 is m * 2^(b - 134), m in [128, 255], so trunc(x^2 * 2^64) is
// the integer m^2 * 2^(2b - 204) when b >= 102, and 0 when b < 95. When
// every value is in one of those two classes and the first spans at most 21
// binades below the largest exponent bmax, each term is an integer below
// 2^58 in units of 2^(2 bmax - 246): (x * 2^(155 - bmax))^2, exact in fp32
// (an 8-bit significand squared), converted exactly to 64 bits and summed;
// the sum is shifted into place once. Otherwise each term goes through
// abs_fixed. `ok` is cleared for |x| >= 2^23 and non-finite x.
template <int NW>
__device__ __forceinline__ u128 sumsq_fixed(const uint32_t (&w)[NW], bool* ok) {
  static_assert(NW <= 32, "64 terms below 2^58 each fit in 64 bits");
  uint32_t e[NW];  // both exponent fields of each word
  uint32_t em = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    e[i] = (w[i] >> 7) & 0x00FF00FFu;
    em = __vmaxu2(em, e[i]);
  }
  const uint32_t bmax = max(em & 0xFFFFu, em >> 16);
  if (bmax >= 150u) {  // 2^23 and above, Inf, NaN
    *ok = false;
    return 0;
  }
  const uint32_t lo = bmax > 123u ? bmax - 21u : 102u;
  uint32_t good = 0xFFFFFFFFu;
  uint32_t keep[NW];  // the values, with those below 2^-32 (whose terms are 0) zeroed
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const uint32_t below = __vcmpltu2(e[i], 0x005F005Fu);  // b < 95
    good &= below | __vcmpgeu2(e[i], lo * 0x00010001u);
    keep[i] = w[i] & ~below;
  }
  if (good == 0xFFFFFFFFu) {
    if (bmax < 102u) return 0;  // every value is below 2^-32
    const float sc = __int_as_float(static_cast<int>(282u - bmax) << 23);  // 2^(155 - bmax)
    uint64_t acc = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const float y0 = __fmul_rn(bf16_bits_to_f32(keep[i] & 0xFFFFu), sc);
      const float y1 = __fmul_rn(bf16_bits_to_f32(keep[i] >> 16), sc);
      acc += __float2ull_rz(__fmul_rn(y0, y0)) + __float2ull_rz(__fmul_rn(y1, y1));
    }
    const int e2 = 2 * static_cast<int>(bmax) - 246;
    return e2 >= 0 ? static_cast<u128>(acc) << e2 : static_cast<u128>(acc >> -e2);  // exact: an integer
  }
  u128 s = 0;
#pragma unroll
  for (int i = 0; i < 2 * NW; ++i) {
    const float f = bf16_bits_to_f32((w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
    u128 a = 0;
    abs_fixed(__fmul_rn(f, f), &a);
    s += a;
  }
  return s;
}

enum RmsOut : int {
  kRmsCodes = 0,  // int8 codes in natural order + bf16 scale
  kRmsPerm = 1,   // codes with 16-element groups transposed 4x4 (the tensor-core
                  // GEMM's activation layout) + scale + the row's code sum
  kRmsZ = 2,      // the normalised bf16 row z itself (for the fused GEMV, which
                  // quantises its own input); `xq` is then bf16 [M, K]
};

// One CTA per row; K % 16 == 0.
template <int MODE>
__global__ void __launch_bounds__(kTernThreads)
    rmsnorm_quant_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                         int32_t* __restrict__ rowsum, const uint16_t* __restrict__ x,
                         const uint16_t* __restrict__ g, float eps, int K) {
  __shared__ uint64_t part[2 * (kTernThreads / 32)];
  __shared__ uint32_t red[kTernThreads / 32];
  __shared__ int reds[kTernThreads / 32];
  __shared__ float r_s;
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const int tid = threadIdx.x;
  const uint2* row = reinterpret_cast<const uint2*>(x + m * K);
  const uint2* gw = reinterpret_cast<const uint2*>(g);
  const int nq = K / 4;

  // 1. exact sum of squares
  u128 s = 0;
  bool ok = true;
  for (int i = tid; i < nq; i += kTernThreads) {
    const uint2 v = __ldg(row + i);
    const uint32_t w2[2] = {v.x, v.y};
    s += sumsq_fixed(w2, &ok);
  }
  if (!ok) atomicOr(&g_device_error, kDevErrValue);
  const u128 total = cta_sum(s, part);
  if (tid == 0) r_s = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean_of(total, static_cast<double>(K)), eps)));
  __syncthreads();
  const float r = r_s;

  if constexpr (MODE == kRmsZ) {
    uint2* zrow = reinterpret_cast<uint2*>(xq) + m * nq;
    for (int i = tid; i < nq; i += kTernThreads) {
      const uint2 v = __ldg(row + i), w = __ldg(gw + i);
      const uint32_t z0 = f32_to_bf16_bits(rms_z(v.x & 0xFFFFu, w.x & 0xFFFFu, r));
      const uint32_t z1 = f32_to_bf16_bits(rms_z(v.x >> 16, w.x >> 16, r));
      const uint32_t z2 = f32_to_bf16_bits(rms_z(v.y & 0xFFFFu, w.y & 0xFFFFu, r));
      const uint32_t z3 = f32_to_bf16_bits(rms_z(v.y >> 16, w.y >> 16, r));
      zrow[i] = make_uint2(z0 | (z1 << 16), z2 | (z3 << 16));
    }
    return;
  }

  // 2. absmax of z
  uint32_t mb = 0;
  for (int i = tid; i < nq; i += kTernThreads) {
    const uint2 v = __ldg(row + i), w = __ldg(gw + i);
    mb = max(mb, __float_as_uint(rms_z(v.x & 0xFFFFu, w.x & 0xFFFFu, r)) & 0x7FFFFFFFu);
    mb = max(mb, __float_as_uint(rms_z(v.x >> 16, w.x >> 16, r)) & 0x7FFFFFFFu);
    mb = max(mb, __float_as_uint(rms_z(v.y & 0xFFFFu, w.y & 0xFFFFu, r)) & 0x7FFFFFFFu);
    mb = max(mb, __float_as_uint(rms_z(v.y >> 16, w.y >> 16, r)) & 0x7FFFFFFFu);
  }
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < kTernThreads / 32 ? red[tid] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  const RowQuant rq = row_quant(__uint_as_float(red[0]));

  // 3. the codes of z
  auto codes4 = [&](int i) {
    const uint2 v = __ldg(row + i), w = __ldg(gw + i);
    return quant4_f32(make_float4(rms_z(v.x & 0xFFFFu, w.x & 0xFFFFu, r),
                                  rms_z(v.x >> 16, w.x >> 16, r),
                                  rms_z(v.y & 0xFFFFu, w.y & 0xFFFFu, r),
                                  rms_z(v.y >> 16, w.y >> 16, r)),
                      rq);
  };
  if constexpr (MODE == kRmsPerm) {
    uint4* qrow = reinterpret_cast<uint4*>(xq + m * K);
    int sum = 0;
    for (int gidx = tid; gidx < K / 16; gidx += kTernThreads) {
      const uint32_t w0 = codes4(4 * gidx), w1 = codes4(4 * gidx + 1);
      const uint32_t w2 = codes4(4 * gidx + 2), w3 = codes4(4 * gidx + 3);
      sum += __dp4a(static_cast<int>(w0), 0x01010101, 0) + __dp4a(static_cast<int>(w1), 0x01010101, 0) +
             __dp4a(static_cast<int>(w2), 0x01010101, 0) + __dp4a(static_cast<int>(w3), 0x01010101, 0);
      // 4x4 byte transpose: out word i byte t = in word t byte i
      const uint32_t t0 = __byte_perm(w0, w1, 0x5140u);
      const uint32_t t1 = __byte_perm(w0, w1, 0x7362u);
      const uint32_t t2 = __byte_perm(w2, w3, 0x5140u);
      const uint32_t t3 = __byte_perm(w2, w3, 0x7362u);
      qrow[gidx] = make_uint4(__byte_perm(t0, t2, 0x5410u), __byte_perm(t0, t2, 0x7632u),
                              __byte_perm(t1, t3, 0x5410u), __byte_perm(t1, t3, 0x7632u));
    }
    sum = __reduce_add_sync(0xFFFFFFFFu, sum);
    if ((tid & 31) == 0) reds[tid >> 5] = sum;
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < kTernThreads / 32; ++w) t += reds[w];
      rowsum[m] = t;
    }
  } else {
    uint32_t* qrow = reinterpret_cast<uint32_t*>(xq + m * K);
    for (int i = tid; i < nq; i += kTernThreads) qrow[i] = codes4(i);
  }
  if (tid == 0) sa[m] = f32_to_bf16_bits(rq.s);
}

// The same with the row held in registers: one read of x from HBM. Each
// thread owns the 16-element groups tid, tid + 256, ... (NG of them, K <=
// 4096 * NG); g, a load-time constant like the packed weights, is read
// before the previous kernel on the stream has finished.
template <int MODE, int NG>
__global__ void __launch_bounds__(kTernThreads)
    rmsnorm_quant_reg_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                             int32_t* __restrict__ rowsum, const uint16_t* __restrict__ x,
                             const uint16_t* __restrict__ g, float eps, int K) {
  __shared__ uint64_t part[2 * (kTernThreads / 32)];
  __shared__ uint32_t red[kTernThreads / 32];
  __shared__ float r_s;
  pdl_launch_dependents();
  const int64_t m = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ng = K / 16;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  const uint4* gw = reinterpret_cast<const uint4*>(g);
  uint4 xv[NG][2], gv[NG][2];
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const int gi = tid + j * kTernThreads;
    gv[j][0] = gi < ng ? __ldg(gw + 2 * gi) : make_uint4(0u, 0u, 0u, 0u);
    gv[j][1] = gi < ng ? __ldg(gw + 2 * gi + 1) : make_uint4(0u, 0u, 0u, 0u);
  }
  pdl_wait();
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const int gi = tid + j * kTernThreads;
    xv[j][0] = gi < ng ? __ldg(row + 2 * gi) : make_uint4(0u, 0u, 0u, 0u);
    xv[j][1] = gi < ng ? __ldg(row + 2 * gi + 1) : make_uint4(0u, 0u, 0u, 0u);
  }

  // exact sum of squares (padding groups hold zeros)
  u128 s = 0;
  bool ok = true;
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const uint32_t w8[8] = {xv[j][0].x, xv[j][0].y, xv[j][0].z, xv[j][0].w,
                            xv[j][1].x, xv[j][1].y, xv[j][1].z, xv[j][1].w};
    s += sumsq_fixed(w8, &ok);
  }
  if (!ok) atomicOr(&g_device_error, kDevErrValue);
  const u128 total = cta_sum(s, part);
  if (tid == 0)
    r_s = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean_of(total, static_cast<double>(K)), eps)));
  __syncthreads();
  const float r = r_s;

  // z = bf16(g * bf16(x * r)) in place of x; its absmax as bf16 magnitude bits
  uint32_t mb = 0;
#pragma unroll
  for (int j = 0; j < NG; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t* xw = reinterpret_cast<uint32_t*>(&xv[j][h]);
      const uint32_t* gww = reinterpret_cast<const uint32_t*>(&gv[j][h]);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t z0 = f32_to_bf16_bits(rms_z(xw[t] & 0xFFFFu, gww[t] & 0xFFFFu, r));
        const uint32_t z1 = f32_to_bf16_bits(rms_z(xw[t] >> 16, gww[t] >> 16, r));
        xw[t] = z0 | (z1 << 16);
        mb = max(mb, max(z0 & 0x7FFFu, z1 & 0x7FFFu));
      }
    }

  if constexpr (MODE == kRmsZ) {
    uint4* zrow = reinterpret_cast<uint4*>(xq) + m * (K / 8);
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      const int gi = tid + j * kTernThreads;
      if (gi < ng) {
        zrow[2 * gi] = xv[j][0];
        zrow[2 * gi + 1] = xv[j][1];
      }
    }
    return;
  }

  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if (lane == 0) red[warp] = mb;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < kTernThreads / 32 ? red[tid] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  const RowQuant rq = row_quant(bf16_bits_to_f32(red[0]));

  uint4* qrow = reinterpret_cast<uint4*>(xq + m * K);
  int sum = 0;
#pragma unroll
  for (int j = 0; j < NG; ++j) {
    const int gi = tid + j * kTernThreads;
    if (gi < ng) {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t* zw = reinterpret_cast<const uint32_t*>(&xv[j][h]);
        w[2 * h] = quant4_f32(make_float4(bf16_bits_to_f32(zw[0] & 0xFFFFu), bf16_bits_to_f32(zw[0] >> 16),
                                          bf16_bits_to_f32(zw[1] & 0xFFFFu), bf16_bits_to_f32(zw[1] >> 16)),
                              rq);
        w[2 * h + 1] = quant4_f32(make_float4(bf16_bits_to_f32(zw[2] & 0xFFFFu), bf16_bits_to_f32(zw[2] >> 16),
                                              bf16_bits_to_f32(zw[3] & 0xFFFFu), bf16_bits_to_f32(zw[3] >> 16)),
                                  rq);
      }
      if constexpr (MODE == kRmsPerm) {
        sum += __dp4a(static_cast<int>(w[0]), 0x01010101, 0) + __dp4a(static_cast<int>(w[1]), 0x01010101, 0) +
               __dp4a(static_cast<int>(w[2]), 0x01010101, 0) + __dp4a(static_cast<int>(w[3]), 0x01010101, 0);
        // 4x4 byte transpose: out word i byte t = in word t byte i
        const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140u);
        const uint32_t t1 = __byte_perm(w[0], w[1], 0x7362u);
        const uint32_t t2 = __byte_perm(w[2], w[3], 0x5140u);
        const uint32_t t3 = __byte_perm(w[2], w[3], 0x7362u);
        qrow[gi] = make_uint4(__byte_perm(t0, t2, 0x5410u), __byte_perm(t0, t2, 0x7632u),
                              __byte_perm(t1, t3, 0x5410u), __byte_perm(t1, t3, 0x7632u));
      } else {
        qrow[gi] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  if constexpr (MODE == kRmsPerm) {
    sum = __reduce_add_sync(0xFFFFFFFFu, sum);
    __syncthreads();  // red[0] has been read by every thread
    if (lane == 0) red[warp] = static_cast<uint32_t>(sum);
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < kTernThreads / 32; ++w) t += static_cast<int>(red[w]);
      rowsum[m] = t;
    }
  }
  if (tid == 0) sa[m] = f32_to_bf16_bits(rq.s);
}

}  // namespace bitnet
