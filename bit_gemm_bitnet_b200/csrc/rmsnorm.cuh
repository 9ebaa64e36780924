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
    const uint32_t h[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float f = bf16_bits_to_f32(h[j]);
      ok &= fabsf(f) < 8388608.0f;  // 2^23 (false for NaN)
      u128 a = 0;
      ok &= abs_fixed(__fmul_rn(f, f), &a);
      s += a;
    }
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

}  // namespace bitnet
