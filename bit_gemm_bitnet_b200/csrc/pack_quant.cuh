// Weight packing and per-token activation quantisation kernels.
#pragma once
#include "common.cuh"

namespace bitnet {

// pack_weights (bitnet-cpu page): code = w + 2, four codes per byte, element
// 4j+i of a row in bits 2i..2i+1 of byte j. One thread per output byte;
// values outside {-1, 0, +1} raise g_pack_bad_value.
__global__ void pack_weights_kernel(uint8_t* __restrict__ out,
                                    const int8_t* __restrict__ w,
                                    int64_t total_bytes) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  unsigned bad = 0;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       j < total_bytes; j += stride) {
    // w is 4-byte aligned and K % 4 == 0, so byte j's four weights are the
    // int32 at element 4j.
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(w) + j);
    uint32_t byte = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int s = static_cast<int8_t>((v >> (8 * i)) & 0xFFu);
      bad |= static_cast<unsigned>(s < -1 || s > 1);
      byte |= (static_cast<uint32_t>(s + 2) & 3u) << (2 * i);
    }
    out[j] = static_cast<uint8_t>(byte);
  }
  if (bad) atomicOr(&g_pack_bad_value, 1u);
}

// |bf16| ordering equals the ordering of the magnitude bits for finite
// values, so the row absmax is a max over (bits & 0x7FFF).
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  uint32_t m = 0;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = max(m, w[i] & 0x7FFFu);
    m = max(m, (w[i] >> 16) & 0x7FFFu);
  }
  return m;
}

// Quantise the 8 bf16 values of v; returns them packed as 8 int8 (uint2),
// natural order.
__device__ __forceinline__ uint2 quant8(const uint4& v, const RowQuant& rq) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int lo = quant_one(bf16_bits_to_f32(w[i] & 0xFFFFu), rq);
    const int hi = quant_one(bf16_bits_to_f32(w[i] >> 16), rq);
    const uint32_t pair = (static_cast<uint32_t>(lo) & 0xFFu) |
                          ((static_cast<uint32_t>(hi) & 0xFFu) << 8);
    o[i >> 1] |= pair << (16 * (i & 1));
  }
  return make_uint2(o[0], o[1]);
}

constexpr int kQuantThreads = 256;

// quantize_activation (bitnet-cpu page), one CTA per row. VPT > 0: the row is
// held in registers (VPT 16-byte vectors per thread, K <= 8 * 256 * VPT);
// VPT == 0: two passes over global memory for longer rows.
template <int VPT>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_rows_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                         const uint16_t* __restrict__ x, int K) {
  __shared__ uint32_t red[kQuantThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  uint2* qrow = reinterpret_cast<uint2*>(xq + m * K);
  const int nvec = K / 8;
  const int tid = threadIdx.x;

  uint4 v[VPT > 0 ? VPT : 1];
  uint32_t mb = 0;
  if constexpr (VPT > 0) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = tid + i * kQuantThreads;
      if (idx < nvec) {
        v[i] = ldg_stream_v4(row + idx);
        mb = max(mb, absmax_bits8(v[i]));
      }
    }
  } else {
    for (int idx = tid; idx < nvec; idx += kQuantThreads)
      mb = max(mb, absmax_bits8(__ldg(row + idx)));
  }
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < kQuantThreads / 32 ? red[tid] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  const RowQuant rq = row_quant(bf16_bits_to_f32(red[0]));
  if constexpr (VPT > 0) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = tid + i * kQuantThreads;
      if (idx < nvec) qrow[idx] = quant8(v[i], rq);
    }
  } else {
    for (int idx = tid; idx < nvec; idx += kQuantThreads)
      qrow[idx] = quant8(__ldg(row + idx), rq);
  }
  if (tid == 0) sa[m] = f32_to_bf16_bits(rq.s);
}

// The same quantiser writing, for the tensor-core GEMM of bitnet_linear, each
// 16-element group of a row transposed 4x4 (element 4t + i at byte 4i + t of
// the group, the order in which the 2-bit planes of a packed weight word come
// out) and the row's sum of codes. GPT > 0: the row is held in registers (GPT
// groups per thread, K <= 16 * 256 * GPT); GPT == 0: two passes.
template <int GPT>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_rows_perm_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                              int32_t* __restrict__ rowsum, const uint16_t* __restrict__ x,
                              int K) {
  __shared__ uint32_t red[kQuantThreads / 32];
  __shared__ int reds[kQuantThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  uint4* qrow = reinterpret_cast<uint4*>(xq + m * K);
  const int ngroups = K / 16;
  const int tid = threadIdx.x;

  uint4 v[GPT > 0 ? GPT : 1][2];
  uint32_t mb = 0;
  if constexpr (GPT > 0) {
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
      const int g = tid + i * kQuantThreads;
      if (g < ngroups) {
        v[i][0] = ldg_stream_v4(row + 2 * g);
        v[i][1] = ldg_stream_v4(row + 2 * g + 1);
        mb = max(mb, max(absmax_bits8(v[i][0]), absmax_bits8(v[i][1])));
      }
    }
  } else {
    for (int g = tid; g < ngroups; g += kQuantThreads)
      mb = max(mb, max(absmax_bits8(__ldg(row + 2 * g)), absmax_bits8(__ldg(row + 2 * g + 1))));
  }
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < kQuantThreads / 32 ? red[tid] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  const RowQuant rq = row_quant(bf16_bits_to_f32(red[0]));
  int sum = 0;
  auto emit = [&](int g, const uint4& a, const uint4& b) {
    const uint2 lo = quant8(a, rq);
    const uint2 hi = quant8(b, rq);
    const uint32_t w0 = lo.x, w1 = lo.y, w2 = hi.x, w3 = hi.y;
    sum += __dp4a(static_cast<int>(w0), 0x01010101, 0) + __dp4a(static_cast<int>(w1), 0x01010101, 0) +
           __dp4a(static_cast<int>(w2), 0x01010101, 0) + __dp4a(static_cast<int>(w3), 0x01010101, 0);
    // 4x4 byte transpose: out word i byte t = in word t byte i
    const uint32_t t0 = __byte_perm(w0, w1, 0x5140u);
    const uint32_t t1 = __byte_perm(w0, w1, 0x7362u);
    const uint32_t t2 = __byte_perm(w2, w3, 0x5140u);
    const uint32_t t3 = __byte_perm(w2, w3, 0x7362u);
    qrow[g] = make_uint4(__byte_perm(t0, t2, 0x5410u), __byte_perm(t0, t2, 0x7632u),
                         __byte_perm(t1, t3, 0x5410u), __byte_perm(t1, t3, 0x7632u));
  };
  if constexpr (GPT > 0) {
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
      const int g = tid + i * kQuantThreads;
      if (g < ngroups) emit(g, v[i][0], v[i][1]);
    }
  } else {
    for (int g = tid; g < ngroups; g += kQuantThreads)
      emit(g, __ldg(row + 2 * g), __ldg(row + 2 * g + 1));
  }
  sum = __reduce_add_sync(0xFFFFFFFFu, sum);
  if ((tid & 31) == 0) reds[tid >> 5] = sum;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kQuantThreads / 32; ++w) t += reds[w];
    rowsum[m] = t;
    sa[m] = f32_to_bf16_bits(rq.s);
  }
}

// ------------------------------------------------ float32 activations

// Row absmax (as fp32 magnitude bits) and the row quantiser of one fp32 row,
// over the CTA; two passes over global memory (K % 4 == 0, 16-byte rows).
__device__ __forceinline__ RowQuant row_quant_f32(const float4* row, int nvec, uint32_t* red) {
  const int tid = threadIdx.x;
  uint32_t mb = 0;
  for (int i = tid; i < nvec; i += kQuantThreads) {
    const float4 v = __ldg(row + i);
    mb = max(mb, max(max(__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu),
                     max(__float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu)));
  }
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  if (tid < 32) {
    uint32_t t = tid < kQuantThreads / 32 ? red[tid] : 0u;
    t = __reduce_max_sync(0xFFFFFFFFu, t);
    if (tid == 0) red[0] = t;
  }
  __syncthreads();
  return row_quant(__uint_as_float(red[0]));
}

// Four fp32 values -> four int8 codes (natural order, one word).
__device__ __forceinline__ uint32_t quant4_f32(const float4& v, const RowQuant& rq) {
  return (static_cast<uint32_t>(quant_one(v.x, rq)) & 0xFFu) |
         ((static_cast<uint32_t>(quant_one(v.y, rq)) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(quant_one(v.z, rq)) & 0xFFu) << 16) |
         (static_cast<uint32_t>(quant_one(v.w, rq)) << 24);
}

// quantize_activation for float32 rows (natural layout), one CTA per row.
__global__ void __launch_bounds__(kQuantThreads)
    quantize_rows_f32_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                             const float* __restrict__ x, int K) {
  __shared__ uint32_t red[kQuantThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const float4* row = reinterpret_cast<const float4*>(x + m * K);
  uint32_t* qrow = reinterpret_cast<uint32_t*>(xq + m * K);
  const int nvec = K / 4;
  const RowQuant rq = row_quant_f32(row, nvec, red);
  for (int i = threadIdx.x; i < nvec; i += kQuantThreads) qrow[i] = quant4_f32(__ldg(row + i), rq);
  if (threadIdx.x == 0) sa[m] = f32_to_bf16_bits(rq.s);
}

// The same with the layout of bitnet_linear's workspace (16-element groups
// transposed 4x4) and the row's code sum, for float32 rows (K % 16 == 0).
__global__ void __launch_bounds__(kQuantThreads)
    quantize_rows_perm_f32_kernel(int8_t* __restrict__ xq, uint16_t* __restrict__ sa,
                                  int32_t* __restrict__ rowsum, const float* __restrict__ x,
                                  int K) {
  __shared__ uint32_t red[kQuantThreads / 32];
  __shared__ int reds[kQuantThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const float4* row = reinterpret_cast<const float4*>(x + m * K);
  uint4* qrow = reinterpret_cast<uint4*>(xq + m * K);
  const int tid = threadIdx.x;
  const RowQuant rq = row_quant_f32(row, K / 4, red);
  int sum = 0;
  for (int g = tid; g < K / 16; g += kQuantThreads) {
    const uint32_t w0 = quant4_f32(__ldg(row + 4 * g), rq);
    const uint32_t w1 = quant4_f32(__ldg(row + 4 * g + 1), rq);
    const uint32_t w2 = quant4_f32(__ldg(row + 4 * g + 2), rq);
    const uint32_t w3 = quant4_f32(__ldg(row + 4 * g + 3), rq);
    sum += __dp4a(static_cast<int>(w0), 0x01010101, 0) + __dp4a(static_cast<int>(w1), 0x01010101, 0) +
           __dp4a(static_cast<int>(w2), 0x01010101, 0) + __dp4a(static_cast<int>(w3), 0x01010101, 0);
    // 4x4 byte transpose: out word i byte t = in word t byte i
    const uint32_t t0 = __byte_perm(w0, w1, 0x5140u);
    const uint32_t t1 = __byte_perm(w0, w1, 0x7362u);
    const uint32_t t2 = __byte_perm(w2, w3, 0x5140u);
    const uint32_t t3 = __byte_perm(w2, w3, 0x7362u);
    qrow[g] = make_uint4(__byte_perm(t0, t2, 0x5410u), __byte_perm(t0, t2, 0x7632u),
                         __byte_perm(t1, t3, 0x5410u), __byte_perm(t1, t3, 0x7632u));
  }
  sum = __reduce_add_sync(0xFFFFFFFFu, sum);
  if ((tid & 31) == 0) reds[tid >> 5] = sum;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kQuantThreads / 32; ++w) t += reds[w];
    rowsum[m] = t;
    sa[m] = f32_to_bf16_bits(rq.s);
  }
}

}  // namespace bitnet
