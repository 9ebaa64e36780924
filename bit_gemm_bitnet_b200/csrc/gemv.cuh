// Decode GEMV with fused per-token quantisation (M < 16), and the same kernel
// reading pre-quantised rows (the SIMT path of bitnet_gemm for shapes the
// tensor-core GEMM does not take).
//
// The work is bound by streaming the packed weights from HBM once:
//   * a producer warp streams blocks of consecutive weight rows (contiguous
//     in memory) into a ring of shared-memory stages with bulk async copies
//     (cp.async.bulk, completion counted on an mbarrier per stage). The first
//     stages are requested before waiting on the previous kernel of the
//     stream (programmatic dependent launch), so a small layer's weights are
//     in flight while its activations are being quantised;
//   * sixteen consumer warps quantise the activation rows into shared memory
//     once per CTA, with every 16-element group transposed 4x4 so that the
//     four 2-bit planes of a packed word, (w >> 2i) & 0x03030303, line up
//     with one activation word each and feed dp4a directly. The codes are
//     used as unsigned c = w + 2 and sum q*w = sum q*c - 2 * sum q;
//   * in a stage, warp w owns RW rows; lane l owns the 32-bit weight words
//     l, l + 32, ... of every row (16 weights each), so each activation word
//     it loads serves RW rows. For one or two activation rows the planes are
//     masked in place, c_i * 4^i = w & (3 << 2i), into four accumulators
//     whose sums are exact multiples of 4^i (recombined with arithmetic
//     shifts): one AND and one dp4a per plane. Row sums are reduced with warp
//     shuffles and the fp32 scale epilogue writes bf16;
//   * CTAs are persistent (as many as fit) and walk the row blocks; loops
//     are kept rolled so the code a launch has to fetch stays small.
#pragma once
#include "common.cuh"
#include "pack_quant.cuh"
#include "rmsnorm.cuh"

namespace bitnet {

constexpr int kGemvMaxConsumerWarps = 16;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvHeaderBytes = 2048;
constexpr int kGemvStageTarget = 40 * 1024;  // bytes per stage (aim)
constexpr int kGemvRingTarget = 160 * 1024;  // bytes of stages per CTA (aim)

#ifdef BITNET_WAIT_TEST
// Failure-path test library only (never in the product library): the ring
// index whose copy CTA 0's producer leaves out, or -1. The consumers waiting
// for that stage then give up their bounded wait.
__device__ int g_wait_test_skip = -1;
#endif

struct GemvParams {
  uint16_t* out;          // bf16 [M, N], or
  int32_t* acc_out;       // int32 [M, N] (test hook)
  const void* x;          // [M, K] bf16, or float32 if x_f32 (fused quantisation)
  const int8_t* xq;       // int8 [M, K] (pre-quantised path)
  const uint16_t* sa_in;  // bf16 [M]    (pre-quantised path)
  const uint8_t* wp;      // uint8 [N, K/4]
  const float* sw;
  int sw_len;
  int M, N, K;
  int rows_per_block;     // CW * RW
  int stages;             // ring depth (<= kGemvMaxStages)
  uint32_t q_bytes;       // shared bytes reserved for the quantised rows
  uint32_t stage_bytes;   // shared bytes per stage (>= rows_per_block * K/4)
  int8_t* dbg_q;          // optional: codes quantised on chip (block 0)
  uint16_t* dbg_sa;       // optional: their scales (block 0)
  int x_f32;              // x holds float32 values
  const uint16_t* bias;   // optional bf16 [N], added to the bf16 output
  const uint16_t* norm_g; // optional bf16 [K]: RMSNorm the rows (weight g) before quantising
  float norm_eps;         // its epsilon
};

// 4x4 byte transpose of a 16-byte group: out word i byte b = in word b byte i.
__device__ __forceinline__ uint4 transpose16(const uint4& a) {
  const uint32_t t0 = prmt(a.x, a.y, 0x5140u);
  const uint32_t t1 = prmt(a.x, a.y, 0x7362u);
  const uint32_t t2 = prmt(a.z, a.w, 0x5140u);
  const uint32_t t3 = prmt(a.z, a.w, 0x7362u);
  return make_uint4(prmt(t0, t2, 0x5410u), prmt(t0, t2, 0x7632u),
                    prmt(t1, t3, 0x5410u), prmt(t1, t3, 0x7632u));
}

__device__ __forceinline__ int bytesum_s8(uint32_t w) {
  return __dp4a(static_cast<int>(w), 0x01010101, 0);
}

// NW words per lane (t0, t0 + 32, ...) of one warp's RW rows against one or
// two activation rows, on four plane accumulators: every shared-memory load is
// issued before the first use, so the warp waits for one round of loads.
// `valid` false (a ragged tail) makes the lane add nothing.
template <int MB, int RW, int NW, bool FULL>
__device__ __forceinline__ void planes_block(int (&acc)[RW][MB][4], const uint32_t* __restrict__ wrow,
                                             int words, const uint8_t* __restrict__ qs, int K,
                                             int Mc, int rows, int t0, bool valid) {
  uint4 Q[NW][MB];
  uint32_t w[NW][RW];
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    const int t = t0 + 32 * j;
#pragma unroll
    for (int m = 0; m < MB; ++m)
      Q[j][m] = (valid && (MB == 1 || m < Mc)) ? *reinterpret_cast<const uint4*>(qs + m * K + 16 * t)
                                               : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < RW; ++r)
      w[j][r] = (valid && (FULL || r < rows)) ? wrow[r * words + t] : 0u;  // zero adds nothing
  }
#pragma unroll
  for (int j = 0; j < NW; ++j)
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const uint32_t v = w[j][r];
      const uint32_t p0 = v & 0x03030303u, p1 = v & 0x0C0C0C0Cu;
      const uint32_t p2 = v & 0x30303030u, p3 = v & 0xC0C0C0C0u;
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        acc[r][m][0] = dp4a_s32(p0, Q[j][m].x, acc[r][m][0]);
        acc[r][m][1] = dp4a_s32(p1, Q[j][m].y, acc[r][m][1]);
        acc[r][m][2] = dp4a_s32(p2, Q[j][m].z, acc[r][m][2]);
        acc[r][m][3] = dp4a_us(p3, Q[j][m].w, acc[r][m][3]);
      }
    }
}

// Four consecutive words per lane (t = base + 4 lane ... + 3) of one warp's RW
// rows: one 128-bit load per row, four 128-bit activation loads (the QUAD
// layout of q_pos), every load issued before the first use.
template <int MB, int RW, bool FULL>
__device__ __forceinline__ void planes_quad(int (&acc)[RW][MB][4], const uint32_t* __restrict__ wrow,
                                            int words, const uint8_t* __restrict__ qs, int K,
                                            int Mc, int rows, int base, int lane) {
  uint4 Q[4][MB];
  uint4 w[RW];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int m = 0; m < MB; ++m)
      Q[j][m] = (MB == 1 || m < Mc)
                    ? *reinterpret_cast<const uint4*>(qs + m * K + 16 * (base + 32 * j + lane))
                    : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int r = 0; r < RW; ++r)
    w[r] = (FULL || r < rows) ? *reinterpret_cast<const uint4*>(wrow + r * words + base + 4 * lane)
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const uint32_t v = j == 0 ? w[r].x : j == 1 ? w[r].y : j == 2 ? w[r].z : w[r].w;
      const uint32_t p0 = v & 0x03030303u, p1 = v & 0x0C0C0C0Cu;
      const uint32_t p2 = v & 0x30303030u, p3 = v & 0xC0C0C0C0u;
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        acc[r][m][0] = dp4a_s32(p0, Q[j][m].x, acc[r][m][0]);
        acc[r][m][1] = dp4a_s32(p1, Q[j][m].y, acc[r][m][1]);
        acc[r][m][2] = dp4a_s32(p2, Q[j][m].z, acc[r][m][2]);
        acc[r][m][3] = dp4a_us(p3, Q[j][m].w, acc[r][m][3]);
      }
    }
}

// Partial dot products of one warp's RW rows of a stage with the quantised
// activation rows, for lane `lane` (words lane, lane + 32, ...).
// PLANES: four plane accumulators per (row, activation row); else one.
template <int MB, int RW, bool PLANES, bool FULL, bool QUAD = false>
__device__ __forceinline__ void gemv_rows(int (&acc)[RW][MB][PLANES ? 4 : 1],
                                          const uint32_t* __restrict__ wrow, int words,
                                          const uint8_t* __restrict__ qs, int K, int Mc,
                                          int rows, int lane) {
  if constexpr (PLANES) {
    // (QUAD) four consecutive words per lane over every whole block of 128
    // words; then two words per lane per iteration while 64 remain, then one
    // word. The loop bounds are warp-uniform.
    int base = 0;
    if constexpr (QUAD) {
#pragma unroll 1
      for (; base + 128 <= words; base += 128)
        planes_quad<MB, RW, FULL>(acc, wrow, words, qs, K, Mc, rows, base, lane);
    }
#pragma unroll 1
    for (; base + 64 <= words; base += 64)
      planes_block<MB, RW, 2, FULL>(acc, wrow, words, qs, K, Mc, rows, base + lane, true);
    if (base + 32 <= words) {
      planes_block<MB, RW, 1, FULL>(acc, wrow, words, qs, K, Mc, rows, base + lane, true);
      base += 32;
    }
    if (base < words)
      planes_block<MB, RW, 1, FULL>(acc, wrow, words, qs, K, Mc, rows, base + lane,
                                    base + lane < words);
  } else {
    // Many activation rows: planes of the warp's rows first, then one
    // activation word at a time (keeps the registers bounded).
#pragma unroll 1
    for (int t = lane; t < words; t += 32) {
      uint32_t e[RW][4];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const uint32_t w = (FULL || r < rows) ? wrow[r * words + t] : 0u;
        e[r][0] = w & 0x03030303u;
        e[r][1] = (w >> 2) & 0x03030303u;
        e[r][2] = (w >> 4) & 0x03030303u;
        e[r][3] = (w >> 6) & 0x03030303u;
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        if (m < Mc) {
          const uint4 Q = *reinterpret_cast<const uint4*>(qs + m * K + 16 * t);
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            int a = acc[r][m][0];
            a = dp4a_s32(e[r][0], Q.x, a);
            a = dp4a_s32(e[r][1], Q.y, a);
            a = dp4a_s32(e[r][2], Q.z, a);
            a = dp4a_s32(e[r][3], Q.w, a);
            acc[r][m][0] = a;
          }
        }
      }
    }
  }
}

// Quantise the Mc activation rows x [Mc, K] (bf16) into shared memory: codes
// with 16-element groups transposed 4x4 (qs), per-row code sums (qsum), the
// bf16-rounded scales as fp32 (saf). All CW consumer warps take part; the
// caller synchronises the consumers (named barrier 1) afterwards. dbg_q /
// dbg_sa, if not null, receive the natural-order codes and the scale bits.
// Four consecutive activations of a row as fp32: bf16 rows are widened
// exactly, float32 rows are read as they are.
__device__ __forceinline__ float4 load_quad(const void* x, bool f32, int64_t row_off, int u) {
  if (f32) return __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + row_off) + u);
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + row_off) + u);
  return make_float4(bf16_bits_to_f32(v.x & 0xFFFFu), bf16_bits_to_f32(v.x >> 16),
                     bf16_bits_to_f32(v.y & 0xFFFFu), bf16_bits_to_f32(v.y >> 16));
}

// Largest magnitude of four fp32 values, as magnitude bits (the order of
// the bits of non-negative floats is the order of their values).
__device__ __forceinline__ uint32_t mag_max4(const float4& v) {
  return max(max(__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu),
             max(__float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu));
}

struct GemvSmem {
  int* qsum;
  float* saf;
  float* rq_s;
  float* rq_r;
  uint32_t* red;
  uint8_t* qs;
};

// Position of 16-byte activation group g in shared memory. With QUAD, the
// groups of every whole block of 128 are permuted so that group 128b + 4l + j
// sits at 128b + 32j + l: lane l's four consecutive groups of a block are then
// read by four conflict-free 128-bit loads (one per j, lanes consecutive).
// Groups after the last whole block keep their place.
template <bool QUAD>
__device__ __forceinline__ int q_pos(int g, int full_end) {
  if constexpr (QUAD) {
    if (g < full_end) return (g & ~127) | ((g & 3) << 5) | ((g >> 2) & 31);
  }
  return g;
}

// The staging of one or two activation rows with at most NQ quads per thread
// (single-problem kernel): every quad is loaded once and kept in registers
// for the quantise pass, and the code sums go to their own slots (no barrier
// to reuse red[]).
// With norm_g, the rows are first RMS-normalised exactly as the norm kernel
// does (rmsnorm.cuh): every CTA derives the same r = 1 / sqrt(mean(x^2) +
// eps) from the exact sum of squares and quantises z = bf16(g * bf16(x * r)).
template <int CW, int MB, int NQ, bool QUAD, bool NORM>
__device__ __forceinline__ void gemv_stage_cached(const GemvSmem& sh, const uint16_t* __restrict__ x,
                                                  int K, int Mc, int8_t* dbg_q, uint16_t* dbg_sa,
                                                  const uint16_t* __restrict__ norm_g,
                                                  float norm_eps) {
  constexpr int kGemvConsumerWarps = CW;
  constexpr int kGemvConsumers = CW * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* qsum = sh.qsum;
  float* saf = sh.saf;
  float* rq_s = sh.rq_s;
  float* rq_r = sh.rq_r;
  uint32_t* red = sh.red;
  uint8_t* qs = sh.qs;
  const int quads = K / 4;
  uint2 v[MB][NQ];
  uint32_t mb[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    const bool live = MB == 1 || m < Mc;
    const uint2* row = reinterpret_cast<const uint2*>(x + static_cast<int64_t>(m) * K);
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const int u = tid + j * kGemvConsumers;
      v[m][j] = (live && u < quads) ? __ldg(row + u) : make_uint2(0u, 0u);
    }
  }
  if constexpr (NORM) {
    // the norm's weights, requested before the sums need the barrier
    const uint2* gw = reinterpret_cast<const uint2*>(norm_g);
    uint2 gv[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const int u = tid + j * kGemvConsumers;
      gv[j] = u < quads ? __ldg(gw + u) : make_uint2(0u, 0u);
    }
    // exact sums of squares: each warp's by butterflies on the two 64-bit
    // halves, one slot pair per warp and row past the reduction scratch
    uint64_t* part = reinterpret_cast<uint64_t*>(red + 256);
    bool ok = true;
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      u128 ss = 0;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const uint32_t w2[2] = {v[m][j].x, v[m][j].y};
        ss += sumsq_fixed(w2, &ok);
      }
      uint64_t lo = static_cast<uint64_t>(ss), hi = static_cast<uint64_t>(ss >> 64);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const uint64_t olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
        const uint64_t ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
        const uint64_t nlo = lo + olo;
        hi = hi + ohi + (nlo < lo ? 1u : 0u);
        lo = nlo;
      }
      if (lane == 0) {
        part[2 * (warp * MB + m)] = lo;
        part[2 * (warp * MB + m) + 1] = hi;
      }
    }
    if (!ok) atomicOr(&g_device_error, kDevErrValue);
    named_barrier_sync(1, kGemvConsumers);
    if (tid < MB) {
      u128 total = 0;
      for (int w = 0; w < kGemvConsumerWarps; ++w)
        total += (static_cast<u128>(part[2 * (w * MB + tid) + 1]) << 64) | part[2 * (w * MB + tid)];
      rq_s[tid] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean_of(total, static_cast<double>(K)), norm_eps)));
    }
    named_barrier_sync(1, kGemvConsumers);
    // z in place of x (padding quads hold zeros in x and g: z = 0)
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const float r = rq_s[m];
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const uint32_t z0 = f32_to_bf16_bits(rms_z(v[m][j].x & 0xFFFFu, gv[j].x & 0xFFFFu, r));
        const uint32_t z1 = f32_to_bf16_bits(rms_z(v[m][j].x >> 16, gv[j].x >> 16, r));
        const uint32_t z2 = f32_to_bf16_bits(rms_z(v[m][j].y & 0xFFFFu, gv[j].y & 0xFFFFu, r));
        const uint32_t z3 = f32_to_bf16_bits(rms_z(v[m][j].y >> 16, gv[j].y >> 16, r));
        v[m][j] = make_uint2(z0 | (z1 << 16), z2 | (z3 << 16));
      }
    }
    // every thread has read r before thread m writes the row's quantiser
    // into rq_s (after the next barrier)
  }
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    mb[m] = 0;
#pragma unroll
    for (int j = 0; j < NQ; ++j)
      mb[m] = max(mb[m], max(max(v[m][j].x & 0x7FFFu, (v[m][j].x >> 16) & 0x7FFFu),
                             max(v[m][j].y & 0x7FFFu, (v[m][j].y >> 16) & 0x7FFFu)));
    mb[m] = __reduce_max_sync(0xFFFFFFFFu, mb[m]);
    if (lane == 0) red[warp * MB + m] = mb[m];
  }
  named_barrier_sync(1, kGemvConsumers);
  if (tid < MB) {
    uint32_t t = 0;
    for (int w = 0; w < kGemvConsumerWarps; ++w) t = max(t, red[w * MB + tid]);
    const RowQuant q = row_quant(bf16_bits_to_f32(t));
    rq_s[tid] = q.s;
    rq_r[tid] = q.r;
    const uint16_t sb = f32_to_bf16_bits(q.s);
    saf[tid] = bf16_bits_to_f32(sb);
    if (dbg_sa != nullptr && tid < Mc) dbg_sa[tid] = sb;
  }
  named_barrier_sync(1, kGemvConsumers);
  uint32_t* red2 = red + kGemvMaxConsumerWarps * MB;  // code sums per warp
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    int part = 0;
    if (MB == 1 || m < Mc) {
      RowQuant rqm;
      rqm.s = rq_s[m];
      rqm.r = rq_r[m];
      uint8_t* qrow = qs + m * K;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const int u = tid + j * kGemvConsumers;
        if (u < quads) {
          const int q0 = quant_one(bf16_bits_to_f32(v[m][j].x & 0xFFFFu), rqm);
          const int q1 = quant_one(bf16_bits_to_f32(v[m][j].x >> 16), rqm);
          const int q2 = quant_one(bf16_bits_to_f32(v[m][j].y & 0xFFFFu), rqm);
          const int q3 = quant_one(bf16_bits_to_f32(v[m][j].y >> 16), rqm);
          part += q0 + q1 + q2 + q3;
          uint8_t* d = qrow + 16 * q_pos<QUAD>(u >> 2, (K / 16) & ~127) + (u & 3);
          d[0] = static_cast<uint8_t>(q0);
          d[4] = static_cast<uint8_t>(q1);
          d[8] = static_cast<uint8_t>(q2);
          d[12] = static_cast<uint8_t>(q3);
          if (dbg_q != nullptr)
            reinterpret_cast<uint32_t*>(dbg_q + static_cast<int64_t>(m) * K)[u] =
                (static_cast<uint32_t>(q0) & 0xFFu) | ((static_cast<uint32_t>(q1) & 0xFFu) << 8) |
                ((static_cast<uint32_t>(q2) & 0xFFu) << 16) | (static_cast<uint32_t>(q3) << 24);
        }
      }
    }
    part = __reduce_add_sync(0xFFFFFFFFu, part);
    if (lane == 0) red2[warp * MB + m] = static_cast<uint32_t>(part);
  }
  named_barrier_sync(1, kGemvConsumers);
  if (tid < MB) {
    int t = 0;
    for (int w = 0; w < kGemvConsumerWarps; ++w) t += static_cast<int>(red2[w * MB + tid]);
    qsum[tid] = t;
  }
}

// CACHE: the single-problem kernel keeps one or two rows' quads in
// registers between the passes (4 or 8 per thread, by K).
template <int CW, int MB, bool QUAD = false, bool CACHE = false, bool NORM = false>
__device__ __forceinline__ void gemv_stage_activations(const GemvSmem& sh, const void* __restrict__ x,
                                                       int K, int Mc, int8_t* dbg_q, uint16_t* dbg_sa,
                                                       bool f32 = false,
                                                       const uint16_t* norm_g = nullptr,
                                                       float norm_eps = 0.0f) {
  constexpr int kGemvConsumerWarps = CW;
  constexpr int kGemvConsumers = CW * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* qsum = sh.qsum;
  float* saf = sh.saf;
  float* rq_s = sh.rq_s;
  float* rq_r = sh.rq_r;
  uint32_t* red = sh.red;
  uint8_t* qs = sh.qs;
  const int quads = K / 4;
  if constexpr (CACHE && MB <= 2) {
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    if (!f32 && quads <= 4 * kGemvConsumers) {
      gemv_stage_cached<CW, MB, 4, QUAD, NORM>(sh, xb, K, Mc, dbg_q, dbg_sa, norm_g, norm_eps);
      return;
    }
    if (!f32 && quads <= 8 * kGemvConsumers) {
      gemv_stage_cached<CW, MB, 8, QUAD, NORM>(sh, xb, K, Mc, dbg_q, dbg_sa, norm_g, norm_eps);
      return;
    }
  }
  // the norm is only fused where the rows stay in registers (the host
  // checks): anything else is reported rather than quantised unnormalised
  if (NORM && tid == 0) atomicOr(&g_device_error, kDevErrValue);
    // absmax of every activation row (as fp32 magnitude bits); each thread
    // owns the 4-element quads tid, tid + 512, ... of a row (loops kept
    // rolled: a small code footprint)
    uint32_t mb[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      mb[m] = 0;
      if (MB == 1 || m < Mc) {
        const int64_t off = static_cast<int64_t>(m) * K;
        // four independent loads in flight per round
#pragma unroll 1
        for (int u0 = tid; u0 < quads; u0 += 4 * kGemvConsumers) {
          float4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int u = u0 + j * kGemvConsumers;
            v[j] = u < quads ? load_quad(x, f32, off, u) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) mb[m] = max(mb[m], mag_max4(v[j]));
        }
      }
      mb[m] = __reduce_max_sync(0xFFFFFFFFu, mb[m]);
      if (lane == 0) red[warp * MB + m] = mb[m];
    }
    named_barrier_sync(1, kGemvConsumers);
    if (tid < MB) {  // one thread per activation row: its quantiser and scale
      uint32_t t = 0;
      for (int w = 0; w < kGemvConsumerWarps; ++w) t = max(t, red[w * MB + tid]);
      const RowQuant q = row_quant(__uint_as_float(t));
      rq_s[tid] = q.s;
      rq_r[tid] = q.r;
      const uint16_t sb = f32_to_bf16_bits(q.s);
      saf[tid] = bf16_bits_to_f32(sb);
      if (dbg_sa != nullptr && tid < Mc) dbg_sa[tid] = sb;
    }
    named_barrier_sync(1, kGemvConsumers);
    // quantise: element 4b + i of 16-group g goes to byte 16g + 4i + b
    int qs_part[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      qs_part[m] = 0;
      if (MB == 1 || m < Mc) {
        RowQuant rqm;
        rqm.s = rq_s[m];
        rqm.r = rq_r[m];
        const int64_t off = static_cast<int64_t>(m) * K;
        uint8_t* qrow = qs + m * K;
#pragma unroll 1
        for (int u = tid; u < quads; u += kGemvConsumers) {
          const float4 v = load_quad(x, f32, off, u);
          const int q0 = quant_one(v.x, rqm);
          const int q1 = quant_one(v.y, rqm);
          const int q2 = quant_one(v.z, rqm);
          const int q3 = quant_one(v.w, rqm);
          qs_part[m] += q0 + q1 + q2 + q3;
          uint8_t* d = qrow + 16 * q_pos<QUAD>(u >> 2, (K / 16) & ~127) + (u & 3);
          d[0] = static_cast<uint8_t>(q0);
          d[4] = static_cast<uint8_t>(q1);
          d[8] = static_cast<uint8_t>(q2);
          d[12] = static_cast<uint8_t>(q3);
          if (dbg_q != nullptr)
            reinterpret_cast<uint32_t*>(dbg_q + static_cast<int64_t>(m) * K)[u] =
                (static_cast<uint32_t>(q0) & 0xFFu) | ((static_cast<uint32_t>(q1) & 0xFFu) << 8) |
                ((static_cast<uint32_t>(q2) & 0xFFu) << 16) | (static_cast<uint32_t>(q3) << 24);
        }
      }
    }
    named_barrier_sync(1, kGemvConsumers);  // red[] reuse
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const int s = __reduce_add_sync(0xFFFFFFFFu, qs_part[m]);
      if (lane == 0) red[warp * MB + m] = static_cast<uint32_t>(s);
    }
    named_barrier_sync(1, kGemvConsumers);
    if (tid < MB) {
      int s = 0;
      for (int w = 0; w < kGemvConsumerWarps; ++w) s += static_cast<int>(red[w * MB + tid]);
      qsum[tid] = s;
    }
}

// Reduce one warp's RW x MB lane partials and write the outputs of rows
// n0 .. n0 + rows - 1: int32 to acc_out if given, else bf16 to out with the
// fp32 epilogue (acc - 2 * qsum[m]) * saf[m] * sw[n or 0].
template <int MB, int RW, bool PLANES>
__device__ __forceinline__ void gemv_reduce_store(const int (&acc)[RW][MB][PLANES ? 4 : 1], int rows,
                                                  int n0, int Mc, int m_base, int N,
                                                  const int* qsum, const float* saf,
                                                  uint16_t* __restrict__ out,
                                                  int32_t* __restrict__ acc_out,
                                                  const float* __restrict__ sw, int sw_len,
                                                  const uint16_t* __restrict__ bias = nullptr) {
  const int lane = threadIdx.x & 31;
  // Reduce the RW x MB lane partials over the warp. One activation row: one
  // warp-wide integer reduction (redux.sync) per value, lane i keeps total i
  // (2 % faster on the decode step). More rows: a butterfly that halves the
  // number of values at each of the first log2(RW * MB) exchanges
  // (reduce-scatter), then plain exchanges for the remaining lane bits
  // (fewer live registers).
  constexpr int V = RW * MB;
  static_assert((V & (V - 1)) == 0 && V <= 32, "V must be a power of two <= 32");
  int vals[V];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      if constexpr (PLANES)
        vals[r * MB + m] = acc[r][m][0] + (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) +
                           (acc[r][m][3] >> 6);
      else
        vals[r * MB + m] = acc[r][m][0];
    }
  int v = 0, idx = 0;
  bool store;
  if constexpr (MB == 1) {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int t = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(vals[i])));
      if (lane == i) v = t;
    }
    idx = lane;
    store = lane < V;
  } else {
#pragma unroll
    for (int h = V / 2, o = 16; h >= 1; h /= 2, o /= 2) {
      const bool hi = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < h; ++i) {
        const int send = hi ? vals[i] : vals[i + h];
        const int keep = hi ? vals[i + h] : vals[i];
        vals[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
      }
      idx += hi ? h : 0;
    }
    v = vals[0];
    constexpr int kDone = V >= 32 ? 32 : V;  // lane bits already summed: log2(V)
#pragma unroll
    for (int o = 32 / kDone / 2; o >= 1; o /= 2) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    // lanes that differ only in the low bits hold the same total; one stores
    store = (lane & (32 / kDone - 1)) == 0;
  }
  if (store) {
    const int r = idx / MB, m = idx % MB;
    if (r < rows && m < Mc) {
      const int n = n0 + r;
      const int a = v - 2 * qsum[m];
      const int64_t o = static_cast<int64_t>(m_base + m) * N + n;
      if (acc_out != nullptr) {
        acc_out[o] = a;
      } else {
        const float s_w = sw[sw_len == 1 ? 0 : n];
        const float y = __fmul_rn(__fmul_rn(__int2float_rn(a), saf[m]), s_w);
        out[o] = add_bias_bf16(f32_to_bf16_bits(y), bias, n);
      }
    }
  }
}

// CW: consumer warps per CTA;
// MB: rows of x per CTA (bucket); RW: weight rows per consumer warp per stage;
// WIDE: K % 64 == 0 (rows 16-byte aligned: one bulk copy per stage),
// otherwise the producer lanes copy the stage in 8-byte pieces;
// PREQ: activations come pre-quantised (x_q + scale_act).
// NORM: the rows are RMS-normalised in the staging (p.norm_g, p.norm_eps).
template <int CW, int MB, int RW, bool WIDE, bool PREQ, bool NORM = false>
__global__ void __launch_bounds__((CW + 1) * 32) gemv_kernel(GemvParams p) {
  constexpr int kGemvConsumerWarps = CW;
  constexpr int kGemvConsumers = CW * 32;
  extern __shared__ __align__(128) uint8_t smem[];
  int* qsum = reinterpret_cast<int*>(smem);                  // [MB]
  float* saf = reinterpret_cast<float*>(smem + 64);          // [MB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 128);  // full[8], empty[8]
  volatile int* abort = reinterpret_cast<volatile int*>(smem + 256);
  float* rq_s = reinterpret_cast<float*>(smem + 320);        // [MB]
  float* rq_r = reinterpret_cast<float*>(smem + 384);        // [MB]
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + 512);   // [16 warps][MB], code sums after
  // (the fused RMSNorm's 128-bit partial sums, [16 warps][MB] pairs of 64-bit
  // words, start at red + 256 words: smem + 1536)
  uint8_t* qs = smem + kGemvHeaderBytes;                     // [Mc][K]
  uint8_t* ring = qs + p.q_bytes;
  static_assert(kGemvMaxConsumerWarps * MB * 4 <= kGemvHeaderBytes - 512, "reduction scratch");
  static_assert(MB > 2 || 1536 + kGemvMaxConsumerWarps * MB * 16 <= kGemvHeaderBytes,
                "the norm's partial sums fit in the header");
  constexpr bool PLANES = MB <= 2;

  const int K = p.K, N = p.N;
  const int KB = K / 4;
  const int words = K / 16;  // 32-bit packed words per row
  const int RPB = p.rows_per_block;
  const int S = p.stages;
  const int nblocks = (N + RPB - 1) / RPB;
  const int m_base = PREQ ? static_cast<int>(blockIdx.y) * MB : 0;
  const int Mc = PREQ ? min(MB, p.M - m_base) : (MB == 1 ? 1 : p.M);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + kGemvMaxStages + s); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), WIDE ? 1u : 32u);
      mbar_init(empty(s), kGemvConsumerWarps);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------------------ producer
    // Weights do not depend on the previous kernel: no griddepcontrol.wait.
#ifdef BITNET_WAIT_TEST
    const int skip = blockIdx.x == 0 ? g_wait_test_skip : -1;
#endif
    uint32_t it = 0;
    for (int b = blockIdx.x; b < nblocks; b += gridDim.x, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1u;
      if (!mbar_wait(empty(s), ph ^ 1u, abort)) break;
#ifdef BITNET_WAIT_TEST
      if (static_cast<int>(it) == skip) continue;  // this stage is never filled
#endif
      const int n0 = b * RPB;
      const int rows = min(RPB, N - n0);
      const uint8_t* src = p.wp + static_cast<int64_t>(n0) * KB;
      uint8_t* dst = ring + static_cast<size_t>(s) * p.stage_bytes;
      if constexpr (WIDE) {
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(rows) * KB;
          mbar_arrive_expect_tx(full(s), bytes);
          bulk_load(smem_u32(dst), src, bytes, full(s));
        }
      } else {
        const int pieces = rows * (KB / 8);
        for (int i = lane; i < pieces; i += 32) cp_async_8(smem_u32(dst + 8 * i), src + 8 * i);
        cp_async_arrive_noinc(full(s));
      }
    }
    // drain: every copy issued has landed before the CTA may exit
    const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0u;
    for (uint32_t j = first; j < it; ++j) {
#ifdef BITNET_WAIT_TEST
      if (static_cast<int>(j) == skip) continue;  // nothing was requested there
#endif
      mbar_wait_drain(full(j % S), (j / S) & 1u);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  if constexpr (!PREQ) {
    // Warm L2 with the activation rows before waiting for their producer.
    // L2 is the point of coherence, so a line fetched early is updated by any
    // later write; the loads that use the values come after the wait.
    const char* xb = reinterpret_cast<const char*>(p.x);
    const int64_t xbytes = static_cast<int64_t>(Mc) * K * (p.x_f32 ? 4 : 2);
    for (int64_t off = static_cast<int64_t>(tid) * 128; off < xbytes; off += kGemvConsumers * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(xb + off));
  }
  pdl_wait();  // the activations may come from the previous kernel
  const int groups16 = K / 16;
  if constexpr (!PREQ) {
    gemv_stage_activations<CW, MB, false, true, NORM>(GemvSmem{qsum, saf, rq_s, rq_r, red, qs}, p.x,
                                   K, Mc, blockIdx.x == 0 ? p.dbg_q : nullptr,
                                   blockIdx.x == 0 ? p.dbg_sa : nullptr, p.x_f32 != 0,
                                   p.norm_g, p.norm_eps);
  } else {
    int qs_part[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      qs_part[m] = 0;
      if (m < Mc) {
        const uint4* row = reinterpret_cast<const uint4*>(p.xq + static_cast<int64_t>(m_base + m) * K);
#pragma unroll 1
        for (int g = tid; g < groups16; g += kGemvConsumers) {
          const uint4 nat = __ldg(row + g);
          qs_part[m] += bytesum_s8(nat.x) + bytesum_s8(nat.y) + bytesum_s8(nat.z) +
                        bytesum_s8(nat.w);
          *reinterpret_cast<uint4*>(qs + m * K + 16 * g) = transpose16(nat);
        }
      }
      const int s = __reduce_add_sync(0xFFFFFFFFu, qs_part[m]);
      if (lane == 0) red[warp * MB + m] = static_cast<uint32_t>(s);
    }
    named_barrier_sync(1, kGemvConsumers);
    if (tid < MB) {
      int s = 0;
      for (int w = 0; w < kGemvConsumerWarps; ++w) s += static_cast<int>(red[w * MB + tid]);
      qsum[tid] = s;
      // the int32 test hook passes no scales
      saf[tid] = (tid < Mc && p.sa_in != nullptr) ? bf16_bits_to_f32(p.sa_in[m_base + tid]) : 0.0f;
    }
  }
  named_barrier_sync(1, kGemvConsumers);

  uint32_t it = 0;
  for (int b = blockIdx.x; b < nblocks; b += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t ph = (it / S) & 1u;
    if (!mbar_wait(full(s), ph, abort)) break;
    const uint8_t* stage = ring + static_cast<size_t>(s) * p.stage_bytes;
    const int r0 = warp * RW;  // this warp's first row in the block
    const int n0 = b * RPB + r0;
    int rows = min(RW, N - n0);
    if (rows < 0) rows = 0;

    int acc[RW][MB][PLANES ? 4 : 1];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m)
#pragma unroll
        for (int i = 0; i < (PLANES ? 4 : 1); ++i) acc[r][m][i] = 0;

    const uint32_t* wrow = reinterpret_cast<const uint32_t*>(stage + static_cast<size_t>(r0) * KB);
    if (rows == RW)
      gemv_rows<MB, RW, PLANES, true>(acc, wrow, words, qs, K, Mc, rows, lane);
    else if (rows > 0)
      gemv_rows<MB, RW, PLANES, false>(acc, wrow, words, qs, K, Mc, rows, lane);
    // the stage's shared memory may be refilled once every warp is done
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));

    gemv_reduce_store<MB, RW, PLANES>(acc, rows, n0, Mc, m_base, N, qsum, saf, p.out, p.acc_out,
                                      p.sw, p.sw_len, p.bias);
  }
}

}  // namespace bitnet
