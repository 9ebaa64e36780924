// Decode GEMV with fused per-token quantisation (M < 16), and the same kernel
// reading pre-quantised rows (a SIMT fallback for shapes the tensor-core GEMM
// does not take).
//
// The work is bound by streaming the packed weights from HBM once. Layout:
//   * L lanes (8, 16 or 32, chosen so that a lane holds at most 8 chunks of a
//     row) share one weight row; 8 warps per CTA; CTAs are persistent (as
//     many as fit at once) and stride over the rows.
//   * a lane issues all loads of its part of a row at once (16-byte streaming
//     loads, 64 weights each), and the next row's loads before using the
//     current one; the first row is requested before waiting on the previous
//     kernel in the stream (programmatic dependent launch), so small layers
//     have their weights in flight while the activations are quantised.
//   * the quantised activations live in shared memory with every 16-element
//     group transposed 4x4, so that the four 2-bit planes of a packed word,
//     (w >> 2i) & 0x03030303, line up with one activation word each and feed
//     dp4a without any byte shuffling. The codes are used as unsigned values
//     c = w + 2, and sum_k q*w = sum_k q*c - 2 * sum_k q is corrected per row.
//   * partial sums are reduced over the 8 lanes with warp shuffles, and the
//     fp32 scale epilogue writes bf16.
#pragma once
#include "common.cuh"
#include "pack_quant.cuh"

namespace bitnet {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvCPL = 8;           // chunks per lane loaded at once
constexpr int kGemvSmallBytes = 1024;  // per-row scalars before the q rows

struct GemvParams {
  uint16_t* out;          // bf16 [M, N], or
  int32_t* acc_out;       // int32 [M, N] (test hook)
  const uint16_t* x;      // bf16 [M, K] (fused quantisation)
  const int8_t* xq;       // int8 [M, K] (pre-quantised path)
  const uint16_t* sa_in;  // bf16 [M]    (pre-quantised path)
  const uint8_t* wp;      // uint8 [N, K/4]
  const float* sw;
  int sw_len;
  int M, N, K;
  int8_t* dbg_q;          // optional: codes quantised on chip (block 0)
  uint16_t* dbg_sa;       // optional: their scales (block 0)
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

// Load the chunks lane `sub` owns in piece `pc` of weight row `n`:
// chunk c = pc * L * CPL + sub + L * i (i < CPL), zero past the row or N.
template <int L, int WPC>
__device__ __forceinline__ void gemv_load_row(uint32_t (&wb)[kGemvCPL][WPC],
                                              const uint8_t* __restrict__ wp, int n,
                                              int pc, int sub, int N, int R, int KB) {
  const int c0 = pc * L * kGemvCPL + sub;
#pragma unroll
  for (int i = 0; i < kGemvCPL; ++i) {
    const int c = c0 + L * i;
    if (n < N && c < R) {
      const uint8_t* ptr = wp + static_cast<int64_t>(n) * KB + c * (4 * WPC);
      if constexpr (WPC == 4) {
        const uint4 v = ldg_stream_v4(ptr);
        wb[i][0] = v.x; wb[i][1] = v.y; wb[i][2] = v.z; wb[i][3] = v.w;
      } else {
        const uint2 v = ldg_stream_v2(ptr);
        wb[i][0] = v.x; wb[i][1] = v.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < WPC; ++j) wb[i][j] = 0u;
    }
  }
}

// MB: rows of x per CTA (bucket); L: lanes per weight row (8, 16 or 32);
// WPC: 32-bit words per chunk (4: 16-byte chunks, needs K % 64 == 0; 2: 8-byte
// chunks); PREQ: activations come pre-quantised (x_q + scale_act).
template <int MB, int L, int WPC, bool PREQ>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(GemvParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  int* qsum = reinterpret_cast<int*>(smem);                  // [MB]
  float* saf = reinterpret_cast<float*>(smem + 64);          // [MB]
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + 128);   // [warps][MB]
  uint8_t* qs = smem + kGemvSmallBytes;                      // [Mc][K]
  static_assert(kGemvWarps * MB * 4 <= kGemvSmallBytes - 128, "reduction scratch");

  pdl_launch_dependents();

  constexpr int G = 32 / L;                  // weight rows per warp at a time
  constexpr int GPC = kGemvWarps * G;        // weight rows per CTA at a time
  const int K = p.K, N = p.N;
  const int m_base = PREQ ? static_cast<int>(blockIdx.y) * MB : 0;
  const int Mc = PREQ ? min(MB, p.M - m_base) : p.M;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % L;
  const int KB = K / 4;
  const int R = K / (16 * WPC);                            // chunks per row
  const int pieces = (R + L * kGemvCPL - 1) / (L * kGemvCPL);
  const int stride = gridDim.x * GPC;
  // n: this group's row; wrow: the warp's first row, which drives the loop so
  // that all 32 lanes take the same trip count.
  int n = static_cast<int>(blockIdx.x) * GPC + warp * G + lane / L;
  int wrow = static_cast<int>(blockIdx.x) * GPC + warp * G;
  int pc = 0;

  // The first row's weights are requested before waiting for the kernel
  // that produces the activations.
  uint32_t cur[kGemvCPL][WPC];
  gemv_load_row<L, WPC>(cur, p.wp, n, 0, sub, N, R, KB);

  pdl_wait();

  // ---- stage the quantised activations (transposed groups) in smem -------
  const int groups16 = K / 16;
  if constexpr (!PREQ) {
    uint32_t mb[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      mb[m] = 0;
      if (m < Mc) {
        const uint4* row = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * K);
        for (int v = tid; v < K / 8; v += kGemvThreads)
          mb[m] = max(mb[m], absmax_bits8(__ldg(row + v)));
      }
      mb[m] = __reduce_max_sync(0xFFFFFFFFu, mb[m]);
      if (lane == 0) red[warp * MB + m] = mb[m];
    }
    __syncthreads();
    RowQuant rq[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      uint32_t t = 0;
#pragma unroll
      for (int w = 0; w < kGemvWarps; ++w) t = max(t, red[w * MB + m]);
      rq[m] = row_quant(bf16_bits_to_f32(t));
    }
    int qs_part[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      qs_part[m] = 0;
      if (m < Mc) {
        const uint4* row = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * K);
        for (int g = tid; g < groups16; g += kGemvThreads) {
          const uint2 lo = quant8(__ldg(row + 2 * g), rq[m]);
          const uint2 hi = quant8(__ldg(row + 2 * g + 1), rq[m]);
          const uint4 nat = make_uint4(lo.x, lo.y, hi.x, hi.y);
          qs_part[m] += bytesum_s8(nat.x) + bytesum_s8(nat.y) +
                        bytesum_s8(nat.z) + bytesum_s8(nat.w);
          *reinterpret_cast<uint4*>(qs + static_cast<int64_t>(m) * K + 16 * g) =
              transpose16(nat);
          if (p.dbg_q != nullptr && blockIdx.x == 0)
            *reinterpret_cast<uint4*>(p.dbg_q + static_cast<int64_t>(m) * K + 16 * g) = nat;
        }
      }
    }
    __syncthreads();  // red[] reuse
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      const int s = __reduce_add_sync(0xFFFFFFFFu, qs_part[m]);
      if (lane == 0) red[warp * MB + m] = static_cast<uint32_t>(s);
    }
    __syncthreads();
    if (tid < MB) {
      int s = 0;
      for (int w = 0; w < kGemvWarps; ++w) s += static_cast<int>(red[w * MB + tid]);
      qsum[tid] = s;
    }
    // every thread holds the same rq[]; thread 0 publishes the scales
    if (tid == 0) {
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        const uint16_t sb = f32_to_bf16_bits(rq[m].s);
        saf[m] = bf16_bits_to_f32(sb);
        if (p.dbg_sa != nullptr && blockIdx.x == 0 && m < Mc) p.dbg_sa[m] = sb;
      }
    }
  } else {
    int qs_part[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      qs_part[m] = 0;
      if (m < Mc) {
        const uint4* row = reinterpret_cast<const uint4*>(
            p.xq + static_cast<int64_t>(m_base + m) * K);
        for (int g = tid; g < groups16; g += kGemvThreads) {
          const uint4 nat = __ldg(row + g);
          qs_part[m] += bytesum_s8(nat.x) + bytesum_s8(nat.y) +
                        bytesum_s8(nat.z) + bytesum_s8(nat.w);
          *reinterpret_cast<uint4*>(qs + static_cast<int64_t>(m) * K + 16 * g) =
              transpose16(nat);
        }
      }
      const int s = __reduce_add_sync(0xFFFFFFFFu, qs_part[m]);
      if (lane == 0) red[warp * MB + m] = static_cast<uint32_t>(s);
    }
    __syncthreads();
    if (tid < MB) {
      int s = 0;
      for (int w = 0; w < kGemvWarps; ++w) s += static_cast<int>(red[w * MB + tid]);
      qsum[tid] = s;
      // the int32 test hook passes no scales
      saf[tid] = (tid < Mc && p.sa_in != nullptr) ? bf16_bits_to_f32(p.sa_in[m_base + tid]) : 0.0f;
    }
  }
  __syncthreads();

  // ---- stream the weights ------------------------------------------------
  int acc[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) acc[m] = 0;

  // One unit = one piece of one row. `use` holds the current unit; the next
  // unit's loads go into `fill` before `use` is consumed. The two buffers
  // alternate (no register copies, which would wait on the loads in flight).
  uint32_t other[kGemvCPL][WPC];
  auto step = [&](uint32_t (&use)[kGemvCPL][WPC], uint32_t (&fill)[kGemvCPL][WPC]) -> bool {
    int pn = pc + 1, nn = n, wn = wrow;
    const bool row_done = pn == pieces;  // warp-uniform
    if (row_done) {
      pn = 0;
      nn = n + stride;
      wn = wrow + stride;
    }
    if (wn < N) gemv_load_row<L, WPC>(fill, p.wp, nn, pn, sub, N, R, KB);

    const int c0 = pc * L * kGemvCPL + sub;
#pragma unroll
    for (int i = 0; i < kGemvCPL; ++i) {
      const int c = c0 + L * i;
      if (c < R) {
#pragma unroll
        for (int j = 0; j < WPC; ++j) {
          const int g = c * WPC + j;
          const uint32_t w = use[i][j];
          const uint32_t e0 = w & 0x03030303u;
          const uint32_t e1 = (w >> 2) & 0x03030303u;
          const uint32_t e2 = (w >> 4) & 0x03030303u;
          const uint32_t e3 = (w >> 6) & 0x03030303u;
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            if (m < Mc) {
              const uint4 Q = *reinterpret_cast<const uint4*>(qs + static_cast<int64_t>(m) * K + 16 * g);
              int a = acc[m];
              a = dp4a_s32(e0, Q.x, a);
              a = dp4a_s32(e1, Q.y, a);
              a = dp4a_s32(e2, Q.z, a);
              a = dp4a_s32(e3, Q.w, a);
              acc[m] = a;
            }
          }
        }
      }
    }

    if (row_done) {
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        int v = acc[m];
#pragma unroll
        for (int o = 1; o < L; o <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        acc[m] = 0;
        if ((m % L) == sub && m < Mc && n < N) {
          const int a = v - 2 * qsum[m];
          const int64_t o = static_cast<int64_t>(m_base + m) * N + n;
          if (p.acc_out != nullptr) {
            p.acc_out[o] = a;
          } else {
            const float s_w = p.sw[p.sw_len == 1 ? 0 : n];
            const float y = __fmul_rn(__fmul_rn(__int2float_rn(a), saf[m]), s_w);
            p.out[o] = f32_to_bf16_bits(y);
          }
        }
      }
    }
    n = nn;
    wrow = wn;
    pc = pn;
    return wrow < N;
  };

  if (wrow < N) {
    while (step(cur, other) && step(other, cur)) {
    }
  }
}

}  // namespace bitnet
