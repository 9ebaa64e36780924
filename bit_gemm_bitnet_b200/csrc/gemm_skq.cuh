// Fused quantise + ternary GEMV for 8 <= M <= 16 activation rows on the 5th-
// generation tensor cores (the decode GEMV of a few tokens).
//
// The grid and the split-K clusters are those of the few-row GEMM
// (gemm_sk.cuh): one 128-row weight tile per cluster, its K loop split over S
// CTAs. There is no quantised copy of the activations in global memory:
//   1. every CTA reads its K-slice of the bf16 rows x[m, k0:k1] and takes
//      their partial absmax; the cluster combines the S partials through
//      distributed shared memory, so every CTA derives the same per-row scale
//      (scale = absmax / 127 with the absmax clamped at 1e-5, as the
//      bitnet-cpu page's quantize_activation);
//   2. the CTA quantises its slice (round half to even, clamp to +-127) into
//      shared memory, directly in the 128-byte-swizzled K-major layout of the
//      MMA's B operand (16 rows; zeros past K; rows past M are computed but
//      never read back), where it stays for the whole K loop;
//   3. only the packed weights stream through TMA, 512 K per stage (one full
//      128-byte line of each of the tile's 128 rows, 128-byte swizzled),
//      requested before the wait for the previous kernel (they are load-time
//      constants); unpack warps expand them into tensor memory (the A
//      operand, 128 columns per stage) and one thread issues the stage's
//      sixteen tcgen05.mma kind::i8;
//   4. the int32 partials are reduced over the cluster and the epilogue
//      bf16((acc * bf16(scale)) * scale_wt) is applied, as in gemm_sk.cuh.
// Shared memory for the resident activations is 16 x 128 bytes per 128-wide
// K block of the slice, so the host picks S with at most MAX_KB such blocks
// (MAX_KB / 4 stages) per CTA.
#pragma once
#include "common.cuh"
#include "gemm_sk.cuh"

namespace bitnet {
namespace skq {

constexpr int BX = 16;                       // MMA N: activation rows (padded)
constexpr int BW = sk::BW;
constexpr int BK = 128;                      // K per resident activation tile
constexpr int BKS = 512;                     // K per weight stage
constexpr int NUM_THREADS = sk::NUM_THREADS;
constexpr int TMEM_COLS = sk::TMEM_COLS;
constexpr int A_COL0 = 32;                   // A stages right after the 16-column accumulator
constexpr int A_COLS = BKS / 4;              // 128 columns per A stage
// Eight unpack warps share every stage (each half the columns of its 32
// tensor-memory lanes); every warp sees every stage in order, so no barrier
// is ever waited on two phases ahead. Three A stages in tensor memory (stage
// it in it % 3) let the next stages be unpacked while the MMAs run.
constexpr int UNPACK_WARPS = 8;
constexpr int GROUPS = 3;                    // A stages
constexpr int ST = 6;                        // weight stages (96 KB in flight)
constexpr int WP_BYTES = BW * BKS / 4;       // 16 KB per stage
constexpr int XT_BYTES = BX * BK;            // one K block of activations, 2 KB
constexpr int ACT_BUDGET = 96 * 1024;        // resident activations per CTA
constexpr int MAX_KB = ACT_BUDGET / XT_BYTES;  // K blocks per CTA (48)
constexpr int QMAX = 24;                     // activation items per thread (registers)
constexpr int PART_BYTES = BX * BW * 4;      // int32 partial tile, 8 KB
constexpr int HDR_BYTES = 3072;              // barriers, per-row and per-column scalars, per-warp maxima
static_assert(2 * ST + 2 * GROUPS + 4 <= 64, "barriers fit below the per-row scalars");
constexpr int SMEM_BYTES = 1024 + HDR_BYTES + ST * WP_BYTES + ACT_BUDGET + PART_BYTES;
static_assert(SMEM_BYTES > 116 * 1024, "one CTA per SM (each holds all TMEM columns)");
static_assert(SMEM_BYTES <= 232448, "too much shared memory");
static_assert(A_COL0 + GROUPS * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(MAX_KB % 4 == 0, "whole stages of resident activations");

// int32 D; A (weights) and B (activations) signed int8; K-major; N = 16.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(BX >> 3) << 17) |
                            (static_cast<uint32_t>(BW >> 4) << 24);

struct Smem {
  uint8_t* base;  // 1024-aligned
  __device__ uint64_t* bars() const { return reinterpret_cast<uint64_t*>(base); }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + ST + s); }
  __device__ uint32_t unpacked(int a) const { return smem_u32(bars() + 2 * ST + a); }
  __device__ uint32_t afree(int a) const { return smem_u32(bars() + 2 * ST + GROUPS + a); }
  __device__ uint32_t tfull() const { return smem_u32(bars() + 2 * ST + 2 * GROUPS); }
  __device__ uint32_t drain() const { return smem_u32(bars() + 2 * ST + 2 * GROUPS + 1); }
  __device__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 2 * ST + 2 * GROUPS + 2);
  }
  __device__ int* abort_flag() const {
    return reinterpret_cast<int*>(bars() + 2 * ST + 2 * GROUPS + 3);
  }
  // per activation row: this CTA's partial absmax (bf16 magnitude bits),
  // the row's quantiser (s, 1/s) and its bf16-rounded scale as fp32
  __device__ uint32_t* amax() const { return reinterpret_cast<uint32_t*>(base + 512); }
  // per warp and activation row: the warp's partial absmax (16 x 16 words)
  __device__ uint32_t* wmax() const { return reinterpret_cast<uint32_t*>(base + 1024); }
  __device__ float* rq_s() const { return reinterpret_cast<float*>(base + 576); }
  __device__ float* rq_r() const { return reinterpret_cast<float*>(base + 640); }
  __device__ float* saf() const { return reinterpret_cast<float*>(base + 704); }
  // per weight row of the tile: fp32 scale and bf16 bias, for the reduction
  __device__ float* col_sw() const { return reinterpret_cast<float*>(base + 2048); }
  __device__ uint16_t* col_bias() const { return reinterpret_cast<uint16_t*>(base + 2560); }
  __device__ uint8_t* wp(int s) const { return base + HDR_BYTES + s * WP_BYTES; }
  // K block j of the CTA's slice: 16 rows x 128 bytes, 128-byte swizzle
  __device__ uint8_t* xt(int j) const { return base + HDR_BYTES + ST * WP_BYTES + j * XT_BYTES; }
  __device__ int32_t* part() const {
    return reinterpret_cast<int32_t*>(base + HDR_BYTES + ST * WP_BYTES + ACT_BUDGET);
  }
};

// i / d without a division: with magic = ceil(2^32 / d), the high word of
// i * magic is floor(i / d) whenever i * d < 2^32 (here i < 2^16, d < 2^12).
__device__ __forceinline__ int div_magic(int i, uint32_t magic) {
  return static_cast<int>(__umulhi(static_cast<uint32_t>(i), magic));
}

// Byte offset of element (row m, k) of a K block in the 128-byte swizzle
// layout: 8-row atoms of 1024 bytes, 16-byte chunks XOR-ed with the row.
__device__ __forceinline__ int sw128_off(int m, int kk) {
  return (m >> 3) * 1024 + (m & 7) * 128 + ((((kk >> 4) ^ m) & 7) << 4) + (kk & 15);
}

// Grid: (N / BW tiles) x S CTAs, clusters of S consecutive CTAs; 1 <= M <= 16;
// K % 64 == 0; x 16-byte aligned. Outputs bf16 [M, N].
// kAccOut (the accumulator hook): the same kernel storing the int32 sums to
// `out` read as int32 [M, N]; every CTA also writes its slice's codes to
// dbg_q (int8 [M, K], natural order) and the CTAs of the first tile the
// scales to dbg_sa (bf16 [M]).
template <bool kAccOut>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemv_i8_skq_kernel(const __grid_constant__ CUtensorMap tmap_w, void* __restrict__ out,
                       const uint16_t* __restrict__ x, const float* __restrict__ scale_wt,
                       int sw_len, int M, int N, int K, int S,
                       const uint16_t* __restrict__ bias, int8_t* __restrict__ dbg_q,
                       uint16_t* __restrict__ dbg_sa) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int n0 = (blockIdx.x / S) * BW;
  const int kstages = (K + BKS - 1) / BKS;
  const int ks0 = kstages * rank / S, ks1 = kstages * (rank + 1) / S;
  const int k0 = ks0 * BKS;
  volatile int* abort = sm.abort_flag();

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), 1);
    }
    for (int a = 0; a < GROUPS; ++a) {
      mbar_init(sm.unpacked(a), UNPACK_WARPS);
      mbar_init(sm.afree(a), 1);
    }
    mbar_init(sm.tfull(), 1);
    mbar_init(sm.drain(), 1);
    *abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < (NUM_THREADS / 32) * BX; i += NUM_THREADS) sm.wmax()[i] = 0u;
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_w);
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_slot()), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot();
  pdl_launch_dependents();

  // the first weight stages: load-time constants, requested before the wait
  const int pre = min(ST, ks1 - ks0);
  if (tid == 0) {
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(sm.full(i), WP_BYTES);
      tma_load_2d(smem_u32(sm.wp(i)), &tmap_w, sm.full(i), (ks0 + i) * (BKS / 4), n0);
    }
  }
  pdl_wait();  // x may come from the previous kernel

  // ---- 1. partial absmax of this CTA's K-slice, per activation row. Each
  // thread loads all its (row, group) items at once (one memory latency for
  // the whole slice) and keeps them in registers for step 2. A warp's 32
  // consecutive items span at most two rows (a slice has a multiple of 16
  // groups), reduced separately into the warp's own slots.
  const int k1 = min(ks1 * BKS, K);
  const int nq = (k1 - k0) / 4;  // 4-element groups of the slice (K % 64 == 0)
  const int items = M * nq;      // <= NUM_THREADS * QMAX (host)
  const uint32_t magic = static_cast<uint32_t>((0x100000000ull + nq - 1) / nq);
  uint2 v[QMAX];
#pragma unroll
  for (int j = 0; j < QMAX; ++j) {
    const int i = tid + j * NUM_THREADS;
    v[j] = make_uint2(0u, 0u);
    if (i < items) {
      const int m = div_magic(i, magic);
      v[j] = __ldg(reinterpret_cast<const uint2*>(x + static_cast<int64_t>(m) * K + k0) + (i - m * nq));
    }
  }
#pragma unroll
  for (int j = 0; j < QMAX; ++j) {
    const int w0 = warp * 32 + j * NUM_THREADS;  // first item of this warp's window
    if (w0 >= items) break;                      // warp-uniform
    const int i = tid + j * NUM_THREADS;
    const uint32_t mag = max(max(v[j].x & 0x7FFFu, (v[j].x >> 16) & 0x7FFFu),
                             max(v[j].y & 0x7FFFu, (v[j].y >> 16) & 0x7FFFu));
    const int m_lo = div_magic(w0, magic);
    const int m = i < items ? div_magic(i, magic) : m_lo;
    const uint32_t a_lo = __reduce_max_sync(0xFFFFFFFFu, m == m_lo ? mag : 0u);
    const uint32_t a_hi = __reduce_max_sync(0xFFFFFFFFu, m != m_lo ? mag : 0u);
    // this warp's own slots: no two warps update the same word
    if (lane == 0) {
      uint32_t* mine = sm.wmax() + warp * BX;
      mine[m_lo] = max(mine[m_lo], a_lo);
      if (a_hi != 0u) mine[m_lo + 1] = max(mine[m_lo + 1], a_hi);
    }
  }
  __syncthreads();
  if (tid < BX) {
    uint32_t a = 0;
    for (int w = 0; w < NUM_THREADS / 32; ++w) a = max(a, sm.wmax()[w * BX + tid]);
    sm.amax()[tid] = a;
  }
  __syncwarp();
  cluster_sync();  // every CTA's partial absmax is visible to the cluster
  if (tid < BX) {
    float sa = 0.0f, qs = 1.0f, qr = 1.0f;
    if (tid < M) {
      uint32_t a = 0;
      for (int q = 0; q < S; ++q)
        a = max(a, dsmem_ld_u32(smem_u32(sm.amax() + tid), static_cast<uint32_t>(q)));
      const RowQuant rq = row_quant(bf16_bits_to_f32(a));
      qs = rq.s;
      qr = rq.r;
      sa = bf16_bits_to_f32(f32_to_bf16_bits(rq.s));
      if (kAccOut && blockIdx.x < static_cast<unsigned>(S)) dbg_sa[tid] = f32_to_bf16_bits(rq.s);
    }
    sm.rq_s()[tid] = qs;
    sm.rq_r()[tid] = qr;
    sm.saf()[tid] = sa;
  }
  __syncthreads();

  // ---- 2. quantise the registers' items into the resident B tiles; the
  // groups past K of a last, partly filled stage are zeros
#pragma unroll
  for (int j = 0; j < QMAX; ++j) {
    const int i = tid + j * NUM_THREADS;
    if (i < items) {
      const int m = div_magic(i, magic), u = i - m * nq;
      RowQuant rq;
      rq.s = sm.rq_s()[m];
      rq.r = sm.rq_r()[m];
      const uint32_t q0 = static_cast<uint32_t>(quant_one(bf16_bits_to_f32(v[j].x & 0xFFFFu), rq)) & 0xFFu;
      const uint32_t q1 = static_cast<uint32_t>(quant_one(bf16_bits_to_f32(v[j].x >> 16), rq)) & 0xFFu;
      const uint32_t q2 = static_cast<uint32_t>(quant_one(bf16_bits_to_f32(v[j].y & 0xFFFFu), rq)) & 0xFFu;
      const uint32_t q3 = static_cast<uint32_t>(quant_one(bf16_bits_to_f32(v[j].y >> 16), rq)) & 0xFFu;
      const int kk = 4 * u;
      *reinterpret_cast<uint32_t*>(sm.xt(kk / BK) + sw128_off(m, kk % BK)) =
          q0 | (q1 << 8) | (q2 << 16) | (q3 << 24);
      if constexpr (kAccOut)
        *reinterpret_cast<uint32_t*>(dbg_q + static_cast<int64_t>(m) * K + k0 + kk) =
            q0 | (q1 << 8) | (q2 << 16) | (q3 << 24);
    }
  }
  {
    const int span = (ks1 - ks0) * (BKS / 4);  // groups incl. the padding
    const int pad = span - nq;                  // a multiple of 16, below 128
    for (int i = tid; i < M * pad; i += NUM_THREADS) {
      const int m = i / pad, kk = 4 * (nq + i - m * pad);
      *reinterpret_cast<uint32_t*>(sm.xt(kk / BK) + sw128_off(m, kk % BK)) = 0u;
    }
  }
  fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA
  __syncthreads();

  // ---- 3. the K loop: weights streamed, activations resident
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = static_cast<uint32_t>(pre);
      for (int ks = ks0 + pre; ks < ks1; ++ks, ++it) {
        const int s = it % ST;
        const uint32_t ph = (it / ST) & 1u;
        if (!mbar_wait(sm.empty(s), ph ^ 1u, abort)) break;
        mbar_arrive_expect_tx(sm.full(s), WP_BYTES);
        tma_load_2d(smem_u32(sm.wp(s)), &tmap_w, sm.full(s), ks * (BKS / 4), n0);
      }
      const uint32_t first = it > ST ? it - ST : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait_drain(sm.full(j % ST), (j / ST) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int ks = ks0; ks < ks1; ++ks, ++it) {
        const int s = it % ST;
        const int a = static_cast<int>(it % GROUPS);
        if (!mbar_wait(sm.unpacked(a), (it / GROUPS) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // sixteen K = 32 MMAs: A columns a0 + 8i, B the stage's four
        // resident 128-wide activation tiles (+32 bytes per step)
        const uint32_t a0 = tmem_base + static_cast<uint32_t>(A_COL0 + a * A_COLS);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.xt(4 * (ks - ks0) + j)));
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mma_i8_tmem_a(tmem_base, a0 + static_cast<uint32_t>(32 * j + 8 * q),
                          bdesc + 2u * static_cast<uint32_t>(q), kIdesc,
                          (ks > ks0 || j > 0 || q > 0) ? 1u : 0u);
        }
        mma_commit(sm.afree(a));
        mma_commit(sm.empty(s));
      }
      if (ok) mma_commit(sm.tfull());
      mma_commit(sm.drain());
      mbar_wait_drain(sm.drain(), 0u);
    }
  } else if (warp == 2 || warp == 3) {
    // the reduction's per-weight-row scalars, staged while the K loop runs
    for (int i = tid - 64; i < BW; i += 64) {
      const int n = n0 + i;
      sm.col_sw()[i] = (!kAccOut && n < N) ? scale_wt[sw_len == 1 ? 0 : n] : 0.0f;
      sm.col_bias()[i] = (bias != nullptr && n < N) ? bias[n] : static_cast<uint16_t>(0);
    }
  } else if (warp >= 4 && warp < 4 + UNPACK_WARPS) {
    // unpack: every stage, lane r of warp w -> weight row 32 (w % 4) + r and
    // the half h = (w - 4) / 4 of its 128 packed bytes: four 16-byte pieces
    // (the 128-byte swizzle puts piece c at c ^ (r % 8)), each expanded to 16
    // tensor-memory columns of the stage's A stage it % 3
    const int sub = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = sub * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
    uint32_t it = 0;
    for (int ks = ks0; ks < ks1; ++ks, ++it) {
      const int s = it % ST;
      const int a = static_cast<int>(it % GROUPS);
      if (!mbar_wait_warp(sm.full(s), (it / ST) & 1u, abort) ||
          !mbar_wait_warp(sm.afree(a), ((it / GROUPS) & 1u) ^ 1u, abort))
        break;
      const uint8_t* row = sm.wp(s) + r * 128;
      const uint32_t col0 = tmem_base + lane_base + static_cast<uint32_t>(A_COL0 + a * A_COLS);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * half + cc;
        const uint4 p = *reinterpret_cast<const uint4*>(row + (((c ^ r) & 7) << 4));
        uint32_t o[16];
        ts::scaled_of(p.x, o + 0);
        ts::scaled_of(p.y, o + 4);
        ts::scaled_of(p.z, o + 8);
        ts::scaled_of(p.w, o + 12);
        tmem_st_32x32b_x16(col0 + static_cast<uint32_t>(16 * c), o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.unpacked(a));
    }
    if (warp < 8) {
      // accumulator -> shared partial tile [16 activation rows][128 weight rows]
      const int quarter = warp & 3;
      if (mbar_wait_warp(sm.tfull(), 0u, abort)) {
        tc_fence_after();
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16), v);
        tmem_ld_wait();
        int32_t* part = sm.part();
#pragma unroll
        for (int j = 0; j < 16; ++j) part[j * BW + r] = static_cast<int32_t>(v[j]) >> ts::kScaledShift;
      }
    }
  }

  // ---- 4. cluster reduction and epilogue
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // every CTA's partial tile (and the scalars) are in shared memory
  {
    const int r_lo = sk::share_row(rank, S), r_hi = sk::share_row(rank + 1, S);
    const int G = (r_hi - r_lo) / 4;
    const int total = M * G;
    const uint32_t part0 = smem_u32(sm.part());
#pragma unroll 1
    for (int idx = tid; idx < total; idx += NUM_THREADS) {
      const int m = idx / G;
      const int rl = r_lo + 4 * (idx - m * G);
      const int n = n0 + rl;
      if (n >= N) continue;
      const uint32_t addr = part0 + static_cast<uint32_t>((m * BW + rl) * 4);
      uint4 v[sk::MAX_SPLIT];
#pragma unroll
      for (int q = 0; q < sk::MAX_SPLIT; ++q)
        if (q < S) v[q] = dsmem_ld_v4(addr, static_cast<uint32_t>(q));
      int a[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < sk::MAX_SPLIT; ++q)
        if (q < S) {
          a[0] += static_cast<int>(v[q].x);
          a[1] += static_cast<int>(v[q].y);
          a[2] += static_cast<int>(v[q].z);
          a[3] += static_cast<int>(v[q].w);
        }
      if constexpr (kAccOut) {
        int32_t* o = static_cast<int32_t*>(out) + static_cast<int64_t>(m) * N + n;
        if (n + 3 < N && (N & 3) == 0) {
          *reinterpret_cast<int4*>(o) = make_int4(a[0], a[1], a[2], a[3]);
        } else {
          for (int j = 0; j < 4 && n + j < N; ++j) o[j] = a[j];
        }
        continue;
      }
      const float sa = sm.saf()[m];
      uint16_t y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        y[j] = f32_to_bf16_bits(__fmul_rn(__fmul_rn(__int2float_rn(a[j]), sa), sm.col_sw()[rl + j]));
        if (bias != nullptr) y[j] = add_bias_bf16_v(y[j], sm.col_bias()[rl + j]);
      }
      uint16_t* o = static_cast<uint16_t*>(out) + static_cast<int64_t>(m) * N + n;
      if (n + 3 < N && (N & 3) == 0) {
        *reinterpret_cast<uint2*>(o) =
            make_uint2(static_cast<uint32_t>(y[0]) | (static_cast<uint32_t>(y[1]) << 16),
                       static_cast<uint32_t>(y[2]) | (static_cast<uint32_t>(y[3]) << 16));
      } else {
        for (int j = 0; j < 4 && n + j < N; ++j) o[j] = y[j];
      }
    }
  }
  cluster_sync();  // the other CTAs have finished reading this CTA's partial tile

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace skq
}  // namespace bitnet
