// Ternary x INT8 GEMM for few activation rows (M <= 256): the 5th-generation
// tensor cores with split-K across a thread-block cluster.
//
// With few activation rows there are too few output tiles to fill the GPU:
// N = 4096 gives 32 tiles of 128 weight rows. So the K loop of a tile is
// split over the S CTAs of one cluster (S <= 8, chosen on the host). Each CTA
// runs the tensor-memory-operand pipeline over its K-slice:
//   - packed weights TMA -> shared memory -> registers (unpack) -> tensor
//     memory (the A operand, 128 weight rows);
//   - activations TMA -> shared memory (the B operand, BX rows, 128-byte
//     swizzle);
//   - int32 accumulators in tensor memory.
// It then stores its int32 partial tile in its own shared memory. After a
// cluster barrier, CTA r of the cluster sums rows [128 r / S, 128 (r+1) / S)
// of the tile over all S partials through distributed shared memory, applies
// the scale epilogue and writes the outputs. The sum is exact (int32), so the
// result does not depend on S.
//
// Warp roles (512 threads, one CTA per SM):
//   warp 0      TMA producer
//   warp 1      tensor-memory owner, MMA issuer (one thread)
//   warps 2-3   stage the epilogue's per-row and per-column scalars
//   warps 4-11  unpack: packed codes -> int8 -> tcgen05.st into an A stage
//               (two groups of four warps, stages in turn); then warps 4-7
//               move the accumulator to the shared-memory partial tile
//   all         the cluster reduction and the epilogue
// Waits on mbarriers are bounded like the other kernels of this library;
// every thread reaches both cluster barriers whatever happens before them.
#pragma once
#include "common.cuh"
#include "gemm_ts.cuh"

namespace bitnet {
namespace sk {

constexpr int BW = 128;                 // weight rows per tile (MMA M)
constexpr int BK = 128;                 // K per stage
constexpr int NUM_THREADS = 512;
constexpr int TMEM_COLS = 512;
constexpr int A_COL0 = 256;             // A stages after the accumulator
constexpr int A_COLS = BK / 4;          // 32 columns per A stage
constexpr int WP_BYTES = BW * BK / 4;   // 4 KB of packed weights per stage
constexpr int BAR_BYTES = 256;
constexpr int MAX_SPLIT = 8;            // CTAs per cluster (portable limit)
// Shared memory is padded to more than half an SM's, so that two CTAs (which
// would both ask for all 512 tensor-memory columns) never share an SM.
constexpr int MIN_SMEM = 120 * 1024;

template <int BX>
struct Cfg {
  static_assert(BX == 16 || BX == 32 || BX == 64 || BX == 128 || BX == 256, "MMA N");
  static constexpr int STAGES = BX == 256 ? 6 : 8;
  static_assert(STAGES % 2 == 0, "stages a multiple of the two unpack groups");
  static constexpr int X_BYTES = BX * BK;
  static constexpr int STAGE_BYTES = X_BYTES + WP_BYTES;
  static constexpr int PART_BYTES = BX * BW * 4;   // int32 partial tile [BX][BW]
  // the reduction's scalars: per activation row fp32 scale and 2 * code sum,
  // per weight row fp32 scale and bf16 bias
  static constexpr int SCAL_BYTES = 2 * BX * 4 + BW * 4 + BW * 2;
  static constexpr int RAW = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + SCAL_BYTES;
  static constexpr int SMEM_BYTES = RAW > MIN_SMEM ? RAW : MIN_SMEM;
  static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(PART_BYTES <= STAGES * STAGE_BYTES, "the partial tile reuses the stages");
  static_assert(A_COL0 + STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(BX <= A_COL0, "accumulator columns");
  static_assert(SMEM_BYTES <= 232448, "too much shared memory");
  // int32 D; B signed int8; A unsigned code planes or signed int8; K-major.
  static constexpr uint32_t kIdescShape = (2u << 4) | (1u << 10) |
                                          (static_cast<uint32_t>(BX >> 3) << 17) |
                                          (static_cast<uint32_t>(BW >> 4) << 24);
};

template <int BX>
struct Smem {
  uint8_t* base;  // 1024-aligned
  static constexpr int ST = Cfg<BX>::STAGES;
  __device__ uint8_t* x(int s) const { return base + s * Cfg<BX>::STAGE_BYTES; }
  __device__ uint8_t* wp(int s) const { return x(s) + Cfg<BX>::X_BYTES; }
  // the int32 partial tile, [BX activation rows][BW weight rows]; written
  // only after the last MMA, when the stages are no longer in use
  __device__ int32_t* part() const { return reinterpret_cast<int32_t*>(base); }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + ST * Cfg<BX>::STAGE_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t unpacked(int s) const { return smem_u32(bars() + ST + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + 2 * ST + s); }
  __device__ uint32_t tfull() const { return smem_u32(bars() + 3 * ST); }
  __device__ uint32_t drain() const { return smem_u32(bars() + 3 * ST + 1); }
  __device__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 3 * ST + 2);
  }
  __device__ int* abort_flag() const { return reinterpret_cast<int*>(bars() + 3 * ST + 3); }
  // the reduction's scalars, staged once per CTA before it
  __device__ float* row_sa() const {
    return reinterpret_cast<float*>(base + ST * Cfg<BX>::STAGE_BYTES + BAR_BYTES);
  }
  __device__ int* row_corr() const { return reinterpret_cast<int*>(row_sa() + BX); }
  __device__ float* col_sw() const { return row_sa() + 2 * BX; }
  __device__ uint16_t* col_bias() const { return reinterpret_cast<uint16_t*>(col_sw() + BW); }
};

// First weight row (within the tile) of CTA `rank`'s share of the reduction:
// multiples of 4, so each share is whole 16-byte groups.
__host__ __device__ constexpr int share_row(int rank, int S) { return 4 * ((32 * rank) / S); }

// kPerm: activations with transposed 16-element groups plus per-row code sums
// (bitnet_linear's workspace); weights enter as unsigned code planes and the
// epilogue subtracts 2 * rowsum[m]. Otherwise natural order, signed weights.
// Grid: (N / BW tiles) x S CTAs, clusters of S consecutive CTAs; M <= BX.
template <int BX, bool kAccOut, bool kPerm>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_sk_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w, void* __restrict__ out,
                      const uint16_t* __restrict__ scale_act,
                      const float* __restrict__ scale_wt, int sw_len,
                      const int32_t* __restrict__ rowsum, int M, int N, int K, int S,
                      const uint16_t* __restrict__ bias) {
  using C = Cfg<BX>;
  constexpr int ST = C::STAGES;
  constexpr uint32_t kIdesc = kPerm ? C::kIdescShape : (C::kIdescShape | (1u << 7));
  constexpr int kShift = kPerm ? 0 : ts::kScaledShift;  // natural order: 64 * w
  extern __shared__ uint8_t smem_raw[];
  Smem<BX> sm;
  sm.base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int tile = blockIdx.x / S;
  const int n0 = tile * BW;
  const int kblocks = (K + BK - 1) / BK;
  const int kb0 = kblocks * rank / S, kb1 = kblocks * (rank + 1) / S;
  volatile int* abort = sm.abort_flag();

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.unpacked(s), 4);
      mbar_init(sm.empty(s), 1);
    }
    mbar_init(sm.tfull(), 1);
    mbar_init(sm.drain(), 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_slot()), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot();

  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // the packed weights are load-time constants: the first stages' weight
      // tiles are requested before waiting for the previous kernel, whose
      // output x_q may be; each stage's barrier expects both tiles' bytes
      const int pre = min(ST, kb1 - kb0);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(sm.full(i), C::STAGE_BYTES);
        tma_load_2d(smem_u32(sm.wp(i)), &tmap_w, sm.full(i), (kb0 + i) * (BK / 4), n0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i)
        tma_load_2d(smem_u32(sm.x(i)), &tmap_x, sm.full(i), (kb0 + i) * BK, 0);
      uint32_t it = static_cast<uint32_t>(pre);
      for (int kb = kb0 + pre; kb < kb1; ++kb, ++it) {
        const int s = it % ST;
        const uint32_t ph = (it / ST) & 1u;
        if (!mbar_wait(sm.empty(s), ph ^ 1u, abort)) break;
        mbar_arrive_expect_tx(sm.full(s), C::STAGE_BYTES);
        tma_load_2d(smem_u32(sm.x(s)), &tmap_x, sm.full(s), kb * BK, 0);
        tma_load_2d(smem_u32(sm.wp(s)), &tmap_w, sm.full(s), kb * (BK / 4), n0);
      }
      const uint32_t first = it > ST ? it - ST : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait_drain(sm.full(j % ST), (j / ST) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      bool ready = false;  // the next block's unpack barrier already completed
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % ST;
        // the unpack warps arrive only after they saw the stage land (full),
        // so this wait also orders the MMA's reads of the stage
        if (!ready && !mbar_wait(sm.unpacked(s), (it / ST) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(A_COL0 + s * A_COLS);
        const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.x(s)));
        const uint32_t nx = it + 1;
        ready = mma4_i8_tmem_a_test(tmem_base, a_tmem, bdesc, kIdesc, kb > kb0 ? 1u : 0u,
                                    sm.unpacked(static_cast<int>(nx % ST)), (nx / ST) & 1u);
        mma_commit(sm.empty(s));
      }
      if (ok) mma_commit(sm.tfull());
      mma_commit(sm.drain());
      mbar_wait_drain(sm.drain(), 0u);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------- epilogue scalars
    // staged while the K loop runs: per activation row the fp32 scale and
    // 2 * code sum, per weight row of the tile the fp32 scale and bf16 bias
    pdl_wait();  // scales and row sums may come from the previous kernel
    for (int m = threadIdx.x - 64; m < BX; m += 64) {
      sm.row_sa()[m] = (!kAccOut && m < M) ? bf16_bits_to_f32(scale_act[m]) : 0.0f;
      sm.row_corr()[m] = (kPerm && m < M) ? 2 * rowsum[m] : 0;
    }
    for (int i = threadIdx.x - 64; i < BW; i += 64) {
      const int n = n0 + i;
      sm.col_sw()[i] = (!kAccOut && n < N) ? scale_wt[sw_len == 1 ? 0 : n] : 0.0f;
      sm.col_bias()[i] = (bias != nullptr && n < N) ? bias[n] : static_cast<uint16_t>(0);
    }
  } else if (warp >= 4 && warp < 12) {
    // -------------------------------------------------------------- unpack
    // Two groups of four warps take the stages in turn, so two stages are
    // unpacked at once (a stage's unpack is a chain of dependent steps: wait,
    // load, unpack, tensor-memory store, wait for the store, arrive). The
    // number of groups divides the number of stages, so a group that waits
    // for a stage's k-th fill is never two fills ahead of the barrier (a
    // parity wait cannot be satisfied by an earlier fill).
    // Warp -> TMEM sub-partition warp % 4 (weight rows 32 * (warp % 4) ...),
    // all 32 columns (128 K elements) of its group's stages.
    const int sub = warp & 3;
    const uint32_t group = static_cast<uint32_t>((warp - 4) >> 2);
    const int r = sub * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
    uint32_t it = 0;
    for (int kb = kb0; kb < kb1; ++kb, ++it) {
      if (it % 2u != group) continue;
      const int s = it % ST;
      const uint32_t ph = (it / ST) & 1u;
      if (!mbar_wait_warp(sm.full(s), ph, abort)) break;
      const uint4 p0 = *reinterpret_cast<const uint4*>(sm.wp(s) + r * 32);
      const uint4 p1 = *reinterpret_cast<const uint4*>(sm.wp(s) + r * 32 + 16);
      uint32_t o[16], o2[16];
      if constexpr (kPerm) {
        ts::planes_of(p0.x, o + 0);
        ts::planes_of(p0.y, o + 4);
        ts::planes_of(p0.z, o + 8);
        ts::planes_of(p0.w, o + 12);
        ts::planes_of(p1.x, o2 + 0);
        ts::planes_of(p1.y, o2 + 4);
        ts::planes_of(p1.z, o2 + 8);
        ts::planes_of(p1.w, o2 + 12);
      } else {
        ts::scaled_of(p0.x, o + 0);
        ts::scaled_of(p0.y, o + 4);
        ts::scaled_of(p0.z, o + 8);
        ts::scaled_of(p0.w, o + 12);
        ts::scaled_of(p1.x, o2 + 0);
        ts::scaled_of(p1.y, o2 + 4);
        ts::scaled_of(p1.z, o2 + 8);
        ts::scaled_of(p1.w, o2 + 12);
      }
      const uint32_t col = tmem_base + lane_base + static_cast<uint32_t>(A_COL0 + s * A_COLS);
      tmem_st_32x32b_x16(col, o);
      tmem_st_32x32b_x16(col + 16u, o2);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.unpacked(s));
    }
    if (warp < 8) {
      // --------------------------------- accumulator -> shared partial tile
      const int quarter = warp & 3;
      if (mbar_wait_warp(sm.tfull(), 0u, abort)) {
        tc_fence_after();
        int32_t* part = sm.part();
#pragma unroll 1
        for (int c = 0; c < BX; c += (BX < 32 ? 16 : 32)) {
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 static_cast<uint32_t>(c);
          if constexpr (BX < 32) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(taddr, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) part[(c + j) * BW + r] = static_cast<int32_t>(v[j]) >> kShift;
          } else {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) part[(c + j) * BW + r] = static_cast<int32_t>(v[j]) >> kShift;
          }
        }
      }
    }
  }

  // --------------------------------------- cluster reduction and epilogue
  pdl_wait();  // the output may still be read by the previous kernel
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // every CTA's partial tile (and the staged scalars) are in shared memory
  {
    const int r_lo = share_row(rank, S), r_hi = share_row(rank + 1, S);
    const int G = (r_hi - r_lo) / 4;  // 16-byte groups per activation row
    const int total = M * G;
    const uint32_t part0 = smem_u32(sm.part());
#pragma unroll 1
    for (int idx = threadIdx.x; idx < total; idx += NUM_THREADS) {
      const int m = idx / G;
      const int rl = r_lo + 4 * (idx - m * G);
      const int n = n0 + rl;
      if (n >= N) continue;
      const uint32_t addr = part0 + static_cast<uint32_t>((m * BW + rl) * 4);
      uint4 v[MAX_SPLIT];
#pragma unroll
      for (int q = 0; q < MAX_SPLIT; ++q)
        if (q < S) v[q] = dsmem_ld_v4(addr, static_cast<uint32_t>(q));
      int a[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < MAX_SPLIT; ++q)
        if (q < S) {
          a[0] += static_cast<int>(v[q].x);
          a[1] += static_cast<int>(v[q].y);
          a[2] += static_cast<int>(v[q].z);
          a[3] += static_cast<int>(v[q].w);
        }
      if constexpr (kPerm) {
        const int corr = sm.row_corr()[m];
#pragma unroll
        for (int j = 0; j < 4; ++j) a[j] -= corr;
      }
      const bool whole = n + 3 < N && (N & 3) == 0;
      if constexpr (kAccOut) {
        int32_t* o = static_cast<int32_t*>(out) + static_cast<int64_t>(m) * N + n;
        if (whole) {
          *reinterpret_cast<int4*>(o) = make_int4(a[0], a[1], a[2], a[3]);
        } else {
          for (int j = 0; j < 4 && n + j < N; ++j) o[j] = a[j];
        }
      } else {
        const float sa = sm.row_sa()[m];
        uint16_t y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          y[j] = f32_to_bf16_bits(__fmul_rn(__fmul_rn(__int2float_rn(a[j]), sa), sm.col_sw()[rl + j]));
          if (bias != nullptr) y[j] = add_bias_bf16_v(y[j], sm.col_bias()[rl + j]);
        }
        uint16_t* o = static_cast<uint16_t*>(out) + static_cast<int64_t>(m) * N + n;
        if (whole) {
          *reinterpret_cast<uint2*>(o) =
              make_uint2(static_cast<uint32_t>(y[0]) | (static_cast<uint32_t>(y[1]) << 16),
                         static_cast<uint32_t>(y[2]) | (static_cast<uint32_t>(y[3]) << 16));
        } else {
          for (int j = 0; j < 4 && n + j < N; ++j) o[j] = y[j];
        }
      }
    }
  }
  cluster_sync();  // the other CTAs have finished reading this CTA's partial tile

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace sk
}  // namespace bitnet
