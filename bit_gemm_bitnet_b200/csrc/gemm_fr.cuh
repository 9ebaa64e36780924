// Ternary x INT8 GEMM for a few activation rows (16 <= M <= 128 after
// padding): tensor-core tiles of 128 weight rows, K streamed in stages of
// 512, the K loop split over the S CTAs of a thread-block cluster only where
// the GPU would otherwise sit idle.
//
// Per stage a CTA receives 16 KB of packed weights (128 rows x 128 bytes:
// one full 128-byte line of every row, 128-byte swizzled, so both the copy
// and the unpacking warps' shared-memory reads run at full width) and the
// activation tile (BX rows x 512 bytes as four 128-byte-swizzled sub-tiles,
// the MMA's B operand). Unpack warps expand the packed codes into tensor
// memory (the MMA's A operand, 128 columns per stage) and one thread issues
// the stage's sixteen tcgen05.mma.kind::i8 (M = 128 weight rows, N = BX, K =
// 32 each) into an int32 accumulator in tensor memory.
//
// With S = 1 (enough weight tiles to fill the GPU) the accumulator goes
// straight to the scale epilogue. With S > 1 each CTA stores its int32
// partial tile in its own shared memory, and after a cluster barrier CTA r
// sums rows [128 r / S, 128 (r + 1) / S) of the tile over the S partials
// through distributed shared memory and writes them (exact: the result does
// not depend on S).
//
// Warp roles (512 threads, one CTA per SM):
//   warp 0      TMA producer
//   warp 1      tensor-memory owner, MMA issuer (one thread)
//   warps 2-3   stage the epilogue's per-row and per-column scalars
//   warps 4-11  unpack: every stage, each warp half the columns of its
//               tensor-memory lanes 32 * (warp % 4) ..; then each moves half
//               the accumulator columns of those lanes out
//   all         the reduction (S > 1) and the epilogue
// Every wait is bounded; every thread reaches both cluster barriers.
#pragma once
#include "common.cuh"
#include "gemm_ts.cuh"

namespace bitnet {
namespace fr {

constexpr int BW = 128;                  // weight rows per tile (MMA M)
constexpr int BKS = 512;                 // K per stage
constexpr int WP_BYTES = BW * BKS / 4;   // 16 KB of packed weights per stage
constexpr int NUM_THREADS = 512;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 128;            // accumulator columns reserved (BX <= 128)
constexpr int A_COLS = BKS / 4;          // 128 columns per A stage
// Eight unpack warps share every stage: warp w expands columns
// [64 (w / 4), 64 (w / 4) + 64) of tensor-memory lanes 32 (w % 4) .., half of
// each row's 128 packed bytes, so a stage is unpacked in half the time one
// warp per row would take. Every warp sees every stage in order, so no
// barrier is ever waited on two phases ahead. Three A stages in tensor
// memory (stage it in it % 3) let the next stages be unpacked while the MMAs
// of stage it run.
constexpr int UNPACK_WARPS = 8;
constexpr int A_STAGES = 3;
constexpr int BAR_BYTES = 256;
// per activation row: fp32 scale, 2 * code sum; per weight row: fp32 scale,
// bf16 bias
constexpr int SCAL_BYTES = 3 * 128 * 4 + 128 * 2;
constexpr int MAX_SPLIT = 8;
constexpr int SMEM_CAP = 225 * 1024;
// Shared memory is padded to more than half an SM's, so that two CTAs (which
// would both ask for all 512 tensor-memory columns) never share an SM.
constexpr int MIN_SMEM = 120 * 1024;

template <int BX>
struct Cfg {
  static_assert(BX == 16 || BX == 32 || BX == 64 || BX == 128, "MMA N");
  static constexpr int X_SUB = BX * 128;            // one 128-byte-wide activation sub-tile
  static constexpr int X_BYTES = 4 * X_SUB;         // BX rows x 512 K
  static constexpr int STAGE_BYTES = WP_BYTES + X_BYTES;
  static constexpr int PART_BYTES = BX * BW * 4;    // int32 partial tile [BX][BW]
  static constexpr int ST0 = (SMEM_CAP - 1024 - BAR_BYTES - SCAL_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = ST0 >= 4 ? 4 : 2;
  static constexpr int RAW = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + SCAL_BYTES;
  static constexpr int SMEM_BYTES = RAW > MIN_SMEM ? RAW : MIN_SMEM;
  static_assert(STAGES >= 2, "at least two stages");
  static_assert(PART_BYTES <= STAGES * STAGE_BYTES, "the partial tile reuses the stages");
  static_assert(8 * 32 * 32 * 4 <= STAGES * STAGE_BYTES, "the epilogue patches reuse the stages");
  static_assert(STAGE_BYTES % 1024 == 0 && X_SUB % 1024 == 0, "1024-byte alignment");
  static_assert(ACC_COLS + A_STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
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
  __device__ uint8_t* wp(int s) const { return base + s * Cfg<BX>::STAGE_BYTES; }
  __device__ uint8_t* x(int s) const { return wp(s) + WP_BYTES; }
  __device__ int32_t* part() const { return reinterpret_cast<int32_t*>(base); }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + ST * Cfg<BX>::STAGE_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + ST + s); }
  __device__ uint32_t unpacked(int a) const { return smem_u32(bars() + 2 * ST + a); }
  __device__ uint32_t afree(int a) const { return smem_u32(bars() + 2 * ST + A_STAGES + a); }
  __device__ uint32_t tfull() const { return smem_u32(bars() + 2 * ST + 2 * A_STAGES); }
  __device__ uint32_t drain() const { return smem_u32(bars() + 2 * ST + 2 * A_STAGES + 1); }
  __device__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 2 * ST + 2 * A_STAGES + 2);
  }
  __device__ int* abort_flag() const {
    return reinterpret_cast<int*>(bars() + 2 * ST + 2 * A_STAGES + 3);
  }
  // the epilogue's per-activation-row scalars, staged once per CTA
  __device__ float* row_sa() const {
    return reinterpret_cast<float*>(base + ST * Cfg<BX>::STAGE_BYTES + BAR_BYTES);
  }
  __device__ int* row_corr() const { return reinterpret_cast<int*>(row_sa() + 128); }
  // the reduction's per-weight-row scalars (S > 1), staged once per CTA
  __device__ float* col_sw() const { return row_sa() + 256; }
  __device__ uint16_t* col_bias() const { return reinterpret_cast<uint16_t*>(row_sa() + 384); }
};

// First weight row (within the tile) of CTA `rank`'s share of the reduction:
// multiples of 4, so each share is whole 16-byte groups.
__host__ __device__ constexpr int share_row(int rank, int S) { return 4 * ((32 * rank) / S); }

// The sixteen K = 32 MMAs of one 512-wide stage: A from tensor memory
// (columns a + 8j), B the stage's four activation sub-tiles (descriptor of
// sub-tile j / 4 plus 32 bytes per step inside its swizzle rows).
template <int BX>
__device__ __forceinline__ void mma_stage(uint32_t d_tmem, uint32_t a_tmem, uint32_t x_smem,
                                          uint32_t idesc, bool first) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint64_t bdesc = smem_desc_sw128(x_smem + static_cast<uint32_t>(j * Cfg<BX>::X_SUB));
    mma_i8_tmem_a(d_tmem, a_tmem + static_cast<uint32_t>(32 * j), bdesc, idesc,
                  (first && j == 0) ? 0u : 1u);
    mma_i8_tmem_a(d_tmem, a_tmem + static_cast<uint32_t>(32 * j + 8), bdesc + 2u, idesc, 1u);
    mma_i8_tmem_a(d_tmem, a_tmem + static_cast<uint32_t>(32 * j + 16), bdesc + 4u, idesc, 1u);
    mma_i8_tmem_a(d_tmem, a_tmem + static_cast<uint32_t>(32 * j + 24), bdesc + 6u, idesc, 1u);
  }
}

// kPerm: activations with transposed 16-element groups plus per-row code
// sums (bitnet_linear's workspace); weights enter as unsigned code planes and
// the epilogue subtracts 2 * rowsum[m]. Otherwise natural order: the weights
// enter as 64 * w (signed), and the sums leave the accumulator shifted right
// by 6. kAccOut: int32 sums to `out` instead of the bf16 epilogue.
// Grid: (N / BW tiles) x S CTAs, clusters of S consecutive CTAs; M <= BX.
template <int BX, bool kAccOut, bool kPerm>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_fr_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w, void* __restrict__ out,
                      const uint16_t* __restrict__ scale_act,
                      const float* __restrict__ scale_wt, int sw_len,
                      const int32_t* __restrict__ rowsum, int M, int N, int K, int S,
                      const uint16_t* __restrict__ bias) {
  using C = Cfg<BX>;
  constexpr int ST = C::STAGES;
  constexpr uint32_t kIdesc = kPerm ? C::kIdescShape : (C::kIdescShape | (1u << 7));
  constexpr int kShift = kPerm ? 0 : ts::kScaledShift;
  extern __shared__ uint8_t smem_raw[];
  Smem<BX> sm;
  sm.base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int tile = blockIdx.x / S;
  const int n0 = tile * BW;
  const int kblocks = (K + BKS - 1) / BKS;
  const int kb0 = kblocks * rank / S, kb1 = kblocks * (rank + 1) / S;
  // Each tile walks its K-slice starting at its own stage (the int32 sum is
  // exact in any order): every tile's CTA reads the same activation tile, and
  // staggered starts spread those reads over the L2 instead of sending every
  // CTA to the same lines at once.
  const int nkb = kb1 - kb0;
  const int rot = nkb > 0 ? tile % nkb : 0;
  auto kb_of = [&](uint32_t it) { return kb0 + static_cast<int>((it + rot) % nkb); };
  volatile int* abort = sm.abort_flag();

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), 1);  // the stage's MMAs have completed
    }
    for (int a = 0; a < A_STAGES; ++a) {
      mbar_init(sm.unpacked(a), UNPACK_WARPS);
      mbar_init(sm.afree(a), 1);
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
      // output the activations may be; each stage's barrier expects both
      const int pre = min(ST, nkb);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(sm.full(i), C::STAGE_BYTES);
        tma_load_2d(smem_u32(sm.wp(i)), &tmap_w, sm.full(i), kb_of(i) * (BKS / 4), n0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d(smem_u32(sm.x(i) + j * C::X_SUB), &tmap_x, sm.full(i),
                      kb_of(i) * BKS + 128 * j, 0);
      uint32_t it = static_cast<uint32_t>(pre);
      for (; it < static_cast<uint32_t>(nkb); ++it) {
        const int s = it % ST;
        const int kb = kb_of(it);
        const uint32_t ph = (it / ST) & 1u;
        if (!mbar_wait(sm.empty(s), ph ^ 1u, abort)) break;
        mbar_arrive_expect_tx(sm.full(s), C::STAGE_BYTES);
        tma_load_2d(smem_u32(sm.wp(s)), &tmap_w, sm.full(s), kb * (BKS / 4), n0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d(smem_u32(sm.x(s) + j * C::X_SUB), &tmap_x, sm.full(s), kb * BKS + 128 * j, 0);
      }
      const uint32_t first = it > ST ? it - ST : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait_drain(sm.full(j % ST), (j / ST) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (uint32_t it = 0; it < static_cast<uint32_t>(nkb); ++it) {
        const int s = it % ST;
        const int a = static_cast<int>(it % A_STAGES);
        // the unpack warps arrive only after they saw the stage land (full),
        // so this wait also orders the MMA's reads of the activation tile
        if (!mbar_wait(sm.unpacked(a), (it / A_STAGES) & 1u, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_stage<BX>(tmem_base, tmem_base + static_cast<uint32_t>(ACC_COLS + a * A_COLS),
                      smem_u32(sm.x(s)), kIdesc, it == 0);
        mma_commit(sm.afree(a));
        mma_commit(sm.empty(s));  // the activation tile may be refilled
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
    if (S == 1) named_barrier_sync(2, 320);  // warps 2-11
  } else if (warp >= 4 && warp < 4 + UNPACK_WARPS) {
    // -------------------------------------------------------------- unpack
    // Lane r of warp w owns weight row 32 * (w % 4) + r and the half
    // h = (w - 4) / 4 of its 128 packed bytes: four 16-byte pieces (64
    // weights each; the 128-byte swizzle puts piece c at c ^ (r % 8)), each
    // expanded to 16 tensor-memory columns of the stage's A stage it % 3.
    const int sub = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = sub * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
    bool ok = true;
    for (uint32_t it = 0; it < static_cast<uint32_t>(nkb); ++it) {
      const int s = it % ST;
      const int a = static_cast<int>(it % A_STAGES);
      if (!mbar_wait_warp(sm.full(s), (it / ST) & 1u, abort) ||
          !mbar_wait_warp(sm.afree(a), ((it / A_STAGES) & 1u) ^ 1u, abort)) {
        ok = false;
        break;
      }
      const uint8_t* row = sm.wp(s) + r * 128;
      const uint32_t col0 = tmem_base + lane_base + static_cast<uint32_t>(ACC_COLS + a * A_COLS);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * half + cc;
        const uint4 p = *reinterpret_cast<const uint4*>(row + (((c ^ r) & 7) << 4));
        uint32_t o[16];
        if constexpr (kPerm) {
          ts::planes_of(p.x, o + 0);
          ts::planes_of(p.y, o + 4);
          ts::planes_of(p.z, o + 8);
          ts::planes_of(p.w, o + 12);
        } else {
          ts::scaled_of(p.x, o + 0);
          ts::scaled_of(p.y, o + 4);
          ts::scaled_of(p.z, o + 8);
          ts::scaled_of(p.w, o + 12);
        }
        tmem_st_32x32b_x16(col0 + static_cast<uint32_t>(16 * c), o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.unpacked(a));
    }
    (void)ok;
    {
      // ------------------------ accumulator -> registers -> (partial tile)
      // Warp w reads the tensor-memory lanes of quarter w % 4 and takes every
      // other chunk of activation rows, from chunk (w - 4) / 4 on.
      const int quarter = warp & 3;
      const int ehalf = (warp - 4) >> 2;
      if (S == 1) {
        pdl_wait();  // the output may still be read by the previous kernel
        named_barrier_sync(2, 320);  // warps 2-11: the scalars are staged
      }
      // lane = weight row n of this warp's quarter of the tile
      const int nq = n0 + quarter * 32;
      const float swn = sm.col_sw()[quarter * 32 + lane];
      const uint16_t bn = sm.col_bias()[quarter * 32 + lane];
      if (mbar_wait_warp(sm.tfull(), 0u, abort)) {
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        if (S == 1) {
          // The epilogue straight from the accumulator (column = activation
          // row m), CH rows at a time. Lane j holds row j's scalars and the
          // shuffles hand them out; the chunk goes through a shared-memory
          // patch (the stage buffers are idle once tfull has fired) and
          // leaves as 16-byte pieces of output rows.
          constexpr int CH = BX < 32 ? BX : 32;
          constexpr int EB = kAccOut ? 4 : 2;        // output element bytes
          constexpr int PER_ROW = 32 * EB / 16;      // 16-byte pieces per patch row
          uint8_t* stg = sm.wp(0) + (warp - 4) * (32 * 32 * 4);
#pragma unroll 1
          for (int c = ehalf * CH; c < BX; c += 2 * CH) {
            const float sa_l = sm.row_sa()[c + (lane & (CH - 1))];
            const int corr_l = sm.row_corr()[c + (lane & (CH - 1))];
            uint32_t v[CH];
            if constexpr (CH == 32) {
              tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), v);
            } else {
              tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(c), v);
            }
            tmem_ld_wait();
            __syncwarp();  // the previous chunk's reads of the patch are done
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              const int acc = (static_cast<int>(v[j]) >> kShift) - __shfl_sync(0xFFFFFFFFu, corr_l, j);
              if constexpr (kAccOut) {
                reinterpret_cast<int32_t*>(stg)[j * 32 + lane] = acc;
              } else {
                const float sa_j = __shfl_sync(0xFFFFFFFFu, sa_l, j);
                const uint16_t y = f32_to_bf16_bits(__fmul_rn(__fmul_rn(__int2float_rn(acc), sa_j), swn));
                reinterpret_cast<uint16_t*>(stg)[j * 32 + lane] =
                    bias != nullptr ? add_bias_bf16_v(y, bn) : y;
              }
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < CH * PER_ROW / 32; ++i) {
              const int piece = lane + 32 * i;
              const int j = piece / PER_ROW;
              const int col = (piece % PER_ROW) * (16 / EB);
              const int m = c + j;
              const int nc = nq + col;
              if (m < M && nc < N) {
                uint8_t* dst = static_cast<uint8_t*>(out) + (static_cast<int64_t>(m) * N + nc) * EB;
                const uint8_t* src = stg + (j * 32 + col) * EB;
                if (nc + 16 / EB <= N && ((N * EB) & 15) == 0) {
                  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
                } else {
                  for (int e = 0; e < 16 / EB && nc + e < N; ++e)
                    for (int b = 0; b < EB; ++b) dst[e * EB + b] = src[e * EB + b];
                }
              }
            }
          }
        } else {
          int32_t* part = sm.part();
          const int rr = quarter * 32 + lane;
#pragma unroll 1
          for (int c = ehalf * 16; c < BX; c += 32) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(c), v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) part[(c + j) * BW + rr] = static_cast<int32_t>(v[j]) >> kShift;
          }
        }
      }
    }
  }

  if (S > 1) {
    // ------------------------------------- cluster reduction and epilogue
    pdl_wait();  // the output may still be read by the previous kernel
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // every CTA's partial tile (and its staged scalars) is in shared memory
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
      int a4[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < MAX_SPLIT; ++q)
        if (q < S) {
          a4[0] += static_cast<int>(v[q].x);
          a4[1] += static_cast<int>(v[q].y);
          a4[2] += static_cast<int>(v[q].z);
          a4[3] += static_cast<int>(v[q].w);
        }
      {
        const int corr = sm.row_corr()[m];
#pragma unroll
        for (int j = 0; j < 4; ++j) a4[j] -= corr;
      }
      const bool whole = n + 3 < N && (N & 3) == 0;
      if constexpr (kAccOut) {
        int32_t* o = static_cast<int32_t*>(out) + static_cast<int64_t>(m) * N + n;
        if (whole) {
          *reinterpret_cast<int4*>(o) = make_int4(a4[0], a4[1], a4[2], a4[3]);
        } else {
          for (int j = 0; j < 4 && n + j < N; ++j) o[j] = a4[j];
        }
      } else {
        const float sa = sm.row_sa()[m];
        uint16_t y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          y[j] = f32_to_bf16_bits(__fmul_rn(__fmul_rn(__int2float_rn(a4[j]), sa), sm.col_sw()[rl + j]));
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
    cluster_sync();  // the other CTAs have finished reading this CTA's partial tile
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace fr
}  // namespace bitnet
