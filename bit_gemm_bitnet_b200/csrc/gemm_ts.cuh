// Batched ternary x INT8 GEMM on the 5th-generation tensor cores with the
// weights as the tensor-memory operand (tcgen05.mma kind::i8, A from TMEM,
// B from shared memory), int32 accumulators in TMEM, scale epilogue fused.
//
// D[n, m] = sum_k W[n, k] * x_q[m, k]: the MMA's M dimension is 128 weight
// rows (TMEM lanes), its N dimension BX = 192 activation rows. Unpacked
// weights go registers -> TMEM (tcgen05.st) and never touch shared memory, so
// per 128-K stage the shared-memory traffic is the activation tile (written
// by TMA, read by the MMA) and the small packed weight tile.
//
// TMEM (512 columns): two 192-column accumulators + four 32-column A stages;
// shared memory holds six stages of activation and packed tiles (the two
// rings are separate, so TMA runs further ahead than tensor memory allows).
// Warp roles (512 threads), persistent (one CTA per SM):
//   warp 0      TMA producer (x tile, 128-byte swizzle; packed weight tile)
//   warp 1      TMEM owner, MMA issuer (one thread)
//   warps 4-7   epilogue: tcgen05.ld, fp32 scales, bf16 (or int32) stores
//   warps 8-15  unpack: packed codes -> int8 -> tcgen05.st into the A stage
//               (two groups of four warps on alternate stages)
// Waits are bounded like the other kernels of this library.
#pragma once
#include "common.cuh"

namespace bitnet {
namespace ts {

constexpr int BW = 128;                 // weight rows per tile (MMA M)
constexpr int BX = 192;                 // activation rows per tile (MMA N)
constexpr int BK = 128;                 // K per stage (four K = 32 MMAs)
constexpr int STAGES = 6;                // shared-memory stages (activation + packed tiles)
constexpr int ASTAGES = 4;               // tensor-memory A stages (unpacked weights)
constexpr int X_BYTES = BX * BK;        // 24 KB
constexpr int WP_BYTES = BW * BK / 4;   //  4 KB
constexpr int STAGE_BYTES = X_BYTES + WP_BYTES;
constexpr int NUM_THREADS = 512;
constexpr int TMEM_COLS = 512;
constexpr int NACC = 2;                 // accumulator buffers (epilogue overlaps the next tile)
constexpr int A_COL0 = NACC * BX;       // first A-stage column
constexpr int A_COLS = BK / 4;          // 32 columns per A stage
constexpr int BAR_BYTES = 256;
constexpr int EPI_BYTES = 4 * 32 * 32 * 4;  // per epilogue warp: one 32 x 32 chunk
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + EPI_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(A_COL0 + ASTAGES * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "too much shared memory");

// int32 D, A (weights) unsigned code planes or signed int8, B signed int8,
// both K-major, N = BX, M = BW.
constexpr uint32_t kIdescShape = (2u << 4) | (1u << 10) |
                                 (static_cast<uint32_t>(BX >> 3) << 17) |
                                 (static_cast<uint32_t>(BW >> 4) << 24);
constexpr uint32_t kIdescUnsignedA = kIdescShape;
constexpr uint32_t kIdescSignedA = kIdescShape | (1u << 7);

struct Smem {
  uint8_t* base;  // 1024-aligned
  __device__ uint8_t* x(int s) const { return base + s * STAGE_BYTES; }
  __device__ uint8_t* wp(int s) const { return base + s * STAGE_BYTES + X_BYTES; }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + STAGES + s); }
  // tensor-memory A stage a: unpacked (4 unpack warps arrive) / free again
  // (the MMAs that read it have completed)
  __device__ uint32_t unpacked(int a) const { return smem_u32(bars() + 2 * STAGES + a); }
  __device__ uint32_t afree(int a) const { return smem_u32(bars() + 2 * STAGES + ASTAGES + a); }
  __device__ uint32_t tfull(int a) const { return smem_u32(bars() + 2 * STAGES + 2 * ASTAGES + a); }
  __device__ uint32_t tempty(int a) const { return smem_u32(bars() + 2 * STAGES + 2 * ASTAGES + 2 + a); }
  __device__ uint32_t drain() const { return smem_u32(bars() + 2 * STAGES + 2 * ASTAGES + 4); }
  __device__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 2 * STAGES + 2 * ASTAGES + 5);
  }
  __device__ int* abort_flag() const {
    return reinterpret_cast<int*>(bars() + 2 * STAGES + 2 * ASTAGES + 6);
  }
  // warp-private staging of one 32 (activation rows) x 32 (weight rows)
  // output chunk, 4 bytes per element (bf16 outputs use the first half)
  __device__ uint8_t* epi(int quarter) const {
    return base + STAGES * STAGE_BYTES + BAR_BYTES + quarter * (32 * 32 * 4);
  }
};

// Packed word -> its four unsigned 2-bit code planes (plane i in word i).
__device__ __forceinline__ void planes_of(uint32_t w, uint32_t* o) {
  o[0] = w & 0x03030303u;
  o[1] = (w >> 2) & 0x03030303u;
  o[2] = (w >> 4) & 0x03030303u;
  o[3] = (w >> 6) & 0x03030303u;
}

// Packed word -> its 16 weights times 64, as int8 in element order (4
// words). Field i of every byte, XOR 2 (the code minus 2, modulo 4), is
// moved to the top two bits of its byte, where it reads as (code - 2) * 64;
// a 4 x 4 byte transpose then puts the fields in element order (field i of
// byte j is element 4j + i). Sums over these weights are 64 times the true
// sums: exact in int32 while 64 * |sum| < 2^31, and shifted back right by 6.
// Twelve integer-pipe operations per word; the three shifts may go to the
// multiply-add pipe.
constexpr int kScaledShift = 6;
__device__ __forceinline__ void scaled_of(uint32_t w, uint32_t* o) {
  const uint32_t e0 = ((w & 0x03030303u) ^ 0x02020202u) * 64u;
  const uint32_t e1 = ((w & 0x0C0C0C0Cu) ^ 0x08080808u) * 16u;
  const uint32_t e2 = ((w & 0x30303030u) ^ 0x20202020u) * 4u;
  const uint32_t e3 = (w & 0xC0C0C0C0u) ^ 0x80808080u;
  const uint32_t t0 = prmt(e0, e1, 0x5140u);
  const uint32_t t1 = prmt(e0, e1, 0x7362u);
  const uint32_t t2 = prmt(e2, e3, 0x5140u);
  const uint32_t t3 = prmt(e2, e3, 0x7362u);
  o[0] = prmt(t0, t2, 0x5410u);
  o[1] = prmt(t0, t2, 0x7632u);
  o[2] = prmt(t1, t3, 0x5410u);
  o[3] = prmt(t1, t3, 0x7632u);
}

// Packed word -> 16 signed int8 weights in element order (4 words).
__device__ __forceinline__ void signed_of(uint32_t w, uint32_t* o) {
  const uint32_t e0 = ((w & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e1 = (((w >> 2) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e2 = (((w >> 4) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e3 = (((w >> 6) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t t0 = prmt(e0, e1, 0x5140u);
  const uint32_t t1 = prmt(e0, e1, 0x7362u);
  const uint32_t t2 = prmt(e2, e3, 0x5140u);
  const uint32_t t3 = prmt(e2, e3, 0x7362u);
  o[0] = prmt(t0, t2, 0x5410u) ^ 0x80808080u;
  o[1] = prmt(t0, t2, 0x7632u) ^ 0x80808080u;
  o[2] = prmt(t1, t3, 0x5410u) ^ 0x80808080u;
  o[3] = prmt(t1, t3, 0x7632u) ^ 0x80808080u;
}

// kPerm: activations with transposed 16-element groups plus per-row code
// sums; weights enter as unsigned code planes and the epilogue subtracts
// 2 * rowsum[m]. Otherwise natural order and signed weights.
template <bool kAccOut, bool kPerm>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_ts_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w, void* __restrict__ out,
                      const uint16_t* __restrict__ scale_act,
                      const float* __restrict__ scale_wt, int sw_len,
                      const int32_t* __restrict__ rowsum, int M, int N, int K,
                      const uint16_t* __restrict__ bias) {
  constexpr uint32_t kIdesc = kPerm ? kIdescUnsignedA : kIdescSignedA;
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int x_tiles = (M + BX - 1) / BX;
  const int w_tiles = (N + BW - 1) / BW;
  const int num_tiles = x_tiles * w_tiles;
  const int kblocks = (K + BK - 1) / BK;
  volatile int* abort = sm.abort_flag();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), 1);
    }
    for (int a = 0; a < ASTAGES; ++a) {
      mbar_init(sm.unpacked(a), 4);
      mbar_init(sm.afree(a), 1);
    }
    for (int a = 0; a < NACC; ++a) {
      mbar_init(sm.tfull(a), 1);
      mbar_init(sm.tempty(a), 4);
    }
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
  pdl_wait();  // x_q, scales and row sums may come from the previous kernel

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int m0 = (t / w_tiles) * BX;
        const int n0 = (t % w_tiles) * BW;
        // The CTAs working on one activation tile (different weight tiles)
        // start their K loops at different blocks (the int32 sum is exact in
        // any order), so they do not all read the same lines at once.
        const int rot = (t % w_tiles) % kblocks;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(sm.empty(s), ph ^ 1u, abort)) { ok = false; break; }
          const int kr = kb + rot < kblocks ? kb + rot : kb + rot - kblocks;
          mbar_arrive_expect_tx(sm.full(s), STAGE_BYTES);
          tma_load_2d(smem_u32(sm.x(s)), &tmap_x, sm.full(s), kr * BK, m0);
          tma_load_2d(smem_u32(sm.wp(s)), &tmap_w, sm.full(s), kr * (BK / 4), n0);
        }
      }
      const uint32_t first = it > STAGES ? it - STAGES : 0u;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait_drain(sm.full(j % STAGES), (j / STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      bool ok = true;
      bool ready = false;  // the next block's unpack barrier already completed
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        const int a = static_cast<int>(local % NACC);
        const uint32_t aph = (local / NACC) & 1u;
        if (!mbar_wait(sm.tempty(a), aph ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * BX);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const int as = static_cast<int>(it % ASTAGES);
          // the unpack warps arrive only after they saw the stage's tiles land
          // (full), so this one wait also orders the activation tile's reads;
          // `ready` is the look-ahead test made with the previous block's MMAs
          if (!ready && !mbar_wait(sm.unpacked(as), (it / ASTAGES) & 1u, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(A_COL0 + as * A_COLS);
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.x(s)));
          // 4 x 32 K bytes: 8 TMEM columns of A each, +32 bytes inside B's
          // swizzle atom; the next block's unpack barrier is tested meanwhile
          const uint32_t nx = it + 1;
          ready = mma4_i8_tmem_a_test(d_tmem, a_tmem, bdesc, kIdesc, kb > 0 ? 1u : 0u,
                                      sm.unpacked(static_cast<int>(nx % ASTAGES)),
                                      (nx / ASTAGES) & 1u);
          mma_commit(sm.empty(s));
          mma_commit(sm.afree(as));
        }
        if (ok) mma_commit(sm.tfull(a));
      }
      mma_commit(sm.drain());
      mbar_wait_drain(sm.drain(), 0u);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    uint32_t local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      const int a = static_cast<int>(local % NACC);
      const uint32_t aph = (local / NACC) & 1u;
      const int m0 = (t / w_tiles) * BX;
      const int n = (t % w_tiles) * BW + quarter * 32 + lane;
      float swn = 0.0f;
      if (!kAccOut && n < N) swn = scale_wt[sw_len == 1 ? 0 : n];
      const uint16_t* bias_n = (bias != nullptr && n < N) ? bias : nullptr;  // lane's weight row
      if (!mbar_wait_warp(sm.tfull(a), aph, abort)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BX / 32; ++c) {
        // lane j fetches the scalars of activation row m0 + 32c + j; they
        // reach the other lanes by shuffles
        const int ml = m0 + c * 32 + lane;
        const float sa_l = (!kAccOut && ml < M) ? bf16_bits_to_f32(scale_act[ml]) : 0.0f;
        const int corr_l = (kPerm && ml < M) ? 2 * rowsum[ml] : 0;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(a * BX + c * 32),
                           v);
        tmem_ld_wait();
        // the chunk goes through this warp's staging patch: lane = weight
        // row n writes column `lane` of 32 activation rows, then the warp
        // writes each activation row's 32 outputs with 16-byte stores
        uint8_t* stg = sm.epi(quarter);
        __syncwarp();  // the previous chunk's reads of the patch are done
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float sa_j = __shfl_sync(0xFFFFFFFFu, sa_l, j);
          const int corr_j = __shfl_sync(0xFFFFFFFFu, corr_l, j);
          const int acc = static_cast<int>(v[j]) - corr_j;
          if constexpr (kAccOut) {
            reinterpret_cast<int32_t*>(stg)[j * 32 + lane] = acc;
          } else {
            const float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), sa_j), swn);
            reinterpret_cast<uint16_t*>(stg)[j * 32 + lane] =
                add_bias_bf16(f32_to_bf16_bits(y), bias_n, n);
          }
        }
        __syncwarp();
        const int nb = (t % w_tiles) * BW + quarter * 32;  // first weight row of the chunk
        constexpr int ebytes = kAccOut ? 4 : 2;
        constexpr int per_row = 32 * ebytes / 16;          // 16-byte pieces per row
#pragma unroll
        for (int i = 0; i < per_row; ++i) {
          const int piece = lane + 32 * i;  // 32 rows x per_row pieces
          const int j = piece / per_row;
          const int col = (piece % per_row) * (16 / ebytes);  // first n within the chunk
          const int m = m0 + c * 32 + j;
          const int n0 = nb + col;
          if (m < M) {
            uint8_t* dst = reinterpret_cast<uint8_t*>(out) + (static_cast<int64_t>(m) * N + n0) * ebytes;
            const uint8_t* src = stg + (j * 32 + col) * ebytes;
            if (n0 + 16 / ebytes <= N && ((N * ebytes) & 15) == 0) {
              *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
            } else {
              for (int e = 0; e < 16 / ebytes && n0 + e < N; ++e)
                for (int b = 0; b < ebytes; ++b) dst[e * ebytes + b] = src[e * ebytes + b];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.tempty(a));
    }
  } else if (warp >= 8) {
    // -------------------------------------------------------------- unpack
    // Two groups of four warps take alternate stages, so two stages are
    // unpacked at once (a stage's unpack is a chain of dependent steps: wait,
    // load, unpack, tensor-memory store, wait for the store, arrive). Warp ->
    // TMEM sub-partition warp % 4 (weight rows 32 * (warp % 4) ...), all 32
    // columns (128 K elements) of its group's stages.
    const int sub = warp & 3;
    const uint32_t group = static_cast<uint32_t>((warp - 8) >> 2);
    const int r = sub * 32 + lane;  // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        if ((it & 1u) != group) continue;
        const int s = it % STAGES;
        const int as = static_cast<int>(it % ASTAGES);
        if (!mbar_wait_warp(sm.full(s), (it / STAGES) & 1u, abort) ||
            !mbar_wait_warp(sm.afree(as), ((it / ASTAGES) & 1u) ^ 1u, abort)) { ok = false; break; }
        const uint4 p0 = *reinterpret_cast<const uint4*>(sm.wp(s) + r * 32);
        const uint4 p1 = *reinterpret_cast<const uint4*>(sm.wp(s) + r * 32 + 16);
        uint32_t o[16], o2[16];
        if constexpr (kPerm) {
          planes_of(p0.x, o + 0);
          planes_of(p0.y, o + 4);
          planes_of(p0.z, o + 8);
          planes_of(p0.w, o + 12);
          planes_of(p1.x, o2 + 0);
          planes_of(p1.y, o2 + 4);
          planes_of(p1.z, o2 + 8);
          planes_of(p1.w, o2 + 12);
        } else {
          signed_of(p0.x, o + 0);
          signed_of(p0.y, o + 4);
          signed_of(p0.z, o + 8);
          signed_of(p0.w, o + 12);
          signed_of(p1.x, o2 + 0);
          signed_of(p1.y, o2 + 4);
          signed_of(p1.z, o2 + 8);
          signed_of(p1.w, o2 + 12);
        }
        const uint32_t col = tmem_base + lane_base + static_cast<uint32_t>(A_COL0 + as * A_COLS);
        tmem_st_32x32b_x16(col, o);
        tmem_st_32x32b_x16(col + 16u, o2);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.unpacked(as));
      }
    }
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

}  // namespace ts
}  // namespace bitnet
