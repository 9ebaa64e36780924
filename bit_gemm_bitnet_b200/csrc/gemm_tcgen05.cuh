// Batched ternary x INT8 GEMM on the 5th-generation tensor cores (tcgen05,
// kind::i8, int32 accumulators in tensor memory), with the scale epilogue
// fused. Persistent: one CTA per SM walks the output tiles.
//
// Tile: 128 rows of x_q (MMA M) x 256 weight rows (MMA N) x 128 K per stage.
// Warp roles (512 threads):
//   warp 0      TMA producer: x_q tile (128-byte swizzle) and the packed
//               weight tile (32 bytes per row) for each stage;
//   warp 1      TMEM owner and MMA issuer (one thread): 4 MMAs of K = 32 per
//               stage into a double-buffered 128 x 256 int32 accumulator;
//   warps 4-7   epilogue: tcgen05.ld of the accumulator, fp32 scaling,
//               bf16 stores (or the raw int32 for the test hook);
//   warps 8-15  unpack: 2-bit codes -> int8 weights written into the
//               128-byte-swizzled K-major layout the MMA reads (signed
//               weights in natural order, or the unsigned code planes when
//               the activations come with transposed 16-element groups).
// Every wait is bounded (see mbar_wait); a role that gives up sets the device
// error word and the CTA drains and exits.
#pragma once
#include "common.cuh"

namespace bitnet {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int STAGES = 4;
constexpr int X_BYTES = BM * BK;        // 16 KB
constexpr int WU_BYTES = BN * BK;       // 32 KB, unpacked int8 weights
constexpr int WP_BYTES = BN * BK / 4;   //  8 KB, packed weights
constexpr int STAGE_BYTES = X_BYTES + WU_BYTES + WP_BYTES;
constexpr int TX_BYTES = X_BYTES + WP_BYTES;
constexpr int NUM_THREADS = 512;
constexpr int UNPACK_WARPS = 8;     // warps 8-15
constexpr int TMEM_COLS = 512;          // 2 accumulators x 256 columns
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + BAR_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "too much shared memory");

// Instruction descriptors: int32 D, signed int8 A, B signed (weights
// -1/0/+1) or unsigned (2-bit codes 0..3), both K-major, N = 256, M = 128.
constexpr uint32_t kIdescShape = (2u << 4) | (1u << 7) |
                                 (static_cast<uint32_t>(BN >> 3) << 17) |
                                 (static_cast<uint32_t>(BM >> 4) << 24);
constexpr uint32_t kIdescSignedB = kIdescShape | (1u << 10);
constexpr uint32_t kIdescUnsignedB = kIdescShape;

struct Smem {
  uint8_t* base;  // 1024-aligned
  __device__ uint8_t* x(int s) const { return base + s * STAGE_BYTES; }
  __device__ uint8_t* wu(int s) const { return base + s * STAGE_BYTES + X_BYTES; }
  __device__ uint8_t* wp(int s) const {
    return base + s * STAGE_BYTES + X_BYTES + WU_BYTES;
  }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t unpacked(int s) const { return smem_u32(bars() + STAGES + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + 2 * STAGES + s); }
  __device__ uint32_t tfull(int a) const { return smem_u32(bars() + 3 * STAGES + a); }
  __device__ uint32_t tempty(int a) const { return smem_u32(bars() + 3 * STAGES + 2 + a); }
  __device__ uint32_t drain() const { return smem_u32(bars() + 3 * STAGES + 4); }
  __device__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 3 * STAGES + 5);
  }
  __device__ int* abort_flag() const {
    return reinterpret_cast<int*>(bars() + 3 * STAGES + 6);
  }
};

// One packed word (16 weights, elements 4t+i in byte t bits 2i) -> 16 signed
// int8 weights in element order, as a 16-byte vector.
__device__ __forceinline__ uint4 unpack_word_s8(uint32_t w) {
  // plane i holds, in byte t, the code of element 4t+i; the 0x80 guard bit
  // keeps the per-byte subtraction of 2 from borrowing across bytes.
  const uint32_t e0 = ((w & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e1 = (((w >> 2) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e2 = (((w >> 4) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  const uint32_t e3 = (((w >> 6) & 0x03030303u) | 0x80808080u) - 0x02020202u;
  // transpose the 4x4 bytes: word t = (e0.t, e1.t, e2.t, e3.t)
  const uint32_t t0 = prmt(e0, e1, 0x5140u);
  const uint32_t t1 = prmt(e0, e1, 0x7362u);
  const uint32_t t2 = prmt(e2, e3, 0x5140u);
  const uint32_t t3 = prmt(e2, e3, 0x7362u);
  return make_uint4(prmt(t0, t2, 0x5410u) ^ 0x80808080u,
                    prmt(t0, t2, 0x7632u) ^ 0x80808080u,
                    prmt(t1, t3, 0x5410u) ^ 0x80808080u,
                    prmt(t1, t3, 0x7632u) ^ 0x80808080u);
}

// One packed word -> its four 2-bit planes as unsigned codes, plane i in
// word i: bytes (c(4t+i)) for t = 0..3. Matches activations whose 16-element
// groups are stored transposed (element 4t + i at byte 4i + t).
__device__ __forceinline__ uint4 unpack_word_planes(uint32_t w) {
  return make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                    (w >> 6) & 0x03030303u);
}

// kPerm: activations come with transposed 16-element groups and per-row code
// sums (from the quantiser of bitnet_linear); the weights then enter the MMA
// as unsigned codes c = w + 2 and the epilogue subtracts 2 * rowsum[m].
// Otherwise activations are in natural order and the weights are expanded to
// signed int8 in natural order.
template <bool kAccOut, bool kPerm>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_i8_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_w,
                           void* __restrict__ out,
                           const uint16_t* __restrict__ scale_act,
                           const float* __restrict__ scale_wt, int sw_len,
                           const int32_t* __restrict__ rowsum,
                           int M, int N, int K) {
  constexpr uint32_t kIdesc = kPerm ? kIdescUnsignedB : kIdescSignedB;
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks = (K + BK - 1) / BK;
  volatile int* abort = sm.abort_flag();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.unpacked(s), UNPACK_WARPS);
      mbar_init(sm.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
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
  pdl_wait();  // x_q and scale_act may come from the previous kernel

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * BM;
        const int n0 = (t % n_tiles) * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(sm.empty(s), ph ^ 1u, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(sm.full(s), TX_BYTES);
          tma_load_2d(smem_u32(sm.x(s)), &tmap_x, sm.full(s), kb * BK, m0);
          tma_load_2d(smem_u32(sm.wp(s)), &tmap_w, sm.full(s), kb * (BK / 4), n0);
        }
      }
      // drain: every load issued has landed before the CTA may exit
      const uint32_t first = it > STAGES ? it - STAGES : 0u;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait_drain(sm.full(j % STAGES), (j / STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        const int a = local & 1;
        const uint32_t aph = (local >> 1) & 1u;
        if (!mbar_wait(sm.tempty(a), aph ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(sm.full(s), ph, abort) ||
              !mbar_wait(sm.unpacked(s), ph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sm.x(s)));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.wu(s)));
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            // +32 bytes along K inside the 128-byte swizzle atom
            mma_i8(d_tmem, adesc + 2u * k, bdesc + 2u * k, kIdesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(sm.empty(s));
        }
        if (ok) mma_commit(sm.tfull(a));
      }
      // drain: no MMA may still be writing TMEM when it is freed
      mma_commit(sm.drain());
      mbar_wait_drain(sm.drain(), 0u);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lanes 32*quarter ...
    const int row = quarter * 32 + lane;   // accumulator row = x_q row in tile
    uint32_t local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      const int a = local & 1;
      const uint32_t aph = (local >> 1) & 1u;
      if (!mbar_wait(sm.tfull(a), aph, abort)) break;
      tc_fence_after();
      const int m = (t / n_tiles) * BM + row;
      const int n_tile0 = (t % n_tiles) * BN;
      float sa = 0.0f;
      if (!kAccOut && m < M) sa = bf16_bits_to_f32(scale_act[m]);
      const int corr = (kPerm && m < M) ? 2 * rowsum[m] : 0;
      const float sw0 = kAccOut ? 0.0f : scale_wt[0];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(a * BN + c * 32),
                           v);
        tmem_ld_wait();
        const int n = n_tile0 + c * 32;
        if (m < M && n < N) {
          if constexpr (kAccOut) {
            int32_t* o = reinterpret_cast<int32_t*>(out) + static_cast<int64_t>(m) * N + n;
            if constexpr (kPerm) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = static_cast<uint32_t>(static_cast<int>(v[j]) - corr);
            }
            if (n + 32 <= N && (N & 3) == 0) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<uint4*>(o + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            } else {
              for (int j = 0; j < 32 && n + j < N; ++j) o[j] = static_cast<int32_t>(v[j]);
            }
          } else {
            uint16_t* o = reinterpret_cast<uint16_t*>(out) + static_cast<int64_t>(m) * N + n;
            uint32_t h[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int nj = n + j;
              const float s0 = sw_len == 1 ? sw0 : (nj < N ? __ldg(scale_wt + nj) : 0.0f);
              const float s1 = sw_len == 1 ? sw0 : (nj + 1 < N ? __ldg(scale_wt + nj + 1) : 0.0f);
              const float y0 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(v[j]) - corr), sa), s0);
              const float y1 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(v[j + 1]) - corr), sa), s1);
              h[j / 2] = static_cast<uint32_t>(f32_to_bf16_bits(y0)) |
                         (static_cast<uint32_t>(f32_to_bf16_bits(y1)) << 16);
            }
            if (n + 32 <= N && (N & 7) == 0) {
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<uint4*>(o + 2 * j) = make_uint4(h[j], h[j + 1], h[j + 2], h[j + 3]);
            } else {
              for (int j = 0; j < 32 && n + j < N; ++j)
                o[j] = static_cast<uint16_t>(h[j / 2] >> (16 * (j & 1)));
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
    // 256 threads, each unpacking two half rows per stage: half row hr
    // (row hr / 2, 16 packed bytes) is read with one conflict-free 16-byte
    // load (consecutive lanes read consecutive 16-byte pieces).
    const int u = threadIdx.x - 256;  // 0..255
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!mbar_wait(sm.full(s), ph, abort)) { ok = false; break; }
        const uint8_t* wp = sm.wp(s);
        uint8_t* wu = sm.wu(s);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int hr = u + 256 * i;
          const int r = hr >> 1, h = hr & 1;
          const uint4 p = *reinterpret_cast<const uint4*>(wp + hr * 16);
          const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
          uint8_t* dst = wu + r * 128;
          const int sw = r & 7;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            // 16-byte chunk j of the row sits at chunk position j ^ (row % 8)
            const int j = 4 * h + jj;
            *reinterpret_cast<uint4*>(dst + ((j ^ sw) << 4)) =
                kPerm ? unpack_word_planes(pw[jj]) : unpack_word_s8(pw[jj]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.unpacked(s));
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

}  // namespace gemm
}  // namespace bitnet
