// Grouped decode GEMV: many independent fused quantise + GEMV problems (same
// M, any K and N) in one persistent launch.
//
// The row blocks ("units") of all problems form one list, in problem order.
// Each CTA owns a contiguous range of it. Its producer warp streams the units'
// packed weights (contiguous rows) through the shared-memory ring with bulk
// async copies, crossing problem boundaries without a pause, while the
// consumer warps quantise a problem's activation rows when they first reach
// one of its units and then reduce its rows exactly as the single-problem
// kernel does. One launch replaces one launch per problem, so the fixed cost
// of a launch and of a CTA's start is paid once for the whole group.
#pragma once
#include "gemv.cuh"

namespace bitnet {

constexpr int kGroupMax = 256;       // problems per launch (kernel parameter space)
constexpr int kGroupGridMax = 512;   // CTAs per launch
// Consumer warps per CTA, by activation-row bucket. One row: 15 (with the
// producer 16 warps, four per scheduler, so each thread may hold 128
// registers: more rows in flight per warp). More rows: 16 (the dp4a work per
// weight grows with the rows and wants every warp).
constexpr int grouped_cw(int mb) { return mb == 1 ? 15 : 16; }
constexpr int kGroupedMaxCW = 16;
// Bytes per unit (aim): large units spread a unit's fixed cost (the wait, the
// warp reduction, the stores) over more rows; two or three stages of the
// ring still cover the memory latency.
constexpr int kGroupedStageTarget = 80 * 1024;

struct GroupedParams {
  int count;               // problems in this launch
  int M;                   // activation rows of every problem (1..15)
  int units;               // total units
  int stages;
  uint32_t q_bytes;        // shared bytes for the quantised rows (M * max K)
  uint32_t stage_bytes;    // shared bytes per stage (the largest unit)
  int unit0[kGroupMax + 1];  // first unit of each problem; unit0[count] = units
  int cta_u0[kGroupGridMax + 1];  // first unit of each CTA; cta_u0[grid] = units
  int8_t rw[kGroupMax];      // weight rows per consumer warp per unit
  int K[kGroupMax];
  int N[kGroupMax];
  int sw_len[kGroupMax];
  const uint16_t* x[kGroupMax];
  const uint8_t* wp[kGroupMax];
  const float* sw[kGroupMax];
  uint16_t* out[kGroupMax];   // bf16 [M, N]; int32 [M, N] in the accumulator hook
};

// The accumulator hook's parameters: the product's, plus where each problem's
// int8 codes [M, K] (natural order) and bf16 scales [M] staged on chip go.
struct GroupedDebugParams : GroupedParams {
  int8_t* dbg_q[kGroupMax];
  uint16_t* dbg_sa[kGroupMax];
};

// One consumer warp's share of a unit: rw == RW rows of a stage (fewer at a
// problem's ragged end), then the release of the stage and the epilogue
// (ACC: the int32 sums are stored instead, to `out` read as int32 [M, N]).
template <int MB, int RW, bool PLANES, bool ACC>
__device__ __forceinline__ void grouped_unit(const uint32_t* wrow, int K, const uint8_t* qs, int Mc,
                                             int rows, int lane, int n0, int N, const int* qsum,
                                             const float* saf, uint16_t* out, const float* sw,
                                             int sw_len, uint32_t empty_bar) {
  int acc[RW][MB][PLANES ? 4 : 1];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int m = 0; m < MB; ++m)
#pragma unroll
      for (int i = 0; i < (PLANES ? 4 : 1); ++i) acc[r][m][i] = 0;
  if (rows == RW)
    gemv_rows<MB, RW, PLANES, true, PLANES>(acc, wrow, K / 16, qs, K, Mc, rows, lane);
  else if (rows > 0)
    gemv_rows<MB, RW, PLANES, false, PLANES>(acc, wrow, K / 16, qs, K, Mc, rows, lane);
  __syncwarp();
  if (lane == 0) mbar_arrive(empty_bar);
  if constexpr (ACC)
    gemv_reduce_store<MB, RW, PLANES>(acc, rows, n0, Mc, 0, N, qsum, saf, nullptr,
                                      reinterpret_cast<int32_t*>(out), sw, sw_len);
  else
    gemv_reduce_store<MB, RW, PLANES>(acc, rows, n0, Mc, 0, N, qsum, saf, out, nullptr, sw, sw_len);
}

// grouped_unit for the power of two rw <= RW: the instantiation with RW = rw.
template <int MB, int RW, bool PLANES, bool ACC>
__device__ __forceinline__ void grouped_unit_rw(int rw, const uint32_t* wrow, int K, const uint8_t* qs,
                                                int Mc, int rows, int lane, int n0, int N,
                                                const int* qsum, const float* saf, uint16_t* out,
                                                const float* sw, int sw_len, uint32_t empty_bar) {
  if constexpr (RW == 1) {
    grouped_unit<MB, 1, PLANES, ACC>(wrow, K, qs, Mc, rows, lane, n0, N, qsum, saf, out, sw,
                                     sw_len, empty_bar);
  } else {
    if (rw >= RW)
      grouped_unit<MB, RW, PLANES, ACC>(wrow, K, qs, Mc, rows, lane, n0, N, qsum, saf, out, sw,
                                        sw_len, empty_bar);
    else
      grouped_unit_rw<MB, RW / 2, PLANES, ACC>(rw, wrow, K, qs, Mc, rows, lane, n0, N, qsum, saf,
                                               out, sw, sw_len, empty_bar);
  }
}

// CW consumer warps; MB activation-row bucket; RW_MAX the most rows a warp
// takes per unit (a problem's own count, a power of two, picks the
// instantiation, so no work is spent on absent rows). Every K is a
// multiple of 64 (16-byte aligned rows). CTA c takes the units
// cta_u0[c] .. cta_u0[c + 1] - 1 (ranges balanced by bytes on the host).
// ACC (the accumulator hook, P = GroupedDebugParams): the same kernel storing
// int32 sums, and every CTA that stages a problem also writes its codes and
// scales (identical values from every such CTA).
template <int CW, int MB, int RW_MAX, bool ACC = false, typename P = GroupedParams>
__global__ void __launch_bounds__((CW + 1) * 32, 1)
    gemv_grouped_kernel(const __grid_constant__ P p) {
  constexpr int kConsumers = CW * 32;
  constexpr bool PLANES = MB <= 2;
  extern __shared__ __align__(128) uint8_t smem[];
  int* qsum = reinterpret_cast<int*>(smem);
  float* saf = reinterpret_cast<float*>(smem + 64);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 128);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + 256);
  float* rq_s = reinterpret_cast<float*>(smem + 320);
  float* rq_r = reinterpret_cast<float*>(smem + 384);
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + 512);
  uint8_t* qs = smem + kGemvHeaderBytes;
  uint8_t* ring = qs + p.q_bytes;
  static_assert(CW * MB * 4 <= kGemvHeaderBytes - 512, "reduction scratch");

  const int S = p.stages;
  const int Mc = MB == 1 ? 1 : p.M;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int u_begin = p.cta_u0[blockIdx.x];
  const int u_end = p.cta_u0[blockIdx.x + 1];
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + kGemvMaxStages + s); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), CW);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // problem of the first unit of this CTA: the last i with unit0[i] <= u_begin
  int pr = 0;
  for (int lo = 0, hi = p.count - 1; lo <= hi;) {
    const int mid = (lo + hi) >> 1;
    if (p.unit0[mid] <= u_begin) {
      pr = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  // the current problem's fields, held in registers: kernel parameters read
  // with a run-time index are fetched again on every use
  int u0 = p.unit0[pr], u1 = p.unit0[pr + 1];

  if (warp == CW) {
    // ------------------------------------------------------------ producer
    int KB = p.K[pr] / 4, rpu = CW * p.rw[pr], N = p.N[pr];
    const uint8_t* wp = p.wp[pr];
    uint32_t it = 0;
    for (int u = u_begin; u < u_end; ++u, ++it) {
      bool next = false;
      while (u >= u1) {
        ++pr;
        u0 = u1;
        u1 = p.unit0[pr + 1];
        KB = p.K[pr] / 4;
        rpu = CW * p.rw[pr];
        N = p.N[pr];
        wp = p.wp[pr];
        next = true;
      }
      if (next) {
        // warm L2 with the problem's activation rows, which the consumers
        // stage when they reach this unit, up to two stages later (2 % on
        // the decode step). L2 is the point of coherence: a line fetched
        // before the previous kernel wrote it is updated by that write.
        const char* xb = reinterpret_cast<const char*>(p.x[pr]);
        const int xbytes = (MB == 1 ? 1 : p.M) * KB * 8;  // bf16 [M, K]
        for (int off = lane * 128; off < xbytes; off += 32 * 128)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(xb + off));
      }
      const int s = it % S;
      const uint32_t ph = (it / S) & 1u;
      if (!mbar_wait(empty(s), ph ^ 1u, abort)) break;
      const int row0 = (u - u0) * rpu;
      const int rows = min(rpu, N - row0);
      if (lane == 0) {
        const uint32_t bytes = static_cast<uint32_t>(rows) * KB;
        mbar_arrive_expect_tx(full(s), bytes);
        bulk_load(smem_u32(ring + static_cast<size_t>(s) * p.stage_bytes),
                  wp + static_cast<int64_t>(row0) * KB, bytes, full(s));
      }
    }
    const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0u;
    for (uint32_t j = first; j < it; ++j) mbar_wait_drain(full(j % S), (j / S) & 1u);
    return;
  }

  // -------------------------------------------------------------- consumers
  pdl_wait();  // activations may come from the previous kernel
  const GemvSmem sh{qsum, saf, rq_s, rq_r, red, qs};
  int staged = -1;     // problem whose activations are in shared memory
  bool dead = false;   // a wait gave up: keep the barrier sequence, skip work
  int K = 0, N = 0, rw = 1, sw_len = 1;
  const float* sw = nullptr;
  uint16_t* out = nullptr;
  uint32_t it = 0;
  for (int u = u_begin; u < u_end; ++u, ++it) {
    while (u >= u1) {
      ++pr;
      u0 = u1;
      u1 = p.unit0[pr + 1];
    }
    if (pr != staged) {
      K = p.K[pr];
      N = p.N[pr];
      rw = p.rw[pr];
      sw_len = p.sw_len[pr];
      sw = p.sw[pr];
      out = p.out[pr];
      // every consumer warp reaches each problem switch at the same unit
      // (the staging only reads the activations, so it also runs after a
      // wait gave up: every consumer warp keeps the same barrier sequence)
      if (staged >= 0) named_barrier_sync(1, kConsumers);
      if constexpr (ACC)
        gemv_stage_activations<CW, MB, PLANES>(sh, p.x[pr], K, Mc, p.dbg_q[pr], p.dbg_sa[pr]);
      else
        gemv_stage_activations<CW, MB, PLANES>(sh, p.x[pr], K, Mc, nullptr, nullptr);
      named_barrier_sync(1, kConsumers);
      staged = pr;
    }
    const int s = it % S;
    const uint32_t ph = (it / S) & 1u;
    if (!dead && !mbar_wait(full(s), ph, abort)) dead = true;
    const int KB = K / 4;
    const int r0 = warp * rw;
    const int n0 = (u - u0) * (CW * rw) + r0;
    int rows = min(rw, N - n0);
    if (rows < 0 || dead) rows = 0;

    const uint32_t* wrow = reinterpret_cast<const uint32_t*>(
        ring + static_cast<size_t>(s) * p.stage_bytes + static_cast<size_t>(r0) * KB);
    grouped_unit_rw<MB, RW_MAX, PLANES, ACC>(rw, wrow, K, qs, Mc, rows, lane, n0, N, qsum, saf, out,
                                             sw, sw_len, empty(s));
  }
}

}  // namespace bitnet
