// libbitnet_b200: C ABI entry points (declared in include/bitnet.h).
//
// Host code only validates arguments, picks a kernel variant and launches it
// on the caller's stream; all arithmetic runs in the kernels included below.
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "../../include/bitnet.h"
#include "common.cuh"
#include "gemm_fr.cuh"
#include "gemm_sk.cuh"
#include "gemm_skq.cuh"
#include "gemm_ts.cuh"
#include "ternarize.cuh"
#include "rmsnorm.cuh"
#include "gemv.cuh"
#include "gemv_grouped.cuh"
#include "pack_quant.cuh"

namespace bitnet {
namespace {

constexpr int kGemvMaxM = 15;
constexpr int kLinearGemvMaxM = 15;

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Launch with programmatic stream serialisation (PDL) enabled.
template <typename Kernel, typename... Args>
bitnet_status launch_pdl(Kernel k, dim3 grid, dim3 block, size_t smem,
                         cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, args...);
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

// PDL launch of clusters of `cluster_x` consecutive CTAs.
template <typename Kernel, typename... Args>
bitnet_status launch_pdl_cluster(Kernel k, dim3 grid, dim3 block, size_t smem, int cluster_x,
                                 cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, args...);
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

struct DeviceInfo {
  int sms = 0;
  bool ready = false;
};

DeviceInfo g_dev[64];
std::mutex g_mu;
std::mutex g_mu_hook;  // the grouped accumulator hook's parameter block

bitnet_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BITNET_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BITNET_ERR_CUDA;
    d.ready = true;
  }
  *out = &d;
  return BITNET_OK;
}

int current_device() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

// The kernel attribute that opens dynamic shared memory beyond 48 KB is a
// driver call: made once per (kernel, device) for the largest size asked
// so far, not on every launch.
bitnet_status ensure_smem(const void* kernel, size_t smem) {
  if (smem <= 48 * 1024) return BITNET_OK;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  const int dev = current_device();
  if (dev < 0) return BITNET_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[std::make_pair(kernel, dev)];
  if (have >= smem) return BITNET_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return BITNET_ERR_CUDA;
  have = smem;
  return BITNET_OK;
}

// Resident CTAs per SM of `kernel` at `threads` and `smem` (an occupancy
// query is a driver call: cached per kernel, device and launch shape).
bitnet_status occupancy(const void* kernel, int threads, size_t smem, int* occ) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
  const int dev = current_device();
  if (dev < 0) return BITNET_ERR_CUDA;
  const auto key = std::make_tuple(kernel, dev, threads, smem);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *occ = it->second;
      return BITNET_OK;
    }
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
    return BITNET_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = n;
  *occ = n;
  return BITNET_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D uint8 tensor map: rows x cols bytes, row pitch `pitch` bytes,
// box of box_rows x box_cols bytes.
bool encode_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint64_t pitch, uint32_t box_rows, uint32_t box_cols,
                   CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// encode_map_u8 through a small cache keyed by every encoded field: a call
// that repeats the operands of an earlier one (a layer's weights, a
// workspace) reuses its map instead of encoding it again.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                 uint64_t pitch, uint32_t box_rows, uint32_t box_cols,
                 CUtensorMapSwizzle swz) {
  using Key = std::tuple<const void*, uint64_t, uint64_t, uint64_t, uint32_t, uint32_t, int>;
  static std::mutex mu;
  static std::map<Key, CUtensorMap> cache;
  constexpr size_t kMaxEntries = 4096;
  const Key key{base, rows, cols, pitch, box_rows, box_cols, static_cast<int>(swz)};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *m = it->second;
      return true;
    }
  }
  if (!encode_map_u8(m, base, rows, cols, pitch, box_rows, box_cols, swz)) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kMaxEntries) cache.clear();
  cache.emplace(key, *m);
  return true;
}

bitnet_status check_compute_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return BITNET_ERR_SHAPE;
  // index arithmetic inside the kernels is 32-bit per dimension
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return BITNET_ERR_SHAPE;
  return BITNET_OK;
}

bitnet_status check_scale_wt(const float* sw, int64_t len, int64_t N) {
  if (sw == nullptr) return BITNET_ERR_NULL;
  if (len != 1 && len != N) return BITNET_ERR_SHAPE;
  if (!aligned(sw, 4)) return BITNET_ERR_ALIGN;
  return BITNET_OK;
}

// ---------------------------------------------------------------- GEMV
size_t align128(size_t v) { return (v + 127) & ~static_cast<size_t>(127); }

constexpr size_t kSmemLimit = 232448;  // per-CTA opt-in maximum on sm_100

// Shared memory of the GEMV for `rows` activation rows of length K and a ring
// of `stages` stages of `rw` rows per warp.
size_t gemv_smem(int rows, int64_t K, int cw, int rw, int stages) {
  return kGemvHeaderBytes + align128(static_cast<size_t>(rows) * K) +
         static_cast<size_t>(stages) * align128(static_cast<size_t>(cw * rw) * (K / 4));
}

// Does the GEMV fit `rows` activation rows of length K (one stage of one
// row per warp of the widest CTA at least)?
bool gemv_fits(int rows, int64_t K) {
  return gemv_smem(rows, K, kGemvMaxConsumerWarps, 1, 1) <= kSmemLimit;
}

int pow2_floor(int64_t v) {
  int r = 1;
  while (static_cast<int64_t>(r) * 2 <= v) r *= 2;
  return r;
}

template <int CW, int MB, int RW, bool WIDE, bool PREQ, bool NORM>
bitnet_status launch_gemv_t(const GemvParams& p, int grid_y, size_t smem, int sms,
                            cudaStream_t st) {
  auto k = gemv_kernel<CW, MB, RW, WIDE, PREQ, NORM>;
  constexpr int threads = (CW + 1) * 32;
  if (ensure_smem(reinterpret_cast<const void*>(k), smem) != BITNET_OK) return BITNET_ERR_CUDA;
  // persistent: no more CTAs than row blocks, nor than can be resident
  int occ = 0;
  if (occupancy(reinterpret_cast<const void*>(k), threads, smem, &occ) != BITNET_OK)
    return BITNET_ERR_CUDA;
  if (occ < 1) occ = 1;
  const int nblocks = (p.N + p.rows_per_block - 1) / p.rows_per_block;
  int gx = nblocks < occ * sms ? nblocks : occ * sms;
  if (gx < 1) gx = 1;
  return launch_pdl(k, dim3(gx, grid_y), dim3(threads), smem, st, p);
}

template <int CW, int MB, bool WIDE, bool PREQ, bool NORM>
bitnet_status launch_gemv_rw(int rw, const GemvParams& p, int gy, size_t smem, int sms,
                             cudaStream_t st) {
  switch (rw) {
    case 1: return launch_gemv_t<CW, MB, 1, WIDE, PREQ, NORM>(p, gy, smem, sms, st);
    case 2: return launch_gemv_t<CW, MB, 2, WIDE, PREQ, NORM>(p, gy, smem, sms, st);
    // instantiated exactly where rw * MB * (MB <= 2 ? 4 : 1) <= 32, the
    // accumulator limit the caller applies
    case 4:
      if constexpr (MB <= 8) return launch_gemv_t<CW, MB, 4, WIDE, PREQ, NORM>(p, gy, smem, sms, st);
      return BITNET_ERR_SHAPE;
    default:
      if constexpr (MB == 1 || MB == 4) return launch_gemv_t<CW, MB, 8, WIDE, PREQ, NORM>(p, gy, smem, sms, st);
      return BITNET_ERR_SHAPE;
  }
}

// NORM (the fused RMSNorm): one or two fused rows only, its own
// instantiations, so that the other kernels carry none of its registers.
template <int CW, bool WIDE, bool PREQ, bool NORM = false>
bitnet_status launch_gemv_mb(int mb, int rw, const GemvParams& p, int gy, size_t smem, int sms,
                             cudaStream_t st) {
  if constexpr (NORM) {
    if (mb == 1) return launch_gemv_rw<CW, 1, WIDE, false, true>(rw, p, gy, smem, sms, st);
    if (mb == 2) return launch_gemv_rw<CW, 2, WIDE, false, true>(rw, p, gy, smem, sms, st);
    return BITNET_ERR_SHAPE;
  } else {
    switch (mb) {
      case 1: return launch_gemv_rw<CW, 1, WIDE, PREQ, false>(rw, p, gy, smem, sms, st);
      case 2: return launch_gemv_rw<CW, 2, WIDE, PREQ, false>(rw, p, gy, smem, sms, st);
      case 4: return launch_gemv_rw<CW, 4, WIDE, PREQ, false>(rw, p, gy, smem, sms, st);
      case 8: return launch_gemv_rw<CW, 8, WIDE, PREQ, false>(rw, p, gy, smem, sms, st);
      default: return launch_gemv_rw<CW, 16, WIDE, PREQ, false>(rw, p, gy, smem, sms, st);
    }
  }
}

template <bool WIDE, bool PREQ, bool NORM = false>
bitnet_status launch_gemv_cw(int cw, int mb, int rw, const GemvParams& p, int gy, size_t smem,
                             int sms, cudaStream_t st) {
  if (cw == 16) return launch_gemv_mb<16, WIDE, PREQ, NORM>(mb, rw, p, gy, smem, sms, st);
  return launch_gemv_mb<8, WIDE, PREQ, NORM>(mb, rw, p, gy, smem, sms, st);
}

int bucket_of(int m) { return m <= 1 ? 1 : m <= 2 ? 2 : m <= 4 ? 4 : m <= 8 ? 8 : 16; }

// Shared by the fused GEMV (PREQ = false, M <= 15) and the pre-quantised
// SIMT path of bitnet_gemm (PREQ = true, any M, row chunks of MB).
bitnet_status run_gemv(GemvParams p, bool preq, cudaStream_t st) {
  DeviceInfo* dev = nullptr;
  bitnet_status s = device_info(&dev);
  if (s != BITNET_OK) return s;
  const int64_t K = p.K;
  int mb, gy, qrows;
  if (!preq) {
    mb = bucket_of(p.M);
    gy = 1;
    qrows = p.M;
  } else {
    mb = 16;
    while (mb > 1 && !gemv_fits(mb, K)) mb /= 2;
    gy = (p.M + mb - 1) / mb;
    qrows = mb;
    if (gy > 65535) return BITNET_ERR_SHAPE;
  }
  if (!gemv_fits(qrows, K)) return BITNET_ERR_SHAPE;
  const int64_t KB = K / 4;
  auto pick_rw = [&](int warps) {
    // rows per warp per stage: a stage near 40 KB, at most 32 accumulator
    // registers per lane, and at least 16 row blocks on small layers
    int r = pow2_floor(kGemvStageTarget / (warps * KB));
    const int acc_per_row = mb * (mb <= 2 ? 4 : 1);
    while (r > 1 && r * acc_per_row > 32) r /= 2;
    if (r > 8) r = 8;
    if (r < 1) r = 1;
    while (r > 1 && (p.N + warps * r - 1) / (warps * r) < 16) r /= 2;
    while (r > 1 && gemv_smem(qrows, K, warps, r, 1) > kSmemLimit) r /= 2;
    return r;
  };
  // 16 consumer warps for large layers (latency hiding in the steady state);
  // 8 for small ones, whose CTAs are short-lived: smaller CTAs let the
  // kernels of independent calls share the SMs.
  int cw = 16;
  int rw = pick_rw(cw);
  // (only while the prologue stays short: at most ~3 activation quads per
  // consumer thread and activation row)
  if ((p.N + cw * rw - 1) / (cw * rw) < 2 * static_cast<int64_t>(dev->sms) &&
      K / 4 <= 3 * 8 * 32) {
    cw = 8;
    rw = pick_rw(cw);
  }
  const size_t stage = align128(static_cast<size_t>(cw * rw) * KB);
  // ring depth: no deeper than the row blocks one CTA will see
  const int64_t nblocks = (p.N + cw * rw - 1) / (cw * rw);
  const int64_t per_cta = (nblocks + dev->sms - 1) / dev->sms;
  int stages = static_cast<int>(kGemvRingTarget / stage);
  if (stages > per_cta) stages = static_cast<int>(per_cta);
  if (stages > kGemvMaxStages) stages = kGemvMaxStages;
  if (stages < 1) stages = 1;
  while (stages > 1 && gemv_smem(qrows, K, cw, rw, stages) > kSmemLimit) --stages;
  p.rows_per_block = cw * rw;
  p.stages = stages;
  p.q_bytes = static_cast<uint32_t>(align128(static_cast<size_t>(qrows) * K));
  p.stage_bytes = static_cast<uint32_t>(stage);
  const size_t smem = gemv_smem(qrows, K, cw, rw, stages);
  const bool wide = (K % 64) == 0;
  if (p.norm_g != nullptr && !preq)
    return wide ? launch_gemv_cw<true, false, true>(cw, mb, rw, p, gy, smem, dev->sms, st)
                : launch_gemv_cw<false, false, true>(cw, mb, rw, p, gy, smem, dev->sms, st);
  if (wide)
    return preq ? launch_gemv_cw<true, true>(cw, mb, rw, p, gy, smem, dev->sms, st)
                : launch_gemv_cw<true, false>(cw, mb, rw, p, gy, smem, dev->sms, st);
  return preq ? launch_gemv_cw<false, true>(cw, mb, rw, p, gy, smem, dev->sms, st)
              : launch_gemv_cw<false, false>(cw, mb, rw, p, gy, smem, dev->sms, st);
}

// ------------------------------------------------------------ grouped GEMV
// Split the units of a group over `grid` CTAs so that every CTA does about the
// same work. Units differ in bytes from problem to problem, and a byte costs
// more when a warp takes fewer rows (each activation load serves fewer rows):
// a unit's cost is its bytes x (rw + 0.72) / rw, and starting a problem (its
// activations quantised into shared memory) costs as much as 110 KB of
// weights. Both figures were fitted to per-CTA cycle counts of the decode
// sweep of a 2B-parameter model.
void partition_units(GroupedParams& gp, int grid, int cw) {
  constexpr int64_t kProblemCost = 110 * 1024;
  auto unit_cost = [&](int i, int64_t rows) {
    const int64_t rw = gp.rw[i];
    return rows * (gp.K[i] / 4) * (100 * rw + 72) / (100 * rw);
  };
  int64_t total = 0;
  for (int i = 0; i < gp.count; ++i) {
    const int64_t n = gp.unit0[i + 1] - gp.unit0[i];
    if (n == 0) continue;
    const int64_t rpu = static_cast<int64_t>(cw) * gp.rw[i];
    total += kProblemCost + (n - 1) * unit_cost(i, rpu) + unit_cost(i, gp.N[i] - (n - 1) * rpu);
  }
  int c = 1;
  int64_t cum = 0;  // cost of the problems before problem i
  gp.cta_u0[0] = 0;
  for (int i = 0; i < gp.count && c < grid; ++i) {
    const int64_t n = gp.unit0[i + 1] - gp.unit0[i];
    if (n == 0) continue;
    const int64_t rpu = static_cast<int64_t>(cw) * gp.rw[i];
    const int64_t cf = unit_cost(i, rpu);
    // cost before unit k of problem i: cum for k = 0, cum + P + k * cf after
    while (c < grid) {
      const int64_t T = total * c / grid;
      if (T <= cum) {
        gp.cta_u0[c++] = gp.unit0[i];
        continue;
      }
      int64_t k = (T - cum - kProblemCost + cf - 1) / cf;
      if (k < 1) k = 1;
      if (k > n - 1) break;
      gp.cta_u0[c++] = gp.unit0[i] + static_cast<int>(k);
    }
    cum += kProblemCost + (n - 1) * cf + unit_cost(i, gp.N[i] - (n - 1) * rpu);
  }
  while (c <= grid) gp.cta_u0[c++] = gp.units;
}

template <int MB, int RW_MAX, bool ACC, typename P>
bitnet_status launch_grouped_t(P& gp, size_t smem, int sms, cudaStream_t st) {
  constexpr int cw = grouped_cw(MB);
  auto k = gemv_grouped_kernel<cw, MB, RW_MAX, ACC, P>;
  constexpr int threads = (cw + 1) * 32;
  if (ensure_smem(reinterpret_cast<const void*>(k), smem) != BITNET_OK) return BITNET_ERR_CUDA;
  int occ = 0;
  if (occupancy(reinterpret_cast<const void*>(k), threads, smem, &occ) != BITNET_OK)
    return BITNET_ERR_CUDA;
  if (occ < 1) occ = 1;
  int grid = occ * sms;
  if (grid > gp.units) grid = gp.units;
  if (grid > kGroupGridMax) grid = kGroupGridMax;
  if (grid < 1) grid = 1;
  partition_units(gp, grid, cw);
  return launch_pdl(k, dim3(grid), dim3(threads), smem, st, gp);
}

// The most weight rows a consumer warp takes per unit, by activation-row
// bucket (at most 32 accumulator registers per lane).
constexpr int grouped_rw_max(int mb) { return mb == 1 ? 8 : mb == 2 ? 4 : mb == 4 ? 8 : mb == 8 ? 4 : 1; }

// Split a group into units for `cw` consumer warps (rows per warp aimed at
// `stage_target` bytes per unit) and size the ring (aimed at `ring` bytes);
// fills gp and returns the dynamic shared memory, or 0 if one stage does not
// fit under `limit`.
template <typename P>
size_t plan_grouped(P& gp, const bitnet_gemv_problem* pr, int count, int M, int sms, int cw,
                    int stage_target, int ring, size_t limit) {
  const int rw_max = grouped_rw_max(bucket_of(M));
  auto rw_of = [&](int i, int shift) {
    int rw = pow2_floor(stage_target / (cw * (pr[i].K / 4)));
    if (rw > rw_max) rw = rw_max;
    rw >>= shift;
    return rw < 1 ? 1 : rw;
  };
  // Smaller units while the group has fewer than two per SM (a small group,
  // or one problem alone), so that every SM streams. (Eight per SM for a
  // single large problem, for a finer balance, measured slower on the 82 MB
  // LM head: 27.6 against 23.6 us.)
  const int64_t min_units = 2 * static_cast<int64_t>(sms);
  int shift = 0;
  for (;; ++shift) {
    int64_t u = 0;
    bool all_one = true;
    for (int i = 0; i < count; ++i) {
      const int rw = rw_of(i, shift);
      all_one = all_one && rw == 1;
      u += (pr[i].N + cw * rw - 1) / (cw * rw);
    }
    if (u >= min_units || all_one) break;
  }
  int units = 0;
  int64_t kmax = 0;
  size_t stage = 0;
  for (int i = 0; i < count; ++i) {
    const int64_t K = pr[i].K, N = pr[i].N, KB = K / 4;
    const int rw = rw_of(i, shift);
    gp.unit0[i] = units;
    gp.rw[i] = static_cast<int8_t>(rw);
    gp.K[i] = static_cast<int>(K);
    gp.N[i] = static_cast<int>(N);
    gp.sw_len[i] = static_cast<int>(pr[i].scale_wt_len);
    gp.x[i] = static_cast<const uint16_t*>(pr[i].x);
    gp.wp[i] = pr[i].w_packed;
    gp.sw[i] = pr[i].scale_wt;
    gp.out[i] = pr[i].out;
    units += static_cast<int>((N + cw * rw - 1) / (cw * rw));
    if (K > kmax) kmax = K;
    const size_t sb = align128(static_cast<size_t>(cw * rw) * KB);
    if (sb > stage) stage = sb;
  }
  gp.unit0[count] = units;
  gp.units = units;
  gp.q_bytes = static_cast<uint32_t>(align128(static_cast<size_t>(M) * kmax));
  gp.stage_bytes = static_cast<uint32_t>(stage);
  int stages = static_cast<int>(ring / stage);
  if (stages > kGemvMaxStages) stages = kGemvMaxStages;
  if (stages < 1) stages = 1;
  while (stages > 1 && kGemvHeaderBytes + gp.q_bytes + stages * stage > limit) --stages;
  gp.stages = stages;
  const size_t smem = kGemvHeaderBytes + gp.q_bytes + static_cast<size_t>(stages) * stage;
  return smem <= limit ? smem : 0;
}

// Launch up to kGroupMax problems (all K % 64 == 0, validated) in one kernel.
// ACC: the accumulator hook (P = GroupedDebugParams, its debug pointers set
// by the caller); the partition and the launch are the product's.
template <bool ACC, typename P>
bitnet_status run_gemv_grouped_t(P& gp, const bitnet_gemv_problem* pr, int count, int M,
                                 cudaStream_t st) {
  DeviceInfo* dev = nullptr;
  bitnet_status s = device_info(&dev);
  if (s != BITNET_OK) return s;
  static_assert(sizeof(P) <= 32000, "kernel parameter space");
  static_assert(grouped_cw(1) <= kGroupedMaxCW && grouped_cw(16) <= kGroupedMaxCW &&
                    kGroupedMaxCW <= kGemvMaxConsumerWarps,
                "the staging's per-warp scratch covers every grouped CTA");
  gp.count = count;
  gp.M = M;
  const int mb = bucket_of(M);
  int64_t total_bytes = 0;
  for (int i = 0; i < count; ++i) total_bytes += pr[i].N * (pr[i].K / 4);
  if (total_bytes == 0) return BITNET_OK;
  const size_t smem = plan_grouped(gp, pr, count, M, dev->sms, grouped_cw(mb),
                                   kGroupedStageTarget, kGemvRingTarget, kSmemLimit);
  if (smem == 0) return BITNET_ERR_SHAPE;
  switch (mb) {
    case 1: return launch_grouped_t<1, grouped_rw_max(1), ACC>(gp, smem, dev->sms, st);
    case 2: return launch_grouped_t<2, grouped_rw_max(2), ACC>(gp, smem, dev->sms, st);
    case 4: return launch_grouped_t<4, grouped_rw_max(4), ACC>(gp, smem, dev->sms, st);
    case 8: return launch_grouped_t<8, grouped_rw_max(8), ACC>(gp, smem, dev->sms, st);
    default: return launch_grouped_t<16, grouped_rw_max(16), ACC>(gp, smem, dev->sms, st);
  }
}

bitnet_status run_gemv_grouped(const bitnet_gemv_problem* pr, int count, int M, cudaStream_t st) {
  GroupedParams gp;
  return run_gemv_grouped_t<false>(gp, pr, count, M, st);
}

// The accumulator hook of the grouped launch: problem i's `out` is its int32
// [M, N] output; its codes and scales go to q[i] and sa[i].
bitnet_status run_gemv_grouped_acc(const bitnet_gemv_problem* pr, int8_t* const* q,
                                   uint16_t* const* sa, int count, int M, cudaStream_t st) {
  static GroupedDebugParams gp;  // 18 KB: kept off the stack (the hook's calls are serialised)
  std::lock_guard<std::mutex> lock(g_mu_hook);
  for (int i = 0; i < count; ++i) {
    gp.dbg_q[i] = q[i];
    gp.dbg_sa[i] = sa[i];
  }
  return run_gemv_grouped_t<true>(gp, pr, count, M, st);
}

// ---------------------------------------------------------------- GEMM
bool gemm_tc_ok(const int8_t* xq, const uint8_t* wp, int64_t K) {
  // TMA: row pitches must be multiples of 16 bytes (K/4 for the packed
  // weights) and base addresses 16-byte aligned.
  return (K % 64) == 0 && aligned(xq, 16) && aligned(wp, 16);
}

// The natural-order few-row and split-K kernels take the weights as 64 * w:
// their int32 sums stay exact while 64 * 256 * K < 2^31 (|x| <= 128,
// |w| <= 2). Longer K goes to the persistent kernel (signed weights).
constexpr int64_t kScaledMaxK = INT32_MAX / (64 * 256) / 64 * 64;

// ------------------------------------------------- few-row GEMM (M <= 256)

constexpr int64_t kSkMaxRows = 256;  // activation rows the split-K kernel takes

// Clusters of `split` CTAs of `kernel` that fit on the GPU at once (cached).
int sk_clusters(const void* kernel, int split, int smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(kernel, split);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(split * 64));
  cfg.blockDim = dim3(sk::NUM_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(split);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) n = 0;
  cache[key] = n;
  return n;
}

// Split of the K loop: the S (1..8, at most the number of K blocks) that
// minimises waves x (K blocks per CTA + a fixed cost of about four K blocks
// per CTA: its start, the reduction and the epilogue).
template <typename Kernel>
int sk_split(Kernel kernel, int smem, int64_t w_tiles, int64_t kblocks) {
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int S = 1; S <= sk::MAX_SPLIT && S <= kblocks; ++S) {
    const int fit = sk_clusters(reinterpret_cast<const void*>(kernel), S, smem);
    if (fit < 1) continue;
    const int64_t waves = (w_tiles + fit - 1) / fit;
    const int64_t cost = waves * ((kblocks + S - 1) / S + 4);
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

template <int BX, bool kAccOut, bool kPerm>
bitnet_status launch_sk(const CUtensorMap& mx, const CUtensorMap& mw, void* out,
                        const uint16_t* sa, const float* sw, int64_t sw_len,
                        const int32_t* rowsum, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                        const uint16_t* bias) {
  auto kernel = sk::gemm_i8_sk_kernel<BX, kAccOut, kPerm>;
  constexpr int smem = sk::Cfg<BX>::SMEM_BYTES;
  if (ensure_smem(reinterpret_cast<const void*>(kernel), smem) != BITNET_OK)
    return BITNET_ERR_CUDA;
  const int64_t w_tiles = (N + sk::BW - 1) / sk::BW;
  const int64_t kblocks = (K + sk::BK - 1) / sk::BK;
  const int S = sk_split(kernel, smem, w_tiles, kblocks);
  if (w_tiles * S > INT32_MAX) return BITNET_ERR_SHAPE;
  return launch_pdl_cluster(kernel, dim3(static_cast<unsigned>(w_tiles * S)),
                            dim3(sk::NUM_THREADS), smem, S, st, mx, mw, out, sa, sw,
                            static_cast<int>(sw_len), rowsum, static_cast<int>(M),
                            static_cast<int>(N), static_cast<int>(K), S, bias);
}

template <int BX>
bitnet_status run_sk_bx(void* out, bool acc_out, const int8_t* xq, const uint8_t* wp,
                        const uint16_t* sa, const float* sw, int64_t sw_len, int64_t M,
                        int64_t N, int64_t K, cudaStream_t st, bool perm,
                        const int32_t* rowsum, const uint16_t* bias) {
  CUtensorMap mx, mw;
  if (!make_map_u8(&mx, xq, M, K, K, BX, sk::BK, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&mw, wp, N, K / 4, K / 4, sk::BW, sk::BK / 4, CU_TENSOR_MAP_SWIZZLE_NONE))
    return BITNET_ERR_CUDA;
  if (acc_out && perm) return launch_sk<BX, true, true>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, nullptr);
  if (acc_out) return launch_sk<BX, true, false>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, nullptr);
  if (perm) return launch_sk<BX, false, true>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, bias);
  return launch_sk<BX, false, false>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, bias);
}

// ------------------------------------- few-row GEMM, 512-wide K stages

// The split of the K loop for the few-row kernel: the S that minimises
// waves x (512-wide K blocks per CTA + a CTA's fixed cost, about four blocks,
// + the cluster reduction's, about one more, when S > 1). The constants are
// fitted to measured times of every forced split at M = 16..128 for K x N =
// 4096 x 4096, 4096 x 2560, 11008 x 4096 and 2560 x 6912.
template <typename Kernel>
int fr_split(Kernel kernel, int smem, int sms, int64_t w_tiles, int64_t kblocks) {
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int S = 1; S <= fr::MAX_SPLIT && S <= kblocks; ++S) {
    const int fit = S == 1 ? sms : sk_clusters(reinterpret_cast<const void*>(kernel), S, smem);
    if (fit < 1) continue;
    const int64_t waves = (w_tiles + fit - 1) / fit;
    const int64_t cost = waves * ((kblocks + S - 1) / S + 4 + (S > 1 ? 1 : 0));
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

template <int BX, bool kAccOut, bool kPerm>
bitnet_status launch_fr(const CUtensorMap& mx, const CUtensorMap& mw, void* out,
                        const uint16_t* sa, const float* sw, int64_t sw_len,
                        const int32_t* rowsum, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                        const uint16_t* bias) {
  auto kernel = fr::gemm_i8_fr_kernel<BX, kAccOut, kPerm>;
  constexpr int smem = fr::Cfg<BX>::SMEM_BYTES;
  if (ensure_smem(reinterpret_cast<const void*>(kernel), smem) != BITNET_OK)
    return BITNET_ERR_CUDA;
  DeviceInfo* dev = nullptr;
  bitnet_status s = device_info(&dev);
  if (s != BITNET_OK) return s;
  const int64_t w_tiles = (N + fr::BW - 1) / fr::BW;
  const int64_t kblocks = (K + fr::BKS - 1) / fr::BKS;
  const int S = fr_split(kernel, smem, dev->sms, w_tiles, kblocks);
  if (w_tiles * S > INT32_MAX) return BITNET_ERR_SHAPE;
  const dim3 grid(static_cast<unsigned>(w_tiles * S)), block(fr::NUM_THREADS);
  if (S == 1)
    return launch_pdl(kernel, grid, block, smem, st, mx, mw, out, sa, sw,
                      static_cast<int>(sw_len), rowsum, static_cast<int>(M), static_cast<int>(N),
                      static_cast<int>(K), 1, bias);
  return launch_pdl_cluster(kernel, grid, block, smem, S, st, mx, mw, out, sa, sw,
                            static_cast<int>(sw_len), rowsum, static_cast<int>(M),
                            static_cast<int>(N), static_cast<int>(K), S, bias);
}

template <int BX>
bitnet_status run_fr_bx(void* out, bool acc_out, const int8_t* xq, const uint8_t* wp,
                        const uint16_t* sa, const float* sw, int64_t sw_len, int64_t M,
                        int64_t N, int64_t K, cudaStream_t st, bool perm,
                        const int32_t* rowsum, const uint16_t* bias) {
  CUtensorMap mx, mw;
  if (!make_map_u8(&mx, xq, M, K, K, BX, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&mw, wp, N, K / 4, K / 4, fr::BW, fr::BKS / 4, CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  if (acc_out && perm) return launch_fr<BX, true, true>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, nullptr);
  if (acc_out) return launch_fr<BX, true, false>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, nullptr);
  if (perm) return launch_fr<BX, false, true>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, bias);
  return launch_fr<BX, false, false>(mx, mw, out, sa, sw, sw_len, rowsum, M, N, K, st, bias);
}

bitnet_status run_gemm_sk(void* out, bool acc_out, const int8_t* xq, const uint8_t* wp,
                          const uint16_t* sa, const float* sw, int64_t sw_len, int64_t M,
                          int64_t N, int64_t K, cudaStream_t st, bool perm,
                          const int32_t* rowsum, const uint16_t* bias) {
  // up to 128 rows: the few-row kernel with 512-wide K stages; more: the
  // split-K kernel's 256-row tile
  if (M <= 16) return run_fr_bx<16>(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
  if (M <= 32) return run_fr_bx<32>(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
  if (M <= 64) return run_fr_bx<64>(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
  if (M <= 128) return run_fr_bx<128>(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
  return run_sk_bx<256>(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
}

// ------------------------------ fused quantise + tensor-core GEMV (4 <= M)

constexpr int64_t kSkqMinRows = 8;  // fewer rows: the dp4a GEMV (measured faster there)

bool skq_ok(const void* x, const uint8_t* wp, int64_t M, int64_t K) {
  return M >= kSkqMinRows && M <= skq::BX && K % 64 == 0 && aligned(x, 16) && aligned(wp, 16);
}

// acc_out (the accumulator hook): int32 sums to `out`, codes to dbg_q and
// scales to dbg_sa, from the same kernel with the epilogue replaced.
bitnet_status run_gemv_skq(void* out, const uint16_t* x, const uint8_t* wp,
                           const float* sw, int64_t sw_len, int64_t M, int64_t N, int64_t K,
                           cudaStream_t st, const uint16_t* bias, bool acc_out = false,
                           int8_t* dbg_q = nullptr, uint16_t* dbg_sa = nullptr) {
  auto kernel = acc_out ? skq::gemv_i8_skq_kernel<true> : skq::gemv_i8_skq_kernel<false>;
  constexpr int smem = skq::SMEM_BYTES;
  if (ensure_smem(reinterpret_cast<const void*>(kernel), smem) != BITNET_OK)
    return BITNET_ERR_CUDA;
  CUtensorMap mw;
  if (!make_map_u8(&mw, wp, N, K / 4, K / 4, skq::BW, skq::BKS / 4, CU_TENSOR_MAP_SWIZZLE_128B))
    return BITNET_ERR_CUDA;
  const int64_t w_tiles = (N + skq::BW - 1) / skq::BW;
  const int64_t kstages = (K + skq::BKS - 1) / skq::BKS;
  // the split: at most MAX_KB / 4 stages per CTA (the resident activations)
  // and at most QMAX activation items per thread; the cost as for the
  // few-row GEMM, in 512-wide stages (a CTA's fixed cost about four, the
  // cluster's activation scales and reduction about four more)
  int best = 0;
  int64_t best_cost = INT64_MAX;
  for (int S = 1; S <= sk::MAX_SPLIT && S <= kstages; ++S) {
    const int64_t per_cta = (kstages + S - 1) / S;
    if (per_cta * 4 > skq::MAX_KB || per_cta * (skq::BKS / 4) * M > skq::NUM_THREADS * skq::QMAX)
      continue;
    const int fit = sk_clusters(reinterpret_cast<const void*>(kernel), S, smem);
    if (fit < 1) continue;
    const int64_t waves = (w_tiles + fit - 1) / fit;
    const int64_t cost = waves * (per_cta + 4 + (S > 1 ? 4 : 0));
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  if (best == 0) return BITNET_ERR_SHAPE;
  if (w_tiles * best > INT32_MAX) return BITNET_ERR_SHAPE;
  return launch_pdl_cluster(kernel, dim3(static_cast<unsigned>(w_tiles * best)),
                            dim3(skq::NUM_THREADS), smem, best, st, mw, out, x, sw,
                            static_cast<int>(sw_len), static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), best, bias, dbg_q, dbg_sa);
}

// perm: x_q has transposed 16-element groups and rowsum holds its per-row
// code sums (the layout of bitnet_linear's workspace); tensor-core path only.
bitnet_status run_gemm(void* out, bool acc_out, const int8_t* xq, const uint8_t* wp,
                       const uint16_t* sa, const float* sw, int64_t sw_len, int64_t M,
                       int64_t N, int64_t K, cudaStream_t st, bool perm = false,
                       const int32_t* rowsum = nullptr, const uint16_t* bias = nullptr) {
  if (M == 0 || N == 0) return BITNET_OK;
  if (!gemm_tc_ok(xq, wp, K)) {
    if (perm) return BITNET_ERR_SHAPE;  // callers only ask for perm when it applies
    GemvParams p = {};
    if (acc_out) p.acc_out = static_cast<int32_t*>(out);
    else p.out = static_cast<uint16_t*>(out);
    p.xq = xq;
    p.sa_in = sa;
    p.wp = wp;
    p.sw = sw;
    p.sw_len = static_cast<int>(sw_len);
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.bias = bias;
    return run_gemv(p, true, st);
  }
  DeviceInfo* dev = nullptr;
  bitnet_status s = device_info(&dev);
  if (s != BITNET_OK) return s;
  // 129..192 rows are one tile of the persistent kernel; where the weight
  // tiles fill at least half the SMs, that beats the split-K kernel's
  // 256-row tile (measured: 21 against 25 us at M = 160..192, N = 11008)
  const bool ts_one_wave = M > 128 && M <= ts::BX && (N + ts::BW - 1) / ts::BW >= dev->sms / 2;
  if (M <= kSkMaxRows && (perm || K <= kScaledMaxK) && !ts_one_wave)
    return run_gemm_sk(out, acc_out, xq, wp, sa, sw, sw_len, M, N, K, st, perm, rowsum, bias);
  CUtensorMap mx, mw;
  if (!make_map_u8(&mx, xq, M, K, K, ts::BX, ts::BK, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_u8(&mw, wp, N, K / 4, K / 4, ts::BW, ts::BK / 4, CU_TENSOR_MAP_SWIZZLE_NONE))
    return BITNET_ERR_CUDA;
  const int64_t tiles = ((M + ts::BX - 1) / ts::BX) * ((N + ts::BW - 1) / ts::BW);
  if (tiles > INT32_MAX) return BITNET_ERR_SHAPE;
  const int grid = static_cast<int>(tiles < dev->sms ? tiles : dev->sms);
  auto go = [&](auto kernel) -> bitnet_status {
    if (ensure_smem(reinterpret_cast<const void*>(kernel), ts::SMEM_BYTES) != BITNET_OK)
      return BITNET_ERR_CUDA;
    return launch_pdl(kernel, dim3(grid), dim3(ts::NUM_THREADS), ts::SMEM_BYTES, st, mx, mw,
                      out, sa, sw, static_cast<int>(sw_len), rowsum, static_cast<int>(M),
                      static_cast<int>(N), static_cast<int>(K), acc_out ? nullptr : bias);
  };
  if (acc_out && perm) return go(ts::gemm_i8_ts_kernel<true, true>);
  if (acc_out) return go(ts::gemm_i8_ts_kernel<true, false>);
  if (perm) return go(ts::gemm_i8_ts_kernel<false, true>);
  return go(ts::gemm_i8_ts_kernel<false, false>);
}

bitnet_status run_quantize(int8_t* xq, uint16_t* sa, const uint16_t* x, int64_t M,
                           int64_t K, cudaStream_t st) {
  if (M == 0) return BITNET_OK;
  if (M > INT32_MAX) return BITNET_ERR_SHAPE;
  const int64_t nvec = K / 8;
  const dim3 grid(static_cast<unsigned>(M)), block(kQuantThreads);
  if (nvec <= 1 * kQuantThreads)
    return launch_pdl(quantize_rows_kernel<1>, grid, block, 0, st, xq, sa, x, static_cast<int>(K));
  if (nvec <= 2 * kQuantThreads)
    return launch_pdl(quantize_rows_kernel<2>, grid, block, 0, st, xq, sa, x, static_cast<int>(K));
  if (nvec <= 4 * kQuantThreads)
    return launch_pdl(quantize_rows_kernel<4>, grid, block, 0, st, xq, sa, x, static_cast<int>(K));
  if (nvec <= 8 * kQuantThreads)
    return launch_pdl(quantize_rows_kernel<8>, grid, block, 0, st, xq, sa, x, static_cast<int>(K));
  return launch_pdl(quantize_rows_kernel<0>, grid, block, 0, st, xq, sa, x, static_cast<int>(K));
}

// float32 activations: the natural-layout quantiser, one CTA per row.
bitnet_status run_quantize_f32(int8_t* xq, uint16_t* sa, const float* x, int64_t M, int64_t K,
                               cudaStream_t st) {
  if (M == 0) return BITNET_OK;
  if (M > INT32_MAX) return BITNET_ERR_SHAPE;
  return launch_pdl(quantize_rows_f32_kernel, dim3(static_cast<unsigned>(M)),
                    dim3(kQuantThreads), 0, st, xq, sa, x, static_cast<int>(K));
}

// float32 activations: the quantiser of bitnet_linear's tensor-core path.
bitnet_status run_quantize_perm_f32(int8_t* xq, uint16_t* sa, int32_t* rowsum, const float* x,
                                    int64_t M, int64_t K, cudaStream_t st) {
  if (M == 0) return BITNET_OK;
  if (M > INT32_MAX) return BITNET_ERR_SHAPE;
  return launch_pdl(quantize_rows_perm_f32_kernel, dim3(static_cast<unsigned>(M)),
                    dim3(kQuantThreads), 0, st, xq, sa, rowsum, x, static_cast<int>(K));
}

// The quantiser of bitnet_linear's tensor-core path: transposed 16-element
// groups plus per-row code sums.
bitnet_status run_quantize_perm(int8_t* xq, uint16_t* sa, int32_t* rowsum, const uint16_t* x,
                                int64_t M, int64_t K, cudaStream_t st) {
  if (M == 0) return BITNET_OK;
  if (M > INT32_MAX) return BITNET_ERR_SHAPE;
  const int64_t groups = K / 16;
  const dim3 grid(static_cast<unsigned>(M)), block(kQuantThreads);
  const int k = static_cast<int>(K);
  if (groups <= 1 * kQuantThreads)
    return launch_pdl(quantize_rows_perm_kernel<1>, grid, block, 0, st, xq, sa, rowsum, x, k);
  if (groups <= 2 * kQuantThreads)
    return launch_pdl(quantize_rows_perm_kernel<2>, grid, block, 0, st, xq, sa, rowsum, x, k);
  if (groups <= 4 * kQuantThreads)
    return launch_pdl(quantize_rows_perm_kernel<4>, grid, block, 0, st, xq, sa, rowsum, x, k);
  return launch_pdl(quantize_rows_perm_kernel<0>, grid, block, 0, st, xq, sa, rowsum, x, k);
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Accumulator hook only: the workspace's codes back in natural order (the
// tensor-core layout transposes every 16-element group 4 x 4, its own
// inverse) and its scales, into the hook's outputs.
__global__ void unpermute_codes_kernel(int8_t* __restrict__ dst, const int8_t* __restrict__ src,
                                       int64_t groups) {
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x)
    reinterpret_cast<uint4*>(dst)[g] = transpose16(reinterpret_cast<const uint4*>(src)[g]);
}

bitnet_status copy_workspace_codes(int8_t* q, uint16_t* sa, const int8_t* ws_q,
                                   const uint16_t* ws_sa, int64_t M, int64_t K, bool permuted,
                                   cudaStream_t st) {
  const int64_t bytes = M * K;
  if (permuted) {
    const int64_t groups = bytes / 16;
    int64_t blocks = (groups + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    unpermute_codes_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, ws_q, groups);
    if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  } else if (cudaMemcpyAsync(q, ws_q, static_cast<size_t>(bytes), cudaMemcpyDeviceToDevice, st) !=
             cudaSuccess) {
    return BITNET_ERR_CUDA;
  }
  if (cudaMemcpyAsync(sa, ws_sa, static_cast<size_t>(M) * 2, cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return BITNET_ERR_CUDA;
  return BITNET_OK;
}

bool linear_uses_gemv(int64_t M, int64_t K) {
  return M >= 1 && M <= kLinearGemvMaxM && K <= INT32_MAX && gemv_fits(static_cast<int>(M), K);
}

}  // namespace
}  // namespace bitnet

using namespace bitnet;

// ---------------------------------------------------------------------------
// Allocation-free linear: built-in scratch.
//
// bitnet_linear needs a workspace for the quantised activations (int8 [M, K])
// and their scales (bf16 [M]) when M >= 16. Callers that cannot allocate
// device memory use bitnet_linear_noalloc instead, which places them in this
// fixed array. It lives in the module's global memory of every GPU that loads
// the library, for the life of the process; all calls on a device share it.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch, looked up once per device. In host
// code the array's name only stands in for the device symbol; kernels must
// be given the address cudaGetSymbolAddress returns.
void* g_noalloc_ptr[64] = {};

bitnet_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BITNET_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return BITNET_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BITNET_OK;
}
}  // namespace

extern "C" {

const char* bitnet_status_string(bitnet_status s) {
  switch (s) {
    case BITNET_OK: return "BITNET_OK";
    case BITNET_ERR_NULL: return "BITNET_ERR_NULL: a required pointer is NULL";
    case BITNET_ERR_SHAPE: return "BITNET_ERR_SHAPE: M, N, K or a length is out of range";
    case BITNET_ERR_DTYPE: return "BITNET_ERR_DTYPE: activation dtype not supported";
    case BITNET_ERR_ALIGN: return "BITNET_ERR_ALIGN: pointer not aligned as required";
    case BITNET_ERR_VALUE: return "BITNET_ERR_VALUE: weight outside {-1, 0, +1}";
    case BITNET_ERR_WORKSPACE: return "BITNET_ERR_WORKSPACE: workspace missing or too small";
    case BITNET_ERR_CUDA: return "BITNET_ERR_CUDA: CUDA call or launch failed";
    case BITNET_ERR_TIMEOUT: return "BITNET_ERR_TIMEOUT: a kernel gave up a bounded wait";
  }
  return "BITNET_ERR_UNKNOWN";
}

bitnet_status bitnet_pack_weights(uint8_t* w_packed, const int8_t* w, int64_t N,
                                  int64_t K, void* stream) {
  if (N < 0 || K < 0 || K % 4 != 0) return BITNET_ERR_SHAPE;
  if (N == 0 || K == 0) return BITNET_OK;
  if (w_packed == nullptr || w == nullptr) return BITNET_ERR_NULL;
  if (!aligned(w, 4)) return BITNET_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  const unsigned zero = 0;
  if (cudaMemcpyToSymbolAsync(g_pack_bad_value, &zero, sizeof zero, 0,
                              cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BITNET_ERR_CUDA;
  const int64_t total = N * (K / 4);
  DeviceInfo* dev = nullptr;
  bitnet_status s = device_info(&dev);
  if (s != BITNET_OK) return s;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8 * dev->sms) blocks = 8 * dev->sms;
  pack_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(w_packed, w, total);
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned bad = 0;
  if (cudaMemcpyFromSymbolAsync(&bad, g_pack_bad_value, sizeof bad, 0,
                                cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BITNET_ERR_CUDA;
  return bad ? BITNET_ERR_VALUE : BITNET_OK;
}

bitnet_status bitnet_ternarize_absmean(int8_t* w_t, float* scale_wt, const float* w, int64_t N,
                                       int64_t K, int per_row, void* stream) {
  if (N < 0 || K <= 0 || K > INT32_MAX || K % (per_row ? 4 : 16) != 0 || N > INT32_MAX)
    return BITNET_ERR_SHAPE;
  if (N == 0) return BITNET_OK;
  if (w_t == nullptr || scale_wt == nullptr || w == nullptr) return BITNET_ERR_NULL;
  if (!aligned(w, 16) || !aligned(w_t, 16) || !aligned(scale_wt, 4)) return BITNET_ERR_ALIGN;
  cudaStream_t st = as_stream(stream);
  const unsigned zero = 0;
  if (cudaMemcpyToSymbolAsync(g_ternarize_bad, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                              st) != cudaSuccess)
    return BITNET_ERR_CUDA;
  const dim3 rows(static_cast<unsigned>(N)), block(kTernThreads);
  const int k = static_cast<int>(K);
  if (per_row) {
    ternarize_rows_kernel<<<rows, block, 0, st>>>(w_t, scale_wt, w, k);
  } else {
    ternarize_rowsum_kernel<<<rows, block, 0, st>>>(w_t, w, k);
    ternarize_total_kernel<<<1, block, 0, st>>>(scale_wt, w_t, N, k);
    ternarize_apply_kernel<<<rows, block, 0, st>>>(w_t, scale_wt, w, k);
    ternarize_round_scale_kernel<<<1, 32, 0, st>>>(scale_wt);
  }
  if (cudaGetLastError() != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned bad = 0;
  if (cudaMemcpyFromSymbolAsync(&bad, g_ternarize_bad, sizeof bad, 0, cudaMemcpyDeviceToHost,
                                st) != cudaSuccess)
    return BITNET_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BITNET_ERR_CUDA;
  return bad ? BITNET_ERR_VALUE : BITNET_OK;
}

bitnet_status bitnet_quantize_act(int8_t* x_q, uint16_t* scale_act, const void* x,
                                  bitnet_dtype dt, int64_t M, int64_t K, void* stream) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (M < 0 || K <= 0 || K % 32 != 0 || K > INT32_MAX) return BITNET_ERR_SHAPE;
  if (M == 0) return BITNET_OK;
  if (x_q == nullptr || scale_act == nullptr || x == nullptr) return BITNET_ERR_NULL;
  if (!aligned(x, 16) || !aligned(x_q, 16) || !aligned(scale_act, 2)) return BITNET_ERR_ALIGN;
  if (dt == BITNET_F32)
    return run_quantize_f32(x_q, scale_act, static_cast<const float*>(x), M, K, as_stream(stream));
  return run_quantize(x_q, scale_act, static_cast<const uint16_t*>(x), M, K,
                      as_stream(stream));
}

bitnet_status bitnet_gemm(uint16_t* out, const int8_t* x_q, const uint8_t* w_packed,
                          const uint16_t* scale_act, const float* scale_wt,
                          int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                          void* stream) {
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M == 0 || N == 0) return BITNET_OK;
  if (out == nullptr || x_q == nullptr || w_packed == nullptr || scale_act == nullptr)
    return BITNET_ERR_NULL;
  s = check_scale_wt(scale_wt, scale_wt_len, N);
  if (s != BITNET_OK) return s;
  if (!aligned(out, 16) || !aligned(x_q, 16) || !aligned(w_packed, 16) ||
      !aligned(scale_act, 2))
    return BITNET_ERR_ALIGN;
  return run_gemm(out, false, x_q, w_packed, scale_act, scale_wt, scale_wt_len, M, N, K,
                  as_stream(stream));
}

bitnet_status bitnet_gemm_acc_i32(int32_t* acc, const int8_t* x_q, const uint8_t* w_packed,
                                  int64_t M, int64_t N, int64_t K, void* stream) {
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M == 0 || N == 0) return BITNET_OK;
  if (acc == nullptr || x_q == nullptr || w_packed == nullptr) return BITNET_ERR_NULL;
  if (!aligned(acc, 16) || !aligned(x_q, 16) || !aligned(w_packed, 16)) return BITNET_ERR_ALIGN;
  return run_gemm(acc, true, x_q, w_packed, nullptr, nullptr, 1, M, N, K, as_stream(stream));
}

static bitnet_status gemv_common(GemvParams& p, const void* x, bitnet_dtype dt,
                                 const uint8_t* w_packed, int64_t M, int64_t N, int64_t K) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M < 1 || M > kGemvMaxM || !gemv_fits(static_cast<int>(M), K)) return BITNET_ERR_SHAPE;
  if (x == nullptr || w_packed == nullptr) return BITNET_ERR_NULL;
  if (!aligned(x, 16) || !aligned(w_packed, 16)) return BITNET_ERR_ALIGN;
  p.x = x;
  p.x_f32 = dt == BITNET_F32 ? 1 : 0;
  p.wp = w_packed;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  return BITNET_OK;
}

// Packed bytes from which a single fused GEMV of one or two rows takes the
// grouped kernel (the 2B model's LM head, 82 MB, does; its layers do not).
constexpr int64_t kGemvViaGroupedBytes = int64_t(32) << 20;

// Where the accumulator hooks send their results: int32 sums instead of the
// bf16 outputs, and the int8 codes [M, K] (natural order) and bf16 scales [M]
// the path quantised. Null for every product call.
struct AccHook {
  int32_t* acc;
  int8_t* q;
  uint16_t* sa;
};

// The fused GEMV's dispatch (shared by bitnet_gemv_fused, bitnet_linear at
// M < 16 and the accumulator hook): the tensor-core GEMV for 8 <= M < 16
// where it applies, else the dp4a GEMV.
static bitnet_status gemv_fused_impl(uint16_t* out, const void* x, bitnet_dtype dt,
                                     const uint8_t* w_packed, const float* scale_wt,
                                     int64_t scale_wt_len, const uint16_t* bias, int64_t M,
                                     int64_t N, int64_t K, void* stream,
                                     const uint16_t* norm_g = nullptr, float norm_eps = 0.0f,
                                     const AccHook* hook = nullptr) {
  GemvParams p = {};
  bitnet_status s = gemv_common(p, x, dt, w_packed, M, N, K);
  if (s != BITNET_OK) return s;
  if (N == 0) return BITNET_OK;
  if (hook == nullptr) {
    if (out == nullptr) return BITNET_ERR_NULL;
    if (!aligned(out, 16)) return BITNET_ERR_ALIGN;
    s = check_scale_wt(scale_wt, scale_wt_len, N);
    if (s != BITNET_OK) return s;
    if (bias != nullptr && !aligned(bias, 2)) return BITNET_ERR_ALIGN;
    p.out = out;
    p.sw = scale_wt;
    p.sw_len = static_cast<int>(scale_wt_len);
    p.bias = bias;
  } else {
    p.acc_out = hook->acc;
    p.dbg_q = hook->q;
    p.dbg_sa = hook->sa;
    p.sw_len = 1;
  }
  p.norm_g = norm_g;
  p.norm_eps = norm_eps;
  // One or two activation rows against a large weight matrix (an LM head):
  // the grouped kernel's one-problem launch (units of up to 80 KB, one CTA
  // per SM, one problem's activations staged once per CTA) streams the
  // weights faster than the single-call kernel's tiling.
  if (M <= 2 && norm_g == nullptr && bias == nullptr && dt == BITNET_BF16 && K % 64 == 0 &&
      N * (K / 4) >= kGemvViaGroupedBytes && aligned(x, 16) && aligned(w_packed, 16)) {
    bitnet_gemv_problem q{hook == nullptr ? out : static_cast<uint16_t*>(static_cast<void*>(hook->acc)),
                          x, w_packed, scale_wt, scale_wt_len, N, K};
    return hook == nullptr ? run_gemv_grouped(&q, 1, static_cast<int>(M), as_stream(stream))
                           : run_gemv_grouped_acc(&q, &hook->q, &hook->sa, 1, static_cast<int>(M),
                                                  as_stream(stream));
  }
  if (norm_g == nullptr && dt == BITNET_BF16 && skq_ok(x, w_packed, M, K) &&
      (K + skq::BKS - 1) / skq::BKS <= sk::MAX_SPLIT * (skq::MAX_KB / 4)) {
    const bitnet_status r =
        hook == nullptr
            ? run_gemv_skq(out, static_cast<const uint16_t*>(x), w_packed, scale_wt,
                           scale_wt_len, M, N, K, as_stream(stream), bias)
            : run_gemv_skq(hook->acc, static_cast<const uint16_t*>(x), w_packed, nullptr, 1, M,
                           N, K, as_stream(stream), nullptr, true, hook->q, hook->sa);
    if (r != BITNET_ERR_SHAPE) return r;
  }
  return run_gemv(p, false, as_stream(stream));
}

bitnet_status bitnet_gemv_fused(uint16_t* out, const void* x, bitnet_dtype dt,
                                const uint8_t* w_packed, const float* scale_wt,
                                int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                                void* stream) {
  return gemv_fused_impl(out, x, dt, w_packed, scale_wt, scale_wt_len, nullptr, M, N, K, stream);
}

// The grouped GEMV's dispatch: problems with K % 64 == 0 and bf16 rows go
// to the grouped kernel, up to kGroupMax per launch; the rest are single
// calls. hq / hsa (the accumulator hook, else null): where each problem's
// codes and scales go; each problem's `out` is then its int32 output.
static bitnet_status grouped_impl(const bitnet_gemv_problem* problems, int64_t count, int64_t M,
                                  bitnet_dtype dt, void* stream, int8_t* const* hq,
                                  uint16_t* const* hsa) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  if (count < 0) return BITNET_ERR_SHAPE;
  if (count == 0) return BITNET_OK;
  if (problems == nullptr) return BITNET_ERR_NULL;
  const bool hook = hq != nullptr;
  // validate everything before anything is enqueued
  for (int64_t i = 0; i < count; ++i) {
    const bitnet_gemv_problem& q = problems[i];
    GemvParams p = {};
    bitnet_status s = gemv_common(p, q.x, dt, q.w_packed, M, q.N, q.K);
    if (s != BITNET_OK) return s;
    if (q.N == 0) continue;
    if (q.out == nullptr) return BITNET_ERR_NULL;
    if (!aligned(q.out, 16)) return BITNET_ERR_ALIGN;
    if (hook) {
      if (hq[i] == nullptr || hsa[i] == nullptr) return BITNET_ERR_NULL;
      if (!aligned(hq[i], 16) || !aligned(hsa[i], 2)) return BITNET_ERR_ALIGN;
    } else {
      s = check_scale_wt(q.scale_wt, q.scale_wt_len, q.N);
      if (s != BITNET_OK) return s;
    }
  }
  cudaStream_t st = as_stream(stream);
  bitnet_gemv_problem batch[kGroupMax];
  int8_t* bq[kGroupMax];
  uint16_t* bsa[kGroupMax];
  int n = 0;
  auto flush = [&]() -> bitnet_status {
    const int k = n;
    n = 0;
    return hook ? run_gemv_grouped_acc(batch, bq, bsa, k, static_cast<int>(M), st)
                : run_gemv_grouped(batch, k, static_cast<int>(M), st);
  };
  for (int64_t i = 0; i < count; ++i) {
    const bitnet_gemv_problem& q = problems[i];
    if (q.N == 0) continue;
    if (q.K % 64 != 0 || dt == BITNET_F32) {  // its own launch (the grouped kernel reads bf16)
      bitnet_status s;
      if (hook) {
        const AccHook h{static_cast<int32_t*>(static_cast<void*>(q.out)), hq[i], hsa[i]};
        s = gemv_fused_impl(nullptr, q.x, dt, q.w_packed, nullptr, 1, nullptr, M, q.N, q.K, stream,
                            nullptr, 0.0f, &h);
      } else {
        s = bitnet_gemv_fused(q.out, q.x, dt, q.w_packed, q.scale_wt, q.scale_wt_len, M, q.N,
                              q.K, stream);
      }
      if (s != BITNET_OK) return s;
      continue;
    }
    batch[n] = q;
    if (hook) {
      bq[n] = hq[i];
      bsa[n] = hsa[i];
    }
    if (++n == kGroupMax) {
      bitnet_status s = flush();
      if (s != BITNET_OK) return s;
    }
  }
  if (n > 0) return flush();
  return BITNET_OK;
}

bitnet_status bitnet_gemv_fused_grouped(const bitnet_gemv_problem* problems, int64_t count,
                                        int64_t M, bitnet_dtype dt, void* stream) {
  return grouped_impl(problems, count, M, dt, stream, nullptr, nullptr);
}

bitnet_status bitnet_gemv_fused_grouped_acc_i32(const bitnet_gemv_problem* problems,
                                                int8_t* const* x_q, uint16_t* const* scale_act,
                                                int64_t count, int64_t M, bitnet_dtype dt,
                                                void* stream) {
  if (count > 0 && (x_q == nullptr || scale_act == nullptr)) return BITNET_ERR_NULL;
  return grouped_impl(problems, count, M, dt, stream, x_q, scale_act);
}

bitnet_status bitnet_gemv_fused_debug(int32_t* acc, int8_t* x_q, uint16_t* scale_act,
                                      const void* x, bitnet_dtype dt,
                                      const uint8_t* w_packed, int64_t M, int64_t N,
                                      int64_t K, void* stream) {
  GemvParams p = {};
  bitnet_status s = gemv_common(p, x, dt, w_packed, M, N, K);
  if (s != BITNET_OK) return s;
  if (acc == nullptr || x_q == nullptr || scale_act == nullptr) return BITNET_ERR_NULL;
  if (!aligned(acc, 16) || !aligned(x_q, 16) || !aligned(scale_act, 2)) return BITNET_ERR_ALIGN;
  p.acc_out = acc;
  p.dbg_q = x_q;
  p.dbg_sa = scale_act;
  p.sw_len = 1;
  if (N == 0) p.N = 0;  // still quantises (block 0) with no weight rows
  return run_gemv(p, false, as_stream(stream));
}

size_t bitnet_linear_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  if (linear_uses_gemv(M, K)) return 0;
  // int8 activations [M, K], bf16 scales [M], int32 per-row code sums [M]
  return align256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
         align256(static_cast<size_t>(M) * 2) + align256(static_cast<size_t>(M) * 4);
}

// bitnet_linear's dispatch (shared with bitnet_linear_bias,
// bitnet_linear_noalloc and the accumulator hook): M < 16 -> the fused GEMV;
// else the quantiser into the workspace, then the GEMM.
static bitnet_status linear_impl(uint16_t* out, const void* x, bitnet_dtype dt,
                                 const uint8_t* w_packed, const float* scale_wt,
                                 int64_t scale_wt_len, const uint16_t* bias, int64_t M, int64_t N,
                                 int64_t K, void* workspace, size_t workspace_bytes,
                                 void* stream, const AccHook* hook = nullptr) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M == 0 || N == 0) return BITNET_OK;
  if (linear_uses_gemv(M, K))
    return gemv_fused_impl(out, x, dt, w_packed, scale_wt, scale_wt_len, bias, M, N, K, stream,
                           nullptr, 0.0f, hook);
  if (bias != nullptr && !aligned(bias, 2)) return BITNET_ERR_ALIGN;
  const size_t need = bitnet_linear_workspace_bytes(M, K);
  if (workspace == nullptr || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return BITNET_ERR_ALIGN;
  if (x == nullptr || w_packed == nullptr) return BITNET_ERR_NULL;
  if (hook == nullptr) {
    if (out == nullptr) return BITNET_ERR_NULL;
    s = check_scale_wt(scale_wt, scale_wt_len, N);
    if (s != BITNET_OK) return s;
    if (!aligned(out, 16)) return BITNET_ERR_ALIGN;
  }
  if (!aligned(x, 16) || !aligned(w_packed, 16)) return BITNET_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  uint16_t* sa = reinterpret_cast<uint16_t*>(ws + align256(static_cast<size_t>(M) * K));
  int32_t* rowsum = reinterpret_cast<int32_t*>(ws + align256(static_cast<size_t>(M) * K) +
                                               align256(static_cast<size_t>(M) * 2));
  cudaStream_t st = as_stream(stream);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const float* xf = static_cast<const float*>(x);
  const bool tc = gemm_tc_ok(xq, w_packed, K);
  if (tc) {
    // tensor-core path: transposed groups + row sums, weights as code planes
    s = dt == BITNET_F32 ? run_quantize_perm_f32(xq, sa, rowsum, xf, M, K, st)
                         : run_quantize_perm(xq, sa, rowsum, xb, M, K, st);
  } else {
    s = dt == BITNET_F32 ? run_quantize_f32(xq, sa, xf, M, K, st)
                         : run_quantize(xq, sa, xb, M, K, st);
  }
  if (s != BITNET_OK) return s;
  if (hook == nullptr)
    return run_gemm(out, false, xq, w_packed, sa, scale_wt, scale_wt_len, M, N, K, st, tc,
                    tc ? rowsum : nullptr, bias);
  s = run_gemm(hook->acc, true, xq, w_packed, sa, nullptr, 1, M, N, K, st, tc,
               tc ? rowsum : nullptr, nullptr);
  if (s != BITNET_OK) return s;
  return copy_workspace_codes(hook->q, hook->sa, xq, sa, M, K, tc, st);
}

bitnet_status bitnet_linear(uint16_t* out, const void* x, bitnet_dtype dt,
                            const uint8_t* w_packed, const float* scale_wt,
                            int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return linear_impl(out, x, dt, w_packed, scale_wt, scale_wt_len, nullptr, M, N, K, workspace,
                     workspace_bytes, stream);
}

bitnet_status bitnet_linear_bias(uint16_t* out, const void* x, bitnet_dtype dt,
                                 const uint8_t* w_packed, const float* scale_wt,
                                 int64_t scale_wt_len, const uint16_t* bias, int64_t M,
                                 int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (bias == nullptr) return BITNET_ERR_NULL;
  return linear_impl(out, x, dt, w_packed, scale_wt, scale_wt_len, bias, M, N, K, workspace,
                     workspace_bytes, stream);
}

bitnet_status bitnet_linear_acc_i32(int32_t* acc, int8_t* x_q, uint16_t* scale_act,
                                    const void* x, bitnet_dtype dt, const uint8_t* w_packed,
                                    int64_t M, int64_t N, int64_t K, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M == 0 || N == 0) return BITNET_OK;
  if (acc == nullptr || x_q == nullptr || scale_act == nullptr) return BITNET_ERR_NULL;
  if (!aligned(acc, 16) || !aligned(x_q, 16) || !aligned(scale_act, 2)) return BITNET_ERR_ALIGN;
  const AccHook hook{acc, x_q, scale_act};
  return linear_impl(nullptr, x, dt, w_packed, nullptr, 1, nullptr, M, N, K, workspace,
                     workspace_bytes, stream, &hook);
}

bitnet_status bitnet_linear_noalloc(uint16_t* out, const void* x, bitnet_dtype dt,
                                    const uint8_t* w_packed, const float* scale_wt,
                                    int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                                    void* stream) {
  if (dt != BITNET_BF16 && dt != BITNET_F32) return BITNET_ERR_DTYPE;
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (M == 0 || N == 0) return BITNET_OK;
  if (out == nullptr || x == nullptr || w_packed == nullptr) return BITNET_ERR_NULL;
  if (linear_uses_gemv(M, K))  // the fused GEMV needs no scratch
    return bitnet_gemv_fused(out, x, dt, w_packed, scale_wt, scale_wt_len, M, N, K, stream);
  const size_t need = bitnet_linear_workspace_bytes(M, K);
  if (need > kNoAllocScratchBytes) return BITNET_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != BITNET_OK) return s;
  // x_q and the scales are written in full by the quantiser before the GEMM
  // reads them, so nothing left from an earlier call is ever used.
  return bitnet_linear(out, x, dt, w_packed, scale_wt, scale_wt_len, M, N, K, scratch,
                       kNoAllocScratchBytes, stream);
}

// ------------------------------------------------ RMSNorm -> quantise

static bitnet_status run_rmsnorm_quant(int8_t* xq, uint16_t* sa, int32_t* rowsum,
                                       const uint16_t* x, const uint16_t* g, float eps,
                                       int64_t M, int64_t K, int mode, cudaStream_t st) {
  if (M == 0) return BITNET_OK;
  if (M > INT32_MAX) return BITNET_ERR_SHAPE;
  const dim3 grid(static_cast<unsigned>(M)), block(kTernThreads);
  const int k = static_cast<int>(K);
  const int64_t per_thread = (K / 16 + kTernThreads - 1) / kTernThreads;  // 16-element groups
  if (per_thread <= 4) {
#define BITNET_RMS_REG(MODE, NG)                                                                  \
  return launch_pdl(rmsnorm_quant_reg_kernel<MODE, NG>, grid, block, 0, st, xq, sa, rowsum, x, g, \
                    eps, k)
#define BITNET_RMS_REG_NG(MODE)       \
  if (per_thread <= 1) BITNET_RMS_REG(MODE, 1); \
  if (per_thread <= 2) BITNET_RMS_REG(MODE, 2); \
  BITNET_RMS_REG(MODE, 4)
    if (mode == kRmsPerm) { BITNET_RMS_REG_NG(kRmsPerm); }
    if (mode == kRmsZ) { BITNET_RMS_REG_NG(kRmsZ); }
    BITNET_RMS_REG_NG(kRmsCodes);
#undef BITNET_RMS_REG_NG
#undef BITNET_RMS_REG
  }
  if (mode == kRmsPerm)
    return launch_pdl(rmsnorm_quant_kernel<kRmsPerm>, grid, block, 0, st, xq, sa, rowsum, x, g,
                      eps, k);
  if (mode == kRmsZ)
    return launch_pdl(rmsnorm_quant_kernel<kRmsZ>, grid, block, 0, st, xq, sa, rowsum, x, g, eps,
                      k);
  return launch_pdl(rmsnorm_quant_kernel<kRmsCodes>, grid, block, 0, st, xq, sa, rowsum, x, g,
                    eps, k);
}

bitnet_status bitnet_rmsnorm_quantize_act(int8_t* x_q, uint16_t* scale_act, const uint16_t* x,
                                          const uint16_t* g, float eps, int64_t M, int64_t K,
                                          void* stream) {
  if (M < 0 || K <= 0 || K % 32 != 0 || K > INT32_MAX) return BITNET_ERR_SHAPE;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BITNET_ERR_VALUE;
  if (M == 0) return BITNET_OK;
  if (x_q == nullptr || scale_act == nullptr || x == nullptr || g == nullptr)
    return BITNET_ERR_NULL;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(x_q, 16) || !aligned(scale_act, 2))
    return BITNET_ERR_ALIGN;
  return run_rmsnorm_quant(x_q, scale_act, nullptr, x, g, eps, M, K, kRmsCodes,
                           as_stream(stream));
}

// One or two rows of up to 16384 that the fused GEMV takes: the GEMV's
// register-cached staging normalises them itself (one launch, no scratch).
bool rmsnorm_in_gemv(int64_t M, int64_t K) { return M <= 2 && K <= 16384 && linear_uses_gemv(M, K); }

size_t bitnet_linear_rmsnorm_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  if (rmsnorm_in_gemv(M, K)) return 0;
  if (linear_uses_gemv(M, K)) return align256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
  return align256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
         align256(static_cast<size_t>(M) * 2) + align256(static_cast<size_t>(M) * 4);
}

bitnet_status bitnet_linear_rmsnorm(uint16_t* out, const uint16_t* x, const uint16_t* g,
                                    float eps, const uint8_t* w_packed, const float* scale_wt,
                                    int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  bitnet_status s = check_compute_shape(M, N, K);
  if (s != BITNET_OK) return s;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BITNET_ERR_VALUE;
  if (M == 0 || N == 0) return BITNET_OK;
  const size_t need = bitnet_linear_rmsnorm_workspace_bytes(M, K);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BITNET_ERR_WORKSPACE;
  if (need > 0 && !aligned(workspace, 256)) return BITNET_ERR_ALIGN;
  if (out == nullptr || x == nullptr || g == nullptr || w_packed == nullptr)
    return BITNET_ERR_NULL;
  s = check_scale_wt(scale_wt, scale_wt_len, N);
  if (s != BITNET_OK) return s;
  if (!aligned(out, 16) || !aligned(x, 16) || !aligned(g, 16) || !aligned(w_packed, 16))
    return BITNET_ERR_ALIGN;
  if (rmsnorm_in_gemv(M, K))
    return gemv_fused_impl(out, x, BITNET_BF16, w_packed, scale_wt, scale_wt_len, nullptr, M, N, K,
                           stream, g, eps);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = as_stream(stream);
  if (linear_uses_gemv(M, K)) {
    // few rows: the normalised bf16 rows, then the fused GEMV quantises them
    int8_t* z = reinterpret_cast<int8_t*>(ws);
    s = run_rmsnorm_quant(z, nullptr, nullptr, x, g, eps, M, K, kRmsZ, st);
    if (s != BITNET_OK) return s;
    return gemv_fused_impl(out, z, BITNET_BF16, w_packed, scale_wt, scale_wt_len, nullptr, M, N,
                           K, stream);
  }
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  uint16_t* sa = reinterpret_cast<uint16_t*>(ws + align256(static_cast<size_t>(M) * K));
  int32_t* rowsum = reinterpret_cast<int32_t*>(ws + align256(static_cast<size_t>(M) * K) +
                                               align256(static_cast<size_t>(M) * 2));
  const bool tc = gemm_tc_ok(xq, w_packed, K);
  s = run_rmsnorm_quant(xq, sa, rowsum, x, g, eps, M, K, tc ? kRmsPerm : kRmsCodes, st);
  if (s != BITNET_OK) return s;
  if (tc)
    return run_gemm(out, false, xq, w_packed, sa, scale_wt, scale_wt_len, M, N, K, st, true,
                    rowsum);
  return run_gemm(out, false, xq, w_packed, sa, scale_wt, scale_wt_len, M, N, K, st);
}

bitnet_status bitnet_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return BITNET_ERR_CUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess)
      return BITNET_ERR_CUDA;
    return (v & kDevErrTimeout) ? BITNET_ERR_TIMEOUT : BITNET_ERR_VALUE;
  }
  return BITNET_OK;
}

}  // extern "C"
