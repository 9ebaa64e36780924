// libbitnet_b200_waittest: the failure-path test library (tests only).
//
// It holds the decode GEMV kernel of gemv.cuh built with a 1 ms wait limit
// and one switch, g_wait_test_skip: the ring stage of CTA 0 that its producer
// leaves unrequested. The consumers waiting for that stage give up their
// bounded wait, set the device error word and return, the producer drains the
// copies it did issue, and the host reads BITNET_ERR_TIMEOUT from the status.
// The kernel holds no tensor memory. Every wait in it is bounded, so the
// context stays usable; the test then runs the same call without the skip.
// The product library (bitnet.cu) is built without any of this.
#define BITNET_WAIT_TEST 1
#define BITNET_WAIT_LIMIT_NS 1000000ull  // 1 ms

#include "../../include/bitnet.h"
#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {
namespace {

size_t round128(size_t v) { return (v + 127) & ~static_cast<size_t>(127); }

}  // namespace
}  // namespace bitnet

using namespace bitnet;

extern "C" {

// One activation row: out (bf16 [1, N]) = the fused GEMV of x (bf16 [1, K])
// with w_packed (uint8 [N, K/4]) and the per-tensor scale *scale_wt, through
// gemv_kernel with 16 consumer warps, one weight row per warp and stage and
// a four-stage ring. skip >= 0 leaves ring index `skip` of CTA 0 unrequested
// (-1: none). 64 <= K <= 4096, K % 64 == 0, 16-byte aligned pointers; N >= 1.
int bitnet_wait_test_gemv(uint16_t* out, const uint16_t* x, const uint8_t* w_packed,
                          const float* scale_wt, int64_t N, int64_t K, int skip, void* stream) {
  if (N < 1 || K < 64 || K % 64 != 0 || K > 4096 || N > (1 << 24)) return BITNET_ERR_SHAPE;
  if (out == nullptr || x == nullptr || w_packed == nullptr || scale_wt == nullptr)
    return BITNET_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyToSymbolAsync(g_wait_test_skip, &skip, sizeof skip, 0, cudaMemcpyHostToDevice,
                              st) != cudaSuccess)
    return BITNET_ERR_CUDA;
  constexpr int kCW = 16, kStages = 4;
  GemvParams p = {};
  p.out = out;
  p.x = x;
  p.wp = w_packed;
  p.sw = scale_wt;
  p.sw_len = 1;
  p.M = 1;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.rows_per_block = kCW;
  p.stages = kStages;
  p.q_bytes = static_cast<uint32_t>(round128(static_cast<size_t>(K)));
  p.stage_bytes = static_cast<uint32_t>(round128(static_cast<size_t>(kCW) * (K / 4)));
  const size_t smem = kGemvHeaderBytes + p.q_bytes + kStages * static_cast<size_t>(p.stage_bytes);
  auto k = gemv_kernel<kCW, 1, 1, true, false, false>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return BITNET_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return BITNET_ERR_CUDA;
  const int64_t nblocks = (N + kCW - 1) / kCW;
  const int grid = static_cast<int>(nblocks < sms ? nblocks : sms);
  k<<<grid, (kCW + 1) * 32, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

// Synchronise `stream`, then read and clear this library's device error
// word: BITNET_ERR_TIMEOUT if a wait gave up, else BITNET_OK.
int bitnet_wait_test_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BITNET_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return BITNET_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess)
    return BITNET_ERR_CUDA;
  return (v & kDevErrTimeout) ? BITNET_ERR_TIMEOUT : (v ? BITNET_ERR_VALUE : BITNET_OK);
}

}  // extern "C"
