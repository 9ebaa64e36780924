/* bitnet.h — C ABI of libbitnet_b200: the BitNet b1.58 W1.58A8 linear layer
 * (ternary weights x per-token INT8 activations) on NVIDIA B200 (sm_100a).
 *
 * The operations are the ones the bitnet-cpu page (torch-ext/bitnet_cpu/
 * __init__.py) defines for the bitnet-tc kernel family:
 *   pack_weights, quantize_activation, bitnet_gemm, bitnet_gemv_fused and
 *   bitnet_linear (dispatch by M).
 *
 * Conventions for every entry point
 *   - Outputs come first, as in the native ops that page calls.
 *   - All array pointers are caller-owned DEVICE pointers on the current CUDA
 *     device; the library keeps no reference to them after the call returns.
 *     Matrices are dense and row-major (last index contiguous).
 *   - bf16 values are passed as their raw 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL means the legacy default stream). All
 *     work is enqueued asynchronously on it; only bitnet_pack_weights and
 *     bitnet_device_status synchronise it.
 *   - Arguments are validated before anything is launched; on any error the
 *     call returns a status other than BITNET_OK and enqueues nothing.
 *   - Shapes: M (tokens), N (output features), K (input features).
 *     Compute entry points need K > 0 and K % 32 == 0 (the page's BitLinear
 *     asserts in_features % 32 == 0); M == 0 or N == 0 is a valid no-op.
 *   - Alignment: x, x_q, w_packed and out must be 16-byte aligned; scale
 *     arrays need their natural alignment.
 *   - Kernels are launched with programmatic stream serialisation: a kernel
 *     of this library may begin while the preceding kernel on the stream is
 *     still running, and reads `w_packed` / `scale_wt` before waiting for it.
 *     Weights and weight scales are therefore load-time constants: they must
 *     not be written by a kernel that is still running on the same stream
 *     when the call is enqueued (bitnet_pack_weights synchronises, so its
 *     output is always safe). Activations and outputs are ordered normally.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BITNET_OK = 0,
  BITNET_ERR_NULL = 1,      /* a required pointer is NULL */
  BITNET_ERR_SHAPE = 2,     /* M, N, K or a length is out of range */
  BITNET_ERR_DTYPE = 3,     /* activation dtype not supported */
  BITNET_ERR_ALIGN = 4,     /* a pointer is not aligned as required */
  BITNET_ERR_VALUE = 5,     /* pack: a weight is outside {-1, 0, +1} */
  BITNET_ERR_WORKSPACE = 6, /* workspace NULL or smaller than required */
  BITNET_ERR_CUDA = 7,      /* a CUDA runtime call or launch failed */
  BITNET_ERR_TIMEOUT = 8    /* a kernel gave up a bounded wait (device) */
} bitnet_status;

typedef enum {
  BITNET_BF16 = 0, /* activations in bf16 */
  BITNET_F32 = 1   /* activations in float32 (the bitnet-cpu page accepts
                      both); other values are rejected */
} bitnet_dtype;

/* Pack ternary weights into 2-bit codes, four per byte.
 * Defined by pack_weights() on the bitnet-cpu page: code = w + 2
 * (-1 -> 1, 0 -> 2, +1 -> 3); byte j of row n holds elements 4j..4j+3 of
 * that row, element 4j+i in bits 2i..2i+1 (element 0 in the low bits).
 *   w_packed  out, uint8 [N, K/4]
 *   w         in,  int8  [N, K], values in {-1, 0, +1}
 * Needs K % 4 == 0 (the page's assert). Synchronises `stream` to report
 * BITNET_ERR_VALUE when any input value is outside {-1, 0, +1}; in that case
 * the contents of w_packed are unspecified. */
bitnet_status bitnet_pack_weights(uint8_t* w_packed, const int8_t* w,
                                  int64_t N, int64_t K, void* stream);

/* Absmean ternarisation of float32 weights, the step before packing:
 * BitLinear.from_dense on the bitnet-cpu page (per_row != 0: one gamma per
 * output row, clamped at 1e-8) or BitLinearKernel (per_row == 0: one gamma
 * for the tensor, clamped at 1e-5):
 *   gamma = max(mean |w|, eps), w_t = clamp(round-half-even(w / gamma), -1, 1),
 *   scale_wt = bf16(gamma), returned widened to fp32.
 * The mean's sum is exact (|w| * 2^64 truncated toward zero, summed as an
 * integer), then mean = float(double(sum) / count * 2^-64): the result does
 * not depend on any summation order.
 *   w_t       out, int8 [N, K] ternary (then bitnet_pack_weights)
 *   scale_wt  out, fp32 [N] (per_row) or [1]
 *   w         in,  fp32 [N, K], finite, |w| < 2^47
 * K % 4 == 0 (per row) or K % 16 == 0 (per tensor; the row sums pass through
 * w_t). Synchronises the stream to report BITNET_ERR_VALUE for a weight that
 * is not finite or too large. */
bitnet_status bitnet_ternarize_absmean(int8_t* w_t, float* scale_wt, const float* w,
                                       int64_t N, int64_t K, int per_row, void* stream);

/* Per-token absmax INT8 activation quantisation.
 * Defined by quantize_activation() on the bitnet-cpu page: for each row m,
 * absmax = max_k |x[m,k]| clamped below at 1e-5, s = absmax / 127 (fp32,
 * IEEE division), x_q[m,k] = clamp(round_half_even(x[m,k] / s), -127, 127),
 * scale_act[m] = bf16(s) (round to nearest even). bf16 inputs are widened to
 * fp32 before any arithmetic.
 *   x_q        out, int8 [M, K]
 *   scale_act  out, bf16 [M]
 *   x          in,  [M, K] of dtype `dt` (BITNET_BF16 or BITNET_F32) */
bitnet_status bitnet_quantize_act(int8_t* x_q, uint16_t* scale_act,
                                  const void* x, bitnet_dtype dt, int64_t M,
                                  int64_t K, void* stream);

/* Ternary x INT8 GEMM with the scale epilogue (bitnet_gemm() on the bitnet-cpu
 * page; batched tensor-core path of the bitnet-tc announcement):
 *   acc[m,n] = sum_k x_q[m,k] * (code(w_packed[n], k) - 2)   (exact int32)
 *   out[m,n] = bf16( (fp32(acc) * fp32(scale_act[m])) * scale_wt[n or 0] )
 *   out        out, bf16 [M, N]
 *   x_q        in,  int8 [M, K]
 *   w_packed   in,  uint8 [N, K/4]
 *   scale_act  in,  bf16 [M]
 *   scale_wt   in,  fp32, scale_wt_len elements: 1 (per tensor) or N
 * Any M >= 0. Kernels: with K % 64 == 0 and 16-byte aligned x_q and
 * w_packed, M <= 256 runs a tensor-core kernel whose K loop is split over a
 * thread-block cluster, and larger M a persistent tensor-core kernel;
 * otherwise a SIMT kernel. The persistent kernel also takes 129..192 rows
 * when the N / 128 weight tiles fill at least half the SMs (one wave of
 * 192-row tiles), and M <= 256 with K > 131008 (the others' int32 sums of
 * 64 * w could overflow). All give the same result. */
bitnet_status bitnet_gemm(uint16_t* out, const int8_t* x_q,
                          const uint8_t* w_packed, const uint16_t* scale_act,
                          const float* scale_wt, int64_t scale_wt_len,
                          int64_t M, int64_t N, int64_t K, void* stream);

/* Fused quantise + ternary GEMV for decode (bitnet_gemv_fused() on the
 * bitnet-cpu page; the fused dp4a GEMV of the bitnet-tc announcement).
 * Same result, bit for bit, as bitnet_quantize_act followed by bitnet_gemm.
 *   out       out, bf16 [M, N]
 *   x         in,  [M, K] of dtype `dt` (BITNET_BF16 or BITNET_F32)
 *   w_packed, scale_wt, scale_wt_len as for bitnet_gemm.
 * Needs 1 <= M <= 15 (the page dispatches M < 16 here), and the quantised
 * rows plus one stage of sixteen weight rows must fit on chip:
 * 2048 + c(M * K) + c(4 * K) <= 232448 with c(v) = v rounded up to a
 * multiple of 128 (about (M + 4) * K <= 230000); otherwise BITNET_ERR_SHAPE.
 * Kernels: with 8 <= M, K % 64 == 0, 16-byte aligned x and w_packed and
 * K <= 128 * 8 * min(48, floor(384 / M)), a tensor-core kernel with the
 * quantisation inside (its K loop split over a thread-block cluster);
 * otherwise a dp4a GEMV (always for BITNET_F32). Both give the same result. */
bitnet_status bitnet_gemv_fused(uint16_t* out, const void* x, bitnet_dtype dt,
                                const uint8_t* w_packed, const float* scale_wt,
                                int64_t scale_wt_len, int64_t M, int64_t N,
                                int64_t K, void* stream);

/* One problem of a grouped decode call (see bitnet_gemv_fused_grouped):
 * the arguments of one bitnet_gemv_fused call, M excepted. */
typedef struct {
  uint16_t* out;            /* bf16 [M, N] */
  const void* x;            /* [M, K] of the group's dtype */
  const uint8_t* w_packed;  /* uint8 [N, K/4] */
  const float* scale_wt;    /* fp32, scale_wt_len elements: 1 or N */
  int64_t scale_wt_len;
  int64_t N;
  int64_t K;
} bitnet_gemv_problem;

/* Many independent bitnet_gemv_fused problems with the same M, in as few
 * launches as possible (one per 256 problems). Each problem's result is the
 * one bitnet_gemv_fused gives, bit for bit. Independent means: no problem
 * reads what another one of the same call writes. Use it for the decode
 * projections that share no data dependency (e.g. Q, K, V of a layer, or the
 * independent calls of a sweep); one persistent launch streams all their
 * weights back to back instead of paying a launch and a prologue per call.
 *   problems  in, HOST array of `count` problem descriptors (read during
 *             the call, not kept)
 * Each problem obeys bitnet_gemv_fused's rules. Problems whose K is not a
 * multiple of 64, and every problem of a BITNET_F32 call, are computed by
 * their own bitnet_gemv_fused launch. The whole call is validated before
 * anything is enqueued. */
bitnet_status bitnet_gemv_fused_grouped(const bitnet_gemv_problem* problems,
                                        int64_t count, int64_t M,
                                        bitnet_dtype dt, void* stream);

/* Workspace bitnet_linear needs for (M, K): 0 when it takes the fused GEMV
 * path, otherwise room for the int8 [M, K] activations, the bf16 [M] scales
 * and int32 [M] per-row sums of the codes, each 256-byte aligned. The layout
 * inside the workspace is private to the library. */
size_t bitnet_linear_workspace_bytes(int64_t M, int64_t K);

/* One-shot BitLinear forward (bitnet_linear() on the bitnet-cpu page):
 * M < 16 (and the fused GEMV's size limit met) -> bitnet_gemv_fused;
 * otherwise bitnet_quantize_act into `workspace`, then bitnet_gemm.
 * The page's version allocates its intermediates; a C ABI takes them from
 * the caller instead: `workspace` (device memory, 256-byte aligned) of at
 * least bitnet_linear_workspace_bytes(M, K) bytes, or NULL when that is 0. */
bitnet_status bitnet_linear(uint16_t* out, const void* x, bitnet_dtype dt,
                            const uint8_t* w_packed, const float* scale_wt,
                            int64_t scale_wt_len, int64_t M, int64_t N,
                            int64_t K, void* workspace, size_t workspace_bytes,
                            void* stream);

/* bitnet_linear followed by the layer's bias, fused into the epilogue
 * (BitLinear.forward on the bitnet-cpu page: y = bitnet_linear(...) + bias,
 * a bf16 addition):
 *   out[m,n] = bf16( fp32(y[m,n]) + fp32(bias[n]) ), y the bf16 result of
 *   bitnet_linear.
 *   bias  in, bf16 [N] (2-byte aligned, not NULL)
 * The other arguments, the workspace and the result are bitnet_linear's. */
bitnet_status bitnet_linear_bias(uint16_t* out, const void* x, bitnet_dtype dt,
                                 const uint8_t* w_packed, const float* scale_wt,
                                 int64_t scale_wt_len, const uint16_t* bias, int64_t M,
                                 int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* RMSNorm fused with the per-token quantiser (BitLinearKernel on the
 * bitnet-cpu page applies the module's rms_norm to its input first). The norm
 * is the usual fp32 RMSNorm with its weight applied after the cast back to
 * bf16, per row:
 *   r = 1 / sqrt(mean(x^2) + eps)   (the sum of squares exact, sqrt and /
 *                                    IEEE fp32)
 *   z = bf16(g * bf16(x * r)),  then quantize_activation(z)
 *   x_q, scale_act  out, as bitnet_quantize_act
 *   x               in,  bf16 [M, K], |x| < 2^23 (else bitnet_device_status
 *                        reports BITNET_ERR_VALUE)
 *   g               in,  bf16 [K], the norm's weight
 *   eps             the norm's epsilon: finite and > 0 (else BITNET_ERR_VALUE;
 *                   a zero row would otherwise divide by zero)
 * K % 32 == 0; x, g and x_q 16-byte aligned. */
bitnet_status bitnet_rmsnorm_quantize_act(int8_t* x_q, uint16_t* scale_act, const uint16_t* x,
                                          const uint16_t* g, float eps, int64_t M, int64_t K,
                                          void* stream);

/* Workspace of bitnet_linear_rmsnorm for (M, K), in bytes. There are three
 * cases:
 *   - M <= 2 and K <= 16384, where bitnet_linear takes the fused GEMV: 0.
 *     The GEMV normalises the rows itself, in one launch.
 *   - Otherwise, where bitnet_linear takes the fused GEMV (M < 16 and the
 *     GEMV's fit rule): the normalised bf16 [M, K] rows, which the GEMV then
 *     quantises.
 *   - Otherwise: the int8 [M, K] codes, the bf16 [M] scales and the int32 [M]
 *     code sums.
 * Each part is 256-byte aligned. The size is 0 for M == 0. */
size_t bitnet_linear_rmsnorm_workspace_bytes(int64_t M, int64_t K);

/* RMSNorm, quantiser and the layer in one call, on the caller's stream. The
 * result equals bitnet_linear applied to bf16(g * bf16(x * r)).
 *   - M <= 2, K <= 16384: the fused GEMV normalises the rows in its own
 *     staging (one launch; workspace unused, may be NULL).
 *   - Otherwise the norm's kernel writes into `workspace` (the quantised
 *     rows, or for few rows the bf16 normalised rows), then the kernels of
 *     bitnet_linear run on it.
 * Arguments as bitnet_rmsnorm_quantize_act and bitnet_linear; x is bf16,
 * workspace 256-byte aligned. */
bitnet_status bitnet_linear_rmsnorm(uint16_t* out, const uint16_t* x, const uint16_t* g,
                                    float eps, const uint8_t* w_packed, const float* scale_wt,
                                    int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* bitnet_linear without a caller workspace, for callers that cannot allocate
 * device memory themselves: code inside a framework that owns all device
 * memory through its own pool and hands out none for a library's scratch, or
 * a latency-critical path that cannot afford an allocation's implicit
 * synchronisation. The bitnet-cpu page has no counterpart; this is a
 * convenience of this library's C ABI.
 * Arguments and result are those of bitnet_linear. When M >= 16 (the split
 * path), the int8 activations and their scales are placed in a scratch array
 * built into the library: 16 MiB (16777216 bytes) per GPU, reserved by every
 * GPU that loads the library until the process exits. Shapes whose
 * bitnet_linear_workspace_bytes(M, K) exceeds it return BITNET_ERR_WORKSPACE
 * and enqueue nothing. The call allocates nothing.
 * The first call on a device looks up the scratch's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. The address is kept for the life of the process: it does not
 * survive a reset of the device's context (cudaDeviceReset), after which this
 * entry point must not be called again in the same process. Every call on a device shares the one scratch array: calls that
 * may run at the same time on the GPU (different streams without ordering
 * between them) race on it and must not overlap. Calls ordered on one stream
 * are safe; each call overwrites whatever an earlier call left there. */
bitnet_status bitnet_linear_noalloc(uint16_t* out, const void* x,
                                    bitnet_dtype dt, const uint8_t* w_packed,
                                    const float* scale_wt, int64_t scale_wt_len,
                                    int64_t M, int64_t N, int64_t K,
                                    void* stream);

/* Synchronise `stream`, then read and clear the device-side error word the
 * kernels set when a bounded wait gives up. BITNET_ERR_TIMEOUT if it was
 * set (the outputs of the affected call are then unspecified), BITNET_OK
 * otherwise, BITNET_ERR_CUDA if the synchronisation itself failed. */
bitnet_status bitnet_device_status(void* stream);

/* Human-readable name of a status. Never NULL. */
const char* bitnet_status_string(bitnet_status s);

/* ---- test hooks: the same kernels with the epilogue replaced ------------
 * Exist so that the exact int32 accumulators (and the fused path's int8
 * codes and scales) can be compared bit for bit with a reference, as the
 * bitnet-tc announcement's "bit-exact across every dispatch path" needs. */

/* The batched GEMM kernel storing acc[m, n] (int32 [M, N]) instead of bf16. */
bitnet_status bitnet_gemm_acc_i32(int32_t* acc, const int8_t* x_q,
                                  const uint8_t* w_packed, int64_t M,
                                  int64_t N, int64_t K, void* stream);

/* The fused GEMV kernel storing acc[m, n] (int32 [M, N]) instead of bf16, and
 * the int8 codes [M, K] and bf16 scales [M] it quantised on chip. */
bitnet_status bitnet_gemv_fused_debug(int32_t* acc, int8_t* x_q,
                                      uint16_t* scale_act, const void* x,
                                      bitnet_dtype dt, const uint8_t* w_packed,
                                      int64_t M, int64_t N, int64_t K,
                                      void* stream);

/* bitnet_linear's own dispatch and kernels (the fused GEMVs for M < 16; the
 * quantiser into `workspace`, then the split-K or persistent GEMM on the
 * tensor-core layout, or the SIMT path, for M >= 16) with the epilogue
 * replaced: acc (int32 [M, N], 16-byte aligned) receives the exact sums,
 * x_q (int8 [M, K], natural order, 16-byte aligned) the codes and scale_act
 * (bf16 [M]) the scales the path quantised. Arguments otherwise as
 * bitnet_linear (no weight scale is read). */
bitnet_status bitnet_linear_acc_i32(int32_t* acc, int8_t* x_q, uint16_t* scale_act,
                                    const void* x, bitnet_dtype dt, const uint8_t* w_packed,
                                    int64_t M, int64_t N, int64_t K, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* bitnet_gemv_fused_grouped's own dispatch and kernel with the epilogue
 * replaced: problems[i].out is problem i's int32 [M, N_i] output (16-byte
 * aligned; scale_wt is not read); x_q[i] (int8 [M, K_i], 16-byte aligned) and
 * scale_act[i] (bf16 [M]) receive the codes and scales it quantised. x_q and
 * scale_act are host arrays of `count` device pointers. */
bitnet_status bitnet_gemv_fused_grouped_acc_i32(const bitnet_gemv_problem* problems,
                                                int8_t* const* x_q, uint16_t* const* scale_act,
                                                int64_t count, int64_t M, bitnet_dtype dt,
                                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
