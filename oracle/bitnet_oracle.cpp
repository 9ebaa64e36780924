// BitNet b1.58 W1.58A8 linear layer: plain scalar CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. This file is the checker that the CUDA library is
// compared against. Nothing in the product path includes, links or calls it;
// only the tests, the smoke check and the bench's CPU-baseline leg do.
// It shares no source, header, table or helper with the CUDA library.
//
// Every function is the plain definition of one step, written in the order
// and notation of the bitnet-cpu page (torch-ext/bitnet_cpu/__init__.py):
//   pack        pack_weights(): code = w + 2, four codes per byte, element 0
//               in the low two bits.
//   unpack      the inverse the pack docstring states: w = code - 2.
//   quantize    quantize_activation(): per-row absmax clamped at eps = 1e-5,
//               scale = absmax / 127, q = clamp(round(x / scale), -127, 127),
//               scale returned as bf16.
//   acc         the int32 ternary x int8 contraction of bitnet_gemm().
//   epilogue    out = bf16(acc * scale_act * scale_wt) in fp32.
//   linear      bitnet_linear(): quantize, then gemm. The fused GEMV of the
//               same page (M < 16) must give the same result, because the
//               bitnet-tc announcement (kernels-community README discussion)
//               states bit-exactness across every dispatch path.
//
// Readings of points the pages leave open (each listed in the design notes):
//   * bf16 input is converted to fp32 before the absmax, the division and the
//     rounding (the torch expression on the page would run in bf16);
//   * the rounding of x / scale is round-half-to-even (torch.round);
//   * the division is a true IEEE fp32 division by the unrounded fp32 scale;
//   * the epilogue multiplies in the order (acc * scale_act) * scale_wt, with
//     scale_act the stored bf16 scale widened to fp32;
//   * code 0b00, which pack never produces, decodes to -2 (code - 2).
//
// Build: g++ -O2 -ffp-contract=off (no -ffast-math), see oracle/build.py.

#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// bf16 <-> fp32, written out from the IEEE formats: bf16 is the top 16 bits
// of an fp32; narrowing rounds to nearest, ties to even.
inline float bf16_bits_to_float(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

inline uint16_t float_to_bf16_bits_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) {
    return static_cast<uint16_t>((u >> 16) | 0x0040u);  // quiet NaN
  }
  const uint32_t lower = u & 0xFFFFu;
  uint32_t upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
  return static_cast<uint16_t>(upper);
}

// Status codes shared in meaning (not in source) with the library's ABI.
enum { OK = 0, ERR_SHAPE = 2, ERR_VALUE = 5, ERR_RANGE = 9 };

}  // namespace

extern "C" {

// pack_weights: w int8 [N, K] in {-1, 0, +1} -> packed uint8 [N, K/4].
// Byte j of row n holds elements 4j..4j+3; element 4j+i sits in bits 2i..2i+1.
int oracle_pack(const int8_t* w, int64_t N, int64_t K, uint8_t* packed) {
  if (N < 0 || K < 0 || K % 4 != 0) return ERR_SHAPE;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      const int v = w[n * K + k];
      if (v < -1 || v > 1) return ERR_VALUE;
    }
  }
  const int64_t KB = K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < KB; ++j) {
      unsigned byte = 0;
      for (int i = 0; i < 4; ++i) {
        const unsigned code = static_cast<unsigned>(w[n * K + 4 * j + i] + 2);
        byte |= code << (2 * i);
      }
      packed[n * KB + j] = static_cast<uint8_t>(byte);
    }
  }
  return OK;
}

// Decode: w = code - 2 for each of the four 2-bit fields of a byte.
int oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* w) {
  if (N < 0 || K < 0 || K % 4 != 0) return ERR_SHAPE;
  const int64_t KB = K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      const unsigned byte = packed[n * KB + k / 4];
      const int code = static_cast<int>((byte >> (2 * (k % 4))) & 3u);
      w[n * K + k] = static_cast<int8_t>(code - 2);
    }
  }
  return OK;
}

// quantize_activation for one row of K fp32 values: absmax clamped at
// eps = 1e-5, s = absmax / 127 (IEEE fp32 division), q = clamp(round-half-
// even(x / s), -127, 127), scale = bf16(s).
static void quantize_row(const float* row, int64_t K, int8_t* q, uint16_t* scale) {
  float absmax = 0.0f;
  for (int64_t k = 0; k < K; ++k) {
    const float a = std::fabs(row[k]);
    if (a > absmax) absmax = a;
  }
  if (absmax < 1e-5f) absmax = 1e-5f;  // clamp(min=eps)
  const float s = absmax / 127.0f;
  for (int64_t k = 0; k < K; ++k) {
    const float v = row[k] / s;
    float r = std::nearbyint(v);  // half-to-even under FE_TONEAREST
    if (r < -127.0f) r = -127.0f;
    if (r > 127.0f) r = 127.0f;
    q[k] = static_cast<int8_t>(r);
  }
  *scale = float_to_bf16_bits_rne(s);
}

// quantize_activation for bf16 rows x [M, K] (given as raw bf16 bits; each
// value is widened to fp32 exactly first). q int8 [M, K]; scale bf16 [M]
// (raw bits).
int oracle_quantize(const uint16_t* x, int64_t M, int64_t K, int8_t* q,
                    uint16_t* scale) {
  if (M < 0 || K <= 0) return ERR_SHAPE;
  std::fesetround(FE_TONEAREST);
  std::vector<float> row(static_cast<size_t>(K));
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) row[k] = bf16_bits_to_float(x[m * K + k]);
    quantize_row(row.data(), K, q + m * K, scale + m);
  }
  return OK;
}

// quantize_activation for fp32 rows x [M, K] (the bitnet-cpu page accepts
// float32 activations as well as bf16).
int oracle_quantize_f32(const float* x, int64_t M, int64_t K, int8_t* q,
                        uint16_t* scale) {
  if (M < 0 || K <= 0) return ERR_SHAPE;
  std::fesetround(FE_TONEAREST);
  for (int64_t m = 0; m < M; ++m) quantize_row(x + m * K, K, q + m * K, scale + m);
  return OK;
}

// acc[m, n] = sum_k q[m, k] * w[n, k], w decoded from the packed bytes.
// Summed in int64; ERR_RANGE if a result does not fit int32.
int oracle_acc(const int8_t* q, const uint8_t* packed, int64_t M, int64_t N,
               int64_t K, int32_t* acc) {
  if (M < 0 || N < 0 || K < 0 || K % 4 != 0) return ERR_SHAPE;
  const int64_t KB = K / 4;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) {
        const unsigned byte = packed[n * KB + k / 4];
        const int w = static_cast<int>((byte >> (2 * (k % 4))) & 3u) - 2;
        sum += static_cast<int64_t>(q[m * K + k]) * w;
      }
      if (sum > INT32_MAX || sum < INT32_MIN) return ERR_RANGE;
      acc[m * N + n] = static_cast<int32_t>(sum);
    }
  }
  return OK;
}

// out[m, n] = bf16( (float(acc) * float(scale_act[m])) * scale_wt[n or 0] ).
int oracle_epilogue(const int32_t* acc, const uint16_t* scale_act,
                    const float* scale_wt, int64_t scale_wt_len, int64_t M,
                    int64_t N, uint16_t* out) {
  if (M < 0 || N < 0) return ERR_SHAPE;
  if (scale_wt_len != 1 && scale_wt_len != N) return ERR_SHAPE;
  for (int64_t m = 0; m < M; ++m) {
    const float sa = bf16_bits_to_float(scale_act[m]);
    for (int64_t n = 0; n < N; ++n) {
      const float sw = scale_wt[scale_wt_len == 1 ? 0 : n];
      const float a = static_cast<float>(acc[m * N + n]);
      const float t = a * sa;
      const float y = t * sw;
      out[m * N + n] = float_to_bf16_bits_rne(y);
    }
  }
  return OK;
}

// bitnet_gemm: int8 activations with bf16 row scales x packed ternary weights.
int oracle_gemm(const int8_t* q, const uint8_t* packed,
                const uint16_t* scale_act, const float* scale_wt,
                int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                uint16_t* out) {
  std::vector<int32_t> acc(static_cast<size_t>(M) * static_cast<size_t>(N));
  int st = oracle_acc(q, packed, M, N, K, acc.data());
  if (st != OK) return st;
  return oracle_epilogue(acc.data(), scale_act, scale_wt, scale_wt_len, M, N,
                         out);
}

// bitnet_linear (and the fused GEMV, which must agree with it): quantize the
// bf16 rows, then gemm.
int oracle_linear(const uint16_t* x, const uint8_t* packed,
                  const float* scale_wt, int64_t scale_wt_len, int64_t M,
                  int64_t N, int64_t K, uint16_t* out) {
  std::vector<int8_t> q(static_cast<size_t>(M) * static_cast<size_t>(K));
  std::vector<uint16_t> sa(static_cast<size_t>(M));
  int st = oracle_quantize(x, M, K, q.data(), sa.data());
  if (st != OK) return st;
  return oracle_gemm(q.data(), packed, sa.data(), scale_wt, scale_wt_len, M, N,
                     K, out);
}

// bitnet_linear for fp32 rows: quantize_f32, then gemm.
int oracle_linear_f32(const float* x, const uint8_t* packed, const float* scale_wt,
                      int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                      uint16_t* out) {
  std::vector<int8_t> q(static_cast<size_t>(M) * static_cast<size_t>(K));
  std::vector<uint16_t> sa(static_cast<size_t>(M));
  int st = oracle_quantize_f32(x, M, K, q.data(), sa.data());
  if (st != OK) return st;
  return oracle_gemm(q.data(), packed, sa.data(), scale_wt, scale_wt_len, M, N,
                     K, out);
}

// The same linear with the output rows split across host threads (each row
// is still the scalar definition above); used only to time the oracle.
int oracle_linear_threads(const uint16_t* x, const uint8_t* packed,
                          const float* scale_wt, int64_t scale_wt_len,
                          int64_t M, int64_t N, int64_t K, uint16_t* out,
                          int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (M < nthreads) nthreads = static_cast<int>(M > 0 ? M : 1);
  std::vector<int> status(static_cast<size_t>(nthreads), OK);
  std::vector<std::thread> pool;
  const int64_t per = (M + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t m0 = t * per;
    const int64_t m1 = (m0 + per < M) ? m0 + per : M;
    if (m0 >= m1) continue;
    pool.emplace_back([=, &status] {
      status[static_cast<size_t>(t)] =
          oracle_linear(x + m0 * K, packed, scale_wt, scale_wt_len, m1 - m0, N,
                        K, out + m0 * N);
    });
  }
  for (auto& th : pool) th.join();
  for (int s : status)
    if (s != OK) return s;
  return OK;
}

// The gemm (pre-quantised rows) split across host threads, for timing.
int oracle_gemm_threads(const int8_t* q, const uint8_t* packed,
                        const uint16_t* scale_act, const float* scale_wt,
                        int64_t scale_wt_len, int64_t M, int64_t N, int64_t K,
                        uint16_t* out, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (M < nthreads) nthreads = static_cast<int>(M > 0 ? M : 1);
  std::vector<int> status(static_cast<size_t>(nthreads), OK);
  std::vector<std::thread> pool;
  const int64_t per = (M + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t m0 = t * per;
    const int64_t m1 = (m0 + per < M) ? m0 + per : M;
    if (m0 >= m1) continue;
    pool.emplace_back([=, &status] {
      status[static_cast<size_t>(t)] =
          oracle_gemm(q + m0 * K, packed, scale_act + m0, scale_wt,
                      scale_wt_len, m1 - m0, N, K, out + m0 * N);
    });
  }
  for (auto& th : pool) th.join();
  for (int s : status)
    if (s != OK) return s;
  return OK;
}

// The same linear with the output columns split across host threads: the
// rows are quantised once, then each thread runs the scalar contraction and
// epilogue above for its slice of weight rows. Used only to time the oracle
// at small M (decode), where a row split would leave threads idle.
int oracle_linear_threads_cols(const uint16_t* x, const uint8_t* packed,
                               const float* scale_wt, int64_t scale_wt_len,
                               int64_t M, int64_t N, int64_t K, uint16_t* out,
                               int nthreads) {
  if (M < 0 || N < 0 || K <= 0 || K % 4 != 0) return ERR_SHAPE;
  if (scale_wt_len != 1 && scale_wt_len != N) return ERR_SHAPE;
  std::vector<int8_t> q(static_cast<size_t>(M) * static_cast<size_t>(K));
  std::vector<uint16_t> sa(static_cast<size_t>(M));
  int st = oracle_quantize(x, M, K, q.data(), sa.data());
  if (st != OK) return st;
  if (nthreads < 1) nthreads = 1;
  if (N < nthreads) nthreads = static_cast<int>(N > 0 ? N : 1);
  std::vector<int> status(static_cast<size_t>(nthreads), OK);
  std::vector<std::thread> pool;
  const int64_t per = (N + nthreads - 1) / nthreads;
  const int64_t KB = K / 4;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t n0 = t * per;
    const int64_t n1 = (n0 + per < N) ? n0 + per : N;
    if (n0 >= n1) continue;
    pool.emplace_back([=, &q, &sa, &status] {
      const int64_t nn = n1 - n0;
      std::vector<int32_t> acc(static_cast<size_t>(M) * static_cast<size_t>(nn));
      std::vector<uint16_t> part(static_cast<size_t>(M) * static_cast<size_t>(nn));
      int s = oracle_acc(q.data(), packed + n0 * KB, M, nn, K, acc.data());
      if (s == OK)
        s = oracle_epilogue(acc.data(), sa.data(),
                            scale_wt + (scale_wt_len == 1 ? 0 : n0),
                            scale_wt_len == 1 ? 1 : nn, M, nn, part.data());
      if (s == OK)
        for (int64_t m = 0; m < M; ++m)
          for (int64_t n = 0; n < nn; ++n)
            out[m * N + n0 + n] = part[static_cast<size_t>(m * nn + n)];
      status[static_cast<size_t>(t)] = s;
    });
  }
  for (auto& th : pool) th.join();
  for (int s : status)
    if (s != OK) return s;
  return OK;
}

// oracle_acc with the weight rows (output columns) split across host
// threads: each thread runs the scalar definition above on its slice. Only
// the order in which independent outputs are computed changes, so the
// result is oracle_acc's; used where a full-size comparison needs it fast.
int oracle_acc_threads(const int8_t* q, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                       int32_t* acc, int nthreads) {
  if (M < 0 || N < 0 || K < 0 || K % 4 != 0) return ERR_SHAPE;
  if (nthreads < 1) nthreads = 1;
  if (N < nthreads) nthreads = static_cast<int>(N > 0 ? N : 1);
  std::vector<int> status(static_cast<size_t>(nthreads), OK);
  std::vector<std::thread> pool;
  const int64_t per = (N + nthreads - 1) / nthreads;
  const int64_t KB = K / 4;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t n0 = t * per;
    const int64_t n1 = (n0 + per < N) ? n0 + per : N;
    if (n0 >= n1) continue;
    pool.emplace_back([=, &status] {
      const int64_t nn = n1 - n0;
      std::vector<int32_t> part(static_cast<size_t>(M) * static_cast<size_t>(nn));
      const int s = oracle_acc(q, packed + n0 * KB, M, nn, K, part.data());
      if (s == OK)
        for (int64_t m = 0; m < M; ++m)
          for (int64_t n = 0; n < nn; ++n) acc[m * N + n0 + n] = part[static_cast<size_t>(m * nn + n)];
      status[static_cast<size_t>(t)] = s;
    });
  }
  for (auto& th : pool) th.join();
  for (int s : status)
    if (s != OK) return s;
  return OK;
}

// Narrowing used by the oracle, exposed so a test can pin it against a
// library conversion on its own.
uint16_t oracle_f32_to_bf16(float f) { return float_to_bf16_bits_rne(f); }

// bitnet_linear followed by the layer's bias (BitLinear.forward on the
// bitnet-cpu page: y = bitnet_linear(...); y = y + bias, both bf16): the
// bf16 output of the layer plus the bf16 bias, added in fp32 and rounded to
// bf16 again. bias is bf16 [N] (raw bits).
int oracle_linear_bias(const uint16_t* x, const uint8_t* packed, const float* scale_wt,
                       int64_t scale_wt_len, const uint16_t* bias, int64_t M, int64_t N,
                       int64_t K, uint16_t* out) {
  int st = oracle_linear(x, packed, scale_wt, scale_wt_len, M, N, K, out);
  if (st != OK) return st;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      const float y = bf16_bits_to_float(out[m * N + n]) + bf16_bits_to_float(bias[n]);
      out[m * N + n] = float_to_bf16_bits_rne(y);
    }
  return OK;
}

// ------------------------------------------------------------------------
// Absmean ternarisation (bitnet-cpu page: BitLinear.from_dense per output
// row, gamma clamped at 1e-8; BitLinearKernel per tensor, clamped at 1e-5):
//   gamma = max(mean |w|, eps), code = clamp(round-half-even(w / gamma), -1, 1),
//   scale = bf16(gamma).
// Reading of the mean (the page computes it with a float32 reduction, whose
// result depends on the summation order): the sum of |w| is exact, as an
// integer in units of 2^-64 (|w| * 2^64 truncated toward zero: exact for
// |w| >= 2^-40, and |w| < 2^47 is required), then
// mean = float(double(sum) / count * 2^-64) with each operation rounded to
// nearest even. Integer addition does not depend on the order.

typedef unsigned __int128 u128;

static bool abs_fixed(float w, u128* out) {
  if (!std::isfinite(w)) return false;
  const float a = std::fabs(w);
  if (a >= 140737488355328.0f) return false;  // 2^47
  if (a == 0.0f) {
    *out = 0;
    return true;
  }
  int e = 0;
  const float fr = std::frexp(a, &e);  // a = fr * 2^e, fr in [0.5, 1)
  const uint64_t m = static_cast<uint64_t>(std::ldexp(fr, 24));  // 24-bit integer
  const int sh = e - 24 + 64;  // a * 2^64 = m * 2^sh
  if (sh >= 0) *out = static_cast<u128>(m) << sh;
  else if (sh > -64) *out = static_cast<u128>(m >> (-sh));
  else *out = 0;
  return true;
}

static float mean_of(u128 sum, int64_t count) {
  const double d = static_cast<double>(sum) / static_cast<double>(count);
  return static_cast<float>(std::ldexp(d, -64));
}

static void ternarize_row(const float* w, int64_t K, float gamma, int8_t* wt) {
  for (int64_t k = 0; k < K; ++k) {
    float r = std::nearbyint(w[k] / gamma);  // half-to-even under FE_TONEAREST
    if (r < -1.0f) r = -1.0f;
    if (r > 1.0f) r = 1.0f;
    wt[k] = static_cast<int8_t>(r);
  }
}

// per_row != 0: scale [N]; per_row == 0: one gamma for the tensor, scale [1].
// scale holds bf16(gamma) widened to fp32. ERR_VALUE for non-finite or huge
// weights.
int oracle_ternarize_absmean(const float* w, int64_t N, int64_t K, int per_row, int8_t* wt,
                             float* scale) {
  if (N < 0 || K <= 0) return ERR_SHAPE;
  std::fesetround(FE_TONEAREST);
  if (per_row) {
    for (int64_t n = 0; n < N; ++n) {
      u128 s = 0;
      for (int64_t k = 0; k < K; ++k) {
        u128 a;
        if (!abs_fixed(w[n * K + k], &a)) return ERR_VALUE;
        s += a;
      }
      float gamma = mean_of(s, K);
      if (gamma < 1e-8f) gamma = 1e-8f;
      ternarize_row(w + n * K, K, gamma, wt + n * K);
      scale[n] = bf16_bits_to_float(float_to_bf16_bits_rne(gamma));
    }
    return OK;
  }
  u128 s = 0;
  for (int64_t i = 0; i < N * K; ++i) {
    u128 a;
    if (!abs_fixed(w[i], &a)) return ERR_VALUE;
    s += a;
  }
  float gamma = N > 0 ? mean_of(s, N * K) : 1e-5f;
  if (gamma < 1e-5f) gamma = 1e-5f;
  for (int64_t n = 0; n < N; ++n) ternarize_row(w + n * K, K, gamma, wt + n * K);
  scale[0] = bf16_bits_to_float(float_to_bf16_bits_rne(gamma));
  return OK;
}

// ------------------------------------------------------------------------
// RMSNorm before the quantiser (BitLinearKernel on the bitnet-cpu page runs
// the module's rms_norm on its input first). The page does not spell the norm
// out; the reading is the usual RMSNorm in fp32 with its weight g applied to
// the result cast back to bf16:
//   var = mean(x^2), r = 1 / sqrt(var + eps), y = bf16(x * r), z = bf16(g * y),
// then quantize_activation(z). The sum of squares is exact (each x^2 of a bf16
// x is exact in fp32, summed as an integer in units of 2^-64, as for the
// absmean), var = float(double(sum) / K * 2^-64), sqrt and 1/. are IEEE.
// ERR_VALUE when some |x| >= 2^23 (x^2 would leave the exact range).

int oracle_rmsnorm(const uint16_t* x, const uint16_t* g, float eps, int64_t M, int64_t K,
                   uint16_t* z) {
  if (M < 0 || K <= 0) return ERR_SHAPE;
  std::fesetround(FE_TONEAREST);
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t* row = x + m * K;
    u128 s = 0;
    for (int64_t k = 0; k < K; ++k) {
      const float v = bf16_bits_to_float(row[k]);
      if (!(std::fabs(v) < 8388608.0f)) return ERR_VALUE;  // 2^23, also NaN
      u128 a;
      if (!abs_fixed(v * v, &a)) return ERR_VALUE;
      s += a;
    }
    const float var = mean_of(s, K);
    const float r = 1.0f / std::sqrt(var + eps);
    for (int64_t k = 0; k < K; ++k) {
      const float y = bf16_bits_to_float(float_to_bf16_bits_rne(bf16_bits_to_float(row[k]) * r));
      z[m * K + k] = float_to_bf16_bits_rne(bf16_bits_to_float(g[k]) * y);
    }
  }
  return OK;
}

int oracle_rmsnorm_quantize(const uint16_t* x, const uint16_t* g, float eps, int64_t M,
                            int64_t K, int8_t* q, uint16_t* scale) {
  std::vector<uint16_t> z(static_cast<size_t>(M) * static_cast<size_t>(K));
  int st = oracle_rmsnorm(x, g, eps, M, K, z.data());
  if (st != OK) return st;
  return oracle_quantize(z.data(), M, K, q, scale);
}

int oracle_linear_rmsnorm(const uint16_t* x, const uint16_t* g, float eps,
                          const uint8_t* packed, const float* scale_wt, int64_t scale_wt_len,
                          int64_t M, int64_t N, int64_t K, uint16_t* out) {
  std::vector<uint16_t> z(static_cast<size_t>(M) * static_cast<size_t>(K));
  int st = oracle_rmsnorm(x, g, eps, M, K, z.data());
  if (st != OK) return st;
  return oracle_linear(z.data(), packed, scale_wt, scale_wt_len, M, N, K, out);
}

}  // extern "C"
