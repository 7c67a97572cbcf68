// Host-side packing of expert weights into 4-bit block-scaled formats, once at load time
// (the weights are constant across steps, like the router's prepared split weight).
//
// Source: handbook digest (agihunt.info), "已确认", bullet "量化与推理": Kimi K3's routed
// experts in MXFP4; NVIDIA's NVFP4 training with key layers kept in BF16.  The pages name
// the formats only; the layouts followed are
//   element  FP4 E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
//            0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7), no infinity or NaN;
//   MXFP4    32 elements share a power-of-two scale 2^E stored as E8M0 (E + 127), with
//            E = floor(log2 amax) - 2, clamped to [-127, 127] (-127 for an all-zero block);
//   NVFP4    16 elements share an FP8 E4M3 scale s_b = E4M3(amax_block / 6 / s_t), and the
//            tensor shares an fp32 scale s_t = amax / (6 * 448) (1 for an all-zero tensor);
//            a block whose scale rounds to 0 stores zeros.
// Elements are w / scale rounded to the nearest E2M1 value, ties to the even mantissa
// bit, magnitudes above 6 saturating.  Storage: codes [rows, K/2] bytes, element 2j in
// the low nibble of byte j and 2j+1 in the high nibble; scales [rows, K/block] bytes.
// All arithmetic is in double from the fp32 inputs; rows are split across host threads.
#include <math.h>

#include <algorithm>
#include <thread>
#include <vector>

#include "common.cuh"

namespace moe {
namespace {

// Nearest E2M1 code of v.  Between consecutive magnitudes the midpoint goes to the even
// code (mantissa bit 0): 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2,
// 3.5 -> 4, 5 -> 4; beyond 5 the code of 6 (saturation).
uint8_t e2m1_code(double v) {
  const double a = fabs(v);
  uint8_t c;
  if (a <= 0.25) c = 0;
  else if (a < 0.75) c = 1;
  else if (a <= 1.25) c = 2;
  else if (a < 1.75) c = 3;
  else if (a <= 2.5) c = 4;
  else if (a < 3.5) c = 5;
  else if (a <= 5.0) c = 6;
  else c = 7;
  return (uint8_t)(signbit(v) ? (c | 8) : c);
}

double e2m1_value(uint8_t code) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double m = mag[code & 7];
  return (code & 8) ? -m : m;
}

// Nearest E4M3 value of a > 0 (ties to even through nearbyint's default mode), saturating
// at 448.  Spacing 2^(e-3) in binade e >= -6; the subnormals share 2^-9.
double e4m3_value(double a) {
  if (a >= 448.0) return 448.0;
  if (a <= 0.0) return 0.0;
  int ex;
  frexp(a, &ex);                              // a = f * 2^ex, f in [0.5, 1)
  const int e = std::max(ex - 1, -6);
  const double r = nearbyint(ldexp(a, 3 - e));
  return std::min(ldexp(r, e - 3), 448.0);
}

uint8_t e4m3_byte(double v) {               // v: 0 or a positive E4M3 value
  if (v <= 0.0) return 0;
  int ex;
  frexp(v, &ex);
  const int e = ex - 1;
  if (e < -6) return (uint8_t)lrint(ldexp(v, 9));                      // subnormal: v / 2^-9
  return (uint8_t)(((e + 7) << 3) | (int)lrint(ldexp(v, 3 - e) - 8.0));  // (1 + m/8) 2^e
}

double e4m3_from_byte(uint8_t b) {
  const int f = (b >> 3) & 15, m = b & 7;
  return f == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, f - 7);
}

template <typename Fn>
void for_rows(long long rows, int threads, Fn fn) {
  int n = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
  if (n < 1) n = 1;
  if (n > rows) n = (int)std::max(1LL, rows);
  if (n == 1) {
    fn(0LL, rows);
    return;
  }
  std::vector<std::thread> pool;
  const long long per = (rows + n - 1) / n;
  for (int i = 0; i < n; ++i) {
    const long long r0 = i * per, r1 = std::min(rows, r0 + per);
    if (r0 < r1) pool.emplace_back(fn, r0, r1);
  }
  for (auto& t : pool) t.join();
}

inline void put(uint8_t* codes, long long row, long long K, long long k, uint8_t c) {
  uint8_t& b = codes[row * (K / 2) + k / 2];
  b = (k & 1) ? (uint8_t)((b & 0x0f) | (c << 4)) : (uint8_t)((b & 0xf0) | c);
}

inline uint8_t get(const uint8_t* codes, long long row, long long K, long long k) {
  const uint8_t b = codes[row * (K / 2) + k / 2];
  return (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0x0f);
}

}  // namespace

int fp4_block(int fmt) { return fmt == MOE_FP4_MX ? 32 : (fmt == MOE_FP4_NV ? 16 : -1); }

moe_status quantize_fp4_host(const float* W, long long rows, long long K, int fmt, uint8_t* codes, uint8_t* scales,
                             float* tensor_scale, int threads) {
  const int B = fp4_block(fmt);
  const long long nb = K / B;
  double st = 1.0;
  if (fmt == MOE_FP4_NV) {
    // the tensor amax, reduced per row range (max is exact in any order)
    std::vector<double> rowmax(rows > 0 ? rows : 1, 0.0);
    for_rows(rows, threads, [&](long long r0, long long r1) {
      for (long long r = r0; r < r1; ++r) {
        double m = 0.0;
        for (long long k = 0; k < K; ++k) m = std::max(m, fabs((double)W[r * K + k]));
        rowmax[r] = m;
      }
    });
    double amax = 0.0;
    for (long long r = 0; r < rows; ++r) amax = std::max(amax, rowmax[r]);
    st = amax > 0.0 ? (double)(float)(amax / (6.0 * 448.0)) : 1.0;
    *tensor_scale = (float)st;
  }
  for_rows(rows, threads, [&](long long r0, long long r1) {
    for (long long r = r0; r < r1; ++r) {
      for (long long b = 0; b < nb; ++b) {
        const float* w = W + r * K + b * B;
        double amax = 0.0;
        for (int i = 0; i < B; ++i) amax = std::max(amax, fabs((double)w[i]));
        if (fmt == MOE_FP4_MX) {
          int E = -127;
          if (amax > 0.0) {
            int ex;
            frexp(amax, &ex);
            E = std::min(127, std::max(-127, ex - 1 - 2));    // floor(log2 amax) - 2
          }
          scales[r * nb + b] = (uint8_t)(E + 127);
          for (int i = 0; i < B; ++i) put(codes, r, K, b * B + i, e2m1_code(ldexp((double)w[i], -E)));
        } else {
          const double sb = e4m3_value(amax / 6.0 / st);
          scales[r * nb + b] = e4m3_byte(sb);
          for (int i = 0; i < B; ++i)
            put(codes, r, K, b * B + i, sb == 0.0 ? (uint8_t)0 : e2m1_code((double)w[i] / (sb * st)));
        }
      }
    }
  });
  return MOE_OK;
}

moe_status dequantize_fp4_host(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, long long rows,
                               long long K, int fmt, float* W, int threads) {
  const int B = fp4_block(fmt);
  const long long nb = K / B;
  const double st = fmt == MOE_FP4_NV ? (double)*tensor_scale : 1.0;
  for_rows(rows, threads, [&](long long r0, long long r1) {
    for (long long r = r0; r < r1; ++r)
      for (long long k = 0; k < K; ++k) {
        const uint8_t s = scales[r * nb + k / B];
        const double e = e2m1_value(get(codes, r, K, k));
        W[r * K + k] = fmt == MOE_FP4_MX ? (float)ldexp(e, (int)s - 127) : (float)(e * e4m3_from_byte(s) * st);
      }
  });
  return MOE_OK;
}

}  // namespace moe
