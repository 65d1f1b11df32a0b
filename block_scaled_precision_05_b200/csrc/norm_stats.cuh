// norm_stats.cuh -- exactly rounded row statistics of the norms fused into the
// NVFP4 quantizers (the producer of a pre-quantized activation:
// hao-ai-lab-FastVideo nvfp4_config.py, NVFP4QuantizeMethod.apply with
// `pre_quantized` from a fused norm+quant call).
//
// The statistics are the exact values of their definitions over the bf16
// inputs, each rounded once to fp32 (round to nearest, ties to even):
//   RMSNorm    ms   = (1/K) sum x_k^2
//   LayerNorm  mean = (1/K) sum x_k,   var = (1/K) sum (x_k - mean_exact)^2
// Each one is decided in two steps, both warp-uniform:
//   1. fast: fp64 sums whose error has a proven bound, and the fp32 rounding
//      of the estimate.  When every real value within the bound of the
//      estimate rounds to that same fp32 (it stays clear of both neighbouring
//      rounding boundaries), it is the correctly rounded statistic.
//   2. otherwise (rows whose statistic lies within about 2^-46 relative of a
//      rounding boundary, or whose mean is 0 or nearly so): the exact sums as
//      integers -- each bf16 is m * 2^e with an 8-bit integer m -- accumulated
//      in shared memory, then an exact long division and the rounding.
// The error bounds (u = 2^-53, D = the additions any one term passes through:
// its lane's sequential sum plus the five levels of the warp butterfly):
//   - a sum of non-negative exact terms is within D*u/(1-D*u) of the exact sum
//     (relative); a signed sum within that times sum |terms|, and
//     sum |x| <= sqrt(K * sum x^2);
//   - multiplying by RN64(1/K) adds two roundings (2u relative);
//   - the LayerNorm variance is the fp64 mean of squares less the square of
//     the fp64 mean, with the bound of ln_fast;
//   - means of bf16 data often lie exactly halfway between two fp32 values
//     (the exact mean has few bits); when the fp64 sum of the row is provably
//     exact (ln_mean_exact) the mean is then decided exactly without the
//     integer path;
//   - every bound below carries a margin of several u (and the check itself is
//     done in fp64 with a margin that covers its own roundings).
#pragma once

#include <stdint.h>

namespace bsp {
namespace normstats {

constexpr double kU = 0x1p-53;

__device__ __forceinline__ double hi_word_double(uint32_t hi) { return __hiloint2double(static_cast<int>(hi), 0); }

// The two bf16 elements of a 32-bit word (element 0 in the low half) as fp32
// bit patterns.
__device__ __forceinline__ uint32_t f32_lo(uint32_t w) { return w << 16; }
__device__ __forceinline__ uint32_t f32_hi(uint32_t w) { return w & 0xFFFF0000u; }

// |x| * 2^-384 of the bf16 element with fp32 pattern f: the fp32 exponent and
// the 7 mantissa bits moved into an fp64 high word whose exponent is offset by
// 512.  Exact for every normal x; a zero or subnormal x gives a value below
// 2^-510 in place of |x| * 2^-384 (<= 2^-510 too), so its square is off by at
// most 2^-1020 (units of 2^-768).
__device__ __forceinline__ double mag_2m384(uint32_t f) {
  return hi_word_double(((f >> 3) & 0x0FFFE000u) | 0x20000000u);
}

// |x| * 2^-896 exactly for every finite x (zero and subnormals included: the
// fp32 exponent field becomes the fp64 one, whose bias is 896 larger).
__device__ __forceinline__ double mag_2m896(uint32_t f) { return hi_word_double((f >> 3) & 0x0FFFE000u); }

// +-2^512 with the sign of the element with fp32 pattern f.
__device__ __forceinline__ double sign_2p512(uint32_t f) { return hi_word_double((f & 0x80000000u) | 0x5FF00000u); }

// acc + x0^2 + x1^2 (units 2^-768) for the two elements of w: exact squares,
// one rounding per addition.
__device__ __forceinline__ double sumsq_word(uint32_t w, double acc) {
  const double d0 = mag_2m384(f32_lo(w)), d1 = mag_2m384(f32_hi(w));
  acc = fma(d0, d0, acc);
  return fma(d1, d1, acc);
}

__device__ __forceinline__ double sumsq8(const uint4& v, double acc) {
  acc = sumsq_word(v.x, acc);
  acc = sumsq_word(v.y, acc);
  acc = sumsq_word(v.z, acc);
  return sumsq_word(v.w, acc);
}

// The LayerNorm sums in real units: |x| exactly (|x| * 2^-896 from the bit
// pattern, zero and subnormals included, times 2^896) and +-1.0 carrying the
// sign, so that s1 + x and s2 + x^2 each round once and a zero adds exactly 0.
__device__ __forceinline__ void sums_elem(uint32_t f, double& s1, double& s2) {
  const double a = mag_2m896(f) * 0x1p896;
  const double sg = hi_word_double((f & 0x80000000u) | 0x3FF00000u);
  s1 = fma(a, sg, s1);
  s2 = fma(a, a, s2);
}

__device__ __forceinline__ void sums8(const uint4& v, double& s1, double& s2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sums_elem(f32_lo(w[i]), s1, s2);
    sums_elem(f32_hi(w[i]), s1, s2);
  }
}

// Running minimum, over 16-bit halves, of (|x| bits - 1) with a zero mapped
// to 0xFFFF: |x| + 0x7FFF cannot carry out of a half (|x| <= 0x7FFF), and the
// top bit of the sum is set exactly when |x| > 0, so flipping it gives
// |x| - 1 for a nonzero x and 0xFFFF for a zero.
__device__ __forceinline__ uint32_t min_nonzero_mag8(const uint4& v, uint32_t m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) m = __vminu2(m, ((w[i] & 0x7FFF7FFFu) + 0x7FFF7FFFu) ^ 0x80008000u);
  return m;
}

// Sum over the warp; every lane ends with the same bits (each butterfly step
// adds the same two values on both partners, and fp addition commutes).
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Additions a term of a row of K elements passes through: the lane's
// sequential sum (16 elements per group, groups strided over the 32 lanes),
// plus the butterfly, plus one.
__host__ __device__ __forceinline__ int sum_depth(int64_t K) { return static_cast<int>(16 * ((K + 511) / 512) + 6); }

// RN32(v) for a real v >= 0 known as v_hat with |v_hat - v| <= err: true (and
// the value in *out) when every real within err of v_hat rounds to the same
// fp32.  c = RN32(v_hat) rounds every real strictly within half the spacing to
// its neighbours; the test keeps [v_hat - err, v_hat + err] inside the smaller
// of the two halves, h: half an ulp of c (2^(e-151) for biased exponent e >= 1),
// a quarter at a power of two (the spacing below halves there), and 2^-150
// among the subnormals and zero.  |v_hat - c| is exact (c is within a factor
// two of v_hat, or both are below 2^-125 where the difference fits), and the
// final sum's rounding is covered by the margins the callers put in err.
__device__ __forceinline__ bool rn32_certain(double v_hat, double err, float* out) {
  if (!(v_hat >= 0.0) || !(err < 1e300)) return false;  // NaN / inf estimates: decided exactly
  const float c = __double2float_rn(v_hat);
  const uint32_t cb = __float_as_uint(c), e = cb >> 23;
  if (e >= 254u) return false;  // at the top of the fp32 range: decided exactly
  const uint32_t he = (e >= 2u && (cb & 0x7FFFFFu) == 0u) ? e - 1u : max(e, 1u);
  const double h = hi_word_double((he + 872u) << 20);  // 2^(he - 151)
  if (!(fabs(v_hat - static_cast<double>(c)) + err < h)) return false;
  *out = c;
  return true;
}

// ms = RN32(S / K) from s_hat = the fp64 sum of squares in units of 2^-768.
__device__ __forceinline__ bool ms_fast(double s_hat, int64_t K, double rK, float* ms) {
  const double v = (s_hat * 0x1p768) * rK;
  // sum: D u relative, plus at most K * 2^-1020 (units 2^-768) from zero and
  // subnormal elements, i.e. 2^-252 per element after the scaling; then 2u
  const double err = (2.0 * sum_depth(K) + 16.0) * kU * v + 0x1p-249;
  return rn32_certain(v, err, ms);
}

// LayerNorm mean and variance from s1_hat = the fp64 sum of x and s2_hat =
// the fp64 sum of x^2 (exact terms), one pass over the row:
//   mean' = S1 / K,  ms' = S2 / K,  var' = ms' - mean'^2.
// With A^2 = S2 / K = var + mean^2 (and |S1| <= K A):
//   |mean' - mean| <= (D + 3) u A
//   |ms' - S2/K|   <= (D + 3) u A^2
//   |var' - var|   <= (3D + 12) u A^2   (with the roundings of mean'^2 and of
//                                        the subtraction)
// A row whose mean is many standard deviations from 0 falls to the exact path
// more often, never to a wrong result.
__device__ __forceinline__ bool ln_fast(double s1_hat, double s2_hat, int64_t K, double rK, float* mean, float* var) {
  const double D = static_cast<double>(sum_depth(K));
  const double mu = s1_hat * rK;
  const double a2 = s2_hat * rK;
  const double v = a2 - mu * mu;
  // sqrt(a2) bounded above with an fp32 square root widened by 1%
  const double a = 1.01 * static_cast<double>(sqrtf(static_cast<float>(a2)));
  const double err_mu = (D + 8.0) * kU * a;
  const double err_var = (3.0 * D + 24.0) * kU * a2 + 0x1p-300;
  if (!(fabs(mu) > 2.0 * err_mu)) return false;  // the mean's sign is certain
  float m;
  if (!rn32_certain(fabs(mu), err_mu, &m)) return false;
  if (!rn32_certain(v, err_var, var)) return false;
  *mean = mu < 0.0 ? -m : m;
  return true;
}

// The variance alone, as in ln_fast (for rows whose mean the fast bound left open).
__device__ __forceinline__ bool ln_var_fast(double s1_hat, double s2_hat, int64_t K, double rK, float* var) {
  const double D = static_cast<double>(sum_depth(K));
  const double mu = s1_hat * rK;
  const double a2 = s2_hat * rK;
  return rn32_certain(a2 - mu * mu, (3.0 * D + 24.0) * kU * a2 + 0x1p-300, var);
}

// When the fp64 sum of a row is exact, the mean's rounding is decided exactly.
// Every element is a multiple of 2^G, G = max(E, 1) - 134 for the exponent
// field E of the smallest nonzero |x| (bf16: 7 fraction bits, subnormals on
// the grid of E = 1), so every partial sum is; and every partial sum is at
// most sum |x| <= sqrt(K S2) in magnitude.  If that is below 2^(G + 53), no
// addition rounds and s1_hat = S1.  Then RN32(S1 / K) is settled by comparing
// |S1| with K times the midpoints around the candidate, products that fp64
// holds exactly (25-bit midpoints, K <= 2^15).
__device__ __forceinline__ bool ln_mean_exact(double s1_hat, double s2_hat, int64_t K, double rK, uint32_t min_mag_m1,
                                              float* mean) {
  if (min_mag_m1 >= 0x7FFFu) {  // no nonzero element: S1 = 0
    *mean = 0.0f;
    return s1_hat == 0.0;
  }
  const int E = static_cast<int>((min_mag_m1 + 1u) >> 7);
  const int G = (E > 1 ? E : 1) - 134;
  const double lim = hi_word_double(static_cast<uint32_t>(2 * G + 106 + 1023) << 20);  // 2^(2G + 106)
  if (!(static_cast<double>(K) * s2_hat * (1.0 + 0x1p-30) < lim)) return false;
  const double a = fabs(s1_hat);
  const float c = __double2float_rn(a * rK);
  const float up = nextafterf(c, __int_as_float(0x7F800000)), dn = c > 0.0f ? nextafterf(c, 0.0f) : 0.0f;
  const double kd = static_cast<double>(K);
  const double k_hi = kd * (0.5 * (static_cast<double>(c) + static_cast<double>(up)));
  const double k_lo = kd * (0.5 * (static_cast<double>(c) + static_cast<double>(dn)));
  const bool c_even = (__float_as_uint(c) & 1u) == 0u;
  float r = c;
  if (a > k_hi)
    r = up;
  else if (a == k_hi)
    r = c_even ? c : up;
  else if (a < k_lo)
    r = dn;
  else if (a == k_lo)
    r = c_even ? c : dn;
  *mean = s1_hat < 0.0 ? -r : r;
  return true;
}

// ---------------------------------------------------------------------------
// Exact path.  A bf16 x with exponent field E and mantissa field F is m * 2^e
// with m = F | 0x80, e = E - 134 (E > 0) or m = F, e = -133 (E = 0).  Then
//   x^2 = m^2 * 2^(2e),  2e + 266 in [0, 506],  m^2 < 2^16
//   x   = m   * 2^e,     e + 133  in [0, 253],  m   < 2^8
// so sum x^2 is an integer in units of 2^-266 below 2^(506 + 16 + 14) (17
// 32-bit digits, K < 2^14) and sum x an integer in units of 2^-133 below
// 2^(253 + 8 + 14) (9 digits).  The terms are added into 64-bit words holding
// 32-bit digits (shared-memory atomics; a word receives at most 2K values
// below 2^32, so it cannot overflow), carried afterwards.
// ---------------------------------------------------------------------------
constexpr int kSqWords = 18;  // digits of sum x^2 (one spare for carries)
constexpr int kS1Words = 10;  // digits of sum x (one spare)

struct ExactSums {
  unsigned long long sq[kSqWords];
  unsigned long long s1[kS1Words];  // two's complement contributions
};

__device__ __forceinline__ void exact_clear(ExactSums* a) {
  const uint32_t lane = threadIdx.x & 31u;
  if (lane < kSqWords) a->sq[lane] = 0ull;
  if (lane < kS1Words) a->s1[lane] = 0ull;
  __syncwarp();
}

__device__ __forceinline__ void exact_add_elem(ExactSums* a, uint32_t b, bool linear) {
  const uint32_t E = (b >> 7) & 0xFFu, F = b & 0x7Fu;
  const uint32_t m = E ? (F | 0x80u) : F;
  if (m == 0u) return;
  const uint32_t p = E ? 2u * E - 2u : 0u;  // 2e + 266
  const unsigned long long v = static_cast<unsigned long long>(m * m) << (p & 31u);
  atomicAdd(&a->sq[p >> 5], v & 0xFFFFFFFFull);
  if (v >> 32) atomicAdd(&a->sq[(p >> 5) + 1], v >> 32);
  if (linear) {
    const uint32_t q = E ? E - 1u : 0u;  // e + 133
    const unsigned long long u = static_cast<unsigned long long>(m) << (q & 31u);
    const bool neg = (b & 0x8000u) != 0u;
    const unsigned long long lo = u & 0xFFFFFFFFull, hi = u >> 32;
    atomicAdd(&a->s1[q >> 5], neg ? 0ull - lo : lo);
    if (hi) atomicAdd(&a->s1[(q >> 5) + 1], neg ? 0ull - hi : hi);
  }
}

__device__ __forceinline__ void exact_add8(ExactSums* a, const uint4& v, bool linear) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    exact_add_elem(a, w[i] & 0xFFFFu, linear);
    exact_add_elem(a, w[i] >> 16, linear);
  }
}

// RN32(num / den * 2^s) for a non-negative integer num of n 32-bit digits
// (least significant first, n <= 20) and 0 < den < 2^31: an exact long
// division of num * 2^64 (so that the quotient holds the fp32 subnormal bits
// for the scales used here, s <= -133), then round to nearest even on the
// quotient's bits, with the remainder as sticky information.
__device__ __noinline__ float rn32_ratio(const uint32_t* num, int n, uint32_t den, int s) {
  uint32_t q[22];
  unsigned long long rem = 0ull;
  const int nq = n + 2;
  for (int i = nq - 1; i >= 0; --i) {
    const unsigned long long cur = (rem << 32) | (i >= 2 ? num[i - 2] : 0u);
    q[i] = static_cast<uint32_t>(cur / den);
    rem = cur % den;
  }
  s -= 64;
  int top = nq - 1;
  while (top >= 0 && q[top] == 0u) --top;
  if (top < 0) return 0.0f;  // below 2^s <= 2^-197
  const int P = 32 * top + (31 - __clz(static_cast<int>(q[top])));
  const int imin = -149 - s;  // bit of 2^-149
  const int L = max(P - 23, imin);
  if (L > P + 2) return 0.0f;  // below 2^-151: rounds to +0
  auto bit = [&](int i) -> uint32_t { return (i < 0 || i >= 32 * nq) ? 0u : (q[i >> 5] >> (i & 31)) & 1u; };
  uint32_t nbits = 0u;
  for (int i = P; i >= L; --i) nbits = (nbits << 1) | bit(i);
  const uint32_t rnd = bit(L - 1);
  bool sticky = rem != 0ull;
  const int lo = L - 1;  // bits below lo
  for (int w = 0; w < (lo >> 5) && !sticky; ++w) sticky = q[w] != 0u;
  if (!sticky && lo > 0 && (lo & 31)) sticky = (q[lo >> 5] & ((1u << (lo & 31)) - 1u)) != 0u;
  if (rnd && (sticky || (nbits & 1u))) ++nbits;
  int Lr = L;
  if (nbits == (1u << 24)) {
    nbits = 1u << 23;
    ++Lr;
  }
  if (nbits >= (1u << 23)) {
    const int E = Lr + s + 23 + 127;
    if (E >= 255) return __int_as_float(0x7F800000);
    return __uint_as_float((static_cast<uint32_t>(E) << 23) | (nbits - (1u << 23)));
  }
  return __uint_as_float(nbits);  // subnormal: Lr + s = -149
}

// Carries the 64-bit words into 32-bit digits (non-negative sum).
__device__ __forceinline__ void carry_unsigned(const unsigned long long* w, int n, uint32_t* d) {
  unsigned long long c = 0ull;
  for (int i = 0; i < n; ++i) {
    const unsigned long long t = w[i] + c;
    d[i] = static_cast<uint32_t>(t);
    c = t >> 32;
  }
}

// ms = RN32(sum x^2 / K) from the exact sums (lane 0 only).
__device__ __noinline__ float exact_ms(const ExactSums* a, uint32_t K) {
  uint32_t d[kSqWords];
  carry_unsigned(a->sq, kSqWords, d);
  return rn32_ratio(d, kSqWords, K, -266);
}

// LayerNorm mean and var from the exact sums (lane 0 only):
//   mean = RN32(S1 / K),  var = RN32((K S2 - S1^2) / K^2)
// with S1 in units of 2^-133 and S2, S1^2 in units of 2^-266.
__device__ __noinline__ void exact_mean_var(const ExactSums* a, uint32_t K, float* mean, float* var) {
  uint32_t s2[kSqWords];
  carry_unsigned(a->sq, kSqWords, s2);
  // signed carry of S1: the final carry is the sign extension (|S1| < 2^275)
  uint32_t s1[kS1Words];
  long long c = 0;
  for (int i = 0; i < kS1Words; ++i) {
    const long long t = static_cast<long long>(a->s1[i]) + c;
    s1[i] = static_cast<uint32_t>(t);
    c = t >> 32;  // arithmetic shift
  }
  const bool neg = c < 0;
  if (neg) {  // |S1| = two's complement negation
    unsigned long long b = 1ull;
    for (int i = 0; i < kS1Words; ++i) {
      const unsigned long long t = static_cast<unsigned long long>(~s1[i]) + b;
      s1[i] = static_cast<uint32_t>(t);
      b = t >> 32;
    }
  }
  const float m = rn32_ratio(s1, kS1Words, K, -133);
  *mean = neg ? -m : m;
  // N = K * S2 - S1^2 (>= 0), 20 digits
  constexpr int kN = 20;
  uint32_t ks2[kN] = {}, sq1[kN] = {};
  unsigned long long cy = 0ull;
  for (int i = 0; i < kSqWords; ++i) {
    const unsigned long long t = static_cast<unsigned long long>(s2[i]) * K + cy;
    ks2[i] = static_cast<uint32_t>(t);
    cy = t >> 32;
  }
  ks2[kSqWords] = static_cast<uint32_t>(cy);
  for (int i = 0; i < kS1Words - 1; ++i) {  // |S1| < 2^275 fits 9 digits
    unsigned long long carry = 0ull;
    for (int j = 0; j < kS1Words - 1; ++j) {
      const unsigned long long t =
          static_cast<unsigned long long>(s1[i]) * s1[j] + sq1[i + j] + carry;
      sq1[i + j] = static_cast<uint32_t>(t);
      carry = t >> 32;
    }
    sq1[i + kS1Words - 1] = static_cast<uint32_t>(carry);
  }
  uint32_t nn[kN];
  long long br = 0;
  for (int i = 0; i < kN; ++i) {
    const long long t = static_cast<long long>(ks2[i]) - static_cast<long long>(sq1[i]) + br;
    nn[i] = static_cast<uint32_t>(t);
    br = t >> 32;  // 0 or -1
  }
  *var = rn32_ratio(nn, kN, K * K, -266);
}

}  // namespace normstats
}  // namespace bsp
