// Exact sums of bf16 values and bf16 x bf16 products, correctly rounded to
// float64, and float64 -> bf16 rounding, written from the IEEE-754 formats.
//
// A finite bf16 pattern with exponent field E and fraction F is the integer
// M = (E ? 128 + F : F) times 2^(max(E,1) - 134).  A product of two such
// values is an integer below 2^16 times 2^(ea + eb), with ea + eb in
// [-266, 240].  Summing those integers in a fixed-point accumulator of 32-bit
// limbs (bit 0 of limb 0 weighs 2^-288) is exact; the result is then rounded
// once to the nearest float64, ties to even.
#pragma once

#include <stdint.h>

namespace sa {

struct ExactAcc {
  static constexpr int kLimbs = 19;   // 608 bits: weights 2^-288 .. 2^319
  static constexpr int kBias = 288;
  int64_t limb[kLimbs];

  __device__ void clear() {
#pragma unroll
    for (int i = 0; i < kLimbs; ++i) limb[i] = 0;
  }
  // Add (neg ? -1 : 1) * m * 2^e, m < 2^16, e in [-266, 240].
  __device__ void add(uint32_t m, int e, bool neg) {
    if (m == 0) return;
    const int off = e + kBias;
    const int li = off >> 5, sh = off & 31;
    const uint64_t v = static_cast<uint64_t>(m) << sh;     // < 2^47
    const int64_t lo = static_cast<int64_t>(v & 0xffffffffull);
    const int64_t hi = static_cast<int64_t>(v >> 32);
    if (neg) {
      limb[li] -= lo;
      limb[li + 1] -= hi;
    } else {
      limb[li] += lo;
      limb[li + 1] += hi;
    }
  }
  // Round the exact value to the nearest float64 (ties to even).
  __device__ double round_to_double() {
    // carry-propagate: limbs 0..kLimbs-2 into [0, 2^32), the top one signed
    for (int i = 0; i < kLimbs - 1; ++i) {
      const int64_t c = limb[i] >> 32;   // arithmetic shift: floor division
      limb[i] -= c * 4294967296ll;
      limb[i + 1] += c;
    }
    bool neg = limb[kLimbs - 1] < 0;
    if (neg) {  // two's complement negation across the limbs
      int64_t carry = 1;
      for (int i = 0; i < kLimbs; ++i) {
        int64_t v = (~limb[i] & 0xffffffffll) + carry;
        carry = v >> 32;
        limb[i] = v & 0xffffffffll;
      }
    }
    int h = kLimbs - 1;
    while (h >= 0 && limb[h] == 0) --h;
    if (h < 0) return 0.0;
    const uint32_t top = static_cast<uint32_t>(limb[h]);
    const int b = 31 - __clz(static_cast<int>(top));          // msb position inside limb h
    const uint64_t l1 = h >= 1 ? static_cast<uint64_t>(limb[h - 1]) : 0;
    const uint64_t l2 = h >= 2 ? static_cast<uint64_t>(limb[h - 2]) : 0;
    bool sticky = false;
    for (int i = h - 3; i >= 0; --i) sticky |= limb[i] != 0;
    // 96-bit window [limb h | limb h-1 | limb h-2] with its msb at bit 64 + b;
    // shift so that the msb lands on bit 63 of a 64-bit word.
    const int s = b + 1;                                        // 1..32
    const uint64_t hi64 = (static_cast<uint64_t>(top) << 32) | l1;   // bits 95..32 of the window
    const uint64_t w = (hi64 << (32 - s)) | (l2 >> s);
    const uint64_t lost = l2 & ((1ull << s) - 1ull);
    sticky |= lost != 0;
    uint64_t mant = w >> 11;                                    // 53 bits
    const bool round = (w >> 10) & 1ull;
    sticky |= (w & 0x3ffull) != 0;
    int exp2 = 32 * h + b - kBias - 52;                         // weight of mant's lsb
    if (round && (sticky || (mant & 1ull))) {
      ++mant;
      if (mant == (1ull << 53)) {
        mant >>= 1;
        ++exp2;
      }
    }
    const double r = scalbn(static_cast<double>(mant), exp2);
    return neg ? -r : r;
  }
};

// Fields of one bf16 pattern: significand integer and the weight of its lsb.
__device__ __forceinline__ void bf16_fields(uint32_t bits, uint32_t& m, int& e, bool& neg) {
  const uint32_t E = (bits >> 7) & 0xffu, F = bits & 0x7fu;
  neg = (bits >> 15) & 1u;
  m = E ? (128u + F) : F;
  e = (E ? static_cast<int>(E) : 1) - 134;
}

// RN64(sum_d a[d] * b[d]) for bf16 patterns a (stride sa) and b (stride 1).
__device__ __forceinline__ double exact_dot_bf16(const uint16_t* a, int sa, const uint16_t* b,
                                                 int n) {
  ExactAcc acc;
  acc.clear();
  for (int d = 0; d < n; ++d) {
    uint32_t ma, mb;
    int ea, eb;
    bool na, nb;
    bf16_fields(a[d * sa], ma, ea, na);
    bf16_fields(b[d], mb, eb, nb);
    acc.add(ma * mb, ea + eb, na != nb);
  }
  return acc.round_to_double();
}

// Nearest bf16 to a float64 (ties to even), for |x| below the bf16 overflow
// threshold.  Works on the binary64 fields: keep the top 8 significant bits
// (fewer for results below 2^-126), round on the rest.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  const uint32_t sign = static_cast<uint32_t>(u >> 63);
  const int E = static_cast<int>((u >> 52) & 0x7ff);
  if (E == 0) return static_cast<uint16_t>(sign << 15);       // zero / f64 subnormal -> 0
  const uint64_t sig = (u & ((1ull << 52) - 1)) | (1ull << 52);   // 53-bit significand
  const int e = E - 1023;                                       // x = sig * 2^(e-52)
  // bf16 lsb weight for this magnitude: 2^(e-7) when normal, 2^-133 below.
  const int lsb = e >= -126 ? e - 7 : -133;
  const int drop = lsb - (e - 52);                              // bits of sig below the lsb
  uint64_t q;
  if (drop >= 64) {
    q = 0;  // far below half the smallest subnormal: rounds to zero
  } else {
    q = sig >> drop;
    const uint64_t rem = sig & ((1ull << drop) - 1);
    const uint64_t half = 1ull << (drop - 1);
    if (rem > half || (rem == half && (q & 1ull))) ++q;
  }
  // q * 2^lsb; rebuild the bf16 pattern (q may have carried into 2^8).
  uint32_t bits;
  if (lsb == -133 && q < 128) {
    bits = static_cast<uint32_t>(q);                            // subnormal
  } else {
    int ee = lsb + 7;                                           // exponent of the leading bit
    if (q >= 256) {
      q >>= 1;
      ++ee;
    }
    bits = (static_cast<uint32_t>(ee + 127) << 7) | static_cast<uint32_t>(q & 0x7f);
  }
  return static_cast<uint16_t>((sign << 15) | bits);
}

}  // namespace sa
