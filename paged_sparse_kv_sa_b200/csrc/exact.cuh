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

#include <math.h>
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
__host__ __device__ __forceinline__ void bf16_fields(uint32_t bits, uint32_t& m, int& e, bool& neg) {
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

// ---------------------------------------------------------------------------
// Warp-cooperative exact dot product.
//
// In one dot product the product exponents usually span a few dozen bits, so
// every product is an integer multiple of 2^emin (emin = the smallest product
// exponent) below 2^(16 + span).  With span <= 100 and n <= 1024 terms, the
// sum of those integers fits a signed 128-bit word: each lane accumulates its
// products there, the lanes' words are added with xor shuffles, and the total
// is rounded once to float64.  A wider span falls back to the superaccumulator
// (one lane).

// Two's complement 128-bit value hi:lo.
struct I128 {
  uint64_t lo, hi;
};
__host__ __device__ __forceinline__ void i128_add(I128& a, uint64_t blo, uint64_t bhi) {
  const uint64_t lo = a.lo + blo;
  a.hi = a.hi + bhi + (lo < a.lo ? 1ull : 0ull);
  a.lo = lo;
}
__host__ __device__ __forceinline__ void i128_sub(I128& a, uint64_t blo, uint64_t bhi) {
  const uint64_t lo = a.lo - blo;
  a.hi = a.hi - bhi - (a.lo < blo ? 1ull : 0ull);
  a.lo = lo;
}
// m << sh as a 128-bit word (sh in [0, 127], m < 2^16).
__host__ __device__ __forceinline__ void shl128(uint64_t m, int sh, uint64_t& lo, uint64_t& hi) {
  if (sh >= 64) {
    lo = 0;
    hi = m << (sh - 64);
  } else {
    lo = m << sh;
    hi = sh ? m >> (64 - sh) : 0ull;
  }
}
__host__ __device__ __forceinline__ int clz64(uint64_t x) {
#ifdef __CUDA_ARCH__
  return __clzll(static_cast<long long>(x));
#else
  return __builtin_clzll(x);
#endif
}
// Nearest float64 (ties to even) to the integer hi:lo times 2^e0; the result
// must be a normal float64.
__host__ __device__ __forceinline__ double i128_to_double_rn(I128 v, int e0) {
  const bool neg = static_cast<int64_t>(v.hi) < 0;
  if (neg) {   // magnitude
    v.lo = ~v.lo + 1ull;
    v.hi = ~v.hi + (v.lo == 0 ? 1ull : 0ull);
  }
  if (v.hi == 0 && v.lo == 0) return 0.0;
  const int msb = v.hi ? 127 - clz64(v.hi) : 63 - clz64(v.lo);
  uint64_t mant;
  int sh = 0;
  if (msb <= 52) {
    mant = v.lo;
  } else {
    sh = msb - 52;                       // bits dropped: 1 .. 75
    // mant = v >> sh (53 bits)
    if (sh >= 64) mant = v.hi >> (sh - 64);
    else mant = (v.lo >> sh) | (v.hi << (64 - sh));
    // round bit = bit sh - 1; sticky = any bit below it
    const int rb = sh - 1;
    const bool round = rb >= 64 ? ((v.hi >> (rb - 64)) & 1ull) : ((v.lo >> rb) & 1ull);
    bool sticky;
    if (rb == 0) sticky = false;
    else if (rb < 64) sticky = (v.lo & ((1ull << rb) - 1ull)) != 0;
    else if (rb == 64) sticky = v.lo != 0;
    else sticky = v.lo != 0 || (v.hi & ((1ull << (rb - 64)) - 1ull)) != 0;
    if (round && (sticky || (mant & 1ull))) {
      ++mant;
      if (mant == (1ull << 53)) {
        mant >>= 1;
        ++sh;
      }
    }
  }
  const double r = scalbn(static_cast<double>(mant), e0 + sh);
  return neg ? -r : r;
}

#ifdef __CUDACC__
// RN64(sum_d a[d] * b[d]) for two bf16 rows of n elements (n % 8 == 0, both
// 16-byte aligned, n <= 256 kMaxC <= 1024), computed by all 32 lanes of a warp
// (each loads its 16-byte chunks once); every lane returns the result.  The
// exponent span of the nonzero products picks the method: up to 26 bits a
// float64 sum that never rounds, up to 100 bits a signed 128-bit fixed-point
// sum anchored at the smallest exponent, beyond that the superaccumulator.
template <int kMaxC>   // 16-byte chunks per lane: n <= 256 kMaxC
__device__ __forceinline__ double warp_exact_dot_bf16(const uint16_t* a, const uint16_t* b, int n) {
  static_assert(kMaxC >= 1 && kMaxC <= 4, "n <= 1024 keeps the float64 path exact");
  const int lane = threadIdx.x & 31;
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  const uint4* b4 = reinterpret_cast<const uint4*>(b);
  const int nc = n >> 3;
  if (nc == 0) return 0.0;
  uint4 xs[kMaxC], ys[kMaxC];
  // every load is issued unconditionally (index clamped, zeroed afterwards), so
  // all of them are in flight together instead of one round trip each
#pragma unroll
  for (int j = 0; j < kMaxC; ++j) {
    const int c = min(lane + 32 * j, nc - 1);
    xs[j] = a4[c];
    ys[j] = b4[c];
  }
#pragma unroll
  for (int j = 0; j < kMaxC; ++j)
    if (lane + 32 * j >= nc) xs[j] = ys[j] = make_uint4(0, 0, 0, 0);
  // pass 1: exponent range of the nonzero products (selects, no branches)
  int emin = 1 << 20, emax = -(1 << 20);
#pragma unroll
  for (int j = 0; j < kMaxC; ++j) {
    const uint32_t xa[4] = {xs[j].x, xs[j].y, xs[j].z, xs[j].w};
    const uint32_t ya[4] = {ys[j].x, ys[j].y, ys[j].z, ys[j].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t ma, mb;
      int ea, eb;
      bool na, nb;
      bf16_fields((xa[i >> 1] >> (16 * (i & 1))) & 0xffffu, ma, ea, na);
      bf16_fields((ya[i >> 1] >> (16 * (i & 1))) & 0xffffu, mb, eb, nb);
      const bool nz = (ma != 0u) & (mb != 0u);
      emin = min(emin, nz ? ea + eb : (1 << 20));
      emax = max(emax, nz ? ea + eb : -(1 << 20));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  if (emax < emin) return 0.0;          // every product is zero
  if (emax - emin <= 26) {
    // Narrow span: every product is an integer multiple of 2^emin below
    // 2^(emax + 16), so every partial sum of at most 1024 of them is a
    // multiple of 2^emin smaller than 2^(emin + 52): float64 represents all
    // of them, and fma(x, y, acc) (x*y exact: 16 significant bits) never
    // rounds.  The float64 sum is the exact sum.
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < kMaxC; ++j) {
      const uint32_t xa[4] = {xs[j].x, xs[j].y, xs[j].z, xs[j].w};
      const uint32_t ya[4] = {ys[j].x, ys[j].y, ys[j].z, ys[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc = fma(static_cast<double>(__uint_as_float(xa[i] << 16)),
                  static_cast<double>(__uint_as_float(ya[i] << 16)), acc);
        acc = fma(static_cast<double>(__uint_as_float(xa[i] & 0xffff0000u)),
                  static_cast<double>(__uint_as_float(ya[i] & 0xffff0000u)), acc);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
  }
  if (emax - emin > 100) {              // wide span: superaccumulator, lane 0
    double r = 0.0;
    if (lane == 0) r = exact_dot_bf16(a, 1, b, n);
    return __shfl_sync(0xffffffffu, r, 0);
  }
  // pass 2: fixed-point sums anchored at 2^emin
  I128 acc{0ull, 0ull};
#pragma unroll
  for (int j = 0; j < kMaxC; ++j) {
    const uint32_t xa[4] = {xs[j].x, xs[j].y, xs[j].z, xs[j].w};
    const uint32_t ya[4] = {ys[j].x, ys[j].y, ys[j].z, ys[j].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t ma, mb;
      int ea, eb;
      bool na, nb;
      bf16_fields((xa[i >> 1] >> (16 * (i & 1))) & 0xffffu, ma, ea, na);
      bf16_fields((ya[i >> 1] >> (16 * (i & 1))) & 0xffffu, mb, eb, nb);
      const uint32_t m = ma * mb;
      if (m) {
        uint64_t lo, hi;
        shl128(m, ea + eb - emin, lo, hi);
        if (na != nb) i128_sub(acc, lo, hi);
        else i128_add(acc, lo, hi);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const uint64_t lo = __shfl_xor_sync(0xffffffffu, acc.lo, o);
    const uint64_t hi = __shfl_xor_sync(0xffffffffu, acc.hi, o);
    i128_add(acc, lo, hi);
  }
  return i128_to_double_rn(acc, emin);
}
#endif

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
