// Shared pieces of the page selectors: order-preserving float keys, a
// two-sequence radix select over shared memory, and exact float64 scores of a
// query row held as float32 copies of bf16 values.
#pragma once

#include "common.cuh"
#include "exact.cuh"

namespace sa {

SA_DEV uint32_t f2key(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
SA_DEV float key2f(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// RN64(q . sigma) for a query row held as float32 copies of bf16 values.
__device__ __forceinline__ double exact_dot_f32q(const float* q, const uint16_t* sig, int n) {
  ExactAcc acc;
  acc.clear();
  for (int d = 0; d < n; ++d) {
    uint32_t ma, mb;
    int ea, eb;
    bool na, nb;
    bf16_fields(__float_as_uint(q[d]) >> 16, ma, ea, na);
    bf16_fields(sig[d], mb, eb, nb);
    acc.add(ma * mb, ea + eb, na != nb);
  }
  return acc.round_to_double();
}

// Radix-select the (k_lo)-th largest key of `lo` and the (k_hi)-th largest of
// `hi` over n entries (1-based ranks; entries with key 0 never match).
SA_DEV void radix_select2(const float* lo, const float* hi, int n, int k_lo, int k_hi,
                          uint32_t* hist /*[2][256]*/, uint32_t* shared_out /*[4]*/,
                          float& out_lo, float& out_hi) {
  uint32_t pre[2] = {0u, 0u}, msk[2] = {0u, 0u};
  int kk[2] = {k_lo, k_hi};
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 512; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const float a = lo[i], c = hi[i];
      const uint32_t ka = f2key(a), kc = f2key(c);
      if (!isnan(a) && (ka & msk[0]) == pre[0]) atomicAdd(&hist[(ka >> shift) & 255u], 1u);
      if (!isnan(c) && (kc & msk[1]) == pre[1]) atomicAdd(&hist[256 + ((kc >> shift) & 255u)], 1u);
    }
    __syncthreads();
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (w < 2) {
      // lane holds bins [255 - 8*lane - 7, 255 - 8*lane], scanned from the top
      uint32_t c8[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c8[j] = hist[w * 256 + 255 - (8 * lane + j)];
        tot += c8[j];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      uint32_t before = incl - tot;   // count in higher bins than this lane's
      const uint32_t want = static_cast<uint32_t>(kk[w]);
      if (before < want && incl >= want) {
        uint32_t run = before;
        for (int j = 0; j < 8; ++j) {
          if (run + c8[j] >= want) {
            shared_out[2 * w] = 255u - (8u * lane + j);
            shared_out[2 * w + 1] = run;
            break;
          }
          run += c8[j];
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      pre[s] |= shared_out[2 * s] << shift;
      msk[s] |= 255u << shift;
      kk[s] -= static_cast<int>(shared_out[2 * s + 1]);
    }
    __syncthreads();
  }
  out_lo = key2f(pre[0]);
  out_hi = key2f(pre[1]);
}



}  // namespace sa
