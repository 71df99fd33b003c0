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
// `hi` over n entries (1-based ranks; NaN entries never match).  Four 8-bit
// digit passes; the histograms and digit results are double-buffered so each
// pass needs two block barriers.  hist: [2][512] words, shared_out: [2][4].
SA_DEV void radix_select2(const float* lo, const float* hi, int n, int k_lo, int k_hi,
                          uint32_t* hist, uint32_t* shared_out, float& out_lo, float& out_hi) {
  uint32_t pre[2] = {0u, 0u}, msk[2] = {0u, 0u};
  int kk[2] = {k_lo, k_hi};
  for (int i = threadIdx.x; i < 512; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = hist + (pass & 1) * 512;
    uint32_t* nxt = hist + ((pass + 1) & 1) * 512;
    uint32_t* so = shared_out + (pass & 1) * 4;
    for (int i = threadIdx.x; i < 512; i += blockDim.x) nxt[i] = 0u;   // next pass's bins
    // warp-aggregated increments: the keys crowd into a few top-digit bins,
    // so lanes with equal bins add their count with one atomic
    const int ln = threadIdx.x & 31;
    for (int i0 = 0; i0 < n; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      uint32_t ba = 0xffffffffu, bc = 0xffffffffu;
      if (i < n) {
        const float a = lo[i], c = hi[i];
        const uint32_t ka = f2key(a), kc = f2key(c);
        if (!isnan(a) && (ka & msk[0]) == pre[0]) ba = (ka >> shift) & 255u;
        if (!isnan(c) && (kc & msk[1]) == pre[1]) bc = 256u + ((kc >> shift) & 255u);
      }
      const uint32_t pa = __match_any_sync(0xffffffffu, ba);
      const uint32_t pc = __match_any_sync(0xffffffffu, bc);
      if (ba != 0xffffffffu && ln == __ffs(pa) - 1) atomicAdd(&h[ba], __popc(pa));
      if (bc != 0xffffffffu && ln == __ffs(pc) - 1) atomicAdd(&h[bc], __popc(pc));
    }
    __syncthreads();
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (w < 2) {
      // lane holds bins [255 - 8*lane - 7, 255 - 8*lane], scanned from the top
      uint32_t c8[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c8[j] = h[w * 256 + 255 - (8 * lane + j)];
        tot += c8[j];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t before = incl - tot;   // count in higher bins than this lane's
      const uint32_t want = static_cast<uint32_t>(kk[w]);
      if (before < want && incl >= want) {
        uint32_t run = before;
        for (int j = 0; j < 8; ++j) {
          if (run + c8[j] >= want) {
            so[2 * w] = 255u - (8u * lane + j);
            so[2 * w + 1] = run;
            break;
          }
          run += c8[j];
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      pre[t] |= so[2 * t] << shift;
      msk[t] |= 255u << shift;
      kk[t] -= static_cast<int>(so[2 * t + 1]);
    }
  }
  __syncthreads();   // the buffers may be reused by the caller
  out_lo = key2f(pre[0]);
  out_hi = key2f(pre[1]);
}

}  // namespace sa
