// Per-page key summaries: sigma = RNE_bf16(RN64(RN64(sum of valid keys) / n)).
//
// One CTA per (logical page, sequence); threads walk the (kv head, feature)
// columns.  With n_new > 0 only the pages holding the last n_new tokens of
// each sequence are rewritten (the pages an append of n_new tokens changed).  The float64 sum of at most P bf16 values is exact whenever the
// values span at most 53 - ceil(log2 P) - 1 bits (every bf16 is an integer
// multiple of its lsb weight); columns that fail that test are re-summed in
// the exact fixed-point accumulator.
//
// Source: "Universal Attention Engine — Declarative Sparse Attention for
// Production", "Content-Dependent Dynamic Routing" (the router scores
// mean(k_blocks), the block-mean key).
#include "common.cuh"
#include "exact.cuh"
#include "internal.h"

namespace sa {
namespace {

__global__ void __launch_bounds__(256)
    summaries_kernel(const uint16_t* __restrict__ k, int64_t ks0, int64_t ks1, int64_t ks2,
                     const PageMap pt, int max_pages,
                     const int32_t* __restrict__ seq_lens, int Hkv, int Dk, int P, int P_pool,
                     int n_new, uint16_t* __restrict__ sig, int32_t* err) {
  pdl_wait_and_release();
  const int b = blockIdx.y;
  const int L = min(seq_lens[b], max_pages * P);
  const int p = (n_new > 0 ? max(L - n_new, 0) / P : 0) + blockIdx.x;
  const int n = min(P, L - p * P);
  if (n <= 0) return;
  const int ph = page_at(pt, b, p);
  if (ph < 0 || ph >= P_pool) {
    if (threadIdx.x == 0) set_dev_error(err, SA_DEVERR_POOL_RANGE);
    return;
  }
  const int lg = 32 - __clz(n);   // >= ceil(log2 n) + 1 for n >= 1
  for (int c = threadIdx.x; c < Hkv * Dk; c += blockDim.x) {
    const int h = c / Dk, d = c % Dk;
    const uint16_t* col = k + ph * ks0 + h * ks1 + d;
    double s = 0.0;
    int emax = -100000, umin = 100000;
    for (int j = 0; j < n; ++j) {
      const uint32_t bits = col[j * ks2];
      if ((bits & 0x7fffu) == 0) continue;
      const int E = (bits >> 7) & 0xff;
      const int eb = E ? E : 1;
      emax = max(emax, eb - 126);   // |x| < 2^(eb - 126)
      umin = min(umin, eb - 134);   // x is a multiple of 2^(eb - 134)
      s += static_cast<double>(bf16_bits_to_float(bits));
    }
    if (emax > -100000 && emax + lg - umin > 53) {
      ExactAcc acc;
      acc.clear();
      for (int j = 0; j < n; ++j) {
        uint32_t m;
        int e;
        bool neg;
        bf16_fields(col[j * ks2], m, e, neg);
        acc.add(m, e, neg);
      }
      s = acc.round_to_double();
    }
    const double mean = s / static_cast<double>(n);
    sig[((int64_t)ph * Hkv + h) * Dk + d] = f64_to_bf16_rne(mean);
  }
}

// FP8 pages: every E4M3 value is a multiple of 2^-9 below 2^9, so the float64
// sum of at most 128 of them is exact; all keys of a (page, kv head) share its
// scale, and scale * sum (24 x 25 significant bits) is exact too: the mean is
// RN64(exact sum of the dequantized keys / n), as for bf16 pages.
__global__ void __launch_bounds__(256)
    summaries_fp8_kernel(const uint8_t* __restrict__ k, int64_t ks0, int64_t ks1, int64_t ks2,
                         const float* __restrict__ k_scale, const PageMap pt,
                         int max_pages, const int32_t* __restrict__ seq_lens, int Hkv, int Dk,
                         int P, int P_pool, uint16_t* __restrict__ sig, int32_t* err) {
  pdl_wait_and_release();
  const int b = blockIdx.y, p = blockIdx.x;
  const int L = min(seq_lens[b], max_pages * P);
  const int n = min(P, L - p * P);
  if (n <= 0) return;
  const int ph = page_at(pt, b, p);
  if (ph < 0 || ph >= P_pool) {
    if (threadIdx.x == 0) set_dev_error(err, SA_DEVERR_POOL_RANGE);
    return;
  }
  for (int c = threadIdx.x; c < Hkv * Dk; c += blockDim.x) {
    const int h = c / Dk, d = c % Dk;
    const uint8_t* col = k + ph * ks0 + h * ks1 + d;
    double s = 0.0;
    for (int j = 0; j < n; ++j) s += static_cast<double>(e4m3_to_float(col[j * ks2]));
    s *= static_cast<double>(k_scale[(int64_t)ph * Hkv + h]);
    sig[((int64_t)ph * Hkv + h) * Dk + d] = f64_to_bf16_rne(s / static_cast<double>(n));
  }
}

}  // namespace

cudaError_t launch_summaries_fp8(const uint8_t* k, const int64_t ks[4], const float* k_scale,
                                 const PageMap& pt, int max_pages, const int32_t* seq_lens, int B,
                                 int Hkv, int Dk, int P, int P_pool, uint16_t* sig, int32_t* err,
                                 cudaStream_t stream) {
  if (B == 0 || max_pages == 0) return cudaSuccess;
  dim3 grid(max_pages, B);
  return launch_pdl(summaries_fp8_kernel, grid, dim3(256), 0, stream, k, ks[0], ks[1], ks[2],
                    k_scale, pt, max_pages, seq_lens, Hkv, Dk, P, P_pool, sig, err);
}

cudaError_t launch_summaries(const uint16_t* k, const int64_t ks[4], const PageMap& pt,
                             int max_pages, const int32_t* seq_lens, int B, int Hkv, int Dk,
                             int P, int P_pool, int n_new, uint16_t* sig, int32_t* err,
                             cudaStream_t stream) {
  if (B == 0 || max_pages == 0) return cudaSuccess;
  // n_new tokens end in at most ceil((n_new - 1) / P) + 1 pages
  const int pages = n_new > 0 ? min(max_pages, (n_new - 1 + P - 1) / P + 1) : max_pages;
  dim3 grid(pages, B);
  return launch_pdl(summaries_kernel, grid, dim3(256), 0, stream, k, ks[0], ks[1], ks[2], pt,
                    max_pages, seq_lens, Hkv, Dk, P, P_pool, n_new, sig, err);
}

}  // namespace sa
