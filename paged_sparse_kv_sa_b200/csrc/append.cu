// Appending tokens to the paged cache in one launch: the new K and V rows are
// written into their pages, and the key summaries of the pages they land in
// are recomputed (sigma = RNE_bf16(RN64(RN64(exact sum of the page's valid
// keys) / n))), so the page router sees the appended tokens without a second
// pass over the cache.
//
// One CTA per (touched page slot, kv head, sequence).  It copies the page's new
// rows of its head (16-byte copies) and then sums each feature column over the
// page's valid rows: the rows that were there before the append are read from
// the cache (this launch never writes them), the new rows from the input
// (never from the rows this CTA is writing).  The float64 sum is exact whenever
// the column's values span at most 53 - ceil(log2 n) - 1 bits; other columns
// are re-summed in the exact fixed-point accumulator.
//
// Source: "Universal Attention Engine — Declarative Sparse Attention for
// Production", "Content-Dependent Dynamic Routing" (the router scores
// mean(k_blocks): a block's mean changes when tokens land in it) and
// "Architecture" (a PagedAttention-compatible cache).
#include "common.cuh"
#include "exact.cuh"
#include "internal.h"

namespace sa {
namespace {

__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
  pdl_wait_and_release();
  const int b = blockIdx.z, h = blockIdx.y, j = blockIdx.x, tid = threadIdx.x;
  int L = a.seq_lens[b];
  int n = a.n_new[b];
  if (n < 0 || n > a.max_new) {
    if (tid == 0 && h == 0 && j == 0) set_dev_error(a.err, SA_DEVERR_COUNT);
    n = n < 0 ? 0 : a.max_new;
  }
  if (L < 0 || L > a.max_pages * a.P) {
    if (tid == 0 && h == 0 && j == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    return;
  }
  if (a.out_seq_lens && tid == 0 && h == 0 && j == 0) a.out_seq_lens[b] = L + n;
  int end = L + n;
  if (end > a.max_pages * a.P) {   // tokens past the page table's row are dropped
    if (tid == 0 && h == 0 && j == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    end = a.max_pages * a.P;
  }
  if (end <= L) return;
  const int P = a.P;
  const int p = L / P + j;
  const int p0 = p * P;
  if (p0 >= end) return;
  const int lo = max(L, p0), hi = min(end, p0 + P);
  const int ph = page_at(a.pt, b, p);
  if (ph < 0 || ph >= a.P_pool) {
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
    return;
  }
  const int D = a.D, cpr = D / 8;   // 16-byte chunks per row
  // ---- the new rows of this page and head
  for (int idx = tid; idx < (hi - lo) * cpr; idx += blockDim.x) {
    const int r = idx / cpr, c = idx % cpr;
    const int pos = lo + r, i = pos - L;
    const uint4 kv = *reinterpret_cast<const uint4*>(a.k_new + b * a.kn0 + i * a.kn1 +
                                                     h * a.kn2 + c * 8);
    const uint4 vv = *reinterpret_cast<const uint4*>(a.v_new + b * a.vn0 + i * a.vn1 +
                                                     h * a.vn2 + c * 8);
    *reinterpret_cast<uint4*>(a.k_cache + ph * a.ks0 + h * a.ks1 + (pos - p0) * a.ks2 + c * 8) =
        kv;
    *reinterpret_cast<uint4*>(a.v_cache + ph * a.vs0 + h * a.vs1 + (pos - p0) * a.vs2 + c * 8) =
        vv;
  }
  // ---- the page's summary for this head over its valid rows [0, hi - p0)
  const int nval = hi - p0, n_old = max(L - p0, 0);
  const int lg = 32 - __clz(nval);   // >= ceil(log2 nval) + 1
  auto key = [&](int r, int d) -> uint32_t {
    return r < n_old ? a.k_cache[ph * a.ks0 + h * a.ks1 + r * a.ks2 + d]
                     : a.k_new[b * a.kn0 + (p0 + r - L) * a.kn1 + h * a.kn2 + d];
  };
  for (int d = tid; d < D; d += blockDim.x) {
    double s = 0.0;
    int emax = -100000, umin = 100000;
    for (int r = 0; r < nval; ++r) {
      const uint32_t bits = key(r, d);
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
      for (int r = 0; r < nval; ++r) {
        uint32_t m;
        int e;
        bool neg;
        bf16_fields(key(r, d), m, e, neg);
        acc.add(m, e, neg);
      }
      s = acc.round_to_double();
    }
    a.sig[((int64_t)ph * a.Hkv + h) * D + d] = f64_to_bf16_rne(s / static_cast<double>(nval));
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.B == 0) return cudaSuccess;
  // n <= max_new tokens starting anywhere cover at most ceil((n - 1) / P) + 1 pages
  const int pages = a.max_new > 0 ? (a.max_new - 1 + a.P - 1) / a.P + 1 : 1;
  return launch_pdl(append_kernel, dim3(pages, a.Hkv, a.B), dim3(256), 0, stream, a);
}

}  // namespace sa
