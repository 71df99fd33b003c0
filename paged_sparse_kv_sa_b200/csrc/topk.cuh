// Shared pieces of the page selectors: order-preserving float / double keys,
// a warp-wide rigorous float32 score bracket, and a two-sequence radix select
// over shared memory.
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

// Order-preserving 64-bit key of a float64 (larger key = larger value; -0 < +0).
SA_DEV unsigned long long d2key(double x) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
SA_DEV double key2d(unsigned long long k) {
  return __longlong_as_double(
      static_cast<long long>((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

// A rigorous float32 bracket [lo, hi] of the exact q . sigma for two bf16 rows
// of n elements (n % 8 == 0, both 16-byte aligned), computed by a whole warp;
// every lane returns it.  Each product of two bf16 values is exact in float32
// and every term passes through at most n roundings on its way to the total,
// so |fl(q.s) - q.s| <= gamma_n sum |q_d s_d| <= gamma_n ||q|| ||s||.
SA_DEV float2 warp_score_bracket(const uint16_t* q, const uint16_t* sg, int n) {
  const int lane = threadIdx.x & 31;
  const uint4* q4 = reinterpret_cast<const uint4*>(q);
  const uint4* s4 = reinterpret_cast<const uint4*>(sg);
  float s = 0.f, qq = 0.f, ss = 0.f;
  for (int c = lane; c < (n >> 3); c += 32) {
    const uint4 x = q4[c], y = s4[c];
    const uint32_t xa[4] = {x.x, x.y, x.z, x.w}, ya[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = __uint_as_float(xa[e] << 16), x1 = __uint_as_float(xa[e] & 0xffff0000u);
      const float y0 = __uint_as_float(ya[e] << 16), y1 = __uint_as_float(ya[e] & 0xffff0000u);
      s = fmaf(x0, y0, s);
      s = fmaf(x1, y1, s);
      qq = fmaf(x0, x0, fmaf(x1, x1, qq));
      ss = fmaf(y0, y0, fmaf(y1, y1, ss));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    qq += __shfl_xor_sync(0xffffffffu, qq, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const float nu = n * 5.96046448e-8f;
  // the float32 sums of squares are within (1 + gamma_n) of the truth
  const float qn = sqrtf(qq * (1.f + 2.f * nu)) * (1.f + 1.2e-7f);
  const float gfac = nu / (1.f - nu) * 1.0001f * qn * 1.0001f;
  const float E = __fmul_ru(gfac, __fsqrt_ru(__fmul_ru(ss, 1.f + 2.f * nu)));
  return make_float2(__fsub_rd(s, E) + 0.f, __fadd_ru(s, E) + 0.f);
}

// Workspace of filtered_select2 (shared memory).
constexpr int kSelGroupsMax = 512;   // n <= 32 * kSelGroupsMax
constexpr int kSelCap = 1024;        // candidates kept per sequence
struct SelScratch {
  float glo[kSelGroupsMax], ghi[kSelGroupsMax];   // per 32-entry group: max lo / hi
  float clo[kSelCap], chi[kSelCap];               // entries at or above the thresholds
  int cnt[2];
  float tau[2], res[2];
};

// The (k_lo)-th largest of lo[0, n) and the (k_hi)-th largest of hi[0, n)
// (1-based ranks; NaN entries never count), by thresholding: the k-th largest
// of the group maxima (groups of gs consecutive entries) is a lower bound of
// the k-th largest entry (k distinct entries reach it), so every entry at or
// above the k-th largest entry is kept by the filter entry >= that bound; the
// answer is then ranked among the kept entries only.  gs (a power of two up
// to 32) is chosen so that there are about 4k groups or more: the bound is
// then close to the answer and few entries pass.  Returns false (results
// unset) when more than kSelGroupsMax groups would be needed or more than
// kSelCap entries pass a filter.  Called by every thread of the block.
SA_DEV bool filtered_select2(const float* lo, const float* hi, int n, int k_lo, int k_hi,
                             SelScratch* sc, float& out_lo, float& out_hi) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int kmax = max(k_lo, k_hi);
  int gs = 32;
  while (gs > 1 && (n + gs - 1) / gs < 4 * kmax && (n + gs / 2 - 1) / (gs / 2) <= kSelGroupsMax)
    gs >>= 1;
  const int ng = (n + gs - 1) / gs;
  if (ng > kSelGroupsMax) return false;
  // lane l of a warp step covers entry 32 i + l, in group (32 i + l) / gs
  for (int i0 = warp * 32; i0 < ng * gs; i0 += nw * 32) {
    const int i = i0 + lane;
    float a = i < n ? lo[i] : -INFINITY, c = i < n ? hi[i] : -INFINITY;
    a = isnan(a) ? -INFINITY : a;
    c = isnan(c) ? -INFINITY : c;
    for (int o = 1; o < gs; o <<= 1) {
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
    }
    if ((lane & (gs - 1)) == 0 && i < ng * gs) {
      sc->glo[i / gs] = a;
      sc->ghi[i / gs] = c;
    }
  }
  if (tid == 0) {
    sc->cnt[0] = sc->cnt[1] = 0;
    sc->tau[0] = sc->tau[1] = -INFINITY;   // fewer groups than k: keep everything
    sc->res[0] = sc->res[1] = -INFINITY;
  }
  __syncthreads();
  // thresholds: the k-th largest group maximum (g values above, e equal:
  // g < k <= g + e)
  for (int x = tid; x < 2 * ng; x += blockDim.x) {
    const int w = x >= ng;
    const float* arr = w ? sc->ghi : sc->glo;
    const int kk = w ? k_hi : k_lo;
    if (ng < kk) continue;
    const float v = arr[x - w * ng];
    int g = 0, e = 0;
    for (int y = 0; y < ng; ++y) {
      g += arr[y] > v;
      e += arr[y] == v;
    }
    if (g < kk && g + e >= kk) sc->tau[w] = v;
  }
  __syncthreads();
  const float t_lo = sc->tau[0], t_hi = sc->tau[1];
  for (int i = tid; i < n; i += blockDim.x) {
    const float a = lo[i], c = hi[i];
    if (a >= t_lo) {
      const int sl = atomicAdd(&sc->cnt[0], 1);
      if (sl < kSelCap) sc->clo[sl] = a;
    }
    if (c >= t_hi) {
      const int sl = atomicAdd(&sc->cnt[1], 1);
      if (sl < kSelCap) sc->chi[sl] = c;
    }
  }
  __syncthreads();
  const int c0 = sc->cnt[0], c1 = sc->cnt[1];
  if (c0 > kSelCap || c1 > kSelCap) {
    __syncthreads();
    return false;
  }
  for (int x = tid; x < c0 + c1; x += blockDim.x) {
    const int w = x >= c0;
    const float* arr = w ? sc->chi : sc->clo;
    const int cn = w ? c1 : c0, kk = w ? k_hi : k_lo;
    const float v = arr[x - w * c0];
    int g = 0, e = 0;
    for (int y = 0; y < cn; ++y) {
      g += arr[y] > v;
      e += arr[y] == v;
    }
    if (g < kk && g + e >= kk) sc->res[w] = v;
  }
  __syncthreads();
  out_lo = sc->res[0];
  out_hi = sc->res[1];
  __syncthreads();   // the scratch may be reused by the caller
  return true;
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
