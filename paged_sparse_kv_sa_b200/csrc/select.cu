// Page scoring and top-k selection (GQA): one CTA per (kv head, sequence).
//
// 1. Every candidate page (neither sink nor local) is scored in float32 with a
//    fixed-order FMA chain per query row, and given a rigorous error bound
//    E = gamma_Dk * max_r ||q_r|| * ||sigma|| (|fl(sum) - sum| <= gamma_n sum|q_d
//    sigma_d| <= gamma_n ||q|| ||sigma||), so the exact score lies in
//    [lo, hi] = [s - E, s + E] (directed rounding).
// 2. Radix selection over the float keys finds H = the (k+1)-th largest hi and
//    Lk = the k-th largest lo.  A page with lo > H is certainly among the top
//    k; a page with hi < Lk certainly is not.
// 3. The few pages left in between are rescored exactly (bf16 products summed
//    in a fixed-point accumulator, rounded once to float64) and ranked by
//    (exact score desc, logical page asc) for the remaining slots.
// 4. Forced and selected pages are written in ascending logical order.
//
// Source: "Universal Attention Engine — Declarative Sparse Attention for
// Production", "Content-Dependent Dynamic Routing" (top_k_blocks over
// q @ mean(k_blocks), at block granularity) and "The Product" (sink + local).
#include "common.cuh"
#include "exact.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxRows = 16;
constexpr int kMaxDk = 256;

SA_DEV uint32_t f2key(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
SA_DEV float key2f(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// RN64(q . sigma) for a query row held as float32 copies of bf16 values.
__device__ double exact_dot_f32q(const float* q, const uint16_t* sig, int n) {
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

// Shared-memory layout (dynamic): lo[Nmax] f32, hi[Nmax] f32, u_list[Nmax] u16,
// flag[Nmax] u8; q rows [R][Dk] f32 in static memory.
struct SelSmem {
  float* lo;
  float* hi;
  uint8_t* flag;   // 0 = not selected, 1 = selected (forced or winner), 2 = uncertain
  uint16_t* u_list;
};

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

__global__ void __launch_bounds__(kThreads) select_gqa_kernel(const SelectArgs a) {
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int G = a.Hq / a.Hkv;
  const int R = a.T * G;
  const int Dk = a.Dk;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {  // a length the page table cannot hold
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  const int N = (L + a.P - 1) / a.P;
  int32_t* outp = a.out_pages + ((int64_t)b * a.Hkv + kvh) * a.budget_pages;
  int32_t* outc = a.out_counts + (int64_t)b * a.Hkv + kvh;

  if (N <= a.budget_pages) {  // every page is selected
    for (int i = tid; i < a.budget_pages; i += blockDim.x) outp[i] = i < N ? i : -1;
    if (tid == 0) *outc = N;
    return;
  }

  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float q_s[kMaxRows * kMaxDk];
  __shared__ uint32_t hist[512];
  __shared__ uint32_t sel_out[4];
  __shared__ float red_f[kThreads / 32];
  __shared__ int red_i[kThreads / 32];
  __shared__ int n_unc, n_certain;
  __shared__ double ex_tmp[kThreads];

  SelSmem S;
  S.lo = reinterpret_cast<float*>(dsm);
  S.hi = S.lo + a.max_pages;
  S.u_list = reinterpret_cast<uint16_t*>(S.hi + a.max_pages);
  S.flag = reinterpret_cast<uint8_t*>(S.u_list + a.max_pages);

  // ---- query rows (t, h in group) as float32 (exact), and max_r ||q_r||
  for (int i = tid; i < R * Dk; i += blockDim.x) {
    const int r = i / Dk, d = i % Dk;
    const int t = r / G, h = kvh * G + r % G;
    q_s[i] = bf16_bits_to_float(a.q[b * a.qs0 + t * a.qs1 + h * a.qs2 + d]);
  }
  if (tid == 0) {
    n_unc = 0;
    n_certain = 0;
  }
  __syncthreads();
  float qn = 0.f;
  {
    const int w = tid >> 5, lane = tid & 31;
    for (int r = w; r < R; r += blockDim.x / 32) {
      float ss = 0.f;
      for (int d = lane; d < Dk; d += 32) ss = fmaf(q_s[r * Dk + d], q_s[r * Dk + d], ss);
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      qn = fmaxf(qn, ss);
    }
    if (lane == 0) red_f[w] = qn;
    __syncthreads();
    qn = 0.f;
    for (int i = 0; i < (int)(blockDim.x / 32); ++i) qn = fmaxf(qn, red_f[i]);
    // sum of squares within (1 + gamma_Dk) of the truth: inflate before sqrt
    qn = sqrtf(qn * (1.f + 2.f * Dk * 5.96046448e-8f)) * (1.f + 1.2e-7f);
  }
  // gamma_n = n u / (1 - n u), u = 2^-24, padded for the products below
  const float nu = Dk * 5.96046448e-8f;
  const float gamma = nu / (1.f - nu) * 1.0001f;
  const float gfac = gamma * qn * 1.0001f;
  const float sq_pad = 1.f + 2.f * nu;

  const int n_sink = min(a.n_sink, N), local0 = max(N - a.n_local, 0);
  const int k = a.k_top;

  // ---- 1. score candidates
  const uint16_t* sig_base = a.sig + (int64_t)kvh * Dk;
  const int64_t sig_page = (int64_t)a.Hkv * Dk;
  const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
  for (int p = tid; p < N; p += blockDim.x) {
    const bool cand = p >= n_sink && p < local0;
    S.flag[p] = cand ? 0 : 1;
    float lo = NAN, hi = NAN;
    if (cand) {
      const int ph = ptrow[p];
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        lo = hi = -INFINITY;     // an unreadable page never wins a slot
      } else {
        const uint4* row = reinterpret_cast<const uint4*>(sig_base + ph * sig_page);
        float acc[kMaxRows];
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
        float ss = 0.f;
        // 64 features per batch: 8 x 16-byte loads, unpacked once, then every
        // query row streams its 64 float32 coefficients from shared memory.
        for (int d0 = 0; d0 < Dk; d0 += 64) {
          uint4 v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = row[d0 / 8 + j];
          float x[64];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              x[8 * j + 2 * e] = __uint_as_float(w4[e] << 16);
              x[8 * j + 2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
            }
          }
#pragma unroll
          for (int i = 0; i < 64; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
          for (int r = 0; r < kMaxRows; ++r) {
            if (r < R) {
              const float4* qr = reinterpret_cast<const float4*>(&q_s[r * Dk + d0]);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float4 qq = qr[i];
                acc[r] = fmaf(qq.x, x[4 * i], acc[r]);
                acc[r] = fmaf(qq.y, x[4 * i + 1], acc[r]);
                acc[r] = fmaf(qq.z, x[4 * i + 2], acc[r]);
                acc[r] = fmaf(qq.w, x[4 * i + 3], acc[r]);
              }
            }
          }
        }
        float s = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
          if (r < R) s = fmaxf(s, acc[r]);
        const float E = __fmul_ru(gfac, __fsqrt_ru(__fmul_ru(ss, sq_pad)));
        lo = __fsub_rd(s, E) + 0.f;     // + 0 turns -0 into +0 (keys order -0 < +0)
        hi = __fadd_ru(s, E) + 0.f;
      }
    }
    S.lo[p] = lo;
    S.hi[p] = hi;
  }
  __syncthreads();

  // ---- 2. order statistics of the bounds (k == 0: streaming, no winners)
  float Lk = INFINITY, H = INFINITY;
  if (k > 0) radix_select2(S.lo, S.hi, N, k, k + 1, hist, sel_out, Lk, H);

  // ---- classify
  for (int p = tid; p < N; p += blockDim.x) {
    if (S.flag[p] != 0) continue;
    if (S.lo[p] > H) {
      S.flag[p] = 1;
      atomicAdd(&n_certain, 1);
    } else if (S.hi[p] >= Lk) {
      S.flag[p] = 2;
      S.u_list[atomicAdd(&n_unc, 1)] = static_cast<uint16_t>(p);
    }
  }
  __syncthreads();
  const int nu_ = n_unc;
  const int slots = k - n_certain;

  // ---- 3. exact scores of the uncertain pages (lo/hi reused as double storage)
  double* ex = reinterpret_cast<double*>(S.lo);
  if (nu_ > 0 && slots > 0) {
    const int per = max(1, kThreads / R);            // uncertain pages per batch
    for (int u0 = 0; u0 < nu_; u0 += per) {
      const int i = tid;
      const int u = u0 + i / R, r = i % R;
      if (i < per * R && u < nu_) {
        const int p = S.u_list[u];
        const int ph = ptrow[p];
        ex_tmp[i] = (ph < 0 || ph >= a.P_pool)
                        ? -INFINITY
                        : exact_dot_f32q(&q_s[r * Dk], sig_base + ph * sig_page, Dk);
      }
      __syncthreads();
      if (i < per && u0 + i < nu_) {
        double m = -INFINITY;
        for (int rr = 0; rr < R; ++rr) m = fmax(m, ex_tmp[i * R + rr]);
        ex[u0 + i] = m;
      }
      __syncthreads();
    }
    // rank among the uncertain pages: (exact desc, logical asc)
    for (int u = tid; u < nu_; u += blockDim.x) {
      const double su = ex[u];
      const int pu = S.u_list[u];
      int rank = 0;
      for (int v = 0; v < nu_; ++v) {
        const double sv = ex[v];
        rank += (sv > su) || (sv == su && S.u_list[v] < pu);
      }
      S.flag[pu] = rank < slots ? 1 : 0;
    }
  } else {
    for (int u = tid; u < nu_; u += blockDim.x) S.flag[S.u_list[u]] = 0;
  }
  __syncthreads();

  // ---- 4. ascending compaction of the selected pages
  const int per_t = (N + blockDim.x - 1) / blockDim.x;
  const int p0 = tid * per_t, p1 = min(N, p0 + per_t);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += S.flag[p] == 1;
  // block exclusive scan of cnt
  const int w = tid >> 5, lane = tid & 31;
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) red_i[w] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int i = 0; i < (int)(blockDim.x / 32); ++i) {
    if (i < w) wbase += red_i[i];
    total += red_i[i];
  }
  int pos = wbase + incl - cnt;
  for (int p = p0; p < p1; ++p)
    if (S.flag[p] == 1 && pos < a.budget_pages) outp[pos++] = p;
  for (int i = total + tid; i < a.budget_pages; i += blockDim.x) outp[i] = -1;
  if (tid == 0) *outc = min(total, a.budget_pages);
}

}  // namespace

cudaError_t launch_select_gqa(const SelectArgs& a, cudaStream_t stream) {
  const size_t dyn = (size_t)a.max_pages * (4 + 4 + 2 + 1) + 16;
  cudaError_t e = cudaFuncSetAttribute(select_gqa_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hkv, a.B);
  select_gqa_kernel<<<grid, kThreads, dyn, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace sa
