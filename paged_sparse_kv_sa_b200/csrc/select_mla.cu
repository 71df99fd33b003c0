// Tiered page selection for one shared latent KV head (MLA + MTP).
//
// Every logical page of a sequence is a candidate; its score is the max over
// all T x Hq query rows of q . sigma (Dk = 576 in DeepSeek-shaped models: a
// 256 x 576 by 576 x N contraction per sequence).  The critical tier is the
// alpha best pages, the ambient tier the next beta, by (score desc, logical
// page asc).  The result is written as two decode lists per sequence: list 0
// = critical pages, list 1 = critical + ambient pages, both ascending.
//
// tiered_score_kernel: one CTA per (64 pages, 64 query rows, sequence); each
// thread owns a 4-page x 4-row register tile and runs float32 FMA chains over
// the 576 features (staged in shared memory in four 144-feature quarters).
// Per page it emits lo/hi = max over its rows of s -+ gamma_Dk ||q_rows|| ||sigma||
// (directed rounding), a rigorous bracket of the exact row-max score.
// tiered_choose_kernel: one CTA per sequence merges the row groups' brackets,
// radix-selects the order statistics for both boundaries (alpha, alpha+beta),
// rescores the undecided pages exactly (fixed-point accumulation of the bf16
// products, one rounding to float64) and writes both lists.
//
// Source: "TileSparse: Arithmetic-Intensity-Aware Sparse Attention for
// Compute-Bound LLM Decoding", "Motivation" (Critical Tier: alpha pages
// computed with all query heads; Ambient Tier: beta pages with h heads).
#include "common.cuh"
#include "exact.cuh"
#include "internal.h"
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kTP = 64;            // pages per scoring CTA
constexpr int kTR = 64;            // query rows per scoring CTA
constexpr int kDq = 144;           // features staged per pass
constexpr int kPad = 4;            // float padding per staged row (bank spread)
constexpr int kChooseThreads = 512;

__global__ void __launch_bounds__(256) tiered_score_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int pc = blockIdx.x, rg = blockIdx.y, b = blockIdx.z;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) L = L < 0 ? 0 : a.max_pages * a.P;
  const int N = (L + a.P - 1) / a.P;
  const int R = a.T * a.Hq;
  const int p0 = pc * kTP, r0 = rg * kTR;
  if (p0 >= N || r0 >= R) return;
  const int Dk = a.Dk;
  extern __shared__ __align__(16) float tsm[];
  float* sg = tsm;                              // [kTP][kDq + kPad]
  float* qs = tsm + kTP * (kDq + kPad);         // [kTR][kDq + kPad]
  __shared__ int phys_s[kTP];
  __shared__ float qn2_s[kTR], sn2_s[kTP];
  const int tid = threadIdx.x;
  if (tid < kTP) {
    const int p = p0 + tid;
    int ph = -1;
    if (p < N) {
      ph = a.page_table[(int64_t)b * a.max_pages + p];
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        ph = -1;
      }
    }
    phys_s[tid] = ph;
    sn2_s[tid] = 0.f;
  }
  if (tid < kTR) qn2_s[tid] = 0.f;
  __syncthreads();
  // thread tile: pages tp + 16i, rows tr + 16j (i, j < 4); consecutive lanes read
  // rows 592 bytes apart, which spreads a quarter-warp over all 16-byte bank slots
  const int tp = tid & 15, tr = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int d0 = 0; d0 < Dk; d0 += kDq) {
    const int dn = min(kDq, Dk - d0);
    // stage summaries and query rows of this feature slice as float32
    for (int i = tid; i < kTP * (kDq / 8); i += 256) {
      const int pg = i / (kDq / 8), c = (i % (kDq / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c < dn && phys_s[pg] >= 0)
        v = *reinterpret_cast<const uint4*>(a.sig + (int64_t)phys_s[pg] * Dk + d0 + c);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float* dst = sg + pg * (kDq + kPad) + c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dst[2 * e] = __uint_as_float(w4[e] << 16);
        dst[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
      }
    }
    for (int i = tid; i < kTR * (kDq / 8); i += 256) {
      const int rr = i / (kDq / 8), c = (i % (kDq / 8)) * 8;
      const int r = r0 + rr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c < dn && r < R) {
        const int t = r / a.Hq, h = r % a.Hq;
        v = *reinterpret_cast<const uint4*>(a.q + b * a.qs0 + t * a.qs1 + h * a.qs2 + d0 + c);
      }
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float* dst = qs + rr * (kDq + kPad) + c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dst[2 * e] = __uint_as_float(w4[e] << 16);
        dst[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
      }
    }
    __syncthreads();
    // squared norms (one thread per page / row; fixed order)
    if (tid < kTP) {
      float s = sn2_s[tid];
      for (int d = 0; d < dn; ++d) s = fmaf(sg[tid * (kDq + kPad) + d], sg[tid * (kDq + kPad) + d], s);
      sn2_s[tid] = s;
    } else if (tid < kTP + kTR) {
      const int rr = tid - kTP;
      float s = qn2_s[rr];
      for (int d = 0; d < dn; ++d) s = fmaf(qs[rr * (kDq + kPad) + d], qs[rr * (kDq + kPad) + d], s);
      qn2_s[rr] = s;
    }
    for (int d = 0; d < dn; d += 4) {
      float4 sv[4], qv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sv[i] = *reinterpret_cast<const float4*>(sg + (tp + 16 * i) * (kDq + kPad) + d);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        qv[j] = *reinterpret_cast<const float4*>(qs + (tr + 16 * j) * (kDq + kPad) + d);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(sv[i].x, qv[j].x, acc[i][j]);
          acc[i][j] = fmaf(sv[i].y, qv[j].y, acc[i][j]);
          acc[i][j] = fmaf(sv[i].z, qv[j].z, acc[i][j]);
          acc[i][j] = fmaf(sv[i].w, qv[j].w, acc[i][j]);
        }
    }
    __syncthreads();
  }
  // bound: gamma_Dk * max_r ||q_r|| * ||sigma|| over this CTA's rows
  __shared__ float qmax_s;
  if (tid == 0) {
    float m = 0.f;
    for (int rr = 0; rr < kTR; ++rr) m = fmaxf(m, qn2_s[rr]);
    qmax_s = m;
  }
  __syncthreads();
  const float nu = Dk * 5.96046448e-8f;
  const float qn = sqrtf(qmax_s * (1.f + 2.f * nu)) * (1.f + 1.2e-7f);
  const float gfac = nu / (1.f - nu) * 1.0001f * qn * 1.0001f;
  // row max per page across the 16 row-threads that share tp (lanes tp, tp+16 in
  // each warp, across 8 warps): reduce through shared memory
  __shared__ float pmax_s[kTP][16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (r0 + tr + 16 * j < R) m = fmaxf(m, acc[i][j]);
    pmax_s[tp + 16 * i][tr] = m;
  }
  __syncthreads();
  if (tid < kTP) {
    const int p = p0 + tid;
    if (p < N) {
      float m = -INFINITY;
      for (int k = 0; k < 16; ++k) m = fmaxf(m, pmax_s[tid][k]);
      float2 out;
      if (phys_s[tid] < 0) {
        out = make_float2(-INFINITY, -INFINITY);
      } else {
        const float E = __fmul_ru(gfac, __fsqrt_ru(__fmul_ru(sn2_s[tid], 1.f + 2.f * nu)));
        out = make_float2(__fsub_rd(m, E) + 0.f, __fadd_ru(m, E) + 0.f);
      }
      a.lohi[((int64_t)b * a.n_rg + rg) * a.max_pages + p] = out;
    }
  }
}

// Block-wide ascending compaction of the pages whose flag has `bit` set.
SA_DEV int compact_pages(const uint8_t* flag, int N, uint8_t bit, int32_t* out, int cap,
                         int* red_i) {
  const int tid = threadIdx.x;
  const int per_t = (N + blockDim.x - 1) / blockDim.x;
  const int p0 = tid * per_t, p1 = min(N, p0 + per_t);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += (flag[p] & bit) != 0;
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
    if ((flag[p] & bit) && pos < cap) out[pos++] = p;
  for (int i = total + tid; i < cap; i += blockDim.x) out[i] = -1;
  __syncthreads();   // red_i is reused by the next call
  return min(total, cap);
}

// Out of line: the exact dot needs many registers, and inlined it would raise
// the register count (and spills) of the whole choose kernel.
__device__ __noinline__ double exact_row_dot(const uint16_t* q, const uint16_t* sg, int n) {
  return warp_exact_dot_bf16<4>(q, sg, n);
}

__global__ void __launch_bounds__(kChooseThreads) tiered_choose_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int b = blockIdx.x, tid = threadIdx.x;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  const int N = (L + a.P - 1) / a.P;
  const int cap = a.alpha + a.beta;
  int32_t* out0 = a.lists + (int64_t)b * 2 * cap;
  int32_t* out1 = out0 + cap;
  extern __shared__ __align__(16) uint8_t dsm[];
  float* lo = reinterpret_cast<float*>(dsm);
  float* hi = lo + a.max_pages;
  uint16_t* u_list = reinterpret_cast<uint16_t*>(hi + a.max_pages);
  uint8_t* flag = reinterpret_cast<uint8_t*>(u_list + a.max_pages);
  __shared__ uint32_t hist[1024];
  __shared__ uint32_t sel_out[8];
  __shared__ SelScratch scratch;
  __shared__ int red_i[kChooseThreads / 32];
  __shared__ int n_unc, n_cert[2];
  __shared__ uint32_t mlo_s[kChooseThreads];
  __shared__ unsigned long long best_s[kChooseThreads];
  const int R = a.T * a.Hq;
  const int kb[2] = {min(a.alpha, N), min(a.alpha + a.beta, N)};
  // flag bits: 1 / 2 = in tier boundary 0 / 1, 4 / 8 = undecided for it
  for (int p = tid; p < N; p += blockDim.x) {
    float l = -INFINITY, h = -INFINITY;
    for (int rg = 0; rg < a.n_rg; ++rg) {
      const float2 v = a.lohi[((int64_t)b * a.n_rg + rg) * a.max_pages + p];
      l = fmaxf(l, v.x);
      h = fmaxf(h, v.y);
    }
    lo[p] = l;
    hi[p] = h;
    flag[p] = 0;
  }
  if (tid == 0) {
    n_unc = 0;
    n_cert[0] = n_cert[1] = 0;
  }
  __syncthreads();
  for (int i = 0; i < 2; ++i) {
    const uint8_t in_bit = 1u << i, unc_bit = 4u << i;
    if (kb[i] >= N) {   // every page is inside this boundary
      for (int p = tid; p < N; p += blockDim.x) flag[p] |= in_bit;
      continue;
    }
    if (kb[i] == 0) continue;
    float Lk, H;
    if (!filtered_select2(lo, hi, N, kb[i], kb[i] + 1, &scratch, Lk, H))
      radix_select2(lo, hi, N, kb[i], kb[i] + 1, hist, sel_out, Lk, H);
    for (int p = tid; p < N; p += blockDim.x) {
      if (lo[p] > H) {
        flag[p] |= in_bit;
        atomicAdd(&n_cert[i], 1);
      } else if (hi[p] >= Lk) {
        if (!(flag[p] & 12u)) u_list[atomicAdd(&n_unc, 1)] = static_cast<uint16_t>(p);
        flag[p] |= unc_bit;
      }
    }
    __syncthreads();
  }
  const int nu_ = n_unc;
  double* ex = reinterpret_cast<double*>(lo);   // lo/hi storage reused as doubles
  if (nu_ > 0) {
    // exact row-max scores of the undecided pages, up to 512 pages per round.
    // Pass 1: a float32 bracket of every (page, row) score, one warp each; per
    // page the largest lower end m.  Pass 2: only rows whose upper end reaches
    // m can hold the page's maximum (the row that attains the exact maximum
    // has exact score >= m); those rows are rescored exactly.
    const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
    const int nw = kChooseThreads / 32, warp = tid >> 5, lane = tid & 31;
    for (int u0 = 0; u0 < nu_; u0 += kChooseThreads) {
      const int np = min(kChooseThreads, nu_ - u0);
      for (int i = tid; i < np; i += blockDim.x) {
        mlo_s[i] = 0u;
        best_s[i] = 0ull;
      }
      __syncthreads();
      const int64_t n_pairs = (int64_t)np * R;
      for (int pass = 0; pass < 2; ++pass) {
        for (int64_t pr = warp; pr < n_pairs; pr += nw) {
          const int uu = static_cast<int>(pr / R), r = static_cast<int>(pr % R);
          const int ph = ptrow[u_list[u0 + uu]];
          if (ph < 0 || ph >= a.P_pool) continue;
          const int t = r / a.Hq, h = r % a.Hq;
          const uint16_t* qr = a.q + b * a.qs0 + t * a.qs1 + h * a.qs2;
          const uint16_t* sg = a.sig + (int64_t)ph * a.Dk;
          const float2 br = warp_score_bracket(qr, sg, a.Dk);
          if (pass == 0) {
            if (lane == 0) atomicMax(&mlo_s[uu], f2key(br.x));
          } else if (br.y >= key2f(mlo_s[uu])) {
            const double e = exact_row_dot(qr, sg, a.Dk);
            if (lane == 0) atomicMax(&best_s[uu], d2key(e));
          }
        }
        __syncthreads();
      }
      for (int i = tid; i < np; i += blockDim.x) {
        const int ph = ptrow[u_list[u0 + i]];
        ex[u0 + i] = (ph < 0 || ph >= a.P_pool) ? -INFINITY : key2d(best_s[i]);
      }
      __syncthreads();
    }
    // per boundary: the undecided pages fill the slots the certain ones left
    for (int i = 0; i < 2; ++i) {
      const uint8_t in_bit = 1u << i, unc_bit = 4u << i;
      const int slots = kb[i] - n_cert[i];
      for (int u = tid; u < nu_; u += blockDim.x) {
        const int pu = u_list[u];
        if (!(flag[pu] & unc_bit)) continue;
        const double su = ex[u];
        int rank = 0;
        for (int v = 0; v < nu_; ++v) {
          const int pv = u_list[v];
          if (!(flag[pv] & unc_bit)) continue;
          const double sv = ex[v];
          rank += (sv > su) || (sv == su && pv < pu);
        }
        if (rank < slots) flag[pu] |= in_bit;
      }
      __syncthreads();
    }
  }
  const int c0 = compact_pages(flag, N, 1u, out0, cap, red_i);
  const int c1 = compact_pages(flag, N, 2u, out1, cap, red_i);
  if (tid == 0) {
    a.counts[2 * b] = c0;
    a.counts[2 * b + 1] = c1;
  }
}

}  // namespace

size_t tiered_workspace_bytes(int B, int T, int Hq, int max_pages) {
  const int n_rg = (T * Hq + kTR - 1) / kTR;
  return (size_t)B * n_rg * max_pages * sizeof(float2);
}

cudaError_t launch_select_tiered(TieredArgs a, cudaStream_t stream) {
  a.n_rg = (a.T * a.Hq + kTR - 1) / kTR;
  const int dyn1 = (kTP + kTR) * (kDq + kPad) * 4;
  cudaError_t e = cudaFuncSetAttribute(tiered_score_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, dyn1);
  if (e != cudaSuccess) return e;
  dim3 g1((a.max_pages + kTP - 1) / kTP, a.n_rg, a.B);
  e = launch_pdl(tiered_score_kernel, g1, dim3(256), dyn1, stream, a);
  if (e != cudaSuccess) return e;
  const size_t dyn2 = (size_t)a.max_pages * (4 + 4 + 2 + 1) + 16;
  e = cudaFuncSetAttribute(tiered_choose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dyn2);
  if (e != cudaSuccess) return e;
  return launch_pdl(tiered_choose_kernel, dim3(a.B), dim3(kChooseThreads), dyn2, stream, a);
}

}  // namespace sa
