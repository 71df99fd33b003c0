// Tiered page selection for one shared latent KV head (MLA + MTP).
//
// Every logical page of a sequence is a candidate; its score is the max over
// all T x Hq query rows of q . sigma (Dk = 576 in DeepSeek-shaped models: a
// 256 x 576 by 576 x N contraction per sequence).  The critical tier is the
// alpha best pages, the ambient tier the next beta, by (score desc, logical
// page asc).  The result is written as two decode lists per sequence: list 0
// = critical pages, list 1 = critical + ambient pages, both ascending.
//
// tiered_score_kernel: one CTA per (64 pages, 64 query rows, sequence) scores
// with warp MMAs and emits, per page and row group, a rigorous bracket of the
// row-max score and the mask of rows that can attain it.
// tiered_choose_kernel: one CTA per sequence merges the row groups' brackets,
// selects the order statistics for both boundaries (alpha, alpha+beta),
// rescores the undecided pages exactly on their flagged rows only (fixed-point
// accumulation of the bf16 products, one rounding to float64) and writes both
// lists.
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
constexpr int kTR = 32;            // query rows per scoring CTA (one 32-bit row mask)
constexpr int kTNT = kTR / 16;     // 8-row MMA tiles per warp
constexpr int kTScoreThreads = 256;
constexpr int kChooseThreads = 512;
constexpr int kChooseCtas = 8;     // CTAs per sequence sharing the exact rescoring

// Scores of 64 pages x 32 query rows of one sequence, S = sigma q^T as warp
// MMAs over the Dk features (m16n8k16, bf16 in, float32 accumulation).  Per
// (page, row) the exact score lies in s -/+ E with (directed rounding)
//   E = c_acc ||q_r|| ||sigma|| + 2^-126 (||q_r||_1 + sqrt(Dk) ||sigma||) + Dk 2^-124,
// c_acc = Dk 2^-20: the accumulation of each 16-product step loses less than
// 2^-17.9 of the running magnitude sum sum_d |q_d sigma_d| <= ||q|| ||sigma||
// even if every addend were truncated at the largest exponent (a margin of
// about 3.5x); the 2^-126 terms cover subnormal inputs flushed to zero inside
// the MMA, Dk 2^-124 products that underflow float32.  The norms are float32
// sums of squares, rounded up.  Emitted per page: [max_r (s_r - E_r),
// max_r (s_r + E_r)] over the CTA's rows, and a mask of the rows whose upper
// end reaches that largest lower end (only those rows can hold the page's
// maximum within this row group).  Summary and query rows arrive with one bulk
// copy each (rows padded by 16 bytes so that ldmatrix row addresses hit
// distinct banks).  Two CTAs fit an SM, so one's loads overlap the other's MMAs.
__global__ void __launch_bounds__(kTScoreThreads) tiered_score_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int pc = blockIdx.x, rg = blockIdx.y, b = blockIdx.z;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) L = L < 0 ? 0 : a.max_pages * a.P;
  const int N = (L + a.P - 1) / a.P;
  const int R = a.T * a.Hq;
  const int p0 = pc * kTP, r0 = rg * kTR;
  if (p0 >= N || r0 >= R) return;
  const int Dk = a.Dk, KP = (Dk + 15) & ~15, RS = KP * 2 + 16;
  // the choose kernel's exact-score slots and completion counter start at 0
  if (rg == 0 && threadIdx.x < kTP && p0 + threadIdx.x < N)
    a.exkey[(int64_t)b * a.max_pages + p0 + threadIdx.x] = 0ull;
  if (pc == 0 && rg == 0 && threadIdx.x == 0) a.counter[b] = 0u;
  extern __shared__ __align__(128) uint8_t tsm[];
  uint8_t* sg_s = tsm;                  // [kTP][RS] summaries
  uint8_t* q_s = tsm + kTP * RS;        // [kTR][RS] query rows
  __shared__ uint64_t ld_bar;
  __shared__ int phys_s[kTP];
  __shared__ float qn_s[kTR];           // ||q_r||_2, rounded up
  __shared__ float fl_s[kTR];           // 2^-126 ||q_r||_1, rounded up
  __shared__ float sn_s[kTP];           // ||sigma_p||_2, rounded up
  __shared__ float2 half_s[4][16];      // rows of the second warp half: per page (lo, hi)
  __shared__ float mlo_s[kTP];          // per page: largest lower end over the rows
  __shared__ unsigned long long mhalf_s[4][16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  }
  if (tid == 0) {
    mbar_init(&ld_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_rows = min(kTR, R - r0);
  const uint32_t rowb = Dk * 2;
  if (warp == 0) {
    const uint32_t m0 = __ballot_sync(0xffffffffu, phys_s[lane] >= 0);
    const uint32_t m1 = __ballot_sync(0xffffffffu, phys_s[32 + lane] >= 0);
    if (lane == 0) mbar_arrive_expect_tx(&ld_bar, (__popc(m0) + __popc(m1) + n_rows) * rowb);
    __syncwarp();
#pragma unroll
    for (int i = lane; i < kTP; i += 32)
      if (phys_s[i] >= 0) bulk_load(sg_s + i * RS, a.sig + (int64_t)phys_s[i] * Dk, rowb, &ld_bar);
  } else if (warp == 1) {
#pragma unroll
    for (int i = lane; i < kTR; i += 32)
      if (i < n_rows) {
        const int r = r0 + i, t = r / a.Hq, h = r % a.Hq;
        bulk_load(q_s + i * RS, a.q + b * a.qs0 + t * a.qs1 + h * a.qs2, rowb, &ld_bar);
      }
  }
  if (KP != Dk)   // the last 8 features of a 16-feature step: zeros
    for (int i = tid; i < kTP + kTR; i += blockDim.x)
      *reinterpret_cast<uint4*>(tsm + i * RS + rowb) = make_uint4(0, 0, 0, 0);
  if (__syncthreads_or(!mbar_wait_bounded(&ld_bar, 0))) {
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
    return;
  }
  // norms: per query row ||q_r||_2 and ||q_r||_1, per page ||sigma_p||_2 (float32
  // sums, within (1 + gamma_Dk) of the truth: padded up); one warp per row
  // 4 lanes per row, 8 rows per warp step, the rows in parallel
  const float pad = 1.f + 2.f * Dk * 5.96046448e-8f;
  for (int rr0 = warp * 8; rr0 < kTR + kTP; rr0 += kTScoreThreads / 4) {
    const int rr = rr0 + (lane >> 2), part = lane & 3;
    const uint8_t* row = rr < kTR ? q_s + rr * RS : sg_s + (rr - kTR) * RS;
    const bool live = rr < kTR + kTP && (rr < kTR ? rr < n_rows : phys_s[rr - kTR] >= 0);
    float s1 = 0.f, s2 = 0.f;
    if (live)
      for (int c = part; c < Dk / 8; c += 4) {
        const uint4 x4 = *reinterpret_cast<const uint4*>(row + c * 16);
        const uint32_t w4[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(w4[e] << 16), x1 = __uint_as_float(w4[e] & 0xffff0000u);
          s1 += fabsf(x0) + fabsf(x1);
          s2 = fmaf(x0, x0, fmaf(x1, x1, s2));
        }
      }
#pragma unroll
    for (int o = 2; o; o >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    if (part == 0 && rr < kTR + kTP) {
      const float n2 = __fmul_ru(__fsqrt_ru(__fmul_ru(s2, pad)), 1.0000002f);
      if (rr < kTR) {
        qn_s[rr] = n2;
        fl_s[rr] = __fmul_ru(__fmul_ru(s1, pad), 1.1754943508222875e-38f);
      } else {
        sn_s[rr - kTR] = n2;
      }
    }
  }
  __syncthreads();

  // warp w: pages 16 (w & 3) .. + 15, query rows 8 kTNT (w >> 2) .. + 8 kTNT - 1
  const int mt = warp & 3, nh = warp >> 2;
  const int gq = lane >> 2, cq = lane & 3;
  const uint32_t a_addr = smem_u32(sg_s) + (16 * mt + (lane & 15)) * RS + 16 * (lane >> 4);
  const uint32_t b_addr =
      smem_u32(q_s) + (8 * kTNT * nh + (lane & 7)) * RS + 16 * ((lane >> 3) & 1);
  float acc[kTNT][4];
#pragma unroll
  for (int nt = 0; nt < kTNT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll 4
  for (int ks = 0; ks < KP / 16; ++ks) {
    uint32_t af[4];
    ldmatrix_x4(af, a_addr + ks * 32);
#pragma unroll
    for (int nt = 0; nt < kTNT; ++nt) {
      uint32_t bq[2];
      ldmatrix_x2(bq, b_addr + nt * 8 * RS + ks * 32);
      mma_bf16_16816(acc[nt], af, bq[0], bq[1]);
    }
  }
  // this lane: pages 16 mt + gq (i = 0, 1) and + 8 (i = 2, 3); rows
  // 8 kTNT nh + 8 nt + 2 cq + (i & 1) of the CTA
  const float c_acc = Dk * 9.5367431640625e-07f;       // Dk * 2^-20
  const float e_abs = Dk * 4.70197740328915e-38f;      // Dk * 2^-124
  const float rt = __fsqrt_ru(static_cast<float>(Dk)) * 1.1754943508222875e-38f;
  float sn[2], en[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    sn[h] = sn_s[16 * mt + gq + 8 * h];
    en[h] = __fadd_ru(__fmul_ru(rt, sn[h]), e_abs);
  }
  float hr[kTNT][4];                    // per element: s + E (for the row mask)
  float lo[2] = {-INFINITY, -INFINITY}, hi[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < kTNT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 8 * kTNT * nh + 8 * nt + 2 * cq + (i & 1);
      const int h = i >> 1;
      hr[nt][i] = -INFINITY;
      if (rr < n_rows) {
        const float E = __fadd_ru(__fmul_ru(__fmul_ru(c_acc, qn_s[rr]), sn[h]),
                                  __fadd_ru(fl_s[rr], en[h]));
        const float sv = acc[nt][i];
        hr[nt][i] = __fadd_ru(sv, E);
        lo[h] = fmaxf(lo[h], __fsub_rd(sv, E));
        hi[h] = fmaxf(hi[h], hr[nt][i]);
      }
    }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      lo[h] = fmaxf(lo[h], __shfl_xor_sync(0xffffffffu, lo[h], o));
      hi[h] = fmaxf(hi[h], __shfl_xor_sync(0xffffffffu, hi[h], o));
    }
  if (nh == 1 && cq == 0)
    for (int h = 0; h < 2; ++h) half_s[mt][gq + 8 * h] = make_float2(lo[h], hi[h]);
  __syncthreads();
  if (nh == 0 && cq == 0)
    for (int h = 0; h < 2; ++h) {
      const int pl = 16 * mt + gq + 8 * h, p = p0 + pl;
      const float2 o2 = half_s[mt][gq + 8 * h];
      const float l2 = fmaxf(lo[h], o2.x), h2 = fmaxf(hi[h], o2.y);
      mlo_s[pl] = l2;
      if (p < N) {
        // + 0 turns -0 into +0 (the radix keys order -0 below +0)
        a.lohi[((int64_t)b * a.n_rg + rg) * a.max_pages + p] =
            phys_s[pl] < 0 ? make_float2(-INFINITY, -INFINITY) : make_float2(l2 + 0.f, h2 + 0.f);
      }
    }
  __syncthreads();
  // rows whose upper end reaches the page's largest lower end
  unsigned long long bits[2] = {0ull, 0ull};
#pragma unroll
  for (int nt = 0; nt < kTNT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 8 * kTNT * nh + 8 * nt + 2 * cq + (i & 1);
      if (hr[nt][i] >= mlo_s[16 * mt + gq + 8 * (i >> 1)]) bits[i >> 1] |= 1ull << rr;
    }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) bits[h] |= __shfl_xor_sync(0xffffffffu, bits[h], o);
  if (nh == 1 && cq == 0)
    for (int h = 0; h < 2; ++h) mhalf_s[mt][gq + 8 * h] = bits[h];
  __syncthreads();
  if (nh == 0 && cq == 0)
    for (int h = 0; h < 2; ++h) {
      const int pl = 16 * mt + gq + 8 * h, p = p0 + pl;
      if (p < N)
        a.rmask[((int64_t)b * a.n_rg + rg) * a.max_pages + p] =
            phys_s[pl] < 0 ? 0ull : (bits[h] | mhalf_s[mt][gq + 8 * h]);
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

// Block-wide ascending list (in shared memory) of the pages whose flag has any
// of `bits` set; returns its length.
SA_DEV int compact_flag_list(const uint8_t* flag, int N, uint8_t bits, uint16_t* list, int* red_i) {
  const int tid = threadIdx.x;
  const int per_t = (N + blockDim.x - 1) / blockDim.x;
  const int p0 = tid * per_t, p1 = min(N, p0 + per_t);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += (flag[p] & bits) != 0;
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
    if (flag[p] & bits) list[pos++] = static_cast<uint16_t>(p);
  __syncthreads();   // red_i is reused; the list is complete
  return total;
}

// Out of line: the exact dot needs many registers, and inlined it would raise
// the register count (and spills) of the whole choose kernel.
__device__ __noinline__ double exact_row_dot(const uint16_t* q, const uint16_t* sg, int n) {
  return warp_exact_dot_bf16<4>(q, sg, n);
}

__global__ void __launch_bounds__(kChooseThreads) tiered_choose_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int b = blockIdx.x, cta = blockIdx.y, tid = threadIdx.x;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
    if (tid == 0 && cta == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
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
  __shared__ int n_cert[2];
  __shared__ int last_s;
  const int kb[2] = {min(a.alpha, N), min(a.alpha + a.beta, N)};
  // flag bits: 1 / 2 = in tier boundary 0 / 1, 4 / 8 = undecided for it
  // (the row groups' brackets of a thread's pages, 8 loads in flight at a time)
  for (int p = tid; p < N; p += blockDim.x) {
    float l = -INFINITY, h = -INFINITY;
    for (int rg0 = 0; rg0 < a.n_rg; rg0 += 8) {
      float2 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = rg0 + j < a.n_rg ? a.lohi[((int64_t)b * a.n_rg + rg0 + j) * a.max_pages + p]
                                : make_float2(-INFINITY, -INFINITY);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        l = fmaxf(l, v[j].x);
        h = fmaxf(h, v[j].y);
      }
    }
    lo[p] = l;
    hi[p] = h;
    flag[p] = 0;
  }
  if (tid == 0) {
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
        flag[p] |= unc_bit;
      }
    }
    __syncthreads();
  }
  // the undecided pages, ascending (the same list in every CTA of the sequence)
  const int nu_ = compact_flag_list(flag, N, 12u, u_list, red_i);
  double* ex = reinterpret_cast<double*>(lo);   // lo/hi storage reused as doubles
  if (nu_ == 0 && cta != 0) return;             // nothing to share: CTA 0 writes
  if (nu_ > 0) {
    // exact row-max scores of the undecided pages: only the query rows the
    // scoring pass flagged for a page (per row group, the rows whose upper end
    // reaches the group's largest lower end) can hold its maximum.  One warp
    // rescores each such (page, row) exactly; the (page, row group) tasks are
    // dealt round-robin over the sequence's CTAs and their warps, the results
    // merged with atomic max in global memory; the last CTA to finish ranks.
    const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
    const int nw = kChooseThreads / 32, warp = tid >> 5, lane = tid & 31;
    unsigned long long* exk = a.exkey + (int64_t)b * a.max_pages;
    for (int x = cta + kChooseCtas * warp; x < nu_ * a.n_rg; x += kChooseCtas * nw) {
      const int uu = x / a.n_rg, g = x % a.n_rg;
      const int pu = u_list[uu];
      const int ph = ptrow[pu];
      if (ph < 0 || ph >= a.P_pool) continue;
      unsigned long long bits = a.rmask[((int64_t)b * a.n_rg + g) * a.max_pages + pu];
      const uint16_t* sg = a.sig + (int64_t)ph * a.Dk;
      while (bits) {
        const int r = g * kTR + __ffsll(static_cast<long long>(bits)) - 1;
        bits &= bits - 1;
        const int t = r / a.Hq, h = r % a.Hq;
        const double e = exact_row_dot(a.q + b * a.qs0 + t * a.qs1 + h * a.qs2, sg, a.Dk);
        if (lane == 0) atomicMax(&exk[uu], d2key(e));
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = atomicAdd(&a.counter[b], 1u) == kChooseCtas - 1;
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    for (int i = tid; i < nu_; i += blockDim.x) {
      const unsigned long long k = __ldcg(&exk[i]);
      const int ph = ptrow[u_list[i]];
      ex[i] = (ph < 0 || ph >= a.P_pool || k == 0ull) ? -INFINITY : key2d(k);
    }
    __syncthreads();
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

// Workspace: score brackets [B, n_rg, max_pages] float2, row masks [B, n_rg,
// max_pages] u64, exact-score keys [B, max_pages] u64, counters [B] u32.
size_t tiered_workspace_bytes(int B, int T, int Hq, int max_pages) {
  const size_t n_rg = (T * Hq + kTR - 1) / kTR;
  const size_t cnt = ((size_t)B * sizeof(unsigned int) + 15) / 16 * 16;
  return (size_t)B * max_pages * (n_rg * (sizeof(float2) + sizeof(unsigned long long)) +
                                   sizeof(unsigned long long)) + cnt;
}

cudaError_t launch_select_tiered(TieredArgs a, cudaStream_t stream) {
  a.n_rg = (a.T * a.Hq + kTR - 1) / kTR;
  const size_t nl = (size_t)a.B * a.n_rg * a.max_pages;
  a.rmask = reinterpret_cast<unsigned long long*>(a.lohi + nl);
  a.exkey = a.rmask + nl;
  a.counter = reinterpret_cast<unsigned int*>(a.exkey + (size_t)a.B * a.max_pages);
  const int RS = ((a.Dk + 15) & ~15) * 2 + 16;
  const int dyn1 = (kTP + kTR) * RS;
  cudaError_t e = cudaFuncSetAttribute(tiered_score_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, dyn1);
  if (e != cudaSuccess) return e;
  dim3 g1((a.max_pages + kTP - 1) / kTP, a.n_rg, a.B);
  e = launch_pdl(tiered_score_kernel, g1, dim3(kTScoreThreads), dyn1, stream, a);
  if (e != cudaSuccess) return e;
  const size_t dyn2 = (size_t)a.max_pages * (4 + 4 + 2 + 1) + 16;
  e = cudaFuncSetAttribute(tiered_choose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dyn2);
  if (e != cudaSuccess) return e;
  return launch_pdl(tiered_choose_kernel, dim3(a.B, kChooseCtas), dim3(kChooseThreads), dyn2,
                    stream, a);
}

}  // namespace sa
