// Tiered page selection for one shared latent KV head (MLA + MTP).
//
// Every logical page of a sequence is a candidate; its score is the max over
// all T x Hq query rows of q . sigma (Dk = 576 in DeepSeek-shaped models: a
// 256 x 576 by 576 x N contraction per sequence).  The critical tier is the
// alpha best pages, the ambient tier the next beta, by (score desc, logical
// page asc).  The result is written as two decode lists per sequence: list 0
// = critical pages, list 1 = critical + ambient pages, both ascending.
//
// tiered_score_kernel: one CTA per (128 pages, 128 query rows, sequence) scores
// on the tensor cores (tcgen05) and emits, per page and row group, a rigorous
// bracket of the row-max score and the mask of rows that can attain it.
// tiered_choose_kernel: up to kChooseCtas CTAs per sequence each merge the row
// groups' brackets and select the order statistics for both boundaries
// (alpha, alpha+beta) in one pass; together they rescore the undecided pages
// exactly on their flagged rows only (fixed-point accumulation of the bf16
// products, one rounding to float64), and the last to finish writes both lists.
//
// Source: "TileSparse: Arithmetic-Intensity-Aware Sparse Attention for
// Compute-Bound LLM Decoding", "Motivation" (Critical Tier: alpha pages
// computed with all query heads; Ambient Tier: beta pages with h heads).
#include "common.cuh"
#include "exact.cuh"
#include "internal.h"
#include "tc05.cuh"
#include "topk.cuh"

#include <algorithm>

namespace sa {
namespace {

constexpr int kTR = 32;            // query rows per row group (one 32-bit row mask)
constexpr int kChooseThreads = 512;
constexpr int kChooseCtas = 16;    // at most this many CTAs per sequence share the exact rescoring

// Scores of 128 pages x 128 query rows of one sequence, S = sigma q^T, on the
// tensor cores: tcgen05.mma (M = 128 pages, N = 128 rows, K = 16 per
// instruction, bf16 in, float32 accumulation in tensor memory) over the Dk
// features in chunks of 64 (one 128-byte swizzle row).  Warps 0-7 gather the
// chunk's summary rows (through the page table) and query rows with 16-byte
// cp.async copies straight into the 128-byte-swizzled K-major layout of a
// kSStages-deep ring, and sum each row's squares from their own copies (packed
// float32 pairs); warp 8 allocates the tensor memory and issues the MMAs;
// warps 0-7 then read the accumulator, one page (TMEM lane) and half of the
// rows per thread.  Per (page, row) the exact score lies in s -/+ E with
// (directed rounding)
//   E = c_acc ||q_r|| ||sigma|| + 2^-126 sqrt(Dk) (||q_r|| + ||sigma||) + Dk 2^-124,
// c_acc = Dk 2^-20: the accumulation of each 16-product step loses less than
// 2^-17.9 of the running magnitude sum sum_d |q_d sigma_d| <= ||q|| ||sigma||
// even if every addend were truncated at the largest exponent (a margin of
// about 3.5x); the 2^-126 terms cover subnormal inputs flushed to zero inside
// the MMA (sum_d |x_d| <= sqrt(Dk) ||x||), Dk 2^-124 products that underflow
// float32.  The norms are float32 sums of squares, padded by (1 + gamma_Dk) and
// rounded up.  Emitted per page and row group of kTR rows: [max_r (s_r - E_r),
// max_r (s_r + E_r)] and the mask of the rows whose upper end reaches that
// largest lower end (only those rows can hold the page's maximum in the group).
constexpr int kSP = 128;                     // pages per CTA (MMA M, TMEM lanes)
constexpr int kSR = 128;                     // query rows per CTA (MMA N, TMEM columns)
constexpr int kSStages = 4;                  // K-chunk ring depth
constexpr int kSLag = kSStages - 1;          // chunks a loader keeps in flight
constexpr int kSChunk = 64;                  // features per K chunk
constexpr int kSTile = kSP * 128;            // bytes of one operand's chunk (16 KB)
constexpr int kSStageBytes = 2 * kSTile;     // summaries, then query rows
constexpr int kSLoaders = 8 * 32;            // warps 0-7: loads, norms, epilogue
constexpr int kSThreads = kSLoaders + 32;     // warp 8: MMA issue
constexpr uint32_t kSIdesc = tc::idesc_bf16_f32(kSP, kSR, false, false);
static_assert(kSR == 4 * kTR && kSP == 128, "epilogue: 4 TMEM lane quarters x 2 halves of 2 row groups");

// acc + (x0^2, x1^2) for the two bf16 of w, as packed float32 (x0 = low half).
SA_DEV unsigned long long fma2_sq(uint32_t w, unsigned long long acc) {
  const unsigned long long x =
      (static_cast<unsigned long long>(w & 0xffff0000u) << 32) | static_cast<unsigned long long>(w << 16);
  asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(x));
  return acc;
}

__global__ void __launch_bounds__(kSThreads, 1) tiered_score_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int pc = blockIdx.x, rt = blockIdx.y, b = blockIdx.z;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) L = L < 0 ? 0 : a.max_pages * a.P;
  const int N = (L + a.P - 1) / a.P;
  const int R = a.T * a.Hq;
  const int p0 = pc * kSP, r0 = rt * kSR;
  if (p0 >= N || r0 >= R) return;
  const int Dk = a.Dk, KC = (Dk + kSChunk - 1) / kSChunk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the choose kernel's exact-score slots and completion counter start at 0
  if (rt == 0 && tid < kSP && p0 + tid < N) a.exkey[(int64_t)b * a.max_pages + p0 + tid] = 0ull;
  if (pc == 0 && rt == 0 && tid == 0) a.counter[b] = 0u;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* ring = tsm_raw + ((1024 - (smem_u32(tsm_raw) & 1023)) & 1023);
  __shared__ uint64_t full[kSStages], empty[kSStages], mma_done;
  __shared__ uint32_t tmem_s;
  __shared__ float sn_s[kSP];                    // ||sigma_p||, rounded up
  __shared__ __align__(16) float cq_s[kSR];      // c_acc ||q_r||, rounded up
  __shared__ __align__(16) float fq_s[kSR];      // 2^-126 sqrt(Dk) ||q_r||, rounded up
  __shared__ int8_t pok_s[kSP];        // page readable
  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&full[s], kSLoaders);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 8) tc::tmem_alloc(&tmem_s, kSR);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_s;
  const uint32_t ring_u = smem_u32(ring);

  if (warp < 8) {
    // this thread: 16-byte unit j of every chunk, rows rb + 32 i (i < 4) of
    // both operands; in the swizzled layout row rr's unit j sits at
    // (rr / 8) * 1024 + (rr % 8) * 128 + ((j ^ (rr % 8)) * 16), and rr % 8 = rb % 8
    const int j = tid & 7, rb = tid >> 3;
    const uint32_t soff = (rb >> 3) * 1024 + (rb & 7) * 128 + ((j ^ (rb & 7)) << 4);
    const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
    const uint16_t* arow[4];
    const uint16_t* brow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = p0 + rb + 32 * i, r = r0 + rb + 32 * i;
      int ph = -1;
      if (p < N) {
        ph = ptrow[p];
        if (ph < 0 || ph >= a.P_pool) {
          if (j == 0) set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
          ph = -1;
        }
      }
      if (j == 0) pok_s[rb + 32 * i] = ph >= 0;
      arow[i] = ph >= 0 ? a.sig + (int64_t)ph * Dk : nullptr;
      brow[i] = r < R ? a.q + b * a.qs0 + (r / a.Hq) * a.qs1 + (r % a.Hq) * a.qs2 : nullptr;
    }
    // sums of squares as packed float32 pairs (even, odd features)
    unsigned long long sa2[4], sb2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sa2[i] = sb2[i] = 0ull;
    for (int kc = 0; kc < KC + kSLag; ++kc) {
      if (kc < KC) {
        const int s = kc % kSStages;
        if (kc >= kSStages && !mbar_wait_bounded(&empty[s], ((kc / kSStages) - 1) & 1))
          set_dev_error(a.err, SA_DEVERR_TIMEOUT);
        const int f0 = kc * kSChunk + 8 * j;      // Dk % 8 == 0: a unit is all in or all out
        const uint32_t da = ring_u + s * kSStageBytes + soff;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool va = arow[i] != nullptr && f0 < Dk, vb = brow[i] != nullptr && f0 < Dk;
          cp_async16(da + 4096 * i, va ? arow[i] + f0 : a.sig, va ? 16u : 0u);
          cp_async16(da + kSTile + 4096 * i, vb ? brow[i] + f0 : a.q, vb ? 16u : 0u);
        }
      }
      cp_async_commit();          // (empty groups past the end keep the count uniform)
      if (kc >= kSLag) {
        cp_async_wait<kSLag>();   // this thread's part of chunk kc - kSLag has landed
        const int s = (kc - kSLag) % kSStages;
        const uint8_t* src = ring + s * kSStageBytes + soff;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 x = *reinterpret_cast<const uint4*>(src + 4096 * i);
          const uint4 y = *reinterpret_cast<const uint4*>(src + kSTile + 4096 * i);
          const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sa2[i] = fma2_sq(xw[e], sa2[i]);
            sb2[i] = fma2_sq(yw[e], sb2[i]);
          }
        }
        tc::fence_proxy_async();   // the copies are read by the tensor core
        mbar_arrive(&full[s]);
      }
    }
    // row norms: the 8 lanes of a row group hold its 8 feature slices
    float na[4], nb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      na[i] = __uint_as_float(static_cast<uint32_t>(sa2[i])) +
              __uint_as_float(static_cast<uint32_t>(sa2[i] >> 32));
      nb[i] = __uint_as_float(static_cast<uint32_t>(sb2[i])) +
              __uint_as_float(static_cast<uint32_t>(sb2[i] >> 32));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        na[i] += __shfl_xor_sync(0xffffffffu, na[i], o);
        nb[i] += __shfl_xor_sync(0xffffffffu, nb[i], o);
      }
    }
    const float pad = 1.f + 2.f * Dk * 5.96046448e-8f;
    const float c_acc = Dk * 9.5367431640625e-07f;                                 // Dk 2^-20
    const float rt_d = __fmul_ru(__fsqrt_ru(static_cast<float>(Dk)), 1.1754943508222875e-38f);
    if (j == 0)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = rb + 32 * i;
        sn_s[rr] = __fmul_ru(__fsqrt_ru(__fmul_ru(na[i], pad)), 1.0000002f);
        const float qn = __fmul_ru(__fsqrt_ru(__fmul_ru(nb[i], pad)), 1.0000002f);
        cq_s[rr] = __fmul_ru(c_acc, qn);
        fq_s[rr] = __fmul_ru(rt_d, qn);
      }
    asm volatile("bar.sync 1, %0;" ::"n"(kSLoaders) : "memory");
    // epilogue: thread = page p0 + 32 (warp % 4) + lane = TMEM lane, row
    // groups 2 (warp / 4) and 2 (warp / 4) + 1
    if (!mbar_wait_bounded(&mma_done, 0)) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
    tc::fence_after_sync();
    const int pl = 32 * (warp & 3) + lane, p = p0 + pl;
    const bool pok = pok_s[pl] != 0;
    const float sn = sn_s[pl];
    const float es = __fadd_ru(__fmul_ru(rt_d, sn), Dk * 4.70197740328915e-38f);   // + Dk 2^-124
    for (int g = 2 * (warp >> 2); g < 2 * (warp >> 2) + 2 && r0 + g * kTR < R; ++g) {
      float sv[32];
      tc::ld32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + g * kTR, sv);
      tc::wait_ld();
      // (no branch per row: a conditional shared load per element would
      // serialise the loop; rows past R are masked by selects)
      const int nv = R - (r0 + g * kTR);   // valid rows of the group (>= 1)
      float lo = -INFINITY, hi = -INFINITY;
#pragma unroll
      for (int c4 = 0; c4 < 32; c4 += 4) {
        const float4 cq = *reinterpret_cast<const float4*>(cq_s + g * kTR + c4);
        const float4 fq = *reinterpret_cast<const float4*>(fq_s + g * kTR + c4);
        const float cqa[4] = {cq.x, cq.y, cq.z, cq.w}, fqa[4] = {fq.x, fq.y, fq.z, fq.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = c4 + e;
          const float E = __fadd_ru(__fmul_ru(cqa[e], sn), __fadd_ru(fqa[e], es));
          const float l = __fsub_rd(sv[c], E), h = __fadd_ru(sv[c], E);
          lo = fmaxf(lo, c < nv ? l : -INFINITY);
          sv[c] = c < nv ? h : -INFINITY;
          hi = fmaxf(hi, sv[c]);
        }
      }
      uint32_t m = 0;
#pragma unroll
      for (int c = 0; c < 32; ++c) m |= static_cast<uint32_t>(sv[c] >= lo) << c;
      if (p < N) {
        const int64_t at = ((int64_t)b * a.n_rg + r0 / kTR + g) * a.max_pages + p;
        // + 0 turns -0 into +0 (the radix keys order -0 below +0)
        a.lohi[at] = pok ? make_float2(lo + 0.f, hi + 0.f) : make_float2(-INFINITY, -INFINITY);
        a.rmask[at] = pok ? m : 0ull;
      }
    }
  } else if (lane == 0) {
    // ================= MMA issuer.  Descriptors advance by (byte offset >> 4).
    const uint64_t da0 = tc::sdesc_sw128(ring_u, 16, 1024);
    const uint64_t db0 = tc::sdesc_sw128(ring_u + kSTile, 16, 1024);
    for (int kc = 0; kc < KC; ++kc) {
      const int s = kc % kSStages;
      if (!mbar_wait_bounded(&full[s], (kc / kSStages) & 1)) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
      tc::fence_after_sync();
      const uint64_t off = static_cast<uint64_t>((s * kSStageBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kSChunk / 16; ++kk)
        tc::mma_bf16(tmem, da0 + off + kk * 2, db0 + off + kk * 2, kSIdesc, (kc | kk) ? 1u : 0u);
      tc::commit(&empty[s]);
    }
    tc::commit(&mma_done);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kSR);
  }
}

// Out of line: the exact dot needs many registers, and inlined it would raise
// the register count (and spills) of the whole choose kernel.
__device__ __noinline__ double exact_row_dot(const uint16_t* q, const uint16_t* sg, int n) {
  return warp_exact_dot_bf16<4>(q, sg, n);
}

// kChoosePairs bounds the (undecided page, row group) pairs whose rescoring
// tasks are flattened to (page, row) and spread evenly over every warp of the
// sequence's CTAs; beyond it each warp takes whole (page, row group) pairs.
constexpr int kChoosePairs = 1024;
// Boundaries up to kChooseGroups pages deep prune the pages by a threshold
// first (below); deeper ones classify every page.
constexpr int kChooseGroups = 256;
// Shared memory per page of the choose kernel: two brackets, two indices, a flag.
constexpr int kChooseBytesPerPage = 8 + 8 + 2 + 2 + 1;
static_assert(kChooseGroups <= kChooseThreads, "one thread clears each group maximum");

// Classification of a page p for a boundary of k pages (k < N), from the
// brackets [lo, hi] of every page's score (rigorous: the exact score lies in
// them), ties to the lower logical page:
//   certainly inside   iff  #{q : hi_q >= lo_p} <= k   (p included: even at
//                            lo_p it cannot be passed by k others)
//   undecided           iff  not inside and #{q : lo_q > hi_p} < k
//   certainly outside   otherwise (k pages are above it whatever the scores).
// Both counts only need the candidate pages, those with hi >= tau, where tau
// is the kmax-th largest of the largest lower ends of G disjoint groups of
// pages (kmax = the deepest boundary, kmax <= G): kmax pages have lo >= tau,
// so a page with hi < tau is outside every boundary, adds nothing to
// #{lo_q > hi_p} for a candidate p, and adds nothing to #{hi_q >= lo_p} when
// lo_p >= tau; a page with lo_p < tau has at least kmax + 1 upper ends at or
// above lo_p, so it is never inside.
__global__ void __launch_bounds__(kChooseThreads) tiered_choose_kernel(const TieredArgs a) {
  pdl_wait_and_release();
  const int b = blockIdx.x, cta = blockIdx.y, n_cta = gridDim.y, tid = threadIdx.x;
  const int nw = kChooseThreads / 32, warp = tid >> 5, lane = tid & 31;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
    if (tid == 0 && cta == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  const int N = (L + a.P - 1) / a.P;
  const int cap = a.alpha + a.beta;
  int32_t* out0 = a.lists + (int64_t)b * 2 * cap;
  int32_t* out1 = out0 + cap;
  // per page: the merged brackets (later (page, flags) of each undecided
  // page), the candidates' brackets (later the physical page of each undecided
  // page, then its exact score), the page of each candidate, the candidate of
  // each undecided page, the candidates' flags
  extern __shared__ __align__(16) uint8_t dsm[];
  float2* lohi = reinterpret_cast<float2*>(dsm);
  int* uf = reinterpret_cast<int*>(dsm);
  float2* c_lohi = reinterpret_cast<float2*>(dsm + 8 * (size_t)a.max_pages);
  int* ph_s = reinterpret_cast<int*>(c_lohi);
  double* ex = reinterpret_cast<double*>(c_lohi);
  uint16_t* c_pg = reinterpret_cast<uint16_t*>(dsm + 16 * (size_t)a.max_pages);
  uint16_t* u_list = c_pg + a.max_pages;
  uint8_t* c_fl = reinterpret_cast<uint8_t*>(u_list + a.max_pages);
  __shared__ __align__(16) uint32_t gmax[kChooseGroups];   // order keys of the groups' largest lower ends
  __shared__ uint32_t cmask[kChoosePairs];   // flagged rows of (candidate, row group), when they fit
  __shared__ uint32_t tau_key;
  __shared__ int pfx[kChoosePairs];          // exclusive prefix of the flagged rows per pair
  __shared__ uint32_t msk[kChoosePairs];     // flagged rows of (undecided page, row group)
  __shared__ int red_i[nw];
  __shared__ int n_cert[2];
  __shared__ int nu_s, last_s;
  const int kb[2] = {min(a.alpha, N), min(a.alpha + a.beta, N)};
  int kmax = 0;
  bool every = false;   // a boundary holds every page: no pruning
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (kb[i] > 0 && kb[i] >= N) every = true;
    if (kb[i] > 0 && kb[i] < N) kmax = max(kmax, kb[i]);
  }
  const int G = min(kChooseGroups, N);   // groups p G / N: none empty
  const bool prune = !every && kmax > 0 && kmax <= G;
  if (tid < kChooseGroups) gmax[tid] = 0u;   // below every non-NaN key
  if (tid == 0) {
    n_cert[0] = n_cert[1] = 0;
    tau_key = 0u;
  }
  __syncthreads();
  // the row groups' brackets of a thread's pages p and p + blockDim.x, 16 loads
  // in flight at a time (indices clamped: the loads are unconditional, and a
  // repeated row group or page does not change a max)
  for (int p = tid; p < N; p += 2 * blockDim.x) {
    const int p2 = p + blockDim.x, pc = min(p2, N - 1);
    float l[2] = {-INFINITY, -INFINITY}, h[2] = {-INFINITY, -INFINITY};
    for (int rg0 = 0; rg0 < a.n_rg; rg0 += 8) {
      float2 v[2][8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t row = ((int64_t)b * a.n_rg + min(rg0 + j, a.n_rg - 1)) * a.max_pages;
        v[0][j] = a.lohi[row + p];
        v[1][j] = a.lohi[row + pc];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          l[i] = fmaxf(l[i], v[i][j].x);
          h[i] = fmaxf(h[i], v[i][j].y);
        }
    }
    lohi[p] = make_float2(l[0], h[0]);
    if (prune) atomicMax(&gmax[p * G / N], f2key(l[0]));
    if (p2 < N) {
      lohi[p2] = make_float2(l[1], h[1]);
      if (prune) atomicMax(&gmax[p2 * G / N], f2key(l[1]));
    }
  }
  __syncthreads();
  float tau = -INFINITY;
  if (prune) {   // tau: the largest group maximum with at least kmax group maxima at or above it
    if (tid < G) {   // (groups G.. hold 0, below every key: never counted)
      const uint32_t mine = gmax[tid];
      const uint4* g4 = reinterpret_cast<const uint4*>(gmax);
      int c = 0;
#pragma unroll 8
      for (int j = 0; j < kChooseGroups / 4; ++j) {
        const uint4 v = g4[j];
        c += (v.x >= mine) + (v.y >= mine) + (v.z >= mine) + (v.w >= mine);
      }
      if (c >= kmax) atomicMax(&tau_key, mine);
    }
    __syncthreads();
    tau = key2f(tau_key);
  }
  // the candidates (hi >= tau), ascending: thread t scans pages [t ppt, (t + 1) ppt)
  int nc;
  {
    const int ppt = (N + blockDim.x - 1) / blockDim.x;
    const int q0 = tid * ppt, q1 = min(N, q0 + ppt);
    int cnt = 0;
    for (int p = q0; p < q1; ++p) cnt += lohi[p].y >= tau;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) red_i[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    nc = 0;
    for (int i = 0; i < nw; ++i) {
      if (i < warp) pos += red_i[i];
      nc += red_i[i];
    }
    for (int p = q0; p < q1; ++p) {
      const float2 v = lohi[p];
      if (v.y >= tau) {
        c_pg[pos] = static_cast<uint16_t>(p);
        c_lohi[pos++] = v;
      }
    }
    __syncthreads();
  }
  // classify the candidates by counting over the candidates, one thread each
  // (every lane reads the same bracket: a broadcast); meanwhile the candidate's
  // row masks are fetched for the exact rescoring, when they fit
  const bool cm = a.n_rg <= 8 && nc * a.n_rg <= kChoosePairs;
  for (int i = tid; i < nc; i += blockDim.x) {
    uint32_t rm[8];
    if (cm) {
#pragma unroll
      for (int g = 0; g < 8; ++g)
        rm[g] = static_cast<uint32_t>(
            a.rmask[((int64_t)b * a.n_rg + min(g, a.n_rg - 1)) * a.max_pages + c_pg[i]]);
    }
    const float2 me = c_lohi[i];
    int n_hi = 0, n_lo = 0;   // #{hi_q >= lo_p}, #{lo_q > hi_p}
#pragma unroll 4
    for (int j = 0; j < nc; ++j) {
      const float2 o = c_lohi[j];
      n_hi += o.y >= me.x;
      n_lo += o.x > me.y;
    }
    uint8_t f = 0;   // bits 1 / 2: inside boundary 0 / 1; 4 / 8: undecided for it
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (kb[k] >= N) {
        if (kb[k] > 0) f |= 1u << k;
      } else if (kb[k] > 0) {
        if (me.x >= tau && n_hi <= kb[k]) {
          f |= 1u << k;
          atomicAdd(&n_cert[k], 1);
        } else if (n_lo < kb[k]) {
          f |= 4u << k;
        }
      }
    }
    c_fl[i] = f;
    if (cm)
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < a.n_rg) cmask[i * a.n_rg + g] = rm[g];
  }
  __syncthreads();
  // the undecided candidates, ascending (one warp, ballots)
  if (warp == 0) {
    int nu = 0;
    for (int j0 = 0; j0 < nc; j0 += 32) {
      const int j = j0 + lane;
      const bool u = j < nc && (c_fl[j] & 12u);
      const uint32_t m = __ballot_sync(0xffffffffu, u);
      if (u) u_list[nu + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
      nu += __popc(m);
    }
    if (lane == 0) nu_s = nu;
  }
  __syncthreads();
  const int nu_ = nu_s;
  if (nu_ == 0 && cta != 0) return;             // nothing to share: CTA 0 writes
  if (nu_ > 0) {
    // exact row-max scores of the undecided pages: only the query rows the
    // scoring pass flagged for a page (per row group, the rows whose upper end
    // reaches the group's largest lower end) can hold its maximum.  One warp
    // rescores each such (page, row) exactly; the results are merged with an
    // atomic max in global memory and the last CTA to finish ranks.
    const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
    const int gw = cta + n_cta * warp, n_gw = n_cta * nw;   // this warp among the sequence's
    unsigned long long* exk = a.exkey + (int64_t)b * a.max_pages;
    const int npair = nu_ * a.n_rg;
    for (int i = tid; i < nu_; i += blockDim.x) {   // (the brackets are dead: ph_s aliases them)
      const int ph = ptrow[c_pg[u_list[i]]];
      ph_s[i] = (ph < 0 || ph >= a.P_pool) ? -1 : ph;
    }
    if (npair <= kChoosePairs) {
      // (page, row) tasks numbered through a block scan of the pairs' row counts
      const int per_t = (npair + blockDim.x - 1) / blockDim.x;
      const int x0 = tid * per_t, x1 = min(npair, x0 + per_t);
      int cnt = 0;
      for (int x = x0; x < x1; ++x) {
        const int uu = x / a.n_rg, g = x % a.n_rg;
        const uint32_t m =
            cm ? cmask[u_list[uu] * a.n_rg + g]
               : static_cast<uint32_t>(
                     a.rmask[((int64_t)b * a.n_rg + g) * a.max_pages + c_pg[u_list[uu]]]);
        msk[x] = m;
        cnt += __popc(m);
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) red_i[warp] = incl;
      __syncthreads();
      int run = incl - cnt, total = 0;
      for (int i = 0; i < nw; ++i) {
        if (i < warp) run += red_i[i];
        total += red_i[i];
      }
      for (int x = x0; x < x1; ++x) {
        pfx[x] = run;
        run += __popc(msk[x]);
      }
      __syncthreads();
      for (int t = gw; t < total; t += n_gw) {
        int l0 = 0, l1 = npair - 1;   // the last pair whose first task is <= t
        while (l0 < l1) {
          const int mid = (l0 + l1 + 1) >> 1;
          if (pfx[mid] <= t) l0 = mid;
          else l1 = mid - 1;
        }
        uint32_t bits = msk[l0];
        for (int j = t - pfx[l0]; j > 0; --j) bits &= bits - 1;
        const int uu = l0 / a.n_rg, r = (l0 % a.n_rg) * kTR + __ffs(bits) - 1;
        const int ph = ph_s[uu];
        if (ph < 0) continue;
        const int tt = r / a.Hq, h = r % a.Hq;
        const double e = exact_row_dot(a.q + b * a.qs0 + tt * a.qs1 + h * a.qs2,
                                       a.sig + (int64_t)ph * a.Dk, a.Dk);
        if (lane == 0) atomicMax(&exk[uu], d2key(e));
      }
    } else {
      __syncthreads();
      for (int x = gw; x < npair; x += n_gw) {
        const int uu = x / a.n_rg, g = x % a.n_rg;
        const int ph = ph_s[uu];
        if (ph < 0) continue;
        unsigned long long bits =
            a.rmask[((int64_t)b * a.n_rg + g) * a.max_pages + c_pg[u_list[uu]]];
        const uint16_t* sg = a.sig + (int64_t)ph * a.Dk;
        while (bits) {
          const int r = g * kTR + __ffsll(static_cast<long long>(bits)) - 1;
          bits &= bits - 1;
          const int tt = r / a.Hq, h = r % a.Hq;
          const double e = exact_row_dot(a.q + b * a.qs0 + tt * a.qs1 + h * a.qs2, sg, a.Dk);
          if (lane == 0) atomicMax(&exk[uu], d2key(e));
        }
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = atomicAdd(&a.counter[b], 1u) == static_cast<unsigned>(n_cta - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    // (no exact result: an unreadable page, scored -inf; ex now aliases ph_s)
    for (int i = tid; i < nu_; i += blockDim.x) {
      const unsigned long long k = __ldcg(&exk[i]);
      ex[i] = k == 0ull ? -INFINITY : key2d(k);
      const int ci = u_list[i];
      uf[i] = c_pg[ci] | (c_fl[ci] << 16);
    }
    __syncthreads();
    // per boundary: the undecided pages fill the slots the certain ones left
    for (int u = tid; u < nu_; u += blockDim.x) {
      const int cu = u_list[u], pu = c_pg[cu];
      const uint8_t fu = c_fl[cu];
      const double su = ex[u];
      int rank[2] = {0, 0};
      for (int v = 0; v < nu_; ++v) {
        const int pf = uf[v], pv = pf & 0xffff, fv = pf >> 16;
        const double sv = ex[v];
        const int ahead = (sv > su) || (sv == su && pv < pu);
        rank[0] += ahead & (fv >> 2);
        rank[1] += ahead & (fv >> 3);
      }
      uint8_t add = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (((fu >> (2 + i)) & 1u) && rank[i] < kb[i] - n_cert[i]) add |= 1u << i;
      if (add) c_fl[cu] = fu | add;
    }
    __syncthreads();
  }
  // both lists: the candidates inside each boundary, ascending, -1 padded
  if (warp == 0) {
    int c[2] = {0, 0};
    for (int j0 = 0; j0 < nc; j0 += 32) {
      const int j = j0 + lane;
      const uint8_t f = j < nc ? c_fl[j] : 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const bool in = (f >> k) & 1u;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        const int pos = c[k] + __popc(m & ((1u << lane) - 1u));
        if (in && pos < cap) (k ? out1 : out0)[pos] = c_pg[j];
        c[k] += __popc(m);
      }
    }
    const int c0 = min(c[0], cap), c1 = min(c[1], cap);
    for (int i = c0 + lane; i < cap; i += 32) out0[i] = -1;
    for (int i = c1 + lane; i < cap; i += 32) out1[i] = -1;
    if (lane == 0) {
      a.counts[2 * b] = c0;
      a.counts[2 * b + 1] = c1;
    }
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
  const int dyn1 = kSStages * kSStageBytes + 1024;   // + alignment slack
  cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(tiered_score_kernel));
  if (e != cudaSuccess) return e;
  dim3 g1((a.max_pages + kSP - 1) / kSP, (a.T * a.Hq + kSR - 1) / kSR, a.B);
  e = launch_pdl(tiered_score_kernel, g1, dim3(kSThreads), dyn1, stream, a);
  if (e != cudaSuccess) return e;
  const size_t dyn2 = (size_t)a.max_pages * kChooseBytesPerPage + 16;
  e = allow_max_dyn_smem(reinterpret_cast<const void*>(tiered_choose_kernel));
  if (e != cudaSuccess) return e;
  // enough CTAs per sequence to spread the exact rescoring over the SMs
  int sms = 0;
  e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const int n_cta = std::max(1, std::min(kChooseCtas, sms / std::max(1, a.B)));
  return launch_pdl(tiered_choose_kernel, dim3(a.B, n_cta), dim3(kChooseThreads), dyn2, stream, a);
}

}  // namespace sa
