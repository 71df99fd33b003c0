// Page scoring and top-k selection (GQA), in two launches.
//
// score_kernel (one CTA per 128 pages of one sequence and a block of kv heads,
// so every SM streams summaries) and choose_kernel (one CTA per (kv head,
// sequence)):
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
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "exact.cuh"
#include "internal.h"
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kThreads = 512;       // choose_kernel
constexpr int kSelGroups = 256;     // choose_kernel: group maxima behind the pruning threshold
constexpr int kCandCap = 1024;      // choose_kernel: candidates classified by counting (more:
                                    // order statistics of the bounds over every page)
static_assert(kSelGroups <= kThreads, "one thread clears each group maximum");
#ifndef SA_SCORE_CHUNK
#define SA_SCORE_CHUNK 128
#endif
constexpr int kScoreChunk = SA_SCORE_CHUNK;   // score_kernel: logical pages per CTA
constexpr int kScoreStages = 2;     // ring slots of 16 pages
constexpr int kScoreMaxHB = 8;      // kv heads per CTA (one consumer warp each)

// Shared-memory layout (dynamic): lo[Nmax] f32, hi[Nmax] f32, u_list[Nmax] u16,
// flag[Nmax] u8; q rows [R][Dk] f32 in static memory.
struct SelSmem {
  float* lo;
  float* hi;
  uint8_t* flag;   // 0 = not selected, 1 = selected (forced or winner), 2 = uncertain
  uint16_t* u_list;
};

// Sequence length clamped to what its page-table row can hold.
SA_DEV int clamped_len(const SelectArgs& a, int b, bool report) {
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
    if (report) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  return L;
}

// lo/hi bounds of every candidate page's score; NaN for forced pages.
//
// Data movement.  Summaries are stored [P_pool, Hkv, Dk], so the rows of
// adjacent kv heads of one page form one contiguous run.  A CTA scores a chunk
// of kScoreChunk logical pages of one sequence for a block of hb adjacent kv
// heads (hb <= 8, hb * Dk * 2 <= 2 KB): warp hb (the producer) looks the pages
// up in the page table and gathers each page's hb-head run with one bulk copy
// into a ring of kScoreStages slots of 16 pages; warps 0 .. hb-1 (one per kv
// head) score the slots.  Gathering whole runs instead of single 256-byte rows
// matters: scattered 256-byte reads reach a fraction of HBM bandwidth.
//
// Arithmetic.  A slot's scores for one head are a (16 pages x Dk) by (Dk x R
// rows) product, done with m16n8k16 bf16 warp MMAs (float32 accumulation),
// which keeps the instruction count per page far below a float32 FMA loop.
// Three products per tile:
//   S = sigma q^T             the scores,
//   T = |sigma| |q|^T          an upper bound of sum_d |q_d sigma_d| per row,
//   U = |sigma| f^T            f_d = 2^-126 where q_d is subnormal, else 0
//                              (only when the head's rows hold a subnormal).
// Every bf16 x bf16 product is exact in float32.  The score bracket of row r is
//   s_r -/+ E_r,  E_r = c_acc T_r + (1 + 2^-10) U_r + 2^-126 ||q_r||_1 + Dk 2^-124
// with directed rounding.  c_acc T_r covers the rounding of the float32
// accumulation (c_acc = Dk 2^-20: the accumulation of each 16-term step loses
// less than 2^-17.9 of the running magnitude sum even if every addend were
// truncated at the largest exponent, a margin of about 3.5x); U_r covers
// subnormal q_d flushed to zero inside the MMA, 2^-126
// ||q_r||_1 the same for sigma_d, and Dk 2^-124 any product that underflows
// float32.  A page's bracket is [max_r (s_r - E_r), max_r (s_r + E_r)].
template <int NT, int DK>   // 8-row tiles of query rows (R <= 8 NT); feature count
__global__ void __launch_bounds__((kScoreMaxHB + 1) * 32) score_kernel(const SelectArgs a, int hb) {
  pdl_wait_and_release();
  constexpr int KS = DK / 16;                      // k-steps
  constexpr int ROWB = DK * 2;                     // bytes per summary row
  constexpr int QS = ROWB + 16;                    // padded query-row stride
  constexpr int QROWS = 8 * NT;
  const int rec = hb * ROWB;                       // bytes per page run
  const int RSB = rec + 16;                        // padded slot-row stride
  extern __shared__ __align__(128) uint8_t score_smem[];
  uint8_t* q_s = score_smem;                                 // [hb][QROWS][QS]
  uint8_t* ring = score_smem + hb * QROWS * QS;              // [stages][16][RSB]
  __shared__ uint64_t full[kScoreStages], empty[kScoreStages];
  __shared__ int8_t stat_s[kScoreStages][16];   // per slot page: 1 scored, 0 forced, -1 bad
  __shared__ float qn1_s[kScoreMaxHB][QROWS];
  __shared__ int sub_s[kScoreMaxHB];
  const int chunk = blockIdx.x, hblk = blockIdx.y, b = blockIdx.z;
  const int L = clamped_len(a, b, false);
  const int N = (L + a.P - 1) / a.P;
  if (N <= a.budget_pages || a.k_top == 0) return;   // no ranking needed
  const int p0 = chunk * kScoreChunk;
  if (p0 >= N) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.Hq / a.Hkv, R = a.T * G, h0 = hblk * hb;
  const int n_groups = (min(kScoreChunk, N - p0) + 15) / 16;
  const int n_sink = min(a.n_sink, N), local0 = max(N - a.n_local, 0);
  if (tid == 0) {
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], hb);
    }
    fence_mbar_init();
  }
  __syncthreads();   // barriers initialised: the producer starts at once

  if (warp < hb) {
    // consumers: the query rows of the block's heads (zero past R) into shared
    // memory, then per head ||q_r||_1 (rounded up) and whether an element is
    // subnormal, while the producer's first gathers are in flight
    // (every thread's loads are issued before any is stored: one round trip)
    constexpr int kPer = QROWS * (ROWB / 16) / 32;   // pieces per consumer thread
    uint4 v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * hb * 32;
      const int r = (i / (ROWB / 16)) % QROWS, w = i / (QROWS * (ROWB / 16));
      v[j] = make_uint4(0, 0, 0, 0);
      if (r < R) {
        const int t = r / G, h = (h0 + w) * G + r % G;
        v[j] = *reinterpret_cast<const uint4*>(a.q + b * a.qs0 + t * a.qs1 + h * a.qs2 +
                                               (i % (ROWB / 16)) * 8);
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * hb * 32;
      const int r = (i / (ROWB / 16)) % QROWS, w = i / (QROWS * (ROWB / 16));
      *reinterpret_cast<uint4*>(q_s + (w * QROWS + r) * QS + (i % (ROWB / 16)) * 16) = v[j];
    }
    asm volatile("bar.sync 1, %0;" ::"r"(hb * 32) : "memory");
    // LPR lanes per query row, each over DK / LPR features in 16-byte pieces
    constexpr int LPR = 32 / QROWS;
    const int r = lane / LPR, part = lane % LPR;
    float s1 = 0.f;
    int sub = 0;
#pragma unroll
    for (int c = 0; c < DK / 8 / LPR; ++c) {
      const uint4 x4 = *reinterpret_cast<const uint4*>(q_s + (warp * QROWS + r) * QS +
                                                      (c * LPR + part) * 16);
      const uint32_t w4[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s1 += fabsf(__uint_as_float(w4[e] << 16)) + fabsf(__uint_as_float(w4[e] & 0xffff0000u));
        sub |= ((w4[e] & 0x7f80u) == 0 && (w4[e] & 0x7fu) != 0) |
               ((w4[e] & 0x7f800000u) == 0 && (w4[e] & 0x7f0000u) != 0);
      }
    }
#pragma unroll
    for (int o = LPR / 2; o; o >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    if (part == 0) qn1_s[warp][r] = s1 * (1.f + DK * 1.2e-7f);
    sub = __any_sync(0xffffffffu, sub);
    if (lane == 0) sub_s[warp] = sub;
    __syncwarp();
  }

  if (warp == hb) {
    // ================= producer: page-table lookups and bulk gathers
    int ph_r[kScoreChunk / 32];
#pragma unroll
    for (int i = 0; i < kScoreChunk / 32; ++i) {
      const int p = p0 + 32 * i + lane;
      ph_r[i] = (p < N && p >= n_sink && p < local0) ? page_at(a.pt, b, p) : -1;
    }
    for (int g = 0; g < n_groups; ++g) {
      const int st = g % kScoreStages;
      if (g >= kScoreStages &&
          !mbar_wait_bounded(&empty[st], ((g / kScoreStages) - 1) & 1)) {
        if (lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
        break;
      }
      int phx = -1;
#pragma unroll
      for (int i = 0; i < kScoreChunk / 32; ++i)
        if (i == (g >> 1)) phx = ph_r[i];
      const int j = lane & 15;                       // page of the slot
      const int p = p0 + 16 * g + j;
      const int ph = __shfl_sync(0xffffffffu, phx, 16 * (g & 1) + j);
      const bool cand = p < N && p >= n_sink && p < local0;
      const bool ok = cand && ph >= 0 && ph < a.P_pool;
      const int st8 = ok ? 1 : (cand ? -1 : 0);
      const uint32_t m = __ballot_sync(0xffffffffu, ok && lane < 16);
      if (lane < 16) stat_s[st][j] = static_cast<int8_t>(st8);
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[st], __popc(m) * rec);
      __syncwarp();
      if (lane < 16 && ok)
        bulk_load(ring + (st * 16 + j) * RSB, a.sig + ((int64_t)ph * a.Hkv + h0) * DK, rec,
                  &full[st]);
    }
  } else if (warp < hb) {
    // ================= consumers: one kv head each
    const int kvh = h0 + warp;
    const bool sub = sub_s[warp] != 0;
    constexpr float c_acc = DK * 9.5367431640625e-07f;   // Dk * 2^-20
    constexpr float e_abs = DK * 4.70197740328915e-38f;  // Dk * 2^-124
    float2* outrow = a.lohi + ((int64_t)b * a.Hkv + kvh) * a.max_pages;
    const int gq = lane >> 2, cq = lane & 3;           // fragment row / column pair
    float fl[NT][2];                                   // per fragment column: 2^-126 ||q_r||_1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) fl[nt][i] = qn1_s[warp][nt * 8 + 2 * cq + i] * 1.1754943508222875e-38f;
    // ldmatrix addresses: A rows = slot pages (lane & 15), k + 8 (lane >> 4);
    // B rows = query rows (lane & 7), k + 8 ((lane >> 3) & 1)
    const uint32_t a_off = (lane & 15) * RSB + warp * ROWB + 16 * (lane >> 4);
    const uint32_t b_base = smem_u32(q_s + (warp * QROWS + (lane & 7)) * QS + 16 * ((lane >> 3) & 1));
    const uint32_t ring_u = smem_u32(ring);
    for (int g = 0; g < n_groups; ++g) {
      const int st = g % kScoreStages;
      if (!mbar_wait_bounded(&full[st], (g / kScoreStages) & 1)) {
        if (lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
        break;
      }
      float acc[3][NT][4];
#pragma unroll
      for (int x = 0; x < 3; ++x)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[x][nt][i] = 0.f;
      const uint32_t a_addr = ring_u + st * 16 * RSB + a_off;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t af[4], aa[4];
        ldmatrix_x4(af, a_addr + ks * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) aa[i] = af[i] & 0x7fff7fffu;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t bq[2];
          ldmatrix_x2(bq, b_base + nt * 8 * QS + ks * 32);
          mma_bf16_16816(acc[0][nt], af, bq[0], bq[1]);
          mma_bf16_16816(acc[1][nt], aa, bq[0] & 0x7fff7fffu, bq[1] & 0x7fff7fffu);
          if (sub) {
            uint32_t bf[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint32_t x = bq[i];
              const bool s0 = (x & 0x7f80u) == 0 && (x & 0x7fu) != 0;
              const bool s1 = (x & 0x7f800000u) == 0 && (x & 0x7f0000u) != 0;
              bf[i] = (s0 ? 0x0080u : 0u) | (s1 ? 0x00800000u : 0u);
            }
            mma_bf16_16816(acc[2][nt], aa, bf[0], bf[1]);
          }
        }
      }
      // epilogue: this lane holds pages gq (i = 0, 1) and gq + 8 (i = 2, 3),
      // query rows 8 nt + 2 cq + (i & 1)
      float lo[2] = {-INFINITY, -INFINITY}, hi[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = nt * 8 + 2 * cq + (i & 1);
          if (r < R) {
            const float E = __fadd_ru(__fadd_ru(__fmul_ru(c_acc, acc[1][nt][i]),
                                                __fmul_ru(1.0009765625f, acc[2][nt][i])),
                                      __fadd_ru(fl[nt][i & 1], e_abs));
            const float sv = acc[0][nt][i];
            lo[i >> 1] = fmaxf(lo[i >> 1], __fsub_rd(sv, E));
            hi[i >> 1] = fmaxf(hi[i >> 1], __fadd_ru(sv, E));
          }
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          lo[h] = fmaxf(lo[h], __shfl_xor_sync(0xffffffffu, lo[h], o));
          hi[h] = fmaxf(hi[h], __shfl_xor_sync(0xffffffffu, hi[h], o));
        }
        const int j = gq + 8 * h;
        const int p = p0 + 16 * g + j;
        if (cq == 0 && p < N) {
          const int stv = stat_s[st][j];
          float2 out;
          if (stv == 0) {
            out = make_float2(NAN, NAN);
          } else if (stv < 0) {
            set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
            out = make_float2(-INFINITY, -INFINITY);   // an unreadable page never wins a slot
          } else {
            // + 0 turns -0 into +0 (the radix keys order -0 below +0)
            out = make_float2(lo[h] + 0.f, hi[h] + 0.f);
          }
          outrow[p] = out;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
  }
}

// Classification of the candidate pages (neither sink nor local) for the k
// slots, from the bracket [lo, hi] of each page's score (rigorous: the exact
// score lies in it), ties to the lower logical page:
//   certainly selected  iff  #{q : hi_q >= lo_p} <= k   (p included)
//   undecided           iff  not certain and #{q : lo_q > hi_p} < k
//   out                 otherwise.
// The counts only need the pages with hi >= tau, where tau is the k-th largest
// of the largest lower ends of G disjoint groups of pages (k <= G): k pages have
// lo >= tau, so a page with hi < tau is out, adds nothing to #{lo_q > hi_p} for
// a kept page p, and adds nothing to #{hi_q >= lo_p} when lo_p >= tau; a page
// with lo_p < tau has at least k + 1 upper ends at or above lo_p and is never
// certain.  With more than kCandCap kept pages the same classification is
// made from the order statistics of the bounds (lo_p > the (k+1)-th largest hi;
// hi_p >= the k-th largest lo) over every page.  The undecided pages are then
// rescored exactly and ranked, and the output is the sink pages, the selected
// pages and the local pages, ascending.
__global__ void __launch_bounds__(kThreads, 2) choose_kernel(const SelectArgs a) {
  pdl_wait_and_release();
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = clamped_len(a, b, tid == 0);
  const int N = (L + a.P - 1) / a.P;
  int32_t* outp = a.out_pages + ((int64_t)b * a.Hkv + kvh) * a.budget_pages;
  int32_t* outc = a.out_counts + (int64_t)b * a.Hkv + kvh;

  if (N <= a.budget_pages) {  // every page is selected
    for (int i = tid; i < a.budget_pages; i += blockDim.x) outp[i] = i < N ? i : -1;
    if (tid == 0) *outc = N;
    return;
  }

  extern __shared__ __align__(16) uint8_t dsm[];
  // the kept pages' bounds and pages (counting path) or the order-statistics
  // scratch (the other path): never both, so they share storage -- which lets
  // two CTAs share an SM at 8192 pages
  union ChooseScratch {
    struct {
      float2 lohi[kCandCap];
      uint16_t pg[kCandCap];
    } kept;
    struct {
      uint32_t hist[1024];
      uint32_t sel_out[8];
      SelScratch sel;
    } stats;
  };
  __shared__ __align__(16) ChooseScratch cs;
  __shared__ int red_i[kThreads / 32];
  __shared__ int n_unc, n_certain;
  __shared__ double ex_tmp[kThreads];
  __shared__ __align__(16) uint32_t gmax[kSelGroups];   // order keys of the groups' largest lo
  __shared__ uint32_t tau_key;
  float2* c_lohi = cs.kept.lohi;                        // the kept pages' bounds, ascending
  uint16_t* c_pg = cs.kept.pg;

  SelSmem S;
  S.lo = reinterpret_cast<float*>(dsm);
  S.hi = S.lo + a.max_pages;
  S.u_list = reinterpret_cast<uint16_t*>(S.hi + a.max_pages);
  S.flag = reinterpret_cast<uint8_t*>(S.u_list + a.max_pages);

  const int G = a.Hq / a.Hkv, R = a.T * G, Dk = a.Dk;
  const int n_sink = min(a.n_sink, N), local0 = max(N - a.n_local, 0);
  const int k = a.k_top;
  const int M = local0 - n_sink;              // candidate pages (more than k here)
  const int Gs = min(kSelGroups, M);          // groups (p - n_sink) Gs / M: none empty
  const bool prune = k > 0 && k <= Gs;
  const float2* lohi = a.lohi + ((int64_t)b * a.Hkv + kvh) * a.max_pages;
  if (tid == 0) {
    n_unc = 0;
    n_certain = 0;
    tau_key = 0u;
  }
  if (tid < kSelGroups) gmax[tid] = 0u;        // below every non-NaN key
  __syncthreads();
  // (loads in batches of 8 per thread, all in flight together)
  for (int p0 = 0; p0 < N; p0 += 8 * kThreads) {
    float2 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int p = p0 + tid + j * kThreads;
      const bool cand = p < N && p >= n_sink && p < local0;
      v[j] = cand && k > 0 ? lohi[p] : make_float2(NAN, NAN);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int p = p0 + tid + j * kThreads;
      if (p < N) {
        S.flag[p] = (p >= n_sink && p < local0) ? 0 : 1;
        S.lo[p] = v[j].x;
        S.hi[p] = v[j].y;
        if (prune && p >= n_sink && p < local0 && !isnan(v[j].x))
          atomicMax(&gmax[(p - n_sink) * Gs / M], f2key(v[j].x));
      }
    }
  }
  __syncthreads();
  float tau = -INFINITY;
  if (prune) {   // the largest group maximum with at least k group maxima at or above it
    if (tid < Gs) {   // (groups Gs.. hold 0, below every key: never counted)
      const uint32_t mine = gmax[tid];
      const uint4* g4 = reinterpret_cast<const uint4*>(gmax);
      int c = 0;
#pragma unroll 8
      for (int j = 0; j < kSelGroups / 4; ++j) {
        const uint4 w = g4[j];
        c += (w.x >= mine) + (w.y >= mine) + (w.z >= mine) + (w.w >= mine);
      }
      if (c >= k) atomicMax(&tau_key, mine);
    }
    __syncthreads();
    tau = key2f(tau_key);
  }
  // the kept candidate pages (hi >= tau), ascending: thread t scans [t ppt, (t + 1) ppt)
  int nc = 0;
  if (k > 0) {
    const int ppt = (N + blockDim.x - 1) / blockDim.x;
    const int q0 = tid * ppt, q1 = min(N, q0 + ppt);
    int cnt = 0;
    for (int p = q0; p < q1; ++p) cnt += S.flag[p] == 0 && S.hi[p] >= tau;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int w = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += w;
    }
    if (lane == 31) red_i[warp] = incl;
    __syncthreads();
    int pos = incl - cnt;
    for (int i = 0; i < kThreads / 32; ++i) {
      if (i < warp) pos += red_i[i];
      nc += red_i[i];
    }
    if (nc <= kCandCap)
      for (int p = q0; p < q1; ++p)
        if (S.flag[p] == 0 && S.hi[p] >= tau) {
          c_pg[pos] = static_cast<uint16_t>(p);
          c_lohi[pos++] = make_float2(S.lo[p], S.hi[p]);
        }
    __syncthreads();
  }
  const bool counted = k > 0 && nc <= kCandCap;
  if (counted) {
    // one thread per kept page; every lane reads the same bound (a broadcast)
    for (int i = tid; i < nc; i += blockDim.x) {
      const float2 me = c_lohi[i];
      int n_hi = 0, n_lo = 0;   // #{hi_q >= lo_p}, #{lo_q > hi_p}
#pragma unroll 4
      for (int j = 0; j < nc; ++j) {
        const float2 o = c_lohi[j];
        n_hi += o.y >= me.x;
        n_lo += o.x > me.y;
      }
      const int p = c_pg[i];
      if (me.x >= tau && n_hi <= k) {
        S.flag[p] = 1;
        atomicAdd(&n_certain, 1);
      } else if (n_lo < k) {
        S.flag[p] = 2;
        S.u_list[atomicAdd(&n_unc, 1)] = static_cast<uint16_t>(p);
      }
    }
  } else if (k > 0) {
    // ---- order statistics of the bounds, then: certainly in (lo > H),
    // undecided (hi >= Lk), else out
    float Lk = INFINITY, H = INFINITY;
    if (!filtered_select2(S.lo, S.hi, N, k, k + 1, &cs.stats.sel, Lk, H))
      radix_select2(S.lo, S.hi, N, k, k + 1, cs.stats.hist, cs.stats.sel_out, Lk, H);
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
  }
  __syncthreads();

  const int nu_ = n_unc;
  const int slots = k - n_certain;

  // ---- exact scores of the undecided pages (lo/hi storage reused as doubles)
  double* ex = reinterpret_cast<double*>(S.lo);
  if (nu_ > 0 && slots > 0) {
    // one warp per (page, query row): exact dot, then the max over the rows
    const int nw = kThreads / 32;
    const int per = max(1, kThreads / R);            // undecided pages per round
    for (int u0 = 0; u0 < nu_; u0 += per) {
      const int np = min(per, nu_ - u0);
      for (int pr = warp; pr < np * R; pr += nw) {
        const int r = pr % R;
        const int ph = page_at(a.pt, b, S.u_list[u0 + pr / R]);
        double e = -INFINITY;
        if (ph >= 0 && ph < a.P_pool) {
          const int t = r / G, h = kvh * G + r % G;
          e = warp_exact_dot_bf16<1>(a.q + b * a.qs0 + t * a.qs1 + h * a.qs2,
                                  a.sig + ((int64_t)ph * a.Hkv + kvh) * Dk, Dk);
        }
        if (lane == 0) ex_tmp[pr] = e;
      }
      __syncthreads();
      if (tid < np) {
        double m = -INFINITY;
        for (int rr = 0; rr < R; ++rr) m = fmax(m, ex_tmp[tid * R + rr]);
        ex[u0 + tid] = m;
      }
      __syncthreads();
    }
    // rank among the undecided pages: (exact desc, logical asc)
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

  if (counted) {
    // ---- sink pages, the selected kept pages (ascending), local pages
    if (warp == 0) {
      for (int i = lane; i < n_sink; i += 32) outp[i] = i;
      int pos = n_sink;
      for (int j0 = 0; j0 < nc; j0 += 32) {
        const int j = j0 + lane;
        const bool sel = j < nc && S.flag[c_pg[j]] == 1;
        const uint32_t m = __ballot_sync(0xffffffffu, sel);
        const int q = pos + __popc(m & ((1u << lane) - 1u));
        if (sel && q < a.budget_pages) outp[q] = c_pg[j];
        pos += __popc(m);
      }
      const int n_loc = N - local0;
      for (int i = lane; i < n_loc; i += 32)
        if (pos + i < a.budget_pages) outp[pos + i] = local0 + i;
      const int total = pos + n_loc;
      for (int i = total + lane; i < a.budget_pages; i += 32) outp[i] = -1;
      if (lane == 0) *outc = min(total, a.budget_pages);
    }
    return;
  }
  // ---- ascending compaction of the selected pages
  const int per_t = (N + blockDim.x - 1) / blockDim.x;
  const int p0 = tid * per_t, p1 = min(N, p0 + per_t);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += S.flag[p] == 1;
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) red_i[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int i = 0; i < (int)(blockDim.x / 32); ++i) {
    if (i < warp) wbase += red_i[i];
    total += red_i[i];
  }
  int pos = wbase + incl - cnt;
  for (int p = p0; p < p1; ++p)
    if (S.flag[p] == 1 && pos < a.budget_pages) outp[pos++] = p;
  for (int i = total + tid; i < a.budget_pages; i += blockDim.x) outp[i] = -1;
  if (tid == 0) *outc = min(total, a.budget_pages);
}

}  // namespace

size_t select_workspace_bytes(int B, int Hkv, int max_pages) {
  return (size_t)B * Hkv * max_pages * sizeof(float2);
}

cudaError_t launch_select_gqa(const SelectArgs& a, cudaStream_t stream) {
  // (an empty page table holds no candidate: the choose pass alone writes the
  // empty selections, without reading any score bound)
  if (a.k_top > 0 && a.max_pages > 0) {
    // kv-head block: the largest divisor of Hkv with hb <= 8 and an hb-head
    // run of at most 2 KB
    int hb = 1;
    for (int d = 1; d <= kScoreMaxHB && d <= a.Hkv; ++d)
      if (a.Hkv % d == 0 && d * a.Dk * 2 <= 2048) hb = d;
    dim3 g1((a.max_pages + kScoreChunk - 1) / kScoreChunk, a.Hkv / hb, a.B);
    const int R = a.T * (a.Hq / a.Hkv);
    auto pick = [&](auto dk) {
      constexpr int DK = decltype(dk)::value;
      auto launch = [&](auto kern, int nt) {
        const int dyn = hb * 8 * nt * (DK * 2 + 16) + kScoreStages * 16 * (hb * DK * 2 + 16);
        cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(kern));
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, g1, dim3((hb + 1) * 32), dyn, stream, a, hb);
      };
      return R <= 8 ? launch(score_kernel<1, DK>, 1) : launch(score_kernel<2, DK>, 2);
    };
    const cudaError_t e = a.Dk == 64    ? pick(std::integral_constant<int, 64>{})
                          : a.Dk == 128 ? pick(std::integral_constant<int, 128>{})
                                        : pick(std::integral_constant<int, 256>{});
    if (e != cudaSuccess) return e;
  }
  const size_t dyn = (size_t)a.max_pages * (4 + 4 + 2 + 1) + 16;
  cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(choose_kernel));
  // the largest shared-memory carveout: two CTAs per SM up to 8192 pages
  if (e == cudaSuccess) e = prefer_max_carveout(reinterpret_cast<const void*>(choose_kernel));
  if (e != cudaSuccess) return e;
  return launch_pdl(choose_kernel, dim3(a.Hkv, a.B), dim3(kThreads), dyn, stream, a);
}


// ---------------------------------------------------------------------------
// Selection without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they select
// pages: code running inside a CUDA-graph capture region, a serving loop
// whose memory pool is sealed after warm-up, or a host framework that owns
// every allocation and hands this library raw pointers only.  For them the
// score bounds live in a fixed-size array in the library's own device memory,
// reserved when the library is loaded (on every GPU that loads it, until the
// process exits).
constexpr size_t kStaticScoreEntries = size_t(1) << 21;   // 2,097,152 pages x 8 bytes = 16 MiB
static __device__ __align__(256) float2 g_static_score_bounds[kStaticScoreEntries];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
// Per device: the array's address in the context it was looked up in.  A
// module's device globals live as long as the context that loaded it, so the
// address is keyed by the context's unique id: after the primary context is
// torn down and created again (cudaDeviceReset, say) the array may sit
// elsewhere, and the next call looks it up afresh.
struct StaticSlot {
  unsigned long long ctx_id;
  float2* ptr;
};
StaticSlot g_static_slot[kMaxDevices] = {};

// Device address of the static array in the current device's context, looked
// up (cudaGetSymbolAddress) on the first call in that context: the host-side
// symbol is only a stand-in and must never reach a kernel.
cudaError_t static_scores_ptr(float2** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // the lookup below also makes the runtime create the context if needed, so
  // read the id after it when there is none yet
  unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticSlot& s = g_static_slot[dev];
  if (!s.ptr || id == 0 || s.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_score_bounds);
    if (e != cudaSuccess) return e;
    s.ptr = static_cast<float2*>(p);
    s.ctx_id = id ? id : current_context_id();
  }
  *out = s.ptr;
  return cudaSuccess;
}
}  // namespace

size_t select_static_capacity() { return kStaticScoreEntries; }

cudaError_t launch_select_gqa_static(SelectArgs a, cudaStream_t stream) {
  float2* p = nullptr;
  cudaError_t e = static_scores_ptr(&p);
  if (e != cudaSuccess) return e;
  a.lohi = p;
  return launch_select_gqa(a, stream);
}

}  // namespace sa
