// Page scoring and top-k selection (GQA), in two launches.
//
// score_kernel (one CTA per 256 pages of one (kv head, sequence), so every SM
// streams summaries) and choose_kernel (one CTA per (kv head, sequence)):
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
constexpr int kScoreThreads = 128;  // score_kernel: 4 warps x 32 pages
constexpr int kScorePages = 128;
constexpr int kMaxRows = 16;
constexpr int kMaxDk = 256;

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

// The group's query rows (t, h) as exact float32 copies in q_s[R][Dk]; returns
// an upper bound on max_r ||q_r||_2.  Called by every thread of the block.
SA_DEV float load_q_rows(const SelectArgs& a, int b, int kvh, float* q_s, float* red) {
  const int G = a.Hq / a.Hkv, R = a.T * G, Dk = a.Dk;
  for (int i = threadIdx.x; i < R * Dk; i += blockDim.x) {
    const int r = i / Dk, d = i % Dk;
    const int t = r / G, h = kvh * G + r % G;
    q_s[i] = bf16_bits_to_float(a.q[b * a.qs0 + t * a.qs1 + h * a.qs2 + d]);
  }
  __syncthreads();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float qn = 0.f;
  for (int r = w; r < R; r += nw) {
    float ss = 0.f;
    for (int d = lane; d < Dk; d += 32) ss = fmaf(q_s[r * Dk + d], q_s[r * Dk + d], ss);
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    qn = fmaxf(qn, ss);
  }
  if (lane == 0) red[w] = qn;
  __syncthreads();
  qn = 0.f;
  for (int i = 0; i < nw; ++i) qn = fmaxf(qn, red[i]);
  // the float32 sum of squares is within (1 + gamma_Dk) of the truth
  return sqrtf(qn * (1.f + 2.f * Dk * 5.96046448e-8f)) * (1.f + 1.2e-7f);
}

SA_DEV void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}

// Packed float32 FMA (two lanes of a 64-bit register pair, each rounded as
// an ordinary fma.rn.f32).
SA_DEV void ffma2(unsigned long long& acc, unsigned long long a, unsigned long long b) {
  asm volatile("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
SA_DEV float hsum2(unsigned long long v) {
  return __uint_as_float(static_cast<uint32_t>(v)) + __uint_as_float(static_cast<uint32_t>(v >> 32));
}
// bf16x2 word -> the two features as a float32 pair (low half first)
SA_DEV unsigned long long unpack2(uint32_t w) {
  return (static_cast<unsigned long long>(w & 0xffff0000u) << 32) |
         static_cast<unsigned long long>(w << 16);
}

// lo/hi bounds of every candidate page's score; NaN for forced pages.
// LPP = Dk / FPL lanes share a page, each holding FPL features of every query
// row in registers; a warp scores 32 / LPP pages per step, reading each page
// row as one coalesced run.  Per page a lane does FPL/2 packed FMAs per row
// (two float32 lanes: even / odd features), then the row sums are reduced over
// the LPP lanes with xor shuffles.  Any summation order obeys the bound
// |fl(q.s) - q.s| <= gamma_Dk ||q|| ||s||, so the bracket stays rigorous.
template <int RP, int DK>   // rows rounded up to a power of two; feature count
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const SelectArgs a) {
  constexpr int FPL = RP <= 8 ? 16 : 8;            // features per lane
  constexpr int LPP = DK / FPL;                    // lanes per page
  constexpr int NSTEPS = LPP;                      // 32 pages / (32 / LPP) per step
  constexpr int HOIST = NSTEPS < 8 ? NSTEPS : 8;   // pages steps loaded at once
  // kv heads vary fastest across the grid: the CTAs reading the Hkv adjacent
  // rows of the same pages run together and share DRAM pages / L2 lines
  const int kvh = blockIdx.x, chunk = blockIdx.y, b = blockIdx.z;
  const int L = clamped_len(a, b, false);
  const int N = (L + a.P - 1) / a.P;
  if (N <= a.budget_pages || a.k_top == 0) return;   // no ranking needed
  const int p0 = chunk * kScorePages;
  if (p0 >= N) return;
  const int G = a.Hq / a.Hkv, R = a.T * G, Dk = DK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int fb = lane % LPP, slot = lane / LPP, pages_per_step = 32 / LPP;
  // lane fb holds features [i*8*LPP + 8*fb, +8) for i < FPL/8: consecutive lanes
  // read consecutive 16-byte pieces of a page row
  // query rows: FPL features each, as float32 pairs; row norms for the bound
  unsigned long long qv[RP][FPL / 2];
  float qn2 = 0.f;
#pragma unroll
  for (int r = 0; r < RP; ++r) {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < FPL / 8; ++i) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (r < R) {
        const int t = r / G, h = kvh * G + r % G;
        w = *reinterpret_cast<const uint4*>(a.q + b * a.qs0 + t * a.qs1 + h * a.qs2 +
                                            i * 8 * LPP + 8 * fb);
      }
      const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[r][4 * i + e] = unpack2(w4[e]);
        const float x0 = __uint_as_float(w4[e] << 16), x1 = __uint_as_float(w4[e] & 0xffff0000u);
        part = fmaf(x0, x0, fmaf(x1, x1, part));
      }
    }
#pragma unroll
    for (int o = LPP / 2; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    qn2 = fmaxf(qn2, part);
  }
  const float nu = Dk * 5.96046448e-8f;
  // the float32 sums of squares are within (1 + gamma_Dk) of the truth
  const float qn = sqrtf(qn2 * (1.f + 2.f * nu)) * (1.f + 1.2e-7f);
  const float gfac = nu / (1.f - nu) * 1.0001f * qn * 1.0001f;
  const float sq_pad = 1.f + 2.f * nu;
  const int n_sink = min(a.n_sink, N), local0 = max(N - a.n_local, 0);
  const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
  float2* outrow = a.lohi + ((int64_t)b * a.Hkv + kvh) * a.max_pages;
  // this warp's 32 pages, pages_per_step at a time, HOIST steps per batch: first
  // every page-table lookup, then every row load, so that they are in flight
  // together, then the arithmetic
  const int wp0 = p0 + warp * 32;
  // the warp's 32 page-table entries in one coalesced load
  const int pt_lane = wp0 + lane < N ? ptrow[wp0 + lane] : -1;
#pragma unroll 1
  for (int sb = 0; sb < NSTEPS; sb += HOIST) {
    int phs[HOIST];
    uint4 v[HOIST][FPL / 8];
#pragma unroll
    for (int k = 0; k < HOIST; ++k) {
      const int p = wp0 + (sb + k) * pages_per_step + slot;
      const int ph = __shfl_sync(0xffffffffu, pt_lane, (sb + k) * pages_per_step + slot);
      phs[k] = -1;
      if (p < N && p >= n_sink && p < local0) phs[k] = (ph < 0 || ph >= a.P_pool) ? -2 : ph;
    }
#pragma unroll
    for (int k = 0; k < HOIST; ++k) {
#pragma unroll
      for (int i = 0; i < FPL / 8; ++i) v[k][i] = make_uint4(0, 0, 0, 0);
      if (phs[k] >= 0) {
        const uint4* src =
            reinterpret_cast<const uint4*>(a.sig + ((int64_t)phs[k] * a.Hkv + kvh) * Dk + 8 * fb);
#pragma unroll
        for (int i = 0; i < FPL / 8; ++i) v[k][i] = __ldcs(src + i * LPP);
      }
    }
#pragma unroll
    for (int k = 0; k < HOIST; ++k) {
      const int p = wp0 + (sb + k) * pages_per_step + slot;
      const bool cand = p < N && p >= n_sink && p < local0;
      const int ph = phs[k];
      if (ph == -2 && fb == 0) set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
      unsigned long long acc[RP], ss = 0ull;
#pragma unroll
      for (int r = 0; r < RP; ++r) acc[r] = 0ull;
#pragma unroll
      for (int i = 0; i < FPL / 8; ++i) {
        const uint32_t w4[4] = {v[k][i].x, v[k][i].y, v[k][i].z, v[k][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const unsigned long long x = unpack2(w4[e]);
          ffma2(ss, x, x);
#pragma unroll
          for (int r = 0; r < RP; ++r) ffma2(acc[r], qv[r][4 * i + e], x);
        }
      }
      float sc = -INFINITY, sq = hsum2(ss);
#pragma unroll
      for (int r = 0; r < RP; ++r) {
        float t = hsum2(acc[r]);
#pragma unroll
        for (int o = LPP / 2; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (r < R) sc = fmaxf(sc, t);
      }
#pragma unroll
      for (int o = LPP / 2; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (fb == 0 && p < N) {
        float2 out;
        if (!cand) {
          out = make_float2(NAN, NAN);
        } else if (ph < 0) {
          out = make_float2(-INFINITY, -INFINITY);   // an unreadable page never wins a slot
        } else {
          const float E = __fmul_ru(gfac, __fsqrt_ru(__fmul_ru(sq, sq_pad)));
          // + 0 turns -0 into +0 (the radix keys order -0 below +0)
          out = make_float2(__fsub_rd(sc, E) + 0.f, __fadd_ru(sc, E) + 0.f);
        }
        outrow[p] = out;
      }
    }
  }
}

// Radix selection of the bounds, exact rescoring of the undecided pages, and
// the ascending output of forced + selected pages.
__global__ void __launch_bounds__(kThreads) choose_kernel(const SelectArgs a) {
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
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
  __shared__ __align__(16) float q_s[kMaxRows * kMaxDk];
  __shared__ uint32_t hist[1024];
  __shared__ uint32_t sel_out[8];
  __shared__ float red_f[kThreads / 32];
  __shared__ int red_i[kThreads / 32];
  __shared__ int n_unc, n_certain;
  __shared__ double ex_tmp[kThreads];

  SelSmem S;
  S.lo = reinterpret_cast<float*>(dsm);
  S.hi = S.lo + a.max_pages;
  S.u_list = reinterpret_cast<uint16_t*>(S.hi + a.max_pages);
  S.flag = reinterpret_cast<uint8_t*>(S.u_list + a.max_pages);

  const int G = a.Hq / a.Hkv, R = a.T * G, Dk = a.Dk;
  const int n_sink = min(a.n_sink, N), local0 = max(N - a.n_local, 0);
  const int k = a.k_top;
  const float2* lohi = a.lohi + ((int64_t)b * a.Hkv + kvh) * a.max_pages;
  if (tid == 0) {
    n_unc = 0;
    n_certain = 0;
  }
  for (int p = tid; p < N; p += blockDim.x) {
    const bool cand = p >= n_sink && p < local0;
    S.flag[p] = cand ? 0 : 1;
    const float2 v = cand && k > 0 ? lohi[p] : make_float2(NAN, NAN);
    S.lo[p] = v.x;
    S.hi[p] = v.y;
  }
  __syncthreads();

  // ---- order statistics of the bounds (k == 0: streaming, no winners)
  float Lk = INFINITY, H = INFINITY;
  if (k > 0) radix_select2(S.lo, S.hi, N, k, k + 1, hist, sel_out, Lk, H);

  // ---- classify: certainly in (lo > H), undecided (hi >= Lk), else out
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

  // ---- exact scores of the undecided pages (lo/hi storage reused as doubles)
  double* ex = reinterpret_cast<double*>(S.lo);
  const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
  if (nu_ > 0 && slots > 0) {
    load_q_rows(a, b, kvh, q_s, red_f);
    const int per = max(1, kThreads / R);            // undecided pages per batch
    for (int u0 = 0; u0 < nu_; u0 += per) {
      const int u = u0 + tid / R, r = tid % R;
      if (tid < per * R && u < nu_) {
        const int ph = ptrow[S.u_list[u]];
        ex_tmp[tid] = (ph < 0 || ph >= a.P_pool)
                          ? -INFINITY
                          : exact_dot_f32q(&q_s[r * Dk],
                                           a.sig + ((int64_t)ph * a.Hkv + kvh) * Dk, Dk);
      }
      __syncthreads();
      if (tid < per && u0 + tid < nu_) {
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

  // ---- ascending compaction of the selected pages
  const int per_t = (N + blockDim.x - 1) / blockDim.x;
  const int p0 = tid * per_t, p1 = min(N, p0 + per_t);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += S.flag[p] == 1;
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

size_t select_workspace_bytes(int B, int Hkv, int max_pages) {
  return (size_t)B * Hkv * max_pages * sizeof(float2);
}

cudaError_t launch_select_gqa(const SelectArgs& a, cudaStream_t stream) {
  if (a.k_top > 0) {
    dim3 g1(a.Hkv, (a.max_pages + kScorePages - 1) / kScorePages, a.B);
    const int R = a.T * (a.Hq / a.Hkv);
    const int rp = R <= 1 ? 1 : R <= 2 ? 2 : R <= 4 ? 4 : R <= 8 ? 8 : 16;
    auto pick = [&](auto dk) {
      constexpr int DK = decltype(dk)::value;
      switch (rp) {
        case 1: score_kernel<1, DK><<<g1, kScoreThreads, 0, stream>>>(a); break;
        case 2: score_kernel<2, DK><<<g1, kScoreThreads, 0, stream>>>(a); break;
        case 4: score_kernel<4, DK><<<g1, kScoreThreads, 0, stream>>>(a); break;
        case 8: score_kernel<8, DK><<<g1, kScoreThreads, 0, stream>>>(a); break;
        default: score_kernel<16, DK><<<g1, kScoreThreads, 0, stream>>>(a); break;
      }
    };
    if (a.Dk == 64) pick(std::integral_constant<int, 64>{});
    else if (a.Dk == 128) pick(std::integral_constant<int, 128>{});
    else pick(std::integral_constant<int, 256>{});
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t dyn = (size_t)a.max_pages * (4 + 4 + 2 + 1) + 16;
  cudaError_t e = cudaFuncSetAttribute(choose_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e != cudaSuccess) return e;
  choose_kernel<<<dim3(a.Hkv, a.B), kThreads, dyn, stream>>>(a);
  return cudaGetLastError();
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
float2* g_static_ptr[kMaxDevices] = {};

// Device address of the static array on the current device; looked up once per
// device (the host-side symbol is only a stand-in and must not reach a kernel).
cudaError_t static_scores_ptr(float2** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_score_bounds);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = static_cast<float2*>(p);
  }
  *out = g_static_ptr[dev];
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
