// The ambient head set of the Critical / Ambient tiers: the h query heads whose
// estimated attention mass falls most on the ambient pages.
//
// For sequence b, query token t and head h, page p of the sequence carries the
// estimated mass n_p exp(scale (q . sigma_p)) (n_p valid tokens, every key of
// the page replaced by the page's mean key, sigma_p); the coverage of (b, t, h)
// is the ambient pages' share of the mass of all the sequence's pages, and a
// head's score is the sum of its coverages over the call's sequences and
// tokens.  The h best heads (ties to the lower head) form the set.
//
//   head_mass_kernel: one CTA per (32 pages, 32 query rows, sequence): the
//     dot products in float64 (bf16 products are exact in float64; the query
//     rows and the transposed summaries sit in shared memory as float32, which
//     holds every bf16 exactly), then per row the chunk's largest scaled score m
//     and the sums of n_p exp(z - m) over all and over the ambient pages.
//   head_pick_kernel: one CTA: each head's score from the chunks' partials
//     (sequences, tokens and chunks in a fixed order), then each head's rank by
//     counting the heads that beat it, and the chosen heads in ascending order.
//
// Source: "TileSparse: Arithmetic-Intensity-Aware Sparse Attention for
// Compute-Bound LLM Decoding", "Motivation" (the Ambient Tier is computed with
// h heads) and "Configuration" (an AutoTuner chooses them per layer by
// estimated attention-mass coverage).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kHPages = 32;     // pages per CTA (one per lane)
constexpr int kHRows = 32;      // query rows per CTA (four per warp)
constexpr int kHThreads = 256;
constexpr int kHMaxDk = 768;

__global__ void __launch_bounds__(kHThreads) head_mass_kernel(const HeadArgs a) {
  pdl_wait_and_release();
  const int chunk = blockIdx.x, rb = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = a.T * a.Hq, Dk = a.Dk;
  extern __shared__ __align__(16) float hsm[];
  float* q_s = hsm;                        // [kHRows][Dk]
  float* s_t = hsm + kHRows * Dk;          // [Dk][kHPages]
  __shared__ int amb_s[kHPages];
  __shared__ float np_s[kHPages];

  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
    if (tid == 0 && chunk == 0 && rb == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  const int nb = (L + a.P - 1) / a.P;
  const int p0 = chunk * kHPages;
  // query rows r = t * Hq + h of this CTA
  for (int i = tid; i < kHRows * Dk; i += kHThreads) {
    const int rr = i / Dk, d = i % Dk, r = rb * kHRows + rr;
    float v = 0.f;
    if (r < R) {
      const int t = r / a.Hq, h = r % a.Hq;
      v = bf16_bits_to_float(a.q[b * a.qs0 + t * a.qs1 + h * a.qs2 + d]);
    }
    q_s[i] = v;
  }
  // the chunk's summaries, transposed (page fastest)
  for (int i = tid; i < kHPages * Dk; i += kHThreads) {
    const int pg = i / Dk, d = i % Dk, p = p0 + pg;
    float v = 0.f;
    if (p < nb) {
      const int ph = a.page_table[(int64_t)b * a.max_pages + p];
      if (ph >= 0 && ph < a.P_pool) v = bf16_bits_to_float(a.sig[(int64_t)ph * Dk + d]);
    }
    s_t[d * kHPages + pg] = v;
  }
  if (tid < kHPages) {
    const int p = p0 + tid;
    bool ok = p < nb, amb = false;
    if (ok) {
      const int ph = a.page_table[(int64_t)b * a.max_pages + p];
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        ok = false;
      }
      // ambient = in list 1 (critical + ambient) and not in list 0 (critical)
      const int32_t* l0 = a.lists + (int64_t)b * 2 * a.cap;
      const int32_t* l1 = l0 + a.cap;
      const int c0 = min(max(a.counts[b * 2], 0), a.cap);
      const int c1 = min(max(a.counts[b * 2 + 1], 0), a.cap);
      for (int i = 0; i < c1; ++i) amb |= l1[i] == p;
      for (int i = 0; i < c0; ++i) amb &= l0[i] != p;
    }
    amb_s[tid] = ok && amb ? 1 : 0;
    np_s[tid] = ok ? static_cast<float>(min(a.P, L - p * a.P)) : 0.f;
  }
  __syncthreads();
  // four rows per warp, one page per lane
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int d = 0; d < Dk; ++d) {
    const double s = static_cast<double>(s_t[d * kHPages + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc[i] = fma(static_cast<double>(q_s[(warp + 8 * i) * Dk + d]), s, acc[i]);
  }
  const bool live = np_s[lane] > 0.f;
  const double n_p = np_s[lane];
  const bool amb = amb_s[lane] != 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rb * kHRows + warp + 8 * i;
    const double z = live ? static_cast<double>(a.scale) * acc[i] : -INFINITY;
    double m = z;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    const double w = live ? n_p * exp(z - m) : 0.0;
    double s_all = w, s_amb = amb ? w : 0.0;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s_all += __shfl_xor_sync(0xffffffffu, s_all, o);
      s_amb += __shfl_xor_sync(0xffffffffu, s_amb, o);
    }
    if (lane == 0 && r < R) {
      double* dst = a.part + (((int64_t)b * a.n_chunks + chunk) * R + r) * 3;
      dst[0] = m;          // -inf: no page of the sequence in this chunk
      dst[1] = s_all;
      dst[2] = s_amb;
    }
  }
}

__global__ void __launch_bounds__(1024) head_pick_kernel(const HeadArgs a) {
  pdl_wait_and_release();
  const int h = threadIdx.x;
  const int R = a.T * a.Hq;
  __shared__ double score_s[1024];
  __shared__ int win_s[1024];
  double score = 0.0;
  if (h < a.Hq) {
    for (int b = 0; b < a.B; ++b)
      for (int t = 0; t < a.T; ++t) {
        const int r = t * a.Hq + h;
        const double* p = a.part + ((int64_t)b * a.n_chunks * R + r) * 3;
        double m = -INFINITY;
        for (int c = 0; c < a.n_chunks; ++c) m = fmax(m, p[(int64_t)c * R * 3]);
        if (m == -INFINITY) continue;   // an empty sequence covers nothing
        double all = 0.0, amb = 0.0;
        for (int c = 0; c < a.n_chunks; ++c) {
          const double mc = p[(int64_t)c * R * 3];
          if (mc == -INFINITY) continue;
          const double f = exp(mc - m);
          all += p[(int64_t)c * R * 3 + 1] * f;
          amb += p[(int64_t)c * R * 3 + 2] * f;
        }
        score += amb / all;
      }
    score_s[h] = score;
  }
  __syncthreads();
  // head h wins iff fewer than k heads beat it by (score desc, head asc)
  int beat = 0;
  if (h < a.Hq)
    for (int j = 0; j < a.Hq; ++j) {
      const double sj = score_s[j];
      beat += sj > score || (sj == score && j < h);
    }
  const int win = h < a.Hq && beat < a.h_keep ? 1 : 0;
  win_s[h] = win;
  if (h < a.Hq && a.scores_out) a.scores_out[h] = score;
  __syncthreads();
  if (win) {   // position among the winners = winners below h
    int pos = 0;
    for (int j = 0; j < h; ++j) pos += win_s[j];
    a.heads_out[pos] = h;
  }
}

}  // namespace

size_t head_workspace_bytes(int B, int T, int Hq, int max_pages) {
  const int n_chunks = (max_pages + kHPages - 1) / kHPages;
  return (size_t)B * (n_chunks > 0 ? n_chunks : 1) * T * Hq * 3 * sizeof(double);
}

int head_max_dk() { return kHMaxDk; }

cudaError_t launch_select_heads(HeadArgs a, cudaStream_t stream) {
  a.n_chunks = (a.max_pages + kHPages - 1) / kHPages;
  if (a.n_chunks == 0) a.n_chunks = 1;
  const int R = a.T * a.Hq;
  const size_t dyn = (size_t)(kHRows + kHPages) * a.Dk * sizeof(float);
  cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(head_mass_kernel));
  if (e != cudaSuccess) return e;
  e = launch_pdl(head_mass_kernel, dim3(a.n_chunks, (R + kHRows - 1) / kHRows, a.B),
                 dim3(kHThreads), dyn, stream, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(head_pick_kernel, dim3(1), dim3(1024), 0, stream, a);
}

}  // namespace sa
