// Block-union KV tables for chunked prefill.
//
// Pass 1 clears the per-group flag rows (the output tables double as flags).
// Pass 2 runs one CTA per (Q-block, head): it flags the sink blocks, the
// diagonal block, and the top_k earlier blocks chosen by repeated block-wide
// argmax over 64-bit keys (score key << 32 | ~index: larger score first,
// then lower index).  Pass 3 runs one CTA per group and compacts its flags
// into an ascending table.
//
// Source: CompactAttention, Block-Union KV Selection (abstract on the page
// titled "Causal Attention on CPU: A Cache-Aware and Load-Balanced Scheduling
// Kernel for Prefill"): Q-block union and intra-group union into per-group KV
// block tables, used in place without KV compaction.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kUThreads = 256;
constexpr int kMaxBlocks = 16384;

SA_DEV uint32_t f2key_u(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void union_clear_kernel(int32_t* tables, int64_t n) {
  pdl_wait_and_release();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    tables[i] = 0;
}

__global__ void __launch_bounds__(kUThreads)
    union_mark_kernel(const float* __restrict__ scores, int Hq, int Hkv, int NQB, int NKB,
                      int q_off, int top_k, int n_sink, int32_t* tables) {
  pdl_wait_and_release();
  const int j = blockIdx.x, h = blockIdx.y;
  const int g = h / (Hq / Hkv);
  const int d = q_off + j;
  int32_t* flags = tables + (int64_t)g * NKB;
  const float* srow = scores + ((int64_t)h * NQB + j) * NKB;
  __shared__ unsigned long long warp_best[kUThreads / 32];
  extern __shared__ unsigned long long keys[];   // [d - n_sink]

  for (int i = threadIdx.x; i < min(n_sink, d + 1); i += blockDim.x) flags[i] = 1;
  if (threadIdx.x == 0) flags[d] = 1;
  const int c0 = n_sink, nc = d - n_sink;
  if (nc <= 0 || top_k <= 0) return;
  for (int i = threadIdx.x; i < nc; i += blockDim.x) {
    const int c = c0 + i;
    keys[i] = (static_cast<unsigned long long>(f2key_u(srow[c])) << 32) |
              static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(c));
  }
  __syncthreads();
  const int rounds = min(top_k, nc);
  for (int r = 0; r < rounds; ++r) {
    unsigned long long m = 0ull;
    for (int i = threadIdx.x; i < nc; i += blockDim.x) m = keys[i] > m ? keys[i] : m;
    for (int o = 16; o; o >>= 1) {
      const unsigned long long v = __shfl_xor_sync(0xffffffffu, m, o);
      m = v > m ? v : m;
    }
    if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long bm = 0ull;
      for (int w = 0; w < kUThreads / 32; ++w) bm = warp_best[w] > bm ? warp_best[w] : bm;
      const int c = static_cast<int>(0xffffffffu - static_cast<uint32_t>(bm & 0xffffffffull));
      flags[c] = 1;
      keys[c - c0] = 0ull;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kUThreads)
    union_compact_kernel(int32_t* tables, int32_t* counts, int NKB) {
  pdl_wait_and_release();
  const int g = blockIdx.x;
  int32_t* row = tables + (int64_t)g * NKB;
  extern __shared__ uint8_t fl[];   // [NKB]
  __shared__ int warp_tot[kUThreads / 32];
  for (int i = threadIdx.x; i < NKB; i += blockDim.x) fl[i] = row[i] != 0;
  __syncthreads();
  const int per = (NKB + blockDim.x - 1) / blockDim.x;
  const int p0 = threadIdx.x * per, p1 = min(NKB, p0 + per);
  int cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += fl[p];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  int base = 0, total = 0;
  for (int i = 0; i < kUThreads / 32; ++i) {
    if (i < w) base += warp_tot[i];
    total += warp_tot[i];
  }
  int pos = base + incl - cnt;
  for (int p = p0; p < p1; ++p)
    if (fl[p]) row[pos++] = p;
  for (int i = total + threadIdx.x; i < NKB; i += blockDim.x) row[i] = -1;
  if (threadIdx.x == 0) counts[g] = total;
}

}  // namespace

cudaError_t launch_block_union(const float* scores, int Hq, int Hkv, int NQB, int NKB, int q_off,
                               int top_k, int n_sink, int32_t* tables, int32_t* counts,
                               cudaStream_t stream) {
  if (NKB > kMaxBlocks) return cudaErrorInvalidValue;
  const int64_t n = (int64_t)Hkv * NKB;
  cudaError_t e =
      launch_pdl(union_clear_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream, tables, n);
  if (e != cudaSuccess) return e;
  const size_t kbytes = sizeof(unsigned long long) * (size_t)NKB;
  e = allow_max_dyn_smem(reinterpret_cast<const void*>(union_mark_kernel));
  if (e != cudaSuccess) return e;
  if (NQB > 0) {
    e = launch_pdl(union_mark_kernel, dim3(NQB, Hq), dim3(kUThreads), kbytes, stream, scores, Hq,
                   Hkv, NQB, NKB, q_off, top_k, n_sink, tables);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(union_compact_kernel, dim3(Hkv), dim3(kUThreads), NKB, stream, tables, counts,
                    NKB);
}

}  // namespace sa
