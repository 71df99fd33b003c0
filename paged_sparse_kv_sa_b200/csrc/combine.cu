// Log-sum-exp merge of split-KV partials: lse = log sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s.  One thread per (row, 4 output columns),
// 16-byte loads and stores, the loads of 8 splits in flight together;
// memory-bound.
//
// Source: the merge step of a split Flash-decode ("TileSparse", section
// "Configuration": mode full = fused Flash-decode).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kCombineBatch = 8;   // splits whose loads are in flight together

__global__ void __launch_bounds__(128)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   int n_splits, int64_t rows, int Dv, float* __restrict__ o_out,
                   uint16_t* __restrict__ o_bf16, float* __restrict__ lse_out) {
  pdl_wait_and_release();
  const int q4 = Dv / 4;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * q4) return;
  const int64_t row = idx / q4;
  const int c = (int)(idx % q4) * 4;
  // running merge over batches of splits: every load of a batch is issued
  // before any of them is used
  float m = -INFINITY, tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n_splits; s0 += kCombineBatch) {
    float ls[kCombineBatch];
    float4 v[kCombineBatch];
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const int s = s0 + i;
      ls[i] = s < n_splits ? lse_part[s * rows + row] : -INFINITY;
      v[i] = s < n_splits ? *reinterpret_cast<const float4*>(o_part + (s * rows + row) * Dv + c)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = m;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) mb = fmaxf(mb, ls[i]);
    if (mb == -INFINITY) continue;
    const float sc = __expf(m - mb);   // 0 while nothing has been merged
    tot *= sc;
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const float w = __expf(ls[i] - mb);
      tot += w;
      // a split without keys (weight 0) adds nothing, whatever its O holds
      if (w > 0.f) {
        acc.x += w * v[i].x;
        acc.y += w * v[i].y;
        acc.z += w * v[i].z;
        acc.w += w * v[i].w;
      }
    }
    m = mb;
  }
  float lse = -INFINITY;
  if (m != -INFINITY) {
    const float inv = 1.f / tot;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    lse = m + logf(tot);
  }
  if (o_out) *reinterpret_cast<float4*>(o_out + row * Dv + c) = acc;
  if (o_bf16) {
    uint2 p;
    p.x = pack_bf16(acc.x, acc.y);
    p.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2*>(o_bf16 + row * Dv + c) = p;
  }
  if (lse_out && c == 0) lse_out[row] = lse;
}

}  // namespace

cudaError_t launch_combine(const float* o_part, const float* lse_part, int n_splits, int64_t rows,
                           int Dv, float* o_out, uint16_t* o_bf16, float* lse_out,
                           cudaStream_t stream) {
  const int64_t n = rows * (Dv / 4);
  if (n == 0) return cudaSuccess;
  const int threads = 128;
  const int64_t blocks = (n + threads - 1) / threads;
  return launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(threads), 0, stream, o_part,
                    lse_part, n_splits, rows, Dv, o_out, o_bf16, lse_out);
}

}  // namespace sa
