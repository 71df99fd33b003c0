// Log-sum-exp merge of split-KV partials: lse = log sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s.  One thread per (row, 4 output columns),
// 16-byte loads and stores, the loads of 8 splits in flight together, no load
// of a split without keys; memory-bound.
//
// Source: the merge step of a split Flash-decode ("TileSparse", section
// "Configuration": mode full = fused Flash-decode).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kCombineBatch = 8;   // splits whose loads are in flight together (many splits)
constexpr int kRegSplits = 16;     // up to this many splits: every load of a phase at once

// 16-byte load that happens only when `pred` holds (a predicated instruction,
// not a branch: a run of them is issued back to back); zeros otherwise.
SA_DEV float4 ld4_if(const float* p, bool pred) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
      " @q ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];\n}\n"
      : "+f"(v.x), "+f"(v.y), "+f"(v.z), "+f"(v.w)
      : "l"(p), "r"(static_cast<int>(pred)));
  return v;
}

// KS: splits handled in registers (n_splits <= KS), 0 = any count in batches.
template <int KS>
__global__ void __launch_bounds__(128)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   int n_splits, int64_t rows, int Dv, float* __restrict__ o_out,
                   uint16_t* __restrict__ o_bf16, float* __restrict__ lse_out) {
  pdl_wait_and_release();
  // (32-bit index arithmetic: the launcher guarantees rows * Dv / 4 < 2^32)
  const uint32_t q4 = static_cast<uint32_t>(Dv) / 4u;
  const uint32_t idx = blockIdx.x * blockDim.x + threadIdx.x;
  const bool live = idx < static_cast<uint32_t>(rows) * q4;
  if (!live) return;
  const uint32_t row_ = idx / q4;
  const int64_t row = row_;
  const int c = static_cast<int>(idx - row_ * q4) * 4;
  // The split LSEs first, then the O rows of the splits that have keys (a
  // split without keys is not read at all); with up to kRegSplits splits every
  // load of a phase is issued before any is used.
  float m = -INFINITY, tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (KS > 0) {
    float w[KS];
#pragma unroll
    for (int s = 0; s < KS; ++s)   // (index clamped: unconditional loads)
      w[s] = __ldg(lse_part + min(s, n_splits - 1) * rows + row);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      if (s >= n_splits) w[s] = -INFINITY;
      m = fmaxf(m, w[s]);
    }
    if (m != -INFINITY) {
      float4 v[KS];
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        w[s] = __expf(w[s] - m);
        v[s] = ld4_if(o_part + (s * rows + row) * Dv + c, w[s] > 0.f);
      }
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        tot += w[s];
        acc.x += w[s] * v[s].x;
        acc.y += w[s] * v[s].y;
        acc.z += w[s] * v[s].z;
        acc.w += w[s] * v[s].w;
      }
    }
  } else {
    for (int s0 = 0; s0 < n_splits; s0 += kCombineBatch) {
      float ls[kCombineBatch];
#pragma unroll
      for (int i = 0; i < kCombineBatch; ++i)
        ls[i] = s0 + i < n_splits ? __ldg(lse_part + (s0 + i) * rows + row) : -INFINITY;
#pragma unroll
      for (int i = 0; i < kCombineBatch; ++i) m = fmaxf(m, ls[i]);
    }
    if (m != -INFINITY)
      for (int s0 = 0; s0 < n_splits; s0 += kCombineBatch) {
        float w[kCombineBatch];
        float4 v[kCombineBatch];
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i)
          w[i] = s0 + i < n_splits ? __expf(__ldg(lse_part + (s0 + i) * rows + row) - m) : 0.f;
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i)
          v[i] = ld4_if(o_part + ((s0 + i) * rows + row) * Dv + c, w[i] > 0.f);
#pragma unroll
        for (int i = 0; i < kCombineBatch; ++i) {
          tot += w[i];
          acc.x += w[i] * v[i].x;
          acc.y += w[i] * v[i].y;
          acc.z += w[i] * v[i].z;
          acc.w += w[i] * v[i].w;
        }
      }
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
  if (n >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
  const int threads = 128;
  const int64_t blocks = (n + threads - 1) / threads;
  auto go = [&](auto kern) {
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(threads), 0, stream, o_part, lse_part,
                      n_splits, rows, Dv, o_out, o_bf16, lse_out);
  };
  if (n_splits <= 4) return go(combine_kernel<4>);
  if (n_splits <= 8) return go(combine_kernel<8>);
  if (n_splits <= kRegSplits) return go(combine_kernel<kRegSplits>);
  return go(combine_kernel<0>);
}

}  // namespace sa
