// Gather-based split-KV Flash-decode over per-head page lists (GQA / MTP).
//
// One CTA per (split, (list, kv head) pair, sequence).  Each warp owns a ring
// of shared-memory stages; its lane 0 gathers 16-token sub-pages of K and V
// straight from the paged pool with TMA tile loads (page ids resolved through
// the list and the page table), and the warp runs QK^T, an online softmax and
// PV on them with m16n8k16 bf16 tensor-core MMAs: the 16 rows of the MMA are
// the query rows (T x heads of the pair), the columns the 16 tokens.  The
// probabilities enter PV as a bf16 hi + lo pair so that their rounding stays
// far below the output tolerance.  Warps merge their (max, sum, O) states in
// shared memory at the end and the CTA writes one normalised partial + LSE.
//
// Sources: "Universal Attention Engine — Declarative Sparse Attention for
// Production" ("Architecture": gather-based sparse KV decode; "Key Design
// Decisions" 3: decode is memory-bound, optimise bytes loaded) and "TileSparse"
// ("Two implementations": a per-head page-list Flash-decode kernel).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kNW = 4;       // warps per CTA
constexpr int kSub = 16;     // tokens per TMA sub-page (one MMA k-step of PV)

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                     // 64-column TMA boxes per row set
  static constexpr int kBoxBytes = kSub * 128;              // 16 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;     // one K (or V) sub-page
  static constexpr int kStageBytes = 2 * kTileBytes;        // K + V
  static constexpr int kStages = D >= 256 ? 2 : 3;
  static constexpr int kRingBytes = kNW * kStages * kStageBytes;
  static constexpr int kMergeBytes = kNW * 16 * (D + 2) * 4;
  static constexpr int kDynBytes = (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes) + 1024;
};

struct __align__(64) DecodeParams {
  DecodeArgs a;
  PairTable pairs;
};

template <int D>
__global__ void __launch_bounds__(kNW * 32)
    decode_gqa_kernel(const __grid_constant__ DecodeParams prm,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
  using C = DecodeCfg<D>;
  const DecodeArgs& a = prm.a;
  const int split = blockIdx.x, pair = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  __shared__ uint64_t bars[kNW][C::kStages];
  __shared__ int phys_s[kMaxSplitEntries];
  __shared__ int page_s[kMaxSplitEntries];

  const int list = prm.pairs.list_of[pair];
  const int kvh = prm.pairs.kvh_of[pair];
  const int nh = prm.pairs.n_heads[pair];
  const int R = a.T * nh;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {  // a length the page table cannot hold
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    L = L < 0 ? 0 : a.max_pages * a.P;
  }
  const int n_log = (L + a.P - 1) / a.P;

  int count = a.counts[b * a.n_lists + list];
  if (count < 0 || count > a.max_list) {
    if (tid == 0) set_dev_error(a.err, SA_DEVERR_COUNT);
    count = count < 0 ? 0 : a.max_list;
  }
  const int chunk = (count + a.n_splits - 1) / a.n_splits;
  const int e0 = min(split * chunk, count);
  const int n_ent = min(chunk, count - e0);

  // Resolve logical -> physical page ids for this split once.
  const int32_t* lrow = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list;
  for (int i = tid; i < n_ent; i += blockDim.x) {
    int p = lrow[e0 + i];
    int ph = -1;
    if (p < 0 || p >= n_log) {
      set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    } else {
      ph = a.page_table[(int64_t)b * a.max_pages + p];
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        ph = -1;
      }
    }
    phys_s[i] = ph;
    page_s[i] = p;
  }
  if (lane == 0)
    for (int s = 0; s < C::kStages; ++s) mbar_init(&bars[warp][s], 1);
  if (tid == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  fence_mbar_init();
  __syncthreads();

  const int subs = a.P / kSub;
  const int n_units = n_ent * subs;
  const int my_units = n_units > warp ? (n_units - warp + kNW - 1) / kNW : 0;
  uint8_t* ring = smem + warp * C::kStages * C::kStageBytes;

  // A unit is (entry, 16-token sub-page); it carries data iff its page is
  // valid and some of its tokens lie before the sequence end.
  auto unit_live = [&](int u, int& ph, int& tok0) {
    const int e = u / subs, st = u % subs;
    ph = phys_s[e];
    tok0 = page_s[e] * a.P + st * kSub;
    return ph >= 0 && tok0 < L;
  };
  auto issue = [&](int k) {  // lane 0 only: unit number k of this warp
    const int u = warp + k * kNW;
    const int slot = k % C::kStages;
    uint64_t* bar = &bars[warp][slot];
    int ph, tok0;
    if (unit_live(u, ph, tok0)) {
      uint8_t* kt = ring + slot * C::kStageBytes;
      uint8_t* vt = kt + C::kTileBytes;
      const int row0 = (u % subs) * kSub;
      mbar_arrive_expect_tx(bar, C::kStageBytes);
#pragma unroll
      for (int bx = 0; bx < C::kBoxes; ++bx) {
        tma_load_4d(kt + bx * C::kBoxBytes, &kmap, bar, bx * 64, row0, kvh, ph);
        tma_load_4d(vt + bx * C::kBoxBytes, &vmap, bar, bx * 64, row0, kvh, ph);
      }
    } else {
      mbar_arrive_expect_tx(bar, 0);
    }
  };
  if (lane == 0)
    for (int k = 0; k < my_units && k < C::kStages; ++k) issue(k);

  // Query fragments (A operand of QK^T), rows r = t * nh + i.
  uint32_t qa[D / 16][4];
  int lim[2];
  {
    const int rows[2] = {gid, gid + 8};
    const uint16_t* qp[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = rows[h];
      if (r < R) {
        const int t = r / nh, head = prm.pairs.heads[pair][r % nh];
        qp[h] = a.q + b * a.qs0 + t * a.qs1 + head * a.qs2;
        lim[h] = L - a.T + t;
      } else {
        qp[h] = nullptr;
        lim[h] = -1;
      }
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * tig;
      qa[kk][0] = qp[0] ? *reinterpret_cast<const uint32_t*>(qp[0] + c) : 0u;
      qa[kk][1] = qp[1] ? *reinterpret_cast<const uint32_t*>(qp[1] + c) : 0u;
      qa[kk][2] = qp[0] ? *reinterpret_cast<const uint32_t*>(qp[0] + c + 8) : 0u;
      qa[kk][3] = qp[1] ? *reinterpret_cast<const uint32_t*>(qp[1] + c + 8) : 0u;
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  int k_fail = -1;

  for (int k = 0; k < my_units; ++k) {
    const int u = warp + k * kNW;
    const int slot = k % C::kStages;
    if (!mbar_wait_bounded(&bars[warp][slot], (k / C::kStages) & 1)) {
      k_fail = k;
      break;
    }
    int ph, tok0;
    if (unit_live(u, ph, tok0)) {
      const uint8_t* kt = ring + slot * C::kStageBytes;
      const uint8_t* vt = kt + C::kTileBytes;
      const uint32_t kbase = smem_u32(kt), vbase = smem_u32(vt);
      // ---- S = Q K^T (16 rows x 16 tokens)
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int colb = (kk & 3) * 16;
        const uint32_t addr = kbase + (kk >> 2) * C::kBoxBytes +
                              swz128(8 * (mi >> 1) + ri, colb + 8 * (mi & 1));
        uint32_t r[4];
        ldmatrix_x4(r, addr);
        mma_bf16_16816(s[0], qa[kk], r[0], r[1]);
        mma_bf16_16816(s[1], qa[kk], r[2], r[3]);
      }
      // ---- mask, online softmax (base 2)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int h = c >> 1;
          const int pos = tok0 + nt * 8 + 2 * tig + (c & 1);
          const bool ok = pos < L && pos <= lim[h];
          s[nt][c] = ok ? s[nt][c] * a.scale_log2 : -INFINITY;
          mx[h] = fmaxf(mx[h], s[nt][c]);
        }
      float alpha[2], base[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float m_new = fmaxf(m_run[h], mx[h]);
        base[h] = m_new == -INFINITY ? 0.f : m_new;
        alpha[h] = exp2f(m_run[h] - base[h]);
        m_run[h] = m_new;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          s[nt][c] = exp2f(s[nt][c] - base[c >> 1]);
          rs[c >> 1] += s[nt][c];
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * alpha[h] + rs[h];
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= alpha[0];
        o[i][1] *= alpha[0];
        o[i][2] *= alpha[1];
        o[i][3] *= alpha[1];
      }
      // ---- O += P V with P = hi + lo (both bf16)
      uint32_t ph_[4], pl_[4];
      {
        const float pv[4][2] = {{s[0][0], s[0][1]}, {s[0][2], s[0][3]},
                                {s[1][0], s[1][1]}, {s[1][2], s[1][3]}};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ph_[i] = pack_bf16(pv[i][0], pv[i][1]);
          const float h0 = bf16_bits_to_float(ph_[i] & 0xffffu);
          const float h1 = bf16_bits_to_float(ph_[i] >> 16);
          pl_[i] = pack_bf16(pv[i][0] - h0, pv[i][1] - h1);
        }
      }
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        const int colb = (n2 & 3) * 16;
        const uint32_t addr = vbase + (n2 >> 2) * C::kBoxBytes +
                              swz128(8 * (mi & 1) + ri, colb + 8 * (mi >> 1));
        uint32_t r[4];
        ldmatrix_x4_trans(r, addr);
        mma_bf16_16816(o[2 * n2], ph_, r[0], r[1]);
        mma_bf16_16816(o[2 * n2], pl_, r[0], r[1]);
        mma_bf16_16816(o[2 * n2 + 1], ph_, r[2], r[3]);
        mma_bf16_16816(o[2 * n2 + 1], pl_, r[2], r[3]);
      }
    }
    __syncwarp();
    if (lane == 0 && k + C::kStages < my_units) issue(k + C::kStages);
  }
  if (k_fail >= 0) {
    if (lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
    // Units k_fail .. k_fail + kStages - 1 were issued; wait for them (again
    // bounded) before the shared memory they target is reused.
    for (int kk = k_fail + 1; kk < my_units && kk < k_fail + C::kStages; ++kk)
      mbar_wait_bounded(&bars[warp][kk % C::kStages], (kk / C::kStages) & 1);
  }

  // ---- merge the warps' states
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
  __syncthreads();  // every warp is done with its ring
  float* mrg = reinterpret_cast<float*>(smem);
  float* mrg_m = mrg;                         // [kNW][16]
  float* mrg_l = mrg + kNW * 16;              // [kNW][16]
  float* mrg_o = mrg + 2 * kNW * 16;          // [kNW][16][D]
  if (tig == 0) {
    mrg_m[warp * 16 + gid] = m_run[0];
    mrg_m[warp * 16 + gid + 8] = m_run[1];
    mrg_l[warp * 16 + gid] = l_run[0];
    mrg_l[warp * 16 + gid + 8] = l_run[1];
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int d = i * 8 + 2 * tig;
    float* r0 = mrg_o + (warp * 16 + gid) * D + d;
    float* r1 = mrg_o + (warp * 16 + gid + 8) * D + d;
    *reinterpret_cast<float2*>(r0) = make_float2(o[i][0], o[i][1]);
    *reinterpret_cast<float2*>(r1) = make_float2(o[i][2], o[i][3]);
  }
  __syncthreads();
  const int64_t row_stride_t = (int64_t)a.Hq;
  for (int idx = tid; idx < R * (D / 4); idx += blockDim.x) {
    const int r = idx / (D / 4), d = (idx % (D / 4)) * 4;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, mrg_m[w * 16 + r]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float f = exp2f(mrg_m[w * 16 + r] - M);
        Lsum += mrg_l[w * 16 + r] * f;
        const float4 v = *reinterpret_cast<const float4*>(mrg_o + (w * 16 + r) * D + d);
        acc.x += v.x * f;
        acc.y += v.y * f;
        acc.z += v.z * f;
        acc.w += v.w * f;
      }
      const float inv = 1.f / Lsum;
      acc.x *= inv;
      acc.y *= inv;
      acc.z *= inv;
      acc.w *= inv;
    }
    const int t = r / nh, head = prm.pairs.heads[pair][r % nh];
    const int64_t row = (((int64_t)split * a.B + b) * a.T + t) * row_stride_t + head;
    *reinterpret_cast<float4*>(a.o_part + row * D + d) = acc;
    if (d == 0) a.lse_part[row] = M == -INFINITY ? -INFINITY : (M + log2f(Lsum)) * kLn2;
  }
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                     const CUtensorMap& vmap, cudaStream_t stream) {
  using C = DecodeCfg<D>;
  DecodeParams prm;
  prm.a = a;
  prm.pairs = pairs;
  cudaError_t e = cudaFuncSetAttribute(decode_gqa_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kDynBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_splits, pairs.n_pairs, a.B);
  decode_gqa_kernel<D><<<grid, kNW * 32, C::kDynBytes, stream>>>(prm, kmap, vmap);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, cudaStream_t stream) {
  switch (a.Dk) {
    case 64: return launch_d<64>(a, pairs, kmap, vmap, stream);
    case 128: return launch_d<128>(a, pairs, kmap, vmap, stream);
    case 256: return launch_d<256>(a, pairs, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
