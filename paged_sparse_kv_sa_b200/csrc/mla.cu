// Sparse MLA decode over per-head page lists on the 5th-generation tensor
// cores: one shared latent KV head, keys of Dk = 576 (512 latent + 64 rope),
// values = the first Dv = 512 key columns (read from the same tile), many
// query rows (T x heads) per list.
//
// One CTA computes 64 query rows of one (list, kv head) pair against its split
// of the list, 32 keys per tile.  The MMAs are M = 64: TMEM then holds a
// 64-row accumulator in the low 16 lanes of each 32-lane subpartition, and a
// second one in the high 16 lanes of the same columns.  O (64 x 512 float32)
// is kept as two such halves — value columns 0-255 in the low lanes, 256-511
// in the high lanes — in TMEM columns [0, 256); the two S buffers (64 x 32)
// sit in columns [256, 320).  So the whole output fits in TMEM next to S and
// no FLOP is spent twice.
//   warp 4      TMA-gathers key tiles (9 column chunks x two 16-key boxes; an
//               absent or invalid group is read at an out-of-range page, which
//               TMA fills with zeros) into a 3-stage ring;
//   warp 5      issues S = Q K^T (36 MMAs of 64x32x16) and O += P V (per value
//               half two MMAs of 64x256x16, V = key columns of the same tile);
//   warps 0-3   own a row each in their low 16 lanes: mask, lazily re-based
//               base-2 online softmax, P to shared memory; the high 16 lanes
//               mirror the row statistics and rescale / write the second value
//               half of O.
//
// Sources: "TileSparse: Arithmetic-Intensity-Aware Sparse Attention for
// Compute-Bound LLM Decoding" ("Motivation": MLA and MTP push decode attention
// above the hardware ridge point; "Two implementations": per-head page-list
// Flash-decode) and "Universal Attention Engine — Declarative Sparse Attention
// for Production" ("Architecture": gather-based sparse KV decode).
#include "common.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace sa {
namespace {

constexpr int kMThreads = 192;
constexpr int kMStages = 3;
constexpr int kMKeys = 32;          // keys per tile
constexpr int kMRows = 64;          // query rows per CTA
constexpr int kMMaxEnt = 512;       // list entries per split
constexpr int kDk = 576, kDv = 512;
constexpr int kKC = kDk / 64;       // 9 key column chunks
constexpr int kQBytes = kKC * kMRows * 128;          // 73728
constexpr int kChunkBytes = kMKeys * 128;            // 4096: one column chunk of a tile
constexpr int kTileBytes = kKC * kChunkBytes;        // 36864
constexpr int kPBytes = kMRows * 128;                // 8192 (32 keys used of 64)
constexpr int kMDyn = kQBytes + kMStages * kTileBytes + 2 * kPBytes + 1024;
constexpr uint32_t kMTmemCols = 512;
constexpr uint32_t kSCol = 256;                      // S buffers at 256 and 288
constexpr uint32_t kHiLanes = 16u << 16;             // second M=64 accumulator
constexpr uint32_t kIdQK = tc::idesc_bf16_f32(kMRows, kMKeys, false, false);
constexpr uint32_t kIdPV = tc::idesc_bf16_f32(kMRows, 256, false, true);
constexpr float kLazyM = 8.f;

struct __align__(64) MlaParams {
  DecodeArgs a;
  PairTable pairs;
};

SA_DEV bool wait_or_abort_m(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// (physical page or -1, first token) of 16-key group g of tile j.
SA_DEV int2 mgroup(const int2* ent, int n_ent, int P, int j, int g) {
  const int key0 = (2 * j + g) * 16;
  const int e = key0 / P;
  if (e >= n_ent) return make_int2(-1, 0);
  const int2 en = ent[e];
  return make_int2(en.x, en.y + key0 % P);
}

__global__ void __launch_bounds__(kMThreads, 1)
    mla_kernel(const __grid_constant__ MlaParams prm, const __grid_constant__ CUtensorMap kmap) {
  const DecodeArgs& a = prm.a;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int qt = blockIdx.x / a.n_splits, split = blockIdx.x % a.n_splits;
  const int nh = prm.pairs.n_heads[pair];
  const int rows_total = a.T * nh;
  if (qt * kMRows >= rows_total) return;             // whole CTA: nothing to do
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int list = prm.pairs.list_of[pair], kvh = prm.pairs.kvh_of[pair];

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  uint8_t* q_s = smem;
  uint8_t* k_s = smem + kQBytes;                              // kMStages tiles
  uint8_t* p_s = k_s + kMStages * kTileBytes;                 // 2 buffers
  __shared__ uint64_t kv_full[kMStages], kv_empty[kMStages];
  __shared__ uint64_t s_full[2], p_full[2], o_done, q_full;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, n_act_s;
  __shared__ int2 ent_s[kMMaxEnt];
  __shared__ int act_s[2 * kMMaxEnt];

  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * a.P) {
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
  const int r0 = qt * kMRows;
  if (n_ent == 0) {   // an empty split: its partial is O = 0, LSE = -inf
    const int nr = min(kMRows, rows_total - r0);
    for (int i = tid; i < nr * (kDv / 4); i += blockDim.x) {
      const int rr = r0 + i / (kDv / 4), c = (i % (kDv / 4)) * 4;
      const int t = rr / nh, head = prm.pairs.heads[pair][rr % nh];
      const int64_t orow = (((int64_t)split * a.B + b) * a.T + t) * a.Hq + head;
      *reinterpret_cast<float4*>(a.o_part + orow * kDv + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c == 0) a.lse_part[orow] = -INFINITY;
    }
    return;
  }
  const int t_last = (min(rows_total, r0 + kMRows) - 1) / nh;
  const int max_q = L - a.T + t_last;

  const int32_t* lrow = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list + e0;
  const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
  for (int i = tid; i < n_ent; i += kMThreads) {
    const int p = lrow[i];
    int ph = -1;
    if (p < 0 || p >= n_log) {
      set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    } else {
      ph = ptrow[p];
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        ph = -1;
      }
    }
    ent_s[i] = make_int2(ph, p * a.P);
  }
  if (tid == 0) {
    for (int s = 0; s < kMStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(&o_done, 1);
    mbar_init(&q_full, 128);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 5) tc::tmem_alloc(&tmem_base_s, kMTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  // tiles with at least one causally visible key, in list order
  const int n_tiles = (n_ent * a.P + kMKeys - 1) / kMKeys;
  if (warp == 0) {
    int n_act = 0;
    for (int j0 = 0; j0 < n_tiles; j0 += 32) {
      const int j = j0 + lane;
      bool live = false;
      if (j < n_tiles)
        for (int g = 0; g < 2; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          live |= gr.x >= 0 && gr.y < L && gr.y <= max_q;
        }
      const uint32_t m = __ballot_sync(0xffffffffu, live);
      if (live) act_s[n_act + __popc(m & ((1u << lane) - 1u))] = j;
      n_act += __popc(m);
    }
    if (lane == 0) n_act_s = n_act;
  }
  __syncthreads();
  const int n_act = n_act_s;
  volatile int* abort_flag = &abort_s;

  if (warp == 4) {
    // ================= producer: TMA gathers of key tiles (values alias them)
    if (lane == 0) {
      prefetch_tmap(&kmap);
      for (int jj = 0; jj < n_act; ++jj) {
        const int st = jj % kMStages;
        if (jj >= kMStages &&
            !wait_or_abort_m(&kv_empty[st], ((jj / kMStages) - 1) & 1, abort_flag))
          break;
        const int j = act_s[jj];
        uint8_t* kt = k_s + st * kTileBytes;
        mbar_arrive_expect_tx(&kv_full[st], kTileBytes);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          const bool ok = gr.x >= 0 && gr.y < L;
          const int page = ok ? gr.x : a.P_pool;     // out of range: zero-filled box
          const int row0 = ok ? gr.y % a.P : 0;
          for (int c = 0; c < kKC; ++c)
            tma_load_4d(kt + c * kChunkBytes + g * 2048, &kmap, &kv_full[st], c * 64, row0, kvh,
                        page);
        }
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer (one thread)
    if (lane == 0 && n_act > 0) {
      const uint32_t q_addr = smem_u32(q_s), k_addr = smem_u32(k_s), p_addr = smem_u32(p_s);
      auto pv = [&](int jp) -> bool {
        const int sb = jp & 1, st = jp % kMStages;
        if (!wait_or_abort_m(&p_full[sb], (jp >> 1) & 1, abort_flag)) return false;
        tc::fence_after_sync();
        const uint32_t kb = k_addr + st * kTileBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < kMKeys / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(p_addr + sb * kPBytes + kk * 32, 16, 1024);
            const uint64_t bd =
                tc::sdesc_sw128(kb + (4 * h) * kChunkBytes + kk * 2048, kChunkBytes, 1024);
            tc::mma_bf16(tmem + (h ? kHiLanes : 0u), ad, bd, kIdPV,
                         (jp > 0 || kk > 0) ? 1u : 0u);
          }
        tc::commit(&o_done);
        tc::commit(&kv_empty[st]);
        return true;
      };
      bool ok = wait_or_abort_m(&q_full, 0, abort_flag);
      tc::fence_after_sync();
      for (int jj = 0; ok && jj < n_act; ++jj) {
        const int st = jj % kMStages, sb = jj & 1;
        if (!wait_or_abort_m(&kv_full[st], (jj / kMStages) & 1, abort_flag)) break;
        tc::fence_after_sync();
        const uint32_t kb = k_addr + st * kTileBytes;
        for (int c = 0; c < kKC; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(q_addr + c * (kMRows * 128) + kk * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(kb + c * kChunkBytes + kk * 32, 16, 1024);
            tc::mma_bf16(tmem + kSCol + sb * kMKeys, ad, bd, kIdQK, (c | kk) ? 1u : 0u);
          }
        tc::commit(&s_full[sb]);
        if (jj >= 1 && !pv(jj - 1)) ok = false;
      }
      if (ok) pv(n_act - 1);
    }
  } else {
    // ================= softmax / epilogue
    // low lanes (l < 16): row 16w + l, keys and value columns 0-255;
    // high lanes: the same row's value columns 256-511
    const bool low = lane < 16;
    const int r = warp * 16 + (lane & 15);
    const int rg = r0 + r;
    const bool row_ok = rg < rows_total;
    const int t = row_ok ? rg / nh : 0;
    const int head = prm.pairs.heads[pair][row_ok ? rg % nh : 0];
    const int qpos = row_ok ? L - a.T + t : -1;
    {
      // query tile: 64 rows x 9 chunks of 128 bytes; two threads per row
      const int qr = tid >> 1, half = tid & 1;
      const int qrg = r0 + qr;
      const bool qok = qrg < rows_total;
      const int qt_ = qok ? qrg / nh : 0;
      const int qh = prm.pairs.heads[pair][qok ? qrg % nh : 0];
      const uint4* src = reinterpret_cast<const uint4*>(a.q + b * a.qs0 + qt_ * a.qs1 + qh * a.qs2);
      for (int ch = half * 36; ch < half * 36 + 36; ++ch) {
        const int c = ch >> 3, sub = ch & 7;
        const uint4 v = qok ? src[ch] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(q_s + c * (kMRows * 128) + qr * 128 + ((sub ^ (qr & 7)) << 4)) = v;
      }
    }
    tc::fence_proxy_async();
    mbar_arrive(&q_full);
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < n_act; ++jj) {
      const int sb = jj & 1, j = act_s[jj];
      if (!wait_or_abort_m(&s_full[sb], (jj >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float x[32];
      tc::ld32(tmem + lane_base + kSCol + sb * kMKeys, x);
      tc::wait_ld();
      float mx = -INFINITY;
      if (low) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          const bool gok = gr.x >= 0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int kp = gr.y + c;
            const bool vis = gok && kp < L && kp <= qpos;
            const float v = vis ? x[g * 16 + c] * a.scale_log2 : -INFINITY;
            x[g * 16 + c] = v;
            mx = fmaxf(mx, v);
          }
        }
      }
      mx = __shfl_sync(0xffffffffu, mx, lane & 15);   // the row's max, in both halves
      if (jj >= 1 && !wait_or_abort_m(&o_done, (jj - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const bool move = mx > m_ref + kLazyM;
      if (__any_sync(0xffffffffu, move)) {
        const float alpha = move ? exp2f(m_ref - mx) : 1.f;
        if (move) m_ref = mx;
        l *= alpha;
        if (jj >= 1) {
          for (int c = 0; c < 256 / 32; ++c) {
            float o[32];
            tc::ld32(tmem + lane_base + c * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::st32(tmem + lane_base + c * 32, o);
          }
          tc::wait_st();
        }
      }
      if (low) {
        const float base = m_ref == -INFINITY ? 0.f : m_ref;
        uint8_t* prow = p_s + sb * kPBytes + r * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float p[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            p[i] = exp2f(x[ch * 8 + i] - base);
            l += p[i];
          }
          uint4 w;
          w.x = pack_bf16(p[0], p[1]);
          w.y = pack_bf16(p[2], p[3]);
          w.z = pack_bf16(p[4], p[5]);
          w.w = pack_bf16(p[6], p[7]);
          *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) = w;
        }
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[sb]);
    }
    if (ok && n_act > 0) ok = wait_or_abort_m(&o_done, (n_act - 1) & 1, abort_flag);
    tc::fence_after_sync();
    l = __shfl_sync(0xffffffffu, l, lane & 15);
    const bool empty = !ok || n_act == 0 || l == 0.f;
    const float inv = empty ? 0.f : 1.f / l;
    const int64_t orow = (((int64_t)split * a.B + b) * a.T + t) * a.Hq + head;
    float* dst = a.o_part + orow * kDv + (low ? 0 : 256);
    for (int c = 0; c < 256 / 32; ++c) {
      float o[32];
      if (n_act > 0) {
        tc::ld32(tmem + lane_base + c * 32, o);
        tc::wait_ld();
      }
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dst + c * 32 + i) =
              empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                    : make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
      }
    }
    if (row_ok && low) a.lse_part[orow] = empty ? -INFINITY : (m_ref + log2f(l)) * kLn2;
    if (!ok && lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kMTmemCols);
  }
}

}  // namespace

int mla_max_split_entries(int P) { return min(kMMaxEnt, 2 * kMMaxEnt * kMKeys / P); }

cudaError_t launch_mla(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                       cudaStream_t stream) {
  MlaParams prm;
  prm.a = a;
  prm.pairs = pairs;
  int max_rows = 0;
  for (int i = 0; i < pairs.n_pairs; ++i) max_rows = max(max_rows, a.T * pairs.n_heads[i]);
  const int qtiles = (max_rows + kMRows - 1) / kMRows;
  cudaError_t e =
      cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMDyn);
  if (e != cudaSuccess) return e;
  dim3 grid(qtiles * a.n_splits, pairs.n_pairs, a.B);
  mla_kernel<<<grid, kMThreads, kMDyn, stream>>>(prm, kmap);
  return cudaGetLastError();
}

}  // namespace sa
