// Sparse attention over per-head page lists for many query rows per (list,
// kv head) pair — chunked prefill over block-union tables, long MTP — on the
// 5th-generation tensor cores.
//
// One CTA computes 256 query rows of a pair (token-major) as two 128-row tiles
// A and B against the keys of its split of the list, 64 keys per tile; each
// K/V tile is loaded once and used by both:
//   warp 8      gathers K and V tiles from the paged pool with TMA (four
//               16-key x 64-column boxes per 64-column chunk; an absent or
//               invalid 16-key group is loaded from an out-of-range page
//               coordinate, which TMA fills with zeros) into a 4-stage ring;
//   warp 9      issues tcgen05.mma, alternating between the tiles: S_A = Q_A K^T
//               and S_B = Q_B K^T (M=128, N=64, K=D) into double-buffered TMEM
//               S buffers, then O_A += P_A V and O_B += P_B V (M=128, N=D) into
//               TMEM with P read from TMEM as the A operand, with
//               tcgen05.commit arrivals on mbarriers;
//   warps 0-3 / 4-7   (one warpgroup per tile) own one query row per thread:
//               Q into shared memory, S rows from TMEM, masking (page validity,
//               sequence end, causal position; skipped for tiles every row sees
//               whole), a base-2 online softmax whose running max only moves when
//               a row's max exceeds it by more than 2^8 (the O rescale through
//               TMEM is then rare), P back into the S buffer it came from, and
//               the epilogue.
// P enters PV as a bf16 pair hi + lo (hi = RNE_bf16(p), lo = RNE_bf16(p - hi)),
// so its rounding is ~2^-17 relative rather than the 2^-9 of a single bf16: two
// MMAs per 16 keys, both reading the pair from the TMEM columns where that
// tile's scores were (64 keys = 32 columns of hi pairs + 32 of lo pairs).
// A softmax warpgroup computes P of tile j while the tensor core still runs
// PV of tile j-1 and QK^T of tile j+1; it waits for PV of tile j-1 only
// before handing P of tile j over (and before the rare rescale of O).
//
// Sources: CompactAttention (abstract on the page titled "Causal Attention on
// CPU: A Cache-Aware and Load-Balanced Scheduling Kernel for Prefill"):
// per-group KV block tables used in place; "Universal Attention Engine —
// Declarative Sparse Attention for Production", "Key Design Decisions" 3:
// prefill is compute-bound, so the FLOPs go to the tensor cores.
#include "common.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace sa {
namespace {

constexpr int kPThreads = 320;    // 2 softmax warpgroups, producer warp, MMA warp
constexpr int kPStages = 4;
constexpr int kKeys = 64;         // keys per tile
constexpr int kM = 128;           // query rows per warpgroup tile
constexpr int kRows = 2 * kM;     // query rows per CTA
constexpr int kMaxEnt = 1024;     // list entries per split
constexpr float kLazyP = 8.f;

template <int D>
struct PCfg {
  static constexpr int kChunks = D / 64;               // 64-column (128-byte) chunks
  static constexpr int kQBytes = kM * D * 2;
  static constexpr int kTileBytes = kKeys * D * 2;     // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kDyn = 2 * kQBytes + kPStages * kStageBytes + 1024;
  // per tile w: S buffers at 128w + {0, 64} (P hi + lo after the softmax:
  // columns +0..31 and +32..63), O at 256 + 128w
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdQK = tc::idesc_bf16_f32(kM, kKeys, false, false);
  static constexpr uint32_t kIdPV = tc::idesc_bf16_f32(kM, D, false, true);
};

struct __align__(64) PrefillParams {
  DecodeArgs a;
  PairTable pairs;
};

// Bounded wait that also gives up as soon as another role has aborted.
SA_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

// (physical page or -1, first token) of 16-key group g of tile j.
SA_DEV int2 group_of(const int2* ent, int n_ent, int P, int j, int g) {
  int e, row0;
  if (P <= kKeys) {
    const int per = kKeys / P;                 // entries per tile
    e = j * per + (g * 16) / P;
    row0 = (g * 16) % P;
  } else {
    const int per = P / kKeys;                 // tiles per entry
    e = j / per;
    row0 = (j % per) * kKeys + g * 16;
  }
  if (e >= n_ent) return make_int2(-1, 0);
  const int2 en = ent[e];
  return make_int2(en.x, en.y + row0);
}

template <int D>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams prm,
                   const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  pdl_wait_and_release();
  using C = PCfg<D>;
  const DecodeArgs& a = prm.a;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int qt = blockIdx.x / a.n_splits, split = blockIdx.x % a.n_splits;
  const int nh = prm.pairs.n_heads[pair];
  const int rows_total = a.T * nh;
  if (qt * kRows >= rows_total) return;               // whole CTA: nothing to do
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int list = prm.pairs.list_of[pair], kvh = prm.pairs.kvh_of[pair];

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  uint8_t* q_s = smem;                                       // 2 tiles
  uint8_t* kv_s = smem + 2 * C::kQBytes;                     // kPStages x (K | V)
  __shared__ uint64_t kv_full[kPStages], kv_empty[kPStages];
  __shared__ uint64_t s_full[2][2], p_full[2], o_done[2], q_full;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, n_act_s;
  __shared__ int2 ent_s[kMaxEnt];
  __shared__ int act_s[kMaxEnt];     // (tile << 1) | needs_mask

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
  // split s holds entries [s c, (s + 1) c) of the list, c = ceil(max_list / n_splits)
  const int chunk = (a.max_list + a.n_splits - 1) / a.n_splits;
  const int e0 = min(split * chunk, count);
  const int n_ent = min(chunk, count - e0);
  const int r0 = qt * kRows;
  if (n_ent == 0) {   // an empty split: its partial is O = 0, LSE = -inf
    const int nr = min(kRows, rows_total - r0);
    for (int i = tid; i < nr * (D / 4); i += blockDim.x) {
      const int rr = r0 + i / (D / 4), c = (i % (D / 4)) * 4;
      const int t = rr / nh, head = prm.pairs.heads[prm.pairs.head_off[pair] + (rr % nh)];
      const int64_t orow = (((int64_t)split * a.B + b) * a.T + t) * a.Hq + head;
      *reinterpret_cast<float4*>(a.o_part + orow * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c == 0) a.lse_part[orow] = -INFINITY;
    }
    return;
  }
  const int t_first = r0 / nh;
  const int t_last = (min(rows_total, r0 + kRows) - 1) / nh;
  const int qb = query_base(a, b, L);
  const int min_q = qb + t_first, max_q = qb + t_last;

  // ---- resolve pages, set up barriers and TMEM
  const int32_t* lrow = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list + e0;
  for (int i = tid; i < n_ent; i += kPThreads) {
    const int p = lrow[i];
    int ph = -1;
    if (p < 0 || p >= n_log) {
      set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
    } else {
      ph = page_at(a.pt, b, p);
      if (ph < 0 || ph >= a.P_pool) {
        set_dev_error(a.err, SA_DEVERR_POOL_RANGE);
        ph = -1;
      }
    }
    ent_s[i] = make_int2(ph, p * a.P);
  }
  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w][0], 1);
      mbar_init(&s_full[w][1], 1);
      mbar_init(&p_full[w], 128);
      mbar_init(&o_done[w], 1);
    }
    mbar_init(&q_full, 256);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 9) tc::tmem_alloc(&tmem_base_s, C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  // ---- tiles with at least one causally visible key, in list order; a tile
  // every row of the CTA sees whole (all groups valid and below min_q) skips
  // the per-element mask
  const int n_tiles = a.P <= kKeys ? (n_ent * a.P + kKeys - 1) / kKeys : n_ent * (a.P / kKeys);
  if (warp == 0) {
    int n_act = 0;
    for (int j0 = 0; j0 < n_tiles; j0 += 32) {
      const int j = j0 + lane;
      bool live = false, whole = true;
      if (j < n_tiles)
        for (int g = 0; g < 4; ++g) {
          const int2 gr = group_of(ent_s, n_ent, a.P, j, g);
          live |= gr.x >= 0 && gr.y < L && gr.y <= max_q;
          whole &= gr.x >= 0 && gr.y + 15 < L && gr.y + 15 <= min_q;
        }
      const uint32_t m = __ballot_sync(0xffffffffu, live);
      if (live) act_s[n_act + __popc(m & ((1u << lane) - 1u))] = (j << 1) | (whole ? 0 : 1);
      n_act += __popc(m);
    }
    if (lane == 0) n_act_s = n_act;
  }
  __syncthreads();
  const int n_act = n_act_s;
  volatile int* abort_flag = &abort_s;

  if (warp == 8) {
    // ================= producer: TMA gathers of K and V tiles
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
      for (int jj = 0; jj < n_act; ++jj) {
        const int st = jj % kPStages;
        if (jj >= kPStages &&
            !wait_or_abort(&kv_empty[st], ((jj / kPStages) - 1) & 1, abort_flag))
          break;
        const int j = act_s[jj] >> 1;
        uint8_t* kt = kv_s + st * C::kStageBytes;
        uint8_t* vt = kt + C::kTileBytes;
        mbar_arrive_expect_tx(&kv_full[st], C::kStageBytes);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int2 gr = group_of(ent_s, n_ent, a.P, j, g);
          const bool ok = gr.x >= 0 && gr.y < L;
          // an out-of-range page coordinate makes TMA write zeros for the box
          const int page = ok ? gr.x : a.P_pool;
          const int row0 = ok ? gr.y % a.P : 0;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            tma_load_4d(kt + c * (kKeys * 128) + g * 2048, &kmap, &kv_full[st], c * 64, row0, kvh,
                        page);
            tma_load_4d(vt + c * (kKeys * 128) + g * 2048, &vmap, &kv_full[st], c * 64, row0, kvh,
                        page);
          }
        }
      }
    }
  } else if (warp == 9) {
    // ================= MMA issuer (one thread), alternating tiles A and B
    if (lane == 0 && n_act > 0) {
      const uint32_t q_addr = smem_u32(q_s), kv_addr = smem_u32(kv_s);
      // O_w += P_w V for tile jp: P (hi, then lo) from the TMEM columns of the
      // S buffer the tile's scores were in.  QK^T of tile jp + 2, issued after
      // this, reuses those columns: MMAs of one thread execute in issue order.
      auto pv = [&](int jp) -> bool {
        const int st = jp % kPStages;
        const uint32_t vbase = kv_addr + st * C::kStageBytes + C::kTileBytes;
        for (int w = 0; w < 2; ++w) {
          if (!wait_or_abort(&p_full[w], jp & 1, abort_flag)) return false;
          tc::fence_after_sync();
          const uint32_t pcol = tmem + 128 * w + (jp & 1) * kKeys;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            const uint64_t bd = tc::sdesc_sw128(vbase + kk * 2048, kKeys * 128, 1024);
            tc::mma_bf16_ts(tmem + 256 + 128 * w, pcol + 8 * kk, bd, C::kIdPV,
                            (jp > 0 || kk > 0) ? 1u : 0u);
            tc::mma_bf16_ts(tmem + 256 + 128 * w, pcol + 32 + 8 * kk, bd, C::kIdPV, 1u);
          }
          tc::commit(&o_done[w]);
        }
        tc::commit(&kv_empty[st]);
        return true;
      };
      bool ok = wait_or_abort(&q_full, 0, abort_flag);
      tc::fence_after_sync();
      for (int jj = 0; ok && jj < n_act; ++jj) {
        const int st = jj % kPStages, sb = jj & 1;
        if (!wait_or_abort(&kv_full[st], (jj / kPStages) & 1, abort_flag)) break;
        tc::fence_after_sync();
        const uint32_t kbase = kv_addr + st * C::kStageBytes;
        for (int w = 0; w < 2; ++w) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(
                q_addr + w * C::kQBytes + (kk >> 2) * (kM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd =
                tc::sdesc_sw128(kbase + (kk >> 2) * (kKeys * 128) + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem + 128 * w + sb * kKeys, ad, bd, C::kIdQK, kk > 0 ? 1u : 0u);
          }
          tc::commit(&s_full[w][sb]);
        }
        if (jj >= 1 && !pv(jj - 1)) ok = false;
      }
      if (ok) pv(n_act - 1);
    }
  } else {
    // ================= softmax / epilogue: one query row per thread
    const int wg = warp >> 2;                       // tile A (0) or B (1)
    const int r = (warp & 3) * 32 + lane;           // row within the tile = TMEM lane
    const int rg = r0 + wg * kM + r;
    const bool row_ok = rg < rows_total;
    const int t = row_ok ? rg / nh : 0;
    const int head = prm.pairs.heads[prm.pairs.head_off[pair] + (row_ok ? rg % nh : 0)];
    const int qpos = row_ok ? qb + t : -1;
    uint8_t* qt_s = q_s + wg * C::kQBytes;
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + b * a.qs0 + t * a.qs1 + head * a.qs2);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = row_ok ? src[c * 8 + ch] : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(qt_s + c * (kM * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
        }
    }
    tc::fence_proxy_async();
    mbar_arrive(&q_full);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = 128 * wg, o_col = 256 + 128 * wg;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < n_act; ++jj) {
      const int sb = jj & 1, code = act_s[jj], j = code >> 1;
      if (!wait_or_abort(&s_full[wg][sb], (jj >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float x[64];
      tc::ld32(tmem + lane_base + s_col + sb * kKeys, *reinterpret_cast<float(*)[32]>(&x[0]));
      tc::ld32(tmem + lane_base + s_col + sb * kKeys + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
      tc::wait_ld();
      // the row max of the scaled scores from the raw ones: x -> x s is monotone
      // (rounding included), so it is s max(x) for s >= 0 and s min(x) for s < 0;
      // invisible keys are NaN here (ignored by the reduction, p = 0 below)
      const float sl = a.scale_log2;
      const bool masked = code & 1;
      if (masked) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int2 gr = group_of(ent_s, n_ent, a.P, j, g);
          const bool gok = gr.x >= 0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int kp = gr.y + c;
            if (!(gok && kp < L && kp <= qpos)) x[g * 16 + c] = NAN;
          }
        }
      }
      const float mr = sl >= 0.f ? reduce_n<false>(x) : reduce_n<true>(x);
      const float mx = mr != mr ? -INFINITY : mr * sl;
      const bool move = mx > m_ref + kLazyP;
      const float m_new = move ? mx : m_ref;
      const float nb = m_new == -INFINITY ? 0.f : -m_new;
      // P = 2^(x sl - m_new) as bf16 hi + lo pairs, written over this tile's
      // scores in TMEM (the S buffer is free: QK^T of the tile is complete and
      // PV of tile jj - 2, the buffer's previous reader, completed before it)
      // (key pairs in packed float32: the same roundings as the scalar ops,
      // half the instructions; the row sum in eight independent chains)
      unsigned long long ls2[4] = {0ull, 0ull, 0ull, 0ull};
      const unsigned long long sl2 = f2_pack(sl, sl), nb2 = f2_pack(nb, nb);
      uint32_t ph[32], pl[32];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float v0 = x[ch * 8 + 2 * i], v1 = x[ch * 8 + 2 * i + 1];
          const float2 z = f2_unpack(f2_fma(f2_pack(v0, v1), sl2, nb2));
          float p0 = ex2_approx(z.x), p1 = ex2_approx(z.y);
          if (masked) {
            p0 = v0 == v0 ? p0 : 0.f;
            p1 = v1 == v1 ? p1 : 0.f;
          }
          const unsigned long long pp = f2_pack(p0, p1);
          ls2[i] = f2_add(ls2[i], pp);
          const uint32_t h = pack_bf16(p0, p1);
          const float2 d = f2_unpack(f2_sub(
              pp, f2_pack(__uint_as_float(h << 16), __uint_as_float(h & 0xffff0000u))));
          ph[ch * 4 + i] = h;
          pl[ch * 4 + i] = pack_bf16(d.x, d.y);
        }
      }
      float ls[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = f2_unpack(ls2[i]);
        ls[2 * i] = v.x;
        ls[2 * i + 1] = v.y;
      }
      tc::st32(tmem + lane_base + s_col + sb * kKeys, *reinterpret_cast<float(*)[32]>(ph));
      tc::st32(tmem + lane_base + s_col + sb * kKeys + 32, *reinterpret_cast<float(*)[32]>(pl));
      tc::wait_st();
      // PV(jj-1) must be done before O is rescaled and before P(jj) is handed
      // over (its completion also keeps this barrier's phases in step)
      if (jj >= 1 && !wait_or_abort(&o_done[wg], (jj - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      if (__any_sync(0xffffffffu, move)) {
        const float alpha = move ? exp2f(m_ref - mx) : 1.f;
        l *= alpha;
        if (jj >= 1) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tc::ld32(tmem + lane_base + o_col + c * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::st32(tmem + lane_base + o_col + c * 32, o);
          }
          tc::wait_st();
        }
      }
      m_ref = m_new;
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      tc::fence_before_sync();
      mbar_arrive(&p_full[wg]);
    }
    if (ok && n_act > 0) ok = wait_or_abort(&o_done[wg], (n_act - 1) & 1, abort_flag);
    tc::fence_after_sync();
    // ---- epilogue: O / l and LSE for this row
    const bool empty = !ok || n_act == 0 || l == 0.f;
    const float inv = empty ? 0.f : 1.f / l;
    float* dst = a.o_part + ((((int64_t)split * a.B + b) * a.T + t) * a.Hq + head) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      if (n_act > 0) {
        tc::ld32(tmem + lane_base + o_col + c * 32, o);
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
    if (row_ok)
      a.lse_part[(((int64_t)split * a.B + b) * a.T + t) * a.Hq + head] =
          empty ? -INFINITY : (m_ref + log2f(l)) * kLn2;
    if (!ok && lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t launch_p(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                     const CUtensorMap& vmap, cudaStream_t stream) {
  using C = PCfg<D>;
  PrefillParams prm;
  prm.a = a;
  prm.pairs = pairs;
  int max_rows = 0;
  for (int i = 0; i < pairs.n_pairs; ++i) max_rows = max(max_rows, a.T * pairs.n_heads[i]);
  const int qtiles = (max_rows + kRows - 1) / kRows;
  cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(prefill_kernel<D>));
  if (e != cudaSuccess) return e;
  dim3 grid(qtiles * a.n_splits, pairs.n_pairs, a.B);
  return launch_pdl(prefill_kernel<D>, grid, dim3(kPThreads), C::kDyn, stream, prm, kmap, vmap);
}

}  // namespace

int prefill_max_split_entries() { return kMaxEnt; }

cudaError_t launch_prefill(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, cudaStream_t stream) {
  switch (a.Dk) {
    case 64: return launch_p<64>(a, pairs, kmap, vmap, stream);
    case 128: return launch_p<128>(a, pairs, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
