// Gather-based split-KV Flash-decode over per-head page lists (GQA / MTP).
//
// The unit of work is a 16-token sub-page of one (list, kv head) pair: its K
// and V arrive by TMA tile loads (64-column x 16-row boxes, 128-byte swizzle;
// FP8 pages: one 128-column box) straight from the paged pool, and one warp
// folds it into an online-softmax state with m16n8k16 tensor-core MMAs: the 16
// MMA rows are the query rows of the pair (T x heads), the columns the 16
// tokens.  Probabilities enter PV as a hi + lo pair so their rounding stays
// ~2^-17 relative; the running max moves only when a row's maximum exceeds it
// by more than 2^8 (so P <= 256 and the O rescale is rare).  One warp takes one
// split of one pair: it resolves its pages, keeps a private two-stage ring of
// units and writes its split's partial from registers.
//
// Sources: "Universal Attention Engine — Declarative Sparse Attention for
// Production" ("Architecture": gather-based sparse KV decode; "Key Design
// Decisions" 3: decode is memory-bound, optimise bytes loaded) and "TileSparse"
// ("Two implementations": a per-head page-list Flash-decode kernel).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

// Diagnostic build (-DSA_DECODE_TIMELINE=1, off in the library): each warp's
// first work item records %globaltimer stamps -- entry, list entries read,
// pages resolved, its first unit computed, each of its first 8 units' data
// arriving, partial stored --
// plus its SM, item and unit count, read back with sa_decode_timeline().
#ifndef SA_DECODE_TIMELINE
#define SA_DECODE_TIMELINE 0
#endif

namespace sa {
#if SA_DECODE_TIMELINE
constexpr int kTlWarps = 8192, kTlSlots = 16;
__device__ unsigned long long g_decode_tl[kTlWarps * kTlSlots];
#endif
namespace {

#if SA_DECODE_TIMELINE
SA_DEV unsigned long long tl_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define SA_TL(slot, value)                                              \
  do {                                                                  \
    if (tl_row >= 0 && lane == 0) g_decode_tl[tl_row + (slot)] = (value); \
  } while (0)
#else
#define SA_TL(slot, value) \
  do {                     \
  } while (0)
#endif

// Build-time shape of a CTA: warps (= splits) per CTA and ring stages per warp.
#ifndef SA_DECODE_WARPS
#define SA_DECODE_WARPS 4
#endif
#ifndef SA_DECODE_STAGES
#define SA_DECODE_STAGES 2
#endif
#ifndef SA_DECODE_STAGES_F8
#define SA_DECODE_STAGES_F8 2
#endif
constexpr int kNW = SA_DECODE_WARPS;
constexpr int kSub = 16;            // tokens per TMA sub-page (one MMA k-step of PV)
constexpr int kWarpEntries = 128;   // list entries one split may hold
constexpr float kLazy = 8.f;        // log2 headroom before the running max moves

// F8: pages hold FP8 E4M3 codes (one byte per element) with a float32 scale per
// (page, kv head); a sub-page arrives as one 128-column box.  The MMAs run in
// f16 (E4M3 -> f16 is one exact instruction per pair): K fragments straight
// from the code tile, V through an f16 staging tile.
template <int D, bool F8 = false>
struct DecodeCfg {
  static_assert(!F8 || D == 128, "FP8 pages: D == 128");
  static constexpr int kBoxes = D / 64;                     // 64-column bf16 boxes per row set
  static constexpr int kBoxBytes = kSub * 128;              // 16 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;     // one bf16 K (or V) sub-page
  static constexpr int kInTile = F8 ? kSub * D : kTileBytes;   // one sub-page as stored
  static constexpr int kStageBytes = 2 * kInTile;           // K + V
  static constexpr int kStages = F8 ? SA_DECODE_STAGES_F8 : (D >= 128 ? SA_DECODE_STAGES : 2 * SA_DECODE_STAGES);
  static constexpr int kWarpBytes = kStages * kStageBytes + (F8 ? kTileBytes : 0);
  static constexpr int kDynBytes = kNW * kWarpBytes + 1024;
};

// One FP8 sub-page (16 rows x 128 codes, 128-byte swizzle) -> f16 in the
// layout of two 64-column swizzled boxes (what the bf16 path's ldmatrix reads).
// Lane l takes row l / 2 and columns 64 (l % 2) .. + 63: four 16-byte code
// chunks in, eight 16-byte f16 chunks out.
SA_DEV void widen_fp8_tile(const uint8_t* src, uint8_t* dst, int lane) {
  const int t = lane >> 1, hb = lane & 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = 4 * hb + i;
    const uint4 c = *reinterpret_cast<const uint4*>(src + t * 128 + (((j ^ t) & 7) << 4));
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint4 o0, o1;
    o0.x = e4m3x2_to_f16x2(w[0]);
    o0.y = e4m3x2_to_f16x2(w[0] >> 16);
    o0.z = e4m3x2_to_f16x2(w[1]);
    o0.w = e4m3x2_to_f16x2(w[1] >> 16);
    o1.x = e4m3x2_to_f16x2(w[2]);
    o1.y = e4m3x2_to_f16x2(w[2] >> 16);
    o1.z = e4m3x2_to_f16x2(w[3]);
    o1.w = e4m3x2_to_f16x2(w[3] >> 16);
    uint8_t* box = dst + hb * (kSub * 128) + t * 128;
    *reinterpret_cast<uint4*>(box + ((((2 * i) ^ t) & 7) << 4)) = o0;
    *reinterpret_cast<uint4*>(box + ((((2 * i + 1) ^ t) & 7) << 4)) = o1;
  }
}

struct __align__(64) DecodeParams {
  DecodeArgs a;
  PairTable pairs;
};

// ---------------------------------------------------------------------------
// Per-warp pieces shared by both kernels: the query fragments of a pair's rows,
// one 16-token unit folded into the online-softmax state, the normalised
// partial of the state.  MMA row r of a pair is query token r / nh, head
// number r % nh of the pair; lane (gid, tig) holds rows gid and gid + 8.
// ---------------------------------------------------------------------------
template <int D>
struct RowState {
  float o[D / 8][4];
  float m_ref[2];   // base-2 reference max per row
  float l_run[2];   // sum of p (the lane's columns; reduced over the quad at the end)
};

template <int D>
SA_DEV void state_clear(RowState<D>& st) {
#pragma unroll
  for (int i = 0; i < D / 8; ++i) st.o[i][0] = st.o[i][1] = st.o[i][2] = st.o[i][3] = 0.f;
  st.m_ref[0] = st.m_ref[1] = -INFINITY;
  st.l_run[0] = st.l_run[1] = 0.f;
}

// Query fragments (A operand of QK^T) of the pair's rows; qt[h] = the query
// token of row gid + 8h, or -1 past the pair's R rows.  FP8: f16 fragments in a
// permuted feature order (k-slots (2 tig, 2 tig + 1) and (2 tig + 8, 2 tig + 9)
// of step kk hold features 16 kk + 4 tig + 0..3), so a key fragment is one
// 4-byte code load; the same permutation on both operands leaves every dot
// product unchanged.  A query value beyond the f16 range sets
// SA_DEVERR_VALUE_RANGE.
template <int D, bool F8>
SA_DEV void load_q_frags(uint32_t (&qa)[D / 16][4], int (&qt)[2], const DecodeArgs& a,
                         const PairTable& pr, int pair, int b, int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  const int nh = pr.n_heads[pair], R = a.T * nh;
  const int rows[2] = {gid, gid + 8};
  const uint16_t* qp[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rows[h];
    qt[h] = r < R ? r / nh : -1;
    qp[h] = r < R ? a.q + b * a.qs0 + qt[h] * a.qs1 + pr.heads[pr.head_off[pair] + (r % nh)] * a.qs2
                  : nullptr;
  }
  if constexpr (F8) {
    bool big = false;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 4 * tig;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 x = qp[h] ? *reinterpret_cast<const uint2*>(qp[h] + c) : make_uint2(0u, 0u);
        const float f0 = bf16_bits_to_float(x.x & 0xffffu), f1 = bf16_bits_to_float(x.x >> 16);
        const float f2 = bf16_bits_to_float(x.y & 0xffffu), f3 = bf16_bits_to_float(x.y >> 16);
        big |= fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3))) > 65504.f;
        qa[kk][h] = pack_f16(f0, f1);
        qa[kk][2 + h] = pack_f16(f2, f3);
      }
    }
    if (big) set_dev_error(a.err, SA_DEVERR_VALUE_RANGE);
  } else {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * tig;
      qa[kk][0] = qp[0] ? *reinterpret_cast<const uint32_t*>(qp[0] + c) : 0u;
      qa[kk][1] = qp[1] ? *reinterpret_cast<const uint32_t*>(qp[1] + c) : 0u;
      qa[kk][2] = qp[0] ? *reinterpret_cast<const uint32_t*>(qp[0] + c + 8) : 0u;
      qa[kk][3] = qp[1] ? *reinterpret_cast<const uint32_t*>(qp[1] + c + 8) : 0u;
    }
  }
}

// Fold one 16-token unit into the state: K tile at kt, V tile at kt + kInTile
// (as the TMA boxes wrote them), tokens tok0 .. tok0 + 15; a token is visible to
// row h when it is below L and at most lim[h].  sl = scale log2(e); ksc scales
// the scores (FP8 key scale, else 1); vsc scales P before PV (FP8 value scale
// over the state's reference, else 1).  FP8 widens the V codes into the warp's
// f16 staging tile `wide` first.
template <int D, bool F8>
SA_DEV void attend_unit(RowState<D>& st, const uint32_t (&qa)[D / 16][4], const uint8_t* kt,
                        uint8_t* wide, int tok0, int L, const int (&lim)[2], float sl, float ksc,
                        float vsc, int lane) {
  using C = DecodeCfg<D, F8>;
  const int gid = lane >> 2, tig = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  uint32_t kbase = smem_u32(kt), vbase = smem_u32(kt + C::kTileBytes);
  if constexpr (F8) {
    widen_fp8_tile(kt + C::kInTile, wide, lane);
    __syncwarp();
    vbase = smem_u32(wide);
  }
  // ---- S = Q K^T (16 rows x 16 tokens): 4 independent accumulation chains
  float s4[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) s4[i][0] = s4[i][1] = s4[i][2] = s4[i][3] = 0.f;
  if constexpr (F8) {
    // key fragments straight from the code tile: token rows gid and gid + 8
    // (both with swizzle row gid), 4 codes per lane per k-step
    const uint8_t* k8 = kt + gid * 128 + 4 * tig;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t w0 = *reinterpret_cast<const uint32_t*>(k8 + ((kk ^ gid) << 4));
      const uint32_t w1 = *reinterpret_cast<const uint32_t*>(k8 + 8 * 128 + ((kk ^ gid) << 4));
      mma_f16_16816(s4[kk & 1], qa[kk], e4m3x2_to_f16x2(w0), e4m3x2_to_f16x2(w0 >> 16));
      mma_f16_16816(s4[2 + (kk & 1)], qa[kk], e4m3x2_to_f16x2(w1), e4m3x2_to_f16x2(w1 >> 16));
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int colb = (kk & 3) * 16;
      const uint32_t addr =
          kbase + (kk >> 2) * C::kBoxBytes + swz128(8 * (mi >> 1) + ri, colb + 8 * (mi & 1));
      uint32_t r[4];
      ldmatrix_x4(r, addr);
      mma_bf16_16816(s4[kk & 1], qa[kk], r[0], r[1]);
      mma_bf16_16816(s4[2 + (kk & 1)], qa[kk], r[2], r[3]);
    }
  }
  float s[2][4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    s[0][c] = s4[0][c] + s4[1][c];
    s[1][c] = s4[2][c] + s4[3][c];
  }
  // ---- mask, lazily re-based online softmax (base 2)
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int h = c >> 1;
      const int pos = tok0 + nt * 8 + 2 * tig + (c & 1);
      const bool ok = pos < L && pos <= lim[h];
      s[nt][c] = ok ? s[nt][c] * (sl * ksc) : -INFINITY;
      mx[h] = fmaxf(mx[h], s[nt][c]);
    }
  bool move[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    move[h] = mx[h] > st.m_ref[h] + kLazy;
  }
  if (__any_sync(0xffffffffu, move[0] || move[1])) {
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      alpha[h] = move[h] ? exp2f(st.m_ref[h] - mx[h]) : 1.f;
      if (move[h]) st.m_ref[h] = mx[h];
      st.l_run[h] *= alpha[h];
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      st.o[i][0] *= alpha[0];
      st.o[i][1] *= alpha[0];
      st.o[i][2] *= alpha[1];
      st.o[i][3] *= alpha[1];
    }
  }
  const float base[2] = {st.m_ref[0] == -INFINITY ? 0.f : st.m_ref[0],
                         st.m_ref[1] == -INFINITY ? 0.f : st.m_ref[1]};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      s[nt][c] = exp2f(s[nt][c] - base[c >> 1]);
      st.l_run[c >> 1] += s[nt][c];
    }
  // ---- O += P V with P = hi + lo (both bf16; FP8: both f16, the value scale
  // riding on P while the denominator l_run does not)
  uint32_t ph_[4], pl_[4];
  {
    const float pv[4][2] = {{s[0][0] * vsc, s[0][1] * vsc}, {s[0][2] * vsc, s[0][3] * vsc},
                            {s[1][0] * vsc, s[1][1] * vsc}, {s[1][2] * vsc, s[1][3] * vsc}};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (F8) {
        ph_[i] = pack_f16(pv[i][0], pv[i][1]);
        const float h0 = f16_bits_to_float(ph_[i] & 0xffffu);
        const float h1 = f16_bits_to_float(ph_[i] >> 16);
        pl_[i] = pack_f16(pv[i][0] - h0, pv[i][1] - h1);
      } else {
        ph_[i] = pack_bf16(pv[i][0], pv[i][1]);
        const float h0 = bf16_bits_to_float(ph_[i] & 0xffffu);
        const float h1 = bf16_bits_to_float(ph_[i] >> 16);
        pl_[i] = pack_bf16(pv[i][0] - h0, pv[i][1] - h1);
      }
    }
  }
#pragma unroll
  for (int n2 = 0; n2 < D / 16; ++n2) {
    const int colb = (n2 & 3) * 16;
    const uint32_t addr =
        vbase + (n2 >> 2) * C::kBoxBytes + swz128(8 * (mi & 1) + ri, colb + 8 * (mi >> 1));
    uint32_t r[4];
    ldmatrix_x4_trans(r, addr);
    if constexpr (F8) {
      mma_f16_16816(st.o[2 * n2], ph_, r[0], r[1]);
      mma_f16_16816(st.o[2 * n2 + 1], ph_, r[2], r[3]);
      mma_f16_16816(st.o[2 * n2], pl_, r[0], r[1]);
      mma_f16_16816(st.o[2 * n2 + 1], pl_, r[2], r[3]);
    } else {
      mma_bf16_16816(st.o[2 * n2], ph_, r[0], r[1]);
      mma_bf16_16816(st.o[2 * n2 + 1], ph_, r[2], r[3]);
      mma_bf16_16816(st.o[2 * n2], pl_, r[0], r[1]);
      mma_bf16_16816(st.o[2 * n2 + 1], pl_, r[2], r[3]);
    }
  }
}

// The state's normalised rows (O * v_ref / l, LSE) into partial slot `slot` of
// the pair's rows; a row without a visible key gets O = 0 and LSE = -inf.
template <int D>
SA_DEV void store_partial(RowState<D>& st, const DecodeArgs& a, const PairTable& pr, int pair,
                          int b, int slot, float v_ref, int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  const int nh = pr.n_heads[pair], R = a.T * nh;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    st.l_run[h] += __shfl_xor_sync(0xffffffffu, st.l_run[h], 1);
    st.l_run[h] += __shfl_xor_sync(0xffffffffu, st.l_run[h], 2);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = gid + 8 * h;
    if (r >= R) continue;
    const int t = r / nh, head = pr.heads[pr.head_off[pair] + (r % nh)];
    const int64_t row = (((int64_t)slot * a.B + b) * a.T + t) * a.Hq + head;
    const bool empty = st.l_run[h] == 0.f;
    const float inv = empty ? 0.f : v_ref / st.l_run[h];
    float* dst = a.o_part + row * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
      *reinterpret_cast<float2*>(dst + i * 8 + 2 * tig) =
          make_float2(st.o[i][2 * h] * inv, st.o[i][2 * h + 1] * inv);
    if (tig == 0)
      a.lse_part[row] = empty ? -INFINITY : (st.m_ref[h] + log2f(st.l_run[h])) * kLn2;
  }
}

// ---------------------------------------------------------------------------
// Split kernel: one warp per split of one (list, kv head) pair of one sequence
// ---------------------------------------------------------------------------
template <int D, bool F8>
__global__ void __launch_bounds__(kNW * 32, D <= 128 ? 3 : 1)
    decode_gqa_kernel(const __grid_constant__ DecodeParams prm,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
  pdl_wait_and_release();
  using C = DecodeCfg<D, F8>;
  const DecodeArgs& a = prm.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#if SA_DECODE_TIMELINE
  const unsigned long long tl_t0 = tl_now();
  const int tl_gw = blockIdx.x * kNW + warp;
  int tl_row = tl_gw < kTlWarps ? tl_gw * kTlSlots : -1;
  SA_TL(0, tl_t0);
#endif

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  __shared__ uint64_t bars[kNW][C::kStages];
  __shared__ int2 ent_s[kNW][kWarpEntries];    // (physical page, first token) per entry
  __shared__ float2 scl_s[F8 ? kNW : 1][F8 ? kWarpEntries : 1];   // FP8: (k, v) scale per entry

  if (lane == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(&bars[warp][s], 1);
    fence_mbar_init();
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  __syncwarp();
  // Work items are (split, pair, sequence) triples, flattened; each warp takes
  // items warp_id, warp_id + total_warps, ... so that every SM gets the same
  // share whatever the grid's shape.  The ring's unit counter `base` runs on
  // across items, which keeps the mbarrier phases in step.
  const int n_items = a.n_splits * prm.pairs.n_pairs * a.B;
  const int total_warps = gridDim.x * kNW;
  uint8_t* ring = smem + warp * C::kWarpBytes;
  uint8_t* wide = ring + C::kStages * C::kStageBytes;   // FP8: the f16 V staging tile
  int base = 0;
  for (int item = blockIdx.x * kNW + warp; item < n_items; item += total_warps) {
    const int split = item % a.n_splits;
    const int pair = (item / a.n_splits) % prm.pairs.n_pairs;
    const int b = item / (a.n_splits * prm.pairs.n_pairs);
    const int list = prm.pairs.list_of[pair];
    const int kvh = prm.pairs.kvh_of[pair];
    // The loads that depend on nothing but the item go out together: the
    // sequence length, the list count and the split's list entries (read up to
    // the split's capacity; only those below the count are used).  The
    // page-table lookups follow in a second round, the query fragments after
    // the first key/value gathers are issued.
    // split s holds entries [s c, (s + 1) c) of the list, c = ceil(max_list / n_splits)
    const int chunk = (a.max_list + a.n_splits - 1) / a.n_splits;
    const int s0 = split * chunk;
    const int32_t* lbase = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list;
    int pre[kWarpEntries / 32];
#pragma unroll
    for (int j = 0; j < kWarpEntries / 32; ++j) {
      const int i = lane + 32 * j;
      pre[j] = (i < chunk && s0 + i < a.max_list) ? lbase[s0 + i] : -1;
    }
    int L = a.seq_lens[b];
    int count = a.counts[b * a.n_lists + list];
    if (L < 0 || L > a.max_pages * a.P) {  // a length the page table cannot hold
      if (lane == 0) set_dev_error(a.err, SA_DEVERR_PAGE_RANGE);
      L = L < 0 ? 0 : a.max_pages * a.P;
    }
    const int n_log = (L + a.P - 1) / a.P;
    if (count < 0 || count > a.max_list) {
      if (lane == 0) set_dev_error(a.err, SA_DEVERR_COUNT);
      count = count < 0 ? 0 : a.max_list;
    }
    const int e0 = min(s0, count);
    const int n_ent = min(chunk, count - e0);
#if SA_DECODE_TIMELINE
    SA_TL(1, tl_now());
#endif

    // Resolve logical -> physical pages of this split.  (FP8: the pages'
    // scales are read after the first copies are issued, so that their round
    // trip overlaps the copies instead of delaying them.)
    int phs[kWarpEntries / 32];
#pragma unroll
    for (int j = 0; j < kWarpEntries / 32; ++j) {
      const int i = lane + 32 * j;
      phs[j] = -1;
      if (i >= n_ent) continue;
      const int p = pre[j];
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
      phs[j] = ph;
      ent_s[warp][i] = make_int2(ph, p * a.P);
    }
    __syncwarp();

    const int subs = a.P / kSub;
    const int n_units = n_ent * subs;
#if SA_DECODE_TIMELINE
    SA_TL(2, tl_now());
    {
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      SA_TL(15, (unsigned long long)smid | ((unsigned long long)n_units << 16) |
                    ((unsigned long long)item << 32));
    }
#endif

    auto unit_live = [&](int u, int& ph, int& tok0) {
      const int2 e = ent_s[warp][u / subs];
      ph = e.x;
      tok0 = e.y + (u % subs) * kSub;
      return ph >= 0 && tok0 < L;
    };
    auto issue = [&](int u) {  // lane 0 only
      const int slot = (base + u) % C::kStages;
      uint64_t* bar = &bars[warp][slot];
      int ph, tok0;
      if (unit_live(u, ph, tok0)) {
        uint8_t* kt = ring + slot * C::kStageBytes;
        uint8_t* vt = kt + C::kInTile;
        const int row0 = (u % subs) * kSub;
        mbar_arrive_expect_tx(bar, C::kStageBytes);
        if constexpr (F8) {
          tma_load_4d(kt, &kmap, bar, 0, row0, kvh, ph);
          tma_load_4d(kt + C::kInTile, &vmap, bar, 0, row0, kvh, ph);
        } else {
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            tma_load_4d(kt + bx * C::kBoxBytes, &kmap, bar, bx * 64, row0, kvh, ph);
            tma_load_4d(vt + bx * C::kBoxBytes, &vmap, bar, bx * 64, row0, kvh, ph);
          }
        }
      } else {
        mbar_arrive_expect_tx(bar, 0);
      }
    };
    if (lane == 0)
      for (int u = 0; u < n_units && u < C::kStages; ++u) issue(u);

    float2 scl[F8 ? kWarpEntries / 32 : 1];
    if constexpr (F8) {
#pragma unroll
      for (int j = 0; j < kWarpEntries / 32; ++j)
        scl[j] = phs[j] >= 0 ? make_float2(a.k_scale[(int64_t)phs[j] * a.Hkv + kvh],
                                           a.v_scale[(int64_t)phs[j] * a.Hkv + kvh])
                             : make_float2(0.f, 0.f);
    }
    uint32_t qa[D / 16][4];
    int qt[2];
    load_q_frags<D, F8>(qa, qt, a, prm.pairs, pair, b, lane);
    if constexpr (F8) {
#pragma unroll
      for (int j = 0; j < kWarpEntries / 32; ++j)
        if (lane + 32 * j < n_ent) scl_s[warp][lane + 32 * j] = scl[j];
      __syncwarp();
    }
    // FP8: values enter PV scaled by (page scale / v_ref), v_ref = the largest
    // value scale of the split's pages (so P stays <= 256 in f16); the output is
    // multiplied back by v_ref.
    float v_ref = 1.f;
    if constexpr (F8) {
      float m = 0.f;
      for (int i = lane; i < n_ent; i += 32) m = fmaxf(m, scl_s[warp][i].y);
#pragma unroll
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      v_ref = m > 0.f ? m : 1.f;
    }
    const int qb = query_base(a, b, L);
    const int lim[2] = {qt[0] >= 0 ? qb + qt[0] : -1, qt[1] >= 0 ? qb + qt[1] : -1};

    RowState<D> st;
    state_clear(st);
    int u_fail = -1;
    for (int u = 0; u < n_units; ++u) {
      const int slot = (base + u) % C::kStages;
      if (!mbar_wait_bounded(&bars[warp][slot], ((base + u) / C::kStages) & 1)) {
        u_fail = u;
        break;
      }
#if SA_DECODE_TIMELINE
      if (u < 8) SA_TL(4 + u, tl_now());
#endif
      int ph, tok0;
      if (unit_live(u, ph, tok0)) {
        float ksc = 1.f, vsc = 1.f;   // FP8: key scale, value scale / v_ref
        if constexpr (F8) {
          const float2 sc = scl_s[warp][u / subs];
          ksc = sc.x;
          vsc = sc.y / v_ref;
        }
        attend_unit<D, F8>(st, qa, ring + slot * C::kStageBytes, wide, tok0, L, lim,
                           a.scale_log2, ksc, vsc, lane);
#if SA_DECODE_TIMELINE
        if (u == 0) SA_TL(3, tl_now());
#endif
      }
      __syncwarp();   // (FP8: the staging tiles are free again)
      if (lane == 0 && u + C::kStages < n_units) issue(u + C::kStages);
    }
    if (u_fail >= 0) {
      if (lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
      // units u_fail .. u_fail + kStages - 1 were issued: wait for them (bounded)
      // before this warp's shared memory can be released
      for (int u = u_fail + 1; u < n_units && u < u_fail + C::kStages; ++u)
        mbar_wait_bounded(&bars[warp][(base + u) % C::kStages], ((base + u) / C::kStages) & 1);
      return;
    }
    store_partial<D>(st, a, prm.pairs, pair, b, split, v_ref, lane);
    base += n_units;
#if SA_DECODE_TIMELINE
    SA_TL(12, tl_now());
    tl_row = -1;   // only the first item of a warp is recorded
#endif
  }  // items
}

template <int D, bool F8 = false>
cudaError_t launch_d(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                     const CUtensorMap& vmap, cudaStream_t stream) {
  using C = DecodeCfg<D, F8>;
  DecodeParams prm;
  prm.a = a;
  prm.pairs = pairs;
  // one wave of resident CTAs (or fewer when there is less work); the set-up
  // queries are answered once per context
  const void* kern = reinterpret_cast<const void*>(decode_gqa_kernel<D, F8>);
  int sms = 0, per_sm = 0;
  cudaError_t e = allow_max_dyn_smem(kern);
  if (e == cudaSuccess) e = sm_count(&sms);
  if (e == cudaSuccess) e = max_blocks_per_sm(kern, kNW * 32, C::kDynBytes, &per_sm);
  if (e != cudaSuccess) return e;
  const long long items = (long long)a.n_splits * pairs.n_pairs * a.B;
  const long long want = (items + kNW - 1) / kNW;
  const int grid = (int)std::min<long long>(want, (long long)std::max(1, per_sm) * sms);
  return launch_pdl(decode_gqa_kernel<D, F8>, grid, dim3(kNW * 32), C::kDynBytes, stream, prm, kmap,
                    vmap);
}

}  // namespace

int decode_max_split_entries() { return kWarpEntries; }
int decode_warps_per_cta() { return kNW; }

cudaError_t decode_default_splits(int D, int n_units, int max_list, int* out) {
  *out = 1;
  if (n_units <= 0 || max_list <= 0) return cudaSuccess;
  const void* kern = D == 64    ? reinterpret_cast<const void*>(decode_gqa_kernel<64, false>)
                     : D == 128 ? reinterpret_cast<const void*>(decode_gqa_kernel<128, false>)
                                : reinterpret_cast<const void*>(decode_gqa_kernel<256, false>);
  const int dyn = D == 64    ? DecodeCfg<64>::kDynBytes
                  : D == 128 ? DecodeCfg<128>::kDynBytes
                             : DecodeCfg<256>::kDynBytes;
  int sms = 0, per_sm = 0;
  cudaError_t e = sm_count(&sms);
  if (e == cudaSuccess) e = max_blocks_per_sm(kern, kNW * 32, dyn, &per_sm);
  if (e != cudaSuccess) return e;
  // as many splits as fill one wave of resident warps, at least enough that no
  // split holds more than a warp's list capacity, at most 64
  int n = std::max(1, std::max(1, per_sm) * kNW * sms / n_units);
  n = std::min(n, max_list);
  while ((max_list + n - 1) / n > kWarpEntries) ++n;
  *out = std::max(1, std::min(n, 64));
  return cudaSuccess;
}

cudaError_t launch_decode_gqa(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, cudaStream_t stream) {
  switch (a.Dk) {
    case 64: return launch_d<64>(a, pairs, kmap, vmap, stream);
    case 128: return launch_d<128>(a, pairs, kmap, vmap, stream);
    case 256: return launch_d<256>(a, pairs, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_gqa_fp8(const DecodeArgs& a, const PairTable& pairs,
                                  const CUtensorMap& kmap, const CUtensorMap& vmap,
                                  cudaStream_t stream) {
  if (a.Dk != 128 || !a.k_scale || !a.v_scale) return cudaErrorInvalidValue;
  return launch_d<128, true>(a, pairs, kmap, vmap, stream);
}

}  // namespace sa

#if SA_DECODE_TIMELINE
// Diagnostic build only: copies the recorded stamps ([8192 warps][16] u64) to
// host memory `out` (n entries at most) and clears them.  Not in the library's
// header: the library proper is built without it.
extern "C" SA_API int sa_decode_timeline(unsigned long long* out, int n) {
  const int total = sa::kTlWarps * sa::kTlSlots;
  if (!out || n <= 0) return SA_ERR_INVALID_ARG;
  const size_t bytes = sizeof(unsigned long long) * (size_t)(n < total ? n : total);
  if (cudaMemcpyFromSymbol(out, sa::g_decode_tl, bytes) != cudaSuccess) return SA_ERR_CUDA;
  void* dev = nullptr;
  if (cudaGetSymbolAddress(&dev, sa::g_decode_tl) != cudaSuccess ||
      cudaMemset(dev, 0, sizeof(unsigned long long) * total) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}
#endif
