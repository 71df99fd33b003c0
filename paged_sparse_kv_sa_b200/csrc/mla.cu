// Sparse MLA decode over per-head page lists on the 5th-generation tensor
// cores: one shared latent KV head, keys of Dk = 576 (512 latent + 64 rope),
// values = the first Dv = 512 key columns (read from the same tile), many
// query rows (T x heads) per list.
//
// One CTA computes 64 query rows of one (list, kv head) pair against its split
// of the list, 64 keys per tile.  The MMAs are M = 64: TMEM then holds a
// 64-row accumulator in the low 16 lanes of each 32-lane subpartition, and a
// second one in the high 16 lanes of the same columns.  O (64 x 512 float32)
// is kept as two such halves — value columns 0-255 in the low lanes, 256-511
// in the high lanes — in TMEM columns [0, 256); the two S buffers (64 x 64)
// sit in columns [256, 320) and [320, 384).  So the whole output fits in TMEM
// next to S and no FLOP is spent twice.
//
// Per 64-key tile S = Q K^T takes 36 MMAs of 64 x 64 x 16 (an MMA of N <= 64
// costs the same issue time as one of N = 32, so 64-key tiles halve the QK
// issue cost per key) and O += P V two halves of four 64 x 256 x 16 MMAs, each
// twice: P enters as bf16 hi + lo (its rounding then ~2^-17 relative), the low
// parts written into the tile's rope chunk, which only QK reads.
// Shared memory: the query tile (72 KB, resident), two key stages of 72 KB and
// one P buffer of 8 KB.  A stage is free only once the PV of its tile is done
// (the values are read from it), so the ring is kept moving by issuing MMAs
// as their inputs arrive: every 64-column chunk of a stage has its own full
// barrier (the QK MMAs of chunk 0 start while chunks 1-8 are in flight), and
// PV of tile j goes out as soon as P of tile j is written, ahead of QK
// chunks of tile j + 1 that have not landed, so the stage of tile j is
// refilled while tile j + 1 is being scored.
//   warp 4      resolves the split's pages, then TMA-gathers key tiles (9
//               column chunks; one 64-row box per chunk when a tile lies in
//               one page, else four 16-row boxes; an absent or invalid group
//               is read at an out-of-range page, which TMA fills with zeros)
//               into the 2-stage ring;
//   warp 5      issues the MMAs in arrival order (descriptors advanced by
//               constants);
//   warps 0-3   stage the query tile (bulk row copies, then a swizzling
//               rearrangement in shared memory), then own a row per
//               lane pair (l, l + 16): mask, lazily re-based base-2 online
//               softmax and P for 32 keys each; the low lane rescales / writes
//               value columns 0-255 of O, the high lane 256-511.
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
constexpr int kMStages = 2;
constexpr int kMKeys = 64;          // keys per tile
constexpr int kMGroups = kMKeys / 16;   // 16-key groups per tile
constexpr int kMRows = 64;          // query rows per CTA
constexpr int kMMaxEnt = 128;       // list entries per split
constexpr int kMMaxTiles = 128;     // tiles per split (tile ids fit 7 bits)
constexpr int kDk = 576, kDv = 512;
constexpr int kKC = kDk / 64;       // 9 key column chunks
constexpr int kQBytes = kKC * kMRows * 128;          // 73728
constexpr int kChunkBytes = kMKeys * 128;            // 8192: one column chunk of a tile
constexpr int kTileBytes = kKC * kChunkBytes;        // 73728
constexpr int kPBytes = kMRows * 128;                // 8192: 64 rows of 64 bf16 keys
constexpr int kMDyn = kQBytes + kMStages * kTileBytes + kPBytes + 1024;
constexpr int kStageRow = kDv * 4 + 16;              // O staging row (padded: no bank conflicts)
static_assert(kMRows * kStageRow <= kMStages * kTileBytes, "O staging must fit the key ring");
static_assert(kQBytes <= kTileBytes, "the raw query rows are staged in the last key stage");
static_assert(kMDyn + 2048 <= 232448, "shared memory per CTA");
constexpr uint32_t kMTmemCols = 512;
constexpr uint32_t kSCol = 256;                      // S buffers at 256 and 320
constexpr uint32_t kHiLanes = 16u << 16;             // second M=64 accumulator
constexpr uint32_t kIdQK = tc::idesc_bf16_f32(kMRows, kMKeys, false, false);
constexpr uint32_t kIdPV = tc::idesc_bf16_f32(kMRows, 256, false, true);
constexpr float kLazyM = 8.f;

constexpr int kMMaxItems = 256;     // (pair, 64-row tile) work items per call

struct __align__(64) MlaParams {
  DecodeArgs a;
  PairTable pairs;
  int n_items;
  int box_rows;                     // rows per TMA box: 64 (tiles within one page) or 16
  int16_t item_pair[kMMaxItems], item_qt[kMMaxItems];
};

SA_DEV bool wait_or_abort_m(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// The same wait taken by a whole warp: true only if it succeeded in every lane,
// so that the lanes leave or stay in a loop together.
SA_DEV bool warp_wait_m(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, wait_or_abort_m(bar, parity, abort_flag));
}
// (physical page or -1, first token) of 16-key group g of tile j.
SA_DEV int2 mgroup(const int2* ent, int n_ent, int P, int j, int g) {
  const int key0 = (kMGroups * j + g) * 16;
  const int e = key0 / P;
  if (e >= n_ent) return make_int2(-1, 0);
  const int2 en = ent[e];
  return make_int2(en.x, en.y + key0 % P);
}

__global__ void __launch_bounds__(kMThreads, 1)
    mla_kernel(const __grid_constant__ MlaParams prm, const __grid_constant__ CUtensorMap kmap) {
  pdl_wait_and_release();
  const DecodeArgs& a = prm.a;
  const int item = blockIdx.x / a.n_splits, split = blockIdx.x % a.n_splits, b = blockIdx.z;
  const int pair = prm.item_pair[item], qt = prm.item_qt[item];
  const int nh = prm.pairs.n_heads[pair];
  const int rows_total = a.T * nh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int list = prm.pairs.list_of[pair], kvh = prm.pairs.kvh_of[pair];

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  uint8_t* q_s = smem;
  uint8_t* k_s = smem + kQBytes;                              // kMStages tiles
  uint8_t* p_s = k_s + kMStages * kTileBytes;                 // one P buffer
  __shared__ uint64_t kv_full[kMStages][kKC], kv_empty[kMStages];   // full: per column chunk
  __shared__ uint64_t s_full[2], p_full, o_done, q_full, q_stage, ent_ready;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, n_act_s;
  __shared__ int2 ent_s[kMMaxEnt];
  __shared__ uint8_t act_s[kMMaxTiles];

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
  const int r0 = qt * kMRows;
  if (n_ent == 0) {   // an empty split: LSE = -inf (and O = 0 when it is the only split)
    const int nr = min(kMRows, rows_total - r0);
    for (int rr = r0 + tid; rr < r0 + nr; rr += blockDim.x) {
      const int t = rr / nh, head = prm.pairs.heads[prm.pairs.head_off[pair] + (rr % nh)];
      a.lse_part[(((int64_t)split * a.B + b) * a.T + t) * a.Hq + head] = -INFINITY;
    }
    if (a.n_splits == 1)
      for (int i = tid; i < nr * (kDv / 4); i += blockDim.x) {
        const int rr = r0 + i / (kDv / 4), c = (i % (kDv / 4)) * 4;
        const int t = rr / nh, head = prm.pairs.heads[prm.pairs.head_off[pair] + (rr % nh)];
        const int64_t orow = (((int64_t)b * a.T + t) * a.Hq + head);
        *reinterpret_cast<float4*>(a.o_part + orow * kDv + c) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    return;
  }
  const int t_last = (min(rows_total, r0 + kMRows) - 1) / nh;
  const int max_q = query_base(a, b, L) + t_last;

  const int n_tiles = min((n_ent * a.P + kMKeys - 1) / kMKeys, kMMaxTiles);
  // query tile: 64 rows x 9 chunks of 128 bytes, 128-byte swizzle.  Each row
  // (1152 contiguous bytes) arrives with one bulk copy in the last key stage,
  // then the softmax warps rearrange it into the swizzled layout; the producer
  // fills that stage only after that (q_full).
  uint8_t* q_raw = k_s + (kMStages - 1) * kTileBytes;
  const int n_qrows = min(kMRows, rows_total - r0);

  // warp 4: the split's entries (list -> page table) and the tiles with a
  // causally visible key (flag 128: the tile also holds a key some row must
  // not see, or an unreadable group).  Done before the CTA barrier, so that
  // these two dependent global reads overlap the barrier and TMEM set-up.
  int n_act = 0;
  if (warp == 4) {
    const int32_t* lrow = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list + e0;
    for (int i = lane; i < n_ent; i += 32) {
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
    __syncwarp();
    const int q_lo = L - a.T + r0 / nh;   // smallest query position among the rows
    for (int j0 = 0; j0 < n_tiles; j0 += 32) {
      const int j = j0 + lane;
      bool live = false, full = true;
      if (j < n_tiles)
        for (int g = 0; g < kMGroups; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          live |= gr.x >= 0 && gr.y < L && gr.y <= max_q;
          full &= gr.x >= 0 && gr.y + 15 < L && gr.y + 15 <= q_lo;
        }
      const uint32_t m = __ballot_sync(0xffffffffu, live);
      if (live)
        act_s[n_act + __popc(m & ((1u << lane) - 1u))] = static_cast<uint8_t>(j | (full ? 0 : 128));
      n_act += __popc(m);
    }
    __syncwarp();
  }
  if (tid == 0) {
    for (int s = 0; s < kMStages; ++s) {
      for (int c = 0; c < kKC; ++c) mbar_init(&kv_full[s][c], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&s_full[s], 1);
    mbar_init(&p_full, 128);
    mbar_init(&o_done, 1);
    mbar_init(&q_full, 1);
    mbar_init(&q_stage, 1);
    mbar_init(&ent_ready, 1);
    abort_s = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(&q_stage, n_qrows * kDk * 2);
  }
  if (warp == 0) {   // the query rows, two per lane, as soon as q_stage exists
    __syncwarp();
    for (int qr = lane; qr < n_qrows; qr += 32) {
      const int qrg = r0 + qr;
      const int qh = prm.pairs.heads[prm.pairs.head_off[pair] + qrg % nh];
      bulk_load(q_raw + qr * (kDk * 2), a.q + b * a.qs0 + (qrg / nh) * a.qs1 + qh * a.qs2,
                kDk * 2, &q_stage);
    }
  }
  if (warp == 5) {
    tc::tmem_alloc(&tmem_base_s, kMTmemCols);
    if (lane == 0) prefetch_tmap(&kmap);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;

  if (warp == 4) {
    // ================= producer: TMA gathers of key tiles (values alias them)
    if (lane == 0) {
      n_act_s = n_act;
      mbar_arrive(&ent_ready);
      const bool box64 = prm.box_rows == 64;
      // (page, first row) of the boxes of tile j: one 64-row box (the tile lies
      // in one page) or four 16-row groups; an absent group reads an
      // out-of-range page (zero-filled)
      auto boxes = [&](int j, int (&page)[kMGroups], int (&row0)[kMGroups]) {
#pragma unroll
        for (int g = 0; g < kMGroups; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          const bool ok = gr.x >= 0 && gr.y < L;
          page[g] = ok ? gr.x : a.P_pool;
          row0[g] = ok ? gr.y % a.P : 0;
        }
      };
      for (int jj = 0; jj < n_act; ++jj) {
        const int st = jj % kMStages;
        if (jj >= kMStages &&
            !wait_or_abort_m(&kv_empty[st], ((jj / kMStages) - 1) & 1, abort_flag))
          break;
        if (jj == kMStages - 1 && !wait_or_abort_m(&q_full, 0, abort_flag)) break;
        int page[kMGroups], row0[kMGroups];
        boxes(act_s[jj] & 127, page, row0);
        uint8_t* kt = k_s + st * kTileBytes;
#pragma unroll
        for (int c = 0; c < kKC; ++c) {
          mbar_arrive_expect_tx(&kv_full[st][c], kChunkBytes);
          if (box64) {
            tma_load_4d(kt + c * kChunkBytes, &kmap, &kv_full[st][c], c * 64, row0[0], kvh,
                        page[0]);
          } else {
#pragma unroll
            for (int g = 0; g < kMGroups; ++g)
              tma_load_4d(kt + c * kChunkBytes + g * 2048, &kmap, &kv_full[st][c], c * 64,
                          row0[g], kvh, page[g]);
          }
        }
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer (one thread).  Descriptors are advanced by
    // adding (byte offset >> 4) to their start-address field.  The MMAs go out
    // in the order their inputs arrive, not tile by tile: PV of tile jp as soon
    // as its P is in shared memory (it frees the tile's stage for the producer),
    // else the next landed column chunk of QK of tile jq.  The tensor pipe runs
    // them in issue order; QK of tile jq writes the S buffer that tile jq - 2
    // used, which is free once PV of tile jq - 2 was issued (jq <= jp + 1).
    const bool ready = warp_wait_m(&ent_ready, 0, abort_flag);
    const int n_act = ready ? n_act_s : 0;
    if (lane == 0 && n_act > 0) {
      const uint64_t dq0 = tc::sdesc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t dk0 = tc::sdesc_sw128(smem_u32(k_s), 16, 1024);
      const uint64_t dp0 = tc::sdesc_sw128(smem_u32(p_s), 16, 1024);
      const uint64_t dv0 = tc::sdesc_sw128(smem_u32(k_s), kChunkBytes, 1024);
      bool ok = wait_or_abort_m(&q_full, 0, abort_flag);
      tc::fence_after_sync();
      int jq = 0, cq = 0, jp = 0;   // next QK tile, its next column chunk; next PV tile
      uint32_t idle = 0;
      while (ok && jp < n_act) {
        if (jp < jq && mbar_test_wait(&p_full, jp & 1)) {
          tc::fence_after_sync();
          const int st = jp % kMStages;
          const uint64_t dv = dv0 + static_cast<uint64_t>((st * kTileBytes) >> 4);
          // P = hi + lo: the low parts sit in the stage's rope chunk (dead after QK)
          const uint64_t dl =
              tc::sdesc_sw128(smem_u32(k_s) + st * kTileBytes + (kKC - 1) * kChunkBytes, 16, 1024);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < kMKeys / 16; ++kk) {
              const uint64_t bv = dv + static_cast<uint64_t>((4 * h * kChunkBytes + kk * 2048) >> 4);
              tc::mma_bf16(tmem + (h ? kHiLanes : 0u), dp0 + static_cast<uint64_t>(kk * 2), bv,
                           kIdPV, (jp > 0 || kk > 0) ? 1u : 0u);
              tc::mma_bf16(tmem + (h ? kHiLanes : 0u), dl + static_cast<uint64_t>(kk * 2), bv,
                           kIdPV, 1u);
            }
          tc::commit(&o_done);
          tc::commit(&kv_empty[st]);
          ++jp;
          idle = 0;
          continue;
        }
        if (jq < n_act && jq <= jp + 1 &&
            mbar_test_wait(&kv_full[jq % kMStages][cq], (jq / kMStages) & 1)) {
          tc::fence_after_sync();
          const uint64_t dk = dk0 + static_cast<uint64_t>(((jq % kMStages) * kTileBytes +
                                                           cq * kChunkBytes) >> 4);
          const uint64_t dq = dq0 + static_cast<uint64_t>((cq * kMRows * 128) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + kSCol + (jq & 1) * kMKeys, dq + static_cast<uint64_t>(kk * 2),
                         dk + static_cast<uint64_t>(kk * 2), kIdQK, (cq | kk) ? 1u : 0u);
          if (++cq == kKC) {
            tc::commit(&s_full[jq & 1]);
            cq = 0;
            ++jq;
          }
          idle = 0;
          continue;
        }
        ++idle;
        if ((idle & 1023u) == 0u && *abort_flag) ok = false;
        if (idle >= kSpinLimit) {
          *abort_flag = 1;
          ok = false;
        }
      }
    }
  } else {
    // ================= softmax / epilogue.  Row 16w + (l & 15) is shared by
    // lanes l and l + 16: the low lane reads its S row from TMEM and hands
    // keys 32-63 to the high lane; each takes the mask, exponentials and P
    // bytes of its 32 keys, and the row statistics are combined across the
    // pair.  For O the low lane owns value columns 0-255, the high lane
    // 256-511 (the two M = 64 accumulators).
    {
      // raw query rows -> swizzled K-major chunks (rows past the CTA's: zeros)
      const bool qok = warp_wait_m(&q_stage, 0, abort_flag);
#pragma unroll 4
      for (int i = tid; i < kMRows * kKC * 8; i += 128) {
        const int row = i / (kKC * 8), ch = i % (kKC * 8);
        uint4 v = *reinterpret_cast<const uint4*>(q_raw + row * (kDk * 2) + ch * 16);
        if (!(qok && row < n_qrows)) v = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(q_s + (ch >> 3) * (kMRows * 128) + row * 128 +
                                  (((ch & 7) ^ (row & 7)) << 4)) = v;
      }
      tc::fence_proxy_async();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) mbar_arrive(&q_full);
    }
    const bool ready = warp_wait_m(&ent_ready, 0, abort_flag);
    const int n_act = ready ? n_act_s : 0;
    const bool low = lane < 16;
    const int r = warp * 16 + (lane & 15);
    const int rg = r0 + r;
    const bool row_ok = rg < rows_total;
    const int t = row_ok ? rg / nh : 0;
    const int head = prm.pairs.heads[prm.pairs.head_off[pair] + (row_ok ? rg % nh : 0)];
    const int qpos = row_ok ? query_base(a, b, L) + t : -1;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = ready;
    for (int jj = 0; jj < n_act; ++jj) {
      const int sb = jj & 1, code = act_s[jj], j = code & 127;
      if (!warp_wait_m(&s_full[sb], (jj >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float v[32];   // this lane's 32 keys: 0-31 (low lane) or 32-63 (high lane)
      {
        float x[32];
        tc::ld32(tmem + lane_base + kSCol + sb * kMKeys, v);
        tc::ld32(tmem + lane_base + kSCol + sb * kMKeys + 32, x);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float hv = __shfl_sync(0xffffffffu, x[i], lane & 15);
          v[i] = low ? v[i] : hv;
        }
      }
      // the row max of the scaled scores from the raw ones: x -> x s is monotone,
      // so it is s max(x) for s >= 0 and s min(x) for s < 0; invisible keys are
      // NaN here (ignored by the reduction, p = 0 below)
      const bool masked = code & 128;
      if (masked) {   // this lane's two 16-key groups
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, (low ? 0 : 2) + gg);
          const bool gok = gr.x >= 0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int kp = gr.y + c;
            if (!(gok && kp < L && kp <= qpos)) v[gg * 16 + c] = NAN;
          }
        }
      }
      const float mr = sl2 >= 0.f ? reduce_n<false>(v) : reduce_n<true>(v);
      float mx = mr != mr ? -INFINITY : mr * sl2;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));   // the row's max, scaled
      // PV of the previous tile done: O is stable and the P buffer free
      if (jj >= 1 && !warp_wait_m(&o_done, (jj - 1) & 1, abort_flag)) {
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
      const float nb = m_ref == -INFINITY ? 0.f : -m_ref;
      // P = hi + lo (both bf16, so its rounding stays ~2^-17 relative): hi into
      // the P buffer, lo into this tile's stage's rope chunk (read by QK only,
      // and QK of this tile is complete)
      uint8_t* prow = p_s + r * 128;
      uint8_t* lrow = k_s + (jj % kMStages) * kTileBytes + (kKC - 1) * kChunkBytes + r * 128;
      // (key pairs in packed float32: the same roundings as the scalar ops)
      const unsigned long long sl2x = f2_pack(sl2, sl2), nb2x = f2_pack(nb, nb);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x0 = v[ch * 8 + 2 * i], x1 = v[ch * 8 + 2 * i + 1];
          const float2 z = f2_unpack(f2_fma(f2_pack(x0, x1), sl2x, nb2x));
          p[2 * i] = ex2_approx(z.x);
          p[2 * i + 1] = ex2_approx(z.y);
          if (masked) {
            p[2 * i] = x0 == x0 ? p[2 * i] : 0.f;
            p[2 * i + 1] = x1 == x1 ? p[2 * i + 1] : 0.f;
          }
        }
        l += ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hw[i] = pack_bf16(p[2 * i], p[2 * i + 1]);
          const float2 d = f2_unpack(f2_sub(f2_pack(p[2 * i], p[2 * i + 1]),
                                            f2_pack(__uint_as_float(hw[i] << 16),
                                                    __uint_as_float(hw[i] & 0xffff0000u))));
          lw[i] = pack_bf16(d.x, d.y);
        }
        const int off = (((low ? 0 : 4) + ch) ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lrow + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full);
    }
    if (ok && n_act > 0) ok = warp_wait_m(&o_done, (n_act - 1) & 1, abort_flag);
    tc::fence_after_sync();
    l += __shfl_xor_sync(0xffffffffu, l, 16);       // the two halves of the row
    const bool empty = !ok || n_act == 0 || l == 0.f;
    const float inv = empty ? 0.f : 1.f / l;
    const int64_t orow = (((int64_t)split * a.B + b) * a.T + t) * a.Hq + head;
    // the normalised O rows are staged in shared memory (the key ring is free:
    // every tile's PV is done) and leave with one 2 KB bulk store per row
    uint8_t* stg = k_s + r * kStageRow;
    for (int c = 0; c < 256 / 32; c += 2) {   // two TMEM loads in flight per wait
      float o[2][32];
      if (n_act > 0) {
        tc::ld32(tmem + lane_base + c * 32, o[0]);
        tc::ld32(tmem + lane_base + (c + 1) * 32, o[1]);
        tc::wait_ld();
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(stg + (low ? 0 : 1024) + ((c + h) * 32 + i) * 4) =
              empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                    : make_float4(o[h][i] * inv, o[h][i + 1] * inv, o[h][i + 2] * inv,
                                  o[h][i + 3] * inv);
    }
    tc::fence_proxy_async();
    __syncwarp();
    if (low && row_ok) {
      bulk_store(a.o_part + orow * kDv, stg, kDv * 4);
      bulk_commit();
    }
    if (row_ok && low) a.lse_part[orow] = empty ? -INFINITY : (m_ref + log2f(l)) * kLn2;
    if (!ok && lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
    if (low && row_ok) bulk_wait_all();   // the staged rows are read before the CTA ends
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kMTmemCols);
  }
}

}  // namespace

int mla_max_split_entries(int P) { return min(kMMaxEnt, kMMaxTiles * kMKeys / P); }

cudaError_t launch_mla(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                       cudaStream_t stream) {
  MlaParams prm;
  prm.a = a;
  prm.pairs = pairs;
  prm.box_rows = a.P % 64 == 0 ? 64 : 16;
  // one work item per (pair, 64-row tile): no CTA for row tiles a pair lacks
  prm.n_items = 0;
  for (int i = 0; i < pairs.n_pairs; ++i)
    for (int qt = 0; qt * kMRows < a.T * pairs.n_heads[i]; ++qt) {
      if (prm.n_items == kMMaxItems) return cudaErrorInvalidConfiguration;
      prm.item_pair[prm.n_items] = static_cast<int16_t>(i);
      prm.item_qt[prm.n_items] = static_cast<int16_t>(qt);
      ++prm.n_items;
    }
  cudaError_t e = allow_max_dyn_smem(reinterpret_cast<const void*>(mla_kernel));
  if (e != cudaSuccess) return e;
  if (prm.n_items == 0) return cudaSuccess;
  dim3 grid(prm.n_items * a.n_splits, 1, a.B);
  return launch_pdl(mla_kernel, grid, dim3(kMThreads), kMDyn, stream, prm, kmap);
}

}  // namespace sa
