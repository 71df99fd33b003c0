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
// sit in columns [256, 288) and [288, 320).  So the whole output fits in TMEM
// next to S and no FLOP is spent twice.
//
// Per 32-key tile S = Q K^T takes 36 MMAs of 64 x 32 x 16 and O += P V two
// halves of two 64 x 256 x 16 MMAs.  Shared memory: the query tile (72 KB,
// resident), four key stages of 36 KB and one P buffer of 8 KB: the deep ring
// is what hides the gather latency (a stage is free only once the PV of its
// tile is done, since the values are read from it).
//   warp 4      resolves the split's pages, then TMA-gathers key tiles (9
//               column chunks x two 16-key boxes; an absent or invalid group
//               is read at an out-of-range page, which TMA fills with zeros)
//               into the 4-stage ring;
//   warp 5      issues the MMAs (fully unrolled, descriptors advanced by
//               constants);
//   warps 0-3   stage the query tile (bulk row copies, then a swizzling
//               rearrangement in shared memory), then own a row per
//               lane pair (l, l + 16): mask, lazily re-based base-2 online
//               softmax and P for 16 keys each; the low lane rescales / writes
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
constexpr int kMStages = 4;
constexpr int kMKeys = 32;          // keys per tile
constexpr int kMRows = 64;          // query rows per CTA
constexpr int kMMaxEnt = 128;       // list entries per split
constexpr int kMMaxTiles = 128;     // tiles per split
constexpr int kDk = 576, kDv = 512;
constexpr int kKC = kDk / 64;       // 9 key column chunks
constexpr int kQBytes = kKC * kMRows * 128;          // 73728
constexpr int kChunkBytes = kMKeys * 128;            // 4096: one column chunk of a tile
constexpr int kTileBytes = kKC * kChunkBytes;        // 36864
constexpr int kPBytes = kMRows * 128;                // 8192: 64 rows of 128 bytes (32 keys used)
constexpr int kMDyn = kQBytes + kMStages * kTileBytes + kPBytes + 1024;
constexpr int kStageRow = kDv * 4 + 16;              // O staging row (padded: no bank conflicts)
static_assert(kMRows * kStageRow <= kMStages * kTileBytes, "O staging must fit the key ring");
constexpr uint32_t kMTmemCols = 512;
constexpr uint32_t kSCol = 256;                      // S buffers at 256 and 288
constexpr uint32_t kHiLanes = 16u << 16;             // second M=64 accumulator
constexpr uint32_t kIdQK = tc::idesc_bf16_f32(kMRows, kMKeys, false, false);
constexpr uint32_t kIdPV = tc::idesc_bf16_f32(kMRows, 256, false, true);
constexpr float kLazyM = 8.f;

constexpr int kMMaxItems = 256;     // (pair, 64-row tile) work items per call

struct __align__(64) MlaParams {
  DecodeArgs a;
  PairTable pairs;
  int n_items;
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
  const int key0 = (2 * j + g) * 16;
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
  __shared__ uint64_t kv_full[kMStages], kv_empty[kMStages];
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
  const int max_q = L - a.T + t_last;

  if (tid == 0) {
    for (int s = 0; s < kMStages; ++s) {
      mbar_init(&kv_full[s], 1);
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
  }
  if (warp == 5) tc::tmem_alloc(&tmem_base_s, kMTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;
  const int n_tiles = min((n_ent * a.P + kMKeys - 1) / kMKeys, kMMaxTiles);

  // query tile: 64 rows x 9 chunks of 128 bytes, 128-byte swizzle.  Each row
  // (1152 contiguous bytes) arrives with one bulk copy in the last two key
  // stages, then the softmax warps rearrange it into the swizzled layout; the
  // producer fills those two stages only after that (q_full).
  uint8_t* q_raw = k_s + (kMStages - 2) * kTileBytes;
  const int n_qrows = min(kMRows, rows_total - r0);
  if (warp < 4) {
    if (tid == 0) mbar_arrive_expect_tx(&q_stage, n_qrows * kDk * 2);
    __syncwarp();
    if (lane < 16) {
      const int qr = warp * 16 + lane;
      if (qr < n_qrows) {
        const int qrg = r0 + qr;
        const int qh = prm.pairs.heads[prm.pairs.head_off[pair] + qrg % nh];
        bulk_load(q_raw + qr * (kDk * 2), a.q + b * a.qs0 + (qrg / nh) * a.qs1 + qh * a.qs2,
                  kDk * 2, &q_stage);
      }
    }
  }
  if (warp == 4) {
    // ================= producer: the split's entries (list -> page table),
    // the tiles with a causally visible key (flag 128: the tile also holds a
    // key some row must not see, or an unreadable group), then TMA gathers of
    // key tiles (values alias them)
    const int32_t* lrow = a.lists + ((int64_t)b * a.n_lists + list) * a.max_list + e0;
    const int32_t* ptrow = a.page_table + (int64_t)b * a.max_pages;
    for (int i = lane; i < n_ent; i += 32) {
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
    __syncwarp();
    const int q_lo = L - a.T + r0 / nh;   // smallest query position among the rows
    int n_act = 0;
    for (int j0 = 0; j0 < n_tiles; j0 += 32) {
      const int j = j0 + lane;
      bool live = false, full = true;
      if (j < n_tiles)
        for (int g = 0; g < 2; ++g) {
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
    if (lane == 0) {
      n_act_s = n_act;
      mbar_arrive(&ent_ready);
      prefetch_tmap(&kmap);
      for (int jj = 0; jj < n_act; ++jj) {
        const int st = jj % kMStages;
        if (jj >= kMStages &&
            !wait_or_abort_m(&kv_empty[st], ((jj / kMStages) - 1) & 1, abort_flag))
          break;
        if (jj == kMStages - 2 && !wait_or_abort_m(&q_full, 0, abort_flag)) break;
        const int j = act_s[jj] & 127;
        uint8_t* kt = k_s + st * kTileBytes;
        mbar_arrive_expect_tx(&kv_full[st], kTileBytes);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int2 gr = mgroup(ent_s, n_ent, a.P, j, g);
          const bool ok = gr.x >= 0 && gr.y < L;
          const int page = ok ? gr.x : a.P_pool;     // out of range: zero-filled box
          const int row0 = ok ? gr.y % a.P : 0;
#pragma unroll
          for (int c = 0; c < kKC; ++c)
            tma_load_4d(kt + c * kChunkBytes + g * 2048, &kmap, &kv_full[st], c * 64, row0, kvh,
                        page);
        }
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer (one thread).  Descriptors are advanced by
    // adding (byte offset >> 4) to their start-address field.
    const bool ready = warp_wait_m(&ent_ready, 0, abort_flag);
    const int n_act = ready ? n_act_s : 0;
    if (lane == 0 && n_act > 0) {
      const uint64_t dq0 = tc::sdesc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t dk0 = tc::sdesc_sw128(smem_u32(k_s), 16, 1024);
      const uint64_t dp0 = tc::sdesc_sw128(smem_u32(p_s), 16, 1024);
      const uint64_t dv0 = tc::sdesc_sw128(smem_u32(k_s), kChunkBytes, 1024);
      auto pv = [&](int jp) -> bool {
        const int st = jp % kMStages;
        if (!wait_or_abort_m(&p_full, jp & 1, abort_flag)) return false;
        tc::fence_after_sync();
        const uint64_t dv = dv0 + static_cast<uint64_t>((st * kTileBytes) >> 4);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < kMKeys / 16; ++kk)
            tc::mma_bf16(tmem + (h ? kHiLanes : 0u), dp0 + static_cast<uint64_t>(kk * 2),
                         dv + static_cast<uint64_t>((4 * h * kChunkBytes + kk * 2048) >> 4),
                         kIdPV, (jp > 0 || kk > 0) ? 1u : 0u);
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
        const uint64_t dk = dk0 + static_cast<uint64_t>((st * kTileBytes) >> 4);
#pragma unroll
        for (int c = 0; c < kKC; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16(tmem + kSCol + sb * kMKeys,
                         dq0 + static_cast<uint64_t>((c * kMRows * 128 + kk * 32) >> 4),
                         dk + static_cast<uint64_t>((c * kChunkBytes + kk * 32) >> 4), kIdQK,
                         (c | kk) ? 1u : 0u);
        tc::commit(&s_full[sb]);
        if (jj >= 1 && !pv(jj - 1)) ok = false;
      }
      if (ok) pv(n_act - 1);
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
      for (int i = tid; i < kMRows * kKC * 8; i += 128) {
        const int row = i / (kKC * 8), ch = i % (kKC * 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (qok && row < n_qrows) v = *reinterpret_cast<const uint4*>(q_raw + row * (kDk * 2) + ch * 16);
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
    const int qpos = row_ok ? L - a.T + t : -1;
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
      float x[32];
      tc::ld32(tmem + lane_base + kSCol + sb * kMKeys, x);
      tc::wait_ld();
      float v[16];   // this lane's 16 keys: 0-15 (low lane) or 16-31 (high lane)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float hv = __shfl_sync(0xffffffffu, x[16 + i], lane & 15);
        v[i] = low ? x[i] : hv;
      }
      if (code & 128) {   // mask this lane's 16-key group
        const int2 gr = mgroup(ent_s, n_ent, a.P, j, low ? 0 : 1);
        const bool gok = gr.x >= 0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int kp = gr.y + c;
          if (!(gok && kp < L && kp <= qpos)) v[c] = -INFINITY;
        }
      }
      float m4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) m4[i] = fmaxf(fmaxf(v[i], v[i + 4]), fmaxf(v[i + 8], v[i + 12]));
      float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16)) * sl2;   // the row's max, scaled
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
      uint8_t* prow = p_s + r * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p[i] = exp2f(fmaf(v[ch * 8 + i], sl2, nb));
          l += p[i];
        }
        uint4 w;
        w.x = pack_bf16(p[0], p[1]);
        w.y = pack_bf16(p[2], p[3]);
        w.z = pack_bf16(p[4], p[5]);
        w.w = pack_bf16(p[6], p[7]);
        *reinterpret_cast<uint4*>(prow + ((((low ? 0 : 2) + ch) ^ (r & 7)) << 4)) = w;
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
    for (int c = 0; c < 256 / 32; ++c) {
      float o[32];
      if (n_act > 0) {
        tc::ld32(tmem + lane_base + c * 32, o);
        tc::wait_ld();
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(stg + (low ? 0 : 1024) + (c * 32 + i) * 4) =
            empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                  : make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
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
  // one work item per (pair, 64-row tile): no CTA for row tiles a pair lacks
  prm.n_items = 0;
  for (int i = 0; i < pairs.n_pairs; ++i)
    for (int qt = 0; qt * kMRows < a.T * pairs.n_heads[i]; ++qt) {
      if (prm.n_items == kMMaxItems) return cudaErrorInvalidConfiguration;
      prm.item_pair[prm.n_items] = static_cast<int16_t>(i);
      prm.item_qt[prm.n_items] = static_cast<int16_t>(qt);
      ++prm.n_items;
    }
  cudaError_t e =
      cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMDyn);
  if (e != cudaSuccess) return e;
  if (prm.n_items == 0) return cudaSuccess;
  dim3 grid(prm.n_items * a.n_splits, 1, a.B);
  return launch_pdl(mla_kernel, grid, dim3(kMThreads), kMDyn, stream, prm, kmap);
}

}  // namespace sa
