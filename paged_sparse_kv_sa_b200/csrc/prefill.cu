// Sparse attention over per-head page lists for many query rows per (list,
// kv head) pair -- chunked prefill over block-union tables, long MTP -- on the
// 5th-generation tensor cores.
//
// One CTA computes 256 query rows of a pair (token-major) as two 128-row tiles
// A and B against the keys of its split of the list, 128 keys per tile; each
// K/V tile is loaded once and used by both:
//   warp 16     gathers K and V tiles from the paged pool with TMA (16-key x
//               64-column boxes; an absent or invalid 16-key group is loaded
//               from an out-of-range page coordinate, which TMA fills with
//               zeros) into separate K and V rings of two (D = 128) or four
//               (D = 64) stages;
//   warp 17     issues tcgen05.mma: S_w = Q_w K^T (M=128, N=128, K=D) into one
//               TMEM S buffer per tile w, and O_w += P_w V (M=128, N=D) with P
//               read from the TMEM columns of S_w as the A operand, in the order
//               PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1): the tensor core works
//               on one tile while the other tile's softmax runs;
//   warps 0-7 / 8-15   (tile A / B) own each query row with two threads, one
//               per 64-key half of every tile (four softmax warps per SM
//               sub-partition, so that they hide one another's latency): Q
//               into shared memory, S from TMEM, masking (page validity,
//               sequence end, causal position; skipped for tiles every row sees
//               whole), the row max from both halves (swapped through shared
//               memory), a base-2 online softmax whose running max only moves
//               when a row's max exceeds it by more than 2^8 (the O rescale
//               through TMEM is then rare), P back into the S columns it came
//               from, and the epilogue (each half of a row writes half of O).
//               The two tiles' softmax warps take turns (A(j) after B(j-1),
//               B(j) after A(j)), so that one tile's softmax runs while the
//               tensor core works on the other tile's PV and QK^T.
// P enters PV as a bf16 pair hi + lo (hi = p truncated to bf16, lo = p - hi,
// exact in float32, truncated to bf16), so hi + lo is within 2^-16 relative of
// p rather than the 2^-9 of a single rounded bf16, at the cost of two
// bitwise operations per key and no conversion instruction: two
// MMAs per 16 keys, reading the pair from the TMEM columns where those keys'
// scores were (per 16 keys: 8 columns of hi pairs, then 8 of lo pairs).
// Single-buffered S costs no wait: the commit that announces S_w(j) tracks
// every MMA issued before it, PV_w(j-1) included, so when the softmax sees
// S_w(j) the previous P is consumed and O_w may be rescaled.
//
// Sources: CompactAttention (abstract on the page titled "Causal Attention on
// CPU: A Cache-Aware and Load-Balanced Scheduling Kernel for Prefill"):
// per-group KV block tables used in place; "Universal Attention Engine —
// Declarative Sparse Attention for Production", "Key Design Decisions" 3:
// prefill is compute-bound, so the FLOPs go to the tensor cores.
#include "common.cuh"
#include "internal.h"
#include "tc05.cuh"

// Diagnostic build (-DSA_PREFILL_TIMELINE=1, off in the library): the first
// kPtCtas CTAs of a launch record SM clock stamps per key tile -- the MMA
// thread's waits and issues and both softmax warpgroups' phases -- read back
// with sa_prefill_timeline().
#ifndef SA_PREFILL_TIMELINE
#define SA_PREFILL_TIMELINE 0
#endif

namespace sa {
#if SA_PREFILL_TIMELINE
constexpr int kPtCtas = 4, kPtIters = 256, kPtSlots = 16;
__device__ long long g_prefill_tl[kPtCtas * kPtIters * kPtSlots];
// every CTA (up to kPtAll): %globaltimer at entry and exit, active tiles, SM id
constexpr int kPtAll = 8192;
__device__ long long g_prefill_cta[kPtAll * 4];
SA_DEV long long pt_now() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
SA_DEV void pt_cta_put(int slot, long long v) {
  const int c = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  if (c < kPtAll) g_prefill_cta[c * 4 + slot] = v;
}
SA_DEV void pt_cta_end(int n_act) {
  uint32_t sm;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
  pt_cta_put(1, pt_now());
  pt_cta_put(2, n_act);
  pt_cta_put(3, sm);
}
#endif
namespace {

constexpr int kSoftWarps = 16;    // two per (row tile, TMEM lane quarter, key half)
constexpr int kProdWarp = kSoftWarps, kMmaWarp = kSoftWarps + 1;
constexpr int kPThreads = 32 * (kSoftWarps + 2);
constexpr int kKeys = 128;        // keys per tile
constexpr int kGroups = kKeys / 16;
constexpr int kM = 128;           // query rows per warpgroup tile
constexpr int kRows = 2 * kM;     // query rows per CTA
constexpr int kMaxEnt = 1024;     // list entries per split
constexpr float kLazyP = 8.f;

template <int D>
struct PCfg {
  static constexpr int kChunks = D / 64;               // 64-column (128-byte) chunks
  static constexpr int kQBytes = kM * D * 2;
  static constexpr int kTileBytes = kKeys * D * 2;     // one K (or V) tile
  static constexpr int kStages = D == 64 ? 4 : 2;      // per ring (K and V)
  static constexpr int kDyn = 2 * kQBytes + 2 * kStages * kTileBytes + 1024;
  // tile w: S (then P hi + lo) at columns 128w .. 128w + 127, O at 256 + D w
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdQK = tc::idesc_bf16_f32(kM, kKeys, false, false);
  static constexpr uint32_t kIdPV = tc::idesc_bf16_f32(kM, D, false, true);
};

struct __align__(64) PrefillParams {
  DecodeArgs a;
  PairTable pairs;
};

// Named barrier `id` over `n` threads: ids 1-8 pair the two key-half warps of
// each (row tile, TMEM lane quarter); 0 is __syncthreads, 9 and 10 the turns.
SA_DEV void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Turn-taking of the two tiles' softmax warps (512 threads): tile A arrives on
// kTurnA when it has handed over P of a key tile, tile B on kTurnB; the other
// tile's warps wait there.
constexpr int kTurnA = 9, kTurnB = 10;
template <int kId>
SA_DEV void turn_wait() { asm volatile("bar.sync %0, 512;" ::"n"(kId) : "memory"); }
template <int kId>
SA_DEV void turn_pass() { asm volatile("bar.arrive %0, 512;" ::"n"(kId) : "memory"); }

// Bounded wait that also gives up as soon as another role has aborted.
SA_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

// (physical page or -1, first token) of 16-key group g of tile j: the tiles cut
// the concatenation of the split's pages into runs of kKeys keys (a page size
// is a multiple of 16, so a group never straddles two pages).
SA_DEV int2 group_of(const int2* ent, int n_ent, int P, int j, int g) {
  const int key0 = (j * kGroups + g) * 16;
  const int e = key0 / P;
  if (e >= n_ent) return make_int2(-1, 0);
  const int2 en = ent[e];
  return make_int2(en.x, en.y + key0 % P);
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
  if (qt * kRows >= rows_total) {                     // whole CTA: nothing to do
#if SA_PREFILL_TIMELINE
    if (threadIdx.x == 0) {
      pt_cta_put(0, pt_now());
      pt_cta_end(0);
    }
#endif
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int list = prm.pairs.list_of[pair], kvh = prm.pairs.kvh_of[pair];
#if SA_PREFILL_TIMELINE
  // slots per key tile: 0 K in (before QK_A), 1 QK_B issued, 2 / 3 second half of
  // P of tiles A / B in (the MMA thread), 4 / 7 S in, 5 / 8 P of keys 0-63
  // written, 6 / 9 P of keys 64-127 written, 12 / 14 partial maxima exchanged,
  // 13 / 15 row max (and any O rescale) done (softmax A / B); tile 0 slot 10:
  // start, slot 11: tiles
  const int pt_cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  long long* pt_row = pt_cta < kPtCtas ? g_prefill_tl + (int64_t)pt_cta * kPtIters * kPtSlots
                                       : nullptr;
  auto pt_mark = [&](int it, int slot) {
    if (pt_row && it >= 0 && it < kPtIters) pt_row[it * kPtSlots + slot] = clock64();
  };
  if (tid == 0) {
    pt_mark(0, 10);
    pt_cta_put(0, pt_now());
  }
#endif

  extern __shared__ uint8_t dyn_smem[];
  uint8_t* smem = dyn_smem + ((1024 - (smem_u32(dyn_smem) & 1023)) & 1023);
  uint8_t* q_s = smem;                                       // 2 tiles
  uint8_t* k_s = smem + 2 * C::kQBytes;                      // kStages K tiles
  uint8_t* v_s = k_s + C::kStages * C::kTileBytes;           // kStages V tiles
  __shared__ uint64_t k_full[C::kStages], k_empty[C::kStages];
  __shared__ uint64_t v_full[C::kStages], v_empty[C::kStages];
  __shared__ uint64_t s_full[2], p_full[2][2], o_done[2], q_full;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, n_act_s;
  __shared__ int2 ent_s[kMaxEnt];
  // partial row maxima (by tile parity), row sums and status of the two key
  // halves of every row
  __shared__ float pmax_s[2][2][2][kM];
  __shared__ float lsum_s[2][2][kM];
  __shared__ int okay_s[2][2][kM];
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
  // split s holds entries [s c, (s + 1) c) of the list, c = ceil(count / n_splits):
  // shares of the list's actual length, so that no split idles while another
  // holds a capacity's worth (c <= ceil(max_list / n_splits), checked on the host)
  const int chunk = (count + a.n_splits - 1) / a.n_splits;
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
#if SA_PREFILL_TIMELINE
    __syncthreads();
    if (tid == 0) pt_cta_end(0);
#endif
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
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w][0], 128);
      mbar_init(&p_full[w][1], 128);
      mbar_init(&o_done[w], 1);
    }
    mbar_init(&q_full, 32 * kSoftWarps);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(&tmem_base_s, C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  // ---- tiles with at least one causally visible key, in list order; a tile
  // every row of the CTA sees whole (all groups valid and below min_q) skips
  // the per-element mask
  const int n_tiles = (n_ent * a.P + kKeys - 1) / kKeys;
  if (warp == 0) {
    int n_act = 0;
    for (int j0 = 0; j0 < n_tiles; j0 += 32) {
      const int j = j0 + lane;
      bool live = false, whole = true;
      if (j < n_tiles)
        for (int g = 0; g < kGroups; ++g) {
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
#if SA_PREFILL_TIMELINE
  if (tid == 0 && pt_row) pt_row[11] = n_act;
#endif

  if (warp == kProdWarp) {
    // ================= producer: TMA gathers of K and V tiles
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
      for (int jj = 0; jj < n_act; ++jj) {
        const int st = jj % C::kStages, j = act_s[jj] >> 1;
        const uint32_t ph = ((jj / C::kStages) - 1) & 1;
        int page[kGroups], row0[kGroups];
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          const int2 gr = group_of(ent_s, n_ent, a.P, j, g);
          const bool ok = gr.x >= 0 && gr.y < L;
          // an out-of-range page coordinate makes TMA write zeros for the box
          page[g] = ok ? gr.x : a.P_pool;
          row0[g] = ok ? gr.y % a.P : 0;
        }
        // K(jj) waits for QK^T of tile jj - kStages, V(jj) for its PV
        if (jj >= C::kStages && !wait_or_abort(&k_empty[st], ph, abort_flag)) break;
        uint8_t* kt = k_s + st * C::kTileBytes;
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(kt + c * (kKeys * 128) + g * 2048, &kmap, &k_full[st], c * 64, row0[g],
                        kvh, page[g]);
        if (jj >= C::kStages && !wait_or_abort(&v_empty[st], ph, abort_flag)) break;
        uint8_t* vt = v_s + st * C::kTileBytes;
        mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(vt + c * (kKeys * 128) + g * 2048, &vmap, &v_full[st], c * 64, row0[g],
                        kvh, page[g]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer (one thread)
    if (lane == 0 && n_act > 0) {
      const uint32_t q_addr = smem_u32(q_s), k_addr = smem_u32(k_s), v_addr = smem_u32(v_s);
      // S_w = Q_w K^T for tile jj into columns [128w, 128w + 128)
      auto qk = [&](int jj, int w) {
        const uint32_t kbase = k_addr + (jj % C::kStages) * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = tc::sdesc_sw128(
              q_addr + w * C::kQBytes + (kk >> 2) * (kM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              tc::sdesc_sw128(kbase + (kk >> 2) * (kKeys * 128) + (kk & 3) * 32, 16, 1024);
          tc::mma_bf16(tmem + 128 * w, ad, bd, C::kIdQK, kk > 0 ? 1u : 0u);
        }
        tc::commit(&s_full[w]);
      };
      // O_w += P_w V over keys [64h, 64h + 64) of tile jj: P hi, then lo, of 16
      // keys kk from columns 128w + 16 kk (+ 8 for lo)
      auto pv = [&](int jj, int w, int h) {
        const uint32_t vbase = v_addr + (jj % C::kStages) * C::kTileBytes;
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
          const uint64_t bd = tc::sdesc_sw128(vbase + kk * 2048, kKeys * 128, 1024);
          const uint32_t hi = tmem + 128 * w + 16 * kk;
          tc::mma_bf16_ts(tmem + 256 + D * w, hi, bd, C::kIdPV, (jj > 0 || kk > 0) ? 1u : 0u);
          tc::mma_bf16_ts(tmem + 256 + D * w, hi + 8, bd, C::kIdPV, 1u);
        }
      };
      bool ok = wait_or_abort(&q_full, 0, abort_flag) && wait_or_abort(&k_full[0], 0, abort_flag);
#if SA_PREFILL_TIMELINE
      pt_mark(0, 0);
#endif
      tc::fence_after_sync();
      if (ok) {
        qk(0, 0);
        qk(0, 1);
        tc::commit(&k_empty[0]);
#if SA_PREFILL_TIMELINE
        pt_mark(0, 1);
#endif
      }
      for (int jj = 0; ok && jj < n_act; ++jj) {
        const int st = jj % C::kStages;
        for (int w = 0; ok && w < 2; ++w) {
          for (int h = 0; h < 2; ++h) {
            if (!wait_or_abort(&p_full[w][h], jj & 1, abort_flag) ||
                (w == 0 && h == 0 &&
                 !wait_or_abort(&v_full[st], (jj / C::kStages) & 1, abort_flag))) {
              ok = false;
              break;
            }
#if SA_PREFILL_TIMELINE
            if (h == 1) pt_mark(jj, 2 + w);
#endif
            tc::fence_after_sync();
            pv(jj, w, h);
          }
          if (!ok) break;
          if (w == 1) tc::commit(&v_empty[st]);
          if (jj + 1 < n_act) {
            const int st1 = (jj + 1) % C::kStages;
            if (w == 0) {
              if (!wait_or_abort(&k_full[st1], ((jj + 1) / C::kStages) & 1, abort_flag)) {
                ok = false;
                break;
              }
#if SA_PREFILL_TIMELINE
              pt_mark(jj + 1, 0);
#endif
              tc::fence_after_sync();
            }
            qk(jj + 1, w);
            if (w == 1) {
              tc::commit(&k_empty[st1]);
#if SA_PREFILL_TIMELINE
              pt_mark(jj + 1, 1);
#endif
            }
          } else {
            tc::commit(&o_done[w]);
          }
        }
      }
    }
  } else {
    // ================= softmax / epilogue: two threads per query row, one per
    // 64-key half of every tile (warps 0-7 tile A, 8-15 tile B; in each, warps
    // 0-3 take keys 0-63 and warps 4-7 keys 64-127 of the same rows, so that
    // four softmax warps share each sub-partition and hide one another's
    // latency).  The two halves of a row swap their partial maxima through
    // shared memory under a named barrier of their two warps.
    const int wg = warp >> 3;                       // tile A (0) or B (1)
    const int kh = (warp >> 2) & 1;                 // key half
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;              // row within the tile = TMEM lane
    const int rg = r0 + wg * kM + r;
    const bool row_ok = rg < rows_total;
    const int t = row_ok ? rg / nh : 0;
    const int head = prm.pairs.heads[prm.pairs.head_off[pair] + (row_ok ? rg % nh : 0)];
    const int qpos = row_ok ? qb + t : -1;
    uint8_t* qt_s = q_s + wg * C::kQBytes;
    {   // this thread's half of the row's 16-byte pieces
      const uint4* src = reinterpret_cast<const uint4*>(a.q + b * a.qs0 + t * a.qs1 + head * a.qs2);
#pragma unroll
      for (int pc = kh * (D / 16); pc < (kh + 1) * (D / 16); ++pc) {
        const int c = pc >> 3, ch = pc & 7;
        const uint4 v = row_ok ? src[pc] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qt_s + c * (kM * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
      }
    }
    tc::fence_proxy_async();
    mbar_arrive(&q_full);
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = 128 * wg + 64 * kh;      // this half's 64 score columns
    const uint32_t o_col = 256 + D * wg + (D / 2) * kh;   // and its half of O
    const int pair_bar = 1 + wg * 4 + quarter;      // the two warps of these rows
    const float sl = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // (after an abort the loop still runs to its end, skipping the work, so
    // that the partner warp's barrier sees every arrival it counts on)
    for (int jj = 0; jj < n_act; ++jj) {
      const int code = act_s[jj], j = code >> 1;
      const bool masked = code & 1;
      // visibility of this half's keys for this row, one bit per key (before
      // the wait: it needs only the list).  A group's keys are consecutive
      // positions: key c of group g is visible iff the group is valid and
      // c < min(L, qpos + 1) - (its first position).
      uint32_t vis[2];
      if (masked) {
        const int vis_end = min(L, qpos + 1);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          uint32_t bits = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int2 gr = group_of(ent_s, n_ent, a.P, j, 4 * kh + 2 * w + h);
            const int lim = gr.x >= 0 ? min(max(vis_end - gr.y, 0), 16) : 0;
            bits |= ((1u << lim) - 1u) << (16 * h);
          }
          vis[w] = bits;
        }
      }
      ok = __all_sync(0xffffffffu, ok && wait_or_abort(&s_full[wg], jj & 1, abort_flag));
#if SA_PREFILL_TIMELINE
      if (r == 0 && kh == 0) pt_mark(jj, 4 + 3 * wg);
#endif
      // The tiles take turns -- A(j) after B(j-1), B(j) after A(j) -- so that
      // one tile's softmax runs while the tensor core works on the other's
      // PV and QK^T, instead of both sharing the sub-partitions at once.
      if (wg == 0) {
        if (jj > 0) turn_wait<kTurnB>();
      } else {
        turn_wait<kTurnA>();
      }
      // the row max of the scaled scores from the raw ones: x -> x s is monotone
      // (rounding included), so it is s max(x) for s >= 0 and s min(x) for s < 0;
      // invisible keys are NaN here (ignored by the reductions, p = 0 below)
      float part = NAN;
      if (ok) {
        tc::fence_after_sync();
        float x[64];
        tc::ld32(tmem + lane_base + s_col, *reinterpret_cast<float(*)[32]>(&x[0]));
        tc::ld32(tmem + lane_base + s_col + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
        tc::wait_ld();
        if (masked) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (!((vis[k >> 5] >> (k & 31)) & 1u)) x[k] = NAN;
        }
        part = sl >= 0.f ? reduce_n<false>(x) : reduce_n<true>(x);
      }
      pmax_s[jj & 1][wg][kh][r] = part;
      named_sync(pair_bar, 64);
      const float other = pmax_s[jj & 1][wg][kh ^ 1][r];
#if SA_PREFILL_TIMELINE
      if (r == 0 && kh == 0) pt_mark(jj, 12 + 2 * wg);
#endif
      if (ok) {
        const float mr = sl >= 0.f ? fmaxf(part, other) : fminf(part, other);
        const float mx = mr != mr ? -INFINITY : mr * sl;
        const bool move = mx > m_ref + kLazyP;
        const float m_new = move ? mx : m_ref;
        const float nb = m_new == -INFINITY ? 0.f : -m_new;
        // this half of O is rescaled before any of this tile's P is handed
        // over; PV of the previous tile, its last writer, completed before
        // these scores arrived
        if (__any_sync(0xffffffffu, move)) {
          const float alpha = move ? exp2f(m_ref - mx) : 1.f;
          l *= alpha;
          if (jj >= 1) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              float o[32];
              tc::ld32(tmem + lane_base + o_col + c * 32, o);
              tc::wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= alpha;
              tc::st32(tmem + lane_base + o_col + c * 32, o);
            }
          }
        }
        m_ref = m_new;
#if SA_PREFILL_TIMELINE
        if (r == 0 && kh == 0) pt_mark(jj, 13 + 2 * wg);
#endif
        // P = 2^(x sl - m_new) as bf16 hi + lo pairs over this half's scores
        // in TMEM, 16 keys at a time (8 columns of hi pairs, then 8 of lo
        // pairs); the scores are read a second time, 32 columns at a time (the
        // other warps of the sub-partition cover the read's latency).  Key
        // pairs in packed float32 (the same roundings as the scalar ops); the
        // row sum in eight chains.
        unsigned long long ls2[4] = {0ull, 0ull, 0ull, 0ull};
        const unsigned long long sl2 = f2_pack(sl, sl), nb2 = f2_pack(nb, nb);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float yc[32];
          tc::ld32(tmem + lane_base + s_col + 32 * c, yc);
          tc::wait_ld();
          const uint32_t vb = masked ? vis[c] : 0xffffffffu;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t ph[8], pl[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int k = 16 * q + 2 * i;        // key within the 32-column chunk
              const float2 z = f2_unpack(f2_fma(f2_pack(yc[k], yc[k + 1]), sl2, nb2));
              float p0 = ex2_approx(z.x), p1 = ex2_approx(z.y);
              if (masked) {
                p0 = (vb >> k) & 1u ? p0 : 0.f;
                p1 = (vb >> (k + 1)) & 1u ? p1 : 0.f;
              }
              const unsigned long long pp = f2_pack(p0, p1);
              ls2[i & 3] = f2_add(ls2[i & 3], pp);
              // hi = p truncated to bf16 (its low 16 bits cleared), lo = p - hi
              // (exact in float32) truncated likewise: integer and byte-permute
              // instructions only, no conversions
              const float h0 = __uint_as_float(__float_as_uint(p0) & 0xffff0000u);
              const float h1 = __uint_as_float(__float_as_uint(p1) & 0xffff0000u);
              const float2 d = f2_unpack(f2_sub(pp, f2_pack(h0, h1)));
              ph[i] = __byte_perm(__float_as_uint(p0), __float_as_uint(p1), 0x7632);
              pl[i] = __byte_perm(__float_as_uint(d.x), __float_as_uint(d.y), 0x7632);
            }
            tc::st8(tmem + lane_base + s_col + 32 * c + 16 * q, ph);
            tc::st8(tmem + lane_base + s_col + 32 * c + 16 * q + 8, pl);
          }
        }
        tc::wait_st();
        tc::fence_before_sync();
        mbar_arrive(&p_full[wg][kh]);
#if SA_PREFILL_TIMELINE
        if (r == 0 && kh == 0) pt_mark(jj, 5 + 3 * wg);
        if (r == 0 && kh == 1) pt_mark(jj, 6 + 3 * wg);
#endif
        float ls[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 v = f2_unpack(ls2[i]);
          ls[2 * i] = v.x;
          ls[2 * i + 1] = v.y;
        }
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      }
      if (wg == 0)
        turn_pass<kTurnA>();
      else
        turn_pass<kTurnB>();
    }
    // tile B's last pass is taken here, so that no arrival is left pending
    if (wg == 0 && n_act > 0) turn_wait<kTurnB>();
    if (ok && n_act > 0) ok = wait_or_abort(&o_done[wg], 0, abort_flag);
    tc::fence_after_sync();
    // ---- epilogue: the row sum and status from both halves, then this half's
    // columns of O / l, and the LSE (from the first half's thread)
    lsum_s[wg][kh][r] = l;
    okay_s[wg][kh][r] = ok ? 1 : 0;
    named_sync(pair_bar, 64);
    const float lt = lsum_s[wg][0][r] + lsum_s[wg][1][r];
    const bool both_ok = okay_s[wg][0][r] && okay_s[wg][1][r];
    const bool empty = !both_ok || n_act == 0 || lt == 0.f;
    const float inv = empty ? 0.f : 1.f / lt;
    float* dst = a.o_part + ((((int64_t)split * a.B + b) * a.T + t) * a.Hq + head) * D +
                 (D / 2) * kh;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
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
    if (row_ok && kh == 0)
      a.lse_part[(((int64_t)split * a.B + b) * a.T + t) * a.Hq + head] =
          empty ? -INFINITY : (m_ref + log2f(lt)) * kLn2;
    if (!ok && lane == 0) set_dev_error(a.err, SA_DEVERR_TIMEOUT);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
#if SA_PREFILL_TIMELINE
  if (tid == 0) pt_cta_end(n_act);
#endif
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

#if SA_PREFILL_TIMELINE
// Diagnostic build only: copies the per-CTA records ([8192][4] int64: entry and
// exit %globaltimer, active tiles, SM id; unlaunched CTAs stay 0) to host memory
// `out` (n entries at most) and clears them.
extern "C" SA_API int sa_prefill_cta_timeline(long long* out, int n) {
  const int total = sa::kPtAll * 4;
  if (!out || n <= 0) return SA_ERR_INVALID_ARG;
  const size_t bytes = sizeof(long long) * (size_t)(n < total ? n : total);
  if (cudaMemcpyFromSymbol(out, sa::g_prefill_cta, bytes) != cudaSuccess) return SA_ERR_CUDA;
  void* dev = nullptr;
  if (cudaGetSymbolAddress(&dev, sa::g_prefill_cta) != cudaSuccess ||
      cudaMemset(dev, 0, sizeof(long long) * total) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}
// Diagnostic build only: copies the recorded stamps ([kPtCtas][kPtIters][16]
// int64, SM clocks) to host memory `out` (n entries at most) and clears them.
extern "C" SA_API int sa_prefill_timeline(long long* out, int n) {
  const int total = sa::kPtCtas * sa::kPtIters * sa::kPtSlots;
  if (!out || n <= 0) return SA_ERR_INVALID_ARG;
  const size_t bytes = sizeof(long long) * (size_t)(n < total ? n : total);
  if (cudaMemcpyFromSymbol(out, sa::g_prefill_tl, bytes) != cudaSuccess) return SA_ERR_CUDA;
  void* dev = nullptr;
  if (cudaGetSymbolAddress(&dev, sa::g_prefill_tl) != cudaSuccess ||
      cudaMemset(dev, 0, sizeof(long long) * total) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}
#endif
