// Host-side declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/sa.h"

namespace sa {

// Launch `kern` as a programmatic dependent of the preceding work in `stream`:
// its CTAs may be scheduled while the preceding kernel finishes; the kernel
// itself waits (pdl_wait_and_release) before touching memory.  Off by default
// (-DSA_PDL=1 turns it on): inside a CUDA graph the measured step time was the
// same or slightly worse with it.
#ifndef SA_PDL
#define SA_PDL 0
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = SA_PDL ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- host-side set-up done once per CUDA context, not once per call
// (a context created anew, after cudaDeviceReset say, is set up again).
// Unique id of the calling thread's current context; 0 if it cannot be read
// (then nothing is cached and every call does the set-up).
unsigned long long current_context_id();
// Let `kern` request up to the device's opt-in maximum of dynamic shared
// memory (a cap only: what a launch uses is what it asks for).
cudaError_t allow_max_dyn_smem(const void* kern);
// Ask for the largest shared-memory carveout for `kern` (more resident CTAs
// when they are limited by shared memory).
cudaError_t prefer_max_carveout(const void* kern);
// Streaming multiprocessors of the current device.
cudaError_t sm_count(int* out);
// Resident CTAs of `kern` per SM at this block size and dynamic shared memory.
cudaError_t max_blocks_per_sm(const void* kern, int threads, size_t dyn_smem, int* out);

constexpr int kMaxPairs = 64;        // (list, kv head) pairs one decode call may touch
constexpr int kMaxHeadsPerPair = 128;
constexpr int kMaxHeads = 256;       // query heads of a decode call
constexpr int kMaxRowsPerPair = 16;  // query rows (T x heads) one warp-MMA tile holds
constexpr int kMaxSplitEntries = 1024;

// Which heads of a call read which (list, kv head) pair; built on the host
// from head_to_list so every CTA knows its query rows without a lookup.
struct PairTable {
  int n_pairs;
  int list_of[kMaxPairs];
  int kvh_of[kMaxPairs];
  int n_heads[kMaxPairs];
  int head_off[kMaxPairs];     // pair i's heads: heads[head_off[i] .. + n_heads[i])
  int16_t heads[kMaxHeads];
};

// A batch's logical -> physical page map.  Flat (blocks null): table is
// [B, stride] physical page ids.  Two-level (the working-set-sized layout):
// table is a directory [B, stride] of block ids, block j of a row covering
// logical pages [j << shift, (j + 1) << shift), and blocks [n_blocks,
// 1 << shift] holds the physical ids; a directory entry outside [0, n_blocks)
// (-1: no block) resolves to -1.  Capacity in logical pages: stride (flat) or
// stride << shift.
struct PageMap {
  const int32_t* table = nullptr;
  const int32_t* blocks = nullptr;
  int stride = 0;
  int shift = 0;
  int n_blocks = 0;
};
inline PageMap flat_map(const int32_t* table, int max_pages) {
  PageMap m;
  m.table = table;
  m.stride = max_pages;
  return m;
}
#ifdef __CUDACC__
__device__ __forceinline__ int page_at(const PageMap& m, int b, int p) {
  if (!m.blocks) return m.table[(int64_t)b * m.stride + p];
  const int blk = m.table[(int64_t)b * m.stride + (p >> m.shift)];
  if (blk < 0 || blk >= m.n_blocks) return -1;
  return m.blocks[((int64_t)blk << m.shift) + (p & ((1 << m.shift) - 1))];
}
#endif

struct DecodeArgs {
  const uint16_t* q;
  int64_t qs0, qs1, qs2;
  PageMap pt;
  int max_pages;          // logical pages a sequence may hold (the map's capacity)
  const int32_t* seq_lens;
  const int32_t* lists;
  const int32_t* counts;
  int n_lists, max_list;
  int B, T, Hq, Hkv, Dk, Dv, P, P_pool;
  float scale_log2;
  int n_splits;
  float* o_part;
  float* lse_part;
  int32_t* err;
  const float* k_scale;   // FP8 pages: [P_pool, Hkv] float32 scales (null for bf16 pages)
  const float* v_scale;
  const int32_t* q_pos;   // [B] position of query token 0 (null: the causal tail L - T)
};

// Position of query token 0 of sequence b of length L (token t sits at this
// + t and sees the keys at positions up to its own): the caller's q_pos[b],
// else the causal tail L - T.
__host__ __device__ inline int query_base(const DecodeArgs& a, int b, int L) {
  return a.q_pos ? a.q_pos[b] : L - a.T;
}

// Encode a 4-D bf16 tensor map over a [P_pool, Hkv, P, D] cache with
// 64-column x box_rows-row boxes (box_rows 16 or 64, at most P) and 128-byte
// swizzle.  false on failure.
bool encode_kv_map(CUtensorMap* map, const void* base, int D, int P, int Hkv, int P_pool,
                   const int64_t strides[4], int box_rows = 16);
// The same over FP8 (one byte per element) pages, D == 128: 128-column x 16-row
// boxes (128-byte rows), 128-byte swizzle.
bool encode_kv_map_u8(CUtensorMap* map, const void* base, int D, int P, int Hkv, int P_pool,
                      const int64_t strides[4]);

int decode_max_split_entries();
int prefill_max_split_entries();
int mla_max_split_entries(int P);
cudaError_t launch_mla(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                       cudaStream_t stream);
cudaError_t launch_prefill(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, cudaStream_t stream);
int decode_warps_per_cta();
// Split count for n_units (sequence, list) pairs of up to max_list pages with
// head dim D: the splits that fill one wave of resident decode warps, at least
// enough that no split exceeds a warp's list capacity, at most 64.
cudaError_t decode_default_splits(int D, int n_units, int max_list, int* out);
cudaError_t launch_decode_gqa(const DecodeArgs& a, const PairTable& pairs, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, cudaStream_t stream);
cudaError_t launch_decode_gqa_fp8(const DecodeArgs& a, const PairTable& pairs,
                                  const CUtensorMap& kmap, const CUtensorMap& vmap,
                                  cudaStream_t stream);

struct SelectArgs {
  const uint16_t* q;
  int64_t qs0, qs1, qs2;
  const uint16_t* sig;
  PageMap pt;
  const int32_t* seq_lens;
  int B, T, Hq, Hkv, Dk, P, max_pages, P_pool;
  int n_sink, n_local, budget_pages, k_top;
  int32_t* out_pages;
  int32_t* out_counts;
  float2* lohi;      // workspace: [B, Hkv, max_pages] score bounds
  int32_t* err;
};
size_t select_workspace_bytes(int B, int Hkv, int max_pages);
cudaError_t launch_select_gqa(const SelectArgs& a, cudaStream_t stream);
size_t select_static_capacity();
cudaError_t launch_select_gqa_static(SelectArgs a, cudaStream_t stream);

struct TieredArgs {
  const uint16_t* q;
  int64_t qs0, qs1, qs2;
  const uint16_t* sig;       // [P_pool, 1, Dk]
  const int32_t* page_table;
  const int32_t* seq_lens;
  int B, T, Hq, Dk, P, max_pages, P_pool, alpha, beta;
  int n_rg;                  // query-row groups of the scoring pass (set by the launcher)
  float2* lohi;              // workspace [B, n_rg, max_pages] score brackets
  unsigned long long* rmask; // workspace [B, n_rg, max_pages] candidate rows (set by the launcher)
  unsigned long long* exkey; // workspace [B, max_pages] exact scores (order keys)
  unsigned int* counter;     // workspace [B] CTAs done with the exact rescoring
  int32_t* lists;            // [B, 2, alpha + beta]
  int32_t* counts;           // [B, 2]
  int32_t* err;
};
size_t tiered_workspace_bytes(int B, int T, int Hq, int max_pages);
cudaError_t launch_select_tiered(TieredArgs a, cudaStream_t stream);

cudaError_t launch_combine(const float* o_part, const float* lse_part, int n_splits, int64_t rows,
                           int Dv, float* o_out, uint16_t* o_bf16, float* lse_out,
                           cudaStream_t stream);

// max_pages: the map's capacity in logical pages
cudaError_t launch_summaries_fp8(const uint8_t* k, const int64_t ks[4], const float* k_scale,
                                 const PageMap& pt, int max_pages, const int32_t* seq_lens, int B,
                                 int Hkv, int Dk, int P, int P_pool, uint16_t* sig, int32_t* err,
                                 cudaStream_t stream);
cudaError_t launch_summaries(const uint16_t* k, const int64_t ks[4], const PageMap& pt,
                             int max_pages, const int32_t* seq_lens, int B, int Hkv, int Dk,
                             int P, int P_pool, int n_new, uint16_t* sig, int32_t* err,
                             cudaStream_t stream);

struct HeadArgs {
  const uint16_t* q;       // [B, T, Hq, Dk]
  int64_t qs0, qs1, qs2;
  const uint16_t* sig;     // [P_pool, 1, Dk]
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  const int32_t* lists;    // [B, 2, cap]: critical, critical + ambient
  const int32_t* counts;   // [B, 2]
  int cap;
  int B, T, Hq, Dk, P, P_pool;
  float scale;
  int h_keep;
  int n_chunks;            // set by the launcher
  double* part;            // workspace [B, n_chunks, T*Hq, 3]
  int32_t* heads_out;      // [h_keep]
  double* scores_out;      // [Hq] (optional)
  int32_t* err;
};
size_t head_workspace_bytes(int B, int T, int Hq, int max_pages);
int head_max_dk();
cudaError_t launch_select_heads(HeadArgs a, cudaStream_t stream);

struct AppendArgs {
  const uint16_t* k_new;   // [B, max_new, Hkv, D]
  int64_t kn0, kn1, kn2;
  const uint16_t* v_new;
  int64_t vn0, vn1, vn2;
  const int32_t* n_new;    // [B]
  int max_new;
  uint16_t* k_cache;       // [P_pool, Hkv, P, D]
  int64_t ks0, ks1, ks2;
  uint16_t* v_cache;
  int64_t vs0, vs1, vs2;
  PageMap pt;
  int max_pages;           // the map's capacity in logical pages
  const int32_t* seq_lens;
  int32_t* out_seq_lens;
  int B, Hkv, D, P, P_pool;
  uint16_t* sig;           // [P_pool, Hkv, D]
  int32_t* err;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

cudaError_t launch_block_union(const float* scores, int Hq, int Hkv, int NQB, int NKB, int q_off,
                               int top_k, int n_sink, int32_t* tables, int32_t* counts,
                               cudaStream_t stream);

}  // namespace sa
