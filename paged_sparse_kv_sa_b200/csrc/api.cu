// C ABI: argument checks on the host, then kernel launches.  Nothing here
// allocates device memory or synchronises.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <map>
#include <mutex>

#include "internal.h"

namespace sa {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Checks shared by the bf16 [*, Hkv, P, D] caches: feature stride 1, the
// other strides multiples of 8 elements (16 bytes), 16-byte aligned base.
int check_cache(const uint16_t* p, const int64_t s[4]) {
  if (!p || !s) return SA_ERR_INVALID_ARG;
  if (!aligned16(p) || s[3] != 1) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (s[i] <= 0 || (s[i] % 8) != 0) return SA_ERR_INVALID_ARG;
  return SA_OK;
}

int check_q(const uint16_t* q, const int64_t s[4]) {
  if (!q || !s) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || s[3] != 1) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (s[i] < 0 || (s[i] % 8) != 0) return SA_ERR_INVALID_ARG;
  return SA_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// The (list, kv head) pairs a decode call reads, the heads of each (in head
// order) and the most query rows (T x heads) one pair holds.
int build_pairs(const int32_t* head_to_list, int Hq, int Hkv, int T, PairTable* out,
                int* max_rows_out) {
  if (Hq > kMaxHeads) return SA_ERR_UNSUPPORTED;
  PairTable& pairs = *out;
  pairs.n_pairs = 0;
  const int G = Hq / Hkv;
  int pair_of[kMaxHeads];
  for (int kvh = 0; kvh < Hkv; ++kvh) {
    for (int h = kvh * G; h < (kvh + 1) * G; ++h) {
      const int l = head_to_list[h];
      int pi = -1;
      for (int i = 0; i < pairs.n_pairs; ++i)
        if (pairs.list_of[i] == l && pairs.kvh_of[i] == kvh) pi = i;
      if (pi < 0) {
        if (pairs.n_pairs == kMaxPairs) return SA_ERR_UNSUPPORTED;
        pi = pairs.n_pairs++;
        pairs.list_of[pi] = l;
        pairs.kvh_of[pi] = kvh;
        pairs.n_heads[pi] = 0;
      }
      if (pairs.n_heads[pi] == kMaxHeadsPerPair) return SA_ERR_UNSUPPORTED;
      ++pairs.n_heads[pi];
      pair_of[h] = pi;
    }
  }
  int max_rows = 0;
  for (int i = 0, off = 0; i < pairs.n_pairs; ++i) {
    pairs.head_off[i] = off;
    off += pairs.n_heads[i];
    max_rows = max_rows > pairs.n_heads[i] * T ? max_rows : pairs.n_heads[i] * T;
    pairs.n_heads[i] = 0;   // refilled below, in head order
  }
  for (int h = 0; h < Hq; ++h) {
    const int pi = pair_of[h];
    pairs.heads[pairs.head_off[pi] + pairs.n_heads[pi]++] = static_cast<int16_t>(h);
  }
  *max_rows_out = max_rows;
  return SA_OK;
}

// FP8 pages: 16-byte aligned base, unit feature stride, other strides
// positive multiples of 16 bytes (= 16 elements).
int check_cache_u8(const uint8_t* p, const int64_t s[4]) {
  if (!p || !s) return SA_ERR_INVALID_ARG;
  if (!aligned16(p) || s[3] != 1) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (s[i] <= 0 || (s[i] % 16) != 0) return SA_ERR_INVALID_ARG;
  return SA_OK;
}


}  // namespace

unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

namespace {
// Values computed once per (context, what, kernel, argument).
struct CacheKey {
  unsigned long long ctx;
  int what;
  const void* fn;
  long long arg;
  bool operator<(const CacheKey& o) const {
    if (ctx != o.ctx) return ctx < o.ctx;
    if (what != o.what) return what < o.what;
    if (fn != o.fn) return fn < o.fn;
    return arg < o.arg;
  }
};
std::mutex g_cache_mu;
std::map<CacheKey, int> g_cache;

template <typename F>
cudaError_t cached(int what, const void* fn, long long arg, int* out, F&& compute) {
  // make sure a context exists before its id is read
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long ctx = current_context_id();
  const CacheKey key{ctx, what, fn, arg};
  if (ctx) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    auto it = g_cache.find(key);
    if (it != g_cache.end()) {
      *out = it->second;
      return cudaSuccess;
    }
  }
  int v = 0;
  e = compute(dev, &v);
  if (e != cudaSuccess) return e;
  if (ctx) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    g_cache[key] = v;
  }
  *out = v;
  return cudaSuccess;
}
}  // namespace

cudaError_t allow_max_dyn_smem(const void* kern) {
  int unused = 0;
  return cached(0, kern, 0, &unused, [&](int dev, int* v) {
    cudaFuncAttributes fa;
    int optin = 0;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               optin - (int)fa.sharedSizeBytes);
    *v = 1;
    return e;
  });
}

cudaError_t prefer_max_carveout(const void* kern) {
  int unused = 0;
  return cached(1, kern, 0, &unused, [&](int, int* v) {
    *v = 1;
    return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
}

cudaError_t sm_count(int* out) {
  return cached(2, nullptr, 0, out, [](int dev, int* v) {
    return cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
  });
}

cudaError_t max_blocks_per_sm(const void* kern, int threads, size_t dyn_smem, int* out) {
  const long long arg = ((long long)threads << 32) | (long long)dyn_smem;
  return cached(3, kern, arg, out, [&](int, int* v) {
    cudaError_t e = allow_max_dyn_smem(kern);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, kern, threads, dyn_smem);
  });
}

bool encode_kv_map(CUtensorMap* map, const void* base, int D, int P, int Hkv, int P_pool,
                   const int64_t strides[4], int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)Hkv, (cuuint64_t)P_pool};
  cuuint64_t gstr[3] = {(cuuint64_t)strides[2] * 2, (cuuint64_t)strides[1] * 2,
                        (cuuint64_t)strides[0] * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, gstr,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_kv_map_u8(CUtensorMap* map, const void* base, int D, int P, int Hkv, int P_pool,
                      const int64_t strides[4]) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)Hkv, (cuuint64_t)P_pool};
  cuuint64_t gstr[3] = {(cuuint64_t)strides[2], (cuuint64_t)strides[1], (cuuint64_t)strides[0]};
  cuuint32_t box[4] = {128, 16, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, gstr, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sa

using namespace sa;

extern "C" {

const char* sa_status_string(int status) {
  switch (status) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    default: return "SA_ERR_UNKNOWN";
  }
}

int sa_abi_version(void) { return 100; }

size_t sa_select_workspace_size(int B, int Hkv, int max_pages) {
  if (B <= 0 || Hkv <= 0 || max_pages <= 0) return 0;
  return select_workspace_bytes(B, Hkv, max_pages);
}

}  // extern "C"

namespace {
// Argument checks and argument block shared by the selection entry points.
int select_args(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                const PageMap& pm, const int32_t* seq_lens, int B, int T, int Hq, int Hkv,
                int Dk, int page_size, int max_pages, int P_pool, int sink_tokens,
                int local_tokens, int budget_tokens, int32_t* out_pages, int32_t* out_counts,
                int32_t* dev_error, SelectArgs* a) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Dk <= 0 || page_size <= 0 ||
      max_pages < 0 || P_pool < 0 || sink_tokens < 0 || local_tokens < 0 || budget_tokens < 0)
    return SA_ERR_INVALID_ARG;
  const int n_sink = (sink_tokens + page_size - 1) / page_size;
  const int n_local = (local_tokens + page_size - 1) / page_size;
  const int budget_pages = budget_tokens / page_size;
  const int k_top = budget_pages - n_sink - n_local;
  if (k_top < 0 || budget_pages <= 0) return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (int r = check_q(q, q_strides)) return r;
  if (!summaries || !pm.table || !seq_lens || !out_pages || !out_counts)
    return SA_ERR_INVALID_ARG;
  if (!aligned16(summaries)) return SA_ERR_INVALID_ARG;
  if (Dk != 64 && Dk != 128 && Dk != 256) return SA_ERR_UNSUPPORTED;
  if (T * (Hq / Hkv) > 16 || max_pages > 16384) return SA_ERR_UNSUPPORTED;
  a->q = q;
  a->qs0 = q_strides[0];
  a->qs1 = q_strides[1];
  a->qs2 = q_strides[2];
  a->sig = summaries;
  a->pt = pm;
  a->seq_lens = seq_lens;
  a->B = B;
  a->T = T;
  a->Hq = Hq;
  a->Hkv = Hkv;
  a->Dk = Dk;
  a->P = page_size;
  a->max_pages = max_pages;
  a->P_pool = P_pool;
  a->n_sink = n_sink;
  a->n_local = n_local;
  a->budget_pages = budget_pages;
  a->k_top = k_top;
  a->out_pages = out_pages;
  a->out_counts = out_counts;
  a->lohi = nullptr;
  a->err = dev_error;
  return SA_OK;
}
}  // namespace

extern "C" {

int sa_select_pages(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                    const int32_t* page_table, const int32_t* seq_lens, int B, int T, int Hq,
                    int Hkv, int Dk, int page_size, int max_pages, int P_pool, int sink_tokens,
                    int local_tokens, int budget_tokens, int32_t* out_pages, int32_t* out_counts,
                    void* workspace, size_t workspace_bytes, int32_t* dev_error, void* stream) {
  SelectArgs a;
  if (int r = select_args(q, q_strides, summaries, flat_map(page_table, max_pages), seq_lens, B,
                          T, Hq, Hkv, Dk,
                          page_size, max_pages, P_pool, sink_tokens, local_tokens, budget_tokens,
                          out_pages, out_counts, dev_error, &a))
    return r;
  if (B == 0) return SA_OK;
  if (a.k_top > 0 && (!workspace || !aligned16(workspace) ||
                      workspace_bytes < select_workspace_bytes(B, Hkv, max_pages)))
    return SA_ERR_WORKSPACE;
  a.lohi = static_cast<float2*>(workspace);
  return cuda_status(launch_select_gqa(a, static_cast<cudaStream_t>(stream)));
}

int sa_select_pages_no_alloc(const uint16_t* q, const int64_t q_strides[4],
                             const uint16_t* summaries, const int32_t* page_table,
                             const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int Dk,
                             int page_size, int max_pages, int P_pool, int sink_tokens,
                             int local_tokens, int budget_tokens, int32_t* out_pages,
                             int32_t* out_counts, int32_t* dev_error, void* stream) {
  SelectArgs a;
  if (int r = select_args(q, q_strides, summaries, flat_map(page_table, max_pages), seq_lens, B,
                          T, Hq, Hkv, Dk,
                          page_size, max_pages, P_pool, sink_tokens, local_tokens, budget_tokens,
                          out_pages, out_counts, dev_error, &a))
    return r;
  if (B == 0) return SA_OK;
  if ((size_t)B * Hkv * max_pages > select_static_capacity()) return SA_ERR_UNSUPPORTED;
  return cuda_status(launch_select_gqa_static(a, static_cast<cudaStream_t>(stream)));
}

size_t sa_select_tiered_workspace_size(int B, int T, int Hq, int max_pages) {
  if (B <= 0 || T <= 0 || Hq <= 0 || max_pages <= 0) return 0;
  return tiered_workspace_bytes(B, T, Hq, max_pages);
}

int sa_select_pages_tiered(const uint16_t* q, const int64_t q_strides[4],
                           const uint16_t* summaries, const int32_t* page_table,
                           const int32_t* seq_lens, int B, int T, int Hq, int Dk, int page_size,
                           int max_pages, int P_pool, int alpha, int beta, int32_t* lists,
                           int32_t* list_counts, void* workspace, size_t workspace_bytes,
                           int32_t* dev_error, void* stream) {
  if (B < 0 || T <= 0 || Hq <= 0 || Dk <= 0 || page_size <= 0 || max_pages < 0 || P_pool < 0 ||
      alpha < 0 || beta < 0 || alpha + beta <= 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0 || max_pages == 0) return SA_OK;
  if (int r = check_q(q, q_strides)) return r;
  if (!summaries || !aligned16(summaries) || !page_table || !seq_lens || !lists || !list_counts)
    return SA_ERR_INVALID_ARG;
  if (Dk % 8 != 0 || Dk > 880 || max_pages > 8192 || B > 65535) return SA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < tiered_workspace_bytes(B, T, Hq, max_pages))
    return SA_ERR_WORKSPACE;
  TieredArgs a;
  a.q = q;
  a.qs0 = q_strides[0];
  a.qs1 = q_strides[1];
  a.qs2 = q_strides[2];
  a.sig = summaries;
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Dk = Dk;
  a.P = page_size;
  a.max_pages = max_pages;
  a.P_pool = P_pool;
  a.alpha = alpha;
  a.beta = beta;
  a.n_rg = 0;
  a.lohi = static_cast<float2*>(workspace);
  a.lists = lists;
  a.counts = list_counts;
  a.err = dev_error;
  return cuda_status(launch_select_tiered(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace sa {
namespace {
// Where a merged call puts its final outputs (any of them null).
struct MergeSpec {
  float* o_out;
  uint16_t* o_bf16;
  float* lse_out;
};

int merge_outputs_ok(const MergeSpec& m) {
  if (!m.o_out && !m.o_bf16 && !m.lse_out) return SA_ERR_INVALID_ARG;
  if ((m.o_out && !aligned16(m.o_out)) ||
      (m.o_bf16 && (reinterpret_cast<uintptr_t>(m.o_bf16) & 7u)))
    return SA_ERR_INVALID_ARG;
  return SA_OK;
}

// Workspace of a merged call: the split partials.
struct AttnWs {
  size_t o_bytes, lse_bytes;
};
AttnWs attn_ws(int B, int T, int Hq, int Dv, int n_splits) {
  auto r16 = [](size_t x) { return (x + 15) / 16 * 16; };
  AttnWs w;
  const size_t rows = (size_t)B * T * Hq;
  w.o_bytes = r16(rows * Dv * n_splits * sizeof(float));
  w.lse_bytes = r16(rows * n_splits * sizeof(float));
  return w;
}

// Where a decode call's partials go: the caller's o_partial / lse_partial
// (ws null), or laid out in a merged call's workspace (n_splits slots).
struct DecodeTarget {
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  const int32_t* q_pos = nullptr;   // [B] query token 0's position (null: causal tail)
  PageMap dir;                      // two-level map (dir.blocks set): page_table is its directory
};

int sparse_decode_impl(const uint16_t* q, const int64_t q_strides[4], const uint16_t* k_cache,
                       const int64_t k_strides[4], const uint16_t* v_cache,
                       const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                       const int32_t* seq_lens, const int32_t* lists, const int32_t* list_counts,
                       int n_lists, int max_list, const int32_t* head_to_list, int B, int T,
                       int Hq, int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                       int n_splits, float* o_partial, float* lse_partial, int32_t* dev_error,
                       void* stream, const MergeSpec* merge, DecodeTarget* tgt) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Dk <= 0 || Dv <= 0 ||
      page_size <= 0 || max_pages < 0 || P_pool <= 0 || n_lists <= 0 || max_list < 0 ||
      n_splits <= 0 || !std::isfinite(scale) || !head_to_list)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (int r = check_q(q, q_strides)) return r;
  if (int r = check_cache(k_cache, k_strides)) return r;
  if (int r = check_cache(v_cache, v_strides)) return r;
  if (!page_table || !seq_lens || !lists || !list_counts) return SA_ERR_INVALID_ARG;
  if (!tgt->ws && (!o_partial || !lse_partial || !aligned16(o_partial)))
    return SA_ERR_INVALID_ARG;
  for (int h = 0; h < Hq; ++h)
    if (head_to_list[h] < 0 || head_to_list[h] >= n_lists) return SA_ERR_INVALID_ARG;
  // MLA: keys of 576 columns whose first 512 are the values (V aliases K)
  const bool mla = Dk == 576 && Dv == 512 && k_cache == v_cache &&
                   std::memcmp(k_strides, v_strides, 4 * sizeof(int64_t)) == 0;
  if (!mla && (Dk != Dv || (Dk != 64 && Dk != 128 && Dk != 256))) return SA_ERR_UNSUPPORTED;
  if (page_size % 16 != 0 || page_size > 128) return SA_ERR_UNSUPPORTED;

  // (list, kv head) pairs and the heads that read them
  PairTable pairs;
  int max_rows = 0;
  if (int r = build_pairs(head_to_list, Hq, Hkv, T, &pairs, &max_rows)) return r;
  // Up to 16 query rows per pair: warp-MMA decode; more: the tcgen05 kernel.
  const bool wide = max_rows > kMaxRowsPerPair;
  const int cap = mla ? mla_max_split_entries(page_size)
                      : (wide ? prefill_max_split_entries() : decode_max_split_entries());
  if (!mla && wide && Dk > 128) return SA_ERR_UNSUPPORTED;
  if (tgt->ws) {
    const AttnWs w = attn_ws(B, T, Hq, Dv, n_splits);
    if (tgt->ws_bytes < w.o_bytes + w.lse_bytes) return SA_ERR_WORKSPACE;
    o_partial = reinterpret_cast<float*>(tgt->ws);
    lse_partial = reinterpret_cast<float*>(tgt->ws + w.o_bytes);
  }
  if ((max_list + n_splits - 1) / n_splits > cap) return SA_ERR_UNSUPPORTED;
  CUtensorMap kmap, vmap;
  // MLA tiles of 64 keys: one 64-row box per column chunk when a tile lies in one page
  const int k_box_rows = mla && page_size % 64 == 0 ? 64 : 16;
  if (!encode_kv_map(&kmap, k_cache, Dk, page_size, Hkv, P_pool, k_strides, k_box_rows) ||
      !encode_kv_map(&vmap, v_cache, Dv, page_size, Hkv, P_pool, v_strides))
    return SA_ERR_CUDA;
  DecodeArgs a{};
  a.q = q;
  a.qs0 = q_strides[0];
  a.qs1 = q_strides[1];
  a.qs2 = q_strides[2];
  a.pt = tgt->dir.blocks ? tgt->dir : flat_map(page_table, max_pages);
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.lists = lists;
  a.counts = list_counts;
  a.n_lists = n_lists;
  a.max_list = max_list;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Dk = Dk;
  a.Dv = Dv;
  a.P = page_size;
  a.P_pool = P_pool;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_splits = n_splits;
  a.o_part = o_partial;
  a.lse_part = lse_partial;
  a.err = dev_error;
  a.k_scale = a.v_scale = nullptr;
  a.q_pos = tgt->q_pos;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (merge && (n_splits > 64 || (int64_t)B * T * Hq * (Dv / 4) >= (int64_t(1) << 32)))
    return SA_ERR_UNSUPPORTED;   // the combine kernel's limits
  cudaError_t e = mla ? launch_mla(a, pairs, kmap, st)
                      : (wide ? launch_prefill(a, pairs, kmap, vmap, st)
                              : launch_decode_gqa(a, pairs, kmap, vmap, st));
  if (e == cudaSuccess && merge)
    e = launch_combine(o_partial, lse_partial, n_splits, (int64_t)B * T * Hq, Dv, merge->o_out,
                       merge->o_bf16, merge->lse_out, st);
  return cuda_status(e);
}

int sparse_decode_fp8_impl(const uint16_t* q, const int64_t q_strides[4],
                           const uint8_t* k_codes, const int64_t k_strides[4],
                           const uint8_t* v_codes, const int64_t v_strides[4],
                           const float* k_scale, const float* v_scale, const int32_t* page_table,
                           int max_pages, const int32_t* seq_lens, const int32_t* lists,
                           const int32_t* list_counts, int n_lists, int max_list,
                           const int32_t* head_to_list, int B, int T, int Hq, int Hkv, int D,
                           int page_size, int P_pool, float scale, int n_splits, float* o_partial,
                           float* lse_partial, int32_t* dev_error, void* stream,
                           const MergeSpec* merge, DecodeTarget* tgt) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || page_size <= 0 ||
      max_pages < 0 || P_pool <= 0 || n_lists <= 0 || max_list < 0 || n_splits <= 0 ||
      !std::isfinite(scale) || !head_to_list)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (int r = check_q(q, q_strides)) return r;
  if (int r = check_cache_u8(k_codes, k_strides)) return r;
  if (int r = check_cache_u8(v_codes, v_strides)) return r;
  if (!k_scale || !v_scale || !page_table || !seq_lens || !lists || !list_counts)
    return SA_ERR_INVALID_ARG;
  if (!tgt->ws && (!o_partial || !lse_partial || !aligned16(o_partial)))
    return SA_ERR_INVALID_ARG;
  for (int h = 0; h < Hq; ++h)
    if (head_to_list[h] < 0 || head_to_list[h] >= n_lists) return SA_ERR_INVALID_ARG;
  if (D != 128 || page_size % 16 != 0 || page_size > 128) return SA_ERR_UNSUPPORTED;
  PairTable pairs;
  int max_rows = 0;
  if (int r = build_pairs(head_to_list, Hq, Hkv, T, &pairs, &max_rows)) return r;
  if (max_rows > kMaxRowsPerPair) return SA_ERR_UNSUPPORTED;
  if (tgt->ws) {
    const AttnWs w = attn_ws(B, T, Hq, D, n_splits);
    if (tgt->ws_bytes < w.o_bytes + w.lse_bytes) return SA_ERR_WORKSPACE;
    o_partial = reinterpret_cast<float*>(tgt->ws);
    lse_partial = reinterpret_cast<float*>(tgt->ws + w.o_bytes);
  }
  if ((max_list + n_splits - 1) / n_splits > decode_max_split_entries())
    return SA_ERR_UNSUPPORTED;
  CUtensorMap kmap, vmap;
  if (!encode_kv_map_u8(&kmap, k_codes, D, page_size, Hkv, P_pool, k_strides) ||
      !encode_kv_map_u8(&vmap, v_codes, D, page_size, Hkv, P_pool, v_strides))
    return SA_ERR_CUDA;
  DecodeArgs a{};
  a.q = q;
  a.qs0 = q_strides[0];
  a.qs1 = q_strides[1];
  a.qs2 = q_strides[2];
  a.pt = tgt->dir.blocks ? tgt->dir : flat_map(page_table, max_pages);
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.lists = lists;
  a.counts = list_counts;
  a.n_lists = n_lists;
  a.max_list = max_list;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Dk = D;
  a.Dv = D;
  a.P = page_size;
  a.P_pool = P_pool;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_splits = n_splits;
  a.o_part = o_partial;
  a.lse_part = lse_partial;
  a.err = dev_error;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.q_pos = tgt->q_pos;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (merge && (n_splits > 64 || (int64_t)B * T * Hq * (D / 4) >= (int64_t(1) << 32)))
    return SA_ERR_UNSUPPORTED;   // the combine kernel's limits
  cudaError_t e = launch_decode_gqa_fp8(a, pairs, kmap, vmap, st);
  if (e == cudaSuccess && merge)
    e = launch_combine(o_partial, lse_partial, n_splits, (int64_t)B * T * Hq, D, merge->o_out,
                       merge->o_bf16, merge->lse_out, st);
  return cuda_status(e);
}
}  // namespace
}  // namespace sa

extern "C" {

int sa_sparse_decode(const uint16_t* q, const int64_t q_strides[4], const uint16_t* k_cache,
                     const int64_t k_strides[4], const uint16_t* v_cache,
                     const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                     const int32_t* seq_lens, const int32_t* lists, const int32_t* list_counts,
                     int n_lists, int max_list, const int32_t* head_to_list, int B, int T, int Hq,
                     int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                     int n_splits, float* o_partial, float* lse_partial, int32_t* dev_error,
                     void* stream) {
  DecodeTarget t;
  return sparse_decode_impl(q, q_strides, k_cache, k_strides, v_cache, v_strides, page_table,
                            max_pages, seq_lens, lists, list_counts, n_lists, max_list,
                            head_to_list, B, T, Hq, Hkv, Dk, Dv, page_size, P_pool, scale,
                            n_splits, o_partial, lse_partial, dev_error, stream, nullptr, &t);
}

int sa_sparse_decode_fp8(const uint16_t* q, const int64_t q_strides[4], const uint8_t* k_codes,
                         const int64_t k_strides[4], const uint8_t* v_codes,
                         const int64_t v_strides[4], const float* k_scale, const float* v_scale,
                         const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                         const int32_t* lists, const int32_t* list_counts, int n_lists,
                         int max_list, const int32_t* head_to_list, int B, int T, int Hq, int Hkv,
                         int D, int page_size, int P_pool, float scale, int n_splits,
                         float* o_partial, float* lse_partial, int32_t* dev_error, void* stream) {
  DecodeTarget t;
  return sparse_decode_fp8_impl(q, q_strides, k_codes, k_strides, v_codes, v_strides, k_scale,
                                v_scale, page_table, max_pages, seq_lens, lists, list_counts,
                                n_lists, max_list, head_to_list, B, T, Hq, Hkv, D, page_size,
                                P_pool, scale, n_splits, o_partial, lse_partial, dev_error, stream,
                                nullptr, &t);
}

size_t sa_sparse_attention_workspace_size(int B, int T, int Hq, int Dv, int n_splits) {
  if (B < 0 || T < 0 || Hq < 0 || Dv < 0 || n_splits < 0) return 0;
  const AttnWs w = attn_ws(B, T, Hq, Dv, n_splits);
  return w.o_bytes + w.lse_bytes;
}

int sa_sparse_attention(const uint16_t* q, const int64_t q_strides[4], const uint16_t* k_cache,
                        const int64_t k_strides[4], const uint16_t* v_cache,
                        const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                        const int32_t* seq_lens, const int32_t* lists, const int32_t* list_counts,
                        int n_lists, int max_list, const int32_t* head_to_list, int B, int T,
                        int Hq, int Hkv, int Dk, int Dv, int page_size, int P_pool, float scale,
                        int n_splits, float* o_out, uint16_t* o_out_bf16, float* lse_out,
                        void* workspace, size_t workspace_bytes, int32_t* dev_error,
                        void* stream) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || n_lists <= 0 || Dv <= 0 || n_splits <= 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (!workspace || !aligned16(workspace)) return SA_ERR_WORKSPACE;
  MergeSpec m{o_out, o_out_bf16, lse_out};
  if (int r = merge_outputs_ok(m)) return r;
  DecodeTarget t{static_cast<uint8_t*>(workspace), workspace_bytes};
  return sparse_decode_impl(q, q_strides, k_cache, k_strides, v_cache, v_strides, page_table,
                            max_pages, seq_lens, lists, list_counts, n_lists, max_list,
                            head_to_list, B, T, Hq, Hkv, Dk, Dv, page_size, P_pool, scale,
                            n_splits, nullptr, nullptr, dev_error, stream, &m, &t);
}

int sa_sparse_decode_at(const uint16_t* q, const int64_t q_strides[4], const uint16_t* k_cache,
                        const int64_t k_strides[4], const uint16_t* v_cache,
                        const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                        const int32_t* seq_lens, const int32_t* q_pos, const int32_t* lists,
                        const int32_t* list_counts, int n_lists, int max_list,
                        const int32_t* head_to_list, int B, int T, int Hq, int Hkv, int Dk, int Dv,
                        int page_size, int P_pool, float scale, int n_splits, float* o_partial,
                        float* lse_partial, int32_t* dev_error, void* stream) {
  if (!q_pos && B > 0) return SA_ERR_INVALID_ARG;
  DecodeTarget t{nullptr, 0, q_pos};
  return sparse_decode_impl(q, q_strides, k_cache, k_strides, v_cache, v_strides, page_table,
                            max_pages, seq_lens, lists, list_counts, n_lists, max_list,
                            head_to_list, B, T, Hq, Hkv, Dk, Dv, page_size, P_pool, scale,
                            n_splits, o_partial, lse_partial, dev_error, stream, nullptr, &t);
}

int sa_sparse_attention_at(const uint16_t* q, const int64_t q_strides[4],
                           const uint16_t* k_cache, const int64_t k_strides[4],
                           const uint16_t* v_cache, const int64_t v_strides[4],
                           const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                           const int32_t* q_pos, const int32_t* lists, const int32_t* list_counts,
                           int n_lists, int max_list, const int32_t* head_to_list, int B, int T,
                           int Hq, int Hkv, int Dk, int Dv, int page_size, int P_pool,
                           float scale, int n_splits, float* o_out, uint16_t* o_out_bf16,
                           float* lse_out, void* workspace, size_t workspace_bytes,
                           int32_t* dev_error, void* stream) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || n_lists <= 0 || Dv <= 0 || n_splits <= 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (!q_pos) return SA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return SA_ERR_WORKSPACE;
  MergeSpec m{o_out, o_out_bf16, lse_out};
  if (int r = merge_outputs_ok(m)) return r;
  DecodeTarget t{static_cast<uint8_t*>(workspace), workspace_bytes, q_pos};
  return sparse_decode_impl(q, q_strides, k_cache, k_strides, v_cache, v_strides, page_table,
                            max_pages, seq_lens, lists, list_counts, n_lists, max_list,
                            head_to_list, B, T, Hq, Hkv, Dk, Dv, page_size, P_pool, scale,
                            n_splits, nullptr, nullptr, dev_error, stream, &m, &t);
}

}  // extern "C"

namespace {
// The split count a step uses (n_splits <= 0: the default policy for this
// device) and its workspace: the selection's score bounds, then the split
// partials.
int step_plan(int B, int T, int Hq, int Hkv, int D, int page_size, int max_pages,
              int budget_tokens, int n_splits, int* splits_out, size_t* sel_bytes,
              size_t* total_bytes) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || page_size <= 0 ||
      max_pages < 0 || budget_tokens < 0)
    return SA_ERR_INVALID_ARG;
  const int budget_pages = budget_tokens / page_size;
  if (budget_pages <= 0) return SA_ERR_INVALID_ARG;
  if (D != 64 && D != 128 && D != 256) return SA_ERR_UNSUPPORTED;
  int s = n_splits;
  if (s <= 0 && cuda_status(decode_default_splits(D, B * Hkv, budget_pages, &s)) != SA_OK)
    return SA_ERR_CUDA;
  *splits_out = s;
  *sel_bytes = (select_workspace_bytes(B, Hkv, max_pages > 0 ? max_pages : 1) + 15) / 16 * 16;
  const AttnWs w = attn_ws(B, T, Hq, D, s);
  *total_bytes = *sel_bytes + w.o_bytes + w.lse_bytes;
  return SA_OK;
}

// FP8 E4M3 pages of a step: codes in place of the bf16 caches, and their
// per-(page, kv head) scales.
struct Fp8Pages {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const float* k_scale;
  const float* v_scale;
};

// sa_sparse_step over either page map (max_pages: the map's capacity); over
// FP8 pages when f8 is given (k_cache / v_cache unused then).
int step_impl(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
              const uint16_t* k_cache, const int64_t k_strides[4], const uint16_t* v_cache,
              const int64_t v_strides[4], const PageMap& pm, int max_pages,
              const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int D, int page_size,
              int P_pool, int sink_tokens, int local_tokens, int budget_tokens, float scale,
              int n_splits, int32_t* out_pages, int32_t* out_counts, float* o_out,
              uint16_t* o_out_bf16, float* lse_out, void* workspace, size_t workspace_bytes,
              int32_t* dev_error, void* stream, const Fp8Pages* f8 = nullptr) {
  int splits = 0;
  size_t sel_bytes = 0, total = 0;
  if (int r = step_plan(B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens, n_splits, &splits,
                        &sel_bytes, &total))
    return r;
  SelectArgs sa_args;
  if (int r = select_args(q, q_strides, summaries, pm, seq_lens, B, T, Hq, Hkv, D,
                          page_size, max_pages, P_pool, sink_tokens, local_tokens, budget_tokens,
                          out_pages, out_counts, dev_error, &sa_args))
    return r;
  if (B == 0) return SA_OK;
  MergeSpec m{o_out, o_out_bf16, lse_out};
  if (int r = merge_outputs_ok(m)) return r;
  if (!workspace || !aligned16(workspace) || workspace_bytes < total) return SA_ERR_WORKSPACE;
  // every argument of both halves is checked before the first launch
  if (f8) {
    if (int r = check_cache_u8(f8->k_codes, k_strides)) return r;
    if (int r = check_cache_u8(f8->v_codes, v_strides)) return r;
    if (!f8->k_scale || !f8->v_scale) return SA_ERR_INVALID_ARG;
    if (D != 128) return SA_ERR_UNSUPPORTED;
  } else {
    if (int r = check_cache(k_cache, k_strides)) return r;
    if (int r = check_cache(v_cache, v_strides)) return r;
  }
  if (P_pool <= 0 || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
  if (page_size % 16 != 0 || page_size > 128) return SA_ERR_UNSUPPORTED;
  const int budget_pages = sa_args.budget_pages;
  if ((budget_pages + splits - 1) / splits > decode_max_split_entries() || splits > 64 ||
      (int64_t)B * T * Hq * (D / 4) >= (int64_t(1) << 32))
    return SA_ERR_UNSUPPORTED;
  int32_t h2l[kMaxHeads];
  if (Hq > kMaxHeads) return SA_ERR_UNSUPPORTED;
  for (int h = 0; h < Hq; ++h) h2l[h] = h / (Hq / Hkv);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  sa_args.lohi = reinterpret_cast<float2*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int r = cuda_status(launch_select_gqa(sa_args, st))) return r;
  DecodeTarget t{ws + sel_bytes, total - sel_bytes};
  if (pm.blocks) t.dir = pm;
  if (f8)
    return sparse_decode_fp8_impl(q, q_strides, f8->k_codes, k_strides, f8->v_codes, v_strides,
                                  f8->k_scale, f8->v_scale, pm.table, max_pages, seq_lens,
                                  out_pages, out_counts, Hkv, budget_pages, h2l, B, T, Hq, Hkv, D,
                                  page_size, P_pool, scale, splits, nullptr, nullptr, dev_error,
                                  stream, &m, &t);
  return sparse_decode_impl(q, q_strides, k_cache, k_strides, v_cache, v_strides, pm.table,
                            max_pages, seq_lens, out_pages, out_counts, Hkv, budget_pages, h2l, B,
                            T, Hq, Hkv, D, D, page_size, P_pool, scale, splits, nullptr, nullptr,
                            dev_error, stream, &m, &t);
}

}  // namespace

extern "C" {

size_t sa_sparse_step_workspace_size(int B, int T, int Hq, int Hkv, int D, int page_size,
                                     int max_pages, int budget_tokens, int n_splits) {
  int s = 0;
  size_t sel = 0, total = 0;
  if (step_plan(B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens, n_splits, &s, &sel,
                &total) != SA_OK)
    return 0;
  return total;
}

int sa_sparse_step(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                   const uint16_t* k_cache, const int64_t k_strides[4], const uint16_t* v_cache,
                   const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                   const int32_t* seq_lens, int B, int T, int Hq, int Hkv, int D, int page_size,
                   int P_pool, int sink_tokens, int local_tokens, int budget_tokens, float scale,
                   int n_splits, int32_t* out_pages, int32_t* out_counts, float* o_out,
                   uint16_t* o_out_bf16, float* lse_out, void* workspace,
                   size_t workspace_bytes, int32_t* dev_error, void* stream) {
  return step_impl(q, q_strides, summaries, k_cache, k_strides, v_cache, v_strides,
                   flat_map(page_table, max_pages), max_pages, seq_lens, B, T, Hq, Hkv, D,
                   page_size, P_pool, sink_tokens, local_tokens, budget_tokens, scale, n_splits,
                   out_pages, out_counts, o_out, o_out_bf16, lse_out, workspace, workspace_bytes,
                   dev_error, stream);
}

int sa_sparse_step_fp8(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                       const uint8_t* k_codes, const int64_t k_strides[4],
                       const uint8_t* v_codes, const int64_t v_strides[4],
                       const float* k_scale, const float* v_scale, const int32_t* page_table,
                       int max_pages, const int32_t* seq_lens, int B, int T, int Hq, int Hkv,
                       int D, int page_size, int P_pool, int sink_tokens, int local_tokens,
                       int budget_tokens, float scale, int n_splits, int32_t* out_pages,
                       int32_t* out_counts, float* o_out, uint16_t* o_out_bf16, float* lse_out,
                       void* workspace, size_t workspace_bytes, int32_t* dev_error,
                       void* stream) {
  const Fp8Pages f8{k_codes, v_codes, k_scale, v_scale};
  return step_impl(q, q_strides, summaries, nullptr, k_strides, nullptr, v_strides,
                   flat_map(page_table, max_pages), max_pages, seq_lens, B, T, Hq, Hkv, D,
                   page_size, P_pool, sink_tokens, local_tokens, budget_tokens, scale, n_splits,
                   out_pages, out_counts, o_out, o_out_bf16, lse_out, workspace, workspace_bytes,
                   dev_error, stream, &f8);
}

int sa_sparse_attention_fp8(const uint16_t* q, const int64_t q_strides[4],
                            const uint8_t* k_codes, const int64_t k_strides[4],
                            const uint8_t* v_codes, const int64_t v_strides[4],
                            const float* k_scale, const float* v_scale,
                            const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                            const int32_t* lists, const int32_t* list_counts, int n_lists,
                            int max_list, const int32_t* head_to_list, int B, int T, int Hq,
                            int Hkv, int D, int page_size, int P_pool, float scale, int n_splits,
                            float* o_out, uint16_t* o_out_bf16, float* lse_out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_error, void* stream) {
  if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || n_lists <= 0 || D <= 0 || n_splits <= 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (!workspace || !aligned16(workspace)) return SA_ERR_WORKSPACE;
  MergeSpec m{o_out, o_out_bf16, lse_out};
  if (int r = merge_outputs_ok(m)) return r;
  DecodeTarget t{static_cast<uint8_t*>(workspace), workspace_bytes};
  return sparse_decode_fp8_impl(q, q_strides, k_codes, k_strides, v_codes, v_strides, k_scale,
                                v_scale, page_table, max_pages, seq_lens, lists, list_counts,
                                n_lists, max_list, head_to_list, B, T, Hq, Hkv, D, page_size,
                                P_pool, scale, n_splits, nullptr, nullptr, dev_error, stream, &m,
                                &t);
}

int sa_combine(const float* o_partial, const float* lse_partial, int n_splits, int64_t rows,
               int Dv, float* o_out, uint16_t* o_out_bf16, float* lse_out, void* stream) {
  if (n_splits <= 0 || rows < 0 || Dv <= 0 || (Dv % 4) != 0) return SA_ERR_INVALID_ARG;
  if (!o_partial || !lse_partial || (!o_out && !o_out_bf16 && !lse_out)) return SA_ERR_INVALID_ARG;
  if (!aligned16(o_partial) || (o_out && !aligned16(o_out)) ||
      (o_out_bf16 && (reinterpret_cast<uintptr_t>(o_out_bf16) & 7u)))
    return SA_ERR_INVALID_ARG;
  if (n_splits > 64 || rows * (Dv / 4) >= (int64_t(1) << 32)) return SA_ERR_UNSUPPORTED;
  if (rows == 0) return SA_OK;
  return cuda_status(launch_combine(o_partial, lse_partial, n_splits, rows, Dv, o_out, o_out_bf16,
                                    lse_out, static_cast<cudaStream_t>(stream)));
}

namespace {
int summaries_call(const uint16_t* k_cache, const int64_t k_strides[4],
                   const PageMap& pm, int max_pages, const int32_t* seq_lens, int B,
                   int Hkv, int Dk, int page_size, int P_pool, int n_new, uint16_t* summaries,
                   int32_t* dev_error, void* stream) {
  if (B < 0 || Hkv <= 0 || Dk <= 0 || page_size <= 0 || max_pages < 0 || P_pool < 0 || n_new < 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0 || max_pages == 0) return SA_OK;
  if (!k_cache || !k_strides || k_strides[3] != 1 || !pm.table || !seq_lens || !summaries)
    return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k_strides[i] <= 0) return SA_ERR_INVALID_ARG;
  if (max_pages > 65535 || B > 65535) return SA_ERR_UNSUPPORTED;
  return cuda_status(launch_summaries(k_cache, k_strides, pm, max_pages, seq_lens, B, Hkv,
                                      Dk, page_size, P_pool, n_new, summaries, dev_error,
                                      static_cast<cudaStream_t>(stream)));
}
}  // namespace

int sa_build_page_summaries(const uint16_t* k_cache, const int64_t k_strides[4],
                            const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                            int B, int Hkv, int Dk, int page_size, int P_pool,
                            uint16_t* summaries, int32_t* dev_error, void* stream) {
  return summaries_call(k_cache, k_strides, flat_map(page_table, max_pages), max_pages, seq_lens,
                        B, Hkv, Dk,
                        page_size, P_pool, 0, summaries, dev_error, stream);
}

int sa_update_page_summaries(const uint16_t* k_cache, const int64_t k_strides[4],
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int B, int Hkv, int Dk, int page_size, int P_pool, int n_new,
                             uint16_t* summaries, int32_t* dev_error, void* stream) {
  if (n_new <= 0) return SA_ERR_INVALID_ARG;
  return summaries_call(k_cache, k_strides, flat_map(page_table, max_pages), max_pages, seq_lens,
                        B, Hkv, Dk,
                        page_size, P_pool, n_new, summaries, dev_error, stream);
}

int sa_build_page_summaries_fp8(const uint8_t* k_codes, const int64_t k_strides[4],
                                const float* k_scale, const int32_t* page_table, int max_pages,
                                const int32_t* seq_lens, int B, int Hkv, int Dk, int page_size,
                                int P_pool, uint16_t* summaries, int32_t* dev_error,
                                void* stream) {
  if (B < 0 || Hkv <= 0 || Dk <= 0 || page_size <= 0 || max_pages < 0 || P_pool < 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0 || max_pages == 0) return SA_OK;
  if (!k_codes || !k_strides || k_strides[3] != 1 || !k_scale || !page_table || !seq_lens ||
      !summaries)
    return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k_strides[i] <= 0) return SA_ERR_INVALID_ARG;
  if (max_pages > 65535 || B > 65535 || page_size > 128) return SA_ERR_UNSUPPORTED;
  return cuda_status(launch_summaries_fp8(k_codes, k_strides, k_scale,
                                          flat_map(page_table, max_pages), max_pages,
                                          seq_lens, B, Hkv, Dk, page_size, P_pool, summaries,
                                          dev_error, static_cast<cudaStream_t>(stream)));
}

int sa_block_union(const float* scores, int Hq, int Hkv, int NQB, int NKB, int q_block_offset,
                   int top_k, int n_sink_blocks, int32_t* tables, int32_t* counts,
                   void* stream) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || NQB < 0 || NKB <= 0 || q_block_offset < 0 ||
      top_k < 0 || n_sink_blocks < 0 || q_block_offset + NQB > NKB)
    return SA_ERR_INVALID_ARG;
  if (!tables || !counts || (NQB > 0 && !scores)) return SA_ERR_INVALID_ARG;
  if (NKB > 16384 || NQB > 65535 || Hq > 65535) return SA_ERR_UNSUPPORTED;
  return cuda_status(launch_block_union(scores, Hq, Hkv, NQB, NKB, q_block_offset, top_k,
                                        n_sink_blocks, tables, counts,
                                        static_cast<cudaStream_t>(stream)));
}

size_t sa_select_ambient_heads_workspace_size(int B, int T, int Hq, int max_pages) {
  if (B <= 0 || T <= 0 || Hq <= 0 || max_pages < 0) return 0;
  return head_workspace_bytes(B, T, Hq, max_pages);
}

int sa_select_ambient_heads(const uint16_t* q, const int64_t q_strides[4],
                            const uint16_t* summaries, const int32_t* page_table, int max_pages,
                            const int32_t* seq_lens, const int32_t* lists,
                            const int32_t* list_counts, int list_cap, int B, int T, int Hq,
                            int Dk, int page_size, int P_pool, float scale, int h,
                            int32_t* out_heads, double* out_scores, void* workspace,
                            size_t workspace_bytes, int32_t* dev_error, void* stream) {
  if (B <= 0 || T <= 0 || Hq <= 0 || Dk <= 0 || page_size <= 0 || max_pages < 0 ||
      P_pool <= 0 || list_cap <= 0 || h < 0 || h > Hq || !std::isfinite(scale))
    return SA_ERR_INVALID_ARG;
  if (int r = check_q(q, q_strides)) return r;
  if (!summaries || !page_table || !seq_lens || !lists || !list_counts || (h > 0 && !out_heads))
    return SA_ERR_INVALID_ARG;
  if (Dk > head_max_dk() || Hq > 1024 || B > 65535 || T * Hq > 65535 * 32)
    return SA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 7u) ||
      workspace_bytes < head_workspace_bytes(B, T, Hq, max_pages))
    return SA_ERR_WORKSPACE;
  HeadArgs a;
  a.q = q;
  a.qs0 = q_strides[0];
  a.qs1 = q_strides[1];
  a.qs2 = q_strides[2];
  a.sig = summaries;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.lists = lists;
  a.counts = list_counts;
  a.cap = list_cap;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Dk = Dk;
  a.P = page_size;
  a.P_pool = P_pool;
  a.scale = scale;
  a.h_keep = h;
  a.n_chunks = 0;
  a.part = static_cast<double*>(workspace);
  a.heads_out = out_heads;
  a.scores_out = out_scores;
  a.err = dev_error;
  return cuda_status(launch_select_heads(a, static_cast<cudaStream_t>(stream)));
}

namespace {
// sa_append_kv over either page map (max_pages: the map's capacity).
int append_impl(const uint16_t* k_new, const int64_t kn_strides[4], const uint16_t* v_new,
                const int64_t vn_strides[4], const int32_t* n_new, int max_new,
                uint16_t* k_cache, const int64_t k_strides[4], uint16_t* v_cache,
                const int64_t v_strides[4], const PageMap& pm, int max_pages,
                const int32_t* seq_lens, int32_t* out_seq_lens, int B, int Hkv, int D,
                int page_size, int P_pool, uint16_t* summaries, int32_t* dev_error,
                void* stream) {
  if (B < 0 || Hkv <= 0 || D <= 0 || page_size <= 0 || max_pages < 0 || P_pool <= 0 ||
      max_new < 0 || D % 8 != 0)
    return SA_ERR_INVALID_ARG;
  if (B == 0) return SA_OK;
  if (int r = check_q(k_new, kn_strides)) return r;   // same rules as q: [B, T, H, D]
  if (int r = check_q(v_new, vn_strides)) return r;
  if (int r = check_cache(k_cache, k_strides)) return r;
  if (int r = check_cache(v_cache, v_strides)) return r;
  if (!n_new || !pm.table || !seq_lens || !summaries) return SA_ERR_INVALID_ARG;
  if (out_seq_lens == seq_lens) return SA_ERR_INVALID_ARG;   // read by every block
  if (B > 65535 || Hkv > 65535) return SA_ERR_UNSUPPORTED;
  AppendArgs a;
  a.k_new = k_new;
  a.kn0 = kn_strides[0];
  a.kn1 = kn_strides[1];
  a.kn2 = kn_strides[2];
  a.v_new = v_new;
  a.vn0 = vn_strides[0];
  a.vn1 = vn_strides[1];
  a.vn2 = vn_strides[2];
  a.n_new = n_new;
  a.max_new = max_new;
  a.k_cache = k_cache;
  a.ks0 = k_strides[0];
  a.ks1 = k_strides[1];
  a.ks2 = k_strides[2];
  a.v_cache = v_cache;
  a.vs0 = v_strides[0];
  a.vs1 = v_strides[1];
  a.vs2 = v_strides[2];
  a.pt = pm;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.out_seq_lens = out_seq_lens;
  a.B = B;
  a.Hkv = Hkv;
  a.D = D;
  a.P = page_size;
  a.P_pool = P_pool;
  a.sig = summaries;
  a.err = dev_error;
  return cuda_status(launch_append(a, static_cast<cudaStream_t>(stream)));
}

// The two-level map of a *_dir call, checked on the host; its capacity in
// logical pages goes to *max_pages.
int dir_map(const int32_t* page_dir, int n_dir, const int32_t* page_blocks, int n_blocks,
            int block_shift, PageMap* m, int* max_pages) {
  if (!page_dir || !page_blocks || n_dir < 0 || n_blocks < 0 || block_shift < 0 ||
      block_shift > 16)
    return SA_ERR_INVALID_ARG;
  const int64_t cap = (int64_t)n_dir << block_shift;
  if (cap > (int64_t(1) << 30)) return SA_ERR_UNSUPPORTED;
  m->table = page_dir;
  m->blocks = page_blocks;
  m->stride = n_dir;
  m->shift = block_shift;
  m->n_blocks = n_blocks;
  *max_pages = (int)cap;
  return SA_OK;
}
}  // namespace

int sa_append_kv(const uint16_t* k_new, const int64_t kn_strides[4], const uint16_t* v_new,
                 const int64_t vn_strides[4], const int32_t* n_new, int max_new,
                 uint16_t* k_cache, const int64_t k_strides[4], uint16_t* v_cache,
                 const int64_t v_strides[4], const int32_t* page_table, int max_pages,
                 const int32_t* seq_lens, int32_t* out_seq_lens, int B, int Hkv, int D,
                 int page_size, int P_pool, uint16_t* summaries, int32_t* dev_error,
                 void* stream) {
  return append_impl(k_new, kn_strides, v_new, vn_strides, n_new, max_new, k_cache, k_strides,
                     v_cache, v_strides, flat_map(page_table, max_pages), max_pages, seq_lens,
                     out_seq_lens, B, Hkv, D, page_size, P_pool, summaries, dev_error, stream);
}

int sa_append_kv_dir(const uint16_t* k_new, const int64_t kn_strides[4], const uint16_t* v_new,
                     const int64_t vn_strides[4], const int32_t* n_new, int max_new,
                     uint16_t* k_cache, const int64_t k_strides[4], uint16_t* v_cache,
                     const int64_t v_strides[4], const int32_t* page_dir, int n_dir,
                     const int32_t* page_blocks, int n_blocks, int block_shift,
                     const int32_t* seq_lens, int32_t* out_seq_lens, int B, int Hkv, int D,
                     int page_size, int P_pool, uint16_t* summaries, int32_t* dev_error,
                     void* stream) {
  PageMap m;
  int max_pages = 0;
  if (int r = dir_map(page_dir, n_dir, page_blocks, n_blocks, block_shift, &m, &max_pages))
    return r;
  return append_impl(k_new, kn_strides, v_new, vn_strides, n_new, max_new, k_cache, k_strides,
                     v_cache, v_strides, m, max_pages, seq_lens, out_seq_lens, B, Hkv, D,
                     page_size, P_pool, summaries, dev_error, stream);
}

int sa_build_page_summaries_dir(const uint16_t* k_cache, const int64_t k_strides[4],
                                const int32_t* page_dir, int n_dir, const int32_t* page_blocks,
                                int n_blocks, int block_shift, const int32_t* seq_lens, int B,
                                int Hkv, int Dk, int page_size, int P_pool, uint16_t* summaries,
                                int32_t* dev_error, void* stream) {
  PageMap m;
  int max_pages = 0;
  if (int r = dir_map(page_dir, n_dir, page_blocks, n_blocks, block_shift, &m, &max_pages))
    return r;
  return summaries_call(k_cache, k_strides, m, max_pages, seq_lens, B, Hkv, Dk, page_size, P_pool,
                        0, summaries, dev_error, stream);
}

int sa_sparse_step_dir(const uint16_t* q, const int64_t q_strides[4], const uint16_t* summaries,
                       const uint16_t* k_cache, const int64_t k_strides[4],
                       const uint16_t* v_cache, const int64_t v_strides[4],
                       const int32_t* page_dir, int n_dir, const int32_t* page_blocks,
                       int n_blocks, int block_shift, const int32_t* seq_lens, int B, int T,
                       int Hq, int Hkv, int D, int page_size, int P_pool, int sink_tokens,
                       int local_tokens, int budget_tokens, float scale, int n_splits,
                       int32_t* out_pages, int32_t* out_counts, float* o_out,
                       uint16_t* o_out_bf16, float* lse_out, void* workspace,
                       size_t workspace_bytes, int32_t* dev_error, void* stream) {
  PageMap m;
  int max_pages = 0;
  if (int r = dir_map(page_dir, n_dir, page_blocks, n_blocks, block_shift, &m, &max_pages))
    return r;
  return step_impl(q, q_strides, summaries, k_cache, k_strides, v_cache, v_strides, m, max_pages,
                   seq_lens, B, T, Hq, Hkv, D, page_size, P_pool, sink_tokens, local_tokens,
                   budget_tokens, scale, n_splits, out_pages, out_counts, o_out, o_out_bf16,
                   lse_out, workspace, workspace_bytes, dev_error, stream);
}

}  // extern "C"
