"""ctypes binding of ``libsa.so``: argument marshalling only.

Each function has the name and argument order of the C entry point it wraps
(include/sa.h); it takes torch tensors, checks dtypes and devices, passes
their data pointers, strides and the current CUDA stream, and raises
``SAError`` on a non-zero status.  Every step of the computation runs in the
library's kernels: there is no fallback when the library or the GPU is
missing; calls raise instead.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PAGED_SPARSE_KV_SA_LIB") or os.path.join(_HERE, "libsa.so")

_c_i64_4 = ctypes.c_int64 * 4
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float

_SIGNATURES = {
    "sa_status_string": (ctypes.c_char_p, [_I]),
    "sa_abi_version": (_I, []),
    "sa_select_pages": (_I, [_P, _c_i64_4, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                             _I, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_select_workspace_size": (ctypes.c_size_t, [_I, _I, _I]),
    "sa_select_pages_no_alloc": (_I, [_P, _c_i64_4, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                      _I, _I, _I, _P, _P, _P, _P]),
    "sa_select_pages_tiered": (_I, [_P, _c_i64_4, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                    _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_select_tiered_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "sa_sparse_decode": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _P, _P, _I,
                              _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _P]),
    "sa_sparse_decode_fp8": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _P, _P, _I, _P,
                                  _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P,
                                  _P, _P]),
    "sa_combine": (_I, [_P, _P, _I, _I64, _I, _P, _P, _P, _P]),
    "sa_sparse_attention_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "sa_sparse_attention": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _P, _P,
                                 _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P,
                                 _P, ctypes.c_size_t, _P, _P]),
    "sa_sparse_attention_fp8": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _P, _P, _I,
                                     _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                     _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_sparse_step_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "sa_sparse_step": (_I, [_P, _c_i64_4, _P, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _I, _I, _I,
                            _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P, _P,
                            ctypes.c_size_t, _P, _P]),
    "sa_sparse_step_fp8": (_I, [_P, _c_i64_4, _P, _P, _c_i64_4, _P, _c_i64_4, _P, _P, _P, _I, _P,
                                _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _P,
                                _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_build_page_summaries": (_I,[_P, _c_i64_4, _P, _I, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sa_update_page_summaries": (_I, [_P, _c_i64_4, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                      _P]),
    "sa_build_page_summaries_fp8": (_I, [_P, _c_i64_4, _P, _P, _I, _P, _I, _I, _I, _I, _I, _P, _P,
                                         _P]),
    "sa_block_union": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sa_select_ambient_heads_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "sa_select_ambient_heads": (_I, [_P, _c_i64_4, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                     _I, _F, _I, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_sparse_decode_at": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _P, _P, _P,
                                 _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P,
                                 _P]),
    "sa_sparse_attention_at": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _P, _P,
                                    _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P,
                                    _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_append_kv": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _c_i64_4, _P, _c_i64_4, _P, _I,
                          _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sa_build_page_summaries_dir": (_I, [_P, _c_i64_4, _P, _I, _P, _I, _I, _P, _I, _I, _I, _I,
                                         _I, _P, _P, _P]),
    "sa_sparse_step_dir": (_I, [_P, _c_i64_4, _P, _P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _I, _I,
                                _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P,
                                _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "sa_append_kv_dir": (_I, [_P, _c_i64_4, _P, _c_i64_4, _P, _I, _P, _c_i64_4, _P, _c_i64_4, _P,
                              _I, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
}

EXPORTED = tuple(_SIGNATURES)


class SAError(RuntimeError):
    pass


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m paged_sparse_kv_sa_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != 0:
        msg = load().sa_status_string(status).decode()
        raise SAError(f"{what} failed: {msg} ({status})")


# While bind() records, the wrappers' C calls are stored instead of issued, and
# every tensor whose pointer is passed is kept alive with the recording.
_REC = threading.local()


def _ptr(t):
    if t is None:
        return None
    keep = getattr(_REC, "keep", None)
    if keep is not None:
        keep.append(t)
    return ctypes.c_void_p(t.data_ptr())


def _call(fn, args, what):
    prog = getattr(_REC, "prog", None)
    if prog is not None:
        prog.append((fn, args, what))
        return
    _check(fn(*args), what)


def bind(fn):
    """Run ``fn()`` once with the library's C calls recorded instead of issued
    (arguments checked and marshalled as usual) and return a zero-argument
    callable that issues the recorded calls, in order, with the same pointers,
    sizes and streams -- for loops that run the same calls over the same
    buffers many times (a serving step over preallocated tensors).  The tensors
    the calls point to are kept alive by the callable; their contents may
    change between calls, their storage must not move."""
    _REC.prog, _REC.keep = [], []
    try:
        fn()
        prog, keep = _REC.prog, _REC.keep
    finally:
        _REC.prog = _REC.keep = None

    def run():
        for f, a, what in prog:
            st = f(*a)
            if st != 0:
                _check(st, what)
    run.keep = keep
    run.n_calls = len(prog)
    return run


def _strides4(t) -> "ctypes.Array":
    s = list(t.stride())
    if len(s) != 4:
        raise ValueError("expected a 4-D tensor")
    return _c_i64_4(*s)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be on the GPU")


def _bf16(t):
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bfloat16")
    return t


def _u8(t):
    if t.dtype != torch.uint8:
        raise TypeError("expected uint8 (FP8 E4M3 codes)")
    return t


def _f32c(t):
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise TypeError("expected a contiguous float32 tensor")
    return t


def _i32(t):
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise TypeError("expected a contiguous int32 tensor")
    return t


def page_budget(sink_tokens: int, local_tokens: int, budget_tokens: int, page_size: int):
    """(n_sink, n_local, budget_pages, k_top): the header's token -> page reading."""
    n_sink = -(-sink_tokens // page_size)
    n_local = -(-local_tokens // page_size)
    budget_pages = budget_tokens // page_size
    return n_sink, n_local, budget_pages, budget_pages - n_sink - n_local


def _select_shapes(q, summaries, page_table, seq_lens, out_pages, out_counts, bp):
    """The shapes the selection kernels assume (dense [P_pool,Hkv,Dk] summaries,
    [B,max_pages] table, [B] lengths, [B,Hkv,budget_pages] / [B,Hkv] outputs):
    a view with other strides would be read or written in the wrong layout."""
    B = q.shape[0]
    Hkv = summaries.shape[1]
    if summaries.dim() != 3 or summaries.shape[2] != q.shape[3]:
        raise ValueError("summaries must be [P_pool, Hkv, Dk] with the query's Dk")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages]")
    if tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be [B]")
    for t, shape, what in ((out_pages, (B, Hkv, max(bp, 1)), "out_pages"),
                           (out_counts, (B, Hkv), "out_counts")):
        if t is None:
            continue
        if t.dtype != torch.int32 or not t.is_contiguous() or tuple(t.shape) != shape:
            raise TypeError(f"{what} must be a contiguous int32 tensor of shape {shape}")


def sa_select_workspace_size(B: int, Hkv: int, max_pages: int) -> int:
    return int(load().sa_select_workspace_size(B, Hkv, max_pages))


def sa_select_pages(q, summaries, page_table, seq_lens, page_size: int, sink_tokens: int,
                    local_tokens: int, budget_tokens: int, out_pages=None, out_counts=None,
                    workspace=None, dev_error=None, P_pool: int = None, stream=None):
    """q [B,T,Hq,Dk] bf16; summaries [P_pool,Hkv,Dk] bf16; page_table [B,max_pages];
    seq_lens [B]; workspace: a uint8 device tensor of sa_select_workspace_size bytes
    (allocated here when None).  Returns (pages [B,Hkv,budget_pages], counts [B,Hkv])."""
    lib = load()
    _need_cuda(q, summaries, page_table, seq_lens)
    _bf16(q), _bf16(summaries), _i32(page_table), _i32(seq_lens)
    B, T, Hq, Dk = q.shape
    P_pool_, Hkv, _ = summaries.shape
    P_pool = P_pool_ if P_pool is None else P_pool
    bp = budget_tokens // page_size
    _select_shapes(q, summaries, page_table, seq_lens, out_pages, out_counts, bp)
    if out_pages is None:
        out_pages = torch.empty((B, Hkv, max(bp, 1)), dtype=torch.int32, device=q.device)
    if out_counts is None:
        out_counts = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    max_pages = page_table.shape[1]
    if workspace is None:
        workspace = torch.empty(max(sa_select_workspace_size(B, Hkv, max_pages), 16),
                                dtype=torch.uint8, device=q.device)
    _call(lib.sa_select_pages, (_ptr(q), _strides4(q), _ptr(summaries.contiguous()), _ptr(page_table),
                             _ptr(seq_lens), B, T, Hq, Hkv, Dk, page_size, max_pages,
                             P_pool, sink_tokens, local_tokens, budget_tokens, _ptr(out_pages),
                             _ptr(out_counts), _ptr(workspace), workspace.numel(),
                             _ptr(dev_error), _stream(stream)), "sa_select_pages")
    return out_pages, out_counts


def sa_select_pages_no_alloc(q, summaries, page_table, seq_lens, page_size: int,
                             sink_tokens: int, local_tokens: int, budget_tokens: int, out_pages,
                             out_counts, dev_error=None, P_pool: int = None, stream=None):
    """sa_select_pages without a workspace: the score bounds go to the library's
    static device array (shared by all calls; calls must not overlap on the GPU).
    The outputs must be preallocated and every tensor laid out as the C call
    assumes (contiguous summaries and outputs): nothing is copied or allocated
    here, so a strided view is refused rather than made contiguous."""
    lib = load()
    _need_cuda(q, summaries, page_table, seq_lens, out_pages, out_counts)
    _bf16(q), _i32(page_table), _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    B, T, Hq, Dk = q.shape
    P_pool_, Hkv, _ = summaries.shape
    P_pool = P_pool_ if P_pool is None else P_pool
    _select_shapes(q, summaries, page_table, seq_lens, out_pages, out_counts,
                   budget_tokens // page_size)
    _call(lib.sa_select_pages_no_alloc, (_ptr(q), _strides4(q), _ptr(summaries), _ptr(page_table),
                                      _ptr(seq_lens), B, T, Hq, Hkv, Dk, page_size,
                                      page_table.shape[1], P_pool, sink_tokens, local_tokens,
                                      budget_tokens, _ptr(out_pages), _ptr(out_counts),
                                      _ptr(dev_error), _stream(stream)), "sa_select_pages_no_alloc")
    return out_pages, out_counts


def sa_select_pages_tiered(q, summaries, page_table, seq_lens, page_size: int, alpha: int,
                           beta: int, lists=None, list_counts=None, workspace=None,
                           dev_error=None, stream=None):
    """q [B,T,Hq,Dk]; summaries [P_pool,1,Dk].  Returns (lists [B,2,alpha+beta],
    counts [B,2]): list 0 = critical pages, list 1 = critical + ambient pages."""
    lib = load()
    _need_cuda(q, summaries, page_table, seq_lens)
    _bf16(q), _bf16(summaries), _i32(page_table), _i32(seq_lens)
    B, T, Hq, Dk = q.shape
    P_pool = summaries.shape[0]
    max_pages = page_table.shape[1]
    if lists is None:
        lists = torch.empty((B, 2, alpha + beta), dtype=torch.int32, device=q.device)
    if list_counts is None:
        list_counts = torch.empty((B, 2), dtype=torch.int32, device=q.device)
    if workspace is None:
        n = int(lib.sa_select_tiered_workspace_size(B, T, Hq, max_pages))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _call(lib.sa_select_pages_tiered, (_ptr(q), _strides4(q), _ptr(summaries.contiguous()),
                                    _ptr(page_table), _ptr(seq_lens), B, T, Hq, Dk, page_size,
                                    max_pages, P_pool, alpha, beta, _ptr(lists),
                                    _ptr(list_counts), _ptr(workspace), workspace.numel(),
                                    _ptr(dev_error), _stream(stream)), "sa_select_pages_tiered")
    return lists, list_counts


def sa_sparse_decode(q, k_cache, v_cache, page_table, seq_lens, lists, list_counts, head_to_list,
                     scale: float, n_splits: int = 1, o_partial=None, lse_partial=None,
                     dev_error=None, stream=None):
    """q [B,T,Hq,Dk]; k_cache [P_pool,Hkv,P,Dk]; v_cache [P_pool,Hkv,P,Dv] (any strides with a
    unit feature stride); lists [B,n_lists,max_list]; list_counts [B,n_lists];
    head_to_list: a host sequence of Hq list ids.  Returns (o_partial, lse_partial)."""
    lib = load()
    _need_cuda(q, k_cache, v_cache, page_table, seq_lens, lists, list_counts)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(page_table), _i32(seq_lens), _i32(lists)
    _i32(list_counts)
    B, T, Hq, Dk = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    Dv = v_cache.shape[-1]
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    if o_partial is None:
        o_partial = torch.empty((n_splits, B, T, Hq, Dv), dtype=torch.float32, device=q.device)
    if lse_partial is None:
        lse_partial = torch.empty((n_splits, B, T, Hq), dtype=torch.float32, device=q.device)
    _call(lib.sa_sparse_decode, (_ptr(q), _strides4(q), _ptr(k_cache), _strides4(k_cache),
                              _ptr(v_cache), _strides4(v_cache), _ptr(page_table),
                              page_table.shape[1], _ptr(seq_lens), _ptr(lists), _ptr(list_counts),
                              n_lists, max_list, ctypes.cast(h2l, ctypes.c_void_p), B, T, Hq, Hkv,
                              Dk, Dv, P, P_pool, float(scale), n_splits, _ptr(o_partial),
                              _ptr(lse_partial), _ptr(dev_error), _stream(stream)), "sa_sparse_decode")
    return o_partial, lse_partial


def sa_sparse_decode_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens, lists,
                         list_counts, head_to_list, scale: float, n_splits: int = 1,
                         o_partial=None, lse_partial=None, dev_error=None, stream=None):
    """sa_sparse_decode over FP8 E4M3 pages: k_codes, v_codes [P_pool,Hkv,P,D] uint8 (unit
    feature stride), k_scale, v_scale [P_pool,Hkv] float32.  Returns (o_partial, lse_partial)."""
    lib = load()
    _need_cuda(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens, lists, list_counts)
    _bf16(q), _u8(k_codes), _u8(v_codes), _f32c(k_scale), _f32c(v_scale)
    _i32(page_table), _i32(seq_lens), _i32(lists), _i32(list_counts)
    B, T, Hq, D = q.shape
    P_pool, Hkv, P, _ = k_codes.shape
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    if o_partial is None:
        o_partial = torch.empty((n_splits, B, T, Hq, D), dtype=torch.float32, device=q.device)
    if lse_partial is None:
        lse_partial = torch.empty((n_splits, B, T, Hq), dtype=torch.float32, device=q.device)
    _call(lib.sa_sparse_decode_fp8, (_ptr(q), _strides4(q), _ptr(k_codes), _strides4(k_codes),
                                  _ptr(v_codes), _strides4(v_codes), _ptr(k_scale), _ptr(v_scale),
                                  _ptr(page_table), page_table.shape[1], _ptr(seq_lens),
                                  _ptr(lists), _ptr(list_counts), n_lists, max_list,
                                  ctypes.cast(h2l, ctypes.c_void_p), B, T, Hq, Hkv, D, P, P_pool,
                                  float(scale), n_splits, _ptr(o_partial), _ptr(lse_partial),
                                  _ptr(dev_error), _stream(stream)), "sa_sparse_decode_fp8")
    return o_partial, lse_partial


def attention_workspace(B, T, Hq, Dv, n_splits, device):
    """A workspace for sa_sparse_attention(_fp8): the split partials."""
    n = int(load().sa_sparse_attention_workspace_size(B, T, Hq, Dv, n_splits))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def _attn_outputs(B, T, Hq, Dv, device, o_out, o_out_bf16, lse_out, want_f32, want_bf16):
    if o_out is None and want_f32:
        o_out = torch.empty((B, T, Hq, Dv), dtype=torch.float32, device=device)
    if o_out_bf16 is None and want_bf16:
        o_out_bf16 = torch.empty((B, T, Hq, Dv), dtype=torch.bfloat16, device=device)
    if lse_out is None:
        lse_out = torch.empty((B, T, Hq), dtype=torch.float32, device=device)
    return o_out, o_out_bf16, lse_out


def sa_sparse_attention(q, k_cache, v_cache, page_table, seq_lens, lists, list_counts,
                        head_to_list, scale: float, n_splits: int = 1, o_out=None,
                        o_out_bf16=None, lse_out=None, want_f32: bool = True,
                        want_bf16: bool = False, workspace=None, dev_error=None, stream=None):
    """sa_sparse_decode + merge in one call.  Inputs as sa_sparse_decode; returns
    (O [B,T,Hq,Dv] f32 or None, O bf16 or None, lse [B,T,Hq]).  `workspace`: from
    attention_workspace (reusable); a fresh one is made when omitted."""
    lib = load()
    _need_cuda(q, k_cache, v_cache, page_table, seq_lens, lists, list_counts)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(page_table), _i32(seq_lens), _i32(lists)
    _i32(list_counts)
    B, T, Hq, Dk = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    Dv = v_cache.shape[-1]
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, Dv, q.device, o_out, o_out_bf16,
                                               lse_out, want_f32, want_bf16)
    if workspace is None:
        workspace = attention_workspace(B, T, Hq, Dv, n_splits, q.device)
    _call(lib.sa_sparse_attention, (_ptr(q), _strides4(q), _ptr(k_cache), _strides4(k_cache),
                                 _ptr(v_cache), _strides4(v_cache), _ptr(page_table),
                                 page_table.shape[1], _ptr(seq_lens), _ptr(lists),
                                 _ptr(list_counts), n_lists, max_list,
                                 ctypes.cast(h2l, ctypes.c_void_p), B, T, Hq, Hkv, Dk, Dv, P,
                                 P_pool, float(scale), n_splits, _ptr(o_out), _ptr(o_out_bf16),
                                 _ptr(lse_out), _ptr(workspace), workspace.numel(),
                                 _ptr(dev_error), _stream(stream)), "sa_sparse_attention")
    return o_out, o_out_bf16, lse_out


def sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens,
                                  n_splits=0) -> int:
    return int(load().sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, page_size, max_pages,
                                                    budget_tokens, n_splits))


def sa_sparse_step(q, summaries, k_cache, v_cache, page_table, seq_lens, page_size: int,
                   sink_tokens: int, local_tokens: int, budget_tokens: int, scale: float,
                   n_splits: int = 0, out_pages=None, out_counts=None, o_out=None,
                   o_out_bf16=None, lse_out=None, want_f32: bool = True, want_bf16: bool = False,
                   workspace=None, dev_error=None, stream=None):
    """Selection + attention + merge in one C call (sa_sparse_step).  q [B,T,Hq,D];
    summaries [P_pool,Hkv,D]; k_cache, v_cache [P_pool,Hkv,P,D]; n_splits 0 = the
    library's default.  Returns (pages, counts, O f32 or None, O bf16 or None, lse)."""
    lib = load()
    _need_cuda(q, summaries, k_cache, v_cache, page_table, seq_lens)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(page_table), _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    B, T, Hq, D = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    if P != page_size:
        raise ValueError("page_size differs from the cache's page dimension")
    bp = budget_tokens // page_size
    _select_shapes(q, summaries, page_table, seq_lens, out_pages, out_counts, bp)
    if out_pages is None:
        out_pages = torch.empty((B, Hkv, max(bp, 1)), dtype=torch.int32, device=q.device)
    if out_counts is None:
        out_counts = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, D, q.device, o_out, o_out_bf16,
                                               lse_out, want_f32, want_bf16)
    max_pages = page_table.shape[1]
    if workspace is None:
        n = sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens,
                                          n_splits)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _call(lib.sa_sparse_step,
          (_ptr(q), _strides4(q), _ptr(summaries), _ptr(k_cache), _strides4(k_cache),
           _ptr(v_cache), _strides4(v_cache), _ptr(page_table), max_pages, _ptr(seq_lens), B, T,
           Hq, Hkv, D, page_size, P_pool, sink_tokens, local_tokens, budget_tokens,
           float(scale), int(n_splits), _ptr(out_pages), _ptr(out_counts), _ptr(o_out),
           _ptr(o_out_bf16), _ptr(lse_out), _ptr(workspace), workspace.numel(),
           _ptr(dev_error), _stream(stream)), "sa_sparse_step")
    return out_pages, out_counts, o_out, o_out_bf16, lse_out


def sa_sparse_step_fp8(q, summaries, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens,
                       page_size: int, sink_tokens: int, local_tokens: int, budget_tokens: int,
                       scale: float, n_splits: int = 0, out_pages=None, out_counts=None,
                       o_out=None, o_out_bf16=None, lse_out=None, want_f32: bool = True,
                       want_bf16: bool = False, workspace=None, dev_error=None, stream=None):
    """sa_sparse_step over FP8 E4M3 pages (codes [P_pool,Hkv,P,D] uint8, scales
    [P_pool,Hkv] float32, D == 128).  Returns (pages, counts, O f32 or None, O bf16
    or None, lse)."""
    lib = load()
    _need_cuda(q, summaries, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens)
    _bf16(q), _u8(k_codes), _u8(v_codes), _f32c(k_scale), _f32c(v_scale), _i32(page_table)
    _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    B, T, Hq, D = q.shape
    P_pool, Hkv, P, _ = k_codes.shape
    if P != page_size:
        raise ValueError("page_size differs from the cache's page dimension")
    bp = budget_tokens // page_size
    _select_shapes(q, summaries, page_table, seq_lens, out_pages, out_counts, bp)
    if out_pages is None:
        out_pages = torch.empty((B, Hkv, max(bp, 1)), dtype=torch.int32, device=q.device)
    if out_counts is None:
        out_counts = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, D, q.device, o_out, o_out_bf16,
                                               lse_out, want_f32, want_bf16)
    max_pages = page_table.shape[1]
    if workspace is None:
        n = sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, page_size, max_pages, budget_tokens,
                                          n_splits)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _call(lib.sa_sparse_step_fp8,
          (_ptr(q), _strides4(q), _ptr(summaries), _ptr(k_codes), _strides4(k_codes),
           _ptr(v_codes), _strides4(v_codes), _ptr(k_scale), _ptr(v_scale), _ptr(page_table),
           max_pages, _ptr(seq_lens), B, T, Hq, Hkv, D, page_size, P_pool, sink_tokens,
           local_tokens, budget_tokens, float(scale), int(n_splits), _ptr(out_pages),
           _ptr(out_counts), _ptr(o_out), _ptr(o_out_bf16), _ptr(lse_out), _ptr(workspace),
           workspace.numel(), _ptr(dev_error), _stream(stream)), "sa_sparse_step_fp8")
    return out_pages, out_counts, o_out, o_out_bf16, lse_out


def sa_sparse_attention_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens, lists,
                            list_counts, head_to_list, scale: float, n_splits: int = 1,
                            o_out=None, o_out_bf16=None, lse_out=None, want_f32: bool = True,
                            want_bf16: bool = False, workspace=None, dev_error=None, stream=None):
    """sa_sparse_decode_fp8 + merge in one call; inputs as sa_sparse_decode_fp8, outputs and
    workspace as sa_sparse_attention."""
    lib = load()
    _need_cuda(q, k_codes, v_codes, k_scale, v_scale, page_table, seq_lens, lists, list_counts)
    _bf16(q), _u8(k_codes), _u8(v_codes), _f32c(k_scale), _f32c(v_scale)
    _i32(page_table), _i32(seq_lens), _i32(lists), _i32(list_counts)
    B, T, Hq, D = q.shape
    P_pool, Hkv, P, _ = k_codes.shape
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, D, q.device, o_out, o_out_bf16, lse_out,
                                               want_f32, want_bf16)
    if workspace is None:
        workspace = attention_workspace(B, T, Hq, D, n_splits, q.device)
    _call(lib.sa_sparse_attention_fp8, (_ptr(q), _strides4(q), _ptr(k_codes), _strides4(k_codes),
                                     _ptr(v_codes), _strides4(v_codes), _ptr(k_scale),
                                     _ptr(v_scale), _ptr(page_table), page_table.shape[1],
                                     _ptr(seq_lens), _ptr(lists), _ptr(list_counts), n_lists,
                                     max_list, ctypes.cast(h2l, ctypes.c_void_p), B, T, Hq, Hkv, D,
                                     P, P_pool, float(scale), n_splits, _ptr(o_out),
                                     _ptr(o_out_bf16), _ptr(lse_out), _ptr(workspace),
                                     workspace.numel(), _ptr(dev_error), _stream(stream)), "sa_sparse_attention_fp8")
    return o_out, o_out_bf16, lse_out


def sa_build_page_summaries_fp8(k_codes, k_scale, page_table, seq_lens, summaries=None,
                                dev_error=None, stream=None):
    """k_codes [P_pool,Hkv,P,Dk] uint8 E4M3, k_scale [P_pool,Hkv] float32 -> summaries
    [P_pool,Hkv,Dk] bf16 (rows of referenced pages written)."""
    lib = load()
    _need_cuda(k_codes, k_scale, page_table, seq_lens)
    _u8(k_codes), _f32c(k_scale), _i32(page_table), _i32(seq_lens)
    P_pool, Hkv, P, Dk = k_codes.shape
    if summaries is None:
        summaries = torch.zeros((P_pool, Hkv, Dk), dtype=torch.bfloat16, device=k_codes.device)
    _call(lib.sa_build_page_summaries_fp8, (_ptr(k_codes), _strides4(k_codes), _ptr(k_scale),
                                         _ptr(page_table), page_table.shape[1], _ptr(seq_lens),
                                         seq_lens.shape[0], Hkv, Dk, P, P_pool, _ptr(summaries),
                                         _ptr(dev_error), _stream(stream)), "sa_build_page_summaries_fp8")
    return summaries


def sa_combine(o_partial, lse_partial, o_out=None, o_out_bf16=None, lse_out=None,
               want_f32: bool = True, stream=None):
    """o_partial [S,...,Dv] f32, lse_partial [S,...] f32 -> (O [...,Dv] f32, O bf16 or None,
    lse [...])."""
    lib = load()
    _need_cuda(o_partial, lse_partial)
    S = o_partial.shape[0]
    Dv = o_partial.shape[-1]
    lead = tuple(o_partial.shape[1:-1])
    rows = lse_partial[0].numel()
    if o_out is None and want_f32:
        o_out = torch.empty(lead + (Dv,), dtype=torch.float32, device=o_partial.device)
    if lse_out is None:
        lse_out = torch.empty(lead, dtype=torch.float32, device=o_partial.device)
    _call(lib.sa_combine, (_ptr(o_partial), _ptr(lse_partial), S, rows, Dv, _ptr(o_out),
                        _ptr(o_out_bf16), _ptr(lse_out), _stream(stream)), "sa_combine")
    return o_out, o_out_bf16, lse_out


def sa_build_page_summaries(k_cache, page_table, seq_lens, summaries=None, dev_error=None,
                            stream=None):
    """k_cache [P_pool,Hkv,P,Dk] bf16 -> summaries [P_pool,Hkv,Dk] bf16 (rows of referenced
    pages written)."""
    lib = load()
    _need_cuda(k_cache, page_table, seq_lens)
    _bf16(k_cache), _i32(page_table), _i32(seq_lens)
    P_pool, Hkv, P, Dk = k_cache.shape
    if summaries is None:
        summaries = torch.zeros((P_pool, Hkv, Dk), dtype=torch.bfloat16, device=k_cache.device)
    _call(lib.sa_build_page_summaries, (_ptr(k_cache), _strides4(k_cache), _ptr(page_table),
                                     page_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], Hkv,
                                     Dk, P, P_pool, _ptr(summaries), _ptr(dev_error),
                                     _stream(stream)), "sa_build_page_summaries")
    return summaries


def sa_update_page_summaries(k_cache, page_table, seq_lens, summaries, n_new: int,
                             dev_error=None, stream=None):
    """Rewrite, in place, the summaries of the pages holding each sequence's last
    n_new tokens (after an append); returns summaries."""
    lib = load()
    _need_cuda(k_cache, page_table, seq_lens, summaries)
    _bf16(k_cache), _i32(page_table), _i32(seq_lens), _bf16(summaries)
    P_pool, Hkv, P, Dk = k_cache.shape
    _call(lib.sa_update_page_summaries, (_ptr(k_cache), _strides4(k_cache), _ptr(page_table),
                                      page_table.shape[1], _ptr(seq_lens), seq_lens.shape[0],
                                      Hkv, Dk, P, P_pool, int(n_new), _ptr(summaries),
                                      _ptr(dev_error), _stream(stream)), "sa_update_page_summaries")
    return summaries


def sa_block_union(scores, Hkv: int, q_block_offset: int, top_k: int, n_sink_blocks: int = 1,
                   tables=None, counts=None, stream=None):
    """scores [Hq,NQB,NKB] f32 -> (tables [Hkv,NKB] int32, counts [Hkv])."""
    lib = load()
    _need_cuda(scores)
    if scores.dtype != torch.float32 or not scores.is_contiguous():
        raise TypeError("scores must be contiguous float32")
    Hq, NQB, NKB = scores.shape
    if tables is None:
        tables = torch.empty((Hkv, NKB), dtype=torch.int32, device=scores.device)
    if counts is None:
        counts = torch.empty((Hkv,), dtype=torch.int32, device=scores.device)
    _call(lib.sa_block_union, (_ptr(scores), Hq, Hkv, NQB, NKB, q_block_offset, top_k,
                            n_sink_blocks, _ptr(tables), _ptr(counts), _stream(stream)), "sa_block_union")
    return tables, counts


def sa_append_kv(k_new, v_new, n_new, k_cache, v_cache, page_table, seq_lens, summaries,
                 out_seq_lens=None, dev_error=None, stream=None):
    """Write sequence b's n_new[b] new tokens (k_new, v_new [B,max_new,Hkv,D] bf16) at
    positions seq_lens[b] + i of the paged caches [P_pool,Hkv,P,D] and rewrite the
    summaries of the pages they land in (in place).  seq_lens: lengths before the
    append; out_seq_lens (optional, not seq_lens) receives the new lengths."""
    lib = load()
    _need_cuda(k_new, v_new, n_new, k_cache, v_cache, page_table, seq_lens, summaries)
    _bf16(k_new), _bf16(v_new), _bf16(k_cache), _bf16(v_cache), _i32(n_new), _i32(page_table)
    _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    if out_seq_lens is not None:
        _i32(out_seq_lens)
    B, max_new, Hkv, D = k_new.shape
    P_pool, _, P, _ = k_cache.shape
    _call(lib.sa_append_kv, (_ptr(k_new), _strides4(k_new), _ptr(v_new), _strides4(v_new),
                             _ptr(n_new), max_new, _ptr(k_cache), _strides4(k_cache),
                             _ptr(v_cache), _strides4(v_cache), _ptr(page_table),
                             page_table.shape[1], _ptr(seq_lens), _ptr(out_seq_lens), B, Hkv, D,
                             P, P_pool, _ptr(summaries), _ptr(dev_error), _stream(stream)),
          "sa_append_kv")
    return out_seq_lens


def sa_select_ambient_heads(q, summaries, page_table, seq_lens, lists, list_counts, page_size: int,
                            scale: float, h: int, out_heads=None, out_scores=None, workspace=None,
                            dev_error=None, stream=None):
    """The h heads of largest estimated ambient attention-mass coverage (ascending,
    [h] int32) and every head's score ([Hq] float64).  lists [B,2,cap] / list_counts
    [B,2]: sa_select_pages_tiered's output."""
    lib = load()
    _need_cuda(q, summaries, page_table, seq_lens, lists, list_counts)
    _bf16(q), _i32(page_table), _i32(seq_lens), _i32(lists), _i32(list_counts)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    B, T, Hq, Dk = q.shape
    P_pool = summaries.shape[0]
    max_pages = page_table.shape[1]
    if out_heads is None:
        out_heads = torch.empty((max(h, 1),), dtype=torch.int32, device=q.device)
    if out_scores is None:
        out_scores = torch.empty((Hq,), dtype=torch.float64, device=q.device)
    if workspace is None:
        n = int(lib.sa_select_ambient_heads_workspace_size(B, T, Hq, max_pages))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _call(lib.sa_select_ambient_heads,
          (_ptr(q), _strides4(q), _ptr(summaries), _ptr(page_table), max_pages, _ptr(seq_lens),
           _ptr(lists), _ptr(list_counts), lists.shape[2], B, T, Hq, Dk, page_size, P_pool,
           float(scale), int(h), _ptr(out_heads), _ptr(out_scores), _ptr(workspace),
           workspace.numel(), _ptr(dev_error), _stream(stream)), "sa_select_ambient_heads")
    return out_heads[:h], out_scores


def sa_sparse_decode_at(q, k_cache, v_cache, page_table, seq_lens, q_pos, lists, list_counts,
                        head_to_list, scale: float, n_splits: int = 1, o_partial=None,
                        lse_partial=None, dev_error=None, stream=None):
    """sa_sparse_decode with explicit query positions: token t of sequence b at
    q_pos[b] + t (q_pos [B] int32 on the GPU).  Returns (o_partial, lse_partial)."""
    lib = load()
    _need_cuda(q, k_cache, v_cache, page_table, seq_lens, q_pos, lists, list_counts)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(page_table), _i32(seq_lens), _i32(q_pos)
    _i32(lists), _i32(list_counts)
    B, T, Hq, Dk = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    Dv = v_cache.shape[-1]
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    if o_partial is None:
        o_partial = torch.empty((n_splits, B, T, Hq, Dv), dtype=torch.float32, device=q.device)
    if lse_partial is None:
        lse_partial = torch.empty((n_splits, B, T, Hq), dtype=torch.float32, device=q.device)
    _call(lib.sa_sparse_decode_at,
          (_ptr(q), _strides4(q), _ptr(k_cache), _strides4(k_cache), _ptr(v_cache),
           _strides4(v_cache), _ptr(page_table), page_table.shape[1], _ptr(seq_lens), _ptr(q_pos),
           _ptr(lists), _ptr(list_counts), n_lists, max_list, ctypes.cast(h2l, ctypes.c_void_p), B,
           T, Hq, Hkv, Dk, Dv, P, P_pool, float(scale), n_splits, _ptr(o_partial),
           _ptr(lse_partial), _ptr(dev_error), _stream(stream)), "sa_sparse_decode_at")
    return o_partial, lse_partial


def sa_sparse_attention_at(q, k_cache, v_cache, page_table, seq_lens, q_pos, lists, list_counts,
                           head_to_list, scale: float, n_splits: int = 1, o_out=None,
                           o_out_bf16=None, lse_out=None, want_f32: bool = True,
                           want_bf16: bool = False, workspace=None, dev_error=None, stream=None):
    """sa_sparse_attention with explicit query positions (q_pos [B] int32 on the GPU)."""
    lib = load()
    _need_cuda(q, k_cache, v_cache, page_table, seq_lens, q_pos, lists, list_counts)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(page_table), _i32(seq_lens), _i32(q_pos)
    _i32(lists), _i32(list_counts)
    B, T, Hq, Dk = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    Dv = v_cache.shape[-1]
    _, n_lists, max_list = lists.shape
    h2l = (ctypes.c_int32 * Hq)(*[int(x) for x in head_to_list])
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, Dv, q.device, o_out, o_out_bf16,
                                               lse_out, want_f32, want_bf16)
    if workspace is None:
        workspace = attention_workspace(B, T, Hq, Dv, n_splits, q.device)
    _call(lib.sa_sparse_attention_at,
          (_ptr(q), _strides4(q), _ptr(k_cache), _strides4(k_cache), _ptr(v_cache),
           _strides4(v_cache), _ptr(page_table), page_table.shape[1], _ptr(seq_lens), _ptr(q_pos),
           _ptr(lists), _ptr(list_counts), n_lists, max_list, ctypes.cast(h2l, ctypes.c_void_p), B,
           T, Hq, Hkv, Dk, Dv, P, P_pool, float(scale), n_splits, _ptr(o_out), _ptr(o_out_bf16),
           _ptr(lse_out), _ptr(workspace), workspace.numel(), _ptr(dev_error), _stream(stream)),
          "sa_sparse_attention_at")
    return o_out, o_out_bf16, lse_out


# ---------------------------------------------------------------------------
# two-level page map: a directory [B, n_dir] of block ids over blocks
# [n_blocks, 2^block_shift] of physical page ids, in place of a flat table
# ---------------------------------------------------------------------------
def _dir_args(page_dir, page_blocks, block_shift: int):
    _i32(page_dir), _i32(page_blocks)
    if page_dir.dim() != 2 or page_blocks.dim() != 2:
        raise ValueError("page_dir must be [B, n_dir] and page_blocks [n_blocks, 2^block_shift]")
    if page_blocks.shape[1] != (1 << block_shift):
        raise ValueError("page_blocks rows must hold 2^block_shift entries")
    return (_ptr(page_dir), page_dir.shape[1], _ptr(page_blocks), page_blocks.shape[0],
            int(block_shift))


def dir_capacity(page_dir, block_shift: int) -> int:
    """Logical pages per sequence a two-level map holds (its flat max_pages)."""
    return page_dir.shape[1] << block_shift


def sa_build_page_summaries_dir(k_cache, page_dir, page_blocks, block_shift: int, seq_lens,
                                summaries=None, dev_error=None, stream=None):
    """sa_build_page_summaries over a two-level page map."""
    lib = load()
    _need_cuda(k_cache, page_dir, page_blocks, seq_lens)
    _bf16(k_cache), _i32(seq_lens)
    P_pool, Hkv, P, Dk = k_cache.shape
    if summaries is None:
        summaries = torch.zeros((P_pool, Hkv, Dk), dtype=torch.bfloat16, device=k_cache.device)
    _call(lib.sa_build_page_summaries_dir,
          (_ptr(k_cache), _strides4(k_cache), *_dir_args(page_dir, page_blocks, block_shift),
           _ptr(seq_lens), seq_lens.shape[0], Hkv, Dk, P, P_pool, _ptr(summaries),
           _ptr(dev_error), _stream(stream)), "sa_build_page_summaries_dir")
    return summaries


def sa_sparse_step_dir(q, summaries, k_cache, v_cache, page_dir, page_blocks, block_shift: int,
                       seq_lens, page_size: int, sink_tokens: int, local_tokens: int,
                       budget_tokens: int, scale: float, n_splits: int = 0, out_pages=None,
                       out_counts=None, o_out=None, o_out_bf16=None, lse_out=None,
                       want_f32: bool = True, want_bf16: bool = False, workspace=None,
                       dev_error=None, stream=None):
    """sa_sparse_step over a two-level page map; returns (pages, counts, O f32 or
    None, O bf16 or None, lse)."""
    lib = load()
    _need_cuda(q, summaries, k_cache, v_cache, page_dir, page_blocks, seq_lens)
    _bf16(q), _bf16(k_cache), _bf16(v_cache), _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    B, T, Hq, D = q.shape
    P_pool, Hkv, P, _ = k_cache.shape
    if P != page_size:
        raise ValueError("page_size differs from the cache's page dimension")
    dargs = _dir_args(page_dir, page_blocks, block_shift)
    bp = budget_tokens // page_size
    if out_pages is None:
        out_pages = torch.empty((B, Hkv, max(bp, 1)), dtype=torch.int32, device=q.device)
    if out_counts is None:
        out_counts = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    _select_shapes(q, summaries, page_dir, seq_lens, out_pages, out_counts, bp)
    o_out, o_out_bf16, lse_out = _attn_outputs(B, T, Hq, D, q.device, o_out, o_out_bf16,
                                               lse_out, want_f32, want_bf16)
    if workspace is None:
        n = sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, page_size,
                                          dir_capacity(page_dir, block_shift), budget_tokens,
                                          n_splits)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _call(lib.sa_sparse_step_dir,
          (_ptr(q), _strides4(q), _ptr(summaries), _ptr(k_cache), _strides4(k_cache),
           _ptr(v_cache), _strides4(v_cache), *dargs, _ptr(seq_lens), B, T, Hq, Hkv, D,
           page_size, P_pool, sink_tokens, local_tokens, budget_tokens, float(scale),
           int(n_splits), _ptr(out_pages), _ptr(out_counts), _ptr(o_out), _ptr(o_out_bf16),
           _ptr(lse_out), _ptr(workspace), workspace.numel(), _ptr(dev_error),
           _stream(stream)), "sa_sparse_step_dir")
    return out_pages, out_counts, o_out, o_out_bf16, lse_out


def sa_append_kv_dir(k_new, v_new, n_new, k_cache, v_cache, page_dir, page_blocks,
                     block_shift: int, seq_lens, summaries, out_seq_lens=None, dev_error=None,
                     stream=None):
    """sa_append_kv over a two-level page map."""
    lib = load()
    _need_cuda(k_new, v_new, n_new, k_cache, v_cache, page_dir, page_blocks, seq_lens, summaries)
    _bf16(k_new), _bf16(v_new), _bf16(k_cache), _bf16(v_cache), _i32(n_new), _i32(seq_lens)
    if summaries.dtype != torch.bfloat16 or not summaries.is_contiguous():
        raise TypeError("summaries must be a contiguous bfloat16 tensor")
    if out_seq_lens is not None:
        _i32(out_seq_lens)
    B, max_new, Hkv, D = k_new.shape
    P_pool, _, P, _ = k_cache.shape
    _call(lib.sa_append_kv_dir,
          (_ptr(k_new), _strides4(k_new), _ptr(v_new), _strides4(v_new), _ptr(n_new), max_new,
           _ptr(k_cache), _strides4(k_cache), _ptr(v_cache), _strides4(v_cache),
           *_dir_args(page_dir, page_blocks, block_shift), _ptr(seq_lens), _ptr(out_seq_lens),
           B, Hkv, D, P, P_pool, _ptr(summaries), _ptr(dev_error), _stream(stream)),
          "sa_append_kv_dir")
    return out_seq_lens
