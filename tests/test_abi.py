"""The C-ABI library loads, exports every entry point include/sa.h declares, and
rejects bad arguments on the host before any launch.  CPU only: no call here
reaches a kernel."""
import ctypes
import os
import re

import pytest

import paged_sparse_kv_sa_b200 as sa
from paged_sparse_kv_sa_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"SA_API\s+[\w\s\*]+?\b(sa_\w+)\s*\(", txt)
    return names


def test_library_exports_every_declared_symbol():
    lib = sa.load()
    names = declared_symbols()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(_lib.EXPORTED)


def test_status_strings_and_version():
    lib = sa.load()
    assert lib.sa_abi_version() == 100
    assert lib.sa_status_string(0) == b"SA_OK"
    assert lib.sa_status_string(1) == b"SA_ERR_INVALID_ARG"
    assert lib.sa_status_string(99) == b"SA_ERR_UNKNOWN"


def _i64x4(*v):
    return (ctypes.c_int64 * 4)(*v)


def test_host_validation_rejects_bad_arguments():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    s = _i64x4(1024, 1024, 128, 1)
    # Hq not a multiple of Hkv
    assert lib.sa_select_pages(fake, s, fake, fake, fake, 1, 1, 6, 4, 128, 16, 8, 8, 32, 64, 256,
                               fake, fake, fake, 1 << 30, None, None) == 1
    # sink + local above the budget
    assert lib.sa_select_pages(fake, s, fake, fake, fake, 1, 1, 8, 2, 128, 16, 8, 8, 512, 512,
                               256, fake, fake, fake, 1 << 30, None, None) == 1
    # null outputs
    assert lib.sa_select_pages(fake, s, fake, fake, fake, 1, 1, 8, 2, 128, 16, 8, 8, 32, 64, 256,
                               None, fake, fake, 1 << 30, None, None) == 1
    # workspace too small
    assert lib.sa_select_pages(fake, s, fake, fake, fake, 1, 1, 8, 2, 128, 16, 8, 8, 32, 64, 256,
                               fake, fake, fake, 16, None, None) == 3
    assert lib.sa_select_workspace_size(2, 8, 100) == 2 * 8 * 100 * 8
    # unsupported head dim
    assert lib.sa_select_pages(fake, _i64x4(96, 96, 96, 1), fake, fake, fake, 1, 1, 8, 2, 96, 16,
                               8, 8, 32, 64, 256, fake, fake, fake, 1 << 30, None, None) == 2
    # misaligned q / non-unit feature stride
    assert lib.sa_select_pages(ctypes.c_void_p(0x1002), s, fake, fake, fake, 1, 1, 8, 2, 128, 16,
                               8, 8, 32, 64, 256, fake, fake, fake, 1 << 30, None, None) == 1
    assert lib.sa_select_pages(fake, _i64x4(1024, 1024, 128, 2), fake, fake, fake, 1, 1, 8, 2, 128,
                               16, 8, 8, 32, 64, 256, fake, fake, fake, 1 << 30, None, None) == 1
    h2l = (ctypes.c_int32 * 8)(0, 0, 0, 0, 1, 1, 1, 5)   # list id out of range
    ks = _i64x4(4096, 2048, 128, 1)
    args = [fake, s, fake, ks, fake, ks, fake, 8, fake, fake, fake, 2, 16,
            ctypes.cast(h2l, ctypes.c_void_p), 1, 1, 8, 2, 128, 128, 16, 64, 0.1, 1, fake, fake,
            None, None]
    assert lib.sa_sparse_decode(*args) == 1
    h2l[7] = 1
    args[22] = float("nan")
    assert lib.sa_sparse_decode(*args) == 1                  # non-finite scale
    args[22] = 0.1
    args[20] = 24                                              # page size not a multiple of 16
    assert lib.sa_sparse_decode(*args) == 2
    args[20] = 16
    args[19] = 64                                              # Dk != Dv
    assert lib.sa_sparse_decode(*args) == 2
    # combine: Dv not a multiple of 4, no outputs
    assert lib.sa_combine(fake, fake, 2, 10, 6, fake, None, None, None) == 1
    assert lib.sa_combine(fake, fake, 2, 10, 8, None, None, None, None) == 1
    # block union: offset past the end
    assert lib.sa_block_union(fake, 8, 2, 4, 10, 8, 2, 1, fake, fake, None) == 1


def test_calls_fail_loudly_without_gpu_tensors():
    import torch
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sa.sa_select_pages(q, torch.zeros((4, 2, 64), dtype=torch.bfloat16),
                           torch.zeros((1, 4), dtype=torch.int32),
                           torch.zeros((1,), dtype=torch.int32), 16, 16, 16, 64)


def test_attention_workspace_size_and_host_checks():
    lib = sa.load()
    # the split partials: [n_splits, rows, Dv] float32 then [n_splits, rows] float32,
    # each rounded up to 16 bytes
    rows, dv, ns = 2 * 1 * 8, 128, 3
    r16 = lambda x: (x + 15) // 16 * 16
    assert lib.sa_sparse_attention_workspace_size(2, 1, 8, dv, ns) == \
        r16(rows * dv * ns * 4) + r16(rows * ns * 4)
    assert lib.sa_sparse_attention_workspace_size(3, 2, 5, 64, 1) == r16(30 * 64 * 4) + r16(30 * 4)
    fake = ctypes.c_void_p(0x1000)
    s = _i64x4(1024, 1024, 128, 1)
    ks = _i64x4(4096, 2048, 128, 1)
    h2l = (ctypes.c_int32 * 8)(0, 0, 0, 0, 1, 1, 1, 1)
    need = lib.sa_sparse_attention_workspace_size(1, 1, 8, 128, 2)

    def call(o_out, ws, ws_bytes):
        return lib.sa_sparse_attention(fake, s, fake, ks, fake, ks, fake, 8, fake, fake, fake, 2,
                                       16, ctypes.cast(h2l, ctypes.c_void_p), 1, 1, 8, 2, 128,
                                       128, 16, 64, 0.1, 2, o_out, None, None, ws, ws_bytes, None,
                                       None)
    assert call(fake, None, need) == 3                        # no workspace
    assert call(fake, fake, need - 16) == 3                   # too small
    assert call(fake, ctypes.c_void_p(0x1008), need) == 3     # not 16-byte aligned
    assert call(None, fake, need) == 1                        # no output at all
    assert call(ctypes.c_void_p(0x1004), fake, need) == 1     # float32 output misaligned
    assert lib.sa_sparse_attention_fp8(fake, s, fake, ks, fake, ks, fake, fake, fake, 8, fake,
                                       fake, fake, 2, 16, ctypes.cast(h2l, ctypes.c_void_p), 1, 1,
                                       8, 2, 128, 16, 64, 0.1, 2, fake, None, None, None, need,
                                       None, None) == 3


def test_step_workspace_size_and_host_checks():
    lib = sa.load()
    r16 = lambda x: (x + 15) // 16 * 16
    # score bounds [B, Hkv, max_pages] x 8 bytes, then the split partials
    B, T, Hq, Hkv, D, P, mp, budget, ns = 16, 1, 32, 8, 128, 16, 2048, 1024, 13
    rows = B * T * Hq
    assert lib.sa_sparse_step_workspace_size(B, T, Hq, Hkv, D, P, mp, budget, ns) == \
        r16(B * Hkv * mp * 8) + r16(rows * D * ns * 4) + r16(rows * ns * 4)
    assert lib.sa_sparse_step_workspace_size(B, T, 30, Hkv, D, P, mp, budget, ns) == 0   # Hq % Hkv
    assert lib.sa_sparse_step_workspace_size(B, T, Hq, Hkv, 96, P, mp, budget, ns) == 0  # head dim
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    s = _i64x4(4096, 4096, 128, 1)
    ks = _i64x4(4096, 2048, 128, 1)
    need = lib.sa_sparse_step_workspace_size(2, 1, 8, 2, 128, 16, 64, 256, 2)

    def call(ws, ws_bytes, o_out=fake, k=fake, scale=0.1, sink=32):
        return lib.sa_sparse_step(fake, s, fake, k, ks, fake, ks, fake, 64, fake, 2, 1, 8, 2, 128,
                                  16, 128, sink, 64, 256, scale, 2, fake, fake, o_out, None, None,
                                  ws, ws_bytes, None, None)
    assert call(None, need) == 3                              # no workspace
    assert call(fake, need - 16) == 3                         # too small
    assert call(ctypes.c_void_p(0x1008), need) == 3           # not 16-byte aligned
    assert call(fake, need, o_out=None) == 1                  # no output at all
    assert call(fake, need, k=ctypes.c_void_p(0x1004)) == 1   # cache base misaligned
    assert call(fake, need, scale=float("inf")) == 1          # scale not finite
    assert call(fake, need, sink=512) == 1                    # sink + local above the budget


def test_append_host_checks():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    kn = _i64x4(40 * 8 * 128, 8 * 128, 128, 1)
    ks = _i64x4(8 * 16 * 128, 16 * 128, 128, 1)

    def call(D=128, kn_=kn, out=None, seq=fake, max_new=40):
        return lib.sa_append_kv(fake, kn_, fake, kn, fake, max_new, fake, ks, fake, ks, fake, 64,
                                seq, out, 4, 8, D, 16, 1000, fake, None, None)
    assert call(D=100) == 1                                   # D not a multiple of 8
    assert call(kn_=_i64x4(40 * 8 * 128, 8 * 128, 128, 2)) == 1   # feature stride not 1
    assert call(kn_=_i64x4(40 * 8 * 128, 8 * 128, 124, 1)) == 1   # head stride not 16 bytes
    assert call(out=fake) == 1                                # new lengths over the old ones
    assert call(seq=None) == 1                                # no lengths
    assert call(max_new=-1) == 1


def test_two_level_map_host_checks():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    ks = _i64x4(8 * 64 * 128, 64 * 128, 128, 1)

    def summ(page_dir=fake, n_dir=4, blocks=fake, n_blocks=3, shift=6, B=2):
        return lib.sa_build_page_summaries_dir(fake, ks, page_dir, n_dir, blocks, n_blocks, shift,
                                               fake, B, 8, 128, 64, 100, fake, None, None)
    assert summ(page_dir=None) == 1
    assert summ(blocks=None) == 1
    assert summ(n_dir=-1) == 1
    assert summ(n_blocks=-1) == 1
    assert summ(shift=-1) == 1
    assert summ(shift=17) == 1
    assert summ(n_dir=1 << 15, shift=16) == 2                 # capacity above 2^30 pages
    assert summ(B=-1) == 1
    assert summ(B=0) == 0                                     # nothing to do, nothing launched

    qs = _i64x4(32 * 128, 32 * 128, 128, 1)
    kvs = _i64x4(8 * 64 * 128, 64 * 128, 128, 1)

    def step(n_dir=4, shift=6, ws_bytes=1 << 30):
        return lib.sa_sparse_step_dir(fake, qs, fake, fake, kvs, fake, kvs, fake, n_dir, fake, 3,
                                      shift, fake, 2, 1, 32, 8, 128, 64, 100, 64, 512, 2048, 0.08,
                                      4, fake, fake, fake, None, None, fake, ws_bytes, None, None)
    assert step(shift=20) == 1
    assert step(n_dir=300) == 2                               # 19200 pages: above the selection's 16384
    assert step(ws_bytes=16) == 3                             # workspace below the size call's
    need = lib.sa_sparse_step_workspace_size(2, 1, 32, 8, 128, 64, 4 << 6, 2048, 4)
    assert need > 0 and step(ws_bytes=need - 16) == 3

    kn = _i64x4(40 * 8 * 128, 8 * 128, 128, 1)

    def app(shift=3, blocks=fake):
        return lib.sa_append_kv_dir(fake, kn, fake, kn, fake, 40, fake, kvs, fake, kvs, fake, 4,
                                    blocks, 3, shift, fake, None, 4, 8, 128, 64, 1000, fake, None,
                                    None)
    assert app(shift=-2) == 1
    assert app(blocks=None) == 1


def test_ambient_heads_host_checks():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)      # never dereferenced: validation fails first
    s = _i64x4(2 * 128 * 576, 128 * 576, 576, 1)
    # partials [B, chunks of 32 pages, T * Hq rows, 3] float64
    assert lib.sa_select_ambient_heads_workspace_size(8, 2, 128, 1024) == 8 * 32 * 256 * 3 * 8
    need = lib.sa_select_ambient_heads_workspace_size(8, 2, 128, 1024)

    def call(h=32, Dk=576, ws=fake, ws_bytes=need, scale=0.04):
        return lib.sa_select_ambient_heads(fake, s, fake, fake, 1024, fake, fake, fake, 32, 8, 2,
                                           128, Dk, 64, 8192, scale, h, fake, None, ws, ws_bytes,
                                           None, None)
    assert call(h=129) == 1                                   # more heads than there are
    assert call(h=-1) == 1
    assert call(scale=float("nan")) == 1
    assert call(Dk=1024) == 2                                 # head dim above what it runs
    assert call(ws=None) == 3
    assert call(ws_bytes=need - 8) == 3


def test_default_split_policy():
    from paged_sparse_kv_sa_b200.pipeline import default_splits
    # one wave of decode warps (12 per SM on 148 SMs) over the (sequence, kv head) units
    assert default_splits(16 * 8, 64, 148) == 13      # Llama-8B-shaped decode
    assert default_splits(32 * 8, 128, 148) == 6      # Llama-70B-shaped decode
    assert default_splits(2, 16, 148) == 16           # never more splits than list entries
    assert default_splits(0, 5, 148) == 1
    for units, max_list in [(4, 1000), (1, 5000), (300, 300), (7, 129)]:
        n = default_splits(units, max_list, 148)
        assert 1 <= n <= 64
        assert -(-max_list // n) <= 128 or n == 64   # a split holds at most 128 entries


def test_tiered_selection_host_checks():
    lib = sa.load()
    fake = ctypes.c_void_p(0x1000)
    s = _i64x4(2 * 128 * 576, 128 * 576, 576, 1)

    def call(max_pages, alpha=8, beta=24, Dk=576, ws_bytes=1 << 40):
        return lib.sa_select_pages_tiered(fake, s, fake, fake, fake, 8, 2, 128, Dk, 64, max_pages,
                                          8192, alpha, beta, fake, fake, fake, ws_bytes, None,
                                          None)
    assert call(8193) == 2                    # above the 8192 pages its choose pass holds
    assert call(1024, Dk=572) == 2            # Dk not a multiple of 8
    assert call(1024, alpha=0, beta=0) == 1   # no page asked for
    assert call(1024, alpha=-1) == 1
    assert call(1024, ws_bytes=16) == 3       # workspace too small
    assert call(0) == 0                       # nothing to select: no launch
    # workspace: brackets and row masks per (sequence, 32-row group, page), exact-score
    # keys per (sequence, page), one counter per sequence (16-byte rounded)
    n_rg = (2 * 128 + 31) // 32
    want = 8 * 1024 * (n_rg * (8 + 8) + 8) + (8 * 4 + 15) // 16 * 16
    assert lib.sa_select_tiered_workspace_size(8, 2, 128, 1024) == want
