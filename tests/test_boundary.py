"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, sizes buffers, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os
import re

import pytest

from block_sparse_long_build_b200 import build as B
from block_sparse_long_build_b200 import native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(N.EXPORTED) == set(names)


def test_version_and_status_strings(lib):
    assert N.bsa_version() >= 100
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert N.status_string(s) and N.status_string(s) != "unknown status"


def _desc(**kw):
    d = dict(B=4, Hq=32, Hkv=8, D=128, kv_dtype=N.BSA_BF16, L_max=65664, stride_b=8 * 65664 * 128,
             stride_h=65664 * 128, stride_t=128)
    d.update(kw)
    return N.KvDesc(**d)


def test_sizes(lib):
    d = _desc()
    p = N.sel_params(16, topk=-1, budget_tokens=4096, sink=256, window=1024)
    assert N.bsa_summary_blocks(d, p) == 65664 // 16
    assert N.bsa_summary_bytes(d, p, N.BSA_SUM_MINMAX) == 32 * (65664 // 16) * 2 * 128 * 2
    assert N.bsa_summary_bytes(d, p, N.BSA_SUM_CENTROID) == 32 * (65664 // 16) * 128 * 4
    assert N.bsa_max_selected(d, p) == 256
    assert N.bsa_max_ranges(d, p) >= 256 + 3
    assert N.bsa_workspace_size(d, p, N.BSA_OP_SELECT) > 0
    assert N.bsa_workspace_size(d, p, N.BSA_OP_DECODE, 0, 5500) > 0


@pytest.mark.parametrize("bad", [dict(D=96), dict(Hq=12), dict(kv_dtype=7), dict(L_max=0),
                                 dict(stride_t=100), dict(B=0)])
def test_bad_descriptor_rejected_on_host(lib, bad):
    d = _desc(**bad)
    p = N.sel_params(16, topk=8)
    fake = 1 << 20   # never dereferenced: validation fails first
    L = N.lib()
    st = L.bsa_decode(ctypes.byref(d), fake, fake, fake, fake, fake, 16, fake, 100, 0.1, fake,
                      None, fake, 1 << 30, None)
    assert st == N.BSA_ERR_ARG
    st = L.bsa_build_summaries(ctypes.byref(d), fake, ctypes.byref(p), 0, 0, 1, fake, None)
    assert st == N.BSA_ERR_ARG


def test_bad_arguments_rejected_on_host(lib):
    L = N.lib()
    d = _desc()
    p = N.sel_params(16, topk=8, sink=4, window=16)
    fake = 1 << 20
    # null output
    assert L.bsa_decode(ctypes.byref(d), fake, fake, fake, fake, fake, 16, fake, 100, 0.1, None,
                        None, fake, 1 << 30, None) == N.BSA_ERR_ARG
    # misaligned K
    assert L.bsa_decode(ctypes.byref(d), fake, fake + 2, fake, fake, fake, 16, fake, 100, 0.1,
                        fake, None, fake, 1 << 30, None) == N.BSA_ERR_ARG
    # non-positive scale
    assert L.bsa_decode(ctypes.byref(d), fake, fake, fake, fake, fake, 16, fake, 100, 0.0, fake,
                        None, fake, 1 << 30, None) == N.BSA_ERR_ARG
    # workspace too small
    assert L.bsa_decode(ctypes.byref(d), fake, fake, fake, fake, fake, 16, fake, 100, 0.1, fake,
                        None, fake, 16, None) == N.BSA_ERR_WORKSPACE
    # summaries past the end of the cache
    assert L.bsa_build_summaries(ctypes.byref(d), fake, ctypes.byref(p), 2, 4100, 10, fake,
                                 None) == N.BSA_ERR_ARG
    # selection buffers smaller than the bound
    assert L.bsa_select(ctypes.byref(d), fake, fake, 2, ctypes.byref(p), fake, 4, fake, fake,
                        64, fake, fake, fake, 1 << 30, None) == N.BSA_ERR_ARG
    # negative sink
    p2 = N.sel_params(16, topk=8, sink=-1)
    assert L.bsa_select(ctypes.byref(d), fake, fake, 2, ctypes.byref(p2), fake, 8, fake, fake,
                        64, fake, fake, fake, 1 << 30, None) == N.BSA_ERR_ARG
    # kernel-count query: bad descriptor, negative token bound
    assert L.bsa_decode_kernels(ctypes.byref(_desc(D=96)), ctypes.byref(p), 100) == N.BSA_ERR_ARG
    assert L.bsa_decode_kernels(ctypes.byref(d), ctypes.byref(p), -1) == N.BSA_ERR_ARG
    # variable blocks without offsets
    p3 = N.sel_params(0, n_blocks=16, topk=-1, budget_tokens=100)
    assert L.bsa_summary_blocks(ctypes.byref(d), ctypes.byref(p3)) == -1
    # grouped prefill outside its domain (fixed blocks)
    assert L.bsa_prefill_grouped(ctypes.byref(d), fake, fake, ctypes.byref(p), fake,
                                 ctypes.byref(d), fake, fake, 0, fake, 0, 16, 0.1, fake, None, fake,
                                 1 << 30, None) in (N.BSA_ERR_ARG, N.BSA_ERR_UNSUPPORTED)


def test_product_path_has_no_oracle_import():
    """The package never imports the oracle (independence of the two sides)."""
    pkg = os.path.join(ROOT, "block_sparse_long_build_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "oracle.c" not in src and "_oracle.so" not in src, f


def test_semantic_index_arguments_rejected_on_host(lib):
    """The index and gather entry points validate on the host and launch
    nothing when an argument is out of range."""
    L = N.lib()
    d = _desc(B=1, Hkv=2, Hq=8, L_max=4096, stride_b=2 * 4096 * 128, stride_h=4096 * 128)
    fake = 1 << 20
    assert N.bsa_index_workspace_size(d, 4096, 64) > 0
    assert N.bsa_index_workspace_size(d, 4097, 64) == 0          # more keys than the cache holds
    assert N.bsa_index_workspace_size(d, 100, 101) == 0           # more clusters than keys
    args = lambda Lk, k, it, ws_bytes: (ctypes.byref(d), fake, Lk, k, it, fake, fake, fake, fake, fake,
                                        fake, ws_bytes, None)
    assert L.bsa_build_semantic_index(*args(4096, 64, 0, 1 << 30)) == N.BSA_ERR_ARG      # no round
    assert L.bsa_build_semantic_index(*args(4096, 0, 5, 1 << 30)) == N.BSA_ERR_ARG       # no cluster
    assert L.bsa_build_semantic_index(*args(4096, 2048, 5, 1 << 30)) == N.BSA_ERR_UNSUPPORTED
    assert L.bsa_build_semantic_index(*args(4096, 64, 5, 16)) == N.BSA_ERR_WORKSPACE
    assert L.bsa_build_semantic_index(ctypes.byref(d), fake, 4096, 64, 5, None, fake, fake, fake, fake,
                                      fake, 1 << 30, None) == N.BSA_ERR_ARG              # no starting rows
    # gather: geometry mismatch, destination overflow, misaligned cache
    d2 = _desc(B=1, Hkv=4, Hq=8, L_max=4096, stride_b=4 * 4096 * 128, stride_h=4096 * 128)
    assert L.bsa_gather_rows(ctypes.byref(d), fake, fake, ctypes.byref(d2), fake, fake, fake, 10, 0,
                             None) == N.BSA_ERR_ARG
    assert L.bsa_gather_rows(ctypes.byref(d), fake, fake, ctypes.byref(d), fake, fake, fake, 100, 4000,
                             None) == N.BSA_ERR_ARG
    assert L.bsa_gather_rows(ctypes.byref(d), fake + 2, fake, ctypes.byref(d), fake, fake, fake, 10, 0,
                             None) == N.BSA_ERR_ARG
    assert L.bsa_gather_rows(ctypes.byref(d), fake, fake, ctypes.byref(d), fake, fake, fake, 0, 0,
                             None) == N.BSA_OK                                           # nothing to do


def test_noalloc_checks_arguments_before_touching_its_scratch(lib):
    """bsa_decode_noalloc makes every check bsa_decode makes before it clears
    its built-in scratch: on a machine without a GPU, a call that got past the
    checks would fail in the CUDA runtime (BSA_ERR_CUDA), so BSA_ERR_ARG here
    shows the rejection came first."""
    L = N.lib()
    d = _desc()
    fake = 1 << 20
    call = lambda q, K, out, scale, max_r: L.bsa_decode_noalloc(
        ctypes.byref(d), q, K, fake, fake, fake, max_r, fake, 100, scale, out, None, None)
    assert call(None, fake, fake, 0.1, 16) == N.BSA_ERR_ARG          # no queries
    assert call(fake, fake + 2, fake, 0.1, 16) == N.BSA_ERR_ARG      # misaligned K
    assert call(fake, fake, None, 0.1, 16) == N.BSA_ERR_ARG          # no output
    assert call(fake, fake, fake, float("nan"), 16) == N.BSA_ERR_ARG
    assert call(fake, fake, fake, 0.1, 0) == N.BSA_ERR_ARG           # no range slot
    g16 = _desc(Hq=8 * 16)
    assert L.bsa_decode_noalloc(ctypes.byref(g16), fake, fake, fake, fake, fake, 16, fake, 100, 0.1,
                                fake, None, None) == N.BSA_ERR_UNSUPPORTED


def test_status_reader_and_test_hook_arguments(lib):
    L = N.lib()
    bits = ctypes.c_uint32(7)
    assert L.bsa_workspace_status(1 << 20, 2, 0, ctypes.byref(bits), None) == N.BSA_ERR_WORKSPACE
    assert L.bsa_workspace_status((1 << 20) + 2, 64, 0, ctypes.byref(bits), None) == N.BSA_ERR_WORKSPACE
    assert L.bsa_test_arm_wait_limit(-1) == N.BSA_ERR_ARG
    assert L.bsa_test_arm_wait_limit(100001) == N.BSA_ERR_ARG
    assert L.bsa_test_arm_wait_limit(0) == N.BSA_OK                  # disarmed


def test_fp8_summary_rows_are_bf16(lib):
    """An FP8 cache's min/max page bounds are stored as exact bf16 pairs: the
    summaries buffer must hold 2 * D * 2 bytes per page (the kernels' rows),
    not 2 * D * 1."""
    d = _desc(kv_dtype=N.BSA_FP8_E4M3)
    p = N.sel_params(16, topk=-1, budget_tokens=4096, sink=256, window=1024)
    nb = 65664 // 16
    assert N.bsa_summary_bytes(d, p, N.BSA_SUM_MINMAX) == 32 * nb * 2 * 128 * 2
    assert N.bsa_summary_bytes(d, p, N.BSA_SUM_CENTROID) == 32 * nb * 128 * 4
    assert N.bsa_summary_bytes(d, p, 7) == 0


def test_paged_descriptor_validation(lib):
    """A paged descriptor needs a table, pages of a multiple of 16 rows and
    L_max = pages_per_seq * page_rows; entry points without a paged path
    refuse it on the host."""
    fake = 1 << 20
    good = dict(B=2, Hkv=2, Hq=8, L_max=64 * 10, stride_b=2 * 64 * 128, stride_h=64 * 128,
                page_rows=64, pages_per_seq=10, page_table=fake, n_pages=25)
    p = N.sel_params(16, topk=4, sink=16, window=32)
    assert N.bsa_summary_blocks(_desc(**good), p) == 40
    for bad in (dict(page_rows=24), dict(page_table=None), dict(L_max=64 * 10 + 16),
                dict(n_pages=0), dict(page_rows=-16)):
        assert N.bsa_summary_blocks(_desc(**{**good, **bad}), p) == -1, bad
    L = N.lib()
    d = _desc(**good)
    assert L.bsa_gather_rows(ctypes.byref(d), fake, fake, ctypes.byref(d), fake, fake, fake, 10, 0,
                             None) == N.BSA_ERR_UNSUPPORTED
    assert L.bsa_build_semantic_index(ctypes.byref(d), fake, 100, 8, 2, fake, fake, fake, fake,
                                      fake, fake, 1 << 30, None) == N.BSA_ERR_UNSUPPORTED


def test_prefill_position_window_rules(lib):
    """The position-ordered window must start at or before pos_limit and cover
    every local key up to q_pos0 + Tq; otherwise the call is refused on the
    host."""
    L = N.lib()
    fake = 1 << 20
    blk = _desc(B=1, Hkv=2, Hq=8, L_max=8192, stride_b=2 * 8192 * 128, stride_h=8192 * 128)
    p = N.sel_params(0, n_blocks=16, block_offsets=fake, kv_pos=fake, topk=-1,
                     budget_tokens=256, pos_limit=4096)
    win = _desc(B=1, Hkv=2, Hq=8, L_max=1024, stride_b=2 * 8192 * 128, stride_h=8192 * 128)

    def call(pos_base, q_pos0, Tq):
        return L.bsa_prefill_grouped(ctypes.byref(blk), fake, fake, ctypes.byref(p), fake,
                                     ctypes.byref(win), fake, fake, pos_base, fake, q_pos0, Tq,
                                     0.1, fake, None, fake, 16, None)

    # valid windows reach the workspace check (too small here)
    assert call(4096, 4096, 1024) == N.BSA_ERR_WORKSPACE
    assert call(4096, 4096, 1025) == N.BSA_ERR_ARG      # past the window's end
    assert call(4097, 4097, 512) == N.BSA_ERR_ARG       # base after pos_limit
    assert call(-1, 4096, 16) == N.BSA_ERR_ARG
