"""ctypes binding of libbsa.so: the C entry points under the same names.

Argument marshalling only -- every step of the computation runs in the CUDA
kernels behind these calls.  Tensors are torch tensors (device memory and
streams come from PyTorch); descriptors are built from them.  There is no
fallback: if the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

(BSA_OK, BSA_ERR_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_CUDA, BSA_ERR_WORKSPACE, BSA_ERR_TIMEOUT,
 BSA_ERR_CAPACITY) = (0, -1, -2, -3, -4, -5, -6)
BSA_SUM_CENTROID, BSA_SUM_CENTROID_NORM, BSA_SUM_MINMAX = 0, 1, 2
BSA_F32, BSA_BF16, BSA_FP8_E4M3 = 0, 1, 2
_DTYPES = {torch.float32: BSA_F32, torch.bfloat16: BSA_BF16, torch.float8_e4m3fn: BSA_FP8_E4M3}
BSA_OP_SELECT, BSA_OP_DECODE, BSA_OP_PREFILL, BSA_OP_APPEND = 0, 1, 2, 3

EXPORTED = ("bsa_version", "bsa_status_string", "bsa_summary_blocks", "bsa_summary_bytes",
            "bsa_max_selected", "bsa_max_ranges", "bsa_decode_kernels", "bsa_workspace_size", "bsa_build_summaries",
            "bsa_select", "bsa_decode", "bsa_decode_noalloc", "bsa_append_kv", "bsa_decode_step",
            "bsa_prefill_grouped", "bsa_index_workspace_size", "bsa_build_semantic_index",
            "bsa_gather_rows", "bsa_workspace_status", "bsa_test_arm_wait_limit")


class BsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")
        self.status = status


class KvDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("kv_dtype", ctypes.c_int32), ("L_max", ctypes.c_int32),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("stride_t", ctypes.c_int64), ("page_rows", ctypes.c_int32),
                ("pages_per_seq", ctypes.c_int32), ("page_table", ctypes.c_void_p),
                ("n_pages", ctypes.c_int64)]


class SelParams(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int32), ("n_blocks", ctypes.c_int32),
                ("block_offsets", ctypes.c_void_p), ("kv_pos", ctypes.c_void_p),
                ("topk", ctypes.c_int32), ("budget_tokens", ctypes.c_int32),
                ("sink", ctypes.c_int32), ("window", ctypes.c_int32),
                ("keep_current_block", ctypes.c_int32), ("local_start", ctypes.c_int32),
                ("pos_limit", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libbsa.so; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbsa.so not built ({LIB_PATH}); run block_sparse_long_build_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                              ctypes.c_float)
        pd, pp = ctypes.POINTER(KvDesc), ctypes.POINTER(SelParams)
        sig = {
            "bsa_version": (I32, []),
            "bsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "bsa_summary_blocks": (I32, [pd, pp]),
            "bsa_summary_bytes": (SZ, [pd, pp, ctypes.c_int]),
            "bsa_max_selected": (I32, [pd, pp]),
            "bsa_max_ranges": (I32, [pd, pp]),
            "bsa_decode_kernels": (I32, [pd, pp, I32]),
            "bsa_index_workspace_size": (SZ, [pd, ctypes.c_int64, I32]),
            "bsa_build_semantic_index": (ctypes.c_int, [pd, P, ctypes.c_int64, I32, I32, P, P, P, P, P, P, SZ, P]),
            "bsa_gather_rows": (ctypes.c_int, [pd, P, P, pd, P, P, P, ctypes.c_int64, ctypes.c_int64, P]),
            "bsa_workspace_size": (SZ, [pd, pp, ctypes.c_int, I32, I32]),
            "bsa_build_summaries": (ctypes.c_int, [pd, P, pp, ctypes.c_int, I32, I32, P, P]),
            "bsa_select": (ctypes.c_int, [pd, P, P, ctypes.c_int, pp, P, I32, P, P, I32, P, P, P,
                                          SZ, P]),
            "bsa_decode": (ctypes.c_int, [pd, P, P, P, P, P, I32, P, I32, F, P, P, P, SZ, P]),
            "bsa_decode_noalloc": (ctypes.c_int, [pd, P, P, P, P, P, I32, P, I32, F, P, P, P]),
            "bsa_append_kv": (ctypes.c_int, [pd, P, P, P, P, P, pp, ctypes.c_int, P, P]),
            "bsa_decode_step": (ctypes.c_int, [pd, P, P, P, P, P, P, pp, ctypes.c_int, P, P, P, I32,
                                               I32, F, P, P, P, SZ, P]),
            "bsa_prefill_grouped": (ctypes.c_int, [pd, P, P, pp, P, pd, P, P, I32, P, I32, I32, F, P,
                                                   P, P, SZ, P]),
            "bsa_workspace_status": (ctypes.c_int, [P, SZ, I32, ctypes.POINTER(ctypes.c_uint32), P]),
            "bsa_test_arm_wait_limit": (ctypes.c_int, [I32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bsa_status_string(status).decode()


def _check(fn: str, status: int):
    if status != BSA_OK:
        raise BsaError(fn, status)


def _p(t):
    """Device (or host) pointer of a tensor, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def kv_desc(K: torch.Tensor, Hq: int) -> KvDesc:
    """Descriptor of a [B, Hkv, L_max, D] cache (D contiguous)."""
    assert K.dim() == 4 and K.stride(3) == 1
    dt = _DTYPES[K.dtype]
    B, H, L, D = K.shape
    return KvDesc(B, Hq, H, D, dt, L, K.stride(0), K.stride(1), K.stride(2), 0, 0, None, 0)


def paged_kv_desc(pool: torch.Tensor, Hq: int, page_table: torch.Tensor) -> KvDesc:
    """Descriptor of a paged cache: pool [n_pages, Hkv, page_rows, D] (D
    contiguous) and page_table int32 [B, pages_per_seq] on the device."""
    assert pool.dim() == 4 and pool.stride(3) == 1
    assert page_table.dtype == torch.int32 and page_table.dim() == 2 and page_table.is_contiguous()
    dt = _DTYPES[pool.dtype]
    n_pages, H, P, D = pool.shape
    B, pps = page_table.shape
    return KvDesc(B, Hq, H, D, dt, pps * P, pool.stride(0), pool.stride(1), pool.stride(2), P, pps,
                  page_table.data_ptr(), n_pages)


def sel_params(block_size=0, n_blocks=0, block_offsets=None, kv_pos=None, topk=-1,
               budget_tokens=0, sink=0, window=0, keep_current_block=False, local_start=0,
               pos_limit=0) -> SelParams:
    return SelParams(block_size, n_blocks, _p(block_offsets), _p(kv_pos), topk, budget_tokens,
                     sink, window, int(bool(keep_current_block)), local_start, pos_limit)


def bsa_version() -> int:
    return lib().bsa_version()


def bsa_summary_blocks(desc, sel) -> int:
    return lib().bsa_summary_blocks(ctypes.byref(desc), ctypes.byref(sel))


def bsa_summary_bytes(desc, sel, kind) -> int:
    return lib().bsa_summary_bytes(ctypes.byref(desc), ctypes.byref(sel), kind)


def bsa_max_selected(desc, sel) -> int:
    return lib().bsa_max_selected(ctypes.byref(desc), ctypes.byref(sel))


def bsa_max_ranges(desc, sel) -> int:
    return lib().bsa_max_ranges(ctypes.byref(desc), ctypes.byref(sel))


def bsa_decode_kernels(desc, sel, tokens_hint) -> int:
    r = lib().bsa_decode_kernels(ctypes.byref(desc), ctypes.byref(sel), tokens_hint)
    if r < 0:
        raise BsaError("bsa_decode_kernels", r)
    return r


def bsa_workspace_size(desc, sel, op, n_queries=0, tokens_hint=0) -> int:
    return lib().bsa_workspace_size(ctypes.byref(desc), ctypes.byref(sel) if sel else None, op,
                                    n_queries, tokens_hint)


def bsa_build_summaries(desc, K, sel, kind, first_block, n_blocks, summaries, stream=None):
    _check("bsa_build_summaries",
           lib().bsa_build_summaries(ctypes.byref(desc), _p(K), ctypes.byref(sel), kind,
                                     first_block, n_blocks, _p(summaries), _stream(stream)))


def bsa_select(desc, q, summaries, kind, sel, cur_len, max_selected, sel_blocks, sel_count,
               max_ranges, ranges, n_ranges, ws, stream=None):
    _check("bsa_select",
           lib().bsa_select(ctypes.byref(desc), _p(q), _p(summaries), kind, ctypes.byref(sel),
                            _p(cur_len), max_selected, _p(sel_blocks), _p(sel_count), max_ranges,
                            _p(ranges), _p(n_ranges), _p(ws), ws.numel() * ws.element_size(),
                            _stream(stream)))


def bsa_decode(desc, q, K, V, ranges, n_ranges, max_ranges, cur_len, tokens_hint, scale, out,
               lse, ws, stream=None):
    _check("bsa_decode",
           lib().bsa_decode(ctypes.byref(desc), _p(q), _p(K), _p(V), _p(ranges), _p(n_ranges),
                            max_ranges, _p(cur_len), tokens_hint, scale, _p(out), _p(lse), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)))


def bsa_decode_noalloc(desc, q, K, V, ranges, n_ranges, max_ranges, cur_len, tokens_hint, scale,
                       out, lse, stream=None):
    """bsa_decode with the library's built-in scratch instead of a workspace,
    for callers that cannot allocate one (see include/bsa.h)."""
    _check("bsa_decode_noalloc",
           lib().bsa_decode_noalloc(ctypes.byref(desc), _p(q), _p(K), _p(V), _p(ranges),
                                    _p(n_ranges), max_ranges, _p(cur_len), tokens_hint, scale,
                                    _p(out), _p(lse), _stream(stream)))


def bsa_append_kv(desc, K, V, k_new, v_new, cur_len, sel, kind, summaries, stream=None):
    _check("bsa_append_kv",
           lib().bsa_append_kv(ctypes.byref(desc), _p(K), _p(V), _p(k_new), _p(v_new),
                               _p(cur_len), ctypes.byref(sel) if sel is not None else None, kind,
                               _p(summaries), _stream(stream)))


def bsa_decode_step(desc, q, K, V, k_new, v_new, cur_len, sel, kind, summaries, ranges, n_ranges,
                    max_ranges, tokens_hint, scale, out, lse, ws, stream=None):
    """bsa_append_kv then bsa_decode, in one launch where the tensor-core
    path applies."""
    _check("bsa_decode_step",
           lib().bsa_decode_step(ctypes.byref(desc), _p(q), _p(K), _p(V), _p(k_new), _p(v_new),
                                 _p(cur_len), ctypes.byref(sel) if sel is not None else None,
                                 kind, _p(summaries), _p(ranges), _p(n_ranges), max_ranges,
                                 tokens_hint, scale, _p(out), _p(lse), _p(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)))


def bsa_prefill_grouped(desc, K, V, sel, summaries, pos_desc, K_pos, V_pos, pos_base, Q, q_pos0,
                        Tq, scale, out, lse, ws, stream=None):
    _check("bsa_prefill_grouped",
           lib().bsa_prefill_grouped(ctypes.byref(desc), _p(K), _p(V), ctypes.byref(sel),
                                     _p(summaries), ctypes.byref(pos_desc), _p(K_pos), _p(V_pos),
                                     pos_base, _p(Q), q_pos0, Tq, scale, _p(out), _p(lse), _p(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def bsa_index_workspace_size(desc, L, n_clusters) -> int:
    return lib().bsa_index_workspace_size(ctypes.byref(desc), L, n_clusters)


def bsa_build_semantic_index(desc, K, L, n_clusters, iters, init, centres, labels, offsets, order, ws,
                             stream=None):
    _check("bsa_build_semantic_index",
           lib().bsa_build_semantic_index(ctypes.byref(desc), _p(K), L, n_clusters, iters, _p(init),
                                          _p(centres), _p(labels), _p(offsets), _p(order), _p(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)))


def bsa_gather_rows(src, K, V, dst, K_out, V_out, rows, n, dst_row0=0, stream=None):
    _check("bsa_gather_rows",
           lib().bsa_gather_rows(ctypes.byref(src), _p(K), _p(V), ctypes.byref(dst), _p(K_out), _p(V_out),
                                 _p(rows), n, dst_row0, _stream(stream)))


def bsa_workspace_status(ws, clear=True, stream=None) -> tuple[int, int]:
    """Waits for `stream`, reads (and by default clears) the sticky device-side
    status word of a workspace tensor; ws=None reads the scratch built into
    the library for bsa_decode_noalloc.  Returns (status, raw bits) without
    raising: BSA_OK, BSA_ERR_TIMEOUT or BSA_ERR_CAPACITY."""
    bits = ctypes.c_uint32(0)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    r = lib().bsa_workspace_status(_p(ws), nbytes, int(bool(clear)), ctypes.byref(bits),
                                   _stream(stream))
    if r not in (BSA_OK, BSA_ERR_TIMEOUT, BSA_ERR_CAPACITY):
        raise BsaError("bsa_workspace_status", r)
    return r, bits.value


def bsa_test_arm_wait_limit(limit_us: int):
    """Test hook: the next tensor-core decode launch makes one warp wait on a
    barrier nothing completes, for at most limit_us microseconds, and report
    it as a timeout (see include/bsa.h)."""
    _check("bsa_test_arm_wait_limit", lib().bsa_test_arm_wait_limit(limit_us))
