"""Plain CPU oracle for block-sparse long-context attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline / reference leg may import this package.  The product
path (the CUDA library and its Python binding) never imports, loads or calls
it, and this package imports nothing from the product path: the two share no
code, table or helper.  Inputs reach both sides from the seeded generators.

What the oracle computes, with the page (title, section) each step follows:

* KV-cache bytes per token -- "Sparse long-context inference with
  self-indexing attention", section "How much memory the KV cache takes":
  2 x layers x kv_heads x head_dim x bytes.
* Block summaries -- mean-pooled key per block (Module 14 "Sparse attention and
  long context", §14.3 MoBA; here the training-free mean stands in for MoBA's
  learned gate key), normalised centre of normalised keys ("Semantic blocks
  for sparse attention", first section), and Quest-style elementwise min/max
  page bounds ("Sparse attention in hybrid LLMs", section "Which parts of the
  context each layer reads").
* Block scores summed over the G query heads of a KV head, ranked by raw score
  (softmax is monotone, so the top-n by probability in "Sparse long-context
  inference...", section "Importance scores and block selection", is the
  top-n by score).
* Selection: the attention sink (Module 14, §14.2), the sliding window of the
  W most recent tokens ("Sparse long-context inference...", section "Sliding
  window"), MoBA's current block (§14.3), plus the top-k candidate blocks or
  the blocks a token budget admits; ties go to the lower block index.
* Exact softmax attention over the selected tokens in fp64 (Module 14,
  Exercise 14.1, attention with an additive mask).
* The semantic index ("Semantic blocks for sparse attention", first section):
  spherical k-means over the unit keys (Lloyd rounds from given starting
  keys, largest fp32 dot wins, lowest centre on ties, normalised-mean update,
  an empty cluster keeps its centre) and the block-ordered store (clusters in
  index order, positions ascending within a cluster).
* A paged cache ("Sparse long-context inference with self-indexing attention",
  "How much memory the KV cache takes"): pages gathered back into the
  sequence's cache through its page table.
* FP8 (E4M3) cache codes decoded exactly ("Attention mechanisms in modern
  LLMs", basic maths and real cost: narrow KV formats such as FP8).

The fp32 arithmetic that decides the selection follows a fixed order written
out in ``oracle.c``; everything compared with a tolerance is fp64.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
except the semantic-centroid arithmetic's exact fp32 rounding, whose pins are
invariants only (unit norm, identical-key blocks); no page prints a worked
example for it.  The k-means is pinned by recovery of well-separated planted
clusters, agreement with an independent fp64 restatement on an input without
near ties, and the tie and empty-cluster rules; its exact fp32 rounding is
likewise unpinned by any printed example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "_oracle.so")
_LOCK = threading.Lock()
_LIB = None

F32, BF16 = 0, 1
CENTROID, CENTROID_NORM, MINMAX = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no fp contraction, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            lib = ctypes.CDLL(build())
            P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_kv_bytes_per_token.argtypes = [L, L, L, L]
            lib.oracle_kv_bytes_per_token.restype = L
            for name in ("oracle_block_centroid", "oracle_block_centroid_normalized"):
                getattr(lib, name).argtypes = [P, I, L, I, P, P, I, P]
                getattr(lib, name).restype = None
            lib.oracle_block_minmax.argtypes = [P, I, L, I, P, P, I, P, P]
            lib.oracle_block_minmax.restype = None
            lib.oracle_block_scores.argtypes = [P, I, I, I, P, P, I, P, P]
            lib.oracle_block_scores.restype = None
            lib.oracle_attend_rows.argtypes = [P, I, I, P, P, I, L, P, L, D, P, P]
            lib.oracle_attend_rows.restype = None
            lib.oracle_spherical_kmeans.argtypes = [P, I, L, I, L, I, I, P, P, P, P, P]
            lib.oracle_spherical_kmeans.restype = None
            lib.oracle_kmeans_assign.argtypes = [P, I, L, I, P, L, P, I, P]
            lib.oracle_kmeans_assign.restype = None
            _LIB = lib
    return _LIB


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _kv_dtype(a: np.ndarray) -> int:
    """fp32 arrays are read as floats; uint16 arrays hold bf16 bit patterns."""
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"KV arrays must be float32 or uint16 (bf16 bits), got {a.dtype}")


def _rows2d(a: np.ndarray) -> tuple[np.ndarray, int]:
    """A [rows, D] view whose rows may be strided; returns (array, row stride)."""
    assert a.ndim == 2 and a.strides[1] == a.itemsize, "D must be contiguous"
    return a, a.strides[0] // a.itemsize


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (u.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# KV-cache arithmetic
# --------------------------------------------------------------------------

def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """2 x layers x kv_heads x head_dim x bytes ("Sparse long-context
    inference with self-indexing attention", "How much memory the KV cache
    takes")."""
    return int(_lib().oracle_kv_bytes_per_token(layers, kv_heads, head_dim, elem_bytes))


def attention_flops(n_pairs: int, head_dim: int) -> int:
    """Module 14, Exercise 14.1: QK^T and the weighted sum of V cost
    2 * pairs * d flops each, 4 * pairs * d in total."""
    return 4 * n_pairs * head_dim


# --------------------------------------------------------------------------
# Summaries and scores
# --------------------------------------------------------------------------

def block_summaries(K_seg: np.ndarray, beg, end, kind: int):
    """Summaries of blocks [beg[b], end[b]) of one segment's keys [rows, D].

    Returns C [nblk, D] float32 for the centroid kinds, (mn, mx) [nblk, D]
    float32 for MINMAX (values exactly those stored in the cache)."""
    K_seg, ld = _rows2d(K_seg)
    beg = np.ascontiguousarray(beg, dtype=np.int64)
    end = np.ascontiguousarray(end, dtype=np.int64)
    nblk, D = len(beg), K_seg.shape[1]
    lib, dt = _lib(), _kv_dtype(K_seg)
    if kind == MINMAX:
        mn = np.zeros((nblk, D), np.float32)
        mx = np.zeros((nblk, D), np.float32)
        lib.oracle_block_minmax(_ptr(K_seg), dt, ld, D, _ptr(beg), _ptr(end), nblk,
                                _ptr(mn), _ptr(mx))
        return mn, mx
    C = np.zeros((nblk, D), np.float32)
    fn = lib.oracle_block_centroid if kind == CENTROID else lib.oracle_block_centroid_normalized
    fn(_ptr(K_seg), dt, ld, D, _ptr(beg), _ptr(end), nblk, _ptr(C))
    return C


def block_scores(q_grp: np.ndarray, summ, kind: int):
    """Scores of every block for the G query heads of one KV head.

    Returns (s32, s64): the fp32 scores in the fixed order (decide the
    selection) and the fp64 scores from the plain formula (list near-ties)."""
    q = np.ascontiguousarray(q_grp, dtype=np.float32)
    G, D = q.shape
    if kind == MINMAX:
        X, X2 = (np.ascontiguousarray(a, dtype=np.float32) for a in summ)
    else:
        X, X2 = np.ascontiguousarray(summ, dtype=np.float32), None
    nblk = X.shape[0]
    s32 = np.zeros(nblk, np.float32)
    s64 = np.zeros(nblk, np.float64)
    _lib().oracle_block_scores(_ptr(q), G, D, kind, _ptr(X), _ptr(X2) if X2 is not None else None,
                               nblk, _ptr(s32), _ptr(s64))
    return s32, s64


# --------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------

def merge_ranges(ranges):
    """Sorted, disjoint, maximal [a, b) intervals covering the union."""
    out = []
    for a, b in sorted((int(a), int(b)) for a, b in ranges if b > a):
        if out and a <= out[-1][1]:
            out[-1][1] = max(out[-1][1], b)
        else:
            out.append([a, b])
    return [tuple(r) for r in out]


def forced_ranges(n: int, sink: int, window: int, block_size: int, keep_current: bool):
    """Tokens every query reads regardless of scores, for a cache holding n
    tokens whose newest (the current token) is n-1:
      sink      [0, sink)                    (Module 14, §14.2)
      window    the W newest tokens [n-W, n) ("Sliding window"; the window
                counts the current token -- the page's w=512 example lists
                513 positions, an off-by-one this reading does not follow)
      current   the block holding n-1, causally up to n-1 (§14.3 MoBA)."""
    r = []
    if sink > 0:
        r.append((0, min(sink, n)))
    if window > 0:
        r.append((max(0, n - window), n))
    if keep_current and n > 0:
        r.append((((n - 1) // block_size) * block_size, n))
    return merge_ranges(r)


def _covered(a: int, b: int, merged) -> bool:
    return any(lo <= a and b <= hi for lo, hi in merged)


def rank_order(s32: np.ndarray, cands):
    """Candidates by fp32 score descending, lower block index first on ties."""
    return sorted(cands, key=lambda j: (-float(s32[j]), j))


def near_ties(s64: np.ndarray, selected, unselected, rel: float = 1e-6):
    """Pairs across the selection cut whose fp64 scores are within `rel`."""
    if not selected or not unselected:
        return []
    lo = min(s64[j] for j in selected)
    hi = max(s64[j] for j in unselected)
    pairs = []
    for a in selected:
        if s64[a] > hi + rel * max(abs(hi), 1e-30):
            continue
        for b in unselected:
            if s64[b] < lo - rel * max(abs(lo), 1e-30):
                continue
            if abs(s64[a] - s64[b]) <= rel * max(abs(s64[a]), abs(s64[b])):
                pairs.append((int(a), int(b)))
    return pairs


def select_fixed(s32, s64, n: int, block_size: int, topk: int, budget_tokens: int,
                 sink: int, window: int, keep_current: bool):
    """Selection over fixed-size blocks for a cache of n tokens.

    Candidates: complete blocks ((j+1)*S <= n) not wholly inside the forced
    set.  k = topk, or budget_tokens // S when topk < 0 (a budget of whole
    pages).  Returns (selected block ids ascending, token ranges, near-ties)."""
    S = block_size
    forced = forced_ranges(n, sink, window, S, keep_current)
    cands = [j for j in range(n // S) if not _covered(j * S, (j + 1) * S, forced)]
    k = topk if topk >= 0 else budget_tokens // S
    order = rank_order(s32, cands)
    sel = sorted(order[:k])
    ties = near_ties(s64, sel, order[k:])
    ranges = merge_ranges(forced + [(j * S, (j + 1) * S) for j in sel])
    return sel, ranges, ties


def select_budget_greedy(s32, s64, visible, budget_tokens: int):
    """Variable-size blocks under a token budget ("Semantic blocks...": budget
    K = L/16 tokens): walk the blocks in rank order, take a block when its
    visible tokens still fit in what is left of the budget, otherwise skip it
    and go on.  `visible[j]` = tokens of block j the query may read; blocks
    with none are not candidates.  Returns (selected ids ascending, ties)."""
    cands = [j for j in range(len(visible)) if visible[j] > 0]
    order = rank_order(s32, cands)
    used, sel = 0, []
    for j in order:
        if used + int(visible[j]) <= budget_tokens:
            sel.append(j)
            used += int(visible[j])
    sel_set = set(sel)
    ties = near_ties(s64, sel, [j for j in order if j not in sel_set])
    return sorted(sel), ties


def ranges_to_rows(ranges) -> np.ndarray:
    if not ranges:
        return np.zeros(0, np.int64)
    return np.concatenate([np.arange(a, b, dtype=np.int64) for a, b in ranges])


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def attend(q_grp: np.ndarray, K_seg: np.ndarray, V_seg: np.ndarray, rows, scale: float):
    """fp64 softmax attention of the G heads in q_grp over the listed rows."""
    q = np.ascontiguousarray(q_grp, dtype=np.float32)
    G, D = q.shape
    K_seg, ld = _rows2d(K_seg)
    V_seg, ldv = _rows2d(V_seg)
    assert ld == ldv and K_seg.dtype == V_seg.dtype
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size:
        assert rows.min() >= 0 and rows.max() < K_seg.shape[0]
    out = np.zeros((G, D), np.float64)
    lse = np.zeros(G, np.float64)
    _lib().oracle_attend_rows(_ptr(q), G, D, _ptr(K_seg), _ptr(V_seg), _kv_dtype(K_seg), ld,
                              _ptr(rows), rows.size, float(scale), _ptr(out), _ptr(lse))
    return out, lse


# --------------------------------------------------------------------------
# Whole steps
# --------------------------------------------------------------------------

def fixed_block_bounds(n: int, block_size: int):
    nb = n // block_size
    beg = np.arange(nb, dtype=np.int64) * block_size
    return beg, beg + block_size


def decode_fixed_segment(q_grp, K_seg, V_seg, n_sel: int, n_now: int, kind: int,
                         block_size: int, topk: int, budget_tokens: int, sink: int,
                         window: int, keep_current: bool, scale: float, q_sel=None):
    """One (batch, KV head) segment of a decode step over fixed-size blocks.

    Selection happens at the last refresh, for a cache of n_sel tokens and
    with that step's queries q_sel (default: q_grp, a refresh now); the pages
    it picked stay selected until the next refresh while the window keeps
    growing, so attention of the current queries q_grp reads the selected
    ranges with the last one extended to the n_now tokens present now
    ("Sparse attention in hybrid LLMs", "Which parts of the context each
    layer reads": selection is refreshed every 32 steps and the window is
    extended in between)."""
    beg, end = fixed_block_bounds(n_sel, block_size)
    summ = block_summaries(K_seg, beg, end, kind)
    s32, s64 = block_scores(q_grp if q_sel is None else q_sel, summ, kind)
    sel, ranges, ties = select_fixed(s32, s64, n_sel, block_size, topk, budget_tokens,
                                     sink, window, keep_current)
    if ranges and n_now > ranges[-1][1]:
        ranges[-1] = (ranges[-1][0], n_now)
    out, lse = attend(q_grp, K_seg, V_seg, ranges_to_rows(ranges), scale)
    return dict(out=out, lse=lse, sel=sel, ranges=ranges, ties=ties, s32=s32, s64=s64)


def semantic_select_positions(q_grp, Kpos_seg, labels, n_blocks: int, pos_limit: int,
                              budget_tokens: int, centroids=None, order=None):
    """Semantic-block selection for one query group, in ORIGINAL positions.

    labels[p] = block of position p.  A block's centre is computed over all
    its keys in ascending position order (the block's stored order); a query
    may read a block's positions below pos_limit.  `centroids` and `order`
    (the stable sort of the positions by label) may be passed in when the
    same labels are reused.  Returns (selected block ids, selected positions
    ascending, ties, centroids)."""
    labels = np.asarray(labels)
    if order is None:
        order = np.argsort(labels, kind="stable")        # (block, position)
    counts = np.bincount(labels, minlength=n_blocks)
    offs = np.zeros(n_blocks + 1, np.int64)
    offs[1:] = np.cumsum(counts)
    if centroids is None:
        Kperm = np.ascontiguousarray(Kpos_seg[order])
        centroids = block_summaries(Kperm, offs[:-1], offs[1:], CENTROID_NORM)
    s32, s64 = block_scores(q_grp, centroids, CENTROID_NORM)
    visible = np.bincount(labels[:pos_limit], minlength=n_blocks)
    sel, ties = select_budget_greedy(s32, s64, visible, budget_tokens)
    pos = [order[offs[j]:offs[j] + visible[j]] for j in sel]
    pos = np.sort(np.concatenate(pos)) if pos else np.zeros(0, np.int64)
    return sel, pos.astype(np.int64), ties, centroids


# --------------------------------------------------------------------------
# Semantic index: spherical k-means and the block-ordered store
# --------------------------------------------------------------------------

def spherical_kmeans(K_seg: np.ndarray, k: int, iters: int, init):
    """Spherical k-means over one segment's keys [L, D] ("Semantic blocks for
    sparse attention", first section: keys are grouped by spherical k-means
    and each group is stored together).  Reading taken where the page is
    silent: start from the unit keys at rows `init` (k distinct rows),
    `iters` assignments (largest fp32 dot with a unit centre, lowest centre
    index on ties) with the normalised-mean update between them, an empty
    cluster keeping its centre.

    Returns (centres [k, D] f32, labels [L] i32, offsets [k+1] i32, order [L]
    i32): the rows of cluster j in the block-ordered store are
    offsets[j]..offsets[j+1], and order[i] is the original position of
    block-ordered row i (clusters in index order, positions ascending)."""
    K_seg, ld = _rows2d(K_seg)
    L, D = K_seg.shape
    init = np.ascontiguousarray(init, dtype=np.int32)
    assert init.shape == (k,) and len(set(init.tolist())) == k and init.min() >= 0 and init.max() < L
    C = np.zeros((k, D), np.float32)
    labels = np.zeros(L, np.int32)
    offsets = np.zeros(k + 1, np.int32)
    order = np.zeros(L, np.int32)
    _lib().oracle_spherical_kmeans(_ptr(K_seg), _kv_dtype(K_seg), ld, D, L, k, iters, _ptr(init),
                                   _ptr(C), _ptr(labels), _ptr(offsets), _ptr(order))
    return C, labels, offsets, order


def kmeans_assign(K_seg: np.ndarray, rows, C: np.ndarray):
    """The assignment step alone for the keys at `rows` against unit centres
    C [k, D] (same arithmetic as ``spherical_kmeans``)."""
    K_seg, ld = _rows2d(K_seg)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    C = np.ascontiguousarray(C, dtype=np.float32)
    out = np.zeros(len(rows), np.int32)
    _lib().oracle_kmeans_assign(_ptr(K_seg), _kv_dtype(K_seg), ld, K_seg.shape[1], _ptr(rows), len(rows),
                                _ptr(C), C.shape[0], _ptr(out))
    return out


# --------------------------------------------------------------------------
# Paged KV ("Sparse long-context inference with self-indexing attention",
# "How much memory the KV cache takes": the cache as fixed-size pages)
# --------------------------------------------------------------------------

def paged_to_contiguous(pool: np.ndarray, page_table, page_size: int, n_tokens: int) -> np.ndarray:
    """One sequence's cache rows [Hkv, n_tokens, D] from a page pool
    [n_pages, Hkv, page_size, D] and its page table (logical page i of the
    sequence is physical page page_table[i]): token t sits in page
    page_table[t // page_size] at row t % page_size.  Attention over a paged
    cache is attention over this gathered cache, so the contiguous oracle
    applies unchanged."""
    page_table = np.asarray(page_table, dtype=np.int64)
    n_pages = -(-n_tokens // page_size)
    assert len(page_table) >= n_pages and (page_table[:n_pages] >= 0).all()
    assert (page_table[:n_pages] < pool.shape[0]).all()
    t = np.arange(n_tokens)
    rows = pool[page_table[t // page_size], :, t % page_size, :]   # [n_tokens, Hkv, D]
    return np.ascontiguousarray(rows.transpose(1, 0, 2))


# --------------------------------------------------------------------------
# FP8 K/V ("Attention mechanisms in modern LLMs", section on the basic maths
# and the real cost: the KV cache may be kept in FP8 and other narrow formats)
# --------------------------------------------------------------------------

def fp8_e4m3_to_f32(codes) -> np.ndarray:
    """Exact values of FP8 E4M3 codes (1 sign bit, 4 exponent bits with bias 7,
    3 mantissa bits; exponent 0 is subnormal, m * 2^-9; S.1111.111 is NaN and
    there is no infinity, so the largest finite value is 448).  The page says
    only "FP8"; E4M3, the usual format for cached keys and values, is the
    reading taken.  An FP8 cache is read through this table, then the
    fp32/fp64 oracle applies unchanged."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return (sign * val).astype(np.float32)
