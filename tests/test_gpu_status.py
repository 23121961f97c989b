"""Device-side status reaches the caller (GPU).

Kernels record a wait that gave up (a copy that never arrived) or a cut
result (a prefill query with more blocks in its budget than the library
keeps) in a sticky word at the start of the workspace;
bsa_workspace_status() reads and clears it.  Here a bounded wait is made to
run out on purpose through the library's test hook -- one warp waits, for one
millisecond, on a barrier that nothing completes, before any copy is issued --
and the capacity limit is crossed with a budget that admits every block.
Nothing here stalls or faults the GPU: every wait ends by its own limit.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

pytestmark = pytest.mark.gpu


def _decoded(cfg):
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    q = wl.decode_query(0)
    sess.select(q)
    sess.decode(q)
    torch.cuda.synchronize()
    return sess, q


QUEST = W.quest(0).scaled(B=2, Hkv=2, Hq=8, L=8192 + 5, budget_tokens=1024, sink=64, window=256)


def test_clean_calls_leave_no_status():
    sess, _ = _decoded(QUEST)
    assert N.bsa_workspace_status(sess.ws) == (N.BSA_OK, 0)


def test_wait_that_gives_up_is_reported():
    sess, q = _decoded(QUEST)
    want_out, want_lse = sess.out.clone(), sess.lse.clone()
    N.bsa_test_arm_wait_limit(1000)          # the next decode launch: a 1 ms wait nothing ends
    sess.out.fill_(float("nan"))
    sess.decode(q)
    st, bits = N.bsa_workspace_status(sess.ws, clear=True)
    assert st == N.BSA_ERR_TIMEOUT and bits & 1
    # the launch still ran to completion, with the same results
    assert torch.equal(sess.out, want_out) and torch.equal(sess.lse, want_lse)
    # the word was cleared and the hook fired once
    sess.decode(q)
    assert N.bsa_workspace_status(sess.ws) == (N.BSA_OK, 0)


def test_fused_step_reports_a_wait_that_gives_up():
    cfg = QUEST.scaled(refresh=4, steps=2)
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    for t in range(2):
        q = wl.decode_query(t)
        k, v = wl.decode_new_kv(t)
        if t == 1:
            N.bsa_test_arm_wait_limit(1000)
        sess.step(t, q, k, v)
    st, _ = N.bsa_workspace_status(sess.ws)
    assert st == N.BSA_ERR_TIMEOUT
    assert int(wl.cur_len[0]) == cfg.L + 2   # the step's append still happened


def _semantic(n_blocks, L=16384, Tq=1024, Hkv=2, Hq=8):
    cfg = W.semantic(0).scaled(L=L, n_blocks=n_blocks, chunk=Tq, steps=1, Hkv=Hkv, Hq=Hq,
                               budget_tokens=L // 16, dense_below=4096)
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    return cfg, wl, sess


def _prefill(cfg, wl, sess, p, budget):
    Tq = cfg.chunk
    sel = N.sel_params(0, cfg.n_blocks, wl.block_offsets, wl.kv_pos, topk=-1, budget_tokens=budget,
                       local_start=wl.local_start, pos_limit=p)
    need = N.bsa_workspace_size(sess.desc, sel, N.BSA_OP_PREFILL, Tq, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty(Tq, cfg.Hq, cfg.D, device="cuda")
    lse = torch.empty(Tq, cfg.Hq, device="cuda")
    Q = wl.prefill_queries(p, Tq)
    Kw, Vw = wl.Kpos[:, :, p:p + Tq], wl.Vpos[:, :, p:p + Tq]   # the chunk's own rows
    N.bsa_prefill_grouped(sess.desc, wl.K, wl.V, sel, sess.summaries, N.kv_desc(Kw, cfg.Hq), Kw, Vw,
                          p, Q, p, Tq, 1 / math.sqrt(cfg.D), out, lse, ws)
    return N.bsa_workspace_status(ws), out


def test_prefill_capacity_is_reported():
    """128 blocks and a budget as large as the prefix: every visible block
    fits, more than the 64 a query keeps."""
    cfg, wl, sess = _semantic(128)
    p = cfg.L - cfg.chunk
    (st, bits), out = _prefill(cfg, wl, sess, p, budget=p)
    assert st == N.BSA_ERR_CAPACITY and bits == 4
    # the same chunk under the configured budget (prefix / 16) stays within it
    (st, bits), out = _prefill(cfg, wl, sess, p, budget=p // 16)
    assert (st, bits) == (N.BSA_OK, 0)
    assert torch.isfinite(out).all()
