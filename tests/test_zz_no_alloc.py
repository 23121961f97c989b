"""bsa_decode_noalloc against bsa_decode and the oracle (GPU).

bsa_decode_noalloc serves callers that cannot allocate device memory for a
workspace, for example code embedded in an application that owns every
device allocation and forbids new ones once it runs, or code that cannot
afford cudaMalloc's implicit synchronisation.  It uses a scratch array built
into the library instead of the caller's workspace.  It runs the same kernels
with the same split count as bsa_decode, so it must give bit-identical
results, call after call (the array keeps the previous call's contents), and
match the fp64 oracle within the decode tests' tolerance.  It refuses
problems larger than its 4 MiB -- checked here at the exact boundary -- and
its status word stays readable until its next call.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

pytestmark = pytest.mark.gpu

ATOL = 2e-3           # the decode tests' tolerance against the fp64 oracle
SCRATCH = 4 << 20     # the built-in scratch, bytes


def _host(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _prepared(cfg):
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    q = wl.decode_query(0)
    sess.select(q)
    sess.decode(q)
    torch.cuda.synchronize()
    return sess, q


def _noalloc(sess, q):
    out = torch.full_like(sess.out, float("nan"))
    lse = torch.full_like(sess.lse, float("nan"))
    N.bsa_decode_noalloc(sess.desc, q, sess.wl.K, sess.wl.V, sess.ranges, sess.n_ranges,
                         sess.max_ranges, sess.wl.cur_len, sess.tokens_hint, sess.scale, out, lse)
    torch.cuda.synchronize()
    return out, lse


def _oracle_check(sess, q, out, lse, segments):
    c = sess.cfg
    qh, oh, lh = _host(q), out.cpu().numpy(), lse.cpu().numpy()
    n = int(sess.wl.cur_len[0])
    for b, g in segments:
        ref = oracle.decode_fixed_segment(
            qh[b, g * c.G:(g + 1) * c.G], _host(sess.wl.K[b, g]), _host(sess.wl.V[b, g]), n, n,
            c.kind, c.block_size, c.topk, c.budget_tokens, c.sink, c.window, c.keep_current,
            1.0 / math.sqrt(c.D))
        assert np.abs(oh[b, g * c.G:(g + 1) * c.G] - ref["out"]).max() <= ATOL
        assert np.abs(lh[b, g * c.G:(g + 1) * c.G] - ref["lse"]).max() <= ATOL


CASES = {
    "quest_small": W.quest(0).scaled(B=2, Hkv=2, Hq=8, L=8192 + 5, budget_tokens=1024, sink=64,
                                     window=256),
    "moba_small": W.moba(0).scaled(Hkv=2, Hq=16, L=128 * 40 + 77, block_size=128, topk=8,
                                   n_needles=6),
    # 12 segments: the splits merge inside thread-block clusters
    "quest_clustered": W.quest(0).scaled(B=3, Hkv=4, Hq=16, L=16 * 700 + 9, budget_tokens=1024,
                                         sink=64, window=256),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_decode_twice(name):
    sess, q = _prepared(CASES[name])
    c = sess.cfg
    for _ in range(2):   # two calls in a row: the shared scratch must not leak state
        out, lse = _noalloc(sess, q)
        assert torch.equal(out, sess.out) and torch.equal(lse, sess.lse)
        assert N.bsa_workspace_status(None) == (N.BSA_OK, 0)
    _oracle_check(sess, q, out, lse, [(b, g) for b in range(c.B) for g in range(c.Hkv)])


def _boundary_batch():
    """Largest batch of an 8-KV-head, G = 8 geometry whose decode scratch fits
    the built-in array, from bsa_workspace_size (the size bsa_decode checks)."""
    def need(B):
        cfg = W.quest(0).scaled(B=B, Hkv=8, Hq=64, L=512, budget_tokens=128, sink=16, window=64)
        desc = N.KvDesc(B, 64, 8, 128, N.BSA_BF16, cfg.L_max, 8 * cfg.L_max * 128,
                        cfg.L_max * 128, 128)
        sel = N.sel_params(16, topk=-1, budget_tokens=128, sink=16, window=64)
        hint = 16 + 64 + 128 + 16 + cfg.refresh + 1   # the session's token bound
        return N.bsa_workspace_size(desc, sel, N.BSA_OP_DECODE, 0, hint), cfg
    B = 1
    while need(B + 1)[0] <= SCRATCH:
        B += 1
    return B, need(B), need(B + 1)


def test_noalloc_at_the_scratch_boundary():
    B, (need_fit, cfg), (need_over, cfg_over) = _boundary_batch()
    assert need_fit <= SCRATCH < need_over
    sess, q = _prepared(cfg)
    assert N.bsa_workspace_size(sess.desc, sess.sel, N.BSA_OP_DECODE, 0, sess.tokens_hint) == need_fit
    out, lse = _noalloc(sess, q)
    assert torch.equal(out, sess.out) and torch.equal(lse, sess.lse)
    _oracle_check(sess, q, out, lse, [(0, 0), (B // 2, 3), (B - 1, 7)])
    del sess
    # one sequence more needs more than the array holds: refused before any launch
    sess, q = _prepared(cfg_over)
    with pytest.raises(N.BsaError) as e:
        _noalloc(sess, q)
    assert e.value.status == N.BSA_ERR_WORKSPACE


def test_noalloc_status_word_reports_a_wait_that_gives_up():
    sess, q = _prepared(CASES["quest_small"])
    N.bsa_test_arm_wait_limit(1000)
    out, lse = _noalloc(sess, q)
    st, bits = N.bsa_workspace_status(None, clear=False)
    assert st == N.BSA_ERR_TIMEOUT and bits & 1
    assert torch.equal(out, sess.out)
    # the next call starts from a zeroed status word
    _noalloc(sess, q)
    assert N.bsa_workspace_status(None) == (N.BSA_OK, 0)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 64 sequences x 64 KV heads of G = 8, head_dim 128: one split's partials
    # already exceed the 4 MiB built-in scratch
    desc = N.KvDesc(64, 512, 64, 128, N.BSA_BF16, 1 << 16, 64 * (1 << 16) * 128,
                    (1 << 16) * 128, 128)
    need = N.bsa_workspace_size(desc, None, N.BSA_OP_DECODE, 0, 1 << 15)
    assert need > SCRATCH
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(N.BsaError) as e:
        N.bsa_decode_noalloc(desc, dummy, dummy, dummy, dummy, dummy, 8, dummy, 1 << 15, 0.1,
                             dummy, dummy)
    assert e.value.status == N.BSA_ERR_WORKSPACE
