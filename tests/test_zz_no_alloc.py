"""bsa_decode_noalloc against bsa_decode (GPU).

bsa_decode_noalloc serves callers that cannot allocate device memory for a
workspace, for example code embedded in an application that owns every
device allocation and forbids new ones once it runs, or code that cannot
afford cudaMalloc's implicit synchronisation.  It uses a scratch array built
into the library instead of the caller's workspace, so it must give the same
result as bsa_decode on the same inputs, call after call (the array keeps
the previous call's contents), and refuse problems larger than its 4 MiB.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

pytestmark = pytest.mark.gpu

ATOL = 2e-3   # the decode tests' tolerance against the fp64 oracle


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


@pytest.mark.parametrize("cfg", [
    W.quest(0).scaled(B=2, Hkv=2, Hq=8, L=8192 + 5, budget_tokens=1024, sink=64, window=256),
    W.moba(0).scaled(Hkv=2, Hq=16, L=128 * 40 + 77, block_size=128, topk=8, n_needles=6),
], ids=["quest_small", "moba_small"])
def test_noalloc_matches_decode_twice(cfg):
    sess, q = _prepared(cfg)
    want_out = sess.out.cpu().numpy()
    want_lse = sess.lse.cpu().numpy()
    for _ in range(2):   # two calls in a row: the shared scratch must not leak state
        out, lse = _noalloc(sess, q)
        assert np.abs(out.cpu().numpy() - want_out).max() <= ATOL
        assert np.abs(lse.cpu().numpy() - want_lse).max() <= ATOL


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 64 sequences x 8 KV heads of G = 8, head_dim 128, few splits' worth of
    # partials already exceed the 4 MiB built-in scratch
    desc = N.KvDesc(64, 512, 64, 128, N.BSA_BF16, 1 << 16, 64 * (1 << 16) * 128,
                    (1 << 16) * 128, 128)
    need = N.bsa_workspace_size(desc, None, N.BSA_OP_DECODE, 0, 1 << 15)
    assert need > (4 << 20)
    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(N.BsaError) as e:
        N.bsa_decode_noalloc(desc, dummy, dummy, dummy, dummy, dummy, 8, dummy, 1 << 15, 0.1,
                             dummy, dummy)
    assert e.value.status == N.BSA_ERR_WORKSPACE
