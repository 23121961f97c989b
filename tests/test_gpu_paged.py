"""GPU parity for a paged KV cache ("Sparse long-context inference with
self-indexing attention", "How much memory the KV cache takes": the cache
held as fixed-size pages).

Each sequence's cache is cut into pages placed at seeded random slots of a
pool with spare, unused slots; the library reads and appends through the
page table (summaries, selection, decode, the fused append + decode step),
and the oracle reads the pool back through the same table with its own
paged_to_contiguous before computing the plain decode.  Selections and
summaries bit for bit, outputs within 2e-3, as for the contiguous cache.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W

from gpu_harness import FixedDecodeCheck, host

pytestmark = pytest.mark.gpu


def _cfg(base, **kw):
    return base.scaled(**kw)


CASES = {
    # pages of 64 rows, page summaries of 16: window starts mid-page, a page
    # of 16 completes inside a fused step (L = 16k + 13, refresh every 4)
    "quest_pages64": (_cfg(W.quest(0), B=2, Hkv=2, Hq=8, L=16 * 500 + 13, budget_tokens=1024,
                           sink=64, window=250, refresh=4, steps=9), 64),
    # pages of 16 rows (one TMA box per page)
    "quest_pages16": (_cfg(W.quest(0), B=2, Hkv=2, Hq=8, L=4096 + 7, budget_tokens=512, sink=40,
                           window=100, refresh=3, steps=5), 16),
    # twelve segments: clustered decode splits, pages of 128
    "largebatch_clustered": (_cfg(W.largebatch(0), B=6, Hkv=2, Hq=8, L=4096 + 31,
                                  budget_tokens=1024, sink=256, window=512, steps=3), 128),
    # MoBA-style current block, G = 8, pages of 256
    "moba_pages256": (_cfg(W.moba(0), Hkv=2, Hq=16, L=128 * 40 + 77, block_size=128, topk=8,
                           n_needles=6, refresh=2, steps=4), 256),
    # head_dim 64 on the tensor-core path
    "quest_d64_pages32": (_cfg(W.quest(0), B=1, Hkv=2, Hq=8, D=64, L=4096 + 9, budget_tokens=512,
                               sink=32, window=128, refresh=2, steps=4), 32),
    # fp32 cache: the CUDA-core decode reads rows through the table
    "moba_f32_pages64": (_cfg(W.moba(0), Hkv=1, Hq=4, kv_dtype=torch.float32, L=64 * 50 + 3,
                              block_size=64, topk=5, n_needles=3, steps=2), 64),
}


@pytest.mark.parametrize("name", list(CASES))
def test_paged_decode_matches_oracle(name):
    cfg, P = CASES[name]
    chk = FixedDecodeCheck(cfg, page_rows=P, spare_pages=5)
    chk.run(cfg.steps)


def test_pool_layout_matches_the_oracle_gather():
    """The pool the library reads is the contiguous cache, gathered back by
    the oracle's own paged_to_contiguous through the page table."""
    cfg, P = CASES["quest_pages64"]
    wl = W.Workload(cfg, "cuda")
    Kp, Vp, table = wl.paged(P, spare_pages=5)
    K, Kp, tab = host(wl.K), host(Kp), table.cpu().numpy()
    assert len(set(tab.ravel().tolist())) == tab.size      # no page used twice
    assert tab.max() < Kp.shape[0] and tab.min() >= 0
    for b in range(cfg.B):
        got = oracle.paged_to_contiguous(Kp, tab[b], P, cfg.L_max)
        assert np.array_equal(got, K[b])


def test_paged_fused_step_is_one_launch():
    """The fused append + decode runs on the paged pool as on a contiguous
    cache (one launch, clustered merge for many segments)."""
    cfg, P = CASES["largebatch_clustered"]
    chk = FixedDecodeCheck(cfg, page_rows=P)
    assert chk.sess.fuses()
    assert N.bsa_decode_kernels(chk.sess.desc, chk.sess.sel, chk.sess.tokens_hint) == \
        chk.sess.decode_kernels
