"""GPU parity: the decode path through the C ABI against the CPU oracle.

Cases span several 16-row pieces, several split-K CTAs and ragged tails; the
small sizes keep the fp64 oracle within seconds.  The workloads at their full
sizes are checked (all or sampled segments, chosen steps) in
test_gpu_fullsize.py.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W

from gpu_harness import FixedDecodeCheck

pytestmark = pytest.mark.gpu


def _cfg(base, **kw):
    return base.scaled(**kw)


CASES = {
    # the tiny configuration exactly as specified (fp32, D 64, CUDA-core path)
    "tiny": W.tiny(0),
    # Quest-style pages of 16, refresh every 4 steps, window extension, ragged L
    "quest_small": _cfg(W.quest(0), B=2, Hkv=2, Hq=8, L=8192 + 5, budget_tokens=1024, sink=64,
                        window=256, refresh=4, steps=9),
    # MoBA-style: G = 8, blocks of 128, top-8, current block
    "moba_small": _cfg(W.moba(0), Hkv=2, Hq=16, L=128 * 40 + 77, block_size=128, topk=8,
                       n_needles=6, steps=3),
    # large-batch shape, pages of 32, selection every step
    "largebatch_small": _cfg(W.largebatch(0), B=6, Hkv=2, Hq=8, L=4096 + 31, budget_tokens=1024,
                             sink=256, window=512, steps=3),
    # head_dim 64 on the tensor-core path
    "quest_d64": _cfg(W.quest(0), B=1, Hkv=2, Hq=8, D=64, L=4096 + 9, budget_tokens=512, sink=32,
                      window=128, refresh=2, steps=4),
    # fp32 cache with D 128 on the CUDA-core path
    "moba_f32": _cfg(W.moba(0), Hkv=1, Hq=4, kv_dtype=torch.float32, L=64 * 50 + 3,
                     block_size=64, topk=5, n_needles=3, steps=2),
    # MSA-shaped: blocks of 128, top-16, current block, clustered keys
    "msa_small": _cfg(W.msa(0), B=2, Hkv=2, Hq=8, L=128 * 40 + 50, steps=3),
    # 600 blocks per segment: the one-warp pick with keys in every register slot
    "msa_600_blocks": _cfg(W.msa(0), B=1, Hkv=2, Hq=8, L=128 * 600 + 17, steps=2),
    # more than 1,024 blocks per segment (the CTA-wide radix pick)
    "msa_many_blocks": _cfg(W.msa(0), B=1, Hkv=2, Hq=8, L=128 * 1100 + 17, steps=2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_decode_matches_oracle(name):
    chk = FixedDecodeCheck(CASES[name])
    worst = chk.run(CASES[name].steps)
    assert worst <= 2e-3


# Steps between refreshes run append + decode as one launch (bsa_decode_step).
# These cases make a fixed block complete during such a step, so the summary
# built inside the decode grid is compared at the next refresh.
FUSED = {
    # pages of 16 (min/max): row 16k+15 is appended at step 2, refresh at 8
    "quest_page_completes": _cfg(W.quest(0), B=2, Hkv=2, Hq=8, L=16 * 300 + 13, budget_tokens=512,
                                 sink=32, window=128, refresh=8, steps=10),
    # blocks of 128 (centroid, current block): row 128k+127 appended at step 1
    "moba_block_completes": _cfg(W.moba(0), Hkv=2, Hq=16, L=128 * 30 + 126, block_size=128,
                                 topk=6, n_needles=4, refresh=4, steps=6),
    # D 64, G 4
    "quest_d64_fused": _cfg(W.quest(0), B=3, Hkv=1, Hq=4, D=64, L=2048 + 14, budget_tokens=256,
                            sink=16, window=64, refresh=5, steps=7),
}


@pytest.mark.parametrize("name", list(FUSED))
def test_fused_step_matches_oracle(name):
    chk = FixedDecodeCheck(FUSED[name])
    assert chk.sess.fuses()
    chk.run(FUSED[name].steps)


def test_unfused_steps_match_oracle():
    """The same step sequence with separate append and decode launches."""
    chk = FixedDecodeCheck(CASES["quest_small"], fused=False)
    chk.run(CASES["quest_small"].steps)


EDGE = {
    # budget 0: sink + window only
    "budget_zero": _cfg(W.quest(0), B=1, Hkv=2, Hq=8, L=3000, budget_tokens=0, sink=16, window=100,
                        refresh=1, steps=2),
    # k larger than the number of candidates: every block (dense attention)
    "k_all": _cfg(W.moba(0), Hkv=2, Hq=8, L=128 * 9 + 5, block_size=128, topk=1000, n_needles=2,
                  steps=2),
    # sink longer than the cache, window covering everything
    "sink_covers": _cfg(W.quest(0), B=1, Hkv=1, Hq=4, L=200, budget_tokens=64, sink=4096,
                        window=64, refresh=1, steps=2),
    # cache shorter than one block: no candidates at all
    "short_cache": _cfg(W.moba(0), Hkv=1, Hq=4, L=40, block_size=64, topk=4, n_needles=0,
                        steps=2),
    # G = 1 (multi-head), pages of 16
    "g1": _cfg(W.quest(0), B=2, Hkv=4, Hq=4, L=2048 + 3, budget_tokens=256, sink=16, window=64,
               refresh=1, steps=2),
    # G = 2: one row per thread in the scoring kernel
    "g2": _cfg(W.quest(0), B=2, Hkv=4, Hq=8, L=2048 + 3, budget_tokens=256, sink=16, window=64,
               refresh=1, steps=2),
    # fp32 cache with min/max page bounds (fp32 pairs, the per-row scoring kernel)
    "minmax_f32": _cfg(W.quest(0), B=2, Hkv=2, Hq=8, kv_dtype=torch.float32, L=2048 + 5,
                       budget_tokens=256, sink=16, window=64, refresh=2, steps=3),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_decode_edge_cases(name):
    chk = FixedDecodeCheck(EDGE[name])
    chk.run(EDGE[name].steps)


def test_needles_recalled_on_gpu():
    """MoBA-style gating with mean-pooled keys selects the planted needle
    blocks (16 needle blocks, top-16) -- the oracle pins the same property."""
    cfg = _cfg(W.moba(0), Hkv=2, Hq=16, L=512 * 40 + 1, block_size=512, topk=16, n_needles=16,
               steps=1)
    chk = FixedDecodeCheck(cfg)
    chk.run(1)
    sel = chk.sess.sel_blocks.cpu().numpy()
    for g in range(cfg.Hkv):
        want = sorted(chk.wl.needle_blocks[0, g].tolist())
        assert sel[g, :16].tolist() == want


def test_values_one_gives_one():
    """V = 1 everywhere: the GPU's softmax weights sum to one."""
    cfg = _cfg(W.quest(0), B=1, Hkv=2, Hq=8, L=4096 + 7, budget_tokens=512, sink=64, window=128,
               refresh=1, steps=1)
    chk = FixedDecodeCheck(cfg)
    chk.wl.V.fill_(1.0)
    chk.sess.build_summaries()
    q = chk.wl.decode_query(0)
    chk.sess.select(q)
    chk.sess.decode(q)
    torch.cuda.synchronize()
    out = chk.sess.out.cpu().numpy()
    assert np.abs(out - 1.0).max() <= 1e-5


def test_workspace_left_clean():
    """Every call leaves its counters at zero (the workspace can be reused)."""
    chk = FixedDecodeCheck(CASES["quest_small"])
    chk.run(3)
    ws = chk.sess.ws.cpu().numpy().view(np.uint32)
    nseg = chk.cfg.B * chk.cfg.Hkv
    assert ws[0] == 0                          # no device-side timeout
    assert np.all(ws[1:1 + 2 * nseg] == 0)     # select and decode counters


def test_decode_kernel_count():
    """Many segments merge inside clusters (one kernel); a single sequence of 8
    KV heads cannot fill the GPU with clusters and takes the merge kernel."""
    def desc(B):
        L = 65536
        return N.KvDesc(B=B, Hq=32, Hkv=8, D=128, kv_dtype=N.BSA_BF16, L_max=L, stride_b=8 * L * 128,
                        stride_h=L * 128, stride_t=128)
    p = N.sel_params(16, topk=-1, budget_tokens=4096, sink=256, window=1024)
    assert N.bsa_decode_kernels(desc(4), p, 5400) == 1
    assert N.bsa_decode_kernels(desc(1), p, 5400) == 2


def test_selection_g16_matches_oracle():
    """G = 16 (the decode stops at 8 query heads per KV head; selection goes to
    16): the paired-row scorer with eight heads per thread, selections and
    ranges bit for bit."""
    import oracle
    from gpu_harness import host, record_ties, current_label
    cfg = _cfg(W.moba(0), Hkv=2, Hq=32, L=128 * 30 + 11, block_size=128, topk=6, n_needles=4,
               steps=1)
    wl = W.Workload(cfg, "cuda")
    from block_sparse_long_build_b200.session import DecodeSession
    sess = DecodeSession(wl)
    sess.build_summaries()
    q = wl.decode_query(0)
    sess.select(q)
    torch.cuda.synchronize()
    qh, K = host(q), host(wl.K)
    n = cfg.L
    sel, cnt = host(sess.sel_blocks), host(sess.sel_count)
    ranges, nr = host(sess.ranges), host(sess.n_ranges)
    for g in range(cfg.Hkv):
        beg, end = oracle.fixed_block_bounds(n, cfg.block_size)
        summ = oracle.block_summaries(K[0, g], beg, end, cfg.kind)
        s32, s64 = oracle.block_scores(qh[0, g * cfg.G:(g + 1) * cfg.G], summ, cfg.kind)
        want, want_r, ties = oracle.select_fixed(s32, s64, n, cfg.block_size, cfg.topk,
                                                 cfg.budget_tokens, cfg.sink, cfg.window,
                                                 cfg.keep_current)
        record_ties(current_label(), ties)
        assert sel[g, :cnt[g]].tolist() == want
        assert [tuple(x) for x in ranges[g, :nr[g]].tolist()] == want_r
