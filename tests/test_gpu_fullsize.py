"""GPU parity at the workloads' own sizes, and on the launch paths the
benchmark takes.

* Quest-style decode at full size (batch 4, 8 KV heads, 65,536 tokens, pages
  of 16, budget 4096, refresh every 32 steps): every segment at steps 0, 1,
  31 and 32 -- two refreshes and the fused append + decode steps between them,
  which run with the split-K merge inside thread-block clusters.
* Large-batch decode at full size (batch 64, 32,768 tokens, pages of 32,
  budget 8192, selection every step): sampled segments at chosen steps.
* MoBA-style decode at full size (131,072 tokens, blocks of 512, top-16, the
  current block): every segment at chosen steps.
* Semantic-block decode at full size (524,288 tokens, 256 variable blocks,
  budget L/16): every KV head at chosen steps.
* Block-grouped prefill at full size (the last and a middle 4,096-query chunk
  of the 524,288-token context, and a 65,536-token context with 256 blocks):
  one query row from every 32-query tile, where each query selects about 16
  blocks (so the merge runs over many partial slots).
* A small Quest-shaped case with enough segments for the clustered decode
  grid, where a page completes inside a fused (clustered) step.
* The FP8 cache at the large-batch size and the Quest configuration on a
  page pool (sampled segments / every segment at chosen steps).

Selections are compared bit for bit, outputs and log-sum-exp within max-abs
2e-3 of the fp64 oracle.  Sampling keeps the oracle's time to seconds per
case; the GPU runs every step in between.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

from gpu_harness import (ATOL, FixedDecodeCheck, assert_status_clean, current_label, host,
                         record_err, record_ties)

pytestmark = pytest.mark.gpu


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_clustered_fused_step_matches_oracle():
    """12 segments: the decode splits form thread-block clusters and the
    append runs inside the clustered grid; L = 16k + 13, so the page of rows
    16k..16k+15 completes at step 2, a fused step, and its summary is compared
    at the refresh of step 4."""
    cfg = W.quest(0).scaled(B=3, Hkv=4, Hq=16, L=16 * 1000 + 13, budget_tokens=1024, sink=64,
                            window=256, refresh=4, steps=9)
    chk = FixedDecodeCheck(cfg)
    assert chk.sess.fuses()
    assert chk.sess.decode_kernels == 1, "expected the clustered (one-kernel) decode"
    chk.run(cfg.steps)
    _free()


def test_quest_full_size():
    cfg = W.quest(0)
    chk = FixedDecodeCheck(cfg)
    assert chk.sess.fuses() and chk.sess.decode_kernels == 1
    chk.run(33, check_steps={0, 1, 31, 32})
    assert chk.compared == 4 * cfg.B * cfg.Hkv
    del chk
    _free()


def test_largebatch_full_size():
    cfg = W.largebatch(0)
    rng = np.random.default_rng(5)
    bs = sorted(set([0, 1, cfg.B - 1] + rng.integers(0, cfg.B, 5).tolist()))
    segs = [(b, g) for b in bs for g in (0, cfg.Hkv - 1)] + [(bs[len(bs) // 2], 3)]
    chk = FixedDecodeCheck(cfg, segments=segs)
    chk.run(20, check_steps={0, 1, 19})
    assert chk.compared == 3 * len(segs)
    del chk
    _free()


def test_largebatch_fp8_full_size():
    """The FP8 (E4M3) cache at the large-batch size, sampled segments."""
    cfg = W.largebatch_fp8(0)
    segs = [(0, 0), (5, 3), (31, 7), (63, 1)]
    chk = FixedDecodeCheck(cfg, segments=segs)
    chk.run(6, check_steps={0, 5})
    assert chk.compared == 2 * len(segs)
    del chk
    _free()


def test_quest_paged_full_size():
    """The Quest-style configuration on a page pool (pages of 256 rows at
    random slots): every segment at a refresh and at the fused steps after it."""
    cfg = W.quest(0)
    chk = FixedDecodeCheck(cfg, page_rows=256, spare_pages=16)
    assert chk.sess.fuses() and chk.sess.decode_kernels == 1
    chk.run(3, check_steps={0, 2})
    assert chk.compared == 2 * cfg.B * cfg.Hkv
    del chk
    _free()


def test_moba_full_size():
    cfg = W.moba(0)
    chk = FixedDecodeCheck(cfg)
    chk.run(cfg.steps, check_steps={0, 1, cfg.steps - 1})
    # the planted needle blocks are among the selected ones at every step
    sel = chk.sess.sel_blocks.cpu().numpy()
    cnt = chk.sess.sel_count.cpu().numpy()
    for g in range(cfg.Hkv):
        assert set(chk.wl.needle_blocks[0, g].tolist()) <= set(sel[g, :cnt[g]].tolist())
    del chk
    _free()


# ------------------------------------------------------------- semantic


@pytest.fixture(scope="module")
def semantic_full():
    cfg = W.semantic(0)
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    torch.cuda.synchronize()
    Kpos, Vpos = host(wl.Kpos), host(wl.Vpos)
    labels = wl.labels.cpu().numpy()
    orders = [np.argsort(labels[0, g], kind="stable") for g in range(cfg.Hkv)]
    # the block centres, bit for bit, once; the oracle's copy serves every query
    summ = sess.summaries.cpu().numpy().view(np.float32).reshape(cfg.Hkv, sess.nb, cfg.D)
    cents = []
    for g in range(cfg.Hkv):
        _, _, _, C = oracle.semantic_select_positions(
            np.zeros((cfg.G, cfg.D), np.float32), Kpos[0, g, :cfg.L], labels[0, g], cfg.n_blocks,
            1, 1, order=orders[g])
        assert np.array_equal(summ[g], C), f"KV head {g}: block centres differ"
        cents.append(C)
    yield cfg, wl, sess, Kpos, Vpos, labels, orders, cents
    del wl, sess
    _free()


def test_semantic_decode_full_size(semantic_full):
    cfg, wl, sess, Kpos, Vpos, labels, orders, cents = semantic_full
    L, loc = cfg.L, cfg.chunk
    Kp, Vp = Kpos.copy(), Vpos.copy()
    label = current_label()
    for t in range(cfg.steps):
        q = wl.decode_query(t)
        k, v = wl.decode_new_kv(t)
        Kp[0, :, L + t] = host(k)[0]
        Vp[0, :, L + t] = host(v)[0]
        sess.step(t, q, k, v)
        torch.cuda.synchronize()
        assert_status_clean(sess.ws, f"after step {t}")
        if t not in (0, 1, cfg.steps - 1):
            continue
        qh = host(q)
        out, lse = sess.out.cpu().numpy(), sess.lse.cpu().numpy()
        sel, cnt = sess.sel_blocks.cpu().numpy(), sess.sel_count.cpu().numpy()
        for g in range(cfg.Hkv):
            qg = qh[0, g * cfg.G:(g + 1) * cfg.G]
            ref_sel, pos, ties, _ = oracle.semantic_select_positions(
                qg, Kp[0, g, :L], labels[0, g], cfg.n_blocks, L - loc, cfg.budget_tokens,
                centroids=cents[g], order=orders[g])
            record_ties(label, ties)
            assert sel[g, :cnt[g]].tolist() == ref_sel, f"step {t} head {g}: near-ties {ties}"
            rows = np.concatenate([pos, np.arange(L - loc, L + t + 1)])
            ref, ref_lse = oracle.attend(qg, Kp[0, g], Vp[0, g], rows, 1 / math.sqrt(cfg.D))
            err = np.abs(out[0, g * cfg.G:(g + 1) * cfg.G] - ref).max()
            lerr = np.abs(lse[0, g * cfg.G:(g + 1) * cfg.G] - ref_lse).max()
            record_err(current_label(), err, lerr)
            assert err <= ATOL, f"step {t} head {g}: max |out - oracle| = {err:.3e}"
            assert lerr <= ATOL, f"step {t} head {g}: max |lse - oracle| = {lerr:.3e}"
    # put the cache length back for the prefill tests sharing the fixture
    wl.cur_len.fill_(L + loc)


def _prefill_rows(cfg, rng, Tq, tile=32):
    """One query row from every 32-query tile of the chunk, plus its ends."""
    rows = [min(Tq - 1, t + int(rng.integers(0, tile))) for t in range(0, Tq, tile)]
    return sorted(set(rows + [0, Tq - 1]))


def _check_prefill(cfg, wl, sess, Kpos, Vpos, labels, orders, cents, p, Tq, heads_per_row=2,
                   seed=0):
    Q = wl.prefill_queries(p, Tq)
    out = torch.full((Tq, cfg.Hq, cfg.D), float("nan"), device="cuda")
    lse = torch.full((Tq, cfg.Hq), float("nan"), device="cuda")
    ws = sess.prefill_chunk(Q, p, out, lse)
    torch.cuda.synchronize()
    assert_status_clean(ws, f"prefill chunk at {p}")
    Qh = host(Q)
    out_h, lse_h = out.cpu().numpy(), lse.cpu().numpy()
    ws_u32 = ws.cpu().numpy().view(np.uint32)
    cb = 256 // 4   # status + counters area of the workspace, in words
    bitmap = ws_u32[cb:cb + Tq * cfg.Hkv * 8].reshape(Tq, cfg.Hkv, 8)
    sparse = p >= cfg.dense_below
    rng = np.random.default_rng(seed + p)
    label = current_label()
    most = 0
    for n_row, i in enumerate(_prefill_rows(cfg, rng, Tq)):
        P = p + i
        for hh in range(heads_per_row):
            g = (n_row + hh * (cfg.Hkv // heads_per_row)) % cfg.Hkv
            qg = oracle.bf16_bits_to_f32(Qh[i, g * cfg.G:(g + 1) * cfg.G])
            if sparse:
                sel, pos, ties, _ = oracle.semantic_select_positions(
                    qg, Kpos[0, g, :cfg.L], labels[0, g], cfg.n_blocks, p, p // 16,
                    centroids=cents[g], order=orders[g])
                got = [j for j in range(cfg.n_blocks) if (bitmap[i, g, j // 32] >> (j % 32)) & 1]
                record_ties(label, ties)
                assert got == sel, f"chunk {p} row {i} head {g}: selection differs; ties {ties}"
                most = max(most, len(sel))
                rws = np.concatenate([pos, np.arange(p, P + 1)])
            else:
                rws = np.arange(0, P + 1)
            ref, ref_lse = oracle.attend(qg, Kpos[0, g], Vpos[0, g], rws, 1 / math.sqrt(cfg.D))
            err = np.abs(out_h[i, g * cfg.G:(g + 1) * cfg.G] - ref).max()
            lerr = np.abs(lse_h[i, g * cfg.G:(g + 1) * cfg.G] - ref_lse).max()
            record_err(current_label(), err, lerr)
            assert err <= ATOL, f"chunk {p} row {i} head {g}: max |out - oracle| = {err:.3e}"
            assert lerr <= ATOL, f"chunk {p} row {i} head {g}: max |lse - oracle| = {lerr:.3e}"
    return most


@pytest.mark.parametrize("which", ["last", "middle"])
def test_semantic_prefill_full_size(semantic_full, which):
    cfg, wl, sess, Kpos, Vpos, labels, orders, cents = semantic_full
    Tq = cfg.chunk
    p = cfg.L - Tq if which == "last" else cfg.L // 2
    most = _check_prefill(cfg, wl, sess, Kpos, Vpos, labels, orders, cents, p, Tq)
    assert most >= 5, f"queries selected at most {most} blocks; the case should reach many slots"


def test_semantic_prefill_dense_chunk_full_size(semantic_full):
    """A chunk below the dense limit of the full configuration (16k): plain
    causal attention over the whole prefix."""
    cfg, wl, sess, Kpos, Vpos, labels, orders, cents = semantic_full
    _check_prefill(cfg, wl, sess, Kpos, Vpos, labels, orders, cents, 8192, cfg.chunk,
                   heads_per_row=1)


def test_prefill_64k_256_blocks():
    """65,536 tokens in 256 blocks (about 256 rows each), 4,096-query chunks:
    each query's budget (prefix / 16) admits about 16 blocks."""
    cfg = W.semantic(0).scaled(L=65536, n_blocks=256, budget_tokens=65536 // 16, steps=1)
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    torch.cuda.synchronize()
    Kpos, Vpos = host(wl.Kpos), host(wl.Vpos)
    labels = wl.labels.cpu().numpy()
    orders = [np.argsort(labels[0, g], kind="stable") for g in range(cfg.Hkv)]
    cents = [oracle.semantic_select_positions(
        np.zeros((cfg.G, cfg.D), np.float32), Kpos[0, g, :cfg.L], labels[0, g], cfg.n_blocks, 1, 1,
        order=orders[g])[3] for g in range(cfg.Hkv)]
    most = _check_prefill(cfg, wl, sess, Kpos, Vpos, labels, orders, cents, cfg.L - cfg.chunk,
                          cfg.chunk)
    assert most >= 5
    del wl, sess
    _free()
