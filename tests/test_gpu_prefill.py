"""GPU parity for the block-grouped prefill (semantic blocks, tcgen05 path).

Sampled query rows of each chunk are recomputed by the oracle in original
positions: dense causal attention while the prefix is short, otherwise the
chunk causally plus the visible positions of the blocks the query selects
(budget = prefix / 16).  The per-row block selections are compared bit for
bit with the selection bitmap the library leaves in its workspace.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

from gpu_harness import ATOL, current_label, host, record_err, record_ties

pytestmark = pytest.mark.gpu


def _setup(L=16384, n_blocks=32, Tq=1024, dense_below=4096, Hkv=2, Hq=8):
    cfg = W.semantic(0).scaled(L=L, n_blocks=n_blocks, chunk=Tq, steps=1, Hkv=Hkv, Hq=Hq,
                               budget_tokens=L // 16, dense_below=dense_below)
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    torch.cuda.synchronize()
    return cfg, wl, sess


def _check_chunk(cfg, wl, sess, p, Tq, rows):
    Q = wl.prefill_queries(p, Tq)
    out = torch.full((Tq, cfg.Hq, cfg.D), float("nan"), device="cuda")
    lse = torch.full((Tq, cfg.Hq), float("nan"), device="cuda")
    ws = sess.prefill_chunk(Q, p, out, lse)
    torch.cuda.synchronize()
    Qh = host(Q)
    Kpos, Vpos = host(wl.Kpos), host(wl.Vpos)
    labels = wl.labels.cpu().numpy()
    out_h, lse_h = out.cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(out_h).all() and np.isfinite(lse_h).all()
    ws_u32 = ws.cpu().numpy().view(np.uint32)
    assert ws_u32[0] == 0, f"device status bits {ws_u32[0]:#x} (timeout or selection overflow)"
    cb = 256 // 4   # status + counters area of the workspace, in words (B*Hkv <= 63)
    bitmap = ws_u32[cb:cb + Tq * cfg.Hkv * 8].reshape(Tq, cfg.Hkv, 8)
    sparse = p >= cfg.dense_below
    worst = 0.0
    for i in rows:
        P = p + i
        for g in range(cfg.Hkv):
            qg = oracle.bf16_bits_to_f32(Qh[i, g * cfg.G:(g + 1) * cfg.G])
            if sparse:
                sel, pos, ties, _ = oracle.semantic_select_positions(
                    qg, Kpos[0, g, :cfg.L], labels[0, g], cfg.n_blocks, p, p // 16)
                got = [j for j in range(cfg.n_blocks) if (bitmap[i, g, j // 32] >> (j % 32)) & 1]
                record_ties(current_label(), ties)
                assert got == sel, f"chunk {p} row {i} head {g}: selection differs; ties {ties}"
                rws = np.concatenate([pos, np.arange(p, P + 1)])
            else:
                assert not bitmap[i, g].any()
                rws = np.arange(0, P + 1)
            ref, ref_lse = oracle.attend(qg, Kpos[0, g], Vpos[0, g], rws, 1 / math.sqrt(cfg.D))
            err = np.abs(out_h[i, g * cfg.G:(g + 1) * cfg.G] - ref).max()
            lerr = np.abs(lse_h[i, g * cfg.G:(g + 1) * cfg.G] - ref_lse).max()
            worst = max(worst, float(err), float(lerr))
            record_err(current_label(), err, lerr)
            assert err <= ATOL, f"chunk {p} row {i} head {g}: max |out - oracle| = {err:.3e}"
            assert lerr <= ATOL, f"chunk {p} row {i} head {g}: max |lse - oracle| = {lerr:.3e}"
    return worst


@pytest.fixture(scope="module")
def small():
    return _setup()


@pytest.mark.parametrize("p", [0, 2048, 8192, 15360], ids=["dense0", "dense2k", "sparse8k", "sparse_last"])
def test_prefill_chunk_matches_oracle(small, p):
    cfg, wl, sess = small
    rng = np.random.default_rng(p + 1)
    Tq = 1024
    rows = sorted(set([0, 1, 31, 32, 127, 128, Tq - 1] + rng.integers(0, Tq, 17).tolist()))
    _check_chunk(cfg, wl, sess, p, Tq, rows)


def test_prefill_ragged_chunk():
    """A chunk whose length is not a multiple of the 32-query tile, G = 8."""
    cfg, wl, sess = _setup(L=12288 + 5, n_blocks=24, Tq=700, dense_below=2048, Hkv=1, Hq=8)
    p = 9000
    _check_chunk(cfg, wl, sess, p, 700, [0, 5, 99, 350, 511, 699])


def test_prefill_single_query_chunk():
    """A chunk of one query at a sparse position: each KV head's local item
    holds G rows, the rest of the item and every grouped item's other rows
    are empty."""
    cfg, wl, sess = _setup(L=16384, n_blocks=32, Tq=1, dense_below=4096)
    _check_chunk(cfg, wl, sess, 12345, 1, [0])


def test_prefill_budget_admits_no_block():
    """Two blocks of ~8k positions and the first sparse chunk at 2,048: the
    budget (128 tokens) is smaller than any block's visible prefix, so every
    query attends only its own chunk and no grouped item exists."""
    cfg, wl, sess = _setup(L=16384, n_blocks=2, Tq=512, dense_below=2048)
    _check_chunk(cfg, wl, sess, 2048, 512, [0, 1, 127, 128, 255, 511])


def test_prefill_first_sparse_chunk():
    """The chunk that starts exactly at the dense limit: the first one whose
    queries select blocks."""
    cfg, wl, sess = _setup(L=16384, n_blocks=32, Tq=1024, dense_below=4096)
    _check_chunk(cfg, wl, sess, 4096, 1024, [0, 1, 63, 64, 511, 1023])
