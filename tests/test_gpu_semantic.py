"""GPU parity for semantic (variable-size) blocks, decode.

The GPU reads a block-ordered store (rows sorted by block, then position,
followed by a position-ordered local part); the oracle works in original
positions from the planted block labels.  Agreement is therefore also a
permutation test of the store layout.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import workloads as W
from block_sparse_long_build_b200.session import DecodeSession

from gpu_harness import ATOL, assert_status_clean, current_label, host, record_err, record_ties

pytestmark = pytest.mark.gpu


def _cfg(L=16384, n_blocks=32, chunk=1024, steps=3, Hkv=2, Hq=8):
    return W.semantic(0).scaled(L=L, n_blocks=n_blocks, chunk=chunk, steps=steps, Hkv=Hkv, Hq=Hq,
                                budget_tokens=L // 16)


@pytest.mark.parametrize("cfg", [_cfg(), _cfg(L=12000 + 7, n_blocks=20, chunk=512, Hkv=1, Hq=4)],
                         ids=["L16k_32blocks", "ragged_20blocks"])
def test_semantic_decode_matches_oracle(cfg):
    wl = W.Workload(cfg, "cuda")
    sess = DecodeSession(wl)
    sess.build_summaries()
    torch.cuda.synchronize()
    Kpos, Vpos = host(wl.Kpos), host(wl.Vpos)
    labels = wl.labels.cpu().numpy()
    L, loc = cfg.L, cfg.chunk
    # summaries: normalised centres, bit-exact
    summ = sess.summaries.cpu().numpy().view(np.float32).reshape(cfg.B * cfg.Hkv, sess.nb, cfg.D)
    for g in range(cfg.Hkv):
        _, _, _, C = oracle.semantic_select_positions(
            np.zeros((cfg.G, cfg.D), np.float32), Kpos[0, g, :L], labels[0, g], cfg.n_blocks, 1, 1)
        assert np.array_equal(summ[g], C), f"KV head {g}: block centres differ"
    for t in range(cfg.steps):
        q = wl.decode_query(t)
        k, v = wl.decode_new_kv(t)
        Kpos[0, :, L + t] = host(k)[0]
        Vpos[0, :, L + t] = host(v)[0]
        sess.step(t, q, k, v)
        torch.cuda.synchronize()
        assert_status_clean(sess.ws, f"after step {t}")
        qh = host(q)
        out = sess.out.cpu().numpy()
        sel = sess.sel_blocks.cpu().numpy()
        cnt = sess.sel_count.cpu().numpy()
        for g in range(cfg.Hkv):
            qg = qh[0, g * cfg.G:(g + 1) * cfg.G]
            ref_sel, pos, ties, _ = oracle.semantic_select_positions(
                qg, Kpos[0, g, :L], labels[0, g], cfg.n_blocks, L - loc, cfg.budget_tokens)
            record_ties(current_label(), ties)
            assert sel[g, :cnt[g]].tolist() == ref_sel, f"step {t} head {g}: near-ties {ties}"
            rows = np.concatenate([pos, np.arange(L - loc, L + t + 1)])
            ref, _ = oracle.attend(qg, Kpos[0, g], Vpos[0, g], rows, 1 / math.sqrt(cfg.D))
            err = np.abs(out[0, g * cfg.G:(g + 1) * cfg.G] - ref).max()
            record_err(current_label(), err)
            assert err <= ATOL, f"step {t} head {g}: max |out - oracle| = {err:.3e}"
