"""Shared driver for the GPU parity tests: runs a decode workload through the
C ABI and through the CPU oracle on the same seeded inputs and compares.

Bars (from the method's statement): selected block ids and token ranges
bit-exact; outputs and log-sum-exp within max-abs 2e-3 of the fp64 oracle.
After every library call sequence the workspace's device-side status word
must read clean (no wait gave up, no capacity cut).

Near-ties (pairs across a selection cut whose fp64 scores lie within 1e-6
relative) are counted per test in NEAR_TIES and printed in pytest's terminal
summary, passing or not.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200.session import DecodeSession
from block_sparse_long_build_b200.workloads import Workload

ATOL = 2e-3

# test label -> [selections compared, selections with a near-tie, near-tie pairs]
NEAR_TIES: dict[str, list[int]] = {}
# largest |GPU - oracle| over outputs and log-sum-exp, per test
MAX_ERR: dict[str, float] = {}


def record_err(label: str, *errs) -> None:
    MAX_ERR[label] = max([MAX_ERR.get(label, 0.0)] + [float(e) for e in errs])


def record_ties(label: str, ties) -> None:
    e = NEAR_TIES.setdefault(label, [0, 0, 0])
    e[0] += 1
    e[1] += 1 if ties else 0
    e[2] += len(ties)


def current_label() -> str:
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def host(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> numpy: bf16 as uint16 bit patterns, FP8 as uint8
    codes, fp32 as float32."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def oracle_kv(a: np.ndarray) -> np.ndarray:
    """A host cache array in a type the oracle reads: FP8 codes decoded by the
    oracle's own fp8_e4m3_to_f32 (exact values as float32), others as is."""
    return oracle.fp8_e4m3_to_f32(a) if a.dtype == np.uint8 else a


def assert_status_clean(ws: torch.Tensor | None, what: str = "") -> None:
    st, bits = N.bsa_workspace_status(ws)
    assert st == N.BSA_OK, f"device status {bits:#x} ({N.status_string(st)}) {what}"


def gpu_summaries(raw: np.ndarray, sess: DecodeSession, s: int, nb: int):
    """Segment s's first nb summaries from the raw summaries buffer."""
    c = sess.cfg
    if sess.kind == N.BSA_SUM_MINMAX:
        esz = 4 if c.kv_dtype == torch.float32 else 2   # bf16 bounds for bf16 and FP8 caches
        row = 2 * c.D * esz
        seg = raw[s * sess.nb * row:(s * sess.nb + nb) * row]
        # (min, max) pairs per dimension
        if esz == 2:
            x = oracle.bf16_bits_to_f32(seg.view(np.uint16)).reshape(nb, c.D, 2)
        else:
            x = seg.view(np.float32).reshape(nb, c.D, 2)
        return x[:, :, 0], x[:, :, 1]
    row = c.D * 4
    return raw[s * sess.nb * row:(s * sess.nb + nb) * row].view(np.float32).reshape(nb, c.D)


class FixedDecodeCheck:
    """Runs fixed-block decode steps on both sides and compares.

    segments: the (b, g) pairs compared (default: all); only their caches are
    copied to the host.  run(check_steps=...) compares only those steps (the
    GPU runs every step in between, as a real decode would).  page_rows > 0
    runs the library on a page pool (seeded random page table); the oracle
    then reads each sequence's cache back through that table with its own
    paged_to_contiguous."""

    def __init__(self, cfg, device="cuda", fused=True, segments=None, page_rows=0,
                 spare_pages=0):
        self.cfg = cfg
        self.wl = Workload(cfg, device)
        self.sess = DecodeSession(self.wl, fused=fused, page_rows=page_rows,
                                  spare_pages=spare_pages)
        self.L_max = self.sess.desc.L_max
        self.segs = segments if segments is not None else [
            (b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
        # the oracle's own copy of each compared segment's cache
        if page_rows:
            Kp, Vp = oracle_kv(host(self.sess.K)), oracle_kv(host(self.sess.V))
            table = self.sess.page_table.cpu().numpy()
            self.K, self.V = {}, {}
            for b in sorted({b for b, _ in self.segs}):
                kb = oracle.paged_to_contiguous(Kp, table[b], page_rows, self.L_max)
                vb = oracle.paged_to_contiguous(Vp, table[b], page_rows, self.L_max)
                for bb, g in self.segs:
                    if bb == b:
                        self.K[(b, g)], self.V[(b, g)] = kb[g].copy(), vb[g].copy()
        else:
            self.K = {(b, g): oracle_kv(host(self.wl.K[b, g])) for b, g in self.segs}
            self.V = {(b, g): oracle_kv(host(self.wl.V[b, g])) for b, g in self.segs}
        self.n = [int(x) for x in self.wl.cur_len.cpu()]
        self.n_sel = list(self.n)
        self.q_sel = None       # queries of the last refresh step
        self.label = current_label()
        self.compared = 0

    def run(self, steps: int, check_summaries=True, check_steps=None):
        c, sess = self.cfg, self.sess
        sess.build_summaries()
        torch.cuda.synchronize()
        worst = 0.0
        for t in range(steps):
            q = self.wl.decode_query(t)
            if t > 0 or c.name != "tiny":
                k, v = self.wl.decode_new_kv(t)
                kh, vh = oracle_kv(host(k)), oracle_kv(host(v))
                for b in range(c.B):
                    if self.n[b] < self.L_max:
                        for bb, g in self.segs:
                            if bb == b:
                                self.K[(b, g)][self.n[b]] = kh[b, g]
                                self.V[(b, g)][self.n[b]] = vh[b, g]
                        self.n[b] += 1
            else:
                k = v = None
            sess.step(t, q, k, v)
            torch.cuda.synchronize()
            assert_status_clean(sess.ws, f"after step {t}")
            refresh = t % c.refresh == 0
            if refresh:
                self.n_sel = list(self.n)
                self.q_sel = host(q)
            if check_steps is None or t in check_steps:
                worst = max(worst, self.compare(q, refresh, check_summaries and refresh))
        return worst

    def compare(self, q, check_sel: bool, check_summaries: bool) -> float:
        c, sess = self.cfg, self.sess
        qh = host(q)
        out, lse = host(sess.out), host(sess.lse)
        assert np.all(host(self.wl.cur_len) == np.array(self.n))
        sel_blocks, sel_count = host(sess.sel_blocks), host(sess.sel_count)
        ranges, n_ranges = host(sess.ranges), host(sess.n_ranges)
        raw = sess.summaries.cpu().numpy() if check_summaries else None
        worst = 0.0
        for b, g in self.segs:
            s = b * c.Hkv + g
            K, V = self.K[(b, g)], self.V[(b, g)]
            qg = qh[b, g * c.G:(g + 1) * c.G]
            qs = self.q_sel[b, g * c.G:(g + 1) * c.G] if self.q_sel is not None else qg
            ref = oracle.decode_fixed_segment(
                qg, K, V, self.n_sel[b], self.n[b], c.kind, c.block_size, c.topk,
                c.budget_tokens, c.sink, c.window, c.keep_current, 1.0 / math.sqrt(c.D), q_sel=qs)
            if check_summaries:
                nb = self.n_sel[b] // c.block_size
                beg, end = oracle.fixed_block_bounds(self.n_sel[b], c.block_size)
                want = oracle.block_summaries(K, beg, end, c.kind)
                got = gpu_summaries(raw, sess, s, nb)
                if c.kind == N.BSA_SUM_MINMAX:
                    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1]), \
                        f"minmax summaries differ (segment {s})"
                else:
                    assert np.array_equal(got, want), f"centroid summaries differ (segment {s})"
            if check_sel:
                record_ties(self.label, ref["ties"])
                gs = sel_blocks[s, :sel_count[s]].tolist()
                assert gs == ref["sel"], (
                    f"segment {s}: selection differs; near-ties {ref['ties']}")
                gr = [tuple(x) for x in ranges[s, :n_ranges[s]].tolist()]
                want_r = oracle.merge_ranges(
                    oracle.forced_ranges(self.n_sel[b], c.sink, c.window, c.block_size,
                                         c.keep_current)
                    + [(j * c.block_size, (j + 1) * c.block_size) for j in ref["sel"]])
                assert gr == want_r, f"segment {s}: ranges differ"
            err = np.abs(out[b, g * c.G:(g + 1) * c.G] - ref["out"]).max()
            lerr = np.abs(lse[b, g * c.G:(g + 1) * c.G] - ref["lse"]).max()
            worst = max(worst, float(err), float(lerr))
            record_err(current_label(), err, lerr)
            assert err <= ATOL, f"segment {s}: max |out - oracle| = {err:.3e}"
            assert lerr <= ATOL, f"segment {s}: max |lse - oracle| = {lerr:.3e}"
            self.compared += 1
        return worst
