"""GPU parity for an FP8 (E4M3) K/V cache ("Attention mechanisms in modern
LLMs", basic maths and the real cost: the cache may be kept in FP8).

The library reads one byte per element: page bounds are built as exact bf16
values, the tensor-core decode loads FP8 boxes by TMA and widens them to f16
in shared memory, the CUDA-core decode decodes codes one by one.  The oracle
reads the same codes through its own fp8_e4m3_to_f32 table (pinned against
torch's float8_e4m3fn on all 256 codes) and computes the plain decode, so
the bars are the same as for bf16: selections and summaries bit for bit,
outputs within 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W

from gpu_harness import FixedDecodeCheck

pytestmark = pytest.mark.gpu

F8 = torch.float8_e4m3fn


def _cfg(base, **kw):
    return base.scaled(kv_dtype=F8, **kw)


CASES = {
    # fused append + decode steps, a page completing inside one, window extension
    "quest_fp8_small": _cfg(W.quest(0), B=2, Hkv=2, Hq=8, L=16 * 500 + 13, budget_tokens=1024,
                            sink=64, window=256, refresh=4, steps=9),
    # twelve segments: clustered decode splits; selection every step
    "largebatch_fp8_clustered": _cfg(W.largebatch(0), B=6, Hkv=2, Hq=8, L=4096 + 31,
                                     budget_tokens=1024, sink=256, window=512, steps=3),
    # MoBA-style: G = 8, centroid summaries from FP8 keys, current block
    "moba_fp8": _cfg(W.moba(0), Hkv=2, Hq=16, L=128 * 40 + 77, block_size=128, topk=8,
                     n_needles=6, steps=3),
    # head_dim 64: the CUDA-core decode decodes the codes itself
    "quest_fp8_d64": _cfg(W.quest(0), B=1, Hkv=2, Hq=8, D=64, L=4096 + 9, budget_tokens=512,
                          sink=32, window=128, refresh=2, steps=4),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_decode_matches_oracle(name):
    chk = FixedDecodeCheck(CASES[name])
    if CASES[name].D == 128:
        assert chk.sess.fuses()
    chk.run(CASES[name].steps)


def test_fp8_paged_decode_matches_oracle():
    cfg = CASES["quest_fp8_small"]
    chk = FixedDecodeCheck(cfg, page_rows=64, spare_pages=3)
    chk.run(cfg.steps)


@pytest.mark.parametrize("D", [128, 64])
def test_fp8_every_code_decodes_exactly(D):
    """Attention over a single row returns that row of V: with V holding
    every finite E4M3 code, the output equals the oracle's decoding of each
    code (the softmax weight is exactly 1)."""
    codes = np.array([c for c in range(256) if c & 0x7f != 0x7f], np.uint8)   # 254 finite codes
    rows = -(-len(codes) // D)
    L = 64
    K = torch.zeros(1, 1, L, D, dtype=F8, device="cuda")
    V = torch.zeros(1, 1, L, D, dtype=F8, device="cuda")
    vbytes = np.zeros((rows, D), np.uint8)
    vbytes.ravel()[:len(codes)] = codes
    V.view(torch.uint8)[0, 0, :rows] = torch.from_numpy(vbytes).cuda()
    K.view(torch.uint8)[0, 0, :rows] = torch.from_numpy(vbytes).cuda()
    desc = N.kv_desc(K, 4)
    q = torch.randn(1, 4, D, device="cuda")
    out = torch.empty(1, 4, D, device="cuda")
    lse = torch.empty(1, 4, device="cuda")
    cur = torch.full((1,), L, dtype=torch.int32, device="cuda")
    ranges = torch.zeros(1, 4, 2, dtype=torch.int32, device="cuda")
    n_ranges = torch.ones(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(N.bsa_workspace_size(desc, None, N.BSA_OP_DECODE, 0, 16), dtype=torch.uint8,
                     device="cuda")
    for j in range(rows):
        ranges[0, 0] = torch.tensor([j, j + 1], dtype=torch.int32)
        # cur_len = j + 1: the last range is not extended past row j
        cur.fill_(j + 1)
        N.bsa_decode(desc, q, K, V, ranges, n_ranges, 4, cur, 16, 1 / math.sqrt(D), out, lse, ws)
        torch.cuda.synchronize()
        want = oracle.fp8_e4m3_to_f32(vbytes[j])
        got = out[0].cpu().numpy()
        assert np.array_equal(got, np.broadcast_to(want, got.shape)), f"row {j}"
        # lse of one token is its scaled logit: q . k / sqrt(D) with k the row's values
        k = oracle.fp8_e4m3_to_f32(vbytes[j]).astype(np.float64)
        ref = q[0].cpu().numpy().astype(np.float64) @ k / math.sqrt(D)
        assert np.abs(lse[0].cpu().numpy() - ref).max() <= 2e-3 * max(1.0, np.abs(ref).max())
