"""GPU parity for the semantic index (spherical k-means and the block-ordered
store, "Semantic blocks for sparse attention").

Small cases are compared with the oracle bit for bit: labels, CSR offsets,
the order of the block-ordered store and the centres (the arithmetic is the
same fixed fp32 order on both sides).  The full-size case (524,288 keys per
KV head, 8 KV heads, 256 clusters, 20 rounds) is checked by properties that
hold at any size: the planted clusters are recovered exactly, the store is a
stable sort by cluster, and sampled keys are assigned as the oracle assigns
them against the centres the GPU returns.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_build_b200 import native as N
from block_sparse_long_build_b200 import workloads as W

from gpu_harness import host

pytestmark = pytest.mark.gpu


def _keys(rng, B, H, L, D, k_planted, noise, dtype):
    cent = rng.standard_normal((B, H, k_planted, D))
    cent /= np.linalg.norm(cent, axis=-1, keepdims=True)
    lab = rng.integers(0, k_planted, (B, H, L))
    X = np.take_along_axis(cent, lab[..., None].repeat(D, -1), axis=2) + noise * rng.standard_normal((B, H, L, D))
    return torch.tensor(X, dtype=torch.float32).to(dtype).cuda()


def _run_index(K, L, k, iters, init):
    d = N.kv_desc(K, K.shape[1])
    nseg = K.shape[0] * K.shape[1]
    ws = torch.zeros(N.bsa_index_workspace_size(d, L, k), dtype=torch.uint8, device="cuda")
    C = torch.zeros(nseg, k, K.shape[3], device="cuda")
    labels = torch.full((nseg, L), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((nseg, k + 1), -1, dtype=torch.int32, device="cuda")
    order = torch.full((nseg, L), -1, dtype=torch.int32, device="cuda")
    N.bsa_build_semantic_index(d, K, L, k, iters, init, C, labels, offsets, order, ws)
    torch.cuda.synchronize()
    return C.cpu().numpy(), labels.cpu().numpy(), offsets.cpu().numpy(), order.cpu().numpy()


@pytest.mark.parametrize("dtype,D,L,k,iters,noise", [
    (torch.bfloat16, 128, 5000 + 37, 22, 5, 0.35),   # ragged chunk, k not a multiple of 4
    (torch.float32, 64, 3000, 16, 4, 0.5),
    (torch.bfloat16, 128, 1024, 1, 2, 0.3),          # one cluster
    (torch.bfloat16, 128, 4096 + 3, 300, 3, 0.4),    # more than 256 clusters (untiled assignment)
])
def test_index_matches_oracle_bit_for_bit(dtype, D, L, k, iters, noise):
    rng = np.random.default_rng(L + k)
    B, H = 1, 2
    K = _keys(rng, B, H, L, D, max(k // 2, 1), noise, dtype)
    init = torch.tensor(np.stack([rng.choice(L, k, replace=False) for _ in range(B * H)]),
                        dtype=torch.int32, device="cuda")
    C, labels, offsets, order = _run_index(K, L, k, iters, init)
    Kh = host(K)
    for s in range(B * H):
        Co, lo, oo, ordo = oracle.spherical_kmeans(Kh[s // H, s % H], k, iters, init[s].cpu().numpy())
        assert (labels[s] == lo).all(), f"segment {s}: {(labels[s] != lo).sum()} labels differ"
        assert (offsets[s] == oo).all()
        assert (order[s] == ordo).all()
        assert (C[s] == Co).all(), f"segment {s}: max |centre diff| {np.abs(C[s] - Co).max():.3e}"


def test_index_empty_cluster_keeps_its_start():
    """Two starting keys with equal values: every tie goes to the lower
    centre, the other stays empty after the first round and keeps its start."""
    rng = np.random.default_rng(3)
    L, D, k = 2048, 128, 6
    K = _keys(rng, 1, 1, L, D, 3, 0.4, torch.bfloat16)
    K[0, 0, 5] = K[0, 0, 9]
    init = torch.tensor([[9, 5, 100, 200, 300, 400]], dtype=torch.int32, device="cuda")
    C, labels, offsets, order = _run_index(K, L, k, 2, init)
    Co, lo, oo, ordo = oracle.spherical_kmeans(host(K)[0, 0], k, 2, init[0].cpu().numpy())
    assert (labels[0] == lo).all() and (order[0] == ordo).all() and (C[0] == Co).all()
    _, l1, o1, _ = _run_index(K, L, k, 1, init)
    assert o1[0][2] - o1[0][1] == 0


def test_full_size_index_recovers_planted_blocks_and_gathers_the_store():
    """The semantic workload at full size: 524,288 keys per KV head in 256
    planted clusters (log-normal sizes), 20 rounds from one key of each
    cluster.  The result must be the planted grouping, stored exactly as the
    workload stores it."""
    cfg = W.semantic(0)
    wl = W.Workload(cfg, "cuda")
    B, H, L, k = cfg.B, cfg.Hkv, cfg.L, cfg.n_blocks
    lab = wl.labels.reshape(B * H, L)
    init = torch.stack([torch.stack([torch.nonzero(lab[s] == j)[0, 0] for j in range(k)])
                        for s in range(B * H)]).to(torch.int32)
    Kpos = wl.Kpos
    C, labels, offsets, order = _run_index(Kpos, L, k, 20, init)
    planted = lab.cpu().numpy()
    assert (labels == planted).all()
    assert (offsets == wl.block_offsets.reshape(B * H, k + 1).cpu().numpy()).all()
    assert (order == wl.kv_pos.reshape(B * H, -1)[:, :L].cpu().numpy()).all()
    assert np.allclose(np.linalg.norm(C.astype(np.float64), axis=-1), 1.0, atol=1e-5)
    # sampled keys are assigned as the oracle assigns them against these centres
    rng = np.random.default_rng(0)
    Kh = host(Kpos)
    for s in (0, B * H - 1):
        rows = rng.choice(L, 256, replace=False)
        ref = oracle.kmeans_assign(Kh[s // H, s % H, :L], rows, C[s])
        assert (labels[s][rows] == ref).all()
    # the block-ordered store from the order, through the gather
    src, dst = N.kv_desc(Kpos, cfg.Hq), N.kv_desc(wl.K, cfg.Hq)
    Kb, Vb = torch.zeros_like(wl.K), torch.zeros_like(wl.V)
    rows_dev = torch.tensor(order, dtype=torch.int32, device="cuda")
    N.bsa_gather_rows(src, Kpos, wl.Vpos, dst, Kb, Vb, rows_dev, L, 0)
    torch.cuda.synchronize()
    assert torch.equal(Kb[:, :, :L], wl.K[:, :, :L]) and torch.equal(Vb[:, :, :L], wl.V[:, :, :L])


def test_gather_skips_rows_outside_the_source():
    K = torch.randn(1, 2, 64, 128, device="cuda").to(torch.bfloat16)
    V = torch.randn_like(K)
    Ko, Vo = torch.zeros_like(K), torch.zeros_like(V)
    rows = torch.tensor([[3, -1, 70, 5], [0, 63, 1, 2]], dtype=torch.int32, device="cuda")
    d = N.kv_desc(K, 2)
    N.bsa_gather_rows(d, K, V, d, Ko, Vo, rows, 4, 10)
    torch.cuda.synchronize()
    assert torch.equal(Ko[0, 0, 10], K[0, 0, 3]) and torch.equal(Ko[0, 0, 13], K[0, 0, 5])
    assert not Ko[0, 0, 11].any() and not Ko[0, 0, 12].any()
    assert torch.equal(Vo[0, 1, 10:14], V[0, 1, torch.tensor([0, 63, 1, 2])])
